// K4 (tensor-core form over SM pairs, bf16, d = 128): dense attention of the chunk over
// its compacted cache (QUOKA page, Figure 1(a): the sub-selected KV cache goes into a
// dense attention kernel; QUILT page: the K/V entries a group of queries selected in
// common are loaded once and reused by all of them).
//
// A cluster of two CTAs on two SMs serves one (sequence, KV head, 2 x TP chunk
// positions); CTA r owns query tile r: 128 rows packing the G query heads of the KV head
// at TP = 128 / G positions, gathered once by TMA (tile::gather4).  The pair runs every
// MMA as one 256-row tcgen05.mma (cta_group::2) issued by one thread of CTA 0:
//   S = Q K^T   (M 256, N 128 keys, K d): A = each CTA's query tile, B = the 128-key
//               tile split by keys, CTA r holding keys 64r .. 64r+63;
//   O += P V    (M 256, N d, K 128 keys): A = P in each CTA's TMEM, B = the V tile
//               split by columns, CTA r holding columns 64r .. 64r+63.
// So each SM loads half of every K and V tile (tiled TMA, 128-byte swizzle, bytes
// counted on CTA 0's barrier) and still feeds 256 query rows per tile pair, and each
// SM's TMEM holds only its own tile: S in two 128-column buffers and O (384 of 512
// columns).  With S double-buffered the tensor cores compute S(j+1) while the softmax
// works on S(j):
//   MMA order   S(0) S(1) | P.V(0) S(2) | P.V(1) S(3) | ...   (P.V(j) waits for P(j))
// P(j) is written as bf16 into S buffer j % 2 and S(j+2) reuses that buffer after
// P.V(j) has read it (one thread issues both, in order).
//
// In each CTA warp 0 loads and warps 2-17 run the softmax, one thread per query row and
// 32-key quarter of the block (four warps per SM sub-partition share a TMEM lane quarter,
// so one warp's loads, exchanges and stores overlap the others' exponentials); the four
// parts of a row agree on the block maximum through shared memory under a 128-thread
// named barrier.  The online softmax keeps the running max per row in fp32 and rescales
// O in TMEM only when it grows by more than 2^8.  Commits of the pair's MMAs arrive on
// the barriers of both CTAs; the softmax warps of CTA 1 arrive on CTA 0's P-ready
// barrier through its cluster address.  Every mbarrier wait is bounded; the only
// unbounded waits are the two cluster barriers, which every thread of both CTAs reaches
// on every path.
#pragma once
#include <cooperative_groups.h>
#include "tc_ptx.cuh"

namespace quoka {

constexpr int AT2_THREADS = 576;   // warp 0 load, warp 1 MMA (CTA 0), warps 2-17 softmax
constexpr int AT2_ST = 4;          // stages of (K half-tile, V half-tile) per block
constexpr float AT2_RESCALE_LOG2 = 8.0f;

struct At2Cfg {
  static constexpr int D = 128;
  static constexpr int Q_BYTES = 128 * D * 2;      // this CTA's query tile
  static constexpr int KH_BYTES = 64 * D * 2;      // 64 keys x 128 dims
  static constexpr int VH_BYTES = 128 * 64 * 2;    // 128 keys x 64 dims
  static constexpr int K_BYTES = AT2_ST * KH_BYTES;
  static constexpr int V_BYTES = AT2_ST * VH_BYTES;
  // qfull, qpeer, stage full/empty ring, sfull[2], pready[2]
  static constexpr int NBAR = 2 + 2 * AT2_ST + 2 + 2;
  static constexpr int XBUF = 2 * 4 * 128 * 4;   // [phase][part][row] exchange slots
  static constexpr int SMEM = 1024 + Q_BYTES + K_BYTES + V_BYTES + NBAR * 8 + 16 + XBUF;
};

struct Attn2Params {
  int h_q, h_kv, G, C, TP;
  long long kc_stride;             // rows per (sequence, KV head) block of the compacted cache
  float scale_log2;                // log2(e) / sqrt(d)
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(AT2_THREADS, 1)
attn_tc2_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ SeqTable tab,
                const __grid_constant__ Attn2Params p, __nv_bfloat16* __restrict__ out) {
  using Cfg = At2Cfg;
  constexpr int D = Cfg::D;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::Q_BYTES;
  uint8_t* sV = sK + Cfg::K_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + Cfg::V_BYTES);
  uint64_t* qfull = bars;                  // this CTA's query tile landed
  uint64_t* qpeer = bars + 1;              // (CTA 0) CTA 1's query tile landed
  // stage s holds K and V of block j (j % AT2_ST == s) for both CTAs; kvfull counts the
  // pair's bytes (CTA 0), kvempty completes when P.V(j) has finished (both CTAs), which
  // also tells the softmax that O holds blocks 0..j
  uint64_t* kvfull = bars + 2;
  uint64_t* kvempty = kvfull + AT2_ST;
  uint64_t* sfull = kvempty + AT2_ST;      // [buffer], both CTAs
  uint64_t* pready = sfull + 2;            // [buffer], CTA 0: 32 softmax warps of the pair
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pready + 2);
  float* xbuf = reinterpret_cast<float*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster.block_rank();
  const int b = blockIdx.z, g = blockIdx.y;
  const int npairs = (p.C + 2 * p.TP - 1) / (2 * p.TP);
  const int pair = npairs - 1 - (int)(blockIdx.x >> 1);     // longest key ranges first
  const int t0 = pair * 2 * p.TP;
  const int nsel = tab.nsel[b];
  const int tend = min(p.C, t0 + 2 * p.TP);                  // positions [t0, tend) of the pair
  const int nkeys = nsel + tend;
  const int nblk = (nkeys + 127) / 128;                      // same for both CTAs
  const int kc_row0 = (int)((long long)(b * p.h_kv + g) * p.kc_stride);
  constexpr uint16_t kBoth = 0x3;

  if (threadIdx.x == 0) {
    ptx::mbar_init(qfull, 1);
    ptx::mbar_init(qpeer, 1);
    for (int s = 0; s < AT2_ST; ++s) { ptx::mbar_init(&kvfull[s], 1); ptx::mbar_init(&kvempty[s], 1); }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sfull[i], 1);
      ptx::mbar_init(&pready[i], 32);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, 512);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  cluster.sync();                          // barriers and TMEM of both CTAs ready
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- loads ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&qmap);
      ptx::prefetch_tmap(&kmap);
      ptx::prefetch_tmap(&vmap);
    }
    // Q: 32 groups of 4 rows; row r is head r / TP, position t0 + rank*TP + r % TP
    // (rows past G*TP or C repeat a valid row; never stored)
    if (lane == 0) ptx::mbar_expect_tx(qfull, (uint32_t)Cfg::Q_BYTES);
    __syncwarp();
    {
      const int r0 = lane * 4;
      int rows[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = r0 + k;
        int hl = r / p.TP, t = t0 + (int)rank * p.TP + r % p.TP;
        if (hl >= p.G || t >= p.C) { hl = 0; t = t0; }
        rows[k] = (b * p.h_q + g * p.G + hl) * p.C + t;
      }
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
        ptx::tma_gather4(sQ + kb * 16384 + r0 * 128, &qmap, qfull, kb * 64, rows[0], rows[1], rows[2], rows[3]);
    }
    if (lane == 0) {
      bool ok = true;
      if (rank == 1) {                     // tell CTA 0 that this CTA's query tile landed
        ok = ptx::mbar_wait_sleep(qfull, 0);
        if (ok) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(qpeer), 0));
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const int st = j % AT2_ST;
        const int row = kc_row0 + j * 128;
        ok = ptx::mbar_wait_sleep(&kvempty[st], ((uint32_t)(j / AT2_ST) & 1u) ^ 1u);
        if (!ok) break;
        if (rank == 0) ptx::mbar_expect_tx(&kvfull[st], 2u * (Cfg::KH_BYTES + Cfg::VH_BYTES));
        const uint32_t fbar = ptx::mapa_shared(ptx::smem_u32(&kvfull[st]), 0);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
          ptx::tma_load_2d_pair(sK + st * Cfg::KH_BYTES + kb * 8192, &kmap, fbar, kb * 64, row + 64 * (int)rank);
        ptx::tma_load_2d_pair(sV + st * Cfg::VH_BYTES, &vmap, fbar, 64 * (int)rank, row);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: one thread of CTA 0 for the pair ----------------
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_s = ptx::idesc_bf16(256, 128, false);
      const uint32_t idesc_o = ptx::idesc_bf16(256, D, true);
      const uint64_t q_d = ptx::sdesc_sw128(ptx::smem_u32(sQ), 16, 1024);
      const uint64_t k_d = ptx::sdesc_sw128(ptx::smem_u32(sK), 16, 1024);
      const uint64_t v_d = ptx::sdesc_sw128(ptx::smem_u32(sV), 16384, 1024);
      const uint32_t q_lo = (uint32_t)q_d, q_hi = (uint32_t)(q_d >> 32);
      const uint32_t k_lo = (uint32_t)k_d, k_hi = (uint32_t)(k_d >> 32);
      const uint32_t v_lo = (uint32_t)v_d, v_hi = (uint32_t)(v_d >> 32);
      // S(j) into buffer j % 2 (columns 128 * (j % 2)); block j's K and V have landed in
      // both CTAs (P.V(j) later reads V(j) from the same stage without another wait)
      auto s_mmas = [&](int j) {
        const int st = j % AT2_ST;
        const uint32_t b0 = k_lo + (uint32_t)(st * (Cfg::KH_BYTES >> 4));
        const uint32_t d = tmem + (uint32_t)((j & 1) * 128);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16_ss_pair(d, q_lo + (uint32_t)(kb * 1024 + k * 2), q_hi,
                                  b0 + (uint32_t)(kb * 512 + k * 2), k_hi, idesc_s, (kb | k) ? 1u : 0u);
      };
      auto kv_landed = [&](int j) -> bool {
        return ptx::mbar_wait_cluster_sleep(&kvfull[j % AT2_ST], (uint32_t)(j / AT2_ST) & 1u);
      };
      bool ok = ptx::mbar_wait_sleep(qfull, 0) && ptx::mbar_wait_cluster_sleep(qpeer, 0);
      for (int j = 0; j < 2 && j < nblk && ok; ++j) {
        ok = kv_landed(j);
        if (!ok) break;
        ptx::tc_fence_after();
        s_mmas(j);
        ptx::tc_commit_pair(&sfull[j & 1], kBoth);
      }
      // Per block: every wait comes before the block's 16 MMAs, which are issued back to
      // back (a wait or commit between them lets the tensor pipe's short queue drain), and
      // both commits come after them.  The stage of block j is released once S(j+2) is
      // done, which also implies P.V(j) is.
      for (int j = 0; j < nblk && ok; ++j) {
        const int st = j % AT2_ST;
        const bool more = j + 2 < nblk;
        if (more) ok = kv_landed(j + 2);
        if (ok) ok = ptx::mbar_wait_cluster_sleep(&pready[j & 1], (uint32_t)(j >> 1) & 1u);
        if (!ok) break;
        ptx::tc_fence_after();
        // O += P(j) V(j); P(j) lies in buffer j % 2: keys 32q .. 32q+31 in columns
        // 32q .. 32q+15 (written by softmax part q)
        const uint32_t b0 = v_lo + (uint32_t)(st * (Cfg::VH_BYTES >> 4));
        const uint32_t pa = tmem + (uint32_t)((j & 1) * 128);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ptx::mma_bf16_ts_pair(tmem + 256u, pa + (uint32_t)((k >> 1) * 32 + (k & 1) * 8),
                                b0 + (uint32_t)(k * 128), v_hi, idesc_o, (j > 0 || k > 0) ? 1u : 0u);
        if (more) {
          s_mmas(j + 2);
          ptx::tc_commit_pair(&sfull[j & 1], kBoth);
        }
        ptx::tc_commit_pair(&kvempty[st], kBoth);
      }
    }
  } else {
    // ---------------- softmax: warps 2-17, one row per thread and key quarter ----------------
    const int part = ((warp - 2) >> 2) & 3;                 // key quarter of each block
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                      // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    constexpr int DP = D / 4;                               // O columns of this part
    const uint32_t o_addr = tmem + lane_off + 256u + (uint32_t)(part * DP);
    const int bar_id = 1 + quarter;
    const uint32_t pready_c0 = ptx::mapa_shared(ptx::smem_u32(pready), 0);   // CTA 0's pready[0]
    // the four parts of a row post their values and each combines all four in part order;
    // slots alternate between two sets, so one barrier per exchange suffices
    int xphase = 0;
    auto exchange = [&](float v, bool is_max) -> float {
      float* slot = xbuf + (xphase & 1) * 512 + r;
      slot[part * 128] = v;
      ptx::named_bar(bar_id, 128);
      const float a0 = slot[0], a1 = slot[128], a2 = slot[256], a3 = slot[384];
      ++xphase;
      return is_max ? fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) : (a0 + a1) + (a2 + a3);
    };
    const int hl = r / p.TP;
    const int t = t0 + (int)rank * p.TP + r % p.TP;
    const bool row_valid = hl < p.G && t < p.C;
    const int tmin = t0 + (int)rank * p.TP;                 // smallest position in this tile
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    // The four warps of a row quarter take part in exactly one exchange per block and one
    // at the end, whatever happens, so the named barrier never waits for a warp that left:
    // after a failed (timed-out) wait a warp skips the work but keeps the exchanges.
    for (int j = 0; j < nblk; ++j) {
      const int buf = j & 1;
      if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&sfull[buf], (uint32_t)(j >> 1) & 1u));
      if (!ok) {
        (void)exchange(0.f, true);
        continue;
      }
      ptx::tc_fence_after();
      // this part's 32 keys of S(j); P(j) goes to the first 16 columns of the same place
      const uint32_t s_addr = tmem + lane_off + (uint32_t)(buf * 128 + part * 32);
      const uint32_t p_addr = s_addr;
      float s[32];
      {
        uint32_t u[32];
        ptx::tmem_ld32(s_addr, u);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = __uint_as_float(u[i]);
      }
      const int kb0 = j * 128 + part * 32;
      if (kb0 + 31 >= nsel + tmin || kb0 + 31 >= nkeys) {   // keys reach the causal part
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int kk = kb0 + c;
          const bool valid = kk < nkeys && (kk < nsel || kk - nsel <= t);
          if (!valid) s[c] = -INFINITY;
        }
      }
      float mx;
      {
        float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
        for (int c = 4; c < 28; c += 8) {
          m0 = ptx::max3(m0, s[c], s[c + 1]);
          m1 = ptx::max3(m1, s[c + 2], s[c + 3]);
          m2 = ptx::max3(m2, s[c + 4], s[c + 5]);
          m3 = ptx::max3(m3, s[c + 6], s[c + 7]);
        }
        m0 = ptx::max3(m0, s[28], s[29]);
        m1 = ptx::max3(m1, s[30], s[31]);
        mx = exchange(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)), true);
      }
      const float m_cand = mx * p.scale_log2;
      const bool grow = m_cand > m_run + AT2_RESCALE_LOG2 || (m_run == -INFINITY && m_cand > -INFINITY);
      float alpha = 1.f;
      if (grow) {
        alpha = (m_run == -INFINITY) ? 0.f : ptx::ex2_approx(m_run - m_cand);
        m_run = m_cand;
        l_run *= alpha;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ptx::ex2_approx(fmaf(s[2 * i], p.scale_log2, -m_use));
          const float p1 = ptx::ex2_approx(fmaf(s[2 * i + 1], p.scale_log2, -m_use));
          ls[i & 3] += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        ptx::tmem_st16(p_addr, pk);
      }
      l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // rescale O (blocks 0..j-1) once P.V(j-1) has finished, i.e. stage (j-1) % ST is
        // released.  The parity wait is unambiguous: the stage's previous release,
        // P.V(j-1-ST), precedes S(j) (which was issued after P.V(j-2)), and its next one,
        // P.V(j-1+ST), needs this warp's P of a later block
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&kvempty[(j - 1) % AT2_ST], (uint32_t)((j - 1) / AT2_ST) & 1u));
        if (ok) ptx::tc_fence_after();
#pragma unroll
        for (int c = 0; c < (ok ? DP : 0); c += 16) {
          uint32_t u[16];
          ptx::tmem_ld16(o_addr + (uint32_t)c, u);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          ptx::tmem_st16(o_addr + (uint32_t)c, u);
        }
      }
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      __syncwarp();
      // relaxed arrive: P and the rescaled O are TMEM stores already completed by
      // tcgen05.wait::st and ordered by the fence above; a cluster-scope release here
      // would stall the warp on its unrelated outstanding memory operations
      if (ok && lane == 0) ptx::mbar_arrive_cluster_relaxed(pready_c0 + (uint32_t)(buf * 8));
    }
    // epilogue: O / l -> bf16 rows of out[b, g*G + hl, t, :], this part's columns, once
    // the last P.V has released its stage (its commit covers every earlier MMA)
    if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&kvempty[(nblk - 1) % AT2_ST], (uint32_t)((nblk - 1) / AT2_ST) & 1u));
    const float l_row = exchange(ok ? l_run : 0.f, false);   // every pair member reaches this
    if (ok) {
      ptx::tc_fence_after();
      const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
      __nv_bfloat16* orow = out + ((size_t)(b * p.h_q + g * p.G + (row_valid ? hl : 0)) * p.C +
                                   (row_valid ? t : 0)) * D + part * DP;
#pragma unroll
      for (int c = 0; c < DP; c += 16) {
        uint32_t u[16];
        ptx::tmem_ld16(o_addr + (uint32_t)c, u);
        ptx::tmem_ld_wait();
        uint4 w0, w1;
        w0.x = pack_bf16x2(__uint_as_float(u[0]) * inv_l, __uint_as_float(u[1]) * inv_l);
        w0.y = pack_bf16x2(__uint_as_float(u[2]) * inv_l, __uint_as_float(u[3]) * inv_l);
        w0.z = pack_bf16x2(__uint_as_float(u[4]) * inv_l, __uint_as_float(u[5]) * inv_l);
        w0.w = pack_bf16x2(__uint_as_float(u[6]) * inv_l, __uint_as_float(u[7]) * inv_l);
        w1.x = pack_bf16x2(__uint_as_float(u[8]) * inv_l, __uint_as_float(u[9]) * inv_l);
        w1.y = pack_bf16x2(__uint_as_float(u[10]) * inv_l, __uint_as_float(u[11]) * inv_l);
        w1.z = pack_bf16x2(__uint_as_float(u[12]) * inv_l, __uint_as_float(u[13]) * inv_l);
        w1.w = pack_bf16x2(__uint_as_float(u[14]) * inv_l, __uint_as_float(u[15]) * inv_l);
        if (row_valid) {
          reinterpret_cast<uint4*>(orow + c)[0] = w0;
          reinterpret_cast<uint4*>(orow + c)[1] = w1;
        }
      }
    }
  }

  ptx::tc_fence_before();
  cluster.sync();                          // the pair's MMAs and loads are over on both SMs
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace quoka
