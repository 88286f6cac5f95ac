// K4 (tensor-core form, bf16): dense attention of the chunk over its compacted cache
// (QUOKA page, Figure 1(a): the sub-selected KV cache goes into a dense attention
// kernel; QUILT page: the K/V entries a group of queries selected in common are loaded
// once and reused by all of them).
//
// One CTA per (sequence, KV head, 2 x TP chunk positions).  Its two 128-row query
// tiles pack the G query heads of the KV head (TP = 128 / G positions each), so every
// K/V tile in shared memory feeds 256 query rows of G heads.  The query tiles are
// gathered once by TMA (tile::gather4).  K/V come from the compacted cache of the
// (sequence, KV head): the selected prefix rows followed by the chunk's own rows,
// contiguous (compact.cuh), so one thread streams each 128-key block with two tiled
// TMA loads per operand (128-byte swizzle) into a 3-stage K ring and a 2-stage V ring.
//
// TMEM holds S0, S1 (128 x 128 fp32 logits of each tile) and O0, O1 (128 x d fp32).
// Warp 0 loads, one thread of warp 1 issues tcgen05.mma, warps 2-9 and 10-17 run the
// softmax of tile 0 and tile 1, so one tile's softmax overlaps the other tile's MMAs.
// Each query row is shared by two warps of the same SM sub-partition, one per 64-key
// half of the block (one thread per row and half): the exponentials of a tile run on
// 8 warps, two per sub-partition, which is what it takes to keep the multi-function
// units busy.  The two halves of a row agree on the block maximum through shared memory
// under a 64-thread named barrier.  P is written back as bf16 into TMEM inside each
// half's own S columns (keys 0-63 -> columns 0-31, keys 64-127 -> columns 96-127) and
// consumed from TMEM by the P.V MMA (A operand in TMEM).
// The online softmax keeps its running max per row in fp32 and rescales O in TMEM
// only when the max grows by more than 2^8, so the exponent stays bounded.
#pragma once
#include "tc_ptx.cuh"

namespace quoka {

constexpr int ATC_THREADS = 576;   // warp 0 load, warp 1 MMA, 2-9 softmax tile 0, 10-17 tile 1
constexpr int ATC_KST = 3;         // K stages
constexpr int ATC_VST = 2;         // V stages
constexpr float ATC_RESCALE_LOG2 = 8.0f;

struct AttnTcParams {
  int h_q, h_kv, G, C, TP, b_max;
  long long kc_stride;             // rows per (sequence, KV head) block of the compacted cache
  long long rows_per_head;
  float scale_log2;                // log2(e) / sqrt(d)
};

template <int D>
struct AtcCfg {
  static constexpr int KB = D / 64;
  static constexpr int TILE_BYTES = 128 * D * 2;  // 128 rows of one operand
  static constexpr int Q_BYTES = 2 * TILE_BYTES;
  static constexpr int K_BYTES = ATC_KST * TILE_BYTES;
  static constexpr int V_BYTES = ATC_VST * TILE_BYTES;
  // qfull, K and V full/empty rings, and per tile sfull, pready, odone
  static constexpr int NBAR = 1 + 2 * ATC_KST + 2 * ATC_VST + 2 + 2 + 2;
  static constexpr int XBUF = 2 * 128 * 4;         // per-row exchange slots of both tiles
  static constexpr int SMEM = 1024 + Q_BYTES + K_BYTES + V_BYTES + NBAR * 8 + 16 + XBUF;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(ATC_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const __grid_constant__ SeqTable tab,
               const __grid_constant__ AttnTcParams p, __nv_bfloat16* __restrict__ out) {
  using Cfg = AtcCfg<D>;
  constexpr int KB = Cfg::KB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::Q_BYTES;
  uint8_t* sV = sK + Cfg::K_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + Cfg::V_BYTES);
  uint64_t* qfull = bars;
  uint64_t* kfull = bars + 1;
  uint64_t* kempty = kfull + ATC_KST;
  uint64_t* vfull = kempty + ATC_KST;
  uint64_t* vempty = vfull + ATC_VST;
  uint64_t* sfull = vempty + ATC_VST;   // [2]
  uint64_t* pready = sfull + 2;         // [2]
  uint64_t* odone = pready + 2;         // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(odone + 2);
  float* xbuf = reinterpret_cast<float*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, g = blockIdx.y;
  const int npairs = (p.C + 2 * p.TP - 1) / (2 * p.TP);
  const int pair = npairs - 1 - (int)blockIdx.x;           // longest key ranges first
  const int t0 = pair * 2 * p.TP;
  const int nsel = tab.nsel[b];
  const int tend = min(p.C, t0 + 2 * p.TP);                  // positions [t0, tend)
  const int nkeys = nsel + tend;                             // selected + chunk keys 0..tend-1
  const int nblk = (nkeys + 127) / 128;
  const int kc_row0 = (int)((long long)(b * p.h_kv + g) * p.kc_stride);

  if (threadIdx.x == 0) {
    ptx::mbar_init(qfull, 1);
    for (int s = 0; s < ATC_KST; ++s) { ptx::mbar_init(&kfull[s], 1); ptx::mbar_init(&kempty[s], 1); }
    for (int s = 0; s < ATC_VST; ++s) { ptx::mbar_init(&vfull[s], 1); ptx::mbar_init(&vempty[s], 1); }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sfull[i], 1);
      ptx::mbar_init(&pready[i], 8);
      ptx::mbar_init(&odone[i], 1);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- loads: Q once by gather4, then K and V blocks by tiled TMA --------
    if (lane == 0) {
      ptx::prefetch_tmap(&qmap);
      ptx::prefetch_tmap(&kmap);
      ptx::prefetch_tmap(&vmap);
    }
    // Q: 2 tiles x 32 groups of 4 rows; row r of tile i is head r / TP, position
    // t0 + i*TP + r % TP (rows past G*TP or C repeat a valid row; never stored)
    if (lane == 0) ptx::mbar_expect_tx(qfull, (uint32_t)Cfg::Q_BYTES);
    __syncwarp();
    for (int grp = lane; grp < 64; grp += 32) {
      const int tile = grp >> 5, r0 = (grp & 31) * 4;
      int rows[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = r0 + k;
        int hl = r / p.TP, t = t0 + tile * p.TP + r % p.TP;
        if (hl >= p.G || t >= p.C) { hl = 0; t = t0; }
        rows[k] = (b * p.h_q + g * p.G + hl) * p.C + t;
      }
#pragma unroll
      for (int kb = 0; kb < KB; ++kb)
        ptx::tma_gather4(sQ + tile * Cfg::TILE_BYTES + kb * 16384 + r0 * 128, &qmap, qfull, kb * 64,
                         rows[0], rows[1], rows[2], rows[3]);
    }
    if (lane == 0) {
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        const int ks = j % ATC_KST, vs = j % ATC_VST;
        const uint32_t kph = (uint32_t)(j / ATC_KST) & 1u, vph = (uint32_t)(j / ATC_VST) & 1u;
        const int row = kc_row0 + j * 128;
        ok = ptx::mbar_wait(&kempty[ks], kph ^ 1u);
        if (!ok) break;
        ptx::mbar_expect_tx(&kfull[ks], (uint32_t)Cfg::TILE_BYTES);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          ptx::tma_load_2d(sK + ks * Cfg::TILE_BYTES + kb * 16384, &kmap, &kfull[ks], kb * 64, row);
        ok = ptx::mbar_wait(&vempty[vs], vph ^ 1u);
        if (!ok) break;
        ptx::mbar_expect_tx(&vfull[vs], (uint32_t)Cfg::TILE_BYTES);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          ptx::tma_load_2d(sV + vs * Cfg::TILE_BYTES + kb * 16384, &vmap, &vfull[vs], kb * 64, row);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc_s = ptx::idesc_bf16(128, 128, false);
      const uint32_t idesc_o = ptx::idesc_bf16(128, D, true);
      bool ok = ptx::mbar_wait(qfull, 0);
      // Descriptor halves: only the start-address field (low half, address >> 4) moves as
      // the MMAs step through k, the tile and the ring stage.
      const uint64_t q_d = ptx::sdesc_sw128(ptx::smem_u32(sQ), 16, 1024);
      const uint64_t k_d = ptx::sdesc_sw128(ptx::smem_u32(sK), 16, 1024);
      const uint64_t v_d = ptx::sdesc_sw128(ptx::smem_u32(sV), 16384, 1024);
      const uint32_t q_lo = (uint32_t)q_d, q_hi = (uint32_t)(q_d >> 32);
      const uint32_t k_lo = (uint32_t)k_d, k_hi = (uint32_t)(k_d >> 32);
      const uint32_t v_lo = (uint32_t)v_d, v_hi = (uint32_t)(v_d >> 32);
      constexpr uint32_t TILE16 = (uint32_t)Cfg::TILE_BYTES >> 4;
      auto issue_s = [&](int i, int j) {
        const uint32_t a0 = q_lo + (uint32_t)i * TILE16;
        const uint32_t b0 = k_lo + (uint32_t)(j % ATC_KST) * TILE16;
        const uint32_t d = tmem + (uint32_t)(i * 128);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16_ss_lh(d, a0 + (uint32_t)(kb * 1024 + k * 2), q_hi, b0 + (uint32_t)(kb * 1024 + k * 2),
                                k_hi, idesc_s, (kb | k) ? 1u : 0u);
        ptx::tc_commit(&sfull[i]);
      };
      auto issue_pv = [&](int i, int j) {
        const uint32_t b0 = v_lo + (uint32_t)(j % ATC_VST) * TILE16;
        const uint32_t d = tmem + (uint32_t)(256 + i * 128), pa = tmem + (uint32_t)(i * 128);
        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
        for (int k = 0; k < 8; ++k)                          // 16 keys per MMA
          ptx::mma_bf16_ts_lh(d, pa + (uint32_t)(k < 4 ? k * 8 : 96 + (k - 4) * 8), b0 + (uint32_t)(k * 128),
                              v_hi, idesc_o, k > 0 ? 1u : acc0);
        ptx::tc_commit(&odone[i]);
      };
      if (ok) ok = ptx::mbar_wait(&kfull[0], 0);
      if (ok) {
        ptx::tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        ptx::tc_commit(&kempty[0]);
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const uint32_t par = (uint32_t)j & 1u;
        ok = ptx::mbar_wait(&vfull[j % ATC_VST], (uint32_t)(j / ATC_VST) & 1u);
        if (ok) ok = ptx::mbar_wait(&pready[0], par);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_pv(0, j);
        const bool more = j + 1 < nblk;
        if (more) {
          ok = ptx::mbar_wait(&kfull[(j + 1) % ATC_KST], (uint32_t)((j + 1) / ATC_KST) & 1u);
          if (!ok) break;
          ptx::tc_fence_after();
          issue_s(0, j + 1);
        }
        ok = ptx::mbar_wait(&pready[1], par);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_pv(1, j);
        ptx::tc_commit(&vempty[j % ATC_VST]);
        if (more) {
          issue_s(1, j + 1);
          ptx::tc_commit(&kempty[(j + 1) % ATC_KST]);
        }
      }
    }
  } else {
    // ---------------- softmax: warps 2-9 tile 0, warps 10-17 tile 1 ----------------
    // Warp w serves TMEM lanes 32 * (w % 4) .. + 31 (one query row per thread) and key
    // half (w - 2) / 4 % 2 of every block; the two warps of a row exchange block maxima
    // (and at the end row sums) through shared memory under a 64-thread named barrier.
    const int tile = (warp - 2) >> 3;
    const int half = ((warp - 2) >> 2) & 1;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                      // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (uint32_t)(tile * 128 + half * 64);
    const uint32_t p_addr = tmem + lane_off + (uint32_t)(tile * 128 + half * 96);
    constexpr int DH = D / 2;                               // O columns of this half
    const uint32_t o_addr = tmem + lane_off + (uint32_t)(256 + tile * 128 + half * DH);
    float* xslot = xbuf + tile * 128 + r;
    const int bar_id = 1 + tile * 4 + quarter;
    // half 0 posts v, half 1 combines it with its own and posts the result for half 0
    auto exchange = [&](float v, bool is_max) -> float {
      if (half == 0) *xslot = v;
      ptx::named_bar(bar_id, 64);
      float res = v;
      if (half == 1) {
        res = is_max ? fmaxf(v, *xslot) : v + *xslot;
        *xslot = res;
      }
      ptx::named_bar(bar_id, 64);
      if (half == 0) res = *xslot;
      return res;
    };
    const int hl = r / p.TP;
    const int t = t0 + tile * p.TP + r % p.TP;
    const bool row_valid = hl < p.G && t < p.C;
    const int tmin = t0 + tile * p.TP;                      // smallest position in this tile
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    // Both warps of a row pair take part in exactly one exchange per block and one at
    // the end, whatever happens, so the named barrier can never wait for a warp that left:
    // after a failed (timed-out) wait a warp skips the work but keeps the exchanges.
    for (int j = 0; j < nblk; ++j) {
      if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait(&sfull[tile], (uint32_t)j & 1u));
      if (!ok) {
        (void)exchange(0.f, true);
        continue;
      }
      ptx::tc_fence_after();
      float s[64];
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t u[32];
        ptx::tmem_ld32(s_addr + (uint32_t)c, u);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c + i] = __uint_as_float(u[i]);
      }
      ptx::tmem_ld_wait();
      const int kb0 = j * 128 + half * 64;
      if (kb0 + 63 >= nsel + tmin || kb0 + 63 >= nkeys) {   // keys reach the causal part
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int kk = kb0 + c;
          const bool valid = kk < nkeys && (kk < nsel || kk - nsel <= t);
          if (!valid) s[c] = -INFINITY;
        }
      }
      float mx;
      {
        float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
        for (int c = 4; c < 60; c += 8) {
          m0 = ptx::max3(m0, s[c], s[c + 1]);
          m1 = ptx::max3(m1, s[c + 2], s[c + 3]);
          m2 = ptx::max3(m2, s[c + 4], s[c + 5]);
          m3 = ptx::max3(m3, s[c + 6], s[c + 7]);
        }
        m0 = ptx::max3(m0, s[60], s[61]);
        m1 = ptx::max3(m1, s[62], s[63]);
        mx = exchange(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)), true);
      }
      const float m_cand = mx * p.scale_log2;
      const bool grow = m_cand > m_run + ATC_RESCALE_LOG2 || (m_run == -INFINITY && m_cand > -INFINITY);
      float alpha = 1.f;
      if (grow) {
        alpha = (m_run == -INFINITY) ? 0.f : ptx::ex2_approx(m_run - m_cand);
        m_run = m_cand;
        l_run *= alpha;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ptx::ex2_approx(fmaf(s[c + 2 * i], p.scale_log2, -m_use));
          const float p1 = ptx::ex2_approx(fmaf(s[c + 2 * i + 1], p.scale_log2, -m_use));
          ls[i & 3] += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
        ptx::tmem_st16(p_addr + (uint32_t)(c / 2), pk);
      }
      l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (ok && j > 0 && __any_sync(0xffffffffu, grow)) {
        // O holds blocks 0..j-1 once the previous P.V of this tile has finished
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&odone[tile], (uint32_t)(j - 1) & 1u));
        if (ok) ptx::tc_fence_after();
#pragma unroll
        for (int c = 0; c < (ok ? DH : 0); c += 16) {
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
      if (ok && lane == 0) ptx::mbar_arrive(&pready[tile]);
    }
    // epilogue: O / l -> bf16 rows of out[b, g*G + hl, t, :], this half's columns
    if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait(&odone[tile], (uint32_t)(nblk - 1) & 1u));
    const float l_row = exchange(ok ? l_run : 0.f, false);   // every pair member reaches this
    if (ok) {
      ptx::tc_fence_after();
      const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
      __nv_bfloat16* orow = out + ((size_t)(b * p.h_q + g * p.G + (row_valid ? hl : 0)) * p.C +
                                   (row_valid ? t : 0)) * D + half * DH;
#pragma unroll
      for (int c = 0; c < DH; c += 16) {
        uint32_t u[16];
        ptx::tmem_ld16(o_addr + (uint32_t)c, u);
        ptx::tmem_ld_wait();
        uint4 w0, w1;
        w0.x = pack_bf16(__uint_as_float(u[0]) * inv_l, __uint_as_float(u[1]) * inv_l);
        w0.y = pack_bf16(__uint_as_float(u[2]) * inv_l, __uint_as_float(u[3]) * inv_l);
        w0.z = pack_bf16(__uint_as_float(u[4]) * inv_l, __uint_as_float(u[5]) * inv_l);
        w0.w = pack_bf16(__uint_as_float(u[6]) * inv_l, __uint_as_float(u[7]) * inv_l);
        w1.x = pack_bf16(__uint_as_float(u[8]) * inv_l, __uint_as_float(u[9]) * inv_l);
        w1.y = pack_bf16(__uint_as_float(u[10]) * inv_l, __uint_as_float(u[11]) * inv_l);
        w1.z = pack_bf16(__uint_as_float(u[12]) * inv_l, __uint_as_float(u[13]) * inv_l);
        w1.w = pack_bf16(__uint_as_float(u[14]) * inv_l, __uint_as_float(u[15]) * inv_l);
        if (row_valid) {
          reinterpret_cast<uint4*>(orow + c)[0] = w0;
          reinterpret_cast<uint4*>(orow + c)[1] = w1;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace quoka
