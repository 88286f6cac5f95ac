// K4 (tensor-core form over SM pairs, bf16, d = 128): dense attention of the chunk over
// its compacted cache (QUOKA page, Figure 1(a): the sub-selected KV cache goes into a
// dense attention kernel; QUILT page: the K/V entries a group of queries selected in
// common are loaded once and reused by all of them).
//
// The same kernel runs per-query selections (QUILT page, summary): each pair of CTAs then
// attends over the union of its 256 rows' key sets, with a per-row membership mask in
// place of the causal rule (perq_tc.cuh builds the union, the masks and the K/V block).
//
// A cluster of two CTAs on two SMs serves (sequence, KV head, 2 x TP chunk positions)
// tiles, listed by sequence (most selected keys first), KV head and pair (longest key
// range first).  Either one cluster per tile (kPersist = false), or (kPersist = true) the
// grid holds as many clusters as can be resident at once and cluster c takes tiles c,
// c + N, c + 2N, ... of the list, keeping its TMEM, barriers and pipeline across tiles, so
// the next tile's query gather (into a second query buffer), K/V loads and first S MMAs
// run while the current tile drains.  CTA r owns query tile r: 128 rows packing the G
// query heads of the KV head at TP = 128 / G positions, gathered by TMA (tile::gather4).
// The pair runs every
// MMA as one 256-row tcgen05.mma (cta_group::2) issued by one thread of CTA 0:
//   S = Q K^T   (M 256, N 128 keys, K d): A = each CTA's query tile, B = the 128-key
//               tile split by keys, CTA r holding keys 64r .. 64r+63;
//   O += P V    (M 256, N d, K 128 keys): A = P in each CTA's TMEM, B = the V tile
//               split by columns, CTA r holding columns 64r .. 64r+63.
// So each SM loads half of every K and V tile (tiled TMA, 128-byte swizzle, bytes
// counted on CTA 0's barrier) and still feeds 256 query rows per tile pair, and each
// SM's TMEM holds only its own tile: S in two 128-column buffers and two O accumulators
// (512 columns).  The key blocks are split by parity between two softmax groups, each
// with its own running max, row sum and O (a split of the key range, combined at the
// end like a split-K reduction):
//   MMA order   S(0) S(1) | P.V(0) S(2) | P.V(1) S(3) | ...   (P.V(j) waits for P(j))
//   P.V(j) accumulates into O_{j % 2}
// P(j) is written as bf16 into S buffer j % 2 and S(j+2) reuses that buffer after
// P.V(j) has read it (one thread issues both, in order).
//
// In each CTA warp 0 loads and warps 2-17 run the softmax: warps 2-9 take the even key
// blocks and warps 10-17 the odd ones, one thread per query row and 64-key half of a
// block.  Each SM sub-partition holds two warps of each group, a block apart, so one
// group's exponentials overlap the other group's TMEM loads, exchange and waits.  The
// halves of a row agree on the block maximum through shared memory under a 64-thread
// named barrier.  The online softmax keeps the running max per row in fp32 and rescales
// its group's O in TMEM only when the max grows by more than 2^8; at the end the two
// groups meet per row quarter and write O = (O_0 f_0 + O_1 f_1) / (l_0 f_0 + l_1 f_1),
// f_g = 2^(m_g - max(m_0, m_1)).  Commits of the pair's MMAs arrive on
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
  static constexpr int Q_BYTES = 128 * D * 2;      // this CTA's query tile (two buffers)
  static constexpr int KH_BYTES = 64 * D * 2;      // 64 keys x 128 dims
  static constexpr int VH_BYTES = 128 * 64 * 2;    // 128 keys x 64 dims
  static constexpr int K_BYTES = AT2_ST * KH_BYTES;
  static constexpr int V_BYTES = AT2_ST * VH_BYTES;
  // qfull[2], qpeer[2], qempty[2], stage full/empty ring, sfull[2], pready[2]
  static constexpr int NBAR = 6 + 2 * AT2_ST + 2 + 2;
  static constexpr int XBUF = (2 * 2 * 2 * 128 + 2 * 2 * 128) * 4;   // exchange slots, then (m, l) per group
  // the persistent form double-buffers the query tile
  static constexpr int smem(bool persist) {
    return 1024 + (persist ? 2 : 1) * Q_BYTES + K_BYTES + V_BYTES + NBAR * 8 + 16 + XBUF;
  }
};

// One tile of the list: (sequence b, KV head g, pair) and its key block.
struct At2Tile {
  int b, g, t0, nsel, nkeys, nblk, kc_row0;
  long long tile;
};

struct Attn2Params {
  int h_q, h_kv, G, C, TP;
  long long kc_stride;             // rows per (sequence, KV head) block of the compacted cache
  float scale_log2;                // log2(e) / sqrt(d)
  int border[QUOKA_MAX_BATCH];     // grid z -> sequence, longest key lists first
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// kMember = false: the chunk step; block (b, g) of the compacted cache holds the n_b
//   selected rows, then the chunk's rows, visible to position t up to its own.
// kMember = true: per-query sets; block `tile` (one per pair of CTAs) holds the union of
//   the tile's sets, ucount[tile] keys, and key u counts for a row when the row's mask
//   word pair of u's 128-key block has u's bit (mask [tile][256 rows][mwords]).
// kPersist = false: one tile per cluster, grid (2 x pairs, KV heads, sequences in the
//   order of border); true: the grid holds the resident clusters, which walk the tile list.
template <bool kMember, bool kPersist>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(AT2_THREADS, 1)
attn_tc2_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ SeqTable tab,
                const __grid_constant__ Attn2Params p, __nv_bfloat16* __restrict__ out,
                const uint32_t* __restrict__ mask, const int32_t* __restrict__ ucount, int mwords) {
  using Cfg = At2Cfg;
  constexpr int D = Cfg::D;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* sQ = smem;                      // one query buffer, or two when persistent
  uint8_t* sK = sQ + (kPersist ? 2 : 1) * Cfg::Q_BYTES;
  uint8_t* sV = sK + Cfg::K_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + Cfg::V_BYTES);
  uint64_t* qfull = bars;                  // [buffer] this CTA's query tile landed
  uint64_t* qpeer = bars + 2;              // [buffer] (CTA 0) CTA 1's query tile landed
  uint64_t* qempty = bars + 4;             // [buffer] the MMAs reading it are done (both CTAs)
  // stage s holds K and V of block jj (jj % AT2_ST == s, jj counted over all the
  // cluster's tiles) for both CTAs; kvfull counts the pair's bytes (CTA 0), kvempty
  // completes when P.V(jj) has finished (both CTAs), which also tells the softmax that O
  // holds the tile's blocks up to jj
  uint64_t* kvfull = bars + 6;
  uint64_t* kvempty = kvfull + AT2_ST;
  uint64_t* sfull = kvempty + AT2_ST;      // [buffer], both CTAs
  uint64_t* pready = sfull + 2;            // [buffer], CTA 0: the 16 warps of one group of the pair
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pready + 2);
  float* xbuf = reinterpret_cast<float*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster.block_rank();
  const int npairs = (p.C + 2 * p.TP - 1) / (2 * p.TP);
  const int ntiles = npairs * p.h_kv * tab.batch;
  const int ncl = (int)(gridDim.x >> 1), cid = (int)(blockIdx.x >> 1);
  // tiles of this cluster (the same for both CTAs)
  const int my_tiles = kPersist ? (cid < ntiles ? (ntiles - 1 - cid) / ncl + 1 : 0) : 1;
  constexpr uint16_t kBoth = 0x3;
  auto tile_at = [&](int it) -> At2Tile {
    int pair;
    At2Tile ti;
    if constexpr (kPersist) {
      const int qi = cid + it * ncl;
      const int rest = qi / npairs;
      pair = npairs - 1 - (qi - rest * npairs);           // longest key ranges first
      ti.g = rest % p.h_kv;
      ti.b = p.border[rest / p.h_kv];
    } else {
      pair = npairs - 1 - cid;
      ti.g = (int)blockIdx.y;
      ti.b = p.border[blockIdx.z];
    }
    ti.t0 = pair * 2 * p.TP;
    ti.tile = ((long long)ti.b * p.h_kv + ti.g) * npairs + pair;
    ti.nsel = kMember ? 0 : tab.nsel[ti.b];
    const int tend = min(p.C, ti.t0 + 2 * p.TP);          // positions [t0, tend) of the pair
    ti.nkeys = kMember ? ucount[ti.tile] : ti.nsel + tend;
    ti.nblk = (ti.nkeys + 127) / 128;                     // same for both CTAs
    ti.kc_row0 = (int)(kMember ? ti.tile * p.kc_stride : (long long)(ti.b * p.h_kv + ti.g) * p.kc_stride);
    return ti;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&qfull[i], 1);
      ptx::mbar_init(&qpeer[i], 1);
      ptx::mbar_init(&qempty[i], 1);
      ptx::mbar_init(&sfull[i], 1);
      ptx::mbar_init(&pready[i], 16);
    }
    for (int s = 0; s < AT2_ST; ++s) { ptx::mbar_init(&kvfull[s], 1); ptx::mbar_init(&kvempty[s], 1); }
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
    bool ok = true;
    int jg = 0;                            // blocks of the earlier tiles
    for (int it = 0; it < my_tiles && ok; ++it) {
      const At2Tile ti = tile_at(it);
      const int qb = kPersist ? (it & 1) : 0;
      // Q: 32 groups of 4 rows; row r is head r / TP, position t0 + rank*TP + r % TP (rows
      // past G*TP or C repeat a valid row; never stored).  The buffer was last read by the
      // MMAs of tile it - 2.
      if (kPersist && lane == 0) ok = ptx::mbar_wait_sleep(&qempty[qb], ((uint32_t)(it >> 1) & 1u) ^ 1u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) ptx::mbar_expect_tx(&qfull[qb], (uint32_t)Cfg::Q_BYTES);
      __syncwarp();
      {
        const int r0 = lane * 4;
        int rows[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = r0 + k;
          int hl = r / p.TP, t = ti.t0 + (int)rank * p.TP + r % p.TP;
          if (hl >= p.G || t >= p.C) { hl = 0; t = ti.t0; }
          rows[k] = (ti.b * p.h_q + ti.g * p.G + hl) * p.C + t;
        }
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
          ptx::tma_gather4(sQ + qb * Cfg::Q_BYTES + kb * 16384 + r0 * 128, &qmap, &qfull[qb], kb * 64,
                           rows[0], rows[1], rows[2], rows[3]);
      }
      if (lane == 0) {
        for (int j = 0; j < ti.nblk && ok; ++j) {
          const int jj = jg + j;
          const int st = jj % AT2_ST;
          const int row = ti.kc_row0 + j * 128;
          ok = ptx::mbar_wait_sleep(&kvempty[st], ((uint32_t)(jj / AT2_ST) & 1u) ^ 1u);
          if (!ok) break;
          if (rank == 0) ptx::mbar_expect_tx(&kvfull[st], 2u * (Cfg::KH_BYTES + Cfg::VH_BYTES));
          const uint32_t fbar = ptx::mapa_shared(ptx::smem_u32(&kvfull[st]), 0);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)
            ptx::tma_load_2d_pair(sK + st * Cfg::KH_BYTES + kb * 8192, &kmap, fbar, kb * 64, row + 64 * (int)rank);
          ptx::tma_load_2d_pair(sV + st * Cfg::VH_BYTES, &vmap, fbar, 64 * (int)rank, row);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      jg += ti.nblk;
    }
  } else if (warp == 1) {
    if (rank == 1 && lane == 0) {
      // ---------------- CTA 1: tell CTA 0 when each of this CTA's query tiles landed ----------------
      const uint32_t qpeer_c0 = ptx::mapa_shared(ptx::smem_u32(qpeer), 0);
      for (int it = 0; it < my_tiles; ++it) {
        const int qb = kPersist ? (it & 1) : 0;
        if (!ptx::mbar_wait_sleep(&qfull[qb], (uint32_t)(it >> 1) & 1u)) break;
        ptx::mbar_arrive_cluster(qpeer_c0 + (uint32_t)(qb * 8));
      }
    }
    // ---------------- MMA issuer: one thread of CTA 0 for the pair ----------------
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_s = ptx::idesc_bf16(256, 128, false);
      const uint32_t idesc_o = ptx::idesc_bf16(256, D, true);
      const uint64_t q_d = ptx::sdesc_sw128(ptx::smem_u32(sQ), 16, 1024);
      const uint64_t k_d = ptx::sdesc_sw128(ptx::smem_u32(sK), 16, 1024);
      const uint64_t v_d = ptx::sdesc_sw128(ptx::smem_u32(sV), 16384, 1024);
      const uint32_t q_hi = (uint32_t)(q_d >> 32);
      const uint32_t k_lo = (uint32_t)k_d, k_hi = (uint32_t)(k_d >> 32);
      const uint32_t v_lo = (uint32_t)v_d, v_hi = (uint32_t)(v_d >> 32);
      // S of global block jj (local j) into buffer j % 2 (columns 128 * (j % 2)); its K and
      // V have landed in both CTAs (P.V later reads V from the same stage without another
      // wait)
      auto s_mmas = [&](int jj, int j, uint32_t q_lo) {
        const int st = jj % AT2_ST;
        const uint32_t b0 = k_lo + (uint32_t)(st * (Cfg::KH_BYTES >> 4));
        const uint32_t d = tmem + (uint32_t)((j & 1) * 128);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16_ss_pair(d, q_lo + (uint32_t)(kb * 1024 + k * 2), q_hi,
                                  b0 + (uint32_t)(kb * 512 + k * 2), k_hi, idesc_s, (kb | k) ? 1u : 0u);
      };
      auto kv_landed = [&](int jj) -> bool {
        return ptx::mbar_wait_cluster_sleep(&kvfull[jj % AT2_ST], (uint32_t)(jj / AT2_ST) & 1u);
      };
      bool ok = true;
      int jg = 0, use0 = 0, use1 = 0;      // blocks, and uses of each S buffer, of earlier tiles
      for (int it = 0; it < my_tiles && ok; ++it) {
        const At2Tile ti = tile_at(it);
        const int qb = kPersist ? (it & 1) : 0, nblk = ti.nblk;
        const uint32_t q_lo = (uint32_t)q_d + (uint32_t)(qb * (Cfg::Q_BYTES >> 4));
        ok = ptx::mbar_wait_sleep(&qfull[qb], (uint32_t)(it >> 1) & 1u) &&
             ptx::mbar_wait_cluster_sleep(&qpeer[qb], (uint32_t)(it >> 1) & 1u);
        for (int j = 0; j < 2 && j < nblk && ok; ++j) {
          ok = kv_landed(jg + j);
          if (!ok) break;
          ptx::tc_fence_after();
          s_mmas(jg + j, j, q_lo);
          ptx::tc_commit_pair(&sfull[j & 1], kBoth);
        }
        // Per block: every wait comes before the block's 16 MMAs, which are issued back to
        // back (a wait or commit between them lets the tensor pipe's short queue drain), and
        // both commits come after them.  The stage of block j is released once S(j+2) is
        // done, which also implies P.V(j) is.
        for (int j = 0; j < nblk && ok; ++j) {
          const int jj = jg + j;
          const int st = jj % AT2_ST;
          const bool more = j + 2 < nblk;
          if (more) ok = kv_landed(jj + 2);
          const uint32_t puse = (uint32_t)(((j & 1) ? use1 : use0) + (j >> 1));
          if (ok) ok = ptx::mbar_wait_cluster_sleep(&pready[j & 1], puse & 1u);
          if (!ok) break;
          ptx::tc_fence_after();
          // O_{j%2} += P(j) V(j); P(j) lies in buffer j % 2: keys 0-63 in columns 0-31, keys
          // 64-127 in columns 96-127
          const uint32_t b0 = v_lo + (uint32_t)(st * (Cfg::VH_BYTES >> 4));
          const uint32_t pa = tmem + (uint32_t)((j & 1) * 128);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            ptx::mma_bf16_ts_pair(tmem + 256u + (uint32_t)((j & 1) * 128), pa + (uint32_t)(k < 4 ? k * 8 : 96 + (k - 4) * 8),
                                  b0 + (uint32_t)(k * 128), v_hi, idesc_o, (j > 1 || k > 0) ? 1u : 0u);
          if (more) {
            s_mmas(jj + 2, j + 2, q_lo);
            ptx::tc_commit_pair(&sfull[j & 1], kBoth);
          }
          ptx::tc_commit_pair(&kvempty[st], kBoth);
        }
        if (!ok) break;
        if (kPersist) ptx::tc_commit_pair(&qempty[qb], kBoth);   // every MMA of the tile: its query buffer is free
        jg += nblk;
        use0 += (nblk + 1) / 2;
        use1 += nblk / 2;
      }
    }
  } else {
    // ---------------- softmax: warps 2-17 in two groups over even / odd key blocks ----------------
    const int grp = ((warp - 2) >> 3) & 1;                  // 0: even blocks, 1: odd blocks
    const int half = ((warp - 2) >> 2) & 1;                 // key half of each block
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                      // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    constexpr int DH = D / 2;
    const uint32_t o_addr = tmem + lane_off + 256u + (uint32_t)(grp * 128 + half * DH);
    const int bar_id = 1 + grp * 4 + quarter;
    const uint32_t pready_c0 = ptx::mapa_shared(ptx::smem_u32(pready), 0);   // CTA 0's pready[0]
    // the two halves of a row in a group post their values and each combines both; slots
    // alternate between two sets, so one barrier per exchange suffices
    int xphase = 0;
    auto exchange = [&](float v, bool is_max) -> float {
      float* slot = xbuf + ((xphase & 1) * 2 + grp) * 256 + r;
      slot[half * 128] = v;
      ptx::named_bar(bar_id, 64);
      const float a0 = slot[0], a1 = slot[128];
      ++xphase;
      return is_max ? fmaxf(a0, a1) : a0 + a1;
    };
    bool ok = true;
    int jg = 0, use = 0;                                    // blocks, and uses of this group's S buffer, of earlier tiles
    for (int it = 0; it < my_tiles; ++it) {
      const At2Tile ti = tile_at(it);
      const int nblk = ti.nblk, nsel = ti.nsel, nkeys = ti.nkeys, t0 = ti.t0;
      const int hl = r / p.TP;
      const int t = t0 + (int)rank * p.TP + r % p.TP;
      const bool row_valid = hl < p.G && t < p.C;
      const int tmin = t0 + (int)rank * p.TP;               // smallest position in this tile
      // membership words of this row and key half, block j at mrow_g[j * 4]
      const uint32_t* mrow_g = kMember ? mask + ((size_t)ti.tile * 256 + rank * 128 + r) * (size_t)mwords + half * 2
                                       : nullptr;
      uint2 mw_next = make_uint2(0u, 0u);
      if (kMember && grp < nblk) mw_next = *reinterpret_cast<const uint2*>(mrow_g + grp * 4);
      float m_run = -INFINITY, l_run = 0.f;
      int jlast = -1;
      // The two warps of a row quarter in a group take part in exactly one exchange per
      // block of the group and one at the end of each tile, whatever happens, so the named
      // barrier never waits for a warp that left: after a failed (timed-out) wait a warp
      // skips the work but keeps the exchanges.
      for (int j = grp; j < nblk; j += 2) {
        const int buf = grp;                                // == j % 2
        const int jj = jg + j;
        jlast = j;
        if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&sfull[buf], (uint32_t)(use + (j >> 1)) & 1u));
        if (!ok) {
          (void)exchange(0.f, true);
          continue;
        }
        ptx::tc_fence_after();
        const uint32_t s_addr = tmem + lane_off + (uint32_t)(buf * 128 + half * 64);
        const uint32_t p_addr = tmem + lane_off + (uint32_t)(buf * 128 + half * 96);
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          uint32_t u[32];
          ptx::tmem_ld32(s_addr + (uint32_t)c, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c + i] = __uint_as_float(u[i]);
        }
        ptx::tmem_ld_wait();
        if constexpr (kMember) {
          const uint2 mw = mw_next;                           // this block's words, loaded a block early
          if (j + 2 < nblk) mw_next = *reinterpret_cast<const uint2*>(mrow_g + (j + 2) * 4);
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const uint32_t wv = c < 32 ? mw.x : mw.y;
            if (!((wv >> (c & 31)) & 1u)) s[c] = -INFINITY;
          }
        } else {
          const int kb0 = j * 128 + half * 64;
          if (kb0 + 63 >= nsel + tmin || kb0 + 63 >= nkeys) {   // keys reach the causal part
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int kk = kb0 + c;
              const bool valid = kk < nkeys && (kk < nsel || kk - nsel <= t);
              if (!valid) s[c] = -INFINITY;
            }
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
        const bool grow = m_cand > m_run + AT2_RESCALE_LOG2 || (m_run == -INFINITY && m_cand > -INFINITY);
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
            pk[i] = pack_bf16x2(p0, p1);
          }
          ptx::tmem_st16(p_addr + (uint32_t)(c / 2), pk);
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        if (j >= 2 && __any_sync(0xffffffffu, grow)) {
          // rescale this group's O (blocks grp, grp + 2, ..., j - 2) once P.V(j-2) has
          // finished, i.e. its stage is released: S(j), which this warp has seen, was issued
          // after P.V(j-2), so the wait does not stall.  The parity wait is unambiguous: the
          // stage's next release needs this group's P of a later block of the tile, or a P
          // of the next tile, which neither group writes before this tile's epilogue
          ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&kvempty[(jj - 2) % AT2_ST], (uint32_t)((jj - 2) / AT2_ST) & 1u));
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
        // relaxed arrive: P and the rescaled O are TMEM stores already completed by
        // tcgen05.wait::st and ordered by the fence above; a cluster-scope release here
        // would stall the warp on its unrelated outstanding memory operations
        if (ok && lane == 0) ptx::mbar_arrive_cluster_relaxed(pready_c0 + (uint32_t)(buf * 8));
      }
      // epilogue: this group's O is final once its last P.V has released its stage (that
      // commit covers every earlier MMA); the two groups then meet per row quarter and each
      // thread writes 32 of the row's output columns from both groups' O:
      //   out = (O_0 f_0 + O_1 f_1) / (l_0 f_0 + l_1 f_1),   f_g = 2^(m_g - max(m_0, m_1))
      if (ok && jlast >= 0)
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&kvempty[(jg + jlast) % AT2_ST], (uint32_t)((jg + jlast) / AT2_ST) & 1u));
      const float l_grp = exchange(ok ? l_run : 0.f, false);   // every pair member reaches this
      float* ml = xbuf + 2 * 2 * 2 * 128;                      // [m, l][group][row]
      if (half == 0) {
        ml[grp * 128 + r] = m_run;
        ml[256 + grp * 128 + r] = ok ? l_grp : 0.f;
      }
      ptx::named_bar(9 + quarter, 128);                         // both groups of this row quarter
      const float m0 = ml[r], m1 = ml[128 + r], l0 = ml[256 + r], l1 = ml[384 + r];
      if (ok) {
        ptx::tc_fence_after();
        const float mm = fmaxf(m0, m1);
        const float f0 = l0 > 0.f ? ptx::ex2_approx(m0 - mm) : 0.f;
        const float f1 = l1 > 0.f ? ptx::ex2_approx(m1 - mm) : 0.f;
        const float l = l0 * f0 + l1 * f1;
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const float g0 = f0 * inv_l, g1 = f1 * inv_l;
        const int c0 = (grp * 2 + half) * 32;                   // this thread's output columns
          const At2Tile te = tile_at(it);                         // (b, g) again, not kept live over the blocks
        __nv_bfloat16* orow = out + ((size_t)(te.b * p.h_q + te.g * p.G + (row_valid ? hl : 0)) * p.C +
                                     (row_valid ? t : 0)) * D + c0;
        const uint32_t oa = tmem + lane_off + 256u + (uint32_t)c0;
#pragma unroll
        for (int c = 0; c < 32; c += 16) {
          uint32_t u0[16], u1[16];
          ptx::tmem_ld16(oa + (uint32_t)c, u0);
          ptx::tmem_ld16(oa + 128u + (uint32_t)c, u1);
          ptx::tmem_ld_wait();
          float o[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            o[i] = (g0 > 0.f ? __uint_as_float(u0[i]) * g0 : 0.f) + (g1 > 0.f ? __uint_as_float(u1[i]) * g1 : 0.f);
          uint4 w0, w1;
          w0.x = pack_bf16x2(o[0], o[1]);   w0.y = pack_bf16x2(o[2], o[3]);
          w0.z = pack_bf16x2(o[4], o[5]);   w0.w = pack_bf16x2(o[6], o[7]);
          w1.x = pack_bf16x2(o[8], o[9]);   w1.y = pack_bf16x2(o[10], o[11]);
          w1.z = pack_bf16x2(o[12], o[13]); w1.w = pack_bf16x2(o[14], o[15]);
          if (row_valid) {
            reinterpret_cast<uint4*>(orow + c)[0] = w0;
            reinterpret_cast<uint4*>(orow + c)[1] = w1;
          }
        }
        ptx::tc_fence_before();
      }
      // both groups of the quarter have read O (and the (m, l) slots) before either one's
      // next P lets the next tile's first P.V overwrite its O
      if (kPersist) ptx::named_bar(9 + quarter, 128);
      jg += nblk;
      use += (nblk - grp + 1) / 2;
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
