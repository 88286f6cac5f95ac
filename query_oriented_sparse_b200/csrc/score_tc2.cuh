// K2 over SM pairs (tensor-core form, bf16, kept queries per head dividing 128): cosine
// scoring of every prefix key against the kept queries with group-aware pooling (QUOKA
// page, method summary: cosine similarity scoring, max pooling over queries, mean
// pooling over the query heads of a GQA group; the selection sweep reads the whole
// prefix once).
//
// A cluster of two CTAs on two SMs takes a contiguous run of work units (sequence, KV
// head, column group, 256-key pair tile); CTA r owns keys 128r .. 128r+127 of each pair
// tile.  Every MMA is one tcgen05.mma.cta_group::2 issued by one thread of CTA 0:
//   S = K_pairtile . Qsel^T   (M 256 keys, N <= 128 kept-query columns, K d)
// A = each CTA's own 128-key tile, B = the slice's kept-query columns split by columns
// (CTA r holds the second half when r = 1), D = 128 keys x N columns in each CTA's
// TMEM.  So each SM reads its own key tile and half of every query slice per MMA
// (96 B/clk of operands at N = 128 instead of 128), and its TMEM holds four 128-column
// accumulators: the column group is cut into slices of 128 columns (whole heads), and
// slice n of the run goes to buffer n % 4 and to epilogue group n % 4.  The tensor pipe
// therefore runs the next slices while earlier ones drain.
//
// Roles per CTA: warp 0 loads (the key tiles by tiled TMA into a ring of 16 KB
// K-block stages, the CTA's half of the column group's kept queries by tiled TMA, and
// the columns' 1/|q| and padding bias by bulk copy); warp 1 issues the pair's MMAs in
// CTA 0 and, in CTA 1, forwards "my tile landed" to CTA 0; warps 2-17 are four epilogue
// groups of four warps (one per TMEM lane quarter).  The group that drains a slice
// takes, for each of its 128 keys, the sum over the slice's heads of the max over the
// head's kept queries of s / |q| (+ bias), plus its share of |k|^2 from the key tile in
// shared memory; the tile's merging group (rotating) adds the slices' partials in slice
// order one tile later and writes score = (sum / G) / |k|.  The score matrix never
// reaches HBM.  Every wait is a bounded mbarrier wait; the only other synchronisation is
// the two cluster barriers, which every thread of both CTAs reaches on every path.
#pragma once
#include <cooperative_groups.h>
#include "tc_ptx.cuh"
#include "score_tc.cuh"

namespace quoka {

constexpr int ST2_PT = 256;          // keys per pair tile (128 per CTA = TMEM lanes)
constexpr int ST2_SLICE = 128;       // MMA N (columns) per accumulator slice
constexpr int ST2_NBUF = 4;          // accumulator slices held in TMEM
constexpr int ST2_MAXCOLS = 512;     // kept-query columns per column group
constexpr int ST2_THREADS = 576;     // warp 0 loads, warp 1 MMA / forwarder, warps 2-17 epilogue
constexpr int ST2_EPI_WARPS = 16;
constexpr int ST2_QBOX = 8;          // rows per TMA box of the kept-query block

template <int D>
struct St2Cfg {
  static constexpr int KB = D / 64;                        // 128-byte K-blocks per row
  static constexpr int STAGE_BYTES = 128 * 128;            // one K-block of this CTA's key tile
  static constexpr int NST = 8;                            // stages in the key ring
  // this CTA's half of every slice: slice s at rows 64 s .. 64 s + N_s / 2 - 1
  static constexpr int QBLK_BYTES = (ST2_MAXCOLS / 2) * 128;
  static constexpr int Q_BYTES = QBLK_BYTES * KB;
  static constexpr int K_BYTES = STAGE_BYTES * NST;
  static constexpr int CP_BYTES = 2 * ST2_MAXCOLS * 4;     // 1/|q| and bias per column
  static constexpr int MERGE_BYTES = 2 * ST2_NBUF * 128 * 8;   // two slots of (sum, |k|^2) per slice
  // kfull, kempty, kpeer [NST]; qfull, qempty, qpeer; accfull, accempty [NBUF]; mfull, mempty [2]
  static constexpr int NBAR = 3 * NST + 3 + 2 * ST2_NBUF + 4;
  static constexpr int SMEM = 1024 + Q_BYTES + K_BYTES + CP_BYTES + MERGE_BYTES + NBAR * 8 + 16;
};

__device__ __forceinline__ void st2_decode(const ScoreTcParams& p, const SeqTable& tab, int u,
                                           int& b, int& g, int& cg, int& pt) {
  b = 0;
  while (b + 1 < tab.batch && p.unit_base[b + 1] <= u) ++b;
  const int rem = u - p.unit_base[b];
  const int tiles = (tab.prefix[b] + ST2_PT - 1) / ST2_PT;
  const int gc = rem / tiles;
  pt = rem - gc * tiles;
  g = gc / p.ncg;
  cg = gc - g * p.ncg;
}

// The unit after (b, g, cg, pt), stepping a cursor instead of decoding from scratch.
__device__ __forceinline__ void st2_next(const ScoreTcParams& p, const SeqTable& tab, int& b,
                                         int& g, int& cg, int& pt, int& tiles) {
  if (++pt < tiles) return;
  pt = 0;
  if (++cg < p.ncg) return;
  cg = 0;
  if (++g < p.h_kv) return;
  g = 0;
  do {                                         // sequences without prefix keys own no units
    ++b;
    tiles = b < tab.batch ? (tab.prefix[b] + ST2_PT - 1) / ST2_PT : 1;
  } while (tiles == 0);
}

// Columns of a column group, and its slices of at most 128 columns (whole heads, since
// the kept queries per head divide 128).
__device__ __forceinline__ int st2_ncols(const ScoreTcParams& p, int cg) {
  const int h0 = cg * p.heads_per_cg;
  return (min(p.G, h0 + p.heads_per_cg) - h0) * p.nkp;
}

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(ST2_THREADS, 1)
score_tc2_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                 const __grid_constant__ SeqTable tab, const __grid_constant__ ScoreTcParams p,
                 const float* __restrict__ qinv, const float* __restrict__ qbias,
                 float* __restrict__ pooled) {
  using Cfg = St2Cfg<D>;
  constexpr int KB = Cfg::KB, NST = Cfg::NST;
  namespace cgrp = cooperative_groups;
  cgrp::cluster_group cluster = cgrp::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::Q_BYTES;
  float* cpi = reinterpret_cast<float*>(sK + Cfg::K_BYTES);     // 1/|q| per column
  float* cpb = cpi + ST2_MAXCOLS;                                 // bias per column
  float2* mslot = reinterpret_cast<float2*>(cpi + 2 * ST2_MAXCOLS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(mslot) + Cfg::MERGE_BYTES);
  uint64_t* kfull = bars;                  // this CTA's K-block landed (local TMA)
  uint64_t* kempty = kfull + NST;          // MMA commit (both CTAs) + this CTA's 16 epilogue warps
  uint64_t* kpeer = kempty + NST;          // (CTA 0) CTA 1's K-block landed
  uint64_t* qfull = kpeer + NST;           // this CTA's query half and the column data landed
  uint64_t* qempty = qfull + 1;            // MMA commit + this CTA's 16 epilogue warps
  uint64_t* qpeer = qfull + 2;             // (CTA 0) CTA 1's query half landed
  uint64_t* accfull = qfull + 3;           // [NBUF] slice's MMAs done (both CTAs)
  uint64_t* accempty = accfull + ST2_NBUF; // [NBUF] (CTA 0) slice drained by both CTAs' groups
  uint64_t* mfull = accempty + ST2_NBUF;   // [2] a tile's slice partials written
  uint64_t* mempty = mfull + 2;            // [2] merged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster.block_rank();
  const long long per = (long long)p.total_units;
  const int nclu = (int)(gridDim.x >> 1), clu = (int)(blockIdx.x >> 1);
  const int u_lo = (int)(per * clu / nclu);
  const int u_hi = (int)(per * (clu + 1) / nclu);
  constexpr uint16_t kBoth = 0x3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      ptx::mbar_init(&kfull[s], 1);
      ptx::mbar_init(&kempty[s], 1 + ST2_EPI_WARPS);
      ptx::mbar_init(&kpeer[s], 1);
    }
    ptx::mbar_init(qfull, 1);
    ptx::mbar_init(qempty, 1 + ST2_EPI_WARPS);
    ptx::mbar_init(qpeer, 1);
    for (int i = 0; i < ST2_NBUF; ++i) {
      ptx::mbar_init(&accfull[i], 1);
      ptx::mbar_init(&accempty[i], 8);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&mfull[i], ST2_NBUF * 128);
      ptx::mbar_init(&mempty[i], 128);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, ST2_NBUF * ST2_SLICE);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  cluster.sync();                          // barriers and TMEM of both CTAs ready
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- loads ----------------
    if (lane == 0 && u_lo < u_hi) {
      ptx::prefetch_tmap(&kmap);
      ptx::prefetch_tmap(&qmap);
      int stage = 0, cur = -1;
      uint32_t kph = 0, qeph = 0;
      bool ok = true;
      int b, g, cg, pt, tiles;
      st2_decode(p, tab, u_lo, b, g, cg, pt);
      tiles = (tab.prefix[b] + ST2_PT - 1) / ST2_PT;
      for (int u = u_lo; u < u_hi && ok; ++u) {
        if (u != u_lo) st2_next(p, tab, b, g, cg, pt, tiles);
        const int key3 = (b * p.h_kv + g) * p.ncg + cg;
        if (key3 != cur) {
          if (cur >= 0) {
            ok = ptx::mbar_wait_sleep(qempty, qeph);
            qeph ^= 1u;
            if (!ok) break;
          }
          const int ncols = st2_ncols(p, cg);
          const int nsl = (ncols + ST2_SLICE - 1) / ST2_SLICE;
          const int qrow0 = (b * p.h_kv + g) * p.G * p.nkp + cg * p.heads_per_cg * p.nkp;
          uint32_t bytes = 2u * (uint32_t)ncols * 4u;
          for (int s = 0; s < nsl; ++s)
            bytes += (uint32_t)(min(ST2_SLICE, ncols - s * ST2_SLICE) / 2) * D * 2;
          ptx::mbar_expect_tx(qfull, bytes);
          for (int s = 0; s < nsl; ++s) {
            const int half = min(ST2_SLICE, ncols - s * ST2_SLICE) / 2;
            const int grow = qrow0 + s * ST2_SLICE + (int)rank * half;
            for (int kb = 0; kb < KB; ++kb)
              for (int r = 0; r < half; r += ST2_QBOX)
                ptx::tma_load_2d(sQ + kb * Cfg::QBLK_BYTES + (s * 64 + r) * 128, &qmap, qfull, kb * 64, grow + r);
          }
          ptx::bulk_load(cpi, qinv + qrow0, (uint32_t)ncols * 4u, qfull);
          ptx::bulk_load(cpb, qbias + qrow0, (uint32_t)ncols * 4u, qfull);
          cur = key3;
        }
        const int krow = (int)(g * p.rows_per_head + tab.kv_off[b]) + pt * ST2_PT + (int)rank * 128;
        for (int kb = 0; kb < KB && ok; ++kb) {
          ok = ptx::mbar_wait_sleep(&kempty[stage], kph ^ 1u);
          if (!ok) break;
          ptx::mbar_expect_tx(&kfull[stage], Cfg::STAGE_BYTES);
          ptx::tma_load_2d(sK + stage * Cfg::STAGE_BYTES, &kmap, &kfull[stage], kb * 64, krow);
          if (++stage == NST) { stage = 0; kph ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 1) {
      // ---------------- CTA 1: forward "landed" to CTA 0, in load order ----------------
      if (lane == 0 && u_lo < u_hi) {
        const uint32_t qpeer_c0 = ptx::mapa_shared(ptx::smem_u32(qpeer), 0);
        const uint32_t kpeer_c0 = ptx::mapa_shared(ptx::smem_u32(kpeer), 0);
        int stage = 0, cur = -1;
        uint32_t kph = 0, qph = 0;
        bool ok = true;
        int b, g, cg, pt, tiles;
        st2_decode(p, tab, u_lo, b, g, cg, pt);
        tiles = (tab.prefix[b] + ST2_PT - 1) / ST2_PT;
        for (int u = u_lo; u < u_hi && ok; ++u) {
          if (u != u_lo) st2_next(p, tab, b, g, cg, pt, tiles);
          const int key3 = (b * p.h_kv + g) * p.ncg + cg;
          if (key3 != cur) {
            ok = ptx::mbar_wait_sleep(qfull, qph);
            qph ^= 1u;
            if (!ok) break;
            ptx::mbar_arrive_cluster(qpeer_c0);
            cur = key3;
          }
          for (int kb = 0; kb < KB && ok; ++kb) {
            ok = ptx::mbar_wait_sleep(&kfull[stage], kph);
            if (!ok) break;
            ptx::mbar_arrive_cluster(kpeer_c0 + (uint32_t)(stage * 8));
            if (++stage == NST) { stage = 0; kph ^= 1u; }
          }
        }
      }
    } else if (lane == 0 && u_lo < u_hi) {
      // ---------------- CTA 0: MMA issuer for the pair ----------------
      int stage = 0, cur = -1, ncols = 0, nsl = 0;
      uint32_t n = 0;                          // slice counter of the run
      uint32_t kph = 0, qph = 0;
      bool ok = true;
      int b, g, cg, pt, tiles;
      st2_decode(p, tab, u_lo, b, g, cg, pt);
      tiles = (tab.prefix[b] + ST2_PT - 1) / ST2_PT;
      for (int u = u_lo; u < u_hi && ok; ++u) {
        if (u != u_lo) st2_next(p, tab, b, g, cg, pt, tiles);
        const int key3 = (b * p.h_kv + g) * p.ncg + cg;
        if (key3 != cur) {
          if (cur >= 0) ptx::tc_commit_pair(qempty, kBoth);
          ok = ptx::mbar_wait_sleep(qfull, qph) && ptx::mbar_wait_cluster_sleep(qpeer, qph);
          qph ^= 1u;
          if (!ok) break;
          ncols = st2_ncols(p, cg);
          nsl = (ncols + ST2_SLICE - 1) / ST2_SLICE;
          cur = key3;
        }
        int st[KB];
        for (int kb = 0; kb < KB; ++kb) {
          st[kb] = stage;
          if (ok) ok = ptx::mbar_wait_sleep(&kfull[stage], kph) && ptx::mbar_wait_cluster_sleep(&kpeer[stage], kph);
          if (++stage == NST) { stage = 0; kph ^= 1u; }
        }
        if (!ok) break;
        for (int s = 0; s < nsl && ok; ++s, ++n) {
          const int buf = (int)(n & 3u);
          ok = ptx::mbar_wait_cluster_sleep(&accempty[buf], ((n >> 2) & 1u) ^ 1u);
          if (!ok) break;
          ptx::tc_fence_after();
          const int w = min(ST2_SLICE, ncols - s * ST2_SLICE);
          const uint32_t idesc = ptx::idesc_bf16(256, w, false);
          const uint32_t d_tmem = tmem + (uint32_t)(buf * ST2_SLICE);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = ptx::sdesc_sw128(ptx::smem_u32(sK + st[kb] * Cfg::STAGE_BYTES), 16, 1024);
            const uint64_t bd = ptx::sdesc_sw128(ptx::smem_u32(sQ + kb * Cfg::QBLK_BYTES + s * 64 * 128), 16, 1024);
            const uint32_t a_lo = (uint32_t)ad, a_hi = (uint32_t)(ad >> 32);
            const uint32_t b_lo = (uint32_t)bd, b_hi = (uint32_t)(bd >> 32);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              ptx::mma_bf16_ss_pair(d_tmem, a_lo + (uint32_t)(ks * 2), a_hi, b_lo + (uint32_t)(ks * 2), b_hi,
                                    idesc, (kb | ks) ? 1u : 0u);
          }
          ptx::tc_commit_pair(&accfull[buf], kBoth);
        }
        for (int kb = 0; kb < KB; ++kb) ptx::tc_commit_pair(&kempty[st[kb]], kBoth);
      }
    }
  } else {
    // ---------------- epilogue: four groups of four warps, one key per thread ----------
    const int e = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t accempty_c0 = ptx::mapa_shared(ptx::smem_u32(accempty), 0);
    constexpr int NCH = D / 8;                   // 16-byte chunks (8 bf16) per key row
    int stage = 0, cur = -1, ncols = 0, nsl = 0, nt = 0;
    uint32_t n = 0, kph = 0, qph = 0;
    bool ok = u_lo < u_hi;
    int b = 0, g = 0, cg = 0, pt = 0, tiles = 1;
    if (ok) {
      st2_decode(p, tab, u_lo, b, g, cg, pt);
      tiles = (tab.prefix[b] + ST2_PT - 1) / ST2_PT;
    }
    int pb = 0, pg = 0, pcg = 0, ppt = 0, pnsl = 0;
    auto merge_tile = [&](int m, int mb, int mg, int mcg, int mpt, int mnsl) -> bool {
      const int slot = m & 1;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_sleep(&mfull[slot], (uint32_t)(m >> 1) & 1u))) return false;
      float2 o[ST2_NBUF];
#pragma unroll
      for (int s = 0; s < ST2_NBUF; ++s)
        o[s] = s < mnsl ? mslot[(slot * ST2_NBUF + s) * 128 + row] : make_float2(0.f, 0.f);
      ptx::mbar_arrive(&mempty[slot]);
      const float msum = ((o[0].x + o[1].x) + o[2].x) + o[3].x;   // slice order
      const float mss = ((o[0].y + o[1].y) + o[2].y) + o[3].y;
      const float knorm = sqrtf(mss);
      const int j = mpt * ST2_PT + (int)rank * 128 + row;
      if (j < tab.prefix[mb]) {
        const float sc = knorm > 0.f ? (p.ncg == 1 ? msum * p.inv_G : msum) / knorm : 0.f;
        pooled[mcg * p.cg_stride + (size_t)(mb * p.h_kv + mg) * p.pooled_stride + j] = sc;
      }
      return true;
    };
    // sum over the heads in [cbase, cbase + ncol) of max over the head's columns of
    // s / |q| (+ bias); columns come 32 (or, at the end of a 16-wide head, 16) at a time
    auto head_max = [&](uint32_t tcol, int cbase, int ncol) -> float {
      const float* ci = cpi + cbase;
      const float* cb = cpb + cbase;
      float run = -INFINITY;
      for (int c = 0; c < ncol; c += 32) {
        const int w = min(32, ncol - c);
        uint32_t r[32];
        if (w == 32) ptx::tmem_ld32(lane_base + tcol + (uint32_t)c, r);
        else ptx::tmem_ld16(lane_base + tcol + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(r));
        ptx::tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q * 16 < w) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 sc = reinterpret_cast<const float4*>(ci + c + q * 16)[i];
              const uint32_t* rr = &r[q * 16 + 4 * i];
              const float2 s01 = make_float2(__uint_as_float(rr[0]), __uint_as_float(rr[1]));
              const float2 s23 = make_float2(__uint_as_float(rr[2]), __uint_as_float(rr[3]));
              float2 v01, v23;
              if (p.padded) {
                const float4 bi = reinterpret_cast<const float4*>(cb + c + q * 16)[i];
                v01 = ptx::fma2(s01, make_float2(sc.x, sc.y), make_float2(bi.x, bi.y));
                v23 = ptx::fma2(s23, make_float2(sc.z, sc.w), make_float2(bi.z, bi.w));
              } else {
                v01 = ptx::mul2(s01, make_float2(sc.x, sc.y));
                v23 = ptx::mul2(s23, make_float2(sc.z, sc.w));
              }
              v[4 * i] = v01.x; v[4 * i + 1] = v01.y; v[4 * i + 2] = v23.x; v[4 * i + 3] = v23.y;
            }
            const float a0 = ptx::max3(v[0], v[1], v[2]), a1 = ptx::max3(v[3], v[4], v[5]);
            const float a2 = ptx::max3(v[6], v[7], v[8]), a3 = ptx::max3(v[9], v[10], v[11]);
            const float a4 = ptx::max3(v[12], v[13], v[14]);
            run = ptx::max3(run, ptx::max3(a0, a1, a2), ptx::max3(a3, a4, v[15]));
          }
        }
      }
      return run;
    };
    for (int u = u_lo; u < u_hi && ok; ++u) {
      if (u != u_lo) st2_next(p, tab, b, g, cg, pt, tiles);
      const int key3 = (b * p.h_kv + g) * p.ncg + cg;
      if (key3 != cur) {
        // done with the previous column group's 1/|q| and bias; wait for this one's
        if (cur >= 0 && lane == 0) ptx::mbar_arrive(qempty);
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(qfull, qph));
        qph ^= 1u;
        if (!ok) break;
        ncols = st2_ncols(p, cg);
        nsl = (ncols + ST2_SLICE - 1) / ST2_SLICE;
        cur = key3;
      }
      // this group's slice of the tile, if any (at most one: nsl <= 4)
      const int s = (int)((uint32_t)e - n) & 3;
      const bool mine = s < nsl;
      int st[KB];
      uint32_t sph[KB];
      for (int kb = 0; kb < KB; ++kb) {
        st[kb] = stage;
        sph[kb] = kph;
        if (++stage == NST) { stage = 0; kph ^= 1u; }
      }
      // Every K-block of the tile has landed before this warp releases it (a release of a
      // slot never waited for could count toward the slot's previous use); the slice's
      // group adds its share of |k|^2 from the swizzled tile.
      for (int kb = 0; kb < KB; ++kb)
        if (ok) ok = ptx::mbar_wait_sleep(&kfull[st[kb]], sph[kb]);
      float ss = 0.f;
      if (ok && mine) {
        const int c_lo = s * NCH / nsl, c_hi = (s + 1) * NCH / nsl;
        for (int c = c_lo; c < c_hi; ++c) {
          const uint8_t* rp = sK + st[c >> 3] * Cfg::STAGE_BYTES + row * 128;
          const uint4 v = *reinterpret_cast<const uint4*>(rp + (((c & 7) ^ (row & 7)) << 4));
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = bf16_lo(wv[i]), hi = bf16_hi(wv[i]);
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
          }
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0)
        for (int kb = 0; kb < KB; ++kb) ptx::mbar_arrive(&kempty[st[kb]]);
      if (!ok) break;

      if (mine) {
        const uint32_t ns = n + (uint32_t)s;
        const int buf = (int)(ns & 3u);
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&accfull[buf], (ns >> 2) & 1u));
        if (!ok) break;
        ptx::tc_fence_after();
        const int c0 = s * ST2_SLICE;
        const int w = min(ST2_SLICE, ncols - c0);
        float sum = 0.f;
        for (int h = 0; h < w; h += p.nkp)
          sum += head_max((uint32_t)(buf * ST2_SLICE + h), c0 + h, p.nkp);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster_relaxed(accempty_c0 + (uint32_t)(buf * 8));
        // hand the partial over; the tile's last slice also arrives for missing slices
        const int slot = nt & 1;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&mempty[slot], ((uint32_t)(nt >> 1) & 1u) ^ 1u));
        if (!ok) break;
        mslot[(slot * ST2_NBUF + s) * 128 + row] = make_float2(sum, ss);
        ptx::mbar_arrive_count(&mfull[slot], s == nsl - 1 ? 1u + (uint32_t)(ST2_NBUF - nsl) : 1u);
      }
      // merge the previous tile, whose partials are all in or on their way
      if (nt > 0 && e == ((nt - 1) & 3)) {
        ok = merge_tile(nt - 1, pb, pg, pcg, ppt, pnsl);
        if (!ok) break;
      }
      pb = b; pg = g; pcg = cg; ppt = pt; pnsl = nsl;
      n += (uint32_t)nsl;
      ++nt;
    }
    if (ok && nt > 0 && e == ((nt - 1) & 3)) merge_tile(nt - 1, pb, pg, pcg, ppt, pnsl);
  }

  ptx::tc_fence_before();
  cluster.sync();                          // the pair's MMAs and loads are over on both SMs
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, ST2_NBUF * ST2_SLICE);
  }
}

}  // namespace quoka
