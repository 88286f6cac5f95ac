// K2 (tensor-core form, bf16): cosine scoring of every prefix key against the kept
// queries with group-aware pooling (QUOKA page, method summary: cosine similarity
// scoring, max pooling over queries, mean pooling over the query heads of a GQA
// group; the selection sweep reads the whole prefix once).
//
// S = K_tile . Qsel^T runs on tcgen05 with raw bf16 operands and fp32 accumulation in
// TMEM (keys on the 128 TMEM lanes, kept-query columns along TMEM columns); 1/|q| and
// the pooling are applied in the epilogue in fp32, and |k| is taken from the key tile
// already in shared memory, so the score matrix never reaches HBM and the only HBM
// traffic is one read of the prefix keys.
//
// Persistent CTAs each take a contiguous run of work units (sequence, KV head, column
// group, 128-key tile).  A column group is up to 2 x 256 kept-query columns (whole
// heads); its operand block stays resident in shared memory while key tiles stream
// through a ring of 16 KB K-block stages loaded by TMA (128-byte swizzle).  Warp 0
// issues TMA, one thread of warp 1 issues the MMAs of each tile as one or two column
// slices (cut on head boundaries) into two 256-column TMEM accumulators, and sixteen
// epilogue warps in four groups drain them: group e takes the heads h with h % 4 == e
// and a quarter of |k|^2.  After a tile every group hands (sum of its head maxima, |k|^2
// share) to the tile's merging group (rotating over the tiles) through a shared-memory
// slot guarded by an mbarrier pair; the merge runs one tile late, so no group waits for
// the slowest one.  Waiting threads sleep on their mbarrier instead of spinning.
#pragma once
#include "tc_ptx.cuh"

namespace quoka {

constexpr int STC_BM = 128;        // keys per tile (TMEM lanes)
constexpr int STC_MAXCOLS = 512;   // kept-query columns per column group
constexpr int STC_SLICE = 256;     // max MMA N per accumulator slice
constexpr int STC_NBUF = 2;        // accumulator slices held in TMEM
constexpr int STC_THREADS = 576;   // warp 0 TMA, warp 1 MMA, warps 2-17 epilogue (4 groups)
constexpr int STC_EPI_WARPS = 16;
constexpr int STC_QBOX = 16;       // rows per TMA box of the kept-query block

struct ScoreTcParams {
  int h_kv, G, nkp, ncg, heads_per_cg;
  int padded;                   // nonzero when heads carry padding columns (bias needed)
  int total_units;
  long long rows_per_head;
  long long pooled_stride;      // floats per (sequence, KV head) row
  long long cg_stride;          // floats between column-group partial-score arrays
  float inv_G;
  int unit_base[QUOKA_MAX_BATCH + 1];
};

template <int D>
struct StcCfg {
  static constexpr int KB = D / 64;                    // 128-byte K-blocks per row
  static constexpr int STAGE_BYTES = STC_BM * 128;     // one K-block of one key tile
  static constexpr int NST = (D == 128) ? 5 : 8;       // stages in the key ring
  static constexpr int QBLK_BYTES = STC_MAXCOLS * 128; // one K-block of the query block
  static constexpr int Q_BYTES = QBLK_BYTES * KB;
  static constexpr int K_BYTES = STAGE_BYTES * NST;
  // 1/|q| and bias per column; twice the columns so the masked tail of a 64-column
  // batch past a slice end still reads inside the arrays
  static constexpr int CP_BYTES = 2 * STC_MAXCOLS * 8;
  static constexpr int NBAR = 2 * NST + 2 + 2 * STC_NBUF + 4;
  // two slots of (partial sum, |k|^2 share) per epilogue group
  static constexpr int MERGE_BYTES = 2 * 4 * STC_BM * 8;
  static constexpr int SMEM = 1024 + Q_BYTES + K_BYTES + CP_BYTES + MERGE_BYTES + NBAR * 8 + 16;
};

__device__ __forceinline__ void stc_decode(const ScoreTcParams& p, const SeqTable& tab, int u,
                                           int& b, int& g, int& cg, int& tile) {
  b = 0;
  while (b + 1 < tab.batch && p.unit_base[b + 1] <= u) ++b;
  const int rem = u - p.unit_base[b];
  const int tiles = (tab.prefix[b] + STC_BM - 1) / STC_BM;
  const int gc = rem / tiles;
  tile = rem - gc * tiles;
  g = gc / p.ncg;
  cg = gc - g * p.ncg;
}

// The unit after (b, g, cg, tile): a CTA walks a contiguous run of units, so after one
// stc_decode it steps without divisions or indexed reads of the sequence table.
__device__ __forceinline__ void stc_next(const ScoreTcParams& p, const SeqTable& tab, int& b,
                                         int& g, int& cg, int& tile, int& tiles) {
  if (++tile < tiles) return;
  tile = 0;
  if (++cg < p.ncg) return;
  cg = 0;
  if (++g < p.h_kv) return;
  g = 0;
  do {                                         // sequences without prefix keys own no units
    ++b;
    tiles = b < tab.batch ? (tab.prefix[b] + STC_BM - 1) / STC_BM : 1;
  } while (tiles == 0);
}

template <int D>
__global__ void __launch_bounds__(STC_THREADS, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                const __grid_constant__ SeqTable tab, const __grid_constant__ ScoreTcParams p,
                const float* __restrict__ qinv, const float* __restrict__ qbias,
                float* __restrict__ pooled) {
  using Cfg = StcCfg<D>;
  constexpr int KB = Cfg::KB, NST = Cfg::NST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::Q_BYTES;
  float* cpi = reinterpret_cast<float*>(sK + Cfg::K_BYTES);     // 1/|q| per column
  float* cpb = cpi + 2 * STC_MAXCOLS;                             // bias per column
  float* merge = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(cpi) + Cfg::CP_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(merge) + Cfg::MERGE_BYTES);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + NST;
  uint64_t* qfull = bars + 2 * NST;
  uint64_t* qempty = qfull + 1;
  uint64_t* accfull = qfull + 2;
  uint64_t* accempty = accfull + STC_NBUF;
  uint64_t* mfull = accempty + STC_NBUF;   // [2] partials of all four groups written
  uint64_t* mempty = mfull + 2;            // [2] slot consumed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long per = (long long)p.total_units;
  const int u_lo = (int)(per * blockIdx.x / gridDim.x);
  const int u_hi = (int)(per * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      ptx::mbar_init(&kfull[s], 1);
      ptx::mbar_init(&kempty[s], 1 + STC_EPI_WARPS);
    }
    ptx::mbar_init(qfull, 1);
    ptx::mbar_init(qempty, 1);
    for (int s = 0; s < STC_NBUF; ++s) {
      ptx::mbar_init(&accfull[s], 1);
      ptx::mbar_init(&accempty[s], STC_EPI_WARPS);
      ptx::mbar_init(&mfull[s], 4 * STC_BM);
      ptx::mbar_init(&mempty[s], STC_BM);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, STC_NBUF * STC_SLICE);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&kmap);
      ptx::prefetch_tmap(&qmap);
      int stage = 0, cur = -1;
      uint32_t kph = 0, qeph = 0;
      bool ok = true;
      int b, g, cg, tile, tiles;
      stc_decode(p, tab, u_lo, b, g, cg, tile);
      tiles = (tab.prefix[b] + STC_BM - 1) / STC_BM;
      for (int u = u_lo; u < u_hi && ok; ++u) {
        if (u != u_lo) stc_next(p, tab, b, g, cg, tile, tiles);
        const int key3 = (b * p.h_kv + g) * p.ncg + cg;
        if (key3 != cur) {
          if (cur >= 0) {
            ok = ptx::mbar_wait_sleep(qempty, qeph);
            qeph ^= 1u;
            if (!ok) break;
          }
          const int h0 = cg * p.heads_per_cg;
          const int nh = min(p.G, h0 + p.heads_per_cg) - h0;
          const int ncols = nh * p.nkp;
          const int qrow0 = (b * p.h_kv + g) * p.G * p.nkp + h0 * p.nkp;
          ptx::mbar_expect_tx(qfull, (uint32_t)(ncols * D * 2));
          for (int kb = 0; kb < KB; ++kb)
            for (int r = 0; r < ncols; r += STC_QBOX)
              ptx::tma_load_2d(sQ + kb * Cfg::QBLK_BYTES + r * 128, &qmap, qfull, kb * 64, qrow0 + r);
          cur = key3;
        }
        const int krow = (int)(g * p.rows_per_head + tab.kv_off[b]) + tile * STC_BM;
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
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0, cur = -1, nsl_done = 0, ncols = 0;
      uint32_t kph = 0, qph = 0;
      bool ok = true;
      int b, g, cg, tile, tiles;
      stc_decode(p, tab, u_lo, b, g, cg, tile);
      tiles = (tab.prefix[b] + STC_BM - 1) / STC_BM;
      for (int u = u_lo; u < u_hi && ok; ++u) {
        if (u != u_lo) stc_next(p, tab, b, g, cg, tile, tiles);
        const int key3 = (b * p.h_kv + g) * p.ncg + cg;
        if (key3 != cur) {
          if (cur >= 0) ptx::tc_commit(qempty);
          ok = ptx::mbar_wait_sleep(qfull, qph);
          qph ^= 1u;
          if (!ok) break;
          const int h0 = cg * p.heads_per_cg;
          ncols = (min(p.G, h0 + p.heads_per_cg) - h0) * p.nkp;
          cur = key3;
        }
        int st[KB];
        for (int kb = 0; kb < KB; ++kb) {
          st[kb] = stage;
          if (ok) ok = ptx::mbar_wait_sleep(&kfull[stage], kph);
          if (++stage == NST) { stage = 0; kph ^= 1u; }
        }
        if (!ok) break;
        ptx::tc_fence_after();
        const int nsl = ncols > STC_SLICE ? 2 : 1;
        const int cols0 = nsl == 2 ? ((ncols / p.nkp + 1) / 2) * p.nkp : ncols;
        for (int sl = 0; sl < nsl && ok; ++sl, ++nsl_done) {
          const int buf = nsl_done & 1;
          const uint32_t bph = (uint32_t)(nsl_done >> 1) & 1u;
          ok = ptx::mbar_wait_sleep(&accempty[buf], bph ^ 1u);
          if (!ok) break;
          ptx::tc_fence_after();
          const int c0 = sl == 0 ? 0 : cols0;
          const int nc = sl == 0 ? cols0 : ncols - cols0;
          const uint32_t idesc = ptx::idesc_bf16(128, nc, false);
          const uint32_t d_tmem = tmem + (uint32_t)(buf * STC_SLICE);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint32_t a0 = ptx::smem_u32(sK + st[kb] * Cfg::STAGE_BYTES);
            const uint32_t b0 = ptx::smem_u32(sQ + kb * Cfg::QBLK_BYTES + c0 * 128);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              ptx::mma_bf16_ss(d_tmem, ptx::sdesc_sw128(a0 + ks * 32, 16, 1024),
                               ptx::sdesc_sw128(b0 + ks * 32, 16, 1024), idesc,
                               (kb | ks) ? 1u : 0u);
            }
          }
          ptx::tc_commit(&accfull[buf]);
        }
        for (int kb = 0; kb < KB; ++kb) ptx::tc_commit(&kempty[st[kb]]);
      }
    }
  } else {
    // ---------------- epilogue: four groups of four warps, one key per thread ----------
    // Group e (warps 2+4e .. 5+4e, one per TMEM lane quarter) takes the query heads h of
    // the column group with h % 4 == e, so a head's columns never leave the thread that
    // owns the key, and a quarter of the key's dimensions for |k|^2.  Every group hands
    // (sum of head maxima, |k|^2 share) to a shared-memory slot; the tile's merging group
    // adds the four in group order one tile later and writes the pooled score.
    // Four warps per SM sub-partition interleave their TMEM loads, which a single warp
    // cannot overlap with its own arithmetic.
    const int e = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    constexpr int DQ = D / 4;                    // dimensions of |k|^2 per group
    constexpr int CHUNKS = DQ / 8;               // 16-byte chunks (8 bf16) per group
    const int kb_e = (e * DQ) / 64;              // K-block holding this group's dimensions
    const int ch0 = ((e * DQ) % 64) / 8;         // first chunk of the 128-byte row
    float2* mslot = reinterpret_cast<float2*>(merge);
    int stage = 0, cur = -1, nsl_done = 0, ncols = 0, nmerge = 0;
    uint32_t kph = 0;
    bool ok = true;
    int b, g, cg, tile, tiles;
    stc_decode(p, tab, u_lo, b, g, cg, tile);
    tiles = (tab.prefix[b] + STC_BM - 1) / STC_BM;
    int pb = 0, pg = 0, pcg = 0, ptile = 0;
    auto merge_tile = [&](int m, int mb, int mg, int mcg, int mtile) -> bool {
      const int slot = m & 1;
      const uint32_t mph = (uint32_t)(m >> 1) & 1u;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_sleep(&mfull[slot], mph))) return false;
      float2 o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) o[q] = mslot[(slot * 4 + q) * STC_BM + row];
      ptx::mbar_arrive(&mempty[slot]);
      const float msum = ((o[0].x + o[1].x) + o[2].x) + o[3].x;   // group order
      const float mss = ((o[0].y + o[1].y) + o[2].y) + o[3].y;
      const float knorm = sqrtf(mss);
      const int j = mtile * STC_BM + row;
      if (j < tab.prefix[mb]) {
        const float sc = knorm > 0.f ? (p.ncg == 1 ? msum * p.inv_G : msum) / knorm : 0.f;
        pooled[mcg * p.cg_stride + (size_t)(mb * p.h_kv + mg) * p.pooled_stride + j] = sc;
      }
      return true;
    };
    for (int u = u_lo; u < u_hi && ok; ++u) {
      if (u != u_lo) stc_next(p, tab, b, g, cg, tile, tiles);
      const int key3 = (b * p.h_kv + g) * p.ncg + cg;
      if (key3 != cur) {
        ptx::named_bar(1, 32 * STC_EPI_WARPS);
        const int h0 = cg * p.heads_per_cg;
        ncols = (min(p.G, h0 + p.heads_per_cg) - h0) * p.nkp;
        const size_t c0 = (size_t)(b * p.h_kv + g) * p.G * p.nkp + (size_t)h0 * p.nkp;
        for (int c = threadIdx.x - 64; c < ncols; c += 32 * STC_EPI_WARPS) {
          cpi[c] = qinv[c0 + c];
          cpb[c] = qbias[c0 + c];
        }
        ptx::named_bar(1, 32 * STC_EPI_WARPS);
        cur = key3;
      }
      const int nh = ncols / p.nkp;                // query heads in this column group
      const int nsl = ncols > STC_SLICE ? 2 : 1;
      const int hs0 = nsl == 2 ? (nh + 1) / 2 : nh; // heads in slice 0 (head-aligned cut)
      int st[KB];
      uint32_t sph[KB];                            // ring slot and its phase per K-block
      for (int kb = 0; kb < KB; ++kb) {
        st[kb] = stage;
        sph[kb] = kph;
        if (++stage == NST) { stage = 0; kph ^= 1u; }
      }
      // Every K-block of the tile has landed before this warp releases it: a release of a
      // slot this warp never waited for could otherwise count toward the slot's previous
      // use.  Then |k|^2 over this group's dimensions from the swizzled tile.
      for (int kb = 0; kb < KB; ++kb)
        if (ok) ok = ptx::mbar_wait_sleep(&kfull[st[kb]], sph[kb]);
      float ss = 0.f;
      if (ok) {
        const uint8_t* rp = sK + st[kb_e] * Cfg::STAGE_BYTES + row * 128;
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(rp + (((ch0 + c) ^ (row & 7)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = bf16_lo(w[i]), hi = bf16_hi(w[i]);
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
          }
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0)
        for (int kb = 0; kb < KB; ++kb) ptx::mbar_arrive(&kempty[st[kb]]);
      if (!ok) break;

      // sum over this group's heads of max over the head's kept queries of s / |q| (+ bias):
      // whole 32-column chunks (one tcgen05.ld each) in straight-line code, then a 16-column
      // tail when the head's width is an odd multiple of 16
      auto range_max = [&](uint32_t tcol, int cbase, int ncol) -> float {
        const float* ci = cpi + cbase;
        const float* cb = cpb + cbase;
        float run = -INFINITY;
        int c = 0;
        for (; c + 32 <= ncol; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(lane_base + tcol + (uint32_t)c, r);
          ptx::tmem_ld_wait();
          float v[32];
          if (p.padded) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 sc = *reinterpret_cast<const float4*>(ci + c + i);
              const float4 bi = *reinterpret_cast<const float4*>(cb + c + i);
              v[i] = fmaf(__uint_as_float(r[i]), sc.x, bi.x);
              v[i + 1] = fmaf(__uint_as_float(r[i + 1]), sc.y, bi.y);
              v[i + 2] = fmaf(__uint_as_float(r[i + 2]), sc.z, bi.z);
              v[i + 3] = fmaf(__uint_as_float(r[i + 3]), sc.w, bi.w);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 sc = *reinterpret_cast<const float4*>(ci + c + i);
              const float2 v01 = ptx::mul2(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), make_float2(sc.x, sc.y));
              const float2 v23 = ptx::mul2(make_float2(__uint_as_float(r[i + 2]), __uint_as_float(r[i + 3])), make_float2(sc.z, sc.w));
              v[i] = v01.x; v[i + 1] = v01.y; v[i + 2] = v23.x; v[i + 3] = v23.y;
            }
          }
          float a[11];
#pragma unroll
          for (int k = 0; k < 10; ++k) a[k] = ptx::max3(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
          a[10] = fmaxf(v[30], v[31]);
          const float b0 = ptx::max3(a[0], a[1], a[2]), b1 = ptx::max3(a[3], a[4], a[5]);
          const float b2 = ptx::max3(a[6], a[7], a[8]), b3 = fmaxf(a[9], a[10]);
          run = ptx::max3(run, ptx::max3(b0, b1, b2), b3);
        }
        if (c < ncol) {                              // 16-column tail
          uint32_t r[16];
          ptx::tmem_ld16(lane_base + tcol + (uint32_t)c, r);
          ptx::tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            const float4 sc = *reinterpret_cast<const float4*>(ci + c + i);
            const float4 bi = p.padded ? *reinterpret_cast<const float4*>(cb + c + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[i] = fmaf(__uint_as_float(r[i]), sc.x, bi.x);
            v[i + 1] = fmaf(__uint_as_float(r[i + 1]), sc.y, bi.y);
            v[i + 2] = fmaf(__uint_as_float(r[i + 2]), sc.z, bi.z);
            v[i + 3] = fmaf(__uint_as_float(r[i + 3]), sc.w, bi.w);
          }
          const float a0 = ptx::max3(v[0], v[1], v[2]), a1 = ptx::max3(v[3], v[4], v[5]);
          const float a2 = ptx::max3(v[6], v[7], v[8]), a3 = ptx::max3(v[9], v[10], v[11]);
          const float a4 = ptx::max3(v[12], v[13], v[14]);
          run = ptx::max3(run, ptx::max3(a0, a1, a2), ptx::max3(a3, a4, v[15]));
        }
        return run;
      };
      float sum = 0.f;
      for (int sl = 0; sl < nsl && ok; ++sl, ++nsl_done) {
        const int buf = nsl_done & 1;
        const uint32_t bph = (uint32_t)(nsl_done >> 1) & 1u;
        // only groups with heads in the slice wait for it; the first of them also releases
        // it for the groups without any, so those move on at once
        const int h_lo = sl == 0 ? 0 : hs0, h_hi = sl == 0 ? hs0 : nh;
        const int h_first = h_lo + ((e - h_lo) & 3);
        if (h_first >= h_hi) continue;
        const int nidle = 4 - min(4, h_hi - h_lo);
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&accfull[buf], bph));
        if (!ok) break;
        ptx::tc_fence_after();
        for (int h = h_first; h < h_hi; h += 4)
          sum += range_max((uint32_t)(buf * STC_SLICE + (h - h_lo) * p.nkp), h * p.nkp, p.nkp);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_count(&accempty[buf], 1u + (e == (h_lo & 3) ? (uint32_t)nidle : 0u));
      }
      if (!ok) break;

      // Hand this tile's partials over, then merge the previous tile, whose partials are
      // all in by now: the merging group rotates, and no group waits for the slowest one.
      {
        const int slot = nmerge & 1;
        const uint32_t mph = (uint32_t)(nmerge >> 1) & 1u;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&mempty[slot], mph ^ 1u));
        if (!ok) break;
        mslot[(slot * 4 + e) * STC_BM + row] = make_float2(sum, ss);
        ptx::mbar_arrive(&mfull[slot]);
      }
      if (nmerge > 0 && e == ((nmerge - 1) & 3)) {
        ok = merge_tile(nmerge - 1, pb, pg, pcg, ptile);
        if (!ok) break;
      }
      pb = b; pg = g; pcg = cg; ptile = tile;
      ++nmerge;
    }
    if (ok && nmerge > 0 && e == ((nmerge - 1) & 3)) merge_tile(nmerge - 1, pb, pg, pcg, ptile);
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, STC_NBUF * STC_SLICE);
  }
}

}  // namespace quoka
