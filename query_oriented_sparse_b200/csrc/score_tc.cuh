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
// group, 128-key tile).  A column group is up to 512 kept-query columns (whole heads);
// its operand block stays resident in shared memory while key tiles stream through a
// ring of 16 KB K-block stages loaded by TMA (128-byte swizzle).  Warp 0 issues TMA,
// one thread of warp 1 issues the MMAs into two 256-column TMEM slices, warps 2-5
// drain one slice while the tensor core fills the other.
#pragma once
#include "tc_ptx.cuh"

namespace quoka {

constexpr int STC_BM = 128;        // keys per tile (TMEM lanes)
constexpr int STC_MAXCOLS = 512;   // kept-query columns per column group
constexpr int STC_SLICE = 256;     // MMA N per accumulator slice
constexpr int STC_NBUF = 2;        // accumulator slices held in TMEM
constexpr int STC_THREADS = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int STC_QBOX = 16;       // rows per TMA box of the kept-query block

struct ScoreTcParams {
  int h_kv, G, nkp, ncg, heads_per_cg;
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
  static constexpr int CP_BYTES = STC_MAXCOLS * 8;     // (1/|q|, bias) per column
  static constexpr int NBAR = 2 * NST + 2 + 2 * STC_NBUF;
  static constexpr int SMEM = 1024 + Q_BYTES + K_BYTES + CP_BYTES + NBAR * 8 + 16;
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

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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
  float2* cp = reinterpret_cast<float2*>(sK + Cfg::K_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(cp) + Cfg::CP_BYTES);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + NST;
  uint64_t* qfull = bars + 2 * NST;
  uint64_t* qempty = qfull + 1;
  uint64_t* accfull = qfull + 2;
  uint64_t* accempty = accfull + STC_NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long per = (long long)p.total_units;
  const int u_lo = (int)(per * blockIdx.x / gridDim.x);
  const int u_hi = (int)(per * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      ptx::mbar_init(&kfull[s], 1);
      ptx::mbar_init(&kempty[s], 1 + 4);
    }
    ptx::mbar_init(qfull, 1);
    ptx::mbar_init(qempty, 1);
    for (int s = 0; s < STC_NBUF; ++s) {
      ptx::mbar_init(&accfull[s], 1);
      ptx::mbar_init(&accempty[s], 4);
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
      for (int u = u_lo; u < u_hi && ok; ++u) {
        int b, g, cg, tile;
        stc_decode(p, tab, u, b, g, cg, tile);
        const int key3 = (b * p.h_kv + g) * p.ncg + cg;
        if (key3 != cur) {
          if (cur >= 0) {
            ok = ptx::mbar_wait(qempty, qeph);
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
          ok = ptx::mbar_wait(&kempty[stage], kph ^ 1u);
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
      for (int u = u_lo; u < u_hi && ok; ++u) {
        int b, g, cg, tile;
        stc_decode(p, tab, u, b, g, cg, tile);
        const int key3 = (b * p.h_kv + g) * p.ncg + cg;
        if (key3 != cur) {
          if (cur >= 0) ptx::tc_commit(qempty);
          ok = ptx::mbar_wait(qfull, qph);
          qph ^= 1u;
          if (!ok) break;
          const int h0 = cg * p.heads_per_cg;
          ncols = (min(p.G, h0 + p.heads_per_cg) - h0) * p.nkp;
          cur = key3;
        }
        int st[KB];
        for (int kb = 0; kb < KB; ++kb) {
          st[kb] = stage;
          if (ok) ok = ptx::mbar_wait(&kfull[stage], kph);
          if (++stage == NST) { stage = 0; kph ^= 1u; }
        }
        if (!ok) break;
        ptx::tc_fence_after();
        for (int sl = 0; sl * STC_SLICE < ncols && ok; ++sl, ++nsl_done) {
          const int buf = nsl_done & 1;
          const uint32_t bph = (uint32_t)(nsl_done >> 1) & 1u;
          ok = ptx::mbar_wait(&accempty[buf], bph ^ 1u);
          if (!ok) break;
          ptx::tc_fence_after();
          const int nc = min(STC_SLICE, ncols - sl * STC_SLICE);
          const uint32_t idesc = ptx::idesc_bf16(128, nc, false);
          const uint32_t d_tmem = tmem + (uint32_t)(buf * STC_SLICE);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint32_t a0 = ptx::smem_u32(sK + st[kb] * Cfg::STAGE_BYTES);
            const uint32_t b0 = ptx::smem_u32(sQ + kb * Cfg::QBLK_BYTES + sl * STC_SLICE * 128);
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
    // ---------------- epilogue: warps 2..5, one key per thread ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    int stage = 0, cur = -1, nsl_done = 0, ncols = 0;
    uint32_t kph = 0;
    bool ok = true;
    for (int u = u_lo; u < u_hi && ok; ++u) {
      int b, g, cg, tile;
      stc_decode(p, tab, u, b, g, cg, tile);
      const int key3 = (b * p.h_kv + g) * p.ncg + cg;
      if (key3 != cur) {
        ptx::named_bar(1, 128);
        const int h0 = cg * p.heads_per_cg;
        ncols = (min(p.G, h0 + p.heads_per_cg) - h0) * p.nkp;
        const size_t c0 = (size_t)(b * p.h_kv + g) * p.G * p.nkp + (size_t)h0 * p.nkp;
        for (int c = threadIdx.x - 64; c < ncols; c += 128) cp[c] = make_float2(qinv[c0 + c], qbias[c0 + c]);
        ptx::named_bar(1, 128);
        cur = key3;
      }
      // |k| of this thread's key from the swizzled tile in shared memory
      float ss = 0.f;
      int st[KB];
      for (int kb = 0; kb < KB; ++kb) {
        st[kb] = stage;
        if (ok) ok = ptx::mbar_wait(&kfull[stage], kph);
        if (ok) {
          const uint8_t* rp = sK + stage * Cfg::STAGE_BYTES + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(rp + ((c ^ (row & 7)) << 4));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float lo = bf16_lo(w[i]), hi = bf16_hi(w[i]);
              ss = fmaf(lo, lo, ss);
              ss = fmaf(hi, hi, ss);
            }
          }
        }
        if (++stage == NST) { stage = 0; kph ^= 1u; }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0)
        for (int kb = 0; kb < KB; ++kb) ptx::mbar_arrive(&kempty[st[kb]]);
      if (!ok) break;
      const float knorm = sqrtf(ss);

      float run = -INFINITY, sum = 0.f;
      for (int sl = 0; sl * STC_SLICE < ncols && ok; ++sl, ++nsl_done) {
        const int buf = nsl_done & 1;
        const uint32_t bph = (uint32_t)(nsl_done >> 1) & 1u;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&accfull[buf], bph));
        if (!ok) break;
        ptx::tc_fence_after();
        const int nc = min(STC_SLICE, ncols - sl * STC_SLICE);
        for (int c0 = 0; c0 < nc; c0 += 64) {
          // up to four 16-column TMEM loads in flight, one wait
          uint32_t r[4][16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            if (c0 + q4 * 16 < nc)
              ptx::tmem_ld16(lane_base + (uint32_t)(buf * STC_SLICE + c0 + q4 * 16), r[q4]);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            if (c0 + q4 * 16 >= nc) break;
            const int col = sl * STC_SLICE + c0 + q4 * 16;
            if (col != 0 && col % p.nkp == 0) {     // a new query head starts here
              sum += run;
              run = -INFINITY;
            }
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 pr = cp[col + i];
              v[i] = fmaf(__uint_as_float(r[q4][i]), pr.x, pr.y);
            }
#pragma unroll
            for (int w = 8; w > 0; w >>= 1)
#pragma unroll
              for (int i = 0; i < w; ++i) v[i] = fmaxf(v[i], v[i + w]);
            run = fmaxf(run, v[0]);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&accempty[buf]);
      }
      if (!ok) break;
      sum += run;
      const int j = tile * STC_BM + row;
      if (j < tab.prefix[b]) {
        const float s = knorm > 0.f ? (p.ncg == 1 ? sum * p.inv_G : sum) / knorm : 0.f;
        pooled[cg * p.cg_stride + (size_t)(b * p.h_kv + g) * p.pooled_stride + j] = s;
      }
    }
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
