// Decode-step scoring on tensor cores, bf16 (QUOKA page, results summary: the method
// also runs in the generation phase; method summary: cosine scoring, max over a head's
// queries, mean over the group's heads).
//
// With every query of a decode step kept and at most 16 query rows per KV head, scoring
// is a stream over the prefix keys with a few dot products per key, so the kernel is
// built to keep HBM busy: TMA streams 128-key tiles (128-byte swizzle) through a ring of
// shared-memory stages, one thread issues S = K_tile . Q^T as a 128 x 16 tcgen05.mma
// (the raw bf16 query rows of the KV head, padded to 16, in shared memory; fp32
// accumulation in TMEM), and four epilogue warps, one thread per key, read the key's 16
// accumulator columns with one tcgen05.ld, take |k|^2 from the key's row in the stage,
// and write
//     s = (1/G) sum_h max_t (q_{h,t} . k / |q_{h,t}|) / |k|.
// 1/|q| of each row is taken once per CTA from the query block in shared memory, so
// the only HBM traffic is one read of the keys and the pooled-score write.  The pooled
// scores are stored with an L2 evict-last policy, so the key stream behind them does not
// push them out before the top-k reads them.
//
// One CTA per (span of SDT_TILES tiles, KV head, sequence); two CTAs fit on an SM, so one
// streams while the other starts or drains.  Warp 0 loads, warp 1 issues the MMAs,
// warps 2-5 run the epilogue (TMEM lane quarter = warp % 4).  Every wait is bounded.
#pragma once
#include "tc_ptx.cuh"

namespace quoka {

constexpr int SDT_THREADS = 192;
constexpr int SDT_TILES = 8;        // 128-key tiles per CTA
constexpr int SDT_NACC = 4;         // 16-column accumulators in TMEM
constexpr int SDT_QROWS = 16;       // query rows per KV head (MMA N)

template <int D>
struct SdtCfg {
  static constexpr int KB = D / 64;                  // 128-byte K-blocks per row
  static constexpr int STAGE = 128 * D * 2;          // one 128-key tile
  static constexpr int NST = (D == 128) ? 3 : 6;     // stages in the key ring
  static constexpr int Q_BYTES = SDT_QROWS * 128 * KB;
  static constexpr int NBAR = 2 * NST + 2 * SDT_NACC + 1;
  static constexpr int SMEM = 1024 + Q_BYTES + NST * STAGE + NBAR * 8 + 16 + SDT_QROWS * 4;
};

// Query rows of KV head g: r = jh * C + t for query head g*G + jh and chunk position t,
// consecutive rows of q [batch, h_q, C, D] starting at (b*h_q + g*G)*C (rows past R are
// loaded but not used).
template <int D>
__global__ void __launch_bounds__(SDT_THREADS)
score_decode_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ SeqTable tab, long long rows_per_head, int h_q, int h_kv,
                       int C, float* __restrict__ pooled, long long pooled_stride) {
  using Cfg = SdtCfg<D>;
  constexpr int KB = Cfg::KB, NST = Cfg::NST;
  const int g = blockIdx.y, b = blockIdx.z;
  const int P = tab.prefix[b];
  const int j0 = blockIdx.x * SDT_TILES * 128;
  if (j0 >= P) return;                                     // uniform over the CTA
  const int ntile = min(SDT_TILES, (P - j0 + 127) / 128);
  const int G = h_q / h_kv, R = G * C;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::Q_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + NST * Cfg::STAGE);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + NST;
  uint64_t* accfull = bars + 2 * NST;
  uint64_t* accempty = accfull + SDT_NACC;
  uint64_t* qfull = accempty + SDT_NACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);
  float* qinv_s = reinterpret_cast<float*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      ptx::mbar_init(&kfull[s], 1);
      ptx::mbar_init(&kempty[s], 1 + 4);                   // MMA commit + 4 epilogue warps
    }
    for (int s = 0; s < SDT_NACC; ++s) {
      ptx::mbar_init(&accfull[s], 1);
      ptx::mbar_init(&accempty[s], 4);
    }
    ptx::mbar_init(qfull, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 64);
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
      const int qrow0 = (b * h_q + g * G) * C;
      ptx::mbar_expect_tx(qfull, (uint32_t)Cfg::Q_BYTES);
      for (int kb = 0; kb < KB; ++kb) ptx::tma_load_2d(sQ + kb * SDT_QROWS * 128, &qmap, qfull, kb * 64, qrow0);
      const int krow0 = (int)(g * rows_per_head + tab.kv_off[b]) + j0;
      for (int t = 0; t < ntile; ++t) {
        const int st = t % NST;
        if (!ptx::mbar_wait_sleep(&kempty[st], ((uint32_t)(t / NST) & 1u) ^ 1u)) break;
        ptx::mbar_expect_tx(&kfull[st], (uint32_t)Cfg::STAGE);
        for (int kb = 0; kb < KB; ++kb)
          ptx::tma_load_2d(sK + st * Cfg::STAGE + kb * 16384, &kmap, &kfull[st], kb * 64, krow0 + t * 128);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16(128, SDT_QROWS, false);
      bool ok = ptx::mbar_wait_sleep(qfull, 0);
      for (int t = 0; t < ntile && ok; ++t) {
        const int st = t % NST, buf = t % SDT_NACC;
        ok = ptx::mbar_wait_sleep(&kfull[st], (uint32_t)(t / NST) & 1u);
        if (ok) ok = ptx::mbar_wait_sleep(&accempty[buf], ((uint32_t)(t / SDT_NACC) & 1u) ^ 1u);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * SDT_QROWS);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
          const uint32_t a0 = ptx::smem_u32(sK + st * Cfg::STAGE + kb * 16384);
          const uint32_t b0 = ptx::smem_u32(sQ + kb * SDT_QROWS * 128);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            ptx::mma_bf16_ss(d_tmem, ptx::sdesc_sw128(a0 + ks * 32, 16, 1024),
                             ptx::sdesc_sw128(b0 + ks * 32, 16, 1024), idesc, (kb | ks) ? 1u : 0u);
        }
        ptx::tc_commit(&accfull[buf]);
        ptx::tc_commit(&kempty[st]);
      }
    }
  } else {
    // ---------------- epilogue: one thread per key ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    // 1/|q| of the query rows: epilogue warp w takes rows w, w+4, ...; lane l reads D/32
    // consecutive dimensions of the row from the swizzled block
    bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(qfull, 0));
    {
      constexpr int E = D / 32;                            // bf16 elements per lane
      const int off = lane * E * 2;                        // byte offset in the D*2-byte row
      const int kb = off >> 7, chunk = (off & 127) >> 4, within = off & 15;
      for (int r = warp - 2; r < SDT_QROWS; r += 4) {
        float ss = 0.f;
        if (ok) {
          const uint8_t* p = sQ + kb * SDT_QROWS * 128 + r * 128 + ((chunk ^ (r & 7)) << 4) + within;
          if constexpr (E == 4) {
            const uint2 v = *reinterpret_cast<const uint2*>(p);
            const float x0 = bf16_lo(v.x), x1 = bf16_hi(v.x);
            const float x2 = bf16_lo(v.y), x3 = bf16_hi(v.y);
            ss = fmaf(x0, x0, fmaf(x1, x1, fmaf(x2, x2, x3 * x3)));
          } else {
            const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
            const float x0 = bf16_lo(v), x1 = bf16_hi(v);
            ss = fmaf(x0, x0, x1 * x1);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) qinv_s[r] = (r < R && ss > 0.f) ? 1.0f / sqrtf(ss) : 0.f;
      }
    }
    ptx::named_bar(1, 128);
    float inv[SDT_QROWS];
#pragma unroll
    for (int r = 0; r < SDT_QROWS; ++r) inv[r] = qinv_s[r];
    float* out = pooled + (size_t)(b * h_kv + g) * pooled_stride;
    const float inv_G = 1.0f / (float)G;
    for (int t = 0; t < ntile && ok; ++t) {
      const int st = t % NST, buf = t % SDT_NACC;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait_sleep(&accfull[buf], (uint32_t)(t / SDT_NACC) & 1u));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t a[16];
      ptx::tmem_ld16(lane_base + (uint32_t)(buf * SDT_QROWS), a);
      // |k|^2 from this key's row of the stage (the MMAs that read it are done; the stage
      // stays until every epilogue warp has released it)
      const uint8_t* rp = sK + st * Cfg::STAGE + row * 128;
      float2 nn2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int kb = 0; kb < KB; ++kb)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(rp + kb * 16384 + ((c ^ (row & 7)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 k2 = make_float2(bf16_lo(w[i]), bf16_hi(w[i]));
            nn2 = ptx::fma2(k2, k2, nn2);
          }
        }
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&accempty[buf]);
        ptx::mbar_arrive(&kempty[st]);
      }
      // rows are head-major (r = jh * C + t): max over each head's C rows, summed
      float s = 0.f, m = -INFINITY;
      int cnt = 0;
#pragma unroll
      for (int r = 0; r < SDT_QROWS; ++r) {
        if (r < R) {
          m = fmaxf(m, __uint_as_float(a[r]) * inv[r]);
          if (++cnt == C) { s += m; m = -INFINITY; cnt = 0; }
        }
      }
      const float nn = nn2.x + nn2.y;
      const int j = j0 + t * 128 + row;
      if (j < P) {                                         // the top-k reads it next: keep it in L2
        const float val = nn > 0.f ? (s * inv_G) / sqrtf(nn) : 0.f;
        uint64_t pol;
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
        asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(out + j), "f"(val), "l"(pol) : "memory");
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 64);
  }
}

}  // namespace quoka
