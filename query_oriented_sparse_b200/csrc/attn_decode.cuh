// Attention of a few query rows per KV head over the selected keys, gathered straight
// from the cache: the decode shape (QUOKA page, results summary: the method also runs in
// the generation phase), where a step brings one new token per sequence (C = 1) or a
// short chunk, so only R = G * C query rows share a KV head.
//
// With so few rows a 128-row tensor-core tile would be almost all padding, and the
// compacted copy would double the bytes moved.  Here each selected K and V row is read
// once from the cache, which is the floor.  Keys are split across CTAs (split-K): each
// CTA keeps a running max, sum and output per row (online softmax) and writes them as a
// partial; attn_decode_combine_kernel merges the partials of each (sequence, KV head).
//
// Per CTA: NW warps, each taking batches of 32 keys of the CTA's split.  A batch's K and V
// rows are gathered into the warp's own shared-memory stage with 16-byte cp.async, K and
// V in separate groups, so the logits start while V is still in flight.
//   QK: lane l owns key l of the batch and computes its R logits over the whole row; the
//       (pre-scaled) query rows are read from shared memory as broadcasts.
//   PV: lane l owns head dims [EPL*l, EPL*l + EPL) of all R output rows.
// Rows are padded by 16 bytes in shared memory, so the row-per-lane reads of QK hit
// distinct banks.
#pragma once
#include "common.cuh"

namespace quoka {

constexpr int ADC_MAX_ROWS = 16;      // query rows per KV head (G * C) this path takes
constexpr int ADC_MIN_SPLIT = 256;    // keys per CTA at least (bounds the partials' bytes)
constexpr int ADC_MAX_SPLIT = 4096;   // unless that would need more than ADC_MAX_NSPLIT splits
constexpr int ADC_MAX_NSPLIT = 512;   // splits per (sequence, KV head) at most
constexpr int ADC_COMBINE_THREADS = 512;

template <typename T, int D>
struct AdcCfg {
  static constexpr int ESZ = (int)sizeof(T);
  static constexpr int VPR = D * ESZ / 16;            // 16-byte vectors per row
  static constexpr int EPV = 16 / ESZ;                // elements per 16-byte vector
  static constexpr int ROW = D * ESZ + 16;            // padded shared-memory row, bytes
  static constexpr int NW = ROW > 300 ? 2 : 4;        // warps per CTA
  static constexpr int THREADS = NW * 32;
  static constexpr int EPL = D / 32;                  // head dims per lane in P.V
  static constexpr int STAGE = 2 * 32 * ROW;          // one warp's K and V rows
  static constexpr int PD = D + 4;                    // floats per partial row: o[D], m, l
};

template <typename T, int D, int R>
constexpr int adc_smem_bytes() {
  using Cfg = AdcCfg<T, D>;
  return R * D * 4 + Cfg::NW * R * 2 * 4 + Cfg::NW * (Cfg::STAGE + 32 * R * 4);
}

__device__ __forceinline__ void adc_cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void adc_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void adc_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// EPV consecutive elements of a 16-byte shared-memory vector as floats
template <typename T>
__device__ __forceinline__ void smem_vec16(const unsigned char* p, float (&x)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void smem_vec16<float>(const unsigned char* p, float (&x)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
template <>
__device__ __forceinline__ void smem_vec16<__nv_bfloat16>(const unsigned char* p, float (&x)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const unsigned int w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    unsigned int wi = w[i];
    const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wi));
    x[2 * i] = f.x; x[2 * i + 1] = f.y;
  }
}

// N consecutive elements (N * sizeof(T) = 4, 8 or 16 bytes) from shared memory as floats
template <typename T, int N>
__device__ __forceinline__ void smem_vecn(const unsigned char* p, float (&x)[N]) {
  if constexpr (sizeof(T) == 4) {
    if constexpr (N == 4) {
      const float4 v = *reinterpret_cast<const float4*>(p);
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(p);
      x[0] = v.x; x[1] = v.y;
    }
  } else {
    if constexpr (N == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      unsigned int a = v.x, b = v.y;
      const float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&b));
      x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
    } else {
      unsigned int a = *reinterpret_cast<const unsigned int*>(p);
      const float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a));
      x[0] = fa.x; x[1] = fa.y;
    }
  }
}

// One CTA per (split s, KV head g, sequence b).  Keys of (b, g): i < n are the selected
// prefix rows idx[b, g, i]; i = n + u (u < C) is the chunk's own row P + u, visible to
// chunk position t when u <= t.
template <typename T, int D, int R>
__global__ void __launch_bounds__(AdcCfg<T, D>::THREADS)
attn_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   long long rows_per_head, const __grid_constant__ SeqTable tab, int h_q,
                   int h_kv, int C, const int32_t* __restrict__ idx, int b_max, int split,
                   int nsplit_ws, float scale_log2, float* __restrict__ part) {
  using Cfg = AdcCfg<T, D>;
  constexpr int NW = Cfg::NW, ROW = Cfg::ROW, VPR = Cfg::VPR, EPV = Cfg::EPV, EPL = Cfg::EPL;
  extern __shared__ __align__(16) unsigned char smem[];
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int n = tab.nsel[b], P = tab.prefix[b];
  const int k0 = s * split;
  const int k1 = min(n + C, k0 + split);
  if (k0 >= k1) return;                                    // uniform over the CTA
  const int G = h_q / h_kv;
  const int rows = G * C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* qs = reinterpret_cast<float*>(smem);              // [R][D], times scale * log2(e)
  float* mls = qs + R * D;                                 // [NW][R][2]: warp m, l
  unsigned char* stage = smem + (R * D + NW * R * 2) * 4 + warp * (Cfg::STAGE + 32 * R * 4);
  unsigned char* vstage = stage + 32 * ROW;
  float* ps = reinterpret_cast<float*>(stage + Cfg::STAGE);   // [32 keys][R]

  for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
    const int r = e / D, d = e - r * D;
    float x = 0.f;
    if (r < rows) {
      const int j = r / C, t = r - j * C;
      x = to_f32(q[(((size_t)b * h_q + (size_t)g * G + j) * C + t) * D + d]) * scale_log2;
    }
    qs[e] = x;
  }
  __syncthreads();

  const T* kb = k + ((size_t)g * rows_per_head + tab.kv_off[b]) * D;
  const T* vb = v + ((size_t)g * rows_per_head + tab.kv_off[b]) * D;
  const int32_t* ib = idx + ((size_t)b * h_kv + g) * b_max;
  float m[R], l[R], acc[R][EPL];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[r][e] = 0.f;
  }

  for (int i0 = k0 + warp * 32; i0 < k1; i0 += NW * 32) {
    const int i = i0 + lane;
    int rr = P;                                            // a valid row for idle lanes
    if (i < min(n, k1)) {
      rr = __ldg(ib + i);
      if (rr < 0 || rr >= P) { flag_error(ERR_BAD_INDEX); rr = P; }
    } else if (i < k1) {
      rr = P + (i - n);
    }
    // gather the batch's K rows, then its V rows (one commit group each)
#pragma unroll 4
    for (int e = lane; e < 32 * VPR; e += 32) {
      const int kk = e / VPR, vv = e - kk * VPR;
      const int rk = __shfl_sync(0xffffffffu, rr, kk);
      adc_cp16(stage + kk * ROW + vv * 16, kb + (size_t)rk * D + vv * EPV);
    }
    adc_commit();
#pragma unroll 4
    for (int e = lane; e < 32 * VPR; e += 32) {
      const int kk = e / VPR, vv = e - kk * VPR;
      const int rk = __shfl_sync(0xffffffffu, rr, kk);
      adc_cp16(vstage + kk * ROW + vv * 16, vb + (size_t)rk * D + vv * EPV);
    }
    adc_commit();
    adc_wait<1>();
    __syncwarp();

    // logits of this lane's key for every row
    float sc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) sc[r] = 0.f;
    const unsigned char* krow = stage + lane * ROW;
#pragma unroll 2
    for (int c = 0; c < VPR; ++c) {
      float kx[EPV];
      smem_vec16<T>(krow + c * 16, kx);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float* qr = qs + r * D + c * EPV;
#pragma unroll
        for (int e4 = 0; e4 < EPV; e4 += 4) {
          const float4 qv = *reinterpret_cast<const float4*>(qr + e4);
          sc[r] = fmaf(qv.x, kx[e4], sc[r]);
          sc[r] = fmaf(qv.y, kx[e4 + 1], sc[r]);
          sc[r] = fmaf(qv.z, kx[e4 + 2], sc[r]);
          sc[r] = fmaf(qv.w, kx[e4 + 3], sc[r]);
        }
      }
    }
    // masks: keys past the split, and chunk keys after the row's position
    const int u = i - n;                                   // chunk key index when >= 0
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int t = r % C;
      if (i >= k1 || (u >= 0 && u > t)) sc[r] = -INFINITY;
    }
    // online softmax per row
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float mx = sc[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mn = fmaxf(m[r], mx);
      float p = 0.f, corr = 1.f;
      if (mn != -INFINITY) {
        p = exp2f(sc[r] - mn);
        corr = exp2f(m[r] - mn);
      }
      float sum = p;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      l[r] = l[r] * corr + sum;
      m[r] = mn;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[r][e] *= corr;
      ps[lane * R + r] = p;
    }
    adc_wait<0>();
    __syncwarp();

    // P.V: this lane's head dims of every row
    const int nk = min(32, k1 - i0);
    for (int kk = 0; kk < nk; ++kk) {
      float vx[EPL];
      smem_vecn<T, EPL>(vstage + kk * ROW + lane * EPL * Cfg::ESZ, vx);
      const float* pk = ps + kk * R;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float pr = pk[r];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[r][e] = fmaf(pr, vx[e], acc[r][e]);
      }
    }
    __syncwarp();                                          // stage free for the next batch
  }

  // merge the warps: each warp parks (m, l) and its output rows, then the CTA combines
  float* wout = reinterpret_cast<float*>(stage);           // [R][D] of this warp
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      mls[(warp * R + r) * 2] = m[r];
      mls[(warp * R + r) * 2 + 1] = l[r];
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int e = 0; e < EPL; ++e) wout[r * D + lane * EPL + e] = acc[r][e];
  __syncthreads();
  float* dst = part + (((size_t)(b * h_kv + g) * nsplit_ws + s) * R) * Cfg::PD;
  for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
    const int r = e / D, d = e - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mls[(w * R + r) * 2]);
    float o = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = mls[(w * R + r) * 2];
        const float* ww = reinterpret_cast<const float*>(smem + (R * D + NW * R * 2) * 4 +
                                                         w * (Cfg::STAGE + 32 * R * 4));
        if (mw != -INFINITY) o += ww[e] * exp2f(mw - M);
      }
    }
    dst[r * Cfg::PD + d] = o;
    if (d == 0) {
      float L = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float mw = mls[(w * R + r) * 2];
          if (mw != -INFINITY) L += mls[(w * R + r) * 2 + 1] * exp2f(mw - M);
        }
      }
      dst[r * Cfg::PD + D] = M;
      dst[r * Cfg::PD + D + 1] = L;
    }
  }
}

// Merges the splits of each (sequence b, KV head g): out = sum_s o_s 2^(m_s - M) /
// sum_s l_s 2^(m_s - M), M the largest m_s.  Every row has at least its own chunk key,
// so the denominator is positive.  The partials were just written and sit in L2, so the
// merge is a few L2 round trips when its loads are in flight together: warp r reads row
// r's (m, l) of every split at once (lane per split) and leaves each split's weight
// 2^(m_s - M) in shared memory; then each thread takes output elements and loads that
// element of up to eight splits before adding them in split order.
template <typename T, int D, int R>
__global__ void __launch_bounds__(ADC_COMBINE_THREADS)
attn_decode_combine_kernel(const float* __restrict__ part, const __grid_constant__ SeqTable tab,
                           int h_q, int h_kv, int C, int split, int nsplit_ws, T* __restrict__ out) {
  constexpr int PD = D + 4;
  extern __shared__ float cw[];                            // [split][R] weights
  __shared__ float Ls[R];
  const int g = blockIdx.x, b = blockIdx.y;
  const int G = h_q / h_kv, rows = G * C;
  const int nkeys = tab.nsel[b] + C;
  const int ns = (nkeys + split - 1) / split;
  const float* src = part + (size_t)(b * h_kv + g) * nsplit_ws * R * PD;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < rows; r += ADC_COMBINE_THREADS / 32) {
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, src[((size_t)s * R + r) * PD + D]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float ms = src[((size_t)s * R + r) * PD + D];
      const float e = ms != -INFINITY ? exp2f(ms - M) : 0.f;   // an empty split weighs 0
      cw[s * R + r] = e;
      if (ms != -INFINITY) L += src[((size_t)s * R + r) * PD + D + 1] * e;
    }
    L = warp_sum(L);
    if (lane == 0) Ls[r] = L;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < rows * D; e += ADC_COMBINE_THREADS) {
    const int r = e / D, d = e - r * D;
    float o = 0.f;
    for (int s0 = 0; s0 < ns; s0 += 8) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = s0 + u < ns ? src[((size_t)(s0 + u) * R + r) * PD + d] : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (s0 + u < ns) o = fmaf(x[u], cw[(s0 + u) * R + r], o);
    }
    const int j = r / C, t = r - j * C;
    out[(((size_t)b * h_q + (size_t)g * G + j) * C + t) * D + d] = from_f32<T>(o / Ls[r]);
  }
}

}  // namespace quoka
