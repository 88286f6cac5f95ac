// K4 (CUDA-core form): attention of the chunk's queries over the compacted cache
// (QUOKA page, Figure 1(a): the sub-selected KV cache is fed to a dense attention
// kernel) - the selected prefix keys of the query head's KV head plus the chunk's own
// keys P..P+t (causal).  Flash-style: key blocks of 64 rows are gathered by index into
// shared memory, logits and the online softmax run in fp32 (base-2 exponent with the
// 1/sqrt(d) scale folded into log2(e)), and the output is normalised once at the end.
//
// One CTA per (sequence, query head, 64 query rows).  Used for fp32 inputs, where the
// 1e-4 relative bound rules out tf32 tensor-core math.
#pragma once
#include "common.cuh"

namespace quoka {

constexpr int ATS_ROWS = 64;
constexpr int ATS_KEYS = 64;
constexpr int ATS_THREADS = 256;

template <int D>
__host__ __device__ constexpr int attn_simt_smem_bytes() {
  return (ATS_ROWS * (D + 1) + ATS_KEYS * (D + 1) + ATS_KEYS * D + ATS_ROWS * (ATS_KEYS + 1)) * 4 +
         ATS_KEYS * 8;
}

template <typename T, int D>
__global__ void __launch_bounds__(ATS_THREADS)
attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k_cache,
                 const T* __restrict__ v_cache, long long rows_per_head,
                 const __grid_constant__ SeqTable tab, int h_q, int h_kv, int C,
                 const int32_t* __restrict__ idx, int b_max, T* __restrict__ out,
                 float scale_log2) {
  constexpr int LD = D + 1;
  constexpr int DJ = D / 16;                  // output columns per thread
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Qs = reinterpret_cast<float*>(smem_raw);
  float* Ks = Qs + ATS_ROWS * LD;
  float* Vs = Ks + ATS_KEYS * LD;
  float* Ps = Vs + ATS_KEYS * D;
  long long* rowid = reinterpret_cast<long long*>(Ps + ATS_ROWS * (ATS_KEYS + 1));

  const int b = blockIdx.z, h = blockIdx.y, t0 = blockIdx.x * ATS_ROWS;
  const int G = h_q / h_kv, g = h / G;
  const int P = tab.prefix[b], nsel = tab.nsel[b];
  const int tid = threadIdx.x, tc = tid & 15, tr = tid >> 4;
  const int tlast = min(C, t0 + ATS_ROWS) - 1;
  const int nkeys = nsel + tlast + 1;
  const size_t head_row0 = (size_t)g * rows_per_head + tab.kv_off[b];
  const T* kh = k_cache + head_row0 * D;
  const T* vh = v_cache + head_row0 * D;
  const int32_t* sel = idx + (size_t)(b * h_kv + g) * b_max;
  const T* qh = q + ((size_t)(b * h_q + h) * C) * D;

  for (int e = tid * 4; e < ATS_ROWS * D; e += ATS_THREADS * 4) {
    const int r = e / D, c = e % D;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (t0 + r < C) load_vec<T, 4>(qh + (size_t)(t0 + r) * D + c, x);
#pragma unroll
    for (int i = 0; i < 4; ++i) Qs[r * LD + c + i] = x[i];
  }

  float m[4], l[4], o[4][DJ];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int j = 0; j < DJ; ++j) o[i][j] = 0.f;
  }

  for (int kb = 0; kb < nkeys; kb += ATS_KEYS) {
    __syncthreads();                           // previous block fully consumed
    if (tid < ATS_KEYS) {
      const int kk = kb + tid;
      long long r = -1;
      if (kk < nsel) {
        r = sel[kk];
        if (r < 0 || r >= P) { flag_error(ERR_BAD_INDEX); r = -1; }   // caller error: skip
      } else if (kk < nkeys) {
        r = P + (kk - nsel);
      }
      rowid[tid] = r;
    }
    __syncthreads();
    for (int e = tid * 4; e < ATS_KEYS * D; e += ATS_THREADS * 4) {
      const int r = e / D, c = e % D;
      float xk[4] = {0.f, 0.f, 0.f, 0.f}, xv[4] = {0.f, 0.f, 0.f, 0.f};
      const long long row = rowid[r];
      if (row >= 0) {
        load_vec<T, 4>(kh + row * D + c, xk);
        load_vec<T, 4>(vh + row * D + c, xv);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        Ks[r * LD + c + i] = xk[i];
        Vs[r * D + c + i] = xv[i];
      }
    }
    __syncthreads();

    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
      float qv[4], kv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) qv[i] = Qs[(tr + 16 * i) * LD + d];
#pragma unroll
      for (int j = 0; j < 4; ++j) kv[j] = Ks[(tc + 16 * j) * LD + d];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = fmaf(qv[i], kv[j], s[i][j]);
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + tr + 16 * i;
      float rmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kk = kb + tc + 16 * j;
        const bool ok = kk < nkeys && (kk < nsel || (kk - nsel) <= t);
        s[i][j] = ok ? s[i][j] * scale_log2 : -INFINITY;
        rmax = fmaxf(rmax, s[i][j]);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, off));
      const float mnew = fmaxf(m[i], rmax);
      const float muse = (mnew == -INFINITY) ? 0.f : mnew;
      const float alpha = exp2f(m[i] - muse);
      float rsum = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = exp2f(s[i][j] - muse);
        rsum += p;
        Ps[(tr + 16 * i) * (ATS_KEYS + 1) + tc + 16 * j] = p;
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, off);
      l[i] = l[i] * alpha + rsum;
      m[i] = mnew;
#pragma unroll
      for (int j = 0; j < DJ; ++j) o[i][j] *= alpha;
    }
    __syncthreads();
    const int klim = min(ATS_KEYS, nkeys - kb);
    for (int kk = 0; kk < klim; ++kk) {
      float pv[4], vv[DJ];
#pragma unroll
      for (int i = 0; i < 4; ++i) pv[i] = Ps[(tr + 16 * i) * (ATS_KEYS + 1) + kk];
#pragma unroll
      for (int j = 0; j < DJ; ++j) vv[j] = Vs[kk * D + tc + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < DJ; ++j) o[i][j] = fmaf(pv[i], vv[j], o[i][j]);
    }
  }

  T* oh = out + ((size_t)(b * h_q + h) * C) * D;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + tr + 16 * i;
    if (t < C) {
      const float inv = l[i] > 0.f ? 1.0f / l[i] : 0.f;
#pragma unroll
      for (int j = 0; j < DJ; ++j) oh[(size_t)t * D + tc + 16 * j] = from_f32<T>(o[i][j] * inv);
    }
  }
}

}  // namespace quoka
