// K2 (CUDA-core form): cosine scoring of every prefix key against the kept queries
// with group-aware pooling (QUOKA page, method summary: cosine scoring, then max
// pooling over queries and mean pooling over the query heads of a GQA group).
//
// One CTA per (sequence, KV head, tile of 64 keys).  The key tile is staged once in
// shared memory (converted to fp32, padded rows), its norms are taken there, and the
// kept queries of the group stream through in chunks of 64 rows.  Each thread holds a
// 4 x 4 block of raw dot products; the epilogue multiplies by 1/|q|, keeps a running
// per-(key, head) maximum in shared memory, and finally writes
//     s_j = (sum_h max_h) / G / |k_j|          (0 for a zero key)
// so the full score matrix never leaves the SM.  Used for fp32 inputs, where the
// tensor cores' tf32 mode would lose precision.
#pragma once
#include "common.cuh"

namespace quoka {

constexpr int SCS_KEYS = 64;
constexpr int SCS_QROWS = 64;
constexpr int SCS_THREADS = 256;

template <int D>
__host__ __device__ constexpr int score_simt_smem_bytes(int G) {
  return (SCS_KEYS * (D + 1) + SCS_QROWS * (D + 1) + SCS_KEYS * (SCS_QROWS + 1) +
          SCS_KEYS * G + SCS_KEYS + 2 * SCS_QROWS) * 4;
}

template <typename T, int D>
__global__ void __launch_bounds__(SCS_THREADS)
score_simt_kernel(const T* __restrict__ k_cache, long long rows_per_head,
                  const __grid_constant__ SeqTable tab, int h_kv, int G, int nkp,
                  const T* __restrict__ qsel, const float* __restrict__ qinv,
                  const float* __restrict__ qbias, float* __restrict__ pooled,
                  long long pooled_stride) {
  constexpr int LD = D + 1;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Ks = reinterpret_cast<float*>(smem_raw);
  float* Qs = Ks + SCS_KEYS * LD;
  float* Sb = Qs + SCS_QROWS * LD;
  float* mx = Sb + SCS_KEYS * (SCS_QROWS + 1);   // [64 keys][G]
  float* knorm = mx + SCS_KEYS * G;
  float* qiv = knorm + SCS_KEYS;
  float* qbs = qiv + SCS_QROWS;

  const int b = blockIdx.z, g = blockIdx.y, j0 = blockIdx.x * SCS_KEYS;
  const int P = tab.prefix[b];
  if (j0 >= P) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const T* kbase = k_cache + ((size_t)g * rows_per_head + tab.kv_off[b]) * D;
  const int nrows = G * nkp;
  const T* qbase = qsel + (size_t)(b * h_kv + g) * nrows * D;
  const float* ibase = qinv + (size_t)(b * h_kv + g) * nrows;
  const float* bbase = qbias + (size_t)(b * h_kv + g) * nrows;

  // stage the key tile (zeros past P) and reset the running maxima
  for (int e = tid * 4; e < SCS_KEYS * D; e += SCS_THREADS * 4) {
    const int r = e / D, c = e % D;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (j0 + r < P) load_vec<T, 4>(kbase + (size_t)(j0 + r) * D + c, x);
#pragma unroll
    for (int i = 0; i < 4; ++i) Ks[r * LD + c + i] = x[i];
  }
  for (int e = tid; e < SCS_KEYS * G; e += SCS_THREADS) mx[e] = -INFINITY;
  __syncthreads();
  if (tid < SCS_KEYS) {
    float s = 0.f;
    for (int d = 0; d < D; ++d) s = fmaf(Ks[tid * LD + d], Ks[tid * LD + d], s);
    knorm[tid] = sqrtf(s);
  }

  for (int q0 = 0; q0 < nrows; q0 += SCS_QROWS) {
    __syncthreads();
    for (int e = tid * 4; e < SCS_QROWS * D; e += SCS_THREADS * 4) {
      const int r = e / D, c = e % D;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (q0 + r < nrows) load_vec<T, 4>(qbase + (size_t)(q0 + r) * D + c, x);
#pragma unroll
      for (int i = 0; i < 4; ++i) Qs[r * LD + c + i] = x[i];
    }
    if (tid < SCS_QROWS) {
      qiv[tid] = (q0 + tid < nrows) ? ibase[q0 + tid] : 0.f;
      qbs[tid] = (q0 + tid < nrows) ? bbase[q0 + tid] : -INFINITY;
    }
    __syncthreads();

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
      float kv[4], qv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = Ks[(ty + 16 * i) * LD + d];
#pragma unroll
      for (int j = 0; j < 4; ++j) qv[j] = Qs[(tx + 16 * j) * LD + d];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(kv[i], qv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        Sb[(ty + 16 * i) * (SCS_QROWS + 1) + tx + 16 * j] =
            fmaf(acc[i][j], qiv[tx + 16 * j], qbs[tx + 16 * j]);
    __syncthreads();
    if (tid < SCS_KEYS) {
      const int lim = min(SCS_QROWS, nrows - q0);
      for (int c = 0; c < lim; ++c) {
        const int hl = (q0 + c) / nkp;
        const float v = Sb[tid * (SCS_QROWS + 1) + c];
        float* m = &mx[tid * G + hl];
        *m = fmaxf(*m, v);
      }
    }
  }
  __syncthreads();
  if (tid < SCS_KEYS && j0 + tid < P) {
    float s = 0.f;
    for (int h = 0; h < G; ++h) s += mx[tid * G + h];
    const float r = knorm[tid];
    pooled[(size_t)(b * h_kv + g) * pooled_stride + j0 + tid] = r > 0.f ? (s / (float)G) / r : 0.f;
  }
}

}  // namespace quoka
