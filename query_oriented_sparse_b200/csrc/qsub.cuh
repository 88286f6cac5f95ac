// K1: query subselection (QUOKA page, method summary and Figure 1(b): the chunk's
// queries are filtered by cosine dissimilarity to their mean; Figure 2: queries far
// from the mean interact with more keys).
//
// One CTA per (sequence, query head).  Pass 1 streams the head's C x D query slab
// once with 8/16-byte vector loads, computes |q_t| with a warp reduction and
// accumulates the sum of unit queries (the mean's direction).  Pass 2 re-reads the
// slab (L2-resident) for c_t = cos(q_t, mean).  A 4-pass block radix select finds the
// Nk-th smallest orderable key, then a scan keeps, in ascending t, every query below
// it plus the lowest-index ties.  The kept rows are copied (raw values) into the
// per-KV-head operand block used by the scoring GEMM, with their fp32 1/|q| and a
// column bias; each head's block is padded to nkp rows (a multiple of 16) with zero
// rows whose bias is -inf, so a padded column can never win the max pooling.
#pragma once
#include "common.cuh"

namespace quoka {

constexpr int QSUB_THREADS = 512;
constexpr int QSUB_WARPS = QSUB_THREADS / 32;

template <int D>
__host__ __device__ constexpr int qsub_smem_bytes(int C) {
  return C * 4 /*inv*/ + C * 4 /*keys*/ + QSUB_WARPS * D * 4 /*partials*/;
}

// Finds the k-th smallest (1-based) of n uint32 keys in shared memory.  Returns the
// key value T and writes to *need_eq how many keys equal to T belong to the k
// smallest.  Every thread of the block must call it.
__device__ __forceinline__ uint32_t block_radix_select_smallest(const uint32_t* keys, int n, int k,
                                                                int* need_eq, int* hist,
                                                                int* misc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int t = tid; t < n; t += blockDim.x) {
      const uint32_t key = keys[t];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (warp == 0) {
      int c[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = hist[lane * 8 + j]; s += c[j]; }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - s;
      if (excl < k && k <= incl) {
        int run = excl, digit = lane * 8 + 7;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + c[j] >= k) { digit = lane * 8 + j; break; }
          run += c[j];
        }
        misc[0] = digit;
        misc[1] = run;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)misc[0] << shift;
    mask |= 0xFFu << shift;
    k -= misc[1];
    __syncthreads();
  }
  *need_eq = k;
  return prefix;
}

template <typename T, int D>
__global__ void __launch_bounds__(QSUB_THREADS)
qsub_kernel(const T* __restrict__ q, int h_q, int C, int nk, int nkp, int nq,
            int32_t* __restrict__ kept_out, T* __restrict__ qsel, float* __restrict__ qinv,
            float* __restrict__ qbias) {
  constexpr int PER = D / 32;                 // elements per lane per row
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* inv = reinterpret_cast<float*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(inv + C);
  float* part = reinterpret_cast<float*>(keys + C);
  __shared__ float mdir[D];
  __shared__ int hist[256];
  __shared__ int scan_scratch[33];
  __shared__ int misc[4];

  const int bh = blockIdx.x;                  // b * h_q + h
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* qh = q + (size_t)bh * C * D;

  // pass 1: norms and the sum of unit queries
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  for (int t = warp; t < C; t += QSUB_WARPS) {
    float x[PER];
    load_vec<T, PER>(qh + (size_t)t * D + lane * PER, x);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) ss = fmaf(x[i], x[i], ss);
    ss = warp_sum(ss);
    const float n = sqrtf(ss);
    const float iv = n > 0.f ? 1.0f / n : 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = fmaf(x[i], iv, acc[i]);
    if (lane == 0) inv[t] = iv;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) part[warp * D + lane * PER + i] = acc[i];
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll 4
    for (int w = 0; w < QSUB_WARPS; ++w) s += part[w * D + tid];
    mdir[tid] = s;
  }
  __syncthreads();
  if (warp == 0) {
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s = fmaf(mdir[d], mdir[d], s);
    s = warp_sum(s);
    if (lane == 0) misc[2] = __float_as_int(s);
  }
  __syncthreads();
  const float mn2 = __int_as_float(misc[2]);
  const float mscale = mn2 > 0.f ? 1.0f / sqrtf(mn2) : 0.f;

  // pass 2: c_t = (q_t . m) / (|q_t| |m|) as ascending-orderable keys
  float mv[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) mv[i] = mdir[lane * PER + i];
  for (int t = warp; t < C; t += QSUB_WARPS) {
    float x[PER];
    load_vec<T, PER>(qh + (size_t)t * D + lane * PER, x);
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) dot = fmaf(x[i], mv[i], dot);
    dot = warp_sum(dot);
    if (lane == 0) keys[t] = float_to_ordered(dot * inv[t] * mscale);
  }
  __syncthreads();

  // select the nk smallest keys, ties to the lower t
  int need_eq = 0;
  uint32_t thr = 0xFFFFFFFFu;
  const bool keep_all = nk >= C;
  if (!keep_all) thr = block_radix_select_smallest(keys, C, nk, &need_eq, hist, misc);

  // compaction in ascending t; kept positions overwrite keys[] (pos <= t, and every
  // key of the current window is read before the scans' barriers)
  int* sel_t = reinterpret_cast<int*>(keys);
  int run_eq = 0, run_sel = 0;
  for (int base = 0; base < C; base += blockDim.x) {
    const int t = base + tid;
    const bool valid = t < C;
    const uint32_t key = valid ? keys[t] : 0xFFFFFFFFu;
    const int is_eq = (valid && !keep_all && key == thr) ? 1 : 0;
    int tot_eq;
    const int eq_rank = block_exclusive_scan(is_eq, scan_scratch, &tot_eq) + run_eq;
    const int is_sel = (valid && (keep_all || key < thr || (is_eq && eq_rank < need_eq))) ? 1 : 0;
    int tot_sel;
    const int pos = block_exclusive_scan(is_sel, scan_scratch, &tot_sel) + run_sel;
    if (is_sel) sel_t[pos] = t;
    run_eq += tot_eq;
    run_sel += tot_sel;
  }
  __syncthreads();

  // outputs: kept positions, 1/|q|, column bias and the raw kept rows (padded to nkp)
  const size_t row0 = (size_t)bh * nkp;       // == ((b*h_kv + g)*G + h%G) * nkp
  for (int i = tid; i < nkp; i += blockDim.x) {
    const bool real = i < nk;
    qinv[row0 + i] = real ? inv[sel_t[i]] : 0.f;
    qbias[row0 + i] = real ? 0.f : -INFINITY;
    if (kept_out && i < nq) kept_out[(size_t)bh * nq + i] = real ? sel_t[i] : -1;
  }
  if (kept_out)
    for (int i = nkp + tid; i < nq; i += blockDim.x) kept_out[(size_t)bh * nq + i] = -1;
  constexpr int VEC = 16 / sizeof(T);          // elements per 16-byte vector
  constexpr int NV = D / VEC;                  // vectors per row
  for (int e = tid; e < nkp * NV; e += blockDim.x) {
    const int i = e / NV, v = e % NV;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (i < nk) val = __ldg(reinterpret_cast<const uint4*>(qh + (size_t)sel_t[i] * D) + v);
    reinterpret_cast<uint4*>(qsel + (row0 + i) * D)[v] = val;
  }
}

}  // namespace quoka
