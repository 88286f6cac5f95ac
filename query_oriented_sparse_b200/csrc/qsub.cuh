// K1: query subselection (QUOKA page, method summary and Figure 1(b): the chunk's
// queries are filtered by cosine dissimilarity to their mean; Figure 2: queries far
// from the mean interact with more keys).
//
// One thread-block cluster of QSUB_CS CTAs per (sequence, query head); CTA r owns a
// contiguous slice of the chunk positions.  Pass 1 streams the slice once with vector
// loads (eight rows in flight per warp), takes |q_t| with a warp reduction and sums the
// unit queries; the CTAs' partial sums meet through distributed shared memory (in rank
// order, so the mean direction is the same on every CTA).  Pass 2 re-reads the slice
// (L2-resident) for c_t = cos(q_t, mean) as orderable keys in shared memory.  A cluster
// radix select keeps the Nk smallest, ties to the lower t, in ascending t
// (cluster_select.cuh).  The kept rows are copied (raw values) into the per-KV-head
// operand block of the scoring GEMM with their fp32 1/|q| and a column bias; each
// head's block is padded to nkp rows (a multiple of 16) with zero rows whose bias is
// -inf, so a padded column can never win the max pooling.
#pragma once
#include "cluster_select.cuh"

namespace quoka {

constexpr int QSUB_CS = 8;                    // CTAs per query head
constexpr int QSUB_THREADS = 512;
constexpr int QSUB_WARPS = QSUB_THREADS / 32;
constexpr int QSUB_MAX_ROWS = (QUOKA_MAX_CHUNK + QSUB_CS - 1) / QSUB_CS;
constexpr int QSUB_UNROLL = 8;

template <typename T, int D>
__global__ void __cluster_dims__(QSUB_CS, 1, 1) __launch_bounds__(QSUB_THREADS)
qsub_kernel(const T* __restrict__ q, int C, int nk, int nkp, int nq,
            int32_t* __restrict__ kept_out, T* __restrict__ qsel, float* __restrict__ qinv,
            float* __restrict__ qbias) {
  constexpr int PER = D / 32;                 // elements per lane per row
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float inv[QSUB_MAX_ROWS];
  __shared__ uint32_t keys[QSUB_MAX_ROWS];
  __shared__ float part[QSUB_WARPS][D];
  __shared__ float cta_sum[D];
  __shared__ float mdir[D];
  __shared__ float mscale_s;
  __shared__ ClusterSelectSmem sm;
  __shared__ int kept_pos[QSUB_MAX_ROWS], kept_t[QSUB_MAX_ROWS];
  __shared__ int n_kept;

  const int rank = (int)cluster.block_rank();
  const int bh = blockIdx.x / QSUB_CS;        // b * h_q + h
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = (C + QSUB_CS - 1) / QSUB_CS;
  const int lo = min(C, rank * S), hi = min(C, lo + S);
  const T* qh = q + (size_t)bh * C * D;

  // pass 1: norms and the sum of unit queries over this CTA's slice
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  for (int t0 = lo + warp; t0 < hi; t0 += QSUB_WARPS * QSUB_UNROLL) {
    float x[QSUB_UNROLL][PER];
#pragma unroll
    for (int u = 0; u < QSUB_UNROLL; ++u) {
      const int t = t0 + u * QSUB_WARPS;
      if (t < hi) load_vec<T, PER>(qh + (size_t)t * D + lane * PER, x[u]);
    }
#pragma unroll
    for (int u = 0; u < QSUB_UNROLL; ++u) {
      const int t = t0 + u * QSUB_WARPS;
      if (t >= hi) break;
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) ss = fmaf(x[u][i], x[u][i], ss);
      ss = warp_sum(ss);
      const float n = sqrtf(ss);
      const float iv = n > 0.f ? 1.0f / n : 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(x[u][i], iv, acc[i]);
      if (lane == 0) inv[t - lo] = iv;
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) part[warp][lane * PER + i] = acc[i];
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < QSUB_WARPS; ++w) s += part[w][tid];
    cta_sum[tid] = s;
  }
  cluster.sync();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < QSUB_CS; ++r) s += cluster.map_shared_rank(cta_sum, r)[tid];
    mdir[tid] = s;
  }
  cluster.sync();                              // remote reads done before anyone moves on
  if (warp == 0) {
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s = fmaf(mdir[d], mdir[d], s);
    s = warp_sum(s);
    if (lane == 0) mscale_s = s > 0.f ? 1.0f / sqrtf(s) : 0.f;
  }
  __syncthreads();
  const float mscale = mscale_s;

  // pass 2: c_t = (q_t . m) / (|q_t| |m|) as ascending-orderable keys
  float mv[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) mv[i] = mdir[lane * PER + i];
  for (int t0 = lo + warp; t0 < hi; t0 += QSUB_WARPS * QSUB_UNROLL) {
    float x[QSUB_UNROLL][PER];
#pragma unroll
    for (int u = 0; u < QSUB_UNROLL; ++u) {
      const int t = t0 + u * QSUB_WARPS;
      if (t < hi) load_vec<T, PER>(qh + (size_t)t * D + lane * PER, x[u]);
    }
#pragma unroll
    for (int u = 0; u < QSUB_UNROLL; ++u) {
      const int t = t0 + u * QSUB_WARPS;
      if (t >= hi) break;
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) dot = fmaf(x[u][i], mv[i], dot);
      dot = warp_sum(dot);
      if (lane == 0) keys[t - lo] = float_to_ordered(dot * inv[t - lo] * mscale);
    }
  }
  __syncthreads();

  // keep the nk smallest (all of them when nk >= C), emitted in ascending t
  const size_t row0 = (size_t)bh * nkp;       // == ((b*h_kv + g)*G + h%G) * nkp
  if (tid == 0) n_kept = 0;
  __syncthreads();
  auto emit = [&](int pos, int t) {
    if (pos >= nk) { flag_error(ERR_BAD_INDEX); return; }   // unreachable when counts agree
    qinv[row0 + pos] = inv[t - lo];
    qbias[row0 + pos] = 0.f;
    if (kept_out) kept_out[(size_t)bh * nq + pos] = t;
    const int slot = atomicAdd(&n_kept, 1);   // rows are copied below, coalesced
    kept_pos[slot] = pos;
    kept_t[slot] = t;
  };
  if (nk >= C) {
    for (int t = lo + tid; t < hi; t += blockDim.x) emit(t, t);
  } else {
    auto key_at = [&](int j) { return keys[j - lo]; };
    uint32_t thr;
    int need_eq;
    cluster_threshold<QSUB_CS, false>(cluster, sm, key_at, lo, hi, nk, &thr, &need_eq);
    cluster_emit<QSUB_CS, false>(cluster, sm, key_at, lo, hi, thr, need_eq, emit);
  }
  __syncthreads();
  {
    constexpr int VPR = D * (int)sizeof(T) / 16;   // 16-byte vectors per row
    const int n = n_kept;
    for (int e = tid; e < n * VPR; e += blockDim.x) {
      const int i = e / VPR, v = e - i * VPR;
      const uint4* src = reinterpret_cast<const uint4*>(qh + (size_t)kept_t[i] * D);
      reinterpret_cast<uint4*>(qsel + (row0 + kept_pos[i]) * D)[v] = __ldg(src + v);
    }
  }

  // padding rows of the head's block and the -1 tail of kept_out
  if (rank == 0) {
    for (int i = nk + tid; i < nkp; i += blockDim.x) {
      qinv[row0 + i] = 0.f;
      qbias[row0 + i] = -INFINITY;
      uint4* dst = reinterpret_cast<uint4*>(qsel + (row0 + i) * D);
      for (int v = 0; v < D * (int)sizeof(T) / 16; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (kept_out)
      for (int i = nk + tid; i < nq; i += blockDim.x) kept_out[(size_t)bh * nq + i] = -1;
  }
}

}  // namespace quoka
