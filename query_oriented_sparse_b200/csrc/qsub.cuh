// K1: query subselection (QUOKA page, method summary and Figure 1(b): the chunk's
// queries are filtered by cosine dissimilarity to their mean; Figure 2: queries far
// from the mean interact with more keys).
//
// One thread-block cluster of CS CTAs per (sequence, query head); CTA r owns a contiguous
// slice of at most QSUB_MAX_ROWS chunk positions.  The call takes the smallest CS that
// covers the chunk and doubles it while the clusters of all heads still fit the SMs at
// once, so a long chunk of few heads spreads over 8 SMs and many short heads each run on
// one (the select's latency chain then runs once per SM, not once per wave of clusters).  Rows are read eight lanes to a row (a warp
// takes four rows per step, each lane one or more 16-byte vectors), several steps in
// flight per warp, so a row's reductions are three shuffles wide instead of a serial
// five-shuffle chain per row.
//   pass 1  |q_t| and the sum of unit queries over this CTA's slice; the CTAs' partial
//           sums meet through distributed shared memory (in rank order, so the mean
//           direction is the same on every CTA);
//   pass 2  re-reads the slice (L2-resident) for c_t = cos(q_t, mean) as orderable keys,
//           stored at their chunk position in a chunk-wide key array;
//   select  after one cluster barrier every CTA copies the other CTAs' keys into its own
//           array (the whole chunk is at most 32 KB of keys) and runs the radix select of
//           the Nk smallest (ties to the lower t) locally, with block barriers only
//           (cluster_select.cuh); each CTA emits the kept positions of its own slice.
// The kept rows are copied (raw values) into the per-KV-head operand block of the scoring
// GEMM with their fp32 1/|q| and a column bias; each head's block is padded to nkp rows
// (a multiple of 16) with zero rows whose bias is -inf, so a padded column can never win
// the max pooling.
#pragma once
#include "cluster_select.cuh"

namespace quoka {

constexpr int QSUB_MAX_CS = 8;                // CTAs per query head at most
constexpr int QSUB_THREADS = 512;
constexpr int QSUB_WARPS = QSUB_THREADS / 32;
constexpr int QSUB_MAX_ROWS = (QUOKA_MAX_CHUNK + QSUB_MAX_CS - 1) / QSUB_MAX_CS;   // chunk positions per CTA
constexpr int QSUB_LPR = 8;                   // lanes per query row
constexpr int QSUB_RPS = 32 / QSUB_LPR;       // rows per warp step
constexpr int QSUB_PULL = (QUOKA_MAX_CHUNK + QSUB_THREADS - 1) / QSUB_THREADS;   // keys pulled per thread

// Per-lane view of a row: NV 16-byte vectors, vector v of lane l8 holding elements
// [(8 v + l8) VE, (8 v + l8 + 1) VE).  U steps are in flight per warp (16 registers of
// raw row data per lane, which keeps two 512-thread CTAs per SM without spills).
template <typename T, int D>
struct QsubShape {
  static constexpr int VE = 16 / (int)sizeof(T);
  static constexpr int NV = D / (QSUB_LPR * VE);
  static constexpr int EPL = NV * VE;
  static constexpr int U = NV >= 4 ? 1 : 4 / NV;
  static_assert(NV * QSUB_LPR * VE == D, "row width must be a multiple of 8 vectors");
};

template <typename T> struct Unpack;
template <> struct Unpack<__nv_bfloat16> {
  __device__ static __forceinline__ void run(const uint4& r, float* x) {
    const unsigned int w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      unsigned int wi = w[i];
      const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wi));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
};
template <> struct Unpack<float> {
  __device__ static __forceinline__ void run(const uint4& r, float* x) {
    x[0] = __uint_as_float(r.x); x[1] = __uint_as_float(r.y);
    x[2] = __uint_as_float(r.z); x[3] = __uint_as_float(r.w);
  }
};

__device__ __forceinline__ float group8_sum(float v) {   // sum over the 8 lanes of a row
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}

template <typename T, int D, int CS>
__global__ void __cluster_dims__(CS, 1, 1) __launch_bounds__(QSUB_THREADS, 2)
qsub_kernel(const T* __restrict__ q, int C, int nk, int nkp, int nq,
            int32_t* __restrict__ kept_out, T* __restrict__ qsel, float* __restrict__ qinv,
            float* __restrict__ qbias) {
  using Sh = QsubShape<T, D>;
  constexpr int VE = Sh::VE, NV = Sh::NV, EPL = Sh::EPL, U = Sh::U;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float inv[QSUB_MAX_ROWS];
  __shared__ float part[QSUB_WARPS][D];
  __shared__ float cta_sum[D];
  __shared__ float mdir[D];
  __shared__ float mscale_s;
  __shared__ SelectSmem sm;
  __shared__ int kept_pos[QSUB_MAX_ROWS], kept_t[QSUB_MAX_ROWS];
  __shared__ int n_kept;
  extern __shared__ uint32_t keys[];          // C entries: c_t keys at chunk position t

  const int rank = (int)cluster.block_rank();
  const int bh = blockIdx.x / CS;             // b * h_q + h
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 3, l8 = lane & 7;
  const int S = (C + CS - 1) / CS;            // <= QSUB_MAX_ROWS (the call picks CS so)
  const int lo = min(C, rank * S), hi = min(C, lo + S);
  const int n = hi - lo;
  const T* qh = q + (size_t)bh * C * D;

  // Row step u of this CTA covers rows lo + 4u .. lo + 4u + 3; warp w takes steps
  // w, w + 16, ...; lanes beyond the slice load zeros and take part in the shuffles.
  auto load_steps = [&](int u0, uint4 (&raw)[U][NV]) {
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int r = (u0 + i * QSUB_WARPS) * QSUB_RPS + g;
      const uint4* src = reinterpret_cast<const uint4*>(qh + (size_t)(lo + r) * D);
#pragma unroll
      for (int v = 0; v < NV; ++v)
        raw[i][v] = r < n ? __ldg(src + v * QSUB_LPR + l8) : make_uint4(0u, 0u, 0u, 0u);
    }
  };

  // pass 1: norms and the sum of unit queries over this CTA's slice
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  for (int u0 = warp; u0 * QSUB_RPS < n; u0 += QSUB_WARPS * U) {
    uint4 raw[U][NV];
    load_steps(u0, raw);
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int r = (u0 + i * QSUB_WARPS) * QSUB_RPS + g;
      float ss = 0.f;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float x[VE];
        Unpack<T>::run(raw[i][v], x);
#pragma unroll
        for (int e = 0; e < VE; ++e) ss = fmaf(x[e], x[e], ss);
      }
      ss = group8_sum(ss);
      const float nrm = sqrtf(ss);
      const float iv = nrm > 0.f ? 1.0f / nrm : 0.f;
      if (r < n) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          float x[VE];
          Unpack<T>::run(raw[i][v], x);
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[v * VE + e] = fmaf(x[e], iv, acc[v * VE + e]);
        }
        if (l8 == 0) inv[r] = iv;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) {             // the warp's four row groups, fixed order
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  }
  if (g == 0) {
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
      for (int e = 0; e < VE; ++e) part[warp][(v * QSUB_LPR + l8) * VE + e] = acc[v * VE + e];
  }
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
    for (int r = 0; r < CS; ++r) s += cluster.map_shared_rank(cta_sum, r)[tid];
    mdir[tid] = s;
  }
  cluster_arrive();                            // remote reads of cta_sum done; waited below
  __syncthreads();
  if (warp == 0) {
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s = fmaf(mdir[d], mdir[d], s);
    s = warp_sum(s);
    if (lane == 0) mscale_s = s > 0.f ? 1.0f / sqrtf(s) : 0.f;
  }
  __syncthreads();
  const float mscale = mscale_s;

  // pass 2: c_t = (q_t . m) / (|q_t| |m|) as ascending-orderable keys
  float mv[EPL];
#pragma unroll
  for (int v = 0; v < NV; ++v)
#pragma unroll
    for (int e = 0; e < VE; ++e) mv[v * VE + e] = mdir[(v * QSUB_LPR + l8) * VE + e];
  for (int u0 = warp; u0 * QSUB_RPS < n; u0 += QSUB_WARPS * U) {
    uint4 raw[U][NV];
    load_steps(u0, raw);
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int r = (u0 + i * QSUB_WARPS) * QSUB_RPS + g;
      float dot = 0.f;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float x[VE];
        Unpack<T>::run(raw[i][v], x);
#pragma unroll
        for (int e = 0; e < VE; ++e) dot = fmaf(x[e], mv[v * VE + e], dot);
      }
      dot = group8_sum(dot);
      if (r < n && l8 == 0) keys[lo + r] = float_to_ordered(dot * inv[r] * mscale);
    }
  }
  cluster_wait();

  // keep the nk smallest (all of them when nk >= C), emitted in ascending t
  const size_t row0 = (size_t)bh * nkp;       // == ((b*h_kv + g)*G + h%G) * nkp
  if (tid == 0) n_kept = 0;
  __syncthreads();
  auto emit = [&](int pos, int t) {
    if (t < lo || t >= hi) return;            // another CTA's position
    if (pos >= nk) { flag_error(ERR_BAD_INDEX); return; }   // unreachable when counts agree
    qinv[row0 + pos] = inv[t - lo];
    qbias[row0 + pos] = 0.f;
    if (kept_out) kept_out[(size_t)bh * nq + pos] = t;
    const int slot = atomicAdd(&n_kept, 1);   // rows are copied below, coalesced
    kept_pos[slot] = pos;
    kept_t[slot] = t;
  };
  const bool select = nk < C;
  if (!select) {
    for (int t = lo + tid; t < hi; t += blockDim.x) emit(t, t);
  } else {
    cluster.sync();                            // every CTA's keys are final
    // all remote loads in flight before any store; 16-byte pulls when every CTA's slice
    // starts on a 16-byte boundary (C a multiple of 32), else 4-byte ones
    if ((S & 3) == 0 && (C & 3) == 0) {
      constexpr int PULL4 = (QSUB_PULL + 3) / 4;
      uint4 v[PULL4];
#pragma unroll
      for (int i = 0; i < PULL4; ++i) {
        const int t = (tid + i * QSUB_THREADS) * 4;
        v[i] = (t < C && t / S != rank)
                   ? *reinterpret_cast<const uint4*>(cluster.map_shared_rank(keys, t / S) + t)
                   : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < PULL4; ++i) {
        const int t = (tid + i * QSUB_THREADS) * 4;
        if (t < C && t / S != rank) *reinterpret_cast<uint4*>(keys + t) = v[i];
      }
    } else {
      uint32_t v[QSUB_PULL];
#pragma unroll
      for (int i = 0; i < QSUB_PULL; ++i) {
        const int t = tid + i * QSUB_THREADS;
        v[i] = (t < C && t / S != rank) ? cluster.map_shared_rank(keys, t / S)[t] : 0u;
      }
#pragma unroll
      for (int i = 0; i < QSUB_PULL; ++i) {
        const int t = tid + i * QSUB_THREADS;
        if (t < C && t / S != rank) keys[t] = v[i];
      }
    }
    cluster_arrive();                          // remote reads of keys done; waited at the end
    __syncthreads();
    auto key_at = [&](int j) { return keys[j]; };
    const SelectThreshold th = block_threshold<false>(sm, key_at, C, nk);
    ordered_emit<false>(sm, key_at, 0, C, th, emit);
  }
  __syncthreads();
  {
    constexpr int VPR = D * (int)sizeof(T) / 16;   // 16-byte vectors per row
    const int nr = n_kept;
    for (int e = tid; e < nr * VPR; e += blockDim.x) {
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
  if (select) cluster_wait();                  // peers' last reads of this CTA's keys
}

}  // namespace quoka
