// K3: per-KV-head top-B of the pooled key scores, ties to the lower index, output in
// ascending index order (QUOKA page, Figure 1(a): the KV cache is sub-selected into a
// compacted cache before dense attention).
//
// One thread-block cluster of CS CTAs per (sequence, KV head); CTA r owns a contiguous
// slice of the prefix.  CS is 16 (a non-portable cluster size, opted into at launch) unless
// the rows' clusters would not all fit the SMs at once (one CTA per SM: 73 registers per
// thread): then it halves, down to 4, while a CTA's slice still fits its staging area, so
// many rows run in one wave of clusters instead of several, each wave paying the whole
// radix select's latency.  The exact B-th largest score is found by a cluster
// radix select over orderable score keys and the kept indices are emitted in index
// order (cluster_select.cuh), so the result is deterministic and sorted without a sort.
// Each CTA first stages its slice's keys in shared memory (coalesced, sixteen loads in
// flight per thread), so the radix passes never wait on L2; slices longer than the
// staging area read their keys from global memory instead.
// When the scoring kernel split a KV head's kept queries into several column groups, a
// first pass adds the groups' partial sums (in group order) and applies 1/G.
#pragma once
#include "cluster_select.cuh"

namespace quoka {

constexpr int TOPK_MAX_CS = 16;               // CTAs per (sequence, KV head) at most
constexpr int TOPK_THREADS = 512;
constexpr int TOPK_STAGE_KEYS = 49152;         // keys staged per CTA (192 KB)
constexpr int TOPK_STAGE_UNROLL = 16;          // staging loads in flight per thread

template <int CS>
__global__ void __cluster_dims__(CS, 1, 1) __launch_bounds__(TOPK_THREADS)
topk_kernel(float* __restrict__ pooled, long long pooled_stride, int ncg, long long cg_stride,
            float inv_G, const __grid_constant__ SeqTable tab, int h_kv, int b_max,
            int32_t* __restrict__ idx_out) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ SelectSmem sm;
  extern __shared__ uint32_t staged[];         // TOPK_STAGE_KEYS entries when used

  const int rank = (int)cluster.block_rank();
  const int head = blockIdx.x / CS;            // b * h_kv + g
  const int b = head / h_kv;
  const int P = tab.prefix[b], B = tab.nsel[b];
  int32_t* out = idx_out + (size_t)head * b_max;
  float* sc = pooled + (size_t)head * pooled_stride;
  const int stride = CS * blockDim.x;

  if (ncg > 1) {                               // sum the column groups' partial scores
    for (int j = rank * blockDim.x + threadIdx.x; j < P; j += stride) {
      float s = sc[j];
      for (int c = 1; c < ncg; ++c) s += sc[c * cg_stride + j];
      sc[j] = s * inv_G;
    }
    __threadfence();
    cluster.sync();
  }

  for (int i = B + rank * blockDim.x + threadIdx.x; i < b_max; i += stride) out[i] = -1;
  if (B >= P) {                                // keep every prefix key (P == 0 included)
    for (int i = rank * blockDim.x + threadIdx.x; i < P; i += stride) out[i] = i;
    return;                                    // uniform across the cluster: no DSMEM used
  }
  if (B == 0) return;

  const int S = (P + CS - 1) / CS;
  const int lo = min(P, rank * S), hi = min(P, lo + S);
  auto emit = [&](int pos, int j) {
    if (pos < B) out[pos] = j;
    else flag_error(ERR_BAD_INDEX);            // unreachable when the counts are consistent
  };
  if (hi - lo <= TOPK_STAGE_KEYS) {
    for (int j0 = lo + threadIdx.x; j0 < hi; j0 += TOPK_STAGE_UNROLL * blockDim.x) {
      float v[TOPK_STAGE_UNROLL];
#pragma unroll
      for (int u = 0; u < TOPK_STAGE_UNROLL; ++u) {
        const int j = j0 + u * blockDim.x;
        v[u] = j < hi ? sc[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < TOPK_STAGE_UNROLL; ++u) {
        const int j = j0 + u * blockDim.x;
        if (j < hi) staged[j - lo] = float_to_ordered(v[u]);
      }
    }
    __syncthreads();
    auto key_at = [&](int j) { return staged[j - lo]; };
    const SelectThreshold th = cluster_threshold<CS, true>(cluster, sm, key_at, lo, hi, B);
    ordered_emit<true>(sm, key_at, lo, hi, th, emit);
  } else {
    auto key_at = [sc](int j) { return float_to_ordered(sc[j]); };
    const SelectThreshold th = cluster_threshold<CS, true>(cluster, sm, key_at, lo, hi, B);
    ordered_emit<true>(sm, key_at, lo, hi, th, emit);
  }
  cluster_wait();                              // peers' last reads of this CTA's histograms
}

}  // namespace quoka
