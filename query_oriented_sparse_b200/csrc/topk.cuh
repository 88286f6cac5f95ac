// K3: per-KV-head top-B of the pooled key scores, ties to the lower index, output in
// ascending index order (QUOKA page, Figure 1(a): the KV cache is sub-selected into a
// compacted cache before dense attention).
//
// One thread-block cluster of TOPK_CS CTAs per (sequence, KV head); CTA r owns a
// contiguous slice of the prefix.  A 4-pass, 8-bit radix select over orderable score
// keys finds the B-th largest key T exactly: each pass builds a shared-memory
// histogram of the slice, the cluster's histograms are summed through distributed
// shared memory (double-buffered, one cluster barrier per pass), and every CTA takes
// the same digit decision.  Keys above T are kept, plus the lowest-index keys equal
// to T; a cluster exchange of per-slice counts and block scans give each kept index
// its output slot, so the result is deterministic and sorted without a sort.
// When the scoring kernel split a KV head's kept queries into several column groups,
// a first pass adds the groups' partial sums (in group order) and applies 1/G.
#pragma once
#include <cooperative_groups.h>
#include "common.cuh"

namespace quoka {

namespace cg = cooperative_groups;

constexpr int TOPK_CS = 8;
constexpr int TOPK_THREADS = 512;

__global__ void __cluster_dims__(TOPK_CS, 1, 1) __launch_bounds__(TOPK_THREADS)
topk_kernel(float* __restrict__ pooled, long long pooled_stride, int ncg, long long cg_stride,
            float inv_G, const __grid_constant__ SeqTable tab, int h_kv, int b_max,
            int32_t* __restrict__ idx_out) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ int hist[2][256];
  __shared__ int tots[256];
  __shared__ int counts[2];
  __shared__ int scan_scratch[33];
  __shared__ int misc[4];

  const int rank = (int)cluster.block_rank();
  const int head = blockIdx.x / TOPK_CS;       // b * h_kv + g
  const int b = head / h_kv;
  const int P = tab.prefix[b], B = tab.nsel[b];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* out = idx_out + (size_t)head * b_max;
  float* sc = pooled + (size_t)head * pooled_stride;
  const int stride = TOPK_CS * blockDim.x;

  if (ncg > 1) {                               // sum the column groups' partial scores
    for (int j = rank * blockDim.x + threadIdx.x; j < P; j += stride) {
      float s = sc[j];
      for (int c = 1; c < ncg; ++c) s += sc[c * cg_stride + j];
      sc[j] = s * inv_G;
    }
    __threadfence();
    cluster.sync();
  }

  for (int i = B + rank * blockDim.x + tid; i < b_max; i += stride) out[i] = -1;
  if (B >= P) {                                // keep every prefix key (P == 0 included)
    for (int i = rank * blockDim.x + tid; i < P; i += stride) out[i] = i;
    return;                                    // uniform across the cluster: no DSMEM used
  }
  if (B == 0) return;

  const int S = (P + TOPK_CS - 1) / TOPK_CS;
  const int lo = min(P, rank * S), hi = min(P, lo + S);

  uint32_t prefix = 0, mask = 0;
  int k = B;                                   // rank from the top among keys matching prefix
  for (int pass = 0; pass < 4; ++pass) {
    int* hcur = hist[pass & 1];
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += blockDim.x) hcur[i] = 0;
    __syncthreads();
    for (int j = lo + tid; j < hi; j += blockDim.x) {
      const uint32_t key = float_to_ordered(sc[j]);
      if ((key & mask) == prefix) atomicAdd(&hcur[(key >> shift) & 255u], 1);
    }
    cluster.sync();
    if (tid < 256) {
      int s = 0;
#pragma unroll
      for (int r = 0; r < TOPK_CS; ++r) s += cluster.map_shared_rank(hcur, r)[tid];
      tots[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {                           // lane L scans bins 255-8L .. 248-8L (descending)
      int c[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = tots[255 - 8 * lane - j]; s += c[j]; }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - s;
      if (excl < k && k <= incl) {
        int run = excl, digit = 248 - 8 * lane;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + c[j] >= k) { digit = 255 - 8 * lane - j; break; }
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
  const uint32_t thr = prefix;
  const int need_eq = k;

  // per-slice counts of keys above / equal to the threshold
  int c_gt = 0, c_eq = 0;
  for (int j = lo + tid; j < hi; j += blockDim.x) {
    const uint32_t key = float_to_ordered(sc[j]);
    c_gt += key > thr;
    c_eq += key == thr;
  }
  int tgt, teq;
  block_exclusive_scan(c_gt, scan_scratch, &tgt);
  block_exclusive_scan(c_eq, scan_scratch, &teq);
  if (tid == 0) { counts[0] = tgt; counts[1] = teq; }
  cluster.sync();
  if (tid == 0) {
    int eq_before = 0, sel_before = 0;
    for (int r = 0; r < rank; ++r) {
      const int* rc = cluster.map_shared_rank(counts, r);
      const int gt_r = rc[0], eq_r = rc[1];
      sel_before += gt_r + max(0, min(need_eq - eq_before, eq_r));
      eq_before += eq_r;
    }
    misc[2] = eq_before;
    misc[3] = sel_before;
  }
  cluster.sync();                              // remote reads finished before any CTA exits

  int run_eq = misc[2], run_sel = misc[3];
  for (int base = lo; base < hi; base += blockDim.x) {
    const int j = base + tid;
    const bool valid = j < hi;
    const uint32_t key = valid ? float_to_ordered(sc[j]) : 0u;
    const int is_eq = (valid && key == thr) ? 1 : 0;
    int tot_eq;
    const int eq_rank = block_exclusive_scan(is_eq, scan_scratch, &tot_eq) + run_eq;
    const int is_sel = (valid && (key > thr || (is_eq && eq_rank < need_eq))) ? 1 : 0;
    int tot_sel;
    const int pos = block_exclusive_scan(is_sel, scan_scratch, &tot_sel) + run_sel;
    if (is_sel) {
      if (pos < B) out[pos] = j;
      else flag_error(ERR_BAD_INDEX);          // unreachable when the counts are consistent
    }
    run_eq += tot_eq;
    run_sel += tot_sel;
  }
}

}  // namespace quoka
