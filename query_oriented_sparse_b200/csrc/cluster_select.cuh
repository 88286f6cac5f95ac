// Cluster-wide exact selection of the k best of n 32-bit orderable keys, spread over the
// CTAs of one thread-block cluster (each CTA owns a contiguous index range [lo, hi)).
// Used for the per-KV-head top-B of pooled key scores (best = largest) and for the
// per-head query subselection (best = smallest cosine).  Ties go to the lower index.
//
//   cluster_threshold  4 passes of an 8-bit radix select.  Each CTA builds a shared
//                      histogram of its keys that match the digits fixed so far
//                      (warp-aggregated: one shared atomic per distinct bin per warp),
//                      the cluster sums histograms through distributed shared memory
//                      (double-buffered, one cluster barrier per pass) and every CTA
//                      takes the same digit decision.  Result: the k-th best key T and
//                      how many keys equal to T belong to the k best.
//   cluster_emit       counts of keys better than / equal to T per CTA are exchanged,
//                      then each CTA walks its range in index order with block scans
//                      and calls emit(position, index) for every selected key, so the
//                      output is in ascending index order without any sort.
#pragma once
#include <cooperative_groups.h>
#include "common.cuh"

namespace quoka {

namespace cg = cooperative_groups;

struct ClusterSelectSmem {
  int hist[2][256];
  int tots[256];
  int counts[2];
  int scan[33];
  int misc[4];
};

template <bool BEST_IS_LARGEST>
__device__ __forceinline__ bool better(uint32_t a, uint32_t b) {
  return BEST_IS_LARGEST ? a > b : a < b;
}

// Every thread of every CTA in the cluster must call it with the same k and n total.
template <int CS, bool BEST_IS_LARGEST, typename KeyFn>
__device__ void cluster_threshold(cg::cluster_group& cl, ClusterSelectSmem& sm, KeyFn key_at,
                                  int lo, int hi, int k, uint32_t* thr_out, int* need_eq_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  for (int pass = 0; pass < 4; ++pass) {
    int* hcur = sm.hist[pass & 1];
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += blockDim.x) hcur[i] = 0;
    __syncthreads();
    for (int base = lo; base < hi; base += blockDim.x) {
      const int j = base + tid;
      int bin = -1;
      if (j < hi) {
        const uint32_t key = key_at(j);
        if ((key & mask) == prefix) bin = (int)((key >> shift) & 255u);
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hcur[bin], __popc(peers));
    }
    cl.sync();
    if (tid < 256) {
      int s = 0;
#pragma unroll
      for (int r = 0; r < CS; ++r) s += cl.map_shared_rank(hcur, r)[tid];
      sm.tots[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      // lane L owns 8 bins in best-first order: bins 255-8L.. (largest first) or 8L..
      int c[8], s = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int bin = BEST_IS_LARGEST ? 255 - 8 * lane - q : 8 * lane + q;
        c[q] = sm.tots[bin];
        s += c[q];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - s;
      if (excl < k && k <= incl) {
        int run = excl, pick = 7;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run + c[q] >= k) { pick = q; break; }
          run += c[q];
        }
        sm.misc[0] = BEST_IS_LARGEST ? 255 - 8 * lane - pick : 8 * lane + pick;
        sm.misc[1] = run;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)sm.misc[0] << shift;
    mask |= 0xFFu << shift;
    k -= sm.misc[1];
    __syncthreads();
  }
  *thr_out = prefix;
  *need_eq_out = k;
}

// Calls emit(pos, j) for each selected index j of this CTA's range, pos being its rank
// among all selected indices of the cluster (ascending index order).  Ends with a
// cluster barrier after the last remote access, so CTAs may exit independently.
template <int CS, bool BEST_IS_LARGEST, typename KeyFn, typename EmitFn>
__device__ void cluster_emit(cg::cluster_group& cl, ClusterSelectSmem& sm, KeyFn key_at, int lo,
                             int hi, uint32_t thr, int need_eq, EmitFn emit) {
  const int tid = threadIdx.x;
  const int rank = (int)cl.block_rank();
  int c_better = 0, c_eq = 0;
  for (int j = lo + tid; j < hi; j += blockDim.x) {
    const uint32_t key = key_at(j);
    c_better += better<BEST_IS_LARGEST>(key, thr);
    c_eq += key == thr;
  }
  int tb, te;
  block_exclusive_scan(c_better, sm.scan, &tb);
  block_exclusive_scan(c_eq, sm.scan, &te);
  if (tid == 0) { sm.counts[0] = tb; sm.counts[1] = te; }
  cl.sync();
  if (tid == 0) {
    int eq_before = 0, sel_before = 0;
    for (int r = 0; r < rank; ++r) {
      const int* rc = cl.map_shared_rank(sm.counts, r);
      sel_before += rc[0] + max(0, min(need_eq - eq_before, rc[1]));
      eq_before += rc[1];
    }
    sm.misc[2] = eq_before;
    sm.misc[3] = sel_before;
  }
  cl.sync();
  int run_eq = sm.misc[2], run_sel = sm.misc[3];
  for (int base = lo; base < hi; base += blockDim.x) {
    const int j = base + tid;
    const bool valid = j < hi;
    const uint32_t key = valid ? key_at(j) : 0u;
    const int is_eq = (valid && key == thr) ? 1 : 0;
    int tot_eq;
    const int eq_rank = block_exclusive_scan(is_eq, sm.scan, &tot_eq) + run_eq;
    const int is_sel =
        (valid && (better<BEST_IS_LARGEST>(key, thr) || (is_eq && eq_rank < need_eq))) ? 1 : 0;
    int tot_sel;
    const int pos = block_exclusive_scan(is_sel, sm.scan, &tot_sel) + run_sel;
    if (is_sel) emit(pos, j);
    run_eq += tot_eq;
    run_sel += tot_sel;
  }
}

}  // namespace quoka
