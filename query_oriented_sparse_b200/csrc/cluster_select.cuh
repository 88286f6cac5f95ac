// Exact selection of the k best of n 32-bit orderable keys, ties to the lower index, the
// result emitted in ascending index order without a sort.  Used for the per-KV-head top-B
// of pooled key scores (best = largest) and for the per-head query subselection (best =
// smallest cosine).
//
//   cluster_threshold  keys spread over the CTAs of a thread-block cluster (each CTA owns a
//                      contiguous index range [lo, hi)).  4 passes of an 8-bit radix select:
//                      each CTA builds a shared histogram of its keys that match the digits
//                      fixed so far (plain shared atomics: on sm_100 they absorb same-bin
//                      conflicts far better than a __match_any_sync aggregation, which costs
//                      an order of magnitude more once a warp's keys spread over many bins);
//                      after one cluster barrier per pass every CTA reads all histograms
//                      through distributed shared memory (double-buffered; the idle buffer
//                      is cleared in the same step) and every warp takes the same digit
//                      decision.  The same reads give, per pass, how many keys of lower-
//                      ranked CTAs fall in bins better than the chosen digit; summed over the
//                      passes that is this CTA's output offset, so emitting needs no further
//                      exchange.  The passes stop early once the chosen bin holds exactly the
//                      keys still to be selected: every key of that bin is selected, so the
//                      bits below cannot matter (keys are then compared under the mask of
//                      the bits fixed so far).  Ends with a cluster barrier arrive after its
//                      last remote read: the caller waits (cluster_wait) before it exits.
//   block_threshold    all n keys in this CTA's shared memory: the same passes with one
//                      block barrier each (three histogram buffers, so clearing the next one
//                      never races a slow warp's decision).
//   ordered_emit       each warp walks a contiguous sub-range of [lo, hi) in index order
//                      with ballots (a count walk, one block barrier for the warp offsets,
//                      an emit walk) and calls emit(position, index) for every selected key.
#pragma once
#include <cooperative_groups.h>
#include "common.cuh"

namespace quoka {

namespace cg = cooperative_groups;

struct SelectSmem {
  __align__(16) int hist[3][256];
  __align__(16) int tots[256];    // cluster total per bin (current pass)
  __align__(16) int bef[256];     // per bin: keys of lower-ranked CTAs (current pass)
  int wcnt[2][32];                // per warp: keys better than / equal to the threshold
};

// The k-th best key thr and this CTA's share of the selection: with keys compared under
// mask (the bits the radix passes fixed), the selected keys are those better than thr and,
// in index order, the first eq_left of this CTA's keys equal to thr.
struct SelectThreshold {
  uint32_t thr;
  uint32_t mask;
  int sel_before;                 // selected keys before this CTA's range
  int eq_left;
};

template <bool BEST_IS_LARGEST>
__device__ __forceinline__ bool better(uint32_t a, uint32_t b) {
  return BEST_IS_LARGEST ? a > b : a < b;
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Eight consecutive ints of a 256-bin table in best-first order: lane L owns best-first
// positions 8L..8L+7, read as two 16-byte vectors (no bank conflicts).
template <bool BEST_IS_LARGEST>
__device__ __forceinline__ void load_bins8(const int* tab, int lane, int (&c)[8]) {
  const int base = BEST_IS_LARGEST ? 248 - 8 * lane : 8 * lane;
  const int4 a = *reinterpret_cast<const int4*>(tab + base);
  const int4 b = *reinterpret_cast<const int4*>(tab + base + 4);
  if (BEST_IS_LARGEST) {
    c[0] = b.w; c[1] = b.z; c[2] = b.y; c[3] = b.x; c[4] = a.w; c[5] = a.z; c[6] = a.y; c[7] = a.x;
  } else {
    c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
  }
}

// One warp's digit decision for the k-th best key from per-bin totals (and, when bef is
// given, per-bin counts of lower-ranked CTAs).  Every lane returns the digit, the number of
// keys in better bins (run), the chosen bin's count and, from bef, the lower ranks' keys in
// better bins (bb).
template <bool BEST_IS_LARGEST, bool WITH_BEF>
__device__ __forceinline__ void decide_digit(const int* tots, const int* bef, int k, int* digit,
                                             int* run_out, int* cnt_out, int* bb_out) {
  const int lane = threadIdx.x & 31;
  int c[8], e[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  load_bins8<BEST_IS_LARGEST>(tots, lane, c);
  if (WITH_BEF) load_bins8<BEST_IS_LARGEST>(bef, lane, e);
  int s = 0, eall = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    s += c[q];
    eall += e[q];
  }
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - s;
  const unsigned owners = __ballot_sync(0xffffffffu, excl < k && k <= incl);
  if (owners == 0u && threadIdx.x == 0) flag_error(ERR_BAD_INDEX);   // counts inconsistent
  const int owner = owners ? __ffs(owners) - 1 : 31;
  int run = excl, pick = 7, eb = 0, cnt = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (run + c[q] >= k) { pick = q; cnt = c[q]; break; }
    run += c[q];
    eb += e[q];
  }
  int bb = lane < owner ? eall : (lane == owner ? eb : 0);
  if (WITH_BEF) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bb += __shfl_xor_sync(0xffffffffu, bb, o);
  }
  pick = __shfl_sync(0xffffffffu, pick, owner);
  *run_out = __shfl_sync(0xffffffffu, run, owner);
  *cnt_out = __shfl_sync(0xffffffffu, cnt, owner);
  *bb_out = WITH_BEF ? bb : 0;
  const int pos = 8 * owner + pick;
  *digit = BEST_IS_LARGEST ? 255 - pos : pos;
}

// Every thread of every CTA of the cluster calls it with the same k and total n.
template <int CS, bool BEST_IS_LARGEST, typename KeyFn>
__device__ SelectThreshold cluster_threshold(cg::cluster_group& cl, SelectSmem& sm, KeyFn key_at,
                                             int lo, int hi, int k) {
  const int tid = threadIdx.x;
  const int rank = (int)cl.block_rank();
  for (int i = tid; i < 2 * 256; i += blockDim.x) (&sm.hist[0][0])[i] = 0;
  __syncthreads();
  uint32_t prefix = 0, mask = 0;
  int better_before = 0, eq_before = 0;
  for (int pass = 0; pass < 4; ++pass) {
    int* hcur = sm.hist[pass & 1];
    const int shift = 24 - 8 * pass;
    for (int j = lo + tid; j < hi; j += blockDim.x) {
      const uint32_t key = key_at(j);
      if ((key & mask) == prefix) atomicAdd(&hcur[(key >> shift) & 255u], 1);
    }
    cl.sync();                                   // every CTA's histogram of this pass is final
    if (tid < 256) {
      int tot = 0, bef = 0;
#pragma unroll
      for (int r = 0; r < CS; ++r) {
        const int v = cl.map_shared_rank(hcur, r)[tid];
        tot += v;
        bef += r < rank ? v : 0;
      }
      sm.tots[tid] = tot;
      sm.bef[tid] = bef;
      sm.hist[(pass + 1) & 1][tid] = 0;          // its remote readers passed the barrier above
    }
    __syncthreads();
    int digit, run, cnt, bb;
    decide_digit<BEST_IS_LARGEST, true>(sm.tots, sm.bef, k, &digit, &run, &cnt, &bb);
    better_before += bb;
    eq_before = sm.bef[digit];
    prefix |= (uint32_t)digit << shift;
    mask |= 0xFFu << shift;
    k -= run;
    if (cnt == k) break;                         // the whole bin is selected
  }
  cluster_arrive();                              // last remote read done
  SelectThreshold t;
  t.thr = prefix;
  t.mask = mask;
  t.sel_before = better_before + min(k, eq_before);
  t.eq_left = max(0, k - eq_before);
  return t;
}

// Every thread of the CTA calls it; key_at(j) for j in [0, n) reads this CTA's memory.
template <bool BEST_IS_LARGEST, typename KeyFn>
__device__ SelectThreshold block_threshold(SelectSmem& sm, KeyFn key_at, int n, int k) {
  const int tid = threadIdx.x;
  for (int i = tid; i < 256; i += blockDim.x) sm.hist[0][i] = 0;
  __syncthreads();
  uint32_t prefix = 0, mask = 0;
  for (int pass = 0; pass < 4; ++pass) {
    int* hcur = sm.hist[pass % 3];
    const int shift = 24 - 8 * pass;
    // the buffer of pass+1 was last read in the decision of pass-2, which every warp
    // finished before the previous barrier
    for (int i = tid; i < 256; i += blockDim.x) sm.hist[(pass + 1) % 3][i] = 0;
    for (int j = tid; j < n; j += blockDim.x) {
      const uint32_t key = key_at(j);
      if ((key & mask) == prefix) atomicAdd(&hcur[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    int digit, run, cnt, bb;
    decide_digit<BEST_IS_LARGEST, false>(hcur, nullptr, k, &digit, &run, &cnt, &bb);
    prefix |= (uint32_t)digit << shift;
    mask |= 0xFFu << shift;
    k -= run;
    if (cnt == k) break;                         // the whole bin is selected
  }
  SelectThreshold t;
  t.thr = prefix;
  t.mask = mask;
  t.sel_before = 0;
  t.eq_left = k;
  return t;
}

// Every thread of the CTA calls it.  Emits the selected keys of [lo, hi) with their output
// positions (t.sel_before + rank among the selected keys of [lo, hi)).
template <bool BEST_IS_LARGEST, typename KeyFn, typename EmitFn>
__device__ void ordered_emit(SelectSmem& sm, KeyFn key_at, int lo, int hi, const SelectThreshold& t,
                             EmitFn emit) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int per = (((hi - lo) + nw - 1) / nw + 31) & ~31;
  const int wlo = min(hi, lo + warp * per), whi = min(hi, wlo + per);
  int cb = 0, ce = 0;
  for (int base = wlo; base < whi; base += 32) {
    const int j = base + lane;
    const bool v = j < whi;
    const uint32_t key = v ? (key_at(j) & t.mask) : 0u;
    cb += __popc(__ballot_sync(0xffffffffu, v && better<BEST_IS_LARGEST>(key, t.thr)));
    ce += __popc(__ballot_sync(0xffffffffu, v && key == t.thr));
  }
  if (lane == 0) {
    sm.wcnt[0][warp] = cb;
    sm.wcnt[1][warp] = ce;
  }
  __syncthreads();
  int bw = lane < warp ? sm.wcnt[0][lane] : 0;   // counts of the warps before this one
  int ew = lane < warp ? sm.wcnt[1][lane] : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    bw += __shfl_xor_sync(0xffffffffu, bw, o);
    ew += __shfl_xor_sync(0xffffffffu, ew, o);
  }
  int pos = t.sel_before + bw + min(t.eq_left, ew);
  int eq_idx = ew;                               // keys equal to thr before this lane's round
  for (int base = wlo; base < whi; base += 32) {
    const int j = base + lane;
    const bool v = j < whi;
    const uint32_t key = v ? (key_at(j) & t.mask) : 0u;
    const bool eq = v && key == t.thr;
    const unsigned meq = __ballot_sync(0xffffffffu, eq);
    const bool sel = (v && better<BEST_IS_LARGEST>(key, t.thr)) ||
                     (eq && eq_idx + __popc(meq & lt) < t.eq_left);
    const unsigned msel = __ballot_sync(0xffffffffu, sel);
    if (sel) emit(pos + __popc(msel & lt), j);
    pos += __popc(msel);
    eq_idx += __popc(meq);
  }
}

}  // namespace quoka
