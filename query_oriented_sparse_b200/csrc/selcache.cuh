// Selected-value cache with miss-only fetch (SQD page, the sparse-attention paragraph:
// the top-k choice keeps scanning the whole cache, attention runs over the chosen
// positions only, the chosen values are kept where attention runs and only the misses
// are sent, ahead of time).
//
// The cache is one block per (sequence, KV head) in the compacted-cache layout the
// attention kernels read: `stride` rows of K (then, in a second array, of V), whose
// slots 0 .. n-1 hold selected prefix rows, n .. n+C-1 the chunk's own rows, and zero
// rows up to the next multiple of 128.  slot_rows[b, g, s] names the cache row slot s
// holds (-1: none).  An update to a new selection keeps every row that is still chosen
// in its slot (a hit), and fetches only the rows that were not held (the misses) into
// the slots that fell free, in ascending row order into ascending free slots.
//
//   selcache_plan_kernel   one CTA per (KV head, sequence): a bitmap of the new
//                          selection in shared memory; each held slot clears its row's
//                          bit if set (hit) or is marked free; the remaining bits are
//                          the misses, matched in order to the free slots through
//                          prefix sums of the two bitmaps' popcounts.
//   selcache_copy_kernel   the misses' K/V rows, the chunk's rows and the zero rows,
//                          16-byte vectors, several CTAs per (sequence, KV head).
#pragma once
#include "common.cuh"

namespace quoka {

constexpr int SCP_THREADS = 512;

__device__ __forceinline__ int nth_set_bit(uint32_t w, int k) {
  for (int i = 0; i < k; ++i) w &= w - 1u;
  return __ffs(w) - 1;
}

// Block-wide exclusive scan of one value per thread (SCP_THREADS threads); returns the
// thread's offset and writes the total to *total.
__device__ __forceinline__ int scp_block_scan(int x, int* sbuf, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int v = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) sbuf[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < SCP_THREADS / 32 ? sbuf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sbuf[32 + lane] = w;                       // inclusive warp totals
  }
  __syncthreads();
  const int base = warp > 0 ? sbuf[32 + warp - 1] : 0;
  *total = sbuf[32 + SCP_THREADS / 32 - 1];
  __syncthreads();                             // sbuf reusable
  return base + v - x;
}

// Shared memory: row bitmap [rw], free-slot bitmap [fw], per-word offsets of both, scan
// scratch.
__host__ __device__ inline size_t selcache_plan_smem(int max_prefix, int b_max) {
  const int rw = (max_prefix + 31) / 32, fw = (b_max + 31) / 32;
  return (size_t)(2 * rw + 2 * fw + 64) * 4;
}

__global__ void __launch_bounds__(SCP_THREADS)
selcache_plan_kernel(const __grid_constant__ SeqTable tab, int h_kv, int b_max,
                     const int32_t* __restrict__ idx, int32_t* __restrict__ slot_rows,
                     int32_t* __restrict__ plan_slot, int32_t* __restrict__ plan_row,
                     int32_t* __restrict__ plan_count, int32_t* __restrict__ misses_out) {
  extern __shared__ __align__(16) uint32_t sm[];
  const int g = blockIdx.x, b = blockIdx.y;
  const int bg = b * h_kv + g;
  const int n = tab.nsel[b], P = tab.prefix[b];
  const int rw = (P + 31) / 32, fw = (n + 31) / 32;
  const int rw_max = (tab.max_prefix + 31) / 32, fw_max = (b_max + 31) / 32;
  uint32_t* rbits = sm;                                   // [rw_max]
  uint32_t* fbits = rbits + rw_max;                       // [fw_max]
  int* roff = reinterpret_cast<int*>(fbits + fw_max);     // [rw_max]
  int* foff = roff + rw_max;                              // [fw_max]
  int* sbuf = foff + fw_max;                              // [64]
  const int32_t* sel = idx + (size_t)bg * b_max;
  int32_t* slots = slot_rows + (size_t)bg * b_max;

  for (int w = threadIdx.x; w < rw; w += SCP_THREADS) rbits[w] = 0u;
  for (int w = threadIdx.x; w < fw; w += SCP_THREADS) fbits[w] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += SCP_THREADS) {
    const int r = __ldg(sel + i);
    if (r < 0 || r >= P) { flag_error(ERR_BAD_INDEX); continue; }
    atomicOr(&rbits[r >> 5], 1u << (r & 31));
  }
  __syncthreads();
  // held slots: a slot inside the live range keeps its row if the row is chosen again
  // (the first slot to claim a row wins, so a duplicated row is fetched only once);
  // every other slot of the range is free; slots past the range are emptied
  for (int s = threadIdx.x; s < b_max; s += SCP_THREADS) {
    const int r = slots[s];
    if (s < n) {
      bool hit = false;
      if (r >= 0 && r < P) {
        const uint32_t bit = 1u << (r & 31);
        hit = (atomicAnd(&rbits[r >> 5], ~bit) & bit) != 0u;
      }
      if (!hit) atomicOr(&fbits[s >> 5], 1u << (s & 31));
    } else if (r != -1) {
      slots[s] = -1;
    }
  }
  __syncthreads();
  // offsets of the misses (remaining row bits) and of the free slots, in ascending order
  int tot_m = 0, tot_f = 0;
  {
    const int per = (rw + SCP_THREADS - 1) / SCP_THREADS;
    const int w0 = threadIdx.x * per, w1 = min(rw, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(rbits[w]);
    int off = scp_block_scan(c, sbuf, &tot_m);
    for (int w = w0; w < w1; ++w) { roff[w] = off; off += __popc(rbits[w]); }
  }
  {
    const int per = (fw + SCP_THREADS - 1) / SCP_THREADS;
    const int w0 = threadIdx.x * per, w1 = min(fw, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(fbits[w]);
    int off = scp_block_scan(c, sbuf, &tot_f);
    for (int w = w0; w < w1; ++w) { foff[w] = off; off += __popc(fbits[w]); }
  }
  __syncthreads();
  if (tot_m != tot_f) {                       // only if the selection held bad indices
    if (threadIdx.x == 0) {
      flag_error(ERR_BAD_INDEX);
      plan_count[bg] = 0;
      if (misses_out) misses_out[bg] = 0;
    }
    return;
  }
  // the k-th miss (ascending row) goes to the k-th free slot (ascending slot)
  for (int w = threadIdx.x; w < rw; w += SCP_THREADS) {
    uint32_t bits = rbits[w];
    int k = roff[w];
    while (bits) {
      const int j = __ffs(bits) - 1;
      bits &= bits - 1u;
      int lo = 0, hi = fw - 1;                // last free word whose offset is <= k
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (foff[mid] <= k) lo = mid; else hi = mid - 1;
      }
      const int bit = lo >= 0 ? nth_set_bit(fbits[lo], k - foff[lo]) : -1;
      const int s = lo * 32 + bit;
      const int r = w * 32 + j;
      const bool good = bit >= 0 && s < n;     // always, when the counts agree
      if (!good) flag_error(ERR_BAD_INDEX);
      plan_slot[(size_t)bg * b_max + k] = good ? s : 0;
      plan_row[(size_t)bg * b_max + k] = good ? r : 0;
      if (good) slots[s] = r;
      ++k;
    }
  }
  if (threadIdx.x == 0) {
    plan_count[bg] = tot_m;
    if (misses_out) misses_out[bg] = tot_m;
  }
}

// Rows q of (sequence b, KV head g): q < M the planned misses, then the C chunk rows at
// slots n .. n+C-1, then zero rows up to the next multiple of 128.  Grid (copiers per
// (b, g), KV heads x sequences).
template <int VPR>
__global__ void __launch_bounds__(256)
selcache_copy_kernel(const uint4* __restrict__ k_cache, const uint4* __restrict__ v_cache,
                     long long rows_per_head, const __grid_constant__ SeqTable tab, int h_kv, int C,
                     int b_max, long long stride, const int32_t* __restrict__ plan_slot,
                     const int32_t* __restrict__ plan_row, const int32_t* __restrict__ plan_count,
                     uint4* __restrict__ kc, uint4* __restrict__ vc) {
  const int bg = blockIdx.y;
  const int b = bg / h_kv, g = bg - b * h_kv;
  const int n = tab.nsel[b], P = tab.prefix[b];
  const int M = plan_count[bg];
  const int nz = (int)(((long long)(n + C) + 127) / 128 * 128) - (n + C);
  const long long total = (long long)(M + C + nz) * VPR;
  const long long src0 = (long long)g * rows_per_head + tab.kv_off[b];
  const long long dst0 = (long long)bg * stride;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int q = (int)(e / VPR), v = (int)(e - (long long)q * VPR);
    if (q >= M + C) {
      const long long d = (dst0 + n + C + (q - M - C)) * VPR + v;
      kc[d] = make_uint4(0u, 0u, 0u, 0u);
      vc[d] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    int slot, row;
    if (q < M) {
      slot = __ldg(plan_slot + (size_t)bg * b_max + q);
      row = __ldg(plan_row + (size_t)bg * b_max + q);
    } else {
      slot = n + (q - M);
      row = P + (q - M);
    }
    const long long s = (src0 + row) * VPR + v;
    const long long d = (dst0 + slot) * VPR + v;
    kc[d] = __ldg(k_cache + s);
    vc[d] = __ldg(v_cache + s);
  }
}

// idx = 0, 1, ..., n - 1: the selected-value cache read as a cache whose selection is
// its own first n slots.
__global__ void iota_kernel(int32_t* __restrict__ out, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) out[i] = i;
}

}  // namespace quoka
