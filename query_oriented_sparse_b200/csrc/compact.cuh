// Compaction of the selected K/V rows (QUOKA page, Figure 1(a): each chunk first
// sub-selects the KV cache into a compacted cache, which then goes into a dense
// attention kernel).
//
// For every (sequence b, KV head g) the compacted block holds, contiguously, the
// n_b = min(budget_b, P_b) selected prefix rows in index order followed by the chunk's
// own C rows (cache rows P_b .. P_b + C - 1), for K and for V:
//     Kc[(b * h_kv + g) * stride + i]   i < n_b + C,   stride = round_up(b_max + C, 128)
// and zeros in the block's remaining rows, so every 128-row tile the attention kernel
// loads lies inside one block and holds finite values (a masked key still meets its V
// row in the P.V product, where 0 * NaN would poison the output).
// In a whole-prompt prefill the chunk's rows are new: they are then read from
// k_new / v_new ([batch, h_kv, C, d] of this chunk) and written to the cache as well, so
// the cache append rides on the compaction pass (append_kv_kernel does it alone for the
// paths without compaction).
// The whole grid streams rows with 16-byte vector loads/stores (a warp moves two
// 256-byte rows per instruction), so the gather runs at HBM bandwidth on every SM.
#pragma once
#include "common.cuh"

namespace quoka {

constexpr int CPT_THREADS = 256;

template <int D>
__global__ void __launch_bounds__(CPT_THREADS)
compact_kv_kernel(const uint4* __restrict__ k_cache, const uint4* __restrict__ v_cache,
                  long long rows_per_head, const __grid_constant__ SeqTable tab, int h_kv, int C,
                  int b_max, long long stride, const int32_t* __restrict__ idx,
                  uint4* __restrict__ kc, uint4* __restrict__ vc, long long total_vecs,
                  const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                  uint4* __restrict__ k_app, uint4* __restrict__ v_app) {
  constexpr int VPR = D * 2 / 16;                   // 16-byte vectors per row
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total_vecs;
       e += (long long)gridDim.x * blockDim.x) {
    const long long rowg = e / VPR;                 // global compacted row
    const int v = (int)(e - rowg * VPR);
    const long long bg = rowg / stride;
    const int i = (int)(rowg - bg * stride);
    const int b = (int)(bg / h_kv), g = (int)(bg - (long long)b * h_kv);
    const int n = tab.nsel[b], P = tab.prefix[b];
    if (i >= n + C) {                               // padding rows of the block
      kc[e] = make_uint4(0u, 0u, 0u, 0u);
      vc[e] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    int r;
    if (i < n) {
      r = __ldg(idx + (size_t)bg * b_max + i);
      if (r < 0 || r >= P) { flag_error(ERR_BAD_INDEX); r = P; }
    } else if (k_new) {                             // a new chunk row: append it as well
      const long long src = ((long long)bg * C + (i - n)) * VPR + v;
      const long long dst = ((long long)g * rows_per_head + tab.kv_off[b] + P + (i - n)) * VPR + v;
      const uint4 kx = __ldg(k_new + src), vx = __ldg(v_new + src);
      k_app[dst] = kx;
      v_app[dst] = vx;
      kc[e] = kx;
      vc[e] = vx;
      continue;
    } else {
      r = P + (i - n);
    }
    const long long src = ((long long)g * rows_per_head + tab.kv_off[b] + r) * VPR + v;
    kc[e] = __ldg(k_cache + src);
    vc[e] = __ldg(v_cache + src);
  }
}

// The chunk's new K/V rows ([batch, h_kv, C, d]) into the cache at rows
// kv_off[b] + P_b + t of each KV head, 16-byte vectors.
__global__ void __launch_bounds__(CPT_THREADS)
append_kv_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                 uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, long long rows_per_head,
                 const __grid_constant__ SeqTable tab, int h_kv, int C, int vpr, long long total_vecs) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total_vecs;
       e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / vpr;                   // (b, g, t) of the new rows
    const int v = (int)(e - row * vpr);
    const int t = (int)(row % C);
    const long long bg = row / C;
    const int b = (int)(bg / h_kv), g = (int)(bg - (long long)b * h_kv);
    const long long dst = ((long long)g * rows_per_head + tab.kv_off[b] + tab.prefix[b] + t) * vpr + v;
    k_cache[dst] = __ldg(k_new + e);
    v_cache[dst] = __ldg(v_new + e);
  }
}

}  // namespace quoka
