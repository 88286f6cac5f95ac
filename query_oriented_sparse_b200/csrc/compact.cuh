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
                  uint4* __restrict__ kc, uint4* __restrict__ vc, long long total_vecs) {
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
    } else {
      r = P + (i - n);
    }
    const long long src = ((long long)g * rows_per_head + tab.kv_off[b] + r) * VPR + v;
    kc[e] = __ldg(k_cache + src);
    vc[e] = __ldg(v_cache + src);
  }
}

}  // namespace quoka
