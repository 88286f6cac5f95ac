// Per-query sparse attention on tensor cores (QUILT page, summary: nearby queries are
// grouped, the key-value entries they selected in common are loaded once and reused, and
// the sharing is organised to fit the accelerator's tiles).
//
// A pair tile is the 256 query rows that one SM pair of the dense attention kernel
// serves: the G heads of a KV head at 2 x TP consecutive positions (TP = 128 / G), 128
// rows per CTA.  Its rows' key sets are merged into one union, the union's K/V rows are
// gathered once into a contiguous block, and the attention kernel runs dense S = Q K^T
// and P V MMAs over that block with a per-row membership mask in place of the causal
// rule: key u of the union counts for row r only if r's own set holds it.
//   perq_tc_union_kernel    one CTA per pair tile: a bitmap of the tile's positions over
//                           the sequence's rows in shared memory, an exclusive scan of
//                           its words' popcounts (the union, ascending, and each key's
//                           union rank), then per row a 128-bit mask per 128-key block of
//                           the union, built in shared memory and written out;
//   perq_tc_gather_kernel   the union's K and V rows into one block per pair tile, zero
//                           rows up to the next multiple of 128.
// The union of a tile holds at most `cap` keys (the caller's bound); a larger union sets
// the device error word and keeps its first `cap` keys.
#pragma once
#include "common.cuh"

namespace quoka {

constexpr int PTC_THREADS = 1024;
constexpr int PTC_MAX_WORDS = 8192;       // sequence bitmap: up to 262144 rows
constexpr int PTC_BATCH = 8;              // set entries a lane has in flight (scalar loads)
constexpr int PTC_BATCH4 = 8;             // 16-byte loads a lane has in flight (32 entries)

// Shared memory of the union kernel: the sequence bitmap, its word offsets, and one
// mask row per warp.
__host__ __device__ inline size_t perq_tc_union_smem(int cap) {
  const int mwords = (cap + 127) / 128 * 4;
  return (size_t)(2 * PTC_MAX_WORDS + (PTC_THREADS / 32) * mwords + 64) * 4;
}

// grid (pair tiles of the chunk, KV heads, sequences).  Row r of CTA rank k of pair
// tile pt: head r / TP, position 2 TP pt + k TP + r % TP (a padding row past G TP or C).
__global__ void __launch_bounds__(PTC_THREADS)
perq_tc_union_kernel(const int32_t* __restrict__ sel, const __grid_constant__ SeqTable tab, int h_q,
                     int h_kv, int C, int S, int TP, int cap, int32_t* __restrict__ uni,
                     int32_t* __restrict__ ucount, uint32_t* __restrict__ mask) {
  extern __shared__ __align__(16) uint32_t ptc_sm[];
  uint32_t* bm = ptc_sm;                                       // [PTC_MAX_WORDS]
  int* roff = reinterpret_cast<int*>(ptc_sm + PTC_MAX_WORDS);  // [PTC_MAX_WORDS]
  const int mwords = (cap + 127) / 128 * 4;
  uint32_t* mrow = ptc_sm + 2 * PTC_MAX_WORDS;                 // [warps][mwords]
  int* sbuf = reinterpret_cast<int*>(mrow + (PTC_THREADS / 32) * mwords);   // [64]
  const int pt = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int npt = gridDim.x;
  const int G = h_q / h_kv;
  const long long N = tab.kv_off[b + 1] - tab.kv_off[b];
  const int W = (int)((N + 31) / 32);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t tile = ((size_t)b * h_kv + g) * npt + pt;

  auto row_of = [&](int rr, int& head, int& pos) -> bool {   // pair-tile row -> (head, position)
    const int k = rr >> 7, r = rr & 127;
    head = r / TP;
    pos = 2 * TP * pt + k * TP + r % TP;
    return head < G && pos < C;
  };

  // every entry of a set row, handed to fn one by one with many loads in flight per lane:
  // 16-byte loads when the rows are 16-byte aligned (S a multiple of 4), else 4-byte ones
  auto for_set = [&](const int32_t* srow, auto&& fn) {
    if ((S & 3) == 0) {
      const int4* s4 = reinterpret_cast<const int4*>(srow);
      const int S4 = S >> 2;
      for (int i0 = 0; i0 < S4; i0 += 32 * PTC_BATCH4) {
        int4 x[PTC_BATCH4];                                    // all loads in flight first
#pragma unroll
        for (int u = 0; u < PTC_BATCH4; ++u) {
          const int i = i0 + u * 32 + lane;
          x[u] = i < S4 ? __ldg(s4 + i) : make_int4(-1, -1, -1, -1);
        }
#pragma unroll
        for (int u = 0; u < PTC_BATCH4; ++u) {
          fn(x[u].x);
          fn(x[u].y);
          fn(x[u].z);
          fn(x[u].w);
        }
      }
    } else {
      for (int i0 = 0; i0 < S; i0 += 32 * PTC_BATCH) {
        int x[PTC_BATCH];
#pragma unroll
        for (int u = 0; u < PTC_BATCH; ++u) {
          const int i = i0 + u * 32 + lane;
          x[u] = i < S ? __ldg(srow + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < PTC_BATCH; ++u) fn(x[u]);
      }
    }
  };

  for (int w = tid; w < W; w += PTC_THREADS) bm[w] = 0u;
  __syncthreads();
  // a warp per row; a bit already set (most of them, when rows share their keys) costs a
  // shared-memory read instead of an atomic
  for (int rr = warp; rr < 256; rr += PTC_THREADS / 32) {
    int head, pos;
    if (!row_of(rr, head, pos)) continue;
    const int32_t* srow = sel + (((size_t)b * h_q + (size_t)g * G + head) * C + pos) * S;
    for_set(srow, [&](int x) {
      if (x < 0) return;
      if (x >= N) { flag_error(ERR_BAD_INDEX); return; }
      const uint32_t bit = 1u << (x & 31);
      if (!(bm[x >> 5] & bit)) atomicOr(&bm[x >> 5], bit);
    });
  }
  __syncthreads();
  // exclusive scan of the words' popcounts (each thread a contiguous run of words)
  const int per = (W + PTC_THREADS - 1) / PTC_THREADS;
  const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
  int mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bm[w]);
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sbuf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = sbuf[lane];                                  // 32 warps
    int iv = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, iv, o);
      if (lane >= o) iv += y;
    }
    sbuf[32 + lane] = iv - v;                                  // exclusive warp offsets
    if (lane == 31) sbuf[0] = iv;                              // total (after the reads above)
  }
  __syncthreads();
  const int total = sbuf[0];
  {
    int off = sbuf[32 + warp] + incl - mine;
    for (int w = w0; w < w1; ++w) { roff[w] = off; off += __popc(bm[w]); }
  }
  const int nu = min(total, cap);
  if (tid == 0) {
    ucount[tile] = nu;
    if (total > cap) flag_error(ERR_UNION_CAP);
  }
  __syncthreads();
  // the union, ascending
  int32_t* U = uni + tile * (size_t)cap;
  for (int w = tid; w < W; w += PTC_THREADS) {
    uint32_t bits = bm[w];
    int k = roff[w];
    while (bits && k < nu) {
      const int j = __ffs(bits) - 1;
      bits &= bits - 1u;
      U[k++] = w * 32 + j;
    }
  }
  // per row: bit (block, key within block) of every union key the row's set holds;
  // a warp builds one row at a time in its shared-memory row
  uint32_t* my = mrow + warp * mwords;
  for (int rr = warp; rr < 256; rr += PTC_THREADS / 32) {
    for (int w = lane; w < mwords; w += 32) my[w] = 0u;
    __syncwarp();
    int head, pos;
    if (row_of(rr, head, pos)) {
      const int32_t* srow = sel + (((size_t)b * h_q + (size_t)g * G + head) * C + pos) * S;
      for_set(srow, [&](int x) {
        if (x < 0 || x >= N) return;
        const uint32_t word = bm[x >> 5];
        const int rank = roff[x >> 5] + __popc(word & ((1u << (x & 31)) - 1u));
        if (rank < nu) atomicOr(&my[rank >> 5], 1u << (rank & 31));
      });
    }
    __syncwarp();
    uint32_t* dst = mask + (tile * 256 + rr) * (size_t)mwords;
    for (int w = lane; w < mwords; w += 32) dst[w] = my[w];
    __syncwarp();
  }
}

// The union's K/V rows of every pair tile into blocks of `stride` rows (ascending union
// order), zero rows up to the next multiple of 128.  Grid (tiles, copiers per tile); each
// CTA strides over its tile's 16-byte vectors.
template <int VPR>
__global__ void __launch_bounds__(256)
perq_tc_gather_kernel(const uint4* __restrict__ k_cache, const uint4* __restrict__ v_cache,
                      long long rows_per_head, const __grid_constant__ SeqTable tab, int h_kv, int npt,
                      int cap, long long stride, const int32_t* __restrict__ uni,
                      const int32_t* __restrict__ ucount, uint4* __restrict__ kc, uint4* __restrict__ vc) {
  const int tile = blockIdx.x;
  const int nu = __ldg(ucount + tile);
  const int nrow = (nu + 127) / 128 * 128;                     // rows the attention reads
  const int bg = tile / npt;
  const int b = bg / h_kv, g = bg - b * h_kv;
  const long long src0 = (long long)g * rows_per_head + tab.kv_off[b];
  const int32_t* U = uni + (size_t)tile * cap;
  uint4* kt = kc + (size_t)tile * stride * VPR;
  uint4* vt = vc + (size_t)tile * stride * VPR;
  for (int e = blockIdx.y * blockDim.x + threadIdx.x; e < nrow * VPR; e += gridDim.y * blockDim.x) {
    const int i = e / VPR, v = e - (e / VPR) * VPR;            // VPR is a power of two
    if (i >= nu) {
      kt[e] = make_uint4(0u, 0u, 0u, 0u);
      vt[e] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const long long src = (src0 + __ldg(U + i)) * VPR + v;
    kt[e] = __ldg(k_cache + src);
    vt[e] = __ldg(v_cache + src);
  }
}

}  // namespace quoka
