// Per-query sparse attention with shared-query loading (QUILT page, summary: nearby
// queries are grouped, the key-value entries they selected are loaded once and reused).
// Every query row has its own set of key positions; a tile of R <= 16 rows (the G heads
// of a KV head x TQ = 16 / G consecutive positions) is processed together:
//   perq_union_kernel    one CTA per tile: the rows' positions set bits of a shared-
//                        memory bitmap over the sequence's rows; an exclusive scan of the
//                        words' popcounts gives every member its union position; writes
//                        the union (ascending) and, per union key, the R-bit mask of the
//                        rows whose own set holds it;
//   perq_attn_kernel     the split-K gather of attn_decode.cuh over the union list, each
//                        union K/V row loaded once for all R rows, the membership bit
//                        deciding which rows see it;
//   perq_combine_kernel  merges the splits of each tile; a row whose set is empty gets
//                        zeros.
#pragma once
#include "common.cuh"
#include "attn_decode.cuh"

namespace quoka {

constexpr int PQ_MAX_ROWS = 16;
constexpr int PQ_UNION_THREADS = 512;
constexpr int PQ_MAX_WORDS = 8192;   // bitmap words: sequences up to 262144 rows

// One CTA per (tile, KV head, sequence).  Workspace per tile: PQ_MAX_ROWS * S entries of
// union positions and of membership masks (the worst case), plus the union size.
__global__ void __launch_bounds__(PQ_UNION_THREADS)
perq_union_kernel(const int32_t* __restrict__ sel, const __grid_constant__ SeqTable tab, int h_q,
                  int h_kv, int C, int S, int TQ, int32_t* __restrict__ uni,
                  uint32_t* __restrict__ memb, int32_t* __restrict__ ucount) {
  extern __shared__ uint32_t pq_sm[];
  __shared__ int wtot[PQ_UNION_THREADS / 32];
  __shared__ int utotal;
  const int tile = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = h_q / h_kv, t0 = tile * TQ, nt = min(TQ, C - t0);
  const long long N = tab.kv_off[b + 1] - tab.kv_off[b];
  const int W = (int)((N + 31) / 32);
  uint32_t* bm = pq_sm;
  int* pre = reinterpret_cast<int*>(pq_sm + PQ_MAX_WORDS);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t base = ((size_t)(b * h_kv + g) * gridDim.x + tile) * (size_t)(PQ_MAX_ROWS * S);

  for (int w = tid; w < W; w += blockDim.x) bm[w] = 0u;
  __syncthreads();
  const int nent = G * TQ * S;
  for (int e = tid; e < nent; e += blockDim.x) {
    const int r = e / S, i = e - r * S;
    const int jh = r / TQ, tt = r - jh * TQ;
    if (tt >= nt) continue;
    const int pos = sel[(((size_t)b * h_q + (size_t)g * G + jh) * C + t0 + tt) * S + i];
    if (pos < 0) continue;
    if (pos >= N) { flag_error(ERR_BAD_INDEX); continue; }
    atomicOr(&bm[pos >> 5], 1u << (pos & 31));
  }
  __syncthreads();
  // exclusive scan of the words' popcounts: each thread a contiguous run of words
  const int per = (W + blockDim.x - 1) / blockDim.x;
  const int lo = min(W, tid * per), hi = min(W, lo + per);
  int mine = 0;
  for (int w = lo; w < hi; ++w) mine += __popc(bm[w]);
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = lane < (int)(blockDim.x >> 5) ? wtot[lane] : 0;
    int iv = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, iv, o);
      if (lane >= o) iv += x;
    }
    if (lane < (int)(blockDim.x >> 5)) wtot[lane] = iv - v;     // exclusive warp offsets
    if (lane == 31) utotal = iv;
  }
  __syncthreads();
  int off = wtot[warp] + incl - mine;
  for (int w = lo; w < hi; ++w) {
    pre[w] = off;
    uint32_t word = bm[w];
    int u = off;
    while (word) {
      const int bit = __ffs(word) - 1;
      uni[base + u++] = (w << 5) + bit;
      word &= word - 1u;
    }
    off = u;
  }
  const int U = utotal;
  for (int u = tid; u < U; u += blockDim.x) memb[base + u] = 0u;
  __syncthreads();                                  // the block's global writes are visible
  for (int e = tid; e < nent; e += blockDim.x) {
    const int r = e / S, i = e - r * S;
    const int jh = r / TQ, tt = r - jh * TQ;
    if (tt >= nt) continue;
    const int pos = sel[(((size_t)b * h_q + (size_t)g * G + jh) * C + t0 + tt) * S + i];
    if (pos < 0 || pos >= N) continue;
    const int w = pos >> 5;
    const int u = pre[w] + __popc(bm[w] & ((1u << (pos & 31)) - 1u));
    atomicOr(&memb[base + u], 1u << r);
  }
  if (tid == 0) ucount[(size_t)(b * h_kv + g) * gridDim.x + tile] = U;
}

// One CTA per (split s, tile, sequence * KV head).  Rows r = jh * TQ + tt.
template <typename T, int D, int R>
__global__ void __launch_bounds__(AdcCfg<T, D>::THREADS)
perq_attn_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 long long rows_per_head, const __grid_constant__ SeqTable tab, int h_q, int h_kv,
                 int C, int S, int TQ, const int32_t* __restrict__ uni,
                 const uint32_t* __restrict__ memb, const int32_t* __restrict__ ucount, int split,
                 int nsplit_ws, float scale_log2, float* __restrict__ part) {
  using Cfg = AdcCfg<T, D>;
  constexpr int NW = Cfg::NW, ROW = Cfg::ROW, VPR = Cfg::VPR, EPV = Cfg::EPV, EPL = Cfg::EPL;
  extern __shared__ __align__(16) unsigned char smem[];
  const int s = blockIdx.x, tile = blockIdx.y, bg = blockIdx.z;
  const int b = bg / h_kv, g = bg - b * h_kv;
  const int ntiles = gridDim.y;
  const size_t tix = (size_t)bg * ntiles + tile;
  const int U = ucount[tix];
  const int k0 = s * split;
  const int k1 = min(U, k0 + split);
  if (k0 >= k1) return;
  const int G = h_q / h_kv, t0 = tile * TQ, nt = min(TQ, C - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* qs = reinterpret_cast<float*>(smem);
  float* mls = qs + R * D;
  unsigned char* stage = smem + (R * D + NW * R * 2) * 4 + warp * (Cfg::STAGE + 32 * R * 4);
  unsigned char* vstage = stage + 32 * ROW;
  float* ps = reinterpret_cast<float*>(stage + Cfg::STAGE);
  for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
    const int r = e / D, d = e - r * D;
    const int jh = r / TQ, tt = r - jh * TQ;
    float x = 0.f;
    if (jh < G && tt < nt)
      x = to_f32(q[(((size_t)b * h_q + (size_t)g * G + jh) * C + t0 + tt) * D + d]) * scale_log2;
    qs[e] = x;
  }
  __syncthreads();
  const T* kb = k + ((size_t)g * rows_per_head + tab.kv_off[b]) * D;
  const T* vb = v + ((size_t)g * rows_per_head + tab.kv_off[b]) * D;
  const size_t ubase = tix * (size_t)(PQ_MAX_ROWS * S);
  float m[R], l[R], acc[R][EPL];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[r][e] = 0.f;
  }
  for (int i0 = k0 + warp * 32; i0 < k1; i0 += NW * 32) {
    const int i = i0 + lane;
    int rr = 0;
    uint32_t mb = 0u;
    if (i < k1) {
      rr = __ldg(uni + ubase + i);
      mb = __ldg(memb + ubase + i);
    }
#pragma unroll 4
    for (int e = lane; e < 32 * VPR; e += 32) {
      const int kk = e / VPR, vv = e - kk * VPR;
      const int rk = __shfl_sync(0xffffffffu, rr, kk);
      adc_cp16(stage + kk * ROW + vv * 16, kb + (size_t)rk * D + vv * EPV);
    }
    adc_commit();
#pragma unroll 4
    for (int e = lane; e < 32 * VPR; e += 32) {
      const int kk = e / VPR, vv = e - kk * VPR;
      const int rk = __shfl_sync(0xffffffffu, rr, kk);
      adc_cp16(vstage + kk * ROW + vv * 16, vb + (size_t)rk * D + vv * EPV);
    }
    adc_commit();
    adc_wait<1>();
    __syncwarp();
    float sc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) sc[r] = 0.f;
    const unsigned char* krow = stage + lane * ROW;
#pragma unroll 2
    for (int c = 0; c < VPR; ++c) {
      float kx[EPV];
      smem_vec16<T>(krow + c * 16, kx);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float* qr = qs + r * D + c * EPV;
#pragma unroll
        for (int e4 = 0; e4 < EPV; e4 += 4) {
          const float4 qv = *reinterpret_cast<const float4*>(qr + e4);
          sc[r] = fmaf(qv.x, kx[e4], sc[r]);
          sc[r] = fmaf(qv.y, kx[e4 + 1], sc[r]);
          sc[r] = fmaf(qv.z, kx[e4 + 2], sc[r]);
          sc[r] = fmaf(qv.w, kx[e4 + 3], sc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (!((mb >> r) & 1u)) sc[r] = -INFINITY;        // not in this row's own set
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float mx = sc[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mn = fmaxf(m[r], mx);
      float p = 0.f, corr = 1.f;
      if (mn != -INFINITY) {
        p = exp2f(sc[r] - mn);
        corr = exp2f(m[r] - mn);
      }
      float sum = p;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      l[r] = l[r] * corr + sum;
      m[r] = mn;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[r][e] *= corr;
      ps[lane * R + r] = p;
    }
    adc_wait<0>();
    __syncwarp();
    const int nk = min(32, k1 - i0);
    for (int kk = 0; kk < nk; ++kk) {
      float vx[EPL];
      smem_vecn<T, EPL>(vstage + kk * ROW + lane * EPL * Cfg::ESZ, vx);
      const float* pk = ps + kk * R;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float pr = pk[r];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[r][e] = fmaf(pr, vx[e], acc[r][e]);
      }
    }
    __syncwarp();
  }
  float* wout = reinterpret_cast<float*>(stage);
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      mls[(warp * R + r) * 2] = m[r];
      mls[(warp * R + r) * 2 + 1] = l[r];
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int e = 0; e < EPL; ++e) wout[r * D + lane * EPL + e] = acc[r][e];
  __syncthreads();
  float* dst = part + ((tix * nsplit_ws + s) * R) * Cfg::PD;
  for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
    const int r = e / D, d = e - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mls[(w * R + r) * 2]);
    float o = 0.f, L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = mls[(w * R + r) * 2];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - M);
        const float* ww = reinterpret_cast<const float*>(smem + (R * D + NW * R * 2) * 4 +
                                                         w * (Cfg::STAGE + 32 * R * 4));
        o += ww[e] * f;
        L += mls[(w * R + r) * 2 + 1] * f;
      }
    }
    dst[r * Cfg::PD + d] = o;
    if (d == 0) {
      dst[r * Cfg::PD + D] = M;
      dst[r * Cfg::PD + D + 1] = L;
    }
  }
}

// Merges the splits of each tile; a row whose set is empty gets zeros.
template <typename T, int D, int R>
__global__ void __launch_bounds__(128)
perq_combine_kernel(const float* __restrict__ part, const int32_t* __restrict__ ucount,
                    int h_q, int h_kv, int C, int TQ, int split, int nsplit_ws,
                    T* __restrict__ out) {
  constexpr int PD = D + 4;
  __shared__ float Ms[R], Ls[R];
  const int tile = blockIdx.x, bg = blockIdx.y;
  const int b = bg / h_kv, g = bg - b * h_kv;
  const int G = h_q / h_kv, t0 = tile * TQ, nt = min(TQ, C - t0);
  const size_t tix = (size_t)bg * gridDim.x + tile;
  const int ns = (ucount[tix] + split - 1) / split;
  const float* src = part + tix * nsplit_ws * R * PD;
  if (threadIdx.x < R) {
    const int r = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, src[((size_t)s * R + r) * PD + D]);
    float L = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < ns; ++s) {
        const float ms = src[((size_t)s * R + r) * PD + D];
        if (ms != -INFINITY) L += src[((size_t)s * R + r) * PD + D + 1] * exp2f(ms - M);
      }
    Ms[r] = M;
    Ls[r] = L;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
    const int r = e / D, d = e - r * D;
    const int jh = r / TQ, tt = r - jh * TQ;
    if (jh >= G || tt >= nt) continue;
    const float M = Ms[r];
    float o = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < ns; ++s) {
        const float ms = src[((size_t)s * R + r) * PD + D];
        if (ms != -INFINITY) o += src[((size_t)s * R + r) * PD + d] * exp2f(ms - M);
      }
    const float L = Ls[r];
    out[(((size_t)b * h_q + (size_t)g * G + jh) * C + t0 + tt) * D + d] =
        from_f32<T>(L > 0.f ? o / L : 0.f);
  }
}

}  // namespace quoka
