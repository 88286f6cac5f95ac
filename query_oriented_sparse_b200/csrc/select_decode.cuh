// Selection for decode steps and short chunks (QUOKA page, results summary: the method
// also runs in the generation phase), where every query of the chunk is kept (Nq >= C)
// and at most 16 query rows share a KV head.
//
// With one or a few kept queries per head the cosine scoring is a stream over the prefix
// keys with a handful of dot products per key, bound by reading the keys.  bf16 keys are
// scored by score_decode_tc_kernel (score_decode_tc.cuh: TMA-streamed tiles, a 128 x 16
// tensor-core MMA per tile); fp32 keys here:
//   kept_all_kernel      writes the kept positions (all of them) when the caller asks;
//   score_decode_kernel  one CTA per (1024-key tile, KV head, sequence), four warps; each
//                        warp streams batches of 32 consecutive key rows into its own
//                        shared-memory stage with 16-byte cp.async (two stages, the next
//                        batch in flight while this one is scored), and lane l scores key
//                        l: its R dot products with the unit queries and its norm, then
//                        s = (1/G) sum_h max_t cos(q_{h,t}, k) (method summary: max over
//                        queries, mean over the group's heads);
//   topk_block_kernel    one CTA per (sequence, KV head) for rows short enough to stage
//                        in shared memory: the radix select and the ordered emit of
//                        cluster_select.cuh with block barriers only.  Taken when there
//                        are at least 32 rows of at most 32768 keys, or rows of at most
//                        8192 keys however few (gqa_8k's 8 rows of 8192: 19.4 us against
//                        23.5 us for 16-CTA clusters).
#pragma once
#include "cluster_select.cuh"
#include "tc_ptx.cuh"
#include "topk.cuh"

namespace quoka {

constexpr int SCD_WARPS = 4;
constexpr int SCD_THREADS = SCD_WARPS * 32;
constexpr int SCD_BATCHES = 8;                              // 32-key batches per warp
constexpr int SCD_KEYS = SCD_WARPS * SCD_BATCHES * 32;      // keys per CTA
constexpr int TOPK_BLOCK_MAX_KEYS = 32768;                  // staged keys (128 KB)
constexpr int TOPK_BLOCK_MIN_ROWS = 32;                     // (sequence, KV head) rows
constexpr int TOPK_BLOCK_ANY_KEYS = 8192;                   // rows this short, however few

__global__ void kept_all_kernel(int32_t* __restrict__ kept_out, int heads, int C, int nq) {
  const long long n = (long long)heads * nq;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(e % nq);
    kept_out[e] = i < C ? i : -1;
  }
}

template <typename T, int D>
struct ScdCfg {
  static constexpr int ESZ = (int)sizeof(T);
  static constexpr int VPR = D * ESZ / 16;          // 16-byte vectors per key row
  static constexpr int EPV = 16 / ESZ;
  static constexpr int ROW = D * ESZ + 16;          // padded shared-memory row
  static constexpr int STAGE = 32 * ROW;
};

template <typename T, int D, int R>
constexpr int scd_smem_bytes() {
  return R * D * 4 + SCD_WARPS * 2 * ScdCfg<T, D>::STAGE;
}

__device__ __forceinline__ void scd_cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void scd_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void scd_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename T>
__device__ __forceinline__ void scd_vec16(const unsigned char* p, float (&x)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const unsigned int w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      unsigned int wi = w[i];
      const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wi));
      x[2 * i] = f.x; x[2 * i + 1] = f.y;
    }
  }
}

// Rows r = j * C + t of a KV head: query head g*G + j, chunk position t (all kept).
template <typename T, int D, int R>
__global__ void __launch_bounds__(SCD_THREADS)
score_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, long long rows_per_head,
                    const __grid_constant__ SeqTable tab, int h_q, int h_kv, int C,
                    float* __restrict__ pooled, long long pooled_stride) {
  using Cfg = ScdCfg<T, D>;
  constexpr int ROW = Cfg::ROW, VPR = Cfg::VPR, EPV = Cfg::EPV;
  extern __shared__ __align__(16) unsigned char smem[];
  const int g = blockIdx.y, b = blockIdx.z;
  const int P = tab.prefix[b];
  const int j0 = blockIdx.x * SCD_KEYS;
  if (j0 >= P) return;                                     // uniform over the CTA
  const int G = h_q / h_kv, rows = G * C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* qs = reinterpret_cast<float*>(smem);              // [R][D] unit queries
  unsigned char* stage = smem + R * D * 4 + warp * 2 * Cfg::STAGE;

  const T* kb = k + ((size_t)g * rows_per_head + tab.kv_off[b]) * D;
  // start the first batch's keys before the queries are prepared
  auto issue = [&](int batch, int buf) {
    const int base = j0 + (warp + SCD_WARPS * batch) * 32;
    unsigned char* dst = stage + buf * Cfg::STAGE;
#pragma unroll 4
    for (int e = lane; e < 32 * VPR; e += 32) {
      const int kk = e / VPR, vv = e - kk * VPR;
      const int j = min(base + kk, P - 1);                 // rows past P: any valid row
      scd_cp16(dst + kk * ROW + vv * 16, kb + (size_t)j * D + vv * EPV);
    }
    scd_commit();
  };
  issue(0, 0);

  for (int e = threadIdx.x; e < R * D; e += SCD_THREADS) {
    const int r = e / D, d = e - r * D;
    float x = 0.f;
    if (r < rows) {
      const int jh = r / C, t = r - jh * C;
      x = to_f32(q[(((size_t)b * h_q + (size_t)g * G + jh) * C + t) * D + d]);
    }
    qs[e] = x;
  }
  __syncthreads();
  for (int r = warp; r < R; r += SCD_WARPS) {              // unit rows (a zero row stays 0)
    float ss = 0.f;
    for (int d = lane; d < D; d += 32) ss = fmaf(qs[r * D + d], qs[r * D + d], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
    for (int d = lane; d < D; d += 32) qs[r * D + d] *= inv;
  }
  __syncthreads();

  float* out = pooled + (size_t)(b * h_kv + g) * pooled_stride;
  const float inv_G = 1.0f / (float)G;
  for (int bt = 0; bt < SCD_BATCHES; ++bt) {
    const int base = j0 + (warp + SCD_WARPS * bt) * 32;
    if (base >= P) break;                                  // uniform over the warp
    const bool more = bt + 1 < SCD_BATCHES && base + SCD_WARPS * 32 < P;
    if (more) {
      issue(bt + 1, (bt + 1) & 1);
      scd_wait<1>();
    } else {
      scd_wait<0>();
    }
    __syncwarp();
    const unsigned char* krow = stage + (bt & 1) * Cfg::STAGE + lane * ROW;
    float dot[R];
    float nn = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) dot[r] = 0.f;
#pragma unroll 2
    for (int c = 0; c < VPR; ++c) {
      float kx[EPV];
      scd_vec16<T>(krow + c * 16, kx);
#pragma unroll
      for (int e = 0; e < EPV; ++e) nn = fmaf(kx[e], kx[e], nn);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float* qr = qs + r * D + c * EPV;
#pragma unroll
        for (int e4 = 0; e4 < EPV; e4 += 4) {
          const float4 qv = *reinterpret_cast<const float4*>(qr + e4);
          dot[r] = fmaf(qv.x, kx[e4], dot[r]);
          dot[r] = fmaf(qv.y, kx[e4 + 1], dot[r]);
          dot[r] = fmaf(qv.z, kx[e4 + 2], dot[r]);
          dot[r] = fmaf(qv.w, kx[e4 + 3], dot[r]);
        }
      }
    }
    float s = 0.f;
    for (int jh = 0; jh < G; ++jh) {
      float m = -INFINITY;
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r >= jh * C && r < (jh + 1) * C) m = fmaxf(m, dot[r]);
      s += m;
    }
    const int j = base + lane;
    if (j < P) out[j] = nn > 0.f ? (s * inv_G) / sqrtf(nn) : 0.f;
    __syncwarp();                                          // stage reused two batches on
  }
}

// One CTA per (sequence, KV head) whose prefix fits the staging area.
__global__ void __launch_bounds__(512)
topk_block_kernel(float* __restrict__ pooled, long long pooled_stride, int ncg, long long cg_stride,
                  float inv_G, const __grid_constant__ SeqTable tab, int h_kv, int b_max,
                  int32_t* __restrict__ idx_out) {
  __shared__ SelectSmem sm;
  extern __shared__ uint32_t staged[];
  const int head = blockIdx.x;                             // b * h_kv + g
  const int b = head / h_kv;
  const int P = tab.prefix[b], B = tab.nsel[b];
  int32_t* out = idx_out + (size_t)head * b_max;
  float* sc = pooled + (size_t)head * pooled_stride;
  if (ncg > 1) {                                           // column groups, in group order
    for (int j = threadIdx.x; j < P; j += blockDim.x) {
      float s = sc[j];
      for (int c = 1; c < ncg; ++c) s += sc[c * cg_stride + j];
      sc[j] = s * inv_G;
    }
    __syncthreads();
  }
  for (int i = B + threadIdx.x; i < b_max; i += blockDim.x) out[i] = -1;
  if (B >= P) {                                            // every prefix key (P == 0 too)
    for (int i = threadIdx.x; i < P; i += blockDim.x) out[i] = i;
    return;
  }
  if (B == 0) return;
  // stage the row's keys: TOPK_STAGE_UNROLL loads in flight per thread (the scores were
  // just written and sit in L2, so the staging costs a few round trips, not one per key)
  for (int j0 = threadIdx.x; j0 < P; j0 += TOPK_STAGE_UNROLL * blockDim.x) {
    float v[TOPK_STAGE_UNROLL];
#pragma unroll
    for (int u = 0; u < TOPK_STAGE_UNROLL; ++u) {
      const int j = j0 + u * blockDim.x;
      v[u] = j < P ? sc[j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < TOPK_STAGE_UNROLL; ++u) {
      const int j = j0 + u * blockDim.x;
      if (j < P) staged[j] = float_to_ordered(v[u]);
    }
  }
  __syncthreads();
  auto key_at = [&](int j) { return staged[j]; };
  auto emit = [&](int pos, int j) {
    if (pos < B) out[pos] = j;
    else flag_error(ERR_BAD_INDEX);                        // unreachable when counts agree
  };
  const SelectThreshold th = block_threshold<true>(sm, key_at, P, B);
  ordered_emit<true>(sm, key_at, 0, P, th, emit);
}

}  // namespace quoka
