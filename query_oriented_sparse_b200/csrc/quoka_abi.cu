// Host side of libquoka.so: argument validation, workspace layout and kernel launches
// behind the C ABI declared in include/quoka.h.  Every check runs before any CUDA
// call, so an invalid call launches nothing.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "qsub.cuh"
#include "score_simt.cuh"
#include "score_tc.cuh"
#include "topk.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "attn_tc2.cuh"
#include "compact.cuh"
#include "attn_decode.cuh"
#include "select_decode.cuh"
#include "score_decode_tc.cuh"
#include "attn_perq.cuh"
#include "selcache.cuh"
#include "perq_tc.cuh"

using namespace quoka;

namespace {

thread_local std::string g_last_error;

quoka_status fail(quoka_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

quoka_status cuda_fail(cudaError_t e, const char* where) {
  return fail(QUOKA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Per-kernel timing (quoka_profile_events): while a caller's event array is set on this
// thread, every launch is followed by a record of the next event on the launch's stream.
struct ProfState {
  void* const* events = nullptr;
  int n = 0, used = 0;
  std::vector<const char*> names;
};
thread_local ProfState g_prof;

void prof_mark(cudaStream_t st, const char* name) {
  if (!g_prof.events || g_prof.used >= g_prof.n) return;
  if (cudaEventRecord(reinterpret_cast<cudaEvent_t>(g_prof.events[g_prof.used]), st) != cudaSuccess)
    return;
  g_prof.names.push_back(name);
  ++g_prof.used;
}

struct Dims {
  int batch, h_q, h_kv, G, D, C;
  quoka_dtype dt;
  int esz;
};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

quoka_status check_shape(const quoka_shape* s, Dims* d) {
  if (!s) return fail(QUOKA_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 1) return fail(QUOKA_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", s->batch);
  if (s->batch > QUOKA_MAX_BATCH)
    return fail(QUOKA_ERR_UNSUPPORTED, "batch %d exceeds QUOKA_MAX_BATCH=%d", s->batch, QUOKA_MAX_BATCH);
  if (s->h_q < 1 || s->h_kv < 1 || s->h_q % s->h_kv != 0)
    return fail(QUOKA_ERR_INVALID_ARG, "h_q=%d must be a positive multiple of h_kv=%d", s->h_q, s->h_kv);
  if (s->h_q / s->h_kv > QUOKA_MAX_GROUP)
    return fail(QUOKA_ERR_UNSUPPORTED, "group size %d exceeds %d", s->h_q / s->h_kv, QUOKA_MAX_GROUP);
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(QUOKA_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", s->head_dim);
  if (s->chunk < 1) return fail(QUOKA_ERR_INVALID_ARG, "chunk must be >= 1 (got %d)", s->chunk);
  if (s->chunk > QUOKA_MAX_CHUNK)
    return fail(QUOKA_ERR_UNSUPPORTED, "chunk %d exceeds QUOKA_MAX_CHUNK=%d", s->chunk, QUOKA_MAX_CHUNK);
  if (s->dtype != QUOKA_F32 && s->dtype != QUOKA_BF16)
    return fail(QUOKA_ERR_UNSUPPORTED, "unknown dtype %d", (int)s->dtype);
  d->batch = s->batch;
  d->h_q = s->h_q;
  d->h_kv = s->h_kv;
  d->G = s->h_q / s->h_kv;
  d->D = s->head_dim;
  d->C = s->chunk;
  d->dt = s->dtype;
  d->esz = s->dtype == QUOKA_F32 ? 4 : 2;
  return QUOKA_OK;
}

// Fills the kernel-side sequence table from the host arrays.
quoka_status build_table(const Dims& d, const int64_t* kv_off, const int32_t* prefix,
                         const int32_t* budget, int b_max, SeqTable* tab, long long* rows) {
  if (!kv_off || !prefix || !budget) return fail(QUOKA_ERR_INVALID_ARG, "kv_off, prefix_len and budget must be non-NULL");
  if (b_max < 1) return fail(QUOKA_ERR_INVALID_ARG, "b_max must be >= 1 (got %d)", b_max);
  if (kv_off[0] < 0) return fail(QUOKA_ERR_INVALID_ARG, "kv_off[0] must be >= 0");
  tab->batch = d.batch;
  tab->max_prefix = 0;
  for (int b = 0; b <= d.batch; ++b) tab->kv_off[b] = kv_off[b];
  for (int b = 0; b < d.batch; ++b) {
    const int P = prefix[b];
    if (P < 0) return fail(QUOKA_ERR_INVALID_ARG, "prefix_len[%d] = %d < 0", b, P);
    if (budget[b] < 0 || budget[b] > b_max)
      return fail(QUOKA_ERR_INVALID_ARG, "budget[%d] = %d outside [0, b_max=%d]", b, budget[b], b_max);
    if (kv_off[b + 1] - kv_off[b] < (int64_t)P + d.C)
      return fail(QUOKA_ERR_INVALID_ARG,
                  "sequence %d owns %lld cache rows, fewer than prefix_len + chunk = %lld", b,
                  (long long)(kv_off[b + 1] - kv_off[b]), (long long)P + d.C);
    tab->prefix[b] = P;
    tab->nsel[b] = budget[b] < P ? budget[b] : P;
    if (P > tab->max_prefix) tab->max_prefix = P;
  }
  for (int b = d.batch; b < QUOKA_MAX_BATCH; ++b) { tab->prefix[b] = 0; tab->nsel[b] = 0; }
  *rows = kv_off[d.batch];
  return QUOKA_OK;
}

struct WsLayout {
  size_t qsel, qinv, qbias, pooled, total;
  long long pooled_stride;  // floats per (sequence, KV head) row
  long long cg_stride;      // floats between column-group partial arrays
  int nk, nkp;              // kept queries per head, and that count padded to 16
  int ncg, heads_per_cg;    // column groups per KV head for the tensor-core scoring
  bool tc;                  // tensor-core scoring (bf16) or CUDA-core scoring (fp32)
  bool dec;                 // every query kept and <= 16 rows per KV head: decode scoring
};

WsLayout ws_layout(const Dims& d, int max_prefix, int nq) {
  WsLayout w;
  w.nk = nq < d.C ? nq : d.C;
  w.nkp = (w.nk + 15) / 16 * 16;
  w.dec = w.nk == d.C && d.G * d.C <= ADC_MAX_ROWS;
  w.tc = !w.dec && d.dt == QUOKA_BF16 && w.nkp <= STC_SLICE;
  if (w.tc) {
    // a column group is at most two head-aligned slices of <= 256 columns
    const int hmax = 2 * (STC_SLICE / w.nkp);
    w.ncg = (d.G + hmax - 1) / hmax;
    w.heads_per_cg = (d.G + w.ncg - 1) / w.ncg;
  } else {
    w.ncg = 1;
    w.heads_per_cg = d.G;
  }
  const size_t rows = (size_t)d.batch * d.h_q * w.nkp;
  size_t off = 0;
  w.qsel = off;
  off = align_up(off + rows * d.D * d.esz, 256);
  w.qinv = off;
  off = align_up(off + rows * 4, 256);
  w.qbias = off;
  off = align_up(off + rows * 4, 256);
  w.pooled_stride = (long long)align_up((size_t)(max_prefix > 0 ? max_prefix : 1), 128);
  w.cg_stride = (long long)d.batch * d.h_kv * w.pooled_stride;
  w.pooled = off;
  off = align_up(off + (size_t)w.ncg * w.cg_stride * 4, 256);
  w.total = off;
  return w;
}

// ---- TMA tensor maps (driver entry point fetched through the runtime) ----------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Row-major [rows, cols] bf16 matrix, box of box_cols x box_rows, 128-byte swizzle.
quoka_status make_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_cols, uint32_t box_rows, const char* what) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(QUOKA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  if (rows >= (1ull << 31)) return fail(QUOKA_ERR_UNSUPPORTED, "%s has more than 2^31 rows", what);
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QUOKA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
  return QUOKA_OK;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// Raises a kernel's dynamic shared-memory limit, once per (kernel, device).
std::mutex g_smem_mu;
std::map<std::pair<const void*, int>, int> g_smem_set;

template <typename K>
cudaError_t ensure_smem(K kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lock(g_smem_mu);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g_smem_set[key] = bytes;
  return e;
}

// Allows a kernel's clusters above the portable size of 8 CTAs (B200 schedules 16).
template <typename K>
cudaError_t ensure_cluster16(K kernel) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::map<std::pair<const void*, int>, bool> done;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lock(g_smem_mu);
  if (done.count(key)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) done[key] = true;
  return e;
}

template <int D>
quoka_status launch_score_tc(const Dims& d, const SeqTable& tab, long long rows, const void* k,
                             unsigned char* ws, const WsLayout& w, cudaStream_t st) {
  ScoreTcParams p;
  p.h_kv = d.h_kv;
  p.G = d.G;
  p.nkp = w.nkp;
  p.ncg = w.ncg;
  p.heads_per_cg = w.heads_per_cg;
  p.padded = w.nk < w.nkp ? 1 : 0;
  p.rows_per_head = rows;
  p.pooled_stride = w.pooled_stride;
  p.cg_stride = w.cg_stride;
  p.inv_G = 1.0f / (float)d.G;
  long long units = 0;
  for (int b = 0; b < d.batch; ++b) {
    p.unit_base[b] = (int)units;
    units += (long long)d.h_kv * w.ncg * ((tab.prefix[b] + STC_BM - 1) / STC_BM);
  }
  for (int b = d.batch; b <= QUOKA_MAX_BATCH; ++b) p.unit_base[b] = (int)units;
  if (units == 0) return QUOKA_OK;
  if (units >= (1ll << 31)) return fail(QUOKA_ERR_UNSUPPORTED, "too many key tiles");
  p.total_units = (int)units;
  CUtensorMap kmap, qmap;
  quoka_status s;
  if ((s = make_map_bf16(&kmap, k, (uint64_t)d.h_kv * rows, D, 64, STC_BM, "k_cache")) != QUOKA_OK) return s;
  if ((s = make_map_bf16(&qmap, ws + w.qsel, (uint64_t)d.batch * d.h_q * w.nkp, D, 64, STC_QBOX,
                         "kept queries")) != QUOKA_OK)
    return s;
  cudaError_t e;
  const int smem = StcCfg<D>::SMEM;
  if ((e = ensure_smem(score_tc_kernel<D>, smem)) != cudaSuccess) return cuda_fail(e, "score_tc smem");
  const int grid = (int)std::min<long long>(units, sm_count());
  score_tc_kernel<D><<<grid, STC_THREADS, smem, st>>>(
      kmap, qmap, tab, p, reinterpret_cast<const float*>(ws + w.qinv),
      reinterpret_cast<const float*>(ws + w.qbias), reinterpret_cast<float*>(ws + w.pooled));
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "score_tc launch");
  prof_mark(st, "score_tc_kernel");
  return QUOKA_OK;
}

// Top-B per (sequence, KV head): one CTA per row when there are many rows short enough to
// stage in shared memory, else a 16-CTA cluster per row.
quoka_status launch_topk(const Dims& d, const SeqTable& tab, int b_max, int32_t* idx_out,
                         const WsLayout& w, float* pooled, cudaStream_t st) {
  cudaError_t e;
  const int nrows = d.batch * d.h_kv;
  // one CTA per row when the rows are many, or so short that a cluster's barriers cost
  // more than it spreads
  if (tab.max_prefix <= TOPK_BLOCK_MAX_KEYS &&
      (nrows >= TOPK_BLOCK_MIN_ROWS || tab.max_prefix <= TOPK_BLOCK_ANY_KEYS)) {
    const int smem = std::max(tab.max_prefix, 1) * 4;
    if ((e = ensure_smem(topk_block_kernel, smem)) != cudaSuccess) return cuda_fail(e, "topk_block smem");
    topk_block_kernel<<<nrows, 512, smem, st>>>(pooled, w.pooled_stride, w.ncg, w.cg_stride,
                                                 1.0f / (float)d.G, tab, d.h_kv, b_max, idx_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "topk_block launch");
    prof_mark(st, "topk_block_kernel");
    return QUOKA_OK;
  }
  // CTAs per row: 16, halved (down to 4) while the rows' clusters would not all fit the
  // SMs at once (one CTA per SM) and a CTA's slice still fits its staging area
  int cs = TOPK_MAX_CS;
  while (cs > 4 && (long long)nrows * cs > (long long)sm_count() &&
         (tab.max_prefix + cs / 2 - 1) / (cs / 2) <= TOPK_STAGE_KEYS)
    cs /= 2;
  const int tk_keys = std::min((tab.max_prefix + cs - 1) / cs, TOPK_STAGE_KEYS);
  const int tk_smem = tk_keys * 4;
  auto topk_launch = [&](auto kern, int csz) -> cudaError_t {
    cudaError_t err = ensure_smem(kern, tk_smem);
    if (err == cudaSuccess && csz > 8) err = ensure_cluster16(kern);
    if (err != cudaSuccess) return err;
    kern<<<nrows * csz, TOPK_THREADS, tk_smem, st>>>(
        pooled, w.pooled_stride, w.ncg, w.cg_stride, 1.0f / (float)d.G, tab, d.h_kv, b_max, idx_out);
    return cudaGetLastError();
  };
  switch (cs) {
    case 4: e = topk_launch(topk_kernel<4>, 4); break;
    case 8: e = topk_launch(topk_kernel<8>, 8); break;
    default: e = topk_launch(topk_kernel<16>, 16); break;
  }
  if (e != cudaSuccess) return cuda_fail(e, "topk launch");
  prof_mark(st, "topk_kernel");
  return QUOKA_OK;
}

template <typename T, int D, int R>
quoka_status launch_score_decode_r(const Dims& d, const SeqTable& tab, long long rows,
                                   const void* q, const void* k, float* pooled, const WsLayout& w,
                                   cudaStream_t st) {
  const int smem = scd_smem_bytes<T, D, R>();
  cudaError_t e;
  if ((e = ensure_smem(score_decode_kernel<T, D, R>, smem)) != cudaSuccess) return cuda_fail(e, "score_decode smem");
  dim3 grid((tab.max_prefix + SCD_KEYS - 1) / SCD_KEYS, d.h_kv, d.batch);
  score_decode_kernel<T, D, R><<<grid, SCD_THREADS, smem, st>>>(
      reinterpret_cast<const T*>(q), reinterpret_cast<const T*>(k), rows, tab, d.h_q, d.h_kv, d.C,
      pooled, w.pooled_stride);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "score_decode launch");
  prof_mark(st, "score_decode_kernel");
  return QUOKA_OK;
}

// bf16 decode scoring on tensor cores: a 128 x 16 MMA per 128-key tile, keys streamed
// by TMA, two CTAs per SM.
template <int D>
quoka_status launch_score_decode_tc(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                                    const void* k, float* pooled, const WsLayout& w, cudaStream_t st) {
  CUtensorMap kmap, qmap;
  quoka_status s;
  if ((s = make_map_bf16(&kmap, k, (uint64_t)d.h_kv * rows, D, 64, 128, "k_cache")) != QUOKA_OK) return s;
  if ((s = make_map_bf16(&qmap, q, (uint64_t)d.batch * d.h_q * d.C, D, 64, SDT_QROWS, "q_chunk")) != QUOKA_OK)
    return s;
  cudaError_t e;
  const int smem = SdtCfg<D>::SMEM;
  if ((e = ensure_smem(score_decode_tc_kernel<D>, smem)) != cudaSuccess) return cuda_fail(e, "score_decode_tc smem");
  dim3 grid((tab.max_prefix + SDT_TILES * 128 - 1) / (SDT_TILES * 128), d.h_kv, d.batch);
  score_decode_tc_kernel<D><<<grid, SDT_THREADS, smem, st>>>(kmap, qmap, tab, rows, d.h_q, d.h_kv, d.C,
                                                             pooled, w.pooled_stride);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "score_decode_tc launch");
  prof_mark(st, "score_decode_tc_kernel");
  return QUOKA_OK;
}

// Every query kept and at most 16 query rows per KV head: the kept positions are all of
// them, and the scoring streams the prefix keys (bf16: tensor cores; fp32: CUDA cores).
template <typename T, int D>
quoka_status launch_select_decode(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                                  const void* k, int nq, int32_t* kept_out, float* pooled,
                                  const WsLayout& w, cudaStream_t st) {
  cudaError_t e;
  if (kept_out) {
    const long long n = (long long)d.batch * d.h_q * nq;
    const int grid = (int)std::min<long long>((n + 255) / 256, (long long)sm_count() * 4);
    kept_all_kernel<<<grid, 256, 0, st>>>(kept_out, d.batch * d.h_q, d.C, nq);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "kept launch");
    prof_mark(st, "kept_all_kernel");
  }
  if (tab.max_prefix == 0) return QUOKA_OK;
  if constexpr (sizeof(T) == 2) {
    return launch_score_decode_tc<D>(d, tab, rows, q, k, pooled, w, st);
  } else {
    int r = 1;
    while (r < d.G * d.C) r *= 2;
    switch (r) {
      case 1: return launch_score_decode_r<T, D, 1>(d, tab, rows, q, k, pooled, w, st);
      case 2: return launch_score_decode_r<T, D, 2>(d, tab, rows, q, k, pooled, w, st);
      case 4: return launch_score_decode_r<T, D, 4>(d, tab, rows, q, k, pooled, w, st);
      case 8: return launch_score_decode_r<T, D, 8>(d, tab, rows, q, k, pooled, w, st);
      default: return launch_score_decode_r<T, D, 16>(d, tab, rows, q, k, pooled, w, st);
    }
  }
}

template <typename T, int D>
quoka_status launch_select(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                           const void* k, int nq, int b_max, int32_t* idx_out, int32_t* kept_out,
                           unsigned char* ws, const WsLayout& w, cudaStream_t st) {
  T* qsel = reinterpret_cast<T*>(ws + w.qsel);
  float* qinv = reinterpret_cast<float*>(ws + w.qinv);
  float* qbias = reinterpret_cast<float*>(ws + w.qbias);
  float* pooled = reinterpret_cast<float*>(ws + w.pooled);
  cudaError_t e;

  if (w.dec) {
    quoka_status s = launch_select_decode<T, D>(d, tab, rows, q, k, nq, kept_out, pooled, w, st);
    if (s != QUOKA_OK) return s;
    return launch_topk(d, tab, b_max, idx_out, w, pooled, st);
  }

  // CTAs per query head: the fewest that cover the chunk, doubled while every head's
  // cluster still fits the SMs at once (two CTAs per SM)
  int cs = 1;
  while (cs < QSUB_MAX_CS && (d.C + cs - 1) / cs > QSUB_MAX_ROWS) cs *= 2;
  while (cs < QSUB_MAX_CS && (long long)d.batch * d.h_q * cs * 2 <= 2LL * sm_count()) cs *= 2;
  const int qs_smem = d.C * 4;                 // the chunk-wide key array
  auto qsub_launch = [&](auto kern, int csz) -> cudaError_t {
    cudaError_t err = ensure_smem(kern, qs_smem);
    if (err != cudaSuccess) return err;
    kern<<<d.batch * d.h_q * csz, QSUB_THREADS, qs_smem, st>>>(
        reinterpret_cast<const T*>(q), d.C, w.nk, w.nkp, nq, kept_out, qsel, qinv, qbias);
    return cudaGetLastError();
  };
  switch (cs) {
    case 1: e = qsub_launch(qsub_kernel<T, D, 1>, 1); break;
    case 2: e = qsub_launch(qsub_kernel<T, D, 2>, 2); break;
    case 4: e = qsub_launch(qsub_kernel<T, D, 4>, 4); break;
    default: e = qsub_launch(qsub_kernel<T, D, 8>, 8); break;
  }
  if (e != cudaSuccess) return cuda_fail(e, "qsub launch");
  prof_mark(st, "qsub_kernel");

  if (tab.max_prefix > 0) {
    if (w.tc) {
      quoka_status s = launch_score_tc<D>(d, tab, rows, k, ws, w, st);
      if (s != QUOKA_OK) return s;
    } else {
      const int s2 = score_simt_smem_bytes<D>(d.G);
      if ((e = ensure_smem(score_simt_kernel<T, D>, s2)) != cudaSuccess) return cuda_fail(e, "score smem");
      dim3 grid((tab.max_prefix + SCS_KEYS - 1) / SCS_KEYS, d.h_kv, d.batch);
      score_simt_kernel<T, D><<<grid, SCS_THREADS, s2, st>>>(
          reinterpret_cast<const T*>(k), rows, tab, d.h_kv, d.G, w.nkp, qsel, qinv, qbias, pooled,
          w.pooled_stride);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "score launch");
      prof_mark(st, "score_simt_kernel");
    }
  }

  return launch_topk(d, tab, b_max, idx_out, w, pooled, st);
}

// Rows per (sequence, KV head) block of the compacted cache.
long long kc_block_rows(const Dims& d, int b_max) {
  return (long long)align_up((size_t)b_max + d.C, 128);
}

// Few query rows per KV head (decode, short chunks): the split-K gather kernel.
bool use_decode(const Dims& d) { return d.G * d.C <= ADC_MAX_ROWS; }

int decode_rows(const Dims& d) {
  int r = 1;
  while (r < d.G * d.C) r *= 2;
  return r;
}

// Splits a (sequence, KV head) can have: the fewest keys per split is ADC_MIN_SPLIT.
int decode_nsplit_ws(const Dims& d, int b_max) {
  return (b_max + d.C + ADC_MIN_SPLIT - 1) / ADC_MIN_SPLIT;
}

size_t attn_ws_bytes(const Dims& d, int b_max) {
  if (use_decode(d))
    return align_up((size_t)d.batch * d.h_kv * decode_nsplit_ws(d, b_max) * decode_rows(d) *
                        (d.D + 4) * 4, 256);
  if (d.dt != QUOKA_BF16) return 0;
  const size_t rows = (size_t)d.batch * d.h_kv * (size_t)kc_block_rows(d, b_max);
  return 2 * align_up(rows * d.D * 2, 256);
}

template <int D>
quoka_status launch_attn_tc_core(const Dims& d, const SeqTable& tab, const void* q, const void* kc,
                                 const void* vc, long long kc_stride, void* out, cudaStream_t st);

template <int D>
quoka_status launch_attn_tc(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                            const void* k, const void* v, const int32_t* idx, int b_max,
                            void* out, unsigned char* ws, cudaStream_t st,
                            const void* k_new = nullptr, const void* v_new = nullptr) {
  AttnTcParams p;
  p.h_q = d.h_q;
  p.h_kv = d.h_kv;
  p.G = d.G;
  p.C = d.C;
  p.TP = 128 / d.G;
  p.b_max = b_max;
  p.kc_stride = kc_block_rows(d, b_max);
  p.rows_per_head = rows;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  const size_t kc_rows = (size_t)d.batch * d.h_kv * p.kc_stride;
  unsigned char* kc = ws;
  unsigned char* vc = ws + attn_ws_bytes(d, b_max) / 2;
  cudaError_t e;
  // 1. the compacted cache: selected rows then the chunk rows, per (sequence, KV head)
  const long long vecs = (long long)kc_rows * (D * 2 / 16);
  const int cgrid = (int)std::min<long long>((vecs + CPT_THREADS - 1) / CPT_THREADS, (long long)sm_count() * 16);
  compact_kv_kernel<D><<<cgrid, CPT_THREADS, 0, st>>>(
      reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), rows, tab, d.h_kv, d.C,
      b_max, p.kc_stride, idx, reinterpret_cast<uint4*>(kc), reinterpret_cast<uint4*>(vc), vecs,
      reinterpret_cast<const uint4*>(k_new), reinterpret_cast<const uint4*>(v_new),
      reinterpret_cast<uint4*>(const_cast<void*>(k)), reinterpret_cast<uint4*>(const_cast<void*>(v)));
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "compact launch");
  prof_mark(st, "compact_kv_kernel");
  // 2. dense attention over it
  return launch_attn_tc_core<D>(d, tab, q, kc, vc, p.kc_stride, out, st);
}

// Grid z -> sequence for the pair attention: sequences with the most keys first, so a
// ragged batch's longest pairs start early and the last wave holds the shortest ones.
// Clusters (SM pairs) of the pair attention kernel that fit on the device at once: the
// persistent grid's size.  Queried once per (device, kernel form).
#ifndef AT2_PERSIST_MAX_BLOCKS
#define AT2_PERSIST_MAX_BLOCKS 100   // mean 128-key blocks per tile up to which the grid is persistent
#endif
template <bool kMember, bool kPersist>
int at2_resident_pairs(int smem) {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * sm_count(), 1, 1);
  cfg.blockDim = dim3(AT2_THREADS, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)attn_tc2_kernel<kMember, kPersist>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = sm_count() / 2;
  }
  cache[dev] = n;
  return n;
}

void fill_border(Attn2Params& p2, const Dims& d, const SeqTable& tab) {
  std::vector<int> order(d.batch);
  for (int b = 0; b < d.batch; ++b) order[b] = b;
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return tab.nsel[x] > tab.nsel[y]; });
  for (int i = 0; i < QUOKA_MAX_BATCH; ++i) p2.border[i] = i < d.batch ? order[i] : 0;
}

// The tensor-core attention over compacted blocks kc / vc of kc_stride rows per
// (sequence, KV head): selected rows first, then the chunk rows, then zero rows.
template <int D>
quoka_status launch_attn_tc_core(const Dims& d, const SeqTable& tab, const void* q, const void* kc,
                                 const void* vc, long long kc_stride, void* out, cudaStream_t st) {
  AttnTcParams p;
  p.h_q = d.h_q;
  p.h_kv = d.h_kv;
  p.G = d.G;
  p.C = d.C;
  p.TP = 128 / d.G;
  p.b_max = 0;
  p.kc_stride = kc_stride;
  p.rows_per_head = 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  const size_t kc_rows = (size_t)d.batch * d.h_kv * kc_stride;
  cudaError_t e;
  CUtensorMap qmap, kmap, vmap;
  quoka_status s;
  if ((s = make_map_bf16(&qmap, q, (uint64_t)d.batch * d.h_q * d.C, D, 64, 1, "q_chunk")) != QUOKA_OK) return s;
  if constexpr (D == 128) {
    // SM pairs: each CTA loads 64-key halves of K tiles and 64-column halves of V tiles
    if ((s = make_map_bf16(&kmap, kc, kc_rows, D, 64, 64, "compacted K")) != QUOKA_OK) return s;
    if ((s = make_map_bf16(&vmap, vc, kc_rows, D, 64, 128, "compacted V")) != QUOKA_OK) return s;
    Attn2Params p2;
    p2.h_q = d.h_q;
    p2.h_kv = d.h_kv;
    p2.G = d.G;
    p2.C = d.C;
    p2.TP = p.TP;
    p2.kc_stride = p.kc_stride;
    p2.scale_log2 = p.scale_log2;
    fill_border(p2, d, tab);
    // One cluster per tile, or, when there are more tiles than resident clusters and the
    // tiles are short (their fill and drain then weigh more than what the hardware's
    // dynamic order of whole tiles gains), as many clusters as fit, each walking the list.
    const int npairs2 = (d.C + 2 * p.TP - 1) / (2 * p.TP);
    const long long tiles = (long long)npairs2 * d.h_kv * d.batch;
    long long blocks = 0;
    for (int b = 0; b < d.batch; ++b)
      for (int pr = 0; pr < npairs2; ++pr)
        blocks += (long long)d.h_kv * ((tab.nsel[b] + std::min(d.C, (pr + 1) * 2 * p.TP) + 127) / 128);
    const int smem_p = At2Cfg::smem(true);
    if ((e = ensure_smem(attn_tc2_kernel<false, true>, smem_p)) != cudaSuccess) return cuda_fail(e, "attn_tc2 smem");
    const long long ncl = at2_resident_pairs<false, true>(smem_p);
    if (tiles > ncl && blocks <= (long long)AT2_PERSIST_MAX_BLOCKS * tiles) {
      attn_tc2_kernel<false, true><<<dim3(2 * (unsigned)ncl), AT2_THREADS, smem_p, st>>>(
          qmap, kmap, vmap, tab, p2, reinterpret_cast<__nv_bfloat16*>(out), nullptr, nullptr, 0);
    } else {
      const int smem2 = At2Cfg::smem(false);
      if ((e = ensure_smem(attn_tc2_kernel<false, false>, smem2)) != cudaSuccess) return cuda_fail(e, "attn_tc2 smem");
      attn_tc2_kernel<false, false><<<dim3(2 * npairs2, d.h_kv, d.batch), AT2_THREADS, smem2, st>>>(
          qmap, kmap, vmap, tab, p2, reinterpret_cast<__nv_bfloat16*>(out), nullptr, nullptr, 0);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_tc2 launch");
    prof_mark(st, "attn_tc2_kernel");
    return QUOKA_OK;
  }
  if ((s = make_map_bf16(&kmap, kc, kc_rows, D, 64, 128, "compacted K")) != QUOKA_OK) return s;
  if ((s = make_map_bf16(&vmap, vc, kc_rows, D, 64, 128, "compacted V")) != QUOKA_OK) return s;
  const int smem = AtcCfg<D>::SMEM;
  if ((e = ensure_smem(attn_tc_kernel<D>, smem)) != cudaSuccess) return cuda_fail(e, "attn_tc smem");
  dim3 grid((d.C + 2 * p.TP - 1) / (2 * p.TP), d.h_kv, d.batch);
  attn_tc_kernel<D><<<grid, ATC_THREADS, smem, st>>>(qmap, kmap, vmap, tab, p,
                                                      reinterpret_cast<__nv_bfloat16*>(out));
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_tc launch");
  prof_mark(st, "attn_tc_kernel");
  return QUOKA_OK;
}

// idx_stride: entries between the idx rows of consecutive (sequence, KV head) pairs
// (b_max, or 0 when every pair reads the same list).
template <typename T, int D, int R>
quoka_status launch_attn_decode_r(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                                  const void* k, const void* v, const int32_t* idx, int b_max,
                                  void* out, unsigned char* ws, cudaStream_t st, int idx_stride) {
  using Cfg = AdcCfg<T, D>;
  long long total = 0;
  int nmax = 0;
  for (int b = 0; b < d.batch; ++b) {
    total += (long long)d.h_kv * (tab.nsel[b] + d.C);
    nmax = std::max(nmax, tab.nsel[b] + d.C);
  }
  // about eight CTAs per SM over the whole call, each at least ADC_MIN_SPLIT keys
  const long long target = (long long)sm_count() * 8;
  long long split = (total + target - 1) / target;
  split = (split + 32 * Cfg::NW - 1) / (32 * Cfg::NW) * (32 * Cfg::NW);
  split = std::min<long long>(std::max<long long>(split, ADC_MIN_SPLIT), ADC_MAX_SPLIT);
  if ((nmax + split - 1) / split > ADC_MAX_NSPLIT) {        // the merge stages one weight per split
    split = (nmax + ADC_MAX_NSPLIT - 1) / ADC_MAX_NSPLIT;
    split = (split + 32 * Cfg::NW - 1) / (32 * Cfg::NW) * (32 * Cfg::NW);
  }
  const int nsplit = (int)((nmax + split - 1) / split);
  const int nsplit_ws = decode_nsplit_ws(d, b_max);
  const int smem = adc_smem_bytes<T, D, R>();
  cudaError_t e;
  if ((e = ensure_smem(attn_decode_kernel<T, D, R>, smem)) != cudaSuccess) return cuda_fail(e, "decode smem");
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  float* part = reinterpret_cast<float*>(ws);
  attn_decode_kernel<T, D, R><<<dim3(nsplit, d.h_kv, d.batch), Cfg::THREADS, smem, st>>>(
      reinterpret_cast<const T*>(q), reinterpret_cast<const T*>(k), reinterpret_cast<const T*>(v),
      rows, tab, d.h_q, d.h_kv, d.C, idx, idx_stride, (int)split, nsplit_ws, scale_log2, part);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "decode launch");
  prof_mark(st, "attn_decode_kernel");
  attn_decode_combine_kernel<T, D, R><<<dim3(d.h_kv, d.batch), ADC_COMBINE_THREADS, nsplit * R * 4, st>>>(
      part, tab, d.h_q, d.h_kv, d.C, (int)split, nsplit_ws, reinterpret_cast<T*>(out));
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "decode combine launch");
  prof_mark(st, "attn_decode_combine_kernel");
  return QUOKA_OK;
}

template <typename T, int D>
quoka_status launch_attn_decode(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                                const void* k, const void* v, const int32_t* idx, int b_max,
                                void* out, unsigned char* ws, cudaStream_t st, int idx_stride = -1) {
  const int is = idx_stride < 0 ? b_max : idx_stride;
  switch (decode_rows(d)) {
    case 1: return launch_attn_decode_r<T, D, 1>(d, tab, rows, q, k, v, idx, b_max, out, ws, st, is);
    case 2: return launch_attn_decode_r<T, D, 2>(d, tab, rows, q, k, v, idx, b_max, out, ws, st, is);
    case 4: return launch_attn_decode_r<T, D, 4>(d, tab, rows, q, k, v, idx, b_max, out, ws, st, is);
    case 8: return launch_attn_decode_r<T, D, 8>(d, tab, rows, q, k, v, idx, b_max, out, ws, st, is);
    default: return launch_attn_decode_r<T, D, 16>(d, tab, rows, q, k, v, idx, b_max, out, ws, st, is);
  }
}

// k_new / v_new (this chunk's new K/V rows, [batch, h_kv, C, d]) or NULL: when given, the
// rows are also appended to the cache, inside the compaction pass where there is one.
template <typename T, int D>
quoka_status launch_attn(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                         const void* k, const void* v, const int32_t* idx, int b_max, void* out,
                         unsigned char* ws, cudaStream_t st, const void* k_new = nullptr,
                         const void* v_new = nullptr) {
  const bool decode = use_decode(d);
  if (d.dt == QUOKA_BF16 && !decode)
    return launch_attn_tc<D>(d, tab, rows, q, k, v, idx, b_max, out, ws, st, k_new, v_new);
  cudaError_t e;
  if (k_new) {
    const int vpr = D * (int)sizeof(T) / 16;
    const long long vecs = (long long)d.batch * d.h_kv * d.C * vpr;
    const int agrid = (int)std::min<long long>((vecs + CPT_THREADS - 1) / CPT_THREADS, (long long)sm_count() * 16);
    append_kv_kernel<<<agrid, CPT_THREADS, 0, st>>>(
        reinterpret_cast<const uint4*>(k_new), reinterpret_cast<const uint4*>(v_new),
        reinterpret_cast<uint4*>(const_cast<void*>(k)), reinterpret_cast<uint4*>(const_cast<void*>(v)),
        rows, tab, d.h_kv, d.C, vpr, vecs);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "append launch");
    prof_mark(st, "append_kv_kernel");
  }
  if (decode) return launch_attn_decode<T, D>(d, tab, rows, q, k, v, idx, b_max, out, ws, st);
  const int s = attn_simt_smem_bytes<D>();
  if ((e = ensure_smem(attn_simt_kernel<T, D>, s)) != cudaSuccess) return cuda_fail(e, "attn smem");
  dim3 grid((d.C + ATS_ROWS - 1) / ATS_ROWS, d.h_q, d.batch);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  attn_simt_kernel<T, D><<<grid, ATS_THREADS, s, st>>>(
      reinterpret_cast<const T*>(q), reinterpret_cast<const T*>(k), reinterpret_cast<const T*>(v),
      rows, tab, d.h_q, d.h_kv, d.C, idx, b_max, reinterpret_cast<T*>(out), scale_log2);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn launch");
  prof_mark(st, "attn_simt_kernel");
  return QUOKA_OK;
}

// ---- per-query selections (shared loading per tile) --------------------------------
struct PerqPlan {
  int TQ, R, ntiles, split, nsplit;
  size_t uni, memb, ucount, part, total;
};

PerqPlan perq_plan(const Dims& d, int S) {
  PerqPlan p;
  p.TQ = std::max(1, PQ_MAX_ROWS / d.G);
  p.R = 1;
  while (p.R < d.G * p.TQ) p.R *= 2;
  p.ntiles = (d.C + p.TQ - 1) / p.TQ;
  // the union of a tile is at most PQ_MAX_ROWS * S keys: up to eight splits of it
  const int nw = d.dt == QUOKA_F32 && d.D == 128 ? 2 : 4;     // AdcCfg<T, D>::NW
  const long long ub = (long long)PQ_MAX_ROWS * S;
  long long split = (ub + 7) / 8;
  split = (split + 32 * nw - 1) / (32 * nw) * (32 * nw);
  p.split = (int)std::min<long long>(std::max<long long>(split, ADC_MIN_SPLIT), ADC_MAX_SPLIT);
  p.nsplit = (int)((ub + p.split - 1) / p.split);
  const size_t nbt = (size_t)d.batch * d.h_kv * p.ntiles;
  size_t off = 0;
  p.uni = off;
  off = align_up(off + nbt * ub * 4, 256);
  p.memb = off;
  off = align_up(off + nbt * ub * 4, 256);
  p.ucount = off;
  off = align_up(off + nbt * 4, 256);
  p.part = off;
  off = align_up(off + nbt * p.nsplit * p.R * (size_t)(d.D + 4) * 4, 256);
  p.total = off;
  return p;
}

template <typename T, int D, int R>
quoka_status launch_perq_r(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                           const void* k, const void* v, const int32_t* sel, int S, void* out,
                           unsigned char* ws, const PerqPlan& pl, cudaStream_t st) {
  using Cfg = AdcCfg<T, D>;
  auto* uni = reinterpret_cast<int32_t*>(ws + pl.uni);
  auto* memb = reinterpret_cast<uint32_t*>(ws + pl.memb);
  auto* ucount = reinterpret_cast<int32_t*>(ws + pl.ucount);
  auto* part = reinterpret_cast<float*>(ws + pl.part);
  cudaError_t e;
  const int usmem = 2 * PQ_MAX_WORDS * 4;
  if ((e = ensure_smem(perq_union_kernel, usmem)) != cudaSuccess) return cuda_fail(e, "perq_union smem");
  perq_union_kernel<<<dim3(pl.ntiles, d.h_kv, d.batch), PQ_UNION_THREADS, usmem, st>>>(
      sel, tab, d.h_q, d.h_kv, d.C, S, pl.TQ, uni, memb, ucount);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "perq_union launch");
  prof_mark(st, "perq_union_kernel");
  const int smem = adc_smem_bytes<T, D, R>();
  if ((e = ensure_smem(perq_attn_kernel<T, D, R>, smem)) != cudaSuccess) return cuda_fail(e, "perq_attn smem");
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  perq_attn_kernel<T, D, R><<<dim3(pl.nsplit, pl.ntiles, d.batch * d.h_kv), Cfg::THREADS, smem, st>>>(
      reinterpret_cast<const T*>(q), reinterpret_cast<const T*>(k), reinterpret_cast<const T*>(v),
      rows, tab, d.h_q, d.h_kv, d.C, S, pl.TQ, uni, memb, ucount, pl.split, pl.nsplit, scale_log2,
      part);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "perq_attn launch");
  prof_mark(st, "perq_attn_kernel");
  perq_combine_kernel<T, D, R><<<dim3(pl.ntiles, d.batch * d.h_kv), 128, 0, st>>>(
      part, ucount, d.h_q, d.h_kv, d.C, pl.TQ, pl.split, pl.nsplit, reinterpret_cast<T*>(out));
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "perq_combine launch");
  prof_mark(st, "perq_combine_kernel");
  return QUOKA_OK;
}

template <typename T, int D>
quoka_status launch_perq(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                         const void* k, const void* v, const int32_t* sel, int S, void* out,
                         unsigned char* ws, const PerqPlan& pl, cudaStream_t st) {
  switch (pl.R) {
    case 1: return launch_perq_r<T, D, 1>(d, tab, rows, q, k, v, sel, S, out, ws, pl, st);
    case 2: return launch_perq_r<T, D, 2>(d, tab, rows, q, k, v, sel, S, out, ws, pl, st);
    case 4: return launch_perq_r<T, D, 4>(d, tab, rows, q, k, v, sel, S, out, ws, pl, st);
    case 8: return launch_perq_r<T, D, 8>(d, tab, rows, q, k, v, sel, S, out, ws, pl, st);
    default: return launch_perq_r<T, D, 16>(d, tab, rows, q, k, v, sel, S, out, ws, pl, st);
  }
}

// One step with the append: select over each sequence's prefix (when any key is to be
// kept), then attend, the chunk's new K/V rows going into the cache on the way (fused
// with the compaction where there is one).
template <typename T, int D>
quoka_status run_step(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                      const void* k_new, const void* v_new, void* k_cache, void* v_cache, int nq,
                      int b_max, int32_t* idx, void* out, unsigned char* ws, unsigned char* aws,
                      cudaStream_t st) {
  bool any = false;
  for (int b = 0; b < d.batch; ++b) any = any || tab.nsel[b] > 0;
  if (any) {
    const WsLayout w = ws_layout(d, tab.max_prefix, nq);
    quoka_status s = launch_select<T, D>(d, tab, rows, q, k_cache, nq, b_max, idx, nullptr, ws, w, st);
    if (s != QUOKA_OK) return s;
  }
  return launch_attn<T, D>(d, tab, rows, q, k_cache, v_cache, idx, b_max, out, aws, st, k_new, v_new);
}

// Whole-prompt chunked prefill: chunk c appends its K/V rows (fused with the compaction
// where there is one), selects over the c * C rows written before it, and attends.
template <typename T, int D>
quoka_status run_prefill(const Dims& d, int n_chunks, const unsigned char* q, const unsigned char* k_new,
                         const unsigned char* v_new, void* k_cache, void* v_cache, const int64_t* kv_off,
                         int nq, const int32_t* budgets, int b_max, int32_t* idx, unsigned char* out,
                         unsigned char* ws, unsigned char* aws, cudaStream_t st) {
  const size_t q_chunk = (size_t)d.batch * d.h_q * d.C * d.D * d.esz;
  const size_t kv_chunk = (size_t)d.batch * d.h_kv * d.C * d.D * d.esz;
  std::vector<int32_t> prefix(d.batch), budget(d.batch);
  for (int c = 0; c < n_chunks; ++c) {
    for (int b = 0; b < d.batch; ++b) {
      prefix[b] = c * d.C;
      budget[b] = budgets[c];
    }
    SeqTable tab;
    long long rows = 0;
    quoka_status s = build_table(d, kv_off, prefix.data(), budget.data(), b_max, &tab, &rows);
    if (s != QUOKA_OK) return s;
    s = run_step<T, D>(d, tab, rows, q + c * q_chunk, k_new + c * kv_chunk, v_new + c * kv_chunk,
                       k_cache, v_cache, nq, b_max, idx, out + c * q_chunk, ws, aws, st);
    if (s != QUOKA_OK) return s;
  }
  return QUOKA_OK;
}


// ---- selected-value cache ------------------------------------------------------------
// The cache: K blocks then V blocks, each [batch * h_kv][kc_block_rows][d] in the dtype.
size_t selcache_bytes(const Dims& d, int b_max) {
  const size_t rows = (size_t)d.batch * d.h_kv * (size_t)kc_block_rows(d, b_max);
  return 2 * align_up(rows * d.D * d.esz, 256);
}

struct SelWs {
  size_t plan_slot, plan_row, plan_count, iota, part, total;
};

// One workspace serves both calls: the update's plan, the attention's slot list and
// (decode shapes) split partials.
SelWs selcache_ws(const Dims& d, int b_max) {
  SelWs w;
  const size_t nbg = (size_t)d.batch * d.h_kv;
  size_t off = 0;
  w.plan_slot = off;
  off = align_up(off + nbg * b_max * 4, 256);
  w.plan_row = off;
  off = align_up(off + nbg * b_max * 4, 256);
  w.plan_count = off;
  off = align_up(off + nbg * 4, 256);
  w.iota = off;
  off = align_up(off + (size_t)b_max * 4, 256);
  w.part = off;
  off = align_up(off + (use_decode(d) ? attn_ws_bytes(d, b_max) : 0), 256);
  w.total = off;
  return w;
}

// Sequence table of the cache's own blocks for the gather kernels: block (b, g) starts
// at row (b * h_kv + g) * stride, so the head stride is `stride` and sequence b starts at
// b * h_kv * stride; the "prefix" is the n_b selected slots, the chunk rows follow them.
SeqTable selcache_table(const Dims& d, const SeqTable& tab, long long stride) {
  SeqTable t = tab;
  t.max_prefix = 0;
  for (int b = 0; b <= d.batch; ++b) t.kv_off[b] = (long long)b * d.h_kv * stride;
  for (int b = 0; b < d.batch; ++b) {
    t.prefix[b] = tab.nsel[b];
    t.max_prefix = std::max(t.max_prefix, tab.nsel[b]);
  }
  return t;
}

template <typename T, int D>
quoka_status launch_attn_selcache(const Dims& d, const SeqTable& tab, const void* q,
                                  const unsigned char* cache, int b_max, void* out,
                                  unsigned char* ws, const SelWs& sw, cudaStream_t st) {
  const long long stride = kc_block_rows(d, b_max);
  const unsigned char* kc = cache;
  const unsigned char* vc = cache + selcache_bytes(d, b_max) / 2;
  if (d.dt == QUOKA_BF16 && !use_decode(d))
    return launch_attn_tc_core<D>(d, tab, q, kc, vc, stride, out, st);
  cudaError_t e;
  auto* iota = reinterpret_cast<int32_t*>(ws + sw.iota);
  iota_kernel<<<(b_max + 255) / 256, 256, 0, st>>>(iota, b_max);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "iota launch");
  prof_mark(st, "iota_kernel");
  const SeqTable t2 = selcache_table(d, tab, stride);
  const long long rows = (long long)d.batch * d.h_kv * stride;
  if (use_decode(d))
    return launch_attn_decode<T, D>(d, t2, stride, q, kc, vc, iota, b_max, out, ws + sw.part, st, 0);
  const int s = attn_simt_smem_bytes<D>();
  if ((e = ensure_smem(attn_simt_kernel<T, D>, s)) != cudaSuccess) return cuda_fail(e, "attn smem");
  dim3 grid((d.C + ATS_ROWS - 1) / ATS_ROWS, d.h_q, d.batch);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  (void)rows;
  attn_simt_kernel<T, D><<<grid, ATS_THREADS, s, st>>>(
      reinterpret_cast<const T*>(q), reinterpret_cast<const T*>(kc), reinterpret_cast<const T*>(vc),
      stride, t2, d.h_q, d.h_kv, d.C, iota, 0, reinterpret_cast<T*>(out), scale_log2);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn launch");
  prof_mark(st, "attn_simt_kernel");
  return QUOKA_OK;
}

template <int VPR>
quoka_status launch_selcache_copy(const Dims& d, const SeqTable& tab, long long rows, const void* k,
                                  const void* v, int b_max, unsigned char* cache, unsigned char* ws,
                                  const SelWs& sw, cudaStream_t st) {
  const long long stride = kc_block_rows(d, b_max);
  const int nbg = d.batch * d.h_kv;
  const int copiers = std::max(1, std::min(64, 2 * sm_count() / nbg));
  selcache_copy_kernel<VPR><<<dim3(copiers, nbg), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), rows, tab, d.h_kv, d.C,
      b_max, stride, reinterpret_cast<const int32_t*>(ws + sw.plan_slot),
      reinterpret_cast<const int32_t*>(ws + sw.plan_row), reinterpret_cast<const int32_t*>(ws + sw.plan_count),
      reinterpret_cast<uint4*>(cache), reinterpret_cast<uint4*>(cache + selcache_bytes(d, b_max) / 2));
  cudaError_t e;
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "selcache_copy launch");
  prof_mark(st, "selcache_copy_kernel");
  return QUOKA_OK;
}

// ---- per-query selections on tensor cores (pair tiles of 256 rows) ----------------------
struct PerqTcPlan {
  int TP, npt, tiles, cap, mwords;
  long long stride;
  size_t uni, ucount, mask, kc, vc, total;
};

PerqTcPlan perq_tc_plan(const Dims& d, int cap) {
  PerqTcPlan p;
  p.TP = 128 / d.G;
  p.npt = (d.C + 2 * p.TP - 1) / (2 * p.TP);
  p.tiles = d.batch * d.h_kv * p.npt;
  p.cap = cap;
  p.mwords = (cap + 127) / 128 * 4;
  p.stride = (long long)align_up((size_t)cap, 128);
  size_t off = 0;
  p.uni = off;
  off = align_up(off + (size_t)p.tiles * cap * 4, 256);
  p.ucount = off;
  off = align_up(off + (size_t)p.tiles * 4, 256);
  p.mask = off;
  off = align_up(off + (size_t)p.tiles * 256 * p.mwords * 4, 256);
  p.kc = off;
  off = align_up(off + (size_t)p.tiles * p.stride * d.D * 2, 256);
  p.vc = off;
  off = align_up(off + (size_t)p.tiles * p.stride * d.D * 2, 256);
  p.total = off;
  return p;
}

quoka_status launch_perq_tc(const Dims& d, const SeqTable& tab, long long rows, const void* q,
                            const void* k, const void* v, const int32_t* sel, int S, void* out,
                            unsigned char* ws, const PerqTcPlan& pl, cudaStream_t st) {
  cudaError_t e;
  auto* uni = reinterpret_cast<int32_t*>(ws + pl.uni);
  auto* ucount = reinterpret_cast<int32_t*>(ws + pl.ucount);
  auto* mask = reinterpret_cast<uint32_t*>(ws + pl.mask);
  const int usmem = (int)perq_tc_union_smem(pl.cap);
  if ((e = ensure_smem(perq_tc_union_kernel, usmem)) != cudaSuccess) return cuda_fail(e, "perq_tc_union smem");
  perq_tc_union_kernel<<<dim3(pl.npt, d.h_kv, d.batch), PTC_THREADS, usmem, st>>>(
      sel, tab, d.h_q, d.h_kv, d.C, S, pl.TP, pl.cap, uni, ucount, mask);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "perq_tc_union launch");
  prof_mark(st, "perq_tc_union_kernel");
  const int copiers = (int)std::max<long long>(1, std::min<long long>((pl.stride * 16 + 255) / 256,
                                                                      (long long)sm_count() * 16 / pl.tiles + 1));
  perq_tc_gather_kernel<16><<<dim3(pl.tiles, copiers), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), rows, tab, d.h_kv, pl.npt,
      pl.cap, pl.stride, uni, ucount, reinterpret_cast<uint4*>(ws + pl.kc), reinterpret_cast<uint4*>(ws + pl.vc));
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "perq_tc_gather launch");
  prof_mark(st, "perq_tc_gather_kernel");
  CUtensorMap qmap, kmap, vmap;
  quoka_status s;
  const uint64_t kc_rows = (uint64_t)pl.tiles * pl.stride;
  if ((s = make_map_bf16(&qmap, q, (uint64_t)d.batch * d.h_q * d.C, 128, 64, 1, "q_chunk")) != QUOKA_OK) return s;
  if ((s = make_map_bf16(&kmap, ws + pl.kc, kc_rows, 128, 64, 64, "union K")) != QUOKA_OK) return s;
  if ((s = make_map_bf16(&vmap, ws + pl.vc, kc_rows, 128, 64, 128, "union V")) != QUOKA_OK) return s;
  Attn2Params p2;
  p2.h_q = d.h_q;
  p2.h_kv = d.h_kv;
  p2.G = d.G;
  p2.C = d.C;
  p2.TP = pl.TP;
  p2.kc_stride = pl.stride;
  p2.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  for (int i = 0; i < QUOKA_MAX_BATCH; ++i) p2.border[i] = i;   // unions are sized on the device
  const int smem2 = At2Cfg::smem(false);
  if ((e = ensure_smem(attn_tc2_kernel<true, false>, smem2)) != cudaSuccess) return cuda_fail(e, "attn_tc2 smem");
  attn_tc2_kernel<true, false><<<dim3(2 * pl.npt, d.h_kv, d.batch), AT2_THREADS, smem2, st>>>(
      qmap, kmap, vmap, tab, p2, reinterpret_cast<__nv_bfloat16*>(out), mask, ucount, pl.mwords);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_tc2 (per-query) launch");
  prof_mark(st, "attn_tc2_kernel");
  return QUOKA_OK;
}

}  // namespace

extern "C" {

int quoka_version(void) { return 101; }

quoka_status quoka_profile_events(void* const* events, int n_events) {
  if (events && n_events < 1) return fail(QUOKA_ERR_INVALID_ARG, "n_events must be >= 1");
  if (events)
    for (int i = 0; i < n_events; ++i)
      if (!events[i]) return fail(QUOKA_ERR_INVALID_ARG, "events[%d] is NULL", i);
  g_prof.events = events;
  g_prof.n = events ? n_events : 0;
  g_prof.used = 0;
  g_prof.names.clear();
  return QUOKA_OK;
}

int quoka_profile_marks(const char** names, int max_names) {
  const int n = g_prof.used;
  for (int i = 0; names && i < n && i < max_names; ++i) names[i] = g_prof.names[i];
  return n;
}

const char* quoka_last_error(void) { return g_last_error.c_str(); }

size_t quoka_select_workspace_size(const quoka_shape* shape, int max_prefix, int nq) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || max_prefix < 0 || nq < 1) return 0;
  return ws_layout(d, max_prefix, nq).total;
}

quoka_status quoka_workspace_pooled_view(const quoka_shape* shape, int max_prefix, int nq,
                                         size_t* offset, size_t* row_stride) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (max_prefix < 0 || nq < 1 || !offset || !row_stride)
    return fail(QUOKA_ERR_INVALID_ARG, "bad max_prefix/nq or NULL output");
  const WsLayout w = ws_layout(d, max_prefix, nq);
  *offset = w.pooled;
  *row_stride = (size_t)w.pooled_stride;
  return QUOKA_OK;
}

quoka_status quoka_select(const quoka_shape* shape, const void* q_chunk, const void* k_cache,
                          const int64_t* kv_off, const int32_t* prefix_len, int nq,
                          const int32_t* budget, int b_max, int32_t* idx_out, int32_t* kept_out,
                          void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (!q_chunk || !k_cache || !idx_out) return fail(QUOKA_ERR_INVALID_ARG, "q_chunk, k_cache and idx_out must be non-NULL");
  if (!aligned(q_chunk, 16) || !aligned(k_cache, 16) || !aligned(idx_out, 16) ||
      (kept_out && !aligned(kept_out, 16)))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (nq < 1) return fail(QUOKA_ERR_INVALID_ARG, "nq must be >= 1 (got %d)", nq);
  SeqTable tab;
  long long rows = 0;
  if ((s = build_table(d, kv_off, prefix_len, budget, b_max, &tab, &rows)) != QUOKA_OK) return s;
  const WsLayout w = ws_layout(d, tab.max_prefix, nq);
  if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", w.total);
  if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < w.total)
    return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, w.total);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  if (d.dt == QUOKA_F32) {
    return d.D == 64 ? launch_select<float, 64>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st)
                     : launch_select<float, 128>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st);
  }
  return d.D == 64 ? launch_select<__nv_bfloat16, 64>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st)
                   : launch_select<__nv_bfloat16, 128>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st);
}

size_t sparse_chunk_attn_workspace_size(const quoka_shape* shape, int b_max) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || b_max < 1) return 0;
  return attn_ws_bytes(d, b_max);
}

quoka_status sparse_chunk_attn(const quoka_shape* shape, const void* q_chunk, const void* k_cache,
                               const void* v_cache, const int64_t* kv_off,
                               const int32_t* prefix_len, const int32_t* budget,
                               const int32_t* idx, int b_max, void* out, void* workspace,
                               size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (!q_chunk || !k_cache || !v_cache || !idx || !out)
    return fail(QUOKA_ERR_INVALID_ARG, "q_chunk, k_cache, v_cache, idx and out must be non-NULL");
  if (!aligned(q_chunk, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(idx, 16) ||
      !aligned(out, 16))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (out == q_chunk || out == k_cache || out == v_cache)
    return fail(QUOKA_ERR_INVALID_ARG, "out must not alias an input");
  SeqTable tab;
  long long rows = 0;
  if ((s = build_table(d, kv_off, prefix_len, budget, b_max, &tab, &rows)) != QUOKA_OK) return s;
  const size_t need = attn_ws_bytes(d, b_max);
  if (need > 0) {
    if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
    if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (ws_bytes < need) return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  if (d.dt == QUOKA_F32) {
    return d.D == 64 ? launch_attn<float, 64>(d, tab, rows, q_chunk, k_cache, v_cache, idx, b_max, out, ws, st)
                     : launch_attn<float, 128>(d, tab, rows, q_chunk, k_cache, v_cache, idx, b_max, out, ws, st);
  }
  return d.D == 64 ? launch_attn<__nv_bfloat16, 64>(d, tab, rows, q_chunk, k_cache, v_cache, idx, b_max, out, ws, st)
                   : launch_attn<__nv_bfloat16, 128>(d, tab, rows, q_chunk, k_cache, v_cache, idx, b_max, out, ws, st);
}

size_t sparse_perq_attn_workspace_size(const quoka_shape* shape, int S) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || S < 1 || d.G > PQ_MAX_ROWS) return 0;
  return perq_plan(d, S).total;
}

quoka_status sparse_perq_attn(const quoka_shape* shape, const void* q_chunk, const void* k_cache,
                              const void* v_cache, const int64_t* kv_off, const int32_t* sel,
                              int S, void* out, void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (d.G > PQ_MAX_ROWS)
    return fail(QUOKA_ERR_UNSUPPORTED, "per-query attention takes at most %d query heads per KV head (got %d)",
                PQ_MAX_ROWS, d.G);
  if (!q_chunk || !k_cache || !v_cache || !kv_off || !sel || !out)
    return fail(QUOKA_ERR_INVALID_ARG, "q_chunk, k_cache, v_cache, kv_off, sel and out must be non-NULL");
  if (!aligned(q_chunk, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(sel, 16) ||
      !aligned(out, 16))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (out == q_chunk || out == k_cache || out == v_cache)
    return fail(QUOKA_ERR_INVALID_ARG, "out must not alias an input");
  if (S < 1 || S > (1 << 20)) return fail(QUOKA_ERR_INVALID_ARG, "S must be in [1, 2^20] (got %d)", S);
  if (kv_off[0] < 0) return fail(QUOKA_ERR_INVALID_ARG, "kv_off[0] must be >= 0");
  SeqTable tab;
  tab.batch = d.batch;
  tab.max_prefix = 0;
  for (int b = 0; b <= d.batch; ++b) tab.kv_off[b] = kv_off[b];
  for (int b = 0; b < QUOKA_MAX_BATCH; ++b) { tab.prefix[b] = 0; tab.nsel[b] = 0; }
  for (int b = 0; b < d.batch; ++b) {
    const long long n = kv_off[b + 1] - kv_off[b];
    if (n < 1) return fail(QUOKA_ERR_INVALID_ARG, "sequence %d owns no cache rows", b);
    if (n > (long long)PQ_MAX_WORDS * 32)
      return fail(QUOKA_ERR_UNSUPPORTED, "sequence %d owns %lld rows; per-query attention takes at most %d",
                  b, n, PQ_MAX_WORDS * 32);
  }
  const PerqPlan pl = perq_plan(d, S);
  if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", pl.total);
  if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < pl.total) return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, pl.total);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* ws = reinterpret_cast<unsigned char*>(workspace);
  const long long rows = kv_off[d.batch];
  if (d.dt == QUOKA_F32)
    return d.D == 64 ? launch_perq<float, 64>(d, tab, rows, q_chunk, k_cache, v_cache, sel, S, out, ws, pl, st)
                     : launch_perq<float, 128>(d, tab, rows, q_chunk, k_cache, v_cache, sel, S, out, ws, pl, st);
  return d.D == 64 ? launch_perq<__nv_bfloat16, 64>(d, tab, rows, q_chunk, k_cache, v_cache, sel, S, out, ws, pl, st)
                   : launch_perq<__nv_bfloat16, 128>(d, tab, rows, q_chunk, k_cache, v_cache, sel, S, out, ws, pl, st);
}

size_t quoka_step_workspace_size(const quoka_shape* shape, int max_prefix, int nq, int b_max) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || max_prefix < 0 || nq < 1 || b_max < 1) return 0;
  return align_up(ws_layout(d, max_prefix, nq).total, 256) + attn_ws_bytes(d, b_max);
}

quoka_status quoka_step(const quoka_shape* shape, const void* q_chunk, const void* k_new,
                        const void* v_new, void* k_cache, void* v_cache, const int64_t* kv_off,
                        const int32_t* prefix_len, int nq, const int32_t* budget, int b_max,
                        int32_t* idx, void* out, void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (!q_chunk || !k_new || !v_new || !k_cache || !v_cache || !idx || !out)
    return fail(QUOKA_ERR_INVALID_ARG,
                "q_chunk, k_new, v_new, k_cache, v_cache, idx and out must be non-NULL");
  if (!aligned(q_chunk, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16) || !aligned(idx, 16) || !aligned(out, 16))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (out == q_chunk || out == k_new || out == v_new || out == k_cache || out == v_cache)
    return fail(QUOKA_ERR_INVALID_ARG, "out must not alias an input");
  if (nq < 1) return fail(QUOKA_ERR_INVALID_ARG, "nq must be >= 1 (got %d)", nq);
  SeqTable tab;
  long long rows = 0;
  if ((s = build_table(d, kv_off, prefix_len, budget, b_max, &tab, &rows)) != QUOKA_OK) return s;
  const size_t sel_bytes = align_up(ws_layout(d, tab.max_prefix, nq).total, 256);
  const size_t need = sel_bytes + attn_ws_bytes(d, b_max);
  if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* ws = reinterpret_cast<unsigned char*>(workspace);
  auto* aws = ws + sel_bytes;
  if (d.dt == QUOKA_F32)
    return d.D == 64 ? run_step<float, 64>(d, tab, rows, q_chunk, k_new, v_new, k_cache, v_cache, nq, b_max, idx, out, ws, aws, st)
                     : run_step<float, 128>(d, tab, rows, q_chunk, k_new, v_new, k_cache, v_cache, nq, b_max, idx, out, ws, aws, st);
  return d.D == 64 ? run_step<__nv_bfloat16, 64>(d, tab, rows, q_chunk, k_new, v_new, k_cache, v_cache, nq, b_max, idx, out, ws, aws, st)
                   : run_step<__nv_bfloat16, 128>(d, tab, rows, q_chunk, k_new, v_new, k_cache, v_cache, nq, b_max, idx, out, ws, aws, st);
}

size_t quoka_prefill_workspace_size(const quoka_shape* shape, int n_chunks, int nq, int b_max) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || n_chunks < 1 || nq < 1 || b_max < 1) return 0;
  const long long max_prefix = (long long)(n_chunks - 1) * d.C;
  if (max_prefix > (1LL << 30)) return 0;
  return align_up(ws_layout(d, (int)max_prefix, nq).total, 256) + attn_ws_bytes(d, b_max);
}

quoka_status quoka_prefill(const quoka_shape* shape, int n_chunks, const void* q, const void* k_new,
                           const void* v_new, void* k_cache, void* v_cache, const int64_t* kv_off,
                           int nq, const int32_t* budgets, int b_max, int32_t* idx, void* out,
                           void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (n_chunks < 1) return fail(QUOKA_ERR_INVALID_ARG, "n_chunks must be >= 1 (got %d)", n_chunks);
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !kv_off || !budgets || !idx || !out)
    return fail(QUOKA_ERR_INVALID_ARG,
                "q, k_new, v_new, k_cache, v_cache, kv_off, budgets, idx and out must be non-NULL");
  if (!aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16) || !aligned(idx, 16) || !aligned(out, 16))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (out == q || out == k_new || out == v_new || out == k_cache || out == v_cache)
    return fail(QUOKA_ERR_INVALID_ARG, "out must not alias an input");
  if (nq < 1) return fail(QUOKA_ERR_INVALID_ARG, "nq must be >= 1 (got %d)", nq);
  if (b_max < 1) return fail(QUOKA_ERR_INVALID_ARG, "b_max must be >= 1 (got %d)", b_max);
  const long long rows_needed = (long long)n_chunks * d.C;
  if (rows_needed > (1LL << 30))
    return fail(QUOKA_ERR_UNSUPPORTED, "a prompt of %lld tokens is too long", rows_needed);
  for (int c = 0; c < n_chunks; ++c)
    if (budgets[c] < 0 || budgets[c] > b_max)
      return fail(QUOKA_ERR_INVALID_ARG, "budgets[%d] = %d outside [0, b_max=%d]", c, budgets[c], b_max);
  if (kv_off[0] < 0) return fail(QUOKA_ERR_INVALID_ARG, "kv_off[0] must be >= 0");
  for (int b = 0; b < d.batch; ++b)
    if (kv_off[b + 1] - kv_off[b] < rows_needed)
      return fail(QUOKA_ERR_INVALID_ARG, "sequence %d owns %lld cache rows, fewer than the prompt's %lld",
                  b, (long long)(kv_off[b + 1] - kv_off[b]), rows_needed);
  const size_t sel_bytes = align_up(ws_layout(d, (int)((n_chunks - 1) * d.C), nq).total, 256);
  const size_t need = sel_bytes + attn_ws_bytes(d, b_max);
  if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* ws = reinterpret_cast<unsigned char*>(workspace);
  auto* aws = ws + sel_bytes;
  const auto* qb = reinterpret_cast<const unsigned char*>(q);
  const auto* kn = reinterpret_cast<const unsigned char*>(k_new);
  const auto* vn = reinterpret_cast<const unsigned char*>(v_new);
  auto* ob = reinterpret_cast<unsigned char*>(out);
  if (d.dt == QUOKA_F32)
    return d.D == 64 ? run_prefill<float, 64>(d, n_chunks, qb, kn, vn, k_cache, v_cache, kv_off, nq, budgets, b_max, idx, ob, ws, aws, st)
                     : run_prefill<float, 128>(d, n_chunks, qb, kn, vn, k_cache, v_cache, kv_off, nq, budgets, b_max, idx, ob, ws, aws, st);
  return d.D == 64 ? run_prefill<__nv_bfloat16, 64>(d, n_chunks, qb, kn, vn, k_cache, v_cache, kv_off, nq, budgets, b_max, idx, ob, ws, aws, st)
                   : run_prefill<__nv_bfloat16, 128>(d, n_chunks, qb, kn, vn, k_cache, v_cache, kv_off, nq, budgets, b_max, idx, ob, ws, aws, st);
}

size_t sparse_perq_attn_tc_workspace_size(const quoka_shape* shape, int S, int max_union) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || S < 1 || max_union < 1) return 0;
  if (d.dt != QUOKA_BF16 || d.D != 128) return 0;
  if (perq_tc_union_smem(max_union) > 227u * 1024u) return 0;
  return perq_tc_plan(d, max_union).total;
}

quoka_status sparse_perq_attn_tc(const quoka_shape* shape, const void* q_chunk, const void* k_cache,
                                 const void* v_cache, const int64_t* kv_off, const int32_t* sel, int S,
                                 int max_union, void* out, void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (d.dt != QUOKA_BF16 || d.D != 128)
    return fail(QUOKA_ERR_UNSUPPORTED, "the tensor-core per-query attention takes bf16 with head_dim 128");
  if (!q_chunk || !k_cache || !v_cache || !kv_off || !sel || !out)
    return fail(QUOKA_ERR_INVALID_ARG, "q_chunk, k_cache, v_cache, kv_off, sel and out must be non-NULL");
  if (!aligned(q_chunk, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(sel, 16) ||
      !aligned(out, 16))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (out == q_chunk || out == k_cache || out == v_cache)
    return fail(QUOKA_ERR_INVALID_ARG, "out must not alias an input");
  if (S < 1 || S > (1 << 20)) return fail(QUOKA_ERR_INVALID_ARG, "S must be in [1, 2^20] (got %d)", S);
  if (max_union < 1) return fail(QUOKA_ERR_INVALID_ARG, "max_union must be >= 1 (got %d)", max_union);
  if (perq_tc_union_smem(max_union) > 227u * 1024u)
    return fail(QUOKA_ERR_UNSUPPORTED, "max_union %d is too large for one tile's masks", max_union);
  if (kv_off[0] < 0) return fail(QUOKA_ERR_INVALID_ARG, "kv_off[0] must be >= 0");
  SeqTable tab;
  tab.batch = d.batch;
  tab.max_prefix = 0;
  for (int b = 0; b <= d.batch; ++b) tab.kv_off[b] = kv_off[b];
  for (int b = d.batch + 1; b <= QUOKA_MAX_BATCH; ++b) tab.kv_off[b] = kv_off[d.batch];
  for (int b = 0; b < QUOKA_MAX_BATCH; ++b) { tab.prefix[b] = 0; tab.nsel[b] = 0; }
  for (int b = 0; b < d.batch; ++b) {
    const long long n = kv_off[b + 1] - kv_off[b];
    if (n < 1) return fail(QUOKA_ERR_INVALID_ARG, "sequence %d owns no cache rows", b);
    if (n > (long long)PTC_MAX_WORDS * 32)
      return fail(QUOKA_ERR_UNSUPPORTED, "sequence %d owns %lld rows; at most %d", b, n, PTC_MAX_WORDS * 32);
  }
  const PerqTcPlan pl = perq_tc_plan(d, max_union);
  if ((long long)pl.tiles * pl.stride >= (1ll << 31))
    return fail(QUOKA_ERR_UNSUPPORTED, "tiles x max_union too large");
  if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", pl.total);
  if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < pl.total) return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, pl.total);
  return launch_perq_tc(d, tab, kv_off[d.batch], q_chunk, k_cache, v_cache, sel, S, out,
                        reinterpret_cast<unsigned char*>(workspace), pl, reinterpret_cast<cudaStream_t>(stream));
}

size_t quoka_selcache_bytes(const quoka_shape* shape, int b_max) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || b_max < 1) return 0;
  return selcache_bytes(d, b_max);
}

size_t quoka_selcache_workspace_size(const quoka_shape* shape, int b_max) {
  Dims d;
  if (check_shape(shape, &d) != QUOKA_OK || b_max < 1) return 0;
  return selcache_ws(d, b_max).total;
}

quoka_status quoka_selcache_update(const quoka_shape* shape, const void* k_cache, const void* v_cache,
                                   const int64_t* kv_off, const int32_t* prefix_len,
                                   const int32_t* budget, const int32_t* idx, int b_max,
                                   void* sel_cache, int32_t* slot_rows, int32_t* misses,
                                   void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (!k_cache || !v_cache || !idx || !sel_cache || !slot_rows)
    return fail(QUOKA_ERR_INVALID_ARG, "k_cache, v_cache, idx, sel_cache and slot_rows must be non-NULL");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(idx, 16) || !aligned(sel_cache, 256) ||
      !aligned(slot_rows, 16) || (misses && !aligned(misses, 16)))
    return fail(QUOKA_ERR_INVALID_ARG,
                "device pointers must be 16-byte aligned (sel_cache 256-byte aligned)");
  if (sel_cache == k_cache || sel_cache == v_cache)
    return fail(QUOKA_ERR_INVALID_ARG, "sel_cache must not alias the cache");
  SeqTable tab;
  long long rows = 0;
  if ((s = build_table(d, kv_off, prefix_len, budget, b_max, &tab, &rows)) != QUOKA_OK) return s;
  const size_t smem = selcache_plan_smem(tab.max_prefix, b_max);
  if (smem > 227u * 1024u)
    return fail(QUOKA_ERR_UNSUPPORTED, "prefix %d with b_max %d is too long for the selected-value cache",
                tab.max_prefix, b_max);
  const SelWs sw = selcache_ws(d, b_max);
  if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", sw.total);
  if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < sw.total) return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, sw.total);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* ws = reinterpret_cast<unsigned char*>(workspace);
  cudaError_t e;
  if ((e = ensure_smem(selcache_plan_kernel, (int)smem)) != cudaSuccess) return cuda_fail(e, "selcache_plan smem");
  selcache_plan_kernel<<<dim3(d.h_kv, d.batch), SCP_THREADS, smem, st>>>(
      tab, d.h_kv, b_max, idx, slot_rows, reinterpret_cast<int32_t*>(ws + sw.plan_slot),
      reinterpret_cast<int32_t*>(ws + sw.plan_row), reinterpret_cast<int32_t*>(ws + sw.plan_count), misses);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "selcache_plan launch");
  prof_mark(st, "selcache_plan_kernel");
  auto* cache = reinterpret_cast<unsigned char*>(sel_cache);
  switch (d.D * d.esz / 16) {
    case 8: return launch_selcache_copy<8>(d, tab, rows, k_cache, v_cache, b_max, cache, ws, sw, st);
    case 16: return launch_selcache_copy<16>(d, tab, rows, k_cache, v_cache, b_max, cache, ws, sw, st);
    default: return launch_selcache_copy<32>(d, tab, rows, k_cache, v_cache, b_max, cache, ws, sw, st);
  }
}

quoka_status sparse_chunk_attn_selcache(const quoka_shape* shape, const void* q_chunk,
                                        const int32_t* prefix_len, const int32_t* budget,
                                        const void* sel_cache, int b_max, void* out,
                                        void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (!q_chunk || !sel_cache || !out || !prefix_len || !budget)
    return fail(QUOKA_ERR_INVALID_ARG, "q_chunk, prefix_len, budget, sel_cache and out must be non-NULL");
  if (!aligned(q_chunk, 16) || !aligned(sel_cache, 256) || !aligned(out, 16))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned (sel_cache 256-byte aligned)");
  if (out == q_chunk || out == sel_cache) return fail(QUOKA_ERR_INVALID_ARG, "out must not alias an input");
  if (b_max < 1) return fail(QUOKA_ERR_INVALID_ARG, "b_max must be >= 1 (got %d)", b_max);
  SeqTable tab;
  tab.batch = d.batch;
  tab.max_prefix = 0;
  for (int b = 0; b <= QUOKA_MAX_BATCH; ++b) tab.kv_off[b] = 0;
  for (int b = 0; b < QUOKA_MAX_BATCH; ++b) { tab.prefix[b] = 0; tab.nsel[b] = 0; }
  for (int b = 0; b < d.batch; ++b) {
    if (prefix_len[b] < 0) return fail(QUOKA_ERR_INVALID_ARG, "prefix_len[%d] = %d < 0", b, prefix_len[b]);
    if (budget[b] < 0 || budget[b] > b_max)
      return fail(QUOKA_ERR_INVALID_ARG, "budget[%d] = %d outside [0, b_max=%d]", b, budget[b], b_max);
    tab.prefix[b] = prefix_len[b];
    tab.nsel[b] = std::min(budget[b], prefix_len[b]);
    tab.max_prefix = std::max(tab.max_prefix, prefix_len[b]);
  }
  const SelWs sw = selcache_ws(d, b_max);
  if (!workspace) return fail(QUOKA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", sw.total);
  if (!aligned(workspace, 256)) return fail(QUOKA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < sw.total) return fail(QUOKA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, sw.total);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* ws = reinterpret_cast<unsigned char*>(workspace);
  const auto* cache = reinterpret_cast<const unsigned char*>(sel_cache);
  if (d.dt == QUOKA_F32)
    return d.D == 64 ? launch_attn_selcache<float, 64>(d, tab, q_chunk, cache, b_max, out, ws, sw, st)
                     : launch_attn_selcache<float, 128>(d, tab, q_chunk, cache, b_max, out, ws, sw, st);
  return d.D == 64 ? launch_attn_selcache<__nv_bfloat16, 64>(d, tab, q_chunk, cache, b_max, out, ws, sw, st)
                   : launch_attn_selcache<__nv_bfloat16, 128>(d, tab, q_chunk, cache, b_max, out, ws, sw, st);
}

}  // extern "C"

// ---- allocation-free variant of quoka_select --------------------------------------
// The scratch is one file-scope device array.  In host code its name is only a
// host-side stand-in, so its device address is looked up per device with
// cudaGetSymbolAddress (with that device current) and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QUOKA_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
// (device ordinal, unique ID of the context current on it) -> device address of the
// array.  A device reset destroys the primary context and the next one loads the module
// again, possibly elsewhere; its new context ID makes the lookup run again.
std::map<std::pair<int, unsigned long long>, void*> g_noalloc_addr;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique ID of the calling thread's current context (0 if the driver cannot say).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur && get_id && get_cur(&ctx) == CUDA_SUCCESS && ctx) get_id(ctx, &id);
  return id;
}

quoka_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = current_context_id();
  if (id != 0) {
    auto it = g_noalloc_addr.find(std::make_pair(dev, id));
    if (it != g_noalloc_addr.end()) {
      *out = it->second;
      return QUOKA_OK;
    }
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // creates the context if need be
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the built-in scratch");
  id = current_context_id();
  if (id != 0) g_noalloc_addr[std::make_pair(dev, id)] = p;   // else: looked up every call
  *out = p;
  return QUOKA_OK;
}
}  // namespace

extern "C" {

quoka_status quoka_select_noalloc(const quoka_shape* shape, const void* q_chunk,
                                  const void* k_cache, const int64_t* kv_off,
                                  const int32_t* prefix_len, int nq, const int32_t* budget,
                                  int b_max, int32_t* idx_out, int32_t* kept_out, void* stream) {
  Dims d;
  quoka_status s = check_shape(shape, &d);
  if (s != QUOKA_OK) return s;
  if (!q_chunk || !k_cache || !idx_out) return fail(QUOKA_ERR_INVALID_ARG, "q_chunk, k_cache and idx_out must be non-NULL");
  if (!aligned(q_chunk, 16) || !aligned(k_cache, 16) || !aligned(idx_out, 16) ||
      (kept_out && !aligned(kept_out, 16)))
    return fail(QUOKA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (nq < 1) return fail(QUOKA_ERR_INVALID_ARG, "nq must be >= 1 (got %d)", nq);
  SeqTable tab;
  long long rows = 0;
  if ((s = build_table(d, kv_off, prefix_len, budget, b_max, &tab, &rows)) != QUOKA_OK) return s;
  const WsLayout w = ws_layout(d, tab.max_prefix, nq);
  if (w.total > (size_t)QUOKA_NOALLOC_SCRATCH_BYTES)
    return fail(QUOKA_ERR_WORKSPACE,
                "this call needs %zu bytes of scratch; the built-in scratch holds %zu "
                "(use quoka_select with a caller workspace)", w.total,
                (size_t)QUOKA_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != QUOKA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(scratch);
  if (d.dt == QUOKA_F32) {
    return d.D == 64 ? launch_select<float, 64>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st)
                     : launch_select<float, 128>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st);
  }
  return d.D == 64 ? launch_select<__nv_bfloat16, 64>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st)
                   : launch_select<__nv_bfloat16, 128>(d, tab, rows, q_chunk, k_cache, nq, b_max, idx_out, kept_out, ws, w, st);
}

quoka_status quoka_device_error(uint32_t* code, void* stream) {
  if (!code) return fail(QUOKA_ERR_INVALID_ARG, "code is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  *code = v;
  return QUOKA_OK;
}

}  // extern "C"
