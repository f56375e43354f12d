// C-ABI layer (include/hyb_attn.h): argument checks, tensor-map encoding,
// launch sequencing.  Host code only; every step of the computation runs in
// the kernels of rope_kv.cu, prefill.cu and decode.cu.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "hyb_attn.h"
#include "common.cuh"
#include "launch.h"

namespace hyb {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static void* const* g_prof_events = nullptr;
static int g_prof_pairs = 0;
static int g_prof_used = 0;
// A failed record (e.g. a handle that is not a live event) disables
// profiling and clears the error, so it never surfaces as a launch failure.
static void profile_record(int idx, cudaStream_t st) {
  if (cudaEventRecord(reinterpret_cast<cudaEvent_t>(g_prof_events[idx]), st) != cudaSuccess) {
    (void)cudaGetLastError();
    g_prof_events = nullptr;
  }
}
void profile_before(cudaStream_t st) {
  if (g_prof_events && g_prof_used < g_prof_pairs) profile_record(2 * g_prof_used, st);
}
void profile_after(cudaStream_t st) {
  if (g_prof_events && g_prof_used < g_prof_pairs) {
    profile_record(2 * g_prof_used + 1, st);
    ++g_prof_used;
  }
}

cudaError_t decode_set_smem_attr();
cudaError_t prefill_set_smem_attr();

}  // namespace hyb

using namespace hyb;

namespace {

thread_local std::string t_err;

hyb_status fail(hyb_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return s;
}

hyb_status cuda_fail(cudaError_t e, const char* what) {
  return fail(HYB_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device one-time set-up: architecture check and the dynamic shared
// memory opt-in of the two large kernels.
std::mutex g_mu;
int g_dev_state[128];  // 0 unknown, 1 ready, -1 unsupported
int g_dev_sms[128];    // multiprocessor count

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128 || g_dev_sms[dev] <= 0) return 148;
  return g_dev_sms[dev];
}

hyb_status ensure_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 128) return fail(HYB_EUNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev_state[dev] == 1) return HYB_OK;
  if (g_dev_state[dev] == -1) return fail(HYB_EUNSUPPORTED, "device %d is not an sm_100 (B200) GPU", dev);
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) {
    g_dev_state[dev] = -1;
    return fail(HYB_EUNSUPPORTED, "device %d has compute capability %d.%d; this library is built for sm_100a",
                dev, major, minor);
  }
  {  // rotation frequencies of both layer types, fp64 on the host
    double f[2][128] = {};
    for (int k = 0; k < RopeCfg<false>::R / 2; ++k)
      f[0][k] = std::pow(RopeCfg<false>::theta, -2.0 * k / RopeCfg<false>::R);
    for (int k = 0; k < RopeCfg<true>::R / 2; ++k)
      f[1][k] = std::pow(RopeCfg<true>::theta, -2.0 * k / RopeCfg<true>::R);
    if ((e = cudaMemcpyToSymbol(g_inv_freq, f, sizeof(f))) != cudaSuccess) return cuda_fail(e, "frequency table");
  }
  if ((e = prefill_set_smem_attr()) != cudaSuccess) return cuda_fail(e, "prefill smem attribute");
  cudaDeviceGetAttribute(&g_dev_sms[dev], cudaDevAttrMultiProcessorCount, dev);
  if ((e = decode_set_smem_attr()) != cudaSuccess) return cuda_fail(e, "decode smem attribute");
  if ((e = gemm_set_smem_attr()) != cudaSuccess) return cuda_fail(e, "linear smem attribute");
  g_dev_state[dev] = 1;
  return HYB_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D map {256 dims, rows, 4 KV heads, batch} of bf16 with boxes of 64 dims x
// box_rows rows and 128-byte swizzle (one box = box_rows rows of 128 bytes).
hyb_status make_kv_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t batch, uint64_t row_bytes,
                       uint64_t head_bytes, uint64_t batch_bytes, uint32_t box_rows, const char* what) {
  auto enc = encode_fn();
  if (!enc) return fail(HYB_EUNSUPPORTED, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[4] = {(cuuint64_t)kD, rows, (cuuint64_t)kHkv, batch};
  cuuint64_t strides[3] = {row_bytes, head_bytes, batch_bytes};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HYB_ECUDA, "cuTensorMapEncodeTiled(%s) failed with CUresult %d", what, (int)r);
  return HYB_OK;
}

// 4-D map {256 dims, 16 heads, T tokens, batch} over query-shaped rows (the
// raw queries, or the output) with boxes of 64 dims x 1 head x box_rows tokens.
hyb_status make_q_map(CUtensorMap* m, const void* base, uint64_t T, uint64_t batch, uint64_t token_bytes,
                      uint32_t box_rows, const char* what) {
  auto enc = encode_fn();
  if (!enc) return fail(HYB_EUNSUPPORTED, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)kHq, T, batch};
  cuuint64_t strides[3] = {(cuuint64_t)kD * 2, token_bytes, T * token_bytes};
  cuuint32_t box[4] = {64, 1, box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HYB_ECUDA, "cuTensorMapEncodeTiled(%s) failed with CUresult %d", what, (int)r);
  return HYB_OK;
}

// 4-D map {256 dims, 16 heads, T tokens, batch} over the bf16 output with boxes
// of 32 dims x 1 head x 32 tokens and 64-byte swizzle: one softmax warp's 32
// rows x 32 dims of the prefill epilogue per store.
hyb_status make_out_map(CUtensorMap* m, void* base, uint64_t T, uint64_t batch) {
  auto enc = encode_fn();
  if (!enc) return fail(HYB_EUNSUPPORTED, "cuTensorMapEncodeTiled is not available from the driver");
  const uint64_t token_bytes = (uint64_t)kHq * kD * 2;
  cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)kHq, T, batch};
  cuuint64_t strides[3] = {(cuuint64_t)kD * 2, token_bytes, T * token_bytes};
  cuuint32_t box[4] = {32, 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HYB_ECUDA, "cuTensorMapEncodeTiled(out) failed with CUresult %d", (int)r);
  return HYB_OK;
}

// Rows per (page or sequence) and pages (or sequences) of a cache's storage:
// a contiguous cache is [batch][4][capacity][256], a paged one
// [n_pages][4][page_size][256].
void cache_geom(const hyb_kv_cache* c, uint64_t* rows, uint64_t* batches) {
  if (c->page_size > 0) {
    *rows = (uint64_t)c->page_size;
    *batches = (uint64_t)c->n_pages;
  } else {
    *rows = (uint64_t)c->capacity;
    *batches = (uint64_t)c->batch;
  }
}

PageMap page_map(const hyb_kv_cache* c) {
  PageMap pm;
  if (c->page_size > 0) {
    pm.table = c->block_table;
    pm.page = c->page_size;
    pm.max_pages = c->max_pages;
    pm.n_pages = (int)c->n_pages;
  }
  return pm;
}

// FP8 cache maps: codes {256, rows, 4, batches} uint8 with 128-dim x 64-row
// boxes (128-byte swizzle), scales {rows, 4, batches} fp32 with 64-row boxes.
hyb_status cache_maps_fp8(const hyb_kv_cache* c, CUtensorMap* mk, CUtensorMap* mv, CUtensorMap* mks,
                          CUtensorMap* mvs) {
  auto enc = encode_fn();
  if (!enc) return fail(HYB_EUNSUPPORTED, "cuTensorMapEncodeTiled is not available from the driver");
  uint64_t cap, nb;
  cache_geom(c, &cap, &nb);
  cuuint64_t dims[4] = {(cuuint64_t)kD, cap, (cuuint64_t)kHkv, (cuuint64_t)nb};
  cuuint64_t strides[3] = {(cuuint64_t)kD, cap * kD, cap * kD * kHkv};
  cuuint32_t box[4] = {128, 64, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  void* bases[2] = {c->k, c->v};
  CUtensorMap* maps[2] = {mk, mv};
  for (int i = 0; i < 2; ++i) {
    CUresult r = enc(maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, bases[i], dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(HYB_ECUDA, "cuTensorMapEncodeTiled(FP8 cache) failed with CUresult %d", (int)r);
  }
  cuuint64_t sdims[3] = {cap, (cuuint64_t)kHkv, (cuuint64_t)nb};
  cuuint64_t sstrides[2] = {cap * 4, cap * 4 * kHkv};
  cuuint32_t sbox[3] = {64, 1, 1};
  cuuint32_t sestr[3] = {1, 1, 1};
  void* sbases[2] = {c->k_scale, c->v_scale};
  CUtensorMap* smaps[2] = {mks, mvs};
  for (int i = 0; i < 2; ++i) {
    CUresult r = enc(smaps[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, sbases[i], sdims, sstrides, sbox, sestr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(HYB_ECUDA, "cuTensorMapEncodeTiled(FP8 scales) failed with CUresult %d", (int)r);
  }
  return HYB_OK;
}

hyb_status check_cache(const hyb_kv_cache* c) {
  if (!c) return fail(HYB_EINVAL, "cache is NULL");
  if (c->type != HYB_SLIDING && c->type != HYB_FULL) return fail(HYB_EINVAL, "cache type %d invalid", c->type);
  if (c->batch <= 0) return fail(HYB_EINVAL, "cache batch %d must be positive", c->batch);
  if (!c->k || !c->v || !c->len) return fail(HYB_EINVAL, "cache k, v and len must be non-NULL");
  if (!aligned16(c->k) || !aligned16(c->v)) return fail(HYB_EALIGN, "cache k/v must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(c->len) & 3u) != 0) return fail(HYB_EALIGN, "cache len must be 4-byte aligned");
  if (c->kv_dtype != HYB_KV_BF16 && c->kv_dtype != HYB_KV_FP8)
    return fail(HYB_EINVAL, "cache kv_dtype %d invalid", c->kv_dtype);
  if (c->kv_dtype == HYB_KV_FP8) {
    if (!c->k_scale || !c->v_scale) return fail(HYB_EINVAL, "an FP8 cache needs k_scale and v_scale buffers");
    if (!aligned16(c->k_scale) || !aligned16(c->v_scale)) return fail(HYB_EALIGN, "cache scales must be 16-byte aligned");
    if (c->capacity % 4) return fail(HYB_ESHAPE, "an FP8 cache needs capacity % 4 == 0, got %lld", (long long)c->capacity);
  }
  if (c->page_size < 0) return fail(HYB_EINVAL, "page_size %d must be >= 0", c->page_size);
  if (c->page_size > 0) {
    if (c->type != HYB_FULL) return fail(HYB_EINVAL, "only full-layer caches can be paged");
    if (c->page_size % 64) return fail(HYB_ESHAPE, "page_size %d must be a multiple of 64", c->page_size);
    if (c->max_pages <= 0) return fail(HYB_EINVAL, "max_pages %d must be positive", c->max_pages);
    if (c->n_pages <= 0 || c->n_pages > (int64_t)0x7fffffff)
      return fail(HYB_EINVAL, "n_pages %lld out of range [1, 2^31)", (long long)c->n_pages);
    if (c->capacity != (int64_t)c->max_pages * c->page_size)
      return fail(HYB_ESHAPE, "capacity %lld must equal max_pages %d x page_size %d", (long long)c->capacity,
                  c->max_pages, c->page_size);
    if (!c->block_table) return fail(HYB_EINVAL, "a paged cache needs a block_table");
    if (reinterpret_cast<uintptr_t>(c->block_table) & 3u) return fail(HYB_EALIGN, "block_table must be 4-byte aligned");
  }
  if (c->type == HYB_SLIDING) {
    if (c->capacity != kWindow) return fail(HYB_ESHAPE, "sliding cache capacity must be 512, got %lld",
                                            (long long)c->capacity);
    if (!c->head || !c->tag) return fail(HYB_EINVAL, "sliding cache needs head and tag buffers");
  } else {
    if (c->capacity <= 0 || c->capacity > (int64_t)0x7fffffff)
      return fail(HYB_ESHAPE, "full cache capacity %lld out of range [1, 2^31)", (long long)c->capacity);
  }
  return HYB_OK;
}

hyb_status cache_maps(const hyb_kv_cache* c, CUtensorMap* mk, CUtensorMap* mv, uint32_t k_box_rows,
                      uint32_t v_box_rows) {
  uint64_t rows, nb;
  cache_geom(c, &rows, &nb);
  const uint64_t row = kD * 2, head = rows * row, batch = head * kHkv;
  hyb_status s = make_kv_map(mk, c->k, rows, nb, row, head, batch, k_box_rows, "cache K");
  if (s != HYB_OK) return s;
  return make_kv_map(mv, c->v, rows, nb, row, head, batch, v_box_rows, "cache V");
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

size_t ctx_rows(int32_t T) { return (size_t)(kWindow - 1) + (size_t)T; }

}  // namespace

extern "C" {

const char* hyb_last_error(void) { return t_err.c_str(); }

uint64_t hyb_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t hyb_build_flags(void) { return hyb::kBuildFlags ? HYB_BUILD_DEBUG_BOUNDS : 0; }

hyb_status hyb_profile_events(void* const* events, int32_t n_pairs) {
  if (n_pairs < 0) return fail(HYB_EINVAL, "n_pairs %d negative", n_pairs);
  hyb::g_prof_events = (n_pairs > 0) ? events : nullptr;
  hyb::g_prof_pairs = (events != nullptr) ? n_pairs : 0;
  hyb::g_prof_used = 0;
  return HYB_OK;
}

int32_t hyb_profile_pairs_used(void) { return hyb::g_prof_used; }

hyb_status hyb_device_error(int32_t* flags, int32_t clear, void* stream) {
  if (!flags) return fail(HYB_EINVAL, "flags is NULL");
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  if ((e = cudaMemcpyFromSymbol(&v, g_dev_err, sizeof(int))) != cudaSuccess) return cuda_fail(e, "read error word");
  *flags = v;
  if (clear) {
    const int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(int))) != cudaSuccess)
      return cuda_fail(e, "clear error word");
  }
  return HYB_OK;
}

namespace {
// 2-D map over a row-major bf16 matrix [rows][ld] (K = cols used), 64 x 128 boxes
hyb_status make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                         const char* what) {
  auto enc = encode_fn();
  if (!enc) return fail(HYB_EUNSUPPORTED, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)gemm_box_k(), (cuuint32_t)gemm_box_rows()};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HYB_ECUDA, "cuTensorMapEncodeTiled(%s) failed with CUresult %d", what, (int)r);
  return HYB_OK;
}

// rope: 0 none; 1 / 2 rotate the 256-wide column tiles below rope_cols as a
// sliding / full layer's heads (see GemmHost)
// rope != 0: RoPE epilogue on the column tiles below rope_cols, with the
// (cos, sin) table of the M rows written first into `rot` (float2 [M][R/2])
// w2 != NULL: a second output group of N2 columns, y2[M][ldy2] = X w2[N2][K]^T,
// computed in the same launch as columns N .. N + N2 - 1 (N a multiple of 256)
hyb_status linear_impl(const void* x, int64_t ldx, const void* w, int64_t ldw, void* y, int64_t ldy, int32_t M,
                       int32_t N, int32_t K, void* stream, int rope = 0, int rope_cols = 0, int32_t T = 0,
                       const int32_t* pos = nullptr, const int32_t* len = nullptr, void* rot = nullptr,
                       const void* w2 = nullptr, int64_t ldw2 = 0, void* y2 = nullptr, int64_t ldy2 = 0,
                       int32_t N2 = 0, bool w_not_written_by_previous = false) {
  if (!x || !w || !y) return fail(HYB_EINVAL, "x, w and y must not be NULL");
  if (M <= 0 || N <= 0 || K <= 0) return fail(HYB_ESHAPE, "M, N, K must be positive (got %d, %d, %d)", M, N, K);
  if (N % 8 || K % 8) return fail(HYB_ESHAPE, "N and K must be multiples of 8 (got %d, %d)", N, K);
  if (ldx < K || ldw < K || ldy < N) return fail(HYB_ESHAPE, "row strides must cover the rows (ldx, ldw >= K; ldy >= N)");
  if (ldx % 8 || ldw % 8 || ldy % 8) return fail(HYB_EALIGN, "row strides must be multiples of 8 elements");
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return fail(HYB_EALIGN, "x, w and y must be 16-byte aligned");
  hyb_status s = ensure_device();
  if (s != HYB_OK) return s;
  if (w2 != nullptr && (N % 256 || N2 <= 0 || N2 % 8 || ldw2 < K || ldy2 < N2 || ldw2 % 8 || ldy2 % 8 || !y2 ||
                        !aligned16(w2) || !aligned16(y2)))
    return fail(HYB_ESHAPE, "second output group: N %% 256, N2 %% 8, strides or alignment");
  if (rope == 0 && smallm_supported(M, N + (w2 ? N2 : 0), K, N)) {
    // a few rows (decode steps): stream W over every SM instead of 256-row tiles
    SmallMHost sh;
    sh.x = x;
    sh.ldx = ldx;
    sh.w = w;
    sh.ldw = ldw;
    sh.w2 = w2;
    sh.ldw2 = ldw2;
    sh.y = y;
    sh.ldy = ldy;
    sh.y2 = y2;
    sh.ldy2 = ldy2;
    sh.n_main = w2 ? N : 0;
    sh.M = M;
    sh.N = N + (w2 ? N2 : 0);
    sh.K = K;
    sh.early_w = w_not_written_by_previous;
    const cudaError_t e = launch_smallm(sh, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "few-row linear launch");
    return HYB_OK;
  }
  GemmHost gh;
  if ((s = make_rows_map(&gh.tm_x, x, (uint64_t)M, (uint64_t)K, (uint64_t)ldx, "x")) != HYB_OK) return s;
  if ((s = make_rows_map(&gh.tm_w, w, (uint64_t)N, (uint64_t)K, (uint64_t)ldw, "w")) != HYB_OK) return s;
  gh.tm_w2 = gh.tm_w;
  gh.y = y;
  gh.ldy = ldy;
  gh.M = M;
  gh.N = N;
  if (w2 != nullptr) {
    if ((s = make_rows_map(&gh.tm_w2, w2, (uint64_t)N2, (uint64_t)K, (uint64_t)ldw2, "w2")) != HYB_OK) return s;
    gh.y2 = y2;
    gh.ldy2 = ldy2;
    gh.n_main = N;
    gh.N = N + N2;
  }
  gh.K = K;
  gh.n_pairs = device_sms() / 2;
  gh.rope = rope;
  gh.rope_cols = rope_cols;
  gh.T = T;
  gh.rot = rot;
  cudaError_t e;
  if (rope != 0) {
    if (!rot) return fail(HYB_EINVAL, "RoPE epilogue without its table");
    if ((e = launch_rope_table(rope == 2, pos, len, T, M, rot, as_stream(stream))) != cudaSuccess)
      return cuda_fail(e, "rope table launch");
  }
  e = launch_gemm(gh, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "linear launch");
  return HYB_OK;
}
}  // namespace

hyb_status hyb_linear(const void* x, int64_t ldx, const void* w, int64_t ldw, void* y, int64_t ldy, int32_t M,
                      int32_t N, int32_t K, void* stream) {
  return linear_impl(x, ldx, w, ldw, y, ldy, M, N, K, stream);
}

hyb_status hyb_selftest_wait_timeout(void* stream) {
  hyb_status s = ensure_device();
  if (s != HYB_OK) return s;
  cudaError_t e = launch_selftest_wait(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return HYB_OK;
}

hyb_status hyb_kv_cache_init(const hyb_kv_cache* c, const int32_t* head0, void* stream) {
  hyb_status s = check_cache(c);
  if (s != HYB_OK) return s;
  if ((s = ensure_device()) != HYB_OK) return s;
  cudaStream_t st = as_stream(stream);
  const bool fp8 = c->kv_dtype == HYB_KV_FP8;
  uint64_t grows, gbatches;
  cache_geom(c, &grows, &gbatches);
  const size_t rows = (size_t)gbatches * kHkv * (size_t)grows;
  const size_t kv_bytes = rows * kD * (fp8 ? 1 : 2);
  cudaError_t e;
  if ((e = cudaMemsetAsync(c->k, 0, kv_bytes, st)) != cudaSuccess) return cuda_fail(e, "zero cache K");
  if ((e = cudaMemsetAsync(c->v, 0, kv_bytes, st)) != cudaSuccess) return cuda_fail(e, "zero cache V");
  if (fp8) {
    if ((e = cudaMemsetAsync(c->k_scale, 0, rows * sizeof(float), st)) != cudaSuccess) return cuda_fail(e, "k_scale");
    if ((e = cudaMemsetAsync(c->v_scale, 0, rows * sizeof(float), st)) != cudaSuccess) return cuda_fail(e, "v_scale");
  }
  if ((e = cudaMemsetAsync(c->len, 0, sizeof(int32_t) * c->batch, st)) != cudaSuccess) return cuda_fail(e, "len");
  if (c->type == HYB_SLIDING) {
    if ((e = launch_fill_i32(c->tag, (int64_t)c->batch * kWindow, -1, st)) != cudaSuccess)
      return cuda_fail(e, "tag fill");
    if (head0) {
      for (int b = 0; b < c->batch; ++b)
        if (head0[b] < 0 || head0[b] >= kWindow) return fail(HYB_ESHAPE, "head0[%d] = %d outside [0,512)", b, head0[b]);
      if ((e = cudaMemcpyAsync(c->head, head0, sizeof(int32_t) * c->batch, cudaMemcpyHostToDevice, st)) !=
          cudaSuccess)
        return cuda_fail(e, "head upload");
      // head0 is pageable host memory: make sure it has been read before returning
      if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "head upload sync");
    } else if ((e = cudaMemsetAsync(c->head, 0, sizeof(int32_t) * c->batch, st)) != cudaSuccess) {
      return cuda_fail(e, "head");
    }
  }
  return HYB_OK;
}

namespace {
hyb_status append_impl(const hyb_kv_cache* c, const void* k, const void* v, int64_t kv_row_stride, const int32_t* pos,
                       int32_t T, void* stream, bool k_rotated) {
  hyb_status s = check_cache(c);
  if (s != HYB_OK) return s;
  if (!k || !v) return fail(HYB_EINVAL, "k and v must be non-NULL");
  if (T <= 0) return fail(HYB_EINVAL, "T = %d must be positive", T);
  if (!aligned16(k) || !aligned16(v)) return fail(HYB_EALIGN, "k/v must be 16-byte aligned");
  if (kv_row_stride < kHkv * kD || kv_row_stride % 8 != 0)
    return fail(HYB_EALIGN, "kv_row_stride %lld must be >= 1024 and a multiple of 8 elements",
                (long long)kv_row_stride);
  if (pos && (reinterpret_cast<uintptr_t>(pos) & 3u)) return fail(HYB_EALIGN, "pos must be 4-byte aligned");
  if ((s = ensure_device()) != HYB_OK) return s;
  cudaStream_t st = as_stream(stream);
  const bool full = c->type == HYB_FULL;
  RopeStoreHost r;
  r.k = k;
  r.v = v;
  r.src_bstride = (int64_t)T * kv_row_stride;
  r.src_tstride = kv_row_stride;
  r.src_hstride = kD;
  r.pos = pos;
  r.dk = c->k;
  r.dv = c->v;
  r.dst_rows = c->capacity;
  r.mode = full ? 0 : 1;
  r.len = c->len;
  r.head = c->head;
  r.tag = c->tag;
  r.B = c->batch;
  r.T = T;
  r.t_first = full ? 0 : (T > kWindow ? T - kWindow : 0);
  r.src_rotated = k_rotated ? 1 : 0;
  r.fp8 = c->kv_dtype == HYB_KV_FP8 ? 1 : 0;
  r.dks = c->k_scale;
  r.dvs = c->v_scale;
  r.pm = page_map(c);
  // a few tokens per sequence (decode steps): one block per sequence writes its rows and
  // advances the cache state in the same launch; long appends spread over the SMs and
  // commit in a second launch
  r.commit = (T - r.t_first) <= 64 ? 1 : 0;
  r.capacity = c->capacity;
  cudaError_t e = launch_rope_store(full, r, st);
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  if (!r.commit && (e = launch_kv_commit(c->len, c->head, c->capacity, !full, c->batch, T, st)) != cudaSuccess)
    return cuda_fail(e, "commit launch");
  return HYB_OK;
}
}  // namespace

hyb_status hyb_kv_append(const hyb_kv_cache* c, const void* k, const void* v, int64_t kv_row_stride,
                         const int32_t* pos, int32_t T, void* stream) {
  return append_impl(c, k, v, kv_row_stride, pos, T, stream, false);
}

namespace {
// Attention scratch: rotated K (standalone) or the sliding context K / V (with
// a cache); rot_q adds the rotated copy of a sliding layer's queries, which
// the attention kernel then reads instead of rotating each query tile itself.
size_t attn_ws(int32_t layer_type, int32_t B, int32_t T, bool with_cache, bool rot_q) {
  if (B <= 0 || T <= 0) return 0;
  const size_t row = (size_t)kHkv * kD * 2;  // one token of K (or V), 4 heads (2 KB: keeps 256-byte alignment)
  size_t n;
  if (!with_cache) n = (size_t)B * (size_t)T * row;                      // rotated K
  else if (layer_type == HYB_FULL) n = 0;                                // reads the cache in place
  else n = 2 * (size_t)B * ctx_rows(T) * row;                            // context K and V
  if (rot_q && layer_type == HYB_SLIDING) n += (size_t)B * (size_t)T * kHq * kD * 2;
  return n;
}
}  // namespace

size_t hyb_attn_prefill_workspace_size(int32_t layer_type, int32_t B, int32_t T, int32_t with_cache) {
  return attn_ws(layer_type, B, T, with_cache != 0, true);
}

namespace {
// Scratch of a prefill with cache `c` (NULL: standalone): full layers read
// their cache in place, bf16 or FP8 (the attention kernel widens the codes
// itself).  rot_q: as attn_ws.
size_t prefill_ws(int32_t layer_type, int32_t B, int32_t T, const hyb_kv_cache* c, bool rot_q) {
  return attn_ws(layer_type, B, T, c != nullptr, rot_q);
}
}  // namespace

size_t hyb_attn_prefill_cache_workspace_size(const hyb_kv_cache* cache, int32_t T) {
  if (!cache || T <= 0 || check_cache(cache) != HYB_OK) return 0;
  return prefill_ws(cache->type, cache->batch, T, cache, true);
}

namespace {
// qk_rotated: q and k arrive rotated (the whole-layer path rotates them in the
// q_k_v_proj epilogue); the attention kernel and the K store then skip RoPE.
hyb_status prefill_impl(const void* q, const void* k, const void* v, const void* gate, const int32_t* pos,
                        int32_t layer_type, int32_t B, int32_t T, int64_t q_row_stride, int64_t kv_row_stride,
                        void* out, const hyb_kv_cache* cache, void* workspace, size_t workspace_bytes, void* stream,
                        bool qk_rotated) {
  if (!q || !k || !v || !out) return fail(HYB_EINVAL, "q, k, v and out must be non-NULL");
  if (layer_type != HYB_SLIDING && layer_type != HYB_FULL) return fail(HYB_EINVAL, "layer_type %d invalid", layer_type);
  if (B <= 0 || T <= 0) return fail(HYB_EINVAL, "B = %d and T = %d must be positive", B, T);
  if ((int64_t)T + kWindow > (int64_t)0x7fffffff) return fail(HYB_EOVERFLOW, "T = %d too large", T);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(HYB_EALIGN, "q, k, v and out must be 16-byte aligned");
  if (q_row_stride < kHq * kD || q_row_stride % 8 != 0)
    return fail(HYB_EALIGN, "q_row_stride %lld must be >= 4096 and a multiple of 8 elements", (long long)q_row_stride);
  if (kv_row_stride < kHkv * kD || kv_row_stride % 8 != 0)
    return fail(HYB_EALIGN, "kv_row_stride %lld must be >= 1024 and a multiple of 8 elements",
                (long long)kv_row_stride);
  if (gate && (reinterpret_cast<uintptr_t>(gate) & 1u)) return fail(HYB_EALIGN, "gate must be 2-byte aligned");
  if (pos && (reinterpret_cast<uintptr_t>(pos) & 3u)) return fail(HYB_EALIGN, "pos must be 4-byte aligned");
  hyb_status s;
  if (cache) {
    if ((s = check_cache(cache)) != HYB_OK) return s;
    if (cache->type != layer_type)
      return fail(HYB_ESHAPE, "cache type %d differs from layer_type %d", cache->type, layer_type);
    if (cache->batch != B) return fail(HYB_ESHAPE, "cache batch %d differs from B = %d", cache->batch, B);
    if (layer_type == HYB_FULL && (int64_t)T > cache->capacity)
      return fail(HYB_ESHAPE, "T = %d exceeds the cache capacity %lld", T, (long long)cache->capacity);
  }
  // sliding layers read a rotated copy of the queries (one pass over them): the
  // attention kernel rotates query tiles itself on full layers only (64 rotary
  // dims), where it costs little next to the long key loop of each tile
  const bool rot_q = layer_type == HYB_SLIDING && !qk_rotated;
  const size_t need = prefill_ws(layer_type, B, T, cache, rot_q);
  if (need > 0) {
    if (!workspace) return fail(HYB_EINVAL, "workspace of %zu bytes required", need);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(HYB_EALIGN, "workspace must be 256-byte aligned");
    if (workspace_bytes < need)
      return fail(HYB_EOVERFLOW, "workspace of %zu bytes given, %zu required", workspace_bytes, need);
  }
  if ((s = ensure_device()) != HYB_OK) return s;

  cudaStream_t st = as_stream(stream);
  const bool full = layer_type == HYB_FULL;
  const uint64_t row_bytes = kD * 2;
  PrefillHost ph;
  cudaError_t e;
  bool q_rot = qk_rotated;
  if (rot_q) {
    void* qr = reinterpret_cast<uint8_t*>(workspace) + prefill_ws(layer_type, B, T, cache, false);
    if ((e = launch_rope_q(false, q, q_row_stride, pos, cache ? cache->len : nullptr, B, T, qr, st)) != cudaSuccess)
      return cuda_fail(e, "query rotation launch");
    q = qr;
    q_row_stride = (int64_t)kHq * kD;
    q_rot = true;
  }
  if ((s = make_q_map(&ph.tm_q, q, T, B, (uint64_t)q_row_stride * 2, prefill_q_box_rows(), "Q")) != HYB_OK) return s;
  if ((s = make_out_map(&ph.tm_o, out, T, B)) != HYB_OK) return s;
  ph.q = q;
  ph.q_stride = q_row_stride;
  ph.gate = gate;
  ph.pos = pos;
  ph.out = out;
  ph.B = B;
  ph.T = T;
  // sliding layers: many short, equal work items -> persistent CTA pairs (one
  // per two SMs); full layers: long items of unequal length -> one item per
  // pair, handed out longest first by the hardware block scheduler.
  ph.n_pairs = full ? (1 << 29) : device_sms() / 2;
  ph.q_rotated = q_rot ? 1 : 0;

  RopeStoreHost r;  // new tokens, token-major input rows
  r.k = k;
  r.src_bstride = (int64_t)T * kv_row_stride;
  r.src_tstride = kv_row_stride;
  r.src_hstride = kD;
  r.pos = pos;
  r.B = B;
  r.T = T;
  r.src_rotated = qk_rotated ? 1 : 0;

  if (!cache) {
    // rotated K into the workspace [B][4][T][256]; V is read in place
    r.dk = workspace;
    r.dst_rows = T;
    r.mode = 2;
    if ((e = launch_rope_store(full, r, st)) != cudaSuccess) return cuda_fail(e, "rope K launch");
    const uint64_t hb = (uint64_t)T * row_bytes;
    if ((s = make_kv_map(&ph.tm_k, workspace, T, B, row_bytes, hb, hb * kHkv, prefill_k_box_rows(), "rotated K")) !=
        HYB_OK)
      return s;
    if ((s = make_kv_map(&ph.tm_v, v, T, B, (uint64_t)kv_row_stride * 2, row_bytes, (uint64_t)T * kv_row_stride * 2,
                         prefill_v_box_rows(), "V")) != HYB_OK)
      return s;
    if ((e = launch_prefill(full, ph, st)) != cudaSuccess) return cuda_fail(e, "prefill launch");
    return HYB_OK;
  }

  const bool fp8 = cache->kv_dtype == HYB_KV_FP8;
  if (full) {
    // append first (rows len .. len+T-1), attend over [0, len+T), then advance len.
    // FP8 caches: the chunk goes in quantized and, like a decode step, attends to
    // its own tokens as the cache stores them
    r.v = v;
    r.dk = cache->k;
    r.dv = cache->v;
    r.dst_rows = cache->capacity;
    r.mode = 0;
    r.len = cache->len;
    r.pm = page_map(cache);
    r.fp8 = fp8 ? 1 : 0;
    r.dks = cache->k_scale;
    r.dvs = cache->v_scale;
    if ((e = launch_rope_store(true, r, st)) != cudaSuccess) return cuda_fail(e, "append launch");
    if (fp8) {
      if ((s = cache_maps_fp8(cache, &ph.tm_k, &ph.tm_v, &ph.tm_ks, &ph.tm_vs)) != HYB_OK) return s;
      ph.fp8 = 1;
    } else if ((s = cache_maps(cache, &ph.tm_k, &ph.tm_v, prefill_k_box_rows(), prefill_v_box_rows())) != HYB_OK) {
      return s;
    }
    ph.pm = page_map(cache);
    ph.qbase = cache->len;
    ph.ctx_mode = 0;
    if ((e = launch_prefill(true, ph, st)) != cudaSuccess) return cuda_fail(e, "prefill launch");
    if ((e = launch_kv_commit(cache->len, cache->head, cache->capacity, false, B, T, st)) != cudaSuccess)
      return cuda_fail(e, "commit launch");
    return HYB_OK;
  }

  // sliding layer with a ring: context = ring's last 511 tokens + the chunk,
  // attend, then write the chunk's last 512 tokens into the ring.
  const size_t rows = ctx_rows(T);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  void* ck = ws;
  void* cv = ws + (size_t)B * rows * kHkv * row_bytes;
  if ((e = launch_ring_gather(cache->k, cache->v, fp8 ? cache->k_scale : nullptr, fp8 ? cache->v_scale : nullptr,
                              cache->len, cache->head, cache->tag, ck, cv, (int64_t)rows, B, st)) != cudaSuccess)
    return cuda_fail(e, "ring gather launch");
  r.v = v;
  r.dk = ck;
  r.dv = cv;
  r.dst_rows = (int64_t)rows;
  r.dst_row_offset = kWindow - 1;
  r.mode = 2;
  r.len = cache->len;  // default positions: len + t
  r.qdq = fp8 ? 1 : 0;  // FP8 ring: the chunk's rows as the ring will store them
  if ((e = launch_rope_store(false, r, st)) != cudaSuccess) return cuda_fail(e, "context rope launch");
  const uint64_t hb = (uint64_t)rows * row_bytes;
  if ((s = make_kv_map(&ph.tm_k, ck, rows, B, row_bytes, hb, hb * kHkv, prefill_k_box_rows(), "context K")) != HYB_OK)
    return s;
  if ((s = make_kv_map(&ph.tm_v, cv, rows, B, row_bytes, hb, hb * kHkv, prefill_v_box_rows(), "context V")) != HYB_OK)
    return s;
  ph.qbase = cache->len;
  ph.ctx_mode = 1;
  if ((e = launch_prefill(false, ph, st)) != cudaSuccess) return cuda_fail(e, "prefill launch");

  RopeStoreHost w;  // ring append: bf16 from the context rows (already rotated); FP8
                    // quantizes the rotated raw keys, as the context rows were made
  if (fp8) {
    w.k = k;
    w.v = v;
    w.src_bstride = (int64_t)T * kv_row_stride;
    w.src_tstride = kv_row_stride;
    w.src_hstride = kD;
    w.src_rotated = qk_rotated ? 1 : 0;
    w.pos = pos;
  } else {
    w.k = reinterpret_cast<const uint8_t*>(ck) + (size_t)(kWindow - 1) * row_bytes;
    w.v = reinterpret_cast<const uint8_t*>(cv) + (size_t)(kWindow - 1) * row_bytes;
    w.src_bstride = (int64_t)kHkv * (int64_t)rows * kD;
    w.src_tstride = kD;
    w.src_hstride = (int64_t)rows * kD;
    w.src_rotated = 1;
  }
  w.dk = cache->k;
  w.dv = cache->v;
  w.dst_rows = kWindow;
  w.mode = 1;
  w.len = cache->len;
  w.head = cache->head;
  w.tag = cache->tag;
  w.B = B;
  w.T = T;
  w.t_first = T > kWindow ? T - kWindow : 0;
  w.fp8 = fp8 ? 1 : 0;
  w.dks = cache->k_scale;
  w.dvs = cache->v_scale;
  if ((e = launch_rope_store(false, w, st)) != cudaSuccess) return cuda_fail(e, "ring append launch");
  if ((e = launch_kv_commit(cache->len, cache->head, cache->capacity, true, B, T, st)) != cudaSuccess)
    return cuda_fail(e, "commit launch");
  return HYB_OK;
}
}  // namespace

hyb_status hyb_attn_prefill(const void* q, const void* k, const void* v, const void* gate, const int32_t* pos,
                            int32_t layer_type, int32_t B, int32_t T, int64_t q_row_stride,
                            int64_t kv_row_stride, void* out, const hyb_kv_cache* cache, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return prefill_impl(q, k, v, gate, pos, layer_type, B, T, q_row_stride, kv_row_stride, out, cache, workspace,
                      workspace_bytes, stream, false);
}

size_t hyb_attn_decode_workspace_size(int32_t layer_type, int32_t B, int64_t max_len) {
  if (B <= 0) return 0;
  // room for either storage type's grid
  const int S = std::max(decode_num_splits(layer_type == HYB_FULL, B, max_len, false),
                         decode_num_splits(layer_type == HYB_FULL, B, max_len, true));
  const size_t rows = (size_t)B * kHq * (size_t)S;
  return rows * kD * sizeof(float) + ((rows * sizeof(float) + 255) & ~size_t(255));
}

namespace {
// out: gated bf16 output; or, with out_o / out_lse set (and out NULL), the
// merged fp32 output and base-2 log-sum-exp over this cache's keys.
hyb_status decode_impl(const void* q, int64_t q_stride, bool q_rotated, const void* gate, const int32_t* pos,
                       const hyb_kv_cache* c, int32_t layer_type, int64_t max_len, void* out, void* workspace,
                       size_t workspace_bytes, void* stream, float* out_o = nullptr, float* out_lse = nullptr) {
  hyb_status s = check_cache(c);
  if (s != HYB_OK) return s;
  if (!q || (!out && !(out_o && out_lse))) return fail(HYB_EINVAL, "q and the output buffers must be non-NULL");
  if (out_o && (!aligned16(out_o) || (reinterpret_cast<uintptr_t>(out_lse) & 3u)))
    return fail(HYB_EALIGN, "part_o must be 16-byte and part_lse 4-byte aligned");
  if (layer_type != c->type) return fail(HYB_ESHAPE, "layer_type %d differs from the cache type %d", layer_type, c->type);
  if (!aligned16(q) || !aligned16(out)) return fail(HYB_EALIGN, "q and out must be 16-byte aligned");
  if (gate && (reinterpret_cast<uintptr_t>(gate) & 1u)) return fail(HYB_EALIGN, "gate must be 2-byte aligned");
  if (pos && (reinterpret_cast<uintptr_t>(pos) & 3u)) return fail(HYB_EALIGN, "pos must be 4-byte aligned");
  if (max_len < 0 || max_len > c->capacity)
    return fail(HYB_ESHAPE, "max_len %lld outside [0, capacity %lld]", (long long)max_len, (long long)c->capacity);
  if (max_len == 0) max_len = c->capacity;
  const size_t need = hyb_attn_decode_workspace_size(layer_type, c->batch, max_len);
  if (!workspace) return fail(HYB_EINVAL, "workspace of %zu bytes required", need);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(HYB_EALIGN, "workspace must be 256-byte aligned");
  if (workspace_bytes < need) return fail(HYB_EOVERFLOW, "workspace of %zu bytes given, %zu required", workspace_bytes, need);
  if ((s = ensure_device()) != HYB_OK) return s;

  DecodeHost d;
  d.fp8 = c->kv_dtype == HYB_KV_FP8 ? 1 : 0;
  if ((s = d.fp8 ? cache_maps_fp8(c, &d.tm_k, &d.tm_v, &d.tm_ks, &d.tm_vs) : cache_maps(c, &d.tm_k, &d.tm_v, 64, 64)) !=
      HYB_OK)
    return s;
  d.q = q;
  d.q_stride = q_stride;
  d.q_rotated = q_rotated ? 1 : 0;
  d.gate = gate;
  d.pos = pos;
  d.len = c->len;
  d.tag = c->type == HYB_SLIDING ? c->tag : nullptr;
  d.out = out;
  d.B = c->batch;
  d.pm = page_map(c);
  d.n_splits = decode_num_splits(layer_type == HYB_FULL, c->batch, max_len, d.fp8 != 0);
  d.part_o = reinterpret_cast<float*>(workspace);
  d.part_lse = d.part_o + (size_t)c->batch * kHq * d.n_splits * kD;
  d.out_o = out_o;
  d.out_lse = out_lse;
  cudaError_t e = launch_decode(layer_type == HYB_FULL, d, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return HYB_OK;
}
}  // namespace

hyb_status hyb_attn_decode(const void* q, const void* gate, const int32_t* pos, const hyb_kv_cache* c,
                           int32_t layer_type, int64_t max_len, void* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return decode_impl(q, (int64_t)kHq * kD, false, gate, pos, c, layer_type, max_len, out, workspace, workspace_bytes,
                     stream);
}

hyb_status hyb_attn_decode_partial(const void* q, const int32_t* pos, const hyb_kv_cache* c, int32_t layer_type,
                                   int64_t max_len, float* part_o, float* part_lse, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (!part_o || !part_lse) return fail(HYB_EINVAL, "part_o and part_lse must be non-NULL");
  return decode_impl(q, (int64_t)kHq * kD, false, nullptr, pos, c, layer_type, max_len, nullptr, workspace,
                     workspace_bytes, stream, part_o, part_lse);
}

hyb_status hyb_attn_decode_merge(const float* part_o, const float* part_lse, int64_t o_stride, int64_t lse_stride,
                                 int32_t n_parts, int32_t B, const void* gate, void* out, void* stream) {
  if (!part_o || !part_lse || !out) return fail(HYB_EINVAL, "part_o, part_lse and out must be non-NULL");
  if (n_parts <= 0 || B <= 0) return fail(HYB_EINVAL, "n_parts = %d and B = %d must be positive", n_parts, B);
  const int64_t rows = (int64_t)B * kHq;
  if (o_stride == 0) o_stride = rows * kD;
  if (lse_stride == 0) lse_stride = rows;
  if (o_stride < rows * kD || lse_stride < rows)
    return fail(HYB_ESHAPE, "part strides (%lld, %lld) below one part (%lld, %lld floats)", (long long)o_stride,
                (long long)lse_stride, (long long)(rows * kD), (long long)rows);
  if ((int64_t)n_parts * o_stride > (int64_t)0x7fffffff || (int64_t)n_parts * lse_stride > (int64_t)0x7fffffff)
    return fail(HYB_EOVERFLOW, "n_parts x part stride exceeds 2^31 elements");
  if (!aligned16(part_o) || !aligned16(out) || (reinterpret_cast<uintptr_t>(part_lse) & 3u))
    return fail(HYB_EALIGN, "part_o and out must be 16-byte aligned, part_lse 4-byte aligned");
  if (gate && (reinterpret_cast<uintptr_t>(gate) & 1u)) return fail(HYB_EALIGN, "gate must be 2-byte aligned");
  hyb_status s;
  if ((s = ensure_device()) != HYB_OK) return s;
  cudaError_t e =
      launch_decode_merge(part_o, part_lse, o_stride, lse_stride, n_parts, (int)rows, gate, out, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return HYB_OK;
}

// Same computation as hyb_attn_decode, with the split partials kept in the
// library's fixed device scratch (decode.cu) instead of a caller workspace,
// so that nothing is allocated by anyone on this call path.
hyb_status hyb_attn_decode_noalloc(const void* q, const void* gate, const int32_t* pos, const hyb_kv_cache* c,
                                   int32_t layer_type, int64_t max_len, void* out, void* stream) {
  hyb_status s = check_cache(c);
  if (s != HYB_OK) return s;
  if (max_len < 0 || max_len > c->capacity)
    return fail(HYB_ESHAPE, "max_len %lld outside [0, capacity %lld]", (long long)max_len, (long long)c->capacity);
  const int64_t ml = max_len == 0 ? c->capacity : max_len;
  const size_t need = hyb_attn_decode_workspace_size(layer_type, c->batch, ml);
  if (need > kNoAllocScratchBytes)
    return fail(HYB_EOVERFLOW,
                "batch %d x 16 heads x %d splits (the larger of the bf16 and FP8 split grids) needs %zu bytes of "
                "split scratch, more than the %zu-byte fixed scratch of hyb_attn_decode_noalloc; use "
                "hyb_attn_decode with a workspace",
                c->batch,
                std::max(decode_num_splits(layer_type == HYB_FULL, c->batch, ml, false),
                         decode_num_splits(layer_type == HYB_FULL, c->batch, ml, true)),
                need, kNoAllocScratchBytes);
  if ((s = ensure_device()) != HYB_OK) return s;
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  cudaError_t e = decode_noalloc_scratch(&scratch, &scratch_bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
  // the same checks and launches as hyb_attn_decode, with the fixed scratch as its workspace
  return decode_impl(q, (int64_t)kHq * kD, false, gate, pos, c, layer_type, max_len, out, scratch, scratch_bytes,
                     stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Whole attention layer: q_k_v_proj + gate projection, the attention core,
// o_proj ("百万 Token 塞进 4B ..." §"省显存的第二板斧").
// ---------------------------------------------------------------------------
namespace {
constexpr int64_t kHidden = 2560;                        // residual width (hidden_size)
constexpr int64_t kQkv = (int64_t)(kHq + 2 * kHkv) * kD;   // 6144: fused q | k | v row
size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }
}  // namespace

// fused q|k|v rows, gate scores, attention output, RoPE table (up to 128
// (cos, sin) pairs per row), then the attention's own scratch
size_t layer_head_bytes(size_t n) {
  return round256(n * kQkv * 2) + round256(n * kHq * 2) + round256(n * kHq * kD * 2) + round256(n * 128 * 8);
}

// (the layer's queries arrive rotated from the q_k_v_proj epilogue: no query copy)
size_t hyb_attn_layer_prefill_workspace_size(int32_t layer_type, int32_t B, int32_t T, int32_t with_cache) {
  if (B <= 0 || T <= 0) return 0;
  return layer_head_bytes((size_t)B * (size_t)T) + attn_ws(layer_type, B, T, with_cache != 0, false);
}

size_t hyb_attn_layer_prefill_cache_workspace_size(const hyb_kv_cache* cache, int32_t T) {
  if (!cache || T <= 0 || check_cache(cache) != HYB_OK) return 0;
  return layer_head_bytes((size_t)cache->batch * (size_t)T) + prefill_ws(cache->type, cache->batch, T, cache, false);
}

hyb_status hyb_attn_layer_prefill(const void* hidden, const void* w_qkv, const void* w_gate, const void* w_o,
                                  const int32_t* pos, int32_t layer_type, int32_t B, int32_t T, void* out,
                                  const hyb_kv_cache* cache, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (!hidden || !w_qkv || !w_o || !out) return fail(HYB_EINVAL, "hidden, w_qkv, w_o and out must be non-NULL");
  if (layer_type != HYB_SLIDING && layer_type != HYB_FULL) return fail(HYB_EINVAL, "layer_type %d invalid", layer_type);
  if (B <= 0 || T <= 0) return fail(HYB_EINVAL, "B = %d and T = %d must be positive", B, T);
  if ((int64_t)B * T > 0x7fffffffLL) return fail(HYB_ESHAPE, "B * T = %lld tokens is too many", (long long)B * T);
  const size_t need = cache ? hyb_attn_layer_prefill_cache_workspace_size(cache, T)
                            : hyb_attn_layer_prefill_workspace_size(layer_type, B, T, 0);
  if (cache && need == 0) {
    hyb_status cs = check_cache(cache);
    return cs != HYB_OK ? cs : fail(HYB_EINVAL, "T = %d must be positive", T);
  }
  if (workspace_bytes < need) return fail(HYB_EOVERFLOW, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(HYB_EALIGN, "workspace must be non-NULL and 256-byte aligned");
  const int32_t M = B * T;
  const size_t n = (size_t)M;
  uint8_t* p = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* qkv = reinterpret_cast<__nv_bfloat16*>(p);
  p += round256(n * kQkv * 2);
  __nv_bfloat16* gate = reinterpret_cast<__nv_bfloat16*>(p);
  p += round256(n * kHq * 2);
  __nv_bfloat16* attn = reinterpret_cast<__nv_bfloat16*>(p);
  p += round256(n * kHq * kD * 2);
  void* rot = p;
  p += round256(n * 128 * 8);
  const size_t attn_ws = prefill_ws(layer_type, B, T, cache, false);
  // q_k_v_proj with RoPE of the q and k heads in the epilogue (positions as
  // hyb_attn_prefill: pos, else the cache length + t, else t); the gate
  // projection's 16 rows as one more column tile of the same launch
  const int32_t* len = cache ? cache->len : nullptr;
  hyb_status s = linear_impl(hidden, kHidden, w_qkv, kHidden, qkv, kQkv, M, (int32_t)kQkv, (int32_t)kHidden, stream,
                             layer_type == HYB_FULL ? 2 : 1, (kHq + kHkv) * kD, T, pos, len, rot, w_gate, kHidden,
                             w_gate ? gate : nullptr, kHq, w_gate ? kHq : 0);
  if (s != HYB_OK) return s;
  s = prefill_impl(qkv, qkv + (int64_t)kHq * kD, qkv + (int64_t)(kHq + kHkv) * kD, w_gate ? gate : nullptr, pos,
                   layer_type, B, T, kQkv, kQkv, attn, cache, attn_ws ? p : nullptr, attn_ws, stream, true);
  if (s != HYB_OK) return s;
  return hyb_linear(attn, (int64_t)kHq * kD, w_o, (int64_t)kHq * kD, out, kHidden, M, (int32_t)kHidden,
                    (int32_t)(kHq * kD), stream);
}

size_t hyb_attn_layer_decode_workspace_size(int32_t layer_type, int32_t B, int64_t max_len) {
  if (B <= 0) return 0;
  return layer_head_bytes((size_t)B) + hyb_attn_decode_workspace_size(layer_type, B, max_len);
}

hyb_status hyb_attn_layer_decode(const void* hidden, const void* w_qkv, const void* w_gate, const void* w_o,
                                 const hyb_kv_cache* cache, int32_t layer_type, int64_t max_len, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  hyb_status s = check_cache(cache);
  if (s != HYB_OK) return s;
  if (!hidden || !w_qkv || !w_o || !out) return fail(HYB_EINVAL, "hidden, w_qkv, w_o and out must be non-NULL");
  if (layer_type != cache->type)
    return fail(HYB_ESHAPE, "layer_type %d differs from the cache type %d", layer_type, cache->type);
  if (max_len < 0 || max_len > cache->capacity)
    return fail(HYB_ESHAPE, "max_len %lld outside [0, capacity %lld]", (long long)max_len, (long long)cache->capacity);
  if (max_len == 0) max_len = cache->capacity;
  const int32_t B = cache->batch;
  const size_t need = hyb_attn_layer_decode_workspace_size(layer_type, B, max_len);
  if (workspace_bytes < need) return fail(HYB_EOVERFLOW, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(HYB_EALIGN, "workspace must be non-NULL and 256-byte aligned");
  const size_t n = (size_t)B;
  uint8_t* p = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* qkv = reinterpret_cast<__nv_bfloat16*>(p);
  p += round256(n * kQkv * 2);
  __nv_bfloat16* gate = reinterpret_cast<__nv_bfloat16*>(p);
  p += round256(n * kHq * 2);
  __nv_bfloat16* attn = reinterpret_cast<__nv_bfloat16*>(p);
  p += round256(n * kHq * kD * 2);
  void* rot = p;
  p += round256(n * 128 * 8);
  // q_k_v_proj and the gate projection in one launch.  Up to 16 sequences the
  // few-row kernel streams the weights and the append and the decode rotate
  // k and q at the new token's position (the cache length); beyond, the
  // tiled GEMM rotates them in its epilogue.
  const bool few = smallm_supported(B, (int)(kQkv + (w_gate ? kHq : 0)), (int)kHidden, (int)kQkv);
  if ((s = linear_impl(hidden, kHidden, w_qkv, kHidden, qkv, kQkv, B, (int32_t)kQkv, (int32_t)kHidden, stream,
                       few ? 0 : (layer_type == HYB_FULL ? 2 : 1), few ? 0 : (kHq + kHkv) * kD, 1, nullptr,
                       cache->len, rot, w_gate, kHidden, w_gate ? gate : nullptr, kHq, w_gate ? kHq : 0)) != HYB_OK)
    return s;
  if ((s = append_impl(cache, qkv + (int64_t)kHq * kD, qkv + (int64_t)(kHq + kHkv) * kD, kQkv, nullptr, 1, stream,
                       !few)) != HYB_OK)
    return s;
  if ((s = decode_impl(qkv, kQkv, !few, w_gate ? gate : nullptr, nullptr, cache, layer_type, max_len, attn, p,
                       hyb_attn_decode_workspace_size(layer_type, B, max_len), stream)) != HYB_OK)
    return s;
  // o_proj right after the library's own attention, which does not write w_o
  return linear_impl(attn, (int64_t)kHq * kD, w_o, (int64_t)kHq * kD, out, kHidden, B, (int32_t)kHidden,
                     (int32_t)(kHq * kD), stream, 0, 0, 0, nullptr, nullptr, nullptr, nullptr, 0, nullptr, 0, 0,
                     true);
}
