// Host-side interface between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hyb {

void count_launch();

// Launches `kernel` with programmatic stream serialization (the kernel calls
// pdl_wait() before reading what earlier kernels of the stream wrote) and,
// with cluster_x > 0, as clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Profiling hook (hyb_profile_events): records a caller-owned event pair
// around the next attention-kernel launches.
void profile_before(cudaStream_t st);
void profile_after(cudaStream_t st);

// Paged full-layer caches: token i of sequence b lives in pool page
// table[b * max_pages + i / page], row i % page.  page == 0: contiguous
// cache, token i of sequence b at row i of batch entry b.
struct PageMap {
  const int32_t* table = nullptr;   // device [B][max_pages]
  int page = 0;
  int max_pages = 0;
  int n_pages = 0;
};

// ---- KV side (rope_kv.cu) --------------------------------------------------
struct RopeStoreHost {
  const void* k = nullptr;
  const void* v = nullptr;
  int64_t src_bstride = 0, src_tstride = 0, src_hstride = 0;  // elements
  int src_rotated = 0;
  const int32_t* pos = nullptr;
  void* dk = nullptr;
  void* dv = nullptr;
  int64_t dst_rows = 0;
  int dst_row_offset = 0;
  int mode = 0;  // 0 linear cache, 1 ring, 2 plain rows
  int32_t* len = nullptr;
  int32_t* head = nullptr;
  int32_t* tag = nullptr;
  int B = 0, T = 0, t_first = 0;
  int fp8 = 0;                 // 1: destination is an FP8 cache (codes + per-row scales)
  float* dks = nullptr;
  float* dvs = nullptr;
  PageMap pm;                  // linear mode: paged destination cache
  int commit = 0;              // 1: advance len / head in the same launch (one block per sequence)
  int qdq = 0;                 // rows mode: write each bf16 row as its e4m3 quantization dequantized
  int64_t capacity = 0;        // commit, linear mode: cache capacity
};
cudaError_t launch_rope_store(bool full, const RopeStoreHost& h, cudaStream_t st);
// rks / rvs: FP8 rings' scales (rk / rv hold e4m3 codes), or null for bf16 rings
cudaError_t launch_ring_gather(const void* rk, const void* rv, const float* rks, const float* rvs,
                               const int32_t* len, const int32_t* head, const int32_t* tag, void* ck, void* cv,
                               int64_t ctx_rows, int B, cudaStream_t st);
cudaError_t launch_kv_commit(int32_t* len, int32_t* head, int64_t capacity, bool ring, int B, int T,
                             cudaStream_t st);
cudaError_t launch_selftest_wait(cudaStream_t st);
// Rotated copy [B][T][16][256] of query rows (16 x 256 at src + (b T + t) src_tstride)
// at position pos[b][t], else (len ? len[b] : 0) + t
cudaError_t launch_rope_q(bool full, const void* src, int64_t src_tstride, const int32_t* pos, const int32_t* len,
                          int B, int T, void* dst, cudaStream_t st);
// (cos, sin) float2 [M][R / 2] of row m's position x frequency k (R = 64 full,
// 256 sliding): row m is token m % T of sequence m / T at position pos[m], else
// (len ? len[m / T] : 0) + m % T
cudaError_t launch_rope_table(bool full, const int32_t* pos, const int32_t* len, int T, int M, void* tab,
                              cudaStream_t st);
cudaError_t launch_fill_i32(int32_t* p, int64_t n, int32_t v, cudaStream_t st);

// ---- linear projections (gemm.cu) -------------------------------------------
struct GemmHost {
  CUtensorMap tm_x, tm_w;      // 2-D maps {K, rows}, 64 x 128 boxes, 128B swizzle
  void* y = nullptr;           // bf16 [M][ldy]
  int64_t ldy = 0;
  // second output group: columns [n_main, N) from tm_w2's rows 0 .. into y2
  // (n_main a multiple of 256); n_main = 0: none
  CUtensorMap tm_w2;
  void* y2 = nullptr;
  int64_t ldy2 = 0;
  int n_main = 0;
  int M = 0, N = 0, K = 0;
  int n_pairs = 74;            // persistent CTA pairs (SMs / 2)
  // RoPE epilogue: 0 none, 1 sliding-layer, 2 full-layer rotation of the
  // 256-wide column tiles below rope_cols, with (cos, sin) from `rot`
  // (launch_rope_table's [M][R / 2] float2 table)
  int rope = 0, rope_cols = 0, T = 0;
  const void* rot = nullptr;
};
cudaError_t launch_gemm(const GemmHost& h, cudaStream_t st);

// ---- few-row projections (smallm.cu) ------------------------------------------
// y[M][ldy] = x[M][ldx] w[N][ldw]^T for M <= 16, K a multiple of 512 up to
// 4096; features n_main .. N - 1 (n_main > 0) from w2's rows into y2.
struct SmallMHost {
  const void* x = nullptr;
  int64_t ldx = 0;
  const void* w = nullptr;
  int64_t ldw = 0;
  const void* w2 = nullptr;
  int64_t ldw2 = 0;
  void* y = nullptr;
  int64_t ldy = 0;
  void* y2 = nullptr;
  int64_t ldy2 = 0;
  int n_main = 0, M = 0, N = 0, K = 0;
  bool early_w = false;   // the kernel launched just before on the stream does not write w / w2
};
bool smallm_supported(int M, int N, int K, int n_main);
cudaError_t launch_smallm(const SmallMHost& h, cudaStream_t st);
cudaError_t gemm_set_smem_attr();
int gemm_box_rows();   // rows of X or W per TMA box
int gemm_box_k();      // K elements per TMA box

// ---- prefill attention (prefill.cu) -----------------------------------------
struct PrefillHost {
  CUtensorMap tm_k, tm_v;      // 4-D maps {256, rows, 4, B}, 64-dim boxes, 128B swizzle
                               // (fp8: uint8 maps of the cache's codes, 128-code boxes)
  CUtensorMap tm_ks, tm_vs;    // fp8: 3-D maps over the row scales {rows, 4, B}, 64-row boxes
  int fp8 = 0;                 // 1: a full layer's keys and values come from an FP8 cache
  CUtensorMap tm_q, tm_o;      // 4-D maps {256, 16, T, B} over q and out, 64-dim x 128-row boxes
  const void* q = nullptr;     // raw queries
  int64_t q_stride = 0;        // elements between tokens
  const void* gate = nullptr;  // [B][T][16] or null
  const int32_t* pos = nullptr;
  void* out = nullptr;         // [B][T][16][256]
  const int32_t* qbase = nullptr;  // [B] sequence index of token 0, or null (0)
  int ctx_mode = 0;            // 1: key row j holds sequence index qbase - 511 + j
  int q_rotated = 0;           // 1: q is already rotated (the kernel skips RoPE)
  int B = 0, T = 0;
  int n_pairs = 74;            // persistent CTA pairs (SMs / 2)
  PageMap pm;                  // K/V maps over a paged cache's pool
};
cudaError_t launch_prefill(bool full, const PrefillHost& h, cudaStream_t st);
int prefill_k_box_rows();   // rows (keys) per TMA box of the K map
int prefill_v_box_rows();   // rows (keys) per TMA box of the V map
int prefill_q_box_rows();   // rows (tokens) per TMA box of the Q and O maps
size_t prefill_smem_bytes();

// ---- decode (decode.cu) -------------------------------------------------------
struct DecodeHost {
  CUtensorMap tm_k, tm_v;      // 4-D maps over the cache {256, capacity, 4, B}
  CUtensorMap tm_ks, tm_vs;    // FP8 caches: 3-D maps over the scales {capacity, 4, B}
  int fp8 = 0;                 // 1: k / v hold e4m3 codes (tm_k / tm_v are uint8 maps, 128-dim boxes)
  const void* q = nullptr;     // [B][16][256] rows q_stride elements apart
  int64_t q_stride = 16 * 256;
  int q_rotated = 0;           // 1: q is already rotated (the kernel skips RoPE)
  const void* gate = nullptr;  // [B][16] or null
  const int32_t* pos = nullptr;
  const int32_t* len = nullptr;
  const int32_t* tag = nullptr;  // ring tags (sliding) or null
  void* out = nullptr;
  float* part_o = nullptr;     // [B][16][S][256]
  float* part_lse = nullptr;   // [B][16][S]
  int B = 0, n_splits = 1;
  PageMap pm;                  // maps over a paged cache's pool {256, page, 4, n_pages}
  float* out_o = nullptr;      // set: write the merged fp32 output [B][16][256] and base-2
  float* out_lse = nullptr;    //   log-sum-exp [B][16] instead of the gated bf16 out
};
cudaError_t launch_decode(bool full, const DecodeHost& h, cudaStream_t st);
// Merges n_parts partials (part p: output [rows][256] at part_o + p * o_stride,
// lse [rows] at part_lse + p * lse_stride, in floats) into gated bf16 out [rows][256].
cudaError_t launch_decode_merge(const float* part_o, const float* part_lse, int64_t o_stride, int64_t lse_stride,
                                int n_parts, int rows, const void* gate, void* out, cudaStream_t st);
int decode_num_splits(bool full, int B, int64_t max_len, bool fp8);
// Address and size of the library's fixed decode scratch on the current
// device (looked up on first use per device).
cudaError_t decode_noalloc_scratch(void** ptr, size_t* bytes);
size_t decode_smem_bytes(bool fp8);

}  // namespace hyb
