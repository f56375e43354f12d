/*
 * hyb_attn.h -- C ABI of the B200 (sm_100a) hybrid GQA attention core.
 *
 * The operation is the per-layer attention of the Spark-X2.5 / X2.6-4B
 * decoder as the following pages describe it (titles abbreviated):
 *
 *  [TEARDOWN] "百万 Token 塞进 4B 是怎么做到的？星火 X2.5 的长上下文架构拆解与显存博弈"
 *  [LAPTOP]   "不用高显存卡也能跑！4B参数挑战百万上下文，笔记本就能玩"
 *  [X26BASE]  the Spark-X2.6-4B-Base config walkthrough (lqnn.cn)
 *
 *  - 16 query heads share 4 KV heads (query head h reads KV head h / 4),
 *    head_dim 256: [TEARDOWN] §"省显存的第二板斧：GQA、融合投影与输出门控",
 *    [LAPTOP] §"分组查询注意力".
 *  - Layer types: sliding layers attend to the last 512 tokens (the query
 *    and the 511 before it) and rotate all 256 dims with RoPE theta 1e4;
 *    full layers attend causally to the whole prefix and rotate only the
 *    first 64 dims with theta 5e6: [TEARDOWN] §"混合注意力：每 4 层只给一层
 *    全量视野" and §"滑动窗口的补救：分层 RoPE 与局部/全局分工";
 *    [X26BASE] §"全局注意力 + 5M 基频 RoPE".  Layer i is full iff i % 4 == 3.
 *  - RoPE is rotate-half: for k < R/2, pair (k, k + R/2) rotates by
 *    pos * theta^(-2k/R); dims >= R are unchanged.
 *  - Softmax scale 1/16; the normalised output of head h is multiplied by
 *    sigmoid(gate[h]) ([TEARDOWN] §"省显存的第二板斧", the head-wise output gate).
 *  - KV cache: a full layer keeps every token (4096 bytes per token per
 *    layer, [TEARDOWN] §"先算一笔账"); a sliding layer keeps the most recent
 *    512 tokens in a ring ([LAPTOP] §"百万上下文的真正瓶颈").
 *
 * Conventions for every call
 *  - All tensors are bfloat16 unless stated; all pointers are DEVICE
 *    pointers owned by the caller, except where a parameter says "host".
 *    The library never allocates or frees device memory.
 *  - Every pointer and every row stride (in bytes) must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Host-side argument checks run
 *    before any launch; on a non-OK status nothing was enqueued and
 *    hyb_last_error() describes the problem.
 *  - Conditions only the device can see (a full-layer cache running out of
 *    capacity, a pipeline wait that exceeded its time limit) set sticky
 *    bits in a per-device error word read by hyb_device_error(); kernels
 *    never trap.
 *  - Token positions: a token's sequence index is its position in its
 *    sequence (0-based, counting cached tokens).  Masks always use sequence
 *    indices; RoPE uses `pos` when given, else the sequence index.
 */
#ifndef HYB_ATTN_H
#define HYB_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HYB_N_Q_HEADS 16
#define HYB_N_KV_HEADS 4
#define HYB_HEAD_DIM 256
#define HYB_WINDOW 512

typedef enum { HYB_SLIDING = 0, HYB_FULL = 1 } hyb_layer_type;

typedef enum {
  HYB_OK = 0,
  HYB_EINVAL = -1,       /* null pointer, bad enum, non-positive size            */
  HYB_ESHAPE = -2,       /* sizes inconsistent with each other or the cache      */
  HYB_EALIGN = -3,       /* pointer or row stride not 16-byte aligned            */
  HYB_EOVERFLOW = -4,    /* workspace too small / size arithmetic overflow       */
  HYB_ECUDA = -5,        /* a CUDA runtime or driver call failed                 */
  HYB_EUNSUPPORTED = -6  /* device is not sm_100 / driver entry point missing    */
} hyb_status;

/* Bits of the per-device error word (hyb_device_error). */
#define HYB_DEV_ERR_CAPACITY 1  /* append past a full-layer cache's capacity: skipped */
#define HYB_DEV_ERR_TIMEOUT 2   /* a pipeline wait exceeded its limit: output invalid */
#define HYB_DEV_ERR_PAGE 4      /* a block-table entry outside [0, n_pages): the write
                                   is skipped, the read gives zero keys and values */
#define HYB_DEV_ERR_BOUNDS 8    /* debug build only (hyb_build_flags): an index outside
                                   its buffer; the access is skipped */

/*
 * KV cache of one layer for `batch` sequences.  All buffers are caller-owned
 * device memory; the struct itself may live on the host stack.
 *   k, v : bf16 [batch][4][capacity][256] (head-major: one KV head's keys of
 *          one sequence are contiguous).  Keys are stored already rotated.
 *   len  : int32 [batch], tokens of each sequence appended so far.
 *   head : SLIDING only, int32 [batch], next ring slot to write.
 *   tag  : SLIDING only, int32 [batch][512], sequence index held by each
 *          slot, -1 = empty.
 * FULL caches keep token i at slot i (capacity >= longest sequence);
 * SLIDING caches have capacity 512 and write token i at slot
 * (head0 + i) % 512, head0 being the head when len was 0.
 */
typedef struct hyb_kv_cache {
  int32_t type;      /* hyb_layer_type */
  int32_t batch;
  int64_t capacity;
  void* k;
  void* v;
  int32_t* len;
  int32_t* head;
  int32_t* tag;
  int32_t kv_dtype;  /* HYB_KV_BF16 (0) or HYB_KV_FP8 (1) */
  float* k_scale;    /* HYB_KV_FP8 only: fp32 [batch][4][capacity], one scale per */
  float* v_scale;    /*   (token, KV head) row; NULL for HYB_KV_BF16 */
  /* Paged storage (FULL caches only; page_size 0 = the contiguous layout above). */
  int32_t page_size;      /* tokens per page, a positive multiple of 64 */
  int32_t max_pages;      /* block_table entries per sequence; capacity == max_pages * page_size */
  int64_t n_pages;        /* pages in the pool that k / v (and the scales) hold */
  int32_t* block_table;   /* device int32 [batch][max_pages] */
} hyb_kv_cache;

/*
 * Paged KV cache (FULL layers): a serving runtime holds one pool of pages for
 * many sequences of mixed length and hands pages out as sequences grow
 * ("不用高显存卡也能跑！..." §3.1 names paged KV caches among the serving
 * engines' means).  With page_size P > 0:
 *   k, v       : pool [n_pages][4][P][256] (bf16, or e4m3 codes),
 *   k_scale, v_scale (FP8): [n_pages][4][P],
 *   block_table: token i of sequence b lives in pool page
 *                block_table[b * max_pages + i / P], row i % P.
 * The library reads only the entries that cover [0, len) (and, for an
 * append of T tokens, [len, len + T)); the others may hold anything, e.g.
 * -1 for pages not handed out yet.  An entry it reads that lies outside
 * [0, n_pages) raises HYB_DEV_ERR_PAGE: appends skip that row, attention
 * reads zero keys and values there.  Pages may be shared by sequences for
 * reading (a common prefix); two sequences that append into one page race.
 * hyb_kv_cache_init zero-fills the whole pool.  P is a multiple of 64 so
 * that every 64-key tile the kernels load lies within one page.
 */

/*
 * KV storage types.  HYB_KV_BF16: k / v hold bf16 [batch][4][capacity][256].
 * HYB_KV_FP8: k / v hold FP8 e4m3 codes (1 byte) [batch][4][capacity][256],
 * and each 256-dim row (one token, one KV head) has an fp32 scale:
 *   scale = amax / 448 (amax = largest |value| of the row, the K row after
 *   RoPE and bf16 rounding as the bf16 cache would hold it),
 *   code  = e4m3(round to nearest even, saturating at +-448)(value * (448 / amax)),
 *   stored value = code * scale (a zero row has scale 0 and zero codes).
 * Halves the cache bytes that decode streams (the pages' deployments keep
 * the KV cache in 8 bits: "不用高显存卡也能跑！..." q8_0 KV in llama.cpp).
 * FP8 caches need capacity % 4 == 0.  Every attention over an FP8 cache
 * reads the keys and values as the cache stores them (code value x scale):
 * decode, the current token included, and prefill, whose chunk is appended
 * quantized and attends to its own tokens in that form as well as to the
 * history.  A full layer's prefill reads the codes in place (no workspace
 * beyond the bf16 cache's); a sliding layer builds its usual bf16 context
 * from the ring's rows and the chunk's rows as the ring will store them.
 */
#define HYB_KV_BF16 0
#define HYB_KV_FP8 1

/*
 * Resets a cache: len = 0, head = head0[b] (host array, NULL = all 0),
 * tag = -1, and zero-fills k and v so that no slot ever holds a non-finite
 * bit pattern (masked keys are multiplied by a zero weight, and 0 * NaN
 * would poison the output).  Must run once on fresh memory.
 * Errors: HYB_EINVAL (null buffer, bad type), HYB_ESHAPE (SLIDING with
 * capacity != 512, head0 outside [0,512)), HYB_EALIGN, HYB_ECUDA.
 */
hyb_status hyb_kv_cache_init(const hyb_kv_cache* cache, const int32_t* head0, void* stream);

/*
 * Appends T tokens to every sequence of the cache (§ KV cache above).
 *   k, v : rows of 4 x 256 bf16 per token, token t of sequence b at
 *          element offset (b*T + t) * kv_row_stride.  kv_row_stride = 1024
 *          for contiguous [B,T,4,256]; 6144 for k/v views into a fused
 *          q_k_v_proj row ([TEARDOWN] §"省显存的第二板斧": q = [:4096],
 *          k = [4096:5120], v = [5120:6144]).
 *   pos  : device int32 [batch][T] RoPE positions, or NULL (sequence index).
 * K is rotated with the cache's layer type before it is stored; V is copied
 * bit for bit.  A full-layer sequence whose len + T exceeds capacity is left
 * unchanged and HYB_DEV_ERR_CAPACITY is raised.  For a sliding layer only
 * the last min(T, 512) tokens are written.
 */
hyb_status hyb_kv_append(const hyb_kv_cache* cache, const void* k, const void* v,
                         int64_t kv_row_stride, const int32_t* pos, int32_t T, void* stream);

/*
 * Prefill attention of T new tokens per sequence, B sequences.
 *   q    : 16 x 256 per token at element offset (b*T + t) * q_row_stride
 *          (4096 contiguous, 6144 for a fused q_k_v_proj row).
 *   k, v : as in hyb_kv_append (kv_row_stride).
 *   gate : bf16 [B][T][16] gate scores, or NULL for no gate.
 *   pos  : device int32 [B][T] RoPE positions, or NULL (sequence index).
 *   out  : bf16 [B][T][16][256].
 *   cache: NULL -> the T tokens are whole sequences (token t has sequence
 *          index t).  Non-NULL -> they continue the cached sequences (token
 *          t has index len[b] + t), attend over the cached keys as well, and
 *          are appended to the cache.  cache->type must equal layer_type and
 *          cache->batch must equal B.
 *   workspace: device scratch of at least
 *          hyb_attn_prefill_workspace_size(layer_type, B, T, cache != NULL)
 *          bytes (256-byte aligned); it holds rotated keys (or a sliding
 *          layer's context keys and values) and, for sliding layers, a
 *          rotated copy of the queries between launches.
 * Errors: HYB_EINVAL, HYB_ESHAPE, HYB_EALIGN, HYB_EOVERFLOW (workspace too
 * small), HYB_EUNSUPPORTED (not an sm_100 device), HYB_ECUDA.
 */
size_t hyb_attn_prefill_workspace_size(int32_t layer_type, int32_t B, int32_t T, int32_t with_cache);
/* Workspace of hyb_attn_prefill with this cache and chunk length: the value
 * above, for bf16 and FP8 caches alike (it does not grow with the cache's
 * capacity).  0 for an invalid cache or T <= 0. */
size_t hyb_attn_prefill_cache_workspace_size(const hyb_kv_cache* cache, int32_t T);
hyb_status hyb_attn_prefill(const void* q, const void* k, const void* v, const void* gate,
                            const int32_t* pos, int32_t layer_type, int32_t B, int32_t T,
                            int64_t q_row_stride, int64_t kv_row_stride, void* out,
                            const hyb_kv_cache* cache, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * One decode step: one query token per sequence against its cache, which
 * must already hold the token itself (call hyb_kv_append first).
 * B is cache->batch: the kernels read q, gate and pos and write out for
 * every sequence of the cache, so each of them must hold B rows (the call
 * has no separate batch argument to check them against).
 *   q    : bf16 [B][16][256] contiguous query (not rotated).
 *   gate : bf16 [B][16] or NULL.
 *   pos  : device int32 [B] RoPE position of the query, or NULL (len - 1).
 *   max_len : host-side upper bound of len over the batch (<= capacity), or
 *          0 for capacity; it sizes the split-KV grid and the workspace.
 *   out  : bf16 [B][16][256].
 *   workspace: at least hyb_attn_decode_workspace_size(layer_type, B,
 *          max_len) bytes of device scratch for the per-split partial
 *          outputs and log-sum-exps.
 * Errors: as hyb_attn_prefill.
 */
size_t hyb_attn_decode_workspace_size(int32_t layer_type, int32_t B, int64_t max_len);
hyb_status hyb_attn_decode(const void* q, const void* gate, const int32_t* pos,
                           const hyb_kv_cache* cache, int32_t layer_type, int64_t max_len,
                           void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sequence-sharded decode.  A long full-layer history can be spread over
 * several caches (one per GPU, each holding any subset of the sequence's
 * tokens, keys rotated at their own positions); attention over the union is
 * the log-sum-exp merge of the attention over each part (the split-KV
 * combination, "百万 Token 塞进 4B ..." §"省显存的第二板斧" for the gate):
 *
 * hyb_attn_decode_partial: attention of the B queries over the keys in
 *   `cache` only, without the gate.
 *   q, pos, cache, layer_type, max_len, workspace: as hyb_attn_decode; pos
 *          should hold the query's position in the whole sequence (NULL
 *          means len - 1 of this cache).
 *   part_o  : fp32 [B][16][256], the softmax-normalised output over these keys.
 *   part_lse: fp32 [B][16], log2 of sum_j exp(q . k_j / 16) over these keys
 *             (-inf for a sequence with no keys here; part_o is then 0).
 * hyb_attn_decode_merge: merges n_parts such partials -- part p's output
 *   [B][16][256] at part_o + p * o_stride and its lse [B][16] at part_lse +
 *   p * lse_stride (strides in floats; 0 = dense, B x 4096 and B x 16) --
 *   weighting part p by 2^lse, applies sigmoid(gate) (bf16 [B][16] or NULL)
 *   and writes bf16 out [B][16][256].  The caller moves the partials between
 *   GPUs (16 KB per sequence per part); with each part's output and lse in
 *   one record of B x 16 x 257 floats (lse after the output), one
 *   all-gather of the records and o_stride = lse_stride = B x 16 x 257 do it.
 * Errors: as hyb_attn_decode; merge: HYB_EINVAL (null buffer, n_parts or
 * B <= 0), HYB_ESHAPE (a stride below one part), HYB_EALIGN, HYB_EOVERFLOW
 * (more than 2^31 elements).
 */
hyb_status hyb_attn_decode_partial(const void* q, const int32_t* pos, const hyb_kv_cache* cache,
                                   int32_t layer_type, int64_t max_len, float* part_o, float* part_lse,
                                   void* workspace, size_t workspace_bytes, void* stream);
hyb_status hyb_attn_decode_merge(const float* part_o, const float* part_lse, int64_t o_stride, int64_t lse_stride,
                                 int32_t n_parts, int32_t B, const void* gate, void* out, void* stream);

/*
 * hyb_attn_decode without a workspace.  The pages describe no counterpart:
 * this entry point exists for callers that may not allocate device memory
 * on their call path -- for example a plugin inside a host application that
 * owns every device allocation, or a latency-critical decode loop in which a
 * cudaMalloc / cudaFree would stall the whole device.  It computes exactly
 * what hyb_attn_decode computes (same arguments, minus the workspace) and
 * allocates nothing; the split partials go to a fixed 4 MiB scratch array
 * inside the library, which every GPU that loads the library holds until
 * the process exits.
 *   Limit: batch x 16 heads x splits x 1028 bytes (plus alignment) must fit
 *   in 4 MiB, i.e. hyb_attn_decode_workspace_size(layer_type, batch,
 *   max_len) <= 4194304; larger calls return HYB_EOVERFLOW and enqueue
 *   nothing.
 *   Set-up: the first call on a device looks up the scratch's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is cached with the CUDA context
 *   it belongs to: after cudaDeviceReset, or from another context, the next
 *   call looks it up again (make that call outside a capture too).
 *   Sharing: every call uses the same scratch, which keeps the previous
 *   call's contents (nothing in it needs to start at zero).  Calls whose
 *   kernels can overlap on the GPU -- e.g. on two streams without ordering
 *   between them -- race on it and give wrong results.
 * Errors: as hyb_attn_decode, plus HYB_EOVERFLOW above the limit.
 */
hyb_status hyb_attn_decode_noalloc(const void* q, const void* gate, const int32_t* pos,
                                   const hyb_kv_cache* cache, int32_t layer_type, int64_t max_len,
                                   void* out, void* stream);

/*
 * Synchronises `stream`, copies the current device's error word to
 * *flags (host) and, if clear != 0, resets it.
 */
hyb_status hyb_device_error(int32_t* flags, int32_t clear, void* stream);

/*
 * Linear projection Y = X W^T, the q_k_v_proj / gate / o_proj GEMMs around the
 * attention core ("百万 Token 塞进 4B ..." §"省显存的第二板斧": the fused
 * q_k_v_proj output is sliced into q, k and v; the gate has one score per
 * head; o_proj maps the 16 x 256 attention output back to the residual
 * width).  Device pointers, caller-owned, row-major bf16:
 *   x [M][ldx] (K used), w [N][ldw] (K used; PyTorch Linear weight layout
 *   [out_features][in_features]), y [M][ldy] (N written).
 * fp32 accumulation; y is rounded to bf16 once.  N, K, ldx, ldw, ldy must be
 * multiples of 8 and the pointers 16-byte aligned (HYB_ESHAPE / HYB_EALIGN
 * otherwise, checked before any launch).  Asynchronous on `stream`.
 * A few rows (M <= 16, K a multiple of 512 up to 4096: the projections of a
 * decode step) run on a kernel that streams W across every SM (split-K in
 * thread-block clusters) instead of the tiled tensor-core GEMM; the
 * result is the same up to fp32 summation order.
 */
hyb_status hyb_linear(const void* x, int64_t ldx, const void* w, int64_t ldw, void* y, int64_t ldy, int32_t M,
                      int32_t N, int32_t K, void* stream);

/*
 * One whole attention layer of the model for prefill ("百万 Token 塞进 4B ..."
 * §"省显存的第二板斧"): the fused q_k_v_proj, the head-wise gate projection,
 * the attention core of hyb_attn_prefill (RoPE, masked GQA, sigmoid gate,
 * cache update) and o_proj.
 *   hidden : bf16 [B][T][2560] contiguous (the layer's input, hidden_size 2560).
 *   w_qkv  : bf16 [6144][2560], rows q (4096) | k (1024) | v (1024).
 *   w_gate : bf16 [16][2560], one gate score per head, or NULL (no gate).
 *   w_o    : bf16 [2560][4096].
 *   pos, layer_type, B, T, cache: as hyb_attn_prefill.
 *   out    : bf16 [B][T][2560].
 *   workspace: at least hyb_attn_layer_prefill_workspace_size(layer_type, B,
 *          T, 0) bytes without a cache, hyb_attn_layer_prefill_cache_
 *          workspace_size(cache, T) with one (the two agree for bf16 caches),
 *          256-byte aligned; it holds the fused q|k|v rows, the gate scores
 *          and the attention output (bf16, as the model's tensors are)
 *          between the steps, the (cos, sin) table of the rows' positions
 *          that the q_k_v_proj epilogue rotates with, and the attention's own
 *          scratch.
 * Errors: as hyb_linear and hyb_attn_prefill.
 */
size_t hyb_attn_layer_prefill_workspace_size(int32_t layer_type, int32_t B, int32_t T, int32_t with_cache);
size_t hyb_attn_layer_prefill_cache_workspace_size(const hyb_kv_cache* cache, int32_t T);
hyb_status hyb_attn_layer_prefill(const void* hidden, const void* w_qkv, const void* w_gate, const void* w_o,
                                  const int32_t* pos, int32_t layer_type, int32_t B, int32_t T, void* out,
                                  const hyb_kv_cache* cache, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * One whole attention layer for a decode step: q_k_v_proj (RoPE of q and k at
 * the new token's position, the cache length), the gate projection, the KV
 * append of the new token, the attention of hyb_attn_decode and o_proj.
 *   hidden : bf16 [B][2560] (one token per sequence, B = cache->batch).
 *   w_qkv, w_gate (or NULL), w_o : as hyb_attn_layer_prefill.
 *   cache, layer_type, max_len : as hyb_attn_decode (max_len bounds the length
 *          after this step's append).
 *   out    : bf16 [B][2560].
 *   workspace: at least hyb_attn_layer_decode_workspace_size(layer_type, B,
 *          max_len) bytes, 256-byte aligned.
 * Errors: as hyb_linear, hyb_kv_append and hyb_attn_decode.
 */
size_t hyb_attn_layer_decode_workspace_size(int32_t layer_type, int32_t B, int64_t max_len);
hyb_status hyb_attn_layer_decode(const void* hidden, const void* w_qkv, const void* w_gate, const void* w_o,
                                 const hyb_kv_cache* cache, int32_t layer_type, int64_t max_len, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Failure-path self-test (no counterpart in the pages).  Launches one block
 * on `stream` whose first thread waits on a shared-memory barrier that
 * nothing completes.  The wait is bounded like every pipeline wait of the
 * library: it gives up after its limit (about 2 s of device time; 1 ms once
 * the error word already holds HYB_DEV_ERR_TIMEOUT), raises
 * HYB_DEV_ERR_TIMEOUT in the error word and the kernel returns, leaving the
 * context usable.  Returns HYB_ECUDA if the launch fails.
 */
hyb_status hyb_selftest_wait_timeout(void* stream);

/* Message for the last non-OK status returned on the calling thread. */
const char* hyb_last_error(void);

/* Number of kernels this library has launched in the process so far. */
uint64_t hyb_launch_count(void);

/*
 * How this copy of the library was built (host only, needs no device):
 * bit HYB_BUILD_DEBUG_BOUNDS is set in the debug build (compiled with
 * -DHYB_DEBUG_BOUNDS, shipped beside the normal one as
 * libhyb_attn_debug.so), whose kernels check the index of every plain
 * global load and store against its buffer, raise HYB_DEV_ERR_BOUNDS and
 * skip the access when it falls outside; they never trap.  The normal build
 * returns 0.
 */
#define HYB_BUILD_DEBUG_BOUNDS 1
int32_t hyb_build_flags(void);

/*
 * Profiling aid.  `events` is a host array of 2 * n_pairs cudaEvent_t handles
 * (passed as void*) owned by the caller.  The next n_pairs launches of an
 * attention kernel (the prefill attention kernel or the decode split-KV
 * kernel) each record events[2i] just before and events[2i+1] just after the
 * launch, on the launch's stream.  n_pairs = 0 (or events = NULL) disables
 * it.  The array must stay valid until all pairs are used or profiling is
 * disabled.  Not thread-safe with concurrent library calls.
 */
hyb_status hyb_profile_events(void* const* events, int32_t n_pairs);
/* Pairs recorded since the last hyb_profile_events call. */
int32_t hyb_profile_pairs_used(void);

#ifdef __cplusplus
}
#endif
#endif /* HYB_ATTN_H */
