// KV-side kernels: rotate keys and place them (with the values) where the
// attention kernels read them, plus the KV-cache bookkeeping.
//
//   * linear append (full layers): token i of a sequence -> slot i;
//   * ring append (sliding layers): token i -> slot (head0 + i) % 512, only the
//     last 512 tokens of a call are written, each slot tagged with the
//     sequence index it holds ("keep only the most recent 512 tokens":
//     "不用高显存卡也能跑！..." §"百万上下文的真正瓶颈");
//   * rotated-key scratch for a cache-less prefill;
//   * the sliding-layer context buffer of a chunked prefill: the ring's last
//     511 tokens in sequence order followed by the chunk's own keys;
//   * the commit step that advances len / head once all writes are done.
//
// Keys are rotated with rotate-half RoPE ("百万 Token 塞进 4B ..." §"滑动窗口
// 的补救：分层 RoPE 与局部/全局分工"): sliding layers theta 1e4 over all 256
// dims, full layers theta 5e6 over the first 64 dims.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace hyb {

// Where a key row goes.
enum DstMode : int {
  kDstLinear = 0,   // cache slot len[b] + t, capacity checked
  kDstRing = 1,     // cache slot (head[b] + t) % 512 for the last 512 tokens, tag written
  kDstRows = 2,     // dst row t (+ row offset) of a [B][4][rows][256] buffer
};

struct RopeStoreArgs {
  const __nv_bfloat16* k;   // source: token t, KV head h of sequence b at
  const __nv_bfloat16* v;   //   b*src_bstride + t*src_tstride + h*src_hstride (elements)
  int64_t src_bstride, src_tstride, src_hstride;   // v may be null: values not copied
  int src_rotated;          // 1: k is already rotated (copy as is)
  const int32_t* pos;       // [B][T] RoPE positions or null (sequence index)
  __nv_bfloat16* dk;        // destination [B][4][dst_rows][256]
  __nv_bfloat16* dv;
  int64_t dst_rows;
  int dst_row_offset;       // kDstRows: first destination row
  int mode;
  int32_t* len;             // cache bookkeeping (linear / ring) and default positions
  int32_t* head;
  int32_t* tag;
  int B, T;
  int t_first;              // first token index written (ring: max(0, T - 512))
  int fp8;                  // 1: dk / dv hold e4m3 codes (1 byte), scales to dks / dvs
  float* dks;               // [B][4][dst_rows]
  float* dvs;
  PageMap pm;               // linear mode, paged cache: destination [n_pages][4][page][256]
  int commit;               // 1: grid = B, block b owns sequence b and advances its len (and
                            //    ring head) after its rows, as kv_commit_kernel would
  int64_t capacity;         // commit, linear mode: the cache capacity
  int qdq;                  // rows mode: each row written as its e4m3 quantization, dequantized
};

// One 256-dim row (one token, one KV head) held by a warp, 8 bf16 values per
// lane in `x`: e4m3 codes with scale amax / 448, codes = satfinite round to
// nearest even of value * (448 / amax) (a zero row: scale 0, codes 0).
// Returns this lane's 8 codes (lowest byte first) and the row's scale.
__device__ __forceinline__ uint2 quantize_row_fp8(uint4 x, float* scale) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  float f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16lo(w[i]);
    f[2 * i + 1] = bf16hi(w[i]);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float inv = amax > 0.f ? 448.f / amax : 0.f;
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {   // element 2i in the low byte
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(f[2 * i + 1] * inv), "f"(f[2 * i] * inv));
    c[i] = h;
  }
  *scale = amax / 448.f;
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}
__device__ __forceinline__ void store_row_fp8(uint4 x, uint8_t* dst, float* dscale, int lane) {
  float sc;
  *reinterpret_cast<uint2*>(dst) = quantize_row_fp8(x, &sc);
  if (lane == 0) *dscale = sc;
}

// Eight e4m3 codes (8 bytes, lowest first) times `scale`, rounded to bf16
// (8 values in 16 bytes, same order).  The codes are widened exactly (value
// x 2^-120 by bit moves, then x 2^120 in fp32), then scaled in fp32.
__device__ __forceinline__ uint4 dequant8_bf16(uint2 codes, float scale) {
  const uint32_t w[2] = {codes.x, codes.y};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t a = e4m3_b02_bf16x2(w[i]), c = e4m3_b13_bf16x2(w[i]);   // codes (0, 2) and (1, 3)
    const float v0 = __uint_as_float(a << 16) * kE4m3WideScale * scale;
    const float v2 = __uint_as_float(a & 0xFFFF0000u) * kE4m3WideScale * scale;
    const float v1 = __uint_as_float(c << 16) * kE4m3WideScale * scale;
    const float v3 = __uint_as_float(c & 0xFFFF0000u) * kE4m3WideScale * scale;
    o[2 * i] = pack_bf16(v0, v1);
    o[2 * i + 1] = pack_bf16(v2, v3);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// One block = one token of one sequence, 128 threads; thread i handles
// 8 consecutive dims (16 bytes) of KV head i / 32.  Rotation partners
// (k, k + R/2) sit in lanes i and i ^ 16 (R = 256) or i ^ 4 (R = 64).  The
// token's R/2 (cos, sin) pairs are computed once (one per thread) into
// shared memory and shared by the 4 heads.  Every branch that skips a job
// depends on the job only, so the whole block takes it.
template <bool FULL>
__global__ void __launch_bounds__(128) rope_store_kernel(RopeStoreArgs a) {
  constexpr int R = RopeCfg<FULL>::R;
  __shared__ double inv_freq[R / 2];
  __shared__ float2 cs[R / 2];
  for (int i = threadIdx.x; i < R / 2; i += blockDim.x) inv_freq[i] = rope_inv_freq<FULL>(i);
  __syncthreads();
  pdl_wait();   // earlier kernels write the keys, values and the cache state read below
  pdl_launch_dependents();

  const int n_tok = a.T - a.t_first;
  const int lane32 = threadIdx.x & 31;
  const int kvh = threadIdx.x >> 5;
  const int d0 = lane32 * 8;
  // jobs token-major: with grid = B (commit) block b takes exactly sequence b's tokens
  int seen_len = 0, seen_head = 0;   // the cache state this thread read (commit: sequence blockIdx.x's)
  bool seen = false;
  for (int job = blockIdx.x; job < a.B * n_tok; job += gridDim.x) {
    const int b = job % a.B;
    const int t = a.t_first + job / a.B;
    const int64_t src = (int64_t)b * a.src_bstride + (int64_t)t * a.src_tstride + (int64_t)kvh * a.src_hstride + d0;
    // the row's K / V loads go out first, with the cache state's: none depends on another
    uint4 kx = *reinterpret_cast<const uint4*>(a.k + src);
    const uint4 vx = a.v != nullptr ? *reinterpret_cast<const uint4*>(a.v + src) : make_uint4(0, 0, 0, 0);
    int64_t dst_row;
    const int L = (a.len != nullptr) ? a.len[b] : 0;
    const int H = a.mode == kDstRing ? a.head[b] : 0;
    seen_len = L;
    seen_head = H;
    seen = true;
    if (a.mode == kDstLinear) {
      if ((int64_t)L + a.T > a.dst_rows) {  // capacity exceeded: leave the sequence unchanged
        if (t == a.t_first && threadIdx.x == 0) raise_err(kErrCapacity);
        continue;
      }
      dst_row = L + t;
    } else if (a.mode == kDstRing) {
      const int slot = (H + t) % kWindow;
      dst_row = slot;
      if (threadIdx.x == 0) a.tag[(int64_t)b * kWindow + slot] = L + t;
    } else {
      dst_row = a.dst_row_offset + t;
    }
    if (!HYB_BOUNDS(dst_row, 0, a.dst_rows)) continue;   // debug build: a row outside the destination
    int64_t row_id = ((int64_t)b * kHkv + kvh) * a.dst_rows + dst_row;   // row of the [..][4][rows] layout
    if (a.mode == kDstLinear && a.pm.page != 0) {
      int prow, ppage;
      kv_coord(a.pm, b, (int)dst_row, prow, ppage);
      if (ppage < 0) continue;   // bad block-table entry: raised, row skipped
      row_id = ((int64_t)ppage * kHkv + kvh) * a.pm.page + prow;
    }
    const int64_t dst = row_id * kD + d0;

    if (!a.src_rotated) {
      const int p = a.pos ? a.pos[(int64_t)b * a.T + t] : L + t;
      __syncthreads();   // the previous job's pairs have been used
      if (threadIdx.x < R / 2) {
        float sn, c;
        rope_sincos(p, inv_freq[threadIdx.x], &sn, &c);
        cs[threadIdx.x] = make_float2(c, sn);
      }
      __syncthreads();
      const uint32_t xs[4] = {kx.x, kx.y, kx.z, kx.w};
      uint32_t ys[4];
      constexpr int xor_mask = (R == 256) ? 16 : 4;
#pragma unroll
      for (int w = 0; w < 4; ++w) ys[w] = __shfl_xor_sync(0xffffffffu, xs[w], xor_mask);
      if (d0 < R) {
        const bool first_half = d0 < R / 2;
        const int kbase = first_half ? d0 : d0 - R / 2;
        uint32_t os[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          float o2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x = e ? bf16hi(xs[w]) : bf16lo(xs[w]);
            const float y = e ? bf16hi(ys[w]) : bf16lo(ys[w]);
            const float2 r = cs[kbase + 2 * w + e];
            // first half: x cos - y sin (y = x[k + R/2]); second half: x cos + y sin (y = x[k])
            o2[e] = first_half ? fmaf(x, r.x, -y * r.y) : fmaf(x, r.x, y * r.y);
          }
          os[w] = pack_bf16(o2[0], o2[1]);
        }
        kx = make_uint4(os[0], os[1], os[2], os[3]);
      }
    }
    if (a.qdq) {   // the rows an FP8 ring will hold, as attention reads them back
      float sc;
      uint2 c = quantize_row_fp8(kx, &sc);
      kx = dequant8_bf16(c, sc);
      if (a.v != nullptr) {
        c = quantize_row_fp8(vx, &sc);
        *reinterpret_cast<uint4*>(a.dv + dst) = dequant8_bf16(c, sc);
      }
      *reinterpret_cast<uint4*>(a.dk + dst) = kx;
      continue;
    }
    if (a.fp8) {
      store_row_fp8(kx, reinterpret_cast<uint8_t*>(a.dk) + dst, a.dks + row_id, lane32);
      if (a.v != nullptr)
        store_row_fp8(vx, reinterpret_cast<uint8_t*>(a.dv) + dst,
                      a.dvs + row_id, lane32);
      continue;
    }
    *reinterpret_cast<uint4*>(a.dk + dst) = kx;
    if (a.v != nullptr) {
      *reinterpret_cast<uint4*>(a.dv + dst) = vx;
    }
  }
  if (a.commit) {
    __syncthreads();   // every row of sequence blockIdx.x has read len / head
    if (threadIdx.x == 0 && blockIdx.x < a.B) {
      const int b = blockIdx.x;
      // the values this thread read above (nothing in this launch writes them before here)
      const int L = seen ? seen_len : a.len[b];
      if (a.mode == kDstRing) {
        a.head[b] = ((seen ? seen_head : a.head[b]) + a.T) % kWindow;
        a.len[b] = L + a.T;
      } else if ((int64_t)L + a.T <= a.capacity) {
        a.len[b] = L + a.T;
      }
    }
  }
}

// Context rows [0, 511) of a chunked sliding prefill: row r holds sequence
// index len - 511 + r, read from the ring (FP8 rings: dequantized to bf16 when
// rks / rvs are given); rows before the start of the sequence (or a slot
// whose tag does not match) are zero-filled so that the masked products stay
// finite.
__global__ void __launch_bounds__(128) ring_gather_kernel(const __nv_bfloat16* rk, const __nv_bfloat16* rv,
                                                          const float* rks, const float* rvs,
                                                          const int32_t* len, const int32_t* head,
                                                          const int32_t* tag, __nv_bfloat16* ck,
                                                          __nv_bfloat16* cv, int64_t ctx_rows, int B) {
  const int lane32 = threadIdx.x & 31;
  const int kvh = threadIdx.x >> 5;
  const int d0 = lane32 * 8;
  constexpr int P = kWindow - 1;
  for (int job = blockIdx.x; job < B * P; job += gridDim.x) {
    const int b = job / P;
    const int r = job % P;
    const int L = len[b];
    const int seq = L - P + r;
    const int slot = ((head[b] - L + seq) % kWindow + kWindow) % kWindow;
    const bool ok = seq >= 0 && HYB_BOUNDS(slot, 0, kWindow) && tag[(int64_t)b * kWindow + slot] == seq;
    if (!HYB_BOUNDS(r, 0, ctx_rows)) continue;   // debug build: a row outside the context buffer
    const int64_t dst = (((int64_t)b * kHkv + kvh) * ctx_rows + r) * kD + d0;
    uint4 kx = make_uint4(0, 0, 0, 0), vx = make_uint4(0, 0, 0, 0);
    if (ok) {
      const int64_t sid = ((int64_t)b * kHkv + kvh) * kWindow + slot;
      if (rks != nullptr) {
        const uint8_t* k8 = reinterpret_cast<const uint8_t*>(rk);
        const uint8_t* v8 = reinterpret_cast<const uint8_t*>(rv);
        kx = dequant8_bf16(*reinterpret_cast<const uint2*>(k8 + sid * kD + d0), rks[sid]);
        vx = dequant8_bf16(*reinterpret_cast<const uint2*>(v8 + sid * kD + d0), rvs[sid]);
      } else {
        kx = *reinterpret_cast<const uint4*>(rk + sid * kD + d0);
        vx = *reinterpret_cast<const uint4*>(rv + sid * kD + d0);
      }
    }
    *reinterpret_cast<uint4*>(ck + dst) = kx;
    *reinterpret_cast<uint4*>(cv + dst) = vx;
  }
}

// Rotated copy of the query rows of a prefill: dst [B][T][16][256] from rows
// of 16 x 256 at src + (b T + t) src_tstride, at position pos[b][t], else
// (len ? len[b] : 0) + t.  One block per token: its R/2 (cos, sin) pairs once
// in shared memory (the fp64-reduced angle), then the 16 heads, one warp per
// head at a time, 8 dims per lane (the partner dims R/2 away in another lane).
template <bool FULL>
__global__ void __launch_bounds__(128) rope_q_kernel(const __nv_bfloat16* src, int64_t src_tstride,
                                                     const int32_t* pos, const int32_t* len, int B, int T,
                                                     __nv_bfloat16* dst) {
  constexpr int R = RopeCfg<FULL>::R;
  __shared__ double inv_freq[R / 2];
  __shared__ float2 cs[R / 2];
  for (int i = threadIdx.x; i < R / 2; i += blockDim.x) inv_freq[i] = rope_inv_freq<FULL>(i);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d0 = lane * 8;
  constexpr int xor_mask = (R == 256) ? 16 : 4;
  for (int64_t m = blockIdx.x; m < (int64_t)B * T; m += gridDim.x) {
    const int b = (int)(m / T), t = (int)(m % T);
    const int p = pos ? pos[m] : (len ? len[b] : 0) + t;
    uint4 qv[kHq / 4];   // this warp's 4 heads, loaded before the angles are ready
#pragma unroll
    for (int j = 0; j < kHq / 4; ++j) qv[j] = *reinterpret_cast<const uint4*>(src + m * src_tstride + (warp + 4 * j) * kD + d0);
    __syncthreads();   // inv_freq written / the previous token's pairs consumed
    for (int k = threadIdx.x; k < R / 2; k += blockDim.x) {
      float sn, c;
      rope_sincos(p, inv_freq[k], &sn, &c);
      cs[k] = make_float2(c, sn);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kHq / 4; ++j) {
      const int h = warp + 4 * j;
      uint4 qx = qv[j];
      const uint32_t xs[4] = {qx.x, qx.y, qx.z, qx.w};
      uint32_t ys[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) ys[w] = __shfl_xor_sync(0xffffffffu, xs[w], xor_mask);
      if (d0 < R) {
        const bool first_half = d0 < R / 2;
        const int kb = first_half ? d0 : d0 - R / 2;
        uint32_t os[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          float o2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x = e ? bf16hi(xs[w]) : bf16lo(xs[w]);
            const float y = e ? bf16hi(ys[w]) : bf16lo(ys[w]);
            const float2 r = cs[kb + 2 * w + e];
            // first half: x cos - y sin (y = x[k + R/2]); second half: x cos + y sin (y = x[k])
            o2[e] = first_half ? fmaf(x, r.x, -y * r.y) : fmaf(x, r.x, y * r.y);
          }
          os[w] = pack_bf16(o2[0], o2[1]);
        }
        qx = make_uint4(os[0], os[1], os[2], os[3]);
      }
      *reinterpret_cast<uint4*>(dst + m * (kHq * kD) + h * kD + d0) = qx;
    }
  }
}

// RoPE (cos, sin) for every (row, frequency) of a projection's output rows,
// the same fp64-reduced angle as the other rotations.
template <bool FULL>
__global__ void __launch_bounds__(256) rope_table_kernel(const int32_t* pos, const int32_t* len, int T, int M,
                                                         float2* tab) {
  constexpr int R = RopeCfg<FULL>::R;
  __shared__ double inv_freq[R / 2];
  for (int i = threadIdx.x; i < R / 2; i += blockDim.x) inv_freq[i] = rope_inv_freq<FULL>(i);
  __syncthreads();
  const int64_t n = (int64_t)M * (R / 2);
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(idx / (R / 2)), k = (int)(idx % (R / 2));
    const int p = pos ? pos[m] : (len ? len[m / T] : 0) + m % T;
    float s, c;
    rope_sincos(p, inv_freq[k], &s, &c);
    tab[idx] = make_float2(c, s);
  }
}

// Advances the cache state after an append of T tokens.  A full-layer
// sequence that would overflow its capacity is not advanced (its rows were
// not written either).
__global__ void kv_commit_kernel(int32_t* len, int32_t* head, int64_t capacity, int is_ring, int B, int T) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  if (is_ring) {
    head[b] = (head[b] + T) % kWindow;
    len[b] += T;
  } else if ((int64_t)len[b] + T <= capacity) {
    len[b] += T;
  }
}

__global__ void fill_i32_kernel(int32_t* p, int64_t n, int32_t v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
static int rope_grid(int jobs) {
  int g = jobs;
  const int cap = 148 * 16;
  return g < cap ? (g > 0 ? g : 1) : cap;
}

cudaError_t launch_rope_store(bool full, const RopeStoreHost& h, cudaStream_t st) {
  RopeStoreArgs a;
  a.k = reinterpret_cast<const __nv_bfloat16*>(h.k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(h.v);
  a.src_bstride = h.src_bstride;
  a.src_tstride = h.src_tstride;
  a.src_hstride = h.src_hstride;
  a.src_rotated = h.src_rotated;
  a.fp8 = h.fp8;
  a.dks = h.dks;
  a.dvs = h.dvs;
  a.pm = h.pm;
  a.pos = h.pos;
  a.dk = reinterpret_cast<__nv_bfloat16*>(h.dk);
  a.dv = reinterpret_cast<__nv_bfloat16*>(h.dv);
  a.dst_rows = h.dst_rows;
  a.dst_row_offset = h.dst_row_offset;
  a.mode = h.mode;
  a.len = h.len;
  a.head = h.head;
  a.tag = h.tag;
  a.B = h.B;
  a.T = h.T;
  a.t_first = h.t_first;
  a.commit = h.commit;
  a.capacity = h.capacity;
  a.qdq = h.qdq;
  const int grid = h.commit ? h.B : rope_grid(h.B * (h.T - h.t_first));
  cudaError_t e = full ? launch_pdl(rope_store_kernel<true>, dim3(grid, 1, 1), dim3(128, 1, 1), 0, st, 0u, a)
                       : launch_pdl(rope_store_kernel<false>, dim3(grid, 1, 1), dim3(128, 1, 1), 0, st, 0u, a);
  count_launch();
  return e;
}

cudaError_t launch_ring_gather(const void* rk, const void* rv, const float* rks, const float* rvs,
                               const int32_t* len, const int32_t* head, const int32_t* tag, void* ck, void* cv,
                               int64_t ctx_rows, int B, cudaStream_t st) {
  ring_gather_kernel<<<rope_grid(B * (kWindow - 1)), 128, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(rk), reinterpret_cast<const __nv_bfloat16*>(rv), rks, rvs, len, head,
      tag, reinterpret_cast<__nv_bfloat16*>(ck), reinterpret_cast<__nv_bfloat16*>(cv), ctx_rows, B);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_rope_table(bool full, const int32_t* pos, const int32_t* len, int T, int M, void* tab,
                              cudaStream_t st) {
  const int64_t n = (int64_t)M * (full ? 32 : 128);
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 148 * 8);
  if (full)
    rope_table_kernel<true><<<grid, 256, 0, st>>>(pos, len, T > 0 ? T : 1, M, reinterpret_cast<float2*>(tab));
  else
    rope_table_kernel<false><<<grid, 256, 0, st>>>(pos, len, T > 0 ? T : 1, M, reinterpret_cast<float2*>(tab));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_rope_q(bool full, const void* src, int64_t src_tstride, const int32_t* pos, const int32_t* len,
                          int B, int T, void* dst, cudaStream_t st) {
  const int64_t n = (int64_t)B * T;
  const int grid = (int)std::min<int64_t>(n, 148 * 16);
  if (full)
    rope_q_kernel<true><<<grid, 128, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(src), src_tstride, pos, len, B,
                                              T, reinterpret_cast<__nv_bfloat16*>(dst));
  else
    rope_q_kernel<false><<<grid, 128, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(src), src_tstride, pos, len, B,
                                               T, reinterpret_cast<__nv_bfloat16*>(dst));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_kv_commit(int32_t* len, int32_t* head, int64_t capacity, bool ring, int B, int T,
                             cudaStream_t st) {
  kv_commit_kernel<<<(B + 127) / 128, 128, 0, st>>>(len, head, capacity, ring ? 1 : 0, B, T);
  count_launch();
  return cudaGetLastError();
}

// One thread waits on a barrier that nothing completes; the bounded wait
// raises the timeout bit and the kernel ends (failure-path self-test).
__global__ void selftest_wait_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    (void)mbar_wait(&bar, 0);
  }
}

cudaError_t launch_selftest_wait(cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>();
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fill_i32(int32_t* p, int64_t n, int32_t v, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  fill_i32_kernel<<<(int)blocks, 256, 0, st>>>(p, n, v);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hyb
