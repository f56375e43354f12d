// Decode attention: one query token per sequence against its KV cache.
//
// Split-KV: CTA (split, kv_head, b) streams a contiguous key range of one KV
// head through a 3-stage TMA ring (64 keys of K and V per stage, 128-byte
// swizzled boxes) and scores the 4 query heads that share the head in one
// pass, so each K/V byte leaves HBM once ("不用高显存卡也能跑！..." §"分组查询
// 注意力": 4 query heads share one KV head).  It writes a partial output
// (normalised, fp32) and its log-sum-exp; a second kernel merges the splits
// and applies the head-wise sigmoid gate ("百万 Token 塞进 4B ..." §"省显存的
// 第二板斧").
//
// The per-key work (4 heads x 256 dims, scores and P.V) runs on mma.sync
// m16n8k16 with the 4 query heads as the M rows (rows 4..15 zero): at about
// 4 flop per byte the kernel is bound by HBM, not by the tensor pipe, and
// the warp-level MMA keeps the instruction count per key low.
//
// Warps 0-3 consume (16 keys each per stage), warp 4 issues the TMA loads.
//
// FP8 caches (e4m3 codes + one fp32 scale per key row): a stage holds the
// codes (half the bytes) and the 64 keys' scales; each consumer warp first
// widens its own 16 key rows of K and V to bf16 (exact: every e4m3 value is
// a bf16 value) in the layout the bf16 path reads, releases the stage, and
// then runs the same MMAs, with the K scale applied to the scores and the V
// scale folded into P.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kDecKeys = 64;                         // keys per stage
constexpr int kDecStages = 3;
constexpr int kDecTileBytes = kDecKeys * kD * 2;     // 32 KB (K or V)
constexpr int kDecStageBytes = 2 * kDecTileBytes;    // K + V
constexpr int kDecThreads = 160;
constexpr int kBoxBytes = kDecKeys * 128;            // one 64-dim box of 64 keys
// FP8 layout inside DecSmem::stage: per stage K codes (2 boxes of 128 dims),
// V codes, K scales, V scales; then the widened bf16 K and V tiles.
constexpr int kDec8TileBytes = kDecKeys * kD;        // 16 KB of codes
constexpr int kDec8Box = kDecKeys * 128;             // 128 dims x 64 keys
constexpr int kDec8StageBytes = 2 * kDec8TileBytes + 2 * kDecKeys * 4 + 512;   // padded to 1 KB multiples
constexpr int kDec8Wide = kDecStages * kDec8StageBytes;                         // widened tiles start here

struct DecSmem {
  // stage buffers first (1024-byte aligned base)
  uint8_t stage[kDecStages][kDecStageBytes];
  float merge_o[4][4][kD];      // [warp][head][dim]
  float merge_m[4][4];
  float merge_l[4][4];
  __nv_bfloat16 qs[4][kD];      // rotated queries of the group
  int32_t tags[kWindow];
  uint64_t full[kDecStages];
  uint64_t empty[kDecStages];
};

size_t decode_smem_bytes() { return sizeof(DecSmem) + 1024; }
static_assert(kDec8StageBytes % 1024 == 0, "FP8 stage must keep 1 KB alignment");
static_assert(kDec8Wide + 2 * kDecTileBytes <= kDecStages * kDecStageBytes, "FP8 stages + widened tiles must fit");

struct DecArgs {
  const __nv_bfloat16* q;
  int64_t q_stride;   // elements between the query rows of consecutive sequences
  int q_rotated;      // 1: the queries arrive rotated
  const int32_t* pos;
  const int32_t* len;
  const int32_t* tag;
  float* part_o;
  float* part_lse;
  int n_splits;
};

template <bool FULL, bool FP8>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                        DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int R = RopeCfg<FULL>::R;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int L = a.len[b];
  const int qseq = L - 1;
  const int n_keys = FULL ? L : kWindow;          // keys (FULL) or ring slots (SLIDING)
  int kps = (n_keys + a.n_splits - 1) / a.n_splits;
  kps = (kps + kDecKeys - 1) / kDecKeys * kDecKeys;
  const int k0 = split * kps;
  const int k1 = min(n_keys, k0 + kps);
  const int n_stages = (k1 > k0 && L > 0) ? (k1 - k0 + kDecKeys - 1) / kDecKeys : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 4);
    }
    fence_barrier_init();
  }
  if (!FULL) {
    for (int i = threadIdx.x; i < kWindow; i += blockDim.x) sm.tags[i] = a.tag[(int64_t)b * kWindow + i];
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------- producer ----------------
    if (lane == 0 && n_stages > 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int i = 0; i < n_stages; ++i) {
        const int slot = i % kDecStages;
        if (i >= kDecStages && !mbar_wait(&sm.empty[slot], ((i / kDecStages) - 1) & 1)) break;
        const int key = k0 + i * kDecKeys;
        if (FP8) {
          mbar_arrive_expect_tx(&sm.full[slot], 2 * kDec8TileBytes + 2 * kDecKeys * 4);
          const uint32_t kdst = smem_u32(sm.stage[0]) + slot * kDec8StageBytes;
          const uint32_t vdst = kdst + kDec8TileBytes;
#pragma unroll
          for (int box = 0; box < 2; ++box) {
            tma_load_4d(kdst + box * kDec8Box, &tm_k, &sm.full[slot], box * 128, key, kvh, b);
            tma_load_4d(vdst + box * kDec8Box, &tm_v, &sm.full[slot], box * 128, key, kvh, b);
          }
          tma_load_3d(vdst + kDec8TileBytes, &tm_ks, &sm.full[slot], key, kvh, b);
          tma_load_3d(vdst + kDec8TileBytes + kDecKeys * 4, &tm_vs, &sm.full[slot], key, kvh, b);
          issued = i + 1;
          continue;
        }
        mbar_arrive_expect_tx(&sm.full[slot], kDecStageBytes);
        const uint32_t kdst = smem_u32(sm.stage[slot]);
        const uint32_t vdst = kdst + kDecTileBytes;
#pragma unroll
        for (int box = 0; box < 4; ++box) {
          tma_load_4d(kdst + box * kBoxBytes, &tm_k, &sm.full[slot], box * 64, key, kvh, b);
          tma_load_4d(vdst + box * kBoxBytes, &tm_v, &sm.full[slot], box * 64, key, kvh, b);
        }
        issued = i + 1;
      }
      // drain: never leave the CTA with copies still landing in shared memory
      for (int i = max(0, issued - kDecStages); i < issued; ++i)
        mbar_wait(&sm.full[i % kDecStages], (i / kDecStages) & 1);
    }
    return;
  }

  // ---------------- consumers: rotate the group's 4 queries ----------------
  {
    const int hh = threadIdx.x >> 5;        // 0..3
    const int d0 = lane * 8;
    const int p = a.pos ? a.pos[b] : qseq;
    uint4 qx = *reinterpret_cast<const uint4*>(a.q + (int64_t)b * a.q_stride + (int64_t)(kvh * kGroup + hh) * kD + d0);
    const uint32_t xs[4] = {qx.x, qx.y, qx.z, qx.w};
    uint32_t ys[4];
    constexpr int xor_mask = (R == 256) ? 16 : 4;
#pragma unroll
    for (int w = 0; w < 4; ++w) ys[w] = __shfl_xor_sync(0xffffffffu, xs[w], xor_mask);
    if (!a.q_rotated && d0 < R) {
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
          float s, c;
          rope_sincos(p, rope_inv_freq(RopeCfg<FULL>::theta, kb + 2 * w + e, R), &s, &c);
          o2[e] = first_half ? fmaf(x, c, -y * s) : fmaf(x, c, y * s);
        }
        os[w] = pack_bf16(o2[0], o2[1]);
      }
      qx = make_uint4(os[0], os[1], os[2], os[3]);
    }
    *reinterpret_cast<uint4*>(&sm.qs[hh][d0]) = qx;
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");

  const int g = lane >> 2, c = lane & 3;
  // A fragments of the rotated queries: row g = head g (g < 4), zero rows otherwise
  uint32_t qa0[16], qa2[16];
#pragma unroll
  for (int s = 0; s < 16; ++s) {
    qa0[s] = (g < 4) ? *reinterpret_cast<const uint32_t*>(&sm.qs[g & 3][16 * s + 2 * c]) : 0u;
    qa2[s] = (g < 4) ? *reinterpret_cast<const uint32_t*>(&sm.qs[g & 3][16 * s + 2 * c + 8]) : 0u;
  }

  const float scale_log2 = 0.0625f * 1.4426950408889634f;  // 1/sqrt(256) * log2(e)
  float m_run = -INFINITY, l_part = 0.f;
  float o[32][4];
#pragma unroll
  for (int n = 0; n < 32; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  const int mi = lane >> 3, rr = lane & 7;
  for (int i = 0; i < n_stages; ++i) {
    const int slot = i % kDecStages;
    if (!mbar_wait(&sm.full[slot], (i / kDecStages) & 1)) break;
    uint32_t kbase = smem_u32(sm.stage[slot]);
    uint32_t vbase = kbase + kDecTileBytes;
    float ksc[4] = {1.f, 1.f, 1.f, 1.f}, vsc[4] = {1.f, 1.f, 1.f, 1.f};   // scales of this thread's keys
    if (FP8) {
      // widen this warp's 16 key rows of K and V to bf16 (the bf16 path's layout)
      uint8_t* st8 = sm.stage[0] + slot * kDec8StageBytes;
      uint8_t* wide = sm.stage[0] + kDec8Wide;
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const uint8_t* src_t = st8 + kv * kDec8TileBytes;
        uint8_t* dst_t = wide + kv * kDecTileBytes;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int job = lane + 32 * it;
          const uint32_t r = warp * 16 + (job >> 4);
          const int cs = job & 15;                         // 16-dim chunk: dims 16 cs .. 16 cs + 15
          const uint4 cw = *reinterpret_cast<const uint4*>(src_t + (cs >> 3) * kDec8Box +
                                                           ((r * 128u) | ((((uint32_t)cs & 7u) ^ (r & 7u)) << 4)));
          const int d0 = 16 * cs;
          const uint4 lo = make_uint4(e4m3x2_to_bf16x2(cw.x & 0xFFFFu), e4m3x2_to_bf16x2(cw.x >> 16),
                                      e4m3x2_to_bf16x2(cw.y & 0xFFFFu), e4m3x2_to_bf16x2(cw.y >> 16));
          const uint4 hi = make_uint4(e4m3x2_to_bf16x2(cw.z & 0xFFFFu), e4m3x2_to_bf16x2(cw.z >> 16),
                                      e4m3x2_to_bf16x2(cw.w & 0xFFFFu), e4m3x2_to_bf16x2(cw.w >> 16));
          *reinterpret_cast<uint4*>(dst_t + (d0 >> 6) * kBoxBytes + sw128_offset(r, (d0 & 63) * 2)) = lo;
          *reinterpret_cast<uint4*>(dst_t + ((d0 + 8) >> 6) * kBoxBytes + sw128_offset(r, ((d0 + 8) & 63) * 2)) = hi;
        }
      }
      const float* kscale = reinterpret_cast<const float*>(st8 + 2 * kDec8TileBytes);
      const float* vscale = kscale + kDecKeys;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kl = warp * 16 + (e >> 1) * 8 + 2 * c + (e & 1);
        ksc[e] = kscale[kl];
        vsc[e] = vscale[kl];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);   // the codes have been read
      kbase = smem_u32(wide);
      vbase = kbase + kDecTileBytes;
    }

    // ---- scores of 16 keys x 4 heads ----
    float acc[2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2) {
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const uint32_t kr = warp * 16 + nb * 8 + rr;
        const uint32_t d = 32 * s2 + 8 * mi;
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kbase + (d >> 6) * kBoxBytes + sw128_offset(kr, (d & 63) * 2), r0, r1, r2, r3);
        mma_16816(acc[nb], qa0[2 * s2], 0u, qa2[2 * s2], 0u, r0, r1);
        mma_16816(acc[nb], qa0[2 * s2 + 1], 0u, qa2[2 * s2 + 1], 0u, r2, r3);
      }
    }
    // ---- mask, online softmax (log2 domain) ----
    float sv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = k0 + i * kDecKeys + warp * 16 + (e >> 1) * 8 + 2 * c + (e & 1);
      bool ok = key < k1;
      if (!FULL && ok) {
        const int tg = sm.tags[key];
        ok = tg >= 0 && tg <= qseq && qseq - tg < kWindow;
      }
      sv[e] = ok ? acc[e >> 1][e & 1] * ksc[e] * scale_log2 : -INFINITY;
    }
    float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = (m_run == -INFINITY) ? 1.f : exp2f(m_run - m_new);
    float pv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) pv[e] = (m_new == -INFINITY || g >= 4) ? 0.f : exp2f(sv[e] - m_new);
    m_run = m_new;
    l_part = l_part * alpha + (pv[0] + pv[1] + pv[2] + pv[3]);
#pragma unroll
    for (int n = 0; n < 32; ++n) {
      o[n][0] *= alpha;
      o[n][1] *= alpha;
    }
    const uint32_t pa0 = pack_bf16(pv[0] * vsc[0], pv[1] * vsc[1]);
    const uint32_t pa2 = pack_bf16(pv[2] * vsc[2], pv[3] * vsc[3]);
    // ---- O += P V over 256 dims ----
#pragma unroll
    for (int i2 = 0; i2 < 16; ++i2) {
      const uint32_t kr = warp * 16 + (mi & 1) * 8 + rr;
      const uint32_t d = 16 * i2 + (mi >> 1) * 8;
      uint32_t r0, r1, r2, r3;
      ldsm_x4_t(vbase + (d >> 6) * kBoxBytes + sw128_offset(kr, (d & 63) * 2), r0, r1, r2, r3);
      mma_16816(o[2 * i2], pa0, 0u, pa2, 0u, r0, r1);
      mma_16816(o[2 * i2 + 1], pa0, 0u, pa2, 0u, r2, r3);
    }
    __syncwarp();
    if (!FP8 && lane == 0) mbar_arrive(&sm.empty[slot]);
  }

  // ---------------- merge the 4 warps, write the split's partial ----------------
  float l_sum = l_part + __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_sum += __shfl_xor_sync(0xffffffffu, l_sum, 2);
  if (g < 4) {
    if (c == 0) {
      sm.merge_m[warp][g] = m_run;
      sm.merge_l[warp][g] = l_sum;
    }
#pragma unroll
    for (int n = 0; n < 32; ++n) {
      sm.merge_o[warp][g][8 * n + 2 * c] = o[n][0];
      sm.merge_o[warp][g][8 * n + 2 * c + 1] = o[n][1];
    }
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  {
    const int hh = threadIdx.x >> 5;
    const int d0 = lane * 8;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm.merge_m[w][hh]);
    float res[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float lse = -INFINITY;
    if (M != -INFINITY) {
      float den = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = sm.merge_m[w][hh];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - M);
        den += f * sm.merge_l[w][hh];
#pragma unroll
        for (int e = 0; e < 8; ++e) res[e] += f * sm.merge_o[w][hh][d0 + e];
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) res[e] *= inv;
      lse = den > 0.f ? M + log2f(den) : -INFINITY;
    }
    const int hq = kvh * kGroup + hh;
    const int64_t row = ((int64_t)b * kHq + hq) * a.n_splits + split;
    float4* dst = reinterpret_cast<float4*>(a.part_o + row * kD + d0);
    dst[0] = make_float4(res[0], res[1], res[2], res[3]);
    dst[1] = make_float4(res[4], res[5], res[6], res[7]);
    if (lane == 0) a.part_lse[row] = lse;
  }
}

// Merges the splits of one (sequence, query head) and applies the gate.
__global__ void __launch_bounds__(256) decode_combine_kernel(const float* part_o, const float* part_lse,
                                                             const __nv_bfloat16* gate, __nv_bfloat16* out,
                                                             int n_splits) {
  const int row = blockIdx.x;  // b * 16 + h
  const int d = threadIdx.x;
  const float* lse = part_lse + (int64_t)row * n_splits;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, lse[s]);
  float acc = 0.f, den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < n_splits; ++s) {
      if (lse[s] == -INFINITY) continue;
      const float w = exp2f(lse[s] - M);
      den += w;
      acc += w * part_o[((int64_t)row * n_splits + s) * kD + d];
    }
  }
  float r = den > 0.f ? acc / den : 0.f;
  if (gate != nullptr) {
    const float gs = __bfloat162float(gate[row]);
    r *= 1.f / (1.f + __expf(-gs));
  }
  out[(int64_t)row * kD + d] = __float2bfloat16_rn(r);
}

int decode_num_splits(bool full, int B, int64_t max_len) {
  const int64_t keys = full ? (max_len > 0 ? max_len : 1) : kWindow;
  const int64_t pairs = (int64_t)B * kHkv;
  const int64_t s_max = keys / 512 > 1 ? keys / 512 : 1;   // >= 8 stages of 64 keys per split
  const int sms = 148;
  int best = 1;
  double best_eff = 0.0;
  for (int64_t s = 1; s <= s_max && s <= 1024; ++s) {
    const int64_t ctas = pairs * s;
    const int64_t waves = (ctas + sms - 1) / sms;
    const double eff = (double)ctas / (double)(waves * sms);
    if (eff >= 0.95) return (int)s;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = (int)s;
    }
  }
  return best;
}

cudaError_t launch_decode(bool full, const DecodeHost& h, cudaStream_t st) {
  DecArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(h.q);
  a.q_stride = h.q_stride;
  a.q_rotated = h.q_rotated;
  a.pos = h.pos;
  a.len = h.len;
  a.tag = h.tag;
  a.part_o = h.part_o;
  a.part_lse = h.part_lse;
  a.n_splits = h.n_splits;
  const dim3 grid(h.n_splits, kHkv, h.B);
  const size_t smem = decode_smem_bytes();
  profile_before(st);
  if (full && h.fp8)
    decode_split_kernel<true, true><<<grid, kDecThreads, smem, st>>>(h.tm_k, h.tm_v, h.tm_ks, h.tm_vs, a);
  else if (full)
    decode_split_kernel<true, false><<<grid, kDecThreads, smem, st>>>(h.tm_k, h.tm_v, h.tm_k, h.tm_v, a);
  else if (h.fp8)
    decode_split_kernel<false, true><<<grid, kDecThreads, smem, st>>>(h.tm_k, h.tm_v, h.tm_ks, h.tm_vs, a);
  else
    decode_split_kernel<false, false><<<grid, kDecThreads, smem, st>>>(h.tm_k, h.tm_v, h.tm_k, h.tm_v, a);
  profile_after(st);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<h.B * kHq, 256, 0, st>>>(h.part_o, h.part_lse,
                                                   reinterpret_cast<const __nv_bfloat16*>(h.gate),
                                                   reinterpret_cast<__nv_bfloat16*>(h.out), h.n_splits);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Fixed scratch for hyb_attn_decode_noalloc.
//
// Some callers may not allocate device memory on their call path -- a plugin
// running inside a host application that owns every device allocation, or a
// latency-critical decode loop where cudaMalloc / cudaFree would stall the
// device.  For them the split partials live in this file-scope array instead
// of a caller workspace.  Every GPU that loads the library holds it (4 MiB)
// until the process exits.  All calls share it and it keeps the previous
// call's contents; nothing in it needs to start at zero, because every split
// CTA writes its partial output and log-sum-exp before the combine kernel
// reads them.  Calls whose kernels overlap on the GPU (different streams
// without ordering between them) race on it.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_decode_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked
// up with cudaGetSymbolAddress, once per device, the first time a device
// uses it (with that device current), and cached.
cudaError_t decode_noalloc_scratch(void** ptr, size_t* bytes) {
  static std::mutex mu;
  static void* addr[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  *bytes = kNoAllocScratchBytes;
  return cudaSuccess;
}

cudaError_t decode_set_smem_attr() {
  const int smem = (int)decode_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_split_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_split_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_split_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

}  // namespace hyb
