// Prefill attention on 5th-generation tensor cores (tcgen05, sm_100a).
//
// One CTA computes a 128-query tile of one query head:
//   O[t] = sum_j softmax_j(q_t . k_j / 16) v_j over the keys j that the layer
//   type lets t see, times sigmoid(gate[t, h]),
// with query head h reading KV head h / 4 (GQA, 16 / 4 heads, head_dim 256:
// "百万 Token 塞进 4B ..." §"省显存的第二板斧：GQA、融合投影与输出门控"), the
// causal mask on full layers and the 512-key band (the query and the 511
// keys before it) on sliding layers (same page, §"混合注意力").  Key tiles
// wholly outside the band are never loaded.
//
// Roles (192 threads):
//   warps 0-3  rotate the query tile (rotate-half RoPE, theta / rotary dim
//              per layer type) into tensor memory, then run the online
//              softmax row by row (one TMEM lane = one query row per thread),
//              and finally the epilogue (1/l, sigmoid gate, bf16 store);
//   warp 4     TMA producer: K and V tiles (64 keys x 256 dims, four 64x64
//              boxes with 128-byte swizzle) into a 6-slot shared-memory ring;
//   warp 5     allocates tensor memory; one lane issues all tcgen05.mma.
// Tensor memory (512 columns x 128 lanes of 32 bit):
//   [0,128)   Q as bf16 pairs (A operand of S = Q K^T)
//   [128,192) S buffer 0, [192,256) S buffer 1 (fp32 64 columns each); P of
//             a tile (bf16 pairs) overwrites the first 32 columns of its S
//             buffer and is the A operand of O += P V
//   [256,512) O accumulator, fp32 128 x 256.
// Softmax in the log2 domain with a lazily updated row maximum: the running
// maximum only moves (and O is only rescaled) when a tile's maximum exceeds
// it by more than 8, so P stays <= 256.
#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kBM = 128;
constexpr int kBN = 64;
constexpr int kSlots = 6;
constexpr int kSlotBytes = kBN * kD * 2;  // 32 KB
constexpr int kPfBox = kBN * 128;         // 8 KB: 64 keys x 64 dims
constexpr int kPfThreads = 192;
constexpr uint32_t kColQ = 0;
constexpr uint32_t kColS0 = 128;
__device__ __forceinline__ uint32_t col_s(int sb) { return sb ? 192u : kColS0; }
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;

struct PfSmem {
  uint8_t slot[kSlots][kSlotBytes];  // 1024-byte aligned
  double inv_freq[128];
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t q_ready;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t mma_done;   // every MMA issued by this CTA has completed (before TMEM is freed)
  uint32_t tmem_base;
};

size_t prefill_smem_bytes() { return sizeof(PfSmem) + 1024; }

struct PfArgs {
  const __nv_bfloat16* q;
  int64_t q_stride;
  const __nv_bfloat16* gate;
  const int32_t* pos;
  __nv_bfloat16* out;
  const int32_t* qbase;
  int ctx_mode;
  int B, T, n_mtiles;
};

// Load order shared by the producer and the MMA issuer:
//   K0, (K1, V0), (K2, V1), ..., (K_{n-1}, V_{n-2}), V_{n-1}
__device__ __forceinline__ void load_of(int i, int n, bool& is_k, int& tile) {
  if (i == 0) { is_k = true; tile = 0; return; }
  if (i == 2 * n - 1) { is_k = false; tile = n - 1; return; }
  if (i & 1) { is_k = true; tile = (i + 1) >> 1; }
  else { is_k = false; tile = (i >> 1) - 1; }
}

// Rotates 32 dims [k0, k0+32) against their partners [k0+R/2, ...) for one
// query row: x1 / x2 hold 16 packed bf16 words each; results replace them.
template <bool FULL>
__device__ __forceinline__ void rotate32(uint32_t (&x1)[16], uint32_t (&x2)[16], int k0, int p,
                                         const double* inv_freq) {
#pragma unroll
  for (int w = 0; w < 16; ++w) {
    float a[2], bb[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float x = e ? bf16hi(x1[w]) : bf16lo(x1[w]);
      const float y = e ? bf16hi(x2[w]) : bf16lo(x2[w]);
      float s, c;
      rope_sincos(p, inv_freq[k0 + 2 * w + e], &s, &c);
      a[e] = fmaf(x, c, -y * s);
      bb[e] = fmaf(y, c, x * s);
    }
    x1[w] = pack_bf16(a[0], a[1]);
    x2[w] = pack_bf16(bb[0], bb[1]);
  }
}

__device__ __forceinline__ void load_words16(const __nv_bfloat16* src, bool valid, uint32_t (&w)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 v = valid ? *reinterpret_cast<const uint4*>(src + 8 * i) : make_uint4(0, 0, 0, 0);
    w[4 * i + 0] = v.x;
    w[4 * i + 1] = v.y;
    w[4 * i + 2] = v.z;
    w[4 * i + 3] = v.w;
  }
}

template <bool FULL>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, PfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  PfSmem& sm = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int R = RopeCfg<FULL>::R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: longest query tiles first, heads of one tile adjacent ----
  const int per_tile = a.B * kHq;
  const int mt = a.n_mtiles - 1 - (int)(blockIdx.x / per_tile);
  const int rem = blockIdx.x % per_tile;
  const int h = rem % kHq;
  const int b = rem / kHq;
  const int kvh = h / kGroup;
  const int m0 = mt * kBM;
  const int qb = a.qbase ? a.qbase[b] : 0;        // sequence index of token 0
  const int kb = a.ctx_mode ? qb - (kWindow - 1) : 0;  // sequence index of key row 0
  const int rows_valid = min(kBM, a.T - m0);
  const int q_lo = qb + m0, q_hi = qb + m0 + rows_valid - 1;
  const int k_lo = FULL ? 0 : max(0, q_lo - (kWindow - 1));
  const int j_lo = (k_lo - kb) / kBN;
  const int j_hi = (q_hi - kb) / kBN;
  const int n = j_hi - j_lo + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.q_ready, kBM);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], kBM);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x < R / 2) sm.inv_freq[threadIdx.x] = rope_inv_freq(RopeCfg<FULL>::theta, threadIdx.x, R);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 4) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int i = 0; i < 2 * n; ++i) {
        bool is_k;
        int tile;
        load_of(i, n, is_k, tile);
        const int slot = i % kSlots;
        if (i >= kSlots && !mbar_wait(&sm.empty[slot], ((i / kSlots) - 1) & 1)) break;
        mbar_arrive_expect_tx(&sm.full[slot], kSlotBytes);
        const uint32_t dst = smem_u32(sm.slot[slot]);
        const int row = (j_lo + tile) * kBN;
        const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
#pragma unroll
        for (int box = 0; box < 4; ++box) tma_load_4d(dst + box * kPfBox, tm, &sm.full[slot], box * 64, row, kvh, b);
        issued = i + 1;
      }
      for (int i = max(0, issued - kSlots); i < issued; ++i) mbar_wait(&sm.full[i % kSlots], (i / kSlots) & 1);
    }
  } else if (warp == 5) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kBM, kBN, false);   // S = Q K^T, B K-major
      constexpr uint32_t idesc_o = idesc_bf16(kBM, kD, true);     // O += P V, B MN-major
      bool ok = mbar_wait(&sm.q_ready, 0);
      tc_fence_after();
      for (int i = 0; ok && i < 2 * n; ++i) {
        bool is_k;
        int tile;
        load_of(i, n, is_k, tile);
        const int slot = i % kSlots;
        if (!(ok = mbar_wait(&sm.full[slot], (i / kSlots) & 1))) break;
        tc_fence_after();
        const uint32_t saddr = smem_u32(sm.slot[slot]);
        const int sb = tile & 1;
        if (is_k) {
#pragma unroll
          for (int s = 0; s < kD / 16; ++s) {
            const uint64_t bdesc = smem_desc_sw128(saddr + (s >> 2) * kPfBox + (s & 3) * 32, 16, 1024);
            mma_ts(tmem + col_s(sb), tmem + kColQ + 8 * s, bdesc, idesc_s, s > 0 ? 1u : 0u);
          }
          mma_commit(&sm.empty[slot]);
          mma_commit(&sm.s_full[sb]);
        } else {
          if (!(ok = mbar_wait(&sm.p_full[sb], (tile >> 1) & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < kBN / 16; ++s) {
            const uint64_t bdesc = smem_desc_sw128(saddr + s * 16 * 128, kPfBox, 1024);
            mma_ts(tmem + kColO, tmem + col_s(sb) + 8 * s, bdesc, idesc_o, (tile > 0 || s > 0) ? 1u : 0u);
          }
          mma_commit(&sm.empty[slot]);
          mma_commit(&sm.o_done);
        }
      }
      // also on an early exit: wait until nothing this thread issued is in flight
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ======================= softmax / epilogue (warps 0-3) =======================
    const int r = threadIdx.x;          // query row in the tile = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const int row = m0 + r;
    const bool valid = row < a.T;
    const int qseq = qb + row;
    const int p = a.pos ? (valid ? a.pos[(int64_t)b * a.T + row] : 0) : qseq;
    const __nv_bfloat16* qrow = a.q + ((int64_t)b * a.T + (valid ? row : 0)) * a.q_stride + (int64_t)h * kD;

    // ---- rotate the query row into TMEM columns [0,128) ----
    if (FULL) {
      uint32_t x1[16], x2[16];
      load_words16(qrow, valid, x1);
      load_words16(qrow + 32, valid, x2);
      rotate32<FULL>(x1, x2, 0, p, sm.inv_freq);
      tmem_st16(trow + kColQ + 0, x1);
      tmem_st16(trow + kColQ + 16, x2);
#pragma unroll
      for (int c = 0; c < 6; ++c) {  // dims 64..255 unchanged
        uint32_t w[16];
        load_words16(qrow + 64 + 32 * c, valid, w);
        tmem_st16(trow + kColQ + 32 + 16 * c, w);
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t x1[16], x2[16];
        load_words16(qrow + 32 * c, valid, x1);
        load_words16(qrow + 128 + 32 * c, valid, x2);
        rotate32<FULL>(x1, x2, 32 * c, p, sm.inv_freq);
        tmem_st16(trow + kColQ + 16 * c, x1);
        tmem_st16(trow + kColQ + 64 + 16 * c, x2);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&sm.q_ready);

    // ---- online softmax over the key tiles ----
    const float scale_log2 = 0.0625f * 1.4426950408889634f;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (j >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      uint32_t sraw[64];
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]);
        tmem_ld32(trow + col_s(sb), lo);
        tmem_ld32(trow + col_s(sb) + 32, hi);
      }
      tmem_wait_ld();
      float s[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sraw[c]);

      const int ks0 = kb + (j_lo + j) * kBN;   // sequence index of the tile's first key
      const bool whole = ks0 >= 0 && ks0 + kBN - 1 <= q_lo && (FULL || q_hi - ks0 <= kWindow - 1);
      if (!whole) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int ks = ks0 + c;
          const bool vis = ks >= 0 && ks <= qseq && (FULL || qseq - ks <= kWindow - 1);
          if (!vis) s[c] = -INFINITY;
        }
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 64; ++c) mx = fmaxf(mx, s[c]);
      const float m_tile = mx * scale_log2;
      const float m_new = fmaxf(m_run, m_tile);
      const bool rescale = m_new > m_run + kRescaleThreshold;
      const float m_use = rescale ? m_new : m_run;
      const float base = (m_use == -INFINITY) ? 0.f : m_use;
      const float alpha = rescale ? exp2f(m_run - m_use) : 1.f;
      float sum = 0.f;
      uint32_t pw[32];
#pragma unroll
      for (int w = 0; w < 32; ++w) {
        const float p0 = exp2f(fmaf(s[2 * w], scale_log2, -base));
        const float p1 = exp2f(fmaf(s[2 * w + 1], scale_log2, -base));
        sum += p0 + p1;
        pw[w] = pack_bf16(p0, p1);
      }
      l_run = l_run * alpha + sum;
      m_run = m_use;
      tmem_st32(trow + col_s(sb), pw);
      tmem_wait_st();
      if (j > 0) {
        // O may only be touched once the previous tile's P.V has landed
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_done, (j - 1) & 1));
        if (!ok) break;
        if (__any_sync(0xffffffffu, rescale)) {
          tc_fence_after();
#pragma unroll 1
          for (int c8 = 0; c8 < 8; ++c8) {
            uint32_t ov[32];
            tmem_ld32(trow + kColO + 32 * c8, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(trow + kColO + 32 * c8, ov);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.p_full[sb]);
    }

    // ---- epilogue: O / l * sigmoid(gate) -> bf16 ----
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_done, (n - 1) & 1));
    if (ok) {
      tc_fence_after();
      float f = l_run > 0.f ? 1.f / l_run : 0.f;
      if (a.gate != nullptr && valid) {
        const float gs = __bfloat162float(a.gate[((int64_t)b * a.T + row) * kHq + h]);
        f *= 1.f / (1.f + __expf(-gs));
      }
      __nv_bfloat16* orow = a.out + (((int64_t)b * a.T + (valid ? row : 0)) * kHq + h) * kD;
#pragma unroll 1
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t ov[32];
        tmem_ld32(trow + kColO + 32 * c8, ov);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c8);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 8 * q4 + 2 * e;
              w4[e] = pack_bf16(__uint_as_float(ov[c]) * f, __uint_as_float(ov[c + 1]) * f);
            }
            dst[q4] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_prefill(bool full, const PrefillHost& h, cudaStream_t st) {
  PfArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(h.q);
  a.q_stride = h.q_stride;
  a.gate = reinterpret_cast<const __nv_bfloat16*>(h.gate);
  a.pos = h.pos;
  a.out = reinterpret_cast<__nv_bfloat16*>(h.out);
  a.qbase = h.qbase;
  a.ctx_mode = h.ctx_mode;
  a.B = h.B;
  a.T = h.T;
  a.n_mtiles = (h.T + kBM - 1) / kBM;
  const long long grid = (long long)a.n_mtiles * h.B * kHq;
  if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const size_t smem = prefill_smem_bytes();
  profile_before(st);
  if (full)
    prefill_kernel<true><<<(unsigned)grid, kPfThreads, smem, st>>>(h.tm_k, h.tm_v, a);
  else
    prefill_kernel<false><<<(unsigned)grid, kPfThreads, smem, st>>>(h.tm_k, h.tm_v, a);
  profile_after(st);
  count_launch();
  return cudaGetLastError();
}

cudaError_t prefill_set_smem_attr() {
  const int smem = (int)prefill_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

}  // namespace hyb
