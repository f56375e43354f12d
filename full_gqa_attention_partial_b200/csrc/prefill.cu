// Prefill attention on 5th-generation tensor cores (tcgen05, sm_100a).
//
// A cluster of two CTAs (a CTA pair) computes one 128-query tile for two
// query heads of the same KV group (GQA, 16 query / 4 KV heads, head_dim 256:
// "百万 Token 塞进 4B ..." §"省显存的第二板斧：GQA、融合投影与输出门控"):
//   O[t] = sum_j softmax_j(q_t . k_j / 16) v_j, times sigmoid(gate[t, h]),
// over the keys j the layer type lets t see: causal on full layers, the
// query and the 511 keys before it on sliding layers (same page, §"混合注意力").
// Key tiles wholly outside the band are never loaded.
//
// The pair shares every K/V tile: each CTA loads half of it (32 of the 64
// keys of a K tile, 128 of the 256 dims of a V tile) and the pair MMAs
// (cta_group::2, M = 256: 128 rows per CTA) read both halves, so each SM
// draws 32 KB from L2 per 64-key tile instead of 64 KB.
//
// Roles in each CTA (192 threads):
//   warps 0-3  rotate this CTA's query head into tensor memory (rotate-half
//              RoPE, theta / rotary dim per layer type), then the online
//              softmax (one TMEM lane = one query row per thread) and the
//              epilogue (1/l, sigmoid gate, bf16 store);
//   warp 4     TMA producer for this CTA's halves of the K/V tiles, into a
//              12-slot ring of 16 KB; bytes are counted on CTA 0's barriers;
//   warp 5     tensor-memory allocation (both CTAs); in CTA 0 the warp runs
//              the MMA loop convergently and one elected lane issues every
//              MMA of the pair and commits to both CTAs.
// Tensor memory, per CTA (512 columns x 128 lanes of 32 bit):
//   [0,128)   Q as bf16 pairs (A operand of S = Q K^T)
//   [128,192) S buffer 0, [192,256) S buffer 1 (fp32, 64 keys each); P of a
//             tile (bf16 pairs) overwrites the first 32 columns of its S
//             buffer and is the A operand of O += P V
//   [256,512) O accumulator, fp32 128 x 256.
// Softmax in the log2 domain with a lazily updated row maximum: the running
// maximum only moves (and O is only rescaled) when a tile's maximum exceeds
// it by more than 8, so P stays <= 256.
#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kBM = 128;                  // query rows per CTA
constexpr int kBN = 64;                   // keys per tile (shared by the pair)
constexpr int kSlots = 12;
constexpr int kSlotBytes = 16384;         // one CTA's half of a K or V tile
constexpr int kKBoxRows = kBN / 2;        // K half: 32 keys x 64 dims per box
constexpr int kKBox = kKBoxRows * 128;    // 4 KB
constexpr int kVBox = kBN * 128;          // V half: 64 keys x 64 dims per box, 8 KB
constexpr int kPfThreads = 192;
constexpr uint32_t kColQ = 0;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;
__device__ __forceinline__ uint32_t col_s(int sb) { return sb ? 192u : 128u; }

struct PfSmem {
  uint8_t slot[kSlots][kSlotBytes];  // 1024-byte aligned
  double inv_freq[128];
  // rotation tables for the tile's rows (positions p_base + 16 i + j):
  //   rot_lo[k][j] = (cos, sin)(j * inv_freq_k),               j < 16
  //   rot_hi[k][i] = (cos, sin)((p_base + 16 i) * inv_freq_k),  i < 8
  float2 rot_lo[128][16];
  float2 rot_hi[128][8];
  uint64_t full[kSlots];   // CTA 0's count both CTAs' bytes
  uint64_t empty[kSlots];  // per CTA, committed by the MMA issuer
  uint64_t q_ready;        // CTA 0: one arrival per softmax warp of the pair
  uint64_t s_full[2];
  uint64_t p_full[2];      // CTA 0: one arrival per softmax warp of the pair
  uint64_t o_done;         // each P.V completed
  uint64_t o_final;        // the last P.V completed
  uint64_t mma_done;       // every MMA of the pair completed
  uint64_t q_full;         // this CTA's query tile landed (ring slots 8..11)
  uint64_t q_free;         // the softmax warps have read it
  uint32_t tmem_base;
};
// The query tile (4 boxes of 64 dims x 128 rows = 64 KB) arrives in ring slots
// 8..11 before the K/V stream first reaches them; the output tile leaves
// through slots 0..3 once every MMA is done.
constexpr int kQSlot = 8;

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

// Load order shared by the producers and the MMA issuer:
//   K0, (K1, V0), (K2, V1), ..., (K_{n-1}, V_{n-2}), V_{n-1}
__device__ __forceinline__ void load_of(int i, int n, bool& is_k, int& tile) {
  if (i == 0) { is_k = true; tile = 0; return; }
  if (i == 2 * n - 1) { is_k = false; tile = n - 1; return; }
  if (i & 1) { is_k = true; tile = (i + 1) >> 1; }
  else { is_k = false; tile = (i >> 1) - 1; }
}

// Rotates 32 dims [k0, k0+32) against their partners [k0+R/2, ...) for one
// query row: x1 / x2 hold 16 packed bf16 words each; results replace them.
// Pair k turns by p * inv_freq_k.  Table form, for a row at p_base + 16 i + j
// (the rows of a tile are consecutive positions): the turn is the product of
// two precomputed unit complex numbers, rot_hi[k][i] * rot_lo[k][j].  General
// form (any other position): the fp64-reduced full angle.
__device__ __forceinline__ void rotate32_table(uint32_t (&x1)[16], uint32_t (&x2)[16], int k0, int i_hi,
                                               int j_lo, const float2 (*rot_lo)[16], const float2 (*rot_hi)[8]) {
#pragma unroll
  for (int w = 0; w < 16; ++w) {
    float a[2], bb[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int k = k0 + 2 * w + e;
      const float x = e ? bf16hi(x1[w]) : bf16lo(x1[w]);
      const float y = e ? bf16hi(x2[w]) : bf16lo(x2[w]);
      const float2 u = rot_hi[k][i_hi];
      const float2 v = rot_lo[k][j_lo];
      const float c = fmaf(u.x, v.x, -u.y * v.y);
      const float s = fmaf(u.y, v.x, u.x * v.y);
      a[e] = fmaf(x, c, -y * s);
      bb[e] = fmaf(y, c, x * s);
    }
    x1[w] = pack_bf16(a[0], a[1]);
    x2[w] = pack_bf16(bb[0], bb[1]);
  }
}
__device__ __noinline__ void rotate32_general(uint32_t (&x1)[16], uint32_t (&x2)[16], int k0, int p,
                                              const double* inv_freq) {
#pragma unroll 4
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
// in_table: warp-uniform (every row of the warp at p_base + [0, 128))
__device__ __forceinline__ void rotate32(uint32_t (&x1)[16], uint32_t (&x2)[16], int k0, int p, int delta,
                                         bool in_table, const PfSmem& sm) {
  if (in_table)
    rotate32_table(x1, x2, k0, delta >> 4, delta & 15, sm.rot_lo, sm.rot_hi);
  else
    rotate32_general(x1, x2, k0, p, sm.inv_freq);
}

template <bool FULL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o, PfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  PfSmem& sm = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int R = RopeCfg<FULL>::R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0 = the CTA that issues the pair's MMAs

  // ---- work item: longest query tiles first; the pairs of one tile adjacent ----
  const int pair = blockIdx.x >> 1;
  const int per_tile = a.B * (kHq / 2);
  const int mt = a.n_mtiles - 1 - pair / per_tile;
  const int rem = pair % per_tile;
  const int hp = rem % (kHq / 2);
  const int b = rem / (kHq / 2);
  const int kvh = hp >> 1;
  const int h = kvh * kGroup + (hp & 1) * 2 + (int)rank;
  const int m0 = mt * kBM;
  const int qb = a.qbase ? a.qbase[b] : 0;             // sequence index of token 0
  const int kb = a.ctx_mode ? qb - (kWindow - 1) : 0;  // sequence index of key row 0
  const int rows_valid = min(kBM, a.T - m0);
  const int q_lo = qb + m0, q_hi = qb + m0 + rows_valid - 1;
  const int k_lo = FULL ? 0 : max(0, q_lo - (kWindow - 1));
  const int j_lo = (k_lo - kb) / kBN;
  const int j_hi = (q_hi - kb) / kBN;
  const int n = j_hi - j_lo + 1;
  // RoPE positions (the tile's first row and this thread's row), loaded early
  // so their latency hides behind the set-up
  const int p_base = a.pos ? a.pos[(int64_t)b * a.T + m0] : qb + m0;
  int p_row = 0;
  if (warp < 4) {
    const int row = m0 + (int)threadIdx.x;
    p_row = a.pos ? (row < a.T ? a.pos[(int64_t)b * a.T + row] : 0) : qb + row;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.q_ready, 8);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 8);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.o_final, 1);
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_free, 4);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  // rotation tables: pair k = t % (R/2) of entry group t / (R/2); 24 entries per pair
  if (threadIdx.x < R / 2) sm.inv_freq[threadIdx.x] = rope_inv_freq(RopeCfg<FULL>::theta, threadIdx.x, R);
  __syncthreads();
  {
    for (int t = threadIdx.x; t < (R / 2) * 24; t += kPfThreads) {
      const int k = t % (R / 2);
      const int e = t / (R / 2);
      const double f = sm.inv_freq[k];
      float sn, cs;
      if (e < 16) {
        small_angle_sincos(e, (float)f, &sn, &cs);
        sm.rot_lo[k][e] = make_float2(cs, sn);
      } else {
        rope_sincos(p_base + 16 * (e - 16), f, &sn, &cs);
        sm.rot_hi[k][e - 16] = make_float2(cs, sn);
      }
    }
  }
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 4) {
    // ======================= TMA producer (both CTAs) =======================
    if (lane == 0) {
      // this CTA's query tile first: 4 boxes of 64 dims x 128 rows of head h
      mbar_arrive_expect_tx(&sm.q_full, 4 * kSlotBytes);
#pragma unroll
      for (int box = 0; box < 4; ++box)
        tma_load_4d(smem_u32(sm.slot[kQSlot + box]), &tm_q, &sm.q_full, box * 64, h, m0, b);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int i = 0; i < 2 * n; ++i) {
        bool is_k;
        int tile;
        load_of(i, n, is_k, tile);
        const int slot = i % kSlots;
        if (i >= kSlots && !mbar_wait(&sm.empty[slot], ((i / kSlots) - 1) & 1)) break;
        if (i == kQSlot && !mbar_wait(&sm.q_free, 0)) break;   // the query tile has been read
        if (rank == 0) mbar_arrive_expect_tx(&sm.full[slot], 2 * kSlotBytes);
        const uint32_t dst = smem_u32(sm.slot[slot]);
        const int row = (j_lo + tile) * kBN;
        if (is_k) {
#pragma unroll
          for (int box = 0; box < 4; ++box)
            tma_load_4d_pair(dst + box * kKBox, &tm_k, &sm.full[slot], box * 64, row + kKBoxRows * (int)rank, kvh, b);
        } else {
#pragma unroll
          for (int box = 0; box < 2; ++box)
            tma_load_4d_pair(dst + box * kVBox, &tm_v, &sm.full[slot], 128 * (int)rank + 64 * box, row, kvh, b);
        }
        issued = i + 1;
      }
      if (rank == 0)  // every load of the pair completes on CTA 0's barriers
        for (int i = max(0, issued - kSlots); i < issued; ++i) mbar_wait(&sm.full[i % kSlots], (i / kSlots) & 1);
    }
  } else if (warp == 5) {
    // ======================= MMA issuer (CTA 0, whole warp, one lane issues) =======================
    if (rank == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(2 * kBM, kBN, false);   // S = Q K^T, B K-major
      constexpr uint32_t idesc_o = idesc_bf16(2 * kBM, kD, true);     // O += P V, B MN-major
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_ready, 0));
      tc_fence_after();
      for (int i = 0; ok && i < 2 * n; ++i) {
        bool is_k;
        int tile;
        load_of(i, n, is_k, tile);
        const int slot = i % kSlots;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[slot], (i / kSlots) & 1)))) break;
        tc_fence_after();
        const uint32_t saddr = smem_u32(sm.slot[slot]);
        const int sb = tile & 1;
        if (is_k) {
#pragma unroll
          for (int s = 0; s < kD / 16; ++s) {
            const uint64_t bdesc = smem_desc_sw128(saddr + (s >> 2) * kKBox + (s & 3) * 32, 16, 1024);
            mma_ts_pair_warp(tmem + col_s(sb), tmem + kColQ + 8 * s, bdesc, idesc_s, s > 0 ? 1u : 0u);
          }
          mma_commit_pair_warp(&sm.empty[slot]);
          mma_commit_pair_warp(&sm.s_full[sb]);
        } else {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.p_full[sb], (tile >> 1) & 1)))) break;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < kBN / 16; ++s) {
            const uint64_t bdesc = smem_desc_sw128(saddr + s * 16 * 128, kVBox, 1024);
            mma_ts_pair_warp(tmem + kColO, tmem + col_s(sb) + 8 * s, bdesc, idesc_o, (tile > 0 || s > 0) ? 1u : 0u);
          }
          mma_commit_pair_warp(&sm.empty[slot]);
          mma_commit_pair_warp(&sm.o_done);
          if (tile == n - 1) mma_commit_pair_warp(&sm.o_final);
        }
      }
      // also on an early exit: wait until nothing the pair issued is in flight
      mma_commit_pair_warp(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ======================= softmax / epilogue (warps 0-3) =======================
    const int r = threadIdx.x;          // query row in the tile = TMEM lane
    bool ok_q = true;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const int row = m0 + r;
    const bool valid = row < a.T;
    const int qseq = qb + row;
    const int p = p_row;
    const int delta = p - p_base;
    const bool small = __all_sync(0xffffffffu, delta >= 0 && delta < kBM);

    // ---- this row of the query tile: shared memory (128-byte swizzled boxes) -> registers ----
    uint4 qv[kD / 8];
    ok_q = __all_sync(0xffffffffu, mbar_wait(&sm.q_full, 0));
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
      const uint32_t off = sw128_offset((uint32_t)r, (uint32_t)(i & 7) * 16);
      qv[i] = *reinterpret_cast<const uint4*>(sm.slot[kQSlot + (i >> 3)] + off);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.q_free);
    // ---- rotate it into TMEM columns [0,128) ----
    auto words16 = [&](int dim0, uint32_t (&w)[16]) {   // 16 packed words = dims [dim0, dim0 + 32)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = qv[dim0 / 8 + i];
        w[4 * i + 0] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
    };
    if (FULL) {
      uint32_t x1[16], x2[16];
      words16(0, x1);
      words16(32, x2);
      rotate32(x1, x2, 0, p, delta, small, sm);
      tmem_st16(trow + kColQ + 0, x1);
      tmem_st16(trow + kColQ + 16, x2);
#pragma unroll
      for (int c = 0; c < 6; ++c) {  // dims 64..255 unchanged
        uint32_t w[16];
        words16(64 + 32 * c, w);
        tmem_st16(trow + kColQ + 32 + 16 * c, w);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t x1[16], x2[16];
        words16(32 * c, x1);
        words16(128 + 32 * c, x2);
        rotate32(x1, x2, 32 * c, p, delta, small, sm);
        tmem_st16(trow + kColQ + 16 * c, x1);
        tmem_st16(trow + kColQ + 64 + 16 * c, x2);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (rank == 0) mbar_arrive(&sm.q_ready);
      else mbar_arrive_remote(&sm.q_ready, 0);
    }

    // ---- online softmax over the key tiles ----
    const float scale_log2 = 0.0625f * 1.4426950408889634f;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = ok_q;
    for (int j = 0; ok && j < n; ++j) {
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
      // row maximum: pairwise tree (short dependency chains)
      float mx[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) mx[c] = fmaxf(s[c], s[c + 32]);
#pragma unroll
      for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
        for (int c = 0; c < w; ++c) mx[c] = fmaxf(mx[c], mx[c + w]);
      const float m_tile = mx[0] * scale_log2;
      const float m_new = fmaxf(m_run, m_tile);
      const bool rescale = m_new > m_run + kRescaleThreshold;
      const float m_use = rescale ? m_new : m_run;
      const float base = (m_use == -INFINITY) ? 0.f : m_use;
      const float alpha = rescale ? ex2(m_run - m_use) : 1.f;
      uint32_t pw[32];
      float ps[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) ps[c] = 0.f;
#pragma unroll
      for (int w = 0; w < 32; ++w) {
        const float p0 = ex2(fmaf(s[2 * w], scale_log2, -base));
        const float p1 = ex2(fmaf(s[2 * w + 1], scale_log2, -base));
        ps[w & 7] += p0 + p1;
        pw[w] = pack_bf16(p0, p1);
      }
      const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      l_run = l_run * alpha + sum;
      m_run = m_use;
      tmem_st32(trow + col_s(sb), pw);
      tmem_wait_st();
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        // O may only be touched once the previous tile's P.V has landed
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_done, (j - 1) & 1));
        if (!ok) break;
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&sm.p_full[sb]);
        else mbar_arrive_remote(&sm.p_full[sb], 0);
      }
    }

    // ---- epilogue: O / l * sigmoid(gate) -> bf16 ----
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_final, 0));
    if (ok) {
      tc_fence_after();
      float f = l_run > 0.f ? 1.f / l_run : 0.f;
      if (a.gate != nullptr && valid) {
        const float gs = __bfloat162float(a.gate[((int64_t)b * a.T + row) * kHq + h]);
        f *= 1.f / (1.f + __expf(-gs));
      }
      // O / l * gate -> bf16 -> ring slots 0..3 in the 128-byte swizzled box
      // layout of the output map; then one thread stores the tile with TMA
      // (rows past T are clipped by the tensor map).
#pragma unroll 1
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t ov[32];
        tmem_ld32(trow + kColO + 32 * c8, ov);
        tmem_wait_ld();
        uint8_t* box = sm.slot[c8 >> 1];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 8 * q4 + 2 * e;
            w4[e] = pack_bf16(__uint_as_float(ov[c]) * f, __uint_as_float(ov[c + 1]) * f);
          }
          const uint32_t off = sw128_offset((uint32_t)r, (uint32_t)(((c8 & 1) * 4 + q4) * 16));
          *reinterpret_cast<uint4*>(box + off) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_proxy_async();
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (ok && r == 0) {
#pragma unroll
      for (int box = 0; box < 4; ++box) tma_store_4d(&tm_o, smem_u32(sm.slot[box]), box * 64, h, m0, b);
      tma_store_commit_and_wait();
    }
  }

  // the peer's shared memory and tensor memory stay alive until both CTAs are done
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
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
  const long long grid = (long long)a.n_mtiles * h.B * kHq;   // one CTA per (tile, head), in pairs
  if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const size_t smem = prefill_smem_bytes();
  profile_before(st);
  if (full)
    prefill_kernel<true><<<(unsigned)grid, kPfThreads, smem, st>>>(h.tm_k, h.tm_v, h.tm_q, h.tm_o, a);
  else
    prefill_kernel<false><<<(unsigned)grid, kPfThreads, smem, st>>>(h.tm_k, h.tm_v, h.tm_q, h.tm_o, a);
  profile_after(st);
  count_launch();
  return cudaGetLastError();
}

// Box rows of the K and V tensor maps this kernel expects (per-CTA halves).
int prefill_k_box_rows() { return kKBoxRows; }
int prefill_v_box_rows() { return kBN; }
int prefill_q_box_rows() { return kBM; }

cudaError_t prefill_set_smem_attr() {
  const int smem = (int)prefill_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

}  // namespace hyb
