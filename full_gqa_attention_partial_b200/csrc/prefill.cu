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
//   warps 0-3  rotate this CTA's query head in place in the shared-memory
//              query tile (rotate-half RoPE, theta / rotary dim per layer
//              type); then the online softmax (one TMEM lane = one query row
//              per thread) and the epilogue (1/l, sigmoid gate, bf16, TMA
//              store);
//   warp 4     lane 0: TMA producer for this CTA's halves of the K/V tiles,
//              into an 8-slot ring of 16 KB, bytes counted on CTA 0's
//              barriers; lane 1: TMA producer of the query tile;
//   warp 5     tensor-memory allocation (both CTAs); in CTA 0 the warp runs
//              the MMA loop convergently and one elected lane issues every
//              MMA of the pair and commits to both CTAs.
// S = Q K^T reads both operands from shared memory: with N = 64 an MMA whose
// A operand sits in tensor memory ran at ~40 % of the tensor rate on B200,
// one reading A from shared memory at ~90 %.
// Tensor memory, per CTA (512 columns x 128 lanes of 32 bit):
//   [0,256)   kNS S buffers (fp32, 64 keys each); P of a tile (bf16 pairs)
//             overwrites the first 32 columns of its S buffer and is the A
//             operand of O += P V
//   [256,512) O accumulator, fp32 128 x 256.
// The pair's MMAs run kNS - 1 key tiles ahead of the softmax (S of tile
// j + kNS - 1 is issued before P.V of tile j), so the time the softmax of a
// tile takes to hand P over is hidden behind tensor-core work.
// Softmax in the log2 domain with a lazily updated row maximum: the running
// maximum only moves (and O is only rescaled) when a tile's maximum exceeds
// it by more than 8, so P stays <= 256.
#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kBM = 128;                  // query rows per CTA
constexpr int kBN = 64;                   // keys per tile (shared by the pair)
constexpr int kSlots = 8;                 // K/V ring
constexpr int kSlotBytes = 16384;         // one CTA's half of a K or V tile
constexpr int kKBoxRows = kBN / 2;        // K half: 32 keys x 64 dims per box
constexpr int kKBox = kKBoxRows * 128;    // 4 KB
constexpr int kVBox = kBN * 128;          // V half: 64 keys x 64 dims per box, 8 KB
constexpr int kPfThreads = 192;
constexpr int kNS = 4;                    // S buffers in tensor memory
constexpr int kAhead = kNS - 1;           // key tiles whose S is issued before the P.V of a tile
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;
__device__ __forceinline__ uint32_t col_s(uint32_t sb) { return 64u * sb; }

struct PfSmem {
  uint8_t slot[kSlots][kSlotBytes];  // 1024-byte aligned
  uint8_t qo[4][kSlotBytes];         // the query tile in (4 boxes of 64 dims x 128 rows, rotated in place:
                                     // the A operand of S = Q K^T), the output tile out
  double inv_freq[128];
  // rotation tables for the tile's rows (positions p_base + 16 i + j):
  //   rot_lo[k / 2][j] = (cos, sin)(j * inv_freq_k), k even then odd,             j < 16
  //   rot_hi[i][k / 2] = (cos, sin)((p_base + 16 i) * inv_freq_k), k even then odd,  i < 8
  // (two frequencies per 16-byte entry: one shared-memory load per pair of them)
  float4 rot_lo[64][16];
  float4 rot_hi[8][64];
  uint8_t ostage[4][2048];           // per softmax warp: 32 rows x 32 output dims (bf16), transposed on the way out
  uint64_t full[kSlots];   // CTA 0's count both CTAs' bytes
  uint64_t empty[kSlots];  // per CTA, committed by the MMA issuer
  uint64_t q_ready;        // CTA 0: one arrival per softmax warp of the pair
  uint64_t s_full[kNS];
  uint64_t p_full[kNS];    // CTA 0: one arrival per softmax warp of the pair
  uint64_t o_done[kNS];    // P.V of a tile in S buffer i completed (two P.Vs may be in flight)
  uint64_t o_final;        // the last P.V completed
  uint64_t mma_done;       // every MMA of the pair completed
  uint64_t q_full;         // this CTA's query tile landed in qo
  uint64_t q_free;         // qo is free again (the item's last S = Q K^T completed)
  uint64_t sync_sm;        // the 128 softmax threads (bounded waits, unlike bar.sync)
  uint32_t tmem_base;
};

size_t prefill_smem_bytes() { return sizeof(PfSmem) + 1024; }
static_assert(sizeof(PfSmem) + 1024 <= 232448, "prefill shared memory exceeds 227 KB");

struct PfArgs {
  const __nv_bfloat16* q;
  int64_t q_stride;
  const __nv_bfloat16* gate;
  const int32_t* pos;
  __nv_bfloat16* out;
  const int32_t* qbase;
  int ctx_mode;
  int q_rotated;   // the queries arrive rotated (by the projection's epilogue)
  int B, T, n_mtiles;
  PageMap pm;      // K/V maps over a paged cache's pool
};

// Load order shared by the K/V producer and the MMA issuer: step s (0 <= s
// < n + kAhead) loads K_s if s < n, then V_{s - kAhead} if 0 <= s - kAhead < n.

// Rotates 32 dims [k0, k0+32) against their partners [k0+R/2, ...) for one
// query row: x1 / x2 hold 16 packed bf16 words each; results replace them.
// Pair k turns by p * inv_freq_k.  Table form, for a row at p_base + 16 i + j
// (the rows of a tile are consecutive positions): the turn is the product of
// two precomputed unit complex numbers (rot_hi for i, rot_lo for j).
// General form (any other position): the fp64-reduced full angle.
__device__ __forceinline__ void rotate32_table(uint32_t (&x1)[16], uint32_t (&x2)[16], int k0, int i_hi,
                                               int j_lo, const float4 (*rot_lo)[16], const float4 (*rot_hi)[64]) {
#pragma unroll
  for (int w = 0; w < 16; ++w) {
    const int kp = k0 / 2 + w;   // frequencies 2 kp and 2 kp + 1
    const float4 u4 = rot_hi[i_hi][kp];
    const float4 v4 = rot_lo[kp][j_lo];
    float a[2], bb[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float x = e ? bf16hi(x1[w]) : bf16lo(x1[w]);
      const float y = e ? bf16hi(x2[w]) : bf16lo(x2[w]);
      const float2 u = e ? make_float2(u4.z, u4.w) : make_float2(u4.x, u4.y);
      const float2 v = e ? make_float2(v4.z, v4.w) : make_float2(v4.x, v4.y);
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

// One work item: a 128-query tile of the two query heads (2 hp + {0, 1}) of KV
// head hp / 2 in sequence b; items are numbered longest first (the query
// tiles of the end of the sequence first), the 8 head pairs of a tile adjacent.
struct Item {
  int b, kvh, h_pair0, m0, qb, kb, q_lo, q_hi, j_lo, n;
};
template <bool FULL>
__device__ __forceinline__ Item item_of(int w, const PfArgs& a) {
  Item it;
  const int per_tile = a.B * (kHq / 2);
  const int mt = a.n_mtiles - 1 - w / per_tile;
  const int rem = w % per_tile;
  const int hp = rem % (kHq / 2);
  it.b = rem / (kHq / 2);
  it.kvh = hp >> 1;
  it.h_pair0 = it.kvh * kGroup + (hp & 1) * 2;
  it.m0 = mt * kBM;
  it.qb = a.qbase ? a.qbase[it.b] : 0;             // sequence index of token 0
  it.kb = a.ctx_mode ? it.qb - (kWindow - 1) : 0;  // sequence index of key row 0
  const int rows_valid = min(kBM, a.T - it.m0);
  it.q_lo = it.qb + it.m0;
  it.q_hi = it.qb + it.m0 + rows_valid - 1;
  const int k_lo = FULL ? 0 : max(0, it.q_lo - (kWindow - 1));
  it.j_lo = (k_lo - it.kb) / kBN;
  it.n = (it.q_hi - it.kb) / kBN - it.j_lo + 1;
  return it;
}

// Item of CTA pair `pair` in round k: the items of a round are the next
// n_pairs of the longest-first order, dealt out in alternating direction
// (pair p gets the p-th of round k when k is even, the p-th from the end
// when k is odd), which evens out the pairs' total work.  -1: none (this pair
// sits out the last, partial round); -2: past the last round.
__device__ __forceinline__ int item_index(int k, int pair, int n_pairs, int n_items) {
  const int base = k * n_pairs;
  if (base >= n_items) return -2;
  const int w = base + ((k & 1) ? n_pairs - 1 - pair : pair);
  return w < n_items ? w : -1;
}

// Persistent: each CTA pair walks its items round by round.
// Barrier phases run on across items: K/V loads by a global load counter,
// S / P buffers by a global tile counter, query / output / last-P.V barriers
// by the item counter.
template <bool FULL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o, PfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  PfSmem& sm = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int R = RopeCfg<FULL>::R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0 = the CTA that issues the pair's MMAs
  const int pair0 = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int n_items = a.n_mtiles * a.B * (kHq / 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.q_ready, 8);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 8);
    }
    for (int s = 0; s < kNS; ++s) mbar_init(&sm.o_done[s], 1);
    mbar_init(&sm.o_final, 1);
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_free, 1);
    mbar_init(&sm.sync_sm, kBM);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  // frequencies and the position-independent rotation table
  if (threadIdx.x < R / 2) sm.inv_freq[threadIdx.x] = rope_inv_freq(RopeCfg<FULL>::theta, threadIdx.x, R);
  __syncthreads();
  for (int t = threadIdx.x; t < (R / 2) * 16; t += kPfThreads) {
    const int k = t % (R / 2), e = t / (R / 2);
    float sn, cs;
    small_angle_sincos(e, (float)sm.inv_freq[k], &sn, &cs);
    reinterpret_cast<float2*>(&sm.rot_lo[k >> 1][e])[k & 1] = make_float2(cs, sn);
  }
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 4) {
    if (lane == 0) {
      // ======================= K/V producer (both CTAs) =======================
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      uint32_t g = 0;   // loads issued so far by this CTA
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int w = item_index(k, pair0, n_pairs, n_items);
        if (w == -2) break;
        if (w < 0) continue;
        const Item it = item_of<FULL>(w, a);
        for (int st = 0; ok && st < it.n + kAhead; ++st) {
#pragma unroll 1
          for (int part = 0; part < 2; ++part) {
            const bool is_k = part == 0;
            const int tile = is_k ? st : st - kAhead;
            if (tile < 0 || tile >= it.n) continue;
            const int slot = g % kSlots;
            if (g >= kSlots && !(ok = mbar_wait(&sm.empty[slot], ((g / kSlots) - 1) & 1))) break;
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[slot], 2 * kSlotBytes);
            const uint32_t dst = smem_u32(sm.slot[slot]);
            int row, cpage;   // the tile's 64 keys lie within one page
            kv_coord(a.pm, it.b, (it.j_lo + tile) * kBN, row, cpage);
            if (is_k) {
#pragma unroll
              for (int box = 0; box < 4; ++box)
                tma_load_4d_pair(dst + box * kKBox, &tm_k, &sm.full[slot], box * 64, row + kKBoxRows * (int)rank,
                                 it.kvh, cpage);
            } else {
#pragma unroll
              for (int box = 0; box < 2; ++box)
                tma_load_4d_pair(dst + box * kVBox, &tm_v, &sm.full[slot], 128 * (int)rank + 64 * box, row, it.kvh,
                                 cpage);
            }
            ++g;
          }
        }
      }
      if (rank == 0)  // every load of the pair completes on CTA 0's barriers
        for (uint32_t i = (g > kSlots ? g - kSlots : 0); i < g; ++i) mbar_wait(&sm.full[i % kSlots], (i / kSlots) & 1);
    } else if (lane == 1) {
      // ======================= query-tile producer (both CTAs) =======================
      prefetch_tmap(&tm_q);
      int item = 0;
      for (int k = 0;; ++k) {
        const int w = item_index(k, pair0, n_pairs, n_items);
        if (w == -2) break;
        if (w < 0) continue;
        const Item it = item_of<FULL>(w, a);
        if (item > 0 && !mbar_wait(&sm.q_free, (item - 1) & 1)) break;
        mbar_arrive_expect_tx(&sm.q_full, 4 * kSlotBytes);
#pragma unroll
        for (int box = 0; box < 4; ++box)
          tma_load_4d(smem_u32(sm.qo[box]), &tm_q, &sm.q_full, box * 64, it.h_pair0 + (int)rank, it.m0, it.b);
        ++item;
      }
      if (item > 0) mbar_wait(&sm.q_full, (item - 1) & 1);   // no copy left landing at exit
    }
  } else if (warp == 5) {
    // ======================= MMA issuer (CTA 0, whole warp, one lane issues) =======================
    if (rank == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(2 * kBM, kBN, false);   // S = Q K^T, B K-major
      constexpr uint32_t idesc_o = idesc_bf16(2 * kBM, kD, true);     // O += P V, B MN-major
      const uint64_t qdesc = smem_desc_sw128(smem_u32(sm.qo[0]), 16, 1024);         // Q, K-major
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(sm.slot[0]), 16, 1024);      // K in slot 0, K-major
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(sm.slot[0]), kVBox, 1024);   // V in slot 0, MN-major
      uint32_t g = 0, J = 0;
      int item = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int w = item_index(k, pair0, n_pairs, n_items);
        if (w == -2) break;
        if (w < 0) continue;
        const Item it = item_of<FULL>(w, a);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_ready, item & 1)))) break;
        tc_fence_after();
        for (int st = 0; ok && st < it.n + kAhead; ++st) {
#pragma unroll 1
          for (int part = 0; part < 2; ++part) {
            const bool is_k = part == 0;
            const int tile = is_k ? st : st - kAhead;
            if (tile < 0 || tile >= it.n) continue;
            const int slot = g % kSlots;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[slot], (g / kSlots) & 1)))) break;
            tc_fence_after();
            const uint32_t jt = J + tile;   // global tile index
            const uint32_t sb = jt % kNS;
            if (is_k) {
              const uint64_t kdesc = desc_advance(kdesc0, slot * kSlotBytes);
#pragma unroll
              for (int s = 0; s < kD / 16; ++s) {
                const uint64_t adesc = desc_advance(qdesc, (s >> 2) * kSlotBytes + (s & 3) * 32);
                const uint64_t bdesc = desc_advance(kdesc, (s >> 2) * kKBox + (s & 3) * 32);
                mma_ss_pair_warp(tmem + col_s(sb), adesc, bdesc, idesc_s, s > 0 ? 1u : 0u);
              }
              mma_commit_pair_warp(&sm.empty[slot]);
              mma_commit_pair_warp(&sm.s_full[sb]);
              if (tile == it.n - 1) mma_commit_pair_warp(&sm.q_free);   // qo is no longer read
            } else {
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.p_full[sb], (jt / kNS) & 1)))) break;
              tc_fence_after();
              const uint64_t vdesc = desc_advance(vdesc0, slot * kSlotBytes);
#pragma unroll
              for (int s = 0; s < kBN / 16; ++s) {
                const uint64_t bdesc = desc_advance(vdesc, s * 16 * 128);
                mma_ts_pair_warp(tmem + kColO, tmem + col_s(sb) + 8 * s, bdesc, idesc_o,
                                 (tile > 0 || s > 0) ? 1u : 0u);
              }
              mma_commit_pair_warp(&sm.empty[slot]);
              mma_commit_pair_warp(&sm.o_done[sb]);
              if (tile == it.n - 1) mma_commit_pair_warp(&sm.o_final);
            }
            ++g;
          }
        }
        J += it.n;
        ++item;
      }
      // also on an early exit: wait until nothing the pair issued is in flight
      mma_commit_pair_warp(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ======================= softmax / epilogue (warps 0-3) =======================
    // Per item: the online softmax over its key tiles; then the next item's
    // query tile is rotated (so the pair's MMAs for it can start), and only
    // then this item's output leaves, straight from TMEM to global memory.
    const int r = threadIdx.x;          // query row in the tile = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const float scale_log2 = 0.0625f * 1.4426950408889634f;
    // barrier among the softmax threads; each thread counts the phases it has
    // passed (none can get two phases ahead: every phase needs all arrivals)
    uint32_t n_sync = 0;
    auto sync_softmax = [&]() -> bool {
      mbar_arrive(&sm.sync_sm);
      return mbar_wait(&sm.sync_sm, (n_sync++) & 1);
    };
    // rotates the query tile of `it` (the item_no-th of this pair) in qo and
    // hands it to the MMA issuer
    auto prepare_q = [&](const Item& it, int item_no) -> bool {
      const int row = it.m0 + r;
      const bool valid = row < a.T;
      const int qseq = it.qb + row;
      const int p_base = a.pos ? a.pos[(int64_t)it.b * a.T + it.m0] : it.qb + it.m0;
      const int p = a.pos ? (valid ? a.pos[(int64_t)it.b * a.T + row] : 0) : qseq;
      const int delta = p - p_base;
      const bool in_table = __all_sync(0xffffffffu, delta >= 0 && delta < kBM);

      // ---- rotation table for this tile's base position ----
      if (!a.q_rotated) {
        for (int t = r; t < (R / 2) * 8; t += kBM) {
          const int k = t % (R / 2), e = t / (R / 2);
          float sn, cs;
          rope_sincos(p_base + 16 * e, sm.inv_freq[k], &sn, &cs);
          reinterpret_cast<float2*>(&sm.rot_hi[e][k >> 1])[k & 1] = make_float2(cs, sn);
        }
        if (!__all_sync(0xffffffffu, sync_softmax())) return false;
      }

      // ---- this row of the query tile: shared memory (128-byte swizzled boxes) -> registers ----
      uint4 qv[kD / 8];
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_full, item_no & 1))) return false;
#pragma unroll
      for (int i = 0; i < kD / 8; ++i) {
        const uint32_t off = sw128_offset((uint32_t)r, (uint32_t)(i & 7) * 16);
        qv[i] = *reinterpret_cast<const uint4*>(sm.qo[i >> 3] + off);
      }
      // ---- rotate it in place (rotated dims go back to where they were read) ----
      auto words16 = [&](int dim0, uint32_t (&wd)[16]) {   // 16 packed words = dims [dim0, dim0 + 32)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = qv[dim0 / 8 + i];
          wd[4 * i + 0] = v.x;
          wd[4 * i + 1] = v.y;
          wd[4 * i + 2] = v.z;
          wd[4 * i + 3] = v.w;
        }
      };
      auto store16 = [&](int dim0, const uint32_t (&wd)[16]) {   // inverse of words16, into qo
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int ci = dim0 / 8 + i;
          const uint32_t off = sw128_offset((uint32_t)r, (uint32_t)(ci & 7) * 16);
          *reinterpret_cast<uint4*>(sm.qo[ci >> 3] + off) = make_uint4(wd[4 * i], wd[4 * i + 1], wd[4 * i + 2], wd[4 * i + 3]);
        }
      };
      if (!a.q_rotated) {
#pragma unroll
        for (int c = 0; c < R / 64; ++c) {   // dims [R, 256) are not rotated and stay as loaded
          uint32_t x1[16], x2[16];
          words16(32 * c, x1);
          words16(R / 2 + 32 * c, x2);
          rotate32(x1, x2, 32 * c, p, delta, in_table, sm);
          store16(32 * c, x1);
          store16(R / 2 + 32 * c, x2);
        }
        fence_proxy_async();              // qo is read by the tensor core
        if (rank != 0) fence_cluster();   // ... through MMAs issued from CTA 0
      }
      tc_fence_before();                // TMEM accesses so far precede the MMAs q_ready releases
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&sm.q_ready);
        else mbar_arrive_remote(&sm.q_ready, 0);
      }
      return true;
    };
    auto next_item = [&](int& k, Item& it) -> bool {
      for (;; ++k) {
        const int w = item_index(k, pair0, n_pairs, n_items);
        if (w == -2) return false;
        if (w >= 0) {
          it = item_of<FULL>(w, a);
          ++k;
          return true;
        }
      }
    };

    uint32_t J = 0;
    int k = 0, item = 0;
    Item it;
    bool have = next_item(k, it);
    bool ok = !have || prepare_q(it, 0);
    while (ok && have) {
      const int h = it.h_pair0 + (int)rank;
      const int row = it.m0 + r;
      const bool valid = row < a.T;
      const int qseq = it.qb + row;

      // ---- online softmax over the key tiles ----
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; ok && j < it.n; ++j) {
        const uint32_t jt = J + j;
        const uint32_t sb = jt % kNS;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (jt / kNS) & 1)))) break;
        tc_fence_after();
        uint32_t sraw[64];
        tmem_ld32(trow + col_s(sb), *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]));
        tmem_ld32(trow + col_s(sb) + 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]));
        tmem_wait_ld();
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sraw[c]);

        const int ks0 = it.kb + (it.j_lo + j) * kBN;   // sequence index of the tile's first key
        const bool whole = ks0 >= 0 && ks0 + kBN - 1 <= it.q_lo && (FULL || it.q_hi - ks0 <= kWindow - 1);
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
        for (int wd = 16; wd >= 1; wd >>= 1)
#pragma unroll
          for (int c = 0; c < wd; ++c) mx[c] = fmaxf(mx[c], mx[c + wd]);
        const float m_row = mx[0];
        const float m_tile = m_row * scale_log2;
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
        for (int wd = 0; wd < 32; ++wd) {
          const float p0 = ex2(fmaf(s[2 * wd], scale_log2, -base));
          const float p1 = ex2(fmaf(s[2 * wd + 1], scale_log2, -base));
          ps[wd & 7] += p0 + p1;
          pw[wd] = pack_bf16(p0, p1);
        }
        const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        l_run = l_run * alpha + sum;
        m_run = m_use;
        tmem_st32(trow + col_s(sb), pw);
        tmem_wait_st();
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O may only be touched once the previous tile's P.V has landed
          const uint32_t jp = jt - 1;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_done[jp % kNS], (jp / kNS) & 1)))) break;
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
      J += it.n;
      if (!ok) break;
      Item nxt{};
      const bool have_next = next_item(k, nxt);
      if (have_next && !(ok = prepare_q(nxt, item + 1))) break;

      // ---- epilogue: O / l * sigmoid(gate) -> bf16 -> global ----
      // 32 dims at a time through the warp's staging area: each thread writes
      // its row (16-byte chunks XOR-swizzled by row, so neither phase has bank
      // conflicts), then each store instruction covers 8 rows x 64 bytes.
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_final, item & 1)))) break;
      tc_fence_after();
      float f = l_run > 0.f ? 1.f / l_run : 0.f;
      if (a.gate != nullptr && valid) {
        const float gs = __bfloat162float(a.gate[((int64_t)it.b * a.T + row) * kHq + h]);
        f *= 1.f / (1.f + __expf(-gs));
      }
      uint8_t* stg = sm.ostage[warp];
      const int rr = lane >> 2, ch = lane & 3;   // store phase: rows rr + 8 t, chunk ch
#pragma unroll 1
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t ov[32];
        tmem_ld32(trow + kColO + 32 * c8, ov);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 8 * q4 + 2 * e;
            w4[e] = pack_bf16(__uint_as_float(ov[c]) * f, __uint_as_float(ov[c + 1]) * f);
          }
          *reinterpret_cast<uint4*>(stg + lane * 64 + 16 * (q4 ^ ((lane >> 1) & 3))) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        __syncwarp();
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int rw = rr + 8 * t;                   // row within this warp's 32
          const int grow = it.m0 + 32 * warp + rw;     // query row in the sequence
          const uint4 v = *reinterpret_cast<const uint4*>(stg + rw * 64 + 16 * (ch ^ ((rw >> 1) & 3)));
          if (grow < a.T)
            *reinterpret_cast<uint4*>(a.out + (((int64_t)it.b * a.T + grow) * kHq + h) * kD + 32 * c8 + 8 * ch) = v;
        }
        __syncwarp();
      }
      it = nxt;
      have = have_next;
      ++item;
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
  a.pm = h.pm;
  a.q_rotated = h.q_rotated;
  a.B = h.B;
  a.T = h.T;
  a.n_mtiles = (h.T + kBM - 1) / kBM;
  const long long n_items = (long long)a.n_mtiles * h.B * (kHq / 2);   // (query tile, head pair)
  if (n_items <= 0 || n_items > 0x3fffffffLL) return cudaErrorInvalidValue;
  const long long grid = 2 * (n_items < h.n_pairs ? n_items : h.n_pairs);   // persistent CTA pairs
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
