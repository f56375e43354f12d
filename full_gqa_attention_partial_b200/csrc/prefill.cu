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
// Key tiles hold 128 keys.  The pair shares every K/V tile: each CTA loads
// half of it (64 of the 128 keys of a K tile, 128 of the 256 dims of a V
// tile) and the pair MMAs (cta_group::2, M = 256: 128 rows per CTA) read
// both halves, so each SM draws 64 KB from L2 per 128-key tile instead of
// 128 KB.  Per 128 keys the pair issues 16 MMAs for S = Q K^T (N = 128) and
// 8 for O += P V (K = 16 keys each): with 64-key tiles the MMA-issuing
// warp, at about 40 cycles per MMA and a few hundred per barrier wait, could
// not keep the tensor pipe fed.
//
// Roles in each CTA (320 threads; sliding layers 448, FP8 caches 384):
//   warps 0-7  two softmax warpgroups.  Both own the tile's 128 query rows
//              (warp w reads TMEM lanes 32 (w % 4) ..); warpgroup g takes
//              keys [64 g, 64 g + 64) of every key tile.  A row's maximum
//              over the tile is exchanged between the two warps of a lane
//              quarter through shared memory, so both decide the same
//              softmax base.  At the end of an item the two warpgroups split
//              the epilogue (1/l, sigmoid gate, bf16, half of the 256 output
//              dims each) and, on full layers given raw queries, the
//              rotation of the next item's query tile (rotate-half RoPE over
//              the first 64 dims, half of the 32 frequencies each).  Sliding
//              layers rotate all 256 dims of every query, which on the item
//              boundary cost more than the separate pass over the queries
//              the host runs first: their queries always arrive rotated;
//   warp 8     lane 0: TMA producer for this CTA's halves of the K/V tiles,
//              into a 4-slot ring of 32 KB, bytes counted on CTA 0's
//              barriers; lane 1: TMA producer of the query tile (with an L2
//              prefetch of the next item's);
//   warp 9     tensor-memory allocation (both CTAs); in CTA 0 the warp runs
//              the MMA loop convergently and one elected lane issues every
//              MMA of the pair and commits to both CTAs;
//   warps 10-13 (sliding layers) the epilogue: a sliding item is only ~5 key
//              tiles, so the softmax warps hand over the row sums and start
//              the next item while these drain the output (the softmax warps
//              fit in the 128 registers 14 warps leave);
//   warps 10-11 (FP8 caches) converters (below).
// Tensor memory, per CTA (512 columns x 128 lanes of 32 bit):
//   [0,256)   two S buffers (fp32, 128 keys each); P of a tile (bf16 pairs)
//             overwrites the first 32 columns of each warpgroup's 64 and is
//             the A operand of O += P V
//   [256,512) O accumulator, fp32 128 x 256.
// The pair's MMAs run one key tile ahead of the softmax (S of tile j + 1 is
// issued before P.V of tile j).
//
// Softmax in the log2 domain with a lazily updated base: every probability
// of a row is 2^(s - base), the base only moves (and O is only rescaled)
// when a tile's maximum exceeds it by more than 8, so P stays <= 256.
//
// FP8 (e4m3) full-layer caches (one fp32 scale per key row and KV head) are
// read in place.  S = Q K^T runs on the tensor cores' e4m3 path
// (kind::f8f6f4) straight from the K codes, which TMA loads into a ring of 16 KB
// entries: the query tile is split into two e4m3 tiles, Q_hi (each element
// rounded, after a power-of-two factor per row that puts the row's largest
// element in [128, 256)) and Q_lo (the remainder, rounded), and S is their
// two MMA passes into one accumulator -- the tensor time of one bf16 pass.  A
// bf16 element has 8 significant bits and each part 4, so the split gives back
// every element of at least 2^-9 of its row's largest exactly and the rest
// within 2^-17 of the largest (a single e4m3 query tile would not meet the
// accuracy bound).  V feeds O += P V in bf16: its
// codes land in the upper half of one of the 32 KB V slots and two converter
// warps (12 warps in all) widen them in place by integer bit moves (value x
// 2^-120, exact; three instructions for two codes).  The row scales never touch the operands: TMA
// loads them into a four-tile ring, the softmax multiplies the scores by the
// K scale and P by the V scale, the query row's factor and the softmax scale
// come in with the row maximum and the exponent, P carries 2^64 (added in the
// exponent's FMA, so O stays far from fp32's subnormals) and the epilogue
// takes back 2^120.
#include <algorithm>
#include <cstddef>

#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kBM = 128;                  // query rows per CTA
constexpr int kBN = 128;                  // keys per tile (shared by the pair)
constexpr int kHalfKeys = 64;             // keys per TMA box row range (a K half, a V quarter)
constexpr int kSlotBytes = 32768;         // one CTA's half of a K or V tile (bf16)
constexpr int kKBox = kHalfKeys * 128;    // K half: 64 keys x 64 dims per box, 8 KB
constexpr int kVChunk = kBN * 128;        // V: 128 keys x 64 dims (two 64-key boxes), 16 KB
constexpr int kSmWarps = 8;               // softmax warps (two warpgroups)
constexpr int kProdWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvWarp = 10;             // FP8: converter warps 10 and 11
constexpr int kSlots = 4;                 // operand ring: 4 x 32 KB
constexpr int kCodeBytes = 16384;         // FP8: one CTA's codes of a K or V tile
constexpr int kNKc = 2;                   // FP8: K code entries (16 KB, two per slot) in the first slots
constexpr int kVSlot0 = kNKc / 2;         // FP8: the V slots follow them ...
constexpr int kNV = kSlots - kVSlot0;     // ... codes land in a V slot's upper half
constexpr int kNF = 4;                    // FP8: K / V row-scale ring (tiles)
constexpr int kEpiWarp0 = 10;             // sliding layers: epilogue warps 10-13
template <bool FULL, bool FP8> struct PfCfg {
  // sliding layers: four warps of their own take each item's epilogue, so the
  // softmax warps start the next item at once (an item is only ~5 key tiles)
  static constexpr bool kEpi = !FULL && !FP8;
  static constexpr int kThreads = FP8 ? 384 : (kEpi ? 448 : 320);
};
constexpr float kTwo120 = 1.329227995784916e36f;    // 2^120
constexpr int kNS = 2;                    // S buffers in tensor memory
constexpr int kAhead = kNS - 1;           // key tiles whose S is issued before the P.V of a tile
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kStageBytes = 2048;         // epilogue transpose area per softmax warp
__device__ __forceinline__ uint32_t col_s(uint32_t sb) { return 128u * sb; }

template <bool FULL, bool FP8>
struct PfSmem {
  static constexpr int R = RopeCfg<FULL>::R;
  // 1024-byte aligned; FP8: the first kVSlot0 slots hold the 16 KB K code entries, the rest the V tiles
  uint8_t slot[kSlots][kSlotBytes];
  uint8_t qo[4][16384];              // the query tile (4 boxes of 64 dims x 128 rows), rotated in place:
                                     // the A operand of S = Q K^T
  // full layers: rotation tables for the tile's rows (positions p_base + 16 i + j), rebuilt per item:
  //   rot_lo[k / 2][j] = (cos, sin)(j * inv_freq_k), k even then odd,             j < 16
  //   rot_hi[i][k / 2] = (cos, sin)((p_base + 16 i) * inv_freq_k), k even then odd,  i < 8
  // (two frequencies per 16-byte entry); warpgroup g owns the entries of its
  // half of the frequencies
  float4 rot_lo[FULL ? R / 4 : 1][16];
  float4 rot_hi[8][FULL ? R / 4 : 1];
  // epilogue staging per softmax warp, the source of its TMA stores (64-byte swizzle: 512-byte periods)
  alignas(1024) uint8_t ostage[kSmWarps][kStageBytes];
  double inv_freq[R / 2];
  float xmax[2][2][kBM];             // [tile parity][warpgroup][row]: a row's maximum over the warpgroup's keys
  float xsum[2][2][kBM];             // [item parity][warpgroup][row]: running sum at item end
  // FP8: the row scales of a tile's 128 keys, by tile % kNF
  alignas(16) float kf[FP8 ? kNF : 1][kBN];
  alignas(16) float vf[FP8 ? kNF : 1][kBN];
  uint64_t f_full[kNF];              // FP8: a tile's scales landed (this CTA's copy)
  uint64_t f_free[kNF];              // FP8: a tile's scales read by every softmax warp
  uint64_t vcode[kNV];               // FP8: this CTA's V codes of a tile landed in its slot
  uint64_t vready[kNV];              // FP8, CTA 0: V widened (one arrival per converter warp of the pair)
  uint64_t vempty[kNV];              // FP8: the V slot's P.V completed
  uint64_t qx_full[4];               // FP8: a query row's largest |element| over each warpgroup's
                                     //   dims (in xsum[item parity]) of lane quarter q written by both warps
  uint64_t full[kSlots];   // CTA 0's count both CTAs' bytes (bf16 slots; FP8 K code entries)
  uint64_t empty[kSlots];  // per CTA, committed by the MMA issuer
  uint64_t q_ready;        // CTA 0: query tile rotated (one arrival per softmax warp of the pair) or
                           //   landed (one arrival per CTA from its query producer)
  uint64_t s_full[kNS];
  uint64_t p_full[kNS];    // CTA 0: one arrival per softmax warp of the pair
  uint64_t o_done[kNS];    // P.V of a tile in S buffer i completed
  uint64_t o_final;        // the item's last P.V completed
  uint64_t o_free;         // CTA 0: every softmax warp of the pair has read O out (epilogue done)
  uint64_t mma_done;       // every MMA of the pair completed
  uint64_t q_full;         // this CTA's query tile landed in qo
  uint64_t q_free;         // qo is free again (the item's last S = Q K^T completed)
  uint64_t xmax_full[2][4];  // xmax[parity] of lane quarter q written by both of its warps
  uint64_t xsum_full;      // both warpgroups' xsum written (one arrival per softmax warp)
  uint64_t sync_wg[2];     // the 128 threads of a warpgroup (bounded waits, unlike bar.sync)
  uint32_t tmem_base;
};

template <bool FULL, bool FP8 = false>
size_t prefill_smem_bytes_t() { return sizeof(PfSmem<FULL, FP8>) + 1024; }
size_t prefill_smem_bytes() {
  return std::max({prefill_smem_bytes_t<true>(), prefill_smem_bytes_t<false>(), prefill_smem_bytes_t<true, true>()});
}
static_assert(sizeof(PfSmem<true, false>) + 1024 <= 232448 && sizeof(PfSmem<false, false>) + 1024 <= 232448 &&
                  sizeof(PfSmem<true, true>) + 1024 <= 232448,
              "prefill shared memory exceeds 227 KB");
using PfSmemFull = PfSmem<true, false>;
using PfSmemSliding = PfSmem<false, false>;
using PfSmemFullFp8 = PfSmem<true, true>;
static_assert(offsetof(PfSmemFull, ostage) % 1024 == 0 && offsetof(PfSmemSliding, ostage) % 1024 == 0 &&
                  offsetof(PfSmemFullFp8, ostage) % 1024 == 0,
              "staging areas must start on a swizzle period");

struct PfArgs {
  const __nv_bfloat16* q;
  int64_t q_stride;
  const __nv_bfloat16* gate;
  const int32_t* pos;
  __nv_bfloat16* out;
  const int32_t* qbase;
  int ctx_mode;
  int q_rotated;   // the queries arrive rotated (by the projection's epilogue or a rotation pass)
  int B, T, n_mtiles;
  PageMap pm;      // K/V maps over a paged cache's pool
};

// ---------------------------------------------------------------------------
// Packed fp32 pairs (sm_100 f32x2 instructions): one issue slot for two lanes
// of arithmetic.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Load order shared by the K/V producer and the MMA issuer, item by item: K of
// tile t + 1 before V of tile t (S of the next tile is issued before P.V of
// this one), the item's last V last.  (Taking the next item's first K before
// the current item's last V was measured slower on sliding layers: the last
// P.V then waits for the next query tile's load, and the epilogue with it.)

// Rotates 2 NW dims [k0, k0 + 2 NW) against their partners [k0 + R/2, ...)
// for one query row: x1 / x2 hold NW packed bf16 words each; results replace
// them.  Pair k turns by p * inv_freq_k.  Table form, for a row at p_base +
// 16 i + j (the rows of a tile are consecutive positions): the turn is the
// product of two precomputed unit complex numbers (rot_hi for i, rot_lo for
// j).  General form (any other position): the fp64-reduced full angle.
template <int NW, int NKP>
__device__ __forceinline__ void rotate_table(uint32_t (&x1)[NW], uint32_t (&x2)[NW], int k0, int i_hi, int j_lo,
                                             const float4 (*rot_lo)[16], const float4 (*rot_hi)[NKP]) {
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int kp = k0 / 2 + w;   // frequencies 2 kp and 2 kp + 1
    const float4 u4 = rot_hi[i_hi][kp];
    const float4 v4 = rot_lo[kp][j_lo];
    // (c, s) of both frequencies as products of the two unit complex numbers
    const float2 ux = make_float2(u4.x, u4.z), uy = make_float2(u4.y, u4.w);
    const float2 vx = make_float2(v4.x, v4.z), vy = make_float2(v4.y, v4.w);
    const float2 uyvy = fmul2(uy, vy), uxvy = fmul2(ux, vy);
    const float2 c = ffma2(ux, vx, make_float2(-uyvy.x, -uyvy.y));
    const float2 s = ffma2(uy, vx, uxvy);
    const float2 x = make_float2(bf16lo(x1[w]), bf16hi(x1[w]));
    const float2 y = make_float2(bf16lo(x2[w]), bf16hi(x2[w]));
    const float2 ys = fmul2(y, s), xs = fmul2(x, s);
    const float2 a = ffma2(x, c, make_float2(-ys.x, -ys.y));
    const float2 bb = ffma2(y, c, xs);
    x1[w] = pack_bf16(a.x, a.y);
    x2[w] = pack_bf16(bb.x, bb.y);
  }
}
template <int NW>
__device__ __noinline__ void rotate_general(uint32_t (&x1)[NW], uint32_t (&x2)[NW], int k0, int p,
                                            const double* inv_freq) {
#pragma unroll 4
  for (int w = 0; w < NW; ++w) {
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
// S / P buffers and the maximum exchange by a global tile counter, query /
// output / sum-exchange barriers by the item counter.
// Warps are dealt round-robin to the SM's four sub-partitions (16,384
// registers each): with 10 (12 for FP8) warps a sub-partition holds three,
// so a thread may use at most 168 registers.
template <bool FULL, bool FP8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PfCfg<FULL, FP8>::kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs, PfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  using Smem = PfSmem<FULL, FP8>;
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    if (FP8) {
      for (int p = 0; p < kNV; ++p) {
        mbar_init(&sm.vcode[p], 1);
        mbar_init(&sm.vready[p], 4);
        mbar_init(&sm.vempty[p], 1);
      }
      for (int p = 0; p < kNF; ++p) {
        mbar_init(&sm.f_full[p], 1);
        mbar_init(&sm.f_free[p], kSmWarps);
      }
      for (int q = 0; q < 4; ++q) mbar_init(&sm.qx_full[q], 2);
    }
    mbar_init(&sm.q_ready, (a.q_rotated && !FP8) ? 2 : 2 * kSmWarps);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 2 * kSmWarps);
      mbar_init(&sm.o_done[s], 1);
    }
    mbar_init(&sm.o_final, 1);
    mbar_init(&sm.o_free, 2 * (PfCfg<FULL, FP8>::kEpi ? 4 : kSmWarps));
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_free, 1);
    for (int p = 0; p < 2; ++p)
      for (int q = 0; q < 4; ++q) mbar_init(&sm.xmax_full[p][q], 2);
    mbar_init(&sm.xsum_full, kSmWarps);
    mbar_init(&sm.sync_wg[0], 128);
    mbar_init(&sm.sync_wg[1], 128);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  if (threadIdx.x < R / 2) sm.inv_freq[threadIdx.x] = rope_inv_freq<FULL>(threadIdx.x);
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kProdWarp) {
    if (lane == 0) {
      // ======================= K/V producer (both CTAs) =======================
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      if (FP8) {
        prefetch_tmap(&tm_ks);
        prefetch_tmap(&tm_vs);
      }
      uint32_t g = 0;   // loads issued so far by this CTA (bf16)
      uint32_t nk = 0, nf = 0, nv = 0;   // FP8: K code, scale and V loads issued (tile index + 1)
      bool ok = true;
      // One load: K (is_k) or V of key tile `tile` of item `it`, whose first tile has the
      // global index Jb.
      auto load = [&](const Item& it, uint32_t Jb, int tile, bool is_k) -> bool {
        const int last_row = it.q_hi - it.kb;   // key row of the item's last visible key
        // (row, page) coordinates of the 64 keys from key row r on; a range past the
        // item's last key is read from an out-of-range page (zeros) instead of
        // touching a block-table entry the sequence may not have
        auto coord = [&](int r, int& row, int& page) {
          if (r > last_row) {
            row = 0;
            page = -1;
          } else {
            kv_coord(a.pm, it.b, r, row, page);
          }
        };
        const int r0 = (it.j_lo + tile) * kBN;   // key row of the tile's first key
        int row, page;
        if constexpr (FP8) {
          const uint32_t jt = Jb + tile;
          if (is_k) {
            // this CTA's 64 keys (codes, dims [0, 128) and [128, 256)) into K entry
            // jt % 4, bytes counted on CTA 0's barrier; then the row scales of all
            // 128 keys (every softmax row needs them) into this CTA's scale ring
            const int e = jt % kNKc;
            if (jt >= kNKc && !(ok = mbar_wait(&sm.empty[e], ((jt / kNKc) - 1) & 1))) return false;
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[e], 2 * kCodeBytes);
            const uint32_t dst = smem_u32(sm.slot[0]) + e * kCodeBytes;
            coord(r0 + kHalfKeys * (int)rank, row, page);
#pragma unroll
            for (int c = 0; c < 2; ++c) tma_load_4d_pair(dst + c * 8192, &tm_k, &sm.full[e], 128 * c, row, it.kvh, page);
            nk = jt + 1;
            const int fe = jt % kNF;
            if (jt >= kNF && !(ok = mbar_wait(&sm.f_free[fe], ((jt / kNF) - 1) & 1))) return false;
            mbar_arrive_expect_tx(&sm.f_full[fe], 2 * kBN * 4);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              coord(r0 + kHalfKeys * h, row, page);
              tma_load_3d(smem_u32(&sm.kf[fe][kHalfKeys * h]), &tm_ks, &sm.f_full[fe], row, it.kvh, page);
              tma_load_3d(smem_u32(&sm.vf[fe][kHalfKeys * h]), &tm_vs, &sm.f_full[fe], row, it.kvh, page);
            }
            nf = jt + 1;
          } else {
            // the tile's 128 keys of this CTA's 128 dims (codes) into the upper half of
            // V slot jt % 2, once the slot's last P.V has completed
            const int v = jt % kNV;
            if (jt >= kNV && !(ok = mbar_wait(&sm.vempty[v], ((jt / kNV) - 1) & 1))) return false;
            mbar_arrive_expect_tx(&sm.vcode[v], kCodeBytes);
            const uint32_t dst = smem_u32(sm.slot[kVSlot0 + v]) + kCodeBytes;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              coord(r0 + kHalfKeys * h, row, page);
              tma_load_4d(dst + h * 8192, &tm_v, &sm.vcode[v], 128 * (int)rank, row, it.kvh, page);
            }
            nv = jt + 1;
          }
          return true;
        }
        const int slot = g % kSlots;
        if (g >= kSlots && !(ok = mbar_wait(&sm.empty[slot], ((g / kSlots) - 1) & 1))) return false;
        if (rank == 0) mbar_arrive_expect_tx(&sm.full[slot], 2 * kSlotBytes);
        const uint32_t dst = smem_u32(sm.slot[slot]);
        if (is_k) {   // this CTA's 64 keys, 4 boxes of 64 dims
          coord(r0 + kHalfKeys * (int)rank, row, page);
#pragma unroll
          for (int box = 0; box < 4; ++box)
            tma_load_4d_pair(dst + box * kKBox, &tm_k, &sm.full[slot], box * 64, row, it.kvh, page);
        } else {      // all 128 keys of this CTA's 128 dims: 2 dim chunks x 2 key halves
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            coord(r0 + kHalfKeys * h, row, page);
#pragma unroll
            for (int d = 0; d < 2; ++d)
              tma_load_4d_pair(dst + d * kVChunk + h * kKBox, &tm_v, &sm.full[slot], 128 * (int)rank + 64 * d,
                               row, it.kvh, page);
          }
        }
        ++g;
        return true;
      };
      // in the order the MMA issuer consumes the loads
      uint32_t J = 0;   // tiles of earlier items
      for (int k = 0; ok; ++k) {
        const int w = item_index(k, pair0, n_pairs, n_items);
        if (w == -2) break;
        if (w < 0) continue;
        const Item it = item_of<FULL>(w, a);
        for (int t = 0; ok && t < it.n; ++t) {
          if (!(ok = load(it, J, t, true))) break;
          if (t > 0) ok = load(it, J, t - 1, false);
        }
        if (ok) ok = load(it, J, it.n - 1, false);
        J += it.n;
      }
      // no copy left landing in shared memory at exit (the pair's loads complete on
      // CTA 0's barriers)
      if constexpr (FP8) {
        for (uint32_t i = (nv > kNV ? nv - kNV : 0); i < nv; ++i) mbar_wait(&sm.vcode[i % kNV], (i / kNV) & 1);
        for (uint32_t i = (nf > kNF ? nf - kNF : 0); i < nf; ++i) mbar_wait(&sm.f_full[i % kNF], (i / kNF) & 1);
        if (rank == 0)
          for (uint32_t i = (nk > kNKc ? nk - kNKc : 0); i < nk; ++i) mbar_wait(&sm.full[i % kNKc], (i / kNKc) & 1);
      } else if (rank == 0) {
        for (uint32_t i = (g > kSlots ? g - kSlots : 0); i < g; ++i) mbar_wait(&sm.full[i % kSlots], (i / kSlots) & 1);
      }
    } else if (lane == 1) {
      // ======================= query-tile producer (both CTAs) =======================
      prefetch_tmap(&tm_q);
      int item = 0;
      bool ok = true;
      for (int k = 0; ok;) {
        int w = item_index(k, pair0, n_pairs, n_items);
        while (w == -1) w = item_index(++k, pair0, n_pairs, n_items);
        if (w == -2) break;
        const Item it = item_of<FULL>(w, a);
        if (item > 0 && !(ok = mbar_wait(&sm.q_free, (item - 1) & 1))) break;
        mbar_arrive_expect_tx(&sm.q_full, 4 * 16384);
#pragma unroll
        for (int box = 0; box < 4; ++box)
          tma_load_4d(smem_u32(sm.qo[box]), &tm_q, &sm.q_full, box * 64, it.h_pair0 + (int)rank, it.m0, it.b);
        // the next item's query tile into L2 while this one is in use
        int k2 = k + 1, w2 = item_index(k2, pair0, n_pairs, n_items);
        while (w2 == -1) w2 = item_index(++k2, pair0, n_pairs, n_items);
        if (w2 >= 0) {
          const Item nx = item_of<FULL>(w2, a);
#pragma unroll
          for (int box = 0; box < 4; ++box) tma_prefetch_l2_4d(&tm_q, box * 64, nx.h_pair0 + (int)rank, nx.m0, nx.b);
        }
        if (a.q_rotated && !FP8) {   // nothing to rotate or permute: the tile is ready once it has landed
          if (!(ok = mbar_wait(&sm.q_full, item & 1))) break;
          if (rank == 0) mbar_arrive(&sm.q_ready);
          else mbar_arrive_remote(&sm.q_ready, 0);
        }
        ++item;
        k = k2;
      }
      if (item > 0) mbar_wait(&sm.q_full, (item - 1) & 1);   // no copy left landing at exit
    }
  } else if (FP8 && warp >= kConvWarp) {
    // ======================= FP8 converters (warps 10, 11; both CTAs) =======================
    // V codes -> bf16 in place, tile by tile: the 128 keys x 128 codes of this
    // CTA's dims sit in the upper half of the V slot (two 64-key boxes, 128-byte
    // swizzle) and become the two 16 KB chunks of 64 dims x 128 keys the P.V
    // MMAs read.  One item is 16 codes (16 dims) of one key: the 8 lanes of a
    // quarter-warp read one 128-byte row (conflict-free under the swizzle) and
    // write its 16 bf16 dims as two 16-byte chunks, lanes 4-7 in the other order
    // so that the 8 lanes' chunks fall in 8 bank groups.  A thread's output in
    // the upper half (dims 64-127) lands on the code row it read from, which
    // only lanes of its own warp read, at the same item: each warp reads a
    // group of four items, then writes them, with no wait on the other warp
    // (four at a time keeps the loop small next to the softmax warps' code in
    // the instruction cache).
    const int ct = (warp - kConvWarp) * 32 + lane;   // 0..63
    // item i of this thread: key 4 i + rq of source box sb, 16 codes q; (4 i) & 7
    // alternates between 0 and 4, so the swizzled chunk indexes take two values
    const int q = ct & 7, sb = (ct >> 3) & 1, rq = ct >> 4;
    const int sx0 = (q ^ rq) << 4, sx1 = (q ^ (rq + 4)) << 4;
    const int c0 = 2 * (q & 3);
    // lanes 4-7 of a quarter-warp store their two chunks in the other order
    const int ca = (q < 4) ? c0 : c0 + 1, cb = (q < 4) ? c0 + 1 : c0;
    const int da0 = (ca ^ rq) << 4, db0 = (cb ^ rq) << 4, da1 = (ca ^ (rq + 4)) << 4, db1 = (cb ^ (rq + 4)) << 4;
    uint32_t J = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int w = item_index(k, pair0, n_pairs, n_items);
      if (w == -2) break;
      if (w < 0) continue;
      const Item it = item_of<FULL>(w, a);
      for (int tile = 0; ok && tile < it.n; ++tile) {
        const uint32_t jt = J + tile;
        const int v = jt % kNV;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.vcode[v], (jt / kNV) & 1)))) break;
        uint8_t* dst = sm.slot[kVSlot0 + v];
        const uint8_t* sp = dst + kCodeBytes + sb * 8192 + rq * 128;
        // 64-dim chunk q / 4, key 64 sb + 4 i + rq
        uint8_t* dp = dst + (q >> 2) * 16384 + (64 * sb + rq) * 128;
#pragma unroll 1
        for (int i0 = 0; i0 < 16; i0 += 4) {
        uint4 cw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) cw[i] = *reinterpret_cast<const uint4*>(sp + (i0 + i) * 512 + ((i & 1) ? sx1 : sx0));
        __syncwarp();   // the group's codes read by every lane before any lane overwrites them
#pragma unroll
        for (int i1 = 0; i1 < 4; ++i1) {
          const int i = i0 + i1;
          const uint32_t wv[4] = {cw[i1].x, cw[i1].y, cw[i1].z, cw[i1].w};
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            o[2 * j] = e4m3_b01_bf16x2(wv[j]);
            o[2 * j + 1] = e4m3_b23_bf16x2(wv[j]);
          }
          const uint4 lo = make_uint4(o[0], o[1], o[2], o[3]), hi = make_uint4(o[4], o[5], o[6], o[7]);
          const uint4 va = (q < 4) ? lo : hi, vb = (q < 4) ? hi : lo;
          uint8_t* rowp = dp + i * 512;
          *reinterpret_cast<uint4*>(rowp + ((i & 1) ? da1 : da0)) = va;
          *reinterpret_cast<uint4*>(rowp + ((i & 1) ? db1 : db0)) = vb;
        }
        }
        fence_proxy_async();              // the slot is read by the tensor core
        if (rank != 0) fence_cluster();   // ... through MMAs issued from CTA 0
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(&sm.vready[v]);
          else mbar_arrive_remote(&sm.vready[v], 0);
        }
      }
      J += it.n;
    }
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer (CTA 0, whole warp, one lane issues) =======================
    if (rank == 0) {
      // S = Q K^T, B K-major (FP8 caches: e4m3 operands, kind::f8f6f4)
      constexpr uint32_t idesc_s = FP8 ? idesc_e4m3(2 * kBM, kBN, false) : idesc_bf16(2 * kBM, kBN, false);
      constexpr uint32_t idesc_o = idesc_bf16(2 * kBM, kD, true);     // O += P V, B MN-major
      const uint64_t qdesc = smem_desc_sw128(smem_u32(sm.qo[0]), 16, 1024);          // Q, K-major
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(sm.slot[0]), 16, 1024);       // K in slot 0, K-major
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(sm.slot[0]), kVChunk, 1024);  // V in slot 0, MN-major
      uint32_t g = 0;
      bool ok = true;
      // One operation: S = Q K^T (is_k) or O += P V of key tile `tile` of item `it`
      // (the pair's ino-th item, whose first tile has the global index Jb).
      auto issue = [&](const Item& it, int ino, uint32_t Jb, int tile, bool is_k) -> bool {
        if (is_k && tile == 0) {   // the item's query tile is ready
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_ready, ino & 1))) return false;
          tc_fence_after();
        }
        const uint32_t jt = Jb + tile;   // global tile index
        const uint32_t sb = jt % kNS;
        // the operand's slot: bf16, the load ring; FP8, K entry jt % 4 or V slot 2 + jt % 2
        const int slot = !FP8 ? (int)(g % kSlots) : is_k ? (int)(jt % kNKc) : kVSlot0 + (int)(jt % kNV);
        if (FP8 && !is_k) {
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.vready[slot - kVSlot0], (jt / kNV) & 1))) return false;
        } else {
          const uint32_t ph = FP8 ? (jt / kNKc) & 1 : (g / kSlots) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[slot], ph))) return false;
        }
        tc_fence_after();
        if (is_k) {
          if constexpr (FP8) {
            // Q_hi K^T then Q_lo K^T into the same accumulator: 32 dims per MMA; the
            // 128 dims of dim block d are Q_hi in qo[2 d], Q_lo in qo[2 d + 1], and
            // codes [128 d, 128 d + 128) of the K entry's 64 keys in its box d
            const uint64_t kdesc = desc_advance(kdesc0, slot * kCodeBytes);
#pragma unroll
            for (int s = 0; s < 2 * kD / 32; ++s) {
              const int s2 = s & 7;
              const uint64_t adesc = desc_advance(qdesc, (s2 >> 2) * 32768 + (s >> 3) * 16384 + (s2 & 3) * 32);
              const uint64_t bdesc = desc_advance(kdesc, (s2 >> 2) * 8192 + (s2 & 3) * 32);
              mma_ss_pair_e4m3_warp(tmem + col_s(sb), adesc, bdesc, idesc_s, s > 0 ? 1u : 0u);
            }
          } else {
            const uint64_t kdesc = desc_advance(kdesc0, slot * kSlotBytes);
#pragma unroll
            for (int s = 0; s < kD / 16; ++s) {
              const uint64_t adesc = desc_advance(qdesc, (s >> 2) * 16384 + (s & 3) * 32);
              const uint64_t bdesc = desc_advance(kdesc, (s >> 2) * kKBox + (s & 3) * 32);
              mma_ss_pair_warp(tmem + col_s(sb), adesc, bdesc, idesc_s, s > 0 ? 1u : 0u);
            }
          }
          mma_commit_pair_warp(&sm.empty[slot]);
          mma_commit_pair_warp(&sm.s_full[sb]);
          if (tile == it.n - 1) mma_commit_pair_warp(&sm.q_free);   // qo is no longer read
        } else {
          // the item's first P.V overwrites O: the previous item's epilogue must have read it
          if (tile == 0 && ino > 0 &&
              !__all_sync(0xffffffffu, mbar_wait(&sm.o_free, (ino - 1) & 1)))
            return false;
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.p_full[sb], (jt / kNS) & 1))) return false;
          tc_fence_after();
          const uint64_t vdesc = desc_advance(vdesc0, slot * kSlotBytes);
#pragma unroll
          for (int s = 0; s < kBN / 16; ++s) {
            // keys [16 s, 16 s + 16): P of warpgroup s / 4 at its columns 64 (s / 4) + 8 (s % 4)
            const uint64_t bdesc = desc_advance(vdesc, s * 16 * 128);
            mma_ts_pair_warp(tmem + kColO, tmem + col_s(sb) + 64 * (s >> 2) + 8 * (s & 3), bdesc, idesc_o,
                             (tile > 0 || s > 0) ? 1u : 0u);
          }
          mma_commit_pair_warp(FP8 ? &sm.vempty[slot - kVSlot0] : &sm.empty[slot]);
          mma_commit_pair_warp(&sm.o_done[sb]);
          if (tile == it.n - 1) mma_commit_pair_warp(&sm.o_final);
        }
        ++g;
        return true;
      };
      // in the producer's load order
      uint32_t J = 0;
      int item = 0;
      for (int k = 0; ok; ++k) {
        const int w = item_index(k, pair0, n_pairs, n_items);
        if (w == -2) break;
        if (w < 0) continue;
        const Item it = item_of<FULL>(w, a);
        for (int t = 0; ok && t < it.n; ++t) {
          if (!(ok = issue(it, item, J, t, true))) break;
          if (t > 0) ok = issue(it, item, J, t - 1, false);
        }
        if (ok) ok = issue(it, item, J, it.n - 1, false);
        J += it.n;
        ++item;
      }
      // also on an early exit: wait until nothing the pair issued is in flight
      mma_commit_pair_warp(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else if (PfCfg<FULL, FP8>::kEpi && warp >= kEpiWarp0) {
    // ======================= epilogue warps (sliding layers: warps 10-13, both CTAs) =======================
    // Warp w reads TMEM lanes 32 (w % 4) ..: O / l * sigmoid(gate) -> bf16 ->
    // global for its 32 rows, all 256 dims, 32 dims at a time through its
    // staging area (64-byte swizzle) and a TMA store, then frees O for the
    // next item's first P.V.  l is the sum of both softmax warpgroups' sums.
    // Items in the same order as the other roles; xsum and o_final of an item
    // cannot advance again before this warp has freed O (the next item's
    // first P.V waits for it, and every later tile of the pair after that).
    const int qtr = warp & 3;
    const int r = qtr * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(qtr * 32) << 16);
    uint8_t* const stg = sm.ostage[warp - kEpiWarp0];
    int item = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int w = item_index(k, pair0, n_pairs, n_items);
      if (w == -2) break;
      if (w < 0) continue;
      const Item it = item_of<FULL>(w, a);
      const int h = it.h_pair0 + (int)rank;
      const int row = it.m0 + r;
      const int64_t gidx = ((int64_t)it.b * a.T + row) * kHq + h;
      const float gscore = (a.gate != nullptr && row < a.T && HYB_BOUNDS(gidx, 0, (int64_t)a.B * a.T * kHq))
                               ? __bfloat162float(a.gate[gidx]) : 0.f;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.xsum_full, item & 1)))) break;
      const float l = sm.xsum[item & 1][0][r] + sm.xsum[item & 1][1][r];   // both at the row's final base
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_final, item & 1)))) break;
      tc_fence_after();
      float f = l > 0.f ? 1.f / l : 0.f;
      if (a.gate != nullptr) f *= 1.f / (1.f + __expf(-gscore));
      const float2 f2 = make_float2(f, f);
      uint32_t ov[32], on[32];
      tmem_ld32(trow + kColO, on);
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = on[e];
        if (c < kD / 32 - 1) tmem_ld32(trow + kColO + 32 * (c + 1), on);   // next chunk in flight
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int cc = 8 * q4 + 2 * e;
            const float2 o = fmul2(make_float2(__uint_as_float(ov[cc]), __uint_as_float(ov[cc + 1])), f2);
            w4[e] = pack_bf16(o.x, o.y);
          }
          *reinterpret_cast<uint4*>(stg + lane * 64 + 16 * (q4 ^ ((lane >> 1) & 3))) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async();   // the staging writes, then the TMA engine's read of them
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(&tm_o, smem_u32(stg), 32 * c, h, it.m0 + 32 * qtr, it.b);
          tma_store_commit();
          tma_store_wait_read();   // the staging area is free again
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&sm.o_free);
        else mbar_arrive_remote(&sm.o_free, 0);
      }
      ++item;
    }
  } else {
    // ======================= softmax / epilogue (warps 0-7) =======================
    const int wg = warp >> 2;            // warpgroup: keys [64 wg, 64 wg + 64) of each tile
    const int qtr = warp & 3;            // lane quarter of tensor memory
    const int r = qtr * 32 + lane;       // query row in the tile = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(qtr * 32) << 16);
    const float scale_log2 = 0.0625f * 1.4426950408889634f;
    const float2 scale2 = make_float2(scale_log2, scale_log2);
    // barrier among the 128 threads of this warpgroup; each thread counts the
    // phases it has passed (none can get two phases ahead: every phase needs
    // all arrivals)
    uint32_t n_sync = 0;
    auto sync_wg = [&]() -> bool {
      mbar_arrive(&sm.sync_wg[wg]);
      return mbar_wait(&sm.sync_wg[wg], (n_sync++) & 1);
    };
    auto arrive_cta0 = [&](uint64_t* bar) {   // lane 0, after __syncwarp: one arrival for the warp
      if (lane == 0) {
        if (rank == 0) mbar_arrive(bar);
        else mbar_arrive_remote(bar, 0);
      }
    };
    float q_row_scale = 1.f;   // FP8: this row's 2^(ex - 7) x the softmax scale (log2) of the last prepared query tile
    // Rotates this warpgroup's half of the frequencies of the query tile of
    // `it` (the item_no-th of this pair) in qo and hands it to the MMA issuer.
    auto prepare_q = [&](const Item& it, int item_no) -> bool {
     if constexpr (!FULL) {
      return false;   // sliding layers: queries always arrive rotated
     } else {
      if (a.q_rotated) {   // FP8 with rotated queries: only the split into Q_hi + Q_lo below
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_full, item_no & 1))) return false;
      } else {
      const int row = it.m0 + r;
      const bool valid = row < a.T;
      const int qseq = it.qb + row;
      const int64_t pidx = (int64_t)it.b * a.T + it.m0;
      const int p_base = a.pos ? (HYB_BOUNDS(pidx, 0, (int64_t)a.B * a.T) ? a.pos[pidx] : 0) : it.qb + it.m0;
      const int p = a.pos ? (valid ? a.pos[(int64_t)it.b * a.T + row] : 0) : qseq;
      const int delta = p - p_base;
      const bool in_table = __all_sync(0xffffffffu, delta >= 0 && delta < kBM);
      constexpr int NF = R / 4;          // frequencies of this warpgroup
      const int f0 = wg * NF;
      // ---- rotation tables of this tile's base position (this warpgroup's frequencies) ----
      if (!__all_sync(0xffffffffu, sync_wg())) return false;   // the area is no longer read or staged in
      for (int t = r; t < NF * 8; t += kBM) {
        const int kf = f0 + t % NF, e = t / NF;
        float sn, cs;
        rope_sincos(p_base + 16 * e, sm.inv_freq[kf], &sn, &cs);
        reinterpret_cast<float2*>(&sm.rot_hi[e][kf >> 1])[kf & 1] = make_float2(cs, sn);
      }
      for (int t = r; t < NF * 16; t += kBM) {
        const int kf = f0 + t % NF, e = t / NF;
        float sn, cs;
        small_angle_sincos(e, (float)sm.inv_freq[kf], &sn, &cs);
        reinterpret_cast<float2*>(&sm.rot_lo[kf >> 1][e])[kf & 1] = make_float2(cs, sn);
      }
      if (!__all_sync(0xffffffffu, sync_wg())) return false;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_full, item_no & 1))) return false;
      // ---- rotate dims [f0, f0 + NF) against [f0 + R/2, ...) in place ----
      constexpr int NW = 8;   // packed words (16 dims of each half) per pass
#pragma unroll
      for (int c = 0; c < NF / (2 * NW); ++c) {
        const int k0 = f0 + 2 * NW * c;
        uint32_t x1[NW], x2[NW];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int dim0 = k0 + h * (R / 2);
#pragma unroll
          for (int i = 0; i < NW / 4; ++i) {
            const int ci = dim0 / 8 + i;
            const uint4 v = *reinterpret_cast<const uint4*>(sm.qo[ci >> 3] + sw128_offset((uint32_t)r, (uint32_t)(ci & 7) * 16));
            uint32_t* xw = h ? x2 : x1;
            xw[4 * i] = v.x;
            xw[4 * i + 1] = v.y;
            xw[4 * i + 2] = v.z;
            xw[4 * i + 3] = v.w;
          }
        }
        if (in_table)
          rotate_table<NW, R / 4>(x1, x2, k0, delta >> 4, delta & 15, sm.rot_lo, sm.rot_hi);
        else
          rotate_general<NW>(x1, x2, k0, p, sm.inv_freq);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int dim0 = k0 + h * (R / 2);
          const uint32_t* xw = h ? x2 : x1;
#pragma unroll
          for (int i = 0; i < NW / 4; ++i) {
            const int ci = dim0 / 8 + i;
            *reinterpret_cast<uint4*>(sm.qo[ci >> 3] + sw128_offset((uint32_t)r, (uint32_t)(ci & 7) * 16)) =
                make_uint4(xw[4 * i], xw[4 * i + 1], xw[4 * i + 2], xw[4 * i + 3]);
          }
        }
      }
      }
      if constexpr (FP8) {
        // The row as Q_hi + Q_lo, both e4m3, for the e4m3 keys: every element times
        // 2^(7 - e), where 2^e <= the row's largest |element| < 2^(e + 1) (found over
        // both warpgroups' halves of the row), so that the largest lies in [128, 256);
        // Q_hi is an element rounded to e4m3, Q_lo the remainder rounded to e4m3:
        // for the tile's bf16 values that is exact down to 2^-9 of the row's largest
        // (8 significant bits = 4 + 4), below within 2^-17 of it.  This warpgroup's
        // 16 chunks of 8 dims for the maximum include every dim it rotated.
        auto chunk_of = [&](int i) { return i < 4 ? 2 * wg + (i & 1) + 4 * (i >> 1) : 8 + 12 * wg + (i - 4); };
        float am = 0.f;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int ci = chunk_of(i);
          const uint4 v = *reinterpret_cast<const uint4*>(sm.qo[ci >> 3] + sw128_offset((uint32_t)r, (uint32_t)(ci & 7) * 16));
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) am = fmaxf(am, fmaxf(fabsf(bf16lo(wv[j])), fabsf(bf16hi(wv[j]))));
        }
        // xsum of the coming item's parity is free: the other warpgroup read it in the
        // epilogue before last, and writes it next after reading this value
        sm.xsum[item_no & 1][wg][r] = am;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.qx_full[qtr]);
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.qx_full[qtr], item_no & 1))) return false;
        am = fmaxf(am, sm.xsum[item_no & 1][wg ^ 1][r]);
        int ex = am > 0.f ? (int)((__float_as_uint(am) >> 23) & 0xFFu) - 127 : 7;   // zero row: factor 1
        ex = max(ex, -100);                     // a subnormal row is scaled as 2^-100 would be
        const float down = __uint_as_float((uint32_t)(127 + 7 - ex) << 23);            // 2^(7 - ex)
        q_row_scale = __uint_as_float((uint32_t)(127 + ex - 7) << 23) * scale_log2;   // 2^(ex - 7), log2 units
        // this warpgroup's dims [128 wg, 128 wg + 128), bf16 in qo[2 wg] and qo[2 wg + 1],
        // become Q_hi in qo[2 wg] and Q_lo in qo[2 wg + 1] (16 dims per 16-byte chunk).
        // Every one is read before any is overwritten; the other warpgroup rotated some
        // of them, and arrived at the exchange above after that.
        uint4 x[16];
#pragma unroll
        for (int m = 0; m < 16; ++m)
          x[m] = *reinterpret_cast<const uint4*>(sm.qo[2 * wg + (m >> 3)] + sw128_offset((uint32_t)r, (uint32_t)(m & 7) * 16));
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t wv[8] = {x[2 * c].x, x[2 * c].y, x[2 * c].z, x[2 * c].w,
                                  x[2 * c + 1].x, x[2 * c + 1].y, x[2 * c + 1].z, x[2 * c + 1].w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {   // dims 4 j .. 4 j + 3 of the chunk
            const float v0 = bf16lo(wv[2 * j]) * down, v1 = bf16hi(wv[2 * j]) * down;
            const float v2 = bf16lo(wv[2 * j + 1]) * down, v3 = bf16hi(wv[2 * j + 1]) * down;
            const uint32_t h01 = f32x2_to_e4m3x2(v0, v1), h23 = f32x2_to_e4m3x2(v2, v3);
            const float2 b01 = e4m3x2_to_f32x2(h01), b23 = e4m3x2_to_f32x2(h23);
            const uint32_t l01 = f32x2_to_e4m3x2(v0 - b01.x, v1 - b01.y), l23 = f32x2_to_e4m3x2(v2 - b23.x, v3 - b23.y);
            hw[j] = h01 | (h23 << 16);
            lw[j] = l01 | (l23 << 16);
          }
          *reinterpret_cast<uint4*>(sm.qo[2 * wg] + sw128_offset((uint32_t)r, (uint32_t)c * 16)) =
              make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sm.qo[2 * wg + 1] + sw128_offset((uint32_t)r, (uint32_t)c * 16)) =
              make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      fence_proxy_async();              // qo is read by the tensor core
      if (rank != 0) fence_cluster();   // ... through MMAs issued from CTA 0
      tc_fence_before();                // TMEM accesses so far precede the MMAs q_ready releases
      __syncwarp();
      arrive_cta0(&sm.q_ready);
      return true;
     }
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
    bool ok = !have || (a.q_rotated && !FP8) || prepare_q(it, 0);
    float rs = q_row_scale;   // the current item's query row factor (FP8)
    while (ok && have) {
      const int h = it.h_pair0 + (int)rank;
      const int row = it.m0 + r;
      const bool valid = row < a.T;
      const int qseq = it.qb + row;
      // the row's gate score, loaded now so that its latency is not on the epilogue's path
      const int64_t gidx = ((int64_t)it.b * a.T + row) * kHq + h;
      const float gscore = (!PfCfg<FULL, FP8>::kEpi && a.gate != nullptr && valid &&
                            HYB_BOUNDS(gidx, 0, (int64_t)a.B * a.T * kHq))
                               ? __bfloat162float(a.gate[gidx]) : 0.f;

      // ---- online softmax over this warpgroup's keys of each tile ----
      float l_run = 0.f, b_run = -INFINITY;   // running sum (this warpgroup's keys) and the row's base
      for (int j = 0; ok && j < it.n; ++j) {
        const uint32_t jt = J + j;
        const uint32_t sb = jt % kNS;
        const uint32_t scol = col_s(sb) + 64 * wg;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (jt / kNS) & 1)))) break;
        tc_fence_after();
        uint32_t sraw[64];
        tmem_ld32(trow + scol, *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]));
        tmem_ld32(trow + scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]));
        tmem_wait_ld();
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sraw[c]);
        if constexpr (FP8) {   // x the key row's scale; the query row's factor and the softmax
                               // scale (rs) come in with the maximum and the exponent
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.f_full[jt % kNF], (jt / kNF) & 1)))) break;
          const float2* kf2 = reinterpret_cast<const float2*>(&sm.kf[jt % kNF][64 * wg]);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float2 v = fmul2(make_float2(s[2 * c], s[2 * c + 1]), kf2[c]);
            s[2 * c] = v.x;
            s[2 * c + 1] = v.y;
          }
        }

        const int ks0 = it.kb + (it.j_lo + j) * kBN + 64 * wg;   // sequence index of this warpgroup's first key
        const bool whole = ks0 >= 0 && ks0 + 63 <= it.q_lo && (FULL || it.q_hi - ks0 <= kWindow - 1);
        if (!whole) {
          // visible columns of this row: c_lo <= c <= c_hi (the band is contiguous);
          // none visible: an empty range past the last column
          int c_lo = max(-ks0, FULL ? 0 : qseq - (kWindow - 1) - ks0);
          int c_hi = qseq - ks0;
          if (c_hi < c_lo) c_lo = c_hi = 64;
          const uint32_t span = (uint32_t)(c_hi - c_lo);
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if ((uint32_t)(c - c_lo) > span) s[c] = -INFINITY;
        }
        // row maximum over this warpgroup's keys: pairwise tree (short dependency chains)
        float mx[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) mx[c] = fmaxf(s[c], s[c + 32]);
#pragma unroll
        for (int wd = 16; wd >= 1; wd >>= 1)
#pragma unroll
          for (int c = 0; c < wd; ++c) mx[c] = fmaxf(mx[c], mx[c + wd]);
        // ---- the maximum over the whole tile, through the partner warp ----
        sm.xmax[jt & 1][wg][r] = mx[0];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.xmax_full[jt & 1][qtr]);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.xmax_full[jt & 1][qtr], (jt >> 1) & 1)))) break;
        const float m_tile = fmaxf(mx[0], sm.xmax[jt & 1][wg ^ 1][r]) * (FP8 ? rs : scale_log2);
        const bool rescale = m_tile > b_run + kRescaleThreshold;
        const float b_new = rescale ? m_tile : b_run;
        const float alpha = rescale ? ex2(b_run - b_new) : 1.f;   // b_run = -inf: O and l are 0

        const float base = (b_new == -INFINITY) ? 0.f : b_new;
        // FP8: P x 2^64 (with V's codes widened x 2^-120, O stays far from fp32's subnormals)
        const float nb = FP8 ? 64.f - base : -base;
        const float2 nbase2 = make_float2(nb, nb);
        const float2 rs2 = make_float2(rs, rs);
        uint32_t pw[32];
        float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // FP8: P for the P.V MMA carries the value row's scale too (the sums do not)
        const float2* vf2 = FP8 ? reinterpret_cast<const float2*>(&sm.vf[jt % kNF][64 * wg]) : nullptr;
#pragma unroll
        for (int wd = 0; wd < 32; ++wd) {
          const float2 x = ffma2(make_float2(s[2 * wd], s[2 * wd + 1]), FP8 ? rs2 : scale2, nbase2);
          const float2 e = make_float2(ex2(x.x), ex2(x.y));
          ps[wd & 3] = fadd2(ps[wd & 3], e);
          if constexpr (FP8) {
            const float2 ev = fmul2(e, vf2[wd]);
            pw[wd] = pack_bf16(ev.x, ev.y);
          } else {
            pw[wd] = pack_bf16(e.x, e.y);
          }
        }
        if constexpr (FP8) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.f_free[jt % kNF]);   // this warp is done with the tile's factors
        }
        const float2 s01 = fadd2(fadd2(ps[0], ps[1]), fadd2(ps[2], ps[3]));
        l_run = l_run * alpha + (s01.x + s01.y);
        b_run = b_new;
        tmem_st32(trow + scol, pw);
        tmem_wait_st();
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O holds tiles < jt at the old base: once tile jt - 1's P.V has landed,
          // bring this warpgroup's half of it to the new one
          const uint32_t jp = jt - 1;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_done[jp % kNS], (jp / kNS) & 1)))) break;
          tc_fence_after();
          const float2 al2 = make_float2(alpha, alpha);
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t ov[32];
            tmem_ld32(trow + kColO + 128 * wg + 32 * c4, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 o = fmul2(make_float2(__uint_as_float(ov[2 * e]), __uint_as_float(ov[2 * e + 1])), al2);
              ov[2 * e] = __float_as_uint(o.x);
              ov[2 * e + 1] = __float_as_uint(o.y);
            }
            tmem_st32(trow + kColO + 128 * wg + 32 * c4, ov);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        arrive_cta0(&sm.p_full[sb]);
      }
      J += it.n;
      if (!ok) break;
      // ---- this warpgroup's sum for the other one ----
      sm.xsum[item & 1][wg][r] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.xsum_full);

      Item nxt{};
      const bool have_next = next_item(k, nxt);
      if (have_next && (!a.q_rotated || FP8) && !(ok = prepare_q(nxt, item + 1))) break;
      const float rs_next = q_row_scale;

      if constexpr (!PfCfg<FULL, FP8>::kEpi) {
      // ---- epilogue: O / l * sigmoid(gate) -> bf16 -> global, this warpgroup's 128 dims ----
      // 32 dims at a time through the warp's staging area: each thread writes
      // its row of 64 bytes, 16-byte chunk q at chunk q ^ ((row / 2) % 4) (no bank
      // conflicts, and the layout of a 64-byte-swizzled tensor map), then one
      // lane issues a TMA store of the 32 rows x 32 dims (rows past T are not
      // written).
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.xsum_full, item & 1)))) break;
      const float l = l_run + sm.xsum[item & 1][wg ^ 1][r];   // both at the row's final base
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_final, item & 1)))) break;
      tc_fence_after();
      float f = l > 0.f ? (FP8 ? kTwo120 : 1.f) / l : 0.f;   // FP8: O and l carry P x 2^64, O V x 2^-120
      if (a.gate != nullptr) f *= 1.f / (1.f + __expf(-gscore));
      const float2 f2 = make_float2(f, f);
      uint8_t* stg = sm.ostage[warp];
      uint32_t ov[32], on[32];
      tmem_ld32(trow + kColO + 128 * wg, on);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = on[e];
        if (c < 3) tmem_ld32(trow + kColO + 128 * wg + 32 * (c + 1), on);   // next chunk in flight
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int cc = 8 * q4 + 2 * e;
            const float2 o = fmul2(make_float2(__uint_as_float(ov[cc]), __uint_as_float(ov[cc + 1])), f2);
            w4[e] = pack_bf16(o.x, o.y);
          }
          *reinterpret_cast<uint4*>(stg + lane * 64 + 16 * (q4 ^ ((lane >> 1) & 3))) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async();   // the staging writes, then the TMA engine's read of them
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(&tm_o, smem_u32(stg), 128 * wg + 32 * c, h, it.m0 + 32 * qtr, it.b);
          tma_store_commit();
          tma_store_wait_read();   // the staging area is free again
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      arrive_cta0(&sm.o_free);
      }
      it = nxt;
      have = have_next;
      rs = rs_next;
      ++item;
    }
  }

  if ((warp < kSmWarps || (PfCfg<FULL, FP8>::kEpi && warp >= kEpiWarp0)) && lane == 0)
    tma_store_commit_and_wait();   // epilogue stores complete
  // the peer's shared memory and tensor memory stay alive until both CTAs are done
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == kMmaWarp) {
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
  if (!full && !h.q_rotated) return cudaErrorInvalidValue;   // sliding layers take rotated queries
  if (!full && h.fp8) return cudaErrorInvalidValue;          // FP8 rings are read through a bf16 context
  const long long grid = 2 * (n_items < h.n_pairs ? n_items : h.n_pairs);   // persistent CTA pairs
  profile_before(st);
  if (full && h.fp8)
    prefill_kernel<true, true><<<(unsigned)grid, PfCfg<true, true>::kThreads, prefill_smem_bytes_t<true, true>(), st>>>(
        h.tm_k, h.tm_v, h.tm_q, h.tm_o, h.tm_ks, h.tm_vs, a);
  else if (full)
    prefill_kernel<true, false><<<(unsigned)grid, PfCfg<true, false>::kThreads, prefill_smem_bytes_t<true>(), st>>>(
        h.tm_k, h.tm_v, h.tm_q, h.tm_o, h.tm_k, h.tm_v, a);
  else
    prefill_kernel<false, false><<<(unsigned)grid, PfCfg<false, false>::kThreads, prefill_smem_bytes_t<false>(), st>>>(
        h.tm_k, h.tm_v, h.tm_q, h.tm_o, h.tm_k, h.tm_v, a);
  profile_after(st);
  count_launch();
  return cudaGetLastError();
}

// Box rows of the K and V tensor maps this kernel expects.
int prefill_k_box_rows() { return kHalfKeys; }
int prefill_v_box_rows() { return kHalfKeys; }
int prefill_q_box_rows() { return kBM; }

cudaError_t prefill_set_smem_attr() {
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prefill_smem_bytes_t<true>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)prefill_smem_bytes_t<true, true>());
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(prefill_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)prefill_smem_bytes_t<false>());
}

}  // namespace hyb
