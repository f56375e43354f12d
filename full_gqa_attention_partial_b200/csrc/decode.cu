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
// m16n8k16 in transposed form: S^T[16 keys x 8 heads] = K Q^T puts a warp's
// 16 keys on the M rows and the group's 4 query heads on half of the N
// columns, the probabilities are turned into the B operand by movmatrix,
// and O^T[256 dims x 8 heads] += V^T P^T.  Half the columns idle instead of
// three quarters of the rows with the heads on M, so a key costs half the
// MMAs and the output accumulator half the registers.  At about 4 flop per
// byte the kernel is bound by HBM, not by the tensor pipe.
//
// Warps 0-3 consume (16 keys each per stage), warp 4 issues the TMA loads.
//
// FP8 caches (e4m3 codes + one fp32 scale per key row): a stage holds the
// codes (half the bytes) and the 64 keys' scales, three stages deep, and
// two FP8 CTAs share an SM.  Each
// lane loads its own codes straight into registers (conflict-free chunk
// orders below), releases the stage, and widens them to bf16 fragments with
// integer bit moves (the value times 2^-120).  The contraction over dims is
// free to take the dims in any order as long as Q's fragments follow the
// same order, which lets a lane pair codes 0/2 and 1/3 of a word.  The K
// scale is applied to the scores after the softmax scale has taken back the
// 2^-120; the V scale (times 2^64) is folded into P and the remaining 2^56
// goes onto the split's output.  P then stays below the bf16 maximum for any
// V row of amax up to 448 * 2^64, and the products P V stay far above the
// fp32 subnormal range.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kDecKeys = 64;                         // keys per stage
constexpr int kDecStages = 3;                        // bf16 stages
constexpr int kDecTileBytes = kDecKeys * kD * 2;     // 32 KB (K or V)
constexpr int kDecStageBytes = 2 * kDecTileBytes;    // K + V
constexpr int kDecThreads = 160;
constexpr int kBoxBytes = kDecKeys * 128;            // one 64-dim box of 64 keys
// FP8 stage: K codes (2 boxes of 128 dims), V codes, K scales, V scales.
// FP8 CTAs take half the shared memory, so two share an SM.
constexpr int kDec8Stages = 3;
constexpr int kDec8TileBytes = kDecKeys * kD;        // 16 KB of codes
constexpr int kDec8Box = kDecKeys * 128;             // 128 dims x 64 keys
constexpr int kDec8StageBytes = 2 * kDec8TileBytes + 2 * kDecKeys * 4 + 512;   // padded to 1 KB multiples

constexpr int kDecClusterMax = 8;   // most splits merged inside a cluster

template <bool FP8>
struct DecSmem {
  static constexpr int kStages = FP8 ? kDec8Stages : kDecStages;
  static constexpr int kRingBytes = FP8 ? kDec8Stages * kDec8StageBytes : kDecStages * kDecStageBytes;
  // stage ring first (1024-byte aligned base); after the last stage it holds
  // the warps' partial outputs, float [warp][head][dim], and in CTA 0 of a
  // cluster, after them, every split's normalised output [split][head][dim]
  // and base-2 log-sum-exp [split][head]
  uint8_t ring[kRingBytes];
  float merge_m[4][4];
  float merge_l[4][4];
  __nv_bfloat16 qs[4][kD];      // rotated queries of the group
  int32_t tags[kWindow];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  static constexpr int kMergeBytes = 4 * 4 * kD * 4;
  static constexpr int kGatherBytes = kDecClusterMax * 4 * kD * 4;
  __device__ float (&merge_o())[4][4][kD] { return *reinterpret_cast<float(*)[4][4][kD]>(ring); }
  __device__ float (&gather_o())[kDecClusterMax][4][kD] {
    return *reinterpret_cast<float(*)[kDecClusterMax][4][kD]>(ring + kMergeBytes);
  }
  __device__ float (&gather_lse())[kDecClusterMax][4] {
    return *reinterpret_cast<float(*)[kDecClusterMax][4]>(ring + kMergeBytes + kGatherBytes);
  }
};
static_assert(DecSmem<true>::kRingBytes >= DecSmem<true>::kMergeBytes + DecSmem<true>::kGatherBytes + 4 * kDecClusterMax * 4 &&
                  DecSmem<false>::kRingBytes >= DecSmem<false>::kMergeBytes + DecSmem<false>::kGatherBytes + 4 * kDecClusterMax * 4,
              "the ring must hold the merge and cluster-gather buffers");

size_t decode_smem_bytes(bool fp8) { return (fp8 ? sizeof(DecSmem<true>) : sizeof(DecSmem<false>)) + 1024; }
static_assert(2 * (sizeof(DecSmem<true>) + 1024 + 1024) <= 228 * 1024, "two FP8 CTAs must share an SM");
static_assert(kDec8StageBytes % 1024 == 0, "FP8 stage must keep 1 KB alignment");

// Chunk orders of the FP8 loads.  A 16-byte load of lanes 4t..4t+7 (rows
// 2t, 2t+1; q = 0..3) is conflict-free when the four lanes of a row read
// 16-byte slots whose indexes differ in their upper two bits (the 128-byte
// swizzle XORs the slot with the row).  K: lane q covers 64 dims of box
// q / 2, chunk dec8_kchunk(q, j) at step j.  V: lane r covers chunk r of
// both boxes (dims 16 r .. 16 r + 15 of each 128), whose parity alternates
// with the row.
__device__ __forceinline__ int dec8_kchunk(int q, int j) {
  return 2 * ((q & 1) + 2 * ((j & 1) ^ (q >> 1))) + (j >> 1);
}
// Dim of row m of MMA block i (O^T rows) for the FP8 V fragments.
__device__ __forceinline__ int dec8_vdim(int i, int m) {
  return 128 * (i >> 3) + 16 * (m & 7) + 4 * ((i >> 1) & 3) + 2 * (i & 1) + (m >> 3);
}

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
  int B;              // sequences (index checks of the debug build)
  PageMap pm;         // paged cache: maps over the pool {.., page, 4, n_pages}
  // cluster merge (the splits of one (sequence, KV head) form a thread-block
  // cluster): CTA 0 of the cluster merges them and writes the result itself
  int cluster_merge;
  const __nv_bfloat16* gate;   // [B][16] or null
  __nv_bfloat16* out;          // [B][16][256] gated bf16, or
  float* out_o;                // [B][16][256] fp32 and
  float* out_lse;              // [B][16] base-2 log-sum-exp
};


template <bool FULL, bool FP8>
__global__ void __launch_bounds__(kDecThreads, FP8 ? 2 : 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                        DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem<FP8>& sm = *reinterpret_cast<DecSmem<FP8>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int R = RopeCfg<FULL>::R;
  constexpr int NST = DecSmem<FP8>::kStages;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();   // the barriers are initialised (before the wait: overlaps the previous kernel)
  // the append before this launch writes len, tags and the new token's row
  pdl_wait();
  pdl_launch_dependents();

  const int L = HYB_BOUNDS(b, 0, a.B) ? a.len[b] : 0;
  const int qseq = L - 1;
  const int n_keys = FULL ? L : kWindow;          // keys (FULL) or ring slots (SLIDING)
  int kps = (n_keys + a.n_splits - 1) / a.n_splits;
  kps = (kps + kDecKeys - 1) / kDecKeys * kDecKeys;
  const int k0 = split * kps;
  const int k1 = min(n_keys, k0 + kps);
  const int n_stages = (k1 > k0 && L > 0) ? (k1 - k0 + kDecKeys - 1) / kDecKeys : 0;
  // this split's normalised output (dims 8 lane .. + 7 of head `warp`) and
  // base-2 log-sum-exp, for the merge inside a cluster
  float cres[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float clse = -INFINITY;

  // The producer issues the first stages as soon as len is known; the
  // consumers meanwhile load the queries and (ring caches) the slot tags.
  if (warp == 4) {
    // ---------------- producer ----------------
    if (lane == 0 && n_stages > 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int i = 0; i < n_stages; ++i) {
        const int slot = i % NST;
        if (i >= NST && !mbar_wait(&sm.empty[slot], ((i / NST) - 1) & 1)) break;
        const int key = k0 + i * kDecKeys;
        int crow, cpage;   // the stage's 64 keys lie within one page
        kv_coord(a.pm, b, key, crow, cpage);
        if (FP8) {
          mbar_arrive_expect_tx(&sm.full[slot], 2 * kDec8TileBytes + 2 * kDecKeys * 4);
          const uint32_t kdst = smem_u32(sm.ring) + slot * kDec8StageBytes;
          const uint32_t vdst = kdst + kDec8TileBytes;
#pragma unroll
          for (int box = 0; box < 2; ++box) {
            tma_load_4d(kdst + box * kDec8Box, &tm_k, &sm.full[slot], box * 128, crow, kvh, cpage);
            tma_load_4d(vdst + box * kDec8Box, &tm_v, &sm.full[slot], box * 128, crow, kvh, cpage);
          }
          tma_load_3d(vdst + kDec8TileBytes, &tm_ks, &sm.full[slot], crow, kvh, cpage);
          tma_load_3d(vdst + kDec8TileBytes + kDecKeys * 4, &tm_vs, &sm.full[slot], crow, kvh, cpage);
          issued = i + 1;
          continue;
        }
        mbar_arrive_expect_tx(&sm.full[slot], kDecStageBytes);
        const uint32_t kdst = smem_u32(sm.ring) + slot * kDecStageBytes;
        const uint32_t vdst = kdst + kDecTileBytes;
#pragma unroll
        for (int box = 0; box < 4; ++box) {
          tma_load_4d(kdst + box * kBoxBytes, &tm_k, &sm.full[slot], box * 64, crow, kvh, cpage);
          tma_load_4d(vdst + box * kBoxBytes, &tm_v, &sm.full[slot], box * 64, crow, kvh, cpage);
        }
        issued = i + 1;
      }
      // drain: never leave the CTA with copies still landing in shared memory
      for (int i = max(0, issued - NST); i < issued; ++i)
        mbar_wait(&sm.full[i % NST], (i / NST) & 1);
    }
    __syncwarp();
    if (a.cluster_merge) cluster_arrive();   // this CTA's ring takes no more copies
  } else {
  // ---------------- consumers: rotate the group's 4 queries ----------------
  {
    const int hh = threadIdx.x >> 5;        // 0..3
    const int d0 = lane * 8;
    const int p = a.pos ? (HYB_BOUNDS(b, 0, a.B) ? a.pos[b] : 0) : qseq;
    uint4 qx = *reinterpret_cast<const uint4*>(a.q + (int64_t)b * a.q_stride + (int64_t)(kvh * kGroup + hh) * kD + d0);
    if (!FULL) {   // in flight with the query's load
      for (int i = threadIdx.x; i < kWindow; i += 128)
        sm.tags[i] = HYB_BOUNDS((int64_t)b * kWindow + i, 0, (int64_t)a.B * kWindow) ? a.tag[(int64_t)b * kWindow + i] : -1;
    }
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
          rope_sincos(p, rope_inv_freq<FULL>(kb + 2 * w + e), &s, &c);
          o2[e] = first_half ? fmaf(x, c, -y * s) : fmaf(x, c, y * s);
        }
        os[w] = pack_bf16(o2[0], o2[1]);
      }
      qx = make_uint4(os[0], os[1], os[2], os[3]);
    }
    *reinterpret_cast<uint4*>(&sm.qs[hh][d0]) = qx;
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");   // queries and tags in shared memory

  // Lane (r, q) = (lane / 4, lane % 4) in the m16n8k16 fragment layouts.
  const int r = lane >> 2, q = lane & 3;
  // B fragments of Q^T per 16-dim k-step: column r = head r (zero for r >= 4).
  // bf16: k-step kk takes dims 16 kk .. 16 kk + 15 in order.  FP8: k-step
  // 4 j + wd takes, for lane q, the 4 dims at 4 wd of the K chunk the lane
  // loads at step j, paired 0/2 and 1/3 like the widened codes.
  uint32_t qb[16][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(&sm.qs[r & 3][0]);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      uint32_t b0, b1;
      if (FP8) {
        const int d = 128 * (q >> 1) + 16 * dec8_kchunk(q, kk >> 2) + 4 * (kk & 3);
        const uint32_t x = qrow[d >> 1], y = qrow[(d >> 1) + 1];
        b0 = prmt(x, y, 0x5410u);
        b1 = prmt(x, y, 0x7632u);
      } else {
        b0 = qrow[8 * kk + q];
        b1 = qrow[8 * kk + q + 4];
      }
      qb[kk][0] = (r < 4) ? b0 : 0u;
      qb[kk][1] = (r < 4) ? b1 : 0u;
    }
  }

  const float scale_log2 = 0.0625f * 1.4426950408889634f;  // 1/sqrt(256) * log2(e)
  const float score_scale = FP8 ? scale_log2 * kE4m3WideScale : scale_log2;
  // running max and (lane-partial) sum for heads 2q and 2q + 1
  float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
  float o[16][4];   // O^T block i: rows = dims, columns = heads 2q, 2q + 1
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  const int mi = lane >> 3, rr = lane & 7;     // ldmatrix: matrix and row this lane addresses
  const int krow = warp * 16 + r;              // this lane's key rows: krow, krow + 8
  for (int i = 0; i < n_stages; ++i) {
    const int slot = i % NST;
    if (!mbar_wait(&sm.full[slot], (i / NST) & 1)) break;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};   // even / odd k-steps
    float ksc[2] = {1.f, 1.f}, vsc[2] = {1.f, 1.f};                 // rows krow, krow + 8
    uint4 vw[4][2];                                                 // FP8 V codes
    uint32_t vbase = 0;
    if (FP8) {
      const uint8_t* st8 = sm.ring + slot * kDec8StageBytes;
      uint4 kw[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = krow + 8 * h;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          kw[h][j] = *reinterpret_cast<const uint4*>(st8 + (q >> 1) * kDec8Box + row * 128 +
                                                     ((dec8_kchunk(q, j) ^ (row & 7)) << 4));
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int row = warp * 16 + 2 * q + (t & 1) + 8 * (t >> 1);
#pragma unroll
        for (int u = 0; u < 2; ++u)
          vw[t][u] = *reinterpret_cast<const uint4*>(st8 + kDec8TileBytes + u * kDec8Box + row * 128 +
                                                     ((r ^ (row & 7)) << 4));
      }
      const float* kscale = reinterpret_cast<const float*>(st8 + 2 * kDec8TileBytes);
      const float* vscale = kscale + kDecKeys;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        ksc[h] = kscale[krow + 8 * h];
        vsc[h] = vscale[krow + 8 * h] * kE4m3PScale;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);   // every code is in registers
      // ---- scores S^T = K Q^T ----
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t w0[4] = {kw[0][j].x, kw[0][j].y, kw[0][j].z, kw[0][j].w};
        const uint32_t w1[4] = {kw[1][j].x, kw[1][j].y, kw[1][j].z, kw[1][j].w};
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          const int kk = 4 * j + wd;
          mma_16816(acc[kk & 1], e4m3_b02_bf16x2(w0[wd]), e4m3_b02_bf16x2(w1[wd]), e4m3_b13_bf16x2(w0[wd]),
                    e4m3_b13_bf16x2(w1[wd]), qb[kk][0], qb[kk][1]);
        }
      }
    } else {
      const uint32_t kbase = smem_u32(sm.ring) + slot * kDecStageBytes;
      vbase = kbase + kDecTileBytes;
      const uint32_t kr = warp * 16 + (mi & 1) * 8 + rr;
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const uint32_t d = 16 * kk + (mi >> 1) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kbase + (d >> 6) * kBoxBytes + sw128_offset(kr, (d & 63) * 2), a0, a1, a2, a3);
        mma_16816(acc[kk & 1], a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
      }
    }
    // ---- mask, online softmax (log2 domain) per head ----
    // sv[h][e]: key row krow + 8 h, head 2 q + e
    float sv[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int key = k0 + i * kDecKeys + krow + 8 * h;
      bool ok = key < k1;
      if (!FULL && ok) {
        const int tg = sm.tags[key];
        ok = tg >= 0 && tg <= qseq && qseq - tg < kWindow;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float sc = acc[0][2 * h + e] + acc[1][2 * h + e];
        // (score * scale) first: with FP8 it restores the widening's 2^-120 before the row scale
        sv[h][e] = ok ? sc * score_scale * ksc[h] : -INFINITY;
      }
    }
    float pv[2][2], alpha[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float mx = fmaxf(sv[0][e], sv[1][e]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_run[e], mx);
      alpha[e] = (m_run[e] == -INFINITY) ? 1.f : exp2f(m_run[e] - m_new);
#pragma unroll
      for (int h = 0; h < 2; ++h) pv[h][e] = (m_new == -INFINITY || q >= 2) ? 0.f : exp2f(sv[h][e] - m_new);
      m_run[e] = m_new;
      l_part[e] = l_part[e] * alpha[e] + (pv[0][e] + pv[1][e]);
    }
    // O moves only when a head's maximum grew somewhere in the warp (times 1
    // otherwise, which changes nothing): past the first stages of a long
    // history that is rare, and the 64 multiplies are a tenth of a stage's work
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[1];
        o[n][2] *= alpha[0];
        o[n][3] *= alpha[1];
      }
    }
    // P^T (keys x heads, C layout) -> B fragments (k = keys, n = heads)
    const uint32_t pb0 = movmatrix_t(pack_bf16(pv[0][0] * vsc[0], pv[0][1] * vsc[0]));
    const uint32_t pb1 = movmatrix_t(pack_bf16(pv[1][0] * vsc[1], pv[1][1] * vsc[1]));
    // ---- O^T += V^T P^T over 256 dims ----
    if (FP8) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t w[4][4] = {{vw[0][u].x, vw[0][u].y, vw[0][u].z, vw[0][u].w},
                                  {vw[1][u].x, vw[1][u].y, vw[1][u].z, vw[1][u].w},
                                  {vw[2][u].x, vw[2][u].y, vw[2][u].z, vw[2][u].w},
                                  {vw[3][u].x, vw[3][u].y, vw[3][u].z, vw[3][u].w}};
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          // keys (2q, 2q+1) and (2q+8, 2q+9), dims 4 wd .. 4 wd + 3 of the lane's chunk:
          // block ib takes dims + 0 (rows r) and + 1 (rows r + 8), block ib + 1 dims + 2 and + 3;
          // each pair of keys is one code from each of two rows' words
          const uint32_t w0 = w[0][wd], w1 = w[1][wd], w2 = w[2][wd], w3 = w[3][wd];
          const int ib = 8 * u + 2 * wd;
          mma_16816(o[ib], e4m3_pair2_bf16x2<0xC480u>(w0, w1), e4m3_pair2_bf16x2<0xD591u>(w0, w1),
                    e4m3_pair2_bf16x2<0xC480u>(w2, w3), e4m3_pair2_bf16x2<0xD591u>(w2, w3), pb0, pb1);
          mma_16816(o[ib + 1], e4m3_pair2_bf16x2<0xE6A2u>(w0, w1), e4m3_pair2_bf16x2<0xF7B3u>(w0, w1),
                    e4m3_pair2_bf16x2<0xE6A2u>(w2, w3), e4m3_pair2_bf16x2<0xF7B3u>(w2, w3), pb0, pb1);
        }
      }
    } else {
      const uint32_t kr = warp * 16 + (mi >> 1) * 8 + rr;
#pragma unroll
      for (int ib = 0; ib < 16; ++ib) {
        const uint32_t d = 16 * ib + (mi & 1) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vbase + (d >> 6) * kBoxBytes + sw128_offset(kr, (d & 63) * 2), a0, a1, a2, a3);
        mma_16816(o[ib], a0, a1, a2, a3, pb0, pb1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }
  }

  // ---------------- merge the 4 warps, write the split's partial ----------------
  // the merge buffer overlays the ring: every consumer warp must be done with its last stage
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (a.cluster_merge) cluster_arrive();   // this CTA is done with its ring
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 4);
    l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 8);
    l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 16);
  }
  if (q < 2) {
    if (r == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        sm.merge_m[warp][2 * q + e] = m_run[e];
        sm.merge_l[warp][2 * q + e] = l_part[e];
      }
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int d0 = FP8 ? dec8_vdim(n, r) : 16 * n + r;
      const int d1 = FP8 ? dec8_vdim(n, r + 8) : 16 * n + 8 + r;
      sm.merge_o()[warp][2 * q][d0] = o[n][0];
      sm.merge_o()[warp][2 * q + 1][d0] = o[n][1];
      sm.merge_o()[warp][2 * q][d1] = o[n][2];
      sm.merge_o()[warp][2 * q + 1][d1] = o[n][3];
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
        for (int e = 0; e < 8; ++e) res[e] += f * sm.merge_o()[w][hh][d0 + e];
      }
      // with FP8, P carried 2^64 and V 2^-120: the output takes back 2^56
      const float inv = den > 0.f ? (FP8 ? kE4m3OutScale : 1.f) / den : 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) res[e] *= inv;
      lse = den > 0.f ? M + log2f(den) : -INFINITY;
    }
    const int hq = kvh * kGroup + hh;
    if (a.cluster_merge) {   // for CTA 0 of the cluster
#pragma unroll
      for (int e = 0; e < 8; ++e) cres[e] = res[e];
      clse = lse;
    } else {
      const int64_t row = ((int64_t)b * kHq + hq) * a.n_splits + split;
      if (HYB_BOUNDS(row, 0, (int64_t)a.B * kHq * a.n_splits)) {
        float4* dst = reinterpret_cast<float4*>(a.part_o + row * kD + d0);
        dst[0] = make_float4(res[0], res[1], res[2], res[3]);
        dst[1] = make_float4(res[4], res[5], res[6], res[7]);
        if (lane == 0) a.part_lse[row] = lse;
      }
    }
  }
  }

  if (a.cluster_merge) {
    // ---------------- merge the cluster's splits in CTA 0 (the log-sum-exp
    // combination of decode_combine_kernel, same order of operations) ----------------
    // Every CTA of the cluster has arrived once it was done with its ring, so
    // once the wait returns CTA 0's ring can take every split's result: each
    // CTA stores its own into CTA 0 (remote stores, no round trips), and after
    // one more barrier CTA 0 merges from its own shared memory.
    cluster_wait();
    if (warp < 4 && HYB_BOUNDS(split, 0, kDecClusterMax)) {
      const int hh = warp, d0 = lane * 8;
      st_cluster_f32x4(mapa_cluster(smem_u32(&sm.gather_o()[split][hh][d0]), 0), cres[0], cres[1], cres[2], cres[3]);
      st_cluster_f32x4(mapa_cluster(smem_u32(&sm.gather_o()[split][hh][d0 + 4]), 0), cres[4], cres[5], cres[6], cres[7]);
      if (lane == 0) st_cluster_f32(mapa_cluster(smem_u32(&sm.gather_lse()[split][hh]), 0), clse);
    }
    cluster_sync();   // every split's result is in CTA 0 (release / acquire)
    if (cluster_ctarank() == 0 && warp < 4) {
      const int hh = warp, d0 = lane * 8;
      const int hq = kvh * kGroup + hh;
      const int64_t orow = (int64_t)b * kHq + hq;
      const int n_parts = min(a.n_splits, kDecClusterMax);
      float M = -INFINITY;
      for (int s2 = 0; s2 < n_parts; ++s2) M = fmaxf(M, sm.gather_lse()[s2][hh]);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, den = 0.f;
      if (M != -INFINITY) {
        for (int s2 = 0; s2 < n_parts; ++s2) {
          const float ls = sm.gather_lse()[s2][hh];
          if (ls == -INFINITY) continue;
          const float w = exp2f(ls - M);
          den += w;
          const float4 o0 = *reinterpret_cast<const float4*>(&sm.gather_o()[s2][hh][d0]);
          const float4 o1 = *reinterpret_cast<const float4*>(&sm.gather_o()[s2][hh][d0 + 4]);
          acc[0] += w * o0.x; acc[1] += w * o0.y; acc[2] += w * o0.z; acc[3] += w * o0.w;
          acc[4] += w * o1.x; acc[5] += w * o1.y; acc[6] += w * o1.z; acc[7] += w * o1.w;
        }
      }
      float r8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) r8[e] = den > 0.f ? acc[e] / den : 0.f;
      if (!HYB_BOUNDS(orow, 0, (int64_t)a.B * kHq)) {
        // debug build: a row outside the output, skipped
      } else if (a.out_o != nullptr) {
        float4* dst = reinterpret_cast<float4*>(a.out_o + orow * kD + d0);
        dst[0] = make_float4(r8[0], r8[1], r8[2], r8[3]);
        dst[1] = make_float4(r8[4], r8[5], r8[6], r8[7]);
        if (lane == 0) a.out_lse[orow] = den > 0.f ? M + log2f(den) : -INFINITY;
      } else {
        if (a.gate != nullptr) {
          const float g = 1.f / (1.f + __expf(-__bfloat162float(a.gate[orow])));
#pragma unroll
          for (int e = 0; e < 8; ++e) r8[e] *= g;
        }
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat16 lo = __float2bfloat16_rn(r8[2 * e]), hi = __float2bfloat16_rn(r8[2 * e + 1]);
          w4[e] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
        }
        *reinterpret_cast<uint4*>(a.out + orow * kD + d0) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  }
}

// Merges n partial results of each (sequence, query head) row.  Partial s
// of row `row` has its normalised output at o + s * o_sstride + row *
// o_rstride and its base-2 log-sum-exp at lse + s * l_sstride + row *
// l_rstride: the merge weighs each by 2^lse (the log-sum-exp combination
// of split softmaxes).  It writes the gated bf16 output, or with out_o set
// the merged fp32 output and log-sum-exp (a partial over the union of the
// keys, for a further merge).
struct CombineArgs {
  const float* o;
  const float* lse;
  int64_t o_sstride, o_rstride, l_sstride, l_rstride;
  int n;
  const __nv_bfloat16* gate;   // [rows] or null (bf16 output only)
  __nv_bfloat16* out;          // [rows][256]
  float* out_o;                // [rows][256] or null
  float* out_lse;              // [rows]
};

__global__ void __launch_bounds__(256) decode_combine_kernel(CombineArgs a) {
  pdl_wait();   // the split kernel's partials
  pdl_launch_dependents();
  const int row = blockIdx.x;  // b * 16 + h
  const int d = threadIdx.x;
  const float* lse = a.lse + (int64_t)row * a.l_rstride;
  const float* po = a.o + (int64_t)row * a.o_rstride + d;
  float M = -INFINITY;
  for (int s = 0; s < a.n; ++s) M = fmaxf(M, lse[s * a.l_sstride]);
  float acc = 0.f, den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.n; ++s) {
      const float ls = lse[s * a.l_sstride];
      if (ls == -INFINITY) continue;
      const float w = exp2f(ls - M);
      den += w;
      acc += w * po[s * a.o_sstride];
    }
  }
  float r = den > 0.f ? acc / den : 0.f;
  if (a.out_o != nullptr) {
    a.out_o[(int64_t)row * kD + d] = r;
    if (d == 0) a.out_lse[row] = den > 0.f ? M + log2f(den) : -INFINITY;
    return;
  }
  if (a.gate != nullptr) {
    const float gs = __bfloat162float(a.gate[row]);
    r *= 1.f / (1.f + __expf(-gs));
  }
  a.out[(int64_t)row * kD + d] = __float2bfloat16_rn(r);
}

cudaError_t launch_decode_merge(const float* part_o, const float* part_lse, int64_t o_stride, int64_t lse_stride,
                                int n_parts, int rows, const void* gate, void* out, cudaStream_t st) {
  CombineArgs c;
  c.o = part_o;
  c.lse = part_lse;
  c.o_sstride = o_stride;
  c.o_rstride = kD;
  c.l_sstride = lse_stride;
  c.l_rstride = 1;
  c.n = n_parts;
  c.gate = reinterpret_cast<const __nv_bfloat16*>(gate);
  c.out = reinterpret_cast<__nv_bfloat16*>(out);
  c.out_o = nullptr;
  c.out_lse = nullptr;
  decode_combine_kernel<<<rows, 256, 0, st>>>(c);
  count_launch();
  return cudaGetLastError();
}

int decode_num_splits(bool full, int B, int64_t max_len, bool fp8) {
  const int64_t keys = full ? (max_len > 0 ? max_len : 1) : kWindow;
  const int64_t pairs = (int64_t)B * kHkv;
  // full layers: >= 8 stages of 64 keys per split; a 512-slot ring may go down to one
  // stage per split, so that a small batch still spreads its rings over the SMs
  const int64_t s_max = full ? (keys / 512 > 1 ? keys / 512 : 1) : kWindow / kDecKeys;
  // whole waves of CTA slots (one bf16 CTA per SM, two FP8 CTAs): the smallest split
  // count that fills its waves exactly, else the smallest within 5 % of that, else
  // the best fill
  const int sms = fp8 ? 2 * 148 : 148;
  int best = 1, first95 = 0;
  double best_eff = 0.0;
  for (int64_t s = 1; s <= s_max && s <= 1024; ++s) {
    const int64_t ctas = pairs * s;
    const int64_t waves = (ctas + sms - 1) / sms;
    const double eff = (double)ctas / (double)(waves * sms);
    if (eff >= 0.999) return (int)s;
    if (eff >= 0.95 && first95 == 0) first95 = (int)s;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = (int)s;
    }
  }
  return first95 ? first95 : best;
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
  a.B = h.B;
  a.pm = h.pm;
  // sliding layers (at most 8 splits of a 512-slot ring): the splits of one
  // (sequence, KV head) run as a cluster and merge in its CTA 0, no second
  // kernel; full layers write per-split partials for decode_combine_kernel
  a.cluster_merge = (!full && h.n_splits <= 8) ? 1 : 0;
  a.gate = reinterpret_cast<const __nv_bfloat16*>(h.gate);
  a.out = reinterpret_cast<__nv_bfloat16*>(h.out);
  a.out_o = h.out_o;
  a.out_lse = h.out_lse;
  const dim3 grid(h.n_splits, kHkv, h.B);
  const size_t smem = decode_smem_bytes(h.fp8);
  profile_before(st);
  cudaError_t e;
  const unsigned cl = a.cluster_merge ? (unsigned)h.n_splits : 0u;
  const dim3 blk(kDecThreads, 1, 1);
  if (full && h.fp8)
    e = launch_pdl(decode_split_kernel<true, true>, grid, blk, smem, st, cl, h.tm_k, h.tm_v, h.tm_ks, h.tm_vs, a);
  else if (full)
    e = launch_pdl(decode_split_kernel<true, false>, grid, blk, smem, st, cl, h.tm_k, h.tm_v, h.tm_k, h.tm_v, a);
  else if (h.fp8)
    e = launch_pdl(decode_split_kernel<false, true>, grid, blk, smem, st, cl, h.tm_k, h.tm_v, h.tm_ks, h.tm_vs, a);
  else
    e = launch_pdl(decode_split_kernel<false, false>, grid, blk, smem, st, cl, h.tm_k, h.tm_v, h.tm_k, h.tm_v, a);
  profile_after(st);
  count_launch();
  if (e != cudaSuccess) return e;
  if (a.cluster_merge) return cudaSuccess;
  CombineArgs c;
  c.o = h.part_o;
  c.lse = h.part_lse;
  c.o_sstride = kD;
  c.o_rstride = (int64_t)h.n_splits * kD;
  c.l_sstride = 1;
  c.l_rstride = h.n_splits;
  c.n = h.n_splits;
  c.gate = reinterpret_cast<const __nv_bfloat16*>(h.gate);
  c.out = reinterpret_cast<__nv_bfloat16*>(h.out);
  c.out_o = h.out_o;
  c.out_lse = h.out_lse;
  e = launch_pdl(decode_combine_kernel, dim3(h.B * kHq, 1, 1), dim3(256, 1, 1), 0, st, 0u, c);
  count_launch();
  return e;
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

// Device address of g_decode_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress, once per device, the first time a device uses it
// (with that device current), and cached together with the CUDA context it
// was found in.  A different current context on that device (after
// cudaDeviceReset, or a context the caller created itself) has the module
// loaded again at another address: the cached entry no longer matches the
// context, and the address is looked up again.
cudaError_t decode_noalloc_scratch(void** ptr, size_t* bytes) {
  static std::mutex mu;
  static void* addr[128] = {};
  static CUcontext ctx_of[128] = {};
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (get_ctx == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
    get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }
  // the caller's earlier runtime calls on this device (its set-up) made a context current
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  if (addr[dev] == nullptr || ctx_of[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  *ptr = addr[dev];
  *bytes = kNoAllocScratchBytes;
  return cudaSuccess;
}

cudaError_t decode_set_smem_attr() {
  const int smem = (int)decode_smem_bytes(false), smem8 = (int)decode_smem_bytes(true);
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_split_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_split_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem8);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_split_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem8);
  return e;
}

}  // namespace hyb
