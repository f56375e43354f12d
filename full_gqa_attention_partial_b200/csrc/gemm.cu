// Linear projections around the attention core (q_k_v_proj, the head-wise
// gate projection and o_proj of "百万 Token 塞进 4B ..." §"省显存的第二板斧"):
//   Y[M, N] = X[M, K] W[N, K]^T   (bf16 in and out, fp32 accumulation),
// with W in the usual [out_features, in_features] layout.
//
// A cluster of two CTAs owns a 256 x 256 output tile: each CTA TMA-loads its
// 128 rows of X and 128 rows of W per 64-wide K block into a 6-stage ring
// (128-byte swizzle), and one warp of CTA 0 issues pair MMAs
// (tcgen05.mma.cta_group::2, M = 256, N = 256, both operands from shared
// memory).  The accumulator (128 x 256 fp32 per CTA) is double-buffered in
// tensor memory, so the 4 epilogue warps drain one tile (TMEM -> bf16 ->
// per-warp 32 x 32 transpose in shared memory -> 64-byte row segments to
// global memory) while the next tile accumulates.  Pairs are persistent and
// walk the tiles row-band first (all column tiles of 256 rows in turn), so
// W and the current rows of X stay in L2.
//
// Roles (192 threads): warps 0-3 epilogue (one TMEM lane = one output row),
// warp 4 lane 0 TMA producer (both CTAs), warp 5 TMEM allocation and, in
// CTA 0, the MMA loop.  Every wait is bounded.
//
// Optional RoPE epilogue (ROPE = 1 sliding layer, theta 1e4 over all 256
// dims; ROPE = 2 full layer, theta 5e6 over the first 64 dims; rotate-half,
// as in the attention core): for q_k_v_proj, output column tiles below
// rope_cols are 256-wide heads (q and k), rotated in fp32 from the
// accumulator at the row's position before the single rounding to bf16.
// The (cos, sin) of each (row, frequency) come from a table computed once
// per call (rope_table_kernel), shared by the row's 20 q and k heads.
//
// Optional second output group: columns n_main .. N - 1 (n_main a multiple
// of the 256-wide tile) take their W rows from a second matrix (tm_w2, from
// its row 0) and go to a second output (y2, column 0 on): the gate
// projection's 16 rows ride in q_k_v_proj's launch as one more column tile
// (rows past the second matrix read as zeros), instead of a launch of their
// own.
#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kGM = 128;            // output rows per CTA (256 per pair)
constexpr int kGN = 256;            // output columns per pair tile
constexpr int kGK = 64;             // K per stage
constexpr int kGStages = 6;
constexpr int kGHalf = 16384;       // one CTA's 128 rows x 64 K of X, or of W
constexpr int kGThreads = 192;

struct GemmSmem {
  uint8_t x[kGStages][kGHalf];      // 1024-byte aligned
  uint8_t w[kGStages][kGHalf];
  uint8_t ostage[4][2048];          // per epilogue warp: 32 rows x 32 columns (bf16)
  uint64_t full[kGStages];          // CTA 0's count both CTAs' bytes
  uint64_t empty[kGStages];
  uint64_t acc_full[2];             // accumulator buffer complete (MMA commit)
  uint64_t acc_empty[2];            // drained: one arrival per epilogue warp of the pair
  uint64_t mma_done;
  uint32_t tmem_base;
};

size_t gemm_smem_bytes() { return sizeof(GemmSmem) + 1024; }
static_assert(sizeof(GemmSmem) + 1024 <= 232448, "GEMM shared memory exceeds 227 KB");

struct GemmArgs {
  __nv_bfloat16* y;
  int64_t ldy;
  __nv_bfloat16* y2;   // columns >= n_main (second output group), or unused
  int64_t ldy2;
  int n_main;
  int M, N, K;
  int tiles_n, n_tiles;
  // RoPE epilogue: row m is token m % T of sequence m / T, at position
  // pos[m] if pos, else (len ? len[m / T] : 0) + m % T
  int rope_cols, T;
  const float2* rot;   // [M][R / 2] (cos, sin) of row m's position x frequency k
};

// Stores 32 columns (col0 ..) of this thread's row through the warp's staging
// area: each thread writes its row (16-byte chunks XOR-swizzled by row), then
// each store instruction covers 8 rows x 64 bytes.
__device__ __forceinline__ void store_cols32(const float (&v)[32], uint8_t* stg, int lane, int row0, int col0,
                                             const GemmArgs& g) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) w4[e] = pack_bf16(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
    *reinterpret_cast<uint4*>(stg + lane * 64 + 16 * (q ^ ((lane >> 1) & 3))) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  __syncwarp();
  const int rr = lane >> 2, ch = lane & 3;   // rows rr + 8 q, 16-byte chunk ch
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int rw = rr + 8 * q;
    const int row = row0 + rw, col = col0 + 8 * ch;
    const uint4 val = *reinterpret_cast<const uint4*>(stg + rw * 64 + 16 * (ch ^ ((rw >> 1) & 3)));
    if (row < g.M && col < g.N) {
      __nv_bfloat16* dst = col < g.n_main ? g.y + (int64_t)row * g.ldy + col
                                          : g.y2 + (int64_t)row * g.ldy2 + (col - g.n_main);
      *reinterpret_cast<uint4*>(dst) = val;
    }
  }
  __syncwarp();
}

template <int ROPE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_w2, GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair0 = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int k_blocks = (g.K + kGK - 1) / kGK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 8);
    }
    mbar_init(&sm.mma_done, 1);
    fence_barrier_init();
  }
  constexpr int R = ROPE == 1 ? 256 : 64;   // rotary dims of the layer type
  if (warp == 5) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // barriers of both CTAs initialised before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 4) {
    if (lane == 0) {
      // ======================= TMA producer (both CTAs) =======================
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_w);
      if (g.n_main < g.N) prefetch_tmap(&tm_w2);
      uint32_t it = 0;   // stages filled so far
      bool ok = true;
      for (int t = pair0; ok && t < g.n_tiles; t += n_pairs) {
        const int mt = t / g.tiles_n, nt = t % g.tiles_n;
        const bool second = nt * kGN >= g.n_main;   // a column tile of the second group
        const CUtensorMap* wmap = second ? &tm_w2 : &tm_w;
        const int wrow = (second ? nt * kGN - g.n_main : nt * kGN) + (int)rank * (kGN / 2);
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % kGStages;
          if (it >= kGStages && !(ok = mbar_wait(&sm.empty[s], ((it / kGStages) - 1) & 1))) break;
          if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 4 * kGHalf);
          tma_load_2d_pair(smem_u32(sm.x[s]), &tm_x, &sm.full[s], kb * kGK, mt * 2 * kGM + (int)rank * kGM);
          tma_load_2d_pair(smem_u32(sm.w[s]), wmap, &sm.full[s], kb * kGK, wrow);
        }
      }
      if (rank == 0)   // every load of the pair completes on CTA 0's barriers
        for (uint32_t i = (it > kGStages ? it - kGStages : 0); i < it; ++i)
          mbar_wait(&sm.full[i % kGStages], (i / kGStages) & 1);
    }
  } else if (warp == 5) {
    // ======================= MMA issuer (CTA 0, whole warp, one lane issues) =======================
    if (rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(2 * kGM, kGN, false);   // both operands K-major
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(sm.x[0]), 16, 1024);
      const uint64_t wdesc0 = smem_desc_sw128(smem_u32(sm.w[0]), 16, 1024);
      uint32_t it = 0, acc = 0;
      bool ok = true;
      for (int t = pair0; ok && t < g.n_tiles; t += n_pairs, ++acc) {
        const uint32_t b = acc & 1;
        if (acc >= 2 && !(ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_empty[b], ((acc >> 1) - 1) & 1)))) break;
        tc_fence_after();
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % kGStages;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[s], (it / kGStages) & 1)))) break;
          tc_fence_after();
          const uint64_t xd = desc_advance(xdesc0, s * kGHalf), wd = desc_advance(wdesc0, s * kGHalf);
#pragma unroll
          for (int k = 0; k < kGK / 16; ++k)
            mma_ss_pair_warp(tmem + b * kGN, desc_advance(xd, k * 32), desc_advance(wd, k * 32), idesc,
                             (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit_pair_warp(&sm.empty[s]);
        }
        if (ok) mma_commit_pair_warp(&sm.acc_full[b]);
      }
      // also on an early exit: wait until nothing the pair issued is in flight
      mma_commit_pair_warp(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ======================= epilogue (warps 0-3, both CTAs) =======================
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* stg = sm.ostage[warp];
    uint32_t acc = 0;
    bool ok = true;
    for (int t = pair0; ok && t < g.n_tiles; t += n_pairs, ++acc) {
      const int mt = t / g.tiles_n, nt = t % g.tiles_n;
      const uint32_t b = acc & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full[b], (acc >> 1) & 1)))) break;
      tc_fence_after();
      const int row0 = mt * 2 * kGM + (int)rank * kGM + warp * 32;   // this warp's first output row
      const bool rotate = ROPE != 0 && nt * kGN < g.rope_cols;      // the tile is one q or k head
      int first_plain = 0;                                            // chunks below were rotated
      if (rotate) {
        const int m = min(row0 + lane, g.M - 1);
        const float4* rot_row = reinterpret_cast<const float4*>(g.rot + (int64_t)m * (R / 2));
#pragma unroll 1
        for (int c = 0; c < R / 64; ++c) {   // dims [32c, 32c+32) against [R/2 + 32c, ...)
          uint32_t u1[32], u2[32];
          tmem_ld32(trow + b * kGN + 32 * c, u1);
          tmem_ld32(trow + b * kGN + R / 2 + 32 * c, u2);
          tmem_wait_ld();
          float a1[32], a2[32];
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) {
            const float4 t = __ldg(rot_row + 16 * c + i2);   // frequencies 32c + 2 i2, + 1
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int i = 2 * i2 + e;
              const float cs = e ? t.z : t.x, sn = e ? t.w : t.y;
              const float x = __uint_as_float(u1[i]), y = __uint_as_float(u2[i]);
              a1[i] = fmaf(x, cs, -y * sn);
              a2[i] = fmaf(y, cs, x * sn);
            }
          }
          store_cols32(a1, stg, lane, row0, nt * kGN + 32 * c, g);
          store_cols32(a2, stg, lane, row0, nt * kGN + R / 2 + 32 * c, g);
        }
        first_plain = R / 32;
      }
#pragma unroll 1
      for (int c = first_plain; c < kGN / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(trow + b * kGN + 32 * c, u);
        tmem_wait_ld();
        float a[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = __uint_as_float(u[i]);
        store_cols32(a, stg, lane, row0, nt * kGN + 32 * c, g);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&sm.acc_empty[b]);
        else mbar_arrive_remote(&sm.acc_empty[b], 0);
      }
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

int gemm_box_rows() { return kGM; }
int gemm_box_k() { return kGK; }

cudaError_t launch_gemm(const GemmHost& h, cudaStream_t st) {
  GemmArgs g;
  g.y = reinterpret_cast<__nv_bfloat16*>(h.y);
  g.ldy = h.ldy;
  g.y2 = reinterpret_cast<__nv_bfloat16*>(h.y2);
  g.ldy2 = h.ldy2;
  g.n_main = h.n_main > 0 ? h.n_main : h.N;
  if (g.n_main < h.N && (g.n_main % kGN != 0 || h.y2 == nullptr)) return cudaErrorInvalidValue;
  g.M = h.M;
  g.N = h.N;
  g.K = h.K;
  const int tiles_m = (h.M + 2 * kGM - 1) / (2 * kGM);
  g.tiles_n = (h.N + kGN - 1) / kGN;
  const long long n_tiles = (long long)tiles_m * g.tiles_n;
  if (n_tiles <= 0 || n_tiles > 0x3fffffffLL) return cudaErrorInvalidValue;
  g.n_tiles = (int)n_tiles;
  g.rope_cols = h.rope_cols;
  g.T = h.T > 0 ? h.T : 1;
  g.rot = reinterpret_cast<const float2*>(h.rot);
  if (h.rope != 0 && h.rot == nullptr) return cudaErrorInvalidValue;
  const long long grid = 2 * (n_tiles < h.n_pairs ? n_tiles : h.n_pairs);
  if (h.rope == 1)
    gemm_kernel<1><<<(unsigned)grid, kGThreads, gemm_smem_bytes(), st>>>(h.tm_x, h.tm_w, h.tm_w2, g);
  else if (h.rope == 2)
    gemm_kernel<2><<<(unsigned)grid, kGThreads, gemm_smem_bytes(), st>>>(h.tm_x, h.tm_w, h.tm_w2, g);
  else
    gemm_kernel<0><<<(unsigned)grid, kGThreads, gemm_smem_bytes(), st>>>(h.tm_x, h.tm_w, h.tm_w2, g);
  count_launch();
  return cudaGetLastError();
}

cudaError_t gemm_set_smem_attr() {
  const int smem = (int)gemm_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

}  // namespace hyb
