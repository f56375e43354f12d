// Projections of a decode step (q_k_v_proj with the gate rows, o_proj of
// "百万 Token 塞进 4B ..." §"省显存的第二板斧") for a few rows:
//   Y[M, N] = X[M, K] W[N, K]^T,  M <= 16 (one token per sequence),
// bf16 in and out, fp32 accumulation.  With M this small the work is
// reading W once (N x K bf16: 31.5 MB for q_k_v_proj, 21 MB for o_proj),
// so the kernel is built to stream W from HBM on every SM, not around the
// tensor cores: the 256-row tiles of the prefill GEMM would be 94 % empty
// and its 25 column tiles could keep only 50 SMs busy.
//
// A cluster of S CTAs (S = K / 512) owns 32 output features: CTA r reads
// K columns [512 r, 512 r + 512) of those 32 rows of W (32 KB) straight
// into registers (16-byte loads, 64 contiguous bytes per row per four
// lanes), multiplies them by X's 16 x 512 slice from shared memory with
// mma.sync m16n8k16 (each warp 8 features); every CTA stores its partial
// tile into CTA 0's shared memory (distributed shared memory, plain stores),
// and after one cluster barrier CTA 0 sums the S tiles in rank order (the
// result does not depend on timing) and writes Y.  When
// the caller knows that the kernel launched just before does not write W
// (o_proj after the library's own attention), W's loads are issued before
// the wait for that kernel, so the weight stream overlaps its tail.
//
// The MMA fragments take the K dims of a 32-wide chunk in a permuted order,
// the same for X and W (a dot product does not depend on the order of its
// terms): thread (g, t) of a warp (g = lane / 4, t = lane % 4) holds the 8
// consecutive dims 8 t .. 8 t + 7 of W's row g, and of those, dims 8 t + 4 j
// .. + 3 feed step j (0, 1) as the fragment's k = 2 t, 2 t + 1, 2 t + 8,
// 2 t + 9; X is read at the same dims.
#include "common.cuh"
#include "launch.h"

namespace hyb {

constexpr int kSmmWarps = 4;
constexpr int kSmmFeat = 8 * kSmmWarps;   // output features per cluster
constexpr int kSmmK = 512;                // K columns per CTA
constexpr int kSmmChunks = kSmmK / 32;    // 32-wide K chunks per CTA
constexpr int kSmmPad = 8;                // X row padding (elements)
constexpr int kSmmMaxS = 8;               // cluster size limit (portable)

struct SmallMArgs {
  const __nv_bfloat16* x;
  int64_t ldx;
  const __nv_bfloat16* w;
  int64_t ldw;
  const __nv_bfloat16* w2;   // rows of features n_main .. N - 1, or unused
  int64_t ldw2;
  __nv_bfloat16* y;
  int64_t ldy;
  __nv_bfloat16* y2;         // features n_main .. N - 1, or unused
  int64_t ldy2;
  int n_main, M, N, K, S;
  int early_w;   // 1: W may be read before the previous kernel has finished
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(32 * kSmmWarps, 5) smallm_kernel(SmallMArgs a) {
  __shared__ __align__(16) __nv_bfloat16 xs[16][kSmmK + kSmmPad];
  __shared__ __align__(16) float part[kSmmMaxS][16][kSmmFeat];   // CTA 0's: the partial tile of every rank
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rank = blockIdx.x % a.S;        // the cluster's CTAs are consecutive in x
  const int n0 = (blockIdx.x / a.S) * kSmmFeat;
  const int k0 = rank * kSmmK;

  // ---- this thread's W: feature n, dims k0 + 32 c + 8 t .. + 7 of every chunk c ----
  const int n = n0 + 8 * warp + g;
  if (!a.early_w) pdl_wait();
  uint4 wr[kSmmChunks];
  if (n < a.N && HYB_BOUNDS(k0 + kSmmK, 1, a.K + 1)) {
    const __nv_bfloat16* row = n < a.n_main ? a.w + (int64_t)n * a.ldw : a.w2 + (int64_t)(n - a.n_main) * a.ldw2;
#pragma unroll
    for (int c = 0; c < kSmmChunks; ++c) wr[c] = ld_stream_v4(row + k0 + 32 * c + 8 * t);
  } else {
#pragma unroll
    for (int c = 0; c < kSmmChunks; ++c) wr[c] = make_uint4(0, 0, 0, 0);
  }
  if (a.early_w) pdl_wait();   // X comes from the previous kernel
  pdl_launch_dependents();

  // ---- X's 16 x 512 slice (rows past M are zero): every load in flight at once ----
  constexpr int kXPer = 16 * (kSmmK / 8) / (32 * kSmmWarps);
  uint4 xv[kXPer];
#pragma unroll
  for (int j = 0; j < kXPer; ++j) {
    const int i = threadIdx.x + j * 32 * kSmmWarps;
    const int m = i / (kSmmK / 8), c8 = i % (kSmmK / 8);
    xv[j] = m < a.M ? *reinterpret_cast<const uint4*>(a.x + (int64_t)m * a.ldx + k0 + 8 * c8) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int j = 0; j < kXPer; ++j) {
    const int i = threadIdx.x + j * 32 * kSmmWarps;
    *reinterpret_cast<uint4*>(&xs[i / (kSmmK / 8)][8 * (i % (kSmmK / 8))]) = xv[j];
  }
  __syncthreads();

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < kSmmChunks; ++c) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int kk = 32 * c + 8 * t + 4 * j;
      const uint2 lo = *reinterpret_cast<const uint2*>(&xs[g][kk]);       // rows g: (a0, a2)
      const uint2 hi = *reinterpret_cast<const uint2*>(&xs[g + 8][kk]);   // rows g + 8: (a1, a3)
      const uint32_t b0 = j ? wr[c].z : wr[c].x, b1 = j ? wr[c].w : wr[c].y;
      mma_16816(acc, lo.x, hi.x, lo.y, hi.y, b0, b1);
    }
  }
  // acc: rows g and g + 8, features 8 warp + 2 t, + 1 -> CTA 0's part[rank]
  st_cluster_f32x2(mapa_cluster(smem_u32(&part[rank][g][8 * warp + 2 * t]), 0), acc[0], acc[1]);
  st_cluster_f32x2(mapa_cluster(smem_u32(&part[rank][g + 8][8 * warp + 2 * t]), 0), acc[2], acc[3]);
  cluster_sync();   // every rank's tile is in CTA 0 (release / acquire); CTA 0 alone reads on
  if (rank == 0) {
    for (int i = threadIdx.x; i < 16 * kSmmFeat / 2; i += blockDim.x) {
      const int m = i / (kSmmFeat / 2), f = 2 * (i % (kSmmFeat / 2));
      const int nn = n0 + f;
      if (m >= a.M || nn >= a.N) continue;
      float s0 = 0.f, s1 = 0.f;
      for (int r = 0; r < a.S; ++r) {   // rank order
        const float2 v = *reinterpret_cast<const float2*>(&part[r][m][f]);
        s0 += v.x;
        s1 += v.y;
      }
      __nv_bfloat16* dst = nn < a.n_main ? a.y + (int64_t)m * a.ldy + nn : a.y2 + (int64_t)m * a.ldy2 + (nn - a.n_main);
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16(s0, s1);
    }
  }
}

bool smallm_supported(int M, int N, int K, int n_main) {
  return M >= 1 && M <= 16 && K % kSmmK == 0 && K / kSmmK >= 1 && K / kSmmK <= kSmmMaxS && N % 8 == 0 &&
         n_main % 2 == 0;
}

cudaError_t launch_smallm(const SmallMHost& h, cudaStream_t st) {
  SmallMArgs a;
  a.x = reinterpret_cast<const __nv_bfloat16*>(h.x);
  a.ldx = h.ldx;
  a.w = reinterpret_cast<const __nv_bfloat16*>(h.w);
  a.ldw = h.ldw;
  a.w2 = reinterpret_cast<const __nv_bfloat16*>(h.w2 ? h.w2 : h.w);
  a.ldw2 = h.w2 ? h.ldw2 : h.ldw;
  a.y = reinterpret_cast<__nv_bfloat16*>(h.y);
  a.ldy = h.ldy;
  a.y2 = reinterpret_cast<__nv_bfloat16*>(h.y2 ? h.y2 : h.y);
  a.ldy2 = h.y2 ? h.ldy2 : h.ldy;
  a.n_main = h.n_main > 0 ? h.n_main : h.N;
  a.M = h.M;
  a.N = h.N;
  a.K = h.K;
  a.S = h.K / kSmmK;
  a.early_w = h.early_w ? 1 : 0;
  if (!smallm_supported(h.M, h.N, h.K, a.n_main)) return cudaErrorInvalidValue;
  const int clusters = (h.N + kSmmFeat - 1) / kSmmFeat;
  const cudaError_t e = launch_pdl(smallm_kernel, dim3(clusters * a.S, 1, 1), dim3(32 * kSmmWarps, 1, 1), 0, st,
                                   (unsigned)a.S, a);
  count_launch();
  return e;
}

}  // namespace hyb
