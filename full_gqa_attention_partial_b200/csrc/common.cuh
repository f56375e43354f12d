// Shared device helpers of the hybrid attention kernels: model constants,
// RoPE angles, mbarrier / TMA / tcgen05 wrappers in inline PTX, and the
// per-device error word.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace hyb {

constexpr int kHq = 16;      // query heads
constexpr int kHkv = 4;      // KV heads
constexpr int kGroup = 4;    // query heads per KV head
constexpr int kD = 256;      // head dim
constexpr int kWindow = 512; // sliding window (keys incl. the query itself)

// RoPE per layer type: sliding theta 1e4 over all 256 dims, full theta 5e6
// over the first 64 dims (partial_rotary_factor 0.25).
template <bool FULL> struct RopeCfg;
template <> struct RopeCfg<false> { static constexpr int R = 256; static constexpr double theta = 1.0e4; };
template <> struct RopeCfg<true>  { static constexpr int R = 64;  static constexpr double theta = 5.0e6; };

// Error word shared by all kernels of the library on one device.  The
// library is built as one translation unit (hyb_attn_lib.cu), so this single
// definition is the one every kernel and the host accessor see.
static __device__ int g_dev_err = 0;
constexpr int kErrCapacity = 1;
constexpr int kErrTimeout = 2;
constexpr int kErrPage = 4;
constexpr int kErrBounds = 8;

__device__ __forceinline__ void raise_err(int bit) { atomicOr(&g_dev_err, bit); }

// Index checks of the debug build (-DHYB_DEBUG_BOUNDS): HYB_BOUNDS(i, lo, hi)
// is true when lo <= i < hi; otherwise it raises kErrBounds and is false, and
// the caller skips the access (nothing traps, no CTA leaves a barrier early).
// In the normal build it is the constant true and the check compiles away.
#ifdef HYB_DEBUG_BOUNDS
__device__ __forceinline__ bool hyb_in_bounds(int64_t i, int64_t lo, int64_t hi) {
  if (i >= lo && i < hi) return true;
  raise_err(kErrBounds);
  return false;
}
#define HYB_BOUNDS(i, lo, hi) (::hyb::hyb_in_bounds((int64_t)(i), (int64_t)(lo), (int64_t)(hi)))
constexpr int kBuildFlags = 1;
#else
#define HYB_BOUNDS(i, lo, hi) true
constexpr int kBuildFlags = 0;
#endif

// Row and batch coordinates of key row `row` of sequence b in a cache's TMA
// map: the identity for contiguous caches; for paged caches the row within
// the page and the pool page from the block table.  A table entry outside
// the pool (or a row past the table) raises kErrPage and returns the page
// coordinate -1, where tensor-map loads read zeros.  Rows of one 64-row
// tile share a page (the page size is a multiple of 64).
__device__ __forceinline__ void kv_coord(const PageMap& pm, int b, int row, int& crow, int& cpage) {
  if (pm.page == 0) {
    crow = row;
    cpage = b;
    return;
  }
  const int lp = row / pm.page;
  int pp = -1;
  if (lp < pm.max_pages) pp = __ldg(pm.table + (int64_t)b * pm.max_pages + lp);
  if (pp < 0 || pp >= pm.n_pages) {
    raise_err(kErrPage);
    pp = -1;
  }
  crow = row - lp * pm.page;
  cpage = pp;
}

// ---------------------------------------------------------------------------
// RoPE angle: phi = pos * inv_freq in fp64, reduced to [-pi, pi] with a
// two-term 2*pi (Cody-Waite style reduction), then sin/cos of the reduced
// angle on the special-function unit (__sincosf: absolute error ~5e-7 on
// [-pi, pi], far below bf16 resolution).  fp32 pos * inv_freq alone would be
// off by ~0.06 rad at pos ~ 2^20.
// ---------------------------------------------------------------------------
// Rotation frequencies inv_freq_k = theta^(-2k/R), k < R/2, of both layer
// types: [0][k] sliding (R = 256, theta 1e4), [1][k] full (R = 64, theta 5e6).
// Computed once per device on the host (fp64) and copied in when the device
// is set up, so that no kernel evaluates pow() itself.
static __device__ double g_inv_freq[2][128];
template <bool FULL>
__device__ __forceinline__ double rope_inv_freq(int k) {
  return __ldg(&g_inv_freq[FULL ? 1 : 0][k]);
}

__device__ __forceinline__ void rope_sincos(int pos, double inv_freq, float* s, float* c) {
  const double two_pi_hi = 6.283185307179586232;      // nearest double to 2*pi
  const double two_pi_lo = 2.4492935982947064e-16;    // 2*pi - two_pi_hi
  const double inv_two_pi = 0.15915494309189533577;
  double phi = (double)pos * inv_freq;
  double n = rint(phi * inv_two_pi);
  double r = fma(-n, two_pi_hi, phi);
  r = fma(-n, two_pi_lo, r);
  __sincosf((float)r, s, c);
}

// 2^x on the special-function unit (flush-to-zero; x <= 8 here)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// sin / cos of x = delta * inv_freq for a small integer delta (|x| <~ 2^8):
// fp32 product, reduction with a two-term fp32 2*pi, then the SFU.
__device__ __forceinline__ void small_angle_sincos(int delta, float inv_freq_f, float* s, float* c) {
  const float x = (float)delta * inv_freq_f;
  const float n = rintf(x * 0.159154943f);
  float r = fmaf(-n, 6.28318548f, x);     // 2*pi rounded to fp32 ...
  r = fmaf(-n, -1.74845553e-7f, r);       // ... and the rest of 2*pi
  __sincosf(r, s, c);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel of its stream is still
// running: pdl_wait() blocks until that kernel has completed and its memory
// is visible, so everything before it must not read what the previous
// kernel writes.  pdl_launch_dependents() lets the next kernel start its own
// launch early.  Without the launch attribute both are no-ops.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// bf16 packing
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers (with bounded waits)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase of `parity` to complete.  Gives up after ~2 s of
// wall time, raises kErrTimeout and returns false: callers then skip the
// rest of their work so that the kernel always terminates.  Once some wait
// on the device has timed out, other waits give up after 1 ms instead, so a
// broken launch drains quickly.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kWaitLimitAfterErrNs = 1000000ull;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u) {
      const uint64_t dt = globaltimer_ns() - t0;
      const bool err = (*reinterpret_cast<volatile int*>(&g_dev_err) & kErrTimeout) != 0;
      if (dt > kWaitLimitNs || (err && dt > kWaitLimitAfterErrNs)) {
        raise_err(kErrTimeout);
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// TMA: 4-D tiled load into shared memory, completion counted on an mbarrier.
// No multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(uint32_t smem_dst, const void* tmap, uint64_t* bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}
// TMA: 3-D tiled load (no swizzle maps, e.g. per-row scales).
__device__ __forceinline__ void tma_load_3d(uint32_t smem_dst, const void* tmap, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// e4m3 -> bf16 by integer bit moves, scaled by 2^-120: the e4m3 sign,
// exponent and mantissa bits land in the bf16 sign, the low four exponent
// bits and the top three mantissa bits, so the code 2^(e-7) (1 + m/8) becomes
// the bf16 2^(e-127) (1 + m/8) and the subnormal code m 2^-9 the bf16
// subnormal m 2^-129, both exact.  Three instructions for two codes: a byte
// permute puts each code in a 16-bit half with its sign bit copied over the
// high byte, a shift by 4 moves sign and magnitude into place, and a mask
// clears the copies and what the low half shifted into the high one.
// A word of four codes (byte 0 lowest) gives two bf16 pairs (low half first).
template <uint32_t SEL>
__device__ __forceinline__ uint32_t e4m3_pair_bf16x2(uint32_t w) {
  return (prmt(w, 0u, SEL) << 4) & 0x87F087F0u;
}
__device__ __forceinline__ uint32_t e4m3_b01_bf16x2(uint32_t w) { return e4m3_pair_bf16x2<0x9180u>(w); }
__device__ __forceinline__ uint32_t e4m3_b23_bf16x2(uint32_t w) { return e4m3_pair_bf16x2<0xB3A2u>(w); }
__device__ __forceinline__ uint32_t e4m3_b02_bf16x2(uint32_t w) { return e4m3_pair_bf16x2<0xA280u>(w); }
__device__ __forceinline__ uint32_t e4m3_b13_bf16x2(uint32_t w) { return e4m3_pair_bf16x2<0xB391u>(w); }
// The same for one code of each of two words a and b (the permute numbers
// a's bytes 0-3 and b's 4-7): e.g. 0xC480 gives (a byte 0, b byte 0), so a
// pair of codes from two key rows costs no extra permute.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t e4m3_pair2_bf16x2(uint32_t a, uint32_t b) {
  return (prmt(a, b, SEL) << 4) & 0x87F087F0u;
}
// Two floats -> two e4m3 codes (lo in the low byte), round to nearest even, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
  return h;
}
// Two e4m3 codes (low byte first) -> their values (exact).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t c) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"((uint16_t)c));
  return __half22float2(*reinterpret_cast<const __half2*>(&d));
}
constexpr float kE4m3WideScale = 1.329227995784916e36f;   // 2^120
constexpr float kE4m3PScale = 18446744073709551616.f;      // 2^64
constexpr float kE4m3OutScale = 72057594037927936.f;       // 2^56

// TMA: 4-D tiled store from shared memory (bulk group); rows outside the
// tensor are not written.
__device__ __forceinline__ void tma_store_4d(const void* tmap, uint32_t smem_src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(tmap),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_src)
               : "memory");
}
__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until every committed bulk store has finished reading its shared-memory source.
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void tma_store_commit_and_wait() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group 0;" ::: "memory");
}
// Prefetch of a 4-D tile into L2 (no shared-memory destination, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_4d(const void* tmap, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(tmap), "r"(c0),
               "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters (CTA pairs)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The two halves of cluster_sync, for work in between (every thread of the
// cluster arrives once, then waits; the warp converged at each).
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// shared::cluster address of the same shared-memory offset in CTA `cta`
__device__ __forceinline__ uint32_t mapa_cluster(uint32_t local_saddr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_saddr), "r"(cta));
  return r;
}
// arrive on the barrier at this offset in CTA `cta` of the cluster
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* bar, uint32_t cta) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(mapa_cluster(smem_u32(bar), cta)) : "memory");
}
// TMA load for a CTA pair: lands in this CTA's shared memory, and its bytes
// are counted on the barrier at `bar`'s offset in CTA 0 of the pair.  No
// multicast.
__device__ __forceinline__ void tma_load_4d_pair(uint32_t smem_dst, const void* tmap, uint64_t* bar, int c0,
                                                 int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(mapa_cluster(smem_u32(bar), 0))
      : "memory");
}

// The same for a 2-D map.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t smem_dst, const void* tmap, uint64_t* bar, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(mapa_cluster(smem_u32(bar), 0))
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// CTA-pair forms: both CTAs of the pair execute alloc / relinquish / dealloc
// from the same warp.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Pair MMA, issued by one thread of CTA 0: D (M = 256 rows, 128 in each CTA's
// tensor memory) (+)= A (each CTA's own 128 rows, from its tensor memory) *
// B (N/2 columns from each CTA's shared memory, same offsets).
__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on the barrier at `bar`'s offset in both CTAs of the pair when
// every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
// Warp-collective forms: the whole warp executes them with warp-uniform
// operands and one elected lane issues.  Keeping the issuing loop convergent
// lets the operands stay warp-uniform, which issues an MMA every ~50 cycles
// instead of ~130 from a lone diverged lane.
__device__ __forceinline__ void mma_ts_pair_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// As mma_ts_pair_warp, with A (K-major, 128-byte swizzle) in shared memory:
// each CTA of the pair supplies its own 128 rows of A from the same offset.
__device__ __forceinline__ void mma_ss_pair_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// As mma_ss_pair_warp on e4m3 operands (kind::f8f6f4, 32 elements of K per MMA:
// in a 128-byte-swizzled K-major operand the same 32 bytes per step as bf16's 16).
__device__ __forceinline__ void mma_ss_pair_e4m3_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                      uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Stores to the shared memory of another CTA of the cluster.
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float x) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(x) : "memory");
}
__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float x, float y) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}
__device__ __forceinline__ void st_cluster_f32x4(uint32_t addr, float x, float y, float z, float w) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(x), "f"(y), "f"(z), "f"(w)
               : "memory");
}
// Orders this thread's earlier memory writes before its later ones for every
// thread of the cluster.
__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }
__device__ __forceinline__ void mma_commit_pair_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]   (kind::f16, bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (format 0), fp32 D, dense
// (the bit fields of the kind::f16 descriptor below).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor, kind::f16: bf16 A/B, fp32 D, dense.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format,
//   15 A major (0 = K), 16 B major (1 = MN), 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   bits 0-13 start >> 4, 16-29 leading byte offset >> 4, 32-45 stride byte
//   offset >> 4, 46-47 version 1, 61-63 layout (2 = SWIZZLE_128B).
// K-major: rows of 128 B (64 bf16 of K), 8-row atoms of 1024 B -> SBO = 1024.
// MN-major: 128 B along MN per K row, 8 K rows per atom -> SBO = 1024 (next
// 8 K rows), LBO = distance to the next 64-element MN chunk.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// The same descriptor `bytes` further on (bytes a multiple of 16, the operand
// inside shared memory, so the start-address field cannot overflow): one
// 32-bit add, which keeps the MMA issue loop short -- with N = 64 the issuing
// warp, not the tensor core, limited the rate when every descriptor was
// rebuilt from its address.
__device__ __forceinline__ uint64_t desc_advance(uint64_t desc, uint32_t bytes) {
  const uint32_t lo = (uint32_t)desc + (bytes >> 4);
  return ((desc >> 32) << 32) | lo;
}

// tcgen05.ld / st, 32 lanes x 32 bit: thread i of the warp gets lane
// (warp % 4) * 32 + i, `N` consecutive columns.
template <int N> struct TmemLd;
#define HYB_TMEM_REGS16(a, o)                                                                      \
  "=r"(a[o + 0]), "=r"(a[o + 1]), "=r"(a[o + 2]), "=r"(a[o + 3]), "=r"(a[o + 4]), "=r"(a[o + 5]), \
      "=r"(a[o + 6]), "=r"(a[o + 7]), "=r"(a[o + 8]), "=r"(a[o + 9]), "=r"(a[o + 10]),             \
      "=r"(a[o + 11]), "=r"(a[o + 12]), "=r"(a[o + 13]), "=r"(a[o + 14]), "=r"(a[o + 15])
#define HYB_TMEM_IREGS16(a, o)                                                                   \
  "r"(a[o + 0]), "r"(a[o + 1]), "r"(a[o + 2]), "r"(a[o + 3]), "r"(a[o + 4]), "r"(a[o + 5]),      \
      "r"(a[o + 6]), "r"(a[o + 7]), "r"(a[o + 8]), "r"(a[o + 9]), "r"(a[o + 10]), "r"(a[o + 11]), \
      "r"(a[o + 12]), "r"(a[o + 13]), "r"(a[o + 14]), "r"(a[o + 15])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
      "[%32];"
      : HYB_TMEM_REGS16(r, 0), HYB_TMEM_REGS16(r, 16)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : HYB_TMEM_REGS16(r, 0)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32};" ::"r"(taddr),
      HYB_TMEM_IREGS16(r, 0), HYB_TMEM_IREGS16(r, 16)
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16};" ::"r"(taddr),
      HYB_TMEM_IREGS16(r, 0)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Legacy warp-level MMA and ldmatrix (used by the HBM-bound decode kernel)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(saddr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(saddr));
}
// D = A(16x16, rows g and g+8) * B(16x8) + C, bf16 in, fp32 accumulate
// (registers only, so the compiler may schedule it freely).
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Transpose of an 8x8 b16 matrix held one row per 4 lanes (two elements each).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(x));
  return d;
}

// Byte offset of element (row, col) inside a TMA box of 128-byte rows with
// SWIZZLE_128B: the 16-byte chunk index is XORed with (row % 8).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t byte_in_row) {
  return row * 128u + ((((byte_in_row >> 4) ^ (row & 7u)) << 4) | (byte_in_row & 15u));
}

}  // namespace hyb
