// Device-side helpers: token permutation index math and sm_100a PTX wrappers
// (mbarrier, TMA, tcgen05).  Included by the .cu files only.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rf_internal.h"

// ---------------------------------------------------------------------------
// Geometry on the device
// ---------------------------------------------------------------------------

// Sequence instance holding global query block `tb` (instances are few; a
// linear scan is cheaper than a table lookup through memory).
__device__ __forceinline__ int rf_seq_of_qblk(const RfGeomDev& g, int tb) {
  int s = 0;
#pragma unroll 1
  for (int i = 1; i < g.n_seqs; ++i)
    if (tb >= g.seq[i].qblk_off) s = i;
  return s;
}

// Element offset of (instance s, head n, row r) in a tensor with `heads` heads.
__device__ __forceinline__ size_t rf_row_offset(const RfGeomDev& g, const RfSeqDev& s, int heads,
                                                int n, int r) {
  if (g.layout == RF_LAYOUT_BNSD)
    return (((size_t)s.batch_idx * heads + n) * (size_t)s.L + (size_t)r) * (size_t)g.d;
  return (((size_t)s.row_off + (size_t)r) * heads + n) * (size_t)g.d;
}

// First row and row count of local block b (prefix blocks tile [0, Lp) with a
// possibly partial last block; sparse blocks tile [Lp, L) exactly).
__host__ __device__ __forceinline__ void rf_block_span(const RfSeqDev& s, int b, int& r0, int& nrows) {
  if (b < s.n_pb) {
    r0 = b * RF_BLOCK;
    nrows = (s.Lp - r0) < RF_BLOCK ? (s.Lp - r0) : RF_BLOCK;
  } else {
    r0 = s.Lp + (b - s.n_pb) * RF_BLOCK;
    nrows = RF_BLOCK;
  }
}

// Key/value blocks of 64 rows (blockShape 128 x 64): ceil(Lp / 64) prefix
// blocks from row 0 (the last may be partial), then 2 * nb blocks from row Lp.
__host__ __device__ __forceinline__ int rf_n_pb64(const RfSeqDev& s) { return (s.Lp + 63) >> 6; }
__host__ __device__ __forceinline__ void rf_kv64_span(const RfSeqDev& s, int b, int& r0, int& nrows) {
  const int n_pb = rf_n_pb64(s);
  if (b < n_pb) {
    r0 = 64 * b;
    nrows = s.Lp - r0 < 64 ? s.Lp - r0 : 64;
  } else {
    r0 = s.Lp + 64 * (b - n_pb);
    nrows = 64;
  }
}

// Original (input-order) row of rearranged row r of one sequence.
//   rearranged = [text | promoted | sparse]; the video part follows V', the
//   video tokens in tile order: aligned tokens by (frame, tile row, tile col,
//   row in tile, col in tile), then the ragged tokens in raster order.
//   With RF_ORDER_FRAME_PAIR the aligned frames 1..t-1 are taken in pairs
//   (xllm PR #1867, frame-pairing approach): frame 0 first, then each pair
//   cube by cube (tile row, tile col; frame in pair, row, col), then an
//   unpaired last frame in tile order.
//   Sparse rows are V'[0, S); promoted rows are V'[S, t*h*w).
__host__ __device__ __forceinline__ int rf_orig_row(const RfSeqDev& s, int r) {
  if (r < s.P) return r;
  int v = (r < s.Lp) ? (s.S + (r - s.P)) : (r - s.Lp);
  int y, x, f;
  if (v < s.A) {
    const int frame = s.h8 * s.w8;
    int rem;  // position of the token in its frame's single-frame tile order
    if (s.order == RF_ORDER_FRAME_PAIR && v >= frame && v < frame * (1 + 2 * ((s.t - 1) >> 1))) {
      // Frame pair (2m+1, 2m+2): cube c holds tile c of both frames, 64 rows each.
      const int u = v - frame;
      const int pair = u / (2 * frame);
      const int c = u - pair * 2 * frame;
      f = 1 + 2 * pair + ((c >> 6) & 1);
      rem = ((c >> 7) << 6) | (c & 63);
    } else {
      f = v / frame;
      rem = v - f * frame;
    }
    const int tile = rem >> 6, within = rem & 63;
    const int tiles_per_row = s.w8 >> 3;
    const int hb = tile / tiles_per_row, wb = tile - hb * tiles_per_row;
    y = (hb << 3) + (within >> 3);
    x = (wb << 3) + (within & 7);
  } else {
    const int q = v - s.A;
    const int per = s.h * s.w - s.h8 * s.w8;  // ragged tokens per frame (> 0 here)
    f = q / per;
    const int q2 = q - f * per;
    const int rw = s.w - s.w8;                 // ragged columns in the top h8 rows
    const int top = s.h8 * rw;
    if (q2 < top) {
      y = q2 / rw;
      x = s.w8 + (q2 - y * rw);
    } else {
      const int q3 = q2 - top;
      y = s.h8 + q3 / s.w;
      x = q3 - (y - s.h8) * s.w;
    }
  }
  return s.P + (f * s.h + y) * s.w + x;
}

// ---------------------------------------------------------------------------
// PTX wrappers (sm_100a)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t rf_smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t rf_globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One test of phase `parity`; the thread may be suspended in hardware (up to
// RF_SUSPEND_HINT_NS, or until the phase completes) instead of spinning, so a
// waiting warp does not take issue slots from the warps sharing its scheduler.
#ifndef RF_SUSPEND_HINT_NS
#define RF_SUSPEND_HINT_NS 1000000u
#endif
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
#if RF_SUSPEND_HINT_NS > 0
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(RF_SUSPEND_HINT_NS)
      : "memory");
#else
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
#endif
  return ok != 0;
}

// One test of phase `parity` without a suspend hint: the thread polls.
__device__ __forceinline__ bool mbar_try_wait_poll(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// One non-blocking test of phase `parity` (mbarrier.test_wait).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of barrier `bar` to complete, for at most
// RF_WAIT_LIMIT_NS; gives up early once *abort is set.  Returns false when it
// gave up (the caller records it and unwinds).  kPoll: poll without the
// suspend hint (for a warp whose wake-up latency is on the critical path).
#define RF_WAIT_LIMIT_NS 1000000000ull
template <bool kPoll = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
#ifdef RF_POLL_TEST_WAIT
  auto test = [&]() { return kPoll ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity); };
#else
  auto test = [&]() { return kPoll ? mbar_try_wait_poll(bar, parity) : mbar_try_wait(bar, parity); };
#endif
  if (test()) return true;
  const uint64_t t0 = rf_globaltimer();
#pragma unroll 1
  for (;;) {
    if (test()) return true;
    if (*abort) return false;
    if (rf_globaltimer() - t0 > RF_WAIT_LIMIT_NS) return false;
  }
}

__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 3-D tiled TMA load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// True on one lane of the (fully active) warp: the lowest one, every time.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 l;\n\t"
      "elect.sync l|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16, fp32 accumulate.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f8f6f4 (E4M3 operands per
// the instruction descriptor), fp32 accumulate.
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16, fp32 accumulate.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f8f6f4 (E4M3 operands per the
// instruction descriptor; A packed four per 32-bit column), fp32 accumulate.
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// Register re-allocation between warpgroups (all warps of a warpgroup execute it).
template <uint32_t kRegs>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <uint32_t kRegs>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float rf_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA and integer pipes, for the share of the softmax
// exponentials taken off the MUFU unit.  Range reduction: x = j + r with
// j = round(x) (adding 1.5 * 2^23 leaves round(x) in the low mantissa bits)
// and r in [-1/2, 1/2]; 2^r from a degree-3 polynomial with p(0) = 1 whose
// coefficients were fitted for minimum relative error on [-1/2, 1/2] by
// csrc/gen_exp2_poly.py (max relative error 1.8e-4 in fp32); 2^j is added to
// the exponent field.  x is clamped at -125.5 so the result stays a normal
// number (2^-125.5 instead of 0 for smaller inputs; irrelevant next to the
// row maximum, whose exponential is >= 2^-8 here).
__device__ __forceinline__ float rf_exp2_poly(float x) {
  constexpr float kShifter = 12582912.0f;  // 1.5 * 2^23
  constexpr float kC1 = 0.6933164596557617f, kC2 = 0.24192412197589874f,
                  kC3 = 0.054602622985839844f;
  x = fmaxf(x, -125.5f);
  const float t = x + kShifter;
  const float r = x - (t - kShifter);
  const int j = __float_as_int(t) - __float_as_int(kShifter);
  float p = fmaf(kC3, r, kC2);
  p = fmaf(p, r, kC1);
  p = fmaf(p, r, 1.0f);
  return __int_as_float(__float_as_int(p) + (j << 23));
}

// Paired fp32 arithmetic (sm_100): two lanes of work per instruction.
__device__ __forceinline__ uint64_t rf_f2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ void rf_f2_split(uint64_t v, float& lo, float& hi) {
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
  lo = __uint_as_float(a);
  hi = __uint_as_float(b);
}
__device__ __forceinline__ uint64_t rf_fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t rf_mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t rf_add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float rf_max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x of two values at once, with the range reduction and polynomial of
// rf_exp2_poly run as paired fp32 instructions (one f32x2 instruction per step
// for both values): x = j + r with j = round(x) from the 1.5 * 2^23 shifter,
// 2^r from the same degree-3 polynomial, 2^j added to the exponent field.
// With t = x + 1.5 * 2^23 rounded to an integer, the bits of t are
// 0x4B400000 + j, and (bits << 23) is j << 23 modulo 2^32 because the low nine
// bits of 0x4B400000 are zero: one shift and one add reassemble the result.
// Inputs are clamped at -125.5 as in rf_exp2_poly.
__device__ __forceinline__ void rf_exp2_poly2(float x0, float x1, float& y0, float& y1) {
  constexpr float kShifter = 12582912.0f;  // 1.5 * 2^23
  constexpr float kC1 = 0.6933164596557617f, kC2 = 0.24192412197589874f,
                  kC3 = 0.054602622985839844f;
  x0 = fmaxf(x0, -125.5f);
  x1 = fmaxf(x1, -125.5f);
  const uint64_t x = rf_f2(__float_as_uint(x0), __float_as_uint(x1));
  const uint64_t sh = rf_f2(__float_as_uint(kShifter), __float_as_uint(kShifter));
  const uint64_t nsh = rf_f2(__float_as_uint(-kShifter), __float_as_uint(-kShifter));
  const uint64_t m1 = rf_f2(__float_as_uint(-1.0f), __float_as_uint(-1.0f));
  const uint64_t t = rf_add2(x, sh);                 // j in the low mantissa bits
  const uint64_t r = rf_fma2(rf_add2(t, nsh), m1, x);  // x - j, exact
  uint64_t p = rf_fma2(rf_f2(__float_as_uint(kC3), __float_as_uint(kC3)), r,
                       rf_f2(__float_as_uint(kC2), __float_as_uint(kC2)));
  p = rf_fma2(p, r, rf_f2(__float_as_uint(kC1), __float_as_uint(kC1)));
  p = rf_fma2(p, r, rf_f2(__float_as_uint(1.0f), __float_as_uint(1.0f)));
  uint32_t t0, t1, p0, p1;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(t0), "=r"(t1) : "l"(t));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(p0), "=r"(p1) : "l"(p));
  y0 = __uint_as_float(p0 + (t0 << 23));
  y1 = __uint_as_float(p1 + (t1 << 23));
}

// Two floats to packed 16-bit (lo = a, hi = b), round to nearest even.
template <bool kBf16>
__device__ __forceinline__ uint32_t rf_pack2(float a, float b) {
  uint32_t r;
  if (kBf16)
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  else
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// ---------------------------------------------------------------------------
// MXFP4: E2M1 elements (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) sharing one
// power-of-two scale per group of 32 (MXAttention abstract: MXFP4 attention
// with Universal Optimal Scaling, boundary Qmax = 7.25).
// ---------------------------------------------------------------------------
constexpr float kMxQmax = 7.25f;
constexpr float kMxLog2Qmax = 2.857980995127572f;  // log2(7.25)

// Two floats rounded to E2M1 (nearest, ties to the even code, saturating at
// +-6), returned as the exact f16 values of the two codes: a in the low half.
__device__ __forceinline__ uint32_t rf_e2m1x2_round(float a, float b) {
  uint32_t r;
  asm("{\n\t.reg .b8 c;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c, %1, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
      : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// ceil(log2(t)) for finite t > 0, from the bits (subnormals scaled up first).
__device__ __forceinline__ int rf_ceil_log2(float t) {
  int off = 0;
  if (t < 1.17549435e-38f) {
    t *= 18446744073709551616.0f;  // 2^64, exact
    off = 64;
  }
  const uint32_t b = __float_as_uint(t);
  return (int)(b >> 23) - 127 + ((b & 0x7FFFFFu) != 0u ? 1 : 0) - off;
}

// 2^k as a float, -126 <= k <= 127.
__device__ __forceinline__ float rf_pow2(int k) { return __int_as_float((127 + k) << 23); }

// x * 2^k for |k| <= 252, as two exact power-of-two products.
__device__ __forceinline__ float rf_scale_pow2(float x, int k) {
  const int k1 = k / 2;
  return x * rf_pow2(k1) * rf_pow2(k - k1);
}

// UOS shared exponent of a group whose largest magnitude is amax: the
// smallest e with amax <= 7.25 * 2^e (0 for an all-zero group).  amax / 7.25
// is a correctly rounded division, so a boundary value 7.25 * 2^k gives k.
__device__ __forceinline__ int rf_uos_exponent(float amax) {
  return amax > 0.f ? rf_ceil_log2(__fdiv_rn(amax, kMxQmax)) : 0;
}

// ---------------------------------------------------------------------------
// UMMA (tcgen05) descriptors
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor for a 128-byte-swizzled tile (1024-byte
// aligned atoms of 8 rows x 128 bytes).  lbo/sbo in bytes.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16 with fp32 accumulation.
//   fmt: 0 = f16, 1 = bf16; b_mn_major: B operand stored N-contiguous.
__host__ __device__ constexpr uint32_t umma_idesc_f16(uint32_t fmt, uint32_t m, uint32_t n,
                                                      uint32_t b_mn_major) {
  return (1u << 4)             // D format: f32
         | (fmt << 7)          // A format
         | (fmt << 10)         // B format
         | (0u << 15)          // A K-major
         | (b_mn_major << 16)  // B major
         | ((n >> 3) << 17) | ((m >> 4) << 24);
}
