// Block-sparse flash attention on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "aclnnRainFusionAttention" API page, "Formula": attentionOut =
// Softmax(scale * query * key^T + atten_mask) * value with the key/value
// blocks of each query block listed in selectIdx (first selectNum entries,
// -1 = unused slot), fp32 softmax (inner precise mode 0), TND and BNSD
// layouts, N1 = G * N2 grouped heads, deterministic.  There is no user mask
// ("RainFusion Attention" user guide, "Geometry handling": no padding mask is
// consumed); the only masked keys are the rows past the dense prefix in its
// last, partial block.
//
// One CTA = one (query block of 128 rows, query head); CTAs are ordered
// head-major so that the K/V of a head (or of a GQA group) stay in L2 while
// its query blocks run, and within a head the dense query blocks (prefix,
// first frame) come first.
//
// Warp roles (384 threads = three warpgroups):
//   warps 0-3  softmax group 0: the even-numbered selected blocks
//   warps 4-7  softmax group 1: the odd-numbered selected blocks
//              (thread = query row = TMEM lane in both groups)
//   warp 8     TMA producer of Q (once) and K_j through a 3-stage ring
//   warp 9     TMEM allocation and the tcgen05.mma issue of S_j = Q K_j^T
//   warp 10    TMA producer of V_j through a 2-stage ring (3 stages with
//              one-byte Q and K, 4 with one-byte V); K and V have separate
//              producers so that a K load never queues behind a V load that
//              waits for an earlier P V product
//   warp 11    the tcgen05.mma issue of O_w += P_j V_j
// One elected thread per issuing warp issues that warp's MMAs.  A single
// issuing thread cannot keep the tensor pipe busy at M = N = 128: every
// barrier check costs it about as much as an MMA's worth of pipe time.
// The kernel launches with 168 registers per thread; the third warpgroup
// gives registers back (72 each) and the softmax groups take them (216 each),
// so that a thread holds its whole 128-column score row: 2*128*216 + 128*72
// = 384*168.
// TMEM columns: one score buffer S at [0, 128); P of group w at
// [128 + 64 w, +64) (128 keys as packed 16-bit pairs, or 32 columns of four
// E4M3 codes); O_w, the accumulator of group w, at [256 + 128 w, +D).
// S_j goes into the score buffer as soon as the softmax has read S_{j-1} into
// registers, so the next block's Q K^T runs while this block's softmax does.
// P_j is the A operand (from TMEM) of O_w += P_j V_j, issued in two halves of
// the key rows: the softmax releases the first 64 keys of P_j before it
// computes the rest.  P buffer w and O_w take block j + 2 once
// P_j V_j is complete.
// Each group keeps its own running max, sum and accumulator over its half of
// the blocks, so the groups never wait for each other; the epilogue merges
// the two halves (a fixed split, so the result is deterministic).  O_w is
// rescaled only when a row max grows by more than 2^8 (a warp-uniform
// decision), right after the row max and before any of P_j is released (O_w
// is at rest then: the group waits for its previous P V product first).
// The softmax works in the exp2 domain.  Column pairs selected by
// RF_EMU_PAIR_MASK take their exponentials from a polynomial on the FMA pipe
// (rf_exp2_poly2, two values per paired instruction) instead of the MUFU unit,
// whose 16 results per clock per SM are otherwise as busy as the tensor pipe
// at D = 128.
// Every wait is bounded: on expiry the CTA records it in the status words and
// unwinds (waiting, again bounded, for its own copies and MMAs in flight).
//
// Precision "mxfp4" (kMx; MXAttention abstract: MXFP4 attention with UOS
// scaling and Pre-Normalization Quantization): Q, K and V arrive already
// rounded to MXFP4 (exact 16-bit values; V as f16).  The softmax keeps its
// running max an integer (log2 units) and, for every group of 32 keys, takes
// the exponentials against m + e, e the group's UOS exponent, so that they
// land in (3.625, 7.25] at the top; it rounds them to E2M1 in hardware,
// accumulates the row sum from the rounded values (PNQ) and hands P V the
// rounded values times 2^e as f16.  Power-of-two scales make the rounded P
// independent of which integer the running max is, so the result does not
// depend on the order the blocks are visited in.  At head dim 128 the MXFP4
// values travel instead as E4M3 codes (an E2M1 value times a power of two in
// range is exact in E4M3), so both products run on the FP8 tensor cores
// (kind::f8f6f4) with unit scales.
//
// Precisions "mix" and "fp8" (user guide, "Configuration"): Q K^T on E4M3
// copies of Q and K with one fp32 scale per (head, block), folded into the
// exponent scale of S_j; "fp8" also runs P V on E4M3: V' per (head, block)
// with a power-of-two scale 2^e_j, and P quantized per block as
// P * 2^(e_j - e_max) so that one output scale 2^e_max serves every block.
#include <cuda.h>
#include <cuda_fp16.h>

#include <mutex>

#include "rf_device.cuh"

namespace {

constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;   // Q and K loads
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10; // V loads
constexpr int kPvWarp = 11;        // P V issue
constexpr int kLaunchRegs = 168;   // 65536 / 384, rounded down to a multiple of 8
constexpr uint32_t kSoftmaxRegs = 216;
constexpr uint32_t kOtherRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
#ifndef RF_EMU_PAIR_MASK
#define RF_EMU_PAIR_MASK 0x0u
#endif
constexpr uint32_t kEmuPairMask = RF_EMU_PAIR_MASK;  // bit i: pair i of every 16 column pairs uses rf_exp2_poly2
constexpr int kStagesK = 3;  // K ring: K_{j+3} is requested as soon as S_j is done
constexpr uint32_t kPCol = 128;  // P of group w at kPCol + 64 w (128 keys as 16-bit pairs)
constexpr uint32_t kOCol = 256;  // O_w, the accumulator of softmax group w, at kOCol + 128 w
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: lazy rescale while growth <= 256x
// Precision mxfp4 with E4M3 carriers (head dim 128): the running max is kept
// exact (threshold 0, so P <= 1) and the E4M3 P values are stored times 2^8
// (at most 256 < 448), which keeps every MXFP4 value of P with 2^e >= 2^-16
// exact in E4M3; the output is multiplied back by 2^-8.
constexpr int kMxP8Up = 8;

// kQk8: Q and K tiles hold E4M3 codes (precisions "mix" and "fp8"), one byte
// per element.  kPv8: V tiles hold E4M3 codes stored transposed (D rows of 128
// keys, precision "fp8").
template <int D, bool kQk8, bool kPv8 = false>
struct __align__(1024) AttnSmem {
  static constexpr int kQkTileBytes = RF_BLOCK * D * (kQk8 ? 1 : 2);
  static constexpr int kVTileBytes = RF_BLOCK * D * (kPv8 ? 1 : 2);
  // V ring: V_{j+kStagesV} is requested as soon as O += P_j V_j is done.  The
  // one-byte Q and K tiles leave room for a third V stage.
  static constexpr int kStagesV = kPv8 ? 4 : (kQk8 ? 3 : 2);
  uint8_t q[kQkTileBytes];
  uint8_t k[kStagesK][kQkTileBytes];
  uint8_t v[kStagesV][kVTileBytes];
  uint64_t bar_q;
  uint64_t bar_k_full[kStagesK], bar_k_empty[kStagesK];
  uint64_t bar_v_full[kStagesV], bar_v_empty[kStagesV];
  uint64_t bar_s_full[2];    // S_j computed (j % 2: one barrier per softmax group, so that
                             // a group never mistakes the other group's S for its own)
  uint64_t bar_s_free;       // S_j read into registers: the score buffer may take S_{j+1}
  uint64_t bar_p_half[2], bar_p_full[2];  // P_j stored, first half / all (j % 2)
  uint64_t bar_pv_done[2];   // O_{j%2} += P_j V_j complete: P buffer j % 2 may take P_{j+2}
  uint64_t bar_final;
  uint64_t bar_drain;
  uint32_t tmem_base;
  int abort;
  int n_valid;
  float row_m[2][RF_BLOCK];
  float row_l[2][RF_BLOCK];
  // compacted selectIdx row; with 64-row key blocks, pairs (a, b) of one
  // 128-key tile each (b = -1: none), hence two spare entries
  int list[RF_MAX_KV_LIST + 2];
  float kscale[kQk8 ? RF_MAX_KV_LIST : 1];  // dequantization scale of K block list[j]
  int vexp[kPv8 ? RF_MAX_KV_LIST : 1];      // power-of-two exponent of V block list[j]
  int vexp_max;                             // the largest of them
};

struct AttnArgs {
  RfGeomDev g;
  const int32_t* sel_idx;
  const int32_t* sel_num;
  uint16_t* o_r;
  uint32_t* status;
  const float* q_scale;  // precisions "mix" and "fp8": E4M3 scales [n1][t_qblk] and [n2][t_qblk]
  const float* k_scale;
  const int32_t* v_exp;  // precision "fp8": V exponents [n2][t_qblk]
  float sl2;  // scale * log2(e)
};

// Warp-wide bounded wait: every lane polls the barrier itself (a lane that
// only waits on a warp shuffle for a polling lane 0 wakes far later), then the
// warp agrees on the outcome.  kPoll = true drops the suspend hint: the MMA
// warp's hand-offs (P ready, V and K tiles landed) sit on the critical path,
// and polling them measured about 2% faster overall than sleeping on them.
template <bool kPoll = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait<kPoll>(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void record_timeout(volatile int* abort, uint32_t* status, int where) {
  *abort = 1;
  atomicOr(status + RF_STATUS_TIMEOUT, 1u << where);
}

__device__ __forceinline__ void softmax_bar_sync() {
  asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight softmax warps
}

// Row max of 128 raw scores (the first vr valid): three-input max, eight chains.
template <bool kFull>
__device__ __forceinline__ float row_max(const uint32_t* sr, int vr) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = -INFINITY;
  if (kFull) {
#pragma unroll
    for (int c = 0; c < 128; c += 2)
      m[(c >> 1) & 7] = rf_max3(m[(c >> 1) & 7], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
  } else {
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if (c < vr) m[c & 7] = fmaxf(m[c & 7], __uint_as_float(sr[c]));
  }
  return rf_max3(rf_max3(m[0], m[1], m[2]), rf_max3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// p = 2^(s * sl2 - m) for the 32 scores c0 .. c0 + 31 of a row (the first vr
// of the row valid), packed pairwise to 16-bit and stored to the 16 TMEM
// columns at p_addr; the fp32 sums go to the four paired accumulators acc (a
// column pair's accumulator does not depend on c0, so the quarters sum in the
// same order as one pass would).  The scale-and-subtract and the sums run as
// paired fp32 instructions (two columns per instruction).  Pairs selected by
// kEmuPairMask use the FMA-pipe polynomial (both values of the pair at once),
// the others ex2.approx.
template <bool kBf16, bool kFull>
__device__ __forceinline__ void quarter_row_exp(const uint32_t* sr, int c0, int vr, float sl2, float neg_m,
                                                uint32_t p_addr, uint64_t* acc) {
  const uint64_t sl2x2 = rf_f2(__float_as_uint(sl2), __float_as_uint(sl2));
  const uint64_t negm2 = rf_f2(__float_as_uint(neg_m), __float_as_uint(neg_m));
  uint32_t pk[16];
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const bool emu = (kEmuPairMask >> ((c >> 1) & 15)) & 1u;
    float x0, x1, p0, p1;
    rf_f2_split(rf_fma2(rf_f2(sr[c0 + c], sr[c0 + c + 1]), sl2x2, negm2), x0, x1);
    if (emu) {
      rf_exp2_poly2(x0, x1, p0, p1);
    } else {
      p0 = rf_ex2(x0);
      p1 = rf_ex2(x1);
    }
    if (!kFull) {
      p0 = c0 + c < vr ? p0 : 0.f;
      p1 = c0 + c + 1 < vr ? p1 : 0.f;
    }
    acc[(c >> 1) & 3] = rf_add2(acc[(c >> 1) & 3], rf_f2(__float_as_uint(p0), __float_as_uint(p1)));
    pk[c >> 1] = rf_pack2<kBf16>(p0, p1);
  }
  tmem_st16(p_addr, pk);
}

// Precision "fp8": p = 2^(s * sl2 - m) for the 32 scores c0 .. c0 + 31 of a row
// (the first vr valid; pairs selected by kEmuPairMask from the FMA-pipe
// polynomial).  The fp32 values go to the row sum (acc, as in
// quarter_row_exp); p * down, down = 2^-shift the power-of-two step from this
// V block's exponent to the row's largest, is rounded to E4M3 (nearest even,
// saturating) and stored four codes per column, the lowest key in the lowest
// byte, to the 8 TMEM columns at p_addr.
template <bool kFull>
__device__ __forceinline__ void quarter_row_exp_f8(const uint32_t* sr, int c0, int vr, float sl2, float neg_m,
                                                   float down, uint32_t p_addr, uint64_t* acc) {
  const uint64_t sl2x2 = rf_f2(__float_as_uint(sl2), __float_as_uint(sl2));
  const uint64_t negm2 = rf_f2(__float_as_uint(neg_m), __float_as_uint(neg_m));
  const uint64_t down2 = rf_f2(__float_as_uint(down), __float_as_uint(down));
  uint32_t pk[8];
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    uint32_t half[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cc = c + 2 * h;
      float x0, x1, p0, p1;
      rf_f2_split(rf_fma2(rf_f2(sr[c0 + cc], sr[c0 + cc + 1]), sl2x2, negm2), x0, x1);
      if ((kEmuPairMask >> ((cc >> 1) & 15)) & 1u) {
        rf_exp2_poly2(x0, x1, p0, p1);
      } else {
        p0 = rf_ex2(x0);
        p1 = rf_ex2(x1);
      }
      if (!kFull) {
        p0 = c0 + cc < vr ? p0 : 0.f;
        p1 = c0 + cc + 1 < vr ? p1 : 0.f;
      }
      const uint64_t pp = rf_f2(__float_as_uint(p0), __float_as_uint(p1));
      acc[(cc >> 1) & 3] = rf_add2(acc[(cc >> 1) & 3], pp);
      float y0, y1;
      rf_f2_split(rf_mul2(pp, down2), y0, y1);
      unsigned short two;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(y1), "f"(y0));
      half[h] = two;
    }
    pk[c >> 2] = half[0] | (half[1] << 16);
  }
  tmem_st8(p_addr, pk);
}

// Maxima of the four 32-column groups of a row of raw scores (the first vr
// valid; a group with no valid column gives -inf).
template <bool kFull>
__device__ __forceinline__ void group_max4(const uint32_t* sr, int vr, float* gm) {
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    float m[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int c = 32 * gi; c < 32 * gi + 32; c += 2) {
      if (kFull) {
        m[(c >> 1) & 1] = rf_max3(m[(c >> 1) & 1], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
      } else {
        if (c < vr) m[0] = fmaxf(m[0], __uint_as_float(sr[c]));
        if (c + 1 < vr) m[1] = fmaxf(m[1], __uint_as_float(sr[c + 1]));
      }
    }
    gm[gi] = fmaxf(m[0], m[1]);
  }
}

// Precision "mxfp4": P over the 32 scores cb .. cb + 31 of a row (one group of
// 32 keys), rounded to MXFP4 and packed as f16 pairs into the 16 TMEM columns
// at p_addr; the rounded values are summed into lsum.  m is the integer
// running max; gmax the group's raw score maximum.  Group exponent (UOS):
// e = ceil(log2(amax / 7.25)) with log2(amax) = gmax * sl2 - m; the
// exponentials are taken as 2^(s * sl2 - (m + e)), rounded to E2M1 (the
// hardware conversion saturates at 6), summed exactly in f16 (at most 32
// values of at most 6 on a 0.5 grid) and scaled by 2^e.
template <bool kFull, bool kOut8 = false>
__device__ __forceinline__ void group_exp_mx(const uint32_t* sr, int cb, int vr, float sl2, float m,
                                             float gmax, uint32_t p_addr, float& lsum) {
  constexpr int kUp = kOut8 ? kMxP8Up : 0;   // E4M3 P is stored times 2^kUp
  const uint64_t sl2x2 = rf_f2(__float_as_uint(sl2), __float_as_uint(sl2));
  const bool live = kFull || cb < vr;
  const int e = live ? (int)ceilf(fmaf(gmax, sl2, -m) - kMxLog2Qmax) : 0;
  const float neg_me = -(m + (float)e);
  const uint64_t negme2 = rf_f2(__float_as_uint(neg_me), __float_as_uint(neg_me));
  // 2^(e + kUp) as f16 (normal from 2^-14, subnormal down to 2^-24; a group
  // whose scale is below that rounds to zero in f16, as its P V terms would)
  const int eu = e + kUp;
  const unsigned short hb = eu >= -14 ? (unsigned short)((15 + eu) << 10)
                                      : (eu >= -24 ? (unsigned short)(1u << (eu + 24)) : (unsigned short)0);
  const __half2 up2 = __half2half2(__ushort_as_half(hb));
  __half2 acc0 = __float2half2_rn(0.f), acc1 = acc0;
  // kOut8: the rounded values times 2^(e + kUp), exact in f16, converted to
  // E4M3 codes four per column (exact for -8 <= e + kUp <= 6); else the f16
  // pairs themselves
  uint32_t pk[kOut8 ? 8 : 16];
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    float x0, x1;
    rf_f2_split(rf_fma2(rf_f2(sr[cb + c], sr[cb + c + 1]), sl2x2, negme2), x0, x1);
    float y0 = rf_ex2(x0), y1 = rf_ex2(x1);
    if (!kFull) {
      y0 = cb + c < vr ? y0 : 0.f;
      y1 = cb + c + 1 < vr ? y1 : 0.f;
    }
    const uint32_t r = rf_e2m1x2_round(y0, y1);
    const __half2 rh = *reinterpret_cast<const __half2*>(&r);
    if (c & 2) acc1 = __hadd2(acc1, rh);
    else       acc0 = __hadd2(acc0, rh);
    const __half2 ph = __hmul2(rh, up2);
    if constexpr (kOut8) {
      unsigned short two;
      asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(two) : "r"(*reinterpret_cast<const uint32_t*>(&ph)));
      if (c & 2) pk[c >> 2] |= (uint32_t)two << 16;
      else       pk[c >> 2] = two;
    } else {
      pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&ph);
    }
  }
  const float2 sum = __half22float2(__hadd2(acc0, acc1));
  if (live && e >= -126) lsum = fmaf(sum.x + sum.y, rf_pow2(e), lsum);
  if constexpr (kOut8) tmem_st8(p_addr, pk);
  else                 tmem_st16(p_addr, pk);
}

__device__ __forceinline__ float acc_sum(const uint64_t* acc) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float a, b;
    rf_f2_split(acc[i], a, b);
    s += a + b;
  }
  return s;
}

template <int D, bool kBf16, bool kQk8, bool kMx, bool kPv8>
__global__ void __launch_bounds__(kThreads, 1)
    rf_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnArgs a) {
  using Smem = AttnSmem<D, kQk8, kPv8>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // Tiles are read as 128-byte-wide swizzle boxes of 128 rows.
  constexpr int kQkBoxes = D * (kQk8 ? 1 : 2) / 128;  // boxes per Q or K tile
  constexpr int kVBoxes = kPv8 ? 1 : D * 2 / 128;     // boxes per V tile
  constexpr uint32_t kQkTileBytes = Smem::kQkTileBytes;
  constexpr uint32_t kVTileBytes = Smem::kVTileBytes;
  constexpr int kStagesV = Smem::kStagesV;
  constexpr uint32_t kBoxBytes = RF_BLOCK * 128;

  const RfGeomDev& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x / g.t_qblk;  // query head (head-major order)
  const int tb = blockIdx.x % g.t_qblk;
  const RfSeqDev& s = g.seq[rf_seq_of_qblk(g, tb)];
  const int qb = tb - s.qblk_off;
  const int nblk = s.n_pb + s.nb;
  const bool kv64 = g.block_kv == 64;                       // blockShape 128 x 64
  const int nkv = kv64 ? rf_n_pb64(s) + 2 * s.nb : nblk;   // key/value blocks of this sequence
  const int gk = n / (g.n1 / g.n2);  // key/value head
  int q_r0, q_rows;
  rf_block_span(s, qb, q_r0, q_rows);
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesK; ++i) {
      mbar_init(rf_smem_u32(&sm.bar_k_full[i]), 1);
      mbar_init(rf_smem_u32(&sm.bar_k_empty[i]), 1);
    }
    for (int i = 0; i < kStagesV; ++i) {
      mbar_init(rf_smem_u32(&sm.bar_v_full[i]), 1);
      mbar_init(rf_smem_u32(&sm.bar_v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(rf_smem_u32(&sm.bar_p_half[i]), 128);
      mbar_init(rf_smem_u32(&sm.bar_p_full[i]), 128);
      mbar_init(rf_smem_u32(&sm.bar_pv_done[i]), 1);
    }
    mbar_init(rf_smem_u32(&sm.bar_s_full[0]), 1);
    mbar_init(rf_smem_u32(&sm.bar_s_full[1]), 1);
    mbar_init(rf_smem_u32(&sm.bar_s_free), 128);
    mbar_init(rf_smem_u32(&sm.bar_final), 2);   // one commit from each issuing warp
    mbar_init(rf_smem_u32(&sm.bar_drain), 2);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    // The Q tile does not depend on the selection: request it first thing.
    mbar_init(rf_smem_u32(&sm.bar_q), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    int c1, c2;
    if (g.layout == RF_LAYOUT_BNSD) { c1 = q_r0; c2 = s.batch_idx * g.n1 + n; }
    else                            { c1 = n; c2 = (int)s.row_off + q_r0; }
    mbar_arrive_expect_tx(rf_smem_u32(&sm.bar_q), kQkTileBytes);
#pragma unroll
    for (int x = 0; x < kQkBoxes; ++x)
      tma_load_3d(rf_smem_u32(sm.q + x * kBoxBytes), &tm_q, rf_smem_u32(&sm.bar_q), x * 64, c1, c2);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(rf_smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  // The selectIdx row (and, with E4M3 Q and K, each entry's K scale) into
  // shared memory: every thread loads, so the row costs one round trip.
  const size_t row_id = (size_t)tb * g.n1 + n;
  const int32_t* row = a.sel_idx + row_id * g.max_kv;
  const int num_raw = a.sel_num[row_id];
  const int num = num_raw < 0 ? 0 : (num_raw > g.max_kv ? g.max_kv : num_raw);
  for (int c = threadIdx.x; c < num; c += kThreads) {
    const int v = row[c];
    sm.list[c] = v;
    // precision mxfp4 carries its values in E4M3 with unit scales: nothing to load
    if constexpr (kQk8 && !kMx)
      if (v >= 0 && v < nkv) sm.kscale[c] = a.k_scale[(size_t)gk * g.t_qblk + s.qblk_off + v];
    if constexpr (kPv8 && !kMx)
      if (v >= 0 && v < nkv) sm.vexp[c] = a.v_exp[(size_t)gk * g.t_qblk + s.qblk_off + v];
  }
  __syncthreads();
  if (warp == 0) {
    // Compact the row in place: keep in-range entries in order, skip -1 (an
    // unused slot), count anything else as a bad index.  A lane writes at or
    // below its own read position, and every lane reads before the ballot.
    int bad = (lane == 0 && num != num_raw) ? 1 : 0;
    int cnt = 0;
    int vmax = kMx ? 0 : -127;  // precision "fp8": the largest V exponent of the row
    const uint32_t lt = (1u << lane) - 1u;
    for (int c0 = 0; c0 < num; c0 += 32) {
      const int c = c0 + lane;
      const int v = c < num ? sm.list[c] : -1;
      float ks = 1.f;
      if constexpr (kQk8 && !kMx) ks = c < num ? sm.kscale[c] : 0.f;
      int ve = kMx ? 0 : -127;
      if constexpr (kPv8 && !kMx) ve = c < num ? sm.vexp[c] : -127;
      const bool ok = c < num && v >= 0 && v < nkv;
      if (c < num && v != -1 && !ok) ++bad;
      const uint32_t ball = __ballot_sync(0xffffffffu, ok);
      if (ok) {
        sm.list[cnt + __popc(ball & lt)] = v;
        if constexpr (kQk8) sm.kscale[cnt + __popc(ball & lt)] = ks;
        if constexpr (kPv8) {
          sm.vexp[cnt + __popc(ball & lt)] = ve;
          vmax = max(vmax, ve);
        }
      }
      cnt += __popc(ball);
    }
    if constexpr (kPv8) {
      vmax = __reduce_max_sync(0xffffffffu, vmax);
      if (lane == 0) sm.vexp_max = vmax;
    }
    bad = __reduce_add_sync(0xffffffffu, bad);
    int units = cnt;  // tiles of 128 keys
    if (kv64) {
      // Pair the 64-row blocks into 128-key tiles: list[2t], list[2t + 1].
      // Valid key rows must run from the tile's first row, so the partial
      // prefix block may be the second of a pair but not the first: if it
      // falls on an even position it stays alone (the entries after it move
      // up by one) -- it can occur at most once.  An odd count leaves the
      // last tile's second half empty.
      const int part_blk = (s.Lp & 63) ? rf_n_pb64(s) - 1 : -1;
      int qpos = -1;
      for (int c0 = 0; c0 < cnt; c0 += 32) {
        const int c = c0 + lane;
        const uint32_t hit = __ballot_sync(0xffffffffu, c < cnt && sm.list[c] == part_blk);
        if (hit && qpos < 0) qpos = c0 + __ffs(hit) - 1;
      }
      const int shift = (qpos >= 0 && (qpos & 1) == 0) ? 1 : 0;
      if (shift) {
        // entries qpos + 1 .. cnt - 1 move to +1, 32 at a time from the end:
        // a chunk reads everything before it writes
        for (int hi = cnt; hi > qpos + 1; hi -= 32) {
          const int c = hi - 1 - lane;
          const bool act = c > qpos;
          const int v = act ? sm.list[c] : 0;
          __syncwarp();
          if (act) sm.list[c + 1] = v;
          __syncwarp();
        }
        if (lane == 0) sm.list[qpos + 1] = -1;
      }
      const int tot = cnt + shift;
      if (lane == 0 && (tot & 1)) sm.list[tot] = -1;
      units = (tot + 1) >> 1;
    }
    if (lane == 0) {
      // A wait that already expired in this workspace (this launch or an
      // earlier one not yet cleared by rf_check_device_status) stops all work.
      const bool stopped = *reinterpret_cast<volatile uint32_t*>(a.status + RF_STATUS_TIMEOUT) != 0;
      sm.n_valid = stopped ? 0 : units;
      if (bad) atomicAdd(a.status + RF_STATUS_BAD_INDEX, (uint32_t)bad);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int nv = sm.n_valid;
  const int vr_last = s.Lp - (s.n_pb - 1) * RF_BLOCK;  // valid rows of the last prefix block
  if (warp >= 8) {
  reg_dealloc<kOtherRegs>();
  if ((warp == kProducerWarp || warp == kVProducerWarp) && lane == 0 && nv > 0) {
    // ---------------- TMA producers: one thread streams Q then K, another V ----------------
    const bool is_k = warp == kProducerWarp;
    const bool bnsd = g.layout == RF_LAYOUT_BNSD;
    auto coords = [&](int heads, int head, int r0, int& c1, int& c2) {
      if (bnsd) { c1 = r0; c2 = s.batch_idx * heads + head; }
      else      { c1 = head; c2 = (int)s.row_off + r0; }
    };
    int c1, c2;
    const uint32_t bq = rf_smem_u32(&sm.bar_q);
    const int stages = is_k ? kStagesK : kStagesV;
    const uint32_t tile_bytes = is_k ? kQkTileBytes : kVTileBytes;
    const int boxes = is_k ? kQkBoxes : kVBoxes;
    uint8_t* tiles = is_k ? &sm.k[0][0] : &sm.v[0][0];
    uint64_t* full = is_k ? sm.bar_k_full : sm.bar_v_full;
    uint64_t* empty = is_k ? sm.bar_k_empty : sm.bar_v_empty;
    const void* map = is_k ? static_cast<const void*>(&tm_k) : static_cast<const void*>(&tm_v);
    int issued = 0;
    for (int j = 0; j < nv; ++j) {
      const int st = j % stages;
      const uint32_t ph = (j / stages) & 1;
      if (j >= stages && !mbar_wait(rf_smem_u32(&empty[st]), ph ^ 1, abort)) {
        record_timeout(abort, a.status, is_k ? 0 : 1);
        break;
      }
      const uint32_t bar = rf_smem_u32(&full[st]);
      mbar_arrive_expect_tx(bar, tile_bytes);
      if (kPv8 && !is_k) {
        // transposed E4M3 V block: D rows of 128 keys, one 128-byte box
        tma_load_3d(rf_smem_u32(tiles + st * tile_bytes), map, bar, 0, 0,
                    gk * g.t_qblk + s.qblk_off + sm.list[j]);
      } else if (!kv64) {
        int r0, nr;
        rf_block_span(s, sm.list[j], r0, nr);
        coords(g.n2, gk, r0, c1, c2);
        for (int x = 0; x < boxes; ++x)
          tma_load_3d(rf_smem_u32(tiles + st * tile_bytes + x * kBoxBytes), map, bar, x * 64, c1, c2);
      } else {
        // two 64-row boxes per column box (the maps have 64-row boxes): block a
        // into tile rows 0..63, block b into rows 64..127; an empty second
        // half loads block a again, so that its (masked) keys stay finite
        const int blk_a = sm.list[2 * j];
        const int blk_b = sm.list[2 * j + 1] >= 0 ? sm.list[2 * j + 1] : blk_a;
        int ra, rb, na, nb2, c1b, c2b;
        rf_kv64_span(s, blk_a, ra, na);
        rf_kv64_span(s, blk_b, rb, nb2);
        coords(g.n2, gk, ra, c1, c2);
        coords(g.n2, gk, rb, c1b, c2b);
        for (int x = 0; x < boxes; ++x) {
          const uint32_t dst = rf_smem_u32(tiles + st * tile_bytes + x * kBoxBytes);
          tma_load_3d(dst, map, bar, x * 64, c1, c2);
          tma_load_3d(dst + 64 * 128, map, bar, x * 64, c1b, c2b);
        }
      }
      issued = j + 1;
    }
    if (*abort) {
      // Let this thread's own copies land before the CTA's shared memory goes
      // away: the newest load of each stage completes last on its barrier.
      volatile int no_abort = 0;
      if (is_k) mbar_wait(bq, 0, &no_abort);
      for (int j = (issued > stages ? issued - stages : 0); j < issued; ++j)
        mbar_wait(rf_smem_u32(&full[j % stages]), (j / stages) & 1, &no_abort);
    }
  } else if ((warp == kMmaWarp || warp == kPvWarp) && nv > 0) {
    // ---------------- tcgen05.mma issue: S products (warp 9), P V products (warp 11) ----------------
    // Two issuing warps: a single thread cannot keep the tensor pipe fed with
    // 128 x 128 x 16 instructions once its barrier checks sit between them.
    // Each warp runs its whole loop (warp-uniform control flow keeps the
    // descriptors in uniform registers); one elected lane issues every MMA and
    // every commit of that warp, so its commits track all of its MMAs.
    const uint32_t fmt = kBf16 ? 1u : 0u;
    bool ok = true;
    if (warp == kMmaWarp) {
      // kind::f8f6f4 takes E4M3 as format 0 in the same descriptor fields.
      const uint32_t idesc_qk = umma_idesc_f16(kQk8 ? 0u : fmt, 128, 128, 0);
      // Adding (bytes >> 4) to a descriptor moves its 14-bit start-address field.
      const uint64_t dq = umma_desc_sw128(rf_smem_u32(sm.q), 16, 1024);
      const uint64_t dk0 = umma_desc_sw128(rf_smem_u32(sm.k[0]), 16, 1024);
      ok = warp_wait<true>(rf_smem_u32(&sm.bar_q), 0, abort);
      for (int j = 0; ok && j < nv; ++j) {
        const int st = j % kStagesK;
        // S_j goes into the score buffer once the softmax has read S_{j-1}.
        if (j > 0 && !warp_wait<true>(rf_smem_u32(&sm.bar_s_free), (j - 1) & 1, abort)) {
          ok = false;
          break;
        }
        if (!warp_wait<true>(rf_smem_u32(&sm.bar_k_full[st]), (j / kStagesK) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
          // S_j = Q K_j^T: every MMA takes a 32-byte slice of the reduction
          // (16 bf16/fp16 or 32 E4M3 elements).
          const uint64_t dk = dk0 + (uint64_t)(st * (kQkTileBytes >> 4));
          const uint32_t d_s = tmem;
#pragma unroll
          for (int kk = 0; kk < (int)(kQkTileBytes / RF_BLOCK / 32); ++kk) {
            const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
            if constexpr (kQk8)
              mma_ss_f8(d_s, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
            else
              mma_ss(d_s, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(rf_smem_u32(&sm.bar_s_full[j & 1]));
          tc_commit(rf_smem_u32(&sm.bar_k_empty[st]));
        }
        __syncwarp();
      }
    } else {
      // precision "mxfp4": P and V are f16 whatever the input type; precision
      // "fp8": both E4M3 (format 0 of kind::f8f6f4), V transposed, so K-major
      const uint32_t idesc_pv = umma_idesc_f16(kMx || kPv8 ? 0u : fmt, 128, D, kPv8 ? 0u : 1u);
      const uint64_t dv0 = kPv8 ? umma_desc_sw128(rf_smem_u32(sm.v[0]), 16, 1024)
                                : umma_desc_sw128(rf_smem_u32(sm.v[0]), kBoxBytes, 1024);
      for (int j = 0; ok && j < nv; ++j) {
        const int b = j & 1, st = j % kStagesV;
        const uint32_t ph = (j >> 1) & 1;
        const uint64_t dv = dv0 + (uint64_t)(st * (kVTileBytes >> 4));
        const uint32_t a_p = tmem + kPCol + (uint32_t)(b * 64);  // P_j
        const uint32_t d_o = tmem + kOCol + (uint32_t)(b * 128);  // O_b
        // O += P_j V_j in two halves of the key rows: the first as soon as the
        // softmax has stored the first 64 columns of P_j, the second when all
        // of P_j is in.
        if (!warp_wait<true>(rf_smem_u32(&sm.bar_p_half[b]), ph, abort)) { ok = false; break; }
        if (!warp_wait<true>(rf_smem_u32(&sm.bar_v_full[st]), (j / kStagesV) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
          if constexpr (kPv8) {
            // 32 keys per MMA: 8 TMEM columns of P', 32 bytes of each V row
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_ts_f8(d_o, a_p + kk * 8, dv + (uint32_t)(kk * 2), idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < RF_BLOCK / 32; ++kk)
              mma_ts(d_o, a_p + kk * 8, dv + (uint32_t)(kk * (2048 >> 4)), idesc_pv,
                     (j >= 2 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
        if (!warp_wait<true>(rf_smem_u32(&sm.bar_p_full[b]), ph, abort)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
          if constexpr (kPv8) {
#pragma unroll
            for (int kk = 2; kk < 4; ++kk) mma_ts_f8(d_o, a_p + kk * 8, dv + (uint32_t)(kk * 2), idesc_pv, 1u);
          } else {
#pragma unroll
            for (int kk = RF_BLOCK / 32; kk < RF_BLOCK / 16; ++kk)
              mma_ts(d_o, a_p + kk * 8, dv + (uint32_t)(kk * (2048 >> 4)), idesc_pv, 1u);
          }
          tc_commit(rf_smem_u32(&sm.bar_v_empty[st]));
          tc_commit(rf_smem_u32(&sm.bar_pv_done[b]));
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) record_timeout(abort, a.status, 2);
    // Every MMA this warp issued (all of them, on the normal path) completes
    // before bar_final, which gates the epilogue, and before bar_drain, which
    // gates freeing TMEM; both barriers count the two issuing warps.
    if (elect_one()) {
      tc_commit(rf_smem_u32(&sm.bar_final));
      tc_commit(rf_smem_u32(&sm.bar_drain));
    }
    __syncwarp();
    volatile int no_abort = 0;
    warp_wait(rf_smem_u32(&sm.bar_drain), 0, &no_abort);
  }
  if (warp == kProducerWarp && lane == 0 && nv == 0) {
    // Nothing to compute (an empty row, or a recorded expiry): the Q copy
    // requested at the start still has to land before the CTA exits.
    volatile int no_abort = 0;
    mbar_wait(rf_smem_u32(&sm.bar_q), 0, &no_abort);
  }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ---------------- softmax + epilogue (warps 0-7) ----------------
    const int wg = warp >> 2;                 // this warpgroup's block parity
    const int row = (warp & 3) * 32 + lane;   // query row = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    // precision "mix": S_j carries the E4M3 scales of the Q block and of K block j
    const float sl2_q = (kQk8 && !kMx) ? a.sl2 * a.q_scale[(size_t)n * g.t_qblk + tb] : a.sl2;
    const int my_blocks = (nv + 1 - wg) >> 1;  // blocks j < nv with j % 2 == wg
    const int vexp_max = kPv8 ? sm.vexp_max : 0;
    const uint32_t scol = lane_base;                          // S_j (both groups in turn)
    const uint32_t pcol = lane_base + kPCol + (uint32_t)(wg * 64);
    const uint32_t ocol = lane_base + kOCol + (uint32_t)(wg * 128);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < my_blocks; ++i) {
      const int j = 2 * i + wg;
      if (!warp_wait(rf_smem_u32(&sm.bar_s_full[wg]), i & 1, abort)) { ok = false; break; }
      tc_fence_after();
      int vr;  // valid key rows of the tile, from its first row; uniform over the CTA
      if (kv64) {
        int r0, na, nb2 = 0;
        rf_kv64_span(s, sm.list[2 * j], r0, na);
        if (sm.list[2 * j + 1] >= 0) rf_kv64_span(s, sm.list[2 * j + 1], r0, nb2);
        vr = na + nb2;
      } else {
        vr = (sm.list[j] == s.n_pb - 1) ? vr_last : RF_BLOCK;
      }
      const float sl2 = (kQk8 && !kMx) ? sl2_q * sm.kscale[j] : sl2_q;
      // precision "fp8": P' = P * 2^-(exp_max - exp_j) for the P V product
      float down = 1.f;
      if constexpr (kPv8) {
        const int shift = vexp_max - sm.vexp[j];
        down = shift <= 126 ? rf_pow2(-shift) : 0.f;
      }
      uint32_t sr[128];
      tmem_ld32(scol, sr);
      tmem_ld32(scol + 32, sr + 32);
      tmem_ld32(scol + 64, sr + 64);
      tmem_ld32(scol + 96, sr + 96);
      tmem_wait_ld();
      // S_j is in registers: the score buffer may take S_{j+1}.
      tc_fence_before();
      mbar_arrive(rf_smem_u32(&sm.bar_s_free));
      float gm[4];
      float mx_t;
      if constexpr (kMx) {
        if (vr == RF_BLOCK) group_max4<true>(sr, vr, gm);
        else                group_max4<false>(sr, vr, gm);
        mx_t = fmaxf(fmaxf(gm[0], gm[1]), fmaxf(gm[2], gm[3])) * sl2;
      } else {
        mx_t = (vr == RF_BLOCK ? row_max<true>(sr, vr) : row_max<false>(sr, vr)) * sl2;
      }
      // P buffer wg and O_wg still serve P_{j-2} V_{j-2} until that product is
      // complete (issued long ago; normally done).
      if (i > 0) {
        if (!warp_wait(rf_smem_u32(&sm.bar_pv_done[wg]), (i - 1) & 1, abort)) { ok = false; break; }
        tc_fence_after();
      }
      constexpr float kThr = (kMx && kPv8) ? 0.f : kRescaleThreshold;
      const bool rescale = __any_sync(0xffffffffu, mx_t > m_run + kThr);
      if (rescale) {
        // mxfp4: the running max stays an integer
        const float m_new = kMx ? ceilf(fmaxf(m_run, mx_t)) : fmaxf(m_run, mx_t);
        const float alpha = rf_ex2(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
        if (i > 0) {
          // O_wg holds this group's earlier P V products and is at rest (its
          // last one is complete, see above).  Rescale it before any of P_j is
          // released.
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(ocol + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(ocol + c0, o);
          }
        }
      }
      // P_j in four quarters of 32 columns (16 TMEM columns each): the first
      // two are released to the MMA warp while the other two are being
      // computed.
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      float lsum = 0.f;
      constexpr uint32_t kQCols = kPv8 ? 8 : 16;   // TMEM columns per 32 keys of P
      if constexpr (kMx) {
        if (vr == RF_BLOCK) {
          group_exp_mx<true, kPv8>(sr, 0, vr, sl2, m_run, gm[0], pcol, lsum);
          group_exp_mx<true, kPv8>(sr, 32, vr, sl2, m_run, gm[1], pcol + kQCols, lsum);
        } else {
          group_exp_mx<false, kPv8>(sr, 0, vr, sl2, m_run, gm[0], pcol, lsum);
          group_exp_mx<false, kPv8>(sr, 32, vr, sl2, m_run, gm[1], pcol + kQCols, lsum);
        }
      } else if constexpr (kPv8) {
        if (vr == RF_BLOCK) {
          quarter_row_exp_f8<true>(sr, 0, vr, sl2, -m_run, down, pcol, acc);
          quarter_row_exp_f8<true>(sr, 32, vr, sl2, -m_run, down, pcol + 8, acc);
        } else {
          quarter_row_exp_f8<false>(sr, 0, vr, sl2, -m_run, down, pcol, acc);
          quarter_row_exp_f8<false>(sr, 32, vr, sl2, -m_run, down, pcol + 8, acc);
        }
      } else {
        if (vr == RF_BLOCK) {
          quarter_row_exp<kBf16, true>(sr, 0, vr, sl2, -m_run, pcol, acc);
          quarter_row_exp<kBf16, true>(sr, 32, vr, sl2, -m_run, pcol + 16, acc);
        } else {
          quarter_row_exp<kBf16, false>(sr, 0, vr, sl2, -m_run, pcol, acc);
          quarter_row_exp<kBf16, false>(sr, 32, vr, sl2, -m_run, pcol + 16, acc);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(rf_smem_u32(&sm.bar_p_half[wg]));
      if constexpr (kMx) {
        if (vr == RF_BLOCK) {
          group_exp_mx<true, kPv8>(sr, 64, vr, sl2, m_run, gm[2], pcol + 2 * kQCols, lsum);
          group_exp_mx<true, kPv8>(sr, 96, vr, sl2, m_run, gm[3], pcol + 3 * kQCols, lsum);
        } else {
          group_exp_mx<false, kPv8>(sr, 64, vr, sl2, m_run, gm[2], pcol + 2 * kQCols, lsum);
          group_exp_mx<false, kPv8>(sr, 96, vr, sl2, m_run, gm[3], pcol + 3 * kQCols, lsum);
        }
        l_run += lsum;
      } else if constexpr (kPv8) {
        if (vr == RF_BLOCK) {
          quarter_row_exp_f8<true>(sr, 64, vr, sl2, -m_run, down, pcol + 16, acc);
          quarter_row_exp_f8<true>(sr, 96, vr, sl2, -m_run, down, pcol + 24, acc);
        } else {
          quarter_row_exp_f8<false>(sr, 64, vr, sl2, -m_run, down, pcol + 16, acc);
          quarter_row_exp_f8<false>(sr, 96, vr, sl2, -m_run, down, pcol + 24, acc);
        }
        l_run += acc_sum(acc);
      } else {
        if (vr == RF_BLOCK) {
          quarter_row_exp<kBf16, true>(sr, 64, vr, sl2, -m_run, pcol + 32, acc);
          quarter_row_exp<kBf16, true>(sr, 96, vr, sl2, -m_run, pcol + 48, acc);
        } else {
          quarter_row_exp<kBf16, false>(sr, 64, vr, sl2, -m_run, pcol + 32, acc);
          quarter_row_exp<kBf16, false>(sr, 96, vr, sl2, -m_run, pcol + 48, acc);
        }
        l_run += acc_sum(acc);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(rf_smem_u32(&sm.bar_p_full[wg]));
    }
    if (!ok) record_timeout(abort, a.status, 3);

    // Epilogue: merge the two groups' (max, sum, O) per row, write this group's
    // half of the columns: O = (2^(m0-m) O_0 + 2^(m1-m) O_1) / (2^(m0-m) l_0 + 2^(m1-m) l_1).
    sm.row_m[wg][row] = m_run;
    sm.row_l[wg][row] = l_run;
    softmax_bar_sync();
    const bool have_o = nv > 0 && !*abort && warp_wait(rf_smem_u32(&sm.bar_final), 0, abort) && !*abort;
    const float m0 = sm.row_m[0][row], m1 = sm.row_m[1][row];
    const float l0 = sm.row_l[0][row], l1 = sm.row_l[1][row];
    const float m = fmaxf(m0, m1);
    const float a0 = l0 > 0.f ? rf_ex2(m0 - m) : 0.f;
    const float a1 = l1 > 0.f ? rf_ex2(m1 - m) : 0.f;
    const float l = a0 * l0 + a1 * l1;
    // precision "fp8": P V ran on P * 2^-exp_max times the V codes
    const float vsc = kMx ? (kPv8 ? rf_pow2(-kMxP8Up) : 1.f)
                          : (kPv8 ? (vexp_max >= -126 ? rf_pow2(vexp_max) : 0.f) : 1.f);
    const float inv = l > 0.f ? vsc / l : 0.f;
    const float s0 = a0 * inv, s1 = a1 * inv;
    const bool use0 = have_o && nv > 0, use1 = have_o && nv > 1;
    uint16_t* dst = a.o_r + rf_row_offset(g, s, g.n1, n, q_r0 + min(row, q_rows - 1));
    if (have_o) tc_fence_after();
#pragma unroll 1
    for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
      uint32_t o0[32], o1[32];
      if (use0) tmem_ld32(lane_base + kOCol + c0, o0);
      if (use1) tmem_ld32(lane_base + kOCol + 128 + c0, o1);
      if (use0 || use1) tmem_wait_ld();
      uint32_t w[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float x0 = 0.f, x1 = 0.f;
        if (use0) {
          x0 = s0 * __uint_as_float(o0[2 * c]);
          x1 = s0 * __uint_as_float(o0[2 * c + 1]);
        }
        if (use1) {
          x0 = fmaf(s1, __uint_as_float(o1[2 * c]), x0);
          x1 = fmaf(s1, __uint_as_float(o1[2 * c + 1]), x1);
        }
        w[c] = rf_pack2<kBf16>(x0, x1);
      }
      if (row < q_rows) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
        d4[2] = make_uint4(w[8], w[9], w[10], w[11]);
        d4[3] = make_uint4(w[12], w[13], w[14], w[15]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Self-test of the two exponential paths the softmax uses.
__global__ void rf_exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                        float* __restrict__ y_mufu, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    y_poly[i] = rf_exp2_poly(x[i]);
    y_mufu[i] = rf_ex2(x[i]);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// Element type of a tensor map: the plan's 16-bit type, E4M3 bytes, or f16.
enum MapElem { kElemPlan = 0, kElemByte = 1, kElemF16 = 2 };

// Tensor map over [rows, heads, D] (TND) or [B*heads, rows, D] (BNSD) with a
// box_rows x 128-byte box and 128-byte swizzle: 64 columns of a 16-bit tensor,
// or 128 columns of a one-byte (E4M3) tensor.  box_rows is 128, or 64 for the
// key/value maps of blockShape 128 x 64.
rf_status_t make_map(CUtensorMap* m, const rf_plan* p, const void* base, int heads, MapElem elem,
                     int box_rows = RF_BLOCK) {
  const bool one_byte = elem == kElemByte;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return rf_fail(RF_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const RfGeomDev& g = p->g;
  const cuuint64_t d = (cuuint64_t)g.d;
  const cuuint64_t esz = one_byte ? 1 : 2;
  const cuuint32_t box_cols = one_byte ? 128 : 64;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  if (g.layout == RF_LAYOUT_BNSD) {
    const cuuint64_t L = (cuuint64_t)g.seq[0].L;
    dims[0] = d; dims[1] = L; dims[2] = (cuuint64_t)p->batch * heads;
    strides[0] = d * esz; strides[1] = L * d * esz;
    box[0] = box_cols; box[1] = (cuuint32_t)box_rows; box[2] = 1;
  } else {
    dims[0] = d; dims[1] = (cuuint64_t)heads; dims[2] = (cuuint64_t)p->rows_total;
    strides[0] = d * esz; strides[1] = (cuuint64_t)heads * d * esz;
    box[0] = box_cols; box[1] = 1; box[2] = (cuuint32_t)box_rows;
  }
  const CUtensorMapDataType dt = one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : (p->dtype == RF_BF16 && elem == kElemPlan) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return rf_fail(RF_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return RF_OK;
}

// Tensor map over precision "fp8"'s transposed E4M3 V codes, uint8
// [n2 * t_qblk][D][128]: one 128 x 128-byte box (128-byte swizzle) per block.
rf_status_t make_map_v8(CUtensorMap* m, const rf_plan* p, const void* base) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return rf_fail(RF_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const RfGeomDev& g = p->g;
  const cuuint64_t d = (cuuint64_t)g.d;
  cuuint64_t dims[3] = {(cuuint64_t)RF_BLOCK, d, (cuuint64_t)g.n2 * (cuuint64_t)g.t_qblk};
  cuuint64_t strides[2] = {(cuuint64_t)RF_BLOCK, (cuuint64_t)RF_BLOCK * d};
  cuuint32_t box[3] = {(cuuint32_t)RF_BLOCK, (cuuint32_t)g.d, 1}, estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return rf_fail(RF_ERR_CUDA, "cuTensorMapEncodeTiled (fp8 V) failed: " + std::to_string((int)r));
  return RF_OK;
}

template <int D, bool kBf16, bool kQk8, bool kMx = false, bool kPv8 = false>
rf_status_t launch_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const AttnArgs& args, unsigned grid, cudaStream_t st) {
  size_t smem = sizeof(AttnSmem<D, kQk8, kPv8>) + 1024;
  // D = 64 tiles are small: ask for enough shared memory that one CTA holds
  // an SM, since each CTA takes all 512 TMEM columns.
  if (smem < 120 * 1024) smem = 120 * 1024;
  auto kern = rf_attn_kernel<D, kBf16, kQk8, kMx, kPv8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return rf_check_launch("cudaFuncSetAttribute(rf_attn_kernel)");
  // The warpgroup register split (setmaxnreg) assumes exactly kLaunchRegs per
  // thread at launch; with fewer, the softmax groups' request could never be
  // met.  Refuse to launch a build that differs.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
    return rf_check_launch("cudaFuncGetAttributes(rf_attn_kernel)");
  if (fa.numRegs != kLaunchRegs)
    return rf_fail(RF_ERR_CUDA, "rf_attn_kernel built with " + std::to_string(fa.numRegs) +
                                    " registers per thread; the register split needs " +
                                    std::to_string(kLaunchRegs));
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, args);
  return rf_check_launch("rf_attn_kernel");
}

}  // namespace

rf_status_t rf_launch_attn(const rf_plan* p, const void* q_r, const void* k_r, const void* v_r,
                           const int32_t* sel_idx, const int32_t* sel_num, float scale, void* o_r,
                           void* ws, cudaStream_t st) {
  const RfGeomDev& g = p->g;
  const long long grid = (long long)g.t_qblk * g.n1;
  if (grid == 0) return RF_OK;
  if (grid > 0x7FFFFFFFll) return rf_fail(RF_ERR_INVALID_ARG, "grid too large");
  CUtensorMap mq, mk, mv;
  rf_status_t s;
  // precision "mix": Q K^T reads the E4M3 copies rf_rearrange wrote into ws;
  // precision "mxfp4": every operand reads the MXFP4 copies in ws (V as f16).
  const bool fp8 = p->precision == RF_PRECISION_FP8;
  const bool mx = p->precision == RF_PRECISION_MXFP4;
  const bool mx8 = mx && g.d == 128;                           // MXFP4 values in E4M3 carriers
  const bool mix = p->precision == RF_PRECISION_MIX || fp8 || mx8;   // E4M3 Q and K
  char* w = static_cast<char*>(ws);
  const void* qsrc = mix ? static_cast<const void*>(w + p->off_q8) : mx ? static_cast<const void*>(w + p->off_qx) : q_r;
  const void* ksrc = mix ? static_cast<const void*>(w + p->off_k8) : mx ? static_cast<const void*>(w + p->off_kx) : k_r;
  const void* vsrc = mx ? static_cast<const void*>(w + p->off_vx) : v_r;
  const MapElem qk_elem = mix ? kElemByte : kElemPlan;
  if ((s = make_map(&mq, p, qsrc, g.n1, qk_elem)) != RF_OK) return s;
  const int kv_box = g.block_kv == 64 ? 64 : RF_BLOCK;
  if ((s = make_map(&mk, p, ksrc, g.n2, qk_elem, kv_box)) != RF_OK) return s;
  if (fp8 || mx8) {
    if ((s = make_map_v8(&mv, p, w + p->off_v8)) != RF_OK) return s;
  } else if ((s = make_map(&mv, p, vsrc, g.n2, mx ? kElemF16 : kElemPlan, kv_box)) != RF_OK) {
    return s;
  }
  AttnArgs args;
  args.g = g;
  args.sel_idx = sel_idx;
  args.sel_num = sel_num;
  args.o_r = static_cast<uint16_t*>(o_r);
  args.status = reinterpret_cast<uint32_t*>(w + p->off_status);
  args.q_scale = (mix && !mx8) ? reinterpret_cast<const float*>(w + p->off_qs) : nullptr;
  args.k_scale = (mix && !mx8) ? reinterpret_cast<const float*>(w + p->off_ks) : nullptr;
  args.v_exp = fp8 ? reinterpret_cast<const int32_t*>(w + p->off_vexp) : nullptr;
  args.sl2 = scale * kLog2e;
  const bool bf = p->dtype == RF_BF16;
  if (g.d == 128) {
    if (mx8)
      return bf ? launch_t<128, true, true, true, true>(mq, mk, mv, args, (unsigned)grid, st)
                : launch_t<128, false, true, true, true>(mq, mk, mv, args, (unsigned)grid, st);
    if (fp8)
      return bf ? launch_t<128, true, true, false, true>(mq, mk, mv, args, (unsigned)grid, st)
                : launch_t<128, false, true, false, true>(mq, mk, mv, args, (unsigned)grid, st);
    if (mix)
      return bf ? launch_t<128, true, true>(mq, mk, mv, args, (unsigned)grid, st)
                : launch_t<128, false, true>(mq, mk, mv, args, (unsigned)grid, st);
    if (mx)
      return bf ? launch_t<128, true, false, true>(mq, mk, mv, args, (unsigned)grid, st)
                : launch_t<128, false, false, true>(mq, mk, mv, args, (unsigned)grid, st);
    return bf ? launch_t<128, true, false>(mq, mk, mv, args, (unsigned)grid, st)
              : launch_t<128, false, false>(mq, mk, mv, args, (unsigned)grid, st);
  }
  if (mx)
    return bf ? launch_t<64, true, false, true>(mq, mk, mv, args, (unsigned)grid, st)
              : launch_t<64, false, false, true>(mq, mk, mv, args, (unsigned)grid, st);
  return bf ? launch_t<64, true, false>(mq, mk, mv, args, (unsigned)grid, st)
            : launch_t<64, false, false>(mq, mk, mv, args, (unsigned)grid, st);
}

rf_status_t rf_launch_exp2_selftest(const float* x, float* y_poly, float* y_mufu, int64_t n,
                                    cudaStream_t st) {
  if (n <= 0) return RF_OK;
  rf_exp2_selftest_kernel<<<1184, 256, 0, st>>>(x, y_poly, y_mufu, (long long)n);
  return rf_check_launch("rf_exp2_selftest_kernel");
}
