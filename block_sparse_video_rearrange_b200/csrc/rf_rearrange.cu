// Token permutation kernels (HBM-bound): rf_rearrange for Q, K and V in one
// launch with the block means of Q and K fused in, the inverse permutation of
// the output, and stand-alone block-mean and E4M3 passes over
// already-rearranged tensors.
//
// "RainFusion Attention" user guide, opening paragraph and "Geometry
// handling": video tokens are arranged in (t, h, w) order with a misaligned
// suffix promoted to the dense prefix; xllm PR #1867 summary: Q, K and V are
// permuted in one call and an inverse restores the original order;
// RainFusion2.0 abstract, insight 1: block means serve as the representative
// token of each 128-token block.
//
// With precision "mix" the rearrange also writes an E4M3 copy of each Q and K
// block with its fp32 scale (amax / 448) while the block is in registers;
// with precision "fp8" also an E4M3 copy of each V block on a power-of-two
// scale, transposed through shared memory (the layout P V's B operand needs).
// With precision "mxfp4" it writes MXFP4-rounded copies instead: Q and K rows
// in groups of 32 columns, V columns in groups of 32 rows of each block, each
// group on its UOS power-of-two scale, stored as the exact 16-bit values.
//
// One CTA moves one 128-row block of one head of one tensor: 16-byte vector
// loads and stores, whole rows per group of D/8 threads, every load of a
// thread issued before its first store.  The source of a rearranged row is
// computed from the geometry (no index table in memory), once per row into
// shared memory, so that the copy loop runs no index arithmetic.
#include <cuda_fp16.h>

#include "rf_device.cuh"

namespace {

enum Mode { kRearrange = 0, kInverse = 1, kPoolOnly = 2, kQuantOnly = 3 };
enum Quant { kQuantNone = 0, kQuantE4M3 = 1, kQuantMx = 2, kQuantFp8 = 3 };

// Outputs of the fused quantization.  Precision "mix": one-byte E4M3 copies of
// Q' and K' in their layouts and one fp32 scale per (head, global block).
// Precision "mxfp4": MXFP4-rounded copies of Q' and K' (input dtype) and of V'
// (always f16, the type of the P V product), in the layouts of q_r, k_r, v_r.
// Precision "fp8": the "mix" outputs, and E4M3 codes of V' transposed per block
// ([n2][t_qblk][D][128] bytes) with one power-of-two exponent per (head, block).
struct QuantOut {
  uint8_t* q8;
  uint8_t* k8;
  float* q_scale;
  float* k_scale;
  uint4* qx;
  uint4* kx;
  uint4* vx;
  uint8_t* v8;
  int32_t* v_exp;
};

// Eight 16-bit values (one 16-byte chunk) rounded to MXFP4, element i on
// shared exponent e[i]: E2M1(x / 2^e) * 2^e, packed as kOutBf16 ? bf16 : f16.
// f16 results saturate at +-65504 (a V group whose rounding would go beyond).
template <class Dec, bool kOutBf16>
__device__ __forceinline__ uint4 rf_mx_round8(const uint4 v, const int* e) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int e0 = e[2 * c], e1 = e[2 * c + 1];
    const uint32_t h = rf_e2m1x2_round(rf_scale_pow2(Dec::lo(w[c]), -e0), rf_scale_pow2(Dec::hi(w[c]), -e1));
    float y0 = rf_scale_pow2(__half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu))), e0);
    float y1 = rf_scale_pow2(__half2float(__ushort_as_half((unsigned short)(h >> 16))), e1);
    if (!kOutBf16) {
      y0 = fminf(fmaxf(y0, -65504.f), 65504.f);
      y1 = fminf(fmaxf(y1, -65504.f), 65504.f);
    }
    o[c] = rf_pack2<kOutBf16>(y0, y1);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The same rounding, the eight values returned as floats (exact: E2M1 times a
// power of two).
template <class Dec>
__device__ __forceinline__ void rf_mx_round8f(const uint4 v, const int* e, float* y) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int e0 = e[2 * c], e1 = e[2 * c + 1];
    const uint32_t h = rf_e2m1x2_round(rf_scale_pow2(Dec::lo(w[c]), -e0), rf_scale_pow2(Dec::hi(w[c]), -e1));
    y[2 * c] = rf_scale_pow2(__half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu))), e0);
    y[2 * c + 1] = rf_scale_pow2(__half2float(__ushort_as_half((unsigned short)(h >> 16))), e1);
  }
}

// Four floats to four E4M3 codes (round to nearest even, saturating at
// +-448), the first in the lowest byte.
__device__ __forceinline__ uint32_t rf_e4m3x4(float a, float b, float c, float d) {
  unsigned short lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

constexpr int kThreads = 256;

// How the fused pooling reads the two 16-bit values packed in a 32-bit word.
struct DecodeBf16 {
  static constexpr bool kBf16 = true;
  __device__ static float lo(uint32_t w) { return __uint_as_float(w << 16); }
  __device__ static float hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
};
struct DecodeF16 {
  static constexpr bool kBf16 = false;
  __device__ static float lo(uint32_t w) {
    return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
  }
  __device__ static float hi(uint32_t w) {
    return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
  }
};

template <int D, int MODE, class Dec, int kQuant>
__global__ void __launch_bounds__(kThreads)
    rf_permute_kernel(const RfGeomDev g, const uint4* __restrict__ q, const uint4* __restrict__ k,
                      const uint4* __restrict__ v, uint4* __restrict__ q_out,
                      uint4* __restrict__ k_out, uint4* __restrict__ v_out,
                      float* __restrict__ pooled_q, float* __restrict__ pooled_k, const QuantOut qo) {
  constexpr int kChunks = D / 8;                  // 16-byte chunks per row
  constexpr int kRowLanes = kThreads / kChunks;   // rows handled in parallel
  constexpr int kRowsPerThread = RF_BLOCK / kRowLanes;
  __shared__ float red[kRowLanes][D + 4];
  __shared__ long long src_off[RF_BLOCK], dst_off[RF_BLOCK];  // row offsets in 16-byte units
  __shared__ uint32_t amax_w[kThreads / 32];

  const int tb = blockIdx.x % g.t_qblk;           // global block
  const int th = blockIdx.x / g.t_qblk;           // tensor-major head index
  int tensor, head, heads;
  if (MODE == kInverse || th < g.n1) {
    tensor = 0; head = th; heads = g.n1;
  } else if (th < g.n1 + g.n2) {
    tensor = 1; head = th - g.n1; heads = g.n2;
  } else {
    tensor = 2; head = th - g.n1 - g.n2; heads = g.n2;
  }
  const RfSeqDev& s = g.seq[rf_seq_of_qblk(g, tb)];
  const int b = tb - s.qblk_off;
  int r0, nrows;
  rf_block_span(s, b, r0, nrows);
  const bool pool = (MODE == kRearrange || MODE == kPoolOnly) && tensor < 2 && b >= s.n_pb;
  if (MODE == kPoolOnly && !pool) return;

  const uint4* src = tensor == 0 ? q : (tensor == 1 ? k : v);
  uint4* dst = tensor == 0 ? q_out : (tensor == 1 ? k_out : v_out);
  const int ch = threadIdx.x % kChunks;
  const int rl = threadIdx.x / kChunks;

  // Source and destination of every row, computed once per row (not once per
  // 16-byte chunk): the permutation's divisions stay off the copy loop.
  if (threadIdx.x < nrows) {
    const int r = r0 + (int)threadIdx.x;
    const int from = (MODE == kRearrange) ? rf_orig_row(s, r) : r;
    const int to = (MODE == kInverse) ? rf_orig_row(s, r) : r;
    src_off[threadIdx.x] = (long long)(rf_row_offset(g, s, heads, head, from) / 8);
    dst_off[threadIdx.x] = (long long)(rf_row_offset(g, s, heads, head, to) / 8);
  }
  __syncthreads();

  uint4 val[kRowsPerThread];
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i) {
    const int rr = rl + i * kRowLanes;
    val[i] = make_uint4(0, 0, 0, 0);
    if (rr < nrows) val[i] = __ldg(src + src_off[rr] + ch);
  }
  if (MODE == kRearrange || MODE == kInverse) {
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int rr = rl + i * kRowLanes;
      if (rr < nrows) dst[dst_off[rr] + ch] = val[i];
    }
  }
  if constexpr (kQuant == kQuantMx && (MODE == kRearrange || MODE == kQuantOnly)) {
    constexpr bool kInBf16 = Dec::kBf16;
    // D = 128: the rounded values are stored as E4M3 codes (every MXFP4 value
    // c * 2^e with -8 <= e <= 6 is one), Q' and K' one byte per element in
    // their layouts, V' transposed per block like precision fp8's.
    constexpr bool kMx8 = D == 128;
    if (tensor < 2) {
      // Q and K: every row in groups of 32 columns.  A group is four 16-byte
      // chunks, held by four consecutive lanes (kChunks is a multiple of 4).
      uint4* dstx = tensor == 0 ? qo.qx : qo.kx;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int rr = rl + i * kRowLanes;
        uint32_t mb = __vmaxu2(__vmaxu2(val[i].x & 0x7FFF7FFFu, val[i].y & 0x7FFF7FFFu),
                               __vmaxu2(val[i].z & 0x7FFF7FFFu, val[i].w & 0x7FFF7FFFu));
        mb = max(mb & 0xFFFFu, mb >> 16);
        mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
        mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
        const int e1 = rf_uos_exponent(Dec::lo(mb));
        const int e[8] = {e1, e1, e1, e1, e1, e1, e1, e1};
        if constexpr (kMx8) {
          if (rr < nrows) {
            float y[8];
            rf_mx_round8f<Dec>(val[i], e, y);
            uint8_t* dst8 = tensor == 0 ? qo.q8 : qo.k8;
            *reinterpret_cast<uint2*>(dst8 + dst_off[rr] * 8 + ch * 8) =
                make_uint2(rf_e4m3x4(y[0], y[1], y[2], y[3]), rf_e4m3x4(y[4], y[5], y[6], y[7]));
          }
        } else {
          if (rr < nrows) dstx[dst_off[rr] + ch] = rf_mx_round8<Dec, kInBf16>(val[i], e);
        }
      }
    } else {
      // V: every column in groups of 32 rows counted from the block's first
      // row (rows past nrows hold zeros and do not raise a group's maximum).
      // A thread holds kRowsPerGroup rows of each group; the other rows of the
      // group sit with the other row lanes of the same chunk.
      constexpr int kRowsPerGroup = 32 / kRowLanes;
      constexpr int kGroups = RF_BLOCK / 32;
      constexpr int kWords = D / 2;  // packed 16-bit pairs per row
      __shared__ uint32_t part[kGroups][kRowLanes][kWords];
      __shared__ uint32_t gmax[kGroups][kWords];
      constexpr int kVTileStride = RF_BLOCK + 4;   // bytes per row of the transposed tile
      __shared__ __align__(16) uint8_t vtile[kMx8 ? D * kVTileStride : 16];
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        uint32_t m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < kRowsPerGroup; ++j) {
          const uint4 x = val[gi * kRowsPerGroup + j];
          m4[0] = __vmaxu2(m4[0], x.x & 0x7FFF7FFFu);
          m4[1] = __vmaxu2(m4[1], x.y & 0x7FFF7FFFu);
          m4[2] = __vmaxu2(m4[2], x.z & 0x7FFF7FFFu);
          m4[3] = __vmaxu2(m4[3], x.w & 0x7FFF7FFFu);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) part[gi][rl][ch * 4 + c] = m4[c];
      }
      __syncthreads();
      if (threadIdx.x < kGroups * kWords) {
        const int gi = threadIdx.x / kWords, wd = threadIdx.x % kWords;
        uint32_t m = 0u;
#pragma unroll 4
        for (int l = 0; l < kRowLanes; ++l) m = __vmaxu2(m, part[gi][l][wd]);
        gmax[gi][wd] = m;
      }
      __syncthreads();
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        int e[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t m = gmax[gi][ch * 4 + c];
          e[2 * c] = rf_uos_exponent(Dec::lo(m));
          e[2 * c + 1] = rf_uos_exponent(Dec::hi(m));
        }
#pragma unroll
        for (int j = 0; j < kRowsPerGroup; ++j) {
          const int i = gi * kRowsPerGroup + j;
          const int rr = rl + i * kRowLanes;
          if constexpr (kMx8) {
            // rows past nrows hold zeros: code 0
            float y[8];
            rf_mx_round8f<Dec>(val[i], e, y);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
              unsigned short two;
              asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(y[c + 1]), "f"(y[c]));
              vtile[(ch * 8 + c) * kVTileStride + rr] = (uint8_t)(two & 0xFFu);
              vtile[(ch * 8 + c + 1) * kVTileStride + rr] = (uint8_t)(two >> 8);
            }
          } else {
            if (rr < nrows) qo.vx[dst_off[rr] + ch] = rf_mx_round8<Dec, false>(val[i], e);
          }
        }
      }
      if constexpr (kMx8) {
        __syncthreads();
        uint32_t* out = reinterpret_cast<uint32_t*>(qo.v8 + ((size_t)head * g.t_qblk + tb) * (size_t)(RF_BLOCK * D));
        for (int wd = threadIdx.x; wd < D * RF_BLOCK / 4; wd += kThreads) {
          const int d = wd / (RF_BLOCK / 4), c4 = wd % (RF_BLOCK / 4);
          out[wd] = *reinterpret_cast<const uint32_t*>(&vtile[d * kVTileStride + 4 * c4]);
        }
      }
    }
  }
  if constexpr ((kQuant == kQuantE4M3 || kQuant == kQuantFp8) && (MODE == kRearrange || MODE == kQuantOnly)) {
    if (tensor < 2) {  // uniform over the CTA: Q and K blocks get an E4M3 copy
      // amax over the block's valid rows (rows past nrows hold zeros).  For
      // finite bf16 and fp16 alike |x| orders as the 15-bit magnitude field,
      // so a packed unsigned 16-bit max of the masked words finds the largest
      // magnitude two elements at a time.
      uint32_t mb = 0u;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        mb = __vmaxu2(mb, val[i].x & 0x7FFF7FFFu);
        mb = __vmaxu2(mb, val[i].y & 0x7FFF7FFFu);
        mb = __vmaxu2(mb, val[i].z & 0x7FFF7FFFu);
        mb = __vmaxu2(mb, val[i].w & 0x7FFF7FFFu);
      }
      mb = __reduce_max_sync(0xffffffffu, max(mb & 0xFFFFu, mb >> 16));
      if ((threadIdx.x & 31) == 0) amax_w[threadIdx.x >> 5] = mb;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < kThreads / 32; ++i) mb = max(mb, amax_w[i]);
      const float amax = Dec::lo(mb);
      const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f;
      const uint64_t inv2 = rf_f2(__float_as_uint(inv), __float_as_uint(inv));
      uint8_t* dst8 = tensor == 0 ? qo.q8 : qo.k8;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int rr = rl + i * kRowLanes;
        if (rr < nrows) {
          const uint32_t w[4] = {val[i].x, val[i].y, val[i].z, val[i].w};
          float y[8];
#pragma unroll
          for (int c = 0; c < 4; ++c)   // x * inv, one IEEE fp32 multiply per element, two per instruction
            rf_f2_split(rf_mul2(rf_f2(__float_as_uint(Dec::lo(w[c])), __float_as_uint(Dec::hi(w[c]))), inv2),
                        y[2 * c], y[2 * c + 1]);
          const uint32_t lo = rf_e4m3x4(y[0], y[1], y[2], y[3]);
          const uint32_t hi = rf_e4m3x4(y[4], y[5], y[6], y[7]);
          // dst_off is in 16-byte units of the 16-bit tensor: 8 elements each.
          *reinterpret_cast<uint2*>(dst8 + dst_off[rr] * 8 + ch * 8) = make_uint2(lo, hi);
        }
      }
      if (threadIdx.x == 0) {
        float* sc = tensor == 0 ? qo.q_scale : qo.k_scale;
        sc[(size_t)head * g.t_qblk + tb] = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      }
    } else if constexpr (kQuant == kQuantFp8) {
      // V (precision "fp8"): E4M3 codes of v * 2^-e, e the smallest integer
      // with amax <= 448 * 2^e (amax / 448 is a correctly rounded division and
      // amax a 16-bit value, so a boundary amax = 448 * 2^k gives exactly 2^k),
      // written transposed: column c of the block holds its 128 keys together.
      constexpr int kTileStride = RF_BLOCK + 4;   // bytes per tile row (33 words)
      __shared__ __align__(16) uint8_t tile[D * kTileStride];
      uint32_t mb = 0u;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        mb = __vmaxu2(mb, val[i].x & 0x7FFF7FFFu);
        mb = __vmaxu2(mb, val[i].y & 0x7FFF7FFFu);
        mb = __vmaxu2(mb, val[i].z & 0x7FFF7FFFu);
        mb = __vmaxu2(mb, val[i].w & 0x7FFF7FFFu);
      }
      mb = __reduce_max_sync(0xffffffffu, max(mb & 0xFFFFu, mb >> 16));
      if ((threadIdx.x & 31) == 0) amax_w[threadIdx.x >> 5] = mb;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < kThreads / 32; ++i) mb = max(mb, amax_w[i]);
      const float amax = Dec::lo(mb);
      // an all-zero block takes the smallest exponent: it never sets a row's largest
      const int e = amax > 0.f ? rf_ceil_log2(__fdiv_rn(amax, 448.0f)) : -127;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int rr = rl + i * kRowLanes;       // rows past nrows hold zeros: code 0
        const uint32_t w[4] = {val[i].x, val[i].y, val[i].z, val[i].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          unsigned short two;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
              : "=h"(two) : "f"(rf_scale_pow2(Dec::hi(w[c]), -e)), "f"(rf_scale_pow2(Dec::lo(w[c]), -e)));
          tile[(ch * 8 + 2 * c) * kTileStride + rr] = (uint8_t)(two & 0xFFu);
          tile[(ch * 8 + 2 * c + 1) * kTileStride + rr] = (uint8_t)(two >> 8);
        }
      }
      __syncthreads();
      uint32_t* out = reinterpret_cast<uint32_t*>(qo.v8 + ((size_t)head * g.t_qblk + tb) * (size_t)(RF_BLOCK * D));
      for (int wd = threadIdx.x; wd < D * RF_BLOCK / 4; wd += kThreads) {
        const int d = wd / (RF_BLOCK / 4), c4 = wd % (RF_BLOCK / 4);
        out[wd] = *reinterpret_cast<const uint32_t*>(&tile[d * kTileStride + 4 * c4]);
      }
      if (threadIdx.x == 0) qo.v_exp[(size_t)head * g.t_qblk + tb] = e;
    }
  }
  if constexpr (MODE == kInverse || MODE == kQuantOnly) {
    return;
  } else {
    if (!pool) return;  // uniform over the CTA

    // Column sums of the block in fp32 and a fixed order (a lane's rows in
    // order, then the lanes in order), then the mean.  Q is pooled over the
    // block's 128 rows.  K is pooled over its key blocks: the same 128 rows,
    // or with 64-row key blocks each half on its own (row lane rl holds rows
    // rl + i * kRowLanes and kRowLanes divides 64, so the first half of every
    // lane's rows is rows 0-63), summed into a second accumulator in the same
    // pass so that no row value outlives its own addition.
    const bool split = tensor == 1 && g.block_kv == 64;  // uniform over the CTA
    static_assert(64 % kRowLanes == 0 && kRowsPerThread % 2 == 0, "64-row halves must split the row lanes");
    float acc[8], acc2[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = acc2[c] = 0.f;
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const uint32_t w[4] = {val[i].x, val[i].y, val[i].z, val[i].w};
      const bool second = split && i >= kRowsPerThread / 2;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (second) {
          acc2[2 * c] += Dec::lo(w[c]);
          acc2[2 * c + 1] += Dec::hi(w[c]);
        } else {
          acc[2 * c] += Dec::lo(w[c]);
          acc[2 * c + 1] += Dec::hi(w[c]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) red[rl][ch * 8 + c] = acc[c];
    __syncthreads();
    const float inv_rows = split ? 1.0f / 64 : 1.0f / RF_BLOCK;
    if (threadIdx.x < D) {
      float sum = 0.f;
#pragma unroll 4
      for (int l = 0; l < kRowLanes; ++l) sum += red[l][threadIdx.x];
      if (tensor == 0)
        pooled_q[((size_t)head * g.pooled_total + (size_t)(s.pool_off + b - s.n_pb)) * D + threadIdx.x] =
            sum * inv_rows;
      else
        pooled_k[((size_t)head * g.pooled_k_total + (size_t)(s.poolk_off + (split ? 2 : 1) * (b - s.n_pb))) * D +
                 threadIdx.x] = sum * inv_rows;
    }
    if (split) {
      __syncthreads();  // the first half's sums have been read
#pragma unroll
      for (int c = 0; c < 8; ++c) red[rl][ch * 8 + c] = acc2[c];
      __syncthreads();
      if (threadIdx.x < D) {
        float sum = 0.f;
#pragma unroll 4
        for (int l = 0; l < kRowLanes; ++l) sum += red[l][threadIdx.x];
        pooled_k[((size_t)head * g.pooled_k_total + (size_t)(s.poolk_off + 2 * (b - s.n_pb) + 1)) * D +
                 threadIdx.x] = sum * inv_rows;
      }
    }
  }
}

template <int MODE>
rf_status_t launch(const rf_plan* p, const void* q, const void* k, const void* v, void* qo,
                   void* ko, void* vo, void* ws, cudaStream_t st, int tensor_heads) {
  const RfGeomDev& g = p->g;
  const long long grid = (long long)g.t_qblk * tensor_heads;
  if (grid == 0) return RF_OK;
  if (grid > 0x7FFFFFFFll) return rf_fail(RF_ERR_INVALID_ARG, "grid too large");
  char* w = static_cast<char*>(ws);
  float* pq = ws ? reinterpret_cast<float*>(w + p->off_pq) : nullptr;
  float* pk = ws ? reinterpret_cast<float*>(w + p->off_pk) : nullptr;
  const bool quant_stage = MODE == kRearrange || MODE == kQuantOnly;
  const bool fp8 = quant_stage && p->precision == RF_PRECISION_FP8;
  const bool quant = quant_stage && (p->precision == RF_PRECISION_MIX || fp8);
  const bool mx = quant_stage && p->precision == RF_PRECISION_MXFP4;
  QuantOut qout{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  if (fp8) {
    qout.v8 = reinterpret_cast<uint8_t*>(w + p->off_v8);
    qout.v_exp = reinterpret_cast<int32_t*>(w + p->off_vexp);
  }
  if (quant) {
    qout.q8 = reinterpret_cast<uint8_t*>(w + p->off_q8);
    qout.k8 = reinterpret_cast<uint8_t*>(w + p->off_k8);
    qout.q_scale = reinterpret_cast<float*>(w + p->off_qs);
    qout.k_scale = reinterpret_cast<float*>(w + p->off_ks);
  }
  if (mx && g.d == 128) {   // E4M3 carriers of the MXFP4 values
    qout.q8 = reinterpret_cast<uint8_t*>(w + p->off_q8);
    qout.k8 = reinterpret_cast<uint8_t*>(w + p->off_k8);
    qout.v8 = reinterpret_cast<uint8_t*>(w + p->off_v8);
  } else if (mx) {
    qout.qx = reinterpret_cast<uint4*>(w + p->off_qx);
    qout.kx = reinterpret_cast<uint4*>(w + p->off_kx);
    qout.vx = reinterpret_cast<uint4*>(w + p->off_vx);
  }
  const uint4* a = static_cast<const uint4*>(q);
  const uint4* b = static_cast<const uint4*>(k);
  const uint4* c = static_cast<const uint4*>(v);
  uint4* x = static_cast<uint4*>(qo);
  uint4* y = static_cast<uint4*>(ko);
  uint4* z = static_cast<uint4*>(vo);
  const bool bf = p->dtype == RF_BF16;
  dim3 grd((unsigned)grid), blk(kThreads);
  if (g.d == 128) {
    if (fp8) {
      if (bf) rf_permute_kernel<128, MODE, DecodeBf16, kQuantFp8><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
      else    rf_permute_kernel<128, MODE, DecodeF16, kQuantFp8><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
    } else if (quant) {
      // precision mix is built for D = 128 only (checked when the plan is made)
      if (bf) rf_permute_kernel<128, MODE, DecodeBf16, kQuantE4M3><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
      else    rf_permute_kernel<128, MODE, DecodeF16, kQuantE4M3><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
    } else if (mx) {
      if (bf) rf_permute_kernel<128, MODE, DecodeBf16, kQuantMx><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
      else    rf_permute_kernel<128, MODE, DecodeF16, kQuantMx><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
    } else {
      if (bf) rf_permute_kernel<128, MODE, DecodeBf16, kQuantNone><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
      else    rf_permute_kernel<128, MODE, DecodeF16, kQuantNone><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
    }
  } else if (mx) {
    if (bf) rf_permute_kernel<64, MODE, DecodeBf16, kQuantMx><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
    else    rf_permute_kernel<64, MODE, DecodeF16, kQuantMx><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
  } else {
    if (bf) rf_permute_kernel<64, MODE, DecodeBf16, kQuantNone><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
    else    rf_permute_kernel<64, MODE, DecodeF16, kQuantNone><<<grd, blk, 0, st>>>(g, a, b, c, x, y, z, pq, pk, qout);
  }
  return rf_check_launch("rf_permute_kernel");
}

}  // namespace

rf_status_t rf_launch_rearrange(const rf_plan* p, const void* q, const void* k, const void* v,
                                void* q_r, void* k_r, void* v_r, void* ws, cudaStream_t st) {
  return launch<kRearrange>(p, q, k, v, q_r, k_r, v_r, ws, st, p->g.n1 + 2 * p->g.n2);
}

rf_status_t rf_launch_pool(const rf_plan* p, const void* q_r, const void* k_r, void* ws,
                           cudaStream_t st) {
  return launch<kPoolOnly>(p, q_r, k_r, nullptr, nullptr, nullptr, nullptr, ws, st,
                           p->g.n1 + p->g.n2);
}

rf_status_t rf_launch_quantize(const rf_plan* p, const void* q_r, const void* k_r, const void* v_r,
                               void* ws, cudaStream_t st) {
  // mix quantizes Q and K; fp8 and mxfp4 also V (the third tensor's heads)
  const int heads = p->g.n1 + p->g.n2 + (p->precision == RF_PRECISION_MIX ? 0 : p->g.n2);
  return launch<kQuantOnly>(p, q_r, k_r, v_r, nullptr, nullptr, nullptr, ws, st, heads);
}

rf_status_t rf_launch_inverse(const rf_plan* p, const void* o_r, void* o, cudaStream_t st) {
  return launch<kInverse>(p, o_r, nullptr, nullptr, o, nullptr, nullptr, nullptr, st, p->g.n1);
}
