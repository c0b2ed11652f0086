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
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread = query row = TMEM lane
//   warp 4     TMA producer: Q once, then K_j / V_j of each selected block
//              through a kStages-deep ring of shared-memory stages
//   warp 5     TMEM allocation and the single-thread tcgen05.mma issue
// TMEM columns: S double buffer [0,128) and [128,256) (fp32 128 x 128), O at
// [256, 256 + D) (fp32 128 x D).  P is written back over its own S buffer as
// packed 16-bit pairs and is the A operand (from TMEM) of O += P V.
// Pipeline per selected block j:
//   MMA:     S_{j+1} = Q K_{j+1}^T   (overlaps softmax of block j)
//   softmax: m, p = exp2(s * scale * log2e - m), l += sum p, P_j -> TMEM;
//            O is rescaled only when the row max grows by more than 2^8
//   MMA:     O += P_j V_j
// Every wait is bounded: on expiry the CTA records it in the status words and
// unwinds (waiting, again bounded, for its own copies and MMAs in flight).
#include <cuda.h>

#include <mutex>

#include "rf_device.cuh"

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: lazy rescale while growth <= 256x

template <int D>
struct __align__(1024) AttnSmem {
  static constexpr int kTileBytes = RF_BLOCK * D * 2;  // 128 rows x D x 16-bit
  uint8_t q[kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t bar_q;
  uint64_t bar_k_full[kStages], bar_k_empty[kStages];
  uint64_t bar_v_full[kStages], bar_v_empty[kStages];
  uint64_t bar_s_full[2], bar_p_full[2];
  uint64_t bar_o_done;
  uint64_t bar_drain;
  uint32_t tmem_base;
  int abort;
  int n_valid;
  int list[RF_MAX_KV_LIST];
};

struct AttnArgs {
  RfGeomDev g;
  const int32_t* sel_idx;
  const int32_t* sel_num;
  uint16_t* o_r;
  uint32_t* status;
  float sl2;  // scale * log2(e)
};

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

__device__ __forceinline__ void record_timeout(volatile int* abort, uint32_t* status, int where) {
  *abort = 1;
  atomicOr(status + RF_STATUS_TIMEOUT, 1u << where);
}

template <int D, bool kBf16>
__global__ void __launch_bounds__(kThreads, 1)
    rf_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D>& sm = *reinterpret_cast<AttnSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int kBoxes = D / 64;  // 64-column (128-byte) swizzle boxes per tile row
  constexpr uint32_t kTileBytes = AttnSmem<D>::kTileBytes;
  constexpr uint32_t kBoxBytes = RF_BLOCK * 128;

  const RfGeomDev& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x / g.t_qblk;  // query head (head-major order)
  const int tb = blockIdx.x % g.t_qblk;
  const RfSeqDev& s = g.seq[rf_seq_of_qblk(g, tb)];
  const int qb = tb - s.qblk_off;
  const int nblk = s.n_pb + s.nb;
  const int gk = n / (g.n1 / g.n2);  // key/value head
  int q_r0, q_rows;
  rf_block_span(s, qb, q_r0, q_rows);
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    mbar_init(rf_smem_u32(&sm.bar_q), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(rf_smem_u32(&sm.bar_k_full[i]), 1);
      mbar_init(rf_smem_u32(&sm.bar_k_empty[i]), 1);
      mbar_init(rf_smem_u32(&sm.bar_v_full[i]), 1);
      mbar_init(rf_smem_u32(&sm.bar_v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(rf_smem_u32(&sm.bar_s_full[i]), 1);
      mbar_init(rf_smem_u32(&sm.bar_p_full[i]), 128);
    }
    mbar_init(rf_smem_u32(&sm.bar_o_done), 1);
    mbar_init(rf_smem_u32(&sm.bar_drain), 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 5) {
    tmem_alloc(rf_smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) {
    // Compact the selectIdx row: keep in-range entries in order, skip -1
    // (an unused slot), count anything else as a bad index.
    const size_t row_id = (size_t)tb * g.n1 + n;
    const int32_t* row = a.sel_idx + row_id * g.max_kv;
    int num = a.sel_num[row_id];
    int bad = 0;
    if (num < 0 || num > g.max_kv) {
      bad = 1;
      num = num < 0 ? 0 : g.max_kv;
    }
    int cnt = 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int c0 = 0; c0 < num; c0 += 32) {
      const int c = c0 + lane;
      const int v = c < num ? row[c] : -1;
      const bool ok = c < num && v >= 0 && v < nblk;
      if (c < num && v != -1 && !ok) ++bad;
      const uint32_t ball = __ballot_sync(0xffffffffu, ok);
      if (ok) sm.list[cnt + __popc(ball & lt)] = v;
      cnt += __popc(ball);
    }
    bad = __reduce_add_sync(0xffffffffu, bad);
    if (lane == 0) {
      // A wait that already expired in this workspace (this launch or an
      // earlier one not yet cleared by rf_check_device_status) stops all work.
      const bool stopped = *reinterpret_cast<volatile uint32_t*>(a.status + RF_STATUS_TIMEOUT) != 0;
      sm.n_valid = stopped ? 0 : cnt;
      if (bad) atomicAdd(a.status + RF_STATUS_BAD_INDEX, (uint32_t)bad);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int nv = sm.n_valid;
  const int vr_last = s.Lp - (s.n_pb - 1) * RF_BLOCK;  // valid rows of the last prefix block

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && nv > 0) {
      const bool bnsd = g.layout == RF_LAYOUT_BNSD;
      auto coords = [&](int heads, int head, int r0, int& c1, int& c2) {
        if (bnsd) { c1 = r0; c2 = s.batch_idx * heads + head; }
        else      { c1 = head; c2 = (int)s.row_off + r0; }
      };
      int c1, c2;
      coords(g.n1, n, q_r0, c1, c2);
      const uint32_t bq = rf_smem_u32(&sm.bar_q);
      mbar_arrive_expect_tx(bq, kTileBytes);
#pragma unroll
      for (int x = 0; x < kBoxes; ++x)
        tma_load_3d(rf_smem_u32(sm.q + x * kBoxBytes), &tm_q, bq, x * 64, c1, c2);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nv; ++j) {
        const int st = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        if (j >= kStages && !mbar_wait(rf_smem_u32(&sm.bar_k_empty[st]), ph ^ 1, abort)) {
          record_timeout(abort, a.status, 0);
          break;
        }
        int r0, nr;
        rf_block_span(s, sm.list[j], r0, nr);
        coords(g.n2, gk, r0, c1, c2);
        const uint32_t bk = rf_smem_u32(&sm.bar_k_full[st]);
        mbar_arrive_expect_tx(bk, kTileBytes);
#pragma unroll
        for (int x = 0; x < kBoxes; ++x)
          tma_load_3d(rf_smem_u32(sm.k[st] + x * kBoxBytes), &tm_k, bk, x * 64, c1, c2);
        k_issued = j + 1;
        if (j >= kStages && !mbar_wait(rf_smem_u32(&sm.bar_v_empty[st]), ph ^ 1, abort)) {
          record_timeout(abort, a.status, 1);
          break;
        }
        const uint32_t bv = rf_smem_u32(&sm.bar_v_full[st]);
        mbar_arrive_expect_tx(bv, kTileBytes);
#pragma unroll
        for (int x = 0; x < kBoxes; ++x)
          tma_load_3d(rf_smem_u32(sm.v[st] + x * kBoxBytes), &tm_v, bv, x * 64, c1, c2);
        v_issued = j + 1;
      }
      if (*abort) {
        // Let this CTA's own copies land before its shared memory goes away:
        // the newest load of each stage completes last on that stage's barrier.
        volatile int no_abort = 0;
        mbar_wait(bq, 0, &no_abort);
        for (int j = (k_issued > kStages ? k_issued - kStages : 0); j < k_issued; ++j)
          mbar_wait(rf_smem_u32(&sm.bar_k_full[j % kStages]), (j / kStages) & 1, &no_abort);
        for (int j = (v_issued > kStages ? v_issued - kStages : 0); j < v_issued; ++j)
          mbar_wait(rf_smem_u32(&sm.bar_v_full[j % kStages]), (j / kStages) & 1, &no_abort);
      }
    }
  } else if (warp == 5) {
    // ---------------- tcgen05.mma issue (one thread) ----------------
    if (lane == 0 && nv > 0) {
      const uint32_t fmt = kBf16 ? 1u : 0u;
      const uint32_t idesc_qk = umma_idesc_f16(fmt, 128, 128, 0);
      const uint32_t idesc_pv = umma_idesc_f16(fmt, 128, D, 1);
      const uint32_t q_addr = rf_smem_u32(sm.q);
      auto issue_qk = [&](int j) {
        const int st = j % kStages, buf = j & 1;
        const uint32_t k_addr = rf_smem_u32(sm.k[st]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_ss(tmem + buf * 128, umma_desc_sw128(q_addr + off, 16, 1024),
                 umma_desc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(rf_smem_u32(&sm.bar_s_full[buf]));
        tc_commit(rf_smem_u32(&sm.bar_k_empty[st]));
      };
      bool ok = mbar_wait(rf_smem_u32(&sm.bar_q), 0, abort);
      if (ok) ok = mbar_wait(rf_smem_u32(&sm.bar_k_full[0]), 0, abort);
      if (ok) {
        tc_fence_after();
        issue_qk(0);
      }
      for (int j = 0; ok && j < nv; ++j) {
        if (j + 1 < nv) {
          const int st = (j + 1) % kStages;
          if (!mbar_wait(rf_smem_u32(&sm.bar_k_full[st]), ((j + 1) / kStages) & 1, abort)) { ok = false; break; }
          tc_fence_after();
          issue_qk(j + 1);
        }
        const int buf = j & 1, st = j % kStages;
        if (!mbar_wait(rf_smem_u32(&sm.bar_p_full[buf]), (j >> 1) & 1, abort)) { ok = false; break; }
        if (!mbar_wait(rf_smem_u32(&sm.bar_v_full[st]), (j / kStages) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t v_addr = rf_smem_u32(sm.v[st]);
#pragma unroll
        for (int kk = 0; kk < RF_BLOCK / 16; ++kk)
          mma_ts(tmem + 256, tmem + buf * 128 + kk * 8,
                 umma_desc_sw128(v_addr + kk * 2048, kBoxBytes, 1024), idesc_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(rf_smem_u32(&sm.bar_o_done));
        tc_commit(rf_smem_u32(&sm.bar_v_empty[st]));
      }
      if (!ok) record_timeout(abort, a.status, 2);
      // Drain: every MMA this thread issued has completed before TMEM is freed.
      tc_commit(rf_smem_u32(&sm.bar_drain));
      volatile int no_abort = 0;
      mbar_wait(rf_smem_u32(&sm.bar_drain), 0, &no_abort);
    }
  } else {
    // ---------------- softmax + epilogue (warps 0-3) ----------------
    const int row = warp * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = a.sl2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nv; ++j) {
      const int buf = j & 1;
      if (!warp_wait(rf_smem_u32(&sm.bar_s_full[buf]), (j >> 1) & 1, abort)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(lane_base + buf * 128 + 0, sr + 0);
      tmem_ld32(lane_base + buf * 128 + 32, sr + 32);
      tmem_ld32(lane_base + buf * 128 + 64, sr + 64);
      tmem_ld32(lane_base + buf * 128 + 96, sr + 96);
      tmem_wait_ld();
      const int vr = (sm.list[j] == s.n_pb - 1) ? vr_last : RF_BLOCK;  // uniform over the CTA
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (c < vr) mx = fmaxf(mx, __uint_as_float(sr[c]));
      const float mx_t = mx * sl2;
      if (__any_sync(0xffffffffu, mx_t > m_run + kRescaleThreshold)) {
        const float m_new = fmaxf(m_run, mx_t);
        const float alpha = rf_ex2(m_run - m_new);
        l_run *= alpha;
        if (j > 0) {
          // O holds P_0..P_{j-1} V: wait for the last of those MMAs, then rescale.
          if (!warp_wait(rf_smem_u32(&sm.bar_o_done), (j - 1) & 1, abort)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(lane_base + 256 + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(lane_base + 256 + c0, o);
          }
          tmem_wait_st();
        }
        m_run = m_new;
      }
      const float neg_m = -m_run;
      float sum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = c < vr ? rf_ex2(fmaf(__uint_as_float(sr[c]), sl2, neg_m)) : 0.f;
        const float p1 = c + 1 < vr ? rf_ex2(fmaf(__uint_as_float(sr[c + 1]), sl2, neg_m)) : 0.f;
        sum += p0 + p1;
        pk[c >> 1] = rf_pack2<kBf16>(p0, p1);
      }
      l_run += sum;
      tmem_st32(lane_base + buf * 128 + 0, pk + 0);
      tmem_st32(lane_base + buf * 128 + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(rf_smem_u32(&sm.bar_p_full[buf]));
    }
    if (!ok) record_timeout(abort, a.status, 3);
    // Epilogue: O / l -> 16-bit, rows of this query block only.
    const bool have_o = ok && nv > 0 && warp_wait(rf_smem_u32(&sm.bar_o_done), (nv - 1) & 1, abort);
    uint16_t* dst = a.o_r + rf_row_offset(g, s, g.n1, n, q_r0 + min(row, q_rows - 1));
    const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
    if (have_o) tc_fence_after();
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld32(lane_base + 256 + c0, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0u;
      }
      uint32_t w[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        w[c] = rf_pack2<kBf16>(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
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
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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

// Tensor map over [rows, heads, D] (TND) or [B*heads, rows, D] (BNSD) with a
// 128-row x 64-column box and 128-byte swizzle.
rf_status_t make_map(CUtensorMap* m, const rf_plan* p, const void* base, int heads) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return rf_fail(RF_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const RfGeomDev& g = p->g;
  const cuuint64_t d = (cuuint64_t)g.d;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  if (g.layout == RF_LAYOUT_BNSD) {
    const cuuint64_t L = (cuuint64_t)g.seq[0].L;
    dims[0] = d; dims[1] = L; dims[2] = (cuuint64_t)p->batch * heads;
    strides[0] = d * 2; strides[1] = L * d * 2;
    box[0] = 64; box[1] = RF_BLOCK; box[2] = 1;
  } else {
    dims[0] = d; dims[1] = (cuuint64_t)heads; dims[2] = (cuuint64_t)p->rows_total;
    strides[0] = d * 2; strides[1] = (cuuint64_t)heads * d * 2;
    box[0] = 64; box[1] = 1; box[2] = RF_BLOCK;
  }
  const CUtensorMapDataType dt =
      p->dtype == RF_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return rf_fail(RF_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return RF_OK;
}

template <int D, bool kBf16>
rf_status_t launch_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const AttnArgs& args, unsigned grid, cudaStream_t st) {
  size_t smem = sizeof(AttnSmem<D>) + 1024;
  // D = 64 tiles are small: ask for enough shared memory that one CTA holds
  // an SM, since each CTA takes all 512 TMEM columns.
  if (smem < 120 * 1024) smem = 120 * 1024;
  auto kern = rf_attn_kernel<D, kBf16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return rf_check_launch("cudaFuncSetAttribute(rf_attn_kernel)");
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
  if ((s = make_map(&mq, p, q_r, g.n1)) != RF_OK) return s;
  if ((s = make_map(&mk, p, k_r, g.n2)) != RF_OK) return s;
  if ((s = make_map(&mv, p, v_r, g.n2)) != RF_OK) return s;
  AttnArgs args;
  args.g = g;
  args.sel_idx = sel_idx;
  args.sel_num = sel_num;
  args.o_r = static_cast<uint16_t*>(o_r);
  args.status = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + p->off_status);
  args.sl2 = scale * kLog2e;
  const bool bf = p->dtype == RF_BF16;
  if (g.d == 128)
    return bf ? launch_t<128, true>(mq, mk, mv, args, (unsigned)grid, st)
              : launch_t<128, false>(mq, mk, mv, args, (unsigned)grid, st);
  return bf ? launch_t<64, true>(mq, mk, mv, args, (unsigned)grid, st)
            : launch_t<64, false>(mq, mk, mv, args, (unsigned)grid, st);
}
