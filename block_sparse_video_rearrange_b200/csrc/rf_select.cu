// Block ranking and selection: selectIdx / selectNum for every (query block,
// query head).
//
// "RainFusion Attention" user guide, opening paragraphs: key blocks are
// pooled, ranked per query block, and the highest-scoring ones are attended;
// prefix rows and first-frame blocks stay dense; segments under 32 blocks run
// dense.  "Configuration": sparsity is the nominal dropped fraction.
// "aclnnRainFusionAttention" API page, constraints: selectIdx is
// [T, headNum, maxKvBlockNum] with -1 in unused slots; selectNum is [T, headNum].
// RainFusion2.0 abstract: block means are the representative tokens; the
// first frame is a sink.
//
// Two kernels:
//  1. rf_scores_kernel: per sparse sequence and query head n, the fp32 matrix
//     scores[i][j] = qbar[n][i] . kbar[n / G][j] over the nb query blocks and
//     the nbk key blocks (nbk = nb, or 2 nb with blockShape 128 x 64, whose
//     key blocks of 64 rows are pooled over their own rows; [API] "Formula":
//     blocks of blockShapeX x blockShapeY) (128 x 128 or 64 x 64 tiles, 8 x 8
//     or 4 x 4 per thread, D chunks double-buffered through shared memory).
//  2. rf_topk_kernel: one warp per selectIdx row.  Keys are the scores mapped
//     to order-preserving 32-bit integers, held in registers (32 lanes x M).
//     A bitwise radix select (over the bits below the keys' common prefix)
//     finds the k-th largest key; ties at the
//     threshold go to the lowest block index; sinks are added; the row is
//     written in ascending order with a ballot prefix sum.  No sorting, no
//     shared memory, no atomics.
#include "rf_device.cuh"

namespace {

constexpr int kKc = 16;  // D chunk staged through shared memory (double-buffered)

// One CTA computes a (16 TT) x (16 TT) tile of scores for one (sequence, query
// head): 256 threads, TT x TT results each (rows q*64 + ty*4 + {0..3} for the
// TT/4 quadrants q, columns likewise with tx), so every inner step is TT/2
// 16-byte shared loads feeding TT*TT fp32 FMAs.  The next D chunk is fetched
// into registers while the current one is multiplied.  TT = 8 (128 x 128
// tiles) for large problems, TT = 4 (64 x 64) when the large tiles would not
// fill the GPU twice over.
template <int TT>
__global__ void __launch_bounds__(256, 2)
    rf_scores_kernel(const RfGeomDev g, const float* __restrict__ pq, const float* __restrict__ pk,
                     float* __restrict__ scores) {
  constexpr int kTile = 16 * TT;
  constexpr int kQ = TT / 4;                       // 64-row quadrants per tile edge
  constexpr int kReps = kTile * kKc / 4 / 256;     // float4 per thread per operand chunk
  __shared__ __align__(16) float As[2][kKc][kTile + 4];
  __shared__ __align__(16) float Bs[2][kKc][kTile + 4];
  // Decode blockIdx.x into (instance, head, tile row, tile col) over the
  // non-dense instances in order.
  int rem = blockIdx.x;
  int si = -1, tiles_r = 0, tiles_c = 0;
  for (int i = 0; i < g.n_seqs; ++i) {
    const RfSeqDev& s = g.seq[i];
    if (s.dense) continue;
    const int tr_n = (s.nb + kTile - 1) / kTile, tc_n = (s.nbk + kTile - 1) / kTile;
    const int cnt = g.n1 * tr_n * tc_n;
    if (rem < cnt) { si = i; tiles_r = tr_n; tiles_c = tc_n; break; }
    rem -= cnt;
  }
  if (si < 0) return;
  const RfSeqDev& s = g.seq[si];
  const int n = rem / (tiles_r * tiles_c);
  const int tr = (rem / tiles_c) % tiles_r;
  const int tc = rem % tiles_c;
  const int gk = n / (g.n1 / g.n2);
  const float* A = pq + ((size_t)n * g.pooled_total + s.pool_off) * g.d;
  const float* B = pk + ((size_t)gk * g.pooled_k_total + s.poolk_off) * g.d;
  const int i0 = tr * kTile, j0 = tc * kTile;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;

  float4 pa[kReps], pb[kReps];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int rep = 0; rep < kReps; ++rep) {
      const int e = threadIdx.x + rep * 256;
      const int row = e >> 2, c4 = e & 3;
      pa[rep] = make_float4(0.f, 0.f, 0.f, 0.f);
      pb[rep] = pa[rep];
      if (i0 + row < s.nb) pa[rep] = *reinterpret_cast<const float4*>(A + (size_t)(i0 + row) * g.d + k0 + 4 * c4);
      if (j0 + row < s.nbk) pb[rep] = *reinterpret_cast<const float4*>(B + (size_t)(j0 + row) * g.d + k0 + 4 * c4);
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int rep = 0; rep < kReps; ++rep) {
      const int e = threadIdx.x + rep * 256;
      const int row = e >> 2, c4 = e & 3;
      As[buf][4 * c4 + 0][row] = pa[rep].x; As[buf][4 * c4 + 1][row] = pa[rep].y;
      As[buf][4 * c4 + 2][row] = pa[rep].z; As[buf][4 * c4 + 3][row] = pa[rep].w;
      Bs[buf][4 * c4 + 0][row] = pb[rep].x; Bs[buf][4 * c4 + 1][row] = pb[rep].y;
      Bs[buf][4 * c4 + 2][row] = pb[rep].z; Bs[buf][4 * c4 + 3][row] = pb[rep].w;
    }
  };

  float acc[TT][TT];
#pragma unroll
  for (int a = 0; a < TT; ++a)
#pragma unroll
    for (int b = 0; b < TT; ++b) acc[a][b] = 0.f;

  fetch(0);
  stash(0);
  __syncthreads();
  const int chunks = g.d / kKc;
#pragma unroll 1
  for (int c = 0; c < chunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < chunks) fetch((c + 1) * kKc);
#pragma unroll
    for (int kk = 0; kk < kKc; ++kk) {
      float av[TT], bv[TT];
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const float4 a4 = *reinterpret_cast<const float4*>(&As[buf][kk][q * 64 + ty * 4]);
        const float4 b4 = *reinterpret_cast<const float4*>(&Bs[buf][kk][q * 64 + tx * 4]);
        av[4 * q] = a4.x; av[4 * q + 1] = a4.y; av[4 * q + 2] = a4.z; av[4 * q + 3] = a4.w;
        bv[4 * q] = b4.x; bv[4 * q + 1] = b4.y; bv[4 * q + 2] = b4.z; bv[4 * q + 3] = b4.w;
      }
#pragma unroll
      for (int x = 0; x < TT; ++x)
#pragma unroll
        for (int y = 0; y < TT; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    if (c + 1 < chunks) stash(buf ^ 1);
    __syncthreads();
  }
  float* C = scores + s.score_off + (size_t)n * s.nb * s.nbk;
#pragma unroll
  for (int x = 0; x < TT; ++x) {
    const int i = i0 + (x >> 2) * 64 + ty * 4 + (x & 3);
    if (i >= s.nb) continue;
#pragma unroll
    for (int y = 0; y < TT; ++y) {
      const int j = j0 + (y >> 2) * 64 + tx * 4 + (y & 3);
      if (j < s.nbk) C[(size_t)i * s.nbk + j] = acc[x][y];
    }
  }
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t rf_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int M>  // keys per lane: nbk <= 32 * M
__global__ void __launch_bounds__(256)
    rf_topk_kernel(const RfGeomDev g, const float* __restrict__ scores, int32_t* __restrict__ sel_idx,
                   int32_t* __restrict__ sel_num) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)g.t_qblk * g.n1;
  if (warp >= rows) return;
  const int tb = warp / g.n1, n = warp % g.n1;
  const RfSeqDev& s = g.seq[rf_seq_of_qblk(g, tb)];
  const int b = tb - s.qblk_off;
  const int nkv = s.npk + s.nbk;  // key blocks of the sequence
  int32_t* row = sel_idx + (size_t)warp * g.max_kv;
  const int i = b - s.n_pb;       // query side: 128-row blocks

  if (s.dense || b < s.n_pb || i < s.ns || s.kk >= s.nbk) {
    for (int c = lane; c < g.max_kv; c += 32) row[c] = c < nkv ? c : -1;
    if (lane == 0) sel_num[warp] = nkv;
    return;
  }

  // Keys of this row; absent slots hold 0, below every real key.
  const float* sc = scores + s.score_off + ((size_t)n * s.nb + i) * s.nbk;
  uint32_t key[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int j = lane + 32 * m;
    key[m] = j < s.nbk ? rf_key(sc[j]) : 0u;
  }
  const int k = s.kk;
  unsigned long long sel = 0;  // bit m: block lane + 32m is kept
  if (k > 0) {
    // Largest T with #{key >= T} >= k, one bit at a time from the top.  All
    // keys of the row share the bits above the highest bit in which the
    // smallest and the largest differ, so T starts as that common prefix and
    // the search runs over the bits below it only.
    uint32_t kmax = 0u, kmin = 0xFFFFFFFFu;
#pragma unroll
    for (int m = 0; m < M; ++m)
      if (lane + 32 * m < s.nbk) {
        kmax = max(kmax, key[m]);
        kmin = min(kmin, key[m]);
      }
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    const uint32_t diff = kmax ^ kmin;
    const int top = diff ? 31 - __clz(diff) : -1;
    uint32_t T = diff ? (kmin & ~((2u << top) - 1u)) : kmin;
#pragma unroll 1
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      int cnt = 0;
#pragma unroll
      for (int m = 0; m < M; ++m) cnt += key[m] >= cand ? 1 : 0;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= k) T = cand;
    }
    int gt = 0;
#pragma unroll
    for (int m = 0; m < M; ++m) gt += key[m] > T ? 1 : 0;
    gt = __reduce_add_sync(0xffffffffu, gt);
    int need = k - gt;  // keys equal to T to take, lowest block index first
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const bool eq = key[m] == T && key[m] != 0u;
      const uint32_t ball = __ballot_sync(0xffffffffu, eq);
      const bool take_eq = eq && (int)__popc(ball & lt_mask) < need;
      need -= min(need, (int)__popc(ball));
      if (key[m] > T || take_eq) sel |= 1ull << m;
    }
  }
  // First-frame sinks.
#pragma unroll
  for (int m = 0; m < M; ++m)
    if (lane + 32 * m < s.nsk) sel |= 1ull << m;

  for (int c = lane; c < s.npk; c += 32) row[c] = c;
  int pos = s.npk;
  const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const bool on = (sel >> m) & 1ull;
    const uint32_t ball = __ballot_sync(0xffffffffu, on);
    if (on) row[pos + __popc(ball & lt_mask)] = s.npk + lane + 32 * m;
    pos += __popc(ball);
  }
  for (int c = pos + lane; c < g.max_kv; c += 32) row[c] = -1;
  if (lane == 0) sel_num[warp] = pos;
}

}  // namespace

rf_status_t rf_launch_select(const rf_plan* p, int32_t* sel_idx, int32_t* sel_num, void* ws,
                             cudaStream_t st) {
  const RfGeomDev& g = p->g;
  const float* pq = reinterpret_cast<const float*>(static_cast<char*>(ws) + p->off_pq);
  const float* pk = reinterpret_cast<const float*>(static_cast<char*>(ws) + p->off_pk);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + p->off_scores);
  // Tiles of 128 x 128 once they fill the GPU at least twice over (two CTAs
  // per SM), else 64 x 64 tiles for more parallelism.
  long long tiles64 = 0, tiles128 = 0;
  for (int i = 0; i < g.n_seqs; ++i) {
    const RfSeqDev& s = g.seq[i];
    if (s.dense) continue;
    tiles64 += (long long)g.n1 * ((s.nb + 63) / 64) * ((s.nbk + 63) / 64);
    tiles128 += (long long)g.n1 * ((s.nb + 127) / 128) * ((s.nbk + 127) / 128);
  }
  if (tiles64 > 0) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaGetLastError();
    if (tiles128 >= 4ll * sms) rf_scores_kernel<8><<<(unsigned)tiles128, 256, 0, st>>>(g, pq, pk, scores);
    else                       rf_scores_kernel<4><<<(unsigned)tiles64, 256, 0, st>>>(g, pq, pk, scores);
    rf_status_t s = rf_check_launch("rf_scores_kernel");
    if (s != RF_OK) return s;
  }
  const long long rows = (long long)g.t_qblk * g.n1;
  if (rows == 0) return RF_OK;
  const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
  if (g.max_nbk <= 256)       rf_topk_kernel<8><<<blocks, 256, 0, st>>>(g, scores, sel_idx, sel_num);
  else if (g.max_nbk <= 512)  rf_topk_kernel<16><<<blocks, 256, 0, st>>>(g, scores, sel_idx, sel_num);
  else if (g.max_nbk <= 640)  rf_topk_kernel<20><<<blocks, 256, 0, st>>>(g, scores, sel_idx, sel_num);
  else if (g.max_nbk <= 1024) rf_topk_kernel<32><<<blocks, 256, 0, st>>>(g, scores, sel_idx, sel_num);
  else if (g.max_nbk <= 1280) rf_topk_kernel<40><<<blocks, 256, 0, st>>>(g, scores, sel_idx, sel_num);
  else                        rf_topk_kernel<64><<<blocks, 256, 0, st>>>(g, scores, sel_idx, sel_num);
  return rf_check_launch("rf_topk_kernel");
}
