// librf host side: plan creation and validation (the first phase of the
// two-phase call on the "aclnnRainFusionAttention" API page), workspace
// layout, status reporting and the whole-path entry point.
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "rf_device.cuh"

namespace {

thread_local std::string g_last_error;

int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// Number of ranked key blocks a sparse query block keeps: ceil((1 - s) * nb),
// with a 1e-6 guard so that (1 - 0.8) * 465 = 92.999... rounds to 93
// ("RainFusion Attention" user guide, "Configuration": nominal dropped fraction).
int keep_count(int nb, double sparsity) {
  double k = std::ceil((1.0 - sparsity) * (double)nb - 1e-6);
  if (k < 0) k = 0;
  if (k > nb) k = nb;
  return (int)k;
}

// Sizes of one sequence under suffix promotion ("RainFusion Attention" user
// guide, "Geometry handling"): the sparse region is the largest whole number of
// 128-row blocks of tokens inside whole 8x8 tiles; every other video token is
// promoted into the always-dense prefix.
RfSeqDev seq_geometry(const rf_seq_geom_t& s, double sparsity, rf_token_order_t order) {
  RfSeqDev d;
  std::memset(&d, 0, sizeof(d));
  d.order = order;
  d.P = s.prefix_len;
  d.t = s.t;
  d.h = s.h;
  d.w = s.w;
  d.h8 = 8 * (s.h / 8);
  d.w8 = 8 * (s.w / 8);
  d.A = s.t * d.h8 * d.w8;
  d.nb = d.A / RF_BLOCK;
  d.S = d.nb * RF_BLOCK;
  d.L = s.prefix_len + s.t * s.h * s.w;
  d.Lp = d.L - d.S;
  d.n_pb = (d.Lp + RF_BLOCK - 1) / RF_BLOCK;
  int first_frame = d.h8 * d.w8;
  d.ns = (first_frame + RF_BLOCK - 1) / RF_BLOCK;
  if (d.ns > d.nb) d.ns = d.nb;
  d.dense = d.nb < RF_DENSE_MIN_BLOCKS ? 1 : 0;
  d.k = d.dense ? d.nb : keep_count(d.nb, sparsity);
  d.npk = d.n_pb;
  d.nbk = d.nb;
  d.nsk = d.ns;
  d.kk = d.k;
  return d;
}

// Key side of the selection with 64-row key blocks ([API] "Formula": blocks of
// blockShapeX x blockShapeY): the prefix tiled from row 0 by ceil(Lp / 64)
// key blocks, the sparse region by 2 nb; the sinks are the key blocks holding
// first-frame tokens; k keeps the nominal fraction of the 64-row key blocks.
void key_side_64(RfSeqDev& d, double sparsity) {
  d.npk = rf_n_pb64(d);
  d.nbk = 2 * d.nb;
  d.nsk = (d.h8 * d.w8 + 63) / 64;
  if (d.nsk > d.nbk) d.nsk = d.nbk;
  d.kk = d.dense ? d.nbk : keep_count(d.nbk, sparsity);
}

}  // namespace

rf_status_t rf_fail(rf_status_t st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

void rf_clear_error() { g_last_error.clear(); }

rf_status_t rf_check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return rf_fail(RF_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return RF_OK;
}

rf_status_t rf_require_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return rf_fail(RF_ERR_UNSUPPORTED_DEVICE, std::string("no CUDA device: ") + cudaGetErrorString(e));
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return rf_fail(RF_ERR_UNSUPPORTED_DEVICE, "cannot query the device's compute capability");
  }
  if (major != 10 || minor != 0)
    return rf_fail(RF_ERR_UNSUPPORTED_DEVICE,
                   "librf is built for sm_100a (B200); device is sm_" + std::to_string(major) +
                       std::to_string(minor));
  return RF_OK;
}

extern "C" {

const char* rf_status_string(rf_status_t s) {
  switch (s) {
    case RF_OK: return "ok";
    case RF_ERR_INVALID_ARG: return "invalid argument";
    case RF_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs sm_100)";
    case RF_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case RF_ERR_CUDA: return "CUDA error";
    case RF_ERR_DEVICE_FAULT: return "device-side fault recorded (bad selectIdx entry or expired wait)";
    case RF_ERR_UNSUPPORTED: return "supported by the method but not built";
  }
  return "unknown status";
}

const char* rf_last_error(void) { return g_last_error.c_str(); }

rf_status_t rf_plan_create(const rf_seq_geom_t* seqs, int32_t n_seqs, int32_t batch, int32_t n1,
                           int32_t n2, int32_t d, rf_layout_t layout, rf_dtype_t dtype,
                           double sparsity, int32_t block_q, int32_t block_kv, rf_plan_t** out) {
  return rf_plan_create_ex(seqs, n_seqs, batch, n1, n2, d, layout, dtype, sparsity, block_q,
                           block_kv, nullptr, out);
}

rf_status_t rf_plan_create_ex(const rf_seq_geom_t* seqs, int32_t n_seqs, int32_t batch,
                              int32_t n1, int32_t n2, int32_t d, rf_layout_t layout,
                              rf_dtype_t dtype, double sparsity, int32_t block_q,
                              int32_t block_kv, const rf_plan_options_t* options,
                              rf_plan_t** out) {
  g_last_error.clear();
  if (!out || !seqs) return rf_fail(RF_ERR_INVALID_ARG, "null seqs or out");
  rf_plan_options_t opt;
  std::memset(&opt, 0, sizeof(opt));
  if (options) opt = *options;
  for (int i = 0; i < 6; ++i)
    if (opt.reserved[i] != 0) return rf_fail(RF_ERR_INVALID_ARG, "reserved option fields must be zero");
  if (opt.token_order != RF_ORDER_TILE && opt.token_order != RF_ORDER_FRAME_PAIR)
    return rf_fail(RF_ERR_INVALID_ARG, "token order must be RF_ORDER_TILE or RF_ORDER_FRAME_PAIR");
  if (opt.precision != RF_PRECISION_NATIVE && opt.precision != RF_PRECISION_MIX &&
      opt.precision != RF_PRECISION_FP8 && opt.precision != RF_PRECISION_MXFP4)
    return rf_fail(RF_ERR_INVALID_ARG, "unknown precision");
  if ((opt.precision == RF_PRECISION_MIX || opt.precision == RF_PRECISION_FP8) && d != 128)
    return rf_fail(RF_ERR_UNSUPPORTED, "precisions mix and fp8 are built for head dim 128 only");
  const rf_token_order_t order = (rf_token_order_t)opt.token_order;
  if (layout != RF_LAYOUT_BNSD && layout != RF_LAYOUT_TND)
    return rf_fail(RF_ERR_INVALID_ARG, "layout must be BNSD or TND");
  if (dtype != RF_BF16 && dtype != RF_FP16)
    return rf_fail(RF_ERR_INVALID_ARG, "dtype must be bf16 or fp16");
  if (!(sparsity >= 0.0 && sparsity <= 1.0) || !std::isfinite(sparsity))
    return rf_fail(RF_ERR_INVALID_ARG, "sparsity must be finite and in [0, 1]");
  if (block_q <= 0 || block_kv <= 0)
    return rf_fail(RF_ERR_INVALID_ARG, "blockShape entries must be > 0");
  if (block_q != RF_BLOCK || (block_kv != RF_BLOCK && block_kv != 64))
    return rf_fail(RF_ERR_UNSUPPORTED, "blockShape must be 128 x 128 or 128 x 64");
  if (block_kv != RF_BLOCK && opt.precision != RF_PRECISION_NATIVE)
    return rf_fail(RF_ERR_UNSUPPORTED, "blockShape 128 x 64 is built for native precision only");
  if (n1 <= 0 || n2 <= 0 || n1 % n2 != 0)
    return rf_fail(RF_ERR_INVALID_ARG, "heads: need n1 > 0, n2 > 0 and n1 % n2 == 0");
  if (d <= 0) return rf_fail(RF_ERR_INVALID_ARG, "head dim must be > 0");
  if (d != 64 && d != 128) return rf_fail(RF_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  if (layout == RF_LAYOUT_BNSD) {
    if (n_seqs != 1) return rf_fail(RF_ERR_INVALID_ARG, "BNSD takes exactly one geometry");
    if (batch < 1 || batch > RF_MAX_SEQS)
      return rf_fail(RF_ERR_INVALID_ARG, "BNSD batch must be in [1, 32]");
  } else {
    if (batch != 1) return rf_fail(RF_ERR_INVALID_ARG, "TND requires batch == 1");
    if (n_seqs < 1 || n_seqs > RF_MAX_SEQS)
      return rf_fail(RF_ERR_INVALID_ARG, "TND takes 1..32 sequences");
  }
  for (int i = 0; i < n_seqs; ++i) {
    const rf_seq_geom_t& s = seqs[i];
    if (s.prefix_len < 0 || s.t < 0 || s.h < 0 || s.w < 0)
      return rf_fail(RF_ERR_INVALID_ARG, "negative geometry");
    int64_t len = (int64_t)s.prefix_len + (int64_t)s.t * s.h * s.w;
    if (len <= 0) return rf_fail(RF_ERR_INVALID_ARG, "empty sequence");
    if (len > (1ll << 30)) return rf_fail(RF_ERR_INVALID_ARG, "sequence too long");
  }

  rf_plan* p = new (std::nothrow) rf_plan();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "out of host memory");
  std::memset(&p->g, 0, sizeof(p->g));
  p->layout = layout;
  p->dtype = dtype;
  p->sparsity = sparsity;
  p->batch = batch;
  p->n_user_seqs = n_seqs;
  RfGeomDev& g = p->g;
  g.layout = layout;
  g.n1 = n1;
  g.n2 = n2;
  g.d = d;
  g.n_seqs = layout == RF_LAYOUT_BNSD ? batch : n_seqs;

  int64_t rows = 0, qblk = 0, pooled = 0, pooled_k = 0, scores = 0, flops = 0;
  int max_kv = 0, max_nb = 0, max_nbk = 0;
  for (int i = 0; i < g.n_seqs; ++i) {
    const rf_seq_geom_t& src = seqs[layout == RF_LAYOUT_BNSD ? 0 : i];
    RfSeqDev s = seq_geometry(src, sparsity, order);
    s.batch_idx = layout == RF_LAYOUT_BNSD ? i : 0;
    s.row_off = layout == RF_LAYOUT_BNSD ? 0 : rows;
    s.qblk_off = (int)qblk;
    s.pool_off = (int)pooled;
    s.score_off = scores;
    if (block_kv != RF_BLOCK) key_side_64(s, sparsity);
    s.poolk_off = (int)pooled_k;
    g.seq[i] = s;
    int nblk = s.n_pb + s.nb;
    // selectIdx rows count key/value blocks of block_kv rows
    const int nkv = s.npk + s.nbk;
    if (nkv > max_kv) max_kv = nkv;
    if (s.nb > max_nb) max_nb = s.nb;
    if (s.nbk > max_nbk) max_nbk = s.nbk;
    rows += s.L;
    qblk += nblk;
    pooled += s.nb;
    pooled_k += s.nbk;
    if (!s.dense) scores += (int64_t)n1 * s.nb * s.nbk;
    flops += 4ll * d * (int64_t)s.L * s.L * n1;
    if (layout == RF_LAYOUT_TND || i == 0) {
      rf_seq_info_t inf;
      inf.row_offset = s.row_off;
      inf.length = s.L;
      inf.lp = s.Lp;
      inf.sparse = s.S;
      inf.promoted = (int64_t)s.L - s.P - s.S;
      inf.n_pb = s.n_pb;
      inf.nb = s.nb;
      inf.ns = s.ns;
      inf.k = s.k;
      inf.qblk_offset = s.qblk_off;
      inf.dense = s.dense;
      inf.n_pb_kv = s.npk;
      inf.nb_kv = s.nbk;
      inf.ns_kv = s.nsk;
      inf.k_kv = s.kk;
      p->info.push_back(inf);
    }
  }
  if (max_kv > RF_MAX_KV_LIST || max_nb > RF_MAX_NB || max_nbk > RF_MAX_NB) {
    delete p;
    return rf_fail(RF_ERR_UNSUPPORTED, "a sequence has more than 2048 blocks (query or key/value)");
  }
  if (qblk * n1 > (1ll << 31) - 1) {
    delete p;
    return rf_fail(RF_ERR_INVALID_ARG, "too many query blocks");
  }
  g.t_qblk = (int)qblk;
  g.max_kv = max_kv;
  g.block_kv = block_kv;
  g.pooled_total = (int)pooled;
  g.pooled_k_total = (int)pooled_k;
  g.max_nb = max_nb;
  g.max_nbk = max_nbk;
  p->rows_total = layout == RF_LAYOUT_BNSD ? (int64_t)batch * g.seq[0].L : rows;
  p->kept_flops_upper = flops;

  // Workspace: [status words | pooled Q fp32 [N1][pooled][D] | pooled K fp32
  // [N2][pooled_k][D] | block scores fp32, per non-dense sequence [N1][nb][nbk]]
  // (nbk = nb, or 2 nb with 64-row key blocks).
  int64_t off = 0;
  p->off_status = off;
  off += 256;
  p->off_pq = off;
  off = align_up(off + (int64_t)n1 * pooled * d * 4, 256);
  p->off_pk = off;
  off = align_up(off + (int64_t)n2 * pooled_k * d * 4, 256);
  p->off_scores = off;
  off = align_up(off + scores * 4, 256);
  // RF_PRECISION_MIX: E4M3 copies of Q' and K' (one byte per element, the
  // layouts of q_r / k_r) and their fp32 scales per (head, query block).
  p->precision = (rf_precision_t)opt.precision;
  p->token_order = order;
  p->off_q8 = p->off_k8 = p->off_qs = p->off_ks = -1;
  p->off_qx = p->off_kx = p->off_vx = -1;
  p->off_v8 = p->off_vexp = -1;
  p->off_quant = off;
  if (p->precision == RF_PRECISION_MIX || p->precision == RF_PRECISION_FP8) {
    p->off_q8 = off;
    off = align_up(off + p->rows_total * n1 * d, 256);
    p->off_k8 = off;
    off = align_up(off + p->rows_total * n2 * d, 256);
    p->off_qs = off;
    off = align_up(off + (int64_t)n1 * qblk * 4, 256);
    p->off_ks = off;
    off = align_up(off + (int64_t)n2 * qblk * 4, 256);
  }
  // RF_PRECISION_FP8 also: E4M3 codes of V' stored transposed per block
  // ([n2][t_qblk][d][128]: the 128 keys of one column contiguous, the layout a
  // K-major B operand of P V needs) and their power-of-two exponents (int32
  // [n2][t_qblk]).
  if (p->precision == RF_PRECISION_FP8) {
    p->off_v8 = off;
    off = align_up(off + (int64_t)n2 * qblk * RF_BLOCK * d, 256);
    p->off_vexp = off;
    off = align_up(off + (int64_t)n2 * qblk * 4, 256);
  }
  // RF_PRECISION_MXFP4: MXFP4-rounded 16-bit copies of Q', K', V' (layouts of
  // q_r / k_r / v_r).
  // D = 128 carries the MXFP4 values as E4M3 codes instead (every value c * 2^e
  // with -8 <= e <= 6 is one): Q' and K' one byte per element in the layouts of
  // q_r / k_r (the mix regions, no scales), V' transposed per block (the fp8
  // region, no exponents); both products then run on the FP8 tensor cores.
  if (p->precision == RF_PRECISION_MXFP4 && d == 128) {
    p->off_q8 = off;
    off = align_up(off + p->rows_total * n1 * d, 256);
    p->off_k8 = off;
    off = align_up(off + p->rows_total * n2 * d, 256);
    p->off_v8 = off;
    off = align_up(off + (int64_t)n2 * qblk * RF_BLOCK * d, 256);
  } else if (p->precision == RF_PRECISION_MXFP4) {
    p->off_qx = off;
    off = align_up(off + p->rows_total * n1 * d * 2, 256);
    p->off_kx = off;
    off = align_up(off + p->rows_total * n2 * d * 2, 256);
    p->off_vx = off;
    off = align_up(off + p->rows_total * n2 * d * 2, 256);
  }
  p->ws_bytes = off;
  *out = p;
  return RF_OK;
}

rf_status_t rf_plan_info(const rf_plan_t* p, rf_plan_info_t* out) {
  if (!p || !out) return rf_fail(RF_ERR_INVALID_ARG, "null plan or out");
  out->rows_total = p->rows_total;
  out->t_qblk = p->g.t_qblk;
  out->max_kv_blocks = p->g.max_kv;
  out->workspace_bytes = p->ws_bytes;
  out->pooled_blocks = p->g.pooled_total;
  out->kept_flops_upper = p->kept_flops_upper;
  out->ws_pooled_q = p->off_pq;
  out->ws_pooled_k = p->off_pk;
  out->n_seqs = p->g.n_seqs;
  out->n1 = p->g.n1;
  out->n2 = p->g.n2;
  out->d = p->g.d;
  out->precision = p->precision;
  out->token_order = p->token_order;
  out->ws_q8 = p->off_q8;
  out->ws_k8 = p->off_k8;
  out->ws_q_scale = p->off_qs;
  out->ws_k_scale = p->off_ks;
  out->ws_q_mx = p->off_qx;
  out->ws_k_mx = p->off_kx;
  out->ws_v_mx = p->off_vx;
  out->ws_v8 = p->off_v8;
  out->ws_v_exp = p->off_vexp;
  out->pooled_k_blocks = p->g.pooled_k_total;
  return RF_OK;
}

rf_status_t rf_plan_seq_info(const rf_plan_t* p, int32_t seq, rf_seq_info_t* out) {
  if (!p || !out) return rf_fail(RF_ERR_INVALID_ARG, "null plan or out");
  if (seq < 0 || seq >= (int)p->info.size()) return rf_fail(RF_ERR_INVALID_ARG, "seq out of range");
  *out = p->info[seq];
  return RF_OK;
}

void rf_plan_destroy(rf_plan_t* p) { delete p; }

rf_status_t rf_plan_permutation(const rf_plan_t* p, int32_t seq, int64_t* src_rows, int64_t n) {
  if (!p || !src_rows) return rf_fail(RF_ERR_INVALID_ARG, "null plan or output");
  if (seq < 0 || seq >= (int)p->info.size()) return rf_fail(RF_ERR_INVALID_ARG, "seq out of range");
  const RfSeqDev& s = p->g.seq[seq];
  if (n != s.L) return rf_fail(RF_ERR_INVALID_ARG, "n must equal the sequence length");
  for (int r = 0; r < s.L; ++r) src_rows[r] = rf_orig_row(s, r);
  return RF_OK;
}

static rf_status_t check_ws(const rf_plan_t* p, const void* ws, size_t ws_bytes) {
  if (!ws) return rf_fail(RF_ERR_INVALID_ARG, "null workspace");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return rf_fail(RF_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((int64_t)ws_bytes < p->ws_bytes)
    return rf_fail(RF_ERR_WORKSPACE_TOO_SMALL,
                   "workspace needs " + std::to_string(p->ws_bytes) + " bytes");
  return RF_OK;
}

static bool aligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; }

rf_status_t rf_rearrange(const rf_plan_t* p, const void* q, const void* k, const void* v,
                         void* q_r, void* k_r, void* v_r, void* ws, size_t ws_bytes,
                         rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (!q || !k || !v || !q_r || !k_r || !v_r) return rf_fail(RF_ERR_INVALID_ARG, "null tensor");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_r) || !aligned16(k_r) ||
      !aligned16(v_r))
    return rf_fail(RF_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (q == q_r || k == k_r || v == v_r) return rf_fail(RF_ERR_INVALID_ARG, "in-place rearrange");
  rf_status_t st = check_ws(p, ws, ws_bytes);
  if (st != RF_OK) return st;
  if ((st = rf_require_device()) != RF_OK) return st;
  return rf_launch_rearrange(p, q, k, v, q_r, k_r, v_r, ws, (cudaStream_t)stream);
}

rf_status_t rf_quantize_qk(const rf_plan_t* p, const void* q_r, const void* k_r, void* ws,
                           size_t ws_bytes, rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (p->precision != RF_PRECISION_MIX)
    return rf_fail(RF_ERR_INVALID_ARG, "rf_quantize_qk needs a plan with precision mix");
  if (!q_r || !k_r || !aligned16(q_r) || !aligned16(k_r))
    return rf_fail(RF_ERR_INVALID_ARG, "q_r and k_r must be non-null and 16-byte aligned");
  rf_status_t st = check_ws(p, ws, ws_bytes);
  if (st != RF_OK) return st;
  if ((st = rf_require_device()) != RF_OK) return st;
  return rf_launch_quantize(p, q_r, k_r, nullptr, ws, (cudaStream_t)stream);
}

rf_status_t rf_quantize_mx(const rf_plan_t* p, const void* q_r, const void* k_r, const void* v_r,
                           void* ws, size_t ws_bytes, rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (p->precision != RF_PRECISION_MXFP4)
    return rf_fail(RF_ERR_INVALID_ARG, "rf_quantize_mx needs a plan with precision mxfp4");
  if (!q_r || !k_r || !v_r || !aligned16(q_r) || !aligned16(k_r) || !aligned16(v_r))
    return rf_fail(RF_ERR_INVALID_ARG, "q_r, k_r and v_r must be non-null and 16-byte aligned");
  rf_status_t st = check_ws(p, ws, ws_bytes);
  if (st != RF_OK) return st;
  if ((st = rf_require_device()) != RF_OK) return st;
  return rf_launch_quantize(p, q_r, k_r, v_r, ws, (cudaStream_t)stream);
}

rf_status_t rf_quantize(const rf_plan_t* p, const void* q_r, const void* k_r, const void* v_r,
                        void* ws, size_t ws_bytes, rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (p->precision == RF_PRECISION_NATIVE)
    return rf_fail(RF_ERR_INVALID_ARG, "a native-precision plan has no quantized copies");
  const bool need_v = p->precision != RF_PRECISION_MIX;
  if (!q_r || !k_r || !aligned16(q_r) || !aligned16(k_r) || (need_v && (!v_r || !aligned16(v_r))))
    return rf_fail(RF_ERR_INVALID_ARG, "inputs must be non-null and 16-byte aligned");
  rf_status_t st = check_ws(p, ws, ws_bytes);
  if (st != RF_OK) return st;
  if ((st = rf_require_device()) != RF_OK) return st;
  return rf_launch_quantize(p, q_r, k_r, need_v ? v_r : nullptr, ws, (cudaStream_t)stream);
}

rf_status_t rf_pool_select(const rf_plan_t* p, const void* q_r, const void* k_r,
                           int32_t* select_idx, int32_t* select_num, void* ws, size_t ws_bytes,
                           rf_pool_mode_t pool_mode, rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (!select_idx || !select_num) return rf_fail(RF_ERR_INVALID_ARG, "null selectIdx/selectNum");
  if (pool_mode != RF_POOL_FROM_WS && pool_mode != RF_POOL_RECOMPUTE)
    return rf_fail(RF_ERR_INVALID_ARG, "bad pool mode");
  if (pool_mode == RF_POOL_RECOMPUTE &&
      (!q_r || !k_r || !aligned16(q_r) || !aligned16(k_r)))
    return rf_fail(RF_ERR_INVALID_ARG, "recompute needs 16-byte aligned q_r and k_r");
  rf_status_t st = check_ws(p, ws, ws_bytes);
  if (st != RF_OK) return st;
  if ((st = rf_require_device()) != RF_OK) return st;
  if (pool_mode == RF_POOL_RECOMPUTE) {
    st = rf_launch_pool(p, q_r, k_r, ws, (cudaStream_t)stream);
    if (st != RF_OK) return st;
  }
  return rf_launch_select(p, select_idx, select_num, ws, (cudaStream_t)stream);
}

rf_status_t rf_block_sparse_attn(const rf_plan_t* p, const void* q_r, const void* k_r,
                                 const void* v_r, const int32_t* select_idx,
                                 const int32_t* select_num, float scale, int32_t inner_precise,
                                 void* o_r, void* ws, size_t ws_bytes, rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (!q_r || !k_r || !v_r || !o_r || !select_idx || !select_num)
    return rf_fail(RF_ERR_INVALID_ARG, "null tensor");
  if (!aligned16(q_r) || !aligned16(k_r) || !aligned16(v_r) || !aligned16(o_r))
    return rf_fail(RF_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (o_r == q_r || o_r == k_r || o_r == v_r) return rf_fail(RF_ERR_INVALID_ARG, "o_r aliases an input");
  if (inner_precise != 0 && inner_precise != 1)
    return rf_fail(RF_ERR_INVALID_ARG, "inner_precise must be 0 or 1");
  if (inner_precise == 1 && p->dtype == RF_BF16)
    return rf_fail(RF_ERR_INVALID_ARG, "bf16 inputs allow only inner_precise 0 (fp32 softmax)");
  if (inner_precise == 1) return rf_fail(RF_ERR_UNSUPPORTED, "fp16 softmax is not built");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return rf_fail(RF_ERR_INVALID_ARG, "scale must be finite and > 0");
  rf_status_t st = check_ws(p, ws, ws_bytes);
  if (st != RF_OK) return st;
  if ((st = rf_require_device()) != RF_OK) return st;
  return rf_launch_attn(p, q_r, k_r, v_r, select_idx, select_num, scale, o_r, ws,
                        (cudaStream_t)stream);
}

rf_status_t rf_inverse_rearrange(const rf_plan_t* p, const void* o_r, void* o, rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (!o_r || !o) return rf_fail(RF_ERR_INVALID_ARG, "null tensor");
  if (!aligned16(o_r) || !aligned16(o)) return rf_fail(RF_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (o_r == o) return rf_fail(RF_ERR_INVALID_ARG, "in-place inverse rearrange");
  rf_status_t st = rf_require_device();
  if (st != RF_OK) return st;
  return rf_launch_inverse(p, o_r, o, (cudaStream_t)stream);
}

rf_status_t rf_forward(const rf_plan_t* p, const void* q, const void* k, const void* v, void* q_r,
                       void* k_r, void* v_r, int32_t* select_idx, int32_t* select_num, float scale,
                       void* o_r, void* o, void* ws, size_t ws_bytes, rf_stream_t stream) {
  rf_status_t st = rf_rearrange(p, q, k, v, q_r, k_r, v_r, ws, ws_bytes, stream);
  if (st != RF_OK) return st;
  st = rf_pool_select(p, nullptr, nullptr, select_idx, select_num, ws, ws_bytes, RF_POOL_FROM_WS,
                      stream);
  if (st != RF_OK) return st;
  st = rf_block_sparse_attn(p, q_r, k_r, v_r, select_idx, select_num, scale, 0, o_r, ws, ws_bytes,
                            stream);
  if (st != RF_OK) return st;
  return rf_inverse_rearrange(p, o_r, o, stream);
}

rf_status_t rf_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n,
                             rf_stream_t stream) {
  g_last_error.clear();
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_mufu))) return rf_fail(RF_ERR_INVALID_ARG, "bad buffers");
  rf_status_t st = rf_require_device();
  if (st != RF_OK) return st;
  return rf_launch_exp2_selftest(x, y_poly, y_mufu, n, (cudaStream_t)stream);
}

rf_status_t rf_selftest_expired_wait(const rf_plan_t* p, void* ws, size_t ws_bytes,
                                    rf_stream_t stream) {
  g_last_error.clear();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  rf_status_t st = check_ws(p, ws, ws_bytes);
  if (st != RF_OK) return st;
  if ((st = rf_require_device()) != RF_OK) return st;
  return rf_launch_expired_wait_selftest(p, ws, (cudaStream_t)stream);
}

rf_status_t rf_check_device_status(const rf_plan_t* p, void* ws, uint32_t* flags_out,
                                   rf_stream_t stream) {
  g_last_error.clear();
  if (!p || !ws) return rf_fail(RF_ERR_INVALID_ARG, "null plan or workspace");
  rf_status_t st = rf_require_device();
  if (st != RF_OK) return st;
  uint32_t words[2] = {0, 0};
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* dev = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + p->off_status);
  if (cudaMemcpyAsync(words, dev, sizeof(words), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess ||
      cudaMemsetAsync(dev, 0, sizeof(words), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return rf_fail(RF_ERR_CUDA, std::string("status read: ") + cudaGetErrorString(cudaGetLastError()));
  if (flags_out) {
    flags_out[0] = words[0];
    flags_out[1] = words[1];
  }
  if (words[0] || words[1])
    return rf_fail(RF_ERR_DEVICE_FAULT, "bad selectIdx entries: " + std::to_string(words[0]) +
                                            ", expired waits: " + std::to_string(words[1]));
  return RF_OK;
}

}  // extern "C"
