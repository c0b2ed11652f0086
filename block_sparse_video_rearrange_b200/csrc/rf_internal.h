// Internal declarations shared by the librf translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "rf.h"

#define RF_BLOCK 128          // query and key block rows ([API] blockShape 128 x 128)
#define RF_MAX_SEQS 32        // sequence instances one plan may hold (BNSD batch or TND seqs)
#define RF_MAX_KV_LIST 2048   // longest selectIdx row the attention kernel accepts
#define RF_MAX_NB 2048        // longest sparse region (blocks) the selection kernel accepts
#define RF_DENSE_MIN_BLOCKS 32  // [UG]: video segments below 32 blocks run dense

// Geometry of one sequence instance, passed to kernels by value.
struct RfSeqDev {
  long long row_off;    // TND: first token row of the sequence; BNSD: 0
  long long score_off;  // float offset of this sequence's [N1, nb, nb] score block in ws
  int batch_idx;        // BNSD: batch element; TND: 0
  int P, t, h, w, h8, w8;
  int A;                // aligned tokens t*h8*w8
  int S;                // sparse rows 128*nb
  int Lp;               // dense prefix rows P + promoted
  int L;                // sequence length
  int n_pb, nb, ns, k, dense;
  int order;            // rf_token_order_t of the aligned video tokens
  int qblk_off;         // first global query block
  int pool_off;         // first pooled query block (sum of nb of earlier instances)
  // Key side of the selection (block_kv rows per key block): prefix key
  // blocks, sparse key blocks, first-frame sink key blocks, ranked blocks
  // kept, and the first pooled key block.  With 128-row key blocks they are
  // n_pb, nb, ns, k and pool_off.
  int npk, nbk, nsk, kk;
  int poolk_off;
};

struct RfGeomDev {
  int n_seqs;           // instances (BNSD: batch, TND: sequences)
  int layout;           // rf_layout_t
  int n1, n2, d;
  int t_qblk;
  int max_kv;
  int block_kv;         // key/value block rows: 128, or 64 ([API] blockShape 128 x 64)
  int pooled_total;     // sum of nb over instances (query block means per head)
  int pooled_k_total;   // sum of nbk over instances (key block means per head)
  int max_nb;
  int max_nbk;
  RfSeqDev seq[RF_MAX_SEQS];
};

struct rf_plan {
  RfGeomDev g;
  rf_layout_t layout;
  rf_dtype_t dtype;
  double sparsity;
  int batch;
  int n_user_seqs;
  std::vector<rf_seq_info_t> info;  // per user sequence
  int64_t rows_total;
  int64_t ws_bytes;
  int64_t off_status, off_pq, off_pk, off_scores;
  rf_precision_t precision;
  rf_token_order_t token_order;
  int64_t off_q8, off_k8, off_qs, off_ks;  // RF_PRECISION_MIX workspace regions, else -1
  int64_t off_qx, off_kx, off_vx;          // RF_PRECISION_MXFP4 workspace regions, else -1
  int64_t off_v8, off_vexp;                // RF_PRECISION_FP8: transposed E4M3 V' and its exponents
  int64_t off_quant;                       // first precision-specific region (ws_bytes if none)
  int64_t kept_flops_upper;
};

// Status words at the start of the workspace.
enum { RF_STATUS_BAD_INDEX = 0, RF_STATUS_TIMEOUT = 1, RF_STATUS_WORDS = 64 };

// Error reporting (thread-local detail string).
rf_status_t rf_fail(rf_status_t st, const std::string& msg);
void rf_clear_error();  // every entry point starts with an empty detail string
rf_status_t rf_check_launch(const char* what);
rf_status_t rf_require_device();  // current device must be sm_100

// Launchers implemented in the .cu files.
rf_status_t rf_launch_rearrange(const rf_plan* p, const void* q, const void* k, const void* v,
                                void* q_r, void* k_r, void* v_r, void* ws, cudaStream_t st);
rf_status_t rf_launch_pool(const rf_plan* p, const void* q_r, const void* k_r, void* ws,
                           cudaStream_t st);
rf_status_t rf_launch_inverse(const rf_plan* p, const void* o_r, void* o, cudaStream_t st);
rf_status_t rf_launch_quantize(const rf_plan* p, const void* q_r, const void* k_r, const void* v_r,
                               void* ws, cudaStream_t st);
rf_status_t rf_launch_select(const rf_plan* p, int32_t* sel_idx, int32_t* sel_num, void* ws,
                             cudaStream_t st);
rf_status_t rf_launch_expired_wait_selftest(const rf_plan* p, void* ws, cudaStream_t st);
rf_status_t rf_launch_exp2_selftest(const float* x, float* y_poly, float* y_mufu, int64_t n,
                                    cudaStream_t st);
rf_status_t rf_launch_attn(const rf_plan* p, const void* q_r, const void* k_r, const void* v_r,
                           const int32_t* sel_idx, const int32_t* sel_num, float scale,
                           void* o_r, void* ws, cudaStream_t st);
