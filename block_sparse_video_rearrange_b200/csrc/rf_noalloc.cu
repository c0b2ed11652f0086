// rf_pool_select_noalloc: block ranking and selection for callers that must
// not allocate device memory.
//
// Who needs it: code that runs inside a host framework whose device memory
// belongs to that framework's own allocator (a serving plugin cannot call
// cudaMalloc behind the allocator's back, and often cannot reach the
// allocator either), and code on a latency-critical path where a cudaMalloc,
// which may synchronise the whole device, is not acceptable.  Such callers can
// still hand over their inputs and outputs; what they cannot provide is the
// selection step's scratch memory (block means and block scores).
//
// This file keeps that scratch in one file-scope device array of
// RF_NOALLOC_SCRATCH_BYTES.  The array belongs to this file's module: every
// GPU on which the module is loaded (the first call of the entry point on that
// device loads it) keeps the array until the process exits.  The work itself
// is done by the same pooling, score and top-k kernels as rf_pool_select in
// RF_POOL_RECOMPUTE mode, pointed at the array instead of a caller workspace.
#include <mutex>
#include <string>

#include "rf_internal.h"

#define RF_NOALLOC_SCRATCH_BYTES (32ull << 20)
#define RF_NOALLOC_MAX_DEVICES 64

static __device__ __align__(256) unsigned char rf_noalloc_scratch[RF_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_mu;
void* g_scratch[RF_NOALLOC_MAX_DEVICES] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached for the life of the
// process; a cudaDeviceReset on that device invalidates it, and the header
// tells callers not to use this entry point after one.
rf_status_t scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return rf_fail(RF_ERR_UNSUPPORTED_DEVICE, "no current CUDA device");
  }
  if (dev < 0 || dev >= RF_NOALLOC_MAX_DEVICES)
    return rf_fail(RF_ERR_UNSUPPORTED_DEVICE, "device ordinal beyond 64");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, rf_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      cudaGetLastError();
      return rf_fail(RF_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    }
    g_scratch[dev] = ptr;
  }
  *out = g_scratch[dev];
  return RF_OK;
}

}  // namespace

extern "C" rf_status_t rf_pool_select_noalloc(const rf_plan_t* p, const void* q_r, const void* k_r,
                                              int32_t* select_idx, int32_t* select_num,
                                              rf_stream_t stream) {
  rf_clear_error();
  if (!p) return rf_fail(RF_ERR_INVALID_ARG, "null plan");
  if (!q_r || !k_r || !select_idx || !select_num)
    return rf_fail(RF_ERR_INVALID_ARG, "null tensor");
  if ((reinterpret_cast<uintptr_t>(q_r) & 15) || (reinterpret_cast<uintptr_t>(k_r) & 15))
    return rf_fail(RF_ERR_INVALID_ARG, "q_r and k_r must be 16-byte aligned");
  // The selection part of the workspace layout (mix and mxfp4 plans put their
  // quantized copies after it; selection never touches them).
  const int64_t sel_bytes = p->off_quant;
  if ((uint64_t)sel_bytes > RF_NOALLOC_SCRATCH_BYTES)
    return rf_fail(RF_ERR_INVALID_ARG,
                   "this problem needs " + std::to_string(sel_bytes) +
                       " bytes of selection scratch; the allocation-free entry point holds " +
                       std::to_string(RF_NOALLOC_SCRATCH_BYTES) + " (use rf_pool_select)");
  rf_status_t st = rf_require_device();
  if (st != RF_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != RF_OK) return st;
  // The array is laid out like a caller workspace.  Nothing in it needs to
  // start at zero: the pooling kernel writes every block mean and the score
  // kernel every score before they are read, within this call.
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = rf_launch_pool(p, q_r, k_r, scratch, s)) != RF_OK) return st;
  return rf_launch_select(p, select_idx, select_num, scratch, s);
}
