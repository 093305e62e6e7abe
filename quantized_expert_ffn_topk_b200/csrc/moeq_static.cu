// moeq_static.cu -- moe_expert_ffn_q_static: the expert FFN call for callers
// that cannot allocate device memory.
//
// moe_expert_ffn_q takes a caller-owned workspace (a control block with the
// device error word, then the SwiGLU activations h that the gate/up kernel
// hands to the down kernel). Some callers have no allocator to get one from:
// code that runs where cudaMalloc is not allowed (inside a stream capture
// that must stay allocation-free, a host callback, a plugin handed only its
// input and output buffers by a host runtime that owns all device memory).
// For them this file keeps one scratch region per GPU as a file-scope
// __device__ array and runs moe_expert_ffn_q on it.
//
// The array lives as long as the library is loaded, on every GPU that loads
// it. Every call on a device shares it, so calls whose kernels overlap on the
// GPU (two streams, two host threads) race on it and must be ordered by the
// caller. Each call clears the control block before its kernels run; h is
// fully written by the gate/up kernel before the down kernel reads it, so
// nothing else needs to start at zero.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "moeq.h"

namespace moeq {
moe_status ffn_check_args(const moe_layer_q* L, const void* x_bf16, int B, const int32_t* idx, const float* y_out);
}

namespace {

constexpr int kMaxDevices = 64;

// The scratch itself. In host code this name is only a stand-in for the
// device object: its address must be fetched with cudaGetSymbolAddress on
// each device before a kernel may be given it.
__device__ __align__(256) unsigned char g_ffn_scratch[MOEQ_STATIC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_ffn_scratch on the current device, looked up once per
// device (the first call on each device).
moe_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ffn_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_expert_ffn_q_static(const moe_layer_q* L, const void* x_bf16, int B, const int32_t* idx,
                                              float* y_out, int32_t* error_out, void* stream) {
  // every argument error returns before anything is queued
  moe_status st = moeq::ffn_check_args(L, x_bf16, B, idx, y_out);
  if (st != MOE_OK) return st;
  if (error_out && (reinterpret_cast<uintptr_t>(error_out) & 3u)) return MOE_ERR_ALIGN;
  const size_t need = moe_workspace_bytes(B, L->K, L->H, L->I, L->E);
  if (need == 0) return MOE_ERR_INVALID_ARG;
  if (need > (size_t)MOEQ_STATIC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  void* ws = nullptr;
  st = scratch_address(&ws);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, sizeof(moeq::WsCtrl), s) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  st = moe_expert_ffn_q(L, x_bf16, B, idx, y_out, ws, need, stream);
  if (st != MOE_OK) return st;
  if (error_out && cudaMemcpyAsync(error_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
