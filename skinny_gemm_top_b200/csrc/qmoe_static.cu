// qmoe_forward_static: the MoE layer forward with its scratch in a fixed
// device array of this library instead of a caller workspace.  It allocates
// nothing (no cudaMalloc / cudaFree, no allocating library call) and runs
// exactly the kernels of qmoe_forward on that array.
//
// Callers that cannot allocate: hosts that own no device allocator or
// memory pool of their own (a plain C embedding without a caching
// allocator), and per-step code that must not call cudaMalloc / cudaFree,
// which synchronise the device and can fail under memory pressure in the
// middle of a step.  Such callers still need scratch for the routing tables,
// the slot rows and the per-tile tickets of qmoe_forward.
//
// Limits and rules:
//  * Scratch: QMOE_STATIC_SCRATCH_BYTES per device (8 MiB).  A call whose
//    qmoe_workspace_size(T) exceeds it is rejected with
//    QMOE_ERR_STATIC_SCRATCH before anything is launched (no row tiling).
//  * Set-up: the first call on a device resolves the array's device address
//    with cudaGetSymbolAddress, with that device current, and caches it; that
//    call can load this library's device code, so it should come before any
//    stream capture.
//  * Zero state: no scratch value needs to start at any particular value.
//    The only values a call reads before writing them are the decode
//    kernel's fp32 accumulator and its last-block ticket, and the reset launch
//    of the same call clears both first; so the array needs no clearing
//    between calls.
//  * One array per device: calls that overlap in time on the same device
//    (other streams, other host threads) race on it.  Serialise them.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "qmoe.h"

namespace {

constexpr int kStaticMaxDevices = 64;

// The scratch: file scope, one instance per device, 256-byte aligned like
// the workspaces qmoe_forward accepts.
static __device__ __align__(256) unsigned char g_static_scratch[QMOE_STATIC_SCRATCH_BYTES];

std::mutex g_static_mu;
void* g_static_ptr[kStaticMaxDevices] = {};

// Device address of the current device's scratch; resolved once per device.
qmoe_status static_scratch(void** out) {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kStaticMaxDevices) return QMOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[d]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr) return QMOE_ERR_CUDA;
    g_static_ptr[d] = p;
  }
  *out = g_static_ptr[d];
  return QMOE_OK;
}

}  // namespace

extern "C" {

qmoe_status qmoe_forward_static(const qmoe_layer* layer, const uint16_t* x, const float* logits, int T,
                                uint16_t* y, void* stream) {
  if (!layer || T <= 0) return QMOE_ERR_INVALID_ARG;
  size_t need = 0;
  qmoe_status s = qmoe_workspace_size(layer, T, &need);
  if (s != QMOE_OK) return s;
  if (need > (size_t)QMOE_STATIC_SCRATCH_BYTES) return QMOE_ERR_STATIC_SCRATCH;
  void* scratch = nullptr;
  s = static_scratch(&scratch);
  if (s != QMOE_OK) return s;
  return qmoe_forward(layer, x, logits, T, y, scratch, (size_t)QMOE_STATIC_SCRATCH_BYTES, stream);
}

}  // extern "C"
