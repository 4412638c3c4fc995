// moe_decode_forward_no_alloc: the layer for callers that cannot give the library device memory.
//
// The scratch the layer needs lives in one file-scope __device__ array of
// MOE_NO_ALLOC_SCRATCH_BYTES bytes. Host code never dereferences or passes the array's name: on
// the host it is only a stand-in symbol. Its device address is looked up once per device with
// cudaGetSymbolAddress (that device current) and handed to the ordinary forward call as its
// workspace. Nothing here allocates or frees memory.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/moe_decode.h"

namespace {

__device__ __align__(256) unsigned char g_no_alloc_scratch[MOE_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_no_alloc_scratch);
    if (e != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int moe_decode_forward_no_alloc(const moe_cfg* cfg, int m, const void* x,
                                           const void* router_w, const float* expert_bias,
                                           const moe_expert_table* routed,
                                           const moe_expert_table* shared,
                                           const void* shared_gate_w, void* out, void* stream) {
  size_t need = 0;
  int rc = moe_workspace_bytes(cfg, m, &need);
  if (rc != MOE_OK) return rc;
  if (need > (size_t)MOE_NO_ALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  // Every remaining argument check of the forward call, with nothing launched: a zero-byte
  // workspace is refused only after all of them have passed.
  alignas(256) static const unsigned char probe[256] = {0};
  rc = moe_decode_forward(cfg, m, x, router_w, expert_bias, routed, shared, shared_gate_w, out,
                          (void*)probe, 0, stream);
  if (rc != MOE_ERR_WORKSPACE) return rc == MOE_OK ? MOE_ERR_WORKSPACE : rc;
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch)) != MOE_OK) return rc;
  if ((rc = moe_workspace_init(scratch, MOE_NO_ALLOC_SCRATCH_BYTES, stream)) != MOE_OK) return rc;
  return moe_decode_forward(cfg, m, x, router_w, expert_bias, routed, shared, shared_gate_w, out,
                            scratch, MOE_NO_ALLOC_SCRATCH_BYTES, stream);
}
