// noalloc.cu -- isa_forward_static: the whole ISA forward with its scratch in
// a fixed device array owned by the library, for callers that cannot hand
// the library a workspace (see include/isa.h).
//
// The array below is a file-scope __device__ object: every GPU that loads the
// library holds it until the process exits.  In host code its name is only a
// host-side stand-in; the device address comes from cudaGetSymbolAddress,
// looked up once per device (with that device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "isa.h"

namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(ISA_STATIC_SCRATCH_BYTES);
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_isa_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_dev[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns an isa_status.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ISA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_isa_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return ISA_ERR_CUDA;
    }
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return ISA_OK;
}

}  // namespace

extern "C" int isa_forward_static(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  uint16_t* out, void* stream) {
  const size_t need = isa_workspace_size(shape);
  // invalid or unsupported shape: isa_forward reports which, before any launch
  if (need == 0) return isa_forward(shape, q, k, v, out, nullptr, 0, stream);
  if (need > kStaticScratchBytes) return ISA_ERR_WORKSPACE;  // beyond the fixed scratch
  void* ws = nullptr;
  int rc = scratch_for_current_device(&ws);
  if (rc != ISA_OK) return rc;
  // The control block (device status word, fault-injection word) must start
  // at zero; everything else in the scratch is written before it is read.
  if (cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess) return ISA_ERR_CUDA;
  return isa_forward(shape, q, k, v, out, ws, kStaticScratchBytes, stream);
}
