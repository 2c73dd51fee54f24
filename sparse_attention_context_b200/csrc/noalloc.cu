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
#include "isa_internal.h"

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
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return isa::record_cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) return isa::record_cuda_status(cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_isa_static_scratch);
    if (e == cudaSuccess && p == nullptr) e = cudaErrorInvalidSymbol;
    if (e != cudaSuccess) {
      cudaGetLastError();  // take it out of the runtime's last-error slot; isa_last_error keeps it
      return isa::record_cuda_status(e);
    }
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return ISA_OK;
}

}  // namespace

extern "C" int isa_forward_static(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  uint16_t* out, void* stream) {
  isa::NvtxRange nvtx_("isa_forward_static");
  const size_t need = isa_workspace_size(shape);
  // invalid or unsupported shape: isa_forward reports which, before any launch
  if (need == 0) return isa_forward(shape, q, k, v, out, nullptr, 0, stream);
  if (need > kStaticScratchBytes) return ISA_ERR_WORKSPACE;  // beyond the fixed scratch
  void* ws = nullptr;
  int rc = scratch_for_current_device(&ws);
  if (rc != ISA_OK) return rc;
  // The control block (device status word, fault-injection word) must start
  // at zero; everything else in the scratch is written before it is read.
  const cudaError_t e = cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return isa::record_cuda_status(e);
  return isa_forward(shape, q, k, v, out, ws, kStaticScratchBytes, stream);
}
