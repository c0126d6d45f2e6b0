// noalloc.cu -- backward entry point whose scratch is a static device array.
//
// Some callers cannot call cudaMalloc (or be handed a workspace) at the point
// where they run the backward: hosts whose memory manager owns every device
// byte and forbids raw allocations, or loops that must not allocate because
// an allocation can synchronise the device. swin_wattn_bwd_noalloc serves
// them: it runs exactly the same kernels as swin_wattn_bwd, but the
// workspace is the file-scope array below, which every GPU that loads the
// library holds until the process exits. The caller still passes all inputs
// and outputs. Nothing here calls cudaMalloc, cudaFree or an allocating
// library routine.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/swin_wattn.h"
#include "kernels.h"

namespace swin {
namespace {

// The scratch itself. In host code `g_scratch` is only a host-side stand-in
// for the symbol: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_scratch[SWIN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per
// device (with that device current) and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = ptr;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace swin

using namespace swin;

extern "C" int swin_wattn_bwd_noalloc(const swin_wattn_desc* desc, const void* q, const void* k,
                                      const void* v, const float* bias_table, const void* dout,
                                      void* dq, void* dk, void* dv, float* dbias_table,
                                      void* stream) {
  // Every argument is checked before anything is queued on the stream.
  int rc = check_bwd_args(desc, q, k, v, bias_table, dout, dq, dk, dv, dbias_table);
  if (rc) return rc;
  if (swin_wattn_path(desc) != 1) return SWIN_ERR_UNSUPPORTED;   // only the tcgen05 kernels run here
  size_t need = 0;
  rc = swin_wattn_workspace_size(desc, &need);
  if (rc) return rc;
  if (need > (size_t)SWIN_NOALLOC_SCRATCH_BYTES) return SWIN_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return SWIN_ERR_CUDA;
  // The status word must start at zero; the bias-gradient table is cleared by
  // the backward's own first kernel. Everything else is overwritten before use.
  if (cudaMemsetAsync(scratch, 0, sizeof(int), (cudaStream_t)stream) != cudaSuccess)
    return SWIN_ERR_CUDA;
  return swin_wattn_bwd(desc, q, k, v, bias_table, dout, dq, dk, dv, dbias_table, scratch,
                        (size_t)SWIN_NOALLOC_SCRATCH_BYTES, stream);
}
