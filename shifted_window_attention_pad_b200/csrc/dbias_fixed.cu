// dbias_fixed.cu -- the two small kernels around the tensor-core kernels:
// the bias table in the layout they read, and the conversion of the exact
// wide-integer bias-gradient sums (dbias_fixed.cuh) to the fp32 output.
#include <cuda_runtime.h>
#include <math.h>

#include "dbias_fixed.cuh"
#include "kernels.h"

namespace swin {
namespace {

constexpr float kLog2eP = 1.4426950408889634f;

// Bias table [bins][heads] -> [heads][bins_pad], times log2(e); clears the
// gradient sums [heads][bins_pad][kLimbStride] when given.
__global__ void bias_prep_kernel(const float* __restrict__ table, int bins, int heads,
                                 int bins_pad, float* __restrict__ out,
                                 long long* __restrict__ acc) {
  // Launched as a programmatic dependent of the kernel before it (which may
  // still read this workspace): nothing is touched before that one completes.
  ptx::grid_dep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= heads * bins_pad) return;
  const int h = i / bins_pad, b = i - h * bins_pad;
  out[i] = b < bins ? table[(size_t)b * heads + h] * kLog2eP : 0.f;
  if (acc) {
#pragma unroll
    for (int k = 0; k < kLimbStride; ++k) acc[(size_t)i * kLimbStride + k] = 0;
  }
}

// dtable[bin][h] = the wide integer of (h, bin) times 2^-kLimbOff, rounded to
// fp32; NaN where a non-finite value reached the sum.
__global__ void dbias_finish_kernel(const long long* __restrict__ acc, int bins, int heads,
                                    int bins_pad, float* __restrict__ dtable) {
  ptx::grid_dep_wait();   // the gradient sums are complete once the kernel before has completed
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= bins * heads) return;
  const int b = i / heads, h = i - b * heads;
  const long long* a = acc + ((size_t)h * bins_pad + b) * kLimbStride;
  if (a[kLimbs] != 0) {
    dtable[i] = __int_as_float(0x7fc00000);
    return;
  }
  long long l[kLimbs];
#pragma unroll
  for (int k = 0; k < kLimbs; ++k) l[k] = a[k];
  // carries upwards: every limb but the top one into [0, 2^32)
#pragma unroll
  for (int k = 0; k + 1 < kLimbs; ++k) {
    const long long c = l[k] >> 32;
    l[k] -= c * 4294967296ll;
    l[k + 1] += c;
  }
  double d = (double)l[kLimbs - 1];
#pragma unroll
  for (int k = kLimbs - 2; k >= 0; --k) d = d * 4294967296.0 + (double)l[k];
  dtable[i] = (float)ldexp(d, -kLimbOff);
}

}  // namespace

size_t dbias_fixed_bytes(const Geo& g) {
  return (size_t)g.heads * bins_padded(g.bins) * kLimbStride * sizeof(long long);
}

size_t dbias_fixed_offset(const Geo& g) {
  return kWsHeader + align256((size_t)g.heads * bins_padded(g.bins) * 4);
}

namespace {
// Launch as a programmatic dependent of the previous kernel on the stream, so
// that the launch overlaps that kernel's last blocks (the kernel itself waits
// for it to complete before touching memory). The tensor-core kernels are
// launched plainly: as dependents of these small kernels they measured slower.
template <typename... Args>
cudaError_t launch_dependent(void (*kernel)(Args...), int n, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n + 255) / 256 > 0 ? (n + 255) / 256 : 1));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}
}  // namespace

cudaError_t prep_bias(const Geo& g, const float* table, float* bias_t, long long* acc,
                      cudaStream_t st) {
  return launch_dependent(bias_prep_kernel, g.heads * bins_padded(g.bins), st, table, g.bins,
                          g.heads, bins_padded(g.bins), bias_t, acc);
}

cudaError_t finish_dbias(const Geo& g, const long long* acc, float* dtable, cudaStream_t st) {
  return launch_dependent(dbias_finish_kernel, g.bins * g.heads, st, acc, g.bins, g.heads,
                          bins_padded(g.bins), dtable);
}

}  // namespace swin
