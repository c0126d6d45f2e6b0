// kernels.h -- launchers shared between the C ABI and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "geometry.cuh"

namespace swin {

// Count of kernel launches made by this library (reported by swin_wattn_launch_count).
void note_launch(int n = 1);

// Workspace layout shared by the launchers: a 256-byte header holding the
// device status word, then 256-byte aligned regions.
constexpr size_t kWsHeader = 256;
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int bins_padded(int bins) { return (bins + 3) & ~3; }

// ---- portable per-token kernels (any supported shape, fp32 or bf16) ----------
size_t generic_workspace(const Geo& g);
cudaError_t generic_forward(const Geo& g, int dtype, const void* q, const void* k, const void* v,
                            const float* table, void* out, float* lse, void* ws,
                            cudaStream_t st);
cudaError_t generic_backward(const Geo& g, int dtype, const void* q, const void* k,
                             const void* v, const float* table, const void* dout, void* dq,
                             void* dk, void* dv, float* dtable, void* ws, cudaStream_t st);
cudaError_t index_map(const Geo& g, int32_t* map, cudaStream_t st);

// Deterministic sum of per-unit bias-gradient partials laid out
// [unit][heads][bins_pad] into dtable [bins][heads].
cudaError_t dbias_reduce(const Geo& g, const float* partial, long long n_units, float* dtable,
                         cudaStream_t st);

// ---- tcgen05 / TMA kernels for sm_100a (bf16) ---------------------------------
bool fast_supported(const Geo& g, int dtype);
size_t fast_workspace(const Geo& g);
cudaError_t fast_forward(const Geo& g, const void* q, const void* k, const void* v,
                         const float* table, void* out, float* lse, void* ws, int flags,
                         cudaStream_t st);
cudaError_t fast_backward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, const void* dout, void* dq, void* dk, void* dv,
                          float* dtable, void* ws, int flags, cudaStream_t st);

// ---- warp-level tensor-core kernels: one CTA per (window, head), windows of
// up to 256 tokens (bf16, head_dim 32 or 64) ----------------------------------
bool tiled_supported(const Geo& g, int dtype);
size_t tiled_workspace(const Geo& g);
cudaError_t tiled_forward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, void* out, float* lse, void* ws, cudaStream_t st);
cudaError_t tiled_backward(const Geo& g, const void* q, const void* k, const void* v,
                           const float* table, const void* dout, void* dq, void* dk, void* dv,
                           float* dtable, void* ws, cudaStream_t st);

}  // namespace swin
