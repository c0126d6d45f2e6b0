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

// Bias table in the layout the tensor-core kernels read ([heads][bins_pad],
// times log2 e), and the exact wide-integer bias-gradient sums they fill
// ([heads][bins_pad][kLimbStride] int64, dbias_fixed.cuh), cleared by
// prep_bias and converted to the fp32 [bins][heads] output by finish_dbias.
size_t dbias_fixed_bytes(const Geo& g);
// Byte offset of those sums in the workspace of either tensor-core family.
size_t dbias_fixed_offset(const Geo& g);
cudaError_t prep_bias(const Geo& g, const float* table, float* bias_t, long long* acc,
                      cudaStream_t st);
cudaError_t finish_dbias(const Geo& g, const long long* acc, float* dtable, cudaStream_t st);

// Host-side checks of swin_wattn_bwd's description and data pointers (null,
// 16-byte alignment), without the workspace: SWIN_OK or a negative status.
int check_bwd_args(const swin_wattn_desc* d, const void* q, const void* k, const void* v,
                   const float* bias_table, const void* dout, const void* dq, const void* dk,
                   const void* dv, const float* dbias_table);

// Deterministic sum of per-unit bias-gradient partials laid out
// [unit][heads][bins_pad] into dtable [bins][heads].
cudaError_t dbias_reduce(const Geo& g, const float* partial, long long n_units, float* dtable,
                         cudaStream_t st);

// ---- tcgen05 / TMA kernels for sm_100a (bf16) ---------------------------------
bool fast_supported(const Geo& g, int dtype);
size_t fast_workspace(const Geo& g);
// `halo` (row band: g.band = 1) gives the halo inputs and outputs; NULL otherwise.
cudaError_t fast_forward(const Geo& g, const void* q, const void* k, const void* v,
                         const float* table, void* out, float* lse, void* ws, int flags,
                         cudaStream_t st, const swin_wattn_halo* halo = nullptr);
cudaError_t fast_backward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, const void* dout, void* dq, void* dk, void* dv,
                          float* dtable, void* ws, int flags, cudaStream_t st,
                          const swin_wattn_halo* halo = nullptr);
// The layout stage exactly as those kernels run it (TMA boxes, row order,
// per-row info): fills `ids` with token ids, then writes the token of every
// window slot (-1 pad, -2 inconsistency) and optionally its region label.
cudaError_t fast_layout_map(const Geo& g, void* ids, int32_t* map, int32_t* labels,
                            cudaStream_t st);

// ---- tcgen05 / TMA kernels for 256-token windows (bf16, head_dim 32 or 64);
// workspace as fast_workspace --------------------------------------------------
bool wide_supported(const Geo& g, int dtype);
cudaError_t wide_forward(const Geo& g, const void* q, const void* k, const void* v,
                         const float* table, void* out, float* lse, void* ws, int flags,
                         cudaStream_t st);
cudaError_t wide_backward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, const void* dout, void* dq, void* dk, void* dv,
                          float* dtable, void* ws, int flags, cudaStream_t st);

// ---- tcgen05 / TMA kernels for 1024-token windows (32 x 32, bf16, head_dim
// 64 or 128) --------------------------------------------------------------------
bool large_supported(const Geo& g, int dtype);
size_t large_workspace(const Geo& g);
cudaError_t large_forward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, void* out, float* lse, void* ws, int flags,
                          cudaStream_t st);
cudaError_t large_backward(const Geo& g, const void* q, const void* k, const void* v,
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
                           float* dtable, void* ws, int flags, cudaStream_t st);

}  // namespace swin
