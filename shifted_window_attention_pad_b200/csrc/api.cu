// api.cu -- the C ABI of libswinwattn.so (declared in include/swin_wattn.h).
//
// Host-side checks, workspace sizing and the choice of kernel family: the
// tcgen05/TMA kernels (bf16, 64-token windows), the warp-level tensor-core
// kernels (bf16, windows of up to 256 tokens) or the portable per-token
// kernels (everything else, fp32 included). No
// device memory is allocated here and no stream is synchronised except by
// swin_wattn_poll_status.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/swin_wattn.h"
#include "kernels.h"

namespace swin {

static std::atomic<uint64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static int check_desc(const swin_wattn_desc* d) {
  if (!d) return SWIN_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->W < 1) return SWIN_ERR_INVALID_ARG;
  if (d->win_h < 1 || d->win_w < 1 || d->win_h > 64 || d->win_w > 64) return SWIN_ERR_INVALID_ARG;
  if (d->shift_h < 0 || d->shift_h >= d->win_h) return SWIN_ERR_INVALID_ARG;
  if (d->shift_w < 0 || d->shift_w >= d->win_w) return SWIN_ERR_INVALID_ARG;
  if (d->heads < 1 || d->head_dim < 8 || d->head_dim > 256 || (d->head_dim & 7))
    return SWIN_ERR_INVALID_ARG;
  if (d->dtype != SWIN_DTYPE_F32 && d->dtype != SWIN_DTYPE_BF16) return SWIN_ERR_UNSUPPORTED;
  if (d->valid_h < 0 || d->valid_h > d->H || d->valid_w < 0 || d->valid_w > d->W)
    return SWIN_ERR_INVALID_ARG;
  const long long Hp = (d->H + d->win_h - 1) / d->win_h * (long long)d->win_h;
  const long long Wp = (d->W + d->win_w - 1) / d->win_w * (long long)d->win_w;
  // Token ids of the index map are int32; grid offsets stay far inside int64.
  if ((long long)d->B * Hp * Wp > 0x7fffffffLL) return SWIN_ERR_INVALID_ARG;
  if ((long long)d->B * Hp * Wp * d->heads * d->head_dim > (1LL << 40)) return SWIN_ERR_INVALID_ARG;
  return SWIN_OK;
}

// 1 = tcgen05/TMA kernels (64-token windows), 3 = tcgen05/TMA kernels
// (256-token windows), 4 = tcgen05/TMA kernels (1024-token windows),
// 2 = warp-level tensor-core kernels, 0 = portable.
static int choose_path(const swin_wattn_desc* d, const Geo& g) {
  if (d->flags & SWIN_FLAG_FORCE_GENERIC) return 0;
  if (!(d->flags & SWIN_FLAG_FORCE_TILED)) {
    if (fast_supported(g, d->dtype)) return 1;
    if (wide_supported(g, d->dtype)) return 3;
    if (large_supported(g, d->dtype)) return 4;
  }
  if (tiled_supported(g, d->dtype)) return 2;
  return 0;
}

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? SWIN_OK : SWIN_ERR_CUDA; }

static size_t need_workspace(const swin_wattn_desc* d, const Geo& g) {
  switch (choose_path(d, g)) {
    case 1: case 3: return fast_workspace(g);
    case 4: return large_workspace(g);
    case 2: return tiled_workspace(g);
    default: return generic_workspace(g);
  }
}

static int check_ws(const swin_wattn_desc* d, const Geo& g, void* ws, size_t bytes) {
  if (!ws || ((uintptr_t)ws & 255u)) return SWIN_ERR_WORKSPACE;
  if (bytes < need_workspace(d, g)) return SWIN_ERR_WORKSPACE;
  return SWIN_OK;
}

int check_bwd_args(const swin_wattn_desc* d, const void* q, const void* k, const void* v,
                   const float* bias_table, const void* dout, const void* dq, const void* dk,
                   const void* dv, const float* dbias_table) {
  const int rc = check_desc(d);
  if (rc) return rc;
  const void* ptrs[] = {q, k, v, bias_table, dout, dq, dk, dv};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SWIN_ERR_INVALID_ARG;
  // dbias_table is not written when the exact sums are left in the workspace
  if (!(d->flags & SWIN_FLAG_DBIAS_SUMS) && !dbias_table) return SWIN_ERR_INVALID_ARG;
  if (dbias_table && !aligned16(dbias_table)) return SWIN_ERR_INVALID_ARG;
  return SWIN_OK;
}

}  // namespace swin

using namespace swin;

extern "C" {

int swin_wattn_path(const swin_wattn_desc* desc) {
  const int rc = check_desc(desc);
  if (rc) return rc;
  return choose_path(desc, make_geo(*desc));
}

int swin_wattn_workspace_size(const swin_wattn_desc* desc, size_t* bytes) {
  const int rc = check_desc(desc);
  if (rc) return rc;
  if (!bytes) return SWIN_ERR_INVALID_ARG;
  *bytes = need_workspace(desc, make_geo(*desc));
  return SWIN_OK;
}

int swin_wattn_fwd(const swin_wattn_desc* desc, const void* q, const void* k, const void* v,
                   const float* bias_table, void* out, float* lse, void* workspace,
                   size_t workspace_bytes, void* stream) {
  int rc = check_desc(desc);
  if (rc) return rc;
  if (!q || !k || !v || !bias_table || !out) return SWIN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(bias_table) || (lse && !aligned16(lse)))
    return SWIN_ERR_INVALID_ARG;
  const Geo g = make_geo(*desc);
  rc = check_ws(desc, g, workspace, workspace_bytes);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int path = choose_path(desc, g);
  if (path == 1)
    return cuda_status(fast_forward(g, q, k, v, bias_table, out, lse, workspace, desc->flags, st));
  if (path == 3)
    return cuda_status(wide_forward(g, q, k, v, bias_table, out, lse, workspace, desc->flags, st));
  if (path == 4)
    return cuda_status(large_forward(g, q, k, v, bias_table, out, lse, workspace, desc->flags, st));
  if (path == 2)
    return cuda_status(tiled_forward(g, q, k, v, bias_table, out, lse, workspace, st));
  return cuda_status(
      generic_forward(g, desc->dtype, q, k, v, bias_table, out, lse, workspace, st));
}

int swin_wattn_bwd(const swin_wattn_desc* desc, const void* q, const void* k, const void* v,
                   const float* bias_table, const void* dout, void* dq, void* dk, void* dv,
                   float* dbias_table, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_bwd_args(desc, q, k, v, bias_table, dout, dq, dk, dv, dbias_table);
  if (rc) return rc;
  const Geo g = make_geo(*desc);
  rc = check_ws(desc, g, workspace, workspace_bytes);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int path = choose_path(desc, g);
  if (path == 0 && (desc->flags & SWIN_FLAG_DBIAS_SUMS)) return SWIN_ERR_UNSUPPORTED;
  if (path == 1)
    return cuda_status(fast_backward(g, q, k, v, bias_table, dout, dq, dk, dv, dbias_table,
                                     workspace, desc->flags, st));
  if (path == 3)
    return cuda_status(wide_backward(g, q, k, v, bias_table, dout, dq, dk, dv, dbias_table,
                                     workspace, desc->flags, st));
  if (path == 4)
    return cuda_status(large_backward(g, q, k, v, bias_table, dout, dq, dk, dv, dbias_table,
                                      workspace, desc->flags, st));
  if (path == 2)
    return cuda_status(tiled_backward(g, q, k, v, bias_table, dout, dq, dk, dv, dbias_table,
                                      workspace, desc->flags, st));
  return cuda_status(generic_backward(g, desc->dtype, q, k, v, bias_table, dout, dq, dk, dv,
                                      dbias_table, workspace, st));
}

// Band geometry: the description is the band's own; the shift wraps into
// the halo tensor, whose rows the band must be able to hold a window of.
static int band_geo(const swin_wattn_desc* desc, const swin_wattn_halo* halo, Geo& g) {
  if (!halo) return SWIN_ERR_INVALID_ARG;
  g = make_geo(*desc);
  if (choose_path(desc, g) != 1) return SWIN_ERR_UNSUPPORTED;
  if (halo->interior && (desc->H % desc->win_h)) return SWIN_ERR_INVALID_ARG;
  if (desc->H < desc->shift_h) return SWIN_ERR_INVALID_ARG;
  if (desc->valid_h && desc->valid_h < desc->H && halo->interior) return SWIN_ERR_INVALID_ARG;
  g.band = 1;
  g.seam_h = halo->interior ? 0 : desc->shift_h;
  return SWIN_OK;
}

int swin_wattn_fwd_band(const swin_wattn_desc* desc, const swin_wattn_halo* halo, const void* q,
                        const void* k, const void* v, const float* bias_table, void* out,
                        float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_desc(desc);
  if (rc) return rc;
  if (!q || !k || !v || !bias_table || !out) return SWIN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(bias_table) || (lse && !aligned16(lse)))
    return SWIN_ERR_INVALID_ARG;
  Geo g;
  rc = band_geo(desc, halo, g);
  if (rc) return rc;
  if (desc->shift_h > 0) {
    const void* hp[] = {halo->q, halo->k, halo->v, halo->out};
    for (const void* p : hp)
      if (!p || !aligned16(p)) return SWIN_ERR_INVALID_ARG;
    if (lse && (!halo->lse || !aligned16(halo->lse))) return SWIN_ERR_INVALID_ARG;
  }
  rc = check_ws(desc, g, workspace, workspace_bytes);
  if (rc) return rc;
  return cuda_status(fast_forward(g, q, k, v, bias_table, out, lse, workspace, desc->flags,
                                  (cudaStream_t)stream, halo));
}

int swin_wattn_bwd_band(const swin_wattn_desc* desc, const swin_wattn_halo* halo, const void* q,
                        const void* k, const void* v, const float* bias_table, const void* dout,
                        void* dq, void* dk, void* dv, float* dbias_table, void* workspace,
                        size_t workspace_bytes, void* stream) {
  int rc = check_bwd_args(desc, q, k, v, bias_table, dout, dq, dk, dv, dbias_table);
  if (rc) return rc;
  Geo g;
  rc = band_geo(desc, halo, g);
  if (rc) return rc;
  if (desc->shift_h > 0) {
    const void* hp[] = {halo->q, halo->k, halo->v, halo->dout, halo->dq, halo->dk, halo->dv};
    for (const void* p : hp)
      if (!p || !aligned16(p)) return SWIN_ERR_INVALID_ARG;
  }
  rc = check_ws(desc, g, workspace, workspace_bytes);
  if (rc) return rc;
  return cuda_status(fast_backward(g, q, k, v, bias_table, dout, dq, dk, dv, dbias_table,
                                   workspace, desc->flags, (cudaStream_t)stream, halo));
}

int swin_wattn_index_map(const swin_wattn_desc* desc, int32_t* map, void* stream) {
  const int rc = check_desc(desc);
  if (rc) return rc;
  if (!map) return SWIN_ERR_INVALID_ARG;
  return cuda_status(index_map(make_geo(*desc), map, (cudaStream_t)stream));
}

int swin_wattn_dbias_sums(const swin_wattn_desc* desc, size_t* offset, size_t* bytes) {
  const int rc = check_desc(desc);
  if (rc) return rc;
  if (!offset || !bytes) return SWIN_ERR_INVALID_ARG;
  const Geo g = make_geo(*desc);
  if (choose_path(desc, g) == 0) return SWIN_ERR_UNSUPPORTED;
  *offset = dbias_fixed_offset(g);
  *bytes = dbias_fixed_bytes(g);
  return SWIN_OK;
}

int swin_wattn_dbias_finish(const swin_wattn_desc* desc, const void* workspace,
                            float* dbias_table, void* stream) {
  const int rc = check_desc(desc);
  if (rc) return rc;
  if (!dbias_table || !aligned16(dbias_table)) return SWIN_ERR_INVALID_ARG;
  if (!workspace || ((uintptr_t)workspace & 255u)) return SWIN_ERR_WORKSPACE;
  const Geo g = make_geo(*desc);
  if (choose_path(desc, g) == 0) return SWIN_ERR_UNSUPPORTED;
  const long long* acc = (const long long*)((const char*)workspace + dbias_fixed_offset(g));
  return cuda_status(finish_dbias(g, acc, dbias_table, (cudaStream_t)stream));
}

int swin_wattn_layout_map(const swin_wattn_desc* desc, void* ids, int32_t* map,
                          int32_t* labels, void* stream) {
  const int rc = check_desc(desc);
  if (rc) return rc;
  if (!ids || !map || !aligned16(ids)) return SWIN_ERR_INVALID_ARG;
  const Geo g = make_geo(*desc);
  if (choose_path(desc, g) != 1) return SWIN_ERR_UNSUPPORTED;
  return cuda_status(fast_layout_map(g, ids, map, labels, (cudaStream_t)stream));
}

int swin_wattn_poll_status(void* workspace, int* device_status, void* stream) {
  if (!workspace || !device_status) return SWIN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SWIN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SWIN_ERR_CUDA;
  *device_status = v;
  if (v != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return SWIN_ERR_CUDA;
  return SWIN_OK;
}

const char* swin_wattn_strerror(int status) {
  switch (status) {
    case SWIN_OK: return "ok";
    case SWIN_ERR_INVALID_ARG: return "invalid argument (null pointer, shape or alignment)";
    case SWIN_ERR_UNSUPPORTED: return "unsupported dtype/size combination or device";
    case SWIN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SWIN_ERR_CUDA: return "CUDA runtime or driver call failed";
    case SWIN_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    default: return "unknown status";
  }
}

uint64_t swin_wattn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
