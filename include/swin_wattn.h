/*
 * swin_wattn.h -- C ABI of libswinwattn.so: forward and backward shifted-window
 * multi-head self-attention (SW-MSA) over a padded token grid on NVIDIA B200
 * (sm_100a).
 *
 * What is computed. Page "TERRA: A Hierarchical Parallel Training and Memory
 * Orchestration Framework for High-Resolution AI-based Earth Modeling":
 * Abstract (window-based Swin Transformer attention with "shifted-window
 * execution" over tokens routed into window layouts) and Table I (H, W the
 * grid; H^, W^ the padded grid). The page gives no formula; the operation is
 * the published Swin shifted-window attention, per batch image b and head h:
 *   1. pad H x W to H^ x W^ (next multiples of the window) at the bottom/right;
 *   2. cyclic shift: rolled (y', x') holds ((y'+shift_h) mod H^, (x'+shift_w) mod W^);
 *   3. cut the rolled grid into win_h x win_w windows, slot i = iy*win_w + ix;
 *   4. in each window a_ij = q_i.k_j / sqrt(head_dim) + T[rel(i,j), h] where
 *      rel(i,j) = (iy-jy+win_h-1)*(2*win_w-1) + (ix-jx+win_w-1); key j is
 *      allowed for query i only when j is a real (non-pad) token and both lie in
 *      the same shift region (each rolled axis splits into [0,n-w), [n-w,n-s),
 *      [n-s,n) when s > 0); P = softmax over allowed keys (others weigh exactly
 *      0); o_i = sum_j P_ij v_j; lse_i = log sum_j exp(a_ij);
 *   5-7. window reverse, reverse shift, crop: o_i lands on its own token.
 * The backward returns dq, dk, dv and dT = sum over windows and pairs of
 * dS_ij = P_ij (dP_ij - D_i), dP_ij = dO_i.v_j, D_i = sum_j P_ij dP_ij. Pad
 * tokens produce and receive nothing.
 *
 * Layouts (all row-major, contiguous):
 *   q, k, v, out, dout, dq, dk, dv : [B, H, W, heads, head_dim] of `dtype`
 *   bias_table, dbias_table        : [(2*win_h-1)*(2*win_w-1), heads] fp32
 *   lse                            : [B, H, W, heads] fp32
 *   index map                      : [B, H^/win_h, W^/win_w, win_h*win_w] int32
 *
 * Ownership and streams. Every data pointer is device memory owned by the
 * caller, who also provides the workspace (size from swin_wattn_workspace_size;
 * 256-byte aligned). The library allocates no device memory, launches its
 * kernels on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 * stream) and never synchronises it, except swin_wattn_poll_status, which says
 * so. Calls are thread-safe; two calls in flight at once must not share a
 * workspace.
 *
 * Errors. Functions return SWIN_OK or a negative status. Arguments are checked
 * on the host before anything is launched (null pointers, shapes, a shift not
 * smaller than the window, misaligned pointers). Asynchronous kernel faults
 * surface at the caller's next synchronisation, as in CUDA. Device-side waits
 * are bounded: a wait that runs out records SWIN_ERR_TIMEOUT in the workspace,
 * the kernel returns, and swin_wattn_poll_status reports it; outputs of that
 * call are then undefined.
 */
#ifndef SWIN_WATTN_H
#define SWIN_WATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum swin_wattn_status {
  SWIN_OK = 0,
  SWIN_ERR_INVALID_ARG = -1, /* null pointer, bad shape or alignment */
  SWIN_ERR_UNSUPPORTED = -2, /* dtype / size combination not built, or not an sm_100 device */
  SWIN_ERR_WORKSPACE = -3,   /* workspace too small or misaligned */
  SWIN_ERR_CUDA = -4,        /* a CUDA runtime or driver call failed */
  SWIN_ERR_TIMEOUT = -5      /* a bounded device wait ran out (see swin_wattn_poll_status) */
};

enum swin_wattn_dtype { SWIN_DTYPE_F32 = 0, SWIN_DTYPE_BF16 = 1 };

enum swin_wattn_flags {
  SWIN_FLAG_FORCE_GENERIC = 1 << 0, /* use the portable per-token kernels even where the
                                       tcgen05 kernels apply (testing, odd shapes) */
  SWIN_FLAG_TEST_TIMEOUT = 1 << 1,  /* testing only: the fast kernels wait on a barrier
                                       nothing arrives on, with a ~1 ms limit, and report
                                       SWIN_ERR_TIMEOUT (no effect on the other kernel
                                       families, which have no device-side waits) */
  SWIN_FLAG_FORCE_TILED = 1 << 2    /* use the warp-level tensor-core kernels where they
                                       apply, even where the tcgen05 kernels would (testing) */
};

/* Problem description. Sizes: B, H, W >= 1; 1 <= win_h, win_w <= 64;
 * 0 <= shift < win per axis; heads >= 1; 8 <= head_dim <= 256 with head_dim a
 * multiple of 8. */
typedef struct swin_wattn_desc {
  int32_t B, H, W;
  int32_t win_h, win_w;
  int32_t shift_h, shift_w;
  int32_t heads, head_dim;
  int32_t dtype; /* enum swin_wattn_dtype: element type of q, k, v, out, dout, dq, dk, dv */
  int32_t flags; /* enum swin_wattn_flags */
} swin_wattn_desc;

/* Kernel family a description runs on:
 *   1 = tcgen05/TMA sm_100a kernels (bf16, 64-token windows, head_dim 32 or 64);
 *   2 = warp-level tensor-core kernels, one CTA per (window, head) with the
 *       whole window in shared memory (bf16, windows of up to 256 tokens, e.g.
 *       16 x 16, head_dim 32 or 64);
 *   0 = portable per-token CUDA kernels (everything else, fp32 included).
 * Returns a negative status for an invalid description. Host only, no CUDA
 * call. */
int swin_wattn_path(const swin_wattn_desc* desc);

/* Bytes of workspace swin_wattn_fwd and swin_wattn_bwd need for `desc`
 * (the larger of the two). Host only, no CUDA call. */
int swin_wattn_workspace_size(const swin_wattn_desc* desc, size_t* bytes);

/* Forward (steps 1-7 above). `lse` may be NULL. `bias_table` is read, never
 * written. Pointers 16-byte aligned. */
int swin_wattn_fwd(const swin_wattn_desc* desc, const void* q, const void* k, const void* v,
                   const float* bias_table, void* out, float* lse, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Backward: dq, dk, dv (same layout and dtype as q) and dbias_table, all
 * overwritten, not accumulated. The softmax rows are recomputed from q, k, v
 * and the table; no forward state is needed. dbias_table is summed in a fixed
 * order, so repeated calls give identical bits. */
int swin_wattn_bwd(const swin_wattn_desc* desc, const void* q, const void* k, const void* v,
                   const float* bias_table, const void* dout, void* dq, void* dk, void* dv,
                   float* dbias_table, void* workspace, size_t workspace_bytes, void* stream);

/* Backward without a workspace argument, for callers that cannot allocate
 * device memory or hand over a workspace when they run it: hosts whose memory
 * manager owns every device byte and forbids raw cudaMalloc, or loops that must
 * not allocate because an allocation can synchronise the device. (The pages
 * have no counterpart; this is a calling convention, not a different
 * computation.)
 *
 * Same arguments, results and kernels as swin_wattn_bwd. The scratch is a
 * static device array of SWIN_NOALLOC_SCRATCH_BYTES inside the library, which
 * every GPU that loads the library holds until the process exits; nothing is
 * allocated or freed. The first call on a device looks the array's address up
 * with that device current (cudaGetSymbolAddress), so make that first call
 * before any stream capture. All calls on a device share the array: calls
 * that overlap on the GPU (other streams, other host threads) race and give
 * undefined results. Each call clears the device status word before it runs;
 * a bounded device wait that runs out leaves the outputs undefined and is not
 * reported by this entry point.
 * Returns SWIN_ERR_UNSUPPORTED when the description does not run on the
 * tcgen05 kernels (swin_wattn_path != 1) and SWIN_ERR_WORKSPACE when the
 * workspace it needs exceeds SWIN_NOALLOC_SCRATCH_BYTES (heads * padded
 * bias-table entries * 12 bytes + 768 bytes must fit). */
#define SWIN_NOALLOC_SCRATCH_BYTES (1u << 20)
int swin_wattn_bwd_noalloc(const swin_wattn_desc* desc, const void* q, const void* k,
                           const void* v, const float* bias_table, const void* dout, void* dq,
                           void* dk, void* dv, float* dbias_table, void* stream);

/* Layout stage alone (steps 1-3): map[b, wy, wx, slot] = (b*H + y)*W + x, the
 * grid token that window slot holds, or -1 for a pad slot. */
int swin_wattn_index_map(const swin_wattn_desc* desc, int32_t* map, void* stream);

/* Synchronises `stream`, then reads the device status word of `workspace`
 * (SWIN_OK or SWIN_ERR_TIMEOUT) into *device_status and clears it. */
int swin_wattn_poll_status(void* workspace, int* device_status, void* stream);

/* Static text for a status code. */
const char* swin_wattn_strerror(int status);

/* Number of kernels this library has launched in the process so far. */
uint64_t swin_wattn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SWIN_WATTN_H */
