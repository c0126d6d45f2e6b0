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
 * Tokens beyond the descriptor's valid extent are pad tokens too.
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
  SWIN_FLAG_FORCE_TILED = 1 << 2,   /* use the warp-level tensor-core kernels where they
                                       apply, even where the tcgen05 kernels would (testing) */
  SWIN_FLAG_DBIAS_SUMS = 1 << 3     /* swin_wattn_bwd on the tensor-core kernels: leave the
                                       exact bias-gradient sums in the workspace instead of
                                       writing dbias_table (which may then be NULL), so that
                                       partial sums of several calls or ranks can be added as
                                       integers (swin_wattn_dbias_sums) and converted once
                                       (swin_wattn_dbias_finish) */
};

/* Problem description. Sizes: B, H, W >= 1; 1 <= win_h, win_w <= 64;
 * 0 <= shift < win per axis; heads >= 1; 8 <= head_dim <= 256 with head_dim a
 * multiple of 8; 0 <= valid_h <= H, 0 <= valid_w <= W.
 *
 * Valid extent (valid_h, valid_w; 0 = H, W): Table I of the page pads the
 * physical field before it is cut into patches, so stored tokens can cover
 * only padded pixels (a 2041 x 4320 field padded to 2048 x 4352 in patches of
 * 8 gives 256 x 544 tokens of which columns 540..543 hold no data; pass
 * valid_h = ceil(field rows / patch), valid_w = ceil(field columns / patch)).
 * Tokens at row >= valid_h or column >= valid_w are padding: they are no key
 * of any query and their outputs (out, lse, dq, dk, dv) are written as zeros.
 * The window grid still follows the stored H x W. */
typedef struct swin_wattn_desc {
  int32_t B, H, W;
  int32_t win_h, win_w;
  int32_t shift_h, shift_w;
  int32_t heads, head_dim;
  int32_t dtype; /* enum swin_wattn_dtype: element type of q, k, v, out, dout, dq, dk, dv */
  int32_t flags; /* enum swin_wattn_flags */
  int32_t valid_h, valid_w; /* valid extent of the token grid; 0 = the whole grid */
} swin_wattn_desc;

/* Kernel family a description runs on:
 *   1 = tcgen05/TMA sm_100a kernels (bf16, 64-token windows, e.g. 8 x 8,
 *       head_dim 32, 64 or 128);
 *   3 = tcgen05/TMA kernels for 256-token windows (bf16, e.g. 16 x 16,
 *       head_dim 32 or 64);
 *   4 = tcgen05/TMA kernels for 1024-token windows (bf16, 32 x 32, head_dim
 *       64 or 128, shifts whose 128-token block sub-boxes are whole 8-row
 *       swizzle atoms, e.g. 16), with an online softmax over 128-token blocks;
 *   2 = warp-level tensor-core kernels, one CTA per (window, head) with the
 *       whole window in shared memory (bf16, windows of up to 256 tokens the
 *       families above do not take, e.g. 7 x 7, head_dim 32 or 64);
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
 * and the table; no forward state is needed. On the tensor-core kernels
 * (paths 1-4) dbias_table is summed exactly in integers whose unit follows
 * the magnitude of each tile's gradients, then rounded once to fp32: repeated
 * calls give identical bits, and the relative error does not depend on the
 * scale of dout. A NaN or infinity reaching a head's gradient makes that
 * head's dbias_table NaN. The portable kernels sum fp32 partials per window in
 * a fixed order (also repeatable). */
int swin_wattn_bwd(const swin_wattn_desc* desc, const void* q, const void* k, const void* v,
                   const float* bias_table, const void* dout, void* dq, void* dk, void* dv,
                   float* dbias_table, void* workspace, size_t workspace_bytes, void* stream);

/* Row bands of a grid split across devices (TERRA page, Fig. 6 and Table III:
 * window layouts placed on devices with boundary-only peer-to-peer
 * exchange). Band r holds rows [r*R, r*R + H) of a grid of Hg rows, R a
 * multiple of win_h; the description of a band call is the band's own: H =
 * its rows (a multiple of win_h except in the last band), everything else as
 * for the whole grid. The shift moves content up by shift_h, so the band's
 * last window row reads the shift_h rows below the band -- the next band's
 * first rows, or for the last band the grid's first rows (the wrap) -- from
 * `q`, `k`, `v`, `dout` here, each [B, shift_h, W, heads, head_dim], and
 * writes the outputs of those rows to `out`, `lse`, `dq`, `dk`, `dv` of the
 * same shape, which belong to the band that owns them. The band's own first
 * shift_h rows are computed, and their outputs written, by the band above.
 * `interior` = 1 for every band but the last one: its last window row lies
 * inside the grid, so no shift-region split applies there. All pointers are
 * device memory, 16-byte aligned; a band call with interior = 0 and halo
 * pointers equal to the band's own first rows is the whole-grid call. */
typedef struct swin_wattn_halo {
  int32_t interior;
  const void* q;
  const void* k;
  const void* v;
  const void* dout; /* backward only */
  void* out;        /* forward only */
  float* lse;       /* forward only; used when the call's lse is not NULL */
  void* dq;         /* backward only */
  void* dk;
  void* dv;
} swin_wattn_halo;

/* Forward and backward of one row band (tcgen05 kernels only:
 * SWIN_ERR_UNSUPPORTED where swin_wattn_path != 1). Arguments as for
 * swin_wattn_fwd / swin_wattn_bwd plus `halo`; dbias_table (or the exact sums
 * under SWIN_FLAG_DBIAS_SUMS) covers the band's windows, so a grid's table is
 * the sum over its bands. */
int swin_wattn_fwd_band(const swin_wattn_desc* desc, const swin_wattn_halo* halo, const void* q,
                        const void* k, const void* v, const float* bias_table, void* out,
                        float* lse, void* workspace, size_t workspace_bytes, void* stream);
int swin_wattn_bwd_band(const swin_wattn_desc* desc, const swin_wattn_halo* halo, const void* q,
                        const void* k, const void* v, const float* bias_table, const void* dout,
                        void* dq, void* dk, void* dv, float* dbias_table, void* workspace,
                        size_t workspace_bytes, void* stream);

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
 * Arguments are checked on the host before anything is queued.
 * Returns SWIN_ERR_UNSUPPORTED when the description does not run on the
 * tcgen05 kernels (swin_wattn_path != 1) and SWIN_ERR_WORKSPACE when the
 * workspace it needs exceeds SWIN_NOALLOC_SCRATCH_BYTES. That workspace is
 * exactly 256 + r(heads * bp * 4) + r(heads * bp * 80) bytes, bp = bias-table
 * entries rounded up to a multiple of 4, r() = round up to 256 (with 8 x 8
 * windows, bp = 228: up to 54 heads fit). */
#define SWIN_NOALLOC_SCRATCH_BYTES (1u << 20)
int swin_wattn_bwd_noalloc(const swin_wattn_desc* desc, const void* q, const void* k,
                           const void* v, const float* bias_table, const void* dout, void* dq,
                           void* dk, void* dv, float* dbias_table, void* stream);

/* Layout stage alone (steps 1-3): map[b, wy, wx, slot] = (b*H + y)*W + x, the
 * grid token that window slot holds, or -1 for a pad slot. */
int swin_wattn_index_map(const swin_wattn_desc* desc, int32_t* map, void* stream);

/* Where the exact bias-gradient sums of a SWIN_FLAG_DBIAS_SUMS backward sit
 * in its workspace: `*offset` bytes from the start, `*bytes` long, int64 words
 * [heads][bins rounded up to 4][10]. Sums of several calls (other images of
 * a batch, other ranks of a data-parallel group) add word by word as int64
 * (no carries needed), and swin_wattn_dbias_finish of the added words equals
 * what one call over all of them would give, bit for bit. Host only;
 * SWIN_ERR_UNSUPPORTED for the portable kernels (path 0). */
int swin_wattn_dbias_sums(const swin_wattn_desc* desc, size_t* offset, size_t* bytes);

/* Converts the exact sums at swin_wattn_dbias_sums' offset of `workspace` to
 * dbias_table ([(2*win_h-1)*(2*win_w-1), heads] fp32, overwritten). */
int swin_wattn_dbias_finish(const swin_wattn_desc* desc, const void* workspace,
                            float* dbias_table, void* stream);

/* Layout stage (steps 1-3) exactly as the tcgen05 kernels run it, for
 * bit-exact checks of their addressing: fills `ids` (caller-owned device
 * memory of B*H*W*heads*head_dim bf16 words, 16-byte aligned, overwritten)
 * with token ids, loads every window's tile with the kernels' own TMA boxes
 * and row order, and writes map[b, wy, wx, slot] = the grid token found in
 * that slot's row (-1 for a pad slot; -2 where the loaded token disagrees
 * with the token the kernels' epilogue would store to). `labels` (same shape,
 * may be NULL) receives each slot's shift-region label 3*r_y + r_x.
 * SWIN_ERR_UNSUPPORTED unless swin_wattn_path(desc) == 1. */
int swin_wattn_layout_map(const swin_wattn_desc* desc, void* ids, int32_t* map, int32_t* labels,
                          void* stream);

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
