// fast_common.cuh -- pieces shared by the tcgen05 / TMA kernel files: launch
// parameters, the shared-memory layout of a tile ring, the layout stage as TMA
// boxes (sub-boxes of a window on the wrap seam, slot order, per-row info),
// the per-row softmax helpers, row stores, and the host-side tensor-map
// encoding. Included by one translation unit per kernel family; everything
// sits in an unnamed namespace, so each unit keeps its own copy.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "dbias_fixed.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace swin {
namespace {

using namespace ptx;

constexpr int kRows = 128;        // tile rows = TMEM lanes = UMMA M
constexpr int kWg = 128;          // threads of one softmax / epilogue warpgroup
constexpr int kNumWg = 2;         // warpgroups 0 (warps 0-3) and 1 (warps 4-7) alternate tiles
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;       // issues S (and dP); allocates and frees TMEM
constexpr int kMma2Warp = 10;     // issues PV (forward) or the gradient products (backward)
constexpr int kFoldWarp = 11;     // backward: folds each tile's bias-gradient bins into global sums
constexpr int kThreads = 384;
constexpr int kMaxMaps = 9;       // box shapes: {full, seam part 1, seam part 2}^2
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kTestLimitNs = 1000000ull;
constexpr float kLog2e = 1.4426950408889634f;

struct FastParams {
  CUtensorMap maps[4][kMaxMaps];  // [q, k, v, dout][ky * 3 + kx]
  Geo g;
  long long n_groups;             // tiles per head: ceil(n_win / G)
  long long n_tiles;              // n_groups * heads
  int bins_pad;
  float scale_log2;               // head_dim^-1/2 * log2(e)
  const float* bias_t;            // [heads][bins_pad], times log2(e)
  void* out0;                     // forward: out;  backward: dq
  void* out1;                     // backward: dk
  void* out2;                     // backward: dv
  float* lse;                     // forward, optional
  void* out0h;                    // row band: outputs of the halo rows (same roles)
  void* out1h;
  void* out2h;
  float* lse_h;
  long long* dt_acc;              // backward: exact bias-gradient sums [heads][bins_pad][kLimbStride]
  int* status;                    // device status word (workspace header)
  int test_timeout;
};

// ---- shared-memory layout (same arithmetic on host and device) ------------------
// A TMA box carries at most 64 channels (128 bytes, the swizzle span), so a
// head_dim of 128 is loaded as two channel halves, each a [128 rows][64]
// region of its own; smaller head_dims are one region of [128 rows][HD].
template <int HD>
struct TileGeom {
  static constexpr int kBoxEl = HD > 64 ? 64 : HD;            // channels of one box
  static constexpr int kHalves = HD / kBoxEl;
  static constexpr uint32_t kRowBytes = kBoxEl * 2;           // a row inside one region
  static constexpr uint32_t kHalfBytes = kRows * kRowBytes;   // one region
  static constexpr int kStepsPerHalf = kBoxEl / 16;           // K steps of 16 per region
};

struct Layout {
  uint32_t tiles, ptile, bias, colinfo, bins_w, bars, misc, total;
};

// NS stages of NTEN input tiles, then PBYTES of P / dS operand blocks, the
// bias rows of the stages, NCOLBUF buffers of key words, int32 bias-gradient
// bins per warp of NBINWG warpgroups (two warps hold a window's rows) and four
// per-warp bounds each, mbarriers and two words (TMEM base, abort flag).
template <int HD, int NS, int NTEN, uint32_t PBYTES, int NCOLBUF = 2 * kNumWg,
          int NBINWG = kNumWg>
__host__ __device__ inline Layout make_layout(int bins_pad) {
  constexpr uint32_t tile_bytes = kRows * HD * 2;
  Layout L;
  L.tiles = 0;
  L.ptile = L.tiles + NS * NTEN * tile_bytes;
  L.bias = L.ptile + PBYTES;
  L.colinfo = L.bias + ((NS * bins_pad * 4 + 15) & ~15);
  L.bins_w = L.colinfo + NCOLBUF * kRows * 4;
  L.bars = (L.bins_w + NBINWG * (4 * bins_pad + 4) * 4 + 7) & ~7u;
  L.misc = L.bars + 8 * 32;
  L.total = L.misc + 16;
  return L;
}

// Rows of the 128-row tile are windows g = row / N; inside a window the rows
// follow the sub-boxes column segment first (x segment, then y segment), each
// row-major -- so within a column segment the window's rows come in their
// natural order whether or not the window wraps at the row seam. A row band
// changes only the wrapping of rows, so a window keeps its slot order (and a
// row's sums add its keys in the same order) in a band and in the whole grid.
struct SubBox {
  int y, x, rows, cols, map_id, row_off;
};

__device__ inline void window_coords(const Geo& g, long long win, int& b, int& wy, int& wx) {
  const long long per_b = (long long)g.nWy * g.nWx;
  b = (int)(win / per_b);
  const int r = (int)(win - (long long)b * per_b);
  wy = r / g.nWx;
  wx = r - wy * g.nWx;
}

// Sub-boxes of window (wy, wx): source start, size, box-shape id, first row.
__device__ inline int plan_window(const Geo& g, int wy, int wx, SubBox* sb) {
  const bool wrap_y = g.sh > 0 && wy == g.nWy - 1;
  const bool wrap_x = g.sw > 0 && wx == g.nWx - 1;
  int ys[2], yl[2], yk[2], xs[2], xl[2], xk[2];
  const int ny = wrap_y ? 2 : 1, nx = wrap_x ? 2 : 1;
  if (wrap_y) {
    ys[0] = 0; yl[0] = g.wh - g.sh; yk[0] = 1;
    ys[1] = g.wh - g.sh; yl[1] = g.sh; yk[1] = 2;
  } else {
    ys[0] = 0; yl[0] = g.wh; yk[0] = 0;
  }
  if (wrap_x) {
    xs[0] = 0; xl[0] = g.ww - g.sw; xk[0] = 1;
    xs[1] = g.ww - g.sw; xl[1] = g.sw; xk[1] = 2;
  } else {
    xs[0] = 0; xl[0] = g.ww; xk[0] = 0;
  }
  int n = 0, off = 0;
  for (int c = 0; c < nx; ++c)
    for (int a = 0; a < ny; ++a) {
      sb[n].y = (wy * g.wh + ys[a] + g.sh) % g.Hp;
      sb[n].x = (wx * g.ww + xs[c] + g.sw) % g.Wp;
      sb[n].rows = yl[a];
      sb[n].cols = xl[c];
      sb[n].map_id = yk[a] * 3 + xk[c];
      sb[n].row_off = off;
      off += yl[a] * xl[c];
      ++n;
    }
  return n;
}

// Slot coordinates (iy, ix) of row r (0..N-1) of window (wy, wx) in sub-box
// order: column segments of w0 and ww - w0 columns, each all wh rows in order.
__device__ inline void row_slot(const Geo& g, int wy, int wx, int r, int& iy, int& ix) {
  const bool wrap_x = g.sw > 0 && wx == g.nWx - 1;
  const int w0 = wrap_x ? g.ww - g.sw : g.ww;
  const int xseg = r >= g.wh * w0;
  const int rr = xseg ? r - g.wh * w0 : r;
  const int wseg = xseg ? g.ww - w0 : w0;
  iy = rr / wseg;
  ix = (xseg ? w0 : 0) + (rr - iy * wseg);
}

// Everything the softmax warpgroup needs to know about its own row.
struct RowInfo {
  bool valid;       // a real token (inside the valid extent)
  bool stored;      // inside the stored grid: its outputs are written
  bool halo;        // row band: a row of the halo tensor (token counts in its [B, sh, W])
  int label;        // shift region 0..8
  int bias_base;    // (iy + wh - 1)(2 ww - 1) + ix + ww - 1
  int key_off;      // iy (2 ww - 1) + ix : subtract from a query's base to index the table
  long long token;  // (b H + y) W + x
};

// Row of slot (iy, ix) of window (wy, wx) of image b.
__device__ inline RowInfo row_info_at(const Geo& g, int b, int wy, int wx, int iy, int ix) {
  RowInfo ri;
  ri.halo = false;
  const int yr = wy * g.wh + iy, xr = wx * g.ww + ix;
  const int y = (yr + g.sh) % g.Hp, x = (xr + g.sw) % g.Wp;
  ri.stored = y < g.H && x < g.W;
  ri.valid = y < g.Hv && x < g.Wv;
  ri.label = 3 * region_1d(yr, g.Hp, g.wh, g.seam_h) + region_1d(xr, g.Wp, g.ww, g.sw);
  ri.bias_base = (iy + g.wh - 1) * (2 * g.ww - 1) + ix + g.ww - 1;
  ri.key_off = iy * (2 * g.ww - 1) + ix;
  ri.token = ((long long)b * g.H + y) * g.W + x;
  if (g.band && yr + g.sh >= g.Hp) {   // wrapped row: source row y < sh of the halo tensor
    ri.halo = true;
    ri.stored = x < g.W;
    ri.valid = x < g.Wv;
    ri.token = ((long long)b * g.sh + y) * g.W + x;
  }
  return ri;
}

__device__ inline RowInfo no_row() {
  RowInfo ri;
  ri.valid = false;
  ri.stored = false;
  ri.halo = false;
  ri.label = 15;
  ri.bias_base = 0;
  ri.key_off = 0;
  ri.token = 0;
  return ri;
}

__device__ inline RowInfo row_info(const Geo& g, long long win, int r) {
  if (win >= g.n_win) return no_row();
  int b, wy, wx, iy, ix;
  window_coords(g, win, b, wy, wx);
  row_slot(g, wy, wx, r, iy, ix);
  return row_info_at(g, b, wy, wx, iy, ix);
}

// ---- windows of more than 256 tokens: 128-token blocks --------------------------
// A window of ww = 32 columns is taken in blocks of 128 slots, 128 / ww whole
// window rows each. Inside a block the slots follow its sub-boxes column
// segment first, as for a whole window, so a block of a window on the column
// seam is two (or, where the block also straddles the row seam, four)
// sub-boxes. Block-row boxes have 128 / ww rows, or the two parts
// (wh - sh) mod (128 / ww) and the rest where a block straddles the row seam.
__device__ inline int plan_block(const Geo& g, int wy, int wx, int blk, SubBox* sb) {
  const int bh = kRows / g.ww;
  const int y0 = blk * bh;
  const int ysplit = g.wh - g.sh;   // first window row whose source row wraps
  const bool split_y = g.sh > 0 && wy == g.nWy - 1 && ysplit > y0 && ysplit < y0 + bh;
  const bool wrap_x = g.sw > 0 && wx == g.nWx - 1;
  int ys[2], yl[2], yk[2], xs[2], xl[2], xk[2];
  const int ny = split_y ? 2 : 1, nx = wrap_x ? 2 : 1;
  if (split_y) {
    ys[0] = y0; yl[0] = ysplit - y0; yk[0] = 1;
    ys[1] = ysplit; yl[1] = y0 + bh - ysplit; yk[1] = 2;
  } else {
    ys[0] = y0; yl[0] = bh; yk[0] = 0;
  }
  if (wrap_x) {
    xs[0] = 0; xl[0] = g.ww - g.sw; xk[0] = 1;
    xs[1] = g.ww - g.sw; xl[1] = g.sw; xk[1] = 2;
  } else {
    xs[0] = 0; xl[0] = g.ww; xk[0] = 0;
  }
  int n = 0, off = 0;
  for (int c = 0; c < nx; ++c)
    for (int a = 0; a < ny; ++a) {
      sb[n].y = (wy * g.wh + ys[a] + g.sh) % g.Hp;
      sb[n].x = (wx * g.ww + xs[c] + g.sw) % g.Wp;
      sb[n].rows = yl[a];
      sb[n].cols = xl[c];
      sb[n].map_id = yk[a] * 3 + xk[c];
      sb[n].row_off = off;
      off += yl[a] * xl[c];
      ++n;
    }
  return n;
}

// Row of window slot r (block r / 128, slot r % 128 of the block).
__device__ inline RowInfo block_row_info(const Geo& g, long long win, int r) {
  if (win >= g.n_win) return no_row();
  int b, wy, wx;
  window_coords(g, win, b, wy, wx);
  const int bh = kRows / g.ww;
  const int blk = r / kRows, rb = r - blk * kRows;
  const bool wrap_x = g.sw > 0 && wx == g.nWx - 1;
  const int w0 = wrap_x ? g.ww - g.sw : g.ww;
  const int xseg = rb >= bh * w0;
  const int rr = xseg ? rb - bh * w0 : rb;
  const int wseg = xseg ? g.ww - w0 : w0;
  const int iy = blk * bh + rr / wseg;
  const int ix = (xseg ? w0 : 0) + (rr - (rr / wseg) * wseg);
  return row_info_at(g, b, wy, wx, iy, ix);
}

// Packed per-key info: low 16 bits key offset into the bias table, bits 16-19
// region label, or 15 for a pad key (never equal to a query's label).
__device__ inline uint32_t key_word(const RowInfo& ri) {
  return (uint32_t)ri.key_off | ((uint32_t)(ri.valid ? ri.label : 15) << 16);
}

// Producer: one elected thread issues every TMA copy of tile `t` into `stage`.
template <int HD, int NTEN>
__device__ inline void issue_tile_loads(const FastParams& p, long long t, uint8_t* tiles,
                                        float* bias_dst, uint64_t* full) {
  const Geo& g = p.g;
  const int G = kRows / g.N;
  const long long group = t / g.heads;
  const int h = (int)(t - group * g.heads);
  using T = TileGeom<HD>;
  constexpr uint32_t row_bytes = T::kRowBytes;
  constexpr uint32_t tile_bytes = kRows * HD * 2;
  for (int gw = 0; gw < G; ++gw) {
    const long long win = group * G + gw;
    const uint32_t row0 = gw * g.N;
    if (win < g.n_win) {
      int b, wy, wx;
      window_coords(g, win, b, wy, wx);
      SubBox sb[4];
      const int n = plan_window(g, wy, wx, sb);
      for (int i = 0; i < n; ++i)
        for (int tt = 0; tt < NTEN; ++tt)
          for (int hf = 0; hf < T::kHalves; ++hf)
            tma_load_5d(tiles + tt * tile_bytes + hf * T::kHalfBytes +
                            (row0 + sb[i].row_off) * row_bytes,
                        &p.maps[tt][sb[i].map_id], full, hf * T::kBoxEl, h, sb[i].x, sb[i].y, b);
    } else {
      // No such window: a box wholly above the grid reads zeros and keeps the
      // transaction count uniform.
      for (int tt = 0; tt < NTEN; ++tt)
        for (int hf = 0; hf < T::kHalves; ++hf)
          tma_load_5d(tiles + tt * tile_bytes + hf * T::kHalfBytes + row0 * row_bytes,
                      &p.maps[tt][0], full, hf * T::kBoxEl, h, 0, -g.wh, 0);
    }
  }
  if (bias_dst) bulk_load(bias_dst, p.bias_t + (size_t)h * p.bins_pad, p.bins_pad * 4, full);
}

// K-major operand, rows of HD bf16 (128-byte swizzle for HD >= 64, 64-byte for
// 32), advanced by k16 steps of 16 elements along K; with two channel
// regions (HD = 128) steps 4-7 move to the second region.
template <int HD>
__device__ inline uint64_t desc_kmajor_tile(uint32_t base, int k16) {
  using T = TileGeom<HD>;
  constexpr uint32_t sw = HD >= 64 ? kSwizzle128 : kSwizzle64;
  return smem_desc(base + (k16 / T::kStepsPerHalf) * T::kHalfBytes +
                       (k16 % T::kStepsPerHalf) * 32,
                   16, 8 * T::kRowBytes, sw);
}
// MN-major operand (the HD columns are N), K = tile rows, 16 rows per step;
// with two channel regions (HD = 128) the second 64 columns of N are the next
// region, one leading byte offset away.
template <int HD>
__device__ inline uint64_t desc_mnmajor_tile(uint32_t base, int k16) {
  using T = TileGeom<HD>;
  constexpr uint32_t sw = HD >= 64 ? kSwizzle128 : kSwizzle64;
  return smem_desc(base + k16 * 16 * T::kRowBytes,
                   T::kHalves > 1 ? T::kHalfBytes : 8 * T::kRowBytes, 8 * T::kRowBytes, sw);
}
// P / dS tile: 128 rows x 128 columns bf16 as two 16 KB regions of 64 columns,
// 128-byte swizzle. As K-major A (M = rows, K = columns):
__device__ inline uint64_t desc_p_kmajor(uint32_t base, int k16) {
  return smem_desc(base + (k16 >> 2) * 16384 + (k16 & 3) * 32, 16, 1024, kSwizzle128);
}

// Writes this thread's row of a P-style tile: columns [col0, col0 + NCOL) from
// `vals` (already scaled), rounded to bf16, 128-byte swizzled.
template <int NCOL>
__device__ inline void store_p_row(uint32_t base, int row, int col0, const float* vals) {
#pragma unroll
  for (int c = 0; c < NCOL / 8; ++c) {
    const int col = col0 + c * 8;
    const uint32_t addr = base + (col >> 6) * 16384 + row * 128 + ((((col >> 3) & 7) ^ (row & 7)) << 4);
    st_shared_v4(addr, pack_bf16(vals[c * 8 + 0], vals[c * 8 + 1]),
                 pack_bf16(vals[c * 8 + 2], vals[c * 8 + 3]),
                 pack_bf16(vals[c * 8 + 4], vals[c * 8 + 5]),
                 pack_bf16(vals[c * 8 + 6], vals[c * 8 + 7]));
  }
}

template <int HD>
__device__ inline void store_row_bf16(void* dst, const float* v, float mul) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < HD / 8; ++c)
    st_global_v4(d + c, pack_bf16(v[c * 8 + 0] * mul, v[c * 8 + 1] * mul),
                 pack_bf16(v[c * 8 + 2] * mul, v[c * 8 + 3] * mul),
                 pack_bf16(v[c * 8 + 4] * mul, v[c * 8 + 5] * mul),
                 pack_bf16(v[c * 8 + 6] * mul, v[c * 8 + 7] * mul));
}

// NCH chunks of 16 bytes of this lane's row, from NCH * 8 values times `mul`,
// rounded to bf16.
template <int NCH>
__device__ inline void pack_chunks(const float* v, float mul, uint4 (&a)[NCH]) {
#pragma unroll
  for (int c = 0; c < NCH; ++c)
    a[c] = make_uint4(pack_bf16(v[c * 8 + 0] * mul, v[c * 8 + 1] * mul),
                      pack_bf16(v[c * 8 + 2] * mul, v[c * 8 + 3] * mul),
                      pack_bf16(v[c * 8 + 4] * mul, v[c * 8 + 5] * mul),
                      pack_bf16(v[c * 8 + 6] * mul, v[c * 8 + 7] * mul));
}

// Warp-collective: the warp's 32 rows (one per lane, NCH chunks of 16 bytes
// each, `dst` = this lane's row or nullptr for a row that is not stored) go
// to global memory so that every store instruction writes whole rows. Lanes
// hold rows and a row's chunks are contiguous in memory, so a plain store
// per chunk would touch 32 separate rows per instruction. Instead, an
// NCH x NCH transpose of the chunks inside each group of NCH lanes (log2 NCH
// butterfly steps of shuffles) leaves lane g*NCH + c with chunk c of the
// group's rows g*NCH + t, t = 0..NCH-1, and each of the NCH stores writes
// 32 / NCH whole rows.
template <int NCH>
__device__ inline void store_rows_coalesced(uint4 (&a)[NCH], const void* dst) {
  const int lane = threadIdx.x & 31;
  const int p = lane & (NCH - 1);
#pragma unroll
  for (int d = NCH / 2; d >= 1; d >>= 1) {
    const bool hi = (p & d) != 0;
#pragma unroll
    for (int q = 0; q < NCH; ++q) {
      if (q & d) continue;   // the pair of positions (q, q + d)
      uint4 v = hi ? a[q] : a[q + d];   // the position whose bit differs from the lane's
      v.x = __shfl_xor_sync(0xffffffffu, v.x, d);
      v.y = __shfl_xor_sync(0xffffffffu, v.y, d);
      v.z = __shfl_xor_sync(0xffffffffu, v.z, d);
      v.w = __shfl_xor_sync(0xffffffffu, v.w, d);
      if (hi) a[q] = v; else a[q + d] = v;
    }
  }
  const int g0 = lane & ~(NCH - 1);
#pragma unroll
  for (int t = 0; t < NCH; ++t) {
    const unsigned long long rp =
        __shfl_sync(0xffffffffu, (unsigned long long)dst, g0 + t);
    if (rp) st_global_v4(reinterpret_cast<uint4*>(rp) + p, a[t].x, a[t].y, a[t].z, a[t].w);
  }
}

// Warp-collective: rows of OC values (OC = 32 or 64, times `mul`) of the
// warp's 32 lanes, coalesced as above.
template <int OC>
__device__ inline void store_rows_bf16(const float* v, float mul, const void* dst) {
  uint4 a[OC / 8];
  pack_chunks<OC / 8>(v, mul, a);
  store_rows_coalesced<OC / 8>(a, dst);
}

// Warp-collective (.sync.aligned): every lane of the warp must reach it.
template <int NCOL>
__device__ inline void tmem_load_cols(uint32_t taddr, float* v) {
  __syncwarp();
#pragma unroll
  for (int c = 0; c < NCOL / 32; ++c) tmem_ld32(taddr + c * 32, v + c * 32);
}

// ================================================================================
// Per-row softmax pieces of the warpgroup
// ================================================================================
// A window is "plain" when it does not straddle the wrap seam and holds no pad
// token: one TMA box, slots in row-major order, a single shift region, all keys
// real. For 8 x 8 windows its key offsets into the bias table are compile-time
// constants, so no per-key word is read and no mask is applied.
template <int WW>
__host__ __device__ constexpr int plain_off(int j) {
  return (j / WW) * (2 * WW - 1) + (j % WW);
}

__device__ inline bool window_plain(const Geo& g, long long win) {
  if (win >= g.n_win) return false;
  int b, wy, wx;
  window_coords(g, win, b, wy, wx);
  if (g.sh > 0 && wy == g.nWy - 1) return false;
  if (g.sw > 0 && wx == g.nWx - 1) return false;
  return wy * g.wh + g.sh + g.wh <= g.Hv && wx * g.ww + g.sw + g.ww <= g.Wv;
}

template <int WW>
__device__ inline RowInfo plain_row_info(const Geo& g, long long win, int r) {
  int b, wy, wx;
  window_coords(g, win, b, wy, wx);
  const int iy = r / (WW > 0 ? WW : 1), ix = r % (WW > 0 ? WW : 1);
  RowInfo ri;
  ri.valid = true;
  ri.stored = true;
  ri.halo = false;
  ri.label = 0;
  ri.bias_base = (iy + WW - 1) * (2 * WW - 1) + ix + WW - 1;
  ri.key_off = iy * (2 * WW - 1) + ix;
  ri.token = ((long long)b * g.H + wy * WW + g.sh + iy) * g.W + wx * WW + g.sw + ix;
  return ri;
}

// Logits in log2 units, x <- scale*log2(e)*s + bias (bias pre-scaled), for
// the N keys of a plain window; returns the row maximum.
// (Pairs of keys go through the packed fp32x2 FMA: the same rounding per
// element, half the instructions.)
template <int N, int WW>
__device__ inline float logits_plain(float* x, const float* bias_q, float c) {
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int j = 0; j < N; j += 4) {
    const float2 a = __ffma2_rn(make_float2(x[j], x[j + 1]), c2,
                                make_float2(bias_q[-plain_off<WW>(j + 0)],
                                            bias_q[-plain_off<WW>(j + 1)]));
    const float2 b = __ffma2_rn(make_float2(x[j + 2], x[j + 3]), c2,
                                make_float2(bias_q[-plain_off<WW>(j + 2)],
                                            bias_q[-plain_off<WW>(j + 3)]));
    x[j + 0] = a.x;
    x[j + 1] = a.y;
    x[j + 2] = b.x;
    x[j + 3] = b.y;
    m0 = fmaxf(m0, a.x);
    m1 = fmaxf(m1, a.y);
    m2 = fmaxf(m2, b.x);
    m3 = fmaxf(m3, b.y);
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// Same for any window: per-key words give the bias offset and the shift region
// (15 = pad key); keys of another region or pad keys get -inf.
template <int N>
__device__ inline float logits_general(float* x, const float* brow, const uint32_t* cw, int base,
                                       int label, float c) {
  float mm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int j0 = 0; j0 < N; j0 += 8) {
#pragma unroll
    for (int j = j0; j < j0 + 8; ++j) {
      const uint32_t w = cw[j];
      const bool ok = (int)(w >> 16) == label;
      x[j] = ok ? fmaf(x[j], c, brow[base - (int)(w & 0xFFFF)]) : -INFINITY;
      mm[j & 3] = fmaxf(mm[j & 3], x[j]);
    }
    asm volatile("" ::: "memory");   // bound the loads in flight (registers)
  }
  return fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3]));
}

// x <- 2^(x - m); returns the sum.
// (Four partial sums over keys j mod 4, as two packed pairs.)
template <int N>
__device__ inline float exp_sum(float* x, float m) {
  float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
  const float2 nm = make_float2(-m, -m);
#pragma unroll
  for (int j = 0; j < N; j += 4) {
    const float2 ta = __fadd2_rn(make_float2(x[j], x[j + 1]), nm);
    const float2 tb = __fadd2_rn(make_float2(x[j + 2], x[j + 3]), nm);
    x[j] = ex2(ta.x);
    x[j + 1] = ex2(ta.y);
    x[j + 2] = ex2(tb.x);
    x[j + 3] = ex2(tb.y);
    la = __fadd2_rn(la, make_float2(x[j], x[j + 1]));
    lb = __fadd2_rn(lb, make_float2(x[j + 2], x[j + 3]));
  }
  return (la.x + la.y) + (lb.x + lb.y);
}

__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Number of tiles CTA `cta` takes in a grid of `grid` CTAs.
__device__ inline long long local_tiles(long long n_tiles, long long cta, long long grid) {
  return cta < n_tiles ? (n_tiles - 1 - cta) / grid + 1 : 0;
}
// ================================================================================
// Host side
// ================================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

int box_len(int kind, int w, int s) { return kind == 0 ? w : (kind == 1 ? w - s : s); }

// The 5-D map [hd, heads, W, rows, B] of one tensor with box [hd, 1, bx, by, 1].
bool encode_map(CUtensorMap* m, const void* base, const Geo& g, int rows, int by, int bx) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[5] = {(cuuint64_t)g.hd, (cuuint64_t)g.heads, (cuuint64_t)g.W,
                              (cuuint64_t)rows, (cuuint64_t)g.B};
  const cuuint64_t es = 2;
  const cuuint64_t strides[4] = {g.hd * es, (cuuint64_t)g.heads * g.hd * es,
                                 (cuuint64_t)g.W * g.heads * g.hd * es,
                                 (cuuint64_t)rows * g.W * g.heads * g.hd * es};
  // at most 64 channels (128 bytes) per box: head_dim 128 is two boxes
  const cuuint32_t box[5] = {(cuuint32_t)(g.hd > 64 ? 64 : g.hd), 1, (cuuint32_t)bx,
                             (cuuint32_t)by, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapSwizzle sw =
      g.hd >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The nine box shapes of one tensor into dst[0..8]. The wrapped row part
// (ky = 2: source rows 0 .. sh-1) reads `halo` ([B, sh, W, heads, hd]) in a
// row band, the tensor itself otherwise.
bool encode_map_set(CUtensorMap* dst, const void* base, const void* halo, const Geo& g) {
  for (int ky = 0; ky < 3; ++ky)
    for (int kx = 0; kx < 3; ++kx) {
      int by = box_len(ky, g.wh, g.sh), bx = box_len(kx, g.ww, g.sw);
      if (by <= 0) by = g.wh;  // shape unused when the axis has no shift
      if (bx <= 0) bx = g.ww;
      const bool from_halo = g.band && ky == 2 && g.sh > 0;
      if (!encode_map(&dst[ky * 3 + kx], from_halo ? halo : base, g, from_halo ? g.sh : g.H, by,
                      bx))
        return false;
    }
  return true;
}
bool encode_maps(FastParams& p, int which, const void* base, const void* halo = nullptr) {
  return encode_map_set(p.maps[which], base, halo, p.g);
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

constexpr size_t kSmemLimit = 227 * 1024;


void fill_common(FastParams& p, const Geo& g, const float* bias_t, int* status, int flags) {
  memset(&p, 0, sizeof(p));
  p.g = g;
  const int G = g.N <= kRows ? kRows / g.N : 1;   // windows per 128-row tile
  p.n_groups = (g.n_win + G - 1) / G;
  p.n_tiles = p.n_groups * g.heads;
  p.bins_pad = bins_padded(g.bins);
  p.scale_log2 = kLog2e / sqrtf((float)g.hd);
  p.bias_t = bias_t;
  p.status = status;
  p.test_timeout = (flags & SWIN_FLAG_TEST_TIMEOUT) ? 1 : 0;
}

template <typename K>
cudaError_t launch(K kernel, const FastParams& p, size_t smem, cudaStream_t st,
                   int threads = kThreads) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = p.n_tiles < num_sms() ? p.n_tiles : num_sms();
  kernel<<<(unsigned)(grid > 0 ? grid : 1), threads, smem, st>>>(p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace
}  // namespace swin
