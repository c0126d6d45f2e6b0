// geometry.cuh -- where every window slot of the padded, shifted grid comes from.
//
// Layout stage of shifted-window attention (TERRA page, Abstract: window-based
// Swin attention with "shifted-window execution"; Table I: H, W the grid,
// H^, W^ its padded size). Nothing is ever copied into the padded, rolled or
// windowed order: these functions give, for window (b, wy, wx) and slot
// (iy, ix), the grid token it reads, whether that token is real or padding, and
// its shift region. The kernels turn the same arithmetic into TMA box
// coordinates (fast path) or per-token addresses (portable path).
#pragma once
#include <stdint.h>

#include "../../include/swin_wattn.h"

namespace swin {

struct Geo {
  int B, H, W, wh, ww, sh, sw, heads, hd;
  int Hv, Wv;               // valid extent: tokens at y >= Hv or x >= Wv are padding
  int Hp, Wp, nWy, nWx, N;  // padded grid, windows per axis, tokens per window
  long long n_win;          // B * nWy * nWx
  int bins;                 // (2 wh - 1) (2 ww - 1)
  // Row band of a larger grid (tcgen05 kernels only): the rows the shift
  // wraps to (source rows 0 .. sh-1 of the last window row) live in a
  // separate halo tensor [B, sh, W, heads, hd] (the next band's first rows),
  // and their outputs go to a halo output tensor of that shape.
  int band;
  int seam_h;               // shift of the row shift-region split (0: none; sh otherwise)
};

inline Geo make_geo(const swin_wattn_desc& d) {
  Geo g;
  g.B = d.B; g.H = d.H; g.W = d.W; g.wh = d.win_h; g.ww = d.win_w;
  g.sh = d.shift_h; g.sw = d.shift_w; g.heads = d.heads; g.hd = d.head_dim;
  g.Hv = d.valid_h > 0 ? d.valid_h : d.H;
  g.Wv = d.valid_w > 0 ? d.valid_w : d.W;
  g.Hp = (d.H + d.win_h - 1) / d.win_h * d.win_h;
  g.Wp = (d.W + d.win_w - 1) / d.win_w * d.win_w;
  g.nWy = g.Hp / d.win_h;
  g.nWx = g.Wp / d.win_w;
  g.N = d.win_h * d.win_w;
  g.n_win = (long long)d.B * g.nWy * g.nWx;
  g.bins = (2 * d.win_h - 1) * (2 * d.win_w - 1);
  g.band = 0;
  g.seam_h = d.shift_h;
  return g;
}

// Shift region of a rolled coordinate t on an axis of padded length n, window w,
// shift s: 0 below n-w (and everywhere when s = 0), 1 on [n-w, n-s), 2 on [n-s, n).
__host__ __device__ inline int region_1d(int t, int n, int w, int s) {
  if (s == 0 || t < n - w) return 0;
  return t < n - s ? 1 : 2;
}

struct SlotInfo {
  int b, y, x;     // source grid position (y < Hp, x < Wp)
  int iy, ix;      // slot coordinates inside the window
  int label;       // 3 * row region + column region
  bool valid;      // a real token: y < Hv and x < Wv
  bool stored;     // in the tensor: y < H and x < W (outputs are written)
};

// Window `win` (flattened over b, wy, wx) and slot -> source token. Rolled
// position (yr, xr) = (wy*wh + iy, wx*ww + ix) holds padded position
// ((yr + sh) mod Hp, (xr + sw) mod Wp).
__host__ __device__ inline SlotInfo slot_info(const Geo& g, long long win, int slot) {
  SlotInfo s;
  const long long per_b = (long long)g.nWy * g.nWx;
  s.b = (int)(win / per_b);
  const int r = (int)(win - (long long)s.b * per_b);
  const int wy = r / g.nWx, wx = r - wy * g.nWx;
  s.iy = slot / g.ww;
  s.ix = slot - s.iy * g.ww;
  const int yr = wy * g.wh + s.iy, xr = wx * g.ww + s.ix;
  s.y = (yr + g.sh) % g.Hp;
  s.x = (xr + g.sw) % g.Wp;
  s.stored = s.y < g.H && s.x < g.W;
  s.valid = s.y < g.Hv && s.x < g.Wv;
  s.label = 3 * region_1d(yr, g.Hp, g.wh, g.seam_h) + region_1d(xr, g.Wp, g.ww, g.sw);
  return s;
}

// Linear token index (b*H + y)*W + x of a stored slot.
__host__ __device__ inline long long token_of(const Geo& g, const SlotInfo& s) {
  return ((long long)s.b * g.H + s.y) * g.W + s.x;
}

// Relative-position bias index for query slot (iy, ix) and key slot (jy, jx).
__host__ __device__ inline int rel_index(const Geo& g, int iy, int ix, int jy, int jx) {
  return (iy - jy + g.wh - 1) * (2 * g.ww - 1) + (ix - jx + g.ww - 1);
}

}  // namespace swin
