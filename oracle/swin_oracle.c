/*
 * swin_oracle.c -- plain, slow, fp64 CPU oracle for shifted-window multi-head
 * self-attention (SW-MSA) over a padded token grid, forward and backward.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark load this library. The GPU library never
 * links, loads or calls it; the two share no source, header, table or helper.
 *
 * What it follows. Page "TERRA: A Hierarchical Parallel Training and Memory
 * Orchestration Framework for High-Resolution AI-based Earth Modeling":
 *   - Abstract: window-based Swin Transformers, "shifted-window execution",
 *     tokens routed into (ragged) window layouts for Transformer execution;
 *   - Table I (notation): H, W spatial resolution; H^, W^ the padded
 *     resolution.
 * The page prints no formula. The Abstract names the Swin Transformer, whose
 * published shifted-window attention (Liu et al., ICCV 2021) is taken as the
 * definition, written out step by step:
 *   1 pad the H x W grid at the bottom/right to H^ x W^ (multiples of the window)
 *   2 cyclic shift: rolled (y', x') holds padded ((y'+s_h) mod H^, (x'+s_w) mod W^)
 *   3 window partition of the rolled grid; region labels of the shift mask
 *   4 per window and head: a = scale*q.k + T[rel(i,j)] on allowed pairs,
 *     softmax over allowed keys, o = P v
 *   5 window reverse, 6 reverse shift, 7 crop back to H x W.
 * Readings taken where the pages are silent (scale = head_dim^-1/2; relative
 * offset = query slot minus key slot; regions on the rolled, padded grid;
 * masked pairs get weight exactly 0; pad keys masked; pad queries produce and
 * receive nothing) are stated next to the step that uses them.
 *
 * Arithmetic is fp64 throughout; every input and output array is fp64 (bf16
 * and fp32 inputs widen exactly).
 * Layouts: q, k, v, dout, out, dq, dk, dv are [B, H, W, heads, head_dim];
 * lse is [B, H, W, heads]; table and dtable are [(2*win_h-1)*(2*win_w-1), heads].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t B, H, W;
  int32_t win_h, win_w;
  int32_t shift_h, shift_w;
  int32_t heads, head_dim;
  int32_t valid_h, valid_w; /* valid extent of the stored grid; 0 = H (or W) */
} swin_oracle_shape;

enum { ORACLE_OK = 0, ORACLE_BAD_SHAPE = -1, ORACLE_NO_MEMORY = -2, ORACLE_EMPTY_ROW = -3 };

static int64_t round_up(int64_t n, int64_t w) { return (n + w - 1) / w * w; }

static int shape_ok(const swin_oracle_shape* s) {
  if (s->B < 0 || s->H < 0 || s->W < 0) return 0;
  if (s->valid_h < 0 || s->valid_h > s->H || s->valid_w < 0 || s->valid_w > s->W) return 0;
  if (s->win_h < 1 || s->win_w < 1 || s->heads < 1 || s->head_dim < 1) return 0;
  if (s->shift_h < 0 || s->shift_h >= s->win_h) return 0;
  if (s->shift_w < 0 || s->shift_w >= s->win_w) return 0;
  return 1;
}

/* Valid extent of the token grid: the tokens that carry field data. Table I
 * pads the physical field itself (H x W to H^ x W^ pixels) before patching,
 * so a stored token can cover only padded pixels. Reading: a token is real
 * when its patch holds at least one real pixel, i.e. the caller passes
 * valid_h = ceil(field rows / patch) (and likewise for columns); tokens at or
 * beyond the valid extent are treated exactly like the pad tokens of step 1.
 * 0 means the whole stored grid is valid. */
static int64_t valid_rows(const swin_oracle_shape* s) { return s->valid_h ? s->valid_h : s->H; }
static int64_t valid_cols(const swin_oracle_shape* s) { return s->valid_w ? s->valid_w : s->W; }

/* ---- Step 1: padding (Table I, H^ x W^) -------------------------------------
 * Reading: pad at the bottom and right, to the smallest multiple of the window;
 * pad values are zero and pad tokens are flagged invalid, as are stored tokens
 * outside the valid extent. One (batch, head) channel slice [H, W, hd] of the
 * [B, H, W, heads, hd] tensor is copied. */
static void step1_pad(const swin_oracle_shape* s, const double* x, int64_t b, int64_t h,
                      int64_t Hp, int64_t Wp, double* xp, unsigned char* valid) {
  const int64_t hd = s->head_dim, C = (int64_t)s->heads * hd;
  const int64_t Hv = valid_rows(s), Wv = valid_cols(s);
  for (int64_t y = 0; y < Hp; ++y)
    for (int64_t xx = 0; xx < Wp; ++xx) {
      const int inside = (y < s->H) && (xx < s->W);
      if (valid) valid[y * Wp + xx] = (unsigned char)((y < Hv) && (xx < Wv));
      for (int64_t e = 0; e < hd; ++e)
        xp[(y * Wp + xx) * hd + e] =
            inside ? x[((b * s->H + y) * s->W + xx) * C + h * hd + e] : 0.0;
    }
}

/* ---- Step 2 and Step 6: cyclic shift and its inverse (Abstract,
 * "shifted-window execution") --------------------------------------------------
 * Reading: the grid content moves up/left by s before partition, so the rolled
 * position (y', x') holds the padded position ((y'+s_h) mod H^, (x'+s_w) mod W^);
 * the inverse puts it back. Elements are `elem` bytes each. */
static void step2_roll(const void* src, void* dst, int64_t Hp, int64_t Wp, size_t elem,
                       int64_t sh, int64_t sw) {
  const unsigned char* a = (const unsigned char*)src;
  unsigned char* d = (unsigned char*)dst;
  for (int64_t yr = 0; yr < Hp; ++yr)
    for (int64_t xr = 0; xr < Wp; ++xr) {
      const int64_t ys = (yr + sh) % Hp, xs = (xr + sw) % Wp;
      memcpy(d + (size_t)(yr * Wp + xr) * elem, a + (size_t)(ys * Wp + xs) * elem, elem);
    }
}

static void step6_unroll(const void* src, void* dst, int64_t Hp, int64_t Wp, size_t elem,
                         int64_t sh, int64_t sw) {
  const unsigned char* a = (const unsigned char*)src;
  unsigned char* d = (unsigned char*)dst;
  for (int64_t yr = 0; yr < Hp; ++yr)
    for (int64_t xr = 0; xr < Wp; ++xr) {
      const int64_t ys = (yr + sh) % Hp, xs = (xr + sw) % Wp;
      memcpy(d + (size_t)(ys * Wp + xs) * elem, a + (size_t)(yr * Wp + xr) * elem, elem);
    }
}

/* ---- Step 3: window partition, and Step 5: window reverse (Abstract,
 * "window-based Swin Transformers") ---------------------------------------------
 * Window (wy, wx) of the rolled grid holds rolled rows wy*win_h .. +win_h-1 and
 * columns wx*win_w .. +win_w-1; slot i = iy*win_w + ix. Windows are numbered
 * wy*(W^/win_w) + wx. */
static void step3_partition(const void* src, void* dst, int64_t Hp, int64_t Wp, int64_t wh,
                            int64_t ww, size_t elem) {
  const unsigned char* a = (const unsigned char*)src;
  unsigned char* d = (unsigned char*)dst;
  const int64_t nWy = Hp / wh, nWx = Wp / ww, N = wh * ww;
  for (int64_t wy = 0; wy < nWy; ++wy)
    for (int64_t wx = 0; wx < nWx; ++wx)
      for (int64_t iy = 0; iy < wh; ++iy)
        for (int64_t ix = 0; ix < ww; ++ix) {
          const int64_t win = wy * nWx + wx, slot = iy * ww + ix;
          const int64_t yr = wy * wh + iy, xr = wx * ww + ix;
          memcpy(d + (size_t)(win * N + slot) * elem, a + (size_t)(yr * Wp + xr) * elem, elem);
        }
}

static void step5_reverse(const void* src, void* dst, int64_t Hp, int64_t Wp, int64_t wh,
                          int64_t ww, size_t elem) {
  const unsigned char* a = (const unsigned char*)src;
  unsigned char* d = (unsigned char*)dst;
  const int64_t nWy = Hp / wh, nWx = Wp / ww, N = wh * ww;
  for (int64_t wy = 0; wy < nWy; ++wy)
    for (int64_t wx = 0; wx < nWx; ++wx)
      for (int64_t iy = 0; iy < wh; ++iy)
        for (int64_t ix = 0; ix < ww; ++ix) {
          const int64_t win = wy * nWx + wx, slot = iy * ww + ix;
          const int64_t yr = wy * wh + iy, xr = wx * ww + ix;
          memcpy(d + (size_t)(yr * Wp + xr) * elem, a + (size_t)(win * N + slot) * elem, elem);
        }
}

/* ---- Step 3b: shift-mask regions ---------------------------------------------
 * Reading (Swin 2021): on the rolled, padded grid each axis splits into
 * [0, n-w), [n-w, n-s), [n-s, n) when s > 0 (one region when s = 0); the label
 * is 3*r_row + r_col. Two tokens of one window may attend to each other only if
 * their labels agree: a window on the wrap seam holds tokens that were far
 * apart before the roll. */
static int32_t region_1d(int64_t t, int64_t n, int64_t w, int64_t s) {
  if (s == 0 || t < n - w) return 0;
  return t < n - s ? 1 : 2;
}

static void step3_region_labels(int64_t Hp, int64_t Wp, const swin_oracle_shape* s,
                                int32_t* label) {
  for (int64_t yr = 0; yr < Hp; ++yr)
    for (int64_t xr = 0; xr < Wp; ++xr)
      label[yr * Wp + xr] = 3 * region_1d(yr, Hp, s->win_h, s->shift_h) +
                            region_1d(xr, Wp, s->win_w, s->shift_w);
}

/* Relative-position bias index (Swin 2021 reading): offset = query slot minus
 * key slot, shifted to be non-negative, row-major over (2w_h-1) x (2w_w-1). */
static int64_t rel_index(const swin_oracle_shape* s, int64_t i, int64_t j) {
  const int64_t iy = i / s->win_w, ix = i % s->win_w, jy = j / s->win_w, jx = j % s->win_w;
  return (iy - jy + s->win_h - 1) * (2 * s->win_w - 1) + (ix - jx + s->win_w - 1);
}

/* ---- Step 4: attention of one window and one head ------------------------------
 * a_ij = scale * q_i.k_j + T[rel(i,j), h] for allowed j (key valid and same
 * region label as the query); P_ij = exp(a_ij - m_i) / sum over allowed keys,
 * P_ij = 0 otherwise; o_i = sum_j P_ij v_j; lse_i = m_i + log(sum). Pad queries
 * (invalid i) are skipped: their rows are dropped by the crop. Returns the
 * softmax rows in P (N x N) for the backward. */
static int step4_window_attention(const swin_oracle_shape* s, int64_t h, const double* T,
                                  const double* qw, const double* kw, const double* vw,
                                  const unsigned char* vld, const int32_t* lab, double* ow,
                                  double* lsew, double* P) {
  const int64_t N = (int64_t)s->win_h * s->win_w, hd = s->head_dim;
  const double scale = 1.0 / sqrt((double)hd);
  for (int64_t i = 0; i < N; ++i) {
    double* Pi = P + i * N;
    for (int64_t j = 0; j < N; ++j) Pi[j] = 0.0;
    for (int64_t e = 0; e < hd; ++e) ow[i * hd + e] = 0.0;
    lsew[i] = 0.0;
    if (!vld[i]) continue;
    double m = -INFINITY;
    for (int64_t j = 0; j < N; ++j) {
      if (!vld[j] || lab[j] != lab[i]) continue;
      double dot = 0.0;
      for (int64_t e = 0; e < hd; ++e) dot += qw[i * hd + e] * kw[j * hd + e];
      Pi[j] = scale * dot + T[rel_index(s, i, j) * s->heads + h];
      if (Pi[j] > m) m = Pi[j];
    }
    if (!(m > -INFINITY)) return ORACLE_EMPTY_ROW; /* impossible: key i == query i is allowed */
    double l = 0.0;
    for (int64_t j = 0; j < N; ++j) {
      if (!vld[j] || lab[j] != lab[i]) continue;
      Pi[j] = exp(Pi[j] - m);
      l += Pi[j];
    }
    for (int64_t j = 0; j < N; ++j) {
      if (!vld[j] || lab[j] != lab[i]) continue;
      Pi[j] /= l;
      for (int64_t e = 0; e < hd; ++e) ow[i * hd + e] += Pi[j] * vw[j * hd + e];
    }
    lsew[i] = m + log(l);
  }
  return ORACLE_OK;
}

/* ---- Backward of step 4 for one window and one head --------------------------
 * With dO given: dP_ij = dO_i.v_j, D_i = sum_j P_ij dP_ij,
 * dS_ij = P_ij (dP_ij - D_i); dq_i = scale sum_j dS_ij k_j,
 * dk_j = scale sum_i dS_ij q_i, dv_j = sum_i P_ij dO_i, and
 * dT[rel(i,j), h] += dS_ij. Pad queries contribute nothing. */
static void step4_window_attention_backward(const swin_oracle_shape* s, const double* qw,
                                            const double* kw, const double* vw,
                                            const double* dow, const unsigned char* vld,
                                            const int32_t* lab, const double* P, double* dqw,
                                            double* dkw, double* dvw, double* dT_bins) {
  const int64_t N = (int64_t)s->win_h * s->win_w, hd = s->head_dim;
  const double scale = 1.0 / sqrt((double)hd);
  for (int64_t t = 0; t < N * hd; ++t) dqw[t] = dkw[t] = dvw[t] = 0.0;
  for (int64_t i = 0; i < N; ++i) {
    if (!vld[i]) continue;
    const double* Pi = P + i * N;
    double D = 0.0;
    for (int64_t j = 0; j < N; ++j) {
      if (!vld[j] || lab[j] != lab[i]) continue;
      double dp = 0.0;
      for (int64_t e = 0; e < hd; ++e) dp += dow[i * hd + e] * vw[j * hd + e];
      D += Pi[j] * dp;
    }
    for (int64_t j = 0; j < N; ++j) {
      if (!vld[j] || lab[j] != lab[i]) continue;
      double dp = 0.0;
      for (int64_t e = 0; e < hd; ++e) dp += dow[i * hd + e] * vw[j * hd + e];
      const double dS = Pi[j] * (dp - D);
      for (int64_t e = 0; e < hd; ++e) {
        dqw[i * hd + e] += scale * dS * kw[j * hd + e];
        dkw[j * hd + e] += scale * dS * qw[i * hd + e];
        dvw[j * hd + e] += Pi[j] * dow[i * hd + e];
      }
      dT_bins[rel_index(s, i, j)] += dS;
    }
  }
}

/* ---- Step 7: crop (inverse of step 1) -----------------------------------------
 * Writes the [H^, W^, width] padded slice back into channel h of a
 * [B, H, W, heads, width] tensor, dropping pad positions. Stored tokens
 * outside the valid extent receive the zeros step 4 leaves for them. */
static void step7_crop(const swin_oracle_shape* s, const double* xp, int64_t b, int64_t h,
                       int64_t Hp, int64_t Wp, int64_t width, double* out) {
  (void)Hp;
  const int64_t C = (int64_t)s->heads * width;
  for (int64_t y = 0; y < s->H; ++y)
    for (int64_t x = 0; x < s->W; ++x)
      for (int64_t e = 0; e < width; ++e)
        out[((b * s->H + y) * s->W + x) * C + h * width + e] = xp[(y * Wp + x) * width + e];
}

/* Layout of one (batch, head) slice through steps 1-3: padded, rolled, windowed. */
typedef struct {
  int64_t Hp, Wp, N, nwin, hd;
  double *tmp_a, *tmp_b;        /* [H^ W^ hd] scratch */
  unsigned char *valid_p, *valid_r, *valid_w;
  int32_t *label_r, *label_w;
} slice_layout;

static void free_layout(slice_layout* L) {
  free(L->tmp_a); free(L->tmp_b); free(L->valid_p); free(L->valid_r); free(L->valid_w);
  free(L->label_r); free(L->label_w);
}

static int make_layout(const swin_oracle_shape* s, slice_layout* L) {
  memset(L, 0, sizeof(*L));
  L->Hp = round_up(s->H, s->win_h);
  L->Wp = round_up(s->W, s->win_w);
  L->N = (int64_t)s->win_h * s->win_w;
  L->nwin = (L->Hp / s->win_h) * (L->Wp / s->win_w);
  L->hd = s->head_dim;
  const size_t cells = (size_t)(L->Hp * L->Wp);
  L->tmp_a = (double*)malloc(cells * L->hd * sizeof(double) + 8);
  L->tmp_b = (double*)malloc(cells * L->hd * sizeof(double) + 8);
  L->valid_p = (unsigned char*)malloc(cells + 1);
  L->valid_r = (unsigned char*)malloc(cells + 1);
  L->valid_w = (unsigned char*)malloc(cells + 1);
  L->label_r = (int32_t*)malloc(cells * sizeof(int32_t) + 4);
  L->label_w = (int32_t*)malloc(cells * sizeof(int32_t) + 4);
  if (!L->tmp_a || !L->tmp_b || !L->valid_p || !L->valid_r || !L->valid_w || !L->label_r ||
      !L->label_w) {
    free_layout(L);
    return ORACLE_NO_MEMORY;
  }
  return ORACLE_OK;
}

/* Steps 1-3 for one tensor slice: pad, roll, partition into `windowed`
 * ([nwin, N, hd]). Fills the validity and label windows when `with_masks`. */
static void layout_in(const swin_oracle_shape* s, slice_layout* L, const double* x, int64_t b,
                      int64_t h, double* windowed, int with_masks) {
  step1_pad(s, x, b, h, L->Hp, L->Wp, L->tmp_a, with_masks ? L->valid_p : NULL);
  step2_roll(L->tmp_a, L->tmp_b, L->Hp, L->Wp, sizeof(double) * L->hd, s->shift_h, s->shift_w);
  step3_partition(L->tmp_b, windowed, L->Hp, L->Wp, s->win_h, s->win_w, sizeof(double) * L->hd);
  if (with_masks) {
    step2_roll(L->valid_p, L->valid_r, L->Hp, L->Wp, 1, s->shift_h, s->shift_w);
    step3_partition(L->valid_r, L->valid_w, L->Hp, L->Wp, s->win_h, s->win_w, 1);
    step3_region_labels(L->Hp, L->Wp, s, L->label_r);
    step3_partition(L->label_r, L->label_w, L->Hp, L->Wp, s->win_h, s->win_w, sizeof(int32_t));
  }
}

/* Steps 5-7 for one output slice of `width` values per token. */
static void layout_out(const swin_oracle_shape* s, slice_layout* L, const double* windowed,
                       int64_t width, int64_t b, int64_t h, double* out) {
  step5_reverse(windowed, L->tmp_a, L->Hp, L->Wp, s->win_h, s->win_w, sizeof(double) * width);
  step6_unroll(L->tmp_a, L->tmp_b, L->Hp, L->Wp, sizeof(double) * width, s->shift_h,
               s->shift_w);
  step7_crop(s, L->tmp_b, b, h, L->Hp, L->Wp, width, out);
}

/* Forward over the whole problem. `lse` may be NULL. */
int swin_oracle_forward(const swin_oracle_shape* s, const double* q, const double* k,
                        const double* v, const double* table, double* out, double* lse) {
  if (!shape_ok(s)) return ORACLE_BAD_SHAPE;
  slice_layout L;
  if (make_layout(s, &L)) return ORACLE_NO_MEMORY;
  const int64_t N = L.N, hd = L.hd, nw = L.nwin;
  double* qw = (double*)malloc(sizeof(double) * nw * N * hd + 8);
  double* kw = (double*)malloc(sizeof(double) * nw * N * hd + 8);
  double* vw = (double*)malloc(sizeof(double) * nw * N * hd + 8);
  double* ow = (double*)malloc(sizeof(double) * nw * N * hd + 8);
  double* lw = (double*)malloc(sizeof(double) * nw * N + 8);
  int status = ORACLE_OK;
  if (!qw || !kw || !vw || !ow || !lw) status = ORACLE_NO_MEMORY;
  for (int64_t b = 0; b < s->B && status == ORACLE_OK; ++b)
    for (int64_t h = 0; h < s->heads && status == ORACLE_OK; ++h) {
      layout_in(s, &L, q, b, h, qw, 1);
      layout_in(s, &L, k, b, h, kw, 0);
      layout_in(s, &L, v, b, h, vw, 0);
      int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
      for (int64_t win = 0; win < nw; ++win) {
        double* P = (double*)malloc(sizeof(double) * N * N);
        if (!P) { bad |= 1; continue; }
        if (step4_window_attention(s, h, table, qw + win * N * hd, kw + win * N * hd,
                                   vw + win * N * hd, L.valid_w + win * N, L.label_w + win * N,
                                   ow + win * N * hd, lw + win * N, P))
          bad |= 2;
        free(P);
      }
      if (bad) { status = (bad & 1) ? ORACLE_NO_MEMORY : ORACLE_EMPTY_ROW; break; }
      layout_out(s, &L, ow, hd, b, h, out);
      if (lse) layout_out(s, &L, lw, 1, b, h, lse);
    }
  free(qw); free(kw); free(vw); free(ow); free(lw);
  free_layout(&L);
  return status;
}

/* Backward over the whole problem: dq, dk, dv and dtable (overwritten). The
 * forward softmax rows are recomputed window by window. dtable is summed in a
 * fixed order (windows in order, then batch and head), so it is deterministic. */
int swin_oracle_backward(const swin_oracle_shape* s, const double* q, const double* k,
                         const double* v, const double* table, const double* dout, double* dq,
                         double* dk, double* dv, double* dtable) {
  if (!shape_ok(s)) return ORACLE_BAD_SHAPE;
  slice_layout L;
  if (make_layout(s, &L)) return ORACLE_NO_MEMORY;
  const int64_t N = L.N, hd = L.hd, nw = L.nwin;
  const int64_t bins = (2 * (int64_t)s->win_h - 1) * (2 * (int64_t)s->win_w - 1);
  const size_t tile = sizeof(double) * nw * N * hd + 8;
  double *qw = (double*)malloc(tile), *kw = (double*)malloc(tile), *vw = (double*)malloc(tile);
  double *dow = (double*)malloc(tile), *dqw = (double*)malloc(tile);
  double *dkw = (double*)malloc(tile), *dvw = (double*)malloc(tile);
  double* bins_w = (double*)malloc(sizeof(double) * nw * bins + 8);
  int status = ORACLE_OK;
  if (!qw || !kw || !vw || !dow || !dqw || !dkw || !dvw || !bins_w) status = ORACLE_NO_MEMORY;
  for (int64_t t = 0; t < bins * s->heads; ++t) dtable[t] = 0.0;
  for (int64_t b = 0; b < s->B && status == ORACLE_OK; ++b)
    for (int64_t h = 0; h < s->heads && status == ORACLE_OK; ++h) {
      layout_in(s, &L, q, b, h, qw, 1);
      layout_in(s, &L, k, b, h, kw, 0);
      layout_in(s, &L, v, b, h, vw, 0);
      layout_in(s, &L, dout, b, h, dow, 0);
      int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
      for (int64_t win = 0; win < nw; ++win) {
        double* P = (double*)malloc(sizeof(double) * N * N);
        double* o_unused = (double*)malloc(sizeof(double) * N * hd);
        double* l_unused = (double*)malloc(sizeof(double) * N);
        if (!P || !o_unused || !l_unused) {
          bad |= 1;
        } else {
          const int64_t off = win * N * hd;
          if (step4_window_attention(s, h, table, qw + off, kw + off, vw + off,
                                     L.valid_w + win * N, L.label_w + win * N, o_unused,
                                     l_unused, P))
            bad |= 2;
          for (int64_t t = 0; t < bins; ++t) bins_w[win * bins + t] = 0.0;
          step4_window_attention_backward(s, qw + off, kw + off, vw + off, dow + off,
                                          L.valid_w + win * N, L.label_w + win * N, P,
                                          dqw + off, dkw + off,
                                          dvw + off, bins_w + win * bins);
        }
        free(P); free(o_unused); free(l_unused);
      }
      if (bad) { status = (bad & 1) ? ORACLE_NO_MEMORY : ORACLE_EMPTY_ROW; break; }
      for (int64_t win = 0; win < nw; ++win)
        for (int64_t t = 0; t < bins; ++t) dtable[t * s->heads + h] += bins_w[win * bins + t];
      layout_out(s, &L, dqw, hd, b, h, dq);
      layout_out(s, &L, dkw, hd, b, h, dk);
      layout_out(s, &L, dvw, hd, b, h, dv);
    }
  free(qw); free(kw); free(vw); free(dow); free(dqw); free(dkw); free(dvw); free(bins_w);
  free_layout(&L);
  return status;
}

/* Index map of steps 1-3: for every (b, window, slot) the source token
 * (b*H + y)*W + x, or -1 where the slot holds a pad position (or a stored
 * token outside the valid extent). Built by pushing token ids through the same
 * pad / roll / partition steps as the data. */
int swin_oracle_index_map(const swin_oracle_shape* s, int64_t* map) {
  if (!shape_ok(s)) return ORACLE_BAD_SHAPE;
  const int64_t Hp = round_up(s->H, s->win_h), Wp = round_up(s->W, s->win_w);
  const int64_t cells = Hp * Wp;
  int64_t* padded = (int64_t*)malloc(sizeof(int64_t) * cells + 8);
  int64_t* rolled = (int64_t*)malloc(sizeof(int64_t) * cells + 8);
  if (!padded || !rolled) { free(padded); free(rolled); return ORACLE_NO_MEMORY; }
  for (int64_t b = 0; b < s->B; ++b) {
    for (int64_t y = 0; y < Hp; ++y)
      for (int64_t x = 0; x < Wp; ++x)
        padded[y * Wp + x] =
            (y < valid_rows(s) && x < valid_cols(s)) ? (b * s->H + y) * s->W + x : -1;
    step2_roll(padded, rolled, Hp, Wp, sizeof(int64_t), s->shift_h, s->shift_w);
    step3_partition(rolled, map + b * cells, Hp, Wp, s->win_h, s->win_w, sizeof(int64_t));
  }
  free(padded); free(rolled);
  return ORACLE_OK;
}

/* Region label of every (window, slot) of one batch image, in window order. */
int swin_oracle_region_labels(const swin_oracle_shape* s, int32_t* labels) {
  if (!shape_ok(s)) return ORACLE_BAD_SHAPE;
  const int64_t Hp = round_up(s->H, s->win_h), Wp = round_up(s->W, s->win_w);
  int32_t* lab = (int32_t*)malloc(sizeof(int32_t) * Hp * Wp + 4);
  if (!lab) return ORACLE_NO_MEMORY;
  step3_region_labels(Hp, Wp, s, lab);
  step3_partition(lab, labels, Hp, Wp, s->win_h, s->win_w, sizeof(int32_t));
  free(lab);
  return ORACLE_OK;
}

/* Round trips used by the identity pins: partition then reverse, roll then
 * unroll, on an int64 grid of H^ x W^ values. `out` receives the result. */
int swin_oracle_roundtrip(const swin_oracle_shape* s, const int64_t* grid, int64_t* out,
                          int which) {
  if (!shape_ok(s)) return ORACLE_BAD_SHAPE;
  const int64_t Hp = round_up(s->H, s->win_h), Wp = round_up(s->W, s->win_w);
  int64_t* mid = (int64_t*)malloc(sizeof(int64_t) * Hp * Wp + 8);
  if (!mid) return ORACLE_NO_MEMORY;
  if (which == 0) {
    step3_partition(grid, mid, Hp, Wp, s->win_h, s->win_w, sizeof(int64_t));
    step5_reverse(mid, out, Hp, Wp, s->win_h, s->win_w, sizeof(int64_t));
  } else {
    step2_roll(grid, mid, Hp, Wp, sizeof(int64_t), s->shift_h, s->shift_w);
    step6_unroll(mid, out, Hp, Wp, sizeof(int64_t), s->shift_h, s->shift_w);
  }
  free(mid);
  return ORACLE_OK;
}

int swin_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
