// tiled_mma.cu -- shifted-window attention for windows of up to 256 tokens
// (16 x 16 windows, odd window sizes, shapes the tcgen05 kernels do not take)
// on warp-level tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulate).
//
// Same operation as the other kernel families (TERRA page, Abstract:
// window-based Swin attention with shifted-window execution; Table I: grid
// H x W padded to H^ x W^): pad, cyclic shift, window partition, softmax of
// q.k / sqrt(hd) + relative-position bias over the keys of the query's own
// shift region, P V, and the inverse layout; backward dq, dk, dv and the
// bias-table gradient.
//
// One CTA owns one (window, head) pair and holds all of the window's q, k, v
// (and dO) rows in shared memory, so every softmax row sees all of its keys
// without a second pass over HBM. Pad, shift and partition are folded into the
// per-slot source addresses (geometry.cuh); pad slots are zero-filled by the
// copy and masked as keys. Windows with N tokens use NP = 64, 128 or 256 slots
// (N rounded up); slots past N are masked like pad.
//
// Forward, warp w, query rows [16w, 16w + 16): S = Q K^T in 64-key chunks with
// an online softmax (running row max and sum, O rescaled), O += P V. A
// 256-slot window runs as two CTAs of 8 warps, one per half of its query rows
// (both load the whole window; the second read of k and v mostly hits L2), so
// two CTAs share an SM and one's loads overlap the other's math.
// Backward, recomputing everything from q, k, v, dO and the table:
//   pass 1, warp w, query rows [16w, 16w + 16): S and dP = dO V^T per 64-key
//     chunk with the same online rescaling give the row max m_i, the row sum
//     l_i and D_i = sum_j P_ij dP_ij;
//   pass 2, warp w, key rows [16w, 16w + 16): per chunk of 64 queries,
//     S^T = K Q^T and dP^T = V dO^T, then P^T and dS^T = P^T (dP^T - D);
//     dV += P^T dO and dK += dS^T Q accumulate in registers, with P and dS
//     split into bf16 high and low parts so the products keep about 16 bits;
//     dS^T goes to shared memory and, after a CTA barrier, the warps compute
//     dQ = dS K for the chunk's 64 queries.
//   The bias-table gradient is summed exactly in integers (dbias_fixed.cuh):
//   pass 1 also gives a bound on |dS| over the tile, which sets the unit 2^-E
//   of the tile's int32 shared bins; the bins are then folded into the
//   workspace's wide integer sums. The result does not depend on the order of
//   the additions, and its relative error not on the scale of the gradients.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/swin_wattn.h"
#include "dbias_fixed.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace swin {
namespace {

using namespace ptx;

constexpr float kLog2eT = 1.4426950408889634f;
constexpr float kLn2T = 0.6931471805599453f;
constexpr size_t kSmemLimitT = 227 * 1024;

struct TiledParams {
  Geo g;
  int bins_pad;
  float scale_log2;   // log2(e) / sqrt(hd): logits in base-2 units
  float dscale;       // 1 / sqrt(hd)
  const uint16_t* q;  // bf16 bits, [B, H, W, heads, hd]
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* dout;
  const float* bias_t;  // [heads][bins_pad], times log2(e)
  uint16_t* out;
  float* lse;
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  long long* dt_acc;    // exact bias-gradient sums [heads][bins_pad][kLimbStride]
};

// ---- shared-memory layout of one tile --------------------------------------
// q, k, v (, dO) as [NP][hd] bf16 with 16-byte chunks XOR-swizzled per row;
// backward: the dS^T buffer of one 64-query chunk, high and low parts, as
// [NP keys][64 queries] bf16; per-slot source offsets and info words; row
// statistics (backward: log-sum-exp and D per query); the head's bias row;
// backward: int32 bias-gradient bins and the tile's bound on |dS|.
struct TLay {
  uint32_t q, k, v, dout, dsh, dsl, off, info, stat, bias, bins, total;
};

template <int HD, int NP>
__host__ __device__ inline TLay tlayout(bool bwd, int bins_pad) {
  TLay L;
  const uint32_t tile = NP * HD * 2;
  L.q = 0;
  L.k = tile;
  L.v = 2 * tile;
  uint32_t o = 3 * tile;
  L.dout = L.dsh = L.dsl = 0;
  if (bwd) {
    L.dout = o;
    o += tile;
    L.dsh = o;
    o += NP * 128;
    L.dsl = o;
    o += NP * 128;
  }
  L.off = o;
  o += NP * 8;
  L.info = o;
  o += NP * 4;
  L.stat = o;
  o += bwd ? NP * 8 : 0;
  L.bias = o;
  o += (uint32_t)bins_pad * 4;
  L.bins = o;
  o += bwd ? (uint32_t)bins_pad * 4 + 16 : 0;
  L.total = o;
  return L;
}

// Byte offset of 16-byte chunk `c` of row `r` in a tile whose rows are RB bytes
// (64 or 128): the chunk index is XORed with row bits so that the eight row
// addresses of one ldmatrix land in eight different bank groups.
template <int RB>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  if constexpr (RB == 128)
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
  else
    return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// ---- warp-level tensor-core and copy wrappers -------------------------------
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// c += a (16x16, row-major fragment) * b (16x8, column-major fragment)
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 16-byte global -> shared copy; src_bytes = 0 fills the chunk with zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// x = hi + lo with hi = x truncated to bf16 and lo = bf16(x - hi), for a pair
// of values packed as bf16x2 (first value in the low half).
__device__ __forceinline__ void split_pair(float x, float y, uint32_t& hi, uint32_t& lo) {
  const uint32_t a = __float_as_uint(x) & 0xFFFF0000u;
  const uint32_t b = __float_as_uint(y) & 0xFFFF0000u;
  hi = __byte_perm(a, b, 0x7632);
  lo = pack_bf16(x - __uint_as_float(a), y - __uint_as_float(b));
}

// Slot info word: bits 0-15 the slot's position iy * (2 ww - 1) + ix, bits
// 16-19 its label as a key (15: pad or past the window, matches nothing), bits
// 20-23 its label as a query (14: no output). Allowed pair <=> key label ==
// query label. The bias index of (query i, key j) is pos_i - pos_j + C0.
// PLAIN: a window with no pad slot and a single shift region, where every
// pair is allowed. (The bias index is in range for every pair, allowed or not.)
template <bool PLAIN>
__device__ __forceinline__ float logit(float s, uint32_t kw, int qp, uint32_t ql,
                                       const float* bias, float sc) {
  const float x = fmaf(s, sc, bias[qp - (int)(kw & 0xFFFFu)]);
  if constexpr (PLAIN)
    return x;
  else
    return ((kw >> 16) & 15u) == ql ? x : -INFINITY;
}

// Common tile prologue: slot table, bias row, cleared bins, and the q, k, v
// (and dO) rows of window `win`, head `h`, copied into swizzled shared tiles.
// Returns true for a plain window (N = NP slots, all real tokens, one shift
// region).
template <int HD, int NP, bool BWD>
__device__ __forceinline__ bool tile_setup(const TiledParams& p, uint8_t* smem, const TLay& L,
                                           long long win, int h) {
  const Geo& g = p.g;
  const int tid = threadIdx.x;
  uint32_t* info = (uint32_t*)(smem + L.info);
  long long* off = (long long*)(smem + L.off);
  int plain = 1;
  if (tid < NP) {
    uint32_t w = (14u << 20) | (15u << 16);
    long long o = -1;
    plain = 0;
    if (tid < g.N) {
      const SlotInfo s = slot_info(g, win, tid);
      const uint32_t pos = (uint32_t)(s.iy * (2 * g.ww - 1) + s.ix);
      plain = s.valid && s.label == slot_info(g, win, 0).label;
      // a stored token beyond the valid extent keeps its address (its
      // outputs are written, as zeros) but matches no query and no key
      w = s.valid ? pos | ((uint32_t)s.label << 16) | ((uint32_t)s.label << 20)
                  : pos | (15u << 16) | (14u << 20);
      if (s.stored) o = (token_of(g, s) * g.heads + h) * HD;
    }
    info[tid] = w;
    off[tid] = o;
  }
  float* bias = (float*)(smem + L.bias);
  for (int b = tid; b < p.bins_pad; b += blockDim.x) bias[b] = p.bias_t[(size_t)h * p.bins_pad + b];
  if (BWD) {
    int* bins = (int*)(smem + L.bins);   // bins, then the tile's |dS| bound (float bits)
    for (int b = tid; b <= p.bins_pad; b += blockDim.x) bins[b] = 0;
  }
  plain = __syncthreads_and(plain);
  constexpr int CH = HD / 8;
  const uint32_t base = smem_u32(smem);
  for (int idx = tid; idx < NP * CH; idx += blockDim.x) {
    const int slot = idx / CH, c = idx - slot * CH;
    const long long o = off[slot];
    const uint32_t d = swz<HD * 2>(slot, c);
    const uint32_t n = o >= 0 ? 16u : 0u;
    const long long e = o >= 0 ? o + c * 8 : 0;
    cp_async16(base + L.q + d, p.q + e, n);
    cp_async16(base + L.k + d, p.k + e, n);
    cp_async16(base + L.v + d, p.v + e, n);
    if (BWD) cp_async16(base + L.dout + d, p.dout + e, n);
  }
  cp_async_wait_all();
  __syncthreads();
  return plain != 0;
}

// ---- forward ------------------------------------------------------------------
template <int HD, int NP, bool PLAIN>
__device__ __forceinline__ void fwd_tile(const TiledParams& p, uint8_t* smem, const TLay& L,
                                         int qbase) {
  const Geo& g = p.g;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3, rr = lane & 7;
  const uint32_t base = smem_u32(smem);
  const uint32_t sq = base + L.q, sk = base + L.k, sv = base + L.v;
  const uint32_t* info = (const uint32_t*)(smem + L.info);
  const long long* off = (const long long*)(smem + L.off);
  const float* bias = (const float*)(smem + L.bias);
  const int C0 = (g.wh - 1) * (2 * g.ww - 1) + g.ww - 1;
  const float sc = p.scale_log2;
  const int r0 = qbase + warp * 16;

  uint32_t qa[HD / 16][4];
#pragma unroll
  for (int ks = 0; ks < HD / 16; ++ks)
    ldsm4(sq + swz<HD * 2>(r0 + (mi & 1) * 8 + rr, 2 * ks + (mi >> 1)), qa[ks]);
  const uint32_t qw0 = info[r0 + g8], qw1 = info[r0 + g8 + 8];
  const int qp0 = (int)(qw0 & 0xFFFFu) + C0, qp1 = (int)(qw1 & 0xFFFFu) + C0;
  const uint32_t ql0 = (qw0 >> 20) & 15u, ql1 = (qw1 >> 20) & 15u;

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[HD / 8][4];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

#pragma unroll 1
  for (int kc = 0; kc < NP / 64; ++kc) {
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        ldsm4(sk + swz<HD * 2>(kc * 64 + np * 16 + (mi >> 1) * 8 + rr, 2 * ks + (mi & 1)), b);
        mma16816(s[2 * np], qa[ks], b[0], b[1]);
        mma16816(s[2 * np + 1], qa[ks], b[2], b[3]);
      }
    float c0 = -INFINITY, c1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const uint2 kw = *(const uint2*)(info + kc * 64 + n * 8 + 2 * t4);
      s[n][0] = logit<PLAIN>(s[n][0], kw.x, qp0, ql0, bias, sc);
      s[n][1] = logit<PLAIN>(s[n][1], kw.y, qp0, ql0, bias, sc);
      s[n][2] = logit<PLAIN>(s[n][2], kw.x, qp1, ql1, bias, sc);
      s[n][3] = logit<PLAIN>(s[n][3], kw.y, qp1, ql1, bias, sc);
      c0 = fmaxf(c0, fmaxf(s[n][0], s[n][1]));
      c1 = fmaxf(c1, fmaxf(s[n][2], s[n][3]));
    }
    c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 1));
    c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 2));
    c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 1));
    c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 2));
    const float n0 = fmaxf(m0, c0), n1 = fmaxf(m1, c1);
    // a row with no allowed key so far keeps max -inf; subtract 0 there
    const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
    const float a0 = ex2(m0 - u0), a1 = ex2(m1 - u1);
    m0 = n0;
    m1 = n1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      s[n][0] = ex2(s[n][0] - u0);
      s[n][1] = ex2(s[n][1] - u0);
      s[n][2] = ex2(s[n][2] - u1);
      s[n][3] = ex2(s[n][3] - u1);
      ps0 += s[n][0] + s[n][1];
      ps1 += s[n][2] + s[n][3];
    }
    l0 = l0 * a0 + ps0;
    l1 = l1 * a1 + ps1;
#pragma unroll
    for (int n = 0; n < HD / 8; ++n) {
      o[n][0] *= a0;
      o[n][1] *= a0;
      o[n][2] *= a1;
      o[n][3] *= a1;
    }
#pragma unroll
    for (int k2 = 0; k2 < 4; ++k2) {
      const uint32_t a[4] = {pack_bf16(s[2 * k2][0], s[2 * k2][1]),
                             pack_bf16(s[2 * k2][2], s[2 * k2][3]),
                             pack_bf16(s[2 * k2 + 1][0], s[2 * k2 + 1][1]),
                             pack_bf16(s[2 * k2 + 1][2], s[2 * k2 + 1][3])};
#pragma unroll
      for (int np = 0; np < HD / 16; ++np) {
        uint32_t b[4];
        ldsm4t(sv + swz<HD * 2>(kc * 64 + k2 * 16 + (mi & 1) * 8 + rr, 2 * np + (mi >> 1)), b);
        mma16816(o[2 * np], a, b[0], b[1]);
        mma16816(o[2 * np + 1], a, b[2], b[3]);
      }
    }
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const long long o0 = off[r0 + g8], o1 = off[r0 + g8 + 8];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n) {
    const int col = n * 8 + 2 * t4;
    if (o0 >= 0) *(uint32_t*)(p.out + o0 + col) = pack_bf16(o[n][0] * i0, o[n][1] * i0);
    if (o1 >= 0) *(uint32_t*)(p.out + o1 + col) = pack_bf16(o[n][2] * i1, o[n][3] * i1);
  }
  if (p.lse && t4 == 0) {
    if (o0 >= 0) p.lse[o0 / HD] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2T : 0.f;
    if (o1 >= 0) p.lse[o1 / HD] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2T : 0.f;
  }
}

// PARTS CTAs per (window, head), each on NP / PARTS query rows.
template <int HD, int NP, int PARTS>
__global__ void __launch_bounds__(NP * 2 / PARTS, 256 * PARTS / NP)
    tiled_fwd_kernel(const __grid_constant__ TiledParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const TLay L = tlayout<HD, NP>(false, p.bins_pad);
  const long long tile = blockIdx.x / PARTS;
  const int qbase = (int)(blockIdx.x % PARTS) * (NP / PARTS);
  const int h = (int)(tile % p.g.heads);
  const long long win = tile / p.g.heads;
  if (tile_setup<HD, NP, false>(p, smem, L, win, h))
    fwd_tile<HD, NP, true>(p, smem, L, qbase);
  else
    fwd_tile<HD, NP, false>(p, smem, L, qbase);
}

// ---- backward -----------------------------------------------------------------
// Adds dS (one value of the tile) to the int32 bin of bias index b, in units
// of 2^-E (qs = 2^E): every term is below 2^22 units and a bin takes at most
// NP <= 256 terms, so the sum cannot overflow.
template <bool PLAIN>
__device__ __forceinline__ void bin_add(int* bins, int b, float ds, float qs) {
  if (!PLAIN && ds == 0.f) return;   // masked pairs of seam and pad windows
  red_add_s32(bins + b, round_to_int(ds * qs));
}

template <int HD, int NP, int QS, bool PLAIN>
__device__ __forceinline__ void bwd_tile(const TiledParams& p, uint8_t* smem, const TLay& L,
                                         int h) {
  constexpr int NW = NP / 16;
  const Geo& g = p.g;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3, rr = lane & 7;
  const uint32_t base = smem_u32(smem);
  const uint32_t sq = base + L.q, sk = base + L.k, sv = base + L.v, sdo = base + L.dout;
  const uint32_t sdh = base + L.dsh, sdl = base + L.dsl;
  const uint32_t* info = (const uint32_t*)(smem + L.info);
  const long long* off = (const long long*)(smem + L.off);
  const float* bias = (const float*)(smem + L.bias);
  float* st_lse = (float*)(smem + L.stat);   // log2 of the row sum of 2^logit
  float* st_d = st_lse + NP;                 // D = sum_j P_ij dP_ij
  int* bins = (int*)(smem + L.bins);
  unsigned* bound_bits = (unsigned*)(bins + p.bins_pad);   // tile max of the row bounds
  const int C0 = (g.wh - 1) * (2 * g.ww - 1) + g.ww - 1;
  const float sc = p.scale_log2;

  // ---- pass 1: log-sum-exp and D per query row ----
  {
    const int r0 = warp * 16;
    uint32_t qa[HD / 16][4], da[HD / 16][4];
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks) {
      ldsm4(sq + swz<HD * 2>(r0 + (mi & 1) * 8 + rr, 2 * ks + (mi >> 1)), qa[ks]);
      ldsm4(sdo + swz<HD * 2>(r0 + (mi & 1) * 8 + rr, 2 * ks + (mi >> 1)), da[ks]);
    }
    const uint32_t qw0 = info[r0 + g8], qw1 = info[r0 + g8 + 8];
    const int qp0 = (int)(qw0 & 0xFFFFu) + C0, qp1 = (int)(qw1 & 0xFFFFu) + C0;
    const uint32_t ql0 = (qw0 >> 20) & 15u, ql1 = (qw1 >> 20) & 15u;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, d0 = 0.f, d1 = 0.f;
    float x0 = 0.f, x1 = 0.f;   // max |dP| of the two rows
#pragma unroll 1
    for (int kc = 0; kc < NP / 64; ++kc) {
      float s[8][4], dp[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks)
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const uint32_t a = swz<HD * 2>(kc * 64 + np * 16 + (mi >> 1) * 8 + rr, 2 * ks + (mi & 1));
          uint32_t b[4];
          ldsm4(sk + a, b);
          mma16816(s[2 * np], qa[ks], b[0], b[1]);
          mma16816(s[2 * np + 1], qa[ks], b[2], b[3]);
          ldsm4(sv + a, b);
          mma16816(dp[2 * np], da[ks], b[0], b[1]);
          mma16816(dp[2 * np + 1], da[ks], b[2], b[3]);
        }
      float c0 = -INFINITY, c1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const uint2 kw = *(const uint2*)(info + kc * 64 + n * 8 + 2 * t4);
        s[n][0] = logit<PLAIN>(s[n][0], kw.x, qp0, ql0, bias, sc);
        s[n][1] = logit<PLAIN>(s[n][1], kw.y, qp0, ql0, bias, sc);
        s[n][2] = logit<PLAIN>(s[n][2], kw.x, qp1, ql1, bias, sc);
        s[n][3] = logit<PLAIN>(s[n][3], kw.y, qp1, ql1, bias, sc);
        c0 = fmaxf(c0, fmaxf(s[n][0], s[n][1]));
        c1 = fmaxf(c1, fmaxf(s[n][2], s[n][3]));
        x0 = fmaxf(x0, fmaxf(fabsf(dp[n][0]), fabsf(dp[n][1])));
        x1 = fmaxf(x1, fmaxf(fabsf(dp[n][2]), fabsf(dp[n][3])));
      }
      c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 1));
      c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 2));
      c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 1));
      c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 2));
      const float n0 = fmaxf(m0, c0), n1 = fmaxf(m1, c1);
      const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
      const float a0 = ex2(m0 - u0), a1 = ex2(m1 - u1);
      m0 = n0;
      m1 = n1;
      float ps0 = 0.f, ps1 = 0.f, pd0 = 0.f, pd1 = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const float e0 = ex2(s[n][0] - u0), e1 = ex2(s[n][1] - u0);
        const float e2 = ex2(s[n][2] - u1), e3 = ex2(s[n][3] - u1);
        ps0 += e0 + e1;
        ps1 += e2 + e3;
        pd0 = fmaf(e0, dp[n][0], fmaf(e1, dp[n][1], pd0));
        pd1 = fmaf(e2, dp[n][2], fmaf(e3, dp[n][3], pd1));
      }
      l0 = l0 * a0 + ps0;
      l1 = l1 * a1 + ps1;
      d0 = d0 * a0 + pd0;
      d1 = d1 * a1 + pd1;
    }
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, x);
      l1 += __shfl_xor_sync(0xffffffffu, l1, x);
      d0 += __shfl_xor_sync(0xffffffffu, d0, x);
      d1 += __shfl_xor_sync(0xffffffffu, d1, x);
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, x));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, x));
    }
    if (t4 == 0) {
      // |dS_ij| = P_ij |dP_ij - D_i| <= (1 / l_i) (max_j |dP_ij| + |D_i|);
      // non-negative floats order like their bit patterns (NaN above all)
      float b0 = l0 > 0.f ? (x0 + fabsf(d0 / l0)) / l0 : 0.f;
      float b1 = l1 > 0.f ? (x1 + fabsf(d1 / l1)) / l1 : 0.f;
      if (!(b0 <= 3.0e38f)) b0 = INFINITY;   // NaN -> +inf: fmaxf would drop a NaN
      if (!(b1 <= 3.0e38f)) b1 = INFINITY;
      atomicMax(bound_bits, __float_as_uint(fmaxf(b0, b1)));
      // P = 2^(logit - lse); rows without an allowed key (pad queries) get
      // lse = +inf, hence P = 0, in pass 2
      st_lse[r0 + g8] = l0 > 0.f ? m0 + log2f(l0) : INFINITY;
      st_d[r0 + g8] = l0 > 0.f ? d0 / l0 : 0.f;
      st_lse[r0 + g8 + 8] = l1 > 0.f ? m1 + log2f(l1) : INFINITY;
      st_d[r0 + g8 + 8] = l1 > 0.f ? d1 / l1 : 0.f;
    }
  }
  __syncthreads();
  const float tile_bound = __uint_as_float(*bound_bits);
  const bool finite = tile_bound <= 3.0e38f;   // false for NaN and infinity
  const int E = tile_exponent(finite ? tile_bound : 0.f);
  const float qs = exp2_int(E);

  // ---- pass 2: key-major dV, dK; dS^T to shared; dQ per 64-query chunk ----
  const int kb = warp * 16;
  const uint32_t kw0 = info[kb + g8], kw1 = info[kb + g8 + 8];
  const int kp0 = (int)(kw0 & 0xFFFFu), kp1 = (int)(kw1 & 0xFFFFu);
  const uint32_t kl0 = (kw0 >> 16) & 15u, kl1 = (kw1 >> 16) & 15u;
  float dv[HD / 8][4], dk[HD / 8][4];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dv[n][e] = dk[n][e] = 0.f;

#pragma unroll 1
  for (int qc = 0; qc < NP / 64; ++qc) {
#pragma unroll 1
    for (int sub = 0; sub < 64 / QS; ++sub) {
      const int qb = qc * 64 + sub * QS;
      constexpr int NT = QS / 8;
      float st[NT][4], dpt[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        uint32_t ak[4], av[4];
        const uint32_t aa = swz<HD * 2>(kb + (mi & 1) * 8 + rr, 2 * ks + (mi >> 1));
        ldsm4(sk + aa, ak);
        ldsm4(sv + aa, av);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          const uint32_t ba = swz<HD * 2>(qb + np * 16 + (mi >> 1) * 8 + rr, 2 * ks + (mi & 1));
          uint32_t b[4];
          ldsm4(sq + ba, b);
          mma16816(st[2 * np], ak, b[0], b[1]);
          mma16816(st[2 * np + 1], ak, b[2], b[3]);
          ldsm4(sdo + ba, b);
          mma16816(dpt[2 * np], av, b[0], b[1]);
          mma16816(dpt[2 * np + 1], av, b[2], b[3]);
        }
      }
      // P^T and dS^T; fixed-point bias-gradient bins
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int i = qb + n * 8 + 2 * t4;
        const uint2 qw = *(const uint2*)(info + i);
        const float2 lq = *(const float2*)(st_lse + i);
        const float2 dq2 = *(const float2*)(st_d + i);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t qwe = (e & 1) ? qw.y : qw.x;
          const float lse = (e & 1) ? lq.y : lq.x;
          const float D = (e & 1) ? dq2.y : dq2.x;
          const int kp = (e >> 1) ? kp1 : kp0;
          const uint32_t kl = (e >> 1) ? kl1 : kl0;
          const int bidx = (int)(qwe & 0xFFFFu) - kp + C0;
          const bool ok = PLAIN || kl == ((qwe >> 20) & 15u);
          const float x = ok ? fmaf(st[n][e], sc, bias[bidx]) : -INFINITY;
          const float pe = ex2(x - lse);
          const float ds = pe * (dpt[n][e] - D);
          if (ok && finite) bin_add<PLAIN>(bins, bidx, ds, qs);
          st[n][e] = pe;
          dpt[n][e] = ds * p.dscale;
        }
      }
      // dV += P^T dO, dK += dS^T Q (high and low parts), dS^T -> shared
#pragma unroll
      for (int k2 = 0; k2 < QS / 16; ++k2) {
        uint32_t ph[4], pl[4], sh[4], sl[4];
        split_pair(st[2 * k2][0], st[2 * k2][1], ph[0], pl[0]);
        split_pair(st[2 * k2][2], st[2 * k2][3], ph[1], pl[1]);
        split_pair(st[2 * k2 + 1][0], st[2 * k2 + 1][1], ph[2], pl[2]);
        split_pair(st[2 * k2 + 1][2], st[2 * k2 + 1][3], ph[3], pl[3]);
        split_pair(dpt[2 * k2][0], dpt[2 * k2][1], sh[0], sl[0]);
        split_pair(dpt[2 * k2][2], dpt[2 * k2][3], sh[1], sl[1]);
        split_pair(dpt[2 * k2 + 1][0], dpt[2 * k2 + 1][1], sh[2], sl[2]);
        split_pair(dpt[2 * k2 + 1][2], dpt[2 * k2 + 1][3], sh[3], sl[3]);
#pragma unroll
        for (int np = 0; np < HD / 16; ++np) {
          const uint32_t ba = swz<HD * 2>(qb + k2 * 16 + (mi & 1) * 8 + rr, 2 * np + (mi >> 1));
          uint32_t bo[4], bq[4];
          ldsm4t(sdo + ba, bo);
          ldsm4t(sq + ba, bq);
          // high parts into four accumulators, then the low parts: no MMA
          // waits on the one issued just before it
          mma16816(dv[2 * np], ph, bo[0], bo[1]);
          mma16816(dv[2 * np + 1], ph, bo[2], bo[3]);
          mma16816(dk[2 * np], sh, bq[0], bq[1]);
          mma16816(dk[2 * np + 1], sh, bq[2], bq[3]);
          mma16816(dv[2 * np], pl, bo[0], bo[1]);
          mma16816(dv[2 * np + 1], pl, bo[2], bo[3]);
          mma16816(dk[2 * np], sl, bq[0], bq[1]);
          mma16816(dk[2 * np + 1], sl, bq[2], bq[3]);
        }
        // fragment word j holds (key row g8 + 8 (j & 1), queries col + 8 (j >> 1))
        const int col = sub * QS + k2 * 16 + 2 * t4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = kb + g8 + 8 * (j & 1), cc = col + 8 * (j >> 1);
          const uint32_t a = swz<128>(r, cc >> 3) + (uint32_t)(cc & 7) * 2;
          sts32(sdh + a, sh[j]);
          sts32(sdl + a, sl[j]);
        }
      }
    }
    __syncthreads();
    // dQ rows [qc*64, qc*64 + 64): warp -> one 16-row block, U n-tiles of 8
    {
      constexpr int NTQ = HD / 8;
      constexpr int UNITS = 4 * NTQ;
      constexpr int U = UNITS / NW < 2 ? 2 : UNITS / NW;
      constexpr int ACTIVE = UNITS / U;
      if (warp < ACTIVE) {
        const int unit0 = warp * U, rb = unit0 / NTQ, n0 = unit0 % NTQ;
        // separate accumulators for the high and low parts of dS (summed at
        // the end) give 2U independent MMA chains; with U >= 4 chains already
        // (few warps), one set keeps the registers in budget
        constexpr int UL = U >= 4 ? 1 : U;
        float acc[U][4], acl[UL][4];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[u][e] = 0.f;
#pragma unroll
        for (int u = 0; u < UL; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) acl[u][e] = 0.f;
#pragma unroll 8
        for (int ks = 0; ks < NP / 16; ++ks) {
          uint32_t ah[4], al[4];
          const uint32_t aa = swz<128>(ks * 16 + (mi >> 1) * 8 + rr, rb * 2 + (mi & 1));
          ldsm4t(sdh + aa, ah);
          ldsm4t(sdl + aa, al);
#pragma unroll
          for (int up = 0; up < U / 2; ++up) {
            uint32_t b[4];
            ldsm4t(sk + swz<HD * 2>(ks * 16 + (mi & 1) * 8 + rr, n0 + 2 * up + (mi >> 1)), b);
            mma16816(acc[2 * up], ah, b[0], b[1]);
            mma16816(acc[2 * up + 1], ah, b[2], b[3]);
            if constexpr (UL == U) {
              mma16816(acl[2 * up], al, b[0], b[1]);
              mma16816(acl[2 * up + 1], al, b[2], b[3]);
            } else {
              mma16816(acc[2 * up], al, b[0], b[1]);
              mma16816(acc[2 * up + 1], al, b[2], b[3]);
            }
          }
        }
        if constexpr (UL == U) {
#pragma unroll
          for (int u = 0; u < U; ++u)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[u][e] += acl[u][e];
        }
        const int row = qc * 64 + rb * 16 + g8;
        const long long o0 = off[row], o1 = off[row + 8];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = (n0 + u) * 8 + 2 * t4;
          if (o0 >= 0) *(uint32_t*)(p.dq + o0 + c) = pack_bf16(acc[u][0], acc[u][1]);
          if (o1 >= 0) *(uint32_t*)(p.dq + o1 + c) = pack_bf16(acc[u][2], acc[u][3]);
        }
      }
    }
    __syncthreads();
  }
  {
    const long long o0 = off[kb + g8], o1 = off[kb + g8 + 8];
#pragma unroll
    for (int n = 0; n < HD / 8; ++n) {
      const int c = n * 8 + 2 * t4;
      if (o0 >= 0) {
        *(uint32_t*)(p.dv + o0 + c) = pack_bf16(dv[n][0], dv[n][1]);
        *(uint32_t*)(p.dk + o0 + c) = pack_bf16(dk[n][0], dk[n][1]);
      }
      if (o1 >= 0) {
        *(uint32_t*)(p.dv + o1 + c) = pack_bf16(dv[n][2], dv[n][3]);
        *(uint32_t*)(p.dk + o1 + c) = pack_bf16(dk[n][2], dk[n][3]);
      }
    }
  }
  // the tile's bins into the workspace's exact sums (the last loop barrier
  // made every shared add visible)
  long long* acc = p.dt_acc + (size_t)h * p.bins_pad * kLimbStride;
  for (int b = threadIdx.x; b < g.bins; b += blockDim.x) {
    const int v = bins[b];
    if (!finite) flag_nonfinite(acc + (size_t)b * kLimbStride);
    else if (v != 0) add_fixed(acc + (size_t)b * kLimbStride, v, E);
  }
}

template <int HD, int NP, int QS>
__global__ void __launch_bounds__(NP * 2, 256 / NP)
    tiled_bwd_kernel(const __grid_constant__ TiledParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const TLay L = tlayout<HD, NP>(true, p.bins_pad);
  const int h = (int)(blockIdx.x % p.g.heads);
  const long long win = blockIdx.x / p.g.heads;
  if (tile_setup<HD, NP, true>(p, smem, L, win, h))
    bwd_tile<HD, NP, QS, true>(p, smem, L, h);
  else
    bwd_tile<HD, NP, QS, false>(p, smem, L, h);
}

int slots_for(int N) { return N <= 64 ? 64 : (N <= 128 ? 128 : 256); }

// Query-chunk width of the backward's key-major pass (register budget).
constexpr int kQS = 32;

template <int HD>
size_t tiled_smem(const Geo& g, bool bwd) {
  const int bp = bins_padded(g.bins);
  switch (slots_for(g.N)) {
    case 64: return tlayout<HD, 64>(bwd, bp).total;
    case 128: return tlayout<HD, 128>(bwd, bp).total;
    default: return tlayout<HD, 256>(bwd, bp).total;
  }
}

size_t tiled_smem_any(const Geo& g, bool bwd) {
  return g.hd == 64 ? tiled_smem<64>(g, bwd) : tiled_smem<32>(g, bwd);
}

void fill_params(TiledParams& p, const Geo& g, const float* bias_t) {
  memset(&p, 0, sizeof(p));
  p.g = g;
  p.bins_pad = bins_padded(g.bins);
  p.dscale = 1.f / sqrtf((float)g.hd);
  p.scale_log2 = kLog2eT * p.dscale;
  p.bias_t = bias_t;
}

template <typename K>
cudaError_t launch_tiled(K kernel, const TiledParams& p, int threads, size_t smem,
                         cudaStream_t st, int parts = 1) {
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long tiles = p.g.n_win * p.g.heads * parts;
  kernel<<<(unsigned)tiles, threads, smem, st>>>(p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool tiled_supported(const Geo& g, int dtype) {
  if (dtype != SWIN_DTYPE_BF16) return false;
  if (g.hd != 64 && g.hd != 32) return false;
  if (g.N > 256) return false;
  if (g.n_win * (long long)g.heads * 2 > 0x7fffffffLL) return false;   // grid size
  return tiled_smem_any(g, true) <= kSmemLimitT && tiled_smem_any(g, false) <= kSmemLimitT;
}

// Workspace: header (status word), bias table [heads][bins_pad] fp32, and the
// exact bias-gradient sums [heads][bins_pad][kLimbStride] int64.
size_t tiled_workspace(const Geo& g) {
  const int bp = bins_padded(g.bins);
  return kWsHeader + align256((size_t)g.heads * bp * 4) + align256(dbias_fixed_bytes(g));
}

cudaError_t tiled_forward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, void* out, float* lse, void* ws, cudaStream_t st) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  TiledParams p;
  fill_params(p, g, bias_t);
  p.q = (const uint16_t*)q;
  p.k = (const uint16_t*)k;
  p.v = (const uint16_t*)v;
  p.out = (uint16_t*)out;
  p.lse = lse;
  cudaError_t e = prep_bias(g, table, bias_t, nullptr, st);
  if (e != cudaSuccess) return e;
  const int NP = slots_for(g.N);
  const size_t smem = tiled_smem_any(g, false);
  if (g.hd == 64) {
    if (NP == 64) return launch_tiled(tiled_fwd_kernel<64, 64, 1>, p, 128, smem, st);
    if (NP == 128) return launch_tiled(tiled_fwd_kernel<64, 128, 1>, p, 256, smem, st);
    return launch_tiled(tiled_fwd_kernel<64, 256, 2>, p, 256, smem, st, 2);
  }
  if (NP == 64) return launch_tiled(tiled_fwd_kernel<32, 64, 1>, p, 128, smem, st);
  if (NP == 128) return launch_tiled(tiled_fwd_kernel<32, 128, 1>, p, 256, smem, st);
  return launch_tiled(tiled_fwd_kernel<32, 256, 2>, p, 256, smem, st, 2);
}

cudaError_t tiled_backward(const Geo& g, const void* q, const void* k, const void* v,
                           const float* table, const void* dout, void* dq, void* dk, void* dv,
                           float* dtable, void* ws, int flags, cudaStream_t st) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  long long* dt_acc = (long long*)((char*)ws + dbias_fixed_offset(g));
  TiledParams p;
  fill_params(p, g, bias_t);
  p.q = (const uint16_t*)q;
  p.k = (const uint16_t*)k;
  p.v = (const uint16_t*)v;
  p.dout = (const uint16_t*)dout;
  p.dq = (uint16_t*)dq;
  p.dk = (uint16_t*)dk;
  p.dv = (uint16_t*)dv;
  p.dt_acc = dt_acc;
  cudaError_t e = prep_bias(g, table, bias_t, dt_acc, st);
  if (e != cudaSuccess) return e;
  const int NP = slots_for(g.N);
  const size_t smem = tiled_smem_any(g, true);
  if (g.hd == 64) {
    if (NP == 64) e = launch_tiled(tiled_bwd_kernel<64, 64, kQS>, p, 128, smem, st);
    else if (NP == 128) e = launch_tiled(tiled_bwd_kernel<64, 128, kQS>, p, 256, smem, st);
    else e = launch_tiled(tiled_bwd_kernel<64, 256, kQS>, p, 512, smem, st);
  } else {
    if (NP == 64) e = launch_tiled(tiled_bwd_kernel<32, 64, kQS>, p, 128, smem, st);
    else if (NP == 128) e = launch_tiled(tiled_bwd_kernel<32, 128, kQS>, p, 256, smem, st);
    else e = launch_tiled(tiled_bwd_kernel<32, 256, kQS>, p, 512, smem, st);
  }
  if (e != cudaSuccess) return e;
  if (flags & SWIN_FLAG_DBIAS_SUMS) return cudaSuccess;   // the caller finishes the sums
  return finish_dbias(g, dt_acc, dtable, st);
}

}  // namespace swin
