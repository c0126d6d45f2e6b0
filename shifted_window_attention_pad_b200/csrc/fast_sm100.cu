// fast_sm100.cu -- tcgen05 / TMA kernels for shifted-window attention on B200.
//
// What they compute: shifted-window multi-head self-attention over a padded
// token grid (TERRA page, Abstract: window-based Swin Transformer with
// "shifted-window execution" over ragged window layouts; Table I: the padded
// resolution H^ x W^), read as the published Swin scheme -- pad, cyclic shift,
// window partition, softmax(q k^T / sqrt(d) + relative-position bias + shift
// mask) v, window reverse, reverse shift -- forward and backward, including the
// gradient of the relative-position bias table.
//
// How, on sm_100a:
//  * Layout stage folded into TMA addressing. Each window is one 5-D TMA box
//    [head_dim, 1 head, win_w, win_h, 1 image] of the [B, H, W, heads, hd] tensor,
//    started at its source position (y0 + s) -- the cyclic shift is a coordinate
//    offset, the zero padding is the TMA out-of-bounds fill. A window on the wrap
//    seam is split into up to 2 x 2 sub-boxes (heights win_h - s_h and s_h,
//    widths likewise); their rows land back to back in shared memory and every
//    consumer knows the resulting slot order. No permuted copy ever exists.
//  * A tile is 128 rows = G = 128 / N windows of one head (N = win_h * win_w).
//    S = Q K^T and O = P V (forward) and S, dP = dO V^T, dV = P^T dO, dQ = dS K,
//    dK = dS^T Q (backward) are tcgen05.mma kind::f16, M = 128, fp32 in TMEM.
//    Entries of S that pair different windows are never read; the P and dS
//    tiles keep zeros there, so they contribute nothing.
//  * One warpgroup reads S (and dP) from TMEM one row per thread, adds the bias
//    from a table row in shared memory, applies the pad and shift-region mask
//    from per-slot coordinates (no mask tensor), runs the softmax in registers
//    (a whole window row is in the tile, so no running rescale is needed), writes
//    P (and dS) to shared memory for the next MMAs, and stores outputs straight
//    to their grid rows. The bias-table gradient is summed exactly in integers
//    (dbias_fixed.cuh): per tile, a bound on |dS| sets the unit 2^-E of int32
//    shared-memory bins, and the tile's bins are folded into wide integer sums
//    in global memory. Integer sums do not depend on the order in which
//    threads or CTAs land, so the result is bitwise repeatable, and the unit
//    follows the magnitude of the gradients, so the relative error does not
//    depend on their scale; a last small kernel converts the sums to fp32.
//  * Warp roles: warps 0-3 and 4-7 two softmax/epilogue warpgroups taking
//    alternate tiles, warp 8 TMA producer, warp 9 issues S (and dP) and owns TMEM,
//    warp 10 issues PV (or the gradient products). Persistent grid of one
//    CTA per SM; tiles go round-robin, head fastest, so the SMs stream
//    neighbouring bytes together.
//  * Every mbarrier wait is bounded (%globaltimer); a wait that runs out records
//    a timeout in the workspace status word and the kernel drains and returns.
#include "fast_common.cuh"

namespace swin {
namespace {

using namespace ptx;

// ================================================================================
// Forward
// ================================================================================
// Per tile: S = Q K^T (MMA) -> softmax row per thread -> P (bf16, smem) ->
// O = P V (MMA) -> normalise and store. Two warpgroups take alternate tiles, so
// while one waits on TMEM loads or an MMA the other computes (two warps per
// scheduler). One thread issues S of each tile as soon as its data and TMEM
// slot are ready, another PV as soon as its P is written.
// P stays in TMEM: S of a tile fills the first 128 columns of its slot, P
// overwrites S's first 64 columns as packed bf16 pairs (the A operand of
// O = P V) once the softmax has read S, and O goes after them. HD <= 64:
// four slots of 128 columns (S | then P in 0-63, O in 64-127) and four input
// stages; HD = 128: two slots of 256 columns (O in 128-255) and two 96 KB
// input stages. (P in shared memory instead, as before: three stages at
// HD = 64 and 8 KB of P stores per row of tiles.)
template <int HD>
struct FwdCfg {
  static constexpr bool kTmemP = true;
  static constexpr int kStages = HD > 64 ? 2 : 4;
  static constexpr int kSlots = HD > 64 ? 2 : 4;
  static constexpr uint32_t kSlotCols = HD > 64 ? 256 : 128;
  static constexpr uint32_t kOCol = HD > 64 ? 128 : 64;    // O inside its slot
  static constexpr uint32_t kPBytes = kTmemP ? 0 : kNumWg * 32768;
};
constexpr int kFwdPBufs = kNumWg;



template <int HD, int WW>
__global__ void __launch_bounds__(kThreads, 1) fwd_kernel(const __grid_constant__ FastParams p) {
  constexpr int N = 64, G = kRows / N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using C = FwdCfg<HD>;
  constexpr int NS = C::kStages, NT = C::kSlots;
  constexpr uint32_t SC = C::kSlotCols;
  constexpr uint32_t tile_bytes = kRows * HD * 2;
  const Geo& g = p.g;
  const Layout L = make_layout<HD, NS, 3, C::kPBytes>(p.bins_pad);
  uint8_t* tiles = smem + L.tiles;
  uint8_t* ptile = smem + L.ptile;
  float* bias = (float*)(smem + L.bias);
  uint32_t* colinfo = (uint32_t*)(smem + L.colinfo);
  uint64_t* bars = (uint64_t*)(smem + L.bars);
  uint64_t* full = bars;
  uint64_t* empty = full + NS;
  uint64_t* s_full = empty + NS;
  uint64_t* p_full = s_full + NT;
  uint64_t* o_full = p_full + NT;
  uint64_t* t_empty = o_full + NT;
  uint64_t* drain = t_empty + NT;   // [2]: one per MMA-issuing thread
  uint64_t* never = drain + 2;
  uint32_t* tmem_slot = (uint32_t*)(smem + L.misc);
  volatile int* abort = (volatile int*)(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_local = local_tiles(p.n_tiles, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < NT; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], kWg);
      mbar_init(&o_full[i], 1); mbar_init(&t_empty[i], kWg);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0)
    for (int tt = 0; tt < 3; ++tt)
      for (int m = 0; m < kMaxMaps; ++m) prefetch_tmap(&p.maps[tt][m]);
  // P tiles start at zero: rows never write the columns of the other window.
  if constexpr (C::kPBytes > 0)
    for (uint32_t i = threadIdx.x; i < C::kPBytes / 16; i += kThreads)
      reinterpret_cast<uint4*>(ptile)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async();
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      long long k = 0;
      for (long long t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++k) {
        const int s = (int)(k % NS);
        const uint32_t ph = (uint32_t)((k / NS) & 1);
        if (!mbar_wait(&empty[s], ph ^ 1, abort, p.status, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&full[s], 3 * tile_bytes + p.bins_pad * 4);
        issue_tile_loads<HD, 3>(p, t, tiles + s * 3 * tile_bytes, bias + s * p.bins_pad, &full[s]);
      }
      if (*abort) {  // let copies already in flight land before the CTA leaves
        const long long first = k > NS ? k - NS : 0;
        for (long long j = first; j < k; ++j)
          mbar_drain(&full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {   // S = Q K^T of every tile, as soon as its data and TMEM slot are ready
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kRows, 0, 0);
      for (long long k = 0; k < n_local; ++k) {
        const int s = (int)(k % NS), sl = (int)(k % NT);
        if (!mbar_wait(&full[s], (uint32_t)((k / NS) & 1), abort, p.status, kWaitLimitNs)) break;
        if (!mbar_wait(&t_empty[sl], (uint32_t)(((k / NT) & 1) ^ 1), abort, p.status,
                       kWaitLimitNs))
          break;
        tc_fence_after();
        const uint32_t q_s = smem_u32(tiles + (s * 3 + 0) * tile_bytes);
        const uint32_t k_s = smem_u32(tiles + (s * 3 + 1) * tile_bytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_ss(tmem + sl * SC, desc_kmajor_tile<HD>(q_s, kk), desc_kmajor_tile<HD>(k_s, kk),
                  idesc_s, kk);
        umma_commit(&s_full[sl]);
      }
      if (*abort) {
        umma_commit(&drain[0]);
        mbar_drain(&drain[0], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == kMma2Warp) {
    if (lane == 0) {   // O = P V of every tile, as soon as its P is written
      constexpr uint32_t idesc_o = idesc_bf16(kRows, HD, 0, 1);
      for (long long k = 0; k < n_local; ++k) {
        const int s = (int)(k % NS), sl = (int)(k % NT);
        if (!mbar_wait(&p_full[sl], (uint32_t)((k / NT) & 1), abort, p.status, kWaitLimitNs))
          break;
        tc_fence_after();
        const uint32_t v_s = smem_u32(tiles + (s * 3 + 2) * tile_bytes);
        if constexpr (C::kTmemP) {
          // A = P from TMEM: 16 keys per step are 8 columns of bf16 pairs
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            umma_ts(tmem + sl * SC + C::kOCol, tmem + sl * SC + kk * 8,
                    desc_mnmajor_tile<HD>(v_s, kk), idesc_o, kk);
        } else {
          const uint32_t p_s = smem_u32(ptile + (k % kFwdPBufs) * 32768);
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            umma_ss(tmem + sl * SC, desc_p_kmajor(p_s, kk), desc_mnmajor_tile<HD>(v_s, kk),
                    idesc_o, kk);
        }
        umma_commit(&o_full[sl]);
        umma_commit(&empty[s]);
      }
      if (*abort) {
        umma_commit(&drain[1]);
        mbar_drain(&drain[1], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp < kNumWg * 4) {
    // Softmax / epilogue warpgroups: thread = tile row = TMEM lane.
    const int wg = warp >> 2;
    const int row = threadIdx.x & (kWg - 1);
    const int gw = row / N, lr = row - gw * N;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t p_s = C::kTmemP ? 0u : smem_u32(ptile + wg * 32768);
    long long k = wg;
    for (long long t = blockIdx.x + wg * (long long)gridDim.x; t < p.n_tiles;
         t += kNumWg * (long long)gridDim.x, k += kNumWg) {
      const int s = (int)(k % NS), sl = (int)(k % NT);
      const uint32_t phs = (uint32_t)((k / NS) & 1), pht = (uint32_t)((k / NT) & 1);
      const long long group = t / g.heads;
      const int h = (int)(t - group * g.heads);
      const long long win = group * G + gw;
      const bool plain = WW > 0 && window_plain(g, win);
      const RowInfo me = plain ? plain_row_info<WW>(g, win, lr) : row_info(g, win, lr);
      uint32_t* ci = colinfo + (wg * 2 + ((k / kNumWg) & 1)) * kRows;
      // A plain window reads no key words, so its two warps need no barrier;
      // the forward has no other warpgroup-wide barrier, so a warp may leave
      // on its own when a wait has run out.
      if (plain && *abort) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(&s_full[sl], pht, abort, p.status, kWaitLimitNs);
      mbar_wait(&full[s], phs, abort, p.status, kWaitLimitNs);
      if (!plain) {
        // key words of the window's rows, published to its two warps only
        // (written once S is ready: every thread of the warpgroup has then
        // read the previous words of this buffer, two tiles back)
        ci[row] = key_word(me);
        if (named_sync_or(1 + 2 * wg + gw, N, *abort)) break;
      }
      tc_fence_after();
      float x[N];
      tmem_load_cols<N>(tmem + lane_base + sl * SC + gw * N, x);
      tmem_wait_ld();
      const float* brow = bias + s * p.bins_pad;
      float m;
      if (plain)
        m = logits_plain<N, (WW > 0 ? WW : 8)>(x, brow + me.bias_base, p.scale_log2);
      else
        m = logits_general<N>(x, brow, ci + gw * N, me.bias_base, me.label, p.scale_log2);
      float l = 1.f;
      if (me.valid) {
        l = exp_sum<N>(x, m);
      } else {
#pragma unroll
        for (int j = 0; j < N; ++j) x[j] = 0.f;
      }
      if constexpr (C::kTmemP) {
        // this row's P as bf16 pairs over the tile's 128 keys: the other
        // window's 64 keys are zeros
        uint32_t w0[32], w1[32];   // columns 0-31 (keys 0-63), 32-63 (keys 64-127)
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const uint32_t w = pack_bf16(x[2 * c], x[2 * c + 1]);
          w0[c] = gw ? 0u : w;
          w1[c] = gw ? w : 0u;
        }
        __syncwarp();
        tmem_st32u(tmem + lane_base + sl * SC + 0, w0);
        tmem_st32u(tmem + lane_base + sl * SC + 32, w1);
        tmem_wait_st();
      } else {
        store_p_row<N>(p_s, row, gw * N, x);
        fence_proxy_async();
      }
      tc_fence_before();
      mbar_arrive(&p_full[sl]);
      // epilogue: O row from TMEM, normalised, straight to its grid token
      // (direct stores measured faster here than staging for a TMA store)
      mbar_wait(&o_full[sl], pht, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      {
        // (rows beyond the valid extent hold P = 0, so O = 0 is stored there)
        __nv_bfloat16* dst = (__nv_bfloat16*)(me.halo ? p.out0h : p.out0) +
                             (me.token * g.heads + h) * HD;
        constexpr int OC = HD > 64 ? 64 : HD;   // columns per TMEM read
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += OC) {
          float o[OC];
          tmem_load_cols<OC>(tmem + lane_base + sl * SC + C::kOCol + c0, o);
          tmem_wait_ld();
          if (c0 + OC == HD) {
            tc_fence_before();
            mbar_arrive(&t_empty[sl]);
          }
          if (me.stored && !*abort) store_row_bf16<OC>(dst + c0, o, 1.f / l);
        }
      }
      float* lse_out = me.halo ? p.lse_h : p.lse;
      if (me.stored && !*abort && lse_out)
        lse_out[me.token * g.heads + h] =
            me.valid ? (m + __log2f(l)) * 0.69314718055994531f : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================================
// Backward
// ================================================================================
// P and scale*dS feed the dV, dQ and dK products. Rounded to bf16 alone they
// would cost up to 2.5% of the output RMS on the largest gradients, so each is
// split into bf16 hi + lo parts (hi = x with the low 16 bits cleared, lo =
// bf16(x - hi); x = hi + lo to ~2^-16 relative) and both parts are accumulated
// in TMEM. The two windows of a tile never mix: each operand is two 64 x 64
// blocks (8 KB, 128-byte swizzle, 128-byte rows) plus shared zero blocks Z1,
// Z2, in this order:
//   [P0h][P0l][dS0h][Z1][dS1h][dS0l][Z2][dS1l][P1h][P1l]
// As a K-major A (dQ = dS K: rows = queries, K = keys) the key half 0 of dS is
// the 16 KB run [dS0 | Z] and the key half 1 is [Z | dS1]. As an MN-major A
// (dV = P^T dO, dK = dS^T Q: M = keys, K = queries) the second 64-key atom is
// addressed through the leading byte offset, so the query half 0 reads
// (X0, Z) and the query half 1 reads (Z, X1) for any X0 < Z < X1.
//
// Two warpgroups take alternate tiles, each with its own TMEM slot of 256
// columns (S | dP, then dV | dQ | dK). The operand blocks are shared: tile k
// writes them as soon as the gradient products of tile k-1 have completed
// (nothing else lives there), and each warpgroup stores its gradient rows
// straight from registers to their grid tokens. One thread issues S and dP of
// each tile as soon as its data and slot are ready, another the gradient
// products as soon as its blocks are written.
//
// Bias-table gradient: per tile, a bound on |dS| (max P of the row times
// max|dP| + |D|, maximised over the tile's rows) sets the exponent of an exact
// fixed-point sum in int32 shared bins; the tile's bins are then added into
// the wide integer sums of the workspace (dbias_fixed.cuh).
// HD <= 64: two input stages, two TMEM slots of 256 columns (S | dP, then
// dV | dQ | dK at 0 / 64 / 128), the two softmax warpgroups on alternate
// tiles. HD = 128: a stage of four 32 KB tiles leaves room for one, and the
// three 128-column gradients need
// 384 columns, so one slot (dV | dQ | dK at 0 / 128 / 256 over S | dP) and
// one softmax warpgroup.
// HD <= 64 also splits every row's 64 keys between two warpgroups (32 each):
// four softmax warpgroups, two per tile in flight, 20 warps at 96 registers a
// thread. The two halves of a row exchange their maxima, sums, D and max |dP|
// through TMEM columns of the other window's S, which that row never reads.
template <int HD>
struct BwdCfg {
  static constexpr bool kWide = HD > 64;
  static constexpr int kStages = kWide ? 1 : 2;
  static constexpr int kSlots = kWide ? 1 : 2;
  static constexpr int kWarpgroups = kWide ? 1 : kNumWg;    // tiles in flight
  static constexpr int kKeySplit = kWide ? 1 : 2;           // warpgroups per tile
  static constexpr int kSoftWg = kWarpgroups * kKeySplit;
  static constexpr int kProducer = kSoftWg > 2 ? kSoftWg * 4 : kProducerWarp;
  static constexpr int kMma = kProducer + 1, kMma2 = kProducer + 2, kFold = kProducer + 3;
  static constexpr int kThreads = (kProducer + 4) * 32;
  static constexpr int kColBufs = kKeySplit > 1 ? kWarpgroups : 2 * kWarpgroups;
  static constexpr uint32_t kGradCols = kWide ? 128 : 64;   // dV, dQ, dK spacing
};
constexpr uint32_t kBlk = 8192;
enum { kP0h = 0, kP0l, kS0h, kZ1, kS1h, kS0l, kZ2, kS1l, kP1h, kP1l, kNumBlk };

__device__ inline uint64_t desc_blk_kmajor(uint32_t base, int blk0, int blk1, int k16) {
  // keys [0,64) read the run starting at blk0, keys [64,128) the run at blk1
  const uint32_t start = base + (k16 < 4 ? blk0 : blk1) * kBlk + (k16 & 3) * 32;
  return smem_desc(start, 16, 1024, kSwizzle128);
}
__device__ inline uint64_t desc_blk_mnmajor(uint32_t base, int x0, int z, int x1, int k16) {
  // query half 0: atoms (x0, z); query half 1: atoms (z, x1)
  const int first = k16 < 4 ? x0 : z, second = k16 < 4 ? z : x1;
  const uint32_t start = base + first * kBlk + (k16 & 3) * 2048;
  return smem_desc(start, (uint32_t)(second - first) * kBlk, 1024, kSwizzle128);
}

// Columns [c0, c0 + NC) of row `lr` (0..63) of the hi and lo blocks of one
// operand, from NC fp32 values v[0..NC).
template <int NC>
__device__ inline void store_split_cols_part(uint32_t blk_hi, uint32_t blk_lo, int lr, int c0,
                                             const float* v) {
#pragma unroll
  for (int cc = 0; cc < NC / 8; ++cc) {
    const int c = c0 / 8 + cc;
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = make_float2(v[cc * 8 + 2 * e], v[cc * 8 + 2 * e + 1]);
      const uint32_t a = __float_as_uint(x.x), b = __float_as_uint(x.y);
      hw[e] = __byte_perm(a, b, 0x7632);   // the top 16 bits of each
      const float2 r = __ffma2_rn(make_float2(__uint_as_float(a & 0xFFFF0000u),
                                              __uint_as_float(b & 0xFFFF0000u)),
                                  make_float2(-1.f, -1.f), x);   // exact remainders
      lw[e] = pack_bf16(r.x, r.y);
    }
    const uint32_t off = lr * 128 + ((c ^ (lr & 7)) << 4);
    st_shared_v4(blk_hi + off, hw[0], hw[1], hw[2], hw[3]);
    st_shared_v4(blk_lo + off, lw[0], lw[1], lw[2], lw[3]);
  }
}

template <int HD, int WW>
__global__ void __launch_bounds__(BwdCfg<HD>::kThreads, 1)
    bwd_kernel(const __grid_constant__ FastParams p) {
  constexpr int N = 64, G = kRows / N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using C = BwdCfg<HD>;
  constexpr int NS = C::kStages, NT = C::kSlots, NWG = C::kWarpgroups;
  constexpr int KS = C::kKeySplit, SW = C::kSoftWg;
  constexpr int KN = 64 / KS;   // keys of a row each thread takes
  constexpr uint32_t GC = C::kGradCols;
  constexpr uint32_t tile_bytes = kRows * HD * 2;
  const Geo& g = p.g;
  const int bp = p.bins_pad;
  const Layout L = make_layout<HD, NS, 4, kNumBlk * kBlk, C::kColBufs, SW>(bp);
  uint8_t* tiles = smem + L.tiles;
  uint8_t* blocks = smem + L.ptile;
  float* bias = (float*)(smem + L.bias);
  uint32_t* colinfo = (uint32_t*)(smem + L.colinfo);
  int* bins = (int*)(smem + L.bins_w);               // [wg][warp][bins_pad] bins
  float* tbound = (float*)(bins + SW * 4 * bp);      // [wg][4] per-warp |dS| bounds
  uint64_t* bars = (uint64_t*)(smem + L.bars);
  uint64_t* full = bars;
  uint64_t* empty = full + NS;
  uint64_t* sdp_full = empty + NS;
  uint64_t* pds_full = sdp_full + NT;
  uint64_t* grad_full = pds_full + NT;
  uint64_t* t_empty = grad_full + NT;
  uint64_t* drain = t_empty + NT;   // [2]: one per MMA-issuing thread
  uint64_t* never = drain + 2;
  uint64_t* gradv_full = never + 1;          // [NT] dV products done
  uint64_t* bins_full = gradv_full + NT;     // [wg] a tile's bins are complete
  uint64_t* bins_empty = bins_full + NWG;    // [pair] ... and folded into global sums
  uint32_t* tmem_slot = (uint32_t*)(smem + L.misc);
  volatile int* abort = (volatile int*)(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_local = local_tiles(p.n_tiles, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < NT; ++i) {
      mbar_init(&sdp_full[i], 1); mbar_init(&pds_full[i], KS * kWg);
      mbar_init(&grad_full[i], 1); mbar_init(&t_empty[i], KS * kWg);
      mbar_init(&gradv_full[i], 1);
    }
    for (int i = 0; i < NWG; ++i) { mbar_init(&bins_full[i], KS * kWg); mbar_init(&bins_empty[i], 32); }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == C::kProducer && lane == 0)
    for (int tt = 0; tt < 4; ++tt)
      for (int m = 0; m < kMaxMaps; ++m) prefetch_tmap(&p.maps[tt][m]);
  for (uint32_t i = threadIdx.x; i < kBlk / 16; i += C::kThreads) {
    reinterpret_cast<uint4*>(blocks + kZ1 * kBlk)[i] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(blocks + kZ2 * kBlk)[i] = make_uint4(0, 0, 0, 0);
  }
  for (int i = threadIdx.x; i < SW * 4 * bp; i += C::kThreads) bins[i] = 0;
  fence_proxy_async();
  if (warp == C::kMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::kProducer) {
    if (lane == 0) {
      long long k = 0;
      for (long long t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++k) {
        const int s = (int)(k % NS);
        const uint32_t ph = (uint32_t)((k / NS) & 1);
        if (!mbar_wait(&empty[s], ph ^ 1, abort, p.status, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&full[s], 4 * tile_bytes + bp * 4);
        issue_tile_loads<HD, 4>(p, t, tiles + s * 4 * tile_bytes, bias + s * bp, &full[s]);
      }
      if (*abort) {
        const long long first = k > NS ? k - NS : 0;
        for (long long j = first; j < k; ++j)
          mbar_drain(&full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == C::kMma) {
    if (lane == 0) {   // S = Q K^T and dP = dO V^T of every tile
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kRows, 0, 0);
      for (long long k = 0; k < n_local; ++k) {
        const int s = (int)(k % NS), sl = (int)(k % NT);
        if (!mbar_wait(&full[s], (uint32_t)((k / NS) & 1), abort, p.status, kWaitLimitNs)) break;
        if (!mbar_wait(&t_empty[sl], (uint32_t)(((k / NT) & 1) ^ 1), abort, p.status,
                       kWaitLimitNs))
          break;
        tc_fence_after();
        const uint32_t q_s = smem_u32(tiles + (s * 4 + 0) * tile_bytes);
        const uint32_t k_s = smem_u32(tiles + (s * 4 + 1) * tile_bytes);
        const uint32_t v_s = smem_u32(tiles + (s * 4 + 2) * tile_bytes);
        const uint32_t do_s = smem_u32(tiles + (s * 4 + 3) * tile_bytes);
        const uint32_t d = tmem + sl * 256;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_ss(d, desc_kmajor_tile<HD>(q_s, kk), desc_kmajor_tile<HD>(k_s, kk), idesc_s, kk);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_ss(d + 128, desc_kmajor_tile<HD>(do_s, kk), desc_kmajor_tile<HD>(v_s, kk), idesc_s,
                  kk);
        umma_commit(&sdp_full[sl]);
      }
      if (*abort) {
        umma_commit(&drain[0]);
        mbar_drain(&drain[0], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == C::kMma2) {
    if (lane == 0) {   // dV, dQ, dK of every tile, once its operand blocks are written
      constexpr uint32_t idesc_t = idesc_bf16(kRows, HD, 1, 1);         // dV, dK: A = X^T
      constexpr uint32_t idesc_q = idesc_bf16(kRows, HD, 0, 1);         // dQ
      const uint32_t bb = smem_u32(blocks);
      // Operand descriptors for K-steps 0 and 4 (the two query / key halves);
      // steps 1-3 and 5-7 only move the start address, which sits in the
      // low 14 bits, so they are a small integer add.
      const uint64_t aPh[2] = {desc_blk_mnmajor(bb, kP0h, kZ1, kP1h, 0),
                               desc_blk_mnmajor(bb, kP0h, kZ1, kP1h, 4)};
      const uint64_t aPl[2] = {desc_blk_mnmajor(bb, kP0l, kZ1, kP1l, 0),
                               desc_blk_mnmajor(bb, kP0l, kZ1, kP1l, 4)};
      const uint64_t aQh[2] = {desc_blk_kmajor(bb, kS0h, kZ1, 0), desc_blk_kmajor(bb, kS0h, kZ1, 4)};
      const uint64_t aQl[2] = {desc_blk_kmajor(bb, kS0l, kZ2, 0), desc_blk_kmajor(bb, kS0l, kZ2, 4)};
      const uint64_t aKh[2] = {desc_blk_mnmajor(bb, kS0h, kZ1, kS1h, 0),
                               desc_blk_mnmajor(bb, kS0h, kZ1, kS1h, 4)};
      const uint64_t aKl[2] = {desc_blk_mnmajor(bb, kS0l, kZ2, kS1l, 0),
                               desc_blk_mnmajor(bb, kS0l, kZ2, kS1l, 4)};
      constexpr uint32_t kStepMN = 2048 >> 4, kStepK = 32 >> 4;
      constexpr uint32_t kStepB = (16 * TileGeom<HD>::kRowBytes) >> 4;
      for (long long k = 0; k < n_local; ++k) {
        const int s = (int)(k % NS), sl = (int)(k % NT);
        if (!mbar_wait(&pds_full[sl], (uint32_t)((k / NT) & 1), abort, p.status, kWaitLimitNs))
          break;
        tc_fence_after();
        const uint64_t bQ = desc_mnmajor_tile<HD>(smem_u32(tiles + (s * 4 + 0) * tile_bytes), 0);
        const uint64_t bK = desc_mnmajor_tile<HD>(smem_u32(tiles + (s * 4 + 1) * tile_bytes), 0);
        const uint64_t bO = desc_mnmajor_tile<HD>(smem_u32(tiles + (s * 4 + 3) * tile_bytes), 0);
        const uint32_t d = tmem + sl * 256;
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {  // dV = P^T dO  (hi, then lo)
          const uint32_t a = (kk & 3) * kStepMN, b = kk * kStepB;
          umma_ss(d + 0, aPh[kk >> 2] + a, bO + b, idesc_t, kk);
          umma_ss(d + 0, aPl[kk >> 2] + a, bO + b, idesc_t, 1);
        }
        umma_commit(&gradv_full[sl]);   // its rows can leave while dQ and dK run
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {  // dQ = dS K
          const uint32_t a = (kk & 3) * kStepK, b = kk * kStepB;
          umma_ss(d + GC, aQh[kk >> 2] + a, bK + b, idesc_q, kk);
          umma_ss(d + GC, aQl[kk >> 2] + a, bK + b, idesc_q, 1);
        }
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {  // dK = dS^T Q
          const uint32_t a = (kk & 3) * kStepMN, b = kk * kStepB;
          umma_ss(d + 2 * GC, aKh[kk >> 2] + a, bQ + b, idesc_t, kk);
          umma_ss(d + 2 * GC, aKl[kk >> 2] + a, bQ + b, idesc_t, 1);
        }
        umma_commit(&grad_full[sl]);
        umma_commit(&empty[s]);
      }
      if (*abort) {
        umma_commit(&drain[1]);
        mbar_drain(&drain[1], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == C::kFold) {
    // Each tile's bins, per warp, into the workspace's exact sums: the warps
    // of a window (two per warpgroup of the tile) add up (exact integers), in
    // the window's own unit.
    for (long long k = 0, t = blockIdx.x; k < n_local; ++k, t += gridDim.x) {
      const int wgk = (int)(k % NWG);
      if (!mbar_wait(&bins_full[wgk], (uint32_t)((k / NWG) & 1), abort, p.status, kWaitLimitNs))
        break;
      const int h = (int)(t - (t / g.heads) * g.heads);
      int* tbk = bins + wgk * KS * 4 * bp;
      const float* bk = tbound + wgk * KS * 4;   // (the key parts' bounds are equal)
      long long* acc = p.dt_acc + (size_t)h * bp * kLimbStride;
      for (int i = lane; i < 2 * g.bins; i += 32) {
        const int w2 = i >= g.bins;
        const int b = i - (w2 ? g.bins : 0);
        const float wbd = fmaxf(bk[2 * w2], bk[2 * w2 + 1]);
        const bool fin = wbd <= 3.0e38f;
        int v = 0;
#pragma unroll
        for (int kh = 0; kh < KS; ++kh) {
          int* b0 = tbk + (kh * 4 + 2 * w2) * bp + b;
          v += b0[0] + b0[bp];
          b0[0] = 0;
          b0[bp] = 0;
        }
        if (!fin) flag_nonfinite(acc + (size_t)b * kLimbStride);
        else if (v != 0) add_fixed(acc + (size_t)b * kLimbStride, v, tile_exponent(wbd));
      }
      mbar_arrive(&bins_empty[wgk]);
    }
  } else if (warp < SW * 4) {
    const int wgi = warp >> 2;       // softmax warpgroup
    const int wg = wgi / KS;         // tile pair: takes tiles wg, wg + NWG, ...
    const int kh = wgi - wg * KS;    // keys kh * KN .. kh * KN + KN - 1 of every row
    const int k0 = kh * KN;
    const int row = threadIdx.x & (kWg - 1);
    const int gw = row / N, lr = row - gw * N;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float dscale = p.scale_log2 * (1.0f / kLog2e);  // head_dim^-1/2
    const uint32_t bb = smem_u32(blocks);
    const uint32_t blk_ph = bb + (gw ? kP1h : kP0h) * kBlk, blk_pl = bb + (gw ? kP1l : kP0l) * kBlk;
    const uint32_t blk_sh = bb + (gw ? kS1h : kS0h) * kBlk, blk_sl = bb + (gw ? kS1l : kS0l) * kBlk;
    int* tb = bins + (wgi * 4 + (warp & 3)) * bp;   // this warp's bins
    float* bnd = tbound + wgi * 4;
    __nv_bfloat16* const outs[3] = {(__nv_bfloat16*)p.out2, (__nv_bfloat16*)p.out0,
                                    (__nv_bfloat16*)p.out1};   // TMEM order: dV, dQ, dK
    __nv_bfloat16* const outs_h[3] = {(__nv_bfloat16*)p.out2h, (__nv_bfloat16*)p.out0h,
                                      (__nv_bfloat16*)p.out1h};
    long long k = wg;
    for (long long t = blockIdx.x + wg * (long long)gridDim.x; t < p.n_tiles;
         t += NWG * (long long)gridDim.x, k += NWG) {
      const int s = (int)(k % NS), sl = (int)(k % NT);
      const uint32_t phs = (uint32_t)((k / NS) & 1), pht = (uint32_t)((k / NT) & 1);
      const long long group = t / g.heads;
      const int h = (int)(t - group * g.heads);
      const long long win = group * G + gw;
      const bool plain = WW > 0 && window_plain(g, win);
      const RowInfo me = plain ? plain_row_info<WW>(g, win, lr) : row_info(g, win, lr);
      // key words: one buffer per tile pair when the keys are split (the
      // exchange barrier below keeps a fast warp's next words behind every
      // read of these), two otherwise
      uint32_t* ci = colinfo + (KS > 1 ? wg : (wg * 2 + (int)((k / NWG) & 1))) * kRows;
      if (kh == 0) ci[row] = key_word(me);
      if (named_sync_or(1 + wg, KS * kWg, *abort)) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(&sdp_full[sl], pht, abort, p.status, kWaitLimitNs);
      mbar_wait(&full[s], phs, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      // S row -> P (registers) -> D from dP; P back into its S columns; dS and
      // the bias-gradient bins from P and dP chunks; scale * dS into the dP
      // columns. All of this runs before the shared operand blocks are free.
      float x[KN];
      const uint32_t s_col = tmem + lane_base + sl * 256 + gw * N + k0;
      const uint32_t dp_col = s_col + 128;
      // (exchange columns: the other window's S in this row's lane)
      const uint32_t x_col = tmem + lane_base + sl * 256 + (1 - gw) * N;
      tmem_load_cols<KN>(s_col, x);
      tmem_wait_ld();
      const float* brow = bias + s * bp;
      const uint32_t* cw = ci + gw * N + k0;
      float m;
      if (plain)
        m = logits_plain<KN, (WW > 0 ? WW : 8)>(x, brow + me.bias_base - plain_off<(WW > 0 ? WW : 8)>(k0),
                                                p.scale_log2);
      else
        m = logits_general<KN>(x, brow, cw, me.bias_base, me.label, p.scale_log2);
      if constexpr (KS > 1) {   // the row's maximum over both key parts
        tmem_st4(x_col + 4 * kh, m, 0.f, 0.f, 0.f);
        tmem_wait_st();
        tc_fence_before();
        named_sync(1 + wg, KS * kWg);
        tc_fence_after();
        float o4[4];
        tmem_ld4(x_col + 4 * (1 - kh), o4);
        tmem_wait_ld();
        m = fmaxf(m, o4[0]);
      }
      // 2^(x - m) (unnormalised), then D = (sum 2^(x - m) dP) / l, max |dP|
      float l = 0.f;
      if (me.valid) {
        l = exp_sum<KN>(x, m);
      } else {
#pragma unroll
        for (int j = 0; j < KN; ++j) x[j] = 0.f;
      }
      // TMEM loads are warp-collective: every lane runs them, valid row or not
      // (x = 0 on invalid rows, so D = 0 and dS = 0 there).
      float2 dda = make_float2(0.f, 0.f), ddb = make_float2(0.f, 0.f);   // keys j mod 4
      float mdp = 0.f;
      {
        float dp[KN];
        tmem_load_cols<KN>(dp_col, dp);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < KN; j += 4) {
          dda = __ffma2_rn(make_float2(x[j], x[j + 1]), make_float2(dp[j], dp[j + 1]), dda);
          ddb = __ffma2_rn(make_float2(x[j + 2], x[j + 3]), make_float2(dp[j + 2], dp[j + 3]), ddb);
          mdp = fmaxf(mdp, fmaxf(fmaxf(fabsf(dp[j]), fabsf(dp[j + 1])),
                                 fmaxf(fabsf(dp[j + 2]), fabsf(dp[j + 3]))));
        }
      }
      float d = (dda.x + dda.y) + (ddb.x + ddb.y);
      if constexpr (KS > 1) {   // sums and max |dP| over both key parts
        tmem_st4(x_col + 8 + 4 * kh, l, d, mdp, 0.f);
        tmem_wait_st();
        tc_fence_before();
        named_sync(1 + wg, KS * kWg);
        tc_fence_after();
        float o4[4];
        tmem_ld4(x_col + 8 + 4 * (1 - kh), o4);
        tmem_wait_ld();
        l += o4[0];
        d += o4[1];
        mdp = fmaxf(mdp, o4[2]);
      }
      const float inv = me.valid ? 1.f / l : 0.f;   // max_j P_ij (= 1 / row sum); 0 on pad rows
      const float D = d * inv;
#pragma unroll
      for (int j = 0; j < KN; j += 2) {
        const float2 pj = __fmul2_rn(make_float2(x[j], x[j + 1]), make_float2(inv, inv));
        x[j] = pj.x;
        x[j + 1] = pj.y;
      }
      __syncwarp();
#pragma unroll
      for (int c = 0; c < KN / 32; ++c) tmem_st32(s_col + 32 * c, x + 32 * c);
      // The bins and bounds are free once the fold warp has taken this
      // tile pair's previous tile.
      if (k >= NWG)
        mbar_wait(&bins_empty[wg], (uint32_t)(((k / NWG) - 1) & 1), abort, p.status,
                  kWaitLimitNs);
      // |dS_ij| = P_ij |dP_ij - D| <= max_j P_ij * (max_j |dP_ij| + |D|); a NaN
      // becomes +inf here, since fmaxf would drop it (both key parts of a row
      // compute the same bound)
      {
        float rb = inv * (mdp + fabsf(D));
        if (!(rb <= 3.0e38f)) rb = INFINITY;
        const float wb = warp_max(rb);
        if (lane == 0) bnd[warp & 3] = wb;
      }
      named_sync(3 + wgi, kWg);
      // Each window has its own unit (warps 2gw and 2gw+1 hold its rows), so
      // its integer sums do not depend on which window shares its tile.
      const float win_bound = fmaxf(bnd[2 * gw], bnd[2 * gw + 1]);
      const bool finite = win_bound <= 3.0e38f;   // false for NaN and infinity
      const int E = tile_exponent(finite ? win_bound : 0.f);
      const float qs = exp2_int(E);
      tmem_wait_st();
      int* bq = tb + me.bias_base - (plain ? plain_off<(WW > 0 ? WW : 8)>(k0) : 0);
#pragma unroll 1
      for (int c = 0; c < KN / 32; ++c) {
        float ds[32], pc[32];
        __syncwarp();
        tmem_ld32(dp_col + 32 * c, ds);
        tmem_ld32(s_col + 32 * c, pc);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 2) {   // dS (0 off the row)
          const float2 v = __fmul2_rn(make_float2(pc[j], pc[j + 1]),
                                      __fadd2_rn(make_float2(ds[j], ds[j + 1]), make_float2(-D, -D)));
          ds[j] = v.x;
          ds[j + 1] = v.y;
        }
        if (me.valid && finite) {
          // bias-gradient bins: integers in units of 2^-E; integer adds
          // commute, so the sums do not depend on the order the lanes land in
          // (unrolled: a runtime index would put ds in local memory)
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            // ds * 2^E is exact, so one fused multiply-add rounds it to an integer
            const float2 q = __ffma2_rn(make_float2(ds[j], ds[j + 1]), make_float2(qs, qs),
                                        make_float2(12582912.0f, 12582912.0f));
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int off = plain ? plain_off<(WW > 0 ? WW : 8)>(32 * c + j + e)
                                    : (int)(lds_u32(cw + 32 * c + j + e) & 0xFFFF);
              red_add_s32(bq - off, __float_as_int(e ? q.y : q.x) - 0x4B400000);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 v = __fmul2_rn(make_float2(ds[j], ds[j + 1]), make_float2(dscale, dscale));
          ds[j] = v.x;
          ds[j + 1] = v.y;
        }
        __syncwarp();
        tmem_st32(dp_col + 32 * c, ds);
      }
      tmem_wait_st();
      mbar_arrive(&bins_full[wg]);   // the fold warp adds them to the global sums
      // The operand blocks are free once the previous tile's gradient
      // products have completed (grad_full of the other slot; this warpgroup
      // saw that barrier's phase before, two tiles ago, so the parity names
      // exactly the phase of tile k-1).
      if (k > 0)
        mbar_wait(&grad_full[(k - 1) % NT], (uint32_t)(((k - 1) / NT) & 1), abort, p.status,
                  kWaitLimitNs);
#pragma unroll 1
      for (int c = 0; c < KN / 32; ++c) {
        float pc[32], ds[32];
        __syncwarp();
        tmem_ld32(s_col + 32 * c, pc);
        tmem_ld32(dp_col + 32 * c, ds);
        tmem_wait_ld();
        store_split_cols_part<32>(blk_ph, blk_pl, lr, k0 + 32 * c, pc);
        store_split_cols_part<32>(blk_sh, blk_sl, lr, k0 + 32 * c, ds);
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&pds_full[sl]);
      // epilogue: dV (as soon as its products are done), then dQ and dK,
      // from TMEM to their grid tokens in whole-row stores (zero rows beyond
      // the valid extent); each key part stores its own HD / KS columns
      constexpr int HC = HD / KS;               // columns of each output this thread stores
      constexpr int OC = HC > 64 ? 64 : HC;     // columns per TMEM read
      const int c_lo = kh * HC;
      const bool st_row = me.stored && !*abort;
      const long long roff = (me.token * g.heads + h) * HD;
      auto store_part = [&](int part, int c0) {
        float o[OC];
        if constexpr (OC == 16) {
          __syncwarp();
          tmem_ld16(tmem + lane_base + sl * 256 + part * GC + c0, o);
        } else {
          tmem_load_cols<OC>(tmem + lane_base + sl * 256 + part * GC + c0, o);
        }
        tmem_wait_ld();
        if (part == 2 && c0 + OC == c_lo + HC) {
          tc_fence_before();
          mbar_arrive(&t_empty[sl]);
        }
        store_rows_bf16<OC>(o, 1.f, st_row ? (const void*)((me.halo ? outs_h[part] : outs[part]) +
                                                            roff + c0)
                                           : nullptr);
      };
      mbar_wait(&gradv_full[sl], pht, abort, p.status, kWaitLimitNs);
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < HC; c0 += OC) store_part(0, c_lo + c0);
      mbar_wait(&grad_full[sl], pht, abort, p.status, kWaitLimitNs);
      tc_fence_after();
#pragma unroll
      for (int part = 1; part < 3; ++part)
#pragma unroll
        for (int c0 = 0; c0 < HC; c0 += OC) store_part(part, c_lo + c0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::kMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================================
// Layout stage as the kernels above run it, for bit-exact checks
// ================================================================================
// ids[token, h, :] holds (token + 1) in its first two 16-bit words and h in
// the third; all else is zero, so a pad slot (TMA zero fill) reads id 0.
__global__ void layout_ids_kernel(Geo g, uint16_t* ids) {
  const long long rows = (long long)g.B * g.H * g.W * g.heads;
  for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < rows;
       r += (long long)gridDim.x * blockDim.x) {
    const long long token = r / g.heads;
    const int h = (int)(r - token * g.heads);
    uint16_t* row = ids + r * g.hd;
    const unsigned long long id = (unsigned long long)token + 1;
    for (int e = 0; e < g.hd; ++e)
      row[e] = e == 0 ? (uint16_t)(id & 0xFFFF) : e == 1 ? (uint16_t)(id >> 16) : e == 2 ? (uint16_t)h : 0;
  }
}

// One CTA per tile: the producer's TMA boxes of tile t land in shared memory
// exactly as in the forward and backward; thread r reads tile row r and
// writes, at the slot that row_slot gives for it, the token it holds (-1 for
// a zero-filled pad row) and the row's shift-region label. A disagreement
// with row_info (validity, token) or with the plain-window row info, or a
// row whose head word is not the tile's head, is written as -2.
template <int HD>
__global__ void __launch_bounds__(kRows) layout_map_kernel(const __grid_constant__ FastParams p,
                                                           int32_t* map, int32_t* labels) {
  constexpr uint32_t row_bytes = TileGeom<HD>::kRowBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tile = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full;
  __shared__ int status;
  __shared__ int abort_flag;
  const Geo& g = p.g;
  const long long t = blockIdx.x;
  if (threadIdx.x == 0) {
    mbar_init(&full, 1);
    status = 0;
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&full, kRows * HD * 2);
    issue_tile_loads<HD, 1>(p, t, tile, nullptr, &full);
  }
  const bool ok = mbar_wait(&full, 0, (volatile int*)&abort_flag, &status, kWaitLimitNs);
  if (!ok) mbar_drain(&full, 0, kWaitLimitNs);
  const int G = kRows / g.N;
  const int r = threadIdx.x, gw = r / g.N, lr = r - gw * g.N;
  const long long group = t / g.heads;
  const int h = (int)(t - group * g.heads);
  const long long win = group * G + gw;
  if (win >= g.n_win || h != g.heads - 1) return;   // the last head exercises the head coordinate
  const uint32_t row_addr = smem_u32(tile) + r * row_bytes;
  const uint32_t swz = HD >= 64 ? ((row_addr >> 7) & 7) : ((row_addr >> 7) & 3);
  const uint16_t* w = (const uint16_t*)(tile + r * row_bytes + (swz << 4));
  const unsigned id = (unsigned)w[0] | ((unsigned)w[1] << 16);
  int b, wy, wx, iy, ix;
  window_coords(g, win, b, wy, wx);
  row_slot(g, wy, wx, lr, iy, ix);
  const RowInfo ri = row_info(g, win, lr);
  int32_t out = (id == 0 || !ri.valid) ? -1 : (int32_t)(id - 1);
  if (!ok || (id != 0) != ri.stored || (ri.stored && (long long)(id - 1) != ri.token) ||
      (id != 0 && w[2] != (uint16_t)h))
    out = -2;
  if (g.wh == 8 && g.ww == 8 && window_plain(g, win)) {
    const RowInfo pi = plain_row_info<8>(g, win, lr);
    if (pi.token != ri.token || pi.bias_base != ri.bias_base || pi.key_off != ri.key_off ||
        pi.label != ri.label || !ri.valid)
      out = -2;
  }
  const long long at = win * g.N + iy * g.ww + ix;
  map[at] = out;
  if (labels) labels[at] = ri.label;
}

template <int HD>
size_t fwd_smem(const Geo& g) {
  using C = FwdCfg<HD>;
  return make_layout<HD, C::kStages, 3, C::kPBytes>(bins_padded(g.bins)).total + 1024;
}
template <int HD>
size_t bwd_smem(const Geo& g) {
  using C = BwdCfg<HD>;
  return make_layout<HD, C::kStages, 4, kNumBlk * kBlk, C::kColBufs, C::kSoftWg>(
             bins_padded(g.bins)).total +
         1024;
}
size_t fwd_smem_any(const Geo& g) {
  return g.hd == 128 ? fwd_smem<128>(g) : g.hd == 64 ? fwd_smem<64>(g) : fwd_smem<32>(g);
}
size_t bwd_smem_any(const Geo& g) {
  return g.hd == 128 ? bwd_smem<128>(g) : g.hd == 64 ? bwd_smem<64>(g) : bwd_smem<32>(g);
}

bool smem_ok(const Geo& g) {
  return fwd_smem_any(g) <= kSmemLimit && bwd_smem_any(g) <= kSmemLimit;
}


}  // namespace

bool fast_supported(const Geo& g, int dtype) {
  if (dtype != SWIN_DTYPE_BF16) return false;
  if (g.hd != 64 && g.hd != 32 && g.hd != 128) return false;
  if (g.N != 64) return false;
  // Every sub-box must be a whole number of 8-row swizzle atoms.
  const int ylen[3] = {g.wh, g.wh - g.sh, g.sh};
  const int xlen[3] = {g.ww, g.ww - g.sw, g.sw};
  for (int a = 0; a < 3; ++a)
    for (int c = 0; c < 3; ++c) {
      if ((a > 0 && g.sh == 0) || (c > 0 && g.sw == 0)) continue;
      if ((ylen[a] * xlen[c]) % 8) return false;
    }
  if (g.bins > 0xFFFF) return false;
  return smem_ok(g);
}

// Workspace: header (status word), bias table [heads][bins_pad] fp32, and the
// exact bias-gradient sums [heads][bins_pad][kLimbStride] int64.
size_t fast_workspace(const Geo& g) {
  const int bp = bins_padded(g.bins);
  return kWsHeader + align256((size_t)g.heads * bp * 4) + align256(dbias_fixed_bytes(g));
}

cudaError_t fast_forward(const Geo& g, const void* q, const void* k, const void* v,
                         const float* table, void* out, float* lse, void* ws, int flags,
                         cudaStream_t st, const swin_wattn_halo* halo) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  static thread_local FastParams p;
  fill_common(p, g, bias_t, (int*)ws, flags);
  p.out0 = out;
  p.lse = lse;
  if (g.band) {
    p.out0h = halo->out;
    p.lse_h = lse ? halo->lse : nullptr;
  }
  if (!encode_maps(p, 0, q, g.band ? halo->q : nullptr) ||
      !encode_maps(p, 1, k, g.band ? halo->k : nullptr) ||
      !encode_maps(p, 2, v, g.band ? halo->v : nullptr))
    return cudaErrorInvalidValue;
  cudaError_t e = prep_bias(g, table, bias_t, nullptr, st);
  if (e != cudaSuccess) return e;
  const bool w8 = g.wh == 8 && g.ww == 8;
  const size_t smem = fwd_smem_any(g);
  if (g.hd == 128)
    return w8 ? launch(fwd_kernel<128, 8>, p, smem, st) : launch(fwd_kernel<128, 0>, p, smem, st);
  if (g.hd == 64)
    return w8 ? launch(fwd_kernel<64, 8>, p, smem, st) : launch(fwd_kernel<64, 0>, p, smem, st);
  return w8 ? launch(fwd_kernel<32, 8>, p, smem, st) : launch(fwd_kernel<32, 0>, p, smem, st);
}

cudaError_t fast_backward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, const void* dout, void* dq, void* dk, void* dv,
                          float* dtable, void* ws, int flags, cudaStream_t st,
                          const swin_wattn_halo* halo) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  long long* dt_acc = (long long*)((char*)ws + dbias_fixed_offset(g));
  static thread_local FastParams p;
  fill_common(p, g, bias_t, (int*)ws, flags);
  p.out0 = dq;
  p.out1 = dk;
  p.out2 = dv;
  p.dt_acc = dt_acc;
  if (g.band) {
    p.out0h = halo->dq;
    p.out1h = halo->dk;
    p.out2h = halo->dv;
  }
  if (!encode_maps(p, 0, q, g.band ? halo->q : nullptr) ||
      !encode_maps(p, 1, k, g.band ? halo->k : nullptr) ||
      !encode_maps(p, 2, v, g.band ? halo->v : nullptr) ||
      !encode_maps(p, 3, dout, g.band ? halo->dout : nullptr))
    return cudaErrorInvalidValue;
  cudaError_t e = prep_bias(g, table, bias_t, dt_acc, st);
  if (e != cudaSuccess) return e;
  const size_t smem = bwd_smem_any(g);
  const bool w8 = g.wh == 8 && g.ww == 8;
  if (g.hd == 128)
    e = w8 ? launch(bwd_kernel<128, 8>, p, smem, st, BwdCfg<128>::kThreads)
           : launch(bwd_kernel<128, 0>, p, smem, st, BwdCfg<128>::kThreads);
  else if (g.hd == 64)
    e = w8 ? launch(bwd_kernel<64, 8>, p, smem, st, BwdCfg<64>::kThreads)
           : launch(bwd_kernel<64, 0>, p, smem, st, BwdCfg<64>::kThreads);
  else
    e = w8 ? launch(bwd_kernel<32, 8>, p, smem, st, BwdCfg<32>::kThreads)
           : launch(bwd_kernel<32, 0>, p, smem, st, BwdCfg<32>::kThreads);
  if (e != cudaSuccess) return e;
  if (flags & SWIN_FLAG_DBIAS_SUMS) return cudaSuccess;   // the caller finishes the sums
  return finish_dbias(g, dt_acc, dtable, st);
}

cudaError_t fast_layout_map(const Geo& g, void* ids, int32_t* map, int32_t* labels,
                            cudaStream_t st) {
  static thread_local FastParams p;
  fill_common(p, g, nullptr, nullptr, 0);
  if (!encode_maps(p, 0, ids)) return cudaErrorInvalidValue;
  const long long rows = (long long)g.B * g.H * g.W * g.heads;
  const int blocks = (int)((rows + 255) / 256 < 4096 ? (rows + 255) / 256 : 4096);
  layout_ids_kernel<<<blocks, 256, 0, st>>>(g, (uint16_t*)ids);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)kRows * g.hd * 2 + 1024;
  if (g.hd == 128) {
    e = cudaFuncSetAttribute(layout_map_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    layout_map_kernel<128><<<(unsigned)p.n_tiles, kRows, smem, st>>>(p, map, labels);
  } else if (g.hd == 64) {
    e = cudaFuncSetAttribute(layout_map_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    layout_map_kernel<64><<<(unsigned)p.n_tiles, kRows, smem, st>>>(p, map, labels);
  } else {
    e = cudaFuncSetAttribute(layout_map_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    layout_map_kernel<32><<<(unsigned)p.n_tiles, kRows, smem, st>>>(p, map, labels);
  }
  note_launch();
  return cudaGetLastError();
}

}  // namespace swin
