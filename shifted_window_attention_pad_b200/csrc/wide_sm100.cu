// wide_sm100.cu -- tcgen05 / TMA kernels for 256-token windows (e.g. 16 x 16).
//
// Same operation as fast_sm100.cu -- shifted-window multi-head self-attention
// over a padded token grid (TERRA page, Abstract: window-based Swin Transformer
// with shifted-window execution; Table I: the padded resolution H^ x W^) --
// for windows of 256 tokens, the downsampled stage of the hierarchy (16 x 16
// windows on the 128 x 272 grid). A window's 256 query rows are two 128-row
// halves, one per softmax warpgroup; each half's row holds all 256 keys:
//  * one input stage per (window, head): Q, K, V as 256-row TMA boxes (up to
//    2 x 2 sub-boxes on the wrap seam, the same planning as the 64-token
//    kernels), plus the head's bias row;
//  * S of a half = Q_half K^T, M = 128, N = 256, fp32 in 256 TMEM columns of the
//    half's slot. The softmax reads S twice in chunks of 32 columns: the first
//    pass adds the bias, applies the pad / shift-region mask, writes the logits
//    back and takes the row maximum; the second exponentiates, sums, and writes
//    P as bf16 pairs over columns 0-127 of the slot (each pair lands on columns
//    already read);
//  * O = P V takes P as its A operand from TMEM (M = 128, N = head_dim,
//    K = 256) into columns 128.. of the slot, and the epilogue normalises and
//    stores each row at its grid token.
// Warp roles: warps 0-3 and 4-7 the softmax warpgroups of halves 0 and 1,
// warp 8 the TMA producer, warp 9 issues S (and owns TMEM), warp 10 issues
// O = P V. Persistent grid of one CTA per SM; (window, head) items round-robin,
// head fastest. Every mbarrier wait is bounded (%globaltimer); a wait that runs
// out records a timeout in the workspace status word, and the kernel drains its
// copies and MMAs and frees TMEM before returning.
#include "fast_common.cuh"

namespace swin {
namespace {

using namespace ptx;

constexpr int kKeys = 256;                 // tokens of a window = keys of every row
constexpr int kHalves = kKeys / kRows;     // query halves per window
// Forward warps: four softmax warpgroups (query half hf, key half kh =
// warpgroup >> 1, & 1), the TMA producer, the S issuer, the O issuer: 19
// warps, 96 registers a thread.
constexpr int kWideFwdWg = 4;
constexpr int kWideThreads = (kWideFwdWg * 4 + 3) * 32;
constexpr int kWideFwdProducer = kWideFwdWg * 4, kWideFwdMma = kWideFwdProducer + 1,
              kWideFwdMma2 = kWideFwdProducer + 2;
constexpr uint32_t kSlotColsW = 256;       // TMEM columns of one half

template <int HD>
struct WideFwdCfg {
  static constexpr uint32_t kRowBytes = HD * 2;
  static constexpr uint32_t kTileBytes = kKeys * kRowBytes;   // one tensor of one item
  static constexpr int kStages = HD > 32 ? 2 : 4;
  static constexpr uint32_t kOCol = 64;                        // O inside a half's slot
};

struct WideLayout {
  uint32_t tiles, bias, colinfo, xch, bars, misc, total;
};

// NS stages of three [256][HD] tiles (Q, K, V), the stages' bias rows, per
// query half two buffers of 256 key words, the row maxima and sums the two
// key-half warpgroups of a row exchange ([max, sum][half][key half][row]),
// mbarriers, two words.
template <int HD>
__host__ __device__ inline WideLayout wide_fwd_layout(int bins_pad) {
  using C = WideFwdCfg<HD>;
  WideLayout L;
  L.tiles = 0;
  L.bias = L.tiles + C::kStages * 3 * C::kTileBytes;
  L.colinfo = L.bias + ((C::kStages * bins_pad * 4 + 15) & ~15);
  L.xch = L.colinfo + kHalves * 2 * kKeys * 4;
  L.bars = (L.xch + 2 * kHalves * 2 * kRows * 4 + 7) & ~7u;
  L.misc = L.bars + 8 * 32;
  L.total = L.misc + 16;
  return L;
}

// K-major operand of [rows][HD] bf16 (128-byte swizzle at HD 64, 64-byte at 32),
// K step k16 of 16 channels.
template <int HD>
__device__ inline uint64_t wdesc_kmajor(uint32_t base, int k16) {
  constexpr uint32_t sw = HD >= 64 ? kSwizzle128 : kSwizzle64;
  return smem_desc(base + k16 * 32, 16, 8 * HD * 2, sw);
}
// MN-major operand (HD columns are N), K = rows, 16 rows per step.
template <int HD>
__device__ inline uint64_t wdesc_mnmajor(uint32_t base, int k16) {
  constexpr uint32_t sw = HD >= 64 ? kSwizzle128 : kSwizzle64;
  return smem_desc(base + k16 * 16 * HD * 2, 8 * HD * 2, 8 * HD * 2, sw);
}

// Producer: every TMA copy of item t (window, head) into one stage: the NTEN
// tensors' 256-row tiles, sub-box by sub-box in slot order, and the bias row.
template <int HD, int NTEN>
__device__ inline void issue_item_loads(const FastParams& p, long long t, uint8_t* tiles,
                                        float* bias_dst, uint64_t* full) {
  const Geo& g = p.g;
  const long long win = t / g.heads;
  const int h = (int)(t - win * g.heads);
  constexpr uint32_t row_bytes = HD * 2, tile_bytes = kKeys * row_bytes;
  int b, wy, wx;
  window_coords(g, win, b, wy, wx);
  SubBox sb[4];
  const int n = plan_window(g, wy, wx, sb);
  for (int i = 0; i < n; ++i)
    for (int tt = 0; tt < NTEN; ++tt)
      tma_load_5d(tiles + tt * tile_bytes + sb[i].row_off * row_bytes, &p.maps[tt][sb[i].map_id],
                  full, 0, h, sb[i].x, sb[i].y, b);
  if (bias_dst) bulk_load(bias_dst, p.bias_t + (size_t)h * p.bins_pad, p.bins_pad * 4, full);
}

// Logits (log2 units) of 32 keys k0.. of this row, in place: plain window
// (compile-time bias offsets for WW x WW windows) or general (per-key words:
// bias offset and region, 15 = pad key). Returns the chunk maximum.
// (k0 a multiple of WW: the chunk starts a window row, so its offsets are
// compile-time constants past the row's own.)
template <int WW>
__device__ inline float chunk_logits_plain(float* x, const float* bias_q, int k0, float c) {
  static_assert(WW > 0 && 32 % WW == 0 || WW % 32 == 0, "chunks start window rows");
  bias_q -= (k0 / WW) * (2 * WW - 1) + k0 % WW;
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float2 v = __ffma2_rn(make_float2(x[j], x[j + 1]), make_float2(c, c),
                                make_float2(bias_q[-plain_off<WW>(j)], bias_q[-plain_off<WW>(j + 1)]));
    x[j] = v.x;
    x[j + 1] = v.y;
    m0 = fmaxf(m0, v.x);
    m1 = fmaxf(m1, v.y);
  }
  return fmaxf(m0, m1);
}

// Pass 1 over the 128 keys k0base .. k0base + 127 of a row (32 at a time):
// logits (scale, bias, mask) written back over S in TMEM; returns their
// maximum.
template <bool PLAIN, int WW>
__device__ inline float wide_pass1(uint32_t slot, int k0base, const float* brow,
                                   const uint32_t* ci, const RowInfo& me, float c) {
  float m = -INFINITY;
#pragma unroll 1
  for (int k0 = k0base; k0 < k0base + kRows; k0 += 32) {
    float x[32];
    __syncwarp();
    tmem_ld32(slot + k0, x);
    tmem_wait_ld_regs(x);
    float cm;
    if constexpr (PLAIN)
      cm = chunk_logits_plain<WW>(x, brow + me.bias_base, k0, c);
    else
      cm = logits_general<32>(x, brow, ci + k0, me.bias_base, me.label, c);
    m = fmaxf(m, cm);
    __syncwarp();
    tmem_st32(slot + k0, x);
  }
  return m;
}

// Pass 2 over the same keys: P = 2^(x - mo) as bf16 pairs, the pair of keys
// k0base + 2c, + 1 in column k0base + c (keys 32 i .. 32 i + 31 of the half
// give columns 16 i .. 16 i + 15, whose logits were read before they are
// overwritten); returns the sum.
__device__ inline float wide_pass2(uint32_t slot, int k0base, float mo) {
  float l = 0.f;
#pragma unroll 1
  for (int i = 0; i < kRows / 32; ++i) {
    float x[32];
    __syncwarp();
    tmem_ld32(slot + k0base + 32 * i, x);
    tmem_wait_ld_regs(x);
    uint32_t w[16];
    float2 l2 = make_float2(0.f, 0.f);
    const float2 nm = make_float2(-mo, -mo);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 t = __fadd2_rn(make_float2(x[2 * j], x[2 * j + 1]), nm);
      const float2 e = make_float2(ex2(t.x), ex2(t.y));
      l2 = __fadd2_rn(l2, e);
      w[j] = pack_bf16(e.x, e.y);
    }
    l += l2.x + l2.y;
    __syncwarp();
    tmem_st16u(slot + k0base + 16 * i, w);
  }
  return l;
}

template <int HD, int WW>
__global__ void __launch_bounds__(kWideThreads, 1)
    wide_fwd_kernel(const __grid_constant__ FastParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using C = WideFwdCfg<HD>;
  constexpr int NS = C::kStages;
  constexpr uint32_t tile_bytes = C::kTileBytes;
  const Geo& g = p.g;
  const WideLayout L = wide_fwd_layout<HD>(p.bins_pad);
  uint8_t* tiles = smem + L.tiles;
  float* bias = (float*)(smem + L.bias);
  uint32_t* colinfo = (uint32_t*)(smem + L.colinfo);
  float* xch = (float*)(smem + L.xch);
  uint64_t* bars = (uint64_t*)(smem + L.bars);
  uint64_t* full = bars;
  uint64_t* empty = full + NS;
  uint64_t* s_full = empty + NS;      // [kHalves]
  uint64_t* p_full = s_full + kHalves;
  uint64_t* o_full = p_full + kHalves;
  uint64_t* t_empty = o_full + kHalves;
  uint64_t* drain = t_empty + kHalves;   // [2]: one per MMA-issuing thread
  uint64_t* never = drain + 2;
  uint32_t* tmem_slot = (uint32_t*)(smem + L.misc);
  volatile int* abort = (volatile int*)(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_local = local_tiles(p.n_tiles, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < kHalves; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 2 * kWg);
      mbar_init(&o_full[i], 1); mbar_init(&t_empty[i], 2 * kWg);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kWideFwdProducer && lane == 0)
    for (int tt = 0; tt < 3; ++tt)
      for (int m = 0; m < kMaxMaps; ++m) prefetch_tmap(&p.maps[tt][m]);
  if (warp == kWideFwdMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWideFwdProducer) {
    if (lane == 0) {
      long long k = 0;
      for (long long t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++k) {
        const int s = (int)(k % NS);
        const uint32_t ph = (uint32_t)((k / NS) & 1);
        if (!mbar_wait(&empty[s], ph ^ 1, abort, p.status, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&full[s], 3 * tile_bytes + p.bins_pad * 4);
        issue_item_loads<HD, 3>(p, t, tiles + s * 3 * tile_bytes, bias + s * p.bins_pad,
                                &full[s]);
      }
      if (*abort) {  // let copies already in flight land before the CTA leaves
        const long long first = k > NS ? k - NS : 0;
        for (long long j = first; j < k; ++j)
          mbar_drain(&full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == kWideFwdMma) {
    if (lane == 0) {   // S = Q_half K^T of both halves of every item
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kKeys, 0, 0);
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        const int s = (int)(k % NS);
        if (!mbar_wait(&full[s], (uint32_t)((k / NS) & 1), abort, p.status, kWaitLimitNs)) break;
        const uint32_t q_s = smem_u32(tiles + (s * 3 + 0) * tile_bytes);
        const uint32_t k_s = smem_u32(tiles + (s * 3 + 1) * tile_bytes);
        for (int hf = 0; hf < kHalves; ++hf) {
          if (!mbar_wait(&t_empty[hf], (uint32_t)((k & 1) ^ 1), abort, p.status,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qh = q_s + hf * kRows * C::kRowBytes;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(tmem + hf * kSlotColsW, wdesc_kmajor<HD>(qh, kk), wdesc_kmajor<HD>(k_s, kk),
                    idesc_s, kk);
          umma_commit(&s_full[hf]);
        }
      }
      if (*abort) {
        umma_commit(&drain[0]);
        mbar_drain(&drain[0], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == kWideFwdMma2) {
    if (lane == 0) {   // O = P V of both halves, as soon as each P is written
      constexpr uint32_t idesc_o = idesc_bf16(kRows, HD, 0, 1);
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        const int s = (int)(k % NS);
        const uint32_t v_s = smem_u32(tiles + (s * 3 + 2) * tile_bytes);
        for (int hf = 0; hf < kHalves; ++hf) {
          if (!mbar_wait(&p_full[hf], (uint32_t)(k & 1), abort, p.status, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t slot = tmem + hf * kSlotColsW;
          // A = P from TMEM: 16 keys per step are 8 columns of bf16 pairs, key
          // half 0 in columns 0-63, key half 1 in 128-191
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            umma_ts(slot + C::kOCol, slot + (kk >> 3) * kRows + (kk & 7) * 8,
                    wdesc_mnmajor<HD>(v_s, kk), idesc_o, kk);
          umma_commit(&o_full[hf]);
        }
        if (ok) umma_commit(&empty[s]);
      }
      if (*abort) {
        umma_commit(&drain[1]);
        mbar_drain(&drain[1], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp < kWideFwdWg * 4) {
    // Softmax / epilogue: warpgroup wg holds query rows 128 hf .. 128 hf + 127
    // (hf = wg >> 1) of every item and their keys 128 kh .. 128 kh + 127
    // (kh = wg & 1); thread = row = TMEM lane. The two key halves of a row
    // exchange their maxima and sums through shared memory.
    const int wg = warp >> 2, hf = wg >> 1, kh = wg & 1;
    const int row = threadIdx.x & (kWg - 1);
    const int lr = hf * kRows + row;               // query slot in the window
    const int lo = (1 - hf) * kRows + row;         // the other half's slot
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t slot = tmem + lane_base + hf * kSlotColsW;
    float* xm = xch + (hf * 2 + kh) * kRows;                  // this thread's maximum, sum
    float* xm_o = xch + (hf * 2 + (1 - kh)) * kRows;          // the other key half's
    constexpr int kSumOff = kHalves * 2 * kRows;
    for (long long k = 0; k < n_local; ++k) {
      const long long t = blockIdx.x + k * (long long)gridDim.x;
      const int s = (int)(k % NS);
      const uint32_t phs = (uint32_t)((k / NS) & 1), pht = (uint32_t)(k & 1);
      const long long win = t / g.heads;
      const int h = (int)(t - win * g.heads);
      const bool plain = WW > 0 && window_plain(g, win);
      const RowInfo me = plain ? plain_row_info<(WW > 0 ? WW : 16)>(g, win, lr)
                               : row_info(g, win, lr);
      uint32_t* ci = colinfo + (hf * 2 + (int)(k & 1)) * kKeys;
      if (!plain) {   // key words of the half's two slots per row: one each
        if (kh == 0) ci[lr] = key_word(me);
        else ci[lo] = key_word(row_info(g, win, lo));
      }
      if (named_sync_or(1 + hf, 2 * kWg, *abort)) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(&s_full[hf], pht, abort, p.status, kWaitLimitNs);
      mbar_wait(&full[s], phs, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      const float* brow = bias + s * p.bins_pad;
      // pass 1: logits written back over S, maximum of this key half (the
      // window kind decides the code path once per item, not per chunk)
      float m;
      if (WW > 0 && plain)
        m = wide_pass1<true, (WW > 0 ? WW : 16)>(slot, kh * kRows, brow, ci, me, p.scale_log2);
      else
        m = wide_pass1<false, 16>(slot, kh * kRows, brow, ci, me, p.scale_log2);
      xm[row] = m;
      tmem_wait_st();
      named_sync(1 + hf, 2 * kWg);
      m = fmaxf(m, xm_o[row]);
      // pass 2: P of this key half; a row that is not a real token subtracts
      // +inf instead of its maximum, so its P is zero without a select
      float l = wide_pass2(slot, kh * kRows, me.valid ? m : INFINITY);
      xm[kSumOff + row] = l;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[hf]);
      named_sync(1 + hf, 2 * kWg);
      l += xm_o[kSumOff + row];
      // epilogue: this key half's warpgroup stores columns (HD / 2) kh .. of
      // the O row, normalised, straight to its grid token
      mbar_wait(&o_full[hf], pht, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      {
        constexpr int OC = HD / 2;
        const float inv = me.valid ? 1.f / l : 0.f;
        __nv_bfloat16* dst = (__nv_bfloat16*)p.out0 + (me.token * g.heads + h) * HD + OC * kh;
        float o[OC];
        __syncwarp();
        if constexpr (OC == 16) tmem_ld16(slot + C::kOCol + OC * kh, o);
        else tmem_ld32(slot + C::kOCol + OC * kh, o);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&t_empty[hf]);
        if (me.stored && !*abort) store_row_bf16<OC>(dst, o, inv);
      }
      if (kh == 0 && me.stored && !*abort && p.lse)
        p.lse[me.token * g.heads + h] = me.valid ? (m + __log2f(l)) * 0.69314718055994531f : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWideFwdMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================================
// Backward
// ================================================================================
// Per (window, head) item, with Q, K, V, dO of the window in shared memory:
//  Phase 1, row statistics, query-major: for each 128-query half qt,
//    S = Q_qt K^T and dP = dO_qt V^T over all 256 keys fill the 512 TMEM
//    columns; warpgroup w (of three) reads the 16-key chunks w, w + 3, ... of
//    every row and keeps an online maximum M, l = sum 2^(x - M),
//    d = sum 2^(x - M) dP and max |dP|; the partials of a row are merged
//    through shared memory into
//    L = M + log2 l (log2 units) and D = d / l = sum_j P_ij dP_ij, and a bound
//    (max_j |dP_ij| + |D|) / l >= |dS_ij| of the row. The largest bound of the
//    window sets the unit 2^-E of its exact bias-gradient sums.
//  Phase 2, gradients, key-major: for each block of 128 keys (kb) x 128
//    queries (qt), S^T = K_kb Q_qt^T and dP^T = V_kb dO_qt^T (M = keys, so a
//    thread holds one key and walks queries); P = 2^(x - L_i) and
//    dS = P (dP - D_i): P goes back into its S^T columns as bf16 hi + lo
//    pairs (the A operand, from TMEM, of dV_kb += P^T dO_qt), dS as hi + lo
//    into shared memory (the A operand of both dK_kb += dS^T Q_qt and
//    dQ_qt += dS K_kb) and into the bias-gradient bins. The scale
//    head_dim^-1/2 of dQ and dK is applied to their fp32 sums at the end.
//    Warpgroup w takes the 16-query chunks w, w + 3, w + 6 of the block.
//    The products overlap the row work: once a block's rows are done, dP^T of
//    the next block goes into the dP^T columns (read already), dV of this
//    block runs, then S^T of the next block replaces P, and dK and dQ of this
//    block run while the next block's rows are worked on (its first write of
//    dS waits for them).
// TMEM: phase 1 S | dP at 0 | 256; phase 2 S^T | dP^T at 0 | 128, dV_kb at
// 256, dK_kb at 320, dQ_0 at 384, dQ_1 at 448. dV and dK of key half 0 leave
// after the third block's rows, the rest after the last block.
template <int HD>
struct WideBwdCfg {
  static constexpr uint32_t kRowBytes = HD * 2;
  static constexpr uint32_t kTileBytes = kKeys * kRowBytes;
  static constexpr int kStages = 1;
  static constexpr uint32_t kOpBytes = 2 * 32768;   // scale * dS, hi and lo
};
// The bias row of the head in four copies, copy m shifted down by m floats,
// so that any 16 consecutive entries are four aligned 16-byte loads from one
// of them. Row stride in floats:
__host__ __device__ inline int bias_copy_stride(int bins_pad) { return bins_pad + 4; }
constexpr uint32_t kColDP1 = 256;                    // phase 1 dP (S at 0)
constexpr uint32_t kColDPT = 128;                    // phase 2 dP^T (S^T at 0)
constexpr uint32_t kColDV = 256, kColDK = 320, kColDQ = 384;
// Backward warps: four softmax warpgroups (0-15), the TMA producer, the MMA
// issuer and the bin fold. Nineteen warps leave 96 registers a thread, which
// the one-buffer chunk loops fit.
constexpr int kWideSoftWg = 4;
constexpr int kWideBwdWarps = kWideSoftWg * 4 + 3;
constexpr int kWideProducerWarp = kWideSoftWg * 4, kWideMmaWarp = kWideProducerWarp + 1,
              kWideFoldWarp = kWideProducerWarp + 2;

struct WideBwdLayout {
  uint32_t tiles, dsop, bias, colinfo, stats, xch, bins, wb, bars, misc, total;
};

template <int HD>
__host__ __device__ inline WideBwdLayout wide_bwd_layout(int bins_pad) {
  using C = WideBwdCfg<HD>;
  WideBwdLayout L;
  L.tiles = 0;
  L.dsop = L.tiles + C::kStages * 4 * C::kTileBytes;
  L.xch = L.dsop;                            // [qt][warpgroup - 1][4][128] partial
                                             // statistics (phase 1 only: the dQ
                                             // operand is free then)
  L.bias = L.dsop + C::kOpBytes;
  L.colinfo = L.bias + C::kStages * 4 * bias_copy_stride(bins_pad) * 4;
  L.stats = L.colinfo + kKeys * 4;           // float2 {L, D} per query
  L.bins = L.stats + kKeys * 8;              // [2][bins_pad] int32 (item parity)
  L.wb = L.bins + 2 * bins_pad * 4;          // [4] warp bounds, [2] E, [2] finite
  L.bars = (L.wb + 64 + 7) & ~7u;
  L.misc = L.bars + 8 * 32;
  L.total = L.misc + 16;
  return L;
}

// dS of a block in shared memory, hi and lo: rows = keys, 128-byte rows of 64
// queries, 128-byte swizzle, 8 KB regions of 64 keys x 64 queries at
// (query half * 2 + key half) * 8 KB. The same bytes are two operands:
// the MN-major A of dQ_qt += dS K_kb (M = queries, K = keys; K step k16 = 16
// keys, the second 64-query atom 16 KB on) and the K-major A of
// dK_kb += dS^T Q_qt (M = keys, K = queries; K step k16 = 16 queries, the 128
// key rows evenly 1 KB per 8).
__device__ inline uint64_t desc_ds_mn(uint32_t base, int k16) {
  return smem_desc(base + (k16 >> 2) * 8192 + (k16 & 3) * 2048, 16384, 1024, kSwizzle128);
}
__device__ inline uint64_t desc_ds_k(uint32_t base, int k16) {
  return smem_desc(base + (k16 >> 2) * 16384 + (k16 & 3) * 32, 16, 1024, kSwizzle128);
}

// Runs work(x, i) over the n chunks i = 0 .. n-1 of a thread's list (n is
// the same for the whole warp): load(x, i) issues the TMEM loads of chunk i.
// One register buffer: with three softmax warpgroups the other warps of the
// scheduler cover the load latency.
template <typename LD, typename WK>
__device__ inline void pipelined_chunks(int n, LD&& load, WK&& work) {
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    float x[32];
    load(x, i);
    tmem_wait_ld_regs(x);
    work(x, i);
  }
}

// Phase 1 over the 16-key chunks w, w + 3, w + 6, ... of one row (S at
// columns s_col + 16 c, dP at dp_col + 16 c for chunk c): online maximum M,
// l = sum 2^(x - M), d = sum 2^(x - M) dP, a = max |dP|. Plain 16 x 16
// windows: the 16 keys of a chunk are one window row, whose table entries
// (bias_base - plain offset of the key) are a run of 16 consecutive floats
// read as four 16-byte loads from the shifted copies.
template <bool PLAIN>
__device__ inline void wide_row_stats(uint32_t s_col, uint32_t dp_col, int w,
                                      const float* bias4, int bstride, const uint32_t* ci,
                                      int bias_base, int label, float c, float& M, float& l,
                                      float& d, float& a) {
  M = -INFINITY;
  float2 l2 = make_float2(0.f, 0.f), d2 = make_float2(0.f, 0.f);
  a = 0.f;
  const int n = (kKeys / 16 - w + kWideSoftWg - 1) / kWideSoftWg;
  auto load = [&](float* x, int i) {
    const int k0 = 16 * (w + kWideSoftWg * i);
    __syncwarp();
    tmem_ld16(s_col + k0, x);
    tmem_ld16(dp_col + k0, x + 16);
  };
  auto work = [&](float* x, int i) {   // x: 16 of S, then 16 of dP
    const int k0 = 16 * (w + kWideSoftWg * i);
    float cm;
    if constexpr (PLAIN) {
      const int lo = bias_base - plain_off<16>(k0) - 15;   // entry of key k0 + 15
      const int m = lo & 3;
      const float4* bp = reinterpret_cast<const float4*>(bias4 + m * bstride + (lo - m));
      float b[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 v = bp[u];   // entries of keys k0 + 15 - 4u .. k0 + 12 - 4u
        b[15 - 4 * u] = v.x;
        b[14 - 4 * u] = v.y;
        b[13 - 4 * u] = v.z;
        b[12 - 4 * u] = v.w;
      }
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float2 v = __ffma2_rn(make_float2(x[j], x[j + 1]), make_float2(c, c),
                                    make_float2(b[j], b[j + 1]));
        x[j] = v.x;
        x[j + 1] = v.y;
        m0 = fmaxf(m0, v.x);
        m1 = fmaxf(m1, v.y);
      }
      cm = fmaxf(m0, m1);
    } else {
      cm = logits_general<16>(x, bias4, ci + k0, bias_base, label, c);
    }
    if (cm > M) {   // rescale the sums to the new maximum
      const float f = ex2(M - cm);
      l2 = __fmul2_rn(l2, make_float2(f, f));
      d2 = __fmul2_rn(d2, make_float2(f, f));
      M = cm;
    }
    const float nM = M == -INFINITY ? 0.f : -M;   // a chunk of masked keys adds zeros
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float2 t = __fadd2_rn(make_float2(x[j], x[j + 1]), make_float2(nM, nM));
      const float2 e = make_float2(ex2(t.x), ex2(t.y));
      l2 = __fadd2_rn(l2, e);
      d2 = __ffma2_rn(e, make_float2(x[16 + j], x[17 + j]), d2);
      a0 = fmaxf(a0, fabsf(x[16 + j]));
      a1 = fmaxf(a1, fabsf(x[17 + j]));
    }
    a = fmaxf(a, fmaxf(a0, a1));
  };
  pipelined_chunks(n, load, work);
  l = l2.x + l2.y;
  d = d2.x + d2.y;
}

// Phase 2, this thread's key over the 16-query chunks kk = w, w + 3, w + 6
// (kk < 8) of one block (i0 = ib0 + 16 kk, the chunk's first query): P and dS
// from S^T and dP^T, P's hi / lo pairs back into its S^T columns, dS's into
// the shared-memory operand (after `op_free`, when given), dS to the
// bias-gradient bins. Bias and bins of pair (i, j) sit at kbase + off(i),
// kbase = C0 - off(j). Plain 16 x 16 windows: a chunk is one window row of
// queries, so its 16 table entries are consecutive and come as four 16-byte
// loads from the shifted bias copies.
template <bool PLAIN>
__device__ inline void wide_grad_block(uint32_t tl, int w, int ib0, const float4* stats4,
                                       const uint32_t* ci, const float* bias4, int bstride,
                                       int kbase, int* bins, uint32_t keylab, bool bins_on,
                                       float c, float qs, uint32_t op_key, int jr,
                                       uint64_t* op_free, uint32_t op_phase, volatile int* abort,
                                       int* status) {
  const int n = (kRows / 16 - w + kWideSoftWg - 1) / kWideSoftWg;
  auto load = [&](float* x, int i) {   // [0, 16) S^T, [16, 32) dP^T of chunk w + 3 i
    const int kk = w + kWideSoftWg * i;
    __syncwarp();
    tmem_ld16(tl + 16 * kk, x);
    tmem_ld16(tl + kColDPT + 16 * kk, x + 16);
  };
  auto work = [&](float* x, int i) {
    const int kk = w + kWideSoftWg * i;
    const int i0 = ib0 + 16 * kk;
    int base = 0, m = 0;
    if constexpr (PLAIN) {
      base = kbase + plain_off<16>(i0);
      m = base & 3;
    }
    const float4* bp = reinterpret_cast<const float4*>(bias4 + m * bstride + (base - m));
    uint32_t pw[16], sw[16];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {   // 4 queries: one 16-byte bias load (plain windows)
      float b4[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (PLAIN) {
        const float4 v = bp[q4];
        b4[0] = v.x;
        b4[1] = v.y;
        b4[2] = v.z;
        b4[3] = v.w;
      }
#pragma unroll
      for (int u2 = 0; u2 < 2; ++u2) {
        const int u = 2 * q4 + u2;
        const float4 st = stats4[(i0 >> 1) + u];   // -L, -D of queries i0 + 2u, i0 + 2u + 1
        const float2 s2 = make_float2(x[2 * u], x[2 * u + 1]);
        float2 lg;
        int idx0, idx1;
        if constexpr (PLAIN) {
          idx0 = base + 2 * u;
          idx1 = idx0 + 1;
          lg = __ffma2_rn(s2, make_float2(c, c), make_float2(b4[2 * u2], b4[2 * u2 + 1]));
        } else {
          const uint32_t w0 = ci[i0 + 2 * u], w1 = ci[i0 + 2 * u + 1];
          idx0 = kbase + (int)(w0 & 0xFFFF);
          idx1 = kbase + (int)(w1 & 0xFFFF);
          lg.x = (w0 >> 16) == keylab ? fmaf(s2.x, c, bias4[idx0]) : -INFINITY;
          lg.y = (w1 >> 16) == keylab ? fmaf(s2.y, c, bias4[idx1]) : -INFINITY;
        }
        const float2 t = __fadd2_rn(lg, make_float2(st.x, st.y));
        const float2 P = make_float2(ex2(t.x), ex2(t.y));
        const float2 dS =
            __fmul2_rn(P, __fadd2_rn(make_float2(x[16 + 2 * u], x[17 + 2 * u]), make_float2(st.z, st.w)));
        if (bins_on) {   // dS in units of 2^-E, rounded to integers (q = 2^E: the product is exact)
          const float2 q = __ffma2_rn(dS, make_float2(qs, qs), make_float2(12582912.0f, 12582912.0f));
          red_add_s32_relaxed(bins + idx0, __float_as_int(q.x) - 0x4B400000);
          red_add_s32_relaxed(bins + idx1, __float_as_int(q.y) - 0x4B400000);
        }
        // hi = the top 16 bits of each value (bf16 truncation), lo = bf16 of the rest
        {
          const uint32_t a = __float_as_uint(P.x), bb = __float_as_uint(P.y);
          pw[u] = __byte_perm(a, bb, 0x7632);
          const float2 r2 = __ffma2_rn(
              make_float2(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(bb & 0xFFFF0000u)),
              make_float2(-1.f, -1.f), P);
          pw[8 + u] = pack_bf16(r2.x, r2.y);
        }
        {
          const uint32_t a = __float_as_uint(dS.x), bb = __float_as_uint(dS.y);
          sw[u] = __byte_perm(a, bb, 0x7632);
          const float2 r2 = __ffma2_rn(
              make_float2(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(bb & 0xFFFF0000u)),
              make_float2(-1.f, -1.f), dS);
          sw[8 + u] = pack_bf16(r2.x, r2.y);
        }
      }
    }
    __syncwarp();
    tmem_st16u(tl + 16 * kk, pw);
    // the dS operand is free once the previous block's dK and dQ are done
    if (i == 0 && op_free) mbar_wait(op_free, op_phase, abort, status, kWaitLimitNs);
    // query half kk / 4, 16-byte chunks 2 (kk % 4) and 2 (kk % 4) + 1 of the key's row
    const uint32_t op_hi = op_key + (kk >> 2) * 16384 + (((2 * (kk & 3)) ^ (jr & 7)) << 4);
    st_shared_v4(op_hi, sw[0], sw[1], sw[2], sw[3]);
    st_shared_v4(op_hi ^ 16u, sw[4], sw[5], sw[6], sw[7]);
    st_shared_v4(op_hi + 32768, sw[8], sw[9], sw[10], sw[11]);
    st_shared_v4((op_hi + 32768) ^ 16u, sw[12], sw[13], sw[14], sw[15]);
  };
  pipelined_chunks(n, load, work);
}

// Rows of one accumulator (HD columns) to the grid tokens of `ri` (lane = row).
template <int HD>
__device__ inline void store_acc_rows(uint32_t taddr, bool stored, long long token,
                                      __nv_bfloat16* out, int heads, int h, float mul) {
  float o[HD];
  tmem_load_cols<HD>(taddr, o);
  tmem_wait_ld();
  store_rows_bf16<HD>(o, mul, stored ? (const void*)(out + (token * heads + h) * HD) : nullptr);
}

template <int HD, int WW>
__global__ void __launch_bounds__(kWideBwdWarps * 32, 1)
    wide_bwd_kernel(const __grid_constant__ FastParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using C = WideBwdCfg<HD>;
  constexpr int NS = C::kStages;
  constexpr uint32_t tile_bytes = C::kTileBytes, RB = C::kRowBytes;
  constexpr int kSoft = kWideSoftWg * kWg;   // threads of the softmax warpgroups
  const Geo& g = p.g;
  const int bp = p.bins_pad;
  const WideBwdLayout L = wide_bwd_layout<HD>(bp);
  uint8_t* tiles = smem + L.tiles;
  float* bias = (float*)(smem + L.bias);
  uint32_t* ci = (uint32_t*)(smem + L.colinfo);
  float2* stats = (float2*)(smem + L.stats);
  float* xch = (float*)(smem + L.xch);
  int* bins = (int*)(smem + L.bins);
  float* wbnd = (float*)(smem + L.wb);
  int* wE = (int*)(smem + L.wb + 16);
  int* wfin = wE + 2;
  uint64_t* bars = (uint64_t*)(smem + L.bars);
  uint64_t* full = bars;
  uint64_t* empty = full + NS;
  uint64_t* s1_full = empty + NS;
  uint64_t* t1_empty = s1_full + 1;
  uint64_t* s2_full = t1_empty + 1;
  uint64_t* pds_full = s2_full + 1;
  uint64_t* grad_done = pds_full + 1;
  uint64_t* gv_done = grad_done + 1;
  uint64_t* acc_free = gv_done + 1;
  uint64_t* t_free = acc_free + 1;
  uint64_t* bins_full = t_free + 1;    // [2]
  uint64_t* bins_empty = bins_full + 2;
  uint64_t* drain = bins_empty + 2;    // [1]
  uint64_t* never = drain + 1;
  uint32_t* tmem_slot = (uint32_t*)(smem + L.misc);
  volatile int* abort = (volatile int*)(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_local = local_tiles(p.n_tiles, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(s1_full, 1);
    mbar_init(t1_empty, kSoft);
    mbar_init(s2_full, 1);
    mbar_init(pds_full, kSoft);
    mbar_init(grad_done, 1);
    mbar_init(gv_done, 1);
    mbar_init(acc_free, kSoft);
    mbar_init(t_free, kSoft);
    for (int i = 0; i < 2; ++i) { mbar_init(&bins_full[i], kSoft); mbar_init(&bins_empty[i], 32); }
    mbar_init(drain, 1);
    mbar_init(never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kWideProducerWarp && lane == 0)
    for (int tt = 0; tt < 4; ++tt)
      for (int m = 0; m < kMaxMaps; ++m) prefetch_tmap(&p.maps[tt][m]);
  for (int i = threadIdx.x; i < 2 * bp; i += kWideBwdWarps * 32) bins[i] = 0;
  if (warp == kWideMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWideProducerWarp) {
    if (lane == 0) {
      long long k = 0;
      for (long long t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++k) {
        const int s = (int)(k % NS);
        const uint32_t ph = (uint32_t)((k / NS) & 1);
        if (!mbar_wait(&empty[s], ph ^ 1, abort, p.status, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&full[s], 4 * tile_bytes + bp * 4);
        issue_item_loads<HD, 4>(p, t, tiles + s * 4 * tile_bytes,
                                bias + s * 4 * bias_copy_stride(bp), &full[s]);
      }
      if (*abort) {
        const long long first = k > NS ? k - NS : 0;
        for (long long j = first; j < k; ++j)
          mbar_drain(&full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == kWideMmaWarp) {
    if (lane == 0) {   // every product, in dependency order
      constexpr uint32_t id_s1 = idesc_bf16(kRows, kKeys, 0, 0);
      constexpr uint32_t id_s2 = idesc_bf16(kRows, kRows, 0, 0);
      constexpr uint32_t id_g = idesc_bf16(kRows, HD, 0, 1);   // dV, dK: A from TMEM
      constexpr uint32_t id_q = idesc_bf16(kRows, HD, 1, 1);   // dQ: A MN-major in smem
      const uint32_t op_hi = smem_u32(smem + L.dsop), op_lo = op_hi + 32768;
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        const int s = (int)(k % NS);
        if (!mbar_wait(&full[s], (uint32_t)((k / NS) & 1), abort, p.status, kWaitLimitNs)) break;
        const uint32_t q_s = smem_u32(tiles + (s * 4 + 0) * tile_bytes);
        const uint32_t k_s = smem_u32(tiles + (s * 4 + 1) * tile_bytes);
        const uint32_t v_s = smem_u32(tiles + (s * 4 + 2) * tile_bytes);
        const uint32_t o_s = smem_u32(tiles + (s * 4 + 3) * tile_bytes);
        // phase 1: S | dP of each query half
        for (int qt = 0; qt < kHalves && ok; ++qt) {
          ok = qt == 0 ? mbar_wait(t_free, (uint32_t)((k & 1) ^ 1), abort, p.status, kWaitLimitNs)
                       : mbar_wait(t1_empty, 0, abort, p.status, kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(tmem, wdesc_kmajor<HD>(q_s + qt * kRows * RB, kk), wdesc_kmajor<HD>(k_s, kk),
                    id_s1, kk);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(tmem + kColDP1, wdesc_kmajor<HD>(o_s + qt * kRows * RB, kk),
                    wdesc_kmajor<HD>(v_s, kk), id_s1, kk);
          umma_commit(s1_full);
        }
        if (!ok || !mbar_wait(t1_empty, 1, abort, p.status, kWaitLimitNs)) break;
        // phase 2: blocks (kb, qt) = (0,0), (0,1), (1,0), (1,1)
        auto issue_st = [&](int b) {   // S^T of block b into columns 0-127
          const uint32_t kq = k_s + (b >> 1) * kRows * RB, qq = q_s + (b & 1) * kRows * RB;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(tmem, wdesc_kmajor<HD>(kq, kk), wdesc_kmajor<HD>(qq, kk), id_s2, kk);
        };
        auto issue_dpt = [&](int b) {   // dP^T of block b into columns 128-255
          const uint32_t vq = v_s + (b >> 1) * kRows * RB, oq = o_s + (b & 1) * kRows * RB;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(tmem + kColDPT, wdesc_kmajor<HD>(vq, kk), wdesc_kmajor<HD>(oq, kk), id_s2, kk);
        };
        tc_fence_after();
        issue_st(0);
        issue_dpt(0);
        umma_commit(s2_full);
        for (int b = 0; b < 4 && ok; ++b) {
          const int kb = b >> 1, qt = b & 1;
          const uint32_t kq = k_s + kb * kRows * RB;
          const uint32_t qq = q_s + qt * kRows * RB, oq = o_s + qt * kRows * RB;
          if (!(ok = mbar_wait(pds_full, (uint32_t)(b & 1), abort, p.status, kWaitLimitNs))) break;
          tc_fence_after();
          if (b < 3) issue_dpt(b + 1);   // its columns were read by the rows of block b
          // dV_1 and dK_1 start over the columns of dV_0 and dK_0: wait for their rows
          if (b == 2 && !(ok = mbar_wait(acc_free, (uint32_t)(k & 1), abort, p.status,
                                         kWaitLimitNs)))
            break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk) {   // dV += P^T dO, 16 queries per step
            const uint32_t acc = (qt > 0 || kk > 0) ? 1u : 0u;
            umma_ts(tmem + kColDV, tmem + 16 * kk, wdesc_mnmajor<HD>(oq, kk), id_g, acc);
            umma_ts(tmem + kColDV, tmem + 16 * kk + 8, wdesc_mnmajor<HD>(oq, kk), id_g, 1);
          }
          umma_commit(gv_done);
          if (b < 3) {   // S^T of the next block over P, once dV has read it
            if (!(ok = mbar_wait(gv_done, (uint32_t)(b & 1), abort, p.status, kWaitLimitNs))) break;
            tc_fence_after();
            issue_st(b + 1);
            umma_commit(s2_full);
          }
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk) {   // dK += dS^T Q, 16 queries per step
            const uint32_t acc = (qt > 0 || kk > 0) ? 1u : 0u;
            umma_ss(tmem + kColDK, desc_ds_k(op_hi, kk), wdesc_mnmajor<HD>(qq, kk), id_g, acc);
            umma_ss(tmem + kColDK, desc_ds_k(op_lo, kk), wdesc_mnmajor<HD>(qq, kk), id_g, 1);
          }
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk) {   // dQ += dS K, 16 keys per step
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            umma_ss(tmem + kColDQ + 64 * qt, desc_ds_mn(op_hi, kk), wdesc_mnmajor<HD>(kq, kk), id_q,
                    acc);
            umma_ss(tmem + kColDQ + 64 * qt, desc_ds_mn(op_lo, kk), wdesc_mnmajor<HD>(kq, kk), id_q,
                    1);
          }
          umma_commit(grad_done);
        }
        if (ok) umma_commit(&empty[s]);
      }
      if (*abort) {
        umma_commit(drain);
        mbar_drain(drain, 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == kWideFoldWarp) {
    // Each item's bins into the workspace's exact sums, in the window's unit.
    for (long long k = 0, t = blockIdx.x; k < n_local; ++k, t += gridDim.x) {
      const int par = (int)(k & 1);
      if (!mbar_wait(&bins_full[par], (uint32_t)((k >> 1) & 1), abort, p.status, kWaitLimitNs))
        break;
      const int h = (int)(t - (t / g.heads) * g.heads);
      int* bk = bins + par * bp;
      const int E = wE[par];
      const bool fin = wfin[par] != 0;
      long long* acc = p.dt_acc + (size_t)h * bp * kLimbStride;
      for (int i = lane; i < g.bins; i += 32) {
        const int v = bk[i];
        bk[i] = 0;
        if (!fin) flag_nonfinite(acc + (size_t)i * kLimbStride);
        else if (v != 0) add_fixed(acc + (size_t)i * kLimbStride, v, E);
      }
      __syncwarp();
      mbar_arrive(&bins_empty[par]);
    }
  } else if (warp < kWideSoftWg * 4) {
    const int wg = warp >> 2;
    const int r = threadIdx.x & (kWg - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tl = tmem + lane_base;
    const float dscale = p.scale_log2 * (1.0f / kLog2e);   // head_dim^-1/2
    const int C0 = (g.wh - 1) * (2 * g.ww - 1) + g.ww - 1;  // table offset of slot (0, 0)
    const uint32_t op_base = smem_u32(smem + L.dsop);
    for (long long k = 0; k < n_local; ++k) {
      const long long t = blockIdx.x + k * (long long)gridDim.x;
      const int s = (int)(k % NS), par = (int)(k & 1);
      const long long win = t / g.heads;
      const int h = (int)(t - win * g.heads);
      const bool plain = WW > 0 && window_plain(g, win);
      // this thread's slots r and 128 + r (query rows of phase 1 and the dQ
      // epilogue, key rows of phase 2)
      // This thread's slots r and 128 + r (query rows of phase 1 and of the dQ
      // epilogue, key rows of phase 2), packed: key offset (bits 0-15), label
      // (16-19), valid (20), stored (21). Grid tokens are recomputed for the
      // epilogues only.
      uint32_t slotw[2];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const RowInfo ri = plain ? plain_row_info<(WW > 0 ? WW : 16)>(g, win, x * kRows + r)
                                 : row_info(g, win, x * kRows + r);
        slotw[x] = (uint32_t)ri.key_off | ((uint32_t)ri.label << 16) | ((uint32_t)ri.valid << 20) |
                   ((uint32_t)ri.stored << 21);
        if (x == wg) ci[wg * kRows + r] = key_word(ri);   // (warpgroups 0 and 1)
      }
      auto slot_token = [&](int x) {
        return (plain ? plain_row_info<(WW > 0 ? WW : 16)>(g, win, x * kRows + r)
                      : row_info(g, win, x * kRows + r)).token;
      };
      if (named_sync_or(1, kSoft, *abort)) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(&full[s], (uint32_t)((k / NS) & 1), abort, p.status, kWaitLimitNs);
      const int bstride = bias_copy_stride(bp);
      float* brow = bias + s * 4 * bstride;   // copy 0 (the loaded row), then copies 1-3
      for (int i = wg * kWg + r; i < g.bins; i += kSoft) {
        const float v = brow[i];
        if (i >= 1) brow[bstride + i - 1] = v;
        if (i >= 2) brow[2 * bstride + i - 2] = v;
        if (i >= 3) brow[3 * bstride + i - 3] = v;
      }
      named_sync(1, kSoft);
      // ---- phase 1 ----
      float bmax = 0.f;
      for (int qt = 0; qt < kHalves; ++qt) {
        const uint32_t qw = qt ? slotw[1] : slotw[0];
        const int q_base = C0 + (int)(qw & 0xFFFF);
        const int q_label = (int)((qw >> 16) & 15);
        const bool q_valid = (qw >> 20) & 1;
        mbar_wait(s1_full, (uint32_t)qt, abort, p.status, kWaitLimitNs);
        tc_fence_after();
        float M, l, d, a;
        if (WW == 16 && plain)
          wide_row_stats<true>(tl, tl + kColDP1, wg, brow, bstride, ci, q_base, q_label,
                               p.scale_log2, M, l, d, a);
        else
          wide_row_stats<false>(tl, tl + kColDP1, wg, brow, bstride, ci, q_base, q_label,
                                p.scale_log2, M, l, d, a);
        tc_fence_before();
        mbar_arrive(t1_empty);
        float* xq = xch + qt * (kWideSoftWg - 1) * 4 * kRows;   // [wg - 1][M, l, d, a][row]
        if (wg > 0) {
          float* xw = xq + (wg - 1) * 4 * kRows;
          xw[r] = M;
          xw[kRows + r] = l;
          xw[2 * kRows + r] = d;
          xw[3 * kRows + r] = a;
        }
        named_sync(1, kSoft);
        if (wg == 0) {
          float Mx = M, a1 = 0.f;
#pragma unroll
          for (int w = 1; w < kWideSoftWg; ++w) {
            Mx = fmaxf(Mx, xq[(w - 1) * 4 * kRows + r]);
            a1 = fmaxf(a1, xq[(w - 1) * 4 * kRows + 3 * kRows + r]);
          }
          const float f0 = ex2(M - Mx);
          float lt = l * f0, dt = d * f0;
#pragma unroll
          for (int w = 1; w < kWideSoftWg; ++w) {
            const float* xw = xq + (w - 1) * 4 * kRows;
            const float f = ex2(xw[r] - Mx);
            lt = fmaf(xw[kRows + r], f, lt);
            dt = fmaf(xw[2 * kRows + r], f, dt);
          }
          float2 st = make_float2(INFINITY, 0.f);   // not a real token: P = 0
          if (q_valid) {
            const float inv = 1.f / lt;
            st = make_float2(Mx + __log2f(lt), dt * inv);
            // |dS_ij| <= max_j P_ij (max_j |dP_ij| + |D|), max_j P_ij = 1 / l;
            // a NaN becomes +inf here, since fmaxf would drop it
            float rb = inv * (fmaxf(a, a1) + fabsf(st.y));
            if (!(rb <= 3.0e38f)) rb = INFINITY;
            bmax = fmaxf(bmax, rb);
          }
          // per query pair: (-L0, -L1, -D0, -D1), so one 16-byte load gives
          // both queries' values as operand pairs of the packed arithmetic
          const int qi = qt * kRows + r;
          float* sp = reinterpret_cast<float*>(stats) + (qi >> 1) * 4 + (qi & 1);
          sp[0] = -st.x;
          sp[2] = -st.y;
        }
      }
      if (wg == 0) {
        const float wb = warp_max(bmax);
        if (lane == 0) wbnd[warp] = wb;
      }
      named_sync(1, kSoft);   // stats and bounds of the whole window are in
      const float win_bound = fmaxf(fmaxf(wbnd[0], wbnd[1]), fmaxf(wbnd[2], wbnd[3]));
      const bool finite = win_bound <= 3.0e38f;   // false for NaN and infinity
      const int E = tile_exponent(finite ? win_bound : 0.f);
      const float qs = exp2_int(E);
      if (k >= 2)   // this parity's bins (and unit) were folded (item k - 2)
        mbar_wait(&bins_empty[par], (uint32_t)(((k >> 1) - 1) & 1), abort, p.status, kWaitLimitNs);
      if (threadIdx.x == 0) {
        wE[par] = E;
        wfin[par] = finite ? 1 : 0;
      }
      int* bins_k = bins + par * bp;
      // ---- phase 2 ----
      const float4* stats4 = reinterpret_cast<const float4*>(stats);
      const int jr = r & 63;
      const uint32_t op_key = op_base + (r >> 6) * 8192 + jr * 128;   // this key's row, query half 0
      for (int b = 0; b < 4; ++b) {
        const int kb = b >> 1, qt = b & 1;
        const uint32_t kw = kb ? slotw[1] : slotw[0];
        const int key_off = (int)(kw & 0xFFFF);
        const bool k_valid = (kw >> 20) & 1;
        const uint32_t keylab = k_valid ? (kw >> 16) & 15 : 14u;   // pad key: no query matches
        mbar_wait(s2_full, (uint32_t)(b & 1), abort, p.status, kWaitLimitNs);
        tc_fence_after();
        const int ib0 = qt * kRows;
        const bool bins_on = finite && k_valid;
        uint64_t* opf = b > 0 ? grad_done : nullptr;   // block b - 1's dK and dQ
        const uint32_t opph = (uint32_t)((b - 1) & 1);
        if (WW == 16 && plain)
          wide_grad_block<true>(tl, wg, ib0, stats4, ci, brow, bstride, C0 - key_off, bins_k,
                                keylab, bins_on, p.scale_log2, qs, op_key, jr, opf, opph, abort,
                                p.status);
        else
          wide_grad_block<false>(tl, wg, ib0, stats4, ci, brow, bstride, C0 - key_off, bins_k,
                                 keylab, bins_on, p.scale_log2, qs, op_key, jr, opf, opph, abort,
                                 p.status);
        tmem_wait_st();
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(pds_full);
        if (b == 2 || b == 3) {
          // b = 2: dV and dK of key half 0 (their last products, block 1's, are
          // done); b = 3: dV and dK of key half 1 and dQ, after the last block
          const int eb = b == 2 ? 1 : 3, ek = b == 2 ? 0 : 1;
          mbar_wait(grad_done, (uint32_t)(eb & 1), abort, p.status, kWaitLimitNs);
          tc_fence_after();
          const bool ok = !*abort;
          // warpgroup 0: dV rows, 1: dK rows (key slots); after the last block
          // warpgroups 2 and 3 the dQ rows of query halves 0 and 1 (query slots
          // r and 128 + r)
          if (wg >= 2) {
            if (b == 3) {
              const int x = wg - 2;
              store_acc_rows<HD>(tl + kColDQ + 64 * x, ok && (((x ? slotw[1] : slotw[0]) >> 21) & 1),
                                 slot_token(x), (__nv_bfloat16*)p.out0, g.heads, h, dscale);
            }
          } else {
            const uint32_t ew = ek ? slotw[1] : slotw[0];
            const bool k_st = ok && ((ew >> 21) & 1);
            const long long k_tok = slot_token(ek);
            if (wg == 0)
              store_acc_rows<HD>(tl + kColDV, k_st, k_tok, (__nv_bfloat16*)p.out2, g.heads, h, 1.f);
            else
              store_acc_rows<HD>(tl + kColDK, k_st, k_tok, (__nv_bfloat16*)p.out1, g.heads, h,
                                 dscale);
          }
          tc_fence_before();
          mbar_arrive(b == 2 ? acc_free : t_free);
        }
      }
      mbar_arrive(&bins_full[par]);   // the fold warp adds them to the global sums
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWideMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int HD>
size_t wide_bwd_smem(const Geo& g) {
  return wide_bwd_layout<HD>(bins_padded(g.bins)).total + 1024;
}

template <int HD>
size_t wide_fwd_smem(const Geo& g) {
  return wide_fwd_layout<HD>(bins_padded(g.bins)).total + 1024;
}

template <typename K>
cudaError_t wide_launch(K kernel, const FastParams& p, size_t smem, int threads,
                        cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = p.n_tiles < num_sms() ? p.n_tiles : num_sms();
  kernel<<<(unsigned)(grid > 0 ? grid : 1), threads, smem, st>>>(p);
  note_launch();
  return cudaGetLastError();
}

void fill_wide(FastParams& p, const Geo& g, const float* bias_t, int* status, int flags) {
  fill_common(p, g, bias_t, status, flags);
  p.n_groups = g.n_win;            // one window per item
  p.n_tiles = g.n_win * g.heads;
}

}  // namespace

bool wide_supported(const Geo& g, int dtype) {
  if (dtype != SWIN_DTYPE_BF16) return false;
  if (g.hd != 64 && g.hd != 32) return false;
  if (g.N != kKeys || g.band) return false;
  if (g.wh > 256 || g.ww > 256) return false;   // one TMA box dimension
  // Every sub-box must be a whole number of 8-row swizzle atoms.
  const int ylen[3] = {g.wh, g.wh - g.sh, g.sh};
  const int xlen[3] = {g.ww, g.ww - g.sw, g.sw};
  for (int a = 0; a < 3; ++a)
    for (int c = 0; c < 3; ++c) {
      if ((a > 0 && g.sh == 0) || (c > 0 && g.sw == 0)) continue;
      if ((ylen[a] * xlen[c]) % 8) return false;
    }
  if (g.bins > 0xFFFF) return false;
  const size_t f = g.hd == 64 ? wide_fwd_smem<64>(g) : wide_fwd_smem<32>(g);
  const size_t b = g.hd == 64 ? wide_bwd_smem<64>(g) : wide_bwd_smem<32>(g);
  return f <= kSmemLimit && b <= kSmemLimit;
}

cudaError_t wide_forward(const Geo& g, const void* q, const void* k, const void* v,
                         const float* table, void* out, float* lse, void* ws, int flags,
                         cudaStream_t st) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  static thread_local FastParams p;
  fill_wide(p, g, bias_t, (int*)ws, flags);
  p.out0 = out;
  p.lse = lse;
  if (!encode_maps(p, 0, q) || !encode_maps(p, 1, k) || !encode_maps(p, 2, v))
    return cudaErrorInvalidValue;
  cudaError_t e = prep_bias(g, table, bias_t, nullptr, st);
  if (e != cudaSuccess) return e;
  const bool w16 = g.wh == 16 && g.ww == 16;
  if (g.hd == 64) {
    const size_t smem = wide_fwd_smem<64>(g);
    return w16 ? wide_launch(wide_fwd_kernel<64, 16>, p, smem, kWideThreads, st)
               : wide_launch(wide_fwd_kernel<64, 0>, p, smem, kWideThreads, st);
  }
  const size_t smem = wide_fwd_smem<32>(g);
  return w16 ? wide_launch(wide_fwd_kernel<32, 16>, p, smem, kWideThreads, st)
             : wide_launch(wide_fwd_kernel<32, 0>, p, smem, kWideThreads, st);
}

cudaError_t wide_backward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, const void* dout, void* dq, void* dk, void* dv,
                          float* dtable, void* ws, int flags, cudaStream_t st) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  long long* dt_acc = (long long*)((char*)ws + dbias_fixed_offset(g));
  static thread_local FastParams p;
  fill_wide(p, g, bias_t, (int*)ws, flags);
  p.out0 = dq;
  p.out1 = dk;
  p.out2 = dv;
  p.dt_acc = dt_acc;
  if (!encode_maps(p, 0, q) || !encode_maps(p, 1, k) || !encode_maps(p, 2, v) ||
      !encode_maps(p, 3, dout))
    return cudaErrorInvalidValue;
  cudaError_t e = prep_bias(g, table, bias_t, dt_acc, st);
  if (e != cudaSuccess) return e;
  const bool w16 = g.wh == 16 && g.ww == 16;
  constexpr int thr = kWideBwdWarps * 32;
  if (g.hd == 64) {
    const size_t smem = wide_bwd_smem<64>(g);
    e = w16 ? wide_launch(wide_bwd_kernel<64, 16>, p, smem, thr, st)
            : wide_launch(wide_bwd_kernel<64, 0>, p, smem, thr, st);
  } else {
    const size_t smem = wide_bwd_smem<32>(g);
    e = w16 ? wide_launch(wide_bwd_kernel<32, 16>, p, smem, thr, st)
            : wide_launch(wide_bwd_kernel<32, 0>, p, smem, thr, st);
  }
  if (e != cudaSuccess) return e;
  if (flags & SWIN_FLAG_DBIAS_SUMS) return cudaSuccess;   // the caller finishes the sums
  return finish_dbias(g, dt_acc, dtable, st);
}

}  // namespace swin
