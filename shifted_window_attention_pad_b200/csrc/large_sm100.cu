// large_sm100.cu -- tcgen05 / TMA kernels for 1024-token windows (32 x 32).
//
// Same operation as fast_sm100.cu and wide_sm100.cu -- shifted-window
// multi-head self-attention over a padded token grid (TERRA page, Abstract:
// window-based Swin Transformer with shifted-window execution; Table I: the
// padded resolution H^ x W^) -- for the 32 x 32 windows of the largest model
// of Table V. A row of 1024 keys does not fit in TMEM (512 columns), so the
// keys are taken in blocks of 128 (four window rows; see plan_block) with an
// online softmax:
//  * forward item = (window, head, pair of query blocks): the two query blocks
//    stay in shared memory while the eight key / value blocks stream through a
//    ring of stages. Per key block and query block, S = Q K^T (M = N = 128,
//    fp32 in TMEM), the softmax (two warpgroups per query block, 64 keys of
//    every row each) writes the logits back, takes the block maximum, and
//    writes P = 2^(x - m) as bf16 hi + lo pairs over the S columns;
//    O += P_hi V + P_lo V takes P from TMEM (tcgen05.mma with A in TMEM). (bf16
//    P alone measured 1.15 of the o error bar over a whole 256 x 544 grid.)
//    The running maximum m of a row
//    moves only when a block raises it by more than 2^8 (P stays below 2^8
//    otherwise); then O and the running sum are scaled by 2^(m_old - m_new)
//    in TMEM before the block's P is written.
//  * TMEM: query block q owns columns 256 q .. 256 q + 255: S / P in the first
//    128, O in the next head_dim.
// Warp roles (forward): warps 0-15 four softmax warpgroups (query block
// q = warpgroup >> 1, key half kh = warpgroup & 1), warp 16 the TMA producer,
// warp 17 issues S (and owns TMEM), warp 18 issues O += P V. Persistent grid
// of one CTA per SM; items round-robin, query-block pair fastest (the four
// items of a window and head share its key and value blocks in L2). Every
// mbarrier wait is bounded (%globaltimer); a wait that runs out records a
// timeout in the workspace status word and the kernel drains its copies and
// products and frees TMEM before returning.
#include "fast_common.cuh"

namespace swin {
namespace {

using namespace ptx;

constexpr int kLargeKeys = 1024;                   // tokens of a window
constexpr int kLargeBlocks = kLargeKeys / kRows;   // 128-token blocks of a window
constexpr int kLargeQPairs = kLargeBlocks / 2;     // forward items per window and head
constexpr int kLargeSoftWg = 4;
constexpr int kLargeThreads = (kLargeSoftWg * 4 + 3) * 32;
constexpr int kLargeProducer = kLargeSoftWg * 4, kLargeMma = kLargeProducer + 1,
              kLargeMma2 = kLargeProducer + 2;
constexpr uint32_t kLargeOCol = 128;   // O after S / P in a query block's 256 columns
constexpr float kRescaleLog2 = 8.f;    // the running maximum moves by more than this

template <int HD>
struct LargeFwdCfg {
  static constexpr uint32_t kTile = kRows * HD * 2;   // one 128-row block of one tensor
  static constexpr int kQBufs = HD > 64 ? 1 : 2;      // query-block pairs in shared memory
  static constexpr int kStages = HD > 64 ? 2 : 3;     // key / value block pairs
};

struct LargeFwdLayout {
  uint32_t q, kv, bias, colinfo, xch, bars, misc, total;
};

// kQBufs pairs of query blocks with their head's bias row, kStages pairs of
// key and value blocks, two buffers of 1024 key words, the maxima and sums
// the two key halves of a row exchange, mbarriers, two words.
template <int HD>
__host__ __device__ inline LargeFwdLayout large_fwd_layout(int bins_pad) {
  using C = LargeFwdCfg<HD>;
  LargeFwdLayout L;
  L.q = 0;
  L.kv = L.q + C::kQBufs * 2 * C::kTile;
  L.bias = L.kv + C::kStages * 2 * C::kTile;
  L.colinfo = L.bias + ((C::kQBufs * bins_pad * 4 + 15) & ~15);
  L.xch = L.colinfo + 2 * kLargeKeys * 4;
  L.bars = (L.xch + 3 * 2 * 2 * kRows * 4 + 7) & ~7u;   // [max x 2 parities, sum][q][kh][row]
  L.misc = L.bars + 8 * 32;
  L.total = L.misc + 16;
  return L;
}

// Producer: the TMA copies of block `blk` of one tensor of window `win`, head
// h, into a [128][HD] tile (channel halves of 64 as separate regions).
template <int HD>
__device__ inline void load_block(const FastParams& p, int tt, long long win, int h, int blk,
                                  uint8_t* tile, uint64_t* full) {
  const Geo& g = p.g;
  using T = TileGeom<HD>;
  int b, wy, wx;
  window_coords(g, win, b, wy, wx);
  SubBox sb[4];
  const int n = plan_block(g, wy, wx, blk, sb);
  for (int i = 0; i < n; ++i)
    for (int hf = 0; hf < T::kHalves; ++hf)
      tma_load_5d(tile + hf * T::kHalfBytes + sb[i].row_off * T::kRowBytes,
                  &p.maps[tt][sb[i].map_id], full, hf * T::kBoxEl, h, sb[i].x, sb[i].y, b);
}

// Logits (log2 units) of the NK keys k0 .. k0 + NK - 1 of a row (32 at a
// time), written back over S in TMEM; returns their maximum. Plain windows
// take compile-time bias offsets (keys in row-major order), others the key
// words (bias offset and region).
template <bool PLAIN, int NK>
__device__ inline float block_pass1(uint32_t s_col, int k0, const float* brow,
                                    const uint32_t* ci, const RowInfo& me, float c) {
  float m = -INFINITY;
#pragma unroll 1
  for (int i = 0; i < NK / 32; ++i) {
    float x[32];
    __syncwarp();
    tmem_ld32(s_col + 32 * i, x);
    tmem_wait_ld_regs(x);
    const int kw = k0 + 32 * i;   // key slot in the window
    float cm;
    if constexpr (PLAIN) {
      const float* bq = brow + me.bias_base - ((kw / 32) * 63 + kw % 32);
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 v = __ffma2_rn(make_float2(x[j], x[j + 1]), make_float2(c, c),
                                    make_float2(bq[-j], bq[-j - 1]));
        x[j] = v.x;
        x[j + 1] = v.y;
        m0 = fmaxf(m0, v.x);
        m1 = fmaxf(m1, v.y);
      }
      cm = fmaxf(m0, m1);
    } else {
      cm = logits_general<32>(x, brow, ci + kw, me.bias_base, me.label, c);
    }
    m = fmaxf(m, cm);
    __syncwarp();
    tmem_st32(s_col + 32 * i, x);
  }
  return m;
}

// 32 fp32 values as bf16 hi + lo pairs over 32 TMEM columns: the top 16 bits
// of each value (pairs in columns col .. col + 15) and the rest rounded to
// bf16 (col + 16 .. col + 31).
__device__ inline void split_to_tmem(uint32_t col, const float* v) {
  uint32_t hw[16], lw[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t a = __float_as_uint(v[2 * e]), b = __float_as_uint(v[2 * e + 1]);
    hw[e] = __byte_perm(a, b, 0x7632);
    const float2 r = __ffma2_rn(make_float2(__uint_as_float(a & 0xFFFF0000u),
                                            __uint_as_float(b & 0xFFFF0000u)),
                                make_float2(-1.f, -1.f), make_float2(v[2 * e], v[2 * e + 1]));
    lw[e] = pack_bf16(r.x, r.y);
  }
  __syncwarp();
  tmem_st16u(col, hw);
  tmem_st16u(col + 16, lw);
}
// A-operand columns of K step kk (16 elements) of such a 128-column operand
__device__ inline uint32_t split_col(int kk) { return 32 * (kk >> 1) + 8 * (kk & 1); }

// P = 2^(x - mu) of the same keys as bf16 hi + lo pairs over their own 32
// columns (split_to_tmem); returns the sum.
template <int NK>
__device__ inline float block_pass2(uint32_t s_col, float mu) {
  float l = 0.f;
#pragma unroll 1
  for (int i = 0; i < NK / 32; ++i) {
    float x[32];
    __syncwarp();
    tmem_ld32(s_col + 32 * i, x);
    tmem_wait_ld_regs(x);
    float2 l2 = make_float2(0.f, 0.f);
    const float2 nm = make_float2(-mu, -mu);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float2 t = __fadd2_rn(make_float2(x[j], x[j + 1]), nm);
      const float2 e = make_float2(ex2(t.x), ex2(t.y));
      l2 = __fadd2_rn(l2, e);
      x[j] = e.x;
      x[j + 1] = e.y;
    }
    l += l2.x + l2.y;
    split_to_tmem(s_col + 32 * i, x);
  }
  return l;
}

template <int HD>
__global__ void __launch_bounds__(kLargeThreads, 1)
    large_fwd_kernel(const __grid_constant__ FastParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using C = LargeFwdCfg<HD>;
  constexpr int NQ = C::kQBufs, NS = C::kStages;
  constexpr uint32_t TB = C::kTile;
  const Geo& g = p.g;
  const int bp = p.bins_pad;
  const LargeFwdLayout L = large_fwd_layout<HD>(bp);
  uint8_t* qbuf = smem + L.q;
  uint8_t* kv = smem + L.kv;
  float* bias = (float*)(smem + L.bias);
  uint32_t* colinfo = (uint32_t*)(smem + L.colinfo);
  float* xch = (float*)(smem + L.xch);
  uint64_t* bars = (uint64_t*)(smem + L.bars);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + NQ;
  uint64_t* kv_full = q_empty + NQ;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;   // [2] per query block
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* t_empty = o_done + 2;
  uint64_t* drain = t_empty + 2;      // [2]: one per MMA-issuing thread
  uint64_t* never = drain + 2;
  uint32_t* tmem_slot = (uint32_t*)(smem + L.misc);
  volatile int* abort = (volatile int*)(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_local = local_tiles(p.n_tiles, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) {
    // a query-block pair (and its bias row) is free once the item's last S
    // products are done and every softmax warp has read its last logits
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1 + kLargeSoftWg * 4);
    }
    for (int i = 0; i < NS; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 2 * kWg);
      mbar_init(&o_done[i], 1); mbar_init(&t_empty[i], 2 * kWg);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kLargeProducer && lane == 0)
    for (int tt = 0; tt < 3; ++tt)
      for (int m = 0; m < kMaxMaps; ++m) prefetch_tmap(&p.maps[tt][m]);
  if (warp == kLargeMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kLargeProducer) {
    if (lane == 0) {
      long long k = 0, e = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x, ++k) {
        const long long wh_item = t / kLargeQPairs;
        const int qp = (int)(t - wh_item * kLargeQPairs);
        const long long win = wh_item / g.heads;
        const int h = (int)(wh_item - win * g.heads);
        const int qs = (int)(k % NQ);
        if (!mbar_wait(&q_empty[qs], (uint32_t)(((k / NQ) & 1) ^ 1), abort, p.status,
                       kWaitLimitNs))
          break;
        mbar_arrive_expect_tx(&q_full[qs], 2 * TB + bp * 4);
        for (int q = 0; q < 2; ++q)
          load_block<HD>(p, 0, win, h, 2 * qp + q, qbuf + (qs * 2 + q) * TB, &q_full[qs]);
        bulk_load(bias + qs * bp, p.bias_t + (size_t)h * bp, bp * 4, &q_full[qs]);
        for (int kb = 0; kb < kLargeBlocks; ++kb, ++e) {
          const int s = (int)(e % NS);
          if (!mbar_wait(&kv_empty[s], (uint32_t)(((e / NS) & 1) ^ 1), abort, p.status,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[s], 2 * TB);
          load_block<HD>(p, 1, win, h, kb, kv + (s * 2 + 0) * TB, &kv_full[s]);
          load_block<HD>(p, 2, win, h, kb, kv + (s * 2 + 1) * TB, &kv_full[s]);
        }
      }
      if (*abort) {  // let copies already in flight land before the CTA leaves
        for (long long j = (e > NS ? e - NS : 0); j < e; ++j)
          mbar_drain(&kv_full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
        for (long long j = (k > NQ ? k - NQ : 0); j < k; ++j)
          mbar_drain(&q_full[j % NQ], (uint32_t)((j / NQ) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == kLargeMma) {
    if (lane == 0) {   // S = Q_q K_kb^T of both query blocks, key block by key block
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kRows, 0, 0);
      long long e = 0;
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        const int qs = (int)(k % NQ);
        if (!mbar_wait(&q_full[qs], (uint32_t)((k / NQ) & 1), abort, p.status, kWaitLimitNs))
          break;
        for (int kb = 0; kb < kLargeBlocks && ok; ++kb, ++e) {
          const int s = (int)(e % NS);
          if (!mbar_wait(&kv_full[s], (uint32_t)((e / NS) & 1), abort, p.status,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t k_s = smem_u32(kv + (s * 2 + 0) * TB);
          for (int q = 0; q < 2; ++q) {
            // the S columns are free once the previous O += P V of this block is done
            if (!mbar_wait(&o_done[q], (uint32_t)(((kb & 1)) ^ 1), abort, p.status,
                           kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t q_s = smem_u32(qbuf + (qs * 2 + q) * TB);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
              umma_ss(tmem + q * 256, desc_kmajor_tile<HD>(q_s, kk), desc_kmajor_tile<HD>(k_s, kk),
                      idesc_s, kk);
            umma_commit(&s_full[q]);
          }
        }
        if (ok) umma_commit(&q_empty[qs]);
      }
      if (*abort) {
        umma_commit(&drain[0]);
        mbar_drain(&drain[0], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == kLargeMma2) {
    if (lane == 0) {   // O += P V_kb of both query blocks, as soon as each P is written
      constexpr uint32_t idesc_o = idesc_bf16(kRows, HD, 0, 1);
      long long e = 0;
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        for (int kb = 0; kb < kLargeBlocks && ok; ++kb, ++e) {
          const int s = (int)(e % NS);
          const uint32_t v_s = smem_u32(kv + (s * 2 + 1) * TB);
          for (int q = 0; q < 2; ++q) {
            // a new item overwrites O: the previous item's epilogue has read it
            if (kb == 0 && !mbar_wait(&t_empty[q], (uint32_t)((k & 1) ^ 1), abort, p.status,
                                      kWaitLimitNs)) {
              ok = false;
              break;
            }
            if (!mbar_wait(&p_full[q], (uint32_t)(kb & 1), abort, p.status, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t base = tmem + q * 256;
            // A = P from TMEM: keys 16 kk .. 16 kk + 15 are 8 columns of bf16
            // hi pairs (split_col) and the 8 lo pairs 16 columns on
#pragma unroll
            for (int kk = 0; kk < kRows / 16; ++kk) {
              const uint64_t bv = desc_mnmajor_tile<HD>(v_s, kk);
              umma_ts(base + kLargeOCol, base + split_col(kk), bv, idesc_o,
                      (kb > 0 || kk > 0) ? 1u : 0u);
              umma_ts(base + kLargeOCol, base + split_col(kk) + 16, bv, idesc_o, 1u);
            }
            umma_commit(&o_done[q]);
          }
          if (ok) umma_commit(&kv_empty[s]);
        }
      }
      if (*abort) {
        umma_commit(&drain[1]);
        mbar_drain(&drain[1], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp < kLargeSoftWg * 4) {
    // Softmax / epilogue: warpgroup wg holds the rows of query block
    // q = wg >> 1 of every item (thread = row = TMEM lane) and keys
    // 64 kh .. 64 kh + 63 (kh = wg & 1) of every key block.
    const int wg = warp >> 2, q = wg >> 1, kh = wg & 1;
    const int row = threadIdx.x & (kWg - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + q * 256 + 64 * kh;
    const uint32_t o_col = tmem + lane_base + q * 256 + kLargeOCol + (HD / 2) * kh;
    float* xmax = xch;                              // [2 parities][q][kh][row]
    float* xsum = xch + 2 * 2 * 2 * kRows;          // [q][kh][row]
    for (long long k = 0; k < n_local; ++k) {
      const long long t = blockIdx.x + k * (long long)gridDim.x;
      const long long wh_item = t / kLargeQPairs;
      const int qp = (int)(t - wh_item * kLargeQPairs);
      const long long win = wh_item / g.heads;
      const int h = (int)(wh_item - win * g.heads);
      const int qs = (int)(k % NQ);
      const bool plain = window_plain(g, win);
      const int slot = (2 * qp + q) * kRows + row;   // query slot in the window
      const RowInfo me = plain ? plain_row_info<32>(g, win, slot) : block_row_info(g, win, slot);
      uint32_t* ci = colinfo + (int)(k & 1) * kLargeKeys;
      if (!plain)   // key words of the window's 1024 slots, two per thread
        for (int j = wg * kWg + row; j < kLargeKeys; j += kLargeSoftWg * kWg)
          ci[j] = key_word(block_row_info(g, win, j));
      if (named_sync_or(1, kLargeSoftWg * kWg, *abort)) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(&q_full[qs], (uint32_t)((k / NQ) & 1), abort, p.status, kWaitLimitNs);
      const float* brow = bias + qs * bp;
      float m_run = -INFINITY, l = 0.f;
      for (int kb = 0; kb < kLargeBlocks; ++kb) {
        mbar_wait(&s_full[q], (uint32_t)(kb & 1), abort, p.status, kWaitLimitNs);
        tc_fence_after();
        const int k0 = kb * kRows + 64 * kh;
        const float mp = plain ? block_pass1<true, 64>(s_col, k0, brow, ci, me, p.scale_log2)
                               : block_pass1<false, 64>(s_col, k0, brow, ci, me, p.scale_log2);
        float* xm = xmax + (kb & 1) * (2 * 2 * kRows) + q * 2 * kRows;
        xm[kh * kRows + row] = mp;
        tmem_wait_st();
        named_sync(2 + q, 2 * kWg);
        const float m_new = fmaxf(m_run, fmaxf(mp, xm[(1 - kh) * kRows + row]));
        // both key halves of a row take the same decision from the same values
        const bool move = m_new > m_run + kRescaleLog2;
        const float f = move ? ex2(m_run - m_new) : 1.f;   // 0 while m_run = -inf
        if (move) {
          l *= f;
          m_run = m_new;
        }
        if (kb > 0 && __any_sync(0xffffffffu, move)) {
          // scale this half's columns of O once the previous O += P V is done
          mbar_wait(&o_done[q], (uint32_t)((kb - 1) & 1), abort, p.status, kWaitLimitNs);
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < HD / 2; c += 16) {
            float o[16];
            __syncwarp();
            tmem_ld16(o_col + c, o);
            tmem_wait_ld_regs16(o);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const float2 v = __fmul2_rn(make_float2(o[j], o[j + 1]), make_float2(f, f));
              o[j] = v.x;
              o[j + 1] = v.y;
            }
            __syncwarp();
            tmem_st16u(o_col + c, reinterpret_cast<const uint32_t*>(o));
          }
        }
        // a row that is not a real token subtracts +inf (P = 0); a row whose
        // keys so far are all masked subtracts 0 (its logits are -inf)
        const float mu = !me.valid ? INFINITY : (m_run == -INFINITY ? 0.f : m_run);
        l += block_pass2<64>(s_col, mu);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[q]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_empty[qs]);   // the bias row is read
      // epilogue: the row sum over both key halves, then this half's HD / 2
      // columns of the O row, normalised, straight to the grid token
      xsum[(q * 2 + kh) * kRows + row] = l;
      named_sync(2 + q, 2 * kWg);
      l += xsum[(q * 2 + 1 - kh) * kRows + row];
      mbar_wait(&o_done[q], 1u, abort, p.status, kWaitLimitNs);   // the item's last product
      tc_fence_after();
      {
        constexpr int OC = HD / 2;
        const float inv = me.valid ? 1.f / l : 0.f;
        __nv_bfloat16* dst = (__nv_bfloat16*)p.out0 + (me.token * g.heads + h) * HD + OC * kh;
        float o[OC];
        __syncwarp();
        if constexpr (OC == 32) tmem_ld32(o_col, o);
        else tmem_load_cols<OC>(o_col, o);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&t_empty[q]);
        if (me.stored && !*abort) store_row_bf16<OC>(dst, o, inv);
      }
      if (kh == 0 && me.stored && !*abort && p.lse)
        p.lse[me.token * g.heads + h] =
            me.valid ? (m_run + __log2f(l)) * 0.69314718055994531f : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kLargeMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================================
// Backward
// ================================================================================
// Two kernels, because dQ sums over the key blocks and dK, dV over the query
// blocks, and neither fits in one CTA's TMEM for a whole window:
// Both take the keys (queries) of a block in two 64-wide sub-blocks, one per
// softmax warpgroup and TMEM buffer, so that one warpgroup's products run
// while the other works on its rows.
//  * query kernel, item = (window, head, query block qb): pass 1 runs
//    S = Q K_u^T and dP = dO V_u^T over the sixteen sub-blocks and keeps, per
//    row and key half, an online maximum M, l = sum 2^(x - M),
//    d = sum 2^(x - M) dP and max |dP|; the halves merge into L = M + log2 l
//    and D = d / l = sum_j P_ij dP_ij, written to the workspace for the key
//    kernel, and a bound (max |dP| + |D|) / l >= |dS| per row sets the unit
//    2^-E of the block's exact bias-gradient sums. Pass 2 recomputes S and
//    dP, P = 2^(x - L), dS = P (dP - D): dS goes into the bias-gradient bins
//    and, times head_dim^-1/2, as bf16 hi + lo pairs over its own dP columns,
//    the A operand (from TMEM) of dQ += dS K_kb.
//  * key kernel, item = (window, head, key block kb): S^T = K_kb Q_qb^T and
//    dP^T = V_kb dO_qb^T (thread = key row, walking queries), P^T and
//    scale * dS^T from the stored L and D as hi + lo pairs over their own
//    columns, dV += P^T dO_qb and dK += dS^T Q_qb with A from TMEM.
// A query block (window rows 4 qb .. 4 qb + 3) meets 35 of the 63 row offsets
// of the bias table, a contiguous run of 35 x 63 bins; so does a key block.
// Only that run of the head's bias row (and, in the query kernel, of its bins)
// is kept in shared memory.
constexpr int kBandBins = (kRows / 32 + 31) * 63;     // 2205
constexpr int kBandPad = (kBandBins + 3) & ~3;        // 2208: whole 16-byte copies
__host__ __device__ inline int qband0(int qb) { return 4 * qb * 63; }
__host__ __device__ inline int kband0(int kb) { return (28 - 4 * kb) * 63; }
// Warps: four softmax warpgroups (two per TMEM buffer, each 32 columns of its
// sub-block), the TMA producer, two MMA issuers and, in the query kernel, the
// bin fold: 20 and 19 warps, 96 registers a thread.
constexpr int kBwdSoftWg = 4;
constexpr int kBwdProducer = kBwdSoftWg * 4, kBwdMma = kBwdProducer + 1,
              kBwdMma2 = kBwdProducer + 2, kBwdFold = kBwdProducer + 3;
constexpr int kBwdQThreads = (kBwdSoftWg * 4 + 4) * 32;
constexpr int kBwdKThreads = (kBwdSoftWg * 4 + 3) * 32;
constexpr uint32_t kColXch = 384;   // query kernel: the warpgroups' row statistics
// TMEM: two buffers of 128 columns, one per softmax warpgroup, each a 64-key
// (query kernel) or 64-query (key kernel) sub-block's S and dP (S^T, dP^T) at
// 128 b and 128 b + 64; the gradient accumulators from column 256.
constexpr uint32_t kColGrad = 256;

template <int HD>
struct LargeBwdCfg {
  static constexpr uint32_t kTile = kRows * HD * 2;
  static constexpr int kStages = HD > 64 ? 2 : 3;   // streamed block pairs
};

struct LargeBwdLayout {
  uint32_t fixed, ring, bias, bins, stats, words, xch, bars, misc, total;
};

// Query kernel: Q and dO of the block, kStages pairs of K, V blocks, the bias
// run, its int32 bins, key words, the halves' statistics and bounds.
// Key kernel: K and V of the block, kStages pairs of Q, dO blocks, the bias
// run, L and D of the window's 1024 queries, query words.
template <int HD, bool KEYS>
__host__ __device__ inline LargeBwdLayout large_bwd_layout() {
  using C = LargeBwdCfg<HD>;
  LargeBwdLayout L;
  L.fixed = 0;
  L.ring = 2 * C::kTile;
  L.bias = L.ring + C::kStages * 2 * C::kTile;
  L.bins = L.bias + kBandPad * 4;
  L.stats = L.bins + (KEYS ? 0 : kBandPad * 4);
  L.words = L.stats + (KEYS ? kLargeKeys * 8 : 0);
  L.xch = L.words + kLargeKeys * 4;
  L.bars = (L.xch + (KEYS ? 0 : (2 * 4 * kRows + 16) * 4) + 7) & ~7u;
  L.misc = L.bars + 8 * 32;
  L.total = L.misc + 16;
  return L;
}

// Logits (log2 units) of 32 keys kw .. kw + 31 of a query row, in place.
template <bool PLAIN>
__device__ inline void row_logits(float* x, const float* brow, const uint32_t* ci, int kw,
                                  const RowInfo& me, float c) {
  if constexpr (PLAIN) {
    const float* bq = brow + me.bias_base - ((kw / 32) * 63 + kw % 32);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float2 v = __ffma2_rn(make_float2(x[j], x[j + 1]), make_float2(c, c),
                                  make_float2(bq[-j], bq[-j - 1]));
      x[j] = v.x;
      x[j + 1] = v.y;
    }
  } else {
    logits_general<32>(x, brow, ci + kw, me.bias_base, me.label, c);
  }
}

template <int HD>
__global__ void __launch_bounds__(kBwdQThreads, 1)
    large_bwdq_kernel(const __grid_constant__ FastParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using C = LargeBwdCfg<HD>;
  constexpr int NS = C::kStages;
  constexpr uint32_t TB = C::kTile;
  const Geo& g = p.g;
  const int bp = p.bins_pad;
  const LargeBwdLayout L = large_bwd_layout<HD, false>();
  uint8_t* qd = smem + L.fixed;   // Q, dO of the block
  uint8_t* ring = smem + L.ring;  // K, V pairs
  float* bias = (float*)(smem + L.bias);
  int* bins = (int*)(smem + L.bins);
  uint32_t* ci = (uint32_t*)(smem + L.words);
  float* wbd = (float*)(smem + L.xch);   // [16] warp bounds, [2][2] (E, finite) per item parity
  uint64_t* bars = (uint64_t*)(smem + L.bars);
  uint64_t* qd_full = bars;
  uint64_t* qd_empty = qd_full + 1;
  uint64_t* kv_full = qd_empty + 1;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* sd_full = kv_empty + NS;   // [2] per TMEM buffer (= softmax warpgroup)
  uint64_t* st_free = sd_full + 2;     // [2] pass 1: the warpgroup has read S and dP
  uint64_t* ds_full = st_free + 2;     // [2]
  uint64_t* dq_done = ds_full + 2;     // [2]
  uint64_t* t_empty = dq_done + 2;
  uint64_t* bins_full = t_empty + 1;
  uint64_t* bins_empty = bins_full + 1;
  uint64_t* drain = bins_empty + 1;   // [2]
  uint64_t* never = drain + 2;
  uint32_t* tmem_slot = (uint32_t*)(smem + L.misc);
  volatile int* abort = (volatile int*)(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_local = local_tiles(p.n_tiles, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    mbar_init(qd_empty, 1 + kBwdSoftWg * 4);   // the last S / dP products and every softmax warp
    for (int i = 0; i < NS; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sd_full[i], 1);
      mbar_init(&st_free[i], 2 * kWg);
      mbar_init(&ds_full[i], 2 * kWg);
      mbar_init(&dq_done[i], 1);
    }
    mbar_init(t_empty, kBwdSoftWg * kWg);
    mbar_init(bins_full, kBwdSoftWg * kWg);
    mbar_init(bins_empty, 32);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kBwdProducer && lane == 0)
    for (int tt = 0; tt < 4; ++tt)
      for (int m = 0; m < kMaxMaps; ++m) prefetch_tmap(&p.maps[tt][m]);
  for (int i = threadIdx.x; i < kBandPad; i += kBwdQThreads) bins[i] = 0;
  if (warp == kBwdMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kBwdProducer) {
    if (lane == 0) {
      long long k = 0, e = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x, ++k) {
        const long long wh_item = t / kLargeBlocks;
        const int qb = (int)(t - wh_item * kLargeBlocks);
        const long long win = wh_item / g.heads;
        const int h = (int)(wh_item - win * g.heads);
        if (!mbar_wait(qd_empty, (uint32_t)((k & 1) ^ 1), abort, p.status, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(qd_full, 2 * TB + kBandPad * 4);
        load_block<HD>(p, 0, win, h, qb, qd, qd_full);
        load_block<HD>(p, 3, win, h, qb, qd + TB, qd_full);
        bulk_load(bias, p.bias_t + (size_t)h * bp + qband0(qb), kBandPad * 4, qd_full);
        for (int st = 0; st < 2 * kLargeBlocks; ++st, ++e) {
          const int s = (int)(e % NS), kb = st & (kLargeBlocks - 1);
          if (!mbar_wait(&kv_empty[s], (uint32_t)(((e / NS) & 1) ^ 1), abort, p.status,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[s], 2 * TB);
          load_block<HD>(p, 1, win, h, kb, ring + (s * 2 + 0) * TB, &kv_full[s]);
          load_block<HD>(p, 2, win, h, kb, ring + (s * 2 + 1) * TB, &kv_full[s]);
        }
      }
      if (*abort) {
        for (long long j = (e > NS ? e - NS : 0); j < e; ++j)
          mbar_drain(&kv_full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
        if (k > 0) mbar_drain(qd_full, (uint32_t)((k - 1) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == kBwdMma) {
    if (lane == 0) {   // S = Q K_u^T and dP = dO V_u^T of 64-key sub-blocks u, both passes
      constexpr uint32_t idesc_s = idesc_bf16(kRows, 64, 0, 0);
      long long e = 0;
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        if (!mbar_wait(qd_full, (uint32_t)(k & 1), abort, p.status, kWaitLimitNs)) break;
        const uint32_t q_s = smem_u32(qd), do_s = smem_u32(qd + TB);
        for (int pass = 0; pass < 2 && ok; ++pass)
          for (int u = 0; u < 2 * kLargeBlocks; ++u) {
            const int b = u & 1, j = u >> 1;   // buffer (= warpgroup), key block
            const int s = (int)(e % NS);
            if (b == 0 && !mbar_wait(&kv_full[s], (uint32_t)((e / NS) & 1), abort, p.status,
                                     kWaitLimitNs)) {
              ok = false;
              break;
            }
            // buffer b is free once its previous sub-block is done with it: in
            // pass 1 once the warpgroup has read S and dP, in pass 2 once the dQ
            // products have read the dS written over dP
            bool w = true;
            if (pass == 0 && j == 0) {
              if (k > 0) w = mbar_wait(&dq_done[b], 1u, abort, p.status, kWaitLimitNs);
            } else if (pass == 0 || j == 0) {
              w = mbar_wait(&st_free[b], (uint32_t)((j - 1) & 1), abort, p.status, kWaitLimitNs);
            } else {
              w = mbar_wait(&dq_done[b], (uint32_t)((j - 1) & 1), abort, p.status, kWaitLimitNs);
            }
            if (!w) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t k_s = smem_u32(ring + (s * 2 + 0) * TB) + b * 64 * TileGeom<HD>::kRowBytes;
            const uint32_t v_s = smem_u32(ring + (s * 2 + 1) * TB) + b * 64 * TileGeom<HD>::kRowBytes;
            const uint32_t d = tmem + 128 * b;
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
              umma_ss(d, desc_kmajor_tile<HD>(q_s, kk), desc_kmajor_tile<HD>(k_s, kk), idesc_s, kk);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
              umma_ss(d + 64, desc_kmajor_tile<HD>(do_s, kk), desc_kmajor_tile<HD>(v_s, kk),
                      idesc_s, kk);
            umma_commit(&sd_full[b]);
            if (b == 1) {
              if (pass == 0) umma_commit(&kv_empty[s]);   // pass 1: K, V of the block read
              ++e;
            }
          }
        if (ok) umma_commit(qd_empty);
      }
      if (*abort) {
        umma_commit(&drain[0]);
        mbar_drain(&drain[0], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == kBwdMma2) {
    if (lane == 0) {   // dQ += scale dS_u K_u (hi, then lo), pass 2, sub-block by sub-block
      constexpr uint32_t idesc_q = idesc_bf16(kRows, HD, 0, 1);
      long long e = 0;
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        e += kLargeBlocks;   // pass 1 entries of the ring
        for (int u = 0; u < 2 * kLargeBlocks; ++u) {
          const int b = u & 1, j = u >> 1;
          const int s = (int)(e % NS);
          if (u == 0 && !mbar_wait(t_empty, (uint32_t)((k & 1) ^ 1), abort, p.status,
                                   kWaitLimitNs)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&ds_full[b], (uint32_t)(j & 1), abort, p.status, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_s = smem_u32(ring + (s * 2 + 0) * TB) + b * 64 * TileGeom<HD>::kRowBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t a = tmem + 128 * b + 64 + split_col(kk);
            const uint64_t bd = desc_mnmajor_tile<HD>(k_s, kk);
            umma_ts(tmem + kColGrad, a, bd, idesc_q, (u > 0 || kk > 0) ? 1u : 0u);
            umma_ts(tmem + kColGrad, a + 16, bd, idesc_q, 1u);
          }
          umma_commit(&dq_done[b]);
          if (b == 1) {
            umma_commit(&kv_empty[s]);
            ++e;
          }
        }
      }
      if (*abort) {
        umma_commit(&drain[1]);
        mbar_drain(&drain[1], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == kBwdFold) {
    // Each item's bins into the workspace's exact sums, in the item's unit.
    for (long long k = 0, t = blockIdx.x; k < n_local; ++k, t += gridDim.x) {
      if (!mbar_wait(bins_full, (uint32_t)(k & 1), abort, p.status, kWaitLimitNs)) break;
      const long long wh_item = t / kLargeBlocks;
      const int qb = (int)(t - wh_item * kLargeBlocks);
      const int h = (int)(wh_item - (wh_item / g.heads) * g.heads);
      const float* eb = wbd + 16 + 2 * (int)(k & 1);
      const int E = (int)eb[0];
      const bool fin = eb[1] != 0.f;
      long long* acc = p.dt_acc + ((size_t)h * bp + qband0(qb)) * kLimbStride;
      for (int i = lane; i < kBandBins; i += 32) {
        const int v = bins[i];
        bins[i] = 0;
        if (!fin) flag_nonfinite(acc + (size_t)i * kLimbStride);
        else if (v != 0) add_fixed(acc + (size_t)i * kLimbStride, v, E);
      }
      mbar_arrive(bins_empty);
    }
  } else {
    // Softmax / epilogue: warpgroup wg holds keys 64 kh + 32 part .. + 31 of
    // every key block (kh = wg >> 1: sub-blocks 2 kb + kh, in TMEM buffer kh;
    // part = wg & 1) for all 128 rows of the query block (thread = row = lane).
    const int wg = warp >> 2, kh = wg >> 1, part = wg & 1;
    const int row = threadIdx.x & (kWg - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + 128 * kh + 32 * part;
    const uint32_t dp_col = s_col + 64;
    const float c = p.scale_log2;
    const float dscale = p.scale_log2 * (1.0f / kLog2e);   // head_dim^-1/2
    for (long long k = 0; k < n_local; ++k) {
      const long long t = blockIdx.x + k * (long long)gridDim.x;
      const long long wh_item = t / kLargeBlocks;
      const int qb = (int)(t - wh_item * kLargeBlocks);
      const long long win = wh_item / g.heads;
      const int h = (int)(wh_item - win * g.heads);
      const bool plain = window_plain(g, win);
      const int slot = qb * kRows + row;
      const RowInfo me = plain ? plain_row_info<32>(g, win, slot) : block_row_info(g, win, slot);
      if (!plain)
        for (int j = wg * kWg + row; j < kLargeKeys; j += kBwdSoftWg * kWg)
          ci[j] = key_word(block_row_info(g, win, j));
      if (named_sync_or(1, kBwdSoftWg * kWg, *abort)) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(qd_full, (uint32_t)(k & 1), abort, p.status, kWaitLimitNs);
      const float* brow = bias - qband0(qb);   // indexed by bin
      // pass 1: statistics of this half's keys
      float m = -INFINITY, l = 0.f, d = 0.f, mdp = 0.f;
#pragma unroll 1
      for (int kb = 0; kb < kLargeBlocks; ++kb) {
        mbar_wait(&sd_full[kh], (uint32_t)(kb & 1), abort, p.status, kWaitLimitNs);
        tc_fence_after();
        {
          const int kw = kb * kRows + 64 * kh + 32 * part;
          float x[32], dp[32];
          __syncwarp();
          tmem_ld32(s_col, x);
          tmem_ld32(dp_col, dp);
          tmem_wait_ld_regs(x);
          reg_fence32(dp);
          // S and dP are in registers: the buffer's next products may start
          tc_fence_before();
          mbar_arrive(&st_free[kh]);
          if (plain) row_logits<true>(x, brow, ci, kw, me, c);
          else row_logits<false>(x, brow, ci, kw, me, c);
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j) cm = fmaxf(cm, x[j]);
          if (cm > m) {
            const float f = ex2(m - cm);   // 0 while m = -inf
            l *= f;
            d *= f;
            m = cm;
          }
          const float mu = m == -INFINITY ? 0.f : m;
          float2 l2 = make_float2(0.f, 0.f), d2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 ev = make_float2(ex2(x[j] - mu), ex2(x[j + 1] - mu));
            l2 = __fadd2_rn(l2, ev);
            d2 = __ffma2_rn(ev, make_float2(dp[j], dp[j + 1]), d2);
            mdp = fmaxf(mdp, fmaxf(fabsf(dp[j]), fabsf(dp[j + 1])));
          }
          l += l2.x + l2.y;
          d += d2.x + d2.y;
        }
      }
      // the four parts of each row merge (through TMEM columns 384 + 4 wg of
      // the row's lane); the block's bound sets its unit
      {
        const uint32_t xc = tmem + lane_base + kColXch;
        tmem_st4(xc + 4 * wg, m, l, d, mdp);
        tmem_wait_st();
        tc_fence_before();
        named_sync(2, kBwdSoftWg * kWg);
        tc_fence_after();
        float o[3][4];
#pragma unroll
        for (int i = 1; i < 4; ++i) tmem_ld4(xc + 4 * ((wg + i) & 3), o[i - 1]);
        tmem_wait_ld();
        float M = m;
#pragma unroll
        for (int i = 0; i < 3; ++i) M = fmaxf(M, o[i][0]);
        const float f0 = m == -INFINITY ? 0.f : ex2(m - M);
        l *= f0;
        d *= f0;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const float fi = o[i][0] == -INFINITY ? 0.f : ex2(o[i][0] - M);
          l += o[i][1] * fi;
          d += o[i][2] * fi;
          mdp = fmaxf(mdp, o[i][3]);
        }
        m = M;
      }
      const float M = m;
      const float Lr = me.valid ? M + __log2f(l) : INFINITY;   // P = 2^(x - L); 0 off real rows
      const float inv = me.valid ? 1.f / l : 0.f;             // max_j P_ij
      const float D = me.valid ? d * inv : 0.f;
      if (wg == 0)
        reinterpret_cast<float2*>(p.lse)[wh_item * kLargeKeys + slot] = make_float2(Lr, D);
      {
        float rb = inv * (mdp + fabsf(D));
        if (!(rb <= 3.0e38f)) rb = INFINITY;
        const float wb = warp_max(rb);
        if (lane == 0) wbd[warp] = wb;
      }
      named_sync(2, kBwdSoftWg * kWg);
      float bound = 0.f;
#pragma unroll
      for (int i = 0; i < kBwdSoftWg * 4; ++i) bound = fmaxf(bound, wbd[i]);
      const bool fin = bound <= 3.0e38f;
      const int E = tile_exponent(fin ? bound : 0.f);
      const float qs = exp2_int(E);
      if (threadIdx.x == 0) {
        wbd[16 + 2 * (int)(k & 1)] = (float)E;
        wbd[17 + 2 * (int)(k & 1)] = fin ? 1.f : 0.f;
      }
      // the bins are free once the fold warp has taken the previous item's
      if (k > 0) mbar_wait(bins_empty, (uint32_t)((k - 1) & 1), abort, p.status, kWaitLimitNs);
      // pass 2: dS into the bins and, scaled, as dQ's operand
#pragma unroll 1
      for (int kb = 0; kb < kLargeBlocks; ++kb) {
        mbar_wait(&sd_full[kh], (uint32_t)(kb & 1), abort, p.status, kWaitLimitNs);
        tc_fence_after();
        {
          const int kw = kb * kRows + 64 * kh + 32 * part;
          float x[32], ds[32];
          __syncwarp();
          tmem_ld32(s_col, x);
          tmem_ld32(dp_col, ds);
          tmem_wait_ld_regs(x);
          reg_fence32(ds);
          if (plain) row_logits<true>(x, brow, ci, kw, me, c);
          else row_logits<false>(x, brow, ci, kw, me, c);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 pj = make_float2(ex2(x[j] - Lr), ex2(x[j + 1] - Lr));
            const float2 v = __fmul2_rn(pj, __fadd2_rn(make_float2(ds[j], ds[j + 1]),
                                                        make_float2(-D, -D)));
            ds[j] = v.x;
            ds[j + 1] = v.y;
          }
          if (me.valid && fin) {
            int* bq = bins - qband0(qb) + me.bias_base;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 qv = __ffma2_rn(make_float2(ds[j], ds[j + 1]), make_float2(qs, qs),
                                           make_float2(12582912.0f, 12582912.0f));
#pragma unroll
              for (int e2 = 0; e2 < 2; ++e2) {
                const int kj = kw + j + e2;
                const int off = plain ? (kj / 32) * 63 + kj % 32 : (int)(ci[kj] & 0xFFFF);
                red_add_s32(bq - off, __float_as_int(e2 ? qv.y : qv.x) - 0x4B400000);
              }
            }
          }
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 v = __fmul2_rn(make_float2(ds[j], ds[j + 1]), make_float2(dscale, dscale));
            ds[j] = v.x;
            ds[j + 1] = v.y;
          }
          split_to_tmem(dp_col, ds);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ds_full[kh]);
      }
      mbar_arrive(bins_full);
      __syncwarp();
      if (lane == 0) mbar_arrive(qd_empty);   // the bias run is read
      // epilogue: this warpgroup's HD / 4 columns of the dQ row, once the
      // item's last product (sub-block 15, buffer 1) is done. A parity wait
      // only names a phase when the barrier is at most one phase behind it:
      // this buffer's own barrier is (its last sub-block's S and dP were
      // issued after the one before had completed), and its last products
      // completing brings buffer 1's there as well (products complete in
      // issue order), so buffer 0's warpgroups wait on their own first.
      mbar_wait(&dq_done[kh], 1u, abort, p.status, kWaitLimitNs);
      mbar_wait(&dq_done[1], 1u, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      {
        constexpr int OC = HD / 4;
        float o[OC];
        __syncwarp();
        if constexpr (OC == 32) tmem_ld32(tmem + lane_base + kColGrad + OC * wg, o);
        else tmem_ld16(tmem + lane_base + kColGrad + OC * wg, o);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(t_empty);
        if (me.stored && !*abort)
          store_row_bf16<OC>((__nv_bfloat16*)p.out0 + (me.token * g.heads + h) * HD + OC * wg, o,
                             1.f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int HD>
__global__ void __launch_bounds__(kBwdKThreads, 1)
    large_bwdk_kernel(const __grid_constant__ FastParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using C = LargeBwdCfg<HD>;
  constexpr int NS = C::kStages;
  constexpr uint32_t TB = C::kTile;
  const Geo& g = p.g;
  const int bp = p.bins_pad;
  const LargeBwdLayout L = large_bwd_layout<HD, true>();
  uint8_t* kvt = smem + L.fixed;  // K, V of the block
  uint8_t* ring = smem + L.ring;  // Q, dO pairs
  float* bias = (float*)(smem + L.bias);
  const float2* stats = (const float2*)(smem + L.stats);   // L, D of every query
  uint32_t* qw = (uint32_t*)(smem + L.words);
  uint64_t* bars = (uint64_t*)(smem + L.bars);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + 1;
  uint64_t* qd_full = kv_empty + 1;
  uint64_t* qd_empty = qd_full + NS;
  uint64_t* sd_full = qd_empty + NS;   // [2] per TMEM buffer (= softmax warpgroup)
  uint64_t* pds_full = sd_full + 2;    // [2]
  uint64_t* grad_done = pds_full + 2;  // [2]
  uint64_t* t_empty = grad_done + 2;
  uint64_t* drain = t_empty + 1;   // [2]
  uint64_t* never = drain + 2;
  uint32_t* tmem_slot = (uint32_t*)(smem + L.misc);
  volatile int* abort = (volatile int*)(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_local = local_tiles(p.n_tiles, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1 + kBwdSoftWg * 4);   // the last S^T / dP^T products and every softmax warp
    for (int i = 0; i < NS; ++i) { mbar_init(&qd_full[i], 1); mbar_init(&qd_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sd_full[i], 1);
      mbar_init(&pds_full[i], 2 * kWg);
      mbar_init(&grad_done[i], 1);
    }
    mbar_init(t_empty, kBwdSoftWg * kWg);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kBwdProducer && lane == 0)
    for (int tt = 0; tt < 4; ++tt)
      for (int m = 0; m < kMaxMaps; ++m) prefetch_tmap(&p.maps[tt][m]);
  if (warp == kBwdMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kBwdProducer) {
    if (lane == 0) {
      long long k = 0, e = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x, ++k) {
        const long long wh_item = t / kLargeBlocks;
        const int kb = (int)(t - wh_item * kLargeBlocks);
        const long long win = wh_item / g.heads;
        const int h = (int)(wh_item - win * g.heads);
        if (!mbar_wait(kv_empty, (uint32_t)((k & 1) ^ 1), abort, p.status, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(kv_full, 2 * TB + kBandPad * 4 + kLargeKeys * 8);
        load_block<HD>(p, 1, win, h, kb, kvt, kv_full);
        load_block<HD>(p, 2, win, h, kb, kvt + TB, kv_full);
        bulk_load(bias, p.bias_t + (size_t)h * bp + kband0(kb), kBandPad * 4, kv_full);
        bulk_load(smem + L.stats, p.lse + (size_t)wh_item * kLargeKeys * 2, kLargeKeys * 8, kv_full);
        for (int qb = 0; qb < kLargeBlocks; ++qb, ++e) {
          const int s = (int)(e % NS);
          if (!mbar_wait(&qd_empty[s], (uint32_t)(((e / NS) & 1) ^ 1), abort, p.status,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&qd_full[s], 2 * TB);
          load_block<HD>(p, 0, win, h, qb, ring + (s * 2 + 0) * TB, &qd_full[s]);
          load_block<HD>(p, 3, win, h, qb, ring + (s * 2 + 1) * TB, &qd_full[s]);
        }
      }
      if (*abort) {
        for (long long j = (e > NS ? e - NS : 0); j < e; ++j)
          mbar_drain(&qd_full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
        if (k > 0) mbar_drain(kv_full, (uint32_t)((k - 1) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == kBwdMma) {
    if (lane == 0) {   // S^T = K Q_u^T and dP^T = V dO_u^T of 64-query sub-blocks u
      constexpr uint32_t idesc_s = idesc_bf16(kRows, 64, 0, 0);
      long long e = 0;
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        if (!mbar_wait(kv_full, (uint32_t)(k & 1), abort, p.status, kWaitLimitNs)) break;
        const uint32_t k_s = smem_u32(kvt), v_s = smem_u32(kvt + TB);
        for (int u = 0; u < 2 * kLargeBlocks; ++u) {
          const int b = u & 1, qb = u >> 1;   // buffer (= warpgroup), query block
          const int s = (int)(e % NS);
          if ((b == 0 && !mbar_wait(&qd_full[s], (uint32_t)((e / NS) & 1), abort, p.status,
                                    kWaitLimitNs)) ||
              // buffer b holds its previous sub-block's P and dS until their products are done
              !mbar_wait(&grad_done[b], (uint32_t)((qb & 1) ^ 1), abort, p.status,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t off = b * 64 * TileGeom<HD>::kRowBytes;
          const uint32_t q_s = smem_u32(ring + (s * 2 + 0) * TB) + off;
          const uint32_t do_s = smem_u32(ring + (s * 2 + 1) * TB) + off;
          const uint32_t d = tmem + 128 * b;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(d, desc_kmajor_tile<HD>(k_s, kk), desc_kmajor_tile<HD>(q_s, kk), idesc_s, kk);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(d + 64, desc_kmajor_tile<HD>(v_s, kk), desc_kmajor_tile<HD>(do_s, kk),
                    idesc_s, kk);
          umma_commit(&sd_full[b]);
          if (b == 1) ++e;
        }
        if (ok) umma_commit(kv_empty);
      }
      if (*abort) {
        umma_commit(&drain[0]);
        mbar_drain(&drain[0], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp == kBwdMma2) {
    if (lane == 0) {   // dV += P^T dO_u, dK += scale dS^T Q_u (hi, then lo), sub-block by sub-block
      constexpr uint32_t idesc_g = idesc_bf16(kRows, HD, 0, 1);
      long long e = 0;
      bool ok = true;
      for (long long k = 0; k < n_local && ok; ++k) {
        for (int u = 0; u < 2 * kLargeBlocks; ++u) {
          const int b = u & 1, qb = u >> 1;
          const int s = (int)(e % NS);
          if (u == 0 && !mbar_wait(t_empty, (uint32_t)((k & 1) ^ 1), abort, p.status,
                                   kWaitLimitNs)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&pds_full[b], (uint32_t)(qb & 1), abort, p.status, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t off = b * 64 * TileGeom<HD>::kRowBytes;
          const uint32_t q_s = smem_u32(ring + (s * 2 + 0) * TB) + off;
          const uint32_t do_s = smem_u32(ring + (s * 2 + 1) * TB) + off;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t a = tmem + 128 * b + split_col(kk);
            const uint64_t bo = desc_mnmajor_tile<HD>(do_s, kk);
            const uint64_t bq = desc_mnmajor_tile<HD>(q_s, kk);
            const uint32_t first = (u > 0 || kk > 0) ? 1u : 0u;
            umma_ts(tmem + kColGrad, a, bo, idesc_g, first);
            umma_ts(tmem + kColGrad, a + 16, bo, idesc_g, 1u);
            umma_ts(tmem + kColGrad + HD, a + 64, bq, idesc_g, first);
            umma_ts(tmem + kColGrad + HD, a + 64 + 16, bq, idesc_g, 1u);
          }
          umma_commit(&grad_done[b]);
          if (b == 1) {
            umma_commit(&qd_empty[s]);
            ++e;
          }
        }
      }
      if (*abort) {
        umma_commit(&drain[1]);
        mbar_drain(&drain[1], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp < kBwdSoftWg * 4) {
    // Softmax / epilogue: thread = key row = lane of the block; warpgroup wg
    // takes queries 64 kh + 32 part .. + 31 of every query block (kh = wg >> 1:
    // sub-blocks 2 qb + kh, in TMEM buffer kh; part = wg & 1).
    const int wg = warp >> 2, kh = wg >> 1, part = wg & 1;
    const int row = threadIdx.x & (kWg - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + 128 * kh + 32 * part;
    const uint32_t dp_col = s_col + 64;
    const float c = p.scale_log2;
    const float dscale = p.scale_log2 * (1.0f / kLog2e);   // head_dim^-1/2
    for (long long k = 0; k < n_local; ++k) {
      const long long t = blockIdx.x + k * (long long)gridDim.x;
      const long long wh_item = t / kLargeBlocks;
      const int kb = (int)(t - wh_item * kLargeBlocks);
      const long long win = wh_item / g.heads;
      const int h = (int)(wh_item - win * g.heads);
      const bool plain = window_plain(g, win);
      const int slot = kb * kRows + row;
      const RowInfo me = plain ? plain_row_info<32>(g, win, slot) : block_row_info(g, win, slot);
      if (!plain)
        for (int j = wg * kWg + row; j < kLargeKeys; j += kBwdSoftWg * kWg)
          qw[j] = key_word(block_row_info(g, win, j));
      if (named_sync_or(1, kBwdSoftWg * kWg, *abort)) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(kv_full, (uint32_t)(k & 1), abort, p.status, kWaitLimitNs);
      // bias of (query j, this key) = brow[bias_base(j) - key_off]; a query's
      // bias_base is its key_off + 31 * 63 + 31
      const float* brow = bias - kband0(kb) - me.key_off + 31 * 63 + 31;
      const bool live = me.valid;   // a pad key: P = 0 in its whole row
#pragma unroll 1
      for (int qb = 0; qb < kLargeBlocks; ++qb) {
        mbar_wait(&sd_full[kh], (uint32_t)(qb & 1), abort, p.status, kWaitLimitNs);
        tc_fence_after();
        {
          const int q0 = qb * kRows + 64 * kh + 32 * part;   // first query slot of the chunk
          float x[32], dp[32];
          __syncwarp();
          tmem_ld32(s_col, x);
          tmem_ld32(dp_col, dp);
          tmem_wait_ld_regs(x);
          reg_fence32(dp);
          // (L, D) of two queries per 16-byte load; eight queries between
          // compiler barriers, so the loads in flight stay bounded (registers)
          const float4* st4 = reinterpret_cast<const float4*>(stats + q0);
          if (plain) {
            const float* bq = brow + (q0 / 32) * 63 + q0 % 32;
#pragma unroll
            for (int j0 = 0; j0 < 32; j0 += 8) {
#pragma unroll
              for (int j = j0; j < j0 + 8; j += 2) {
                const float4 ld = st4[j >> 1];
                const float2 t = __fadd2_rn(
                    __ffma2_rn(make_float2(x[j], x[j + 1]), make_float2(c, c),
                               make_float2(bq[j], bq[j + 1])),
                    make_float2(-ld.x, -ld.z));
                const float2 pj = make_float2(ex2(t.x), ex2(t.y));
                const float2 v = __fmul2_rn(pj, __fadd2_rn(make_float2(dp[j], dp[j + 1]),
                                                           make_float2(-ld.y, -ld.w)));
                x[j] = pj.x;
                x[j + 1] = pj.y;
                dp[j] = v.x;
                dp[j + 1] = v.y;
              }
              asm volatile("" ::: "memory");
            }
          } else {
#pragma unroll
            for (int j0 = 0; j0 < 32; j0 += 8) {
#pragma unroll
              for (int j = j0; j < j0 + 8; j += 2) {
                const float4 ld = st4[j >> 1];
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                  const uint32_t w = qw[q0 + j + e2];
                  const bool ok = live && (int)(w >> 16) == me.label;
                  const float pj =
                      ok ? ex2(fmaf(x[j + e2], c, brow[(int)(w & 0xFFFF)]) - (e2 ? ld.z : ld.x))
                         : 0.f;
                  x[j + e2] = pj;
                  dp[j + e2] = pj * (dp[j + e2] - (e2 ? ld.w : ld.y));
                }
              }
              asm volatile("" ::: "memory");
            }
          }
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 v = __fmul2_rn(make_float2(dp[j], dp[j + 1]), make_float2(dscale, dscale));
            dp[j] = v.x;
            dp[j + 1] = v.y;
          }
          split_to_tmem(s_col, x);
          split_to_tmem(dp_col, dp);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&pds_full[kh]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(kv_empty);   // bias run, statistics and query words read
      // epilogue: this warpgroup's HD / 4 columns of the dV and dK rows of this key
      // sub-block 15's products (buffer 1); buffer 0's warpgroups first wait
      // for their own last products, which leaves buffer 1's barrier at most
      // one phase behind the one the parity names (as in the query kernel)
      mbar_wait(&grad_done[kh], 1u, abort, p.status, kWaitLimitNs);
      mbar_wait(&grad_done[1], 1u, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      {
        constexpr int OC = HD / 4;
        const long long roff = (me.token * g.heads + h) * HD + OC * wg;
#pragma unroll 1
        for (int gi = 0; gi < 2; ++gi) {
          float o[OC];
          const uint32_t col = tmem + lane_base + kColGrad + gi * HD + OC * wg;
          __syncwarp();
          if constexpr (OC == 32) tmem_ld32(col, o);
          else tmem_ld16(col, o);
          tmem_wait_ld();
          if (gi == 1) {
            tc_fence_before();
            mbar_arrive(t_empty);
          }
          if (me.stored && !*abort)
            store_row_bf16<OC>((__nv_bfloat16*)(gi ? p.out1 : p.out2) + roff, o, 1.f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================================
// Host side
// ================================================================================
template <int HD>
size_t large_fwd_smem(const Geo& g) {
  return large_fwd_layout<HD>(bins_padded(g.bins)).total + 1024;
}
template <int HD, bool KEYS>
size_t large_bwd_smem() {
  return large_bwd_layout<HD, KEYS>().total + 1024;
}

template <typename K>
cudaError_t large_launch(K kernel, const FastParams& p, size_t smem, int threads,
                         cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = p.n_tiles < num_sms() ? p.n_tiles : num_sms();
  kernel<<<(unsigned)(grid > 0 ? grid : 1), threads, smem, st>>>(p);
  note_launch();
  return cudaGetLastError();
}

// The nine box shapes of one tensor for 128-token blocks: rows 128 / ww, or
// the two parts of a block on the row seam; columns as for whole windows.
bool encode_block_maps(FastParams& p, int which, const void* base) {
  const Geo& g = p.g;
  const int bh = kRows / g.ww;
  const int r1 = (g.wh - g.sh) % bh;
  for (int ky = 0; ky < 3; ++ky)
    for (int kx = 0; kx < 3; ++kx) {
      int by = ky == 0 ? bh : (ky == 1 ? r1 : bh - r1);
      int bx = box_len(kx, g.ww, g.sw);
      if (by <= 0) by = bh;   // shape unused
      if (bx <= 0) bx = g.ww;
      if (!encode_map(&p.maps[which][ky * 3 + kx], base, g, g.H, by, bx)) return false;
    }
  return true;
}

}  // namespace

bool large_supported(const Geo& g, int dtype) {
  if (dtype != SWIN_DTYPE_BF16) return false;
  if (g.hd != 64 && g.hd != 128) return false;
  if (g.wh != 32 || g.ww != 32 || g.band) return false;
  // Every sub-box of a block must be a whole number of 8-row swizzle atoms.
  const int bh = kRows / g.ww;
  const int r1 = (g.wh - g.sh) % bh;
  const int ylen[3] = {bh, r1, bh - r1};
  const int xlen[3] = {g.ww, g.ww - g.sw, g.sw};
  for (int a = 0; a < 3; ++a)
    for (int c = 0; c < 3; ++c) {
      if ((a > 0 && (g.sh == 0 || r1 == 0)) || (c > 0 && g.sw == 0)) continue;
      if ((ylen[a] * xlen[c]) % 8) return false;
    }
  if (g.bins != 63 * 63 || bins_padded(g.bins) < kband0(0) + kBandPad) return false;
  const size_t f = g.hd == 64 ? large_fwd_smem<64>(g) : large_fwd_smem<128>(g);
  const size_t bq = g.hd == 64 ? large_bwd_smem<64, false>() : large_bwd_smem<128, false>();
  const size_t bk = g.hd == 64 ? large_bwd_smem<64, true>() : large_bwd_smem<128, true>();
  return f <= kSmemLimit && bq <= kSmemLimit && bk <= kSmemLimit;
}

cudaError_t large_forward(const Geo& g, const void* q, const void* k, const void* v,
                          const float* table, void* out, float* lse, void* ws, int flags,
                          cudaStream_t st) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  static thread_local FastParams p;
  fill_common(p, g, bias_t, (int*)ws, flags);
  p.n_groups = g.n_win;
  p.n_tiles = g.n_win * g.heads * kLargeQPairs;
  p.out0 = out;
  p.lse = lse;
  if (!encode_block_maps(p, 0, q) || !encode_block_maps(p, 1, k) || !encode_block_maps(p, 2, v))
    return cudaErrorInvalidValue;
  cudaError_t e = prep_bias(g, table, bias_t, nullptr, st);
  if (e != cudaSuccess) return e;
  if (g.hd == 128)
    return large_launch(large_fwd_kernel<128>, p, large_fwd_smem<128>(g), kLargeThreads, st);
  return large_launch(large_fwd_kernel<64>, p, large_fwd_smem<64>(g), kLargeThreads, st);
}

// The bias table, the exact bias-gradient sums (as for the 64-token kernels),
// then L and D of every query ([windows * heads][1024] float2).
size_t large_workspace(const Geo& g) {
  return fast_workspace(g) + align256((size_t)g.n_win * g.heads * kLargeKeys * 8);
}

cudaError_t large_backward(const Geo& g, const void* q, const void* k, const void* v,
                           const float* table, const void* dout, void* dq, void* dk, void* dv,
                           float* dtable, void* ws, int flags, cudaStream_t st) {
  float* bias_t = (float*)((char*)ws + kWsHeader);
  long long* dt_acc = (long long*)((char*)ws + dbias_fixed_offset(g));
  static thread_local FastParams p;
  fill_common(p, g, bias_t, (int*)ws, flags);
  p.n_groups = g.n_win;
  p.n_tiles = g.n_win * g.heads * kLargeBlocks;
  p.out0 = dq;
  p.out1 = dk;
  p.out2 = dv;
  p.dt_acc = dt_acc;
  p.lse = (float*)((char*)ws + fast_workspace(g));   // L and D of every query
  if (!encode_block_maps(p, 0, q) || !encode_block_maps(p, 1, k) ||
      !encode_block_maps(p, 2, v) || !encode_block_maps(p, 3, dout))
    return cudaErrorInvalidValue;
  cudaError_t e = prep_bias(g, table, bias_t, dt_acc, st);
  if (e != cudaSuccess) return e;
  if (g.hd == 128) {
    e = large_launch(large_bwdq_kernel<128>, p, large_bwd_smem<128, false>(), kBwdQThreads, st);
    if (e == cudaSuccess)
      e = large_launch(large_bwdk_kernel<128>, p, large_bwd_smem<128, true>(), kBwdKThreads, st);
  } else {
    e = large_launch(large_bwdq_kernel<64>, p, large_bwd_smem<64, false>(), kBwdQThreads, st);
    if (e == cudaSuccess)
      e = large_launch(large_bwdk_kernel<64>, p, large_bwd_smem<64, true>(), kBwdKThreads, st);
  }
  if (e != cudaSuccess) return e;
  if (flags & SWIN_FLAG_DBIAS_SUMS) return cudaSuccess;   // the caller finishes the sums
  return finish_dbias(g, dt_acc, dtable, st);
}

}  // namespace swin
