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
constexpr int kWideThreads = 352;          // 11 warps
constexpr uint32_t kSlotColsW = 256;       // TMEM columns of one half

template <int HD>
struct WideFwdCfg {
  static constexpr uint32_t kRowBytes = HD * 2;
  static constexpr uint32_t kTileBytes = kKeys * kRowBytes;   // one tensor of one item
  static constexpr int kStages = HD > 32 ? 2 : 4;
  static constexpr uint32_t kOCol = 128;                       // O inside a half's slot
};

struct WideLayout {
  uint32_t tiles, bias, colinfo, bars, misc, total;
};

// NS stages of three [256][HD] tiles (Q, K, V), the stages' bias rows, per
// warpgroup two buffers of 256 key words, mbarriers, two words.
template <int HD>
__host__ __device__ inline WideLayout wide_fwd_layout(int bins_pad) {
  using C = WideFwdCfg<HD>;
  WideLayout L;
  L.tiles = 0;
  L.bias = L.tiles + C::kStages * 3 * C::kTileBytes;
  L.colinfo = L.bias + ((C::kStages * bins_pad * 4 + 15) & ~15);
  L.bars = (L.colinfo + kHalves * 2 * kKeys * 4 + 7) & ~7u;
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
    x[j] = fmaf(x[j], c, bias_q[-plain_off<WW>(j)]);
    x[j + 1] = fmaf(x[j + 1], c, bias_q[-plain_off<WW>(j + 1)]);
    m0 = fmaxf(m0, x[j]);
    m1 = fmaxf(m1, x[j + 1]);
  }
  return fmaxf(m0, m1);
}

// The row's 256 columns in chunks of 32, two register buffers: the TMEM load
// of chunk c + 1 is in flight while chunk c is worked on.
template <typename F>
__device__ inline void for_row_chunks(uint32_t slot, F&& work) {
  float xa[32], xb[32];
  __syncwarp();
  tmem_ld32(slot, xa);
#pragma unroll 1
  for (int k0 = 0; k0 < kKeys; k0 += 64) {
    tmem_wait_ld_regs(xa);
    __syncwarp();
    tmem_ld32(slot + k0 + 32, xb);
    work(xa, k0);
    tmem_wait_ld_regs(xb);
    if (k0 + 64 < kKeys) {
      __syncwarp();
      tmem_ld32(slot + k0 + 64, xa);
    }
    work(xb, k0 + 32);
  }
}

// Pass 1 over a row of 256 keys: logits (scale, bias, mask) written back over
// S in TMEM; returns the row maximum.
template <bool PLAIN, int WW>
__device__ inline float wide_pass1(uint32_t slot, const float* brow, const uint32_t* ci,
                                   const RowInfo& me, float c) {
  float m = -INFINITY;
  for_row_chunks(slot, [&](float* x, int k0) {
    float cm;
    if constexpr (PLAIN)
      cm = chunk_logits_plain<WW>(x, brow + me.bias_base, k0, c);
    else
      cm = logits_general<32>(x, brow, ci + k0, me.bias_base, me.label, c);
    m = fmaxf(m, cm);
    __syncwarp();
    tmem_st32(slot + k0, x);
  });
  return m;
}

// Pass 2: P = 2^(x - mo) as bf16 pairs over columns 0-127 (pair columns
// k0/2 .. k0/2 + 15 come from keys k0 .. k0 + 31, whose logits columns were
// read before they are overwritten); returns the row sum.
__device__ inline float wide_pass2(uint32_t slot, float mo) {
  float l = 0.f;
  for_row_chunks(slot, [&](float* x, int k0) {
    uint32_t w[16];
    float la = 0.f, lb = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float a = ex2(x[2 * j] - mo);
      const float b = ex2(x[2 * j + 1] - mo);
      la += a;
      lb += b;
      w[j] = pack_bf16(a, b);
    }
    l += la + lb;
    __syncwarp();
    tmem_st16u(slot + k0 / 2, w);
  });
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
        issue_item_loads<HD, 3>(p, t, tiles + s * 3 * tile_bytes, bias + s * p.bins_pad,
                                &full[s]);
      }
      if (*abort) {  // let copies already in flight land before the CTA leaves
        const long long first = k > NS ? k - NS : 0;
        for (long long j = first; j < k; ++j)
          mbar_drain(&full[j % NS], (uint32_t)((j / NS) & 1), kTestLimitNs * 100);
      }
    }
  } else if (warp == kMmaWarp) {
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
  } else if (warp == kMma2Warp) {
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
          // A = P from TMEM: 16 keys per step are 8 columns of bf16 pairs
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            umma_ts(slot + C::kOCol, slot + kk * 8, wdesc_mnmajor<HD>(v_s, kk), idesc_o, kk);
          umma_commit(&o_full[hf]);
        }
        if (ok) umma_commit(&empty[s]);
      }
      if (*abort) {
        umma_commit(&drain[1]);
        mbar_drain(&drain[1], 0, kTestLimitNs * 100);
      }
    }
  } else if (warp < kHalves * 4) {
    // Softmax / epilogue: warpgroup hf holds query rows 128 hf .. 128 hf + 127
    // of every item; thread = row = TMEM lane.
    const int hf = warp >> 2;
    const int row = threadIdx.x & (kWg - 1);
    const int lr = hf * kRows + row;               // query slot in the window
    const int lo = (1 - hf) * kRows + row;         // the other half's slot
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t slot = tmem + lane_base + hf * kSlotColsW;
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
      if (!plain) {
        ci[lr] = key_word(me);
        ci[lo] = key_word(row_info(g, win, lo));
      }
      if (named_sync_or(1 + hf, kWg, *abort)) break;
      if (p.test_timeout) mbar_wait(never, 0, abort, p.status, kTestLimitNs);
      mbar_wait(&s_full[hf], pht, abort, p.status, kWaitLimitNs);
      mbar_wait(&full[s], phs, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      const float* brow = bias + s * p.bins_pad;
      // pass 1: logits written back over S, row maximum (the window kind
      // decides the code path once per item, not per chunk)
      float m;
      if (WW > 0 && plain)
        m = wide_pass1<true, (WW > 0 ? WW : 16)>(slot, brow, ci, me, p.scale_log2);
      else
        m = wide_pass1<false, 16>(slot, brow, ci, me, p.scale_log2);
      tmem_wait_st();
      // pass 2: P over columns 0-127; a row that is not a real token
      // subtracts +inf instead of its maximum, so its P is zero without a select
      const float l = wide_pass2(slot, me.valid ? m : INFINITY);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[hf]);
      // epilogue: O row from TMEM, normalised, straight to its grid token
      mbar_wait(&o_full[hf], pht, abort, p.status, kWaitLimitNs);
      tc_fence_after();
      {
        const float inv = me.valid ? 1.f / l : 0.f;
        __nv_bfloat16* dst = (__nv_bfloat16*)p.out0 + (me.token * g.heads + h) * HD;
        float o[HD];
        tmem_load_cols<HD>(slot + C::kOCol, o);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&t_empty[hf]);
        if (me.stored && !*abort) store_row_bf16<HD>(dst, o, inv);
      }
      if (me.stored && !*abort && p.lse)
        p.lse[me.token * g.heads + h] = me.valid ? (m + __log2f(l)) * 0.69314718055994531f : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
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
  const size_t sm = g.hd == 64 ? wide_fwd_smem<64>(g) : wide_fwd_smem<32>(g);
  return sm <= kSmemLimit;
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

}  // namespace swin
