// dbias_fixed.cuh -- exact, order-independent and scale-invariant sums for the
// gradient of the relative-position bias table.
//
// The bias-table gradient of one head is dT[b] = sum of dS_ij over every pair
// (i, j) of every window whose relative offset is bin b (TERRA page, Abstract:
// the Swin window attention trained end to end, so the learned bias table gets
// a gradient). Many threads and CTAs add into the same bin, and floating-point
// adds done in the order they land would change the last bits from run to run.
// Integer adds commute, so the kernels sum integers:
//
//  * per tile, every term is rounded to an integer multiple of 2^-E, where the
//    exponent E comes from a bound on |dS| over the tile (bound < 2^e gives
//    E = 22 - e, so every term is below 2^22 units and a bin of up to 256 terms
//    stays below 2^30); the rounding error of a term is at most 2^-23 of the
//    tile's bound, whatever the magnitude of the gradients;
//  * the tile's int32 bin sums are exact and do not depend on the order of
//    the shared-memory adds;
//  * each tile's bin v (units 2^-E) is added into a wide signed integer per
//    (head, bin) held as kLimbs 32-bit limbs in int64 words, value =
//    sum_k limb_k * 2^(32 k - kLimbOff): v * 2^(kLimbOff - E) straddles two
//    limbs, so two 64-bit global reductions add it exactly. Any order of
//    tiles gives the same limbs.
// A last kernel normalises the carries and converts each sum to fp32.
#pragma once
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace swin {

constexpr int kLimbs = 9;           // 288 bits: positions 2^-128 .. 2^160
constexpr int kLimbStride = 10;     // kLimbs words, then a non-finite flag
constexpr int kLimbOff = 128;       // limb 0 holds the bits of 2^-128 .. 2^-97
constexpr int kTileExpMin = -106;   // bound < 2^128
constexpr int kTileExpMax = 126;    // bounds below 2^-104 keep fewer than 22 bits

// Exponent E of a tile whose |dS| is at most `bound` (finite, >= 0): terms are
// rounded to multiples of 2^-E and stay below 2^22 units.
__host__ __device__ inline int tile_exponent(float bound) {
  union { float f; uint32_t u; } c;
  c.f = bound;
  const int e = (int)((c.u >> 23) & 0xFFu) - 126;   // bound < 2^e (also for 0 and subnormals)
  int E = 22 - e;
  if (E < kTileExpMin) E = kTileExpMin;
  if (E > kTileExpMax) E = kTileExpMax;
  return E;
}

// 2^E as a float, for E in [-126, 127].
__host__ __device__ inline float exp2_int(int E) {
  union { uint32_t u; float f; } c;
  c.u = (uint32_t)(E + 127) << 23;
  return c.f;
}

// x (|x| < 2^23) rounded to the nearest integer with the float adder: adding
// 1.5 * 2^23 leaves round(x) in the low mantissa bits.
__device__ __forceinline__ int round_to_int(float x) {
  return __float_as_int(x + 12582912.0f) - 0x4B400000;
}

// Adds v * 2^-E (|v| < 2^31, E in [kTileExpMin, kTileExpMax]) to the wide
// integer at acc[0 .. kLimbs).
__device__ __forceinline__ void add_fixed(long long* acc, int v, int E) {
  const int p0 = kLimbOff - E;            // bit position of 2^-E: 2 .. 234
  const int L = p0 >> 5, r = p0 & 31;
  const long long u = (long long)v << r;  // |u| < 2^62
  ptx::red_add_global_s64(acc + L, u & 0xFFFFFFFFll);
  ptx::red_add_global_s64(acc + L + 1, u >> 32);
}

// Marks the (head, bin) sum as not finite (a NaN or infinity reached dS).
__device__ __forceinline__ void flag_nonfinite(long long* acc) {
  ptx::red_add_global_s64(acc + kLimbs, 1);
}

}  // namespace swin
