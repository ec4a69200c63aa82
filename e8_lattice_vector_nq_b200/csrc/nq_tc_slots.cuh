// nq_tc_slots.cuh -- the order in which the tensor-core decode feeds a
// vector's 128 b-bit codes to the MMA as f16 values (host and device).
//
// A code j sits in the mantissa of an f16 whose exponent field is that of
// 1024: bits 0x6400 | (j << d) are the value 1024 + j * 2^d, exact for
// j * 2^d < 1024.  Two codes share a 32-bit register (lanes at bits 0 and 16),
// so one AND with a two-field mask and one OR with 0x64006400 turn a shifted
// view of the packed code string into an f16 pair.  Since a 3-bit field never
// starts 16 bits after another, the two lanes take codes at different
// mantissa shifts d, and the MMA's B operand undoes each slot's 2^d (a power
// of two, exact).  The slot order is free: the B operand's rows are permuted
// to match, so tc_unpack emits whatever the masks produce and tc_slot tells
// which code and shift each slot holds.
//
//  * b = 2: word m holds codes 16m .. 16m+15; masks at bits (2i, 16 + 2i),
//    i = 0..4, give the pairs (16m + i, 16m + 8 + i) with d = 2i; the word
//    shifted right by 10 gives (16m + 5 + i, 16m + 13 + i), d = 2i, i = 0..2.
//  * b = 3: for a = 0, 10, ..., 110, the window starting one bit before code
//    a gives (a + r, a + 5 + r) with d = (3r + 1, 3r), r = 0..2, and the
//    window one bit before code a + 3 gives (a + 3 + r, a + 8 + r), r = 0..1;
//    codes 120..127 take one window before code 120 (three pairs) and one
//    pair (123, 124) assembled from two windows with a byte permute.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define NQ_HD __host__ __device__ __forceinline__
#else
#define NQ_HD inline
#endif

namespace nq {

constexpr uint32_t kF16Pair1024 = 0x64006400u;  // f16 pair (1024, 1024)

NQ_HD uint32_t shr_funnel(uint32_t lo, uint32_t hi, int s) {  // bits [s, s+32) of hi:lo
#if defined(__CUDA_ARCH__)
  return __funnelshift_r(lo, hi, s);
#else
  return s == 0 ? lo : (lo >> s) | (hi << (32 - s));
#endif
}

NQ_HD uint32_t perm_bytes(uint32_t x, uint32_t y, uint32_t sel) {
#if defined(__CUDA_ARCH__)
  return __byte_perm(x, y, sel);
#else
  const uint64_t v = (static_cast<uint64_t>(y) << 32) | x;
  uint32_t r = 0;
  for (int i = 0; i < 4; ++i) r |= static_cast<uint32_t>((v >> (8 * ((sel >> (4 * i)) & 7))) & 0xFF) << (8 * i);
  return r;
#endif
}

// Bits [s, s + 32) of the vector's code string (code k at bits [b k, b k + b)
// of its little-endian words), zeros outside it; s >= -31.
template <int BITS>
NQ_HD uint32_t code_window(const uint32_t (&w)[4 * BITS], int s) {
  if (s < 0) return w[0] << (-s);
  const int i = s >> 5, o = s & 31;
  const uint32_t lo = w[i], hi = i + 1 < 4 * BITS ? w[i + 1] : 0u;
  return o == 0 ? lo : shr_funnel(lo, hi, o);
}

NQ_HD uint32_t f16_pair(uint32_t v, uint32_t mask) { return (v & mask) | kF16Pair1024; }

// The 128 codes as 64 f16 pairs, h[q] = slots 2q (low half) and 2q + 1.
template <int BITS>
NQ_HD void tc_unpack(const uint32_t (&w)[4 * BITS], uint32_t (&h)[64]) {
  if (BITS == 2) {
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint32_t v0 = w[m], v1 = w[m] >> 10;
#pragma unroll
      for (int i = 0; i < 5; ++i) h[8 * m + i] = f16_pair(v0, (3u << (2 * i)) | (3u << (16 + 2 * i)));
#pragma unroll
      for (int i = 0; i < 3; ++i)
        h[8 * m + 5 + i] = f16_pair(v1, (3u << (2 * i)) | (3u << (16 + 2 * i)));
    }
  } else {
#pragma unroll
    for (int blk = 0; blk < 12; ++blk) {
      const int a = 10 * blk;
      const uint32_t v1 = code_window<BITS>(w, 3 * a - 1), v2 = code_window<BITS>(w, 3 * a + 8);
#pragma unroll
      for (int r = 0; r < 3; ++r) h[5 * blk + r] = f16_pair(v1, (7u << (3 * r + 1)) | (7u << (16 + 3 * r)));
#pragma unroll
      for (int r = 0; r < 2; ++r)
        h[5 * blk + 3 + r] = f16_pair(v2, (7u << (3 * r + 1)) | (7u << (16 + 3 * r)));
    }
    const uint32_t v1 = code_window<BITS>(w, 359);
#pragma unroll
    for (int r = 0; r < 3; ++r) h[60 + r] = f16_pair(v1, (7u << (3 * r + 1)) | (7u << (16 + 3 * r)));
    // code 123 at bit 0 of one window, code 124 at bit 16 of another
    const uint32_t v = perm_bytes(code_window<BITS>(w, 369), code_window<BITS>(w, 356), 0x7610u);
    h[63] = f16_pair(v, 7u | (7u << 16));
  }
}

// Slot p (0..127) -> the code it holds and its mantissa shift d.
template <int BITS>
NQ_HD void tc_slot(int p, int& code, int& shift) {
  const int q = p >> 1, lane = p & 1;
  if (BITS == 2) {
    const int m = q >> 3, i = q & 7;
    code = 16 * m + i + 8 * lane;
    shift = 2 * (i < 5 ? i : i - 5);
  } else if (q < 63) {
    const int blk = q < 60 ? q / 5 : 12, r5 = q < 60 ? q % 5 : q - 60;
    const int r = r5 < 3 ? r5 : r5 - 3;
    code = 10 * blk + r5 + 5 * lane;
    shift = lane ? 3 * r : 3 * r + 1;
  } else {
    code = 123 + lane;
    shift = 0;
  }
}

}  // namespace nq
