// nq_codec_math.cuh -- the codec arithmetic shared by the decode kernel and
// the attention kernel (sm_100a): the in-thread Walsh-Hadamard transform of a
// half vector, code unpacking, and the reconstruction x = fp32(w * kappa) of
// one thread's 64 coordinates from a packed vector.
//
// Thread layout: two threads own one 128-vector; half h holds the coordinate
// pairs (x_i, x_{i+64}) for i in [32h, 32h+32) as packed fp32x2 registers.
#pragma once

#include "nq_device.cuh"

namespace nq {

// ------------------------------------------------------ Hadamard (fp32)
// Unnormalised Sylvester transform, stages h = 1, 2, ..., 64 in this order.
// v[j] = (x_{32h+j}, x_{32h+j+64}); stage 32 pairs this thread's j with the
// partner's j (x_i with x_{i+32}); stage 64 is the pair's own butterfly.
// Every output is the IEEE fp32 sum / difference of the same two operands as
// the scalar butterfly network.
__device__ __forceinline__ void fwht_half(float2 (&v)[32], int half) {
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (!(j & s)) {
        const float2 A = v[j], B = v[j + s];
        v[j] = add2(A, B);
        v[j + s] = sub2(A, B);
      }
    }
  }
  // half 0 holds x_i (a), half 1 holds x_{i+32} (b): a+b = fma(a, 1, b) and
  // a-b = fma(b, -1, a), each one rounding of the exact sum or difference
  const float sg = half ? -1.0f : 1.0f;
  const float2 sg2 = make_float2(sg, sg);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, v[j].x, 16),
                                 __shfl_xor_sync(0xffffffffu, v[j].y, 16));
    v[j] = fma2(v[j], sg2, o);
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float a = v[j].x, b = v[j].y;
    v[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
}

// 2^22 + j as an fp32 bit pattern for the code j of coordinate c of a
// 32-coordinate block held in BITS words (code c at bits [BITS*c, BITS*c +
// BITS) of the block's little-endian words): the code is moved to bit 1 with
// one (funnel) shift and masked into the mantissa of 2^22 with one LOP3.
template <int BITS>
__device__ __forceinline__ float code_as_float(const uint32_t (&w)[BITS], int c) {
  const int p = BITS * c;
  const int wi = p >> 5, off = p & 31;
  const int wn = wi + 1 < BITS ? wi + 1 : wi;  // never read past the block
  uint32_t x;
  if (off == 0) {
    x = w[wi] << 1;
  } else if (off + BITS <= 32) {
    x = w[wi] >> (off - 1);
  } else {
    x = __funnelshift_r(w[wi], w[wn], off - 1);
  }
  return __uint_as_float((x & (((1u << BITS) - 1u) << 1)) | 0x4A800000u);
}

// This thread's half of a packed vector, reconstructed in fp32 before RoPE:
// 2q = 2j - 2^b + 2 - h_g from the codes, the unnormalised Hadamard transform
// (exact: integers below 2^10), then x = fp32(w * kappa) with
// kappa = fp32(fp32(sigma / 2) * C).  v[j] = (x_{32h+j}, x_{32h+j+64}).
template <int BITS>
__device__ __forceinline__ void reconstruct_half(const uint32_t (&w)[4 * BITS], uint32_t meta,
                                                 int half, float2 (&v)[32]) {
  // This half's blocks: coordinates [32h, 32h+32) and [64+32h, 96+32h), each
  // BITS words starting at word BITS*h and BITS*(2+h).
  uint32_t wa[BITS], wb[BITS];
#pragma unroll
  for (int k = 0; k < BITS; ++k) {
    wa[k] = half ? w[BITS + k] : w[k];
    wb[k] = half ? w[3 * BITS + k] : w[2 * BITS + k];
  }
  // x = 2^22 + j (the fp32 spacing at 2^22 is 1/2, so the mantissa holds 2j);
  // t = 2x - 2^23 - (2^b - 2) - h, every constant below 2^24: exact.
  constexpr float kBase = -8388608.0f - static_cast<float>((1 << BITS) - 2);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ga = 4 * half + q, gb = 8 + 4 * half + q;
    const float2 kg = make_float2(kBase - static_cast<float>((meta >> ga) & 1u),
                                  kBase - static_cast<float>((meta >> gb) & 1u));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float xa = code_as_float<BITS>(wa, 8 * q + i);
      const float xb = code_as_float<BITS>(wb, 8 * q + i);
      v[8 * q + i] = fma2(make_float2(xa, xb), make_float2(2.0f, 2.0f), kg);
    }
  }
  fwht_half(v, half);
  const float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(meta >> 16)));
  const float kappa = __fmul_rn(__fmul_rn(sig, 0.5f), __uint_as_float(kCBits));
  const float2 k2 = make_float2(kappa, kappa);
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = mul2(v[j], k2);
}

}  // namespace nq
