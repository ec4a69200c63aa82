// nq_codec_math.cuh -- the codec arithmetic shared by the encode, decode and
// attention kernels (sm_100a): the in-thread Walsh-Hadamard transform of a
// half vector, code unpacking, the reconstruction x = fp32(w * kappa) of one
// thread's 64 coordinates from a packed vector, and the staging of the
// two-level RoPE table for tiles of 16 vectors.
//
// Thread layout: two threads own one 128-vector; half h holds the coordinate
// pairs (x_i, x_{i+64}) for i in [32h, 32h+32) as packed fp32x2 registers.
#pragma once

#include "nq_device.cuh"

namespace nq {

constexpr int kSlots = 16;                  // vectors per tile: one warp = 16 slots x 2 halves
constexpr int kCsBytes = 32 * kSlots * 16;  // float4 cs[32][16]

// ------------------------------------------------------ RoPE table rows
// The table holds cos/sin of the angles 256a * theta_i (rows a < n_a) and
// b * theta_i (rows n_a + b, b < 256) as 64 (c, s) pairs per row.  The rows of
// a tile are staged raw: for each of the 16 slots the A row of its position
// p = 256a + b and its B row, 512 bytes each, at a padded stride of kRawSlot
// bytes per slot.  Warp w copies the rows of slots w, w + nwarps, ...: one
// 16-byte chunk per lane per row.  src_lane is the position minus pos_base of
// the lane's slot (lanes l and l+16 share slot l % 16), -1 for an empty slot.
constexpr int kRawSlot = 1024 + 16;
constexpr int kRawBytes = kSlots * kRawSlot;

__device__ __forceinline__ void issue_rope_rows(const float2* tab, int64_t n_a, int64_t pos_base,
                                                int32_t src_lane, uint32_t raw, int warp,
                                                int nwarps, int lane) {
  for (int slot = warp; slot < kSlots; slot += nwarps) {  // warp-uniform
    const int32_t src = __shfl_sync(0xffffffffu, src_lane, slot);
    if (src < 0) continue;
    const int64_t pos = pos_base + src;
    int64_t hi = pos >> 8;
    hi = hi < 0 ? 0 : (hi >= n_a ? n_a - 1 : hi);  // out-of-contract positions stay in bounds
    const char* rowA = reinterpret_cast<const char*>(tab + hi * kHalf);
    const char* rowB = reinterpret_cast<const char*>(tab + (n_a + (pos & 255)) * kHalf);
    const uint32_t dst = raw + slot * kRawSlot + lane * 16;
    cp_async16(dst, rowA + lane * 16);
    cp_async16(dst + 512, rowB + lane * 16);
  }
}

// cs table of one tile from its raw rows: float4 cs[j][slot] = (c_2j, s_2j,
// c_2j+1, s_2j+1) with c = fmaf(cA, cB, -(sA sB)), s = fmaf(sA, cB, cA sB)
// (the angle-sum rule); a thread of half h later reads j in [16h, 16h+16).
__device__ __forceinline__ void combine_rope_rows(uint32_t raw, float4* cs, int tid,
                                                  int nthreads) {
  for (int e = tid; e < 32 * kSlots; e += nthreads) {
    const int slot = e & 15, j = e >> 4;
    const float4 A = lds128f(raw + slot * kRawSlot + j * 16);
    const float4 B = lds128f(raw + slot * kRawSlot + 512 + j * 16);
    float4 v;
    v.x = __fmaf_rn(A.x, B.x, -__fmul_rn(A.y, B.y));
    v.y = __fmaf_rn(A.y, B.x, __fmul_rn(A.x, B.y));
    v.z = __fmaf_rn(A.z, B.z, -__fmul_rn(A.w, B.w));
    v.w = __fmaf_rn(A.w, B.z, __fmul_rn(A.z, B.w));
    cs[j * kSlots + slot] = v;
  }
}

// Rotation of this thread's half vector at its position:
// o_i = fmaf(x_i, c, -(x_{i+64} s)), o_{i+64} = fmaf(x_{i+64}, c, x_i s), with
// (c, s) read from the cs table at csa = cs + (16 half * kSlots + slot) * 16.
__device__ __forceinline__ void rope_half(float2 (&v)[32], uint32_t csa) {
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) {
    const float4 t = lds128f(csa + jj * (kSlots * 16));
#pragma unroll
    for (int ww = 0; ww < 2; ++ww) {
      const float c = ww ? t.z : t.x, s = ww ? t.w : t.y;
      const float2 P = v[2 * jj + ww];
      const float2 Q = mul2(P, make_float2(s, s));
      v[2 * jj + ww] = make_float2(__fmaf_rn(P.x, c, -Q.y), __fmaf_rn(P.y, c, Q.x));
    }
  }
}

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
