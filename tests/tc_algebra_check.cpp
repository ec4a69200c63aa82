// Host check of the tensor-core decode's algebra (compiled and run by
// tests/test_tc_algebra.py with the system C++ compiler; no GPU).
//
// 1. tc_unpack / tc_slot: every one of the 128 codes of a vector sits in
//    exactly one f16 slot, as the value 1024 + j * 2^d with j * 2^d < 1024.
// 2. The product the kernel asks of the tensor cores, D[n] = sum_p A[p] B[n][p]
//    with A and B built by the rules of decode_tc_kernel (code slots
//    2^(1-d) H, coset slots 2 h_g against -(1/2) of the group's H row sum,
//    16 constant slots of 1 against the parts of beta_n, each part an f16
//    value), equals the integer transform w = H t, t_k = 2 j_k - 2^b + 2 - h,
//    for every output column and random vectors, and every sum of term
//    magnitudes stays below 2^18 (so fp32 accumulation is exact in any order).
// Exit status 0 when both hold.
#include <cmath>
#include <cstdio>
#include <random>

#include "../e8_lattice_vector_nq_b200/csrc/nq_tc_slots.cuh"

static int parity(unsigned x) { return __builtin_popcount(x) & 1; }

// f16 bits -> value (normal numbers and zero, the only ones used here)
static double f16_value(uint32_t bits) {
  if ((bits & 0x7FFF) == 0) return 0.0;
  const int e = (bits >> 10) & 31, m = bits & 1023;
  const double v = std::ldexp(1.0 + m / 1024.0, e - 15);
  return (bits >> 15) ? -v : v;
}

// an integer of magnitude <= 16384 that is a multiple of 8, as f16 (exact)
static double f16_int(int v, bool* exact) {
  const double x = v;
  if (v != 0) {
    int e;
    std::frexp(std::fabs(x), &e);  // |x| in [2^(e-1), 2^e)
    const double ulp = std::ldexp(1.0, e - 11);
    if (std::fmod(std::fabs(x), ulp) != 0.0) *exact = false;
  }
  return x;
}

// output coordinate of TMEM column n (decode_tc_kernel's tc_coord)
static int coord(int n) { return 2 * (n >> 2) + (n & 1) + 64 * ((n >> 1) & 1); }

template <int B>
static int run() {
  std::mt19937 rng(7 + B);
  int bad = 0;
  bool exact = true;
  // 1. slot map
  for (int it = 0; it < 2000; ++it) {
    uint32_t w[4 * B] = {0};
    int code[128];
    for (int k = 0; k < 128; ++k) {
      code[k] = rng() % (1 << B);
      const int p = B * k;
      w[p >> 5] |= static_cast<uint32_t>(code[k]) << (p & 31);
      if ((p & 31) + B > 32) w[(p >> 5) + 1] |= static_cast<uint32_t>(code[k]) >> (32 - (p & 31));
    }
    uint32_t h[64];
    nq::tc_unpack<B>(w, h);
    int seen[128] = {0};
    for (int p = 0; p < 128; ++p) {
      int c, d;
      nq::tc_slot<B>(p, c, d);
      if (c < 0 || c > 127) { ++bad; continue; }
      ++seen[c];
      const uint32_t bits = (h[p >> 1] >> (16 * (p & 1))) & 0xFFFF;
      if (bits != (0x6400u | (static_cast<uint32_t>(code[c]) << d)) || (code[c] << d) >= 1024) ++bad;
    }
    for (int k = 0; k < 128; ++k) bad += seen[k] != 1;
  }
  // 2. the product
  static double Bm[128][160];
  for (int n = 0; n < 128; ++n) {
    const int cn = coord(n);
    int beta = cn == 0 ? (2 - (1 << B)) * 128 : 0;
    for (int p = 0; p < 128; ++p) {
      int c, d;
      nq::tc_slot<B>(p, c, d);
      const double sgn = parity(cn & c) ? -1.0 : 1.0;
      Bm[n][p] = sgn * std::ldexp(1.0, 1 - d);
      beta += parity(cn & c) ? (1 << (11 - d)) : -(1 << (11 - d));
    }
    for (int g = 0; g < 16; ++g)
      Bm[n][128 + g] = (cn & 7) ? 0.0 : (parity(cn & (8 * g)) ? 4.0 : -4.0);
#ifdef PLANT_COSET_SIGN  // a planted mistake the check must catch
    for (int g = 0; g < 16; ++g) Bm[n][128 + g] = -Bm[n][128 + g];
#endif
    for (int s = 0; s < 16; ++s) {
      const int part = beta > 16384 ? 16384 : (beta < -16384 ? -16384 : beta);
      beta -= part;
      Bm[n][144 + s] = f16_int(part, &exact);
    }
    if (beta != 0) ++bad;
  }
  double maxabs = 0;
  for (int it = 0; it < 1500; ++it) {
    uint32_t w[4 * B] = {0};
    int code[128];
    for (int k = 0; k < 128; ++k) {
      code[k] = rng() % (1 << B);
      const int p = B * k;
      w[p >> 5] |= static_cast<uint32_t>(code[k]) << (p & 31);
      if ((p & 31) + B > 32) w[(p >> 5) + 1] |= static_cast<uint32_t>(code[k]) >> (32 - (p & 31));
    }
    const uint32_t mask = rng() & 0xFFFF;
    uint32_t h[64];
    nq::tc_unpack<B>(w, h);
    double A[160];
    for (int p = 0; p < 128; ++p) A[p] = f16_value((h[p >> 1] >> (16 * (p & 1))) & 0xFFFF);
    const uint32_t y = mask | (mask << 15);  // the kernel's coset slots: 2.0 for a set bit
    for (int u = 0; u < 8; ++u) {
      const uint32_t cw = (y << (14 - 2 * u)) & 0x40004000u;
      A[128 + 2 * u] = f16_value(cw & 0xFFFF);
      A[129 + 2 * u] = f16_value(cw >> 16);
    }
    for (int s = 0; s < 16; ++s) A[144 + s] = 1.0;
    for (int n = 0; n < 128; ++n) {
      const int cn = coord(n);
      double ref = 0, D = 0, mag = 0;
      for (int k = 0; k < 128; ++k) {
        const double t = 2.0 * code[k] - (1 << B) + 2 - ((mask >> (k / 8)) & 1);
        ref += parity(cn & k) ? -t : t;
      }
      for (int p = 0; p < 160; ++p) {
        D += A[p] * Bm[n][p];
        mag += std::fabs(A[p] * Bm[n][p]);
      }
      if (mag > maxabs) maxabs = mag;
      if (D != ref) ++bad;
    }
  }
  if (!exact || maxabs >= 262144.0) ++bad;
  std::printf("bits %d: %d failures, largest sum of term magnitudes %.0f\n", B, bad, maxabs);
  return bad;
}

int main() { return (run<2>() + run<3>()) ? 1 : 0; }
