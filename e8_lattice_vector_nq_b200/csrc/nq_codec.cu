// nq_codec.cu -- E8 lattice encode / decode kernels for sm_100a.
//
// Method: NexusQuant ("NexusQuant: training-free 10-33x KV cache
// compression", zingnex.cn, sections "E8 lattice quantisation" and
// "Implementation details"; "Como comprimir o KV cache do seu LLM em 33x sem
// treino", dev.to, "Como funciona", steps 3-5): remove RoPE from the kept
// keys, rotate every 128-vector with a Walsh-Hadamard transform, scale it by
// one fp16 absmax scale, snap each group of 8 coordinates to the nearest E8
// point (Conway-Sloane, D8 u D8+1/2), clamp to b-bit codes and pack; decode
// inverts the chain and writes bf16.
//
// Design (B200).  Two threads own one 128-coordinate vector: half h holds
// the coordinate pairs (i, i+64) for i in [32h, 32h+32) as packed fp32x2
// registers.  With that layout the RoPE pairs, the Hadamard stages 1..16 and
// 64, and the E8 groups all stay inside a thread; only Hadamard stage 32
// crosses to the partner lane (lane ^ 16, one shuffle per coordinate).  The
// two lanes of an fp32x2 register hold groups g and g+8, so the E8 search
// runs two groups per packed instruction (__fadd2_rn / __ffma2_rn /
// __fmul2_rn: per-lane IEEE round-to-nearest, the same bits as scalar code).
// A persistent CTA of HG warps (HG heads) walks tiles of 16 slots x HG heads
// (encode: 16 (unit, slot) pairs of the flat pair list, so a tile may span
// units; decode: 16 slots of one unit).  The E8 decision is taken from the
// integer coset's rounding alone when the two coset distances are clearly
// apart, with the full two-coset decision as the exact fallback (e8_choose).
// Encode stages the input rows with warp-cooperative 16-byte async copies
// (each warp instruction moves two whole 256-byte rows, gathered through the
// kept list) into padded shared-memory rows, double buffered, so the loads of
// tile k+2 overlap the arithmetic of tile k; the RoPE (cos, sin) pairs of a
// tile are combined once per CTA from table rows staged a tile ahead and
// shared by its heads.  Decode loads the next tile's codes one tile ahead,
// double-buffers the table rows (one CTA barrier per tile) and writes each
// warp's 16 reconstructed rows into a 128-byte-swizzled shared tile that one
// lane stores with two TMA tensor stores (cp.async.bulk.tensor, 4-D map of the
// output).  Every (bits, RoPE) variant is its own kernel: keys and values are
// two launches.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "nq_codec_math.cuh"
#include "nq_internal.h"
#include "nq_tc_slots.cuh"
#include "nq_tcgen05.cuh"

namespace nq {

// Division by a fixed divisor for numerators below 2^31 (round-up method of
// Granlund and Montgomery): q = (n * m) >> (31 + l), l = ceil(log2 d),
// m = floor(2^(31+l) / d) + 1.
struct FastDiv {
  uint64_t m;
  uint32_t d, shift;
};

static FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  FastDiv f;
  f.d = d;
  f.shift = 31 + l;
  f.m = ((1ull << f.shift) / d) + 1;
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return static_cast<uint32_t>((static_cast<uint64_t>(n) * f.m) >> f.shift);
}

struct CodecArgs {
  const uint16_t* kv;  // encode: bf16 input; decode: bf16 output
  int64_t su, sh, st;  // element strides of the bf16 tensor
  uint32_t* codes;
  uint32_t* meta;
  int64_t pu, ph;      // vector strides of the packed store
  int heads, hg, ngroups;
  int64_t T_in;        // encode: input tokens per (unit, head)
  int64_t n, slot0, pos_base;
  const int32_t* idx;  // encode: kept (source tokens); decode: positions
  int64_t idx_stride;
  const float2* tab;
  int64_t n_a;
  int64_t slot_tiles, num_tiles;
  FastDiv div_groups, div_stiles;
  int64_t pairs;  // encode: units * n (unit, slot) pairs, below 2^31
  FastDiv div_n;  // encode: division by n
  // tensor-core decode: a tile holds tc_m slot tiles of one head group
  int tc_m;
  int64_t tc_sgroups;  // ceil(slot_tiles / tc_m)
  FastDiv div_sgroups;
};

struct Tile {
  int group, unit;
  int64_t stile;
};

// Tile index -> (unit, slot tile, head group); tile counts stay below 2^31.
__device__ __forceinline__ Tile tile_of(const CodecArgs& a, int64_t t64) {
  const uint32_t t = static_cast<uint32_t>(t64);
  const uint32_t q = fdiv(t, a.div_groups);
  const uint32_t u = fdiv(q, a.div_stiles);
  Tile r;
  r.group = static_cast<int>(t - q * a.div_groups.d);
  r.stile = static_cast<int64_t>(q - u * a.div_stiles.d);
  r.unit = static_cast<int>(u);
  return r;
}

// Source token of slot stile * 16 + slot_l of a unit: the kept-list entry, or
// the slot itself; -1 past the last slot.
__device__ __forceinline__ int32_t slot_src_at(const CodecArgs& a, int unit, int64_t stile,
                                               int slot_l) {
  const int64_t slot = stile * kSlots + slot_l;
  if (slot >= a.n) return -1;
  return a.idx ? __ldg(a.idx + static_cast<int64_t>(unit) * a.idx_stride + slot)
               : static_cast<int32_t>(slot);
}
// The same for this lane's slot (lanes l and l+16 share slot l % 16) in tile tl.
__device__ __forceinline__ int32_t slot_src(const CodecArgs& a, const Tile& tl, int slot_l) {
  return slot_src_at(a, tl.unit, tl.stile, slot_l);
}

// Encode tiles walk the (unit, slot) pairs of all units as one list, 16 pairs
// per tile (pair p = unit * n + slot), so a tile may span units: an append of
// one token per unit fills whole tiles.  Tile index -> (head group, p0).
struct EncTile {
  int group;
  int64_t p0;
};
__device__ __forceinline__ EncTile enc_tile(const CodecArgs& a, int64_t t64) {
  const uint32_t t = static_cast<uint32_t>(t64);
  const uint32_t q = fdiv(t, a.div_groups);
  EncTile r;
  r.group = static_cast<int>(t - q * a.div_groups.d);
  r.p0 = static_cast<int64_t>(q) * kSlots;
  return r;
}
// This lane's pair of a tile (lanes l and l+16 share pair p0 + l % 16).
struct EncPair {
  bool valid;
  int64_t unit, slot;
};
__device__ __forceinline__ EncPair enc_pair(const CodecArgs& a, int64_t p0, int slot_l) {
  EncPair e;
  const int64_t p = p0 + slot_l;
  e.valid = p < a.pairs;
  const uint32_t pp = static_cast<uint32_t>(e.valid ? p : 0);
  const uint32_t u = fdiv(pp, a.div_n);
  e.unit = u;
  e.slot = static_cast<int64_t>(pp) - static_cast<int64_t>(u) * a.n;
  return e;
}
// Source token of a pair (its RoPE position is pos_base + src), -1 if invalid.
__device__ __forceinline__ int32_t enc_src(const CodecArgs& a, const EncPair& e) {
  if (!e.valid) return -1;
  return a.idx ? __ldg(a.idx + e.unit * a.idx_stride + e.slot) : static_cast<int32_t>(e.slot);
}

// ---------------------------------------------------------- E8 (fp32x2)
// Nearest E8 point of two groups at once (lane x: group g, lane y: group
// g+8), Conway-Sloane: per coset (shift 0 and 1/2) u = y - shift, f = rint(u)
// (ties to even via the 1.5*2^23 trick), e = u - f, d = e0^2 then an fma
// chain, an odd sum of f adds 1 - 2 max|e| (moving the first largest-error
// coordinate toward u); the half coset wins only when strictly closer.
// e8_decide is that decision written out for both cosets; e8_choose reaches
// the same decision from the integer coset alone when the two distances are
// not close, and e8_codes then recomputes the chosen coset and packs it.
// e8_decide returns, per lane, whether the half coset wins, whether its
// coordinate sum was odd (a fix is needed) and the largest rounding error of
// the chosen coset.
struct E8Choice {
  float2 hh;     // 1 for the half coset, 0 for the integer coset
  float mx, my;  // largest |e| of the chosen coset
  bool oddx, oddy;
};

__device__ __forceinline__ E8Choice e8_decide(const float2 (&y)[8]) {
  const float2 M2 = make_float2(kMagicRound, kMagicRound);
  const float2 H2 = make_float2(0.5f, 0.5f);
  float2 d0 = make_float2(0.f, 0.f), d1 = make_float2(0.f, 0.f);
  float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);  // sums of f (exact)
  float m0x = 0.f, m0y = 0.f, m1x = 0.f, m1y = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f0 = sub2(add2(y[i], M2), M2);
    const float2 e0 = sub2(y[i], f0);
    const float2 u = sub2(y[i], H2);
    const float2 f1 = sub2(add2(u, M2), M2);
    const float2 e1 = sub2(u, f1);
    s0 = add2(s0, f0);
    s1 = add2(s1, f1);
    d0 = i == 0 ? mul2(e0, e0) : fma2(e0, e0, d0);
    d1 = i == 0 ? mul2(e1, e1) : fma2(e1, e1, d1);
    m0x = fmaxf(m0x, fabsf(e0.x));
    m0y = fmaxf(m0y, fabsf(e0.y));
    m1x = fmaxf(m1x, fabsf(e1.x));
    m1y = fmaxf(m1y, fabsf(e1.y));
  }
  // parity of an integer-valued sum: the LSB of its 1.5*2^23-biased bits
  const float2 b0 = add2(s0, M2), b1 = add2(s1, M2);
  const bool o0x = __float_as_uint(b0.x) & 1u, o0y = __float_as_uint(b0.y) & 1u;
  const bool o1x = __float_as_uint(b1.x) & 1u, o1y = __float_as_uint(b1.y) & 1u;
  const float2 m0 = make_float2(m0x, m0y), m1 = make_float2(m1x, m1y);
  const float2 fix0 = add2(d0, fma2(make_float2(-2.f, -2.f), m0, make_float2(1.f, 1.f)));
  const float2 fix1 = add2(d1, fma2(make_float2(-2.f, -2.f), m1, make_float2(1.f, 1.f)));
  const float D0x = o0x ? fix0.x : d0.x, D0y = o0y ? fix0.y : d0.y;
  const float D1x = o1x ? fix1.x : d1.x, D1y = o1y ? fix1.y : d1.y;
  const bool halfx = D1x < D0x, halfy = D1y < D0y;
  E8Choice c;
  c.hh = make_float2(halfx ? 1.f : 0.f, halfy ? 1.f : 0.f);
  c.mx = halfx ? m1x : m0x;
  c.my = halfy ? m1y : m0y;
  c.oddx = halfx ? o1x : o0x;
  c.oddy = halfy ? o1y : o0y;
  return c;
}

// max of eight non-negative values as chains of three-input maxima.
__device__ __forceinline__ float max8(const float (&a)[8]) {
  return fmaxf(fmaxf(fmaxf(fmaxf(a[0], a[1]), a[2]), fmaxf(fmaxf(a[3], a[4]), a[5])),
               fmaxf(a[6], a[7]));
}

// fp32 fma with the result saturated to [0, 1] (one instruction).
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Coset choice without the half coset's rounding.  Let e = y - rint(y) (exact)
// and a_i = |e_i|.  Up to the rounding of y - 1/2 (below 2^-22 for |y| < 8)
// the half coset's errors are 1/2 - a_i, so in exact arithmetic
//   d1 - d0 = 2 - sum(a) + odd1 * 2 min(a) - odd0 * (1 - 2 max(a)),
// with odd0 the parity of sum rint(y) (the LSB of each 1.5*2^23-biased value)
// and, once every a_i >= 2^-20 (so that the rounding of y - 1/2 cannot move
// its nearest integer), odd1 = odd0 xor (number of negative e_i).  The
// decoder's two fp32 distances (eight fma roundings each on sums <= 2, plus
// the fix term and the y - 1/2 roundings) and this fp32 estimate each stay
// within 4e-6 of their exact values, so when the estimate is at least 6e-5
// away from zero its sign is the sign of the fp32 comparison d1 < d0.  Any
// other lane makes its warp run the full two-coset decision (e8_decide).
// Per lane: whether the half coset wins and whether its rounded sum is odd.
constexpr float kFastMargin = 6e-5f;
constexpr float kFastMinErr = 9.5367431640625e-7f;  // 2^-20

__device__ __forceinline__ void e8_fast_lane(const float (&a)[8], const uint32_t (&tb)[8],
                                             const uint32_t (&eb)[8], bool& half, bool& odd,
                                             bool& slow) {
  const float A = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  const float mx = max8(a);
  const float mn = fminf(fminf(fminf(fminf(a[0], a[1]), a[2]), fminf(fminf(a[3], a[4]), a[5])),
                         fminf(a[6], a[7]));
  const uint32_t P = (tb[0] ^ tb[1] ^ tb[2]) ^ (tb[3] ^ tb[4] ^ tb[5]) ^ (tb[6] ^ tb[7]);
  const uint32_t S = (eb[0] ^ eb[1] ^ eb[2]) ^ (eb[3] ^ eb[4] ^ eb[5]) ^ (eb[6] ^ eb[7]);
  const bool odd0 = P & 1u;
  const bool odd1 = odd0 ^ static_cast<bool>(S >> 31);
  float d = __fsub_rn(2.0f, A);
  if (odd1) d = __fmaf_rn(2.0f, mn, d);
  if (odd0) d = __fsub_rn(d, __fmaf_rn(-2.0f, mx, 1.0f));
  slow = !(fabsf(d) >= kFastMargin) || !(mn >= kFastMinErr);
  half = d < 0.0f;
  odd = half ? odd1 : odd0;
}

// Coset and parity of the chosen coset for the two groups of y (lanes x, y).
// The estimate above needs |y| < 7 (the y - 1/2 rounding bound); a lane whose
// groups may exceed it passes force and always takes the full decision.
__device__ __forceinline__ void e8_choose(const float2 (&y)[8], bool force, bool& halfx,
                                          bool& halfy, bool& oddx, bool& oddy) {
  const float2 M2 = make_float2(kMagicRound, kMagicRound);
  float ax[8], ay[8];
  uint32_t tx[8], ty[8], ex[8], ey[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 t = add2(y[i], M2);
    const float2 e = sub2(y[i], sub2(t, M2));
    ax[i] = fabsf(e.x);
    ay[i] = fabsf(e.y);
    tx[i] = __float_as_uint(t.x);
    ty[i] = __float_as_uint(t.y);
    ex[i] = __float_as_uint(e.x);
    ey[i] = __float_as_uint(e.y);
  }
  bool slowx, slowy;
  e8_fast_lane(ax, tx, ex, halfx, oddx, slowx);
  e8_fast_lane(ay, ty, ey, halfy, oddy, slowy);
  slowx = slowx || force;
  slowy = slowy || force;
  if (__any_sync(0xffffffffu, slowx || slowy)) {
    const E8Choice c = e8_decide(y);
    if (slowx) {
      halfx = c.hh.x != 0.f;
      oddx = c.oddx;
    }
    if (slowy) {
      halfy = c.hh.y != 0.f;
      oddy = c.oddy;
    }
  }
}

// Codes of the chosen cosets for the two groups of y (lanes x, y): the
// coset's rounding is recomputed (U = y - shift with a +0 shift for the
// integer coset, so U is never -0; F = rint(U), E = U - F), m = max |E|; when
// the sum was odd the first coordinate with |E| = m moves one step toward U
// (E >= 0: up).  The clamp to [lo, lo + R] (R = 2^b - 1 for the half coset,
// 2^b - 2 for the integer one) and the code j = F - lo come from
// a = sat((F - lo) / R), evaluated as one saturating fma with fp32 1/R and
// -lo/R (error below 1e-6 in a*R for |F| < 8, so a*R + 2^23 rounds to
// 2^23 + j exactly; values beyond the range saturate to 0 or 1), then
// J = fma(a, R, 2^23), whose low mantissa bits hold j.  Code i is packed at
// bits [BITS*i, BITS*i + BITS).
template <int BITS>
__device__ __forceinline__ void e8_codes(const float2 (&y)[8], bool halfx, bool halfy, bool oddx,
                                         bool oddy, uint32_t& gx, uint32_t& gy) {
  const float2 M2 = make_float2(kMagicRound, kMagicRound);
  constexpr float kRH = static_cast<float>((1 << BITS) - 1);
  constexpr float kRI = static_cast<float>((1 << BITS) - 2);
  constexpr float kInvH = 1.0f / kRH, kInvI = 1.0f / kRI;
  constexpr float kCH = static_cast<float>(1 << (BITS - 1)) / kRH;
  constexpr float kCI = static_cast<float>((1 << (BITS - 1)) - 1) / kRI;
  // per-lane coset constants from the coset flag hf in {0, 1} with packed fmas
  // (1/R and -lo/R need not be exact: only a*R + 2^23 must round to 2^23 + j)
  const float2 hf = make_float2(halfx ? 1.0f : 0.0f, halfy ? 1.0f : 0.0f);
  const float2 sh = fma2(hf, make_float2(-1.0f, -1.0f), make_float2(0.0f, 0.0f));
  const float2 H2 = make_float2(0.5f, 0.5f);
  float2 F[8], E[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 U = fma2(sh, H2, y[i]);
    F[i] = sub2(add2(U, M2), M2);
    E[i] = sub2(U, F[i]);
  }
  float ex[8], ey[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ex[i] = fabsf(E[i].x);
    ey[i] = fabsf(E[i].y);
  }
  const float mx = max8(ex), my = max8(ey);
  const float2 R2 = add2(hf, make_float2(kRI, kRI));
  const float2 i2 = fma2(hf, make_float2(kInvH - kInvI, kInvH - kInvI), make_float2(kInvI, kInvI));
  const float2 c2 = fma2(hf, make_float2(kCH - kCI, kCH - kCI), make_float2(kCI, kCI));
  const float ix = i2.x, iy = i2.y, cx = c2.x, cy = c2.y;
  const float2 B2 = make_float2(kTwo23, kTwo23);
  bool fx = !oddx, fy = !oddy;  // "fix done" flags
  uint32_t ax = 0u, ay = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float2 f = F[i];
    const bool hitx = !fx && ex[i] == mx;
    const bool hity = !fy && ey[i] == my;
    fx = fx || hitx;
    fy = fy || hity;
    if (hitx) f.x = __fadd_rn(f.x, copysignf(1.0f, E[i].x));
    if (hity) f.y = __fadd_rn(f.y, copysignf(1.0f, E[i].y));
    const float2 a2 = make_float2(fma_sat(f.x, ix, cx), fma_sat(f.y, iy, cy));
    const float2 J = fma2(a2, R2, B2);  // 2^23 + code: the code sits in the low mantissa bits
    ax = mad_u32(__float_as_uint(J.x), 1u << (BITS * i), ax);
    ay = mad_u32(__float_as_uint(J.y), 1u << (BITS * i), ay);
  }
  constexpr uint32_t kMask = (1u << (8 * BITS)) - 1u;
  gx = ax & kMask;
  gy = ay & kMask;
}

// ------------------------------------------- E8 inside the code box (fp32x2)
// The exact (24/16-bit) packing stores each group's coset bit in place of the
// low bit of its last code, which needs every coded point in E8: the nearest
// E8 point inside the b-bit code box, per coset the Conway-Sloane D8 step with
// the box.  For two groups at once (lanes x, y) and one coset (shift 0, f in
// [-(2^(b-1)-1), 2^(b-1)-1]; shift 1/2, f in [-2^(b-1), 2^(b-1)-1]):
// u = y - shift, f = clamp(rint(u), lo, hi) (ties to even), e = u - f (exact),
// d = e0^2 then an fma chain; when the sum of f is odd, the one coordinate
// whose move by dir = (e >= 0 ? +1 : -1), reversed when that leaves the box,
// costs least moves, cost fmaf(-2 dir, e, 1), the first index on ties, and d
// gains that cost.  The half coset wins only when strictly closer.
// The move for one lane, without branches (a lane-dependent branch here made
// warps run both paths): every coordinate's move and cost, then the first
// coordinate of least cost moves and d gains that cost, only when the sum is
// odd.  The first index attaining the minimum is the one a scan keeping the
// first strictly smaller cost finds.
__device__ __forceinline__ void box_fix_bf(float (&f)[8], const float (&e)[8], float lo, float hi,
                                           bool odd, float& d) {
  float c[8], u[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool p = e[i] >= 0.0f;
    float v = p ? 1.0f : -1.0f;
    if (f[i] == (p ? hi : lo)) v = -v;  // f is on the grid in [lo, hi]: f + dir leaves it
    c[i] = __fmaf_rn(-2.0f * v, e[i], 1.0f);
    u[i] = v;
  }
  const float m = fminf(fminf(fminf(fminf(c[0], c[1]), c[2]), fminf(fminf(c[3], c[4]), c[5])),
                        fminf(c[6], c[7]));
  bool done = !odd;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hit = !done && c[i] == m;
    done = done || hit;
    if (hit) f[i] = __fadd_rn(f[i], u[i]);
  }
  if (odd) d = __fadd_rn(d, m);
}

__device__ __forceinline__ void d8_box2(const float2 (&y)[8], float shift, float lo, float hi,
                                        float (&fx)[8], float (&fy)[8], float& dx, float& dy) {
  const float2 M2 = make_float2(kMagicRound, kMagicRound);
  const float2 S2 = make_float2(-shift, -shift);
  float ex[8], ey[8];
  float2 d = make_float2(0.f, 0.f), sum = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 u = add2(y[i], S2);  // y + (-shift): the rounding of y - shift
    const float2 r = sub2(add2(u, M2), M2);
    const float2 f = make_float2(fminf(fmaxf(r.x, lo), hi), fminf(fmaxf(r.y, lo), hi));
    const float2 e = sub2(u, f);
    d = i == 0 ? mul2(e, e) : fma2(e, e, d);
    sum = add2(sum, f);
    fx[i] = f.x;
    fy[i] = f.y;
    ex[i] = e.x;
    ey[i] = e.y;
  }
  const float2 b = add2(sum, M2);  // parity of the integer sum: LSB of the biased value
  dx = d.x;
  dy = d.y;
  box_fix_bf(fx, ex, lo, hi, __float_as_uint(b.x) & 1u, dx);
  box_fix_bf(fy, ey, lo, hi, __float_as_uint(b.y) & 1u, dy);
}

// Folded codes of two groups (lanes x, y) at their nearest E8 point inside the
// box: code j = f - lo of the chosen coset at bits [b i, b i + b), then the low
// bit of code 7 replaced by the coset bit (1 = half coset).
template <int BITS>
__device__ __forceinline__ void e8_box_codes(const float2 (&y)[8], uint32_t& gx, uint32_t& gy) {
  constexpr float kH = static_cast<float>(1 << (BITS - 1));
  float f0x[8], f0y[8], f1x[8], f1y[8], d0x, d0y, d1x, d1y;
  d8_box2(y, 0.0f, 1.0f - kH, kH - 1.0f, f0x, f0y, d0x, d0y);
  d8_box2(y, 0.5f, -kH, kH - 1.0f, f1x, f1y, d1x, d1y);
  const bool hx = d1x < d0x, hy = d1y < d0y;
  uint32_t ax = 0u, ay = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // 2^23 + j, exact: the code sits in the low mantissa bits
    const float jx = hx ? __fadd_rn(f1x[i], kH + kTwo23) : __fadd_rn(f0x[i], kH - 1.0f + kTwo23);
    const float jy = hy ? __fadd_rn(f1y[i], kH + kTwo23) : __fadd_rn(f0y[i], kH - 1.0f + kTwo23);
    ax = mad_u32(__float_as_uint(jx), 1u << (BITS * i), ax);
    ay = mad_u32(__float_as_uint(jy), 1u << (BITS * i), ay);
  }
  constexpr uint32_t kMask = (1u << (8 * BITS)) - 1u;
  constexpr uint32_t kCos = 1u << (7 * BITS);
  gx = ((ax & kMask) & ~kCos) | (hx ? kCos : 0u);
  gy = ((ay & kMask) & ~kCos) | (hy ? kCos : 0u);
}

// --------------------------------------------------------------- encode
// Staged bf16 row -> this half's 64 coordinates; keys: RoPE removed.
template <bool ROPE>
__device__ __forceinline__ void load_half(float2 (&v)[32], uint32_t row, uint32_t csa, int half) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 A = lds128(row + 16 * (4 * half + q));      // x_{32h+8q .. +7}
    const uint4 B = lds128(row + 16 * (8 + 4 * half + q));  // x_{64+32h+8q .. +7}
    const uint32_t a[4] = {A.x, A.y, A.z, A.w}, b[4] = {B.x, B.y, B.z, B.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      v[8 * q + 2 * t] = make_float2(bf16lo(a[t]), bf16lo(b[t]));
      v[8 * q + 2 * t + 1] = make_float2(bf16hi(a[t]), bf16hi(b[t]));
    }
  }
  if (ROPE) {
    // u_i = fmaf(k_i, c, k_{i+64} s),  u_{i+64} = fmaf(k_{i+64}, c, -(k_i s))
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const float4 t = lds128f(csa + jj * (kSlots * 16));
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const float c = w ? t.z : t.x, s = w ? t.w : t.y;
        const float2 P = v[2 * jj + w];
        const float2 Q = mul2(P, make_float2(s, s));
        v[2 * jj + w] = make_float2(__fmaf_rn(P.x, c, Q.y), __fmaf_rn(P.y, c, -Q.x));
      }
    }
  }
}

// Rotation, scale, E8 step and packing of this thread's half vector; the meta
// word (regular layout) or the fp16 scale (exact layout) is written by half 0.
template <int BITS, bool EXACT>
__device__ __forceinline__ void quantise_half(float2 (&v)[32], int half, bool valid,
                                              uint32_t* codes, void* meta) {
  fwht_half(v, half);
  float m4[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four chains for latency
#pragma unroll
  for (int j = 0; j < 32; ++j) m4[j & 3] = fmaxf(fmaxf(m4[j & 3], fabsf(v[j].x)), fabsf(v[j].y));
  float M = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));
  const float G = __uint_as_float(BITS == 3 ? kG3Bits : kG2Bits);
  const float C = __uint_as_float(kCBits);
  const float P = __fmul_rn(M, G);
  const __half sh = __float2half_rn(fminf(P, 65504.0f));
  // Unsaturated, sigma >= P / 1.5 (fp16 subnormals included), so |y| <=
  // 1.5 * A_b <= 5.25; a saturated scale can leave |y| larger.
  const bool big = !(P <= 65504.0f);
  const float sig = __half2float(sh);
  const float r = (sig == 0.0f) ? 0.0f : __fdiv_rn(C, sig);
  const float2 r2 = make_float2(r, r);

  uint32_t gx[4], gy[4];
  uint32_t cm = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float2 y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = mul2(v[8 * q + i], r2);
    if (EXACT) {
      e8_box_codes<BITS>(y, gx[q], gy[q]);
    } else {
      bool hx, hy, ox, oy;
      e8_choose(y, big, hx, hy, ox, oy);
      e8_codes<BITS>(y, hx, hy, ox, oy, gx[q], gy[q]);
      cm |= (static_cast<uint32_t>(hx) << (4 * half + q)) |
            (static_cast<uint32_t>(hy) << (8 + 4 * half + q));
    }
  }
  if (!EXACT) cm |= __shfl_xor_sync(0xffffffffu, cm, 16);
  if (!valid) return;
  if (BITS == 3) {
    // groups 4h..4h+3 -> words 3h..3h+2; groups 8+4h.. -> words 6+3h..
    const uint32_t a0 = gx[0] | (gx[1] << 24), a1 = (gx[1] >> 8) | (gx[2] << 16),
                   a2 = (gx[2] >> 16) | (gx[3] << 8);
    const uint32_t b0 = gy[0] | (gy[1] << 24), b1 = (gy[1] >> 8) | (gy[2] << 16),
                   b2 = (gy[2] >> 16) | (gy[3] << 8);
    if (half == 0) {
      *reinterpret_cast<uint2*>(codes + 0) = make_uint2(a0, a1);
      codes[2] = a2;
      *reinterpret_cast<uint2*>(codes + 6) = make_uint2(b0, b1);
      codes[8] = b2;
    } else {
      codes[3] = a0;
      *reinterpret_cast<uint2*>(codes + 4) = make_uint2(a1, a2);
      codes[9] = b0;
      *reinterpret_cast<uint2*>(codes + 10) = make_uint2(b1, b2);
    }
  } else {
    // groups 4h..4h+3 -> words 2h, 2h+1; groups 8+4h.. -> words 4+2h, 5+2h
    *reinterpret_cast<uint2*>(codes + 2 * half) =
        make_uint2(gx[0] | (gx[1] << 16), gx[2] | (gx[3] << 16));
    *reinterpret_cast<uint2*>(codes + 4 + 2 * half) =
        make_uint2(gy[0] | (gy[1] << 16), gy[2] | (gy[3] << 16));
  }
  if (half == 0) {
    if (EXACT)
      *static_cast<uint16_t*>(meta) = __half_as_ushort(sh);
    else
      *static_cast<uint32_t*>(meta) = cm | (static_cast<uint32_t>(__half_as_ushort(sh)) << 16);
  }
}

template <int BITS, bool ROPE, bool EXACT>
__global__ void __launch_bounds__(256, 2) encode_kernel(const CodecArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int nthreads = blockDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot_l = lane & 15, half = lane >> 4;
  const int rows_bytes = (nthreads / 2) * kRowPad;
  const int stage_bytes = rows_bytes + (ROPE ? kCsBytes : 0);
  const uint32_t raw = smem_u32(smem + 2 * stage_bytes);  // RoPE rows of the next tile
  const int row_idx = warp * kSlots + slot_l;             // this vector's staged row

  const int64_t first = blockIdx.x, step = gridDim.x;
  const int64_t my_tiles = first < a.num_tiles ? (a.num_tiles - 1 - first) / step + 1 : 0;
  auto tile = [&](int64_t k) { return enc_tile(a, first + k * step); };

  // The warp's 16 rows (one head, 16 pairs) with 16-byte async copies: in copy
  // j, lane l moves chunk l%16 of row 2j + l/16, two whole rows per
  // instruction.  Each lane supplies its pair's row offset in elements
  // (unit * su + token * st, -1 past the last pair) through a shuffle.
  auto issue_rows = [&](const EncTile& tl, const EncPair& ep, int32_t src, int s) {
    const int h = tl.group * a.hg + warp;
    const int64_t tok = src < a.T_in ? src : a.T_in - 1;
    const long long roff = src >= 0 ? static_cast<long long>(ep.unit * a.su + tok * a.st) : -1ll;
    const uint16_t* base = a.kv + h * a.sh + slot_l * 8;
    const uint32_t dst0 = smem_u32(smem + s * stage_bytes + warp * kSlots * kRowPad) + slot_l * 16;
#pragma unroll
    for (int j = 0; j < kSlots / 2; ++j) {
      const int r = 2 * j + half;
      const long long ro = __shfl_sync(0xffffffffu, roff, r);
      if (ro >= 0) cp_async16(dst0 + r * kRowPad, base + ro);
    }
  };
  // cross-warp data (the shared RoPE table) needs the CTA barrier; value
  // tiles only touch the warp's own rows
  auto sync = [&]() {
    if (ROPE) __syncthreads();
    else __syncwarp();
  };

  // prologue: tile 0 (rows + its RoPE table), then tile 1 in flight
  EncPair pp_pref{};
  int32_t src_pref = -1;
  if (my_tiles > 0) {
    const EncTile t0 = tile(0);
    const EncPair p0 = enc_pair(a, t0.p0, slot_l);
    const int32_t s0 = enc_src(a, p0);
    if (ROPE) issue_rope_rows(a.tab, a.n_a, a.pos_base, s0, raw, warp, nthreads / 32, lane);
    issue_rows(t0, p0, s0, 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  sync();
  if (ROPE && my_tiles > 0) combine_rope_rows(raw, reinterpret_cast<float4*>(smem + rows_bytes), tid, nthreads);
  sync();
  if (my_tiles > 1) {
    const EncTile t1 = tile(1);
    const EncPair p1 = enc_pair(a, t1.p0, slot_l);
    const int32_t s1 = enc_src(a, p1);
    if (ROPE) issue_rope_rows(a.tab, a.n_a, a.pos_base, s1, raw, warp, nthreads / 32, lane);
    cp_async_commit();
    issue_rows(t1, p1, s1, 1);
    cp_async_commit();
  } else {
    cp_async_commit();
    cp_async_commit();
  }
  if (my_tiles > 2) {
    pp_pref = enc_pair(a, tile(2).p0, slot_l);
    src_pref = enc_src(a, pp_pref);
  }

  // Per iteration two groups are committed, [RoPE rows of k+2] then [rows of
  // k+2]; waiting for all but the newest leaves only rows(k+1) in flight.
  for (int64_t k = 0; k < my_tiles; ++k) {
    const int s = static_cast<int>(k & 1);
    cp_async_wait<1>();
    sync();

    const EncTile tl = tile(k);
    const int h = tl.group * a.hg + warp;
    const EncPair ep = enc_pair(a, tl.p0, slot_l);
    unsigned char* st = smem + s * stage_bytes;
    // lanes past the last pair run on whatever their staging row holds; none
    // of their results is stored
    float2 v[32];
    load_half<ROPE>(v, smem_u32(st + row_idx * kRowPad),
                    smem_u32(st + rows_bytes) + (16 * half * kSlots + slot_l) * 16, half);
    if (ROPE && k + 1 < my_tiles)  // RoPE table of tile k+1 into the other stage
      combine_rope_rows(raw, reinterpret_cast<float4*>(smem + (s ^ 1) * stage_bytes + rows_bytes), tid,
                  nthreads);
    sync();  // stage s and the raw rows are free
    if (k + 2 < my_tiles) {
      if (ROPE) issue_rope_rows(a.tab, a.n_a, a.pos_base, src_pref, raw, warp, nthreads / 32, lane);
      cp_async_commit();
      issue_rows(tile(k + 2), pp_pref, src_pref, s);
      cp_async_commit();
      if (k + 3 < my_tiles) {  // used next iteration
        pp_pref = enc_pair(a, tile(k + 3).p0, slot_l);
        src_pref = enc_src(a, pp_pref);
      }
    } else {
      cp_async_commit();
      cp_async_commit();
    }
    const int64_t vec = ep.unit * a.pu + h * a.ph + a.slot0 + ep.slot;
    void* meta = EXACT ? static_cast<void*>(reinterpret_cast<uint16_t*>(a.meta) + vec)
                       : static_cast<void*>(a.meta + vec);
    quantise_half<BITS, EXACT>(v, half, ep.valid, a.codes + vec * (4 * BITS), meta);
  }
  cp_async_wait<0>();
}

// --------------------------------------------------------------- decode
template <int BITS, bool ROPE>
__device__ __forceinline__ void decode_half(const uint32_t (&w)[4 * BITS], uint32_t meta,
                                            uint32_t csa, uint32_t row, int rsw, int half) {
  float2 v[32];
  reconstruct_half<BITS>(w, meta, half, v);
  if (ROPE) rope_half(v, csa);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t A[4], B[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const __nv_bfloat162 pa = __floats2bfloat162_rn(v[8 * q + 2 * t].x, v[8 * q + 2 * t + 1].x);
      const __nv_bfloat162 pb = __floats2bfloat162_rn(v[8 * q + 2 * t].y, v[8 * q + 2 * t + 1].y);
      A[t] = *reinterpret_cast<const uint32_t*>(&pa);
      B[t] = *reinterpret_cast<const uint32_t*>(&pb);
    }
    // chunk 4h+q of columns 0-63 and of columns 64-127, swizzled by row % 8
    const uint32_t cc = static_cast<uint32_t>(((4 * half + q) ^ rsw) << 4);
    sts128(row + cc, make_uint4(A[0], A[1], A[2], A[3]));
    sts128(row + kSlots * 128 + cc, make_uint4(B[0], B[1], B[2], B[3]));
  }
}

// Exact layout -> regular layout in registers: each group's coset bit sits in
// place of the low bit of its code 7, whose true value is the parity of codes
// 0..6 (the codes of a point of E8 have an even sum).  Restores that bit in
// the words and returns the regular meta word (coset mask | sigma << 16).
template <int BITS>
__device__ __forceinline__ uint32_t unfold_exact(uint32_t (&w)[4 * BITS], uint32_t sig16) {
  constexpr int kGB = 8 * BITS;                                 // bits per group
  constexpr uint32_t kLsb8 = BITS == 3 ? 0x249249u : 0x5555u;  // low bits of codes 0..7
  uint32_t mask = 0u;
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    // the parity of the low bits of codes 0..7 (the stored coset bit included)
    // is the coset bit xor the true low bit of code 7, so xor-ing it into the
    // stored bit restores that bit; groups cross a word boundary only for 3
    // bits, and never past the last word
    const int p = kGB * g, wi = p >> 5, off = p & 31;
    uint32_t x = w[wi] & (kLsb8 << off);
    if (off + kGB > 32) x ^= w[wi + 1] & (kLsb8 >> (32 - off));
    const int q = p + 7 * BITS, qw = q >> 5, qb = q & 31;
    mask |= ((w[qw] >> qb) & 1u) << g;
    w[qw] ^= (static_cast<uint32_t>(__popc(x)) & 1u) << qb;
  }
  return mask | (sig16 << 16);
}

// Codes and meta of the vector (unit, head h, slot stile * 16 + slot_l), if
// that slot is below n (registers, loaded one tile ahead).  RAW (exact layout
// only): meta is the raw fp16 scale and the words stay folded, for the caller
// to unfold when it uses them (so that the loads are not waited for here).
template <int BITS, bool EXACT, bool RAW = false>
__device__ __forceinline__ void load_codes_at(const CodecArgs& a, int unit, int h, int64_t stile,
                                              int slot_l, uint32_t (&w)[4 * BITS],
                                              uint32_t& meta) {
  const int64_t slot = stile * kSlots + slot_l;
  if (slot < a.n) {
    const int64_t vec = unit * a.pu + h * a.ph + a.slot0 + slot;
    const uint4* src = reinterpret_cast<const uint4*>(a.codes + vec * (4 * BITS));
#pragma unroll
    for (int c = 0; c < BITS; ++c) {
      const uint4 q = __ldg(src + c);
      w[4 * c] = q.x;
      w[4 * c + 1] = q.y;
      w[4 * c + 2] = q.z;
      w[4 * c + 3] = q.w;
    }
    if (EXACT && RAW)
      meta = __ldg(reinterpret_cast<const unsigned short*>(a.meta) + vec);
    else if (EXACT)
      meta = unfold_exact<BITS>(w, __ldg(reinterpret_cast<const unsigned short*>(a.meta) + vec));
    else
      meta = __ldg(a.meta + vec);
  }
}

// Codes and meta of this thread's vector in tile t (warp: its head in the group).
template <int BITS, bool EXACT>
__device__ __forceinline__ void load_codes(const CodecArgs& a, int64_t t, int warp, int slot_l,
                                           uint32_t (&w)[4 * BITS], uint32_t& meta) {
  const Tile tl = tile_of(a, t);
  load_codes_at<BITS, EXACT>(a, tl.unit, tl.group * a.hg + warp, tl.stile, slot_l, w, meta);
}

// Output tile of one warp: 16 rows x 256 bytes as two 16 x 128-byte boxes
// (columns 0-63 and 64-127) in the 128-byte swizzled layout of the tensor
// store: 16-byte chunk c of row r sits at chunk (c ^ (r % 8)) of its box row.
constexpr int kOutTileBytes = 2 * kSlots * 128;

template <int BITS, bool ROPE, bool EXACT>
__global__ void __launch_bounds__(256, 2)
    decode_kernel(const CodecArgs a, const __grid_constant__ CUtensorMap out_map) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzled tiles need a 1024-byte aligned base (1 KB of slack is allocated)
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int nthreads = blockDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot_l = lane & 15, half = lane >> 4;
  const int nwarps = nthreads / 32;
  const uint32_t tile_base = smem_u32(smem) + warp * kOutTileBytes;
  unsigned char* cs_base = smem + nwarps * kOutTileBytes;  // two cs buffers, kCsBytes each

  const int64_t first = blockIdx.x, step = gridDim.x;
  const int64_t my_tiles = first < a.num_tiles ? (a.num_tiles - 1 - first) / step + 1 : 0;

  uint32_t w[4 * BITS];
  uint32_t meta = 0;
#pragma unroll
  for (int i = 0; i < 4 * BITS; ++i) w[i] = 0;
  // RoPE rows of tiles k+1 and k+2 in two raw buffers: one CTA barrier per tile
  const uint32_t raw0 = smem_u32(cs_base + 2 * kCsBytes);
  auto raw_of = [&](int64_t k) { return raw0 + static_cast<uint32_t>(k & 1) * kRawBytes; };
  auto tile = [&](int64_t k) { return tile_of(a, first + k * step); };
  auto cs_of = [&](int64_t k) { return reinterpret_cast<float4*>(cs_base + (k & 1) * kCsBytes); };

  // prologue: rows of tiles 0 and 1 in flight, table of tile 0 combined
  int32_t src_pref = -1;
  if (ROPE) {
    if (my_tiles > 0) issue_rope_rows(a.tab, a.n_a, a.pos_base, slot_src(a, tile(0), slot_l), raw_of(0), warp, nwarps, lane);
    cp_async_commit();
    if (my_tiles > 1) issue_rope_rows(a.tab, a.n_a, a.pos_base, slot_src(a, tile(1), slot_l), raw_of(1), warp, nwarps, lane);
    cp_async_commit();
    if (my_tiles > 2) src_pref = slot_src(a, tile(2), slot_l);
    cp_async_wait<1>();
    __syncthreads();
    if (my_tiles > 0) combine_rope_rows(raw_of(0), cs_of(0), tid, nthreads);
  }
  if (my_tiles > 0) load_codes<BITS, EXACT>(a, first, warp, slot_l, w, meta);

  for (int64_t k = 0; k < my_tiles; ++k) {
    if (ROPE) {
      // rows of tile k+1 landed (everyone's), table k combined, tile k-1 decoded
      cp_async_wait<0>();
      __syncthreads();
      if (k + 2 < my_tiles) issue_rope_rows(a.tab, a.n_a, a.pos_base, src_pref, raw_of(k), warp, nwarps, lane);
      cp_async_commit();
      if (k + 3 < my_tiles) src_pref = slot_src(a, tile(k + 3), slot_l);
      if (k + 1 < my_tiles) combine_rope_rows(raw_of(k + 1), cs_of(k + 1), tid, nthreads);
    }
    const Tile tl = tile(k);
    const int h = tl.group * a.hg + warp;
    uint32_t wc[4 * BITS];
#pragma unroll
    for (int i = 0; i < 4 * BITS; ++i) wc[i] = w[i];
    const uint32_t mc = meta;
    if (k + 1 < my_tiles) load_codes<BITS, EXACT>(a, first + (k + 1) * step, warp, slot_l, w, meta);
    // the warp's previous tensor store has finished reading the tile
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
    const uint32_t csa = smem_u32(cs_of(k)) + (16 * half * kSlots + slot_l) * 16;
    decode_half<BITS, ROPE>(wc, mc, csa, tile_base + slot_l * 128, slot_l & 7, half);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      // rows past n are clipped by the tensor map (its token extent is n)
      const int y = static_cast<int>(tl.stile * kSlots);
      tma_store_4d(&out_map, tile_base, 0, y, h, tl.unit);
      tma_store_4d(&out_map, tile_base + kSlots * 128, 64, y, h, tl.unit);
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait_all();
}

// ------------------------------------------------ decode on the tensor cores
// The transform inside decode is an exact integer matrix product: per vector
// w = H t with H the 128 x 128 Sylvester matrix, t_k = 2 j_k - 2^b + 2 - h_g(k)
// and |w| <= 896.  decode_tc_kernel runs it on the tensor cores
// (tcgen05.mma kind::f16, fp32 accumulators in TMEM) for tiles of 128 vectors
// (8 / hg slot tiles of 16 slots for a group of hg heads; with hg = 3, 5, 6 or
// 7 some of the 8 row blocks idle): D = A B^T with
//  * A (128 x 160, f16): per vector, its 128 codes as 1024 + j 2^d in the slot
//    order of tc_unpack, 16 slots 2 h_g (the group coset bits) and 16 slots 1;
//  * B (128 x 160, f16, the same for every tile): row n is output coordinate
//    c(n) = tc_coord(n) (columns 4k .. 4k+3: 2k, 2k+1, 2k+64, 2k+65, two RoPE
//    pairs as two register pairs); code slot p holds 2^(1-d_p) H[c(n)][code_p], coset
//    slot g holds -(1/2) sum over group g of H[c(n)][k] (0 or +-4), and the
//    16 constant slots split beta_n = (2 - 2^b) 128 [c(n) = 0]
//    - sum_p 2^(11-d_p) H[c(n)][code_p] (which cancels the 1024 offsets) into
//    parts of at most 2^14, each exact in f16.
// Every product and partial sum is an integer of magnitude below 2^18, so
// D = w exactly whatever the summation order.  The epilogue (one thread per
// vector) then forms x = fp32(w kappa), applies the RoPE rotation and the bf16
// rounding with the same operations as decode_half, and writes the 128-byte
// swizzled boxes of the same TMA stores.
//
// One CTA per SM holds NWG = 4 warpgroups of 128 threads.  Each owns 128 TMEM
// columns, an A tile whose rows double as the output staging of the same
// rows (so a warp waits only for its own earlier stores before it writes its
// rows of the next tile), its coset slots and a RoPE table, and walks its own
// tiles: write A -> one thread issues the ten MMAs and commits them to the
// warpgroup's mbarrier -> combine the tile's RoPE table and prefetch the next
// tile's codes and table rows -> wait for the mbarrier (bounded: past
// kTcWaitLimit polls the device error word gets kErrMmaTimeout and the
// warpgroup stops) -> epilogue -> TMA stores.  The output bytes a SM can
// have in flight are its staging tiles, so the layout gives them as much of
// the 227 KB as it can: four warpgroups of 32 KB.
constexpr int kTcA = 32768;    // A: 128 rows x 128 f16 in two 128-byte swizzled K blocks; then
                               // the output staging: per block of 16 rows two 2 KB boxes
constexpr int kTcAx = 4096;    // coset slots: 128 rows x 16 f16 as two 2 KB chunk columns
constexpr int kTcB = 32768;    // B: 128 rows x 128 f16, the layout of A
constexpr int kTcBx = 8192;    // B extra: coset and constant slots, four 2 KB chunk columns
constexpr int kTcOnes = 4096;  // A constant slots (1.0), shared by the warpgroups
constexpr int kTcTab = 1024;   // setup: slot table (code, shift) and per-row constants
constexpr int kTcShared = kTcB + kTcBx + kTcOnes + kTcTab;
// RoPE table of one slot tile: entry (j, slot) = (c_2j, c_2j+1, s_2j, s_2j+1) of
// the slot's position at j * kTcCsPitch + slot * 16.  The pitch is 17 chunks of
// 16 bytes, so both access patterns are free of bank conflicts: a quarter warp
// writing eight consecutive j of one slot, and one reading entry j of eight
// consecutive slots.
constexpr int kTcCsPitch = 17 * 16;
constexpr int kTcCsBytes = 32 * kTcCsPitch;
constexpr uint32_t kTcIdesc = idesc_f16_f32(128, 128);
constexpr uint32_t kTcWaitLimit = 1u << 20;
constexpr uint32_t kErrMmaTimeout = 2u;

// A warpgroup's A tile, coset slots and tables, rounded up to 1024 bytes so
// that every warpgroup's A tile keeps the swizzle atom's 1024-byte alignment.
template <int TABLES>
__host__ __device__ constexpr int tc_wg_bytes() {
  return (kTcA + kTcAx + TABLES * kTcCsBytes + 1023) / 1024 * 1024;
}
template <int NWG, int TABLES>
__host__ __device__ constexpr int tc_smem_bytes() {
  return 1024 + kTcShared + NWG * tc_wg_bytes<TABLES>() + 64;
}

// AND of pred over the `count` threads of named barrier `id`.
__device__ __forceinline__ bool bar_and(uint32_t id, uint32_t count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0u;
}

// Output coordinate of row n of B (TMEM column n): columns 4k .. 4k+3 hold
// coordinates 2k, 2k+1, 2k+64, 2k+65, so a thread's register pairs are
// (x_2k, x_2k+1) and their RoPE partners (x_2k+64, x_2k+65).
__host__ __device__ constexpr int tc_coord(int n) {
  return 2 * (n >> 2) + (n & 1) + 64 * ((n >> 1) & 1);
}

// The constant operands (see above), built once per CTA: B main in the
// 128-byte swizzled K-major layout; B extra as four 2 KB chunk columns
// (chunk c of row n at c * 2048 + n * 16: coset slots 0..15, constant slots
// 16..31); the A constant slots (1.0) as two chunk columns.  tab: generic
// pointer to kTcTab bytes of scratch (slot codes, shifts, per-row beta).
template <int BITS>
__device__ void tc_build_constants(uint32_t b_main, uint32_t b_x, uint32_t ones,
                                   unsigned char* tab, int tid, int nthreads) {
  unsigned char* s_code = tab;
  unsigned char* s_shift = tab + 128;
  int* s_beta = reinterpret_cast<int*>(tab + 256);
  for (int i = tid; i < 128; i += nthreads) {
    int code, d;
    tc_slot<BITS>(i, code, d);
    s_code[i] = static_cast<unsigned char>(code);
    s_shift[i] = static_cast<unsigned char>(d);
    const int cn = tc_coord(i);  // row i's coordinate
    s_beta[i] = cn == 0 ? (2 - (1 << BITS)) * 128 : 0;
  }
  for (int i = tid; i < kTcOnes / 16; i += nthreads)
    sts128(ones + i * 16, make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u));
  __syncthreads();
  for (int e = tid; e < 128 * 16; e += nthreads) {
    const int n = e >> 4, c = e & 15;
    const int cn = tc_coord(n);
    uint32_t v[4];
    int part = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t pair = 0u;
#pragma unroll
      for (int l = 0; l < 2; ++l) {
        const int p = 8 * c + 2 * u + l;
        const int code = s_code[p], d = s_shift[p];
        const uint32_t neg = static_cast<uint32_t>(__popc(cn & code) & 1);
        pair |= ((neg << 15) | (static_cast<uint32_t>(16 - d) << 10)) << (16 * l);  // +-2^(1-d)
        part += neg ? (1 << (11 - d)) : -(1 << (11 - d));  // -2^(11-d) H
      }
      v[u] = pair;
    }
    sts128(b_main + (c >> 3) * 16384 + (n >> 3) * 1024 + (n & 7) * 128 + (((c & 7) ^ (n & 7)) << 4),
           make_uint4(v[0], v[1], v[2], v[3]));
    atomicAdd(s_beta + n, part);
  }
  __syncthreads();
  for (int n = tid; n < 128; n += nthreads) {
    const int cn = tc_coord(n);
    uint32_t cw[8], bw[8];
    int beta = s_beta[n];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      uint32_t pc = 0u, pb = 0u;
#pragma unroll
      for (int l = 0; l < 2; ++l) {
        const int g = 2 * u + l;  // -4 (-1)^popc(c & 8g) where c % 8 == 0, else 0
        pc |= ((cn & 7) ? 0u : ((__popc(cn & (8 * g)) & 1) ? 0x4400u : 0xC400u)) << (16 * l);
        const int part = beta > 16384 ? 16384 : (beta < -16384 ? -16384 : beta);
        beta -= part;
        pb |= static_cast<uint32_t>(__half_as_ushort(__int2half_rn(part))) << (16 * l);
      }
      cw[u] = pc;
      bw[u] = pb;
    }
    sts128(b_x + n * 16, make_uint4(cw[0], cw[1], cw[2], cw[3]));
    sts128(b_x + 2048 + n * 16, make_uint4(cw[4], cw[5], cw[6], cw[7]));
    sts128(b_x + 4096 + n * 16, make_uint4(bw[0], bw[1], bw[2], bw[3]));
    sts128(b_x + 6144 + n * 16, make_uint4(bw[4], bw[5], bw[6], bw[7]));
  }
}

// Row r of A: the 128 codes (16 chunks of 8 slots) and the 16 coset slots
// (2.0 for a set bit g of meta, else 0).
template <int BITS>
__device__ __forceinline__ void tc_write_a(const uint32_t (&w)[4 * BITS], uint32_t meta,
                                           uint32_t a_main, uint32_t a_x, int r) {
  uint32_t h[64];
  tc_unpack<BITS>(w, h);
  const uint32_t rowb = a_main + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
  for (int c = 0; c < 16; ++c)
    sts128(rowb + (c >> 3) * 16384 + (((c & 7) ^ (r & 7)) << 4),
           make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]));
  // y = mask | mask << 15: bit 2u of mask at bit 2u, bit 2u+1 at bit 16 + 2u
  const uint32_t mask = meta & 0xFFFFu, y = mask | (mask << 15);
  uint32_t cw[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) cw[u] = (y << (14 - 2 * u)) & 0x40004000u;
  sts128(a_x + r * 16, make_uint4(cw[0], cw[1], cw[2], cw[3]));
  sts128(a_x + 2048 + r * 16, make_uint4(cw[4], cw[5], cw[6], cw[7]));
}

// Columns 32q .. 32q+31 of this thread's row of D (d: their bits) -> bf16
// coordinates 16q .. 16q+15 and 64+16q .. 79+16q in the swizzled boxes at
// rowb (box 1 at +16384).  Columns 32q + 4g .. +3 are X = (x_2k, x_2k+1) and
// Y = (x_2k+64, x_2k+65), k = 8q + g; the table entry of k is (c_2k, c_2k+1,
// s_2k, s_2k+1), so one packed multiply and one packed fma per half rotate two
// pairs with each lane's own roundings fmaf(x, c, -(y s)), fmaf(y, c, x s).
template <bool ROPE>
__device__ __forceinline__ void tc_chunk(const uint32_t (&d)[32], int q, float2 k2, uint32_t csa,
                                         uint32_t rowb, int rsw) {
  float2 X[8], Y[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    X[g] = mul2(make_float2(__uint_as_float(d[4 * g]), __uint_as_float(d[4 * g + 1])), k2);
    Y[g] = mul2(make_float2(__uint_as_float(d[4 * g + 2]), __uint_as_float(d[4 * g + 3])), k2);
  }
  if (ROPE) {
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const float4 t = lds128f(csa + (8 * q + g) * kTcCsPitch);
      const float2 C = make_float2(t.x, t.y), S = make_float2(t.z, t.w);
      const float2 T = mul2(Y[g], S), U = mul2(X[g], S);
      X[g] = fma2(X[g], C, make_float2(-T.x, -T.y));
      Y[g] = fma2(Y[g], C, U);
    }
  }
#pragma unroll
  for (int h8 = 0; h8 < 2; ++h8) {
    uint32_t A[4], B[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const __nv_bfloat162 pa = __floats2bfloat162_rn(X[4 * h8 + t].x, X[4 * h8 + t].y);
      const __nv_bfloat162 pb = __floats2bfloat162_rn(Y[4 * h8 + t].x, Y[4 * h8 + t].y);
      A[t] = *reinterpret_cast<const uint32_t*>(&pa);
      B[t] = *reinterpret_cast<const uint32_t*>(&pb);
    }
    const uint32_t cc = static_cast<uint32_t>(((2 * q + h8) ^ rsw) << 4);
    sts128(rowb + cc, make_uint4(A[0], A[1], A[2], A[3]));
    sts128(rowb + 16384 + cc, make_uint4(B[0], B[1], B[2], B[3]));
  }
}

// This thread's row of D (taddr: its TMEM lane, the warpgroup's columns) ->
// bf16 in the output staging at out.
template <bool ROPE>
__device__ __forceinline__ void tc_epilogue(uint32_t taddr, uint32_t meta, uint32_t out,
                                            uint32_t csa, int r) {
  const float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(meta >> 16)));
  const float kappa = __fmul_rn(__fmul_rn(sig, 0.5f), __uint_as_float(kCBits));
  const float2 k2 = make_float2(kappa, kappa);
  const uint32_t rowb = out + (r >> 3) * 1024 + (r & 7) * 128;
  const int rsw = r & 7;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t d[32];
    tmem_ld32(taddr + 32 * q, d);
    tmem_ld_wait(d);
    tc_chunk<ROPE>(d, q, k2, csa, rowb, rsw);
  }
}

// TABLES: RoPE tables per warpgroup (one per slot tile of a tile; 0 for
// values).  HG: the head-group size when it is 8 (one slot tile per tile) or
// 4 (two), which folds the tiling to constants; 0: taken from the arguments.
template <int BITS, bool ROPE, bool EXACT, int NWG, int TABLES, int HG>
__global__ void __launch_bounds__(128 * NWG, 1)
    decode_tc_kernel(const CodecArgs a, const __grid_constant__ CUtensorMap out_map) {
  static_assert(ROPE == (TABLES > 0), "keys carry one table per slot tile, values none");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const int tid = threadIdx.x, wg = tid >> 7, t = tid & 127, wl = (tid >> 5) & 3, lane = tid & 31;
  constexpr uint32_t kWg = static_cast<uint32_t>(tc_wg_bytes<TABLES>());
  constexpr uint32_t kCols = NWG <= 2 ? 256u : 512u;
  static_assert(128 * NWG <= 512, "one accumulator of 128 columns per warpgroup");
  static_assert(kTcShared % 1024 == 0 && kWg % 1024 == 0, "A tiles on 1024-byte boundaries");
  const uint32_t b_main = base, b_x = base + kTcB, ones = b_x + kTcBx, tab = ones + kTcOnes;
  const uint32_t a_main = base + kTcShared + wg * kWg, a_x = a_main + kTcA, cs = a_x + kTcAx;
  const uint32_t bars = base + kTcShared + NWG * kWg;
  const uint32_t mbar = bars + 8 * wg, tslot = bars + 8 * NWG;

  if (tid < 32) {
    tmem_alloc(tslot, kCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int g = 0; g < NWG; ++g) mbar_init(bars + 8 * g, 1);
    fence_mbar_init();
  }
  tc_build_constants<BITS>(b_main, b_x, ones, smem_raw + (tab - raw), tid, blockDim.x);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = lds32(tslot) + static_cast<uint32_t>(128 * wg);
  const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * wl) << 16);

  const int64_t first = static_cast<int64_t>(blockIdx.x) * NWG + wg;
  const int64_t step = static_cast<int64_t>(gridDim.x) * NWG;
  const int64_t my_tiles = first < a.num_tiles ? (a.num_tiles - 1 - first) / step + 1 : 0;
  // Row t of a tile: row block rb = t / 16 is slot tile mi of the tile (rb / hg)
  // for head rb % hg of the head group, slot t % 16; blocks past m * hg idle.
  // Keys in head groups of 8 or 4 pair their rows instead: warp w serves slot
  // tile mi = w / (hg / 2) and heads hp, hp + 1 of it (hp = 2 (w % (hg / 2))),
  // lanes 2i and 2i+1 slot i of the two heads, so the two lanes that read one
  // RoPE table entry sit in the same quarter warp (one shared-memory access
  // serves both), and a warp's 32 rows are one box of 2 heads x 16 tokens.
  constexpr bool PAIRS = ROPE && (HG == 8 || HG == 4);
  const int hg = HG ? HG : a.hg, m = HG ? 8 / HG : a.tc_m;
  const int rb = t >> 4, slot = PAIRS ? (lane >> 1) : (t & 15);
  const bool rb_used = PAIRS || rb < m * hg;
  const int mi = PAIRS ? wl / (hg / 2) : (rb_used ? rb / hg : 0);
  const int hp = PAIRS ? 2 * (wl % (hg / 2)) : 0;
  const int hrel = PAIRS ? hp + (lane & 1) : (rb_used ? rb % hg : 0);
  // A tile index -> (head group, unit, first slot tile).
  auto tile_at = [&](int64_t t64, int& group, int& unit, int64_t& stile0) {
    const uint32_t tt = static_cast<uint32_t>(t64);
    const uint32_t q = fdiv(tt, a.div_groups);
    const uint32_t u = fdiv(q, a.div_sgroups);
    group = static_cast<int>(tt - q * a.div_groups.d);
    unit = static_cast<int>(u);
    stile0 = static_cast<int64_t>(q - u * a.div_sgroups.d) * m;
  };
  auto load_row = [&](int64_t t64, uint32_t (&wr)[4 * BITS], uint32_t& mr) {
    int group, unit;
    int64_t stile0;
    tile_at(t64, group, unit, stile0);
    const int64_t st = stile0 + mi;
    if (HG == 8 || (rb_used && st < a.slot_tiles))
      load_codes_at<BITS, EXACT, !ROPE>(a, unit, group * hg + hrel, st, slot, wr, mr);
  };
  uint32_t w[4 * BITS];
  uint32_t meta = 0u;
#pragma unroll
  for (int i = 0; i < 4 * BITS; ++i) w[i] = 0u;
  // RoPE table rows of this thread's four table entries (fslot, j = fj + 8u)
  // of each table of the next tile, fetched a tile ahead: eight lanes read one
  // 128-byte run of a slot's two table rows.
  const int fslot = t >> 3, fj = t & 7;
  constexpr int kT = TABLES > 0 ? TABLES : 1;
  float4 ra[kT][4], rbw[kT][4];
  bool rvalid[kT];
#pragma unroll
  for (int x = 0; x < kT; ++x) rvalid[x] = false;
  auto fetch_rope = [&](int64_t t64) {
    int group, unit;
    int64_t stile0;
    tile_at(t64, group, unit, stile0);
#pragma unroll
    for (int x = 0; x < kT; ++x) {
      const int32_t src = HG == 8 || stile0 + x < a.slot_tiles
                              ? slot_src_at(a, unit, stile0 + x, fslot) : -1;
      rvalid[x] = src >= 0;
      if (rvalid[x]) {
        const int64_t pos = a.pos_base + src;
        int64_t hi = pos >> 8;
        hi = hi < 0 ? 0 : (hi >= a.n_a ? a.n_a - 1 : hi);  // out-of-contract positions stay in bounds
        const float4* ta = reinterpret_cast<const float4*>(a.tab + hi * kHalf);
        const float4* tb = reinterpret_cast<const float4*>(a.tab + (a.n_a + (pos & 255)) * kHalf);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          ra[x][u] = __ldg(ta + fj + 8 * u);
          rbw[x][u] = __ldg(tb + fj + 8 * u);
        }
      }
    }
  };
  if (my_tiles > 0) {
    load_row(first, w, meta);
    if (ROPE) fetch_rope(first);
  }

  for (int64_t k = 0; k < my_tiles; ++k) {
    // this warp's rows of A are its output staging: its last stores must have read them
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
    // exact-layout values were loaded raw a tile ago (keys unfold at the load:
    // deferred, their kernel spills)
    if (EXACT && !ROPE) meta = unfold_exact<BITS>(w, meta & 0xFFFFu);
    tc_write_a<BITS>(w, meta, a_main, a_x, t);
    const uint32_t mk = meta;
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar_sync(1 + wg, 128);  // also: every epilogue of tile k-1 has read the RoPE tables
    if (t == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
        umma_f16(tmem, desc_sw128(a_main + off), desc_sw128(b_main + off), kTcIdesc, s > 0);
      }
      umma_f16(tmem, desc_plain(a_x, 2048, 128), desc_plain(b_x, 2048, 128), kTcIdesc, 1u);
      umma_f16(tmem, desc_plain(ones, 2048, 128), desc_plain(b_x + 4096, 2048, 128), kTcIdesc, 1u);
      umma_commit(mbar);
    }
    if (ROPE) {
#pragma unroll
      for (int x = 0; x < kT; ++x) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (rvalid[x]) {  // (c_2j, c_2j+1, s_2j, s_2j+1)
            const float4 A = ra[x][u], B = rbw[x][u];
            v.x = __fmaf_rn(A.x, B.x, -__fmul_rn(A.y, B.y));
            v.z = __fmaf_rn(A.y, B.x, __fmul_rn(A.x, B.y));
            v.y = __fmaf_rn(A.z, B.z, -__fmul_rn(A.w, B.w));
            v.w = __fmaf_rn(A.w, B.z, __fmul_rn(A.z, B.w));
          }
          sts128(cs + x * kTcCsBytes + (fj + 8 * u) * kTcCsPitch + fslot * 16,
                 make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
                            __float_as_uint(v.w)));
        }
      }
    }
    if (k + 1 < my_tiles) load_row(first + (k + 1) * step, w, meta);
    // the MMAs are done (A has been read: its rows become the staging) and, by
    // the same barrier, every thread's part of the RoPE tables is written
    bool done = false;
    for (uint32_t spin = 0; spin < kTcWaitLimit && !done; ++spin)
      done = mbar_try_wait(mbar, static_cast<uint32_t>(k & 1));
    if (!bar_and(1 + wg, 128, done)) {
      if (t == 0) atomicOr(&g_nq_error, kErrMmaTimeout);
      break;
    }
    tc_fence_after();
    tc_epilogue<ROPE>(t_row, mk, a_main, cs + (ROPE ? mi : 0) * kTcCsBytes + slot * 16, t);
    tc_fence_before();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      // rows past n are clipped by the tensor map (its token extent is n)
      int group, unit;
      int64_t stile0;
      tile_at(first + k * step, group, unit, stile0);
      if (PAIRS && (HG == 8 || stile0 + mi < a.slot_tiles)) {
        // rows 32 wl .. 32 wl + 31: heads hp, hp + 1 of the 16 tokens of slot tile mi
        const int y = static_cast<int>((stile0 + mi) * kSlots), h = group * hg + hp;
        const uint32_t src = a_main + wl * 4096;
        tma_store_4d(&out_map, src, 0, h, y, unit);
        tma_store_4d(&out_map, src + 16384, 64, h, y, unit);
      }
#pragma unroll
      for (int b2 = 0; b2 < (PAIRS ? 0 : 2); ++b2) {
        const int rbi = 2 * wl + b2;
        if (rbi >= m * hg) continue;
        const int64_t st = stile0 + rbi / hg;
        if (HG != 8 && st >= a.slot_tiles) continue;
        const int y = static_cast<int>(st * kSlots);
        const int h = group * hg + rbi % hg;
        const uint32_t src = a_main + rbi * 2048;
        tma_store_4d(&out_map, src, 0, y, h, unit);
        tma_store_4d(&out_map, src + 16384, 64, y, h, unit);
      }
      bulk_commit();
    }
    if (ROPE && k + 1 < my_tiles) fetch_rope(first + (k + 1) * step);
  }
  if (lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (tid < 32) {
    tc_fence_after();
    tmem_dealloc(lds32(tslot), kCols);
  }
}

// ---------------------------------------------------------------- launch
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D map of a bf16 [units][heads][n][128] output: boxes of 64 coordinates x
// 16 tokens, 128-byte swizzle.  Strides in bytes; a unit dimension of extent
// 1 may carry any stride, so it is given a valid one.  head_pairs: the head
// dimension is listed before the token one, with boxes of 64 coordinates x 2
// heads x 16 tokens (shared-memory rows token-major: row 2 * token + head).
static cudaError_t make_out_map(CUtensorMap* m, const CodecArgs& a, int units,
                                bool head_pairs = false) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return cudaErrorNotSupported;
  const uint64_t st = static_cast<uint64_t>(a.st) * 2;
  uint64_t sh = static_cast<uint64_t>(a.sh) * 2, su = static_cast<uint64_t>(a.su) * 2;
  if (a.heads == 1 || sh == 0) sh = st * static_cast<uint64_t>(a.n);
  if (units == 1 || su == 0) su = sh * static_cast<uint64_t>(a.heads);
  cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(a.n), static_cast<cuuint64_t>(a.heads),
                        static_cast<cuuint64_t>(units)};
  cuuint64_t strides[3] = {st, sh, su};
  cuuint32_t box[4] = {64, kSlots, 1, 1};
  if (head_pairs) {
    dims[1] = static_cast<cuuint64_t>(a.heads);
    dims[2] = static_cast<cuuint64_t>(a.n);
    strides[0] = sh;
    strides[1] = st;
    box[1] = 2;
    box[2] = kSlots;
  }
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(a.kv), dims,
                  strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

static std::atomic<int> g_decode_engine{NQ_DECODE_AUTO};
void set_decode_engine(int engine) { g_decode_engine.store(engine); }
int decode_engine() { return g_decode_engine.load(); }

// Tensor-core decode tiles: 128 rows = m slot tiles x hg heads x 16 slots,
// m = 8 / hg (rows past m * hg * 16 idle).  Keys need one RoPE table per slot
// tile, so they take hg >= 3 (m <= 2) and, with two tables, three warpgroups
// (shared memory); values take any hg.
static int tc_slot_tiles_per_tile(int hg, bool rope) {
  const int m = 8 / hg;
  return rope && m > 2 ? 0 : m;
}

template <int BITS, bool ROPE, bool EXACT, int NWG, int TABLES, int HG>
static cudaError_t launch_decode_tc_on(const CodecArgs& a, const CUtensorMap& map, int sms,
                                       cudaStream_t stream) {
  const void* fn =
      reinterpret_cast<const void*>(decode_tc_kernel<BITS, ROPE, EXACT, NWG, TABLES, HG>);
  constexpr int smem = tc_smem_bytes<NWG, TABLES>();
  static_assert(smem <= 232448, "one CTA per SM within 227 KB");
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int64_t grid = min64((a.num_tiles + NWG - 1) / NWG, static_cast<int64_t>(sms));
  decode_tc_kernel<BITS, ROPE, EXACT, NWG, TABLES, HG>
      <<<static_cast<unsigned>(grid), 128 * NWG, smem, stream>>>(a, map);
  return cudaGetLastError();
}

// Runs the tensor-core decode when the engine setting and the call allow it
// (*used = true), else leaves the call to the CUDA-core kernel.
template <int BITS, bool ROPE, bool EXACT>
static cudaError_t launch_decode_tc(CodecArgs a, const CUtensorMap& map, int units,
                                    cudaStream_t stream, bool* used) {
  *used = false;
  const int engine = decode_engine();
  const int m = tc_slot_tiles_per_tile(a.hg, ROPE);
  if (engine == NQ_DECODE_CUDA_CORES || m == 0) return cudaSuccess;
  const int nwg = ROPE && m == 2 ? 3 : 4;
  a.tc_m = m;
  a.tc_sgroups = (a.slot_tiles + m - 1) / m;
  a.num_tiles = static_cast<int64_t>(a.num_tiles / a.slot_tiles) * a.tc_sgroups;  // units * groups * sgroups
  a.div_sgroups = make_fastdiv(static_cast<uint32_t>(a.tc_sgroups));
  int dev = 0, sms = 0;
  cudaError_t err;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  // the per-CTA setup (the constant B operand) pays from about two tiles per warpgroup on
  if (engine == NQ_DECODE_AUTO && a.num_tiles < static_cast<int64_t>(2) * nwg * sms)
    return cudaSuccess;
  *used = true;
  if constexpr (!ROPE) {
    if (a.hg == 8) return launch_decode_tc_on<BITS, ROPE, EXACT, 4, 0, 8>(a, map, sms, stream);
    if (a.hg == 4) return launch_decode_tc_on<BITS, ROPE, EXACT, 4, 0, 4>(a, map, sms, stream);
    return launch_decode_tc_on<BITS, ROPE, EXACT, 4, 0, 0>(a, map, sms, stream);
  } else {
    if (a.hg == 8 || a.hg == 4) {
      CUtensorMap pairs;  // keys: rows in head pairs (see decode_tc_kernel)
      if ((err = make_out_map(&pairs, a, units, true)) != cudaSuccess) return err;
      if (a.hg == 8) return launch_decode_tc_on<BITS, ROPE, EXACT, 4, 1, 8>(a, pairs, sms, stream);
      return launch_decode_tc_on<BITS, ROPE, EXACT, 3, 2, 4>(a, pairs, sms, stream);
    }
    if (m == 1) return launch_decode_tc_on<BITS, ROPE, EXACT, 4, 1, 0>(a, map, sms, stream);
    return launch_decode_tc_on<BITS, ROPE, EXACT, 3, 2, 0>(a, map, sms, stream);
  }
}

template <int BITS, bool ROPE, bool EXACT>
static cudaError_t launch_one(bool decode, CodecArgs a, int units, cudaStream_t stream) {
  a.hg = pick_head_group(a.heads);
  a.ngroups = a.heads / a.hg;
  a.slot_tiles = (a.n + kSlots - 1) / kSlots;
  if (decode) {
    a.num_tiles = static_cast<int64_t>(units) * a.slot_tiles * a.ngroups;
  } else {
    // encode: tiles of 16 (unit, slot) pairs over all units
    a.pairs = static_cast<int64_t>(units) * a.n;
    if (a.pairs >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    a.num_tiles = (a.pairs + kSlots - 1) / kSlots * a.ngroups;
    if (a.n > 0) a.div_n = make_fastdiv(static_cast<uint32_t>(a.n));
  }
  if (a.num_tiles == 0) return cudaSuccess;
  if (a.num_tiles >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  a.div_groups = make_fastdiv(static_cast<uint32_t>(a.ngroups));
  a.div_stiles = make_fastdiv(static_cast<uint32_t>(a.slot_tiles));
  const int threads = 32 * a.hg;
  const int rows_bytes = (threads / 2) * kRowPad;
  size_t smem;
  const void* fn;
  CUtensorMap map;
  if (decode) {
    cudaError_t e = make_out_map(&map, a, units);
    if (e != cudaSuccess) return e;
    bool used = false;
    if ((e = launch_decode_tc<BITS, ROPE, EXACT>(a, map, units, stream, &used)) != cudaSuccess ||
        used)
      return e;
    smem = 1024 + static_cast<size_t>(threads / 32) * kOutTileBytes +
           (ROPE ? 2 * kCsBytes + 2 * kRawBytes : 0);
    fn = reinterpret_cast<const void*>(decode_kernel<BITS, ROPE, EXACT>);
  } else {
    smem = 2 * (static_cast<size_t>(rows_bytes) + (ROPE ? kCsBytes : 0)) + (ROPE ? kRawBytes : 0);
    fn = reinterpret_cast<const void*>(encode_kernel<BITS, ROPE, EXACT>);
  }
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 0, per_sm = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem)) !=
      cudaSuccess)
    return err;
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = min64(a.num_tiles, static_cast<int64_t>(sms) * per_sm);
  if (decode)
    decode_kernel<BITS, ROPE, EXACT><<<static_cast<unsigned>(grid), threads, smem, stream>>>(a, map);
  else
    encode_kernel<BITS, ROPE, EXACT><<<static_cast<unsigned>(grid), threads, smem, stream>>>(a);
  return cudaGetLastError();
}

static cudaError_t launch_kind(bool decode, const CodecArgs& a, int bits, bool rope, bool exact,
                               int units, cudaStream_t stream) {
  if (exact) {
    if (bits == 3)
      return rope ? launch_one<3, true, true>(decode, a, units, stream)
                  : launch_one<3, false, true>(decode, a, units, stream);
    return rope ? launch_one<2, true, true>(decode, a, units, stream)
                : launch_one<2, false, true>(decode, a, units, stream);
  }
  if (bits == 3)
    return rope ? launch_one<3, true, false>(decode, a, units, stream)
                : launch_one<3, false, false>(decode, a, units, stream);
  return rope ? launch_one<2, true, false>(decode, a, units, stream)
              : launch_one<2, false, false>(decode, a, units, stream);
}

cudaError_t codec_read_clear_error(uint32_t* flags) {
  cudaError_t err = cudaDeviceSynchronize();
  if (err != cudaSuccess) return err;
  unsigned int v = 0, zero = 0;
  if ((err = cudaMemcpyFromSymbol(&v, g_nq_error, sizeof(v))) != cudaSuccess) return err;
  if ((err = cudaMemcpyToSymbol(g_nq_error, &zero, sizeof(zero))) != cudaSuccess) return err;
  *flags = v;
  return cudaSuccess;
}

static CodecArgs common_args(int heads, int64_t n, int64_t slot0, int64_t pos_base,
                             const int32_t* idx, int64_t idx_stride, const float* tab,
                             int64_t max_pos) {
  CodecArgs a{};
  a.heads = heads;
  a.n = n;
  a.slot0 = slot0;
  a.pos_base = pos_base;
  a.idx = idx;
  a.idx_stride = idx_stride;
  a.tab = reinterpret_cast<const float2*>(tab);
  a.n_a = (max_pos + 255) / 256;
  return a;
}

cudaError_t launch_encode(const EncodeLaunch& L, cudaStream_t stream) {
  CodecArgs a = common_args(L.heads, L.n, L.slot0, L.pos_base, L.kept, L.kept_stride, L.rope_tab,
                            L.rope_max_pos);
  a.T_in = L.T_in;
  if (L.K) {
    CodecArgs k = a;
    k.kv = static_cast<const uint16_t*>(L.K);
    k.su = L.ks.unit;
    k.sh = L.ks.head;
    k.st = L.ks.token;
    k.codes = L.k_out.codes;
    k.meta = L.k_out.meta;
    k.pu = L.k_out.unit_stride;
    k.ph = L.k_out.head_stride;
    cudaError_t err = launch_kind(false, k, L.k_out.bits, true, L.exact, L.units, stream);
    if (err != cudaSuccess) return err;
  }
  if (L.V) {
    CodecArgs v = a;
    v.kv = static_cast<const uint16_t*>(L.V);
    v.su = L.vs.unit;
    v.sh = L.vs.head;
    v.st = L.vs.token;
    v.codes = L.v_out.codes;
    v.meta = L.v_out.meta;
    v.pu = L.v_out.unit_stride;
    v.ph = L.v_out.head_stride;
    return launch_kind(false, v, L.v_out.bits, false, L.exact, L.units, stream);
  }
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream) {
  CodecArgs a = common_args(L.heads, L.n, L.slot0, L.pos_base, L.positions, L.pos_stride,
                            L.rope_tab, L.rope_max_pos);
  if (L.K_out) {
    CodecArgs k = a;
    k.kv = static_cast<const uint16_t*>(L.K_out);
    k.su = L.kos.unit;
    k.sh = L.kos.head;
    k.st = L.kos.token;
    k.codes = L.k_in.codes;
    k.meta = L.k_in.meta;
    k.pu = L.k_in.unit_stride;
    k.ph = L.k_in.head_stride;
    cudaError_t err = launch_kind(true, k, L.k_in.bits, true, L.exact, L.units, stream);
    if (err != cudaSuccess) return err;
  }
  if (L.V_out) {
    CodecArgs v = a;
    v.kv = static_cast<const uint16_t*>(L.V_out);
    v.su = L.vos.unit;
    v.sh = L.vos.head;
    v.st = L.vos.token;
    v.codes = L.v_in.codes;
    v.meta = L.v_in.meta;
    v.pu = L.v_in.unit_stride;
    v.ph = L.v_in.head_stride;
    return launch_kind(true, v, L.v_in.bits, false, L.exact, L.units, stream);
  }
  return cudaSuccess;
}

// ------------------------------------------------------ E8 quantiser alone
// One thread per pair of groups (2p in lane x, 2p + 1 in lane y) of a
// [groups][8] fp32 array, with the encode kernels' decision and code
// functions: the regular step (nearest point, then clamp) or, with BOX, the
// nearest point inside the code box with the coset bit folded into code 7.
// The CTA loop bound is uniform across each warp (threads past the end run on
// zeros), as the warp vote in e8_choose needs.
template <int BITS, bool BOX>
__global__ void __launch_bounds__(256) e8_quantise_kernel(const float* __restrict__ y,
                                                          int64_t groups, uint32_t* codes,
                                                          uint8_t* coset) {
  const int64_t pairs = (groups + 1) / 2;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x; base < pairs;
       base += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = base + threadIdx.x;
    const int64_t g0 = 2 * p, g1 = 2 * p + 1;
    float a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a[i] = g0 < groups ? __ldg(y + 8 * g0 + i) : 0.0f;
      b[i] = g1 < groups ? __ldg(y + 8 * g1 + i) : 0.0f;
    }
    float2 yy[8];
    float big = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      yy[i] = make_float2(a[i], b[i]);
      big = fmaxf(big, fmaxf(fabsf(a[i]), fabsf(b[i])));
    }
    uint32_t cx, cy;
    bool hx, hy;
    if (BOX) {
      e8_box_codes<BITS>(yy, cx, cy);
      hx = (cx >> (7 * BITS)) & 1u;
      hy = (cy >> (7 * BITS)) & 1u;
    } else {
      bool ox, oy;
      e8_choose(yy, !(big < 7.0f), hx, hy, ox, oy);
      e8_codes<BITS>(yy, hx, hy, ox, oy, cx, cy);
    }
    if (g0 < groups) {
      codes[g0] = cx;
      coset[g0] = hx ? 1 : 0;
    }
    if (g1 < groups) {
      codes[g1] = cy;
      coset[g1] = hy ? 1 : 0;
    }
  }
}

template <bool BOX>
static cudaError_t launch_e8(const float* y, int64_t groups, int bits, uint32_t* codes,
                             uint8_t* coset, cudaStream_t stream) {
  if (groups <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  const int64_t pairs = (groups + 1) / 2;
  const int64_t grid = min64((pairs + 255) / 256, static_cast<int64_t>(sms) * 8);
  if (bits == 3)
    e8_quantise_kernel<3, BOX><<<static_cast<unsigned>(grid), 256, 0, stream>>>(y, groups, codes,
                                                                                coset);
  else
    e8_quantise_kernel<2, BOX><<<static_cast<unsigned>(grid), 256, 0, stream>>>(y, groups, codes,
                                                                                coset);
  return cudaGetLastError();
}

cudaError_t launch_e8_quantise(const float* y, int64_t groups, int bits, uint32_t* codes,
                               uint8_t* coset, cudaStream_t stream) {
  return launch_e8<false>(y, groups, bits, codes, coset, stream);
}

cudaError_t launch_e8_box_quantise(const float* y, int64_t groups, int bits, uint32_t* codes,
                                   uint8_t* coset, cudaStream_t stream) {
  return launch_e8<true>(y, groups, bits, codes, coset, stream);
}

}  // namespace nq
