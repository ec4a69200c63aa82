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
// Design (B200): one thread owns one 128-coordinate vector in registers
// (64 packed fp32 pairs), so the Hadamard butterflies, the RoPE pairs
// (i, i+64) and the 8-coordinate E8 groups need no shuffles.  A persistent
// CTA of HG warps walks tiles of 32 slots x HG heads; every thread stages its
// own 256-byte row with a bulk async copy (TMA engine, mbarrier completion)
// into a padded shared-memory row, double buffered, so that HBM reads of the
// next tiles overlap the arithmetic of the current one.  The per-position
// RoPE (cos, sin) pairs of a tile are combined once per CTA and shared by the
// HG heads.  Decode writes each reconstructed row to shared memory and
// stores it with a bulk async copy.
#include "nq_internal.h"

namespace nq {

// ------------------------------------------------------------- tile map
struct KindParams {
  const uint16_t* src;   // encode: bf16 input; decode: bf16 output (as uint16_t*)
  int64_t su, sh, st;    // element strides of the bf16 tensor
  uint32_t* codes;
  uint32_t* meta;
  int64_t pu, ph;        // vector strides of the packed store
  int bits;
  int rope;
};

struct CodecArgs {
  KindParams kind[2];
  int nkinds;
  int heads, hg, ngroups;
  int64_t T_in;          // encode: input tokens per (unit, head)
  int64_t n, slot0, pos_base;
  const int32_t* idx;    // encode: kept (source tokens); decode: positions
  int64_t idx_stride;
  const float2* tab;
  int64_t n_a;
  int64_t slot_tiles, num_tiles;
};

struct Tile {
  int kind, group, unit;
  int64_t stile;
};

__device__ __forceinline__ Tile tile_of(const CodecArgs& a, int64_t t) {
  Tile r;
  r.kind = static_cast<int>(t % a.nkinds);
  t /= a.nkinds;
  r.group = static_cast<int>(t % a.ngroups);
  t /= a.ngroups;
  r.stile = t % a.slot_tiles;
  r.unit = static_cast<int>(t / a.slot_tiles);
  return r;
}

// cs table of one tile in shared memory: float4 cs[32 pair-pairs][32 slots],
// entry (j, slot) = (c_2j, c_2j+1, s_2j, s_2j+1) at that slot's position.
constexpr int kCsBytes = 32 * kTileSlots * 16;

__device__ __forceinline__ void fill_cs(const CodecArgs& a, const Tile& tl, bool use_idx,
                                        float4* cs, int tid, int nthreads) {
  for (int e = tid; e < 32 * kTileSlots; e += nthreads) {
    const int slot_l = e % kTileSlots;
    const int j = e / kTileSlots;
    const int64_t slot = tl.stile * kTileSlots + slot_l;
    float4 v = make_float4(1.f, 1.f, 0.f, 0.f);
    if (slot < a.n) {
      int64_t p = slot;
      if (use_idx && a.idx) p = __ldg(a.idx + static_cast<int64_t>(tl.unit) * a.idx_stride + slot);
      p += a.pos_base;
      const float2 c0 = rope_cs(a.tab, a.n_a, p, 2 * j);
      const float2 c1 = rope_cs(a.tab, a.n_a, p, 2 * j + 1);
      v = make_float4(c0.x, c1.x, c0.y, c1.y);
    }
    cs[j * kTileSlots + slot_l] = v;
  }
}

// --------------------------------------------------------- Hadamard (fp32)
// Unnormalised Sylvester transform on 128 coordinates held as 64 pairs
// v[j] = (x_2j, x_2j+1); stage order h = 1, 2, ..., 64 as in the reference
// definition.  Every output is the IEEE fp32 sum / difference of the same
// two operands as in the scalar butterfly network.
__device__ __forceinline__ void fwht128(float2 (&v)[64]) {
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const float a = v[j].x, b = v[j].y;
    v[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
#pragma unroll
  for (int hp = 1; hp < 64; hp <<= 1) {
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      if (!(j & hp)) {
        const float2 A = v[j], B = v[j + hp];
        v[j] = add2(A, B);
        v[j + hp] = sub2(A, B);
      }
    }
  }
}

// ------------------------------------------------------------ E8 (fp32)
// One D8 + shift decode (shift 0 or 1/2), Conway-Sloane:
//   u = y - shift; f = rint(u) (ties to even, via the 1.5*2^23 round trick);
//   e = u - f; d = e0^2 then fma chain; parity = sum f mod 2 (LSB of the
//   rounded float's bits); m = max |e|.
struct D8 {
  float f[8], e[8];
  float d, m;
  uint32_t par;
};

__device__ __forceinline__ void d8_decode(const float (&y)[8], float shift, D8& o) {
  uint32_t par = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float u = __fsub_rn(y[i], shift);
    const float rr = __fadd_rn(u, kMagicRound);
    o.f[i] = __fsub_rn(rr, kMagicRound);
    o.e[i] = __fsub_rn(u, o.f[i]);
    par ^= __float_as_uint(rr);
  }
  float d = __fmul_rn(o.e[0], o.e[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) d = __fmaf_rn(o.e[i], o.e[i], d);
  float m = fabsf(o.e[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, fabsf(o.e[i]));
  o.par = par & 1u;
  // an odd sum re-rounds the worst coordinate: |e|^2 grows by 1 - 2|e_k|
  o.d = o.par ? __fadd_rn(d, __fmaf_rn(-2.0f, m, 1.0f)) : d;
  o.m = m;
}

// Nearest E8 point of y and its b-bit codes, packed as BITS*8 bits
// (code i at bits [BITS*i, BITS*i + BITS)); returns the coset (1 = half).
template <int BITS>
__device__ __forceinline__ uint32_t e8_codes(const float (&y)[8], uint32_t& half_out) {
  D8 c0, c1;
  d8_decode(y, 0.0f, c0);
  d8_decode(y, 0.5f, c1);
  const bool half = c1.d < c0.d;
  const float m = half ? c1.m : c0.m;
  bool found = !(half ? c1.par : c0.par);  // even sum: nothing to fix
  constexpr float kOffHalf = static_cast<float>(1 << (BITS - 1));
  constexpr float kOffInt = static_cast<float>((1 << (BITS - 1)) - 1);
  constexpr float kMaxHalf = static_cast<float>((1 << BITS) - 1);
  constexpr float kMaxInt = static_cast<float>((1 << BITS) - 2);
  const float off = half ? kOffHalf : kOffInt;
  const float jmax = half ? kMaxHalf : kMaxInt;
  uint32_t acc = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float e = half ? c1.e[i] : c0.e[i];
    float f = half ? c1.f[i] : c0.f[i];
    const bool hit = !found && (fabsf(e) == m);
    found = found || hit;
    if (hit) f = __fadd_rn(f, e >= 0.0f ? 1.0f : -1.0f);
    const float jf = fminf(fmaxf(__fadd_rn(f, off), 0.0f), jmax);
    acc += __float_as_uint(__fadd_rn(jf, kTwo23)) << (BITS * i);
  }
  half_out = half ? 1u : 0u;
  return acc & ((1u << (8 * BITS)) - 1u);
}

// ----------------------------------------------------------- encode core
// Staged bf16 row -> fp32 pairs; keys: RoPE removed at the slot's position.
template <bool ROPE>
__device__ __forceinline__ void load_row(float2 (&v)[64], uint32_t row_addr, uint32_t cs_addr) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint4 q = lds128(row_addr + 16 * c);
    v[4 * c + 0] = make_float2(bf16lo(q.x), bf16hi(q.x));
    v[4 * c + 1] = make_float2(bf16lo(q.y), bf16hi(q.y));
    v[4 * c + 2] = make_float2(bf16lo(q.z), bf16hi(q.z));
    v[4 * c + 3] = make_float2(bf16lo(q.w), bf16hi(q.w));
  }
  if (ROPE) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float4 t = lds128f(cs_addr + j * (kTileSlots * 16));
      const float2 c2 = make_float2(t.x, t.y), s2 = make_float2(t.z, t.w);
      const float2 A = v[j], B = v[j + 32];
      const float2 bs = mul2(B, s2);
      const float2 as = mul2(A, s2);
      v[j] = fma2(A, c2, bs);
      v[j + 32] = fma2(B, c2, make_float2(-as.x, -as.y));
    }
  }
}

// Rotate, scale, E8-quantise and pack one vector.
template <int BITS>
__device__ __forceinline__ void quantise(float2 (&v)[64], uint32_t* codes, uint32_t* meta) {
  fwht128(v);
  float M = 0.0f;
#pragma unroll
  for (int j = 0; j < 64; ++j) M = fmaxf(M, fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
  const float G = __uint_as_float(BITS == 3 ? kG3Bits : kG2Bits);
  const float C = __uint_as_float(kCBits);
  const float sm = fminf(__fmul_rn(M, G), 65504.0f);
  const __half sh = __float2half_rn(sm);
  const float sig = __half2float(sh);
  const float r = (sig == 0.0f) ? 0.0f : __fdiv_rn(C, sig);
  const float2 r2 = make_float2(r, r);

  uint32_t gw[16];
  uint32_t cmask = 0;
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    const float2 p0 = mul2(v[4 * g + 0], r2), p1 = mul2(v[4 * g + 1], r2);
    const float2 p2 = mul2(v[4 * g + 2], r2), p3 = mul2(v[4 * g + 3], r2);
    const float y[8] = {p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y};
    uint32_t half;
    gw[g] = e8_codes<BITS>(y, half);
    cmask |= half << g;
  }
  uint4* dst = reinterpret_cast<uint4*>(codes);
  if (BITS == 3) {
    // three words per 32 coordinates (four 24-bit groups)
    uint32_t w[12];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t g0 = gw[4 * q], g1 = gw[4 * q + 1], g2 = gw[4 * q + 2], g3 = gw[4 * q + 3];
      w[3 * q + 0] = g0 | (g1 << 24);
      w[3 * q + 1] = (g1 >> 8) | (g2 << 16);
      w[3 * q + 2] = (g2 >> 16) | (g3 << 8);
    }
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
  } else {
    uint32_t w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) w[q] = gw[2 * q] | (gw[2 * q + 1] << 16);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  *meta = cmask | (static_cast<uint32_t>(__half_as_ushort(sh)) << 16);
}

// ----------------------------------------------------------- decode core
template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[4 * BITS], int c) {
  const int p = BITS * c;
  const int wi = p >> 5, off = p & 31;
  uint32_t x;
  if (off + BITS <= 32) {
    x = w[wi] >> off;
  } else {
    x = __funnelshift_r(w[wi], w[wi + 1], off);
  }
  return x & ((1u << BITS) - 1u);
}

template <int BITS, bool ROPE>
__device__ __forceinline__ void decode_vector(const uint32_t (&w)[4 * BITS], uint32_t meta,
                                              uint32_t cs_addr, uint32_t out_addr) {
  float2 v[64];
  // x = 2^22 + j (the fp32 spacing at 2^22 is 1/2, so the mantissa holds 2j);
  // t = 2x - 2^23 - (2^b - 2) - h, every constant below 2^24: exact.
  constexpr float kBase = -8388608.0f - static_cast<float>((1 << BITS) - 2);
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    const float kg = kBase - static_cast<float>((meta >> g) & 1u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 8 * g + 2 * k;
      const float x0 = __uint_as_float(0x4A800000u | (code_at<BITS>(w, c) << 1));
      const float x1 = __uint_as_float(0x4A800000u | (code_at<BITS>(w, c + 1) << 1));
      v[4 * g + k] = fma2(make_float2(x0, x1), make_float2(2.0f, 2.0f), make_float2(kg, kg));
    }
  }
  fwht128(v);
  const float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(meta >> 16)));
  const float kappa = __fmul_rn(__fmul_rn(sig, 0.5f), __uint_as_float(kCBits));
  const float2 k2 = make_float2(kappa, kappa);
#pragma unroll
  for (int j = 0; j < 64; ++j) v[j] = mul2(v[j], k2);
  if (ROPE) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float4 t = lds128f(cs_addr + j * (kTileSlots * 16));
      const float2 c2 = make_float2(t.x, t.y), s2 = make_float2(t.z, t.w);
      const float2 A = v[j], B = v[j + 32];
      const float2 bs = mul2(B, s2);
      const float2 as = mul2(A, s2);
      v[j] = fma2(A, c2, make_float2(-bs.x, -bs.y));
      v[j + 32] = fma2(B, c2, as);
    }
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    uint32_t q[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[4 * c + k].x, v[4 * c + k].y);
      q[k] = *reinterpret_cast<const uint32_t*>(&b);
    }
    sts128(out_addr + 16 * c, make_uint4(q[0], q[1], q[2], q[3]));
  }
}

// ------------------------------------------------------------- encode
__global__ void __launch_bounds__(256, 1) encode_kernel(const CodecArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int nthreads = blockDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rows_bytes = nthreads * kRowPad;
  const int stage_bytes = rows_bytes + kCsBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * stage_bytes);

  const int64_t first = blockIdx.x, step = gridDim.x;
  const int64_t my_tiles = first < a.num_tiles ? (a.num_tiles - 1 - first) / step + 1 : 0;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](int64_t k, int s) {
    const Tile tl = tile_of(a, first + k * step);
    const KindParams& kp = a.kind[tl.kind];
    unsigned char* st = smem + s * stage_bytes;
    const int h = tl.group * a.hg + warp;
    const int64_t slot = tl.stile * kTileSlots + lane;
    const int64_t valid = min64(kTileSlots, a.n - tl.stile * kTileSlots);
    if (tid == 0) mbar_arrive_expect_tx(&bars[s], static_cast<uint32_t>(valid * a.hg * 256));
    if (slot < a.n) {
      int64_t src = slot;
      if (a.idx) src = __ldg(a.idx + static_cast<int64_t>(tl.unit) * a.idx_stride + slot);
      src = src < 0 ? 0 : (src >= a.T_in ? a.T_in - 1 : src);
      const uint16_t* g = kp.src + tl.unit * kp.su + h * kp.sh + src * kp.st;
      bulk_g2s(st + tid * kRowPad, g, 256, &bars[s]);
    }
    if (kp.rope) fill_cs(a, tl, true, reinterpret_cast<float4*>(st + rows_bytes), tid, nthreads);
  };

  if (my_tiles > 0) issue(0, 0);
  if (my_tiles > 1) issue(1, 1);
  __syncthreads();

  for (int64_t k = 0; k < my_tiles; ++k) {
    const int s = static_cast<int>(k & 1);
    const uint32_t parity = static_cast<uint32_t>((k >> 1) & 1);
    const bool ok = mbar_wait_bounded(&bars[s], parity);
    if (!__syncthreads_and(ok)) return;  // a copy never landed: error word set, stop

    const Tile tl = tile_of(a, first + k * step);
    const KindParams& kp = a.kind[tl.kind];
    const int h = tl.group * a.hg + warp;
    const int64_t slot = tl.stile * kTileSlots + lane;
    unsigned char* st = smem + s * stage_bytes;
    const uint32_t row = smem_u32(st + tid * kRowPad);
    const uint32_t csa = smem_u32(st + rows_bytes) + lane * 16;
    const bool valid = slot < a.n;
    // The staged row (and its RoPE pairs) moves to registers, then the stage
    // is refilled with tile k+2 while this tile is quantised.
    float2 v[64];
    if (valid) {
      if (kp.rope) load_row<true>(v, row, csa);
      else load_row<false>(v, row, csa);
    }
    __syncthreads();  // everyone is done with stage s
    if (k + 2 < my_tiles) issue(k + 2, s);
    if (valid) {
      const int64_t vec = tl.unit * kp.pu + h * kp.ph + a.slot0 + slot;
      uint32_t* codes = kp.codes + vec * (4 * kp.bits);
      uint32_t* meta = kp.meta + vec;
      if (kp.bits == 3) quantise<3>(v, codes, meta);
      else quantise<2>(v, codes, meta);
    }
  }
}

// ------------------------------------------------------------- decode
__global__ void __launch_bounds__(256, 1) decode_kernel(const CodecArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int nthreads = blockDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned char* out_rows = smem;
  float4* cs_buf[2] = {reinterpret_cast<float4*>(smem + nthreads * kRowPad),
                       reinterpret_cast<float4*>(smem + nthreads * kRowPad + kCsBytes)};
  const uint32_t row = smem_u32(out_rows + tid * kRowPad);

  const int64_t first = blockIdx.x, step = gridDim.x;
  const int64_t my_tiles = first < a.num_tiles ? (a.num_tiles - 1 - first) / step + 1 : 0;

  uint32_t w[12];
  uint32_t meta = 0;
  auto load_in = [&](int64_t k) {
    const Tile tl = tile_of(a, first + k * step);
    const KindParams& kp = a.kind[tl.kind];
    const int h = tl.group * a.hg + warp;
    const int64_t slot = tl.stile * kTileSlots + lane;
    if (slot < a.n) {
      const int64_t vec = tl.unit * kp.pu + h * kp.ph + a.slot0 + slot;
      const uint4* src = reinterpret_cast<const uint4*>(kp.codes + vec * (4 * kp.bits));
      const uint4 q0 = __ldg(src), q1 = __ldg(src + 1);
      w[0] = q0.x; w[1] = q0.y; w[2] = q0.z; w[3] = q0.w;
      w[4] = q1.x; w[5] = q1.y; w[6] = q1.z; w[7] = q1.w;
      if (kp.bits == 3) {
        const uint4 q2 = __ldg(src + 2);
        w[8] = q2.x; w[9] = q2.y; w[10] = q2.z; w[11] = q2.w;
      }
      meta = __ldg(kp.meta + vec);
    }
  };
  auto prep_cs = [&](int64_t k, int b) {
    const Tile tl = tile_of(a, first + k * step);
    if (a.kind[tl.kind].rope) fill_cs(a, tl, true, cs_buf[b], tid, nthreads);
  };

  if (my_tiles > 0) {
    prep_cs(0, 0);
    load_in(0);
  }
  __syncthreads();
  for (int64_t k = 0; k < my_tiles; ++k) {
    const Tile tl = tile_of(a, first + k * step);
    const KindParams& kp = a.kind[tl.kind];
    const int h = tl.group * a.hg + warp;
    const int64_t slot = tl.stile * kTileSlots + lane;
    uint32_t wc[12];
#pragma unroll
    for (int i = 0; i < 12; ++i) wc[i] = w[i];
    const uint32_t mc = meta;
    if (k + 1 < my_tiles) load_in(k + 1);  // next tile's codes in flight during this one
    if (slot < a.n) {
      const uint32_t csa = smem_u32(cs_buf[k & 1]) + lane * 16;
      bulk_wait_read_all();  // this thread's previous row store has left smem
      if (kp.bits == 3) {
        const uint32_t(&w3)[12] = wc;
        if (kp.rope) decode_vector<3, true>(w3, mc, csa, row);
        else decode_vector<3, false>(w3, mc, csa, row);
      } else {
        const uint32_t(&w2)[8] = *reinterpret_cast<const uint32_t(*)[8]>(wc);
        if (kp.rope) decode_vector<2, true>(w2, mc, csa, row);
        else decode_vector<2, false>(w2, mc, csa, row);
      }
      fence_proxy_async_smem();
      uint16_t* dst = const_cast<uint16_t*>(kp.src) + tl.unit * kp.su + h * kp.sh + slot * kp.st;
      bulk_s2g(dst, out_rows + tid * kRowPad, 256);
      bulk_commit();
    }
    if (k + 1 < my_tiles) prep_cs(k + 1, static_cast<int>((k + 1) & 1));
    __syncthreads();
  }
  bulk_wait_all();
}

// ---------------------------------------------------------------- launch
static int pick_head_group(int heads) {
  for (int g = 8; g >= 1; --g)
    if (heads % g == 0) return g;
  return 1;
}

static cudaError_t launch_codec(bool decode, CodecArgs& a, int units, cudaStream_t stream) {
  a.hg = pick_head_group(a.heads);
  a.ngroups = a.heads / a.hg;
  a.slot_tiles = (a.n + kTileSlots - 1) / kTileSlots;
  a.num_tiles = static_cast<int64_t>(units) * a.slot_tiles * a.ngroups * a.nkinds;
  if (a.num_tiles == 0) return cudaSuccess;
  const int threads = 32 * a.hg;
  size_t smem;
  const void* fn;
  if (decode) {
    smem = static_cast<size_t>(threads) * kRowPad + 2 * kCsBytes;
    fn = reinterpret_cast<const void*>(decode_kernel);
  } else {
    smem = 2 * (static_cast<size_t>(threads) * kRowPad + kCsBytes) + 16;
    fn = reinterpret_cast<const void*>(encode_kernel);
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
    decode_kernel<<<static_cast<unsigned>(grid), threads, smem, stream>>>(a);
  else
    encode_kernel<<<static_cast<unsigned>(grid), threads, smem, stream>>>(a);
  return cudaGetLastError();
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

cudaError_t launch_encode(const EncodeLaunch& L, cudaStream_t stream) {
  CodecArgs a{};
  int nk = 0;
  if (L.K) {
    a.kind[nk++] = KindParams{static_cast<const uint16_t*>(L.K), L.ks.unit, L.ks.head, L.ks.token,
                              L.k_out.codes, L.k_out.meta, L.k_out.unit_stride,
                              L.k_out.head_stride, L.k_out.bits, 1};
  }
  if (L.V) {
    a.kind[nk++] = KindParams{static_cast<const uint16_t*>(L.V), L.vs.unit, L.vs.head, L.vs.token,
                              L.v_out.codes, L.v_out.meta, L.v_out.unit_stride,
                              L.v_out.head_stride, L.v_out.bits, 0};
  }
  a.nkinds = nk;
  a.heads = L.heads;
  a.T_in = L.T_in;
  a.n = L.n;
  a.slot0 = L.slot0;
  a.pos_base = L.pos_base;
  a.idx = L.kept;
  a.idx_stride = L.kept_stride;
  a.tab = reinterpret_cast<const float2*>(L.rope_tab);
  a.n_a = (L.rope_max_pos + 255) / 256;
  return launch_codec(false, a, L.units, stream);
}

cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream) {
  CodecArgs a{};
  int nk = 0;
  if (L.K_out) {
    a.kind[nk++] = KindParams{static_cast<const uint16_t*>(L.K_out), L.kos.unit, L.kos.head,
                              L.kos.token, L.k_in.codes, L.k_in.meta, L.k_in.unit_stride,
                              L.k_in.head_stride, L.k_in.bits, 1};
  }
  if (L.V_out) {
    a.kind[nk++] = KindParams{static_cast<const uint16_t*>(L.V_out), L.vos.unit, L.vos.head,
                              L.vos.token, L.v_in.codes, L.v_in.meta, L.v_in.unit_stride,
                              L.v_in.head_stride, L.v_in.bits, 0};
  }
  a.nkinds = nk;
  a.heads = L.heads;
  a.T_in = 0;
  a.n = L.n;
  a.slot0 = L.slot0;
  a.pos_base = L.pos_base;
  a.idx = L.positions;
  a.idx_stride = L.pos_stride;
  a.tab = reinterpret_cast<const float2*>(L.rope_tab);
  a.n_a = (L.rope_max_pos + 255) / 256;
  return launch_codec(true, a, L.units, stream);
}

}  // namespace nq
