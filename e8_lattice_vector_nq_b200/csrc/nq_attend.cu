// nq_attend.cu -- decode-phase attention over the packed cache for sm_100a,
// reconstructing keys and values inside the attention instead of writing the
// bf16 cache first (the on-demand reconstruction within FlashAttention of
// "VQKV" (section "Decoding"), applied to the E8-coded NexusQuant cache).
//
// For unit u and query head j (KV head h = j / G):
//   s_t = scale * q_j . k_t,  o_j = sum_t softmax(s)_t v_t,  lse_j = log sum_t exp(s_t)
// over the n kept tokens, where k_t, v_t are the fp32 reconstructions that the
// decode kernel rounds to bf16 (keys re-rotated at their positions).
//
// Design (B200).  Split-K over the tokens (flash decoding): a CTA takes one
// (unit, KV head, chunk of kChunk tokens) and all G query heads of the group.
//   pass 1: two threads per token rebuild the key half by half (the decode
//           kernel's arithmetic: unpack, Hadamard, kappa, RoPE with the
//           two-level table rows read through L1) and dot it with the G
//           queries held in shared memory as (q_i, q_{i+64}) pairs;
//   softmax: one warp per query head: chunk max m, l = sum exp(s - m), and
//           the weights w_t = exp(s_t - m) * kappa_t in place;
//   pass 2: values stay in the code domain: since v_t = kappa_t * H t_t (H the
//           unnormalised Hadamard matrix, t_t the 2q integers), the chunk
//           accumulates a = sum_t w_t t_t per coordinate (thread = coordinate,
//           two token streams), and H is applied once per query head when the
//           chunks are combined (o = H A / L).
// The combine kernel merges the chunks' (m, l, a) with the usual rescaling,
// applies the 128-point Hadamard transform across one warp and writes o, lse.
#include "nq_codec_math.cuh"
#include "nq_internal.h"

namespace nq {

constexpr int kChunk = 512;         // tokens per CTA
constexpr int kAttThreads = 256;
constexpr int kMaxGroup = 8;        // query heads per KV head
constexpr int kPartFloats = 2 + kD;  // m, l, a[128]

struct AttendArgs {
  const float* q;  // [units][heads * G][128]
  const uint32_t *kc, *km, *vc, *vm;
  int64_t kpu, kph, vpu, vph;  // vector strides of the packed stores
  int heads, G, GT;  // GT: query heads computed per CTA (G rounded up to 1, 2, 4 or 8)
  int64_t n, slot0;
  const int32_t* pos;
  int64_t pos_stride, pos_base;
  const float2* tab;
  int64_t n_a;
  float scale;
  int64_t nsplit;
  float* part;  // [units][heads][nsplit][G][kPartFloats]
};

constexpr int kStreams = 8;  // token streams of pass 2 (one per warp)

// Dynamic shared memory of the partial kernel for GT query heads per CTA.
template <int BV, int GT>
struct AttSmem {
  static constexpr int kQ = GT * 64 * 8;          // float2 qp[GT][64]
  static constexpr int kSc = kChunk * GT * 4;     // float sc[kChunk][GT]
  static constexpr int kVw = kChunk * 4 * BV * 4;  // uint32 vw[kChunk][4 BV]
  static constexpr int kMeta = kChunk * 4;        // uint32 vmeta[kChunk]
  static constexpr int kAcc = kStreams * GT * kD * 4;  // float acc[kStreams][GT][128]
  static constexpr int kRed = GT * 2 * 4;         // float red[GT][2]
  static constexpr int bytes = kQ + kSc + kVw + kMeta + kAcc + kRed;
};

template <int BK, int BV, int GT>
__global__ void __launch_bounds__(kAttThreads, 2) attend_partial_kernel(const AttendArgs a) {
  extern __shared__ __align__(16) unsigned char att_smem[];
  using S = AttSmem<BV, GT>;
  float2(*qp)[64] = reinterpret_cast<float2(*)[64]>(att_smem);                     // (q_i, q_{i+64})
  float* sc = reinterpret_cast<float*>(att_smem + S::kQ);                          // [kChunk][GT]
  uint32_t* vw = reinterpret_cast<uint32_t*>(att_smem + S::kQ + S::kSc);           // value codes
  uint32_t* vmeta = reinterpret_cast<uint32_t*>(att_smem + S::kQ + S::kSc + S::kVw);
  float* accs = reinterpret_cast<float*>(att_smem + S::kQ + S::kSc + S::kVw + S::kMeta);
  float* red = accs + kStreams * GT * kD;                                          // [GT][2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot_l = lane & 15, half = lane >> 4;
  const int64_t split = blockIdx.x % a.nsplit;
  const int64_t uh = blockIdx.x / a.nsplit;
  const int h = static_cast<int>(uh % a.heads);
  const int64_t u = uh / a.heads;
  const int G = a.G;  // G <= GT; heads G..GT-1 of the CTA are zero queries
  const int64_t t0 = split * kChunk;
  const int nt = static_cast<int>(min64(kChunk, a.n - t0));

  // queries of the group, and the chunk's value codes (cp.async) and meta
  const float* qg = a.q + (u * a.heads * G + static_cast<int64_t>(h) * G) * kD;
  for (int e = tid; e < GT * 64; e += kAttThreads) {
    const int g = e >> 6, i = e & 63;
    qp[g][i] = g < G ? make_float2(__ldg(qg + g * kD + i), __ldg(qg + g * kD + i + 64))
                     : make_float2(0.f, 0.f);
  }
  const int64_t vbase = u * a.vpu + h * a.vph + a.slot0 + t0;
  {
    const char* src = reinterpret_cast<const char*>(a.vc + vbase * (4 * BV));
    const uint32_t dst = smem_u32(vw);
    for (int c = tid; c < nt * BV; c += kAttThreads) cp_async16(dst + c * 16, src + c * 16);
    cp_async_commit();
  }
  for (int t = tid; t < nt; t += kAttThreads) vmeta[t] = __ldg(a.vm + vbase + t);
  __syncthreads();  // qp ready

  // ---- pass 1: keys and scores (16 tokens per warp per round); each round's
  // codes, meta and position are loaded one round ahead
  uint32_t wn_[4 * BK];
  uint32_t meta_n = 0;
  int64_t pos_n = 0;
  auto load_round = [&](int r) {
    const int tt = r * 128 + warp * 16 + slot_l;
#pragma unroll
    for (int i = 0; i < 4 * BK; ++i) wn_[i] = 0;
    meta_n = 0;
    pos_n = 0;
    if (tt < nt) {
      const int64_t vec = u * a.kpu + h * a.kph + a.slot0 + t0 + tt;
      const uint4* src = reinterpret_cast<const uint4*>(a.kc + vec * (4 * BK));
#pragma unroll
      for (int c = 0; c < BK; ++c) {
        const uint4 x = __ldg(src + c);
        wn_[4 * c] = x.x;
        wn_[4 * c + 1] = x.y;
        wn_[4 * c + 2] = x.z;
        wn_[4 * c + 3] = x.w;
      }
      meta_n = __ldg(a.km + vec);
      pos_n = a.pos_base + (a.pos ? static_cast<int64_t>(__ldg(a.pos + u * a.pos_stride + t0 + tt))
                                  : t0 + tt);
    }
  };
  load_round(0);
  for (int r = 0; r < kChunk / 128; ++r) {
    const int tt = r * 128 + warp * 16 + slot_l;
    const bool valid = tt < nt;
    uint32_t w[4 * BK];
#pragma unroll
    for (int i = 0; i < 4 * BK; ++i) w[i] = wn_[i];
    const uint32_t meta = meta_n;
    const int64_t pos = pos_n;
    if (r + 1 < kChunk / 128 && (r + 1) * 128 < nt) load_round(r + 1);
    float2 v[32];
    reconstruct_half<BK>(w, meta, half, v);
    // RoPE: o_i = fmaf(x_i, c, -(x_{i+64} s)), o_{i+64} = fmaf(x_{i+64}, c, x_i s) with
    // c = fmaf(cA, cB, -(sA sB)), s = fmaf(sA, cB, cA sB) from the table rows of
    // p = 256 hi + lo (clamped into the table for out-of-contract positions)
    int64_t hi = pos >> 8;
    hi = hi < 0 ? 0 : (hi >= a.n_a ? a.n_a - 1 : hi);
    const float4* rowA = reinterpret_cast<const float4*>(a.tab + hi * kHalf + 32 * half);
    const float4* rowB =
        reinterpret_cast<const float4*>(a.tab + (a.n_a + (pos & 255)) * kHalf + 32 * half);
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const float4 A = __ldg(rowA + jj), B = __ldg(rowB + jj);
#pragma unroll
      for (int ww = 0; ww < 2; ++ww) {
        const float cA = ww ? A.z : A.x, sA = ww ? A.w : A.y;
        const float cB = ww ? B.z : B.x, sB = ww ? B.w : B.y;
        const float c = __fmaf_rn(cA, cB, -__fmul_rn(sA, sB));
        const float s = __fmaf_rn(sA, cB, __fmul_rn(cA, sB));
        const float2 P = v[2 * jj + ww];
        const float2 Q = mul2(P, make_float2(s, s));
        v[2 * jj + ww] = make_float2(__fmaf_rn(P.x, c, -Q.y), __fmaf_rn(P.y, c, Q.x));
      }
    }
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      float2 d0 = make_float2(0.f, 0.f), d1 = d0;
      const float4* qh = reinterpret_cast<const float4*>(&qp[g][32 * half]);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float4 qq = qh[j];
        d0 = fma2(v[2 * j], make_float2(qq.x, qq.y), d0);
        d1 = fma2(v[2 * j + 1], make_float2(qq.z, qq.w), d1);
      }
      float d = (d0.x + d0.y) + (d1.x + d1.y);
      d += __shfl_xor_sync(0xffffffffu, d, 16);
      if (half == 0 && valid) sc[tt * GT + g] = a.scale * d;
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- softmax statistics per query head (warp g), weights in place
  if (warp < GT) {
    const int g = warp;
    float m = -INFINITY;
    for (int t = lane; t < nt; t += 32) m = fmaxf(m, sc[t * GT + g]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int t = lane; t < nt; t += 32) {
      const float p = __expf(sc[t * GT + g] - m);
      l += p;
      const float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(vmeta[t] >> 16)));
      const float kappa = __fmul_rn(__fmul_rn(sig, 0.5f), __uint_as_float(kCBits));
      sc[t * GT + g] = p * kappa;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      red[2 * g] = m;
      red[2 * g + 1] = l;
    }
  }
  __syncthreads();

  // ---- pass 2: a[g][i] = sum_t w[t][g] * t_{t,i}.  Thread (stream, quad) owns
  // coordinates 4 quad .. 4 quad + 3 (one coset group) for tokens t = stream mod 8.
  // Code k of the quad sits at bits BV*(4 quad + k) of the token's words;
  // 2q = 2 (2^22 + j) - 2^23 - (2^b - 2) - h, with 2^22 + j built by one LOP3
  // (the code at mantissa bit 1: the fp32 spacing at 2^22 is 1/2) and every
  // constant an integer below 2^24: exact.
  {
    const int quad = lane, strm = warp;
    const int bitpos = BV * 4 * quad;
    const int wi = bitpos >> 5, off = bitpos & 31;
    const int wn = wi + 1 < 4 * BV ? wi + 1 : wi;
    const int grp = quad >> 1;
    constexpr float kBase = -8388608.0f - static_cast<float>((1 << BV) - 2);
    constexpr uint32_t kMask2 = ((1u << BV) - 1u) << 1;
    // heads in pairs as fp32x2 lanes (GT = 1: one lane unused)
    constexpr int GP = (GT + 1) / 2;
    float2 acc[GP][4];
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[g][k] = make_float2(0.f, 0.f);
    for (int t = strm; t < nt; t += kStreams) {
      const uint32_t* ww = vw + t * (4 * BV);
      const uint32_t x =
          (off + 4 * BV <= 32 ? (ww[wi] >> off) : __funnelshift_r(ww[wi], ww[wn], off)) << 1;
      const float kg = ((vmeta[t] >> grp) & 1u) ? kBase - 1.0f : kBase;
      float2 wt[GP];
      if (GT >= 4) {
#pragma unroll
        for (int g = 0; g < GP; g += 2) {
          const float4 w4 = *reinterpret_cast<const float4*>(sc + t * GT + 2 * g);
          wt[g] = make_float2(w4.x, w4.y);
          wt[g + 1 < GP ? g + 1 : g] = make_float2(w4.z, w4.w);
        }
      } else if (GT == 2) {
        wt[0] = *reinterpret_cast<const float2*>(sc + t * GT);
      } else {
        wt[0] = make_float2(sc[t * GT], 0.f);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float J = __uint_as_float(((x >> (BV * k)) & kMask2) | 0x4A800000u);
        const float tq = __fmaf_rn(J, 2.0f, kg);
#pragma unroll
        for (int g = 0; g < GP; ++g) acc[g][k] = fma2(wt[g], make_float2(tq, tq), acc[g][k]);
      }
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      *reinterpret_cast<float4*>(accs + (strm * GT + 2 * g) * kD + 4 * quad) =
          make_float4(acc[g][0].x, acc[g][1].x, acc[g][2].x, acc[g][3].x);
      if (2 * g + 1 < GT)
        *reinterpret_cast<float4*>(accs + (strm * GT + 2 * g + 1) * kD + 4 * quad) =
            make_float4(acc[g][0].y, acc[g][1].y, acc[g][2].y, acc[g][3].y);
    }
  }
  __syncthreads();
  // sum the streams in a fixed order and write the chunk's (m, l, a)
  float* out = a.part + (uh * a.nsplit + split) * GT * kPartFloats;
  for (int e = tid; e < GT * kD; e += kAttThreads) {
    const int g = e / kD, i = e % kD;
    float sum = 0.f;
#pragma unroll
    for (int st = 0; st < kStreams; ++st) sum += accs[(st * GT + g) * kD + i];
    out[g * kPartFloats + 2 + i] = sum;
  }
  if (tid < 2 * GT) out[(tid >> 1) * kPartFloats + (tid & 1)] = red[tid];
}

// One warp per (unit, query head): merge the chunks, o = H A / L, lse = M + log L.
// Lane l holds coordinates l, l+32, l+64, l+96: Hadamard stages 32 and 64 in
// the lane, stages 1..16 across lanes.
__global__ void __launch_bounds__(32) attend_combine_kernel(const AttendArgs a, float* out,
                                                            float* lse) {
  const int lane = threadIdx.x;
  const int64_t uj = blockIdx.x;  // u * (heads * G) + j
  const int Hq = a.heads * a.G;
  const int64_t u = uj / Hq;
  const int j = static_cast<int>(uj % Hq);
  const int h = j / a.G, g = j % a.G;
  const float* base = a.part + ((u * a.heads + h) * a.nsplit) * a.GT * kPartFloats + g * kPartFloats;
  const int64_t sstride = static_cast<int64_t>(a.GT) * kPartFloats;
  float M = -INFINITY;
#pragma unroll 8
  for (int64_t s = 0; s < a.nsplit; ++s) M = fmaxf(M, base[s * sstride]);
  float L = 0.f, A[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int64_t s = 0; s < a.nsplit; ++s) {
    const float* p = base + s * sstride;
    const float f = __expf(p[0] - M);
    L = __fmaf_rn(f, p[1], L);
#pragma unroll
    for (int r = 0; r < 4; ++r) A[r] = __fmaf_rn(f, p[2 + lane + 32 * r], A[r]);
  }
  // unnormalised Sylvester transform: stages 1..16 across lanes, 32 and 64 in the lane
#pragma unroll
  for (int st = 1; st < 32; st <<= 1) {
    const bool upper = lane & st;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float o = __shfl_xor_sync(0xffffffffu, A[r], st);
      A[r] = upper ? o - A[r] : A[r] + o;
    }
  }
  {
    const float x0 = A[0] + A[1], x1 = A[0] - A[1], x2 = A[2] + A[3], x3 = A[2] - A[3];
    A[0] = x0 + x2;
    A[2] = x0 - x2;
    A[1] = x1 + x3;
    A[3] = x1 - x3;
  }
  const float invL = 1.0f / L;
  float* o = out + uj * kD;
#pragma unroll
  for (int r = 0; r < 4; ++r) o[lane + 32 * r] = A[r] * invL;
  if (lse && lane == 0) lse[uj] = M + __logf(L);
}

static int group_tile(int G) { return G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8)); }

size_t attend_workspace_floats(int units, int heads, int G, int64_t n) {
  const int64_t nsplit = (n + kChunk - 1) / kChunk;
  return static_cast<size_t>(units) * heads * nsplit * group_tile(G) * kPartFloats;
}

template <int BK, int BV, int GT>
static cudaError_t launch_partial_gt(const AttendArgs& a, int64_t grid, cudaStream_t stream) {
  constexpr int smem = AttSmem<BV, GT>::bytes;
  cudaError_t err = cudaFuncSetAttribute(attend_partial_kernel<BK, BV, GT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  attend_partial_kernel<BK, BV, GT><<<static_cast<unsigned>(grid), kAttThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int BK, int BV>
static cudaError_t launch_partial(const AttendArgs& a, int64_t grid, cudaStream_t stream) {
  switch (a.GT) {
    case 1: return launch_partial_gt<BK, BV, 1>(a, grid, stream);
    case 2: return launch_partial_gt<BK, BV, 2>(a, grid, stream);
    case 4: return launch_partial_gt<BK, BV, 4>(a, grid, stream);
    default: return launch_partial_gt<BK, BV, 8>(a, grid, stream);
  }
}

cudaError_t launch_attend(const AttendLaunch& L, cudaStream_t stream) {
  AttendArgs a{};
  a.q = L.q;
  a.kc = L.k_in.codes;
  a.km = L.k_in.meta;
  a.vc = L.v_in.codes;
  a.vm = L.v_in.meta;
  a.kpu = L.k_in.unit_stride;
  a.kph = L.k_in.head_stride;
  a.vpu = L.v_in.unit_stride;
  a.vph = L.v_in.head_stride;
  a.heads = L.heads;
  a.G = L.G;
  a.GT = group_tile(L.G);
  a.n = L.n;
  a.slot0 = L.slot0;
  a.pos = L.positions;
  a.pos_stride = L.pos_stride;
  a.pos_base = L.pos_base;
  a.tab = reinterpret_cast<const float2*>(L.rope_tab);
  a.n_a = (L.rope_max_pos + 255) / 256;
  a.scale = L.scale;
  a.nsplit = (L.n + kChunk - 1) / kChunk;
  a.part = static_cast<float*>(L.ws);
  const int64_t grid = static_cast<int64_t>(L.units) * L.heads * a.nsplit;
  const int bk = L.k_in.bits, bv = L.v_in.bits;
  cudaError_t err;
  if (bk == 3 && bv == 2) err = launch_partial<3, 2>(a, grid, stream);
  else if (bk == 3 && bv == 3) err = launch_partial<3, 3>(a, grid, stream);
  else if (bk == 2 && bv == 2) err = launch_partial<2, 2>(a, grid, stream);
  else err = launch_partial<2, 3>(a, grid, stream);
  if (err != cudaSuccess) return err;
  attend_combine_kernel<<<static_cast<unsigned>(static_cast<int64_t>(L.units) * L.heads * L.G), 32,
                          0, stream>>>(a, L.out, L.lse);
  return cudaGetLastError();
}

}  // namespace nq
