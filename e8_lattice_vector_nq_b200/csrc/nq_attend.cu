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
// (unit, group of up to 8 KV heads, chunk of tokens), one warp per KV head
// with all G query heads of that KV head, and walks the chunk in tiles of 16
// tokens.  All heads of a unit share the tokens' positions, so:
//   - the RoPE table rows of a tile are staged two tiles ahead (cp.async) and
//     combined once into a cos/sin table that every warp of the CTA reads;
//   - keys: two lanes per token rebuild the key half by half exactly as the
//     decode kernel does (unpack, Hadamard, kappa, RoPE from the shared
//     table) and dot it with the warp's queries, held in shared memory as
//     (q_i, q_{i+64}) pairs;
//   - online softmax per query head: running max m and sum l, the sums
//     rescaled by exp(m_old - m_new) when the max grows; token weights
//     w_t = exp(s_t - m) * kappa_t;
//   - values stay in the code domain: since v_t = kappa_t * H t_t (H the
//     unnormalised Hadamard matrix, t_t the 2q integers), the warp
//     accumulates a = sum_t w_t t_t, lane l owning coordinates 4l..4l+3 (half
//     a coset group), from value codes staged one tile ahead; H is applied
//     once per query head when the chunks are merged (o = H A / L).
// One CTA barrier per tile (the shared table); everything else is per warp.
// The combine kernel merges the chunks' (m, l, a) with the usual rescaling,
// applies the 128-point Hadamard transform across one warp and writes o, lse.
#include "nq_codec_math.cuh"
#include "nq_internal.h"

namespace nq {

constexpr int kPartFloats = 2 + kD;  // m, l, a[128]
constexpr int kMinChunk = 64;        // tokens per CTA at least
// Splits are chosen so that a launch has about this many CTAs: four waves of
// two 256-thread CTAs per SM on 148 SMs.
constexpr int64_t kTargetCtas = 8 * 148;

struct AttendArgs {
  const float* q;  // [units][heads * G][128]
  const uint32_t *kc, *km, *vc, *vm;
  int64_t kpu, kph, vpu, vph;  // vector strides of the packed stores
  int heads, hg, ngroups;      // KV heads, KV heads per CTA, CTAs per (unit, split)
  int G, GT;  // GT: query heads computed per warp (G rounded up to 1, 2, 4 or 8)
  int64_t n, slot0;
  const int32_t* pos;
  int64_t pos_stride, pos_base;
  const float2* tab;
  int64_t n_a;
  float scale;
  int64_t chunk, nsplit;  // tokens per CTA (a multiple of 16), chunks per (unit, head)
  float* part;            // [units][heads][nsplit][GT][kPartFloats]
};

// Dynamic shared memory of the partial kernel: per CTA the raw RoPE rows and
// the cos/sin tables of two tiles; per warp its queries, the key and value
// codes of two tiles, and the current tile's weights and value meta.  Key
// codes sit at a stride of 48 bytes per token (3 bits: exactly the codes;
// 2 bits: padded), so the 16-byte reads of 8 consecutive tokens hit
// distinct bank groups.
constexpr int kKStride = 48;
template <int BV, int GT>
struct AttSmem {
  static constexpr int kRaw = 2 * kRawBytes;
  static constexpr int kCs = 2 * kCsBytes;
  static constexpr int kQ = GT * 64 * 8;               // float2 qp[GT][64]
  static constexpr int kKc = 2 * kSlots * kKStride;    // key codes [2][16][48 bytes]
  static constexpr int kVc = 2 * kSlots * 4 * BV * 4;  // uint32 codes[2][16][4 BV]
  static constexpr int kW = kSlots * GT * 4;           // float w[16][GT]
  static constexpr int kVm = kSlots * 4;               // uint32 vmeta[16]
  static constexpr int kWarp = kQ + kKc + kVc + kW + kVm;
  static constexpr int bytes(int warps) { return kRaw + kCs + warps * kWarp; }
};

template <int BK, int BV, int GT>
__global__ void __launch_bounds__(256, GT == 8 ? 1 : 2) attend_partial_kernel(const AttendArgs a) {
  extern __shared__ __align__(16) unsigned char att_smem[];
  using S = AttSmem<BV, GT>;
  constexpr int GP = (GT + 1) / 2;  // query heads in fp32x2 pairs (GT = 1: one lane unused)
  constexpr int kVWords = 4 * BV;   // value code words per token
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  const int slot_l = lane & 15, half = lane >> 4;

  const int64_t split = blockIdx.x % a.nsplit;
  const int64_t ug = blockIdx.x / a.nsplit;
  const int h = static_cast<int>(ug % a.ngroups) * a.hg + warp;
  const int64_t u = ug / a.ngroups;
  const int64_t t0 = split * a.chunk;
  const int nt = static_cast<int>(min64(a.chunk, a.n - t0));  // >= 1
  const int ntiles = (nt + kSlots - 1) / kSlots;

  const uint32_t raw0 = smem_u32(att_smem);
  unsigned char* cs0 = att_smem + S::kRaw;
  unsigned char* wsm = att_smem + S::kRaw + S::kCs + warp * S::kWarp;
  float2(*qp)[64] = reinterpret_cast<float2(*)[64]>(wsm);
  const uint32_t kcb = smem_u32(wsm + S::kQ);
  uint32_t* vcb = reinterpret_cast<uint32_t*>(wsm + S::kQ + S::kKc);
  float* wts = reinterpret_cast<float*>(wsm + S::kQ + S::kKc + S::kVc);
  uint32_t* vmb = reinterpret_cast<uint32_t*>(wsm + S::kQ + S::kKc + S::kVc + S::kW);
  auto raw_of = [&](int k) { return raw0 + static_cast<uint32_t>(k & 1) * kRawBytes; };
  auto cs_of = [&](int k) { return reinterpret_cast<float4*>(cs0 + (k & 1) * kCsBytes); };

  // position minus pos_base of this lane's token in tile k, -1 past the chunk
  // (out-of-contract negative positions are taken as 0)
  auto src_of = [&](int k) -> int32_t {
    const int tt = k * kSlots + slot_l;
    if (tt >= nt) return -1;
    const int32_t p =
        a.pos ? __ldg(a.pos + u * a.pos_stride + t0 + tt) : static_cast<int32_t>(t0 + tt);
    return p < 0 ? 0 : p;
  };
  const int64_t kv0 = u * a.kpu + h * a.kph + a.slot0 + t0;  // first key vector of the chunk
  const int64_t vv0 = u * a.vpu + h * a.vph + a.slot0 + t0;  // first value vector
  // key and value codes of tile k (its valid tokens) into the warp's buffers k & 1
  auto issue_codes = [&](int k) {
    const int nv = min(kSlots, nt - k * kSlots);
    const char* ks = reinterpret_cast<const char*>(a.kc + (kv0 + k * kSlots) * (4 * BK));
    const uint32_t kd = kcb + (k & 1) * (kSlots * kKStride);
    for (int c = lane; c < nv * BK; c += 32) {
      const int tok = c / BK;
      cp_async16(kd + tok * kKStride + (c - tok * BK) * 16, ks + c * 16);
    }
    const char* vs = reinterpret_cast<const char*>(a.vc + (vv0 + k * kSlots) * kVWords);
    const uint32_t vd = smem_u32(vcb + (k & 1) * (kSlots * kVWords));
    for (int c = lane; c < nv * BV; c += 32) cp_async16(vd + c * 16, vs + c * 16);
  };
  // key and value meta of this lane's token in tile k (zero past the chunk)
  uint32_t kmeta = 0, vmeta = 0;
  auto load_meta = [&](int k) {
    const int tt = k * kSlots + slot_l;
    kmeta = tt < nt ? __ldg(a.km + kv0 + tt) : 0u;
    vmeta = tt < nt ? __ldg(a.vm + vv0 + tt) : 0u;
  };

  // the warp's queries (heads G..GT-1 are zero)
  const float* qg = a.q + (u * a.heads + h) * static_cast<int64_t>(a.G) * kD;
  for (int e = lane; e < GT * 64; e += 32) {
    const int g = e >> 6, i = e & 63;
    qp[g][i] = g < a.G ? make_float2(__ldg(qg + g * kD + i), __ldg(qg + g * kD + i + 64))
                       : make_float2(0.f, 0.f);
  }

  // prologue: rows of tiles 0 and 1 and the value codes of tile 0 in flight,
  // the table of tile 0 combined
  int32_t src_pref = -1;
  issue_rope_rows(a.tab, a.n_a, a.pos_base, src_of(0), raw_of(0), warp, nwarps, lane);
  issue_codes(0);
  cp_async_commit();
  if (ntiles > 1)
    issue_rope_rows(a.tab, a.n_a, a.pos_base, src_of(1), raw_of(1), warp, nwarps, lane);
  cp_async_commit();
  if (ntiles > 2) src_pref = src_of(2);
  load_meta(0);
  cp_async_wait<1>();
  __syncthreads();
  combine_rope_rows(raw_of(0), cs_of(0), tid, nthreads);

  // running max and sum of query head g live in lane g
  float m_lane = -INFINITY, l_lane = 0.f;
  float2 acc[GP][4];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[g][c] = make_float2(0.f, 0.f);

  // Lane l's value coordinates 4l..4l+3: codes at bits BV*4l.. of the token's
  // words, coset group l/2.  2q = 2 (2^22 + j) - 2^23 - (2^b - 2) - h, with
  // 2^22 + j built by one LOP3 (the code at mantissa bit 1: the fp32 spacing
  // at 2^22 is 1/2) and every constant an integer below 2^24: exact.
  const int bitpos = BV * 4 * lane;
  const int wi = bitpos >> 5, off = bitpos & 31;
  const int wn = wi + 1 < kVWords ? wi + 1 : wi;
  const int vgrp = lane >> 1;
  constexpr float kBase = -8388608.0f - static_cast<float>((1 << BV) - 2);
  constexpr uint32_t kMask2 = ((1u << BV) - 1u) << 1;

  for (int k = 0; k < ntiles; ++k) {
    // rows of tile k+1 and codes of tile k landed (everyone's), table k
    // combined, tile k-1 done by every warp
    cp_async_wait<0>();
    __syncthreads();
    if (k + 2 < ntiles)
      issue_rope_rows(a.tab, a.n_a, a.pos_base, src_pref, raw_of(k), warp, nwarps, lane);
    if (k + 1 < ntiles) issue_codes(k + 1);
    cp_async_commit();
    if (k + 3 < ntiles) src_pref = src_of(k + 3);
    if (k + 1 < ntiles) combine_rope_rows(raw_of(k + 1), cs_of(k + 1), tid, nthreads);

    const bool valid = k * kSlots + slot_l < nt;
    const uint32_t kmc = kmeta, vmc = vmeta;
    if (k + 1 < ntiles) load_meta(k + 1);

    // ---- keys and scores (a token past the chunk has kappa 0 and score -inf)
    float sc[GT];
    {
      // only this half's code words are read, and each is placed in both
      // halves' positions, so that every index into wc is a constant (a
      // runtime index would put the array in local memory)
      uint32_t wc[4 * BK];
      const uint32_t kt = kcb + (k & 1) * (kSlots * kKStride) + slot_l * kKStride;
#pragma unroll
      for (int c = 0; c < BK; ++c) {
        const uint32_t wa = lds32(kt + 4 * (BK * half + c));
        const uint32_t wb = lds32(kt + 4 * (2 * BK + BK * half + c));
        wc[c] = wa;
        wc[BK + c] = wa;
        wc[2 * BK + c] = wb;
        wc[3 * BK + c] = wb;
      }
      float2 v[32];
      reconstruct_half<BK>(wc, kmc, half, v);
      rope_half(v, smem_u32(cs_of(k)) + (16 * half * kSlots + slot_l) * 16);
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
        sc[g] = valid ? a.scale * d : -INFINITY;
      }
    }

    // ---- online softmax over the tile (lanes l and l+16 hold the same token)
    const float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(vmc >> 16)));
    const float kappa = __fmul_rn(__fmul_rn(sig, 0.5f), __uint_as_float(kCBits));
    float wt[GT], al[GT];
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      float mt = sc[g];
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
      const float mo = __shfl_sync(0xffffffffu, m_lane, g);
      const float mn = fmaxf(mo, mt);  // finite: every tile holds a valid token
      al[g] = __expf(mo - mn);         // 0 on the first tile
      const float p = valid ? __expf(sc[g] - mn) : 0.f;
      float ps = p;
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      const float lo = __shfl_sync(0xffffffffu, l_lane, g);
      if (lane == g) {
        m_lane = mn;
        l_lane = __fmaf_rn(lo, al[g], ps);
      }
      wt[g] = valid ? p * kappa : 0.f;
    }
    if (half == 0) {
      float* wd = wts + slot_l * GT;
      if (GT >= 4) {
#pragma unroll
        for (int g = 0; g < GT; g += 4)
          *reinterpret_cast<float4*>(wd + g) = make_float4(wt[g], wt[g + 1], wt[g + 2], wt[g + 3]);
      } else if (GT == 2) {
        *reinterpret_cast<float2*>(wd) = make_float2(wt[0], wt[1]);
      } else {
        wd[0] = wt[0];
      }
      vmb[slot_l] = vmc;
    }
    __syncwarp();
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float2 a2 = make_float2(al[2 * g], al[2 * g + 1 < GT ? 2 * g + 1 : 2 * g]);
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[g][c] = mul2(acc[g][c], a2);
    }

    // ---- values: a[g][4l + c] += w[t][g] * t_{t, 4l + c}; tokens past the
    // chunk carry weight 0 (their staged codes are stale but decode to finite values)
    const uint32_t* vcur = vcb + (k & 1) * (kSlots * kVWords);
#pragma unroll
    for (int t = 0; t < kSlots; ++t) {
      const uint32_t* ww = vcur + t * kVWords;
      const uint32_t x =
          (off + 4 * BV <= 32 ? (ww[wi] >> off) : __funnelshift_r(ww[wi], ww[wn], off)) << 1;
      const float kg = ((vmb[t] >> vgrp) & 1u) ? kBase - 1.0f : kBase;
      float2 wp[GP];
      if (GT >= 4) {
#pragma unroll
        for (int g = 0; g < GP; g += 2) {
          const float4 w4 = *reinterpret_cast<const float4*>(wts + t * GT + 2 * g);
          wp[g] = make_float2(w4.x, w4.y);
          wp[g + 1 < GP ? g + 1 : g] = make_float2(w4.z, w4.w);
        }
      } else if (GT == 2) {
        wp[0] = *reinterpret_cast<const float2*>(wts + t * GT);
      } else {
        wp[0] = make_float2(wts[t], 0.f);
      }
#pragma unroll
      for (int cp = 0; cp < 2; ++cp) {
        const float J0 = __uint_as_float(((x >> (BV * 2 * cp)) & kMask2) | 0x4A800000u);
        const float J1 = __uint_as_float(((x >> (BV * (2 * cp + 1))) & kMask2) | 0x4A800000u);
        const float2 tq = fma2(make_float2(J0, J1), make_float2(2.0f, 2.0f), make_float2(kg, kg));
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          acc[g][2 * cp] = fma2(wp[g], make_float2(tq.x, tq.x), acc[g][2 * cp]);
          acc[g][2 * cp + 1] = fma2(wp[g], make_float2(tq.y, tq.y), acc[g][2 * cp + 1]);
        }
      }
    }
  }

  // the chunk's (m, l, a) for each query head of the warp
  float* out = a.part + ((u * a.heads + h) * a.nsplit + split) * (GT * kPartFloats);
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    float* o0 = out + (2 * g) * kPartFloats + 2 + 4 * lane;
    *reinterpret_cast<float2*>(o0) = make_float2(acc[g][0].x, acc[g][1].x);
    *reinterpret_cast<float2*>(o0 + 2) = make_float2(acc[g][2].x, acc[g][3].x);
    if (2 * g + 1 < GT) {
      float* o1 = o0 + kPartFloats;
      *reinterpret_cast<float2*>(o1) = make_float2(acc[g][0].y, acc[g][1].y);
      *reinterpret_cast<float2*>(o1 + 2) = make_float2(acc[g][2].y, acc[g][3].y);
    }
  }
  if (lane < GT) {
    out[lane * kPartFloats] = m_lane;
    out[lane * kPartFloats + 1] = l_lane;
  }
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

// Tokens per CTA: about kTargetCtas CTAs per launch, a multiple of the tile,
// at least kMinChunk.
static int64_t attend_chunk(int units, int heads, int64_t n) {
  int64_t per_split = static_cast<int64_t>(units) * (heads / pick_head_group(heads));
  if (per_split < 1) per_split = 1;
  const int64_t want = (kTargetCtas + per_split - 1) / per_split;
  int64_t chunk = (n + want - 1) / want;
  chunk = (chunk + kSlots - 1) / kSlots * kSlots;
  return chunk < kMinChunk ? kMinChunk : chunk;
}

static int64_t attend_nsplit(int units, int heads, int64_t n) {
  const int64_t c = attend_chunk(units, heads, n);
  return (n + c - 1) / c;
}

size_t attend_workspace_floats(int units, int heads, int G, int64_t n) {
  return static_cast<size_t>(units) * heads * attend_nsplit(units, heads, n) * group_tile(G) *
         kPartFloats;
}

int64_t attend_ctas(int units, int heads, int64_t n) {
  return static_cast<int64_t>(units) * (heads / pick_head_group(heads)) *
         attend_nsplit(units, heads, n);
}

template <int BK, int BV, int GT>
static cudaError_t launch_partial_gt(const AttendArgs& a, int64_t grid, cudaStream_t stream) {
  const int smem = AttSmem<BV, GT>::bytes(a.hg);
  cudaError_t err = cudaFuncSetAttribute(attend_partial_kernel<BK, BV, GT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  attend_partial_kernel<BK, BV, GT><<<static_cast<unsigned>(grid), 32 * a.hg, smem, stream>>>(a);
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
  a.hg = pick_head_group(L.heads);
  a.ngroups = L.heads / a.hg;
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
  a.chunk = attend_chunk(L.units, L.heads, L.n);
  a.nsplit = (L.n + a.chunk - 1) / a.chunk;
  a.part = static_cast<float*>(L.ws);
  const int64_t grid = static_cast<int64_t>(L.units) * a.ngroups * a.nsplit;
  if (grid >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
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
