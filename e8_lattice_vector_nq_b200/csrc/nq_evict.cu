// nq_evict.cu -- key-key proxy scoring and token selection for sm_100a.
//
// Method: NexusQuant ("NexusQuant: training-free 10-33x KV cache
// compression", zingnex.cn, sections "Token eviction" and "Implementation
// details": a fast key-key proxy score; always keep BOS and a recent sliding
// window, drop the low scorers; "Como comprimir o KV cache...", dev.to,
// "Como funciona", steps 1-2: rank tokens by a cross-head inner product).
//
//   window_mean_kernel: m[u][h][d] = fp32(fp64 sum of the last W keys / W)
//   score_kernel:       scores[u][t] = sum_h sum_d K[u][h][t][d] * m[u][h][d]
//                       in fp64 (one coalesced pass over K)
//   select_kernel:      per unit (one cluster of 4 CTAs sharing histograms
//                       through distributed shared memory), an MSD radix
//                       select (11-bit digits, after the prefix that every
//                       middle key shares) of the
//                       (score desc, position asc) threshold on
//                       order-preserving 64-bit keys; once at most 8192 keys
//                       share the prefix they move to shared memory and the
//                       remaining digits are read from there; then an
//                       ordered compaction with warp ballots.
#include <cooperative_groups.h>

#include <cuda.h>

#include <mutex>

#include "nq_internal.h"

namespace nq {
namespace cg = cooperative_groups;

// ----------------------------------------------------------- window mean
__global__ void window_mean_kernel(const uint16_t* __restrict__ K, nq_kv_strides ks, int heads,
                                   int64_t T, int W, float* __restrict__ mean) {
  const int u = blockIdx.x / heads, h = blockIdx.x % heads, d = threadIdx.x;
  const uint16_t* p = K + u * ks.unit + h * ks.head + d;
  double S = 0.0;  // every partial sum of bf16 values is exact in fp64 here
  for (int64_t t = T - W; t < T; ++t) S += static_cast<double>(bf16lo(__ldg(p + t * ks.token)));
  mean[(static_cast<int64_t>(u) * heads + h) * kD + d] = static_cast<float>(S / W);
}

// ---------------------------------------------------------------- score
constexpr int kScoreTok = 128;     // tokens per CTA
constexpr int kScoreThreads = 256;

// 4 CTAs (32 warps) per SM: more 16-byte loads in flight per SM (a few
// registers spill to L1).
// SHARE: fewer heads than warps, so wph = floor(8 / heads) (2, 4 or 8) warps
// share a head, each taking 1 / wph of the tile's tokens and every warp loads;
// otherwise one warp per head.
template <bool SHARE>
__global__ void __launch_bounds__(kScoreThreads, 4) score_kernel(const uint16_t* __restrict__ K,
                                                              nq_kv_strides ks, int heads,
                                                              int64_t T,
                                                              const float* __restrict__ mean,
                                                              double* __restrict__ scores) {
  extern __shared__ double part[];  // [heads][kScoreTok]
  const int64_t tiles = (T + kScoreTok - 1) / kScoreTok;
  const int u = static_cast<int>(blockIdx.x / tiles);
  const int64_t t0 = (blockIdx.x % tiles) * kScoreTok;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, chunk = lane & 15;
  const int nwarps = kScoreThreads / 32;
  constexpr int kPairs = kScoreTok / 2;  // iterations of two tokens per warp and head
  const int wph = SHARE ? nwarps / heads : 1;
  const int span = SHARE ? kPairs / wph : kPairs;

  for (int hw = warp; hw < heads * wph; hw += nwarps) {
    const int h = SHARE ? hw % heads : hw, it_begin = SHARE ? (hw / heads) * span : 0;
    const float* mh = mean + (static_cast<int64_t>(u) * heads + h) * kD + chunk * 8;
    double m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = static_cast<double>(__ldg(mh + i));
    const uint16_t* base = K + u * ks.unit + h * ks.head + chunk * 8;
    // 8 independent 16-byte loads per lane are in flight before any math
    constexpr int kBatch = 8;
#pragma unroll 1
    for (int it0 = it_begin; it0 < it_begin + span; it0 += kBatch) {
      uint4 q[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int64_t t = t0 + 2 * (it0 + b) + half;
        q[b] = t < T ? __ldg(reinterpret_cast<const uint4*>(base + t * ks.token))
                     : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const uint32_t w[4] = {q[b].x, q[b].y, q[b].z, q[b].w};
        double acc = 0.0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc = fma(static_cast<double>(bf16lo(w[k])), m[2 * k], acc);
          acc = fma(static_cast<double>(bf16hi(w[k])), m[2 * k + 1], acc);
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (chunk == 0) part[h * kScoreTok + 2 * (it0 + b) + half] = acc;
      }
    }
  }
  __syncthreads();
  for (int tl = threadIdx.x; tl < kScoreTok; tl += blockDim.x) {
    const int64_t t = t0 + tl;
    if (t < T) {
      double s = 0.0;
      for (int h = 0; h < heads; ++h) s += part[h * kScoreTok + tl];
      scores[static_cast<int64_t>(u) * T + t] = s;
    }
  }
}

// --------------------------------------------------------------- select
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;

// Order-preserving map of a finite double to uint64 (larger score -> larger
// key); -0 is folded onto +0 so that the two compare equal.
__device__ __forceinline__ uint64_t score_key(double x) {
  if (x == 0.0) x = 0.0;
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ void block_exclusive_scan32(int* vals /*[32] smem*/) {
  // small serial scan by one thread: 32 warps
  if (threadIdx.x == 0) {
    int run = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      const int c = vals[w];
      vals[w] = run;
      run += c;
    }
  }
  __syncthreads();
}

constexpr int kDigitBits = 11;
constexpr int kUnroll = 8;  // independent score loads in flight per thread
constexpr int kBins = 1 << kDigitBits;  // 2 bins per thread
constexpr int kCandCap = 8192;          // candidate keys kept in shared memory
constexpr int kSelCluster = 4;          // CTAs (one cluster) per unit

// One unit per cluster of kSelCluster CTAs (thread-block cluster, distributed
// shared memory).  CTA r owns the r-th contiguous slice of the middle range for
// the radix passes and the r-th contiguous segment of positions for the
// ordered compaction.  Every radix pass builds a local histogram, then each
// CTA sums the cluster's histograms for its two bins through DSMEM and runs
// the same descending scan, so all CTAs derive the same prefix and rank; the
// compaction offsets are exclusive sums over the lower-ranked CTAs' counts.
// Every CTA of a cluster executes the same sequence of cluster barriers.
__global__ void __launch_bounds__(kSelThreads) select_kernel(const double* __restrict__ scores,
                                                             int64_t T, int W, int64_t n_kept,
                                                             int32_t* __restrict__ kept,
                                                             int64_t kept_stride) {
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  extern __shared__ uint32_t flagbits[];  // this CTA's segment flag words, then candidate keys
  __shared__ unsigned int hist[kBins];
  __shared__ uint64_t s_min[kSelWarps], s_max[kSelWarps];
  __shared__ uint64_t c_minmax[2];        // this CTA's min and max key (read by the cluster)
  __shared__ unsigned int s_wsum[kSelWarps];
  __shared__ uint64_t s_prefix;
  __shared__ int64_t s_k;
  __shared__ int64_t s_eq;
  __shared__ int warp_cnt[kSelWarps];
  __shared__ long long c_count[2];        // this CTA's tie and kept counts (read by the cluster)
  __shared__ unsigned int s_ncand;

  const int u = blockIdx.x / kSelCluster;
  const double* s = scores + static_cast<int64_t>(u) * T;
  int32_t* out = kept + static_cast<int64_t>(u) * kept_stride;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this CTA's segment of positions, a multiple of 32 wide
  const int64_t seg_cta = ((T + kSelCluster - 1) / kSelCluster + 31) / 32 * 32;
  const int64_t S0 = min64(T, rank * seg_cta), S1 = min64(T, S0 + seg_cta);
  uint64_t* cand = reinterpret_cast<uint64_t*>(flagbits + ((seg_cta + 63) / 64) * 2);

  if (n_kept >= T) {  // the same branch in every CTA: no barrier pending
    for (int64_t t = S0 + tid; t < S1; t += blockDim.x) out[t] = static_cast<int32_t>(t);
    return;
  }
  const int64_t lo = 1, hi = T - W;  // middle range [lo, hi)
  const int64_t n_mid = n_kept - 1 - W;
  // this CTA's slice of the middle range
  const int64_t sl = (hi - lo + kSelCluster - 1) / kSelCluster;
  const int64_t A0 = min64(hi, lo + rank * sl), A1 = min64(hi, A0 + sl);

  // --- radix select: the n_mid-th largest key among the middle tokens
  uint64_t prefix = 0;
  int64_t k = n_mid;
  int64_t n_eq = hi - lo;  // keys equal to the threshold (all, until a radix pass splits them)
  if (n_mid > 0) {
    // every candidate key lies in [kmin, kmax], so they share its common prefix
    uint64_t kmin = ~0ull, kmax = 0ull;
    for (int64_t t0 = A0 + tid; t0 < A1; t0 += kUnroll * blockDim.x) {
      double v[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int64_t t = t0 + j * blockDim.x;
        v[j] = t < A1 ? __ldg(s + t) : 0.0;
      }
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        if (t0 + j * blockDim.x < A1) {
          const uint64_t key = score_key(v[j]);
          kmin = key < kmin ? key : kmin;
          kmax = key > kmax ? key : kmax;
        }
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const uint64_t a = __shfl_xor_sync(0xffffffffu, kmin, o);
      const uint64_t b = __shfl_xor_sync(0xffffffffu, kmax, o);
      kmin = a < kmin ? a : kmin;
      kmax = b > kmax ? b : kmax;
    }
    if (lane == 0) {
      s_min[warp] = kmin;
      s_max[warp] = kmax;
    }
    __syncthreads();
    if (tid == 0) {
      uint64_t mn = ~0ull, mx = 0ull;
      for (int w = 0; w < kSelWarps; ++w) {
        mn = s_min[w] < mn ? s_min[w] : mn;
        mx = s_max[w] > mx ? s_max[w] : mx;
      }
      c_minmax[0] = mn;
      c_minmax[1] = mx;
    }
    cl.sync();  // every CTA's min/max published
    uint64_t mn = ~0ull, mx = 0ull;
    for (int r = 0; r < kSelCluster; ++r) {
      const uint64_t* mm = cl.map_shared_rank(c_minmax, r);
      mn = mm[0] < mn ? mm[0] : mn;
      mx = mm[1] > mx ? mm[1] : mx;
    }
    const uint64_t diff = mn ^ mx;
    int rem = diff ? 64 - __clzll(static_cast<long long>(diff)) : 0;  // bits still undecided
    prefix = mn & (rem == 64 ? 0ull : ~((1ull << rem) - 1ull));
    int64_t ncand = -1;  // >= 0 once this CTA's candidates sit in cand[]
    while (rem > 0) {
      const int width = rem < kDigitBits ? rem : kDigitBits;
      const int shift = rem - width;
      const uint64_t pmask = rem == 64 ? 0ull : ~((1ull << rem) - 1ull);
      for (int i = tid; i < kBins; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      if (ncand >= 0) {
        for (int64_t i = tid; i < ncand; i += blockDim.x) {
          const uint64_t key = cand[i];
          if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & ((1u << width) - 1u)], 1u);
        }
      } else {
        for (int64_t t0 = A0 + tid; t0 < A1; t0 += kUnroll * blockDim.x) {
          double v[kUnroll];
#pragma unroll
          for (int j = 0; j < kUnroll; ++j) {
            const int64_t t = t0 + j * blockDim.x;
            v[j] = t < A1 ? __ldg(s + t) : 0.0;
          }
#pragma unroll
          for (int j = 0; j < kUnroll; ++j) {
            const uint64_t key = score_key(v[j]);
            const bool in = t0 + j * blockDim.x < A1 && (key & pmask) == prefix;
            if (in) atomicAdd(&hist[(key >> shift) & ((1u << width) - 1u)], 1u);
          }
        }
      }
      cl.sync();  // every CTA's histogram complete
      // descending bins: thread t owns bins 2047-2t and 2046-2t, summed over the cluster
      const int b0 = kBins - 1 - 2 * tid, b1 = b0 - 1;
      unsigned int c0 = 0, c1 = 0;
      for (int r = 0; r < kSelCluster; ++r) {
        const unsigned int* hr = cl.map_shared_rank(hist, r);
        c0 += hr[b0];
        c1 += hr[b1];
      }
      const unsigned int own = c0 + c1;
      unsigned int inc = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      if (lane == 31) s_wsum[warp] = inc;
      __syncthreads();
      if (warp == 0) {
        unsigned int w = s_wsum[lane], wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned int v = __shfl_up_sync(0xffffffffu, wi, o);
          if (lane >= o) wi += v;
        }
        s_wsum[lane] = wi - w;  // exclusive prefix of warp totals
      }
      __syncthreads();
      const int64_t before = static_cast<int64_t>(s_wsum[warp]) + (inc - own);  // keys in higher bins
      if (before < k && k <= before + own) {
        const bool first = k <= before + c0;
        const int d = first ? b0 : b1;
        s_k = k - before - (first ? 0 : c0);
        s_prefix = prefix | (static_cast<uint64_t>(d) << shift);
        s_eq = first ? c0 : c1;  // keys sharing the prefix so far (all of it after the last pass)
      }
      __syncthreads();
      prefix = s_prefix;
      k = s_k;
      n_eq = s_eq;
      rem = shift;
      cl.sync();  // every CTA has read the cluster's histograms: they may be cleared
      if (ncand < 0 && rem > 0 && n_eq <= kCandCap) {
        // few keys share the prefix now: copy this CTA's ones to shared memory
        // once, so the remaining passes read cand[] instead of every score
        if (tid == 0) s_ncand = 0;
        __syncthreads();
        const uint64_t pm = ~((1ull << rem) - 1ull);
        for (int64_t t0 = A0 + tid; t0 < A1; t0 += kUnroll * blockDim.x) {
          double v[kUnroll];
#pragma unroll
          for (int j = 0; j < kUnroll; ++j) {
            const int64_t t = t0 + j * blockDim.x;
            v[j] = t < A1 ? __ldg(s + t) : 0.0;
          }
#pragma unroll
          for (int j = 0; j < kUnroll; ++j) {
            const uint64_t key = score_key(v[j]);
            if (t0 + j * blockDim.x < A1 && (key & pm) == prefix) cand[atomicAdd(&s_ncand, 1u)] = key;
          }
        }
        __syncthreads();
        ncand = s_ncand;
      }
    }
  }
  const uint64_t kstar = prefix;  // threshold key
  const int64_t need_eq = k;      // how many keys equal to kstar are taken, lowest positions first

  // --- ordered compaction: each warp owns a contiguous part of the CTA's segment
  const int64_t seg = ((S1 - S0 + kSelWarps - 1) / kSelWarps + 31) / 32 * 32;
  const int64_t s0 = min64(S1, S0 + warp * seg), s1 = min64(S1, s0 + seg);

  // pass A (only when ties at the threshold must be split by position):
  // keys equal to the threshold, per warp
  const bool rank_ties = n_mid > 0 && need_eq < n_eq;
  int eq = 0;
  if (rank_ties) {
    for (int64_t b0 = s0; b0 < s1; b0 += 32 * kUnroll) {
      double v[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int64_t t = b0 + 32 * j + lane;
        v[j] = (t < s1 && t >= lo && t < hi) ? __ldg(s + t) : 0.0;
      }
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int64_t t = b0 + 32 * j + lane;
        const bool is_eq = t < s1 && t >= lo && t < hi && score_key(v[j]) == kstar;
        eq += __popc(__ballot_sync(0xffffffffu, is_eq));
      }
    }
  }
  if (lane == 0) warp_cnt[warp] = eq;
  __syncthreads();
  if (tid == 0) {
    long long tot = 0;
    for (int w = 0; w < kSelWarps; ++w) tot += warp_cnt[w];
    c_count[0] = tot;
  }
  block_exclusive_scan32(warp_cnt);
  cl.sync();  // every CTA's tie count published
  long long eq_base = 0;
  for (int r = 0; r < rank; ++r) eq_base += cl.map_shared_rank(c_count, r)[0];
  int64_t eq_rank = eq_base + warp_cnt[warp];
  __syncthreads();

  // pass B: keep flags (bitmask in smem) and per-warp kept counts
  int cnt = 0;
  for (int64_t b0 = s0; b0 < s1; b0 += 32 * kUnroll) {
    double v[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const int64_t t = b0 + 32 * j + lane;
      v[j] = (t < s1 && t >= lo && t < hi && n_mid > 0) ? __ldg(s + t) : 0.0;
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const int64_t b = b0 + 32 * j;
      if (b >= s1) break;
      const int64_t t = b + lane;
      const bool in_range = t < s1;
      const bool mid = in_range && t >= lo && t < hi;
      const uint64_t key = mid ? score_key(v[j]) : 0ull;
      const bool is_eq = mid && n_mid > 0 && key == kstar;
      const uint32_t eqb = __ballot_sync(0xffffffffu, is_eq);
      const int64_t r = eq_rank + __popc(eqb & ((1u << lane) - 1u));
      const bool keep = in_range && (!mid || (n_mid > 0 && (key > kstar ||
                                                           (is_eq && (!rank_ties || r < need_eq)))));
      const uint32_t kb = __ballot_sync(0xffffffffu, keep);
      eq_rank += __popc(eqb);
      if (lane == 0) flagbits[(b - S0) >> 5] = kb;
      cnt += __popc(kb);
    }
  }
  if (lane == 0) warp_cnt[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    long long tot = 0;
    for (int w = 0; w < kSelWarps; ++w) tot += warp_cnt[w];
    c_count[1] = tot;
  }
  block_exclusive_scan32(warp_cnt);
  cl.sync();  // every CTA's kept count published
  long long out_base = 0;
  for (int r = 0; r < rank; ++r) out_base += cl.map_shared_rank(c_count, r)[1];

  // pass C: write kept positions in ascending order
  int64_t o = out_base + warp_cnt[warp];
  for (int64_t b = s0; b < s1; b += 32) {
    const uint32_t kb = flagbits[(b - S0) >> 5];
    const int64_t idx = o + __popc(kb & ((1u << lane) - 1u));
    if (((kb >> lane) & 1u) && idx < n_kept) out[idx] = static_cast<int32_t>(b + lane);
    o += __popc(kb);
  }
  cl.sync();  // no CTA leaves while another may still read its shared memory
}

// ---------------------------------------------------------------- launch
cudaError_t launch_score(const void* K, nq_kv_strides ks, int units, int heads, int64_t T, int W,
                         double* scores, float* mean_ws, cudaStream_t stream) {
  window_mean_kernel<<<units * heads, kD, 0, stream>>>(static_cast<const uint16_t*>(K), ks, heads,
                                                       T, W, mean_ws);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t tiles = (T + kScoreTok - 1) / kScoreTok;
  const size_t smem = static_cast<size_t>(heads) * kScoreTok * sizeof(double);
  const bool share = heads < kScoreThreads / 32;
  const void* fn = share ? reinterpret_cast<const void*>(score_kernel<true>)
                         : reinterpret_cast<const void*>(score_kernel<false>);
  if (smem > 48 * 1024) {
    err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  if (share)
    score_kernel<true><<<static_cast<unsigned>(units * tiles), kScoreThreads, smem, stream>>>(
        static_cast<const uint16_t*>(K), ks, heads, T, mean_ws, scores);
  else
    score_kernel<false><<<static_cast<unsigned>(units * tiles), kScoreThreads, smem, stream>>>(
        static_cast<const uint16_t*>(K), ks, heads, T, mean_ws, scores);
  return cudaGetLastError();
}

// ------------------------------------------ score without any allocation
// Scratch for the window means of nq_score_static: a fixed array in the
// library's own device memory, present on every GPU that loads the library
// until the process exits.  All calls share it and it keeps the last call's
// contents; the window-mean kernel overwrites every entry a call reads, so
// nothing has to be cleared.  Two calls whose kernels overlap on a GPU race
// on it.
static __device__ __align__(256) float g_score_scratch[NQ_SCORE_STATIC_MAX_VECTORS * kD];

namespace {
constexpr int kMaxDevices = 256;
std::mutex g_scratch_mu;
float* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}
}  // namespace

// Device address of g_score_scratch on the current device.  Host code only
// sees a host-side stand-in under the array's name, so the address is looked
// up with the device current and cached per device, together with the
// context it belongs to: after a device reset (a new primary context, the
// module loaded again) the next call looks the address up again.
static cudaError_t score_scratch_address(float** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (!get_ctx) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!ctx || !g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
    // the lookup also makes the device's primary context current if none is
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_score_scratch);
    if (err != cudaSuccess) return err;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    g_scratch_addr[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

cudaError_t launch_score_static(const void* K, nq_kv_strides ks, int units, int heads, int64_t T,
                                int W, double* scores, cudaStream_t stream) {
  float* mean = nullptr;
  cudaError_t err = score_scratch_address(&mean);
  if (err != cudaSuccess) return err;
  return launch_score(K, ks, units, heads, T, W, scores, mean, stream);
}

cudaError_t launch_select(const double* scores, int units, int64_t T, int W, int evict_pct,
                          int64_t n_kept, int32_t* kept, int64_t kept_stride,
                          cudaStream_t stream) {
  (void)evict_pct;
  // this CTA's flag words rounded up to an even count (8-byte alignment of the
  // keys), then the keys
  const int64_t seg_cta = ((T + kSelCluster - 1) / kSelCluster + 31) / 32 * 32;
  const size_t smem = static_cast<size_t>((seg_cta + 63) / 64) * 2 * sizeof(uint32_t) +
                      static_cast<size_t>(kCandCap) * sizeof(uint64_t);
  cudaError_t err = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units) * kSelCluster);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSelCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, select_kernel, scores, T, W, n_kept, kept, kept_stride);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace nq
