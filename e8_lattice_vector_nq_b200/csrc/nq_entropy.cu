// nq_entropy.cu -- delta + entropy coding of the lattice indices of a packed
// store for sm_100a.  The NexusQuant pages close their pipeline with it:
// consecutive tokens give similar lattice indices, so the difference to the
// previous token is stored and the result compressed (zingnex.cn
// "Implementation details"; dev.to step 6, which uses zstd).  zstd is a
// third-party library; the coder here is range-variant asymmetric numeral
// systems (rANS, J. Duda, "Asymmetric numeral systems", 2013) with a static
// frequency table per (unit, head).
//
// Format (the decoder's contract):
//   streams  one per (unit, head, segment of kSeg tokens, coordinate c), in
//            that order, coordinate fastest; symbols d_t = (j_t - j_{t-1})
//            mod 2^b within the segment, d = j at its first token (d_t = j_t
//            when the difference is off); j_t is the b-bit code of c;
//   table    per (unit, head) over the symbols of all its streams:
//            F_s = 0 for an absent symbol, else max(1, floor(count_s M / total)),
//            M = 4096, the remainder M - sum F added to the largest F (the
//            lowest symbol on ties); C_s = sum_{r<s} F_r;
//   coder    state x in [2^16, 2^32) from 2^16, symbols last to first: if
//            x >= F_s 2^20, emit x mod 2^16 and shift x right by 16; then
//            x = floor(x / F_s) M + (x mod F_s) + C_s;
//   stream   the final state (low, high 16 bits), then the emitted words from
//            the last emitted to the first; offsets[i] is the first word of
//            stream i in the dense output, offsets[streams] the total.
//
// Design (B200).  One thread per stream: a CTA of 128 threads takes the 128
// coordinate streams of one (unit, head, segment).  The segment's code words
// move between HBM and shared memory in chunks of 64 tokens (16-byte cp.async
// loads, 16-byte stores), so the 32 lanes of a warp read a token's words with
// one broadcast LDS and, decoding, build them back with one warp
// OR-reduction per word.  Encode passes: count (per-lane counters in shared
// memory, warp sums, one atomic per symbol and warp), table (a thread per
// (unit, head)), encode into fixed slots of kSeg + 2 words per stream in the
// workspace (a step emits at most one word), an exclusive scan of the stream
// lengths (tile sums, their scan, per-tile scans), and a copy to the dense
// output (a warp per stream).  Decoding looks the symbol of a slot up in a
// per-CTA table of 4096 16-bit entries (s | F_s << 3).  The division by F_s uses
// floor(x * floor(2^32 / F_s) / 2^32), which is floor(x / F_s) or one less,
// and one correction step.
#include "nq_internal.h"

namespace nq {

constexpr int kSeg = 2048;         // tokens per stream segment
constexpr int kCap = kSeg + 2;     // words of one stream at most
constexpr uint32_t kAnsM = 4096u;  // table total
constexpr uint32_t kAnsL = 65536u;  // lower bound of the state

struct EntArgs {
  uint32_t* codes;  // packed code words (read by encode, written by decode)
  int64_t pu, ph;   // vector strides
  int heads;
  int64_t n, slot0, nseg;
  int delta;
};

struct StreamPos {
  int64_t uh, g;  // (unit * heads + head), segment
  int m;          // tokens of the segment
  int64_t vec0;   // first vector of the segment
};

__device__ __forceinline__ StreamPos stream_pos(const EntArgs& a) {
  StreamPos p;
  const int64_t blk = blockIdx.x;
  p.g = blk % a.nseg;
  p.uh = blk / a.nseg;
  const int64_t u = p.uh / a.heads;
  const int h = static_cast<int>(p.uh % a.heads);
  const int64_t t0 = p.g * kSeg;
  p.m = static_cast<int>(min64(kSeg, a.n - t0));
  p.vec0 = u * a.pu + h * a.ph + a.slot0 + t0;
  return p;
}

// Where the code of coordinate c sits in a vector's words.
struct CodeAt {
  int wi, off;
  bool straddle;
};
template <int BITS>
__device__ __forceinline__ CodeAt code_at(int c) {
  CodeAt r;
  const int bp = BITS * c;
  r.wi = bp >> 5;
  r.off = bp & 31;
  r.straddle = r.off + BITS > 32;
  return r;
}
template <int BITS>
__device__ __forceinline__ uint32_t code_of(const uint32_t* w, const CodeAt& at) {
  uint32_t x = w[at.wi] >> at.off;
  if (at.straddle) x |= w[at.wi + 1] << (32 - at.off);
  return x & ((1u << BITS) - 1u);
}

// The code words of a segment pass through shared memory in chunks of
// kChunk tokens (contiguous vectors, 16 BITS bytes each), copied by the whole
// CTA with 16-byte cp.async; a warp then reads its token's word with one
// broadcast LDS instead of one dependent global load per token.
constexpr int kChunk = 64;
template <int BITS>
__device__ __forceinline__ void issue_chunk(uint32_t dst, const uint32_t* seg, int k, int m,
                                            int tid) {
  const int nt = min(kChunk, m - k * kChunk);
  const char* src = reinterpret_cast<const char*>(seg + static_cast<int64_t>(k) * kChunk * 4 * BITS);
  for (int i = tid; i < nt * BITS; i += 128) cp_async16(dst + i * 16, src + i * 16);
}

template <int BITS>
__global__ void __launch_bounds__(128) entropy_count_kernel(const EntArgs a, uint32_t* counts) {
  constexpr int A = 1 << BITS;
  constexpr int VW = 4 * BITS;
  constexpr uint32_t kMask = A - 1;
  __shared__ __align__(16) uint32_t stage[2][kChunk * VW];
  __shared__ uint32_t cnt[4][A][32];  // per warp, symbol and lane: the bank is the lane
  const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
  const StreamPos p = stream_pos(a);
  const CodeAt at = code_at<BITS>(c);
  const uint32_t* seg = a.codes + p.vec0 * VW;
  const int nch = (p.m + kChunk - 1) / kChunk;
  issue_chunk<BITS>(smem_u32(stage[0]), seg, 0, p.m, c);
  cp_async_commit();
  uint32_t* my = &cnt[warp][0][lane];  // this thread's counter of symbol s: my[32 s]
#pragma unroll
  for (int s = 0; s < A; ++s) my[32 * s] = 0;
  uint32_t prev = 0;
  for (int k = 0; k < nch; ++k) {
    if (k + 1 < nch) issue_chunk<BITS>(smem_u32(stage[(k + 1) & 1]), seg, k + 1, p.m, c);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t* buf = stage[k & 1];
    const int nt = min(kChunk, p.m - k * kChunk);
#pragma unroll 4
    for (int t = 0; t < nt; ++t) {
      const uint32_t j = code_of<BITS>(buf + t * VW, at);
      const uint32_t s = a.delta ? ((j - prev) & kMask) : j;
      prev = j;
      my[32 * s] += 1u;
    }
    __syncthreads();  // the buffer is refilled next iteration
  }
#pragma unroll
  for (int s = 0; s < A; ++s) {
    const uint32_t sum = __reduce_add_sync(0xffffffffu, my[32 * s]);
    if (lane == 0 && sum) atomicAdd(counts + p.uh * 8 + s, sum);
  }
}

__global__ void entropy_table_kernel(const uint32_t* counts, int A, int64_t nuh, uint16_t* freq) {
  const int64_t uh = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (uh >= nuh) return;
  uint64_t total = 0;
  for (int s = 0; s < A; ++s) total += counts[uh * 8 + s];
  uint32_t F[8];
  int64_t sum = 0;
  int best = 0;
  for (int s = 0; s < A; ++s) {
    const uint64_t cnt = counts[uh * 8 + s];
    uint64_t f = 0;
    if (cnt) {
      f = cnt * kAnsM / total;
      if (f < 1) f = 1;
    }
    F[s] = static_cast<uint32_t>(f);
    sum += static_cast<int64_t>(f);
    if (F[s] > F[best]) best = s;
  }
  F[best] = static_cast<uint32_t>(static_cast<int64_t>(F[best]) + (kAnsM - sum));
  for (int s = 0; s < A; ++s) freq[uh * A + s] = static_cast<uint16_t>(F[s]);
}

// One rANS step (the coder of the format above): returns the new state and
// emits at most one word at out[--pos].
__device__ __forceinline__ uint32_t ans_put(uint32_t x, uint32_t e, uint32_t rc, uint16_t* out,
                                            int& pos) {
  const uint32_t F = e >> 16, C = e & 0xFFFFu;
  if (F < kAnsM && x >= (F << 20)) {
    out[--pos] = static_cast<uint16_t>(x & 0xFFFFu);
    x >>= 16;
  }
  uint32_t q = F == 1 ? x : __umulhi(x, rc);
  uint32_t r = x - q * F;
  if (r >= F) {
    q += 1;
    r -= F;
  }
  return (q << 12) + r + C;
}

template <int BITS>
__global__ void __launch_bounds__(128) entropy_encode_kernel(const EntArgs a, const uint16_t* freq,
                                                             uint16_t* scratch, uint32_t* sizes) {
  constexpr int A = 1 << BITS;
  constexpr int VW = 4 * BITS;
  constexpr uint32_t kMask = A - 1;
  __shared__ __align__(16) uint32_t stage[2][kChunk * VW];
  __shared__ uint2 sym_tab[A];  // (F << 16 | C, floor(2^32 / F) for F >= 2): one 64-bit load
  const int c = threadIdx.x;
  const StreamPos p = stream_pos(a);
  if (c == 0) {
    uint32_t C = 0;
    for (int s = 0; s < A; ++s) {
      const uint32_t F = freq[p.uh * A + s];
      sym_tab[s] = make_uint2((F << 16) | C, F > 1 ? static_cast<uint32_t>(0x100000000ull / F) : 0u);
      C += F;
    }
  }
  const CodeAt at = code_at<BITS>(c);
  const uint32_t* seg = a.codes + p.vec0 * VW;
  const int nch = (p.m + kChunk - 1) / kChunk;
  const int64_t stream = static_cast<int64_t>(blockIdx.x) * 128 + c;
  uint16_t* out = scratch + stream * kCap;
  int pos = kCap;
  uint32_t x = kAnsL;
  // Symbols are coded last to first.  With the difference, reading token r
  // completes the symbol of token r+1, d_{r+1} = j_{r+1} - j_r, so only the
  // chunk being read is needed; d_0 = j_0 comes last.
  uint32_t jn = 0;
  issue_chunk<BITS>(smem_u32(stage[(nch - 1) & 1]), seg, nch - 1, p.m, c);
  cp_async_commit();
  for (int k = nch - 1; k >= 0; --k) {
    if (k > 0) issue_chunk<BITS>(smem_u32(stage[(k - 1) & 1]), seg, k - 1, p.m, c);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t* buf = stage[k & 1];
    const int nt = min(kChunk, p.m - k * kChunk);
#pragma unroll 4
    for (int t = nt - 1; t >= 0; --t) {
      const uint32_t j = code_of<BITS>(buf + t * VW, at);
      if (a.delta) {
        if (k * kChunk + t < p.m - 1) {
          const uint2 e = sym_tab[(jn - j) & kMask];
          x = ans_put(x, e.x, e.y, out, pos);
        }
        jn = j;
      } else {
        const uint2 e = sym_tab[j];
        x = ans_put(x, e.x, e.y, out, pos);
      }
    }
    __syncthreads();  // the buffer is refilled next iteration
  }
  if (a.delta) x = ans_put(x, sym_tab[jn].x, sym_tab[jn].y, out, pos);
  out[--pos] = static_cast<uint16_t>(x >> 16);
  out[--pos] = static_cast<uint16_t>(x & 0xFFFFu);
  sizes[stream] = static_cast<uint32_t>(kCap - pos);
}

// Exclusive scan of S lengths by one CTA of 1024 threads (used on the tile
// sums): each thread sums a contiguous run, the run sums are scanned across
// the CTA, and each thread writes its run's offsets; offsets[S] is the total.
__global__ void __launch_bounds__(1024) entropy_scan_kernel(const uint32_t* sizes, int64_t S,
                                                            uint32_t* offsets) {
  __shared__ uint32_t wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t per = (S + 1023) / 1024;
  const int64_t b = tid * per, e = min64(S, b + per);
  uint32_t local = 0;
  for (int64_t i = b; i < e; ++i) local += sizes[i];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = wsum[lane], wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    wsum[lane] = wi - w;  // exclusive over warps
  }
  __syncthreads();
  uint32_t run = wsum[warp] + incl - local;
  for (int64_t i = b; i < e; ++i) {
    offsets[i] = run;
    run += sizes[i];
  }
  if (tid == 1023) offsets[S] = run;
}

// The offsets of many streams in three passes: sums of tiles of kScanTile
// lengths (a CTA each), the scan of the tile sums (entropy_scan_kernel, one
// CTA), and per tile a CTA-wide exclusive scan plus the tile's offset.
constexpr int kScanTile = 2048;  // 256 threads x 8 lengths

__global__ void __launch_bounds__(256) entropy_tile_sum_kernel(const uint32_t* sizes, int64_t S,
                                                               uint32_t* tile_sums) {
  __shared__ uint32_t ws[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile;
  uint32_t v = 0;
  for (int i = tid; i < kScanTile; i += 256)
    if (base + i < S) v += sizes[base + i];
  v = __reduce_add_sync(0xffffffffu, v);
  if (lane == 0) ws[warp] = v;
  __syncthreads();
  if (tid == 0) {
    uint32_t t = 0;
    for (int w = 0; w < 8; ++w) t += ws[w];
    tile_sums[blockIdx.x] = t;
  }
}

__global__ void __launch_bounds__(256) entropy_offsets_kernel(const uint32_t* sizes, int64_t S,
                                                              const uint32_t* tile_off,
                                                              int64_t ntiles, uint32_t* offsets) {
  __shared__ uint32_t wsum[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile + tid * 8;
  uint32_t v[8], local = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[k] = base + k < S ? sizes[base + k] : 0u;
    local += v[k];
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < 8 ? wsum[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < 8) wsum[lane] = wi - w;
  }
  __syncthreads();
  uint32_t run = tile_off[blockIdx.x] + wsum[warp] + incl - local;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (base + k < S) offsets[base + k] = run;
    run += v[k];
  }
  if (blockIdx.x == 0 && tid == 0) offsets[S] = tile_off[ntiles];
}

// A warp per stream: its words, tail-aligned in the stream's slot, to the
// dense output.
__global__ void __launch_bounds__(256) entropy_compact_kernel(const uint16_t* scratch,
                                                              const uint32_t* sizes,
                                                              const uint32_t* offsets, int64_t S,
                                                              uint16_t* words) {
  const int64_t s = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (s >= S) return;
  const int lane = threadIdx.x & 31;
  const uint32_t len = sizes[s];
  const uint16_t* src = scratch + s * kCap + (kCap - len);
  uint16_t* dst = words + offsets[s];
#pragma unroll 4
  for (uint32_t i = lane; i < len; i += 32) dst[i] = src[i];
}

template <int BITS>
__global__ void __launch_bounds__(128) entropy_decode_kernel(const EntArgs a, const uint16_t* words,
                                                             const uint32_t* offsets,
                                                             const uint16_t* freq) {
  constexpr int A = 1 << BITS;
  constexpr int VW = 4 * BITS;
  constexpr uint32_t kMask = A - 1;
  __shared__ __align__(16) uint32_t stage[kChunk * VW];
  __shared__ uint32_t fc[A];             // F << 16 | C
  __shared__ uint16_t slot_tab[kAnsM];   // slot -> s | F_s << 3 (the symbol whose range holds it)
  const int c = threadIdx.x, lane = c & 31, blk32 = c >> 5;
  const StreamPos p = stream_pos(a);
  if (c == 0) {
    uint32_t C = 0;
    for (int s = 0; s < A; ++s) {
      const uint32_t F = freq[p.uh * A + s];
      fc[s] = (F << 16) | C;
      C += F;
    }
  }
  __syncthreads();
  {
    uint32_t cum[A];  // C_1 .. C_{A-1} (cum[0] unused)
#pragma unroll
    for (int s = 0; s < A; ++s) cum[s] = fc[s] & 0xFFFFu;
    // thread c fills slots 32c .. 32c+31: s = the number of C_q <= slot, q >= 1
    for (int q = 0; q < static_cast<int>(kAnsM) / 128; ++q) {
      const uint32_t slot = static_cast<uint32_t>(c) * (kAnsM / 128) + q;
      uint32_t s = 0;
#pragma unroll
      for (int k = 1; k < A; ++k) s += slot >= cum[k] ? 1u : 0u;
      slot_tab[slot] = static_cast<uint16_t>(s | ((fc[s] >> 16) << 3));
    }
  }
  __syncthreads();
  const int64_t stream = static_cast<int64_t>(blockIdx.x) * 128 + c;
  const uint32_t o0 = offsets[stream];
  const uint32_t len = offsets[stream + 1] - o0;
  const uint16_t* in = words + o0;
  // a stream that ends early (not written by the encoder) reads zeros, never
  // past its end; the next word is fetched one renormalisation ahead
  uint32_t x = (len > 0 ? in[0] : 0u) | (static_cast<uint32_t>(len > 1 ? in[1] : 0u) << 16);
  uint32_t nxt = len > 2 ? in[2] : 0u;
  uint32_t i = 3;
  // this lane's code within its warp's 32-coordinate block of BITS words
  const CodeAt at = code_at<BITS>(lane);
  uint32_t* seg = a.codes + p.vec0 * VW;
  const int nch = (p.m + kChunk - 1) / kChunk;
  uint32_t j = 0;
  for (int k = 0; k < nch; ++k) {
    const int nt = min(kChunk, p.m - k * kChunk);
#pragma unroll 4
    for (int t = 0; t < nt; ++t) {
      const uint32_t slot = x & (kAnsM - 1u);
      const uint32_t e = slot_tab[slot];
      const uint32_t s = e & 7u;
      x = (e >> 3) * (x >> 12) + slot - (fc[s] & 0xFFFFu);
      if (x < kAnsL) {
        x = (x << 16) | nxt;
        nxt = i < len ? in[i] : 0u;
        ++i;
      }
      j = a.delta ? ((j + s) & kMask) : s;
      const uint32_t lo = j << at.off;
      const uint32_t hi = at.straddle ? (j >> (32 - at.off)) : 0u;
#pragma unroll
      for (int w = 0; w < BITS; ++w) {
        const uint32_t v = (at.wi == w ? lo : 0u) | (at.straddle && at.wi + 1 == w ? hi : 0u);
        const uint32_t word = __reduce_or_sync(0xffffffffu, v);
        if (lane == w) stage[t * VW + blk32 * BITS + w] = word;
      }
    }
    __syncthreads();  // the chunk's words are complete
    uint4* dst = reinterpret_cast<uint4*>(seg + static_cast<int64_t>(k) * kChunk * VW);
    const uint4* src = reinterpret_cast<const uint4*>(stage);
    for (int q = c; q < nt * BITS; q += 128) dst[q] = src[q];
    __syncthreads();  // the stage is rewritten by the next chunk
  }
}

// ---------------------------------------------------------------- launch
int64_t entropy_streams(int units, int heads, int64_t n) {
  return static_cast<int64_t>(units) * heads * ((n + kSeg - 1) / kSeg) * kD;
}

static size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

size_t entropy_workspace_bytes(int units, int heads, int64_t n) {
  const int64_t S = entropy_streams(units, heads, n);
  const int64_t ntiles = (S + kScanTile - 1) / kScanTile;
  return align256(static_cast<size_t>(units) * heads * 8 * sizeof(uint32_t)) +
         align256(static_cast<size_t>(S) * sizeof(uint32_t)) +
         2 * align256(static_cast<size_t>(ntiles + 1) * sizeof(uint32_t)) +
         static_cast<size_t>(S) * kCap * sizeof(uint16_t);
}

int64_t entropy_max_words(int units, int heads, int64_t n) {
  return entropy_streams(units, heads, n) * kCap;
}

static EntArgs ent_args(const nq_packed& pk, int heads, int64_t n, int64_t slot0, int delta) {
  EntArgs a{};
  a.codes = pk.codes;
  a.pu = pk.unit_stride;
  a.ph = pk.head_stride;
  a.heads = heads;
  a.n = n;
  a.slot0 = slot0;
  a.nseg = (n + kSeg - 1) / kSeg;
  a.delta = delta;
  return a;
}

cudaError_t launch_entropy_encode(const nq_packed& in, int units, int heads, int64_t n,
                                  int64_t slot0, int delta, uint16_t* freq, uint32_t* offsets,
                                  uint16_t* words, void* ws, cudaStream_t stream) {
  const EntArgs a = ent_args(in, heads, n, slot0, delta);
  const int64_t nuh = static_cast<int64_t>(units) * heads;
  const int64_t blocks = nuh * a.nseg;
  const int64_t S = blocks * kD;
  const int A = 1 << in.bits;
  char* w = static_cast<char*>(ws);
  uint32_t* counts = reinterpret_cast<uint32_t*>(w);
  w += align256(static_cast<size_t>(nuh) * 8 * sizeof(uint32_t));
  uint32_t* sizes = reinterpret_cast<uint32_t*>(w);
  w += align256(static_cast<size_t>(S) * sizeof(uint32_t));
  const int64_t ntiles = (S + kScanTile - 1) / kScanTile;
  uint32_t* tile_sums = reinterpret_cast<uint32_t*>(w);
  w += align256(static_cast<size_t>(ntiles + 1) * sizeof(uint32_t));
  uint32_t* tile_off = reinterpret_cast<uint32_t*>(w);
  w += align256(static_cast<size_t>(ntiles + 1) * sizeof(uint32_t));
  uint16_t* scratch = reinterpret_cast<uint16_t*>(w);
  cudaError_t err = cudaMemsetAsync(counts, 0, static_cast<size_t>(nuh) * 8 * sizeof(uint32_t),
                                    stream);
  if (err != cudaSuccess) return err;
  const unsigned grid = static_cast<unsigned>(blocks);
  if (in.bits == 3) entropy_count_kernel<3><<<grid, 128, 0, stream>>>(a, counts);
  else entropy_count_kernel<2><<<grid, 128, 0, stream>>>(a, counts);
  entropy_table_kernel<<<static_cast<unsigned>((nuh + 127) / 128), 128, 0, stream>>>(counts, A,
                                                                                     nuh, freq);
  if (in.bits == 3) entropy_encode_kernel<3><<<grid, 128, 0, stream>>>(a, freq, scratch, sizes);
  else entropy_encode_kernel<2><<<grid, 128, 0, stream>>>(a, freq, scratch, sizes);
  entropy_tile_sum_kernel<<<static_cast<unsigned>(ntiles), 256, 0, stream>>>(sizes, S, tile_sums);
  entropy_scan_kernel<<<1, 1024, 0, stream>>>(tile_sums, ntiles, tile_off);
  entropy_offsets_kernel<<<static_cast<unsigned>(ntiles), 256, 0, stream>>>(sizes, S, tile_off,
                                                                            ntiles, offsets);
  entropy_compact_kernel<<<static_cast<unsigned>((S + 7) / 8), 256, 0, stream>>>(scratch, sizes,
                                                                               offsets, S, words);
  return cudaGetLastError();
}

cudaError_t launch_entropy_decode(const uint16_t* words, const uint32_t* offsets,
                                  const uint16_t* freq, int units, int heads, int64_t n,
                                  int delta, const nq_packed& out, int64_t slot0,
                                  cudaStream_t stream) {
  const EntArgs a = ent_args(out, heads, n, slot0, delta);
  const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(units) * heads * a.nseg);
  if (out.bits == 3)
    entropy_decode_kernel<3><<<grid, 128, 0, stream>>>(a, words, offsets, freq);
  else
    entropy_decode_kernel<2><<<grid, 128, 0, stream>>>(a, words, offsets, freq);
  return cudaGetLastError();
}

}  // namespace nq
