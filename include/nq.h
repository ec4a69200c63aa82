/*
 * nq.h -- C ABI of libnq: B200 (sm_100a) kernels for training-free KV-cache
 * compression by token eviction plus E8 lattice vector quantisation.
 *
 * The method follows two descriptions of NexusQuant:
 *   [NQ-zh]  "NexusQuant: training-free 10-33x KV cache compression"
 *            (zingnex.cn), sections "Token eviction", "E8 lattice
 *            quantisation", "Implementation details";
 *   [NQ-pt]  "Como comprimir o KV cache do seu LLM em 33x sem treino"
 *            (dev.to), section "Como funciona (em 6 passos)", steps 1-6
 *            (step 6, the coding of the lattice indices: nq_entropy_*).
 * The pages give no formulas or code; the concrete arithmetic below (fp32
 * operation order, tie rules, scale rule, packed layout) is this library's
 * reading and is restated next to each call.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every tensor pointer is a DEVICE pointer that the caller allocates and
 *   owns; the library never allocates, frees or retains memory, except
 *   nq_rope_tables_fill_host, which writes a caller-owned HOST buffer.  The
 *   one exception: nq_encode's K and V inputs may also be pinned host memory
 *   (cudaHostAlloc / cudaHostRegister), which the kernels read in place, so
 *   only the rows encoded (the kept tokens) cross the bus; memory the device
 *   cannot read is refused with NQ_ERR_INVALID before any launch.
 * - Every compute call is asynchronous on the caller's CUDA stream and
 *   returns as soon as its kernels are queued.  Nothing synchronises.
 * - Return value: nq_status.  NQ_ERR_INVALID for bad arguments (checked on the
 *   host before anything is launched; nothing is launched then),
 *   NQ_ERR_WORKSPACE for a workspace smaller than required, NQ_ERR_CUDA when a
 *   launch reports an error.  nq_last_error() gives a message for the calling
 *   thread.  No C++ exception, exit() or device trap crosses the ABI.
 * - A KV tensor (bf16) holds, for each (unit, head, token), one vector of 128
 *   contiguous bf16 coordinates.  Its three strides are in ELEMENTS and must
 *   be multiples of 8, and the base pointer 16-byte aligned (16-byte vector
 *   loads).  A "unit" is one layer of one sequence.
 * - Inputs must be finite with |x| <= 2^30; other values are out of
 *   contract (no fault: the kernels stay within their buffers, the codes of
 *   such a vector are unspecified).
 * - Staging uses cp.async groups and bulk-copy groups, whose waits complete
 *   in hardware.  The one polled wait is decode's wait for its own
 *   tensor-core products (an mbarrier that the MMA unit signals on
 *   completion); it is bounded (2^20 polls), and when it expires the kernel
 *   sets bit 1 of the device error word and its warpgroup stops (that call's
 *   output is then incomplete).  nq_device_error() reads the device error
 *   word; it reads 0 after any sequence of valid calls.
 */
#ifndef NQ_H
#define NQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nq_stream_t; /* = cudaStream_t; NULL = legacy default stream */

typedef enum {
    NQ_OK = 0,
    NQ_ERR_INVALID = 1,
    NQ_ERR_WORKSPACE = 2,
    NQ_ERR_CUDA = 3,
    NQ_ERR_UNSUPPORTED = 4
} nq_status;

#define NQ_HEAD_DIM 128

/* Strides, in bf16 elements, of a [units][heads][tokens][128] KV tensor. */
typedef struct {
    int64_t unit;
    int64_t head;
    int64_t token;
} nq_kv_strides;

/* A packed store of E8 codes for one of K or V.
 *   codes: uint32 words, 4*bits words per vector.  The b-bit code of
 *          coordinate c (0..127) of a vector sits at bits [b*c, b*c + b) of
 *          the vector's little-endian stream of words (b = 3: 12 words,
 *          b = 2: 8 words).
 *   meta:  one uint32 per vector: bits 0..15 = coset mask (bit g set when
 *          group g, coordinates 8g..8g+7, lies in the half-integer coset
 *          D8 + 1/2), bits 16..31 = the vector's fp16 scale sigma.
 *   Vector (unit u, head h, slot i) is at index u*unit_stride + h*head_stride
 *   + i (in vectors) of both arrays.  16-byte aligned codes pointer. */
typedef struct {
    uint32_t *codes;
    uint32_t *meta;
    int64_t unit_stride;
    int64_t head_stride;
    int32_t bits; /* 2 or 3 */
} nq_packed;

/* Thread-local message for the last non-OK status (never NULL). */
const char *nq_last_error(void);

/* ABI version, bumped on incompatible changes. */
int nq_version(void);

/* Bytes of raw packed storage per vector: 4*(4*bits) + 4 (52 for K3, 36 for V2). */
int64_t nq_packed_bytes_per_vector(int bits);

/* ----------------------------------------------------------- RoPE tables
 * Split-half rotary embedding ([NQ-zh] "Supported models": split-half RoPE
 * only; interleaved RoPE is not supported), pairs (i, i+64), frequencies
 * w_i = theta^(-i/64).  For position p = 256a + b the tables hold fp32
 * roundings of fp64 cos/sin:
 *   A[a][i] = (cos(256a*w_i), sin(256a*w_i)),  a < ceil(max_pos/256)
 *   B[b][i] = (cos(b*w_i),    sin(b*w_i)),     b < 256
 * as float2 pairs, A first then B.  The kernels combine them in fp32:
 *   c = fmaf(cA, cB, -(sA*sB)),  s = fmaf(sA, cB, cA*sB).
 * The caller copies the filled host buffer to device memory (16-byte
 * aligned) once per theta and passes that device pointer with the same
 * max_pos. */
size_t nq_rope_tables_bytes(int64_t max_pos);
nq_status nq_rope_tables_fill_host(double theta, int64_t max_pos, void *host_buf, size_t bytes);

/* ----------------------------------------------------------------- score
 * Key-key proxy importance ([NQ-zh] "Implementation details": fast key-key
 * proxy; [NQ-pt] step 1: cross-head inner product), on the stored, rotated
 * keys:
 *   m[u][h][d]   = fp32( (sum over t in [T-W, T) of K[u][h][t][d], fp64) / W )
 *   scores[u][t] = sum over h, d of (double)K[u][h][t][d] * (double)m[u][h][d]
 * (fp64 accumulation; products are exact, summation order is the kernel's).
 * K: bf16 [units][heads][T][128] with strides ks.  scores: fp64
 * [units][T], row-contiguous.  ws: device workspace of at least
 * nq_score_workspace_bytes(units, heads) bytes (holds m), 16-byte aligned.
 * 1 <= W <= T; heads <= 128 (more: NQ_ERR_UNSUPPORTED). */
size_t nq_score_workspace_bytes(int units, int heads);
nq_status nq_score(const void *K, nq_kv_strides ks, int units, int heads, int64_t T, int W,
                   double *scores, void *ws, size_t ws_bytes, nq_stream_t stream);

/* ------------------------------------------- score with no allocation
 * This entry point has no counterpart in the method description; it exists
 * for callers of this library that cannot allocate device memory: code
 * embedded in a host framework that owns every byte of the GPU (a serving
 * engine whose memory planner reserved all of HBM for its KV pool up front),
 * or a latency-critical loop where a cudaMalloc/cudaFree would block or
 * synchronise the device.  Such callers cannot provide nq_score's workspace.
 *
 * nq_score_static computes exactly what nq_score computes, with the same
 * arguments minus the workspace.  The window means live instead in a fixed
 * array inside the library's own device memory, sized for at most
 * NQ_SCORE_STATIC_MAX_VECTORS (unit, head) pairs (1 MiB); every GPU that
 * loads the library holds that array until the process exits.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   - units * heads above the maximum, or heads above 128: NQ_ERR_UNSUPPORTED,
 *     nothing launched.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it with the device's context; the
 *     first call after a device reset (a new context) looks it up again.
 *     Make the first call on a device, and after a reset, before any stream
 *     capture.
 *   - All calls share the array and it keeps the last call's contents (each
 *     call overwrites every entry it reads, so nothing needs clearing).
 *     Calls whose kernels overlap on the same GPU (different streams, or
 *     different host threads) race on it and give undefined scores:
 *     serialise them. */
#define NQ_SCORE_STATIC_MAX_VECTORS 2048
nq_status nq_score_static(const void *K, nq_kv_strides ks, int units, int heads, int64_t T, int W,
                          double *scores, nq_stream_t stream);

/* ---------------------------------------------------------------- select
 * Token eviction ([NQ-zh] "Token eviction": always keep BOS and a recent
 * sliding window, drop the low scorers; [NQ-pt] step 2).  Per unit:
 *   mid = T - 1 - W, n_evict = floor(mid * evict_pct / 100),
 *   kept = {0} u top (mid - n_evict) of positions [1, T-W) by
 *          (score descending, position ascending) u [T-W, T),
 * written in ascending order to kept[u*kept_stride + 0 .. n-1], n =
 * nq_kept_count(T, W, evict_pct) (every unit keeps the same count).
 * T <= 1 + W or evict_pct == 0 keeps everything.  scores: fp64 [units][T]
 * row-contiguous (as written by nq_score); kept_stride >= n. */
int64_t nq_kept_count(int64_t T, int64_t W, int evict_pct);
nq_status nq_select(const double *scores, int units, int64_t T, int W, int evict_pct,
                    int32_t *kept, int64_t kept_stride, nq_stream_t stream);

/* ---------------------------------------------------------------- encode
 * RoPE removal, Hadamard rotation and E8 quantisation ([NQ-zh] "E8 lattice
 * quantisation", "Implementation details"; [NQ-pt] steps 3-5).  For slot i
 * (0 <= i < n) of every (unit u, head h):
 *   src = kept ? kept[u*kept_stride + i] : i      (input token, < T_in)
 *   pos = pos_base + src                          (RoPE position)
 *   keys:   v = RoPE^-1(K[u][h][src]) at pos:
 *             v_i    = fmaf(k_i,    c, k_{i+64}*s)
 *             v_i+64 = fmaf(k_i+64, c, -(k_i*s))
 *   values: v = V[u][h][src]
 *   v <- unnormalised Walsh-Hadamard (Sylvester order, stages 1, 2, ..., 64,
 *        butterfly (a, b) -> (a+b, a-b), fp32)
 *   sigma = fp16(min(fp32(max|v| * G_b), 65504)), G_b = fp32(1/(A_b*sqrt(128))),
 *           A_3 = 3.5, A_2 = 1.5;  r = fp32(C/sigma) (0 if sigma == 0),
 *           C = fp32(1/sqrt(128));  y = fp32(v * r)
 *   each group of 8 coordinates of y -> nearest E8 point (Conway-Sloane:
 *           decode D8 and D8 + 1/2 in fp32 -- round to nearest even, fix an
 *           odd sum on the first largest-error coordinate, fp32 squared
 *           distance, ties to the integer coset)
 *   2q clamped to the b-bit symmetric range (half coset |2q| <= 2^b-1,
 *           integer coset |2q| <= 2^b-2), code = (2q + lim)/2,
 *   written to slot slot0 + i of k_out / v_out.
 * K and/or V may be NULL (then its k_out/v_out is ignored).  bits: K and V
 * may differ (K3V2).  rope_tab: device tables from nq_rope_tables_fill_host
 * (required when K != NULL), positions must be < rope_max_pos.
 * units * n must stay below 2^31 (NQ_ERR_UNSUPPORTED otherwise). */
nq_status nq_encode(const void *K, nq_kv_strides ks, const void *V, nq_kv_strides vs, int units,
                    int heads, int64_t T_in, int64_t n, const int32_t *kept, int64_t kept_stride,
                    int64_t pos_base, const float *rope_tab, int64_t rope_max_pos,
                    const nq_packed *k_out, const nq_packed *v_out, int64_t slot0,
                    nq_stream_t stream);

/* ---------------------------------------------------------------- decode
 * Inverse path: for slot slot0 + i (0 <= i < n) of every (unit, head):
 *   t_c   = 2 j_c - 2^b + 2 - h_g       (= 2q, h_g the group's coset bit)
 *   w     = Walsh-Hadamard(t)           (integers, exact in fp32)
 *   x_c   = fp32(w_c * kappa),  kappa = fp32(fp32(sigma/2) * C)
 *   keys: re-apply RoPE at pos = pos_base + (positions ?
 *         positions[u*pos_stride + i] : i) ([NQ-zh] "Implementation
 *         details": RoPE restored after quantisation):
 *           o_i = fmaf(x_i, c, -(x_{i+64}*s)),  o_i+64 = fmaf(x_i+64, c, x_i*s)
 *   bf16 round-to-nearest-even into K_out/V_out[u][h][i] (strides kos/vos).
 * k_in/v_in may be NULL (that output is skipped).  The transform runs on the
 * tensor cores as an exact f16 product with fp32 accumulation (every partial
 * sum an integer below 2^18) in tiles of 128 vectors (8 / hg slot tiles of a
 * group of hg heads, hg the largest divisor of heads up to 8; keys need
 * hg >= 3), or on the CUDA cores (see nq_set_decode_engine); both give the
 * bits above. */
nq_status nq_decode(const nq_packed *k_in, const nq_packed *v_in, int units, int heads,
                    int64_t n, int64_t slot0, const int32_t *positions, int64_t pos_stride,
                    int64_t pos_base, const float *rope_tab, int64_t rope_max_pos, void *K_out,
                    nq_kv_strides kos, void *V_out, nq_kv_strides vos, nq_stream_t stream);

/* --------------------------------------- exact (24/16-bit) index packing
 * The lattice step at exactly b bits per coordinate plus the scale ([NQ-pt]
 * step 5 stores the E8 indices at "2 bits/dim"): the coset bit of each group
 * rides in the low bit of the group's last code, which a point of E8 does
 * not need -- its codes j = q + 2^(b-1) - 1 (integer coset) or
 * j = (q - 1/2) + 2^(b-1) (half coset) have an even sum, so the low bit of
 * j_7 is the parity of j_0 .. j_6.  This needs every coded point in E8, so the
 * lattice step is the nearest E8 point INSIDE the b-bit code box (the
 * library's parity-preserving reading of the clamp), per coset:
 *   u = y - shift (shift 0: f in [-(2^(b-1)-1), 2^(b-1)-1];
 *                  shift 1/2: f in [-2^(b-1), 2^(b-1)-1]),
 *   f_i = clamp(rint(u_i), lo, hi) (ties to even), e_i = u_i - f_i,
 *   d = e_0^2 then fmaf chain; when sum f is odd the one coordinate whose move
 *   by dir = (e >= 0 ? +1 : -1), reversed when that leaves the box, costs
 *   least -- cost fmaf(-2 dir, e, 1), first index on ties -- moves, d += cost;
 *   the half coset wins only when d1 < d0.
 * It equals nq_encode's point whenever that point lies in the box.
 * Layout (nq_packed_exact): codes as in nq_packed (4*bits uint32 words per
 * vector, code c at bits [b*c, b*c + b)), except that the low bit of code
 * 8g+7 holds group g's coset bit (1 = half coset); sigma: one fp16 scale per
 * vector (uint16, 2-byte aligned).  4*(4*bits) + 2 bytes per vector: 50 for
 * K3 (3.125 bits per coordinate), 34 for V2 (2.125).
 * nq_encode_exact / nq_decode_exact take the same arguments, with the same
 * rules and errors, as nq_encode / nq_decode, with exact-layout stores; the
 * steps before and after the lattice step are theirs.  Decode restores each
 * code 7's low bit from the parity of codes 0..6.  The codes of an exact
 * store can go through nq_entropy_encode / nq_entropy_decode as they are (an
 * nq_packed with the same codes, strides and bits; its meta is not read). */
typedef struct {
    uint32_t *codes;
    uint16_t *sigma;
    int64_t unit_stride;
    int64_t head_stride;
    int32_t bits; /* 2 or 3 */
} nq_packed_exact;

int64_t nq_packed_exact_bytes_per_vector(int bits);
nq_status nq_encode_exact(const void *K, nq_kv_strides ks, const void *V, nq_kv_strides vs,
                          int units, int heads, int64_t T_in, int64_t n, const int32_t *kept,
                          int64_t kept_stride, int64_t pos_base, const float *rope_tab,
                          int64_t rope_max_pos, const nq_packed_exact *k_out,
                          const nq_packed_exact *v_out, int64_t slot0, nq_stream_t stream);
nq_status nq_decode_exact(const nq_packed_exact *k_in, const nq_packed_exact *v_in, int units,
                          int heads, int64_t n, int64_t slot0, const int32_t *positions,
                          int64_t pos_stride, int64_t pos_base, const float *rope_tab,
                          int64_t rope_max_pos, void *K_out, nq_kv_strides kos, void *V_out,
                          nq_kv_strides vos, nq_stream_t stream);

/* ----------------------------------------------------- decode attention
 * Decode-phase attention over the packed cache, reconstructing keys and
 * values inside the attention (the on-demand reconstruction within
 * FlashAttention described for VQKV, section "Decoding"; the NexusQuant pages
 * give no attention formula, so this reading is the library's):
 *   for unit u, query head j (KV head h = j / G), over the n slots
 *   slot0 .. slot0+n-1 of (u, h):
 *     s_t = scale * dot(q[u][j], k_t)      k_t: the fp32 key that nq_decode
 *                                          rounds to bf16 (RoPE re-applied at
 *                                          pos = pos_base + (positions ?
 *                                          positions[u*pos_stride + t] : t))
 *     out[u][j] = sum_t softmax(s)_t v_t   v_t: the fp32 value before bf16
 *     lse[u][j] = log(sum_t exp(s_t))      (natural log; lse may be NULL)
 * fp32 arithmetic in the kernels' own order (scores, fp32 exp, a running
 * max and sum over tiles of 16 tokens within each chunk, chunks merged at
 * the end), so results agree with an exact evaluation to about 1e-5
 * relative, not bit for bit.  q: fp32 [units][heads*G][128], 16-byte aligned.
 * out: fp32 [units][heads*G][128].  k_in/v_in: packed stores as for
 * nq_decode (any bits 2/3).  1 <= G <= 8, 1 <= n < 2^31 (larger n returns
 * NQ_ERR_UNSUPPORTED).  ws: device workspace of
 * nq_attend_workspace_bytes(units, heads, G, n) bytes, 16-byte aligned
 * (per-chunk partial results; the token chunk per CTA depends on units,
 * heads and n only).  rope_tab as for nq_decode. */
size_t nq_attend_workspace_bytes(int units, int heads, int G, int64_t n);
nq_status nq_attend(const float *q, int units, int heads, int G, const nq_packed *k_in,
                    const nq_packed *v_in, int64_t n, int64_t slot0, const int32_t *positions,
                    int64_t pos_stride, int64_t pos_base, const float *rope_tab,
                    int64_t rope_max_pos, float scale, float *out, float *lse, void *ws,
                    size_t ws_bytes, nq_stream_t stream);

/* --------------------------------------------- delta + entropy coding
 * Lossless coding of the lattice indices (the b-bit codes) of a packed store,
 * the last step of the NexusQuant pipeline: consecutive tokens give similar
 * lattice indices, so the difference to the previous token is stored and the
 * result compressed ([NQ-zh] "Implementation details"; [NQ-pt] step 6, which
 * names zstd).  The coder is rANS (Duda, "Asymmetric numeral systems", 2013)
 * with a static table per (unit, head); this format is the library's:
 *   streams: one per (unit, head, segment of 2048 slots, coordinate c), in
 *     that order (coordinate fastest), over slots slot0 .. slot0+n-1;
 *     symbols d_t = (j_t - j_{t-1}) mod 2^b inside the segment, d = j at the
 *     segment's first slot (delta = 1), or d_t = j_t (delta = 0);
 *   freq [units][heads][2^b] uint16: F_s = 0 for an absent symbol, else
 *     max(1, floor(count_s * 4096 / total)), the remainder 4096 - sum F added
 *     to the largest F (lowest symbol on ties);
 *   words: stream i is words[offsets[i] .. offsets[i+1]) (uint16): the final
 *     coder state (low, high 16 bits) then the emitted words from the last
 *     emitted to the first; offsets [streams + 1] uint32, offsets[streams] =
 *     the total words.
 * Meta words (coset bits, fp16 scale) are not part of the streams.
 * nq_entropy_encode reads the code words of `in` and writes freq, offsets and
 * words (capacity words_cap >= nq_entropy_max_words, the worst case of one
 * word per symbol plus two per stream); ws: device workspace of
 * nq_entropy_workspace_bytes, 16-byte aligned.  nq_entropy_decode writes the
 * code words of `out` (slots slot0 .. slot0+n-1; meta untouched) from the
 * output of nq_entropy_encode with the same units, heads, n, bits and delta;
 * other inputs are out of contract (no fault: a stream never reads past its
 * offsets, but the codes are then unspecified).  All arrays are device
 * memory owned by the caller.  1 <= n < 2^25; units * heads * streams must
 * keep the worst case below 2^32 words (else NQ_ERR_UNSUPPORTED). */
int64_t nq_entropy_streams(int units, int heads, int64_t n);
int64_t nq_entropy_max_words(int units, int heads, int64_t n);
size_t nq_entropy_workspace_bytes(int units, int heads, int64_t n);
nq_status nq_entropy_encode(const nq_packed *in, int units, int heads, int64_t n, int64_t slot0,
                            int delta, uint16_t *freq, uint32_t *offsets, uint16_t *words,
                            int64_t words_cap, void *ws, size_t ws_bytes, nq_stream_t stream);
nq_status nq_entropy_decode(const uint16_t *words, const uint32_t *offsets, const uint16_t *freq,
                            int units, int heads, int64_t n, int delta, const nq_packed *out,
                            int64_t slot0, nq_stream_t stream);

/* ------------------------------------------------------ E8 quantiser
 * The lattice step of nq_encode on its own ([NQ-zh] "E8 lattice
 * quantisation"; [NQ-pt] step 4), for coordinates that are already rotated
 * and scaled: each row g of y ([groups][8] fp32, contiguous) is snapped to
 * the nearest E8 point with exactly nq_encode's fp32 decoder (D8 and
 * D8 + 1/2, round to nearest even, the odd-sum fix on the first
 * largest-error coordinate, fp32 fma distance chains, a tie keeps the
 * integer coset), then clamped and coded as in nq_encode:
 *   codes[g]: the 8 b-bit codes of the group, code i at bits [b*i, b*i + b)
 *   coset[g]: 1 when the point lies in D8 + 1/2, else 0.
 * y, codes (uint32 [groups]) and coset (uint8 [groups]) are device arrays
 * owned by the caller; y and codes 4-byte aligned.  bits is 2 or 3;
 * groups = 0 launches nothing.  y must be finite with |y| < 2^22; other
 * values are out of contract (no fault, unspecified codes). */
nq_status nq_e8_quantise(const float *y, int64_t groups, int bits, uint32_t *codes,
                         uint8_t *coset, nq_stream_t stream);

/* The lattice step of nq_encode_exact on its own: each row of y is snapped
 * to the nearest E8 point inside the b-bit code box (see nq_encode_exact),
 * codes[g] holds its 8 codes (code i at bits [b*i, b*i + b)) with the low
 * bit of code 7 replaced by the coset bit, coset[g] the coset (1 = half).
 * Same arguments, alignment rules and errors as nq_e8_quantise. */
nq_status nq_e8_box_quantise(const float *y, int64_t groups, int bits, uint32_t *codes,
                             uint8_t *coset, nq_stream_t stream);

/* ------------------------------------------------------- decode engine
 * Which kernel nq_decode / nq_decode_exact run (process-wide, default
 * NQ_DECODE_AUTO):
 *   NQ_DECODE_AUTO          the tensor cores where they apply (see nq_decode)
 *                           and the call has at least two 128-vector tiles per
 *                           warpgroup of the SMs (8 or 6 tiles per SM; below
 *                           that the per-CTA setup of the tensor-core kernel
 *                           outweighs it), else the CUDA cores;
 *   NQ_DECODE_TENSOR_CORES  the tensor cores wherever they apply;
 *   NQ_DECODE_CUDA_CORES    always the CUDA-core kernel.
 * Both give the same bits.  Returns NQ_ERR_INVALID for another value.  Not
 * synchronised with launches in flight: set it between calls. */
typedef enum {
  NQ_DECODE_AUTO = 0,
  NQ_DECODE_TENSOR_CORES = 1,
  NQ_DECODE_CUDA_CORES = 2
} nq_decode_engine;
nq_status nq_set_decode_engine(int engine);
int nq_get_decode_engine(void);

/* -------------------------------------------------------------- status
 * Reads and clears the device error word of in-kernel failure reports
 * (bit 1: a tensor-core product of nq_decode / nq_decode_exact did not
 * complete within its bounded wait).  Synchronises the current device, so a
 * pending launch error surfaces here as NQ_ERR_CUDA. */
nq_status nq_device_error(uint32_t *flags_out);

#ifdef __cplusplus
}
#endif
#endif /* NQ_H */
