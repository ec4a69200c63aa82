/*
 * nq_oracle.c -- plain, slow, single-threaded CPU oracle of the NexusQuant
 * KV-cache hot path: key-key token scoring, eviction, RoPE removal, Hadamard
 * rotation, per-vector fp16 scale, E8 lattice quantisation, bit packing and
 * the inverse path; decode attention on the packed cache; the delta + rANS
 * coding of the lattice indices; and the nearest E8 point inside the code box
 * with the exact (coset bit folded) packing.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline of the benchmark may load this file.  It shares no code, header,
 * table or constant generator with the CUDA library; every step is written
 * out here from the method description:
 *
 *   - "NexusQuant: training-free 10-33x KV cache compression"
 *     (zingnex.cn, sections "Token eviction", "E8 lattice quantisation",
 *     "Implementation details")
 *   - "Como comprimir o KV cache do seu LLM em 33x sem treino"
 *     (dev.to, section "Como funciona (em 6 passos)", steps 1-6)
 *
 * The pages leave every formula open; the readings taken (fp32 operation
 * order, tie rules, scale rule, packed layout) are stated next to each
 * function below.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no SIMD intrinsics, no OpenMP).  -ffp-contract=off matters: every fused
 * multiply-add below is an explicit fmaf(), every other product is rounded.
 *
 * Parity status: every function is pinned by tests under tests/ (closed
 * forms, brute force, library routines); end-to-end model quality is
 * "parity unpinned" (it needs models and datasets).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OQ_D 128
#define OQ_HALF 64

/* ---------------------------------------------------------------- floats */

static float oq_u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t oq_f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* 1/sqrt(128) rounded to fp32, and 1/(A_b * sqrt(128)) for A_3 = 3.5 and
 * A_2 = 1.5 (the largest code magnitude of a b-bit symmetric code), each the
 * fp32 nearest to the real number. */
#define OQ_C_BITS 0x3DB504F3u
#define OQ_G3_BITS 0x3CCEE116u
#define OQ_G2_BITS 0x3D715BEFu

float oq_bf16_to_f32(uint16_t h) { return oq_u2f((uint32_t)h << 16); }

/* IEEE round-to-nearest-even of an fp32 value to bfloat16 (finite inputs;
 * NaN is kept quiet). */
uint16_t oq_f32_to_bf16(float f)
{
    uint32_t u = oq_f2u(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* IEEE binary16 round-to-nearest-even of a finite fp32 value, written from
 * the format definition (1 sign, 5 exponent, 10 fraction bits, bias 15).
 * Overflow gives +-inf here; the scale rule saturates separately. */
uint16_t oq_f32_to_f16(float f)
{
    uint32_t u = oq_f2u(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7FFFFFFFu;
    if (a >= 0x7F800000u) /* inf / nan */
        return (uint16_t)(sign | 0x7C00u | (a > 0x7F800000u ? 0x200u : 0u));
    int e = (int)(a >> 23) - 127;    /* unbiased exponent */
    uint32_t m = (a & 0x7FFFFFu);
    if (a == 0) return sign;
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    uint32_t full;  /* significand with hidden bit, 24 bits */
    int shift;      /* bits to drop */
    uint32_t ebits;
    if (e >= -14) { /* normal binary16 range */
        full = m | 0x800000u;
        shift = 13;
        ebits = (uint32_t)(e + 15);
    } else {        /* subnormal binary16: value = frac * 2^-24 */
        if ((int)(a >> 23) == 0) return sign; /* fp32 subnormal: far below 2^-25 */
        full = m | 0x800000u;
        shift = 13 + (-14 - e);
        if (shift > 24) return sign; /* below half of the smallest subnormal */
        ebits = 0;
    }
    uint32_t keep = full >> shift;
    uint32_t rem = full & ((1u << shift) - 1u);
    uint32_t halfway = 1u << (shift - 1);
    if (rem > halfway || (rem == halfway && (keep & 1u))) keep += 1u;
    uint32_t out;
    if (ebits) {
        /* keep has the hidden bit at position 10; a carry to bit 11 bumps the
         * exponent, which the addition below does by itself */
        out = ((ebits - 1u) << 10) + keep;
    } else {
        out = keep; /* may round up into the smallest normal, also correct */
    }
    if (out >= 0x7C00u) out = 0x7C00u;
    return (uint16_t)(sign | out);
}

float oq_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu, m = h & 0x3FFu;
    if (e == 0) {
        float v = (float)m * oq_u2f(0x33800000u); /* m * 2^-24, exact */
        return sign ? -v : v;
    }
    if (e == 31) return oq_u2f(sign | 0x7F800000u | (m << 13));
    return oq_u2f(sign | ((e - 15 + 127) << 23) | (m << 13));
}

/* ------------------------------------------------------------ rope table */

/* Split-half rotary embedding (pairs (i, i+64)), frequencies
 * omega_i = theta^(-2i/D) (NexusQuant, "Supported models": standard
 * split-half RoPE only).  The angle at position p = 256a + b is split into
 * two exactly-known parts; each part's cos/sin is evaluated in fp64 and
 * rounded to fp32, then combined with the angle-addition identity in fp32:
 *   c = fmaf(cos A, cos B, -(sin A * sin B)),
 *   s = fmaf(sin A, cos B,  (cos A * sin B)). */
void oq_rope_cs(double theta, int64_t pos, float *c, float *s)
{
    int64_t a = pos >> 8, b = pos & 255;
    for (int i = 0; i < OQ_HALF; i++) {
        double w = pow(theta, -(double)i / 64.0);
        double angA = (double)(256 * a) * w;
        double angB = (double)b * w;
        float ca = (float)cos(angA), sa = (float)sin(angA);
        float cb = (float)cos(angB), sb = (float)sin(angB);
        float ss = sa * sb, cs = ca * sb;
        c[i] = fmaf(ca, cb, -ss);
        s[i] = fmaf(sa, cb, cs);
    }
}

/* Remove the rotation that RoPE applied at this position (rotate by -angle):
 *   u_i    = fmaf(k_i,    c, k_{i+64} * s)
 *   u_i+64 = fmaf(k_i+64, c, -(k_i * s))          (NexusQuant step 3) */
void oq_rope_undo(float *v, const float *c, const float *s)
{
    for (int i = 0; i < OQ_HALF; i++) {
        float a = v[i], b = v[i + OQ_HALF];
        float bs = b * s[i], as = a * s[i];
        v[i] = fmaf(a, c[i], bs);
        v[i + OQ_HALF] = fmaf(b, c[i], -as);
    }
}

/* Re-apply the rotation after reconstruction (rotate by +angle). */
void oq_rope_redo(float *v, const float *c, const float *s)
{
    for (int i = 0; i < OQ_HALF; i++) {
        float a = v[i], b = v[i + OQ_HALF];
        float bs = b * s[i], as = a * s[i];
        v[i] = fmaf(a, c[i], -bs);
        v[i + OQ_HALF] = fmaf(b, c[i], as);
    }
}

/* ----------------------------------------------------------------- FWHT */

/* Unnormalised Walsh-Hadamard transform in Sylvester (natural) order:
 * stages h = 1, 2, 4, ..., 64, each butterfly (a, b) -> (a + b, a - b).
 * The 1/sqrt(128) normalisation is folded into the scale (NexusQuant
 * step 4: rotate so that no outlier dominates the quantisation scale). */
void oq_fwht128(float *v)
{
    for (int h = 1; h < OQ_D; h <<= 1)
        for (int i = 0; i < OQ_D; i++)
            if (!(i & h)) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

/* ------------------------------------------------------------ E8 decode */

/* Nearest point of D8 + shift (shift 0: D8 = integer vectors with even sum;
 * shift 1/2: D8 + (1/2,...,1/2)), following the Conway-Sloane decoder for
 * D_n: round every coordinate to the nearest integer, and if the sum is odd,
 * re-round the coordinate with the largest rounding error the other way.
 *
 * fp32, in this order:
 *   u_i = y_i - shift                 (rounded; exact for shift 0)
 *   f_i = rint(u_i)                   (nearest, ties to even)
 *   e_i = u_i - f_i                   (exact)
 *   d   = e_0*e_0, then d = fmaf(e_i, e_i, d) for i = 1..7
 *   if sum(f) is odd:
 *     k   = first index of max |e_i|
 *     f_k += (e_k >= 0 ? 1 : -1)
 *     d   = d + fmaf(-2, |e_k|, 1)     (= |e|^2 after the move, since
 *                                      (1-|e_k|)^2 - e_k^2 = 1 - 2|e_k|)
 * Output: g[i] = f_i (the point is g + shift), return value d. */
static float oq_d8_decode(const float *y, float shift, int32_t *g)
{
    float u[8], e[8];
    int32_t f[8];
    int32_t sum = 0;
    for (int i = 0; i < 8; i++) {
        u[i] = y[i] - shift;
        float r = rintf(u[i]);
        e[i] = u[i] - r;
        f[i] = (int32_t)r;
        sum += f[i];
    }
    float d = e[0] * e[0];
    for (int i = 1; i < 8; i++) d = fmaf(e[i], e[i], d);
    if (sum & 1) {
        int k = 0;
        float m = fabsf(e[0]);
        for (int i = 1; i < 8; i++)
            if (fabsf(e[i]) > m) { m = fabsf(e[i]); k = i; }
        f[k] += (e[k] >= 0.0f) ? 1 : -1;
        d = d + fmaf(-2.0f, m, 1.0f);
    }
    for (int i = 0; i < 8; i++) g[i] = f[i];
    return d;
}

/* Nearest E8 point, E8 = D8 u (D8 + 1/2) (Conway-Sloane): decode both cosets
 * and keep the closer; a tie keeps the integer coset.  t[i] = 2*q_i (all even
 * for the integer coset, all odd for the half coset).  Returns the coset
 * (0 integer, 1 half) and the chosen fp32 distance in *dist. */
int oq_e8_nearest(const float *y, int32_t *t, float *dist)
{
    int32_t g0[8], g1[8];
    float d0 = oq_d8_decode(y, 0.0f, g0);
    float d1 = oq_d8_decode(y, 0.5f, g1);
    if (d1 < d0) {
        for (int i = 0; i < 8; i++) t[i] = 2 * g1[i] + 1;
        if (dist) *dist = d1;
        return 1;
    }
    for (int i = 0; i < 8; i++) t[i] = 2 * g0[i];
    if (dist) *dist = d0;
    return 0;
}

/* ---------------------------------------------- E8 within the code box
 * The nearest point of E8 restricted to the b-bit code box, this library's
 * parity-preserving reading of the clamp, which the exact (coset bit folded)
 * packing below needs.  The pages give no clamp rule; the encoder's own rule
 * (nearest E8 point, then each 2q clamped) can leave E8 when it clamps.
 * Box: the integer coset q in [-(2^(b-1) - 1), 2^(b-1) - 1], the half coset
 * q in [-(2^(b-1) - 1/2), 2^(b-1) - 1/2] (the code ranges of oq_code).
 * Per coset (shift 0 or 1/2, f = q - shift integers in [lo, hi]): each
 * coordinate takes f = clamp(rint(u), lo, hi) (u = y - shift, ties to even),
 * e = u - f; an odd sum of f moves the one coordinate whose move to the
 * nearest in-range value of the other parity (toward u when that is in
 * range, else away) costs least, cost (e - dir)^2 - e^2 = 1 - 2 dir e, the
 * first index on ties.  The costs are separable and non-negative, so this is
 * the nearest point of the coset inside the box (Conway-Sloane's D8 step
 * with the box).  Distance: e0^2 then an fmaf chain, plus the move's cost;
 * the half coset wins only when strictly closer.  When the unconstrained
 * decoder's point lies in the box, this returns the same point. */
static float oq_d8_box_decode(const float *y, float shift, int32_t lo, int32_t hi, int32_t *g)
{
    float u[8], e[8];
    int32_t f[8];
    int32_t sum = 0;
    for (int i = 0; i < 8; i++) {
        u[i] = y[i] - shift;
        int32_t r = (int32_t)rintf(u[i]);
        f[i] = r < lo ? lo : (r > hi ? hi : r);
        e[i] = u[i] - (float)f[i];
        sum += f[i];
    }
    float d = e[0] * e[0];
    for (int i = 1; i < 8; i++) d = fmaf(e[i], e[i], d);
    if (sum & 1) {
        int k = -1, kdir = 0;
        float best = 0.0f;
        for (int i = 0; i < 8; i++) {
            int32_t dir = (e[i] >= 0.0f) ? 1 : -1;
            if (f[i] + dir > hi || f[i] + dir < lo) dir = -dir;
            float cost = fmaf(-2.0f * (float)dir, e[i], 1.0f);
            if (k < 0 || cost < best) {
                best = cost;
                k = i;
                kdir = dir;
            }
        }
        f[k] += kdir;
        d = d + best;
    }
    for (int i = 0; i < 8; i++) g[i] = f[i];
    return d;
}

/* Box-constrained nearest E8 point: t[i] = 2 q_i; returns the coset (0
 * integer, 1 half), the fp32 distance in *dist. */
int oq_e8_box_nearest(const float *y, int bits, int32_t *t, float *dist)
{
    int32_t g0[8], g1[8];
    int32_t h = 1 << (bits - 1);
    float d0 = oq_d8_box_decode(y, 0.0f, -(h - 1), h - 1, g0);
    float d1 = oq_d8_box_decode(y, 0.5f, -h, h - 1, g1);
    const int half = d1 < d0; /* the half coset only when strictly closer */
    for (int i = 0; i < 8; i++) t[i] = half ? 2 * g1[i] + 1 : 2 * g0[i];
    if (dist) *dist = half ? d1 : d0;
    return half;
}

/* Exact packing of one group of a box-constrained point.  The codes are
 * j = q + 2^(b-1) - 1 (integer coset) and j = (q - 1/2) + 2^(b-1) (half
 * coset); a point of E8 has sum q even (integer coset) or sum (q - 1/2) even
 * (half coset: D8 + 1/2), so sum j is even in both, the low bit of j_7 is the
 * parity of j_0 .. j_6, and its place carries the coset bit:
 * bits [b i, b i + b) hold j_i for i < 7, bit 7b the coset, bits
 * [7b + 1, 8b) the high bits of j_7. */
uint32_t oq_exact_pack_group(const uint32_t *j, int half, int bits)
{
    uint32_t w = 0;
    for (int i = 0; i < 7; i++) w |= j[i] << (bits * i);
    w |= ((j[7] & ~1u) | (uint32_t)(half & 1)) << (7 * bits);
    return w;
}

void oq_exact_unpack_group(uint32_t w, int bits, uint32_t *j, int *half)
{
    uint32_t mask = (1u << bits) - 1u, par = 0;
    for (int i = 0; i < 7; i++) {
        j[i] = (w >> (bits * i)) & mask;
        par ^= j[i] & 1u;
    }
    uint32_t last = (w >> (7 * bits)) & mask;
    *half = (int)(last & 1u);
    j[7] = (last & ~1u) | par;
}

/* Batch: box-constrained codes of n groups of 8 (codes packed plainly, code
 * i at bits [b i, b i + b)), coset flags and distances. */
void oq_e8_box_code_batch(const float *y, int64_t n, int bits, uint32_t *codes, int32_t *coset,
                          float *dist)
{
    for (int64_t g = 0; g < n; g++) {
        int32_t t[8];
        float d;
        int half = oq_e8_box_nearest(y + 8 * g, bits, t, &d);
        const int32_t offs = half ? (1 << bits) - 1 : (1 << bits) - 2; /* the code range */
        uint32_t w = 0;
        for (int i = 0; i < 8; i++) w |= (uint32_t)((t[i] + offs) / 2) << (bits * i);
        codes[g] = w;
        coset[g] = half;
        dist[g] = d;
    }
}

/* Clamp 2q to the b-bit symmetric code range and return the code:
 *   half coset (t odd):     t in [-(2^b-1), 2^b-1],  j = (t + 2^b - 1)/2
 *   integer coset (t even): t in [-(2^b-2), 2^b-2],  j = (t + 2^b - 2)/2
 * Sets *clamped when t had to move. */
static uint32_t oq_code(int32_t t, int half, int bits, int *clamped)
{
    int32_t lim = (1 << bits) - (half ? 1 : 2);
    int32_t tc = t < -lim ? -lim : (t > lim ? lim : t);
    if (tc != t) *clamped += 1;
    return (uint32_t)((tc + lim) / 2);
}

/* The b-bit code of coordinate c sits at bits [b*c, b*c + b) of a vector's
 * little-endian stream of 32-bit words. */
static uint32_t oq_get_code(const uint32_t *words, int bits, int c)
{
    uint32_t j = 0;
    int bitpos = bits * c;
    for (int k = 0; k < bits; k++)
        j |= ((words[(bitpos + k) >> 5] >> ((bitpos + k) & 31)) & 1u) << k;
    return j;
}

static void oq_put_code(uint32_t *words, int bits, int c, uint32_t j)
{
    int bitpos = bits * c;
    for (int k = 0; k < bits; k++)
        if (j & (1u << k)) words[(bitpos + k) >> 5] |= 1u << ((bitpos + k) & 31);
}

/* --------------------------------------------------------------- encode */

/* Encode one 128-vector (NexusQuant steps 3-5 plus packing):
 *  1. bf16 -> fp32; for keys, undo RoPE at this position (c, s given).
 *  2. unnormalised FWHT-128.
 *  3. M = max|v|; sigma = fp16(fp32(M * G_b)), saturated at 65504;
 *     r = fp32(C / sigma) (0 when sigma is 0); y_i = fp32(v_i * r), with a
 *     zero product taken as +0.
 *  4. each group of 8 consecutive coordinates -> nearest E8 point -> codes.
 *  5. pack: the b-bit code of coordinate c sits at bits [b*c, b*c + b) of the
 *     vector's little-endian stream of 4*b 32-bit words; meta word =
 *     coset mask (bit g = group g in the half coset) | fp16(sigma) << 16.
 * Returns the number of clamped coordinates.  With box set, step 4 takes the
 * nearest E8 point inside the code box instead (oq_e8_box_nearest; nothing
 * is clamped then). */
static int oq_encode_vector_mode(const uint16_t *x, int rope, const float *c, const float *s,
                                 int bits, int box, uint32_t *words, uint32_t *meta)
{
    float v[OQ_D];
    for (int i = 0; i < OQ_D; i++) v[i] = oq_bf16_to_f32(x[i]);
    if (rope) oq_rope_undo(v, c, s);
    oq_fwht128(v);

    float M = 0.0f;
    for (int i = 0; i < OQ_D; i++) M = fmaxf(M, fabsf(v[i]));
    float G = oq_u2f(bits == 3 ? OQ_G3_BITS : OQ_G2_BITS);
    float C = oq_u2f(OQ_C_BITS);
    float sm = M * G;
    if (sm > 65504.0f) sm = 65504.0f;
    uint16_t sig16 = oq_f32_to_f16(sm);
    float sig = oq_f16_to_f32(sig16);
    float r = (sig == 0.0f) ? 0.0f : C / sig;

    int nw = 4 * bits, clamped = 0;
    for (int w = 0; w < nw; w++) words[w] = 0;
    uint32_t cmask = 0;
    for (int g = 0; g < 16; g++) {
        float y[8];
        for (int i = 0; i < 8; i++) {
            float p = v[8 * g + i] * r;
            y[i] = (p == 0.0f) ? 0.0f : p;
        }
        int32_t t[8];
        int half = box ? oq_e8_box_nearest(y, bits, t, NULL) : oq_e8_nearest(y, t, NULL);
        if (half) cmask |= 1u << g;
        for (int i = 0; i < 8; i++)
            oq_put_code(words, bits, 8 * g + i, oq_code(t[i], half, bits, &clamped));
    }
    *meta = cmask | ((uint32_t)sig16 << 16);
    return clamped;
}

int oq_encode_vector(const uint16_t *x, int rope, const float *c, const float *s,
                     int bits, uint32_t *words, uint32_t *meta)
{
    return oq_encode_vector_mode(x, rope, c, s, bits, 0, words, meta);
}

int oq_encode_vector_box(const uint16_t *x, int rope, const float *c, const float *s,
                         int bits, uint32_t *words, uint32_t *meta)
{
    return oq_encode_vector_mode(x, rope, c, s, bits, 1, words, meta);
}

/* The exact layout of a vector of box-constrained points from the regular one:
 * group g's codes occupy bits [8b g, 8b g + 8b) of the vector's words in both;
 * the exact layout holds the coset bit h_g where the regular one holds the low
 * bit of j_{8g+7} (the parity of j_{8g} .. j_{8g+6} for a point of E8), and of
 * the meta word it keeps only sigma. */
void oq_fold_exact(const uint32_t *words, uint32_t meta, int bits, uint32_t *out,
                   uint16_t *sig16)
{
    for (int w = 0; w < 4 * bits; w++) out[w] = words[w];
    for (int g = 0; g < 16; g++) {
        int pos = bits * (8 * g + 7);
        uint32_t h = (meta >> g) & 1u;
        out[pos >> 5] = (out[pos >> 5] & ~(1u << (pos & 31))) | (h << (pos & 31));
    }
    *sig16 = (uint16_t)(meta >> 16);
}

void oq_unfold_exact(const uint32_t *in, uint16_t sig16, int bits, uint32_t *words,
                     uint32_t *meta)
{
    uint32_t cmask = 0;
    for (int w = 0; w < 4 * bits; w++) words[w] = in[w];
    for (int g = 0; g < 16; g++) {
        int pos = bits * (8 * g + 7);
        cmask |= ((in[pos >> 5] >> (pos & 31)) & 1u) << g;
        uint32_t par = 0;
        for (int i = 0; i < 7; i++) par ^= oq_get_code(words, bits, 8 * g + i) & 1u;
        words[pos >> 5] = (words[pos >> 5] & ~(1u << (pos & 31))) | (par << (pos & 31));
    }
    *meta = cmask | ((uint32_t)sig16 << 16);
}

/* --------------------------------------------------------------- decode */

/* Inverse of oq_encode_vector:
 *  t_c = 2 j_c - 2^b + 2 - h_g   (h_g = coset bit of the group, t_c = 2 q_c)
 *  w   = FWHT(t)                 (integers, |w| <= 896: exact in fp32)
 *  kappa = fp32(fp32(sigma / 2) * C);  x_c = fp32(w_c * kappa)
 *  keys: re-apply RoPE at this position; then bf16 round-to-nearest-even. */
/* The fp32 reconstruction of one packed vector, before the bf16 rounding of
 * the decode output: codes -> 2q -> Walsh-Hadamard -> x = fp32(w * kappa),
 * keys re-rotated (RoPE at the (c, s) row given). */
void oq_reconstruct_vector(const uint32_t *words, uint32_t meta, int rope, const float *c,
                           const float *s, int bits, float *w)
{
    for (int cidx = 0; cidx < OQ_D; cidx++) {
        uint32_t j = oq_get_code(words, bits, cidx);
        int h = (meta >> (cidx >> 3)) & 1u;
        int32_t t = 2 * (int32_t)j - (1 << bits) + 2 - h;
        w[cidx] = (float)t;
    }
    oq_fwht128(w);
    float sig = oq_f16_to_f32((uint16_t)(meta >> 16));
    float kappa = (sig * 0.5f) * oq_u2f(OQ_C_BITS);
    for (int i = 0; i < OQ_D; i++) w[i] = w[i] * kappa;
    if (rope) oq_rope_redo(w, c, s);
}

void oq_decode_vector(const uint32_t *words, uint32_t meta, int rope, const float *c,
                      const float *s, int bits, uint16_t *out)
{
    float w[OQ_D];
    oq_reconstruct_vector(words, meta, rope, c, s, bits, w);
    for (int i = 0; i < OQ_D; i++) out[i] = oq_f32_to_bf16(w[i]);
}

/* ---------------------------------------------------------------- score */

/* Key-key proxy importance (NexusQuant "Implementation details": fast
 * key-key proxy; dev.to step 1: cross-head inner product), on the stored
 * (RoPE'd) keys of one layer K[h][t][d] (bf16, contiguous):
 *   m[h][d]  = fp32( (sum over t in [T-W, T) of K[h][t][d], fp64, t rising) / W )
 *   score[t] = sum over h, then d, of (double)K[h][t][d] * (double)m[h][d] */
void oq_score(const uint16_t *K, int H, int T, int W, double *score, float *mean_out)
{
    float *m = (float *)malloc(sizeof(float) * (size_t)H * OQ_D);
    for (int h = 0; h < H; h++)
        for (int d = 0; d < OQ_D; d++) {
            double S = 0.0;
            for (int t = T - W; t < T; t++)
                S += (double)oq_bf16_to_f32(K[((size_t)h * T + t) * OQ_D + d]);
            m[h * OQ_D + d] = (float)(S / (double)W);
        }
    for (int t = 0; t < T; t++) {
        double acc = 0.0;
        for (int h = 0; h < H; h++)
            for (int d = 0; d < OQ_D; d++)
                acc += (double)oq_bf16_to_f32(K[((size_t)h * T + t) * OQ_D + d]) *
                       (double)m[h * OQ_D + d];
        score[t] = acc;
    }
    if (mean_out) memcpy(mean_out, m, sizeof(float) * (size_t)H * OQ_D);
    free(m);
}

/* --------------------------------------------------------------- select */

/* Kept-token count: always BOS and the last W tokens (NexusQuant "Token
 * eviction"); of the T-1-W middle tokens, floor(T_mid * pct / 100) are
 * evicted.  Everything is kept when T <= 1 + W or pct == 0. */
int64_t oq_kept_count(int64_t T, int64_t W, int pct)
{
    if (T <= 1 + W || pct <= 0) return T;
    int64_t mid = T - 1 - W;
    return T - (mid * pct) / 100;
}

typedef struct { double s; int32_t t; } oq_pair;

static int oq_pair_cmp(const void *pa, const void *pb)
{
    const oq_pair *a = (const oq_pair *)pa, *b = (const oq_pair *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->t > b->t) - (a->t < b->t);
}

/* Kept positions in ascending order: 0, the top n_mid middle positions by
 * (score descending, position ascending), and [T-W, T).  Returns n. */
int64_t oq_select(const double *score, int64_t T, int64_t W, int pct, int32_t *kept)
{
    int64_t n = oq_kept_count(T, W, pct);
    if (n == T) {
        for (int64_t t = 0; t < T; t++) kept[t] = (int32_t)t;
        return T;
    }
    int64_t mid = T - 1 - W, n_mid = n - 1 - W;
    oq_pair *p = (oq_pair *)malloc(sizeof(oq_pair) * (size_t)mid);
    for (int64_t i = 0; i < mid; i++) {
        double s = score[1 + i];
        p[i].s = (s == 0.0) ? 0.0 : s; /* -0 and +0 compare equal anyway */
        p[i].t = (int32_t)(1 + i);
    }
    qsort(p, (size_t)mid, sizeof(oq_pair), oq_pair_cmp);
    uint8_t *flag = (uint8_t *)calloc((size_t)T, 1);
    flag[0] = 1;
    for (int64_t i = 0; i < n_mid; i++) flag[p[i].t] = 1;
    for (int64_t t = T - W; t < T; t++) flag[t] = 1;
    int64_t k = 0;
    for (int64_t t = 0; t < T; t++)
        if (flag[t]) kept[k++] = (int32_t)t;
    free(flag);
    free(p);
    return k;
}

/* ------------------------------------------------------ unit-level driver */

/* Encode n slots of one (layer) unit.  K/V are [H][T_in][128] bf16
 * (contiguous; either may be NULL).  Slot i reads input token
 * src = kept ? kept[i] : i, at RoPE position pos_base + src, and writes
 * codes[h][i][4*bits] / meta[h][i].  Returns the clamp count. */
int64_t oq_encode_unit(const uint16_t *K, const uint16_t *V, int H, int64_t T_in, int64_t n,
                       const int32_t *kept, int64_t pos_base, double theta, int bits_k,
                       int bits_v, uint32_t *k_codes, uint32_t *k_meta, uint32_t *v_codes,
                       uint32_t *v_meta)
{
    int64_t clamped = 0;
    float c[OQ_HALF], s[OQ_HALF];
    for (int64_t i = 0; i < n; i++) {
        int64_t src = kept ? kept[i] : i;
        if (K) oq_rope_cs(theta, pos_base + src, c, s);
        for (int h = 0; h < H; h++) {
            size_t vec = (size_t)h * n + (size_t)i;
            if (K)
                clamped += oq_encode_vector(K + ((size_t)h * T_in + src) * OQ_D, 1, c, s, bits_k,
                                            k_codes + vec * 4 * bits_k, k_meta + vec);
            if (V)
                clamped += oq_encode_vector(V + ((size_t)h * T_in + src) * OQ_D, 0, c, s, bits_v,
                                            v_codes + vec * 4 * bits_v, v_meta + vec);
        }
    }
    return clamped;
}

/* Decode n slots of one unit into K_out/V_out [H][n][128] bf16; slot i is at
 * RoPE position pos_base + (positions ? positions[i] : i). */
void oq_decode_unit(const uint32_t *k_codes, const uint32_t *k_meta, const uint32_t *v_codes,
                    const uint32_t *v_meta, int H, int64_t n, const int32_t *positions,
                    int64_t pos_base, double theta, int bits_k, int bits_v, uint16_t *K_out,
                    uint16_t *V_out)
{
    float c[OQ_HALF], s[OQ_HALF];
    for (int64_t i = 0; i < n; i++) {
        int64_t pos = pos_base + (positions ? (int64_t)positions[i] : i);
        if (K_out) oq_rope_cs(theta, pos, c, s);
        for (int h = 0; h < H; h++) {
            size_t vec = (size_t)h * n + (size_t)i;
            if (K_out)
                oq_decode_vector(k_codes + vec * 4 * bits_k, k_meta[vec], 1, c, s, bits_k,
                                 K_out + vec * OQ_D);
            if (V_out)
                oq_decode_vector(v_codes + vec * 4 * bits_v, v_meta[vec], 0, c, s, bits_v,
                                 V_out + vec * OQ_D);
        }
    }
}

/* ------------------------------------------------------ decode attention */

/* Attention of G query heads per KV head over one packed unit (decode phase:
 * one query vector per head).  This is the reading taken for attention on
 * the compressed cache (the pages only say that reconstruction happens inside
 * the attention computation, VQKV "Decoding": rebuild the needed KV pieces on
 * demand within FlashAttention): scaled dot-product softmax attention over the
 * fp32 reconstructions of the n kept tokens, keys re-rotated at their
 * positions.  Query head j attends with KV head j / G.  Everything after the
 * fp32 reconstruction is fp64:
 *   s_t = scale * sum_i q_i k_t,i,  m = max_t s_t,  l = sum_t exp(s_t - m),
 *   o   = sum_t exp(s_t - m) v_t / l,  lse = m + log(l).
 * q [H*G][128] fp32, out [H*G][128] fp64, lse [H*G] fp64.  Codes/meta are
 * [H][n] vectors as in oq_decode_unit.  n >= 1. */
void oq_attend_unit(const uint32_t *k_codes, const uint32_t *k_meta, const uint32_t *v_codes,
                    const uint32_t *v_meta, int H, int G, int64_t n, const int32_t *positions,
                    int64_t pos_base, double theta, int bits_k, int bits_v, const float *q,
                    double scale, double *out, double *lse)
{
    float c[OQ_HALF], sn[OQ_HALF], k[OQ_D], v[OQ_D];
    double *sc = (double *)malloc((size_t)n * (size_t)G * sizeof(double));
    for (int h = 0; h < H; h++) {
        for (int64_t t = 0; t < n; t++) {
            int64_t pos = pos_base + (positions ? (int64_t)positions[t] : t);
            size_t vec = (size_t)h * n + (size_t)t;
            oq_rope_cs(theta, pos, c, sn);
            oq_reconstruct_vector(k_codes + vec * 4 * bits_k, k_meta[vec], 1, c, sn, bits_k, k);
            for (int g = 0; g < G; g++) {
                const float *qj = q + (size_t)(h * G + g) * OQ_D;
                double dot = 0.0;
                for (int i = 0; i < OQ_D; i++) dot += (double)qj[i] * (double)k[i];
                sc[(size_t)t * G + g] = scale * dot;
            }
        }
        for (int g = 0; g < G; g++) {
            double m = -INFINITY, l = 0.0, acc[OQ_D];
            for (int64_t t = 0; t < n; t++) m = fmax(m, sc[(size_t)t * G + g]);
            for (int i = 0; i < OQ_D; i++) acc[i] = 0.0;
            for (int64_t t = 0; t < n; t++) {
                size_t vec = (size_t)h * n + (size_t)t;
                double p = exp(sc[(size_t)t * G + g] - m);
                l += p;
                oq_reconstruct_vector(v_codes + vec * 4 * bits_v, v_meta[vec], 0, c, sn, bits_v, v);
                for (int i = 0; i < OQ_D; i++) acc[i] += p * (double)v[i];
            }
            for (int i = 0; i < OQ_D; i++) out[(size_t)(h * G + g) * OQ_D + i] = acc[i] / l;
            lse[h * G + g] = m + log(l);
        }
    }
    free(sc);
}

/* fp32 reconstructions of a batch of vectors (keys: rope = 1 with c, s rows). */
void oq_reconstruct_batch(const uint32_t *words, const uint32_t *meta, int64_t n, int rope,
                          const float *c, const float *s, int bits, float *out)
{
    for (int64_t i = 0; i < n; i++)
        oq_reconstruct_vector(words + 4 * bits * i, meta[i], rope, c + OQ_HALF * i,
                              s + OQ_HALF * i, bits, out + OQ_D * i);
}

/* ------------------------------------------------ helpers for the pins */

/* Batched E8 on [n][8] fp32 groups: t_out [n][8] = 2q, coset_out [n],
 * dist_out [n]. */
void oq_e8_batch(const float *y, int64_t n, int32_t *t_out, int32_t *coset_out, float *dist_out)
{
    for (int64_t i = 0; i < n; i++)
        coset_out[i] = oq_e8_nearest(y + 8 * i, t_out + 8 * i, dist_out + i);
}

/* Batched E8 step with codes: nearest point (oq_e8_nearest), then the clamp
 * and code rule (oq_code); codes_out[i] holds the 8 b-bit codes of group i,
 * code k at bits [b*k, b*k + b). */
void oq_e8_code_batch(const float *y, int64_t n, int bits, uint32_t *codes_out,
                      int32_t *coset_out)
{
    for (int64_t i = 0; i < n; i++) {
        int32_t t[8];
        int clamped = 0;
        int half = oq_e8_nearest(y + 8 * i, t, NULL);
        uint32_t w = 0;
        for (int k = 0; k < 8; k++) w |= oq_code(t[k], half, bits, &clamped) << (bits * k);
        codes_out[i] = w;
        coset_out[i] = half;
    }
}

void oq_fwht_batch(float *v, int64_t n)
{
    for (int64_t i = 0; i < n; i++) oq_fwht128(v + OQ_D * i);
}

void oq_f32_to_f16_batch(const float *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oq_f32_to_f16(x[i]);
}

void oq_f32_to_bf16_batch(const float *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oq_f32_to_bf16(x[i]);
}

void oq_rope_batch(double theta, const int64_t *pos, int64_t n, float *c, float *s)
{
    for (int64_t i = 0; i < n; i++) oq_rope_cs(theta, pos[i], c + OQ_HALF * i, s + OQ_HALF * i);
}

/* Apply undo (dir = -1) or redo (dir = +1) to [n][128] fp32 vectors whose
 * (c, s) rows are given [n][64]. */
void oq_rope_apply_batch(float *v, const float *c, const float *s, int64_t n, int dir)
{
    for (int64_t i = 0; i < n; i++) {
        if (dir < 0) oq_rope_undo(v + OQ_D * i, c + OQ_HALF * i, s + OQ_HALF * i);
        else oq_rope_redo(v + OQ_D * i, c + OQ_HALF * i, s + OQ_HALF * i);
    }
}

/* Encode a batch of vectors with per-vector positions (c, s rows given). */
int64_t oq_encode_batch(const uint16_t *x, int64_t n, int rope, const float *c, const float *s,
                        int bits, uint32_t *words, uint32_t *meta)
{
    int64_t clamped = 0;
    for (int64_t i = 0; i < n; i++)
        clamped += oq_encode_vector(x + OQ_D * i, rope, c + OQ_HALF * i, s + OQ_HALF * i, bits,
                                    words + 4 * bits * i, meta + i);
    return clamped;
}

void oq_decode_batch(const uint32_t *words, const uint32_t *meta, int64_t n, int rope,
                     const float *c, const float *s, int bits, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++)
        oq_decode_vector(words + 4 * bits * i, meta[i], rope, c + OQ_HALF * i, s + OQ_HALF * i,
                         bits, out + OQ_D * i);
}

/* Batches of the box-constrained encoder and of the exact-layout conversions. */
int64_t oq_encode_box_batch(const uint16_t *x, int64_t n, int rope, const float *c,
                            const float *s, int bits, uint32_t *words, uint32_t *meta)
{
    int64_t clamped = 0;
    for (int64_t i = 0; i < n; i++)
        clamped += oq_encode_vector_box(x + OQ_D * i, rope, c + OQ_HALF * i, s + OQ_HALF * i, bits,
                                        words + 4 * bits * i, meta + i);
    return clamped;
}

void oq_fold_exact_batch(const uint32_t *words, const uint32_t *meta, int64_t n, int bits,
                         uint32_t *out, uint16_t *sig16)
{
    for (int64_t i = 0; i < n; i++)
        oq_fold_exact(words + 4 * bits * i, meta[i], bits, out + 4 * bits * i, sig16 + i);
}

void oq_unfold_exact_batch(const uint32_t *in, const uint16_t *sig16, int64_t n, int bits,
                           uint32_t *words, uint32_t *meta)
{
    for (int64_t i = 0; i < n; i++)
        oq_unfold_exact(in + 4 * bits * i, sig16[i], bits, words + 4 * bits * i, meta + i);
}

/* -------------------------------------- decision margins (parity accounting)
 * How near each decision of the encoder lies to its boundary.  The parity rule
 * for the GPU path excuses a mismatch with the oracle only where the oracle's
 * value sits within a small relative distance (1e-5) of the boundary of a
 * decision; these functions give that distance (0 = on the boundary, capped
 * at 1).  They take the decisions exactly as oq_d8_decode, oq_e8_nearest and
 * oq_encode_vector_mode take them.  Per group of 8 scaled coordinates y, for
 * the integer coset (shift 0) and the half coset (shift 1/2), with
 * u = fl32(y - shift), f = rint(u), e = u - f:
 *   rounding      | |e_i| - 1/2 | / (1/2)       (u_i at a rounding tie)
 *   parity move   (m1 - m2) / m1, when sum f is odd, m1 >= m2 the two
 *                 largest |e_i| (which coordinate moves)
 * and between the cosets |d1 - d0| / max(d0, d1) with the fp32 distances of
 * oq_d8_decode.  Per vector, also the scale's fp16 rounding: |P - mid| / P,
 * P = fp32(M * G_b), mid = the midpoint of the two fp16 values around P. */
static double oq_min(double a, double b) { return a < b ? a : b; }

static double oq_coset_margin(const float *y, float shift)
{
    double mg = 1.0, m1 = 0.0, m2 = 0.0;
    int32_t sum = 0;
    for (int i = 0; i < 8; i++) {
        float u = y[i] - shift;
        float f = rintf(u);
        double a = fabs((double)(u - f));
        mg = oq_min(mg, fabs(a - 0.5) / 0.5);
        sum += (int32_t)f;
        if (a > m1) { m2 = m1; m1 = a; }
        else if (a > m2) { m2 = a; }
    }
    if ((sum & 1) && m1 > 0.0) mg = oq_min(mg, (m1 - m2) / m1);
    return mg;
}

double oq_e8_margin(const float *y)
{
    int32_t g[8];
    double d0 = oq_d8_decode(y, 0.0f, g), d1 = oq_d8_decode(y, 0.5f, g);
    double mg = oq_min(oq_coset_margin(y, 0.0f), oq_coset_margin(y, 0.5f));
    double big = d0 > d1 ? d0 : d1;
    if (big > 0.0) mg = oq_min(mg, fabs(d1 - d0) / big);
    return mg;
}

/* Smallest decision margin of the encode of one 128-vector (steps as in
 * oq_encode_vector_mode: RoPE undo for keys, FWHT, scale, then the E8 step
 * per group).  A zero vector (sigma 0) takes no decision: margin 1. */
double oq_encode_margin(const uint16_t *x, int rope, const float *c, const float *s, int bits)
{
    float v[OQ_D];
    for (int i = 0; i < OQ_D; i++) v[i] = oq_bf16_to_f32(x[i]);
    if (rope) oq_rope_undo(v, c, s);
    oq_fwht128(v);
    float M = 0.0f;
    for (int i = 0; i < OQ_D; i++) M = fmaxf(M, fabsf(v[i]));
    float P = M * oq_u2f(bits == 3 ? OQ_G3_BITS : OQ_G2_BITS);
    double mg = 1.0;
    if (P > 65504.0f) P = 65504.0f; /* saturated: the clamp decides, not a rounding */
    else if (P > 0.0f) {
        uint16_t h = oq_f32_to_f16(P);
        double near = oq_f16_to_f32(h);
        double other = (double)P >= near ? oq_f16_to_f32((uint16_t)(h + 1))
                                         : oq_f16_to_f32((uint16_t)(h - 1));
        mg = oq_min(mg, fabs((double)P - 0.5 * (near + other)) / (double)P);
    }
    float sig = oq_f16_to_f32(oq_f32_to_f16(P));
    if (sig == 0.0f) return mg;
    float r = oq_u2f(OQ_C_BITS) / sig;
    for (int g = 0; g < 16; g++) {
        float y[8];
        for (int i = 0; i < 8; i++) {
            float p = v[8 * g + i] * r;
            y[i] = (p == 0.0f) ? 0.0f : p;
        }
        mg = oq_min(mg, oq_e8_margin(y));
    }
    return mg;
}

void oq_encode_margin_batch(const uint16_t *x, int64_t n, int rope, const float *c,
                            const float *s, int bits, double *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oq_encode_margin(x + OQ_D * i, rope, c + OQ_HALF * i, s + OQ_HALF * i, bits);
}

void oq_e8_margin_batch(const float *y, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oq_e8_margin(y + 8 * i);
}

/* ------------------------------------------------- delta + entropy stage */

/* The lattice indices (the b-bit codes) of a packed store, coded the way the
 * NexusQuant pages describe their last step: consecutive tokens give similar
 * lattice indices, so the difference to the previous token is stored and the
 * result compressed ("Implementation details" of the zingnex.cn page; step 6
 * of the dev.to page, which names zstd).  zstd is a third-party library, so
 * the compressor here is range-variant asymmetric numeral systems (rANS,
 * J. Duda, "Asymmetric numeral systems", 2013) with a static frequency table;
 * streams, table rule and word format are the library's reading:
 *
 *   streams  one per (unit, head, segment of OQ_SEG tokens, coordinate c),
 *            in that order (coordinate fastest); symbols
 *            d_t = (j_t - j_{t-1}) mod 2^b inside the segment, d = j at the
 *            segment's first token (or d_t = j_t when the difference is off);
 *   table    per (unit, head), over the symbols of all its streams:
 *            F_s = 0 for an absent symbol, else max(1, floor(count_s M / total))
 *            with M = 4096, and the remainder M - sum F added to the largest F
 *            (the lowest symbol on ties); C_s = sum_{r<s} F_r;
 *   encoder  state x in [2^16, 2^32), starting at 2^16, symbols taken last to
 *            first: if x >= F_s 2^20, emit x mod 2^16 and x = floor(x / 2^16);
 *            then x = floor(x / F_s) M + (x mod F_s) + C_s;
 *   stream   the final state (low 16 bits, high 16 bits), then the emitted
 *            words from the last emitted to the first;
 *   decoder  slot = x mod M; s = the symbol with C_s <= slot < C_s + F_s;
 *            x = F_s floor(x / M) + slot - C_s; if x < 2^16, x = x 2^16 + the
 *            next word. */
#define OQ_ANS_M 4096u
#define OQ_ANS_L 65536u
#define OQ_SEG 2048

void oq_ans_table(const uint64_t *counts, int A, uint16_t *F)
{
    uint64_t total = 0;
    for (int s = 0; s < A; s++) total += counts[s];
    int64_t sum = 0;
    for (int s = 0; s < A; s++) {
        uint64_t f = 0;
        if (counts[s]) {
            f = counts[s] * OQ_ANS_M / total;
            if (f < 1) f = 1;
        }
        F[s] = (uint16_t)f;
        sum += (int64_t)f;
    }
    int best = 0;
    for (int s = 1; s < A; s++)
        if (F[s] > F[best]) best = s;
    F[best] = (uint16_t)((int64_t)F[best] + ((int64_t)OQ_ANS_M - sum));
}

static void oq_ans_cum(const uint16_t *F, int A, uint32_t *C)
{
    C[0] = 0;
    for (int s = 0; s < A; s++) C[s + 1] = C[s] + F[s];
}

/* One stream: returns its length in 16-bit words (written to out[0..len)),
 * -1 when cap words do not suffice, -2 for a symbol of frequency 0. */
int64_t oq_ans_encode(const uint8_t *sym, int64_t count, const uint16_t *F, int A, uint16_t *out,
                      int64_t cap)
{
    uint32_t C[257];
    oq_ans_cum(F, A, C);
    int64_t p = cap; /* emitted words fill out[] from the end */
    uint32_t x = OQ_ANS_L;
    for (int64_t t = count - 1; t >= 0; t--) {
        uint32_t s = sym[t], f = F[s];
        if (f == 0) return -2;
        if ((uint64_t)x >= ((uint64_t)f << 20)) {
            if (p == 0) return -1;
            out[--p] = (uint16_t)(x & 0xFFFFu);
            x >>= 16;
        }
        x = (x / f) * OQ_ANS_M + (x % f) + C[s];
    }
    if (p < 2) return -1;
    out[--p] = (uint16_t)(x >> 16);
    out[--p] = (uint16_t)(x & 0xFFFFu);
    int64_t len = cap - p;
    memmove(out, out + p, (size_t)len * sizeof(uint16_t));
    return len;
}

/* Inverse of oq_ans_encode: count symbols from a stream of len words;
 * returns the words read, -1 if the stream ends early. */
int64_t oq_ans_decode(const uint16_t *in, int64_t len, const uint16_t *F, int A, uint8_t *sym,
                      int64_t count)
{
    uint32_t C[257];
    oq_ans_cum(F, A, C);
    if (len < 2) return -1;
    uint32_t x = (uint32_t)in[0] | ((uint32_t)in[1] << 16);
    int64_t i = 2;
    for (int64_t t = 0; t < count; t++) {
        uint32_t slot = x & (OQ_ANS_M - 1u);
        int s = 0;
        while (s + 1 < A && C[s + 1] <= slot) s++;
        sym[t] = (uint8_t)s;
        x = F[s] * (x >> 12) + slot - C[s];
        if (x < OQ_ANS_L) {
            if (i >= len) return -1;
            x = (x << 16) | in[i++];
        }
    }
    return i;
}

/* Symbols of the stream (segment g, coordinate c) of one (unit, head):
 * codes holds its n vectors of 4*bits words. */
static int64_t oq_stream_symbols(const uint32_t *codes, int64_t n, int bits, int delta, int64_t g,
                                 int c, uint8_t *sym)
{
    int64_t t0 = g * OQ_SEG, t1 = t0 + OQ_SEG < n ? t0 + OQ_SEG : n;
    uint32_t mask = (1u << bits) - 1u, prev = 0;
    for (int64_t t = t0; t < t1; t++) {
        uint32_t j = oq_get_code(codes + 4 * bits * t, bits, c);
        sym[t - t0] = (uint8_t)(delta ? ((j - prev) & mask) : j);
        prev = j;
    }
    return t1 - t0;
}

/* Encode the codes of units x heads x n vectors (codes: [units][heads][n][4 bits]
 * contiguous): freq [units][heads][2^bits], offsets [streams + 1] (stream i
 * occupies words[offsets[i] .. offsets[i+1])).  Returns the total words, -1
 * if cap words do not suffice. */
int64_t oq_entropy_encode_store(const uint32_t *codes, int64_t units, int heads, int64_t n,
                                int bits, int delta, uint16_t *freq, uint32_t *offsets,
                                uint16_t *words, int64_t cap)
{
    int A = 1 << bits;
    int64_t nseg = (n + OQ_SEG - 1) / OQ_SEG, stream = 0, off = 0;
    uint8_t *sym = malloc(OQ_SEG);
    for (int64_t uh = 0; uh < units * heads; uh++) {
        const uint32_t *cu = codes + uh * n * 4 * bits;
        uint64_t counts[8] = {0};
        for (int64_t g = 0; g < nseg; g++)
            for (int c = 0; c < OQ_D; c++) {
                int64_t m = oq_stream_symbols(cu, n, bits, delta, g, c, sym);
                for (int64_t t = 0; t < m; t++) counts[sym[t]]++;
            }
        uint16_t *F = freq + uh * A;
        oq_ans_table(counts, A, F);
        for (int64_t g = 0; g < nseg; g++)
            for (int c = 0; c < OQ_D; c++) {
                int64_t m = oq_stream_symbols(cu, n, bits, delta, g, c, sym);
                int64_t len = oq_ans_encode(sym, m, F, A, words + off, cap - off);
                if (len < 0) {
                    free(sym);
                    return -1;
                }
                offsets[stream++] = (uint32_t)off;
                off += len;
            }
    }
    offsets[stream] = (uint32_t)off;
    free(sym);
    return off;
}

/* Inverse of oq_entropy_encode_store: rebuilds the code words (meta is not
 * part of the streams).  Returns 0, or -1 if a stream is inconsistent. */
int oq_entropy_decode_store(const uint16_t *words, const uint32_t *offsets, const uint16_t *freq,
                            int64_t units, int heads, int64_t n, int bits, int delta,
                            uint32_t *codes)
{
    int A = 1 << bits;
    uint32_t mask = (1u << bits) - 1u;
    int64_t nseg = (n + OQ_SEG - 1) / OQ_SEG, stream = 0;
    uint8_t *sym = malloc(OQ_SEG);
    memset(codes, 0, (size_t)(units * heads * n * 4 * bits) * sizeof(uint32_t));
    for (int64_t uh = 0; uh < units * heads; uh++) {
        uint32_t *cu = codes + uh * n * 4 * bits;
        const uint16_t *F = freq + uh * A;
        for (int64_t g = 0; g < nseg; g++)
            for (int c = 0; c < OQ_D; c++, stream++) {
                int64_t t0 = g * OQ_SEG, t1 = t0 + OQ_SEG < n ? t0 + OQ_SEG : n;
                int64_t len = (int64_t)offsets[stream + 1] - (int64_t)offsets[stream];
                int64_t used = oq_ans_decode(words + offsets[stream], len, F, A, sym, t1 - t0);
                if (used != len) {
                    free(sym);
                    return -1;
                }
                uint32_t j = 0;
                for (int64_t t = t0; t < t1; t++) {
                    j = delta ? ((j + sym[t - t0]) & mask) : sym[t - t0];
                    oq_put_code(cu + 4 * bits * t, bits, c, j);
                }
            }
    }
    free(sym);
    return 0;
}
