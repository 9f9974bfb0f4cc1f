/*
 * hq_oracle.c -- plain, slow CPU oracle of the HyperQuant per-tile codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library) shares no code, header, table or constant with it.
 *
 * Sources, cited by page title and section:
 *   [V1] "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline for
 *        Large Language and Diffusion Models" (mlsanity.com paper page),
 *        section "Abstract (arXiv)", ingredients (i)-(iv).
 *   [V2] "HyperQuant: A Near-Entropy-Optimal Lattice Quantization Pipeline
 *        for Large Language and Diffusion Models" (acceptodds.com ICLR 2027
 *        page), abstract.
 *   [CS82] Conway & Sloane, "Fast quantizing and decoding algorithms for
 *        lattice quantizers and codes", IEEE Trans. IT 28(2), 1982:
 *        nearest point of Z^n, D_n and of a union of cosets.
 *   [SM64] Steele, Lea & Flood, "Fast splittable pseudorandom number
 *        generators", OOPSLA 2014: the SplitMix64 output function.
 *
 * The pages state the pipeline (per-tile random-sign Hadamard rotation,
 * lattice E8/D4/A2/Z, lossless strip of the bits membership fixes, Rice code
 * of the remainder, subtractive dither for the KV cache) but none of its
 * constants, tie rules or the stream layout.  Every such choice below is a
 * stated reading; the same readings are listed, with reasons, in the design
 * notes that ship with the repository.
 *
 * Parity unpinned: the stream layout (hqo_pack_tile / the unpacker) -- no
 * page prints a stream, so it is checked only against layouts worked out by
 * hand from this file's own specification (tests/golden/rice_layout.json)
 * and by round trips, not against anything the pages fix.
 *
 * Precision: every step whose floating-point result decides an integer (the
 * lattice point, the Rice parameter, the stream) runs in IEEE binary32 with
 * round-to-nearest-even, one rounding per operation (compile with
 * -ffp-contract=off, no fast-math).  The decode reconstruction and the GEMV
 * reference run in binary64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define HQO_MAX_TILE 1024

/* status bits shared by encode/decode (values are this oracle's own) */
#define HQO_NONFINITE 1
#define HQO_CAPACITY 2
#define HQO_CORRUPT 4

/* ------------------------------------------------------------------ */
/* Counter-based randomness [SM64]: the pages ask for random signs and a
 * seeded dither without naming a generator; this one is our choice. */

uint64_t hqo_mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

/* H(seed, tag, a, b): three chained mixes of a golden-gamma offset seed. */
uint64_t hqo_hash(uint64_t seed, uint64_t tag, uint64_t a, uint64_t b)
{
    uint64_t h = hqo_mix64(seed + 0x9E3779B97F4A7C15ULL * (tag + 1));
    h = hqo_mix64(h ^ a);
    return hqo_mix64(h ^ b);
}

/* Random sign of coordinate i of column tile j (the random signs of the
 * per-tile Hadamard rotation, [V1] (i), [V2]): bit (i mod 64) of
 * H(seed, 1, j, i / 64), set
 * bit = -1.  Signs depend on the column tile only, so every row of a
 * column tile shares them. */
int hqo_sign(uint64_t seed, uint64_t j, uint32_t i)
{
    uint64_t h = hqo_hash(seed, 1, j, i >> 6);
    return ((h >> (i & 63)) & 1) ? -1 : 1;
}

/* Uniform r_i in [0,1) on the 16-bit grid, for coordinate i of tile t
 * (dither).  One hash serves coordinates 4m .. 4m+3: coordinate 4m + k takes
 * bits 16k .. 16k+15 of H(seed, 2, t, m). */
float hqo_uniform(uint64_t seed, uint64_t t, uint32_t i)
{
    uint64_t h = hqo_hash(seed, 2, t, i >> 2);
    uint32_t r = (uint32_t)((h >> (16 * (i & 3))) & 0xFFFFu);
    return (float)r * 0x1p-16f;
}

/* ------------------------------------------------------------------ */
/* Walsh-Hadamard transform [V1 (i), V2]: unnormalised Sylvester matrix
 * H[a][b] = (-1)^popcount(a & b).  Butterfly stages h = 1, 2, 4, ..., n/2
 * in that order; the pair (a, a+h) with bit h of a clear becomes
 * (v_a + v_{a+h}, v_a - v_{a+h}). */
void hqo_fwht_f32(float *v, int n)
{
    for (int h = 1; h < n; h <<= 1)
        for (int a = 0; a < n; a++)
            if (!(a & h)) {
                float p = v[a], q = v[a + h];
                v[a] = p + q;
                v[a + h] = p - q;
            }
}

void hqo_fwht_f64(double *v, int n)
{
    for (int h = 1; h < n; h <<= 1)
        for (int a = 0; a < n; a++)
            if (!(a & h)) {
                double p = v[a], q = v[a + h];
                v[a] = p + q;
                v[a + h] = p - q;
            }
}

/* ------------------------------------------------------------------ */
/* Per-tile scale for the target rate (the pages name such a scale but give
 * no rule; reading): the high-resolution entropy of a lattice quantizer of
 * cell volume V and step D on i.i.d. N(0, s^2) coordinates is
 * log2(sqrt(2 pi e) s) - log2(D V^(1/d)) bits per dimension; setting it to
 * R gives D = s sqrt(2 pi e) 2^-R V^(-1/d).  With the unnormalised
 * Hadamard transform the rotated coordinates have variance sum_i w_i^2. */

static double cell_volume(int lattice)
{
    switch (lattice) {
    case 8: return 1.0;             /* E8: unimodular */
    case 4: return 2.0;             /* D4: index 2 in Z^4 */
    case 2: return sqrt(3.0) / 2.0; /* A2 with minimal norm 1 */
    default: return 1.0;            /* Z */
    }
}

float hqo_rate_constant(int lattice, float bps)
{
    double c = sqrt(2.0 * M_PI * M_E) * pow(2.0, -(double)bps) *
               pow(cell_volume(lattice), -1.0 / (double)lattice);
    return (float)c;
}

/* sum of squares by a fixed pairwise tree: level l adds the partial sums of
 * indices that differ in bit l (l = 0 first). */
float hqo_sumsq(const float *w, int n)
{
    float a[HQO_MAX_TILE];
    for (int i = 0; i < n; i++) a[i] = w[i] * w[i];
    for (int h = 1; h < n; h <<= 1)
        for (int i = 0; i < n; i++)
            if (!(i & h)) a[i] = a[i] + a[i + h];
    return a[0];
}

/* binary32 -> bfloat16 bit pattern, round to nearest even (finite input) */
static uint16_t bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Delta = bf16(c * sqrt(S)).  A non-finite S marks the tile non-finite;
 * a non-finite tile, a tile with S < 2^-96 (energy so small that squares of
 * its entries underflow, which would let S understate the tile and the
 * rotated coordinates outgrow the payload bound) and a zero or subnormal
 * Delta are all stored as Delta = 0 with all lattice points zero. */
uint16_t hqo_tile_scale(float S, float c, int *nonfinite)
{
    *nonfinite = !isfinite(S);
    if (*nonfinite) return 0;
    if (S < 0x1p-96f) return 0;
    float sigma = sqrtf(S);
    float d32 = c * sigma;
    uint16_t b = bf16_bits(d32);
    if ((b & 0x7F80u) == 0) return 0;
    return b;
}

/* ------------------------------------------------------------------ */
/* Nearest lattice points [CS82].  Each returns the coset bit c (E8, A2;
 * else 0), the integer coordinates z that the stream stores before the
 * strip, and the point itself in binary32.
 *   Z  : points Z;           z = y.
 *   D_n: points of Z^n with even sum; z = y.
 *   E8 : D8 u (D8 + 1/2);    z = y - c/2 (in D8).
 *   A2 : points (a + c/2, (b + c/2) sqrt3);  z = (a, b).
 * Tie rules (reading): rint ties to even; D_n flips the first coordinate of
 * largest |x - rint(x)|, towards x (upwards when x is an integer); A2 keeps
 * the integer coset when the two squared distances are equal.
 *
 * E8 (reading of [CS82]'s two-candidate decoder): with f = rint(x) and
 * e = x - f, the D8 candidate is f with the first coordinate of largest |e|
 * moved towards x when sum(f) is odd.  The D8 + 1/2 candidate starts from the
 * nearest half-integers floor(x) + 1/2 (an integer x goes up): their
 * distances to x are exactly 1/2 - |e_i|, so when sum(floor(x)) is odd the
 * first coordinate of smallest |e| moves towards x (up when its fractional
 * part is at least 1/2).  The squared distances then differ by
 *   d0 - d1 = sum|e| - 2 + [sum f odd](1 - 2 max|e|) - [sum floor odd] 2 min|e|,
 * evaluated in binary32 in that order (|e| summed for i = 0..7); d0 - d1 <= 0
 * keeps the integer coset. */

static void dn_round(const float *x, int d, int32_t *f)
{
    float e[8];
    int32_t sum = 0;
    for (int i = 0; i < d; i++) {
        float r = rintf(x[i]);
        f[i] = (int32_t)r;
        e[i] = x[i] - r;
        sum += f[i];
    }
    if (sum & 1) {
        int b = 0;
        for (int i = 1; i < d; i++)
            if (fabsf(e[i]) > fabsf(e[b])) b = i;
        f[b] += (e[b] >= 0.0f) ? 1 : -1;
    }
}

static float sqdist(const float *x, const float *p, int d)
{
    float s = 0.0f;
    for (int i = 0; i < d; i++) {
        float t = x[i] - p[i];
        s = s + t * t;
    }
    return s;
}

static void e8_nearest(const float *x, int *c, int32_t *z, float *pt)
{
    float e[8], ae[8];
    int32_t f[8], g[8], sf = 0, sg = 0;
    for (int i = 0; i < 8; i++) {
        float r = rintf(x[i]);
        f[i] = (int32_t)r;
        g[i] = (int32_t)floorf(x[i]);
        e[i] = x[i] - r;
        ae[i] = fabsf(e[i]);
        sf += f[i];
        sg += g[i];
    }
    int bmax = 0, bmin = 0;
    for (int i = 1; i < 8; i++) {
        if (ae[i] > ae[bmax]) bmax = i;
        if (ae[i] < ae[bmin]) bmin = i;
    }
    float s = 0.0f;
    for (int i = 0; i < 8; i++) s = s + ae[i];
    float dd = s - 2.0f;
    if (sf & 1) dd = dd + (1.0f - 2.0f * ae[bmax]);
    if (sg & 1) dd = dd - 2.0f * ae[bmin];
    if (dd <= 0.0f) {
        *c = 0;
        for (int i = 0; i < 8; i++) z[i] = f[i];
        if (sf & 1) z[bmax] += (e[bmax] >= 0.0f) ? 1 : -1;
        for (int i = 0; i < 8; i++) pt[i] = (float)z[i];
    } else {
        *c = 1;
        for (int i = 0; i < 8; i++) z[i] = g[i];
        if (sg & 1) z[bmin] += (x[bmin] - (float)g[bmin] >= 0.5f) ? 1 : -1;
        for (int i = 0; i < 8; i++) pt[i] = (float)z[i] + 0.5f;
    }
}

void hqo_nearest(int lattice, const float *x, int *c, int32_t *z, float *pt)
{
    *c = 0;
    if (lattice == 1) {
        float r = rintf(x[0]);
        z[0] = (int32_t)r;
        pt[0] = r;
    } else if (lattice == 4) {
        dn_round(x, 4, z);
        for (int i = 0; i < 4; i++) pt[i] = (float)z[i];
    } else if (lattice == 8) {
        e8_nearest(x, c, z, pt);
    } else { /* A2 */
        const float S3 = (float)sqrt(3.0);
        const float T = (float)(1.0 / sqrt(3.0));
        float y1 = x[1] * T;
        float a0 = rintf(x[0]), b0 = rintf(y1);
        float a1 = rintf(x[0] - 0.5f), b1 = rintf(y1 - 0.5f);
        float p0[2] = { a0, b0 * S3 };
        float p1[2] = { a1 + 0.5f, (b1 + 0.5f) * S3 };
        float d0 = sqdist(x, p0, 2), d1 = sqdist(x, p1, 2);
        if (d0 <= d1) {
            z[0] = (int32_t)a0; z[1] = (int32_t)b0; pt[0] = p0[0]; pt[1] = p0[1];
        } else {
            *c = 1;
            z[0] = (int32_t)a1; z[1] = (int32_t)b1; pt[0] = p1[0]; pt[1] = p1[1];
        }
    }
}

/* ------------------------------------------------------------------ */
/* Subtractive dither for the KV cache [V2].  The pages ask for subtractive
 * dither under an idealised sampler without fixing its law.  Reading: delta
 * is uniform on a box that is a fundamental domain of a sublattice L' of the
 * lattice L -- L' = D_d for E8 and D4 (box [-1/2,1/2)^(d-1) x [-1,1)),
 * Z x sqrt3 Z for A2 ([-1/2,1/2) x sqrt3 [-1/2,1/2)), Z for Z ([-1/2,1/2)).
 * Then delta mod L is uniform, so the error Q(x + delta) - delta - x is
 * uniform on the Voronoi cell and independent of x (the subtractive-dither
 * property) with no nearest-point step in drawing delta.  On the 16-bit
 * grid of the uniforms every value is exact in binary32 except the A2
 * second coordinate, rounded once.  Vector v of tile t. */
void hqo_dither(int lattice, uint64_t seed, uint64_t t, uint32_t v, float *delta)
{
    int d = lattice;
    for (int m = 0; m < d; m++) {
        float r = hqo_uniform(seed, t, v * (uint32_t)d + (uint32_t)m);
        if ((lattice == 8 || lattice == 4) && m == d - 1) delta[m] = 2.0f * r - 1.0f;
        else if (lattice == 2 && m == 1) delta[m] = (r - 0.5f) * (float)sqrt(3.0);
        else delta[m] = r - 0.5f;
    }
}

/* ------------------------------------------------------------------ */
/* Lossless strip and zigzag ([V1] (iii); [V2]: the strip drops what being a
 * lattice point already determines).  Reading: for D-type vectors
 * (D4, and E8 after its coset bit is removed) the coordinate sum is even,
 * so the parity of the last coordinate is implied: it is stored halved
 * (floor).  A2 keeps the coset bit c and its two integers.  Z strips
 * nothing.  Zigzag maps 0,-1,1,-2,... to 0,1,2,3,... */

static int32_t floor_half(int32_t z) { return (z - (z & 1)) / 2; }

static uint32_t zigzag(int32_t z) { return z >= 0 ? 2u * (uint32_t)z : 2u * (uint32_t)(-(int64_t)z) - 1u; }

static int32_t unzigzag(uint32_t u) { return (u & 1) ? -(int32_t)((u + 1) / 2) : (int32_t)(u / 2); }

void hqo_symbols(int lattice, const int32_t *z, uint32_t *u)
{
    int d = lattice;
    for (int i = 0; i < d; i++) {
        int32_t s = z[i];
        if ((lattice == 8 || lattice == 4) && i == d - 1) s = floor_half(z[i]);
        u[i] = zigzag(s);
    }
}

void hqo_unsymbols(int lattice, const uint32_t *u, int32_t *z)
{
    int d = lattice;
    int32_t sum = 0;
    for (int i = 0; i < d; i++) z[i] = unzigzag(u[i]);
    if (lattice == 8 || lattice == 4) {
        for (int i = 0; i < d - 1; i++) sum += z[i];
        z[d - 1] = 2 * z[d - 1] + (sum & 1);
    }
}

/* ------------------------------------------------------------------ */
/* Rice code of what remains after the strip ([V1] (iii), [V2]):
 * code(u, k) = q = floor(u / 2^k) zero bits, one 1 bit, and the k low bits
 * of u; length q + 1 + k.  Per-tile k in [0, 15] minimising the tile's total
 * length, smallest k on ties (brute force over all 16 values). */
uint64_t hqo_rice_cost(const uint32_t *u, int n, int k)
{
    uint64_t s = 0;
    for (int i = 0; i < n; i++) s += (uint64_t)(u[i] >> k) + 1u + (uint64_t)k;
    return s;
}

int hqo_best_k(const uint32_t *u, int n)
{
    int bk = 0;
    uint64_t best = hqo_rice_cost(u, n, 0);
    for (int k = 1; k <= 15; k++) {
        uint64_t c = hqo_rice_cost(u, n, k);
        if (c < best) { best = c; bk = k; }
    }
    return bk;
}

/* Tile stream layout (this build's format; the pages print none).  Bits are
 * numbered LSB-first within little-endian 32-bit words.
 *   [0, C)            coset bit of vector v at bit v (C = n/d for E8, A2)
 *   [C, C + n k)      low k bits of code i at C + i k, LSB first
 *   [C + n k, ...)    unary parts: q_i zero bits then a one bit, i = 0..n-1
 * then zero padding to a whole word.  Same bits as the interleaved Rice
 * code, grouped by kind. */
static int put_bit(uint32_t *w, uint64_t cap_bits, uint64_t pos, int b)
{
    if (pos >= cap_bits) return 0;
    if (b) w[pos >> 5] |= 1u << (pos & 31);
    return 1;
}

static int get_bit(const uint32_t *w, uint64_t pos) { return (int)((w[pos >> 5] >> (pos & 31)) & 1u); }

/* returns the number of words, or -1 if cap_words is too small */
int hqo_pack_tile(int lattice, int n, int k, const uint8_t *coset, const uint32_t *u,
                  uint32_t *words, int cap_words)
{
    uint64_t cap = (uint64_t)cap_words * 32u, pos = 0;
    int d = lattice;
    int nv = n / d;
    memset(words, 0, sizeof(uint32_t) * (size_t)cap_words);
    if (lattice == 8 || lattice == 2)
        for (int v = 0; v < nv; v++)
            if (!put_bit(words, cap, pos++, coset[v])) return -1;
    for (int i = 0; i < n; i++)
        for (int b = 0; b < k; b++)
            if (!put_bit(words, cap, pos++, (int)((u[i] >> b) & 1u))) return -1;
    for (int i = 0; i < n; i++) {
        pos += u[i] >> k;
        if (!put_bit(words, cap, pos++, 1)) return -1;
    }
    return (int)((pos + 31) / 32);
}

/* Parse one tile; 0 on success, HQO_CORRUPT if the words do not hold a
 * canonical tile (a read past the end, a one bit in the padding, or -- when
 * `exact` -- a word count other than ceil(bits / 32); a fixed-rate slot may
 * end in whole words of zero padding). */
static int unpack_words(int lattice, int n, int k, const uint32_t *words, int nwords,
                        uint8_t *coset, uint32_t *u, int exact)
{
    uint64_t end = (uint64_t)nwords * 32u, pos = 0;
    int d = lattice;
    int nv = n / d;
    if (k < 0 || k > 15) return HQO_CORRUPT;
    if (lattice == 8 || lattice == 2) {
        for (int v = 0; v < nv; v++) {
            if (pos >= end) return HQO_CORRUPT;
            coset[v] = (uint8_t)get_bit(words, pos++);
        }
    } else {
        for (int v = 0; v < nv; v++) coset[v] = 0;
    }
    for (int i = 0; i < n; i++) {
        uint32_t low = 0;
        for (int b = 0; b < k; b++) {
            if (pos >= end) return HQO_CORRUPT;
            low |= (uint32_t)get_bit(words, pos++) << b;
        }
        u[i] = low;
    }
    for (int i = 0; i < n; i++) {
        uint32_t q = 0;
        for (;;) {
            if (pos >= end) return HQO_CORRUPT;
            if (get_bit(words, pos++)) break;
            q++;
        }
        if (q > (1u << 16)) return HQO_CORRUPT;
        u[i] |= q << k;
    }
    for (uint64_t p = pos; p < end; p++)
        if (get_bit(words, p)) return HQO_CORRUPT;
    if (exact && (pos + 31) / 32 != (uint64_t)nwords) return HQO_CORRUPT;
    return 0;
}

int hqo_unpack_tile(int lattice, int n, int k, const uint32_t *words, int nwords,
                    uint8_t *coset, uint32_t *u)
{
    return unpack_words(lattice, n, k, words, nwords, coset, u, 1);
}

/* ------------------------------------------------------------------ */
/* Quantize the rotated tile v at the scale with bf16 bits sb (0: all-zero
 * tile): y = Q(v / Delta [+ delta]) per vector, then the strip and zigzag of
 * its integer coordinates into the symbols u. */
static void quantize_tile(const float *v, int n, int lattice, uint16_t sb, uint64_t seed, uint64_t t,
                          int dither, int32_t *z, uint8_t *coset, uint32_t *u)
{
    int d = lattice, nv = n / lattice;
    if (sb == 0) {
        for (int i = 0; i < n; i++) z[i] = 0;
        for (int q = 0; q < nv; q++) coset[q] = 0;
    } else {
        float inv = 1.0f / bf16_to_float(sb);
        for (int q = 0; q < nv; q++) {
            float x[8], pt[8], del[8];
            int c;
            if (dither) hqo_dither(lattice, seed, t, (uint32_t)q, del);
            for (int m = 0; m < d; m++) {
                x[m] = v[q * d + m] * inv;
                if (dither) x[m] = x[m] + del[m];
            }
            hqo_nearest(lattice, x, &c, &z[q * d], pt);
            coset[q] = (uint8_t)c;
        }
    }
    for (int q = 0; q < nv; q++) hqo_symbols(lattice, &z[q * d], &u[q * d]);
}

/* One tile, end to end [V1 (i)-(iv), V2].
 * w: n binary32 inputs (bf16 inputs are widened exactly by the caller).
 * j: column tile (signs), t: tile index (dither).  Outputs the bf16 bits of
 * Delta, k, the words, and optionally the pre-strip integer coordinates
 * z[n] and coset bits c[n/d].  Returns the word count, -1 if cap_words is
 * too small.  *status gets HQO_NONFINITE for a non-finite tile. */
int hqo_encode_tile(const float *w, int n, int lattice, float bps, uint64_t seed,
                    uint64_t j, uint64_t t, int dither, uint16_t *scale_out, uint8_t *k_out,
                    uint32_t *words, int cap_words, int32_t *z_out, uint8_t *c_out, int *status)
{
    float v[HQO_MAX_TILE];
    int32_t z[HQO_MAX_TILE];
    uint32_t u[HQO_MAX_TILE];
    uint8_t coset[HQO_MAX_TILE];
    int nv = n / lattice, nonfinite = 0;

    for (int i = 0; i < n; i++) v[i] = (float)hqo_sign(seed, j, (uint32_t)i) * w[i];
    hqo_fwht_f32(v, n);
    float S = hqo_sumsq(w, n);
    uint16_t sb = hqo_tile_scale(S, hqo_rate_constant(lattice, bps), &nonfinite);
    if (nonfinite) *status |= HQO_NONFINITE;

    quantize_tile(v, n, lattice, sb, seed, t, dither, z, coset, u);
    int k = hqo_best_k(u, n);
    *scale_out = sb;
    *k_out = (uint8_t)k;
    if (z_out) memcpy(z_out, z, sizeof(int32_t) * (size_t)n);
    if (c_out) memcpy(c_out, coset, (size_t)nv);
    return hqo_pack_tile(lattice, n, k, coset, u, words, cap_words);
}

/* Decode one tile into binary64 (before any output rounding):
 * w_hat = s . H(Delta (p - delta)) / n with p the lattice point.
 * Returns 0 or HQO_CORRUPT (output zeroed).  `exact`: the words are the
 * tile's own (variable-rate stream); else a fixed-rate slot. */
static int decode_words(const uint32_t *words, int nwords, int n, int lattice, uint16_t scale,
                        int k, uint64_t seed, uint64_t j, uint64_t t, int dither, double *out, int exact)
{
    uint32_t u[HQO_MAX_TILE];
    uint8_t coset[HQO_MAX_TILE];
    int32_t z[8];
    double v[HQO_MAX_TILE];
    int d = lattice, nv = n / lattice;
    int st = unpack_words(lattice, n, k, words, nwords, coset, u, exact);
    /* the encoder only writes Delta = 0 or a positive, normal, finite bf16 */
    if (scale != 0 && ((scale & 0x8000u) || (scale & 0x7F80u) == 0 || (scale & 0x7F80u) == 0x7F80u))
        st = HQO_CORRUPT;
    if (st) {
        for (int i = 0; i < n; i++) out[i] = 0.0;
        return st;
    }
    double delta_f = (double)bf16_to_float(scale);
    for (int q = 0; q < nv; q++) {
        double p[8];
        float del[8];
        hqo_unsymbols(lattice, &u[q * d], z);
        if (lattice == 2) {
            p[0] = (double)z[0] + 0.5 * coset[q];
            p[1] = ((double)z[1] + 0.5 * coset[q]) * sqrt(3.0);
        } else {
            for (int m = 0; m < d; m++) p[m] = (double)z[m] + 0.5 * coset[q];
        }
        if (dither && scale != 0) {
            hqo_dither(lattice, seed, t, (uint32_t)q, del);
            for (int m = 0; m < d; m++) p[m] -= (double)del[m];
        }
        for (int m = 0; m < d; m++) v[q * d + m] = delta_f * p[m];
    }
    hqo_fwht_f64(v, n);
    for (int i = 0; i < n; i++) out[i] = (double)hqo_sign(seed, j, (uint32_t)i) * v[i] / (double)n;
    return 0;
}

int hqo_decode_tile(const uint32_t *words, int nwords, int n, int lattice, uint16_t scale,
                    int k, uint64_t seed, uint64_t j, uint64_t t, int dither, double *out)
{
    return decode_words(words, nwords, n, lattice, scale, k, seed, j, t, dither, out, 1);
}

/* ------------------------------------------------------------------ */
/* Fixed-rate tiles: compact headers and exact rate control.  The pages
 * quote whole-model ratios that count every bit spent (about 3.9x for the
 * weights, 3.79x for the KV cache at 4 bps: [V1] abstract "End-to-end ...
 * compresses"), and name the per-tile scale as the rate's control.  Reading:
 * every tile gets a slot of S words; its tile offset is then t S and is not
 * stored, k is stored in 4 bits, so a tile's side information is the bf16
 * Delta and k (20 bits).  Delta is searched so that the coded tile fits its
 * slot, which makes the rate exact: (32 S + 20) / n bits per coordinate.
 * The slot holds the same tile layout as a variable-rate tile, followed by
 * zero words up to S.
 *
 * Coded size at the scale with bf16 bits c: C + n (1 + k) + sum(u >> k)
 * with u the tile's symbols at that scale and k their best Rice parameter
 * (C = coset bits).  A scale fits if that size is at most 32 S bits.
 *
 * Search (bf16 bit patterns of positive normal numbers are ordered like the
 * numbers; 128 patterns per octave).  c0 = the closed-form scale at the
 * slot's rate.  Bounds: lo_lim = max(0x0080, c0 - 512), hi_lim = min(0x7F7F,
 * c0 + 512) (four octaves either way).
 *   Predict: one pattern step changes every coordinate's rate by 1/128 bit,
 *             so the size moves by about n / 128 bits per step; from c0's
 *             size b0 the start is s = c0 + floor(128 (b0 - budget) / n),
 *             clamped to [lo_lim, hi_lim] (s = c0 reuses c0's size).
 *   s fits:   step down from s by 1, 2, 4, ... (clamped at lo_lim) while
 *             the candidate fits; the first that does not becomes lo (the
 *             last that fits is hi).  If lo_lim itself fits, the answer is
 *             lo_lim.
 *   otherwise: step up likewise from s (clamped at hi_lim) until a
 *             candidate fits (hi; the last that did not is lo).  If hi_lim
 *             does not fit, the tile is stored as an all-zero tile
 *             (Delta = 0), which always fits a legal slot.
 *   Then bisect: while hi - lo > 1, mid = floor((lo + hi) / 2) replaces hi
 *   if it fits, else lo.  The answer is hi: a fitting scale whose next
 *   smaller bf16 value does not fit (when the search ended by bisection).
 * A tile whose closed-form scale is 0 (non-finite, zero or negligible
 * energy) is the all-zero tile, as in the variable-rate stream. */

/* smallest legal slot: the all-zero tile (k = 0, n one bits, C coset bits) */
int hqo_min_slot_words(int n, int lattice)
{
    int c = (lattice == 8 || lattice == 2) ? n / lattice : 0;
    return (c + n + 31) / 32;
}

/* slot for a total rate of `bps` bits per coordinate including the 20 bits
 * of side information: floor((bps n - 20) / 32), or -1 below the minimum */
int hqo_fixed_slot_words(int n, int lattice, float bps)
{
    double s = floor(((double)bps * (double)n - 20.0) / 32.0);
    if (s < (double)hqo_min_slot_words(n, lattice)) return -1;
    return (int)s;
}

static uint64_t coded_bits(const float *v, int n, int lattice, uint16_t c, uint64_t seed, uint64_t t,
                           int dither)
{
    int32_t z[HQO_MAX_TILE];
    uint32_t u[HQO_MAX_TILE];
    uint8_t coset[HQO_MAX_TILE];
    quantize_tile(v, n, lattice, c, seed, t, dither, z, coset, u);
    uint64_t cb = (lattice == 8 || lattice == 2) ? (uint64_t)(n / lattice) : 0;
    return cb + hqo_rice_cost(u, n, hqo_best_k(u, n));
}

/* The fixed-rate scale search above; *trials counts the sizes evaluated. */
uint16_t hqo_fixed_scale(const float *v, int n, int lattice, uint16_t c0, uint64_t budget_bits,
                         uint64_t seed, uint64_t t, int dither, int *trials)
{
    int tr = 0;
    if (c0 == 0) {
        if (trials) *trials = 0;
        return 0;
    }
    int lo_lim = (int)c0 - 512 > 0x0080 ? (int)c0 - 512 : 0x0080;
    int hi_lim = (int)c0 + 512 < 0x7F7F ? (int)c0 + 512 : 0x7F7F;
    int lo, hi, step = 1;
    tr++;
    uint64_t b0 = coded_bits(v, n, lattice, c0, seed, t, dither);
    int64_t num = 128 * ((int64_t)b0 - (int64_t)budget_bits);
    int64_t shift = num >= 0 ? num / n : -((-num + n - 1) / n); /* floor(num / n) */
    int64_t s64 = (int64_t)c0 + shift;
    int start = s64 < lo_lim ? lo_lim : (s64 > hi_lim ? hi_lim : (int)s64);
    int fits_start;
    if (start == (int)c0) {
        fits_start = b0 <= budget_bits;
    } else {
        tr++;
        fits_start = coded_bits(v, n, lattice, (uint16_t)start, seed, t, dither) <= budget_bits;
    }
    if (fits_start) {
        hi = start;
        for (;;) {
            if (hi == lo_lim) {
                if (trials) *trials = tr;
                return (uint16_t)hi;
            }
            int cand = hi - step > lo_lim ? hi - step : lo_lim;
            tr++;
            if (coded_bits(v, n, lattice, (uint16_t)cand, seed, t, dither) <= budget_bits) {
                hi = cand;
                step *= 2;
            } else {
                lo = cand;
                break;
            }
        }
    } else {
        lo = start;
        for (;;) {
            if (lo == hi_lim) {
                if (trials) *trials = tr;
                return 0;
            }
            int cand = lo + step < hi_lim ? lo + step : hi_lim;
            tr++;
            if (coded_bits(v, n, lattice, (uint16_t)cand, seed, t, dither) <= budget_bits) {
                hi = cand;
                break;
            }
            lo = cand;
            step *= 2;
        }
    }
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        tr++;
        if (coded_bits(v, n, lattice, (uint16_t)mid, seed, t, dither) <= budget_bits) hi = mid;
        else lo = mid;
    }
    if (trials) *trials = tr;
    return (uint16_t)hi;
}

/* Closed-form start of the search: the scale rule at the slot's payload
 * rate 32 S / n less 5/32 bit (about what the Rice code and the coset bits
 * spend over the closed form's entropy on Gaussian tiles, so the search
 * starts a few bf16 steps from its answer), at most 8 bits per coordinate.
 * The start only steers the search; every answer fits the slot. */
float hqo_fixed_start_rate(int n, int slot_words)
{
    double r = 32.0 * (double)slot_words / (double)n - 0.15625;
    return (float)(r < 8.0 ? r : 8.0);
}

/* One fixed-rate tile: fills all slot_words words of `slot` (the tile, then
 * zeros).  Returns the tile's own word count, -1 if the slot is below the
 * minimum.  *status gets HQO_NONFINITE for a non-finite tile. */
int hqo_encode_tile_fixed(const float *w, int n, int lattice, int slot_words, uint64_t seed, uint64_t j,
                          uint64_t t, int dither, uint16_t *scale_out, uint8_t *k_out, uint32_t *slot,
                          int *trials, int *status)
{
    float v[HQO_MAX_TILE];
    int32_t z[HQO_MAX_TILE];
    uint32_t u[HQO_MAX_TILE];
    uint8_t coset[HQO_MAX_TILE];
    int nonfinite = 0;
    if (slot_words < hqo_min_slot_words(n, lattice)) return -1;

    for (int i = 0; i < n; i++) v[i] = (float)hqo_sign(seed, j, (uint32_t)i) * w[i];
    hqo_fwht_f32(v, n);
    float S = hqo_sumsq(w, n);
    float c = hqo_rate_constant(lattice, hqo_fixed_start_rate(n, slot_words));
    uint16_t c0 = hqo_tile_scale(S, c, &nonfinite);
    if (nonfinite) *status |= HQO_NONFINITE;
    uint16_t sb = hqo_fixed_scale(v, n, lattice, c0, 32u * (uint64_t)slot_words, seed, t, dither, trials);

    quantize_tile(v, n, lattice, sb, seed, t, dither, z, coset, u);
    int k = hqo_best_k(u, n);
    *scale_out = sb;
    *k_out = (uint8_t)k;
    return hqo_pack_tile(lattice, n, k, coset, u, slot, slot_words);
}

/* Tiles [t0, t1) of a matrix (as in hqo_encode_tiles) into consecutive
 * slots; trials[t - t0] gets each tile's search length. */
int hqo_encode_tiles_fixed(const void *x, int dtype, int64_t cols, int n, int lattice, int slot_words,
                           uint64_t seed, int dither, int64_t t0, int64_t t1, uint32_t *slots,
                           uint16_t *scale, uint8_t *kk, int32_t *trials)
{
    float w[HQO_MAX_TILE];
    int64_t tpr = cols / n;
    int status = 0;
    for (int64_t t = t0; t < t1; t++) {
        int64_t r = t / tpr, j = t % tpr;
        int64_t base = r * cols + j * n;
        for (int i = 0; i < n; i++) {
            if (dtype == 0) w[i] = bf16_to_float(((const uint16_t *)x)[base + i]);
            else w[i] = ((const float *)x)[base + i];
        }
        int tr = 0;
        int nw = hqo_encode_tile_fixed(w, n, lattice, slot_words, seed, (uint64_t)j, (uint64_t)t, dither,
                                       &scale[t - t0], &kk[t - t0], slots + (t - t0) * (int64_t)slot_words,
                                       &tr, &status);
        if (nw < 0) return -1;
        trials[t - t0] = tr;
    }
    return status;
}

/* Decode tiles [t0, t1) of a fixed-rate stream: tile t is words
 * [t S, t S + S) of the payload (cap words), k[t] unpacked by the caller. */
int hqo_decode_tiles_fixed(const uint32_t *payload, uint64_t cap, int slot_words, const uint16_t *scale,
                           const uint8_t *kk, int64_t cols, int n, int lattice, uint64_t seed, int dither,
                           int64_t t0, int64_t t1, double *out)
{
    int64_t tpr = cols / n;
    int status = 0;
    for (int64_t t = t0; t < t1; t++) {
        int64_t r = t / tpr, j = t % tpr;
        if ((uint64_t)(t + 1) * (uint64_t)slot_words > cap) {
            for (int i = 0; i < n; i++) out[r * cols + j * n + i] = 0.0;
            status |= HQO_CORRUPT;
            continue;
        }
        status |= decode_words(payload + t * (int64_t)slot_words, slot_words, n, lattice, scale[t], kk[t], seed,
                               (uint64_t)j, (uint64_t)t, dither, out + r * cols + j * n, 0);
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* Whole matrices, tile by tile.  x is row-major rows x cols, dtype 0 =
 * bf16 bit patterns (uint16), 1 = binary32.  Tile t = r (cols/n) + j covers
 * x[r][j n .. j n + n).  Tiles [t0, t1) are encoded into fixed slots of
 * slot_words words each: words for tile t start at slots + (t - t0) slot_words
 * and their count goes to nwords[t - t0].  The caller forms the offsets
 * (an exclusive prefix sum of nwords) and the payload (the slots
 * concatenated); the prefix sum is the format's only cross-tile step. */
int hqo_encode_tiles(const void *x, int dtype, int64_t rows, int64_t cols, int n, int lattice,
                     float bps, uint64_t seed, int dither, int64_t t0, int64_t t1,
                     uint32_t *slots, int slot_words, int32_t *nwords, uint16_t *scale,
                     uint8_t *kk)
{
    float w[HQO_MAX_TILE];
    int64_t tpr = cols / n;
    int status = 0;
    (void)rows;
    for (int64_t t = t0; t < t1; t++) {
        int64_t r = t / tpr, j = t % tpr;
        int64_t base = r * cols + j * n;
        for (int i = 0; i < n; i++) {
            if (dtype == 0) w[i] = bf16_to_float(((const uint16_t *)x)[base + i]);
            else w[i] = ((const float *)x)[base + i];
        }
        int nw = hqo_encode_tile(w, n, lattice, bps, seed, (uint64_t)j, (uint64_t)t, dither,
                                 &scale[t - t0], &kk[t - t0], slots + (t - t0) * (int64_t)slot_words,
                                 slot_words, NULL, NULL, &status);
        if (nw < 0) return -1;
        nwords[t - t0] = nw;
    }
    return status;
}

/* Decode tiles [t0, t1) of a stream given its offsets (off[t] .. off[t+1]
 * are the words of tile t, all below cap) into out (binary64, row-major
 * rows x cols, only the decoded tiles are written).  A tile whose offsets
 * are out of order or past cap is corrupt.  Returns the OR of tile
 * statuses. */
int hqo_decode_tiles(const uint32_t *payload, uint64_t cap, const uint32_t *off,
                     const uint16_t *scale, const uint8_t *kk, int64_t rows, int64_t cols, int n,
                     int lattice, uint64_t seed, int dither, int64_t t0, int64_t t1, double *out)
{
    int64_t tpr = cols / n;
    int status = 0;
    (void)rows;
    for (int64_t t = t0; t < t1; t++) {
        int64_t r = t / tpr, j = t % tpr;
        int nw = (off[t + 1] >= off[t] && off[t + 1] <= cap) ? (int)(off[t + 1] - off[t]) : -1;
        if (nw < 0) {
            for (int i = 0; i < n; i++) out[r * cols + j * n + i] = 0.0;
            status |= HQO_CORRUPT;
            continue;
        }
        status |= hqo_decode_tile(payload + off[t], nw, n, lattice, scale[t], kk[t], seed,
                                  (uint64_t)j, (uint64_t)t, dither, out + r * cols + j * n);
    }
    return status;
}

/* GEMV reference: y_r = sum_c w_hat[r][c] x[c], in binary64, from the
 * binary64 decode of rows [r0, r1). */
int hqo_gemv_rows(const uint32_t *payload, uint64_t cap, const uint32_t *off, const uint16_t *scale,
                  const uint8_t *kk, int64_t rows, int64_t cols, int n, int lattice, uint64_t seed,
                  const double *x, int64_t r0, int64_t r1, double *y)
{
    int64_t tpr = cols / n;
    int status = 0;
    double *row = (double *)malloc(sizeof(double) * (size_t)cols);
    if (!row) return -1;
    (void)rows;
    for (int64_t r = r0; r < r1; r++) {
        for (int64_t j = 0; j < tpr; j++) {
            int64_t t = r * tpr + j;
            int nw = (off[t + 1] >= off[t] && off[t + 1] <= cap) ? (int)(off[t + 1] - off[t]) : -1;
            if (nw < 0) {
                for (int i = 0; i < n; i++) row[j * n + i] = 0.0;
                status |= HQO_CORRUPT;
                continue;
            }
            status |= hqo_decode_tile(payload + off[t], nw, n, lattice, scale[t], kk[t], seed,
                                      (uint64_t)j, (uint64_t)t, 0, row + j * n);
        }
        double acc = 0.0;
        for (int64_t c = 0; c < cols; c++) acc += row[c] * x[c];
        y[r - r0] = acc;
    }
    free(row);
    return status;
}

/* ------------------------------------------------------------------ */
/* Integer tensor-core product ([V1] abstract: the 8-bit MMA paths, int8
 * ahead of fp8 on the lattice output after the rotation).  Reading: the
 * doubled lattice coordinates 2y are integers for E8 (y in Z or Z + 1/2),
 * D4 and Z, so A = 2y is exact in int8 while |2y| <= 127; A2's second
 * coordinate carries sqrt3 and has no integer form.  The activations are
 * rotated like the weights, x~ = H (s_j . x_bj) in binary32, and quantized
 * per (batch row, column tile) to q = rint(x~ 127 / max|x~|) with scale
 * s = max|x~| / 127 (all binary32, so q is decided exactly).  Then
 *   Y[b][r] = sum_j Delta_rj s_bj / (2 n) sum_i A_rji q_bji.
 * Coordinates with |2y| > 127 are saturated to +-127 and flagged. */

/* q and s for one activation tile x (n binary32 values, column tile j). */
void hqo_act_quant_i8(const float *x, int n, uint64_t seed, uint64_t j, int8_t *q, float *scale)
{
    float v[HQO_MAX_TILE];
    float amax = 0.0f;
    for (int i = 0; i < n; i++) v[i] = (float)hqo_sign(seed, j, (uint32_t)i) * x[i];
    hqo_fwht_f32(v, n);
    for (int i = 0; i < n; i++)
        if (fabsf(v[i]) > amax || isnan(v[i])) amax = isnan(v[i]) ? v[i] : fabsf(v[i]);
    if (amax == 0.0f || !isfinite(amax)) {
        for (int i = 0; i < n; i++) q[i] = 0;
        *scale = amax;  /* 0, or the non-finite value, which then propagates */
        return;
    }
    float inv = 127.0f / amax;
    for (int i = 0; i < n; i++) q[i] = (int8_t)rintf(v[i] * inv);
    *scale = amax / 127.0f;
}

/* Doubled lattice coordinates of one tile's points (E8, D4, Z): a[i] = 2 y_i
 * saturated to [-127, 127]; *sat counts the saturated coordinates.  Returns
 * the parse status (HQO_CORRUPT: a is zero). */
int hqo_tile_points_i8(const uint32_t *words, int nwords, int n, int lattice, int k, int exact, int8_t *a,
                       int *sat)
{
    uint32_t u[HQO_MAX_TILE];
    uint8_t coset[HQO_MAX_TILE];
    int32_t z[8];
    int d = lattice, nv = n / lattice;
    int st = unpack_words(lattice, n, k, words, nwords, coset, u, exact);
    if (st || lattice == 2) {
        for (int i = 0; i < n; i++) a[i] = 0;
        return st ? st : HQO_CORRUPT;
    }
    for (int q = 0; q < nv; q++) {
        hqo_unsymbols(lattice, &u[q * d], z);
        for (int m = 0; m < d; m++) {
            int32_t v2 = 2 * z[m] + coset[q];
            if (v2 > 127 || v2 < -127) {
                (*sat)++;
                v2 = v2 > 0 ? 127 : -127;
            }
            a[q * d + m] = (int8_t)v2;
        }
    }
    return 0;
}

/* Y for rows [r0, r1) and all `batch` rows of X: Q (batch x cols int8) and
 * S (batch x cols/n scales) from hqo_act_quant_i8; the stream is
 * variable-rate (off != NULL) or fixed-rate (slot words, off == NULL) with
 * one k per tile in kk.  Y is batch x (r1 - r0), binary64.  Returns the OR
 * of the tile statuses; *sat gets the saturated coordinates. */
int hqo_gemm_i8_rows(const uint32_t *payload, uint64_t cap, const uint32_t *off, int slot_words,
                     const uint16_t *scale, const uint8_t *kk, int64_t cols, int n, int lattice, const int8_t *Q,
                     const float *S, int64_t batch, int64_t r0, int64_t r1, double *Y, int *sat)
{
    int8_t a[HQO_MAX_TILE];
    int64_t tpr = cols / n;
    int status = 0;
    for (int64_t r = r0; r < r1; r++) {
        for (int64_t b = 0; b < batch; b++) Y[b * (r1 - r0) + (r - r0)] = 0.0;
        for (int64_t j = 0; j < tpr; j++) {
            int64_t t = r * tpr + j;
            const uint32_t *w;
            int nw;
            if (off) {
                if (off[t + 1] < off[t] || off[t + 1] > cap) {
                    status |= HQO_CORRUPT;
                    continue;
                }
                w = payload + off[t];
                nw = (int)(off[t + 1] - off[t]);
            } else {
                if ((uint64_t)(t + 1) * (uint64_t)slot_words > cap) {
                    status |= HQO_CORRUPT;
                    continue;
                }
                w = payload + t * (int64_t)slot_words;
                nw = slot_words;
            }
            int st = hqo_tile_points_i8(w, nw, n, lattice, kk[t], off != NULL, a, sat);
            status |= st;
            if (st) continue;
            double delta = (double)bf16_to_float(scale[t]);
            for (int64_t b = 0; b < batch; b++) {
                int64_t dot = 0;
                const int8_t *q = Q + b * cols + j * n;
                for (int i = 0; i < n; i++) dot += (int64_t)a[i] * (int64_t)q[i];
                Y[b * (r1 - r0) + (r - r0)] += delta * (double)S[b * tpr + j] / (2.0 * n) * (double)dot;
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* fp8 tensor-core product ([V1] abstract: the fp8-e4m3 MMA path, which the
 * pages find behind int8 on the lattice output).  Same construction as the
 * integer product with both operands in OCP FP8 E4M3 (1 sign, 4 exponent
 * bits with bias 7, 3 mantissa bits, subnormals, no infinity, largest
 * finite 448, NaN = S.1111.111): A = e4m3(2y) -- exact only while |2y| <= 16
 * or on the format's coarser grid beyond -- and q = e4m3(x~ 448 / max|x~|),
 * s = max|x~| / 448.  Conversion rounds to nearest, ties to even, and
 * saturates finite values to +-448. */

/* binary32 -> E4M3 bits, round to nearest even, saturating (NaN -> 0x7F). */
uint8_t hqo_e4m3(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;  /* 448 or above (ties at 464 would round up past the largest) */
    int e;
    if (a < 0x1p-6) {
        e = -6;  /* subnormal range: quantum 2^-9 */
    } else {
        e = (int)floor(log2(a));
        if (ldexp(1.0, e) > a) e--;  /* guard the log against rounding */
        if (ldexp(1.0, e + 1) <= a) e++;
    }
    double quantum = ldexp(1.0, e - 3);
    double m = a / quantum;  /* exact: a power-of-two scale */
    double r = floor(m);
    double frac = m - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double v = r * quantum;  /* the rounded magnitude */
    if (v >= 448.0) return sign | 0x7E;
    if (v < 0x1p-6) return sign | (uint8_t)(v / 0x1p-9);  /* subnormal: exponent field 0 */
    int ev;
    double mant = frexp(v, &ev);  /* v = mant 2^ev, mant in [0.5, 1) */
    int E = ev - 1;               /* v = 1.f 2^E */
    int f = (int)((mant * 2.0 - 1.0) * 8.0);
    return sign | (uint8_t)(((E + 7) << 3) | f);
}

float hqo_e4m3_value(uint8_t b)
{
    int s = b >> 7, E = (b >> 3) & 15, f = b & 7;
    if (E == 15 && f == 7) return NAN;
    double v = E == 0 ? ldexp((double)f, -9) : ldexp(1.0 + f / 8.0, E - 7);
    return (float)(s ? -v : v);
}

/* q (E4M3 bits) and s for one activation tile x (column tile j). */
void hqo_act_quant_e4m3(const float *x, int n, uint64_t seed, uint64_t j, uint8_t *q, float *scale)
{
    float v[HQO_MAX_TILE];
    float amax = 0.0f;
    for (int i = 0; i < n; i++) v[i] = (float)hqo_sign(seed, j, (uint32_t)i) * x[i];
    hqo_fwht_f32(v, n);
    for (int i = 0; i < n; i++)
        if (fabsf(v[i]) > amax || isnan(v[i])) amax = isnan(v[i]) ? v[i] : fabsf(v[i]);
    if (amax == 0.0f || !isfinite(amax)) {
        for (int i = 0; i < n; i++) q[i] = 0;
        *scale = amax;
        return;
    }
    float inv = 448.0f / amax;
    for (int i = 0; i < n; i++) q[i] = hqo_e4m3(v[i] * inv);
    *scale = amax / 448.0f;
}

/* Y for rows [r0, r1): as hqo_gemm_i8_rows with A = e4m3(2y) (saturated to
 * +-448 and counted in *sat) and Q holding E4M3 bits; the products of E4M3
 * values are summed exactly in binary64. */
int hqo_gemm_e4m3_rows(const uint32_t *payload, uint64_t cap, const uint32_t *off, int slot_words,
                       const uint16_t *scale, const uint8_t *kk, int64_t cols, int n, int lattice,
                       const uint8_t *Q, const float *S, int64_t batch, int64_t r0, int64_t r1, double *Y, int *sat)
{
    uint32_t u[HQO_MAX_TILE];
    uint8_t coset[HQO_MAX_TILE];
    double a[HQO_MAX_TILE];
    int32_t z[8];
    int64_t tpr = cols / n;
    int status = 0, d = lattice, nv = n / lattice;
    for (int64_t r = r0; r < r1; r++) {
        for (int64_t b = 0; b < batch; b++) Y[b * (r1 - r0) + (r - r0)] = 0.0;
        for (int64_t j = 0; j < tpr; j++) {
            int64_t t = r * tpr + j;
            const uint32_t *w;
            int nw;
            if (off) {
                if (off[t + 1] < off[t] || off[t + 1] > cap) {
                    status |= HQO_CORRUPT;
                    continue;
                }
                w = payload + off[t];
                nw = (int)(off[t + 1] - off[t]);
            } else {
                if ((uint64_t)(t + 1) * (uint64_t)slot_words > cap) {
                    status |= HQO_CORRUPT;
                    continue;
                }
                w = payload + t * (int64_t)slot_words;
                nw = slot_words;
            }
            int st = lattice == 2 ? HQO_CORRUPT : unpack_words(lattice, n, kk[t], w, nw, coset, u, off != NULL);
            status |= st;
            if (st) continue;
            for (int q = 0; q < nv; q++) {
                hqo_unsymbols(lattice, &u[q * d], z);
                for (int m = 0; m < d; m++) {
                    float v2 = (float)(2 * z[m] + coset[q]);
                    if (fabsf(v2) > 448.0f) (*sat)++;
                    a[q * d + m] = (double)hqo_e4m3_value(hqo_e4m3(v2));
                }
            }
            double delta = (double)bf16_to_float(scale[t]);
            for (int64_t b = 0; b < batch; b++) {
                double dot = 0.0;
                const uint8_t *qq = Q + b * cols + j * n;
                for (int i = 0; i < n; i++) dot += a[i] * (double)hqo_e4m3_value(qq[i]);
                Y[b * (r1 - r0) + (r - r0)] += delta * (double)S[b * tpr + j] / (2.0 * n) * dot;
            }
        }
    }
    return status;
}

/* Nearest points of `count` vectors stored back to back (d floats each). */
void hqo_nearest_batch(int lattice, const float *x, int64_t count, int32_t *c, int32_t *z,
                       float *pt)
{
    int d = lattice;
    for (int64_t q = 0; q < count; q++) {
        int cc;
        hqo_nearest(lattice, x + q * d, &cc, z + q * d, pt + q * d);
        c[q] = cc;
    }
}
