// hq_device.cuh -- device building blocks of the sm_100a HyperQuant codec.
//
// A tile of n coordinates is held by a group of LPT = n / EPL lanes of one
// warp, EPL coordinates per lane, coordinate i = lane_in_group * EPL + r.
// Index bits below log2(EPL) live in registers, the others across lanes, so
// butterfly stages and pairwise reductions over index bit b run in
// registers for b < log2(EPL) and as __shfl_xor over lanes otherwise.
//
// Every floating-point step that decides an integer (rotation, scale,
// nearest point, dither) uses the _rn intrinsics so nothing is contracted
// into an FMA and each operation rounds once to nearest-even, as the
// method's definition of the codec does.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace hq {

constexpr unsigned FULL = 0xffffffffu;
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

// SplitMix64 output function (Steele, Lea & Flood 2014).
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

// Per-call hash key of a tag: H(seed, tag, a, b) = mix64(mix64(key ^ a) ^ b).
__host__ __forceinline__ uint64_t hash_key(uint64_t seed, uint64_t tag)
{
    return mix64(seed + kGamma * (tag + 1));
}

// ------------------------------------------------------------- division
// Unsigned 32-bit division by a divisor fixed per call (Granlund & Montgomery,
// "Division by invariant integers using multiplication", 1994): q = n / d.
struct FastDiv {
    uint32_t d, m, s1, s2;
};

__host__ inline FastDiv make_fastdiv(uint32_t d)
{
    FastDiv f{ d, 0, 0, 0 };
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < d) ++l;
    f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
    f.s1 = l > 0 ? 1 : 0;
    f.s2 = l > 0 ? l - 1 : 0;
    return f;
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv &f)
{
    const uint32_t t = __umulhi(f.m, n);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

// ------------------------------------------------------------- groups
template <int LPT>
__device__ __forceinline__ unsigned group_mask(int lane)
{
    if constexpr (LPT == 32) return FULL;
    else return ((1u << LPT) - 1u) << (lane & ~(LPT - 1));
}

template <int LPT>
__device__ __forceinline__ uint32_t group_sum(unsigned mask, uint32_t v)
{
    return __reduce_add_sync(mask, v);
}

template <int LPT>
__device__ __forceinline__ uint32_t group_max(unsigned mask, uint32_t v)
{
    return __reduce_max_sync(mask, v);
}

// exclusive prefix sum over the lanes of a group
template <int LPT>
__device__ __forceinline__ uint32_t group_excl_scan(unsigned mask, uint32_t v, int l)
{
    uint32_t incl = v;
#pragma unroll
    for (int d = 1; d < LPT; d <<= 1) {
        uint32_t o = __shfl_up_sync(mask, incl, d, LPT);
        if (l >= d) incl += o;
    }
    return incl - v;
}

// ------------------------------------------------------------- rotation
// Unnormalised Walsh-Hadamard transform, stages h = 1, 2, ..., n/2 in that
// order; the lower index of each pair keeps the sum, the upper the
// difference (lower - upper).  For lane stages the upper lane computes
// other - own as fma(-1, own, other), exactly one rounding of the same
// difference.
template <int EPL, int LPT>
__device__ __forceinline__ void fwht(float (&v)[EPL], unsigned mask, int l)
{
#pragma unroll
    for (int h = 1; h < EPL; h <<= 1) {
#pragma unroll
        for (int a = 0; a < EPL; a++) {
            if (!(a & h)) {
                float p = v[a], q = v[a + h];
                v[a] = __fadd_rn(p, q);
                v[a + h] = __fsub_rn(p, q);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < LPT; m <<= 1) {
        const float sg = (l & m) ? -1.0f : 1.0f;
#pragma unroll
        for (int a = 0; a < EPL; a++) {
            float o = __shfl_xor_sync(mask, v[a], m);
            v[a] = __fmaf_rn(sg, v[a], o);
        }
    }
}

// Sum of squares by the pairwise tree over index bits (bit 0 first).
template <int EPL, int LPT>
__device__ __forceinline__ float sumsq(const float (&w)[EPL], unsigned mask)
{
    float a[EPL];
#pragma unroll
    for (int i = 0; i < EPL; i++) a[i] = __fmul_rn(w[i], w[i]);
#pragma unroll
    for (int h = 1; h < EPL; h <<= 1)
#pragma unroll
        for (int i = 0; i < EPL; i++)
            if (!(i & h) && (i % (2 * h)) == 0) a[i] = __fadd_rn(a[i], a[i + h]);
    float s = a[0];
#pragma unroll
    for (int m = 1; m < LPT; m <<= 1) s = __fadd_rn(s, __shfl_xor_sync(mask, s, m));
    return s;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Delta as bf16 bits: 0 for a non-finite S (flagged), S < 2^-96, or a zero /
// subnormal result.
__device__ __forceinline__ uint32_t tile_scale_bits(float S, float c, bool &nonfinite)
{
    nonfinite = (__float_as_uint(S) & 0x7f800000u) == 0x7f800000u;
    if (nonfinite || S < 0x1p-96f) return 0;
    float d32 = __fmul_rn(c, __fsqrt_rn(S));
    uint32_t b = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(d32));
    return (b & 0x7f80u) ? b : 0u;
}

// ------------------------------------------------------------- lattices
// Conway & Sloane (1982) nearest points.  Ties: rint to even; D_n flips the
// first coordinate of largest |x - rint x| towards x (up when exact); E8 and
// A2 keep coset 0 when both squared distances are equal.
template <int D>
__device__ __forceinline__ void dn_round(const float (&x)[D], float (&f)[D])
{
    float e[D];
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < D; i++) {
        f[i] = rintf(x[i]);
        e[i] = __fsub_rn(x[i], f[i]);
        sum = __fadd_rn(sum, f[i]);   // small integers: exact
    }
    if (__float2int_rn(sum) & 1) {
        int b = 0;
        float ab = fabsf(e[0]), eb = e[0];
#pragma unroll
        for (int i = 1; i < D; i++) {
            float a = fabsf(e[i]);
            if (a > ab) { ab = a; eb = e[i]; b = i; }
        }
        const float dir = (eb >= 0.0f) ? 1.0f : -1.0f;
#pragma unroll
        for (int i = 0; i < D; i++)
            if (i == b) f[i] = __fadd_rn(f[i], dir);
    }
}

struct A2Consts {
    float s3;     // fp32(sqrt 3)
    float inv_s3; // fp32(1 / sqrt 3)
};

// Nearest point of one D-dimensional vector: coset bit, integer coordinates
// (pre-strip), and the point in binary32.
template <int D>
__device__ __forceinline__ void nearest(const float (&x)[D], int &c, int (&z)[D], float (&p)[D],
                                        const A2Consts &a2)
{
    c = 0;
    if constexpr (D == 1) {
        p[0] = rintf(x[0]);
        z[0] = __float2int_rn(p[0]);
    } else if constexpr (D == 4) {
        dn_round<4>(x, p);
#pragma unroll
        for (int i = 0; i < 4; i++) z[i] = __float2int_rn(p[i]);
    } else if constexpr (D == 8) {
        // Two candidates: D8 from f = rint(x) and D8 + 1/2 from floor(x) + 1/2,
        // whose coordinates lie exactly 1/2 - |e_i| from x (e = x - f), so
        //   d0 - d1 = sum|e| - 2 + [sum f odd](1 - 2 max|e|) - [sum floor odd] 2 min|e|
        // (binary32, in this order); d0 - d1 <= 0 keeps the integer coset.
        float f[8], g[8], e[8], ae[8];
        float sf = 0.0f, sg = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            f[i] = rintf(x[i]);
            g[i] = floorf(x[i]);
            e[i] = __fsub_rn(x[i], f[i]);
            ae[i] = fabsf(e[i]);
            sf = __fadd_rn(sf, f[i]);  // small integers: exact
            sg = __fadd_rn(sg, g[i]);
        }
        const bool odd0 = __float2int_rn(sf) & 1, odd1 = __float2int_rn(sg) & 1;
        float mx = ae[0], mn = ae[0], s = ae[0];
#pragma unroll
        for (int i = 1; i < 8; i++) {
            mx = fmaxf(mx, ae[i]);
            mn = fminf(mn, ae[i]);
            s = __fadd_rn(s, ae[i]);
        }
        float dd = __fsub_rn(s, 2.0f);
        if (odd0) dd = __fadd_rn(dd, __fsub_rn(1.0f, 2.0f * mx));
        if (odd1) dd = __fsub_rn(dd, 2.0f * mn);
        const bool one = !(dd <= 0.0f);
        c = one ? 1 : 0;
        // the coordinate the parity fix moves: first index of max|e| (D8) or
        // min|e| (D8 + 1/2); towards x
        const bool fix = one ? odd1 : odd0;
        const float target = one ? mn : mx;
        int b = 0;
#pragma unroll
        for (int i = 7; i >= 0; i--)
            if (ae[i] == target) b = i;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            float base = one ? g[i] : f[i];
            if (fix && i == b) {
                const bool up = one ? (__fsub_rn(x[i], g[i]) >= 0.5f) : (e[i] >= 0.0f);
                base = __fadd_rn(base, up ? 1.0f : -1.0f);
            }
            z[i] = __float2int_rn(base);
            p[i] = one ? __fadd_rn(base, 0.5f) : base;
        }
    } else {  // A2: points (a + c/2, (b + c/2) sqrt3)
        float y1 = __fmul_rn(x[1], a2.inv_s3);
        float a0 = rintf(x[0]), b0 = rintf(y1);
        float a1 = rintf(__fsub_rn(x[0], 0.5f)), b1 = rintf(__fsub_rn(y1, 0.5f));
        float p00 = a0, p01 = __fmul_rn(b0, a2.s3);
        float p10 = __fadd_rn(a1, 0.5f), p11 = __fmul_rn(__fadd_rn(b1, 0.5f), a2.s3);
        float t0 = __fsub_rn(x[0], p00), t1 = __fsub_rn(x[1], p01);
        float d0 = __fadd_rn(__fmul_rn(t0, t0), __fmul_rn(t1, t1));
        float u0 = __fsub_rn(x[0], p10), u1 = __fsub_rn(x[1], p11);
        float d1 = __fadd_rn(__fmul_rn(u0, u0), __fmul_rn(u1, u1));
        const bool one = !(d0 <= d1);
        c = one ? 1 : 0;
        z[0] = __float2int_rn(one ? a1 : a0);
        z[1] = __float2int_rn(one ? b1 : b0);
        p[0] = one ? p10 : p00;
        p[1] = one ? p11 : p01;
    }
}

// ------------------------------------------------------------- dither
// Four uniforms on the 16-bit grid of [0,1) for coordinates 4g .. 4g+3 of a
// tile: coordinate 4g + k takes bits 16k .. 16k+15 of mix64(tile_key ^ g).
__device__ __forceinline__ void uniform4(uint64_t tile_key, uint32_t g, float (&r)[4])
{
    const uint64_t h = mix64(tile_key ^ (uint64_t)g);
    const uint32_t lo = (uint32_t)h, hi = (uint32_t)(h >> 32);
    r[0] = (float)(lo & 0xffffu) * 0x1p-16f;
    r[1] = (float)(lo >> 16) * 0x1p-16f;
    r[2] = (float)(hi & 0xffffu) * 0x1p-16f;
    r[3] = (float)(hi >> 16) * 0x1p-16f;
}

// Dither coordinate m of a D-vector from its uniform r: a centred box that
// is a fundamental domain of a sublattice (D_d for E8 and D4: [-1/2,1/2)^(d-1)
// x [-1,1); Z x sqrt3 Z for A2; Z for Z).  Exact except the A2 second
// coordinate (one rounding).
template <int D>
__device__ __forceinline__ float box_dither(float r, int m, const A2Consts &a2)
{
    if constexpr (D == 8 || D == 4) {
        return m == D - 1 ? __fmaf_rn(2.0f, r, -1.0f) : __fsub_rn(r, 0.5f);
    } else if constexpr (D == 2) {
        return m == 1 ? __fmul_rn(__fsub_rn(r, 0.5f), a2.s3) : __fsub_rn(r, 0.5f);
    } else {
        return __fsub_rn(r, 0.5f);
    }
}

// Dither of vector q of lane l (coordinates l*EPL + q*D ...).  For D < 4 one
// hash serves 4/D consecutive vectors: r4 carries it from the vector that
// starts a group of four coordinates to the next ones (call with q in order).
template <int D, int EPL>
__device__ __forceinline__ void dither_vec(uint64_t tile_key, int l, int q, float (&r4)[4], float (&delta)[D],
                                           const A2Consts &a2)
{
    const uint32_t g0 = (uint32_t)l * (EPL / 4) + (uint32_t)(q * D) / 4;
    if constexpr (D >= 4) {
#pragma unroll
        for (int b = 0; b < D / 4; b++) {
            uniform4(tile_key, g0 + b, r4);
#pragma unroll
            for (int k = 0; k < 4; k++) delta[4 * b + k] = box_dither<D>(r4[k], 4 * b + k, a2);
        }
    } else {
        if (((q * D) & 3) == 0) uniform4(tile_key, g0, r4);
#pragma unroll
        for (int m = 0; m < D; m++) delta[m] = box_dither<D>(r4[((q * D) & 3) + m], m, a2);
    }
}

// Subtract the dither from lane l's EPL lattice coordinates.
template <int D, int EPL>
__device__ __forceinline__ void sub_dither(uint64_t tile_key, int l, float (&pt)[EPL], const A2Consts &a2)
{
    float r4[4];
#pragma unroll
    for (int q = 0; q < EPL / D; q++) {
        float dl[D];
        dither_vec<D, EPL>(tile_key, l, q, r4, dl, a2);
#pragma unroll
        for (int m = 0; m < D; m++) pt[q * D + m] = __fsub_rn(pt[q * D + m], dl[m]);
    }
}

// ------------------------------------------------------------- symbols
__device__ __forceinline__ uint32_t zigzag(int z) { return ((uint32_t)z << 1) ^ (uint32_t)(z >> 31); }
__device__ __forceinline__ int unzigzag(uint32_t u) { return (int)(u >> 1) ^ -(int)(u & 1u); }

// ------------------------------------------------------------- bits
// v << s with s >= 32 giving 0 (PTX clamps the shift amount)
__device__ __forceinline__ uint32_t shl32(uint32_t v, uint32_t s)
{
    uint32_t r;
    asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(s));
    return r;
}

// OR `len` (<= 64) bits of v into a shared-memory bit buffer at bit `pos`.
// The shifted value spans at most three words.
__device__ __forceinline__ void or_bits(uint32_t *buf, uint32_t pos, uint64_t v, int len)
{
    if (len <= 0 || v == 0) return;
    const uint32_t w = pos >> 5, sh = pos & 31;
    const uint32_t b0 = (uint32_t)(v << sh);
    const uint32_t b1 = sh ? (uint32_t)(v >> (32 - sh)) : (uint32_t)(v >> 32);
    const uint32_t b2 = sh ? (uint32_t)(v >> (64 - sh)) : 0u;
    if (b0) atomicOr(&buf[w], b0);
    if (len + (int)sh > 32 && b1) atomicOr(&buf[w + 1], b1);
    if (len + (int)sh > 64 && b2) atomicOr(&buf[w + 2], b2);
}

// OR `len` (<= 32) bits of v into a shared-memory bit buffer at bit `pos`
// (at most two words).
__device__ __forceinline__ void or_bits32(uint32_t *buf, uint32_t pos, uint32_t v, int len)
{
    const uint32_t w = pos >> 5, sh = pos & 31;
    atomicOr(&buf[w], v << sh);
    if (sh && (int)sh + len > 32) atomicOr(&buf[w + 1], v >> (32 - sh));
}

// or_bits32 confined to the buffer's first `limit` words: a write past them
// is dropped (the caller's lengths already keep every write inside; this
// only guards the buffer against an inconsistent length).
__device__ __forceinline__ void or_bits32_lim(uint32_t *buf, uint32_t pos, uint32_t v, int len, uint32_t limit)
{
    const uint32_t w = pos >> 5, sh = pos & 31;
    if (w < limit) atomicOr(&buf[w], v << sh);
    if (sh && (int)sh + len > 32 && w + 1 < limit) atomicOr(&buf[w + 1], v >> (32 - sh));
}

// `len` (<= 32) bits at bit `pos` of a word buffer (buf[pos/32 + 1] must be
// readable).
__device__ __forceinline__ uint32_t get_bits(const uint32_t *buf, uint32_t pos, int len)
{
    uint32_t w = pos >> 5, sh = pos & 31;
    uint64_t v = (uint64_t)buf[w] | ((uint64_t)buf[w + 1] << 32);
    uint32_t r = (uint32_t)(v >> sh);
    return len >= 32 ? r : (r & ((1u << len) - 1u));
}

}  // namespace hq
