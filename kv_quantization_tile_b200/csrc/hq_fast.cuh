// hq_fast.cuh -- packed-pair building blocks of the sm_100a codec kernels.
//
// Layout.  A group of LPT = n / EPL lanes holds one tile, EPL coordinates per
// lane, as EPL / 2 float2 pairs: pair m holds coordinates 2m and 2m + 1 of the
// lane's slice, so element-wise steps run as one f32x2 instruction per pair
// (add / sub / mul / fma .rn, add .rm), each lane of the pair rounded once to
// nearest-even (or down) exactly like the scalar binary32 operation.
//
// Half-exchange Walsh-Hadamard transform.  The loaded tile has index bits
// 0 .. e-1 in registers (e = log2 EPL, lane l holds coordinates l EPL ..) and
// bits e .. e+p-1 across the group's lanes (p = log2 LPT).  Stages run on
// index bits 0, 1, 2, ... in that order, each mapping a pair (a, c) (a the
// lower index) to (a + c, a - c) in binary32.  The stages on register bits
// run in registers.  The stage on lane bit j swaps that lane bit with the top
// register bit (the passenger): each lane keeps the half of its registers
// whose passenger value equals its lane bit and sends the other half to its
// partner (EPL / 2 shuffles instead of EPL), so after the stage the passenger
// register bit holds the stage's index bit and lane bit j the passenger's
// old one.  Every lane sends the same physical half because a lane whose next
// lane bit is set stores its two halves swapped; the swap is a +-1 factor in
// the fma that forms each output, chosen per lane.  The outputs are then
// exactly the reference transform's values up to a sign per (lane, half):
// sigma_A = (-1)^popc(l & (l >> 1)) for the low half and sigma_B = sigma_A
// (-1)^(top lane bit) for the high half.  After the transform lane l holds two
// runs of EPL / 2 consecutive coordinates: run A = l EPL/2 .., run B =
// n/2 + l EPL/2 .. (pairs 0 .. EPL/4 - 1 and EPL/4 .. EPL/2 - 1).
//
// Method: [V1] "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline
// for Large Language and Diffusion Models", abstract (i) per-tile randomized
// Hadamard transform, (ii) E8 nearest point (Conway & Sloane 1982).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "hq_device.cuh"

namespace hq {

// ------------------------------------------------------------- f32x2
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 add2_rd(float2 a, float2 b) { return __fadd2_rd(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b)
{
    float2 r;
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 b, {%4, %5};\n\t"
        "sub.rn.f32x2 d, a, b;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// ------------------------------------------------------------- transform
// Forward transform of one tile held as EPL / 2 pairs per lane (see above).
// l is the lane's index in its group, mask the group's lanes.
template <int EPL, int LPT>
__device__ __forceinline__ void fwht_hx(float2 (&P)[EPL / 2], unsigned mask, int l)
{
    constexpr int NP = EPL / 2, HP = NP / 2;
    static_assert(EPL >= 4 && (EPL & (EPL - 1)) == 0 && LPT >= 2, "layout");
#pragma unroll
    for (int m = 0; m < NP; m++) {  // index bit 0: inside each pair
        const float a = P[m].x, c = P[m].y;
        P[m] = make_float2(__fadd_rn(a, c), __fsub_rn(a, c));
    }
#pragma unroll
    for (int h = 1; h < HP; h <<= 1) {  // index bits 1 .. e-2: between pairs
#pragma unroll
        for (int m = 0; m < NP; m++) {
            if (!(m & h)) {
                const float2 a = P[m], c = P[m + h];
                P[m] = add2(a, c);
                P[m + h] = sub2(a, c);
            }
        }
    }
    {  // index bit e-1 (the passenger): halves stored swapped where lane bit 0 is set
        const float s = (l & 1) ? -1.0f : 1.0f;
        const float2 cp = splat2(s), cn = splat2(-s);
#pragma unroll
        for (int m = 0; m < HP; m++) {
            const float2 a = P[m], c = P[m + HP];
            P[m] = fma2(c, cp, a);
            P[m + HP] = fma2(c, cn, a);
        }
    }
#pragma unroll
    for (int j = 0; (1 << j) < LPT; j++) {  // lane bit j <-> passenger
        float2 r[HP];
#pragma unroll
        for (int m = 0; m < HP; m++)
            r[m] = make_float2(__shfl_xor_sync(mask, P[m + HP].x, 1 << j), __shfl_xor_sync(mask, P[m + HP].y, 1 << j));
        if ((2 << j) < LPT) {  // place for the next lane stage
            const float s = ((l >> (j + 1)) & 1) ? -1.0f : 1.0f;
            const float2 cp = splat2(s), cn = splat2(-s);
#pragma unroll
            for (int m = 0; m < HP; m++) {
                const float2 k = P[m];
                P[m] = fma2(r[m], cp, k);
                P[m + HP] = fma2(r[m], cn, k);
            }
        } else {
#pragma unroll
            for (int m = 0; m < HP; m++) {
                const float2 k = P[m];
                P[m] = add2(k, r[m]);
                P[m + HP] = sub2(k, r[m]);
            }
        }
    }
}

// Signs the half-exchange transform leaves on lane l's two runs: bit 0 set
// if run A is negated, bit 1 if run B is.
template <int LPT>
__device__ __forceinline__ uint32_t hx_sigma_bits(int l)
{
    const uint32_t a = (uint32_t)__popc((uint32_t)l & ((uint32_t)l >> 1)) & 1u;
    const uint32_t top = ((uint32_t)l >> (__ffs(LPT) - 2)) & 1u;
    return a | ((a ^ top) << 1);
}

// ------------------------------------------------------------- sum of squares
// Sum of squares of lane-contiguous coordinates by the pairwise tree over
// index bits (bit 0 first): pair sums, then between pairs, then across lanes.
// EXACT_SQ: every square is exact in binary32 (bf16 inputs), so a pair sum may
// fuse its second square into one fma.
template <int EPL, int LPT, bool EXACT_SQ>
__device__ __forceinline__ float sumsq_pairs(const float2 (&P)[EPL / 2], unsigned mask)
{
    constexpr int NP = EPL / 2;
    float a[NP];
#pragma unroll
    for (int m = 0; m < NP; m++) {
        if constexpr (EXACT_SQ) {
            a[m] = __fmaf_rn(P[m].y, P[m].y, __fmul_rn(P[m].x, P[m].x));
        } else {
            a[m] = __fadd_rn(__fmul_rn(P[m].x, P[m].x), __fmul_rn(P[m].y, P[m].y));
        }
    }
#pragma unroll
    for (int h = 1; h < NP; h <<= 1)
#pragma unroll
        for (int m = 0; m < NP; m += 2 * h) a[m] = __fadd_rn(a[m], a[m + h]);
    float s = a[0];
#pragma unroll
    for (int d = 1; d < LPT; d <<= 1) s = __fadd_rn(s, __shfl_xor_sync(mask, s, d));
    return s;
}

// ------------------------------------------------------------- signs
// A lane's random signs as one word Y, arranged so the XOR mask of pair m's
// two bf16 halves is (Y << m) & 0x80008000: the sign of the pair's first
// coordinate sits at bit 15 - m, of its second at bit 31 - m.  `neg(i)` gives
// the sign bit (1 = negative) of the lane's coordinate i (i < EPL, in pair
// order: pair m holds i = 2m, 2m + 1).
template <int EPL, typename F>
__host__ __device__ __forceinline__ uint32_t sign_word(F neg)
{
    uint32_t y = 0;
    for (int m = 0; m < EPL / 2; m++) {
        y |= (uint32_t)neg(2 * m) << (15 - m);
        y |= (uint32_t)neg(2 * m + 1) << (31 - m);
    }
    return y;
}

// ------------------------------------------------------------- E8
constexpr int32_t kMagicBias = 0x4B400000;  // bits of 1.5 * 2^23: B + k is the float 1.5 2^23 + k

// E8 nearest point and symbols of one vector (4 pairs of x = v / Delta
// [+ dither]): the Conway-Sloane two-coset rule with the exact distance
// identity (see nearest<8> in hq_device.cuh), branch-free and in binary32
// arithmetic on exact small integers (the fma pipe).
//   R = x + 1.5 2^23 rounded to nearest (rint x, biased), F = the same add
//   rounded down (floor x, biased), e = x - rint x, all exact for |x| < 2^22.
//   d0 - d1 = sum|e| - 2 + [sum rint odd](1 - 2 max|e|) - [sum floor odd] 2 min|e|
//   (binary32, this order); d0 - d1 <= 0 keeps the integer coset.
//   The parity fix moves the coordinate of largest |e| (integer coset) or
//   smallest |e| (half-integer coset) one step towards x.  With C = F - R
//   (0, or -1 where rint = floor + 1) and h = +1 (integer coset) or -1
//   (half-integer coset) at the moved coordinate, 0 elsewhere,
//     z = F - [integer coset] C + h (1 + 2C)   (biased by 1.5 2^23, then removed)
//   is the stored integer y - c/2, and the zigzag of an integer z is
//   |2z + 1/2| - 1/2 (2z for z >= 0, -2z - 1 below).  The last coordinate is
//   stored as floor(z / 2) (an fma rounded down against 1.5 2^23).
// U gets the 8 symbols as exact binary32 integers; returns the coset bit.
// When |e| == T holds for more than one coordinate, the rule moves the first
// of them (index order), so h keeps only the first hit.
__device__ __forceinline__ int e8_symbols(const float2 (&X)[4], float2 (&U)[4])
{
    constexpr float kM = 12582912.0f;  // 1.5 * 2^23
    const float2 M2 = splat2(kM);
    float2 R[4], F[4], E[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        R[i] = add2(X[i], M2);
        F[i] = add2_rd(X[i], M2);
        E[i] = sub2(X[i], sub2(R[i], M2));
    }
    const float ae[8] = { fabsf(E[0].x), fabsf(E[0].y), fabsf(E[1].x), fabsf(E[1].y),
                          fabsf(E[2].x), fabsf(E[2].y), fabsf(E[3].x), fabsf(E[3].y) };
    float s = ae[0];
#pragma unroll
    for (int i = 1; i < 8; i++) s = __fadd_rn(s, ae[i]);  // in index order: the rounding is part of the rule
    float mx = ae[0], mn = ae[0];
#pragma unroll
    for (int i = 1; i < 8; i++) {
        mx = fmaxf(mx, ae[i]);
        mn = fminf(mn, ae[i]);
    }
    const int32_t px = __float_as_int(R[0].x) ^ __float_as_int(R[0].y) ^ __float_as_int(R[1].x) ^
                       __float_as_int(R[1].y) ^ __float_as_int(R[2].x) ^ __float_as_int(R[2].y) ^
                       __float_as_int(R[3].x) ^ __float_as_int(R[3].y);
    const int32_t py = __float_as_int(F[0].x) ^ __float_as_int(F[0].y) ^ __float_as_int(F[1].x) ^
                       __float_as_int(F[1].y) ^ __float_as_int(F[2].x) ^ __float_as_int(F[2].y) ^
                       __float_as_int(F[3].x) ^ __float_as_int(F[3].y);
    const bool odd0 = px & 1, odd1 = py & 1;
    float dd = __fsub_rn(s, 2.0f);
    if (odd0) dd = __fadd_rn(dd, __fmaf_rn(mx, -2.0f, 1.0f));  // 1 - 2 max|e|: one rounding
    if (odd1) dd = __fmaf_rn(mn, -2.0f, dd);                    // dd - 2 min|e|: one rounding
    const bool one = dd > 0.0f;
    const bool fix = one ? odd1 : odd0;
    const float T = fix ? (one ? mn : mx) : -1.0f;
    const float sc = one ? -1.0f : 1.0f;
    // H: 1 at the coordinates whose |e| is T, else 0
    float2 H[4];
#pragma unroll
    for (int i = 0; i < 4; i++) H[i] = make_float2(ae[2 * i] == T ? 1.0f : 0.0f, ae[2 * i + 1] == T ? 1.0f : 0.0f);
    const float2 hs = add2(add2(H[0], H[1]), add2(H[2], H[3]));
    if (__fadd_rn(hs.x, hs.y) > 1.5f) {  // a tie: only the first hit (in index order) moves
        float seen = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float hx = H[i].x, hy = H[i].y;
            H[i].x = hx * (1.0f - seen);
            seen = fmaxf(seen, hx);
            H[i].y = hy * (1.0f - seen);
            seen = fmaxf(seen, hy);
        }
    }
    const float2 mq0 = splat2(one ? 0.0f : -1.0f), two = splat2(2.0f), half = splat2(0.5f);
    const float2 sc2 = splat2(2.0f * sc), sc1 = splat2(sc);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 C = sub2(F[i], R[i]);
        const float2 base = fma2(C, mq0, F[i]);
        const float2 zb = fma2(H[i], fma2(C, sc2, sc1), base);  // h (1 + 2C), h = sc at a hit
        const float2 z = sub2(zb, M2);
        if (i < 3) {
            const float2 t = fma2(z, two, half);
            U[i] = make_float2(__fsub_rn(fabsf(t.x), 0.5f), __fsub_rn(fabsf(t.y), 0.5f));
        } else {
            const float t6 = __fmaf_rn(z.x, 2.0f, 0.5f);
            const float s7 = __fsub_rn(__fmaf_rd(z.y, 0.5f, kM), kM);  // floor(z / 2)
            const float t7 = __fmaf_rn(s7, 2.0f, 0.5f);
            U[i] = make_float2(__fsub_rn(fabsf(t6), 0.5f), __fsub_rn(fabsf(t7), 0.5f));
        }
    }
    return one ? 1 : 0;
}

}  // namespace hq
