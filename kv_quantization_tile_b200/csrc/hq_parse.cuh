// hq_parse.cuh -- tile parser shared by the decoder, the decode-GEMV and the
// KV-cache attention kernels (see hq_decode.cu for the method).
//
// A group of LPT lanes parses one tile; lane l owns codes l*EPL .. l*EPL+EPL-1.
//   * The tile's words are staged in shared memory (plus zero guard words).
//   * Coset bits and the fixed-width low parts are read at computed offsets.
//   * Unary parts: one pass popcounts the unary words (a lane per word) and
//     records the running count of terminators per word; each lane then
//     selects the terminator of rank l*EPL - 1 (the end of the previous lane's
//     codes), which gives its start bit, and parses its EPL codes
//     sequentially from a bit-reversed 64-bit window with one count-leading-
//     zeros per code.  A lane whose codes span more than 64 bits parses from
//     shared memory word by word instead.
// Every read stays inside the tile's own words.  A tile that is not canonical
// (offsets out of order or past the capacity, k > 15, a scale that is not 0
// or a positive normal bf16, a terminator count other than n, a word count
// other than its bits need) parses to zeros and is reported as bad.
#pragma once

#include "hq_internal.h"

namespace hq {

// words of shared memory per group: staged tile words + 4 guard words, then
// the running terminator count of each unary word
__host__ __device__ constexpr uint32_t group_words(uint32_t wmax) { return 2 * wmax + 4; }

// position of the r-th (0-based) set bit of v (v has more than r set bits)
__device__ __forceinline__ uint32_t select_bit(uint32_t v, uint32_t r)
{
    uint32_t c = __popc(v & 0xffffu);
    uint32_t base = 0;
    if (r >= c) { r -= c; v >>= 16; base = 16; }
    c = __popc(v & 0xffu);
    if (r >= c) { r -= c; v >>= 8; base += 8; }
    for (uint32_t i = 0; i < r; i++) v &= v - 1;
    return base + (__ffs(v) - 1);
}

// Parse tile t into lattice point coordinates pt (binary32).  Returns true
// if the tile is not canonical (pt is then zero and sb is 0).
template <int N, int D, int EPL>
__device__ __forceinline__ bool parse_tile(const DecodeArgs &a, int64_t t, uint32_t *wbuf,
                                           unsigned mask, int l, float (&pt)[EPL], uint32_t &sb)
{
    constexpr int LPT = N / EPL;
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;
    constexpr int VPL = EPL / D;
    uint32_t *cnt = wbuf + a.wmax + 4;

    const uint32_t o0 = a.off[t], o1 = a.off[t + 1];
    const int k = a.kk[t];
    sb = a.scale[t];
    // Delta is 0 or a positive, normal, finite bf16 in any canonical tile
    const uint32_t ex = sb & 0x7f80u;
    bool bad = (o1 < o0) || (o1 - o0 > a.wmax) || ((uint64_t)o1 > a.cap) || (k > 15) ||
               (sb & 0x8000u) || ex == 0x7f80u || (sb != 0 && ex == 0);
    const uint32_t U0 = (uint32_t)C + (uint32_t)N * (uint32_t)k;
    const uint32_t W0 = bad ? 0u : o1 - o0;
    if (!bad && U0 + (uint32_t)N > 32u * W0) bad = true;
    const uint32_t W = bad ? 0u : W0;

    for (uint32_t i = l; i < W; i += LPT) wbuf[i] = __ldg(a.payload + o0 + i);
    if (l < 4) wbuf[W + l] = 0u;
    __syncwarp(mask);

    // ---- unary terminators: running count per unary word
    const uint32_t wu0 = U0 >> 5;
    const uint32_t nwu = W > wu0 ? W - wu0 : 0;  // unary words (the first shared with the low parts)
    uint32_t found = 0;
    for (uint32_t wb = 0; wb < nwu; wb += LPT) {
        const uint32_t wi = wb + l;
        uint32_t v = wi < nwu ? wbuf[wu0 + wi] : 0u;
        if (wi == 0) v &= 0xffffffffu << (U0 & 31);
        const uint32_t c = __popc(v);
        uint32_t incl = c;
#pragma unroll
        for (int d = 1; d < LPT; d <<= 1) {
            const uint32_t o = __shfl_up_sync(mask, incl, d, LPT);
            if (l >= d) incl += o;
        }
        if (wi < nwu) cnt[wi] = found + incl;
        found += __shfl_sync(mask, incl, LPT - 1, LPT);
    }
    if (!bad && found != (uint32_t)N) bad = true;
    __syncwarp(mask);
    // canonical word count: the last word holds the last terminator
    if (!bad && cnt[nwu - 1] == (nwu > 1 ? cnt[nwu - 2] : 0u)) bad = true;

#pragma unroll
    for (int r = 0; r < EPL; r++) pt[r] = 0.0f;
    if (bad) {
        sb = 0;
        return true;
    }

    // ---- this lane's first unary bit (relative to U0): after terminator l*EPL - 1
    uint32_t start = 0;
    if (l > 0) {
        const uint32_t R = (uint32_t)l * EPL - 1;
        uint32_t wi = (uint32_t)(((uint64_t)R * nwu) / (uint32_t)N);  // estimate, then step
        if (wi >= nwu) wi = nwu - 1;
        while (wi > 0 && cnt[wi - 1] > R) --wi;
        while (cnt[wi] <= R) ++wi;
        const uint32_t before = wi ? cnt[wi - 1] : 0u;
        uint32_t v = wbuf[wu0 + wi];
        if (wi == 0) v &= 0xffffffffu << (U0 & 31);
        start = (wu0 + wi) * 32u + select_bit(v, R - before) + 1u - U0;
    }
    // the next lane's start bounds this lane's codes
    uint32_t end = __shfl_down_sync(mask, start, 1, LPT);
    if (l == LPT - 1) {
        const uint32_t v = wbuf[W - 1] & (nwu == 1 ? (0xffffffffu << (U0 & 31)) : 0xffffffffu);
        end = (W - 1) * 32u + (31u - __clz(v)) + 1u - U0;
    }

    // ---- coset bits and low parts
    uint32_t cb = 0;
    if constexpr (C > 0) cb = get_bits(wbuf, (uint32_t)l * VPL, VPL);
    uint32_t low[EPL];
    if (k == 0) {
#pragma unroll
        for (int r = 0; r < EPL; r++) low[r] = 0;
    } else if (k <= 4) {
        const uint32_t lowmask = (1u << k) - 1u;
        const uint32_t base = (uint32_t)C + (uint32_t)l * EPL * (uint32_t)k;
#pragma unroll
        for (int r0 = 0; r0 < EPL; r0 += 8) {
            uint32_t f = get_bits(wbuf, base + (uint32_t)r0 * k, 8 * k);
#pragma unroll
            for (int m = 0; m < 8; m++) {
                low[r0 + m] = f & lowmask;
                f >>= k;
            }
        }
    } else {
        const uint32_t base = (uint32_t)C + (uint32_t)l * EPL * (uint32_t)k;
#pragma unroll
        for (int r = 0; r < EPL; r++) low[r] = get_bits(wbuf, base + (uint32_t)r * k, k);
    }

    // ---- unary parts
    uint32_t q[EPL];
    const uint32_t span = end - start;
    const uint32_t p0 = U0 + start;
    if (span <= 64) {
        const uint32_t w0 = p0 >> 5, sh = p0 & 31;
        const uint32_t b0 = wbuf[w0], b1 = wbuf[w0 + 1], b2 = wbuf[w0 + 2];
        uint32_t rh = __brev(__funnelshift_r(b0, b1, sh));  // next stream bit at the MSB
        uint32_t rl = __brev(__funnelshift_r(b1, b2, sh));
#pragma unroll
        for (int r = 0; r < EPL; r++) {
            uint32_t z = __clz(rh);
            if (z < 32) {
                const uint32_t s = z + 1;
                rh = __funnelshift_lc(rl, rh, s);
                rl = shl32(rl, s);
            } else {  // q >= 32: the terminator sits in the low word
                z = 32 + __clz(rl);
                rh = shl32(rl, z - 31);
                rl = 0;
            }
            q[r] = z;
        }
    } else {
        uint32_t p = p0;
#pragma unroll
        for (int r = 0; r < EPL; r++) {
            uint32_t qq = 0;
            for (;;) {
                const uint32_t w = get_bits(wbuf, p, 32);
                if (w) {
                    const uint32_t z = __ffs(w) - 1;
                    qq += z;
                    p += z + 1;
                    break;
                }
                qq += 32;
                p += 32;
            }
            q[r] = qq;
        }
    }

    // ---- symbols -> lattice point
#pragma unroll
    for (int qv = 0; qv < VPL; qv++) {
        int z[D];
#pragma unroll
        for (int m = 0; m < D; m++) z[m] = unzigzag((q[qv * D + m] << k) | low[qv * D + m]);
        if constexpr (D == 8 || D == 4) {
            int s = 0;
#pragma unroll
            for (int m = 0; m < D - 1; m++) s += z[m];
            z[D - 1] = 2 * z[D - 1] + (s & 1);
        }
        const float half = ((cb >> qv) & 1u) ? 0.5f : 0.0f;
        if constexpr (D == 2) {
            pt[qv * 2] = (float)z[0] + half;
            pt[qv * 2 + 1] = __fmul_rn((float)z[1] + half, a.a2.s3);
        } else {
#pragma unroll
            for (int m = 0; m < D; m++) pt[qv * D + m] = (float)z[m] + half;
        }
    }
    return false;
}

template <int N, int EPL>
__device__ __forceinline__ uint32_t sign_bits(const unsigned long long *tab, int sign_words, uint64_t sign_key,
                                              uint64_t j, int l)
{
    constexpr int WPT = N / 64 > 0 ? N / 64 : 1;
    const uint32_t i0 = (uint32_t)l * EPL;
    const uint64_t w = sign_words ? tab[j * WPT + (i0 >> 6)] : mix64(mix64(sign_key ^ j) ^ (uint64_t)(i0 >> 6));
    return (uint32_t)(w >> (i0 & 63));
}

template <int N>
__device__ __forceinline__ void build_sign_table(unsigned long long *tab, int sign_words, uint64_t sign_key)
{
    constexpr int WPT = N / 64 > 0 ? N / 64 : 1;
    for (int i = threadIdx.x; i < sign_words; i += blockDim.x)
        tab[i] = mix64(mix64(sign_key ^ (uint64_t)(i / WPT)) ^ (uint64_t)(i % WPT));
}

}  // namespace hq
