// hq_parse.cuh -- tile parser shared by the decoder, the decode-GEMV and the
// KV-cache attention kernels (see hq_decode.cu for the method).
//
// A group of LPT lanes parses one tile; lane l owns codes l*EPL .. l*EPL+EPL-1.
//   * The tile's words are staged in shared memory (plus zero guard words).
//   * Coset bits and the fixed-width low parts are read at computed offsets.
//   * Unary parts: one pass popcounts the unary words (two per lane) and
//     scans the counts across the group; lane m finds the word holding
//     terminator m*EPL - 1 by a binary search over the scanned counts and
//     selects the bit (its start is the bit after that terminator), all
//     lanes in step.  Each lane then parses its EPL codes
//     from a bit-reversed 64-bit window with one count-leading-zeros and two
//     funnel shifts per code, once it has checked that no zero run of its
//     span reaches 32 bits; otherwise (and for spans over 64 bits) it parses
//     from shared memory word by word.
// Every read stays inside the tile's own words.  A tile that is not canonical
// (offsets out of order or past the capacity, k > 15, a scale that is not 0
// or a positive normal bf16, a terminator count other than n, a word count
// other than its bits need) parses to zeros and is reported as bad.
// A fixed-rate stream (FIXED, a.slot > 0) puts tile t at words [t S, t S + S) and
// its k in 4 bits; the slot may end in zero words, so only the word-count
// rule is dropped.  For both kinds the last lane's span ends at the last one
// bit of the tile's words (a max over the group finds its word).
#pragma once

#include "hq_internal.h"

namespace hq {

// words of shared memory per group: staged tile words + 4 guard words
__host__ __device__ constexpr uint32_t group_words(uint32_t wmax) { return wmax + 4; }

// position of the r-th (0-based) set bit of v (v has more than r set bits):
// a branch-free binary search on popcounts of halves
__device__ __forceinline__ uint32_t select_bit(uint32_t v, uint32_t r)
{
    uint32_t pos = 0, c;
    c = __popc(v & 0xffffu);
    if (r >= c) { r -= c; pos = 16; }
    c = __popc((v >> pos) & 0xffu);
    if (r >= c) { r -= c; pos += 8; }
    c = __popc((v >> pos) & 0xfu);
    if (r >= c) { r -= c; pos += 4; }
    c = __popc((v >> pos) & 0x3u);
    if (r >= c) { r -= c; pos += 2; }
    c = (v >> pos) & 1u;
    if (r >= c) pos += 1;
    return pos;
}

// A tile's header as the parser reads it: word offset, words (0 if the header
// is not canonical), Rice parameter and scale bits.
struct TileHdr {
    uint32_t o0, W, sb;
    int k;
    bool bad;
};

// Load tile t's header and check it (offsets in order and inside the
// capacity, k <= 15, Delta zero or a positive normal finite bf16, enough
// words for the coset bits, the low parts and n terminators).
template <int N, int D, bool FIXED>
__device__ __forceinline__ TileHdr tile_header(const DecodeArgs &a, int64_t t)
{
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;
    TileHdr h;
    uint32_t o1;
    if constexpr (FIXED) {
        h.o0 = (uint32_t)t * a.slot;  // the host keeps ntiles * slot below 2^32
        o1 = h.o0 + a.slot;
        h.k = (a.kk[t >> 1] >> ((t & 1) * 4)) & 15;
    } else {
        h.o0 = a.off[t];
        o1 = a.off[t + 1];
        h.k = a.kk[t];
    }
    h.sb = a.scale[t];
    const uint32_t ex = h.sb & 0x7f80u;
    h.bad = (o1 < h.o0) || (o1 - h.o0 > a.wmax) || ((uint64_t)o1 > a.cap) || (h.k > 15) || (h.sb & 0x8000u) ||
            ex == 0x7f80u || (h.sb != 0 && ex == 0);
    const uint32_t U0 = (uint32_t)C + (uint32_t)N * (uint32_t)h.k;
    const uint32_t W0 = h.bad ? 0u : o1 - h.o0;
    if (!h.bad && U0 + (uint32_t)N > 32u * W0) h.bad = true;
    h.W = h.bad ? 0u : W0;
    return h;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Start copying the tile's words into the group's staging buffer (cp.async,
// no registers held; each lane copies words l, l + LPT, ...) and write the
// four zero guard words.  The caller commits the group and waits for it.
template <int LPT>
__device__ __forceinline__ void stage_async(const DecodeArgs &a, const TileHdr &h, uint32_t *wbuf, int l)
{
    for (uint32_t i = l; i < h.W; i += LPT)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(wbuf + i)), "l"(a.payload + h.o0 + i)
                     : "memory");
    if (l < 4) wbuf[h.W + l] = 0u;
}

__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Parse a staged tile (header h, words in wbuf) into lane l's symbols u
// (zigzagged stripped coordinates, code order) and coset bits cb (bit q: the
// lane's vector q).  Returns true if the tile is not canonical (u, cb and sb
// are then zero).  small: every code's unary part is shorter than 32 bits, so
// u < 2^20.
template <int N, int D, int EPL, bool FIXED>
__device__ __forceinline__ bool parse_staged(const DecodeArgs &a, const TileHdr &h, uint32_t *wbuf, unsigned mask,
                                             int l, uint32_t (&u)[EPL], uint32_t &cb, uint32_t &sb, bool &small)
{
    constexpr int LPT = N / EPL;
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;
    constexpr int VPL = EPL / D;
    constexpr bool fixed = FIXED;
    const int k = h.k;
    bool bad = h.bad;
    const uint32_t W = h.W;
    sb = h.sb;
    const uint32_t U0 = (uint32_t)C + (uint32_t)N * (uint32_t)k;

    // ---- unary terminators: lane l counts the ones of unary words 2l, 2l + 1
    // of each pass of 2 LPT words, the counts are scanned across the group,
    // and lane m (m >= 1) finds the word pair holding terminator m EPL - 1
    // by a binary search over the scanned counts (shuffles, no divergence),
    // then the bit by a select: its start is the bit after that terminator.
    const uint32_t wu0 = U0 >> 5;
    const uint32_t nwu = W > wu0 ? W - wu0 : 0;  // unary words (the first shared with the low parts)
    uint32_t found = 0, last_nz = 0;  // last_nz: 1 + the last unary word holding a one bit
    uint32_t start = 0;
    const uint32_t target = (uint32_t)l * EPL - 1u;  // lane l's terminator (l >= 1)
    for (uint32_t wb = 0; wb < nwu; wb += 2 * LPT) {
        const uint32_t wi = wb + 2 * (uint32_t)l;
        uint32_t v0 = wi < nwu ? wbuf[wu0 + wi] : 0u;
        const uint32_t v1 = wi + 1 < nwu ? wbuf[wu0 + wi + 1] : 0u;
        if (wi == 0) v0 &= 0xffffffffu << (U0 & 31);
        const uint32_t c0 = __popc(v0), c = c0 + __popc(v1);
        uint32_t incl = c;
#pragma unroll
        for (int d = 1; d < LPT; d <<= 1) {
            const uint32_t o = __shfl_up_sync(mask, incl, d, LPT);
            if (l >= d) incl += o;
        }
        if (v1) last_nz = wi + 2;
        else if (v0) last_nz = wi + 1;
        const uint32_t total = __shfl_sync(mask, incl, LPT - 1, LPT);
        const uint32_t rel = target - found;  // wraps for a target before this pass
        int w = 0;  // first lane whose inclusive count exceeds rel
#pragma unroll
        for (int sh = LPT / 2; sh >= 1; sh >>= 1) {
            const uint32_t o = __shfl_sync(mask, incl, w + sh - 1, LPT);
            if (o <= rel) w += sh;
        }
        const uint32_t ex = __shfl_sync(mask, incl - c, w, LPT);
        const uint32_t a0 = __shfl_sync(mask, v0, w, LPT), a1 = __shfl_sync(mask, v1, w, LPT);
        const uint32_t ac0 = __shfl_sync(mask, c0, w, LPT);
        if (l > 0 && rel < total) {
            const uint32_t r = rel - ex;
            const uint32_t bit = r < ac0 ? select_bit(a0, r) : 32u + select_bit(a1, r - ac0);
            start = (wu0 + wb + 2u * (uint32_t)w) * 32u + bit + 1u - U0;
        }
        found += total;
    }
    last_nz = group_max<LPT>(mask, last_nz);
    // a variable-rate tile ends in its last word (no whole word of padding)
    if (!bad && (found != (uint32_t)N || (!fixed && last_nz != nwu))) bad = true;

#pragma unroll
    for (int r = 0; r < EPL; r++) u[r] = 0;
    cb = 0;
    small = true;
    if (bad) {
        sb = 0;
        return true;
    }

    // the next lane's start bounds this lane's codes
    uint32_t end = __shfl_down_sync(mask, start, 1, LPT);
    if (l == LPT - 1) {
        // the word of the tile's last terminator: the last unary word holding
        // a one bit (the last word of a variable-rate tile)
        const uint32_t wl = wu0 + last_nz - 1u;
        const uint32_t v = wbuf[wl] & (wl == wu0 ? (0xffffffffu << (U0 & 31)) : 0xffffffffu);
        end = wl * 32u + (31u - __clz(v)) + 1u - U0;
    }

    // ---- coset bits and low parts
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
    // the lane's span in a bit-reversed 64-bit window (next bit at the MSB);
    // bits past the span are set so they cannot lengthen a zero run
    const uint32_t w0 = p0 >> 5, sh = p0 & 31;
    const uint32_t b0 = wbuf[w0], b1 = wbuf[w0 + 1], b2 = wbuf[w0 + 2];
    uint32_t rh = __brev(__funnelshift_r(b0, b1, sh));
    uint32_t rl = __brev(__funnelshift_r(b1, b2, sh));
    if (span < 64) {
        rl |= span >= 32 ? (0xffffffffu >> (span - 32)) : 0xffffffffu;
        rh |= span < 32 ? (0xffffffffu >> span) : 0u;
    }
    // every zero run shorter than 32 bits: each terminator sits in rh
    if (span <= 64 && rh != 0 && rl != 0 && (__ffs(rh) - 1u) + __clz(rl) < 32u) {
#pragma unroll
        for (int r = 0; r < EPL; r++) {
            const uint32_t z = __clz(rh);
            q[r] = z;
            rh = __funnelshift_lc(rl, rh, z + 1);  // a shift of 32 moves rl into rh
            rl = shl32(rl, z + 1);
        }
    } else {
        small = false;
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

    const uint32_t p2k = 1u << k;
#pragma unroll
    for (int r = 0; r < EPL; r++) u[r] = q[r] * p2k + low[r];  // (q << k) | low: the low part is below 2^k
    return false;
}

// Load, stage and parse tile t (parse_staged with synchronous staging).
template <int N, int D, int EPL, bool FIXED>
__device__ __forceinline__ bool parse_symbols(const DecodeArgs &a, int64_t t, uint32_t *wbuf, unsigned mask, int l,
                                              uint32_t (&u)[EPL], uint32_t &cb, uint32_t &sb, bool &small)
{
    constexpr int LPT = N / EPL;
    const TileHdr h = tile_header<N, D, FIXED>(a, t);
    __syncwarp(mask);  // the group is done with the previous tile's words
    for (uint32_t i = l; i < h.W; i += LPT) wbuf[i] = __ldg(a.payload + h.o0 + i);
    if (l < 4) wbuf[h.W + l] = 0u;
    __syncwarp(mask);
    return parse_staged<N, D, EPL, FIXED>(a, h, wbuf, mask, l, u, cb, sb, small);
}

// Lattice point coordinates (binary32) of lane's vectors from their symbols.
template <int D, int EPL>
__device__ __forceinline__ void points_from_symbols(const uint32_t (&u)[EPL], uint32_t cb, const A2Consts &a2,
                                                    float (&pt)[EPL])
{
    constexpr int VPL = EPL / D;
#pragma unroll
    for (int qv = 0; qv < VPL; qv++) {
        int z[D];
#pragma unroll
        for (int m = 0; m < D; m++) z[m] = unzigzag(u[qv * D + m]);
        if constexpr (D == 8 || D == 4) {
            int s = 0;
#pragma unroll
            for (int m = 0; m < D - 1; m++) s += z[m];
            z[D - 1] = 2 * z[D - 1] + (s & 1);
        }
        const float half = ((cb >> qv) & 1u) ? 0.5f : 0.0f;
        if constexpr (D == 2) {
            pt[qv * 2] = (float)z[0] + half;
            pt[qv * 2 + 1] = __fmul_rn((float)z[1] + half, a2.s3);
        } else {
#pragma unroll
            for (int m = 0; m < D; m++) pt[qv * D + m] = (float)z[m] + half;
        }
    }
}

// Doubled lattice coordinates t = 2y of lane's vectors from their symbols
// (D = 1, 4, 8: integer points, E8's half-integer coset odd).  With z the
// unzigzagged symbol, 2z = u ^ -(u & 1); a stripped last coordinate s =
// floor(z / 2) is restored as 2z = 2 (2s) + 2 parity(sum of the others), that
// parity being bit 1 of the XOR of the others' 2z.  `bias` is added to every
// coordinate (with the coset), e.g. the bit pattern of 1.5 2^23.
template <int D, int EPL>
__device__ __forceinline__ void doubled_from_symbols(const uint32_t (&u)[EPL], uint32_t cb, int32_t (&t)[EPL],
                                                     int32_t bias = 0)
{
    static_assert(D != 2, "A2 has no integer form");
    constexpr int VPL = EPL / D;
#pragma unroll
    for (int qv = 0; qv < VPL; qv++) {
        int32_t d2[D];
#pragma unroll
        for (int m = 0; m < D; m++) d2[m] = (int32_t)(u[qv * D + m] ^ (0u - (u[qv * D + m] & 1u)));
        if constexpr (D == 8 || D == 4) {
            int32_t x = 0;
#pragma unroll
            for (int m = 0; m < D - 1; m++) x ^= d2[m];
            d2[D - 1] = 2 * d2[D - 1] + (x & 2);
        }
        const int32_t c = ((D == 8) ? (int32_t)((cb >> qv) & 1u) : 0) + bias;
#pragma unroll
        for (int m = 0; m < D; m++) t[qv * D + m] = d2[m] + c;
    }
}

// Parse tile t into lattice point coordinates pt (binary32).  Returns true
// if the tile is not canonical (pt is then zero and sb is 0).
template <int N, int D, int EPL, bool FIXED>
__device__ __forceinline__ bool parse_tile(const DecodeArgs &a, int64_t t, uint32_t *wbuf, unsigned mask, int l,
                                           float (&pt)[EPL], uint32_t &sb)
{
    uint32_t u[EPL], cb;
    bool small;
    const bool bad = parse_symbols<N, D, EPL, FIXED>(a, t, wbuf, mask, l, u, cb, sb, small);
    points_from_symbols<D, EPL>(u, cb, a.a2, pt);
    return bad;
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
