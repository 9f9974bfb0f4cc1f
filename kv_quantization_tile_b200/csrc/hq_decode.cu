// hq_decode.cu -- tile decoder and fused batch-1 decode-GEMV for sm_100a.
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
// other than its bits need) decodes to zeros with HQ_ST_CORRUPT.
//
// Decode:  w_hat = s . H ((Delta / n) (y [- dither]))  (register + shuffle
//          Walsh-Hadamard transform, 128-bit stores).
// GEMV:    y_r = sum_j (Delta_rj / n) <y_rj, H (s_j . x_j)>; each block first
//          rotates x into shared memory (the per-tile inverse transform drops
//          out because H is symmetric), then each warp streams its rows.
//
// Method: [V2] "HyperQuant: A Near-Entropy-Optimal Lattice Quantization
// Pipeline for Large Language and Diffusion Models", abstract (algebraic
// decoding; batch-1 decode against bf16 GEMV; subtractive dither).
#include <cuda_bf16.h>

#include "hq_internal.h"

namespace hq {

namespace {

constexpr int kDecodeWarps = 8;

// words of shared memory per group: staged tile words + 4 guard words, then
// the running terminator count of each unary word
__host__ __device__ constexpr uint32_t group_words(uint32_t wmax) { return 2 * wmax + 4; }

__device__ __forceinline__ uint32_t shl32(uint32_t v, uint32_t s)
{
    uint32_t r;
    asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(s));
    return r;
}

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

}  // namespace

template <int N, int D, int EPL, bool DITHER, bool F32OUT>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const DecodeArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = kDecodeWarps * TPW;
    constexpr int VPL = EPL / D;
    extern __shared__ __align__(16) uint32_t sm[];
    unsigned long long *sign_tab = reinterpret_cast<unsigned long long *>(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    uint32_t *wbuf = sm + 2 * a.sign_words + gid * group_words(a.wmax);
    build_sign_table<N>(sign_tab, a.sign_words, a.sign_key);
    __syncthreads();

    for (int64_t t = (int64_t)blockIdx.x * GPB + gid; t < a.ntiles; t += (int64_t)gridDim.x * GPB) {
        float pt[EPL];
        uint32_t sb;
        const bool bad = parse_tile<N, D, EPL>(a, t, wbuf, mask, l, pt, sb);
        if constexpr (DITHER) {
            if (!bad && sb) {
                const uint64_t tkey = mix64(a.dither_key ^ (uint64_t)t);
#pragma unroll
                for (int q = 0; q < VPL; q++) {
                    float dl[D];
                    dither<D>(tkey, (uint32_t)(l * VPL + q), dl, a.a2);
#pragma unroll
                    for (int m = 0; m < D; m++) pt[q * D + m] = __fsub_rn(pt[q * D + m], dl[m]);
                }
            }
        }
        const float scale = bf16_bits_to_float(sb) * (1.0f / N);  // exact: a power-of-two step
        float v[EPL];
#pragma unroll
        for (int r = 0; r < EPL; r++) v[r] = pt[r] * scale;
        fwht<EPL, LPT>(v, mask, l);
        const uint64_t j = (uint32_t)t - fast_div((uint32_t)t, a.tpr_div) * (uint32_t)a.tiles_per_row;
        const uint32_t sbits = sign_bits<N, EPL>(sign_tab, a.sign_words, a.sign_key, j, l);
#pragma unroll
        for (int r = 0; r < EPL; r++) v[r] = __uint_as_float(__float_as_uint(v[r]) ^ ((sbits << (31 - r)) & 0x80000000u));
        const int64_t e0 = t * N + (int64_t)l * EPL;
        if constexpr (F32OUT) {
            float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(a.y) + e0);
#pragma unroll
            for (int i = 0; i < EPL / 4; i++) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
            uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.y) + e0);
#pragma unroll
            for (int i = 0; i < EPL / 8; i++) {
                uint32_t qq[4];
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    const __nv_bfloat162 p2 = __floats2bfloat162_rn(v[8 * i + 2 * h], v[8 * i + 2 * h + 1]);
                    qq[h] = *reinterpret_cast<const uint32_t *>(&p2);
                }
                o[i] = make_uint4(qq[0], qq[1], qq[2], qq[3]);
            }
        }
        if (bad && l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
    }
}

template <int N, int D, int EPL>
__global__ void __launch_bounds__(kDecodeWarps * 32) gemv_kernel(const DecodeArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = kDecodeWarps * TPW;
    constexpr int SW = EPL / 4 - 1;
    extern __shared__ __align__(16) uint32_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    const int64_t tpr = a.tiles_per_row;
    unsigned long long *sign_tab = reinterpret_cast<unsigned long long *>(sm);
    float *xt = reinterpret_cast<float *>(sm + 2 * a.sign_words);
    uint32_t *wbuf = sm + 2 * a.sign_words + tpr * N + gid * group_words(a.wmax);
    build_sign_table<N>(sign_tab, a.sign_words, a.sign_key);
    __syncthreads();

    // rotated x: xt_j = H (s_j . x_j); lane l's EPL values stored as EPL/4
    // 16-byte chunks, chunk c at slot c ^ (l & SW) (conflict-free 128-bit reads)
    for (int64_t j = gid; j < tpr; j += GPB) {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(a.x) + j * N + l * EPL);
        float v[EPL];
#pragma unroll
        for (int i = 0; i < EPL / 8; i++) {
            uint4 q = __ldg(p + i);
            const uint32_t qq[4] = { q.x, q.y, q.z, q.w };
#pragma unroll
            for (int h = 0; h < 4; h++) {
                v[8 * i + 2 * h] = __uint_as_float(qq[h] << 16);
                v[8 * i + 2 * h + 1] = __uint_as_float(qq[h] & 0xffff0000u);
            }
        }
        const uint32_t sbits = sign_bits<N, EPL>(sign_tab, a.sign_words, a.sign_key, (uint64_t)j, l);
#pragma unroll
        for (int r = 0; r < EPL; r++) v[r] = __uint_as_float(__float_as_uint(v[r]) ^ ((sbits << (31 - r)) & 0x80000000u));
        fwht<EPL, LPT>(v, mask, l);
        float4 *dst = reinterpret_cast<float4 *>(xt + j * N + l * EPL);
#pragma unroll
        for (int c = 0; c < EPL / 4; c++)
            dst[c ^ (l & SW)] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
    __syncthreads();

    for (int64_t row = (int64_t)blockIdx.x * kDecodeWarps + warp; row < a.rows; row += (int64_t)gridDim.x * kDecodeWarps) {
        float acc = 0.0f;
        for (int64_t j = lane / LPT; j < tpr; j += TPW) {
            const int64_t t = row * tpr + j;
            float pt[EPL];
            uint32_t sb;
            const bool bad = parse_tile<N, D, EPL>(a, t, wbuf, mask, l, pt, sb);
            const float4 *src = reinterpret_cast<const float4 *>(xt + j * N + l * EPL);
            float dot = 0.0f;
#pragma unroll
            for (int c = 0; c < EPL / 4; c++) {
                const float4 xv = src[c ^ (l & SW)];
                dot = fmaf(pt[4 * c], xv.x, dot);
                dot = fmaf(pt[4 * c + 1], xv.y, dot);
                dot = fmaf(pt[4 * c + 2], xv.z, dot);
                dot = fmaf(pt[4 * c + 3], xv.w, dot);
            }
            acc = fmaf(bf16_bits_to_float(sb) * (1.0f / N), dot, acc);
            if (bad && l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
        }
        __syncwarp();
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(FULL, acc, m);
        if (lane == 0) a.gy[row] = acc;
    }
}

// ------------------------------------------------------------------ launch
namespace {

template <int N>
constexpr int epl_for() { return N == 64 ? 8 : (N <= 256 ? 16 : 32); }

template <int N>
constexpr int groups_per_block() { return kDecodeWarps * (32 / (N / epl_for<N>())); }

template <typename K>
cudaError_t grid_for(K kern, size_t smem, int64_t work_blocks, unsigned &blocks)
{
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t b = (int64_t)sm_count() * per_sm;
    if (b > work_blocks) b = work_blocks;
    if (b < 1) b = 1;
    blocks = (unsigned)b;
    return cudaSuccess;
}

template <int N, int D, bool DITHER, bool F32OUT>
cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t s)
{
    constexpr int EPL = epl_for<N>(), GPB = groups_per_block<N>();
    const size_t smem = (size_t)a.sign_words * 8 + (size_t)GPB * group_words(a.wmax) * 4;
    auto kern = decode_kernel<N, D, EPL, DITHER, F32OUT>;
    unsigned blocks = 0;
    cudaError_t e = grid_for(kern, smem, (a.ntiles + GPB - 1) / GPB, blocks);
    if (e != cudaSuccess) return e;
    kern<<<blocks, kDecodeWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int N, int D>
cudaError_t launch_decode_nd(bool dither, int dtype, const DecodeArgs &a, cudaStream_t s)
{
    if (dither) return dtype ? launch_decode_t<N, D, true, true>(a, s) : launch_decode_t<N, D, true, false>(a, s);
    return dtype ? launch_decode_t<N, D, false, true>(a, s) : launch_decode_t<N, D, false, false>(a, s);
}

template <int N>
cudaError_t launch_decode_n(int lattice, bool dither, int dtype, const DecodeArgs &a, cudaStream_t s)
{
    switch (lattice) {
    case 1: return launch_decode_nd<N, 1>(dither, dtype, a, s);
    case 2: return launch_decode_nd<N, 2>(dither, dtype, a, s);
    case 4: return launch_decode_nd<N, 4>(dither, dtype, a, s);
    default: return launch_decode_nd<N, 8>(dither, dtype, a, s);
    }
}

template <int N, int D>
cudaError_t launch_gemv_t(const DecodeArgs &a, int64_t cols, cudaStream_t s)
{
    constexpr int EPL = epl_for<N>(), GPB = groups_per_block<N>();
    const size_t smem = (size_t)a.sign_words * 8 + (size_t)cols * 4 + (size_t)GPB * group_words(a.wmax) * 4;
    auto kern = gemv_kernel<N, D, EPL>;
    unsigned blocks = 0;
    cudaError_t e = grid_for(kern, smem, (a.rows + kDecodeWarps - 1) / kDecodeWarps, blocks);
    if (e != cudaSuccess) return e;
    kern<<<blocks, kDecodeWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int N>
cudaError_t launch_gemv_n(int lattice, const DecodeArgs &a, int64_t cols, cudaStream_t s)
{
    switch (lattice) {
    case 1: return launch_gemv_t<N, 1>(a, cols, s);
    case 2: return launch_gemv_t<N, 2>(a, cols, s);
    case 4: return launch_gemv_t<N, 4>(a, cols, s);
    default: return launch_gemv_t<N, 8>(a, cols, s);
    }
}

}  // namespace

cudaError_t launch_decode(int tile, int lattice, bool dither, int dtype, const DecodeArgs &a,
                          cudaStream_t s)
{
    switch (tile) {
    case 64: return launch_decode_n<64>(lattice, dither, dtype, a, s);
    case 128: return launch_decode_n<128>(lattice, dither, dtype, a, s);
    case 256: return launch_decode_n<256>(lattice, dither, dtype, a, s);
    case 512: return launch_decode_n<512>(lattice, dither, dtype, a, s);
    default: return launch_decode_n<1024>(lattice, dither, dtype, a, s);
    }
}

cudaError_t launch_gemv(int tile, int lattice, const DecodeArgs &a, int64_t cols, cudaStream_t s)
{
    switch (tile) {
    case 64: return launch_gemv_n<64>(lattice, a, cols, s);
    case 128: return launch_gemv_n<128>(lattice, a, cols, s);
    case 256: return launch_gemv_n<256>(lattice, a, cols, s);
    case 512: return launch_gemv_n<512>(lattice, a, cols, s);
    default: return launch_gemv_n<1024>(lattice, a, cols, s);
    }
}

}  // namespace hq
