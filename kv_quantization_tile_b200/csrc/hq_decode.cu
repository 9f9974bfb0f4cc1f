// hq_decode.cu -- tile decoder and fused batch-1 decode-GEMV for sm_100a.
//
// A group of LPT lanes parses one tile: its words are staged in shared
// memory; coset bits and the fixed-width low parts are read at computed bit
// offsets; the unary parts are located in parallel (each lane takes one word,
// popcounts it, a group prefix sum ranks its one bits, and each one bit's
// position is stored under its rank, so q_i = P_i - P_{i-1} - 1).  Every read
// stays inside the tile's own words; a tile that is not canonical (offsets out
// of order or past the capacity, k > 15, a count of one bits other than n, a
// word count other than the bits need) decodes to zeros with HQ_ST_CORRUPT.
//
// Decode:  w_hat = s . H (Delta (y [- dither])) / n   (register + shuffle
//          Walsh-Hadamard transform, 128-bit stores).
// GEMV:    y_r = sum_j (Delta_rj / n) <y_rj, H (s_j . x_j)>; each block first
//          rotates x into shared memory (the per-tile inverse transform drops
//          out because H is symmetric), then each warp streams the tiles of
//          its rows.
//
// Method: [V2] "HyperQuant: A Near-Entropy-Optimal Lattice Quantization
// Pipeline for Large Language and Diffusion Models", abstract (algebraic
// decoding; batch-1 decode against bf16 GEMV; subtractive dither).
#include <cuda_bf16.h>

#include "hq_internal.h"

namespace hq {

namespace {

// Parse tile t into the lattice point coordinates pt (binary32).  Returns
// true if the tile is not canonical (pt is then zero).  sb receives the bf16
// bits of Delta.  Group-uniform control flow; uses wbuf (wmax + 2 words) and
// pos (N entries) of this group.
template <int N, int D, int EPL>
__device__ __forceinline__ bool parse_tile(const DecodeArgs &a, int64_t t, uint32_t *wbuf,
                                           uint16_t *pos, unsigned mask, int l, float (&pt)[EPL],
                                           uint32_t &sb)
{
    constexpr int LPT = N / EPL;
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;
    constexpr int VPL = EPL / D;

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
    if (l < 2) wbuf[W + l] = 0u;
    __syncwarp(mask);

    uint32_t cb = 0, low[EPL];
#pragma unroll
    for (int r = 0; r < EPL; r++) low[r] = 0;
    if (!bad) {
        if constexpr (C > 0) cb = get_bits(wbuf, (uint32_t)l * VPL, VPL);
        if (k) {
#pragma unroll
            for (int r = 0; r < EPL; r++) low[r] = get_bits(wbuf, (uint32_t)C + ((uint32_t)l * EPL + r) * k, k);
        }
        uint32_t found = 0;
        const uint32_t wu0 = U0 >> 5;
        for (uint32_t wb = wu0; wb < W; wb += LPT) {
            const uint32_t wi = wb + l;
            uint32_t val = wi < W ? wbuf[wi] : 0u;
            if (wi == wu0) val &= 0xffffffffu << (U0 & 31);
            const uint32_t cnt = __popc(val);
            uint32_t r = found + group_excl_scan<LPT>(mask, cnt, l);
            while (val) {
                const uint32_t b = __ffs(val) - 1;
                val &= val - 1;
                if (r < (uint32_t)N) pos[r] = (uint16_t)(wi * 32u + b - U0);
                ++r;
            }
            found += group_sum<LPT>(mask, cnt);
        }
        if (found != (uint32_t)N) bad = true;
    }
    __syncwarp(mask);
    if (!bad && ((U0 + (uint32_t)pos[N - 1]) >> 5) != W - 1) bad = true;

#pragma unroll
    for (int r = 0; r < EPL; r++) pt[r] = 0.0f;
    if (bad) sb = 0;
    if (!bad) {
        uint32_t u[EPL];
#pragma unroll
        for (int r = 0; r < EPL; r++) {
            const int i = l * EPL + r;
            const int p1 = pos[i];
            const int p0 = i ? (int)pos[i - 1] : -1;
            u[r] = ((uint32_t)(p1 - p0 - 1) << k) | low[r];
        }
#pragma unroll
        for (int q = 0; q < VPL; q++) {
            int z[D];
#pragma unroll
            for (int m = 0; m < D; m++) z[m] = unzigzag(u[q * D + m]);
            if constexpr (D == 8 || D == 4) {
                int s = 0;
#pragma unroll
                for (int m = 0; m < D - 1; m++) s += z[m];
                z[D - 1] = 2 * z[D - 1] + (s & 1);
            }
            const float half = ((cb >> q) & 1u) ? 0.5f : 0.0f;
            if constexpr (D == 2) {
                pt[q * 2] = (float)z[0] + half;
                pt[q * 2 + 1] = __fmul_rn((float)z[1] + half, a.a2.s3);
            } else {
#pragma unroll
                for (int m = 0; m < D; m++) pt[q * D + m] = (float)z[m] + half;
            }
        }
    }
    return bad;
}

template <int EPL>
__device__ __forceinline__ uint32_t sign_bits(uint64_t sign_key, uint64_t j, int l)
{
    const uint32_t i0 = (uint32_t)l * EPL;
    return (uint32_t)(mix64(mix64(sign_key ^ j) ^ (uint64_t)(i0 >> 6)) >> (i0 & 63));
}

}  // namespace

template <int N, int D, int EPL, bool DITHER, bool F32OUT, int NWARPS>
__global__ void __launch_bounds__(NWARPS * 32) decode_kernel(const DecodeArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = NWARPS * TPW;
    constexpr int VPL = EPL / D;
    extern __shared__ uint32_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    uint32_t *wbuf = sm + gid * (a.wmax + 2);
    uint16_t *pos = reinterpret_cast<uint16_t *>(sm + GPB * (a.wmax + 2)) + gid * N;

    for (int64_t t = (int64_t)blockIdx.x * GPB + gid; t < a.ntiles; t += (int64_t)gridDim.x * GPB) {
        float pt[EPL];
        uint32_t sb;
        const bool bad = parse_tile<N, D, EPL>(a, t, wbuf, pos, mask, l, pt, sb);
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
        const float delta = bf16_bits_to_float(sb);
        float v[EPL];
#pragma unroll
        for (int r = 0; r < EPL; r++) v[r] = __fmul_rn(delta, pt[r]);
        fwht<EPL, LPT>(v, mask, l);
        const uint64_t j = (uint64_t)(t % a.tiles_per_row);
        const uint32_t sbits = sign_bits<EPL>(a.sign_key, j, l);
        constexpr float inv_n = 1.0f / N;
#pragma unroll
        for (int r = 0; r < EPL; r++)
            v[r] = __uint_as_float(__float_as_uint(__fmul_rn(v[r], inv_n)) ^ (((sbits >> r) & 1u) << 31));
        const int64_t e0 = t * N + (int64_t)l * EPL;
        if constexpr (F32OUT) {
            float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(a.y) + e0);
#pragma unroll
            for (int i = 0; i < EPL / 4; i++) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
            uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.y) + e0);
#pragma unroll
            for (int i = 0; i < EPL / 8; i++) {
                uint32_t q[4];
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[8 * i + 2 * h]));
                    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[8 * i + 2 * h + 1]));
                    q[h] = lo | (hi << 16);
                }
                o[i] = make_uint4(q[0], q[1], q[2], q[3]);
            }
        }
        if (bad && l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
    }
}

template <int N, int D, int EPL, int NWARPS>
__global__ void __launch_bounds__(NWARPS * 32) gemv_kernel(const DecodeArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = NWARPS * TPW;
    extern __shared__ uint32_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    const int64_t tpr = a.tiles_per_row;
    float *xt = reinterpret_cast<float *>(sm);
    uint32_t *wbuf = sm + tpr * N + gid * (a.wmax + 2);
    uint16_t *pos = reinterpret_cast<uint16_t *>(sm + tpr * N + GPB * (a.wmax + 2)) + gid * N;

    // rotated x: xt_j = H (s_j . x_j) for every column tile j
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
        const uint32_t sbits = sign_bits<EPL>(a.sign_key, (uint64_t)j, l);
#pragma unroll
        for (int r = 0; r < EPL; r++) v[r] = __uint_as_float(__float_as_uint(v[r]) ^ (((sbits >> r) & 1u) << 31));
        fwht<EPL, LPT>(v, mask, l);
#pragma unroll
        for (int r = 0; r < EPL; r++) xt[j * N + l * EPL + r] = v[r];
    }
    __syncthreads();

    constexpr float inv_n = 1.0f / N;
    for (int64_t row = (int64_t)blockIdx.x * NWARPS + warp; row < a.rows; row += (int64_t)gridDim.x * NWARPS) {
        float acc = 0.0f;
        for (int64_t j = lane / LPT; j < tpr; j += TPW) {
            const int64_t t = row * tpr + j;
            float pt[EPL];
            uint32_t sb;
            const bool bad = parse_tile<N, D, EPL>(a, t, wbuf, pos, mask, l, pt, sb);
            const float *xr = xt + j * N + l * EPL;
            float dot = 0.0f;
#pragma unroll
            for (int r = 0; r < EPL; r++) dot = fmaf(pt[r], xr[r], dot);
            acc = fmaf(bf16_bits_to_float(sb) * inv_n, dot, acc);
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

constexpr int kDecodeWarps = 8;

template <int N>
constexpr int epl_for() { return N <= 256 ? 8 : N / 32; }

template <int N>
constexpr int groups_per_block() { return kDecodeWarps * (32 / (N / epl_for<N>())); }

template <typename K>
cudaError_t prepare(K kern, size_t smem)
{
    if (smem > 48 * 1024)
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return cudaSuccess;
}

template <int N, int D, bool DITHER, bool F32OUT>
cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t s)
{
    constexpr int EPL = epl_for<N>(), GPB = groups_per_block<N>();
    const size_t smem = (size_t)GPB * (a.wmax + 2) * 4 + (size_t)GPB * N * 2;
    auto kern = decode_kernel<N, D, EPL, DITHER, F32OUT, kDecodeWarps>;
    cudaError_t e = prepare(kern, smem);
    if (e != cudaSuccess) return e;
    int64_t blocks = (a.ntiles + GPB - 1) / GPB;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    kern<<<(unsigned)blocks, kDecodeWarps * 32, smem, s>>>(a);
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
    const size_t smem = (size_t)cols * 4 + (size_t)GPB * (a.wmax + 2) * 4 + (size_t)GPB * N * 2;
    auto kern = gemv_kernel<N, D, EPL, kDecodeWarps>;
    cudaError_t e = prepare(kern, smem);
    if (e != cudaSuccess) return e;
    int64_t blocks = (a.rows + kDecodeWarps - 1) / kDecodeWarps;
    int per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = (int64_t)sm_count() * per_sm;
    if (blocks > cap) blocks = cap;
    kern<<<(unsigned)blocks, kDecodeWarps * 32, smem, s>>>(a);
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
