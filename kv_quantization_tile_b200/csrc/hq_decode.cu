// hq_decode.cu -- tile decoder and fused batch-1 decode-GEMV for sm_100a.
//
// The tile parser (hq_parse.cuh) stages a tile in shared memory, finds each
// lane's start with one select and parses the unary parts with one CLZ per
// code; non-canonical tiles decode to zeros with HQ_ST_CORRUPT.
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

#include "hq_fast.cuh"
#include "hq_parse.cuh"

namespace hq {

namespace {

constexpr int kDecodeWarps = 8;

}  // namespace

// Output sign word of lane l of column tile j after the half-exchange transform
// (see sign_word): pair m < EPL/4 holds tile coordinates RL l + 2m, + 1 (run
// A), pair m >= EPL/4 coordinates N/2 + RL l + 2(m - EPL/4), + 1 (run B), RL =
// EPL / 2; the transform's own signs on each run are folded in.
template <int N, int EPL>
__device__ __forceinline__ uint32_t decode_sign_word(uint64_t sign_key, uint64_t j, int l)
{
    constexpr int LPT = N / EPL, RL = EPL / 2, HP = EPL / 4;
    const uint32_t sig = hx_sigma_bits<LPT>(l);
    const uint32_t a0 = (uint32_t)l * RL, b0 = (uint32_t)N / 2 + (uint32_t)l * RL;
    const uint64_t wa = mix64(mix64(sign_key ^ j) ^ (uint64_t)(a0 >> 6));
    const uint64_t wb = mix64(mix64(sign_key ^ j) ^ (uint64_t)(b0 >> 6));
    const uint32_t sa = (uint32_t)(wa >> (a0 & 63)), sbb = (uint32_t)(wb >> (b0 & 63));
    return sign_word<EPL>([&](int i) {
        const int m = i >> 1;
        return m < HP ? (((sa >> i) & 1u) ^ (sig & 1u)) : (((sbb >> (i - 2 * HP)) & 1u) ^ (sig >> 1));
    });
}

template <int N, int D, int EPL, bool DITHER, bool F32OUT, bool FIXED>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const DecodeArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = kDecodeWarps * TPW;
    constexpr int NP = EPL / 2, HP = NP / 2, RL = EPL / 2;
    extern __shared__ __align__(16) uint32_t sm[];
    const int ywords = a.sign_words ? (int)a.tiles_per_row * LPT : 0;  // sign words cached per block
    uint32_t *ytab = sm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    // two staging buffers per group: the next tile's words arrive (cp.async)
    // while this one is parsed
    uint32_t *wb0 = sm + ((ywords + 3) & ~3) + gid * 2 * group_words(a.wmax);
    uint32_t *wb1 = wb0 + group_words(a.wmax);
    for (int i = threadIdx.x; i < ywords; i += blockDim.x)
        ytab[i] = decode_sign_word<N, EPL>(a.sign_key, (uint64_t)(i / LPT), i % LPT);
    __syncthreads();

    const int64_t stride = (int64_t)gridDim.x * GPB;
    int64_t t = (int64_t)blockIdx.x * GPB + gid;
    TileHdr h{};
    if (t < a.ntiles) {
        h = tile_header<N, D, FIXED>(a, t);
        stage_async<LPT>(a, h, wb0, l);
    }
    async_commit();
    for (; t < a.ntiles; t += stride) {
        const int64_t tn = t + stride;
        TileHdr hn{};
        if (tn < a.ntiles) {
            hn = tile_header<N, D, FIXED>(a, tn);
            stage_async<LPT>(a, hn, wb1, l);
        }
        async_commit();
        async_wait<1>();   // this tile's words have arrived
        __syncwarp(mask);  // ... for every lane of the group
        uint32_t u[EPL], cb, sb;
        bool small;
        const bool bad = parse_staged<N, D, EPL, FIXED>(a, h, wb0, mask, l, u, cb, sb, small);
        h = hn;
        uint32_t *tmp = wb0;
        wb0 = wb1;
        wb1 = tmp;
        __syncwarp(mask);  // the group is done with the words the next prefetch overwrites
        float2 v[NP];
        if constexpr (D != 2 && !DITHER) {
            // v = (Delta / n) y = (Delta / 2n) t with t = 2y an integer: t + 1.5 2^23
            // read as a float, times Delta / 2n, minus 1.5 2^23 Delta / 2n (exact:
            // 9 significant bits) in one fma -- the single rounding of t Delta / 2n.
            // Exact while |t| < 2^22, which a lane whose codes all have unary
            // parts under 32 bits guarantees (u < 2^20); otherwise convert.
            int32_t tt[EPL];  // t + 1.5 2^23 (bit patterns) where small, else t
            doubled_from_symbols<D, EPL>(u, cb, tt, small ? kMagicBias : 0);
            const float s2 = bf16_bits_to_float(sb) * (0.5f / N);  // exact: a power-of-two step
            if (small) {
                const float2 sc = splat2(s2), off = splat2(-12582912.0f * s2);
#pragma unroll
                for (int m = 0; m < NP; m++)
                    v[m] = fma2(make_float2(__int_as_float(tt[2 * m]), __int_as_float(tt[2 * m + 1])), sc, off);
            } else {
#pragma unroll
                for (int m = 0; m < NP; m++) v[m] = make_float2((float)tt[2 * m] * s2, (float)tt[2 * m + 1] * s2);
            }
        } else {
            float pt[EPL];
            points_from_symbols<D, EPL>(u, cb, a.a2, pt);
            if constexpr (DITHER) {
                if (!bad && sb) sub_dither<D, EPL>(mix64(a.dither_key ^ (uint64_t)t), l, pt, a.a2);
            }
            const float2 scale = splat2(bf16_bits_to_float(sb) * (1.0f / N));  // exact: a power-of-two step
#pragma unroll
            for (int m = 0; m < NP; m++) v[m] = mul2(make_float2(pt[2 * m], pt[2 * m + 1]), scale);
        }
        fwht_hx<EPL, LPT>(v, mask, l);
        const uint64_t j = (uint32_t)t - fast_div((uint32_t)t, a.tpr_div) * (uint32_t)a.tiles_per_row;
        const uint32_t Y = ywords ? ytab[j * LPT + l] : decode_sign_word<N, EPL>(a.sign_key, j, l);
        const int64_t eA = t * N + (int64_t)l * RL, eB = eA + N / 2;
        if constexpr (F32OUT) {
#pragma unroll
            for (int run = 0; run < 2; run++) {
                float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(a.y) + (run ? eB : eA));
#pragma unroll
                for (int i = 0; i < RL / 4; i++) {
                    const int m0 = run * HP + 2 * i;
                    const uint32_t s0 = Y << m0, s1 = Y << (m0 + 1);
                    o[i] = make_float4(__uint_as_float(__float_as_uint(v[m0].x) ^ ((s0 << 16) & 0x80000000u)),
                                       __uint_as_float(__float_as_uint(v[m0].y) ^ (s0 & 0x80000000u)),
                                       __uint_as_float(__float_as_uint(v[m0 + 1].x) ^ ((s1 << 16) & 0x80000000u)),
                                       __uint_as_float(__float_as_uint(v[m0 + 1].y) ^ (s1 & 0x80000000u)));
                }
            }
        } else {
#pragma unroll
            for (int run = 0; run < 2; run++) {
                uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.y) + (run ? eB : eA));
#pragma unroll
                for (int i = 0; i < RL / 8; i++) {
                    uint32_t qq[4];
#pragma unroll
                    for (int h = 0; h < 4; h++) {
                        const int m = run * HP + 4 * i + h;
                        const __nv_bfloat162 p2 = __floats2bfloat162_rn(v[m].x, v[m].y);
                        qq[h] = *reinterpret_cast<const uint32_t *>(&p2) ^ ((Y << m) & 0x80008000u);
                    }
                    o[i] = make_uint4(qq[0], qq[1], qq[2], qq[3]);
                }
            }
        }
        if (bad && l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
    }
}

template <int N, int D, int EPL, int W, bool FIXED>
__global__ void __launch_bounds__(W * 32, N <= 256 ? 32 / W : 1) gemv_kernel(const DecodeArgs a)  // 64 registers up to 256
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = W * TPW;
    constexpr int SW = EPL / 4 - 1;
    extern __shared__ __align__(16) uint32_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    const int64_t tpr = a.tiles_per_row;
    unsigned long long *sign_tab = reinterpret_cast<unsigned long long *>(sm);
    float *xt = reinterpret_cast<float *>(sm + 2 * a.sign_words);
    uint32_t *wb0 = sm + 2 * a.sign_words + tpr * N + gid * 2 * group_words(a.wmax);
    uint32_t *wb1 = wb0 + group_words(a.wmax);
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

    for (int64_t row = (int64_t)blockIdx.x * W + warp; row < a.rows; row += (int64_t)gridDim.x * W) {
        float acc = 0.0f;
        // the row's tiles j = group, group + TPW, ...: the next one's words
        // arrive (cp.async) while this one is parsed
        int64_t j = lane / LPT;
        TileHdr h{};
        if (j < tpr) {
            h = tile_header<N, D, FIXED>(a, row * tpr + j);
            stage_async<LPT>(a, h, wb0, l);
        }
        async_commit();
        for (; j < tpr; j += TPW) {
            const int64_t t = row * tpr + j;
            TileHdr hn{};
            if (j + TPW < tpr) {
                hn = tile_header<N, D, FIXED>(a, t + TPW);
                stage_async<LPT>(a, hn, wb1, l);
            }
            async_commit();
            async_wait<1>();
            __syncwarp(mask);
            uint32_t u[EPL], cb, sb;
            bool small;
            const bool bad = parse_staged<N, D, EPL, FIXED>(a, h, wb0, mask, l, u, cb, sb, small);
            h = hn;
            uint32_t *tmp = wb0;
            wb0 = wb1;
            wb1 = tmp;
            __syncwarp(mask);
            const float4 *src = reinterpret_cast<const float4 *>(xt + j * N + l * EPL);
            float2 d2 = make_float2(0.0f, 0.0f);
            float step;  // the tile's weight on the dot: Delta / n for points, Delta / 2n for doubled points
            if constexpr (D != 2) {
                // t = 2y: t + 1.5 2^23 read as a float minus 1.5 2^23 is exact while
                // |t| < 2^22 (every unary part under 32 bits); otherwise convert
                int32_t tt[EPL];  // t + 1.5 2^23 (bit patterns) where small, else t
                doubled_from_symbols<D, EPL>(u, cb, tt, small ? kMagicBias : 0);
                const float2 moff = splat2(-12582912.0f);
#pragma unroll
                for (int c = 0; c < EPL / 4; c++) {
                    const float4 xv = src[c ^ (l & SW)];
                    float2 p0, p1;
                    if (small) {
                        p0 = add2(make_float2(__int_as_float(tt[4 * c]), __int_as_float(tt[4 * c + 1])), moff);
                        p1 = add2(make_float2(__int_as_float(tt[4 * c + 2]), __int_as_float(tt[4 * c + 3])), moff);
                    } else {
                        p0 = make_float2((float)tt[4 * c], (float)tt[4 * c + 1]);
                        p1 = make_float2((float)tt[4 * c + 2], (float)tt[4 * c + 3]);
                    }
                    d2 = fma2(p0, make_float2(xv.x, xv.y), d2);
                    d2 = fma2(p1, make_float2(xv.z, xv.w), d2);
                }
                step = bf16_bits_to_float(sb) * (0.5f / N);
            } else {
                float pt[EPL];
                points_from_symbols<D, EPL>(u, cb, a.a2, pt);
#pragma unroll
                for (int c = 0; c < EPL / 4; c++) {
                    const float4 xv = src[c ^ (l & SW)];
                    d2 = fma2(make_float2(pt[4 * c], pt[4 * c + 1]), make_float2(xv.x, xv.y), d2);
                    d2 = fma2(make_float2(pt[4 * c + 2], pt[4 * c + 3]), make_float2(xv.z, xv.w), d2);
                }
                step = bf16_bits_to_float(sb) * (1.0f / N);
            }
            acc = fmaf(step, __fadd_rn(d2.x, d2.y), acc);
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
// the decoder: at least 16 per lane (the half-exchange transform's two runs
// then hold whole vectors and 16-byte stores)
template <int N>
constexpr int epl_dec() { return N <= 256 ? 16 : 32; }

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
    constexpr int EPL = epl_dec<N>(), GPB = kDecodeWarps * (32 / (N / EPL));
    const size_t ywords = a.sign_words ? (size_t)a.tiles_per_row * (N / EPL) : 0;
    const size_t smem = ((ywords + 3) & ~(size_t)3) * 4 + (size_t)GPB * 2 * group_words(a.wmax) * 4;
    auto kern = a.slot ? decode_kernel<N, D, EPL, DITHER, F32OUT, true> : decode_kernel<N, D, EPL, DITHER, F32OUT, false>;
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

// Blocks of W warps each hold the rotated x (cols floats) in shared memory;
// when that copy is large, 16-warp blocks keep as many warps resident as
// 8-warp blocks do with a small one.  Resident blocks per SM come from the
// kernel's registers and shared memory and the device limits.
template <int N, int D, int W>
cudaError_t launch_gemv_w(const DecodeArgs &a, int64_t cols, cudaStream_t s)
{
    constexpr int EPL = epl_for<N>(), GPB = W * (32 / (N / EPL));
    const size_t smem = (size_t)a.sign_words * 8 + (size_t)cols * 4 + (size_t)GPB * 2 * group_words(a.wmax) * 4;
    auto kern = a.slot ? gemv_kernel<N, D, EPL, W, true> : gemv_kernel<N, D, EPL, W, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa{};
    int dev = 0, smem_sm = 0, reserved = 0, regs_sm = 0, thr_sm = 0;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev)) != cudaSuccess) return e;
    const int threads = W * 32;
    int per_sm = thr_sm / threads;
    const int by_regs = regs_sm / (threads * (fa.numRegs > 0 ? fa.numRegs : 64));
    const int by_smem = (int)((size_t)smem_sm / (smem + fa.sharedSizeBytes + (size_t)reserved));
    if (by_regs < per_sm) per_sm = by_regs;
    if (by_smem < per_sm) per_sm = by_smem;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t blocks = (int64_t)sm_count() * per_sm, work = (a.rows + W - 1) / W;
    if (blocks > work) blocks = work;
    if (blocks < 1) blocks = 1;
    kern<<<(unsigned)blocks, threads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int N, int D>
cudaError_t launch_gemv_t(const DecodeArgs &a, int64_t cols, cudaStream_t s)
{
    // 32 coordinates per lane (tiles of 512, 1024) need more than 64
    // registers, so those keep 8-warp blocks
    if constexpr (N <= 256) {
        if (cols * 4 > 32 * 1024) return launch_gemv_w<N, D, 16>(a, cols, s);
    }
    return launch_gemv_w<N, D, 8>(a, cols, s);
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
