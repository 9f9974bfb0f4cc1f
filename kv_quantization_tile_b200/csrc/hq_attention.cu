// hq_attention.cu -- batch-1 attention over a dithered compressed KV cache
// (sm_100a).
//
// K and V are KV-codec streams laid out as (heads * tokens) rows of one tile
// (head_dim = n coordinates) each: tile t = h * tokens + token.  Decoding a
// tile gives  v_hat = s . H (z) / n  with z = Delta (y - delta) the
// dequantised rotated vector, so, H being symmetric,
//   <q, k_hat_t>      = <H (s_K . q), z_t> / n
//   sum_t p_t v_hat_t = s_V . H (sum_t p_t z_t) / n.
// A block therefore rotates its queries once, scores every token straight
// from the K stream, and accumulates p_t z_t over the V stream in the rotated
// domain; one inverse transform per query at the very end.  Grouped-query
// attention: a block serves up to GB query heads that share one KV head, so
// each K and V tile is parsed once for all of them.
//
// Tokens are split across blocks (flash-decoding): a block writes, per query,
// its maximum score m, its sum of exp(s - m) and its unnormalised rotated
// output to the workspace; the last block of a (KV head, query chunk) to
// finish -- found with a counter, no waiting -- merges the splits.
//
// Method: [V2] "HyperQuant: A Near-Entropy-Optimal Lattice Quantization
// Pipeline for Large Language and Diffusion Models", abstract (subtractive
// dither keeps each cached vector's inner products unbiased);
// [V1] "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline for
// Large Language and Diffusion Models", abstract (iv) (inner products kept
// for attention).
#include <cuda_bf16.h>

#include "hq_parse.cuh"

namespace hq {

namespace {

constexpr int kAttnWarps = 8, kAttnThreads = kAttnWarps * 32;
constexpr int kFactorChunk = 256;  // splits merged per pass of the combine
constexpr int kAttnWaves = 1;      // waves of resident blocks the token splits aim to fill

// Block-wide max or sum of GB values per thread (one per query); every
// thread gets the results.  `red` holds kAttnWarps * GB floats.
template <int GB, bool MAX>
__device__ __forceinline__ void block_reduce(float (&v)[GB], float *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int g = 0; g < GB; g++)
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            const float o = __shfl_xor_sync(FULL, v[g], m);
            v[g] = MAX ? fmaxf(v[g], o) : v[g] + o;
        }
    __syncthreads();
    if (lane == 0)
#pragma unroll
        for (int g = 0; g < GB; g++) red[warp * GB + g] = v[g];
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GB; g++) {
        float r = red[g];
        for (int w = 1; w < kAttnWarps; w++) r = MAX ? fmaxf(r, red[w * GB + g]) : r + red[w * GB + g];
        v[g] = r;
    }
}

}  // namespace

// Shared memory: K and V sign words | rotated queries (GB x n, float4 chunk c
// of lane l at (g * EPL/4 + c) * LPT + l) | region U, first the per-group
// staged tiles, the scores (GB x tokens_per_split) and each warp's value
// staging rows (TPW x n) and weights (TPW x GB), later reused for the
// cross-warp partial outputs and the combine.
// Resident blocks per SM the register allocation targets: four, fewer where
// the GB x n/32 column accumulators of head_dim 256 would spill.
constexpr int attn_min_blocks(int n, int gb) { return n * gb >= 2048 ? 2 : (n == 256 && n * gb >= 1024 ? 3 : 4); }

template <int N, int D, int EPL, int GB, bool FIXED>
__global__ void __launch_bounds__(kAttnThreads, attn_min_blocks(N, GB)) kv_attention_kernel(const AttnArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = kAttnWarps * TPW, C4 = EPL / 4;
    constexpr int WPT = N / 64;
    constexpr float inv_n = 1.0f / N;
    const int sp = blockIdx.x, h = blockIdx.y, z = blockIdx.z;
    const int g0 = z * GB;
    const int G = a.group - g0 < GB ? a.group - g0 : GB;  // queries of this block
    const int tps = a.tokens_per_split;
    const int64_t t0 = (int64_t)sp * tps;
    const int nt = (int)(a.tokens - t0 < tps ? a.tokens - t0 : tps);  // >= 1
    const int64_t qh0 = (int64_t)h * a.group + g0;                    // first query head

    extern __shared__ __align__(16) uint32_t sm[];
    unsigned long long *sk = reinterpret_cast<unsigned long long *>(sm);
    unsigned long long *sv = sk + WPT;
    float4 *qt4 = reinterpret_cast<float4 *>(sv + WPT);
    float *U = reinterpret_cast<float *>(qt4 + GB * N / 4);
    const uint32_t wmax = a.k.wmax > a.v.wmax ? a.k.wmax : a.v.wmax;
    __shared__ float s_red[kAttnWarps * GB];
    __shared__ float s_stat[2 * GB];  // this split's m_g and l_g
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    uint32_t *wbuf = reinterpret_cast<uint32_t *>(U) + gid * group_words(wmax);
    float *scores = U + GPB * group_words(wmax);  // [GB][tps]

    if (tid < WPT) {
        sk[tid] = mix64(mix64(a.k.sign_key) ^ (uint64_t)tid);  // column tile 0
        sv[tid] = mix64(mix64(a.v.sign_key) ^ (uint64_t)tid);
    }
    __syncthreads();

    // ---- rotated queries q~_g = H (s_K . q_g); zero for g >= G
    for (int g = gid; g < GB; g += GPB) {
        float v[EPL];
        if (g < G) {
            const uint4 *p = reinterpret_cast<const uint4 *>(a.q + (qh0 + g) * N + l * EPL);
#pragma unroll
            for (int i = 0; i < EPL / 8; i++) {
                const uint4 w = __ldg(p + i);
                const uint32_t ww[4] = { w.x, w.y, w.z, w.w };
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    v[8 * i + 2 * k] = __uint_as_float(ww[k] << 16);
                    v[8 * i + 2 * k + 1] = __uint_as_float(ww[k] & 0xffff0000u);
                }
            }
            const uint32_t sb = sign_bits<N, EPL>(sk, WPT, 0, 0, l);
#pragma unroll
            for (int r = 0; r < EPL; r++)
                v[r] = __uint_as_float(__float_as_uint(v[r]) ^ ((sb << (31 - r)) & 0x80000000u));
            fwht<EPL, LPT>(v, mask, l);
        } else {
#pragma unroll
            for (int r = 0; r < EPL; r++) v[r] = 0.0f;
        }
#pragma unroll
        for (int c = 0; c < C4; c++)
            qt4[(g * C4 + c) * LPT + l] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
    __syncthreads();

    // ---- scores s_gt = scale (Delta_t / n) <y_t - delta_t, q~_g>
    for (int i = gid; i < nt; i += GPB) {
        const int64_t tg = (int64_t)h * a.tokens + t0 + i;
        float pt[EPL];
        uint32_t sbits;
        const bool bad = parse_tile<N, D, EPL, FIXED>(a.k, tg, wbuf, mask, l, pt, sbits);
        if (!bad && sbits) sub_dither<D, EPL>(mix64(a.k.dither_key ^ (uint64_t)tg), l, pt, a.k.a2);
        float dot[GB];
#pragma unroll
        for (int g = 0; g < GB; g++) {
            dot[g] = 0.0f;
#pragma unroll
            for (int c = 0; c < C4; c++) {
                const float4 qv = qt4[(g * C4 + c) * LPT + l];
                dot[g] = fmaf(pt[4 * c], qv.x, dot[g]);
                dot[g] = fmaf(pt[4 * c + 1], qv.y, dot[g]);
                dot[g] = fmaf(pt[4 * c + 2], qv.z, dot[g]);
                dot[g] = fmaf(pt[4 * c + 3], qv.w, dot[g]);
            }
#pragma unroll
            for (int m = 1; m < LPT; m <<= 1) dot[g] += __shfl_xor_sync(mask, dot[g], m);
        }
        if (l == 0) {
            const float f = a.scale * (bf16_bits_to_float(sbits) * inv_n);
#pragma unroll
            for (int g = 0; g < GB; g++) scores[g * tps + i] = f * dot[g];
            if (bad && a.status) atomicOr(a.status, kStatusCorrupt);
        }
    }
    __syncthreads();

    // ---- softmax statistics of this split: m_g, then p = exp(s - m_g), l_g
    float mx[GB], ls[GB];
#pragma unroll
    for (int g = 0; g < GB; g++) mx[g] = -INFINITY;
    for (int i = tid; i < nt; i += kAttnThreads)
#pragma unroll
        for (int g = 0; g < GB; g++) mx[g] = fmaxf(mx[g], scores[g * tps + i]);
    block_reduce<GB, true>(mx, s_red);
#pragma unroll
    for (int g = 0; g < GB; g++) ls[g] = 0.0f;
    for (int i = tid; i < nt; i += kAttnThreads)
#pragma unroll
        for (int g = 0; g < GB; g++) {
            const float p = expf(scores[g * tps + i] - mx[g]);
            scores[g * tps + i] = p;
            ls[g] += p;
        }
    block_reduce<GB, false>(ls, s_red);  // its barriers also publish the weights
    if (tid == 0)
#pragma unroll
        for (int g = 0; g < GB; g++) {
            s_stat[g] = mx[g];
            s_stat[GB + g] = ls[g];
        }

    // ---- values: acc_g = sum_t p_gt Delta_t (y_t - delta_t), rotated domain.
    // The groups of a warp parse one token each into the warp's staging rows
    // (lane l's chunk c at slot c ^ swz(l), conflict-free 128-bit stores) with
    // the token's weights p_gt Delta_t; then every lane accumulates columns
    // lane + 32 c of all staged tokens for all GB queries.
    constexpr int CPL = N / 32;           // columns per lane
    constexpr int U4 = EPL / 4;
    float *stage = scores + ((GB * tps + 3) & ~3);
    float *zw = stage + warp * TPW * N;                            // [TPW][n]
    float *ww = stage + kAttnWarps * TPW * N + warp * TPW * GB;    // [TPW][GB]
    int pos[CPL];  // staging position of column lane + 32 c
#pragma unroll
    for (int c = 0; c < CPL; c++) {
        const int i = lane + 32 * c, li = i / EPL, cc = (i % EPL) / 4;
        pos[c] = li * EPL + 4 * (cc ^ ((li * U4 >> 3) & (U4 - 1))) + (i & 3);
    }
    float acc[GB][CPL];
#pragma unroll
    for (int g = 0; g < GB; g++)
#pragma unroll
        for (int c = 0; c < CPL; c++) acc[g][c] = 0.0f;
    const int grp = lane / LPT;
    for (int base = warp * TPW; base < nt; base += GPB) {
        const int i = base + grp;
        if (i < nt) {
            const int64_t tg = (int64_t)h * a.tokens + t0 + i;
            float pt[EPL];
            uint32_t sbits;
            const bool bad = parse_tile<N, D, EPL, FIXED>(a.v, tg, wbuf, mask, l, pt, sbits);
            if (!bad && sbits) sub_dither<D, EPL>(mix64(a.v.dither_key ^ (uint64_t)tg), l, pt, a.v.a2);
            float4 *row = reinterpret_cast<float4 *>(zw + grp * N + l * EPL);
            const int sw = (l * U4 >> 3) & (U4 - 1);
#pragma unroll
            for (int c = 0; c < U4; c++) row[c ^ sw] = make_float4(pt[4 * c], pt[4 * c + 1], pt[4 * c + 2], pt[4 * c + 3]);
            if (l < GB) ww[grp * GB + l] = scores[l * tps + i] * bf16_bits_to_float(sbits);
            if (bad && l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
        } else {  // past the split's end: weight 0 on a zero row
            float4 *row = reinterpret_cast<float4 *>(zw + grp * N + l * EPL);
#pragma unroll
            for (int c = 0; c < U4; c++) row[c] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (l < GB) ww[grp * GB + l] = 0.0f;
        }
        __syncwarp();
#pragma unroll
        for (int s = 0; s < TPW; s++) {
            float w[GB];
#pragma unroll
            for (int g = 0; g < GB; g++) w[g] = ww[s * GB + g];
#pragma unroll
            for (int c = 0; c < CPL; c++) {
                const float z = zw[s * N + pos[c]];
#pragma unroll
                for (int g = 0; g < GB; g++) acc[g][c] = fmaf(w[g], z, acc[g][c]);
            }
        }
        __syncwarp();
    }
    __syncthreads();  // U (staged tiles, weights) is free from here on
    float *red = U;   // [warps][GB][n]
#pragma unroll
    for (int g = 0; g < GB; g++)
#pragma unroll
        for (int c = 0; c < CPL; c++) red[(warp * GB + g) * N + lane + 32 * c] = acc[g][c];
    __syncthreads();
    for (int e = tid; e < G * N; e += kAttnThreads) {
        const int g = e / N, i = e % N;
        float o = red[g * N + i];
        for (int w = 1; w < kAttnWarps; w++) o += red[(w * GB + g) * N + i];
        float *part = a.part + ((qh0 + g) * a.splits + sp) * (N + 2);
        part[2 + i] = o;
        if (i == 0) {
            part[0] = s_stat[g];
            part[1] = s_stat[GB + g];
        }
    }

    // ---- the last block of this (KV head, query chunk) merges the splits
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(a.counter + (int64_t)h * gridDim.z + z, 1u) == (unsigned)(a.splits - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int S = a.splits;
    // warp g: M_g = max_s m_gs, L_g = sum_s l_gs exp(m_gs - M_g)
    float *sM = s_red, *sL = s_red + GB;
    if (warp < G) {
        const float *ph = a.part + (qh0 + warp) * S * (int64_t)(N + 2);
        float M = -INFINITY;
        for (int s = lane; s < S; s += 32) M = fmaxf(M, __ldcg(ph + (int64_t)s * (N + 2)));
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, m));
        float L = 0.0f;
        for (int s = lane; s < S; s += 32) {
            const float *p = ph + (int64_t)s * (N + 2);
            L += __ldcg(p + 1) * expf(__ldcg(p) - M);
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) L += __shfl_xor_sync(FULL, L, m);
        if (lane == 0) {
            sM[warp] = M;
            sL[warp] = L;
        }
    }
    __syncthreads();
    // O_g = sum_s exp(m_gs - M_g) O_gs, a chunk of split factors at a time
    constexpr int PPT = (GB * N + kAttnThreads - 1) / kAttnThreads;
    float *fac = U;                     // [GB][kFactorChunk]
    float *ob = U + GB * kFactorChunk;  // [GB][n]
    float o[PPT];
#pragma unroll
    for (int k = 0; k < PPT; k++) o[k] = 0.0f;
    for (int s0 = 0; s0 < S; s0 += kFactorChunk) {
        const int sc = S - s0 < kFactorChunk ? S - s0 : kFactorChunk;
        for (int e = tid; e < G * sc; e += kAttnThreads) {
            const int g = e / sc, s = e % sc;
            fac[g * kFactorChunk + s] =
                expf(__ldcg(a.part + ((qh0 + g) * S + s0 + s) * (int64_t)(N + 2)) - sM[g]);
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < PPT; k++) {
            const int e = tid + k * kAttnThreads;
            if (e < G * N) {
                const int g = e / N, i = e % N;
                const float *p = a.part + ((qh0 + g) * S + s0) * (int64_t)(N + 2) + 2 + i;
                float acc1 = o[k];
                for (int s = 0; s < sc; s++)
                    acc1 = fmaf(fac[g * kFactorChunk + s], __ldcg(p + (int64_t)s * (N + 2)), acc1);
                o[k] = acc1;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < PPT; k++) {
        const int e = tid + k * kAttnThreads;
        if (e < G * N) ob[e] = o[k] / sL[e / N];
    }
    __syncthreads();
    // out_g = s_V . H (O_g / L_g) / n
    for (int g = gid; g < G; g += GPB) {
        float v[EPL];
#pragma unroll
        for (int r = 0; r < EPL; r++) v[r] = ob[g * N + l * EPL + r];
        fwht<EPL, LPT>(v, mask, l);
        const uint32_t sb = sign_bits<N, EPL>(sv, WPT, 0, 0, l);
        float4 *dst = reinterpret_cast<float4 *>(a.out + (qh0 + g) * N + l * EPL);
#pragma unroll
        for (int c = 0; c < C4; c++) {
            float w[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const int r = 4 * c + k;
                w[k] = __uint_as_float(__float_as_uint(v[r] * inv_n) ^ ((sb << (31 - r)) & 0x80000000u));
            }
            dst[c] = make_float4(w[0], w[1], w[2], w[3]);
        }
    }
}

// ------------------------------------------------------------------ launch
namespace {

// Coordinates per lane of a parsed tile.
template <int N, int GB>
constexpr int attn_epl() { return N == 64 ? 8 : 16; }

template <int N, int GB>
size_t attn_smem(uint32_t wmax, int tps)
{
    constexpr int EPL = attn_epl<N, GB>(), GPB = kAttnWarps * (32 / (N / EPL));
    const size_t staged = (size_t)GPB * group_words(wmax) * 4 + (size_t)((GB * tps + 3) & ~3) * 4 +
                          (size_t)kAttnWarps * (32 / (N / EPL)) * (N + GB) * 4;
    const size_t red = (size_t)kAttnWarps * GB * N * 4;
    const size_t merge = (size_t)GB * (kFactorChunk + N) * 4;
    size_t u = staged > red ? staged : red;
    if (merge > u) u = merge;
    return 2 * (N / 64) * 8 + (size_t)GB * N * 4 + u;
}

// Splits from the kernel's occupancy at the largest split, then the launch.
template <int N, int D, int GB>
cudaError_t launch_attention_t(AttnArgs a, int zchunks, cudaStream_t s)
{
    constexpr int EPL = attn_epl<N, GB>();
    const uint32_t wmax = a.k.wmax > a.v.wmax ? a.k.wmax : a.v.wmax;
    auto kern = a.k.slot ? kv_attention_kernel<N, D, EPL, GB, true> : kv_attention_kernel<N, D, EPL, GB, false>;
    const size_t smem_max = attn_smem<N, GB>(wmax, 4096 / GB);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kAttnThreads, smem_max);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    attention_splits(a.heads, a.tokens, a.group, per_sm, &a.splits, &a.tokens_per_split);
    const size_t smem = attn_smem<N, GB>(wmax, a.tokens_per_split);
    kern<<<dim3((unsigned)a.splits, (unsigned)a.heads, (unsigned)zchunks), kAttnThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int N, int D>
cudaError_t launch_attention_nd(int gb, const AttnArgs &a, int zchunks, cudaStream_t s)
{
    switch (gb) {
    case 1: return launch_attention_t<N, D, 1>(a, zchunks, s);
    case 2: return launch_attention_t<N, D, 2>(a, zchunks, s);
    case 4: return launch_attention_t<N, D, 4>(a, zchunks, s);
    default: return launch_attention_t<N, D, 8>(a, zchunks, s);
    }
}

template <int N>
cudaError_t launch_attention_n(int lattice, int gb, const AttnArgs &a, int zchunks, cudaStream_t s)
{
    switch (lattice) {
    case 1: return launch_attention_nd<N, 1>(gb, a, zchunks, s);
    case 2: return launch_attention_nd<N, 2>(gb, a, zchunks, s);
    case 4: return launch_attention_nd<N, 4>(gb, a, zchunks, s);
    default: return launch_attention_nd<N, 8>(gb, a, zchunks, s);
    }
}

}  // namespace

int attention_queries_per_block(int group) { return group <= 1 ? 1 : group <= 2 ? 2 : group <= 4 ? 4 : 8; }

// Token splits: enough to fill kAttnWaves waves of resident blocks
// (blocks_per_sm per SM) over the heads x query-chunk blocks, but no fewer
// than 128 tokens per split where the sequence allows and no more than
// 4096 / GB tokens per split (the GB rows of scores stay within 16 KB of
// shared memory).  Every split is non-empty.  The count never grows when
// blocks_per_sm shrinks, so blocks_per_sm = 8 (the most 256-thread blocks an
// SM holds) bounds the workspace of any launch.
void attention_splits(int64_t heads, int64_t tokens, int group, int blocks_per_sm, int *splits,
                      int *tokens_per_split)
{
    const int gb = attention_queries_per_block(group);
    const int64_t zc = (group + gb - 1) / gb;
    const int64_t tmax = 4096 / gb;
    const int64_t smin = (tokens + tmax - 1) / tmax;
    const int64_t blocks = heads * zc > 0 ? heads * zc : 1;
    int64_t s = (int64_t)kAttnWaves * sm_count() * (blocks_per_sm > 0 ? blocks_per_sm : 1) / blocks;
    const int64_t s128 = (tokens + 127) / 128;
    if (s > s128) s = s128;
    if (s < smin) s = smin;
    if (s < 1) s = 1;
    const int64_t tps = tokens > 0 ? (tokens + s - 1) / s : 1;
    s = tokens > 0 ? (tokens + tps - 1) / tps : 1;
    *splits = (int)s;
    *tokens_per_split = (int)tps;
}

cudaError_t launch_attention(int head_dim, int lattice, AttnArgs a, cudaStream_t s)
{
    const int gb = attention_queries_per_block(a.group);
    const int zchunks = (a.group + gb - 1) / gb;
    switch (head_dim) {
    case 64: return launch_attention_n<64>(lattice, gb, a, zchunks, s);
    case 128: return launch_attention_n<128>(lattice, gb, a, zchunks, s);
    default: return launch_attention_n<256>(lattice, gb, a, zchunks, s);
    }
}

}  // namespace hq
