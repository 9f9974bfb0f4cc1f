// hq_stats.cu -- rate accounting of a stream: its bits by kind and a
// histogram of its symbols.
//
// Method: [V2] "HyperQuant: A Near-Entropy-Optimal Lattice Quantization
// Pipeline for Large Language and Diffusion Models", abstract (itemized rate
// accounting; the Rice code's distance from the lattice's rate-distortion
// ideal).  Per canonical tile, with k its Rice parameter, C its coset bits
// (n / 8 for E8, n / 2 for A2, 0 otherwise) and u its n symbols:
//   low-part bits = n k, unary bits = sum(u >> k) + n, padding = 32 W - C -
//   n k - unary (W the tile's words), headers = offset (32, none in a
//   fixed-rate stream) + scale (16) + Rice parameter (8, or 4 packed).
// The histogram keeps the symbols of the stripped last coordinate of D4 / E8
// vectors apart (row 1) from all others (row 0): the two follow different
// laws, so their empirical entropies are taken separately.
#include <cuda_bf16.h>

#include "../../include/hq.h"
#include "hq_parse.cuh"

namespace hq {

namespace {

constexpr int kStatsWarps = 8;

template <int N, int D, int EPL, bool FIXED>
__global__ void __launch_bounds__(kStatsWarps * 32) stats_kernel(const DecodeArgs a, unsigned long long *counts,
                                                                  unsigned long long *hist, int bins)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = kStatsWarps * TPW;
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;
    extern __shared__ __align__(16) uint32_t sm[];
    uint32_t *h = sm;                                   // [2][bins] symbol counts
    unsigned long long *c = reinterpret_cast<unsigned long long *>(sm + ((2 * bins + 1) & ~1));  // [8]
    uint32_t *wbase = reinterpret_cast<uint32_t *>(c + 8);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    uint32_t *wbuf = wbase + gid * group_words(a.wmax);
    for (int i = tid; i < 2 * bins; i += blockDim.x) h[i] = 0;
    if (tid < 8) c[tid] = 0;
    __syncthreads();

    unsigned long long tiles = 0, low = 0, unary = 0, pad = 0;
    for (int64_t t = (int64_t)blockIdx.x * GPB + gid; t < a.ntiles; t += (int64_t)gridDim.x * GPB) {
        uint32_t u[EPL], cb, sb;
        bool small;
        const TileHdr hd = tile_header<N, D, FIXED>(a, t);
        __syncwarp(mask);  // the group is done with the previous tile's words
        for (uint32_t i = l; i < hd.W; i += LPT) wbuf[i] = __ldg(a.payload + hd.o0 + i);
        if (l < 4) wbuf[hd.W + l] = 0u;
        __syncwarp(mask);
        const bool bad = parse_staged<N, D, EPL, FIXED>(a, hd, wbuf, mask, l, u, cb, sb, small);
        if (bad) {
            if (l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
            continue;  // group-uniform
        }
        uint32_t q = 0;
#pragma unroll
        for (int r = 0; r < EPL; r++) {
            q += u[r] >> hd.k;
            const int row = ((D == 8 || D == 4) && (r % D) == D - 1) ? 1 : 0;
            atomicAdd(&h[row * bins + (u[r] < (uint32_t)bins - 1 ? u[r] : (uint32_t)bins - 1)], 1u);
        }
        const uint32_t un = group_sum<LPT>(mask, q) + (uint32_t)N;
        if (l == 0) {
            tiles += 1;
            low += (unsigned long long)N * (unsigned long long)hd.k;
            unary += un;
            pad += 32ull * hd.W - (unsigned long long)C - (unsigned long long)N * hd.k - un;
        }
    }
    if (l == 0) {
        atomicAdd(&c[0], tiles);
        atomicAdd(&c[2], low);
        atomicAdd(&c[3], unary);
        atomicAdd(&c[4], pad);
    }
    __syncthreads();
    for (int i = tid; i < 2 * bins; i += blockDim.x)
        if (h[i]) atomicAdd(&hist[i], (unsigned long long)h[i]);
    if (tid == 0) {
        const unsigned long long nt = c[0];
        atomicAdd(&counts[0], nt);
        atomicAdd(&counts[1], nt * (unsigned long long)C);
        atomicAdd(&counts[2], c[2]);
        atomicAdd(&counts[3], c[3]);
        atomicAdd(&counts[4], c[4]);
        atomicAdd(&counts[5], FIXED ? 0ull : 32ull * nt);
        atomicAdd(&counts[6], 16ull * nt);
        atomicAdd(&counts[7], (FIXED ? 4ull : 8ull) * nt);
    }
}

template <int N>
constexpr int epl_stats() { return N <= 256 ? 16 : 32; }

template <int N, int D>
cudaError_t launch_stats_nd(const DecodeArgs &a, unsigned long long *counts, unsigned long long *hist, int bins,
                            cudaStream_t s)
{
    constexpr int EPL = epl_stats<N>(), GPB = kStatsWarps * (32 / (N / EPL));
    const size_t smem = (size_t)((2 * bins + 1) & ~1) * 4 + 8 * 8 + (size_t)GPB * group_words(a.wmax) * 4;
    auto kern = a.slot ? stats_kernel<N, D, EPL, true> : stats_kernel<N, D, EPL, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kStatsWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t blocks = (int64_t)sm_count() * per_sm, work = (a.ntiles + GPB - 1) / GPB;
    if (blocks > work) blocks = work;
    if (blocks < 1) blocks = 1;
    kern<<<(unsigned)blocks, kStatsWarps * 32, smem, s>>>(a, counts, hist, bins);
    return cudaGetLastError();
}

template <int N>
cudaError_t launch_stats_n(int lattice, const DecodeArgs &a, unsigned long long *counts, unsigned long long *hist,
                           int bins, cudaStream_t s)
{
    switch (lattice) {
    case 1: return launch_stats_nd<N, 1>(a, counts, hist, bins, s);
    case 2: return launch_stats_nd<N, 2>(a, counts, hist, bins, s);
    case 4: return launch_stats_nd<N, 4>(a, counts, hist, bins, s);
    default: return launch_stats_nd<N, 8>(a, counts, hist, bins, s);
    }
}

}  // namespace

cudaError_t launch_stats(int tile, int lattice, const DecodeArgs &a, uint64_t *counts, uint64_t *hist, int bins,
                         cudaStream_t s)
{
    auto *c = reinterpret_cast<unsigned long long *>(counts);
    auto *h = reinterpret_cast<unsigned long long *>(hist);
    switch (tile) {
    case 64: return launch_stats_n<64>(lattice, a, c, h, bins, s);
    case 128: return launch_stats_n<128>(lattice, a, c, h, bins, s);
    case 256: return launch_stats_n<256>(lattice, a, c, h, bins, s);
    case 512: return launch_stats_n<512>(lattice, a, c, h, bins, s);
    default: return launch_stats_n<1024>(lattice, a, c, h, bins, s);
    }
}

}  // namespace hq
