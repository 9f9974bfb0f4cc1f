// hq_encode.cu -- single-pass tile encoder for sm_100a.
//
// One thread block encodes one chunk of T consecutive tiles (a contiguous
// span of the row-major input), one tile per group of LPT lanes:
//   load (128-bit) -> random signs -> pairwise sum of squares -> register +
//   shuffle Walsh-Hadamard transform -> Delta -> v / Delta [+ dither] ->
//   nearest lattice point -> strip + zigzag -> per-tile Rice k (convex
//   descent on the exact code length) -> per-lane code lengths.
// The chunk's word count is then published for a decoupled look-back prefix
// scan over chunks (chunk ids come from an atomic ticket, so every chunk a
// block waits on belongs to a block that is already running); the tiles'
// bits are OR-ed into a shared-memory image of the chunk and written out
// with coalesced stores.  Every wait is bounded: a block that gives up
// raises HQ_ST_TIMEOUT, publishes its own prefix and writes nothing.
//
// Method: [V1] "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline
// for Large Language and Diffusion Models", abstract (i)-(iv); [V2]
// "HyperQuant: A Near-Entropy-Optimal Lattice Quantization Pipeline for
// Large Language and Diffusion Models", abstract (strip, Rice code,
// subtractive dither).
#include <cuda_bf16.h>

#include "hq_internal.h"

namespace hq {

namespace {

__device__ __forceinline__ void st_release(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Decoupled look-back (thread 0 of a block): publish this chunk's aggregate,
// sum predecessors' aggregates until an inclusive prefix is found, publish
// the inclusive prefix.  Returns the exclusive prefix; `timed_out` is set if
// a predecessor published nothing within the poll limit.
__device__ uint64_t chunk_lookback(unsigned long long *lb, uint32_t chunk, uint64_t agg,
                                   bool &timed_out)
{
    timed_out = false;
    if (chunk == 0) {
        st_release(&lb[0], kFlagInclusive | agg);
        return 0;
    }
    st_release(&lb[chunk], kFlagAggregate | agg);
    uint64_t excl = 0;
    int64_t p = (int64_t)chunk - 1;
    uint32_t polls = 0;
    while (p >= 0) {
        unsigned long long s = ld_acquire(&lb[p]);
        const uint64_t flag = s & ~kValueMask;
        if (flag == 0) {
            if (++polls > kSpinLimit) {
                timed_out = true;
                break;
            }
            __nanosleep(64);
            continue;
        }
        excl += s & kValueMask;
        if (flag == kFlagInclusive) break;
        --p;
    }
    st_release(&lb[chunk], kFlagInclusive | ((excl + agg) & kValueMask));
    return excl;
}

template <int EPL, bool F32IN>
__device__ __forceinline__ void load_tile_part(const void *x, int64_t e0, float (&w)[EPL])
{
    if constexpr (F32IN) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) + e0);
#pragma unroll
        for (int i = 0; i < EPL / 4; i++) {
            float4 f = __ldg(p + i);
            w[4 * i] = f.x; w[4 * i + 1] = f.y; w[4 * i + 2] = f.z; w[4 * i + 3] = f.w;
        }
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + e0);
#pragma unroll
        for (int i = 0; i < EPL / 8; i++) {
            uint4 q = __ldg(p + i);
            const uint32_t qq[4] = { q.x, q.y, q.z, q.w };
#pragma unroll
            for (int h = 0; h < 4; h++) {
                w[8 * i + 2 * h] = __uint_as_float(qq[h] << 16);
                w[8 * i + 2 * h + 1] = __uint_as_float(qq[h] & 0xffff0000u);
            }
        }
    }
}

}  // namespace

template <int N, int D, int EPL, bool DITHER, bool F32IN, int NWARPS>
__global__ void __launch_bounds__(NWARPS * 32) encode_kernel(const EncodeArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, T = NWARPS * TPW;
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;  // coset bits per tile
    constexpr int VPL = EPL / D;                          // vectors per lane
    static_assert(EPL % D == 0 && LPT <= 32 && (32 % LPT) == 0, "layout");

    extern __shared__ uint32_t chunk_buf[];  // T * wmax words
    __shared__ uint32_t s_tile_words[T];
    __shared__ uint32_t s_tile_off[T];
    __shared__ uint32_t s_chunk, s_total;
    __shared__ unsigned long long s_base;
    __shared__ int s_timeout;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT;
    const int tl = warp * TPW + lane / LPT;  // tile within the chunk
    const unsigned mask = group_mask<LPT>(lane);

    if (tid == 0) s_chunk = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t chunk = s_chunk;
    const int64_t t = (int64_t)chunk * T + tl;
    const bool active = t < a.ntiles;

    // ---- load + signs
    float w[EPL];
    if (active) {
        load_tile_part<EPL, F32IN>(a.x, t * N + (int64_t)l * EPL, w);
    } else {
#pragma unroll
        for (int r = 0; r < EPL; r++) w[r] = 0.0f;
    }
    const uint64_t j = active ? (uint64_t)(t % a.tiles_per_row) : 0;
    const uint32_t i0 = (uint32_t)l * EPL;
    const uint32_t sbits = (uint32_t)(mix64(mix64(a.sign_key ^ j) ^ (uint64_t)(i0 >> 6)) >> (i0 & 63));
    float v[EPL];
#pragma unroll
    for (int r = 0; r < EPL; r++) v[r] = __uint_as_float(__float_as_uint(w[r]) ^ (((sbits >> r) & 1u) << 31));

    // ---- scale + rotation
    const float S = sumsq<EPL, LPT>(w, mask);
    fwht<EPL, LPT>(v, mask, l);
    bool nonfinite;
    const uint32_t sb = tile_scale_bits(S, a.c, nonfinite);
    if (active && nonfinite && l == 0 && a.status) atomicOr(a.status, kStatusNonfinite);

    // ---- nearest point, strip, zigzag
    uint32_t u[EPL];
    uint32_t cbits = 0;
#pragma unroll
    for (int r = 0; r < EPL; r++) u[r] = 0;
    if (sb != 0) {
        const float inv = __frcp_rn(bf16_bits_to_float(sb));
        const uint64_t tkey = DITHER ? mix64(a.dither_key ^ (uint64_t)t) : 0ull;
#pragma unroll
        for (int q = 0; q < VPL; q++) {
            float x[D], p[D];
            int z[D], c;
#pragma unroll
            for (int m = 0; m < D; m++) x[m] = __fmul_rn(v[q * D + m], inv);
            if constexpr (DITHER) {
                float dl[D];
                dither<D>(tkey, (uint32_t)(l * VPL + q), dl, a.a2);
#pragma unroll
                for (int m = 0; m < D; m++) x[m] = __fadd_rn(x[m], dl[m]);
            }
            nearest<D>(x, c, z, p, a.a2);
            cbits |= (uint32_t)c << q;
#pragma unroll
            for (int m = 0; m < D; m++) {
                int s = z[m];
                if constexpr (D == 8 || D == 4) {
                    if (m == D - 1) s >>= 1;  // floor(z / 2): parity is implied by the even sum
                }
                u[q * D + m] = zigzag(s);
            }
        }
    }

    // ---- per-tile Rice parameter: smallest k in [0, 15] with
    //      sum_i ceil(floor(u_i / 2^k) / 2) <= N (the code length is convex in k
    //      and this is where its forward difference turns non-negative).
    uint32_t lsum = 0;
#pragma unroll
    for (int r = 0; r < EPL; r++) lsum += u[r];
    const uint32_t tot = group_sum<LPT>(mask, lsum);
    const uint32_t mean = tot / N;
    int k = mean ? 31 - __clz(mean) : 0;
    k = k > 15 ? 15 : k;
    auto halfsum = [&](int kk) {
        uint32_t s = 0;
#pragma unroll
        for (int r = 0; r < EPL; r++) s += (u[r] + (1u << kk)) >> (kk + 1);
        return group_sum<LPT>(mask, s);
    };
    if (k < 15 && halfsum(k) > (uint32_t)N) {
        do {
            ++k;
        } while (k < 15 && halfsum(k) > (uint32_t)N);
    } else {
        while (k > 0 && halfsum(k - 1) <= (uint32_t)N) --k;
    }

    // ---- lengths
    uint32_t ul = 0;
#pragma unroll
    for (int r = 0; r < EPL; r++) ul += (u[r] >> k) + 1u;
    const uint32_t uoff = group_excl_scan<LPT>(mask, ul, l);
    const uint32_t utot = group_sum<LPT>(mask, ul);
    const uint32_t bits = (uint32_t)C + (uint32_t)N * (uint32_t)k + utot;
    uint32_t W = active ? (bits + 31) >> 5 : 0;
    const bool overflow = W > a.wmax;  // excluded by the bound; guards the shared image
    if (overflow) W = a.wmax;
    if (l == 0) s_tile_words[tl] = W;
    __syncthreads();

    // ---- chunk prefix (in block) and across chunks (look-back)
    if (tid == 0) {
        uint32_t acc = 0;
        for (int i = 0; i < T; i++) {
            s_tile_off[i] = acc;
            acc += s_tile_words[i];
        }
        s_total = acc;
        bool to;
        s_base = chunk_lookback(a.lb, chunk, acc, to);
        s_timeout = to;
        if (to && a.status) atomicOr(a.status, kStatusTimeout);
    }
    __syncthreads();

    // ---- pack this tile into the chunk image
    const uint32_t tb = s_tile_off[tl];
    uint32_t *tbuf = chunk_buf + tb;
    for (uint32_t i = l; i < W; i += LPT) tbuf[i] = 0u;
    __syncwarp();
    if (active && !overflow) {
        if constexpr (C > 0) or_bits(tbuf, (uint32_t)l * VPL, cbits, VPL);
        if (k) {
            const uint32_t lowmask = (1u << k) - 1u;
#pragma unroll
            for (int r0 = 0; r0 < EPL; r0 += 4) {
                uint64_t val = 0;
#pragma unroll
                for (int m = 0; m < 4; m++) val |= (uint64_t)(u[r0 + m] & lowmask) << (m * k);
                or_bits(tbuf, (uint32_t)C + ((uint32_t)l * EPL + r0) * (uint32_t)k, val, 4 * k);
            }
        }
        const uint32_t upos = (uint32_t)C + (uint32_t)N * (uint32_t)k + uoff;
        if (ul <= 64) {
            uint64_t val = 0;
            uint32_t rel = 0;
#pragma unroll
            for (int r = 0; r < EPL; r++) {
                rel += u[r] >> k;
                val |= 1ull << rel;
                ++rel;
            }
            or_bits(tbuf, upos, val, (int)ul);
        } else {
            uint32_t rel = 0;
#pragma unroll
            for (int r = 0; r < EPL; r++) {
                rel += u[r] >> k;
                const uint32_t pbit = upos + rel;
                atomicOr(&tbuf[pbit >> 5], 1u << (pbit & 31));
                ++rel;
            }
        }
    }
    if (overflow && l == 0 && a.status) atomicOr(a.status, kStatusCapacity);
    __syncthreads();

    // ---- write the chunk and the tile headers
    const uint64_t base = s_base;
    const uint32_t total = s_total;
    if (s_timeout) return;
    const bool fits = base + total <= a.cap;
    if (!fits && tid == 0 && a.status) atomicOr(a.status, kStatusCapacity);
    if (fits) {
        for (uint32_t i = tid; i < total; i += NWARPS * 32) a.payload[base + i] = chunk_buf[i];
    }
    if (active && l == 0) {
        a.off[t] = (uint32_t)(base + tb);
        a.scale[t] = (uint16_t)sb;
        a.kk[t] = (uint8_t)k;
    }
    if (tid == 0 && chunk == a.nchunks - 1) a.off[a.ntiles] = (uint32_t)(base + total);
}

// ------------------------------------------------------------------ launch
namespace {

constexpr int kEncodeWarps = 8;

template <int N>
constexpr int epl_for() { return N <= 256 ? 8 : N / 32; }

template <int N, int D, bool DITHER, bool F32IN>
cudaError_t launch_encode_t(const EncodeArgs &a, cudaStream_t s)
{
    constexpr int EPL = epl_for<N>();
    constexpr int T = kEncodeWarps * (32 / (N / EPL));
    const size_t smem = (size_t)T * a.wmax * sizeof(uint32_t);
    auto kern = encode_kernel<N, D, EPL, DITHER, F32IN, kEncodeWarps>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<a.nchunks, kEncodeWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int N, int D>
cudaError_t launch_encode_nd(bool dither, int dtype, const EncodeArgs &a, cudaStream_t s)
{
    if (dither) return dtype ? launch_encode_t<N, D, true, true>(a, s) : launch_encode_t<N, D, true, false>(a, s);
    return dtype ? launch_encode_t<N, D, false, true>(a, s) : launch_encode_t<N, D, false, false>(a, s);
}

template <int N>
cudaError_t launch_encode_n(int lattice, bool dither, int dtype, const EncodeArgs &a, cudaStream_t s)
{
    switch (lattice) {
    case 1: return launch_encode_nd<N, 1>(dither, dtype, a, s);
    case 2: return launch_encode_nd<N, 2>(dither, dtype, a, s);
    case 4: return launch_encode_nd<N, 4>(dither, dtype, a, s);
    default: return launch_encode_nd<N, 8>(dither, dtype, a, s);
    }
}

}  // namespace

int encode_chunk_tiles(int tile)
{
    const int epl = tile <= 256 ? 8 : tile / 32;
    return kEncodeWarps * (32 / (tile / epl));
}

cudaError_t launch_encode(int tile, int lattice, bool dither, int dtype, const EncodeArgs &a,
                          cudaStream_t s)
{
    switch (tile) {
    case 64: return launch_encode_n<64>(lattice, dither, dtype, a, s);
    case 128: return launch_encode_n<128>(lattice, dither, dtype, a, s);
    case 256: return launch_encode_n<256>(lattice, dither, dtype, a, s);
    case 512: return launch_encode_n<512>(lattice, dither, dtype, a, s);
    default: return launch_encode_n<1024>(lattice, dither, dtype, a, s);
    }
}

}  // namespace hq
