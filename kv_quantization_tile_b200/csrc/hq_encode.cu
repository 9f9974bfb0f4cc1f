// hq_encode.cu -- single-pass tile encoder for sm_100a.
//
// Persistent blocks take chunks of T consecutive tiles (a contiguous span of
// the row-major input) from an atomic ticket, so chunks are started in order.
// Within a block, a group of LPT = N / EPL lanes owns G consecutive tiles of
// the chunk and, per tile:
//   loads it (128-bit, the next tile's load in flight), applies the random
//   signs (per-block table), forms the pairwise sum of squares, runs the
//   register + shuffle Walsh-Hadamard transform, derives Delta, quantizes
//   v / Delta [+ dither] to the nearest lattice point, strips and zigzags,
//   picks the Rice parameter (exact argmin: one pass evaluates k-1, k, k+1
//   around the rate's typical k and walks further only if needed), and packs
//   the tile into the group's shared-memory image.
// The chunk's word count is then published for a decoupled look-back prefix
// scan over chunks; one warp polls 32 predecessor slots at a time.  Every
// wait is bounded: a block that gives up raises HQ_ST_TIMEOUT, publishes its
// own prefix so later chunks proceed, and writes nothing.  Finally each group
// stores its image with coalesced stores and the block writes the chunk's
// tile headers.
//
// Method: [V1] "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline
// for Large Language and Diffusion Models", abstract (i)-(iv); [V2]
// "HyperQuant: A Near-Entropy-Optimal Lattice Quantization Pipeline for
// Large Language and Diffusion Models", abstract (strip, Rice code,
// subtractive dither).
#include <cuda_bf16.h>

#include "hq_fast.cuh"
#include "hq_internal.h"

namespace hq {

namespace {

constexpr int kEncodeWarps = 8;

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

// Named barriers between the compute warps and the store warp (0 is
// __syncthreads): image b ready / image b free again / ticket broadcast.
constexpr int kBarReady0 = 1, kBarFree0 = 3, kBarTicket = 5;

__device__ __forceinline__ void named_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void named_arrive(int id, int threads)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Decoupled look-back run by one whole warp: publish this chunk's aggregate,
// then sum predecessors 32 at a time until an inclusive prefix is found.
// Returns the exclusive prefix (same value in every lane).  A chunk that gives
// up waiting, or meets a poisoned predecessor before any inclusive prefix,
// publishes poison instead of a prefix and reports timed_out, so every later
// chunk also gives up without writing rather than using a wrong offset.

__device__ uint64_t chunk_lookback_warp(unsigned long long *lb, uint32_t chunk, uint64_t agg, int lane,
                                        bool publish, bool &timed_out)
{
    timed_out = false;
    if (chunk == 0) {
        if (lane == 0 && publish) st_release(&lb[0], kFlagInclusive | agg);
        return 0;
    }
    if (lane == 0 && publish) st_release(&lb[chunk], kFlagAggregate | agg);
    uint64_t excl = 0;
    int64_t top = (int64_t)chunk - 1;  // newest predecessor not yet summed
    uint32_t polls = 0;
    const uint64_t t0 = global_ns();
    while (top >= 0) {
        const int64_t p = top - lane;
        unsigned long long s = p >= 0 ? ld_acquire(&lb[p]) : (kFlagInclusive | 0ull);
        const uint64_t flag = s & ~kValueMask;
        const unsigned incl = __ballot_sync(FULL, flag == kFlagInclusive || flag == kFlagPoison);
        const unsigned none = __ballot_sync(FULL, flag == 0);
        // lanes up to and including the nearest inclusive (or poisoned) slot
        const unsigned upto = incl ? ((incl & -incl) << 1) - 1u : FULL;
        if (none & upto) {  // a needed predecessor has not published yet
            if (++polls > kSpinLimit || global_ns() - t0 > kWaitLimitNs) {
                timed_out = true;
                break;
            }
            __nanosleep(64);
            continue;
        }
        if (incl && __shfl_sync(FULL, flag, __ffs(incl) - 1) == kFlagPoison) {
            timed_out = true;  // an earlier chunk gave up: no valid prefix exists
            break;
        }
        uint64_t v = ((1u << lane) & upto) ? (s & kValueMask) : 0;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(FULL, v, m);
        excl += v;
        if (incl) break;
        top -= 32;
    }
    if (lane == 0 && publish)
        st_release(&lb[chunk], timed_out ? kFlagPoison : (kFlagInclusive | ((excl + agg) & kValueMask)));
    return excl;
}

template <int EPL, bool F32IN>
struct RawTile {
    uint4 q[F32IN ? EPL / 4 : EPL / 8];
};

template <int EPL, bool F32IN>
__device__ __forceinline__ void load_raw(const void *x, int64_t e0, RawTile<EPL, F32IN> &r)
{
    const uint4 *p = F32IN ? reinterpret_cast<const uint4 *>(static_cast<const float *>(x) + e0)
                           : reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + e0);
#pragma unroll
    for (int i = 0; i < (F32IN ? EPL / 4 : EPL / 8); i++) r.q[i] = __ldg(p + i);
}

// ---------------------------------------------------------------- packed path
// Unpack lane l's EPL raw coordinates into pairs and apply the random signs of
// the sign word Y (pair m's mask is (Y << m) & 0x80008000, see sign_word).
template <int EPL, bool F32IN>
__device__ __forceinline__ void unpack_signed(const RawTile<EPL, F32IN> &r, uint32_t Y, float2 (&P)[EPL / 2])
{
    if constexpr (F32IN) {
#pragma unroll
        for (int i = 0; i < EPL / 4; i++) {
            const uint32_t qq[4] = { r.q[i].x, r.q[i].y, r.q[i].z, r.q[i].w };
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int m = 2 * i + h;
                const uint32_t sm = Y << m;
                P[m] = make_float2(__uint_as_float(qq[2 * h] ^ ((sm << 16) & 0x80000000u)),
                                   __uint_as_float(qq[2 * h + 1] ^ (sm & 0x80000000u)));
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < EPL / 8; i++) {
            const uint32_t qq[4] = { r.q[i].x, r.q[i].y, r.q[i].z, r.q[i].w };
#pragma unroll
            for (int h = 0; h < 4; h++) {
                const int m = 4 * i + h;
                const uint32_t w = qq[h] ^ ((Y << m) & 0x80008000u);
                P[m] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
            }
        }
    }
}

// The sign word of lane l of column tile j (see sign_word): the lane's
// coordinates l EPL .. l EPL + EPL - 1 in pair order.
template <int N, int EPL>
__device__ __forceinline__ uint32_t encode_sign_word(uint64_t sign_key, uint64_t j, int l)
{
    const uint32_t i0 = (uint32_t)l * EPL;
    const uint64_t w = mix64(mix64(sign_key ^ j) ^ (uint64_t)(i0 >> 6));
    const uint32_t sb = (uint32_t)(w >> (i0 & 63));
    return sign_word<EPL>([&](int i) { return (sb >> i) & 1u; });
}

// Dither of the D-vector whose first coordinate is tile coordinate c0 (c0 a
// multiple of D); for D < 4, r4 carries one hash over the vectors of a group
// of four coordinates (call with consecutive vectors in order).
template <int D>
__device__ __forceinline__ void dither_at(uint64_t tile_key, uint32_t c0, float (&r4)[4], float (&delta)[D],
                                          const A2Consts &a2)
{
    if constexpr (D >= 4) {
#pragma unroll
        for (int b = 0; b < D / 4; b++) {
            uniform4(tile_key, c0 / 4 + b, r4);
#pragma unroll
            for (int k = 0; k < 4; k++) delta[4 * b + k] = box_dither<D>(r4[k], 4 * b + k, a2);
        }
    } else {
        if ((c0 & 3) == 0) uniform4(tile_key, c0 / 4, r4);
#pragma unroll
        for (int m = 0; m < D; m++) delta[m] = box_dither<D>(r4[(c0 & 3) + m], m, a2);
    }
}

// Nearest points of lane l's two runs after the half-exchange transform (run
// A: tile coordinates RL l .., run B: N/2 + RL l .., RL = EPL / 2) of
// v / Delta [+ dither], stripped and zigzagged, as exact binary32 integers in
// pairs (U[m]: symbols 2m, 2m + 1 of the lane's run-A-then-run-B order, each
// run in coordinate order).  sig: the transform's signs (bit 0: run A
// negated, bit 1: run B).  Returns the coset bits (bit q: run A's vector q,
// bit RL / D + q: run B's).  sb = 0: the all-zero tile.  E8 uses e8_symbols
// (the fma pipe), the other lattices the scalar nearest point.
template <int N, int D, int EPL, bool DITHER>
__device__ __forceinline__ uint32_t quantize_hx_f(const float2 (&P)[EPL / 2], uint32_t sb, uint32_t sig,
                                                  uint64_t tkey, int l, const A2Consts &a2, float2 (&U)[EPL / 2])
{
    constexpr int NP = EPL / 2, HP = NP / 2, RL = EPL / 2, VPR = RL / D;
#pragma unroll
    for (int m = 0; m < NP; m++) U[m] = make_float2(0.0f, 0.0f);
    if (sb == 0) return 0;
    uint32_t cbits = 0;
    const float inv = __frcp_rn(bf16_bits_to_float(sb));
    const float2 ia = splat2((sig & 1u) ? -inv : inv), ib = splat2((sig & 2u) ? -inv : inv);
    float2 X[NP];
#pragma unroll
    for (int m = 0; m < NP; m++) X[m] = mul2(P[m], m < HP ? ia : ib);
    float r4[4];
#pragma unroll
    for (int run = 0; run < 2; run++) {
        const uint32_t cbase = (run ? (uint32_t)N / 2 : 0u) + (uint32_t)l * RL;
#pragma unroll
        for (int q = 0; q < VPR; q++) {
            float x[D];
#pragma unroll
            for (int m = 0; m < D; m++) {
                const int i = q * D + m;  // coordinate within the run: pair i / 2, element i & 1
                x[m] = (i & 1) ? X[run * HP + i / 2].y : X[run * HP + i / 2].x;
            }
            if constexpr (DITHER) {
                float dl[D];
                dither_at<D>(tkey, cbase + (uint32_t)(q * D), r4, dl, a2);
#pragma unroll
                for (int m = 0; m < D; m++) x[m] = __fadd_rn(x[m], dl[m]);
            }
            float us[D];
            int c = 0;
            if constexpr (D == 8) {
                float2 V[4], W[4];
#pragma unroll
                for (int i = 0; i < 4; i++) V[i] = make_float2(x[2 * i], x[2 * i + 1]);
                c = e8_symbols(V, W);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    us[2 * i] = W[i].x;
                    us[2 * i + 1] = W[i].y;
                }
            } else {
                int z[D];
                float p[D];
                nearest<D>(x, c, z, p, a2);
#pragma unroll
                for (int m = 0; m < D; m++) {
                    int sv = z[m];
                    if constexpr (D == 8 || D == 4) {
                        if (m == D - 1) sv >>= 1;  // floor(z / 2): its parity follows from the even sum
                    }
                    us[m] = (float)zigzag(sv);
                }
            }
#pragma unroll
            for (int m = 0; m < D; m++) {
                const int i = q * D + m;
                if (i & 1) U[run * HP + i / 2].y = us[m];
                else U[run * HP + i / 2].x = us[m];
            }
            cbits |= (uint32_t)c << (run * VPR + q);
        }
    }
    return cbits;
}

// 2^e as a binary32 (e in -126 .. 127)
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// Sums over run A and run B of floor(u / 2^k) for one k: an fma rounded down
// against 1.5 2^23 leaves 1.5 2^23 + floor(u 2^-k), whose bit patterns are
// added as integers (the common bias removed at the end).
template <int EPL>
__device__ __forceinline__ void shifted_sums(const float2 (&U)[EPL / 2], int k, uint32_t &sa, uint32_t &sbv)
{
    constexpr int NP = EPL / 2, HP = NP / 2;
    const float2 sk = splat2(exp2i(-k)), M2 = splat2(12582912.0f);
    uint32_t a = 0, b = 0;
#pragma unroll
    for (int m = 0; m < NP; m++) {
        const float2 qb = __ffma2_rd(U[m], sk, M2);
        const uint32_t pair = (uint32_t)__float_as_int(qb.x) + (uint32_t)__float_as_int(qb.y);
        if (m < HP) a += pair;
        else b += pair;
    }
    constexpr uint32_t kBiasRun = (uint32_t)kMagicBias * (uint32_t)(EPL / 2);  // EPL / 2 biases, mod 2^32
    sa = a - kBiasRun;
    sbv = b - kBiasRun;
}

// Rice parameter: the smallest k minimising sum(u >> k) + N (1 + k) over the
// group's symbols.  One pass gives the sums at k0-1, k0, k0+1 (k0 = the
// rate's typical k); the cost is convex in k, so k0 is optimal iff
// C(k0-1) > C(k0) <= C(k0+1), and only otherwise does the search walk on.
// partA / partB: this lane's sum(u >> k) over run A / run B at the returned k.
template <int N, int EPL, int LPT>
__device__ __forceinline__ int rice_param_f(const float2 (&U)[EPL / 2], unsigned mask, int k_hint, uint32_t &partA,
                                            uint32_t &partB)
{
    int k = k_hint;
    const int km = k > 0 ? k - 1 : 0;
    uint32_t a0, b0, a1, b1, a2, b2;
    shifted_sums<EPL>(U, km, a0, b0);
    shifted_sums<EPL>(U, km + 1, a1, b1);
    shifted_sums<EPL>(U, km + 2, a2, b2);
    const uint32_t S0 = group_sum<LPT>(mask, a0 + b0), S1 = group_sum<LPT>(mask, a1 + b1),
                   S2 = group_sum<LPT>(mask, a2 + b2);
    bool up = false, down = false;
    if (k == 0) {
        if (S0 - S1 <= (uint32_t)N) {
            partA = a0; partB = b0;          // C(1) >= C(0)
        } else if (S1 - S2 <= (uint32_t)N) {
            k = 1; partA = a1; partB = b1;   // C(1) < C(0), C(2) >= C(1)
        } else {
            k = 2; partA = a2; partB = b2; up = true;
        }
    } else if (S0 - S1 <= (uint32_t)N) {     // C(k0 - 1) <= C(k0)
        k = km; partA = a0; partB = b0; down = true;
    } else if (S1 - S2 > (uint32_t)N && k < 15) {  // C(k0 + 1) < C(k0)
        k = k + 1; partA = a2; partB = b2; up = true;
    } else {
        partA = a1; partB = b1;
    }
    while (down && k > 0) {
        uint32_t da, db;
        shifted_sums<EPL>(U, k - 1, da, db);
        if (group_sum<LPT>(mask, da + db) - group_sum<LPT>(mask, partA + partB) > (uint32_t)N) break;
        --k; partA = da; partB = db;
    }
    while (up && k < 15) {
        uint32_t ua, ub;
        shifted_sums<EPL>(U, k + 1, ua, ub);
        if (group_sum<LPT>(mask, partA + partB) - group_sum<LPT>(mask, ua + ub) <= (uint32_t)N) break;
        ++k; partA = ua; partB = ub;
    }
    return k;
}

// Low parts and unary parts of one run of 8 float symbols (4 pairs) for
// k <= 4 and a unary span of at most 32 bits: the low word is sum_i low_i 2^(k i)
// formed exactly in binary32 as two halves of 4 codes (16 bits at most), the
// unary bitmap by Horner from the last code, bm = ((bm << 1) | 1) << q, with q
// taken from the biased floor pattern (its low 5 bits are q's).
__device__ __forceinline__ void run_words8(const float2 *U, int k, uint32_t &low, uint32_t &unary)
{
    const float2 sk = splat2(exp2i(-k)), M2 = splat2(12582912.0f), mpk = splat2(-exp2i(k));
    const float pk = exp2i(k), pk2 = exp2i(2 * k);
    float c[4];
    uint32_t qb[8];
#pragma unroll
    for (int m = 0; m < 4; m++) {
        const float2 b = __ffma2_rd(U[m], sk, M2);              // 1.5 2^23 + q
        const float2 lo = fma2(sub2(b, M2), mpk, U[m]);         // u - 2^k q
        c[m] = __fmaf_rn(lo.y, pk, lo.x);
        qb[2 * m] = (uint32_t)__float_as_int(b.x);
        qb[2 * m + 1] = (uint32_t)__float_as_int(b.y);
    }
    const float h0 = __fmaf_rn(c[1], pk2, c[0]), h1 = __fmaf_rn(c[3], pk2, c[2]);  // < 2^16: exact
    const uint32_t b0 = (uint32_t)__float_as_int(__fadd_rn(h0, 8388608.0f));       // 2^23 + h0
    const uint32_t b1 = (uint32_t)__float_as_int(__fadd_rn(h1, 8388608.0f));
    low = (b1 << (4 * k)) + b0 - (0x4B000000u << (4 * k)) - 0x4B000000u;
    uint32_t bm = 0;
#pragma unroll
    for (int i = 7; i >= 0; i--) bm = __funnelshift_l(0u, bm * 2u + 1u, qb[i]);
    unary = bm;
}

// OR `cnt` codes' k low bits (code i at bit pos + i k) into a zeroed image,
// four codes at a time, writes confined to the image's first `limit` words.
template <int CNT>
__device__ __forceinline__ void pack_low_run_lim(uint32_t *tbuf, uint32_t pos, int k, const uint32_t *u, uint32_t limit)
{
    const uint32_t lowmask = (1u << k) - 1u;
#pragma unroll
    for (int r0 = 0; r0 < CNT; r0 += 4) {  // 4 codes of up to 15 bits: at most 60 bits, as two 32-bit halves
        uint64_t acc = 0;
#pragma unroll
        for (int m = 3; m >= 0; m--) acc = (acc << k) | (u[r0 + m] & lowmask);
        const uint32_t p = pos + (uint32_t)r0 * k;
        or_bits32_lim(tbuf, p, (uint32_t)acc, 4 * k < 32 ? 4 * k : 32, limit);
        if (4 * k > 32) or_bits32_lim(tbuf, p + 32, (uint32_t)(acc >> 32), 4 * k - 32, limit);
    }
}

// OR `cnt` codes' unary parts into a zeroed image one terminator at a time,
// writes confined to the image's first `limit` words.
template <int CNT>
__device__ __forceinline__ void pack_unary_run_lim(uint32_t *tbuf, uint32_t pos, int k, const uint32_t *u,
                                                   uint32_t limit)
{
#pragma unroll
    for (int m = 0; m < CNT; m++) {
        pos += u[m] >> k;
        if ((pos >> 5) < limit) atomicOr(&tbuf[pos >> 5], 1u << (pos & 31));
        ++pos;
    }
}

// Pack lane l's two runs of float symbols into a zeroed shared-memory image:
// coset bits, low parts, and unary parts starting uoffA / uoffB bits into the
// unary section.  spanA / spanB: the runs' unary bits (sum of q + 1); limit:
// the words of the group's image from tbuf on (no write goes past them);
// mask: the group's lanes (all of them call this together).
template <int N, int D, int EPL>
__device__ __forceinline__ void pack_hx_f(uint32_t *tbuf, int l, int k, uint32_t cbits, const float2 (&U)[EPL / 2],
                                          uint32_t uoffA, uint32_t uoffB, uint32_t spanA, uint32_t spanB,
                                          uint32_t limit, unsigned mask)
{
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;
    constexpr int RL = EPL / 2, VPR = RL / D, HP = EPL / 4, LPT = N / EPL;
    if constexpr (C > 0 && VPR == 1 && 2 * LPT <= 32) {
        // one coset bit per run and lane: the group's bits by two ballots,
        // run A's in lane order, then run B's, OR-ed in by the first lane
        const int base = (threadIdx.x & 31) & ~(LPT - 1);
        const uint32_t gm = LPT == 32 ? 0xffffffffu : (1u << LPT) - 1u;
        const uint32_t ba = (__ballot_sync(mask, cbits & 1u) >> base) & gm;
        const uint32_t bb = (__ballot_sync(mask, cbits & 2u) >> base) & gm;
        if (l == 0) or_bits32_lim(tbuf, 0u, ba | (bb << LPT), C, limit);
    } else if constexpr (C > 0) {
        or_bits32_lim(tbuf, (uint32_t)l * VPR, cbits & ((1u << VPR) - 1u), VPR, limit);
        or_bits32_lim(tbuf, (uint32_t)(N / (2 * D)) + (uint32_t)l * VPR, cbits >> VPR, VPR, limit);
    }
    const uint32_t lowA = (uint32_t)C + (uint32_t)l * RL * (uint32_t)k;
    const uint32_t lowB = (uint32_t)C + ((uint32_t)N / 2 + (uint32_t)l * RL) * (uint32_t)k;
    const uint32_t ubase = (uint32_t)C + (uint32_t)N * (uint32_t)k;
    if (RL == 8 && k <= 4 && spanA <= 32 && spanB <= 32) {
        uint32_t wl, wu;
        run_words8(U, k, wl, wu);
        if (k) or_bits32_lim(tbuf, lowA, wl, 8 * k, limit);
        or_bits32_lim(tbuf, ubase + uoffA, wu, (int)spanA, limit);
        run_words8(U + HP, k, wl, wu);
        if (k) or_bits32_lim(tbuf, lowB, wl, 8 * k, limit);
        or_bits32_lim(tbuf, ubase + uoffB, wu, (int)spanB, limit);
    } else {
        uint32_t u[EPL];
#pragma unroll
        for (int m = 0; m < EPL / 2; m++) {
            u[2 * m] = (uint32_t)U[m].x;
            u[2 * m + 1] = (uint32_t)U[m].y;
        }
        if (k) {
            pack_low_run_lim<RL>(tbuf, lowA, k, u, limit);
            pack_low_run_lim<RL>(tbuf, lowB, k, u + RL, limit);
        }
        pack_unary_run_lim<RL>(tbuf, ubase + uoffA, k, u, limit);
        pack_unary_run_lim<RL>(tbuf, ubase + uoffB, k, u + RL, limit);
    }
}

}  // namespace

// Resident blocks per SM the compiler must fit registers for: 4 (64 registers)
// where the tile state fits, fewer for 32 coordinates per lane or dithered E8.
constexpr int encode_min_blocks(int epl, int d, bool dither) { return epl >= 32 ? 2 : ((dither && d == 8) ? 3 : 4); }

template <int N, int D, int EPL, bool DITHER, bool F32IN>
__global__ void __launch_bounds__(kEncodeWarps * 32, encode_min_blocks(EPL, D, DITHER))
    encode_kernel(const EncodeArgs a)
{
    constexpr int NCW = kEncodeWarps - 1;  // compute warps; the last warp scans and stores
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = NCW * TPW;
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;  // coset bits per tile
    constexpr int RL = EPL / 2;                        // coordinates per run
    static_assert(EPL % D == 0 && RL % D == 0 && LPT <= 32 && (32 % LPT) == 0 && EPL <= 32 && LPT >= 2, "layout");
    constexpr int kAll = kEncodeWarps * 32, kCompute = NCW * 32;

    const int G = a.tiles_per_group;
    const int T = GPB * G;  // tiles per chunk
    const int ywords = a.sign_words ? (int)a.tiles_per_row * LPT : 0;  // sign words cached per block
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *ytab = smem;                                                     // [tiles_per_row][LPT]
    const uint32_t gstride = ((uint32_t)G * a.wmax + 3u) & ~3u;                // words per group image
    uint32_t *stage0 = smem + ((ywords + 3) & ~3);                             // 2 x GPB x gstride
    uint32_t *meta0 = stage0 + (size_t)2 * GPB * gstride;                      // 2 x (2T + GPB)
    __shared__ uint32_t s_chunk[2];
    __shared__ uint32_t s_goff[64];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // per-block table of every column tile's sign words
    for (int i = tid; i < ywords; i += kAll)
        ytab[i] = encode_sign_word<N, EPL>(a.sign_key, (uint64_t)(i / LPT), i % LPT);
    __syncthreads();

    if (warp < NCW) {
        // ================= compute warps: encode chunks into alternating images
        const int l = lane % LPT;
        const int gid = warp * TPW + lane / LPT;
        const unsigned mask = group_mask<LPT>(lane);
        const uint32_t sig = hx_sigma_bits<LPT>(l);
        for (int it = 0;; it++) {
            const int b = it & 1;
            if (it >= 2) named_sync(kBarFree0 + b, kAll);  // the store warp is done with image b
            if (tid == 0) s_chunk[b] = atomicAdd(a.ticket, 1u);
            named_sync(kBarTicket, kCompute);
            const uint32_t chunk = s_chunk[b];
            if (chunk >= a.nchunks) {
                named_arrive(kBarReady0 + b, kAll);  // tells the store warp to finish
                // consume the store warp's last "image free" so every arrival is matched
                if (it >= 1) named_sync(kBarFree0 + ((it - 1) & 1), kAll);
                break;
            }
            uint32_t *gstage = stage0 + ((size_t)b * GPB + gid) * gstride;
            uint32_t *tile_w = meta0 + (size_t)b * (2 * T + GPB);  // T: word offset in group
            uint32_t *tile_hdr = tile_w + T;                         // T: scale | k << 16
            uint32_t *grp_w = tile_hdr + T;                          // GPB: words per group
            const int64_t t_first = (int64_t)chunk * T + (int64_t)gid * G;  // this group's first tile
            const uint32_t tpr = (uint32_t)a.tiles_per_row;
            uint32_t jj = 0;  // column tile of the current tile (consecutive tiles: j + 1 mod tpr)
            if (t_first < a.ntiles) jj = (uint32_t)t_first - fast_div((uint32_t)t_first, a.tpr_div) * tpr;
            {
                uint4 *zs = reinterpret_cast<uint4 *>(gstage);
                for (uint32_t i = l; i < gstride / 4; i += LPT) zs[i] = make_uint4(0u, 0u, 0u, 0u);
                __syncwarp(mask);
            }

            uint32_t goff = 0;  // words staged by this group so far
            RawTile<EPL, F32IN> raw;
            if (t_first < a.ntiles) load_raw<EPL, F32IN>(a.x, t_first * N + (int64_t)l * EPL, raw);
            for (int gi = 0; gi < G; gi++) {
                const int64_t t = t_first + gi;
                const bool active = t < a.ntiles;
                // ---- signs (v = s . w), as pairs
                const uint32_t Y = ywords ? ytab[jj * LPT + l] : encode_sign_word<N, EPL>(a.sign_key, jj, l);
                float2 v[EPL / 2];
                if (active) {
                    unpack_signed<EPL, F32IN>(raw, Y, v);
                    if (gi + 1 < G && t + 1 < a.ntiles) load_raw<EPL, F32IN>(a.x, (t + 1) * N + (int64_t)l * EPL, raw);
                } else {
#pragma unroll
                    for (int m = 0; m < EPL / 2; m++) v[m] = make_float2(0.0f, 0.0f);
                }
                if (++jj == tpr) jj = 0;

                // ---- scale (sum of squares is sign-blind) + rotation
                const float S = sumsq_pairs<EPL, LPT, !F32IN>(v, mask);
                fwht_hx<EPL, LPT>(v, mask, l);
                bool nonfinite;
                const uint32_t sb = tile_scale_bits(S, a.c, nonfinite);
                if (active && nonfinite && l == 0 && a.status) atomicOr(a.status, kStatusNonfinite);

                // ---- nearest point, strip, zigzag (symbols as exact binary32 integers)
                float2 U[EPL / 2];
                const uint64_t tkey = DITHER ? mix64(a.dither_key ^ (uint64_t)t) : 0ull;
                const uint32_t cbits = quantize_hx_f<N, D, EPL, DITHER>(v, sb, sig, tkey, l, a.a2, U);

                // ---- Rice parameter (exact argmin); this lane's sum(u >> k) per run
                uint32_t partA, partB;
                const int k = rice_param_f<N, EPL, LPT>(U, mask, a.k_hint, partA, partB);

                // ---- lengths: run A's unary parts precede run B's in the tile
                const uint32_t ulA = partA + RL, ulB = partB + RL;
                const uint32_t totA = group_sum<LPT>(mask, ulA);
                const uint32_t uoffA = group_excl_scan<LPT>(mask, ulA, l);
                const uint32_t uoffB = totA + group_excl_scan<LPT>(mask, ulB, l);
                const uint32_t utot = totA + group_sum<LPT>(mask, ulB);
                const uint32_t bits = (uint32_t)C + (uint32_t)N * (uint32_t)k + utot;
                uint32_t W = active ? (bits + 31) >> 5 : 0;
                const bool overflow = W > a.wmax;  // excluded by the bound; guards the image
                if (overflow) W = a.wmax;

                // ---- pack into the group's image (zeroed at chunk start)
                uint32_t *tbuf = gstage + goff;
                if (active && !overflow) pack_hx_f<N, D, EPL>(tbuf, l, k, cbits, U, uoffA, uoffB, ulA, ulB, gstride - goff, mask);
                if (overflow && l == 0 && a.status) atomicOr(a.status, kStatusCapacity);
                if (l == 0) {
                    tile_w[gid * G + gi] = goff;
                    tile_hdr[gid * G + gi] = sb | ((uint32_t)k << 16);
                }
                goff += W;
            }
            if (l == 0) grp_w[gid] = goff;
            named_arrive(kBarReady0 + b, kAll);
        }
    } else {
        // ================= store warp: chunk prefix, look-back, coalesced stores
        for (int it = 0;; it++) {
            const int b = it & 1;
            named_sync(kBarReady0 + b, kAll);
            const uint32_t chunk = s_chunk[b];
            if (chunk >= a.nchunks) break;
            const uint32_t *stage = stage0 + (size_t)b * GPB * gstride;
            const uint32_t *tile_w = meta0 + (size_t)b * (2 * T + GPB);
            const uint32_t *tile_hdr = tile_w + T;
            const uint32_t *grp_w = tile_hdr + T;
            // groups lane and lane + 32 (a block has at most 64 groups): their
            // word offsets in the chunk by one scan over the 64 counts in order
            static_assert(GPB <= 64, "store warp scans at most 64 groups");
            const uint32_t mine = lane < GPB ? grp_w[lane] : 0u;
            const uint32_t mine2 = lane + 32 < GPB ? grp_w[lane + 32] : 0u;
            uint32_t incl = mine, incl2 = mine2;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t o = __shfl_up_sync(FULL, incl, d), o2 = __shfl_up_sync(FULL, incl2, d);
                if (lane >= d) {
                    incl += o;
                    incl2 += o2;
                }
            }
            const uint32_t half = __shfl_sync(FULL, incl, 31);
            const uint32_t total = half + __shfl_sync(FULL, incl2, 31);
            const uint32_t gexcl = incl - mine;           // group `lane`'s word offset in the chunk
            const uint32_t gexcl2 = half + incl2 - mine2;  // group `lane + 32`'s
            bool to;
            const uint64_t base = chunk_lookback_warp(a.lb, chunk, total, lane, chunk != a.stall_chunk, to);
            if (to) {
                if (lane == 0 && a.status) atomicOr(a.status, kStatusTimeout);
            } else {
                const bool fits = base + total <= a.cap;
                if (!fits && lane == 0 && a.status) atomicOr(a.status, kStatusCapacity);
                if (fits) {
                    for (int g = 0; g < GPB; g++) {
                        const uint32_t go = g < 32 ? __shfl_sync(FULL, gexcl, g) : __shfl_sync(FULL, gexcl2, g - 32);
                        const uint32_t gw = g < 32 ? __shfl_sync(FULL, mine, g) : __shfl_sync(FULL, mine2, g - 32);
                        const uint32_t *src = stage + (size_t)g * gstride;
                        uint32_t *dst = a.payload + base + go;
                        uint32_t i = lane;
                        for (; i + 96 < gw; i += 128) {  // four loads in flight per lane
                            const uint32_t w0 = src[i], w1 = src[i + 32], w2 = src[i + 64], w3 = src[i + 96];
                            dst[i] = w0;
                            dst[i + 32] = w1;
                            dst[i + 64] = w2;
                            dst[i + 96] = w3;
                        }
                        for (; i < gw; i += 32) dst[i] = src[i];
                    }
                }
                if (lane < GPB) s_goff[lane] = gexcl;
                if (lane + 32 < GPB) s_goff[lane + 32] = gexcl2;
                __syncwarp();
                const int64_t t0 = (int64_t)chunk * T;
                for (int i = lane; i < T; i += 32) {
                    const int64_t t = t0 + i;
                    if (t < a.ntiles) {
                        a.off[t] = (uint32_t)(base + s_goff[i / G] + tile_w[i]);
                        a.scale[t] = (uint16_t)(tile_hdr[i] & 0xffffu);
                        a.kk[t] = (uint8_t)(tile_hdr[i] >> 16);
                    }
                }
                if (lane == 0 && chunk == a.nchunks - 1) a.off[a.ntiles] = (uint32_t)(base + total);
                __syncwarp();
            }
            named_arrive(kBarFree0 + b, kAll);
        }
    }
}

// ------------------------------------------------------------ fixed rate
// Fixed-rate tiles: every tile owns a slot of S words at word t S, so no
// offsets are computed or stored and tiles are independent.  Per tile the
// scale Delta is searched over bf16 bit patterns so that the coded tile fits
// its slot: the closed-form scale c0's size predicts a start (a pattern step
// moves the size by about N / 128 bits), then steps of 1, 2, 4, ... patterns
// towards the boundary (down while it fits, up until it fits; four octaves
// from c0 at most either way), then bisection to a fitting scale whose next
// finer pattern does not fit.  If no scale of the range fits, the tile is stored
// as the all-zero tile, which a legal slot always holds.  Each probe
// quantizes the rotated tile (held in registers) and prices it with the Rice
// parameter search; the probe's size is group-uniform, so each group walks
// its own search.  A group encodes the pair of tiles 2p, 2p + 1, which share
// the byte of packed 4-bit Rice parameters, into a zeroed shared-memory slot
// image and stores it whole.

constexpr int kFixedWarps = 8, kFixedThreads = kFixedWarps * 32;
// Resident blocks the registers are budgeted for: the rotated tile, the
// next tile's raw words and a probe's symbols are live together.  At 80
// registers (3 blocks per SM) E8 spills a few words, yet the Llama layer
// encodes faster than with 128 registers and no spills (2 blocks: 2.04 vs
// 1.87 ms) and level with 64 (4 blocks: 1.88 ms).
constexpr int fixed_min_blocks(int epl) { return epl >= 32 ? 1 : 3; }
constexpr int kFixedMaxProbes = 64;  // the search needs at most about 20
enum { kPredict, kStart, kDown, kUp, kBisect, kFinal };  // scale search phases

template <int N, int D, int EPL, bool DITHER, bool F32IN>
__global__ void __launch_bounds__(kFixedWarps * 32, fixed_min_blocks(EPL))
    encode_fixed_kernel(const EncodeArgs a)
{
    constexpr int LPT = N / EPL, TPW = 32 / LPT, GPB = kFixedWarps * TPW;
    constexpr int C = (D == 8 || D == 2) ? N / D : 0;
    constexpr int NP = EPL / 2, RL = EPL / 2;
    static_assert(EPL % D == 0 && RL % D == 0 && LPT <= 32 && (32 % LPT) == 0 && EPL <= 32 && LPT >= 2, "layout");
    const uint32_t S = a.slot_words;
    const uint32_t istride = (S + 1 + 3) & ~3u;  // slot image + a guard word, 16-byte multiple
    const int ywords = a.sign_words ? (int)a.tiles_per_row * LPT : 0;  // sign words cached per block
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *ytab = smem;                                       // [tiles_per_row][LPT]
    uint32_t *images = smem + ((ywords + 3) & ~3);
    float *sym = reinterpret_cast<float *>(images + (size_t)GPB * istride);  // [NP * 2 + 4][threads]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < ywords; i += kFixedThreads)
        ytab[i] = encode_sign_word<N, EPL>(a.sign_key, (uint64_t)(i / LPT), i % LPT);
    __syncthreads();

    const int l = lane % LPT;
    const int gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    const uint32_t sig = hx_sigma_bits<LPT>(l);
    uint32_t *img = images + (size_t)gid * istride;
    const int64_t npairs = (a.ntiles + 1) >> 1;
    const uint32_t tpr = (uint32_t)a.tiles_per_row;
    const uint32_t budget = 32u * S;
    uint32_t *keep = reinterpret_cast<uint32_t *>(sym);

    for (int64_t p = (int64_t)blockIdx.x * GPB + gid; p < npairs; p += (int64_t)gridDim.x * GPB) {
        uint32_t kbyte = 0;
        RawTile<EPL, F32IN> raw;
        const int64_t tp = 2 * p;
        load_raw<EPL, F32IN>(a.x, tp * N + (int64_t)l * EPL, raw);
        uint32_t jj = (uint32_t)tp - fast_div((uint32_t)tp, a.tpr_div) * tpr;
#pragma unroll 1
        for (int h = 0; h < 2; h++) {
            const int64_t t = tp + h;
            if (t >= a.ntiles) break;  // group-uniform
            // ---- signs (as pairs), then prefetch the pair's second tile
            const uint32_t Y = ywords ? ytab[jj * LPT + l] : encode_sign_word<N, EPL>(a.sign_key, jj, l);
            float2 v[NP];
            unpack_signed<EPL, F32IN>(raw, Y, v);
            if (h == 0 && t + 1 < a.ntiles) load_raw<EPL, F32IN>(a.x, (t + 1) * N + (int64_t)l * EPL, raw);
            if (++jj == tpr) jj = 0;

            // ---- rotation, closed-form start, scale search
            const float Ssq = sumsq_pairs<EPL, LPT, !F32IN>(v, mask);
            fwht_hx<EPL, LPT>(v, mask, l);
            bool nonfinite;
            const uint32_t c0 = tile_scale_bits(Ssq, a.c, nonfinite);
            if (nonfinite && l == 0 && a.status) atomicOr(a.status, kStatusNonfinite);
            const uint64_t tkey = DITHER ? mix64(a.dither_key ^ (uint64_t)t) : 0ull;

            // ---- scale search: one probe site (quantize + Rice parameter), a
            // state machine picking the next pattern.  Every fitting probe's
            // symbols are kept in shared memory, so the answer (the last
            // fitting probe) never needs a final pass; only the all-zero tile
            // runs one, on zeros.
            const int lo_lim = (int)c0 - 512 > 0x0080 ? (int)c0 - 512 : 0x0080;
            const int hi_lim = (int)c0 + 512 < 0x7f7f ? (int)c0 + 512 : 0x7f7f;
            int phase = c0 ? kPredict : kFinal, lo = 0, hi = (int)c0, step = 1, c = (int)c0;
            float2 U[NP];
            uint32_t cbits, partA, partB;
            int k;
            for (int probe = 0;; probe++) {
                cbits = quantize_hx_f<N, D, EPL, DITHER>(v, (uint32_t)c, sig, tkey, l, a.a2, U);
                k = rice_param_f<N, EPL, LPT>(U, mask, a.k_hint, partA, partB);
                if (phase == kFinal) break;
                const uint32_t bits = (uint32_t)C + (uint32_t)N * (uint32_t)(k + 1) + group_sum<LPT>(mask, partA + partB);
                const bool f = bits <= budget;
                if (f) {  // keep a fitting probe's symbols: the search's answer is its last fitting probe
#pragma unroll
                    for (int m = 0; m < NP; m++) {
                        sym[(2 * m) * kFixedThreads + tid] = U[m].x;
                        sym[(2 * m + 1) * kFixedThreads + tid] = U[m].y;
                    }
                    keep[(EPL + 0) * kFixedThreads + tid] = cbits;
                    keep[(EPL + 1) * kFixedThreads + tid] = (uint32_t)k;
                    keep[(EPL + 2) * kFixedThreads + tid] = partA;
                    keep[(EPL + 3) * kFixedThreads + tid] = partB;
                }
                if (phase == kPredict) {
                    // a pattern step moves the size by about N / 128 bits: start
                    // from c0 + floor(128 (bits - budget) / N), clamped
                    const int num = 128 * ((int)bits - (int)budget);
                    const int shift = num >= 0 ? num / N : -((-num + N - 1) / N);
                    const int start = c + shift < lo_lim ? lo_lim : (c + shift > hi_lim ? hi_lim : c + shift);
                    phase = kStart;
                    if (start != c) {
                        c = start;
                        continue;
                    }
                }
                if (phase == kStart) {
                    if (f) { hi = c; phase = kDown; } else { lo = c; phase = kUp; }
                } else if (phase == kDown) {
                    if (f) { hi = c; step *= 2; } else { lo = c; phase = kBisect; }
                } else if (phase == kUp) {
                    if (f) { hi = c; phase = kBisect; } else { lo = c; step *= 2; }
                } else {
                    if (f) hi = c; else lo = c;
                }
                int next = -1, answer = -1;  // the next probe, or the search's answer
                if (phase == kDown) {
                    if (hi == lo_lim) answer = hi;
                    else next = hi - step > lo_lim ? hi - step : lo_lim;
                } else if (phase == kUp) {
                    if (lo == hi_lim) answer = 0;  // no scale of the range fits: the all-zero tile
                    else next = lo + step < hi_lim ? lo + step : hi_lim;
                } else {
                    if (hi - lo <= 1) answer = hi;
                    else next = (lo + hi) >> 1;
                }
                if (answer < 0 && probe + 1 >= kFixedMaxProbes)  // not reached: the search ends well before
                    answer = phase == kUp ? 0 : hi;
                if (answer < 0) {
                    c = next;
                } else {
                    if (answer == c && f) break;  // the last probe is the answer
                    c = answer;
                    if (answer != 0) {  // an earlier fitting probe: its kept symbols
#pragma unroll
                        for (int m = 0; m < NP; m++)
                            U[m] = make_float2(sym[(2 * m) * kFixedThreads + tid], sym[(2 * m + 1) * kFixedThreads + tid]);
                        cbits = keep[(EPL + 0) * kFixedThreads + tid];
                        k = (int)keep[(EPL + 1) * kFixedThreads + tid];
                        partA = keep[(EPL + 2) * kFixedThreads + tid];
                        partB = keep[(EPL + 3) * kFixedThreads + tid];
                        break;
                    }
                    phase = kFinal;  // the all-zero tile
                }
            }
            const uint32_t sb = (uint32_t)c;

            // ---- pack the chosen symbols (run A's unary parts precede run B's), store the slot
            const uint32_t ulA = partA + RL, ulB = partB + RL;
            const uint32_t totA = group_sum<LPT>(mask, ulA);
            const uint32_t uoffA = group_excl_scan<LPT>(mask, ulA, l);
            const uint32_t uoffB = totA + group_excl_scan<LPT>(mask, ulB, l);
            for (uint32_t i = l; i < istride; i += LPT) img[i] = 0u;
            __syncwarp(mask);
            pack_hx_f<N, D, EPL>(img, l, k, cbits, U, uoffA, uoffB, ulA, ulB, istride, mask);
            __syncwarp(mask);
            uint32_t *dst = a.payload + (uint64_t)t * S;
            for (uint32_t i = l; i < S; i += LPT) dst[i] = img[i];
            __syncwarp(mask);  // the image is reused by the next tile
            if (l == 0) a.scale[t] = (uint16_t)sb;
            kbyte |= (uint32_t)k << (4 * h);
        }
        if (l == 0) a.kk[p] = (uint8_t)kbyte;
    }
}

// ------------------------------------------------------------------ launch
namespace {

// coordinates per lane (both encoders): at least 16, so each of a lane's two
// runs after the half-exchange transform holds whole E8 vectors
template <int N>
constexpr int epl_var() { return N <= 256 ? 16 : 32; }

template <int N>
constexpr int groups_per_block() { return (kEncodeWarps - 1) * (32 / (N / epl_var<N>())); }

template <int N, int D, bool DITHER, bool F32IN>
cudaError_t launch_encode_t(const EncodeArgs &a0, cudaStream_t s)
{
    constexpr int EPL = epl_var<N>(), GPB = groups_per_block<N>();
    EncodeArgs a = a0;
    const int T = GPB * a.tiles_per_group;
    const size_t gstride = ((size_t)a.tiles_per_group * a.wmax + 3) & ~(size_t)3;
    const size_t ywords = a.sign_words ? (size_t)a.tiles_per_row * (N / EPL) : 0;
    const size_t smem = ((ywords + 3) & ~(size_t)3) * 4 + 2 * (size_t)GPB * gstride * 4 +
                        2 * ((size_t)T * 8 + (size_t)GPB * 4);
    auto kern = encode_kernel<N, D, EPL, DITHER, F32IN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kEncodeWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t blocks = (int64_t)sm_count() * per_sm;
    if (blocks > a.nchunks) blocks = a.nchunks;
    kern<<<(unsigned)blocks, kEncodeWarps * 32, smem, s>>>(a);
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

template <int N, int D, bool DITHER, bool F32IN>
cudaError_t launch_encode_fixed_t(const EncodeArgs &a, cudaStream_t s)
{
    constexpr int EPL = epl_var<N>(), GPB = kFixedWarps * (32 / (N / EPL));
    const size_t istride = (a.slot_words + 1 + 3) & ~(size_t)3;
    const size_t ywords = a.sign_words ? (size_t)a.tiles_per_row * (N / EPL) : 0;
    const size_t smem = ((ywords + 3) & ~(size_t)3) * 4 + (size_t)GPB * istride * 4 +
                        (size_t)(EPL + 4) * kFixedThreads * 4;
    auto kern = encode_fixed_kernel<N, D, EPL, DITHER, F32IN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFixedWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t npairs = (a.ntiles + 1) / 2;
    int64_t blocks = (npairs + GPB - 1) / GPB;
    const int64_t wave = (int64_t)sm_count() * per_sm;
    if (blocks > wave) blocks = wave;
    kern<<<(unsigned)blocks, kFixedWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int N, int D>
cudaError_t launch_encode_fixed_nd(bool dither, int dtype, const EncodeArgs &a, cudaStream_t s)
{
    if (dither)
        return dtype ? launch_encode_fixed_t<N, D, true, true>(a, s) : launch_encode_fixed_t<N, D, true, false>(a, s);
    return dtype ? launch_encode_fixed_t<N, D, false, true>(a, s) : launch_encode_fixed_t<N, D, false, false>(a, s);
}

template <int N>
cudaError_t launch_encode_fixed_n(int lattice, bool dither, int dtype, const EncodeArgs &a, cudaStream_t s)
{
    switch (lattice) {
    case 1: return launch_encode_fixed_nd<N, 1>(dither, dtype, a, s);
    case 2: return launch_encode_fixed_nd<N, 2>(dither, dtype, a, s);
    case 4: return launch_encode_fixed_nd<N, 4>(dither, dtype, a, s);
    default: return launch_encode_fixed_nd<N, 8>(dither, dtype, a, s);
    }
}

int groups_for(int tile)
{
    switch (tile) {
    case 64: return groups_per_block<64>();
    case 128: return groups_per_block<128>();
    case 256: return groups_per_block<256>();
    case 512: return groups_per_block<512>();
    default: return groups_per_block<1024>();
    }
}

}  // namespace

// Tiles per group per chunk: as many as keep the two staged images within
// 48 KB (at most 8), so a chunk spans up to 8 x (groups per block) tiles.
int encode_tiles_per_group(int tile, uint32_t wmax, int64_t ntiles)
{
    const int gpb = groups_for(tile);
    int g = (int)((48u * 1024u) / (2u * (uint32_t)gpb * wmax * 4u));  // two staging images in 48 KB
    g = g < 1 ? 1 : (g > 8 ? 8 : g);
    // small matrices: smaller chunks, so every resident block gets about one
    // (measured best against one-tile and three-per-block chunks)
    const int64_t blocks = 4 * (int64_t)sm_count();
    const int64_t gp = ntiles / ((int64_t)gpb * blocks);
    if (gp < g) g = gp < 1 ? 1 : (int)gp;
    return g;
}

// Smallest chunk for a tile length (one tile per group): sizes the workspace.
int encode_chunk_tiles(int tile) { return groups_for(tile); }

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

cudaError_t launch_encode_fixed(int tile, int lattice, bool dither, int dtype, const EncodeArgs &a,
                                cudaStream_t s)
{
    switch (tile) {
    case 64: return launch_encode_fixed_n<64>(lattice, dither, dtype, a, s);
    case 128: return launch_encode_fixed_n<128>(lattice, dither, dtype, a, s);
    case 256: return launch_encode_fixed_n<256>(lattice, dither, dtype, a, s);
    case 512: return launch_encode_fixed_n<512>(lattice, dither, dtype, a, s);
    default: return launch_encode_fixed_n<1024>(lattice, dither, dtype, a, s);
    }
}

}  // namespace hq
