// hq_gemm.cu -- batched decode + matrix product on the 5th-generation tensor
// cores (sm_100a: tcgen05.mma with TMEM accumulators).
//
//   Y[b][r] = sum_c x[b][c] w_hat[r][c]
//           = (1/n) sum_j < H (s_j . x_bj), Delta_rj y_rj >     (H symmetric)
//
// so the weights never leave the rotated domain: a block parses 128 rows of
// one column tile j straight from the stream into a bf16 A operand
// (Delta_rj * y, row-major along K), the rotated activations
// X~ = H (s_j . x_bj) (rotated once per call by rotate_x_kernel) form the B
// operand, and one thread issues the 16 K=16 MMAs of the tile into an fp32
// accumulator in tensor memory.  The parse is the cost; the MMAs take a
// small fraction of it.  Column tiles may be split across blocks (split-K);
// the partial sums are added in a fixed order by splitk_reduce_kernel.
//
// Method: [V2] "HyperQuant: A Near-Entropy-Optimal Lattice Quantization
// Pipeline for Large Language and Diffusion Models", abstract (algebraic
// decoding, the decode path against bf16 matrix products); [V1]
// "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline for Large
// Language and Diffusion Models", abstract (low-bit MMA decode paths).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "hq_parse.cuh"

namespace hq {

namespace {

constexpr int kGemmWarps = 16, kGemmThreads = kGemmWarps * 32;
constexpr int kGemmM = 128;  // weight rows per block (the MMA's M)
constexpr int kGemmN = 256;  // tile length handled here
// Operand layout (SWIZZLE_NONE, K-major): 16-byte chunks of 8 bf16; chunk
// (m, kc) at 16 B x ((m % 8) + 8 (m / 8) + LBO kc).  SBO = 8 chunks (one
// 8 x 16 B core matrix per 8 rows); an odd LBO (rows x 16 B + 16 B) spreads
// the 16 lanes writing one row's chunks over the shared-memory banks.
__host__ __device__ constexpr uint32_t gemm_lbo(int rows) { return (uint32_t)rows + 1; }
__host__ __device__ constexpr uint32_t gemm_operand_bytes(int rows) { return 32u * gemm_lbo(rows) * 16u; }

// ---------------------------------------------------------------- PTX
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t make_smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3fffu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    return d;                // base offset 0, LBO mode 0, layout SWIZZLE_NONE
}

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, M x N.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int m, int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// kind::i8 instruction descriptor: s32 accumulator, signed 8-bit A and B,
// both K-major, M x N.
__host__ __device__ constexpr uint32_t make_idesc_i8(int m, int n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// 8-bit operands: a 256-element row is 16 chunks of 16 bytes (same chunk
// layout as the bf16 operands, half the chunks).
__host__ __device__ constexpr uint32_t gemm_operand_bytes_i8(int rows) { return 16u * gemm_lbo(rows) * 16u; }

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// kind::f8f6f4 instruction descriptor: fp32 accumulator, E4M3 A and B (type
// code 0), both K-major, M x N.
__host__ __device__ constexpr uint32_t make_idesc_e4m3(int m, int n)
{
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void umma_e4m3(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// E4M3 bits of x, round to nearest even, saturating to +-448 (NaN stays NaN)
__device__ __forceinline__ uint32_t e4m3_bits(float x)
{
    return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ void umma_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

// Bounded wait for phase `parity` of an mbarrier (2^24 polls or 0.5 s of
// the global timer, whichever first); false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity)
{
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kSpinLimit; i++) {
        if ((i & 1023u) == 1023u && global_ns() - t0 > kWaitLimitNs) return false;
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16-byte global -> shared copy through L2 (cp.async, no registers held)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}

}  // namespace

// ------------------------------------------------------------ rotate x
// X~[b][j n + i] = bf16(H (s_j . x_bj))_i for b < batch, 0 for the padding
// rows up to batch_pad.  One 16-lane group per (b, j) tile.
__global__ void __launch_bounds__(256) rotate_x_kernel(const GemmArgs a)
{
    constexpr int N = kGemmN, EPL = 16, LPT = 16, GPB = 16;
    const int lane = threadIdx.x & 31, l = lane % LPT;
    const unsigned mask = group_mask<LPT>(lane);
    const int64_t ntiles = (int64_t)a.batch_pad * a.tiles_per_row;
    for (int64_t t = (int64_t)blockIdx.x * GPB + threadIdx.x / LPT; t < ntiles; t += (int64_t)gridDim.x * GPB) {
        const int64_t b = t / a.tiles_per_row, j = t % a.tiles_per_row;
        float v[EPL];
        if (b < a.batch) {
            const uint4 *p = reinterpret_cast<const uint4 *>(a.x + b * a.cols + j * N + l * EPL);
#pragma unroll
            for (int i = 0; i < EPL / 8; i++) {
                const uint4 q = __ldg(p + i);
                const uint32_t qq[4] = { q.x, q.y, q.z, q.w };
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    v[8 * i + 2 * h] = __uint_as_float(qq[h] << 16);
                    v[8 * i + 2 * h + 1] = __uint_as_float(qq[h] & 0xffff0000u);
                }
            }
            const uint32_t i0 = (uint32_t)l * EPL;
            const uint64_t w = mix64(mix64(a.sign_key ^ (uint64_t)j) ^ (uint64_t)(i0 >> 6));
            const uint32_t sb = (uint32_t)(w >> (i0 & 63));
#pragma unroll
            for (int r = 0; r < EPL; r++) v[r] = __uint_as_float(__float_as_uint(v[r]) ^ ((sb << (31 - r)) & 0x80000000u));
            fwht<EPL, LPT>(v, mask, l);
        } else {
#pragma unroll
            for (int r = 0; r < EPL; r++) v[r] = 0.0f;
        }
        uint4 *o = reinterpret_cast<uint4 *>(a.xt + b * a.cols + j * N + l * EPL);
#pragma unroll
        for (int i = 0; i < EPL / 8; i++)
            o[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                              pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
    }
}

// ------------------------------------------------------------ decode + MMA
// Blocks take work items (row block of 128 weight rows, batch block of NB
// rows, K split of column tiles [j0, j1)) in turn.  Per column
// tile: every 16-lane group parses rows into A (bf16 Delta y, K-major), all
// threads copy X~ into B, one thread issues 16 MMAs (K = 16 each) into the
// TMEM accumulator and commits them to an mbarrier that the next tile's
// writers wait on (bounded).  After an item's last tile, warps 0-3 read the
// accumulator (row = TMEM lane) and store it.
template <int D, int NB, bool FIXED>
__global__ void __launch_bounds__(kGemmThreads, 2) gemm_tc_kernel(const GemmArgs a)
{
    constexpr int N = kGemmN, EPL = 16, LPT = 16, TPW = 2, GPB = kGemmWarps * TPW;
    constexpr uint32_t LBO_A = gemm_lbo(kGemmM) * 16u, LBO_B = gemm_lbo(NB) * 16u;
    constexpr uint32_t NCOLS = NB < 32 ? 32u : (uint32_t)NB;  // TMEM columns: a power of two >= 32
    constexpr uint32_t IDESC = make_idesc_bf16(kGemmM, NB);
    extern __shared__ __align__(128) uint8_t smraw[];
    uint8_t *sA = smraw;
    uint8_t *sB = sA + gemm_operand_bytes(kGemmM);
    uint32_t *wbase = reinterpret_cast<uint32_t *>(sB + gemm_operand_bytes(NB));
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    uint32_t *wbuf = wbase + gid * group_words(a.w.wmax);
    const uint32_t bar = smem_u32(&mbar);

    if (warp == 0) tmem_alloc(smem_u32(&tmem_base), NCOLS);
    if (tid == 0) {
        mbar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t aA = smem_u32(sA), aB = smem_u32(sB);
    const int64_t row_blocks = (a.rows + kGemmM - 1) / kGemmM, batch_blocks = a.batch_pad / NB;
    const int64_t items = row_blocks * batch_blocks * a.ksplit;

    uint32_t parity = 0;
    bool fail = false, pending = false;  // pending: an MMA commit not yet waited for
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int ks = (int)(it % a.ksplit);
        const int64_t rb = (it / a.ksplit) % row_blocks, bb = it / (a.ksplit * row_blocks);
        const int64_t r0 = rb * kGemmM;
        const int b0 = (int)bb * NB;
        const int64_t j0 = (int64_t)ks * a.tiles_per_split;
        const int64_t j1 = j0 + a.tiles_per_split < a.tiles_per_row ? j0 + a.tiles_per_split : a.tiles_per_row;
        for (int64_t j = j0; j < j1; j++) {
            if (pending) {  // the previous MMAs have read A and B
                const bool ok = mbar_wait(bar, parity);
                parity ^= 1u;
                pending = false;
                // Every thread leaves together.  The wait gives up only when a
                // tile's MMAs were never issued and committed (the stall hook
                // withholds them); committed MMAs finish in microseconds, so no
                // tensor-core work is in flight when the block then frees TMEM.
                if (__syncthreads_or(!ok)) {
                    fail = true;
                    break;
                }
            }
            // B: X~ rows b0 .. b0 + NB - 1 of tile j (consecutive threads:
            // consecutive rows), copied asynchronously while A is parsed
            for (int e = tid; e < NB * 32; e += kGemmThreads) {
                const int n = e % NB, kc = e / NB;
                cp_async16(aB + (uint32_t)((n & 7) + 8 * (n >> 3)) * 16u + (uint32_t)kc * LBO_B,
                           a.xt + (int64_t)(b0 + n) * a.cols + j * N + kc * 8);
            }
            cp_async_commit();
            // A: rows r0 .. r0 + 127 of column tile j, lane l's chunks 2l and 2l + 1
            for (int m = gid; m < kGemmM; m += GPB) {
                const int64_t r = r0 + m;
                float pt[EPL];
                uint32_t sb = 0;
                bool bad = false;
                if (r < a.rows) {
                    bad = parse_tile<N, D, EPL, FIXED>(a.w, r * a.tiles_per_row + j, wbuf, mask, l, pt, sb);
                } else {
#pragma unroll
                    for (int i = 0; i < EPL; i++) pt[i] = 0.0f;
                }
                const float delta = bf16_bits_to_float(sb);
                uint8_t *row = sA + (uint32_t)((m & 7) + 8 * (m >> 3)) * 16u;
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    const float *q = pt + 8 * h;
                    *reinterpret_cast<uint4 *>(row + (uint32_t)(2 * l + h) * LBO_A) =
                        make_uint4(pack_bf16x2(delta * q[0], delta * q[1]), pack_bf16x2(delta * q[2], delta * q[3]),
                                   pack_bf16x2(delta * q[4], delta * q[5]), pack_bf16x2(delta * q[6], delta * q[7]));
                }
                if (bad && l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
            }
            cp_async_wait_all();  // this thread's B chunks have landed
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0 && j != a.stall_tile) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < N / 16; s++) {
                    const uint64_t ad = make_smem_desc(aA + 2u * s * LBO_A, LBO_A, 128u);
                    const uint64_t bd = make_smem_desc(aB + 2u * s * LBO_B, LBO_B, 128u);
                    umma_bf16(tmem, ad, bd, IDESC, (j > j0 || s > 0) ? 1u : 0u);
                }
                umma_commit(bar);
            }
            pending = true;
        }
        if (pending) {
            const bool ok = mbar_wait(bar, parity);
            parity ^= 1u;
            pending = false;
            if (__syncthreads_or(!ok)) fail = true;
        }
        tc_fence_after();
        // epilogue: warp w < 4 owns TMEM lanes (rows) 32 w .. 32 w + 31; after
        // a wait that gave up the accumulator is not read (zeros are stored)
        if (warp < 4) {
            const int64_t r = r0 + warp * 32 + lane;
#pragma unroll
            for (int c = 0; c < NB; c += 16) {
                float v[16];
                if (!fail) {
                    tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; i++) v[i] = 0.0f;
                }
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const int b = b0 + c + i;
                    if (r < a.rows && b < a.batch) {
                        const float val = (j1 > j0 && !fail) ? v[i] * (1.0f / N) : 0.0f;
                        if (a.ksplit == 1) a.y[(int64_t)b * a.rows + r] = val;
                        else a.part[((int64_t)ks * a.batch_pad + b) * a.rows + r] = val;
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();  // the accumulator is read before the next item overwrites it
        tc_fence_after();
        if (fail) break;  // block-uniform: stop after a wait that gave up
    }
    if (fail && tid == 0 && a.status) atomicOr(a.status, kStatusTimeout);
    if (warp == 0) tmem_dealloc(tmem, NCOLS);
}

// y[b][r] = sum over K splits s (in order) of part[s][b][r].
__global__ void splitk_reduce_kernel(const GemmArgs a)
{
    const int64_t n = (int64_t)a.batch * a.rows;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = e / a.rows, r = e % a.rows;
        float s = 0.0f;
        for (int k = 0; k < a.ksplit; k++) s += a.part[((int64_t)k * a.batch_pad + b) * a.rows + r];
        a.y[e] = s;
    }
}

// ------------------------------------------------------------ int8 product
// The integer variant ([V1]: 8-bit MMA paths, int8 ahead of fp8 on the
// lattice output after the rotation).  The doubled lattice coordinates 2y are
// exact integers for E8 (y in Z or Z + 1/2), D4 and Z, so A = 2y in int8
// (saturated to +-127, flagged); the activations, rotated like the weights,
// are quantized per (batch row, column tile) to q = rint(x~ 127 / max|x~|)
// with scale s = max|x~| / 127.  Per column tile the tensor cores form the
// exact int32 sums A q; the epilogue scales them by Delta_rj s_bj / (2 n) and
// accumulates in fp32:  Y[b][r] = sum_j Delta_rj s_bj / (2 n) sum_i A_rji q_bji.

// Q[b][j n + i] and S[b][j] for b < batch_pad (zero for the padding rows);
// FP8: q = e4m3(x~ 448 / max|x~|), s = max|x~| / 448 (the fp8 variant).
template <bool FP8>
__global__ void __launch_bounds__(256) rotate_quant_x_kernel(const GemmArgs a)
{
    constexpr float kQmax = FP8 ? 448.0f : 127.0f;
    constexpr int N = kGemmN, EPL = 16, LPT = 16, GPB = 16;
    const int lane = threadIdx.x & 31, l = lane % LPT;
    const unsigned mask = group_mask<LPT>(lane);
    const int64_t ntiles = (int64_t)a.batch_pad * a.tiles_per_row;
    for (int64_t t = (int64_t)blockIdx.x * GPB + threadIdx.x / LPT; t < ntiles; t += (int64_t)gridDim.x * GPB) {
        const int64_t b = t / a.tiles_per_row, j = t % a.tiles_per_row;
        float v[EPL];
        if (b < a.batch) {
            const uint4 *p = reinterpret_cast<const uint4 *>(a.x + b * a.cols + j * N + l * EPL);
#pragma unroll
            for (int i = 0; i < EPL / 8; i++) {
                const uint4 q = __ldg(p + i);
                const uint32_t qq[4] = { q.x, q.y, q.z, q.w };
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    v[8 * i + 2 * h] = __uint_as_float(qq[h] << 16);
                    v[8 * i + 2 * h + 1] = __uint_as_float(qq[h] & 0xffff0000u);
                }
            }
            const uint32_t i0 = (uint32_t)l * EPL;
            const uint64_t w = mix64(mix64(a.sign_key ^ (uint64_t)j) ^ (uint64_t)(i0 >> 6));
            const uint32_t sb = (uint32_t)(w >> (i0 & 63));
#pragma unroll
            for (int r = 0; r < EPL; r++) v[r] = __uint_as_float(__float_as_uint(v[r]) ^ ((sb << (31 - r)) & 0x80000000u));
            fwht<EPL, LPT>(v, mask, l);
        } else {
#pragma unroll
            for (int r = 0; r < EPL; r++) v[r] = 0.0f;
        }
        // max |x~|: bit patterns of non-negative floats order like the values
        // (a NaN above infinity, which then propagates through the scale)
        uint32_t mb = 0;
#pragma unroll
        for (int r = 0; r < EPL; r++) mb = max(mb, __float_as_uint(fabsf(v[r])));
        mb = __reduce_max_sync(mask, mb);
        const float amax = __uint_as_float(mb);
        uint32_t wq[4] = { 0u, 0u, 0u, 0u };
        float scale = amax;
        if (mb != 0u && mb < 0x7f800000u) {
            const float inv = __fdiv_rn(kQmax, amax);
#pragma unroll
            for (int r = 0; r < EPL; r++) {
                const float xs = __fmul_rn(v[r], inv);
                const uint32_t q = FP8 ? e4m3_bits(xs) : ((uint32_t)__float2int_rn(xs) & 0xffu);  // |q| <= 127
                wq[r >> 2] |= q << (8 * (r & 3));
            }
            scale = __fdiv_rn(amax, kQmax);
        }
        *reinterpret_cast<uint4 *>(a.xq + b * a.cols + j * N + l * EPL) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
        if (l == 0) a.sx[b * a.tiles_per_row + j] = scale;
    }
}

// Work items as in gemm_tc_kernel.  Per column tile: every 16-lane group
// parses rows into A (int8 2y, K-major) and keeps each row's Delta, all
// threads copy Q into B and its scales, one thread issues 8 MMAs (K = 32
// each) into an s32 TMEM accumulator.  After the MMAs of tile j complete,
// warps 0-3 read the accumulator (row = TMEM lane), scale each sum by
// Delta s / (2 n) and add it to the item's fp32 sums in shared memory while
// the other warps parse tile j + 1 (the row and batch scales are double
// buffered); the item's sums are stored after its last tile.
template <int D, int NB, bool FIXED, bool FP8>
__global__ void __launch_bounds__(kGemmThreads, 2) gemm_i8_kernel(const GemmArgs a)
{
    constexpr int N = kGemmN, EPL = 16, LPT = 16, TPW = 2, GPB = kGemmWarps * TPW;
    constexpr uint32_t LBO_A = gemm_lbo(kGemmM) * 16u, LBO_B = gemm_lbo(NB) * 16u;
    constexpr uint32_t NCOLS = NB < 32 ? 32u : (uint32_t)NB;
    constexpr uint32_t IDESC = FP8 ? make_idesc_e4m3(kGemmM, NB) : make_idesc_i8(kGemmM, NB);
    static_assert(NB == 16 || NB == 32 || NB == 64 || NB == 128, "8-bit batch block");
    extern __shared__ __align__(128) uint8_t smraw[];
    uint8_t *sA = smraw;
    uint8_t *sB = sA + gemm_operand_bytes_i8(kGemmM);
    float *acc = reinterpret_cast<float *>(sB + gemm_operand_bytes_i8(NB));  // [NB][128] fp32 sums
    float *dlt = acc + NB * kGemmM;                                          // [2][128] Delta per row
    float *sxs = dlt + 2 * kGemmM;                                           // [2][NB] scale per batch row
    uint32_t *wbase = reinterpret_cast<uint32_t *>(sxs + 2 * NB);
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane % LPT, gid = warp * TPW + lane / LPT;
    const unsigned mask = group_mask<LPT>(lane);
    uint32_t *wbuf = wbase + gid * group_words(a.w.wmax);
    const uint32_t bar = smem_u32(&mbar);

    if (warp == 0) tmem_alloc(smem_u32(&tmem_base), NCOLS);
    if (tid == 0) {
        mbar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t aA = smem_u32(sA), aB = smem_u32(sB);
    const int64_t row_blocks = (a.rows + kGemmM - 1) / kGemmM, batch_blocks = a.batch_pad / NB;
    const int64_t items = row_blocks * batch_blocks * a.ksplit;
    constexpr float kInv2N = 1.0f / (2.0f * N);  // a power of two: exact

    // warps 0-3: add tile buffer pb's scaled int32 sums to row `warp * 32 + lane`'s fp32 sums
    auto epilogue = [&](int pb) {
        const int row = warp * 32 + lane;
        const float d = dlt[pb * kGemmM + row];
#pragma unroll
        for (int c = 0; c < NB; c += 16) {
            float v[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const float sum = FP8 ? v[i] : (float)__float_as_int(v[i]);  // fp32 (fp8) or s32 (int8) accumulator
                const float term = __fmul_rn(__fmul_rn(d, sxs[pb * NB + c + i]), sum);
                acc[(c + i) * kGemmM + row] = __fadd_rn(acc[(c + i) * kGemmM + row], __fmul_rn(term, kInv2N));
            }
        }
    };

    uint32_t parity = 0;
    bool fail = false, pending = false;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int ks = (int)(it % a.ksplit);
        const int64_t rb = (it / a.ksplit) % row_blocks, bb = it / (a.ksplit * row_blocks);
        const int64_t r0 = rb * kGemmM;
        const int b0 = (int)bb * NB;
        const int64_t j0 = (int64_t)ks * a.tiles_per_split;
        const int64_t j1 = j0 + a.tiles_per_split < a.tiles_per_row ? j0 + a.tiles_per_split : a.tiles_per_row;
        for (int e = tid; e < NB * kGemmM; e += kGemmThreads) acc[e] = 0.0f;
        for (int64_t j = j0; j < j1; j++) {
            const int pb = (int)((j - j0) & 1);
            if (pending) {  // the previous tile's MMAs are complete: A and B are free, its sums readable
                const bool ok = mbar_wait(bar, parity);
                parity ^= 1u;
                pending = false;
                if (__syncthreads_or(!ok)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                if (warp < 4) epilogue(pb ^ 1);
            }
            // A: rows r0 .. r0 + 127 of column tile j; lane l holds K bytes 16 l .. 16 l + 15 (chunk l)
            for (int m = gid; m < kGemmM; m += GPB) {
                const int64_t r = r0 + m;
                float pt[EPL];
                uint32_t sb = 0;
                bool bad = false;
                if (r < a.rows) {
                    bad = parse_tile<N, D, EPL, FIXED>(a.w, r * a.tiles_per_row + j, wbuf, mask, l, pt, sb);
                } else {
#pragma unroll
                    for (int i = 0; i < EPL; i++) pt[i] = 0.0f;
                }
                uint32_t wa[4] = { 0u, 0u, 0u, 0u };
                bool sat = false;
#pragma unroll
                for (int i = 0; i < EPL; i++) {
                    const float y2 = 2.0f * pt[i];  // exact: 2y is an integer
                    uint32_t b8;
                    if constexpr (FP8) {
                        sat |= fabsf(y2) > 448.0f;
                        b8 = e4m3_bits(y2);
                    } else {
                        int v2 = __float2int_rn(y2);
                        if (v2 > 127 || v2 < -127) {
                            sat = true;
                            v2 = v2 > 0 ? 127 : -127;
                        }
                        b8 = (uint32_t)v2 & 0xffu;
                    }
                    wa[i >> 2] |= b8 << (8 * (i & 3));
                }
                *reinterpret_cast<uint4 *>(sA + (uint32_t)((m & 7) + 8 * (m >> 3)) * 16u + (uint32_t)l * LBO_A) =
                    make_uint4(wa[0], wa[1], wa[2], wa[3]);
                if (l == 0) dlt[pb * kGemmM + m] = bf16_bits_to_float(sb);
                if (bad && l == 0 && a.status) atomicOr(a.status, kStatusCorrupt);
                if (__any_sync(mask, sat) && l == 0 && a.status) atomicOr(a.status, kStatusRange);
            }
            // B: Q rows b0 .. b0 + NB - 1 of tile j, and their scales
            for (int e = tid; e < NB * 16; e += kGemmThreads) {
                const int n = e % NB, kc = e / NB;
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.xq + (int64_t)(b0 + n) * a.cols + j * N + kc * 16));
                *reinterpret_cast<uint4 *>(sB + (uint32_t)((n & 7) + 8 * (n >> 3)) * 16u + (uint32_t)kc * LBO_B) = v;
            }
            for (int n = tid; n < NB; n += kGemmThreads) sxs[pb * NB + n] = a.sx[(int64_t)(b0 + n) * a.tiles_per_row + j];
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0 && j != a.stall_tile) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < N / 32; s++) {
                    const uint64_t ad = make_smem_desc(aA + 2u * s * LBO_A, LBO_A, 128u);
                    const uint64_t bd = make_smem_desc(aB + 2u * s * LBO_B, LBO_B, 128u);
                    if constexpr (FP8) umma_e4m3(tmem, ad, bd, IDESC, s > 0 ? 1u : 0u);
                    else umma_i8(tmem, ad, bd, IDESC, s > 0 ? 1u : 0u);
                }
                umma_commit(bar);
            }
            pending = true;
        }
        if (pending) {
            const bool ok = mbar_wait(bar, parity);
            parity ^= 1u;
            pending = false;
            if (__syncthreads_or(!ok)) fail = true;
            tc_fence_after();
            if (!fail && warp < 4) epilogue((int)((j1 - 1 - j0) & 1));
        }
        // warps 0-3 store the sums of their rows (the threads that accumulated them)
        if (warp < 4) {
            const int64_t r = r0 + warp * 32 + lane;
            for (int c = 0; c < NB; c++) {
                const int b = b0 + c;
                if (r < a.rows && b < a.batch) {
                    const float val = fail ? 0.0f : acc[c * kGemmM + warp * 32 + lane];
                    if (a.ksplit == 1) a.y[(int64_t)b * a.rows + r] = val;
                    else a.part[((int64_t)ks * a.batch_pad + b) * a.rows + r] = val;
                }
            }
        }
        tc_fence_before();
        __syncthreads();  // sums stored and the accumulator read before the next item
        tc_fence_after();
        if (fail) break;
    }
    if (fail && tid == 0 && a.status) atomicOr(a.status, kStatusTimeout);
    if (warp == 0) tmem_dealloc(tmem, NCOLS);
}

// ------------------------------------------------------------------ launch
int gemm_block_batch(int64_t batch)
{
    return batch <= 16 ? 16 : batch <= 32 ? 32 : batch <= 64 ? 64 : batch <= 128 ? 128 : 256;
}

// Column splits: enough work items for about three waves of resident
// blocks (blocks_per_sm per SM), so the last wave is nearly full.  The count
// never grows when blocks_per_sm shrinks; two (the register limit of 512
// threads x 64 registers) bounds the workspace.
void gemm_plan(int64_t rows, int64_t cols, int64_t batch, int blocks_per_sm, GemmPlan *p)
{
    p->nb = gemm_block_batch(batch);
    p->batch_pad = (int)(((batch + p->nb - 1) / p->nb) * p->nb);
    const int64_t tpr = cols / kGemmN;
    const int64_t blocks = ((rows + kGemmM - 1) / kGemmM) * (p->batch_pad / p->nb);
    const int64_t slots = 3 * (int64_t)sm_count() * (blocks_per_sm > 0 ? blocks_per_sm : 1);
    int64_t ks = (slots + blocks - 1) / (blocks > 0 ? blocks : 1);
    if (ks > tpr) ks = tpr;
    if (ks < 1) ks = 1;
    int64_t tps = (tpr + ks - 1) / ks;
    if (tps < 1) tps = 1;
    p->tiles_per_split = (int)tps;
    p->ksplit = (int)(tpr > 0 ? (tpr + tps - 1) / tps : 1);
    p->xt_bytes = (uint64_t)p->batch_pad * (uint64_t)cols * 2;
    p->part_bytes = p->ksplit > 1 ? (uint64_t)p->ksplit * (uint64_t)p->batch_pad * (uint64_t)rows * 4 : 0;
}

void gemm_plan_i8(int64_t rows, int64_t cols, int64_t batch, int blocks_per_sm, GemmPlan *p)
{
    gemm_plan(rows, cols, batch < 128 ? batch : 128, blocks_per_sm, p);  // splits for one batch block of <= 128
    p->batch_pad = (int)(((batch + p->nb - 1) / p->nb) * p->nb);
    const int64_t tpr = cols / kGemmN;
    const uint64_t q_bytes = ((uint64_t)p->batch_pad * (uint64_t)cols + 255) / 256 * 256;
    p->xt_bytes = q_bytes + (uint64_t)p->batch_pad * (uint64_t)tpr * 4;
    p->part_bytes = p->ksplit > 1 ? (uint64_t)p->ksplit * (uint64_t)p->batch_pad * (uint64_t)rows * 4 : 0;
}

namespace {

template <int D, int NB>
cudaError_t launch_gemm_t(GemmArgs a, cudaStream_t s)
{
    const size_t smem = gemm_operand_bytes(kGemmM) + gemm_operand_bytes(NB) +
                        (size_t)kGemmWarps * 2 * group_words(a.w.wmax) * 4;
    auto kern = a.w.slot ? gemm_tc_kernel<D, NB, true> : gemm_tc_kernel<D, NB, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // Resident blocks per SM: the register limit of 512 threads x 64
    // registers is two; shared memory may allow fewer.  (Computed from the
    // device limits: the occupancy query reported one block where two are
    // resident.)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    int dev = 0, smem_sm = 0, reserved = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
    int per_sm = (int)((size_t)smem_sm / (smem + 256 + (size_t)reserved));
    if (per_sm > 2) per_sm = 2;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    GemmPlan p{};
    gemm_plan(a.rows, a.cols, a.batch, per_sm, &p);  // never more splits than the workspace holds
    a.ksplit = p.ksplit;
    a.tiles_per_split = p.tiles_per_split;
    // one block per work item (measured faster than a persistent grid here)
    const int64_t items = ((a.rows + kGemmM - 1) / kGemmM) * (a.batch_pad / NB) * a.ksplit;
    if (items >= ((int64_t)1 << 31)) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)(items > 0 ? items : 1), kGemmThreads, smem, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.ksplit == 1) return e;
    int64_t n = (int64_t)a.batch * a.rows, blocks = (n + 255) / 256;
    if (blocks > 8 * (int64_t)sm_count()) blocks = 8 * (int64_t)sm_count();
    splitk_reduce_kernel<<<(unsigned)(blocks > 0 ? blocks : 1), 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_gemm_d(const GemmArgs &a, cudaStream_t s)
{
    switch (a.nb) {
    case 16: return launch_gemm_t<D, 16>(a, s);
    case 32: return launch_gemm_t<D, 32>(a, s);
    case 64: return launch_gemm_t<D, 64>(a, s);
    case 128: return launch_gemm_t<D, 128>(a, s);
    default: return launch_gemm_t<D, 256>(a, s);
    }
}

}  // namespace

cudaError_t launch_gemm(int lattice, const GemmArgs &a, cudaStream_t s)
{
    const int64_t xtiles = (int64_t)a.batch_pad * a.tiles_per_row;
    int64_t rb = (xtiles + 15) / 16;
    if (rb > 4 * (int64_t)sm_count()) rb = 4 * (int64_t)sm_count();
    rotate_x_kernel<<<(unsigned)(rb > 0 ? rb : 1), 256, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (lattice) {
    case 1: return launch_gemm_d<1>(a, s);
    case 2: return launch_gemm_d<2>(a, s);
    case 4: return launch_gemm_d<4>(a, s);
    default: return launch_gemm_d<8>(a, s);
    }
}

namespace {

template <int D, int NB, bool FP8>
cudaError_t launch_gemm_i8_t(GemmArgs a, cudaStream_t s)
{
    const size_t smem = gemm_operand_bytes_i8(kGemmM) + gemm_operand_bytes_i8(NB) +
                        ((size_t)NB * kGemmM + 2 * kGemmM + 2 * NB) * 4 +
                        (size_t)kGemmWarps * 2 * group_words(a.w.wmax) * 4;
    auto kern = a.w.slot ? gemm_i8_kernel<D, NB, true, FP8> : gemm_i8_kernel<D, NB, false, FP8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    int dev = 0, smem_sm = 0, reserved = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
    int per_sm = (int)((size_t)smem_sm / (smem + 256 + (size_t)reserved));
    if (per_sm > 2) per_sm = 2;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    GemmPlan p{};
    gemm_plan_i8(a.rows, a.cols, a.batch, per_sm, &p);  // never more splits than the workspace holds
    a.ksplit = p.ksplit;
    a.tiles_per_split = p.tiles_per_split;
    const int64_t items = ((a.rows + kGemmM - 1) / kGemmM) * (a.batch_pad / NB) * a.ksplit;
    if (items >= ((int64_t)1 << 31)) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)(items > 0 ? items : 1), kGemmThreads, smem, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.ksplit == 1) return e;
    int64_t n = (int64_t)a.batch * a.rows, blocks = (n + 255) / 256;
    if (blocks > 8 * (int64_t)sm_count()) blocks = 8 * (int64_t)sm_count();
    splitk_reduce_kernel<<<(unsigned)(blocks > 0 ? blocks : 1), 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D, bool FP8>
cudaError_t launch_gemm_i8_d(const GemmArgs &a, cudaStream_t s)
{
    switch (a.nb) {
    case 16: return launch_gemm_i8_t<D, 16, FP8>(a, s);
    case 32: return launch_gemm_i8_t<D, 32, FP8>(a, s);
    case 64: return launch_gemm_i8_t<D, 64, FP8>(a, s);
    default: return launch_gemm_i8_t<D, 128, FP8>(a, s);
    }
}

template <bool FP8>
cudaError_t launch_lowbit(int lattice, const GemmArgs &a, cudaStream_t s)
{
    const int64_t xtiles = (int64_t)a.batch_pad * a.tiles_per_row;
    int64_t rb = (xtiles + 15) / 16;
    if (rb > 4 * (int64_t)sm_count()) rb = 4 * (int64_t)sm_count();
    rotate_quant_x_kernel<FP8><<<(unsigned)(rb > 0 ? rb : 1), 256, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (lattice) {
    case 1: return launch_gemm_i8_d<1, FP8>(a, s);
    case 4: return launch_gemm_i8_d<4, FP8>(a, s);
    default: return launch_gemm_i8_d<8, FP8>(a, s);  // A2 has no integer form: refused by the host API
    }
}

}  // namespace

cudaError_t launch_gemm_i8(int lattice, const GemmArgs &a, cudaStream_t s) { return launch_lowbit<false>(lattice, a, s); }

cudaError_t launch_gemm_e4m3(int lattice, const GemmArgs &a, cudaStream_t s) { return launch_lowbit<true>(lattice, a, s); }

}  // namespace hq
