// hq_internal.h -- argument blocks and launchers shared by the host API and
// the kernel translation units (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "hq_device.cuh"

namespace hq {

constexpr int kStatusNonfinite = 1, kStatusCapacity = 2, kStatusCorrupt = 4, kStatusTimeout = 8, kStatusRange = 16;

// Look-back slot: bits 62..63 flag (1 = chunk aggregate, 2 = inclusive
// prefix, 3 = poisoned: the chunk gave up waiting, so no prefix from it on is
// valid), bits 0..61 the word count.
constexpr uint64_t kFlagAggregate = 1ull << 62, kFlagInclusive = 2ull << 62, kFlagPoison = 3ull << 62;
constexpr uint64_t kValueMask = (1ull << 62) - 1;
constexpr uint32_t kSpinLimit = 1u << 24;          // polls before a wait gives up ...
constexpr uint64_t kWaitLimitNs = 500ull * 1000000;  // ... or 0.5 s of waiting, whichever first

// Nanoseconds of the GPU's global timer (bounds every wait).
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

struct EncodeArgs {
    const void *x;
    int64_t ntiles;
    int64_t tiles_per_row;
    float c;
    A2Consts a2;
    uint64_t sign_key;    // hash key of tag 1 (signs)
    uint64_t dither_key;  // hash key of tag 2 (dither)
    uint32_t *payload;
    uint64_t cap;
    uint32_t *off;
    uint16_t *scale;
    uint8_t *kk;
    uint32_t *ticket;
    unsigned long long *lb;
    int32_t *status;
    uint32_t wmax;        // worst-case words of one tile
    uint32_t nchunks;
    int tiles_per_group;  // G: consecutive tiles each lane group encodes per chunk
    int sign_words;       // sign words cached per block (0: hash them per tile)
    int k_hint;           // the rate's typical Rice parameter (search start)
    FastDiv tpr_div;      // division by tiles_per_row
    uint32_t stall_chunk; // test hook: this chunk never publishes its prefix (0xffffffff: none)
    uint32_t slot_words;  // fixed-rate encode: words per tile slot (kk then holds packed 4-bit k)
};

struct DecodeArgs {
    const uint32_t *payload;
    uint64_t cap;
    const uint32_t *off;
    const uint16_t *scale;
    const uint8_t *kk;
    int64_t ntiles;
    int64_t tiles_per_row;
    A2Consts a2;
    uint64_t sign_key;
    uint64_t dither_key;
    int32_t *status;
    uint32_t wmax;
    void *y;              // decode output
    const void *x;        // gemv input (bf16)
    float *gy;            // gemv output
    int64_t rows;
    int sign_words;       // sign words cached per block (0: hash them per tile)
    FastDiv tpr_div;      // division by tiles_per_row
    uint32_t slot;        // fixed-rate stream: words per tile slot, tile t at t * slot, k packed
                          // two per byte (0: variable rate, offsets from off[], one k per byte)
};

// Batch-1 attention over K and V codec streams (one tile per cached vector).
struct AttnArgs {
    DecodeArgs k, v;        // rows = heads * tokens, one tile of head_dim per row
    const uint16_t *q;      // bf16 [heads * group][head_dim]
    float *out;             // fp32 [heads * group][head_dim]
    float *part;            // [heads * group][splits][head_dim + 2] partial results
    uint32_t *counter;      // [heads][query chunks] finished splits, zero at launch
    int64_t heads, tokens;
    int group;              // query heads per KV head
    int splits, tokens_per_split;
    float scale;
    int32_t *status;
};

// Batched decode + matrix product (tile 256): Y = X W_hat^T.
struct GemmArgs {
    DecodeArgs w;               // weight stream, rows x cols
    const uint16_t *x;          // bf16 [batch][cols]
    uint16_t *xt;               // bf16 [batch_pad][cols]: rotated activations (workspace)
    int8_t *xq;                 // 8-bit products: quantized rotated activations [batch_pad][cols]
                                // (int8, or E4M3 bits for the fp8 variant; workspace)
    float *sx;                  // 8-bit products: their scales [batch_pad][tiles_per_row] (workspace)
    float *y;                   // fp32 [batch][rows]
    float *part;                // fp32 [ksplit][batch_pad][rows] split-K partials (workspace)
    int64_t rows, cols, tiles_per_row;
    int batch, batch_pad, nb;   // nb: batch rows per block (16, 32, 64, 128 or 256)
    int ksplit, tiles_per_split;
    uint64_t sign_key;
    int32_t *status;
    int64_t stall_tile;         // test hook: this column tile never commits its MMAs (-1: none)
};

struct GemmPlan {
    int nb, batch_pad, ksplit, tiles_per_split;
    uint64_t xt_bytes, part_bytes;  // workspace: X~ (int8 product: Q, then the scales), then the partials
};

// Launch helpers; return a cudaError_t.
cudaError_t launch_encode(int tile, int lattice, bool dither, int dtype, const EncodeArgs &a,
                          cudaStream_t s);
cudaError_t launch_encode_fixed(int tile, int lattice, bool dither, int dtype, const EncodeArgs &a,
                                cudaStream_t s);
cudaError_t launch_decode(int tile, int lattice, bool dither, int dtype, const DecodeArgs &a,
                          cudaStream_t s);
cudaError_t launch_gemv(int tile, int lattice, const DecodeArgs &a, int64_t cols, cudaStream_t s);
cudaError_t launch_gemm(int lattice, const GemmArgs &a, cudaStream_t s);
// Plan for blocks_per_sm resident blocks; the launch re-plans from the
// kernel's occupancy (never more splits than for two blocks per SM).
void gemm_plan(int64_t rows, int64_t cols, int64_t batch, int blocks_per_sm, GemmPlan *p);
// The 8-bit products (int8 or E4M3 operands); see gemm_plan_i8 in hq_gemm.cu.
void gemm_plan_i8(int64_t rows, int64_t cols, int64_t batch, int blocks_per_sm, GemmPlan *p);
cudaError_t launch_gemm_i8(int lattice, const GemmArgs &a, cudaStream_t s);
// The fp8 variant: A = e4m3(2y), activations in E4M3 scaled to +-448 (same workspace).
cudaError_t launch_gemm_e4m3(int lattice, const GemmArgs &a, cudaStream_t s);
// Rate accounting of a stream: counts[8] and hist[2][bins] (device, added to).
cudaError_t launch_stats(int tile, int lattice, const DecodeArgs &a, uint64_t *counts, uint64_t *hist, int bins,
                         cudaStream_t s);
// Fills a.splits / a.tokens_per_split from the kernel's occupancy, then launches.
cudaError_t launch_attention(int head_dim, int lattice, AttnArgs a, cudaStream_t s);

// Query heads one attention block serves (1, 2, 4 or 8), and the token
// splits for `blocks_per_sm` resident blocks (every split non-empty; never
// more splits for fewer resident blocks).
int attention_queries_per_block(int group);
void attention_splits(int64_t heads, int64_t tokens, int group, int blocks_per_sm, int *splits,
                      int *tokens_per_split);

// Smallest encode chunk (tiles) for a tile length; sizes the workspace.
int encode_chunk_tiles(int tile);
// Tiles per lane group per chunk for a tile length, worst-case tile words and
// the call's tile count (small calls get small chunks to spread over the GPU).
int encode_tiles_per_group(int tile, uint32_t wmax, int64_t ntiles);
int sm_count();

}  // namespace hq
