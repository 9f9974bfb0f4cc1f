// hq_api.cu -- host side of the C ABI declared in include/hq.h: argument
// validation, sizing rules, hash keys and kernel dispatch.  No allocation,
// no synchronisation; everything is enqueued on the caller's stream.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_internal.h"

namespace hq {

int sm_count()
{
    static std::atomic<int> cached[64];  // zero-initialised; a race only stores the same value twice
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

}  // namespace hq

namespace {

using namespace hq;

bool valid_tile(int tile) { return tile == 64 || tile == 128 || tile == 256 || tile == 512 || tile == 1024; }
bool valid_lattice(int d) { return d == HQ_Z || d == HQ_A2 || d == HQ_D4 || d == HQ_E8; }
bool valid_bps(float b) { return std::isfinite(b) && b > 0.0f && b <= 8.0f; }
bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

double cell_volume(int lattice)
{
    switch (lattice) {
    case HQ_E8: return 1.0;
    case HQ_D4: return 2.0;
    case HQ_A2: return std::sqrt(3.0) / 2.0;
    default: return 1.0;
    }
}

float rate_constant(int lattice, float bps)
{
    const double c = std::sqrt(2.0 * M_PI * M_E) * std::pow(2.0, -(double)bps) *
                     std::pow(cell_volume(lattice), -1.0 / (double)lattice);
    return (float)c;
}

// Largest zigzag symbol a tile can produce, from |v_i| <= sqrt(n sum w^2):
// |x_i| <= sqrt(n) / c (1 + 2^-7) covering the rounding of S, sqrt, c and
// bf16(Delta); dither adds at most 1 per coordinate, each coset's rounding
// moves a coordinate at most 1.5, so |z| <= X + 2.5 and u <= 2 |z|.
uint32_t tile_bound_words(int tile, int lattice, float bps)
{
    const double c = (double)rate_constant(lattice, bps);
    const double X = std::sqrt((double)tile) / c * (1.0 + 1.0 / 128.0) + 3.0;
    const uint64_t umax = 2ull * (uint64_t)std::ceil(X);
    int kb = 0;
    while (kb < 63 && (umax >> kb) != 0) ++kb;
    const int k = kb < 15 ? kb : 15;
    const uint64_t coset = (lattice == HQ_E8 || lattice == HQ_A2) ? (uint64_t)(tile / lattice) : 0;
    const uint64_t bits = coset + (uint64_t)tile * (1 + k) + (uint64_t)tile * (umax >> k);
    return (uint32_t)((bits + 31) / 32);
}

// Where the Rice search starts: Delta puts every tile's coordinates at RMS
// about 1/c, so the optimal k sits near log2(1/c) for all tiles of a call.
int rice_hint(float c)
{
    const double k = std::floor(std::log2(1.0 / (double)c) + 0.5);
    return k < 0 ? 0 : (k > 15 ? 15 : (int)k);
}

A2Consts a2_consts() { return A2Consts{ (float)std::sqrt(3.0), (float)(1.0 / std::sqrt(3.0)) }; }

int check_stream(const hq_stream *s, int64_t ntiles, bool need_payload)
{
    if (!s) return HQ_ERR_ARG;
    if (!s->slot_words && !s->tile_off) return HQ_ERR_ARG;  // fixed-rate streams keep no offsets
    if (ntiles > 0 && (!s->tile_scale || !s->tile_k || (need_payload && !s->payload))) return HQ_ERR_ARG;
    return HQ_OK;
}

// Fixed-rate slots.  The smallest holds the all-zero tile (coset bits and n
// one bits); the largest allowed is 8 bits per coordinate.
uint32_t min_slot_words(int tile, int lattice)
{
    const uint32_t coset = (lattice == HQ_E8 || lattice == HQ_A2) ? (uint32_t)(tile / lattice) : 0u;
    return (coset + (uint32_t)tile + 31u) / 32u;
}

bool valid_slot(int tile, int lattice, uint32_t slot)
{
    return slot >= min_slot_words(tile, lattice) && slot <= (uint32_t)tile / 4u;
}

// Start of the fixed-rate scale search: the closed-form rule at the slot's
// payload rate less 5/32 bit (about what the Rice code and the coset bits
// spend over the rule's entropy on Gaussian tiles), at most 8 bits.
float fixed_start_rate(int tile, uint32_t slot)
{
    const double r = 32.0 * (double)slot / (double)tile - 0.15625;
    return (float)(r < 8.0 ? r : 8.0);
}

// Fixed-rate stream of `ntiles` tiles: slot legal, every slot inside the
// payload, offsets t * slot within 32 bits.
int check_fixed_stream(const hq_stream *s, int64_t ntiles, int tile, int lattice)
{
    if (!valid_slot(tile, lattice, s->slot_words)) return HQ_ERR_ARG;
    const uint64_t need = (uint64_t)ntiles * s->slot_words;
    if (need >= (1ull << 32)) return HQ_ERR_UNSUPPORTED;
    if (s->payload_capacity_words < need) return HQ_ERR_CAPACITY;
    return HQ_OK;
}

int common_shape(int64_t rows, int64_t cols, int tile, int lattice, float bps, int64_t *ntiles)
{
    if (rows < 0 || cols < 0 || !valid_tile(tile) || !valid_lattice(lattice) || !valid_bps(bps)) return HQ_ERR_ARG;
    if (cols % tile) return HQ_ERR_ARG;
    const int64_t tpr = cols / tile;
    if (tpr && rows > (int64_t)(INT64_MAX / 2) / tpr) return HQ_ERR_UNSUPPORTED;
    *ntiles = rows * tpr;
    if (*ntiles >= (int64_t)1 << 32 || tpr >= (int64_t)1 << 32) return HQ_ERR_UNSUPPORTED;
    return HQ_OK;
}

int64_t nchunks_for(int64_t ntiles, int tile)
{
    const int T = encode_chunk_tiles(tile);
    return (ntiles + T - 1) / T;
}

int encode_impl(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                uint64_t seed, const hq_stream *out, void *workspace, uint64_t workspace_bytes,
                void *stream, int32_t *d_status, bool dither, uint32_t stall_chunk = 0xffffffffu)
{
    int64_t ntiles = 0;
    int rc = common_shape(rows, cols, tile, lattice, bps, &ntiles);
    if (rc) return rc;
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if ((rc = check_stream(out, ntiles, true))) return rc;
    if (out->slot_words) return HQ_ERR_ARG;  // a fixed-rate stream: hq_encode_fixed
    cudaStream_t s = (cudaStream_t)stream;
    if (ntiles == 0) return cudaMemsetAsync(out->tile_off, 0, sizeof(uint32_t), s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
    if (!x || !aligned(x, 16)) return HQ_ERR_ARG;
    const uint32_t wmax = tile_bound_words(tile, lattice, bps);
    const uint64_t need = (uint64_t)ntiles * wmax;
    if (need >= (1ull << 32)) return HQ_ERR_UNSUPPORTED;
    if (out->payload_capacity_words < need) return HQ_ERR_CAPACITY;
    const int G = encode_tiles_per_group(tile, wmax, ntiles);
    const int64_t chunk_tiles = (int64_t)encode_chunk_tiles(tile) * G;
    const int64_t nchunks = (ntiles + chunk_tiles - 1) / chunk_tiles;
    const uint64_t ws_need = 256 + 8 * (uint64_t)nchunks;
    if (!workspace || !aligned(workspace, 8) || workspace_bytes < ws_need) return HQ_ERR_WORKSPACE;
    if (nchunks >= (int64_t)1 << 31) return HQ_ERR_UNSUPPORTED;

    if (cudaMemsetAsync(workspace, 0, ws_need, s) != cudaSuccess) return HQ_ERR_CUDA;
    EncodeArgs a{};
    a.x = x;
    a.ntiles = ntiles;
    a.tiles_per_row = cols / tile;
    a.c = rate_constant(lattice, bps);
    a.a2 = a2_consts();
    a.sign_key = hash_key(seed, 1);
    a.dither_key = hash_key(seed, 2);
    a.payload = out->payload;
    a.cap = out->payload_capacity_words;
    a.off = out->tile_off;
    a.scale = out->tile_scale;
    a.kk = out->tile_k;
    a.ticket = static_cast<uint32_t *>(workspace);
    a.lb = reinterpret_cast<unsigned long long *>(static_cast<char *>(workspace) + 256);
    a.status = d_status;
    a.wmax = wmax;
    a.nchunks = (uint32_t)nchunks;
    a.tiles_per_group = G;
    const int64_t sign_words = (cols / tile) * (tile >= 64 ? tile / 64 : 1);
    a.sign_words = sign_words <= 2048 ? (int)sign_words : 0;
    a.k_hint = rice_hint(a.c);
    a.tpr_div = make_fastdiv((uint32_t)(cols / tile));
    a.stall_chunk = stall_chunk;
    return launch_encode(tile, lattice, dither, dtype, a, s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

int encode_fixed_impl(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice, uint64_t seed,
                      const hq_stream *out, void *stream, int32_t *d_status, bool dither)
{
    int64_t ntiles = 0;
    int rc = common_shape(rows, cols, tile, lattice, 1.0f, &ntiles);
    if (rc) return rc;
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (!out || !out->slot_words) return HQ_ERR_ARG;
    if ((rc = check_stream(out, ntiles, true))) return rc;
    if ((rc = check_fixed_stream(out, ntiles, tile, lattice))) return rc;
    if (ntiles == 0) return HQ_OK;
    if (!x || !aligned(x, 16)) return HQ_ERR_ARG;
    EncodeArgs a{};
    a.x = x;
    a.ntiles = ntiles;
    a.tiles_per_row = cols / tile;
    a.c = rate_constant(lattice, fixed_start_rate(tile, out->slot_words));
    a.a2 = a2_consts();
    a.sign_key = hash_key(seed, 1);
    a.dither_key = hash_key(seed, 2);
    a.payload = out->payload;
    a.cap = out->payload_capacity_words;
    a.scale = out->tile_scale;
    a.kk = out->tile_k;
    a.status = d_status;
    a.wmax = out->slot_words;
    const int64_t sign_words = (cols / tile) * (tile >= 64 ? tile / 64 : 1);
    a.sign_words = sign_words <= 2048 ? (int)sign_words : 0;
    a.k_hint = rice_hint(a.c);
    a.tpr_div = make_fastdiv((uint32_t)(cols / tile));
    a.stall_chunk = 0xffffffffu;
    a.slot_words = out->slot_words;
    return launch_encode_fixed(tile, lattice, dither, dtype, a, (cudaStream_t)stream) == cudaSuccess ? HQ_OK
                                                                                                     : HQ_ERR_CUDA;
}

int decode_common(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                  uint64_t seed, DecodeArgs &a, int64_t *ntiles)
{
    int rc = common_shape(rows, cols, tile, lattice, bps, ntiles);
    if (rc) return rc;
    if ((rc = check_stream(in, *ntiles, true))) return rc;
    if (in->slot_words && (rc = check_fixed_stream(in, *ntiles, tile, lattice))) return rc;
    a.payload = in->payload;
    a.cap = in->payload_capacity_words;
    a.off = in->tile_off;
    a.scale = in->tile_scale;
    a.kk = in->tile_k;
    a.ntiles = *ntiles;
    a.tiles_per_row = tile ? cols / tile : 0;
    a.a2 = a2_consts();
    a.sign_key = hash_key(seed, 1);
    a.dither_key = hash_key(seed, 2);
    a.wmax = in->slot_words ? in->slot_words : tile_bound_words(tile, lattice, bps);
    a.slot = in->slot_words;
    a.rows = rows;
    const int64_t sign_words = (cols / tile) * (tile >= 64 ? tile / 64 : 1);
    a.sign_words = sign_words <= 2048 ? (int)sign_words : 0;
    a.tpr_div = make_fastdiv((uint32_t)(tile ? cols / tile : 1));
    return HQ_OK;
}

int decode_impl(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                uint64_t seed, void *y, int dtype, void *stream, int32_t *d_status, bool dither)
{
    DecodeArgs a{};
    int64_t ntiles = 0;
    int rc = decode_common(in, rows, cols, tile, lattice, bps, seed, a, &ntiles);
    if (rc) return rc;
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (ntiles == 0) return HQ_OK;
    if (!y || !aligned(y, 16)) return HQ_ERR_ARG;
    a.y = y;
    a.status = d_status;
    return launch_decode(tile, lattice, dither, dtype, a, (cudaStream_t)stream) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

bool valid_head_dim(int d) { return d == 64 || d == 128 || d == 256; }

// Workspace of an attention call: counters, then the per-split partials.
struct AttnWorkspace {
    int splits, tokens_per_split;
    uint64_t counter_bytes, total_bytes;
};

AttnWorkspace attention_workspace(int64_t heads, int64_t tokens, int head_dim, int group)
{
    AttnWorkspace w{};
    attention_splits(heads, tokens, group, 8, &w.splits, &w.tokens_per_split);  // the largest split count
    const int gb = attention_queries_per_block(group);
    const uint64_t counters = (uint64_t)heads * (uint64_t)((group + gb - 1) / gb);
    w.counter_bytes = (counters * 4 + 255) / 256 * 256;
    w.total_bytes = w.counter_bytes + (uint64_t)heads * (uint64_t)group * (uint64_t)w.splits *
                                          (uint64_t)(head_dim + 2) * 4;
    return w;
}

}  // namespace

extern "C" {

const char *hq_error_string(int code)
{
    switch (code) {
    case HQ_OK: return "ok";
    case HQ_ERR_ARG: return "invalid argument";
    case HQ_ERR_UNSUPPORTED: return "unsupported size or configuration";
    case HQ_ERR_CAPACITY: return "payload capacity below the worst-case bound";
    case HQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case HQ_ERR_CUDA: return "CUDA call or kernel launch failed";
    case HQ_ERR_FORMAT: return "not a valid, intact checkpoint container";
    default: return "unknown error";
    }
}

int hq_version(void) { return 100; }

int hq_rate_constant(int lattice, float bps, float *out)
{
    if (!out || !valid_lattice(lattice) || !valid_bps(bps)) return HQ_ERR_ARG;
    *out = rate_constant(lattice, bps);
    return HQ_OK;
}

int hq_tile_bound_words(int tile, int lattice, float bps, uint32_t *out)
{
    if (!out || !valid_tile(tile) || !valid_lattice(lattice) || !valid_bps(bps)) return HQ_ERR_ARG;
    *out = tile_bound_words(tile, lattice, bps);
    return HQ_OK;
}

int hq_max_payload_words(int64_t rows, int64_t cols, int tile, int lattice, float bps, uint64_t *out)
{
    int64_t ntiles = 0;
    if (!out) return HQ_ERR_ARG;
    int rc = common_shape(rows, cols, tile, lattice, bps, &ntiles);
    if (rc) return rc;
    const uint64_t w = (uint64_t)ntiles * tile_bound_words(tile, lattice, bps);
    if (w >= (1ull << 32)) return HQ_ERR_UNSUPPORTED;
    *out = w;
    return HQ_OK;
}

int hq_min_slot_words(int tile, int lattice, uint32_t *out)
{
    if (!out || !valid_tile(tile) || !valid_lattice(lattice)) return HQ_ERR_ARG;
    *out = min_slot_words(tile, lattice);
    return HQ_OK;
}

int hq_fixed_slot_words(int tile, int lattice, float bps, uint32_t *out)
{
    if (!out || !valid_tile(tile) || !valid_lattice(lattice) || !valid_bps(bps)) return HQ_ERR_ARG;
    const double s = std::floor(((double)bps * (double)tile - 20.0) / 32.0);
    if (s < (double)min_slot_words(tile, lattice)) return HQ_ERR_ARG;
    *out = (uint32_t)s;
    return HQ_OK;
}

int hq_encode_fixed(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice, uint64_t seed,
                    const hq_stream *out, void *stream, int32_t *d_status)
{
    return encode_fixed_impl(x, dtype, rows, cols, tile, lattice, seed, out, stream, d_status, false);
}

int hq_kv_encode_fixed(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice, uint64_t seed,
                       const hq_stream *out, void *stream, int32_t *d_status)
{
    return encode_fixed_impl(x, dtype, rows, cols, tile, lattice, seed, out, stream, d_status, true);
}

int hq_encode_workspace_bytes(int64_t rows, int64_t cols, int tile, uint64_t *out)
{
    if (!out || rows < 0 || cols < 0 || !valid_tile(tile) || cols % tile) return HQ_ERR_ARG;
    const int64_t tpr = cols / tile;
    if (tpr && rows > (int64_t)(INT64_MAX / 2) / tpr) return HQ_ERR_UNSUPPORTED;  // rows * tpr would overflow
    const int64_t ntiles = rows * tpr;
    *out = 256 + 8 * (uint64_t)nchunks_for(ntiles, tile);
    return HQ_OK;
}

int hq_encode(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice, float bps,
              uint64_t seed, const hq_stream *out, void *workspace, uint64_t workspace_bytes, void *stream,
              int32_t *d_status)
{
    return encode_impl(x, dtype, rows, cols, tile, lattice, bps, seed, out, workspace, workspace_bytes, stream,
                       d_status, false);
}

int hq_kv_encode(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                 uint64_t seed, const hq_stream *out, void *workspace, uint64_t workspace_bytes, void *stream,
                 int32_t *d_status)
{
    return encode_impl(x, dtype, rows, cols, tile, lattice, bps, seed, out, workspace, workspace_bytes, stream,
                       d_status, true);
}

int hq_test_encode_stalled(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                           uint64_t seed, const hq_stream *out, void *workspace, uint64_t workspace_bytes,
                           void *stream, int32_t *d_status, uint32_t stalled_chunk)
{
    return encode_impl(x, dtype, rows, cols, tile, lattice, bps, seed, out, workspace, workspace_bytes, stream,
                       d_status, false, stalled_chunk);
}

int hq_decode(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice, float bps, uint64_t seed,
              void *y, int dtype, void *stream, int32_t *d_status)
{
    return decode_impl(in, rows, cols, tile, lattice, bps, seed, y, dtype, stream, d_status, false);
}

int hq_kv_decode(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                 uint64_t seed, void *y, int dtype, void *stream, int32_t *d_status)
{
    return decode_impl(in, rows, cols, tile, lattice, bps, seed, y, dtype, stream, d_status, true);
}

int hq_stream_stats(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                    uint64_t *counts, uint64_t *hist, int bins, void *stream, int32_t *d_status)
{
    DecodeArgs a{};
    int64_t ntiles = 0;
    int rc = decode_common(in, rows, cols, tile, lattice, bps, 0, a, &ntiles);
    if (rc) return rc;
    if (!counts || !hist || bins < 2 || bins > 4096 || !aligned(counts, 8) || !aligned(hist, 8)) return HQ_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(counts, 0, 8 * sizeof(uint64_t), s) != cudaSuccess ||
        cudaMemsetAsync(hist, 0, 2 * (size_t)bins * sizeof(uint64_t), s) != cudaSuccess)
        return HQ_ERR_CUDA;
    if (ntiles == 0) return HQ_OK;
    a.status = d_status;
    return launch_stats(tile, lattice, a, counts, hist, bins, s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

int hq_decode_gemv(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                   uint64_t seed, const void *x, float *y, void *stream, int32_t *d_status)
{
    DecodeArgs a{};
    int64_t ntiles = 0;
    int rc = decode_common(w, rows, cols, tile, lattice, bps, seed, a, &ntiles);
    if (rc) return rc;
    if (cols > 40960) return HQ_ERR_UNSUPPORTED;
    if (rows > 0 && !y) return HQ_ERR_ARG;
    if (ntiles == 0) {
        if (rows > 0)
            return cudaMemsetAsync(y, 0, sizeof(float) * (size_t)rows, (cudaStream_t)stream) == cudaSuccess
                       ? HQ_OK : HQ_ERR_CUDA;
        return HQ_OK;
    }
    if (!x || !aligned(x, 16)) return HQ_ERR_ARG;
    a.x = x;
    a.gy = y;
    a.status = d_status;
    return launch_gemv(tile, lattice, a, cols, (cudaStream_t)stream) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

int hq_decode_gemm_workspace_bytes(int64_t rows, int64_t cols, int64_t batch, uint64_t *out)
{
    if (!out || rows < 0 || cols < 0 || batch < 0 || cols % 256) return HQ_ERR_ARG;
    if (batch > (int64_t)1 << 24) return HQ_ERR_UNSUPPORTED;
    GemmPlan p{};
    gemm_plan(rows, cols, batch, 2, &p);  // the most splits any launch picks
    *out = (p.xt_bytes + 255) / 256 * 256 + p.part_bytes;
    return HQ_OK;
}

}  // extern "C"

namespace {

int decode_gemm_impl(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                     uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                     uint64_t workspace_bytes, void *stream, int32_t *d_status, int64_t stall_tile,
                     int lowbit = 0)  // 0: bf16 operands, 1: int8, 2: fp8 (E4M3)
{
    GemmArgs a{};
    int64_t ntiles = 0;
    int rc = decode_common(w, rows, cols, tile, lattice, bps, seed, a.w, &ntiles);
    if (rc) return rc;
    if (tile != 256) return HQ_ERR_UNSUPPORTED;
    const bool int8 = lowbit != 0;  // both 8-bit products share the workspace layout and plan
    if (int8 && lattice == HQ_A2) return HQ_ERR_UNSUPPORTED;  // A2 points have no integer form
    if (batch < 0) return HQ_ERR_ARG;
    if (batch > (int64_t)1 << 24) return HQ_ERR_UNSUPPORTED;
    if (batch == 0 || rows == 0) return HQ_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (!y || !aligned(y, 4)) return HQ_ERR_ARG;
    if (cols == 0)
        return cudaMemsetAsync(y, 0, sizeof(float) * (size_t)(batch * rows), s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
    if (!x || !aligned(x, 16)) return HQ_ERR_ARG;
    GemmPlan p{};
    if (int8) gemm_plan_i8(rows, cols, batch, 2, &p);  // workspace bound; the launch re-plans
    else gemm_plan(rows, cols, batch, 2, &p);
    const uint64_t xt_span = (p.xt_bytes + 255) / 256 * 256;
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < xt_span + p.part_bytes) return HQ_ERR_WORKSPACE;
    a.x = static_cast<const uint16_t *>(x);
    a.xt = static_cast<uint16_t *>(workspace);
    if (int8) {  // Q (batch_pad x cols int8, 256-byte rounded), then the scales
        a.xq = static_cast<int8_t *>(workspace);
        a.sx = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                         ((uint64_t)p.batch_pad * (uint64_t)cols + 255) / 256 * 256);
    }
    a.y = y;
    a.part = reinterpret_cast<float *>(static_cast<char *>(workspace) + xt_span);
    a.rows = rows;
    a.cols = cols;
    a.tiles_per_row = cols / 256;
    a.batch = (int)batch;
    a.batch_pad = p.batch_pad;
    a.nb = p.nb;
    a.ksplit = p.ksplit;
    a.tiles_per_split = p.tiles_per_split;
    a.sign_key = hash_key(seed, 1);
    a.status = d_status;
    a.stall_tile = stall_tile;
    if (lowbit == 2) return launch_gemm_e4m3(lattice, a, s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
    if (lowbit == 1) return launch_gemm_i8(lattice, a, s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
    return launch_gemm(lattice, a, s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

}  // namespace

extern "C" {

int hq_decode_gemm(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps, uint64_t seed,
                   const void *x, int64_t batch, float *y, void *workspace, uint64_t workspace_bytes, void *stream,
                   int32_t *d_status)
{
    return decode_gemm_impl(w, rows, cols, tile, lattice, bps, seed, x, batch, y, workspace, workspace_bytes, stream,
                            d_status, -1);
}

int hq_decode_gemm_int8_workspace_bytes(int64_t rows, int64_t cols, int64_t batch, uint64_t *out)
{
    if (!out || rows < 0 || cols < 0 || batch < 0 || cols % 256) return HQ_ERR_ARG;
    if (batch > (int64_t)1 << 24) return HQ_ERR_UNSUPPORTED;
    GemmPlan p{};
    gemm_plan_i8(rows, cols, batch, 2, &p);  // the most splits any launch picks
    *out = (p.xt_bytes + 255) / 256 * 256 + p.part_bytes;
    return HQ_OK;
}

int hq_decode_gemm_int8(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                        uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                        uint64_t workspace_bytes, void *stream, int32_t *d_status)
{
    return decode_gemm_impl(w, rows, cols, tile, lattice, bps, seed, x, batch, y, workspace, workspace_bytes, stream,
                            d_status, -1, 1);
}

int hq_decode_gemm_fp8(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                       uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                       uint64_t workspace_bytes, void *stream, int32_t *d_status)
{
    return decode_gemm_impl(w, rows, cols, tile, lattice, bps, seed, x, batch, y, workspace, workspace_bytes, stream,
                            d_status, -1, 2);
}

int hq_test_gemm_stalled(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                         uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                         uint64_t workspace_bytes, void *stream, int32_t *d_status, int64_t stalled_tile)
{
    return decode_gemm_impl(w, rows, cols, tile, lattice, bps, seed, x, batch, y, workspace, workspace_bytes, stream,
                            d_status, stalled_tile);
}

int hq_kv_attention_workspace_bytes(int64_t heads, int64_t tokens, int head_dim, int group, uint64_t *out)
{
    if (!out || heads < 0 || tokens < 0 || !valid_head_dim(head_dim) || group < 1) return HQ_ERR_ARG;
    if (heads > 65535 || tokens >= (int64_t)1 << 32 || group > 65535 * 8) return HQ_ERR_UNSUPPORTED;
    *out = attention_workspace(heads, tokens, head_dim, group).total_bytes;
    return HQ_OK;
}

int hq_kv_attention(const hq_stream *k, const hq_stream *v, int64_t heads, int64_t tokens, int head_dim,
                    int group, int lattice, float bps_k, float bps_v, uint64_t seed_k, uint64_t seed_v,
                    const void *q, float scale, float *out, void *workspace, uint64_t workspace_bytes,
                    void *stream, int32_t *d_status)
{
    if (heads < 0 || tokens < 0 || !valid_head_dim(head_dim) || group < 1 || !std::isfinite(scale))
        return HQ_ERR_ARG;
    if (heads > 65535 || tokens >= (int64_t)1 << 32 || group > 65535 * 8) return HQ_ERR_UNSUPPORTED;
    if (heads > 0 && tokens > (int64_t)(((uint64_t)1 << 32) - 1) / heads) return HQ_ERR_UNSUPPORTED;
    AttnArgs a{};
    int64_t nk = 0, nv = 0;
    int rc = decode_common(k, heads * tokens, head_dim, head_dim, lattice, bps_k, seed_k, a.k, &nk);
    if (rc) return rc;
    if ((rc = decode_common(v, heads * tokens, head_dim, head_dim, lattice, bps_v, seed_v, a.v, &nv))) return rc;
    if ((a.k.slot != 0) != (a.v.slot != 0)) return HQ_ERR_UNSUPPORTED;  // K and V of one kind
    if (heads == 0) return HQ_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (!out || !aligned(out, 16)) return HQ_ERR_ARG;
    if (tokens == 0)
        return cudaMemsetAsync(out, 0, sizeof(float) * (size_t)(heads * group * head_dim), s) == cudaSuccess
                   ? HQ_OK : HQ_ERR_CUDA;
    if (!q || !aligned(q, 16)) return HQ_ERR_ARG;
    const AttnWorkspace w = attention_workspace(heads, tokens, head_dim, group);
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < w.total_bytes) return HQ_ERR_WORKSPACE;
    if (cudaMemsetAsync(workspace, 0, w.counter_bytes, s) != cudaSuccess) return HQ_ERR_CUDA;
    a.q = static_cast<const uint16_t *>(q);
    a.out = out;
    a.counter = static_cast<uint32_t *>(workspace);
    a.part = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.counter_bytes);
    a.heads = heads;
    a.tokens = tokens;
    a.group = group;
    a.scale = scale;
    a.status = d_status;
    return launch_attention(head_dim, lattice, a, s) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

}  // extern "C"
