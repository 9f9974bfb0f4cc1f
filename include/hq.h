/*
 * hq.h -- C ABI of the B200 (sm_100a) HyperQuant per-tile codec.
 *
 * The method (sources cited by page title and section):
 *   [V1] "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline for
 *        Large Language and Diffusion Models", section "Abstract (arXiv)":
 *        (i) per-tile randomized Hadamard transform, (ii) quantization to a
 *        low-dimensional lattice E8, D4, A2 or Z, (iii) lossless
 *        bit-stripping and Rice coding of the lattice indices, (iv) a KV-cache
 *        bias correction keeping inner products unbiased.
 *   [V2] "HyperQuant: A Near-Entropy-Optimal Lattice Quantization Pipeline
 *        for Large Language and Diffusion Models", abstract: the rotation
 *        whitens each tile, the strip removes the bits lattice membership
 *        fixes, a Rice code carries the remainder, decoding is algebraic, and
 *        the KV cache uses subtractive dither; a batch-1 decode path is
 *        compared with a bf16 GEMV.
 *
 * Data model.  A matrix is row-major, `rows` x `cols`, `cols` a multiple of
 * the tile length n.  Tile t = r * (cols / n) + j is the row segment
 * x[r][j n .. j n + n).  For every tile the codec computes
 *     v = H (s_j . w)           s_j: seeded random signs of column tile j,
 *                               H: unnormalised Sylvester-Hadamard matrix
 *     Delta = bf16(c(lattice, bps) * sqrt(sum w^2))
 *     y = Q_lattice(v / Delta [+ dither])
 * strips the bits membership fixes, zigzags the remaining integers and
 * Rice-codes them with the tile's own parameter k.  Decoding returns
 *     w_hat = s_j . H (Delta (y [- dither])) / n.
 *
 * Stream.  The caller owns every buffer (device memory, e.g. from
 * torch.empty); the library never allocates, never synchronises, and runs
 * every call asynchronously on the given CUDA stream (`stream` is a
 * cudaStream_t passed as void*; NULL = the legacy default stream).
 *   payload     32-bit words; tile t occupies words [tile_off[t], tile_off[t+1])
 *   tile_off    ntiles + 1 word offsets; tile_off[0] = 0,
 *               tile_off[ntiles] = total payload words
 *   tile_scale  ntiles bf16 bit patterns of Delta (0 = all-zero tile)
 *   tile_k      ntiles Rice parameters, 0..15
 * (A fixed-rate stream, hq_stream.slot_words > 0, has no offsets and packs k
 * in 4 bits: see hq_stream and hq_encode_fixed.)
 * Tile layout, bits LSB-first in little-endian words: the n/d coset bits
 * (E8 and A2 only), then k low bits of each of the n codes in coordinate
 * order, then for each code q = u >> k zero bits and a one bit, then zero
 * padding to a word.
 *
 * Errors.  Functions return HQ_OK or an HQ_ERR_* code synchronously for bad
 * arguments or a failed launch; nothing is launched then.  Conditions found
 * on the device are OR-ed into *d_status (a caller-owned device int32; pass
 * NULL to skip): HQ_ST_NONFINITE (a tile held NaN/Inf or its sum of squares
 * overflowed: it is encoded as an all-zero tile), HQ_ST_CAPACITY (payload
 * too small: words past the capacity are not written), HQ_ST_CORRUPT (a
 * decoded tile is not a canonical tile: its output is zero), HQ_ST_TIMEOUT
 * (a bounded wait between thread blocks gave up: the call's output is
 * invalid), HQ_ST_RANGE (the integer product saturated a doubled lattice
 * coordinate to +-127).
 *
 * The same seed must be given to encode and decode: signs and dither are
 * regenerated from it, not stored.
 */
#ifndef HQ_H
#define HQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* lattices; the value is the lattice dimension d */
enum { HQ_Z = 1, HQ_A2 = 2, HQ_D4 = 4, HQ_E8 = 8 };

/* element types of dense inputs / outputs */
enum { HQ_BF16 = 0, HQ_F32 = 1 };

/* synchronous return codes */
enum {
    HQ_OK = 0,
    HQ_ERR_ARG = 1,          /* null pointer, bad size, tile, lattice, bps or dtype */
    HQ_ERR_UNSUPPORTED = 2,  /* valid request outside what this build handles */
    HQ_ERR_CAPACITY = 3,     /* payload capacity below the worst-case bound */
    HQ_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
    HQ_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    HQ_ERR_FORMAT = 6        /* a checkpoint buffer is not a valid, intact container */
};

/* device status bits OR-ed into *d_status */
enum { HQ_ST_NONFINITE = 1, HQ_ST_CAPACITY = 2, HQ_ST_CORRUPT = 4, HQ_ST_TIMEOUT = 8, HQ_ST_RANGE = 16 };

/* A compressed matrix.  Host struct; all pointers are device memory owned by
 * the caller.
 * Variable rate (slot_words = 0): payload >= hq_max_payload_words(...) words
 * for encode (the exact count is tile_off[ntiles] afterwards), tile_off
 * ntiles + 1, tile_scale ntiles, tile_k ntiles.
 * Fixed rate (slot_words = S > 0, written by hq_encode_fixed /
 * hq_kv_encode_fixed): tile t occupies payload words [t S, t S + S) (the
 * tile layout above, then zero words), payload >= ntiles S words, tile_off
 * is not used (may be NULL), tile_scale ntiles, tile_k (ntiles + 1) / 2
 * bytes holding k of tile t in bits 4 (t mod 2) .. 4 (t mod 2) + 3 of byte
 * t / 2.  Every decoder below accepts either kind. */
typedef struct hq_stream {
    uint32_t *payload;
    uint64_t payload_capacity_words;
    uint32_t *tile_off;
    uint16_t *tile_scale;
    uint8_t *tile_k;
    uint32_t slot_words;
} hq_stream;

/* Static description of a return code (never NULL). */
const char *hq_error_string(int code);

/* Library version: major * 10000 + minor * 100 + patch. */
int hq_version(void);

/* c(lattice, bps) = fp32(sqrt(2 pi e) 2^-bps V^(-1/d)), V the lattice cell
 * volume (E8 1, D4 2, A2 sqrt3/2, Z 1): Delta = bf16(c sqrt(sum w^2)) puts
 * the high-resolution entropy of the lattice indices at `bps` bits per
 * coordinate for Gaussian tiles.  The pages name a per-tile scale for the
 * target rate but not its rule; this is the reading ([V1] (ii), [V2]).
 * Host only.  HQ_ERR_ARG for a bad lattice, bps outside (0, 8] or out == NULL. */
int hq_rate_constant(int lattice, float bps, float *out);

/* Worst-case words of one tile: n/d coset bits + n (1 + kb) bits rounded up,
 * kb the bits of the largest zigzag symbol a tile can produce (the rotated
 * coordinates obey |v_i| <= sqrt(n sum w^2)).  Host only. */
int hq_tile_bound_words(int tile, int lattice, float bps, uint32_t *out);

/* ntiles * hq_tile_bound_words: a payload this large never overflows.
 * HQ_ERR_UNSUPPORTED if the bound reaches 2^32 words (offsets are 32-bit). */
int hq_max_payload_words(int64_t rows, int64_t cols, int tile, int lattice, float bps,
                         uint64_t *out);

/* Bytes of device workspace hq_encode / hq_kv_encode need for this shape
 * (a chunk counter and one 64-bit prefix slot per chunk of tiles, used by
 * the single-pass decoupled look-back scan that assigns tile offsets).
 * Host only. */
int hq_encode_workspace_bytes(int64_t rows, int64_t cols, int tile, uint64_t *out);

/* Encode ([V1] (i)-(iii), [V2]).
 *   x          device, rows x cols, HQ_BF16 or HQ_F32 (`dtype`), 16-byte aligned
 *   rows, cols rows >= 0, cols >= 0, cols % tile == 0 (0 rows or cols: empty
 *              stream, tile_off[0] = 0)
 *   tile       n in {64, 128, 256, 512, 1024}
 *   lattice    HQ_E8, HQ_D4, HQ_A2 or HQ_Z
 *   bps        target bits per coordinate, 0 < bps <= 8
 *   seed       signs of the rotation
 *   out        stream to fill; payload_capacity_words >= hq_max_payload_words
 *   workspace  device, >= hq_encode_workspace_bytes, 8-byte aligned; its
 *              contents are overwritten (it is cleared on `stream` first)
 * Tiles are encoded independently except for their offsets, which a single
 * pass assigns with a decoupled look-back prefix scan over chunks of tiles. */
int hq_encode(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice,
              float bps, uint64_t seed, const hq_stream *out, void *workspace,
              uint64_t workspace_bytes, void *stream, int32_t *d_status);

/* KV-cache encode ([V1] (iv), [V2] subtractive dither): as hq_encode, with a
 * seeded dither added before the nearest-point step: uniform (16-bit grid)
 * on a centred box that is a fundamental domain of a sublattice (D_d for E8
 * and D4, Z x sqrt3 Z for A2, Z for Z), so the decoded error is uniform on
 * the Voronoi cell and independent of the input.  A KV slab is laid out as (heads * tokens) rows of
 * head_dim columns, tile = head_dim, so each tile is one cached vector. */
int hq_kv_encode(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice,
                 float bps, uint64_t seed, const hq_stream *out, void *workspace,
                 uint64_t workspace_bytes, void *stream, int32_t *d_status);

/* ------------------------------------------------------------------
 * Fixed rate: compact headers and exact rate control.  The pages quote
 * whole-model compression ratios that count every stored bit (about 3.9x
 * for the weights and 3.79x for the KV cache at 4 bps, [V1] abstract) and
 * name the per-tile scale as the control of the rate.  Reading: each tile
 * gets a slot of S words, so its offset t S is implicit, k is kept in 4
 * bits, and the tile's only side information is the bf16 Delta and k (20
 * bits): (32 S + 20) / n bits per coordinate, exactly.  Delta is searched
 * per tile so the coded tile fits its slot: the size at the closed-form
 * scale c0 (rate 32 S / n - 5/32) predicts a start (one bf16 step moves the
 * size by about n / 128 bits), then steps of 1, 2, 4, ... bf16 patterns
 * towards the boundary (within four octaves of c0), then bisection, ending
 * at a fitting Delta whose next finer bf16 value does not fit.  A tile that fits
 * at no scale of that range (possible only with dither at very small slots)
 * is stored as the all-zero tile. */

/* Smallest slot: the all-zero tile, (n/d coset bits (E8, A2) + n) / 32
 * rounded up.  Host only. */
int hq_min_slot_words(int tile, int lattice, uint32_t *out);

/* Slot for a total rate of `bps` bits per coordinate, side information
 * included: floor((bps n - 20) / 32).  HQ_ERR_ARG if that is below
 * hq_min_slot_words or an argument is invalid.  Host only. */
int hq_fixed_slot_words(int tile, int lattice, float bps, uint32_t *out);

/* Fixed-rate encode.  Arguments as hq_encode except:
 *   out        out->slot_words = S with hq_min_slot_words <= S <= n / 4;
 *              payload_capacity_words >= ntiles S (< 2^32); tile_off unused
 * No workspace: tiles are independent.  Every tile's slot is written whole
 * (zero words after the tile), tile_scale[t] and the packed k. */
int hq_encode_fixed(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice,
                    uint64_t seed, const hq_stream *out, void *stream, int32_t *d_status);

/* Fixed-rate KV-cache encode: as hq_encode_fixed with the subtractive
 * dither of hq_kv_encode; decode with hq_kv_decode or hq_kv_attention. */
int hq_kv_encode_fixed(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice,
                       uint64_t seed, const hq_stream *out, void *stream, int32_t *d_status);

/* Decode ([V2] algebraic decoding): y = s . H (Delta y_lattice) / n per tile,
 * rounded to `dtype` (bf16 round-to-nearest-even, or fp32).
 *   in         stream written by hq_encode with the same shape, tile,
 *              lattice, bps and seed, or by hq_encode_fixed with the same
 *              shape, tile, lattice and seed (bps must still be valid; the
 *              slot sets the rate)
 *   y          device, rows x cols, 16-byte aligned
 * A tile whose words are not a canonical tile (bad offsets, k > 15, wrong
 * symbol count, a set padding bit) is written as zeros and HQ_ST_CORRUPT is
 * raised; no read leaves [tile_off[t], tile_off[t+1]) (the slot, for a
 * fixed-rate stream) or the capacity. */
int hq_decode(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice, float bps,
              uint64_t seed, void *y, int dtype, void *stream, int32_t *d_status);

/* KV-cache decode: as hq_decode, subtracting the same dither
 * (w_hat = s . H (Delta (y - delta)) / n). */
int hq_kv_decode(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice,
                 float bps, uint64_t seed, void *y, int dtype, void *stream, int32_t *d_status);

/* Fused decode + GEMV at batch 1 ([V2] batch-1 decode path):
 *   y[r] = sum_c w_hat[r][c] x[c], fp32 accumulation, without forming w_hat.
 * Because H is symmetric, each tile contributes
 *   (Delta / n) <y_lattice, H (s_j . x_j)>,
 * so x is rotated once per column tile and the per-tile inverse rotation
 * disappears.
 *   w          stream of a rows x cols matrix (no dither)
 *   x          device bf16, cols entries, 16-byte aligned
 *   y          device fp32, rows entries
 * cols * 4 bytes of rotated x must fit in shared memory (cols <= 40960). */
int hq_decode_gemv(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice,
                   float bps, uint64_t seed, const void *x, float *y, void *stream,
                   int32_t *d_status);

/* Rate accounting of a stream ([V2] abstract: itemized rate accounting;
 * the Rice code's distance from the lattice's rate-distortion ideal).  The
 * stream is read, not changed; any stream kind (variable or fixed rate).
 * counts: device uint64[8], cleared by the call, then: canonical tiles, coset
 * bits, low-part bits (n k per tile), unary bits (sum(u >> k) + n), padding
 * bits (the tile's words minus those), offset-header bits (32 per tile; 0 in
 * a fixed-rate stream), scale-header bits (16), Rice-parameter bits (8; 4
 * packed in a fixed-rate stream).  hist: device uint64[2][bins] (2 <= bins
 * <= 4096), cleared by the call: counts of symbol values 0 .. bins - 2 and of
 * values >= bins - 1 in the last bin; row 1 holds the stripped last
 * coordinates of D4 / E8 vectors, row 0 every other symbol.  Both pointers
 * 8-byte aligned, caller-owned.  Asynchronous on `stream`; tiles that are not
 * canonical are skipped and raise HQ_ST_CORRUPT.  HQ_ERR_ARG for bad
 * pointers or bins, the decode calls' shape errors otherwise. */
int hq_stream_stats(const hq_stream *in, int64_t rows, int64_t cols, int tile, int lattice,
                    float bps, uint64_t *counts, uint64_t *hist, int bins, void *stream,
                    int32_t *d_status);

/* Bytes of device workspace hq_decode_gemm needs for this shape: the
 * rotated activations (bf16, batch rounded up to the block's batch rows x
 * cols), then, when column tiles are split across blocks, fp32 partial
 * results (splits x padded batch x rows).  Depends on the SM count of the
 * current device.  Host only.  HQ_ERR_ARG for negative sizes, a cols that is
 * not a multiple of 256 or out == NULL. */
int hq_decode_gemm_workspace_bytes(int64_t rows, int64_t cols, int64_t batch, uint64_t *out);

/* Batched decode + matrix product on the tensor cores ([V2] decode path
 * beside bf16 matrix products; [V1] MMA decode paths):
 *   y[b][r] = sum_c x[b][c] w_hat[r][c]   (Y = X W_hat^T)
 * computed as (1/n) sum_j <H(s_j . x_bj), Delta_rj y_rj>: the weights stay in
 * the rotated domain and are parsed straight into bf16 tensor-core operands
 * (Delta y rounded once to bf16, as a bf16 decode would); the activations are
 * rotated once per call and rounded to bf16; products accumulate in fp32
 * (tcgen05.mma, tensor memory).
 *   w          stream of a rows x cols matrix (no dither), tile 256
 *              (HQ_ERR_UNSUPPORTED for other tiles)
 *   x          device bf16 [batch][cols], 16-byte aligned
 *   batch      >= 0 activation rows
 *   y          device fp32 [batch][rows]
 *   workspace  device, >= hq_decode_gemm_workspace_bytes, 16-byte aligned
 * Corrupt tiles count as zero rows of W and raise HQ_ST_CORRUPT; a bounded
 * wait on the tensor cores that gives up raises HQ_ST_TIMEOUT. */
int hq_decode_gemm(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                   uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                   uint64_t workspace_bytes, void *stream, int32_t *d_status);

/* Bytes of device workspace hq_decode_gemm_int8 (and hq_decode_gemm_fp8) needs: the quantized
 * activations (int8, batch rounded up to the block's batch rows (at most 128)
 * x cols, 256-byte rounded), their scales (fp32, padded batch x cols / 256),
 * then fp32 split-K partials.  Host only; as hq_decode_gemm_workspace_bytes. */
int hq_decode_gemm_int8_workspace_bytes(int64_t rows, int64_t cols, int64_t batch, uint64_t *out);

/* Batched decode + integer tensor-core product ([V1] abstract: 8-bit MMA
 * paths, int8 ahead of fp8 on the lattice output after the rotation):
 *   y[b][r] = sum_j Delta_rj s_bj / (2 n) sum_i A_rji q_bji
 * with A = 2y, the doubled lattice coordinates (exact integers for E8, D4
 * and Z; saturated to +-127 with HQ_ST_RANGE raised where they leave int8),
 * and q_bj = rint(x~_bj 127 / max|x~_bj|), s_bj = max|x~_bj| / 127 the
 * rotated activations x~_bj = H (s_j . x_bj) quantized per (batch row,
 * column tile) in binary32.  The int32 sums over each column tile are exact
 * (tcgen05.mma kind::i8, TMEM accumulator); scaling and the sum over column
 * tiles are fp32.  The activation rounding makes this an approximation of
 * X W_hat^T (each term moves by at most s_bj / 2).  Arguments as
 * hq_decode_gemm; lattice HQ_A2 returns HQ_ERR_UNSUPPORTED (its points carry
 * sqrt 3).  Non-finite activations give non-finite outputs. */
int hq_decode_gemm_int8(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                        uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                        uint64_t workspace_bytes, void *stream, int32_t *d_status);

/* Batched decode + fp8 tensor-core product ([V1] abstract: the fp8-e4m3
 * MMA path, which the pages find behind int8 on the lattice output): as
 * hq_decode_gemm_int8 with both operands in OCP FP8 E4M3 (largest finite
 * 448): A = e4m3(2y), exact while |2y| <= 16 and rounded to nearest even on
 * the format's coarser grid beyond (HQ_ST_RANGE where |2y| > 448, saturated),
 * and q_bj = e4m3(x~_bj 448 / max|x~_bj|), s_bj = max|x~_bj| / 448.  Products
 * accumulate in fp32 on the tensor cores (tcgen05.mma kind::f8f6f4).
 * Workspace: hq_decode_gemm_int8_workspace_bytes.  A2 returns
 * HQ_ERR_UNSUPPORTED. */
int hq_decode_gemm_fp8(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                       uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                       uint64_t workspace_bytes, void *stream, int32_t *d_status);

/* Testing hook for failure detection (no counterpart on the pages):
 * hq_decode_gemm in which column tile `stalled_tile` never issues or commits
 * its tensor-core products, so the bounded wait for them runs out (0.5 s):
 * the blocks that reach it raise HQ_ST_TIMEOUT, leave with no tensor-core
 * work in flight, free their tensor memory and return; the output is
 * invalid, the device stays usable.  Not for production use. */
int hq_test_gemm_stalled(const hq_stream *w, int64_t rows, int64_t cols, int tile, int lattice, float bps,
                         uint64_t seed, const void *x, int64_t batch, float *y, void *workspace,
                         uint64_t workspace_bytes, void *stream, int32_t *d_status, int64_t stalled_tile);

/* Bytes of device workspace hq_kv_attention needs: 256-byte-rounded
 * counters (heads * ceil(group / queries per block) uint32) followed by
 * heads * group * splits * (head_dim + 2) floats of per-split partial
 * results, for the largest number of token splits a call of this shape can
 * choose (a call picks its splits from the kernel's occupancy and never
 * exceeds this).  Depends on (heads, tokens, head_dim, group) and the SM
 * count of the current device, so query it on the device the call will run
 * on.  Host only.  HQ_ERR_ARG for negative sizes, head_dim not 64/128/256,
 * group < 1 or out == NULL. */
int hq_kv_attention_workspace_bytes(int64_t heads, int64_t tokens, int head_dim, int group,
                                    uint64_t *out);

/* Batch-1 attention over a dithered compressed KV cache ([V2] subtractive
 * dither keeps each cached inner product unbiased; [V1] (iv) the KV codec
 * serves attention).  For query head qh = h * group + g (grouped-query
 * attention: `group` query heads share KV head h):
 *   out[qh] = sum_t softmax_t(scale <q[qh], k_hat_t>) v_hat_t
 * with k_hat_t, v_hat_t what hq_kv_decode returns for tile h * tokens + t of
 * each stream, in fp32, without forming them: q is rotated once with the K
 * signs, scores come from the K stream's lattice points, and values are
 * accumulated in the rotated domain with one inverse rotation per query.
 *   k, v        streams written by hq_kv_encode (or both by
 *               hq_kv_encode_fixed; a variable-rate K with a fixed-rate V,
 *               or the reverse, is HQ_ERR_UNSUPPORTED) of a (heads * tokens)
 *               x head_dim slab, tile = head_dim, with lattice, bps_k / bps_v
 *               and seed_k / seed_v
 *   heads       KV heads (<= 65535), tokens >= 0 cached vectors per head
 *   head_dim    64, 128 or 256
 *   group       query heads per KV head, >= 1
 *   q           device bf16 [heads * group][head_dim], 16-byte aligned
 *   scale       finite softmax scale (typically 1 / sqrt(head_dim))
 *   out         device fp32 [heads * group][head_dim], 16-byte aligned
 *   workspace   device, >= hq_kv_attention_workspace_bytes, 16-byte
 *               aligned; its counters are cleared on `stream` first, so calls
 *               sharing one workspace must be ordered
 * tokens == 0 writes zeros.  A non-canonical tile counts as a zero vector and
 * raises HQ_ST_CORRUPT.  Non-finite q or scores propagate to out. */
int hq_kv_attention(const hq_stream *k, const hq_stream *v, int64_t heads, int64_t tokens,
                    int head_dim, int group, int lattice, float bps_k, float bps_v, uint64_t seed_k,
                    uint64_t seed_v, const void *q, float scale, float *out, void *workspace,
                    uint64_t workspace_bytes, void *stream, int32_t *d_status);

/* Testing hook for failure detection (no counterpart on the pages): hq_encode
 * in which the chunk of tiles numbered `stalled_chunk` (in encode-chunk order)
 * never publishes its word count to the cross-block prefix scan, so the
 * next chunk's bounded wait runs out.  The call still returns: the waiting
 * block raises HQ_ST_TIMEOUT after at most 0.5 s, publishes its own prefix
 * so later chunks proceed, and the stream it leaves is invalid.  The device
 * stays usable.  Not for production use. */
int hq_test_encode_stalled(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice,
                           float bps, uint64_t seed, const hq_stream *out, void *workspace,
                           uint64_t workspace_bytes, void *stream, int32_t *d_status,
                           uint32_t stalled_chunk);

/* Encode without a caller-provided workspace.  No counterpart on the pages:
 * this entry point exists for callers that cannot allocate device memory --
 * engines that hand out memory only from their own pre-reserved pool and
 * forbid cudaMalloc after start-up, plug-ins living inside another
 * framework's allocator, or paths where cudaMalloc may not run because it
 * can block or synchronise the device.
 * Same arguments, output and device status as hq_encode, minus the
 * workspace.  Its scratch is a fixed 512 KiB + 256 B array in each GPU's
 * global memory, held by every GPU that loads the library until the process
 * exits; a call may use at most 65536 encode chunks (that is,
 * hq_encode_workspace_bytes(rows, cols, tile) <= 256 + 8 * 65536), larger
 * shapes return HQ_ERR_UNSUPPORTED with nothing launched.  The call allocates
 * nothing.  Every call looks up the current device's scratch address
 * (cudaGetSymbolAddress, with that device current), so the address is right
 * again after a cudaDeviceReset; the first call on a device may load the
 * library's device code, so make that first call before any stream capture.
 * Every call on a device shares the one
 * array and clears the part it uses on `stream` before its kernel runs, so
 * calls whose work overlaps on the GPU (different streams, no ordering)
 * race on it and must be serialised by the caller. */
int hq_encode_noalloc(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice,
                      float bps, uint64_t seed, const hq_stream *out, void *stream,
                      int32_t *d_status);

/* ---------------------------------------------------------------- file
 * Packed checkpoint container for one compressed matrix ([I9] a packed
 * Rice-coded lattice-index format).  Host memory only: the caller copies the
 * stream's arrays to the host (and back after reading).  Layout,
 * little-endian, sections 8-byte aligned: a 128-byte header (magic "HQF1",
 * version 1, flags, rows, cols, tile, lattice, bps, seed, ntiles,
 * payload_words, section offsets, FNV-1a 64-bit checksums of the body and of
 * the header), then tile_off (uint32 x ntiles + 1), tile_scale (uint16 x
 * ntiles), tile_k (uint8 x ntiles) and the payload (uint32 x payload_words).
 * A fixed-rate stream (flags bit 1, slot_words in the header word after bps)
 * has no tile_off section, its tile_k section holds the packed 4-bit k
 * ((ntiles + 1) / 2 bytes) and its payload is ntiles x slot_words words. */
typedef struct hq_file_info {
    int64_t rows, cols;
    int32_t tile, lattice;
    float bps;
    uint32_t flags;          /* bit 0: KV stream (decode with dither); bit 1: fixed-rate stream */
    uint64_t seed;
    uint64_t ntiles;         /* rows * cols / tile */
    uint64_t payload_words;  /* tile_off[ntiles]; fixed rate: ntiles * slot_words */
    uint32_t slot_words;     /* fixed rate: the slot (hq_min_slot_words .. tile / 4); else 0 */
} hq_file_info;

/* Bytes of the container for `info`.  HQ_ERR_ARG if the fields are not a
 * valid shape and codec parameter set (ntiles must equal rows * cols / tile). */
int hq_file_bytes(const hq_file_info *info, uint64_t *out);

/* Write the container into buf (host, >= hq_file_bytes).  tile_off must end
 * at payload_words (fixed rate: tile_off is not read and may be NULL).
 * HQ_ERR_CAPACITY if buf is too small. */
int hq_file_write(const hq_file_info *info, const uint32_t *tile_off, const uint16_t *tile_scale,
                  const uint8_t *tile_k, const uint32_t *payload, void *buf, uint64_t buf_bytes);

/* Check a container (magic, version, header and body checksums, section
 * layout, parameters, offsets non-decreasing from 0 to the payload size,
 * k <= 15; fixed rate: a legal slot, payload = ntiles x slot, the unused
 * half of an odd tile count's last k byte zero) and return its info and
 * pointers into buf (any pointer argument may be NULL; *tile_off is NULL for
 * a fixed-rate stream).  HQ_ERR_FORMAT for anything that does not check out. */
int hq_file_read(const void *buf, uint64_t buf_bytes, hq_file_info *info, const uint32_t **tile_off,
                 const uint16_t **tile_scale, const uint8_t **tile_k, const uint32_t **payload);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
