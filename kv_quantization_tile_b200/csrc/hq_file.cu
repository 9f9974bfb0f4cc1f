// hq_file.cu -- packed checkpoint container for one compressed matrix (host
// code only; the arrays are the stream's own, copied by the caller to host
// memory).
//
// Layout (little-endian), every section 8-byte aligned:
//   header (128 bytes)                       see struct FileHeader
//   tile_off    uint32 x (ntiles + 1)        (none for a fixed-rate stream)
//   tile_scale  uint16 x ntiles              bf16 bits of Delta
//   tile_k      uint8  x ntiles              (fixed rate: (ntiles + 1) / 2 bytes, 4 bits per tile)
//   payload     uint32 x payload_words       (fixed rate: ntiles x slot words)
// The header carries the shape and codec parameters a decoder needs (tile,
// lattice, bits per sample, seed, dither flag, fixed-rate slot) and an
// FNV-1a 64-bit checksum of everything after it plus one of the header
// itself.
//
// Method: [I9] "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline
// ... #9" (a packed Rice-coded lattice-index checkpoint format).
#include <cstdint>
#include <cstring>

#include "../../include/hq.h"

namespace {

constexpr char kMagic[4] = { 'H', 'Q', 'F', '1' };
constexpr uint32_t kVersion = 1, kHeaderBytes = 128;

struct FileHeader {
    char magic[4];
    uint32_t version;
    uint32_t header_bytes;
    uint32_t flags;  // bit 0: KV stream (subtractive dither); bit 1: fixed-rate stream
    int64_t rows, cols;
    int32_t tile, lattice;
    float bps;
    uint32_t slot_words;  // fixed-rate slot (0 for a variable-rate stream)
    uint64_t seed;
    uint64_t ntiles, payload_words;
    uint64_t sec_off, sec_scale, sec_k, sec_payload, total_bytes;
    uint64_t body_checksum;   // FNV-1a 64 of bytes [header_bytes, total_bytes)
    uint64_t header_checksum; // FNV-1a 64 of this header with this field zero
};
static_assert(sizeof(FileHeader) <= kHeaderBytes, "header fits its 128 bytes");

uint64_t fnv1a(const uint8_t *p, uint64_t n, uint64_t h = 0xcbf29ce484222325ull)
{
    for (uint64_t i = 0; i < n; i++) {
        h ^= p[i];
        h *= 0x100000001b3ull;
    }
    return h;
}

uint64_t align8(uint64_t v) { return (v + 7) & ~7ull; }

constexpr uint32_t kFlagDither = 1u, kFlagFixed = 2u;

bool is_fixed(const hq_file_info *f) { return (f->flags & kFlagFixed) != 0; }

bool valid_info(const hq_file_info *f)
{
    if (!f || f->rows < 0 || f->cols < 0) return false;
    if (!(f->tile == 64 || f->tile == 128 || f->tile == 256 || f->tile == 512 || f->tile == 1024)) return false;
    if (!(f->lattice == HQ_Z || f->lattice == HQ_A2 || f->lattice == HQ_D4 || f->lattice == HQ_E8)) return false;
    if (!(f->bps > 0.0f && f->bps <= 8.0f)) return false;
    if (f->cols % f->tile) return false;
    const int64_t tpr = f->cols / f->tile;
    if (tpr && f->rows > INT64_MAX / 2 / tpr) return false;
    if ((uint64_t)(f->rows * tpr) != f->ntiles) return false;
    if (f->ntiles >= (1ull << 32) || f->payload_words >= (1ull << 32)) return false;
    if ((f->flags & ~(kFlagDither | kFlagFixed)) != 0) return false;
    if (is_fixed(f)) {
        // the slot limits of the fixed-rate encoder: the all-zero tile up to 8 bits per coordinate
        const uint32_t coset = (f->lattice == HQ_E8 || f->lattice == HQ_A2) ? (uint32_t)(f->tile / f->lattice) : 0u;
        const uint32_t min_slot = (coset + (uint32_t)f->tile + 31u) / 32u;
        if (f->slot_words < min_slot || f->slot_words > (uint32_t)f->tile / 4u) return false;
        if (f->payload_words != f->ntiles * f->slot_words) return false;
    } else if (f->slot_words != 0) {
        return false;
    }
    return true;
}

// section offsets for an info; false on overflow
bool layout(const hq_file_info *f, FileHeader &h)
{
    const uint64_t n = f->ntiles;
    const bool fixed = is_fixed(f);
    h.sec_off = kHeaderBytes;
    h.sec_scale = align8(h.sec_off + (fixed ? 0 : 4 * (n + 1)));
    h.sec_k = align8(h.sec_scale + 2 * n);
    h.sec_payload = align8(h.sec_k + (fixed ? (n + 1) / 2 : n));
    h.total_bytes = h.sec_payload + 4 * f->payload_words;
    return h.total_bytes >= h.sec_payload;
}

}  // namespace

extern "C" {

int hq_file_bytes(const hq_file_info *info, uint64_t *out)
{
    if (!out || !valid_info(info)) return HQ_ERR_ARG;
    FileHeader h{};
    if (!layout(info, h)) return HQ_ERR_UNSUPPORTED;
    *out = h.total_bytes;
    return HQ_OK;
}

int hq_file_write(const hq_file_info *info, const uint32_t *tile_off, const uint16_t *tile_scale,
                  const uint8_t *tile_k, const uint32_t *payload, void *buf, uint64_t buf_bytes)
{
    const bool fixed = info && is_fixed(info);
    if (!valid_info(info) || !buf || (!fixed && !tile_off)) return HQ_ERR_ARG;
    if (info->ntiles && (!tile_scale || !tile_k)) return HQ_ERR_ARG;
    if (info->payload_words && !payload) return HQ_ERR_ARG;
    if (!fixed && tile_off[info->ntiles] != info->payload_words) return HQ_ERR_ARG;  // the stream's own end offset
    FileHeader h{};
    if (!layout(info, h)) return HQ_ERR_UNSUPPORTED;
    if (buf_bytes < h.total_bytes) return HQ_ERR_CAPACITY;
    uint8_t *b = static_cast<uint8_t *>(buf);
    std::memset(b, 0, h.total_bytes);
    if (!fixed) std::memcpy(b + h.sec_off, tile_off, 4 * (info->ntiles + 1));
    if (info->ntiles) {
        std::memcpy(b + h.sec_scale, tile_scale, 2 * info->ntiles);
        std::memcpy(b + h.sec_k, tile_k, fixed ? (info->ntiles + 1) / 2 : info->ntiles);
    }
    if (info->payload_words) std::memcpy(b + h.sec_payload, payload, 4 * info->payload_words);
    std::memcpy(h.magic, kMagic, 4);
    h.version = kVersion;
    h.header_bytes = kHeaderBytes;
    h.flags = info->flags;
    h.rows = info->rows;
    h.cols = info->cols;
    h.tile = info->tile;
    h.lattice = info->lattice;
    h.bps = info->bps;
    h.slot_words = info->slot_words;
    h.seed = info->seed;
    h.ntiles = info->ntiles;
    h.payload_words = info->payload_words;
    h.body_checksum = fnv1a(b + kHeaderBytes, h.total_bytes - kHeaderBytes);
    h.header_checksum = 0;
    h.header_checksum = fnv1a(reinterpret_cast<const uint8_t *>(&h), sizeof(h));
    std::memcpy(b, &h, sizeof(h));
    return HQ_OK;
}

int hq_file_read(const void *buf, uint64_t buf_bytes, hq_file_info *info, const uint32_t **tile_off,
                 const uint16_t **tile_scale, const uint8_t **tile_k, const uint32_t **payload)
{
    if (!buf || !info) return HQ_ERR_ARG;
    if (buf_bytes < kHeaderBytes) return HQ_ERR_FORMAT;
    FileHeader h;
    std::memcpy(&h, buf, sizeof(h));
    if (std::memcmp(h.magic, kMagic, 4) != 0 || h.version != kVersion || h.header_bytes != kHeaderBytes)
        return HQ_ERR_FORMAT;
    const uint64_t hc = h.header_checksum;
    FileHeader z = h;
    z.header_checksum = 0;
    if (fnv1a(reinterpret_cast<const uint8_t *>(&z), sizeof(z)) != hc) return HQ_ERR_FORMAT;
    hq_file_info f{};
    f.rows = h.rows;
    f.cols = h.cols;
    f.tile = h.tile;
    f.lattice = h.lattice;
    f.bps = h.bps;
    f.flags = h.flags;
    f.slot_words = h.slot_words;
    f.seed = h.seed;
    f.ntiles = h.ntiles;
    f.payload_words = h.payload_words;
    if (!valid_info(&f)) return HQ_ERR_FORMAT;
    FileHeader want{};
    if (!layout(&f, want) || want.sec_off != h.sec_off || want.sec_scale != h.sec_scale || want.sec_k != h.sec_k ||
        want.sec_payload != h.sec_payload || want.total_bytes != h.total_bytes)
        return HQ_ERR_FORMAT;
    if (buf_bytes < h.total_bytes) return HQ_ERR_FORMAT;
    const uint8_t *b = static_cast<const uint8_t *>(buf);
    if (fnv1a(b + kHeaderBytes, h.total_bytes - kHeaderBytes) != h.body_checksum) return HQ_ERR_FORMAT;
    const bool fixed = is_fixed(&f);
    if (!fixed) {
        // stream-level checks: offsets start at 0, never decrease, end at the payload size
        uint32_t prev = 0, first;
        std::memcpy(&first, b + h.sec_off, 4);
        if (first != 0) return HQ_ERR_FORMAT;
        for (uint64_t t = 1; t <= f.ntiles; t++) {
            uint32_t o;
            std::memcpy(&o, b + h.sec_off + 4 * t, 4);
            if (o < prev) return HQ_ERR_FORMAT;
            prev = o;
        }
        if (prev != f.payload_words) return HQ_ERR_FORMAT;
        for (uint64_t t = 0; t < f.ntiles; t++)
            if (b[h.sec_k + t] > 15) return HQ_ERR_FORMAT;
    } else if (f.ntiles & 1) {
        if (b[h.sec_k + f.ntiles / 2] >> 4) return HQ_ERR_FORMAT;  // the unused half of the last byte
    }
    *info = f;
    if (tile_off) *tile_off = fixed ? nullptr : reinterpret_cast<const uint32_t *>(b + h.sec_off);
    if (tile_scale) *tile_scale = reinterpret_cast<const uint16_t *>(b + h.sec_scale);
    if (tile_k) *tile_k = b + h.sec_k;
    if (payload) *payload = reinterpret_cast<const uint32_t *>(b + h.sec_payload);
    return HQ_OK;
}

}  // extern "C"
