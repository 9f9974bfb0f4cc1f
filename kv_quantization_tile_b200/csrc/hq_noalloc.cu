// hq_noalloc.cu -- hq_encode_noalloc: the encoder for callers that cannot
// allocate device memory.
//
// hq_encode needs a small scratch workspace (a chunk counter and one 64-bit
// prefix slot per chunk of tiles for its single-pass offset scan) that the
// caller allocates.  Some callers cannot do that: engines that hand out
// device memory only through their own pre-reserved pool and forbid raw
// cudaMalloc after start-up, plug-ins that run inside a host framework's
// memory manager, and latency-critical paths where cudaMalloc is not allowed
// because it can block or implicitly synchronise the device.  This entry
// point takes no workspace: the scratch lives in a fixed array below, in
// every GPU's global memory, for as long as the library stays loaded.
//
// The kernel launched is the same encoder hq_encode launches; only where its
// scratch comes from differs.
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_internal.h"

namespace {

// 256 bytes for the chunk counter, then one 8-byte slot per chunk.
constexpr uint64_t kNoallocChunks = 65536;
constexpr uint64_t kNoallocScratchBytes = 256 + 8 * kNoallocChunks;

// Device-resident scratch shared by every call on a device.  In host code
// this name is only a stand-in; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the scratch array on the current device.  It is looked
// up on every call (a host-side table lookup once the module is loaded, no
// allocation), so the address stays right after a device reset reloads the
// module at a new place.
int scratch_address(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HQ_ERR_CUDA;
    *out = p;
    return HQ_OK;
}

}  // namespace

extern "C" int hq_encode_noalloc(const void *x, int dtype, int64_t rows, int64_t cols, int tile, int lattice,
                                 float bps, uint64_t seed, const hq_stream *out, void *stream,
                                 int32_t *d_status)
{
    // Scratch bytes this shape needs; reject anything beyond the fixed array.
    uint64_t need = 0;
    int rc = hq_encode_workspace_bytes(rows, cols, tile, &need);
    if (rc != HQ_OK) return rc;
    if (need > kNoallocScratchBytes) return HQ_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((rc = scratch_address(&scratch)) != HQ_OK) return rc;
    // hq_encode clears the `need` bytes it uses on `stream` before launching,
    // so what an earlier call left in the array does not matter.
    return hq_encode(x, dtype, rows, cols, tile, lattice, bps, seed, out, scratch, need, stream, d_status);
}
