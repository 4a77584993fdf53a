// Position table without a caller workspace: ipe_mrope_rope_index_static.
//
// Some callers cannot hand the library device memory at call time: a serving
// loop that reserved all device memory up front and forbids allocation on its
// hot path, or a plain C host program with no device allocator of its own.
// For them this entry point runs ipe_mrope_rope_index on a scratch buffer the
// library owns: one statically sized device array per device, compiled into
// this library, so the call itself allocates nothing.
//
// The buffer's address is looked up once per device (cudaGetSymbolAddress,
// with that device current) by the first call made on that device; that call
// therefore does the set-up work and should come before any stream capture.
// Later calls check that the remembered address still names device memory of
// that device, and look it up again after a device reset.
// Every call first clears what must start at zero (a memset of the tile
// flags, the per-sample records and the tile ticket) and every other word is
// written before it is read, so the caller clears nothing between calls.  All calls on one device share the
// buffer: calls whose kernels overlap in time (other streams, other host
// threads) race with each other.
#include <cstdio>
#include <mutex>

#include "ipe.h"
#include "ipe_internal.h"

namespace ipe {
int set_error(int code, const char *msg);
}  // namespace ipe

// The library-owned scratch, IPE_ROPE_INDEX_STATIC_BYTES on every device.
static __device__ __align__(256) unsigned char g_rope_index_scratch[IPE_ROPE_INDEX_STATIC_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Address of the scratch on the current device (set up on first use).
int scratch_address(void **out)
{
    char msg[256];
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        snprintf(msg, sizeof msg, "cudaGetDevice: %s", cudaGetErrorString(e));
        return ipe::set_error(IPE_ECUDA, msg);
    }
    if (dev < 0 || dev >= kMaxDevices) {
        snprintf(msg, sizeof msg, "device %d is beyond the %d this entry point serves", dev, kMaxDevices);
        return ipe::set_error(IPE_ELIMIT, msg);
    }
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] != nullptr) {
        // A device reset (cudaDeviceReset, or the primary context released
        // and created again) unloads the library's module and may map it
        // elsewhere: an address that no longer names device memory of this
        // device is looked up again.
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, g_scratch_addr[dev]) != cudaSuccess || at.type != cudaMemoryTypeDevice ||
            at.device != dev) {
            cudaGetLastError();
            g_scratch_addr[dev] = nullptr;
        }
    }
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_rope_index_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the position-table scratch: %s",
                     e != cudaSuccess ? cudaGetErrorString(e) : "null address");
            return ipe::set_error(IPE_ECUDA, msg);
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return IPE_OK;
}

}  // namespace

extern "C" int ipe_mrope_rope_index_static(const void *mm_token_type_ids, const void *attention_mask, int id_bytes,
                                           int64_t B, int64_t L, const void *image_grid_thw, int n_images,
                                           const void *video_grid_thw, int n_videos, int grid_bytes,
                                           int spatial_merge, int32_t *position_ids, int32_t *rope_deltas,
                                           void *stream)
{
    const size_t need = ipe_mrope_rope_index_workspace(B, L, n_images, n_videos);
    if (need == 0 && B > 0)   // the sizes themselves are out of range: let the checked call say why
        return ipe_mrope_rope_index(mm_token_type_ids, attention_mask, id_bytes, B, L, image_grid_thw, n_images,
                                    video_grid_thw, n_videos, grid_bytes, spatial_merge, position_ids, rope_deltas,
                                    nullptr, 0, stream);
    if (need > (size_t)IPE_ROPE_INDEX_STATIC_BYTES) {
        char msg[160];
        snprintf(msg, sizeof msg, "these sizes need %zu bytes of scratch, above the %u this entry point has", need,
                 (unsigned)IPE_ROPE_INDEX_STATIC_BYTES);
        return ipe::set_error(IPE_ELIMIT, msg);
    }
    void *scratch = nullptr;
    if (int rc = scratch_address(&scratch)) return rc;
    return ipe_mrope_rope_index(mm_token_type_ids, attention_mask, id_bytes, B, L, image_grid_thw, n_images,
                                video_grid_thw, n_videos, grid_bytes, spatial_merge, position_ids, rope_deltas, scratch,
                                (size_t)IPE_ROPE_INDEX_STATIC_BYTES, stream);
}
