// tt_emb_forward_noalloc: the forward pass for callers that cannot allocate
// device memory (see include/tt_emb.h).  Its scratch is this file's fixed
// device array; the host side looks up the array's device address once per
// device and passes that address to the kernels.  The paper has no
// counterpart; this is a deployment variant of the library.
#include <mutex>
#include <string.h>

#include "tt_common.cuh"

namespace tt {
int handle_device(tt_emb_t h);
int record_error(tt_emb_t h, int rc);
size_t scratch_bytes_for(tt_emb_t h, int64_t num_lookups);
int forward_with_scratch(tt_emb_t h, char* scratch, size_t scratch_bytes, const int64_t* indices,
                         const int64_t* offsets, int64_t num_lookups, int64_t batch, float* out,
                         cudaStream_t s);
}  // namespace tt

namespace {

constexpr size_t kScratchBytes = TT_EMB_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a usable address: the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up on the first
// call per device (with that device current) and cached.  The handle's cores and
// status block live on the device it was created on; a call made while another
// device is current is refused rather than mixing the two devices' memory.
int scratch_on_current_device(tt_emb_t h, char** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TT_ERR_CUDA;
    if (dev != tt::handle_device(h)) return TT_ERR_STATE;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TT_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = (char*)g_scratch_ptr[dev];
    return TT_OK;
}

}  // namespace

static int forward_noalloc(tt_emb_t h, const int64_t* indices, const int64_t* offsets, int64_t num_lookups,
                           int64_t batch, float* out, tt_stream_t stream)
{
    if (!h || !offsets || !out || num_lookups < 0 || batch < 1) return TT_ERR_ARG;
    if (num_lookups > TT_EMB_NOALLOC_MAX_LOOKUPS) return TT_ERR_WORKSPACE;
    if (tt::scratch_bytes_for(h, num_lookups) > kScratchBytes) return TT_ERR_WORKSPACE;
    char* scratch = nullptr;
    const int rc = scratch_on_current_device(h, &scratch);
    if (rc != TT_OK) return rc;
    return tt::forward_with_scratch(h, scratch, kScratchBytes, indices, offsets, num_lookups, batch,
                                    out, (cudaStream_t)stream);
}

extern "C" int tt_emb_forward_noalloc(tt_emb_t h, const int64_t* indices, const int64_t* offsets,
                                      int64_t num_lookups, int64_t batch, float* out,
                                      tt_stream_t stream)
{
    return tt::record_error(h, forward_noalloc(h, indices, offsets, num_lookups, batch, out, stream));
}
