// moe_capacity_noalloc: the capacity stage without a caller-supplied
// workspace, for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or ask their framework
// for a buffer) at the point where they run the capacity step: for example a
// serving loop whose device memory is planned once at start-up and may not
// grow afterwards, or a host application whose device memory belongs to
// another allocator that must not be bypassed.  They still own and pass the
// inputs and outputs; only the stage's scratch moves into the library.
//
// The scratch is a file-scope __device__ array, so every GPU that loads the
// library holds it (256 KiB) until the process exits.  In host code the
// array's name is only a host-side stand-in for the symbol, never a device
// address: the device address is looked up with cudaGetSymbolAddress once per
// device, with that device current, and cached.
#include "internal.cuh"

#include <mutex>

namespace {

// one int32 table: the per-block histograms, room for one entry per (block
// of 256 tokens, rank, expert) (token order uses one per (block, expert))
constexpr int64_t kTableInts = 65536;
static __device__ __align__(256) int32_t g_capacity_scratch[kTableInts];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int32_t *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on the
// first call for that device).
cudaError_t scratch_on_current_device(int32_t **out)
{
    int dev = -1;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void *addr = nullptr;
        err = cudaGetSymbolAddress(&addr, g_capacity_scratch);
        if (err != cudaSuccess)
            return err;
        g_scratch_addr[dev] = static_cast<int32_t *>(addr);
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_capacity_noalloc(const moe_config *cfg, const int32_t *topk_idx,
                                           int32_t *counts, int32_t *pos, uint8_t *keep,
                                           int32_t *kept, int32_t *offsets, uint8_t *dropped,
                                           int32_t *n_dropped, moe_stream_t stream)
{
    if (!cfg)
        return MOE_ERR_NULL;
    const moe_config &c = *cfg;
    moe_status st = moe::validate(c);
    if (st != MOE_OK)
        return st;
    if (c.priority == MOE_PRIORITY_SCORE)
        return MOE_ERR_DTYPE;   // the score order needs scores and more scratch
    if (!counts || !kept || !offsets || !n_dropped ||
        (c.T > 0 && (!topk_idx || !pos || !keep || !dropped)))
        return MOE_ERR_NULL;
    // the table holds one int32 per (token block of 256, rank, expert)
    if ((int64_t)moe::cap_blocks(c) * c.k * c.E > kTableInts)
        return MOE_ERR_WORKSPACE;
    int32_t *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess)
        return MOE_ERR_CUDA;
    // The table is written in full by this call before it is read, so
    // whatever an earlier call left in it does not matter.
    cudaError_t err = moe::launch_capacity(c, moe::capacity_of(c), topk_idx, counts, pos, keep,
                                           kept, offsets, dropped, n_dropped, scratch,
                                           reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
