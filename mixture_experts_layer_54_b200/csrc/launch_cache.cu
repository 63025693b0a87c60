// Launch-shape queries answered once per device and kernel.  The driver's
// answers (SM count, blocks or clusters resident at once) do not change while
// the process runs, and a kernel's shared-memory opt-in only has to be raised
// once, so the launchers ask here instead of asking the driver on every call.

#include <array>
#include <map>
#include <mutex>

#include "internal.cuh"

namespace moe {
namespace {

using Key = std::array<intptr_t, 6>;

std::mutex g_mu;
std::map<Key, int> g_memo;

int current_device(cudaError_t *err)
{
    int dev = 0;
    *err = cudaGetDevice(&dev);
    return dev;
}

bool lookup(const Key &k, int *out)
{
    std::lock_guard<std::mutex> g(g_mu);
    auto it = g_memo.find(k);
    if (it == g_memo.end())
        return false;
    *out = it->second;
    return true;
}

void store(const Key &k, int v)
{
    std::lock_guard<std::mutex> g(g_mu);
    g_memo[k] = v;
}

}  // namespace

int device_sms()
{
    cudaError_t err;
    const int dev = current_device(&err);
    const Key k{0, dev, 0, 0, 0, 0};
    int n = 0;
    if (err == cudaSuccess && lookup(k, &n))
        return n;
    n = 148;
    if (err == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
        store(k, n);
    return n;
}

cudaError_t raise_smem_limit(const void *kernel, int bytes)
{
    cudaError_t err;
    const int dev = current_device(&err);
    if (err != cudaSuccess)
        return err;
    const Key k{reinterpret_cast<intptr_t>(kernel), dev, 1, 0, 0, 0};
    int have = 0;
    if (lookup(k, &have) && have >= bytes)
        return cudaSuccess;
    // raised, never lowered: a launch asking for less than an earlier one
    // stays within the limit that launch set
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err == cudaSuccess)
        store(k, bytes);
    return err;
}

cudaError_t cached_blocks_per_sm(const void *kernel, int threads, int smem, int *out)
{
    cudaError_t err;
    const int dev = current_device(&err);
    if (err != cudaSuccess)
        return err;
    const Key k{reinterpret_cast<intptr_t>(kernel), dev, 2, threads, smem, 0};
    if (lookup(k, out))
        return cudaSuccess;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, kernel, threads, (size_t)smem);
    if (err == cudaSuccess)
        store(k, *out);
    return err;
}

cudaError_t cached_active_clusters(const void *kernel, int threads, int smem, int cluster,
                                   int *out)
{
    cudaError_t err;
    const int dev = current_device(&err);
    if (err != cudaSuccess)
        return err;
    const Key k{reinterpret_cast<intptr_t>(kernel), dev, 3, threads, smem, cluster};
    if (lookup(k, out))
        return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)cluster);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    err = cudaOccupancyMaxActiveClusters(out, kernel, &cfg);
    if (err == cudaSuccess)
        store(k, *out);
    return err;
}

}  // namespace moe
