// Balancing losses from the router's per-block partial sums and the
// capacity stage's counts, reduced in a fixed order (deterministic).
//
// Page "Lab 18 - Mixture of experts", section 2:
//   L_aux = E * sum_i f_i P_i, f_i = counts_i / (T k), P_i = mean_t p_{t,i}
//   L_z   = (1/T) sum_t (logsumexp_i z_{t,i})^2
// "Lab 01", where to start step 3: f divides by the T k slots.
#include "internal.cuh"

namespace moe {
namespace {

constexpr int THREADS = 256;

__global__ void __launch_bounds__(THREADS)
losses_kernel(const int32_t *counts, const float *partials, int nblk, int T, int k, int E,
              float *aux, float *zloss)
{
    __shared__ double term[THREADS];
    double acc = 0.0;
    // expert i: P_i summed over blocks in block order, times f_i
    for (int i = threadIdx.x; i < E; i += THREADS) {
        double P = 0.0;
        for (int b = 0; b < nblk; ++b)
            P += (double)partials[(int64_t)b * (E + 1) + i];
        acc += ((double)counts[i] / ((double)T * (double)k)) * (P / (double)T);
    }
    term[threadIdx.x] = acc;
    __syncthreads();
    for (int s = THREADS / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s)
            term[threadIdx.x] += term[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        double z = 0.0;
        for (int b = 0; b < nblk; ++b)
            z += (double)partials[(int64_t)b * (E + 1) + E];
        *aux = (float)((double)E * term[0]);
        *zloss = (float)(z / (double)T);
    }
}

}  // namespace

cudaError_t launch_losses(const moe_config &c, const int32_t *counts, const float *partials,
                          float *aux, float *zloss, cudaStream_t s)
{
    losses_kernel<<<1, THREADS, 0, s>>>(counts, partials, route_blocks(c), c.T > 0 ? c.T : 1,
                                        c.k, c.E, aux, zloss);
    return cudaGetLastError();
}

}  // namespace moe
