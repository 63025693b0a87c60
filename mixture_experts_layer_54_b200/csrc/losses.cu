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

constexpr int THREADS = 1024;
constexpr int WARPS = THREADS / 32;

// Column c of the partials (expert c < E, or the lse^2 column c = E) belongs
// to warp c mod 32; lane l sums rows l, l + 32, ... in order (double), then
// the 32 lane sums meet by xor shuffles in a fixed pattern: a fixed reduction
// tree, so the result does not depend on timing.
__global__ void __launch_bounds__(THREADS)
losses_kernel(const int32_t *__restrict__ counts, const float *__restrict__ partials, int rows,
              int T, int k, int E, float *aux, float *zloss)
{
    __shared__ double term[kMaxE + 1];
    const int C = E + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int col = warp; col < C; col += WARPS) {
        double s = 0.0;
#pragma unroll 4
        for (int r = lane; r < rows; r += 32)
            s += (double)__ldg(partials + (int64_t)r * C + col);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0)
            term[col] = col < E ? ((double)counts[col] / ((double)T * (double)k)) * (s / (double)T)
                                : s / (double)T;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0;
        for (int i = 0; i < E; ++i)
            a += term[i];
        *aux = (float)((double)E * a);
        *zloss = (float)term[E];
    }
}

}  // namespace

cudaError_t launch_losses(const moe_config &c, const int32_t *counts, const float *partials,
                          float *aux, float *zloss, cudaStream_t s)
{
    losses_kernel<<<1, THREADS, 0, s>>>(counts, partials, partial_rows(c), c.T > 0 ? c.T : 1,
                                        c.k, c.E, aux, zloss);
    return cudaGetLastError();
}

}  // namespace moe
