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

// Column c of the partials (expert c < E, or the lse^2 column c = E) is
// summed by ny threads, each over rows y, y + ny, ... in order, then the ny
// partial sums in order: a fixed reduction tree, so the result does not depend
// on timing.
__global__ void __launch_bounds__(THREADS)
losses_kernel(const int32_t *counts, const float *partials, int rows, int T, int k, int E,
              float *aux, float *zloss)
{
    extern __shared__ double part[];   // [ny][C]
    __shared__ double term[kMaxE + 1];
    const int C = E + 1;
    const int ny = THREADS / C;
    const int tx = threadIdx.x % C, ty = threadIdx.x / C;
    if (ty < ny) {
        double s = 0.0;
        for (int r = ty; r < rows; r += ny)
            s += (double)partials[(int64_t)r * C + tx];
        part[ty * C + tx] = s;
    }
    __syncthreads();
    if (threadIdx.x < C) {
        double s = 0.0;
        for (int y = 0; y < ny; ++y)
            s += part[y * C + threadIdx.x];
        term[threadIdx.x] = threadIdx.x < E
                                ? ((double)counts[threadIdx.x] / ((double)T * (double)k)) *
                                      (s / (double)T)
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
    const int C = c.E + 1;
    const size_t smem = sizeof(double) * (THREADS / C) * C;
    losses_kernel<<<1, THREADS, smem, s>>>(counts, partials, partial_rows(c),
                                           c.T > 0 ? c.T : 1, c.k, c.E, aux, zloss);
    return cudaGetLastError();
}

}  // namespace moe
