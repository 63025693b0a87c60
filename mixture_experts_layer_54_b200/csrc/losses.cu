// Balancing losses from the router's per-block partial sums and the
// capacity stage's counts, reduced in a fixed order (deterministic).
//
// Page "Lab 18 - Mixture of experts", section 2:
//   L_aux = E * sum_i f_i P_i, f_i = counts_i / (T k), P_i = mean_t p_{t,i}
//   L_z   = (1/T) sum_t (logsumexp_i z_{t,i})^2
// "Lab 01", where to start step 3: f divides by the T k slots.
#include "internal.cuh"
#include "losses_common.cuh"

namespace moe {
namespace {

constexpr int THREADS = kLossUnits;

// One block: thread u computes the phase sum of work unit u (losses_common.cuh)
// into shared memory, then the terms in the fixed order of
// losses_from_phase_sums: the same bits as the forward's capacity stage.
__global__ void __launch_bounds__(THREADS)
losses_kernel(const int32_t *__restrict__ counts, const float *__restrict__ partials, int rows,
              int T, int k, int E, float *aux, float *zloss)
{
    __shared__ double term[kMaxE + 1];
    __shared__ double ps[kLossUnits];
    pdl_wait();   // counts and partials come from the capacity and route stages
    pdl_trigger();
    const int C = E + 1;
    if ((int)threadIdx.x < loss_phases(C) * C)
        ps[threadIdx.x] = loss_phase_sum(partials, rows, C, threadIdx.x);
    __syncthreads();
    losses_from_phase_sums(counts, ps, T, k, E, aux, zloss, term);
}

}  // namespace

cudaError_t launch_losses(const moe_config &c, const int32_t *counts, const float *partials,
                          float *aux, float *zloss, cudaStream_t s)
{
    return launch_pdl(losses_kernel, dim3(1), dim3(THREADS), 0, s, counts, partials,
                      partial_rows(c), c.T > 0 ? c.T : 1, c.k, c.E, aux, zloss);
}

}  // namespace moe
