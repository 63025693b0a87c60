// The fixed-order reduction of the loss partials, shared by the losses kernel
// and the capacity stage of the whole forward (which computes the losses in
// its two launches), so that both give the same bits.
//
// Page "Lab 18 - Mixture of experts", section 2:
//   L_aux = E * sum_i f_i P_i, f_i = counts_i / (T k), P_i = mean_t p_{t,i}
//   L_z   = (1/T) sum_t (logsumexp_i z_{t,i})^2
// "Lab 01", where to start step 3: f divides by the T k slots.
#pragma once

#include "internal.cuh"

namespace moe {

// The partials are [rows][C], C = E + 1 (expert columns, then the lse^2
// column).  Column col is summed in G = max(1, 1024 / C) row phases: phase g
// adds rows g, g + G, g + 2G, ... in order in double, and the G phase sums are
// then added in phase order.  G depends on C alone, so whichever threads or
// blocks compute the phases, the bits are the same.  Phase g of column col is
// work unit u = g * C + col (G * C <= kLossUnits units).
constexpr int kLossBatch = 32;   // loads in flight per unit

__host__ __device__ __forceinline__ int loss_phases(int C)
{
    return C >= kLossUnits ? 1 : kLossUnits / C;
}

// The phase sum of work unit u (u < loss_phases(C) * C).  Consecutive units
// read consecutive columns of one row (coalesced).
__device__ __forceinline__ double loss_phase_sum(const float *partials, int rows, int C, int u)
{
    const int G = loss_phases(C), col = u % C, g = u / C;
    double s = 0.0;
    for (int r0 = g; r0 < rows; r0 += kLossBatch * G) {
        float v[kLossBatch];
#pragma unroll
        for (int i = 0; i < kLossBatch; ++i) {
            const int r = r0 + i * G;
            v[i] = r < rows ? partials[(int64_t)r * C + col] : 0.f;
        }
        // adding +0 for the rows past the end leaves s unchanged (s >= 0)
#pragma unroll
        for (int i = 0; i < kLossBatch; ++i)
            s += (double)v[i];
    }
    return s;
}

// The loss terms from the phase sums ps[g * C + col] (ps in shared memory,
// complete): the G phase sums of a column added in phase order, then one
// thread adds the E terms in expert order.  term: shared scratch of kMaxE + 1
// doubles.  Every thread of the block calls it.
__device__ __forceinline__ void losses_from_phase_sums(const int32_t *counts, const double *ps,
                                                       int T, int k, int E, float *aux,
                                                       float *zloss, double *term)
{
    const int C = E + 1, G = loss_phases(C);
    for (int col = threadIdx.x; col < C; col += blockDim.x) {
        double s = 0.0;
        for (int g = 0; g < G; ++g)
            s += ps[g * C + col];
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

}  // namespace moe
