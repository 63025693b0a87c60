// The fixed-order reduction of the loss partials, shared by the losses kernel
// and the capacity stage of the whole forward (which computes the losses in
// the same launch), so that both give the same bits.
//
// Page "Lab 18 - Mixture of experts", section 2:
//   L_aux = E * sum_i f_i P_i, f_i = counts_i / (T k), P_i = mean_t p_{t,i}
//   L_z   = (1/T) sum_t (logsumexp_i z_{t,i})^2
// "Lab 01", where to start step 3: f divides by the T k slots.
#pragma once

#include "internal.cuh"

namespace moe {

// Column col of the partials [rows][C] (expert col < E, or the lse^2 column
// col = E), summed by one warp: lane l adds rows l, l + 32, ... in order in
// double, then the 32 lane sums meet by xor shuffles in a fixed pattern.  The
// result (in every lane) does not depend on timing or on which warp runs it.
__device__ __forceinline__ double loss_column_sum(const float *partials, int rows, int C, int col,
                                                  int lane)
{
    double s = 0.0;
#pragma unroll 4
    for (int r = lane; r < rows; r += 32)
        s += (double)partials[(int64_t)r * C + col];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// The block's warps take the columns in turn (warp w: columns w, w + warps,
// ...); then one thread adds the E terms in expert order.  counts[e]: the
// assignments of expert e before capacity.  term: shared scratch [E + 1].
__device__ __forceinline__ void block_losses(const int32_t *counts, const float *partials,
                                             int rows, int T, int k, int E, float *aux,
                                             float *zloss, double *term)
{
    const int C = E + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = blockDim.x >> 5;
    for (int col = warp; col < C; col += warps) {
        const double s = loss_column_sum(partials, rows, C, col, lane);
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

}  // namespace moe
