// Load balancing beyond the batch Switch loss: the sequence-wise balance loss
// and the auxiliary-loss-free bias step of DeepSeek-V3.
//
// Page "Lab 18 - Mixture of experts", section 2 (L_aux = E sum_i f_i P_i; the
// DeepSeek-V3 bias b_i on the selection scores only, moved after each step by
// a fixed amount against the expert's load; a small sequence-wise balance
// loss kept beside it); cs336 lecture 4 field map, "Training a router you
// cannot differentiate" (the balancing unit, batch or sequence, is where the
// variants differ; add gamma to underloaded experts, subtract it from
// overloaded ones).
//
// Both read what the forward already produced: the top-k indices, the
// route's loss partials (one row per 32 tokens: the per-expert probability
// sums and the lse^2 sum of those tokens) and the per-expert counts.
#include "internal.cuh"

namespace moe {
namespace {

// One block per sequence of L tokens (L a multiple of 32, so the sequence owns
// whole rows of the loss partials).  Counts: shared-memory integer histogram
// of the sequence's assignments.  P sums: the sequence's partial rows added in
// row order, in double.  Value: E sum_i (count_i / (L k)) (P_i / L), the terms
// added in expert order.
__global__ void __launch_bounds__(256)
seq_loss_kernel(const int32_t *__restrict__ topk, const float *__restrict__ partials, int E,
                int k, int L, float *__restrict__ per_seq)
{
    __shared__ int32_t cnt[kMaxE];
    __shared__ double term[kMaxE];
    const int b = blockIdx.x;
    for (int i = threadIdx.x; i < E; i += blockDim.x)
        cnt[i] = 0;
    __syncthreads();
    const int64_t a0 = (int64_t)b * L * k, a1 = a0 + (int64_t)L * k;
    for (int64_t a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
        const int e = topk[a];
        if (e >= 0 && e < E)
            atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    const int rows = L / kPartialTokens;
    const int64_t r0 = (int64_t)b * rows;
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        double P = 0.0;
        for (int r = 0; r < rows; ++r)
            P += (double)partials[(r0 + r) * (E + 1) + i];
        term[i] = ((double)cnt[i] / ((double)L * (double)k)) * (P / (double)L);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int i = 0; i < E; ++i)
            s += term[i];
        per_seq[b] = (float)((double)E * s);
    }
}

// Mean over the B sequences: a fixed-order reduction in one block.
__global__ void __launch_bounds__(256) seq_mean_kernel(const float *__restrict__ per_seq, int B,
                                                       float *loss)
{
    __shared__ double part[256];
    double s = 0.0;
    for (int b = threadIdx.x; b < B; b += 256)
        s += (double)per_seq[b];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        *loss = (float)(part[0] / (double)B);
}

// b_i -= gamma when E counts_i > T k (overloaded), += gamma when below, kept
// at exactly the balanced load: one fp32 addition, in place.
__global__ void bias_update_kernel(const int32_t *__restrict__ counts, int E, long long balanced,
                                   float gamma, float *bias)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= E)
        return;
    const long long load = (long long)E * counts[i];
    float b = bias[i];
    if (load > balanced)
        b = __fsub_rn(b, gamma);
    else if (load < balanced)
        b = __fadd_rn(b, gamma);
    bias[i] = b;
}

}  // namespace

cudaError_t launch_seq_loss(const moe_config &c, int L, const int32_t *topk,
                            const float *partials, float *per_seq, float *loss, cudaStream_t s)
{
    const int B = c.T / L;
    seq_loss_kernel<<<B, 256, 0, s>>>(topk, partials, c.E, c.k, L, per_seq);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess)
        return err;
    seq_mean_kernel<<<1, 256, 0, s>>>(per_seq, B, loss);
    return cudaGetLastError();
}

cudaError_t launch_bias_update(const moe_config &c, const int32_t *counts, float gamma,
                               float *bias, cudaStream_t s)
{
    bias_update_kernel<<<(unsigned)ceil_div(c.E, 256), 256, 0, s>>>(
        counts, c.E, (long long)c.T * c.k, gamma, bias);
    return cudaGetLastError();
}

}  // namespace moe
