// Device helpers shared by the two routers (fp32 tiled, bf16 tensor-core).
#pragma once

#include "internal.cuh"

#include <math.h>

namespace moe {

struct RouteArgs {
    const void *x;
    const float *W_r, *logit_bias, *select_bias;
    int32_t *topk;
    float *gates, *partials, *logits_out, *scores_out;
    int T, d, E, k, score, renorm;
};

// Better of two (key, index) candidates: larger key, then lower index.
__device__ __forceinline__ bool better(float ka, int ia, float kb, int ib)
{
    return ka > kb || (ka == kb && ia < ib);
}


// Softmax / sigmoid, top-k, gates and loss partials of the TB tokens of one
// batch: lane L holds the logit of (token L / E_T, expert L % E_T).
// On return, lanes 0..E_T-1 hold in *pc the batch's sum of expert lane's
// probability (sigmoid: s / sum s) and every lane holds in *zc the batch's sum
// of lse^2, both summed over the tokens in a fixed order.  lbias and sbias
// are the logit and selection biases of expert lane % E_T (read only when
// the layer has them), loaded once by the caller.
template <int E_T>
__device__ __forceinline__ void small_epilogue(const RouteArgs &a, float z, int t0, int lane,
                                               bool renorm, float lbias, float sbias,
                                               float *pc_out, float *zc_out)
{
    const int E = a.E, T = a.T;
    const int gl = lane % E_T;
    const int gbase = lane - gl;
    const int t = t0 + lane / E_T;
    const bool tok = t < T;
    const bool valid = tok && gl < E;
    if (valid && a.logit_bias)
        z += lbias;
    float m = valid ? z : -INFINITY;
#pragma unroll
    for (int o = 1; o < E_T; o <<= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float ex = valid ? expf(z - m) : 0.f;
    float sum = ex;
#pragma unroll
    for (int o = 1; o < E_T; o <<= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float lse = m + logf(sum);
    float v, key;
    if (a.score == MOE_SCORE_SOFTMAX) {
        v = valid ? ex / sum : 0.f;
        key = valid ? z : -INFINITY;
    } else {
        v = valid ? 1.f / (1.f + expf(-z)) : 0.f;
        key = valid ? v + (a.select_bias ? sbias : 0.f) : -INFINITY;
    }
    float ssum = v;
#pragma unroll
    for (int o = 1; o < E_T; o <<= 1)
        ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
    if (valid && a.logits_out)
        a.logits_out[(int64_t)t * E + gl] = z;
    if (valid && a.scores_out)
        a.scores_out[(int64_t)t * E + gl] = v;
    // top-k: k rounds of a group argmax over (key, expert), lower index on
    // ties; lane gl == j keeps round j's expert and value, so the k outputs go
    // out from k lanes at once (the gate sum adds the values in round order)
    bool taken = false;
    int my_idx = 0;
    float my_v = 0.f, sel_sum = 0.f;
#pragma unroll 1
    for (int j = 0; j < a.k; ++j) {
        float bk = (!taken && valid) ? key : -INFINITY;
        int bi = (!taken && valid) ? gl : 0x7fffffff;
#pragma unroll
        for (int o = 1; o < E_T; o <<= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (better(ok, oi, bk, bi)) {
                bk = ok;
                bi = oi;
            }
        }
        const float bv = __shfl_sync(0xffffffffu, v, gbase + (bi < E_T ? bi : 0));
        if (gl == bi)
            taken = true;
        if (gl == j) {
            my_idx = bi;
            my_v = bv;
        }
        sel_sum += bv;
    }
    if (tok && gl < a.k) {
        a.topk[(int64_t)t * a.k + gl] = my_idx;
        a.gates[(int64_t)t * a.k + gl] = renorm ? my_v / sel_sum : my_v;
    }
    // loss sums over the batch's tokens (lanes of the same expert), fixed order
    float pc = valid ? (a.score == MOE_SCORE_SOFTMAX ? v : v / ssum) : 0.f;
    float zc = (tok && gl == 0) ? lse * lse : 0.f;
#pragma unroll
    for (int o = E_T; o < 32; o <<= 1)
        pc += __shfl_xor_sync(0xffffffffu, pc, o);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        zc += __shfl_xor_sync(0xffffffffu, zc, o);
    *pc_out = pc;
    *zc_out = zc;
}


}  // namespace moe
