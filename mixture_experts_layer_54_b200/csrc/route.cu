// Router stage: z = x W_r in fp32, scores, top-k, gates and the per-block
// partial sums of the balancing losses, one kernel.
//
// Page "Lab 18 - Mixture of experts", section 1 (z = x W_r, p = softmax(z),
// gate values: renormalized for k > 1, raw for k = 1; sigmoid scores for the
// DeepSeek-V3 style), section 2 (P_i for the load-balance loss, logsumexp for
// the z-loss, selection-only bias); "Lab 01" traps (stable softmax, ties to
// the lower expert index).
//
// This file holds the fp32 router (bf16 layers use the tensor-core router in
// route_tc.cu): one block = 32 tokens; phase 1 is a register-tiled fp32 GEMM of
// the block's x rows against W_r, staged through shared memory in chunks of 32
// columns of d; phase 2 gives each warp whole tokens (the E logits of a token
// spread over the lanes, max / sum / argmax as warp shuffles); phase 3 sums
// each expert's probability over the block's 32 tokens in token order, so the loss
// partials are deterministic.
#include "internal.cuh"
#include "route_common.cuh"

#include <math.h>

namespace moe {
namespace {

constexpr int RT = kRouteTokens;   // tokens per block
constexpr int KC = 32;             // d columns per chunk
constexpr int THREADS = 256;

template <typename T> __device__ __forceinline__ float ld_f32(const T *p, int64_t i);
template <> __device__ __forceinline__ float ld_f32<float>(const float *p, int64_t i) { return p[i]; }
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i)
{
    return __bfloat162float(p[i]);
}

template <typename Tin, int TM, int TN>
__global__ void __launch_bounds__(THREADS) route_kernel(RouteArgs a)
{
    extern __shared__ float smem[];
    const int E = a.E, d = a.d, T = a.T;
    const int NX = (E + TN - 1) / TN;          // threads along experts
    const int NY = RT / TM;                     // threads along tokens
    const int Epad = NX * TN;
    float *xs = smem;                           // [RT][KC + 1]
    float *wsm = xs + RT * (KC + 1);            // [KC][Epad]
    float *zs = wsm + KC * Epad;                // [RT][E + 1]
    float *lse_s = zs + RT * (E + 1);           // [RT]

    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * RT;
    const Tin *x = static_cast<const Tin *>(a.x);
    const int tx = tid % NX, ty = tid / NX;
    const bool computes = ty < NY;

    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j)
            acc[i][j] = 0.f;

    for (int c0 = 0; c0 < d; c0 += KC) {
        for (int idx = tid; idx < RT * KC; idx += THREADS) {
            int r = idx / KC, c = idx % KC;
            int t = t0 + r, col = c0 + c;
            xs[r * (KC + 1) + c] = (t < T && col < d) ? ld_f32(x, (int64_t)t * d + col) : 0.f;
        }
        for (int idx = tid; idx < KC * Epad; idx += THREADS) {
            int r = idx / Epad, e = idx % Epad;
            int col = c0 + r;
            wsm[idx] = (col < d && e < E) ? a.W_r[(int64_t)col * E + e] : 0.f;
        }
        __syncthreads();
        if (computes) {
#pragma unroll 8
            for (int kk = 0; kk < KC; ++kk) {
                float xv[TM], wv[TN];
#pragma unroll
                for (int i = 0; i < TM; ++i)
                    xv[i] = xs[(ty + i * NY) * (KC + 1) + kk];
#pragma unroll
                for (int j = 0; j < TN; ++j)
                    wv[j] = wsm[kk * Epad + tx + j * NX];
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j)
                        acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
            }
        }
        __syncthreads();
    }
    if (computes) {
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) {
                int e = tx + j * NX;
                if (e < E)
                    zs[(ty + i * NY) * (E + 1) + e] =
                        acc[i][j] + (a.logit_bias ? a.logit_bias[e] : 0.f);
            }
    }
    __syncthreads();

    // ---- phase 2: one warp per token ----
    const int lane = tid & 31, warp = tid >> 5;
    const int per_lane = (E + 31) / 32;        // <= 8
    const bool renorm = a.renorm < 0 ? (a.k > 1) : (a.renorm != 0);
    for (int tl = warp; tl < RT; tl += THREADS / 32) {
        const int t = t0 + tl;
        float *zrow = zs + tl * (E + 1);
        if (t >= T) {
            for (int e = lane; e < E; e += 32)
                zrow[e] = 0.f;
            if (lane == 0)
                lse_s[tl] = 0.f;
            continue;
        }
        float z[8], v[8], key[8];
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int e = lane + 32 * i;
            z[i] = (i < per_lane && e < E) ? zrow[e] : -INFINITY;
            m = fmaxf(m, z[i]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int e = lane + 32 * i;
            if (i < per_lane && e < E)
                sum += expf(z[i] - m);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float lse = m + logf(sum);
        float ssum = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int e = lane + 32 * i;
            bool ok = i < per_lane && e < E;
            if (a.score == MOE_SCORE_SOFTMAX) {
                v[i] = ok ? expf(z[i] - m) / sum : 0.f;
                key[i] = ok ? z[i] : -INFINITY;      // same order as p
            } else {
                v[i] = ok ? 1.f / (1.f + expf(-z[i])) : 0.f;
                key[i] = ok ? v[i] + (a.select_bias ? a.select_bias[e] : 0.f) : -INFINITY;
                ssum += v[i];
            }
        }
        if (a.score == MOE_SCORE_SIGMOID) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
        }
        if (a.logits_out || a.scores_out) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int e = lane + 32 * i;
                if (i < per_lane && e < E) {
                    if (a.logits_out)
                        a.logits_out[(int64_t)t * E + e] = z[i];
                    if (a.scores_out)
                        a.scores_out[(int64_t)t * E + e] = v[i];
                }
            }
        }
        // top-k: k rounds of a warp argmax over (key, index)
        unsigned taken = 0;
        int sel_idx[kMaxK];
        float sel_v[kMaxK];
        float sel_sum = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            sel_idx[j] = 0;
            sel_v[j] = 0.f;
            if (j >= a.k)
                continue;
            float bk = -INFINITY;
            int bi = 0x7fffffff;
            float bv = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int e = lane + 32 * i;
                if (i < per_lane && e < E && !((taken >> i) & 1u) && better(key[i], e, bk, bi)) {
                    bk = key[i];
                    bi = e;
                    bv = v[i];
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ok = __shfl_xor_sync(0xffffffffu, bk, o);
                int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                if (better(ok, oi, bk, bi)) {
                    bk = ok;
                    bi = oi;
                    bv = ov;
                }
            }
            if ((bi & 31) == lane)
                taken |= 1u << (bi >> 5);
            sel_idx[j] = bi;
            sel_v[j] = bv;
            sel_sum += bv;
        }
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                if (j < a.k) {
                    a.topk[(int64_t)t * a.k + j] = sel_idx[j];
                    a.gates[(int64_t)t * a.k + j] = renorm ? sel_v[j] / sel_sum : sel_v[j];
                }
            lse_s[tl] = lse * lse;
        }
        // probability mass entering P_i (sigmoid: s_i / sum_j s_j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int e = lane + 32 * i;
            if (i < per_lane && e < E)
                zrow[e] = a.score == MOE_SCORE_SOFTMAX ? v[i] : v[i] / ssum;
        }
    }
    __syncthreads();

    // ---- phase 3: sums over the block's row of 32 tokens, in token order ----
    constexpr int G = RT / kPartialTokens;
    const int rows = (T + kPartialTokens - 1) / kPartialTokens;
    for (int i = tid; i < G * (E + 1); i += THREADS) {
        const int g = i / (E + 1), e = i % (E + 1);
        const int row = blockIdx.x * G + g;
        if (row >= rows)
            continue;
        float s = 0.f;
        for (int tl = g * kPartialTokens; tl < (g + 1) * kPartialTokens; ++tl)
            s += e < E ? zs[tl * (E + 1) + e] : lse_s[tl];
        a.partials[(int64_t)row * (E + 1) + e] = s;
    }
}

template <typename Tin, int TM, int TN>
cudaError_t launch_tiled(const RouteArgs &a, int blocks, cudaStream_t s)
{
    const int NX = (a.E + TN - 1) / TN;
    const int Epad = NX * TN;
    size_t smem = sizeof(float) * (RT * (KC + 1) + KC * Epad + RT * (a.E + 1) + RT);
    auto kern = route_kernel<Tin, TM, TN>;
    cudaError_t err = raise_smem_limit((const void *)kern, (int)smem);
    if (err != cudaSuccess)
        return err;
    kern<<<blocks, THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_typed(const RouteArgs &a, int blocks, cudaStream_t s)
{
    // thread tile: (32 / TM) token rows x ceil(E / TN) expert columns <= 256 threads
    if (a.E <= 8)
        return launch_tiled<Tin, 1, 1>(a, blocks, s);
    if (a.E <= 32)
        return launch_tiled<Tin, 4, 1>(a, blocks, s);
    if (a.E <= 64)
        return launch_tiled<Tin, 4, 2>(a, blocks, s);
    if (a.E <= 128)
        return launch_tiled<Tin, 4, 4>(a, blocks, s);
    return launch_tiled<Tin, 4, 8>(a, blocks, s);
}

}  // namespace

cudaError_t launch_route(const moe_config &c, const void *x, const float *W_r,
                         const float *logit_bias, const float *select_bias,
                         int32_t *topk, float *gates, float *partials,
                         float *logits_out, float *scores_out, cudaStream_t s)
{
    if (c.T == 0)
        return cudaSuccess;
    RouteArgs a{x, W_r, logit_bias, select_bias, topk, gates, partials, logits_out,
                scores_out, c.T, c.d, c.E, c.k, c.score, c.renorm};
    const int blocks = route_blocks(c);
    if (c.dtype == MOE_DTYPE_BF16)
        return launch_typed<__nv_bfloat16>(a, blocks, s);
    return launch_typed<float>(a, blocks, s);
}

}  // namespace moe
