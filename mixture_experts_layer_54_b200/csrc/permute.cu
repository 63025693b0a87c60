// Dispatch (permute token rows into expert-grouped order) and combine (gated
// sum of the expert outputs plus shared experts), both HBM-bound row copies.
//
// Page "Lab 18 - Mixture of experts": tips (gather each expert's tokens, run
// the expert once, index_add the gated result back), section 1 (y = sum of
// g_i FFN_i(x)), section 3 (a dropped slot contributes nothing; a fully
// dropped token passes through the residual).
//
// Dispatch reads each token row once and writes it to each of its kept
// destinations, so it moves T*d + N_kept*d elements.  Combine reads the k
// expert rows of a token, its shared-expert row (and residual) and writes y,
// summing in fp32 in slot order.  Rows move as 16-byte vectors; a block of 128
// threads owns one token per iteration of a grid-stride loop.
#include "internal.cuh"

namespace moe {
namespace {

constexpr int THREADS = 128;

__global__ void __launch_bounds__(THREADS)
dispatch_vec_kernel(const uint4 *x, int T, int k, int E, int nvec, const int32_t *topk,
                    const int32_t *pos, const uint8_t *keep, const int32_t *offsets,
                    uint4 *x_perm)
{
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        uint4 *dst[kMaxK];
        int nd = 0;
        for (int j = 0; j < k; ++j) {
            int64_t a = (int64_t)t * k + j;
            const int e = topk[a];
            if (keep[a] && e >= 0 && e < E) {
                int64_t row = (int64_t)offsets[e] + pos[a];
                dst[nd++] = x_perm + row * nvec;
            }
        }
        if (nd == 0)
            continue;
        const uint4 *src = x + (int64_t)t * nvec;
        for (int v = threadIdx.x; v < nvec; v += THREADS) {
            uint4 val = __ldg(src + v);
            for (int j = 0; j < nd; ++j)
                __stcs(dst[j] + v, val);
        }
    }
}

// 8 values of a 16-byte vector, widened to fp32
template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const uint4 &u, float *f)
    {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 p = __bfloat1622float2(h[i]);
            f[2 * i] = p.x;
            f[2 * i + 1] = p.y;
        }
    }
    __device__ static uint4 store(const float *f)
    {
        uint4 u;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        return u;
    }
};
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ static void load(const uint4 &u, float *f)
    {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
    __device__ static uint4 store(const float *f)
    {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};

template <typename Elem>
__global__ void __launch_bounds__(THREADS)
combine_vec_kernel(const uint4 *Y_perm, const uint4 *Y_sh, const float *gates,
                   const int32_t *topk, const int32_t *pos, const uint8_t *keep,
                   const int32_t *offsets, const uint4 *residual, uint4 *y, int T, int k,
                   int E, int nvec)
{
    constexpr int N = Vec<Elem>::N;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const uint4 *src[kMaxK];
        float g[kMaxK];
        int ns = 0;
        for (int j = 0; j < k; ++j) {
            int64_t a = (int64_t)t * k + j;
            const int e = topk[a];
            if (keep[a] && e >= 0 && e < E) {
                int64_t row = (int64_t)offsets[e] + pos[a];
                src[ns] = Y_perm + row * nvec;
                g[ns++] = gates[a];
            }
        }
        for (int v = threadIdx.x; v < nvec; v += THREADS) {
            float acc[N], f[N];
#pragma unroll
            for (int i = 0; i < N; ++i)
                acc[i] = 0.f;
            for (int j = 0; j < ns; ++j) {
                Vec<Elem>::load(__ldcs(src[j] + v), f);
#pragma unroll
                for (int i = 0; i < N; ++i)
                    acc[i] = fmaf(g[j], f[i], acc[i]);
            }
            if (Y_sh) {
                Vec<Elem>::load(__ldcs(Y_sh + (int64_t)t * nvec + v), f);
#pragma unroll
                for (int i = 0; i < N; ++i)
                    acc[i] += f[i];
            }
            if (residual) {
                Vec<Elem>::load(__ldg(residual + (int64_t)t * nvec + v), f);
#pragma unroll
                for (int i = 0; i < N; ++i)
                    acc[i] += f[i];
            }
            y[(int64_t)t * nvec + v] = Vec<Elem>::store(acc);
        }
    }
}

int grid_for(int T)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int g = sms * 16;
    return T < g ? T : g;
}

}  // namespace

cudaError_t launch_dispatch(const moe_config &c, const void *x, const int32_t *topk,
                            const int32_t *pos, const uint8_t *keep, const int32_t *offsets,
                            void *x_perm, cudaStream_t s)
{
    if (c.T == 0)
        return cudaSuccess;
    const int nvec = (int)((int64_t)c.d * dtype_bytes(c.dtype) / 16);
    dispatch_vec_kernel<<<grid_for(c.T), THREADS, 0, s>>>(
        static_cast<const uint4 *>(x), c.T, c.k, c.E, nvec, topk, pos, keep, offsets,
        static_cast<uint4 *>(x_perm));
    return cudaGetLastError();
}

cudaError_t launch_combine(const moe_config &c, const void *Y_perm, const void *Y_sh,
                           const float *gates, const int32_t *topk, const int32_t *pos,
                           const uint8_t *keep, const int32_t *offsets, const void *residual,
                           void *y, cudaStream_t s)
{
    if (c.T == 0)
        return cudaSuccess;
    const int nvec = (int)((int64_t)c.d * dtype_bytes(c.dtype) / 16);
    auto args = [&](auto kern) {
        kern<<<grid_for(c.T), THREADS, 0, s>>>(
            static_cast<const uint4 *>(Y_perm), static_cast<const uint4 *>(Y_sh), gates, topk,
            pos, keep, offsets, static_cast<const uint4 *>(residual), static_cast<uint4 *>(y),
            c.T, c.k, c.E, nvec);
    };
    if (c.dtype == MOE_DTYPE_BF16)
        args(combine_vec_kernel<__nv_bfloat16>);
    else
        args(combine_vec_kernel<float>);
    return cudaGetLastError();
}

}  // namespace moe
