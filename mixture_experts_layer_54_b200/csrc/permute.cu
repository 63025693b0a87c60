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
// summing in fp32 in slot order.  A warp owns one token at a time (grid-stride
// over tokens).  It looks up the slots of its next 32 / k tokens at once (lane
// l: slot l mod k of the (l / k)-th of them; two dependent loads, so they are
// paid once per 32 / k tokens) and hands each token its rows by shuffle; then
// the rows move as 16-byte vectors, several per lane in flight.
#include "internal.cuh"

namespace moe {
namespace {

constexpr int THREADS = 256;   // 8 warps, one token per warp at a time
constexpr int WARPS = THREADS / 32;
constexpr int UNROLL = 4;      // 16-byte vectors in flight per lane

// x_perm nullable: only the slot table.  src_slot nullable: row r of a kept
// slot gets its assignment t k + j.  zero_rows nullable: the row of a token
// with every slot dropped is set to zero there.
__global__ void __launch_bounds__(THREADS)
dispatch_vec_kernel(const uint4 *__restrict__ x, int T, int k, int E, int nvec,
                    const int32_t *__restrict__ topk, const int32_t *__restrict__ pos,
                    const uint8_t *__restrict__ keep, const int32_t *__restrict__ offsets,
                    uint4 *__restrict__ x_perm, int32_t *__restrict__ src_slot,
                    uint4 *__restrict__ zero_rows)
{
    pdl_wait();   // the slots come from the capacity stage
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * WARPS + (threadIdx.x >> 5);
    const int stride = gridDim.x * WARPS;
    const int tpb = 32 / k;   // tokens whose slots one lookup round covers
    for (int tb = gw; tb < T; tb += stride * tpb) {
        // the slots of this warp's next tpb tokens at once: lane l takes slot
        // l mod k of token tb + (l / k) stride
        int64_t mine = -1;
        {
            const int i = lane / k, j = lane % k, t = tb + i * stride;
            if (i < tpb && t < T) {
                const int64_t a = (int64_t)t * k + j;
                const int e = topk[a];
                if (keep[a] && e >= 0 && e < E)
                    mine = (int64_t)offsets[e] + pos[a];
            }
        }
        for (int ti = 0; ti < tpb; ++ti) {
            const int t = tb + ti * stride;
            if (t >= T)
                break;
            int64_t rows[kMaxK];   // rows[j], j < k: slot j's row or -1
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                rows[j] = __shfl_sync(0xffffffffu, mine, (ti * k + j) & 31);
            bool any = false;
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                any |= j < k && rows[j] >= 0;
            if (src_slot) {   // lane j records slot j's row
#pragma unroll
                for (int j = 0; j < kMaxK; ++j)
                    if (j == lane && j < k && rows[j] >= 0)
                        src_slot[rows[j]] = t * k + j;
            }
            if (!any) {
                if (zero_rows)
                    for (int v = lane; v < nvec; v += 32)
                        zero_rows[(int64_t)t * nvec + v] = make_uint4(0u, 0u, 0u, 0u);
                continue;
            }
            if (!x_perm)
                continue;
            const uint4 *src = x + (int64_t)t * nvec;
            for (int v0 = 0; v0 < nvec; v0 += 32 * UNROLL) {
                uint4 val[UNROLL];
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec)
                        val[u] = __ldcs(src + v);
                }
#pragma unroll
                for (int j = 0; j < kMaxK; ++j) {
                    if (j >= k || rows[j] < 0)
                        continue;
                    uint4 *dst = x_perm + rows[j] * nvec;
#pragma unroll
                    for (int u = 0; u < UNROLL; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < nvec)
                            __stcs(dst + v, val[u]);
                    }
                }
            }
        }
    }
}

// Dispatch fused into the expert GEMM: instead of copying rows, record for
// every kept assignment a = (t, j) that permuted row offsets[e] + pos[t, j]
// holds it (token a / k).  Padding rows keep the -1 the table was cleared to.
__global__ void dispatch_rows_kernel(const int32_t *__restrict__ topk,
                                     const int32_t *__restrict__ pos,
                                     const uint8_t *__restrict__ keep,
                                     const int32_t *__restrict__ offsets, int64_t A, int E,
                                     int32_t *__restrict__ src_slot)
{
    pdl_wait();   // the slots come from the capacity stage
    pdl_trigger();
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < A;
         a += (int64_t)gridDim.x * blockDim.x) {
        const int e = topk[a];
        if (keep[a] && e >= 0 && e < E)
            src_slot[offsets[e] + pos[a]] = (int32_t)a;
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

// KS = the layer's k (slots per token).  A chunk of U vectors per lane is
// loaded for every slot before any arithmetic (U * KS >= 8 loads in flight,
// at least two per slot), then summed in fp32 in slot order, then the shared
// experts and the residual.
template <typename Elem, int KS>
__global__ void __launch_bounds__(THREADS, 2)
combine_vec_kernel(const uint4 *__restrict__ Y_perm, const uint4 *__restrict__ Y_sh,
                   const float *__restrict__ gates, const int32_t *__restrict__ topk,
                   const int32_t *__restrict__ pos, const uint8_t *__restrict__ keep,
                   const int32_t *__restrict__ offsets, const uint4 *__restrict__ residual,
                   uint4 *__restrict__ y, int T, int E, int nvec)
{
    pdl_wait();   // the expert rows come from the expert GEMMs
    pdl_trigger();
    constexpr int N = Vec<Elem>::N;
    // 16-byte vectors per slot row and lane in flight (k = 1: 4, so that the
    // shared-expert and residual rows fit beside them in 128 registers)
    constexpr int U = KS >= 4 ? 2 : (KS == 1 ? 4 : 8 / KS);
    constexpr int TPB = 32 / KS;   // tokens whose slots one lookup round covers
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * WARPS + (threadIdx.x >> 5);
    const int stride = gridDim.x * WARPS;
    for (int tb = gw; tb < T; tb += stride * TPB) {
        // the slots of this warp's next TPB tokens at once: lane l takes slot
        // l mod KS of token tb + (l / KS) stride (the row or -1, and the gate)
        int64_t mine = -1;
        float gmine = 0.f;
        {
            const int i = lane / KS, j = lane % KS, t = tb + i * stride;
            if (i < TPB && t < T) {
                const int64_t a = (int64_t)t * KS + j;
                const int e = topk[a];
                if (keep[a] && e >= 0 && e < E)
                    mine = (int64_t)offsets[e] + pos[a];
                gmine = gates[a];
            }
        }
        for (int ti = 0; ti < TPB; ++ti) {
            const int t = tb + ti * stride;
            if (t >= T)
                break;
            int64_t rows[KS];
            float g[KS];
#pragma unroll
            for (int j = 0; j < KS; ++j) {
                rows[j] = __shfl_sync(0xffffffffu, mine, ti * KS + j);
                g[j] = __shfl_sync(0xffffffffu, gmine, ti * KS + j);
            }
            const uint4 *extra[2] = {Y_sh ? Y_sh + (int64_t)t * nvec : nullptr,
                                     residual ? residual + (int64_t)t * nvec : nullptr};
            for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
                // the slot rows and the shared-expert / residual rows in flight together
                uint4 raw[KS][U], ex[2][U];
#pragma unroll
                for (int j = 0; j < KS; ++j)
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int v = v0 + u * 32 + lane;
                        raw[j][u] = (rows[j] >= 0 && v < nvec) ? __ldcs(Y_perm + rows[j] * nvec + v)
                                                               : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                for (int q = 0; q < 2; ++q)
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int v = v0 + u * 32 + lane;
                        ex[q][u] = (extra[q] && v < nvec) ? __ldcs(extra[q] + v)
                                                          : make_uint4(0u, 0u, 0u, 0u);
                    }
                float acc[U][N];
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int i = 0; i < N; ++i)
                        acc[u][i] = 0.f;
                // slots in order, then the shared experts, then the residual
#pragma unroll
                for (int j = 0; j < KS; ++j) {
                    if (rows[j] < 0)
                        continue;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        float f[N];
                        Vec<Elem>::load(raw[j][u], f);
#pragma unroll
                        for (int i = 0; i < N; ++i)
                            acc[u][i] = fmaf(g[j], f[i], acc[u][i]);
                    }
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    if (!extra[q])
                        continue;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < nvec) {
                            float f[N];
                            Vec<Elem>::load(ex[q][u], f);
#pragma unroll
                            for (int i = 0; i < N; ++i)
                                acc[u][i] += f[i];
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec)
                        y[(int64_t)t * nvec + v] = Vec<Elem>::store(acc[u]);
                }
            }
        }
    }
}

// The combine after the gate was applied in the expert GEMM: the k gated rows
// of a token are contiguous (Y_slot row t k + j); their kept ones are summed
// in fp32 in slot order, then the shared experts and the residual.
template <typename Elem, int KS>
__global__ void __launch_bounds__(THREADS)
combine_slots_kernel(const uint4 *__restrict__ Y_slot, const uint4 *__restrict__ Y_sh,
                     const uint8_t *__restrict__ keep, const uint4 *__restrict__ residual,
                     uint4 *__restrict__ y, int T, int nvec)
{
    pdl_wait();   // the gated rows come from the expert GEMM
    pdl_trigger();
    constexpr int N = Vec<Elem>::N;
    constexpr int U = KS >= 4 ? 2 : 8 / KS;
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * WARPS + (threadIdx.x >> 5);
    for (int t = gw; t < T; t += gridDim.x * WARPS) {
        const int mk = lane < KS ? keep[(int64_t)t * KS + lane] : 0;
        bool kp[KS];
#pragma unroll
        for (int j = 0; j < KS; ++j)
            kp[j] = __shfl_sync(0xffffffffu, mk, j) != 0;
        const uint4 *rows = Y_slot + (int64_t)t * KS * nvec;
        for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
            uint4 raw[KS][U];
#pragma unroll
            for (int j = 0; j < KS; ++j)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    raw[j][u] = (kp[j] && v < nvec) ? __ldcs(rows + (int64_t)j * nvec + v)
                                                    : make_uint4(0u, 0u, 0u, 0u);
                }
            float acc[U][N];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < N; ++i)
                    acc[u][i] = 0.f;
#pragma unroll
            for (int j = 0; j < KS; ++j) {
                if (!kp[j])
                    continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float f[N];
                    Vec<Elem>::load(raw[j][u], f);
#pragma unroll
                    for (int i = 0; i < N; ++i)
                        acc[u][i] += f[i];
                }
            }
            const uint4 *extra[2] = {Y_sh ? Y_sh + (int64_t)t * nvec : nullptr,
                                     residual ? residual + (int64_t)t * nvec : nullptr};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                if (!extra[q])
                    continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) {
                        float f[N];
                        Vec<Elem>::load(__ldcs(extra[q] + v), f);
#pragma unroll
                        for (int i = 0; i < N; ++i)
                            acc[u][i] += f[i];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec)
                    y[(int64_t)t * nvec + v] = Vec<Elem>::store(acc[u]);
            }
        }
    }
}

// As many blocks of 8 token-warps as are resident at once, fewer for small T.
template <typename K>
int grid_for(K kernel, int T)
{
    const int sms = device_sms();
    int per_sm = 1;
    if (cached_blocks_per_sm((const void *)kernel, THREADS, 0, &per_sm) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int need = (T + WARPS - 1) / WARPS;
    const int g = sms * per_sm;
    return need < g ? need : g;
}

}  // namespace

cudaError_t launch_dispatch(const moe_config &c, const void *x, const int32_t *topk,
                            const int32_t *pos, const uint8_t *keep, const int32_t *offsets,
                            void *x_perm, cudaStream_t s, int32_t *src_slot, void *zero_rows)
{
    if (c.T == 0)
        return cudaSuccess;
    const int nvec = (int)((int64_t)c.d * dtype_bytes(c.dtype) / 16);
    return launch_pdl(dispatch_vec_kernel, dim3(grid_for(dispatch_vec_kernel, c.T)), dim3(THREADS),
                      0, s, static_cast<const uint4 *>(x), c.T, c.k, c.E, nvec, topk, pos, keep,
                      offsets, static_cast<uint4 *>(x_perm), src_slot,
                      static_cast<uint4 *>(zero_rows));
}

cudaError_t launch_dispatch_rows(const moe_config &c, const int32_t *topk, const int32_t *pos,
                                 const uint8_t *keep, const int32_t *offsets, int32_t *src_slot,
                                 cudaStream_t s)
{
    // every entry -1 (all bytes 0xFF), then the kept rows
    cudaError_t err = cudaMemsetAsync(src_slot, 0xFF, sizeof(int32_t) * (size_t)perm_rows(c), s);
    if (err != cudaSuccess || c.T == 0)
        return err;
    const int64_t A = (int64_t)c.T * c.k;
    const int blocks = (int)(ceil_div(A, 256) < 1184 ? ceil_div(A, 256) : 1184);
    return launch_pdl(dispatch_rows_kernel, dim3(blocks), dim3(256), 0, s, topk, pos, keep,
                      offsets, A, c.E, src_slot);
}

cudaError_t launch_combine_slots(const moe_config &c, const void *Y_slot, const void *Y_sh,
                                 const uint8_t *keep, const void *residual, void *y,
                                 cudaStream_t s)
{
    if (c.T == 0)
        return cudaSuccess;
    const int nvec = (int)((int64_t)c.d * dtype_bytes(c.dtype) / 16);
    cudaError_t err = cudaSuccess;
    auto args = [&](auto kern) {
        err = launch_pdl(kern, dim3(grid_for(kern, c.T)), dim3(THREADS), 0, s,
                         static_cast<const uint4 *>(Y_slot), static_cast<const uint4 *>(Y_sh),
                         keep, static_cast<const uint4 *>(residual), static_cast<uint4 *>(y),
                         c.T, nvec);
    };
    auto by_k = [&](auto elem) {
        using El = decltype(elem);
        switch (c.k) {
        case 1: args(combine_slots_kernel<El, 1>); break;
        case 2: args(combine_slots_kernel<El, 2>); break;
        case 3: args(combine_slots_kernel<El, 3>); break;
        case 4: args(combine_slots_kernel<El, 4>); break;
        case 5: args(combine_slots_kernel<El, 5>); break;
        case 6: args(combine_slots_kernel<El, 6>); break;
        case 7: args(combine_slots_kernel<El, 7>); break;
        default: args(combine_slots_kernel<El, 8>); break;
        }
    };
    if (c.dtype == MOE_DTYPE_BF16)
        by_k(__nv_bfloat16());
    else
        by_k(float());
    return err;
}

cudaError_t launch_combine(const moe_config &c, const void *Y_perm, const void *Y_sh,
                           const float *gates, const int32_t *topk, const int32_t *pos,
                           const uint8_t *keep, const int32_t *offsets, const void *residual,
                           void *y, cudaStream_t s)
{
    if (c.T == 0)
        return cudaSuccess;
    const int nvec = (int)((int64_t)c.d * dtype_bytes(c.dtype) / 16);
    cudaError_t err = cudaSuccess;
    auto args = [&](auto kern) {
        err = launch_pdl(kern, dim3(grid_for(kern, c.T)), dim3(THREADS), 0, s,
                         static_cast<const uint4 *>(Y_perm), static_cast<const uint4 *>(Y_sh),
                         gates, topk, pos, keep, offsets, static_cast<const uint4 *>(residual),
                         static_cast<uint4 *>(y), c.T, c.E, nvec);
    };
    auto by_k = [&](auto elem) {
        using El = decltype(elem);
        switch (c.k) {
        case 1: args(combine_vec_kernel<El, 1>); break;
        case 2: args(combine_vec_kernel<El, 2>); break;
        case 3: args(combine_vec_kernel<El, 3>); break;
        case 4: args(combine_vec_kernel<El, 4>); break;
        case 5: args(combine_vec_kernel<El, 5>); break;
        case 6: args(combine_vec_kernel<El, 6>); break;
        case 7: args(combine_vec_kernel<El, 7>); break;
        default: args(combine_vec_kernel<El, 8>); break;
        }
    };
    if (c.dtype == MOE_DTYPE_BF16)
        by_k(__nv_bfloat16());
    else
        by_k(float());
    return err;
}

}  // namespace moe
