// Expert FFNs in fp32 on the CUDA cores (the fp32 layer configuration).
//
// Page "Lab 18 - Mixture of experts", section 1: an expert is W2 gelu(W1 x)
// (two matrices) or W2 (silu(W1 x) * (W3 x)) (three matrices); tips: run each
// expert once on its gathered tokens.
//
// One tiled kernel serves both GEMMs of both expert kinds:
//   routed: rows of segment e of the permuted buffer against expert e's
//           weights; a 32-row tile never straddles segments because segments
//           start on multiples of 128 rows;
//   shared: all T token rows; GEMM1 puts shared expert s in columns
//           [s Fs, (s+1) Fs) of the hidden buffer, GEMM2 runs K over all
//           shared experts so their outputs are summed in the accumulator.
#include "internal.cuh"

#include <math.h>

namespace moe {
namespace {

constexpr int TILE = 32;
constexpr int KC = 32;
constexpr int THREADS = 256;   // 32 x 32 outputs, 4 per thread

enum { ACT_NONE = 0, ACT_GELU = 1, ACT_SWIGLU = 2 };

struct SimtGemm {
    const float *A;
    int64_t lda;
    int rows;                    // dense row count (shared)
    const int32_t *offsets;      // routed: segment table, E + 1 entries
    int E;
    const float *B, *B3;         // [groups][N][Kg]
    int64_t b_group_stride;
    int N, Kg;                   // N per group, K per group
    int k_groups;                // > 1: K runs over this many groups (A columns g*Kg + kk)
    float *C;
    int64_t ldc;
    int64_t c_group_col;         // dense, blockIdx.z = group: C column offset per group
    const int32_t *a_slot;       // non-null: row r of A is row a_slot[r] / a_div of the A
    int a_div;                   // tensor (a_slot[r] = assignment t k + j, -1 = none)
    // non-null: the combine's gate fused (routed GEMM2): kept row r of group e
    // (r - offsets[e] < kept[e]) goes, times gates[a], to row a = a_slot[r] of C
    const int32_t *kept;
    const float *gates;
};

__device__ __forceinline__ float gelu_erf(float u) { return 0.5f * u * (1.f + erff(u * 0.70710678118654752f)); }

template <int ACT>
__global__ void __launch_bounds__(THREADS) simt_gemm_kernel(SimtGemm p)
{
    __shared__ float As[TILE][KC + 1];
    __shared__ float Bs[TILE][KC + 1];
    __shared__ float B3s[TILE][KC + 1];
    const int n0 = blockIdx.x * TILE;
    const int m0 = blockIdx.y * TILE;
    int group = blockIdx.z;
    int row_end;
    if (p.offsets) {
        row_end = p.offsets[p.E];
        if (m0 >= row_end)
            return;
        int lo = 0, hi = p.E;   // last e with offsets[e] <= m0
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (p.offsets[mid] <= m0)
                lo = mid;
            else
                hi = mid;
        }
        group = lo;
    } else {
        row_end = p.rows;
        if (m0 >= row_end)
            return;
    }
    const int tx = threadIdx.x % TILE, ty = threadIdx.x / TILE;   // ty in 0..7
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc3[4] = {0.f, 0.f, 0.f, 0.f};
    const int groups_k = p.k_groups > 1 ? p.k_groups : 1;
    for (int gk = 0; gk < groups_k; ++gk) {
        const int bg = p.k_groups > 1 ? gk : group;
        const float *B = p.B + (int64_t)bg * p.b_group_stride;
        const float *B3 = p.B3 ? p.B3 + (int64_t)bg * p.b_group_stride : nullptr;
        const int64_t a_col0 = p.k_groups > 1 ? (int64_t)gk * p.Kg : 0;
        for (int k0 = 0; k0 < p.Kg; k0 += KC) {
            for (int i = threadIdx.x; i < TILE * KC; i += THREADS) {
                int r = i / KC, c = i % KC;
                int row = m0 + r, kk = k0 + c, n = n0 + r;
                int64_t arow = row;
                if (row < row_end && p.a_slot && !p.kept) {
                    const int a = p.a_slot[row];
                    arow = a >= 0 ? a / p.a_div : 0;
                }
                As[r][c] = (row < row_end && kk < p.Kg) ? p.A[arow * p.lda + a_col0 + kk] : 0.f;
                Bs[r][c] = (n < p.N && kk < p.Kg) ? B[(int64_t)n * p.Kg + kk] : 0.f;
                if (ACT == ACT_SWIGLU)
                    B3s[r][c] = (n < p.N && kk < p.Kg) ? B3[(int64_t)n * p.Kg + kk] : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int kk = 0; kk < KC; ++kk) {
                float b = Bs[tx][kk];
                float b3 = ACT == ACT_SWIGLU ? B3s[tx][kk] : 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float a = As[ty + 8 * i][kk];
                    acc[i] = fmaf(a, b, acc[i]);
                    if (ACT == ACT_SWIGLU)
                        acc3[i] = fmaf(a, b3, acc3[i]);
                }
            }
            __syncthreads();
        }
    }
    const int n = n0 + tx;
    if (n >= p.N)
        return;
    const int64_t col = (p.offsets ? 0 : (int64_t)blockIdx.z * p.c_group_col) + n;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int row = m0 + ty + 8 * i;
        if (row >= row_end)
            continue;
        float v = acc[i];
        if (ACT == ACT_GELU)
            v = gelu_erf(v);
        else if (ACT == ACT_SWIGLU)
            v = v / (1.f + expf(-v)) * acc3[i];
        if (p.kept) {   // gated: to the assignment's row, kept rows only
            if (row - p.offsets[group] >= p.kept[group])
                continue;
            const int a = p.a_slot[row];
            p.C[(int64_t)a * p.ldc + col] = p.gates[a] * v;
        } else {
            p.C[(int64_t)row * p.ldc + col] = v;
        }
    }
}

cudaError_t run(const SimtGemm &p, int act, int grid_m, int grid_z, cudaStream_t s)
{
    dim3 grid((unsigned)ceil_div(p.N, TILE), (unsigned)grid_m, (unsigned)grid_z);
    if (grid_m == 0)
        return cudaSuccess;
    if (act == ACT_GELU)
        simt_gemm_kernel<ACT_GELU><<<grid, THREADS, 0, s>>>(p);
    else if (act == ACT_SWIGLU)
        simt_gemm_kernel<ACT_SWIGLU><<<grid, THREADS, 0, s>>>(p);
    else
        simt_gemm_kernel<ACT_NONE><<<grid, THREADS, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_simt(const moe_config &c, const void *x_perm, const int32_t *offsets,
                            const int32_t *src_slot, const void *W1, const void *W3, const void *W2,
                            const void *x, const void *Ws1, const void *Ws3, const void *Ws2,
                            void *Y_perm, void *Y_sh, void *H, void *H_sh, cudaStream_t s,
                            const int32_t *kept, const float *gates, void *slot_out)
{
    const int act1 = c.act == MOE_ACT_SWIGLU ? ACT_SWIGLU : ACT_GELU;
    const int R = (int)perm_rows(c);
    const int gm = (int)ceil_div(R, TILE);
    cudaError_t err;
    // routed GEMM1: H = act(x_perm W1^T), or without x_perm the rows of x
    // through src_slot
    SimtGemm g1{static_cast<const float *>(x_perm ? x_perm : x), c.d, 0, offsets, c.E,
                static_cast<const float *>(W1), static_cast<const float *>(W3),
                (int64_t)c.d_ff * c.d, c.d_ff, c.d, 1, static_cast<float *>(H), c.d_ff, 0,
                x_perm ? nullptr : src_slot, c.k};
    if ((err = run(g1, act1, gm, 1, s)) != cudaSuccess)
        return err;
    // routed GEMM2: Y_perm = H W2^T, or gated rows to slot_out
    SimtGemm g2{static_cast<const float *>(H), c.d_ff, 0, offsets, c.E,
                static_cast<const float *>(W2), nullptr, (int64_t)c.d * c.d_ff, c.d, c.d_ff, 1,
                static_cast<float *>(slot_out ? slot_out : Y_perm), c.d, 0,
                slot_out ? src_slot : nullptr, c.k, slot_out ? kept : nullptr, gates};
    if ((err = run(g2, ACT_NONE, gm, 1, s)) != cudaSuccess)
        return err;
    if (c.n_shared > 0 && c.T > 0) {
        const int S = c.n_shared, Fs = c.d_ff_shared;
        const int gt = (int)ceil_div(c.T, TILE);
        SimtGemm s1{static_cast<const float *>(x), c.d, c.T, nullptr, 0,
                    static_cast<const float *>(Ws1), static_cast<const float *>(Ws3),
                    (int64_t)Fs * c.d, Fs, c.d, 1, static_cast<float *>(H_sh), (int64_t)S * Fs,
                    Fs};
        if ((err = run(s1, act1, gt, S, s)) != cudaSuccess)
            return err;
        SimtGemm s2{static_cast<const float *>(H_sh), (int64_t)S * Fs, c.T, nullptr, 0,
                    static_cast<const float *>(Ws2), nullptr, (int64_t)c.d * Fs, c.d, Fs, S,
                    static_cast<float *>(Y_sh), c.d, 0};
        if ((err = run(s2, ACT_NONE, gt, 1, s)) != cudaSuccess)
            return err;
    }
    return cudaSuccess;
}

}  // namespace moe
