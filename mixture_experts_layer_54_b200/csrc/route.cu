// Router stage: z = x W_r in fp32, scores, top-k, gates and the per-block
// partial sums of the balancing losses, one kernel.
//
// Page "Lab 18 - Mixture of experts", section 1 (z = x W_r, p = softmax(z),
// gate values: renormalized for k > 1, raw for k = 1; sigmoid scores for the
// DeepSeek-V3 style), section 2 (P_i for the load-balance loss, logsumexp for
// the z-loss, selection-only bias); "Lab 01" traps (stable softmax, ties to
// the lower expert index).
//
// Two kernels.  The tiled one (any E, any d): one block = 32 tokens; phase 1 is
// a register-tiled fp32 GEMM of the block's x rows against W_r, staged through
// shared memory in chunks of 32 columns of d; phase 2 gives each warp whole
// tokens (the E logits of a token spread over the lanes, max / sum / argmax as
// warp shuffles); phase 3 sums each expert's probability over every 4 tokens
// in token order, so the loss partials are deterministic.  The small-E one is
// described at its definition below.
#include "internal.cuh"

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

    // ---- phase 3: sums over each row of 4 tokens, in token order ----
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

// ---------------------------------------------------------------------------
// Small-E variant (E <= 8 on rows of up to 4096 bf16): every compute thread
// keeps its slice of W_r (NV vectors of CPT columns, all E_T experts) in
// registers for the whole kernel, so the fp32 FMAs read only x.  x arrives by
// TMA: batches of TB = 32 / E_T consecutive token rows are one contiguous
// block of memory, copied by thread 0 with one bulk copy into a ring of
// shared-memory stages; each warp releases a stage through an mbarrier when it
// is done with it.  A batch gives each lane 32 partial
// logits; one butterfly reduce-scatter (31 shuffles) leaves lane L with its
// warp's sum for (token L / E_T, expert L % E_T).  After every 8 batches the
// 8 warps' sums meet in shared memory and each warp finishes one batch's
// tokens.  Batches are spread over a persistent grid; one loss-partials row
// per 4 tokens.

// v[0..N) summed over the warp: the N values are split over the lanes by
// halving exchanges, then the lanes that share a value finish with xor sums.
// Lane L returns the total of v[L / (32 / N)].
template <int N>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[N], int lane)
{
    int n = N;
#pragma unroll
    for (int o = 16; o >= 32 / N; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            if (i < n / 2) {
                const float send = upper ? v[i] : v[i + n / 2];
                const float keep = upper ? v[i + n / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        n >>= 1;
    }
    float r = v[0];
#pragma unroll
    for (int o = 32 / N / 2; o >= 1; o >>= 1)
        r += __shfl_xor_sync(0xffffffffu, r, o);
    return r;
}

template <int CPT> struct XVec;
template <> struct XVec<8> {   // 8 bf16 = 16 bytes
    __device__ static void load(const uint8_t *p, float *f)
    {
        uint4 u = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 q = __bfloat1622float2(h[i]);
            f[2 * i] = q.x;
            f[2 * i + 1] = q.y;
        }
    }
};
template <> struct XVec<4> {   // 4 bf16 = 8 bytes
    __device__ static void load(const uint8_t *p, float *f)
    {
        uint2 u = *reinterpret_cast<const uint2 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float2 q = __bfloat1622float2(h[i]);
            f[2 * i] = q.x;
            f[2 * i + 1] = q.y;
        }
    }
};

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bounded wait on an mbarrier phase (about 2 s of wall clock); false on expiry
// or, when `abort` is given, as soon as another thread has given up.
__device__ __noinline__ bool route_wait(uint32_t bar, uint32_t parity, volatile int *abort)
{
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok)
            return true;
        if ((i & 63u) == 0) {
            if (abort && *abort)
                return false;
            uint64_t now;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
            if (i == 0) {
                t0 = now;
            } else if (now - t0 > 2000000000ull) {
                if (abort)
                    *abort = 1;
                return false;
            }
        }
    }
}

constexpr int RING_BYTES = 192 * 1024;   // shared-memory ring for the x batches
constexpr int MAX_STAGES = 6;

__device__ __forceinline__ void mbar_init_route(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_route(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Softmax / sigmoid, top-k, gates and loss partials of the TB tokens of one
// batch: lane L holds the logit of (token L / E_T, expert L % E_T).
template <int E_T>
__device__ __forceinline__ void small_epilogue(const RouteArgs &a, float z, int t0, int lane,
                                               bool renorm)
{
    constexpr int TB = 32 / E_T;
    (void)TB;
    const int E = a.E, T = a.T;
    const int gl = lane % E_T;
    const int gbase = lane - gl;
    const int t = t0 + lane / E_T;
    const bool tok = t < T;
    const bool valid = tok && gl < E;
    if (valid && a.logit_bias)
        z += a.logit_bias[gl];
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
        key = valid ? v + (a.select_bias ? a.select_bias[gl] : 0.f) : -INFINITY;
    }
    float ssum = v;
#pragma unroll
    for (int o = 1; o < E_T; o <<= 1)
        ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
    if (valid && a.logits_out)
        a.logits_out[(int64_t)t * E + gl] = z;
    if (valid && a.scores_out)
        a.scores_out[(int64_t)t * E + gl] = v;
    // top-k: k rounds of a group argmax over (key, expert), lower index on ties
    bool taken = false;
    int sel_idx[kMaxK];
    float sel_v[kMaxK];
    float sel_sum = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        sel_idx[j] = 0;
        sel_v[j] = 0.f;
        if (j < a.k) {
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
            sel_idx[j] = bi;
            sel_v[j] = bv;
            sel_sum += bv;
        }
    }
    if (tok && gl == 0) {
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j < a.k) {
                a.topk[(int64_t)t * a.k + j] = sel_idx[j];
                a.gates[(int64_t)t * a.k + j] = renorm ? sel_v[j] / sel_sum : sel_v[j];
            }
    }
    // loss partials: one row per 4 tokens (4 * E_T lanes), tokens in order
    float pc = valid ? (a.score == MOE_SCORE_SOFTMAX ? v : v / ssum) : 0.f;
    float zc = (tok && gl == 0) ? lse * lse : 0.f;
#pragma unroll
    for (int o = E_T; o < kPartialTokens * E_T; o <<= 1) {
        pc += __shfl_xor_sync(0xffffffffu, pc, o);
        zc += __shfl_xor_sync(0xffffffffu, zc, o);
    }
    const int row = t0 / kPartialTokens + lane / (kPartialTokens * E_T);
    const bool row_lane = (lane % (kPartialTokens * E_T)) < E_T;
    if (row_lane && row * kPartialTokens < T) {
        float *out = a.partials + (int64_t)row * (E + 1);
        if (gl < E)
            out[gl] = pc;
        if (gl == 0)
            out[E] = zc;
    }
}

template <int E_T, int CPT, int NV>
__global__ void __launch_bounds__(THREADS, 1) route_small_kernel(RouteArgs a, int stages)
{
    constexpr int TB = 32 / E_T;       // tokens per reduce-scatter batch
    constexpr int NW = THREADS / 32;   // warps (8: two per SM sub-partition)
    constexpr int GROUP = NW;          // batches per round of epilogues
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t full[MAX_STAGES];
    __shared__ __align__(8) uint64_t empty[MAX_STAGES];
    __shared__ float red[GROUP][NW][32];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, T = a.T, d = a.d;
    const uint8_t *x = static_cast<const uint8_t *>(a.x);
    const int row_bytes = d * 2;
    const int stage_bytes = TB * row_bytes;
    const int nbatch = (T + TB - 1) / TB;
    const int G = gridDim.x;
    const int n_my = blockIdx.x < nbatch ? (nbatch - 1 - blockIdx.x) / G + 1 : 0;
    const bool producer = tid == 0;

    if (producer) {
        for (int q = 0; q < stages; ++q) {
            mbar_init_route(smem_addr(&full[q]), 1);
            mbar_init_route(smem_addr(&empty[q]), NW);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_flag = 0;
    }
    __syncthreads();

    // Thread 0 also issues the copies: batch i goes into stage i % stages once
    // every warp has released batch i - stages.  Before computing batch `it`
    // it tops the ring up to batch it + stages - 1, which only needs batch
    // it - 1 released, so no warp ever waits on a copy that is not issued.
    int next_issue = 0;
    int last_issue[MAX_STAGES];
    for (int q = 0; q < MAX_STAGES; ++q)
        last_issue[q] = -1;
    auto issue_upto = [&](int limit) {
        while (next_issue < limit && !abort_flag) {
            const int i = next_issue, s = i % stages, round = i / stages;
            if (round > 0 &&
                !route_wait(smem_addr(&empty[s]), (uint32_t)((round - 1) & 1), &abort_flag))
                return;
            const int b = blockIdx.x + i * G;
            const uint32_t bytes = (uint32_t)(min(TB, T - b * TB) * row_bytes);
            const uint32_t bar = smem_addr(&full[s]);
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                         "r"(bytes)
                         : "memory");
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], "
                "%2, [%3];" ::"r"(smem_addr(ring + s * stage_bytes)),
                "l"(x + (int64_t)b * stage_bytes), "r"(bytes), "r"(bar)
                : "memory");
            last_issue[s] = i;
            ++next_issue;
        }
    };
    if (producer)
        issue_upto(min(stages, n_my));

    const bool renorm = a.renorm < 0 ? (a.k > 1) : (a.renorm != 0);
    float w[NV][CPT][E_T];
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int col = (v * THREADS + tid) * CPT + i;
            const float *wr = a.W_r + (int64_t)col * E;
            if (E == E_T) {   // whole 16-byte rows of W_r
#pragma unroll
                for (int e = 0; e < E_T; e += 4) {
                    const float4 q = __ldg(reinterpret_cast<const float4 *>(wr + e));
                    w[v][i][e] = q.x;
                    w[v][i][e + 1] = q.y;
                    w[v][i][e + 2] = q.z;
                    w[v][i][e + 3] = q.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < E_T; ++e)
                    w[v][i][e] = e < E ? __ldg(wr + e) : 0.f;
            }
        }

    for (int g0 = 0; g0 < n_my; g0 += GROUP) {
        const int gn = min(GROUP, n_my - g0);
        for (int j = 0; j < gn; ++j) {
            const int it = g0 + j;
            const int s = it % stages;
            const int t0 = (blockIdx.x + it * G) * TB;
            if (producer)
                issue_upto(min(it + stages, n_my));
            __syncwarp();
            const bool ok = !abort_flag && route_wait(smem_addr(&full[s]),
                                                      (uint32_t)((it / stages) & 1), &abort_flag);
            // one token at a time keeps the loop body small (instruction cache)
            const uint8_t *st = ring + s * stage_bytes;
#pragma unroll 1
            for (int tk = 0; tk < TB; ++tk) {
                float acc[E_T];
#pragma unroll
                for (int e = 0; e < E_T; ++e)
                    acc[e] = 0.f;
                if (ok && t0 + tk < T) {
#pragma unroll
                    for (int v = 0; v < NV; ++v) {
                        float xv[CPT];
                        XVec<CPT>::load(st + tk * row_bytes + (v * THREADS + tid) * CPT * 2, xv);
#pragma unroll
                        for (int q = 0; q < CPT; ++q)
#pragma unroll
                            for (int e = 0; e < E_T; ++e)
                                acc[e] = fmaf(xv[q], w[v][q][e], acc[e]);
                    }
                }
                // lanes 32/E_T * e .. hold expert e's warp total
                const float sum = warp_reduce_scatter<E_T>(acc, lane);
                if ((lane & (32 / E_T - 1)) == 0)
                    red[j][warp][tk * E_T + lane / (32 / E_T)] = sum;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive_route(smem_addr(&empty[s]));   // this warp is done with stage s
        }
        __syncthreads();
        if (warp < gn) {
            const int it = g0 + warp;
            const int t0 = (blockIdx.x + it * G) * TB;
            if (!abort_flag) {
                float z = 0.f;
#pragma unroll
                for (int ww = 0; ww < NW; ++ww)
                    z += red[warp][ww][lane];
                small_epilogue<E_T>(a, z, t0, lane, renorm);
            } else {
                // an expired wait: mark the batch's tokens with expert -1
                for (int q = lane; q < TB * a.k; q += 32)
                    if (t0 + q / a.k < T)
                        a.topk[(int64_t)t0 * a.k + q] = -1;
            }
        }
        __syncthreads();
    }
    // every copy issued has landed before the block exits (bounded)
    if (producer)
        for (int q = 0; q < stages; ++q)
            if (last_issue[q] >= 0)
                route_wait(smem_addr(&full[q]), (uint32_t)((last_issue[q] / stages) & 1), nullptr);
}

int sm_count()
{
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int E_T, int CPT, int NV>
cudaError_t launch_small(const RouteArgs &a, cudaStream_t s)
{
    constexpr int TB = 32 / E_T;
    const int stage_bytes = TB * a.d * 2;
    int stages = RING_BYTES / stage_bytes;
    stages = stages > MAX_STAGES ? MAX_STAGES : stages;
    const int nbatch = (a.T + TB - 1) / TB;
    const int grid = nbatch < sm_count() ? nbatch : sm_count();
    const int smem = stages * stage_bytes;
    auto kern = route_small_kernel<E_T, CPT, NV>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    kern<<<grid, THREADS, smem, s>>>(a, stages);
    return cudaGetLastError();
}

// Launches the register-resident variant when the W_r slice fits (at most 128
// floats per thread), x is 16-byte aligned and a ring of at least two batches
// fits; sets *done.  Leaves *done false otherwise.
template <int E_T>
cudaError_t try_small(const RouteArgs &a, cudaStream_t s, bool *done)
{
    *done = false;
    const int d = a.d;
    if ((reinterpret_cast<uintptr_t>(a.x) & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(a.W_r) & 15u) != 0 || 2 * (32 / E_T) * d * 2 > RING_BYTES)
        return cudaSuccess;
    *done = true;
    if (d % (THREADS * 8) == 0) {
        const int nv = d / (THREADS * 8);
        if (nv == 1) return launch_small<E_T, 8, 1>(a, s);
        if (nv == 2) return launch_small<E_T, 8, 2>(a, s);
    }
    if (d % (THREADS * 4) == 0) {
        const int nv = d / (THREADS * 4);
        if (nv == 1) return launch_small<E_T, 4, 1>(a, s);
        if (nv == 2) return launch_small<E_T, 4, 2>(a, s);
        if constexpr (E_T <= 4) {
            if (nv == 4) return launch_small<E_T, 4, 4>(a, s);
        }
    }
    *done = false;
    return cudaSuccess;
}

template <typename Tin, int TM, int TN>
cudaError_t launch_tiled(const RouteArgs &a, int blocks, cudaStream_t s)
{
    const int NX = (a.E + TN - 1) / TN;
    const int Epad = NX * TN;
    size_t smem = sizeof(float) * (RT * (KC + 1) + KC * Epad + RT * (a.E + 1) + RT);
    auto kern = route_kernel<Tin, TM, TN>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
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
    if (c.dtype == MOE_DTYPE_BF16 && c.E >= 3 && c.E <= 8) {
        bool done = false;
        cudaError_t err = c.E <= 4 ? try_small<4>(a, s, &done) : try_small<8>(a, s, &done);
        if (done)
            return err;
    }
    if (c.dtype == MOE_DTYPE_BF16)
        return launch_typed<__nv_bfloat16>(a, blocks, s);
    return launch_typed<float>(a, blocks, s);
}

}  // namespace moe
