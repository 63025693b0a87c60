// Router on the tensor cores for bf16 layers.
//
// Page "Lab 18 - Mixture of experts", section 1 (z = x W_r, softmax, top-k,
// gate values), section 2 (P_i, logsumexp); "Lab 01" traps (ties to the lower
// expert index); routers are computed in fp32 (cs336 lecture 4, "Stability,
// fine-tuning, and upcycling").
//
// x is bf16, so x W_r needs no fp32 inputs to stay exact: every fp32 weight is
// the exact sum of three bf16 numbers (hi = bf16(w), mid = bf16(w - hi),
// lo = w - hi - mid, each rounding exact because the remainders keep at most
// 16 and 8 significant bits), and bf16 x bf16 products are exact in fp32.  So
//     z = x W_hi + x W_mid + x W_lo
// accumulated in fp32 is the fp32 router, computed by three bf16 MMAs per K
// step into one TMEM accumulator.  Three kernels:
//   split  - W_r [d, E] fp32 -> W3 [3][E_pad][d] bf16 (K-major, zero rows past E);
//   logits - grid (token tile of 128, expert chunk of up to 64, K part): TMA ring
//            of x and W3 tiles, tcgen05.mma from one thread, the accumulator
//            read back with tcgen05.ld and written as fp32 partial logits
//            [K part][T][E_pad];
//   select - sums the K parts in order, adds the logit bias, softmax or
//            sigmoid, top-k by warp argmax, gates, and one loss-partials row per
//            block of 32 tokens: one warp per token, or for E <= 8 one warp per
//            4 (or 8) tokens with E_T lanes each.
#include "internal.cuh"
#include "route_common.cuh"

#include <cuda.h>
#include <math.h>

namespace moe {
namespace rtc {

constexpr int BM = 128, BK = 64;
constexpr int THREADS = 128;   // warp 0: TMA producer, warp 1: MMA; then all 4 read TMEM
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB

// -------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t saddr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Bounded wait (about 2 s of wall clock); false on expiry or once `abort` is set.
__device__ __noinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                      int32_t *status)
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
        if ((i & 31u) == 0) {
            if (abort && *abort)
                return false;
            uint64_t now;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
            if (i == 0) {
                t0 = now;
            } else if (now - t0 > 2000000000ull) {
                if (abort)
                    *abort = 1;
                if (status)
                    atomicExch(status, (int32_t)MOE_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t a)
{
    return (uint64_t)((a & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

struct __align__(64) LogitParams {
    CUtensorMap tmX;   // x as (d, T, 1)
    CUtensorMap tmW;   // W3 as (d, E_pad, 3)
    float *partial;    // [k_parts][T][E_pad]
    int T, E_pad, n_chunk, kb_per_part, k_blocks;
    int32_t *status;
};

// ---------------------------------------------------------------- split

__global__ void __launch_bounds__(256) split_kernel(const float *__restrict__ W_r, int d, int E,
                                                    int E_pad, __nv_bfloat16 *__restrict__ W3)
{
    __shared__ float tile[32][33];
    const int c0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int c = c0 + r, e = e0 + tx;
        tile[r][tx] = (c < d && e < E) ? W_r[(int64_t)c * E + e] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int e = e0 + r, c = c0 + tx;
        if (e < E_pad && c < d) {
            const float w = tile[tx][r];
            const __nv_bfloat16 hi = __float2bfloat16_rn(w);
            const float r1 = w - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
            const int64_t o = (int64_t)e * d + c;
            W3[o] = hi;
            W3[(int64_t)E_pad * d + o] = mid;
            W3[2 * (int64_t)E_pad * d + o] = lo;
        }
    }
}

// ---------------------------------------------------------------- logits

template <int N>
__global__ void __launch_bounds__(THREADS, 1) logits_kernel(const __grid_constant__ LogitParams p)
{
    constexpr int B_BYTES = N * BK * 2;                 // one split's tile
    constexpr int STAGE = A_BYTES + 3 * B_BYTES;
    constexpr uint32_t TMEM_COLS = N <= 32 ? 32 : (N <= 64 ? 64 : 128);   // power of two >= 32
    constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
                               ((uint32_t)(BM >> 4) << 24);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], done;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * N;
    const int kb0 = blockIdx.z * p.kb_per_part;
    const int kb1 = min(kb0 + p.kb_per_part, p.k_blocks);
    const int nk = kb1 - kb0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            bar_init(saddr(&full[s]), 1);
            bar_init(saddr(&empty[s]), 1);
        }
        bar_init(saddr(&done), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(&tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---- TMA producer ----
        int last_issue[STAGES];
        for (int s = 0; s < STAGES; ++s)
            last_issue[s] = -1;
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            if (i >= STAGES && !bar_wait(saddr(&empty[s]), (uint32_t)(((i / STAGES) - 1) & 1),
                                         &abort_flag, p.status))
                break;
            const uint32_t fb = saddr(&full[s]);
            const uint32_t dst = saddr(smem + s * STAGE);
            const int kc = (kb0 + i) * BK;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb),
                         "r"(STAGE)
                         : "memory");
            asm volatile(
                "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
                " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
                "l"(reinterpret_cast<uint64_t>(&p.tmX)), "r"(kc), "r"(m0), "r"(0), "r"(fb)
                : "memory");
#pragma unroll
            for (int sp = 0; sp < 3; ++sp)
                asm volatile(
                    "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
                    " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst + A_BYTES + sp * B_BYTES),
                    "l"(reinterpret_cast<uint64_t>(&p.tmW)), "r"(kc), "r"(n0), "r"(sp), "r"(fb)
                    : "memory");
            last_issue[s] = i;
        }
        // copies in flight land before the block exits (bounded)
        for (int s = 0; s < STAGES; ++s)
            if (last_issue[s] >= 0)
                bar_wait(saddr(&full[s]), (uint32_t)((last_issue[s] / STAGES) & 1), nullptr,
                         nullptr);
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: three bf16 MMAs (hi, mid, lo) per K step of 16 ----
        bool any = false;
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            if (!bar_wait(saddr(&full[s]), (uint32_t)((i / STAGES) & 1), &abort_flag, p.status))
                break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t a = saddr(smem + s * STAGE);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
                for (int sp = 0; sp < 3; ++sp) {
                    const uint32_t acc = (i | kk | sp) != 0 ? 1u : 0u;
                    asm volatile(
                        "{\n\t.reg .pred q;\n\t"
                        "setp.ne.b32 q, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q;\n\t}" ::"r"(tmem),
                        "l"(sdesc_sw128(a + kk * 32)),
                        "l"(sdesc_sw128(a + A_BYTES + sp * B_BYTES + kk * 32)), "r"(IDESC),
                        "r"(acc)
                        : "memory");
                }
            asm volatile(
                "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    saddr(&empty[s]))
                : "memory");
            any = true;
        }
        if (any)
            asm volatile(
                "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    saddr(&done))
                : "memory");
        else
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&done)) : "memory");
    }
    __syncwarp();

    // ---- all four warps: accumulator rows -> fp32 partial logits ----
    const bool ok = bar_wait(saddr(&done), 0, nullptr, p.status) && !abort_flag;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const int row = m0 + warp * 32 + lane;
    float *out = p.partial + ((int64_t)blockIdx.z * p.T + row) * p.E_pad + n0;
#pragma unroll
    for (int c = 0; c < N; c += 16) {
        uint32_t r[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
              "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
              "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (row < p.T) {
#pragma unroll
            for (int q = 0; q < 16; q += 4) {
                float4 v;
                v.x = ok ? __uint_as_float(r[q]) : NAN;
                v.y = ok ? __uint_as_float(r[q + 1]) : NAN;
                v.z = ok ? __uint_as_float(r[q + 2]) : NAN;
                v.w = ok ? __uint_as_float(r[q + 3]) : NAN;
                *reinterpret_cast<float4 *>(out + c + q) = v;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------- select

struct SelectArgs {
    const float *partial;
    int parts, E_pad;
    const float *logit_bias, *select_bias;
    int32_t *topk;
    float *gates, *loss_partials, *logits_out, *scores_out;
    int T, E, k, score, renorm;
};

// fp32 -> unsigned integer of the same order (-0 made +0; keys are never NaN),
// and back: lets a warp take a max with one redux.sync instead of a shuffle
// tree.
__device__ __forceinline__ uint32_t ord_key(float f)
{
    const uint32_t u = __float_as_uint(f + 0.f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_key(uint32_t u)
{
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// The token's logits: the K parts summed in order, plus the logit bias.
template <int PL>
__device__ __forceinline__ void load_logits(const SelectArgs &a, int t, int lane, float *z)
{
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        const int e = lane + 32 * i;
        z[i] = -INFINITY;
        if (t < a.T && e < a.E) {
            float s = 0.f;
            for (int q = 0; q < a.parts; ++q)
                s += a.partial[((int64_t)q * a.T + t) * a.E_pad + e];
            if (a.logit_bias)
                s += a.logit_bias[e];
            z[i] = s;
        }
    }
}

// One block = 32 tokens = one row of the loss partials, one warp per token
// (with four tokens per warp in series, eight warps per block left the
// schedulers half idle); the warps' sums meet in shared memory in warp order.
// Lane l holds experts l, l + 32, ... (PL of them).  Each top-k round is two
// integer warp reductions: the largest key, then the lowest expert index
// holding it (ties go to the lower index).
template <int PL>
__global__ void __launch_bounds__(32 * kPartialTokens, 1) select_kernel(SelectArgs a)
{
    constexpr int W = kPartialTokens;   // warps per block, one token each
    __shared__ float pw[W][kMaxE + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E;
    const bool renorm = a.renorm < 0 ? (a.k > 1) : (a.renorm != 0);
    const int t = blockIdx.x * kPartialTokens + warp;
    float pacc[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i)
        pacc[i] = 0.f;
    float zacc = 0.f;
    if (t < a.T) {
        float z[PL];
        load_logits<PL>(a, t, lane, z);
        uint32_t mo = 0;
#pragma unroll
        for (int i = 0; i < PL; ++i)
            if (lane + 32 * i < E)
                mo = max(mo, ord_key(z[i]));
        const float m = unord_key(__reduce_max_sync(0xffffffffu, mo));
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i)
            if (lane + 32 * i < E)
                sum += expf(z[i] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float lse = m + logf(sum);
        float v[PL];
        uint32_t okey[PL];   // 0: not an expert of this layer
        float ssum = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int e = lane + 32 * i;
            const bool okk = e < E;
            float key;
            if (a.score == MOE_SCORE_SOFTMAX) {
                v[i] = okk ? expf(z[i] - m) / sum : 0.f;
                key = z[i];
            } else {
                v[i] = okk ? 1.f / (1.f + expf(-z[i])) : 0.f;
                key = v[i] + (a.select_bias && okk ? a.select_bias[e] : 0.f);
                ssum += v[i];
            }
            okey[i] = okk ? ord_key(key) : 0u;
            if (okk && a.logits_out)
                a.logits_out[(int64_t)t * E + e] = z[i];
            if (okk && a.scores_out)
                a.scores_out[(int64_t)t * E + e] = v[i];
        }
        if (a.score == MOE_SCORE_SIGMOID) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
        }
        int sel_idx[kMaxK];
        float sel_v[kMaxK];
        float sel_sum = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            sel_idx[j] = 0;
            sel_v[j] = 0.f;
            if (j >= a.k)
                continue;
            uint32_t lk = 0;
#pragma unroll
            for (int i = 0; i < PL; ++i)
                lk = max(lk, okey[i]);
            const uint32_t mk = __reduce_max_sync(0xffffffffu, lk);
            uint32_t li = 0xffffffffu;
#pragma unroll
            for (int i = PL - 1; i >= 0; --i)
                if (okey[i] == mk && mk != 0u)
                    li = (uint32_t)(lane + 32 * i);
            const uint32_t bi = __reduce_min_sync(0xffffffffu, li);
            const int slot = (int)(bi >> 5);
            float mine = v[0];
#pragma unroll
            for (int i = 1; i < PL; ++i)
                if (slot == i)
                    mine = v[i];
            const float bv = __shfl_sync(0xffffffffu, mine, (int)(bi & 31u));
            if ((int)(bi & 31u) == lane) {
#pragma unroll
                for (int i = 0; i < PL; ++i)
                    if (slot == i)
                        okey[i] = 0u;   // taken
            }
            sel_idx[j] = (int)bi;
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
            zacc += lse * lse;
        }
#pragma unroll
        for (int i = 0; i < PL; ++i)
            if (lane + 32 * i < E)
                pacc[i] += a.score == MOE_SCORE_SOFTMAX ? v[i] : v[i] / ssum;
    }
#pragma unroll
    for (int i = 0; i < PL; ++i)
        if (lane + 32 * i < E)
            pw[warp][lane + 32 * i] = pacc[i];
    if (lane == 0)
        pw[warp][E] = zacc;
    __syncthreads();
    float *out = a.loss_partials + (int64_t)blockIdx.x * (E + 1);
    for (int e = threadIdx.x; e <= E; e += 32 * W) {
        float acc = 0.f;
        for (int w = 0; w < W; ++w)
            acc += pw[w][e];
        out[e] = acc;
    }
}

// Small E (<= 8): a warp holds 32 / E_T tokens at once, lane L = (token
// L / E_T, expert L % E_T), so softmax, top-k and the loss sums are segmented
// shuffles over E_T lanes; E_T warps make one block of 32 tokens, one row of
// the loss partials.
template <int E_T>
__global__ void __launch_bounds__(32 * E_T) select_small_kernel(SelectArgs s)
{
    constexpr int TB = 32 / E_T;
    __shared__ float pw[E_T][E_T];
    __shared__ float zw[E_T];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * kPartialTokens + warp * TB;
    const int gl = lane % E_T;
    const int t = t0 + lane / E_T;
    float z = -INFINITY;
    if (t < s.T && gl < s.E) {
        z = 0.f;
        for (int q = 0; q < s.parts; ++q)
            z += s.partial[((int64_t)q * s.T + t) * s.E_pad + gl];
    }
    RouteArgs a{nullptr, nullptr, s.logit_bias, s.select_bias, s.topk, s.gates,
                s.loss_partials, s.logits_out, s.scores_out, s.T, 0, s.E, s.k, s.score, s.renorm};
    const bool renorm = s.renorm < 0 ? (s.k > 1) : (s.renorm != 0);
    float pc, zc;
    small_epilogue<E_T>(a, z, t0, lane, renorm, &pc, &zc);
    if (lane < E_T)
        pw[warp][lane] = pc;
    if (lane == 0)
        zw[warp] = zc;
    __syncthreads();
    float *out = s.loss_partials + (int64_t)blockIdx.x * (s.E + 1);
    if (threadIdx.x <= s.E) {
        float acc = 0.f;
        for (int w = 0; w < E_T; ++w)
            acc += threadIdx.x < s.E ? pw[w][threadIdx.x] : zw[w];
        out[threadIdx.x] = acc;
    }
}

// ---------------------------------------------------------------- host

typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder()
{
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    }
    return fn;
}

bool map3(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
          uint64_t s2, uint32_t b0, uint32_t b1)
{
    EncodeTiled enc = encoder();
    if (!enc)
        return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int N>
cudaError_t launch_logits(const LogitParams &p, dim3 grid, cudaStream_t s)
{
    constexpr int smem = STAGES * (A_BYTES + 3 * N * BK * 2) + 1024;
    auto kern = logits_kernel<N>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    kern<<<grid, THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace rtc

RoutePlan route_plan(const moe_config &c)
{
    RoutePlan r{};
    r.tensor_cores = c.dtype == MOE_DTYPE_BF16 && c.d % 64 == 0;
    r.E_pad = c.E <= 64 ? (int)align_up((size_t)c.E, 16) : (int)align_up((size_t)c.E, 64);
    r.n_chunk = r.E_pad <= 64 ? r.E_pad : 64;
    const int n_chunks = r.E_pad / r.n_chunk;
    const int m_tiles = (int)ceil_div(c.T, rtc::BM);
    const int k_blocks = (int)ceil_div(c.d, rtc::BK);
    const int base = m_tiles * n_chunks > 0 ? m_tiles * n_chunks : 1;
    // fill about one wave of SMs (two blocks per SM fit when the expert chunk
    // is 16 wide); keep at least 4 K blocks per part
    const int want = (r.n_chunk <= 16 ? 296 : 148) / base;
    int parts = want < k_blocks / 4 ? want : k_blocks / 4;
    r.k_parts = parts < 1 ? 1 : parts;
    r.kb_per_part = (int)ceil_div(k_blocks, r.k_parts);
    r.k_parts = (int)ceil_div(k_blocks, r.kb_per_part);
    return r;
}

size_t route_scratch_bytes(const moe_config &c)
{
    const RoutePlan r = route_plan(c);
    if (!r.tensor_cores)
        return 0;
    return align_up((size_t)3 * r.E_pad * c.d * 2, 256) +
           align_up((size_t)r.k_parts * c.T * r.E_pad * 4, 256);
}

cudaError_t launch_route_tc(const moe_config &c, const void *x, const float *W_r,
                            const float *logit_bias, const float *select_bias, int32_t *topk,
                            float *gates, float *partials, float *logits_out, float *scores_out,
                            void *scratch, int32_t *status, cudaStream_t s)
{
    using namespace rtc;
    const RoutePlan r = route_plan(c);
    __nv_bfloat16 *W3 = static_cast<__nv_bfloat16 *>(scratch);
    float *plog = reinterpret_cast<float *>(static_cast<char *>(scratch) +
                                            align_up((size_t)3 * r.E_pad * c.d * 2, 256));
    dim3 sg((unsigned)ceil_div(c.d, 32), (unsigned)ceil_div(r.E_pad, 32));
    split_kernel<<<sg, 256, 0, s>>>(W_r, c.d, c.E, r.E_pad, W3);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess)
        return err;
    LogitParams p;
    memset(&p, 0, sizeof p);
    bool ok = map3(&p.tmX, x, c.d, c.T, 1, (uint64_t)c.d * 2, (uint64_t)c.d * 2 * c.T, BK, BM);
    ok &= map3(&p.tmW, W3, c.d, r.E_pad, 3, (uint64_t)c.d * 2, (uint64_t)c.d * 2 * r.E_pad, BK,
               r.n_chunk);
    if (!ok)
        return cudaErrorInvalidValue;
    p.partial = plog;
    p.T = c.T;
    p.E_pad = r.E_pad;
    p.n_chunk = r.n_chunk;
    p.kb_per_part = r.kb_per_part;
    p.k_blocks = (int)ceil_div(c.d, BK);
    p.status = status;
    dim3 grid((unsigned)ceil_div(c.T, BM), (unsigned)(r.E_pad / r.n_chunk), (unsigned)r.k_parts);
    switch (r.n_chunk) {
    case 16: err = launch_logits<16>(p, grid, s); break;
    case 32: err = launch_logits<32>(p, grid, s); break;
    case 48: err = launch_logits<48>(p, grid, s); break;
    default: err = launch_logits<64>(p, grid, s); break;
    }
    if (err != cudaSuccess)
        return err;
    SelectArgs a{plog, r.k_parts, r.E_pad, logit_bias, select_bias, topk, gates, partials,
                 logits_out, scores_out, c.T, c.E, c.k, c.score, c.renorm};
    const unsigned rows = (unsigned)ceil_div(c.T, kPartialTokens);
    if (c.E <= 4)
        select_small_kernel<4><<<rows, 4 * 32, 0, s>>>(a);
    else if (c.E <= 8)
        select_small_kernel<8><<<rows, 8 * 32, 0, s>>>(a);
    else if (c.E <= 32)
        select_kernel<1><<<rows, 32 * kPartialTokens, 0, s>>>(a);
    else if (c.E <= 64)
        select_kernel<2><<<rows, 32 * kPartialTokens, 0, s>>>(a);
    else if (c.E <= 128)
        select_kernel<4><<<rows, 32 * kPartialTokens, 0, s>>>(a);
    else
        select_kernel<8><<<rows, 32 * kPartialTokens, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
