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
// in fp32 is the fp32 router.
//
// Up to 16 experts: one kernel (details at route_kernel).  The blocks of a
// thread-block cluster split K for one 128-token tile; each splits its part of
// W_r into the three terms stage by stage as the tile's x streams (hi, mid and
// lo stacked as 3 x 16 rows of the MMA's B operand, so one MMA per K step
// gives the three products side by side in TMEM).  Each block then selects
// its share of the tile's tokens, summing the K parts' partial logits in
// order through distributed shared memory: softmax or sigmoid, top-k (ties to
// the lower index), gates, optional logits/scores, and the rows of the loss
// partials (32 tokens per row) in a fixed order.
//
// More experts: three launches (split once, logits, select), below.
#include "internal.cuh"
#include "route_common.cuh"

#include <cuda.h>
#include <math.h>

namespace moe {
namespace rtc {

constexpr int BM = 128, BK = 64;
constexpr int THREADS = 512;   // one-kernel router: 16 warps, roles below, then all select
constexpr int WARPS = THREADS / 32;
constexpr int STAGES = 4;              // TMA ring of either kernel
constexpr int A_BYTES = BM * BK * 2;   // 16 KB: one x tile of a K block
constexpr int CONV_WARP0 = 4;          // warps 4-7 split W_r, then read TMEM
constexpr int COPY_WARP0 = 8;          // warps 8-11 copy W_r
constexpr int CONV_LANES = 128;        // lanes of either role
constexpr int MAX_CLUSTER = 4;

// -------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t saddr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void bar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait (about 2 s of wall clock); false on expiry or once `abort` is
// set.  (A suspend-time hint on the tries, letting the thread sleep until the
// phase completes, measured slower here: woken threads resumed up to
// microseconds after the phase completed.)
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

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory offset in block `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

__device__ __forceinline__ float ld_peer(uint32_t a)
{
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}

// Sum of the float at offset off in the parts blocks whose shared bases are
// rb[0 .. parts - 1] (parts <= MAX_CLUSTER), in part order.  Every remote load
// is issued before the first add, so the parts cost one round trip.
__device__ __forceinline__ float sum_parts(const uint32_t *rb, int parts, uint32_t off)
{
    float v[MAX_CLUSTER];
#pragma unroll
    for (int q = 0; q < MAX_CLUSTER; ++q)
        v[q] = q < parts ? ld_peer(rb[q] + off) : 0.f;
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < MAX_CLUSTER; ++q)
        if (q < parts)
            s += v[q];
    return s;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const float *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// Arrives on the mbarrier once this thread's earlier cp.async copies land.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

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

// Two bf16 terms packed low-k first, as a K-major row stores them.
__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 a, __nv_bfloat16 b)
{
    return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}

struct __align__(64) RouteParams {
    CUtensorMap tmX;   // x as (d, T, 1)
    const float *W_r;  // [d, E] fp32
    const float *logit_bias, *select_bias;
    int32_t *topk;
    float *gates, *loss_partials, *logits_out, *scores_out;
    int T, d, E, k, score, renorm;
    int cs, k_parts, kb_per_part, k_blocks;
    int clear_status;               // 1: block 0 clears the status word first
    int32_t *status;
};

// ------------------------------------------------------------- selection

// The fields selection reads, copied out of the kernel parameters once so
// that they stay in registers across a token's global stores (read through
// the parameter block they could be re-read after every store).
struct SelArgs {
    int32_t *topk;
    float *gates, *logits_out, *scores_out;
    const float *select_bias;
    int E, k, score;
};
__device__ __forceinline__ SelArgs sel_args(const RouteParams &p)
{
    return SelArgs{p.topk, p.gates, p.logits_out, p.scores_out, p.select_bias, p.E, p.k, p.score};
}

// NT tokens held by a whole warp, lane l holding experts l, l + 32, ... (PL
// of them) of each: softmax or sigmoid, top-k and gates; adds the loss terms
// of the tokens with tv set to pacc / zacc in token order.  The NT tokens'
// steps are independent, so the warp keeps NT dependency chains in flight
// instead of one.  SB_REG: sb holds the lane's selection biases (0 without);
// otherwise they are read from a.select_bias.  Each top-k round is two integer
// warp reductions: the largest key, then the lowest expert index holding it
// (ties go to the lower index); lane j keeps round j's expert and value, so
// the k outputs go out from k lanes at once (the gate sum still adds the
// values in round order).  A token with tv clear takes part in the warp
// reductions (with finite logits) and writes nothing.
template <int PL, int NT, bool SB_REG>
__device__ __forceinline__ void select_tokens(const SelArgs &a, bool renorm, const int (&t)[NT],
                                              const bool (&tv)[NT], int lane,
                                              const float (&z)[NT][PL], const float (&sb)[PL],
                                              float (&pacc)[PL], float &zacc)
{
    const int E = a.E;
    float m[NT], sum[NT], lse[NT], ssum[NT], v[NT][PL];
    uint32_t okey[NT][PL];   // 0: not an expert of this layer, or taken
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        uint32_t mo = 0;
#pragma unroll
        for (int i = 0; i < PL; ++i)
            if (lane + 32 * i < E)
                mo = max(mo, ord_key(z[n][i]));
        m[n] = unord_key(__reduce_max_sync(0xffffffffu, mo));
    }
    float ex[NT][PL];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        sum[n] = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            ex[n][i] = lane + 32 * i < E ? expf(z[n][i] - m[n]) : 0.f;
            sum[n] += ex[n][i];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int n = 0; n < NT; ++n)
            sum[n] += __shfl_xor_sync(0xffffffffu, sum[n], o);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        lse[n] = m[n] + logf(sum[n]);
        ssum[n] = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int e = lane + 32 * i;
            const bool okk = e < E;
            float key;
            if (a.score == MOE_SCORE_SOFTMAX) {
                v[n][i] = okk ? ex[n][i] / sum[n] : 0.f;
                key = z[n][i];
            } else {
                v[n][i] = okk ? 1.f / (1.f + expf(-z[n][i])) : 0.f;
                key = v[n][i] + (SB_REG ? sb[i] : (a.select_bias && okk ? a.select_bias[e] : 0.f));
                ssum[n] += v[n][i];
            }
            okey[n][i] = okk ? ord_key(key) : 0u;
            if (okk && tv[n] && a.logits_out)
                a.logits_out[(int64_t)t[n] * E + e] = z[n][i];
            if (okk && tv[n] && a.scores_out)
                a.scores_out[(int64_t)t[n] * E + e] = v[n][i];
        }
    }
    if (a.score == MOE_SCORE_SIGMOID) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int n = 0; n < NT; ++n)
                ssum[n] += __shfl_xor_sync(0xffffffffu, ssum[n], o);
    }
    int my_idx[NT];
    float my_v[NT], sel_sum[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        my_idx[n] = 0;
        my_v[n] = 0.f;
        sel_sum[n] = 0.f;
    }
#pragma unroll 1
    for (int j = 0; j < a.k; ++j) {
        uint32_t mk[NT];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            uint32_t lk = 0;
#pragma unroll
            for (int i = 0; i < PL; ++i)
                lk = max(lk, okey[n][i]);
            mk[n] = __reduce_max_sync(0xffffffffu, lk);
        }
        uint32_t bi[NT];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            uint32_t li = 0xffffffffu;
#pragma unroll
            for (int i = PL - 1; i >= 0; --i)
                if (okey[n][i] == mk[n] && mk[n] != 0u)
                    li = (uint32_t)(lane + 32 * i);
            bi[n] = __reduce_min_sync(0xffffffffu, li);
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int slot = (int)(bi[n] >> 5);
            float mine = v[n][0];
#pragma unroll
            for (int i = 1; i < PL; ++i)
                if (slot == i)
                    mine = v[n][i];
            const float bv = __shfl_sync(0xffffffffu, mine, (int)(bi[n] & 31u));
            if ((int)(bi[n] & 31u) == lane) {
#pragma unroll
                for (int i = 0; i < PL; ++i)
                    if (slot == i)
                        okey[n][i] = 0u;   // taken
            }
            if (lane == j) {
                my_idx[n] = (int)bi[n];
                my_v[n] = bv;
            }
            sel_sum[n] += bv;
        }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        if (!tv[n])
            continue;
        if (lane < a.k) {
            a.topk[(int64_t)t[n] * a.k + lane] = my_idx[n];
            a.gates[(int64_t)t[n] * a.k + lane] = renorm ? my_v[n] / sel_sum[n] : my_v[n];
        }
        if (lane == 0)
            zacc += lse[n] * lse[n];
#pragma unroll
        for (int i = 0; i < PL; ++i)
            if (lane + 32 * i < E)
                pacc[i] += a.score == MOE_SCORE_SOFTMAX ? v[n][i] : v[n][i] / ssum[n];
    }
}

template <int PL, bool SB_REG>
__device__ __forceinline__ void select_token(const SelArgs &a, bool renorm, int t, int lane,
                                             const float (&z)[PL], const float (&sb)[PL],
                                             float (&pacc)[PL], float &zacc)
{
    const int tt[1] = {t};
    const bool tv[1] = {true};
    float zz[1][PL];
#pragma unroll
    for (int i = 0; i < PL; ++i)
        zz[0][i] = z[i];
    select_tokens<PL, 1, SB_REG>(a, renorm, tt, tv, lane, zz, sb, pacc, zacc);
}

// ---------------------------------------------------------------- kernel

// One 128-token tile per cluster of k_parts blocks (block `rank` owns K
// blocks [rank kbp, (rank + 1) kbp)), two blocks per SM, 16 warps:
//   warp 0       TMA ring of x tiles (4 stages, one thread);
//   warp 1       one MMA of N = 3 x 16 per K step of 16 into TMEM;
//   warps 8-11   copy each stage's fp32 W_r slice into a staging slot
//                (4-byte cp.async, arriving on the stage's barrier when landed);
//   warps 4-7    split the staged slice into the three bf16 terms (128-byte
//                swizzle, the stage's B operand), then read the accumulator
//                back (hi + (mid + lo)) into the block's partial-logit tile;
//   all 16       after a cluster barrier, select the block's 128 / P tokens,
//                summing the P partial tiles in part order (ld.shared::cluster).
// So W_r is split while x streams, and the stage ring is the only pipeline.
// N: experts per block (launched with 16).  Selection: E_T > 0 takes E <= E_T
// experts with E_T lanes per token (32 / E_T tokens per warp at once); E_T == 0
// takes a warp per token with PL experts per lane.
template <int N, int E_T, int PL>
__global__ void __launch_bounds__(THREADS, N <= 16 ? 2 : 1)
    route_kernel(const __grid_constant__ RouteParams p)
{
    constexpr int B_BYTES = N * BK * 2;   // one bf16 term of the W slice
    constexpr int STAGE = A_BYTES + 3 * B_BYTES;
    constexpr int RAW = BK * N * 4;        // fp32 W_r slice of a stage, as staged
    constexpr int N3 = 3 * N;   // hi, mid, lo rows of the B operand
    constexpr uint32_t TMEM_COLS = N3 <= 64 ? 64 : (N3 <= 128 ? 128 : 256);   // power of two
    constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N3 >> 3) << 17) |
                               ((uint32_t)(BM >> 4) << 24);
    constexpr int LS = N + 4;   // row stride (floats) of the partial-logit tile
    constexpr int L_BYTES = BM * LS * 4;
    constexpr int CPL = N * 8 / CONV_LANES;   // 16-byte W chunks per converter lane per stage
    static_assert(N * 8 % CONV_LANES == 0, "chunk split");
    static_assert(L_BYTES + WARPS * (kMaxE + 1) * 4 <= STAGES * STAGE, "select scratch");
    static_assert(STAGES * (STAGE + RAW) + 1024 <= 227 * 1024, "shared memory");
    static_assert(COPY_WARP0 + CONV_LANES / 32 <= WARPS, "roles");
    static_assert(N == 16, "one block per K part covers the layer's E <= 16 experts");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], wfull[STAGES], done;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_rank();
    const int chunk = rank / p.k_parts, part = rank % p.k_parts;
    const int m0 = (blockIdx.x / p.cs) * BM, n0 = chunk * N;
    const int kb0 = part * p.kb_per_part;
    const int kb1 = min(kb0 + p.kb_per_part, p.k_blocks);
    const int nk = kb1 > kb0 ? kb1 - kb0 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            bar_init(saddr(&full[s]), 1 + CONV_LANES / 32);
            bar_init(saddr(&empty[s]), 1);
            bar_init(saddr(&wfull[s]), CONV_LANES);
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
    // inputs (x, W_r, biases) may come from the previous kernel in the stream
    pdl_wait();
    pdl_trigger();
    if (p.clear_status && blockIdx.x == 0 && threadIdx.x == 0)
        *p.status = 0;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer: the x tile of each K block ----
            int last_issue[STAGES];
            for (int s = 0; s < STAGES; ++s)
                last_issue[s] = -1;
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES;
                if (i >= STAGES && !bar_wait(saddr(&empty[s]), (uint32_t)(((i / STAGES) - 1) & 1),
                                             &abort_flag, p.status))
                    break;
                const uint32_t fb = saddr(&full[s]);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb),
                             "r"(A_BYTES)
                             : "memory");
                asm volatile(
                    "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
                    " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(saddr(smem + s * STAGE)),
                    "l"(reinterpret_cast<uint64_t>(&p.tmX)), "r"((kb0 + i) * BK), "r"(m0), "r"(0),
                    "r"(fb)
                    : "memory");
                last_issue[s] = i;
            }
            // copies in flight land before the block moves on (bounded)
            for (int s = 0; s < STAGES; ++s)
                if (last_issue[s] >= 0)
                    bar_wait(saddr(&full[s]), (uint32_t)((last_issue[s] / STAGES) & 1), nullptr,
                             nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer: one bf16 MMA of N = 3 x chunk per K step of 16 ----
            bool any = false;
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES;
                if (!bar_wait(saddr(&full[s]), (uint32_t)((i / STAGES) & 1), &abort_flag,
                              p.status))
                    break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t a = saddr(smem + s * STAGE);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
                    asm volatile(
                        "{\n\t.reg .pred q;\n\t"
                        "setp.ne.b32 q, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q;\n\t}" ::"r"(tmem),
                        "l"(sdesc_sw128(a + kk * 32)), "l"(sdesc_sw128(a + A_BYTES + kk * 32)),
                        "r"(IDESC), "r"(acc)
                        : "memory");
                }
                asm volatile(
                    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
                    "[%0];" ::"r"(saddr(&empty[s]))
                    : "memory");
                any = true;
            }
            if (any)
                asm volatile(
                    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
                    "[%0];" ::"r"(saddr(&done))
                    : "memory");
            else
                bar_arrive(saddr(&done));
        }
    } else if (warp >= COPY_WARP0 && warp < COPY_WARP0 + CONV_LANES / 32) {
        // ---- W_r slice of each K block -> staging slot, 4-byte cp.async ----
        // Lane cl stages the 8 K values of its chunks c = cl + 128 u, where
        // chunk c = (expert row el = c % N, 8-wide K group j = c / N); value q
        // of chunk u sits at (8 u + q) x 128 + cl, so a warp's copies fill
        // consecutive words.
        const int cl = threadIdx.x - COPY_WARP0 * 32;
        float *raw = reinterpret_cast<float *>(smem + STAGES * STAGE);
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            if (i >= STAGES) {
                int ok = 0;
                if (lane == 0)
                    ok = bar_wait(saddr(&empty[s]), (uint32_t)(((i / STAGES) - 1) & 1),
                                  &abort_flag, p.status);
                if (!__shfl_sync(0xffffffffu, ok, 0))
                    break;
            }
            const int kc = (kb0 + i) * BK;
            float *dst = raw + s * (RAW / 4);
#pragma unroll
            for (int u = 0; u < CPL; ++u) {
                const int c = cl + CONV_LANES * u;
                const int el = c % N, j = c / N;
                const int e = n0 + el;
                if (e < p.E) {
                    const float *src = p.W_r + (int64_t)(kc + 8 * j) * p.E + e;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        cp_async4(saddr(dst + (u * 8 + q) * CONV_LANES + cl),
                                  src + (int64_t)q * p.E);
                }
            }
            cp_async_arrive(saddr(&wfull[s]));
        }
        cp_async_wait_all();
    } else if (warp >= CONV_WARP0 && warp < CONV_WARP0 + CONV_LANES / 32) {
        // ---- staged W_r slice -> three bf16 terms, 128-byte swizzle ----
        // Chunk c's 16 bytes sit at row el, position j ^ (el & 7) of the
        // row's eight.  A stage's staging slot is complete once wfull fires,
        // which also means the MMA reading the slot's previous B tiles is done
        // (the copies waited for it).
        const int cl = threadIdx.x - CONV_WARP0 * 32;
        const float *raw = reinterpret_cast<const float *>(smem + STAGES * STAGE);
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            if (!__all_sync(0xffffffffu, bar_wait(saddr(&wfull[s]), (uint32_t)((i / STAGES) & 1),
                                                  &abort_flag, p.status)))
                break;
            uint8_t *b = smem + s * STAGE + A_BYTES;
            const float *src = raw + s * (RAW / 4);
#pragma unroll
            for (int u = 0; u < CPL; ++u) {
                const int c = cl + CONV_LANES * u;
                const int el = c % N, j = c / N;
                float w[8];
                const bool live = n0 + el < p.E;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    w[q] = live ? src[(u * 8 + q) * CONV_LANES + cl] : 0.f;
                uint32_t hi[4], mid[4], lo[4];
#pragma unroll
                for (int q = 0; q < 8; q += 2) {
                    __nv_bfloat16 h[2], md[2], l[2];
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const float x = w[q + r];
                        h[r] = __float2bfloat16_rn(x);
                        const float r1 = x - __bfloat162float(h[r]);
                        md[r] = __float2bfloat16_rn(r1);
                        l[r] = __float2bfloat16_rn(r1 - __bfloat162float(md[r]));
                    }
                    hi[q / 2] = pack2(h[0], h[1]);
                    mid[q / 2] = pack2(md[0], md[1]);
                    lo[q / 2] = pack2(l[0], l[1]);
                }
                const int off = el * 128 + ((j ^ (el & 7)) << 4);
                *reinterpret_cast<uint4 *>(b + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(b + B_BYTES + off) =
                    make_uint4(mid[0], mid[1], mid[2], mid[3]);
                *reinterpret_cast<uint4 *>(b + 2 * B_BYTES + off) =
                    make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            // generic-proxy stores, read next by the tensor core (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0)
                bar_arrive(saddr(&full[s]));
        }

        // ---- accumulator rows -> fp32 partial-logit tile (reuses the ring) ----
        const int ew = warp - CONV_WARP0;   // TMEM lanes 32 ew .. 32 ew + 31
        const bool ok = bar_wait(saddr(&done), 0, nullptr, p.status) && !abort_flag;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        float *L = reinterpret_cast<float *>(smem) + (ew * 32 + lane) * LS;
#pragma unroll
        for (int c = 0; c < N; c += 16) {
            uint32_t r[3][16];
            if (nk > 0) {
#pragma unroll
                for (int sp = 0; sp < 3; ++sp)
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
                        "[%16];"
                        : "=r"(r[sp][0]), "=r"(r[sp][1]), "=r"(r[sp][2]), "=r"(r[sp][3]),
                          "=r"(r[sp][4]), "=r"(r[sp][5]), "=r"(r[sp][6]), "=r"(r[sp][7]),
                          "=r"(r[sp][8]), "=r"(r[sp][9]), "=r"(r[sp][10]), "=r"(r[sp][11]),
                          "=r"(r[sp][12]), "=r"(r[sp][13]), "=r"(r[sp][14]), "=r"(r[sp][15])
                        : "r"(tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(sp * N + c)));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            }
#pragma unroll
            for (int q = 0; q < 16; q += 4) {
                float v[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    // x W_hi + (x W_mid + x W_lo)
                    const float z = __uint_as_float(r[0][q + h]) +
                                    (__uint_as_float(r[1][q + h]) + __uint_as_float(r[2][q + h]));
                    v[h] = nk == 0 ? 0.f : (ok ? z : NAN);
                }
                *reinterpret_cast<float4 *>(L + c + q) = make_float4(v[0], v[1], v[2], v[3]);
            }
        }
    }
    __syncwarp();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();   // every block's partial-logit tile is written
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }

    // ---- selection: this block's share of the tile's tokens ----
    const int TPC = BM / p.cs;                // 128, 64 or 32 tokens
    const int tl0 = rank * TPC;               // first token of the share, within the tile
    const int row0 = (m0 + tl0) / kPartialTokens;
    const bool renorm = p.renorm < 0 ? (p.k > 1) : (p.renorm != 0);
    const uint32_t lbase = saddr(smem);
    uint32_t rb[MAX_CLUSTER];
#pragma unroll
    for (int q = 0; q < MAX_CLUSTER; ++q)
        rb[q] = q < p.cs ? peer_addr(lbase, (uint32_t)q) : 0u;
    float *scratch = reinterpret_cast<float *>(smem + L_BYTES);
    const int E = p.E;

    if constexpr (E_T > 0) {
        // a group = the 32 / E_T tokens one warp holds at once; E_T groups
        // make a row of the loss partials
        constexpr int TB = 32 / E_T;
        const int groups = TPC / TB;
        const int gl = lane % E_T;
        RouteArgs ra{nullptr, nullptr, p.logit_bias, p.select_bias, p.topk, p.gates,
                     p.loss_partials, p.logits_out, p.scores_out, p.T, 0, E, p.k, p.score,
                     p.renorm};
        // the biases of this lane's expert, loaded once
        const float lbv = p.logit_bias && gl < E ? p.logit_bias[gl] : 0.f;
        const float sbv = p.select_bias && gl < E ? p.select_bias[gl] : 0.f;
        for (int g = warp; g < groups; g += WARPS) {
            const int tg = tl0 + g * TB;
            const int tl = tg + lane / E_T;
            float z = -INFINITY;
            if (m0 + tl < p.T && gl < E)
                z = sum_parts(rb, p.k_parts, (uint32_t)(tl * LS + gl) * 4u);
            float pc, zc;
            small_epilogue<E_T>(ra, z, m0 + tg, lane, renorm, lbv, sbv, &pc, &zc);
            if (lane < E_T)
                scratch[g * (E_T + 1) + lane] = pc;
            if (lane == 0)
                scratch[g * (E_T + 1) + E_T] = zc;
        }
        __syncthreads();
        const int rows = TPC / kPartialTokens;
        for (int idx = threadIdx.x; idx < rows * (E + 1); idx += THREADS) {
            const int r = idx / (E + 1), e = idx % (E + 1);
            if ((int64_t)(row0 + r) * kPartialTokens >= p.T)
                continue;
            float acc = 0.f;
            for (int w = 0; w < E_T; ++w)
                acc += scratch[(r * E_T + w) * (E_T + 1) + (e < E ? e : E_T)];
            p.loss_partials[(int64_t)(row0 + r) * (E + 1) + e] = acc;
        }
    } else {
        // a warp per token: warp w takes tokens w, w + 16 of each row of 32;
        // the row's sums meet in shared memory in warp order
        float(*pw)[kMaxE + 1] = reinterpret_cast<float(*)[kMaxE + 1]>(scratch);
        const SelArgs sa = sel_args(p);
        const int rows = TPC / kPartialTokens;
        float lb[PL], sb[PL];   // per-expert biases of this lane, loaded once
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int e = lane + 32 * i;
            lb[i] = p.logit_bias && e < E ? p.logit_bias[e] : 0.f;
            sb[i] = p.select_bias && e < E ? p.select_bias[e] : 0.f;
        }
        for (int r = 0; r < rows; ++r) {
            float pacc[PL];
#pragma unroll
            for (int i = 0; i < PL; ++i)
                pacc[i] = 0.f;
            float zacc = 0.f;
            for (int u = warp; u < kPartialTokens; u += WARPS) {
                const int tl = tl0 + r * kPartialTokens + u;
                const int t = m0 + tl;
                if (t >= p.T)
                    break;
                float z[PL];
#pragma unroll
                for (int i = 0; i < PL; ++i) {
                    const int e = lane + 32 * i;
                    z[i] = -INFINITY;
                    if (e < E) {
                        // one block per tile covers all experts (E <= N)
                        float s = sum_parts(rb, p.k_parts, (uint32_t)(tl * LS + e) * 4u);
                        if (p.logit_bias)
                            s += lb[i];
                        z[i] = s;
                    }
                }
                select_token<PL, true>(sa, renorm, t, lane, z, sb, pacc, zacc);
            }
#pragma unroll
            for (int i = 0; i < PL; ++i)
                if (lane + 32 * i < E)
                    pw[warp][lane + 32 * i] = pacc[i];
            if (lane == 0)
                pw[warp][E] = zacc;
            __syncthreads();
            if ((int64_t)(row0 + r) * kPartialTokens < p.T) {
                float *out = p.loss_partials + (int64_t)(row0 + r) * (E + 1);
                for (int e = threadIdx.x; e <= E; e += THREADS) {
                    float acc = 0.f;
                    for (int w = 0; w < WARPS; ++w)
                        acc += pw[w][e];
                    out[e] = acc;
                }
            }
            __syncthreads();
        }
    }
    cluster_sync();   // the cluster's reads of this block's tile are done
}

// ======================================================= three-launch path
//
// For wider expert sets (E > 16) the W_r split runs once per call instead of
// once per token tile:
//   split  - W_r [d, E] fp32 -> W3 [3][E_pad][d] bf16 (K-major, zero rows past E);
//   logits - grid (token tile of 128, expert chunk of up to 64, K part): TMA ring
//            of x and W3 tiles, three bf16 MMAs per K step, fp32 partial logits
//            [K part][T][E_pad];
//   select - sums the K parts in order, then selects as above.

constexpr int LOGIT_THREADS = 128;   // warp 0: TMA, warp 1: MMA; then all 4 read TMEM

struct __align__(64) LogitParams {
    CUtensorMap tmX;   // x as (d, T, 1)
    CUtensorMap tmW;   // W3 as (d, E_pad, 3)
    float *partial;    // [k_parts][T][E_pad]
    int T, E_pad, n_chunk, kb_per_part, k_blocks;
    int32_t *status;
};

// ---------------------------------------------------------------- split

__global__ void __launch_bounds__(256) split_kernel(const float *__restrict__ W_r, int d, int E,
                                                    int E_pad, __nv_bfloat16 *__restrict__ W3,
                                                    int32_t *status)
{
    pdl_wait();   // W_r may come from the previous kernel in the stream
    pdl_trigger();
    if (status && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        *status = 0;   // cleared before the launches whose waits may set it
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
__global__ void __launch_bounds__(LOGIT_THREADS, 1) logits_kernel(const __grid_constant__ LogitParams p)
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
    pdl_wait();   // the split weights (and x) come from earlier kernels
    pdl_trigger();

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

// Selection of the three-launch path: one block per row of 32 tokens, a warp
// per token, the K parts summed in order; the warps' sums meet in shared
// memory in warp order.
// One block per row of 32 tokens (a row of the loss partials): 32 / NT warps,
// warp w taking tokens w, w + 32 / NT, ... of the row, its NT tokens at once.
// The row's sums meet in shared memory in warp order.  Launched with NT = 4 up
// to 64 experts (four blocks per SM fit, so one wave; 5% faster on the
// DeepSeekMoE shape) and NT = 1 above (eight experts per lane: two tokens per
// warp in 16-warp blocks measured 18% slower on the DeepSeek-V3 shape).
// ONE: a single K part (its logits read straight, no loop over parts).
template <int PL, int NT, bool ONE>
__global__ void __launch_bounds__(32 * kPartialTokens / NT)
    select_kernel(const __grid_constant__ RouteParams a, const float *__restrict__ partial,
                  int parts, int E_pad)
{
    constexpr int W = kPartialTokens / NT;   // warps per block
    __shared__ float pw[W][kMaxE + 1];
    pdl_wait();   // the partial logits come from the logits kernel
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E;
    const bool renorm = a.renorm < 0 ? (a.k > 1) : (a.renorm != 0);
    float pacc[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i)
        pacc[i] = 0.f;
    float zacc = 0.f;
    int tt[NT];
    bool tv[NT];
    float z[NT][PL], sb[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i)
        sb[i] = 0.f;   // unused: the selection biases are read in place
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        tt[n] = blockIdx.x * kPartialTokens + warp + n * W;
        tv[n] = tt[n] < a.T;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int e = lane + 32 * i;
            float s = 0.f;
            if (e < E && tv[n]) {
                if (ONE)
                    s = partial[(int64_t)tt[n] * E_pad + e];
                else
                    for (int q = 0; q < parts; ++q)
                        s += partial[((int64_t)q * a.T + tt[n]) * E_pad + e];
                if (a.logit_bias)
                    s += a.logit_bias[e];
            }
            z[n][i] = s;
        }
    }
    const SelArgs sa = sel_args(a);
    select_tokens<PL, NT, false>(sa, renorm, tt, tv, lane, z, sb, pacc, zacc);
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

// ---------------------------------------------------------------- host

typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (a function-local static is
// initialised once even when several host threads make their first call
// together); null when the driver does not provide it.
EncodeTiled encoder()
{
    static const EncodeTiled fn = []() -> EncodeTiled {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiled>(ptr);
        return nullptr;
    }();
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

// Launch attributes: a cluster of `cluster` blocks, and programmatic
// dependent launch (the kernel may start while the previous kernel in the
// stream finishes; it waits for it with griddepcontrol.wait).
struct LaunchAttrs {
    cudaLaunchAttribute at[2];
    int n = 0;
    LaunchAttrs(int cluster, bool pdl)
    {
        if (cluster >= 1) {
            at[n].id = cudaLaunchAttributeClusterDimension;
            at[n].val.clusterDim.x = (unsigned)cluster;
            at[n].val.clusterDim.y = 1;
            at[n].val.clusterDim.z = 1;
            ++n;
        }
        if (pdl) {
            at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            at[n].val.programmaticStreamSerializationAllowed = 1;
            ++n;
        }
    }
};

template <int N, int E_T, int PL>
cudaError_t launch(const RouteParams &p, unsigned grid, cudaStream_t s)
{
    constexpr int smem = STAGES * (A_BYTES + 3 * N * BK * 2 + BK * N * 4) + 1024;
    auto kern = route_kernel<N, E_T, PL>;
    cudaError_t err = raise_smem_limit((const void *)kern, smem);
    if (err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    LaunchAttrs la(p.cs, true);   // cluster of the K parts; programmatic dependent launch
    cfg.attrs = la.at;
    cfg.numAttrs = la.n;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int N>
cudaError_t launch_logits(const LogitParams &p, dim3 grid, cudaStream_t s)
{
    constexpr int smem = STAGES * (A_BYTES + 3 * N * BK * 2) + 1024;
    auto kern = logits_kernel<N>;
    cudaError_t err = raise_smem_limit((const void *)kern, smem);
    if (err != cudaSuccess)
        return err;
    return launch_pdl(kern, grid, dim3(LOGIT_THREADS), smem, s, p);
}

}  // namespace rtc

RoutePlan route_plan(const moe_config &c)
{
    RoutePlan r{};
    r.tensor_cores = c.dtype == MOE_DTYPE_BF16 && c.d % rtc::BK == 0;
    r.k_blocks = (int)ceil_div(c.d, rtc::BK);
    const int m_tiles = (int)ceil_div(c.T, rtc::BM);
    // One kernel up to 16 experts: each block splits its 16-expert slice of
    // W_r stage by stage as its x tiles stream.  Wider expert sets split W_r
    // once (three launches): a one-kernel form measured slower inside the
    // layer step on the 64- and 256-expert layers.
    if (c.E <= 16) {
        r.fused = true;
        r.n_chunk = 16;
        r.n_chunks = 1;
        r.E_pad = 16;
        // K parts: the most of 4, 2, 1 that keeps the grid within one wave
        // (two blocks per SM) and at least 4 K blocks per part
        r.k_parts = 1;
        for (int kp = rtc::MAX_CLUSTER; kp >= 2; kp /= 2)
            if ((int64_t)m_tiles * kp <= 296 && r.k_blocks / kp >= 4) {
                r.k_parts = kp;
                break;
            }
        r.kb_per_part = (int)ceil_div(r.k_blocks, r.k_parts);
        r.cluster = r.k_parts;
        r.blocks = m_tiles * r.cluster;
        return r;
    }
    r.fused = false;
    r.E_pad = c.E <= 64 ? (int)align_up((size_t)c.E, 16) : (int)align_up((size_t)c.E, 64);
    r.n_chunk = r.E_pad <= 64 ? r.E_pad : 64;
    r.n_chunks = r.E_pad / r.n_chunk;
    const int base = m_tiles * r.n_chunks > 0 ? m_tiles * r.n_chunks : 1;
    // fill about one wave of SMs; keep at least 4 K blocks per part
    const int want = 148 / base;
    int parts = want < r.k_blocks / 4 ? want : r.k_blocks / 4;
    r.k_parts = parts < 1 ? 1 : parts;
    r.kb_per_part = (int)ceil_div(r.k_blocks, r.k_parts);
    r.k_parts = (int)ceil_div(r.k_blocks, r.kb_per_part);
    r.cluster = 1;
    r.blocks = m_tiles * r.n_chunks * r.k_parts;
    return r;
}

size_t route_scratch_bytes(const moe_config &c)
{
    const RoutePlan r = route_plan(c);
    if (!r.tensor_cores || r.fused)
        return 0;
    return align_up((size_t)3 * r.E_pad * c.d * 2, 256) +
           align_up((size_t)r.k_parts * c.T * r.E_pad * 4, 256);
}

cudaError_t launch_route_tc(const moe_config &c, const void *x, const float *W_r,
                            const float *logit_bias, const float *select_bias, int32_t *topk,
                            float *gates, float *partials, float *logits_out, float *scores_out,
                            void *scratch, int32_t *status, bool clear_status, cudaStream_t s)
{
    using namespace rtc;
    const RoutePlan r = route_plan(c);
    RouteParams p;
    memset(&p, 0, sizeof p);
    if (!map3(&p.tmX, x, c.d, c.T, 1, (uint64_t)c.d * 2, (uint64_t)c.d * 2 * c.T, BK, BM))
        return cudaErrorInvalidValue;
    p.W_r = W_r;
    p.logit_bias = logit_bias;
    p.select_bias = select_bias;
    p.topk = topk;
    p.gates = gates;
    p.loss_partials = partials;
    p.logits_out = logits_out;
    p.scores_out = scores_out;
    p.T = c.T;
    p.d = c.d;
    p.E = c.E;
    p.k = c.k;
    p.score = c.score;
    p.renorm = c.renorm;
    p.cs = r.cluster;
    p.k_parts = r.k_parts;
    p.kb_per_part = r.kb_per_part;
    p.k_blocks = r.k_blocks;
    p.status = status;
    p.clear_status = clear_status ? 1 : 0;
    if (r.fused) {
        const unsigned grid = (unsigned)r.blocks;
        if (c.E <= 4)
            return launch<16, 4, 1>(p, grid, s);
        if (c.E <= 8)
            return launch<16, 8, 1>(p, grid, s);
        return launch<16, 0, 1>(p, grid, s);
    }

    // three launches: split, logits, select
    __nv_bfloat16 *W3 = static_cast<__nv_bfloat16 *>(scratch);
    float *plog = reinterpret_cast<float *>(static_cast<char *>(scratch) +
                                            align_up((size_t)3 * r.E_pad * c.d * 2, 256));
    dim3 sg((unsigned)ceil_div(c.d, 32), (unsigned)ceil_div(r.E_pad, 32));
    cudaError_t err = launch_pdl(split_kernel, sg, dim3(256), 0, s, W_r, c.d, c.E, r.E_pad, W3,
                                 clear_status ? status : nullptr);
    if (err != cudaSuccess)
        return err;
    LogitParams lp;
    memset(&lp, 0, sizeof lp);
    lp.tmX = p.tmX;
    if (!map3(&lp.tmW, W3, c.d, r.E_pad, 3, (uint64_t)c.d * 2, (uint64_t)c.d * 2 * r.E_pad, BK,
              r.n_chunk))
        return cudaErrorInvalidValue;
    lp.partial = plog;
    lp.T = c.T;
    lp.E_pad = r.E_pad;
    lp.n_chunk = r.n_chunk;
    lp.kb_per_part = r.kb_per_part;
    lp.k_blocks = r.k_blocks;
    lp.status = status;
    dim3 grid((unsigned)ceil_div(c.T, BM), (unsigned)r.n_chunks, (unsigned)r.k_parts);
    switch (r.n_chunk) {
    case 16: err = launch_logits<16>(lp, grid, s); break;
    case 32: err = launch_logits<32>(lp, grid, s); break;
    case 48: err = launch_logits<48>(lp, grid, s); break;
    default: err = launch_logits<64>(lp, grid, s); break;
    }
    if (err != cudaSuccess)
        return err;
    const unsigned rows = (unsigned)ceil_div(c.T, kPartialTokens);
    const float *pl = plog;
    const bool one = r.k_parts == 1;
    if (c.E <= 32)
        err = one ? launch_pdl(select_kernel<1, 4, true>, dim3(rows), dim3(32 * kPartialTokens / 4),
                               0, s, p, pl, r.k_parts, r.E_pad)
                  : launch_pdl(select_kernel<1, 4, false>, dim3(rows),
                               dim3(32 * kPartialTokens / 4), 0, s, p, pl, r.k_parts, r.E_pad);
    else if (c.E <= 64)
        err = one ? launch_pdl(select_kernel<2, 4, true>, dim3(rows), dim3(32 * kPartialTokens / 4),
                               0, s, p, pl, r.k_parts, r.E_pad)
                  : launch_pdl(select_kernel<2, 4, false>, dim3(rows),
                               dim3(32 * kPartialTokens / 4), 0, s, p, pl, r.k_parts, r.E_pad);
    else if (c.E <= 128)
        err = one ? launch_pdl(select_kernel<4, 1, true>, dim3(rows), dim3(32 * kPartialTokens), 0,
                               s, p, pl, r.k_parts, r.E_pad)
                  : launch_pdl(select_kernel<4, 1, false>, dim3(rows), dim3(32 * kPartialTokens),
                               0, s, p, pl, r.k_parts, r.E_pad);
    else
        err = one ? launch_pdl(select_kernel<8, 1, true>, dim3(rows), dim3(32 * kPartialTokens), 0,
                               s, p, pl, r.k_parts, r.E_pad)
                  : launch_pdl(select_kernel<8, 1, false>, dim3(rows), dim3(32 * kPartialTokens),
                               0, s, p, pl, r.k_parts, r.E_pad);
    return err;
}

}  // namespace moe
