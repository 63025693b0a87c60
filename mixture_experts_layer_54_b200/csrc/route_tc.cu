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
// Up to 64 experts: one persistent kernel (details at route_kernel).  The
// blocks of a thread-block cluster split K; each splits its part of W_r into
// the three terms once, keeps them in shared memory as the MMA's B operand
// (hi, mid and lo stacked as 3 E_pad rows, so one MMA per K step gives the
// three products side by side in TMEM), and streams 128-token x tiles by TMA
// through a double-buffered TMEM accumulator.  Each block then selects its
// share of a tile's tokens, summing the K parts' partial logits in order
// through distributed shared memory: softmax or sigmoid, top-k (ties to the
// lower index), gates, optional logits/scores, and the rows of the loss
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
constexpr int STAGES = 4;              // TMA ring of the three-launch logits kernel
constexpr int A_BYTES = BM * BK * 2;   // 16 KB: one x tile of a K block

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
// set.  CLUSTER: acquire at cluster scope, for barriers that blocks of the
// cluster complete remotely.  (A suspend-time hint on the tries, letting the
// thread sleep until the phase completes, measured slower here: woken threads
// resumed up to microseconds after the phase completed.)
template <bool CLUSTER>
__device__ __noinline__ bool bar_wait_t(uint32_t bar, uint32_t parity, volatile int *abort,
                                        int32_t *status)
{
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t ok;
        if (CLUSTER)
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(ok)
                : "r"(bar), "r"(parity)
                : "memory");
        else
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

__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                         int32_t *status)
{
    return bar_wait_t<false>(bar, parity, abort, status);
}

// The same wait for a whole warp: every lane polls, the warp agrees on the
// outcome.  (Polling by lane 0 alone, the others waiting at a shuffle,
// measured slower: 9.4 against 12.1 us for the Switch-shaped router.)
template <bool CLUSTER>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          int32_t *status)
{
    return __all_sync(0xffffffffu, bar_wait_t<CLUSTER>(bar, parity, abort, status));
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
    int tiles, nclusters, stages;   // one-kernel router: token tiles, clusters, x stages
    int clear_status;               // 1: block 0 clears the status word first
    int w_bulk;                     // 1: W_r is 16-byte aligned (its K parts copied in bulk)
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
//
// One kernel for up to 64 experts.  The blocks of a cluster split K into P
// parts (P = cluster size, 1, 2 or 4); block `rank` owns K blocks
// [rank kbp, (rank + 1) kbp).  The cluster walks token tiles of 128
// (tile = cluster, cluster + clusters, ...), so one cluster may take several.
//   prologue     warps 2-13 split this block's K part of W_r into the three
//                bf16 terms, K-major in the 128-byte swizzle, once (all of a
//                thread's loads issued before any conversion): the B operand
//                of every tile stays in shared memory;
//   warp 0       TMA ring of x tiles (one thread), as deep as shared memory
//                allows;
//   warp 1       one MMA of N = 3 NE per K step of 16 into one of two TMEM
//                accumulators (tile i uses buffer i mod 2);
//   warps 2-5    read an accumulator back (hi + (mid + lo)) and push each
//                token's partial logits into buffer i mod 2 of the block that
//                selects that token (st.async, slot = this block's K part):
//                each store's bytes count on that block's lfull barrier, so
//                no fence or remote arrive follows the pushes;
//   warps 6-13   select 128 / P tokens of the tile from their own buffer once
//                its BM x NE floats have landed, summing the P parts in part
//                order; then arm the buffer's barrier for its next use and
//                tell every block that the buffer may be filled again.
// So one tile's read-back and selection run while the next tile's x streams,
// and no warp waits on a remote load.

constexpr int PR_THREADS = 448;   // 14 warps
constexpr int RB_WARP0 = 2;       // warps 2-5: TMEM read-back
constexpr int SEL_WARP0 = 6;      // warps 6-13: selection
constexpr int SEL_WARPS = 8;
constexpr int SEL_THREADS = SEL_WARPS * 32;
static_assert(RB_WARP0 == 2 && SEL_WARP0 == RB_WARP0 + 4, "warps 0, 1: TMA, MMA; then 4 read-back");
constexpr int CONV_WARP0 = 2;     // warps 2-13 split W_r first
constexpr int CONV_THREADS = PR_THREADS - CONV_WARP0 * 32;
constexpr int MAX_STAGES = 8;
constexpr int W_MAX_BYTES = 112 * 1024;   // resident split weights per block

// This warp's 32 TMEM lanes x 16 (or 8) consecutive fp32 columns from taddr.
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

// Asynchronous store of four floats to shared memory of a block of the
// cluster (a and bar are cluster shared addresses of that block): when the 16
// bytes have landed they count against the transaction bytes the block's
// mbarrier bar expects, so the reader needs no fence or arrive from the writer.
__device__ __forceinline__ void st_async4(uint32_t a, float4 v, uint32_t bar)
{
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, "
        "[%5];" ::"r"(a),
        "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
        : "memory");
}

// Arrive on a barrier of this block, first raising the transaction bytes its
// current phase waits for.
__device__ __forceinline__ void arrive_expect(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// Named barriers (id 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Arrive on the mbarrier at the same shared offset in block `rank` of the
// cluster, with no memory ordering: a bare "go" signal.
__device__ __forceinline__ void arrive_remote_relaxed(uint32_t bar, uint32_t rank)
{
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                     peer_addr(bar, rank))
                 : "memory");
}

// Shared-memory plan of the kernel (host and device agree on it).
struct RouteSmem {
    int w, x, l, scratch, total;
};
__host__ __device__ inline RouteSmem route_smem(int NE, int kbp, int stages)
{
    RouteSmem s;
    const int N3 = (3 * NE + 15) / 16 * 16;   // the MMA's N: hi, mid, lo rows, padded
    s.w = 0;
    s.x = (kbp * N3 * 128 + 1023) / 1024 * 1024;
    s.l = s.x + stages * A_BYTES;
    const int l_bytes = BM * (NE + 4) * 4;
    s.scratch = s.l + 2 * l_bytes;
    // selection sums: a row per selection warp, or (E <= 8) up to 32 groups of 9
    const int sc = SEL_WARPS * (NE + 1) > 32 * 9 ? SEL_WARPS * (NE + 1) : 32 * 9;
    s.total = s.scratch + sc * 4 + 1024;   // + alignment slack
    return s;
}

// NE: experts per MMA (E padded to 8, 16, 32, 48 or 64).  Selection: E_T > 0
// (NE = 8) takes E <= E_T experts with E_T lanes per token (32 / E_T tokens per
// warp at once); E_T == 0 takes a warp per token with NE / 32 (rounded up)
// experts per lane, four tokens per warp at once.
template <int NE, int E_T>
__global__ void __launch_bounds__(PR_THREADS, 1) route_kernel(const __grid_constant__ RouteParams p)
{
    constexpr int N3 = (3 * NE + 15) / 16 * 16;      // hi, mid, lo rows of B (+ zero rows)
    constexpr int WT_BYTES = N3 * 128;               // one K block of B
    constexpr uint32_t ACC = N3 <= 64 ? 64 : (N3 <= 128 ? 128 : 256);   // columns per buffer
    constexpr uint32_t TMEM_COLS = 2 * ACC;
    constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N3 >> 3) << 17) |
                               ((uint32_t)(BM >> 4) << 24);
    constexpr int LS = NE + 4;                       // row stride (floats) of a logit buffer
    constexpr int L_BYTES = BM * LS * 4;
    constexpr int L_PUSH = BM * NE * 4;              // bytes pushed into a buffer per tile
    static_assert(N3 % 16 == 0 && N3 <= 256, "MMA N");
    static_assert(NE == 8 || NE % 16 == 0, "experts per MMA: 8 or a multiple of 16");
    static_assert((E_T > 0) == (NE == 8), "narrow selection exactly on the 8-expert layout");
    constexpr int PL = (NE + 31) / 32;               // experts per lane, a warp per token

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[MAX_STAGES], empty[MAX_STAGES], wready, wbar, tfull[2],
        tempty[2], lfull[2], lempty[2], drain;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    // Set by a read-back (selection) warp whose bounded wait gave up, read by
    // its whole group after a named barrier, so the group leaves its loop
    // together and no warp waits at a named barrier for one that left.
    __shared__ int rb_fail, sel_fail;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.cs, ST = p.stages;
    const int rank = (int)cluster_rank();
    const int cl = blockIdx.x / P, ncl = p.nclusters;
    const int kbp = p.kb_per_part, kb0 = rank * kbp;
    const RouteSmem sm = route_smem(NE, kbp, ST);
    uint8_t *Wres = smem + sm.w;
    uint8_t *X = smem + sm.x;
    const uint32_t lbase = saddr(smem + sm.l);
    const int TPC = BM / P;   // tokens of a tile this block selects (128, 64 or 32)

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            bar_init(saddr(&full[s]), 1);
            bar_init(saddr(&empty[s]), 1);
        }
        bar_init(saddr(&wready), CONV_THREADS / 32);
        bar_init(saddr(&wbar), 1);
        for (int a = 0; a < 2; ++a) {
            bar_init(saddr(&tfull[a]), 1);
            bar_init(saddr(&tempty[a]), 4);
            // a phase of lfull[a]: this block's own arrive, which also sets the
            // bytes the cluster's read-back pushes into buffer a (BM rows of NE
            // floats: TPC rows from each of the P blocks)
            bar_init(saddr(&lfull[a]), 1);
            bar_init(saddr(&lempty[a]), (uint32_t)P);
        }
        bar_init(saddr(&drain), 1);
        abort_flag = 0;
        rb_fail = 0;
        sel_fail = 0;
        for (int a = 0; a < 2; ++a)   // the first use of each buffer
            arrive_expect(saddr(&lfull[a]), (uint32_t)L_PUSH);
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
    cluster_sync();   // every block's barriers exist before anyone arrives remotely
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_slot;

    // inputs (x, W_r, biases) may come from the previous kernel in the stream
    pdl_wait();
    pdl_trigger();
    if (p.clear_status && blockIdx.x == 0 && threadIdx.x == 0)
        *p.status = 0;

    if (warp >= CONV_WARP0) {
        // ---- prologue: this block's K part of W_r -> three bf16 terms ----
        // Chunk c = (K block i, 8-wide K group j, expert e < E), e fastest;
        // its 16 bytes of each term go to row e (+ NE, + 2 NE) of K block i's
        // tile, at position j ^ (row & 7) of the row's eight (128-byte
        // swizzle).  The part (kbp x 64 rows of E floats, contiguous in W_r)
        // arrives by bulk copies into the tail of the split-weight region,
        // issued by the TMA thread ahead of any x tile; every thread reads all
        // of its chunks (at most CB: 8 kbp E <= 8 kbp NE <= CB x 384 on every
        // layer this kernel takes) before any thread writes a term over the
        // staged part.  Without 16-byte alignment the threads load the part
        // from global memory themselves.
        constexpr int CB = 6;
        const int ct = threadIdx.x - CONV_WARP0 * 32;
        const int E = p.E, nchunk = kbp * 8 * E;
        const float *stage =
            reinterpret_cast<const float *>(Wres + kbp * WT_BYTES - kbp * BK * E * 4);
        if (p.w_bulk)   // expiry: recorded, go on
            warp_wait<false>(saddr(&wbar), 0, &abort_flag, p.status);
        float w[CB][8];
#pragma unroll
        for (int b = 0; b < CB; ++b) {
            const int c = ct + b * CONV_THREADS;
            const int e = c % E, j = (c / E) % 8, i = c / (E * 8);
            const int r0 = i * BK + 8 * j;   // row of the part
#pragma unroll
            for (int u = 0; u < 8; ++u)
                w[b][u] = c >= nchunk ? 0.f
                          : p.w_bulk  ? stage[(r0 + u) * E + e]
                                      : p.W_r[((int64_t)kb0 * BK + r0 + u) * E + e];
        }
        named_sync(3, CONV_THREADS);   // the staged part is read: terms may overwrite it
#pragma unroll
        for (int b = 0; b < CB; ++b) {
            const int c = ct + b * CONV_THREADS;
            if (c >= nchunk)
                break;
            const int e = c % E, j = (c / E) % 8, i = c / (E * 8);
            uint32_t hi[4], mid[4], lo[4];
#pragma unroll
            for (int u = 0; u < 8; u += 2) {
                __nv_bfloat16 h[2], md[2], l[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float x = w[b][u + r];
                    h[r] = __float2bfloat16_rn(x);
                    const float r1 = x - __bfloat162float(h[r]);
                    md[r] = __float2bfloat16_rn(r1);
                    l[r] = __float2bfloat16_rn(r1 - __bfloat162float(md[r]));
                }
                hi[u / 2] = pack2(h[0], h[1]);
                mid[u / 2] = pack2(md[0], md[1]);
                lo[u / 2] = pack2(l[0], l[1]);
            }
            uint8_t *tile = Wres + i * WT_BYTES;
            const uint32_t *terms[3] = {hi, mid, lo};
#pragma unroll
            for (int sp = 0; sp < 3; ++sp) {
                const int row = sp * NE + e;
                *reinterpret_cast<uint4 *>(tile + row * 128 + ((j ^ (row & 7)) << 4)) =
                    make_uint4(terms[sp][0], terms[sp][1], terms[sp][2], terms[sp][3]);
            }
        }
        // zero rows: the padding experts E .. NE - 1 of every term, and the
        // rows 3 NE .. N3 - 1 that round the MMA's N up to a multiple of 16
        const int dead = NE - E, zrows = 3 * dead + (N3 - 3 * NE), nz = kbp * zrows * 8;
        for (int z = ct; z < nz; z += CONV_THREADS) {
            const int q16 = z % 8, zr = (z / 8) % zrows, i = z / (8 * zrows);
            const int row = zr < 3 * dead ? (zr / dead) * NE + E + zr % dead : 3 * NE + zr - 3 * dead;
            *reinterpret_cast<uint4 *>(Wres + i * WT_BYTES + row * 128 + q16 * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        // generic-proxy stores, read next by the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0)
            bar_arrive(saddr(&wready));
    }

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer: the x tile of every K block of every tile ----
            int it = 0;
            int last_issue[MAX_STAGES];
            for (int s = 0; s < MAX_STAGES; ++s)
                last_issue[s] = -1;
            // this block's K part of W_r first, in pieces of up to 16 KB
            const uint32_t wbytes = (uint32_t)(kbp * BK * p.E * 4);
            if (p.w_bulk) {
                const uint32_t wb = saddr(&wbar);
                const uint32_t dst = saddr(Wres + kbp * WT_BYTES) - wbytes;
                const char *src = reinterpret_cast<const char *>(p.W_r + (int64_t)kb0 * BK * p.E);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(wb),
                             "r"(wbytes)
                             : "memory");
                for (uint32_t o = 0; o < wbytes; o += 16384) {
                    const uint32_t n = wbytes - o < 16384 ? wbytes - o : 16384;
                    asm volatile(
                        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], "
                        "%2, [%3];" ::"r"(dst + o),
                        "l"(src + o), "r"(n), "r"(wb)
                        : "memory");
                }
            }
            // x waits until the terms are written: issued together, the whole
            // grid's first x tiles (stages x 16 KB per block) would share the
            // memory system with W_r, and the converters' proxy fence would
            // wait for them to land
            bool ok = bar_wait(saddr(&wready), 0, &abort_flag, p.status);
            for (int tile = cl; ok && tile < p.tiles; tile += ncl) {
                for (int i = 0; i < kbp; ++i, ++it) {
                    const int s = it % ST;
                    if (it >= ST && !bar_wait(saddr(&empty[s]), (uint32_t)(((it / ST) - 1) & 1),
                                              &abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = saddr(&full[s]);
                    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb),
                                 "r"(A_BYTES)
                                 : "memory");
                    asm volatile(
                        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::"
                        "bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(saddr(X + s * A_BYTES)),
                        "l"(reinterpret_cast<uint64_t>(&p.tmX)), "r"((kb0 + i) * BK),
                        "r"(tile * BM), "r"(0), "r"(fb)
                        : "memory");
                    last_issue[s] = it;
                }
            }
            // copies in flight land before the block moves on (bounded)
            if (p.w_bulk)
                bar_wait(saddr(&wbar), 0, nullptr, nullptr);
            for (int s = 0; s < ST; ++s)
                if (last_issue[s] >= 0)
                    bar_wait(saddr(&full[s]), (uint32_t)((last_issue[s] / ST) & 1), nullptr,
                             nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer ----
            bool ok = bar_wait(saddr(&wready), 0, &abort_flag, p.status);
            bool any = false;
            int it = 0, tc = 0;
            for (int tile = cl; ok && tile < p.tiles; tile += ncl, ++tc) {
                const int a = tc & 1;
                if (!bar_wait(saddr(&tempty[a]), (uint32_t)(((tc >> 1) & 1) ^ 1), &abort_flag,
                              p.status))
                    break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t d = tmem + (uint32_t)a * ACC;
                for (int i = 0; i < kbp; ++i, ++it) {
                    const int s = it % ST;
                    if (!bar_wait(saddr(&full[s]), (uint32_t)((it / ST) & 1), &abort_flag,
                                  p.status)) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t xa = saddr(X + s * A_BYTES), wb = saddr(Wres + i * WT_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred q;\n\t"
                            "setp.ne.b32 q, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q;\n\t}" ::"r"(d),
                            "l"(sdesc_sw128(xa + kk * 32)), "l"(sdesc_sw128(wb + kk * 32)),
                            "r"(IDESC), "r"(acc)
                            : "memory");
                    }
                    asm volatile(
                        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
                        "[%0];" ::"r"(saddr(&empty[s]))
                        : "memory");
                    any = true;
                }
                if (!ok)
                    break;
                asm volatile(
                    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
                    "[%0];" ::"r"(saddr(&tfull[a]))
                    : "memory");
            }
            if (any) {   // every MMA issued has completed before TMEM is freed
                asm volatile(
                    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
                    "[%0];" ::"r"(saddr(&drain))
                    : "memory");
                bar_wait(saddr(&drain), 0, nullptr, p.status);
            }
        }
    } else if (warp < SEL_WARP0) {
        // ---- accumulator -> this block's partial-logit buffer ----
        const int q = warp & 3;   // TMEM lanes 32 q .. 32 q + 31
        int tc = 0;
        for (int tile = cl; tile < p.tiles; tile += ncl, ++tc) {
            const int a = tc & 1, n = tc >> 1;
            bool okw = warp_wait<false>(saddr(&tfull[a]), (uint32_t)(n & 1), &abort_flag, p.status);
            // the cluster's selection of the tile that last used this buffer is done
            if (okw)
                okw = warp_wait<false>(saddr(&lempty[a]), (uint32_t)((n & 1) ^ 1), &abort_flag,
                                       p.status);
            if (!okw && lane == 0)
                rb_fail = 1;
            named_sync(1, 128);
            if (rb_fail)
                break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // this lane's token row goes to the block selecting it, slot
            // `rank`; the owner's lfull[a] counts the bytes as they land
            const int row = q * 32 + lane, owner = row / TPC, tl = row % TPC;
            const uint32_t dst = peer_addr(lbase, (uint32_t)owner) +
                                 (uint32_t)(a * L_BYTES + (rank * TPC + tl) * LS * 4);
            const uint32_t dbar = peer_addr(saddr(&lfull[a]), (uint32_t)owner);
            const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)a * ACC;
            constexpr int CW = NE < 16 ? NE : 16;   // columns per load and term
#pragma unroll
            for (int c = 0; c < NE; c += CW) {
                uint32_t r[3][CW];
#pragma unroll
                for (int sp = 0; sp < 3; ++sp)
                    tmem_ld_cols(tb + (uint32_t)(sp * NE + c), r[sp]);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (int h = 0; h < CW; h += 4) {
                    float v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)   // x W_hi + (x W_mid + x W_lo)
                        v[u] = __uint_as_float(r[0][h + u]) +
                               (__uint_as_float(r[1][h + u]) + __uint_as_float(r[2][h + u]));
                    st_async4(dst + (uint32_t)((c + h) * 4), make_float4(v[0], v[1], v[2], v[3]),
                              dbar);
                }
            }
            // accumulator free for the tile after next
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0)
                bar_arrive(saddr(&tempty[a]));
        }
    } else {
        // ---- selection: this block's share of every tile's tokens ----
        // buffer a holds [part q][token tl of the share][expert]
        const int st = threadIdx.x - SEL_WARP0 * 32;
        const int E = p.E;
        const int sw = warp - SEL_WARP0;   // selection warp 0..7
        const int tl0 = rank * TPC;
        const bool renorm = p.renorm < 0 ? (p.k > 1) : (p.renorm != 0);
        const SelArgs sa = sel_args(p);
        float *scratch = reinterpret_cast<float *>(smem + sm.scratch);
        float lb[PL], sb[PL];   // per-expert biases of this lane, loaded once
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int e = lane + 32 * i;
            lb[i] = p.logit_bias && e < E ? p.logit_bias[e] : 0.f;
            sb[i] = p.select_bias && e < E ? p.select_bias[e] : 0.f;
        }
        // narrow layers: lane L serves expert L % E_T
        const int gle = E_T > 0 ? lane % (E_T > 0 ? E_T : 1) : 0;
        const float lbv = E_T > 0 && p.logit_bias && gle < E ? p.logit_bias[gle] : 0.f;
        const float sbv = E_T > 0 && p.select_bias && gle < E ? p.select_bias[gle] : 0.f;
        int tc = 0;
        for (int tile = cl; tile < p.tiles; tile += ncl, ++tc) {
            const int a = tc & 1, n = tc >> 1;
            const bool okw =
                warp_wait<true>(saddr(&lfull[a]), (uint32_t)(n & 1), &abort_flag, p.status);
            if (!okw && lane == 0)
                sel_fail = 1;
            named_sync(2, SEL_THREADS);
            if (sel_fail)
                break;
            const int m0 = tile * BM;
            const int row0 = (m0 + tl0) / kPartialTokens;
            const int rows = TPC / kPartialTokens;
            const float *Lb = reinterpret_cast<const float *>(smem + sm.l + a * L_BYTES);
            if constexpr (E_T > 0) {
                // a group = the 32 / E_T tokens one warp holds at once; E_T
                // groups make a row of the loss partials
                constexpr int TB = 32 / E_T;
                const int groups = TPC / TB;
                const int gl = lane % E_T;
                RouteArgs ra{nullptr, nullptr, p.logit_bias, p.select_bias, p.topk, p.gates,
                             p.loss_partials, p.logits_out, p.scores_out, p.T, 0, E, p.k,
                             p.score, p.renorm};
                for (int g = sw; g < groups; g += SEL_WARPS) {
                    const int tg = tl0 + g * TB;
                    const int tl = tg + lane / E_T;
                    float z = -INFINITY;
                    if (m0 + tl < p.T && gl < E) {
                        z = 0.f;
                        for (int q = 0; q < P; ++q)
                            z += Lb[(q * TPC + tl - tl0) * LS + gl];
                    }
                    float pc, zc;
                    small_epilogue<E_T>(ra, z, m0 + tg, lane, renorm, lbv, sbv, &pc, &zc);
                    if (lane < E_T)
                        scratch[g * (E_T + 1) + lane] = pc;
                    if (lane == 0)
                        scratch[g * (E_T + 1) + E_T] = zc;
                }
                named_sync(2, SEL_THREADS);   // every group's sums are in scratch
                for (int idx = st; idx < rows * (E + 1); idx += SEL_THREADS) {
                    const int r = idx / (E + 1), e = idx % (E + 1);
                    if ((int64_t)(row0 + r) * kPartialTokens >= p.T)
                        continue;
                    float acc = 0.f;
                    for (int w = 0; w < E_T; ++w)
                        acc += scratch[(r * E_T + w) * (E_T + 1) + (e < E ? e : E_T)];
                    p.loss_partials[(int64_t)(row0 + r) * (E + 1) + e] = acc;
                }
                named_sync(2, SEL_THREADS);   // scratch free, every read of the buffers done
            } else {
                // selection warp w takes tokens w, w + 8, w + 16 and w + 24 of
                // each row of 32, all four at once, a whole warp per token; the
                // row's sums meet in shared memory in warp order
                for (int r = 0; r < rows; ++r) {
                    float pacc[PL];
#pragma unroll
                    for (int i = 0; i < PL; ++i)
                        pacc[i] = 0.f;
                    float zacc = 0.f;
                    // the warp's tokens of the row (sw, sw + 8, ...) at once
                    constexpr int NT = kPartialTokens / SEL_WARPS;
                    int tt[NT];
                    bool tv[NT];
                    float z[NT][PL];
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const int tl = tl0 + r * kPartialTokens + sw + n * SEL_WARPS;
                        tt[n] = m0 + tl;
                        tv[n] = tt[n] < p.T;
#pragma unroll
                        for (int i = 0; i < PL; ++i) {
                            const int e = lane + 32 * i;
                            float sum = 0.f;
                            if (e < E && tv[n]) {
                                for (int q = 0; q < P; ++q)
                                    sum += Lb[(q * TPC + tl - tl0) * LS + e];
                                if (p.logit_bias)
                                    sum += lb[i];
                            }
                            z[n][i] = sum;
                        }
                    }
                    select_tokens<PL, NT, true>(sa, renorm, tt, tv, lane, z, sb, pacc, zacc);
#pragma unroll
                    for (int i = 0; i < PL; ++i)
                        if (lane + 32 * i < E)
                            scratch[sw * (NE + 1) + lane + 32 * i] = pacc[i];
                    if (lane == 0)
                        scratch[sw * (NE + 1) + E] = zacc;
                    named_sync(2, SEL_THREADS);
                    if ((int64_t)(row0 + r) * kPartialTokens < p.T) {
                        float *out = p.loss_partials + (int64_t)(row0 + r) * (E + 1);
                        for (int e = st; e <= E; e += SEL_THREADS) {
                            float acc = 0.f;
                            for (int w = 0; w < SEL_WARPS; ++w)
                                acc += scratch[w * (NE + 1) + e];
                            out[e] = acc;
                        }
                    }
                    named_sync(2, SEL_THREADS);
                }
            }
            // this block is done reading buffer a: arm it for its next use,
            // then let every block of the cluster push into it again
            if (st == 0) {
                arrive_expect(saddr(&lfull[a]), (uint32_t)L_PUSH);
                // relaxed: every read of the buffer returned its value before
                // the named barrier above, so later pushes cannot change them
                for (int r = 0; r < P; ++r)
                    arrive_remote_relaxed(saddr(&lempty[a]), (uint32_t)r);
            }
        }
    }

    // ---- tear-down: no block leaves while the cluster may read its buffers ----
    __syncwarp();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }
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
template <int PL>
__global__ void __launch_bounds__(32 * kPartialTokens, 1)
    select_kernel(const __grid_constant__ RouteParams a, const float *__restrict__ partial,
                  int parts, int E_pad)
{
    constexpr int W = kPartialTokens;
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
        float z[PL], sb[PL];
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int e = lane + 32 * i;
            z[i] = -INFINITY;
            sb[i] = 0.f;   // unused: the biases are read in place
            if (e < E) {
                float s = 0.f;
                for (int q = 0; q < parts; ++q)
                    s += partial[((int64_t)q * a.T + t) * E_pad + e];
                if (a.logit_bias)
                    s += a.logit_bias[e];
                z[i] = s;
            }
        }
        const SelArgs sa = sel_args(a);
        select_token<PL, false>(sa, renorm, t, lane, z, sb, pacc, zacc);
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

template <int NE, int E_T>
cudaError_t launch(RouteParams p, cudaStream_t s)
{
    auto kern = route_kernel<NE, E_T>;
    const int smem = route_smem(NE, p.kb_per_part, p.stages).total;
    cudaError_t err = raise_smem_limit((const void *)kern, smem);
    if (err != cudaSuccess)
        return err;
    // as many clusters as fit at once (every block must be resident: blocks of
    // a cluster wait on one another), at most one per tile, the tiles spread
    // evenly over them
    int fit = 0;
    err = cached_active_clusters((const void *)kern, PR_THREADS, smem, p.cs, &fit);
    if (err != cudaSuccess)
        return err;
    if (fit < 1)
        return cudaErrorInvalidConfiguration;
    const int per = (int)ceil_div(p.tiles, fit);
    p.nclusters = (int)ceil_div(p.tiles, per);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.blockDim = dim3(PR_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.gridDim = dim3((unsigned)(p.nclusters * p.cs));
    LaunchAttrs lp(p.cs, true);
    cfg.attrs = lp.at;
    cfg.numAttrs = lp.n;
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
    kern<<<grid, LOGIT_THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace rtc

RoutePlan route_plan(const moe_config &c)
{
    RoutePlan r{};
    r.tensor_cores = c.dtype == MOE_DTYPE_BF16 && c.d % rtc::BK == 0;
    r.k_blocks = (int)ceil_div(c.d, rtc::BK);
    const int m_tiles = (int)ceil_div(c.T, rtc::BM);
    // One kernel up to 64 experts when a block's K part of the split weights
    // (3 E_pad rows, padded to a multiple of 16, x 128 bytes per K block;
    // E_pad = 8 up to 8 experts, else E rounded up to 16) stays resident in
    // shared memory: K split in P = 4 parts (or 2, 1 for short K), at least 4
    // K blocks each.
    if (c.E <= 64) {
        const int E_pad = c.E <= 8 ? 8 : (int)align_up((size_t)c.E, 16);
        const int N3 = (3 * E_pad + 15) / 16 * 16;
        int P = 4;
        while (P > 1 && (r.k_blocks % P != 0 || r.k_blocks / P < 4))
            P /= 2;
        const int kbp = r.k_blocks / P;
        int stages = rtc::MAX_STAGES;
        while (stages > 2 && rtc::route_smem(E_pad, kbp, stages).total > 227 * 1024)
            --stages;
        if (kbp * N3 * 128 <= rtc::W_MAX_BYTES &&
            rtc::route_smem(E_pad, kbp, stages).total <= 227 * 1024) {
            r.fused = true;
            r.E_pad = E_pad;
            r.n_chunk = E_pad;
            r.n_chunks = 1;
            r.k_parts = P;
            r.kb_per_part = kbp;
            r.cluster = P;
            r.stages = stages;
            r.blocks = m_tiles * P;   // upper bound; the launch sizes the persistent grid
            return r;
        }
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
    // a K part of W_r (kbp x 64 rows of E floats, contiguous) comes in by bulk
    // copies when W_r is 16-byte aligned, else by per-thread loads
    p.w_bulk = reinterpret_cast<uintptr_t>(W_r) % 16 == 0 ? 1 : 0;
    if (r.fused) {
        p.tiles = (int)ceil_div(c.T, BM);
        p.stages = r.stages;
        if (c.E <= 4)
            return launch<8, 4>(p, s);
        if (c.E <= 8)
            return launch<8, 8>(p, s);
        if (c.E <= 16)
            return launch<16, 0>(p, s);
        if (c.E <= 32)
            return launch<32, 0>(p, s);
        if (c.E <= 48)
            return launch<48, 0>(p, s);
        return launch<64, 0>(p, s);
    }

    // three launches: split, logits, select
    __nv_bfloat16 *W3 = static_cast<__nv_bfloat16 *>(scratch);
    float *plog = reinterpret_cast<float *>(static_cast<char *>(scratch) +
                                            align_up((size_t)3 * r.E_pad * c.d * 2, 256));
    dim3 sg((unsigned)ceil_div(c.d, 32), (unsigned)ceil_div(r.E_pad, 32));
    split_kernel<<<sg, 256, 0, s>>>(W_r, c.d, c.E, r.E_pad, W3, clear_status ? status : nullptr);
    cudaError_t err = cudaGetLastError();
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
    if (c.E <= 32)
        select_kernel<1><<<rows, 32 * kPartialTokens, 0, s>>>(p, plog, r.k_parts, r.E_pad);
    else if (c.E <= 64)
        select_kernel<2><<<rows, 32 * kPartialTokens, 0, s>>>(p, plog, r.k_parts, r.E_pad);
    else if (c.E <= 128)
        select_kernel<4><<<rows, 32 * kPartialTokens, 0, s>>>(p, plog, r.k_parts, r.E_pad);
    else
        select_kernel<8><<<rows, 32 * kPartialTokens, 0, s>>>(p, plog, r.k_parts, r.E_pad);
    return cudaGetLastError();
}

}  // namespace moe
