// Capacity stage: each assignment's queue position in its expert, the keep
// mask, per-expert counts and the padded segment offsets of the permuted
// buffers.
//
// Page "Lab 18 - Mixture of experts", section 3 (C = ceil(cf T k / E); the
// assignment beyond C is dropped; GShard rank-major priority); "Lab 01",
// where to start step 4 (first come first served in token order).
//
// The sequential definition is a walk over the T*k assignments in priority
// order with one counter per expert.  It is computed here in three launches:
//   count  - each block of 256 tokens histograms its assignments per (rank j,
//            expert e) in shared memory (integer atomics, order-free);
//   scan   - one block turns the histograms into, for every block, the number
//            of assignments to each expert that come before the block in
//            priority order, plus counts, kept, offsets and the drop total;
//   place  - each block walks its own assignments in priority order, 256 at a
//            time, ranking equal experts inside a warp with __match_any_sync
//            and across warps through a per-warp count table.
// Integers only, so the result is bit-exact with the sequential walk.
#include "internal.cuh"

namespace moe {
namespace {

constexpr int CT = kCapTokens;   // tokens per block (also the thread count)

__global__ void __launch_bounds__(CT) cap_count_kernel(const int32_t *topk, int T, int k, int E,
                                                       int32_t *hist)
{
    extern __shared__ int32_t h[];   // [k][E]
    for (int i = threadIdx.x; i < k * E; i += CT)
        h[i] = 0;
    __syncthreads();
    const int t = blockIdx.x * CT + threadIdx.x;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            int e = topk[(int64_t)t * k + j];
            if (e >= 0 && e < E)
                atomicAdd(&h[j * E + e], 1);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < k * E; i += CT)
        hist[(int64_t)blockIdx.x * k * E + i] = h[i];
}

__global__ void __launch_bounds__(1024)
cap_scan_kernel(const int32_t *__restrict__ hist, int nblk, int k, int E, int priority,
                long long C, int32_t *__restrict__ base, int32_t *__restrict__ counts,
                int32_t *__restrict__ kept, int32_t *__restrict__ offsets,
                int32_t *__restrict__ n_dropped)
{
    __shared__ int32_t total[kMaxK * kMaxE];   // per (j, e), all blocks
    __shared__ int32_t cnt[kMaxE];
    const int cols = k * E;
    // exclusive scan over blocks of each (j, e) column
    for (int col = threadIdx.x; col < cols; col += blockDim.x) {
        int run = 0;
#pragma unroll 8
        for (int b = 0; b < nblk; ++b) {
            int v = hist[(int64_t)b * cols + col];
            base[(int64_t)b * cols + col] = run;
            run += v;
        }
        total[col] = run;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int s = 0;
        for (int j = 0; j < k; ++j)
            s += total[j * E + e];
        cnt[e] = s;
        counts[e] = s;
        kept[e] = (long long)s < C ? s : (int32_t)C;
    }
    __syncthreads();
    if (priority == MOE_PRIORITY_TOKEN) {
        // assignments to e in earlier blocks, any rank: stored in the j = 0 slot
        for (int i = threadIdx.x; i < nblk * E; i += blockDim.x) {
            int b = i / E, e = i % E;
            int s = 0;
            for (int j = 0; j < k; ++j)
                s += base[(int64_t)b * cols + j * E + e];
            base[(int64_t)b * cols + e] = s;
        }
    } else {
        // rank-major: every rank j' < j of all tokens comes first
        for (int i = threadIdx.x; i < nblk * cols; i += blockDim.x) {
            int col = i % cols;
            int j = col / E, e = col % E;
            int s = 0;
            for (int jj = 0; jj < j; ++jj)
                s += total[jj * E + e];
            base[i] += s;
        }
    }
    if (threadIdx.x == 0) {
        int off = 0;
        long long drop = 0;
        for (int e = 0; e < E; ++e) {
            offsets[e] = off;
            int kv = (long long)cnt[e] < C ? cnt[e] : (int)C;
            drop += cnt[e] - kv;
            off += (kv + MOE_ROW_ALIGN - 1) / MOE_ROW_ALIGN * MOE_ROW_ALIGN;
        }
        offsets[E] = off;
        *n_dropped = (int32_t)drop;
    }
}

__global__ void __launch_bounds__(CT)
cap_place_kernel(const int32_t *topk, int T, int k, int E, int priority, long long C,
                 const int32_t *base, int32_t *pos, uint8_t *keep, uint8_t *dropped)
{
    __shared__ int32_t run[kMaxE];
    __shared__ int32_t wcnt[CT / 32][kMaxE];
    __shared__ uint8_t keep_s[CT * kMaxK];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * CT;
    const int ntok = min(CT, T - t0);
    const int cols = k * E;
    const int32_t *bb = base + (int64_t)blockIdx.x * cols;
    for (int i = tid; i < (CT / 32) * kMaxE; i += CT)
        (&wcnt[0][0])[i] = 0;
    const unsigned lt_mask = (1u << lane) - 1u;

    // one pass = a sequence of `len` assignments, element n -> (t_local, j)
    const int passes = priority == MOE_PRIORITY_TOKEN ? 1 : k;
    for (int p = 0; p < passes; ++p) {
        for (int e = tid; e < E; e += CT)
            run[e] = 0;
        __syncthreads();
        const int len = priority == MOE_PRIORITY_TOKEN ? ntok * k : ntok;
        for (int c0 = 0; c0 < len; c0 += CT) {
            const int n = c0 + tid;
            const bool valid = n < len;
            int tl = 0, j = 0, e = E;   // E = sentinel for idle lanes
            if (valid) {
                if (priority == MOE_PRIORITY_TOKEN) {
                    tl = n / k;
                    j = n % k;
                } else {
                    tl = n;
                    j = p;
                }
                e = topk[(int64_t)(t0 + tl) * k + j];
                if (e < 0 || e >= E)
                    e = E;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int inwarp = __popc(peers & lt_mask);
            const bool leader = (peers & lt_mask) == 0;
            if (leader && e < E)
                wcnt[warp][e] = __popc(peers);
            __syncthreads();
            if (valid) {
                if (e < E) {
                    int prior = 0;
                    for (int w = 0; w < warp; ++w)
                        prior += wcnt[w][e];
                    const int boff = priority == MOE_PRIORITY_TOKEN ? e : j * E + e;
                    const long long position = (long long)bb[boff] + run[e] + prior + inwarp;
                    pos[(int64_t)(t0 + tl) * k + j] = (int32_t)position;
                    keep_s[tl * k + j] = position < C ? 1 : 0;
                } else {
                    pos[(int64_t)(t0 + tl) * k + j] = -1;
                    keep_s[tl * k + j] = 0;
                }
            }
            __syncthreads();
            for (int ee = tid; ee < E; ee += CT) {
                int s = 0;
                for (int w = 0; w < CT / 32; ++w) {
                    s += wcnt[w][ee];
                    wcnt[w][ee] = 0;
                }
                run[ee] += s;
            }
            __syncthreads();
        }
    }
    if (tid < ntok) {
        int any = 0;
        for (int j = 0; j < k; ++j) {
            any |= keep_s[tid * k + j];
            keep[(int64_t)(t0 + tid) * k + j] = keep_s[tid * k + j];
        }
        dropped[t0 + tid] = any ? 0 : 1;
    }
}

}  // namespace

cudaError_t launch_capacity(const moe_config &c, int64_t C, const int32_t *topk,
                            int32_t *counts, int32_t *pos, uint8_t *keep, int32_t *kept,
                            int32_t *offsets, uint8_t *dropped, int32_t *n_dropped,
                            int32_t *hist, int32_t *base, cudaStream_t s)
{
    const int nblk = cap_blocks(c);
    if (nblk > 0) {
        cap_count_kernel<<<nblk, CT, sizeof(int32_t) * c.k * c.E, s>>>(topk, c.T, c.k, c.E, hist);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess)
            return err;
    }
    cap_scan_kernel<<<1, 1024, 0, s>>>(hist, nblk, c.k, c.E, c.priority, (long long)C, base,
                                       counts, kept, offsets, n_dropped);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || nblk == 0)
        return err;
    cap_place_kernel<<<nblk, CT, 0, s>>>(topk, c.T, c.k, c.E, c.priority, (long long)C, base, pos,
                                         keep, dropped);
    return cudaGetLastError();
}

}  // namespace moe
