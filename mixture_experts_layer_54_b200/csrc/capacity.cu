// Capacity stage: each assignment's queue position in its expert, the keep
// mask, per-expert counts and the padded segment offsets of the permuted
// buffers.
//
// Page "Lab 18 - Mixture of experts", section 3 (C = ceil(cf T k / E); the
// assignment beyond C is dropped; GShard rank-major priority); "Lab 01",
// where to start step 4 (first come first served in token order).
//
// The sequential definition is a walk over the T*k assignments in priority
// order with one counter per expert.  It is computed here in two launches:
//   count  - each block of 256 tokens histograms its assignments per (rank j,
//            expert e) in shared memory (integer atomics, order-free) and
//            writes it per (j, e), or in token order per expert (the k ranks
//            summed: a later block's base needs no more);
//   place  - each block sums the histograms of the blocks before it (and,
//            rank-major, all blocks' lower ranks): the number of assignments
//            to each expert that come before the block in priority order;
//            then each warp walks its 32 tokens' assignments in priority
//            order, 32 at a time, ranking equal experts with __match_any_sync,
//            after one scan over the block's warps has given each warp its
//            start per expert.  One more block computes counts, kept, offsets
//            and the drop total (and, for the whole forward, the losses).
// Integers only, so the result is bit-exact with the sequential walk.
//
// Batch-prioritized order ("Lab 18" section 3, V-MoE: assignments ranked by
// router score) adds three launches after the token-order ones, which give
// the counts, kept, offsets and drop total (the same for every order) and each
// assignment's token-order place in its expert's list:
//   list   - every assignment writes a 64-bit key into its expert's list at
//            that place: high word the score's bits mapped to an unsigned
//            order, low word ~a, so a larger key means a higher score, or an
//            equal score and an earlier assignment;
//   rank   - a block per 256 entries of one expert's list; each entry's queue
//            position is the number of larger keys in the list (keys are
//            distinct, so positions are a permutation), read from shared
//            memory in tiles;
//   drop   - a token is dropped when none of its k slots was kept.
#include "internal.cuh"
#include "losses_common.cuh"

namespace moe {
namespace {

constexpr int CT = kCapTokens;   // tokens per block (also the thread count)

__global__ void __launch_bounds__(CT) cap_count_kernel(const int32_t *topk, int T, int k, int E,
                                                       int hcols, int32_t *hist, int nblk,
                                                       const float *partials, int prows,
                                                       double *loss_ps)
{
    if ((int)blockIdx.x >= nblk) {
        // the whole forward's extra blocks: phase sums of the loss partials,
        // thread u of these blocks taking work unit u (losses_common.cuh)
        pdl_wait();   // the partials come from the router
        pdl_trigger();
        const int C = E + 1, u = ((int)blockIdx.x - nblk) * CT + (int)threadIdx.x;
        if (u < loss_phases(C) * C)
            loss_ps[u] = loss_phase_sum(partials, prows, C, u);
        return;
    }
    extern __shared__ int32_t h[];   // [k][E]
    for (int i = threadIdx.x; i < k * E; i += CT)
        h[i] = 0;
    pdl_wait();   // topk comes from the router
    pdl_trigger();
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
    if (hcols == E) {
        // token order: one column per expert, the k slots summed
        for (int e = threadIdx.x; e < E; e += CT) {
            int v = 0;
            for (int j = 0; j < k; ++j)
                v += h[j * E + e];
            hist[(int64_t)blockIdx.x * E + e] = v;
        }
    } else {
        for (int i = threadIdx.x; i < k * E; i += CT)
            hist[(int64_t)blockIdx.x * k * E + i] = h[i];
    }
}

// Column sums of the per-block histograms [nblk][cols]: before[col] = blocks
// [0, upto), and (total != nullptr) total[col] = all blocks; BATCH loads of a
// column in flight per thread.  With fewer columns than threads the blocks
// are split into P parts (thread t: column t mod cols, blocks t / cols,
// + P, ...) whose sums meet in shared memory (integers: exact in any order).
// Every thread of the block calls it; it ends with the block synchronised.
__device__ __forceinline__ void hist_sums(const int32_t *__restrict__ hist, int nblk, int cols,
                                          int upto, int32_t *before, int32_t *total)
{
    constexpr int BATCH = 16;
    __shared__ int32_t pb[kCapTokens], pt[kCapTokens];
    const int end = total ? nblk : upto;
    const int P = cols >= (int)blockDim.x ? 1 : (int)blockDim.x / cols;
    if (P == 1) {
        for (int col = threadIdx.x; col < cols; col += blockDim.x) {
            int bsum = 0, tsum = 0;
            for (int b0 = 0; b0 < end; b0 += BATCH) {
                int v[BATCH];
#pragma unroll
                for (int i = 0; i < BATCH; ++i)
                    v[i] = b0 + i < end ? hist[(int64_t)(b0 + i) * cols + col] : 0;
#pragma unroll
                for (int i = 0; i < BATCH; ++i) {
                    bsum += b0 + i < upto ? v[i] : 0;
                    tsum += v[i];
                }
            }
            before[col] = bsum;
            if (total)
                total[col] = tsum;
        }
        __syncthreads();
        return;
    }
    const int t = threadIdx.x, col = t % cols, part = t / cols;
    if (part < P) {
        int bsum = 0, tsum = 0;
        for (int b0 = part; b0 < end; b0 += BATCH * P) {
            int v[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const int b = b0 + i * P;
                v[i] = b < end ? hist[(int64_t)b * cols + col] : 0;
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                bsum += b0 + i * P < upto ? v[i] : 0;
                tsum += v[i];
            }
        }
        pb[t] = bsum;
        pt[t] = tsum;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < cols; c += blockDim.x) {
        int sb = 0, st = 0;
        for (int q = 0; q < P; ++q) {
            sb += pb[q * cols + c];
            st += pt[q * cols + c];
        }
        before[c] = sb;
        if (total)
            total[c] = st;
    }
    __syncthreads();
}

// The block after the placement blocks: counts, kept, the padded segment
// offsets and the drop total from the histograms of all blocks; with
// partials, also the two balancing losses (the forward's losses stage, in the
// same fixed order as moe_losses).
__device__ void capacity_totals(const int32_t *__restrict__ hist, int nblk, int k, int E,
                                int hcols, long long C, const int32_t *__restrict__ count_base,
                                int T,
                                int32_t *__restrict__ counts, int32_t *__restrict__ kept,
                                int32_t *__restrict__ offsets, int32_t *__restrict__ n_dropped,
                                const double *loss_ps, float *aux, float *zloss,
                                int32_t *colsum)
{
    __shared__ int32_t cnt[kMaxE];
    __shared__ int32_t kept_s[kMaxE];
    __shared__ double term[kMaxE + 1];
    __shared__ double ps[kLossUnits];
    hist_sums(hist, nblk, hcols, nblk, colsum, nullptr);
    const int ranks = hcols == E ? 1 : k;   // histogram rows per expert column
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int s = 0;
        for (int j = 0; j < ranks; ++j)
            s += colsum[j * E + e];
        // slots left for this batch: C, less what earlier shards of the same
        // global batch already took (count_base, sharded capacity only)
        long long room = C - (count_base ? (long long)count_base[e] : 0LL);
        room = room < 0 ? 0 : room;
        const int32_t kv = (long long)s < room ? s : (int32_t)room;
        cnt[e] = s;
        counts[e] = s;
        kept_s[e] = kv;
        kept[e] = kv;
    }
    __syncthreads();
    // segment offsets: kept counts rounded up to MOE_ROW_ALIGN, exclusive scan
    // by one warp; the drop total summed in a fixed order
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int carry = 0;
        long long drop = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            int padded = 0;
            if (e < E) {
                const int kv = kept_s[e];
                drop += cnt[e] - kv;
                padded = (kv + MOE_ROW_ALIGN - 1) / MOE_ROW_ALIGN * MOE_ROW_ALIGN;
            }
            int incl = padded;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += n;
            }
            if (e < E)
                offsets[e] = carry + incl - padded;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            drop += __shfl_xor_sync(0xffffffffu, drop, o);
        if (lane == 0) {
            offsets[E] = carry;
            *n_dropped = (int32_t)drop;
        }
    }
    if (loss_ps) {
        // the phase sums from the count launch's extra blocks, then the terms
        const int units = loss_phases(E + 1) * (E + 1);
        for (int u = threadIdx.x; u < units; u += blockDim.x)
            ps[u] = loss_ps[u];
        __syncthreads();
        losses_from_phase_sums(cnt, ps, T > 0 ? T : 1, k, E, aux, zloss, term);
    }
}

// Each warp owns 32 consecutive tokens of the block.  Per pass (token order:
// one pass over all slots; rank-major: one pass per slot j): (A) the warp
// counts its assignments per expert; (B) one exclusive scan over the warps
// turns the counts into each warp's start inside the block; (C) the warp walks
// its assignments in priority order, 32 at a time, ranking equal experts with
// __match_any_sync and keeping its own running count per expert.
//
// Each block first takes its bases from the histograms: token order, the
// assignments to e of earlier blocks (any rank); rank-major, those of rank j
// in earlier blocks plus every assignment of a lower rank.  Block nblk
// computes the totals instead (capacity_totals).
__global__ void __launch_bounds__(CT)
cap_place_kernel(const int32_t *__restrict__ topk, int T, int k, int E, int priority, long long C,
                 const int32_t *__restrict__ count_base, const int32_t *__restrict__ hist,
                 int nblk, int32_t *__restrict__ pos, uint8_t *__restrict__ keep,
                 uint8_t *__restrict__ dropped, int32_t *__restrict__ counts,
                 int32_t *__restrict__ kept, int32_t *__restrict__ offsets,
                 int32_t *__restrict__ n_dropped, const double *loss_ps, float *aux, float *zloss)
{
    __shared__ int32_t wrun[CT / 32][kMaxE];
    __shared__ uint8_t keep_s[CT * kMaxK];
    __shared__ int32_t before[kMaxK * kMaxE], total[kMaxK * kMaxE];
    pdl_wait();   // topk from the router, the histograms from cap_count
    pdl_trigger();
    const int cols = k * E;
    const bool token_order = priority == MOE_PRIORITY_TOKEN;
    const int hcols = token_order ? E : cols;   // cap_count's histogram columns
    if (blockIdx.x == nblk) {
        capacity_totals(hist, nblk, k, E, hcols, C, count_base, T, counts, kept, offsets,
                        n_dropped, loss_ps, aux, zloss, before);
        return;
    }
    // token order: before[e] = the base of expert e (any rank)
    hist_sums(hist, nblk, hcols, blockIdx.x, before, token_order ? nullptr : total);
    if (!token_order) {
        for (int col = threadIdx.x; col < cols; col += CT) {
            const int j = col / E, e = col % E;
            int s = 0;
            for (int jj = 0; jj < j; ++jj)
                s += total[jj * E + e];
            before[col] += s;
        }
    }
    __syncthreads();
    const int32_t *bb = before;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int tw = blockIdx.x * CT + warp * 32;   // this warp's first token
    const int nw = max(0, min(32, T - tw));       // its tokens
    const int passes = token_order ? 1 : k;
    for (int p = 0; p < passes; ++p) {
        const int len = token_order ? nw * k : nw;   // <= 32 kMaxK
        // this pass's experts, entry i * 32 + lane in ev[i], all loads in flight
        int ev[kMaxK];
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
            const int n = i * 32 + lane;
            int e = E;   // sentinel for idle lanes and invalid experts
            if (n < len) {
                const int tl = token_order ? n / k : n, j = token_order ? n % k : p;
                e = topk[(int64_t)(tw + tl) * k + j];
                if (e < 0 || e >= E)
                    e = E;
            }
            ev[i] = e;
        }
        // (A) this warp's assignments per expert
        for (int i = lane; i < E; i += 32)
            wrun[warp][i] = 0;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
            if (i * 32 >= len)
                break;
            const int e = ev[i];
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            if ((peers & lt_mask) == 0 && e < E)
                wrun[warp][e] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        // (B) earlier warps' assignments to each expert
        for (int e = tid; e < E; e += CT) {
            int run = 0;
#pragma unroll
            for (int w = 0; w < CT / 32; ++w) {
                const int v = wrun[w][e];
                wrun[w][e] = run;
                run += v;
            }
        }
        __syncthreads();
        // (C) positions, in priority order
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
            if (i * 32 >= len)
                break;
            const int n = i * 32 + lane;
            const int e = ev[i];
            const int tl = token_order ? n / k : n, j = token_order ? n % k : p;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            if (n < len) {
                const int64_t a = (int64_t)(tw + tl) * k + j;
                uint8_t kv = 0;
                if (e < E) {
                    const int boff = token_order ? e : j * E + e;
                    const long long position =
                        (long long)bb[boff] + wrun[warp][e] + __popc(peers & lt_mask);
                    pos[a] = (int32_t)position;
                    // kept while the slot's place in the whole (global) batch is below C
                    kv = position + (count_base ? count_base[e] : 0) < C ? 1 : 0;
                } else {
                    pos[a] = -1;
                }
                keep_s[(warp * 32 + tl) * k + j] = kv;
            }
            __syncwarp();
            if ((peers & lt_mask) == 0 && e < E)
                wrun[warp][e] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();   // every warp done with the tables before the next pass
    }
    if (lane < nw) {
        int any = 0;
        for (int j = 0; j < k; ++j) {
            const uint8_t kv = keep_s[(warp * 32 + lane) * k + j];
            any |= kv;
            keep[(int64_t)(tw + lane) * k + j] = kv;
        }
        dropped[tw + lane] = any ? 0 : 1;
    }
}

// fp32 bits to an unsigned key with the same order (-0 and +0 equal)
__device__ __forceinline__ uint32_t score_order(float v)
{
    uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive scan of the counts into shared memory (E <= 256, one warp)
__device__ __forceinline__ void list_offsets(const int32_t *counts, int E, int32_t *lofs)
{
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int carry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < E ? counts[e] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += n;
            }
            if (e < E)
                lofs[e] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(256)
cap_list_kernel(const int32_t *__restrict__ topk, const float *__restrict__ scores, int T, int k,
                int E, const int32_t *__restrict__ counts, const int32_t *__restrict__ pos_tok,
                unsigned long long *__restrict__ keys)
{
    __shared__ int32_t lofs[kMaxE];
    list_offsets(counts, E, lofs);
    const int64_t A = (int64_t)T * k;
    for (int64_t a = (int64_t)blockIdx.x * 256 + threadIdx.x; a < A; a += (int64_t)gridDim.x * 256) {
        const int e = topk[a];
        if (e < 0 || e >= E)
            continue;
        const float v = scores[(a / k) * E + e];
        keys[lofs[e] + pos_tok[a]] =
            ((unsigned long long)score_order(v) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)a);
    }
}

__global__ void __launch_bounds__(256)
cap_rank_kernel(const unsigned long long *__restrict__ keys, const int32_t *__restrict__ counts,
                int E, int k, long long C, int32_t *__restrict__ pos, uint8_t *__restrict__ keep)
{
    __shared__ int32_t lofs[kMaxE];
    __shared__ unsigned long long tile[256];
    const int e = blockIdx.y;
    const int n = counts[e];
    const int m = blockIdx.x * 256 + threadIdx.x;
    if (blockIdx.x * 256 >= n)
        return;   // whole block: no entries of this expert here
    list_offsets(counts, E, lofs);
    const unsigned long long *list = keys + lofs[e];
    const unsigned long long mine = m < n ? list[m] : 0ull;
    int ahead = 0;
    for (int t0 = 0; t0 < n; t0 += 256) {
        __syncthreads();
        if (t0 + threadIdx.x < n)
            tile[threadIdx.x] = list[t0 + threadIdx.x];
        __syncthreads();
        const int len = min(256, n - t0);
        for (int j = 0; j < len; ++j)
            ahead += tile[j] > mine ? 1 : 0;
    }
    if (m < n) {
        const int64_t a = (int64_t)(0xFFFFFFFFu - (uint32_t)(mine & 0xFFFFFFFFull));
        pos[a] = ahead;
        keep[a] = (long long)ahead < C ? 1 : 0;
    }
}

__global__ void cap_drop_kernel(const uint8_t *__restrict__ keep, int T, int k,
                                uint8_t *__restrict__ dropped)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T)
        return;
    int any = 0;
    for (int j = 0; j < k; ++j)
        any |= keep[(int64_t)t * k + j];
    dropped[t] = any ? 0 : 1;
}

}  // namespace

cudaError_t launch_capacity_scored(const moe_config &c, int64_t C, const int32_t *topk,
                                   const float *scores, int32_t *counts, int32_t *pos,
                                   uint8_t *keep, int32_t *kept, int32_t *offsets,
                                   uint8_t *dropped, int32_t *n_dropped, int32_t *hist,
                                   unsigned long long *keys, cudaStream_t s)
{
    // token order first: counts, kept, offsets, drop total, and each
    // assignment's place in its expert's list (written to pos, then replaced)
    moe_config tok = c;
    tok.priority = MOE_PRIORITY_TOKEN;
    cudaError_t err = launch_capacity(tok, C, topk, counts, pos, keep, kept, offsets, dropped,
                                      n_dropped, hist, s);
    if (err != cudaSuccess || c.T == 0)
        return err;
    const int64_t A = (int64_t)c.T * c.k;
    const int list_blocks = (int)(ceil_div(A, 256) < 1184 ? ceil_div(A, 256) : 1184);
    cap_list_kernel<<<list_blocks, 256, 0, s>>>(topk, scores, c.T, c.k, c.E, counts, pos, keys);
    if ((err = cudaGetLastError()) != cudaSuccess)
        return err;
    // an expert holds at most T assignments (a token's k experts are distinct)
    dim3 grid((unsigned)ceil_div(c.T, 256), (unsigned)c.E);
    cap_rank_kernel<<<grid, 256, 0, s>>>(keys, counts, c.E, c.k, (long long)C, pos, keep);
    if ((err = cudaGetLastError()) != cudaSuccess)
        return err;
    cap_drop_kernel<<<(unsigned)ceil_div(c.T, 256), 256, 0, s>>>(keep, c.T, c.k, dropped);
    return cudaGetLastError();
}

// count_base[e] = sum over the shards before `shard` of their counts
// (shard_counts [n_shards][E]), in shard order.
__global__ void shard_base_kernel(const int32_t *__restrict__ shard_counts, int shard, int E,
                                  int32_t *__restrict__ count_base)
{
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int s = 0;
        for (int r = 0; r < shard; ++r)
            s += shard_counts[(int64_t)r * E + e];
        count_base[e] = s;
    }
}

cudaError_t launch_shard_base(const moe_config &c, const int32_t *shard_counts, int shard,
                              int32_t *count_base, cudaStream_t s)
{
    shard_base_kernel<<<1, 256, 0, s>>>(shard_counts, shard, c.E, count_base);
    return cudaGetLastError();
}

cudaError_t launch_capacity(const moe_config &c, int64_t C, const int32_t *topk,
                            int32_t *counts, int32_t *pos, uint8_t *keep, int32_t *kept,
                            int32_t *offsets, uint8_t *dropped, int32_t *n_dropped,
                            int32_t *hist, cudaStream_t s, const int32_t *count_base,
                            const float *partials, double *loss_ps, float *aux, float *zloss)
{
    const int nblk = cap_blocks(c);
    // with the losses: extra count blocks for the phase sums of the partials
    const int lblk = partials ? (loss_phases(c.E + 1) * (c.E + 1) + CT - 1) / CT : 0;
    if (nblk + lblk > 0) {
        // token order: histogram rows of one column per expert
        const int hcols = c.priority == MOE_PRIORITY_TOKEN ? c.E : c.k * c.E;
        cudaError_t err = launch_pdl(cap_count_kernel, dim3(nblk + lblk), dim3(CT),
                                     sizeof(int32_t) * c.k * c.E, s, topk, c.T, c.k, c.E, hcols,
                                     hist, nblk, partials, partial_rows(c), loss_ps);
        if (err != cudaSuccess)
            return err;
    }
    // placement blocks, then the totals block (and the losses when asked)
    return launch_pdl(cap_place_kernel, dim3(nblk + 1), dim3(CT), 0, s, topk, c.T, c.k, c.E,
                      c.priority, (long long)C, count_base, (const int32_t *)hist, nblk, pos,
                      keep, dropped, counts, kept, offsets, n_dropped,
                      partials ? (const double *)loss_ps : nullptr, aux, zloss);
}

}  // namespace moe
