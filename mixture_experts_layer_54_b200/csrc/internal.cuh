// Library-private declarations shared by the CUDA translation units of
// libmoe_b200.so.  Nothing here is visible through the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kMaxE = 256;
constexpr int kMaxK = 8;
constexpr int kRouteTokens = 32;   // tokens per block of the tiled route kernel
constexpr int kPartialTokens = 32;  // tokens per row of the loss partials
constexpr int kCapTokens = 256;    // tokens per capacity block
constexpr int kLossUnits = 1024;   // most (row phase, column) units of the loss reduction

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline int dtype_bytes(int dtype) { return dtype == MOE_DTYPE_BF16 ? 2 : 4; }

// ---- programmatic dependent launch ----
// The forward's kernels are launched so that each may start while the
// previous kernel in the stream is finishing: its blocks become resident and
// run their set-up, then wait in pdl_wait() until the previous kernel has
// completed and its writes are visible.  pdl_trigger() lets the next kernel
// start launching; every kernel launched with launch_pdl calls pdl_wait()
// before it reads anything an earlier kernel wrote (both are no-ops for a
// kernel launched without the attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    return err != cudaSuccess ? err : cudaGetLastError();
}

// ---- launch-shape queries, answered once per device and kernel ----
int device_sms();
// Raises (never lowers) the kernel's dynamic shared-memory opt-in to bytes.
cudaError_t raise_smem_limit(const void *kernel, int bytes);
cudaError_t cached_blocks_per_sm(const void *kernel, int threads, int smem, int *out);
// Clusters of `cluster` blocks resident at once (the kernel's opt-in must
// already cover smem).
cudaError_t cached_active_clusters(const void *kernel, int threads, int smem, int cluster,
                                   int *out);

// Shape limits and codes; also the capacity factor rule.
moe_status validate(const moe_config &c);
int64_t capacity_of(const moe_config &c);          // valid config only
int64_t perm_rows(const moe_config &c);            // valid config only
int route_blocks(const moe_config &c);   // blocks of the tiled route kernel
int partial_rows(const moe_config &c);   // rows of the loss partials, ceil(T / 32)
int cap_blocks(const moe_config &c);

// Tensor-core router layout (bf16 layers).  Fused (E <= 16): one kernel, a
// cluster of k_parts blocks per 128-token tile.  Otherwise three launches:
// experts padded to E_pad in n_chunks chunks of n_chunk, K (k_blocks of 64)
// split in k_parts of kb_per_part, through scratch.
struct RoutePlan {
    bool tensor_cores, fused;
    int E_pad, n_chunk, n_chunks, k_blocks, k_parts, kb_per_part, cluster, blocks;
};
RoutePlan route_plan(const moe_config &c);
size_t route_scratch_bytes(const moe_config &c);

// Scratch carving of the stage workspace: the status word, then one region
// that the route, capacity and expert-FFN calls share (a call only uses it
// while it runs, and calls on one stream do not overlap).
struct StageScratch {
    int32_t *status;      // device status word (timeouts)
    void *route;          // tensor-core router (three launches): split weights, partial logits
    int32_t *hist;        // [cap_blocks][k][E]
    double *loss_ps;      // [kLossUnits] the whole forward's loss phase sums
    int32_t *count_base;  // [E] sharded capacity: earlier shards' assignments
    unsigned long long *keys;   // [T k] batch-prioritized capacity: per-expert lists
    void *H;              // [perm_rows][F] dtype
    void *H_sh;           // [S][T][Fs] dtype
};
size_t stage_scratch_bytes(const moe_config &c);
StageScratch carve_stage(const moe_config &c, void *ws);

// ---- launches (return the first CUDA error, cudaSuccess otherwise) ----
cudaError_t launch_route(const moe_config &c, const void *x, const float *W_r,
                         const float *logit_bias, const float *select_bias,
                         int32_t *topk, float *gates, float *partials,
                         float *logits_out, float *scores_out, cudaStream_t s);

cudaError_t launch_route_tc(const moe_config &c, const void *x, const float *W_r,
                            const float *logit_bias, const float *select_bias, int32_t *topk,
                            float *gates, float *partials, float *logits_out, float *scores_out,
                            void *scratch, int32_t *status, bool clear_status, cudaStream_t s);

cudaError_t launch_shard_base(const moe_config &c, const int32_t *shard_counts, int shard,
                              int32_t *count_base, cudaStream_t s);

// hist: scratch [cap_blocks][k][E] int32.  count_base (nullable, [E]):
// assignments to each expert in earlier shards of the same global batch
// (token order); C is then the global batch's capacity.  partials (nullable,
// the router's loss partials): the same two launches also write aux and
// zloss, with the phase sums in loss_ps (scratch of kLossUnits doubles).
cudaError_t launch_capacity(const moe_config &c, int64_t C, const int32_t *topk,
                            int32_t *counts, int32_t *pos, uint8_t *keep,
                            int32_t *kept, int32_t *offsets, uint8_t *dropped,
                            int32_t *n_dropped, int32_t *hist, cudaStream_t s,
                            const int32_t *count_base = nullptr,
                            const float *partials = nullptr, double *loss_ps = nullptr,
                            float *aux = nullptr, float *zloss = nullptr);

cudaError_t launch_capacity_scored(const moe_config &c, int64_t C, const int32_t *topk,
                                   const float *scores, int32_t *counts, int32_t *pos,
                                   uint8_t *keep, int32_t *kept, int32_t *offsets,
                                   uint8_t *dropped, int32_t *n_dropped, int32_t *hist,
                                   unsigned long long *keys, cudaStream_t s);

cudaError_t launch_seq_loss(const moe_config &c, int L, const int32_t *topk,
                            const float *partials, float *per_seq, float *loss, cudaStream_t s);

cudaError_t launch_bias_update(const moe_config &c, const int32_t *counts, float gamma,
                               float *bias, cudaStream_t s);

// src_slot[offsets[e] + pos[t, j]] = t k + j for every kept (t, j), -1 for
// every other row.
cudaError_t launch_dispatch_rows(const moe_config &c, const int32_t *topk, const int32_t *pos,
                                 const uint8_t *keep, const int32_t *offsets, int32_t *src_slot,
                                 cudaStream_t s);

// x_perm nullable (only the table), src_slot nullable (no table; padding rows
// are not written), zero_rows nullable: rows of tokens with every slot
// dropped are set to 0 there (the fused combine of a top-1 layer).
cudaError_t launch_dispatch(const moe_config &c, const void *x, const int32_t *topk,
                            const int32_t *pos, const uint8_t *keep,
                            const int32_t *offsets, void *x_perm, cudaStream_t s,
                            int32_t *src_slot = nullptr, void *zero_rows = nullptr);

// y[t] = sum over kept slots j of Y_slot[t k + j] (+ Y_sh[t]) (+ residual[t]),
// fp32 in slot order.
cudaError_t launch_combine_slots(const moe_config &c, const void *Y_slot, const void *Y_sh,
                                 const uint8_t *keep, const void *residual, void *y,
                                 cudaStream_t s);

cudaError_t launch_combine(const moe_config &c, const void *Y_perm, const void *Y_sh,
                           const float *gates, const int32_t *topk, const int32_t *pos,
                           const uint8_t *keep, const int32_t *offsets,
                           const void *residual, void *y, cudaStream_t s);

cudaError_t launch_losses(const moe_config &c, const int32_t *counts,
                          const float *partials, float *aux, float *zloss,
                          cudaStream_t s);

// one bounded wait on a barrier nobody arrives on (diagnostic)
cudaError_t launch_wait_probe(int32_t *status, unsigned long long timeout_ns, cudaStream_t s);

// fp32 expert FFNs on the CUDA cores (x_perm, src_slot, kept, gates and
// slot_out as for launch_ffn_tcgen05)
cudaError_t launch_ffn_simt(const moe_config &c, const void *x_perm, const int32_t *offsets,
                            const int32_t *src_slot, const void *W1, const void *W3, const void *W2,
                            const void *x, const void *Ws1, const void *Ws3,
                            const void *Ws2, void *Y_perm, void *Y_sh, void *H,
                            void *H_sh, cudaStream_t s, const int32_t *kept = nullptr,
                            const float *gates = nullptr, void *slot_out = nullptr);

// bf16 expert FFNs on the tensor cores (tcgen05 + TMEM + TMA).  x_perm NULL:
// GEMM1 gathers its routed rows from x through src_slot (row r holds
// assignment src_slot[r], token src_slot[r] / k).  slot_out non-NULL: GEMM2
// writes gates[a] * FFN(row) to row a = src_slot[r] of slot_out [T k, d] for
// every kept row (r - offsets[e] < kept[e]) instead of Y_perm.
cudaError_t launch_ffn_tcgen05(const moe_config &c, const void *x_perm,
                               const int32_t *offsets, const int32_t *src_slot,
                               const void *W1, const void *W3,
                               const void *W2, const void *x, const void *Ws1,
                               const void *Ws3, const void *Ws2, void *Y_perm,
                               void *Y_sh, void *H, void *H_sh, int32_t *status,
                               bool clear_status, cudaStream_t s,
                               const int32_t *kept = nullptr, const float *gates = nullptr,
                               void *slot_out = nullptr);

}  // namespace moe
