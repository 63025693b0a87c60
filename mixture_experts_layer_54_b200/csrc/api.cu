// Host side of the C ABI declared in include/moe_b200.h: argument checks,
// workspace carving and the stage launches.  Nothing here allocates device
// memory or synchronises, except moe_device_status which reads the status
// word back.
#include "internal.cuh"

#include <math.h>
#include <string.h>

namespace moe {

moe_status validate(const moe_config &c)
{
    if (c.T < 0 || c.d < 1 || c.E < 1 || c.E > kMaxE || c.k < 1 || c.k > c.E || c.k > kMaxK ||
        c.d_ff < 1 || c.n_shared < 0 || (c.n_shared > 0 && c.d_ff_shared < 1))
        return MOE_ERR_SHAPE;
    if ((c.act != MOE_ACT_GELU && c.act != MOE_ACT_SWIGLU) ||
        (c.score != MOE_SCORE_SOFTMAX && c.score != MOE_SCORE_SIGMOID) ||
        (c.dtype != MOE_DTYPE_F32 && c.dtype != MOE_DTYPE_BF16) ||
        (c.priority != MOE_PRIORITY_TOKEN && c.priority != MOE_PRIORITY_RANK &&
         c.priority != MOE_PRIORITY_SCORE) || c.renorm < -1 ||
        c.renorm > 1)
        return MOE_ERR_DTYPE;
    if (!(c.capacity_factor >= 1.0))   // also rejects NaN
        return MOE_ERR_CAPACITY_FACTOR;
    if ((int64_t)c.T * c.k > INT32_MAX / 2)
        return MOE_ERR_SHAPE;
    if (c.dtype == MOE_DTYPE_BF16) {
        // 128-byte K steps and 16-byte rows for TMA
        if (c.d % 64 || c.d_ff % 64 || (c.n_shared > 0 && c.d_ff_shared % 64))
            return MOE_ERR_SHAPE;
    } else if (c.d % 4) {
        return MOE_ERR_SHAPE;   // 16-byte rows for the row copies
    }
    return MOE_OK;
}

int64_t capacity_of(const moe_config &c)
{
    if (isinf(c.capacity_factor))
        return c.T;
    // A token's k experts are distinct, so an expert receives at most T
    // assignments: any C >= T keeps them all.  Holding C at T changes no
    // decision and keeps the conversion defined for huge finite factors.
    const double C = ceil(c.capacity_factor * (double)((int64_t)c.T * c.k) / (double)c.E);
    return C >= (double)c.T ? (int64_t)c.T : (int64_t)C;
}

int64_t perm_rows(const moe_config &c)
{
    int64_t kept = (int64_t)c.T * c.k;
    const int64_t cap_total = capacity_of(c) * c.E;
    if (cap_total < kept)
        kept = cap_total;
    const int64_t rows = kept + (int64_t)c.E * (MOE_ROW_ALIGN - 1);
    return (int64_t)align_up((size_t)rows, MOE_ROW_ALIGN);
}

int route_blocks(const moe_config &c) { return (int)ceil_div(c.T, kRouteTokens); }
int partial_rows(const moe_config &c) { return (int)ceil_div(c.T, kPartialTokens); }
int cap_blocks(const moe_config &c) { return (int)ceil_div(c.T, kCapTokens); }

namespace {

constexpr size_t kAlign = 256;

struct Carver {
    char *base;
    size_t off = 0;
    void *take(size_t bytes)
    {
        void *p = base ? base + off : nullptr;
        off = align_up(off + bytes, kAlign);
        return p;
    }
};

void carve_stage_into(const moe_config &c, Carver &cv, StageScratch &s)
{
    const int64_t R = perm_rows(c);
    const size_t esz = dtype_bytes(c.dtype);
    const size_t hk = (size_t)cap_blocks(c) * c.k * c.E * sizeof(int32_t);
    s.status = static_cast<int32_t *>(cv.take(kAlign));
    // one shared region: the largest of the three stages' scratch
    const size_t off = cv.off;
    Carver route_cv{cv.base, off}, cap_cv{cv.base, off}, ffn_cv{cv.base, off};
    s.route = route_cv.take(route_scratch_bytes(c));
    s.hist = static_cast<int32_t *>(cap_cv.take(hk));
    s.loss_ps = static_cast<double *>(cap_cv.take(kLossUnits * sizeof(double)));
    s.count_base = static_cast<int32_t *>(cap_cv.take((size_t)c.E * 4));
    s.keys = static_cast<unsigned long long *>(
        cap_cv.take(c.priority == MOE_PRIORITY_SCORE ? (size_t)c.T * c.k * 8 : 0));
    s.H = ffn_cv.take((size_t)R * c.d_ff * esz);
    s.H_sh = ffn_cv.take((size_t)c.n_shared * c.T * (c.n_shared ? c.d_ff_shared : 0) * esz);
    cv.off = route_cv.off > cap_cv.off ? route_cv.off : cap_cv.off;
    if (ffn_cv.off > cv.off)
        cv.off = ffn_cv.off;
}

struct ForwardBufs {
    int32_t *topk, *counts, *kept, *offsets, *n_dropped, *pos, *slot;
    float *gates, *partials, *scores;
    uint8_t *keep, *dropped;
    void *x_perm, *Y_perm, *Y_sh;
};

void carve_forward_into(const moe_config &c, Carver &cv, ForwardBufs &f)
{
    const int64_t R = perm_rows(c);
    const size_t esz = dtype_bytes(c.dtype);
    const size_t A = (size_t)c.T * c.k;
    f.topk = static_cast<int32_t *>(cv.take(A * 4));
    f.gates = static_cast<float *>(cv.take(A * 4));
    f.partials = static_cast<float *>(cv.take((size_t)partial_rows(c) * (c.E + 1) * 4));
    // router scores [T, E], kept only for the batch-prioritized capacity order
    f.scores = static_cast<float *>(
        cv.take(c.priority == MOE_PRIORITY_SCORE ? (size_t)c.T * c.E * 4 : 0));
    f.counts = static_cast<int32_t *>(cv.take((size_t)c.E * 4));
    f.kept = static_cast<int32_t *>(cv.take((size_t)c.E * 4));
    f.offsets = static_cast<int32_t *>(cv.take((size_t)(c.E + 1) * 4));
    f.n_dropped = static_cast<int32_t *>(cv.take(4));
    f.pos = static_cast<int32_t *>(cv.take(A * 4));
    f.keep = static_cast<uint8_t *>(cv.take(A));
    f.dropped = static_cast<uint8_t *>(cv.take((size_t)c.T));
    f.x_perm = cv.take((size_t)R * c.d * esz);
    f.Y_perm = cv.take((size_t)R * c.d * esz);
    f.Y_sh = c.n_shared > 0 ? cv.take((size_t)c.T * c.d * esz) : nullptr;
    f.slot = static_cast<int32_t *>(cv.take((size_t)R * 4));   // row -> assignment
}

}  // namespace

size_t stage_scratch_bytes(const moe_config &c)
{
    Carver cv{nullptr};
    StageScratch s;
    carve_stage_into(c, cv, s);
    return cv.off;
}

StageScratch carve_stage(const moe_config &c, void *ws)
{
    Carver cv{static_cast<char *>(ws)};
    StageScratch s;
    carve_stage_into(c, cv, s);
    return s;
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status check_cfg(const moe_config *cfg)
{
    if (!cfg)
        return MOE_ERR_NULL;
    return validate(*cfg);
}

}  // namespace

extern "C" {

const char *moe_status_string(moe_status s)
{
    switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_NULL: return "a required pointer is NULL";
    case MOE_ERR_SHAPE: return "shape outside the supported limits";
    case MOE_ERR_CAPACITY_FACTOR: return "capacity factor must be >= 1.0";
    case MOE_ERR_ALIGN: return "pointer or row pitch not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_DTYPE: return "unknown dtype, activation, score or priority code";
    case MOE_ERR_CUDA: return "CUDA launch failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "a device-side wait timed out";
    }
    return "unknown status";
}

moe_status moe_validate(const moe_config *cfg) { return check_cfg(cfg); }

moe_status moe_capacity_value(const moe_config *cfg, int64_t *C)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (!C)
        return MOE_ERR_NULL;
    *C = capacity_of(*cfg);
    return MOE_OK;
}

int64_t moe_perm_rows(const moe_config *cfg)
{
    return check_cfg(cfg) == MOE_OK ? perm_rows(*cfg) : -1;
}

int64_t moe_loss_partials_count(const moe_config *cfg)
{
    return check_cfg(cfg) == MOE_OK ? (int64_t)partial_rows(*cfg) * (cfg->E + 1) : -1;
}

size_t moe_stage_workspace_size(const moe_config *cfg)
{
    return check_cfg(cfg) == MOE_OK ? stage_scratch_bytes(*cfg) : 0;
}

size_t moe_workspace_size(const moe_config *cfg)
{
    if (check_cfg(cfg) != MOE_OK)
        return 0;
    Carver cv{nullptr};
    StageScratch s;
    ForwardBufs f;
    carve_stage_into(*cfg, cv, s);
    carve_forward_into(*cfg, cv, f);
    return cv.off;
}

namespace {

moe_status route_impl(const moe_config *cfg, const void *x, const float *W_r,
                      const float *logit_bias, const float *select_bias, int32_t *topk_idx,
                      float *gates, float *loss_partials, float *logits_out, float *scores_out,
                      void *ws, size_t ws_bytes, moe_stream_t stream, bool clear_status)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (cfg->T == 0)
        return MOE_OK;
    if (!x || !W_r || !topk_idx || !gates || !loss_partials || !ws)
        return MOE_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_ALIGN;
    if (ws_bytes < stage_scratch_bytes(*cfg))
        return MOE_ERR_WORKSPACE;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const RoutePlan plan = route_plan(*cfg);
    if (plan.tensor_cores) {
        if (!aligned16(x))
            return MOE_ERR_ALIGN;
        // the router's first kernel clears the status word itself
        StageScratch s = carve_stage(*cfg, ws);
        return cuda_status(launch_route_tc(*cfg, x, W_r, logit_bias, select_bias, topk_idx,
                                           gates, loss_partials, logits_out, scores_out, s.route,
                                           s.status, clear_status, cs));
    }
    if (clear_status && cudaMemsetAsync(ws, 0, sizeof(int32_t), cs) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(launch_route(*cfg, x, W_r, logit_bias, select_bias, topk_idx, gates,
                                    loss_partials, logits_out, scores_out, cs));
}

}  // namespace

moe_status moe_route(const moe_config *cfg, const void *x, const float *W_r,
                     const float *logit_bias, const float *select_bias, int32_t *topk_idx,
                     float *gates, float *loss_partials, float *logits_out, float *scores_out,
                     void *ws, size_t ws_bytes, moe_stream_t stream)
{
    return route_impl(cfg, x, W_r, logit_bias, select_bias, topk_idx, gates, loss_partials,
                      logits_out, scores_out, ws, ws_bytes, stream, true);
}

moe_status moe_capacity(const moe_config *cfg, const int32_t *topk_idx, int32_t *counts,
                        int32_t *pos, uint8_t *keep, int32_t *kept, int32_t *offsets,
                        uint8_t *dropped, int32_t *n_dropped, void *ws, size_t ws_bytes,
                        moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (cfg->priority == MOE_PRIORITY_SCORE)
        return MOE_ERR_DTYPE;   // the score order needs the scores: moe_capacity_scored
    if (!counts || !kept || !offsets || !n_dropped || !ws ||
        (cfg->T > 0 && (!topk_idx || !pos || !keep || !dropped)))
        return MOE_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_ALIGN;
    if (ws_bytes < stage_scratch_bytes(*cfg))
        return MOE_ERR_WORKSPACE;
    StageScratch s = carve_stage(*cfg, ws);
    return cuda_status(launch_capacity(*cfg, capacity_of(*cfg), topk_idx, counts, pos, keep, kept,
                                       offsets, dropped, n_dropped, s.hist,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_capacity_sharded(const moe_config *cfg, int64_t capacity,
                                const int32_t *shard_counts, int32_t n_shards, int32_t shard,
                                const int32_t *topk_idx,
                                int32_t *counts, int32_t *pos, uint8_t *keep, int32_t *kept,
                                int32_t *offsets, uint8_t *dropped, int32_t *n_dropped, void *ws,
                                size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (cfg->priority != MOE_PRIORITY_TOKEN)
        return MOE_ERR_DTYPE;   // across shards only the token order is a prefix sum
    if (capacity < 0 || n_shards < 1 || shard < 0 || shard >= n_shards)
        return MOE_ERR_SHAPE;
    if (!shard_counts || !counts || !kept || !offsets || !n_dropped || !ws ||
        (cfg->T > 0 && (!topk_idx || !pos || !keep || !dropped)))
        return MOE_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_ALIGN;
    if (ws_bytes < stage_scratch_bytes(*cfg))
        return MOE_ERR_WORKSPACE;
    StageScratch s = carve_stage(*cfg, ws);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_shard_base(*cfg, shard_counts, shard, s.count_base, cs);
    if (e != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(launch_capacity(*cfg, capacity, topk_idx, counts, pos, keep, kept, offsets,
                                       dropped, n_dropped, s.hist, cs, s.count_base));
}

moe_status moe_capacity_scored(const moe_config *cfg, const int32_t *topk_idx,
                               const float *scores, int32_t *counts, int32_t *pos, uint8_t *keep,
                               int32_t *kept, int32_t *offsets, uint8_t *dropped,
                               int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (cfg->priority != MOE_PRIORITY_SCORE)
        return MOE_ERR_DTYPE;
    if (!counts || !kept || !offsets || !n_dropped || !ws ||
        (cfg->T > 0 && (!topk_idx || !scores || !pos || !keep || !dropped)))
        return MOE_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_ALIGN;
    if (ws_bytes < stage_scratch_bytes(*cfg))
        return MOE_ERR_WORKSPACE;
    StageScratch s = carve_stage(*cfg, ws);
    return cuda_status(launch_capacity_scored(*cfg, capacity_of(*cfg), topk_idx, scores, counts,
                                              pos, keep, kept, offsets, dropped, n_dropped,
                                              s.hist, s.keys,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch_rows(const moe_config *cfg, const int32_t *topk_idx, const int32_t *pos,
                             const uint8_t *keep, const int32_t *offsets, int32_t *src_slot,
                             moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (!offsets || !src_slot || (cfg->T > 0 && (!topk_idx || !pos || !keep)))
        return MOE_ERR_NULL;
    return cuda_status(launch_dispatch_rows(*cfg, topk_idx, pos, keep, offsets, src_slot,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                        const int32_t *pos, const uint8_t *keep, const int32_t *offsets,
                        void *x_perm, int32_t *src_slot, void *zero_rows, moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (cfg->T == 0)
        return MOE_OK;
    if (!x || !topk_idx || !pos || !keep || !offsets || !x_perm)
        return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(x_perm) || (zero_rows && !aligned16(zero_rows)))
        return MOE_ERR_ALIGN;
    return cuda_status(launch_dispatch(*cfg, x, topk_idx, pos, keep, offsets, x_perm,
                                       reinterpret_cast<cudaStream_t>(stream), src_slot,
                                       zero_rows));
}

namespace {

// x_perm NULL: routed rows gathered from x through src_slot.  slot_out
// non-NULL: GEMM2 writes gates[a] * FFN(row) to row a of slot_out (src_slot,
// kept, gates required) instead of Y_perm.
moe_status expert_ffn_impl(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                           const int32_t *src_slot, const void *W1, const void *W3,
                           const void *W2, const void *x, const void *Ws1, const void *Ws3,
                           const void *Ws2, void *Y_perm,
                           void *Y_shared, void *ws, size_t ws_bytes, moe_stream_t stream,
                           bool clear_status, const int32_t *kept = nullptr,
                           const float *gates = nullptr, void *slot_out = nullptr)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    const moe_config &c = *cfg;
    const bool swiglu = c.act == MOE_ACT_SWIGLU;
    const bool shared = c.n_shared > 0;
    if (!offsets || !W1 || !W2 || !ws || (swiglu && !W3) || (!slot_out && !Y_perm))
        return MOE_ERR_NULL;
    if (!x_perm && (!src_slot || (c.T > 0 && !x)))   // routed rows: x_perm, or gathered from x
        return MOE_ERR_NULL;
    if (slot_out && (!src_slot || !kept || !gates))
        return MOE_ERR_NULL;
    if (shared && (!x || !Ws1 || !Ws2 || !Y_shared || (swiglu && !Ws3)))
        return MOE_ERR_NULL;
    const void *ptrs[] = {x_perm, W1, W3, W2, x, Ws1, Ws3, Ws2, Y_perm, Y_shared, slot_out};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return MOE_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_ALIGN;
    if (ws_bytes < stage_scratch_bytes(c))
        return MOE_ERR_WORKSPACE;
    StageScratch s = carve_stage(c, ws);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    // bf16: GEMM1 clears the status word itself before any of its waits
    if (clear_status && c.dtype != MOE_DTYPE_BF16 &&
        cudaMemsetAsync(s.status, 0, sizeof(int32_t), cs) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (c.dtype == MOE_DTYPE_BF16)
        e = launch_ffn_tcgen05(c, x_perm, offsets, src_slot, W1, W3, W2, x, Ws1, Ws3, Ws2, Y_perm,
                               Y_shared, s.H, s.H_sh, s.status, clear_status, cs, kept, gates,
                               slot_out);
    else
        e = launch_ffn_simt(c, x_perm, offsets, src_slot, W1, W3, W2, x, Ws1, Ws3, Ws2, Y_perm,
                            Y_shared, s.H, s.H_sh, cs, kept, gates, slot_out);
    return cuda_status(e);
}

}  // namespace

moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                          const void *W1, const void *W3, const void *W2, const void *x,
                          const void *Ws1, const void *Ws3, const void *Ws2, void *Y_perm,
                          void *Y_shared, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    return expert_ffn_impl(cfg, x_perm, offsets, nullptr, W1, W3, W2, x, Ws1, Ws3, Ws2, Y_perm,
                           Y_shared, ws, ws_bytes, stream, true);
}

moe_status moe_expert_ffn_gather(const moe_config *cfg, const void *x, const int32_t *src_slot,
                                 const int32_t *offsets, const void *W1, const void *W3,
                                 const void *W2, const void *Ws1, const void *Ws3, const void *Ws2,
                                 void *Y_perm, void *Y_shared, void *ws, size_t ws_bytes,
                                 moe_stream_t stream)
{
    if (!src_slot)
        return MOE_ERR_NULL;
    return expert_ffn_impl(cfg, nullptr, offsets, src_slot, W1, W3, W2, x, Ws1, Ws3, Ws2, Y_perm,
                           Y_shared, ws, ws_bytes, stream, true);
}

moe_status moe_expert_ffn_slots(const moe_config *cfg, const void *x_perm, const void *x,
                                const int32_t *src_slot, const int32_t *offsets,
                                const int32_t *kept, const float *gates, const void *W1,
                                const void *W3, const void *W2, const void *Ws1, const void *Ws3,
                                const void *Ws2, void *Y_slot, void *Y_shared, void *ws,
                                size_t ws_bytes, moe_stream_t stream)
{
    if (!src_slot || !kept || !gates || !Y_slot)
        return MOE_ERR_NULL;
    return expert_ffn_impl(cfg, x_perm, offsets, src_slot, W1, W3, W2, x, Ws1, Ws3, Ws2, nullptr,
                           Y_shared, ws, ws_bytes, stream, true, kept, gates, Y_slot);
}

moe_status moe_combine_slots(const moe_config *cfg, const void *Y_slot, const void *Y_shared,
                             const uint8_t *keep, const void *residual, void *y,
                             moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (cfg->T == 0)
        return MOE_OK;
    if (!Y_slot || !keep || !y || (cfg->n_shared > 0 && !Y_shared))
        return MOE_ERR_NULL;
    const void *ptrs[] = {Y_slot, Y_shared, residual, y};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return MOE_ERR_ALIGN;
    return cuda_status(launch_combine_slots(*cfg, Y_slot, Y_shared, keep, residual, y,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_config *cfg, const void *Y_perm, const void *Y_shared,
                       const float *gates, const int32_t *topk_idx, const int32_t *pos,
                       const uint8_t *keep, const int32_t *offsets, const void *residual,
                       void *y, moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (cfg->T == 0)
        return MOE_OK;
    if (!Y_perm || !gates || !topk_idx || !pos || !keep || !offsets || !y ||
        (cfg->n_shared > 0 && !Y_shared))
        return MOE_ERR_NULL;
    const void *ptrs[] = {Y_perm, Y_shared, residual, y};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return MOE_ERR_ALIGN;
    return cuda_status(launch_combine(*cfg, Y_perm, Y_shared, gates, topk_idx, pos, keep,
                                      offsets, residual, y,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_losses(const moe_config *cfg, const int32_t *counts, const float *loss_partials,
                      float *aux, float *zloss, moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (!counts || !aux || !zloss || (cfg->T > 0 && !loss_partials))
        return MOE_ERR_NULL;
    return cuda_status(launch_losses(*cfg, counts, loss_partials, aux, zloss,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_seq_balance_loss(const moe_config *cfg, int32_t seq_len, const int32_t *topk_idx,
                                const float *loss_partials, float *per_seq, float *loss,
                                moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (seq_len < kPartialTokens || seq_len % kPartialTokens || cfg->T < 1 || cfg->T % seq_len)
        return MOE_ERR_SHAPE;
    if (!topk_idx || !loss_partials || !per_seq || !loss)
        return MOE_ERR_NULL;
    return cuda_status(launch_seq_loss(*cfg, seq_len, topk_idx, loss_partials, per_seq, loss,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_bias_update(const moe_config *cfg, const int32_t *counts, float gamma,
                           float *select_bias, moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (!isfinite(gamma))
        return MOE_ERR_SHAPE;
    if (!counts || !select_bias)
        return MOE_ERR_NULL;
    return cuda_status(launch_bias_update(*cfg, counts, gamma, select_bias,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_forward(const moe_config *cfg, const moe_weights *w, const void *x,
                       const moe_outputs *out, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK)
        return st;
    if (!w || !out || !ws || !out->aux || !out->zloss || !w->W_r || !w->W1 || !w->W2)
        return MOE_ERR_NULL;
    const moe_config &c = *cfg;
    if (c.T > 0 && (!x || !out->y))
        return MOE_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_ALIGN;
    if (ws_bytes < moe_workspace_size(cfg))
        return MOE_ERR_WORKSPACE;
    Carver cv{static_cast<char *>(ws)};
    StageScratch s;
    ForwardBufs f;
    carve_stage_into(c, cv, s);
    carve_forward_into(c, cv, f);
    if (out->topk_idx) f.topk = out->topk_idx;
    if (out->gates) f.gates = out->gates;
    if (out->keep) f.keep = out->keep;
    if (out->dropped) f.dropped = out->dropped;
    if (out->counts) f.counts = out->counts;
    if (out->n_dropped) f.n_dropped = out->n_dropped;
    const size_t ssz = stage_scratch_bytes(c);
    if (c.T == 0 && (st = moe_clear_device_status(ws, stream)) != MOE_OK)
        return st;
    const bool scored = c.priority == MOE_PRIORITY_SCORE;
    // the router clears the status word once for the whole layer
    if ((st = route_impl(cfg, x, w->W_r, w->logit_bias, w->select_bias, f.topk, f.gates,
                         f.partials, nullptr, scored ? f.scores : nullptr, ws, ssz, stream,
                         true)) != MOE_OK)
        return st;
    if (scored)
        st = moe_capacity_scored(cfg, f.topk, f.scores, f.counts, f.pos, f.keep, f.kept,
                                 f.offsets, f.dropped, f.n_dropped, ws, ssz, stream);
    else   // token or rank order: the capacity launch also writes the two losses
        st = cuda_status(launch_capacity(c, capacity_of(c), f.topk, f.counts, f.pos, f.keep,
                                         f.kept, f.offsets, f.dropped, f.n_dropped, s.hist,
                                         reinterpret_cast<cudaStream_t>(stream), nullptr,
                                         f.partials, s.loss_ps, out->aux, out->zloss));
    if (st != MOE_OK)
        return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (c.k == 1 && c.n_shared == 0) {
        // one slot per token and no shared expert: the combine is the gate,
        // applied in GEMM2's epilogue, which writes y's rows directly; the
        // dispatch records each row's assignment and zeroes dropped tokens' y
        if ((st = cuda_status(launch_dispatch(c, x, f.topk, f.pos, f.keep, f.offsets, f.x_perm, cs,
                                              f.slot, out->y))) != MOE_OK)
            return st;
        if ((st = expert_ffn_impl(cfg, f.x_perm, f.offsets, f.slot, w->W1, w->W3, w->W2, x,
                                  w->Ws1, w->Ws3, w->Ws2, nullptr, nullptr, ws, ssz, stream,
                                  false, f.kept, f.gates, out->y)) != MOE_OK)
            return st;
    } else {
        if ((st = cuda_status(launch_dispatch(c, x, f.topk, f.pos, f.keep, f.offsets, f.x_perm,
                                              cs))) != MOE_OK)
            return st;
        if ((st = expert_ffn_impl(cfg, f.x_perm, f.offsets, nullptr, w->W1, w->W3, w->W2, x,
                                  w->Ws1, w->Ws3, w->Ws2, f.Y_perm, f.Y_sh, ws, ssz, stream,
                                  false)) != MOE_OK)
            return st;
        if ((st = moe_combine(cfg, f.Y_perm, f.Y_sh, f.gates, f.topk, f.pos, f.keep, f.offsets,
                              nullptr, out->y, stream)) != MOE_OK)
            return st;
    }
    return scored ? moe_losses(cfg, f.counts, f.partials, out->aux, out->zloss, stream) : MOE_OK;
}

moe_status moe_device_status(const void *ws, int32_t *status, moe_stream_t stream)
{
    if (!ws || !status)
        return MOE_ERR_NULL;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(status, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(cs));
}

moe_status moe_probe_wait_timeout(void *ws, uint64_t timeout_ns, moe_stream_t stream)
{
    if (!ws)
        return MOE_ERR_NULL;
    if (timeout_ns > 2000000000ull)
        return MOE_ERR_SHAPE;
    return cuda_status(launch_wait_probe(static_cast<int32_t *>(ws), timeout_ns,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_clear_device_status(void *ws, moe_stream_t stream)
{
    if (!ws)
        return MOE_ERR_NULL;
    return cuda_status(
        cudaMemsetAsync(ws, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
