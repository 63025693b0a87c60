// Expert FFNs in bf16 on the 5th-generation tensor cores: a persistent,
// warp-specialised grouped GEMM (TMA -> shared memory -> tcgen05.mma -> TMEM
// -> epilogue -> TMA store) over the variable-length expert segments.
//
// Page "Lab 18 - Mixture of experts": section 1 (experts are W2 gelu(W1 x) or
// W2 (silu(W1 x) * (W3 x))), tips ("production kernels do the same thing as one
// grouped matrix multiply over all experts"); shared experts run on every token
// ("Lab 18" section 1, DeepSeekMoE row).
//
// Two launches: GEMM1 (hidden = act(A W1^T), SwiGLU fuses W3) and GEMM2
// (out = hidden W2^T).  GEMM1's routed A rows come either from the permuted
// buffer x_perm or, with the dispatch fused in, straight from x: four more
// warps copy each stage's 128 rows with 16-byte cp.async through the per-row
// assignment table that moe_dispatch_rows writes (a TMA row gather, 4 rows
// per instruction, was bound by the TMA issue rate: 64 instructions per stage
// instead of 2).  GEMM2 may take the combine's gate too: each kept
// row, times its assignment's gate, goes straight to that assignment's row of
// a [T k, d] output (EPI_GATED).  Each launch covers two tile sets:
//   set 0, routed: for expert e the rows [offsets[e], offsets[e+1]) of the
//          permuted buffer, read from device memory (no host sync); segments
//          start on multiples of 128 rows, so a 128-row tile has one expert;
//   set 1, shared: all T token rows.  GEMM1 spreads the S shared experts over
//          the N tiles (each writes its own column block of the hidden
//          buffer); GEMM2 runs K over all S experts so their outputs add up in
//          the TMEM accumulator.
// Tile = 128 rows x 256 accumulator columns, K step 64 (one 128-byte swizzle
// atom of bf16), 4-stage TMA ring, double-buffered TMEM accumulator (2 x 256
// of the 512 columns) so the epilogue of one tile overlaps the MMAs of the
// next.  SwiGLU tiles load 128 rows of W1 and the same 128 rows of W3 into one
// 256-row B tile: accumulator columns [0,128) hold x W1^T, [128,256) x W3^T.
//
// Warps: 0 = TMA producer, 1 = MMA issuer (and TMEM owner), 2..9 = epilogue
// (warp w reads TMEM lanes 32 (w mod 4) .. +31; warps 2..5 take the first half
// of the tile's columns, warps 6..9 the second), 10..13 = gather warps (only
// when GEMM1 reads its rows from x).  Every wait on an mbarrier is
// bounded by a wall-clock limit; on expiry the CTA records
// MOE_ERR_DEVICE_TIMEOUT in the status word, every role leaves its loop, the
// CTA drains what it issued (bounded as well), frees TMEM and returns.
#include "internal.cuh"

#include <cuda.h>

namespace moe {
namespace tc {

constexpr int BM = 128, BK = 64, BN = 256, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B_BYTES = BN * BK * 2;                 // 32 KB
constexpr int EPI_WARPS = 8;                          // two per TMEM lane quarter
constexpr int THREADS = 64 + 32 * EPI_WARPS;         // 320
// Epilogue: a warp moves CHUNK accumulator columns of its 32 rows per step,
// through STG_BUFS staging buffers of its own (a buffer is written again only
// once the TMA store issued from it STG_BUFS steps earlier has read it), as
// 32 rows of 2 CHUNK bytes in the swizzle of the store map (16-byte chunk c of
// row r at c ^ ((r >> (3 - SWZ_BITS)) & (2^SWZ_BITS - 1))).
constexpr int CHUNK = 32;                            // epilogue columns per step
constexpr int STG_BUFS = 1;
constexpr int STG_BYTES = 32 * CHUNK * 2;            // one buffer: 32 rows x CHUNK bf16
constexpr int STG_WARP = STG_BUFS * STG_BYTES;       // a warp's buffers
constexpr int SWZ_BITS = CHUNK == 16 ? 1 : (CHUNK == 32 ? 2 : 3);   // 32, 64 or 128 B rows
constexpr uint32_t TMEM_COLS = 512;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_STG = OFF_B + STAGES * B_BYTES;
constexpr int OFF_BAR = OFF_STG + EPI_WARPS * STG_WARP;
constexpr int OFF_TILES = OFF_BAR + 256;
constexpr int SMEM_BYTES = OFF_TILES + 2 * 4 * (kMaxE + 1) + 1024;   // + alignment slack

// EPI_GATED: GEMM2 with the combine's gate fused (routed rows only): row r
// of expert e's segment, when kept (r - offsets[e] < kept[e]), holds
// assignment a = src_slot[r]; gates[a] * acc goes, rounded to bf16, to row a
// of slot_out.  Shared-expert tiles store as EPI_NONE.
enum Epi { EPI_NONE = 0, EPI_GELU = 1, EPI_SWIGLU = 2, EPI_GATED = 3 };

struct SetDesc {
    int routed;     // 1: rows and B group from the segment table
    int rows;       // dense row count (shared set)
    int n_tiles;    // N tiles per N group
    int n_groups;   // groups the N tiles run over (shared GEMM1: S), else 1
    int k_blocks;   // K blocks per tile
    int kbg;        // > 0: K runs over groups, kbg blocks each (shared GEMM2)
    int c_cols;     // columns of the output tensor (chunks at or past it are skipped)
};

struct __align__(64) Params {
    CUtensorMap tmA[2], tmB[2], tmB3[2], tmC[2];
    SetDesc set[2];
    int nsets;
    int E;
    int gather;                  // 1: routed A rows gathered from x through src_slot
    const __nv_bfloat16 *xg;     // x [T][x_ld] (gathered A rows)
    int x_ld;
    int n_rows;                  // rows of the permuted buffers (entries of src_slot)
    int k;                       // experts per token: token of assignment a = a / k
    const int32_t *src_slot;     // [n_rows] assignment t k + j of each permuted row (-1: none)
    const int32_t *kept;         // [E] kept rows of each segment (EPI_GATED)
    const float *gates;          // [T k] (EPI_GATED)
    __nv_bfloat16 *slot_out;     // [T k][slot_ld] (EPI_GATED)
    int slot_ld;
    const int32_t *offsets;
    int32_t *status;
    int clear_status;            // 1: block 0 clears the status word before any wait
    unsigned long long timeout_ns;
};

// ------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// CL: acquire at cluster scope (the barrier's arrivals include writes of the
// other CTA of an SM pair made by its threads, not by TMA)
template <bool CL = false>
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    if (CL)
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
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

struct Ctl {
    volatile int *abort;
    int32_t *status;
    uint64_t timeout_ns;
};

// Wait for the phase of `bar` with the given parity to complete.  Gives up
// (returns false) when the time limit passed or, if honor_abort, when another
// role already gave up.  Drain waits pass honor_abort = false: they must see
// their own copies land even after an abort, but stay bounded.
template <bool CL = false>
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl &c,
                                      bool honor_abort = true)
{
    if (mbar_try<CL>(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try<CL>(bar, parity))
            return true;
        if ((i & 31u) == 0) {
            if (honor_abort && *c.abort)
                return false;
            if (global_ns() - t0 > c.timeout_ns) {
                *c.abort = 1;
                atomicExch(c.status, (int32_t)MOE_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

// ---- gathered A rows (the dispatch fused into GEMM1) ----
// GATHER_WARPS extra warps copy the tile's 128 rows of each stage straight
// from x with 16-byte cp.async, into the 128-byte swizzled layout a TMA box
// would give (row r of a 64-wide box at r * 128 bytes, its 16-byte chunk j at
// position j ^ (r & 7)).  A warp copies whole rows: with KS boxes per stage a
// row is 8 KS chunks, so one instruction moves 32 / (8 KS) rows.
constexpr int GATHER_WARPS = 4;

// 16 bytes, or (src_bytes = 0) 16 zero bytes without reading src
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int KS>
struct GatherLanes {
    static constexpr int CPR = 8 * KS;      // 16-byte chunks of a row per stage
    static constexpr int RPI = 32 / CPR;    // rows per warp instruction
    static constexpr int NI = 32 / RPI;     // instructions per warp per stage (32 rows)
};

// This lane's copies of one stage: gather warp gw owns rows [32 gw, 32 gw + 32)
// of the CTA's 128; tok[i] is the token of its row in instruction i.  Columns
// at or past the row length x_ld (the second box of a stage when d is an odd
// multiple of 64) are zero-filled, as TMA fills a box past the tensor.
template <int KS>
__device__ __forceinline__ void gather_stage(uint32_t a_stage, uint32_t box_stride,
                                             const __nv_bfloat16 *x, int x_ld, int kcol,
                                             const int *tok, int gw, int lane)
{
    using G = GatherLanes<KS>;
    const int c = lane % G::CPR, sub = lane / G::CPR;
    const int box = c >> 3, j = c & 7;
    const bool inside = kcol + c * 8 < x_ld;
#pragma unroll
    for (int i = 0; i < G::NI; ++i) {
        const int row = 32 * gw + G::RPI * i + sub;
        const __nv_bfloat16 *src = inside ? x + (int64_t)tok[i] * x_ld + kcol + c * 8 : x;
        cp_async16(a_stage + box * box_stride + row * 128 + ((j ^ (row & 7)) << 4), src,
                   inside ? 16u : 0u);
    }
}

// A stage's copies by this lane have landed (cp.async.wait_group before this):
// make them visible to the tensor core (async proxy), then one arrive per
// warp on the stage's full barrier; PAIR: the leader CTA's barrier, releasing
// at cluster scope.
template <bool PAIR>
__device__ __forceinline__ void gather_arrive(uint32_t full, int lane)
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
        if (PAIR) {
            uint32_t remote;
            asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(remote) : "r"(full));
            asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                             remote)
                         : "memory");
        } else {
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(full) : "memory");
        }
    }
}

// the token whose x row permuted row r holds (padding rows, and rows past the
// table, read token 0; their results are never used)
__device__ __forceinline__ int gather_row(const Params &p, int r)
{
    const int a = r < p.n_rows ? p.src_slot[r] : -1;
    return a >= 0 ? a / p.k : 0;
}

// EPI_GATED: the assignment a routed row `row` of expert e holds (-1 for a
// padding row) and its gate.
__device__ __forceinline__ int gated_slot(const Params &p, int e, int row, float *gate)
{
    const int a = row - p.offsets[e] < p.kept[e] ? p.src_slot[row] : -1;
    *gate = a >= 0 ? p.gates[a] : 0.f;
    return a;
}

// EPI_GATED: CHUNK accumulator columns of one row, times the gate, rounded to
// bf16, to 2 CHUNK bytes of the slot's output row.
__device__ __forceinline__ void store_gated(const Params &p, int a, float gate, int col,
                                            const float *v)
{
    uint4 *dst = reinterpret_cast<uint4 *>(p.slot_out + (int64_t)a * p.slot_ld + col);
#pragma unroll
    for (int q = 0; q < CHUNK / 8; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(gate * v[8 * q + 2 * i],
                                                     gate * v[8 * q + 2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int c0, int c1,
                                             int c2)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::
                     "l"(reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(src)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the TMA stores issued from this thread, all but the last n, have read their source
template <int N>
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand tile in shared memory, 128-byte swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart (stride byte offset 64 x 16 B), leading byte
// offset unused for this layout (1), descriptor version 1, layout code 2.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                     "r"(bar)
                 : "memory");
}

// 32 lanes x 16 consecutive fp32 columns: thread i gets lane (base + i)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 32 consecutive fp32 columns: thread i gets lane (base + i)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------ tile schedule

struct Tile {
    int set;
    int m0;       // first row of A and C
    int b_group;  // group of the B tensor (K not split)
    int b_row;    // first B row inside the group
    int c_col;    // first C column
    int c_group;  // group of the C tensor
};

// Tile `tile` of 128 rows: routed tiles expert by expert, N outer and row
// tiles inner; then the shared set over its dense rows.
__device__ __forceinline__ Tile decode(const Params &p, const int *tstart, const int *mtiles,
                                       int routed_total, int tile, int bn_b, int bn_out)
{
    Tile t;
    if (tile < routed_total) {
        int lo = 0, hi = p.E;   // last e with tstart[e] <= tile
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (tstart[mid] <= tile)
                lo = mid;
            else
                hi = mid;
        }
        const int e = lo, i = tile - tstart[e], mt = mtiles[e];
        const int n = i / mt, m = i % mt;
        t.set = 0;
        t.m0 = p.offsets[e] + m * BM;
        t.b_group = e;
        t.b_row = n * bn_b;
        t.c_col = n * bn_out;
        t.c_group = 0;
    } else {
        const SetDesc &s = p.set[1];
        const int i = tile - routed_total;
        const int mt = (s.rows + BM - 1) / BM;
        const int n = i / mt, m = i % mt;
        const int g = n / s.n_tiles, nn = n % s.n_tiles;
        t.set = 1;
        t.m0 = m * BM;
        t.b_group = g;
        t.b_row = nn * bn_b;
        t.c_col = nn * bn_out;
        t.c_group = g;
    }
    return t;
}

// CHUNK columns of this thread's accumulator row
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, float *v)
{
    if (CHUNK == 16)
        tmem_ld16(taddr, v);
    else
        tmem_ld32(taddr, v);
}

// Stage this thread's row of packed bf16 (2 CHUNK bytes) into a staging buffer
// in the store map's swizzle.
__device__ __forceinline__ void stage_row(uint8_t *buf, int lane, const uint32_t *packed)
{
    uint8_t *row = buf + lane * (CHUNK * 2);
#pragma unroll
    for (int ch = 0; ch < CHUNK / 8; ++ch) {
        const int phys = ch ^ ((lane >> (3 - SWZ_BITS)) & ((1 << SWZ_BITS) - 1));
        *reinterpret_cast<uint4 *>(row + phys * 16) =
            make_uint4(packed[4 * ch], packed[4 * ch + 1], packed[4 * ch + 2], packed[4 * ch + 3]);
    }
}

template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const float *g, const float *u, uint32_t *packed)
{
#pragma unroll
    for (int i = 0; i < CHUNK; i += 2) {
        float a, b;
        if (EPI == EPI_SWIGLU) {   // silu(g) * u, fast reciprocal (output is bf16)
            a = __fdividef(g[i], 1.f + __expf(-g[i])) * u[i];
            b = __fdividef(g[i + 1], 1.f + __expf(-g[i + 1])) * u[i + 1];
        } else if (EPI == EPI_GELU) {
            a = 0.5f * g[i] * (1.f + erff(g[i] * 0.70710678118654752f));
            b = 0.5f * g[i + 1] * (1.f + erff(g[i + 1] * 0.70710678118654752f));
        } else {
            a = g[i];
            b = g[i + 1];
        }
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        packed[i / 2] = *reinterpret_cast<uint32_t *>(&h);
    }
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(THREADS + (GATHER ? 32 * GATHER_WARPS : 0), 1)
    grouped_gemm_kernel(const __grid_constant__ Params p)
{
    constexpr int BN_B = EPI == EPI_SWIGLU ? BN / 2 : BN;     // B rows per tensor per tile
    constexpr int BN_OUT = EPI == EPI_SWIGLU ? BN / 2 : BN;   // output columns per tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sA = smem_u32(smem + OFF_A);
    const uint32_t sB = smem_u32(smem + OFF_B);
    const uint32_t sStg = smem_u32(smem + OFF_STG);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    // full[0..S), empty[S..2S), tfull[2S, 2S+2), tempty[2S+2, 2S+4), drain 2S+4
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8 * (2 * STAGES + 5));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *tstart = reinterpret_cast<int *>(smem + OFF_TILES);    // [E + 1]
    int *mtiles = tstart + (kMaxE + 1);                         // [E]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Ctl ctl{abort_flag, p.status, p.timeout_ns};

    // ---- set-up: barriers, TMEM, tile table ----
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // the producer's expect_tx arrive, and one arrive per gather warp
            mbar_init(full_bar(s), 1 + (GATHER ? GATHER_WARPS : 0));
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), EPI_WARPS);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // the segment table and the A rows come from the previous kernels
    pdl_wait();
    pdl_trigger();
    if (p.clear_status && blockIdx.x == 0 && threadIdx.x == 0)
        *p.status = 0;
    int routed_total = 0;
    if (p.set[0].routed && p.nsets > 0) {
        for (int e = threadIdx.x; e < p.E; e += blockDim.x)
            mtiles[e] = (p.offsets[e + 1] - p.offsets[e]) / BM;
        __syncthreads();
        if (threadIdx.x == 0) {
            int acc = 0;
            for (int e = 0; e < p.E; ++e) {
                tstart[e] = acc;
                acc += mtiles[e] * p.set[0].n_tiles;
            }
            tstart[p.E] = acc;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (p.set[0].routed && p.nsets > 0)
        routed_total = tstart[p.E];
    int shared_total = 0;
    if (p.nsets > 1) {
        const SetDesc &s = p.set[1];
        shared_total = (s.rows + BM - 1) / BM * s.n_tiles * s.n_groups;
    }
    const int total = routed_total + shared_total;
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ================= TMA producer =================
        // Lane 0 owns the barrier waits and the box copies (with gathered A
        // rows, the B boxes only: the gather warps copy A).
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued[STAGES];
            uint32_t last_phase[STAGES];
            for (int s = 0; s < STAGES; ++s)
                issued[s] = 0, last_phase[s] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                const Tile t = decode(p, tstart, mtiles, routed_total, tile, BN_B, BN_OUT);
                const SetDesc &sd = p.set[t.set];
                const bool gath = GATHER && t.set == 0;
                for (int kb = 0; kb < sd.k_blocks; ++kb) {
                    if (!wait_bar(empty_bar(stage), phase ^ 1u, ctl)) {
                        ok = false;
                        break;
                    }
                    int kcol = kb * BK, ga = 0, gb = t.b_group;
                    if (sd.kbg > 0) {
                        ga = gb = kb / sd.kbg;
                        kcol = (kb % sd.kbg) * BK;
                    }
                    const uint32_t fb = full_bar(stage);
                    mbar_expect_tx(fb, (gath ? 0 : A_BYTES) + B_BYTES);
                    if (!gath)
                        tma_load_3d(sA + stage * A_BYTES, &p.tmA[t.set], fb, kcol, t.m0, ga);
                    const uint32_t b0 = sB + stage * B_BYTES;
                    if (EPI == EPI_SWIGLU) {
                        tma_load_3d(b0, &p.tmB[t.set], fb, kcol, t.b_row, gb);
                        tma_load_3d(b0 + B_BYTES / 2, &p.tmB3[t.set], fb, kcol, t.b_row, gb);
                    } else {
                        tma_load_3d(b0, &p.tmB[t.set], fb, kcol, t.b_row, gb);
                    }
                    issued[stage] = 1;
                    last_phase[stage] = phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain: every load this CTA issued has landed before it exits
            for (int s = 0; s < STAGES; ++s)
                if (issued[s])
                    wait_bar(full_bar(s), last_phase[s], ctl, false);
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, any = false;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                const Tile t = decode(p, tstart, mtiles, routed_total, tile, BN_B, BN_OUT);
                const SetDesc &sd = p.set[t.set];
                if (!wait_bar(tempty_bar(acc), acc_phase ^ 1u, ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tmem_d = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < sd.k_blocks; ++kb) {
                    if (!wait_bar(full_bar(stage), phase, ctl)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = sA + stage * A_BYTES, b_base = sB + stage * B_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_bf16(tmem_d, sdesc_sw128(a_base + kk * 32), sdesc_sw128(b_base + kk * 32),
                                 (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(empty_bar(stage));
                    any = true;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                mma_commit(tfull_bar(acc));
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (any) {   // all MMAs issued by this thread complete before TMEM is freed
                mma_commit(drain_bar);
                wait_bar(drain_bar, 0, ctl, false);
            }
        }
    } else if (GATHER && warp >= 2 + EPI_WARPS) {
        // ================= gather warps: routed A rows from x =================
        // A stage is signalled D issues after its copies were issued, so the
        // copies of D + 1 stages are in flight while the MMA has a full stage
        // to work on.
        using G = GatherLanes<1>;
        constexpr int D = STAGES - 2;
        const int gw = warp - (2 + EPI_WARPS);
        const int sub = lane / G::CPR;
        int stage = 0, seq = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
            const Tile t = decode(p, tstart, mtiles, routed_total, tile, BN_B, BN_OUT);
            const SetDesc &sd = p.set[t.set];
            const bool gath = t.set == 0;   // shared-expert tiles: TMA boxes of x
            int tok[G::NI];
#pragma unroll
            for (int i = 0; i < G::NI; ++i)
                tok[i] = gath ? gather_row(p, t.m0 + 32 * gw + G::RPI * i + sub) : 0;
            for (int kb = 0; kb < sd.k_blocks; ++kb) {
                int okw = lane == 0 ? (wait_bar(empty_bar(stage), phase ^ 1u, ctl) ? 1 : 0) : 1;
                if (!__shfl_sync(0xffffffffu, okw, 0)) {
                    ok = false;
                    break;
                }
                if (gath)
                    gather_stage<1>(sA + stage * A_BYTES, 0, p.xg, p.x_ld, kb * BK, tok, gw, lane);
                cp_async_commit();
                if (seq >= D) {
                    cp_async_wait<D>();
                    gather_arrive<false>(full_bar((stage + STAGES - D) % STAGES), lane);
                }
                ++seq;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        cp_async_wait<0>();   // the last stages' copies, then their arrivals
        for (int q = seq < D ? seq : D; q > 0; --q)
            gather_arrive<false>(full_bar((stage + STAGES - q) % STAGES), lane);
    } else {
        // ================= epilogue (warps 2..9) =================
        const int q = warp & 3;                      // TMEM lane quarter
        const int ew = warp - 2;                     // staging buffer owner
        const int half = ew >> 2;                    // which half of the columns
        const uint32_t stg = sStg + ew * STG_WARP;
        uint8_t *stg_ptr = smem + OFF_STG + ew * STG_WARP;
        int acc = 0, nchunk = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Tile t = decode(p, tstart, mtiles, routed_total, tile, BN_B, BN_OUT);
            if (!wait_bar(tfull_bar(acc), acc_phase, ctl))
                break;
            tc_fence_after();
            const int c_end = min((half + 1) * (BN_OUT / 2), p.set[t.set].c_cols - t.c_col);
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const int row0 = t.m0 + q * 32;   // this warp's 32 rows
            if (EPI == EPI_GATED && t.set == 0) {
                // gate and scatter: this lane's row goes to its assignment's row
                float gate;
                const int a = gated_slot(p, t.b_group, row0 + lane, &gate);
#pragma unroll 1
                for (int c = half * (BN_OUT / 2); c < c_end; c += CHUNK) {
                    float g[CHUNK];
                    tmem_ld_chunk(tbase + c, g);
                    if (a >= 0)
                        store_gated(p, a, gate, t.c_col + c, g);
                }
            } else {
#pragma unroll 1
            for (int c = half * (BN_OUT / 2); c < c_end; c += CHUNK, ++nchunk) {
                float g[CHUNK], u[CHUNK];
                uint32_t packed[CHUNK / 2];
                tmem_ld_chunk(tbase + c, g);
                if (EPI == EPI_SWIGLU) {
                    tmem_ld_chunk(tbase + BN / 2 + c, u);
                    epilogue_chunk<EPI>(g, u, packed);
                } else {
                    epilogue_chunk<EPI>(g, g, packed);
                }
                const int b = nchunk % STG_BUFS;   // this chunk's staging buffer
                if (lane == 0)
                    bulk_wait_read<STG_BUFS - 1>();
                __syncwarp();
                stage_row(stg_ptr + b * STG_BYTES, lane, packed);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&p.tmC[t.set], stg + b * STG_BYTES, t.c_col + c, row0,
                                 t.c_group);
                    bulk_commit();
                }
            }
            }
            // this warp's reads of the accumulator are done
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tempty_bar(acc));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0)
            bulk_wait_all();
        __syncwarp();
    }

    // ---- tear-down ----
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ===================================================================== 2-SM
// The same grouped GEMM on SM pairs (cta_group::2): a 2-CTA cluster owns a
// 256-row x 256-column accumulator tile, each CTA holding 128 rows of it in
// its own TMEM.  Each CTA loads its 128 rows of A and its half of the B tile
// (SwiGLU: CTA 0 the W1 rows, CTA 1 the same W3 rows), so 64 of K move 32 KB
// into each SM instead of 48 KB.  A stage holds K = 128 (two 64-wide boxes of
// A and of B, 64 KB per SM, three stages): eight MMAs per full/empty barrier
// round trip instead of four, which measured 10% faster than six stages of
// K = 64 with the same bytes in flight (the per-stage hand-over, not memory,
// held the tensor pipe back).  The leader CTA's MMA
// thread issues the M = 256 MMAs for both; its commits are multicast to the
// empty / accumulator-full barriers of both CTAs; both CTAs' TMA loads report
// to the leader's full barriers; both CTAs' epilogues report to the leader's
// accumulator-empty barriers.  A 256-row pair tile lies inside one expert's
// segment; when the segment ends after the first 128 rows, CTA 1 computes
// rows it does not store.

constexpr int STAGES2 = 3;
constexpr int KSUB = 2;                              // 64-wide K boxes per stage
constexpr int HALF_BYTES = 128 * BK * 2;             // 16 KB: 128 rows x 64 bf16
constexpr int OFF2_A = 0;
constexpr int OFF2_B = OFF2_A + STAGES2 * KSUB * HALF_BYTES;
constexpr int OFF2_STG = OFF2_B + STAGES2 * KSUB * HALF_BYTES;
constexpr int OFF2_BAR = OFF2_STG + EPI_WARPS * STG_WARP;
constexpr int OFF2_TILES = OFF2_BAR + 256;
constexpr int SMEM2_BYTES = OFF2_TILES + 2 * 4 * (kMaxE + 1) + 1024;

// kind::f16, fp32 accumulator, bf16 A and B, K-major, N = 256, M = 256
constexpr uint32_t IDESC2 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared variable in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
    return out;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                     "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t bar_leader, int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar_leader)
        : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(IDESC2), "r"(accumulate)
        : "memory");
}

// arrive on the barrier at this shared offset in both CTAs of the pair
__device__ __forceinline__ void mma_commit_pair(uint32_t bar)
{
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void mma_commit_local2(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                     "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

struct Tile2 {
    int set;
    int m0;        // first row of the pair tile
    int b_group;   // B group when K is not split
    int n_idx;     // N tile index inside the group
    int c_group;
    bool second;   // rows m0 + 128 .. belong to the tile's segment
};

__device__ __forceinline__ Tile2 decode2(const Params &p, const int *tstart, const int *mpairs,
                                         int routed_total, int tile)
{
    Tile2 t;
    if (tile < routed_total) {
        int lo = 0, hi = p.E;
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (tstart[mid] <= tile)
                lo = mid;
            else
                hi = mid;
        }
        const int e = lo, i = tile - tstart[e], mp = mpairs[e];
        t.set = 0;
        t.m0 = p.offsets[e] + (i % mp) * 256;
        t.second = t.m0 + 128 < p.offsets[e + 1];
        t.b_group = e;
        t.n_idx = i / mp;
        t.c_group = 0;
    } else {
        const SetDesc &sd = p.set[1];
        const int i = tile - routed_total;
        const int mp = (sd.rows + 255) / 256;
        const int n = i / mp;
        t.set = 1;
        t.m0 = (i % mp) * 256;
        t.second = t.m0 + 128 < sd.rows;
        t.b_group = n / sd.n_tiles;
        t.n_idx = n % sd.n_tiles;
        t.c_group = t.b_group;
    }
    return t;
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(THREADS + (GATHER ? 32 * GATHER_WARPS : 0), 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ Params p)
{
    constexpr int BN_OUT = EPI == EPI_SWIGLU ? BN / 2 : BN;   // output columns per tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sA = smem_u32(smem + OFF2_A);
    const uint32_t sB = smem_u32(smem + OFF2_B);
    const uint32_t sStg = smem_u32(smem + OFF2_STG);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF2_BAR);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES2 + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES2 + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES2 + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES2 + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF2_BAR + 8 * (2 * STAGES2 + 5));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *tstart = reinterpret_cast<int *>(smem + OFF2_TILES);   // [E + 1]
    int *mpairs = tstart + (kMaxE + 1);                        // [E]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const Ctl ctl{abort_flag, p.status, p.timeout_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) {
            // the leader producer's expect_tx arrive, and (gathered A rows) one
            // arrive per gather warp of both CTAs
            mbar_init(full_bar(s), 1 + (GATHER ? 2 * GATHER_WARPS : 0));
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 2 * EPI_WARPS);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    // the segment table and the A rows come from the previous kernels
    pdl_wait();
    pdl_trigger();
    if (p.clear_status && blockIdx.x == 0 && threadIdx.x == 0)
        *p.status = 0;
    int routed_total = 0;
    if (p.set[0].routed && p.nsets > 0) {
        for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
            const int mt = (p.offsets[e + 1] - p.offsets[e]) / BM;
            mpairs[e] = (mt + 1) / 2;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int acc = 0;
            for (int e = 0; e < p.E; ++e) {
                tstart[e] = acc;
                acc += mpairs[e] * p.set[0].n_tiles;
            }
            tstart[p.E] = acc;
        }
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised, TMEM allocated, tables ready
    tc_fence_after();
    if (p.set[0].routed && p.nsets > 0)
        routed_total = tstart[p.E];
    int shared_total = 0;
    if (p.nsets > 1) {
        const SetDesc &sd = p.set[1];
        shared_total = (sd.rows + 255) / 256 * sd.n_tiles * sd.n_groups;
    }
    const int total = routed_total + shared_total;
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ================= TMA producer (both CTAs) =================
        // Lane 0 owns the barrier waits and the box copies (with gathered A
        // rows, the B boxes only: the gather warps copy A).
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued[STAGES2];
            uint32_t last_phase[STAGES2];
            for (int s = 0; s < STAGES2; ++s)
                issued[s] = 0, last_phase[s] = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < total; tile += nclusters) {
                const Tile2 t = decode2(p, tstart, mpairs, routed_total, tile);
                const SetDesc &sd = p.set[t.set];
                const int brow = EPI == EPI_SWIGLU ? t.n_idx * (BN / 2)
                                                   : t.n_idx * BN + (int)rank * (BN / 2);
                const CUtensorMap *bmap =
                    (EPI == EPI_SWIGLU && rank == 1) ? &p.tmB3[t.set] : &p.tmB[t.set];
                const bool gath = GATHER && t.set == 0;
                for (int kb = 0; kb < sd.k_blocks; ++kb) {
                    if (!wait_bar(empty_bar(stage), phase ^ 1u, ctl)) {
                        ok = false;
                        break;
                    }
                    int kcol = kb * BK * KSUB, ga = 0, gb = t.b_group;
                    if (sd.kbg > 0) {
                        ga = gb = kb / sd.kbg;
                        kcol = (kb % sd.kbg) * BK * KSUB;
                    }
                    if (leader)   // both CTAs' B boxes (and A boxes unless gathered)
                        mbar_expect_tx(full_bar(stage), (gath ? 2 : 4) * KSUB * HALF_BYTES);
                    const uint32_t fb = map_to_rank(full_bar(stage), 0);
                    for (int ks = 0; ks < KSUB; ++ks) {
                        const uint32_t a_dst = sA + (stage * KSUB + ks) * HALF_BYTES;
                        if (!gath)
                            tma_load_3d_pair(a_dst, &p.tmA[t.set], fb, kcol + ks * BK,
                                             t.m0 + (int)rank * 128, ga);
                        tma_load_3d_pair(sB + (stage * KSUB + ks) * HALF_BYTES, bmap, fb,
                                         kcol + ks * BK, brow, gb);
                    }
                    issued[stage] = 1;
                    last_phase[stage] = phase;
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the leader's full barriers count both CTAs' bytes: drain there
            if (leader)
                for (int s = 0; s < STAGES2; ++s)
                    if (issued[s])
                        wait_bar<GATHER>(full_bar(s), last_phase[s], ctl, false);
        }
    } else if (warp == 1) {
        // ================= MMA issuer (leader CTA only) =================
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, any = false;
            for (int tile = cluster_id; ok && tile < total; tile += nclusters) {
                const Tile2 t = decode2(p, tstart, mpairs, routed_total, tile);
                const SetDesc &sd = p.set[t.set];
                if (!wait_bar(tempty_bar(acc), acc_phase ^ 1u, ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tmem_d = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < sd.k_blocks; ++kb) {
                    // gathered rows: arrivals of the other CTA's threads too
                    if (!wait_bar<GATHER>(full_bar(stage), phase, ctl)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < KSUB; ++ks) {
                        const uint32_t a_base = sA + (stage * KSUB + ks) * HALF_BYTES,
                                       b_base = sB + (stage * KSUB + ks) * HALF_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_bf16_pair(tmem_d, sdesc_sw128(a_base + kk * 32),
                                          sdesc_sw128(b_base + kk * 32),
                                          (kb | ks | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(empty_bar(stage));
                    any = true;
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                mma_commit_pair(tfull_bar(acc));
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (any) {
                mma_commit_local2(drain_bar);
                wait_bar(drain_bar, 0, ctl, false);
            }
        }
    } else if (GATHER && warp >= 2 + EPI_WARPS) {
        // ================= gather warps: routed A rows from x (both CTAs) =====
        // Each CTA's four gather warps copy its 128 rows of the pair tile and
        // arrive on the leader's full barrier; a stage is signalled one issue
        // after its copies were issued (two stages' copies in flight).
        using G = GatherLanes<KSUB>;
        constexpr int D = STAGES2 - 2;
        const int gw = warp - (2 + EPI_WARPS);
        const int sub = lane / G::CPR;
        int stage = 0, seq = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = cluster_id; ok && tile < total; tile += nclusters) {
            const Tile2 t = decode2(p, tstart, mpairs, routed_total, tile);
            const SetDesc &sd = p.set[t.set];
            const bool gath = t.set == 0;   // shared-expert tiles: TMA boxes of x
            int tok[G::NI];
#pragma unroll
            for (int i = 0; i < G::NI; ++i)
                tok[i] = gath ? gather_row(p, t.m0 + (int)rank * 128 + 32 * gw + G::RPI * i + sub)
                              : 0;
            for (int kb = 0; kb < sd.k_blocks; ++kb) {
                int okw = lane == 0 ? (wait_bar(empty_bar(stage), phase ^ 1u, ctl) ? 1 : 0) : 1;
                if (!__shfl_sync(0xffffffffu, okw, 0)) {
                    ok = false;
                    break;
                }
                if (gath)
                    gather_stage<KSUB>(sA + stage * KSUB * HALF_BYTES, HALF_BYTES, p.xg, p.x_ld,
                                       kb * BK * KSUB, tok, gw, lane);
                cp_async_commit();
                if (seq >= D) {
                    cp_async_wait<D>();
                    gather_arrive<true>(full_bar((stage + STAGES2 - D) % STAGES2), lane);
                }
                ++seq;
                if (++stage == STAGES2) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        cp_async_wait<0>();   // the last stages' copies, then their arrivals
        for (int q = seq < D ? seq : D; q > 0; --q)
            gather_arrive<true>(full_bar((stage + STAGES2 - q) % STAGES2), lane);
    } else {
        // ================= epilogue (warps 2..9, both CTAs) =================
        const int q = warp & 3;
        const int ew = warp - 2;
        const int half = ew >> 2;
        const uint32_t stg = sStg + ew * STG_WARP;
        uint8_t *stg_ptr = smem + OFF2_STG + ew * STG_WARP;
        int acc = 0, nchunk = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster_id; tile < total; tile += nclusters) {
            const Tile2 t = decode2(p, tstart, mpairs, routed_total, tile);
            if (!wait_bar(tfull_bar(acc), acc_phase, ctl))
                break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const int c_col = t.n_idx * BN_OUT;
            const int c_end = (rank == 0 || t.second)
                                  ? min((half + 1) * (BN_OUT / 2), p.set[t.set].c_cols - c_col)
                                  : 0;
            const int row = t.m0 + (int)rank * 128 + q * 32;
            if (EPI == EPI_GATED && t.set == 0) {
                // gate and scatter: this lane's row goes to its assignment's row
                float gate;
                const int a = gated_slot(p, t.b_group, row + lane, &gate);
#pragma unroll 1
                for (int c = half * (BN_OUT / 2); c < c_end; c += CHUNK) {
                    float g[CHUNK];
                    tmem_ld_chunk(tbase + c, g);
                    if (a >= 0)
                        store_gated(p, a, gate, c_col + c, g);
                }
            } else {
#pragma unroll 1
            for (int c = half * (BN_OUT / 2); c < c_end; c += CHUNK, ++nchunk) {
                float g[CHUNK], u[CHUNK];
                uint32_t packed[CHUNK / 2];
                tmem_ld_chunk(tbase + c, g);
                if (EPI == EPI_SWIGLU) {
                    tmem_ld_chunk(tbase + BN / 2 + c, u);
                    epilogue_chunk<EPI>(g, u, packed);
                } else {
                    epilogue_chunk<EPI>(g, g, packed);
                }
                const int b = nchunk % STG_BUFS;   // this chunk's staging buffer
                if (lane == 0)
                    bulk_wait_read<STG_BUFS - 1>();
                __syncwarp();
                stage_row(stg_ptr + b * STG_BYTES, lane, packed);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&p.tmC[t.set], stg + b * STG_BYTES, c_col + c, row, t.c_group);
                    bulk_commit();
                }
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_remote(map_to_rank(tempty_bar(acc), 0));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0)
            bulk_wait_all();
        __syncwarp();
    }

    // ---- tear-down: both CTAs done with the pair's TMEM before it is freed ----
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------- host side

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

// 3-D bf16 tensor: dim0 (contiguous) x dim1 x dim2 with byte strides s1, s2.
bool make_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw)
{
    EncodeTiled enc = encoder();
    if (!enc)
        return false;
    cuuint64_t dims[3] = {d0, d1, d2 > 0 ? d2 : 1};
    cuuint64_t strides[2] = {s1, s2 > 0 ? s2 : s1 * (d1 > 0 ? d1 : 1)};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count() { return device_sms(); }

template <int EPI, bool GATHER = false>
cudaError_t launch_2sm(const Params &p, cudaStream_t s)
{
    auto kern = grouped_gemm_2sm_kernel<EPI, GATHER>;
    const int threads = THREADS + (GATHER ? 32 * GATHER_WARPS : 0);
    cudaError_t err = raise_smem_limit((const void *)kern, SMEM2_BYTES);
    if (err != cudaSuccess)
        return err;
    int clusters = 0;
    err = cached_active_clusters((const void *)kern, threads, SMEM2_BYTES, 2, &clusters);
    if (err != cudaSuccess)
        return err;
    if (clusters < 1)
        return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = SMEM2_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.numAttrs = 2;   // cluster pair and programmatic dependent launch
    err = cudaLaunchKernelEx(&cfg, kern, p);
    if (err != cudaSuccess)
        return err;
    return cudaGetLastError();
}

template <int EPI, bool GATHER = false>
cudaError_t launch(const Params &p, cudaStream_t s)
{
    auto kern = grouped_gemm_kernel<EPI, GATHER>;
    cudaError_t err = raise_smem_limit((const void *)kern, SMEM_BYTES);
    if (err != cudaSuccess)
        return err;
    return launch_pdl(kern, dim3(sm_count()), dim3(THREADS + (GATHER ? 32 * GATHER_WARPS : 0)),
                      SMEM_BYTES, s, p);
}

template <int EPI>
cudaError_t launch_1sm(const Params &p, cudaStream_t s)
{
    return p.gather ? launch<EPI, true>(p, s) : launch<EPI, false>(p, s);
}

// Diagnostic for the timeout path: one thread waits, with the same bounded
// wait the GEMM roles use, on an mbarrier that nothing ever arrives on.  The
// wait must give up after timeout_ns and record MOE_ERR_DEVICE_TIMEOUT; no
// copy or MMA is in flight, so the kernel simply returns.
__global__ void wait_probe_kernel(int32_t *status, unsigned long long timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const Ctl ctl{&abort_flag, status, timeout_ns};
    wait_bar(b, 0, ctl);
}

}  // namespace tc

cudaError_t launch_wait_probe(int32_t *status, unsigned long long timeout_ns, cudaStream_t s)
{
    tc::wait_probe_kernel<<<1, 1, 0, s>>>(status, timeout_ns);
    return cudaGetLastError();
}

cudaError_t launch_ffn_tcgen05(const moe_config &c, const void *x_perm, const int32_t *offsets,
                               const int32_t *src_slot, const void *W1, const void *W3,
                               const void *W2, const void *x, const void *Ws1, const void *Ws3,
                               const void *Ws2, void *Y_perm, void *Y_sh, void *H, void *H_sh,
                               int32_t *status, bool clear_status, cudaStream_t s,
                               const int32_t *kept, const float *gates, void *slot_out)
{
    using namespace tc;
    const uint64_t R = (uint64_t)perm_rows(c), d = c.d, F = c.d_ff, E = c.E;
    const uint64_t T = c.T, S = c.n_shared, Fs = c.d_ff_shared;
    const bool swiglu = c.act == MOE_ACT_SWIGLU;
    // SM-pair tiles (256 rows) when experts average at least 512 rows; single-SM
    // tiles (128 rows) for small segments, where a 256-row tile would mostly
    // compute padding.
    const bool pair = (int64_t)c.T * c.k >= (int64_t)512 * c.E;
    // B rows one TMA box brings into one CTA: half the 256-column accumulator
    // for SwiGLU (W1 and W3 halves) and for every SM-pair tile (one half per
    // CTA), the whole 256 otherwise.  The box must match what the kernel
    // expects, or the stage's byte count is wrong.
    const int bn_b = (swiglu || pair) ? BN / 2 : BN;
    const int bn2_b = pair ? BN / 2 : BN;
    const int bn_out = swiglu ? BN / 2 : BN;
    const CUtensorMapSwizzle SW128 = CU_TENSOR_MAP_SWIZZLE_128B;
    // epilogue store boxes: CHUNK columns x 32 rows, swizzled as stage_row writes them
    const CUtensorMapSwizzle SWC = SWZ_BITS == 1 ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : (SWZ_BITS == 2 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_128B);
    const bool shared = S > 0 && T > 0;

    // ---- GEMM1: H = act(x_perm W1^T [, x_perm W3^T]); H_sh likewise from x ----
    Params p1;
    memset(&p1, 0, sizeof p1);
    p1.E = c.E;
    p1.offsets = offsets;
    p1.status = status;
    p1.clear_status = clear_status ? 1 : 0;
    p1.timeout_ns = 2000000000ull;
    p1.nsets = shared ? 2 : 1;
    bool ok = true;
    if (!x_perm) {
        // dispatch fused in: tile rows gathered from x by the gather warps
        p1.gather = 1;
        p1.src_slot = src_slot;
        p1.n_rows = (int)R;
        p1.k = c.k;
        p1.xg = static_cast<const __nv_bfloat16 *>(x);
        p1.x_ld = (int)d;
    } else {
        ok &= make_map(&p1.tmA[0], x_perm, d, R, 1, d * 2, 0, BK, BM, SW128);
    }
    ok &= make_map(&p1.tmB[0], W1, d, F, E, d * 2, F * d * 2, BK, bn_b, SW128);
    if (swiglu)
        ok &= make_map(&p1.tmB3[0], W3, d, F, E, d * 2, F * d * 2, BK, bn_b, SW128);
    ok &= make_map(&p1.tmC[0], H, F, R, 1, F * 2, 0, CHUNK, 32, SWC);
    const int KB = pair ? KSUB * BK : BK;   // K per stage: the pair kernel takes 128

    p1.set[0] = SetDesc{1, 0, (int)ceil_div(F, bn_out), 1, (int)ceil_div(d, KB), 0, (int)F};
    if (shared) {
        ok &= make_map(&p1.tmA[1], x, d, T, 1, d * 2, 0, BK, BM, SW128);
        ok &= make_map(&p1.tmB[1], Ws1, d, Fs, S, d * 2, Fs * d * 2, BK, bn_b, SW128);
        if (swiglu)
            ok &= make_map(&p1.tmB3[1], Ws3, d, Fs, S, d * 2, Fs * d * 2, BK, bn_b, SW128);
        // H_sh [S][T][Fs]: shared expert s owns one [T][Fs] slab
        ok &= make_map(&p1.tmC[1], H_sh, Fs, T, S, Fs * 2, T * Fs * 2, CHUNK, 32, SWC);
        p1.set[1] = SetDesc{0, (int)T, (int)ceil_div(Fs, bn_out), (int)S, (int)ceil_div(d, KB), 0,
                            (int)Fs};
    }
    if (!ok)
        return cudaErrorInvalidValue;
    cudaError_t err;
    if (pair)
        err = p1.gather ? (swiglu ? launch_2sm<EPI_SWIGLU, true>(p1, s)
                                  : launch_2sm<EPI_GELU, true>(p1, s))
                        : (swiglu ? launch_2sm<EPI_SWIGLU>(p1, s) : launch_2sm<EPI_GELU>(p1, s));
    else
        err = swiglu ? launch_1sm<EPI_SWIGLU>(p1, s)
                     : launch_1sm<EPI_GELU>(p1, s);
    if (err != cudaSuccess)
        return err;

    // ---- GEMM2: Y_perm = H W2^T; Y_sh = sum_s H_sh[:, s] Ws2[s]^T ----
    Params p2;
    memset(&p2, 0, sizeof p2);
    p2.E = c.E;
    p2.offsets = offsets;
    p2.status = status;
    p2.timeout_ns = 2000000000ull;
    p2.nsets = shared ? 2 : 1;
    ok = true;
    ok &= make_map(&p2.tmA[0], H, F, R, 1, F * 2, 0, BK, BM, SW128);
    ok &= make_map(&p2.tmB[0], W2, F, d, E, F * 2, d * F * 2, BK, bn2_b, SW128);
    if (slot_out) {
        // the combine's gate fused: row r of expert e -> row src_slot[r] of slot_out
        p2.src_slot = src_slot;
        p2.n_rows = (int)R;
        p2.k = c.k;
        p2.kept = kept;
        p2.gates = gates;
        p2.slot_out = static_cast<__nv_bfloat16 *>(slot_out);
        p2.slot_ld = (int)d;
    } else {
        ok &= make_map(&p2.tmC[0], Y_perm, d, R, 1, d * 2, 0, CHUNK, 32, SWC);
    }
    p2.set[0] = SetDesc{1, 0, (int)ceil_div(d, BN), 1, (int)ceil_div(F, KB), 0, (int)d};
    if (shared) {
        ok &= make_map(&p2.tmA[1], H_sh, Fs, T, S, Fs * 2, T * Fs * 2, BK, BM, SW128);
        ok &= make_map(&p2.tmB[1], Ws2, Fs, d, S, Fs * 2, d * Fs * 2, BK, bn2_b, SW128);
        ok &= make_map(&p2.tmC[1], Y_sh, d, T, 1, d * 2, 0, CHUNK, 32, SWC);
        const int kbg = (int)ceil_div(Fs, KB);
        p2.set[1] = SetDesc{0, (int)T, (int)ceil_div(d, BN), 1, kbg * (int)S, kbg, (int)d};
    }
    if (!ok)
        return cudaErrorInvalidValue;
    if (slot_out)
        return pair ? launch_2sm<EPI_GATED>(p2, s) : launch_1sm<EPI_GATED>(p2, s);
    return pair ? launch_2sm<EPI_NONE>(p2, s) : launch_1sm<EPI_NONE>(p2, s);
}

}  // namespace moe
