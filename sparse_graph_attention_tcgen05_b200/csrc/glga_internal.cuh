// glga_internal.cuh -- shared declarations of libglga's CUDA sources (not installed).
//
// Device helpers wrap the sm_100a instructions the kernels use: mbarrier waits with an
// upper bound, TMA 2-D tiled loads (no cluster multicast anywhere in this library),
// tcgen05 TMEM allocation, MMA issue/commit and TMEM loads.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "glga.h"

namespace glga {

// ---------------------------------------------------------------------------------------
// error reporting
// ---------------------------------------------------------------------------------------
void set_error(const char *fmt, ...);
glga_status cuda_fail(cudaError_t e, const char *what);
glga_status cuda_ok(cudaError_t e);   // GLGA_OK, or cuda_fail's status for an error

#define GLGA_CUDA(call)                                                    \
    do {                                                                   \
        cudaError_t _e = (call);                                           \
        if (_e != cudaSuccess) return ::glga::cuda_fail(_e, #call);        \
    } while (0)

// Device-side error flag bits (ctx->dev_flag).
enum : unsigned {
    kDevErrTimeout = 1u,   // a bounded mbarrier wait gave up
    kDevErrBounds = 2u,    // a device-side check found an out-of-range index
};

// Validation flag bits for topology checks.
enum : unsigned {
    kGraphBadRowPtr0 = 1u,
    kGraphBadRowPtrEnd = 2u,
    kGraphNotMonotone = 4u,
    kGraphColOutOfRange = 8u,
};

// ---------------------------------------------------------------------------------------
// context
// ---------------------------------------------------------------------------------------
struct TensorMap2D {
    CUtensorMap map;
    bool valid = false;
};

enum Stage { kStagePrep = 0, kStageGemm, kStageStats, kStageLocal, kStageReadout, kStageEnd, kNumEvents };

struct Ctx {
    int device = 0;
    int num_sms = 148;
    int64_t N = 0, E = 0;
    int32_t d = 0, H = 0, r = 0, D = 0;
    glga_dtype io = GLGA_F32;
    int elem = 4;                 // bytes per io element
    glga_options opts{};

    // topology (owned copies)
    int32_t *row_ptr = nullptr, *col_idx = nullptr;
    int64_t nb[4] = {0, 0, 0, 0};   // bucket sizes and chunk count
    int32_t *warp_rows = nullptr, *cta_rows = nullptr, *split_rows = nullptr;
    int32_t *chunk_row = nullptr, *chunk_begin = nullptr;
    int32_t *task_start = nullptr;      // bucket-0 warp tasks: [n_tasks + 1] list positions
    int64_t n_tasks = 0;
    unsigned *chunk_ticket = nullptr;   // one counter per chunk slot (first chunk of a row)
    float *chunk_part = nullptr;        // per chunk: m[H], l[H], acc[D]

    // projection
    int32_t dp = 0;               // padded input width (multiple of the K tile)
    int32_t Dp = 0;               // padded GEMM width: 3*D + gate column + padding
    int32_t BN = 0, bn_last = 0, n_tiles = 0, stages = 0, tmem_cols = 0;
    bool gemm_tma_epi = false;    // Q/K/V stored through shared memory + TMA
    int32_t gemm_sbufs = 2;       // staging buffers of that epilogue (1 or 2)
    TensorMap2D tmKVs, tmQs;      // K|V and Q store maps (64-column x 32-row boxes)
    int split = 1;                // 1: bf16 MMA; 3: 3-term tf32 split (fp32 io)
    bool x_direct = false;        // A operand read straight from the caller's X
    void *Wt = nullptr;           // [planes][Dp][dp]
    void *Xp = nullptr;           // [planes][N][dp] (prepared A operand when !x_direct)
    TensorMap2D tmB[2], tmA[2];

    // row sharding: the context's N target rows are rows row0 .. row0+N-1 of n_src nodes;
    // its CSR columns and the K/V buffer index all n_src nodes (n_src = N, row0 = 0 when
    // the context holds the whole graph)
    int64_t n_src = 0, row0 = 0;
    bool sharded = false;
    bool kv_external = false;     // KV is the caller's buffer (not freed here)

    // intermediates
    void *Q = nullptr;            // io [N, D]
    void *KV = nullptr;           // io [n_src, 2D]  (k_j | v_j)
    void *kv_own = nullptr;       // KV + row0 rows: the rows this context projects
    float *t = nullptr;           // [N] gate logits
    float *Spart = nullptr;       // [P][H][r][r+1] partial sums of the row ranges
    float *Sz = nullptr;          // S [n_seg][H][r][r] followed by z [n_seg][H][r]
    int32_t stats_parts = 0;
    int64_t stats_rows_per_part = 0;
    int32_t *part_ptr = nullptr;  // row ranges of the statistics kernel [stats_parts + 1]
    TensorMap2D tmK, tmV;         // K and V halves of KV for the statistics kernel

    // readout GEMM (phi(Q) x [S | z] per head group, blended with L)
    int32_t ro_groups = 0, ro_hg = 0, ro_kp = 0, ro_bn = 0;
    bool ro_tma_epi = false;      // L in / Y out through TMA boxes (group width fits boxes)
    void *Bro = nullptr;          // [planes][groups][ro_bn][ro_kp] K-major, io type
    TensorMap2D tmBro[2], tmQ, tmL;
    void *L = nullptr;            // io [N, D] local-branch output

    // segments (a batch of graphs as contiguous node ranges, each with its own S and z)
    int64_t n_seg = 1;
    std::vector<int64_t> seg_ptr;     // host copy [n_seg + 1]
    int32_t *seg_part_ptr = nullptr;  // statistics ranges of each segment [n_seg + 1]
    bool stats_direct = false;        // every non-empty segment one range: no reduction pass
    bool stats_fused = false;         // S | z partials from the projection epilogue (one per CTA)
    int32_t stats_fused_parts = 0;    // ... the projection's grid size
    int32_t *part_seg = nullptr;      // ... and the segment of each range
    int32_t *tile_seg = nullptr;      // segment of each 128-row readout tile's first row
    int32_t *fix_row = nullptr;       // rows whose segment differs from their tile's
    int32_t *fix_seg = nullptr;       //   ... and that segment
    int64_t n_fix = 0;

    // block around the layer (Z = LayerNorm(X + Y Wo))
    int32_t blk_kp = 0;           // K = H*r padded to the K tile
    bool blk_y_direct = false;    // Y read in place as the A operand
    void *Wo_t = nullptr;         // [planes][d][blk_kp] K-major Wo^T
    void *Yp = nullptr;           // [planes][N][blk_kp] padded / split Y when not direct

    // backward pass workspaces (opts.backward)
    int32_t *t_row_ptr = nullptr, *t_col = nullptr;   // transposed CSR: rows by source
    void *bw_dL = nullptr;                            // [N, D] in the io type
    float *bw_dnum = nullptr;                         // [N, D + 16]
    float *bw_dden = nullptr, *bw_dg = nullptr, *bw_lse = nullptr, *bw_Dd = nullptr;   // [N, H]
    float *bw_dZ = nullptr;                           // [N, 3D + 1]: dQ | dK | dV | dt
    float *bw_dsz_part = nullptr, *bw_dSz = nullptr;  // dS | dz partials and sum
    float *bw_ST = nullptr, *bw_dST = nullptr;        // per-head transposes of S and dS
    float *bw_Wall = nullptr;                         // [d][dz_ld] fp32 [W_Q | W_K | W_V | w_g]
    float *bw_dSc = nullptr;                          // dS [H][R][R] then dz [H][R]
    int2 *bw_q_chunks = nullptr, *bw_k_chunks = nullptr;  // heavy rows' edge chunks {row, first}
    int32_t *bw_q_cptr = nullptr, *bw_k_cptr = nullptr;   // chunk offsets per heavy row
    int64_t bw_nq_chunks = 0, bw_nk_chunks = 0;
    float *bw_q_part = nullptr, *bw_kv_part = nullptr;  // chunk shares
    cudaStream_t bw_side = nullptr;                   // second stream of the backward (source side)
    float *bw_dwtc_part = nullptr;                    // [P][d][3D] tensor-core dW range partials
    int64_t bw_dwtc_rpp = 0;                          // ... rows per range (multiple of 64)
    int32_t bw_dwtc_parts = 0;                        // ... ranges
    float *bw_dW3 = nullptr;                          // [d][3D] their sum
    __nv_bfloat16 *bw_dZb = nullptr;                  // [N][3D] dQ | dK | dV in bf16 (global parts, then the finals)
    int32_t *bw_perm = nullptr;                       // [E] forward CSR entry -> its transposed CSR position
    uint32_t *bw_pds = nullptr;                       // [E][H] (p_ij, ds_ij) as bf16 pairs, transposed order
    cudaEvent_t bw_ev_q = nullptr;                    // the target side has written bw_pds
    cudaEvent_t bw_ev_fork = nullptr, bw_ev_join = nullptr;
    float *bw_dbg_part = nullptr;                     // [wparts] row-range sums of dt
    float *bw_dw_part = nullptr;                      // [wparts][d][3D + 1]
    int32_t *bw_q_rows = nullptr, *bw_k_rows = nullptr;   // light rows, then heavy rows
    int64_t bw_nq_light = 0, bw_nq_heavy = 0, bw_nk_light = 0, bw_nk_heavy = 0;
    int64_t bw_dz_ld = 0;
    int32_t bw_parts = 0, bw_wparts = 0;
    int32_t bw_dsz_parts = 0;                         // dS | dz row ranges and their rows
    int64_t bw_dsz_rpp = 0;
    int32_t bw_fx_parts = 0;                          // thread blocks of the one-pass dX / dW kernel (0: off)

    unsigned *dev_flag = nullptr;
    int64_t bytes = 0;
    int64_t alloc_calls = 0;      // device allocations made by create (debug_fail_alloc)
    int64_t launches = 0;         // kernels launched by glga_forward so far

    bool timing = false;
    cudaEvent_t ev[kNumEvents] = {};
    bool ev_recorded = false;
};

// One thread waits on an mbarrier nothing arrives on, with the bounded wait of the
// tensor-core kernels, and sets kDevErrTimeout in *flag after limit_ns (test entry points).
glga_status launch_bounded_wait_probe(unsigned *flag, uint64_t limit_ns, cudaStream_t s);

struct Ctx;
// Records stage event `stage` of the context on s (an event record node of the graph when
// s is being captured, so graph replays record it too).
cudaError_t record_stage(Ctx *c, int stage, cudaStream_t s);

// allocation helper that tracks bytes
glga_status dev_alloc(Ctx *c, void **p, size_t bytes);
// Counts one device allocation of create; GLGA_ERR_OOM when it is the one
// opts.debug_fail_alloc names (test hook of the clean-up path).
glga_status debug_alloc_hook(Ctx *c);

// topology.cu
glga_status validate_csr(Ctx *c, cudaStream_t s);
glga_status build_buckets(Ctx *c, cudaStream_t s);
glga_status exclusive_scan_i32(const int32_t *in, int32_t *out, int64_t n, int32_t *total_dev,
                               cudaStream_t s, void *tmp, size_t tmp_bytes);
size_t scan_tmp_bytes(int64_t n);

// projection.cu
glga_status projection_setup(Ctx *c);
glga_status projection_run(Ctx *c, const void *X, const void *WQ, const void *WK,
                           const void *WV, const void *wg, cudaStream_t s, bool time_prep);
// C [M][ldc] (float32, columns < ncols written) = A [M][K] * B [ncols][K]^T on the tcgen05
// tensor cores: A and B row-major with leading dimensions lda, ldb (elements, 16-byte
// multiples), element type t (GLGA_BF16: kind::f16; GLGA_F32: kind::tf32, one term).
// Stream-ordered; the persistent projection kernel with a float32 epilogue.
glga_status gemm_nt_f32out(Ctx *c, glga_dtype t, const void *A, int64_t M, int64_t lda, const void *B,
                           int64_t ncols, int64_t ldb, int64_t K, float *C, int64_t ldc, cudaStream_t s);

// global_stats.cu
glga_status stats_setup(Ctx *c);
glga_status stats_run(Ctx *c, cudaStream_t s);
// row-sharded forward: this context's partial S | z (flat [H][r][r+1]) ...
glga_status stats_run_partial(Ctx *c, float *own, cudaStream_t s);
// ... and the final reduction of all ranks' partials ([P][H][r][r+1], in rank order)
glga_status stats_finish(Ctx *c, const float *partials, int P, cudaStream_t s);

// local.cu
glga_status local_setup(Ctx *c);
glga_status local_run(Ctx *c, cudaStream_t s);

// block.cu
bool block_supported(const Ctx *c);
glga_status block_setup(Ctx *c);
glga_status block_run(Ctx *c, const void *Y, const void *X, const void *Wo, const void *gamma,
                      const void *beta, float ln_eps, void *Z, cudaStream_t s);

// backward.cu
glga_status backward_setup(Ctx *c, cudaStream_t s);
glga_status backward_run(Ctx *c, const void *X, const void *WQ, const void *WK, const void *WV,
                         const void *wg, float b_g, float eps, const void *dY, float *dX, float *dWQ,
                         float *dWK, float *dWV, float *dwg, float *db_g, cudaStream_t s);

// readout.cu
glga_status readout_setup(Ctx *c);
glga_status readout_run(Ctx *c, float b_g, float eps, void *Y, cudaStream_t s);

// tensor maps (driver entry point resolved at run time; no libcuda link dependency)
glga_status encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base,
                           uint64_t inner, uint64_t outer, uint64_t row_bytes,
                           uint32_t box_inner, uint32_t box_outer,
                           CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

// ---------------------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but a thread whose phase is still open may be suspended for up to
// `hint_ns` nanoseconds (or until the phase completes) instead of the hardware's
// default window, so a waiting warp takes no issue slots while it waits.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Suspend-time hint of one poll (ns): the thread may sleep up to this long unless the
// phase completes first.
#ifndef GLGA_MBAR_SUSPEND_NS
#define GLGA_MBAR_SUSPEND_NS 1000000u
#endif

// Waits for the phase with the given parity to complete.  Each poll may suspend the
// thread for up to GLGA_MBAR_SUSPEND_NS (1 ms); gives up after about `limit_ns`
// nanoseconds of wall time or 2^26 polls, whichever comes first, and returns false; the
// caller records the timeout and winds down.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns = 1000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1; it < (1u << 26); ++it) {
        if (mbar_try_wait_suspend(bar, parity, GLGA_MBAR_SUSPEND_NS)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// Position in a ring of n mbarrier-guarded slots: the slot and the parity of the
// current pass over the ring, advanced without divisions.
struct RingPos {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n) {
        if (++slot == n) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

// Walks the tiles start, start + step, start + 2 step, ... of a row-major grid with
// `cols` tiles per row, keeping (row, col) by increments instead of divisions.
struct TileWalk {
    int32_t row, col, step_row, step_col, cols;
    __device__ __forceinline__ TileWalk(int32_t start, int32_t step, int32_t cols_)
        : row(start / cols_), col(start % cols_), step_row(step / cols_), step_col(step % cols_),
          cols(cols_) {}
    __device__ __forceinline__ void next() {
        col += step_col;
        row += step_row;
        if (col >= cols) {
            col -= cols;
            ++row;
        }
    }
};

// 2-D tiled TMA load global -> shared, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// 2-D tiled TMA store shared -> global (bulk async group).  Elements outside the tensor
// are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t x,
                                             int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until at most the most recently committed bulk-store group is still reading.
__device__ __forceinline__ void bulk_wait_group_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later async-proxy
// (TMA, tcgen05) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also returns the OR of `pred` over the participating threads.
__device__ __forceinline__ bool named_barrier_or(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, p;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "barrier.cta.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// --- tcgen05 ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start address, leading
// and stride byte offsets (16-byte units), version 1, swizzle mode in bits 61..63
// (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swz) {
    uint64_t dsc = 0;
    dsc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    dsc |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    dsc |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    dsc |= static_cast<uint64_t>(1u) << 46;
    dsc |= static_cast<uint64_t>(swz & 7u) << 61;
    return dsc;
}

// Instruction descriptor for kind::f16 / kind::tf32 with an f32 accumulator.
// fmt: 1 = bf16, 2 = tf32.  a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, uint32_t fmt, bool a_mn,
                                                  bool b_mn) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((static_cast<uint32_t>(N) >> 3) << 17) |
           ((static_cast<uint32_t>(M) >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrives on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// TMEM -> registers: 32 lanes x 32 consecutive 32-bit columns (one row per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr)
        : "memory");
}
// TMEM -> registers: 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
// TMEM -> registers: 32 lanes x N (1, 2 or 4) consecutive 32-bit columns.
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&v)[N]) {
    static_assert(N == 1 || N == 2 || N == 4, "tmem_ld_n: 1, 2 or 4 columns");
    if constexpr (N == 1) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
                     : "=r"(v[0]) : "r"(taddr) : "memory");
    } else if constexpr (N == 2) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                     : "=r"(v[0]), "=r"(v[1]) : "r"(taddr) : "memory");
    } else {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(taddr) : "memory");
    }
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// phi of two bf16 values in one word, on packed bf16x2 arithmetic:
//   phi(x) = elu(x) + 1 = 2^(min(x, 0) log2 e) + max(x, 0),
// which is x + 1 for x > 0 (2^0 = 1, then one rounding of x + 1, as in float32 followed
// by the bf16 rounding of the operand) and e^x for x <= 0.  log2 e enters as a bf16 pair
// hi + lo (sum within 5e-6 of it, so e^x carries no systematic scale error) and the
// exponent is rounded to bf16 once: at most |x| 2^-9 relative in e^x, an absolute error
// of at most 2^-9 / e beside the bf16 rounding of the result (checked over every bf16
// x <= 0: worst total 2.6e-3 against 2.0e-3 for float32 e^x rounded to bf16).
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t x) {
    uint32_t y;
    asm("{\n\t.reg .b32 neg, pos, t;\n\t"
        "min.bf16x2 neg, %1, %2;\n\t"
        "max.bf16x2 pos, %1, %2;\n\t"
        "mul.rn.bf16x2 t, neg, %4;\n\t"
        "fma.rn.bf16x2 t, neg, %3, t;\n\t"
        "ex2.approx.ftz.bf16x2 t, t;\n\t"
        "add.rn.bf16x2 %0, t, pos;\n\t}"
        : "=r"(y) : "r"(x), "r"(0u), "r"(0x3FB93FB9u), "r"(0xBB2CBB2Cu));   // 0, log2 e = hi + lo
    return y;
}

// d = a * b + c for the bf16 half AH of a and BH of b (1 = the high half): fma.rn.f32.bf16,
// the product exact, one f32 rounding (the same value as float32 fmaf of the widened halves).
template <int AH, int BH>
__device__ __forceinline__ float fma_bf16h(uint32_t a, uint32_t b, float c) {
    float d;
    if constexpr (AH == 0 && BH == 0)
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a0, b0, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else if constexpr (AH == 1 && BH == 1)
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a1, b1, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else if constexpr (AH == 0 && BH == 1)
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a0, b1, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a1, b0, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}

// acc + the dot product of the 2W bf16 values of a and b (W words each), element order.
template <int W>
__device__ __forceinline__ float dot_bf16w(const uint32_t *a, const uint32_t *b, float acc) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
        acc = fma_bf16h<0, 0>(a[w], b[w], acc);
        acc = fma_bf16h<1, 1>(a[w], b[w], acc);
    }
    return acc;
}

// acc[2w + e] += s x[w].half(e) for the bf16 s in the low half of s2.
template <int W>
__device__ __forceinline__ void axpy_bf16w(uint32_t s2, const uint32_t *x, float *acc) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
        acc[2 * w] = fma_bf16h<0, 0>(s2, x[w], acc[2 * w]);
        acc[2 * w + 1] = fma_bf16h<0, 1>(s2, x[w], acc[2 * w + 1]);
    }
}

// x rounded to bf16 (nearest even) in both halves of a word.
__device__ __forceinline__ uint32_t bf16_splat(float x) {
    uint32_t w;
    asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(w) : "f"(x));
    return w;
}

// 16-byte asynchronous copy global -> shared (L2 only), its group commit and the wait for
// all but the N most recent groups of this thread.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Round-to-nearest (ties away) conversion of an f32 to tf32, kept in an f32 container.
__device__ __forceinline__ float to_tf32(float x) {
    uint32_t u;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(u) : "f"(x));
    return __uint_as_float(u);
}

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace glga
