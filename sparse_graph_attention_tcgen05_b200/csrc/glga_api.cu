// glga_api.cu -- the C ABI of libglga (declared in include/glga.h).
//
// Argument checking, context lifetime, workspace allocation, stage ordering on the
// caller's stream and error reporting.  All arithmetic happens in the kernels of
// projection.cu, global_stats.cu, local.cu and topology.cu.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>

#include <nvtx3/nvToolsExt.h>

#include "glga_internal.cuh"

namespace glga {

namespace {
thread_local char g_msg[512] = "no error";

// One thread waits on an mbarrier that nothing arrives on, with the bounded wait of the
// tensor-core kernels; it gives up after limit_ns and raises the timeout flag.
__global__ void bounded_wait_probe_kernel(unsigned *flag, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(flag, kDevErrTimeout);
}
}  // namespace

glga_status launch_bounded_wait_probe(unsigned *flag, uint64_t limit_ns, cudaStream_t s) {
    bounded_wait_probe_kernel<<<1, 32, 0, s>>>(flag, limit_ns);
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
}

glga_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? GLGA_OK : cuda_fail(e, "CUDA call"); }

cudaError_t record_stage(Ctx *c, int stage, cudaStream_t s) {
    // while the stream is being captured into a CUDA graph the event becomes an event
    // record node, so every replay of the graph records it
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return e;
    if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(c->ev[stage], s, cudaEventRecordExternal);
    return cudaEventRecord(c->ev[stage], s);
}

glga_status cuda_fail(cudaError_t e, const char *what) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    if (e == cudaErrorMemoryAllocation) return GLGA_ERR_OOM;
    return GLGA_ERR_CUDA;
}

glga_status debug_alloc_hook(Ctx *c) {
    ++c->alloc_calls;
    if (c->opts.debug_fail_alloc > 0 && c->alloc_calls == c->opts.debug_fail_alloc) {
        set_error("simulated failure of device allocation %lld (debug_fail_alloc)",
                  static_cast<long long>(c->alloc_calls));
        return GLGA_ERR_OOM;
    }
    return GLGA_OK;
}

glga_status dev_alloc(Ctx *c, void **p, size_t bytes) {
    if (bytes == 0) bytes = 16;
    *p = nullptr;
    const glga_status hook = debug_alloc_hook(c);
    if (hook != GLGA_OK) return hook;
    cudaError_t e = cudaMalloc(p, bytes);
    if (e != cudaSuccess) {
        *p = nullptr;
        return cuda_fail(e, "cudaMalloc");
    }
    c->bytes += static_cast<int64_t>(bytes);
    return GLGA_OK;
}

// Releases every device resource held by the context (the host object is freed by the
// caller).
static void release_ctx(Ctx *c) {
    if (!c) return;
    if (c->kv_external) c->KV = nullptr;   // the caller's buffer
    void *ptrs[] = {c->row_ptr, c->col_idx, c->warp_rows, c->cta_rows, c->split_rows,
                    c->chunk_row, c->chunk_begin, c->chunk_ticket, c->chunk_part, c->Wt,
                    c->Xp, c->Q, c->KV, c->t, c->Spart, c->Sz, c->Bro, c->L, c->task_start,
                    c->part_ptr, c->seg_part_ptr, c->tile_seg, c->fix_row, c->fix_seg,
                    c->Wo_t, c->Yp, c->t_row_ptr, c->t_col, c->bw_dL, c->bw_dnum, c->bw_dden,
                    c->bw_dg, c->bw_lse, c->bw_Dd, c->bw_dZ, c->bw_dsz_part, c->bw_dSz,
                    c->bw_dw_part, c->bw_q_rows, c->bw_k_rows, c->bw_ST, c->bw_dST, c->bw_Wall, c->bw_dbg_part,
                    c->bw_dSc, c->bw_q_chunks, c->bw_k_chunks, c->bw_q_cptr, c->bw_k_cptr,
                    c->bw_q_part, c->bw_kv_part, c->bw_dwtc_part, c->bw_dW3, c->bw_dZb, c->bw_perm, c->bw_pds,
                    c->part_seg, c->dev_flag};
    for (void *p : ptrs)
        if (p) cudaFree(p);
    for (auto &e : c->ev)
        if (e) cudaEventDestroy(e);
    if (c->bw_ev_fork) cudaEventDestroy(c->bw_ev_fork);
    if (c->bw_ev_join) cudaEventDestroy(c->bw_ev_join);
    if (c->bw_ev_q) cudaEventDestroy(c->bw_ev_q);
    if (c->bw_side) cudaStreamDestroy(c->bw_side);
}

}  // namespace glga

using namespace glga;

struct glga_ctx {
    Ctx c;
};

namespace {
glga_status create_impl(glga_ctx **out, int64_t N, int32_t d, int32_t H, int32_t r, glga_dtype io,
                        const int32_t *row_ptr, const int32_t *col_idx, int64_t E,
                        const int64_t *seg_ptr, int64_t n_seg, const glga_options *opts,
                        void *stream, int64_t n_src, int64_t row0, void *kv_ext);
}  // namespace

extern "C" {

const char *glga_status_string(glga_status s) {
    switch (s) {
        case GLGA_OK: return "ok";
        case GLGA_ERR_INVALID_ARG: return "invalid argument";
        case GLGA_ERR_BAD_GRAPH: return "invalid graph";
        case GLGA_ERR_UNSUPPORTED: return "unsupported shape";
        case GLGA_ERR_OOM: return "out of device memory";
        case GLGA_ERR_CUDA: return "CUDA error";
        case GLGA_ERR_TIMEOUT: return "device-side wait timed out";
        case GLGA_ERR_DEVICE: return "device-side check failed";
    }
    return "unknown status";
}

const char *glga_last_error_message(void) { return g_msg; }

glga_status glga_default_options(glga_options *opts) {
    if (!opts) {
        set_error("glga_default_options: null pointer");
        return GLGA_ERR_INVALID_ARG;
    }
    opts->warp_max_degree = 256;
    opts->chunk_edges = 2048;
    opts->debug_checks = 0;
    opts->debug_fail_alloc = 0;
    opts->backward = 0;
    opts->fuse_stats = 0;
    return GLGA_OK;
}

glga_status glga_create(glga_ctx **out, int64_t N, int32_t d, int32_t H, int32_t r,
                        glga_dtype io, const int32_t *row_ptr, const int32_t *col_idx, int64_t E,
                        const glga_options *opts, void *stream) {
    const int64_t seg[2] = {0, N};
    return glga_create_segmented(out, N, d, H, r, io, row_ptr, col_idx, E, seg, 1, opts, stream);
}

glga_status glga_create_segmented(glga_ctx **out, int64_t N, int32_t d, int32_t H, int32_t r,
                                  glga_dtype io, const int32_t *row_ptr, const int32_t *col_idx,
                                  int64_t E, const int64_t *seg_ptr, int64_t n_seg,
                                  const glga_options *opts, void *stream) {
    return create_impl(out, N, d, H, r, io, row_ptr, col_idx, E, seg_ptr, n_seg, opts, stream, N, 0,
                       nullptr);
}

glga_status glga_create_sharded(glga_ctx **out, int64_t n_nodes, int64_t row_begin, int64_t row_end,
                                int32_t d, int32_t H, int32_t r, glga_dtype io,
                                const int32_t *row_ptr, const int32_t *col_idx, int64_t E,
                                void *kv, const glga_options *opts, void *stream) {
    if (n_nodes < 0 || n_nodes > 2147483646LL || row_begin < 0 || row_end < row_begin ||
        row_end > n_nodes || !kv || (reinterpret_cast<uintptr_t>(kv) & 15u)) {
        if (out) *out = nullptr;
        set_error("glga_create_sharded: need 0 <= row_begin <= row_end <= n_nodes < 2^31-1 and a "
                  "16-byte aligned K/V buffer");
        return GLGA_ERR_INVALID_ARG;
    }
    const int64_t n_own = row_end - row_begin;
    const int64_t seg[2] = {0, n_own};
    return create_impl(out, n_own, d, H, r, io, row_ptr, col_idx, E, seg, 1, opts, stream, n_nodes,
                       row_begin, kv);
}
}  // extern "C"

namespace {
glga_status create_impl(glga_ctx **out, int64_t N, int32_t d, int32_t H, int32_t r, glga_dtype io,
                        const int32_t *row_ptr, const int32_t *col_idx, int64_t E,
                        const int64_t *seg_ptr, int64_t n_seg, const glga_options *opts,
                        void *stream, int64_t n_src, int64_t row0, void *kv_ext) {
    if (!out) {
        set_error("glga_create: out is NULL");
        return GLGA_ERR_INVALID_ARG;
    }
    *out = nullptr;
    if (N < 0 || N > 2147483646LL || E < 0 || E > 2147483647LL || d < 1 || H < 1) {
        set_error("glga_create: need 0 <= N < 2^31-1, 0 <= E < 2^31, d >= 1, H >= 1");
        return GLGA_ERR_INVALID_ARG;
    }
    if (io != GLGA_F32 && io != GLGA_BF16) {
        set_error("glga_create: io must be GLGA_F32 or GLGA_BF16");
        return GLGA_ERR_INVALID_ARG;
    }
    if (!(r == 8 || r == 16 || r == 32 || r == 64 || r == 128)) {
        set_error("glga_create: r must be one of 8, 16, 32, 64, 128 (got %d)", r);
        return GLGA_ERR_UNSUPPORTED;
    }
    const int elem = io == GLGA_F32 ? 4 : 2;
    const int64_t D = static_cast<int64_t>(H) * r;
    if (D * elem > 2048) {
        set_error("glga_create: H*r*sizeof(io) = %lld bytes exceeds 2048",
                  static_cast<long long>(D * elem));
        return GLGA_ERR_UNSUPPORTED;
    }
    if (!row_ptr || (E > 0 && !col_idx)) {
        set_error("glga_create: null CSR pointer");
        return GLGA_ERR_INVALID_ARG;
    }
    glga_options o;
    glga_default_options(&o);
    if (opts) o = *opts;
    if (o.warp_max_degree < 0 || o.chunk_edges < 1 || o.warp_max_degree > o.chunk_edges) {
        set_error("glga_create: need 0 <= warp_max_degree <= chunk_edges, chunk_edges >= 1");
        return GLGA_ERR_INVALID_ARG;
    }
    if (o.debug_fail_alloc < 0) {
        set_error("glga_create: debug_fail_alloc must be >= 0");
        return GLGA_ERR_INVALID_ARG;
    }
    if (!seg_ptr || n_seg < 1 || n_seg > 2147483647LL || seg_ptr[0] != 0 || seg_ptr[n_seg] != N) {
        set_error("glga_create: seg_ptr must hold n_seg + 1 >= 2 offsets from 0 to N");
        return GLGA_ERR_INVALID_ARG;
    }
    for (int64_t k = 0; k < n_seg; ++k)
        if (seg_ptr[k + 1] < seg_ptr[k]) {
            set_error("glga_create: seg_ptr decreases at segment %lld", static_cast<long long>(k));
            return GLGA_ERR_INVALID_ARG;
        }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    glga_ctx *h = new (std::nothrow) glga_ctx();
    if (!h) {
        set_error("glga_create: host allocation failed");
        return GLGA_ERR_OOM;
    }
    Ctx *c = &h->c;
    c->N = N;
    c->E = E;
    c->d = d;
    c->H = H;
    c->r = r;
    c->D = static_cast<int32_t>(D);
    c->io = io;
    c->elem = elem;
    c->opts = o;
    c->n_seg = n_seg;
    c->seg_ptr.assign(seg_ptr, seg_ptr + n_seg + 1);
    c->n_src = n_src;
    c->row0 = row0;
    c->sharded = kv_ext != nullptr;
    glga_status st = GLGA_OK;
    cudaError_t e = cudaGetDevice(&c->device);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
    int cc_major = 0, cc_minor = 0;
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, c->device);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&cc_minor, cudaDevAttrComputeCapabilityMinor, c->device);
    if (e != cudaSuccess) st = cuda_fail(e, "device query");
    if (st == GLGA_OK && !(cc_major == 10 && cc_minor == 0)) {
        set_error("glga_create: needs an sm_100 device (B200); found sm_%d%d", cc_major, cc_minor);
        st = GLGA_ERR_UNSUPPORTED;
    }
#define TRY(x) \
    if (st == GLGA_OK) st = (x)
    TRY(dev_alloc(c, reinterpret_cast<void **>(&c->dev_flag), 64));
    TRY(dev_alloc(c, reinterpret_cast<void **>(&c->row_ptr), (N + 1) * sizeof(int32_t)));
    TRY(dev_alloc(c, reinterpret_cast<void **>(&c->col_idx), (E > 0 ? E : 1) * sizeof(int32_t)));
    if (st == GLGA_OK) {
        e = cudaMemcpyAsync(c->row_ptr, row_ptr, (N + 1) * sizeof(int32_t),
                            cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess && E > 0)
            e = cudaMemcpyAsync(c->col_idx, col_idx, E * sizeof(int32_t),
                                cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) st = cuda_fail(e, "CSR copy");
    }
    TRY(validate_csr(c, s));
    TRY(build_buckets(c, s));
    TRY(dev_alloc(c, &c->Q, static_cast<size_t>(N) * D * elem));
    if (kv_ext) {
        c->KV = kv_ext;
        c->kv_external = true;
    } else {
        TRY(dev_alloc(c, &c->KV, static_cast<size_t>(n_src) * 2 * D * elem));
    }
    if (st == GLGA_OK) c->kv_own = static_cast<uint8_t *>(c->KV) + static_cast<size_t>(row0) * 2 * D * elem;
    TRY(dev_alloc(c, reinterpret_cast<void **>(&c->t), static_cast<size_t>(N) * sizeof(float)));
    TRY(projection_setup(c));
    TRY(readout_setup(c));
    TRY(stats_setup(c));
    TRY(local_setup(c));
    TRY(block_setup(c));
    TRY(backward_setup(c, s));
    if (st == GLGA_OK) {
        e = cudaMemsetAsync(c->dev_flag, 0, 64, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) st = cuda_fail(e, "create sync");
    }
#undef TRY
    if (st != GLGA_OK) {
        cudaStreamSynchronize(s);
        release_ctx(c);
        delete h;
        return st;
    }
    *out = h;
    return GLGA_OK;
}
}  // namespace

extern "C" {

glga_status glga_forward(glga_ctx *h, const void *X, const void *W_Q, const void *W_K,
                         const void *W_V, const void *w_g, float b_g, float eps, void *Y,
                         void *stream) {
    if (!h) {
        set_error("glga_forward: ctx is NULL");
        return GLGA_ERR_INVALID_ARG;
    }
    Ctx *c = &h->c;
    if (!W_Q || !W_K || !W_V || !w_g || (c->N > 0 && (!X || !Y))) {
        set_error("glga_forward: null pointer argument");
        return GLGA_ERR_INVALID_ARG;
    }
    if (!(eps > 0.f) || !std::isfinite(eps) || !std::isfinite(b_g)) {
        set_error("glga_forward: eps must be finite and > 0, b_g finite");
        return GLGA_ERR_INVALID_ARG;
    }
    const uintptr_t align_or = reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Y);
    if (align_or & 15u) {
        set_error("glga_forward: X and Y must be 16-byte aligned");
        return GLGA_ERR_INVALID_ARG;
    }
    if (c->sharded) {
        set_error("glga_forward: a row-sharded context runs glga_forward_begin / glga_forward_end");
        return GLGA_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (c->timing) {
        for (auto &ev : c->ev)
            if (!ev) GLGA_CUDA(cudaEventCreate(&ev));
        GLGA_CUDA(record_stage(c, kStagePrep, s));
    }
    // NVTX ranges mark the host-side enqueue of each stage (visible to profilers that
    // attach an NVTX tool; no-ops otherwise)
    struct Range {
        explicit Range(const char *name) { nvtxRangePushA(name); }
        ~Range() { nvtxRangePop(); }
    } whole("glga_forward");
    glga_status st;
    {
        Range r("glga.projection");
        st = projection_run(c, X, W_Q, W_K, W_V, w_g, s, c->timing);
    }
    if (st != GLGA_OK) return st;
    if (c->timing) GLGA_CUDA(record_stage(c, kStageStats, s));
    {
        Range r("glga.global_stats");
        st = stats_run(c, s);
    }
    if (st != GLGA_OK) return st;
    if (c->timing) GLGA_CUDA(record_stage(c, kStageLocal, s));
    {
        Range r("glga.local");
        st = local_run(c, s);
    }
    if (st != GLGA_OK) return st;
    if (c->timing) GLGA_CUDA(record_stage(c, kStageReadout, s));
    {
        Range r("glga.readout");
        st = readout_run(c, b_g, eps, Y, s);
    }
    if (st != GLGA_OK) return st;
    if (c->timing) {
        GLGA_CUDA(record_stage(c, kStageEnd, s));
        c->ev_recorded = true;
    }
    return GLGA_OK;
}

glga_status glga_forward_begin(glga_ctx *h, const void *X, const void *W_Q, const void *W_K,
                               const void *W_V, const void *w_g, float *own_partial, void *stream) {
    if (!h || !h->c.sharded) {
        set_error("glga_forward_begin: needs a context from glga_create_sharded");
        return GLGA_ERR_INVALID_ARG;
    }
    Ctx *c = &h->c;
    if (!W_Q || !W_K || !W_V || !w_g || !own_partial || (c->N > 0 && !X) ||
        (reinterpret_cast<uintptr_t>(X) & 15u)) {
        set_error("glga_forward_begin: null or misaligned pointer argument");
        return GLGA_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (c->timing) {
        for (auto &ev : c->ev)
            if (!ev) GLGA_CUDA(cudaEventCreate(&ev));
        GLGA_CUDA(record_stage(c, kStagePrep, s));
    }
    nvtxRangePushA("glga_forward_begin");
    glga_status st = projection_run(c, X, W_Q, W_K, W_V, w_g, s, c->timing);
    if (st == GLGA_OK && c->timing) st = cuda_ok(record_stage(c, kStageStats, s));
    if (st == GLGA_OK) st = stats_run_partial(c, own_partial, s);
    nvtxRangePop();
    return st;
}

glga_status glga_forward_end(glga_ctx *h, const float *partials, int32_t P, float b_g, float eps,
                             void *Y, void *stream) {
    if (!h || !h->c.sharded) {
        set_error("glga_forward_end: needs a context from glga_create_sharded");
        return GLGA_ERR_INVALID_ARG;
    }
    Ctx *c = &h->c;
    if (!partials || P < 1 || (c->N > 0 && !Y) || (reinterpret_cast<uintptr_t>(Y) & 15u)) {
        set_error("glga_forward_end: need partials of P >= 1 ranks and a 16-byte aligned Y");
        return GLGA_ERR_INVALID_ARG;
    }
    if (!(eps > 0.f) || !std::isfinite(eps) || !std::isfinite(b_g)) {
        set_error("glga_forward_end: eps must be finite and > 0, b_g finite");
        return GLGA_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (c->timing && !c->ev[kStagePrep]) {
        set_error("glga_forward_end: timing is on but glga_forward_begin ran without it");
        return GLGA_ERR_INVALID_ARG;
    }
    nvtxRangePushA("glga_forward_end");
    glga_status st = stats_finish(c, partials, P, s);
    if (st == GLGA_OK && c->timing) st = cuda_ok(record_stage(c, kStageLocal, s));
    if (st == GLGA_OK) st = local_run(c, s);
    if (st == GLGA_OK && c->timing) st = cuda_ok(record_stage(c, kStageReadout, s));
    if (st == GLGA_OK) st = readout_run(c, b_g, eps, Y, s);
    if (st == GLGA_OK && c->timing) {
        st = cuda_ok(record_stage(c, kStageEnd, s));
        c->ev_recorded = st == GLGA_OK;
    }
    nvtxRangePop();
    return st;
}

glga_status glga_backward(glga_ctx *h, const void *X, const void *W_Q, const void *W_K,
                          const void *W_V, const void *w_g, float b_g, float eps, const void *dY,
                          float *dX, float *dW_Q, float *dW_K, float *dW_V, float *dw_g, float *db_g,
                          void *stream) {
    if (!h || !h->c.opts.backward) {
        set_error("glga_backward: needs a context created with glga_options.backward = 1");
        return GLGA_ERR_INVALID_ARG;
    }
    Ctx *c = &h->c;
    if (!W_Q || !W_K || !W_V || !w_g || !dW_Q || !dW_K || !dW_V || !dw_g || !db_g ||
        (c->N > 0 && (!X || !dY || !dX))) {
        set_error("glga_backward: null pointer argument");
        return GLGA_ERR_INVALID_ARG;
    }
    if (!(eps > 0.f) || !std::isfinite(eps) || !std::isfinite(b_g)) {
        set_error("glga_backward: eps must be finite and > 0, b_g finite");
        return GLGA_ERR_INVALID_ARG;
    }
    nvtxRangePushA("glga_backward");
    const glga_status st = backward_run(c, X, W_Q, W_K, W_V, w_g, b_g, eps, dY, dX, dW_Q, dW_K, dW_V,
                                        dw_g, db_g, static_cast<cudaStream_t>(stream));
    nvtxRangePop();
    return st;
}

glga_status glga_block_output(glga_ctx *h, const void *Y, const void *X, const void *Wo,
                              const void *gamma, const void *beta, float ln_eps, void *Z,
                              void *stream) {
    if (!h) {
        set_error("glga_block_output: ctx is NULL");
        return GLGA_ERR_INVALID_ARG;
    }
    Ctx *c = &h->c;
    if (!Wo || !gamma || !beta || (c->N > 0 && (!Y || !X || !Z))) {
        set_error("glga_block_output: null pointer argument");
        return GLGA_ERR_INVALID_ARG;
    }
    const uintptr_t a = reinterpret_cast<uintptr_t>(Y) | reinterpret_cast<uintptr_t>(X) |
                        reinterpret_cast<uintptr_t>(Z);
    if ((a & 15u) || !(ln_eps >= 0.f) || !std::isfinite(ln_eps)) {
        set_error("glga_block_output: Y, X, Z must be 16-byte aligned and ln_eps finite, >= 0");
        return GLGA_ERR_INVALID_ARG;
    }
    nvtxRangePushA("glga_block_output");
    const glga_status st = block_run(c, Y, X, Wo, gamma, beta, ln_eps, Z, static_cast<cudaStream_t>(stream));
    nvtxRangePop();
    return st;
}

glga_status glga_destroy(glga_ctx *h) {
    if (!h) return GLGA_OK;
    cudaDeviceSynchronize();
    release_ctx(&h->c);
    delete h;
    return GLGA_OK;
}

glga_status glga_bucket_counts(const glga_ctx *h, int64_t *counts) {
    if (!h || !counts) {
        set_error("glga_bucket_counts: null pointer");
        return GLGA_ERR_INVALID_ARG;
    }
    for (int k = 0; k < 4; ++k) counts[k] = h->c.nb[k];
    return GLGA_OK;
}

glga_status glga_get_buckets(const glga_ctx *h, int32_t *warp_rows, int32_t *cta_rows,
                             int32_t *split_rows, int32_t *chunk_row, int32_t *chunk_begin,
                             void *stream) {
    if (!h) {
        set_error("glga_get_buckets: ctx is NULL");
        return GLGA_ERR_INVALID_ARG;
    }
    const Ctx *c = &h->c;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    struct {
        int32_t *dst;
        const int32_t *src;
        int64_t n;
    } items[] = {{warp_rows, c->warp_rows, c->nb[0]}, {cta_rows, c->cta_rows, c->nb[1]},
                 {split_rows, c->split_rows, c->nb[2]}, {chunk_row, c->chunk_row, c->nb[3]},
                 {chunk_begin, c->chunk_begin, c->nb[3]}};
    for (auto &it : items)
        if (it.dst && it.n > 0)
            GLGA_CUDA(cudaMemcpyAsync(it.dst, it.src, it.n * sizeof(int32_t),
                                      cudaMemcpyDeviceToDevice, s));
    return GLGA_OK;
}

glga_status glga_get_intermediates(const glga_ctx *h, void *Q, void *K, void *V, float *t,
                                   float *S, float *z, void *L, void *stream) {
    if (!h) {
        set_error("glga_get_intermediates: ctx is NULL");
        return GLGA_ERR_INVALID_ARG;
    }
    const Ctx *c = &h->c;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t row = static_cast<size_t>(c->D) * c->elem;
    if (c->N > 0) {
        if (Q) GLGA_CUDA(cudaMemcpyAsync(Q, c->Q, c->N * row, cudaMemcpyDeviceToDevice, s));
        if (K)
            GLGA_CUDA(cudaMemcpy2DAsync(K, row, c->kv_own, 2 * row, row, c->N,
                                        cudaMemcpyDeviceToDevice, s));
        if (V)
            GLGA_CUDA(cudaMemcpy2DAsync(V, row, static_cast<const uint8_t *>(c->kv_own) + row, 2 * row,
                                        row, c->N, cudaMemcpyDeviceToDevice, s));
        if (t) GLGA_CUDA(cudaMemcpyAsync(t, c->t, c->N * sizeof(float), cudaMemcpyDeviceToDevice, s));
        if (L) GLGA_CUDA(cudaMemcpyAsync(L, c->L, c->N * row, cudaMemcpyDeviceToDevice, s));
    }
    // Sz holds S [n_seg][H][r][r] followed by z [n_seg][H][r]
    const size_t s_floats = static_cast<size_t>(c->n_seg) * c->H * c->r * c->r;
    if (S) GLGA_CUDA(cudaMemcpyAsync(S, c->Sz, s_floats * sizeof(float), cudaMemcpyDeviceToDevice, s));
    if (z)
        GLGA_CUDA(cudaMemcpyAsync(z, c->Sz + s_floats,
                                  static_cast<size_t>(c->n_seg) * c->H * c->r * sizeof(float),
                                  cudaMemcpyDeviceToDevice, s));
    return GLGA_OK;
}

glga_status glga_set_timing(glga_ctx *h, int enable) {
    if (!h) {
        set_error("glga_set_timing: ctx is NULL");
        return GLGA_ERR_INVALID_ARG;
    }
    h->c.timing = enable != 0;
    h->c.ev_recorded = false;
    return GLGA_OK;
}

glga_status glga_stage_times(glga_ctx *h, float *ms, int32_t n_max, int32_t *n_written) {
    if (!h || !ms || !n_written) {
        set_error("glga_stage_times: null pointer");
        return GLGA_ERR_INVALID_ARG;
    }
    Ctx *c = &h->c;
    *n_written = 0;
    if (!c->timing || !c->ev_recorded) {
        set_error("glga_stage_times: timing disabled or no forward recorded");
        return GLGA_ERR_INVALID_ARG;
    }
    GLGA_CUDA(cudaEventSynchronize(c->ev[kStageEnd]));
    float v[6];
    GLGA_CUDA(cudaEventElapsedTime(&v[0], c->ev[kStagePrep], c->ev[kStageGemm]));
    GLGA_CUDA(cudaEventElapsedTime(&v[1], c->ev[kStageGemm], c->ev[kStageStats]));
    GLGA_CUDA(cudaEventElapsedTime(&v[2], c->ev[kStageStats], c->ev[kStageLocal]));
    GLGA_CUDA(cudaEventElapsedTime(&v[3], c->ev[kStageLocal], c->ev[kStageReadout]));
    GLGA_CUDA(cudaEventElapsedTime(&v[4], c->ev[kStageReadout], c->ev[kStageEnd]));
    GLGA_CUDA(cudaEventElapsedTime(&v[5], c->ev[kStagePrep], c->ev[kStageEnd]));
    const int n = n_max < 6 ? n_max : 6;
    for (int i = 0; i < n; ++i) ms[i] = v[i];
    *n_written = n;
    return GLGA_OK;
}

glga_status glga_kernel_launches(const glga_ctx *h, int64_t *n) {
    if (!h || !n) {
        set_error("glga_kernel_launches: null pointer");
        return GLGA_ERR_INVALID_ARG;
    }
    *n = h->c.launches;
    return GLGA_OK;
}

glga_status glga_workspace_bytes(const glga_ctx *h, int64_t *bytes) {
    if (!h || !bytes) {
        set_error("glga_workspace_bytes: null pointer");
        return GLGA_ERR_INVALID_ARG;
    }
    *bytes = h->c.bytes;
    return GLGA_OK;
}

glga_status glga_debug_bounded_wait(glga_ctx *h, int64_t limit_ns, void *stream) {
    if (!h || limit_ns < 1000 || limit_ns > 10000000000LL) {
        set_error("glga_debug_bounded_wait: need a context and 1e3 <= limit_ns <= 1e10");
        return GLGA_ERR_INVALID_ARG;
    }
    return launch_bounded_wait_probe(h->c.dev_flag, static_cast<uint64_t>(limit_ns),
                                     static_cast<cudaStream_t>(stream));
}

glga_status glga_debug_set_col_idx(glga_ctx *h, int64_t e, int32_t value, void *stream) {
    if (!h || !h->c.opts.debug_checks || e < 0 || e >= h->c.E) {
        set_error("glga_debug_set_col_idx: needs a context made with debug_checks and 0 <= e < E");
        return GLGA_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the value is copied from this function's stack: wait for the copy before returning
    GLGA_CUDA(cudaMemcpyAsync(h->c.col_idx + e, &value, sizeof(int32_t), cudaMemcpyHostToDevice, s));
    GLGA_CUDA(cudaStreamSynchronize(s));
    return GLGA_OK;
}

glga_status glga_last_device_error(glga_ctx *h, void *stream) {
    if (!h) {
        set_error("glga_last_device_error: ctx is NULL");
        return GLGA_ERR_INVALID_ARG;
    }
    Ctx *c = &h->c;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned f = 0;
    GLGA_CUDA(cudaMemcpyAsync(&f, c->dev_flag, sizeof(unsigned), cudaMemcpyDeviceToHost, s));
    GLGA_CUDA(cudaStreamSynchronize(s));
    GLGA_CUDA(cudaMemsetAsync(c->dev_flag, 0, sizeof(unsigned), s));
    if (f & kDevErrTimeout) {
        set_error("a bounded device-side wait timed out");
        return GLGA_ERR_TIMEOUT;
    }
    if (f) {
        set_error("device-side check failed (flags 0x%x)", f);
        return GLGA_ERR_DEVICE;
    }
    return GLGA_OK;
}

}  // extern "C"
