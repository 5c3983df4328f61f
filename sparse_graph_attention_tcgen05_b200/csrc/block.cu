// block.cu -- the block around the layer: Z = LayerNorm(X + Y Wo).
//
// Method page "Gated Local-Global Graph Attention", Implementation notes, item 2: the
// layer returns LayerNorm(X + Wo(g*L + (1-g)*G)), i.e. the output projection Wo
// ([H*r, d], no bias), the residual and a LayerNorm over the d features (per-feature gain
// and bias, population variance).
//
// One CTA per 128-row tile (192 threads): warp 4 issues TMA loads of the Y tile (K-major
// A operand; fp32 Y goes through a tf32 hi/lo split copy) and of the packed Wo^T (K-major
// B operand) through an mbarrier ring, warp 5 issues tcgen05.mma into a d-column fp32
// TMEM accumulator (two N halves when d > 256), and warps 0-3 (one thread per row) run
// the epilogue straight from TMEM: u = acc + x, mean, centred variance, then
// (u - mean) * rsqrt(var + eps) * gamma + beta, stored as Z.  Y Wo never goes to HBM.
#include <algorithm>

#include "glga_internal.cuh"

namespace glga {
namespace {

constexpr int kBM = 128;
constexpr int kRowBytes = 128;
constexpr int kMaxStages = 4;
constexpr int kThreads = 192;
constexpr int kProdWarp = 4;
constexpr int kMmaWarp = 5;

template <typename T>
__device__ __forceinline__ float ld1(const T *p);
template <>
__device__ __forceinline__ float ld1<float>(const float *p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ T st1(float v);
template <>
__device__ __forceinline__ float st1<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 st1<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Wt[c][k] = Wo[k][c] (c < d, k < Kp; zero for k >= D): the K-major B operand, as tf32
// hi/lo planes for SPLIT = 3.
template <int SPLIT, typename T>
__global__ void pack_wo_kernel(const T *__restrict__ Wo, int D, int d, int Kp, T *__restrict__ Wt) {
    const int64_t total = static_cast<int64_t>(d) * Kp;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(idx / Kp), k = static_cast<int>(idx % Kp);
        const float v = k < D ? ld1<T>(Wo + static_cast<int64_t>(k) * d + c) : 0.f;
        if (SPLIT == 3) {
            const float hi = to_tf32(v);
            Wt[idx] = st1<T>(hi);
            Wt[total + idx] = st1<T>(to_tf32(v - hi));
        } else {
            Wt[idx] = st1<T>(v);
        }
    }
}

// Y copied to [planes][N][Kp], zero for k >= D; for SPLIT = 3 as tf32 hi/lo planes.
template <int SPLIT, typename T>
__global__ void prep_y_kernel(const T *__restrict__ Y, int64_t N, int D, int Kp, T *__restrict__ Yp) {
    const int64_t total = N * Kp;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = idx / Kp;
        const int k = static_cast<int>(idx % Kp);
        const float v = k < D ? ld1<T>(Y + i * D + k) : 0.f;
        if (SPLIT == 3) {
            const float hi = to_tf32(v);
            Yp[idx] = st1<T>(hi);
            Yp[total + idx] = st1<T>(to_tf32(v - hi));
        } else {
            Yp[idx] = st1<T>(v);
        }
    }
}

struct BlockParams {
    int64_t M;
    int32_t d, nk, stages, halves;
    uint32_t a_bytes, b_bytes, stage_bytes;   // b_bytes: one plane of the d-row B box(es)
    uint32_t tmem_cols;
    const void *X;
    const void *gamma, *beta;
    void *Z;
    float ln_eps;
    unsigned *flag;
};

template <int SPLIT, typename T>
__global__ void __launch_bounds__(kThreads, 1) block_kernel(const __grid_constant__ CUtensorMap tmA0,
                                                             const __grid_constant__ CUtensorMap tmA1,
                                                             const __grid_constant__ CUtensorMap tmB0,
                                                             const __grid_constant__ CUtensorMap tmB1,
                                                             BlockParams p) {
    constexpr int kPlanes = SPLIT == 3 ? 2 : 1;
    constexpr int kPairs = SPLIT == 3 ? 3 : 1;
    constexpr uint32_t kFmt = SPLIT == 3 ? 2u : 1u;
    constexpr int KT = kRowBytes / static_cast<int>(sizeof(T));
    constexpr int VE = 16 / static_cast<int>(sizeof(T));

    extern __shared__ uint8_t dsmem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_base_sh;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t m0 = static_cast<int32_t>(blockIdx.x) * kBM;
    const int dh = p.d / p.halves;                  // columns per MMA (<= 256)

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&done_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_base_sh, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kProdWarp) {
        if (lane == 0) {
            RingPos rp;
            int issued = 0;
            bool ok = true;
            for (int kb = 0; kb < p.nk; ++kb, rp.next(p.stages)) {
                const int s = rp.slot;
                if (kb >= p.stages && !mbar_wait_bounded(&empty_bar[s], rp.phase ^ 1u)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
                mbar_arrive_expect_tx(&full_bar[s], kPlanes * (p.a_bytes + p.b_bytes));
                tma_load_2d(st, &tmA0, &full_bar[s], kb * KT, m0);
                if (kPlanes == 2) tma_load_2d(st + p.a_bytes, &tmA1, &full_bar[s], kb * KT, m0);
                uint8_t *bst = st + kPlanes * p.a_bytes;
                for (int hh = 0; hh < p.halves; ++hh) {
                    const uint32_t off = static_cast<uint32_t>(hh * dh) * kRowBytes;
                    tma_load_2d(bst + off, &tmB0, &full_bar[s], kb * KT, hh * dh);
                    if (kPlanes == 2) tma_load_2d(bst + p.b_bytes + off, &tmB1, &full_bar[s], kb * KT, hh * dh);
                }
                ++issued;
            }
            if (!ok) {
                atomicOr(p.flag, kDevErrTimeout);
                for (int k = std::max(0, issued - p.stages); k < issued; ++k)
                    mbar_wait_bounded(&full_bar[k % p.stages], static_cast<uint32_t>(k / p.stages) & 1u);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t idesc = instr_desc(kBM, dh, kFmt, false, false);
            RingPos rp;
            bool ok = true;
            for (int kb = 0; kb < p.nk; ++kb, rp.next(p.stages)) {
                const int s = rp.slot;
                if (!mbar_wait_bounded(&full_bar[s], rp.phase)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + static_cast<size_t>(s) * p.stage_bytes);
                const uint32_t b_addr = a_addr + kPlanes * p.a_bytes;
                for (int hh = 0; hh < p.halves; ++hh) {
                    const uint32_t boff = static_cast<uint32_t>(hh * dh) * kRowBytes;
#pragma unroll
                    for (int k = 0; k < kRowBytes / 32; ++k) {
#pragma unroll
                        for (int pr = 0; pr < kPairs; ++pr) {
                            const uint32_t ap = (pr == 2) ? 1u : 0u;
                            const uint32_t bp = (pr == 1) ? 1u : 0u;
                            const uint64_t ad = smem_desc(a_addr + ap * p.a_bytes + k * 32, 16, 1024, 2);
                            const uint64_t bd = smem_desc(b_addr + bp * p.b_bytes + boff + k * 32, 16, 1024, 2);
                            const uint32_t acc = (kb | k | pr) != 0;
                            if (SPLIT == 3)
                                umma_tf32(tmem + static_cast<uint32_t>(hh * dh), ad, bd, idesc, acc);
                            else
                                umma_bf16(tmem + static_cast<uint32_t>(hh * dh), ad, bd, idesc, acc);
                        }
                    }
                }
                umma_commit(&empty_bar[s]);
            }
            if (!ok) atomicOr(p.flag, kDevErrTimeout);
            umma_commit(&done_bar);          // also retires every MMA issued so far
        }
    } else {
        // ---------------- epilogue: one thread per row, straight from TMEM ----------------
        // warp-uniform, since the TMEM loads below are warp-collective
        const bool done = __all_sync(0xffffffffu, mbar_wait_bounded(&done_bar, 0));
        tc_fence_after();
        const int rt = warp * 32 + lane;
        const int64_t row = static_cast<int64_t>(m0) + rt;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        if (!done) {
            if (lane == 0) atomicOr(p.flag, kDevErrTimeout);
        } else {
            const T *X = static_cast<const T *>(p.X) + row * p.d;
            T *Z = static_cast<T *>(p.Z) + row * p.d;
            const T *G = static_cast<const T *>(p.gamma);
            const T *B = static_cast<const T *>(p.beta);
            const bool live = row < p.M;
            float sum = 0.f, sq = 0.f, mean = 0.f;
            // pass 0: mean of u = acc + x; pass 1: centred variance; pass 2: normalise, store
            for (int pass = 0; pass < 3; ++pass) {
                const float rstd = pass == 2 ? rsqrtf(sq / static_cast<float>(p.d) + p.ln_eps) : 0.f;
                for (int c0 = 0; c0 < p.d; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_base + static_cast<uint32_t>(c0), v);
                    tmem_ld_wait();
                    if (!live) continue;
                    float u[32];
#pragma unroll
                    for (int q = 0; q < 32 / VE; ++q) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(X + c0 + q * VE);
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int e = 0; e < VE; ++e) {
                            float xv;
                            if (sizeof(T) == 4)
                                xv = __uint_as_float(w[e]);
                            else
                                xv = __uint_as_float(e & 1 ? (w[e / 2] & 0xffff0000u) : (w[e / 2] << 16));
                            u[q * VE + e] = __uint_as_float(v[q * VE + e]) + xv;
                        }
                    }
                    if (pass == 0) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) sum += u[j];
                    } else if (pass == 1) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) sq = fmaf(u[j] - mean, u[j] - mean, sq);
                    } else {
#pragma unroll
                        for (int q = 0; q < 32 / VE; ++q) {
                            uint32_t w[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                if (sizeof(T) == 4) {
                                    const int j = q * VE + k;
                                    w[k] = __float_as_uint((u[j] - mean) * rstd * ld1<T>(G + c0 + j) + ld1<T>(B + c0 + j));
                                } else {
                                    const int j = q * VE + 2 * k;
                                    const float z0 = (u[j] - mean) * rstd * ld1<T>(G + c0 + j) + ld1<T>(B + c0 + j);
                                    const float z1 = (u[j + 1] - mean) * rstd * ld1<T>(G + c0 + j + 1) + ld1<T>(B + c0 + j + 1);
                                    __nv_bfloat162 h = __floats2bfloat162_rn(z0, z1);
                                    w[k] = *reinterpret_cast<uint32_t *>(&h);
                                }
                            }
                            *reinterpret_cast<uint4 *>(Z + c0 + q * VE) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                if (pass == 0) mean = sum / static_cast<float>(p.d);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

}  // namespace

bool block_supported(const Ctx *c) {
    return c->d % 32 == 0 && c->d <= 512;
}

glga_status block_setup(Ctx *c) {
    if (!block_supported(c)) return GLGA_OK;         // glga_block_output reports it
    const int kt = kRowBytes / c->elem;
    c->blk_kp = static_cast<int32_t>(ceil_div(c->D, kt) * kt);
    const int planes = c->split == 3 ? 2 : 1;
    glga_status st = dev_alloc(c, &c->Wo_t, static_cast<size_t>(planes) * c->d * c->blk_kp * c->elem);
    // Y is read in place only as bf16 rows of whole 64-column boxes; otherwise a padded
    // (and for fp32, tf32-split) copy is the A operand
    c->blk_y_direct = c->split == 1 && c->D % kt == 0;
    if (st == GLGA_OK && !c->blk_y_direct && c->N > 0)
        st = dev_alloc(c, &c->Yp, static_cast<size_t>(planes) * c->N * c->blk_kp * c->elem);
    return st;
}

glga_status block_run(Ctx *c, const void *Y, const void *X, const void *Wo, const void *gamma,
                      const void *beta, float ln_eps, void *Z, cudaStream_t s) {
    if (!block_supported(c)) {
        set_error("glga_block_output: needs d a multiple of 32 and d <= 512 (d = %d)", c->d);
        return GLGA_ERR_UNSUPPORTED;
    }
    const int kt = kRowBytes / c->elem;
    const int planes = c->split == 3 ? 2 : 1;
    const int64_t wt_total = static_cast<int64_t>(c->d) * c->blk_kp;
    const unsigned wb = static_cast<unsigned>(std::min<int64_t>(ceil_div(wt_total, 256), 2048));
    if (c->split == 3)
        pack_wo_kernel<3, float><<<wb, 256, 0, s>>>(static_cast<const float *>(Wo), c->D, c->d, c->blk_kp,
                                                   static_cast<float *>(c->Wo_t));
    else
        pack_wo_kernel<1, __nv_bfloat16><<<wb, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(Wo), c->D, c->d,
                                                           c->blk_kp, static_cast<__nv_bfloat16 *>(c->Wo_t));
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    if (c->N == 0) return GLGA_OK;
    const CUtensorMapDataType dt =
        c->io == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap a0, a1, b0, b1;
    glga_status st;
    if (!c->blk_y_direct) {
        const int64_t total = c->N * c->blk_kp;
        const unsigned yb = static_cast<unsigned>(std::min<int64_t>(ceil_div(total, 256), 8192));
        if (c->split == 3)
            prep_y_kernel<3, float><<<yb, 256, 0, s>>>(static_cast<const float *>(Y), c->N, c->D, c->blk_kp,
                                                      static_cast<float *>(c->Yp));
        else
            prep_y_kernel<1, __nv_bfloat16><<<yb, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(Y), c->N, c->D,
                                                              c->blk_kp, static_cast<__nv_bfloat16 *>(c->Yp));
        GLGA_CUDA(cudaGetLastError());
        c->launches += 1;
        const uint64_t rb = static_cast<uint64_t>(c->blk_kp) * c->elem;
        st = encode_tmap_2d(&a0, dt, c->Yp, c->blk_kp, c->N, rb, kt, kBM);
        if (st == GLGA_OK && planes == 2)
            st = encode_tmap_2d(&a1, dt, static_cast<uint8_t *>(c->Yp) + static_cast<size_t>(total) * c->elem,
                                c->blk_kp, c->N, rb, kt, kBM);
        else
            a1 = a0;
    } else {
        // bf16 rows of whole 64-column boxes: Y itself is the A operand
        st = encode_tmap_2d(&a0, dt, Y, c->D, c->N, static_cast<uint64_t>(c->D) * c->elem, kt, kBM);
        a1 = a0;
    }
    if (st != GLGA_OK) return st;
    const int halves = c->d > 256 ? 2 : 1;
    const int dh = c->d / halves;
    const uint64_t wrb = static_cast<uint64_t>(c->blk_kp) * c->elem;
    st = encode_tmap_2d(&b0, dt, c->Wo_t, c->blk_kp, c->d, wrb, kt, dh);
    if (st == GLGA_OK && planes == 2)
        st = encode_tmap_2d(&b1, dt, static_cast<uint8_t *>(c->Wo_t) + static_cast<size_t>(c->d) * wrb,
                            c->blk_kp, c->d, wrb, kt, dh);
    else
        b1 = b0;
    if (st != GLGA_OK) return st;

    BlockParams p;
    p.M = c->N;
    p.d = c->d;
    p.nk = c->blk_kp / kt;
    p.halves = halves;
    p.a_bytes = kBM * kRowBytes;
    p.b_bytes = static_cast<uint32_t>(c->d) * kRowBytes;
    p.stage_bytes = planes * (p.a_bytes + p.b_bytes);
    p.stages = std::max(1, std::min(std::min(kMaxStages, p.nk), static_cast<int>((200u * 1024u) / p.stage_bytes)));
    uint32_t tc = 32;
    while (tc < static_cast<uint32_t>(c->d)) tc <<= 1;
    p.tmem_cols = tc;
    p.X = X;
    p.gamma = gamma;
    p.beta = beta;
    p.Z = Z;
    p.ln_eps = ln_eps;
    p.flag = c->dev_flag;
    const size_t smem = static_cast<size_t>(p.stages) * p.stage_bytes + 1024;
    const unsigned grid = static_cast<unsigned>(ceil_div(c->N, kBM));
    if (c->split == 3) {
        GLGA_CUDA(cudaFuncSetAttribute(block_kernel<3, float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
        block_kernel<3, float><<<grid, kThreads, smem, s>>>(a0, a1, b0, b1, p);
    } else {
        GLGA_CUDA(cudaFuncSetAttribute(block_kernel<1, __nv_bfloat16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
        block_kernel<1, __nv_bfloat16><<<grid, kThreads, smem, s>>>(a0, a1, b0, b1, p);
    }
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    return GLGA_OK;
}

}  // namespace glga
