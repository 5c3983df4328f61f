// readout.cu -- global readout fused with the gate blend, on the tcgen05 tensor cores.
//
// Method page "Gated Local-Global Graph Attention", Key formulas:
//   G_i = phi(q_i)^T S / (phi(q_i)^T z + eps),   Y_i = g_i L_i + (1 - g_i) G_i,
//   g_i = sigmoid(x_i w_g + b_g), per head, heads concatenated.
// For a group of hg heads starting at head h0 the numerators and denominators of all
// rows come from one GEMM:  [num | den] = phi(Q[:, h0 r .. (h0+hg) r)) B_g,
// where B_g (K = hg*r, N = hg*r + hg) holds S_h block-diagonally and z_h in column
// hg*r + h.  B_g is written by the statistics reduction each forward.
//
// Kernel: 128-row tiles, 192 threads.  Warp 4 issues TMA loads (128-byte swizzle): the
// group's L tile once, and the q tile and B_g through an mbarrier ring.  Warps 0-3
// apply phi to each landed q tile in shared memory (for fp32 also splitting it into tf32
// hi/lo planes), fence it for the async proxy and arrive on a "ready" barrier; warp 5
// issues tcgen05.mma into TMEM.  Epilogue (warps 0-3, one row per thread): numerators
// and denominators from TMEM, L and the blend in shared memory in place, then TMA bulk
// stores of the Y tile.  Shapes whose head group is not a whole number of 128-byte
// column boxes fall back to per-thread global loads and stores.
#include <algorithm>

#include "glga_internal.cuh"

namespace glga {
namespace {

constexpr int kBM = 128;
constexpr int kRowBytes = 128;
constexpr int kMaxStages = 4;
constexpr int kWorkers = 256;        // warps 0-7: phi pass and epilogue
constexpr int kProdWarp = 8;         // TMA producer
constexpr int kMmaWarp = 9;          // TMEM owner and MMA issuer
constexpr int kThreads = 320;
constexpr uint32_t kBoxBytes = kBM * kRowBytes;   // one 128-row x 128-byte TMA box

struct ReadoutParams {
    int64_t M;              // rows
    int32_t D, r, hg, n_groups;
    int32_t nk;             // K tiles per group
    int32_t BNr;            // GEMM N per group (>= hg*r + hg, multiple of 16)
    int32_t stages, tmem_cols;
    int32_t lboxes;         // 128-byte column boxes of the group's L/Y tile (0: no TMA path)
    uint32_t a_bytes, b_bytes, stage_bytes;
    const void *L;          // io [N, D]
    const float *t;         // [N]
    void *Y;                // io [N, D]
    float b_g, eps;
    unsigned *flag;
};

template <typename T>
struct IoT;
template <>
struct IoT<float> {
    static constexpr int VE = 4;      // elements per 16 bytes
    __device__ __forceinline__ static void unpack(const uint4 &u, float *v) {
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
        v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ static uint4 pack(const float *v) {
        return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                          __float_as_uint(v[3]));
    }
    __device__ __forceinline__ static float get(const float *p) { return *p; }
    __device__ __forceinline__ static void put(float *p, float x) { *p = x; }
};
template <>
struct IoT<__nv_bfloat16> {
    static constexpr int VE = 8;
    __device__ __forceinline__ static void unpack(const uint4 &u, float *v) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[2 * k] = __uint_as_float(w[k] << 16);
            v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float *v) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
            w[k] = *reinterpret_cast<uint32_t *>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ __forceinline__ static float get(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    __device__ __forceinline__ static void put(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// phi applied in place to one 16-byte chunk of the q tile (bf16: 8 values).
__device__ __forceinline__ void phi_chunk_bf16(uint4 *p) {
    uint4 u = *p;
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float a = phi(__uint_as_float(w[k] << 16));
        const float b = phi(__uint_as_float(w[k] & 0xffff0000u));
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        w[k] = *reinterpret_cast<uint32_t *>(&h);
    }
    *p = make_uint4(w[0], w[1], w[2], w[3]);
}

// fp32: phi, then split into tf32 hi (in place) and lo (same offset in the lo plane).
__device__ __forceinline__ void phi_split_chunk_f32(float4 *hi, float4 *lo) {
    float4 u = *hi;
    float v[4] = {phi(u.x), phi(u.y), phi(u.z), phi(u.w)};
    float h[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        h[k] = to_tf32(v[k]);
        l[k] = to_tf32(v[k] - h[k]);
    }
    *hi = make_float4(h[0], h[1], h[2], h[3]);
    *lo = make_float4(l[0], l[1], l[2], l[3]);
}

template <int SPLIT, typename T, int R>
__global__ void __launch_bounds__(kThreads, 1) readout_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmB0,
                                                              const __grid_constant__ CUtensorMap tmB1,
                                                              const __grid_constant__ CUtensorMap tmL,
                                                              const __grid_constant__ CUtensorMap tmY,
                                                              ReadoutParams p) {
    constexpr int kPlanes = SPLIT == 3 ? 2 : 1;
    constexpr int kPairs = SPLIT == 3 ? 3 : 1;
    constexpr uint32_t kFmt = SPLIT == 3 ? 2u : 1u;
    constexpr int KT = kRowBytes / static_cast<int>(sizeof(T));   // elements per tile row
    constexpr int VE = IoT<T>::VE;
    constexpr int kChunks32 = 32 / VE;                              // 16-byte chunks per 32 columns

    extern __shared__ uint8_t dsmem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t ready_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ __align__(8) uint64_t l_bar;
    __shared__ uint32_t tmem_base_sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *lbuf = smem + static_cast<size_t>(p.stages) * p.stage_bytes;   // L, then Y, tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x;                          // head group
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
    const int h0 = g * p.hg;
    const int hg = std::min(p.hg, p.D / R - h0);       // heads in this group
    const int qx0 = h0 * R;                            // first q / L / Y column of the group

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&ready_bar[s], kWorkers);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&done_bar, 1);
        mbar_init(&l_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_base_sh, static_cast<uint32_t>(p.tmem_cols));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kProdWarp) {
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            if (p.lboxes > 0) {
                mbar_arrive_expect_tx(&l_bar, p.lboxes * kBoxBytes);
                for (int b = 0; b < p.lboxes; ++b)
                    tma_load_2d(lbuf + b * kBoxBytes, &tmL, &l_bar, qx0 + b * KT, static_cast<int32_t>(m0));
            }
            int issued = 0;
            bool ok = true;
            for (int kb = 0; kb < p.nk; ++kb) {
                const int s = kb % p.stages;
                const uint32_t ph = static_cast<uint32_t>(kb / p.stages) & 1u;
                if (kb >= p.stages && !mbar_wait_bounded(&empty_bar[s], ph ^ 1u)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
                const uint32_t tx = p.a_bytes + kPlanes * p.b_bytes;
                mbar_arrive_expect_tx(&full_bar[s], tx);
                tma_load_2d(st, &tmQ, &full_bar[s], qx0 + kb * KT, static_cast<int32_t>(m0));
                uint8_t *bst = st + kPlanes * p.a_bytes;
                tma_load_2d(bst, &tmB0, &full_bar[s], kb * KT, g * p.BNr);
                if (kPlanes == 2) tma_load_2d(bst + p.b_bytes, &tmB1, &full_bar[s], kb * KT, g * p.BNr);
                ++issued;
            }
            if (!ok) {
                atomicOr(p.flag, kDevErrTimeout);
                for (int kb = std::max(0, issued - p.stages); kb < issued; ++kb)
                    mbar_wait_bounded(&full_bar[kb % p.stages], static_cast<uint32_t>(kb / p.stages) & 1u);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t idesc = instr_desc(kBM, p.BNr, kFmt, false, false);
            bool ok = true;
            for (int kb = 0; kb < p.nk; ++kb) {
                const int s = kb % p.stages;
                const uint32_t ph = static_cast<uint32_t>(kb / p.stages) & 1u;
                if (!mbar_wait_bounded(&ready_bar[s], ph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + static_cast<size_t>(s) * p.stage_bytes);
                const uint32_t b_addr = a_addr + kPlanes * p.a_bytes;
#pragma unroll
                for (int k = 0; k < kRowBytes / 32; ++k) {
#pragma unroll
                    for (int pr = 0; pr < kPairs; ++pr) {
                        const uint32_t ap = (pr == 2) ? 1u : 0u;
                        const uint32_t bp = (pr == 1) ? 1u : 0u;
                        const uint64_t ad = smem_desc(a_addr + ap * p.a_bytes + k * 32, 16, 1024, 2);
                        const uint64_t bd = smem_desc(b_addr + bp * p.b_bytes + k * 32, 16, 1024, 2);
                        const uint32_t acc = (kb | k | pr) != 0;
                        if (SPLIT == 3)
                            umma_tf32(tmem, ad, bd, idesc, acc);
                        else
                            umma_bf16(tmem, ad, bd, idesc, acc);
                    }
                }
                umma_commit(&empty_bar[s]);
            }
            if (!ok) atomicOr(p.flag, kDevErrTimeout);
            umma_commit(&done_bar);
        }
    } else {
        // ---------------- warps 0-7: phi on the landed q tiles ----------------
        bool ok = true;
        for (int kb = 0; kb < p.nk && ok; ++kb) {
            const int s = kb % p.stages;
            const uint32_t ph = static_cast<uint32_t>(kb / p.stages) & 1u;
            if (!mbar_wait_bounded(&full_bar[s], ph)) {
                ok = false;
                break;
            }
            uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
            // threads 2t and 2t+1 own row t of the tile: 4 chunks of 16 bytes each
            uint4 *row = reinterpret_cast<uint4 *>(st + (threadIdx.x >> 1) * kRowBytes) + (threadIdx.x & 1) * 4;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (SPLIT == 3) {
                    float4 *hi = reinterpret_cast<float4 *>(row + c);
                    float4 *lo = reinterpret_cast<float4 *>(reinterpret_cast<uint8_t *>(row + c) + p.a_bytes);
                    phi_split_chunk_f32(hi, lo);
                } else {
                    phi_chunk_bf16(row + c);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&ready_bar[s]);
        }
        if (!ok && lane == 0) atomicOr(p.flag, kDevErrTimeout);
    }
    __syncwarp();

    if (warp < 8) {
        // ---------------- epilogue: G = num / (den + eps), blend with L, write Y ----------------
        // warp w reads TMEM lanes 32*(w%4).. (its rows); warpgroup w/4 takes every other
        // 32-column chunk
        const bool done = mbar_wait_bounded(&done_bar, 0);
        const bool lok = p.lboxes == 0 || mbar_wait_bounded(&l_bar, 0);
        tc_fence_after();
        const int quad = warp & 3, wg = warp >> 2;
        const int rt = quad * 32 + lane;
        const int64_t row = m0 + rt;
        const bool live = row < p.M;
        if (!done || !lok) {
            if (lane == 0) atomicOr(p.flag, kDevErrTimeout);
        } else {
            const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
            const float gt = live ? __ldg(p.t + row) + p.b_g : 0.f;
            const float gate = 1.f / (1.f + __expf(-gt));
            const int ncol = hg * R;
            for (int c0 = wg * 32; c0 < ncol; c0 += 64) {
                uint32_t v[32], dv[32];
                tmem_ld32(tmem + lane_base + static_cast<uint32_t>(c0), v);
                // denominators of the heads this chunk touches: column hg*R + head
                tmem_ld32(tmem + lane_base + static_cast<uint32_t>(ncol + c0 / R), dv);
                tmem_ld_wait();
                float gv[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    gv[j] = (1.f - gate) * __uint_as_float(v[j]) /
                            (__uint_as_float(dv[R >= 32 ? 0 : j / R]) + p.eps);
                if (p.lboxes > 0) {
                    // L from the swizzled shared tile, Y written back in place
                    const int b = c0 / KT, e0 = c0 % KT;
                    uint8_t *base = lbuf + b * kBoxBytes + rt * kRowBytes;
#pragma unroll
                    for (int q = 0; q < kChunks32; ++q) {
                        const int ch = (e0 / VE + q) ^ (rt & 7);
                        uint4 *pch = reinterpret_cast<uint4 *>(base + ch * 16);
                        float lv[VE], y[VE];
                        IoT<T>::unpack(*pch, lv);
#pragma unroll
                        for (int e = 0; e < VE; ++e) y[e] = gate * lv[e] + gv[q * VE + e];
                        *pch = IoT<T>::pack(y);
                    }
                } else if (live) {
                    const T *L = static_cast<const T *>(p.L) + row * p.D + qx0;
                    T *Y = static_cast<T *>(p.Y) + row * p.D + qx0;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c0 + j < ncol)
                            IoT<T>::put(Y + c0 + j, gate * IoT<T>::get(L + c0 + j) + gv[j]);
                }
            }
        }
        if (p.lboxes > 0) {
            fence_proxy_async_smem();
            named_barrier_sync(1, kWorkers);
            if (threadIdx.x == 0 && done && lok) {
                for (int b = 0; b < p.lboxes; ++b)
                    tma_store_2d(&tmY, lbuf + b * kBoxBytes, qx0 + b * KT, static_cast<int32_t>(m0));
                bulk_commit_group();
                bulk_wait_group_read0();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
    }
}

template <int SPLIT, typename T>
glga_status launch_readout_r(Ctx *c, const ReadoutParams &p, size_t smem, const CUtensorMap &q,
                             const CUtensorMap &b0, const CUtensorMap &b1, const CUtensorMap &ml,
                             const CUtensorMap &my, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>(p.n_groups), static_cast<unsigned>(ceil_div(p.M, kBM)));
#define GLGA_RO(RR)                                                                              \
    case RR: {                                                                                   \
        auto kern = readout_kernel<SPLIT, T, RR>;                                                \
        GLGA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,      \
                                       static_cast<int>(smem)));                                 \
        kern<<<grid, kThreads, smem, s>>>(q, b0, b1, ml, my, p);                                 \
        break;                                                                                   \
    }
    switch (p.r) {
        GLGA_RO(8) GLGA_RO(16) GLGA_RO(32) GLGA_RO(64) GLGA_RO(128)
        default: set_error("unsupported r"); return GLGA_ERR_UNSUPPORTED;
    }
#undef GLGA_RO
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    return GLGA_OK;
}

}  // namespace

glga_status readout_setup(Ctx *c) {
    const int kt = kRowBytes / c->elem;
    // hg*r + hg + 32 <= 256: numerators, denominators and the 32-column read past them
    // fit one 256-column TMEM allocation.  Groups span at most 128 columns (one head for
    // r >= 64): narrower groups let more CTAs share an SM and overlap their phases.
    const int hg_max = std::max(1, std::min(224 / (c->r + 1), (c->r >= 64 ? 64 : 128) / c->r));
    c->ro_groups = static_cast<int32_t>(ceil_div(c->H, hg_max));
    c->ro_hg = static_cast<int32_t>(ceil_div(c->H, c->ro_groups));
    c->ro_kp = static_cast<int32_t>(ceil_div(static_cast<int64_t>(c->ro_hg) * c->r, kt) * kt);
    c->ro_bn = static_cast<int32_t>(ceil_div(c->ro_hg * c->r + c->ro_hg, 16) * 16);
    const int last = c->H - (c->ro_groups - 1) * c->ro_hg;
    c->ro_tma_epi = (c->ro_hg * c->r) % kt == 0 && (last * c->r) % kt == 0;
    const int planes = c->split == 3 ? 2 : 1;
    const size_t plane = static_cast<size_t>(c->ro_groups) * c->ro_bn * c->ro_kp * c->elem;
    glga_status st = dev_alloc(c, &c->Bro, planes * plane);
    if (st != GLGA_OK) return st;
    cudaError_t e = cudaMemset(c->Bro, 0, planes * plane);   // off-diagonal blocks stay zero
    if (e != cudaSuccess) return cuda_fail(e, "readout operand init");
    const CUtensorMapDataType dt =
        c->io == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    for (int pl = 0; pl < planes; ++pl) {
        st = encode_tmap_2d(&c->tmBro[pl].map, dt, static_cast<uint8_t *>(c->Bro) + pl * plane,
                            c->ro_kp, static_cast<uint64_t>(c->ro_groups) * c->ro_bn,
                            static_cast<uint64_t>(c->ro_kp) * c->elem, kt, c->ro_bn);
        if (st != GLGA_OK) return st;
        c->tmBro[pl].valid = true;
    }
    st = dev_alloc(c, &c->L, static_cast<size_t>(c->N) * c->D * c->elem);
    if (st != GLGA_OK) return st;
    if (c->N > 0) {
        const uint64_t rb = static_cast<uint64_t>(c->D) * c->elem;
        st = encode_tmap_2d(&c->tmQ.map, dt, c->Q, c->D, c->N, rb, kt, kBM);
        if (st == GLGA_OK) st = encode_tmap_2d(&c->tmL.map, dt, c->L, c->D, c->N, rb, kt, kBM);
        if (st != GLGA_OK) return st;
        c->tmQ.valid = c->tmL.valid = true;
    }
    return GLGA_OK;
}

glga_status readout_run(Ctx *c, float b_g, float eps, void *Y, cudaStream_t s) {
    if (c->N == 0) return GLGA_OK;
    const int kt = kRowBytes / c->elem;
    ReadoutParams p;
    p.M = c->N;
    p.D = c->D;
    p.r = c->r;
    p.hg = c->ro_hg;
    p.n_groups = c->ro_groups;
    p.nk = c->ro_kp / kt;
    p.BNr = c->ro_bn;
    // the epilogue reads 32 columns starting at a denominator column (<= hg*r + hg - 1)
    int tc = 32;
    while (tc < p.BNr || tc < p.hg * p.r + p.hg + 32) tc <<= 1;
    p.tmem_cols = tc;
    const int planes = c->split == 3 ? 2 : 1;
    p.a_bytes = kBM * kRowBytes;
    p.b_bytes = static_cast<uint32_t>(p.BNr) * kRowBytes;
    p.stage_bytes = planes * (p.a_bytes + p.b_bytes);
    p.lboxes = c->ro_tma_epi ? static_cast<int32_t>(ceil_div(static_cast<int64_t>(p.hg) * p.r, kt)) : 0;
    const uint32_t lbytes = static_cast<uint32_t>(p.lboxes) * kBoxBytes;
    p.stages = std::max(1, std::min(std::min(p.nk, kMaxStages),
                                    static_cast<int>((200u * 1024u - lbytes) / p.stage_bytes)));
    p.L = c->L;
    p.t = c->t;
    p.Y = Y;
    p.b_g = b_g;
    p.eps = eps;
    p.flag = c->dev_flag;
    const CUtensorMapDataType dt =
        c->io == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap my = c->tmL.map;   // placeholder when the TMA store path is off
    if (p.lboxes > 0) {
        glga_status st = encode_tmap_2d(&my, dt, Y, c->D, c->N, static_cast<uint64_t>(c->D) * c->elem,
                                        kt, kBM);
        if (st != GLGA_OK) return st;
    }
    const size_t smem = static_cast<size_t>(p.stages) * p.stage_bytes + lbytes + 1024;
    const CUtensorMap &b1 = planes == 2 ? c->tmBro[1].map : c->tmBro[0].map;
    if (c->io == GLGA_F32)
        return launch_readout_r<3, float>(c, p, smem, c->tmQ.map, c->tmBro[0].map, b1, c->tmL.map, my, s);
    return launch_readout_r<1, __nv_bfloat16>(c, p, smem, c->tmQ.map, c->tmBro[0].map, b1, c->tmL.map, my, s);
}

}  // namespace glga
