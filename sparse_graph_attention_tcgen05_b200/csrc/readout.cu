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
// Persistent kernel, one CTA per SM walking (row tile, head group) tiles round-robin;
// W worker warps (a multiple of 4) and three single-thread roles:
//   warp W     TMA producer: the q tile's K blocks through an mbarrier ring (and B_g's,
//              unless B_g is resident)
//   warp W+1   MMA issuer: accumulates tile i into TMEM buffer i & 1 (256 columns each)
//   warp W+2   TMA producer: the group's L tile into one of 2-3 L/Y buffers
//   warps 0..W-1  phi on each landed q block (fp32: also the tf32 hi/lo split), then the
//              epilogue of the previous tile: numerators and denominators from TMEM, the
//              blend with L and the gate in shared memory, TMA bulk stores of Y
// so the loads and MMAs of tile i overlap the epilogue of tile i - 1.  When the grid is
// a multiple of the number of head groups every CTA keeps one group, and B_g (a few tens
// of KB) is loaded once and stays in shared memory.  The Y stores of a tile are waited
// for one tile later, when their buffer is handed back to the L producer.  Shapes whose
// head group is not a whole number of 128-byte column boxes use per-thread global loads
// and stores in the epilogue instead of the L/Y buffers.
#include <algorithm>
#include <vector>

#include "glga_internal.cuh"

namespace glga {
namespace {

constexpr int kBM = 128;
constexpr int kRowBytes = 128;
constexpr int kMaxStages = 8;
constexpr int kWorkerWarps = 16;     // phi pass and epilogue
constexpr int kWorkers = kWorkerWarps * 32;
constexpr int kWG = kWorkerWarps / 4;         // worker warpgroups (TMEM lane quarters x kWG)
constexpr int kTPR = kWorkers / 128;          // phi-pass threads per tile row
constexpr int kProdWarp = kWorkerWarps;       // TMA producer (q, B_g)
constexpr int kMmaWarp = kWorkerWarps + 1;    // TMEM owner and MMA issuer
constexpr int kLWarp = kWorkerWarps + 2;      // L tile loader
constexpr int kThreads = kWorkers + 96;
constexpr int kMaxLBufs = 3;
static_assert(kWorkerWarps % 4 == 0 && 8 % kTPR == 0, "worker warps: 4, 8 or 16");
constexpr uint32_t kBoxBytes = kBM * kRowBytes;   // one 128-row x 128-byte TMA box
constexpr uint32_t kAccCols = 256;                // TMEM columns per accumulator buffer

struct ReadoutParams {
    int64_t M;              // rows
    int64_t n_total;        // row tiles x head groups
    int32_t D, r, hg, n_groups;
    int32_t nk;             // K tiles per group
    int32_t BNr;            // GEMM N per group (>= hg*r + hg, multiple of 16)
    int32_t stages;
    int32_t lboxes;         // 128-byte column boxes of the group's L/Y tile (0: no TMA path)
    int32_t lbufs;          // L/Y staging buffers (2 or 3)
    int32_t b_resident;     // B_g loaded once per CTA (grid is a multiple of n_groups)
    const int32_t *tile_seg;  // segment of each row tile (NULL: one segment)
    uint32_t a_bytes, b_bytes, stage_bytes;
    uint32_t bres_bytes;    // resident B_g: planes x nk x b_bytes (0 when streamed)
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
    const uint4 u = *p;
    *p = make_uint4(phi_bf16x2(u.x), phi_bf16x2(u.y), phi_bf16x2(u.z), phi_bf16x2(u.w));
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
    constexpr int kHeads = R >= 32 ? 1 : 32 / R;                    // heads per 32 columns
    constexpr int kCPT = 8 / kTPR;                                  // phi chunks per thread and row

    extern __shared__ uint8_t dsmem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t ready_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2];    // MMA -> epilogue: accumulator complete
    __shared__ __align__(8) uint64_t acce_bar[2];    // epilogue -> MMA: accumulator drained
    __shared__ __align__(8) uint64_t lfull_bar[kMaxLBufs];   // L tile landed in buffer b
    __shared__ __align__(8) uint64_t lfree_bar[kMaxLBufs];   // Y stores finished reading b
    __shared__ __align__(8) uint64_t bres_bar;       // resident B_g landed
    __shared__ __align__(8) uint64_t drain_bar;      // error path: issued MMAs retired
    __shared__ uint32_t tmem_base_sh;

    // shared memory: [resident B_g][K ring: stages x stage_bytes][L/Y: lbufs x lbytes]
    uint8_t *bres = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *smem = bres + p.bres_bytes;
    const uint32_t lbytes = static_cast<uint32_t>(p.lboxes) * kBoxBytes;
    uint8_t *lbase = smem + static_cast<size_t>(p.stages) * p.stage_bytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t n_my = p.n_total > blockIdx.x
                             ? static_cast<int32_t>((p.n_total - blockIdx.x + gridDim.x - 1) / gridDim.x)
                             : 0;
    const uint32_t a_planes = kPlanes * p.a_bytes;   // q part of a ring stage

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&ready_bar[s], kWorkerWarps);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf_bar[b], 1);
            mbar_init(&acce_bar[b], kWorkerWarps);
        }
        for (int b = 0; b < kMaxLBufs; ++b) {
            mbar_init(&lfull_bar[b], 1);
            mbar_init(&lfree_bar[b], 1);
        }
        mbar_init(&bres_bar, 1);
        mbar_init(&drain_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_base_sh, 2 * kAccCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kProdWarp) {
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            if (p.b_resident && n_my > 0) {
                // every tile of this CTA belongs to head group blockIdx.x % n_groups
                const int g = static_cast<int>(blockIdx.x % p.n_groups);
                mbar_arrive_expect_tx(&bres_bar, p.bres_bytes);
                for (int kb = 0; kb < p.nk; ++kb) {
                    uint8_t *dst = bres + static_cast<size_t>(kb) * kPlanes * p.b_bytes;
                    tma_load_2d(dst, &tmB0, &bres_bar, kb * KT, g * p.BNr);
                    if (kPlanes == 2) tma_load_2d(dst + p.b_bytes, &tmB1, &bres_bar, kb * KT, g * p.BNr);
                }
            }
            int it = 0;
            RingPos rp;
            TileWalk tw(blockIdx.x, gridDim.x, p.n_groups);
            // with segments, B_g of the tile's segment: rows (seg * n_groups + g) * BNr of
            // the operand; the segment id is loaded one tile ahead
            int seg_next = (p.tile_seg && n_my > 0) ? __ldg(p.tile_seg + tw.row) : 0;
            bool ok = true;
            for (int i = 0; i < n_my && ok; ++i, tw.next()) {
                const int g = tw.col;
                const int32_t m0 = tw.row * kBM;
                const int qx0 = g * p.hg * R;
                const int seg = seg_next;
                if (p.tile_seg && i + 1 < n_my) {
                    TileWalk nx = tw;
                    nx.next();
                    seg_next = __ldg(p.tile_seg + nx.row);
                }
                const int32_t brow = (seg * p.n_groups + g) * p.BNr;
                for (int kb = 0; kb < p.nk; ++kb, ++it, rp.next(p.stages)) {
                    const int s = rp.slot;
                    if (it >= p.stages && !mbar_wait_bounded(&empty_bar[s], rp.phase ^ 1u)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
                    // TMA brings the raw q box (the fp32 lo plane is written by the
                    // phi pass) and, when streamed, B_g's K block
                    mbar_arrive_expect_tx(&full_bar[s], p.b_resident ? p.a_bytes
                                                                     : p.a_bytes + kPlanes * p.b_bytes);
                    tma_load_2d(st, &tmQ, &full_bar[s], qx0 + kb * KT, m0);
                    if (!p.b_resident) {
                        uint8_t *bst = st + a_planes;
                        tma_load_2d(bst, &tmB0, &full_bar[s], kb * KT, brow);
                        if (kPlanes == 2) tma_load_2d(bst + p.b_bytes, &tmB1, &full_bar[s], kb * KT, brow);
                    }
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA can exit
                atomicOr(p.flag, kDevErrTimeout);
                for (int q = std::max(0, it - p.stages); q < it; ++q)
                    mbar_wait_bounded(&full_bar[q % p.stages], static_cast<uint32_t>(q / p.stages) & 1u);
                if (p.b_resident) mbar_wait_bounded(&bres_bar, 0);
            }
        }
    } else if (warp == kLWarp) {
        if (lane == 0 && p.lboxes > 0) {
            // the L tile of tile i goes into buffer i % lbufs once the Y stores of tile
            // i - lbufs have been read out of it
            tma_prefetch_desc(&tmL);
            int i = 0;
            RingPos lp;
            TileWalk tw(blockIdx.x, gridDim.x, p.n_groups);
            bool ok = true;
            for (; i < n_my; ++i, lp.next(p.lbufs), tw.next()) {
                const int b = lp.slot;
                if (i >= p.lbufs && !mbar_wait_bounded(&lfree_bar[b], lp.phase ^ 1u)) {
                    ok = false;
                    break;
                }
                const int g = tw.col;
                const int32_t m0 = tw.row * kBM;
                mbar_arrive_expect_tx(&lfull_bar[b], lbytes);
                for (int bx = 0; bx < p.lboxes; ++bx)
                    tma_load_2d(lbase + b * lbytes + bx * kBoxBytes, &tmL, &lfull_bar[b],
                                g * p.hg * R + bx * KT, m0);
            }
            if (!ok) {
                atomicOr(p.flag, kDevErrTimeout);
                for (int q = std::max(0, i - p.lbufs); q < i; ++q)
                    mbar_wait_bounded(&lfull_bar[q % p.lbufs], static_cast<uint32_t>(q / p.lbufs) & 1u);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t idesc = instr_desc(kBM, p.BNr, kFmt, false, false);
            RingPos rp;
            bool ok = !p.b_resident || n_my == 0 || mbar_wait_bounded(&bres_bar, 0);
            const uint32_t bres_addr = smem_u32(bres);
            for (int i = 0; i < n_my && ok; ++i) {
                const int buf = static_cast<int>(i & 1);
                if (i >= 2 && !mbar_wait_bounded(&acce_bar[buf], static_cast<uint32_t>((i >> 1) - 1) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem + static_cast<uint32_t>(buf) * kAccCols;
                for (int kb = 0; kb < p.nk; ++kb, rp.next(p.stages)) {
                    const int s = rp.slot;
                    if (!mbar_wait_bounded(&ready_bar[s], rp.phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + static_cast<size_t>(s) * p.stage_bytes);
                    const uint32_t b_addr = p.b_resident
                                                ? bres_addr + static_cast<uint32_t>(kb) * kPlanes * p.b_bytes
                                                : a_addr + a_planes;
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
                                umma_tf32(dcol, ad, bd, idesc, acc);
                            else
                                umma_bf16(dcol, ad, bd, idesc, acc);
                        }
                    }
                    umma_commit(&empty_bar[s]);
                }
                if (ok) umma_commit(&accf_bar[buf]);
            }
            if (!ok) {
                // drain the MMAs already issued before TMEM is released
                atomicOr(p.flag, kDevErrTimeout);
                umma_commit(&drain_bar);
                mbar_wait_bounded(&drain_bar, 0);
            }
        }
    } else {
        // ------------ worker warps: phi of tile i, then the epilogue of tile i - 1 ------------
        const int quad = warp & 3, wg = warp >> 2;
        const int rt = quad * 32 + lane;                 // epilogue row inside the tile
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const int trow = threadIdx.x / kTPR;             // phi-pass row
        const int tpart = threadIdx.x % kTPR;
        float t_prev = 0.f;                              // gate logit of tile i - 1's row
        RingPos rp, lp;                                  // K ring; L/Y buffers (epilogue)
        int lp_prev = 0;                                 // L/Y buffer of the previous epilogue
        TileWalk tw(blockIdx.x, gridDim.x, p.n_groups);   // tile i (phi pass)
        TileWalk te = tw;                                // tile i - 1 (epilogue)
        bool ok = true;
        // a bounded wait of a phi pass that gave up: the workers agree on it at the next
        // epilogue's barrier (one per tile), so all of them leave the loop together
        bool bad = false;
        for (int i = 0; i <= n_my && ok; ++i) {
            float t_cur = 0.f;
            if (i < n_my) {
                // the gate logit of this tile's row, consumed one iteration later
                const int64_t row = static_cast<int64_t>(tw.row) * kBM + rt;
                if (row < p.M) t_cur = __ldg(p.t + row);
                tw.next();
                for (int kb = 0; kb < p.nk; ++kb, rp.next(p.stages)) {
                    const int s = rp.slot;
                    // the warp agrees on the outcome (it stays converged for its arrival)
                    if (!__all_sync(0xffffffffu, !bad && mbar_wait_bounded(&full_bar[s], rp.phase))) {
                        bad = true;        // (the MMA warp's own bounded wait then gives up too)
                        continue;
                    }
                    uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
                    // kTPR threads share a tile row, kCPT of its 8 16-byte chunks each; the
                    // chunk order is rotated by the row so that the 8 threads of a
                    // shared-memory phase touch 8 different bank groups
                    uint4 *rowp = reinterpret_cast<uint4 *>(st + trow * kRowBytes);
#pragma unroll
                    for (int c = 0; c < kCPT; ++c) {
                        const int ch = (tpart * kCPT + c) ^ (trow & 7);
                        if (SPLIT == 3) {
                            float4 *hi = reinterpret_cast<float4 *>(rowp + ch);
                            float4 *lo = reinterpret_cast<float4 *>(reinterpret_cast<uint8_t *>(rowp + ch) + p.a_bytes);
                            phi_split_chunk_f32(hi, lo);
                        } else {
                            phi_chunk_bf16(rowp + ch);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ready_bar[s]);
                }
            }
            if (i > 0) {
                // ---- epilogue of tile k = i - 1 ----
                const int k = i - 1;
                const int buf = k & 1;
                const int g = te.col;
                const int64_t m0 = static_cast<int64_t>(te.row) * kBM;
                te.next();
                const int h0 = g * p.hg;
                const int hg = std::min(p.hg, p.D / R - h0);
                const int qx0 = h0 * R;
                const int ncol = hg * R;
                const int64_t row = m0 + rt;
                const bool live = row < p.M;
                const int lb_i = lp.slot;
                bool got = !bad && mbar_wait_bounded(&accf_bar[buf], static_cast<uint32_t>(k >> 1) & 1u);
                if (p.lboxes > 0) got = got && mbar_wait_bounded(&lfull_bar[lb_i], lp.phase);
                if (named_barrier_or(1, kWorkers, !got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float gate = 1.f / (1.f + __expf(-(t_prev + p.b_g)));
                const uint32_t acc = tmem + lane_base + static_cast<uint32_t>(buf) * kAccCols;
                uint8_t *lb = lbase + lb_i * lbytes;
                for (int c0 = wg * 32; c0 < ncol; c0 += 32 * kWG) {
                    uint32_t v[32], dv[kHeads];
                    tmem_ld32(acc + static_cast<uint32_t>(c0), v);
                    // denominators of the heads this chunk touches: column hg*R + head
                    tmem_ld_n<kHeads>(acc + static_cast<uint32_t>(ncol + c0 / R), dv);
                    tmem_ld_wait();
                    float scale[kHeads];
#pragma unroll
                    for (int h = 0; h < kHeads; ++h)
                        scale[h] = (1.f - gate) / (__uint_as_float(dv[h]) + p.eps);
                    if (p.lboxes > 0) {
                        // L from the swizzled shared tile, Y written back in place
                        const int bx = c0 / KT, e0 = c0 % KT;
                        uint8_t *base = lb + bx * kBoxBytes + rt * kRowBytes;
#pragma unroll
                        for (int q = 0; q < kChunks32; ++q) {
                            const int ch = (e0 / VE + q) ^ (rt & 7);
                            uint4 *pch = reinterpret_cast<uint4 *>(base + ch * 16);
                            float lv[VE], y[VE];
                            IoT<T>::unpack(*pch, lv);
#pragma unroll
                            for (int e = 0; e < VE; ++e) {
                                const int j = q * VE + e;
                                y[e] = gate * lv[e] + __uint_as_float(v[j]) * scale[j / R < kHeads ? j / R : 0];
                            }
                            *pch = IoT<T>::pack(y);
                        }
                    } else if (live) {
                        const T *L = static_cast<const T *>(p.L) + row * p.D + qx0;
                        T *Y = static_cast<T *>(p.Y) + row * p.D + qx0;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c0 + j < ncol)
                                IoT<T>::put(Y + c0 + j, gate * IoT<T>::get(L + c0 + j) +
                                                            __uint_as_float(v[j]) *
                                                                scale[j / R < kHeads ? j / R : 0]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce_bar[buf]);   // accumulator buffer may be reused
                if (p.lboxes > 0) {
                    fence_proxy_async_smem();
                    named_barrier_sync(2, kWorkers);
                    if (threadIdx.x == 0) {
                        for (int bx = 0; bx < p.lboxes; ++bx)
                            tma_store_2d(&tmY, lb + bx * kBoxBytes, qx0 + bx * KT, static_cast<int32_t>(m0));
                        bulk_commit_group();
                        // the previous tile's stores have now been read out of their buffer,
                        // which may take a new L tile
                        bulk_wait_group_read1();
                        if (k > 0) mbar_arrive(&lfree_bar[lp_prev]);
                    }
                }
                lp_prev = lb_i;
                lp.next(p.lbufs);
            }
            t_prev = t_cur;
        }
        if (!ok && lane == 0) atomicOr(p.flag, kDevErrTimeout);
        if (threadIdx.x == 0) bulk_wait_group_read0();   // shared memory outlives the stores
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kAccCols);
    }
}

template <int SPLIT, typename T>
glga_status launch_readout_r(Ctx *c, const ReadoutParams &p, unsigned grid, size_t smem,
                             const CUtensorMap &q, const CUtensorMap &b0, const CUtensorMap &b1,
                             const CUtensorMap &ml, const CUtensorMap &my, cudaStream_t s) {
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

// Rows whose segment differs from the segment of their 128-row tile's first row (tiles
// that straddle a segment boundary): the tile GEMM used the first row's S, z for them,
// so they are redone here on the CUDA cores, one warp per row, with their own segment's
// fp32 statistics: G_i = phi(q_i)^T S / (phi(q_i)^T z + eps), then the same gate blend
// with L_i as the tile epilogue.
constexpr int kFixRowsPerBlock = 4;
constexpr int kFixMaxD = 1024;

template <typename T>
__global__ void __launch_bounds__(32 * kFixRowsPerBlock) readout_fixup_kernel(
    const int32_t *__restrict__ rows, const int32_t *__restrict__ segs, int64_t n,
    const T *__restrict__ Q, const T *__restrict__ L, const float *__restrict__ t,
    const float *__restrict__ Sz, int64_t n_seg, int H, int R, float b_g, float eps, T *__restrict__ Y) {
    __shared__ float ph[kFixRowsPerBlock][kFixMaxD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m = static_cast<int64_t>(blockIdx.x) * kFixRowsPerBlock + warp;
    if (m >= n) return;   // warp-uniform; no block-wide barrier follows
    const int64_t row = rows[m], seg = segs[m];
    const int D = H * R;
    for (int c = lane; c < D; c += 32) ph[warp][c] = phi(IoT<T>::get(Q + row * D + c));
    __syncwarp();
    const float gate = 1.f / (1.f + __expf(-(t[row] + b_g)));
    const int64_t hrr = static_cast<int64_t>(H) * R * R;
    const float *S = Sz + seg * hrr;
    const float *z = Sz + n_seg * hrr + seg * H * R;
    for (int c = lane; c < D; c += 32) {
        const int h = c / R, cc = c - h * R;
        float num = 0.f, den = 0.f;
        for (int a = 0; a < R; ++a) {
            const float f = ph[warp][h * R + a];
            num = fmaf(f, S[(static_cast<int64_t>(h) * R + a) * R + cc], num);
            den = fmaf(f, z[h * R + a], den);
        }
        const float y = gate * IoT<T>::get(L + row * D + c) + (1.f - gate) * num / (den + eps);
        IoT<T>::put(Y + row * D + c, y);
    }
}

}  // namespace

glga_status readout_setup(Ctx *c) {
    const int kt = kRowBytes / c->elem;
    // hg*r + hg + 32 <= 256: numerators, denominators and the 32-column read past them
    // fit one 256-column TMEM buffer.  Groups span at most 128 columns (one head for
    // r >= 64), which bounds the two L/Y staging buffers to 2 x 64 KB.
    const int hg_max = std::max(1, std::min(224 / (c->r + 1), (c->r >= 64 ? 64 : 128) / c->r));
    c->ro_groups = static_cast<int32_t>(ceil_div(c->H, hg_max));
    c->ro_hg = static_cast<int32_t>(ceil_div(c->H, c->ro_groups));
    c->ro_kp = static_cast<int32_t>(ceil_div(static_cast<int64_t>(c->ro_hg) * c->r, kt) * kt);
    c->ro_bn = static_cast<int32_t>(ceil_div(c->ro_hg * c->r + c->ro_hg, 16) * 16);
    const int last = c->H - (c->ro_groups - 1) * c->ro_hg;
    c->ro_tma_epi = (c->ro_hg * c->r) % kt == 0 && (last * c->r) % kt == 0;
    const int planes = c->split == 3 ? 2 : 1;
    // one operand per segment and group: [planes][n_seg][groups][BNr][Kp]
    const uint64_t b_rows = static_cast<uint64_t>(c->n_seg) * c->ro_groups * c->ro_bn;
    const size_t plane = static_cast<size_t>(b_rows) * c->ro_kp * c->elem;
    if (b_rows >= (uint64_t{1} << 31) || planes * plane > (size_t{4} << 30)) {
        set_error("glga_create: %lld segments need more than 4 GiB of readout operands",
                  static_cast<long long>(c->n_seg));
        return GLGA_ERR_UNSUPPORTED;
    }
    glga_status st = dev_alloc(c, &c->Bro, planes * plane);
    if (st != GLGA_OK) return st;
    cudaError_t e = cudaMemset(c->Bro, 0, planes * plane);   // off-diagonal blocks stay zero
    if (e != cudaSuccess) return cuda_fail(e, "readout operand init");
    const CUtensorMapDataType dt =
        c->io == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    for (int pl = 0; pl < planes; ++pl) {
        st = encode_tmap_2d(&c->tmBro[pl].map, dt, static_cast<uint8_t *>(c->Bro) + pl * plane,
                            c->ro_kp, b_rows, static_cast<uint64_t>(c->ro_kp) * c->elem, kt, c->ro_bn);
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
    if (c->n_seg > 1 && c->N > 0) {
        // segment of every tile's first row, and the rows whose segment differs from it
        const int64_t m_tiles = ceil_div(c->N, kBM);
        std::vector<int32_t> ts(static_cast<size_t>(m_tiles)), fr, fs;
        int64_t k = 0;
        for (int64_t row = 0; row < c->N; ++row) {
            while (c->seg_ptr[k + 1] <= row) ++k;   // skips empty segments
            if (row % kBM == 0) ts[static_cast<size_t>(row / kBM)] = static_cast<int32_t>(k);
            else if (k != ts[static_cast<size_t>(row / kBM)]) {
                fr.push_back(static_cast<int32_t>(row));
                fs.push_back(static_cast<int32_t>(k));
            }
        }
        c->n_fix = static_cast<int64_t>(fr.size());
        st = dev_alloc(c, reinterpret_cast<void **>(&c->tile_seg), ts.size() * sizeof(int32_t));
        if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->fix_row), (fr.size() + 1) * sizeof(int32_t));
        if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->fix_seg), (fs.size() + 1) * sizeof(int32_t));
        if (st != GLGA_OK) return st;
        e = cudaMemcpy(c->tile_seg, ts.data(), ts.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
        if (e == cudaSuccess && !fr.empty())
            e = cudaMemcpy(c->fix_row, fr.data(), fr.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
        if (e == cudaSuccess && !fs.empty())
            e = cudaMemcpy(c->fix_seg, fs.data(), fs.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "segment tables");
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
    p.n_total = ceil_div(c->N, kBM) * c->ro_groups;
    p.nk = c->ro_kp / kt;
    p.BNr = c->ro_bn;
    const int planes = c->split == 3 ? 2 : 1;
    p.a_bytes = kBM * kRowBytes;
    p.b_bytes = static_cast<uint32_t>(p.BNr) * kRowBytes;
    p.lboxes = c->ro_tma_epi ? static_cast<int32_t>(ceil_div(static_cast<int64_t>(p.hg) * p.r, kt)) : 0;
    // Dynamic shared memory: resident B_g (when it fits), the K ring, and 2-3 L/Y
    // buffers (a third when two ring stages still fit beside it).
    constexpr int64_t kBudget = 220 * 1024;
    const int64_t lb1 = static_cast<int64_t>(p.lboxes) * kBoxBytes;
    const int64_t bres = static_cast<int64_t>(planes) * p.nk * p.b_bytes;
    p.b_resident = 0;
    p.lbufs = 0;
    // B_g stays resident only with one segment (otherwise it changes with the tile)
    for (int resident = c->n_seg == 1 ? 1 : 0; resident >= 0 && p.lbufs == 0; --resident) {
        const int64_t stage = planes * (p.a_bytes + (resident ? 0 : p.b_bytes));
        const int64_t fixed = resident ? bres : 0;
        for (int nb = 3; nb >= 2 && p.lbufs == 0; --nb) {
            const int64_t left = kBudget - fixed - nb * lb1;
            if (left >= (nb == 3 ? 2 : 1) * stage) {
                p.b_resident = resident;
                p.lbufs = nb;
                p.stage_bytes = static_cast<uint32_t>(stage);
                p.stages = static_cast<int32_t>(std::min<int64_t>(kMaxStages, left / stage));
            }
        }
    }
    if (p.lbufs == 0) {
        set_error("readout: shared memory plan does not fit");
        return GLGA_ERR_UNSUPPORTED;
    }
    p.bres_bytes = p.b_resident ? static_cast<uint32_t>(bres) : 0u;
    const uint32_t lbytes = static_cast<uint32_t>(p.lbufs * lb1);
    // persistent: one CTA per SM (it holds all 512 TMEM columns); with resident B_g the
    // grid is a multiple of the group count so every CTA stays on one group
    int64_t grid = std::min<int64_t>(p.n_total, c->num_sms);
    if (p.b_resident) {
        grid = grid / p.n_groups * p.n_groups;
        if (grid == 0) {
            p.b_resident = 0;
            p.bres_bytes = 0;
            grid = std::min<int64_t>(p.n_total, c->num_sms);
            p.stage_bytes = planes * (p.a_bytes + p.b_bytes);
            p.stages = static_cast<int32_t>(std::min<int64_t>(
                kMaxStages, (kBudget - static_cast<int64_t>(lbytes)) / p.stage_bytes));
            if (p.stages < 1) {
                set_error("readout: shared memory plan does not fit");
                return GLGA_ERR_UNSUPPORTED;
            }
        }
    }
    p.L = c->L;
    p.t = c->t;
    p.Y = Y;
    p.b_g = b_g;
    p.eps = eps;
    p.flag = c->dev_flag;
    p.tile_seg = c->n_seg > 1 ? c->tile_seg : nullptr;
    const CUtensorMapDataType dt =
        c->io == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap my = c->tmL.map;   // placeholder when the TMA store path is off
    if (p.lboxes > 0) {
        glga_status st = encode_tmap_2d(&my, dt, Y, c->D, c->N, static_cast<uint64_t>(c->D) * c->elem,
                                        kt, kBM);
        if (st != GLGA_OK) return st;
    }
    const size_t smem = static_cast<size_t>(p.bres_bytes) + static_cast<size_t>(p.stages) * p.stage_bytes +
                        lbytes + 1024;
    const CUtensorMap &b1 = planes == 2 ? c->tmBro[1].map : c->tmBro[0].map;
    glga_status st =
        c->io == GLGA_F32
            ? launch_readout_r<3, float>(c, p, static_cast<unsigned>(grid), smem, c->tmQ.map,
                                         c->tmBro[0].map, b1, c->tmL.map, my, s)
            : launch_readout_r<1, __nv_bfloat16>(c, p, static_cast<unsigned>(grid), smem, c->tmQ.map,
                                                 c->tmBro[0].map, b1, c->tmL.map, my, s);
    if (st != GLGA_OK || c->n_fix == 0) return st;
    // rows in a later segment than their tile's first row: redo them with their own S, z
    const unsigned fgrid = static_cast<unsigned>(ceil_div(c->n_fix, kFixRowsPerBlock));
    if (c->io == GLGA_F32)
        readout_fixup_kernel<float><<<fgrid, 32 * kFixRowsPerBlock, 0, s>>>(
            c->fix_row, c->fix_seg, c->n_fix, static_cast<const float *>(c->Q),
            static_cast<const float *>(c->L), c->t, c->Sz, c->n_seg, c->H, c->r, b_g, eps,
            static_cast<float *>(Y));
    else
        readout_fixup_kernel<__nv_bfloat16><<<fgrid, 32 * kFixRowsPerBlock, 0, s>>>(
            c->fix_row, c->fix_seg, c->n_fix, static_cast<const __nv_bfloat16 *>(c->Q),
            static_cast<const __nv_bfloat16 *>(c->L), c->t, c->Sz, c->n_seg, c->H, c->r, b_g, eps,
            static_cast<__nv_bfloat16 *>(Y));
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    return GLGA_OK;
}

}  // namespace glga
