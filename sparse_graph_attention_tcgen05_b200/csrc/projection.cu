// projection.cu -- fused Q/K/V/gate projection on the tcgen05 tensor cores.
//
// One GEMM computes [Q | K | V | t] = X [W_Q | W_K | W_V | w_g] (method page "Gated
// Local-Global Graph Attention", Key formulas: q = x W_Q, k = x W_K, v = x W_V and the
// gate logit x w_g).  The weights are packed once per forward into one K-major operand
// Wt [rows][dp] (row c = output column c; rows past 3D+1 are zero).  Output columns
// [0, D) go to Q, [D, 3D) to KV (k_j | v_j per row, the layout the local kernel
// gathers), column 3D to the float32 gate logit t.
//
// Kernel shape: 128 x BN tiles (BN <= 256, one MMA per 32-byte K step), K tiles of 128
// bytes per row loaded by TMA with the 128-byte swizzle, an mbarrier ring of `stages`
// buffers, one elected thread issuing tcgen05.mma into a TMEM accumulator, and all four
// warps draining TMEM (tcgen05.ld 32x32b) into global memory.
//
// float32 I/O uses kind::tf32 with a 3-term split: every operand x is stored as
// hi = tf32(x) and lo = tf32(x - hi) and the accumulator receives hi*hi + hi*lo + lo*hi,
// which keeps ~2^-21 relative accuracy (plain tf32 would give ~2^-11).
//
// The same kernel also serves as a plain GEMM with a float32 output (gemm_nt_f32out):
// C [M][ncols] = A [M][K] B [ncols][K]^T, both operands K-major, bf16 on kind::f16 or
// float32 on kind::tf32 with one term (the backward pass's input gradient).
#include <algorithm>
#include <cstdio>

#include "glga_internal.cuh"

namespace glga {

namespace {
constexpr int kBM = 128;
constexpr int kRowBytes = 128;            // bytes of K per smem row (one swizzle span)
constexpr int kMaxStages = 6;
constexpr int kProdWarp = 8;             // TMA producer
constexpr int kMmaWarp = 9;              // TMEM owner and MMA issuer
constexpr int kGemmThreads = 320;        // warps 0-7 drain TMEM in the epilogue

struct GemmParams {
    int64_t M;
    int64_t n_total_tiles;   // m-tiles x n-tiles
    int32_t n_tiles;         // column tiles
    int32_t nk;          // K tiles
    int32_t BN;          // columns per tile (multiple of 16, <= 256)
    int32_t bn_last;     // columns of the last column tile (BN, or BN + 16 with the gate)
    int32_t tma_epi;     // 1: Q/K/V leave through smem + TMA stores (BN multiple of 64)
    int32_t sbufs;       // staging buffers of the TMA-store epilogue (1 or 2)
    uint32_t stage_area; // bytes of the stage ring (staging buffers follow it)
    int32_t stages;
    int32_t tmem_cols;
    int32_t D;
    uint32_t a_bytes, b_bytes, stage_bytes;
    void *Q;
    void *KV;
    float *t;
    float *C;            // plain GEMM: float32 output [M][ldc] (first ncols columns), else null
    int64_t ldc;
    int32_t ncols;
    unsigned *flag;
    // statistics in the epilogue (bf16, D = 128, heads inside 64-feature groups): column
    // tiles are [K_g | V_g] for the feature groups g, then [Q | gate]; each CTA walks whole
    // row blocks and accumulates phi(K_g)^T [V_g | 1] in TMEM across them
    int32_t fuse;
    int32_t groups;          // feature groups of 64 (KV column tiles)
    int32_t R;               // head width r
    uint32_t acc_stride;     // TMEM columns between the two projection accumulators
    uint32_t stats_col0;     // first TMEM column of the statistics accumulators
    float *part;             // [gridDim.x][H][r][r + 1] per-CTA partial sums
};

constexpr uint32_t kStatsCols = 96;      // TMEM columns per feature group: S (64) | z (16)
constexpr uint32_t kFusedAccStride = 160; // projection accumulators (<= 144 columns) when fused

// Tile i of this CTA: tiles blockIdx.x + i * gridDim.x of the row-major tile grid, or, when
// the statistics are fused, column tile i % n_tiles of row block blockIdx.x + (i / n_tiles)
// * gridDim.x (a CTA owns whole row blocks, so K_g and V_g of a row meet in one CTA).
__device__ __forceinline__ void tile_at(const GemmParams &p, int32_t i, int32_t &row, int32_t &col) {
    if (p.fuse) {
        row = static_cast<int32_t>(blockIdx.x) + (i / p.n_tiles) * static_cast<int32_t>(gridDim.x);
        col = i % p.n_tiles;
    } else {
        const int64_t t = static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(i) * gridDim.x;
        row = static_cast<int32_t>(t / p.n_tiles);
        col = static_cast<int32_t>(t % p.n_tiles);
    }
}


template <typename T>
__device__ __forceinline__ void store_vec32(T *dst, const uint32_t (&v)[32]);

template <>
__device__ __forceinline__ void store_vec32<float>(float *dst, const uint32_t (&v)[32]) {
    float4 *o = reinterpret_cast<float4 *>(dst);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        o[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                           __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

template <>
__device__ __forceinline__ void store_vec32<__nv_bfloat16>(__nv_bfloat16 *dst,
                                                           const uint32_t (&v)[32]) {
    uint4 *o = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 q;
        q.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
        q.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
        q.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
        q.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
        o[i] = q;
    }
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Routes 32 consecutive accumulator columns [gc0, gc0+32) of one row to Q / KV / t.
// Columns at or past n_end belong to the next column tile (or are padding) and are
// skipped: TMEM past the tile's width holds no MMA result.
template <typename T>
__device__ __forceinline__ void store_row_cols(const GemmParams &p, int64_t row, int gc0,
                                               int n_end, const uint32_t (&v)[32]) {
    const int D = p.D;
    T *Q = static_cast<T *>(p.Q);
    T *KV = static_cast<T *>(p.KV);
    const bool whole = gc0 + 32 <= n_end;
    if (whole && gc0 + 32 <= D) {
        store_vec32<T>(Q + row * D + gc0, v);
    } else if (whole && gc0 >= D && gc0 + 32 <= 3 * D) {
        store_vec32<T>(KV + row * 2 * D + (gc0 - D), v);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int gc = gc0 + j;
            const float x = __uint_as_float(v[j]);
            if (gc >= n_end)
                continue;
            if (gc < D)
                Q[row * D + gc] = from_f32<T>(x);
            else if (gc < 3 * D)
                KV[row * 2 * D + (gc - D)] = from_f32<T>(x);
            else if (gc == 3 * D)
                p.t[row] = x;
        }
    }
}

// Persistent: CTA b walks tiles b, b + gridDim.x, ... (tile t = m-tile t / n_tiles,
// n-tile t % n_tiles).  The producer streams every K block of every tile through the
// stage ring; the MMA warp accumulates tile i into TMEM buffer i & 1 (256 columns each)
// once the epilogue has drained that buffer's previous tile; warps 0-7 drain buffer
// i & 1 while tile i + 1 accumulates in the other one.
// SPLIT = 1: bf16 operands, one MMA per K step.  SPLIT = 3: tf32 hi/lo planes.
template <int SPLIT, typename T>
__global__ void __launch_bounds__(kGemmThreads, 1) proj_gemm_kernel(
    const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
    const __grid_constant__ CUtensorMap tmQs, const __grid_constant__ CUtensorMap tmKVs,
    GemmParams p) {
    constexpr int kPlanes = SPLIT == 3 ? 2 : 1;
    constexpr int kPairs = SPLIT == 3 ? 3 : 1;
    constexpr uint32_t kFmt = sizeof(T) == 4 ? 2u : 1u;   // tf32 or bf16 operands

    extern __shared__ uint8_t dsmem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2];    // MMA -> epilogue: buffer holds a tile
    __shared__ __align__(8) uint64_t acce_bar[2];    // epilogue -> MMA: buffer drained
    __shared__ __align__(8) uint64_t staged_bar[2];  // epilogue -> MMA: staging b written (fused)
    __shared__ __align__(8) uint64_t sdone_bar[2];   // MMA -> epilogue: staging b read (fused)
    __shared__ uint32_t tmem_base_sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t n_my;
    if (p.fuse) {
        const int64_t nrb = p.n_total_tiles / p.n_tiles;   // row blocks
        n_my = nrb > blockIdx.x ? static_cast<int32_t>((nrb - blockIdx.x + gridDim.x - 1) / gridDim.x) * p.n_tiles
                                : 0;
    } else {
        n_my = p.n_total_tiles > blockIdx.x
                   ? static_cast<int32_t>((p.n_total_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x)
                   : 0;
    }
    const uint32_t box_bytes = kBM * kRowBytes;          // one 128-row x 64-column bf16 box
    // fused statistics: two staging buffers of three boxes each (K_g | phi(K_g) | V_g, or
    // the two Q boxes; tile i uses buffer i & 1), then the "ones" operand of the z MMA
    uint8_t *ones = smem + p.stage_area + 6 * box_bytes;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf_bar[b], 1);
            mbar_init(&acce_bar[b], 8);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&staged_bar[b], 8);
            mbar_init(&sdone_bar[b], 1);
        }
        fence_mbar_init();
    }
    if (p.fuse && threadIdx.x < 256) {
        // ones tile (16 rows of 128 bytes, K-major): row 0 = 1.0, rows 1..15 = 0; the
        // swizzle permutes 16-byte chunks inside a row only, so row 0 reads as ones at
        // every K offset
        uint32_t *o = reinterpret_cast<uint32_t *>(ones);
        for (int k = threadIdx.x; k < 16 * kRowBytes / 4; k += 256) o[k] = k < kRowBytes / 4 ? 0x3F803F80u : 0u;
        fence_proxy_async_smem();
    }
    if (warp == kProdWarp && lane == 0) {
        tma_prefetch_desc(&tmA0);
        tma_prefetch_desc(&tmB0);
        if (kPlanes == 2) {
            tma_prefetch_desc(&tmA1);
            tma_prefetch_desc(&tmB1);
        }
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_base_sh, static_cast<uint32_t>(p.tmem_cols));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kProdWarp && lane == 0) {
        // ---------------- TMA producer: every K block of every tile of this CTA ----------
        int it = 0;           // K blocks issued so far
        RingPos rp;           // stage ring position
        bool ok = true;
        for (int i = 0; i < n_my && ok; ++i) {
            int32_t trow, tcol;
            tile_at(p, i, trow, tcol);
            const int32_t m0 = trow * kBM;
            const int32_t n0 = tcol * p.BN;
            for (int kb = 0; kb < p.nk; ++kb, ++it, rp.next(p.stages)) {
                const int s = rp.slot;
                if (it >= p.stages && !mbar_wait_bounded(&empty_bar[s], rp.phase ^ 1u)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
                mbar_arrive_expect_tx(&full_bar[s], p.stage_bytes);
                const int kx = kb * (kRowBytes / static_cast<int>(sizeof(T)));
                tma_load_2d(st, &tmA0, &full_bar[s], kx, m0);
                if (kPlanes == 2) tma_load_2d(st + p.a_bytes, &tmA1, &full_bar[s], kx, m0);
                uint8_t *bst = st + kPlanes * p.a_bytes;
                tma_load_2d(bst, &tmB0, &full_bar[s], kx, n0);
                if (kPlanes == 2) tma_load_2d(bst + p.b_bytes, &tmB1, &full_bar[s], kx, n0);
            }
        }
        if (!ok) {
            atomicOr(p.flag, kDevErrTimeout);
            // let the copies already in flight land before the block can exit
            for (int k = std::max(0, it - p.stages); k < it; ++k)
                mbar_wait_bounded(&full_bar[k % p.stages], static_cast<uint32_t>(k / p.stages) & 1u);
        }
    } else if (warp == kMmaWarp && lane == 0) {
        // ---------------- MMA issuer ----------------
        const uint32_t idesc_main = instr_desc(kBM, p.BN, kFmt, false, false);
        const uint32_t idesc_last = instr_desc(kBM, p.bn_last, kFmt, false, false);
        // fused statistics of tile j (its staging buffer is written): for a [K_g | V_g]
        // tile, S_g += phi(K_g)^T V_g and z_g += phi(K_g)^T 1 with the node rows as the
        // contraction; A = [phi(K_g) | V_g] (M = 128, MN-major, the upper 64 rows of the
        // product are not used), B = V_g (N = 64, MN-major) and the ones tile (N = 16)
        const uint32_t idS = instr_desc(128, 64, 1u, true, true);
        const uint32_t idZ = instr_desc(128, 16, 1u, true, false);
        auto stats_step = [&](int32_t j) -> bool {
            // staging buffer j & 1 is written for the (j >> 1)-th time
            if (!mbar_wait_bounded(&staged_bar[j & 1], static_cast<uint32_t>(j >> 1) & 1u)) return false;
            tc_fence_after();
            const int32_t col = j % p.n_tiles;
            if (col < p.groups) {
                const uint32_t sbase = smem_u32(smem + p.stage_area + (j & 1) * 3 * box_bytes);
                const uint32_t acc_s = tmem + p.stats_col0 + static_cast<uint32_t>(col) * kStatsCols;
                const uint64_t dones = smem_desc(smem_u32(ones), 16, 1024, 2);
#pragma unroll
                for (int ks = 0; ks < kBM / 16; ++ks) {
                    const uint64_t ad = smem_desc(sbase + box_bytes + ks * 16 * kRowBytes, box_bytes, 1024, 2);
                    const uint64_t bd = smem_desc(sbase + 2 * box_bytes + ks * 16 * kRowBytes, box_bytes, 1024, 2);
                    const uint32_t acc = (j >= p.n_tiles || ks > 0) ? 1u : 0u;
                    umma_bf16(acc_s, ad, bd, idS, acc);
                    umma_bf16(acc_s + 64, ad, dones, idZ, acc);
                }
            }
            umma_commit(&sdone_bar[j & 1]);   // the staging buffer may be rewritten
            return true;
        };
        bool ok = true;
        RingPos rp;
        for (int i = 0; i < n_my && ok; ++i) {
            int32_t trow, tcol;
            tile_at(p, i, trow, tcol);
            (void)trow;
            const int buf = i & 1;
            const uint32_t acc_col = static_cast<uint32_t>(buf) * p.acc_stride;
            const uint32_t idesc = (tcol == p.n_tiles - 1) ? idesc_last : idesc_main;
            // wait until the epilogue drained this buffer's previous tile (tile i - 2)
            if (i >= 2 && !mbar_wait_bounded(&acce_bar[buf], static_cast<uint32_t>((i >> 1) - 1) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int kb = 0; kb < p.nk; ++kb, rp.next(p.stages)) {
                const int s = rp.slot;
                if (!mbar_wait_bounded(&full_bar[s], rp.phase)) {
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
                        const uint32_t ap = (pr == 2) ? 1u : 0u;   // (hi,hi) (hi,lo) (lo,hi)
                        const uint32_t bp = (pr == 1) ? 1u : 0u;
                        const uint64_t ad = smem_desc(a_addr + ap * p.a_bytes + k * 32, 16, 1024, 2);
                        const uint64_t bd = smem_desc(b_addr + bp * p.b_bytes + k * 32, 16, 1024, 2);
                        const uint32_t acc = (kb | k | pr) != 0;
                        if (SPLIT == 3)
                            umma_tf32(tmem + acc_col, ad, bd, idesc, acc);
                        else
                            umma_bf16(tmem + acc_col, ad, bd, idesc, acc);
                    }
                }
                umma_commit(&empty_bar[s]);   // stage reusable once these MMAs finish
            }
            if (ok) umma_commit(&accf_bar[buf]);   // the tile's accumulator is complete
            // the previous tile's statistics, while this tile's MMAs run
            if (ok && p.fuse && i >= 1 && !stats_step(i - 1)) ok = false;
        }
        if (ok && p.fuse && n_my > 0 && !stats_step(n_my - 1)) ok = false;
        if (!ok) atomicOr(p.flag, kDevErrTimeout);
    }
    __syncwarp();

    // ---------------- epilogue (warps 0-7): TMEM -> registers -> Q / KV / t ----------------
    // warp w drains TMEM lanes 32*(w%4).. (its rows); warpgroup w/4 takes every other
    // 32-column chunk
    if (warp < 8) {
        const int quad = warp & 3, wg = warp >> 2;
        const int rt = quad * 32 + lane;                 // row inside the tile
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const int nbox = p.BN / 64;
        bool ok = true;
        for (int i = 0; i < n_my; ++i) {
            int32_t trow, tcol;
            tile_at(p, i, trow, tcol);
            const int buf = i & 1;
            const uint32_t acc = tmem + lane_base + static_cast<uint32_t>(buf) * p.acc_stride;
            // no barrier spans the epilogue warps: each warp agrees on its own wait (the
            // TMEM loads below are warp-collective)
            const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&accf_bar[buf], static_cast<uint32_t>(i >> 1) & 1u));
            if (!got) {
                if (lane == 0) atomicOr(p.flag, kDevErrTimeout);
                ok = false;
                break;
            }
            tc_fence_after();
            const int64_t m0 = static_cast<int64_t>(trow) * kBM;
            const int64_t row = m0 + rt;
            const int ntile = tcol;
            const int n0 = ntile * p.BN;
            const int bn = ntile == p.n_tiles - 1 ? p.bn_last : p.BN;
            if (p.C) {
                // plain GEMM: float32 rows of C, columns below ncols
                for (int c0 = wg * 32; c0 < bn; c0 += 64) {
                    uint32_t v[32];
                    tmem_ld32(acc + static_cast<uint32_t>(c0), v);
                    tmem_ld_wait();
                    const int gc0 = n0 + c0;
                    if (row < p.M) {
                        float *crow = p.C + row * p.ldc + gc0;
                        if (gc0 + 32 <= p.ncols && (p.ldc & 3) == 0) {
                            store_vec32<float>(crow, v);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (gc0 + j < p.ncols) crow[j] = __uint_as_float(v[j]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce_bar[buf]);
            } else if (p.fuse) {
                // Staging buffer i & 1 of three boxes.  [K_g | V_g] tile: warpgroup g & 1
                // stages K_g (box 0) and phi(K_g) (box 1, zero past row M), the other V_g
                // (box 2); [Q | gate] tile: warpgroup w stages Q box w, warpgroup 1 the gate
                // column.  A buffer is rewritten only after the statistics MMAs of its
                // previous tile (i - 2) and this warp's TMA stores out of it have read it.
                uint8_t *sb = smem + p.stage_area + buf * 3 * box_bytes;
                if (i >= 2 && !__all_sync(0xffffffffu, mbar_wait_bounded(&sdone_bar[buf], static_cast<uint32_t>((i >> 1) - 1) & 1u))) {
                    if (lane == 0) atomicOr(p.flag, kDevErrTimeout);
                    ok = false;
                    break;
                }
                if (lane == 0) bulk_wait_group_read1();   // (the other buffer's stores may still run)
                __syncwarp();
                const bool kv = ntile < p.groups;
                const bool kwarp = kv && wg == (ntile & 1);
                const int box = kv ? (kwarp ? 0 : 2) : wg;
                const uint32_t c_src = kv ? (kwarp ? 0u : 64u) : static_cast<uint32_t>(wg * 64);
                const bool valid = row < p.M;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t v[32];
                    tmem_ld32(acc + c_src + static_cast<uint32_t>(half * 32), v);
                    tmem_ld_wait();
                    uint8_t *rp = sb + box * box_bytes + rt * kRowBytes;
                    uint8_t *fp = sb + box_bytes + rt * kRowBytes;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = pack_bf16x2(__uint_as_float(v[8 * q + 2 * e]), __uint_as_float(v[8 * q + 2 * e + 1]));
                        const int chunk = ((half * 4 + q) ^ (rt & 7)) * 16;
                        *reinterpret_cast<uint4 *>(rp + chunk) = make_uint4(w[0], w[1], w[2], w[3]);
                        if (kwarp) {
                            // phi of the stored (bf16) k, as the statistics kernel forms it;
                            // rows past M contribute nothing to z
#pragma unroll
                            for (int e = 0; e < 4; ++e) w[e] = valid ? phi_bf16x2(w[e]) : 0u;
                            *reinterpret_cast<uint4 *>(fp + chunk) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                if (!kv && wg == 1) {
                    uint32_t v[32];
                    tmem_ld32(acc + static_cast<uint32_t>(p.BN), v);
                    tmem_ld_wait();
                    if (valid) p.t[row] = __uint_as_float(v[0]);   // gate logit column
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce_bar[buf]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int64_t y = m0 + quad * 32;
                    if (y < p.M) {
                        const uint8_t *src = sb + box * box_bytes + quad * 32 * kRowBytes;
                        if (kv)
                            tma_store_2d(&tmKVs, src, (kwarp ? 0 : p.D) + ntile * 64, static_cast<int32_t>(y));
                        else
                            tma_store_2d(&tmQs, src, wg * 64, static_cast<int32_t>(y));
                    }
                    bulk_commit_group();
                    mbar_arrive(&staged_bar[buf]);   // phi(K_g) and V_g are in place for the MMA
                }
            } else if (p.tma_epi) {
                // Each warp owns whole 64-column boxes of its 32 rows (boxes wg, wg + 2, ...;
                // in the last column tile warpgroup 1 also takes the gate column past them):
                // it stages them in shared memory (buffer i & 1 when there are two) and
                // stores them with its own TMA bulk stores, waiting only for its own
                // earlier stores out of that buffer, so no barrier spans the warps.
                const int sbuf = p.sbufs == 2 ? buf : 0;
                uint8_t *sb = smem + p.stage_area + static_cast<size_t>(sbuf) * nbox * box_bytes;
                if (lane == 0) {
                    if (p.sbufs == 2)
                        bulk_wait_group_read1();
                    else
                        bulk_wait_group_read0();
                }
                __syncwarp();
                for (int b = wg; b < nbox; b += 2) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t v[32];
                        tmem_ld32(acc + static_cast<uint32_t>(b * 64 + half * 32), v);
                        tmem_ld_wait();
                        uint8_t *rp = sb + b * box_bytes + rt * kRowBytes;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                            w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                            w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                            w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                            *reinterpret_cast<uint4 *>(rp + (((half * 4 + q) ^ (rt & 7)) * 16)) = w;
                        }
                    }
                }
                if (bn > p.BN && wg == 1) {
                    uint32_t v[32];
                    tmem_ld32(acc + static_cast<uint32_t>(p.BN), v);
                    tmem_ld_wait();
                    if (row < p.M) p.t[row] = __uint_as_float(v[0]);   // gate logit column
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce_bar[buf]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int64_t y = m0 + quad * 32;
                    for (int b = wg; b < nbox && y < p.M; b += 2) {
                        const int gc = n0 + b * 64;
                        const uint8_t *src = sb + b * box_bytes + quad * 32 * kRowBytes;
                        if (gc < p.D)
                            tma_store_2d(&tmQs, src, gc, static_cast<int32_t>(y));
                        else
                            tma_store_2d(&tmKVs, src, gc - p.D, static_cast<int32_t>(y));
                    }
                    bulk_commit_group();
                }
            } else {
                for (int c0 = wg * 32; c0 < bn; c0 += 64) {
                    uint32_t v[32];
                    tmem_ld32(acc + static_cast<uint32_t>(c0), v);
                    tmem_ld_wait();
                    if (row < p.M) store_row_cols<T>(p, row, n0 + c0, n0 + bn, v);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce_bar[buf]);
            }
        }
        if (p.fuse && quad < 2 && wg < p.groups) {
            // this CTA's statistics: warps of quads 0-1 in warpgroup g read feature group g
            // (TMEM lanes = its 64 features) and write the rows of their heads' blocks
            const int g = wg;
            const int f = g * 64 + quad * 32 + lane;            // feature
            const int h = f / p.R;
            const int hc0 = h * p.R - g * 64;                   // the head's first V column
            uint32_t s0[32], s1[32], zv[32];
            // the last tile's commit follows every statistics MMA of the CTA
            const int32_t jl = n_my - 1;
            const bool got = ok && n_my > 0 &&
                             __all_sync(0xffffffffu, mbar_wait_bounded(&sdone_bar[jl & 1], static_cast<uint32_t>(jl >> 1) & 1u));
            if (ok && n_my > 0 && !got && lane == 0) atomicOr(p.flag, kDevErrTimeout);
            tc_fence_after();
            const uint32_t acc_s = tmem + lane_base + p.stats_col0 + static_cast<uint32_t>(g) * kStatsCols;
            tmem_ld32(acc_s, s0);
            tmem_ld32(acc_s + 32, s1);
            tmem_ld32(acc_s + 64, zv);
            tmem_ld_wait();
            float *dst = p.part + (static_cast<int64_t>(blockIdx.x) * p.D + f) * (p.R + 1);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if (j >= hc0 && j < hc0 + p.R) dst[j - hc0] = got ? __uint_as_float(s0[j]) : 0.f;
                if (j + 32 >= hc0 && j + 32 < hc0 + p.R) dst[j + 32 - hc0] = got ? __uint_as_float(s1[j]) : 0.f;
            }
            dst[p.R] = got ? __uint_as_float(zv[0]) : 0.f;
        }
        if ((p.tma_epi || p.fuse) && lane == 0) bulk_wait_group_read0();   // shared memory outlives the stores
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
    }
}

// ---------------------------------------------------------------------------------------
// operand preparation
// ---------------------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float ld_f32(const T *p);
template <>
__device__ __forceinline__ float ld_f32<float>(const float *p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
}

// Wt[c][k] (k < dp, c < rows): the packed K-major weight operand.
template <int SPLIT, typename T>
__global__ void pack_weights_kernel(const T *__restrict__ WQ, const T *__restrict__ WK,
                                    const T *__restrict__ WV, const T *__restrict__ wg, int d,
                                    int D, int dp, int rows, int fused, T *__restrict__ Wt) {
    const int64_t total = static_cast<int64_t>(rows) * dp;
    const int64_t plane = total;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(idx / dp);
        const int k = static_cast<int>(idx % dp);
        float v = 0.f;
        if (k < d && fused && c < 2 * D) {
            // [K_g | V_g] for the 64-feature groups g, then Q and the gate
            const int g = c / 128, w = c % 128;
            const T *src = w < 64 ? WK : WV;
            v = ld_f32<T>(src + static_cast<int64_t>(k) * D + g * 64 + (w & 63));
        } else if (k < d && fused) {
            if (c < 3 * D)
                v = ld_f32<T>(WQ + static_cast<int64_t>(k) * D + (c - 2 * D));
            else if (c == 3 * D)
                v = ld_f32<T>(wg + k);
        } else if (k < d) {
            if (c < D)
                v = ld_f32<T>(WQ + static_cast<int64_t>(k) * D + c);
            else if (c < 2 * D)
                v = ld_f32<T>(WK + static_cast<int64_t>(k) * D + (c - D));
            else if (c < 3 * D)
                v = ld_f32<T>(WV + static_cast<int64_t>(k) * D + (c - 2 * D));
            else if (c == 3 * D)
                v = ld_f32<T>(wg + k);
        }
        if (SPLIT == 3) {
            const float hi = to_tf32(v);
            Wt[idx] = from_f32<T>(hi);
            Wt[plane + idx] = from_f32<T>(to_tf32(v - hi));
        } else {
            Wt[idx] = from_f32<T>(v);
        }
    }
}

// Xp[i][k] (k < dp): zero-padded copy of X (and its tf32 hi/lo split for SPLIT = 3).
template <int SPLIT, typename T>
__global__ void prep_x_kernel(const T *__restrict__ X, int64_t N, int d, int dp,
                              T *__restrict__ Xp) {
    const int64_t total = N * dp;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = idx / dp;
        const int k = static_cast<int>(idx % dp);
        const float v = k < d ? ld_f32<T>(X + i * d + k) : 0.f;
        if (SPLIT == 3) {
            const float hi = to_tf32(v);
            Xp[idx] = from_f32<T>(hi);
            Xp[total + idx] = from_f32<T>(to_tf32(v - hi));
        } else {
            Xp[idx] = from_f32<T>(v);
        }
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

template <int SPLIT, typename T>
glga_status launch_gemm(Ctx *c, cudaStream_t s) {
    GemmParams p;
    p.M = c->N;
    p.n_tiles = c->n_tiles;
    p.n_total_tiles = ceil_div(c->N, kBM) * c->n_tiles;
    p.nk = c->dp / (kRowBytes / c->elem);
    p.BN = c->BN;
    p.bn_last = c->bn_last;
    p.tma_epi = c->gemm_tma_epi ? 1 : 0;
    p.sbufs = c->gemm_sbufs;
    p.stages = c->stages;
    p.tmem_cols = c->tmem_cols;   // two 256-column accumulators
    p.D = c->D;
    const int planes = SPLIT == 3 ? 2 : 1;
    p.a_bytes = kBM * kRowBytes;
    p.b_bytes = static_cast<uint32_t>(c->bn_last) * kRowBytes;
    p.stage_bytes = planes * (p.a_bytes + p.b_bytes);
    p.stage_area = static_cast<uint32_t>(p.stages) * p.stage_bytes;
    p.Q = c->Q;
    p.KV = c->kv_own;
    p.t = c->t;
    p.C = nullptr;
    p.ldc = 0;
    p.ncols = 0;
    p.flag = c->dev_flag;
    p.fuse = c->stats_fused ? 1 : 0;
    p.groups = c->stats_fused ? c->D / 64 : 0;
    p.R = c->r;
    p.acc_stride = c->stats_fused ? kFusedAccStride : 256u;
    p.stats_col0 = 2 * kFusedAccStride;
    p.part = c->Spart;
    // fused: two staging buffers of three boxes and the 2 KB ones tile
    const uint32_t staging = c->stats_fused ? 6u * kBM * kRowBytes + 2048u
                             : p.tma_epi ? static_cast<uint32_t>(p.sbufs) * (c->BN / 64) * kBM * kRowBytes : 0u;
    const size_t smem = static_cast<size_t>(p.stage_area) + staging + 1024;
    auto kern = proj_gemm_kernel<SPLIT, T>;
    GLGA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem)));
    // persistent: one CTA per SM (it holds all 512 TMEM columns); fused statistics give
    // each CTA whole row blocks
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(
        c->stats_fused ? p.n_total_tiles / p.n_tiles : p.n_total_tiles, c->num_sms));
    const CUtensorMap &a1 = planes == 2 ? c->tmA[1].map : c->tmA[0].map;
    const CUtensorMap &b1 = planes == 2 ? c->tmB[1].map : c->tmB[0].map;
    const CUtensorMap &qs = c->gemm_tma_epi ? c->tmQs.map : c->tmB[0].map;     // unused otherwise
    const CUtensorMap &kvs = c->gemm_tma_epi ? c->tmKVs.map : c->tmB[0].map;
    kern<<<grid, kGemmThreads, smem, s>>>(c->tmA[0].map, a1, c->tmB[0].map, b1, qs, kvs, p);
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    return GLGA_OK;
}

}  // namespace

glga_status gemm_nt_f32out(Ctx *c, glga_dtype t, const void *A, int64_t M, int64_t lda, const void *B,
                           int64_t ncols, int64_t ldb, int64_t K, float *C, int64_t ldc, cudaStream_t s) {
    if (M <= 0 || ncols <= 0) return GLGA_OK;
    const int elem = t == GLGA_F32 ? 4 : 2;
    const int kt = kRowBytes / elem;                      // K elements per tile row
    if ((lda * elem) % 16 || (ldb * elem) % 16 || K < 1 || K > lda || K > ldb || ncols > 1 << 20) {
        set_error("gemm_nt_f32out: operand rows must be 16-byte multiples and hold K elements");
        return GLGA_ERR_INVALID_ARG;
    }
    GemmParams p;
    p.M = M;
    p.BN = static_cast<int32_t>(std::min<int64_t>(256, ceil_div(ncols, 16) * 16));
    p.n_tiles = static_cast<int32_t>(ceil_div(ncols, p.BN));
    p.bn_last = static_cast<int32_t>(ceil_div(ncols - static_cast<int64_t>(p.n_tiles - 1) * p.BN, 16) * 16);
    p.n_total_tiles = ceil_div(M, kBM) * p.n_tiles;
    p.nk = static_cast<int32_t>(ceil_div(K, kt));
    p.tma_epi = 0;
    p.sbufs = 1;
    p.tmem_cols = 512;
    p.D = 0;
    p.a_bytes = kBM * kRowBytes;
    p.b_bytes = static_cast<uint32_t>(p.BN) * kRowBytes;
    p.stage_bytes = p.a_bytes + p.b_bytes;
    p.stages = std::max(1, std::min(kMaxStages, static_cast<int>((220u * 1024u) / p.stage_bytes)));
    p.stage_area = static_cast<uint32_t>(p.stages) * p.stage_bytes;
    p.Q = p.KV = nullptr;
    p.t = nullptr;
    p.C = C;
    p.ldc = ldc;
    p.ncols = static_cast<int32_t>(ncols);
    p.flag = c->dev_flag;
    p.fuse = 0;
    p.groups = 0;
    p.R = 0;
    p.acc_stride = 256;
    p.stats_col0 = 0;
    p.part = nullptr;
    const CUtensorMapDataType dt = t == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap ma, mb;
    glga_status r = encode_tmap_2d(&ma, dt, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                                   static_cast<uint64_t>(lda) * elem, kt, kBM);
    if (r == GLGA_OK)
        r = encode_tmap_2d(&mb, dt, B, static_cast<uint64_t>(K), static_cast<uint64_t>(ncols),
                           static_cast<uint64_t>(ldb) * elem, kt, static_cast<uint32_t>(p.BN));
    if (r != GLGA_OK) return r;
    const size_t smem = static_cast<size_t>(p.stage_area) + 1024;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(p.n_total_tiles, c->num_sms));
    if (t == GLGA_F32) {
        auto kern = proj_gemm_kernel<1, float>;
        GLGA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
        kern<<<grid, kGemmThreads, smem, s>>>(ma, ma, mb, mb, mb, mb, p);
    } else {
        auto kern = proj_gemm_kernel<1, __nv_bfloat16>;
        GLGA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
        kern<<<grid, kGemmThreads, smem, s>>>(ma, ma, mb, mb, mb, mb, p);
    }
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

glga_status encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base,
                           uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                           uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        set_error("cuTensorMapEncodeTiled unavailable from the driver");
        return GLGA_ERR_CUDA;
    }
    if ((reinterpret_cast<uintptr_t>(base) & 15u) || (row_bytes & 15u)) {
        set_error("tensor map base/stride not 16-byte aligned");
        return GLGA_ERR_INVALID_ARG;
    }
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) dims=%llu,%llu box=%u,%u", static_cast<int>(r),
                  static_cast<unsigned long long>(inner), static_cast<unsigned long long>(outer),
                  box_inner, box_outer);
        return GLGA_ERR_CUDA;
    }
    return GLGA_OK;
}

glga_status projection_setup(Ctx *c) {
    c->split = (c->io == GLGA_F32) ? 3 : 1;
    const int kt = kRowBytes / c->elem;                  // K elements per tile row
    c->dp = static_cast<int32_t>(ceil_div(c->d, kt) * kt);
    const int D3 = 3 * c->D;
    c->gemm_tma_epi = false;
    // global statistics in the epilogue (on request): bf16, D = 128 (two 64-feature
    // groups), heads inside a group, one segment
    c->stats_fused = c->opts.fuse_stats && c->split == 1 && c->D == 128 && 64 % c->r == 0 &&
                     c->n_seg == 1 && c->N > 0;
    c->stats_fused_parts = c->stats_fused ? static_cast<int32_t>(std::min<int64_t>(ceil_div(c->N, kBM), c->num_sms)) : 0;
    if (c->stats_fused) {
        // column tiles [K_0 | V_0], [K_1 | V_1], [Q | gate + 15 zero columns]
        c->BN = 128;
        c->n_tiles = 3;
        c->bn_last = c->BN + 16;
        c->Dp = D3 + 16;
        c->gemm_tma_epi = true;
    } else if (c->split == 1 && c->D % 64 == 0) {
        // Column tiles of BN (a multiple of the 64-column store box) over Q | K | V; the
        // last tile also carries the gate column (+15 zero columns).  Q/K/V leave through
        // shared memory and TMA stores.
        c->BN = 64;
        for (int bn = 192; bn >= 64; bn -= 64)
            if (D3 % bn == 0) {
                c->BN = bn;
                break;
            }
        c->n_tiles = D3 / c->BN;
        c->bn_last = c->BN + 16;
        c->Dp = D3 + 16;
        c->gemm_tma_epi = true;
    } else {
        const int Dp = D3 + 1;
        c->n_tiles = static_cast<int32_t>(ceil_div(Dp, 256));
        c->BN = static_cast<int32_t>(ceil_div(ceil_div(Dp, c->n_tiles), 16) * 16);
        c->bn_last = c->BN;
        c->Dp = c->n_tiles * c->BN;
    }
    c->tmem_cols = 512;
    const int planes = c->split == 3 ? 2 : 1;
    const uint32_t stage_bytes = planes * (kBM * kRowBytes + c->bn_last * kRowBytes);
    // One persistent CTA per SM: as many ring stages as fit beside the epilogue's staging
    // buffers (loads run ahead across tiles).  Two staging buffers let a tile's TMA store
    // overlap the next tile's epilogue; one is used when two would leave fewer than four
    // ring stages, since the operand loads in flight bound the MMA rate.
    constexpr uint32_t kBudget = 220u * 1024u;
    // (fused statistics: always two buffers of three boxes, plus the 2 KB ones tile)
    const uint32_t stg1 = c->stats_fused ? 3u * kBM * kRowBytes
                          : c->gemm_tma_epi ? (c->BN / 64) * kBM * kRowBytes : 0u;
    c->gemm_sbufs = c->stats_fused || (kBudget - 2u * stg1) / stage_bytes >= 4u ? 2 : 1;
    const uint32_t budget = kBudget - static_cast<uint32_t>(c->gemm_sbufs) * stg1 - (c->stats_fused ? 2048u : 0u);
    int st = static_cast<int>(budget / stage_bytes);
    c->stages = std::max(1, std::min(st, kMaxStages));

    const size_t wt_bytes = static_cast<size_t>(planes) * c->Dp * c->dp * c->elem;
    glga_status r = dev_alloc(c, &c->Wt, wt_bytes);
    if (r != GLGA_OK) return r;
    const CUtensorMapDataType dt =
        c->io == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    for (int pl = 0; pl < planes; ++pl) {
        const uint8_t *base = static_cast<const uint8_t *>(c->Wt) +
                              static_cast<size_t>(pl) * c->Dp * c->dp * c->elem;
        r = encode_tmap_2d(&c->tmB[pl].map, dt, base, c->dp, c->Dp,
                           static_cast<uint64_t>(c->dp) * c->elem, kt, c->bn_last);
        if (r != GLGA_OK) return r;
        c->tmB[pl].valid = true;
    }
    if (c->gemm_tma_epi && c->N > 0) {
        // store maps: 64-column x 32-row boxes, one per epilogue warp and box
        r = encode_tmap_2d(&c->tmKVs.map, dt, c->kv_own, 2 * static_cast<uint64_t>(c->D), c->N,
                           2 * static_cast<uint64_t>(c->D) * c->elem, 64, 32);
        if (r != GLGA_OK) return r;
        c->tmKVs.valid = true;
        r = encode_tmap_2d(&c->tmQs.map, dt, c->Q, static_cast<uint64_t>(c->D), c->N,
                           static_cast<uint64_t>(c->D) * c->elem, 64, 32);
        if (r != GLGA_OK) return r;
        c->tmQs.valid = true;
    }
    // The A operand is read from the caller's X when it is bf16 with 16-byte rows;
    // otherwise from a padded (and, for fp32, split) copy.
    c->x_direct = (c->split == 1) && ((static_cast<int64_t>(c->d) * c->elem) % 16 == 0);
    if (!c->x_direct && c->N > 0) {
        const size_t xp_bytes = static_cast<size_t>(planes) * c->N * c->dp * c->elem;
        r = dev_alloc(c, &c->Xp, xp_bytes);
        if (r != GLGA_OK) return r;
        for (int pl = 0; pl < planes; ++pl) {
            const uint8_t *base = static_cast<const uint8_t *>(c->Xp) +
                                  static_cast<size_t>(pl) * c->N * c->dp * c->elem;
            r = encode_tmap_2d(&c->tmA[pl].map, dt, base, c->dp, c->N,
                               static_cast<uint64_t>(c->dp) * c->elem, kt, kBM);
            if (r != GLGA_OK) return r;
            c->tmA[pl].valid = true;
        }
    }
    return GLGA_OK;
}

glga_status projection_run(Ctx *c, const void *X, const void *WQ, const void *WK, const void *WV,
                           const void *wg, cudaStream_t s, bool time_prep) {
    (void)time_prep;
    const int64_t wt_total = static_cast<int64_t>(c->Dp) * c->dp;
    const unsigned wblocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(wt_total, 256), 2048));
    if (c->io == GLGA_F32) {
        pack_weights_kernel<3, float><<<wblocks, 256, 0, s>>>(
            static_cast<const float *>(WQ), static_cast<const float *>(WK),
            static_cast<const float *>(WV), static_cast<const float *>(wg), c->d, c->D, c->dp,
            c->Dp, 0, static_cast<float *>(c->Wt));
    } else {
        pack_weights_kernel<1, __nv_bfloat16><<<wblocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(WQ), static_cast<const __nv_bfloat16 *>(WK),
            static_cast<const __nv_bfloat16 *>(WV), static_cast<const __nv_bfloat16 *>(wg), c->d,
            c->D, c->dp, c->Dp, c->stats_fused ? 1 : 0, static_cast<__nv_bfloat16 *>(c->Wt));
    }
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    if (c->N == 0) {
        if (c->timing) GLGA_CUDA(record_stage(c, kStageGemm, s));
        return GLGA_OK;
    }
    const CUtensorMapDataType dt =
        c->io == GLGA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (c->x_direct) {
        glga_status r = encode_tmap_2d(&c->tmA[0].map, dt, X, c->d, c->N,
                                       static_cast<uint64_t>(c->d) * c->elem,
                                       kRowBytes / c->elem, kBM);
        if (r != GLGA_OK) return r;
        c->tmA[0].valid = true;
    } else {
        const int64_t total = c->N * c->dp;
        const unsigned xblocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(total, 256), 8192));
        if (c->io == GLGA_F32)
            prep_x_kernel<3, float><<<xblocks, 256, 0, s>>>(static_cast<const float *>(X), c->N,
                                                            c->d, c->dp, static_cast<float *>(c->Xp));
        else
            prep_x_kernel<1, __nv_bfloat16><<<xblocks, 256, 0, s>>>(
                static_cast<const __nv_bfloat16 *>(X), c->N, c->d, c->dp,
                static_cast<__nv_bfloat16 *>(c->Xp));
        GLGA_CUDA(cudaGetLastError());
        c->launches += 1;
    }
    if (c->timing) GLGA_CUDA(record_stage(c, kStageGemm, s));
    if (c->io == GLGA_F32) return launch_gemm<3, float>(c, s);
    return launch_gemm<1, __nv_bfloat16>(c, s);
}

}  // namespace glga
