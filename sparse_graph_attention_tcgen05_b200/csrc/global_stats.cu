// global_stats.cu -- global statistics of the linear-attention branch on tensor cores.
//
// Method page "Gated Local-Global Graph Attention", Key formulas:
//   S_h = sum_j phi(k_j^h) (v_j^h)^T,  z_h = sum_j phi(k_j^h),  phi = elu + 1,
// summed over all N nodes.  For a block of 128 features the kernel forms
//   [S_blk | z_blk] = phi(K_blk)^T [V_blk | 1]
// with tcgen05.mma: A = phi(K) and B = V are used in place as MN-major operands (the
// node index is the contraction dimension), straight from the 128-byte-swizzled TMA
// tiles after warps 0-3 apply phi (and, for fp32, the tf32 hi/lo split); z comes from a
// second MMA against a constant "ones" column.  Only the diagonal r x r blocks (one per
// head) are kept.
//
// Deterministic split-N tree: the nodes are cut into P fixed ranges; the CTAs of a
// feature block walk the ranges g, g + G, g + 2G, ... (persistent when ranges are many,
// as with per-segment statistics), accumulating each range in TMEM in node-tile order
// (two accumulators, so a range's epilogue overlaps the next range's MMAs) and writing
// its partial sums; a reduction adds the P partials in range order.  The reduction also
// writes S and z into the block-diagonal operand of the readout GEMM.  Output layout:
// S [H][r][r], z [H][r].
#include <algorithm>
#include <mutex>
#include <vector>

#include "glga_internal.cuh"

namespace glga {
namespace {

constexpr int kFB = 128;             // features per block: MMA M (phi(K)) and N (V)
constexpr int kRowBytes = 128;
constexpr int kMaxStages = 6;
constexpr int kWorkers = 512;        // warps 0-15: phi / split passes
constexpr int kWorkerWarps = kWorkers / 32;
constexpr int kProdWarp = 16;        // TMA producer
constexpr int kMmaWarp = 17;         // TMEM owner and MMA issuer
constexpr int kEpiWarp0 = 18;        // warps 18-21: epilogue (partial sums of each range)
constexpr int kThreads = 704;
constexpr uint32_t kAccStride = 256; // TMEM columns between the two accumulators

template <typename T>
struct StatsGeom {
    static constexpr int kRows = sizeof(T) == 2 ? 64 : 32;           // node rows per stage
    static constexpr int kStages = sizeof(T) == 2 ? 6 : 2;
    static constexpr int kUK = sizeof(T) == 2 ? 16 : 8;              // rows per MMA
    static constexpr int kBoxes = kFB * static_cast<int>(sizeof(T)) / kRowBytes;
    static constexpr uint32_t kBoxBytes = kRows * kRowBytes;
    static constexpr uint32_t kOpBytes = kBoxes * kBoxBytes;           // one operand plane
};

struct StatsParams {
    int64_t N;
    int32_t D, H;
    int32_t n_parts;         // P row ranges, walked by gridDim.x CTAs per feature block
    int64_t rows_per_part;   // multiple of the stage height (when part_ptr is NULL)
    const int32_t *part_ptr; // explicit row ranges [P + 1] (segments), or NULL
    int32_t stages;
    uint32_t stage_bytes;
    uint32_t scratch_off;    // epilogue staging in dynamic shared memory (0: direct stores)
    float *part;             // [P][H][r][r+1]
    unsigned *flag;
    // final statistics written by the epilogue (every non-empty segment is one range, so
    // a range's sums are its segment's S and z): range -> segment, S | z and the readout
    // operand (layouts of stats_reduce_kernel); null part_seg: partial sums only
    const int32_t *part_seg;
    int64_t n_seg;
    float *Sz;
    void *Bro;
    int32_t hg, BNr, Kp;
    int64_t seg_stride, plane;
};

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int SPLIT, typename T, int R>
__global__ void __launch_bounds__(kThreads, 1) stats_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                               const __grid_constant__ CUtensorMap tmV,
                                                               StatsParams p) {
    using G = StatsGeom<T>;
    constexpr uint32_t kFmt = SPLIT == 3 ? 2u : 1u;
    extern __shared__ uint8_t dsmem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t ready_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2];   // MMA -> epilogue: a range is accumulated
    __shared__ __align__(8) uint64_t acce_bar[2];   // epilogue -> MMA: the accumulator is drained
    __shared__ uint32_t tmem_base_sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ones = smem + static_cast<size_t>(p.stages) * p.stage_bytes;   // 16 x 128 B, K-major
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int fb = blockIdx.y;
    // this CTA's ranges: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int n_my = p.n_parts > static_cast<int>(blockIdx.x)
                         ? (p.n_parts - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
                         : 0;
    // row range [r0, r1) of range `part`; rows of its last tile past r1 get phi(k) = 0
    auto range_of = [&](int part, int64_t &r0, int64_t &r1) {
        r0 = p.part_ptr ? p.part_ptr[part] : static_cast<int64_t>(part) * p.rows_per_part;
        r1 = p.part_ptr ? p.part_ptr[part + 1] : std::min<int64_t>(p.N, r0 + p.rows_per_part);
    };
    auto tiles_of = [&](int64_t r0, int64_t r1) {
        return r1 > r0 ? static_cast<int>(ceil_div(r1 - r0, G::kRows)) : 0;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&ready_bar[s], kWorkerWarps);   // one arrival per worker warp
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf_bar[b], 1);
            mbar_init(&acce_bar[b], 4);
        }
        fence_mbar_init();
    }
    if (threadIdx.x < kWorkers) {
        // ones tile: row 0 = 1.0 everywhere, rows 1..15 = 0 (the swizzle only permutes
        // 16-byte chunks inside a row, so row 0 reads as ones at any K offset)
        uint32_t *o = reinterpret_cast<uint32_t *>(ones);
        const uint32_t one = sizeof(T) == 2 ? 0x3F803F80u : 0x3F800000u;
        for (int i = threadIdx.x; i < 16 * kRowBytes / 4; i += kWorkers) o[i] = (i < kRowBytes / 4) ? one : 0u;
        fence_async_smem();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_base_sh, 512u);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kProdWarp) {
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued = 0;
            RingPos rp;
            bool ok = true;
            for (int k = 0; k < n_my && ok; ++k) {
                int64_t r0, r1;
                range_of(static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), r0, r1);
                const int ntiles = tiles_of(r0, r1);
                for (int it = 0; it < ntiles; ++it, rp.next(p.stages)) {
                    const int s = rp.slot;
                    if (issued >= p.stages && !mbar_wait_bounded(&empty_bar[s], rp.phase ^ 1u)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
                    mbar_arrive_expect_tx(&full_bar[s], 2 * G::kOpBytes);
                    const int32_t y = static_cast<int32_t>(r0 + static_cast<int64_t>(it) * G::kRows);
#pragma unroll
                    for (int b = 0; b < G::kBoxes; ++b) {
                        const int32_t x = fb * kFB + b * (kRowBytes / static_cast<int>(sizeof(T)));
                        tma_load_2d(st + b * G::kBoxBytes, &tmK, &full_bar[s], x, y);
                        tma_load_2d(st + G::kOpBytes + b * G::kBoxBytes, &tmV, &full_bar[s], x, y);
                    }
                    ++issued;
                }
            }
            if (!ok) {
                atomicOr(p.flag, kDevErrTimeout);
                for (int it = std::max(0, issued - p.stages); it < issued; ++it)
                    mbar_wait_bounded(&full_bar[it % p.stages], static_cast<uint32_t>(it / p.stages) & 1u);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t idS = instr_desc(128, kFB, kFmt, true, true);
            const uint32_t idZ = instr_desc(128, 16, kFmt, true, false);
            const uint32_t idSk = instr_desc(128, kFB, kFmt, false, false);
            const uint32_t idZk = instr_desc(128, 16, kFmt, false, false);
            const uint64_t dones = smem_desc(smem_u32(ones), 16, 1024, 2);
            bool ok = true;
            RingPos rp;
            for (int k = 0; k < n_my && ok; ++k) {
                const int buf = k & 1;
                const uint32_t acc_base = tmem + static_cast<uint32_t>(buf) * kAccStride;
                // the epilogue must have drained this accumulator's previous range (k - 2)
                if (k >= 2 && !mbar_wait_bounded(&acce_bar[buf], static_cast<uint32_t>((k >> 1) - 1) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                int64_t r0, r1;
                range_of(static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), r0, r1);
                const int ntiles = tiles_of(r0, r1);
                for (int it = 0; it < ntiles; ++it, rp.next(p.stages)) {
                    const int s = rp.slot;
                    if (!mbar_wait_bounded(&ready_bar[s], rp.phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t kb = smem_u32(smem + static_cast<size_t>(s) * p.stage_bytes);
                    const uint32_t vb = kb + G::kOpBytes;
#pragma unroll
                    for (int ks = 0; ks < G::kRows / G::kUK; ++ks) {
                        const uint32_t off = ks * G::kUK * kRowBytes;
                        const uint32_t acc0 = (it | ks) != 0;
                        if (SPLIT == 3) {
                            // tf32 operands were transposed to K-major planes by the workers
                            // (MN-major tf32 would need the 32-byte-atom swizzle)
                            const uint32_t kt = ks * 32;   // 8 node rows of tf32 = 32 bytes
                            const uint32_t ah = kb + 2 * G::kOpBytes, al = kb + 3 * G::kOpBytes;
                            const uint32_t bh = kb + 4 * G::kOpBytes, bl = kb + 5 * G::kOpBytes;
                            const uint64_t akh = smem_desc(ah + kt, 16, 1024, 2);
                            const uint64_t akl = smem_desc(al + kt, 16, 1024, 2);
                            const uint64_t bvh = smem_desc(bh + kt, 16, 1024, 2);
                            const uint64_t bvl = smem_desc(bl + kt, 16, 1024, 2);
                            umma_tf32(acc_base, akh, bvh, idSk, acc0);
                            umma_tf32(acc_base, akh, bvl, idSk, 1u);
                            umma_tf32(acc_base, akl, bvh, idSk, 1u);
                            umma_tf32(acc_base + kFB, akh, dones, idZk, acc0);
                            umma_tf32(acc_base + kFB, akl, dones, idZk, 1u);
                            (void)off;
                        } else {
                            const uint64_t ak = smem_desc(kb + off, G::kBoxBytes, 1024, 2);
                            const uint64_t bv = smem_desc(vb + off, G::kBoxBytes, 1024, 2);
                            umma_bf16(acc_base, ak, bv, idS, acc0);
                            umma_bf16(acc_base + kFB, ak, dones, idZ, acc0);
                        }
                    }
                    umma_commit(&empty_bar[s]);
                }
                // (a range without rows commits at once; its epilogue writes zeros)
                if (ok) umma_commit(&accf_bar[buf]);
            }
            if (!ok) atomicOr(p.flag, kDevErrTimeout);
        }
    } else if (warp < kWorkerWarps) {
        // ---------------- warps 0-15: phi(K) (zero past the range), tf32 split ----------
        bool ok = true;
        constexpr int kChunksPerBox = G::kBoxBytes / 16;
        RingPos rp;
        for (int k = 0; k < n_my && ok; ++k) {
            int64_t r0, r1;
            range_of(static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), r0, r1);
            const int ntiles = tiles_of(r0, r1);
            for (int it = 0; it < ntiles && ok; ++it, rp.next(p.stages)) {
                const int s = rp.slot;
                // the warp agrees on the outcome, so it stays converged for its arrival
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[s], rp.phase))) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + static_cast<size_t>(s) * p.stage_bytes;
                const int64_t y0 = r0 + static_cast<int64_t>(it) * G::kRows;
                if (SPLIT == 3) {
                    // Transpose the [node][feature] TMA tiles (128-byte swizzle) into K-major
                    // planes [feature][node] with the same swizzle, applying phi and the tf32
                    // split on the way: element (m, k) of a plane sits at
                    // (m/8)*1024 + (m%8)*128 + (((k/4) ^ (m%8)) * 16) + (k%4)*4.
                    const float *rk = reinterpret_cast<const float *>(st);
                    const float *rv = reinterpret_cast<const float *>(st + G::kOpBytes);
                    float *ah = reinterpret_cast<float *>(st + 2 * G::kOpBytes);
                    float *al = reinterpret_cast<float *>(st + 3 * G::kOpBytes);
                    float *bh = reinterpret_cast<float *>(st + 4 * G::kOpBytes);
                    float *bl = reinterpret_cast<float *>(st + 5 * G::kOpBytes);
                    for (int idx = threadIdx.x; idx < G::kRows * kFB; idx += kWorkers) {
                        const int kr = idx / kFB, m = idx % kFB;
                        const int e = m % 32;
                        const int src = ((m / 32) * G::kBoxBytes + kr * kRowBytes +
                                         (((e / 4) ^ (kr % 8)) * 16) + (e % 4) * 4) / 4;
                        const int dst = ((m / 8) * 1024 + (m % 8) * kRowBytes +
                                         (((kr / 4) ^ (m % 8)) * 16) + (kr % 4) * 4) / 4;
                        const bool valid = y0 + kr < r1;
                        const float f = valid ? phi(rk[src]) : 0.f;
                        const float v = rv[src];
                        const float fh = to_tf32(f), vh = to_tf32(v);
                        ah[dst] = fh;
                        al[dst] = to_tf32(f - fh);
                        bh[dst] = vh;
                        bl[dst] = to_tf32(v - vh);
                    }
                }
                for (int c = threadIdx.x; SPLIT != 3 && c < G::kBoxes * kChunksPerBox; c += kWorkers) {
                    const int row = (c % kChunksPerBox) / 8;
                    const bool valid = y0 + row < r1;
                    uint4 *kp = reinterpret_cast<uint4 *>(st) + c;
                    const uint4 u = *kp;
                    *kp = valid ? make_uint4(phi_bf16x2(u.x), phi_bf16x2(u.y), phi_bf16x2(u.z), phi_bf16x2(u.w))
                                : make_uint4(0u, 0u, 0u, 0u);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ready_bar[s]);
            }
        }
        if (!ok && lane == 0) atomicOr(p.flag, kDevErrTimeout);
    } else {
        // ---------------- warps 18-21: diagonal head blocks of S and z -> partials ----------
        const int quad = warp & 3;                        // TMEM lanes this warp may read
        const int t = quad * 32 + lane;                   // TMEM lane = feature in the block
        const int f = fb * kFB + t;
        const bool live = f < p.D;
        const int h = live ? f / R : 0, a = f % R;
        const int hc0 = h * R - fb * kFB;                 // head's first column in the block
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        bool ok = true;
        for (int k = 0; k < n_my; ++k) {
            const int buf = k & 1;
            const int part = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
            int64_t r0, r1;
            range_of(part, r0, r1);
            const bool have = ok && tiles_of(r0, r1) > 0;
            if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(&accf_bar[buf], static_cast<uint32_t>(k >> 1) & 1u))) {
                ok = false;
                if (lane == 0) atomicOr(p.flag, kDevErrTimeout);
            }
            tc_fence_after();
            // this feature's row of the range's partial sums ([H][R][R+1] layout: the row
            // of feature f = h*R + a starts at f*(R+1)); with staging, the warp's 32 rows
            // (one contiguous block of 32*(R+1) floats) go through shared memory and leave
            // as coalesced stores
            float *sw = p.scratch_off ? reinterpret_cast<float *>(dsmem_raw + p.scratch_off) +
                                            (warp - kEpiWarp0) * 32 * (R + 1)
                                      : nullptr;
            float *dst = sw ? sw + lane * (R + 1)
                            : p.part + ((static_cast<int64_t>(part) * p.H + h) * R + a) * (R + 1);
            const uint32_t acc = tmem + lane_base + static_cast<uint32_t>(buf) * kAccStride;
#pragma unroll
            for (int q = 0; q < kFB / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(acc + q * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int col = q * 32 + j;
                    if (live && col >= hc0 && col < hc0 + R) dst[col - hc0] = have ? __uint_as_float(v[j]) : 0.f;
                }
            }
            uint32_t v[32];
            tmem_ld32(acc + kFB, v);
            tmem_ld_wait();
            if (live) dst[R] = have ? __uint_as_float(v[0]) : 0.f;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar[buf]);
            if (sw && p.part_seg) {
                // the range is its segment: S rows (coalesced, from the staging), z, and the
                // segment's readout operand block (transposed S_h and z_h; consecutive
                // features write consecutive K positions)
                __syncwarp();
                const int64_t seg = p.part_seg[part];
                const int f0 = fb * kFB + quad * 32;
                const int rows = max(0, min(32, p.D - f0));
                const int64_t hrr = static_cast<int64_t>(p.H) * R * R;
                float *gS = p.Sz + seg * hrr + static_cast<int64_t>(f0) * R;
                for (int i = lane; i < rows * R; i += 32) gS[i] = sw[(i / R) * (R + 1) + i % R];
                if (live) {
                    p.Sz[p.n_seg * hrr + seg * p.H * R + f] = sw[lane * (R + 1) + R];
                    const int gi = h / p.hg, hl = h - gi * p.hg, hga = min(p.hg, p.H - gi * p.hg);
                    const int64_t base = seg * p.seg_stride + static_cast<int64_t>(gi) * p.BNr * p.Kp + hl * R + a;
                    for (int cc = 0; cc <= R; ++cc) {
                        const float x = sw[lane * (R + 1) + cc];
                        const int n = cc < R ? hl * R + cc : hga * R + hl;
                        const int64_t idx = base + static_cast<int64_t>(n) * p.Kp;
                        if (sizeof(T) == 4) {
                            const float hi = to_tf32(x);
                            reinterpret_cast<float *>(p.Bro)[idx] = hi;
                            reinterpret_cast<float *>(p.Bro)[p.plane + idx] = to_tf32(x - hi);
                        } else {
                            reinterpret_cast<__nv_bfloat16 *>(p.Bro)[idx] = __float2bfloat16_rn(x);
                        }
                    }
                }
                __syncwarp();
            } else if (sw) {
                // rows fb*128 + quad*32 .. (those below D) of the range's block
                const int f0 = fb * kFB + quad * 32;
                const int rows = max(0, min(32, p.D - f0));
                float *g = p.part + (static_cast<int64_t>(part) * p.H * R + f0) * (R + 1);
                for (int i = lane; i < rows * (R + 1); i += 32) g[i] = sw[i];
                __syncwarp();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512u);
    }
}

// Segment k = blockIdx.y sums its parts (seg_part_ptr[k] .. seg_part_ptr[k+1] - 1, or
// 0..P-1 when seg_part_ptr is NULL) in order.  Writes S_k [H][R][R] at Sz + k*H*R*R and
// z_k [H][R] at Sz + n_seg*H*R*R + k*H*R and, when Bro is given, segment k's readout
// operand at Bro + k*seg_stride: group gi = h / hg holds, K-major, S_h at rows (n)
// hl*R + c and columns (k) hl*R + a, and z_h at row hga*R + hl (hl = h - gi*hg, hga =
// heads in group gi).  Every other entry of Bro stays zero from its initialisation.
// Block of 256 threads = 8 warps for 32 consecutive outputs: warp w adds parts
// w, w+8, w+16, ... in order, then warp 0 adds the 8 warp sums in warp order.
template <typename T>
__global__ void __launch_bounds__(256) stats_reduce_kernel(const float *__restrict__ part, int P,
                                    const int32_t *__restrict__ seg_part_ptr, int64_t n_seg,
                                    int H, int R, float *__restrict__ Sz, T *__restrict__ Bro,
                                    int hg, int BNr, int Kp, int64_t seg_stride, int64_t plane,
                                    float *__restrict__ flat) {
    __shared__ float ws[8][32];
    const int per_head = R * (R + 1);
    const int total = H * per_head;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int o = blockIdx.x * 32 + lane;
    // segments blockIdx.y, blockIdx.y + gridDim.y, ... (the grid's y extent is capped)
    for (int64_t seg = blockIdx.y; seg < n_seg; seg += gridDim.y) {
    const int q0 = seg_part_ptr ? seg_part_ptr[seg] : 0;
    const int q1 = seg_part_ptr ? seg_part_ptr[seg + 1] : P;
    float acc = 0.f;
    if (o < total) {
        int q = q0 + w;
        for (; q + 24 < q1; q += 32) {
            const float a0 = part[static_cast<int64_t>(q) * total + o];
            const float a1 = part[static_cast<int64_t>(q + 8) * total + o];
            const float a2 = part[static_cast<int64_t>(q + 16) * total + o];
            const float a3 = part[static_cast<int64_t>(q + 24) * total + o];
            acc += a0; acc += a1; acc += a2; acc += a3;
        }
        for (; q < q1; q += 8) acc += part[static_cast<int64_t>(q) * total + o];
    }
    ws[w][lane] = acc;
    __syncthreads();
    float s = 0.f;
    if (w == 0 && o < total) {
#pragma unroll
        for (int k = 0; k < 8; ++k) s += ws[k][lane];
    }
    if (w == 0 && o < total && flat) {
        // the sum of these ranges in the partial layout [H][R][R+1] (one row shard's
        // contribution, exchanged between ranks before the final reduction)
        flat[o] = s;
    } else if (w == 0 && o < total) {
        const int h = o / per_head, rem = o % per_head, a = rem / (R + 1), c = rem % (R + 1);
        const int64_t hrr = static_cast<int64_t>(H) * R * R;
        if (c < R)
            Sz[seg * hrr + (static_cast<int64_t>(h) * R + a) * R + c] = s;
        else
            Sz[n_seg * hrr + seg * H * R + h * R + a] = s;
        if (Bro) {
            const int gi = h / hg, hl = h - gi * hg, hga = min(hg, H - gi * hg);
            const int n = c < R ? hl * R + c : hga * R + hl;
            const int64_t idx = seg * seg_stride + (static_cast<int64_t>(gi) * BNr + n) * Kp + hl * R + a;
            if (sizeof(T) == 4) {
                const float hi = to_tf32(s);
                reinterpret_cast<float *>(Bro)[idx] = hi;
                reinterpret_cast<float *>(Bro)[plane + idx] = to_tf32(s - hi);
            } else {
                Bro[idx] = __float2bfloat16_rn(s);
            }
        }
    }
    __syncthreads();   // ws is rewritten by the next segment
    }
}

// Segment-major reduction for batches of segments: block (h, y) reduces head h of
// segments y, y + gridDim.y, ...: it adds each segment's ranges one after another in
// range order (deterministic) into shared memory with coalesced reads of the partials,
// then writes S_h and z_h of the segment to Sz and its block of the readout operand
// (rows n of the K-major operand, R consecutive k each) with coalesced writes.  Layouts as
// in stats_reduce_kernel.
template <typename T>
__global__ void __launch_bounds__(256) stats_reduce_segments_kernel(
    const float *__restrict__ part, const int32_t *__restrict__ seg_part_ptr, int64_t n_seg, int H,
    int R, float *__restrict__ Sz, T *__restrict__ Bro, int hg, int BNr, int Kp, int64_t seg_stride,
    int64_t plane) {
    extern __shared__ float red[];                  // [R][R + 1] of one head
    const int h = blockIdx.x;
    const int per_head = R * (R + 1);
    const int total = H * per_head;
    const int64_t hrr = static_cast<int64_t>(H) * R * R;
    const int gi = h / hg, hl = h - gi * hg, hga = min(hg, H - gi * hg);
    for (int64_t seg = blockIdx.y; seg < n_seg; seg += gridDim.y) {
        const int q0 = seg_part_ptr[seg], q1 = seg_part_ptr[seg + 1];
        // 8 outputs per thread at a time, so 8 independent loads are in flight
        constexpr int kIlp = 8;
        for (int i0 = threadIdx.x; i0 < per_head; i0 += kIlp * blockDim.x) {
            float acc[kIlp];
#pragma unroll
            for (int k = 0; k < kIlp; ++k) acc[k] = 0.f;
            for (int q = q0; q < q1; ++q) {
                const float *src = part + static_cast<int64_t>(q) * total + h * per_head;
#pragma unroll
                for (int k = 0; k < kIlp; ++k) {
                    const int i = i0 + k * blockDim.x;
                    if (i < per_head) acc[k] += src[i];
                }
            }
#pragma unroll
            for (int k = 0; k < kIlp; ++k) {
                const int i = i0 + k * blockDim.x;
                if (i < per_head) red[i] = acc[k];
            }
        }
        __syncthreads();
        float *S = Sz + seg * hrr + static_cast<int64_t>(h) * R * R;
        for (int i = threadIdx.x; i < R * R; i += blockDim.x) S[i] = red[(i / R) * (R + 1) + i % R];
        float *z = Sz + n_seg * hrr + seg * H * R + h * R;
        for (int a = threadIdx.x; a < R; a += blockDim.x) z[a] = red[a * (R + 1) + R];
        if (Bro) {
            // operand rows n = hl*R + c (S_h column c) and n = hga*R + hl (z_h); k = hl*R + a
            T *B = Bro + seg * seg_stride + static_cast<int64_t>(gi) * BNr * Kp;
            for (int i = threadIdx.x; i < (R + 1) * R; i += blockDim.x) {
                const int c = i / R, a = i % R;          // c == R: the z row
                const float v = red[a * (R + 1) + c];
                const int n = c < R ? hl * R + c : hga * R + hl;
                const int64_t idx = static_cast<int64_t>(n) * Kp + hl * R + a;
                if (sizeof(T) == 4) {
                    const float hi = to_tf32(v);
                    reinterpret_cast<float *>(B)[idx] = hi;
                    reinterpret_cast<float *>(B)[plane + idx] = to_tf32(v - hi);
                } else {
                    B[idx] = __float2bfloat16_rn(v);
                }
            }
        }
        __syncthreads();                            // red is rewritten by the next segment
    }
}

// Ring stages that fit beside the epilogue's staging buffer (4 warps x 32 rows x (r + 1)
// floats), or 0 when fewer than two do.
size_t stats_scratch_bytes(int r) { return static_cast<size_t>(4) * 32 * (r + 1) * sizeof(float); }
int stats_stages_with_scratch(uint32_t stage_bytes, int stages, int r) {
    constexpr size_t kSmemMax = 226 * 1024;   // dynamic shared memory, leaving room for the static part
    const int st = static_cast<int>(
        std::min<size_t>(stages, (kSmemMax - 2048 - 1024 - stats_scratch_bytes(r)) / stage_bytes));
    return st >= 2 ? st : 0;
}

// P = p.n_parts row ranges per feature block, walked by min(P, num_sms / nblk) CTAs each
// (one range per CTA when the ranges are about one per SM).
template <typename T>
glga_status launch_stats(const CUtensorMap &mk, const CUtensorMap &mv, const StatsParams &p, int num_sms,
                         int nblk, int r, cudaStream_t s) {
    const int g = std::max(1, std::min(p.n_parts, std::max(1, num_sms / nblk)));
    dim3 grid(static_cast<unsigned>(g), static_cast<unsigned>(nblk));
    // several ranges per CTA, or final statistics written by the epilogue: the epilogue
    // stages each range's sums in shared memory (coalesced stores) when two or more ring
    // stages still fit beside the staging buffer
    StatsParams q = p;
    q.scratch_off = 0;
    const size_t scratch = stats_scratch_bytes(r);
    if (g < p.n_parts || p.part_seg) {
        const int st = stats_stages_with_scratch(p.stage_bytes, p.stages, r);
        if (st >= 2) {
            q.stages = st;
            q.scratch_off = static_cast<uint32_t>(1024 + static_cast<size_t>(st) * p.stage_bytes + 2048);
        } else if (p.part_seg) {
            set_error("statistics: the epilogue staging does not fit beside the ring");
            return GLGA_ERR_UNSUPPORTED;
        }
    }
    const size_t smem = static_cast<size_t>(q.stages) * q.stage_bytes + 2048 + 1024 + (q.scratch_off ? scratch : 0);
    constexpr int SPLIT = sizeof(T) == 4 ? 3 : 1;
#define GLGA_ST(RR)                                                                          \
    case RR: {                                                                               \
        auto kern = stats_tc_kernel<SPLIT, T, RR>;                                           \
        GLGA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                       static_cast<int>(smem)));                             \
        kern<<<grid, kThreads, smem, s>>>(mk, mv, q);                                        \
        break;                                                                               \
    }
    switch (r) {
        GLGA_ST(8) GLGA_ST(16) GLGA_ST(32) GLGA_ST(64) GLGA_ST(128)
        default: set_error("unsupported r"); return GLGA_ERR_UNSUPPORTED;
    }
#undef GLGA_ST
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

// Row ranges: a multiple of the stage height, about one CTA (range x feature block) per
// SM in total.
void plan_parts(int64_t N, int nblk, int num_sms, int rows, int64_t max_parts, int *parts,
                int64_t *rows_per_part) {
    const int64_t want = std::max<int64_t>(1, ceil_div(num_sms, nblk));
    const int64_t tiles = std::max<int64_t>(1, ceil_div(std::max<int64_t>(N, 1), rows));
    int64_t P = std::max<int64_t>(1, std::min(std::min(want, tiles), max_parts));
    const int64_t per = ceil_div(tiles, P) * rows;
    P = std::max<int64_t>(1, ceil_div(std::max<int64_t>(N, 1), per));
    *parts = static_cast<int>(P);
    *rows_per_part = per;
}

glga_status encode_kv_maps(const void *KV, int64_t N, int D, int elem, CUtensorMap *mk, CUtensorMap *mv,
                           int rows) {
    const CUtensorMapDataType dt =
        elem == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint64_t stride = static_cast<uint64_t>(2) * D * elem;
    glga_status st = encode_tmap_2d(mk, dt, KV, D, N, stride, kRowBytes / elem, rows);
    if (st != GLGA_OK) return st;
    return encode_tmap_2d(mv, dt, static_cast<const uint8_t *>(KV) + static_cast<size_t>(D) * elem,
                          D, N, stride, kRowBytes / elem, rows);
}

// bf16: K and V tiles (phi applied in place).  fp32: K and V tiles plus four K-major
// tf32 planes (phi(K) hi/lo, V hi/lo).
template <typename T>
uint32_t stage_bytes() {
    return (sizeof(T) == 4 ? 6 : 2) * StatsGeom<T>::kOpBytes;
}

}  // namespace

glga_status stats_setup(Ctx *c) {
    const int nblk = static_cast<int>(ceil_div(c->D, kFB));
    const int rows = c->io == GLGA_F32 ? StatsGeom<float>::kRows : StatsGeom<__nv_bfloat16>::kRows;
    int parts = 1;
    int64_t per = 0;
    plan_parts(c->N, nblk, c->num_sms, rows, 1 << 20, &parts, &per);
    // Row ranges of at most `per` rows that never cross a segment boundary: each
    // non-empty segment is cut into ceil(len / per) ranges, summed by the reduction in
    // order.  Without segments this is the plain cut into `per`-row ranges.
    std::vector<int32_t> pp(1, 0), sp(1, 0);
    for (int64_t k = 0; k < c->n_seg; ++k) {
        const int64_t a = c->seg_ptr[k], b = c->seg_ptr[k + 1];
        for (int64_t r0 = a; r0 < b; r0 += per) pp.push_back(static_cast<int32_t>(std::min(b, r0 + per)));
        sp.push_back(static_cast<int32_t>(pp.size() - 1));
    }
    parts = static_cast<int>(pp.size() - 1);
    c->stats_parts = parts;
    c->stats_rows_per_part = per;
    // every non-empty segment one range: the statistics kernel's epilogue writes the final
    // S, z and readout operand of each segment, and no reduction runs
    std::vector<int32_t> pseg;
    bool one_each = c->n_seg > 1 && c->N > 0;
    for (int64_t k = 0; k < c->n_seg && one_each; ++k) {
        const int32_t cnt = sp[k + 1] - sp[k];
        if (cnt > 1) one_each = false;
        if (cnt == 1) pseg.push_back(static_cast<int32_t>(k));
    }
    const uint32_t sb = c->io == GLGA_F32 ? stage_bytes<float>() : stage_bytes<__nv_bfloat16>();
    const int kst = c->io == GLGA_F32 ? StatsGeom<float>::kStages : StatsGeom<__nv_bfloat16>::kStages;
    c->stats_direct = one_each && stats_stages_with_scratch(sb, kst, c->r) >= 2;
    const size_t one = static_cast<size_t>(c->H) * c->r * (c->r + 1) * sizeof(float);
    if (one * std::max(parts, 1) > (size_t{4} << 30)) {
        set_error("glga_create: %d statistics ranges need more than 4 GiB of partial sums", parts);
        return GLGA_ERR_UNSUPPORTED;
    }
    // (the projection epilogue writes one partial per CTA when the statistics are fused)
    glga_status st = dev_alloc(c, reinterpret_cast<void **>(&c->Spart),
                               one * std::max(std::max(parts, c->stats_fused_parts), 1));
    if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->Sz), one * c->n_seg);
    if (st == GLGA_OK) {
        // empty segments keep zero statistics (the direct epilogue never writes them)
        cudaError_t e = cudaMemset(c->Sz, 0, one * c->n_seg);
        if (e != cudaSuccess) return cuda_fail(e, "statistics init");
    }
    if (st == GLGA_OK && c->stats_direct) {
        st = dev_alloc(c, reinterpret_cast<void **>(&c->part_seg), pseg.size() * sizeof(int32_t));
        if (st == GLGA_OK) {
            cudaError_t e = cudaMemcpy(c->part_seg, pseg.data(), pseg.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
            if (e != cudaSuccess) return cuda_fail(e, "statistics segments");
        }
    }
    if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->part_ptr), pp.size() * sizeof(int32_t));
    if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->seg_part_ptr), sp.size() * sizeof(int32_t));
    if (st == GLGA_OK) {
        cudaError_t e = cudaMemcpy(c->part_ptr, pp.data(), pp.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
        if (e == cudaSuccess)
            e = cudaMemcpy(c->seg_part_ptr, sp.data(), sp.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "statistics ranges");
    }
    if (st == GLGA_OK && c->N > 0)
        st = encode_kv_maps(c->kv_own, c->N, c->D, c->elem, &c->tmK.map, &c->tmV.map, rows);
    return st;
}

namespace {
// Partial sums of S | z over the context's row ranges (Spart).
glga_status stats_partials(Ctx *c, cudaStream_t s) {
    if (c->N > 0 && !c->stats_fused) {
        StatsParams p;
        p.N = c->N;
        p.D = c->D;
        p.H = c->H;
        p.n_parts = c->stats_parts;
        p.rows_per_part = c->stats_rows_per_part;
        p.part_ptr = c->part_ptr;
        p.part_seg = c->stats_direct ? c->part_seg : nullptr;
        p.n_seg = c->n_seg;
        p.Sz = c->Sz;
        p.Bro = c->Bro;
        p.hg = c->ro_hg;
        p.BNr = c->ro_bn;
        p.Kp = c->ro_kp;
        p.seg_stride = static_cast<int64_t>(c->ro_groups) * c->ro_bn * c->ro_kp;
        p.plane = c->n_seg * p.seg_stride;
        p.stages = c->io == GLGA_F32 ? StatsGeom<float>::kStages : StatsGeom<__nv_bfloat16>::kStages;
        p.part = c->Spart;
        p.flag = c->dev_flag;
        const int nblk = static_cast<int>(ceil_div(c->D, kFB));
        glga_status st;
        if (c->io == GLGA_F32) {
            p.stage_bytes = stage_bytes<float>();
            st = launch_stats<float>(c->tmK.map, c->tmV.map, p, c->num_sms, nblk, c->r, s);
        } else {
            p.stage_bytes = stage_bytes<__nv_bfloat16>();
            st = launch_stats<__nv_bfloat16>(c->tmK.map, c->tmV.map, p, c->num_sms, nblk, c->r, s);
        }
        if (st != GLGA_OK) return st;
        c->launches += 1;
    }
    return GLGA_OK;
}

// Final reduction of P partials (flat layout [P][H][r][r+1]) into S, z and the readout
// operand; the order of the sums is fixed (the same on every rank).
template <typename T>
glga_status reduce_into_stats(Ctx *c, const float *part, int P, float *flat, cudaStream_t s) {
    const int total = c->H * c->r * (c->r + 1);
    const int64_t seg_stride = static_cast<int64_t>(c->ro_groups) * c->ro_bn * c->ro_kp;
    stats_reduce_kernel<T><<<static_cast<unsigned>(ceil_div(total, 32)), 256, 0, s>>>(
        part, P, nullptr, 1, c->H, c->r, c->Sz, static_cast<T *>(c->Bro), c->ro_hg, c->ro_bn, c->ro_kp,
        seg_stride, seg_stride, flat);
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    return GLGA_OK;
}
}  // namespace

glga_status stats_run_partial(Ctx *c, float *own, cudaStream_t s) {
    glga_status st = stats_partials(c, s);
    if (st != GLGA_OK) return st;
    const int P = c->N == 0 ? 0 : c->stats_fused ? c->stats_fused_parts : c->stats_parts;
    return c->io == GLGA_F32 ? reduce_into_stats<float>(c, c->Spart, P, own, s)
                             : reduce_into_stats<__nv_bfloat16>(c, c->Spart, P, own, s);
}

glga_status stats_finish(Ctx *c, const float *partials, int P, cudaStream_t s) {
    return c->io == GLGA_F32 ? reduce_into_stats<float>(c, partials, P, nullptr, s)
                             : reduce_into_stats<__nv_bfloat16>(c, partials, P, nullptr, s);
}

glga_status stats_run(Ctx *c, cudaStream_t s) {
    glga_status st0 = stats_partials(c, s);
    if (st0 != GLGA_OK) return st0;
    if (c->stats_direct) return GLGA_OK;   // the epilogue wrote S, z and the readout operand
    const int total = c->H * c->r * (c->r + 1);
    const int P = c->N == 0 ? 0 : c->stats_fused ? c->stats_fused_parts : c->stats_parts;
    const int64_t seg_stride = static_cast<int64_t>(c->ro_groups) * c->ro_bn * c->ro_kp;
    const int64_t plane = c->n_seg * seg_stride;
    const dim3 rgrid(static_cast<unsigned>(ceil_div(total, 32)),
                     static_cast<unsigned>(std::min<int64_t>(c->n_seg, 65535)));
    // with no rows every segment's sums are zero (no ranges to add); the fused partials
    // (one segment) are parts 0 .. P-1
    const int32_t *spp = c->N > 0 && !c->stats_fused ? c->seg_part_ptr : nullptr;
    if (c->n_seg > 1 && spp) {
        const dim3 sgrid(static_cast<unsigned>(c->H),
                         static_cast<unsigned>(std::min<int64_t>(c->n_seg, 65535)));
        const size_t red_bytes = static_cast<size_t>(c->r) * (c->r + 1) * sizeof(float);   // <= 66 KB
        if (c->io == GLGA_F32) {
            GLGA_CUDA(cudaFuncSetAttribute(stats_reduce_segments_kernel<float>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(red_bytes)));
            stats_reduce_segments_kernel<float><<<sgrid, 256, red_bytes, s>>>(
                c->Spart, spp, c->n_seg, c->H, c->r, c->Sz, static_cast<float *>(c->Bro), c->ro_hg,
                c->ro_bn, c->ro_kp, seg_stride, plane);
        } else {
            GLGA_CUDA(cudaFuncSetAttribute(stats_reduce_segments_kernel<__nv_bfloat16>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(red_bytes)));
            stats_reduce_segments_kernel<__nv_bfloat16><<<sgrid, 256, red_bytes, s>>>(
                c->Spart, spp, c->n_seg, c->H, c->r, c->Sz, static_cast<__nv_bfloat16 *>(c->Bro),
                c->ro_hg, c->ro_bn, c->ro_kp, seg_stride, plane);
        }
        GLGA_CUDA(cudaGetLastError());
        c->launches += 1;
        return GLGA_OK;
    }
    if (c->io == GLGA_F32)
        stats_reduce_kernel<float><<<rgrid, 256, 0, s>>>(
            c->Spart, P, spp, c->n_seg, c->H, c->r, c->Sz, static_cast<float *>(c->Bro), c->ro_hg,
            c->ro_bn, c->ro_kp, seg_stride, plane, nullptr);
    else
        stats_reduce_kernel<__nv_bfloat16><<<rgrid, 256, 0, s>>>(
            c->Spart, P, spp, c->n_seg, c->H, c->r, c->Sz, static_cast<__nv_bfloat16 *>(c->Bro),
            c->ro_hg, c->ro_bn, c->ro_kp, seg_stride, plane, nullptr);
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    return GLGA_OK;
}

// ---------------------------------------------------------------------------------------
// glga_global_stats_static: the same global statistics for callers that cannot allocate
// device memory.  The per-range partial sums live in a fixed 2 MiB array that is part of
// this library's device image (every GPU that loads the library keeps it until the
// process exits), so the call allocates nothing.
// ---------------------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchFloats = 512u * 1024u;   // 2 MiB of float partial sums
constexpr int kMaxDevices = 64;

__device__ __align__(256) float g_static_stats_scratch[kStaticScratchFloats];
__device__ unsigned g_static_stats_flag;   // bounded-wait timeouts of these calls

std::mutex g_static_mu;
struct StaticSlot {
    void *ctx = nullptr;          // the CUDA context the addresses belong to
    float *scratch = nullptr;
    unsigned *flag = nullptr;
    int num_sms = 0;
};
StaticSlot g_static_slot[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The current CUDA context (driver entry point resolved at run time), or null.
void *current_context() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    }
    CUcontext cx = nullptr;
    if (!fn || fn(&cx) != CUDA_SUCCESS) return nullptr;
    return cx;
}

// Device addresses of the scratch array and its flag on the current device.  Their names
// in host code are host-side stand-ins, never device addresses.  The lookup runs once per
// device and again whenever the device's context is not the one the cached addresses
// belong to (after cudaDeviceReset, the module is loaded anew at other addresses).
glga_status static_scratch(int dev, float **ptr, unsigned **flag, int *num_sms) {
    void *cx = current_context();
    cudaError_t e = cudaSuccess;
    if (!cx) {
        // no context current yet: cudaSetDevice initialises the device's primary context
        e = cudaSetDevice(dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
        cx = current_context();
    }
    std::lock_guard<std::mutex> lock(g_static_mu);
    StaticSlot &sl = g_static_slot[dev];
    if (!sl.scratch || cx != sl.ctx) {
        void *q = nullptr, *f = nullptr;
        e = cudaGetSymbolAddress(&q, g_static_stats_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static stats scratch)");
        e = cudaGetSymbolAddress(&f, g_static_stats_flag);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static stats flag)");
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        sl.ctx = cx;
        sl.scratch = static_cast<float *>(q);
        sl.flag = static_cast<unsigned *>(f);
        sl.num_sms = sms;
    }
    *ptr = sl.scratch;
    *flag = sl.flag;
    *num_sms = sl.num_sms;
    return GLGA_OK;
}

glga_status static_device(int *dev) {
    GLGA_CUDA(cudaGetDevice(dev));
    if (*dev < 0 || *dev >= kMaxDevices) {
        set_error("static statistics scratch: device ordinal %d not supported", *dev);
        return GLGA_ERR_UNSUPPORTED;
    }
    return GLGA_OK;
}

}  // namespace
}  // namespace glga

extern "C" glga_status glga_global_stats_static(const void *KV, int64_t N, int32_t H, int32_t r,
                                                glga_dtype io, float *Sz, void *stream) {
    using namespace glga;
    if (N < 0 || N > 2147483647LL || H < 1 || (N > 0 && !KV) || !Sz) {
        set_error("glga_global_stats_static: need 0 <= N < 2^31, H >= 1, non-null KV (when N > 0) and Sz");
        return GLGA_ERR_INVALID_ARG;
    }
    if (io != GLGA_F32 && io != GLGA_BF16) {
        set_error("glga_global_stats_static: io must be GLGA_F32 or GLGA_BF16");
        return GLGA_ERR_INVALID_ARG;
    }
    if (!(r == 8 || r == 16 || r == 32 || r == 64 || r == 128)) {
        set_error("glga_global_stats_static: r must be one of 8, 16, 32, 64, 128 (got %d)", r);
        return GLGA_ERR_UNSUPPORTED;
    }
    const int64_t per_part = static_cast<int64_t>(H) * r * (r + 1);
    if (per_part > static_cast<int64_t>(kStaticScratchFloats)) {
        set_error("glga_global_stats_static: H*r*(r+1)*4 = %lld bytes of partial sums exceed the "
                  "%zu-byte static scratch (use glga_forward, which sizes its own workspace)",
                  static_cast<long long>(per_part * 4), kStaticScratchFloats * sizeof(float));
        return GLGA_ERR_UNSUPPORTED;
    }
    const int elem = io == GLGA_F32 ? 4 : 2;
    const int64_t D = static_cast<int64_t>(H) * r;
    if (N > 0 && (reinterpret_cast<uintptr_t>(KV) & 15u)) {
        set_error("glga_global_stats_static: KV must be 16-byte aligned");
        return GLGA_ERR_INVALID_ARG;
    }
    int dev = 0;
    glga_status st = static_device(&dev);
    if (st != GLGA_OK) return st;
    float *scratch = nullptr;
    unsigned *flag = nullptr;
    int sms = 0;
    st = static_scratch(dev, &scratch, &flag, &sms);
    if (st != GLGA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int parts = 0;
    if (N > 0) {
        const int nblk = static_cast<int>(ceil_div(D, kFB));
        const int rows = io == GLGA_F32 ? StatsGeom<float>::kRows : StatsGeom<__nv_bfloat16>::kRows;
        int64_t per = 0;
        plan_parts(N, nblk, sms, rows, static_cast<int64_t>(kStaticScratchFloats) / per_part, &parts, &per);
        CUtensorMap mk, mv;
        st = encode_kv_maps(KV, N, static_cast<int>(D), elem, &mk, &mv, rows);
        if (st != GLGA_OK) return st;
        StatsParams p;
        p.N = N;
        p.D = static_cast<int32_t>(D);
        p.H = H;
        p.n_parts = parts;
        p.rows_per_part = per;
        p.part_ptr = nullptr;
        p.part_seg = nullptr;
        p.stages = io == GLGA_F32 ? StatsGeom<float>::kStages : StatsGeom<__nv_bfloat16>::kStages;
        p.part = scratch;
        p.flag = flag;
        if (io == GLGA_F32) {
            p.stage_bytes = stage_bytes<float>();
            st = launch_stats<float>(mk, mv, p, sms, nblk, r, s);
        } else {
            p.stage_bytes = stage_bytes<__nv_bfloat16>();
            st = launch_stats<__nv_bfloat16>(mk, mv, p, sms, nblk, r, s);
        }
        if (st != GLGA_OK) return st;
    }
    const int total = static_cast<int>(per_part);
    stats_reduce_kernel<float><<<static_cast<unsigned>(ceil_div(total, 32)), 256, 0, s>>>(
        scratch, parts, nullptr, 1, H, r, static_cast<float *>(Sz), static_cast<float *>(nullptr), 1, 1, 1, 0, 0,
        nullptr);
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

extern "C" glga_status glga_global_stats_static_error(void *stream) {
    using namespace glga;
    int dev = 0;
    glga_status st = static_device(&dev);
    if (st != GLGA_OK) return st;
    float *scratch = nullptr;
    unsigned *flag = nullptr;
    int sms = 0;
    st = static_scratch(dev, &scratch, &flag, &sms);
    if (st != GLGA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned f = 0;
    GLGA_CUDA(cudaMemcpyAsync(&f, flag, sizeof(unsigned), cudaMemcpyDeviceToHost, s));
    GLGA_CUDA(cudaStreamSynchronize(s));
    if (f) {
        GLGA_CUDA(cudaMemsetAsync(flag, 0, sizeof(unsigned), s));
        GLGA_CUDA(cudaStreamSynchronize(s));
    }
    if (f & kDevErrTimeout) {
        set_error("glga_global_stats_static: a bounded device-side wait timed out; the S and z of "
                  "that call are incomplete");
        return GLGA_ERR_TIMEOUT;
    }
    if (f) {
        set_error("glga_global_stats_static: device-side check failed (flags 0x%x)", f);
        return GLGA_ERR_DEVICE;
    }
    return GLGA_OK;
}

extern "C" glga_status glga_debug_static_bounded_wait(int64_t limit_ns, void *stream) {
    using namespace glga;
    if (limit_ns < 1000 || limit_ns > 10000000000LL) {
        set_error("glga_debug_static_bounded_wait: need 1e3 <= limit_ns <= 1e10");
        return GLGA_ERR_INVALID_ARG;
    }
    int dev = 0;
    glga_status st = static_device(&dev);
    if (st != GLGA_OK) return st;
    float *scratch = nullptr;
    unsigned *flag = nullptr;
    int sms = 0;
    st = static_scratch(dev, &scratch, &flag, &sms);
    if (st != GLGA_OK) return st;
    return launch_bounded_wait_probe(flag, static_cast<uint64_t>(limit_ns), static_cast<cudaStream_t>(stream));
}
