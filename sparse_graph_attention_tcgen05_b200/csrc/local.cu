// local.cu -- per-target kernel: the local softmax branch.
//
// Method page "Gated Local-Global Graph Attention", Key formulas:
//   L_i = sum_{j in N(i)} softmax_j(q_i . k_j / sqrt r) v_j
// evaluated per head for every target row and written to L [N, H*r]; the global readout
// and the gate blend run afterwards in the readout GEMM's epilogue (readout.cu).  The
// softmax is the stable one of the tinymesh page ("Target softmax"), computed in a
// single pass: the state (m, l, acc) of a partial sum holds l = sum 2^(x_j - m) and
// acc = sum 2^(x_j - m) v_j for base-2 scores x_j = s_ij log2(e) and a reference m.  Any
// reference gives the same acc / l; m is raised (and l, acc rescaled by 2^(m_old - m_new))
// only when a score exceeds it by more than 2^kTau, so most edge steps skip the rescale
// and every weight stays below 2^kTau.  Two partial states merge the same way, so edges
// may be split across lanes, warps and thread blocks and merged in a fixed order.  No
// per-edge value is stored.
//
// Work is scheduled by the degree buckets built at create time:
//   chunk blocks   bucket-2 rows cut into chunk_edges-edge chunks; each block merges its
//                  8 warps, writes (m, l, acc) to scratch, and the last block of a row
//                  (ticket counter) merges the row's chunks in chunk order and finishes
//   row blocks     bucket-1 rows: 8 warps split the edges, merged in warp order
//   task warps     bucket-0 rows (descending degree) in tasks of <= 32 rows and about
//                  kTaskEdges edges; each edge slot of the warp takes its own row
// Heavy work comes first in block order so it starts early.
//
// Debug instantiations (DBG, chosen by glga_options.debug_checks) check every column
// index they read against [0, N) and every row taken from a schedule list; a bad one
// raises kDevErrBounds on the context's flag and is skipped, so no access leaves its
// buffer.  The default instantiations compile without the checks.
//
// Lane layout: a 16-byte vector holds VE = 16/sizeof(T) consecutive features; an edge's
// k_j (or v_j) row is LPE lanes x VPL vectors; EPW = 32/LPE edge slots per warp; the r
// features of a head live in LPH adjacent lanes, which reduce dot products with butterfly
// shuffles.  In the joint layout (J) a lane's VPL vectors are consecutive features of one
// head, so the lane keeps one softmax state for all of them.  Each slot walks a
// contiguous edge range U edges at a time; the column indices of the next step (and, for
// task rows, the next row's q and first columns) are loaded one step ahead so the
// k_j/v_j gathers do not wait behind them.  Options of the compile-time layouts, chosen per
// shape by measurement: PIPE issues the next step's gathers before the current step is
// consumed (two register buffers), CB loads the column indices of several steps at once.
//
// Arithmetic: q_i and k_j stay in the io type; for bf16 the dot product runs on the
// mixed-precision fma.rn.f32.bf16 (bf16 operands, exact products, f32 accumulation), so
// the gathered rows are never unpacked.  The score scale log2(e)/sqrt(r) is applied to
// the f32 dot product inside the exponent.  The v_j side accumulates in f32 with f32
// weights (bf16 v_j widened exactly).
#include <algorithm>
#include <cmath>
#include <vector>

#include "glga_internal.cuh"

namespace glga {
namespace {

constexpr int kLocalWarps = 8;
constexpr int kLocalThreads = kLocalWarps * 32;
constexpr int kTaskRows = 32;
constexpr int64_t kTaskEdges = 256;
// Start of the running reference: a finite stand-in for -infinity, so that an empty state
// merges without inf - inf.
constexpr float kMInit = -3.0e38f;
// The reference is raised only when a base-2 score exceeds it by more than this.
constexpr float kTau = 8.f;

// d = a * b + c with a and b the bf16 halves (AH / BH: high half) of 32-bit words:
// exact product, one f32 rounding.
template <int AH, int BH>
__device__ __forceinline__ float mfma(uint32_t a, uint32_t b, float c) {
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

// Two f32 values rounded to bf16 (nearest even) in one word: lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t w;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(hi), "f"(lo));
    return w;
}

template <typename T>
struct Io;
template <>
struct Io<float> {
    static constexpr int VE = 4;
    __device__ __forceinline__ static float dot(const uint4 &q, const uint4 &k, float acc) {
        acc = fmaf(__uint_as_float(q.x), __uint_as_float(k.x), acc);
        acc = fmaf(__uint_as_float(q.y), __uint_as_float(k.y), acc);
        acc = fmaf(__uint_as_float(q.z), __uint_as_float(k.z), acc);
        return fmaf(__uint_as_float(q.w), __uint_as_float(k.w), acc);
    }
    __device__ __forceinline__ static void unpack(const uint4 &u, float (&f)[VE]) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[VE]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};
template <>
struct Io<__nv_bfloat16> {
    static constexpr int VE = 8;
    __device__ __forceinline__ static float dot(const uint4 &q, const uint4 &k, float acc) {
        // two chains, so consecutive FMAs do not wait on each other
        float a2 = mfma<1, 1>(q.x, k.x, 0.f);
        acc = mfma<0, 0>(q.x, k.x, acc);
        acc = mfma<0, 0>(q.y, k.y, acc);
        a2 = mfma<1, 1>(q.y, k.y, a2);
        acc = mfma<0, 0>(q.z, k.z, acc);
        a2 = mfma<1, 1>(q.z, k.z, a2);
        acc = mfma<0, 0>(q.w, k.w, acc);
        a2 = mfma<1, 1>(q.w, k.w, a2);
        return acc + a2;
    }
    __device__ __forceinline__ static void unpack(const uint4 &u, float (&f)[VE]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[VE]) {
        return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                          pack_bf16x2(f[6], f[7]));
    }
};

// Per-shape kernel options (bit flags of the OPT template parameter), chosen by
// measurement for each hot shape:
constexpr int kOptWB = 1;   // bf16 softmax weights, two edges per mixed-precision FMA word
constexpr int kOptAsync = 2;   // gathers by cp.async into a two-step shared-memory ring per
                               // warp: the next step's loads wait in shared memory, not in
                               // registers, while the current step is computed

constexpr int kRingSteps = 2;
// Dynamic shared memory of the cp.async ring: [warp][step % 2][U][VPL][k | v][lane] x 16 B.
constexpr size_t async_ring_bytes(int U, int VPL) {
    return static_cast<size_t>(kLocalWarps) * kRingSteps * U * VPL * 2 * 32 * 16;
}


// volatile: the load must stay under its guard (it is never speculated)
__device__ __forceinline__ uint4 ld_gather(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

struct LocalParams {
    const int32_t *row_ptr;
    const int32_t *col_idx;
    const int32_t *warp_rows;
    const int32_t *task_start;   // [n_tasks + 1] positions in warp_rows
    const int32_t *cta_rows;
    const int32_t *chunk_row;
    const int32_t *chunk_begin;
    int64_t n_tasks, n_cta, n_chunks;
    int64_t task_blocks;
    int32_t chunk_edges;
    const void *Q;
    const void *KV;
    float *part;         // per chunk: m[H] l[H] acc[D]
    unsigned *ticket;
    void *L;             // io [N, D] local-branch output
    float *lse;          // [N, H] log-sum-exp of the row's scores for the backward pass, or null
    int32_t D, r, H, nvec, lpe, epw, lph;
    float score_scale;   // log2(e) / sqrt(r)
    int32_t N;           // source nodes: bound of column indices (debug checks)
    int32_t n_rows;      // target rows of this context: bound of scheduled rows (debug checks)
    unsigned *flag;      // device error flag (debug checks)
};

// 2^x by the PTX ex2.approx.ftz instruction.  The arguments are scores minus a reference
// (<= kTau); results below 2^-126 flush to zero.
__device__ __forceinline__ float exp2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A column index read from the CSR; debug builds mask (and report) one outside [0, N).
template <bool DBG>
__device__ __forceinline__ int32_t checked_col(const LocalParams &p, int32_t j) {
    if constexpr (DBG) {
        if (j < 0 || j >= p.N) {
            atomicOr(p.flag, kDevErrBounds);
            return -1;
        }
    }
    return j;
}

// A row taken from a schedule list; debug builds report one outside [0, n_rows).
template <bool DBG>
__device__ __forceinline__ bool row_ok(const LocalParams &p, int64_t row) {
    if constexpr (DBG) {
        if (row < 0 || row >= p.n_rows) {
            atomicOr(p.flag, kDevErrBounds);
            return false;
        }
    }
    return true;
}

constexpr int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Compile-time shape of one instantiation.  NV (16-byte vectors per q/k/v row) and LPH
// (lanes per head) are fixed for the hot shapes and 0 for the generic build, which reads
// them from the parameters.
template <typename T, int NV, int LPH, int VPL, bool J>
struct Shape {
    static constexpr int VE = Io<T>::VE;
    static constexpr int NH = J ? 1 : VPL;   // heads (softmax states) per lane
    __device__ __forceinline__ static int nvec(const LocalParams &p) { return NV ? NV : p.nvec; }
    __device__ __forceinline__ static int lph(const LocalParams &p) { return LPH ? LPH : p.lph; }
    __device__ __forceinline__ static int lpe(const LocalParams &p) {
        if constexpr (NV != 0) return J ? NV / VPL : (NV >= 32 ? 32 : pow2_at_least(NV));
        return p.lpe;
    }
    __device__ __forceinline__ static int epw(const LocalParams &p) { return 32 / lpe(p); }
    // vector index (within a row) of the lane's vector v; its head is vid * VE / r
    __device__ __forceinline__ static int vid(int v, int li) { return J ? li * VPL + v : v * 32 + li; }
    // lanes per edge of a compile-time layout (0: read from the parameters)
    static constexpr int kLpe = NV == 0 ? 0 : (J ? NV / VPL : (NV >= 32 ? 32 : pow2_at_least(NV)));
    // every vector of a compile-time layout that fills its lanes is in range
    static constexpr bool kFull =
        NV != 0 && (J || NV == 32 * VPL || (VPL == 1 && NV < 32 && (NV & (NV - 1)) == 0));
    __device__ __forceinline__ static bool lane_ok(const LocalParams &p, int v, int li) {
        if constexpr (kFull) return true;
        return vid(v, li) < nvec(p);
    }
    // byte offset of the lane's vector v inside a k (or v, q, L) row
    __device__ __forceinline__ static int voff(int v) { return J ? v * 16 : v * 512; }
};

template <typename T, int VPL, bool J>
struct State {
    static constexpr int VE = Io<T>::VE;
    static constexpr int NH = J ? 1 : VPL;
    float m[NH], l[NH], acc[VPL][VE];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            m[h] = kMInit;
            l[h] = 0.f;
        }
#pragma unroll
        for (int v = 0; v < VPL; ++v)
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[v][e] = 0.f;
    }
    __device__ __forceinline__ static constexpr int head_of(int v) { return J ? 0 : v; }
    // merge another partial state (m2, l2, a2) into this one
    __device__ __forceinline__ void merge(const float (&m2)[NH], const float (&l2)[NH], const float (&a2)[VPL][VE]) {
        float c1[NH], c2[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const float mn = fmaxf(m[h], m2[h]);
            c1[h] = exp2_ftz(m[h] - mn);
            c2[h] = exp2_ftz(m2[h] - mn);
            l[h] = l[h] * c1[h] + l2[h] * c2[h];
            m[h] = mn;
        }
#pragma unroll
        for (int v = 0; v < VPL; ++v)
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[v][e] = acc[v][e] * c1[head_of(v)] + a2[v][e] * c2[head_of(v)];
    }
};

struct Lane {
    int lane, slot, li;
};

// Column indices of a slot's range as held by the lanes that later broadcast them: lane
// li (< CB) of the slot holds col_idx[e0 + li].  CB = U (one step's edges) for runtime
// layouts, the slot's lane count for compile-time ones (a batch of several steps).
template <int CB, bool DBG>
__device__ __forceinline__ int32_t first_cols(const LocalParams &p, int64_t e0, int64_t e1, const Lane &ln) {
    return (ln.li < CB && e0 + ln.li < e1) ? checked_col<DBG>(p, __ldg(p.col_idx + e0 + ln.li)) : -1;
}

// Column indices per load: a batch of the slot's LPE lanes (CB, compile-time layouts
// only) or one step's U.
template <typename T, int NV, int LPH, int VPL, int U, bool J, bool CB>
constexpr int col_batch() {
    return (CB && Shape<T, NV, LPH, VPL, J>::kLpe != 0) ? Shape<T, NV, LPH, VPL, J>::kLpe : U;
}

// One slot walks the CSR entries [e0, e1) U at a time (the trip count is the warp's
// maximum over slots); `cols` holds the first column batch (first_cols).  With PIPE the
// k_j / v_j gathers of step i + 1 are issued before step i is consumed (two register
// buffers), so a warp keeps a step's loads in flight while it computes the previous one.
// On return each lane holds its slot's partial state for its feature vectors.
template <typename T, int NV, int LPH, int VPL, int U, bool DBG, bool J, bool PIPE, bool CB, int OPT>
__device__ __forceinline__ void slot_edges(const LocalParams &p, const uint4 (&q)[VPL], int64_t e0,
                                           int64_t e1, int32_t cols, const Lane &ln,
                                           State<T, VPL, J> &st) {
    using Sh = Shape<T, NV, LPH, VPL, J>;
    using St = State<T, VPL, J>;
    constexpr int VE = Io<T>::VE;
    constexpr int NH = Sh::NH;
    st.init();
    const int iters_mine = e1 > e0 ? static_cast<int>((e1 - e0 + U - 1) / U) : 0;
    const int iters = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(iters_mine));
    const int nvec = Sh::nvec(p);
    const uint32_t row_bytes = 32u * static_cast<uint32_t>(nvec);   // k_j | v_j
    const char *kvl = static_cast<const char *>(p.KV) + 16 * Sh::vid(0, ln.li);
    const int src0 = ln.slot * Sh::lpe(p);
    const int lph = Sh::lph(p);
    const float scale = p.score_scale;
    bool ok[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) ok[v] = Sh::lane_ok(p, v, ln.li);
    // column indices arrive in batches of NB edges (NB / U steps each; NB = U without
    // batching); the next batch is loaded while the current one is used.  The batches
    // follow the load stream.
    constexpr int NB = col_batch<T, NV, LPH, VPL, U, J, CB>();
    constexpr int PER = NB / U;
    static_assert(NB % U == 0, "a batch holds whole steps");
    int32_t c_cur = cols;
    int32_t c_next = -1;
    if (PER > 1 && iters > PER) {
        const int64_t nb = e0 + NB;
        c_next = (ln.li < NB && nb + ln.li < e1) ? checked_col<DBG>(p, __ldg(p.col_idx + nb + ln.li)) : -1;
    }
    // issues the gathers of step `step` into (kb, vb); jb gets its column indices (-1:
    // no edge; such a slot keeps its previous, finite contents and gets weight 0)
    // the column indices of step `step` (taken in step order)
    auto cols_of = [&](int step, int32_t (&jb)[U]) {
        const int sub = PER > 1 ? step % PER : 0;
#pragma unroll
        for (int u = 0; u < U; ++u) jb[u] = __shfl_sync(0xffffffffu, c_cur, src0 + sub * U + u);
        if (sub == PER - 1) {
            if (PER > 1) {
                c_cur = c_next;
                const int64_t nb = e0 + static_cast<int64_t>(step / PER + 2) * NB;
                c_next = (ln.li < NB && nb + ln.li < e1) ? checked_col<DBG>(p, __ldg(p.col_idx + nb + ln.li)) : -1;
            } else {
                const int64_t nb = e0 + static_cast<int64_t>(step + 1) * U;
                c_cur = (ln.li < U && nb + ln.li < e1) ? checked_col<DBG>(p, __ldg(p.col_idx + nb + ln.li)) : -1;
            }
        }
    };
    auto load = [&](int step, uint4 (&kb)[U][VPL], uint4 (&vb)[U][VPL], int32_t (&jb)[U]) {
        cols_of(step, jb);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (jb[u] >= 0) {
                const char *rowp = kvl + static_cast<size_t>(static_cast<uint32_t>(jb[u])) * row_bytes;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    if (ok[v]) {
                        kb[u][v] = ld_gather(rowp + Sh::voff(v));
                        vb[u][v] = ld_gather(rowp + 16 * nvec + Sh::voff(v));
                    }
                }
            }
        }
    };
    // folds one step's edges into the state
    auto consume = [&](const uint4 (&kb)[U][VPL], const uint4 (&vb)[U][VPL], const int32_t (&jb)[U]) {
        // scores (f32 dot products, unscaled), reduced over the head's lanes
        float sc[U][NH];
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                float dot = 0.f;
#pragma unroll
                for (int v = 0; v < VPL; ++v)
                    if (St::head_of(v) == h) dot = Io<T>::dot(q[v], kb[u][v], dot);
                if constexpr (LPH != 0) {
#pragma unroll
                    for (int o = 1; o < LPH; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                } else {
                    for (int o = 1; o < lph; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                }
                sc[u][h] = (jb[u] >= 0) ? dot : -INFINITY;
            }
        }
        // raise the reference only when a score exceeds it by more than kTau
        float mx[NH];
        bool need = false;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            mx[h] = sc[0][h];
#pragma unroll
            for (int u = 1; u < U; ++u) mx[h] = fmaxf(mx[h], sc[u][h]);
            mx[h] *= scale;
            need |= mx[h] > st.m[h] + kTau;
        }
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const float mn = fmaxf(st.m[h], mx[h]);
                const float corr = exp2_ftz(st.m[h] - mn);
                st.l[h] *= corr;
                st.m[h] = mn;
#pragma unroll
                for (int v = 0; v < VPL; ++v)
                    if (St::head_of(v) == h)
#pragma unroll
                        for (int e = 0; e < VE; ++e) st.acc[v][e] *= corr;
            }
        }
        if constexpr (sizeof(T) == 2 && (OPT & kOptWB) != 0) {
            // weights rounded to bf16 (as attention kernels round P before the P V
            // product), two edges per 32-bit word on the mixed-precision FMA; l sums
            // exactly the rounded weights, so each row's weights still sum to one
            constexpr uint32_t kOne = 0x3f803f80u;
#pragma unroll
            for (int u = 0; u < U; u += 2) {
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const float p0 = exp2_ftz(fmaf(sc[u][h], scale, -st.m[h]));
                    const float p1 = u + 1 < U ? exp2_ftz(fmaf(sc[u + 1][h], scale, -st.m[h])) : 0.f;
                    const uint32_t w = pack_bf16x2(p0, p1);
                    st.l[h] = mfma<0, 0>(w, kOne, st.l[h]);
                    if (u + 1 < U) st.l[h] = mfma<1, 0>(w, kOne, st.l[h]);
#pragma unroll
                    for (int v = 0; v < VPL; ++v) {
                        if (St::head_of(v) != h) continue;
                        const uint32_t a[4] = {vb[u][v].x, vb[u][v].y, vb[u][v].z, vb[u][v].w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            st.acc[v][2 * i] = mfma<0, 0>(w, a[i], st.acc[v][2 * i]);
                            st.acc[v][2 * i + 1] = mfma<0, 1>(w, a[i], st.acc[v][2 * i + 1]);
                        }
                        if (u + 1 < U) {
                            const uint32_t b[4] = {vb[u + 1][v].x, vb[u + 1][v].y, vb[u + 1][v].z, vb[u + 1][v].w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                st.acc[v][2 * i] = mfma<1, 0>(w, b[i], st.acc[v][2 * i]);
                                st.acc[v][2 * i + 1] = mfma<1, 1>(w, b[i], st.acc[v][2 * i + 1]);
                            }
                        }
                    }
                }
            }
            return;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float pr[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                pr[h] = exp2_ftz(fmaf(sc[u][h], scale, -st.m[h]));
                st.l[h] += pr[h];
            }
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const float w = pr[St::head_of(v)];
                float vf[VE];
                Io<T>::unpack(vb[u][v], vf);
#pragma unroll
                for (int e = 0; e < VE; ++e) st.acc[v][e] = fmaf(w, vf[e], st.acc[v][e]);
            }
        }
    };
    uint4 kA[U][VPL], vA[U][VPL];
    int32_t jA[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
        for (int v = 0; v < VPL; ++v) kA[u][v] = vA[u][v] = make_uint4(0, 0, 0, 0);
    if constexpr ((OPT & kOptAsync) != 0 && !PIPE) {
        // this lane's slots of the warp's ring (written and read by the lane alone, so the
        // lane's own cp.async.wait_group makes them visible; never-written slots hold
        // zeros or an earlier edge's finite values and get weight 0)
        constexpr int S = kRingSteps;
        extern __shared__ uint4 local_ring[];
        uint4 *ring = local_ring + (threadIdx.x >> 5) * (S * U * VPL * 2 * 32) + ln.lane;
        auto slot = [&](int stage, int u, int v, int kv) { return ring + (((stage * U + u) * VPL + v) * 2 + kv) * 32; };
        auto issue = [&](int step, int32_t (&jb)[U]) {
            cols_of(step, jb);
            const int stage = step % S;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (jb[u] >= 0) {
                    const char *rowp = kvl + static_cast<size_t>(static_cast<uint32_t>(jb[u])) * row_bytes;
#pragma unroll
                    for (int v = 0; v < VPL; ++v) {
                        if (ok[v]) {
                            cp_async16(slot(stage, u, v, 0), rowp + Sh::voff(v));
                            cp_async16(slot(stage, u, v, 1), rowp + 16 * nvec + Sh::voff(v));
                        }
                    }
                }
            }
            cp_async_commit();
        };
        // step it + 1's gathers are issued before step it is waited for and consumed
        int32_t jN[U];
        if (iters > 0) issue(0, jA);
        for (int it = 0; it < iters; ++it) {
            if (it + 1 < iters) {
                issue(it + 1, jN);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            const int stage = it % S;
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    kA[u][v] = *slot(stage, u, v, 0);
                    vA[u][v] = *slot(stage, u, v, 1);
                }
            consume(kA, vA, jA);
            if (it + 1 < iters) {
#pragma unroll
                for (int u = 0; u < U; ++u) jA[u] = jN[u];
            }
        }
    } else if constexpr (!PIPE) {
        for (int it = 0; it < iters; ++it) {
            load(it, kA, vA, jA);
            consume(kA, vA, jA);
        }
    } else {
        uint4 kB[U][VPL], vB[U][VPL];
        int32_t jB[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int v = 0; v < VPL; ++v) kB[u][v] = vB[u][v] = make_uint4(0, 0, 0, 0);
        if (iters > 0) load(0, kA, vA, jA);
        for (int it = 0; it < iters; it += 2) {
            if (it + 1 < iters) load(it + 1, kB, vB, jB);
            consume(kA, vA, jA);
            if (it + 1 < iters) {
                if (it + 2 < iters) load(it + 2, kA, vA, jA);
                consume(kB, vB, jB);
            }
        }
    }
}

// Merges the edge slots of the warp (lanes li, li + LPE, ...): afterwards every lane
// holds the state over all slots.
template <typename T, int NV, int LPH, int VPL, bool J>
__device__ __forceinline__ void merge_slots(const LocalParams &p, State<T, VPL, J> &st) {
    using Sh = Shape<T, NV, LPH, VPL, J>;
    constexpr int VE = Io<T>::VE;
    constexpr int NH = Sh::NH;
    for (int o = Sh::lpe(p); o < 32; o <<= 1) {
        float m2[NH], l2[NH], a2[VPL][VE];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            m2[h] = __shfl_xor_sync(0xffffffffu, st.m[h], o);
            l2[h] = __shfl_xor_sync(0xffffffffu, st.l[h], o);
        }
#pragma unroll
        for (int v = 0; v < VPL; ++v)
#pragma unroll
            for (int e = 0; e < VE; ++e) a2[v][e] = __shfl_xor_sync(0xffffffffu, st.acc[v][e], o);
        st.merge(m2, l2, a2);
    }
}

template <typename T, int NV, int LPH, int VPL, bool J, int OPT>
__device__ __forceinline__ void load_q(const LocalParams &p, int64_t row, const Lane &ln, bool valid,
                                       uint4 (&qr)[VPL]) {
    using Sh = Shape<T, NV, LPH, VPL, J>;
    const char *Q = static_cast<const char *>(p.Q) + row * 16 * Sh::nvec(p) + 16 * Sh::vid(0, ln.li);
#pragma unroll
    for (int v = 0; v < VPL; ++v)
        qr[v] = (valid && Sh::lane_ok(p, v, ln.li)) ? __ldg(reinterpret_cast<const uint4 *>(Q + Sh::voff(v)))
                                                    : make_uint4(0, 0, 0, 0);
}

// lse_i = ln sum_j exp(s_ij) per head, ln 2 (m + log2 l) since the state keeps base-2
// scores (0 for a row without edges), from the vector holding the head's first features.
// Compiled in only for the LSE instantiations (contexts made for the backward pass), so
// the plain forward's code is untouched.
template <typename T, int NV, int LPH, int VPL, bool J, bool LSE>
__device__ __forceinline__ void store_lse(const LocalParams &p, int64_t row, const State<T, VPL, J> &st,
                                          const Lane &ln, bool mine) {
    if constexpr (!LSE) return;
    using Sh = Shape<T, NV, LPH, VPL, J>;
    constexpr int VE = Io<T>::VE;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int vid = Sh::vid(v, ln.li);
        const int h = State<T, VPL, J>::head_of(v);
        if (mine && Sh::lane_ok(p, v, ln.li) && (vid * VE) % p.r == 0)
            p.lse[row * p.H + vid * VE / p.r] =
                st.l[h] > 0.f ? 0.69314718055994531f * (st.m[h] + __log2f(st.l[h])) : 0.f;
    }
}

// L_i = acc / l per head (0 for a row without edges), stored from lanes with `mine`.
template <typename T, int NV, int LPH, int VPL, bool J, bool LSE, int OPT>
__device__ __forceinline__ void finish_row(const LocalParams &p, int64_t row, const State<T, VPL, J> &st,
                                           const Lane &ln, bool mine) {
    using Sh = Shape<T, NV, LPH, VPL, J>;
    constexpr int VE = Io<T>::VE;
    constexpr int NH = Sh::NH;
    float inv_l[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) inv_l[h] = st.l[h] > 0.f ? 1.f / st.l[h] : 0.f;
    char *Lout = static_cast<char *>(p.L) + row * 16 * Sh::nvec(p) + 16 * Sh::vid(0, ln.li);
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        float y[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) y[e] = st.acc[v][e] * inv_l[State<T, VPL, J>::head_of(v)];
        if (mine && Sh::lane_ok(p, v, ln.li)) *reinterpret_cast<uint4 *>(Lout + Sh::voff(v)) = Io<T>::pack(y);
    }
    store_lse<T, NV, LPH, VPL, J, LSE>(p, row, st, ln, mine);
}

template <typename T, int VPL, bool J>
struct BlockScratch {
    static constexpr int VE = Io<T>::VE;
    static constexpr int NH = J ? 1 : VPL;
    float m[kLocalWarps][NH][32];
    float l[kLocalWarps][NH][32];
    float acc[kLocalWarps][VPL][VE][32];
};

// 8 warps split [e0, e1) (each warp's share split again across its slots); warp 0
// returns the merge of all warps in warp order.
template <typename T, int NV, int LPH, int VPL, int U, bool DBG, bool J, bool PIPE, bool CB, int OPT>
__device__ __forceinline__ void block_edges(const LocalParams &p, const uint4 (&q)[VPL], int64_t e0,
                                            int64_t e1, const Lane &ln, int warp,
                                            BlockScratch<T, VPL, J> &sh, State<T, VPL, J> &st) {
    using Sh = Shape<T, NV, LPH, VPL, J>;
    constexpr int VE = Io<T>::VE;
    constexpr int NH = Sh::NH;
    const int64_t per = ceil_div(e1 - e0, kLocalWarps);
    const int64_t a = std::min(e1, e0 + warp * per), b = std::min(e1, a + per);
    const int64_t per_s = ceil_div(b - a, Sh::epw(p));
    const int64_t sa = std::min(b, a + ln.slot * per_s), sb = std::min(b, sa + per_s);
    slot_edges<T, NV, LPH, VPL, U, DBG, J, PIPE, CB, OPT>(p, q, sa, sb,
                                               first_cols<col_batch<T, NV, LPH, VPL, U, J, CB>(), DBG>(p, sa, sb, ln),
                                               ln, st);
    merge_slots<T, NV, LPH, VPL, J>(p, st);
#pragma unroll
    for (int h = 0; h < NH; ++h) {
        sh.m[warp][h][ln.lane] = st.m[h];
        sh.l[warp][h][ln.lane] = st.l[h];
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v)
#pragma unroll
        for (int e = 0; e < VE; ++e) sh.acc[warp][v][e][ln.lane] = st.acc[v][e];
    __syncthreads();
    if (warp == 0) {
        for (int w = 1; w < kLocalWarps; ++w) {
            float m2[NH], l2[NH], a2[VPL][VE];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                m2[h] = sh.m[w][h][ln.lane];
                l2[h] = sh.l[w][h][ln.lane];
            }
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VE; ++e) a2[v][e] = sh.acc[w][v][e][ln.lane];
            st.merge(m2, l2, a2);
        }
    }
}

// Blocks per SM the register budget aims at: 3 (at most 85 registers) while the gather
// buffers take at most 32 registers (8 per edge step and vector, doubled when pipelined),
// else 2.
constexpr int local_min_blocks(int VPL, int U, bool PIPE) {
    return ((PIPE ? 2 : 1) * U * VPL * 8 <= 32 && VPL <= 2) ? 3 : 2;
}
// The gather-ring layout with one vector per lane runs four blocks per SM (64 registers);
// the log-sum-exp store would otherwise take it to 71 registers and three blocks.
constexpr int local_min_blocks_opt(int VPL, int U, bool PIPE, bool LSE, int OPT) {
    return (LSE && (OPT & kOptAsync) != 0 && VPL == 1 && U <= 2 && !PIPE) ? 4 : local_min_blocks(VPL, U, PIPE);
}
template <typename T, int NV, int LPH, int VPL, int U, bool DBG, bool J, bool LSE, bool PIPE, bool CB, int OPT>
__global__ void __launch_bounds__(kLocalThreads, local_min_blocks_opt(VPL, U, PIPE, LSE, OPT))
    local_kernel(const LocalParams p) {
    using Sh = Shape<T, NV, LPH, VPL, J>;
    using St = State<T, VPL, J>;
    constexpr int VE = Io<T>::VE;
    constexpr int NH = Sh::NH;
    __shared__ BlockScratch<T, VPL, J> sh;
    const int warp = threadIdx.x >> 5;
    Lane ln;
    ln.lane = threadIdx.x & 31;
    ln.slot = ln.lane / Sh::lpe(p);
    ln.li = ln.lane % Sh::lpe(p);
    if constexpr ((OPT & kOptAsync) != 0) {
        // the gather ring starts at zero (slots of masked edges are read with weight 0)
        extern __shared__ uint4 local_ring[];
        constexpr int S = kRingSteps;
        uint4 *ring = local_ring + warp * (S * U * VPL * 2 * 32) + ln.lane;
#pragma unroll
        for (int k = 0; k < S * U * VPL * 2; ++k) ring[k * 32] = make_uint4(0u, 0u, 0u, 0u);
    }
    int64_t bid = blockIdx.x;
    uint4 q[VPL];
    St st;

    if (bid < p.n_chunks) {
        // ---------------- chunk of a bucket-2 row ----------------
        const int64_t c = bid;
        const int64_t row = p.chunk_row[c];
        if (!row_ok<DBG>(p, row)) return;
        const int64_t rb = p.row_ptr[row], re = p.row_ptr[row + 1];
        const int64_t e0 = p.chunk_begin[c];
        const int64_t e1 = std::min<int64_t>(re, e0 + p.chunk_edges);
        const int64_t nch = ceil_div(re - rb, p.chunk_edges);
        const int64_t first = c - (e0 - rb) / p.chunk_edges;
        load_q<T, NV, LPH, VPL, J, OPT>(p, row, ln, true, q);
        block_edges<T, NV, LPH, VPL, U, DBG, J, PIPE, CB, OPT>(p, q, e0, e1, ln, warp, sh, st);
        const int64_t stride = 2 * p.H + p.D;
        if (warp == 0) {
            float *dst = p.part + c * stride;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const int vid = Sh::vid(v, ln.li);
                if (Sh::lane_ok(p, v, ln.li) && ln.slot == 0) {
#pragma unroll
                    for (int e = 0; e < VE; ++e) dst[2 * p.H + vid * VE + e] = st.acc[v][e];
                    if ((vid * VE) % p.r == 0) {
                        const int h = vid * VE / p.r;
                        dst[h] = st.m[St::head_of(v)];
                        dst[p.H + h] = st.l[St::head_of(v)];
                    }
                }
            }
            __threadfence();
            __syncwarp();
            int last = 0;
            if (ln.lane == 0) {
                const unsigned prev = atomicAdd(p.ticket + first, 1u);
                last = (prev == static_cast<unsigned>(nch - 1));
                if (last) p.ticket[first] = 0u;   // ready for the next forward
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                __threadfence();
                st.init();
                for (int64_t k = 0; k < nch; ++k) {
                    const float *src = p.part + (first + k) * stride;
                    float m2[NH], l2[NH], a2[VPL][VE];
#pragma unroll
                    for (int v = 0; v < VPL; ++v) {
                        const int vid = Sh::vid(v, ln.li);
                        const bool okv = Sh::lane_ok(p, v, ln.li);
                        const int h = okv ? vid * VE / p.r : 0;
#pragma unroll
                        for (int e = 0; e < VE; ++e) a2[v][e] = okv ? __ldcg(src + 2 * p.H + vid * VE + e) : 0.f;
                        if (St::head_of(v) == v || v == 0) {
                            m2[St::head_of(v)] = okv ? __ldcg(src + h) : kMInit;
                            l2[St::head_of(v)] = okv ? __ldcg(src + p.H + h) : 0.f;
                        }
                    }
                    st.merge(m2, l2, a2);
                }
                finish_row<T, NV, LPH, VPL, J, LSE, OPT>(p, row, st, ln, ln.slot == 0);
            }
        }
        return;
    }
    bid -= p.n_chunks;
    if (bid < p.n_cta) {
        // ---------------- bucket-1 row: one block ----------------
        const int64_t row = p.cta_rows[bid];
        if (!row_ok<DBG>(p, row)) return;
        load_q<T, NV, LPH, VPL, J, OPT>(p, row, ln, true, q);
        block_edges<T, NV, LPH, VPL, U, DBG, J, PIPE, CB, OPT>(p, q, p.row_ptr[row], p.row_ptr[row + 1], ln, warp, sh, st);
        if (warp == 0) finish_row<T, NV, LPH, VPL, J, LSE, OPT>(p, row, st, ln, ln.slot == 0);
        return;
    }
    bid -= p.n_cta;
    // ---------------- bucket-0 task: up to 32 rows, one per slot per step ----------------
    const int64_t task = bid * kLocalWarps + warp;
    if (task >= p.n_tasks) return;
    const int t0 = p.task_start[task];
    const int n = p.task_start[task + 1] - t0;
    const int epw = Sh::epw(p);
    int32_t myrow = 0, mybeg = 0, myend = 0;
    if (ln.lane < n) {
        myrow = __ldg(p.warp_rows + t0 + ln.lane);
        if (row_ok<DBG>(p, myrow)) {
            mybeg = __ldg(p.row_ptr + myrow);
            myend = __ldg(p.row_ptr + myrow + 1);
        } else {
            myrow = -1;   // (debug only) no edges, no output
        }
    }
    const int steps = (n + epw - 1) / epw;
    // step 0 prefetch: this slot's first row
    int k = ln.slot;
    int32_t row = __shfl_sync(0xffffffffu, myrow, k & 31);
    int32_t beg = __shfl_sync(0xffffffffu, mybeg, k & 31);
    int32_t end = __shfl_sync(0xffffffffu, myend, k & 31);
    if (k >= n) beg = end = 0;
    uint4 qn[VPL];
    load_q<T, NV, LPH, VPL, J, OPT>(p, row, ln, k < n && (!DBG || row >= 0), qn);
    int32_t cols = first_cols<col_batch<T, NV, LPH, VPL, U, J, CB>(), DBG>(p, beg, end, ln);
    for (int step = 0; step < steps; ++step) {
        const bool valid = k < n;
        const int32_t row_c = row;
        const int64_t beg_c = beg, end_c = end;
        const int32_t cols_c = cols;
#pragma unroll
        for (int v = 0; v < VPL; ++v) q[v] = qn[v];
        // prefetch the next step's row while this one's gathers are in flight
        k += epw;
        row = __shfl_sync(0xffffffffu, myrow, k & 31);
        beg = __shfl_sync(0xffffffffu, mybeg, k & 31);
        end = __shfl_sync(0xffffffffu, myend, k & 31);
        if (k >= n) beg = end = 0;
        load_q<T, NV, LPH, VPL, J, OPT>(p, row, ln, k < n && (!DBG || row >= 0), qn);
        cols = first_cols<col_batch<T, NV, LPH, VPL, U, J, CB>(), DBG>(p, beg, end, ln);
        slot_edges<T, NV, LPH, VPL, U, DBG, J, PIPE, CB, OPT>(p, q, beg_c, end_c, cols_c, ln, st);
        // every slot finishes its own row
        if (valid && (!DBG || row_c >= 0)) finish_row<T, NV, LPH, VPL, J, LSE, OPT>(p, row_c, st, ln, true);
    }
}

template <typename T, int NV, int LPH, int VPL, int U, bool J, bool PIPE = false, bool CB = false, int OPT = 0>
glga_status launch_local(Ctx *c, LocalParams p, cudaStream_t s) {
    using Sh = Shape<T, NV, LPH, VPL, J>;
    if constexpr (NV != 0) {
        // compile-time layout: its lane geometry replaces the generic one
        p.lpe = Sh::kLpe;
        p.epw = 32 / Sh::kLpe;
        p.lph = LPH != 0 ? LPH : p.r / (Io<T>::VE * (J ? VPL : 1));
    }
    const int64_t blocks = p.n_chunks + p.n_cta + p.task_blocks;
    if (blocks == 0) return GLGA_OK;
    const unsigned g = static_cast<unsigned>(blocks);
    const size_t dyn = (OPT & kOptAsync) != 0 ? async_ring_bytes(U, VPL) : 0;
    auto go = [&](auto kern) -> glga_status {
        if (dyn > 0) GLGA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn)));
        kern<<<g, kLocalThreads, dyn, s>>>(p);
        return GLGA_OK;
    };
    glga_status st;
    if (c->opts.debug_checks) {
        st = p.lse ? go(local_kernel<T, NV, LPH, VPL, U, true, J, true, PIPE, CB, OPT>)
                   : go(local_kernel<T, NV, LPH, VPL, U, true, J, false, PIPE, CB, OPT>);
    } else {
        st = p.lse ? go(local_kernel<T, NV, LPH, VPL, U, false, J, true, PIPE, CB, OPT>)
                   : go(local_kernel<T, NV, LPH, VPL, U, false, J, false, PIPE, CB, OPT>);
    }
    if (st != GLGA_OK) return st;
    GLGA_CUDA(cudaGetLastError());
    c->launches += 1;
    return GLGA_OK;
}

}  // namespace

glga_status local_setup(Ctx *c) {
    const int64_t nc = c->nb[3];
    glga_status st = GLGA_OK;
    if (nc > 0) {
        st = dev_alloc(c, reinterpret_cast<void **>(&c->chunk_part),
                       static_cast<size_t>(nc) * (2 * c->H + c->D) * sizeof(float));
        if (st == GLGA_OK)
            st = dev_alloc(c, reinterpret_cast<void **>(&c->chunk_ticket), nc * sizeof(unsigned));
        if (st == GLGA_OK) {
            cudaError_t e = cudaMemset(c->chunk_ticket, 0, nc * sizeof(unsigned));
            if (e != cudaSuccess) return cuda_fail(e, "ticket init");
        }
    }
    if (st != GLGA_OK) return st;
    // bucket-0 tasks: consecutive rows of the (descending-degree) list, at most kTaskRows
    // rows and about kTaskEdges edges each
    const int64_t n0 = c->nb[0];
    std::vector<int32_t> ts(1, 0);
    if (n0 > 0) {
        std::vector<int32_t> rp(static_cast<size_t>(c->N) + 1), rows(static_cast<size_t>(n0));
        cudaError_t e = cudaMemcpy(rp.data(), c->row_ptr, rp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
        if (e == cudaSuccess)
            e = cudaMemcpy(rows.data(), c->warp_rows, rows.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "task build");
        int cnt = 0;
        int64_t edges = 0;
        for (int64_t i = 0; i < n0; ++i) {
            const int64_t deg = rp[rows[i] + 1] - rp[rows[i]];
            if (cnt > 0 && (cnt == kTaskRows || edges + deg > kTaskEdges)) {
                ts.push_back(static_cast<int32_t>(i));
                cnt = 0;
                edges = 0;
            }
            ++cnt;
            edges += deg;
        }
        ts.push_back(static_cast<int32_t>(n0));
    }
    c->n_tasks = static_cast<int64_t>(ts.size()) - 1;
    st = dev_alloc(c, reinterpret_cast<void **>(&c->task_start), ts.size() * sizeof(int32_t));
    if (st != GLGA_OK) return st;
    cudaError_t e = cudaMemcpy(c->task_start, ts.data(), ts.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "task upload");
    return GLGA_OK;
}

glga_status local_run(Ctx *c, cudaStream_t s) {
    LocalParams p;
    p.row_ptr = c->row_ptr;
    p.col_idx = c->col_idx;
    p.warp_rows = c->warp_rows;
    p.task_start = c->task_start;
    p.cta_rows = c->cta_rows;
    p.chunk_row = c->chunk_row;
    p.chunk_begin = c->chunk_begin;
    p.n_tasks = c->n_tasks;
    p.n_cta = c->nb[1];
    p.n_chunks = c->nb[3];
    p.task_blocks = ceil_div(p.n_tasks, kLocalWarps);
    p.chunk_edges = c->opts.chunk_edges;
    p.Q = c->Q;
    p.KV = c->KV;
    p.part = c->chunk_part;
    p.ticket = c->chunk_ticket;
    p.L = c->L;
    p.lse = c->opts.backward ? c->bw_lse : nullptr;
    p.D = c->D;
    p.r = c->r;
    p.H = c->H;
    const int VE = 16 / c->elem;
    p.nvec = c->D / VE;
    int lpe = 1;
    while (lpe < p.nvec && lpe < 32) lpe <<= 1;
    p.lpe = lpe;
    p.epw = 32 / lpe;
    p.lph = c->r / VE;
    p.score_scale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->r)));
    p.N = static_cast<int32_t>(c->n_src);   // column indices range over all source nodes
    p.n_rows = static_cast<int32_t>(c->N);
    p.flag = c->dev_flag;
    const int vpl = static_cast<int>(ceil_div(p.nvec, 32));
    if (c->io == GLGA_BF16) {
        using B = __nv_bfloat16;
        // hot shapes with compile-time layouts, chosen by measurement: a lane's vector
        // interleaved across the row (D = 128 and 256: one vector per lane, 2 edges per
        // step, 64 registers); at D = 512 two consecutive vectors of one head per lane,
        // the next step's gathers issued before the current one is consumed, column
        // indices in batches
        // (D = 128 and 256: gathers through the cp.async ring, 2 edges per slot step;
        // D = 128 also with bf16 weights)
        if (p.nvec == 16 && c->r == 32) return launch_local<B, 16, 4, 1, 2, false, false, false, kOptWB | kOptAsync>(c, p, s);
        if (p.nvec == 32 && c->r == 32) return launch_local<B, 32, 4, 1, 2, false, false, false, kOptAsync>(c, p, s);
        if (p.nvec == 64 && c->r == 64) return launch_local<B, 64, 4, 2, 2, true, true, true>(c, p, s);
        if (p.nvec == 64 && c->r >= 16) return launch_local<B, 64, 0, 2, 2, true, false>(c, p, s);
        if (vpl == 1 && lpe >= 4) return launch_local<B, 0, 0, 1, 4, false, false>(c, p, s);
        if (vpl == 1 && lpe == 2) return launch_local<B, 0, 0, 1, 2, false, false>(c, p, s);
        if (vpl == 1) return launch_local<B, 0, 0, 1, 1, false, false>(c, p, s);
        if (vpl == 2) return launch_local<B, 0, 0, 2, 2, false, false>(c, p, s);
        if (vpl <= 4) return launch_local<B, 0, 0, 4, 1, false, false>(c, p, s);
    } else {
        // U edges per slot step; U <= LPE so the slot's lanes can hold its column indices
        if (vpl == 1 && lpe >= 4) return launch_local<float, 0, 0, 1, 4, false, false>(c, p, s);
        if (vpl == 1 && lpe == 2) return launch_local<float, 0, 0, 1, 2, false, false>(c, p, s);
        if (vpl == 1) return launch_local<float, 0, 0, 1, 1, false, false>(c, p, s);
        if (vpl == 2) return launch_local<float, 0, 0, 2, 2, false, false>(c, p, s);
        if (vpl <= 4) return launch_local<float, 0, 0, 4, 1, false, false>(c, p, s);
    }
    set_error("row width too large for the local kernel");
    return GLGA_ERR_UNSUPPORTED;
}

}  // namespace glga
