// local.cu -- per-target kernel: the local softmax branch.
//
// Method page "Gated Local-Global Graph Attention", Key formulas:
//   L_i = sum_{j in N(i)} softmax_j(q_i . k_j / sqrt r) v_j
// evaluated per head for every target row and written to L [N, H*r]; the global readout
// and the gate blend run afterwards in the readout GEMM's epilogue (readout.cu).  The
// softmax is the stable one of the tinymesh page ("Target softmax"), computed in a
// single pass with a running maximum: the state (m, l, acc) of a partial sum is rescaled
// by 2^(m_old - m_new) whenever the maximum grows, and two partial states merge the same
// way, so edges may be split across lanes, warps and thread blocks and merged in a fixed
// order.  No per-edge value is stored.
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
// features of a head live in LPH = r/VE adjacent lanes, which reduce dot products with
// butterfly shuffles.  Each slot walks a contiguous edge range U edges at a time; the
// column indices of the next step (and, for task rows, the next row's q and first
// columns) are loaded one step ahead so the k_j/v_j gathers do not wait behind them.
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

template <typename T>
struct Io;
template <>
struct Io<float> {
    static constexpr int VE = 4;
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
    __device__ __forceinline__ static void unpack(const uint4 &u, float (&f)[VE]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[VE]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

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

// 2^x by the PTX ex2.approx.ftz instruction.  The arguments are differences from a
// running maximum (<= 0); results below 2^-126 of the maximum flush to zero.
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

template <typename T, int VPL>
struct State {
    static constexpr int VE = Io<T>::VE;
    float m[VPL], l[VPL], acc[VPL][VE];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            m[v] = -INFINITY;
            l[v] = 0.f;
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[v][e] = 0.f;
        }
    }
    // merge another partial state into this one (per vector)
    __device__ __forceinline__ void merge(int v, float m2, float l2, const float (&a2)[VE]) {
        const float mn = fmaxf(m[v], m2);
        if (mn == -INFINITY) return;
        const float c1 = exp2_ftz(m[v] - mn), c2 = exp2_ftz(m2 - mn);
        l[v] = l[v] * c1 + l2 * c2;
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[v][e] = acc[v][e] * c1 + a2[e] * c2;
        m[v] = mn;
    }
};

struct Lane {
    int lane, slot, li;
};

// The 16-byte vector index (within a q / k / v / L row) of vector v of lane li.  J = false:
// vectors v*32 + li (lanes interleave; a head spans r/VE lanes).  J = true ("joint"): the
// lane's VPL vectors are consecutive, li*VPL + v, and all lie in one head (VPL*VE <= r),
// so the lane computes one score per edge for all of them.
template <bool J, int VPL>
__device__ __forceinline__ int vid_of(int v, int li) {
    return J ? li * VPL + v : v * 32 + li;
}

// First column index of a slot's range as held by the lane that later broadcasts it:
// lane li (< U) of the slot holds col_idx[e0 + li].
template <int U, bool DBG>
__device__ __forceinline__ int32_t first_cols(const LocalParams &p, int64_t e0, int64_t e1, const Lane &ln) {
    return (ln.li < U && e0 + ln.li < e1) ? checked_col<DBG>(p, __ldg(p.col_idx + e0 + ln.li)) : -1;
}

// One slot walks the CSR entries [e0, e1) U at a time (the trip count is the warp's
// maximum over slots); `cols` holds the first step's column indices (first_cols).
// On return each lane holds its slot's partial state for its feature vectors.
template <typename T, int VPL, int U, bool DBG, bool J>
__device__ __forceinline__ void slot_edges(const LocalParams &p, const float (&q)[VPL][Io<T>::VE],
                                           int64_t e0, int64_t e1, int32_t cols, const Lane &ln,
                                           State<T, VPL> &st) {
    constexpr int VE = Io<T>::VE;
    st.init();
    const int iters_mine = e1 > e0 ? static_cast<int>((e1 - e0 + U - 1) / U) : 0;
    const int iters = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(iters_mine));
    const uint4 *KV = static_cast<const uint4 *>(p.KV);
    const int64_t row_vecs = 2 * static_cast<int64_t>(p.nvec);
    const int src0 = ln.slot * p.lpe;
    int32_t c_next = cols;
    for (int it = 0; it < iters; ++it) {
        const int32_t c_cur = c_next;
        const int64_t nb = e0 + static_cast<int64_t>(it + 1) * U;
        c_next = (ln.li < U && nb + ln.li < e1) ? checked_col<DBG>(p, __ldg(p.col_idx + nb + ln.li)) : -1;
        int32_t j[U];
#pragma unroll
        for (int u = 0; u < U; ++u) j[u] = __shfl_sync(0xffffffffu, c_cur, src0 + u);
        uint4 kr[U][VPL], vr[U][VPL];
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const int vid = vid_of<J, VPL>(v, ln.li);
                if (j[u] >= 0 && vid < p.nvec) {
                    // (a masked-off slot never forms an address: j < 0 takes the else branch)
                    const uint4 *rowp = KV + static_cast<int64_t>(j[u]) * row_vecs;
                    kr[u][v] = ld_gather(rowp + vid);
                    vr[u][v] = ld_gather(rowp + p.nvec + vid);
                } else {
                    kr[u][v] = make_uint4(0, 0, 0, 0);
                    vr[u][v] = make_uint4(0, 0, 0, 0);
                }
            }
        }
        if constexpr (J) {
            // one score per edge for the lane's VPL vectors (one head): one exp, one max
            // and one rescale per edge instead of VPL
            float s1[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float dot = 0.f;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float kf[VE];
                    Io<T>::unpack(kr[u][v], kf);
#pragma unroll
                    for (int e = 0; e < VE; ++e) dot = fmaf(q[v][e], kf[e], dot);
                }
                for (int o = 1; o < p.lph; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                s1[u] = (j[u] >= 0) ? dot : -INFINITY;
            }
            float mx = s1[0];
#pragma unroll
            for (int u = 1; u < U; ++u) mx = fmaxf(mx, s1[u]);
            const float mn = fmaxf(st.m[0], mx);
            if (mn != -INFINITY) {
                const float corr = exp2_ftz(st.m[0] - mn);
                st.l[0] *= corr;
#pragma unroll
                for (int v = 0; v < VPL; ++v)
#pragma unroll
                    for (int e = 0; e < VE; ++e) st.acc[v][e] *= corr;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const float pr = exp2_ftz(s1[u] - mn);
                    st.l[0] += pr;
#pragma unroll
                    for (int v = 0; v < VPL; ++v) {
                        float vf[VE];
                        Io<T>::unpack(vr[u][v], vf);
#pragma unroll
                        for (int e = 0; e < VE; ++e) st.acc[v][e] = fmaf(pr, vf[e], st.acc[v][e]);
                    }
                }
                st.m[0] = mn;
            }
            continue;
        }
        float s[U][VPL];
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                float kf[VE];
                Io<T>::unpack(kr[u][v], kf);
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < VE; ++e) dot = fmaf(q[v][e], kf[e], dot);
                for (int o = 1; o < p.lph; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                s[u][v] = (j[u] >= 0) ? dot : -INFINITY;
            }
        }
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            float mx = s[0][v];
#pragma unroll
            for (int u = 1; u < U; ++u) mx = fmaxf(mx, s[u][v]);
            const float mn = fmaxf(st.m[v], mx);
            if (mn == -INFINITY) continue;
            const float corr = exp2_ftz(st.m[v] - mn);
            st.l[v] *= corr;
#pragma unroll
            for (int e = 0; e < VE; ++e) st.acc[v][e] *= corr;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float pr = exp2_ftz(s[u][v] - mn);
                float vf[VE];
                Io<T>::unpack(vr[u][v], vf);
                st.l[v] += pr;
#pragma unroll
                for (int e = 0; e < VE; ++e) st.acc[v][e] = fmaf(pr, vf[e], st.acc[v][e]);
            }
            st.m[v] = mn;
        }
    }
    if constexpr (J) {
        // every vector of the lane carries the head's (m, l): the merges work per vector
#pragma unroll
        for (int v = 1; v < VPL; ++v) {
            st.m[v] = st.m[0];
            st.l[v] = st.l[0];
        }
    }
}

// Merges the edge slots of the warp (lanes li, li + LPE, ...): afterwards every lane
// holds the state over all slots.
template <typename T, int VPL>
__device__ __forceinline__ void merge_slots(const LocalParams &p, State<T, VPL> &st) {
    constexpr int VE = Io<T>::VE;
    for (int o = p.lpe; o < 32; o <<= 1) {
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            const float m2 = __shfl_xor_sync(0xffffffffu, st.m[v], o);
            const float l2 = __shfl_xor_sync(0xffffffffu, st.l[v], o);
            float a2[VE];
#pragma unroll
            for (int e = 0; e < VE; ++e) a2[e] = __shfl_xor_sync(0xffffffffu, st.acc[v][e], o);
            st.merge(v, m2, l2, a2);
        }
    }
}

template <typename T, int VPL, bool J>
__device__ __forceinline__ void load_q_raw(const LocalParams &p, int64_t row, const Lane &ln, bool ok,
                                           uint4 (&qr)[VPL]) {
    const uint4 *Q = static_cast<const uint4 *>(p.Q) + row * p.nvec;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int vid = vid_of<J, VPL>(v, ln.li);
        qr[v] = (ok && vid < p.nvec) ? __ldg(Q + vid) : make_uint4(0, 0, 0, 0);
    }
}

template <typename T, int VPL>
__device__ __forceinline__ void scale_q(const LocalParams &p, const uint4 (&qr)[VPL], float (&q)[VPL][Io<T>::VE]) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        Io<T>::unpack(qr[v], q[v]);
#pragma unroll
        for (int e = 0; e < Io<T>::VE; ++e) q[v][e] *= p.score_scale;   // log2(e)/sqrt(r) folded in
    }
}

// lse_i = ln sum_j exp(s_ij) per head, ln 2 (m + log2 l) since the state keeps base-2
// scores (0 for a row without edges), from the vector holding the head's first features.
// Compiled in only for the LSE instantiations (contexts made for the backward pass), so
// the plain forward's code is untouched.
template <typename T, int VPL, bool J, bool LSE>
__device__ __forceinline__ void store_lse(const LocalParams &p, int64_t row, const State<T, VPL> &st,
                                          const Lane &ln, bool mine) {
    if constexpr (!LSE) return;
    constexpr int VE = Io<T>::VE;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int vid = vid_of<J, VPL>(v, ln.li);
        if (mine && vid < p.nvec && (vid * VE) % p.r == 0)
            p.lse[row * p.H + vid * VE / p.r] =
                st.l[v] > 0.f ? 0.69314718055994531f * (st.m[v] + __log2f(st.l[v])) : 0.f;
    }
}

// L_i = acc / l per head (0 for a row without edges); stores L[row] from `slot`'s lanes.
template <typename T, int VPL, bool J, bool LSE>
__device__ __forceinline__ void finish_row(const LocalParams &p, int64_t row, const State<T, VPL> &st,
                                           const Lane &ln, int slot) {
    constexpr int VE = Io<T>::VE;
    uint4 *Lout = static_cast<uint4 *>(p.L) + row * p.nvec;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int vid = vid_of<J, VPL>(v, ln.li);
        const float inv_l = st.l[v] > 0.f ? 1.f / st.l[v] : 0.f;
        float y[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) y[e] = st.acc[v][e] * inv_l;
        if (vid < p.nvec && ln.slot == slot) Lout[vid] = Io<T>::pack(y);
    }
    store_lse<T, VPL, J, LSE>(p, row, st, ln, ln.slot == slot);
}

template <typename T, int VPL>
struct BlockScratch {
    static constexpr int VE = Io<T>::VE;
    float m[kLocalWarps][VPL][32];
    float l[kLocalWarps][VPL][32];
    float acc[kLocalWarps][VPL][VE][32];
};

// 8 warps split [e0, e1) (each warp's share split again across its slots); warp 0
// returns the merge of all warps in warp order.
template <typename T, int VPL, int U, bool DBG, bool J>
__device__ __forceinline__ void block_edges(const LocalParams &p, const float (&q)[VPL][Io<T>::VE],
                                            int64_t e0, int64_t e1, const Lane &ln, int warp,
                                            BlockScratch<T, VPL> &sh, State<T, VPL> &st) {
    constexpr int VE = Io<T>::VE;
    const int64_t per = ceil_div(e1 - e0, kLocalWarps);
    const int64_t a = std::min(e1, e0 + warp * per), b = std::min(e1, a + per);
    const int64_t per_s = ceil_div(b - a, p.epw);
    const int64_t sa = std::min(b, a + ln.slot * per_s), sb = std::min(b, sa + per_s);
    slot_edges<T, VPL, U, DBG, J>(p, q, sa, sb, first_cols<U, DBG>(p, sa, sb, ln), ln, st);
    merge_slots<T, VPL>(p, st);
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        sh.m[warp][v][ln.lane] = st.m[v];
        sh.l[warp][v][ln.lane] = st.l[v];
#pragma unroll
        for (int e = 0; e < VE; ++e) sh.acc[warp][v][e][ln.lane] = st.acc[v][e];
    }
    __syncthreads();
    if (warp == 0) {
        for (int w = 1; w < kLocalWarps; ++w) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                float a2[VE];
#pragma unroll
                for (int e = 0; e < VE; ++e) a2[e] = sh.acc[w][v][e][ln.lane];
                st.merge(v, sh.m[w][v][ln.lane], sh.l[w][v][ln.lane], a2);
            }
        }
    }
}

template <typename T, int VPL, int U, bool DBG, bool J, bool LSE>
__global__ void __launch_bounds__(kLocalThreads, VPL == 1 ? 3 : 2) local_kernel(const LocalParams p) {
    constexpr int VE = Io<T>::VE;
    __shared__ BlockScratch<T, VPL> sh;
    const int warp = threadIdx.x >> 5;
    Lane ln;
    ln.lane = threadIdx.x & 31;
    ln.slot = ln.lane / p.lpe;
    ln.li = ln.lane % p.lpe;
    int64_t bid = blockIdx.x;
    float q[VPL][VE];
    uint4 qr[VPL];
    State<T, VPL> st;

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
        load_q_raw<T, VPL, J>(p, row, ln, true, qr);
        scale_q<T, VPL>(p, qr, q);
        block_edges<T, VPL, U, DBG, J>(p, q, e0, e1, ln, warp, sh, st);
        const int64_t stride = 2 * p.H + p.D;
        if (warp == 0) {
            float *dst = p.part + c * stride;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const int vid = vid_of<J, VPL>(v, ln.li);
                if (vid < p.nvec && ln.slot == 0) {
#pragma unroll
                    for (int e = 0; e < VE; ++e) dst[2 * p.H + vid * VE + e] = st.acc[v][e];
                    if ((ln.li & (p.lph - 1)) == 0) {
                        const int h = vid * VE / p.r;
                        dst[h] = st.m[v];
                        dst[p.H + h] = st.l[v];
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
#pragma unroll
                    for (int v = 0; v < VPL; ++v) {
                        const int vid = vid_of<J, VPL>(v, ln.li);
                        const int h = vid < p.nvec ? vid * VE / p.r : 0;
                        float a2[VE];
#pragma unroll
                        for (int e = 0; e < VE; ++e)
                            a2[e] = vid < p.nvec ? __ldcg(src + 2 * p.H + vid * VE + e) : 0.f;
                        st.merge(v, __ldcg(src + h), __ldcg(src + p.H + h), a2);
                    }
                }
                finish_row<T, VPL, J, LSE>(p, row, st, ln, 0);
            }
        }
        return;
    }
    bid -= p.n_chunks;
    if (bid < p.n_cta) {
        // ---------------- bucket-1 row: one block ----------------
        const int64_t row = p.cta_rows[bid];
        if (!row_ok<DBG>(p, row)) return;
        load_q_raw<T, VPL, J>(p, row, ln, true, qr);
        scale_q<T, VPL>(p, qr, q);
        block_edges<T, VPL, U, DBG, J>(p, q, p.row_ptr[row], p.row_ptr[row + 1], ln, warp, sh, st);
        if (warp == 0) finish_row<T, VPL, J, LSE>(p, row, st, ln, 0);
        return;
    }
    bid -= p.n_cta;
    // ---------------- bucket-0 task: up to 32 rows, one per slot per step ----------------
    const int64_t task = bid * kLocalWarps + warp;
    if (task >= p.n_tasks) return;
    const int t0 = p.task_start[task];
    const int n = p.task_start[task + 1] - t0;
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
    const int steps = (n + p.epw - 1) / p.epw;
    // step 0 prefetch: this slot's first row
    int k = ln.slot;
    int32_t row = __shfl_sync(0xffffffffu, myrow, k & 31);
    int32_t beg = __shfl_sync(0xffffffffu, mybeg, k & 31);
    int32_t end = __shfl_sync(0xffffffffu, myend, k & 31);
    if (k >= n) beg = end = 0;
    load_q_raw<T, VPL, J>(p, row, ln, k < n && (!DBG || row >= 0), qr);
    int32_t cols = first_cols<U, DBG>(p, beg, end, ln);
    for (int step = 0; step < steps; ++step) {
        const bool valid = k < n;
        const int32_t row_c = row;
        const int64_t beg_c = beg, end_c = end;
        const int32_t cols_c = cols;
        scale_q<T, VPL>(p, qr, q);
        // prefetch the next step's row while this one's gathers are in flight
        k += p.epw;
        row = __shfl_sync(0xffffffffu, myrow, k & 31);
        beg = __shfl_sync(0xffffffffu, mybeg, k & 31);
        end = __shfl_sync(0xffffffffu, myend, k & 31);
        if (k >= n) beg = end = 0;
        load_q_raw<T, VPL, J>(p, row, ln, k < n && (!DBG || row >= 0), qr);
        cols = first_cols<U, DBG>(p, beg, end, ln);
        slot_edges<T, VPL, U, DBG, J>(p, q, beg_c, end_c, cols_c, ln, st);
        if (valid && (!DBG || row_c >= 0)) {
            // every slot finishes its own row
            constexpr int VEc = Io<T>::VE;
            uint4 *Lout = static_cast<uint4 *>(p.L) + static_cast<int64_t>(row_c) * p.nvec;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const int vid = vid_of<J, VPL>(v, ln.li);
                const float inv_l = st.l[v] > 0.f ? 1.f / st.l[v] : 0.f;
                float y[VEc];
#pragma unroll
                for (int e = 0; e < VEc; ++e) y[e] = st.acc[v][e] * inv_l;
                if (vid < p.nvec) Lout[vid] = Io<T>::pack(y);
            }
            store_lse<T, VPL, J, LSE>(p, row_c, st, ln, true);
        }
    }
}

template <typename T, int VPL, int U, bool J = false>
glga_status launch_local(Ctx *c, const LocalParams &p, cudaStream_t s) {
    const int64_t blocks = p.n_chunks + p.n_cta + p.task_blocks;
    if (blocks == 0) return GLGA_OK;
    const unsigned g = static_cast<unsigned>(blocks);
    if (c->opts.debug_checks) {
        if (p.lse) local_kernel<T, VPL, U, true, J, true><<<g, kLocalThreads, 0, s>>>(p);
        else local_kernel<T, VPL, U, true, J, false><<<g, kLocalThreads, 0, s>>>(p);
    } else {
        if (p.lse) local_kernel<T, VPL, U, false, J, true><<<g, kLocalThreads, 0, s>>>(p);
        else local_kernel<T, VPL, U, false, J, false><<<g, kLocalThreads, 0, s>>>(p);
    }
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
    // bf16 rows of 64 vectors (D = 512) with heads of >= 16 features: the joint layout,
    // two consecutive vectors (16 features of one head) per lane.  (Measured: faster than
    // the interleaved layout at D = 512, slower at D = 128, where its 118 registers leave
    // 16 warps per SM instead of 24.)
    if (c->io == GLGA_BF16 && c->r >= 16 && p.nvec == 64) {
        p.lpe = p.nvec / 2;
        p.epw = 32 / p.lpe;
        p.lph = c->r / 16;
        return launch_local<__nv_bfloat16, 2, 2, true>(c, p, s);
    }
    // U edges per slot step; U <= LPE so the slot's lanes can hold its column indices
    if (c->io == GLGA_F32) {
        if (vpl == 1 && lpe >= 4) return launch_local<float, 1, 4>(c, p, s);
        if (vpl == 1 && lpe == 2) return launch_local<float, 1, 2>(c, p, s);
        if (vpl == 1) return launch_local<float, 1, 1>(c, p, s);
        if (vpl == 2) return launch_local<float, 2, 2>(c, p, s);
        if (vpl <= 4) return launch_local<float, 4, 1>(c, p, s);
    } else {
        if (vpl == 1 && lpe >= 4) return launch_local<__nv_bfloat16, 1, 4>(c, p, s);
        if (vpl == 1 && lpe == 2) return launch_local<__nv_bfloat16, 1, 2>(c, p, s);
        if (vpl == 1) return launch_local<__nv_bfloat16, 1, 1>(c, p, s);
        if (vpl == 2) return launch_local<__nv_bfloat16, 2, 2>(c, p, s);
        if (vpl <= 4) return launch_local<__nv_bfloat16, 4, 1>(c, p, s);
    }
    set_error("row width too large for the local kernel");
    return GLGA_ERR_UNSUPPORTED;
}

}  // namespace glga
