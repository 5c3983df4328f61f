// backward.cu -- gradients of the layer (training): dX, dW_Q, dW_K, dW_V, dw_g, db_g from dY.
//
// Method page "Gated Local-Global Graph Attention", Key formulas, differentiated:
//   Y = g L + (1 - g) G,  g = sigmoid(t + b_g):  dL = g dY,  dG = (1 - g) dY,
//       dt_i = g (1 - g) sum_c dY_ic (L_ic - G_ic)
//   G = num / den, num = phi(q)^T S, den = phi(q)^T z + eps:
//       dnum = dG / den,  dden = -(dG . G) / den,  dphi(q) = S dnum + z dden,
//       dS = sum_i phi(q_i) dnum_i^T,  dz = sum_i phi(q_i) dden_i,
//       dphi(k_j) = dS v_j + dz,  dv_j += dS^T phi(k_j),  phi'(x) = 1 (x > 0) or e^x
//   L_i = sum_j p_ij v_j, p = softmax_j(s), s_ij = q_i . k_j / sqrt(r)  (the segment
//   maximum cancels; tinymesh "Target softmax" detaches it):
//       D_i = dL_i . L_i,  ds_ij = p_ij (dL_i . v_j - D_i),
//       dq_i += sum_j ds_ij k_j / sqrt(r),  dk_j += sum_i ds_ij q_i / sqrt(r),
//       dv_j += sum_i p_ij dL_i
//   [Q | K | V | t] = X [W_Q | W_K | W_V | w_g]:  dW = X^T dZ,  dX = dZ W^T with
//       dZ = [dQ | dK | dV | dt].
// The target-grouped terms (dq) walk the forward CSR; the source-grouped terms (dk, dv)
// walk a transposed CSR built at create, so every sum has a fixed order and there are no
// atomics (two runs give identical bits).  Plain CUDA-core kernels with fp32 arithmetic
// (one thread per row and head, tiled GEMMs for the projections); gradients are fp32.
#include <algorithm>
#include <cmath>
#include <vector>

#include "glga_internal.cuh"

namespace glga {
namespace {

template <typename T>
__device__ __forceinline__ float ldf(const T *p);
template <>
__device__ __forceinline__ float ldf<float>(const float *p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ float dphi(float x) { return x > 0.f ? 1.f : __expf(x); }

// (ld_row / head_reduce: see the warp-cooperative row kernels below)
template <typename T, int EPL>
__device__ __forceinline__ void ld_row(const T *row, int lane, bool act, float (&x)[EPL]);
__device__ __forceinline__ float head_reduce(float x, int lph);

// One warp per row i (lanes over features, EPL each): the gate, readout and blend
// backward.  Writes dL [N, D], dnum [N, D], dden [N, H], the global part of dQ into
// dZ [:, 0:D] and dt into dZ [:, 3D] (dg summed over the whole row in lane order).
template <typename T, int EPL>
__global__ void __launch_bounds__(256) bwd_readout_kernel(
    const T *__restrict__ Q, const T *__restrict__ L, const float *__restrict__ t, const float *__restrict__ Sz,
    const float *__restrict__ ST, const T *__restrict__ dY, int64_t N, int H, int R, float b_g, float eps,
    float *__restrict__ dL,
    float *__restrict__ dnum, float *__restrict__ dden, float *__restrict__ dZ, int64_t dz_ld) {
    const int64_t i = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (i >= N) return;                                   // warp-uniform
    const int D = H * R;
    const bool act = lane * EPL < D;
    const int lph = R / EPL, h = act ? lane * EPL / R : 0;
    const float *S = Sz + static_cast<int64_t>(h) * R * R;
    const float *z = Sz + static_cast<int64_t>(H) * R * R + h * R;
    const T *qh = Q + i * D + h * R;                      // the lane's head
    float q[EPL], dy[EPL], lv[EPL];
    ld_row<T, EPL>(Q + i * D, lane, act, q);
    ld_row<T, EPL>(dY + i * D, lane, act, dy);
    ld_row<T, EPL>(L + i * D, lane, act, lv);
    const int f0 = lane * EPL - h * R;                    // in-head index of the lane's first feature
    float den = 0.f;
    if (act) {
#pragma unroll
        for (int x = 0; x < EPL; ++x) den = fmaf(phi(q[x]), z[f0 + x], den);
    }
    den = head_reduce(den, lph) + eps;
    // num_c = sum_a phi(q_a) S[a][c] for the lane's features c (phi(q_a) read back from
    // the row, the same for the head's lanes)
    float G[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) G[x] = 0.f;
    if (act)
        for (int a = 0; a < R; ++a) {
            const float pa = phi(ldf<T>(qh + a));
#pragma unroll
            for (int x = 0; x < EPL; ++x) G[x] = fmaf(pa, S[a * R + f0 + x], G[x]);
        }
    const float g = 1.f / (1.f + __expf(-(t[i] + b_g)));
    float dgp = 0.f, dGG = 0.f;
    const int64_t o = i * D + lane * EPL;
#pragma unroll
    for (int x = 0; x < EPL; ++x) {
        G[x] /= den;
        dgp = fmaf(dy[x], lv[x] - G[x], dgp);
        const float dG = (1.f - g) * dy[x];
        dGG = fmaf(dG, G[x], dGG);
        if (act) {
            dL[o + x] = g * dy[x];
            dnum[o + x] = dG / den;
        }
    }
    const float dd = -head_reduce(dGG, lph) / den;
    if (act && (lane % lph) == 0) dden[i * H + h] = dd;
    __syncwarp();                                         // dnum of the row is written
    const float *dn = dnum + i * D + h * R;
    const float *STh = ST + static_cast<int64_t>(h) * R * R;   // STh[c][a] = S[a][c]
    if (act) {
#pragma unroll
        for (int x = 0; x < EPL; ++x) {
            float acc = z[f0 + x] * dd;
            for (int c = 0; c < R; ++c) acc = fmaf(STh[c * R + f0 + x], dn[c], acc);
            dZ[i * dz_ld + lane * EPL + x] = acc * dphi(q[x]);
        }
    }
    for (int w = 16; w > 0; w >>= 1) dgp += __shfl_xor_sync(0xffffffffu, dgp, w);
    if (lane == 0) dZ[i * dz_ld + 3 * D] = g * (1.f - g) * dgp;
}

// Partial sums of dS | dz over the row range of block column p, per head h =
// blockIdx.y, in the layout [H][R][R+1] (column R is dz):
//   part[p][h][a][c] = sum_i phi(q_i[h R + a]) * (c < R ? dnum_i[h R + c] : dden_i[h]).
// 32-row tiles of phi(Q_h) and [dnum_h | dden_h] are staged in shared memory; each thread
// owns outputs o = tid, tid + 256, ... of the head's R (R + 1).
template <typename T, int R>
__global__ void __launch_bounds__(256) bwd_dsz_partial_kernel(const T *__restrict__ Q, const float *__restrict__ dnum,
                                                              const float *__restrict__ dden, int64_t N, int H,
                                                              int64_t rows_per_part, float *__restrict__ part) {
    extern __shared__ float tile[];                      // [32][R] phi(q) then [32][R + 1] dnum | dden
    constexpr int kRowsT = 32;
    const int h = blockIdx.y;
    const int D = H * R;
    const int per_head = R * (R + 1);
    float *pq = tile, *pw = tile + kRowsT * R;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_part;
    const int64_t r1 = std::min<int64_t>(N, r0 + rows_per_part);
    constexpr int kMaxOut = (R * (R + 1) + 255) / 256;
    float acc[kMaxOut];
    const int n_out = (per_head - static_cast<int>(threadIdx.x) + 255) / 256;
#pragma unroll
    for (int u = 0; u < kMaxOut; ++u) acc[u] = 0.f;
    for (int64_t i0 = r0; i0 < r1; i0 += kRowsT) {
        for (int l = threadIdx.x; l < kRowsT * (R + 1); l += 256) {
            const int rr = l / (R + 1), c = l % (R + 1);
            const int64_t i = i0 + rr;
            const bool in = i < r1;
            if (c < R) {
                pq[rr * R + c] = in ? phi(ldf<T>(Q + i * D + h * R + c)) : 0.f;
                pw[rr * (R + 1) + c] = in ? dnum[i * D + h * R + c] : 0.f;
            } else {
                pw[rr * (R + 1) + R] = in ? dden[i * H + h] : 0.f;
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kMaxOut; ++u) {
            if (u < n_out) {
                const int oo = threadIdx.x + u * 256;
                const int a = oo / (R + 1), c = oo % (R + 1);
                float sacc = acc[u];
                for (int rr = 0; rr < kRowsT; ++rr) sacc = fmaf(pq[rr * R + a], pw[rr * (R + 1) + c], sacc);
                acc[u] = sacc;
            }
        }
        __syncthreads();
    }
    const int total = H * per_head;
    float *out = part + static_cast<int64_t>(blockIdx.x) * total + h * per_head;
#pragma unroll
    for (int u = 0; u < kMaxOut; ++u)
        if (u < n_out) out[threadIdx.x + u * 256] = acc[u];
}

// dst[h][c][a] = src[h][a][c] (a, c < R) for per-head R x R blocks with row stride ld.
__global__ void bwd_transpose_heads_kernel(const float *__restrict__ src, int ld, int H, int R,
                                           float *__restrict__ dst) {
    const int64_t total = static_cast<int64_t>(H) * R * R;
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < total;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int h = static_cast<int>(o / (static_cast<int64_t>(R) * R));
        const int c = static_cast<int>((o / R) % R), a = static_cast<int>(o % R);
        dst[o] = src[static_cast<int64_t>(h) * R * ld + static_cast<int64_t>(a) * ld + c];
    }
}

// out[o] = sum over p = 0 .. P-1, in order, of part[p][o].
__global__ void bwd_sum_parts_kernel(const float *__restrict__ part, int P, int64_t total, float *__restrict__ out) {
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < total;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float acc = 0.f;
        for (int p = 0; p < P; ++p) acc += part[static_cast<int64_t>(p) * total + o];
        out[o] = acc;
    }
}

// Warp-cooperative row kernels: one warp per row, lane l holds the EPL consecutive
// features l*EPL .. l*EPL+EPL-1 of every row it reads (contiguous across the warp, so a
// row is one coalesced read), and a head's r features lie in LPH = r/EPL adjacent lanes,
// whose dot products meet in a butterfly of shuffles.

template <typename T, int EPL>
__device__ __forceinline__ void ld_row(const T *row, int lane, bool act, float (&x)[EPL]) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) x[e] = act ? ldf<T>(row + lane * EPL + e) : 0.f;
}

__device__ __forceinline__ float head_reduce(float x, int lph) {
    for (int o = 1; o < lph; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

constexpr int kEU = 4;           // edges whose rows are loaded before any is used
constexpr int kHeavyWarps = 32;  // warps per heavy row (one 1024-thread block)

// Online (max, sum) of exp(s) over the edges [a, b) of target row q (this warp's lanes).
template <typename T, int EPL>
__device__ __forceinline__ void q_lse_range(const int32_t *col_idx, const T *KV, int D, int lane, bool act,
                                            int lph, float inv_sqrt_r, const float (&q)[EPL], int32_t a,
                                            int32_t b, float &m, float &l) {
    for (int32_t e = a; e < b; e += kEU) {
        float k[kEU][EPL];
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
            const bool live = e + u < b;
            const int64_t jj = live ? col_idx[e + u] : 0;
            ld_row<T, EPL>(KV + jj * 2 * D, lane, act && live, k[u]);
        }
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
            float s = 0.f;
#pragma unroll
            for (int x = 0; x < EPL; ++x) s = fmaf(q[x], k[u][x], s);
            s = head_reduce(s, lph) * inv_sqrt_r;
            if (e + u < b) {
                const float mn = fmaxf(m, s);
                l = l * __expf(m - mn) + __expf(s - mn);
                m = mn;
            }
        }
    }
}

// dq += sum over edges [a, b) of ds_ij k_j (ds already scaled by 1/sqrt(r)).
template <typename T, int EPL>
__device__ __forceinline__ void q_grad_range(const int32_t *col_idx, const T *KV, int D, int lane, bool act,
                                             int lph, float inv_sqrt_r, const float (&q)[EPL],
                                             const float (&dl)[EPL], float ls, float dd, int32_t a, int32_t b,
                                             float (&dq)[EPL]) {
    for (int32_t e = a; e < b; e += kEU) {
        float k[kEU][EPL], v[kEU][EPL];
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
            const bool live = e + u < b;
            const T *row = KV + (live ? static_cast<int64_t>(col_idx[e + u]) : 0) * 2 * D;
            ld_row<T, EPL>(row, lane, act && live, k[u]);
            ld_row<T, EPL>(row + D, lane, act && live, v[u]);
        }
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int x = 0; x < EPL; ++x) {
                s = fmaf(q[x], k[u][x], s);
                dp = fmaf(dl[x], v[u][x], dp);
            }
            s = head_reduce(s, lph);
            dp = head_reduce(dp, lph);
            const float ds = e + u < b ? __expf(s * inv_sqrt_r - ls) * (dp - dd) * inv_sqrt_r : 0.f;
#pragma unroll
            for (int x = 0; x < EPL; ++x) dq[x] = fmaf(ds, k[u][x], dq[x]);
        }
    }
}

// Target rows of the forward CSR: per head the softmax's log-sum-exp and D_i = dL_i . L_i,
// and the local part of dq_i added into dZ [:, 0:D].  Light rows (the `rows` list): one
// warp each.  Heavy rows (HEAVY): one 1024-thread block each, its 32 warps taking
// contiguous shares of the edges; their partial (max, sum) and dq are combined in warp
// order through shared memory.
template <typename T, int EPL, bool HEAVY>
__global__ void __launch_bounds__(HEAVY ? 1024 : 256) bwd_local_q_kernel(
    const int32_t *__restrict__ rows, int64_t n_rows, const int32_t *__restrict__ row_ptr,
    const int32_t *__restrict__ col_idx, const T *__restrict__ Q, const T *__restrict__ KV,
    const T *__restrict__ L, const float *__restrict__ dL, int H, int R, float inv_sqrt_r,
    float *__restrict__ lse, float *__restrict__ Dd, float *__restrict__ dZ, int64_t dz_ld) {
    __shared__ float sm_m[HEAVY ? kHeavyWarps : 1][32], sm_l[HEAVY ? kHeavyWarps : 1][32];
    __shared__ float sm_dq[HEAVY ? 32 * 32 : 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t slot = HEAVY ? blockIdx.x : (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (slot >= n_rows) return;                           // uniform per warp (per block when HEAVY)
    const int64_t i = rows[slot];
    const int D = H * R;
    const bool act = lane * EPL < D;
    const int lph = R / EPL, h = act ? lane * EPL / R : 0;
    float q[EPL], dl[EPL], lv[EPL];
    ld_row<T, EPL>(Q + i * D, lane, act, q);
    ld_row<float, EPL>(dL + i * D, lane, act, dl);
    ld_row<T, EPL>(L + i * D, lane, act, lv);
    const int32_t r0 = row_ptr[i], r1 = row_ptr[i + 1];
    int32_t a = r0, b = r1;
    if (HEAVY) {
        const int32_t per = (r1 - r0 + kHeavyWarps - 1) / kHeavyWarps;
        a = min(r1, r0 + warp * per);
        b = min(r1, a + per);
    }
    float m = -INFINITY, l = 0.f;
    q_lse_range<T, EPL>(col_idx, KV, D, lane, act, lph, inv_sqrt_r, q, a, b, m, l);
    if (HEAVY) {
        sm_m[warp][lane] = m;
        sm_l[warp][lane] = l;
        __syncthreads();
        m = -INFINITY;
        l = 0.f;
        for (int w = 0; w < kHeavyWarps; ++w) {          // warp order
            const float m2 = sm_m[w][lane], l2 = sm_l[w][lane];
            const float mn = fmaxf(m, m2);
            if (mn != -INFINITY) {
                l = l * __expf(m - mn) + l2 * __expf(m2 - mn);
                m = mn;
            }
        }
    }
    const float ls = r1 > r0 ? m + __logf(l) : 0.f;
    float dd = 0.f;
#pragma unroll
    for (int x = 0; x < EPL; ++x) dd = fmaf(dl[x], lv[x], dd);
    dd = head_reduce(dd, lph);
    if (act && (lane % lph) == 0 && (!HEAVY || warp == 0)) {
        lse[i * H + h] = ls;
        Dd[i * H + h] = dd;
    }
    float dq[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) dq[x] = 0.f;
    q_grad_range<T, EPL>(col_idx, KV, D, lane, act, lph, inv_sqrt_r, q, dl, ls, dd, a, b, dq);
    if (HEAVY) {
        // add the warps' dq in warp order, one 32 * EPL-feature slice at a time
        for (int w = 0; w < kHeavyWarps; ++w) {
            if (warp == w) {
#pragma unroll
                for (int x = 0; x < EPL; ++x) {
                    const int f = lane * EPL + x;
                    if (f < 32 * 32) sm_dq[f] = (w == 0 ? 0.f : sm_dq[f]) + dq[x];
                }
            }
            __syncthreads();
        }
        if (warp == 0) {
#pragma unroll
            for (int x = 0; x < EPL; ++x) dq[x] = sm_dq[lane * EPL + x];
        } else {
            return;
        }
    }
    if (act) {
#pragma unroll
        for (int x = 0; x < EPL; ++x) dZ[i * dz_ld + lane * EPL + x] += dq[x];
    }
}

// dk, dv += the terms of targets [a, b) of source row j (this warp's lanes).
template <typename T, int EPL>
__device__ __forceinline__ void kv_grad_range(const int32_t *t_col, const T *Q, const float *dL,
                                              const float *lse, const float *Dd, int H, int D, int lane,
                                              bool act, int lph, int h, float inv_sqrt_r, const float (&k)[EPL],
                                              const float (&v)[EPL], int32_t a, int32_t b, float (&dk)[EPL],
                                              float (&dv)[EPL]) {
    for (int32_t e = a; e < b; e += kEU) {
        float q[kEU][EPL], dl[kEU][EPL], ls[kEU], dd[kEU];
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
            const bool live = e + u < b;
            const int64_t i = live ? t_col[e + u] : 0;
            ld_row<T, EPL>(Q + i * D, lane, act && live, q[u]);
            ld_row<float, EPL>(dL + i * D, lane, act && live, dl[u]);
            ls[u] = live ? lse[i * H + h] : 0.f;
            dd[u] = live ? Dd[i * H + h] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int x = 0; x < EPL; ++x) {
                s = fmaf(q[u][x], k[x], s);
                dp = fmaf(dl[u][x], v[x], dp);
            }
            s = head_reduce(s, lph);
            dp = head_reduce(dp, lph);
            const bool live = e + u < b;
            const float p = live ? __expf(s * inv_sqrt_r - ls[u]) : 0.f;
            const float ds = p * (dp - dd[u]) * inv_sqrt_r;
#pragma unroll
            for (int x = 0; x < EPL; ++x) {
                dv[x] = fmaf(p, dl[u][x], dv[x]);
                dk[x] = fmaf(ds, q[u][x], dk[x]);
            }
        }
    }
}

// Source rows of the transposed CSR (the targets i of j): the local terms of dk_j and
// dv_j, plus the global terms through phi(k_j), written to dZ [:, D:2D] and [:, 2D:3D].
// dSz holds dS | dz as [H][R][R+1].  Light rows one warp each, heavy rows one block each
// (warp shares combined in warp order), as bwd_local_q_kernel.
template <typename T, int EPL, bool HEAVY>
__global__ void __launch_bounds__(HEAVY ? 1024 : 256) bwd_local_kv_kernel(
    const int32_t *__restrict__ rows, int64_t n_rows, const int32_t *__restrict__ t_row_ptr,
    const int32_t *__restrict__ t_col, const T *__restrict__ Q, const T *__restrict__ KV,
    const float *__restrict__ dL, const float *__restrict__ lse, const float *__restrict__ Dd,
    const float *__restrict__ dSz, const float *__restrict__ dST, int H, int R, float inv_sqrt_r,
    float *__restrict__ dZ, int64_t dz_ld) {
    __shared__ float sm_dk[HEAVY ? 32 * 32 : 1], sm_dv[HEAVY ? 32 * 32 : 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t slot = HEAVY ? blockIdx.x : (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (slot >= n_rows) return;
    const int64_t j = rows[slot];
    const int D = H * R;
    const bool act = lane * EPL < D;
    const int lph = R / EPL, h = act ? lane * EPL / R : 0;
    const T *krow = KV + j * 2 * D;
    float k[EPL], v[EPL], dk[EPL], dv[EPL];
    ld_row<T, EPL>(krow, lane, act, k);
    ld_row<T, EPL>(krow + D, lane, act, v);
#pragma unroll
    for (int x = 0; x < EPL; ++x) dk[x] = dv[x] = 0.f;
    const int32_t r0 = t_row_ptr[j], r1 = t_row_ptr[j + 1];
    int32_t a = r0, b = r1;
    if (HEAVY) {
        const int32_t per = (r1 - r0 + kHeavyWarps - 1) / kHeavyWarps;
        a = min(r1, r0 + warp * per);
        b = min(r1, a + per);
    }
    kv_grad_range<T, EPL>(t_col, Q, dL, lse, Dd, H, D, lane, act, lph, h, inv_sqrt_r, k, v, a, b, dk, dv);
    if (HEAVY) {
        for (int w = 0; w < kHeavyWarps; ++w) {
            if (warp == w) {
#pragma unroll
                for (int x = 0; x < EPL; ++x) {
                    const int f = lane * EPL + x;
                    if (f < 32 * 32) {
                        sm_dk[f] = (w == 0 ? 0.f : sm_dk[f]) + dk[x];
                        sm_dv[f] = (w == 0 ? 0.f : sm_dv[f]) + dv[x];
                    }
                }
            }
            __syncthreads();
        }
        if (warp != 0) return;
#pragma unroll
        for (int x = 0; x < EPL; ++x) {
            dk[x] = sm_dk[lane * EPL + x];
            dv[x] = sm_dv[lane * EPL + x];
        }
    }
    // global branch, S = sum phi(k) v^T and z = sum phi(k): for the lane's features
    // (head h, in-head index f = lane*EPL + x - h*R)
    if (act) {
        const float *dS = dSz + static_cast<int64_t>(h) * R * (R + 1);
        const float *dSTh = dST + static_cast<int64_t>(h) * R * R;   // dSTh[c][f] = dS[f][c]
        const T *kh = krow + h * R, *vh = krow + D + h * R;
#pragma unroll
        for (int x = 0; x < EPL; ++x) {
            const int f = lane * EPL + x - h * R;
            float dphk = dS[f * (R + 1) + R];             // dz_f
            float dvg = 0.f;
            for (int c = 0; c < R; ++c) {
                dphk = fmaf(dSTh[c * R + f], ldf<T>(vh + c), dphk);
                dvg = fmaf(dS[c * (R + 1) + f], phi(ldf<T>(kh + c)), dvg);
            }
            dk[x] = fmaf(dphk, dphi(k[x]), dk[x]);
            dv[x] += dvg;
        }
#pragma unroll
        for (int x = 0; x < EPL; ++x) {
            dZ[j * dz_ld + D + lane * EPL + x] = dk[x];
            dZ[j * dz_ld + 2 * D + lane * EPL + x] = dv[x];
        }
    }
}

// db_g = sum_i dt_i in a fixed order: thread k sums i = k, k + 1024, ...; then a tree.
__global__ void __launch_bounds__(1024) bwd_dbg_kernel(const float *__restrict__ dZ, int64_t N, int64_t dz_ld,
                                                       int64_t col, float *__restrict__ db_g) {
    __shared__ float red[1024];
    float s = 0.f;
    for (int64_t i = threadIdx.x; i < N; i += 1024) s += dZ[i * dz_ld + col];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *db_g = red[0];
}

constexpr int kTile = 64, kTk = 16;

// part[p][a][k] = sum over rows i of range p of X[i][a] * dZ[i][k]  (a < d, k < Dz):
// 64 x 64 output tiles, 16 rows per shared-memory step, 4 x 4 outputs per thread.
template <typename T>
__global__ void __launch_bounds__(256) bwd_dw_kernel(const T *__restrict__ X, const float *__restrict__ dZ,
                                                     int64_t N, int d, int Dz, int64_t rows_per_part,
                                                     float *__restrict__ part) {
    __shared__ float As[kTk][kTile], Bs[kTk][kTile];
    const int a0 = blockIdx.x * kTile, k0 = blockIdx.y * kTile;
    const int64_t r0 = static_cast<int64_t>(blockIdx.z) * rows_per_part;
    const int64_t r1 = std::min<int64_t>(N, r0 + rows_per_part);
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int64_t i0 = r0; i0 < r1; i0 += kTk) {
        for (int l = threadIdx.x; l < kTk * kTile; l += 256) {
            const int rr = l / kTile, cc = l % kTile;
            const int64_t i = i0 + rr;
            As[rr][cc] = (i < r1 && a0 + cc < d) ? ldf<T>(X + i * d + a0 + cc) : 0.f;
            Bs[rr][cc] = (i < r1 && k0 + cc < Dz) ? dZ[i * Dz + k0 + cc] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < kTk; ++rr) {
            float av[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                av[u] = As[rr][ty * 4 + u];
                bv[u] = Bs[rr][tx * 4 + u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
        }
        __syncthreads();
    }
    float *out = part + static_cast<int64_t>(blockIdx.z) * d * Dz;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int a = a0 + ty * 4 + u, k = k0 + tx * 4 + w;
            if (a < d && k < Dz) out[static_cast<int64_t>(a) * Dz + k] = acc[u][w];
        }
}

// dW_Q | dW_K | dW_V | dw_g from the row-range parts, summed in range order.
__global__ void bwd_dw_reduce_kernel(const float *__restrict__ part, int P, int d, int D, int Dz,
                                     float *__restrict__ dWQ, float *__restrict__ dWK, float *__restrict__ dWV,
                                     float *__restrict__ dwg) {
    const int64_t total = static_cast<int64_t>(d) * Dz;
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < total;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float acc = 0.f;
        for (int p = 0; p < P; ++p) acc += part[static_cast<int64_t>(p) * total + o];
        const int a = static_cast<int>(o / Dz), k = static_cast<int>(o % Dz);
        if (k < D) dWQ[static_cast<int64_t>(a) * D + k] = acc;
        else if (k < 2 * D) dWK[static_cast<int64_t>(a) * D + k - D] = acc;
        else if (k < 3 * D) dWV[static_cast<int64_t>(a) * D + k - 2 * D] = acc;
        else dwg[a] = acc;
    }
}

// Column k of [W_Q | W_K | W_V | w_g] at row a.
template <typename T>
__device__ __forceinline__ float w_all(const T *WQ, const T *WK, const T *WV, const T *wg, int D, int a, int k) {
    if (k < D) return ldf<T>(WQ + static_cast<int64_t>(a) * D + k);
    if (k < 2 * D) return ldf<T>(WK + static_cast<int64_t>(a) * D + k - D);
    if (k < 3 * D) return ldf<T>(WV + static_cast<int64_t>(a) * D + k - 2 * D);
    return ldf<T>(wg + a);
}

// dX[i][a] = sum_k dZ[i][k] * W_all[a][k]: 64 x 64 tiles of (rows, a), 16 k per step.
template <typename T>
__global__ void __launch_bounds__(256) bwd_dx_kernel(const float *__restrict__ dZ, const T *__restrict__ WQ,
                                                     const T *__restrict__ WK, const T *__restrict__ WV,
                                                     const T *__restrict__ wg, int64_t N, int d, int D, int Dz,
                                                     float *__restrict__ dX) {
    __shared__ float As[kTk][kTile], Bs[kTk][kTile];
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kTile;
    const int a0 = blockIdx.y * kTile;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < Dz; k0 += kTk) {
        for (int l = threadIdx.x; l < kTk * kTile; l += 256) {
            const int kk = l % kTk, rr = l / kTk;
            const int64_t i = i0 + rr;
            As[kk][rr] = (i < N && k0 + kk < Dz) ? dZ[i * Dz + k0 + kk] : 0.f;
            Bs[kk][rr] = (a0 + rr < d && k0 + kk < Dz) ? w_all<T>(WQ, WK, WV, wg, D, a0 + rr, k0 + kk) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kTk; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                av[u] = As[kk][ty * 4 + u];
                bv[u] = Bs[kk][tx * 4 + u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int64_t i = i0 + ty * 4 + u;
            const int a = a0 + tx * 4 + w;
            if (i < N && a < d) dX[i * d + a] = acc[u][w];
        }
}

// expand the CSR's rows: tgt[e] = i for e in [row_ptr[i], row_ptr[i+1])
__global__ void bwd_expand_rows_kernel(const int32_t *__restrict__ row_ptr, int64_t N, int32_t *__restrict__ tgt) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < N;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        for (int32_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) tgt[e] = static_cast<int32_t>(i);
}

// Features per lane of the warp-cooperative kernels: the smallest power of two with
// 32 * EPL >= D (a lane must stay inside one head, so EPL <= r is required).
int lane_features(int D) {
    int e = 1;
    while (32 * e < D) e <<= 1;
    return e;
}

// Both local backward kernels with EPL = lane_features(D): light rows one warp each,
// heavy rows (more than kHeavyDegree entries) one block each.
template <typename T>
void launch_local_bwd(Ctx *c, const T *Q, const T *KV, const T *L, float isr, int64_t Dz, cudaStream_t s) {
    const int H = c->H, R = c->r;
    const unsigned gq = static_cast<unsigned>(std::max<int64_t>(1, ceil_div(c->bw_nq_light * 32, 256)));
    const unsigned gk = static_cast<unsigned>(std::max<int64_t>(1, ceil_div(c->bw_nk_light * 32, 256)));
#define GLGA_LB(E)                                                                                        \
    case E:                                                                                               \
        if (c->bw_nq_light)                                                                               \
            bwd_local_q_kernel<T, E, false><<<gq, 256, 0, s>>>(c->bw_q_rows, c->bw_nq_light, c->row_ptr,   \
                c->col_idx, Q, KV, L, c->bw_dL, H, R, isr, c->bw_lse, c->bw_Dd, c->bw_dZ, Dz);            \
        if (c->bw_nq_heavy)                                                                               \
            bwd_local_q_kernel<T, E, true><<<static_cast<unsigned>(c->bw_nq_heavy), 1024, 0, s>>>(        \
                c->bw_q_rows + c->bw_nq_light, c->bw_nq_heavy, c->row_ptr, c->col_idx, Q, KV, L, c->bw_dL, \
                H, R, isr, c->bw_lse, c->bw_Dd, c->bw_dZ, Dz);                                            \
        if (c->bw_nk_light)                                                                               \
            bwd_local_kv_kernel<T, E, false><<<gk, 256, 0, s>>>(c->bw_k_rows, c->bw_nk_light,             \
                c->t_row_ptr, c->t_col, Q, KV, c->bw_dL, c->bw_lse, c->bw_Dd, c->bw_dSz, c->bw_dST, H, R, isr, \
                c->bw_dZ, Dz);                                                                            \
        if (c->bw_nk_heavy)                                                                               \
            bwd_local_kv_kernel<T, E, true><<<static_cast<unsigned>(c->bw_nk_heavy), 1024, 0, s>>>(       \
                c->bw_k_rows + c->bw_nk_light, c->bw_nk_heavy, c->t_row_ptr, c->t_col, Q, KV, c->bw_dL,    \
                c->bw_lse, c->bw_Dd, c->bw_dSz, c->bw_dST, H, R, isr, c->bw_dZ, Dz);                                 \
        break;
    switch (lane_features(c->D)) {
        GLGA_LB(1) GLGA_LB(2) GLGA_LB(4) GLGA_LB(8) GLGA_LB(16) GLGA_LB(32)
        default: break;
    }
#undef GLGA_LB
}

template <typename T>
void launch_readout_bwd(Ctx *c, const T *Q, const T *dY, float b_g, float eps, int64_t Dz, cudaStream_t s) {
    const unsigned grid = static_cast<unsigned>(ceil_div(c->N * 32, 256));
#define GLGA_RB(E)                                                                                       \
    case E:                                                                                              \
        bwd_readout_kernel<T, E><<<grid, 256, 0, s>>>(Q, static_cast<const T *>(c->L), c->t, c->Sz, c->bw_ST, dY, \
                                                      c->N, c->H, c->r, b_g, eps, c->bw_dL, c->bw_dnum,  \
                                                      c->bw_dden, c->bw_dZ, Dz);                         \
        break;
    switch (lane_features(c->D)) {
        GLGA_RB(1) GLGA_RB(2) GLGA_RB(4) GLGA_RB(8) GLGA_RB(16) GLGA_RB(32)
        default: break;
    }
#undef GLGA_RB
}

template <typename T>
void launch_dsz_bwd(Ctx *c, const T *Q, int64_t rpp, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>(c->bw_parts), static_cast<unsigned>(c->H));
    const size_t smem = (32 * c->r + 32 * (c->r + 1)) * sizeof(float);
#define GLGA_DZ(RR)                                                                                      \
    case RR:                                                                                             \
        bwd_dsz_partial_kernel<T, RR><<<grid, 256, smem, s>>>(Q, c->bw_dnum, c->bw_dden, c->N, c->H, rpp, \
                                                              c->bw_dsz_part);                           \
        break;
    switch (c->r) {
        GLGA_DZ(8) GLGA_DZ(16) GLGA_DZ(32) GLGA_DZ(64) GLGA_DZ(128)
        default: break;
    }
#undef GLGA_DZ
}

// Light rows first, then heavy ones (more than kHeavyDegree entries), by a CSR's offsets.
constexpr int64_t kHeavyDegree = 128;
void split_rows(const std::vector<int32_t> &rp, std::vector<int32_t> &rows, int64_t &n_light, int64_t &n_heavy) {
    const int64_t n = static_cast<int64_t>(rp.size()) - 1;
    rows.clear();
    for (int64_t i = 0; i < n; ++i)
        if (rp[i + 1] - rp[i] <= kHeavyDegree) rows.push_back(static_cast<int32_t>(i));
    n_light = static_cast<int64_t>(rows.size());
    for (int64_t i = 0; i < n; ++i)
        if (rp[i + 1] - rp[i] > kHeavyDegree) rows.push_back(static_cast<int32_t>(i));
    n_heavy = static_cast<int64_t>(rows.size()) - n_light;
}

int64_t ceil_parts(int64_t N, int64_t want) { return std::max<int64_t>(1, std::min<int64_t>(want, N)); }

}  // namespace

glga_status backward_setup(Ctx *c, cudaStream_t s) {
    if (!c->opts.backward) return GLGA_OK;
    if (c->sharded || c->n_seg != 1) {
        set_error("glga_create: the backward pass is for whole-graph, one-segment contexts");
        return GLGA_ERR_UNSUPPORTED;
    }
    if (lane_features(c->D) > c->r) {
        set_error("glga_create: the backward pass needs H*r <= 32*r (at most 32 heads)");
        return GLGA_ERR_UNSUPPORTED;
    }
    const int64_t N = c->N, E = c->E, D = c->D, H = c->H, R = c->r;
    c->bw_dz_ld = 3 * D + 1;
    c->bw_parts = static_cast<int32_t>(ceil_parts(N, c->num_sms));
    const int64_t tiles = ceil_div(c->d, kTile) * ceil_div(c->bw_dz_ld, kTile);
    c->bw_wparts = static_cast<int32_t>(ceil_parts(N, std::max<int64_t>(1, 2 * c->num_sms / tiles)));
    const size_t f = sizeof(float);
    const int64_t nz = std::max<int64_t>(N, 1);
    glga_status st = GLGA_OK;
#define BTRY(x) \
    if (st == GLGA_OK) st = (x)
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->t_row_ptr), (N + 1) * sizeof(int32_t)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->t_col), std::max<int64_t>(E, 1) * sizeof(int32_t)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dL), nz * D * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dnum), nz * D * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dden), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_lse), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_Dd), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dZ), nz * c->bw_dz_ld * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dsz_part), static_cast<size_t>(c->bw_parts) * H * R * (R + 1) * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dSz), static_cast<size_t>(H) * R * (R + 1) * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_ST), static_cast<size_t>(H) * R * R * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dST), static_cast<size_t>(H) * R * R * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dw_part),
                   static_cast<size_t>(c->bw_wparts) * c->d * c->bw_dz_ld * f));
#undef BTRY
    if (st != GLGA_OK) return st;
    // transposed CSR: rows by source j, listing the targets i of j's out-edges in order
    int32_t *tgt = nullptr;
    if (E > 0) {
        st = debug_alloc_hook(c);
        if (st != GLGA_OK) return st;
        GLGA_CUDA(cudaMalloc(&tgt, E * sizeof(int32_t)));
        bwd_expand_rows_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(N, 256), 4096)), 256, 0, s>>>(
            c->row_ptr, N, tgt);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) {
            cudaFree(tgt);
            return cuda_fail(e, "backward transpose");
        }
    }
    st = glga_csr_from_coo(N, E, tgt, c->col_idx, c->t_row_ptr, c->t_col, s);
    if (tgt) {
        cudaStreamSynchronize(s);
        cudaFree(tgt);
    }
    if (st != GLGA_OK) return st;
    // row lists of the two local backward kernels: light rows first, then heavy rows
    std::vector<int32_t> rp(static_cast<size_t>(N) + 1), trp(static_cast<size_t>(N) + 1), qr, kr;
    GLGA_CUDA(cudaMemcpy(rp.data(), c->row_ptr, rp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost));
    GLGA_CUDA(cudaMemcpy(trp.data(), c->t_row_ptr, trp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost));
    split_rows(rp, qr, c->bw_nq_light, c->bw_nq_heavy);
    split_rows(trp, kr, c->bw_nk_light, c->bw_nk_heavy);
    st = dev_alloc(c, reinterpret_cast<void **>(&c->bw_q_rows), (qr.size() + 1) * sizeof(int32_t));
    if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->bw_k_rows), (kr.size() + 1) * sizeof(int32_t));
    if (st != GLGA_OK) return st;
    if (!qr.empty()) GLGA_CUDA(cudaMemcpy(c->bw_q_rows, qr.data(), qr.size() * sizeof(int32_t), cudaMemcpyHostToDevice));
    if (!kr.empty()) GLGA_CUDA(cudaMemcpy(c->bw_k_rows, kr.data(), kr.size() * sizeof(int32_t), cudaMemcpyHostToDevice));
    return GLGA_OK;
}

glga_status backward_run(Ctx *c, const void *X, const void *WQ, const void *WK, const void *WV,
                         const void *wg, float b_g, float eps, const void *dY, float *dX, float *dWQ,
                         float *dWK, float *dWV, float *dwg, float *db_g, cudaStream_t s) {
    const int64_t N = c->N;
    const int H = c->H, R = c->r, D = c->D, d = c->d;
    const int Dz = static_cast<int>(c->bw_dz_ld);
    const float isr = 1.f / std::sqrt(static_cast<float>(R));
    const int total = H * R * (R + 1);
    const int64_t rpp = ceil_div(std::max<int64_t>(N, 1), c->bw_parts);
    const int64_t wrpp = ceil_div(std::max<int64_t>(N, 1), c->bw_wparts);
    const int64_t wtotal = static_cast<int64_t>(d) * Dz;
#define BWD_LAUNCHES(T)                                                                                   \
    do {                                                                                                  \
        const T *Q = static_cast<const T *>(c->Q);                                                        \
        const T *KV = static_cast<const T *>(c->KV);                                                      \
        const unsigned tgrid = static_cast<unsigned>(ceil_div(static_cast<int64_t>(H) * R * R, 256));    \
        if (N > 0) {                                                                                      \
            bwd_transpose_heads_kernel<<<tgrid, 256, 0, s>>>(c->Sz, R, H, R, c->bw_ST);                  \
            launch_readout_bwd<T>(c, Q, static_cast<const T *>(dY), b_g, eps, Dz, s);                  \
            launch_dsz_bwd<T>(c, Q, rpp, s);                                                              \
        }                                                                                                 \
        bwd_sum_parts_kernel<<<static_cast<unsigned>(ceil_div(total, 256)), 256, 0, s>>>(                 \
            c->bw_dsz_part, N > 0 ? c->bw_parts : 0, total, c->bw_dSz);                                   \
        if (N > 0) {                                                                                      \
            bwd_transpose_heads_kernel<<<tgrid, 256, 0, s>>>(c->bw_dSz, R + 1, H, R, c->bw_dST);         \
            launch_local_bwd<T>(c, Q, KV, static_cast<const T *>(c->L), isr, Dz, s);                  \
            bwd_dw_kernel<T><<<dim3(ceil_div(d, kTile), ceil_div(Dz, kTile), c->bw_wparts), 256, 0, s>>>( \
                static_cast<const T *>(X), c->bw_dZ, N, d, Dz, wrpp, c->bw_dw_part);                     \
            bwd_dx_kernel<T><<<dim3(ceil_div(N, kTile), ceil_div(d, kTile)), 256, 0, s>>>(                \
                c->bw_dZ, static_cast<const T *>(WQ), static_cast<const T *>(WK),                         \
                static_cast<const T *>(WV), static_cast<const T *>(wg), N, d, D, Dz, dX);                \
        }                                                                                                 \
    } while (0)
    if (c->io == GLGA_F32)
        BWD_LAUNCHES(float);
    else
        BWD_LAUNCHES(__nv_bfloat16);
#undef BWD_LAUNCHES
    if (N > 0) {
        bwd_dw_reduce_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(wtotal, 256), 4096)), 256, 0, s>>>(
            c->bw_dw_part, c->bw_wparts, d, D, Dz, dWQ, dWK, dWV, dwg);
        bwd_dbg_kernel<<<1, 1024, 0, s>>>(c->bw_dZ, N, Dz, 3 * D, db_g);
    } else {
        GLGA_CUDA(cudaMemsetAsync(dWQ, 0, static_cast<size_t>(d) * D * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(dWK, 0, static_cast<size_t>(d) * D * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(dWV, 0, static_cast<size_t>(d) * D * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(dwg, 0, static_cast<size_t>(d) * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(db_g, 0, sizeof(float), s));
    }
    GLGA_CUDA(cudaGetLastError());
    c->launches += N > 0 ? 12 : 1;
    return GLGA_OK;
}

}  // namespace glga
