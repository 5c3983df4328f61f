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

constexpr int kMaxR = 128;

// One thread per (row i, head h): the gate, readout and blend backward.  Writes
// dL [N, D], dnum [N, D], dden [N, H], the gate partial dg [N, H] and the global part of
// dQ into dZ [:, 0:D].
template <typename T>
__global__ void bwd_readout_kernel(const T *__restrict__ Q, const T *__restrict__ L, const float *__restrict__ t,
                                   const float *__restrict__ Sz, const T *__restrict__ dY, int64_t N, int H,
                                   int R, float b_g, float eps, float *__restrict__ dL,
                                   float *__restrict__ dnum, float *__restrict__ dden, float *__restrict__ dg,
                                   float *__restrict__ dZ, int64_t dz_ld) {
    const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (idx >= N * H) return;
    const int64_t i = idx / H;
    const int h = static_cast<int>(idx % H);
    const int D = H * R;
    const float *S = Sz + static_cast<int64_t>(h) * R * R;
    const float *z = Sz + static_cast<int64_t>(H) * R * R + h * R;
    const T *q = Q + i * D + h * R;
    float phq[kMaxR];
    float den = eps;
    for (int a = 0; a < R; ++a) {
        phq[a] = phi(ldf<T>(q + a));
        den = fmaf(phq[a], z[a], den);
    }
    const float g = 1.f / (1.f + __expf(-(t[i] + b_g)));
    float dgp = 0.f, dG_dot_G = 0.f;
    const int64_t o = i * D + h * R;
    for (int c = 0; c < R; ++c) {
        float num = 0.f;
        for (int a = 0; a < R; ++a) num = fmaf(phq[a], S[a * R + c], num);
        const float Gc = num / den;
        const float dy = ldf<T>(dY + o + c);
        dgp = fmaf(dy, ldf<T>(L + o + c) - Gc, dgp);
        dL[o + c] = g * dy;
        const float dGc = (1.f - g) * dy;
        dnum[o + c] = dGc / den;
        dG_dot_G = fmaf(dGc, Gc, dG_dot_G);
    }
    const float dd = -dG_dot_G / den;
    dden[idx] = dd;
    dg[idx] = dgp;
    for (int a = 0; a < R; ++a) {
        float acc = z[a] * dd;
        for (int c = 0; c < R; ++c) acc = fmaf(S[a * R + c], dnum[o + c], acc);
        dZ[i * dz_ld + h * R + a] = acc * dphi(ldf<T>(q + a));
    }
}

// Partial sums over the row range of part p of dS | dz in the layout [H][R][R+1]
// (column R is dz): part[p][h][a][c] = sum_i phi(q_i[h R + a]) * (dnum_i[h R + c] or
// dden_i[h]).
template <typename T>
__global__ void bwd_dsz_partial_kernel(const T *__restrict__ Q, const float *__restrict__ dnum,
                                       const float *__restrict__ dden, int64_t N, int H, int R,
                                       int64_t rows_per_part, float *__restrict__ part) {
    const int total = H * R * (R + 1);
    const int o = blockIdx.y * blockDim.x + threadIdx.x;
    if (o >= total) return;
    const int per_head = R * (R + 1);
    const int h = o / per_head, rem = o % per_head, a = rem / (R + 1), c = rem % (R + 1);
    const int D = H * R;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_part;
    const int64_t r1 = std::min<int64_t>(N, r0 + rows_per_part);
    float acc = 0.f;
    for (int64_t i = r0; i < r1; ++i) {
        const float w = c < R ? dnum[i * D + h * R + c] : dden[i * H + h];
        acc = fmaf(phi(ldf<T>(Q + i * D + h * R + a)), w, acc);
    }
    part[static_cast<int64_t>(blockIdx.x) * total + o] = acc;
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

// One thread per (target i, head h) over the forward CSR: the softmax's log-sum-exp,
// D_i = dL_i . L_i, and the local part of dq_i added into dZ [:, 0:D].
template <typename T>
__global__ void bwd_local_q_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                                   const T *__restrict__ Q, const T *__restrict__ KV, const T *__restrict__ L,
                                   const float *__restrict__ dL, int64_t N, int H, int R, float inv_sqrt_r,
                                   float *__restrict__ lse, float *__restrict__ Dd, float *__restrict__ dZ,
                                   int64_t dz_ld) {
    const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (idx >= N * H) return;
    const int64_t i = idx / H;
    const int h = static_cast<int>(idx % H);
    const int D = H * R;
    const T *q = Q + i * D + h * R;
    const int32_t e0 = row_ptr[i], e1 = row_ptr[i + 1];
    float m = -INFINITY, l = 0.f;
    for (int32_t e = e0; e < e1; ++e) {
        const T *k = KV + static_cast<int64_t>(col_idx[e]) * 2 * D + h * R;
        float s = 0.f;
        for (int a = 0; a < R; ++a) s = fmaf(ldf<T>(q + a), ldf<T>(k + a), s);
        s *= inv_sqrt_r;
        const float mn = fmaxf(m, s);
        l = l * __expf(m - mn) + __expf(s - mn);
        m = mn;
    }
    const float ls = e1 > e0 ? m + __logf(l) : 0.f;
    float dd = 0.f;
    const int64_t o = i * D + h * R;
    for (int c = 0; c < R; ++c) dd = fmaf(dL[o + c], ldf<T>(L + o + c), dd);
    lse[idx] = ls;
    Dd[idx] = dd;
    float dq[kMaxR];
    for (int a = 0; a < R; ++a) dq[a] = 0.f;
    for (int32_t e = e0; e < e1; ++e) {
        const T *k = KV + static_cast<int64_t>(col_idx[e]) * 2 * D + h * R;
        const T *v = k + D;
        float s = 0.f, dp = 0.f;
        for (int a = 0; a < R; ++a) {
            s = fmaf(ldf<T>(q + a), ldf<T>(k + a), s);
            dp = fmaf(dL[o + a], ldf<T>(v + a), dp);
        }
        const float p = __expf(s * inv_sqrt_r - ls);
        const float ds = p * (dp - dd) * inv_sqrt_r;
        for (int a = 0; a < R; ++a) dq[a] = fmaf(ds, ldf<T>(k + a), dq[a]);
    }
    for (int a = 0; a < R; ++a) dZ[i * dz_ld + h * R + a] += dq[a];
}

// One thread per (source j, head h) over the transposed CSR (the targets i of j): the
// local terms of dk_j and dv_j, plus the global terms through phi(k_j), written to
// dZ [:, D:2D] and [:, 2D:3D].  dSz holds dS | dz as [H][R][R+1].
template <typename T>
__global__ void bwd_local_kv_kernel(const int32_t *__restrict__ t_row_ptr, const int32_t *__restrict__ t_col,
                                    const T *__restrict__ Q, const T *__restrict__ KV,
                                    const float *__restrict__ dL, const float *__restrict__ lse,
                                    const float *__restrict__ Dd, const float *__restrict__ dSz, int64_t N,
                                    int H, int R, float inv_sqrt_r, float *__restrict__ dZ, int64_t dz_ld) {
    const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (idx >= N * H) return;
    const int64_t j = idx / H;
    const int h = static_cast<int>(idx % H);
    const int D = H * R;
    const T *k = KV + j * 2 * D + h * R;
    const T *v = k + D;
    float dk[kMaxR], dv[kMaxR];
    for (int a = 0; a < R; ++a) dk[a] = dv[a] = 0.f;
    const int32_t e0 = t_row_ptr[j], e1 = t_row_ptr[j + 1];
    for (int32_t e = e0; e < e1; ++e) {
        const int64_t i = t_col[e];
        const T *q = Q + i * D + h * R;
        const float *dl = dL + i * D + h * R;
        float s = 0.f, dp = 0.f;
        for (int a = 0; a < R; ++a) {
            s = fmaf(ldf<T>(q + a), ldf<T>(k + a), s);
            dp = fmaf(dl[a], ldf<T>(v + a), dp);
        }
        const float p = __expf(s * inv_sqrt_r - lse[i * H + h]);
        const float ds = p * (dp - Dd[i * H + h]) * inv_sqrt_r;
        for (int a = 0; a < R; ++a) {
            dv[a] = fmaf(p, dl[a], dv[a]);
            dk[a] = fmaf(ds, ldf<T>(q + a), dk[a]);
        }
    }
    // global branch: S = sum phi(k) v^T, z = sum phi(k)
    const float *dS = dSz + static_cast<int64_t>(h) * R * (R + 1);
    for (int a = 0; a < R; ++a) {
        const float ka = ldf<T>(k + a);
        float dphk = dS[a * (R + 1) + R];            // dz_a
        for (int c = 0; c < R; ++c) dphk = fmaf(dS[a * (R + 1) + c], ldf<T>(v + c), dphk);
        dk[a] = fmaf(dphk, dphi(ka), dk[a]);
        const float pk = phi(ka);
        for (int c = 0; c < R; ++c) dv[c] = fmaf(dS[a * (R + 1) + c], pk, dv[c]);
    }
    for (int a = 0; a < R; ++a) {
        dZ[j * dz_ld + D + h * R + a] = dk[a];
        dZ[j * dz_ld + 2 * D + h * R + a] = dv[a];
    }
}

// dt_i = g (1 - g) sum_h dg[i][h], the gate logit column of dZ.
__global__ void bwd_dt_kernel(const float *__restrict__ t, const float *__restrict__ dg, int64_t N, int H,
                              float b_g, float *__restrict__ dZ, int64_t dz_ld, int64_t col) {
    const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (i >= N) return;
    float s = 0.f;
    for (int h = 0; h < H; ++h) s += dg[i * H + h];
    const float g = 1.f / (1.f + __expf(-(t[i] + b_g)));
    dZ[i * dz_ld + col] = g * (1.f - g) * s;
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

int64_t ceil_parts(int64_t N, int64_t want) { return std::max<int64_t>(1, std::min<int64_t>(want, N)); }

}  // namespace

glga_status backward_setup(Ctx *c, cudaStream_t s) {
    if (!c->opts.backward) return GLGA_OK;
    if (c->sharded || c->n_seg != 1) {
        set_error("glga_create: the backward pass is for whole-graph, one-segment contexts");
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
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dg), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_lse), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_Dd), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dZ), nz * c->bw_dz_ld * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dsz_part), static_cast<size_t>(c->bw_parts) * H * R * (R + 1) * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dSz), static_cast<size_t>(H) * R * (R + 1) * f));
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
    return st;
}

glga_status backward_run(Ctx *c, const void *X, const void *WQ, const void *WK, const void *WV,
                         const void *wg, float b_g, float eps, const void *dY, float *dX, float *dWQ,
                         float *dWK, float *dWV, float *dwg, float *db_g, cudaStream_t s) {
    const int64_t N = c->N;
    const int H = c->H, R = c->r, D = c->D, d = c->d;
    const int Dz = static_cast<int>(c->bw_dz_ld);
    const float isr = 1.f / std::sqrt(static_cast<float>(R));
    const int64_t nh = N * H;
    const unsigned gnh = static_cast<unsigned>(std::max<int64_t>(1, ceil_div(nh, 128)));
    const int total = H * R * (R + 1);
    const int64_t rpp = ceil_div(std::max<int64_t>(N, 1), c->bw_parts);
    const int64_t wrpp = ceil_div(std::max<int64_t>(N, 1), c->bw_wparts);
    const int64_t wtotal = static_cast<int64_t>(d) * Dz;
#define BWD_LAUNCHES(T)                                                                                   \
    do {                                                                                                  \
        const T *Q = static_cast<const T *>(c->Q);                                                        \
        const T *KV = static_cast<const T *>(c->KV);                                                      \
        if (N > 0) {                                                                                      \
            bwd_readout_kernel<T><<<gnh, 128, 0, s>>>(Q, static_cast<const T *>(c->L), c->t, c->Sz,       \
                                                      static_cast<const T *>(dY), N, H, R, b_g, eps,      \
                                                      c->bw_dL, c->bw_dnum, c->bw_dden, c->bw_dg,         \
                                                      c->bw_dZ, Dz);                                      \
            bwd_dsz_partial_kernel<T><<<dim3(c->bw_parts, ceil_div(total, 256)), 256, 0, s>>>(           \
                Q, c->bw_dnum, c->bw_dden, N, H, R, rpp, c->bw_dsz_part);                                 \
        }                                                                                                 \
        bwd_sum_parts_kernel<<<static_cast<unsigned>(ceil_div(total, 256)), 256, 0, s>>>(                 \
            c->bw_dsz_part, N > 0 ? c->bw_parts : 0, total, c->bw_dSz);                                   \
        if (N > 0) {                                                                                      \
            bwd_local_q_kernel<T><<<gnh, 128, 0, s>>>(c->row_ptr, c->col_idx, Q, KV,                      \
                                                      static_cast<const T *>(c->L), c->bw_dL, N, H, R,    \
                                                      isr, c->bw_lse, c->bw_Dd, c->bw_dZ, Dz);            \
            bwd_local_kv_kernel<T><<<gnh, 128, 0, s>>>(c->t_row_ptr, c->t_col, Q, KV, c->bw_dL,           \
                                                       c->bw_lse, c->bw_Dd, c->bw_dSz, N, H, R, isr,      \
                                                       c->bw_dZ, Dz);                                     \
            bwd_dt_kernel<<<static_cast<unsigned>(ceil_div(N, 256)), 256, 0, s>>>(c->t, c->bw_dg, N, H,   \
                                                                                  b_g, c->bw_dZ, Dz,      \
                                                                                  3 * D);                 \
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
    c->launches += N > 0 ? 10 : 1;
    return GLGA_OK;
}

}  // namespace glga
