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
// atomics (two runs give identical bits).  The gathers run on the CUDA cores (one row, or
// one 64-edge chunk of a heavy row, per warp or per 16-lane half), bf16 rows kept packed
// for fma.rn.f32.bf16 with f32 accumulation; for bf16 layers each edge's (p, ds) is formed
// once, by the target side, and handed to the source side at the edge's transposed
// position.  Every dense product of bf16 layers with H*r = 128 runs on the tcgen05 tensor
// cores (the readout backward, dS | dz, the source side's global terms, dX | dW in one
// pass); fp32 layers and other widths use register-tiled CUDA-core kernels.  Gradients are
// fp32.  The log-sum-exp of each row's scores comes from the forward.
#include <algorithm>
#include <cmath>
#include <type_traits>
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

// Warp-cooperative row kernels: one warp per row (or per chunk of a row's edges), lane l
// holds the EPL consecutive features l*EPL .. l*EPL+EPL-1 of every row it reads
// (contiguous across the warp, so a row is one coalesced read), and a head's r features
// lie in LPH = r/EPL adjacent lanes, whose dot products meet in a butterfly of shuffles.
// r is a power of two and EPL <= r, so LPH is a power of two, D is a multiple of EPL and
// every lane's slice starts on an EPL-element boundary (the vector loads below rely on it).

template <int EPL>
__device__ __forceinline__ void unpack_bf16(const uint32_t *w, float *x) {
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) {
        const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162 *>(&w[e]);
        const float2 f = __bfloat1622float2(p);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}

template <typename T, int EPL>
__device__ __forceinline__ void ld_row(const T *row, int lane, bool act, float (&x)[EPL]) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) x[e] = 0.f;
    if (!act) return;
    const T *p = row + lane * EPL;
    if constexpr (std::is_same<T, float>::value) {
        if constexpr (EPL % 4 == 0) {
#pragma unroll
            for (int v = 0; v < EPL / 4; ++v) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(p) + v);
                x[4 * v] = f.x; x[4 * v + 1] = f.y; x[4 * v + 2] = f.z; x[4 * v + 3] = f.w;
            }
        } else if constexpr (EPL == 2) {
            const float2 f = __ldg(reinterpret_cast<const float2 *>(p));
            x[0] = f.x; x[1] = f.y;
        } else {
            x[0] = __ldg(p);
        }
    } else {
        if constexpr (EPL % 8 == 0) {
#pragma unroll
            for (int v = 0; v < EPL / 8; ++v) {
                const uint4 w = __ldg(reinterpret_cast<const uint4 *>(p) + v);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                unpack_bf16<8>(ww, x + 8 * v);
            }
        } else if constexpr (EPL == 4) {
            const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
            const uint32_t ww[2] = {w.x, w.y};
            unpack_bf16<4>(ww, x);
        } else if constexpr (EPL == 2) {
            const uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(p));
            unpack_bf16<2>(&w, x);
        } else {
            x[0] = __bfloat162float(*p);
        }
    }
}

// x = p[0 .. EPL-1] of an fp32 matrix row (p on an EPL-float boundary).  NC: through the
// read-only path (data the kernel does not write); otherwise plain loads.
template <int EPL, bool NC = true>
__device__ __forceinline__ void ld_mrow(const float *p, float (&x)[EPL]) {
    if constexpr (EPL % 4 == 0) {
#pragma unroll
        for (int v = 0; v < EPL / 4; ++v) {
            const float4 *a = reinterpret_cast<const float4 *>(p) + v;
            const float4 f = NC ? __ldg(a) : *a;
            x[4 * v] = f.x; x[4 * v + 1] = f.y; x[4 * v + 2] = f.z; x[4 * v + 3] = f.w;
        }
    } else if constexpr (EPL == 2) {
        const float2 *a = reinterpret_cast<const float2 *>(p);
        const float2 f = NC ? __ldg(a) : *a;
        x[0] = f.x; x[1] = f.y;
    } else {
        x[0] = NC ? __ldg(p) : *p;
    }
}

// p[0 .. EPL-1] = x for an fp32 row slice on an EPL-float boundary.
template <int EPL>
__device__ __forceinline__ void st_mrow(float *p, const float (&x)[EPL]) {
    if constexpr (EPL % 4 == 0) {
#pragma unroll
        for (int v = 0; v < EPL / 4; ++v)
            reinterpret_cast<float4 *>(p)[v] = make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
    } else if constexpr (EPL == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    } else {
        p[0] = x[0];
    }
}

// p[0 .. EPL-1] = x rounded to T, for a row slice on an EPL-element boundary.
template <typename T, int EPL>
__device__ __forceinline__ void st_row(T *p, const float (&x)[EPL]) {
    if constexpr (std::is_same<T, float>::value) {
        st_mrow<EPL>(p, x);
    } else if constexpr (EPL == 1) {
        p[0] = __float2bfloat16_rn(x[0]);
    } else {
        uint32_t w[EPL / 2];
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t *>(&h);
        }
        if constexpr (EPL % 8 == 0) {
#pragma unroll
            for (int v = 0; v < EPL / 8; ++v)
                reinterpret_cast<uint4 *>(p)[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        } else if constexpr (EPL == 4) {
            *reinterpret_cast<uint2 *>(p) = make_uint2(w[0], w[1]);
        } else {
            *reinterpret_cast<uint32_t *>(p) = w[0];
        }
    }
}

// Two floats rounded to bf16 (nearest even) in one word, lo in bits 0..15.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 2^x by the PTX ex2.approx.ftz instruction (the arguments are scores minus the row's
// log-sum-exp, at most a few units above zero).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// acc[2w + e] += s x[w].half(e) for the bf16 s in the HIGH half of s2.
template <int W>
__device__ __forceinline__ void axpy_bf16w_hi(uint32_t s2, const uint32_t *x, float *acc) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
        acc[2 * w] = fma_bf16h<1, 0>(s2, x[w], acc[2 * w]);
        acc[2 * w + 1] = fma_bf16h<1, 1>(s2, x[w], acc[2 * w + 1]);
    }
}

// (p, ds) rounded to bf16 in one word: p in the low half, ds in the high half.
__device__ __forceinline__ uint32_t pack_p_ds(float p, float ds) {
    uint32_t w;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(ds), "f"(p));
    return w;
}

// x = the EPL bf16 values at p (p on an EPL-element boundary), by plain loads
// (the kernel may write the same place afterwards).
template <int EPL>
__device__ __forceinline__ void ld_bf16_slice(const __nv_bfloat16 *p, float (&x)[EPL]) {
    if constexpr (EPL == 1) {
        x[0] = __bfloat162float(*p);
        return;
    }
    uint32_t w[EPL > 1 ? EPL / 2 : 1];
    if constexpr (EPL % 8 == 0) {
#pragma unroll
        for (int v = 0; v < EPL / 8; ++v) {
            const uint4 u = reinterpret_cast<const uint4 *>(p)[v];
            w[4 * v] = u.x; w[4 * v + 1] = u.y; w[4 * v + 2] = u.z; w[4 * v + 3] = u.w;
        }
    } else if constexpr (EPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        w[0] = u.x; w[1] = u.y;
    } else {
        w[0] = *reinterpret_cast<const uint32_t *>(p);
    }
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}

// x as a T row stores it.
template <typename T>
__device__ __forceinline__ float round_to(float x) {
    if constexpr (std::is_same<T, float>::value) return x;
    else return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float head_reduce(float x, int lph) {
    for (int o = 1; o < lph; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// out[k][x] += sum over c < R of M[c * R + f0 + x] * u[k]_c for one head and each of the
// warp's RPW rows k: M is a row-major R x R fp32 block, and u[k]_c is held by the head's
// lanes (lane hb + c / EPL, element c % EPL), so it travels by shuffle; each row of M is
// loaded once for all RPW rows.  LPH = R / EPL when known at compile time (the loop is
// then unrolled), else 0 and lph gives it.  Every lane of the warp takes part (lanes
// outside D pass f0 = 0 and hb = 0 and discard the result).
template <int EPL, int LPH, int RPW>
__device__ __forceinline__ void head_matvec(const float *M, int R, int f0, int hb, int lph,
                                            const float (&u)[RPW][EPL], float (&out)[RPW][EPL]) {
    auto step = [&](int sl) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            float m[EPL];
            ld_mrow<EPL>(M + static_cast<int64_t>(sl * EPL + e) * R + f0, m);
#pragma unroll
            for (int k = 0; k < RPW; ++k) {
                const float uc = __shfl_sync(0xffffffffu, u[k][e], hb + sl);
#pragma unroll
                for (int x = 0; x < EPL; ++x) out[k][x] = fmaf(m[x], uc, out[k][x]);
            }
        }
    };
    if constexpr (LPH > 0) {
#pragma unroll 4
        for (int sl = 0; sl < LPH; ++sl) step(sl);
    } else {
        for (int sl = 0; sl < lph; ++sl) step(sl);
    }
}

// One row (the source side's global terms).
template <int EPL>
__device__ __forceinline__ void head_matvec(const float *M, int R, int f0, int hb, int lph, const float (&u)[EPL],
                                            float (&out)[EPL]) {
    head_matvec<EPL, 0, 1>(M, R, f0, hb, lph, reinterpret_cast<const float (&)[1][EPL]>(u),
                           reinterpret_cast<float (&)[1][EPL]>(out));
}

// The lane's head h, in-head feature offset f0 and the head's first lane hb.
struct LaneHead {
    bool act;
    int lph, h, f0, hb;
    __device__ __forceinline__ LaneHead(int lane, int EPL, int D, int R) {
        act = lane * EPL < D;
        lph = R / EPL;
        h = act ? lane * EPL / R : 0;
        f0 = act ? lane * EPL - h * R : 0;
        hb = act ? h * lph : 0;
    }
};

// One warp per RPW consecutive rows i: the gate, readout and blend backward.  Writes dL
// [N, D], D_i = dL_i . L_i per head into Dd [N, H], dnum [N, D], dden [N, H], the global
// part of dQ into dZ [:, 0:D] and dt into dZ [:, 3D] (dg summed over the whole row in lane
// order).  Sz holds S [H][R][R] then z [H][R]; ST [H][R][R] is S transposed per head.
// Rows past N (in the last warp) compute on zeros and store nothing.
template <typename T, int EPL, int LPH, int RPW>
__global__ void __launch_bounds__(256, EPL <= 8 ? 2 : 1) bwd_readout_kernel(
    const T *__restrict__ Q, const T *__restrict__ L, const float *__restrict__ t, const float *__restrict__ Sz,
    const float *__restrict__ ST, const T *__restrict__ dY, int64_t N, int H, int R, float b_g, float eps,
    T *__restrict__ dL, float *__restrict__ Dd, float *__restrict__ dnum, float *__restrict__ dden,
    float *__restrict__ dZ, int64_t dz_ld) {
    const int64_t i0 = ((blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5) * RPW;
    const int lane = threadIdx.x & 31;
    if (i0 >= N) return;                                  // warp-uniform
    const int D = H * R;
    const LaneHead lh(lane, EPL, D, R);
    const int lph = LPH > 0 ? LPH : lh.lph;              // lanes per head (a constant when known)
    const float *S = Sz + static_cast<int64_t>(lh.h) * R * R;
    float q[RPW][EPL], dy[RPW][EPL], lv[RPW][EPL], ph[RPW][EPL], zz[EPL];
    bool live[RPW];
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        const int64_t i = i0 + k;
        live[k] = i < N;
        ld_row<T, EPL>(Q + i * D, lane, lh.act && live[k], q[k]);
        ld_row<T, EPL>(dY + i * D, lane, lh.act && live[k], dy[k]);
        ld_row<T, EPL>(L + i * D, lane, lh.act && live[k], lv[k]);
    }
    ld_mrow<EPL>(Sz + static_cast<int64_t>(H) * R * R + lh.h * R + lh.f0, zz);
    float den[RPW], G[RPW][EPL];
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        den[k] = 0.f;
#pragma unroll
        for (int x = 0; x < EPL; ++x) {
            ph[k][x] = phi(q[k][x]);
            den[k] = fmaf(ph[k][x], zz[x], den[k]);
            G[k][x] = 0.f;
        }
        den[k] = head_reduce(den[k], lph) + eps;
    }
    head_matvec<EPL, LPH, RPW>(S, R, lh.f0, lh.hb, lh.lph, ph, G);  // num_f = sum_a phi(q_a) S[a][f]
    float dn[RPW][EPL], acc[RPW][EPL], dgp[RPW], gk[RPW];
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        const int64_t i = i0 + k;
        const float g = live[k] ? 1.f / (1.f + __expf(-(t[i] + b_g))) : 0.f;
        gk[k] = g;
        float dGG = 0.f, dLL = 0.f, gl[EPL];
        const float inv_den = 1.f / den[k];              // one division per row and head
        dgp[k] = 0.f;
#pragma unroll
        for (int x = 0; x < EPL; ++x) {
            G[k][x] *= inv_den;
            gl[x] = round_to<T>(g * dy[k][x]);            // dL as stored; D_i from the same values
            dLL = fmaf(gl[x], lv[k][x], dLL);
            dgp[k] = fmaf(dy[k][x], lv[k][x] - G[k][x], dgp[k]);
            const float dG = (1.f - g) * dy[k][x];
            dGG = fmaf(dG, G[k][x], dGG);
            dn[k][x] = dG * inv_den;
        }
        const int64_t o = i * D + lane * EPL;
        if (lh.act && live[k]) {
            st_row<T, EPL>(dL + o, gl);
            st_mrow<EPL>(dnum + o, dn[k]);
        }
        const float dd = -head_reduce(dGG, lph) * inv_den;
        dLL = head_reduce(dLL, lph);
        if (lh.act && live[k] && (lane % lph) == 0) {
            dden[i * H + lh.h] = dd;
            Dd[i * H + lh.h] = dLL;
        }
#pragma unroll
        for (int x = 0; x < EPL; ++x) acc[k][x] = zz[x] * dd;
    }
    // dphi(q)_f = sum_c S[f][c] dnum_c + z_f dden, through ST's rows c
    head_matvec<EPL, LPH, RPW>(ST + static_cast<int64_t>(lh.h) * R * R, R, lh.f0, lh.hb, lh.lph, dn, acc);
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        const int64_t i = i0 + k;
#pragma unroll
        for (int x = 0; x < EPL; ++x) acc[k][x] *= dphi(q[k][x]);
        if (lh.act && live[k]) st_mrow<EPL>(dZ + i * dz_ld + lane * EPL, acc[k]);
        float d = dgp[k];
        for (int w = 16; w > 0; w >>= 1) d += __shfl_xor_sync(0xffffffffu, d, w);
        if (lane == 0 && live[k]) dZ[i * dz_ld + 3 * D] = gk[k] * (1.f - gk[k]) * d;
    }
}

// Partial sums of dS | dz over the row range of block column p, per head h =
// blockIdx.y, in the layout [H][R][R+1] (column R is dz):
//   part[p][h][a][c] = sum_i phi(q_i[h R + a]) * (c < R ? dnum_i[h R + c] : dden_i[h]).
// Row tiles (32 rows; 8 at R = 128) of phi(Q_h), dnum_h and dden_h are staged in shared
// memory, the next one prefetched into registers during the current one; each thread
// owns 4 (a) x 4 (c) output tiles (NT of them when R >= 64) and, for the first column
// tile, the dz entries of its 4 a's.  For R <= 32 the block's threads form G row groups
// (group g takes rows g, g + G, ... of each staged tile), added in group order at the end.
template <typename T, int R>
__global__ void __launch_bounds__(256) bwd_dsz_partial_kernel(const T *__restrict__ Q, const float *__restrict__ dnum,
                                                              const float *__restrict__ dden, int64_t N, int H,
                                                              int64_t rows_per_part, float *__restrict__ part) {
    constexpr int kRowsT = R >= 128 ? 8 : 32, TR = R / 4, NTILE = TR * TR;   // rows per staged tile
    constexpr int G = NTILE >= 256 ? 1 : 256 / NTILE;
    constexpr int NT = NTILE >= 256 ? NTILE / 256 : 1;
    constexpr int PH = R * (R + 1);                      // outputs per head
    extern __shared__ float4 dsm4[];
    float *pq = reinterpret_cast<float *>(dsm4);          // [32][R] phi(q)
    float *pw = pq + kRowsT * R;                          // [32][R] dnum
    float *pd = pw + kRowsT * R;                          // [32] dden
    float *red = pd + kRowsT;                             // [G][PH] when G > 1
    const int h = blockIdx.y, t = threadIdx.x;
    const int D = H * R;
    const int g = G > 1 ? t / NTILE : 0;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_part;
    const int64_t r1 = std::min<int64_t>(N, r0 + rows_per_part);
    float acc[NT][4][4], accz[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            accz[n][u] = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[n][u][w] = 0.f;
        }
    // the next tile's inputs are loaded into registers while the current one is multiplied
    constexpr int kPer = (kRowsT * R + 255) / 256;
    float rq[kPer], rw[kPer], rd = 0.f;
    auto fetch = [&](int64_t i0) {
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int l = t + u * 256;
            const int64_t i = i0 + l / R;
            const bool in = l < kRowsT * R && i < r1;
            rq[u] = in ? phi(ldf<T>(Q + i * D + h * R + l % R)) : 0.f;
            rw[u] = in ? dnum[i * D + h * R + l % R] : 0.f;
        }
        if (t < kRowsT) rd = i0 + t < r1 ? dden[(i0 + t) * H + h] : 0.f;
    };
    if (r0 < r1) fetch(r0);
    for (int64_t i0 = r0; i0 < r1; i0 += kRowsT) {
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int l = t + u * 256;
            if (l < kRowsT * R) {
                pq[l] = rq[u];
                pw[l] = rw[u];
            }
        }
        if (t < kRowsT) pd[t] = rd;
        __syncthreads();
        if (i0 + kRowsT < r1) fetch(i0 + kRowsT);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int tile = G > 1 ? t % NTILE : t + n * 256;
            const int a0 = (tile / TR) * 4, c0 = (tile % TR) * 4;
            for (int rr = g; rr < kRowsT; rr += G) {
                const float4 av = *reinterpret_cast<const float4 *>(pq + rr * R + a0);
                const float4 bv = *reinterpret_cast<const float4 *>(pw + rr * R + c0);
                const float a4[4] = {av.x, av.y, av.z, av.w}, b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc[n][u][w] = fmaf(a4[u], b4[w], acc[n][u][w]);
                if (c0 == 0) {
                    const float dd = pd[rr];
#pragma unroll
                    for (int u = 0; u < 4; ++u) accz[n][u] = fmaf(a4[u], dd, accz[n][u]);
                }
            }
        }
        __syncthreads();
    }
    float *out = part + static_cast<int64_t>(blockIdx.x) * H * PH + static_cast<int64_t>(h) * PH;
    float *dst = G > 1 ? red + g * PH : out;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int tile = G > 1 ? t % NTILE : t + n * 256;
        const int a0 = (tile / TR) * 4, c0 = (tile % TR) * 4;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int w = 0; w < 4; ++w) dst[(a0 + u) * (R + 1) + c0 + w] = acc[n][u][w];
            if (c0 == 0) dst[(a0 + u) * (R + 1) + R] = accz[n][u];
        }
    }
    if constexpr (G > 1) {
        __syncthreads();
        for (int o = t; o < PH; o += 256) {
            float v = 0.f;
            for (int gg = 0; gg < G; ++gg) v += red[gg * PH + o];
            out[o] = v;
        }
    }
}

// Per-head R x R blocks of src (row stride ld, head stride R * ld): dstT[h][c][a] =
// src[h][a][c] and, when dstC is given, the compact copy dstC[h][a][c] = src[h][a][c]
// followed by column R of src as dstC[H R R + h R + a] (so dstC has the [S | z] layout).
__global__ void bwd_heads_prep_kernel(const float *__restrict__ src, int ld, int H, int R, float *__restrict__ dstT,
                                      float *__restrict__ dstC) {
    const int64_t RR = static_cast<int64_t>(R) * R, total = static_cast<int64_t>(H) * RR;
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < total;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t h = o / RR;
        const int u = static_cast<int>((o / R) % R), w = static_cast<int>(o % R);
        dstT[o] = src[(h * R + w) * ld + u];
        if (dstC) {
            dstC[o] = src[(h * R + u) * ld + w];
            if (w == 0) dstC[total + h * R + u] = src[(h * R + u) * ld + R];
        }
    }
}

// out[o] = sum over p of part[p][o], in a fixed order: a block takes 32 consecutive
// outputs o; its warp g adds the partials p = g, g + 8, g + 16, ... in order (coalesced
// 128-byte rows, four loads in flight), and warp 0 adds the 8 warp sums in warp order.
constexpr int kSumThreads = 256, kSumOut = 32;
__global__ void __launch_bounds__(kSumThreads) bwd_sum_parts_kernel(const float *__restrict__ part, int P,
                                                                    int64_t total, float *__restrict__ out) {
    __shared__ float red[kSumThreads / 32][kSumOut];
    const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
    constexpr int kG = kSumThreads / 32;
    const int64_t o = static_cast<int64_t>(blockIdx.x) * kSumOut + lane;
    float acc = 0.f;
    if (o < total) {
        int p = g;
        for (; p + 3 * kG < P; p += 4 * kG) {
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = __ldg(part + static_cast<int64_t>(p + u * kG) * total + o);
#pragma unroll
            for (int u = 0; u < 4; ++u) acc += v[u];
        }
        for (; p < P; p += kG) acc += __ldg(part + static_cast<int64_t>(p) * total + o);
    }
    red[g][lane] = acc;
    __syncthreads();
    if (g == 0 && o < total) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kG; ++w) sum += red[w][lane];
        out[o] = sum;
    }
}
unsigned sum_parts_grid(int64_t total) { return static_cast<unsigned>(ceil_div(total, kSumOut)); }

// out[a] = sum over p of part[p * sp + a * sa] (a < n), one warp per output: lane l adds
// p = l, l + 32, ... in order, then a fixed butterfly adds the lanes.
__global__ void __launch_bounds__(256) bwd_strided_sum_kernel(const float *__restrict__ part, int P, int64_t sp,
                                                              int64_t sa, int n, float *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int a = static_cast<int>((blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5);
    if (a >= n) return;                                   // warp-uniform
    float acc = 0.f;
    for (int p = lane; p < P; p += 32) acc += __ldg(part + static_cast<int64_t>(p) * sp + a * sa);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (lane == 0) out[a] = acc;
}

constexpr int kEU = 4;            // edges whose rows are loaded before any is used
constexpr int kChunk = 64;        // edges per chunk of a heavy row (one warp each)

// The lane's EPL bf16 values of a row (EPL even) as EPL / 2 packed words (zero if !act).
template <int EPL>
__device__ __forceinline__ void ld_words(const __nv_bfloat16 *row, int lane, bool act, uint32_t (&w)[EPL / 2]) {
#pragma unroll
    for (int x = 0; x < EPL / 2; ++x) w[x] = 0u;
    if (!act) return;
    const __nv_bfloat16 *p = row + lane * EPL;
    if constexpr (EPL % 8 == 0) {
#pragma unroll
        for (int v = 0; v < EPL / 8; ++v) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + v);
            w[4 * v] = u.x; w[4 * v + 1] = u.y; w[4 * v + 2] = u.z; w[4 * v + 3] = u.w;
        }
    } else if constexpr (EPL == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        w[0] = u.x; w[1] = u.y;
    } else {
        w[0] = __ldg(reinterpret_cast<const unsigned int *>(p));
    }
}

// EPL values that are bf16 numbers, packed into EPL / 2 words (exact).
template <int EPL>
__device__ __forceinline__ void pack_words(const float (&x)[EPL], uint32_t (&w)[EPL / 2]) {
#pragma unroll
    for (int i = 0; i < EPL / 2; ++i) w[i] = bf16x2_bits(x[2 * i], x[2 * i + 1]);
}

// dq += sum over edges [a, b) of ds_ij k_j (ds already scaled by 1/sqrt(r)).  bf16 rows
// stay packed (fma.rn.f32.bf16, ds rounded to bf16 for dq).
template <typename T, int EPL>
__device__ __forceinline__ void q_grad_range(const int32_t *col_idx, const T *KV, int D, int lane, bool act,
                                             int lph, float inv_sqrt_r, const float (&q)[EPL],
                                             const float (&dl)[EPL], float ls, float dd, int32_t a, int32_t b,
                                             float (&dq)[EPL]) {
    if constexpr (sizeof(T) == 2 && EPL % 2 == 0) {
        constexpr int W = EPL / 2;
        uint32_t qw[W], dw[W];
        pack_words<EPL>(q, qw);
        pack_words<EPL>(dl, dw);
        for (int32_t e = a; e < b; e += kEU) {
            uint32_t k[kEU][W], v[kEU][W];
#pragma unroll
            for (int u = 0; u < kEU; ++u) {
                const bool live = e + u < b;
                const T *row = KV + (live ? static_cast<int64_t>(col_idx[e + u]) : 0) * 2 * D;
                ld_words<EPL>(row, lane, act && live, k[u]);
                ld_words<EPL>(row + D, lane, act && live, v[u]);
            }
#pragma unroll
            for (int u = 0; u < kEU; ++u) {
                float s = dot_bf16w<W>(qw, k[u], 0.f), dp = dot_bf16w<W>(dw, v[u], 0.f);
                s = head_reduce(s, lph);
                dp = head_reduce(dp, lph);
                const float ds = e + u < b ? __expf(s * inv_sqrt_r - ls) * (dp - dd) * inv_sqrt_r : 0.f;
                axpy_bf16w<W>(bf16_splat(ds), k[u], dq);
            }
        }
    } else {
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
}

// Light target rows of the forward CSR (one warp each, the `rows` list): the local part
// of dq_i added into dZ [:, 0:D].  lse holds the softmax's log-sum-exp per row and head
// (written by the forward's local kernel), Dd holds D_i = dL_i . L_i (the readout's).
template <typename T, int EPL>
__global__ void __launch_bounds__(256) bwd_local_q_kernel(
    const int32_t *__restrict__ rows, int64_t n_rows, const int32_t *__restrict__ row_ptr,
    const int32_t *__restrict__ col_idx, const T *__restrict__ Q, const T *__restrict__ KV,
    const T *__restrict__ dL, int H, int R, float inv_sqrt_r, const float *__restrict__ lse,
    const float *__restrict__ Dd, float *__restrict__ dZ, int64_t dz_ld) {
    const int lane = threadIdx.x & 31;
    const int64_t slot = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (slot >= n_rows) return;                           // warp-uniform
    const int64_t i = rows[slot];
    const int D = H * R;
    const LaneHead lh(lane, EPL, D, R);
    const int32_t r0 = row_ptr[i], r1 = row_ptr[i + 1];
    if (r0 == r1) return;                                 // no local term
    float q[EPL], dl[EPL];
    ld_row<T, EPL>(Q + i * D, lane, lh.act, q);
    ld_row<T, EPL>(dL + i * D, lane, lh.act, dl);
    const float ls = __ldg(lse + i * H + lh.h), dd = __ldg(Dd + i * H + lh.h);
    float dq[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) dq[x] = 0.f;
    q_grad_range<T, EPL>(col_idx, KV, D, lane, lh.act, lh.lph, inv_sqrt_r, q, dl, ls, dd, r0, r1, dq);
    if (lh.act) {
        float *o = dZ + i * dz_ld + lane * EPL;
        float cur[EPL];
        ld_mrow<EPL, false>(o, cur);
#pragma unroll
        for (int x = 0; x < EPL; ++x) cur[x] += dq[x];
        st_mrow<EPL>(o, cur);
    }
}

// bf16 rows with 4 features per lane (8 per half-lane: one 16-byte slice) take
// bwd_q_pair_kernel, with a shared-memory ring of cp.async gathers.
template <typename T, int EPL>
constexpr bool kQRing = sizeof(T) == 2 && EPL == 4;
constexpr size_t kQRingBytes = 8 * 2 * 2 * 2 * 32 * 16;   // 8 warps x 2 steps x kU x (k, v) x 32 lanes

// Light target rows with two edges per step (the layout of bwd_local_kv2_kernel): the
// warp's 16-lane halves take alternate edges of the row, lane hl of a half holding the
// EPL2 = 2 EPL features hl*EPL2 .. hl*EPL2+EPL2-1 of q_i, dL_i and of the gathered k_j,
// v_j, so a step's two edges share one shuffle butterfly and one exponential per lane.
// The halves' dq are added (the same sum in both) and the lower half's lanes add their
// EPL2-feature slices into dZ [:, 0:D] (or dZb).  Needs 2 EPL <= r.
// With CH the warps take the chunks of heavy rows instead (chunk w = {row, first entry},
// kChunk entries at most) and write their shares of dq_i to part[w][0:D].
template <typename T, int EPL, bool CH = false>
__global__ void __launch_bounds__(256, 3) bwd_local_q2_kernel(
    const int32_t *__restrict__ rows, int64_t n_rows, const int32_t *__restrict__ row_ptr,
    const int32_t *__restrict__ col_idx, const T *__restrict__ Q, const T *__restrict__ KV,
    const T *__restrict__ dL, int H, int R, float inv_sqrt_r, const float *__restrict__ lse,
    const float *__restrict__ Dd, float *__restrict__ dZ, int64_t dz_ld, __nv_bfloat16 *__restrict__ dZb,
    const int2 *__restrict__ chunks, float *__restrict__ part) {
    constexpr int EPL2 = 2 * EPL, kU = 2;             // kU edges per slot per step
    const int lane = threadIdx.x & 31, slot = lane >> 4, hl = lane & 15;
    const int64_t w = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (w >= n_rows) return;                              // warp-uniform
    int64_t i;
    int32_t a, b;
    if constexpr (CH) {
        const int2 ch = chunks[w];
        i = ch.x;
        a = ch.y;
        b = min(row_ptr[i + 1], ch.y + kChunk);
    } else {
        i = rows[w];
        a = row_ptr[i];
        b = row_ptr[i + 1];
    }
    const int D = H * R;
    if (!CH && a == b) return;                            // no local term (dq_i = its global part)
    const bool act2 = hl * EPL2 < D;
    const int lph2 = R / EPL2, h2 = act2 ? hl * EPL2 / R : 0;
    float q2[EPL2], dl2[EPL2], dq2[EPL2];
    ld_row<T, EPL2>(Q + i * D, hl, act2, q2);
    ld_row<T, EPL2>(dL + i * D, hl, act2, dl2);
    const float ls = __ldg(lse + i * H + h2), dd = __ldg(Dd + i * H + h2);
#pragma unroll
    for (int x = 0; x < EPL2; ++x) dq2[x] = 0.f;
    // the edges of step it (kU per half)
    auto use_step = [&](int32_t e0, const float (&k)[kU][EPL2], const float (&v)[kU][EPL2]) {
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            float sc = 0.f, dp = 0.f;
#pragma unroll
            for (int x = 0; x < EPL2; ++x) {
                sc = fmaf(q2[x], k[u][x], sc);
                dp = fmaf(dl2[x], v[u][x], dp);
            }
            sc = head_reduce(sc, lph2);
            dp = head_reduce(dp, lph2);
            const bool live = e0 + 2 * u + slot < b;
            const float ds = live ? __expf(sc * inv_sqrt_r - ls) * (dp - dd) * inv_sqrt_r : 0.f;
#pragma unroll
            for (int x = 0; x < EPL2; ++x) dq2[x] = fmaf(ds, k[u][x], dq2[x]);
        }
    };
    for (int32_t e0 = a; e0 < b; e0 += 2 * kU) {          // the same trip count in both halves
        float k[kU][EPL2], v[kU][EPL2];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int32_t e = e0 + 2 * u + slot;
            const bool live = e < b;
            const T *row = KV + (live ? static_cast<int64_t>(col_idx[e]) : 0) * 2 * D;
            ld_row<T, EPL2>(row, hl, act2 && live, k[u]);
            ld_row<T, EPL2>(row + D, hl, act2 && live, v[u]);
        }
        use_step(e0, k, v);
    }
#pragma unroll
    for (int x = 0; x < EPL2; ++x) dq2[x] += __shfl_xor_sync(0xffffffffu, dq2[x], 16);
    // the lower half's lanes hold the row's features hl*EPL2 .. hl*EPL2 + EPL2 - 1
    if (slot != 0 || !act2) return;
    if constexpr (CH) {
        st_mrow<EPL2>(part + w * D + hl * EPL2, dq2);
        return;
    }
    {                                                     // the global part + the local one
        float *o = dZ + i * dz_ld + hl * EPL2;
        __nv_bfloat16 *ob = dZb + i * 3 * D + hl * EPL2;
        float cur[EPL2];
        if (dZb) ld_bf16_slice<EPL2>(ob, cur);
        else ld_mrow<EPL2, false>(o, cur);
#pragma unroll
        for (int x = 0; x < EPL2; ++x) cur[x] += dq2[x];
        if (dZb) st_row<__nv_bfloat16, EPL2>(ob, cur);
        else st_mrow<EPL2>(o, cur);
    }
}

// Light target rows (or, with CH, chunks of heavy rows: chunk = {row, first entry},
// kChunk entries at most) of bf16 layers with 8 features per half-lane (EPL = 4), one
// row per 16-lane half: lane hl of a half holds features hl*8 .. hl*8+7 of its row's q_i
// and dL_i and of the gathered k_j, v_j (through a two-step cp.async ring per warp), kU
// edges of its own row per step; the warp steps as long as
// its longer row (rows come sorted by degree, so the two are alike).  No combine across
// the halves: each writes its row's dq_i (or, with CH, its chunk's share to part) and,
// with pds, each edge's (p, ds) at its transposed position.
template <bool CH>
__global__ void __launch_bounds__(256, 4) bwd_q_pair_kernel(
    const int32_t *__restrict__ rows, int64_t n_items, const int32_t *__restrict__ row_ptr,
    const int32_t *__restrict__ col_idx, const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ KV,
    const __nv_bfloat16 *__restrict__ dL, int H, int R, float inv_sqrt_r, const float *__restrict__ lse,
    const float *__restrict__ Dd, float *__restrict__ dZ, int64_t dz_ld, __nv_bfloat16 *__restrict__ dZb,
    const int2 *__restrict__ chunks, float *__restrict__ part, const int32_t *__restrict__ perm,
    uint32_t *__restrict__ pds) {
    constexpr int EPL2 = 8, kU = 2;
    const int lane = threadIdx.x & 31, slot = lane >> 4, hl = lane & 15;
    const int64_t w = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (2 * w >= n_items) return;                         // warp-uniform
    const int64_t item = 2 * w + slot;
    const bool have = item < n_items;
    int64_t i = 0;
    int32_t a = 0, b = 0;
    if (have) {
        if constexpr (CH) {
            const int2 ch = chunks[item];
            i = ch.x;
            a = ch.y;
            b = min(row_ptr[i + 1], ch.y + kChunk);
        } else {
            i = rows[item];
            a = row_ptr[i];
            b = row_ptr[i + 1];
        }
    }
    const int D = H * R;
    const bool act2 = have && hl * EPL2 < D;
    const int lph2 = R / EPL2, h2 = hl * EPL2 < D ? hl * EPL2 / R : 0;
    uint32_t qw[4] = {0u, 0u, 0u, 0u}, dw[4] = {0u, 0u, 0u, 0u};
    if (act2) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(Q + i * D + hl * EPL2));
        const uint4 y = __ldg(reinterpret_cast<const uint4 *>(dL + i * D + hl * EPL2));
        qw[0] = x.x; qw[1] = x.y; qw[2] = x.z; qw[3] = x.w;
        dw[0] = y.x; dw[1] = y.y; dw[2] = y.z; dw[3] = y.w;
    }
    const float ls = have ? __ldg(lse + i * H + h2) : 0.f, dd = have ? __ldg(Dd + i * H + h2) : 0.f;
    // p = 2^(sc log2(e) / sqrt(r) - lse log2(e)), ds = p (dp / sqrt(r) - D_i / sqrt(r))
    const float sc2 = inv_sqrt_r * 1.4426950408889634f, ls2 = ls * 1.4426950408889634f, dd_s = dd * inv_sqrt_r;
    float dq2[EPL2];
#pragma unroll
    for (int x = 0; x < EPL2; ++x) dq2[x] = 0.f;
    // never-written cells (edges past the row's end) are read with ds = 0: keep them finite
    extern __shared__ uint4 q_ring[];
    uint4 *ring = q_ring + (threadIdx.x >> 5) * (2 * kU * 2 * 32) + lane;
    auto cell = [&](int st, int u, int kv) { return ring + ((st * kU + u) * 2 + kv) * 32; };
#pragma unroll
    for (int c = 0; c < 2 * kU * 2; ++c) ring[c * 32] = make_uint4(0u, 0u, 0u, 0u);
    auto issue = [&](int32_t e0, int st, int32_t (&pe)[kU]) {
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int32_t e = e0 + u;
            if (e < b && act2) {
                const __nv_bfloat16 *row = KV + static_cast<int64_t>(col_idx[e]) * 2 * D + hl * EPL2;
                cp_async16(cell(st, u, 0), row);
                cp_async16(cell(st, u, 1), row + D);
            }
            pe[u] = (pds && e < b) ? __ldg(perm + e) : 0;
        }
        cp_async_commit();
    };
    const int mine = (b - a + kU - 1) / kU;
    const int n_steps = max(mine, __shfl_xor_sync(0xffffffffu, mine, 16));
    const bool head_lead = act2 && (hl & (lph2 - 1)) == 0;   // one lane per head writes (p, ds)
    int32_t pc[kU], pn[kU];
    issue(a, 0, pc);
    for (int it = 0; it < n_steps; ++it) {
        const int32_t e0 = a + it * kU;
        if (it + 1 < n_steps) {
            issue(e0 + kU, (it + 1) & 1, pn);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const uint4 kv4 = *cell(it & 1, u, 0), vv4 = *cell(it & 1, u, 1);
            const uint32_t kk[4] = {kv4.x, kv4.y, kv4.z, kv4.w}, vv[4] = {vv4.x, vv4.y, vv4.z, vv4.w};
            float sc = dot_bf16w<4>(qw, kk, 0.f), dp = dot_bf16w<4>(dw, vv, 0.f);
            sc = head_reduce(sc, lph2);
            dp = head_reduce(dp, lph2);
            const bool live = e0 + u < b;
            const float p = ex2_approx(fmaf(sc, sc2, -ls2));
            const float ds = live ? p * fmaf(dp, inv_sqrt_r, -dd_s) : 0.f;
            axpy_bf16w<4>(bf16_splat(ds), kk, dq2);
            if (pds && live && head_lead) pds[static_cast<int64_t>(pc[u]) * H + h2] = pack_p_ds(p, ds);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) pc[u] = pn[u];
    }
    if (!act2) return;
    if constexpr (CH) {
        st_mrow<EPL2>(part + item * D + hl * EPL2, dq2);
    } else {
        if (a == b) return;                               // no local term (dq_i = its global part)
        float *o = dZ + i * dz_ld + hl * EPL2;
        __nv_bfloat16 *ob = dZb + i * 3 * D + hl * EPL2;
        float cur[EPL2];
        if (dZb) ld_bf16_slice<EPL2>(ob, cur);
        else ld_mrow<EPL2, false>(o, cur);
#pragma unroll
        for (int x = 0; x < EPL2; ++x) cur[x] += dq2[x];
        if (dZb) st_row<__nv_bfloat16, EPL2>(ob, cur);
        else st_mrow<EPL2>(o, cur);
    }
}

// Chunks of heavy target rows, one warp each: chunk c covers the edges
// [chunks[c].y, min(chunks[c].y + kChunk, row end)) of row chunks[c].x, and writes its
// share of dq_i into part[c][0:D].
template <typename T, int EPL>
__global__ void __launch_bounds__(256) bwd_q_chunk_kernel(
    const int2 *__restrict__ chunks, int64_t n_chunks, const int32_t *__restrict__ row_ptr,
    const int32_t *__restrict__ col_idx, const T *__restrict__ Q, const T *__restrict__ KV,
    const T *__restrict__ dL, int H, int R, float inv_sqrt_r, const float *__restrict__ lse,
    const float *__restrict__ Dd, float *__restrict__ part) {
    const int lane = threadIdx.x & 31;
    const int64_t c = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (c >= n_chunks) return;                            // warp-uniform
    const int2 ch = chunks[c];
    const int64_t i = ch.x;
    const int32_t a = ch.y, b = min(row_ptr[i + 1], ch.y + kChunk);
    const int D = H * R;
    const LaneHead lh(lane, EPL, D, R);
    float q[EPL], dl[EPL], dq[EPL];
    ld_row<T, EPL>(Q + i * D, lane, lh.act, q);
    ld_row<T, EPL>(dL + i * D, lane, lh.act, dl);
#pragma unroll
    for (int x = 0; x < EPL; ++x) dq[x] = 0.f;
    const float ls = __ldg(lse + i * H + lh.h), dd = __ldg(Dd + i * H + lh.h);
    q_grad_range<T, EPL>(col_idx, KV, D, lane, lh.act, lh.lph, inv_sqrt_r, q, dl, ls, dd, a, b, dq);
    if (lh.act) st_mrow<EPL>(part + c * D + lane * EPL, dq);
}

// Heavy rows are merged by one block of kMW warps each: warp w takes the row's chunks
// c0 + w, c0 + w + kMW, ... (in order, kMU loads in flight), and warp 0 then combines the
// warps' results in warp order through shared memory, so the order is fixed.
constexpr int kMW = 8, kMU = 8;

// Heavy target rows over their chunks [chunk_ptr[s], chunk_ptr[s + 1]): dq_i = the
// chunks' shares summed, added into dZ [:, 0:D].  Dynamic shared memory: kMW * D floats.
template <int EPL>
__global__ void __launch_bounds__(kMW * 32) bwd_q_heavy_kernel(
    const int32_t *__restrict__ rows, int64_t n_rows, const int32_t *__restrict__ chunk_ptr,
    const float *__restrict__ part, int H, int R, float *__restrict__ dZ, int64_t dz_ld,
    __nv_bfloat16 *__restrict__ dZb) {
    extern __shared__ float msm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t slot = blockIdx.x;
    if (slot >= n_rows) return;                           // block-uniform
    const int64_t i = rows[slot];
    const int D = H * R;
    const LaneHead lh(lane, EPL, D, R);
    const int32_t c0 = chunk_ptr[slot], c1 = chunk_ptr[slot + 1];
    float dq[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) dq[x] = 0.f;
    if (lh.act) {
        for (int32_t c = c0 + warp; c < c1; c += kMU * kMW) {
            float pv[kMU][EPL];
#pragma unroll
            for (int u = 0; u < kMU; ++u) {
                const int32_t cc = c + u * kMW;
                if (cc < c1) {
                    ld_mrow<EPL>(part + static_cast<int64_t>(cc) * D + lane * EPL, pv[u]);
                } else {
#pragma unroll
                    for (int x = 0; x < EPL; ++x) pv[u][x] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kMU; ++u)
#pragma unroll
                for (int x = 0; x < EPL; ++x) dq[x] += pv[u][x];
        }
        st_mrow<EPL>(msm + warp * D + lane * EPL, dq);
    }
    __syncthreads();
    if (warp != 0 || !lh.act) return;
    float acc[EPL], pv[EPL];
    float *o = dZ + i * dz_ld + lane * EPL;
    if (dZb) ld_bf16_slice<EPL>(dZb + i * 3 * D + lane * EPL, acc);   // the global part of dq_i
    else ld_mrow<EPL, false>(o, acc);
#pragma unroll
    for (int x = 0; x < EPL; ++x) dq[x] = 0.f;
    for (int w = 0; w < kMW; ++w) {
        ld_mrow<EPL, false>(msm + w * D + lane * EPL, pv);
#pragma unroll
        for (int x = 0; x < EPL; ++x) dq[x] += pv[x];
    }
#pragma unroll
    for (int x = 0; x < EPL; ++x) acc[x] += dq[x];
    if (dZb) st_row<__nv_bfloat16, EPL>(dZb + i * 3 * D + lane * EPL, acc);
    else st_mrow<EPL>(o, acc);
}

// dk, dv += the terms of targets [a, b) of source row j (this warp's lanes).
template <typename T, int EPL>
__device__ __forceinline__ void kv_grad_range(const int32_t *t_col, const T *Q, const T *dL,
                                              const float *lse, const float *Dd, int H, int D, int lane,
                                              bool act, int lph, int h, float inv_sqrt_r, const float (&k)[EPL],
                                              const float (&v)[EPL], int32_t a, int32_t b, float (&dk)[EPL],
                                              float (&dv)[EPL]) {
    if constexpr (sizeof(T) == 2 && EPL % 2 == 0) {
        // bf16 rows stay packed (fma.rn.f32.bf16; p and ds rounded to bf16 for dv and dk)
        constexpr int W = EPL / 2;
        uint32_t kw[W], vw[W];
        pack_words<EPL>(k, kw);
        pack_words<EPL>(v, vw);
        for (int32_t e = a; e < b; e += kEU) {
            uint32_t q[kEU][W], dl[kEU][W];
            float ls[kEU], dd[kEU];
#pragma unroll
            for (int u = 0; u < kEU; ++u) {
                const bool live = e + u < b;
                const int64_t i = live ? t_col[e + u] : 0;
                ld_words<EPL>(Q + i * D, lane, act && live, q[u]);
                ld_words<EPL>(dL + i * D, lane, act && live, dl[u]);
                ls[u] = live ? __ldg(lse + i * H + h) : 0.f;
                dd[u] = live ? __ldg(Dd + i * H + h) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kEU; ++u) {
                float s = dot_bf16w<W>(q[u], kw, 0.f), dp = dot_bf16w<W>(dl[u], vw, 0.f);
                s = head_reduce(s, lph);
                dp = head_reduce(dp, lph);
                const bool live = e + u < b;
                const float p = live ? __expf(s * inv_sqrt_r - ls[u]) : 0.f;
                const float ds = p * (dp - dd[u]) * inv_sqrt_r;
                axpy_bf16w<W>(bf16_splat(p), dl[u], dv);
                axpy_bf16w<W>(bf16_splat(ds), q[u], dk);
            }
        }
    } else {
        for (int32_t e = a; e < b; e += kEU) {
            float q[kEU][EPL], dl[kEU][EPL], ls[kEU], dd[kEU];
#pragma unroll
            for (int u = 0; u < kEU; ++u) {
                const bool live = e + u < b;
                const int64_t i = live ? t_col[e + u] : 0;
                ld_row<T, EPL>(Q + i * D, lane, act && live, q[u]);
                ld_row<T, EPL>(dL + i * D, lane, act && live, dl[u]);
                ls[u] = live ? __ldg(lse + i * H + h) : 0.f;
                dd[u] = live ? __ldg(Dd + i * H + h) : 0.f;
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
}

// The global terms of source row j and the store, in the 32-lane layout (every lane of
// the warp takes part in the shuffles):
//   dphi(k_j)_f = sum_c dS[f][c] v_c + dz_f,  dv_j,f += sum_c dS[c][f] phi(k_c)
// (S = sum phi(k) v^T, z = sum phi(k)); dk, dv hold the local terms on entry.  With GTC
// the global terms are already in dZ (bwd_kv_global_tc_kernel) and the local terms are
// added to them.
template <int EPL, bool GTC>
__device__ __forceinline__ void kv_finish(const LaneHead &lh, int lane, int64_t j, const float (&k)[EPL],
                                          const float (&v)[EPL], float (&dk)[EPL], float (&dv)[EPL],
                                          const float *dSc, const float *dST, int H, int R, float *dZ,
                                          int64_t dz_ld, __nv_bfloat16 *dZb) {
    const int D = H * R;
    if constexpr (GTC) {
        if (lh.act) {
            float *pk = dZ + j * dz_ld + D + lane * EPL, *pv = pk + D;
            float gk[EPL], gv[EPL];
            if (dZb) {
                ld_bf16_slice<EPL>(dZb + j * 3 * D + D + lane * EPL, gk);
                ld_bf16_slice<EPL>(dZb + j * 3 * D + 2 * D + lane * EPL, gv);
            } else {
                ld_mrow<EPL, false>(pk, gk);
                ld_mrow<EPL, false>(pv, gv);
            }
#pragma unroll
            for (int x = 0; x < EPL; ++x) {
                dk[x] += gk[x];
                dv[x] += gv[x];
            }
            if (dZb) {                                    // the final values in bf16
                st_row<__nv_bfloat16, EPL>(dZb + j * 3 * D + D + lane * EPL, dk);
                st_row<__nv_bfloat16, EPL>(dZb + j * 3 * D + 2 * D + lane * EPL, dv);
            } else {
                st_mrow<EPL>(pk, dk);
                st_mrow<EPL>(pv, dv);
            }
        }
        return;
    } else {
    float dphk[EPL], dvg[EPL], pk[EPL];
    ld_mrow<EPL>(dSc + static_cast<int64_t>(H) * R * R + lh.h * R + lh.f0, dphk);
#pragma unroll
    for (int x = 0; x < EPL; ++x) {
        dvg[x] = 0.f;
        pk[x] = phi(k[x]);
    }
    head_matvec<EPL>(dST + static_cast<int64_t>(lh.h) * R * R, R, lh.f0, lh.hb, lh.lph, v, dphk);
    head_matvec<EPL>(dSc + static_cast<int64_t>(lh.h) * R * R, R, lh.f0, lh.hb, lh.lph, pk, dvg);
    if (lh.act) {
#pragma unroll
        for (int x = 0; x < EPL; ++x) {
            dk[x] = fmaf(dphk[x], dphi(k[x]), dk[x]);
            dv[x] += dvg[x];
        }
        st_mrow<EPL>(dZ + j * dz_ld + D + lane * EPL, dk);
        st_mrow<EPL>(dZ + j * dz_ld + 2 * D + lane * EPL, dv);
    }
    }
}

// Source rows of the transposed CSR (the targets i of j): the local terms of dk_j and
// dv_j, plus the global terms through phi(k_j), written to dZ [:, D:2D] and [:, 2D:3D].
// Light rows (PARTS false, one warp each) walk their edges; heavy rows (PARTS true, one
// block of kMW warps each) sum their chunks' shares part[c][0:D] | part[c][D:2D], c in
// [chunk_ptr[s], chunk_ptr[s + 1]), warp-strided and then in warp order.  dSc holds dS [H][R][R] then dz [H][R]; dST is dS transposed per head.
template <typename T, int EPL, bool PARTS, bool GTC = false>
__global__ void __launch_bounds__(PARTS ? kMW * 32 : 256) bwd_local_kv_kernel(
    const int32_t *__restrict__ rows, int64_t n_rows, const int32_t *__restrict__ t_row_ptr,
    const int32_t *__restrict__ t_col, const int32_t *__restrict__ chunk_ptr, const float *__restrict__ part,
    const T *__restrict__ Q, const T *__restrict__ KV, const T *__restrict__ dL,
    const float *__restrict__ lse, const float *__restrict__ Dd, const float *__restrict__ dSc,
    const float *__restrict__ dST, int H, int R, float inv_sqrt_r, float *__restrict__ dZ, int64_t dz_ld,
    __nv_bfloat16 *__restrict__ dZb) {
    extern __shared__ float msm[];                       // PARTS: [kMW][2D]
    const int lane = threadIdx.x & 31;
    const int64_t slot = PARTS ? blockIdx.x : (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (slot >= n_rows) return;                           // warp-uniform (block-uniform with PARTS)
    const int64_t j = rows[slot];
    const int D = H * R;
    const LaneHead lh(lane, EPL, D, R);
    const T *krow = KV + j * 2 * D;
    float k[EPL], v[EPL], dk[EPL], dv[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) dk[x] = dv[x] = 0.f;
    if constexpr (PARTS) {
        const int warp = threadIdx.x >> 5;
        const int32_t c0 = chunk_ptr[slot], c1 = chunk_ptr[slot + 1];
        if (lh.act) {
            for (int32_t c = c0 + warp; c < c1; c += kMU * kMW) {
                float pk[kMU][EPL], pv[kMU][EPL];
#pragma unroll
                for (int u = 0; u < kMU; ++u) {
                    const int32_t cc = c + u * kMW;
                    if (cc < c1) {
                        const float *pc = part + static_cast<int64_t>(cc) * 2 * D + lane * EPL;
                        ld_mrow<EPL>(pc, pk[u]);
                        ld_mrow<EPL>(pc + D, pv[u]);
                    } else {
#pragma unroll
                        for (int x = 0; x < EPL; ++x) pk[u][x] = pv[u][x] = 0.f;
                    }
                }
#pragma unroll
                for (int u = 0; u < kMU; ++u)
#pragma unroll
                    for (int x = 0; x < EPL; ++x) {
                        dk[x] += pk[u][x];
                        dv[x] += pv[u][x];
                    }
            }
            st_mrow<EPL>(msm + warp * 2 * D + lane * EPL, dk);
            st_mrow<EPL>(msm + warp * 2 * D + D + lane * EPL, dv);
        }
        __syncthreads();
        if (warp != 0) return;
        if (lh.act) {
#pragma unroll
            for (int x = 0; x < EPL; ++x) dk[x] = dv[x] = 0.f;
            for (int w = 0; w < kMW; ++w) {
                float pk[EPL], pv[EPL];
                ld_mrow<EPL, false>(msm + w * 2 * D + lane * EPL, pk);
                ld_mrow<EPL, false>(msm + w * 2 * D + D + lane * EPL, pv);
#pragma unroll
                for (int x = 0; x < EPL; ++x) {
                    dk[x] += pk[x];
                    dv[x] += pv[x];
                }
            }
        }
    }
    ld_row<T, EPL>(krow, lane, lh.act, k);
    ld_row<T, EPL>(krow + D, lane, lh.act, v);
    if constexpr (!PARTS) {
        kv_grad_range<T, EPL>(t_col, Q, dL, lse, Dd, H, D, lane, lh.act, lh.lph, lh.h, inv_sqrt_r, k, v,
                              t_row_ptr[j], t_row_ptr[j + 1], dk, dv);
    }
    kv_finish<EPL, GTC>(lh, lane, j, k, v, dk, dv, dSc, dST, H, R, dZ, dz_ld, dZb);
}

// Light source rows with two edges per step: the warp's halves (slots) take alternate
// edges of the row, lane hl = lane % 16 of a half holding the EPL2 = 2 EPL features
// hl*EPL2 .. hl*EPL2+EPL2-1 (a head's r features in r/EPL2 lanes of the half), so the two
// edges of a step share one shuffle butterfly and one exponential per lane.  The halves'
// dk, dv are then added (lower + upper, the same sum in both) and moved to the 32-lane
// layout for kv_finish.  Needs 2 EPL <= r.
// With CH the warps take the chunks of heavy rows instead (chunk w = {row, first entry},
// kChunk entries at most) and write their shares of dk_j | dv_j to part[w][0:2D].
// With the target side's stored (p, ds), bwd_kv_pair_kernel takes these rows instead
// (kPdsEdges edges per half-warp step, gathers through a two-step shared-memory ring).
constexpr int kPdsEdges = 2;
constexpr size_t kKvRingBytes = 8 * 2 * kPdsEdges * 2 * 32 * 16;   // 8 warps x 2 steps x edges x (q, dL) x 32 lanes
template <typename T, int EPL, bool GTC = false, bool CH = false>
__global__ void __launch_bounds__(256, 4) bwd_local_kv2_kernel(
    const int32_t *__restrict__ rows, int64_t n_rows, const int32_t *__restrict__ t_row_ptr,
    const int32_t *__restrict__ t_col, const T *__restrict__ Q, const T *__restrict__ KV,
    const T *__restrict__ dL, const float *__restrict__ lse, const float *__restrict__ Dd,
    const float *__restrict__ dSc, const float *__restrict__ dST, int H, int R, float inv_sqrt_r,
    float *__restrict__ dZ, int64_t dz_ld, __nv_bfloat16 *__restrict__ dZb, const int2 *__restrict__ chunks,
    float *__restrict__ part) {
    constexpr int EPL2 = 2 * EPL, kU = 2;             // kU edges per slot per step
    const int lane = threadIdx.x & 31, slot = lane >> 4, hl = lane & 15;
    const int64_t w = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (w >= n_rows) return;                              // warp-uniform
    const int64_t j = CH ? static_cast<int64_t>(chunks[w].x) : static_cast<int64_t>(rows[w]);
    const int D = H * R;
    const bool act2 = hl * EPL2 < D;
    const int lph2 = R / EPL2, h2 = act2 ? hl * EPL2 / R : 0;
    const T *krow = KV + j * 2 * D;
    float k2[EPL2], v2[EPL2], dk2[EPL2], dv2[EPL2];
    ld_row<T, EPL2>(krow, hl, act2, k2);
    ld_row<T, EPL2>(krow + D, hl, act2, v2);
#pragma unroll
    for (int x = 0; x < EPL2; ++x) dk2[x] = dv2[x] = 0.f;
    const int32_t a = CH ? chunks[w].y : t_row_ptr[j];
    const int32_t b = CH ? min(t_row_ptr[j + 1], chunks[w].y + kChunk) : t_row_ptr[j + 1];
    auto use_step = [&](int32_t e0, const float (&q)[kU][EPL2], const float (&dl)[kU][EPL2], const float (&ls)[kU],
                        const float (&dd)[kU]) {
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            float sc = 0.f, dp = 0.f;
#pragma unroll
            for (int x = 0; x < EPL2; ++x) {
                sc = fmaf(q[u][x], k2[x], sc);
                dp = fmaf(dl[u][x], v2[x], dp);
            }
            sc = head_reduce(sc, lph2);
            dp = head_reduce(dp, lph2);
            const bool live = e0 + 2 * u + slot < b;
            const float p = live ? __expf(sc * inv_sqrt_r - ls[u]) : 0.f;
            const float ds = p * (dp - dd[u]) * inv_sqrt_r;
#pragma unroll
            for (int x = 0; x < EPL2; ++x) {
                dv2[x] = fmaf(p, dl[u][x], dv2[x]);
                dk2[x] = fmaf(ds, q[u][x], dk2[x]);
            }
        }
    };
    if constexpr (sizeof(T) == 2 && EPL2 == 8) {
        // k_j, v_j and the gathered q_i, dL_i stay packed: the dot products, dv and dk run on
        // fma.rn.f32.bf16 (p and ds rounded to bf16 for dv and dk)
        uint32_t kw[4] = {0u, 0u, 0u, 0u}, vw[4] = {0u, 0u, 0u, 0u};
        if (act2) {
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(krow + hl * EPL2));
            const uint4 y = __ldg(reinterpret_cast<const uint4 *>(krow + D + hl * EPL2));
            kw[0] = x.x; kw[1] = x.y; kw[2] = x.z; kw[3] = x.w;
            vw[0] = y.x; vw[1] = y.y; vw[2] = y.z; vw[3] = y.w;
        }
        for (int32_t e0 = a; e0 < b; e0 += 2 * kU) {  // the same trip count in both halves
            uint4 q4[kU], d4[kU];
            float ls[kU], dd[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int32_t e = e0 + 2 * u + slot;
                const bool live = e < b;
                const int64_t i = live ? t_col[e] : 0;
                q4[u] = d4[u] = make_uint4(0u, 0u, 0u, 0u);
                if (act2 && live) {
                    q4[u] = __ldg(reinterpret_cast<const uint4 *>(Q + i * D + hl * EPL2));
                    d4[u] = __ldg(reinterpret_cast<const uint4 *>(dL + i * D + hl * EPL2));
                }
                ls[u] = live ? __ldg(lse + i * H + h2) : 0.f;
                dd[u] = live ? __ldg(Dd + i * H + h2) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const uint32_t qq[4] = {q4[u].x, q4[u].y, q4[u].z, q4[u].w};
                const uint32_t ll[4] = {d4[u].x, d4[u].y, d4[u].z, d4[u].w};
                float sc = dot_bf16w<4>(qq, kw, 0.f), dp = dot_bf16w<4>(ll, vw, 0.f);
                sc = head_reduce(sc, lph2);
                dp = head_reduce(dp, lph2);
                const bool live = e0 + 2 * u + slot < b;
                const float p = live ? __expf(sc * inv_sqrt_r - ls[u]) : 0.f;
                const float ds = p * (dp - dd[u]) * inv_sqrt_r;
                axpy_bf16w<4>(bf16_splat(p), ll, dv2);
                axpy_bf16w<4>(bf16_splat(ds), qq, dk2);
            }
        }
    } else {
        for (int32_t e0 = a; e0 < b; e0 += 2 * kU) {  // the same trip count in both halves
            float q[kU][EPL2], dl[kU][EPL2], ls[kU], dd[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int32_t e = e0 + 2 * u + slot;
                const bool live = e < b;
                const int64_t i = live ? t_col[e] : 0;
                ld_row<T, EPL2>(Q + i * D, hl, act2 && live, q[u]);
                ld_row<T, EPL2>(dL + i * D, hl, act2 && live, dl[u]);
                ls[u] = live ? __ldg(lse + i * H + h2) : 0.f;
                dd[u] = live ? __ldg(Dd + i * H + h2) : 0.f;
            }
            use_step(e0, q, dl, ls, dd);
        }
    }
#pragma unroll
    for (int x = 0; x < EPL2; ++x) {
        dk2[x] += __shfl_xor_sync(0xffffffffu, dk2[x], 16);
        dv2[x] += __shfl_xor_sync(0xffffffffu, dv2[x], 16);
    }
    if constexpr (CH) {                                   // the chunk's share, 8-feature slices
        if (slot == 0 && act2) {
            st_mrow<EPL2>(part + w * 2 * D + hl * EPL2, dk2);
            st_mrow<EPL2>(part + w * 2 * D + D + hl * EPL2, dv2);
        }
        return;
    }
    if constexpr (GTC) {
        // the global terms are in dZ already: the lower half adds its 8-feature slices
        if (slot == 0 && act2) {
            float *pk = dZ + j * dz_ld + D + hl * EPL2, *pv = pk + D;
            float gk[EPL2], gv[EPL2];
            if (dZb) {
                ld_bf16_slice<EPL2>(dZb + j * 3 * D + D + hl * EPL2, gk);
                ld_bf16_slice<EPL2>(dZb + j * 3 * D + 2 * D + hl * EPL2, gv);
            } else {
                ld_mrow<EPL2, false>(pk, gk);
                ld_mrow<EPL2, false>(pv, gv);
            }
#pragma unroll
            for (int x = 0; x < EPL2; ++x) {
                dk2[x] += gk[x];
                dv2[x] += gv[x];
            }
            if (dZb) {                                    // the final values in bf16
                st_row<__nv_bfloat16, EPL2>(dZb + j * 3 * D + D + hl * EPL2, dk2);
                st_row<__nv_bfloat16, EPL2>(dZb + j * 3 * D + 2 * D + hl * EPL2, dv2);
            } else {
                st_mrow<EPL2>(pk, dk2);
                st_mrow<EPL2>(pv, dv2);
            }
        }
        return;
    }
    // to the 32-lane layout: lane l's features l*EPL .. are half-lane l/2's, part l % 2
    const LaneHead lh(lane, EPL, D, R);
    const int src = lane >> 1;
    const bool hi = lane & 1;
    float k[EPL], v[EPL], dk[EPL], dv[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) {
        const float k0 = __shfl_sync(0xffffffffu, dk2[x], src), k1 = __shfl_sync(0xffffffffu, dk2[EPL + x], src);
        const float v0 = __shfl_sync(0xffffffffu, dv2[x], src), v1 = __shfl_sync(0xffffffffu, dv2[EPL + x], src);
        dk[x] = hi ? k1 : k0;
        dv[x] = hi ? v1 : v0;
    }
    ld_row<T, EPL>(krow, lane, lh.act, k);
    ld_row<T, EPL>(krow + D, lane, lh.act, v);
    kv_finish<EPL, GTC>(lh, lane, j, k, v, dk, dv, dSc, dST, H, R, dZ, dz_ld, dZb);
}

// The source side with stored (p, ds) (bf16 layers, 8 features per half-lane, global terms
// already in dZ / dZb), one row (or, with CH, one chunk of a heavy row) per 16-lane half:
// lane hl of a half gathers features hl*8 .. hl*8+7 of q_i and dL_i through a two-step
// cp.async ring per warp, kPdsEdges edges of its own row per step, and accumulates
// dv_j += p dL_i, dk_j += ds q_i; the warp steps as long as its longer row.  Each half then
// adds its row's local terms to the global ones in place (or, with CH, writes its chunk's
// share of dk_j | dv_j to part).
template <bool CH>
__global__ void __launch_bounds__(256, 4) bwd_kv_pair_kernel(
    const int32_t *__restrict__ rows, int64_t n_items, const int32_t *__restrict__ t_row_ptr,
    const int32_t *__restrict__ t_col, const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ dL,
    int H, int R, float *__restrict__ dZ, int64_t dz_ld, __nv_bfloat16 *__restrict__ dZb,
    const int2 *__restrict__ chunks, float *__restrict__ part, const uint32_t *__restrict__ pds) {
    constexpr int EPL2 = 8, kP = kPdsEdges;
    const int lane = threadIdx.x & 31, slot = lane >> 4, hl = lane & 15;
    const int64_t w = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (2 * w >= n_items) return;                         // warp-uniform
    const int64_t item = 2 * w + slot;
    const bool have = item < n_items;
    int64_t j = 0;
    int32_t a = 0, b = 0;
    if (have) {
        if constexpr (CH) {
            const int2 ch = chunks[item];
            j = ch.x;
            a = ch.y;
            b = min(t_row_ptr[j + 1], ch.y + kChunk);
        } else {
            j = rows[item];
            a = t_row_ptr[j];
            b = t_row_ptr[j + 1];
        }
    }
    const int D = H * R;
    const bool act2 = have && hl * EPL2 < D;
    const int h2 = hl * EPL2 < D ? hl * EPL2 / R : 0;
    float dk2[EPL2], dv2[EPL2];
#pragma unroll
    for (int x = 0; x < EPL2; ++x) dk2[x] = dv2[x] = 0.f;
    extern __shared__ uint4 kv_ring[];
    uint4 *ring = kv_ring + (threadIdx.x >> 5) * (2 * kP * 2 * 32) + lane;
    auto cell = [&](int st, int u, int which) { return ring + ((st * kP + u) * 2 + which) * 32; };
    // never-written cells are read with p = ds = 0: keep them finite
#pragma unroll
    for (int c = 0; c < 2 * kP * 2; ++c) ring[c * 32] = make_uint4(0u, 0u, 0u, 0u);
    auto issue = [&](int32_t e0, int st, uint32_t (&pw)[kP]) {
#pragma unroll
        for (int u = 0; u < kP; ++u) {
            const int32_t e = e0 + u;
            pw[u] = 0u;
            if (e < b && act2) {
                const int64_t i = t_col[e];
                cp_async16(cell(st, u, 0), Q + i * D + hl * EPL2);
                cp_async16(cell(st, u, 1), dL + i * D + hl * EPL2);
                pw[u] = __ldg(pds + static_cast<int64_t>(e) * H + h2);
            }
        }
        cp_async_commit();
    };
    const int mine = (b - a + kP - 1) / kP;
    const int n_steps = max(mine, __shfl_xor_sync(0xffffffffu, mine, 16));
    uint32_t pc[kP], pn[kP];
    issue(a, 0, pc);
    for (int it = 0; it < n_steps; ++it) {
        const int32_t e0 = a + it * kP;
        if (it + 1 < n_steps) {
            issue(e0 + kP, (it + 1) & 1, pn);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
#pragma unroll
        for (int u = 0; u < kP; ++u) {
            const uint4 q4 = *cell(it & 1, u, 0), d4 = *cell(it & 1, u, 1);
            const uint32_t qq[4] = {q4.x, q4.y, q4.z, q4.w};
            const uint32_t ll[4] = {d4.x, d4.y, d4.z, d4.w};
            axpy_bf16w<4>(pc[u], ll, dv2);
            axpy_bf16w_hi<4>(pc[u], qq, dk2);
        }
#pragma unroll
        for (int u = 0; u < kP; ++u) pc[u] = pn[u];
    }
    if (!act2) return;
    if constexpr (CH) {
        st_mrow<EPL2>(part + item * 2 * D + hl * EPL2, dk2);
        st_mrow<EPL2>(part + item * 2 * D + D + hl * EPL2, dv2);
    } else {
        float gk[EPL2], gv[EPL2];
        if (dZb) {
            __nv_bfloat16 *pk = dZb + j * 3 * D + D + hl * EPL2, *pv = pk + D;
            ld_bf16_slice<EPL2>(pk, gk);
            ld_bf16_slice<EPL2>(pv, gv);
#pragma unroll
            for (int x = 0; x < EPL2; ++x) {
                gk[x] += dk2[x];
                gv[x] += dv2[x];
            }
            st_row<__nv_bfloat16, EPL2>(pk, gk);
            st_row<__nv_bfloat16, EPL2>(pv, gv);
        } else {
            float *pk = dZ + j * dz_ld + D + hl * EPL2, *pv = pk + D;
            ld_mrow<EPL2, false>(pk, gk);
            ld_mrow<EPL2, false>(pv, gv);
#pragma unroll
            for (int x = 0; x < EPL2; ++x) {
                gk[x] += dk2[x];
                gv[x] += dv2[x];
            }
            st_mrow<EPL2>(pk, gk);
            st_mrow<EPL2>(pv, gv);
        }
    }
}

// Chunks of heavy source rows, one warp each (layout as bwd_q_chunk_kernel's, over the
// transposed CSR): the chunk's shares of dk_j | dv_j into part[c][0:D] | part[c][D:2D].
template <typename T, int EPL>
__global__ void __launch_bounds__(256) bwd_kv_chunk_kernel(
    const int2 *__restrict__ chunks, int64_t n_chunks, const int32_t *__restrict__ t_row_ptr,
    const int32_t *__restrict__ t_col, const T *__restrict__ Q, const T *__restrict__ KV,
    const T *__restrict__ dL, const float *__restrict__ lse, const float *__restrict__ Dd, int H, int R,
    float inv_sqrt_r, float *__restrict__ part) {
    const int lane = threadIdx.x & 31;
    const int64_t c = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    if (c >= n_chunks) return;
    const int2 ch = chunks[c];
    const int64_t j = ch.x;
    const int32_t a = ch.y, b = min(t_row_ptr[j + 1], ch.y + kChunk);
    const int D = H * R;
    const LaneHead lh(lane, EPL, D, R);
    float k[EPL], v[EPL], dk[EPL], dv[EPL];
    ld_row<T, EPL>(KV + j * 2 * D, lane, lh.act, k);
    ld_row<T, EPL>(KV + j * 2 * D + D, lane, lh.act, v);
#pragma unroll
    for (int x = 0; x < EPL; ++x) dk[x] = dv[x] = 0.f;
    kv_grad_range<T, EPL>(t_col, Q, dL, lse, Dd, H, D, lane, lh.act, lh.lph, lh.h, inv_sqrt_r, k, v, a, b, dk, dv);
    if (lh.act) {
        float *pc = part + c * 2 * D + lane * EPL;
        st_mrow<EPL>(pc, dk);
        st_mrow<EPL>(pc + D, dv);
    }
}

// dw_g and db_g over row range p = blockIdx.x (rows [p rpp, (p + 1) rpp)), dt = dZ[:, Kc]:
// part[p][a][Kc] = sum_i X[i][a] dt_i for the 32 columns a of blockIdx.y, the block's
// 8 warps taking rows i = r0 + w, r0 + w + 8, ... and their sums added in warp order;
// blocks with blockIdx.y == 0 also sum dt_i over the range (thread-strided, then a
// fixed tree) into dbg_part[p].
template <typename T>
__global__ void __launch_bounds__(256) bwd_dwg_kernel(const T *__restrict__ X, const float *__restrict__ dZ,
                                                      int64_t N, int d, int64_t dz_ld, int Kc, int Dc, int64_t rpp,
                                                      float *__restrict__ part, float *__restrict__ dbg_part) {
    __shared__ float red[256];
    const int t = threadIdx.x, w = t >> 5, col = t & 31;
    const int a = blockIdx.y * 32 + col;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rpp;
    const int64_t r1 = std::min<int64_t>(N, r0 + rpp);
    float acc = 0.f;
    if (a < d) {
        int64_t i = r0 + w;
        for (; i + 24 < r1; i += 32) {
            float xv[4], tv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                xv[u] = ldf<T>(X + (i + 8 * u) * d + a);
                tv[u] = __ldg(dZ + (i + 8 * u) * dz_ld + Kc);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) acc = fmaf(xv[u], tv[u], acc);
        }
        for (; i < r1; i += 8) acc = fmaf(ldf<T>(X + i * d + a), __ldg(dZ + i * dz_ld + Kc), acc);
    }
    red[t] = acc;
    __syncthreads();
    if (w == 0 && a < d) {
        float s = 0.f;
        for (int ww = 0; ww < 8; ++ww) s += red[ww * 32 + col];
        part[static_cast<int64_t>(blockIdx.x) * d * Dc + static_cast<int64_t>(a) * Dc + Kc] = s;
    }
    if (blockIdx.y != 0) return;                          // block-uniform
    __syncthreads();
    float sdt = 0.f;
    for (int64_t i = r0 + t; i < r1; i += 256) sdt += __ldg(dZ + i * dz_ld + Kc);
    red[t] = sdt;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (t < o) red[t] += red[t + o];
        __syncthreads();
    }
    if (t == 0) dbg_part[blockIdx.x] = red[0];
}

// Register-tiled fp32 GEMM tiles for the weight and input gradients: a 128 x 128 output
// tile per 256-thread block, 8 reduction steps per shared-memory stage (two stages, the
// next one loaded into registers while the current one is multiplied), and 8 x 8 outputs
// per thread at rows {4ty.., 64 + 4ty..} and columns {4tx.., 64 + 4tx..} so that every
// shared-memory read is a conflict-free float4.
constexpr int kGT = 128, kGK = 8, kGPad = 4;

__device__ __forceinline__ void gemm_stage(const float (&As)[kGK][kGT + kGPad], const float (&Bs)[kGK][kGT + kGPad],
                                           int ty, int tx, float (&acc)[8][8]) {
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
        float av[8], bv[8];
        const float4 a0 = *reinterpret_cast<const float4 *>(&As[kk][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4 *>(&As[kk][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[kk][64 + tx * 4]);
        av[0] = a0.x; av[1] = a0.y; av[2] = a0.z; av[3] = a0.w;
        av[4] = a1.x; av[5] = a1.y; av[6] = a1.z; av[7] = a1.w;
        bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w;
        bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int w = 0; w < 8; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
    }
}


// part[p][a][k] = sum over rows i of range p of X[i][a] * dZ[i][k]  (a < d, k < Kc = 3D;
// column Kc is bwd_dwg_kernel's).  Stage: 8 rows of X (scalar loads, 128 columns) and
// 8 rows of dZ (float4 loads, dz_ld % 4 == 0).
template <typename T>
__global__ void __launch_bounds__(256, 2) bwd_dw_kernel(const T *__restrict__ X, const float *__restrict__ dZ,
                                                        int64_t N, int d, int64_t dz_ld, int Kc, int Dc,
                                                        int64_t rows_per_part, float *__restrict__ part) {
    __shared__ __align__(16) float As[2][kGK][kGT + kGPad];
    __shared__ __align__(16) float Bs[2][kGK][kGT + kGPad];
    const int a0 = blockIdx.x * kGT, k0 = blockIdx.y * kGT;
    const int64_t r0 = static_cast<int64_t>(blockIdx.z) * rows_per_part;
    const int64_t r1 = std::min<int64_t>(N, r0 + rows_per_part);
    const int t = threadIdx.x, tx = t % 16, ty = t / 16;
    // loader roles: X column t % 128, rows t / 128 + 2j; dZ row t / 32, float4 (t % 32)
    const int xa = t % kGT, xr = t / kGT;
    const int zr = t / 32, zc = (t % 32) * 4;
    float xa_reg[4];
    float4 zb_reg;
    auto load = [&](int64_t i0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t i = i0 + xr + 2 * j;
            xa_reg[j] = (i < r1 && a0 + xa < d) ? ldf<T>(X + i * d + a0 + xa) : 0.f;
        }
        const int64_t i = i0 + zr;
        const int k = k0 + zc;
        zb_reg = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < r1 && k < Kc) {
            zb_reg = *reinterpret_cast<const float4 *>(dZ + i * dz_ld + k);
            if (k + 1 >= Kc) zb_reg.y = 0.f;
            if (k + 2 >= Kc) zb_reg.z = 0.f;
            if (k + 3 >= Kc) zb_reg.w = 0.f;
        }
    };
    auto store = [&](int b) {
#pragma unroll
        for (int j = 0; j < 4; ++j) As[b][xr + 2 * j][xa] = xa_reg[j];
        *reinterpret_cast<float4 *>(&Bs[b][zr][zc]) = zb_reg;
    };
    float acc[8][8] = {};
    const int64_t steps = ceil_div(std::max<int64_t>(r1 - r0, 0), kGK);
    if (steps > 0) {
        load(r0);
        store(0);
        __syncthreads();
        for (int64_t st = 0; st < steps; ++st) {
            const bool more = st + 1 < steps;
            if (more) load(r0 + (st + 1) * kGK);
            gemm_stage(As[st & 1], Bs[st & 1], ty, tx, acc);
            if (more) store((st + 1) & 1);
            __syncthreads();
        }
    }
    float *out = part + static_cast<int64_t>(blockIdx.z) * d * Dc;
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const int a = a0 + (u < 4 ? ty * 4 + u : 64 + ty * 4 + u - 4);
            const int k = k0 + (w < 4 ? tx * 4 + w : 64 + tx * 4 + w - 4);
            if (a < d && k < Kc) out[static_cast<int64_t>(a) * Dc + k] = acc[u][w];
        }
}

// dW_Q | dW_K | dW_V | dw_g from the row-range parts, summed in range order; when w3 is
// given (the tensor cores' sums of the columns k < 3D, as w3[a][k] with row stride 3D)
// those columns are copied from it and column 3D (dw_g) is left to bwd_strided_sum_kernel.
__global__ void bwd_dw_reduce_kernel(const float *__restrict__ part, int P, const float *__restrict__ w3, int d,
                                     int D, int Dc, float *__restrict__ dWQ, float *__restrict__ dWK,
                                     float *__restrict__ dWV, float *__restrict__ dwg) {
    const int64_t total = static_cast<int64_t>(d) * Dc;
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < total;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int a = static_cast<int>(o / Dc), k = static_cast<int>(o % Dc);
        if (w3 && k >= 3 * D) continue;                   // dw_g: bwd_strided_sum_kernel
        float acc = 0.f;
        if (w3) {
            acc = w3[static_cast<int64_t>(a) * 3 * D + k];
        } else {
            for (int p = 0; p < P; ++p) acc += part[static_cast<int64_t>(p) * total + o];
        }
        if (k < D) dWQ[static_cast<int64_t>(a) * D + k] = acc;
        else if (k < 2 * D) dWK[static_cast<int64_t>(a) * D + k - D] = acc;
        else if (k < 3 * D) dWV[static_cast<int64_t>(a) * D + k - 2 * D] = acc;
        else dwg[a] = acc;
    }
}

// Wall[a][k] = column k of [W_Q | W_K | W_V | w_g] at row a, fp32, zero for Dc <= k < ld.
template <typename T>
__global__ void bwd_pack_w_kernel(const T *__restrict__ WQ, const T *__restrict__ WK, const T *__restrict__ WV,
                                  const T *__restrict__ wg, int d, int D, int64_t ld, float *__restrict__ Wall) {
    const int64_t total = static_cast<int64_t>(d) * ld;
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < total;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t a = o / ld;
        const int k = static_cast<int>(o % ld);
        float v = 0.f;
        if (k < D) v = ldf<T>(WQ + a * D + k);
        else if (k < 2 * D) v = ldf<T>(WK + a * D + k - D);
        else if (k < 3 * D) v = ldf<T>(WV + a * D + k - 2 * D);
        else if (k == 3 * D) v = ldf<T>(wg + a);
        Wall[o] = v;
    }
}

// dX[i][a] = sum_{k < Dc} dZ[i][k] * Wall[a][k]: 128 x 128 tiles of (rows, a).  Stage:
// 8 columns k of 128 rows of dZ and of Wall (a float4 per thread each, stored transposed).
__global__ void __launch_bounds__(256, 2) bwd_dx_kernel(const float *__restrict__ dZ, const float *__restrict__ Wall,
                                                        int64_t N, int d, int64_t ld, int Dc, float *__restrict__ dX) {
    __shared__ __align__(16) float As[2][kGK][kGT + kGPad];
    __shared__ __align__(16) float Bs[2][kGK][kGT + kGPad];
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kGT;
    const int a0 = blockIdx.y * kGT;
    const int t = threadIdx.x, tx = t % 16, ty = t / 16;
    const int lr = t / 2, lc = (t % 2) * 4;           // loader: row lr, columns lc .. lc + 3
    float4 ar, br;
    auto ld4 = [&](const float *base, int64_t row, int64_t rows, int k) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row < rows && k < Dc) {
            v = *reinterpret_cast<const float4 *>(base + row * ld + k);
            if (k + 1 >= Dc) v.y = 0.f;
            if (k + 2 >= Dc) v.z = 0.f;
            if (k + 3 >= Dc) v.w = 0.f;
        }
        return v;
    };
    auto load = [&](int k0) {
        ar = ld4(dZ, i0 + lr, N, k0 + lc);
        br = ld4(Wall, a0 + lr, d, k0 + lc);
    };
    auto store = [&](int b) {
        As[b][lc + 0][lr] = ar.x; As[b][lc + 1][lr] = ar.y; As[b][lc + 2][lr] = ar.z; As[b][lc + 3][lr] = ar.w;
        Bs[b][lc + 0][lr] = br.x; Bs[b][lc + 1][lr] = br.y; Bs[b][lc + 2][lr] = br.z; Bs[b][lc + 3][lr] = br.w;
    };
    float acc[8][8] = {};
    const int steps = (Dc + kGK - 1) / kGK;
    load(0);
    store(0);
    __syncthreads();
    for (int st = 0; st < steps; ++st) {
        const bool more = st + 1 < steps;
        if (more) load((st + 1) * kGK);
        gemm_stage(As[st & 1], Bs[st & 1], ty, tx, acc);
        if (more) store((st + 1) & 1);
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + (u < 4 ? ty * 4 + u : 64 + ty * 4 + u - 4);
        if (i >= N) continue;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const int a = a0 + (w < 4 ? tx * 4 + w : 64 + tx * 4 + w - 4);
            if (a < d) dX[i * d + a] = acc[u][w];
        }
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

unsigned warp_grid(int64_t n) {
    return static_cast<unsigned>(std::max<int64_t>(1, ceil_div(n * 32, 256)));
}

// Whether bwd_kv_global_tc_kernel writes the source side's global terms (defined with it).
bool kv_global_tc(const Ctx *c);

// Light source rows: two edges per warp step where a head spans at least two of the
// 16-lane half's slices (2 EPL <= r, EPL <= 4), else one edge per step.
template <typename T, int E>
void launch_kv_light(Ctx *c, const T *Q, const T *KV, float isr, int64_t Dz, cudaStream_t sk) {
    const int64_t nkl = c->bw_nk_light;
    if constexpr (E == 4 && sizeof(T) == 2) {
        if (kv_global_tc(c)) {                    // (2 E <= r holds: r >= 16)
            if (c->bw_pds) {                      // stored (p, ds): one row per half-warp
                bwd_kv_pair_kernel<false><<<warp_grid(ceil_div(nkl, 2)), 256, kKvRingBytes, sk>>>(c->bw_k_rows, nkl,
                    c->t_row_ptr, c->t_col, Q, static_cast<const T *>(c->bw_dL), c->H, c->r, c->bw_dZ, Dz, c->bw_dZb,
                    nullptr, nullptr, c->bw_pds);
                return;
            }
            bwd_local_kv2_kernel<T, E, true><<<warp_grid(nkl), 256, 0, sk>>>(c->bw_k_rows, nkl, c->t_row_ptr, c->t_col,
                Q, KV, static_cast<const T *>(c->bw_dL), c->bw_lse, c->bw_Dd, nullptr, nullptr, c->H, c->r, isr, c->bw_dZ, Dz, c->bw_dZb,
                nullptr, nullptr);
            return;
        }
    }
    if constexpr (E <= 4) {
        if (2 * E <= c->r) {
            bwd_local_kv2_kernel<T, E><<<warp_grid(nkl), 256, 0, sk>>>(c->bw_k_rows, nkl, c->t_row_ptr, c->t_col,
                Q, KV, static_cast<const T *>(c->bw_dL), c->bw_lse, c->bw_Dd, c->bw_dSc, c->bw_dST, c->H, c->r, isr, c->bw_dZ, Dz, nullptr,
                nullptr, nullptr);
            return;
        }
    }
    bwd_local_kv_kernel<T, E, false><<<warp_grid(nkl), 256, 0, sk>>>(c->bw_k_rows, nkl, c->t_row_ptr, c->t_col,
        nullptr, nullptr, Q, KV, static_cast<const T *>(c->bw_dL), c->bw_lse, c->bw_Dd, c->bw_dSc, c->bw_dST, c->H, c->r, isr, c->bw_dZ, Dz, nullptr);
}

// Light target rows: two edges per warp step under the same condition as the source side.
template <typename T, int E>
void launch_q_light(Ctx *c, const T *Q, const T *KV, float isr, int64_t Dz, cudaStream_t sq) {
    const int64_t nql = c->bw_nq_light;
    if constexpr (kQRing<T, E>) {
        if (2 * E <= c->r) {                      // one row per half-warp
            bwd_q_pair_kernel<false><<<warp_grid(ceil_div(nql, 2)), 256, kQRingBytes, sq>>>(c->bw_q_rows, nql,
                c->row_ptr, c->col_idx, Q, KV, static_cast<const T *>(c->bw_dL), c->H, c->r, isr, c->bw_lse,
                c->bw_Dd, c->bw_dZ, Dz, c->bw_dZb, nullptr, nullptr, c->bw_perm, c->bw_pds);
            return;
        }
    }
    if constexpr (E <= 4 && !kQRing<T, E>) {
        if (2 * E <= c->r) {
            bwd_local_q2_kernel<T, E><<<warp_grid(nql), 256, 0, sq>>>(c->bw_q_rows, nql, c->row_ptr, c->col_idx,
                Q, KV, static_cast<const T *>(c->bw_dL), c->H, c->r, isr, c->bw_lse, c->bw_Dd, c->bw_dZ, Dz, c->bw_dZb,
                nullptr, nullptr);
            return;
        }
    }
    bwd_local_q_kernel<T, E><<<warp_grid(nql), 256, 0, sq>>>(c->bw_q_rows, nql, c->row_ptr, c->col_idx, Q, KV,
        static_cast<const T *>(c->bw_dL), c->H, c->r, isr, c->bw_lse, c->bw_Dd, c->bw_dZ, Dz);
}

// Chunks of heavy source / target rows: the two-edges-per-step kernels in chunk mode where
// the light rows use them, else one edge per step across the warp.
template <typename T, int E>
void launch_kv_chunks(Ctx *c, const T *Q, const T *KV, float isr, cudaStream_t sk) {
    const int64_t nkc = c->bw_nk_chunks;
    if constexpr (E <= 4) {
        if (2 * E <= c->r) {
            if constexpr (sizeof(T) == 2 && E == 4) {
                if (c->bw_pds) {                  // stored (p, ds): one chunk per half-warp
                    bwd_kv_pair_kernel<true><<<warp_grid(ceil_div(nkc, 2)), 256, kKvRingBytes, sk>>>(nullptr, nkc,
                        c->t_row_ptr, c->t_col, Q, static_cast<const T *>(c->bw_dL), c->H, c->r, nullptr, 0, nullptr,
                        c->bw_k_chunks, c->bw_kv_part, c->bw_pds);
                    return;
                }
            }
            bwd_local_kv2_kernel<T, E, false, true><<<warp_grid(nkc), 256, 0, sk>>>(nullptr, nkc, c->t_row_ptr,
                c->t_col, Q, KV, static_cast<const T *>(c->bw_dL), c->bw_lse, c->bw_Dd, nullptr, nullptr, c->H, c->r,
                isr, nullptr, 0, nullptr, c->bw_k_chunks, c->bw_kv_part);
            return;
        }
    }
    bwd_kv_chunk_kernel<T, E><<<warp_grid(nkc), 256, 0, sk>>>(c->bw_k_chunks, nkc, c->t_row_ptr, c->t_col, Q, KV,
        static_cast<const T *>(c->bw_dL), c->bw_lse, c->bw_Dd, c->H, c->r, isr, c->bw_kv_part);
}
template <typename T, int E>
void launch_q_chunks(Ctx *c, const T *Q, const T *KV, float isr, cudaStream_t sq) {
    const int64_t nqc = c->bw_nq_chunks;
    if constexpr (kQRing<T, E>) {
        if (2 * E <= c->r) {                      // one chunk per half-warp
            bwd_q_pair_kernel<true><<<warp_grid(ceil_div(nqc, 2)), 256, kQRingBytes, sq>>>(nullptr, nqc, c->row_ptr,
                c->col_idx, Q, KV, static_cast<const T *>(c->bw_dL), c->H, c->r, isr, c->bw_lse, c->bw_Dd, nullptr, 0,
                nullptr, c->bw_q_chunks, c->bw_q_part, c->bw_perm, c->bw_pds);
            return;
        }
    }
    if constexpr (E <= 4 && !kQRing<T, E>) {
        if (2 * E <= c->r) {
            bwd_local_q2_kernel<T, E, true><<<warp_grid(nqc), 256, 0, sq>>>(nullptr, nqc,
                c->row_ptr, c->col_idx, Q, KV, static_cast<const T *>(c->bw_dL), c->H, c->r, isr, c->bw_lse, c->bw_Dd,
                nullptr, 0, nullptr, c->bw_q_chunks, c->bw_q_part);
            return;
        }
    }
    bwd_q_chunk_kernel<T, E><<<warp_grid(nqc), 256, 0, sq>>>(c->bw_q_chunks, nqc, c->row_ptr, c->col_idx, Q, KV,
        static_cast<const T *>(c->bw_dL), c->H, c->r, isr, c->bw_lse, c->bw_Dd, c->bw_q_part);
}

// Heavy source rows: chunk sums, then the global terms (or, with the tensor-core global
// terms, the local sums added to them).
template <typename T, int E>
void launch_kv_heavy(Ctx *c, const T *Q, const T *KV, float isr, int64_t Dz, const int32_t *kh, int64_t nkh,
                     cudaStream_t sk) {
    const size_t sm = static_cast<size_t>(kMW) * 2 * c->D * 4;
    auto go = [&](auto kern, const float *dSc, const float *dST, __nv_bfloat16 *dZb) {
        if (sm > 48 * 1024)
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
        kern<<<static_cast<unsigned>(nkh), kMW * 32, sm, sk>>>(kh, nkh, c->t_row_ptr, c->t_col, c->bw_k_cptr,
                                                               c->bw_kv_part, Q, KV, static_cast<const T *>(c->bw_dL), c->bw_lse, c->bw_Dd,
                                                               dSc, dST, c->H, c->r, isr, c->bw_dZ, Dz, dZb);
    };
    if constexpr (E == 4 && sizeof(T) == 2) {
        if (kv_global_tc(c)) return go(bwd_local_kv_kernel<T, E, true, true>, nullptr, nullptr, c->bw_dZb);
    }
    go(bwd_local_kv_kernel<T, E, true>, c->bw_dSc, c->bw_dST, nullptr);
}

// Both local backward kernels with EPL = lane_features(D): light rows one warp each;
// heavy rows (more than kHeavyDegree entries) as kChunk-edge chunks, one warp each, whose
// shares the per-row kernels merge in chunk order.  The target-side (dq) kernels go to
// stream sq and the source-side (dk, dv) kernels to sk: they read the same inputs and
// write disjoint columns of dZ.
template <typename T>
void launch_local_bwd(Ctx *c, const T *Q, const T *KV, float isr, int64_t Dz, cudaStream_t sq, cudaStream_t sk) {
    const int H = c->H, R = c->r;
    const size_t D = static_cast<size_t>(c->D);
    const int64_t nql = c->bw_nq_light, nqh = c->bw_nq_heavy, nkl = c->bw_nk_light, nkh = c->bw_nk_heavy;
    const int32_t *qh = c->bw_q_rows + nql, *kh = c->bw_k_rows + nkl;
    // with stored (p, ds) the source side reads what the target side wrote: it waits for
    // the target side's light rows and chunks (ev_q), else the two sides run side by side
#define GLGA_LB(E)                                                                                        \
    case E:                                                                                               \
        if (c->bw_pds) {                                                                                  \
            if (nql) launch_q_light<T, E>(c, Q, KV, isr, Dz, sq);                                        \
            if (nqh) launch_q_chunks<T, E>(c, Q, KV, isr, sq);                                           \
            cudaEventRecord(c->bw_ev_q, sq);                                                              \
            cudaStreamWaitEvent(sk, c->bw_ev_q, 0);                                                       \
        }                                                                                                 \
        if (nkl) launch_kv_light<T, E>(c, Q, KV, isr, Dz, sk);                                           \
        if (nkh) {                                                                                        \
            launch_kv_chunks<T, E>(c, Q, KV, isr, sk);                                                   \
            launch_kv_heavy<T, E>(c, Q, KV, isr, Dz, kh, nkh, sk);                                      \
        }                                                                                                 \
        if (!c->bw_pds && nql) launch_q_light<T, E>(c, Q, KV, isr, Dz, sq);                              \
        if (nqh) {                                                                                        \
            if (!c->bw_pds) launch_q_chunks<T, E>(c, Q, KV, isr, sq);                                    \
            bwd_q_heavy_kernel<E><<<static_cast<unsigned>(nqh), kMW * 32, kMW * D * 4, sq>>>(qh, nqh,      \
                c->bw_q_cptr, c->bw_q_part, H, R, c->bw_dZ, Dz, c->bw_dZb);                                          \
        }                                                                                                 \
        break;
    switch (lane_features(c->D)) {
        GLGA_LB(1) GLGA_LB(2) GLGA_LB(4) GLGA_LB(8) GLGA_LB(16) GLGA_LB(32)
        default: break;
    }
#undef GLGA_LB
}

int local_bwd_launches(const Ctx *c) {
    return (c->bw_nq_light > 0) + 2 * (c->bw_nq_heavy > 0) + (c->bw_nk_light > 0) + 2 * (c->bw_nk_heavy > 0);
}

// ---------------------------------------------------------------------------------------
// Readout backward on the tensor cores (bf16 layers, H*r = 128, r <= 64, one head group):
// per 128-row tile,
//   [num | den] = phi(Q) B_g            (tcgen05, B_g = the forward's readout operand)
//   epilogue:  G, dL = g dY, dnum = (1-g) dY / den, dden = -(dG . G)/den, D_i, dt
//   dphi = dnum blockdiag(S_h)          (tcgen05, A = dnum rounded to bf16)
//   dq_global = (dphi + z dden) phi'(q)
// 16 warps, one CTA per SM: warp w reads TMEM lanes 32 (w % 4) (its 32 tile rows) and
// owns columns 32 (w / 4) .. +31, one thread per row.  The Q, dY and L tiles arrive by
// TMA (128-byte swizzle, the MMA operand layout): Q in two buffers (the next tile's lands
// while this one runs), dY and L issued as soon as this tile is done with them.  phi(Q)
// is formed in place as the first A operand and dnum in place of dY as the second; a
// tile the threads have read doubles as the 2 KB-per-warp staging area of the coalesced
// row stores (8 rows x 64 B per instruction).  phi'(q) = min(phi(q), 1) from the bf16
// phi(q).  Per-head and per-row sums that span column quarters meet in shared memory.
constexpr int kBroTcD = 128;
constexpr int kBroTcBN = kBroTcD + 16;            // num | den (H <= 8) | zero columns
constexpr int kBroTcWarps = 16;
constexpr uint32_t kBroTcAtom = 128 * 128;        // one 64-column atom of a 128-row operand
constexpr uint32_t kBroTcB1Atom = kBroTcBN * 128; // one 64-column atom of B_g (144 rows)
constexpr uint32_t kBroTcStage = 4096;            // staging bytes per warp (source side)
constexpr size_t kBroTcSmem = 1024 + 4 * 2 * kBroTcAtom + 2 * kBroTcB1Atom + 2 * kBroTcAtom +
                              (kBroTcD + 3 * 4 * 128) * 4;

// byte offset of element (row, k) of a K-major operand with 64-element atoms of `rows` rows
__device__ __forceinline__ uint32_t swz_off(int row, int k, uint32_t atom_bytes) {
    return static_cast<uint32_t>(k >> 6) * atom_bytes + static_cast<uint32_t>(row) * 128u +
           ((static_cast<uint32_t>((k & 63) >> 3) ^ static_cast<uint32_t>(row & 7)) << 4) +
           static_cast<uint32_t>(k & 7) * 2u;
}

// The lane's 32 floats (its row, columns c0 .. c0 + 31) to a row-major float32 matrix:
// each 4-float piece p into the staging area (row r at byte r * 128, piece p at slot
// p ^ (r & 7)) as it is computed, then eight coalesced stores of 4 rows x 128 B.  Rows at
// or past N are not written.
__device__ __forceinline__ void stage_f32_piece(uint8_t *stage, int lane, int p, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(stage + lane * 128 + ((p ^ (lane & 7)) << 4)) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void warp_rows_f32_flush(float *dst, int64_t ld, int64_t r0, int64_t N, int c0,
                                                    uint8_t *stage, int lane) {
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = 4 * i + (lane >> 3), p = lane & 7;
        const int64_t gr = r0 + r;
        const float4 x = *reinterpret_cast<const float4 *>(stage + r * 128 + ((p ^ (r & 7)) << 4));
        if (gr < N) reinterpret_cast<float4 *>(dst + gr * ld + c0)[p] = x;
    }
    __syncwarp();
}

// The lane's 64 bytes of a row (lane = row: 32 bf16 or 16 float32 values) to a row-major
// matrix: four 16-byte pieces into a 2 KB staging area (row r at byte r * 64, piece p at
// slot p ^ ((r >> 1) & 3)), then four coalesced stores of 8 rows x 64 B to dst + row * ld
// (bytes).  Rows at or past N are not written.
__device__ __forceinline__ void stage_row64_piece(uint8_t *stage, int lane, int p, uint4 v) {
    *reinterpret_cast<uint4 *>(stage + lane * 64 + ((p ^ ((lane >> 1) & 3)) << 4)) = v;
}
__device__ __forceinline__ void warp_rows64_flush(uint8_t *dst, int64_t ld, int64_t r0, int64_t N, uint8_t *stage,
                                                  int lane) {
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = 8 * i + (lane >> 2), p = lane & 3;
        const int64_t gr = r0 + r;
        const uint4 x = *reinterpret_cast<const uint4 *>(stage + r * 64 + ((p ^ ((r >> 1) & 3)) << 4));
        if (gr < N) reinterpret_cast<uint4 *>(dst + (r0 + r) * ld)[p] = x;
    }
    __syncwarp();
}

template <int R>
__global__ void __launch_bounds__(kBroTcWarps * 32, 1) bwd_readout_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmY,
    const __grid_constant__ CUtensorMap tmL, const float *__restrict__ t, const __nv_bfloat16 *__restrict__ Bg,
    int ro_kp, const float *__restrict__ Sz, int64_t N, int H, float b_g, float eps, __nv_bfloat16 *__restrict__ dL,
    float *__restrict__ Dd, __nv_bfloat16 *__restrict__ dnum, float *__restrict__ dZ, int64_t dz_ld,
    __nv_bfloat16 *__restrict__ dZb, unsigned *flag) {
    constexpr int D = kBroTcD;
    constexpr int kHQ = R >= 32 ? 1 : 32 / R;     // heads in a 32-column quarter
    constexpr uint32_t kTile = 2 * kBroTcAtom;    // a [128][128] bf16 tile
    extern __shared__ uint8_t bro_raw[];
    __shared__ __align__(8) uint64_t q_full[2], y_full, l_full, mma_bar;
    __shared__ uint32_t tmem_sh;
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(bro_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sQb = sm;                             // [2] Q tiles: phi(Q) in place is the first A
    uint8_t *sY = sQb + 2 * kTile;                 // dY tile; dnum in place is the second A
    uint8_t *sL = sY + kTile;                      // L tile, then the first epilogue's staging
    uint8_t *sB1 = sL + kTile;                     // B_g: 2 atoms of 144 rows
    uint8_t *sB2 = sB1 + 2 * kBroTcB1Atom;         // blockdiag(S_h): 2 atoms
    float *zf = reinterpret_cast<float *>(sB2 + 2 * kBroTcAtom);
    float *xdt = zf + D;                           // [4 quarters][128 rows] dt partials
    float *xdd = xdt + 4 * 128;                    // ... (dG . G) partials (r = 64: a head spans 2)
    float *xDd = xdd + 4 * 128;                    // ... (dL . L) partials
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cq = warp >> 2;     // TMEM lane quarter, column quarter
    const int rt = quad * 32 + lane;               // row in the tile
    const int c0 = cq * 32;                        // first column of this warp
    const float *z = Sz + static_cast<int64_t>(H) * R * R;

    // operands that stay for the whole launch: B_g, blockdiag(S_h), z
    for (int ch = tid; ch < kBroTcBN * (D / 8); ch += blockDim.x) {
        const int n = ch / (D / 8), k8 = (ch % (D / 8)) * 8;
        const uint4 v = *reinterpret_cast<const uint4 *>(Bg + static_cast<int64_t>(n) * ro_kp + k8);
        *reinterpret_cast<uint4 *>(sB1 + swz_off(n, k8, kBroTcB1Atom)) = v;
    }
    for (int ch = tid; ch < D * (D / 8); ch += blockDim.x) {
        const int f = ch / (D / 8), c8 = (ch % (D / 8)) * 8;
        const int h = f / R;
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = 0.f;
        if (c8 / R == h) {   // 8 columns of head h: S_h[f - h R][c8 - h R ..]
            const float4 *sp = reinterpret_cast<const float4 *>(Sz + (static_cast<int64_t>(h) * R + (f - h * R)) * R + (c8 - h * R));
            const float4 a0 = __ldg(sp), a1 = __ldg(sp + 1);
            v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w; v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
        }
        *reinterpret_cast<uint4 *>(sB2 + swz_off(f, c8, kBroTcAtom)) =
            make_uint4(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]), bf16x2_bits(v[4], v[5]), bf16x2_bits(v[6], v[7]));
    }
    for (int f = tid; f < D; f += blockDim.x) zf[f] = z[f];
    const int64_t n_tiles = ceil_div(N, 128);
    const int my = blockIdx.x < n_tiles ? static_cast<int>((n_tiles - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    // the rows of this block's k-th tile of one input into a tile buffer (two 64-column boxes)
    auto issue = [&](const CUtensorMap *m, uint64_t *bar, uint8_t *dst, int k) {
        const int32_t y = static_cast<int32_t>((blockIdx.x + static_cast<int64_t>(k) * gridDim.x) * 128);
        mbar_arrive_expect_tx(bar, kTile);
        tma_load_2d(dst, m, bar, 0, y);
        tma_load_2d(dst + kBroTcAtom, m, bar, 64, y);
    };
    int nq = 0, ny = 0, nl = 0;                    // loads issued (thread 0)
    if (tid == 0) {
        mbar_init(&q_full[0], 1);
        mbar_init(&q_full[1], 1);
        mbar_init(&y_full, 1);
        mbar_init(&l_full, 1);
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
        for (; nq < my && nq < 2; ++nq) issue(&tmQ, &q_full[nq], sQb + nq * kTile, nq);
        if (my > 0) {
            issue(&tmY, &y_full, sY, 0);
            issue(&tmL, &l_full, sL, 0);
            ny = nl = 1;
        }
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(&tmem_sh, 256u);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sh;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t idesc1 = instr_desc(128, kBroTcBN, 1u, false, false);
    const uint32_t idesc2 = instr_desc(128, D, 1u, false, false);
    uint32_t phase = 0;
    // the tile's MMAs: 8 K steps of 16 over the two atoms of A and B, one thread
    auto mma = [&](const uint8_t *sa, const uint8_t *sb, uint32_t b_atom, uint32_t idesc) {
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t ko = static_cast<uint32_t>(ks >> 2), kb = static_cast<uint32_t>(ks & 3) * 32u;
                umma_bf16(tmem, smem_desc(a0 + ko * kBroTcAtom + kb, 16, 1024, 2),
                          smem_desc(b0 + ko * b_atom + kb, 16, 1024, 2), idesc, ks != 0);
            }
            umma_commit(&mma_bar);
        }
    };
    // every thread waits; the block leaves together if any wait gave up
    auto wait_all = [&](uint64_t *bar, uint32_t par) -> bool {
        const bool got = mbar_wait_bounded(bar, par);
        const bool bad = __syncthreads_or(!got) != 0;
        if (bad && tid == 0) atomicOr(flag, kDevErrTimeout);
        return !bad;
    };
    auto bf = [](const uint4 (&w)[4], int j) {
        const uint32_t word = (&w[j / 8].x)[(j % 8) / 2];
        return __uint_as_float((j & 1) ? (word & 0xffff0000u) : (word << 16));
    };
    // the warp's 32 rows x 32 columns of a landed tile (lane = row)
    auto slice = [&](const uint8_t *tile, uint4 (&w)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = *reinterpret_cast<const uint4 *>(tile + swz_off(rt, c0 + 8 * i, kBroTcAtom));
    };
    // the gate pre-activation of this thread's row, one tile ahead
    auto t_of = [&](int kk) {
        const int64_t rr = (blockIdx.x + static_cast<int64_t>(kk) * gridDim.x) * 128 + rt;
        return kk < my && rr < N ? __ldg(t + rr) : 0.f;
    };
    float t_next = t_of(0);
    int k = 0;
    for (; k < my; ++k) {
        const int64_t m0 = (blockIdx.x + static_cast<int64_t>(k) * gridDim.x) * 128, r0 = m0 + quad * 32;
        const int64_t row = m0 + rt;
        const bool valid = row < N;
        const float t_row = t_next;
        t_next = t_of(k + 1);
        uint8_t *sQ = sQb + (k & 1) * kTile;
        if (!wait_all(&q_full[k & 1], static_cast<uint32_t>(k >> 1) & 1u)) break;
        // ---- A = phi(q) in place (rows past N hold zeros: phi = 1, never stored) ----
        for (int ch = tid; ch < static_cast<int>(kTile / 16); ch += blockDim.x) {
            uint4 *p = reinterpret_cast<uint4 *>(sQ + ch * 16);
            const uint4 u = *p;
            *p = make_uint4(phi_bf16x2(u.x), phi_bf16x2(u.y), phi_bf16x2(u.z), phi_bf16x2(u.w));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        mma(sQ, sB1, kBroTcB1Atom, idesc1);
        const bool m1 = wait_all(&mma_bar, phase);
        phase ^= 1u;
        if (!m1) break;
        tc_fence_after();
        // ---- epilogue 1 ----
        uint32_t dv[8];
        tmem_ld_n<4>(tmem + lane_base + D, *reinterpret_cast<uint32_t (*)[4]>(&dv[0]));
        tmem_ld_n<4>(tmem + lane_base + D + 4, *reinterpret_cast<uint32_t (*)[4]>(&dv[4]));
        tmem_ld_wait();
        const float g = valid ? 1.f / (1.f + __expf(-(t_row + b_g))) : 0.f;
        float inv[kHQ], dda[kHQ], Dda[kHQ];
#pragma unroll
        for (int hq = 0; hq < kHQ; ++hq) {
            const int h = c0 / R + hq;
            inv[hq] = 1.f / (__uint_as_float(dv[h < 8 ? h : 0]) + eps);
            dda[hq] = 0.f;
            Dda[hq] = 0.f;
        }
        const uint32_t yl_par = static_cast<uint32_t>(k) & 1u;
        if (!wait_all(&y_full, yl_par) || !wait_all(&l_full, yl_par)) break;
        uint4 yw[4], lw[4];
        slice(sY, yw);
        slice(sL, lw);
        __syncthreads();   // every warp holds its dY and L slices: the L tile is the staging
        uint8_t *stg = sL + warp * 2048;
        // dL = g dY stored in bf16, and D_i from the stored values
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = 8 * p + 2 * e, hq = j / R < kHQ ? j / R : 0;
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(g * bf(yw, j), g * bf(yw, j + 1));
                const float2 v = __bfloat1622float2(h2);
                Dda[hq] = fmaf(v.x, bf(lw, j), Dda[hq]);
                Dda[hq] = fmaf(v.y, bf(lw, j + 1), Dda[hq]);
                w[e] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            stage_row64_piece(stg, lane, p, make_uint4(w[0], w[1], w[2], w[3]));
        }
        warp_rows64_flush(reinterpret_cast<uint8_t *>(dL + c0), static_cast<int64_t>(D) * 2, r0, N, stg, lane);
        float dtp = 0.f;
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {           // 16 columns at a time
            uint32_t nv[16];
            tmem_ld16(tmem + lane_base + static_cast<uint32_t>(c0 + 16 * hb), nv);
            tmem_ld_wait();
            float dn[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 16 * hb + e, hq = j / R < kHQ ? j / R : 0;
                const float y = bf(yw, j);
                const float G = __uint_as_float(nv[e]) * inv[hq];
                const float dG = (1.f - g) * y;
                dn[e] = dG * inv[hq];
                dda[hq] = fmaf(dG, G, dda[hq]);
                dtp = fmaf(y, bf(lw, j) - G, dtp);
            }
            // dnum in bf16: the second MMA's A operand, in place of the warp's own dY slice,
            // and the rows the dS | dz kernel reads
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint4 wv = make_uint4(bf16x2_bits(dn[8 * i], dn[8 * i + 1]), bf16x2_bits(dn[8 * i + 2], dn[8 * i + 3]),
                                            bf16x2_bits(dn[8 * i + 4], dn[8 * i + 5]), bf16x2_bits(dn[8 * i + 6], dn[8 * i + 7]));
                *reinterpret_cast<uint4 *>(sY + swz_off(rt, c0 + 16 * hb + 8 * i, kBroTcAtom)) = wv;
                stage_row64_piece(stg, lane, 2 * hb + i, wv);
            }
        }
        warp_rows64_flush(reinterpret_cast<uint8_t *>(dnum + c0), static_cast<int64_t>(D + 16) * 2, r0, N, stg, lane);
        xdt[cq * 128 + rt] = dtp;
        xdd[cq * 128 + rt] = dda[0];
        xDd[cq * 128 + rt] = Dda[0];
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        mma(sY, sB2, kBroTcAtom, idesc2);
        if (tid == 0 && nl < my) {                 // the staging is done: the next L tile
            issue(&tmL, &l_full, sL, nl);
            ++nl;
        }
        // per-row and per-head sums across the column quarters; dden, D_i and dt out
        float ddh[kHQ];
        if constexpr (R == 64) {
            const int q0 = cq & ~1;                // the head's two quarters
            const float s_dd = xdd[q0 * 128 + rt] + xdd[(q0 + 1) * 128 + rt];
            const float s_Dd = xDd[q0 * 128 + rt] + xDd[(q0 + 1) * 128 + rt];
            ddh[0] = -s_dd * inv[0];
            if (valid && (cq & 1) == 0) {
                dnum[row * (D + 16) + D + c0 / R] = __float2bfloat16_rn(ddh[0]);
                Dd[row * H + c0 / R] = s_Dd;
            }
        } else {
#pragma unroll
            for (int hq = 0; hq < kHQ; ++hq) {
                ddh[hq] = -dda[hq] * inv[hq];
                if (valid) {
                    dnum[row * (D + 16) + D + c0 / R + hq] = __float2bfloat16_rn(ddh[hq]);
                    Dd[row * H + c0 / R + hq] = Dda[hq];
                }
            }
        }
        if (cq == 0 && valid)
            dZ[row * dz_ld + 3 * D] = g * (1.f - g) * (xdt[rt] + xdt[128 + rt] + xdt[256 + rt] + xdt[384 + rt]);
        const bool m2 = wait_all(&mma_bar, phase);
        phase ^= 1u;
        if (!m2) break;
        tc_fence_after();
        if (tid == 0 && ny < my) {                 // the second MMA has read dnum: the next dY tile
            issue(&tmY, &y_full, sY, ny);
            ++ny;
        }
        // ---- epilogue 2: dq_global = (dphi + z dden) phi'(q), phi'(q) = min(phi(q), 1) ----
        uint4 pw[4];
        slice(sQ, pw);
        __syncthreads();   // every warp holds its phi(q) slice: the Q tile is the staging
        stg = sQ + warp * 2048;
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            uint32_t av[16];
            tmem_ld16(tmem + lane_base + static_cast<uint32_t>(c0 + 16 * hb), av);
            tmem_ld_wait();
            float o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 16 * hb + e, hq = j / R < kHQ ? j / R : 0;
                o[e] = fmaf(zf[c0 + j], ddh[hq], __uint_as_float(av[e])) * fminf(bf(pw, j), 1.f);
            }
            if (dZb) {                         // bf16 rows of 3D columns: both halves, one store
#pragma unroll
                for (int i = 0; i < 2; ++i)
                    stage_row64_piece(stg, lane, 2 * hb + i,
                                      make_uint4(bf16x2_bits(o[8 * i], o[8 * i + 1]), bf16x2_bits(o[8 * i + 2], o[8 * i + 3]),
                                                 bf16x2_bits(o[8 * i + 4], o[8 * i + 5]), bf16x2_bits(o[8 * i + 6], o[8 * i + 7])));
                if (hb == 1)
                    warp_rows64_flush(reinterpret_cast<uint8_t *>(dZb + c0), static_cast<int64_t>(3 * D) * 2, r0, N, stg, lane);
            } else {
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    stage_row64_piece(stg, lane, p, make_uint4(__float_as_uint(o[4 * p]), __float_as_uint(o[4 * p + 1]),
                                                               __float_as_uint(o[4 * p + 2]), __float_as_uint(o[4 * p + 3])));
                warp_rows64_flush(reinterpret_cast<uint8_t *>(dZ + c0 + 16 * hb), dz_ld * 4, r0, N, stg, lane);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();   // TMEM, the cross-quarter sums and the Q tile are free
        if (tid == 0 && nq < my) {
            issue(&tmQ, &q_full[nq & 1], sQb + (nq & 1) * kTile, nq);
            ++nq;
        }
    }
    // the block leaves only after its copies have landed (already so when all went well)
    if (tid == 0) {
        for (int i = std::max(0, nq - 2); i < nq; ++i) mbar_wait_bounded(&q_full[i & 1], static_cast<uint32_t>(i >> 1) & 1u);
        if (ny > 0) mbar_wait_bounded(&y_full, static_cast<uint32_t>(ny - 1) & 1u);
        if (nl > 0) mbar_wait_bounded(&l_full, static_cast<uint32_t>(nl - 1) & 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256u);
    }
}

// The source side's global terms on the tensor cores (bf16 layers, H*r = 128, r <= 64):
// per 128-row tile of source rows j,
//   G_k = V blockdiag(dS_h)^T       (tcgen05: dphi(k_j)_f = sum_c dS_h[f][c] v_jc)
//   G_v = phi(K) blockdiag(dS_h)    (tcgen05: dv_jf = sum_c dS_h[c][f] phi(k_jc))
//   dZ[j, D + f] = (G_k + dz_f) phi'(k_jf),   dZ[j, 2D + f] = G_v
// written before the source-side gather kernels, which then add their local terms.
// 16 warps, each with 32 rows x 32 columns of the epilogue; the block's tiles stream in by
// TMA (K | V rows, two stages: the next tile lands while this one is multiplied and
// written), and a landed stage, once read, stages the warps' coalesced row stores.
constexpr int kKvgStages = 2;
constexpr uint32_t kKvgStage = 4 * kBroTcAtom;     // the K tile (2 atoms), then the V tile
constexpr size_t kKvgSmem = 1024 + kKvgStages * kKvgStage + 6 * kBroTcAtom + kBroTcD * 4;
static_assert(kBroTcWarps * kBroTcStage <= kKvgStage, "a landed stage doubles as the output staging");

template <int R>
__global__ void __launch_bounds__(kBroTcWarps * 32, 1) bwd_kv_global_tc_kernel(
    const __grid_constant__ CUtensorMap tmKV, const float *__restrict__ dSc, const float *__restrict__ dST,
    int64_t N, int H, float *__restrict__ dZ, int64_t dz_ld, __nv_bfloat16 *__restrict__ dZb, unsigned *flag) {
    constexpr int D = kBroTcD;
    extern __shared__ uint8_t kvg_raw[];
    __shared__ __align__(8) uint64_t full_bar[kKvgStages];
    __shared__ __align__(8) uint64_t mma_bar;
    __shared__ uint32_t tmem_sh;
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(kvg_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sS = sm;                                          // [kKvgStages] K | V tiles (TMA)
    uint8_t *sP = sS + kKvgStages * kKvgStage;                 // A of the second MMA: phi(K)
    uint8_t *sB1 = sP + 2 * kBroTcAtom;                        // blockdiag(dS_h)^T as [f][c] = dS_h[f][c]
    uint8_t *sB2 = sB1 + 2 * kBroTcAtom;                       // blockdiag(dS_h) as [f][c] = dS_h[c][f]
    float *dzf = reinterpret_cast<float *>(sB2 + 2 * kBroTcAtom);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cq = warp >> 2;
    const int rt = quad * 32 + lane;
    const int c0 = cq * 32;
    const float *dz = dSc + static_cast<int64_t>(H) * R * R;
    for (int ch = tid; ch < D * (D / 8); ch += blockDim.x) {
        const int f = ch / (D / 8), c8 = (ch % (D / 8)) * 8;
        const int h = f / R, fl = f - h * R;
        float v1[8], v2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v1[e] = v2[e] = 0.f;
        if (c8 / R == h) {   // 8 columns of head h: dS_h[fl][cl ..] and dS_h^T[fl][cl ..] (= dS_h[cl ..][fl])
            const int64_t o = (static_cast<int64_t>(h) * R + fl) * R + (c8 - h * R);
            const float4 a0 = __ldg(reinterpret_cast<const float4 *>(dSc + o)), a1 = __ldg(reinterpret_cast<const float4 *>(dSc + o) + 1);
            const float4 b0 = __ldg(reinterpret_cast<const float4 *>(dST + o)), b1 = __ldg(reinterpret_cast<const float4 *>(dST + o) + 1);
            v1[0] = a0.x; v1[1] = a0.y; v1[2] = a0.z; v1[3] = a0.w; v1[4] = a1.x; v1[5] = a1.y; v1[6] = a1.z; v1[7] = a1.w;
            v2[0] = b0.x; v2[1] = b0.y; v2[2] = b0.z; v2[3] = b0.w; v2[4] = b1.x; v2[5] = b1.y; v2[6] = b1.z; v2[7] = b1.w;
        }
        *reinterpret_cast<uint4 *>(sB1 + swz_off(f, c8, kBroTcAtom)) =
            make_uint4(bf16x2_bits(v1[0], v1[1]), bf16x2_bits(v1[2], v1[3]), bf16x2_bits(v1[4], v1[5]), bf16x2_bits(v1[6], v1[7]));
        *reinterpret_cast<uint4 *>(sB2 + swz_off(f, c8, kBroTcAtom)) =
            make_uint4(bf16x2_bits(v2[0], v2[1]), bf16x2_bits(v2[2], v2[3]), bf16x2_bits(v2[4], v2[5]), bf16x2_bits(v2[6], v2[7]));
    }
    for (int f = tid; f < D; f += blockDim.x) dzf[f] = dz[f];
    const int64_t n_tiles = ceil_div(N, 128);
    const int my = blockIdx.x < n_tiles ? static_cast<int>((n_tiles - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    // the K | V rows of this block's k-th tile into stage k % 2
    auto issue = [&](int k) {
        const int s = k % kKvgStages;
        const int32_t y = static_cast<int32_t>((blockIdx.x + static_cast<int64_t>(k) * gridDim.x) * 128);
        uint8_t *st = sS + s * kKvgStage;
        mbar_arrive_expect_tx(&full_bar[s], kKvgStage);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(st + b * kBroTcAtom, &tmKV, &full_bar[s], b * 64, y);
    };
    if (tid == 0) {
        for (int s = 0; s < kKvgStages; ++s) mbar_init(&full_bar[s], 1);
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmKV);
        for (int k = 0; k < my && k < kKvgStages; ++k) issue(k);
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(&tmem_sh, 256u);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sh;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t idesc = instr_desc(128, D, 1u, false, false);
    auto bf = [](const uint4 (&w)[4], int j) {
        const uint32_t word = (&w[j / 8].x)[(j % 8) / 2];
        return __uint_as_float((j & 1) ? (word & 0xffff0000u) : (word << 16));
    };
    int k = 0;
    for (; k < my; ++k) {
        const int s = k % kKvgStages;
        uint8_t *sK = sS + s * kKvgStage, *sV = sK + 2 * kBroTcAtom;
        const bool got = mbar_wait_bounded(&full_bar[s], static_cast<uint32_t>(k / kKvgStages) & 1u);
        if (__syncthreads_or(!got)) {
            if (tid == 0) atomicOr(flag, kDevErrTimeout);
            break;
        }
        // phi(K) into the second MMA's A operand: elementwise, so at the same byte offsets
        for (int ch = tid; ch < static_cast<int>(2 * kBroTcAtom / 16); ch += blockDim.x) {
            const uint32_t off = static_cast<uint32_t>(ch) * 16u;
            const uint4 u = *reinterpret_cast<const uint4 *>(sK + off);
            *reinterpret_cast<uint4 *>(sP + off) = make_uint4(phi_bf16x2(u.x), phi_bf16x2(u.y), phi_bf16x2(u.z), phi_bf16x2(u.w));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t v0 = smem_u32(sV), p0 = smem_u32(sP), b10 = smem_u32(sB1), b20 = smem_u32(sB2);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t ko = static_cast<uint32_t>(ks >> 2) * kBroTcAtom, kb = static_cast<uint32_t>(ks & 3) * 32u;
                umma_bf16(tmem, smem_desc(v0 + ko + kb, 16, 1024, 2), smem_desc(b10 + ko + kb, 16, 1024, 2), idesc, ks != 0);
                umma_bf16(tmem + D, smem_desc(p0 + ko + kb, 16, 1024, 2), smem_desc(b20 + ko + kb, 16, 1024, 2), idesc,
                          ks != 0);
            }
            umma_commit(&mma_bar);
        }
        // the warp's k slice (rows rt, columns c0 .. c0 + 31) for phi'(k)
        uint4 kw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) kw[i] = *reinterpret_cast<const uint4 *>(sK + swz_off(rt, c0 + 8 * i, kBroTcAtom));
        const bool done = mbar_wait_bounded(&mma_bar, static_cast<uint32_t>(k) & 1u);
        if (__syncthreads_or(!done)) {   // also: every warp holds its k slice, the stage is free
            if (tid == 0) atomicOr(flag, kDevErrTimeout);
            break;
        }
        tc_fence_after();
        uint8_t *stg = sK + warp * kBroTcStage;
        // dk: (G_k + dz) phi'(k); dv: G_v
        const int64_t r0 = (blockIdx.x + static_cast<int64_t>(k) * gridDim.x) * 128 + quad * 32;
        // the k or v half's 32 columns of this warp: float rows of dZ, or bf16 rows of dZb
        auto put = [&](const float (&o)[16], int hb, int col0) {
            if (dZb) {
#pragma unroll
                for (int i = 0; i < 2; ++i)
                    stage_row64_piece(stg, lane, 2 * hb + i,
                                      make_uint4(bf16x2_bits(o[8 * i], o[8 * i + 1]), bf16x2_bits(o[8 * i + 2], o[8 * i + 3]),
                                                 bf16x2_bits(o[8 * i + 4], o[8 * i + 5]), bf16x2_bits(o[8 * i + 6], o[8 * i + 7])));
                if (hb == 1)
                    warp_rows64_flush(reinterpret_cast<uint8_t *>(dZb + col0 + c0), static_cast<int64_t>(3 * D) * 2, r0, N,
                                      stg, lane);
            } else {
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    stage_f32_piece(stg, lane, 4 * hb + p, o[4 * p], o[4 * p + 1], o[4 * p + 2], o[4 * p + 3]);
                if (hb == 1) warp_rows_f32_flush(dZ + col0, dz_ld, r0, N, c0, stg, lane);
            }
        };
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            uint32_t a[16];
            tmem_ld16(tmem + lane_base + static_cast<uint32_t>(c0 + 16 * hb), a);
            tmem_ld_wait();
            float o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = (__uint_as_float(a[e]) + dzf[c0 + 16 * hb + e]) * dphi(bf(kw, 16 * hb + e));
            put(o, hb, D);
        }
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            uint32_t a[16];
            tmem_ld16(tmem + lane_base + static_cast<uint32_t>(D + c0 + 16 * hb), a);
            tmem_ld_wait();
            float o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __uint_as_float(a[e]);
            put(o, hb, 2 * D);
        }
        fence_proxy_async_smem();   // the staging writes come before the stage's next TMA load
        tc_fence_before();
        __syncthreads();            // TMEM, phi(K) and the stage are free
        if (tid == 0 && k + kKvgStages < my) issue(k + kKvgStages);
    }
    // the block leaves only after its copies have landed (already so when all went well)
    if (tid == 0)
        for (int kk = k; kk < my && kk < k + kKvgStages; ++kk)
            mbar_wait_bounded(&full_bar[kk % kKvgStages], static_cast<uint32_t>(kk / kKvgStages) & 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256u);
    }
}

// bf16 layers with H*r = 128 and r <= 64: the source side's global terms run on the tensor
// cores before the gather kernels (which then get dST = nullptr and add to them).
bool kv_global_tc(const Ctx *c) {
    return c->io == GLGA_BF16 && c->D == kBroTcD && (c->r == 16 || c->r == 32 || c->r == 64);
}

template <int R>
glga_status launch_kv_global_r(Ctx *c, int64_t Dz, cudaStream_t s) {
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ceil_div(c->N, 128), c->num_sms));
    cudaFuncSetAttribute(bwd_kv_global_tc_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(kKvgSmem));
    CUtensorMap m;
    const glga_status st = encode_tmap_2d(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->KV, 2 * kBroTcD,
                                          static_cast<uint64_t>(c->N), 4 * kBroTcD, 64, 128);
    if (st != GLGA_OK) return st;
    bwd_kv_global_tc_kernel<R><<<grid, kBroTcWarps * 32, kKvgSmem, s>>>(m, c->bw_dSc, c->bw_dST, c->N, c->H, c->bw_dZ, Dz, c->bw_dZb,
                                                                       c->dev_flag);
    return GLGA_OK;
}
glga_status launch_kv_global(Ctx *c, int64_t Dz, cudaStream_t s) {
    if (!kv_global_tc(c) || c->N == 0) return GLGA_OK;
    if (c->r == 32) return launch_kv_global_r<32>(c, Dz, s);
    if (c->r == 16) return launch_kv_global_r<16>(c, Dz, s);
    return launch_kv_global_r<64>(c, Dz, s);
}

// Two rows per warp for up to 4 features per lane (one above that); the head loop
// unrolled for the lane layout of H*r = 128 with r = 32.
template <typename T, int EPL, int LPH>
void launch_readout_bwd_e(Ctx *c, const T *Q, const T *dY, float b_g, float eps, int64_t Dz, cudaStream_t s) {
    constexpr int kRpw = EPL <= 4 ? 2 : 1;
    const unsigned grid = static_cast<unsigned>(ceil_div(ceil_div(c->N, kRpw) * 32, 256));
    bwd_readout_kernel<T, EPL, LPH, kRpw><<<grid, 256, 0, s>>>(Q, static_cast<const T *>(c->L), c->t, c->Sz,
                                                               c->bw_ST, dY, c->N, c->H, c->r, b_g, eps, static_cast<T *>(c->bw_dL),
                                                               c->bw_Dd, c->bw_dnum, c->bw_dden, c->bw_dZ, Dz);
}

// The readout backward on the tensor cores (and with it dS | dz from [dnum | dden] rows):
// bf16 layers with H*r = 128, r in {16, 32, 64}, one head group.
bool readout_bwd_tc(const Ctx *c) {
    return c->io == GLGA_BF16 && c->D == kBroTcD && c->ro_groups == 1 && c->ro_kp == kBroTcD &&
           c->ro_bn == kBroTcBN && c->n_seg == 1 && (c->r == 16 || c->r == 32 || c->r == 64);
}

template <int R>
glga_status launch_readout_bwd_tc(Ctx *c, const __nv_bfloat16 *Q, const __nv_bfloat16 *dY, float b_g, float eps,
                                  int64_t Dz, cudaStream_t s) {
    const int64_t tiles = ceil_div(c->N, 128);
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, c->num_sms));
    cudaFuncSetAttribute(bwd_readout_tc_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(kBroTcSmem));
    CUtensorMap mq, my, ml;
    const uint64_t n = static_cast<uint64_t>(c->N);
    glga_status st = encode_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, kBroTcD, n, 2 * kBroTcD, 64, 128);
    if (st == GLGA_OK)
        st = encode_tmap_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, kBroTcD, n, 2 * kBroTcD, 64, 128);
    if (st == GLGA_OK)
        st = encode_tmap_2d(&ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->L, kBroTcD, n, 2 * kBroTcD, 64, 128);
    if (st != GLGA_OK) return st;
    bwd_readout_tc_kernel<R><<<grid, kBroTcWarps * 32, kBroTcSmem, s>>>(
        mq, my, ml, c->t, static_cast<const __nv_bfloat16 *>(c->Bro), c->ro_kp, c->Sz, c->N, c->H, b_g, eps,
        static_cast<__nv_bfloat16 *>(c->bw_dL), c->bw_Dd, reinterpret_cast<__nv_bfloat16 *>(c->bw_dnum), c->bw_dZ, Dz,
        c->bw_dZb, c->dev_flag);
    return GLGA_OK;
}

// The readout backward runs on the tensor cores for bf16 layers with H*r = 128, r in
// {16, 32, 64} and one head group (the forward's readout operand then holds every head);
// elsewhere on the CUDA cores.
template <typename T>
glga_status launch_readout_bwd(Ctx *c, const T *Q, const T *dY, float b_g, float eps, int64_t Dz, cudaStream_t s) {
    if constexpr (sizeof(T) == 2) {
        if (readout_bwd_tc(c)) {
            if (c->r == 32) return launch_readout_bwd_tc<32>(c, Q, dY, b_g, eps, Dz, s);
            if (c->r == 16) return launch_readout_bwd_tc<16>(c, Q, dY, b_g, eps, Dz, s);
            return launch_readout_bwd_tc<64>(c, Q, dY, b_g, eps, Dz, s);
        }
    }
    const int E = lane_features(c->D), lph = c->r / E;
    if (E == 4 && lph == 8) {
        launch_readout_bwd_e<T, 4, 8>(c, Q, dY, b_g, eps, Dz, s);
        return GLGA_OK;
    }
    switch (E) {
        case 1: launch_readout_bwd_e<T, 1, 0>(c, Q, dY, b_g, eps, Dz, s); break;
        case 2: launch_readout_bwd_e<T, 2, 0>(c, Q, dY, b_g, eps, Dz, s); break;
        case 4: launch_readout_bwd_e<T, 4, 0>(c, Q, dY, b_g, eps, Dz, s); break;
        case 8: launch_readout_bwd_e<T, 8, 0>(c, Q, dY, b_g, eps, Dz, s); break;
        case 16: launch_readout_bwd_e<T, 16, 0>(c, Q, dY, b_g, eps, Dz, s); break;
        case 32: launch_readout_bwd_e<T, 32, 0>(c, Q, dY, b_g, eps, Dz, s); break;
        default: break;
    }
    return GLGA_OK;
}


// Work lists over one CSR's offsets: light rows (at most kHeavyDegree entries) sorted by
// degree, longest first (stable), so a block's warps carry similar loads; then heavy rows
// in index order, each cut into chunks of kChunk entries (chunks[c] = {row, first entry})
// with chunk_ptr[s] .. chunk_ptr[s + 1] the chunks of heavy row s.
constexpr int64_t kHeavyDegree = 64;
struct RowPlan {
    std::vector<int32_t> rows, chunk_ptr;
    std::vector<int2> chunks;
    int64_t n_light = 0, n_heavy = 0;
};
void plan_rows(const std::vector<int32_t> &rp, RowPlan &p) {
    const int64_t n = static_cast<int64_t>(rp.size()) - 1;
    auto deg = [&](int32_t i) { return rp[i + 1] - rp[i]; };
    p.rows.clear();
    p.chunks.clear();
    p.chunk_ptr.assign(1, 0);
    for (int64_t i = 0; i < n; ++i)
        if (deg(static_cast<int32_t>(i)) <= kHeavyDegree) p.rows.push_back(static_cast<int32_t>(i));
    std::stable_sort(p.rows.begin(), p.rows.end(), [&](int32_t x, int32_t y) { return deg(x) > deg(y); });
    p.n_light = static_cast<int64_t>(p.rows.size());
    for (int64_t i = 0; i < n; ++i) {
        if (deg(static_cast<int32_t>(i)) <= kHeavyDegree) continue;
        p.rows.push_back(static_cast<int32_t>(i));
        for (int32_t e = rp[i]; e < rp[i + 1]; e += kChunk) p.chunks.push_back(make_int2(static_cast<int>(i), e));
        p.chunk_ptr.push_back(static_cast<int32_t>(p.chunks.size()));
    }
    p.n_heavy = static_cast<int64_t>(p.rows.size()) - p.n_light;
}

int64_t ceil_parts(int64_t N, int64_t want) { return std::max<int64_t>(1, std::min<int64_t>(want, N)); }

// ---------------------------------------------------------------------------------------
// Weight gradient of bf16 layers on the tcgen05 tensor cores:
//   part[p][a][k] = sum over the rows i of range p of X[i][a] dZ[i][k]   (a < d, k < 3D)
// for 128 x 128 blocks (block fa of 128 input features, block fb of 128 dZ columns); the
// node index is the contraction dimension.  Per 64-row stage a TMA producer loads the X
// tile [64][128] (bf16, two 64-column boxes, 128-byte swizzle) and the dZ tile [64][128]
// (float32, four 32-column boxes); warps 0-7 round dZ to bf16 into a third tile laid out
// as TMA lays out bf16 (rows past the range are zeroed); one thread issues tcgen05.mma
// with both operands MN-major (X^T as A, the bf16 dZ tile as B), accumulating the block
// in TMEM over the range in row order.  Warps 0-3 write the block to the range's partial
// sums, which bwd_sum_parts_kernel adds in range order (the result is the same on every
// call).  Every mbarrier wait is bounded: on expiry the kernel raises the context's flag,
// lets its copies land and returns.
constexpr int kDwRows = 64;
constexpr int kDwStages = 3;
constexpr int kDwWorkers = 256;
constexpr int kDwProd = 8, kDwMma = 9, kDwThreads = 320;
constexpr uint32_t kDwBox = kDwRows * 128;                 // one 64-row box of 128-byte rows
constexpr uint32_t kDwXBytes = 2 * kDwBox;                 // X tile (bf16)
constexpr uint32_t kDwZBytes = 4 * kDwBox;                 // dZ tile (float32)
constexpr uint32_t kDwStage = kDwXBytes + kDwZBytes + 2 * kDwBox;   // + dZ rounded to bf16
// the dS | dz form: bf16 [dnum | dden] rows of 144 columns loaded by TMA straight into a B
// tile of three 64-column atoms (columns 144 .. 191 past the rows' end read as zero); four
// stages
constexpr int kDszStages = 4;
constexpr uint32_t kDszZBytes = 0;
constexpr uint32_t kDszStage = kDwXBytes + 3 * kDwBox;
static_assert(kDszStage % 1024 == 0, "1024-byte aligned tiles");

struct DwParams {
    int64_t N;
    int32_t d, Kc;            // X columns; dZ columns in use (3D)
    int64_t rows_per_part;
    float *part;              // [P][d][Kc]
    unsigned *flag;
    int32_t H, R;             // DSZ: heads and head width
};

// With DSZ the same kernel forms the readout's dS | dz partials: X = Q with phi applied to
// each landed tile, dZ = [dnum | dden] (bf16 rows of D + 16 columns, dden_h in column
// D + h, loaded as the B operand itself: the ranges are whole 64-row tiles, so no row
// needs zeroing), one M = 128, N = 144 MMA per 16 rows, and the epilogue keeps the
// diagonal head blocks and the dden column in the layout [P][H][R][R + 1] (column R = dz)
// that bwd_sum_parts_kernel adds.
template <bool DSZ>
__global__ void __launch_bounds__(kDwThreads, 1) bwd_dw_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                                                                  const __grid_constant__ CUtensorMap tmZ,
                                                                  DwParams p) {
    constexpr int kStages = DSZ ? kDszStages : kDwStages;
    constexpr uint32_t kZBytes = DSZ ? kDszZBytes : kDwZBytes;
    constexpr uint32_t kStageBytes = DSZ ? kDszStage : kDwStage;
    constexpr int kNCols = DSZ ? 144 : 128;                   // MMA N
    constexpr uint32_t kTmemCols = DSZ ? 256u : 128u;
    extern __shared__ uint8_t dsmem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t ready_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_base_sh;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = blockIdx.x, fa = blockIdx.y, fb = blockIdx.z;
    const int64_t r0 = static_cast<int64_t>(part) * p.rows_per_part;
    const int64_t r1 = std::min<int64_t>(p.N, r0 + p.rows_per_part);
    const int ntiles = r1 > r0 ? static_cast<int>(ceil_div(r1 - r0, kDwRows)) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&ready_bar[s], kDwWorkers / 32);   // one arrival per worker warp
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&done_bar, 1);
        fence_mbar_init();
    }
    if (warp == kDwMma) {
        tmem_alloc(&tmem_base_sh, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kDwProd) {
        if (lane == 0) {
            tma_prefetch_desc(&tmX);
            tma_prefetch_desc(&tmZ);
            int issued = 0;
            RingPos rp;
            bool ok = true;
            for (int it = 0; it < ntiles; ++it, rp.next(kStages)) {
                const int s = rp.slot;
                if (it >= kStages && !mbar_wait_bounded(&empty_bar[s], rp.phase ^ 1u)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + static_cast<size_t>(s) * kStageBytes;
                const int32_t y = static_cast<int32_t>(r0 + static_cast<int64_t>(it) * kDwRows);
                if constexpr (DSZ) {
                    mbar_arrive_expect_tx(&full_bar[s], kDszStage);
                    for (int b = 0; b < 2; ++b) tma_load_2d(st + b * kDwBox, &tmX, &full_bar[s], b * 64, y);
                    for (int b = 0; b < 3; ++b) tma_load_2d(st + kDwXBytes + b * kDwBox, &tmZ, &full_bar[s], b * 64, y);
                } else {
                    mbar_arrive_expect_tx(&full_bar[s], kDwXBytes + kZBytes);
                    for (int b = 0; b < 2; ++b)
                        tma_load_2d(st + b * kDwBox, &tmX, &full_bar[s], fa * 128 + b * 64, y);
                    for (int b = 0; b < 4; ++b)
                        tma_load_2d(st + kDwXBytes + b * kDwBox, &tmZ, &full_bar[s], fb * 128 + b * 32, y);
                }
                ++issued;
            }
            if (!ok) {
                atomicOr(p.flag, kDevErrTimeout);
                for (int it = std::max(0, issued - kStages); it < issued; ++it)
                    mbar_wait_bounded(&full_bar[it % kStages], static_cast<uint32_t>(it / kStages) & 1u);
            }
        }
    } else if (warp == kDwMma) {
        if (lane == 0) {
            const uint32_t idesc = instr_desc(128, kNCols, 1u, true, true);
            bool ok = true;
            RingPos rp;
            for (int it = 0; it < ntiles; ++it, rp.next(kStages)) {
                const int s = rp.slot;
                if (!mbar_wait_bounded(&ready_bar[s], rp.phase)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t xb = smem_u32(smem + static_cast<size_t>(s) * kStageBytes);
                const uint32_t bb = xb + kDwXBytes + kZBytes;
#pragma unroll
                for (int ks = 0; ks < kDwRows / 16; ++ks) {
                    const uint32_t off = ks * 16 * 128;
                    umma_bf16(tmem, smem_desc(xb + off, kDwBox, 1024, 2), smem_desc(bb + off, kDwBox, 1024, 2),
                              idesc, (it | ks) != 0);
                }
                umma_commit(&empty_bar[s]);
            }
            if (!ok) atomicOr(p.flag, kDevErrTimeout);
            umma_commit(&done_bar);
        }
    } else {
        // ---------------- warps 0-7: dZ float32 -> bf16 (zero past the range) ----------
        bool ok = true;
        RingPos rp;
        for (int it = 0; it < ntiles && ok; ++it, rp.next(kStages)) {
            const int s = rp.slot;
            // the warp agrees on the outcome, so it stays converged for its arrival
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[s], rp.phase))) {
                ok = false;
                break;
            }
            const uint8_t *z = smem + static_cast<size_t>(s) * kStageBytes + kDwXBytes;
            uint8_t *bt = smem + static_cast<size_t>(s) * kStageBytes + kDwXBytes + kZBytes;
            const int64_t y0 = r0 + static_cast<int64_t>(it) * kDwRows;
            if constexpr (DSZ) {
                // phi of the q tile in place (rows past N are zero in both tiles)
                uint4 *xq = reinterpret_cast<uint4 *>(smem + static_cast<size_t>(s) * kStageBytes);
                for (int cidx = threadIdx.x; cidx < static_cast<int>(kDwXBytes / 16); cidx += kDwWorkers) {
                    const uint4 u = xq[cidx];
                    xq[cidx] = make_uint4(phi_bf16x2(u.x), phi_bf16x2(u.y), phi_bf16x2(u.z), phi_bf16x2(u.w));
                }
            }
            // one 16-byte chunk of the bf16 tile (8 consecutive columns of one row) per step
            for (int cidx = threadIdx.x; !DSZ && cidx < kDwRows * 16; cidx += kDwWorkers) {
                const int k = cidx >> 4, ch = cidx & 15;
                const int bo = ch >> 3, co = ch & 7;            // bf16 box, chunk in its row
                const int g0 = bo * 64 + co * 8;                // first column in the tile
                const int bi = g0 >> 5, j0 = (g0 & 31) >> 2;    // float32 box, its first chunk
                uint4 w = make_uint4(0, 0, 0, 0);
                if (y0 + k < r1) {
                    const uint8_t *zr = z + bi * kDwBox + k * 128;
                    const float4 a = *reinterpret_cast<const float4 *>(zr + ((j0 ^ (k & 7)) * 16));
                    const float4 b = *reinterpret_cast<const float4 *>(zr + (((j0 + 1) ^ (k & 7)) * 16));
                    __nv_bfloat162 h0 = __floats2bfloat162_rn(a.x, a.y), h1 = __floats2bfloat162_rn(a.z, a.w);
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(b.x, b.y), h3 = __floats2bfloat162_rn(b.z, b.w);
                    w = make_uint4(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1),
                                   *reinterpret_cast<uint32_t *>(&h2), *reinterpret_cast<uint32_t *>(&h3));
                }
                *reinterpret_cast<uint4 *>(bt + bo * kDwBox + k * 128 + ((co ^ (k & 7)) * 16)) = w;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready_bar[s]);
        }
        if (!ok && lane == 0) atomicOr(p.flag, kDevErrTimeout);
    }
    __syncwarp();

    if (warp < 4) {
        // ---------------- epilogue: the 128 x 128 block -> the range's partial sums ---------
        const bool done = ntiles == 0 ? true : mbar_wait_bounded(&done_bar, 0);
        tc_fence_after();
        if (!done && lane == 0) atomicOr(p.flag, kDevErrTimeout);
        const bool have = ntiles > 0 && done;
        const int a = fa * 128 + warp * 32 + lane;         // TMEM lane = input feature
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        if constexpr (DSZ) {
            // feature a = h R + al: its head's block row (columns h R ..) and its dz (column D + h)
            const int h = a / p.R, al = a - h * p.R;
            float *dst = p.part + ((static_cast<int64_t>(part) * p.H + h) * p.R + al) * (p.R + 1);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + q * 32, v);
                tmem_ld_wait();
                if (a < p.d) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = q * 32 + j;
                        if (col / p.R == h) dst[col - h * p.R] = have ? __uint_as_float(v[j]) : 0.f;
                    }
                }
            }
            uint32_t v[16];
            tmem_ld16(tmem + lane_base + p.d, v);
            tmem_ld_wait();
            float dz = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (j == h) dz = __uint_as_float(v[j]);
            if (a < p.d) dst[p.R] = have ? dz : 0.f;
        } else {
        float *dst = p.part + (static_cast<int64_t>(part) * p.d + a) * p.Kc;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + q * 32, v);
            tmem_ld_wait();
            const int k0 = fb * 128 + q * 32;
            if (a < p.d) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (k0 + j < p.Kc) dst[k0 + j] = have ? __uint_as_float(v[j]) : 0.f;
            }
        }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kDwMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Whether the bf16 tensor-core GEMMs serve this context's backward: bf16 layers whose X
// rows are 16-byte multiples (TMA).  Other layers keep the CUDA-core GEMM kernels.
bool bwd_tc_gemms(const Ctx *c) { return c->io == GLGA_BF16 && c->d % 8 == 0 && c->N > 0; }

// dW (columns < 3D) and dX of a bf16 layer on the tensor cores:
//   dW3 [d][3D] = sum of the range partials of bwd_dw_tc_kernel, in range order;
//   dX [N][d] = dZ [N][3D + 1] Wall^T, the persistent GEMM on kind::tf32 (fp32 dZ and
//   Wall read as tf32).
glga_status tc_gemms(Ctx *c, const void *X, float *dX, cudaStream_t s) {
    const int64_t N = c->N;
    const int d = c->d, D = c->D, Kc = 3 * D;
    CUtensorMap mx, mz;
    glga_status st = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(d),
                                    static_cast<uint64_t>(N), static_cast<uint64_t>(d) * 2, 64, kDwRows);
    if (st == GLGA_OK)
        st = encode_tmap_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, c->bw_dZ, static_cast<uint64_t>(Kc),
                            static_cast<uint64_t>(N), static_cast<uint64_t>(c->bw_dz_ld) * 4, 32, kDwRows);
    if (st != GLGA_OK) return st;
    DwParams p;
    p.N = N;
    p.d = d;
    p.Kc = Kc;
    p.rows_per_part = c->bw_dwtc_rpp;
    p.part = c->bw_dwtc_part;
    p.flag = c->dev_flag;
    p.H = p.R = 0;
    const size_t smem = static_cast<size_t>(kDwStages) * kDwStage + 1024;
    GLGA_CUDA(cudaFuncSetAttribute(bwd_dw_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem)));
    const dim3 grid(static_cast<unsigned>(c->bw_dwtc_parts), static_cast<unsigned>(ceil_div(d, 128)),
                    static_cast<unsigned>(ceil_div(Kc, 128)));
    bwd_dw_tc_kernel<false><<<grid, kDwThreads, smem, s>>>(mx, mz, p);
    GLGA_CUDA(cudaGetLastError());
    const int64_t total = static_cast<int64_t>(d) * Kc;
    bwd_sum_parts_kernel<<<sum_parts_grid(total), kSumThreads, 0, s>>>(
        c->bw_dwtc_part, c->bw_dwtc_parts, total, c->bw_dW3);
    GLGA_CUDA(cudaGetLastError());
    return gemm_nt_f32out(c, GLGA_F32, c->bw_dZ, N, c->bw_dz_ld, c->bw_Wall, d, c->bw_dz_ld, Kc + 1, dX, d, s);
}

// ---------------------------------------------------------------------------------------
// dX, dW, dw_g and db_g of a bf16 layer with d = 128 in one pass over dZ (tcgen05):
//   dX[i][a] = sum_k dZ[i][k] W[a][k] + dt_i w_g[a]            (W = [W_Q | W_K | W_V])
//   dW[a][k] = sum_i X[i][a] dZ[i][k],  dw_g[a] = sum_i X[i][a] dt_i,  db_g = sum_i dt_i
// dZ's columns 0 .. 3D - 1 come as the bf16 copy the gather kernels write with their
// final values (dZb [N][3D]); dt stays in the float dZ.  A persistent grid: thread block
// b takes the 128-row tiles b, b + G, ...  Per tile one producer thread loads by TMA the
// X tile (two [128][64] bf16 boxes) with dt (a [128][4] float box at column 3D), then per
// 64-column chunk the [128][64] bf16 dZ box and the [128 a][64 k] block of W it
// multiplies, into a four-stage ring.  One thread issues per chunk the dX MMAs (the dZ
// chunk K-major as A, the W block K-major as B: M = 128 rows, N = 128 features) into
// TMEM columns 0-127 and the dW MMAs (X^T MN-major as A, the dZ chunk MN-major as B:
// M = 128 features, N = 64) into the chunk's columns of a [128][3D] accumulator that stays
// in TMEM over all the block's tiles.  Warps 0-7 add X^T dt and the sum of dt on the CUDA
// cores; warps 10-13 drain dX per tile (adding dt w_g) through a staging area into
// coalesced row stores, and after the last tile write the block's dW partial sums; the
// range-order reductions add the blocks' partials (the result is the same on every call).
// Every wait is bounded: on expiry the kernel raises the context's flag, lets its copies
// land, waits for its MMAs and returns.
constexpr int kFxRows = 128;
constexpr int kFxXStages = 2, kFxBStages = 4;
constexpr uint32_t kFxBox = kFxRows * 128;                  // a [128][128 B] box: 16 KB
constexpr uint32_t kFxXStage = 2 * kFxBox + kFxRows * 16;   // X tile, then the dt box
constexpr uint32_t kFxBStage = 2 * kFxBox;                  // bf16 dZ chunk, then the W block
constexpr uint32_t kFxEpi = kFxXStages * kFxXStage + kFxBStages * kFxBStage;
constexpr uint32_t kFxEpiStage = 4096;                      // per epilogue warp
constexpr size_t kFxSmem = 1024 + kFxEpi + 4 * kFxEpiStage + (128 + 256 + 2) * sizeof(float);
constexpr int kFxWorkers = 256, kFxProd = 8, kFxMma = 9, kFxEpi0 = 10, kFxThreads = 448;
static_assert(kFxXStage % 1024 == 0 && kFxEpi % 1024 == 0, "stages stay 1024-byte aligned");

struct FxParams {
    int64_t N;
    int32_t D, Kc, ntiles;          // W blocks of D columns; 3D dZ columns; 128-row tiles
    const __nv_bfloat16 *wg;        // [128]
    float *dX;                      // [N][128]
    float *dw_part;                 // [P][128][3D]
    float *g_part;                  // [P][128][3D + 1]: column 3D holds dw_g
    float *b_part;                  // [P]
    unsigned *flag;
};

__global__ void __launch_bounds__(kFxThreads, 1) bwd_dxdw_tc_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmZ,
    const __grid_constant__ CUtensorMap tmDt, const __grid_constant__ CUtensorMap tmWq,
    const __grid_constant__ CUtensorMap tmWk, const __grid_constant__ CUtensorMap tmWv, FxParams p) {
    extern __shared__ uint8_t dsmem_raw[];
    __shared__ __align__(8) uint64_t x_full[kFxXStages], x_empty[kFxXStages];
    __shared__ __align__(8) uint64_t b_full[kFxBStages], b_empty[kFxBStages];
    __shared__ __align__(8) uint64_t dx_full, dx_empty, mma_done;
    __shared__ uint32_t tmem_base_sh;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sX = smem;                                      // [kFxXStages] X tile + dt
    uint8_t *sB = sX + kFxXStages * kFxXStage;               // [kFxBStages] dZ chunk + W block
    uint8_t *sE = smem + kFxEpi;                             // epilogue staging
    float *swg = reinterpret_cast<float *>(sE + 4 * kFxEpiStage);   // w_g as float
    float *sred = swg + 128;                                 // [256] + [2] worker sums
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, blk = blockIdx.x;
    const int my = blk < p.ntiles ? (p.ntiles - 1 - blk) / G + 1 : 0;   // this block's tiles
    const int nc = p.Kc / 64, cpm = p.D / 64;               // chunks per tile, per W matrix

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFxXStages; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1 + kFxWorkers / 32 + 4);   // MMA commit, workers, epilogue
        }
        for (int s = 0; s < kFxBStages; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        mbar_init(&dx_full, 1);
        mbar_init(&dx_empty, 4);
        mbar_init(&mma_done, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 128) swg[threadIdx.x] = __bfloat162float(p.wg[threadIdx.x]);
    if (warp == kFxMma) {
        tmem_alloc(&tmem_base_sh, 512u);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kFxProd) {
        if (lane == 0) {
            tma_prefetch_desc(&tmX);
            tma_prefetch_desc(&tmZ);
            bool ok = true;
            int nx = 0, nb = 0;                                  // loads issued per ring
            for (int j = 0; j < my && ok; ++j) {
                const int32_t y = (blk + j * G) * kFxRows;
                const int xs = nx % kFxXStages;
                if (nx >= kFxXStages && !mbar_wait_bounded(&x_empty[xs], ((nx / kFxXStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                uint8_t *xst = sX + xs * kFxXStage;
                mbar_arrive_expect_tx(&x_full[xs], kFxXStage);
                tma_load_2d(xst, &tmX, &x_full[xs], 0, y);
                tma_load_2d(xst + kFxBox, &tmX, &x_full[xs], 64, y);
                tma_load_2d(xst + 2 * kFxBox, &tmDt, &x_full[xs], p.Kc, y);
                ++nx;
                for (int cc = 0; cc < nc; ++cc) {
                    const int bs = nb % kFxBStages;
                    if (nb >= kFxBStages && !mbar_wait_bounded(&b_empty[bs], ((nb / kFxBStages) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    const CUtensorMap *wm = cc < cpm ? &tmWq : (cc < 2 * cpm ? &tmWk : &tmWv);
                    uint8_t *bst = sB + bs * kFxBStage;
                    mbar_arrive_expect_tx(&b_full[bs], kFxBStage);
                    tma_load_2d(bst, &tmZ, &b_full[bs], cc * 64, y);
                    tma_load_2d(bst + kFxBox, wm, &b_full[bs], (cc % cpm) * 64, 0);
                    ++nb;
                }
            }
            if (!ok) atomicOr(p.flag, kDevErrTimeout);
            // the block leaves only after its copies have landed (already so when all went well)
            for (int i = std::max(0, nx - kFxXStages); i < nx; ++i)
                mbar_wait_bounded(&x_full[i % kFxXStages], (i / kFxXStages) & 1);
            for (int i = std::max(0, nb - kFxBStages); i < nb; ++i)
                mbar_wait_bounded(&b_full[i % kFxBStages], (i / kFxBStages) & 1);
        }
    } else if (warp == kFxMma) {
        if (lane == 0) {
            const uint32_t id_dx = instr_desc(128, 128, 1u, false, false);
            const uint32_t id_dw = instr_desc(128, 64, 1u, true, true);
            bool ok = true;
            int nb = 0;
            for (int j = 0; j < my && ok; ++j) {
                const int xs = j % kFxXStages;
                if (!mbar_wait_bounded(&x_full[xs], (j / kFxXStages) & 1) ||
                    (j > 0 && !mbar_wait_bounded(&dx_empty, (j - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t xa = smem_u32(sX + xs * kFxXStage);
                for (int cc = 0; cc < nc; ++cc, ++nb) {
                    const int bs = nb % kFxBStages;
                    if (!mbar_wait_bounded(&b_full[bs], static_cast<uint32_t>(nb / kFxBStages) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t zb = smem_u32(sB + bs * kFxBStage), wb = zb + kFxBox;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)        // dX += dZ chunk (K-major) W block^T
                        umma_bf16(tmem, smem_desc(zb + ks * 32, 16, 1024, 2), smem_desc(wb + ks * 32, 16, 1024, 2),
                                  id_dx, (cc | ks) != 0);
#pragma unroll
                    for (int ks = 0; ks < kFxRows / 16; ++ks)   // dW chunk += X^T dZ chunk
                        umma_bf16(tmem + 128 + cc * 64, smem_desc(xa + ks * 2048, kFxBox, 1024, 2),
                                  smem_desc(zb + ks * 2048, kFxBox, 1024, 2), id_dw, (j | ks) != 0);
                    umma_commit(&b_empty[bs]);
                }
                if (!ok) break;
                umma_commit(&x_empty[xs]);
                umma_commit(&dx_full);
            }
            if (!ok) atomicOr(p.flag, kDevErrTimeout);
            umma_commit(&mma_done);
        }
    } else if (warp < kFxWorkers / 32) {
        // ---------------- warps 0-7: X^T dt and the sum of dt ----------------------------
        const int t = threadIdx.x, fa = t & 127, hh = t >> 7;   // feature, half of the tile's rows
        bool ok = true;
        float accg = 0.f, accb = 0.f;
        for (int j = 0; j < my && ok; ++j) {
            const int xs = j % kFxXStages;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&x_full[xs], (j / kFxXStages) & 1))) {
                ok = false;
                break;
            }
            const uint8_t *xt = sX + xs * kFxXStage + (fa >> 6) * kFxBox;
            const float *dt = reinterpret_cast<const float *>(sX + xs * kFxXStage + 2 * kFxBox);
            const int cb = (fa & 63) >> 3, wi = (fa & 7) * 2;   // 16-byte chunk in the row, byte in it
            for (int r = hh * 64; r < hh * 64 + 64; ++r) {
                const float x = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16 *>(xt + r * 128 + ((cb ^ (r & 7)) << 4) + wi));
                const float dv = dt[r * 4];
                accg = fmaf(x, dv, accg);
                accb += dv;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&x_empty[xs]);
        }
        if (!ok && lane == 0) atomicOr(p.flag, kDevErrTimeout);
        // the two row halves of each feature, added in a fixed order
        sred[t] = accg;
        if (t == 0 || t == 128) sred[256 + hh] = accb;
        asm volatile("bar.sync 1, %0;" ::"n"(kFxWorkers) : "memory");
        if (t < 128)
            p.g_part[(static_cast<int64_t>(blk) * 128 + t) * (p.Kc + 1) + p.Kc] = sred[t] + sred[t + 128];
        if (t == 0) p.b_part[blk] = sred[256] + sred[257];
    } else if (warp >= kFxEpi0) {
        // ---------------- warps 10-13: dX per tile, then the block's dW ---------------------
        const int qw = warp & 3;                              // TMEM lane quarter
        uint8_t *stg = sE + (warp - kFxEpi0) * kFxEpiStage;
        const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
        bool ok = true;
        for (int j = 0; j < my && ok; ++j) {
            const int xs = j % kFxXStages;
            const bool got = mbar_wait_bounded(&dx_full, j & 1) && mbar_wait_bounded(&x_full[xs], (j / kFxXStages) & 1);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int64_t r0 = static_cast<int64_t>(blk + j * G) * kFxRows + qw * 32;
            const float dv = reinterpret_cast<const float *>(sX + xs * kFxXStage + 2 * kFxBox)[(qw * 32 + lane) * 4];
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + q * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int pc = 0; pc < 8; ++pc) {
                    const float *g = swg + q * 32 + pc * 4;
                    stage_f32_piece(stg, lane, pc, fmaf(dv, g[0], __uint_as_float(v[4 * pc])),
                                    fmaf(dv, g[1], __uint_as_float(v[4 * pc + 1])),
                                    fmaf(dv, g[2], __uint_as_float(v[4 * pc + 2])),
                                    fmaf(dv, g[3], __uint_as_float(v[4 * pc + 3])));
                }
                warp_rows_f32_flush(p.dX, 128, r0, p.N, q * 32, stg, lane);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&dx_empty);
                mbar_arrive(&x_empty[xs]);
            }
        }
        if (!ok && lane == 0) atomicOr(p.flag, kDevErrTimeout);
        if (ok && my > 0) {
            // the last tile's dX commit covers every MMA of the block: dW is complete
            float *dst = p.dw_part + static_cast<int64_t>(blk) * 128 * p.Kc;
#pragma unroll 1
            for (int q = 0; q < p.Kc / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + 128 + q * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int pc = 0; pc < 8; ++pc)
                    stage_f32_piece(stg, lane, pc, __uint_as_float(v[4 * pc]), __uint_as_float(v[4 * pc + 1]),
                                    __uint_as_float(v[4 * pc + 2]), __uint_as_float(v[4 * pc + 3]));
                warp_rows_f32_flush(dst, p.Kc, qw * 32, 128, q * 32, stg, lane);
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kFxMma) {
        // every MMA issued has completed before the columns are freed
        if (lane == 0 && !mbar_wait_bounded(&mma_done, 0)) atomicOr(p.flag, kDevErrTimeout);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512u);
    }
}

// Whether dX and the weight gradients of this context take the one-pass kernel: bf16
// layers with d = 128 whose readout backward and source-side global terms run on the
// tensor cores (H*r = 128, r in {16, 32, 64}, one head group): dX and dW fit TMEM
// together, and dZ's columns 0 .. 3D - 1 live in bf16 (dZb) from the start: the two
// tensor-core kernels write the global parts there and the gather kernels (light rows two
// edges per step, heavy rows chunk sums) add the local parts in place.
bool bwd_fx(const Ctx *c) {
    return c->io == GLGA_BF16 && c->d == 128 && kv_global_tc(c) && readout_bwd_tc(c) && c->N > 0;
}

// dX, and the dW / dw_g / db_g partials that the reductions after it add
// (over c->bw_fx_parts blocks), in one pass over dZ.
glga_status fx_gemms(Ctx *c, const void *X, const void *WQ, const void *WK, const void *WV, const void *wg,
                     float *dX, cudaStream_t s) {
    const int64_t N = c->N, D = c->D, Kc = 3 * D;
    const uint64_t zrow = static_cast<uint64_t>(c->bw_dz_ld) * 4;
    CUtensorMap mx, mz, mdt, mq, mk, mv;
    glga_status st = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, 128, static_cast<uint64_t>(N), 256,
                                    64, kFxRows);
    if (st == GLGA_OK)
        st = encode_tmap_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->bw_dZb, static_cast<uint64_t>(Kc),
                            static_cast<uint64_t>(N), static_cast<uint64_t>(Kc) * 2, 64, kFxRows);
    if (st == GLGA_OK)
        st = encode_tmap_2d(&mdt, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, c->bw_dZ, static_cast<uint64_t>(c->bw_dz_ld),
                            static_cast<uint64_t>(N), zrow, 4, kFxRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    const void *wm[3] = {WQ, WK, WV};
    CUtensorMap *mw[3] = {&mq, &mk, &mv};
    for (int m = 0; m < 3 && st == GLGA_OK; ++m)
        st = encode_tmap_2d(mw[m], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, wm[m], static_cast<uint64_t>(D), 128,
                            static_cast<uint64_t>(D) * 2, 64, 128);
    if (st != GLGA_OK) return st;
    FxParams p;
    p.N = N;
    p.D = static_cast<int32_t>(D);
    p.Kc = static_cast<int32_t>(Kc);
    p.ntiles = static_cast<int32_t>(ceil_div(N, kFxRows));
    p.wg = static_cast<const __nv_bfloat16 *>(wg);
    p.dX = dX;
    p.dw_part = c->bw_dwtc_part;
    p.g_part = c->bw_dw_part;
    p.b_part = c->bw_dbg_part;
    p.flag = c->dev_flag;
    GLGA_CUDA(cudaFuncSetAttribute(bwd_dxdw_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(kFxSmem)));
    bwd_dxdw_tc_kernel<<<static_cast<unsigned>(c->bw_fx_parts), kFxThreads, kFxSmem, s>>>(mx, mz, mdt, mq, mk, mv, p);
    GLGA_CUDA(cudaGetLastError());
    const int64_t total = 128 * Kc;
    bwd_sum_parts_kernel<<<sum_parts_grid(total), kSumThreads, 0, s>>>(
        c->bw_dwtc_part, c->bw_fx_parts, total, c->bw_dW3);
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

// dS | dz partials over c->bw_dsz_parts row ranges of c->bw_dsz_rpp rows.
template <typename T>
glga_status launch_dsz_bwd(Ctx *c, const T *Q, cudaStream_t s) {
    const int64_t rpp = c->bw_dsz_rpp;
    if constexpr (sizeof(T) == 2) {
        if (readout_bwd_tc(c)) {
            // tcgen05: X = Q [N][D] (phi applied per tile), dZ = bf16 [dnum | dden] [N][D + 16]
            const int64_t N = c->N, D = c->D;
            CUtensorMap mx, mz;
            glga_status st = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, static_cast<uint64_t>(D),
                                            static_cast<uint64_t>(N), static_cast<uint64_t>(D) * 2, 64, kDwRows);
            if (st == GLGA_OK)
                st = encode_tmap_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->bw_dnum, static_cast<uint64_t>(D + 16),
                                    static_cast<uint64_t>(N), static_cast<uint64_t>(D + 16) * 2, 64, kDwRows);
            if (st != GLGA_OK) return st;
            DwParams p;
            p.N = N;
            p.d = static_cast<int32_t>(D);
            p.Kc = static_cast<int32_t>(D + 16);
            p.rows_per_part = rpp;
            p.part = c->bw_dsz_part;
            p.flag = c->dev_flag;
            p.H = c->H;
            p.R = c->r;
            const size_t smem = static_cast<size_t>(kDszStages) * kDszStage + 1024;
            GLGA_CUDA(cudaFuncSetAttribute(bwd_dw_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem)));
            bwd_dw_tc_kernel<true><<<static_cast<unsigned>(c->bw_dsz_parts), kDwThreads, smem, s>>>(mx, mz, p);
            GLGA_CUDA(cudaGetLastError());
            return GLGA_OK;
        }
    }
    const dim3 grid(static_cast<unsigned>(c->bw_dsz_parts), static_cast<unsigned>(c->H));
    const int R = c->r, tiles = (R / 4) * (R / 4), G = tiles >= 256 ? 1 : 256 / tiles;
    const size_t smem = (2 * 32 * R + 32 + (G > 1 ? static_cast<size_t>(G) * R * (R + 1) : 0)) * sizeof(float);
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
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

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
    c->bw_dz_ld = ceil_div(3 * D + 1, 4) * 4;        // rows start on 16 bytes (float4 GEMM loads)
    c->bw_parts = static_cast<int32_t>(ceil_parts(N, c->num_sms));
    const int64_t tiles = ceil_div(c->d, kGT) * ceil_div(3 * D, kGT);
    c->bw_wparts = static_cast<int32_t>(ceil_parts(N, std::max<int64_t>(1, 2 * c->num_sms / tiles)));
    const size_t f = sizeof(float);
    const int64_t nz = std::max<int64_t>(N, 1);
    glga_status st = GLGA_OK;
#define BTRY(x) \
    if (st == GLGA_OK) st = (x)
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->t_row_ptr), (N + 1) * sizeof(int32_t)));
    if (st == GLGA_OK) {
        cudaError_t e = cudaStreamCreateWithFlags(&c->bw_side, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->bw_ev_fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->bw_ev_join, cudaEventDisableTiming);
        if (e != cudaSuccess) st = cuda_fail(e, "backward side stream");
    }
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->t_col), std::max<int64_t>(E, 1) * sizeof(int32_t)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dL), nz * D * c->elem));
    // bf16 [dnum | dden] rows of D + 16 columns (dden_h in column D + h) for the tensor-core
    // dS | dz; float dnum rows of D columns and dden [N, H] on the other paths
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dnum), nz * (D + 16) * f));
    if (st == GLGA_OK) {
        const cudaError_t e = cudaMemsetAsync(c->bw_dnum, 0, nz * (D + 16) * f, s);
        if (e != cudaSuccess) st = cuda_fail(e, "backward buffers");
    }
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dden), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_lse), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_Dd), nz * H * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dZ), nz * c->bw_dz_ld * f));
    if (readout_bwd_tc(c)) {
        // 64-row-aligned ranges, one thread block per SM
        c->bw_dsz_rpp = ceil_div(ceil_div(N, std::max<int64_t>(1, c->num_sms)), kDwRows) * kDwRows;
    } else {
        c->bw_dsz_rpp = ceil_div(std::max<int64_t>(N, 1), c->bw_parts);
    }
    c->bw_dsz_parts = static_cast<int32_t>(std::max<int64_t>(1, ceil_div(std::max<int64_t>(N, 1), c->bw_dsz_rpp)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dsz_part),
                   static_cast<size_t>(c->bw_dsz_parts) * H * R * (R + 1) * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dSz), static_cast<size_t>(H) * R * (R + 1) * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_ST), static_cast<size_t>(H) * R * R * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dST), static_cast<size_t>(H) * R * R * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dSc), static_cast<size_t>(H) * R * (R + 1) * f));
    // the one-pass dX / dW kernel: one thread block per SM, each with at least one row tile
    c->bw_fx_parts = bwd_fx(c) ? static_cast<int32_t>(std::min<int64_t>(c->num_sms, ceil_div(N, kFxRows))) : 0;
    if (bwd_fx(c))   // the bf16 copy of dZ's columns 0 .. 3D - 1 it reads
        BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dZb), nz * 3 * D * sizeof(__nv_bfloat16)));
    const int64_t gparts = std::max<int64_t>(c->bw_wparts, c->bw_fx_parts);
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dw_part),
                   static_cast<size_t>(gparts) * c->d * (3 * D + 1) * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dbg_part), static_cast<size_t>(gparts) * f));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_Wall), static_cast<size_t>(c->d) * c->bw_dz_ld * f));
    if (bwd_tc_gemms(c)) {
        // weight-gradient partials of the tensor-core GEMM: 64-row-aligned ranges, about
        // one thread block per SM over the (feature block, column block) grid
        const int64_t blocks = ceil_div(c->d, 128) * ceil_div(3 * D, 128);
        const int64_t want = std::max<int64_t>(1, c->num_sms / blocks);
        const int64_t rpp = ceil_div(ceil_div(N, want), kDwRows) * kDwRows;
        c->bw_dwtc_rpp = rpp;
        c->bw_dwtc_parts = static_cast<int32_t>(ceil_div(N, rpp));
        BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dwtc_part),
                       static_cast<size_t>(std::max(c->bw_dwtc_parts, c->bw_fx_parts)) * c->d * 3 * D * f));
        BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_dW3), static_cast<size_t>(c->d) * 3 * D * f));
    }
#undef BTRY
    if (st != GLGA_OK) return st;
    // dZ's padding columns (3D + 1 .. dz_ld - 1) are never written: zero them once
    GLGA_CUDA(cudaMemset(c->bw_dZ, 0, static_cast<size_t>(nz) * c->bw_dz_ld * f));
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
    std::vector<int32_t> rp(static_cast<size_t>(N) + 1), trp(static_cast<size_t>(N) + 1);
    GLGA_CUDA(cudaMemcpy(rp.data(), c->row_ptr, rp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost));
    GLGA_CUDA(cudaMemcpy(trp.data(), c->t_row_ptr, trp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost));
    RowPlan qp, kp;
    plan_rows(rp, qp);
    plan_rows(trp, kp);
    // the hand-over of each edge's (p, ds) from the target side to the source side (bf16
    // layers on the two-edges-per-step kernels): perm maps a forward CSR entry to its
    // position in the transposed CSR (a source row's entries in target order, ties in
    // entry order), checked entry by entry against the transposed CSR; without a match
    // the source side recomputes p and ds
    if (kv_global_tc(c) && E > 0) {
        std::vector<int32_t> ci(static_cast<size_t>(E)), tci(static_cast<size_t>(E)), perm(static_cast<size_t>(E));
        GLGA_CUDA(cudaMemcpy(ci.data(), c->col_idx, ci.size() * sizeof(int32_t), cudaMemcpyDeviceToHost));
        GLGA_CUDA(cudaMemcpy(tci.data(), c->t_col, tci.size() * sizeof(int32_t), cudaMemcpyDeviceToHost));
        std::vector<int32_t> cur(trp.begin(), trp.end() - 1);
        bool match = true;
        for (int64_t i = 0; i < N && match; ++i) {
            for (int32_t e = rp[i]; e < rp[i + 1]; ++e) {
                const int32_t j = ci[e];
                if (j < 0 || j >= N || cur[j] >= trp[j + 1] || tci[cur[j]] != i) {
                    match = false;
                    break;
                }
                perm[e] = cur[j]++;
            }
        }
        if (match) {
            st = dev_alloc(c, reinterpret_cast<void **>(&c->bw_perm), perm.size() * sizeof(int32_t));
            if (st == GLGA_OK)
                st = dev_alloc(c, reinterpret_cast<void **>(&c->bw_pds), static_cast<size_t>(E) * H * sizeof(uint32_t));
            if (st != GLGA_OK) return st;
            GLGA_CUDA(cudaMemcpy(c->bw_perm, perm.data(), perm.size() * sizeof(int32_t), cudaMemcpyHostToDevice));
            GLGA_CUDA(cudaEventCreateWithFlags(&c->bw_ev_q, cudaEventDisableTiming));
        }
    }
    c->bw_nq_light = qp.n_light;
    c->bw_nq_heavy = qp.n_heavy;
    c->bw_nk_light = kp.n_light;
    c->bw_nk_heavy = kp.n_heavy;
    c->bw_nq_chunks = static_cast<int64_t>(qp.chunks.size());
    c->bw_nk_chunks = static_cast<int64_t>(kp.chunks.size());
    const int64_t nqc = std::max<int64_t>(c->bw_nq_chunks, 1), nkc = std::max<int64_t>(c->bw_nk_chunks, 1);
#define BTRY(x) \
    if (st == GLGA_OK) st = (x)
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_q_rows), (qp.rows.size() + 1) * sizeof(int32_t)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_k_rows), (kp.rows.size() + 1) * sizeof(int32_t)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_q_cptr), qp.chunk_ptr.size() * sizeof(int32_t)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_k_cptr), kp.chunk_ptr.size() * sizeof(int32_t)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_q_chunks), nqc * sizeof(int2)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_k_chunks), nkc * sizeof(int2)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_q_part), nqc * D * sizeof(float)));
    BTRY(dev_alloc(c, reinterpret_cast<void **>(&c->bw_kv_part), nkc * 2 * D * sizeof(float)));
#undef BTRY
    if (st != GLGA_OK) return st;
    auto up = [](void *dst, const void *src, size_t bytes) {
        return bytes ? cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice) : cudaSuccess;
    };
    GLGA_CUDA(up(c->bw_q_rows, qp.rows.data(), qp.rows.size() * sizeof(int32_t)));
    GLGA_CUDA(up(c->bw_k_rows, kp.rows.data(), kp.rows.size() * sizeof(int32_t)));
    GLGA_CUDA(up(c->bw_q_cptr, qp.chunk_ptr.data(), qp.chunk_ptr.size() * sizeof(int32_t)));
    GLGA_CUDA(up(c->bw_k_cptr, kp.chunk_ptr.data(), kp.chunk_ptr.size() * sizeof(int32_t)));
    GLGA_CUDA(up(c->bw_q_chunks, qp.chunks.data(), qp.chunks.size() * sizeof(int2)));
    GLGA_CUDA(up(c->bw_k_chunks, kp.chunks.data(), kp.chunks.size() * sizeof(int2)));
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
    const int64_t wrpp = ceil_div(std::max<int64_t>(N, 1), c->bw_wparts);
    const int Dc = 3 * D + 1;                         // columns of dZ in use: dQ | dK | dV | dt
    const int64_t wtotal = static_cast<int64_t>(d) * Dc;
#define BWD_LAUNCHES(T)                                                                                   \
    do {                                                                                                  \
        const T *Q = static_cast<const T *>(c->Q);                                                        \
        const T *KV = static_cast<const T *>(c->KV);                                                      \
        const unsigned tgrid = static_cast<unsigned>(ceil_div(static_cast<int64_t>(H) * R * R, 256));    \
        if (N > 0) {                                                                                      \
            bwd_heads_prep_kernel<<<tgrid, 256, 0, s>>>(c->Sz, R, H, R, c->bw_ST, nullptr);              \
            {                                                                                             \
                const glga_status rs = launch_readout_bwd<T>(c, Q, static_cast<const T *>(dY), b_g, eps, Dz, s); \
                if (rs != GLGA_OK) return rs;                                                             \
            }                                                                                             \
            /* fork: the dS | dz chain and the source-side kernels on the side stream */                 \
            GLGA_CUDA(cudaEventRecord(c->bw_ev_fork, s));                                                 \
            GLGA_CUDA(cudaStreamWaitEvent(c->bw_side, c->bw_ev_fork, 0));                                 \
            {                                                                                             \
                const glga_status ds = launch_dsz_bwd<T>(c, Q, c->bw_side);                               \
                if (ds != GLGA_OK) return ds;                                                             \
            }                                                                                             \
            bwd_sum_parts_kernel<<<sum_parts_grid(total), kSumThreads, 0, c->bw_side>>>(                 \
                c->bw_dsz_part, c->bw_dsz_parts, total, c->bw_dSz);                                       \
            bwd_heads_prep_kernel<<<tgrid, 256, 0, c->bw_side>>>(c->bw_dSz, R + 1, H, R, c->bw_dST,      \
                                                                c->bw_dSc);                               \
            {                                                                                             \
                const glga_status gs = launch_kv_global(c, Dz, c->bw_side);                               \
                if (gs != GLGA_OK) return gs;                                                             \
            }                                                                                             \
            launch_local_bwd<T>(c, Q, KV, isr, Dz, s, c->bw_side);                                        \
            GLGA_CUDA(cudaEventRecord(c->bw_ev_join, c->bw_side));                                        \
            GLGA_CUDA(cudaStreamWaitEvent(s, c->bw_ev_join, 0));                                          \
            if (bwd_fx(c)) {                                                                              \
                const glga_status gs = fx_gemms(c, X, WQ, WK, WV, wg, dX, s);                             \
                if (gs != GLGA_OK) return gs;                                                             \
                break;                                                                                    \
            }                                                                                             \
            if (bwd_tc_gemms(c)) {                                                                        \
                bwd_pack_w_kernel<T><<<static_cast<unsigned>(std::min<int64_t>(ceil_div(d * Dz, 256), 1024)), \
                                       256, 0, s>>>(static_cast<const T *>(WQ), static_cast<const T *>(WK), \
                                                    static_cast<const T *>(WV), static_cast<const T *>(wg), \
                                                    d, D, Dz, c->bw_Wall);                                  \
                const glga_status gs = tc_gemms(c, X, dX, s);                                             \
                if (gs != GLGA_OK) return gs;                                                             \
                bwd_dwg_kernel<T><<<dim3(static_cast<unsigned>(c->bw_wparts), ceil_div(d, 32)), 256, 0, s>>>( \
                    static_cast<const T *>(X), c->bw_dZ, N, d, Dz, 3 * D, Dc, wrpp, c->bw_dw_part,         \
                    c->bw_dbg_part);                                                                       \
                break;                                                                                    \
            }                                                                                             \
            bwd_pack_w_kernel<T><<<static_cast<unsigned>(std::min<int64_t>(ceil_div(d * Dz, 256), 1024)),   \
                                   256, 0, s>>>(static_cast<const T *>(WQ), static_cast<const T *>(WK),     \
                                                static_cast<const T *>(WV), static_cast<const T *>(wg), d, \
                                                D, Dz, c->bw_Wall);                                         \
            bwd_dw_kernel<T><<<dim3(ceil_div(d, kGT), ceil_div(3 * D, kGT), c->bw_wparts), 256, 0, s>>>(   \
                static_cast<const T *>(X), c->bw_dZ, N, d, Dz, 3 * D, Dc, wrpp, c->bw_dw_part);            \
            bwd_dwg_kernel<T><<<dim3(static_cast<unsigned>(c->bw_wparts), ceil_div(d, 32)), 256, 0, s>>>(   \
                static_cast<const T *>(X), c->bw_dZ, N, d, Dz, 3 * D, Dc, wrpp, c->bw_dw_part,             \
                c->bw_dbg_part);                                                                           \
            bwd_dx_kernel<<<dim3(static_cast<unsigned>(ceil_div(N, kGT)), ceil_div(d, kGT)), 256, 0, s>>>( \
                c->bw_dZ, c->bw_Wall, N, d, Dz, Dc, dX);                                                   \
        }                                                                                                 \
    } while (0)
    if (c->io == GLGA_F32)
        BWD_LAUNCHES(float);
    else
        BWD_LAUNCHES(__nv_bfloat16);
#undef BWD_LAUNCHES
    if (N > 0) {
        const int wp = bwd_fx(c) ? c->bw_fx_parts : c->bw_wparts;   // partials of dw_g (and dW)
        const bool tcg = bwd_tc_gemms(c);
        bwd_dw_reduce_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(wtotal, 256), 4096)), 256, 0, s>>>(
            c->bw_dw_part, wp, tcg ? c->bw_dW3 : nullptr, d, D, Dc, dWQ, dWK, dWV, dwg);
        if (tcg)   // dw_g: column 3D of the partials, one warp per feature
            bwd_strided_sum_kernel<<<static_cast<unsigned>(ceil_div(d, 8)), 256, 0, s>>>(
                c->bw_dw_part + 3 * D, wp, static_cast<int64_t>(d) * Dc, Dc, d, dwg);
        bwd_strided_sum_kernel<<<1, 32, 0, s>>>(c->bw_dbg_part, wp, 1, 0, 1, db_g);
    } else {
        GLGA_CUDA(cudaMemsetAsync(dWQ, 0, static_cast<size_t>(d) * D * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(dWK, 0, static_cast<size_t>(d) * D * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(dWV, 0, static_cast<size_t>(d) * D * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(dwg, 0, static_cast<size_t>(d) * sizeof(float), s));
        GLGA_CUDA(cudaMemsetAsync(db_g, 0, sizeof(float), s));
    }
    // (N == 0: no dS | dz to sum, and every gradient is zero)
    GLGA_CUDA(cudaGetLastError());
    c->launches += N > 0 ? (bwd_tc_gemms(c) ? 12 : 11) + local_bwd_launches(c) : 0;
    return GLGA_OK;
}

}  // namespace glga
