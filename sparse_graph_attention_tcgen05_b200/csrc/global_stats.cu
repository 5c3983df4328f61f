// global_stats.cu -- global statistics of the linear-attention branch.
//
// Method page "Gated Local-Global Graph Attention", Key formulas:
//   S_h = sum_j phi(k_j^h) (v_j^h)^T,  z_h = sum_j phi(k_j^h),  phi = elu + 1,
// summed over all N nodes.  Deterministic: the node range is cut into P fixed parts,
// every part's sums are formed in node order by one thread per output, and the parts
// are then added in part order.  Output layout: S [H][r][r] followed by z [H][r].
#include <algorithm>

#include "glga_internal.cuh"

namespace glga {
namespace {

constexpr int kStatsThreads = 256;
constexpr int kStatsRows = 32;      // node rows staged per shared-memory tile

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : expf(x); }

// grid: (P parts, H heads).  part[p][h][a][c] for c < r is S, c == r is z.
template <typename T, int R>
__global__ void __launch_bounds__(kStatsThreads) stats_part_kernel(const T *__restrict__ KV,
                                                                   int64_t N, int D,
                                                                   int64_t rows_per_part,
                                                                   float *__restrict__ part) {
    constexpr int kOut = R * (R + 1);
    constexpr int kPer = (kOut + kStatsThreads - 1) / kStatsThreads;
    __shared__ float sk[kStatsRows][R];
    __shared__ float sv[kStatsRows][R + 1];
    const int h = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_part;
    const int64_t r1 = std::min<int64_t>(N, r0 + rows_per_part);
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
    for (int64_t base = r0; base < r1; base += kStatsRows) {
        const int nrow = static_cast<int>(std::min<int64_t>(kStatsRows, r1 - base));
        __syncthreads();
        for (int idx = threadIdx.x; idx < kStatsRows * R; idx += kStatsThreads) {
            const int rr = idx / R, a = idx % R;
            float kx = 0.f, vx = 0.f;
            if (rr < nrow) {
                const T *row = KV + (base + rr) * 2 * static_cast<int64_t>(D);
                kx = phi(to_f<T>(row[h * R + a]));
                vx = to_f<T>(row[D + h * R + a]);
            }
            sk[rr][a] = kx;
            sv[rr][a] = vx;
            if (a == 0) sv[rr][R] = rr < nrow ? 1.f : 0.f;
        }
        __syncthreads();
        for (int rr = 0; rr < nrow; ++rr) {
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int o = threadIdx.x + i * kStatsThreads;
                if (o < kOut) acc[i] += sk[rr][o / (R + 1)] * sv[rr][o % (R + 1)];
            }
        }
    }
    float *dst = part + (static_cast<int64_t>(blockIdx.x) * gridDim.y + h) * kOut;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int o = threadIdx.x + i * kStatsThreads;
        if (o < kOut) dst[o] = acc[i];
    }
}

// Sz: S [H][r][r] then z [H][r]; sums parts 0..P-1 in order.
__global__ void stats_reduce_kernel(const float *__restrict__ part, int P, int H, int R,
                                    float *__restrict__ Sz) {
    const int per_head = R * (R + 1);
    const int total = H * per_head;
    for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < total; o += gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int p = 0; p < P; ++p) s += part[static_cast<int64_t>(p) * total + o];
        const int h = o / per_head, rem = o % per_head, a = rem / (R + 1), c = rem % (R + 1);
        if (c < R)
            Sz[(static_cast<int64_t>(h) * R + a) * R + c] = s;
        else
            Sz[static_cast<int64_t>(H) * R * R + h * R + a] = s;
    }
}

template <typename T>
glga_status launch_parts(Ctx *c, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>(c->stats_parts), static_cast<unsigned>(c->H));
    const T *kv = static_cast<const T *>(c->KV);
    switch (c->r) {
        case 8: stats_part_kernel<T, 8><<<grid, kStatsThreads, 0, s>>>(kv, c->N, c->D, c->stats_rows_per_part, c->Spart); break;
        case 16: stats_part_kernel<T, 16><<<grid, kStatsThreads, 0, s>>>(kv, c->N, c->D, c->stats_rows_per_part, c->Spart); break;
        case 32: stats_part_kernel<T, 32><<<grid, kStatsThreads, 0, s>>>(kv, c->N, c->D, c->stats_rows_per_part, c->Spart); break;
        case 64: stats_part_kernel<T, 64><<<grid, kStatsThreads, 0, s>>>(kv, c->N, c->D, c->stats_rows_per_part, c->Spart); break;
        case 128: stats_part_kernel<T, 128><<<grid, kStatsThreads, 0, s>>>(kv, c->N, c->D, c->stats_rows_per_part, c->Spart); break;
        default: set_error("unsupported r"); return GLGA_ERR_UNSUPPORTED;
    }
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

}  // namespace

glga_status stats_setup(Ctx *c) {
    const int64_t want = std::max<int64_t>(1, ceil_div(2 * c->num_sms, c->H));
    const int64_t parts = std::max<int64_t>(1, std::min<int64_t>(want, ceil_div(std::max<int64_t>(c->N, 1), kStatsRows)));
    c->stats_parts = static_cast<int32_t>(parts);
    c->stats_rows_per_part = static_cast<int32_t>(ceil_div(std::max<int64_t>(c->N, 1), parts));
    const size_t per = static_cast<size_t>(c->H) * c->r * (c->r + 1) * sizeof(float);
    glga_status st = dev_alloc(c, reinterpret_cast<void **>(&c->Spart), per * parts);
    if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->Sz), per);
    return st;
}

glga_status stats_run(Ctx *c, cudaStream_t s) {
    glga_status st = (c->io == GLGA_F32) ? launch_parts<float>(c, s) : launch_parts<__nv_bfloat16>(c, s);
    if (st != GLGA_OK) return st;
    const int total = c->H * c->r * (c->r + 1);
    stats_reduce_kernel<<<static_cast<unsigned>(ceil_div(total, 256)), 256, 0, s>>>(
        c->Spart, c->stats_parts, c->H, c->r, c->Sz);
    GLGA_CUDA(cudaGetLastError());
    c->launches += 2;
    return GLGA_OK;
}

}  // namespace glga

// ---------------------------------------------------------------------------------------
// glga_global_stats_static: the same global statistics for callers that cannot allocate
// device memory.  The per-range partial sums live in a fixed 2 MiB array that is part of
// this library's device image (every GPU that loads the library keeps it until the
// process exits), so the call allocates nothing.
// ---------------------------------------------------------------------------------------
#include <mutex>

namespace glga {
namespace {

constexpr size_t kStaticScratchFloats = 512u * 1024u;   // 2 MiB of float partial sums
constexpr int kMaxDevices = 64;

__device__ __align__(256) float g_static_stats_scratch[kStaticScratchFloats];

std::mutex g_static_mu;
float *g_static_scratch_addr[kMaxDevices] = {};
int g_static_num_sms[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
// The array's name in host code is only a host-side stand-in, never a device address.
glga_status static_scratch(int dev, float **ptr, int *num_sms) {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_scratch_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_stats_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static stats scratch)");
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        g_static_scratch_addr[dev] = static_cast<float *>(p);
        g_static_num_sms[dev] = sms;
    }
    *ptr = g_static_scratch_addr[dev];
    *num_sms = g_static_num_sms[dev];
    return GLGA_OK;
}

template <typename T>
glga_status launch_static_parts(const T *kv, int64_t N, int H, int r, int64_t rows_per_part,
                                      int parts, float *scratch, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>(parts), static_cast<unsigned>(H));
    const int D = H * r;
    switch (r) {
        case 8: stats_part_kernel<T, 8><<<grid, kStatsThreads, 0, s>>>(kv, N, D, rows_per_part, scratch); break;
        case 16: stats_part_kernel<T, 16><<<grid, kStatsThreads, 0, s>>>(kv, N, D, rows_per_part, scratch); break;
        case 32: stats_part_kernel<T, 32><<<grid, kStatsThreads, 0, s>>>(kv, N, D, rows_per_part, scratch); break;
        case 64: stats_part_kernel<T, 64><<<grid, kStatsThreads, 0, s>>>(kv, N, D, rows_per_part, scratch); break;
        case 128: stats_part_kernel<T, 128><<<grid, kStatsThreads, 0, s>>>(kv, N, D, rows_per_part, scratch); break;
        default: set_error("unsupported r"); return GLGA_ERR_UNSUPPORTED;
    }
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

}  // namespace

}  // namespace glga

extern "C" glga_status glga_global_stats_static(const void *KV, int64_t N, int32_t H, int32_t r,
                                                glga_dtype io, float *Sz, void *stream) {
    using namespace glga;
    if (N < 0 || H < 1 || (N > 0 && !KV) || !Sz) {
        set_error("glga_global_stats_static: need N >= 0, H >= 1, non-null KV (when N > 0) and Sz");
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
    int dev = 0;
    GLGA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("glga_global_stats_static: device ordinal %d not supported", dev);
        return GLGA_ERR_UNSUPPORTED;
    }
    float *scratch = nullptr;
    int sms = 0;
    glga_status st = static_scratch(dev, &scratch, &sms);
    if (st != GLGA_OK) return st;
    const int64_t fit = static_cast<int64_t>(kStaticScratchFloats) / per_part;
    const int64_t want = std::max<int64_t>(1, ceil_div(2 * sms, H));
    const int64_t parts = std::max<int64_t>(
        1, std::min<int64_t>(std::min(want, fit), ceil_div(std::max<int64_t>(N, 1), kStatsRows)));
    const int64_t rows_per_part = ceil_div(std::max<int64_t>(N, 1), parts);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = (io == GLGA_F32)
             ? launch_static_parts<float>(static_cast<const float *>(KV), N, H, r, rows_per_part,
                                          static_cast<int>(parts), scratch, s)
             : launch_static_parts<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(KV), N, H, r,
                                                  rows_per_part, static_cast<int>(parts), scratch, s);
    if (st != GLGA_OK) return st;
    const int total = static_cast<int>(per_part);
    stats_reduce_kernel<<<static_cast<unsigned>(ceil_div(total, 256)), 256, 0, s>>>(
        scratch, static_cast<int>(parts), H, r, Sz);
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}
