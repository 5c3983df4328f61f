// topology.cu -- integer graph preparation: prefix scans, CSR validation, degree buckets
// and the CSR-from-COO builder.
//
// The target-grouped CSR is the form the tinymesh page ("Sparse attention experiment",
// section "Target softmax") reduces over: one row per destination.  Everything here is
// integer work and deterministic; its results are compared bit for bit with the oracle.
#include <algorithm>
#include <cstdio>
#include <vector>

#include "glga_internal.cuh"

namespace glga {

// ---------------------------------------------------------------------------------------
// exclusive prefix scan of int32 (tiles of 4096, recursive over tile sums)
// ---------------------------------------------------------------------------------------
constexpr int kScanThreads = 1024;
constexpr int kScanIpt = 4;
constexpr int64_t kScanTile = kScanThreads * kScanIpt;

__global__ void __launch_bounds__(kScanThreads) scan_tile_kernel(const int32_t *__restrict__ in,
                                                                 int32_t *__restrict__ out,
                                                                 int64_t n,
                                                                 int32_t *__restrict__ tile_sums) {
    __shared__ int32_t warp_tot[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile + threadIdx.x * kScanIpt;
    int32_t v[kScanIpt], loc[kScanIpt];
    int32_t s = 0;
#pragma unroll
    for (int i = 0; i < kScanIpt; ++i) {
        v[i] = (base + i < n) ? in[base + i] : 0;
        loc[i] = s;
        s += v[i];
    }
    int32_t x = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
        int32_t t = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_tot[lane] = t;
    }
    __syncthreads();
    const int32_t warp_off = (w > 0) ? warp_tot[w - 1] : 0;
    const int32_t off = warp_off + x - s;
#pragma unroll
    for (int i = 0; i < kScanIpt; ++i)
        if (base + i < n) out[base + i] = off + loc[i];
    if (threadIdx.x == kScanThreads - 1 && tile_sums) tile_sums[blockIdx.x] = warp_off + x;
}

__global__ void scan_add_kernel(int32_t *__restrict__ out, int64_t n,
                                const int32_t *__restrict__ tile_off) {
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile;
    const int32_t add = tile_off[blockIdx.x];
    for (int64_t i = threadIdx.x; i < kScanTile; i += blockDim.x)
        if (base + i < n) out[base + i] += add;
}

__global__ void scan_total_kernel(const int32_t *in, const int32_t *out, int64_t n,
                                  int32_t *total) {
    *total = n > 0 ? out[n - 1] + in[n - 1] : 0;
}

size_t scan_tmp_bytes(int64_t n) {
    size_t b = 0;
    while (n > kScanTile) {
        int64_t t = ceil_div(n, kScanTile);
        b += 2 * static_cast<size_t>(t) * sizeof(int32_t);
        n = t;
    }
    return b + 256;
}

glga_status exclusive_scan_i32(const int32_t *in, int32_t *out, int64_t n, int32_t *total_dev,
                               cudaStream_t s, void *tmp, size_t tmp_bytes) {
    if (n <= 0) {
        if (total_dev) GLGA_CUDA(cudaMemsetAsync(total_dev, 0, sizeof(int32_t), s));
        return GLGA_OK;
    }
    const int64_t tiles = ceil_div(n, kScanTile);
    if (tiles == 1) {
        scan_tile_kernel<<<1, kScanThreads, 0, s>>>(in, out, n, nullptr);
    } else {
        if (tmp_bytes < 2 * tiles * sizeof(int32_t)) {
            set_error("scan scratch too small");
            return GLGA_ERR_INVALID_ARG;
        }
        int32_t *sums = static_cast<int32_t *>(tmp);
        int32_t *offs = sums + tiles;
        scan_tile_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, s>>>(in, out, n, sums);
        glga_status st = exclusive_scan_i32(sums, offs, tiles, nullptr, s, offs + tiles,
                                            tmp_bytes - 2 * tiles * sizeof(int32_t));
        if (st != GLGA_OK) return st;
        scan_add_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(out, n, offs);
    }
    GLGA_CUDA(cudaGetLastError());
    if (total_dev) scan_total_kernel<<<1, 1, 0, s>>>(in, out, n, total_dev);
    GLGA_CUDA(cudaGetLastError());
    return GLGA_OK;
}

// ---------------------------------------------------------------------------------------
// CSR validation
// ---------------------------------------------------------------------------------------
__global__ void validate_csr_kernel(const int32_t *__restrict__ rp, const int32_t *__restrict__ col,
                                    int64_t N, int64_t E, int64_t n_cols, unsigned *flag) {
    unsigned bad = 0;
    const int64_t lim = (N + 1 > E) ? N + 1 : E;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < lim;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (i == 0 && rp[0] != 0) bad |= kGraphBadRowPtr0;
        if (i == N && static_cast<int64_t>(rp[N]) != E) bad |= kGraphBadRowPtrEnd;
        if (i < N && rp[i + 1] < rp[i]) bad |= kGraphNotMonotone;
        if (i < E && (col[i] < 0 || static_cast<int64_t>(col[i]) >= n_cols)) bad |= kGraphColOutOfRange;
    }
    if (bad) atomicOr(flag, bad);
}

glga_status validate_csr(Ctx *c, cudaStream_t s) {
    GLGA_CUDA(cudaMemsetAsync(c->dev_flag, 0, sizeof(unsigned), s));
    const int64_t lim = (c->N + 1 > c->E) ? c->N + 1 : c->E;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(lim, 256), 4096));
    // rows are the context's targets; columns index all n_src nodes whose k/v it reads
    validate_csr_kernel<<<blocks, 256, 0, s>>>(c->row_ptr, c->col_idx, c->N, c->E, c->n_src, c->dev_flag);
    GLGA_CUDA(cudaGetLastError());
    unsigned h = 0;
    GLGA_CUDA(cudaMemcpyAsync(&h, c->dev_flag, sizeof(unsigned), cudaMemcpyDeviceToHost, s));
    GLGA_CUDA(cudaStreamSynchronize(s));
    if (h) {
        set_error("invalid CSR:%s%s%s%s", (h & kGraphBadRowPtr0) ? " row_ptr[0]!=0" : "",
                  (h & kGraphBadRowPtrEnd) ? " row_ptr[N]!=E" : "",
                  (h & kGraphNotMonotone) ? " row_ptr decreasing" : "",
                  (h & kGraphColOutOfRange) ? " col_idx outside [0, node count)" : "");
        return GLGA_ERR_BAD_GRAPH;
    }
    return GLGA_OK;
}

// ---------------------------------------------------------------------------------------
// degree buckets
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int bucket_of(int64_t deg, int32_t wmax, int32_t chunk) {
    return deg <= wmax ? 0 : (deg <= chunk ? 1 : 2);
}

__global__ void bucket_flags_kernel(const int32_t *__restrict__ rp, int64_t N, int32_t wmax,
                                    int32_t chunk, int32_t *f0, int32_t *f1, int32_t *f2,
                                    int32_t *fc) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < N;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t deg = static_cast<int64_t>(rp[i + 1]) - rp[i];
        const int b = bucket_of(deg, wmax, chunk);
        f0[i] = b == 0;
        f1[i] = b == 1;
        f2[i] = b == 2;
        fc[i] = b == 2 ? static_cast<int32_t>(ceil_div(deg, chunk)) : 0;
    }
}

__global__ void bucket_scatter_kernel(const int32_t *__restrict__ rp, int64_t N, int32_t wmax,
                                      int32_t chunk, const int32_t *o0, const int32_t *o1,
                                      const int32_t *o2, const int32_t *oc, int32_t *warp_rows,
                                      int32_t *cta_rows, int32_t *split_rows, int32_t *chunk_row,
                                      int32_t *chunk_begin) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < N;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t deg = static_cast<int64_t>(rp[i + 1]) - rp[i];
        const int b = bucket_of(deg, wmax, chunk);
        if (b == 0) {
            warp_rows[o0[i]] = static_cast<int32_t>(i);
        } else if (b == 1) {
            cta_rows[o1[i]] = static_cast<int32_t>(i);
        } else {
            split_rows[o2[i]] = static_cast<int32_t>(i);
            const int32_t n = static_cast<int32_t>(ceil_div(deg, chunk));
            for (int32_t k = 0; k < n; ++k) {
                chunk_row[oc[i] + k] = static_cast<int32_t>(i);
                chunk_begin[oc[i] + k] = rp[i] + k * chunk;
            }
        }
    }
}

glga_status build_buckets(Ctx *c, cudaStream_t s) {
    const int64_t N = c->N;
    if (N == 0) return GLGA_OK;
    const size_t tmpb = scan_tmp_bytes(N);
    void *scratch = nullptr;
    const size_t nbytes = 8 * static_cast<size_t>(N) * sizeof(int32_t) + 4 * sizeof(int32_t) + tmpb;
    const glga_status hook = debug_alloc_hook(c);
    if (hook != GLGA_OK) return hook;
    GLGA_CUDA(cudaMalloc(&scratch, nbytes));
    int32_t *f = static_cast<int32_t *>(scratch);
    int32_t *o = f + 4 * N;
    int32_t *tot = o + 4 * N;
    void *tmp = tot + 4;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(N, 256), 8192));
    glga_status st = GLGA_OK;
    bucket_flags_kernel<<<blocks, 256, 0, s>>>(c->row_ptr, N, c->opts.warp_max_degree,
                                               c->opts.chunk_edges, f, f + N, f + 2 * N, f + 3 * N);
    for (int k = 0; k < 4 && st == GLGA_OK; ++k)
        st = exclusive_scan_i32(f + k * N, o + k * N, N, tot + k, s, tmp, tmpb);
    int32_t h[4] = {0, 0, 0, 0};
    if (st == GLGA_OK) {
        cudaError_t e = cudaMemcpyAsync(h, tot, sizeof(h), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) st = cuda_fail(e, "bucket sizes");
    }
    if (st == GLGA_OK) {
        for (int k = 0; k < 4; ++k) c->nb[k] = h[k];
        st = dev_alloc(c, reinterpret_cast<void **>(&c->warp_rows), (h[0] + 1) * sizeof(int32_t));
        if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->cta_rows), (h[1] + 1) * sizeof(int32_t));
        if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->split_rows), (h[2] + 1) * sizeof(int32_t));
        if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->chunk_row), (h[3] + 1) * sizeof(int32_t));
        if (st == GLGA_OK) st = dev_alloc(c, reinterpret_cast<void **>(&c->chunk_begin), (h[3] + 1) * sizeof(int32_t));
    }
    if (st == GLGA_OK) {
        bucket_scatter_kernel<<<blocks, 256, 0, s>>>(
            c->row_ptr, N, c->opts.warp_max_degree, c->opts.chunk_edges, o, o + N, o + 2 * N,
            o + 3 * N, c->warp_rows, c->cta_rows, c->split_rows, c->chunk_row, c->chunk_begin);
        cudaError_t e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) st = cuda_fail(e, "bucket scatter");
    }
    cudaFree(scratch);
    // Bucket 0 by descending degree, ties by ascending row: rows of similar degree share a
    // warp task and the heaviest start first.
    if (st == GLGA_OK && h[0] > 1) {
        std::vector<int32_t> rp(static_cast<size_t>(N) + 1), rows(static_cast<size_t>(h[0]));
        cudaError_t e = cudaMemcpy(rp.data(), c->row_ptr, rp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
        if (e == cudaSuccess)
            e = cudaMemcpy(rows.data(), c->warp_rows, rows.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
        if (e == cudaSuccess) {
            std::stable_sort(rows.begin(), rows.end(), [&rp](int32_t a, int32_t b) {
                return rp[a + 1] - rp[a] > rp[b + 1] - rp[b];
            });
            e = cudaMemcpy(c->warp_rows, rows.data(), rows.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
        }
        if (e != cudaSuccess) st = cuda_fail(e, "bucket-0 order");
    }
    return st;
}

// ---------------------------------------------------------------------------------------
// CSR from COO: key = (dst << b) | src sorted by an LSD radix sort (8-bit digits, stable
// per pass), then col_idx = low bits and row_ptr from the row boundaries.
// ---------------------------------------------------------------------------------------
constexpr int kRsThreads = 256;
constexpr int kRsIpt = 16;
constexpr int64_t kRsTile = kRsThreads * kRsIpt;
constexpr int kRsWarps = kRsThreads / 32;

__global__ void coo_check_keys_kernel(const int32_t *__restrict__ src, const int32_t *__restrict__ dst,
                                      int64_t E, int64_t N, int bits, uint64_t *__restrict__ keys,
                                      unsigned *flag) {
    unsigned bad = 0;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < E;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t a = src[e], b = dst[e];
        if (a < 0 || a >= N || b < 0 || b >= N) {
            bad = 1;
            keys[e] = 0;
        } else {
            keys[e] = (static_cast<uint64_t>(b) << bits) | static_cast<uint64_t>(a);
        }
    }
    if (bad) atomicOr(flag, 1u);
}

__global__ void __launch_bounds__(kRsThreads) radix_hist_kernel(const uint64_t *__restrict__ keys,
                                                                int64_t n, int shift,
                                                                int32_t *__restrict__ counts,
                                                                int64_t nblocks) {
    __shared__ int32_t h[256];
    h[threadIdx.x] = 0;
    __syncthreads();
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kRsTile;
#pragma unroll 4
    for (int i = 0; i < kRsIpt; ++i) {
        const int64_t idx = base + i * kRsThreads + threadIdx.x;
        if (idx < n) atomicAdd(&h[(keys[idx] >> shift) & 255u], 1);
    }
    __syncthreads();
    counts[threadIdx.x * nblocks + blockIdx.x] = h[threadIdx.x];
}

__global__ void __launch_bounds__(kRsThreads) radix_scatter_kernel(const uint64_t *__restrict__ in,
                                                                   uint64_t *__restrict__ out,
                                                                   int64_t n, int shift,
                                                                   const int32_t *__restrict__ offs,
                                                                   int64_t nblocks) {
    __shared__ int32_t base[256];
    __shared__ int32_t wcnt[kRsWarps][256];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    base[t] = offs[t * nblocks + blockIdx.x];
    const int64_t tile = static_cast<int64_t>(blockIdx.x) * kRsTile;
    for (int round = 0; round < kRsIpt; ++round) {
#pragma unroll
        for (int k = 0; k < kRsWarps; ++k) wcnt[k][t] = 0;
        __syncthreads();
        const int64_t idx = tile + round * kRsThreads + t;
        const bool valid = idx < n;
        const uint64_t key = valid ? in[idx] : 0ull;
        const uint32_t dig = valid ? static_cast<uint32_t>((key >> shift) & 255u) : 256u;
        const uint32_t peers = __match_any_sync(0xffffffffu, dig);
        const int rank = __popc(peers & lt_mask);
        if (valid && rank == 0) wcnt[w][dig] = __popc(peers);
        __syncthreads();
        int32_t run = 0;
#pragma unroll
        for (int k = 0; k < kRsWarps; ++k) {
            const int32_t cnt = wcnt[k][t];
            wcnt[k][t] = run;
            run += cnt;
        }
        __syncthreads();
        if (valid) out[base[dig] + wcnt[w][dig] + rank] = key;
        __syncthreads();
        base[t] += run;
    }
}

__global__ void csr_emit_kernel(const uint64_t *__restrict__ keys, int64_t E, int64_t N, int bits,
                                int32_t *__restrict__ row_ptr, int32_t *__restrict__ col_idx) {
    const uint64_t mask = (bits >= 64) ? ~0ull : ((1ull << bits) - 1ull);
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e <= E;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t prev = e > 0 ? static_cast<int64_t>(keys[e - 1] >> bits) : -1;
        const int64_t cur = e < E ? static_cast<int64_t>(keys[e] >> bits) : N;
        if (e < E) col_idx[e] = static_cast<int32_t>(keys[e] & mask);
        for (int64_t row = prev + 1; row <= cur && row <= N; ++row)
            row_ptr[row] = static_cast<int32_t>(e);
    }
}

}  // namespace glga

using namespace glga;

extern "C" glga_status glga_csr_from_coo(int64_t N, int64_t E, const int32_t *src,
                                         const int32_t *dst, int32_t *row_ptr, int32_t *col_idx,
                                         void *stream) {
    if (N < 0 || E < 0 || N > 2147483647LL || E > 2147483647LL) {
        set_error("glga_csr_from_coo: N and E must be in [0, 2^31)");
        return GLGA_ERR_INVALID_ARG;
    }
    if (!row_ptr || (E > 0 && (!src || !dst || !col_idx))) {
        set_error("glga_csr_from_coo: null pointer");
        return GLGA_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int bits = 1;
    while ((1LL << bits) < N) ++bits;
    const int64_t nblocks = ceil_div(E, kRsTile);
    const int64_t ncount = 256 * nblocks;
    const size_t tmpb = scan_tmp_bytes(ncount);
    const size_t bytes = 2 * static_cast<size_t>(E) * sizeof(uint64_t) +
                         2 * static_cast<size_t>(ncount) * sizeof(int32_t) + tmpb + 256;
    void *scratch = nullptr;
    GLGA_CUDA(cudaMalloc(&scratch, bytes));
    uint64_t *ka = static_cast<uint64_t *>(scratch);
    uint64_t *kb = ka + E;
    int32_t *counts = reinterpret_cast<int32_t *>(kb + E);
    int32_t *offs = counts + ncount;
    unsigned *flag = reinterpret_cast<unsigned *>(offs + ncount);
    void *tmp = flag + 64;
    glga_status st = GLGA_OK;
    cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) st = cuda_fail(e, "memset");
    if (st == GLGA_OK && E > 0) {
        const unsigned g = static_cast<unsigned>(std::min<int64_t>(ceil_div(E, 256), 8192));
        coo_check_keys_kernel<<<g, 256, 0, s>>>(src, dst, E, N, bits, ka, flag);
        unsigned h = 0;
        e = cudaMemcpyAsync(&h, flag, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) {
            st = cuda_fail(e, "COO check");
        } else if (h) {
            set_error("glga_csr_from_coo: an endpoint is outside [0, N)");
            st = GLGA_ERR_BAD_GRAPH;
        }
        for (int shift = 0; st == GLGA_OK && shift < 2 * bits; shift += 8) {
            radix_hist_kernel<<<static_cast<unsigned>(nblocks), kRsThreads, 0, s>>>(ka, E, shift,
                                                                                   counts, nblocks);
            st = exclusive_scan_i32(counts, offs, ncount, nullptr, s, tmp, tmpb);
            if (st != GLGA_OK) break;
            radix_scatter_kernel<<<static_cast<unsigned>(nblocks), kRsThreads, 0, s>>>(
                ka, kb, E, shift, offs, nblocks);
            e = cudaGetLastError();
            if (e != cudaSuccess) st = cuda_fail(e, "radix pass");
            uint64_t *x = ka;
            ka = kb;
            kb = x;
        }
    }
    if (st == GLGA_OK) {
        const unsigned g = static_cast<unsigned>(std::min<int64_t>(ceil_div(E + 1, 256), 8192));
        csr_emit_kernel<<<g, 256, 0, s>>>(ka, E, N, bits, row_ptr, col_idx);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) st = cuda_fail(e, "CSR emit");
    }
    cudaStreamSynchronize(s);
    cudaFree(scratch);
    return st;
}
