// backward.cu -- the backward passes a trainer needs around the invariant
// forward kernels (xitu-tech news, "强化学习的突破": on-policy RL wants the
// trainer to reproduce the sampler's numbers, so every pass runs on fixed,
// deterministic reduction orders).
//
//   RMSNorm   dx: one block per row, every sum in a fixed order that depends
//             on H only, so a row's dx does not depend on the batch.
//             dw: a sum over rows -- in chunks of 64 rows counted from row 0,
//             each chunk's rows in ascending order, then the chunks in
//             ascending order: the same bits on every run.
//   matmul    through the invariant GEMM: dA = dC W as dC (W^T)^T and
//             dW = dC^T A as (dC^T) (A^T)^T, the transposes made by
//             transpose_kernel (bit copies).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"

namespace bi {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kDwChunk = 64;   // rows per partial sum of dw
constexpr int kDwBatch = 8;    // rows whose loads are in flight together

__device__ __forceinline__ float lo_f(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi_f(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_rn(float a, float b)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&p);
}

// Block-wide sum in a fixed order: a xor butterfly in each warp, then the
// warp totals added in warp order.  Every thread gets the result.
__device__ float block_sum_fixed(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // red is free
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.0f;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) s = __fadd_rn(s, red[w]);
    return s;
}

// dx of one row per block iteration; r of each row to rs (for dw).
__global__ void __launch_bounds__(kBwdThreads)
rmsnorm_bwd_rows_kernel(const uint4 *__restrict__ x, const uint4 *__restrict__ w,
                        const uint4 *__restrict__ dy, void *__restrict__ dx, float *__restrict__ rs,
                        int64_t M, int64_t H, float eps, int out_f32)
{
    __shared__ float red[kBwdThreads / 32];
    const int64_t pieces = H / 8;
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        const uint4 *xr = x + m * pieces;
        const uint4 *dr = dy + m * pieces;
        float sq = 0.0f, dot = 0.0f;
        for (int64_t p = threadIdx.x; p < pieces; p += blockDim.x) {
            const uint4 a = xr[p], b = dr[p], c = __ldg(w + p);
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
            const uint32_t cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float x0 = lo_f(av[j]), x1 = hi_f(av[j]);
                sq = __fadd_rn(sq, __fmul_rn(x0, x0));
                sq = __fadd_rn(sq, __fmul_rn(x1, x1));
                dot = __fadd_rn(dot, __fmul_rn(__fmul_rn(lo_f(cv[j]), lo_f(bv[j])), x0));
                dot = __fadd_rn(dot, __fmul_rn(__fmul_rn(hi_f(cv[j]), hi_f(bv[j])), x1));
            }
        }
        sq = block_sum_fixed(sq, red);
        dot = block_sum_fixed(dot, red);
        const float r = rsqrtf(__fadd_rn(__fdiv_rn(sq, float(H)), eps));
        // dx_j = r w_j dy_j - x_j (r^3 / H) dot
        const float c = __fmul_rn(__fmul_rn(__fmul_rn(r, r), r), __fdiv_rn(dot, float(H)));
        if (threadIdx.x == 0) rs[m] = r;
        for (int64_t p = threadIdx.x; p < pieces; p += blockDim.x) {
            const uint4 a = xr[p], b = dr[p], cw = __ldg(w + p);
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
            const uint32_t cv[4] = {cw.x, cw.y, cw.z, cw.w};
            float o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                o[2 * j] = __fsub_rn(__fmul_rn(__fmul_rn(r, lo_f(cv[j])), lo_f(bv[j])),
                                     __fmul_rn(lo_f(av[j]), c));
                o[2 * j + 1] = __fsub_rn(__fmul_rn(__fmul_rn(r, hi_f(cv[j])), hi_f(bv[j])),
                                         __fmul_rn(hi_f(av[j]), c));
            }
            if (out_f32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(dx) + m * H + 8 * p);
                dst[0] = make_float4(o[0], o[1], o[2], o[3]);
                dst[1] = make_float4(o[4], o[5], o[6], o[7]);
            } else {
                static_cast<uint4 *>(dx)[m * pieces + p] =
                    make_uint4(pack_rn(o[0], o[1]), pack_rn(o[2], o[3]), pack_rn(o[4], o[5]),
                               pack_rn(o[6], o[7]));
            }
        }
    }
}

// partial[c, j] = sum over the rows of chunk c (ascending) of dy_j x_j r.
// One thread per 8 columns of one chunk.
__global__ void rmsnorm_bwd_dw_partial_kernel(const uint4 *__restrict__ x,
                                              const uint4 *__restrict__ dy,
                                              const float *__restrict__ rs, int64_t M, int64_t H,
                                              float *__restrict__ partial)
{
    const int64_t pieces = H / 8;
    const int64_t chunks = (M + kDwChunk - 1) / kDwChunk;
    const int64_t n = chunks * pieces;
    for (int64_t it = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; it < n;
         it += int64_t(gridDim.x) * blockDim.x) {
        const int64_t ch = it / pieces, p = it - ch * pieces;
        const int64_t m1 = (ch + 1) * kDwChunk < M ? (ch + 1) * kDwChunk : M;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int64_t m0 = ch * kDwChunk; m0 < m1; m0 += kDwBatch) {
            // the loads of up to kDwBatch rows first, then their terms in row order
            uint4 a[kDwBatch], b[kDwBatch];
            float r[kDwBatch];
#pragma unroll
            for (int u = 0; u < kDwBatch; ++u) {
                const bool in = m0 + u < m1;
                a[u] = in ? __ldg(x + (m0 + u) * pieces + p) : make_uint4(0u, 0u, 0u, 0u);
                b[u] = in ? __ldg(dy + (m0 + u) * pieces + p) : make_uint4(0u, 0u, 0u, 0u);
                r[u] = in ? __ldg(rs + m0 + u) : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < kDwBatch; ++u) {
                if (m0 + u >= m1) break;
                const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
                const uint32_t bv[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[2 * j] =
                        __fadd_rn(acc[2 * j], __fmul_rn(__fmul_rn(lo_f(bv[j]), lo_f(av[j])), r[u]));
                    acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1],
                                               __fmul_rn(__fmul_rn(hi_f(bv[j]), hi_f(av[j])), r[u]));
                }
            }
        }
        float4 *dst = reinterpret_cast<float4 *>(partial + ch * H + 8 * p);
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

// dw_j = sum over chunks (ascending) of partial[c, j].
__global__ void rmsnorm_bwd_dw_final_kernel(const float *__restrict__ partial, int64_t chunks,
                                            int64_t H, void *__restrict__ dw, int out_f32)
{
    for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < H;
         j += int64_t(gridDim.x) * blockDim.x) {
        float s = 0.0f;
        for (int64_t c = 0; c < chunks; ++c) s = __fadd_rn(s, partial[c * H + j]);
        if (out_f32)
            static_cast<float *>(dw)[j] = s;
        else
            static_cast<__nv_bfloat16 *>(dw)[j] = __float2bfloat16_rn(s);
    }
}

// out[c, r] = a[r, c] for r < R; out[c, r] = 0 for R <= r < ld_out.  32 x 32
// tiles through shared memory (one padding column against bank conflicts).
__global__ void transpose_kernel(const uint16_t *__restrict__ a, uint16_t *__restrict__ out,
                                 int64_t R, int64_t C, int64_t ld_out)
{
    __shared__ uint16_t tile[32][33];
    const int64_t tiles_r = (ld_out + 31) / 32, tiles_c = (C + 31) / 32;
    for (int64_t t = blockIdx.x; t < tiles_r * tiles_c; t += gridDim.x) {
        const int64_t r0 = (t / tiles_c) * 32, c0 = (t % tiles_c) * 32;
        __syncthreads();
        for (int i = threadIdx.y; i < 32; i += blockDim.y) {
            const int64_t r = r0 + i, c = c0 + threadIdx.x;
            tile[i][threadIdx.x] = (r < R && c < C) ? a[r * C + c] : uint16_t(0);
        }
        __syncthreads();
        for (int i = threadIdx.y; i < 32; i += blockDim.y) {
            const int64_t c = c0 + i, r = r0 + threadIdx.x;
            if (c < C && r < ld_out) out[c * ld_out + r] = tile[threadIdx.x][i];
        }
    }
}

}  // namespace

size_t rmsnorm_backward_ws_bytes(int64_t M, int64_t H)
{
    const int64_t chunks = (M + kDwChunk - 1) / kDwChunk;
    const size_t rs = (size_t(M) * 4 + 255) / 256 * 256;
    return rs + size_t(chunks) * size_t(H) * 4;
}

cudaError_t launch_rmsnorm_backward(const void *x, const void *w, const void *dy, void *dx,
                                    void *dw, int64_t M, int64_t H, float eps, bool out_f32,
                                    void *ws, int num_sms, cudaStream_t s)
{
    float *rs = static_cast<float *>(ws);
    float *partial = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) +
                                               (size_t(M) * 4 + 255) / 256 * 256);
    const int64_t cap = int64_t(num_sms) * 8;
    rmsnorm_bwd_rows_kernel<<<static_cast<unsigned>(M < cap ? M : cap), kBwdThreads, 0, s>>>(
        static_cast<const uint4 *>(x), static_cast<const uint4 *>(w),
        static_cast<const uint4 *>(dy), dx, rs, M, H, eps, out_f32 ? 1 : 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t chunks = (M + kDwChunk - 1) / kDwChunk;
    const int64_t items = chunks * (H / 8);
    const int64_t blocks = (items + 127) / 128;
    rmsnorm_bwd_dw_partial_kernel<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 128, 0,
                                    s>>>(static_cast<const uint4 *>(x),
                                         static_cast<const uint4 *>(dy), rs, M, H, partial);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t fb = (H + 255) / 256;
    rmsnorm_bwd_dw_final_kernel<<<static_cast<unsigned>(fb), 256, 0, s>>>(partial, chunks, H, dw,
                                                                          out_f32 ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_transpose(const void *a, void *out, int64_t R, int64_t C, int64_t ld_out,
                             int num_sms, cudaStream_t s)
{
    const int64_t tiles = ((ld_out + 31) / 32) * ((C + 31) / 32);
    const int64_t cap = int64_t(num_sms) * 16;
    transpose_kernel<<<static_cast<unsigned>(tiles < cap ? tiles : cap), dim3(32, 8), 0, s>>>(
        static_cast<const uint16_t *>(a), static_cast<uint16_t *>(out), R, C, ld_out);
    return cudaGetLastError();
}

}  // namespace bi
