// rmsnorm.cu -- batch-invariant RMSNorm.
//
// xitu-tech news, "构建确定性解决方案", RMSNorm item, and neican.ai insight,
// "技术原理与创新点解析", data-parallel RMSNorm bullet: each batch row is
// reduced entirely by one core (here: one thread block), with one reduction
// strategy for every batch size -- never a split reduction across blocks.
//
// Per row r (fp32 arithmetic, bf16 in):
//   ss      = sum_j x[r,j]^2          (order fixed by H alone, see below)
//   rstd    = rsqrt(ss / H + eps)
//   y[r,j]  = round((x[r,j] * rstd) * w[j])
//
// Order of the sum of squares: thread t of the block owns 16-byte chunks
// t, t+T, ..., t+(ITEMS-1)T of the row and accumulates their elements in
// index order with fused multiply-adds; the T partial sums are combined by a
// 5-level xor-butterfly inside each warp and then warp 0..T/32-1 in order.
// T and ITEMS depend only on H, so a row gets the same bits whatever M is,
// whichever block handles it and wherever it sits in the batch.
//
// Memory: rows are loaded once into registers with 128-bit loads (a block
// loads all of its R rows before reducing any, to keep more bytes in
// flight), the output is written with 128-bit stores.  The grid strides
// over groups of R rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"

namespace bi {
namespace {

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ float sumsq8(const uint4 &v, float acc)
{
    acc = __fmaf_rn(bf_lo(v.x), bf_lo(v.x), acc);
    acc = __fmaf_rn(bf_hi(v.x), bf_hi(v.x), acc);
    acc = __fmaf_rn(bf_lo(v.y), bf_lo(v.y), acc);
    acc = __fmaf_rn(bf_hi(v.y), bf_hi(v.y), acc);
    acc = __fmaf_rn(bf_lo(v.z), bf_lo(v.z), acc);
    acc = __fmaf_rn(bf_hi(v.z), bf_hi(v.z), acc);
    acc = __fmaf_rn(bf_lo(v.w), bf_lo(v.w), acc);
    acc = __fmaf_rn(bf_hi(v.w), bf_hi(v.w), acc);
    return acc;
}

__device__ __forceinline__ float scale1(float x, float rstd, float w)
{
    return __fmul_rn(__fmul_rn(x, rstd), w);
}

template <bool OUT_F32>
__device__ __forceinline__ void store8(void *y, int64_t idx, const uint4 &xv, const uint4 &wv,
                                       float rstd)
{
    float o[8];
    o[0] = scale1(bf_lo(xv.x), rstd, bf_lo(wv.x));
    o[1] = scale1(bf_hi(xv.x), rstd, bf_hi(wv.x));
    o[2] = scale1(bf_lo(xv.y), rstd, bf_lo(wv.y));
    o[3] = scale1(bf_hi(xv.y), rstd, bf_hi(wv.y));
    o[4] = scale1(bf_lo(xv.z), rstd, bf_lo(wv.z));
    o[5] = scale1(bf_hi(xv.z), rstd, bf_hi(wv.z));
    o[6] = scale1(bf_lo(xv.w), rstd, bf_lo(wv.w));
    o[7] = scale1(bf_hi(xv.w), rstd, bf_hi(wv.w));
    if constexpr (OUT_F32) {
        float4 *yr = reinterpret_cast<float4 *>(y) + idx * 2;
        __stcs(yr, make_float4(o[0], o[1], o[2], o[3]));
        __stcs(yr + 1, make_float4(o[4], o[5], o[6], o[7]));
    } else {
        uint4 ov;
        __nv_bfloat162 p0 = __floats2bfloat162_rn(o[0], o[1]);
        __nv_bfloat162 p1 = __floats2bfloat162_rn(o[2], o[3]);
        __nv_bfloat162 p2 = __floats2bfloat162_rn(o[4], o[5]);
        __nv_bfloat162 p3 = __floats2bfloat162_rn(o[6], o[7]);
        ov.x = *reinterpret_cast<uint32_t *>(&p0);
        ov.y = *reinterpret_cast<uint32_t *>(&p1);
        ov.z = *reinterpret_cast<uint32_t *>(&p2);
        ov.w = *reinterpret_cast<uint32_t *>(&p3);
        __stcs(reinterpret_cast<uint4 *>(y) + idx, ov);
    }
}

// A block handles R rows at a time: all R rows are loaded before any is
// reduced, so that more bytes are in flight.  R changes only how rows are
// grouped into blocks; each row's arithmetic is the same for every R.
template <int ITEMS, int R, bool OUT_F32, int MAXT>
__global__ void __launch_bounds__(MAXT, MAXT <= 256 ? 2 : 1) rmsnorm_kernel(const uint4 *__restrict__ x,
                                                       const uint4 *__restrict__ w,
                                                       void *__restrict__ y, int64_t M, int H,
                                                       float eps)
{
    __shared__ float part[R][32];
    const int chunks = H >> 3;
    const int T = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float h_den = static_cast<float>(H);

    for (int64_t row0 = int64_t(blockIdx.x) * R; row0 < M; row0 += int64_t(gridDim.x) * R) {
        uint4 v[R][ITEMS];
        float acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            acc[r] = 0.0f;
            const int64_t row = row0 + r;
#pragma unroll
            for (int it = 0; it < ITEMS; ++it) {
                const int c = threadIdx.x + it * T;
                if (row < M && c < chunks) v[r][it] = __ldcs(x + row * chunks + c);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
            for (int it = 0; it < ITEMS; ++it) {
                const int c = threadIdx.x + it * T;
                if (row0 + r < M && c < chunks) acc[r] = sumsq8(v[r][it], acc[r]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                acc[r] = __fadd_rn(acc[r], __shfl_xor_sync(0xffffffffu, acc[r], off));
            if (lane == 0) part[r][warp] = acc[r];
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t row = row0 + r;
            if (row >= M) break;
            float tot = 0.0f;
            for (int i = 0; i < (T >> 5); ++i) tot = __fadd_rn(tot, part[r][i]);
            const float rstd = rsqrtf(__fadd_rn(__fdiv_rn(tot, h_den), eps));
#pragma unroll
            for (int it = 0; it < ITEMS; ++it) {
                const int c = threadIdx.x + it * T;
                if (c < chunks) store8<OUT_F32>(y, row * chunks + c, v[r][it], __ldg(w + c), rstd);
            }
        }
        __syncthreads();  // part[] is reused by the next group of rows
    }
}

template <int ITEMS, int R, int MAXT>
cudaError_t launch_rows(const void *x, const void *w, void *y, int64_t M, int H, float eps,
                        bool out_f32, int threads, cudaStream_t s)
{
    const int64_t cap = int64_t(1) << 20;
    const int64_t groups = (M + R - 1) / R;
    const unsigned grid = static_cast<unsigned>(groups < cap ? groups : cap);
    if (out_f32)
        rmsnorm_kernel<ITEMS, R, true, MAXT><<<grid, threads, 0, s>>>(
            static_cast<const uint4 *>(x), static_cast<const uint4 *>(w), y, M, H, eps);
    else
        rmsnorm_kernel<ITEMS, R, false, MAXT><<<grid, threads, 0, s>>>(
            static_cast<const uint4 *>(x), static_cast<const uint4 *>(w), y, M, H, eps);
    return cudaGetLastError();
}

// Rows per block R with ITEMS * R 16-byte chunks held per thread: up to 16
// (64 registers) for blocks of at most 256 threads, two blocks per SM;
// up to 8 for wider blocks.
template <int ITEMS>
cudaError_t launch_items(const void *x, const void *w, void *y, int64_t M, int H, float eps,
                         bool out_f32, int threads, int rows_per_block, cudaStream_t s)
{
    if (threads <= 256) {
        if constexpr (ITEMS <= 2)
            if (rows_per_block >= 8)
                return launch_rows<ITEMS, 8, 256>(x, w, y, M, H, eps, out_f32, threads, s);
        if constexpr (ITEMS <= 4)
            if (rows_per_block >= 4)
                return launch_rows<ITEMS, 4, 256>(x, w, y, M, H, eps, out_f32, threads, s);
        if (rows_per_block >= 2) return launch_rows<ITEMS, 2, 256>(x, w, y, M, H, eps, out_f32, threads, s);
        return launch_rows<ITEMS, 1, 256>(x, w, y, M, H, eps, out_f32, threads, s);
    }
    if constexpr (ITEMS <= 4)
        if (rows_per_block >= 2)
            return launch_rows<ITEMS, 2, 1024>(x, w, y, M, H, eps, out_f32, threads, s);
    return launch_rows<ITEMS, 1, 1024>(x, w, y, M, H, eps, out_f32, threads, s);
}

}  // namespace

// Block shape of a row: ITEMS 16-byte chunks per thread, T threads; a
// function of H alone.
void rmsnorm_shape(int64_t H, int *items, int *threads)
{
    const int64_t chunks = H / 8;
    int it = 1;
    while (it < 8 && (chunks + it - 1) / it > 256) it *= 2;
    int64_t t = (chunks + it - 1) / it;
    t = (t + 31) / 32 * 32;
    *items = it;
    *threads = static_cast<int>(t);
}

cudaError_t launch_rmsnorm(const void *x, const void *w, void *y, int64_t M, int64_t H,
                           float eps, bool out_f32, int num_sms, cudaStream_t s)
{
    int items, threads;
    rmsnorm_shape(H, &items, &threads);
#if !BI_INVARIANT
    // Variant-off: a small batch spreads each row over twice as many
    // threads, which changes the order of its sum of squares with M.
    if (M < 2 * num_sms && items > 1) {
        items /= 2;
        int64_t t = (H / 8 + items - 1) / items;
        threads = static_cast<int>((t + 31) / 32 * 32);
    }
#endif
    // Rows per block: enough that two blocks per SM cover M in one wave,
    // within the registers a thread may hold (ITEMS * R <= 16; 8 for blocks
    // wider than 256 threads).
    const int64_t blocks = int64_t(num_sms) * (threads <= 256 ? 2 : 1);
    const int cap = threads <= 256 ? 16 : 8;
    int rpb = 1;
    while (rpb < 8 && int64_t(rpb) * blocks < M && items * rpb * 2 <= cap) rpb *= 2;
    const int h = static_cast<int>(H);
    switch (items) {
    case 1: return launch_items<1>(x, w, y, M, h, eps, out_f32, threads, rpb, s);
    case 2: return launch_items<2>(x, w, y, M, h, eps, out_f32, threads, rpb, s);
    case 4: return launch_items<4>(x, w, y, M, h, eps, out_f32, threads, rpb, s);
    default: return launch_items<8>(x, w, y, M, h, eps, out_f32, threads, rpb, s);
    }
}

}  // namespace bi
