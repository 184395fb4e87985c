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
// Residual form (between the sublayers of a pre-norm decoder): x is first
// replaced by round(x + delta) (fp32 add, bf16 RNE) and written back, then
// normalised by the same code, so its y equals the plain form's y of the
// updated row bit for bit.
//
// Memory: a row is loaded once into registers with 128-bit streaming loads
// and written with 128-bit stores.  One row per block at a time, with many
// small blocks resident per SM (8 of 256 threads at H = 4096) so that the
// loads of some rows overlap the reduction and stores of others; the grid
// strides over rows.
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

__device__ __forceinline__ uint32_t add_pair(uint32_t a, uint32_t b)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(__fadd_rn(bf_lo(a), bf_lo(b)),
                                             __fadd_rn(bf_hi(a), bf_hi(b)));
    return *reinterpret_cast<uint32_t *>(&p);
}

// x <- round(x + delta), element by element in fp32.
__device__ __forceinline__ uint4 add8(const uint4 &a, const uint4 &b)
{
    return make_uint4(add_pair(a.x, b.x), add_pair(a.y, b.y), add_pair(a.z, b.z),
                      add_pair(a.w, b.w));
}

// One row per block iteration; the grid strides over rows.
// ADD: the residual form -- x is first replaced by round(x + delta) (and
// written back), then normalised exactly as the plain form normalises it.
// STATS: only the row's rstd is written, to ((float *) y)[row].
template <int ITEMS, bool OUT_F32, int MAXT, bool ADD, int MINB, bool STATS = false>
__global__ void __launch_bounds__(MAXT, MINB) rmsnorm_kernel(uint4 *x,
                                                       const uint4 *__restrict__ delta,
                                                       const uint4 *__restrict__ w,
                                                       void *__restrict__ y, int64_t M, int H,
                                                       float eps)
{
    __shared__ float part[32];
    const int chunks = H >> 3;
    const int T = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float h_den = static_cast<float>(H);

    for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
        uint4 v[ITEMS];
        uint4 dv[ADD ? ITEMS : 1];
#pragma unroll
        for (int it = 0; it < ITEMS; ++it) {
            const int c = threadIdx.x + it * T;
            if (c < chunks) {
                v[it] = __ldcs(x + row * chunks + c);
                if constexpr (ADD) dv[it] = __ldcs(delta + row * chunks + c);
            }
        }
        float acc = 0.0f;
#pragma unroll
        for (int it = 0; it < ITEMS; ++it) {
            const int c = threadIdx.x + it * T;
            if (c < chunks) {
                if constexpr (ADD) {
                    v[it] = add8(v[it], dv[it]);
                    x[row * chunks + c] = v[it];
                }
                acc = sumsq8(v[it], acc);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
        if (lane == 0) part[warp] = acc;
        __syncthreads();
        float tot = 0.0f;
        for (int i = 0; i < (T >> 5); ++i) tot = __fadd_rn(tot, part[i]);
        const float rstd = rsqrtf(__fadd_rn(__fdiv_rn(tot, h_den), eps));
        if constexpr (STATS) {
            if (threadIdx.x == 0) static_cast<float *>(y)[row] = rstd;
        } else {
#pragma unroll
            for (int it = 0; it < ITEMS; ++it) {
                const int c = threadIdx.x + it * T;
                if (c < chunks) store8<OUT_F32>(y, row * chunks + c, v[it], __ldg(w + c), rstd);
            }
        }
        __syncthreads();  // part[] is reused by the next row
    }
}

struct NormArgs {
    void *x;
    const void *delta;  // non-null: the residual form
    bool stats;         // write only each row's rstd (y is float [M])
    const void *w;
    void *y;
    int64_t M;
    int H;
    float eps;
    bool out_f32;
    int threads;
    int num_sms;
};

// Blocks resident per SM: as many as the 2048 threads of an SM hold, within
// the registers a thread needs (the row's ITEMS 16-byte chunks, twice that
// for the residual form).
template <int ITEMS, int MAXT, bool ADD>
constexpr int min_blocks()
{
    constexpr int full = 2048 / MAXT;                     // 8 or 2
    constexpr int data_regs = 4 * ITEMS * (ADD ? 2 : 1);  // registers of row data
    return data_regs <= 8 ? full : (data_regs <= 16 ? full / 2 : full / 4 > 0 ? full / 4 : 1);
}

template <int ITEMS, int MAXT, bool ADD>
cudaError_t launch_shape(const NormArgs &a, cudaStream_t s)
{
    constexpr int MINB = min_blocks<ITEMS, MAXT, ADD>();
    // Up to two waves of rows: every block takes rows in turn (grid of the
    // resident blocks); more rows: one block per row, the hardware refills.
    const int64_t resident = int64_t(a.num_sms) * MINB;
    const int64_t cap = int64_t(1) << 20;
    int64_t grid = a.M <= 2 * resident ? (a.M < resident ? a.M : resident) : a.M;
    if (grid > cap) grid = cap;
    uint4 *x = static_cast<uint4 *>(a.x);
    const uint4 *d = static_cast<const uint4 *>(a.delta);
    const uint4 *w = static_cast<const uint4 *>(a.w);
    const unsigned g = static_cast<unsigned>(grid);
    if (a.stats)
        rmsnorm_kernel<ITEMS, false, MAXT, false, MINB, true><<<g, a.threads, 0, s>>>(
            x, d, w, a.y, a.M, a.H, a.eps);
    else if (a.out_f32)
        rmsnorm_kernel<ITEMS, true, MAXT, ADD, MINB><<<g, a.threads, 0, s>>>(x, d, w, a.y, a.M,
                                                                             a.H, a.eps);
    else
        rmsnorm_kernel<ITEMS, false, MAXT, ADD, MINB><<<g, a.threads, 0, s>>>(x, d, w, a.y, a.M,
                                                                              a.H, a.eps);
    return cudaGetLastError();
}

template <int ITEMS, bool ADD>
cudaError_t launch_items(const NormArgs &a, cudaStream_t s)
{
    return a.threads <= 256 ? launch_shape<ITEMS, 256, ADD>(a, s)
                            : launch_shape<ITEMS, 1024, ADD>(a, s);
}

template <bool ADD>
cudaError_t launch_norm(const NormArgs &a, int items, cudaStream_t s)
{
    switch (items) {
    case 1: return launch_items<1, ADD>(a, s);
    case 2: return launch_items<2, ADD>(a, s);
    case 4: return launch_items<4, ADD>(a, s);
    default: return launch_items<8, ADD>(a, s);
    }
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

static cudaError_t launch_any(void *x, const void *delta, const void *w, void *y, int64_t M,
                              int64_t H, float eps, bool out_f32, int num_sms, cudaStream_t s,
                              bool stats = false)
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
    const NormArgs a{x, delta, stats, w, y, M, static_cast<int>(H), eps, out_f32, threads, num_sms};
    return delta ? launch_norm<true>(a, items, s) : launch_norm<false>(a, items, s);
}

cudaError_t launch_rmsnorm(const void *x, const void *w, void *y, int64_t M, int64_t H,
                           float eps, bool out_f32, int num_sms, cudaStream_t s)
{
    return launch_any(const_cast<void *>(x), nullptr, w, y, M, H, eps, out_f32, num_sms, s);
}

cudaError_t launch_add_rmsnorm(void *x, const void *delta, const void *w, void *y, int64_t M,
                               int64_t H, float eps, bool out_f32, int num_sms, cudaStream_t s)
{
    return launch_any(x, delta, w, y, M, H, eps, out_f32, num_sms, s);
}

cudaError_t launch_row_rstd(const void *x, float *r, int64_t M, int64_t H, float eps, int num_sms,
                            cudaStream_t s)
{
    return launch_any(const_cast<void *>(x), nullptr, nullptr, r, M, H, eps, false, num_sms, s,
                      true);
}

}  // namespace bi
