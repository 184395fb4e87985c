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
//   SwiGLU    elementwise: each gradient from its own (gate, up, dout) only.
//   RoPE      elementwise per pair: the rotation by the negative angle, with
//             the forward's angles (double precision, rounded to float).
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

// ---------------------------------------------------------------- SwiGLU
// With s = 1 / (1 + e^-g) (the sigmoid), out = g s u:
//   dup   = dout (g s)
//   dgate = (dout u) (s + (g s) s'),   s' = 1 / (1 + e^g) = 1 - s
// s' is evaluated as its own sigmoid rather than as 1 - s, which loses the
// small values of 1 - s for large g; neither form overflows to NaN.  fp32,
// every operation rounded; one thread per 8 outputs of each half.
template <bool OUT_F32>
__global__ void swiglu_bwd_kernel(const uint4 *__restrict__ gu, const uint4 *__restrict__ dout,
                                  void *__restrict__ dgu, int64_t T, int64_t fp)
{
    const int64_t n = T * fp;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = i / fp;
        const int64_t c = i - t * fp;
        const uint4 g4 = __ldcs(gu + t * 2 * fp + c);
        const uint4 u4 = __ldcs(gu + t * 2 * fp + fp + c);
        const uint4 d4 = __ldcs(dout + i);
        const uint32_t gv[4] = {g4.x, g4.y, g4.z, g4.w};
        const uint32_t uv[4] = {u4.x, u4.y, u4.z, u4.w};
        const uint32_t dv[4] = {d4.x, d4.y, d4.z, d4.w};
        float dg[8], du[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float g = (k & 1) ? hi_f(gv[k >> 1]) : lo_f(gv[k >> 1]);
            const float u = (k & 1) ? hi_f(uv[k >> 1]) : lo_f(uv[k >> 1]);
            const float d = (k & 1) ? hi_f(dv[k >> 1]) : lo_f(dv[k >> 1]);
            const float s = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-g)));
            const float sc = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(g)));
            const float gs = __fmul_rn(g, s);
            du[k] = __fmul_rn(d, gs);
            dg[k] = __fmul_rn(__fmul_rn(d, u), __fadd_rn(s, __fmul_rn(gs, sc)));
        }
        const int64_t og = t * 2 * fp + c, ou = og + fp;  // 8-value pieces of dgate, dup
        if constexpr (OUT_F32) {
            float4 *o = static_cast<float4 *>(dgu);
            o[2 * og] = make_float4(dg[0], dg[1], dg[2], dg[3]);
            o[2 * og + 1] = make_float4(dg[4], dg[5], dg[6], dg[7]);
            o[2 * ou] = make_float4(du[0], du[1], du[2], du[3]);
            o[2 * ou + 1] = make_float4(du[4], du[5], du[6], du[7]);
        } else {
            uint4 *o = static_cast<uint4 *>(dgu);
            o[og] = make_uint4(pack_rn(dg[0], dg[1]), pack_rn(dg[2], dg[3]), pack_rn(dg[4], dg[5]),
                               pack_rn(dg[6], dg[7]));
            o[ou] = make_uint4(pack_rn(du[0], du[1]), pack_rn(du[2], du[3]), pack_rn(du[4], du[5]),
                               pack_rn(du[6], du[7]));
        }
    }
}

// ---------------------------------------------------------------- RoPE
// The forward rotates the pair (x_i, x_{i+d/2}) by the angle
// a_i = pos theta^(-2i/d); its transpose rotates the upstream gradient back:
//   dx_i       = round(round(dy_i cos) + round(dy_{i+d/2} sin))
//   dx_{i+d/2} = round(round(dy_{i+d/2} cos) - round(dy_i sin))
// with cos and sin evaluated in double precision and rounded to float, as
// the forward does.  One block per token (grid-stride); each thread rotates
// a pair of 8-value pieces of one head.  dy and dx rows are ld_dy / ld_dx
// values apart (a head set inside a wider row, e.g. the q part of a fused
// q/k/v gradient).
constexpr int kRopeBwdThreads = 256;

template <bool OUT_F32>
__global__ void __launch_bounds__(kRopeBwdThreads)
rope_bwd_kernel(const uint16_t *__restrict__ dy, int64_t ld_dy, const int32_t *__restrict__ pos,
                void *__restrict__ dx, int64_t ld_dx, int64_t T, int nh, int d, double theta)
{
    __shared__ float cs[64], sn[64];
    const int half = d / 2, hp = half / 8;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const int32_t p = __ldg(pos + t);
        __syncthreads();  // the previous token's angles are no longer read
        if (threadIdx.x < half) {
            const double inv = pow(theta, -2.0 * double(threadIdx.x) / double(d));
            double sv, cv;
            sincos(double(p) * inv, &sv, &cv);
            cs[threadIdx.x] = static_cast<float>(cv);
            sn[threadIdx.x] = static_cast<float>(sv);
        }
        __syncthreads();
        for (int it = threadIdx.x; it < nh * hp; it += blockDim.x) {
            const int h = it / hp, c = it - h * hp;
            const uint16_t *row = dy + t * ld_dy + int64_t(h) * d;
            const uint4 a = *reinterpret_cast<const uint4 *>(row + 8 * c);
            const uint4 b = *reinterpret_cast<const uint4 *>(row + half + 8 * c);
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
            float lo[8], hi[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int i = 8 * c + k;
                const float l = (k & 1) ? hi_f(av[k >> 1]) : lo_f(av[k >> 1]);
                const float u = (k & 1) ? hi_f(bv[k >> 1]) : lo_f(bv[k >> 1]);
                lo[k] = __fadd_rn(__fmul_rn(l, cs[i]), __fmul_rn(u, sn[i]));
                hi[k] = __fsub_rn(__fmul_rn(u, cs[i]), __fmul_rn(l, sn[i]));
            }
            const int64_t o = t * ld_dx + int64_t(h) * d;
            if constexpr (OUT_F32) {
                float *orow = static_cast<float *>(dx) + o;
                float4 *ol = reinterpret_cast<float4 *>(orow + 8 * c);
                float4 *oh = reinterpret_cast<float4 *>(orow + half + 8 * c);
                ol[0] = make_float4(lo[0], lo[1], lo[2], lo[3]);
                ol[1] = make_float4(lo[4], lo[5], lo[6], lo[7]);
                oh[0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
                oh[1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
            } else {
                uint16_t *orow = static_cast<uint16_t *>(dx) + o;
                *reinterpret_cast<uint4 *>(orow + 8 * c) =
                    make_uint4(pack_rn(lo[0], lo[1]), pack_rn(lo[2], lo[3]), pack_rn(lo[4], lo[5]),
                               pack_rn(lo[6], lo[7]));
                *reinterpret_cast<uint4 *>(orow + half + 8 * c) =
                    make_uint4(pack_rn(hi[0], hi[1]), pack_rn(hi[2], hi[3]), pack_rn(hi[4], hi[5]),
                               pack_rn(hi[6], hi[7]));
            }
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

cudaError_t launch_swiglu_backward(const void *gu, const void *dout, void *dgu, int64_t T,
                                   int64_t F, bool out_f32, int num_sms, cudaStream_t s)
{
    const int64_t fp = F / 8, items = T * fp;
    const int64_t blocks = (items + 255) / 256, cap = int64_t(num_sms) * 8;
    const unsigned g = static_cast<unsigned>(blocks < cap ? blocks : cap);
    const uint4 *a = static_cast<const uint4 *>(gu), *b = static_cast<const uint4 *>(dout);
    if (out_f32)
        swiglu_bwd_kernel<true><<<g, 256, 0, s>>>(a, b, dgu, T, fp);
    else
        swiglu_bwd_kernel<false><<<g, 256, 0, s>>>(a, b, dgu, T, fp);
    return cudaGetLastError();
}

cudaError_t launch_rope_backward(const void *dy, int64_t ld_dy, const int32_t *pos, void *dx,
                                 int64_t ld_dx, int64_t T, int nh, int d, double theta,
                                 bool out_f32, int num_sms, cudaStream_t s)
{
    const int64_t cap = int64_t(num_sms) * 8;
    const unsigned g = static_cast<unsigned>(T < cap ? T : cap);
    const uint16_t *src = static_cast<const uint16_t *>(dy);
    if (out_f32)
        rope_bwd_kernel<true><<<g, kRopeBwdThreads, 0, s>>>(src, ld_dy, pos, dx, ld_dx, T, nh, d,
                                                              theta);
    else
        rope_bwd_kernel<false><<<g, kRopeBwdThreads, 0, s>>>(src, ld_dy, pos, dx, ld_dx, T, nh, d,
                                                               theta);
    return cudaGetLastError();
}

}  // namespace bi
