// moe.cu -- the mixture-of-experts feed-forward around the batch-invariant
// matmul: router top-k, grouping of tokens by expert, gate-weighted combine.
//
// The model of the reports' experiment is a mixture of experts (Qwen3-235B-
// A22B; xitu-tech news, "显著成果与高昂成本"; neican.ai insight,
// "技术原理与创新点解析"); they describe no router.  Each token picks its k
// experts by largest router logit (lowest index on ties); its gate weights
// are the softmax of the selected logits; its output is the gate-weighted
// sum of its experts' outputs in rank order.  Every step depends on the
// token's own row only; the expert matmuls run through bi_matmul, whose rows
// do not depend on how many tokens an expert received.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"

namespace bi {
namespace {

// ---------------------------------------------------------------- route
// One warp per token; lane l holds the logits of experts l, l + 32, ...
__global__ void moe_route_kernel(const float *__restrict__ logits, int64_t T, int E, int k,
                                 int32_t *__restrict__ experts, float *__restrict__ weights)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
         t += warps) {
        const float *row = logits + t * E;
        uint32_t taken = 0u;  // bit s: expert lane + 32 s already chosen
        int32_t chosen[kMaxMoeTopK];
        float val[kMaxMoeTopK];
        for (int i = 0; i < k; ++i) {
            float bv = -INFINITY;
            int be = INT32_MAX;
            for (int s = 0, e = lane; e < E; ++s, e += 32) {
                if (taken & (1u << s)) continue;
                const float x = row[e];
                if (x > bv || (x == bv && e < be)) {
                    bv = x;
                    be = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (ov > bv || (ov == bv && oe < be)) {
                    bv = ov;
                    be = oe;
                }
            }
            if (be == INT32_MAX) be = 0;  // no finite logit left (not expected)
            chosen[i] = be;
            val[i] = bv;
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
        }
        if (lane == 0) {
            float e[kMaxMoeTopK], s = 0.0f;
            for (int i = 0; i < k; ++i) {
                e[i] = expf(__fsub_rn(val[i], val[0]));
                s = __fadd_rn(s, e[i]);
            }
            for (int i = 0; i < k; ++i) {
                experts[t * k + i] = chosen[i];
                weights[t * k + i] = __fdiv_rn(e[i], s);
            }
        }
    }
}

// ---------------------------------------------------------------- dispatch
// One block.  Counts per expert, their exclusive scan (offsets), then the
// entries in index order, 1024 at a time: an entry's rank among the earlier
// entries of its expert is its rank inside its warp (__match_any_sync) plus
// the counts of the earlier warps of the chunk plus the earlier chunks'.
// Integer arithmetic only: the grouping is exact.
constexpr int kDispatchThreads = 1024;

__global__ void __launch_bounds__(kDispatchThreads)
moe_dispatch_kernel(const int32_t *__restrict__ experts, int64_t N, int E, int k,
                    int64_t *__restrict__ offsets, int64_t *__restrict__ order,
                    int64_t *__restrict__ pos, int32_t *__restrict__ token_sorted,
                    unsigned *status)
{
    __shared__ int64_t start[kMaxMoeExperts + 1];
    __shared__ int64_t done[kMaxMoeExperts];
    __shared__ int wcnt[kDispatchThreads / 32][kMaxMoeExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nw = kDispatchThreads / 32;
    for (int e = tid; e < E; e += blockDim.x) done[e] = 0;
    __syncthreads();
    // counts (the order of integer additions does not matter)
    for (int64_t i = tid; i < N; i += blockDim.x) {
        const int e = experts[i];
        if (e < 0 || e >= E) {
            record_status(status, BI_DEV_BAD_INDEX);
            continue;
        }
        atomicAdd(reinterpret_cast<unsigned long long *>(&done[e]), 1ull);
    }
    __syncthreads();
    if (tid == 0) {
        int64_t acc = 0;
        for (int e = 0; e < E; ++e) {
            start[e] = acc;
            offsets[e] = acc;
            acc += done[e];
        }
        start[E] = acc;
        offsets[E] = acc;
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) done[e] = 0;
    for (int64_t c0 = 0; c0 < N; c0 += kDispatchThreads) {
        for (int idx = tid; idx < nw * kMaxMoeExperts; idx += blockDim.x)
            (&wcnt[0][0])[idx] = 0;
        __syncthreads();
        const int64_t i = c0 + tid;
        int e = -1;
        if (i < N) {
            e = experts[i];
            if (e < 0 || e >= E) {
                e = -1;
                pos[i] = -1;  // flagged above; combine skips it
            }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int64_t p = start[e] + done[e] + rank;
            for (int w = 0; w < warp; ++w) p += wcnt[w][e];
            order[p] = i;
            pos[i] = p;
            token_sorted[p] = static_cast<int32_t>(i / k);
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x) {
            int64_t s = 0;
            for (int w = 0; w < nw; ++w) s += wcnt[w][ee];
            done[ee] += s;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- combine
// out[t, :] = round( sum_{i < k} w[t, i] * y[pos[t k + i], :] ), fp32, the
// terms added in rank order; one thread per 8 outputs.
__global__ void moe_combine_kernel(const uint4 *__restrict__ y, const int64_t *__restrict__ pos,
                                   const float *__restrict__ weights, int64_t T, int k,
                                   int64_t pieces, int64_t rows, uint4 *__restrict__ out,
                                   unsigned *status)
{
    const int64_t n = T * pieces;
    for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
         idx += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = idx / pieces;
        const int64_t c = idx - t * pieces;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int i = 0; i < k; ++i) {
            const float w = weights[t * k + i];
            const int64_t p = pos[t * k + i];
            if (p < 0 || p >= rows) {  // an entry the dispatch could not place
                if (c == 0) record_status(status, BI_DEV_BAD_INDEX);
                continue;
            }
            const uint4 v = __ldg(y + p * pieces + c);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[2 * j] = __fadd_rn(acc[2 * j], __fmul_rn(w, __uint_as_float(u[j] << 16)));
                acc[2 * j + 1] =
                    __fadd_rn(acc[2 * j + 1], __fmul_rn(w, __uint_as_float(u[j] & 0xFFFF0000u)));
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
            o[j] = *reinterpret_cast<uint32_t *>(&p);
        }
        out[idx] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_moe_route(const float *logits, int64_t T, int E, int k, int32_t *experts,
                             float *weights, int num_sms, cudaStream_t s)
{
    const int64_t blocks = (T + 7) / 8;  // 8 warps a block, a warp per token
    const int64_t cap = int64_t(num_sms) * 8;
    moe_route_kernel<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 256, 0, s>>>(
        logits, T, E, k, experts, weights);
    return cudaGetLastError();
}

cudaError_t launch_moe_dispatch(const int32_t *experts, int64_t N, int E, int k, int64_t *offsets,
                                int64_t *order, int64_t *pos, int32_t *token_sorted,
                                unsigned *status, cudaStream_t s)
{
    moe_dispatch_kernel<<<1, kDispatchThreads, 0, s>>>(experts, N, E, k, offsets, order, pos,
                                                       token_sorted, status);
    return cudaGetLastError();
}

cudaError_t launch_moe_combine(const void *y, const int64_t *pos, const float *weights, int64_t T,
                               int k, int64_t H, void *out, unsigned *status, int num_sms,
                               cudaStream_t s)
{
    const int64_t pieces = H / 8;
    const int64_t blocks = (T * pieces + 255) / 256;
    const int64_t cap = int64_t(num_sms) * 8;
    moe_combine_kernel<<<static_cast<unsigned>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap), 256,
                         0, s>>>(static_cast<const uint4 *>(y), pos, weights, T, k, pieces,
                                 T * k, static_cast<uint4 *>(out), status);
    return cudaGetLastError();
}

}  // namespace bi
