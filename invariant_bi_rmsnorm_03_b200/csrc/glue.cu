// glue.cu -- the elementwise and per-row operations of a decoder layer around
// the three batch-invariant kernels: token embedding, rotary position
// embedding fused with the KV-cache write, SwiGLU, and the greedy argmax.
//
// The reports on "Defeating Nondeterminism in LLM Inference" measure
// invariance end to end by completing one prompt greedily many times among
// other requests and counting the distinct completions (xitu-tech news,
// "显著成果与高昂成本"; liuwei.blog, "实验成果").  They name no layer beyond
// RMSNorm, matmul and attention; the decoder is read as the plain pre-norm
// transformer.  Every operation here computes each output element (or each
// row's argmax) from its own row's inputs only, in an order fixed by the
// row's shape, so it is batch-invariant by construction.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"

namespace bi {
namespace {

__device__ __forceinline__ float lo16(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi16(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack2(float a, float b)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&p);
}

// ---------------------------------------------------------------- embedding
// out[t, :] = table[ids[t], :]: one thread per 16-byte piece.
__global__ void embedding_kernel(const uint4 *__restrict__ table, int64_t V, int pieces,
                                 const int32_t *__restrict__ ids, uint4 *__restrict__ out,
                                 int64_t T, unsigned *status)
{
    const int64_t n = T * pieces;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = i / pieces;
        const int p = static_cast<int>(i - t * pieces);
        const int64_t id = __ldg(ids + t);
        if (id < 0 || id >= V) {
            if (p == 0) record_status(status, BI_DEV_BAD_INDEX);
            continue;
        }
        out[i] = __ldg(table + id * pieces + p);
    }
}

// ---------------------------------------------------------------- RoPE
// One block per token (grid-stride).  The token's d/2 rotation angles
// angle_i = pos * theta^(-2i/d) and their cosine and sine are evaluated in
// double precision once per token and rounded to float; then each 16-byte
// piece pair (values 8c..8c+7 and d/2+8c..d/2+8c+7) of every q and k head
// is rotated in fp32:
//   lo' = round(round(lo cos) - round(hi sin)),  hi' = round(round(hi cos) + round(lo sin))
// and rounded to bf16.  q goes to q_out [T, Hq, d]; the rotated k and the
// unchanged v go to the token's cache slot (page blocks in core-matrix
// order: value 8vg + c of token 8kg + r at piece (kg * d/8 + vg) * 8 + r).
constexpr int kRopeThreads = 256;
constexpr int kMaxHalf = 64;  // head_dim <= 128

__global__ void __launch_bounds__(kRopeThreads)
rope_kv_kernel(const uint4 *__restrict__ qkv, const int32_t *__restrict__ pos,
               const int64_t *__restrict__ slots, uint4 *__restrict__ q_out, uint4 *k_cache,
               uint4 *v_cache, int64_t num_pages, int Hq, int Hkv, int d, double theta, int64_t T,
               unsigned *status)
{
    __shared__ float cs[kMaxHalf], sn[kMaxHalf];
    const int half = d / 2;
    const int pieces = d / 8;          // 16-byte pieces of a head
    const int hp = half / 8;           // pieces of a half head
    const int row_pieces = (Hq + 2 * Hkv) * pieces;
    const int rot_items = (Hq + Hkv) * hp;    // rotated piece pairs of q and k
    const int items = rot_items + Hkv * pieces;  // + plain v pieces
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const int32_t p = __ldg(pos + t);
        const int64_t slot = __ldg(slots + t);
        __syncthreads();  // the previous token's angles are no longer read
        if (threadIdx.x < half) {
            const double inv = pow(theta, -2.0 * double(threadIdx.x) / double(d));
            double s, c;
            sincos(double(p) * inv, &s, &c);
            cs[threadIdx.x] = static_cast<float>(c);
            sn[threadIdx.x] = static_cast<float>(s);
        }
        __syncthreads();
        bool write_kv = slot >= 0;
        if (slot >= num_pages * kPage) {
            write_kv = false;
            if (threadIdx.x == 0) record_status(status, BI_DEV_BAD_INDEX);
        }
        const int64_t page = slot / kPage;
        const int off = static_cast<int>(slot % kPage);
        // piece of the cache block holding token `off`, value piece vg
        const int64_t blk_row = (off >> 3) * (8 * pieces) + (off & 7);
        const uint4 *row = qkv + t * row_pieces;
        for (int it = threadIdx.x; it < items; it += blockDim.x) {
            if (it < rot_items) {
                const int h = it / hp;          // 0..Hq-1 q heads, then k heads
                const int c = it - h * hp;      // piece of the low half
                const uint4 a = row[h * pieces + c];
                const uint4 b = row[h * pieces + hp + c];
                const uint32_t av[4] = {a.x, a.y, a.z, a.w};
                const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i0 = 8 * c + 2 * k;
                    const float c0 = cs[i0], s0 = sn[i0], c1 = cs[i0 + 1], s1 = sn[i0 + 1];
                    const float a0 = lo16(av[k]), a1 = hi16(av[k]);
                    const float b0 = lo16(bv[k]), b1 = hi16(bv[k]);
                    lo[k] = pack2(__fsub_rn(__fmul_rn(a0, c0), __fmul_rn(b0, s0)),
                                  __fsub_rn(__fmul_rn(a1, c1), __fmul_rn(b1, s1)));
                    hi[k] = pack2(__fadd_rn(__fmul_rn(b0, c0), __fmul_rn(a0, s0)),
                                  __fadd_rn(__fmul_rn(b1, c1), __fmul_rn(a1, s1)));
                }
                const uint4 lo4 = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                const uint4 hi4 = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                if (h < Hq) {
                    uint4 *qo = q_out + (t * Hq + h) * pieces;
                    qo[c] = lo4;
                    qo[hp + c] = hi4;
                } else if (write_kv) {
                    const int g = h - Hq;
                    uint4 *blk = k_cache + (page * Hkv + g) * (kPage * pieces) + blk_row;
                    blk[c * 8] = lo4;
                    blk[(hp + c) * 8] = hi4;
                }
            } else if (write_kv) {
                const int j = it - rot_items;
                const int g = j / pieces;
                const int vg = j - g * pieces;
                v_cache[(page * Hkv + g) * (kPage * pieces) + blk_row + vg * 8] =
                    row[(Hq + Hkv + g) * pieces + vg];
            }
        }
    }
}

// ---------------------------------------------------------------- SwiGLU
// out[t, j] = round( silu(g) * u ),  g = gu[t, j], u = gu[t, F + j],
// silu(g) = g / (1 + e^-g), fp32; one thread per 8 outputs.
__global__ void swiglu_kernel(const uint4 *__restrict__ gu, uint4 *__restrict__ out, int64_t T,
                              int64_t fp)
{
    const int64_t n = T * fp;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = i / fp;
        const int64_t c = i - t * fp;
        const uint4 g4 = __ldcs(gu + t * 2 * fp + c);
        const uint4 u4 = __ldcs(gu + t * 2 * fp + fp + c);
        const uint32_t gv[4] = {g4.x, g4.y, g4.z, g4.w};
        const uint32_t uv[4] = {u4.x, u4.y, u4.z, u4.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float g0 = lo16(gv[k]), g1 = hi16(gv[k]);
            const float s0 = __fdiv_rn(g0, __fadd_rn(1.0f, expf(-g0)));
            const float s1 = __fdiv_rn(g1, __fadd_rn(1.0f, expf(-g1)));
            o[k] = pack2(__fmul_rn(s0, lo16(uv[k])), __fmul_rn(s1, hi16(uv[k])));
        }
        __stcs(out + i, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

// The same angles as a table [P, d/2] of (cos, sin), for the QKV epilogue
// of the matmul: the same expressions, so the same floats.
__global__ void rope_table_kernel(float2 *__restrict__ table, int P, int d, double theta)
{
    const int half = d / 2;
    const int64_t n = int64_t(P) * half;
    for (int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; k < n;
         k += int64_t(gridDim.x) * blockDim.x) {
        const int p = static_cast<int>(k / half);
        const int i = static_cast<int>(k - int64_t(p) * half);
        const double inv = pow(theta, -2.0 * double(i) / double(d));
        double sv, cv;
        sincos(double(p) * inv, &sv, &cv);
        table[k] = make_float2(static_cast<float>(cv), static_cast<float>(sv));
    }
}

// ---------------------------------------------------------------- norm-weight fold
// wf[n, k] = round(W[n, k] * w[k]): the product of two bf16 values is exact
// in fp32, so this is the correctly rounded product.  Eight per thread.
__global__ void fold_norm_weight_kernel(const uint4 *__restrict__ W, const uint4 *__restrict__ w,
                                        uint4 *__restrict__ wf, int64_t N, int64_t kp)
{
    const int64_t n = N * kp;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t k = i % kp;
        const uint4 a = W[i], b = __ldg(w + k);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = pack2(__fmul_rn(lo16(av[j]), lo16(bv[j])), __fmul_rn(hi16(av[j]), hi16(bv[j])));
        wf[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ---------------------------------------------------------------- argmax
// One block per row (grid-stride): each thread scans its float4 pieces in
// index order, then the (value, index) pairs are combined by a warp
// butterfly and across warps.  The combination keeps the larger value and,
// on equal values, the lower index: an exact selection, the same whatever
// the order of combination.  NaN entries are never selected.
constexpr int kArgmaxThreads = 512;

struct Best {
    float v;
    int32_t i;
};

__device__ __forceinline__ Best better(Best a, Best b)
{
    return (b.v > a.v || (b.v == a.v && b.i < a.i)) ? b : a;
}

__global__ void __launch_bounds__(kArgmaxThreads)
argmax_kernel(const float4 *__restrict__ logits, int64_t T, int64_t V, int32_t *__restrict__ out)
{
    __shared__ Best part[kArgmaxThreads / 32];
    const int64_t q = V / 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        Best b{-INFINITY, INT32_MAX};
        const float4 *row = logits + t * q;
        for (int64_t c = threadIdx.x; c < q; c += blockDim.x) {
            const float4 v = __ldcs(row + c);
            const int32_t j = static_cast<int32_t>(4 * c);
            b = better(b, Best{v.x, j});
            b = better(b, Best{v.y, j + 1});
            b = better(b, Best{v.z, j + 2});
            b = better(b, Best{v.w, j + 3});
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            Best o;
            o.v = __shfl_xor_sync(0xffffffffu, b.v, off);
            o.i = __shfl_xor_sync(0xffffffffu, b.i, off);
            b = better(b, o);
        }
        if (lane == 0) part[warp] = b;
        __syncthreads();
        if (threadIdx.x == 0) {
            Best r = part[0];
            for (int k = 1; k < int(blockDim.x >> 5); ++k) r = better(r, part[k]);
            out[t] = r.i == INT32_MAX ? 0 : r.i;  // a row of NaN only: index 0
        }
        __syncthreads();  // part[] is reused by the next row
    }
}

// ---------------------------------------------------------------- sampling
// One block per row (grid-stride), the row's weights cached in shared
// memory.  Every reduction has an order fixed by V and the block size alone:
// thread i takes elements i, i + T, ... in turn, then a warp xor-butterfly
// (commutative, so every lane gets the same bits), then warps 0..W-1 in
// order.  The row's draw comes from Philox4x32-10 (Salmon et al., SC 2011)
// keyed by the request's seed at a counter made of its offset.
constexpr int kSampleThreads = 512;

struct Philox {
    uint32_t c[4];
    uint32_t k[2];
};

__device__ __forceinline__ uint32_t philox_word0(uint64_t seed, uint64_t offset)
{
    uint32_t c0 = uint32_t(offset), c1 = uint32_t(offset >> 32), c2 = 0u, c3 = 0u;
    uint32_t k0 = uint32_t(seed), k1 = uint32_t(seed >> 32);
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
        const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
        const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
        k0 += 0x9E3779B9u;  // the key for the next round
        k1 += 0xBB67AE85u;
    }
    return c0;
}

// Sum over the block of one value per thread: butterfly in each warp, then
// the warp sums in order.  `red` holds kSampleThreads / 32 floats.
__device__ __forceinline__ float block_sum(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();  // red[] free
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float tot = 0.0f;
    for (int i = 0; i < int(blockDim.x >> 5); ++i) tot = __fadd_rn(tot, red[i]);
    return tot;
}

__device__ __forceinline__ float block_max(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float m = red[0];
    for (int i = 1; i < int(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
    return m;
}

__device__ __forceinline__ int block_min_int(int v, int *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int m = red[0];
    for (int i = 1; i < int(blockDim.x >> 5); ++i) m = min(m, red[i]);
    return m;
}

__global__ void __launch_bounds__(kSampleThreads)
sample_kernel(const float *__restrict__ logits, int64_t T, int V,
              const float *__restrict__ temperature, const float *__restrict__ top_p,
              const uint64_t *__restrict__ seed, const uint64_t *__restrict__ offset,
              int32_t *__restrict__ out)
{
    extern __shared__ float w[];                 // [V] weights of the row
    __shared__ float redf[kSampleThreads / 32];
    __shared__ int redi[kSampleThreads / 32];
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const float *row = logits + t * int64_t(V);
        const float temp = temperature[t];
        if (!(temp > 0.0f)) {
            // greedy: the largest logit, lowest index on ties
            float bv = -INFINITY;
            int bi = INT32_MAX;
            for (int j = tid; j < V; j += nt) {
                const float x = row[j];
                if (x > bv || (x == bv && j < bi)) {
                    bv = x;
                    bi = j;
                }
            }
            const float m = block_max(bv, redf);
            const int idx = block_min_int(bv == m ? bi : INT32_MAX, redi);
            if (tid == 0) out[t] = idx == INT32_MAX ? 0 : idx;
            continue;
        }
        // z_j = logit_j / temperature; weights w_j = e^(z_j - max z)
        float mx = -INFINITY;
        for (int j = tid; j < V; j += nt) mx = fmaxf(mx, __fdiv_rn(row[j], temp));
        mx = block_max(mx, redf);
        float part = 0.0f;
        for (int j = tid; j < V; j += nt) {
            const float e = expf(__fsub_rn(__fdiv_rn(row[j], temp), mx));
            w[j] = e;
            part = __fadd_rn(part, e);
        }
        const float total = block_sum(part, redf);
        // nucleus threshold: the largest tau with sum_{w >= tau} w >= top_p * total,
        // found by bisection on the bit pattern (positive floats order like
        // their bits); each probe is a sum in the fixed order above.
        uint32_t lo = 0u, hi = 0x3F800001u;  // S(0) = total, S(> 1) = 0
        float zk = total;
        const float tp = top_p[t];
        if (tp < 1.0f) {
            const float need = __fmul_rn(tp, total);
            while (hi - lo > 1u) {
                const uint32_t mid = lo + ((hi - lo) >> 1);
                const float tau = __uint_as_float(mid);
                float ps = 0.0f;
                for (int j = tid; j < V; j += nt)
                    if (w[j] >= tau) ps = __fadd_rn(ps, w[j]);
                const float S = block_sum(ps, redf);
                if (S >= need) {
                    lo = mid;
                    zk = S;
                } else {
                    hi = mid;
                }
            }
            if (lo == 0u) zk = total;
        }
        const float tau = __uint_as_float(lo);
        // the draw and the target mass
        const float u = float(philox_word0(seed[t], offset[t]) >> 8) * (1.0f / 16777216.0f);
        const float target = __fmul_rn(u, zk);
        // walk the kept weights in index order: thread i owns the contiguous
        // range [i C, (i+1) C); range sums, an exclusive scan of them over the
        // threads (a fixed tree), then each thread walks its range.
        const int C = (V + nt - 1) / nt;
        const int j0 = tid * C, j1 = min(V, j0 + C);
        float rs = 0.0f;
        for (int j = j0; j < j1; ++j)
            if (w[j] >= tau) rs = __fadd_rn(rs, w[j]);
        float inc = rs;
        const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc = __fadd_rn(inc, y);
        }
        __syncthreads();
        if (lane == 31) redf[warp] = inc;
        __syncthreads();
        float before = 0.0f;  // sum of the warps before this one, in order
        for (int i = 0; i < warp; ++i) before = __fadd_rn(before, redf[i]);
        float run = __fadd_rn(before, __fsub_rn(inc, rs));  // exclusive prefix
        int cand = INT32_MAX, last = -1;
        for (int j = j0; j < j1; ++j) {
            if (!(w[j] >= tau)) continue;
            last = j;
            run = __fadd_rn(run, w[j]);
            if (run > target) {
                cand = j;
                break;
            }
        }
        int tok = block_min_int(cand, redi);
        if (tok == INT32_MAX) tok = -block_min_int(-last, redi);  // past the end: the last kept
        if (tid == 0) out[t] = tok < 0 ? 0 : tok;
        __syncthreads();  // w[] and the scratch are reused by the next row
    }
}

unsigned grid_for(int64_t items, int threads, int num_sms)
{
    const int64_t blocks = (items + threads - 1) / threads;
    const int64_t cap = int64_t(num_sms) * 8;
    return static_cast<unsigned>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

size_t sample_smem_bytes(int64_t V) { return size_t(V) * sizeof(float); }

cudaError_t launch_sample(const float *logits, int64_t T, int64_t V, const float *temperature,
                          const float *top_p, const uint64_t *seed, const uint64_t *offset,
                          int32_t *out, int num_sms, cudaStream_t s)
{
    const size_t smem = sample_smem_bytes(V);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(kMaxSampleVocab * sizeof(float)));
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int64_t cap = int64_t(num_sms);
    const unsigned grid = static_cast<unsigned>(T < cap ? T : cap);
    sample_kernel<<<grid, kSampleThreads, smem, s>>>(logits, T, int(V), temperature, top_p, seed,
                                                     offset, out);
    return cudaGetLastError();
}

cudaError_t launch_embedding(const void *table, int64_t V, int64_t H, const int32_t *ids,
                             void *out, int64_t T, unsigned *status, int num_sms, cudaStream_t s)
{
    const int pieces = static_cast<int>(H / 8);
    embedding_kernel<<<grid_for(T * pieces, 256, num_sms), 256, 0, s>>>(
        static_cast<const uint4 *>(table), V, pieces, ids, static_cast<uint4 *>(out), T, status);
    return cudaGetLastError();
}

cudaError_t launch_rope_kv(const void *qkv, const int32_t *pos, const int64_t *slots,
                           void *q_out, void *k_cache, void *v_cache, int64_t num_pages, int Hq,
                           int Hkv, int d, double theta, int64_t T, unsigned *status, int num_sms,
                           cudaStream_t s)
{
    const int64_t cap = int64_t(num_sms) * 8;
    const unsigned grid = static_cast<unsigned>(T < cap ? T : cap);
    rope_kv_kernel<<<grid, kRopeThreads, 0, s>>>(
        static_cast<const uint4 *>(qkv), pos, slots, static_cast<uint4 *>(q_out),
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), num_pages, Hq, Hkv, d,
        theta, T, status);
    return cudaGetLastError();
}

cudaError_t launch_swiglu(const void *gu, void *out, int64_t T, int64_t F, int num_sms,
                          cudaStream_t s)
{
    const int64_t fp = F / 8;
    swiglu_kernel<<<grid_for(T * fp, 256, num_sms), 256, 0, s>>>(
        static_cast<const uint4 *>(gu), static_cast<uint4 *>(out), T, fp);
    return cudaGetLastError();
}

cudaError_t launch_rope_table(float *table, int P, int d, double theta, int num_sms,
                              cudaStream_t s)
{
    rope_table_kernel<<<grid_for(int64_t(P) * (d / 2), 256, num_sms), 256, 0, s>>>(
        reinterpret_cast<float2 *>(table), P, d, theta);
    return cudaGetLastError();
}

cudaError_t launch_fold_norm_weight(const void *W, const void *w, void *wf, int64_t N, int64_t K,
                                    int num_sms, cudaStream_t s)
{
    const int64_t kp = K / 8;
    fold_norm_weight_kernel<<<grid_for(N * kp, 256, num_sms), 256, 0, s>>>(
        static_cast<const uint4 *>(W), static_cast<const uint4 *>(w), static_cast<uint4 *>(wf), N,
        kp);
    return cudaGetLastError();
}

cudaError_t launch_argmax(const float *logits, int64_t T, int64_t V, int32_t *out, int num_sms,
                          cudaStream_t s)
{
    const int64_t cap = int64_t(num_sms) * 4;
    const unsigned grid = static_cast<unsigned>(T < cap ? T : cap);
    argmax_kernel<<<grid, kArgmaxThreads, 0, s>>>(reinterpret_cast<const float4 *>(logits), T, V,
                                                  out);
    return cudaGetLastError();
}

}  // namespace bi
