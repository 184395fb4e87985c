// gemm.cu -- batch-invariant matrix product C = A W^T on the 5th-generation
// tensor cores (tcgen05), fed by TMA.
//
// xitu-tech news, "构建确定性解决方案", matmul item: no split-K chosen from the
// input size; one fixed kernel configuration with one tile size.  neican.ai
// insight, "技术原理与创新点解析", data-parallel matmul bullet: the output is cut
// into 2-D tiles and each core computes its tiles' whole dot products.
//
// One configuration for every shape: 256 x 256 output tiles, each computed
// by a pair of SMs (a 2-CTA cluster, tcgen05.mma.cta_group::2), K consumed
// in 64-wide slices in ascending order, four K=16 MMAs per slice
// accumulating in fp32 in tensor memory.  Row m of A always lands in tile
// m / 256 at row m % 256 (CTA (m % 256) / 128 of the pair) and column n of
// W in tile n / 256, whatever M is; the K loop of an output element never
// depends on M, N or on which pair runs the tile.  Rows past M and K past
// the end are zero-filled by TMA.
//
// Each CTA of a pair: 192 threads, one per SM, persistent over tiles:
//   warp 0     TMA producer: this CTA's 128 rows of the A slice and 128 rows
//              of the W slice (128-byte swizzle, 32 KB a stage, 7 stages),
//              completing on the leader's barrier
//   warp 1     TMEM allocation (512 columns: two 128 x 256 fp32
//              accumulators, the pair allocating together) and, in the
//              leader, MMA issue by one thread
//   warps 2-5  epilogue: tcgen05.ld of this CTA's accumulator rows (each warp
//              its 32-lane quarter), fp32 -> bf16 rounding, global stores;
//              the second accumulator lets the next tile's MMAs run meanwhile.
//
// Fused forms (the RMSNorm and residual steps around a transformer block's
// matmuls, adjacent to the matmul item of xitu-tech news, "构建确定性解决方案"):
//   norm      C[m, :] = r[m] * (A W^T)[m, :], r[m] = rsqrt(mean_k A[m, k]^2 +
//             eps) computed beforehand by the RMSNorm kernel's own reduction
//             (one read of A, M floats written), with the norm weight folded
//             into W beforehand: the epilogue scales its row by r[m].  The MMA
//             operands are the stored bf16 values, and A is not read again
//             from shared memory for the statistics (which, done once per
//             output tile, took shared-memory bandwidth the tensor cores
//             need).
//   residual  C[m, :] = round(R[m, :] + round(acc[m, :])), R read in the
//             epilogue (it may be C itself).
//   QKV       the columns are q, k and v heads: the rounded product goes
//             through RoPE and the cache write in the epilogue (qkv_epilogue);
//             the library uses it together with the norm form.
// None of them changes the K order of the product; all of them act per row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"
#include "bi_ptx.cuh"

namespace bi {
namespace {

struct Unit {
    int mb, nb, split, kb0, kb1;
    int64_t row0;    // first row of A and C of the tile
    int64_t row_end; // rows at or past this one are not stored
    int64_t w_row0;  // first row of W (stacked groups: group * N + column)
};

__device__ __forceinline__ Unit unit_of(int u, int num_m, int k_splits, int kblocks, int kb_per)
{
    Unit r;
    r.split = u % k_splits;
    const int tile = u / k_splits;
    r.mb = tile % num_m;
    r.nb = tile / num_m;
    r.kb0 = r.split * kb_per;
    r.kb1 = min(kblocks, r.kb0 + kb_per);
    return r;
}

// Waits without looking at the abort flag: used only to let in-flight
// asynchronous copies and MMAs land before a block that gave up exits.
__device__ bool wait_drain(uint64_t *bar, uint32_t parity, uint64_t timeout_ns)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs))
        if (global_ns() - t0 > timeout_ns) return false;
    return true;
}

__device__ __forceinline__ void store_row32(const uint32_t (&r)[32], void *c, float *ws,
                                            int64_t row, int col0, int N, int M, int split,
                                            int k_splits, int out_f32)
{
    if (k_splits > 1 || out_f32) {
        float *dst = (k_splits > 1 ? ws + (int64_t(split) * M + row) * N
                                   : static_cast<float *>(c) + row * N) +
                     col0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (col0 + 8 * g < N) {
                float4 *p = reinterpret_cast<float4 *>(dst + 8 * g);
                p[0] = make_float4(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]),
                                   __uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
                p[1] = make_float4(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]),
                                   __uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
            }
        }
    } else {
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(c) + row * N + col0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (col0 + 8 * g < N) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
                v.y = pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
                v.z = pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
                v.w = pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
                *reinterpret_cast<uint4 *>(dst + 8 * g) = v;
            }
        }
    }
}

// The residual row[col0 .. col0+31] (pieces past N read as zero).
__device__ __forceinline__ void load_res32(const void *res, int64_t row, int col0, int N,
                                           uint4 (&v)[4])
{
    const uint4 *src =
        reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(res) + row * N + col0);
#pragma unroll
    for (int g = 0; g < 4; ++g)
        v[g] = (col0 + 8 * g < N) ? __ldcs(src + g) : make_uint4(0u, 0u, 0u, 0u);
}

// out[row, col0 .. col0+31] = round(res + round(acc)) in bf16, res loaded
// beforehand (it may be c itself).
__device__ __forceinline__ void store_row32_res(const uint32_t (&r)[32], void *c,
                                                const uint4 (&rv)[4], int64_t row, int col0, int N)
{
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(c) + row * N + col0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        if (col0 + 8 * g < N) {
            const uint32_t ru[4] = {rv[g].x, rv[g].y, rv[g].z, rv[g].w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                // round the product to bf16 first, as a separate matmul would
                const uint32_t p = pack_bf16x2(__uint_as_float(r[8 * g + 2 * j]),
                                               __uint_as_float(r[8 * g + 2 * j + 1]));
                const float lo = __fadd_rn(__uint_as_float(ru[j] << 16), __uint_as_float(p << 16));
                const float hi = __fadd_rn(__uint_as_float(ru[j] & 0xFFFF0000u),
                                           __uint_as_float(p & 0xFFFF0000u));
                o[j] = pack_bf16x2(lo, hi);
            }
            *reinterpret_cast<uint4 *>(dst + 8 * g) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// QKV form of the epilogue, for one accumulator row (one token): the tile's
// 256 columns are 256 / d whole heads of the (Hq + 2 Hkv) d columns.  Each
// value is first rounded to bf16 exactly as the product's output would be
// (after the norm scale), then q and k heads are rotated with the table's
// angles for the token's position using rope_kv_kernel's fp32 operations,
// so that the result is the plain product followed by bi_rope_kv_write bit
// for bit.  q goes to q_out, k and v to the token's cache slot (page blocks
// in core-matrix order).  The tensor-memory loads are warp-wide; only the
// stores depend on the row.
__device__ __noinline__ void qkv_epilogue(const GemmEpi &epi, uint32_t tbase, int nb, int64_t row,
                                          bool row_ok, float rscale, int N, unsigned *status)
{
    const int d = epi.head_dim, half = d / 2, pieces = d / 8;
    int32_t p = 0;
    int64_t slot = -1;
    if (row_ok) {
        p = __ldg(epi.pos + row);
        slot = __ldg(epi.slots + row);
        if (p < 0 || p >= epi.max_pos) record_status(status, BI_DEV_BAD_INDEX);
        if (slot >= epi.num_pages * kPage) {
            record_status(status, BI_DEV_BAD_INDEX);
            slot = -1;
        }
    }
    const bool ok = row_ok && p >= 0 && p < epi.max_pos;  // else the row writes nothing
    const int64_t page = slot >= 0 ? slot / kPage : 0;
    const int off = slot >= 0 ? int(slot % kPage) : 0;
    const int64_t blk_row = (off >> 3) * (8 * pieces) + (off & 7);
#pragma unroll 1
    for (int hh = 0; hh < 256 / d; ++hh) {
        const int n0 = nb * 256 + hh * d;
        if (n0 >= N) break;  // the same for the whole warp
        const int gh = n0 / d;  // q heads, then k heads, then v heads
        const bool rotated = gh < epi.Hq + epi.Hkv;
#pragma unroll 1
        for (int a = 0; a < half / 32; ++a) {
            uint32_t lo[32], hi[32];
            tmem_ld32(tbase + uint32_t(hh * d + 32 * a), lo);
            tmem_ld32(tbase + uint32_t(hh * d + half + 32 * a), hi);
            tmem_wait_ld(lo);
            tmem_wait_ld(hi);
            uint32_t plo[16], phi[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                plo[j] = pack_bf16x2(__fmul_rn(__uint_as_float(lo[2 * j]), rscale),
                                     __fmul_rn(__uint_as_float(lo[2 * j + 1]), rscale));
                phi[j] = pack_bf16x2(__fmul_rn(__uint_as_float(hi[2 * j]), rscale),
                                     __fmul_rn(__uint_as_float(hi[2 * j + 1]), rscale));
            }
            if (!ok) continue;
            if (rotated) {
                const float4 *cs =
                    reinterpret_cast<const float4 *>(epi.rope + (int64_t(p) * half + 32 * a) * 2);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 c = __ldg(cs + j);  // cos, sin of values 2j and 2j + 1
                    const float a0 = __uint_as_float(plo[j] << 16);
                    const float a1 = __uint_as_float(plo[j] & 0xFFFF0000u);
                    const float b0 = __uint_as_float(phi[j] << 16);
                    const float b1 = __uint_as_float(phi[j] & 0xFFFF0000u);
                    plo[j] = pack_bf16x2(__fsub_rn(__fmul_rn(a0, c.x), __fmul_rn(b0, c.y)),
                                         __fsub_rn(__fmul_rn(a1, c.z), __fmul_rn(b1, c.w)));
                    phi[j] = pack_bf16x2(__fadd_rn(__fmul_rn(b0, c.x), __fmul_rn(a0, c.y)),
                                         __fadd_rn(__fmul_rn(b1, c.z), __fmul_rn(a1, c.w)));
                }
            }
            if (gh < epi.Hq) {
                uint4 *qo = static_cast<uint4 *>(epi.q_out) + (row * epi.Hq + gh) * pieces;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    qo[4 * a + u] = make_uint4(plo[4 * u], plo[4 * u + 1], plo[4 * u + 2], plo[4 * u + 3]);
                    qo[half / 8 + 4 * a + u] =
                        make_uint4(phi[4 * u], phi[4 * u + 1], phi[4 * u + 2], phi[4 * u + 3]);
                }
            } else if (slot >= 0) {
                const int g = rotated ? gh - epi.Hq : gh - epi.Hq - epi.Hkv;
                uint4 *blk = static_cast<uint4 *>(rotated ? epi.k_cache : epi.v_cache) +
                             (page * epi.Hkv + g) * (kPage * pieces) + blk_row;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    blk[(4 * a + u) * 8] =
                        make_uint4(plo[4 * u], plo[4 * u + 1], plo[4 * u + 2], plo[4 * u + 3]);
                    blk[(half / 8 + 4 * a + u) * 8] =
                        make_uint4(phi[4 * u], phi[4 * u + 1], phi[4 * u + 2], phi[4 * u + 3]);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ 2-SM kernel
//
// One 256 x 256 output tile per pair of SMs (a cluster of two CTAs): CTA r
// of the pair owns rows 128r..128r+127 of the tile in its TMEM and holds,
// per 64-wide K slice, its own 128 rows of A and W rows 128r..128r+127 of
// the tile's 256 columns; the leader (r = 0) issues tcgen05.mma.cta_group::2
// with M = 256, N = 256, which reads both CTAs' shared memory.  A CTA reads
// 32 KB per K slice instead of 48, so seven stages fit.
namespace pair {

constexpr int BM = 256, BN = 256, BK = kGemmBK, STAGES = 7;
constexpr int A_BYTES = kGemmCtaRows * BK * 2;  // 16 KB: this CTA's half of the A slice
constexpr int W_BYTES = kGemmCtaRows * BK * 2;  // 16 KB: this CTA's half of the W slice
constexpr int STAGE_BYTES = A_BYTES + W_BYTES;
static_assert(2 * kGemmCtaRows == BM && 2 * kGemmCtaRows == BN, "a pair's two CTAs cover the tile");
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;     // two 128-lane x 256-column fp32 accumulators
constexpr int BAR_BYTES = 256;
constexpr int CUM_BYTES = (kMaxGemmGroups + 1) * 4;  // grouped mode: tiles before each group
static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barriers, TMEM address and abort flag");
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + CUM_BYTES;
// shared addresses fit the 14-bit field (16-byte units) of a matrix descriptor
static_assert(SMEM_BYTES + 4096 <= (1 << 18), "descriptor address field");

// The tile of work unit u.  Plain: tiles m-fastest over an M x N output
// (split-K units only in the variant-off build).  Grouped: the rows of group
// g are offsets[g] .. offsets[g+1]-1 of A and C and its weight is rows
// g*N .. g*N+N-1 of W; its tiles (m-fastest) follow those of group g-1.
__device__ __forceinline__ Unit unit_at(int u, int num_m, int num_n, int k_splits, int kblocks,
                                        int kb_per, int M, int N, const int64_t *goff,
                                        const int *cum, int groups)
{
    if (!goff) {
        Unit t = unit_of(u, num_m, k_splits, kblocks, kb_per);
        t.row0 = int64_t(t.mb) * BM;
        t.row_end = M;
        t.w_row0 = int64_t(t.nb) * BN;
        return t;
    }
    int g = 0;
    while (g + 1 < groups && cum[g + 1] <= u) ++g;
    const int64_t r0 = goff[g], r1 = goff[g + 1];
    const int mt = int((r1 - r0 + BM - 1) / BM);
    const int local = u - cum[g];
    Unit t;
    t.split = 0;
    t.kb0 = 0;
    t.kb1 = kblocks;
    t.mb = local % mt;
    t.nb = local / mt;
    t.row0 = r0 + int64_t(t.mb) * BM;
    t.row_end = r1;
    t.w_row0 = int64_t(g) * N + int64_t(t.nb) * BN;
    (void)num_m;
    (void)num_n;
    return t;
}

template <bool FUSED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmw,
                     void *c, float *__restrict__ ws, int M, int N, int K, int out_f32,
                     int k_splits, const int64_t *__restrict__ goff, int groups, GemmEpi epi,
                     unsigned *status, uint64_t timeout_ns)
{
#if BI_INVARIANT
    k_splits = 1;  // the invariant build never splits K
#endif
    // fused forms: plain tiles only (no groups, no split K)
    const float *row_scale = FUSED ? epi.rs : nullptr;
    const void *res = FUSED ? epi.residual : nullptr;
    if (FUSED) {
        k_splits = 1;
        goff = nullptr;
    }
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
    uint8_t *sA = smem;
    uint8_t *sW = smem + STAGES * A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);  // leader's used
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;   // leader's used: 8 arrivals (4 epilogue warps x 2 CTAs)
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *cum = reinterpret_cast<int *>(smem + STAGES * STAGE_BYTES + BAR_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int num_n = (N + BN - 1) / BN;
    if (goff && threadIdx.x == 64) {
        // tiles before each group (read once: the offsets come from the device)
        int acc = 0;
        for (int g = 0; g < groups; ++g) {
            cum[g] = acc;
            const int64_t n = goff[g + 1] - goff[g];
            acc += int((n > 0 ? (n + BM - 1) / BM : 0) * num_n);
        }
        cum[groups] = acc;
    }

    if (threadIdx.x == 0) {
        // the producer's first loads will need both descriptors
        tma_prefetch_desc(&tma);
        tma_prefetch_desc(&tmw);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 8);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers and TMEM of both CTAs exist before either uses them
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtl ctl{abort_flag, status, timeout_ns};

    const int num_m = (M + BM - 1) / BM;
    const int kblocks = (K + BK - 1) / BK;
    const int kb_per = (kblocks + k_splits - 1) / k_splits;
    const int units = goff ? cum[groups] : num_m * num_n * k_splits;
    auto unit = [&](int u) {
        return unit_at(u, num_m, num_n, k_splits, kblocks, kb_per, M, N, goff, cum, groups);
    };
    const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = pair_id; ok && u < units; u += num_pairs) {
                const Unit t = unit(u);
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    if (!wait_spin(&empty[stage], phase ^ 1u, ctl)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = map_to_cta(smem_u32(&full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
                    tma_load_2d_pair(sA + stage * A_BYTES, &tma, bar, kb * BK,
                                     int(t.row0) + int(rank) * kGemmCtaRows);
                    tma_load_2d_pair(sW + stage * W_BYTES, &tmw, bar, kb * BK,
                                     int(t.w_row0) + int(rank) * kGemmCtaRows);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issue (leader)
            const uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
            const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA), 16, 1024);
            const uint64_t w_desc0 = sdesc_sw128(smem_u32(sW), 16, 1024);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int u = pair_id; ok && u < units; u += num_pairs) {
                const Unit t = unit(u);
                if (!wait_spin(&tempty[acc], acc_phase ^ 1u, ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + uint32_t(acc * BN);
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    if (!wait_spin(&full[stage], phase, ctl)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // the descriptors of stage 0 plus the stage's and the K
                    // step's offsets, in the 16-byte units of the address
                    // field (every address stays below 2^18 bytes, so the
                    // sums never carry out of the field)
                    const uint64_t ad = a_desc0 + uint64_t(stage * (A_BYTES >> 4));
                    const uint64_t wd = w_desc0 + uint64_t(stage * (W_BYTES >> 4));
                    mma_ss_pair(d, ad, wd, idesc, kb > t.kb0 ? 1u : 0u);
#pragma unroll
                    for (int k = 1; k < BK / 16; ++k)
                        mma_ss_pair(d, ad + 2 * k, wd + 2 * k, idesc, 1u);
                    mma_commit_pair(&empty[stage], 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(&tfull[acc], 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                mma_commit_pair(drain, 0x1);
                wait_drain(drain, 0, timeout_ns);
            }
        }
    } else if (warp < 6) {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;
        const uint32_t tempty_leader0 = map_to_cta(smem_u32(&tempty[0]), 0);
        const uint32_t tempty_leader1 = map_to_cta(smem_u32(&tempty[1]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = pair_id; u < units; u += num_pairs) {
            const Unit t = unit(u);
            const int64_t row = t.row0 + int(rank) * 128 + 32 * q + lane;
            const bool row_ok = row >= 0 && row < M && row < t.row_end;
            // residual form: this row's 256 residual values are fetched while
            // the MMAs still run (into L2, and the first 32 into registers),
            // so that the stores below do not wait on memory in turn
            uint4 rcur[4];
            if (FUSED && res && row_ok) {
                const __nv_bfloat16 *rp = static_cast<const __nv_bfloat16 *>(res) + row * N;
#pragma unroll
                for (int l = 0; l < BN / 64; ++l) {
                    const int col = t.nb * BN + 64 * l;
                    if (col < N) prefetch_l2(rp + col);
                }
                load_res32(res, row, t.nb * BN, N, rcur);
            }
            if (!wait(&tfull[acc], acc_phase, ctl)) break;
            tc_fence_after();
            // norm form: this row's rsqrt (computed before the launch)
            const float rscale = (row_scale && row_ok) ? __ldg(row_scale + row) : 1.0f;
            if (FUSED && epi.rope) {
                qkv_epilogue(epi, tmem_addr(tmem, 32 * q, acc * BN), t.nb, row, row_ok, rscale, N,
                             status);
            } else {
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint4 rnext[4];
                if (FUSED && res && row_ok && cc + 1 < BN / 32)
                    load_res32(res, row, t.nb * BN + (cc + 1) * 32, N, rnext);
                uint32_t r[32];
                tmem_ld32(tmem_addr(tmem, 32 * q, acc * BN + cc * 32), r);
                tmem_wait_ld(r);
                if (row_scale) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        r[j] = __float_as_uint(__fmul_rn(__uint_as_float(r[j]), rscale));
                }
                const int col0 = t.nb * BN + cc * 32;
                if (row_ok && col0 < N) {
                    if (FUSED && res)
                        store_row32_res(r, c, rcur, row, col0, N);
                    else
                        store_row32(r, c, ws, row, col0, N, M, t.split, k_splits, out_f32);
                }
                if (FUSED && res) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) rcur[g] = rnext[g];
                }
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its peer may still touch its memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

}  // namespace pair

// Variant-off only: C = sum over splits of the fp32 partials, in split order.
__global__ void splitk_reduce_kernel(const float *__restrict__ ws, void *__restrict__ c,
                                     int64_t MN, int k_splits, int out_f32)
{
    const int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (i >= MN) return;
    float4 acc = *reinterpret_cast<const float4 *>(ws + i);
    for (int s = 1; s < k_splits; ++s) {
        const float4 v = *reinterpret_cast<const float4 *>(ws + int64_t(s) * MN + i);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
    }
    if (out_f32) {
        *reinterpret_cast<float4 *>(static_cast<float *>(c) + i) = acc;
    } else {
        uint2 v;
        v.x = pack_bf16x2(acc.x, acc.y);
        v.y = pack_bf16x2(acc.z, acc.w);
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(c) + i) = v;
    }
}

}  // namespace

size_t gemm_smem_bytes() { return pair::SMEM_BYTES; }

int gemm_k_splits(int64_t M, int64_t N, int64_t K, int num_sms)
{
#if BI_INVARIANT
    (void)M, (void)N, (void)K, (void)num_sms;
    return 1;
#else
    // Variant-off: split K when the tiles cannot fill the GPU, with the
    // count that minimises a simple time model: the K slices the busiest
    // pair walks (waves x slices per split, ~0.6 us a slice, measured on a
    // B200 at M = 256) plus one pass of the fp32 partial sums out to memory
    // and back (~6.5 TB/s) and the reduction's launch (~3 us); taken only
    // when the model saves a fifth or more.
    const int64_t tiles = ((M + pair::BM - 1) / pair::BM) * ((N + pair::BN - 1) / pair::BN);
    const int64_t kblocks = (K + pair::BK - 1) / pair::BK;
    const int64_t pairs = num_sms / 2;
    if (tiles >= pairs || kblocks < 8 || pairs < 1) return 1;
    const double slice_us = 0.6, bytes_per_us = 6.5e6, reduce_us = 3.0;
    const double whole_us = double(kblocks) * slice_us;  // one wave of whole-K tiles
    int64_t best = 1;
    double best_us = 0.8 * whole_us;
    for (int64_t ks = 2; ks <= 16 && ks <= kblocks / 4; ++ks) {
        const int64_t per = (kblocks + ks - 1) / ks;
        const int64_t splits = (kblocks + per - 1) / per;
        const int64_t waves = (tiles * splits + pairs - 1) / pairs;
        const double us = double(waves * per) * slice_us +
                          2.0 * double(splits) * double(M) * double(N) * 4.0 / bytes_per_us +
                          reduce_us;
        if (us < best_us) {
            best = splits;
            best_us = us;
        }
    }
    return static_cast<int>(best);
#endif
}

// Pairs of SMs that can be resident at once on this device (not every SM can
// pair up); the persistent grid is this many clusters.
static cudaError_t resident_pairs(int num_sms, int *out)
{
    cudaError_t e = cudaFuncSetAttribute(pair::gemm_pair_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         pair::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(pair::gemm_pair_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, pair::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // as many pairs as can be resident at once (not every SM can pair up)
    static int max_pairs[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (max_pairs[dev] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
        cfg.blockDim = dim3(pair::THREADS, 1, 1);
        cfg.dynamicSmemBytes = pair::SMEM_BYTES;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        e = cudaOccupancyMaxActiveClusters(&clusters, pair::gemm_pair_kernel<false>, &cfg);
        if (e != cudaSuccess) return e;
        max_pairs[dev] = clusters > 0 ? clusters : 1;
    }
    *out = max_pairs[dev];
    return cudaSuccess;
}

cudaError_t launch_gemm_grouped(const CUtensorMap &ta, const CUtensorMap &tw, void *c, int rows,
                                int N, int K, bool out_f32, const int64_t *offsets, int groups,
                                int num_sms, unsigned *status, uint64_t timeout_ns,
                                cudaStream_t s)
{
    int pairs = 0;
    cudaError_t e = resident_pairs(num_sms, &pairs);
    if (e != cudaSuccess) return e;
    // the tile count is only known on the device: every resident pair runs
    pair::gemm_pair_kernel<false><<<2 * pairs, pair::THREADS, pair::SMEM_BYTES, s>>>(
        ta, tw, c, nullptr, rows, N, K, out_f32 ? 1 : 0, 1, offsets, groups, GemmEpi{}, status,
        timeout_ns);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tw, void *c, int M, int N,
                        int K, bool out_f32, float *ws, int k_splits, int num_sms,
                        unsigned *status, uint64_t timeout_ns, cudaStream_t s)
{
    int max_pairs = 0;
    cudaError_t e = resident_pairs(num_sms, &max_pairs);
    if (e != cudaSuccess) return e;
    const int64_t units = int64_t((M + pair::BM - 1) / pair::BM) * ((N + pair::BN - 1) / pair::BN) *
                          k_splits;
    const int pairs = static_cast<int>(units < max_pairs ? units : max_pairs);
    pair::gemm_pair_kernel<false><<<2 * pairs, pair::THREADS, pair::SMEM_BYTES, s>>>(
        ta, tw, c, ws, M, N, K, out_f32 ? 1 : 0, k_splits, nullptr, 0, GemmEpi{}, status,
        timeout_ns);
    e = cudaGetLastError();
    if (e != cudaSuccess || k_splits <= 1) return e;
    const int64_t MN = int64_t(M) * N;
    const int64_t thr = (MN / 4 + 255) / 256;
    splitk_reduce_kernel<<<static_cast<unsigned>(thr), 256, 0, s>>>(ws, c, MN, k_splits,
                                                                    out_f32 ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_gemm_fused(const CUtensorMap &ta, const CUtensorMap &tw, void *c, int M, int N,
                              int K, bool out_f32, const GemmEpi &epi, int num_sms,
                              unsigned *status, uint64_t timeout_ns, cudaStream_t s)
{
    int max_pairs = 0;
    cudaError_t e = resident_pairs(num_sms, &max_pairs);
    if (e != cudaSuccess) return e;
    const int64_t units = int64_t((M + pair::BM - 1) / pair::BM) * ((N + pair::BN - 1) / pair::BN);
    const int pairs = static_cast<int>(units < max_pairs ? units : max_pairs);
    pair::gemm_pair_kernel<true><<<2 * pairs, pair::THREADS, pair::SMEM_BYTES, s>>>(
        ta, tw, c, nullptr, M, N, K, out_f32 ? 1 : 0, 1, nullptr, 0, epi, status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace bi
