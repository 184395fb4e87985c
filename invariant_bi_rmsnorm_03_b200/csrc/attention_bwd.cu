// attention_bwd.cu -- backward of the paged causal attention, for the trainer
// side of on-policy RL (xitu-tech news, "强化学习的突破": the trainer must
// reproduce the sampler's numbers, so its passes run on fixed, deterministic
// reduction orders).
//
// For a query row i (absolute position t_i, visible keys j <= t_i) with the
// forward's log-sum-exp lse_i and output o_i, and an upstream gradient dO_i:
//   P_ij  = exp(scale q_i . k_j - lse_i)                 (the forward's weights)
//   dP_ij = dO_i . v_j,   Delta_i = dO_i . o_i           (= sum_j P_ij dP_ij)
//   dS_ij = P_ij (dP_ij - Delta_i)
//   dq_i  = scale sum_j dS_ij k_j
//   dk_j  = scale sum_i dS_ij q_i,   dv_j = sum_i P_ij dO_i
// where the sums for dk_j and dv_j run over every query row of the sequence's
// chunk that sees key j, in all query heads of k_j's group.
//
// Three kernels, no atomics:
//   attn_bwd_prep_kernel   Delta_i (fp32, a fixed order) and lse_i log2(e).
//   attn_bwd_dkv_kernel    one block per (sequence, kv head, 128-key block):
//                          for each query head of the group (ascending) and
//                          each 128-row query tile (ascending):
//                            S^T = K Q^T,  dP^T = V dO^T        (tcgen05)
//                            P^T, dS^T elementwise (a key row per TMEM lane)
//                            dV += P^T dO,  dK += dS^T Q         (P^T, dS^T
//                                                                 from TMEM)
//                          so a key's dk and dv are sums in one fixed order
//                          over its own sequence's rows.
//   attn_bwd_dq_kernel     one block per (sequence, query head, 128-row tile):
//                          for each 128-key block ascending:
//                            S = Q K^T,  dP = dO V^T;  P, dS elementwise (a
//                            query row per TMEM lane);  dQ += dS K.
//                          A row's dq depends on that row alone.
// P and dS are rounded to bf16 to enter the tensor core (as the forward
// rounds P before P V); every other quantity is fp32.
//
// Shared-memory operands: a 128-row tile of q or dO is loaded by TMA as
// 64-value boxes of 128 rows with the 128-byte swizzle, which serves both as
// a K-major operand (for S^T, dP^T, S, dP) and as an MN-major one (for dV,
// dK); a 128-key block of the cache is its eight page blocks, already in the
// no-swizzle core-matrix order, copied whole (the dK/dV kernel's, once, by
// the threads; the dQ kernel's, per step, by one bulk copy per page block).
// The next step's tiles or block land in a second buffer while the current
// step computes.  Rows a masked product could meet as 0 x NaN are zeroed in
// shared memory first: q/dO rows past the chunk in the dK/dV kernel (they
// enter dV and dK through a zero P or dS) and keys past the sequence in the
// dQ kernel (they enter dQ through a zero dS).
//
// Block of 256 threads (8 warps; warps w and w + 4 share TMEM lanes
// 32(w%4) .. +31, each taking half of the columns).  Thread 0 issues the
// MMAs; every wait is bounded and its outcome is agreed on by the whole
// block (__syncthreads_and), so that a timeout ends every thread's loop at
// the same point.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"
#include "bi_ptx.cuh"

namespace bi {
namespace {

constexpr int kBwdThreads = 256;  // 8 warps: two per TMEM lane quarter
constexpr int kKeyBlock = 128;  // keys per block of the dk/dv kernel and per step of dq
constexpr int kQTile = 128;     // query rows per tile
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
    static constexpr int TILE_BYTES = kQTile * D * 2;          // q or dO tile
    static constexpr int BOX_BYTES = kQTile * 64 * 2;          // 64 values of 128 rows
    static constexpr int PAGE_BYTES = kPage * D * 2;           // one page block
    static constexpr int KGROUP_BYTES = PAGE_BYTES / 2;        // 8-key groups
    static constexpr int BLOCK_BYTES = (kKeyBlock / kPage) * PAGE_BYTES;  // 128 keys
    static constexpr int VEC_BYTES = 2 * kQTile * 4;           // lse2, Delta of 128 rows
    static constexpr int SLACK = 1024;
    // two buffers of what streams (q and dO tiles in the dk/dv kernel, key
    // blocks in the dq kernel), one of what stays
    static constexpr int SMEM = SLACK + 4 * TILE_BYTES + 2 * BLOCK_BYTES + 2 * VEC_BYTES + 64;
    // shared addresses fit the 14-bit field (16-byte units) of a matrix
    // descriptor, so descriptors are formed by adding offsets to one
    static_assert(SMEM + 4096 <= (1 << 18), "descriptor address field");
    static_assert(4 * TILE_BYTES + 2 * BLOCK_BYTES == 2 * TILE_BYTES + 4 * BLOCK_BYTES,
                  "both kernels fit the same shared-memory size");
    // TMEM columns: S (128), dP (128), two d-wide accumulators (dV, dK) or one (dQ)
    static constexpr uint32_t S_COL = 0, DP_COL = 128, ACC0 = 256, ACC1 = 256 + D;
    static constexpr uint32_t TMEM_COLS = 512;
};

// The two warps of a TMEM lane quarter each turn half of the 128 fp32
// columns of S (or dP) into bf16 pairs and store them back in place.  Chunk c
// (columns 32c .. 32c+31) packs into 16 columns inside its own half
// [64 (c/2), 64 (c/2) + 64), which only that half's warp reads, and only
// after it has read them: one warp never overwrites a column the other has
// still to read.  packed_step_col(j) is where values 16 j .. 16 j + 15 (the
// K step j of the product that reads them) start.
static_assert(kQTile == 128 && kKeyBlock == 128, "four 32-column chunks, two per half");
__device__ __forceinline__ uint32_t packed_chunk_col(int c) { return 64u * (c >> 1) + 16u * (c & 1); }
__device__ __forceinline__ uint32_t packed_step_col(int j) { return 64u * (j >> 2) + 8u * (j & 3); }

// Byte offset, inside a page block of head dim D, of values 8c .. 8c+7 of key r.
template <int D>
__device__ __forceinline__ uint32_t page_off(int r, int c)
{
    return uint32_t(r >> 3) * (D * 16) + uint32_t(c) * 128u + uint32_t(r & 7) * 16u;
}

__device__ __forceinline__ uint32_t pack2(float a, float b)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&p);
}

// Keys k0 .. k0+127 of kv head g of one sequence (its page-table row `bt`)
// into eight page blocks, asynchronously; keys at or past kv_len are zero.
template <int D>
__device__ __forceinline__ void copy_keys(uint8_t *dst, const uint8_t *cache, const int32_t *bt,
                                          int k0, int kv_len, int Hkv, int g, int num_pages,
                                          unsigned *status)
{
    using C = BwdCfg<D>;
    constexpr int PP = C::PAGE_BYTES / 16;  // 16-byte pieces of a page block
    constexpr int ITER = (kKeyBlock / kPage) * PP / kBwdThreads;
#pragma unroll
    for (int i = 0; i < ITER; ++i) {
        const int e = threadIdx.x + i * kBwdThreads;
        const int pg = e / PP, piece = e - pg * PP;
        const uint32_t off = uint32_t(piece) * 16u;
        // piece -> key: off = kg * 16D + c * 128 + r * 16
        const int kg = int(off / (D * 16)), r = int(off % 128) / 16;
        const int key = k0 + pg * kPage + kg * 8 + r;
        const uint8_t *src = cache;
        bool ok = false;
        if (key < kv_len) {
            const int phys = __ldg(bt + (k0 / kPage + pg));
            if (phys >= 0 && phys < num_pages) {
                src = cache + (int64_t(phys) * Hkv + g) * int64_t(C::PAGE_BYTES) + off;
                ok = true;
            } else if (piece == 0) {
                record_status(status, BI_DEV_BAD_INDEX);
            }
        }
        cp_async16(dst + pg * C::PAGE_BYTES + off, src, ok);
    }
}

// Waits for phase `parity` of `bar` on every thread; the block agrees on the
// outcome (true only if every thread saw the phase complete).  The whole
// block waits on each step's products, so the wait polls before it sleeps.
__device__ __forceinline__ bool block_wait(uint64_t *bar, uint32_t parity, const WaitCtl &ctl)
{
    const bool ok = wait_spin(bar, parity, ctl);
    return __syncthreads_and(ok ? 1 : 0) != 0;
}

__device__ bool drain_wait(uint64_t *bar, uint32_t parity, uint64_t timeout_ns)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs))
        if (global_ns() - t0 > timeout_ns) return false;
    return true;
}

// ---------------------------------------------------------------- prep
// delta[r] = sum_v dO[r, v] o[r, v] (fp32: lane-strided fused multiply-adds
// in value order, then a xor butterfly); lse2[r] = lse[r] log2(e).  One warp
// per (token, head) row.
__global__ void attn_bwd_prep_kernel(const uint16_t *__restrict__ o, const uint16_t *__restrict__ dout,
                                     const float *__restrict__ lse, int64_t rows, int d,
                                     float *__restrict__ lse2, float *__restrict__ delta)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        float acc = 0.0f;
        for (int v = lane; v < d; v += 32) {
            const float a = __uint_as_float(uint32_t(o[r * d + v]) << 16);
            const float b = __uint_as_float(uint32_t(dout[r * d + v]) << 16);
            acc = __fmaf_rn(a, b, acc);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
        if (lane == 0) {
            delta[r] = acc;
            lse2[r] = __fmul_rn(lse[r], kLog2e);
        }
    }
}

// ---------------------------------------------------------------- dK, dV

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tq,
                                                              const __grid_constant__ CUtensorMap tdo,
                                                              const AttnBwdParams p)
{
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
    // q tiles [2], dO tiles [2] (the step's and the next step's), K, V
    auto sQ = [&](int buf) { return smem + buf * C::TILE_BYTES; };
    auto sDO = [&](int buf) { return smem + (2 + buf) * C::TILE_BYTES; };
    uint8_t *sK = smem + 4 * C::TILE_BYTES;
    uint8_t *sV = sK + C::BLOCK_BYTES;
    float *sLse = reinterpret_cast<float *>(sV + C::BLOCK_BYTES);  // [2][128]
    float *sDelta = sLse + 2 * kQTile;                             // [2][128]
    uint64_t *bar = reinterpret_cast<uint64_t *>(sDelta + 2 * kQTile);
    uint64_t *drain = bar + 1;
    uint64_t *tbar = drain + 1;  // [2] the q and dO tiles of buffer b landed (TMA)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tbar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    // block -> (sequence, kv head, key block)
    // (key blocks slowest, ascending: the blocks with the most query tiles
    // start first -- a longest-first schedule of the waves)
    const int bh = blockIdx.x % (p.B * p.Hkv);
    const int kb = blockIdx.x / (p.B * p.Hkv);
    const int g = bh % p.Hkv;
    const int b = bh / p.Hkv;
    const int q0 = p.cu_q[b], n = p.cu_q[b + 1] - q0, ctx = p.ctx_lens[b];
    const int kv_len = ctx + n;
    const int k0 = kb * kKeyBlock;
    if (n <= 0 || k0 >= kv_len) return;
    if (kv_len > p.max_pages * kPage) {  // the page table cannot hold the sequence
        if (threadIdx.x == 0) record_status(p.status, BI_DEV_BAD_INDEX);
        return;
    }

    // Steps j = hh * ntiles + qt: query head hh of the group (ascending),
    // then the chunk's 128-row tile qt (ascending); a tile whose last row
    // comes before this key block sees none of it and is skipped.
    const int ntiles = (n + kQTile - 1) / kQTile;
    const int nsteps = p.group * ntiles;
    auto sees = [&](int j) {
        const int qt = j % ntiles;
        return ctx + min(n, (qt + 1) * kQTile) - 1 >= k0;
    };
    auto next_step = [&](int j) {
        while (j < nsteps && !sees(j)) ++j;
        return j;
    };
    // the step's q and dO tiles (TMA, thread 0: 64-value boxes of 128 rows,
    // 128-byte swizzle, rows past the tensor zero) and this thread's row of
    // its lse2 / Delta
    uint32_t tphase = 0, tpending = 0;  // per buffer: parity to wait for, copy in flight
    auto fetch = [&](int j, int buf, float &lse_r, float &delta_r) {
        const int h = g * p.group + j / ntiles, qt = j % ntiles;
        const int rows = min(kQTile, n - qt * kQTile);
        const int64_t row0 = int64_t(q0) + int64_t(qt) * kQTile;
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(&tbar[buf], 2u * C::TILE_BYTES);
#pragma unroll
            for (int x = 0; x < D / 64; ++x) {
                tma_load_3d(sQ(buf) + x * C::BOX_BYTES, &tq, &tbar[buf], 64 * x, h, int(row0));
                tma_load_3d(sDO(buf) + x * C::BOX_BYTES, &tdo, &tbar[buf], 64 * x, h, int(row0));
            }
        }
        tpending |= 1u << buf;
        const int r = threadIdx.x;  // threads 0..127: one row each
        lse_r = r < rows ? p.lse2[(row0 + r) * p.Hq + h] : 0.0f;
        delta_r = r < rows ? p.delta[(row0 + r) * p.Hq + h] : 0.0f;
    };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        mbar_init(drain, 1);
        mbar_init(&tbar[0], 1);
        mbar_init(&tbar[1], 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    const int32_t *bt = p.block_table + int64_t(b) * p.max_pages;
    copy_keys<D>(sK, static_cast<const uint8_t *>(p.k_cache), bt, k0, kv_len, p.Hkv, g,
                 p.num_pages, p.status);
    copy_keys<D>(sV, static_cast<const uint8_t *>(p.v_cache), bt, k0, kv_len, p.Hkv, g,
                 p.num_pages, p.status);
    cp_async_commit();
    int j = next_step(0);  // (the sequence's last row sees every key block of it)
    float lse_r = 0.0f, delta_r = 0.0f;
    fetch(j, 0, lse_r, delta_r);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
    // warps w and w + 4 share TMEM lane quarter w % 4, each taking half of
    // the columns
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t lane_base = tmem_addr(tmem, 32 * quarter, 0);
    const int key = k0 + 32 * quarter + lane;  // this thread's key (TMEM lane)
    const float cs = p.scale_log2;

    const uint32_t idesc_s = idesc_bf16_f32(128, kQTile, 0, 0);
    const uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);
    const uint32_t kb_addr = smem_u32(sK), vb_addr = smem_u32(sV);
    const uint64_t kd0 = sdesc_plain(kb_addr, 128, C::KGROUP_BYTES);  // K, V: K-major
    const uint64_t vd0 = sdesc_plain(vb_addr, 128, C::KGROUP_BYTES);
    uint32_t phase = 0;
    bool ok = true, first = true;
    int buf = 0;
    while (ok && j < nsteps) {
        const int qt = j % ntiles;
        const int rows = min(kQTile, n - qt * kQTile);
        const int pos0 = ctx + qt * kQTile;
        const uint32_t q_addr = smem_u32(sQ(buf)), do_addr = smem_u32(sDO(buf));
        float *lse_s = sLse + buf * kQTile, *delta_s = sDelta + buf * kQTile;
        if (threadIdx.x < kQTile) {
            lse_s[threadIdx.x] = lse_r;
            delta_s[threadIdx.x] = delta_r;
        }
        cp_async_wait<0>();  // (first step) this thread's part of the key block landed
        ok = block_wait(&tbar[buf], (tphase >> buf) & 1u, ctl);  // this step's tiles
        if (!ok) break;
        tphase ^= 1u << buf;
        tpending &= ~(1u << buf);
        if (rows < kQTile) {
            // rows past the chunk (the next sequence's, or zeros past the
            // tensor) become zeros: 128 bytes a row in each box (the swizzle
            // moves 16-byte pieces only within their row)
            const int per = (kQTile - rows) * 8;  // 16-byte pieces per box
            for (int e = threadIdx.x; e < 2 * (D / 64) * per; e += kBwdThreads) {
                const int box = e / per, off = e - box * per;
                uint8_t *t = (box & 1 ? sDO(buf) : sQ(buf)) + (box >> 1) * C::BOX_BYTES;
                reinterpret_cast<uint4 *>(t + rows * 128)[off] = make_uint4(0, 0, 0, 0);
            }
        }
        fence_proxy_async_smem();  // the tiles (and the zeros) are read by the tensor core
        tc_fence_before();
        __syncthreads();
        // ------------------------------------------------ S^T, dP^T
        if (threadIdx.x == 0) {
            tc_fence_after();
            // descriptors by offset (16-byte units) from the step-0 ones
            const uint64_t qd = sdesc_sw128(q_addr, 16, 1024), dd = sdesc_sw128(do_addr, 16, 1024);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                // q and dO as K-major operands: 16 values = 32 bytes of a
                // swizzled 128-byte row, 64-value boxes BOX_BYTES apart
                const uint32_t koff = ((k >> 2) * C::BOX_BYTES + (k & 3) * 32) / 16;
                mma_ss(tmem + C::S_COL, kd0 + 16 * k, qd + koff, idesc_s, k > 0 ? 1u : 0u);
                mma_ss(tmem + C::DP_COL, vd0 + 16 * k, dd + koff, idesc_s, k > 0 ? 1u : 0u);
            }
            mma_commit(bar);
        }
        // the next step's tiles stream into the other buffer meanwhile (the
        // previous step's products, which read it, have completed)
        const int jn = next_step(j + 1);
        if (jn < nsteps) fetch(jn, buf ^ 1, lse_r, delta_r);
        ok = block_wait(bar, phase, ctl);
        phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
        // ------------------------------------------------ P^T, dS^T (row = key)
#pragma unroll 1
        for (int c = half * (kQTile / 64); c < (half + 1) * (kQTile / 64); ++c) {
            uint32_t sv[32], dp[32];
            tmem_ld32(lane_base + C::S_COL + 32 * c, sv);
            tmem_ld32(lane_base + C::DP_COL + 32 * c, dp);
            tmem_wait_ld(sv);
            tmem_wait_ld(dp);
            uint32_t pk[16], dk[16];
#pragma unroll
            for (int jj = 0; jj < 32; jj += 2) {
                float pv[2], dv[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int i = 32 * c + jj + u;  // query column
                    const bool vis = i < rows && key <= pos0 + i;
                    const float pr = ex2(__fmaf_rn(__uint_as_float(sv[jj + u]), cs, -lse_s[i]));
                    const float ds = __fmul_rn(pr, __fsub_rn(__uint_as_float(dp[jj + u]), delta_s[i]));
                    pv[u] = vis ? pr : 0.0f;
                    dv[u] = vis ? ds : 0.0f;
                }
                pk[jj / 2] = pack2(pv[0], pv[1]);
                dk[jj / 2] = pack2(dv[0], dv[1]);
            }
            tmem_st16(lane_base + C::S_COL + packed_chunk_col(c), pk);
            tmem_st16(lane_base + C::DP_COL + packed_chunk_col(c), dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        // ------------------------------------------------ dV += P^T dO, dK += dS^T Q
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint64_t dd = sdesc_sw128(do_addr, C::BOX_BYTES, 1024);
            const uint64_t qd = sdesc_sw128(q_addr, C::BOX_BYTES, 1024);
#pragma unroll
            for (int jj = 0; jj < kQTile / 16; ++jj) {
                const uint32_t acc = (first && jj == 0) ? 0u : 1u;
                // dO and q as MN-major operands (N = head dim): 16 rows =
                // 2048 bytes per K step, 8-row groups 1024 bytes apart,
                // 64-value boxes BOX_BYTES apart along N
                mma_ts(tmem + C::ACC0, tmem + C::S_COL + packed_step_col(jj), dd + 128 * jj, idesc_acc,
                       acc);
                mma_ts(tmem + C::ACC1, tmem + C::DP_COL + packed_step_col(jj), qd + 128 * jj, idesc_acc,
                       acc);
            }
            mma_commit(bar);
        }
        first = false;
        ok = block_wait(bar, phase, ctl);
        phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
        buf ^= 1;
        j = jn;
    }
    cp_async_wait<0>();  // no copy may still be landing when the block leaves
    if (!ok) {
        if (threadIdx.x == 0) {
            mma_commit(drain);
            drain_wait(drain, 0, p.timeout_ns);
            for (int bb = 0; bb < 2; ++bb)
                if (tpending & (1u << bb)) drain_wait(&tbar[bb], (tphase >> bb) & 1u, p.timeout_ns);
        }
    } else {
        // ---------------------------------------------------- write dV, dK
        // The keys of this block in pages the sequence owns (slots past its
        // length are zeros: their rows of P^T and dS^T were zero).
        const int n_pages = (kv_len + kPage - 1) / kPage;
        const int lp = key / kPage;
        const bool mine = lp < n_pages;
        int phys = -1;
        if (mine) phys = __ldg(bt + lp);
        const bool good = mine && phys >= 0 && phys < p.num_pages;
        const int r = key % kPage;
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            uint8_t *dst = static_cast<uint8_t *>(which ? p.dk : p.dv);
            const float mul = which ? p.scale : 1.0f;
            const uint32_t col = which ? C::ACC1 : C::ACC0;
#pragma unroll 1
            for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
                uint32_t a[32];
                tmem_ld32(lane_base + col + 32 * c, a);
                tmem_wait_ld(a);
                if (good) {
                    uint8_t *blk = dst + (int64_t(phys) * p.Hkv + g) * int64_t(C::PAGE_BYTES);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 v;
                        v.x = pack2(__fmul_rn(__uint_as_float(a[8 * q + 0]), mul),
                                    __fmul_rn(__uint_as_float(a[8 * q + 1]), mul));
                        v.y = pack2(__fmul_rn(__uint_as_float(a[8 * q + 2]), mul),
                                    __fmul_rn(__uint_as_float(a[8 * q + 3]), mul));
                        v.z = pack2(__fmul_rn(__uint_as_float(a[8 * q + 4]), mul),
                                    __fmul_rn(__uint_as_float(a[8 * q + 5]), mul));
                        v.w = pack2(__fmul_rn(__uint_as_float(a[8 * q + 6]), mul),
                                    __fmul_rn(__uint_as_float(a[8 * q + 7]), mul));
                        *reinterpret_cast<uint4 *>(blk + page_off<D>(r, 4 * c + q)) = v;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- dQ

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tq,
                                                             const __grid_constant__ CUtensorMap tdo,
                                                             const AttnBwdParams p)
{
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
    uint8_t *sQ = smem;
    uint8_t *sDO = sQ + C::TILE_BYTES;
    // K blocks [2], V blocks [2]: the step's and the next step's
    uint8_t *kv_base = sDO + C::TILE_BYTES;
    auto sK = [&](int buf) { return kv_base + buf * C::BLOCK_BYTES; };
    auto sV = [&](int buf) { return kv_base + (2 + buf) * C::BLOCK_BYTES; };
    uint64_t *bar = reinterpret_cast<uint64_t *>(kv_base + 4 * C::BLOCK_BYTES + 2 * C::VEC_BYTES);
    uint64_t *drain = bar + 1;
    uint64_t *kvbar = drain + 1;  // [2] the K and V pages of buffer b landed (bulk copies)
    uint64_t *qbar = kvbar + 2;   // the q and dO tiles landed (TMA)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(qbar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    // block -> (sequence, query head, query tile)
    // (tiles slowest, the last -- longest -- first: a longest-first
    // schedule of the waves)
    const int nqt = p.num_q_tiles;
    const int bh = blockIdx.x % (p.B * p.Hq);
    const int qt = nqt - 1 - blockIdx.x / (p.B * p.Hq);
    const int h = bh % p.Hq;
    const int b = bh / p.Hq;
    const int q0 = p.cu_q[b], n = p.cu_q[b + 1] - q0, ctx = p.ctx_lens[b];
    const int kv_len = ctx + n;
    if (qt * kQTile >= n) return;
    if (kv_len > p.max_pages * kPage) {
        if (threadIdx.x == 0) record_status(p.status, BI_DEV_BAD_INDEX);
        return;
    }
    const int rows = min(kQTile, n - qt * kQTile);
    const int pos0 = ctx + qt * kQTile;
    const int g = h / p.group;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        mbar_init(drain, 1);
        mbar_init(&kvbar[0], 1);
        mbar_init(&kvbar[1], 1);
        mbar_init(qbar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    const int64_t row0 = int64_t(q0) + qt * kQTile;
    const int32_t *bt = p.block_table + int64_t(b) * p.max_pages;
    // Page pg of key block kb: its physical page, or -1 when no key of it
    // is in the sequence or its id is out of range (then it is zeroed).
    auto page_of = [&](int kb, int pg) -> int {
        const int lp = kb * (kKeyBlock / kPage) + pg;
        if (lp * kPage >= kv_len) return -1;
        const int phys = __ldg(bt + lp);
        return (phys >= 0 && phys < p.num_pages) ? phys : -1;
    };
    // The block's K and V pages, one bulk copy per page block (thread 0).
    uint32_t kvphase = 0, kvpending = 0;
    auto fetch = [&](int kb, int buf) {
        if (threadIdx.x == 0) {
            uint32_t bytes = 0;
            for (int pg = 0; pg < kKeyBlock / kPage; ++pg)
                if (page_of(kb, pg) >= 0) bytes += 2u * C::PAGE_BYTES;
            mbar_arrive_expect_tx(&kvbar[buf], bytes);
            for (int pg = 0; pg < kKeyBlock / kPage; ++pg) {
                const int phys = page_of(kb, pg);
                const int lp = kb * (kKeyBlock / kPage) + pg;
                if (phys < 0) {
                    if (lp * kPage < kv_len) record_status(p.status, BI_DEV_BAD_INDEX);
                    continue;
                }
                const int64_t off = (int64_t(phys) * p.Hkv + g) * int64_t(C::PAGE_BYTES);
                bulk_load(sK(buf) + pg * C::PAGE_BYTES, static_cast<const uint8_t *>(p.k_cache) + off,
                          C::PAGE_BYTES, &kvbar[buf]);
                bulk_load(sV(buf) + pg * C::PAGE_BYTES, static_cast<const uint8_t *>(p.v_cache) + off,
                          C::PAGE_BYTES, &kvbar[buf]);
            }
        }
        kvpending |= 1u << buf;
    };
    // the tile's q and dO rows (TMA, 64-value boxes, 128-byte swizzle; rows
    // past the chunk are other rows' data or zeros, and a row's dQ depends
    // on that row alone, so they are left as they land)
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(qbar, 2u * C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < D / 64; ++x) {
            tma_load_3d(sQ + x * C::BOX_BYTES, &tq, qbar, 64 * x, h, int(row0));
            tma_load_3d(sDO + x * C::BOX_BYTES, &tdo, qbar, 64 * x, h, int(row0));
        }
    }
    bool qpending = true;
    fetch(0, 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
    // warps w and w + 4 share TMEM lane quarter w % 4, each taking half of
    // the columns
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t lane_base = tmem_addr(tmem, 32 * quarter, 0);
    const int i = 32 * quarter + lane;  // this thread's query row (TMEM lane)
    const bool row_ok = i < rows;
    const int t = pos0 + i;          // its absolute position
    const float lse2 = row_ok ? p.lse2[(row0 + i) * p.Hq + h] : 0.0f;
    const float delta = row_ok ? p.delta[(row0 + i) * p.Hq + h] : 0.0f;
    const float cs = p.scale_log2;

    const uint32_t idesc_s = idesc_bf16_f32(128, kKeyBlock, 0, 0);
    const uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);
    const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sDO);
    const uint64_t qd0 = sdesc_sw128(q_addr, 16, 1024);  // q, dO: K-major, swizzled
    const uint64_t dd0 = sdesc_sw128(do_addr, 16, 1024);
    uint32_t phase = 0;
    bool ok = true;
    const int last_key = pos0 + rows - 1;  // the tile's last visible key
    int buf = 0;
    for (int kb = 0; ok && kb * kKeyBlock <= last_key; ++kb) {
        const int k0 = kb * kKeyBlock;
        const uint32_t kb_addr = smem_u32(sK(buf)), vb_addr = smem_u32(sV(buf));
        if (qpending) {  // (first step) the q and dO tiles
            ok = block_wait(qbar, 0, ctl);
            if (!ok) break;
            qpending = false;
        }
        ok = block_wait(&kvbar[buf], (kvphase >> buf) & 1u, ctl);  // this block's K and V
        if (!ok) break;
        kvphase ^= 1u << buf;
        kvpending &= ~(1u << buf);
        // Pages not copied become zeros, and so do the keys past the sequence
        // in its last page: K enters dQ += dS K, where a masked key's zero
        // dS must not meet a stale NaN (V only enters dP, masked by
        // selection, but is zeroed alike).
        {
            constexpr int PP = C::PAGE_BYTES / 16;  // 16-byte pieces of a page block
            for (int pg = 0; pg < kKeyBlock / kPage; ++pg) {
                const int key0 = k0 + pg * kPage;
                const bool whole = page_of(kb, pg) < 0;
                if (!whole && key0 + kPage <= kv_len) continue;  // copied, every key in
                const int valid = whole ? 0 : kv_len - key0;     // keys of the page in the sequence
                for (int e = threadIdx.x; e < 2 * PP; e += kBwdThreads) {
                    const int piece = e % PP;
                    const uint32_t off = uint32_t(piece) * 16u;
                    const int r = int(off / (D * 16)) * 8 + int(off % 128) / 16;  // key of the piece
                    if (r < valid) continue;
                    uint8_t *dst = (e < PP ? sK(buf) : sV(buf)) + pg * C::PAGE_BYTES + off;
                    *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            // descriptors by offset (16-byte units) from the step-0 ones
            const uint64_t kd = sdesc_plain(kb_addr, 128, C::KGROUP_BYTES);
            const uint64_t vd = sdesc_plain(vb_addr, 128, C::KGROUP_BYTES);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t koff = ((k >> 2) * C::BOX_BYTES + (k & 3) * 32) / 16;  // K-major, swizzled
                mma_ss(tmem + C::S_COL, qd0 + koff, kd + 16 * k, idesc_s, k > 0 ? 1u : 0u);
                mma_ss(tmem + C::DP_COL, dd0 + koff, vd + 16 * k, idesc_s, k > 0 ? 1u : 0u);
            }
            mma_commit(bar);
        }
        // the next key block streams into the other buffer meanwhile (the
        // previous block's products, which read it, have completed)
        if ((kb + 1) * kKeyBlock <= last_key) fetch(kb + 1, buf ^ 1);
        ok = block_wait(bar, phase, ctl);
        phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
        // ---------------------------------------------------- dS (row = query)
#pragma unroll 1
        for (int c = half * (kKeyBlock / 64); c < (half + 1) * (kKeyBlock / 64); ++c) {
            uint32_t sv[32], dp[32];
            tmem_ld32(lane_base + C::S_COL + 32 * c, sv);
            tmem_ld32(lane_base + C::DP_COL + 32 * c, dp);
            tmem_wait_ld(sv);
            tmem_wait_ld(dp);
            uint32_t dk[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float dv[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int key = k0 + 32 * c + j + u;
                    const bool vis = row_ok && key <= t;
                    const float pr = ex2(__fmaf_rn(__uint_as_float(sv[j + u]), cs, -lse2));
                    const float ds = __fmul_rn(pr, __fsub_rn(__uint_as_float(dp[j + u]), delta));
                    dv[u] = vis ? ds : 0.0f;
                }
                dk[j / 2] = pack2(dv[0], dv[1]);
            }
            tmem_st16(lane_base + C::S_COL + packed_chunk_col(c), dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        // ---------------------------------------------------- dQ += dS K
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint64_t kd = sdesc_plain(kb_addr, C::KGROUP_BYTES, 128);
#pragma unroll
            for (int jj = 0; jj < kKeyBlock / 16; ++jj)
                mma_ts(tmem + C::ACC0, tmem + C::S_COL + packed_step_col(jj),
                       kd + uint64_t(jj) * (C::PAGE_BYTES / 16), idesc_acc, (kb > 0 || jj > 0) ? 1u : 0u);
            mma_commit(bar);
        }
        ok = block_wait(bar, phase, ctl);
        phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
        buf ^= 1;
    }
    cp_async_wait<0>();  // no copy may still be landing when the block leaves
    if (!ok) {
        if (threadIdx.x == 0) {
            mma_commit(drain);
            drain_wait(drain, 0, p.timeout_ns);
            for (int bb = 0; bb < 2; ++bb)
                if (kvpending & (1u << bb)) drain_wait(&kvbar[bb], (kvphase >> bb) & 1u, p.timeout_ns);
            if (qpending) drain_wait(qbar, 0, p.timeout_ns);
        }
    } else {
        // every thread takes part in the warp's TMEM loads; rows past the
        // chunk store nothing
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.dq) + ((row0 + i) * p.Hq + h) * D;
#pragma unroll 1
        for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
            uint32_t a[32];
            tmem_ld32(lane_base + C::ACC0 + 32 * c, a);
            tmem_wait_ld(a);
            if (!row_ok) continue;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 v;
                v.x = pack2(__fmul_rn(__uint_as_float(a[8 * q + 0]), p.scale),
                            __fmul_rn(__uint_as_float(a[8 * q + 1]), p.scale));
                v.y = pack2(__fmul_rn(__uint_as_float(a[8 * q + 2]), p.scale),
                            __fmul_rn(__uint_as_float(a[8 * q + 3]), p.scale));
                v.z = pack2(__fmul_rn(__uint_as_float(a[8 * q + 4]), p.scale),
                            __fmul_rn(__uint_as_float(a[8 * q + 5]), p.scale));
                v.w = pack2(__fmul_rn(__uint_as_float(a[8 * q + 6]), p.scale),
                            __fmul_rn(__uint_as_float(a[8 * q + 7]), p.scale));
                reinterpret_cast<uint4 *>(dst + 32 * c)[q] = v;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace

size_t attn_bwd_ws_bytes(int64_t rows) { return size_t(rows) * 2 * sizeof(float); }

cudaError_t launch_attention_backward(const CUtensorMap &tq, const CUtensorMap &tdo,
                                      const AttnBwdParams &p_in, int head_dim, int64_t rows,
                                      int num_sms, cudaStream_t s)
{
    AttnBwdParams p = p_in;
    // Delta and lse2 of every (token, head) row, in the workspace
    {
        const int64_t blocks = (rows + 7) / 8, cap = int64_t(num_sms) * 16;
        attn_bwd_prep_kernel<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 256, 0, s>>>(
            static_cast<const uint16_t *>(p.o), static_cast<const uint16_t *>(p.dout), p.lse, rows,
            head_dim, p.lse2, p.delta);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int64_t dkv_blocks = int64_t(p.B) * p.Hkv * p.num_key_blocks;
    const int64_t dq_blocks = int64_t(p.B) * p.Hq * p.num_q_tiles;
    if (dkv_blocks > INT32_MAX || dq_blocks > INT32_MAX) return cudaErrorInvalidValue;
    cudaError_t e;
    if (head_dim == 128) {
        using C = BwdCfg<128>;
        if ((e = cudaFuncSetAttribute(attn_bwd_dkv_kernel<128>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(attn_bwd_dq_kernel<128>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)) != cudaSuccess)
            return e;
        attn_bwd_dkv_kernel<128><<<unsigned(dkv_blocks), kBwdThreads, C::SMEM, s>>>(tq, tdo, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        attn_bwd_dq_kernel<128><<<unsigned(dq_blocks), kBwdThreads, C::SMEM, s>>>(tq, tdo, p);
    } else {
        using C = BwdCfg<64>;
        if ((e = cudaFuncSetAttribute(attn_bwd_dkv_kernel<64>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(attn_bwd_dq_kernel<64>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)) != cudaSuccess)
            return e;
        attn_bwd_dkv_kernel<64><<<unsigned(dkv_blocks), kBwdThreads, C::SMEM, s>>>(tq, tdo, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        attn_bwd_dq_kernel<64><<<unsigned(dq_blocks), kBwdThreads, C::SMEM, s>>>(tq, tdo, p);
    }
    return cudaGetLastError();
}

}  // namespace bi
