// attention.cu -- batch-invariant attention over a paged KV cache.
//
// neican.ai insight, "技术原理与创新点解析", batch-invariant attention bullet:
// the KV-cache page table is updated before the kernel launches, and a
// split reduction fixes the SIZE of each split rather than the number of
// splits, so the reduction order is the same however many query tokens are
// processed.  liuwei.blog, "破解之道": FlashAttention-2 parallelises over
// queries and reduces over keys/values, and the order in which the keys of a
// token are reduced must not depend on whether the cache was empty (prefill)
// or full (decode).  xitu-tech news, "构建确定性解决方案", attention item.
//
// The method as built here.  For a query row at absolute position t the keys
// 0..t are cut into splits of 256 keys aligned to key 0.  For each split s,
// on its own:
//   S      = Q K_s^T                    tcgen05, M=128 rows, N=256 keys, fp32
//   c      = scale * log2(e); keys j > t are masked out
//   m_s    = round(c * max_j S_j)        (= max_j round(c S_j): c > 0)
//   p_j    = 2^fma(S_j, c, -m_s),  l_s = sum_j p_j   (a fixed order, tree8 below)
//   O_s    = bf16(p) V_s                tcgen05, P read from tensor memory
// and the partials are merged from split 0 upwards, always in that order:
//   m' = max(m, m_s), a = 2^(m - m'), c = 2^(m_s - m')
//   l' = l a + l_s c,  O' = O a + O_s c          (separately rounded fp32)
//   out = O / l,  lse = (m + log2 l) ln 2.
// One kernel body serves decode (rows = the Hq/Hkv query heads of one
// token) and prefill (rows = 128 tokens of one head); a row's arithmetic is
// the same instruction sequence in both, so a token's output has the same
// bits in decode, full prefill and chunked prefill of any chunk size.
//
// Decode divides a sequence's splits among blocks (`splits_per_cta`).  A
// block whose range starts at split 0 merges in registers; every other block
// writes each split's own partial (m_s, l_s, O_s) to the workspace, and
// attn_combine continues the merge from where block 0 stopped, split by
// split, with the same merge function.  The bits therefore do not depend on
// how many blocks served a sequence.
//
// Block of 640 threads, one per SM (about 225 KB shared memory; 512 TMEM
// columns as two 256-column buffers, each holding a split's logits, then
// its P in columns 0-127 and O_s in columns 128-255):
//   warp 0     producer: Q by TMA once; per split the 16 pages of K and of
//              V, one bulk copy per page block (gathered through the page
//              table; the cache keeps each page block in the tensor core's
//              core-matrix order, so it is used in place), into a 3-slot
//              ring, in the order K0 K1 V0 K2 V1 ...; V rows past the
//              sequence end are zero (copies of a zero page, explicit stores
//              for the partial page) so that 0 * stale never reaches O.
//   warp 1     TMEM allocation and MMA issue (one thread): QK^T of split
//              s+1 runs while split s is in softmax (double-buffered TMEM).
//   warps 4-7, 16-19  softmax of one split, two warps per TMEM lane
//              quarter (warp w may only reach lanes 32(w%4)..+31): warps
//              4-7 take the first 16 lanes of their quarter, 16-19 the last
//              16, four threads a row (softmax_lanes16).  Decode spreads the
//              query heads over the four lane quarters.
//   warps 8-15 merge ("fold") of O_s into the running output, two per lane
//              quarter (one per half of the head dim), overlapping the next
//              split's softmax; warps 2-3 idle (they fill the producer's
//              warpgroup, whose registers go to the fold warps).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"
#include "bi_ptx.cuh"

namespace bi {
namespace {

// Warp roles, by warpgroup (four warps): group 0 = producer (warp 0), MMA
// (warp 1) and two idle warps; group 1 (warps 4-7) and group 4 (16-19)
// softmax; groups 2 and 3 (warps 8-15) merge ("fold").  Softmax and fold
// warp w serve TMEM lane quarter w % 4; softmax warps 4-7 take lanes 0-15 of
// their quarter, 16-19 lanes 16-31; fold warps 8-11 take the first half of
// the head dim, 12-15 the second.  The block is launched with 96 registers a
// thread; group 0 gives back all but kRegsCtl and the fold groups take
// kRegsFold (setmaxnreg), so that a fold thread holds its half row of the
// output in registers:
//   128 (kRegsCtl + 96 + 2 kRegsFold + 96) <= 640 * 96.
constexpr int THREADS = 640;
constexpr int kLaunchRegs = 96;
constexpr int kRegsCtl = 56, kRegsFold = 104;
static_assert(128 * (kRegsCtl + 2 * kLaunchRegs + 2 * kRegsFold) <= THREADS * kLaunchRegs,
              "the register split must fit the block's launch allocation");
constexpr int kFoldThreads = 256;
constexpr float kLn2 = 0.693147180559945309f;

template <int D>
struct Cfg {
    static constexpr int KB = D / 64;                   // 128-byte column blocks of a row
    static constexpr int Q_KB_BYTES = 128 * 128;        // one column block of the Q tile
    static constexpr int Q_BYTES = KB * Q_KB_BYTES;
    // A cache page block (16 keys x D) in core-matrix order: 2 key groups
    // of D/8 core matrices (8 keys x 8 values, 128 contiguous bytes).
    static constexpr int PAGE_BYTES = kPage * D * 2;
    static constexpr int KGROUP_BYTES = PAGE_BYTES / 2;  // stride between 8-key groups
    static constexpr int KV_BYTES = (kSplit / kPage) * PAGE_BYTES;  // one split of K or V
    static constexpr int NSLOT = 3;
    static constexpr int ML_BYTES = 2 * 128 * 2 * 4;   // (m_s, l_s) per row, two buffers
    static constexpr int BAR_BYTES = 256;
    static constexpr int SLACK = 768;                  // alignment slack of the base
    static constexpr int SMEM = SLACK + ML_BYTES + Q_BYTES + NSLOT * KV_BYTES + BAR_BYTES;
    // shared addresses fit the 14-bit field (16-byte units) of a matrix descriptor
    static_assert(SMEM + 4096 <= (1 << 18), "descriptor address field");
    // TMEM: two buffers of 256 columns.  In buffer b: S over all 256
    // columns; P (bf16 pairs) written over its first 128; O_s in the next D.
    static constexpr uint32_t BUF_COLS = 256, P_OFF = 0, O_OFF = 128, TMEM_COLS = 512;
    static constexpr int REC = D + 4;                   // floats per spilled partial
};

// Source of the all-zero value pages past a sequence's end.
__device__ __align__(128) uint8_t g_zero_page[kPage * 128 * 2];

// ---------------------------------------------------------------- merge

__device__ __forceinline__ void merge_scales(float m, float ms, float &mn, float &a, float &c)
{
    mn = fmaxf(m, ms);
    a = ex2(__fsub_rn(m, mn));
    c = ex2(__fsub_rn(ms, mn));
}

__device__ __forceinline__ float merge_val(float x, float a, float xs, float c)
{
    return __fadd_rn(__fmul_rn(x, a), __fmul_rn(xs, c));
}

__device__ __forceinline__ float finish_lse(float m, float l)
{
    return __fmul_rn(__fadd_rn(m, log2f(l)), kLn2);
}

template <int D>
__device__ __forceinline__ void write_out(const float (&O)[D], float l, float m,
                                          __nv_bfloat16 *orow, float *lse_ptr)
{
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        uint4 v;
        v.x = pack_bf16x2(__fdiv_rn(O[8 * c + 0], l), __fdiv_rn(O[8 * c + 1], l));
        v.y = pack_bf16x2(__fdiv_rn(O[8 * c + 2], l), __fdiv_rn(O[8 * c + 3], l));
        v.z = pack_bf16x2(__fdiv_rn(O[8 * c + 4], l), __fdiv_rn(O[8 * c + 5], l));
        v.w = pack_bf16x2(__fdiv_rn(O[8 * c + 6], l), __fdiv_rn(O[8 * c + 7], l));
        reinterpret_cast<uint4 *>(orow)[c] = v;
    }
    if (lse_ptr) *lse_ptr = finish_lse(m, l);
}

__device__ bool wait_drain(uint64_t *bar, uint32_t parity, uint64_t timeout_ns)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs))
        if (global_ns() - t0 > timeout_ns) return false;
    return true;
}

// ---------------------------------------------------------------- work item

struct Item {
    int b, g, h;          // sequence, kv head, query head (prefill)
    int s0, s1, n_splits; // split range of this block; splits of the sequence
    int kv_len;           // keys in the cache for this sequence
    int key0, kend;       // keys key0 .. kend-1 of the sequence are this block's;
                          // split s covers key0 + (s - s0) 256 .. +255 (below kend)
    int q_row0;           // prefill: first packed token of the tile
    int rows;             // prefill: valid tokens in the tile
    int pos0;             // prefill: absolute position of the tile's first row
};

__device__ __forceinline__ int key_of(const Item &it, int s) { return it.key0 + (s - it.s0) * kSplit; }

// Decode work division: blocks per sequence, and the splits a block of a
// sequence of n splits covers (its first block merges splits 0 .. c-1).
// With blocks_per_seq set, each sequence is cut into that many blocks of
// ceil(n / blocks_per_seq) splits, so a long sequence gets long blocks and a
// short one short blocks; otherwise every block covers splits_per_cta.
// The division never changes the output bits.
__device__ __forceinline__ int decode_blocks(const AttnParams &p)
{
    return p.blocks_per_seq > 0 ? p.blocks_per_seq
                                : (p.max_splits + p.splits_per_cta - 1) / p.splits_per_cta;
}
#if BI_INVARIANT
__device__ __forceinline__ int decode_chunk(const AttnParams &p, int n)
{
    return p.blocks_per_seq > 0 ? max(1, (n + p.blocks_per_seq - 1) / p.blocks_per_seq)
                                : p.splits_per_cta;
}
#endif

// Decode: whether this block alone covers the whole sequence, and the index
// of the record a block that does not hands its merged range over in.
__device__ __forceinline__ bool item_whole(const Item &it)
{
    return it.key0 == 0 && it.kend == it.kv_len && it.s1 == it.n_splits;
}
__device__ __forceinline__ int item_rec(const Item &it)
{
#if BI_INVARIANT
    return it.s1 - 1;  // its last split
#else
    return it.s0;      // its block number
#endif
}

#if !BI_INVARIANT
// Variant-off decode: the sequence's keys are cut into cnt ranges of R keys
// (R a whole number of pages), cnt = min(blocks per sequence, its 256-key
// splits) -- the split SIZE follows the load.  Block x covers keys x R ..
// min((x + 1) R, L) - 1 in 256-key pieces counted from x R.
__device__ __forceinline__ int variant_range(int L, int nblk)
{
    const int n = (L + kSplit - 1) / kSplit;
    const int cnt = min(nblk, n);
    const int per = (L + cnt - 1) / cnt;
    return (per + kPage - 1) / kPage * kPage;
}
#endif

// Work item idx of a launch.  Decode: idx = x + nblk (g + Hkv z), block x of
// the split range of kv head g of the z-th sequence of the launch order
// (longest first).  Prefill: idx = h + Hq (xr + tiles b), query head h of
// tile tiles-1-xr (longest first) of sequence b.  Items past a sequence's
// end are empty (false).
__device__ __forceinline__ bool make_item(const AttnParams &p, int idx, Item &it)
{
    if (p.decode) {
        const int nblk = decode_blocks(p);
        const int x = idx % nblk, r = idx / nblk;
        const int z = r / p.Hkv;
        it.b = p.order ? p.order[z] : z;
        it.g = r - z * p.Hkv;
        it.h = 0;
        it.kv_len = p.seq_lens[it.b];
        it.n_splits = (it.kv_len + kSplit - 1) / kSplit;
        if (it.n_splits > p.max_splits) {  // longer than the declared maximum
            if (threadIdx.x == 0) record_status(p.status, BI_DEV_BAD_INDEX);
            return false;
        }
        if (it.kv_len <= 0) return false;
#if BI_INVARIANT
        const int c = decode_chunk(p, it.n_splits);
        it.s0 = x * c;
        if (it.s0 >= it.n_splits) return false;
        it.s1 = min(it.n_splits, it.s0 + c);
        it.key0 = it.s0 * kSplit;
        it.kend = it.kv_len;
#else
        const int R = variant_range(it.kv_len, nblk);
        it.key0 = x * R;
        if (it.key0 >= it.kv_len) return false;
        it.kend = min(it.kv_len, it.key0 + R);
        it.s0 = x;
        it.s1 = x + (it.kend - it.key0 + kSplit - 1) / kSplit;
#endif
        it.q_row0 = it.rows = it.pos0 = 0;
    } else {
        const int r = idx / p.Hq;
        it.h = idx - r * p.Hq;
        it.b = r / p.num_q_tiles;
        it.g = it.h / p.group;
        const int tile = p.num_q_tiles - 1 - (r - it.b * p.num_q_tiles);  // long tiles first
        const int q0 = p.cu_q[it.b];
        const int n = p.cu_q[it.b + 1] - q0;
        if (tile * 128 >= n) return false;
        const int ctx = p.ctx_lens[it.b];
        it.kv_len = ctx + n;
        it.q_row0 = q0 + tile * 128;
        it.rows = min(128, n - tile * 128);
        it.pos0 = ctx + tile * 128;
        const int t_max = it.pos0 + it.rows - 1;
        it.s0 = 0;
        it.s1 = t_max / kSplit + 1;
        it.n_splits = (it.kv_len + kSplit - 1) / kSplit;
        it.key0 = 0;
        it.kend = it.kv_len;
    }
    return true;
}

// Byte offset, inside a page block in core-matrix order, of the 16 bytes
// holding values 8c..8c+7 of key r.
template <int D>
__device__ __forceinline__ uint32_t page_off(int r, int c)
{
    return uint32_t(r >> 3) * (D * 16) + uint32_t(c) * 128u + uint32_t(r & 7) * 16u;
}

// ---------------------------------------------------------------- kernel

// The order of the split sum l_s, shared by both softmax paths below.  The
// 256 keys of a split are cut into 32-key chunks; inside a chunk, key
// 32c + 8i + 2u + j (i < 4, u < 4, j < 2) belongs to class u.  For each class
// u, S_u accumulates, chunk by chunk in key order, the chunk's eight class-u
// values summed as ((a0 + b0) + (a1 + b1)) + ((a2 + b2) + (a3 + b3)) with
// a_i = p[32c + 8i + 2u], b_i = p[32c + 8i + 2u + 1].  Then
// l_s = (S_0 + S_1) + (S_2 + S_3).
__device__ __forceinline__ float tree8(float a0, float b0, float a1, float b1, float a2, float b2,
                                       float a3, float b3)
{
    return __fadd_rn(__fadd_rn(__fadd_rn(a0, b0), __fadd_rn(a1, b1)),
                     __fadd_rn(__fadd_rn(a2, b2), __fadd_rn(a3, b3)));
}

// p = 2^(S * cs - m_s), one rounding (fused multiply-add).  Both softmax
// paths below use it, so a key's p has the same bits in decode and prefill.
__device__ __forceinline__ float logit(float s, float cs, float m_s)
{
    return ex2(__fmaf_rn(s, cs, -m_s));
}

// Softmax of one split for 16 TMEM lanes of a lane quarter (one warp; the
// quarter's other 16 lanes belong to its second softmax warp).  Thread
// t = u + 4 v holds rows v and v + 8 of the 16 lanes and, of each row and
// each 32-key chunk c, the keys 32c + 8i + 2u and 32c + 8i + 2u + 1 (i < 4)
// -- class u of the order above -- read with the 16-lane TMEM shape, a chunk
// a load, the next load in flight.  Pass 1 takes the row maximum (exact in
// any order; four accumulators a row break the chain, two xor shuffles join
// the row's four threads).  Pass 2 computes p, writes the chunk's packed P
// (P column 16c + 4i + u, the matching 16-lane store) over columns this warp
// has already read, and adds the chunk's eight class-u values to the class
// sum as tree8 does; the two xor shuffles at the end give
// (S_u + S_u^1) + (S_u^2 + S_u^3), which commutativity makes
// (S_0 + S_1) + (S_2 + S_3) on every thread.  So a row's m_s, l_s and P have
// the same bits whichever lanes and warp hold the row.  sb is the TMEM
// address of the first of the 16 lanes at the buffer's first column; t_lo
// and t_hi are the last visible keys of rows v and v + 8; HI says whether
// rows 8..15 are computed.  A chunk whose 32 keys every row of the thread
// sees takes a path without masks.
template <bool HI>
__device__ __forceinline__ void softmax_lanes16(uint32_t sb, int k0, int t_lo, int t_hi, float cs,
                                                float (&m_s)[2], float (&l_s)[2])
{
    constexpr int NC = kSplit / 32;  // 32-key chunks
    const int u = threadIdx.x & 3;
    // last key visible to both of this thread's rows; a chunk whose keys all
    // come at or before it takes the path without masks
    const int t_min = HI ? min(t_lo, t_hi) : t_lo;
    // r[4 i + 2 h + j] of chunk c: key k0 + 32 c + 8 i + 2 u + j of row h
    auto key = [&](int c, int i, int j) { return k0 + 32 * c + 8 * i + 2 * u + j; };
    auto whole = [&](int c) { return k0 + 32 * c + 31 <= t_min; };
    float mx[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) mx[0][i] = mx[1][i] = -INFINITY;
    auto chunk_max = [&](const uint32_t *r, int c) {
        if (whole(c)) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    mx[0][i] = fmaxf(mx[0][i], __uint_as_float(r[4 * i + j]));
                    if (HI) mx[1][i] = fmaxf(mx[1][i], __uint_as_float(r[4 * i + 2 + j]));
                }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int kj = key(c, i, j);
                    if (kj <= t_lo) mx[0][i] = fmaxf(mx[0][i], __uint_as_float(r[4 * i + j]));
                    if (HI && kj <= t_hi)
                        mx[1][i] = fmaxf(mx[1][i], __uint_as_float(r[4 * i + 2 + j]));
                }
        }
    };
    // Pass 1 holds four chunks' loads in flight (two 64-key loads, one
    // wait): a TMEM load under the block's load takes ~150 cycles, far more
    // than the 16 maxima of a chunk.
    {
        uint32_t ra[32], rb[32];
#pragma unroll 1
        for (int c = 0; c < NC; c += 4) {
            tmem_ld_16x256b_x8(sb + 32 * c, ra);
            tmem_ld_16x256b_x8(sb + 32 * (c + 2), rb);
            tmem_wait_ld(ra);
            tmem_wait_ld(rb);
            chunk_max(ra, c);
            chunk_max(ra + 16, c + 1);
            chunk_max(rb, c + 2);
            chunk_max(rb + 16, c + 3);
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float mr = fmaxf(fmaxf(mx[h][0], mx[h][1]), fmaxf(mx[h][2], mx[h][3]));
        mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, 1));
        mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, 2));
        m_s[h] = __fmul_rn(mr, cs);
    }

    // Chunk c's P goes to columns 16c .. 16c + 15, which the loads of chunks
    // c/2 .. c have read (waited for); the load in flight reads columns from
    // 32(c + 1) on.
    float S[2] = {0.0f, 0.0f};
    auto chunk_exp = [&](const uint32_t (&r)[16], int c) {
        float e0[8], e1[8];
        if (whole(c)) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    e0[2 * i + j] = logit(__uint_as_float(r[4 * i + j]), cs, m_s[0]);
                    e1[2 * i + j] = HI ? logit(__uint_as_float(r[4 * i + 2 + j]), cs, m_s[1]) : 0.0f;
                }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int kj = key(c, i, j);
                    const float x0 = logit(__uint_as_float(r[4 * i + j]), cs, m_s[0]);
                    e0[2 * i + j] = kj <= t_lo ? x0 : 0.0f;
                    e1[2 * i + j] = 0.0f;
                    if (HI) {
                        const float x1 = logit(__uint_as_float(r[4 * i + 2 + j]), cs, m_s[1]);
                        e1[2 * i + j] = kj <= t_hi ? x1 : 0.0f;
                    }
                }
        }
        S[0] = __fadd_rn(S[0], tree8(e0[0], e0[1], e0[2], e0[3], e0[4], e0[5], e0[6], e0[7]));
        if (HI) S[1] = __fadd_rn(S[1], tree8(e1[0], e1[1], e1[2], e1[3], e1[4], e1[5], e1[6], e1[7]));
        uint32_t pk[8];  // 16x128b.x4 store operands: [2 i + row h]
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            pk[2 * i] = pack_bf16x2(e0[2 * i], e0[2 * i + 1]);
            pk[2 * i + 1] = HI ? pack_bf16x2(e1[2 * i], e1[2 * i + 1]) : 0u;
        }
        __syncwarp();  // the rows of a warp may have taken different paths
        tmem_st_16x128b_x4(sb + 16 * c, pk);
    };
    // loops kept rolled (a small instruction footprint: the block's other
    // warps run other code on the same sub-partitions), two chunks a trip
    uint32_t ra[16], rb[16];
    tmem_ld_16x256b_x4(sb, ra);
#pragma unroll 1
    for (int c = 0; c < NC; c += 2) {
        tmem_wait_ld16(ra);
        tmem_ld_16x256b_x4(sb + 32 * (c + 1), rb);
        chunk_exp(ra, c);
        tmem_wait_ld16(rb);
        if (c + 2 < NC) tmem_ld_16x256b_x4(sb + 32 * (c + 2), ra);
        chunk_exp(rb, c + 1);
    }
    tmem_wait_st();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        S[h] = __fadd_rn(S[h], __shfl_xor_sync(0xffffffffu, S[h], 1));
        S[h] = __fadd_rn(S[h], __shfl_xor_sync(0xffffffffu, S[h], 2));
        l_s[h] = S[h];
    }
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    attn_split_kernel(const __grid_constant__ CUtensorMap tq, const AttnParams p)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024 - (raw & 1023)) & 1023;
    if (pad > uint32_t(C::SLACK)) {  // cannot happen with a 1 KB-aligned base
        if (threadIdx.x == 0) record_status(p.status, BI_DEV_BAD_INDEX);
        return;
    }
    uint8_t *smem = smem_raw + pad;
    float *sML = reinterpret_cast<float *>(smem);               // [2][128][2]
    uint8_t *sQ = smem + C::ML_BYTES;
    uint8_t *sKV = sQ + C::Q_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(sKV + C::NSLOT * C::KV_BYTES);
    uint64_t *empty = full + C::NSLOT;
    uint64_t *barQ = empty + C::NSLOT;
    uint64_t *barQfree = barQ + 1;  // the item's last QK done: Q may be replaced
    uint64_t *barS = barQfree + 1;  // [2] S of buffer b computed
    uint64_t *barP = barS + 2;      // [2] P and (m_s, l_s) of buffer b written (256 arrivals)
    uint64_t *barO = barP + 2;      // [2] O_s of buffer b computed
    uint64_t *barF = barO + 2;      // [2] O_s of buffer b merged, buffer free
    uint64_t *drain = barF + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(barQ, 1);
        mbar_init(barQfree, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&barS[b], 1);
            mbar_init(&barP[b], 256);
            mbar_init(&barO[b], 1);
            mbar_init(&barF[b], kFoldThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
    // The item of this block's r-th round: items are ordered longest first
    // and dealt to the blocks in a snake (round r even: block b takes item
    // r G + b; odd: r G + G - 1 - b), so that every block's total is close to
    // the mean instead of block 0 taking the longest item of every round.
    // Every role walks the same sequence.
    const auto item_of = [&](int rnd) {
        const int G = int(gridDim.x), b = int(blockIdx.x);
        return rnd * G + ((rnd & 1) ? G - 1 - b : b);
    };

    // The block serves work items item_of(0), item_of(1), ...
    // (longest first).  Every role walks the same items and counts the
    // splits it has seen (gs): split number gs uses TMEM buffer gs & 1 with
    // barrier parity (gs >> 1) & 1, and its loads are numbers 2 gs, 2 gs + 1
    // of the ring.  An item's last QK releases the Q buffer for the next.
    // Each warpgroup sets its registers once, at one instruction for all its
    // warps, before its warps take their roles: warpgroup 0 gives back, the
    // fold warpgroups take, the softmax ones keep the launch's.
    if (warp < 4) {
        regs_release<kRegsCtl>();
        if (warp == 0) {
            // ====================================================== producer
            bool ok = true;
            uint32_t armed = 0, armed_parity = 0;
            int gs = 0, nq = 0;
            int64_t li = 0;  // running load number: slot li % NSLOT
            for (int rnd = 0, idx = item_of(0); ok && idx < p.items; idx = item_of(++rnd)) {
                Item it;
                if (!make_item(p, idx, it)) continue;
                const int32_t *bt_row = p.block_table + int64_t(it.b) * p.max_pages;
                auto lookup = [&](int s) -> int {
                    const int lp = key_of(it, s) / kPage + lane;  // logical page
                    if (lane >= kSplit / kPage || lp * kPage >= it.kend) return -1;
                    return lp < p.max_pages ? __ldg(bt_row + lp) : -2;
                };
                // Load list (relative split j, n splits): K0, K1, V0, K2, V1, K3,
                // ..., V(n-2), V(n-1): keys two splits ahead of values, the order
                // in which the MMA warp consumes them.  Lane i < 16 looks up page
                // i of a split ahead of use (4 splits in flight) and issues that
                // page's copy itself; the id is checked where it is used.
                const int n = it.s1 - it.s0;
                int pages[4];
    #pragma unroll
                for (int e = 0; e < 4; ++e) pages[e] = e < n ? lookup(it.s0 + e) : -1;
                auto emit = [&](int which, int j) -> bool {
                    const int s = it.s0 + j;
                    const int slot = int(li % C::NSLOT);
                    const uint32_t phase = uint32_t(li / C::NSLOT) & 1u;
                    int phys = pages[j & 3];
                    if (phys == -2 || phys >= p.num_pages || phys < -1) {  // bad id: zero page, flagged
                        if (which == 0) record_status(p.status, BI_DEV_BAD_INDEX);
                        phys = -1;
                    }
                    const int nk = min(kSplit, it.kend - key_of(it, s));  // valid keys, >= 1
                    const int full_pages = nk / kPage;
                    const int npages = (nk + kPage - 1) / kPage;
                    int got = 1;
                    if (lane == 0) got = wait_inl(&empty[slot], phase ^ 1u, ctl) ? 1 : 0;
                    got = __shfl_sync(0xffffffffu, got, 0);
                    if (!got) return false;
                    uint8_t *dst = sKV + slot * C::KV_BYTES;
                    const uint8_t *cache = static_cast<const uint8_t *>(which ? p.v_cache : p.k_cache);
                    const int partial_phys = __shfl_sync(0xffffffffu, phys, full_pages & 31);
                    // V: the partial last page is copied by the whole warp, with
                    // the keys past the sequence end set to zero.
                    if (which == 1 && full_pages < npages) {
                        const int pg = full_pages;
                        const bool good = partial_phys >= 0;
                        const int valid = nk - pg * kPage;
                        const uint8_t *blk =
                            cache + (int64_t(partial_phys) * p.Hkv + it.g) * int64_t(C::PAGE_BYTES);
                        for (int e = lane; e < kPage * (D / 8); e += 32) {
                            const int r = e / (D / 8), c = e % (D / 8);
                            const uint32_t off = page_off<D>(r, c);
                            uint4 v = make_uint4(0, 0, 0, 0);
                            if (good && r < valid) v = __ldg(reinterpret_cast<const uint4 *>(blk + off));
                            *reinterpret_cast<uint4 *>(dst + pg * C::PAGE_BYTES + off) = v;
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                    // K: the pages holding valid keys.  V: whole valid pages plus
                    // all-zero pages past the end.  One bulk copy per page.
                    const int copies = which ? (kSplit / kPage) - (npages - full_pages) : npages;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[slot], uint32_t(copies) * C::PAGE_BYTES);
                        armed |= 1u << slot;
                        armed_parity = (armed_parity & ~(1u << slot)) | (phase << slot);
                    }
                    __syncwarp();
                    const int pg = lane;
                    bool issue;
                    const uint8_t *src = g_zero_page;
                    if (which == 0) {
                        issue = pg < npages;
                        if (phys >= 0) src = cache + (int64_t(phys) * p.Hkv + it.g) * int64_t(C::PAGE_BYTES);
                    } else {
                        issue = pg < kSplit / kPage && !(pg == full_pages && full_pages < npages);
                        if (pg < full_pages && phys >= 0)
                            src = cache + (int64_t(phys) * p.Hkv + it.g) * int64_t(C::PAGE_BYTES);
                    }
                    if (issue) bulk_load(dst + pg * C::PAGE_BYTES, src, C::PAGE_BYTES, &full[slot]);
                    __syncwarp();
                    ++li;
                    return true;
                };
                // the first keys go out before Q (their slots free up earlier)
                if (n > 0) ok = emit(0, 0);
                if (ok && n > 1) ok = emit(0, 1);
                // Q of this item once the previous item's QK products are done
                int gotq = 1;
                if (lane == 0) {
                    if (nq > 0) gotq = wait_inl(barQfree, uint32_t(nq - 1) & 1u, ctl) ? 1 : 0;
                    if (gotq) {
                        if (p.decode) {
                            const int rpq = p.rows_per_q;
                            mbar_arrive_expect_tx(barQ, 4u * C::KB * rpq * 128u);
                            for (int q = 0; q < 4; ++q)
                                for (int kb = 0; kb < C::KB; ++kb)
                                    tma_load_3d(sQ + kb * C::Q_KB_BYTES + q * 32 * 128, &tq, barQ,
                                                kb * 64, it.g * p.group + q * rpq, it.b);
                        } else {
                            mbar_arrive_expect_tx(barQ, uint32_t(C::Q_BYTES));
                            for (int kb = 0; kb < C::KB; ++kb)
                                tma_load_3d(sQ + kb * C::Q_KB_BYTES, &tq, barQ, kb * 64, it.h, it.q_row0);
                        }
                    }
                }
                gotq = __shfl_sync(0xffffffffu, gotq, 0);
                ok = ok && gotq;
                ++nq;
                for (int j = 0; ok && j < n; ++j) {
                    ok = emit(1, j);
                    // split j is done with its page ids: look up split j + 4
                    pages[j & 3] = (j + 4 < n) ? lookup(it.s0 + j + 4) : -1;
                    if (ok && j + 2 < n) ok = emit(0, j + 2);
                }
                gs += n;
            }
            if (!ok && lane == 0) {
                for (int s = 0; s < C::NSLOT; ++s)
                    if (armed & (1u << s)) wait_drain(&full[s], (armed_parity >> s) & 1u, p.timeout_ns);
                if (nq > 0) wait_drain(barQ, uint32_t(nq - 1) & 1u, p.timeout_ns);
            }
            (void)gs;
        } else if (warp == 1) {
            // ====================================================== MMA issue
            // Per item, tensor-pipe order QK(0), QK(1), PV(0), QK(2), PV(1), ...
            // -- the order of the producer's load list.  QK of split gs reuses
            // TMEM buffer gs & 1 once the fold warps have merged split gs - 2,
            // which may belong to the previous item.
            if (lane == 0) {
                const uint32_t idesc_qk = idesc_bf16_f32(128, kSplit, 0, 0);
                const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
                const uint32_t q_base = smem_u32(sQ);
                const uint64_t q_desc0 = sdesc_sw128(q_base, 16, 1024);
                bool ok = true;
                int gs = 0, nq = 0;
                for (int rnd = 0, idx = item_of(0); ok && idx < p.items; idx = item_of(++rnd)) {
                    Item it;
                    if (!make_item(p, idx, it)) continue;
                    const int n = it.s1 - it.s0;
                    const int64_t base = 2 * int64_t(gs);  // load number of K0
                    // load numbers of K(j) and V(j) in the list K0, K1, V0, K2, V1, ...
                    auto k_load = [&](int j) { return base + (j < 2 ? j : 2 * j - 1); };
                    auto v_load = [&](int j) { return base + min(2 + 2 * j, 2 * n - 1); };
                    auto issue_qk = [&](int j) -> bool {
                        const int g = gs + j;
                        if (g >= 2) {  // buffer g & 1 still holds split g - 2 until merged
                            if (!wait_inl(&barF[g & 1], uint32_t((g - 2) >> 1) & 1u, ctl)) return false;
                            tc_fence_after();
                        }
                        const int64_t i = k_load(j);
                        const int slot = int(i % C::NSLOT);
                        if (!wait_inl(&full[slot], uint32_t(i / C::NSLOT) & 1u, ctl)) return false;
                        tc_fence_after();
                        const uint32_t d = tmem + C::BUF_COLS * uint32_t(g & 1);
                        const uint32_t k_base = smem_u32(sKV + slot * C::KV_BYTES);
                        // K: K-major, core matrices; 16 values of the head
                        // dim are two core matrices 128 bytes apart, 8-key
                        // groups KGROUP_BYTES apart (also across pages).
                        // Descriptors by offset (16-byte units) from the
                        // step-0 ones: shared addresses stay below 2^18, so
                        // no sum carries out of the address field.
                        const uint64_t kd0 = sdesc_plain(k_base, 128, C::KGROUP_BYTES);
    #pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t kb = k >> 2, kk = k & 3;
                            mma_ss(d, q_desc0 + (kb * C::Q_KB_BYTES + kk * 32) / 16, kd0 + 16 * k,
                                   idesc_qk, k > 0 ? 1u : 0u);
                        }
                        mma_commit(&barS[g & 1]);
                        mma_commit(&empty[slot]);
                        if (j == n - 1) mma_commit(barQfree);  // the item's last use of Q
                        return true;
                    };
                    ok = wait_inl(barQ, uint32_t(nq) & 1u, ctl);
                    ++nq;
                    if (ok) ok = issue_qk(0);
                    if (ok && n > 1) ok = issue_qk(1);
                    for (int j = 0; ok && j < n; ++j) {
                        const int g = gs + j;
                        const int b = g & 1;
                        const uint32_t par = uint32_t(g >> 1) & 1u;
                        const int64_t i = v_load(j);
                        const int slot = int(i % C::NSLOT);
                        if (!wait_inl(&full[slot], uint32_t(i / C::NSLOT) & 1u, ctl)) {
                            ok = false;
                            break;
                        }
                        const uint32_t buf = tmem + C::BUF_COLS * uint32_t(b);
                        const uint32_t v_base = smem_u32(sKV + slot * C::KV_BYTES);
                        if (!wait_inl(&barP[b], par, ctl)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        // V: MN-major, core matrices; step jj is page jj;
                        // its two 8-key groups are KGROUP_BYTES apart, 8-value
                        // blocks of the head dim 128 bytes apart.
                        const uint64_t vd0 = sdesc_plain(v_base, C::KGROUP_BYTES, 128);
    #pragma unroll
                        for (int jj = 0; jj < kSplit / 16; ++jj)
                            mma_ts(buf + C::O_OFF, buf + C::P_OFF + 8 * jj,
                                   vd0 + uint64_t(jj) * (C::PAGE_BYTES / 16), idesc_pv, jj > 0 ? 1u : 0u);
                        mma_commit(&barO[b]);
                        mma_commit(&empty[slot]);
                        if (j + 2 < n) ok = issue_qk(j + 2);
                    }
                    gs += n;
                }
                if (!ok) {
                    mma_commit(drain);
                    wait_drain(drain, 0, p.timeout_ns);
                }
            }
        }
        // warps 2 and 3: no role
    } else if ((warp >= 4 && warp < 8) || warp >= 16) {
        // ====================================================== softmax
        // The softmax warps of lane quarter q (two, 16 lanes each) and its
        // fold warps (two, one per half of the head dim) serve the same 32
        // rows; each role walks the items on its own, so that the code after
        // a role's register budget is that role's alone.
        const int q = warp & 3;
        int gs = 0;
        bool ok = true;
        for (int rnd = 0, idx = item_of(0); ok && idx < p.items; idx = item_of(++rnd)) {
            Item it;
            if (!make_item(p, idx, it)) continue;
            // whether lane quarter q holds any row of the item
            const bool active = p.decode ? q * p.rows_per_q < p.group : 32 * q < it.rows;
            const float cs = p.scale_log2;
            // this warp's 16 lanes of the quarter: lane0 .. lane0 + 15;
            // this thread's rows lane0 + v and lane0 + v + 8
            const int lane0 = 32 * q + (warp >= 16 ? 16 : 0), v = lane >> 2;
            // lanes of the quarter that hold rows (from lane 0 up)
            const int n_lanes = !active ? 0
                                : p.decode ? min(p.rows_per_q, p.group - q * p.rows_per_q)
                                           : min(32, it.rows - 32 * q);
            const bool lo = n_lanes > lane0 - 32 * q, hi = n_lanes > lane0 - 32 * q + 8;
            const int t_lo = p.decode ? it.kend - 1 : it.pos0 + lane0 + v;
            const int t_hi = p.decode ? it.kend - 1 : it.pos0 + lane0 + v + 8;
            const uint32_t lanes16 = tmem_addr(tmem, uint32_t(lane0), 0);
            for (int s = it.s0; s < it.s1; ++s) {
                const int g = gs + (s - it.s0);
                const int b = g & 1;
                const uint32_t par = uint32_t(g >> 1) & 1u;
                if (!wait_inl(&barS[b], par, ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float m_s[2] = {-INFINITY, -INFINITY}, l_s[2] = {0.0f, 0.0f};
                const uint32_t sb = lanes16 + C::BUF_COLS * uint32_t(b) + C::P_OFF;
                if (hi)
                    softmax_lanes16<true>(sb, key_of(it, s), t_lo, t_hi, cs, m_s, l_s);
                else if (lo)
                    softmax_lanes16<false>(sb, key_of(it, s), t_lo, t_hi, cs, m_s, l_s);
                if ((lane & 3) == 0) {
                    float *ml = sML + (b * 128 + lane0 + v) * 2;
                    ml[0] = m_s[0];
                    ml[1] = l_s[0];
                    ml[16] = m_s[1];  // row lane0 + v + 8
                    ml[17] = l_s[1];
                }
                tc_fence_before();
                mbar_arrive(&barP[b]);
            }
            gs += it.s1 - it.s0;
        }
    } else {
        // ====================================================== fold
        regs_take<kRegsFold>();
        const int q = warp & 3;
        const uint32_t lane_base = tmem_addr(tmem, 32 * q, 0);
        const int row_id = 32 * q + lane;  // TMEM lane of this row
        // This thread's row of an item: its last visible key t, whether its
        // lane quarter holds any row, whether the row is a real one, and
        // where its output goes.
        auto row_of = [&](const Item &it, int &t, bool &active, bool &valid, int64_t &out_row) {
            if (p.decode) {
                const int local = q * p.rows_per_q + lane;
                valid = lane < p.rows_per_q && local < p.group;
                t = it.kend - 1;  // the block's last key (the sequence's, but for a
                                  // variant-off range that ends before it)
                out_row = int64_t(it.b) * p.Hq + it.g * p.group + local;
                active = q * p.rows_per_q < p.group;
            } else {
                const int local = 32 * q + lane;
                valid = local < it.rows;
                t = it.pos0 + local;
                out_row = int64_t(it.q_row0 + local) * p.Hq + it.h;
                active = 32 * q < it.rows;
            }
        };
        int gs = 0;
        bool ok = true;
        for (int rnd = 0, idx = item_of(0); ok && idx < p.items; idx = item_of(++rnd)) {
            Item it;
            if (!make_item(p, idx, it)) continue;
            bool valid, active;
            int t;
            int64_t out_row;
            row_of(it, t, active, valid, out_row);
            // This warp merges columns col0 .. col0 + HW - 1 of its rows.
            constexpr int HW = D / 2;
            const int half = warp >= 12 ? 1 : 0;
            const int col0 = half * HW;
#if BI_INVARIANT
            // blocks after a sequence's first write every split's own partial
            const bool spill = p.decode && it.s0 > 0;
#else
            // variant-off: every block merges its own range (the grouping
            // of the merge then depends on how many blocks served it)
            const bool spill = false;
#endif
            float m = -INFINITY, l = 0.0f;
            float O[HW];
#pragma unroll
            for (int j = 0; j < HW; ++j) O[j] = 0.0f;
            for (int s = it.s0; s < it.s1; ++s) {
                const int g = gs + (s - it.s0);
                const int b = g & 1;
                const uint32_t par = uint32_t(g >> 1) & 1u;
                const uint32_t ob = lane_base + C::BUF_COLS * uint32_t(b) + C::O_OFF + col0;
                const int k0 = key_of(it, s);
                // barP: (m_s, l_s) of this split are in shared memory;
                // barO: O_s is in TMEM.
                if (!wait_inl(&barP[b], par, ctl) || !wait_inl(&barO[b], par, ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                bool released = false;
                const float m_s = sML[(b * 128 + row_id) * 2 + 0];
                const float l_s = sML[(b * 128 + row_id) * 2 + 1];
                if (active) {
                    // 16-column TMEM loads (HW / 16 per split): one at a
                    // time when a partial is written out, the next one in
                    // flight while the current one merges
                    constexpr int NCH16 = HW / 16;
                    if (spill) {
                        // not the first block of this sequence: write the
                        // split's own partial for attn_combine
                        float *rec = p.ws + ((out_row * p.max_splits) + s) * C::REC + 4 + col0;
#pragma unroll 1
                        for (int c = 0; c < NCH16; ++c) {
                            uint32_t r[16];
                            tmem_ld32x16(ob + 16 * c, r);
                            tmem_wait_ld16(r);
                            if (valid) {
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    reinterpret_cast<float4 *>(rec + 16 * c)[j] = make_float4(
                                        __uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]),
                                        __uint_as_float(r[4 * j + 3]));
                            }
                        }
                        if (valid && half == 0) {
                            rec[-4] = m_s;
                            rec[-3] = l_s;
                        }
                    } else {
                        const bool first = (s == it.s0);
                        const bool take = k0 <= t;  // the row sees at least key k0
                        float mn, a, cc;
                        merge_scales(m, m_s, mn, a, cc);
                        // the next 16 columns load while these merge
                        uint32_t r2[2][16];
                        tmem_ld32x16(ob, r2[0]);
#pragma unroll
                        for (int c = 0; c < NCH16; ++c) {
                            uint32_t(&r)[16] = r2[c & 1];
                            tmem_wait_ld16(r);
                            if (c + 1 < NCH16) tmem_ld32x16(ob + 16 * (c + 1), r2[(c + 1) & 1]);
                            if (c == NCH16 - 1) {  // O_s read: the buffer is free
                                tc_fence_before();
                                mbar_arrive(&barF[b]);
                                released = true;
                            }
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const float o = __uint_as_float(r[j]);
                                if (first)
                                    O[16 * c + j] = o;
                                else if (take)
                                    O[16 * c + j] = merge_val(O[16 * c + j], a, o, cc);
                            }
                        }
                        if (first) {
                            m = m_s;
                            l = l_s;
                        } else if (take) {
                            l = merge_val(l, a, l_s, cc);
                            m = mn;
                        }
                    }
                }
                if (!released) {
                    tc_fence_before();
                    mbar_arrive(&barF[b]);
                }
            }
            if (ok && active && valid && !spill) {
                if (!p.decode || item_whole(it)) {
                    write_out<HW>(O, l, m,
                                  static_cast<__nv_bfloat16 *>(p.o) + out_row * D + col0,
                                  (p.lse && half == 0) ? p.lse + out_row : nullptr);
                } else {
                    // a block of a sequence served by several: hand the
                    // merged state over its range (ending at split s1-1)
                    // to attn_combine (in the invariant build only the
                    // first block gets here; the others write every split)
                    float *rec = p.ws + ((out_row * p.max_splits) + item_rec(it)) * C::REC;
                    if (half == 0) {
                        rec[0] = m;
                        rec[1] = l;
                    }
#pragma unroll
                    for (int j = 0; j < HW / 4; ++j)
                        reinterpret_cast<float4 *>(rec + 4 + col0)[j] =
                            make_float4(O[4 * j], O[4 * j + 1], O[4 * j + 2], O[4 * j + 3]);
                }
            }
            gs += it.s1 - it.s0;
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Launch order of decode sequences: longest first (by split count), so that
// the block scheduler, which starts blocks in index order, ends with short
// ones (a greedy longest-processing-time schedule).  A counting sort over
// at most 1024 length buckets; the order inside a bucket is whatever the
// atomics give -- it changes which block runs when, never what a block
// computes.
__global__ void __launch_bounds__(1024) attn_order_kernel(const int32_t *__restrict__ seq_lens,
                                                          int B, int32_t *__restrict__ order)
{
    __shared__ int cnt[1024];
    __shared__ int warp_tot[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    cnt[tid] = 0;
    __syncthreads();
    auto bucket = [](int L) {
        const int n = L > 0 ? (L + kSplit - 1) / kSplit : 0;
        return 1023 - (n < 1023 ? n : 1023);  // longest in bucket 0
    };
    for (int b = tid; b < B; b += 1024) atomicAdd(&cnt[bucket(seq_lens[b])], 1);
    __syncthreads();
    // exclusive prefix sum of cnt over the buckets
    const int v = cnt[tid];
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    cnt[tid] = x - v + (warp > 0 ? warp_tot[warp - 1] : 0);
    __syncthreads();
    for (int b = tid; b < B; b += 1024) order[atomicAdd(&cnt[bucket(seq_lens[b])], 1)] = b;
}

// Continues the merge of a decode row past the first block's range, record
// by record in ascending order; one block per (sequence, query head).  The
// row's records (the first block's state, then one per later split) lie
// contiguously in the workspace; warps 1-3 copy them into shared memory,
// CH records at a time and the next chunk while warp 0 merges the current
// one, so the sequential merge reads shared memory instead of waiting on a
// memory latency every few records.  Warp 0 does exactly the merges of the
// one-warp form, in the same order, with the same functions, so CH (chosen
// from the number of rows) never changes a bit.
constexpr int kCombineThreads = 128;

template <int D, int CH>
constexpr size_t combine_smem_bytes()
{
    return size_t(2) * CH * Cfg<D>::REC * sizeof(float);
}

template <int D, int CH>
__global__ void __launch_bounds__(kCombineThreads) attn_combine_kernel(const AttnParams p)
{
    using C = Cfg<D>;
    constexpr int PER = D / 32;  // columns per lane of warp 0
    static_assert(C::REC % 4 == 0, "records of whole 16-byte pieces");
    extern __shared__ float4 s_rec4[];  // [2][CH * REC]
    float *s_rec = reinterpret_cast<float *>(s_rec4);
    const int64_t row = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (row >= int64_t(p.B) * p.Hq) return;
    const int b = static_cast<int>(row / p.Hq);
    const int L = p.seq_lens[b];
    const int n = (L + kSplit - 1) / kSplit;
    const float *base = p.ws + row * p.max_splits * C::REC;
#if BI_INVARIANT
    if (L <= 0 || n > p.max_splits) return;
    const int first_end = decode_chunk(p, n);  // splits merged by the first block
    if (n <= first_end) return;
    const int rec0 = first_end, count = n - first_end;  // records split by split
#else
    // variant-off: one record per block of keys x R .. (x + 1) R - 1
    const int nblk = decode_blocks(p);
    if (L <= 0 || n > p.max_splits) return;
    const int R = variant_range(L, nblk);
    if (R >= L) return;  // one block: its output is written
    const int rec0 = 1, count = (L + R - 1) / R - 1;    // records block by block
#endif
    // records rec0 - 1 (the state to continue from) .. rec0 + count - 1
    const float4 *src = reinterpret_cast<const float4 *>(base + int64_t(rec0 - 1) * C::REC);
    const int total = count + 1;
    const int nchunk = (total + CH - 1) / CH;
    auto copy_chunk = [&](int c, int t, int nt) {
        const int n4 = min(CH, total - c * CH) * (C::REC / 4);
        const float4 *g = src + int64_t(c) * CH * (C::REC / 4);
        float4 *d = s_rec4 + (c & 1) * CH * (C::REC / 4);
        for (int i = t; i < n4; i += nt) d[i] = __ldg(g + i);
    };
    copy_chunk(0, threadIdx.x, kCombineThreads);
    __syncthreads();
    float m = 0.0f, l = 0.0f, O[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) O[j] = 0.0f;
    for (int c = 0; c < nchunk; ++c) {
        if (warp > 0) {
            if (c + 1 < nchunk) copy_chunk(c + 1, threadIdx.x - 32, kCombineThreads - 32);
        } else {
            const float *buf = s_rec + (c & 1) * CH * C::REC;
            const int nr = min(CH, total - c * CH);
            int i = 0;
            if (c == 0) {
                m = buf[0];
                l = buf[1];
#pragma unroll
                for (int j = 0; j < PER; ++j) O[j] = buf[4 + lane * PER + j];
                i = 1;
            }
#pragma unroll 4
            for (; i < nr; ++i) {
                const float *r = buf + i * C::REC;
                float ro[PER];
#pragma unroll
                for (int j = 0; j < PER; ++j) ro[j] = r[4 + lane * PER + j];
                float mn, a, cc;
                merge_scales(m, r[0], mn, a, cc);
#pragma unroll
                for (int j = 0; j < PER; ++j) O[j] = merge_val(O[j], a, ro[j], cc);
                l = merge_val(l, a, r[1], cc);
                m = mn;
            }
        }
        __syncthreads();  // chunk c is merged and chunk c + 1 has landed
    }
    if (warp != 0) return;
    __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(p.o) + row * D + lane * PER;
#pragma unroll
    for (int j = 0; j < PER; j += 2)
        *reinterpret_cast<uint32_t *>(orow + j) = pack_bf16x2(__fdiv_rn(O[j], l), __fdiv_rn(O[j + 1], l));
    if (p.lse && lane == 0) p.lse[row] = finish_lse(m, l);
}

}  // namespace

size_t attn_smem_bytes(int head_dim) { return head_dim == 64 ? Cfg<64>::SMEM : Cfg<128>::SMEM; }

size_t attn_ws_bytes(int B, int Hq, int head_dim, int max_splits, int max_chunks)
{
    if (max_chunks <= 1) return 0;
    return size_t(B) * Hq * max_splits * (head_dim + 4) * sizeof(float);
}

// The block's register split (setmaxnreg: warpgroup 0 down to kRegsCtl,
// the fold warpgroups up to kRegsFold) must fit the registers the block is
// launched with, i.e. what the compiled kernel declares a thread -- a split
// above that would leave the fold warps waiting for registers forever.
// Checked once per kernel; a kernel that does not fit is never launched.
template <int D>
cudaError_t check_register_split()
{
    static int split_fits = 0;  // 0 not yet checked, 1 fits, -1 does not
    if (split_fits == 0) {
        cudaFuncAttributes a;
        const cudaError_t e = cudaFuncGetAttributes(&a, attn_split_kernel<D>);
        if (e != cudaSuccess) return e;
        const long r = a.numRegs;
        split_fits = (128L * (kRegsCtl + 2 * r + 2 * kRegsFold) <= long(THREADS) * r) ? 1 : -1;
    }
    return split_fits > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

cudaError_t launch_attention(const CUtensorMap &tq, const AttnParams &p_in, int head_dim,
                             cudaStream_t s)
{
    // Prefill: persistent, one block per SM (at most), each walking its
    // items in the snake order of item_of (longest first; the tiles'
    // lengths fall in steps, so the static assignment stays balanced, and a
    // block's next item overlaps the current one's tail).  Decode: one block
    // per item -- request lengths vary too much for a static assignment, and
    // the hardware hands each free SM the next block of the longest-first
    // order.
    AttnParams p = p_in;
    int64_t items;
    if (p.decode)
        items = int64_t(p.blocks_per_seq > 0 ? p.blocks_per_seq
                                             : (p.max_splits + p.splits_per_cta - 1) / p.splits_per_cta) *
                p.Hkv * p.B;
    else
        items = int64_t(p.num_q_tiles) * p.Hq * p.B;
    if (items > INT32_MAX) return cudaErrorInvalidValue;
    p.items = static_cast<int32_t>(items);
    if (p.items == 0) return cudaSuccess;
    static int sms[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (sms[dev] == 0) {
        cudaError_t e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    const unsigned grid =
        static_cast<unsigned>(p.decode ? p.items : (p.items < sms[dev] ? p.items : sms[dev]));
    cudaError_t e = head_dim == 128 ? check_register_split<128>() : check_register_split<64>();
    if (e != cudaSuccess) return e;
    if (head_dim == 128) {
        e = cudaFuncSetAttribute(attn_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<128>::SMEM);
        if (e != cudaSuccess) return e;
        attn_split_kernel<128><<<grid, THREADS, Cfg<128>::SMEM, s>>>(tq, p);
    } else {
        e = cudaFuncSetAttribute(attn_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<64>::SMEM);
        if (e != cudaSuccess) return e;
        attn_split_kernel<64><<<grid, THREADS, Cfg<64>::SMEM, s>>>(tq, p);
    }
    return cudaGetLastError();
}

cudaError_t launch_attn_order(const int32_t *seq_lens, int B, int32_t *order, cudaStream_t s)
{
    attn_order_kernel<<<1, 1024, 0, s>>>(seq_lens, B, order);
    return cudaGetLastError();
}

template <int D, int CH>
static cudaError_t launch_combine(const AttnParams &p, unsigned blocks, cudaStream_t s)
{
    constexpr size_t smem = combine_smem_bytes<D, CH>();
    const cudaError_t e = cudaFuncSetAttribute(attn_combine_kernel<D, CH>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attn_combine_kernel<D, CH><<<blocks, kCombineThreads, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_attn_combine(const AttnParams &p, int head_dim, cudaStream_t s)
{
    const int64_t rows = int64_t(p.B) * p.Hq;
    if (rows > INT32_MAX) return cudaErrorInvalidValue;
    const unsigned blocks = static_cast<unsigned>(rows);
    // few rows: long chunks (fewer copy rounds per row); many rows: short
    // ones (more blocks resident per SM); measured crossover ~500 rows
    const bool few = rows <= 512;
    if (head_dim == 128)
        return few ? launch_combine<128, 64>(p, blocks, s) : launch_combine<128, 32>(p, blocks, s);
    return few ? launch_combine<64, 64>(p, blocks, s) : launch_combine<64, 32>(p, blocks, s);
}

}  // namespace bi
