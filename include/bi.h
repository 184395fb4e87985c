/*
 * bi.h -- C ABI of the batch-invariant forward kernels for B200 (sm_100a).
 *
 * Every output row of every call below is bitwise identical whatever else is
 * in the batch: the batch size, the other rows or requests, their order, the
 * physical pages of the KV cache, how full the cache pool is, whether a token
 * is processed by decode, full prefill or chunked prefill, and how the work is
 * divided among thread blocks.  The reports on "Defeating Nondeterminism in
 * LLM Inference" trace run-to-run differences of served models to kernels
 * whose reduction strategy changes with the batch (xitu-tech news, section
 * "揭露真正元凶"; neican.ai insight, section "技术原理与创新点解析") and name the
 * three operations that need batch-invariant versions: RMSNorm, matmul and
 * attention (same sections, and xitu-tech news, section "构建确定性解决方案").
 *
 * Conventions for every entry point
 *   - Pointers marked "device" are CUDA device pointers on the current device;
 *     pointers marked "host" are host memory.  The caller owns every buffer;
 *     the library never allocates device memory.
 *   - bfloat16 tensors are dense and row-major (last index fastest).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on it and returns without synchronising.
 *   - Argument errors are detected on the host before anything is launched
 *     and return BI_ERR_INVALID (or BI_ERR_UNSUPPORTED / BI_ERR_WORKSPACE);
 *     a failed launch returns BI_ERR_CUDA.  Errors that only the device can
 *     see (an out-of-range page id or slot, a bounded wait that ran out) are
 *     recorded in a per-device status word that bi_device_status() reads.
 *   - No C++ exception crosses this boundary.
 */
#ifndef BI_H
#define BI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BI_OK = 0,
    BI_ERR_INVALID = 1,      /* bad pointer, size, alignment or layout        */
    BI_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. head_dim 96)        */
    BI_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed             */
    BI_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out            */
    BI_ERR_WORKSPACE = 5,    /* workspace missing or smaller than required    */
    BI_ERR_DEVICE_INDEX = 6  /* the device met an out-of-range page id / slot */
} bi_status;

typedef enum {
    BI_BF16 = 0,
    BI_F32 = 1
} bi_dtype;

/* Tokens per KV-cache page. */
#define BI_PAGE_SIZE 16
/* Keys per attention split: the fixed split SIZE (not split count). */
#define BI_SPLIT_KEYS 256

/*
 * Paged KV cache (vLLM-style paging, as the neican.ai insight describes in
 * section "技术原理与创新点解析", batch-invariant attention bullet).
 *   k_cache, v_cache : device, bf16.  num_pages x num_kv_heads page blocks of
 *                      16 x head_dim values, each block contiguous
 *                      (32 * head_dim bytes) and stored in core-matrix order:
 *                        block[kg][vg][r][c] = X[token 8*kg + r][value 8*vg + c]
 *                      for kg in 0..1, vg in 0..head_dim/8-1, r, c in 0..7
 *                      (token = position inside the page).  This is the
 *                      order the tensor core reads its operands in, so a page
 *                      block is copied to shared memory unchanged.  Blocks
 *                      are indexed [page][kv head].  Both caches start
 *                      16-byte aligned.  bi_kv_write produces this layout.
 *   block_table      : device, int32 [num_seqs, max_pages_per_seq];
 *                      block_table[b][i] is the physical page holding tokens
 *                      16*i .. 16*i+15 of sequence b.  Entries past a
 *                      sequence's last page are never read.
 *   page_size        : must be 16.
 *   head_dim         : 64 or 128.
 */
typedef struct bi_paged_kv {
    void *k_cache;
    void *v_cache;
    const int32_t *block_table;
    int32_t max_pages_per_seq;
    int32_t num_pages;
    int32_t page_size;
    int32_t num_kv_heads;
    int32_t head_dim;
} bi_paged_kv;

/*
 * bi_rmsnorm -- batch-invariant RMSNorm (xitu-tech news, "构建确定性解决方案",
 * RMSNorm item; neican.ai insight, "技术原理与创新点解析", data-parallel
 * RMSNorm bullet: one batch row per core, its whole reduction inside that
 * core, never a split reduction).
 *
 *   y[r, j] = round( x[r, j] * rsqrt( sum_i x[r, i]^2 / H + eps ) * w[j] )
 *
 *   x : device, bf16 [M, H];  w : device, bf16 [H];
 *   y : device, [M, H] of out_dtype (BI_BF16: round to nearest even; BI_F32).
 *   Requirements: H % 8 == 0, 8 <= H <= 65536, x, w, y 16-byte aligned,
 *   y must not overlap x.  M == 0 is a no-op.
 *   fp32 arithmetic; each row is reduced by one thread block in an order that
 *   depends only on H.
 */
bi_status bi_rmsnorm(const void *x, const void *w, void *y, int64_t M, int64_t H, float eps,
                     bi_dtype out_dtype, void *stream);

/*
 * bi_add_rmsnorm -- the residual form of bi_rmsnorm used between the
 * sublayers of a pre-norm decoder: the residual stream x takes the
 * sublayer's output, then is normalised.
 *
 *   x[r, j] <- round( x[r, j] + delta[r, j] )          (fp32 add, bf16 RNE)
 *   y[r, :]  = bi_rmsnorm(x[r, :]) of the updated row, bit for bit
 *
 *   x : device, bf16 [M, H], read and written;  delta : device, bf16 [M, H];
 *   w, y, eps, out_dtype, requirements: as bi_rmsnorm; y overlaps neither x
 *   nor delta.  Same one-block-per-row order, fixed by H alone.
 */
bi_status bi_add_rmsnorm(void *x, const void *delta, const void *w, void *y, int64_t M,
                         int64_t H, float eps, bi_dtype out_dtype, void *stream);

/*
 * bi_matmul -- batch-invariant matrix product (xitu-tech news,
 * "构建确定性解决方案", matmul item: no split-K chosen from the input size, one
 * fixed kernel configuration with one tile size; neican.ai insight,
 * "技术原理与创新点解析", data-parallel matmul bullet: 2-D output tiles, each
 * core computes its whole dot products).
 *
 *   C[m, n] = round( sum_k A[m, k] * W[n, k] )        (C = A W^T)
 *
 *   a : device, bf16 [M, K];  w : device, bf16 [N, K] (output-feature-major,
 *   the nn.Linear weight layout);  c : device, [M, N] of out_dtype.
 *   Requirements: K % 8 == 0, N % 8 == 0, M, N, K >= 1, all three pointers
 *   16-byte aligned, c not overlapping a or w.  M == 0 is a no-op.
 *   One fixed 256 x 256 output tile computed by a pair of SMs, K consumed in
 *   64-wide slices in ascending order with fp32 accumulation on the tensor
 *   cores; there is no split-K and no choice of kernel by shape.
 *   ws / ws_bytes: workspace (device); the invariant build needs none
 *   (bi_matmul_workspace_bytes returns 0, ws may be NULL).  The variant-off
 *   build uses it for split-K partial sums.
 */
bi_status bi_matmul(const void *a, const void *w, void *c, int64_t M, int64_t N, int64_t K,
                    bi_dtype out_dtype, void *ws, size_t ws_bytes, void *stream);
size_t bi_matmul_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * bi_matmul_grouped -- many matrix products of one shape family in one
 * launch, as bi_matmul computes each: the rows offsets[g] .. offsets[g+1]-1
 * of A and C (group g, e.g. the tokens routed to expert g) are multiplied
 * by group g's weight, rows g*N .. g*N+N-1 of w:
 *
 *   C[r, n] = round( sum_k A[r, k] * w[g*N + n, k] )    offsets[g] <= r < offsets[g+1]
 *
 *   a : device, bf16 [rows, K];  w : device, bf16 [groups * N, K] (the
 *   groups' weights stacked, each output-feature-major);  c : device,
 *   [rows, N] of out_dtype;  offsets : device, int64 [groups + 1],
 *   non-decreasing within 0..rows (rows outside every group are left
 *   unwritten).  The tile list is built on the device from the offsets (no
 *   read-back): each group's rows are cut into the same fixed 256 x 256 tiles
 *   as bi_matmul, with the same K order, so a row's bits do not depend on
 *   how many rows its group holds.  1 <= groups <= 256; K, N % 8 == 0;
 *   pointers 16-byte aligned.  No split-K in either build.
 */
bi_status bi_matmul_grouped(const void *a, const void *w, void *c, const int64_t *offsets,
                            int32_t groups, int64_t rows, int64_t N, int64_t K, bi_dtype out_dtype,
                            void *stream);

/*
 * Fused forms of the RMSNorm and residual steps around a transformer block's
 * matmuls (the RMSNorm item beside the matmul item of xitu-tech news,
 * "构建确定性解决方案").  Both run the bi_matmul product (same tiles, same
 * K order, no split-K in either build) and change only its epilogue, row by
 * row, so every row stays independent of M.
 *
 * bi_fold_norm_weight -- wf[n, k] = round(W[n, k] * w[k]): a matmul weight
 *   with the preceding RMSNorm's weight folded in (once, at load time).
 *   W, wf : device, bf16 [N, K];  w : device, bf16 [K].  K % 8 == 0, N >= 0,
 *   16-byte aligned; wf may be W (in place), no other overlap.  The product
 *   of two bf16 values is exact in fp32, so wf is the correctly rounded
 *   product.
 *
 * bi_rmsnorm_matmul -- RMSNorm of each row of x followed by the product with
 *   a folded weight:
 *
 *     r[m]    = rsqrt( (1/K) * sum_k x[m, k]^2 + eps )          (fp32)
 *     C[m, n] = round( r[m] * sum_k x[m, k] * wf[n, k] )
 *
 *   x : device, bf16 [M, K];  wf : device, bf16 [N, K];  c : device, [M, N]
 *   of out_dtype.  r is computed first by bi_rmsnorm's own reduction (the
 *   same order, so r[m] has the bits of bi_rmsnorm's rstd of that row) into
 *   the workspace -- M floats instead of the normalised [M, K] rows -- and
 *   the matmul's epilogue scales each row by it; the normalised row is never
 *   rounded to bf16.  ws : device workspace of
 *   bi_rmsnorm_matmul_workspace_bytes(M) bytes, 16-byte aligned.
 *   Requirements as bi_matmul, K <= 65536, and eps finite and >= 0.
 *
 * bi_matmul_residual -- the product added to a residual stream:
 *
 *     C[m, n] = round( R[m, n] + round( sum_k A[m, k] * W[n, k] ) )
 *
 *   (the inner rounding is bi_matmul's, so the result equals bi_matmul
 *   followed by the addition bit for bit).  a : bf16 [M, K];  w : bf16
 *   [N, K];  r, c : bf16 [M, N], c may be r (in place), no other overlap.
 *   Requirements as bi_matmul.
 */
/*
 * Backward passes for a trainer that must reproduce the sampler's numbers
 * (on-policy RL; xitu-tech news, "强化学习的突破").  Every reduction runs in
 * a fixed order, so the results are the same bits on every run.
 *
 * bi_rmsnorm_backward -- gradients of y = RMSNorm(x) * w (bi_rmsnorm) for an
 *   upstream gradient dy, with r = rsqrt(mean_i x_i^2 + eps):
 *     dx[m, j] = r w_j dy[m, j] - x[m, j] (r^3 / H) sum_i w_i dy[m, i] x[m, i]
 *     dw[j]    = sum_m dy[m, j] x[m, j] r[m]
 *   x, dy : device bf16 [M, H];  w : bf16 [H];  dx : [M, H], dw : [H] of
 *   out_dtype.  A row's dx depends on that row only (one block per row, sums
 *   in an order fixed by H); dw adds the rows in chunks of 64 from row 0,
 *   each chunk ascending, then the chunks ascending.  ws : device workspace
 *   of bi_rmsnorm_backward_workspace_bytes(M, H) bytes.  H % 8 == 0,
 *   8 <= H <= 65536, 16-byte aligned pointers.
 *
 * bi_transpose -- out[c, r] = a[r, c] for bf16 a [R, C]; out has rows of
 *   ld_out >= R values, those past R set to 0.  A bit copy.
 *
 * bi_matmul_backward -- for C = A W^T (bi_matmul):  dA = dC W  [M, K]  and
 *   dW = dC^T A  [N, K], both on the invariant matmul (the transposes of W,
 *   dC and A made in the workspace by bi_transpose; dW's sum over the M rows
 *   is that matmul's K loop, rows padded to a multiple of 8 with zeros).
 *   dc : bf16 [M, N];  a : bf16 [M, K];  w : bf16 [N, K];  da, dw : of
 *   out_dtype, either may be NULL.  ws : bi_matmul_backward_workspace_bytes
 *   (M, N, K) bytes.  Requirements as bi_matmul.  A row of dA depends on
 *   that row of dC only.
 *
 * bi_swiglu_backward -- gradients of out = silu(g) * u (bi_swiglu) for an
 *   upstream gradient dout, with s = 1 / (1 + e^-g):
 *     dgate = dout * u * (s + g s (1 - s)),   dup = dout * g * s
 *   (1 - s evaluated as 1 / (1 + e^g)); fp32, every operation rounded.
 *   gu : device, bf16 [T, 2F] (gate columns, then up);  dout : device, bf16
 *   [T, F];  dgu : device, [T, 2F] of out_dtype (dgate, then dup: the layout
 *   of gu, ready for the stacked gate/up matmul's backward).  F % 8 == 0,
 *   16-byte aligned pointers, dgu overlapping neither input.  Each element
 *   depends on its own inputs only.
 *
 * bi_rope_backward -- gradient of bi_rope_kv_write's rotation: the rotation
 *   by the negative angle,
 *     dx_i       = dy_i cos(a) + dy_{i+d/2} sin(a)
 *     dx_{i+d/2} = dy_{i+d/2} cos(a) - dy_i sin(a),   a = pos * theta^(-2i/d)
 *   with cos and sin evaluated in double precision and rounded to float as
 *   the forward evaluates them; fp32, every product and sum rounded.
 *   dy : device, bf16, T rows of num_heads heads of head_dim values, rows
 *   ld_dy values apart;  dx : device, of out_dtype, same shape, rows ld_dx
 *   values apart (so a head set inside a wider row, e.g. the q or k part of
 *   a fused q/k/v gradient, can be read and written in place of a copy);
 *   positions : device, int32 [T].  head_dim in {64, 128}, ld % 8 == 0,
 *   ld >= num_heads * head_dim, theta > 1, 16-byte aligned dy and dx.
 */
size_t bi_rmsnorm_backward_workspace_bytes(int64_t M, int64_t H);
bi_status bi_rmsnorm_backward(const void *x, const void *w, const void *dy, void *dx, void *dw,
                              int64_t M, int64_t H, float eps, bi_dtype out_dtype, void *ws,
                              size_t ws_bytes, void *stream);
bi_status bi_transpose(const void *a, void *out, int64_t R, int64_t C, int64_t ld_out,
                       void *stream);
bi_status bi_swiglu_backward(const void *gu, const void *dout, void *dgu, int64_t T, int64_t F,
                             bi_dtype out_dtype, void *stream);
bi_status bi_rope_backward(const void *dy, int64_t ld_dy, const int32_t *positions, void *dx,
                           int64_t ld_dx, int64_t T, int32_t num_heads, int32_t head_dim,
                           float theta, bi_dtype out_dtype, void *stream);
size_t bi_matmul_backward_workspace_bytes(int64_t M, int64_t N, int64_t K);
bi_status bi_matmul_backward(const void *dc, const void *a, const void *w, void *da, void *dw,
                             int64_t M, int64_t N, int64_t K, bi_dtype out_dtype, void *ws,
                             size_t ws_bytes, void *stream);

/*
 * bi_rope_table -- the rotary angles of bi_rope_kv_write as a table:
 *   table[p, i] = ( cos(p theta^(-2i/d)), sin(p theta^(-2i/d)) ),  p < max_pos, i < d/2
 * evaluated in double precision and rounded to fp32 exactly as
 * bi_rope_kv_write evaluates them (the same floats).  table : device, fp32
 * [max_pos, d/2, 2], 16-byte aligned.  d = head_dim in {64, 128}; theta > 1.
 *
 * bi_rmsnorm_matmul_rope_kv -- the attention input of a transformer block:
 * RMSNorm of x folded into the QKV matmul (as bi_rmsnorm_matmul, wf the
 * folded [N, K] weight, N = (Hq + 2 Hkv) d, its row statistics in ws, of
 * bi_rmsnorm_matmul_workspace_bytes(T) bytes), then RoPE of the q and k
 * heads and the cache write of k and v, in the matmul's epilogue.  The
 * result is bi_rmsnorm_matmul followed by bi_rope_kv_write bit for bit (the
 * product is rounded to bf16 first, the rotation uses the table's angles
 * and the same fp32 operations); the [T, N] product is never stored.
 *   x : device, bf16 [T, K];  positions : device, int32 [T], each in
 *   [0, max_pos) (a row outside writes nothing and sets BI_ERR_DEVICE_INDEX
 *   in the status word);  slot_mapping : device, int64 [T] (< 0: no cache
 *   write; >= num_pages * 16: no write and BI_ERR_DEVICE_INDEX);  q_out :
 *   device, bf16 [T, Hq, d];  the cache as in bi_kv_write.  Requirements as
 *   bi_matmul for (T, N, K), Hq % Hkv == 0.  The cache pages written must be
 *   distinct from the pages the same launch's other rows write (one slot per
 *   token).
 */
bi_status bi_rope_table(float *table, int32_t max_pos, int32_t head_dim, float theta,
                        void *stream);
bi_status bi_rmsnorm_matmul_rope_kv(const void *x, const void *wf, float eps,
                                    const bi_paged_kv *kv, const float *rope_table,
                                    int32_t max_pos, const int32_t *positions,
                                    const int64_t *slot_mapping, void *q_out, int64_t T,
                                    int64_t K, int32_t Hq, void *ws, size_t ws_bytes,
                                    void *stream);
bi_status bi_fold_norm_weight(const void *W, const void *w, void *wf, int64_t N, int64_t K,
                              void *stream);
size_t bi_rmsnorm_matmul_workspace_bytes(int64_t M);
bi_status bi_rmsnorm_matmul(const void *x, const void *wf, void *c, int64_t M, int64_t N,
                            int64_t K, float eps, bi_dtype out_dtype, void *ws, size_t ws_bytes,
                            void *stream);
bi_status bi_matmul_residual(const void *a, const void *w, const void *r, void *c, int64_t M,
                             int64_t N, int64_t K, void *stream);

/*
 * bi_kv_write -- write the step's new keys and values into the paged cache
 * before attention runs, so that the attention kernel sees one consistent
 * KV layout (neican.ai insight, "技术原理与创新点解析", batch-invariant
 * attention bullet: the page table is updated before the kernel launches).
 *
 *   k_new, v_new : device, bf16 [T, num_kv_heads, head_dim]
 *   slot_mapping : device, int64 [T]; token t goes to page slot/16, offset
 *                  slot%16.  slot < 0 skips the token.  A slot at or past
 *                  num_pages*16 is skipped and flags BI_ERR_DEVICE_INDEX.
 *   Bit copy.  T == 0 is a no-op.  Two tokens of one call must not share a
 *   slot.
 */
bi_status bi_kv_write(const bi_paged_kv *kv, const void *k_new, const void *v_new,
                      const int64_t *slot_mapping, int64_t T, void *stream);

/*
 * bi_attention_decode -- one new query token per sequence against the paged
 * cache (neican.ai insight, "技术原理与创新点解析", batch-invariant attention
 * bullet: fix the SIZE of each split rather than the number of splits, so
 * the reduction order does not depend on how many query tokens are
 * processed; xitu-tech news, "构建确定性解决方案", attention item).
 *
 *   q        : device, bf16 [B, Hq, head_dim] (the token at position L_b - 1)
 *   o        : device, bf16 [B, Hq, head_dim]
 *   lse      : device, fp32 [B, Hq] natural-log sum of exp of the scaled
 *              logits, or NULL
 *   seq_lens : device, int32 [B]; L_b >= 1 includes the new token, whose K/V
 *              bi_kv_write has already placed in the cache.
 *   max_seq_len : host int, >= every L_b (sizes the grid and workspace).
 *   scale    : softmax scale (usually 1/sqrt(head_dim)).
 *   splits_per_cta : how many 256-key splits one thread block handles; 0
 *              picks a value from B, Hq/Hkv and the SM count.  It changes
 *              only the speed: the output bits do not depend on it.
 *   ws, ws_bytes : device workspace of at least
 *              bi_attention_decode_workspace_bytes(...) bytes, 16-byte
 *              aligned: the launch order of the sequences (longest first)
 *              and, when a sequence spans several blocks, the fp32 split
 *              partials.
 *   Query head h reads kv head h / (Hq / num_kv_heads).  Keys are reduced in
 *   splits of 256 aligned to position 0; each split's partial (max, sum,
 *   weighted values) is formed on its own and the partials are merged from
 *   split 0 upwards, in that order, whichever block computed them.
 *   Requirements: Hq % num_kv_heads == 0, Hq / num_kv_heads <= 128,
 *   head_dim in {64, 128}, q and o 16-byte aligned.
 */
bi_status bi_attention_decode(const bi_paged_kv *kv, const void *q, void *o, float *lse,
                              const int32_t *seq_lens, int32_t B, int32_t Hq,
                              int32_t max_seq_len, float scale, int32_t splits_per_cta,
                              void *ws, size_t ws_bytes, void *stream);
size_t bi_attention_decode_workspace_bytes(const bi_paged_kv *kv, int32_t B, int32_t Hq,
                                           int32_t max_seq_len, int32_t splits_per_cta);

/*
 * bi_attention_decode_noalloc -- bi_attention_decode for callers that cannot
 * allocate device memory.  (The pages have no counterpart of this entry
 * point; it is an interface convenience of this library.)
 *
 * Some callers may not call cudaMalloc or any allocating routine: code that
 * runs inside a host framework which owns every device allocation through
 * its own pool, latency-critical serving loops where an allocation could
 * synchronise the device or fail under fragmentation, and embedders whose
 * memory budget is fixed when the process starts.  This variant takes no
 * workspace: its scratch (the launch order of the sequences and the fp32
 * split partials) lives in one fixed array of BI_NOALLOC_SCRATCH_BYTES
 * inside the library, which every GPU that loads the library holds until
 * the process exits.  The caller still passes q, o, lse and seq_lens.
 *
 * Arguments, layouts and output bits are exactly those of
 * bi_attention_decode (both entry points share one launcher).  With
 * splits_per_cta == 0 the work division is picked so that the scratch fits
 * (falling back to one block per sequence, which changes only the speed);
 * an explicit splits_per_cta whose partials exceed the array returns
 * BI_ERR_WORKSPACE before any launch.  (The launch order of the largest
 * batch, 65535 sequences, always fits.)
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any
 * stream capture.  The address is kept for the life of the process: this
 * entry point does not support a device reset (cudaDeviceReset) between
 * calls.  Every call on a device shares the one array and each call writes
 * all of the scratch it later reads, so nothing has to start at zero; two
 * calls whose work overlaps on the GPU (different streams without ordering)
 * race on the array and must not be issued.  No device memory is allocated
 * or freed.
 */
#define BI_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
bi_status bi_attention_decode_noalloc(const bi_paged_kv *kv, const void *q, void *o, float *lse,
                                      const int32_t *seq_lens, int32_t B, int32_t Hq,
                                      int32_t max_seq_len, float scale, int32_t splits_per_cta,
                                      void *stream);

/*
 * bi_attention_prefill -- causal attention of a batch of prompt chunks
 * against the paged cache (liuwei.blog, "破解之道": the order in which the
 * keys of token 1000 are reduced must not depend on whether the cache was
 * empty (prefill) or full (decode); neican.ai insight, "技术原理与创新点解析").
 *
 *   q        : device, bf16 [T_total, Hq, head_dim], sequences packed
 *   o        : device, bf16 [T_total, Hq, head_dim]
 *   lse      : device, fp32 [T_total, Hq] or NULL
 *   cu_q     : device, int32 [B + 1]; sequence b owns rows cu_q[b]..cu_q[b+1]-1
 *   ctx_lens : device, int32 [B]; tokens of sequence b already in the cache
 *              before this chunk.  The chunk's own K/V must already be in the
 *              cache (bi_kv_write), so the cache holds ctx_lens[b] +
 *              (cu_q[b+1]-cu_q[b]) tokens of sequence b.
 *   max_q_len : host int, >= every chunk length.
 *   The row at absolute position t attends keys 0..t with the same 256-key
 *   splits, the same per-split arithmetic and the same merge order as
 *   bi_attention_decode, so a token's output is bitwise the same in decode,
 *   full prefill and chunked prefill of any chunk size.
 *   ws / ws_bytes: reserved, pass NULL / 0 (bi_attention_prefill_workspace_bytes
 *   returns 0).
 */
bi_status bi_attention_prefill(const bi_paged_kv *kv, const void *q, void *o, float *lse,
                               const int32_t *cu_q, const int32_t *ctx_lens, int32_t B,
                               int32_t Hq, int64_t T_total, int32_t max_q_len, float scale,
                               void *ws, size_t ws_bytes, void *stream);
size_t bi_attention_prefill_workspace_bytes(const bi_paged_kv *kv, int32_t B, int32_t Hq,
                                            int32_t max_q_len);

/*
 * bi_attention_backward -- gradients of bi_attention_prefill (and of decode,
 * which is prefill with one row per sequence) for an upstream gradient dO,
 * for the trainer side of on-policy RL (xitu-tech news, "强化学习的突破").
 * With P_ij = exp(scale q_i.k_j - lse_i) over the visible keys j <= t_i,
 * dP_ij = dO_i.v_j, Delta_i = dO_i.o_i and dS_ij = P_ij (dP_ij - Delta_i):
 *   dq_i = scale sum_j dS_ij k_j
 *   dk_j = scale sum_i dS_ij q_i,   dv_j = sum_i P_ij dO_i
 * the sums for dk_j, dv_j over every row of the call's chunk of key j's
 * sequence that sees it, in all query heads of its kv group.
 *
 *   kv, q, cu_q, ctx_lens, B, Hq, T_total, max_q_len, scale : as the
 *     bi_attention_prefill call whose gradient is taken;
 *   o    : device, bf16 [T_total, Hq, d], that call's output;
 *   lse  : device, fp32 [T_total, Hq], that call's lse (natural log);
 *   dout : device, bf16 [T_total, Hq, d], the upstream gradient;
 *   max_kv_len : host int >= every ctx_lens[b] + chunk length;
 *   dq   : device, bf16 [T_total, Hq, d];
 *   dk_cache, dv_cache : device, bf16, shaped and laid out like the caches
 *     (page blocks in core-matrix order).  For each sequence, every slot of
 *     its pages up to its last key is written (slots past its length in the
 *     last page get 0); other pages are not touched.  No page may belong to
 *     two sequences of the call; dk_cache and dv_cache overlap neither cache
 *     nor each other.
 *   ws, ws_bytes : device workspace of bi_attention_backward_workspace_bytes
 *     (Hq, T_total) bytes (Delta and lse log2 e per row), 16-byte aligned.
 * Fixed orders: dk_j and dv_j sum the query heads of the group ascending,
 * then the 128-row query tiles of the chunk ascending, each tile's rows
 * reduced on the tensor core; dq_i sums the 128-key blocks from key 0
 * ascending -- a row's dq depends on that row only.  P and dS enter the
 * tensor core as bf16 (as the forward's P does); the rest is fp32.
 * Requirements: as bi_attention_prefill; d in {64, 128}.
 */
size_t bi_attention_backward_workspace_bytes(int32_t Hq, int64_t T_total);
bi_status bi_attention_backward(const bi_paged_kv *kv, const void *q, const void *o,
                                const void *dout, const float *lse, const int32_t *cu_q,
                                const int32_t *ctx_lens, int32_t B, int32_t Hq, int64_t T_total,
                                int32_t max_q_len, int32_t max_kv_len, float scale, void *dq,
                                void *dk_cache, void *dv_cache, void *ws, size_t ws_bytes,
                                void *stream);

/*
 * Decoder glue.  The reports measure invariance end to end by completing one
 * prompt greedily many times among other requests and counting the distinct
 * completions (xitu-tech news, "显著成果与高昂成本"; liuwei.blog, "实验成果").
 * They name no layer beyond RMSNorm, matmul and attention; the decoder around
 * them is read as the plain pre-norm transformer.  Each operation below
 * computes an output row from its own input row only.
 */

/*
 * bi_embedding -- out[t, :] = table[ids[t], :]  (bit copy; also a row gather
 * of any [V, H] bf16 matrix).
 *   table : device, bf16 [V, H];  ids : device, int32 [T];
 *   out : device, bf16 [T, H].  H % 8 == 0, table and out 16-byte aligned.
 *   An id outside 0..V-1 leaves its row unwritten and flags
 *   BI_ERR_DEVICE_INDEX.  T == 0 is a no-op.
 */
bi_status bi_embedding(const void *table, int64_t V, int64_t H, const int32_t *ids, void *out,
                       int64_t T, void *stream);

/*
 * bi_rope_kv_write -- rotary position embedding of the new tokens' queries
 * and keys, fused with the write of their keys and values into the paged
 * cache (the cache is updated before attention runs, as bi_kv_write does).
 *
 *   qkv : device, bf16 [T, (Hq + 2 Hkv) * d], each row [q heads | k heads |
 *         v heads] (the output of one matmul with the stacked q, k, v
 *         weights);  positions : device, int32 [T], absolute positions;
 *   slot_mapping : device, int64 [T], as bi_kv_write (slot < 0 skips the
 *         token's K/V; a slot past the pool flags BI_ERR_DEVICE_INDEX);
 *   q_out : device, bf16 [T, Hq, d], the rotated queries.
 *   For i < d/2, angle = pos * theta^(-2i/d) (evaluated in double, its
 *   cosine and sine rounded to float); the pair (x_i, x_{i + d/2}) becomes
 *     (x_i cos - x_{i+d/2} sin,  x_{i+d/2} cos + x_i sin)
 *   in fp32 with every product and sum rounded, then bf16 RNE.  V is copied
 *   unchanged.  Requirements: Hq % Hkv == 0, d in {64, 128}, theta > 1,
 *   qkv and q_out 16-byte aligned.
 */
bi_status bi_rope_kv_write(const bi_paged_kv *kv, const void *qkv, const int32_t *positions,
                           const int64_t *slot_mapping, void *q_out, int64_t T, int32_t Hq,
                           float theta, void *stream);

/*
 * bi_swiglu -- out[t, j] = round( silu(g) * u ),  g = gu[t, j],
 * u = gu[t, F + j], silu(g) = g / (1 + e^-g), fp32.
 *   gu : device, bf16 [T, 2F] (gate columns first, then up: the output of
 *   one matmul with the stacked gate and up weights);  out : device, bf16
 *   [T, F].  F % 8 == 0, both 16-byte aligned.
 */
bi_status bi_swiglu(const void *gu, void *out, int64_t T, int64_t F, void *stream);

/*
 * bi_argmax -- greedy choice: out[t] = the lowest index j of the maximum of
 * logits[t, :].  An exact selection (no rounding), so it does not depend on
 * the order of the search.  NaN entries are never chosen; a row of NaN only
 * gives 0.
 *   logits : device, fp32 [T, V], 16-byte aligned, V % 4 == 0;
 *   out : device, int32 [T].
 */
bi_status bi_argmax(const float *logits, int64_t T, int64_t V, int32_t *out, void *stream);

/*
 * bi_sample -- one token per row, the random draw belonging to the request,
 * so that a request's token never depends on the rest of the batch.  The
 * reports tie bitwise-identical sampling to on-policy reinforcement learning
 * (xitu-tech news, "强化学习的突破"; neican.ai insight, "未来发展路径预测") and
 * set the random seed aside as the cause of run-to-run differences
 * (vpshk.cn, "AI随机性的根源探析"); they describe no sampler, so this one is
 * the plainest reading.
 *
 *   temperature[t] <= 0: the greedy choice (as bi_argmax).  Otherwise, with
 *   z_j = logits[t, j] / temperature[t] and w_j = e^(z_j - max z):
 *     kept set K = { j : w_j >= tau }, tau the largest value such that the
 *       weights >= tau hold at least top_p[t] of the total (ties at tau are
 *       all kept; top_p >= 1 keeps everything);
 *     u = (x >> 8) * 2^-24, x the first output word of Philox4x32-10
 *       (Salmon et al., SC 2011) with key (seed lo, seed hi) and counter
 *       (offset lo, offset hi, 0, 0) -- e.g. seed per request, offset = the
 *       token's position;
 *     the token is the first j of K, in index order, at which the running
 *       sum of w over K exceeds u * sum_K w.
 *   Every sum has an order fixed by V alone (fp32).
 *   logits : device, fp32 [T, V], 1 <= V <= 53248;  temperature, top_p :
 *   device, fp32 [T];  seed, offset : device, uint64 [T];  out : device,
 *   int32 [T].  T == 0 is a no-op.
 */
bi_status bi_sample(const float *logits, int64_t T, int64_t V, const float *temperature,
                    const float *top_p, const uint64_t *seed, const uint64_t *offset, int32_t *out,
                    void *stream);

/*
 * Mixture-of-experts feed-forward.  The model of the reports' experiment is
 * a mixture of experts (Qwen3-235B-A22B; xitu-tech news, "显著成果与高昂成本";
 * neican.ai insight, "技术原理与创新点解析"); they describe no router.  The
 * plainest reading: each token picks its k experts by largest router logit
 * (lowest index on ties), its gate weights are the softmax of the selected
 * logits, its output is the gate-weighted sum of its experts' outputs in
 * rank order.  The experts' matmuls go through bi_matmul, whose rows do not
 * depend on how many tokens an expert received, so a token's output does
 * not depend on the batch.
 */

/*
 * bi_moe_route -- experts[t, i] = index of the i-th largest of
 * logits[t, 0..E-1] (ties: lower index first); weights[t, i] =
 * e^(l_i - l_0) / sum_j e^(l_j - l_0) over the chosen k (fp32, summed in
 * rank order).
 *   logits : device, fp32 [T, E] (finite);  experts : device, int32 [T, k];
 *   weights : device, fp32 [T, k].  1 <= k <= min(E, 16), E <= 256.
 */
bi_status bi_moe_route(const float *logits, int64_t T, int32_t E, int32_t k, int32_t *experts,
                       float *weights, void *stream);

/*
 * bi_moe_dispatch -- groups the T*k entries (entry t*k + i = token t's i-th
 * expert) by expert, keeping entry order inside an expert: offsets[e] ..
 * offsets[e+1]-1 are expert e's positions; order[p] is the entry at position
 * p, pos[entry] its position, token_sorted[p] = order[p] / k (the rows to
 * gather, e.g. with bi_embedding).  Integer work, exact.  An expert id
 * outside 0..E-1 is skipped (pos = -1) and flags BI_ERR_DEVICE_INDEX.
 * T == 0 only zeroes the offsets (the other arrays may then be NULL).
 *   experts : device, int32 [T, k];  offsets : device, int64 [E + 1];
 *   order, pos : device, int64 [T*k];  token_sorted : device, int32 [T*k].
 */
bi_status bi_moe_dispatch(const int32_t *experts, int64_t T, int32_t k, int32_t E,
                          int64_t *offsets, int64_t *order, int64_t *pos, int32_t *token_sorted,
                          void *stream);

/*
 * bi_moe_combine -- out[t, :] = round( sum_{i<k} weights[t, i] *
 * y[pos[t*k + i], :] ), fp32, terms added in rank order, bf16 RNE.
 *   y : device, bf16 [T*k, H] (the experts' outputs in dispatch order);
 *   pos : device, int64 [T*k] (from bi_moe_dispatch);  weights : device,
 *   fp32 [T, k];  out : device, bf16 [T, H].  H % 8 == 0, y and out 16-byte
 *   aligned.
 */
bi_status bi_moe_combine(const void *y, const int64_t *pos, const float *weights, int64_t T,
                         int32_t k, int64_t H, void *out, void *stream);

/* Human-readable name of a status code (static string). */
const char *bi_status_string(bi_status s);

/* 1 for the batch-invariant build, 0 for the variant-off build (split-K
 * matmul, split count chosen from the load, split-reduction RMSNorm) that
 * exists to measure what invariance costs. */
int bi_build_invariant(void);

/*
 * bi_device_status -- synchronise `stream`, then read and clear the current
 * device's status word.  Returns BI_OK, BI_ERR_TIMEOUT or
 * BI_ERR_DEVICE_INDEX (the first error recorded since the last read), or
 * BI_ERR_CUDA if the synchronisation itself failed.
 */
bi_status bi_device_status(void *stream);

/*
 * bi_debug_bounded_wait -- launches one thread block that waits on a
 * barrier nothing ever arrives at, using the same bounded wait as every
 * kernel of the library, with a limit of `timeout_ns` nanoseconds
 * (1e3 .. 1e9).  The wait gives up, records BI_ERR_TIMEOUT in the status
 * word and the kernel returns normally: the context stays usable.  It exists
 * so that a test can check the timeout path without faulting the GPU.
 */
bi_status bi_debug_bounded_wait(uint64_t timeout_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_H */
