// bi_launch.h -- host-side launchers of the kernels (internal to the library;
// the public boundary is include/bi.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace bi {

// ---------------------------------------------------------------- RMSNorm
void rmsnorm_shape(int64_t H, int *items, int *threads);
cudaError_t launch_rmsnorm(const void *x, const void *w, void *y, int64_t M, int64_t H,
                           float eps, bool out_f32, int num_sms, cudaStream_t s);
// x <- round(x + delta); y <- RMSNorm(x) exactly as launch_rmsnorm computes it
cudaError_t launch_add_rmsnorm(void *x, const void *delta, const void *w, void *y, int64_t M,
                               int64_t H, float eps, bool out_f32, int num_sms, cudaStream_t s);
// r[m] = rsqrt(sum_k x[m, k]^2 / H + eps): launch_rmsnorm's reduction of the
// row (the same order, the same bits as its rstd), with nothing else written
cudaError_t launch_row_rstd(const void *x, float *r, int64_t M, int64_t H, float eps, int num_sms,
                            cudaStream_t s);

// ---------------------------------------------------------------- matmul
constexpr int kGemmBK = 64;  // K slice; the output tile is 256 x 256 per SM pair
// Rows of A and of W that each CTA of a pair loads per K slice: the box of
// both tensor maps (every form encodes them through one function) and the
// kernel's stage layout.
constexpr int kGemmCtaRows = 128;
size_t gemm_smem_bytes();
// k_splits > 1 only in the variant-off build: fp32 partial sums go to ws
// ([k_splits, M, N]) and a second kernel adds them.
int gemm_k_splits(int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tw, void *c, int M, int N,
                        int K, bool out_f32, float *ws, int k_splits, int num_sms,
                        unsigned *status, uint64_t timeout_ns, cudaStream_t s);
// Grouped: group g's rows offsets[g] .. offsets[g+1]-1 of A and C use rows
// g*N .. g*N+N-1 of W (the groups' weights stacked); offsets on the device.
constexpr int kMaxGemmGroups = 256;
cudaError_t launch_gemm_grouped(const CUtensorMap &ta, const CUtensorMap &tw, void *c, int rows,
                                int N, int K, bool out_f32, const int64_t *offsets, int groups,
                                int num_sms, unsigned *status, uint64_t timeout_ns,
                                cudaStream_t s);
// Fused epilogues of the plain product (never split along K):
//   norm:     C[m, :] = round(rs[m] * acc[m, :]), rs[m] = rsqrt(mean_k A[m, k]^2 + eps)
//             from launch_row_rstd
//   residual: C[m, :] = round(R[m, :] + round(acc[m, :]))   (R may be C)
//   QKV (rope non-null): the N = (Hq + 2 Hkv) head_dim columns of the
//             rounded product are q, k and v heads; q and k are rotated by
//             the angles of the row's position (rope_kv_kernel's arithmetic)
//             and q goes to q_out [M, Hq, head_dim], k and v to the row's
//             cache slot; C is not written.
struct GemmEpi {
    const float *rs;        // [M] row scales (norm form) or null
    const void *residual;
    const float *rope;      // [max_pos, head_dim / 2, 2]: cos, sin
    int max_pos;
    const int32_t *pos;     // [M]
    const int64_t *slots;   // [M]; < 0: no cache write
    void *q_out, *k_cache, *v_cache;
    int64_t num_pages;
    int Hq, Hkv, head_dim;
};
cudaError_t launch_gemm_fused(const CUtensorMap &ta, const CUtensorMap &tw, void *c, int M, int N,
                              int K, bool out_f32, const GemmEpi &epi, int num_sms,
                              unsigned *status, uint64_t timeout_ns, cudaStream_t s);
// table[p, i] = (cos, sin) of p theta^(-2i/d), evaluated as rope_kv_kernel does
cudaError_t launch_rope_table(float *table, int P, int d, double theta, int num_sms,
                              cudaStream_t s);
// wf[n, k] = round(W[n, k] * w[k])
cudaError_t launch_fold_norm_weight(const void *W, const void *w, void *wf, int64_t N, int64_t K,
                                    int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- backward
size_t rmsnorm_backward_ws_bytes(int64_t M, int64_t H);
cudaError_t launch_rmsnorm_backward(const void *x, const void *w, const void *dy, void *dx,
                                    void *dw, int64_t M, int64_t H, float eps, bool out_f32,
                                    void *ws, int num_sms, cudaStream_t s);
// out[c, r] = a[r, c] (bf16), rows of out padded with zeros to ld_out >= R
cudaError_t launch_transpose(const void *a, void *out, int64_t R, int64_t C, int64_t ld_out,
                             int num_sms, cudaStream_t s);
// dgu [T, 2F] = [dgate | dup] of out = silu(gate) * up for the upstream dout [T, F]
cudaError_t launch_swiglu_backward(const void *gu, const void *dout, void *dgu, int64_t T,
                                   int64_t F, bool out_f32, int num_sms, cudaStream_t s);
// dx = the transpose of the rotary rotation applied to dy ([T, nh, d] heads,
// rows ld_dy / ld_dx values apart)
cudaError_t launch_rope_backward(const void *dy, int64_t ld_dy, const int32_t *pos, void *dx,
                                 int64_t ld_dx, int64_t T, int nh, int d, double theta,
                                 bool out_f32, int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- KV write
cudaError_t launch_kv_write(void *k_cache, void *v_cache, int64_t num_pages, int Hkv, int d,
                            const void *k_new, const void *v_new, const int64_t *slots,
                            int64_t T, unsigned *status, cudaStream_t s);

// ---------------------------------------------------------------- attention
struct AttnParams {
    // cache (page blocks in core-matrix order, see include/bi.h)
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_table;
    int32_t max_pages;
    int32_t num_pages;
    int32_t Hkv;
    int32_t Hq;
    int32_t group;         // Hq / Hkv
    int32_t rows_per_q;    // decode: query rows per TMEM lane quarter
    // mode
    int32_t decode;        // 1 decode, 0 prefill
    int32_t B;
    const int32_t *seq_lens;   // decode
    const int32_t *order;      // decode: launch order of the sequences (or null)
    const int32_t *cu_q;       // prefill
    const int32_t *ctx_lens;   // prefill
    int32_t splits_per_cta;    // decode work division: splits per block (uniform) ...
    int32_t blocks_per_seq;    // ... or, if > 0, this many blocks per sequence, each of
                               // ceil(its splits / blocks_per_seq) splits
    int32_t max_splits;        // decode: splits of the longest sequence
    int32_t num_q_tiles;       // prefill: tiles of the longest chunk
    int32_t items;             // work items of the launch (set by launch_attention)
    float scale_log2;          // softmax scale * log2(e)
    // outputs
    void *o;
    float *lse;
    float *ws;                 // decode split partials
    unsigned *status;
    uint64_t timeout_ns;
};

size_t attn_smem_bytes(int head_dim);
size_t attn_ws_bytes(int B, int Hq, int head_dim, int max_splits, int max_chunks);
cudaError_t launch_attention(const CUtensorMap &tq, const AttnParams &p, int head_dim,
                             cudaStream_t s);
cudaError_t launch_attn_combine(const AttnParams &p, int head_dim, cudaStream_t s);
cudaError_t launch_attn_order(const int32_t *seq_lens, int B, int32_t *order, cudaStream_t s);

// ---------------------------------------------------------------- attention backward
struct AttnBwdParams {
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_table;
    int32_t max_pages;
    int32_t num_pages;
    int32_t Hkv;
    int32_t Hq;
    int32_t group;             // Hq / Hkv
    int32_t B;
    const int32_t *cu_q;       // [B + 1]
    const int32_t *ctx_lens;   // [B]
    int32_t num_q_tiles;       // 128-row tiles of the longest chunk
    int32_t num_key_blocks;    // 128-key blocks of the longest sequence
    float scale;               // softmax scale
    float scale_log2;          // scale * log2(e)
    const void *q, *o, *dout;  // [T, Hq, d] bf16
    const float *lse;          // [T, Hq] natural log
    float *lse2, *delta;       // workspace [T, Hq] each
    void *dq;                  // [T, Hq, d] bf16
    void *dk, *dv;             // cache-shaped bf16
    unsigned *status;
    uint64_t timeout_ns;
};
size_t attn_bwd_ws_bytes(int64_t rows);
// tq, tdo: 3D tensor maps (D, Hq, T) of q and dO, boxes of 64 x 1 x 128,
// 128-byte swizzle (the dK/dV kernel's tile loads).
cudaError_t launch_attention_backward(const CUtensorMap &tq, const CUtensorMap &tdo,
                                      const AttnBwdParams &p, int head_dim, int64_t rows,
                                      int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- decoder glue
cudaError_t launch_embedding(const void *table, int64_t V, int64_t H, const int32_t *ids,
                             void *out, int64_t T, unsigned *status, int num_sms, cudaStream_t s);
cudaError_t launch_rope_kv(const void *qkv, const int32_t *pos, const int64_t *slots,
                           void *q_out, void *k_cache, void *v_cache, int64_t num_pages, int Hq,
                           int Hkv, int d, double theta, int64_t T, unsigned *status, int num_sms,
                           cudaStream_t s);
cudaError_t launch_swiglu(const void *gu, void *out, int64_t T, int64_t F, int num_sms,
                          cudaStream_t s);
cudaError_t launch_argmax(const float *logits, int64_t T, int64_t V, int32_t *out, int num_sms,
                          cudaStream_t s);
constexpr int64_t kMaxSampleVocab = 53248;  // the row's weights live in shared memory
size_t sample_smem_bytes(int64_t V);
cudaError_t launch_sample(const float *logits, int64_t T, int64_t V, const float *temperature,
                          const float *top_p, const uint64_t *seed, const uint64_t *offset,
                          int32_t *out, int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- mixture of experts
constexpr int kMaxMoeExperts = 256;
constexpr int kMaxMoeTopK = 16;
cudaError_t launch_moe_route(const float *logits, int64_t T, int E, int k, int32_t *experts,
                             float *weights, int num_sms, cudaStream_t s);
cudaError_t launch_moe_dispatch(const int32_t *experts, int64_t N, int E, int k, int64_t *offsets,
                                int64_t *order, int64_t *pos, int32_t *token_sorted,
                                unsigned *status, cudaStream_t s);
cudaError_t launch_moe_combine(const void *y, const int64_t *pos, const float *weights, int64_t T,
                               int k, int64_t H, void *out, unsigned *status, int num_sms,
                               cudaStream_t s);

// ---------------------------------------------------------------- debug
cudaError_t launch_bounded_wait_probe(unsigned *status, uint64_t timeout_ns, cudaStream_t s);

}  // namespace bi
