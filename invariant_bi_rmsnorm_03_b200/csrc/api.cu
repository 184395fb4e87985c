// api.cu -- the C ABI declared in include/bi.h: argument checks, TMA
// descriptor encoding, launches and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "bi.h"
#include "bi_common.cuh"
#include "bi_launch.h"

// The per-device status word: first error recorded by any kernel.
__device__ unsigned g_bi_status;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool ready = false;
    unsigned *status = nullptr;
    int num_sms = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bi_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BI_OK : BI_ERR_CUDA; }

// Looks up the current device's status-word address and SM count (once).
bi_status device_state(DeviceState **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bi_status) != cudaSuccess) return BI_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BI_ERR_CUDA;
        d.status = static_cast<unsigned *>(p);
        d.num_sms = sms;
        d.ready = true;
    }
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                             cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return BI_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = &d;
    return BI_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// bf16 tensor map, 128-byte swizzle, zero fill out of bounds.  dims[0] is
// the contiguous dimension; strides are in bytes for dims 1.. .
bool encode(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
            const uint64_t *strides, const uint32_t *box)
{
    uint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                                const_cast<void *>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool kv_ok(const bi_paged_kv *kv)
{
    if (!kv || !kv->k_cache || !kv->v_cache || !kv->block_table) return false;
    if (kv->page_size != BI_PAGE_SIZE) return false;
    if (kv->num_kv_heads < 1 || kv->num_pages < 1 || kv->max_pages_per_seq < 1) return false;
    if (!aligned16(kv->k_cache) || !aligned16(kv->v_cache)) return false;
    // page ids and (page, head) block indices are 32-bit
    if (int64_t(kv->num_pages) * kv->num_kv_heads >= (int64_t(1) << 31)) return false;
    return true;
}

bool head_dim_ok(int d) { return d == 64 || d == 128; }

// Decode workspace: the launch order of the sequences (int32 [B], padded to
// 256 bytes), then the split partials when a sequence spans several blocks.
size_t order_bytes(int B) { return (size_t(B) * 4 + 255) / 256 * 256; }

int decode_splits_per_cta(int B, int Hkv, int max_splits, int requested, int num_sms)
{
    if (requested > 0) return requested < max_splits ? requested : max_splits;
    // Blocks per sequence: about one and a half waves of blocks over the SMs,
    // one wave when there are at most 8 (sequence, kv head) units.  Fewer
    // blocks pay fewer start-ups and leave fewer split records to merge (one
    // block per sequence needs no merge at all); more spread the longest
    // sequences.  Measured on lengths U(1, 32768), GQA 64/4: against two
    // waves, B = 1, 2 and 64 took 16%, 13% and 12% less time, B = 4 and 8
    // 3-4% less, B = 32 and 256 the same, B = 16 3% more.  The division never
    // changes a bit of the output.
    const int units = B * Hkv;
    const int twice = units <= 8 ? 2 : 3;  // twice the waves
    int k = (twice * num_sms + 2 * units - 1) / (2 * units);
    if (k < 1) k = 1;
    int c = (max_splits + k - 1) / k;
    return c < 1 ? 1 : c;
}

}  // namespace

extern "C" {

const char *bi_status_string(bi_status s)
{
    switch (s) {
    case BI_OK: return "ok";
    case BI_ERR_INVALID: return "invalid argument";
    case BI_ERR_UNSUPPORTED: return "unsupported configuration";
    case BI_ERR_CUDA: return "CUDA error";
    case BI_ERR_TIMEOUT: return "device-side wait timed out";
    case BI_ERR_WORKSPACE: return "workspace missing or too small";
    case BI_ERR_DEVICE_INDEX: return "device met an out-of-range page id or slot";
    }
    return "unknown status";
}

int bi_build_invariant(void) { return BI_INVARIANT ? 1 : 0; }

bi_status bi_rmsnorm(const void *x, const void *w, void *y, int64_t M, int64_t H, float eps,
                     bi_dtype out_dtype, void *stream)
{
    if (M < 0 || H < 8 || H % 8 != 0 || H > 65536) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BI_ERR_INVALID;
    if (M == 0) return BI_OK;
    if (!x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_rmsnorm(x, w, y, M, H, eps, out_dtype == BI_F32, d->num_sms,
                                        static_cast<cudaStream_t>(stream)));
}

static bi_status gemm_maps(const void *a, const void *w, int64_t M, int64_t N, int64_t K,
                           CUtensorMap *ta, CUtensorMap *tw)
{
    const uint64_t da[2] = {uint64_t(K), uint64_t(M)}, sa[1] = {uint64_t(K) * 2};
    const uint64_t dw[2] = {uint64_t(K), uint64_t(N)}, sw[1] = {uint64_t(K) * 2};
    // each CTA of a pair loads kGemmCtaRows rows of A and of W per K slice
    const uint32_t box[2] = {uint32_t(bi::kGemmBK), uint32_t(bi::kGemmCtaRows)};
    if (!encode(ta, a, 2, da, sa, box) || !encode(tw, w, 2, dw, sw, box)) return BI_ERR_CUDA;
    return BI_OK;
}

bi_status bi_matmul_grouped(const void *a, const void *w, void *c, const int64_t *offsets,
                            int32_t groups, int64_t rows, int64_t N, int64_t K, bi_dtype out_dtype,
                            void *stream)
{
    if (rows < 0 || N < 1 || K < 1 || N % 8 != 0 || K % 8 != 0) return BI_ERR_INVALID;
    if (groups < 1 || groups > bi::kMaxGemmGroups) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (rows > INT32_MAX || int64_t(groups) * N > INT32_MAX || K > INT32_MAX) return BI_ERR_INVALID;
    if (rows == 0) return BI_OK;
    if (!a || !w || !c || !offsets || !aligned16(a) || !aligned16(w) || !aligned16(c))
        return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    CUtensorMap ta, tw;
    if ((st = gemm_maps(a, w, rows, int64_t(groups) * N, K, &ta, &tw)) != BI_OK) return st;
    return from_cuda(bi::launch_gemm_grouped(ta, tw, c, int(rows), int(N), int(K),
                                             out_dtype == BI_F32, offsets, groups, d->num_sms,
                                             d->status, bi::kDefaultTimeoutNs,
                                             static_cast<cudaStream_t>(stream)));
}

static bool gemm_shape_ok(int64_t M, int64_t N, int64_t K)
{
    return M >= 0 && N >= 1 && K >= 1 && N % 8 == 0 && K % 8 == 0 && M <= INT32_MAX &&
           N <= INT32_MAX && K <= INT32_MAX;
}


bi_status bi_fold_norm_weight(const void *W, const void *w, void *wf, int64_t N, int64_t K,
                              void *stream)
{
    if (N < 0 || K < 8 || K % 8 != 0) return BI_ERR_INVALID;
    if (N == 0) return BI_OK;
    if (!W || !w || !wf || !aligned16(W) || !aligned16(w) || !aligned16(wf)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_fold_norm_weight(W, w, wf, N, K, d->num_sms,
                                                 static_cast<cudaStream_t>(stream)));
}

size_t bi_rmsnorm_matmul_workspace_bytes(int64_t M)
{
    return M > 0 ? (size_t(M) * sizeof(float) + 255) / 256 * 256 : 0;
}

bi_status bi_rmsnorm_matmul(const void *x, const void *wf, void *c, int64_t M, int64_t N,
                            int64_t K, float eps, bi_dtype out_dtype, void *ws, size_t ws_bytes,
                            void *stream)
{
    if (!gemm_shape_ok(M, N, K) || K > 65536) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BI_ERR_INVALID;
    if (M == 0) return BI_OK;
    if (!x || !wf || !c || !aligned16(x) || !aligned16(wf) || !aligned16(c)) return BI_ERR_INVALID;
    if (!ws || ws_bytes < bi_rmsnorm_matmul_workspace_bytes(M) || !aligned16(ws))
        return BI_ERR_WORKSPACE;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    CUtensorMap ta, tw;
    if ((st = gemm_maps(x, wf, M, N, K, &ta, &tw)) != BI_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *r = static_cast<float *>(ws);
    cudaError_t e = bi::launch_row_rstd(x, r, M, K, eps, d->num_sms, s);
    if (e != cudaSuccess) return from_cuda(e);
    bi::GemmEpi epi{};
    epi.rs = r;
    return from_cuda(bi::launch_gemm_fused(ta, tw, c, int(M), int(N), int(K), out_dtype == BI_F32,
                                           epi, d->num_sms, d->status, bi::kDefaultTimeoutNs, s));
}

bi_status bi_rope_table(float *table, int32_t max_pos, int32_t head_dim, float theta,
                        void *stream)
{
    if (max_pos < 1 || !head_dim_ok(head_dim)) return BI_ERR_INVALID;
    if (!(theta > 1.0f) || !std::isfinite(theta)) return BI_ERR_INVALID;
    if (!table || !aligned16(table)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_rope_table(table, max_pos, head_dim, double(theta), d->num_sms,
                                           static_cast<cudaStream_t>(stream)));
}

bi_status bi_rmsnorm_matmul_rope_kv(const void *x, const void *wf, float eps,
                                    const bi_paged_kv *kv, const float *rope_table,
                                    int32_t max_pos, const int32_t *positions,
                                    const int64_t *slot_mapping, void *q_out, int64_t T,
                                    int64_t K, int32_t Hq, void *ws, size_t ws_bytes,
                                    void *stream)
{
    if (!kv_ok(kv) || !head_dim_ok(kv->head_dim)) return BI_ERR_INVALID;
    if (Hq < 1 || Hq % kv->num_kv_heads != 0 || max_pos < 1) return BI_ERR_INVALID;
    const int64_t N = int64_t(Hq + 2 * kv->num_kv_heads) * kv->head_dim;
    if (!gemm_shape_ok(T, N, K) || K > 65536) return BI_ERR_INVALID;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!x || !wf || !rope_table || !positions || !slot_mapping || !q_out || !aligned16(x) ||
        !aligned16(wf) || !aligned16(rope_table) || !aligned16(q_out))
        return BI_ERR_INVALID;
    if (!ws || ws_bytes < bi_rmsnorm_matmul_workspace_bytes(T) || !aligned16(ws))
        return BI_ERR_WORKSPACE;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    CUtensorMap ta, tw;
    if ((st = gemm_maps(x, wf, T, N, K, &ta, &tw)) != BI_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *r = static_cast<float *>(ws);
    cudaError_t e = bi::launch_row_rstd(x, r, T, K, eps, d->num_sms, s);
    if (e != cudaSuccess) return from_cuda(e);
    bi::GemmEpi epi{};
    epi.rs = r;
    epi.rope = rope_table;
    epi.max_pos = max_pos;
    epi.pos = positions;
    epi.slots = slot_mapping;
    epi.q_out = q_out;
    epi.k_cache = kv->k_cache;
    epi.v_cache = kv->v_cache;
    epi.num_pages = kv->num_pages;
    epi.Hq = Hq;
    epi.Hkv = kv->num_kv_heads;
    epi.head_dim = kv->head_dim;
    return from_cuda(bi::launch_gemm_fused(ta, tw, nullptr, int(T), int(N), int(K), false, epi,
                                           d->num_sms, d->status, bi::kDefaultTimeoutNs, s));
}

bi_status bi_matmul_residual(const void *a, const void *w, const void *r, void *c, int64_t M,
                             int64_t N, int64_t K, void *stream)
{
    if (!gemm_shape_ok(M, N, K)) return BI_ERR_INVALID;
    if (M == 0) return BI_OK;
    if (!a || !w || !r || !c || !aligned16(a) || !aligned16(w) || !aligned16(r) || !aligned16(c))
        return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    CUtensorMap ta, tw;
    if ((st = gemm_maps(a, w, M, N, K, &ta, &tw)) != BI_OK) return st;
    bi::GemmEpi epi{};
    epi.residual = r;
    return from_cuda(bi::launch_gemm_fused(ta, tw, c, int(M), int(N), int(K), false, epi,
                                           d->num_sms, d->status, bi::kDefaultTimeoutNs,
                                           static_cast<cudaStream_t>(stream)));
}

size_t bi_rmsnorm_backward_workspace_bytes(int64_t M, int64_t H)
{
    if (M <= 0 || H <= 0) return 0;
    return bi::rmsnorm_backward_ws_bytes(M, H);
}

bi_status bi_rmsnorm_backward(const void *x, const void *w, const void *dy, void *dx, void *dw,
                              int64_t M, int64_t H, float eps, bi_dtype out_dtype, void *ws,
                              size_t ws_bytes, void *stream)
{
    if (M < 0 || H < 8 || H % 8 != 0 || H > 65536) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BI_ERR_INVALID;
    if (M == 0) return BI_OK;
    if (!x || !w || !dy || !dx || !dw || !aligned16(x) || !aligned16(w) || !aligned16(dy) ||
        !aligned16(dx) || !aligned16(dw))
        return BI_ERR_INVALID;
    if (!ws || ws_bytes < bi::rmsnorm_backward_ws_bytes(M, H) || !aligned16(ws))
        return BI_ERR_WORKSPACE;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_rmsnorm_backward(x, w, dy, dx, dw, M, H, eps, out_dtype == BI_F32,
                                                 ws, d->num_sms,
                                                 static_cast<cudaStream_t>(stream)));
}

bi_status bi_transpose(const void *a, void *out, int64_t R, int64_t C, int64_t ld_out,
                       void *stream)
{
    if (R < 0 || C < 0 || ld_out < R) return BI_ERR_INVALID;
    if (R == 0 || C == 0) return BI_OK;
    if (!a || !out) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_transpose(a, out, R, C, ld_out, d->num_sms,
                                          static_cast<cudaStream_t>(stream)));
}

namespace {
int64_t round8(int64_t v) { return (v + 7) / 8 * 8; }
size_t region(int64_t elems) { return (size_t(elems) * 2 + 255) / 256 * 256; }
}  // namespace

size_t bi_matmul_backward_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    const int64_t M8 = round8(M);
    return region(K * N) + region(N * M8) + region(K * M8);
}

bi_status bi_matmul_backward(const void *dc, const void *a, const void *w, void *da, void *dw,
                             int64_t M, int64_t N, int64_t K, bi_dtype out_dtype, void *ws,
                             size_t ws_bytes, void *stream)
{
    if (!gemm_shape_ok(M, N, K)) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (M == 0) return BI_OK;
    if (!dc || !a || !w || (!da && !dw)) return BI_ERR_INVALID;
    if (!aligned16(dc) || !aligned16(a) || !aligned16(w) || (da && !aligned16(da)) ||
        (dw && !aligned16(dw)))
        return BI_ERR_INVALID;
    const int64_t M8 = round8(M);
    if (M8 > INT32_MAX) return BI_ERR_INVALID;
    if (!ws || ws_bytes < bi_matmul_backward_workspace_bytes(M, N, K) || !aligned16(ws))
        return BI_ERR_WORKSPACE;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *base = static_cast<uint8_t *>(ws);
    void *wt = base;                                  // W^T  [K, N]
    void *dct = base + region(K * N);                 // dC^T [N, M8]
    void *at = base + region(K * N) + region(N * M8); // A^T  [K, M8]
    const bool f32 = out_dtype == BI_F32;
    cudaError_t e;
    if (da) {
        // dA [M, K] = dC [M, N] (W^T [K, N])^T
        if ((e = bi::launch_transpose(w, wt, N, K, N, d->num_sms, s)) != cudaSuccess)
            return from_cuda(e);
        CUtensorMap ta, tw;
        if ((st = gemm_maps(dc, wt, M, K, N, &ta, &tw)) != BI_OK) return st;
        if ((e = bi::launch_gemm(ta, tw, da, int(M), int(K), int(N), f32, nullptr, 1, d->num_sms,
                                 d->status, bi::kDefaultTimeoutNs, s)) != cudaSuccess)
            return from_cuda(e);
    }
    if (dw) {
        // dW [N, K] = dC^T [N, M8] (A^T [K, M8])^T; the zero columns past M add nothing
        if ((e = bi::launch_transpose(dc, dct, M, N, M8, d->num_sms, s)) != cudaSuccess)
            return from_cuda(e);
        if ((e = bi::launch_transpose(a, at, M, K, M8, d->num_sms, s)) != cudaSuccess)
            return from_cuda(e);
        CUtensorMap ta, tw;
        if ((st = gemm_maps(dct, at, N, K, M8, &ta, &tw)) != BI_OK) return st;
        if ((e = bi::launch_gemm(ta, tw, dw, int(N), int(K), int(M8), f32, nullptr, 1, d->num_sms,
                                 d->status, bi::kDefaultTimeoutNs, s)) != cudaSuccess)
            return from_cuda(e);
    }
    return BI_OK;
}

bi_status bi_swiglu_backward(const void *gu, const void *dout, void *dgu, int64_t T, int64_t F,
                             bi_dtype out_dtype, void *stream)
{
    if (T < 0 || F < 8 || F % 8 != 0) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!gu || !dout || !dgu || !aligned16(gu) || !aligned16(dout) || !aligned16(dgu))
        return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_swiglu_backward(gu, dout, dgu, T, F, out_dtype == BI_F32,
                                                d->num_sms, static_cast<cudaStream_t>(stream)));
}

bi_status bi_rope_backward(const void *dy, int64_t ld_dy, const int32_t *positions, void *dx,
                           int64_t ld_dx, int64_t T, int32_t num_heads, int32_t head_dim,
                           float theta, bi_dtype out_dtype, void *stream)
{
    if (T < 0 || num_heads < 1 || !head_dim_ok(head_dim)) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (!(theta > 1.0f) || !std::isfinite(theta)) return BI_ERR_INVALID;
    const int64_t row = int64_t(num_heads) * head_dim;
    if (ld_dy < row || ld_dx < row || ld_dy % 8 != 0 || ld_dx % 8 != 0) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!dy || !positions || !dx || !aligned16(dy) || !aligned16(dx)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_rope_backward(dy, ld_dy, positions, dx, ld_dx, T, num_heads,
                                              head_dim, double(theta), out_dtype == BI_F32,
                                              d->num_sms, static_cast<cudaStream_t>(stream)));
}

bi_status bi_add_rmsnorm(void *x, const void *delta, const void *w, void *y, int64_t M,
                         int64_t H, float eps, bi_dtype out_dtype, void *stream)
{
    if (M < 0 || H < 8 || H % 8 != 0 || H > 65536) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BI_ERR_INVALID;
    if (M == 0) return BI_OK;
    if (!x || !delta || !w || !y) return BI_ERR_INVALID;
    if (!aligned16(x) || !aligned16(delta) || !aligned16(w) || !aligned16(y)) return BI_ERR_INVALID;
    if (x == y || delta == y) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_add_rmsnorm(x, delta, w, y, M, H, eps, out_dtype == BI_F32,
                                            d->num_sms, static_cast<cudaStream_t>(stream)));
}

size_t bi_matmul_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    DeviceState *d;
    if (device_state(&d) != BI_OK) return 0;
    const int ks = bi::gemm_k_splits(M, N, K, d->num_sms);
    return ks > 1 ? size_t(ks) * M * N * sizeof(float) : 0;
}

bi_status bi_matmul(const void *a, const void *w, void *c, int64_t M, int64_t N, int64_t K,
                    bi_dtype out_dtype, void *ws, size_t ws_bytes, void *stream)
{
    if (M < 0 || N < 1 || K < 1 || N % 8 != 0 || K % 8 != 0) return BI_ERR_INVALID;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return BI_ERR_INVALID;
    if (out_dtype != BI_BF16 && out_dtype != BI_F32) return BI_ERR_INVALID;
    if (M == 0) return BI_OK;
    if (!a || !w || !c || !aligned16(a) || !aligned16(w) || !aligned16(c)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    const int ks = bi::gemm_k_splits(M, N, K, d->num_sms);
    if (ks > 1) {
        if (!ws || ws_bytes < size_t(ks) * M * N * sizeof(float) || !aligned16(ws))
            return BI_ERR_WORKSPACE;
    }
    CUtensorMap ta, tw;
    if ((st = gemm_maps(a, w, M, N, K, &ta, &tw)) != BI_OK) return st;
    return from_cuda(bi::launch_gemm(ta, tw, c, int(M), int(N), int(K), out_dtype == BI_F32,
                                     static_cast<float *>(ws), ks, d->num_sms, d->status,
                                     bi::kDefaultTimeoutNs, static_cast<cudaStream_t>(stream)));
}

bi_status bi_kv_write(const bi_paged_kv *kv, const void *k_new, const void *v_new,
                      const int64_t *slot_mapping, int64_t T, void *stream)
{
    if (!kv_ok(kv) || !head_dim_ok(kv->head_dim) || T < 0) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new))
        return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_kv_write(kv->k_cache, kv->v_cache, kv->num_pages, kv->num_kv_heads,
                                         kv->head_dim, k_new, v_new, slot_mapping, T, d->status,
                                         static_cast<cudaStream_t>(stream)));
}

bi_status bi_embedding(const void *table, int64_t V, int64_t H, const int32_t *ids, void *out,
                       int64_t T, void *stream)
{
    if (V < 1 || H < 8 || H % 8 != 0 || T < 0) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!table || !ids || !out || !aligned16(table) || !aligned16(out)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_embedding(table, V, H, ids, out, T, d->status, d->num_sms,
                                          static_cast<cudaStream_t>(stream)));
}

bi_status bi_rope_kv_write(const bi_paged_kv *kv, const void *qkv, const int32_t *positions,
                           const int64_t *slot_mapping, void *q_out, int64_t T, int32_t Hq,
                           float theta, void *stream)
{
    if (!kv_ok(kv) || !head_dim_ok(kv->head_dim) || T < 0) return BI_ERR_INVALID;
    if (Hq < 1 || Hq % kv->num_kv_heads != 0) return BI_ERR_INVALID;
    if (!(theta > 1.0f) || !std::isfinite(theta)) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!qkv || !positions || !slot_mapping || !q_out || !aligned16(qkv) || !aligned16(q_out))
        return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_rope_kv(qkv, positions, slot_mapping, q_out, kv->k_cache,
                                        kv->v_cache, kv->num_pages, Hq, kv->num_kv_heads,
                                        kv->head_dim, double(theta), T, d->status, d->num_sms,
                                        static_cast<cudaStream_t>(stream)));
}

bi_status bi_swiglu(const void *gu, void *out, int64_t T, int64_t F, void *stream)
{
    if (T < 0 || F < 8 || F % 8 != 0) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!gu || !out || !aligned16(gu) || !aligned16(out)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_swiglu(gu, out, T, F, d->num_sms, static_cast<cudaStream_t>(stream)));
}

bi_status bi_argmax(const float *logits, int64_t T, int64_t V, int32_t *out, void *stream)
{
    if (T < 0 || V < 4 || V % 4 != 0 || V > INT32_MAX) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!logits || !out || !aligned16(logits)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_argmax(logits, T, V, out, d->num_sms, static_cast<cudaStream_t>(stream)));
}

bi_status bi_sample(const float *logits, int64_t T, int64_t V, const float *temperature,
                    const float *top_p, const uint64_t *seed, const uint64_t *offset, int32_t *out,
                    void *stream)
{
    if (T < 0 || V < 1 || V > bi::kMaxSampleVocab) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!logits || !temperature || !top_p || !seed || !offset || !out) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_sample(logits, T, V, temperature, top_p, seed, offset, out,
                                       d->num_sms, static_cast<cudaStream_t>(stream)));
}

bi_status bi_moe_route(const float *logits, int64_t T, int32_t E, int32_t k, int32_t *experts,
                       float *weights, void *stream)
{
    if (T < 0 || E < 1 || E > bi::kMaxMoeExperts || k < 1 || k > bi::kMaxMoeTopK || k > E)
        return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!logits || !experts || !weights) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_moe_route(logits, T, E, k, experts, weights, d->num_sms,
                                          static_cast<cudaStream_t>(stream)));
}

bi_status bi_moe_dispatch(const int32_t *experts, int64_t T, int32_t k, int32_t E,
                          int64_t *offsets, int64_t *order, int64_t *pos, int32_t *token_sorted,
                          void *stream)
{
    if (T < 0 || E < 1 || E > bi::kMaxMoeExperts || k < 1 || k > bi::kMaxMoeTopK)
        return BI_ERR_INVALID;
    if (T > (int64_t(1) << 31) / k) return BI_ERR_INVALID;
    if (!offsets) return BI_ERR_INVALID;
    if (T > 0 && (!experts || !order || !pos || !token_sorted)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_moe_dispatch(experts, T * k, E, k, offsets, order, pos,
                                             token_sorted, d->status,
                                             static_cast<cudaStream_t>(stream)));
}

bi_status bi_moe_combine(const void *y, const int64_t *pos, const float *weights, int64_t T,
                         int32_t k, int64_t H, void *out, void *stream)
{
    if (T < 0 || k < 1 || k > bi::kMaxMoeTopK || H < 8 || H % 8 != 0) return BI_ERR_INVALID;
    if (T == 0) return BI_OK;
    if (!y || !pos || !weights || !out || !aligned16(y) || !aligned16(out)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_moe_combine(y, pos, weights, T, k, H, out, d->status, d->num_sms,
                                            static_cast<cudaStream_t>(stream)));
}

static bool attn_common_ok(const bi_paged_kv *kv, int32_t Hq)
{
    if (!kv_ok(kv)) return false;
    if (Hq < 1 || Hq % kv->num_kv_heads != 0) return false;
    if (Hq / kv->num_kv_heads > 128) return false;
    return true;
}

size_t bi_attention_decode_workspace_bytes(const bi_paged_kv *kv, int32_t B, int32_t Hq,
                                           int32_t max_seq_len, int32_t splits_per_cta)
{
    if (!kv || B < 1 || Hq < 1 || max_seq_len < 1 || kv->num_kv_heads < 1) return 0;
    DeviceState *d;
    if (device_state(&d) != BI_OK) return 0;
    const int max_splits = (max_seq_len + bi::kSplit - 1) / bi::kSplit;
    const int c = decode_splits_per_cta(B, kv->num_kv_heads, max_splits, splits_per_cta, d->num_sms);
    const int chunks = (max_splits + c - 1) / c;
    return order_bytes(B) + bi::attn_ws_bytes(B, Hq, kv->head_dim, max_splits, chunks);
}

// Argument checks shared by both decode entry points.
static bi_status decode_args_ok(const bi_paged_kv *kv, const void *q, const void *o,
                                const int32_t *seq_lens, int32_t B, int32_t Hq,
                                int32_t max_seq_len, float scale, int32_t splits_per_cta)
{
    if (!attn_common_ok(kv, Hq)) return BI_ERR_INVALID;
    if (!head_dim_ok(kv->head_dim)) return BI_ERR_UNSUPPORTED;
    if (B < 0 || max_seq_len < 1 || splits_per_cta < 0 || !std::isfinite(scale))
        return BI_ERR_INVALID;
    if (int64_t(max_seq_len) > int64_t(kv->max_pages_per_seq) * BI_PAGE_SIZE) return BI_ERR_INVALID;
    if (B == 0) return BI_OK;
    if (B > 65535) return BI_ERR_UNSUPPORTED;
    if (!q || !o || !seq_lens || !aligned16(q) || !aligned16(o)) return BI_ERR_INVALID;
    return BI_OK;
}

// The launches of one decode call, given its scratch: `order` (int32 [B],
// the launch order of the sequences) and, when a sequence is split over
// several blocks (chunks > 1), `partials` (the fp32 split records).  Both
// decode entry points go through here, so they launch the same kernels with
// the same parameters and give the same bits.
static bi_status decode_launch(const DeviceState *d, const bi_paged_kv *kv, const void *q,
                               void *o, float *lse, const int32_t *seq_lens, int32_t B,
                               int32_t Hq, int max_splits, int splits_per_cta, int chunks,
                               bool per_sequence, float scale, int32_t *order, float *partials,
                               cudaStream_t s)
{
    const int D = kv->head_dim, Hkv = kv->num_kv_heads, group = Hq / Hkv;
    bi::AttnParams p{};
    p.k_cache = kv->k_cache;
    p.v_cache = kv->v_cache;
    p.block_table = kv->block_table;
    p.max_pages = kv->max_pages_per_seq;
    p.num_pages = kv->num_pages;
    p.Hkv = Hkv;
    p.Hq = Hq;
    p.group = group;
    p.rows_per_q = (group + 3) / 4;
    p.decode = 1;
    p.B = B;
    p.seq_lens = seq_lens;
    // The launch order only decides which blocks start first; when every
    // block of the launch fits in one wave (one block per SM) nothing waits,
    // so the sorting launch is skipped (the kernel reads a null order as the
    // identity).
    const int64_t items = int64_t(per_sequence ? chunks : (max_splits + splits_per_cta - 1) /
                                                              splits_per_cta) * Hkv * B;
    const bool sort = B > 1 && items > d->num_sms;
    p.order = sort ? order : nullptr;
    p.splits_per_cta = splits_per_cta;
    // a division chosen from the load cuts each sequence into `chunks`
    // blocks of its own length; an explicit one uses splits_per_cta for all
    p.blocks_per_seq = per_sequence ? chunks : 0;
    p.max_splits = max_splits;
    p.scale_log2 = float(double(scale) * 1.4426950408889634);
    p.o = o;
    p.lse = lse;
    p.ws = partials;
    p.status = d->status;
    p.timeout_ns = bi::kDefaultTimeoutNs;

    CUtensorMap tq;
    const uint64_t dq[3] = {uint64_t(D), uint64_t(Hq), uint64_t(B)};
    const uint64_t sq[2] = {uint64_t(D) * 2, uint64_t(Hq) * D * 2};
    const uint32_t bq[3] = {64, uint32_t(p.rows_per_q), 1};
    if (!encode(&tq, q, 3, dq, sq, bq)) return BI_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    if (sort) {
        e = bi::launch_attn_order(seq_lens, B, order, s);
        if (e != cudaSuccess) return BI_ERR_CUDA;
    }
    e = bi::launch_attention(tq, p, D, s);
    if (e != cudaSuccess) return BI_ERR_CUDA;
    if (chunks > 1) e = bi::launch_attn_combine(p, D, s);
    return from_cuda(e);
}

bi_status bi_attention_decode(const bi_paged_kv *kv, const void *q, void *o, float *lse,
                              const int32_t *seq_lens, int32_t B, int32_t Hq,
                              int32_t max_seq_len, float scale, int32_t splits_per_cta,
                              void *ws, size_t ws_bytes, void *stream)
{
    bi_status st = decode_args_ok(kv, q, o, seq_lens, B, Hq, max_seq_len, scale, splits_per_cta);
    if (st != BI_OK || B == 0) return st;
    DeviceState *d;
    if ((st = device_state(&d)) != BI_OK) return st;

    const int max_splits = (max_seq_len + bi::kSplit - 1) / bi::kSplit;
    const int c = decode_splits_per_cta(B, kv->num_kv_heads, max_splits, splits_per_cta, d->num_sms);
    const int chunks = (max_splits + c - 1) / c;
    const size_t need = order_bytes(B) + bi::attn_ws_bytes(B, Hq, kv->head_dim, max_splits, chunks);
    if (!ws || ws_bytes < need || !aligned16(ws)) return BI_ERR_WORKSPACE;
    int32_t *order = static_cast<int32_t *>(ws);
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + order_bytes(B));
    return decode_launch(d, kv, q, o, lse, seq_lens, B, Hq, max_splits, c, chunks,
                         splits_per_cta == 0, scale, order, partials,
                         static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- no-alloc decode
//
// bi_attention_decode_noalloc: the same decode attention for callers that
// cannot allocate device memory.  Its scratch (the launch order of the
// sequences and the split partials) is this fixed array, which every GPU
// that loads the library holds until the process exits.
static __device__ __align__(256) uint8_t g_decode_scratch[BI_NOALLOC_SCRATCH_BYTES];

// The launch order of the largest batch always fits beside some partials.
static_assert(((65535 * 4 + 255) / 256) * 256 < BI_NOALLOC_SCRATCH_BYTES,
              "the launch order of 65535 sequences fits in the scratch array");

static std::mutex g_scratch_mu;
static void *g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device.  (In host code the array's name is a host-side stand-in, not a
// device address, so it is never handed to a kernel directly.)
static bi_status decode_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr)
            return BI_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return BI_OK;
}

bi_status bi_attention_decode_noalloc(const bi_paged_kv *kv, const void *q, void *o, float *lse,
                                      const int32_t *seq_lens, int32_t B, int32_t Hq,
                                      int32_t max_seq_len, float scale, int32_t splits_per_cta,
                                      void *stream)
{
    bi_status st = decode_args_ok(kv, q, o, seq_lens, B, Hq, max_seq_len, scale, splits_per_cta);
    if (st != BI_OK || B == 0) return st;
    DeviceState *d;
    if ((st = device_state(&d)) != BI_OK) return st;
    void *scratch = nullptr;
    if ((st = decode_scratch(&scratch)) != BI_OK) return st;

    const int max_splits = (max_seq_len + bi::kSplit - 1) / bi::kSplit;
    int c = decode_splits_per_cta(B, kv->num_kv_heads, max_splits, splits_per_cta, d->num_sms);
    int chunks = (max_splits + c - 1) / c;
    size_t need = order_bytes(B) + bi::attn_ws_bytes(B, Hq, kv->head_dim, max_splits, chunks);
    if (need > BI_NOALLOC_SCRATCH_BYTES && splits_per_cta == 0) {
        // The work division chosen from the load would need more partials
        // than the array holds: give each sequence one block instead (the
        // output bits do not depend on the division).
        c = max_splits;
        chunks = 1;
        need = order_bytes(B);
    }
    if (need > BI_NOALLOC_SCRATCH_BYTES) return BI_ERR_WORKSPACE;
    int32_t *order = static_cast<int32_t *>(scratch);
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + order_bytes(B));
    return decode_launch(d, kv, q, o, lse, seq_lens, B, Hq, max_splits, c, chunks,
                         splits_per_cta == 0, scale, order, partials,
                         static_cast<cudaStream_t>(stream));
}

size_t bi_attention_prefill_workspace_bytes(const bi_paged_kv *kv, int32_t B, int32_t Hq,
                                            int32_t max_q_len)
{
    (void)kv, (void)B, (void)Hq, (void)max_q_len;
    return 0;
}

bi_status bi_attention_prefill(const bi_paged_kv *kv, const void *q, void *o, float *lse,
                               const int32_t *cu_q, const int32_t *ctx_lens, int32_t B,
                               int32_t Hq, int64_t T_total, int32_t max_q_len, float scale,
                               void *ws, size_t ws_bytes, void *stream)
{
    (void)ws, (void)ws_bytes;
    if (!attn_common_ok(kv, Hq)) return BI_ERR_INVALID;
    if (!head_dim_ok(kv->head_dim)) return BI_ERR_UNSUPPORTED;
    if (B < 0 || T_total < 0 || max_q_len < 0 || !std::isfinite(scale)) return BI_ERR_INVALID;
    if (T_total > INT32_MAX) return BI_ERR_UNSUPPORTED;
    if (B == 0 || T_total == 0 || max_q_len == 0) return BI_OK;
    if (B > 65535 || Hq > 65535) return BI_ERR_UNSUPPORTED;
    if (!q || !o || !cu_q || !ctx_lens || !aligned16(q) || !aligned16(o)) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;

    const int D = kv->head_dim, Hkv = kv->num_kv_heads;
    bi::AttnParams p{};
    p.k_cache = kv->k_cache;
    p.v_cache = kv->v_cache;
    p.block_table = kv->block_table;
    p.max_pages = kv->max_pages_per_seq;
    p.num_pages = kv->num_pages;
    p.Hkv = Hkv;
    p.Hq = Hq;
    p.group = Hq / Hkv;
    p.rows_per_q = 32;
    p.decode = 0;
    p.B = B;
    p.cu_q = cu_q;
    p.ctx_lens = ctx_lens;
    p.num_q_tiles = (max_q_len + 127) / 128;
    p.scale_log2 = float(double(scale) * 1.4426950408889634);
    p.o = o;
    p.lse = lse;
    p.status = d->status;
    p.timeout_ns = bi::kDefaultTimeoutNs;

    CUtensorMap tq;
    const uint64_t dq[3] = {uint64_t(D), uint64_t(Hq), uint64_t(T_total)};
    const uint64_t sq[2] = {uint64_t(D) * 2, uint64_t(Hq) * D * 2};
    const uint32_t bq[3] = {64, 1, 128};
    if (!encode(&tq, q, 3, dq, sq, bq)) return BI_ERR_CUDA;
    return from_cuda(bi::launch_attention(tq, p, D, static_cast<cudaStream_t>(stream)));
}

size_t bi_attention_backward_workspace_bytes(int32_t Hq, int64_t T_total)
{
    if (Hq < 1 || T_total < 1) return 0;
    return bi::attn_bwd_ws_bytes(int64_t(Hq) * T_total);
}

bi_status bi_attention_backward(const bi_paged_kv *kv, const void *q, const void *o,
                                const void *dout, const float *lse, const int32_t *cu_q,
                                const int32_t *ctx_lens, int32_t B, int32_t Hq, int64_t T_total,
                                int32_t max_q_len, int32_t max_kv_len, float scale, void *dq,
                                void *dk_cache, void *dv_cache, void *ws, size_t ws_bytes,
                                void *stream)
{
    if (!attn_common_ok(kv, Hq)) return BI_ERR_INVALID;
    if (!head_dim_ok(kv->head_dim)) return BI_ERR_UNSUPPORTED;
    if (B < 0 || T_total < 0 || max_q_len < 0 || max_kv_len < 0 || !std::isfinite(scale))
        return BI_ERR_INVALID;
    if (int64_t(max_kv_len) > int64_t(kv->max_pages_per_seq) * BI_PAGE_SIZE) return BI_ERR_INVALID;
    if (T_total > INT32_MAX) return BI_ERR_UNSUPPORTED;
    if (B == 0 || T_total == 0 || max_q_len == 0) return BI_OK;
    if (max_kv_len < max_q_len) return BI_ERR_INVALID;
    if (B > 65535) return BI_ERR_UNSUPPORTED;
    if (!q || !o || !dout || !lse || !cu_q || !ctx_lens || !dq || !dk_cache || !dv_cache)
        return BI_ERR_INVALID;
    if (!aligned16(q) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk_cache) || !aligned16(dv_cache))
        return BI_ERR_INVALID;
    if (dk_cache == kv->k_cache || dk_cache == kv->v_cache || dv_cache == kv->k_cache ||
        dv_cache == kv->v_cache || dk_cache == dv_cache)
        return BI_ERR_INVALID;
    const int64_t rows = T_total * Hq;
    if (!ws || ws_bytes < bi::attn_bwd_ws_bytes(rows) || !aligned16(ws)) return BI_ERR_WORKSPACE;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;

    bi::AttnBwdParams p{};
    p.k_cache = kv->k_cache;
    p.v_cache = kv->v_cache;
    p.block_table = kv->block_table;
    p.max_pages = kv->max_pages_per_seq;
    p.num_pages = kv->num_pages;
    p.Hkv = kv->num_kv_heads;
    p.Hq = Hq;
    p.group = Hq / kv->num_kv_heads;
    p.B = B;
    p.cu_q = cu_q;
    p.ctx_lens = ctx_lens;
    p.num_q_tiles = (max_q_len + 127) / 128;
    p.num_key_blocks = (max_kv_len + 127) / 128;
    p.scale = scale;
    p.scale_log2 = float(double(scale) * 1.4426950408889634);
    p.q = q;
    p.o = o;
    p.dout = dout;
    p.lse = lse;
    p.lse2 = static_cast<float *>(ws);
    p.delta = static_cast<float *>(ws) + rows;
    p.dq = dq;
    p.dk = dk_cache;
    p.dv = dv_cache;
    p.status = d->status;
    p.timeout_ns = bi::kDefaultTimeoutNs;
    CUtensorMap tq, tdo;
    const int D = kv->head_dim;
    const uint64_t dq3[3] = {uint64_t(D), uint64_t(Hq), uint64_t(T_total)};
    const uint64_t sq3[2] = {uint64_t(D) * 2, uint64_t(Hq) * D * 2};
    const uint32_t bq3[3] = {64, 1, 128};
    if (!encode(&tq, q, 3, dq3, sq3, bq3) || !encode(&tdo, dout, 3, dq3, sq3, bq3))
        return BI_ERR_CUDA;
    return from_cuda(bi::launch_attention_backward(tq, tdo, p, kv->head_dim, rows, d->num_sms,
                                                   static_cast<cudaStream_t>(stream)));
}

bi_status bi_device_status(void *stream)
{
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return BI_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, d->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return BI_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(d->status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
            return BI_ERR_CUDA;
    }
    switch (v) {
    case 0: return BI_OK;
    case bi::BI_DEV_TIMEOUT: return BI_ERR_TIMEOUT;
    case bi::BI_DEV_BAD_INDEX: return BI_ERR_DEVICE_INDEX;
    default: return BI_ERR_CUDA;
    }
}

bi_status bi_debug_bounded_wait(uint64_t timeout_ns, void *stream)
{
    if (timeout_ns < 1000 || timeout_ns > 1000000000ull) return BI_ERR_INVALID;
    DeviceState *d;
    bi_status st = device_state(&d);
    if (st != BI_OK) return st;
    return from_cuda(bi::launch_bounded_wait_probe(d->status, timeout_ns,
                                                   static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
