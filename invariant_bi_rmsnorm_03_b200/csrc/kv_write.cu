// kv_write.cu -- write the step's new keys and values into the paged cache
// before attention launches (neican.ai insight, "技术原理与创新点解析",
// batch-invariant attention bullet: the KV-cache page table is updated
// before the kernel starts, so the kernel always sees one consistent
// layout).
//
// Cache layout: page blocks [num_pages, Hkv] of 16 x d bf16, each block in
// core-matrix order [2 key groups][d/8 value groups][8 keys][8 values] (the
// order the attention kernel's tensor-core operands use, so a block is
// copied to shared memory as it is).  Token t of the step with slot
// s = slot_mapping[t] lands at page s / 16, key s % 16 for every kv head.
// One thread moves one 16-byte piece (8 values of one key); a bit copy, so
// trivially invariant.
//
// Also here: the probe kernel of the bounded-wait path (bi_debug_bounded_wait).
#include <cuda_runtime.h>

#include <cstdint>

#include "bi_common.cuh"
#include "bi_launch.h"
#include "bi_ptx.cuh"

namespace bi {
namespace {

__global__ void kv_write_kernel(uint4 *__restrict__ kc, uint4 *__restrict__ vc, int64_t num_pages,
                                int Hkv, int d, const uint4 *__restrict__ kn,
                                const uint4 *__restrict__ vn, const int64_t *__restrict__ slots,
                                int64_t T, unsigned *status)
{
    const int pieces = d >> 3;  // 16-byte pieces per (token, head)
    const int64_t total = T * Hkv * pieces;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int piece = static_cast<int>(i % pieces);
        const int64_t th = i / pieces;
        const int g = static_cast<int>(th % Hkv);
        const int64_t t = th / Hkv;
        const int64_t slot = slots[t];
        if (slot < 0) continue;
        if (slot >= num_pages * kPage) {
            if (piece == 0 && g == 0) record_status(status, BI_DEV_BAD_INDEX);
            continue;
        }
        const int64_t page = slot / kPage;
        const int off = static_cast<int>(slot % kPage);
        // page block in core-matrix order: [key group][value group][8 keys][8 values]
        const int64_t dst = (page * Hkv + g) * (kPage * pieces) + (off >> 3) * (8 * pieces) +
                            piece * 8 + (off & 7);
        kc[dst] = kn[i];
        vc[dst] = vn[i];
    }
}

// One block whose thread 0 waits on a barrier that nothing arrives at.
__global__ void bounded_wait_probe_kernel(unsigned *status, uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitCtl ctl{&abort_flag, status, timeout_ns};
        (void)wait(&bar, 0, ctl);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_kv_write(void *k_cache, void *v_cache, int64_t num_pages, int Hkv, int d,
                            const void *k_new, const void *v_new, const int64_t *slots,
                            int64_t T, unsigned *status, cudaStream_t s)
{
    const int64_t total = T * Hkv * (d / 8);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (1 << 20)) blocks = 1 << 20;
    kv_write_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), num_pages, Hkv, d,
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slots, T, status);
    return cudaGetLastError();
}

cudaError_t launch_bounded_wait_probe(unsigned *status, uint64_t timeout_ns, cudaStream_t s)
{
    bounded_wait_probe_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace bi
