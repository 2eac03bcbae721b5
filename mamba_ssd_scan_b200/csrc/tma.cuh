// tma.cuh -- tensor-memory-accelerator (TMA) loads: the host builds a tiled
// tensor map (cuTensorMapEncodeTiled, reached through the runtime's driver
// entry point so the library does not link libcuda) and one thread per CTA
// issues cp.async.bulk.tensor loads that complete on an mbarrier (and bulk
// stores tracked by bulk async groups).  Never with cluster multicast.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// 4-D bf16 tensor [d3][d2][d1][d0] (d0 innermost, dense), a box of
// {64, box1, box2, 1} elements with the 128-byte swizzle: it lands in shared
// memory as box1 * box2 128-byte rows in the SW128 layout.  Elements outside
// the tensor read as zero.  Returns false if the encoder is unavailable or
// rejects the arguments.
bool make_tmap_bf16_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                       uint64_t d2, uint64_t d3, uint32_t box1, uint32_t box2);
// A 2-D fp32 tensor [d1][d0] (d0 innermost, a multiple of 4 elements) read or
// written in boxes of {32, box1} elements with the 128-byte swizzle: box1
// 128-byte rows in the SW128 layout.
bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint32_t box1);

namespace tc {

__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :
                 : "r"(mbar), "r"(bytes)
                 : "memory");
}

// One box of a 4-D tensor map into shared memory; completes `bytes` on mbar.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t mbar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar), "r"(c0), "r"(c1), "r"(c2),
          "r"(c3)
        : "memory");
}

// One box from shared memory to a 4-D tensor in global memory (bulk async
// group of the issuing thread; elements outside the tensor are not written).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
        :
        : "l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
// One box from shared memory to a 2-D tensor in global memory (bulk async
// group of the issuing thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 :
                 : "l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
// One contiguous run of `bytes` from global into shared memory (both
// addresses 16-byte aligned, bytes a multiple of 16); completes `bytes` on
// mbar.  A plain bulk copy, never multicast.
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes,
                                             uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :
        : "r"(dst), "l"(src), "r"(bytes), "r"(mbar)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until the bulk groups of this thread have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until the bulk groups of this thread have completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Bring one box of a 4-D tensor map into L2 only (no shared memory, no
// completion signal), so a later tma_load_4d of the same box hits L2.
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* map, int c0, int c1, int c2,
                                                   int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];"
                 :
                 : "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" : : "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

}  // namespace tc
}  // namespace ssd
