// Shared device helpers: the device status word, bf16 conversion and the
// paged-cache row resolver used by every kernel that touches the pool.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mla_b200.h"

namespace mla {

// First device-side fault since the last mla_get_device_error() call.
__device__ int g_device_status;

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_device_status, 0, code);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t v) {
    return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return static_cast<uint32_t>(f32_to_bf16(lo)) | (static_cast<uint32_t>(f32_to_bf16(hi)) << 16);
}

// Pool row of token t of sequence b:
//   block_table[b][t / block_size] * block_size + t % block_size
// (the page walk of a paged latent cache). Returns -1 if b is outside
// [0, num_seqs), the page index is outside the table row or the block id is
// outside [0, num_blocks).
__device__ __forceinline__ int64_t resolve_row(const int32_t* __restrict__ block_table, int32_t num_seqs,
                                               int32_t max_blocks_per_seq, int64_t num_blocks,
                                               int32_t block_size, int32_t b, int32_t t) {
    if (t < 0 || b < 0 || b >= num_seqs) return -1;
    const int32_t page = t / block_size;
    if (page >= max_blocks_per_seq) return -1;
    const int32_t blk = __ldg(block_table + static_cast<int64_t>(b) * max_blocks_per_seq + page);
    if (blk < 0 || blk >= num_blocks) return -1;
    return static_cast<int64_t>(blk) * block_size + (t - page * block_size);
}

// Programmatic dependent launch: every kernel of the library is launched
// with programmatic stream serialization, so the next kernel in the stream may
// start (launch, set up shared memory, barriers and tensor memory) while this
// one finishes. pdl_wait() blocks until the preceding grid has completed and
// its memory is visible; every kernel calls it before its first global access
// of data another kernel produces or consumes (so the chain of waits also
// orders it after all earlier work). pdl_trigger() lets the next kernel launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

}  // namespace mla
