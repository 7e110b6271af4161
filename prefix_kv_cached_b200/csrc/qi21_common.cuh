// Device helpers shared by every kernel family (storage conversion, reductions).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qi21 {

typedef __nv_bfloat16 bf16;

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

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

// Sum over the block; `red` holds >= 32 floats of shared memory. All threads
// receive the total.
__device__ __forceinline__ float block_sum(float v, float *red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : 0.f;
    t = warp_sum(t);
    return t;
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

// Programmatic dependent launch. A kernel launched with the programmatic
// stream-serialisation attribute may be scheduled while the kernel before it in
// the stream is still running; pdl_wait() returns once every preceding kernel
// has completed and its memory is visible, so a kernel calls it before its
// first global-memory access (after any prologue that touches only its own
// shared memory, TMEM and kernel parameters). pdl_launch_dependents() allows
// the next kernel to be scheduled. Both are no-ops in a normal launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Error word in the workspace: kernels set a code and return instead of
// trapping; the host reads it with qi21_check_device_error.
enum : uint32_t { DEV_ERR_NONE = 0, DEV_ERR_TIMEOUT = 1, DEV_ERR_LAYOUT = 2 };

__device__ __forceinline__ void raise_device_error(uint32_t *err, uint32_t code) {
    if (err) atomicCAS(err, 0u, code);
}

}  // namespace qi21
