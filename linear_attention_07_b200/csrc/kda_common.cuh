// Shared device/host helpers of libkda.so (no method arithmetic here).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "../../include/kda.h"

namespace kda {

// Counts every kernel launch made by the library (kda_launch_count()).
void note_launches(int n);

// Kernel attributes (the dynamic shared-memory limit) and memory-pool
// settings apply to one device only, so one-time setup is kept per device
// ordinal.  The setup calls are idempotent: two host threads that race on a
// device's first call may both run them, which is harmless.
constexpr int MAX_DEVICES = 64;
using DeviceFlags = std::atomic<bool>[MAX_DEVICES];

// Runs setup(device) on the current device unless it has already succeeded
// there; returns its error, or cudaSuccess.
template <typename F>
cudaError_t once_per_device(DeviceFlags& done, F&& setup)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool tracked = dev >= 0 && dev < MAX_DEVICES;
    if (tracked && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = setup(dev);
    if (e == cudaSuccess && tracked) done[dev].store(true, std::memory_order_release);
    return e;
}

// Number of SMs of the current device (queried once per device); 0 if the
// query fails.
int current_sm_count();

// Keep freed stream-ordered workspace in the current device's default pool
// between calls (release threshold: never), once per device, so that a call
// does not map its workspace anew every time.
void keep_pool_memory();
// Limit of every bounded device-side wait: 2 s, or KDA_WAIT_LIMIT_NS
// (0 .. 2e9 ns) for tests that make the waits run out.
uint64_t bounded_wait_limit_ns();

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace kda
