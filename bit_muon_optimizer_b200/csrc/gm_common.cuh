// Internal helpers shared by the libgmuon translation units (not installed).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/gmuon.h"

namespace gm {

constexpr int kGrid = GM_GRID_BLOCK;   // 128 x 128 grid-quant blocks
constexpr int kMaxK = GM_MAX_K;

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline long long cdivll(long long a, long long b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- dtypes
__device__ __forceinline__ float load_as_float(const void* p, long long idx, int dt) {
  if (dt == GM_F32) return static_cast<const float*>(p)[idx];
  if (dt == GM_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[idx]);
  return __half2float(static_cast<const __half*>(p)[idx]);
}

// 16-bit float bits <-> float, for operands stored as raw uint16 (bf16 or f16)
__device__ __forceinline__ float h16_to_float(uint16_t v, bool f16) {
  if (f16) return __half2float(__ushort_as_half(v));
  return __bfloat162float(__ushort_as_bfloat16(v));
}
__device__ __forceinline__ uint16_t float_to_h16(float v, bool f16) {
  if (f16) return __half_as_ushort(__float2half_rn(v));
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ void store_from_float(void* p, long long idx, int dt, float v) {
  if (dt == GM_F32) static_cast<float*>(p)[idx] = v;
  else if (dt == GM_BF16) static_cast<__nv_bfloat16*>(p)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(p)[idx] = __float2half_rn(v);
}

// Four consecutive elements from fp32 values (idx a multiple of 4, aligned).
__device__ __forceinline__ void store4_from_float(void* p, long long idx, int dt, float4 v) {
  if (dt == GM_F32) {
    *reinterpret_cast<float4*>(static_cast<float*>(p) + idx) = v;
  } else {
    const bool f16 = dt == GM_F16;
    uint2 w;
    w.x = (uint32_t)float_to_h16(v.x, f16) | ((uint32_t)float_to_h16(v.y, f16) << 16);
    w.y = (uint32_t)float_to_h16(v.z, f16) | ((uint32_t)float_to_h16(v.w, f16) << 16);
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p) + idx) = w;
  }
}

// ----------------------------------------------------- splitmix64 (Steele et al.)
__host__ __device__ inline uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// ------------------------------------------------- per-device one-time set-up
// Kernel attributes and looked-up device addresses belong to a device (its
// primary context), so every cache of them is keyed by the current device.
constexpr int kMaxDevices = 64;

// SM count of the current device (cached per device; 148 if the query fails).
inline int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Runs `fn` once per device (the current one when called), thread-safe; a
// failed `fn` is retried on the next call.
class DeviceOnce {
 public:
  template <typename F>
  cudaError_t run(F&& fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const uint64_t bit = 1ull << dev;
    if (done_.load(std::memory_order_acquire) & bit) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_.load(std::memory_order_relaxed) & bit) return cudaSuccess;
    e = fn();
    if (e == cudaSuccess) done_.fetch_or(bit, std::memory_order_release);
    return e;
  }

 private:
  std::mutex mu_;
  std::atomic<uint64_t> done_{0};
};

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes) once per device.
template <typename K>
cudaError_t smem_attr_once(DeviceOnce& once, K kernel, size_t bytes) {
  return once.run([&] {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  });
}

// --------------------------------------------------------------- errors
// Host-side error bookkeeping lives in gm_api.cu.
gm_status set_error(gm_status s, const char* fmt, ...);

}  // namespace gm
