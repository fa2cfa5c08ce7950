// The weight update of the GRASP step on its own: W <- W - eta (O + wd W) from
// an orthogonalized update O that is already in memory ("Achieving low-bit Muon
// through subspace preservation and grid quantization", worked step 6, last
// line). The step's own path fuses this update into the epilogue of its last
// Newton-Schulz product; this pass serves callers that move O between devices
// first (a data-parallel set split by ownership exchanges the 16-bit O, half
// the bytes of the fp32 weights, and every rank then applies the same update
// to its copy of W).
//
// k_put_status hands a batch's device status (the step's skip flag) to the ranks
// that receive its O, one int32 per matrix.
//
// HBM-bound: W read and written (8 B per element) and O read (2 or 4 B). Each
// thread moves one float4 of W and the matching four values of O per trip; the
// grid's y index is the matrix, so a matrix that its skip flag marks keeps its
// weights without a single load.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gm_common.cuh"
#include "gm_internal.h"

namespace gm {
namespace {

constexpr int kUpdThreads = 256;

template <int ODT>
__device__ __forceinline__ void load_o4(const void* O, long long i, float (&o)[4]) {
  if constexpr (ODT == GM_F32) {
    const float4 v = reinterpret_cast<const float4*>(O)[i];
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  } else {
    const uint2 v = reinterpret_cast<const uint2*>(O)[i];
    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint16_t lo = (uint16_t)(w[h] & 0xFFFFu), hi = (uint16_t)(w[h] >> 16);
      if constexpr (ODT == GM_BF16) {
        o[2 * h] = __uint_as_float((uint32_t)lo << 16);
        o[2 * h + 1] = __uint_as_float((uint32_t)hi << 16);
      } else {
        o[2 * h] = __half2float(__ushort_as_half(lo));
        o[2 * h + 1] = __half2float(__ushort_as_half(hi));
      }
    }
  }
}

template <int ODT>
__global__ void __launch_bounds__(kUpdThreads) k_weight_update(long long per4, float eta, float wd,
                                                               const void* __restrict__ O,
                                                               float* __restrict__ W,
                                                               const int32_t* __restrict__ skip,
                                                               int skip_stride) {
  const int b = blockIdx.y;
  if (skip && skip[(long long)b * skip_stride]) return;
  const long long base = (long long)b * per4;
  for (long long i = (long long)blockIdx.x * kUpdThreads + threadIdx.x; i < per4;
       i += (long long)gridDim.x * kUpdThreads) {
    float4 w = reinterpret_cast<float4*>(W)[base + i];
    float o[4];
    load_o4<ODT>(O, base + i, o);
    w.x -= eta * (o[0] + wd * w.x);
    w.y -= eta * (o[1] + wd * w.y);
    w.z -= eta * (o[2] + wd * w.z);
    w.w -= eta * (o[3] + wd * w.w);
    reinterpret_cast<float4*>(W)[base + i] = w;
  }
}

struct PeerFlags {
  int32_t* flag[kMaxPeers];
};

// Every destination's flag of every matrix of the batch gets the batch's status.
__global__ void k_put_status(int B, int npeers, const __grid_constant__ PeerFlags pf,
                             const int64_t* __restrict__ dst_index, const int32_t* __restrict__ status) {
  const int32_t v = *status;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const long long at = dst_index ? dst_index[b] : b;
#pragma unroll
    for (int r = 0; r < kMaxPeers; ++r)
      if (r < npeers) pf.flag[r][at] = v;
  }
}

}  // namespace

cudaError_t launch_put_status(int B, int npeers, int32_t* const* flags, const int64_t* dst_index,
                              const int32_t* status, cudaStream_t s) {
  if (npeers < 1 || npeers > kMaxPeers) return cudaErrorInvalidValue;
  PeerFlags pf{};
  for (int r = 0; r < npeers; ++r) pf.flag[r] = flags[r];
  k_put_status<<<1, 256, 0, s>>>(B, npeers, pf, dst_index, status);
  return cudaGetLastError();
}

cudaError_t launch_weight_update(int B, int m, int n, float eta, float wd, const void* O, int odt,
                                 float* W, const int32_t* skip, int skip_stride, cudaStream_t s) {
  const long long per4 = (long long)m * n / 4;   // m, n multiples of 16
  // about eight CTAs of 256 threads per SM over the whole batch
  const long long want = (8LL * sm_count() + B - 1) / B;
  const int gx = (int)max(1LL, min(want, (per4 + kUpdThreads - 1) / kUpdThreads));
  const dim3 grid(gx, B);
  switch (odt) {
    case GM_F32:
      k_weight_update<GM_F32><<<grid, kUpdThreads, 0, s>>>(per4, eta, wd, O, W, skip, skip_stride);
      break;
    case GM_BF16:
      k_weight_update<GM_BF16><<<grid, kUpdThreads, 0, s>>>(per4, eta, wd, O, W, skip, skip_stride);
      break;
    case GM_F16:
      k_weight_update<GM_F16><<<grid, kUpdThreads, 0, s>>>(per4, eta, wd, O, W, skip, skip_stride);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace gm
