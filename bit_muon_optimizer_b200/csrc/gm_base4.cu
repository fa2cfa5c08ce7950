// The 4bit-Muon-base codec: blockwise 4-bit quantization of the whole
// momentum matrix, the direct quantization of Muon's state that the GRASP
// note ("Achieving low-bit Muon through subspace preservation and grid
// quantization") measures its own codec against.
//
// Layout: groups of 128 consecutive row-major elements, one absmax scale each.
// m and n are multiples of 16, so m n is a multiple of 256: no group is ragged
// or straddles two matrices of the batch, and the batch is one flat run of
// B m n / 128 groups.
//
// Both passes are HBM-bound (4.53 B per element in total): one warp owns one
// group at a time, lane l holds its elements 4l .. 4l + 3 as one float4, so a
// warp moves the group's 512 bytes in one coalesced request and its 64 code
// bytes as 32 two-byte stores. A grid of eight CTAs per SM walks the groups.

#include <math.h>

#include "gm_common.cuh"
#include "gm_internal.h"

namespace gm {
namespace {

constexpr int kGroup = 128;
constexpr int kB4Threads = 256;
constexpr int kB4Warps = kB4Threads / 32;
constexpr int kB4MaxBlocks = 8 * 148;

// q = clamp(rint(fp32(x / s) * 7), -7, 7) for |x| <= s, as a nibble. The
// product z = x * fl(7 / s) differs from fl(x / s) * 7 by a few units in the
// last place, so away from a rounding tie (|z - rint(z)| < 0.5 - 2^-16) both
// round alike; near one the IEEE division decides.
__device__ __forceinline__ uint32_t code4(float x, float s, float r7) {
  const float z = __fmul_rn(x, r7), zr = rintf(z);
  int q;
  if (fabsf(__fsub_rn(z, zr)) < 0.49998474f)   // 0.5 - 2^-16
    q = (int)zr;
  else
    q = (int)rintf(__fmul_rn(__fdiv_rn(x, s), 7.0f));
  q = max(-7, min(7, q));
  return (uint32_t)q & 0xFu;
}

__global__ void __launch_bounds__(kB4Threads) k_group_quant4(long long ngroups,
                                                              const float* __restrict__ X,
                                                              uint8_t* __restrict__ codes4,
                                                              float* __restrict__ gscale) {
  const int lane = threadIdx.x & 31;
  const long long stride = (long long)gridDim.x * kB4Warps;
  for (long long g = (long long)blockIdx.x * kB4Warps + (threadIdx.x >> 5); g < ngroups;
       g += stride) {
    const float4 v = reinterpret_cast<const float4*>(X)[g * 32 + lane];
    // |x| as unsigned bits orders like the values, and a NaN (above every
    // other pattern) carries into the scale: its group then keeps code 0
    const uint32_t a = max(max(__float_as_uint(fabsf(v.x)), __float_as_uint(fabsf(v.y))),
                           max(__float_as_uint(fabsf(v.z)), __float_as_uint(fabsf(v.w))));
    const float s = __uint_as_float(__reduce_max_sync(0xffffffffu, a));
    uint32_t w = 0;
    if (s > 0.f) {
      const float r7 = __fdiv_rn(7.0f, s);
      // element 4 lane + e sits in nibble e: low nibble = even column
      w = code4(v.x, s, r7) | (code4(v.y, s, r7) << 4) | (code4(v.z, s, r7) << 8) |
          (code4(v.w, s, r7) << 12);
    }
    reinterpret_cast<uint16_t*>(codes4)[g * 32 + lane] = (uint16_t)w;
    if (lane == 0) gscale[g] = s;
  }
}

__global__ void __launch_bounds__(kB4Threads) k_group_dequant4(long long ngroups,
                                                                const uint8_t* __restrict__ codes4,
                                                                const float* __restrict__ gscale,
                                                                float* __restrict__ X) {
  __shared__ float deq[16];   // fl(q / 7) for the nibble q (two's complement)
  if (threadIdx.x < 16)
    deq[threadIdx.x] = __fdiv_rn((float)((threadIdx.x & 8) ? (int)threadIdx.x - 16 : (int)threadIdx.x),
                                 7.0f);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long long stride = (long long)gridDim.x * kB4Warps;
  for (long long g = (long long)blockIdx.x * kB4Warps + (threadIdx.x >> 5); g < ngroups;
       g += stride) {
    const float s = gscale[g];
    const uint32_t w = reinterpret_cast<const uint16_t*>(codes4)[g * 32 + lane];
    float4 o;
    o.x = __fmul_rn(deq[w & 0xF], s);
    o.y = __fmul_rn(deq[(w >> 4) & 0xF], s);
    o.z = __fmul_rn(deq[(w >> 8) & 0xF], s);
    o.w = __fmul_rn(deq[(w >> 12) & 0xF], s);
    reinterpret_cast<float4*>(X)[g * 32 + lane] = o;
  }
}

int base4_blocks(long long ngroups) {
  return (int)max(1LL, min((long long)kB4MaxBlocks, cdivll(ngroups, kB4Warps)));
}

// ---------------------------------------------------------------- mu-law codec
// MuonQ's mu-law companding, read as: each group of 128 consecutive elements is
// normalised by its absmax s, companded by F(y) = sign(y) ln(1 + mu |y|) /
// ln(1 + mu) and coded q = clamp(rint(7 F(x / s)), -7, 7). Since F is
// increasing, |q| >= j exactly when |x| / s >= t_j = F^-1((j - 1/2) / 7), so
// the code needs no logarithm per element: the seven thresholds t_j come from
// the host in fp64, each lane scales them by its group's s (fp64) and rounds
// up to fp32, and since |x| is an fp32 value, |x| >= fl_up(t_j s) decides what
// |x| / s >= t_j does unless t_j s lies within fp64 rounding of an fp32 value.
// Decoding multiplies the fp32 level F^-1(|q| / 7) (also from the host) by s.
struct MulawTables {
  double t[7];   // t[j - 1] = F^-1((j - 1/2) / 7), j = 1..7
  float level[8];   // level[j] = F^-1(j / 7), j = 0..7
};

__device__ __forceinline__ uint32_t mulaw_code(float x, const float (&T)[7]) {
  const float a = fabsf(x);
  int q = 0;
#pragma unroll
  for (int j = 0; j < 7; ++j) q += a >= T[j] ? 1 : 0;
  if (x < 0.f) q = -q;
  return (uint32_t)q & 0xFu;
}

__global__ void __launch_bounds__(kB4Threads) k_mulaw_quant4(long long ngroups, MulawTables tab,
                                                              const float* __restrict__ X,
                                                              uint8_t* __restrict__ codes4,
                                                              float* __restrict__ gscale) {
  const int lane = threadIdx.x & 31;
  const long long stride = (long long)gridDim.x * kB4Warps;
  for (long long g = (long long)blockIdx.x * kB4Warps + (threadIdx.x >> 5); g < ngroups;
       g += stride) {
    const float4 v = reinterpret_cast<const float4*>(X)[g * 32 + lane];
    const uint32_t a = max(max(__float_as_uint(fabsf(v.x)), __float_as_uint(fabsf(v.y))),
                           max(__float_as_uint(fabsf(v.z)), __float_as_uint(fabsf(v.w))));
    const float s = __uint_as_float(__reduce_max_sync(0xffffffffu, a));
    uint32_t w = 0;
    if (s > 0.f) {   // false for s = 0 and for a NaN scale: codes 0
      float T[7];
#pragma unroll
      for (int j = 0; j < 7; ++j) T[j] = __double2float_ru(tab.t[j] * (double)s);
      w = mulaw_code(v.x, T) | (mulaw_code(v.y, T) << 4) | (mulaw_code(v.z, T) << 8) |
          (mulaw_code(v.w, T) << 12);
    }
    reinterpret_cast<uint16_t*>(codes4)[g * 32 + lane] = (uint16_t)w;
    if (lane == 0) gscale[g] = s;
  }
}

__global__ void __launch_bounds__(kB4Threads) k_mulaw_dequant4(long long ngroups, MulawTables tab,
                                                                const uint8_t* __restrict__ codes4,
                                                                const float* __restrict__ gscale,
                                                                float* __restrict__ X) {
  __shared__ float deq[16];   // the signed level of nibble q (two's complement)
  if (threadIdx.x < 16) {
    const int q = (threadIdx.x & 8) ? (int)threadIdx.x - 16 : (int)threadIdx.x;
    const float l = tab.level[q < 0 ? (q < -7 ? 7 : -q) : q];
    deq[threadIdx.x] = q < 0 ? -l : l;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long long stride = (long long)gridDim.x * kB4Warps;
  for (long long g = (long long)blockIdx.x * kB4Warps + (threadIdx.x >> 5); g < ngroups;
       g += stride) {
    const float s = gscale[g];
    const uint32_t w = reinterpret_cast<const uint16_t*>(codes4)[g * 32 + lane];
    float4 o;
    o.x = __fmul_rn(deq[w & 0xF], s);
    o.y = __fmul_rn(deq[(w >> 4) & 0xF], s);
    o.z = __fmul_rn(deq[(w >> 8) & 0xF], s);
    o.w = __fmul_rn(deq[(w >> 12) & 0xF], s);
    reinterpret_cast<float4*>(X)[g * 32 + lane] = o;
  }
}

// The thresholds and levels of F for this mu, from the definition in fp64:
// F^-1(z) = ((1 + mu)^z - 1) / mu = expm1(z ln(1 + mu)) / mu.
MulawTables mulaw_tables(float mu) {
  MulawTables tab;
  const double lm = log1p((double)mu);
  for (int j = 1; j <= 7; ++j) tab.t[j - 1] = expm1((j - 0.5) / 7.0 * lm) / (double)mu;
  for (int j = 0; j <= 7; ++j) tab.level[j] = j == 7 ? 1.0f : (float)(expm1(j / 7.0 * lm) / (double)mu);
  return tab;
}

}  // namespace

cudaError_t launch_mulaw_quant4(int B, int m, int n, float mu, const float* X, uint8_t* codes4,
                                float* gscale, cudaStream_t s) {
  const long long ngroups = (long long)B * m * n / kGroup;
  k_mulaw_quant4<<<base4_blocks(ngroups), kB4Threads, 0, s>>>(ngroups, mulaw_tables(mu), X, codes4,
                                                              gscale);
  return cudaGetLastError();
}

cudaError_t launch_mulaw_dequant4(int B, int m, int n, float mu, const uint8_t* codes4,
                                  const float* gscale, float* X, cudaStream_t s) {
  const long long ngroups = (long long)B * m * n / kGroup;
  k_mulaw_dequant4<<<base4_blocks(ngroups), kB4Threads, 0, s>>>(ngroups, mulaw_tables(mu), codes4,
                                                                gscale, X);
  return cudaGetLastError();
}

cudaError_t launch_group_quant4(int B, int m, int n, const float* X, uint8_t* codes4,
                                float* gscale, cudaStream_t s) {
  const long long ngroups = (long long)B * m * n / kGroup;
  k_group_quant4<<<base4_blocks(ngroups), kB4Threads, 0, s>>>(ngroups, X, codes4, gscale);
  return cudaGetLastError();
}

cudaError_t launch_group_dequant4(int B, int m, int n, const uint8_t* codes4, const float* gscale,
                                  float* X, cudaStream_t s) {
  const long long ngroups = (long long)B * m * n / kGroup;
  k_group_dequant4<<<base4_blocks(ngroups), kB4Threads, 0, s>>>(ngroups, codes4, gscale, X);
  return cudaGetLastError();
}

}  // namespace gm
