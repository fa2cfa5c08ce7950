// Codec and power-iteration kernels of the GRASP step (CUDA cores, HBM bound).
//
// Step order follows "Achieving low-bit Muon through subspace preservation
// and grid quantization", worked step 1-5:
//   S1 rebuild + momentum  -> M (fp32), |M|^2 tile partials, non-finite flag
//   S2 warm start          -> Q = column-normalised R_{t-1} (or Rademacher)
//   S3 projection          -> P~ = M Q (fp32 chunks, fp64 accumulation)
//   S4 orthonormalisation  -> P = P~ L^-T  (fp64 Cholesky of P~^T P~)
//   S5 back-projection     -> R = M^T P, plus the normalised NS input X
//   S6 8-bit quant of P, R; S7 residual M - P R^T -> 4-bit grid codes
// Every reduction runs in a fixed order, so results are bit-reproducible.
// Quantization decisions use IEEE fp32 division and round-half-to-even.

#include <math.h>

#include "gm_common.cuh"
#include "gm_internal.h"

namespace gm {

namespace {

constexpr int kThreads = 256;
constexpr int kTargetCtas = 2 * 148;   // two waves' worth of CTAs on a B200


__device__ __forceinline__ float deq8(int8_t q, float s) {
  return __fmul_rn(__fdiv_rn((float)q, 127.0f), s);
}


__device__ __forceinline__ double block_sum_d(double v, double* red) {
  const int t = threadIdx.x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((t & 31) == 0) red[t >> 5] = v;
  __syncthreads();
  double s = 0.0;
  if (t == 0)
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
  __syncthreads();
  return s;   // valid in thread 0
}

// ------------------------------------------------- warp tensor-core helpers
// The rank-k contractions of the codec passes (at most 32 deep) run as
// warp-level mma.sync: too shallow for the tcgen05 pipeline to pay, and on the
// FMA pipe they made these HBM-bound passes issue-bound. Fragment layouts follow
// the PTX ISA for mma.m16n8k8 .tf32 and mma.m16n8k16 .bf16 (row.col): lane =
// 4 g + t; A holds rows g and g + 8, B column g, C/D rows g and g + 8 at
// columns 2 t and 2 t + 1.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// x = hi + lo + rest, |rest| <= 2^-22 |x|: hi keeps the top 11 significant bits
// (a tf32 by truncation, exact), lo is the remainder rounded to tf32. Products
// of two such pairs summed as lo*hi + hi*lo + hi*hi reach fp32-level accuracy
// (the 3xTF32 emulation); the small terms go first.
__device__ __forceinline__ uint32_t tf32_hi(float x) { return __float_as_uint(x) & 0xFFFFE000u; }
// The remainder's rounding to tf32 is round-to-nearest with ties away from zero on
// the magnitude (the rna rounding of the tf32 conversion): adding half of the last
// kept bit to the sign-magnitude pattern and clearing the 13 dropped bits gives it
// for every finite value (a carry out of the mantissa rounds up into the next
// binade), in two integer operations where the conversion instruction costs about four.
__device__ __forceinline__ uint32_t tf32_lo(float x, uint32_t hi) {
  return (__float_as_uint(__fsub_rn(x, __uint_as_float(hi))) + 0x1000u) & 0xFFFFE000u;
}

// x = p0 + p1 + p2 with every part a bf16: exact for normal fp32 (3 x 8
// significant bits). Two values per word, the first in the low half.
__device__ __forceinline__ void bf16_split3(float x, float y, uint32_t (&w)[3]) {
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    w[p] = *reinterpret_cast<const uint32_t*>(&h);
    x = __fsub_rn(x, __low2float(h));
    y = __fsub_rn(y, __high2float(h));
  }
}

// 16-byte asynchronous global -> shared copies (zero-filled when !valid; the
// source address is then not read).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Copy `bytes` (a multiple of 16, both ends 16-byte aligned) from global to
// shared memory with all threads of the block; the copies stay in flight.
__device__ __forceinline__ void cp_async_block(void* smem, const void* gmem, int bytes) {
  for (int c = threadIdx.x; c < (bytes >> 4); c += blockDim.x)
    cp_async16(static_cast<uint8_t*>(smem) + 16 * c, static_cast<const uint8_t*>(gmem) + 16 * c, true);
}

// As above, zero-filling the bytes at and beyond `valid`.
__device__ __forceinline__ void cp_async_block_zf(void* smem, const void* gmem, int bytes, int valid) {
  for (int c = threadIdx.x; c < (bytes >> 4); c += blockDim.x) {
    const bool ok = 16 * c < valid;
    cp_async16(static_cast<uint8_t*>(smem) + 16 * c,
               ok ? static_cast<const uint8_t*>(gmem) + 16 * c : gmem, ok);
  }
}


__host__ __device__ constexpr int kb16(int KP) { return KP < 16 ? 16 : KP; }

// ---------------------------------------------- fragment-ordered factor copies
// The rank-k factors are small (rows x k), so each is laid out once per step in
// the order the warps' MMA fragments read it; a CTA then copies its slice into
// shared memory with cp.async, as is. kp = factor_width(k), nl = kp / 8,
// ksb = max(kp, 16) / 16, nsl = ceil(n / 64) column slabs; padding is zero.
//   QF [B][nsl][8 s][nl][32][4]    Q hi, lo: B operand of the projection
//   RF [B][nsl][8 nt][ksb][32][2]  R codes as bf16: B operand of the rebuild
//   PF [B][m/16][ksb][3][32][4]    P codes x c_l, three bf16 parts: its A operand
//   PA [B][m/16][nl][2][32][4]     -P hi, lo: A operand of the residual
//   RB [B][nsl][8 nt][nl][32][4]   R hi, lo: B operand of the residual
//   PB [B][m/8][nl][32][4]         P hi, lo: B operand of the back-projection
// Column j of a slab sits in n-tile ((j & 15) >> 1) at fragment column
// 2 (j >> 4 & 3) + (j & 1) for the rebuild / residual, and at k-step
// ((j & 15) >> 1), k-slot (j >> 4 & 3) (+4 when j is odd) for the projection.
__device__ __forceinline__ long long qf_at(int b, int nsl, int nl, int j, int l) {   // + 0/1 hi, + 2/3 lo
  const int slab = j >> 6, jj = j & 63;
  return ((((long long)(b * nsl + slab) * 8 + ((jj & 15) >> 1)) * nl + (l >> 3)) * 32 + 4 * (l & 7) +
          (jj >> 4)) * 4 + (jj & 1);
}
__device__ __forceinline__ long long rf_at16(int b, int nsl, int ksb, int j, int l) {   // 16-bit index
  const int slab = j >> 6, jj = j & 63, ll = l & 15;
  return (((((long long)(b * nsl + slab) * 8 + ((jj & 15) >> 1)) * ksb + (l >> 4)) * 32 +
           4 * (2 * (jj >> 4) + (jj & 1)) + ((ll >> 1) & 3)) * 2 + (ll >> 3)) * 2 + (ll & 1);
}
__device__ __forceinline__ long long pf_at16(int b, int m16, int ksb, int i, int l, int part) {
  const int r = i & 15, ll = l & 15;
  return (((((long long)(b * m16 + (i >> 4)) * ksb + (l >> 4)) * 3 + part) * 32 + 4 * (r & 7) +
           ((ll >> 1) & 3)) * 4 + (r >> 3) + 2 * (ll >> 3)) * 2 + (ll & 1);
}
__device__ __forceinline__ long long pa_at(int b, int m16, int nl, int i, int l) {   // + 128 lo
  const int r = i & 15, ll = l & 7;
  return (((((long long)(b * m16 + (i >> 4)) * nl + (l >> 3)) * 2) * 32 + 4 * (r & 7) + (ll & 3)) * 4 +
          (r >> 3) + 2 * (ll >> 2));
}
__device__ __forceinline__ long long rb_at(int b, int nsl, int nl, int j, int l) {   // + 2 lo
  const int slab = j >> 6, jj = j & 63, ll = l & 7;
  return ((((long long)(b * nsl + slab) * 8 + ((jj & 15) >> 1)) * nl + (l >> 3)) * 32 +
          4 * (2 * (jj >> 4) + (jj & 1)) + (ll & 3)) * 4 + (ll >> 2);
}
__device__ __forceinline__ uint16_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

// ------------------------------------------------------------------ S2
__global__ void __launch_bounds__(kThreads) k_warm_start(int n, int k, const int8_t* R8,
                                                          const float* Rscale, const float* Rprev,
                                                          uint64_t seed, const int64_t* ids,
                                                          float* Q, uint32_t* QF,
                                                          const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.x, t = threadIdx.x;
  const uint64_t bid = ids ? (uint64_t)ids[b] : (uint64_t)b;   // the matrix's counter index
  const long long off = (long long)b * n * k;
  __shared__ double red[kThreads];
  __shared__ double nrm2[kMaxK];
  auto rhat = [&](int j, int l) -> float {
    if (Rprev) return Rprev[off + (long long)j * k + l];
    if (R8) return deq8(R8[off + (long long)j * k + l], Rscale[(long long)b * k + l]);
    return 0.0f;
  };
  const int groups = kThreads / k;
  double acc = 0.0;
  if (t < groups * k) {
    const int l = t % k, g = t / k;
    for (int j = g; j < n; j += groups) {
      const double v = rhat(j, l);
      acc += v * v;
    }
  }
  red[t] = acc;
  __syncthreads();
  if (t < k) {
    double s = 0.0;
    for (int g = 0; g < groups; ++g) s += red[g * k + t];
    nrm2[t] = s > 0.0 ? 1.0 / sqrt(s) : 0.0;   // inverse column norm; 0 marks a zero column
  }
  __syncthreads();
  const float rad = (float)(1.0 / sqrt((double)n));
  const int kp = factor_width(k), nsl = cdiv(n, 64);
  for (long long e = t; e < (long long)nsl * 64 * kp; e += kThreads) {
    const int j = (int)(e / kp), l = (int)(e % kp);
    float q = 0.f;
    if (j < n && l < k) {
      const double inv = nrm2[l];
      if (inv == 0.0) {
        const uint64_t ctr = seed ^ (bid << 48) ^ ((uint64_t)j << 16) ^ (uint64_t)l;
        q = (splitmix64(ctr) >> 63) ? -rad : rad;
      } else {
        q = (float)((double)rhat(j, l) * inv);
      }
      Q[off + (long long)j * k + l] = q;
    }
    if (QF) {
      const long long at = qf_at(b, nsl, kp / 8, j, l);
      const uint32_t hi = tf32_hi(q);
      QF[at] = hi;
      QF[at + 2] = tf32_lo(q, hi);
    }
  }
}

// S2 on the stored 8-bit state. Q[:, l] = R^[:, l] / |R^[:, l]| with
// R^[:, l] = (r8[:, l] / 127) s_l equals sign(s_l) r8[:, l] / |r8[:, l]|, so the
// column norms are exact integer sums of squared codes. Integer atomics make the
// sum independent of the order the CTAs arrive in. A zero code column or a zero
// scale gives the Rademacher column.
__global__ void __launch_bounds__(kThreads) k_colnorm_int(int n, int k, const int8_t* __restrict__ R8,
                                                           int* __restrict__ norm2,
                                                           const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y, t = threadIdx.x;
  __shared__ int red[kThreads];
  const int groups = kThreads / k;
  const int j0 = blockIdx.x * kThreads;
  const int j1 = min(n, j0 + kThreads);
  int acc = 0;
  if (t < groups * k) {
    const int l = t % k, g = t / k;
    for (int j = j0 + g; j < j1; j += groups) {
      const int v = R8[((long long)b * n + j) * k + l];
      acc += v * v;
    }
  }
  red[t] = acc;
  __syncthreads();
  if (t < k) {
    int s = 0;
    for (int g = 0; g < groups; ++g) s += red[g * k + t];
    if (s) atomicAdd(&norm2[b * k + t], s);
  }
}

// Blocks [0, nbq) cover the nsl * 64 x kb elements of Q and R: Q, its fragments
// QF and the R code fragments RF; blocks [nbq, ..) the m x kb elements of P:
// the P code fragments PF (c_l = Pscale_l Rscale_l / 127^2).
__global__ void __launch_bounds__(kThreads) k_warm_q(int m, int n, int k, int nbq,
                                                      const int8_t* __restrict__ R8,
                                                      const float* __restrict__ Rscale,
                                                      const int8_t* __restrict__ P8,
                                                      const float* __restrict__ Pscale,
                                                      const int* __restrict__ norm2, uint64_t seed,
                                                      const int64_t* __restrict__ ids,
                                                      float* __restrict__ Q, uint32_t* __restrict__ QF,
                                                      uint16_t* __restrict__ RF, uint16_t* __restrict__ PF,
                                                      const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y, t = threadIdx.x;
  const int kp = factor_width(k), kb = kb16(kp), nsl = cdiv(n, 64);
  __shared__ double inv[kMaxK];
  __shared__ float cf[kMaxK];
  if (t < k) {
    const int s2 = norm2[b * k + t];
    const float sc = Rscale[b * k + t];
    inv[t] = (s2 > 0 && sc != 0.f) ? (sc > 0.f ? 1.0 : -1.0) / sqrt((double)s2) : 0.0;
    cf[t] = __fdiv_rn(__fmul_rn(Pscale[b * k + t], sc), 16129.0f);
  }
  __syncthreads();
  if ((int)blockIdx.x < nbq) {
    const float rad = (float)(1.0 / sqrt((double)n));
    const long long base = (long long)blockIdx.x * kThreads * 4;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long e = base + u * kThreads + t;
      if (e >= (long long)nsl * 64 * kb) break;
      const int j = (int)(e / kb), l = (int)(e % kb);
      const bool valid = j < n && l < k;
      const float rq = valid ? (float)R8[((long long)b * n + j) * k + l] : 0.f;
      if (l < kp) {
        float q = 0.f;
        if (valid) {
          const double iv = inv[l];
          if (iv == 0.0) {
            const uint64_t bid = ids ? (uint64_t)ids[b] : (uint64_t)b;
            const uint64_t ctr = seed ^ (bid << 48) ^ ((uint64_t)j << 16) ^ (uint64_t)l;
            q = (splitmix64(ctr) >> 63) ? -rad : rad;
          } else {
            q = (float)((double)rq * iv);
          }
          Q[((long long)b * n + j) * k + l] = q;
        }
        const long long at = qf_at(b, nsl, kp / 8, j, l);
        const uint32_t hi = tf32_hi(q);
        QF[at] = hi;
        QF[at + 2] = tf32_lo(q, hi);
      }
      RF[rf_at16(b, nsl, kb / 16, j, l)] = bf16_bits(rq);
    }
  } else {
    const long long base = (long long)(blockIdx.x - nbq) * kThreads * 4;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long e = base + u * kThreads + t;
      if (e >= (long long)m * kb) break;
      const int i = (int)(e / kb), l = (int)(e % kb);
      float x = l < k ? __fmul_rn((float)P8[((long long)b * m + i) * k + l], cf[l]) : 0.f;
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const uint16_t h = bf16_bits(x);
        PF[pf_at16(b, m >> 4, kb / 16, i, l, part)] = h;
        x = __fsub_rn(x, __bfloat162float(__ushort_as_bfloat16(h)));
      }
    }
  }
}

// ------------------------------------------------------------------ S1 + S3
// Rebuild + momentum, fused with the projection P~ = M Q (k_rebuild_pipe below).
// Tile: 64 rows x 128 columns (half a grid block), 8 warps, two CTAs per SM.
// Warp w owns the rows 16 (w & 3) .. + 15 and the 64-column slab w >> 2; lane
// (g, t) the rows g and g + 8 of the warp's 16 and the 16 consecutive columns
// 16 t .. 16 t + 15 of the slab, so its loads and stores are whole 16-column runs.
// Column 16 t + 2 s + e of the slab is column 2 t + e of n-tile s in the C
// fragments, which makes
//   * the rank-k rebuild P^ R^T eight n-tiles of bf16 mma.m16n8k16 with
//     A = the 8-bit P codes times c_l = Pscale_l Rscale_l / 127^2, split into
//     three bf16 parts (exact), and B = the R codes (exact in bf16);
//   * the projection a tf32 mma.m16n8k8 whose A operand is M read straight from
//     those fragments (k-step s = slab columns 16 t + 2 s + {0, 1} of every t)
//     and whose B is Q, both split hi + lo (3xTF32).
// The decoded nibble value q / 7 comes from a 16-entry table filled with IEEE
// divisions, so it is bit-identical to (float)q / 7.0f. No block-wide reduction is
// needed per tile: the two warps of the same rows (one per 64-column slab) add
// their P~ partials through shared memory (a named barrier of the pair) and the
// slab-0 warp writes the sum over the 128-column block to Ppart[b][bj][row][l];
// each warp writes |M|^2 over its 16 x 64 part to norm2_part[b][row tile][column
// block][warp]; the orthonormalisation sums them in fp64 in a fixed order.
constexpr int kRB = 64;     // rows per rebuild tile

// Named barrier of the two warps (one per 64-column slab) that own row block rb
// of a rebuild tile (barriers 1..4; 0 is the block-wide one).
__device__ __forceinline__ void pair_sync(int rb) {
  switch (rb) {
    case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
    case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
    case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
    default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
  }
}
constexpr int kRBT = 256;  // threads per rebuild CTA

enum RebuildSrc { SRC_STATE = 0, SRC_DENSE = 1, SRC_ZERO = 2 };

// The rebuild alone (the rebuild-only entry point: M_{t-1} from the stored
// state, no gradient, no step workspace): one tile per CTA, the factors' MMA
// fragments built in the CTA from the raw codes, which are copied to shared
// memory with cp.async while the element loads are in flight.
__host__ __device__ constexpr int dequant_smem_words(int KP) {
  return 2 * 8 * (kb16(KP) / 16) * 32 * 2 + 4 * (kb16(KP) / 16) * 3 * 32 * 4 + (kGrid + kRB) * KP / 4;
}

template <int KP>   // the factor width k rounded up to 8, 16 or 32 (columns beyond k are zero)
__global__ void __launch_bounds__(kRBT, 2) k_dequant_rebuild(
    int m, int n, int k, const uint8_t* __restrict__ codes4, const float* __restrict__ rscale,
    const float* __restrict__ cscale, const int8_t* __restrict__ P8,
    const float* __restrict__ Pscale, const int8_t* __restrict__ R8,
    const float* __restrict__ Rscale, float* __restrict__ M) {
  constexpr int KSB = kb16(KP) / 16;
  const int bj = blockIdx.x, bi = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, tq = lane & 3, rb = warp & 3, slab = warp >> 2;
  const int r0 = bi * kRB, c0 = bj * kGrid;
  const int nrows = min(kRB, m - r0), ncols = min(kGrid, n - c0);   // multiples of 16
  extern __shared__ __align__(16) uint32_t smd[];
  uint32_t* RF = smd;                                                // [slab][nt][KSB][lane][2]
  uint32_t* PF = RF + 2 * 8 * KSB * 32 * 2;                          // [rb][KSB][part][lane][4]
  int8_t* R8raw = reinterpret_cast<int8_t*>(PF + 4 * KSB * 3 * 32 * 4);   // [128][k]
  int8_t* P8raw = R8raw + kGrid * KP;                                     // [64][k]
  __shared__ float deq4[16];
  __shared__ float cfac[32];
  const long long mn = (long long)m * n;
  const int cb = c0 + 64 * slab + 16 * tq;   // n % 16 == 0: the run is all in or all out
  const bool colok = cb < n;

  // 1. element loads (codes, scales), then the raw factors
  uint2 cw[2];
  float rsc[2], cs[16];
  bool ok[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int gi = r0 + 16 * rb + g + 8 * h;
    ok[h] = gi < m && colok;
    cw[h] = ok[h] ? *reinterpret_cast<const uint2*>(codes4 + ((long long)b * m + gi) * (n / 2) + cb / 2)
                  : make_uint2(0u, 0u);
    rsc[h] = gi < m ? rscale[((long long)b * m + gi) * nb + bj] : 0.f;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 v = colok ? *reinterpret_cast<const float4*>(cscale + ((long long)b * cdiv(m, kGrid) + r0 / kGrid) * n + cb + 4 * u)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    cs[4 * u] = v.x; cs[4 * u + 1] = v.y; cs[4 * u + 2] = v.z; cs[4 * u + 3] = v.w;
  }
  cp_async_block(R8raw, R8 + ((long long)b * n + c0) * k, ncols * k);
  cp_async_block(P8raw, P8 + ((long long)b * m + r0) * k, nrows * k);
  cp_async_commit();
  if (t < 16) deq4[t] = __fdiv_rn((float)((t & 8) ? t - 16 : t), 7.0f);
  if (t < 32) cfac[t] = t < k ? __fdiv_rn(__fmul_rn(Pscale[b * k + t], Rscale[b * k + t]), 16129.0f) : 0.f;
  cp_async_wait<0>();
  __syncthreads();

  // 2. fragments: R codes as the B operand of n-tile (jj & 15) / 2, column
  // 2 (jj / 16) + jj % 2; P codes x c_l as the A operand in three bf16 parts
#pragma unroll
  for (int it = 0; it < kGrid * KSB * 8 / kRBT; ++it) {
    const int e = t + it * kRBT;
    const int jl = e / (KSB * 8), l = 2 * (e % (KSB * 8));
    const int8_t* rr = R8raw + jl * k;
    const float v0 = (jl < ncols && l < k) ? (float)rr[l] : 0.f;
    const float v1 = (jl < ncols && l + 1 < k) ? (float)rr[l + 1] : 0.f;
    const int jj = jl & 63, ll = l & 15;
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
    RF[((((jl >> 6) * 8 + ((jj & 15) >> 1)) * KSB + (l >> 4)) * 32 + 4 * (2 * (jj >> 4) + (jj & 1)) +
        ((ll >> 1) & 3)) * 2 + (ll >> 3)] = *reinterpret_cast<const uint32_t*>(&h2);
  }
#pragma unroll
  for (int it = 0; it < kRB * KSB * 8 / kRBT; ++it) {
    const int e = t + it * kRBT;
    const int il = e / (KSB * 8), l = 2 * (e % (KSB * 8));
    const int8_t* pr = P8raw + il * k;
    const float v0 = (il < nrows && l < k) ? __fmul_rn((float)pr[l], cfac[l]) : 0.f;
    const float v1 = (il < nrows && l + 1 < k) ? __fmul_rn((float)pr[l + 1], cfac[l + 1]) : 0.f;
    uint32_t w3[3];
    bf16_split3(v0, v1, w3);
    const int r = il & 15, ll = l & 15;
    uint32_t* dst = PF + (((il >> 4) * KSB + (l >> 4)) * 3) * 128 +
                    (4 * (r & 7) + ((ll >> 1) & 3)) * 4 + (r >> 3) + 2 * (ll >> 3);
    dst[0] = w3[0];
    dst[128] = w3[1];
    dst[256] = w3[2];
  }
  __syncthreads();

  // 3. rank-k rebuild P^ R^T, then M = q/7 * s + P^ R^T
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KSB; ++ks) {
    uint32_t a[3][4];
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      const uint4 v = reinterpret_cast<const uint4*>(PF)[((rb * KSB + ks) * 3 + p) * 32 + lane];
      a[p][0] = v.x; a[p][1] = v.y; a[p][2] = v.z; a[p][3] = v.w;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const uint2 bv = reinterpret_cast<const uint2*>(RF)[((slab * 8 + nt) * KSB + ks) * 32 + lane];
      mma_bf16(acc[nt], a[2], bv.x, bv.y);
      mma_bf16(acc[nt], a[1], bv.x, bv.y);
      mma_bf16(acc[nt], a[0], bv.x, bv.y);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (!ok[h]) continue;
    float o[16];
#pragma unroll
    for (int ce = 0; ce < 16; ++ce) {
      const uint32_t word = ce < 8 ? cw[h].x : cw[h].y;
      const float sc = fminf(rsc[h], cs[ce]);
      o[ce] = __fadd_rn(__fmul_rn(deq4[(word >> (4 * (ce & 7))) & 0xF], sc), acc[ce >> 1][2 * h + (ce & 1)]);
    }
    float4* dst = reinterpret_cast<float4*>(M + (long long)b * mn + (long long)(r0 + 16 * rb + g + 8 * h) * n + cb);
#pragma unroll
    for (int u = 0; u < 4; ++u) dst[u] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
  }
}

// The fused pass, pipelined: a CTA owns one 128-column block and walks up to
// kRebuildTiles 64-row tiles of it (rows
// blockIdx.y, + gridDim.y, ...). Q's and R's fragments are copied once; every
// input of tile i + 1 (its P fragments, gradient, codes, row and column scales,
// dense M_{t-1}) streams into the other of two shared-memory stages with
// cp.async while tile i is multiplied, so the memory latency of one tile hides
// behind the work of the previous one. Each thread copies its own gradient (and
// M_{t-1}) chunks and reads only those back; the shared inputs become visible at
// the barrier after the copies complete.
constexpr int kRebuildTiles = 4;

__host__ __device__ constexpr int pipe_g_chunks(int GDT) { return GDT == GM_F32 ? 8 : 4; }
// words of one stage: P fragments, codes (64 rows x 64 B), column and row scales,
// the per-thread gradient chunks, the per-thread dense M_{t-1} chunks
__host__ __device__ constexpr int pipe_stage_words(int SRC, int GDT, int KP) {
  return (SRC == SRC_STATE ? 4 * (kb16(KP) / 16) * 3 * 128 + 64 * 16 + kGrid + kRB : 0) +
         pipe_g_chunks(GDT) * kRBT * 4 + (SRC == SRC_DENSE ? 8 * kRBT * 4 : 0);
}
__host__ __device__ constexpr int pipe_smem_words(int SRC, int GDT, int KP) {
  return 2 * 8 * (KP / 8) * 32 * 4 + (SRC == SRC_STATE ? 2 * 8 * (kb16(KP) / 16) * 32 * 2 : 0) +
         2 * pipe_stage_words(SRC, GDT, KP) + (SRC == SRC_STATE ? 0 : (kRB / 16) * (KP / 8) * 4 * 32);
}

template <int SRC, int GDT, int KP>
__global__ void __launch_bounds__(kRBT, 2) k_rebuild_pipe(
    int m, int n, int k, const uint8_t* __restrict__ codes4, const float* __restrict__ rscale,
    const float* __restrict__ cscale, const float* __restrict__ Mprev, float mu,
    const void* __restrict__ G, const uint32_t* __restrict__ QFg, const uint32_t* __restrict__ RFg,
    const uint32_t* __restrict__ PFg, float* __restrict__ M, double* __restrict__ norm2_part,
    float* __restrict__ Ppart, int32_t* status) {
  constexpr bool ST = SRC == SRC_STATE, DN = SRC == SRC_DENSE, G32 = GDT == GM_F32;
  constexpr int NL = KP / 8, KSB = kb16(KP) / 16, GCH = pipe_g_chunks(GDT);
  constexpr int QW = 8 * NL * 128, RW = 8 * KSB * 64, PW = KSB * 3 * 128;   // words per slab / block
  constexpr int SW = pipe_stage_words(SRC, GDT, KP);
  const int bj = blockIdx.x, b = blockIdx.z;
  const int nb = gridDim.x, nrb = cdiv(m, kRB), mbg = cdiv(m, kGrid);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, tq = lane & 3, rb = warp & 3, slab = warp >> 2;
  const int c0 = bj * kGrid;
  const int cb = c0 + 64 * slab + 16 * tq;   // n % 16 == 0: the run is all in or all out
  const bool colok = cb < n;
  const int ncols = min(kGrid, n - c0);
  const int nsl = cdiv(n, 64), vs = min(2, nsl - 2 * bj);
  const long long mn = (long long)m * n;
  extern __shared__ __align__(16) uint32_t smp[];
  uint32_t* QF = smp;                          // [slab][s][NL][lane][4]
  uint32_t* RF = QF + 2 * QW;                  // [slab][nt][KSB][lane][2]
  uint32_t* stg = RF + (ST ? 2 * RW : 0);      // two stages of SW words
  float* PXd = reinterpret_cast<float*>(stg + 2 * SW);   // [rb][NL][4][lane] (without a state)
  __shared__ float deq4[16];

  // stage layout
  auto PFs = [&](int s) { return stg + s * SW; };                                  // [rb][KSB][part][lane][4]
  auto CDs = [&](int s) { return stg + s * SW + (ST ? 4 * PW : 0); };              // codes [64][16 words]
  auto CSs = [&](int s) { return reinterpret_cast<float*>(CDs(s) + (ST ? 64 * 16 : 0)); };   // [128]
  auto RSs = [&](int s) { return CSs(s) + (ST ? kGrid : 0); };                     // [64]
  auto GSs = [&](int s) { return reinterpret_cast<uint4*>(RSs(s) + (ST ? kRB : 0)); };        // [GCH][256]
  auto MPs = [&](int s) { return GSs(s) + GCH * kRBT; };                           // [8][256]

  auto issue = [&](int rbi, int s) {
    const int r0 = rbi * kRB;
    if constexpr (ST) {
      const int vb = min(kRB / 16, (m >> 4) - r0 / 16);
      cp_async_block_zf(PFs(s), PFg + ((long long)b * (m >> 4) + r0 / 16) * PW, (kRB / 16) * PW * 4, vb * PW * 4);
      {   // codes: 64 rows x 64 bytes, one 16-byte chunk (32 columns) per thread; a
          // chunk half past the last column (ncols % 32 == 16) copies 8 bytes. A codes
          // row is n / 2 bytes, so rows start 16-byte aligned only when n % 32 == 0;
          // otherwise (n % 32 == 16) the chunk goes as two 8-byte copies, which need
          // only the 8-byte alignment that n % 16 == 0 gives.
        const int r = t >> 2, ch = t & 3, gi = r0 + r;
        const int nbytes = gi < m ? max(0, min(16, (ncols - 32 * ch) / 2)) : 0;
        const uint32_t sa = (uint32_t)__cvta_generic_to_shared(CDs(s) + r * 16 + ch * 4);
        const uint8_t* src = nbytes ? codes4 + ((long long)b * m + gi) * (n / 2) + c0 / 2 + 16 * ch : codes4;
        if ((n & 31) == 0) {
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(src), "r"(nbytes)
                       : "memory");
        } else {
          asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(sa), "l"(src),
                       "r"(min(nbytes, 8))
                       : "memory");
          asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(sa + 8u),
                       "l"(nbytes > 8 ? src + 8 : codes4), "r"(max(nbytes - 8, 0))
                       : "memory");
        }
      }
      if (t < kGrid / 4) {   // column scales of the grid-block row
        const bool ok = 4 * t < ncols;
        cp_async16(CSs(s) + 4 * t, ok ? cscale + ((long long)b * mbg + r0 / kGrid) * n + c0 + 4 * t : cscale, ok);
      }
      if (t < kRB) {   // row scales (stride ceil(n / 128) in memory)
        const int gi = r0 + t;
        const uint32_t sa = (uint32_t)__cvta_generic_to_shared(RSs(s) + t);
        if (gi < m)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa),
                       "l"(rscale + ((long long)b * m + gi) * nb + bj) : "memory");
        else
          RSs(s)[t] = 0.f;
      }
    }
    // this thread's gradient (and dense M_{t-1}) chunks: rows g, g + 8 of its warp's 16
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gi = r0 + 16 * rb + g + 8 * h;
      const bool ok = gi < m && colok && G;
      const long long base = (long long)b * mn + (long long)gi * n + cb;
#pragma unroll
      for (int u = 0; u < GCH / 2; ++u) {
        const void* src = ok ? (G32 ? (const void*)(static_cast<const float*>(G) + base + 4 * u)
                                    : (const void*)(static_cast<const uint16_t*>(G) + base + 8 * u))
                             : G ? G : (Mprev ? (const void*)Mprev : (const void*)M);
        cp_async16(&GSs(s)[(h * (GCH / 2) + u) * kRBT + t], src, ok);
      }
      if constexpr (DN) {
        const bool okm = gi < m && colok;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          cp_async16(&MPs(s)[(h * 4 + u) * kRBT + t], okm ? Mprev + base + 4 * u : Mprev, okm);
      }
    }
  };

  const int first = blockIdx.y, stride = gridDim.y;
  int ntl = 0;
  for (int rbi = first; rbi < nrb && ntl < kRebuildTiles; rbi += stride) ++ntl;
  // Q and R fragments of the column block, and the first tile's stage
  cp_async_block_zf(QF, QFg + ((long long)b * nsl + 2 * bj) * QW, 2 * QW * 4, vs * QW * 4);
  if constexpr (ST) cp_async_block_zf(RF, RFg + ((long long)b * nsl + 2 * bj) * RW, 2 * RW * 4, vs * RW * 4);
  if (t < 16) deq4[t] = __fdiv_rn((float)((t & 8) ? t - 16 : t), 7.0f);
  if (ntl > 0) issue(first, 0);
  cp_async_commit();

  bool bad = false;
  for (int i = 0; i < ntl; ++i) {
    const int s = i & 1, rbi = first + i * stride, r0 = rbi * kRB;
    __syncthreads();   // every thread is done with stage s ^ 1 (tile i - 1)
    if (i + 1 < ntl) {
      issue(rbi + stride, s ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();   // stage s (and the fragments) complete and visible

    // rank-k rebuild P^ R^T
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    if constexpr (ST) {
      const uint32_t* PF = PFs(s);
#pragma unroll
      for (int ks = 0; ks < KSB; ++ks) {
        uint32_t a[3][4];
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          const uint4 v = reinterpret_cast<const uint4*>(PF)[((rb * KSB + ks) * 3 + p) * 32 + lane];
          a[p][0] = v.x; a[p][1] = v.y; a[p][2] = v.z; a[p][3] = v.w;
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const uint2 bv = reinterpret_cast<const uint2*>(RF)[((slab * 8 + nt) * KSB + ks) * 32 + lane];
          mma_bf16(acc[nt], a[2], bv.x, bv.y);
          mma_bf16(acc[nt], a[1], bv.x, bv.y);
          mma_bf16(acc[nt], a[0], bv.x, bv.y);
        }
      }
    }

    // M = mu M_prev + G
    float cs[16];
    if constexpr (ST) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 v = reinterpret_cast<const float4*>(CSs(s))[16 * slab + 4 * tq + u];
        cs[4 * u] = v.x; cs[4 * u + 1] = v.y; cs[4 * u + 2] = v.z; cs[4 * u + 3] = v.w;
      }
    }
    float nsq = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rl = 16 * rb + g + 8 * h, gi = r0 + rl;
      const bool ok = gi < m && colok;
      uint32_t gw[GCH / 2 * 4];
#pragma unroll
      for (int u = 0; u < GCH / 2; ++u) {
        const uint4 v = GSs(s)[(h * (GCH / 2) + u) * kRBT + t];
        gw[4 * u] = v.x; gw[4 * u + 1] = v.y; gw[4 * u + 2] = v.z; gw[4 * u + 3] = v.w;
      }
      uint2 cw = make_uint2(0u, 0u);
      float rsc = 0.f;
      if constexpr (ST) {
        cw = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(CDs(s)) + rl * 64 + 32 * slab + 8 * tq);
        rsc = RSs(s)[rl];
      }
      float mpv[16];
      if constexpr (DN) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 v = reinterpret_cast<const float4*>(MPs(s))[(h * 4 + u) * kRBT + t];
          mpv[4 * u] = v.x; mpv[4 * u + 1] = v.y; mpv[4 * u + 2] = v.z; mpv[4 * u + 3] = v.w;
        }
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int ce = 2 * nt + e;
          float gv;
          if constexpr (G32) gv = __uint_as_float(gw[ce]);
          else gv = h16_to_float((uint16_t)(gw[ce >> 1] >> (16 * (ce & 1))), GDT == GM_F16);
          float mp = 0.f;
          if constexpr (ST) {
            const uint32_t word = ce < 8 ? cw.x : cw.y;
            const float sc = fminf(rsc, cs[ce]);
            mp = __fadd_rn(__fmul_rn(deq4[(word >> (4 * (ce & 7))) & 0xF], sc), acc[nt][2 * h + e]);
          } else if constexpr (DN) {
            mp = mpv[ce];
          }
          const float o = ok ? __fadd_rn(__fmul_rn(mu, mp), gv) : 0.f;
          acc[nt][2 * h + e] = o;
          nsq = fmaf(o, o, nsq);
        }
      }
      if (ok && M) {   // M == NULL: the projection alone (a repeated power-iteration step)
        float4* dst = reinterpret_cast<float4*>(M + (long long)b * mn + (long long)gi * n + cb);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_float4(acc[2 * u][2 * h], acc[2 * u][2 * h + 1], acc[2 * u + 1][2 * h],
                               acc[2 * u + 1][2 * h + 1]);
      }
    }
    // a non-finite M_t makes nsq non-finite; only then (or when the finite squares
    // overflowed) are the thread's 32 values checked one by one
    if (!(fabsf(nsq) <= 3.402823466e38f)) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) bad |= !(fabsf(acc[nt][r]) <= 3.402823466e38f);
    }
    // |M|^2 partial of this warp's 16 x 64 part of the tile (fixed shuffle tree)
    double wsq = (double)nsq;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsq += __shfl_xor_sync(0xffffffffu, wsq, o);
    if (lane == 0 && norm2_part) norm2_part[(((long long)b * nrb + rbi) * nb + bj) * (kRBT / 32) + warp] = wsq;

    // projection partials of this warp's 64-column slab
    float pt[NL][4];
#pragma unroll
    for (int nl = 0; nl < NL; ++nl) pt[nl][0] = pt[nl][1] = pt[nl][2] = pt[nl][3] = 0.f;
#pragma unroll
    for (int sk = 0; sk < 8; ++sk) {
      const float xa[4] = {acc[sk][0], acc[sk][2], acc[sk][1], acc[sk][3]};
      uint32_t ah[4], al[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ah[j] = tf32_hi(xa[j]);
        al[j] = tf32_lo(xa[j], ah[j]);
      }
#pragma unroll
      for (int nl = 0; nl < NL; ++nl) {
        const uint4 qv = reinterpret_cast<const uint4*>(QF)[((slab * 8 + sk) * NL + nl) * 32 + lane];
        mma_tf32(pt[nl], al, qv.x, qv.y);
        mma_tf32(pt[nl], ah, qv.z, qv.w);
        mma_tf32(pt[nl], ah, qv.x, qv.y);
      }
    }
    // the slab-1 warp hands its partials to the slab-0 warp of the same rows (a
    // slab beyond the last column holds zeros). With a state the hand-over goes
    // through this pair's own P-fragment rows of the current stage, which only
    // the pair reads (in its rebuild, before the first pair barrier) and which
    // are refilled only after the block-wide barrier at the top of the next tile
    float* PX = ST ? reinterpret_cast<float*>(PFs(s) + rb * KSB * 3 * 128) : PXd + rb * NL * 128;
    static_assert(!ST || NL * 4 * 32 <= KSB * 3 * 128, "hand-over fits the pair's P fragments");
    pair_sync(rb);
    if (slab == 1) {
#pragma unroll
      for (int nl = 0; nl < NL; ++nl)
#pragma unroll
        for (int r = 0; r < 4; ++r) PX[(nl * 4 + r) * 32 + lane] = pt[nl][r];
    }
    pair_sync(rb);
    if (slab == 0) {
      const long long pbase = ((long long)b * nb + bj) * m;
#pragma unroll
      for (int nl = 0; nl < NL; ++nl)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int rl = 16 * rb + g + 8 * (r >> 1), l = 8 * nl + 2 * tq + (r & 1);
          const float v = __fadd_rn(pt[nl][r], PX[(nl * 4 + r) * 32 + lane]);
          if (r0 + rl < m && l < k) Ppart[(pbase + r0 + rl) * k + l] = v;
        }
    }
  }
  if (bad && status) atomicExch(status, GM_E_NONFINITE);
}

// ------------------------------------------------------------------ S4
// (a) P~ = sum of column-split partials (fixed order); partial Gram P~^T P~.
__global__ void __launch_bounds__(kThreads) k_orth_gram(int m, int k, int csplit, int rsplit,
                                                         const float* __restrict__ Ppart,
                                                         double* __restrict__ Ptil,
                                                         double* __restrict__ gram_part,
                                                         const int32_t* skip) {
  if (skip && *skip) return;
  const int split = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int per = cdiv(m, rsplit);
  const int i0 = split * per, i1 = min(m, i0 + per);
  constexpr int CH = 32;
  __shared__ double Ps[CH][kMaxK];
  const int npairs = k * (k + 1) / 2;
  double acc[3] = {0.0, 0.0, 0.0};
  int pa[3], pc[3];
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const int p = t + s * kThreads;
    int a = 0, rem = p;
    while (a < k && rem >= k - a) { rem -= k - a; ++a; }
    pa[s] = a; pc[s] = a + rem;
  }
  for (int c = i0; c < i1; c += CH) {
    for (int e = t; e < CH * k; e += kThreads) {
      const int rr = e / k, l = e % k, gi = c + rr;
      double v = 0.0;
      if (gi < i1) {
        for (int s = 0; s < csplit; ++s) v += (double)Ppart[(((long long)b * csplit + s) * m + gi) * k + l];
        Ptil[((long long)b * m + gi) * k + l] = v;
      }
      Ps[rr][l] = v;
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      if (t + s * kThreads < npairs) {
        for (int rr = 0; rr < CH; ++rr) acc[s] = fma(Ps[rr][pa[s]], Ps[rr][pc[s]], acc[s]);
      }
    }
    __syncthreads();
  }
  double* g = gram_part + ((long long)b * rsplit + split) * k * k;
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    if (t + s * kThreads < npairs) {
      g[pa[s] * k + pc[s]] = acc[s];
      g[pc[s] * k + pa[s]] = acc[s];
    }
  }
}

// (b) Cholesky G = L L^T of the Gram (fp64) with dead-column exclusion, right
// looking: lane i holds row i of G in registers; after step j it holds L[i][j] in
// slot j and has subtracted L[i][j] L[c][j] from its slots c > j (L[c][j] by
// shuffle from lane c), in ascending j as the textbook left-looking sums do.
// Writes L below the diagonal and the reciprocal diagonal on it (0 for a dead
// column) for the forward substitution in (c); NS scale 1 / (|M_t|_F + eps).
constexpr int kCholThreads = 256;
__global__ void __launch_bounds__(kCholThreads) k_orth_chol(int k, int rsplit, const double* __restrict__ gram_part,
                                                   double* __restrict__ Lmat,
                                                   const double* __restrict__ norm2_part, int ntiles,
                                                   float eps, float* __restrict__ scale,
                                                   const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  constexpr unsigned kAll = 0xffffffffu;
  __shared__ double Gs[kMaxK][kMaxK + 1];
  __shared__ double wsum[kCholThreads / 32];
  // the Gram, each entry summed over the row splits in order (all the block's
  // threads, several splits' loads in flight: these sums are latency-bound)
  for (int e = t; e < k * k; e += kCholThreads) {
    const double* gp = gram_part + (long long)b * rsplit * k * k + e;
    double acc = 0.0;
#pragma unroll 8
    for (int p = 0; p < rsplit; ++p) acc += gp[(long long)p * k * k];
    Gs[e / k][e % k] = acc;
  }
  // |M_t|^2 from the rebuild's partials: 256 thread-strided chains, then a fixed tree
  double nsq = 0.0;
  const double* np = norm2_part + (long long)b * ntiles;
#pragma unroll 8
  for (int p = t; p < ntiles; p += kCholThreads) nsq += np[p];
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) nsq += __shfl_xor_sync(kAll, nsq, off);
  if (lane == 0) wsum[warp] = nsq;
  __syncthreads();
  if (warp != 0) return;   // the factorisation is one warp's (no block barrier follows)
  double ns2 = 0.0;
#pragma unroll
  for (int w = 0; w < kCholThreads / 32; ++w) ns2 += wsum[w];
  // row `lane` of the Gram
  double g[kMaxK];
#pragma unroll
  for (int c = 0; c < kMaxK; ++c) g[c] = (lane < k && c < k) ? Gs[lane][c] : 0.0;
  // dead-column tolerance: (1e-6 * max column norm)^2
  double maxn2 = 0.0;
#pragma unroll
  for (int c = 0; c < kMaxK; ++c)
    if (c == lane) maxn2 = g[c];
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) maxn2 = fmax(maxn2, __shfl_xor_sync(kAll, maxn2, off));
  const double tol2 = 1e-12 * maxn2;
  double rinv = 0.0;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j >= k) break;
    const double d = __shfl_sync(kAll, g[j], j);
    const bool alive = (d > tol2) && (d > 0.0);
    const double ljj = alive ? sqrt(d) : 0.0;
    const double rj = alive ? 1.0 / ljj : 0.0;
    const double lij = lane > j ? g[j] * rj : (lane == j ? ljj : 0.0);
    if (lane >= j) g[j] = lij;
    if (lane == j) rinv = rj;
#pragma unroll
    for (int c = j + 1; c < kMaxK; ++c) {
      const double lcj = __shfl_sync(kAll, lij, c);
      if (lane >= c && c < k) g[c] = fma(-lij, lcj, g[c]);
    }
  }
  if (lane < k) {
    double* out = Lmat + ((long long)b * k + lane) * k;
#pragma unroll
    for (int c = 0; c < kMaxK; ++c)
      if (c < k) out[c] = c < lane ? g[c] : (c == lane ? rinv : 0.0);
  }
  if (lane == 0 && scale) scale[b] = (float)(1.0 / (sqrt(ns2) + (double)eps));
}

// (c) P = P~ L^-T by forward substitution (fp64), one row of P per thread:
// P[i][l] = (P~[i][l] - sum_{a<l} P[i][a] L[l][a]) / L[l][l], zero for a dead
// column. Stored fp32 and as fragments: PB for the back-projection (PB[b][i / 8]
// [l / 8][lane][4] = {hi(P[8 s + t][l]), hi(P[8 s + t + 4][l]), lo, lo}, lane =
// 4 (l % 8) + t) and PA (-P) for the residual (nullable); zero for k <= l < KP.
// PT (nullable): the tensor-core residual's operand rows, tf32 hi then lo halves
// ([2][B][m][32], columns beyond k zero).
// The column absolute maxima of P go to Pmax (fp32 bits, atomicMax; nullable).
template <int KP>
__global__ void __launch_bounds__(kThreads) k_orth_apply(int m, int k, const double* __restrict__ Ptil,
                                                          const double* __restrict__ Lmat,
                                                          float* __restrict__ P,
                                                          uint32_t* __restrict__ PB,
                                                          uint32_t* __restrict__ PA,
                                                          float* __restrict__ PT,
                                                          unsigned* __restrict__ Pmax,
                                                          const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y, t = threadIdx.x, lane = t & 31;
  __shared__ double Ls[KP][KP];   // L below the diagonal, 1 / L[l][l] on it
  __shared__ unsigned cmax[KP];
  for (int e = t; e < KP * KP; e += kThreads) {
    const int l = e / KP, a = e % KP;
    Ls[l][a] = (a < k && l < k) ? Lmat[((long long)b * k + l) * k + a] : 0.0;
  }
  if (t < KP) cmax[t] = 0u;
  __syncthreads();
  const int i = blockIdx.x * kThreads + t;
  const bool in = i < m;
  double row[KP];
#pragma unroll
  for (int a = 0; a < KP; ++a) row[a] = (in && a < k) ? Ptil[((long long)b * m + i) * k + a] : 0.0;
#pragma unroll
  for (int l = 0; l < KP; ++l) {
    double v = row[l];
#pragma unroll
    for (int a = 0; a < l; ++a) v = fma(-row[a], Ls[l][a], v);   // row[a] holds P[i][a] by now
    row[l] = v * Ls[l][l];
    const float f = (float)row[l];   // 0 outside the matrix
    const unsigned mx = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(f)));
    if (lane == 0 && mx) atomicMax(&cmax[l], mx);
    if (!in) continue;
    if (l < k) P[((long long)b * m + i) * k + l] = f;
    if (PB) {
      uint32_t* dst = PB + ((((long long)b * (m >> 3) + (i >> 3)) * (KP / 8) + (l >> 3)) * 32 +
                            4 * (l & 7) + (i & 3)) * 4 + ((i & 7) >> 2);
      const uint32_t hi = tf32_hi(f);
      dst[0] = hi;
      dst[2] = tf32_lo(f, hi);
    }
    if (PA) {
      const long long at = pa_at(b, m >> 4, KP / 8, i, l);
      const uint32_t hi = tf32_hi(-f);
      PA[at] = hi;
      PA[at + 128] = tf32_lo(-f, hi);
    }
  }
  if (PT && in) {   // the operand row, 16-byte stores; columns beyond KP are zero
    float4* hi4 = reinterpret_cast<float4*>(PT + ((long long)b * m + i) * 32);
    float4* lo4 = reinterpret_cast<float4*>(PT + (long long)gridDim.y * m * 32 + ((long long)b * m + i) * 32);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float h[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int l = 4 * q + e;
        const float f = l < KP ? (float)row[l < KP ? l : 0] : 0.f;   // 0 beyond k (row is 0 there)
        const uint32_t hb = tf32_hi(f);
        h[e] = __uint_as_float(hb);
        lo[e] = __uint_as_float(tf32_lo(f, hb));
      }
      hi4[q] = make_float4(h[0], h[1], h[2], h[3]);
      lo4[q] = make_float4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  __syncthreads();
  if (Pmax && t < k && cmax[t]) atomicMax(&Pmax[b * k + t], cmax[t]);
}

// ------------------------------------------------------------------ S5
// R = M^T P over row splits, and the normalised wide-form NS input
// X = round16(scale * M) (X = M^T when m > n).
// CTA: 64 columns x the rows of its split, in chunks of 128 rows; 8 warps. Warp
// w owns the 32-column half w & 1 and the rows 32 (w >> 1) .. + 31 of each chunk
// as four k-steps of 8 rows. Per k-step, lane (g, t) loads the float4
// M[i][4 g .. 4 g + 3] of rows i = 8 s + t and 8 s + t + 4 (one load instruction
// reads four whole 128-byte row segments), through a two-stage cp.async ring
// in shared memory (each thread reads back only its own copies, so the next
// chunk streams in while this one is multiplied); element 2 mt + h of the float4 is row
// g + 8 h of m-tile mt in the A fragment of M^T (tf32 mma.m16n8k8, 3xTF32
// against P's precomputed fragments). fp32 sums over at most 1024 rows per
// split, the four row warps added in order, fp64 across splits.
// Two fp32 values rounded to a packed pair of 16-bit floats (a in the low half).
template <bool F16>
__device__ __forceinline__ uint32_t pack_h16x2(float a, float b) {
  if constexpr (F16) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

template <int KP, bool F16>   // F16: the NS input in fp16 (Gram NS), else bf16
__global__ void __launch_bounds__(kThreads, 2) k_backproject(int m, int n, int k, int rsplit,
                                                              const float* __restrict__ M,
                                                              const uint32_t* __restrict__ PB,
                                                              const float* __restrict__ scale,
                                                              uint16_t* __restrict__ X16,
                                                              double* __restrict__ Rpart,
                                                              const int32_t* skip) {
  if (skip && *skip) return;
  // per-warp transpose tile [col][row]; rows of 36 halves (72 B): the 2-byte stores
  // of a warp (8 columns 4 apart) fall on 2-way shared banks, the 8-byte row reads
  // on distinct ones
  constexpr int NL = KP / 8, CH = 128, XS = 36;
  __shared__ __align__(16) uint16_t Xt[8][32][XS];
  __shared__ float redR[64][KP + 1];
  extern __shared__ __align__(16) float4 Ms[];       // [stage][warp][slot][lane]
  const int cbk = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, tq = lane & 3, half = warp & 1, rg = warp >> 1;
  const int c0 = cbk * 64 + 32 * half;   // the warp's 32 columns
  const int cq = c0 + 4 * g;             // this lane's float4 (n % 16 == 0: all in or out)
  const bool colok = cq < n;
  const int nchunks = cdiv(m, CH);
  const int per = cdiv(nchunks, rsplit);
  const int ch0 = split * per, ch1 = min(nchunks, ch0 + per);
  const float* Mb = M + (long long)b * m * n;
  const uint4* PBb = reinterpret_cast<const uint4*>(PB) + (long long)b * (m >> 3) * NL * 32;
  const bool tall = m > n;
  const float sc = X16 ? scale[b] : 0.f;
  uint16_t* Xb = X16 ? X16 + (long long)b * m * n : nullptr;

  float acc[2][NL][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nl = 0; nl < NL; ++nl) acc[mt][nl][0] = acc[mt][nl][1] = acc[mt][nl][2] = acc[mt][nl][3] = 0.f;

  auto issue = [&](int chn, int st) {
    const int i0 = chn * CH + 32 * rg;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gi = i0 + 8 * (j >> 1) + tq + 4 * (j & 1);
      const bool ok = gi < m && colok;
      cp_async16(&Ms[((st * 8 + warp) * 8 + j) * 32 + lane], ok ? Mb + (long long)gi * n + cq : Mb, ok);
    }
    cp_async_commit();
  };
  // P fragments of the warp's k-step sequence (chunk c, step s: rows c * 128 +
  // 32 rg + 8 s), loaded one k-step ahead from L2
  const int nq = (ch1 - ch0) * 4;
  auto pb_load = [&](int q, uint4 (&dst)[NL]) {
    const int i8 = (ch0 + (q >> 2)) * CH + 32 * rg + 8 * (q & 3);
    const bool ok = q < nq && i8 < m;
#pragma unroll
    for (int nl = 0; nl < NL; ++nl)
      dst[nl] = ok ? PBb[((long long)(i8 >> 3) * NL + nl) * 32 + lane] : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 pbn[NL];
  pb_load(0, pbn);
  if (ch0 < ch1) issue(ch0, 0);
  for (int chn = ch0; chn < ch1; ++chn) {
    const int i0 = chn * CH + 32 * rg;   // the warp's 32 rows
    const int st = (chn - ch0) & 1;
    if (chn + 1 < ch1) {
      issue(chn + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    float4 v[4][2];
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) v[s][hh] = Ms[((st * 8 + warp) * 8 + 2 * s + hh) * 32 + lane];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int i8 = i0 + 8 * s;
      uint4 pb[NL];
#pragma unroll
      for (int nl = 0; nl < NL; ++nl) pb[nl] = pbn[nl];
      pb_load((chn - ch0) * 4 + s + 1, pbn);
      if (i8 >= m) continue;   // m % 8 == 0: a k-step is all in or all out (warp-uniform)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const float xa[4] = {mt ? v[s][0].z : v[s][0].x, mt ? v[s][0].w : v[s][0].y,
                             mt ? v[s][1].z : v[s][1].x, mt ? v[s][1].w : v[s][1].y};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ah[i] = tf32_hi(xa[i]);
          al[i] = tf32_lo(xa[i], ah[i]);
        }
#pragma unroll
        for (int nl = 0; nl < NL; ++nl) {
          mma_tf32(acc[mt][nl], al, pb[nl].x, pb[nl].y);
          mma_tf32(acc[mt][nl], ah, pb[nl].z, pb[nl].w);
          mma_tf32(acc[mt][nl], ah, pb[nl].x, pb[nl].y);
        }
      }
    }
    if (Xb) {
      if (!tall) {
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int gi = i0 + 8 * s + tq + 4 * hh;
            if (gi < m && colok) {
              const float4 x = v[s][hh];
              uint2 w;
              w.x = pack_h16x2<F16>(x.x * sc, x.y * sc);
              w.y = pack_h16x2<F16>(x.z * sc, x.w * sc);
              *reinterpret_cast<uint2*>(Xb + (long long)gi * n + cq) = w;
            }
          }
      } else {
        // X[j][i] = M[i][j]: through the warp's tile, then 32-byte row runs of X
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int ii = 8 * s + tq + 4 * hh;
            const float4 x = v[s][hh];
            const uint32_t p01 = pack_h16x2<F16>(x.x * sc, x.y * sc);
            const uint32_t p23 = pack_h16x2<F16>(x.z * sc, x.w * sc);
            Xt[warp][4 * g][ii] = (uint16_t)(p01 & 0xFFFFu);
            Xt[warp][4 * g + 1][ii] = (uint16_t)(p01 >> 16);
            Xt[warp][4 * g + 2][ii] = (uint16_t)(p23 & 0xFFFFu);
            Xt[warp][4 * g + 3][ii] = (uint16_t)(p23 >> 16);
          }
        __syncwarp();
        if (c0 + lane < n) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            if (i0 + 16 * q < m) {   // m % 16 == 0: 16-row runs are all in or all out
              const uint2* src = reinterpret_cast<const uint2*>(&Xt[warp][lane][16 * q]);
              uint4* dst = reinterpret_cast<uint4*>(Xb + (long long)(c0 + lane) * m + i0 + 16 * q);
              const uint2 a = src[0], b2 = src[1], c = src[2], d = src[3];
              dst[0] = make_uint4(a.x, a.y, b2.x, b2.y);
              dst[1] = make_uint4(c.x, c.y, d.x, d.y);
            }
          }
        }
        __syncwarp();
      }
    }
  }
  // the four row warps of each half, added in order
  for (int w = 3; w >= 0; --w) {
    if (rg == w) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nl = 0; nl < NL; ++nl)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            float* slot = &redR[32 * half + 4 * g + 2 * mt + (r >> 1)][8 * nl + 2 * tq + (r & 1)];
            *slot = (w == 3) ? acc[mt][nl][r] : (*slot + acc[mt][nl][r]);
          }
    }
    __syncthreads();
  }
  double* out = Rpart + ((long long)b * rsplit + split) * n * k;
  for (int e = t; e < 64 * k; e += kThreads) {
    const int cc = e / k, l = e % k;
    if (cbk * 64 + cc < n) out[(long long)(cbk * 64 + cc) * k + l] = (double)redR[cc][l];
  }
}

// R = the sum of the row splits (fp64, in order), and its residual fragments RB
// over the padded nsl * 64 x kp range (zero outside n x k).
// The column absolute maxima of R go to Rmax (fp32 bits, atomicMax; nullable).
__global__ void __launch_bounds__(kThreads) k_finalize_r(int n, int k, int rsplit,
                                                          const double* __restrict__ Rpart,
                                                          float* __restrict__ R,
                                                          uint32_t* __restrict__ RB,
                                                          float* __restrict__ RT,
                                                          unsigned* __restrict__ Rmax,
                                                          const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y, t = threadIdx.x;
  const int kp = factor_width(k), nsl = cdiv(n, 64);
  __shared__ unsigned cmax[kMaxK];
  if (t < kMaxK) cmax[t] = 0u;
  __syncthreads();
  const long long e = (long long)blockIdx.x * kThreads + t;
  const bool in = e < (long long)nsl * 64 * kp;
  const int j = (int)(e / kp), l = (int)(e % kp);
  float f = 0.f;
  if (in && j < n && l < k) {
    double s = 0.0;
    for (int p = 0; p < rsplit; ++p) s += Rpart[(((long long)b * rsplit + p) * n + j) * k + l];
    f = (float)s;
    R[((long long)b * n + j) * k + l] = f;
    if (f != 0.f) atomicMax(&cmax[l], __float_as_uint(fabsf(f)));
  }
  __syncthreads();
  if (Rmax && t < k && cmax[t]) atomicMax(&Rmax[b * k + t], cmax[t]);
  if (!in) return;
  if (RB) {
    const long long at = rb_at(b, nsl, kp >> 3, j, l);
    const uint32_t hi = tf32_hi(f);
    RB[at] = hi;
    RB[at + 2] = tf32_lo(f, hi);
  }
  if (RT && j < n) {   // the tensor-core residual's operand rows ([2][B][n][32], tf32 hi, lo)
    const long long row = ((long long)b * n + j) * 32, lo_off = (long long)gridDim.y * n * 32;
    const uint32_t hi = tf32_hi(f);
    RT[row + l] = __uint_as_float(hi);
    RT[lo_off + row + l] = __uint_as_float(tf32_lo(f, hi));
    if (l == kp - 1)
      for (int c = kp; c < 32; ++c) RT[row + c] = RT[lo_off + row + c] = 0.f;
  }
}

// ------------------------------------------------------------------ S7
// One 128 x 128 grid block per CTA of 8 warps (two CTAs per SM, so that one
// CTA's loads overlap the other's arithmetic). Warp w owns the rows 16 w +
// {g, g + 8} of the block and, in each of its two 64-column slabs, the columns
// 64 slab + 16 t .. + 15 (lane = 4 g + t): the C fragments of the rank-k
// products, as in the rebuild. The residual x = M - P R^T is formed in those
// fragments: M is loaded as the accumulator, A = -P and B = R^T are tf32 hi + lo
// pairs (3xTF32, mma.m16n8k8). A row's absolute maximum over the block's 128
// columns is complete inside its warp (the four lanes of the row); the column
// maxima need one exchange of 8 x 128 values through shared memory. Then the
// codes q = rint(fp32(x / s) * 7) with s = min(row max, column max). Since
// |x| <= s, the quotient taken as z = x * fl(7 / s) is within 7 * 2^-22 of
// fp32(x / s) * 7; where z lies at least 2^-16 away from a rounding tie, rint(z)
// is the code, elsewhere the IEEE division decides.
// FR: -P and R come as ready-made fragments (PA, RB); otherwise from raw rows.
// Q8 (given with the P and R column maxima): the CTAs of block column 0 also
// write the 8-bit codes of their 128 rows of P, those of block row 0 of their
// 128 rows of R (q = rint(fp32(x / s) * 127), s the column absolute maximum;
// the worked step's step 5), after their 4-bit codes; block (0, 0) the scales
// and the step count.
constexpr int kRT = 256;   // threads of the residual CTAs (8 warps)
struct Quant8Out {
  const unsigned* Pmax;
  const unsigned* Rmax;
  int8_t* P8;
  float* Pscale;
  int8_t* R8;
  float* Rscale;
  int64_t* step;
};

// q = rint(fp32(x / s) * 127) for |x| <= s. Taken as rint(x * fl(127 / s)) where
// that product lies at least 2^-12 away from a rounding tie (the two differ by at
// most 127 * 2^-22), else by the IEEE division.
__device__ __forceinline__ int8_t code8(float x, float s, float r127) {
  if (!(s > 0.f)) return 0;
  const float z = __fmul_rn(x, r127), zr = rintf(z);
  int q;
  if (fabsf(__fsub_rn(z, zr)) < 0.49975586f)   // 0.5 - 2^-12
    q = (int)zr;
  else
    q = (int)rintf(__fmul_rn(__fdiv_rn(x, s), 127.0f));
  return (int8_t)max(-127, min(127, q));
}

// The residual-from-codes variant: the residual pass's factor fragments PA (-P^)
// and RB (R^) rebuilt from this step's 8-bit codes, P^ = deq8(code8(P)) and
// R^ = deq8(code8(R)), instead of the unquantized P and R. Pmax / Rmax hold the
// complete column absolute maxima (the 8-bit scales). Elements [0, m k) are P's,
// [m k, (m + n) k) R's; fragment slots of columns l >= k keep their zeros.
template <int KP>
__global__ void __launch_bounds__(kThreads) k_codes_frags(int m, int n, int k,
                                                           const float* __restrict__ P,
                                                           const float* __restrict__ R,
                                                           const unsigned* __restrict__ Pmax,
                                                           const unsigned* __restrict__ Rmax,
                                                           uint32_t* __restrict__ PA,
                                                           uint32_t* __restrict__ RB,
                                                           float* __restrict__ PT,
                                                           float* __restrict__ RT,
                                                           const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y, t = threadIdx.x;
  __shared__ float s8[2][kMaxK], r127[2][kMaxK];
  if (t < 2 * kMaxK) {
    const int w = t / kMaxK, l = t % kMaxK;
    const float sv = l < k ? __uint_as_float((w ? Rmax : Pmax)[b * k + l]) : 0.f;
    s8[w][l] = sv;
    r127[w][l] = sv > 0.f ? __fdiv_rn(127.0f, sv) : 0.f;
  }
  __syncthreads();
  const long long e = (long long)blockIdx.x * kThreads + t;
  const long long np = (long long)m * k, nr = (long long)n * k;
  if (e < np) {
    const int i = (int)(e / k), l = (int)(e % k);
    const float x = P[(long long)b * np + e];
    const float v = -deq8(code8(x, s8[0][l], r127[0][l]), s8[0][l]);
    const long long at = pa_at(b, m >> 4, KP / 8, i, l);
    const uint32_t hi = tf32_hi(v);
    PA[at] = hi;
    PA[at + 128] = tf32_lo(v, hi);
    if (PT) {   // +P^ for the tensor-core residual
      const long long pt = ((long long)b * m + i) * 32 + l;
      const uint32_t ph = tf32_hi(-v);
      PT[pt] = __uint_as_float(ph);
      PT[(long long)gridDim.y * m * 32 + pt] = __uint_as_float(tf32_lo(-v, ph));
    }
  } else if (e < np + nr) {
    const long long e2 = e - np;
    const int j = (int)(e2 / k), l = (int)(e2 % k);
    const float x = R[(long long)b * nr + e2];
    const float v = deq8(code8(x, s8[1][l], r127[1][l]), s8[1][l]);
    const long long at = rb_at(b, cdiv(n, 64), KP / 8, j, l);
    const uint32_t hi = tf32_hi(v);
    RB[at] = hi;
    RB[at + 2] = tf32_lo(v, hi);
    if (RT) {
      const long long rt = ((long long)b * n + j) * 32 + l;
      RT[rt] = __uint_as_float(hi);
      RT[(long long)gridDim.y * n * 32 + rt] = __uint_as_float(tf32_lo(v, hi));
    }
  }
}

template <int KP, bool FR>   // KP = 0: no rank-k term
__global__ void __launch_bounds__(kRT, 2) k_residual_quant4(
    int m, int n, int k, const float* __restrict__ X, const float* __restrict__ P,
    const float* __restrict__ R, const uint32_t* __restrict__ PA, const uint32_t* __restrict__ RB,
    uint8_t* __restrict__ codes4, float* __restrict__ rscale, float* __restrict__ cscale,
    Quant8Out q8, const int32_t* skip) {
  if (skip && *skip) return;
  constexpr int NL = KP / 8;
  const int bj = blockIdx.x, bi = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, mb = gridDim.y;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, tq = lane & 3, rb = warp;
  const int r0 = bi * kGrid, c0 = bj * kGrid;
  extern __shared__ __align__(16) uint32_t smq[];
  uint32_t* AF = smq;                      // [rb][ks][part][lane][4]: -P hi, lo
  uint32_t* BF = smq + 8 * NL * 2 * 128;   // [slab][nt][ks][lane][4]: {b0, b1} hi, {b0, b1} lo
  float* Praw = reinterpret_cast<float*>(BF + 2 * 8 * NL * 32 * 4);   // [128][k]
  float* Rraw = Praw + kGrid * KP;                                     // [128][k]
  const int nrows = min(kGrid, m - r0), ncols = min(kGrid, n - c0);   // multiples of 16
  __shared__ __align__(16) float CM[8][kGrid];    // per warp: column maxima of its 16 rows
  __shared__ __align__(16) float r7c[kGrid];
  __shared__ float smax_c[kGrid];

  // M as the accumulator: acc[slab][nt][2 h + e] = element (row g + 8 h, column
  // 64 slab + 16 t + 2 nt + e)
  float acc[2][8][4];
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    const int cb = c0 + 64 * sl + 16 * tq;   // n % 16 == 0: the run is all in or all out
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gi = r0 + 16 * rb + g + 8 * h;
      const bool ok = gi < m && cb < n;
      const float4* src = reinterpret_cast<const float4*>(X + ((long long)b * m + gi) * n + cb);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 v = ok ? src[u] : make_float4(0.f, 0.f, 0.f, 0.f);
        acc[sl][2 * u][2 * h] = v.x;
        acc[sl][2 * u][2 * h + 1] = v.y;
        acc[sl][2 * u + 1][2 * h] = v.z;
        acc[sl][2 * u + 1][2 * h + 1] = v.w;
      }
    }
  }
  if constexpr (KP > 0 && FR) {
    const int nsl = cdiv(n, 64), vs = min(2, nsl - 2 * bj), vb = min(8, (m >> 4) - r0 / 16);
    constexpr int aw = NL * 2 * 128, bw = 8 * NL * 128;   // words per row block / slab
    cp_async_block_zf(AF, PA + ((long long)b * (m >> 4) + r0 / 16) * aw, 8 * aw * 4, vb * aw * 4);
    cp_async_block_zf(BF, RB + ((long long)b * nsl + 2 * bj) * bw, 2 * bw * 4, vs * bw * 4);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
  }
  if constexpr (KP > 0 && !FR) {
    cp_async_block(Praw, P + ((long long)b * m + r0) * k, nrows * k * 4);
    cp_async_block(Rraw, R + ((long long)b * n + c0) * k, ncols * k * 4);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
#pragma unroll 4
    for (int it = 0; it < kGrid * KP / kRT; ++it) {
      const int e = t + it * kRT;
      const int il = e / KP, l = e % KP;
      const float pv = (il < nrows && l < k) ? -Praw[il * k + l] : 0.f;
      const float rv = (il < ncols && l < k) ? Rraw[il * k + l] : 0.f;
      {
        const int r = il & 15;
        uint32_t* dst = AF + (((il >> 4) * NL + (l >> 3)) * 2) * 128 + (4 * (r & 7) + (l & 3)) * 4 +
                        (r >> 3) + 2 * ((l & 7) >> 2);
        const uint32_t hi = tf32_hi(pv);
        dst[0] = hi;
        dst[128] = tf32_lo(pv, hi);
      }
      {
        const int jj = il & 63;
        uint32_t* dst = BF + ((((il >> 6) * 8 + ((jj & 15) >> 1)) * NL + (l >> 3)) * 32 +
                              4 * (2 * (jj >> 4) + (jj & 1)) + (l & 3)) * 4 + ((l & 7) >> 2);
        const uint32_t hi = tf32_hi(rv);
        dst[0] = hi;
        dst[2] = tf32_lo(rv, hi);
      }
    }
    __syncthreads();
  }
  if constexpr (KP > 0) {
#pragma unroll
    for (int ks = 0; ks < NL; ++ks) {
      uint32_t ah[4], al[4];
      {
        const uint4 h4 = reinterpret_cast<const uint4*>(AF)[((rb * NL + ks) * 2) * 32 + lane];
        const uint4 l4 = reinterpret_cast<const uint4*>(AF)[((rb * NL + ks) * 2 + 1) * 32 + lane];
        ah[0] = h4.x; ah[1] = h4.y; ah[2] = h4.z; ah[3] = h4.w;
        al[0] = l4.x; al[1] = l4.y; al[2] = l4.z; al[3] = l4.w;
      }
#pragma unroll
      for (int sl = 0; sl < 2; ++sl)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const uint4 bv = reinterpret_cast<const uint4*>(BF)[((sl * 8 + nt) * NL + ks) * 32 + lane];
          mma_tf32(acc[sl][nt], al, bv.x, bv.y);
          mma_tf32(acc[sl][nt], ah, bv.z, bv.w);
          mma_tf32(acc[sl][nt], ah, bv.x, bv.y);
        }
    }
  }
  // rows and columns outside the matrix are 0 (loaded as 0; their P rows are 0)
  // row maxima over the block's 128 columns: the thread's 32, then the 4 lanes of the row
  float rmax[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float v = 0.f;
#pragma unroll
    for (int sl = 0; sl < 2; ++sl)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        v = fmaxf(v, fmaxf(fabsf(acc[sl][nt][2 * h]), fabsf(acc[sl][nt][2 * h + 1])));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    rmax[h] = v;
    const int gi = r0 + 16 * rb + g + 8 * h;
    if (tq == 0 && gi < m) rscale[((long long)b * m + gi) * nb + bj] = v;
  }
  // column maxima over the warp's 16 rows (the 8 lanes g of each column), then
  // over the 8 warps
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = fmaxf(fabsf(acc[sl][nt][e]), fabsf(acc[sl][nt][2 + e]));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        if (g == 0) CM[rb][64 * sl + 16 * tq + 2 * nt + e] = v;
      }
    }
  }
  __syncthreads();
  if (t < kGrid) {
    float v = CM[0][t];
#pragma unroll
    for (int w = 1; w < 8; ++w) v = fmaxf(v, CM[w][t]);
    smax_c[t] = v;
    r7c[t] = v > 0.f ? __fdiv_rn(7.0f, v) : 0.f;
    if (c0 + t < n) cscale[((long long)b * mb + bi) * n + c0 + t] = v;
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int rl = 16 * rb + g + 8 * h, gi = r0 + rl;
    const float rr7 = rmax[h] > 0.f ? __fdiv_rn(7.0f, rmax[h]) : 0.f;
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      const int cb = c0 + 64 * sl + 16 * tq;
      if (gi >= m || cb >= n) continue;
      float rc7[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 v = *reinterpret_cast<const float4*>(&r7c[64 * sl + 16 * tq + 4 * u]);
        rc7[4 * u] = v.x; rc7[4 * u + 1] = v.y; rc7[4 * u + 2] = v.z; rc7[4 * u + 3] = v.w;
      }
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int ce = 0; ce < 16; ++ce) {
        const float x = acc[sl][ce >> 1][2 * h + (ce & 1)];
        const float z = __fmul_rn(x, fmaxf(rr7, rc7[ce]));
        const float zr = rintf(z);
        int q;
        if (fabsf(__fsub_rn(z, zr)) < 0.49998474f) {   // 0.5 - 2^-16
          q = (int)zr;
        } else {
          const float sv = fminf(rmax[h], smax_c[64 * sl + 16 * tq + ce]);
          q = sv > 0.f ? (int)rintf(__fmul_rn(__fdiv_rn(x, sv), 7.0f)) : 0;
        }
        q = max(-7, min(7, q));
        w[ce >> 3] |= (uint32_t)(q & 0xF) << (4 * (ce & 7));
      }
      *reinterpret_cast<uint2*>(codes4 + ((long long)b * m + gi) * (n / 2) + cb / 2) = make_uint2(w[0], w[1]);
    }
  }
  // 8-bit codes of P (block column 0) and R (block row 0), after the block's own
  // codes: the factor values are loaded only now, so they hold no registers above
  if (q8.Pmax && (bj == 0 || bi == 0)) {
    for (int which = 0; which < 2; ++which) {
      const bool doit = which == 0 ? bj == 0 : bi == 0;
      if (!doit) continue;
      const unsigned* mx = which == 0 ? q8.Pmax : q8.Rmax;
      const float* src = which == 0 ? P + ((long long)b * m + r0) * k : R + ((long long)b * n + c0) * k;
      int8_t* dst = which == 0 ? q8.P8 + ((long long)b * m + r0) * k : q8.R8 + ((long long)b * n + c0) * k;
      const int cnt = (which == 0 ? nrows : ncols) * k;
      for (int e = t; e < cnt; e += kRT) {
        const int l = e % k;
        const float sv = __uint_as_float(mx[b * k + l]);
        const float r127 = sv > 0.f ? __fdiv_rn(127.0f, sv) : 0.f;
        dst[e] = code8(src[e], sv, r127);
      }
    }
    if (bi == 0 && bj == 0 && t < k) {
      q8.Pscale[b * k + t] = __uint_as_float(q8.Pmax[b * k + t]);
      q8.Rscale[b * k + t] = __uint_as_float(q8.Rmax[b * k + t]);
    }
  }
  if (q8.step && b == 0 && bi == 0 && bj == 0 && t == 0) *q8.step += 1;
}

// ---------------------------------------------- S7 on the 5th-generation tensor cores
// The step's residual pass, one persistent CTA per SM walking a contiguous run of
// 128 x 128 grid blocks (batch, block row, block column; columns fastest), with the
// rank-k product on tcgen05 (kind::tf32) and the block held in tensor memory:
//   warp 0      : TMA producer: the block's M tile (four 128 x 32 fp32 boxes,
//                 128-byte swizzle) into a two-stage ring; the block's R operand
//                 rows and, when the block row changes, its P rows, as tf32 hi / lo
//                 pairs (pre-split by the kernels that produce P and R; the k <= 32
//                 factor columns zero-padded to 32, one 128-byte swizzled row each:
//                 the K-major operand layout);
//   warp 1      : allocates 256 TMEM columns; lane 0 issues the 3xTF32 product
//                 D = P_hi R_hi^T + P_hi R_lo^T + P_lo R_hi^T (M = N = 128, K = 8 per
//                 instruction) into one of two 128-column accumulators;
//   warps 2..17 : the block sweeps, while the next block's M streams in and its
//                 product runs. Warp w owns the TMEM lanes (rows) 32 (w & 3) .. + 31
//                 and a 32-column group of the block: it reads D in 16-column chunks,
//                 forms x = M - D from its rows of the swizzled M stage, keeps the row
//                 maxima in the thread, reduces the column maxima over its 32 rows
//                 with redux.sync and writes x back into TMEM; the column groups of a
//                 row and the four row quarters of a column meet in shared memory. A
//                 second sweep over TMEM turns x into codes q = rint(fp32(x / s) * 7),
//                 s = min(row max, column max), with the same fl(7 / s) shortcut and
//                 IEEE fallback as k_residual_quant4 (one tie test per 16-element
//                 run, the rounding on the FMA pipe), and stores each thread's 8 code
//                 bytes per chunk. The 8-bit codes of P's rows of block row bi are
//                 written by the block (bi, bi mod nb), those of R's rows of block
//                 column bj by the block (bj mod mb, bj): one job per block row and
//                 column, spread over the grid; block (0, 0) writes the scales and
//                 the step count.
// Operand tiles are single-buffered: the next block's R (and P) rows load as soon as
// the product that read them has completed. Every wait is bounded (~2 s of
// %globaltimer) and gives up at once when another role has aborted; a timeout records
// GM_E_TIMEOUT in `status`, every role leaves its loop, the producer and the MMA
// issuer wait (bounded) for their copies and products still in flight, and the
// tensor memory is freed.
constexpr int kTcTmemCols = 128;   // one accumulator: 128 lanes x 128 fp32 columns

__device__ __forceinline__ uint32_t tc_smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ bool tc_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::tf32: D f32, A and B tf32, both K-major, M = N = 128.
constexpr uint32_t kTcIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tc_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

constexpr int kWsEpiWarps = 16;
constexpr int kWsColGroups = kWsEpiWarps / 4;          // column groups of a block
constexpr int kWsCols = kGrid / kWsColGroups;          // columns per epilogue warp
constexpr int kWsChunks = kWsCols / 16;
constexpr int kWsThreads = (2 + kWsEpiWarps) * 32;
constexpr int kQ8Per = kGrid * kMaxK / (kWsEpiWarps * 32);   // 8-bit codes per thread and job
constexpr uint32_t kWsTile = 128 * 32 * 4;                        // one 128 x 32 fp32 box
constexpr uint32_t kWsOps = 4 * kWsTile;                          // P hi, lo, R hi, lo
constexpr uint32_t kWsStage = 4 * kWsTile;                        // M: four boxes
constexpr uint32_t kWsSmemBytes = kWsOps + 2 * kWsStage + 1024;   // + alignment

struct ResidualWsMaps {
  CUtensorMap P, Plo, R, Rlo;   // [B][rows][32] fp32 operand rows, {32, 128, 1} boxes, 128-byte swizzle
  CUtensorMap M;                // [B][m][n] fp32, {32, 128, 1} boxes, 128-byte swizzle
};

__device__ __forceinline__ bool ws_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (tc_try_wait(bar, parity)) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t it = 1;; ++it) {
    if (tc_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > 2000000000ull) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ void ws_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void ws_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void ws_tma3(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                        int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void ws_epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kWsEpiWarps * 32) : "memory");
}
// true in every epilogue thread when `pred` holds in any of them
__device__ __forceinline__ bool ws_epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 2, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(kWsEpiWarps * 32)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kWsThreads, 1) k_residual_ws(
    const __grid_constant__ ResidualWsMaps maps, int m, int n, int k, int nb, int mb, int total,
    const float* __restrict__ P, const float* __restrict__ R, uint8_t* __restrict__ codes4,
    float* __restrict__ rscale, float* __restrict__ cscale, Quant8Out q8, const int32_t* skip,
    int32_t* status) {
  if (skip && *skip) return;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // this CTA's contiguous run of blocks (runs differ in length by at most one)
  const int blk0 = (int)((long long)blockIdx.x * total / gridDim.x);
  const int blk1 = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
  extern __shared__ __align__(1024) uint8_t wsm[];
  uint8_t* sbase = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wsm) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[10];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_word;
  __shared__ float RMX[kWsColGroups][kGrid];
  __shared__ uint32_t CMX[4][kGrid];
  __shared__ float smax_c[kGrid];
  __shared__ __align__(16) float r7c[kGrid];
  volatile int* abort_flag = &abort_word;
  const uint32_t ops_full = tc_smem_u32(&bars[0]), ops_empty = tc_smem_u32(&bars[1]);
  auto m_full = [&](int s) { return tc_smem_u32(&bars[2 + s]); };
  auto m_empty = [&](int s) { return tc_smem_u32(&bars[4 + s]); };
  auto acc_full = [&](int a) { return tc_smem_u32(&bars[6 + a]); };
  auto acc_empty = [&](int a) { return tc_smem_u32(&bars[8 + a]); };
  const uint32_t sP = tc_smem_u32(sbase), sPlo = sP + kWsTile, sR = sP + 2 * kWsTile, sRlo = sP + 3 * kWsTile;
  auto sM = [&](int s) { return tc_smem_u32(sbase + kWsOps + s * kWsStage); };

  if (t == 0) {
    abort_word = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(ops_full) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(ops_empty) : "memory");
    for (int i = 0; i < 2; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(m_full(i)) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(m_empty(i)), "r"(kWsEpiWarps) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(acc_full(i)) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(acc_empty(i)), "r"(kWsEpiWarps) : "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     tc_smem_u32(&tmem_slot)),
                 "r"(2 * kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_slot;
  auto decode = [&](int blk, int& b, int& bi, int& bj) {
    bj = blk % nb;
    bi = (blk / nb) % mb;
    b = blk / (nb * mb);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ producer
      int pb = -1, pbi = -1;
      int j = 0, last_ops = -1, m_issued = 0;
      for (int blk = blk0; blk < blk1; ++blk, ++j) {
        int b, bi, bj;
        decode(blk, b, bi, bj);
        const int s = j & 1;
        if (j >= 2 && !ws_wait(m_empty(s), ((j >> 1) - 1) & 1, abort_flag)) break;
        ws_expect(m_full(s), kWsStage);
#pragma unroll
        for (int q = 0; q < 4; ++q) ws_tma3(sM(s) + q * kWsTile, &maps.M, m_full(s), bj * kGrid + 32 * q, bi * kGrid, b);
        m_issued = j + 1;
        if (j >= 1 && !ws_wait(ops_empty, (j - 1) & 1, abort_flag)) break;
        const bool newrow = b != pb || bi != pbi;
        ws_expect(ops_full, (newrow ? 4 : 2) * kWsTile);
        ws_tma3(sR, &maps.R, ops_full, 0, bj * kGrid, b);
        ws_tma3(sRlo, &maps.Rlo, ops_full, 0, bj * kGrid, b);
        if (newrow) {
          ws_tma3(sP, &maps.P, ops_full, 0, bi * kGrid, b);
          ws_tma3(sPlo, &maps.Plo, ops_full, 0, bi * kGrid, b);
          pb = b;
          pbi = bi;
        }
        last_ops = j;
      }
      // the copies issued last have landed before the CTA may exit (these waits do not
      // give up on an abort, only on their time limit)
      volatile int no_abort = 0;
      for (int jj = max(0, m_issued - 2); jj < m_issued; ++jj) ws_wait(m_full(jj & 1), (jj >> 1) & 1, &no_abort);
      if (last_ops >= 0) ws_wait(ops_full, last_ops & 1, &no_abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int j = 0, mma_issued = 0;
      for (int blk = blk0; blk < blk1; ++blk, ++j) {
        const int a = j & 1;
        if (j >= 2 && !ws_wait(acc_empty(a), ((j >> 1) - 1) & 1, abort_flag)) break;
        if (!ws_wait(ops_full, j & 1, abort_flag)) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t d = tmem + (uint32_t)(a * kTcTmemCols);
        const uint32_t as[3] = {sP, sP, sPlo}, bs[3] = {sR, sRlo, sR};
#pragma unroll
        for (int term = 0; term < 3; ++term)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = tc_sdesc(as[term] + 32 * kk), bd = tc_sdesc(bs[term] + 32 * kk);
            const uint32_t acc = (term | kk) ? 1u : 0u;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
                "l"(ad), "l"(bd), "r"(kTcIdesc), "r"(acc)
                : "memory");
          }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         ops_empty)
                     : "memory");
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         acc_full(a))
                     : "memory");
        mma_issued = j + 1;
      }
      // every product issued above has completed before the tensor memory is freed
      volatile int no_abort = 0;
      if (mma_issued > 0) ws_wait(acc_full((mma_issued - 1) & 1), ((mma_issued - 1) >> 1) & 1, &no_abort);
    }
  } else {
    // -------------------------------------------------- epilogue warps
    const int ew = warp - 2;
    const int quarter = warp & 3;          // TMEM lanes 32 (warp % 4) .. + 31
    const int half = ew >> 2;              // column group of the block
    const int rl = 32 * quarter + lane;    // this thread's row of the block
    const int et = ew * 32 + lane;         // 0 .. 255
    int j = 0;
    for (int blk = blk0; blk < blk1; ++blk, ++j) {
      int b, bi, bj;
      decode(blk, b, bi, bj);
      const int a = j & 1, s = j & 1;
      const int r0 = bi * kGrid, c0 = bj * kGrid, gi = r0 + rl;
      const int cbase = c0 + kWsCols * half;
      const bool row_ok = gi < m;
      bool ok = ws_wait(acc_full(a), (j >> 1) & 1, abort_flag);
      ok = ok && ws_wait(m_full(s), (j >> 1) & 1, abort_flag);
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (ws_epi_any(!ok)) break;   // leave together: the epilogue warps share named barriers
      const uint32_t tbase = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(a * kTcTmemCols + kWsCols * half);
      const uint32_t mrow = sM(s) + (uint32_t)rl * 128u;   // this row in each of the four boxes
      // sweep 1: x = M - P R^T, row and column maxima, x back into TMEM
      float rmax = 0.f;
#pragma unroll 1
      for (int ch = 0; ch < kWsChunks; ++ch) {
        __syncwarp();
        const int cl0 = kWsCols * half + 16 * ch;            // first column (in the block) of the chunk
        const uint32_t box = mrow + (uint32_t)(cl0 >> 5) * kWsTile;
        float mv[16];
#pragma unroll
        for (int pcs = 0; pcs < 4; ++pcs) {             // four 16-byte pieces of the 128-byte row
          const int piece = ((cl0 & 31) >> 2) + pcs;
          const uint32_t addr = box + (uint32_t)(((piece ^ (rl & 7)) & 7) << 4);
          float4 v;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                       : "r"(addr));
          mv[4 * pcs] = v.x; mv[4 * pcs + 1] = v.y; mv[4 * pcs + 2] = v.z; mv[4 * pcs + 3] = v.w;
        }
        float x[16];
        tc_ld16(tbase + 16 * ch, x);
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = __fsub_rn(mv[e], x[e]);
        if (!row_ok || cbase + 16 * ch >= n) {
#pragma unroll
          for (int e = 0; e < 16; ++e) x[e] = 0.f;   // rows and columns outside the matrix
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          rmax = fmaxf(rmax, fabsf(x[e]));
          uint32_t cm;
          asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(cm) : "r"(__float_as_uint(fabsf(x[e]))));
          if (lane == e) CMX[quarter][cl0 + e] = cm;
        }
        __syncwarp();
        tc_st16(tbase + 16 * ch, x);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      __syncwarp();
      if (lane == 0) ws_arrive(m_empty(s));     // this warp is done with the M stage
      RMX[half][rl] = rmax;
      ws_epi_bar();
      if (et < kGrid) {
        const uint32_t v = max(max(CMX[0][et], CMX[1][et]), max(CMX[2][et], CMX[3][et]));
        const float f = __uint_as_float(v);
        smax_c[et] = f;
        r7c[et] = f > 0.f ? __fdiv_rn(7.0f, f) : 0.f;
        if (c0 + et < n) cscale[((long long)b * mb + bi) * n + c0 + et] = f;
      }
      ws_epi_bar();
      rmax = RMX[0][rl];
#pragma unroll
      for (int h = 1; h < kWsColGroups; ++h) rmax = fmaxf(rmax, RMX[h][rl]);
      if (half == 0 && row_ok) rscale[((long long)b * m + gi) * nb + bj] = rmax;
      const float rr7 = rmax > 0.f ? __fdiv_rn(7.0f, rmax) : 0.f;
      // sweep 2: the codes
#pragma unroll 1
      for (int ch = 0; ch < kWsChunks; ++ch) {
        const int c = cbase + 16 * ch;
        float x[16];
        __syncwarp();
        tc_ld16(tbase + 16 * ch, x);
        if (row_ok && c < n) {
          // q = rint(x fl(7 / s)) away from rounding ties; |x| <= s (s is the smaller of
          // x's row and column maxima), so |q| <= 7 there without a clamp. A tie
          // candidate anywhere in the chunk sends the thread through the IEEE division
          // for those elements (rare: one branch per chunk instead of one per element).
          const int cl0 = kWsCols * half + 16 * ch;
          float r7v[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 v = reinterpret_cast<const float4*>(r7c + cl0)[u];
            r7v[4 * u] = v.x; r7v[4 * u + 1] = v.y; r7v[4 * u + 2] = v.z; r7v[4 * u + 3] = v.w;
          }
          int q[16];
          bool tie = false;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float z = __fmul_rn(x[e], fmaxf(rr7, r7v[e]));
            // rint(z) by adding and removing 1.5 * 2^23 (exact round-to-nearest-even
            // for |z| < 2^22) on the FMA pipe; the integer is the sum's low bits
            const float zm = __fadd_rn(z, 12582912.0f);
            const float zr = __fsub_rn(zm, 12582912.0f);
            q[e] = __float_as_int(zm) - 0x4B400000;
            tie |= !(fabsf(__fsub_rn(z, zr)) < 0.49998474f);   // 0.5 - 2^-16
          }
          if (tie) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float z = __fmul_rn(x[e], fmaxf(rr7, r7v[e]));
              if (!(fabsf(__fsub_rn(z, rintf(z))) < 0.49998474f)) {
                const float sv = fminf(rmax, smax_c[cl0 + e]);
                const int qq = sv > 0.f ? (int)rintf(__fmul_rn(__fdiv_rn(x[e], sv), 7.0f)) : 0;
                q[e] = max(-7, min(7, qq));
              }
            }
          }
          uint32_t w[2] = {0u, 0u};
#pragma unroll
          for (int e = 0; e < 16; ++e)
            asm("bfi.b32 %0, %1, %0, %2, 4;" : "+r"(w[e >> 3]) : "r"((uint32_t)q[e]), "r"(4 * (e & 7)));
          *reinterpret_cast<uint2*>(codes4 + ((long long)b * m + gi) * (n / 2) + c / 2) = make_uint2(w[0], w[1]);
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) ws_arrive(acc_empty(a));   // this warp is done with the accumulator
      // 8-bit codes of P's 128 rows of block row bi (in the block whose column is
      // bi mod nb) and of R's 128 rows of block column bj (in the block whose row is
      // bj mod mb): one job per block row and per block column, spread over the
      // grid instead of piling up in block row 0 of each matrix; scales, step count
      const bool pjob = bj == bi % nb, rjob = bi == bj % mb;
      if (q8.Pmax && (pjob || rjob)) {
        const int nrows = min(kGrid, m - r0), ncols = min(kGrid, n - c0);
        for (int which = 0; which < 2; ++which) {
          if (!(which == 0 ? pjob : rjob)) continue;
          const unsigned* mx = which == 0 ? q8.Pmax : q8.Rmax;
          const float* src = which == 0 ? P + ((long long)b * m + r0) * k : R + ((long long)b * n + c0) * k;
          int8_t* dst = which == 0 ? q8.P8 + ((long long)b * m + r0) * k : q8.R8 + ((long long)b * n + c0) * k;
          const int cnt = (which == 0 ? nrows : ncols) * k;
          // all of this thread's loads first (at most kQ8Per), then the codes
          float v[kQ8Per];
#pragma unroll
          for (int u = 0; u < kQ8Per; ++u) {
            const int e = et + u * kWsEpiWarps * 32;
            v[u] = e < cnt ? __ldg(src + e) : 0.f;
          }
#pragma unroll
          for (int u = 0; u < kQ8Per; ++u) {
            const int e = et + u * kWsEpiWarps * 32;
            if (e < cnt) {
              const int l = e % k;
              const float sv = __uint_as_float(__ldg(mx + b * k + l));
              const float r127 = sv > 0.f ? __fdiv_rn(127.0f, sv) : 0.f;
              dst[e] = code8(v[u], sv, r127);
            }
          }
        }
        if (bi == 0 && bj == 0 && et < k) {
          q8.Pscale[b * k + et] = __uint_as_float(q8.Pmax[b * k + et]);
          q8.Rscale[b * k + et] = __uint_as_float(q8.Rmax[b * k + et]);
        }
      }
      if (q8.step && b == 0 && bi == 0 && bj == 0 && et == 0) *q8.step += 1;
      ws_epi_bar();   // RMX, smax_c and r7c are rewritten by the next block
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kTcTmemCols)
                 : "memory");
  if (t == 0 && *abort_flag && status) atomicExch(status, (int32_t)GM_E_TIMEOUT);
}

// ------------------------------------------------------------------ S6
// blockIdx.x selects the matrix (0: X0 with rows0 rows, 1: X1), blockIdx.y the batch,
// blockIdx.z a share of the rows. Every block reduces the column absmax over all
// rows (the factors are small and L2-resident), then quantizes its share; thread
// t owns column t % k of rows t / k, t / k + 256 / k, ... (no division per element).
constexpr int kQuant8Split = 8;
__global__ void __launch_bounds__(kThreads) k_quant8(int rows0, int rows1, int k,
                                                      const float* __restrict__ X0,
                                                      int8_t* __restrict__ c0, float* __restrict__ s0,
                                                      const float* __restrict__ X1,
                                                      int8_t* __restrict__ c1, float* __restrict__ s1,
                                                      int64_t* step, const int32_t* skip) {
  if (skip && *skip) return;
  const int which = blockIdx.x, b = blockIdx.y, z = blockIdx.z, t = threadIdx.x;
  const int rows = which ? rows1 : rows0;
  const float* X = (which ? X1 : X0) + (long long)b * rows * k;
  int8_t* C = (which ? c1 : c0) + (long long)b * rows * k;
  float* S = (which ? s1 : s0) + (long long)b * k;
  __shared__ float red[kThreads];
  __shared__ float sc[kMaxK];
  const int groups = kThreads / k;
  const int l = t % k, g = t / k;
  const bool active = t < groups * k;
  float mx = 0.f;
  if (active)
    for (int i = g; i < rows; i += groups) mx = fmaxf(mx, fabsf(X[(long long)i * k + l]));
  red[t] = mx;
  __syncthreads();
  if (t < k) {
    float v = 0.f;
    for (int gg = 0; gg < groups; ++gg) v = fmaxf(v, red[gg * k + t]);
    sc[t] = v;
    if (z == 0) S[t] = v;
  }
  __syncthreads();
  const int per = cdiv(rows, kQuant8Split);
  const int i0 = z * per, i1 = min(rows, i0 + per);
  if (active) {
    const float s = sc[l];
    for (int i = i0 + g; i < i1; i += groups) {
      const long long e = (long long)i * k + l;
      int q = 0;
      if (s > 0.f) {
        q = (int)rintf(__fmul_rn(__fdiv_rn(X[e], s), 127.0f));
        q = max(-127, min(127, q));
      }
      C[e] = (int8_t)q;
    }
  }
  if (step && which == 0 && b == 0 && z == 0 && t == 0) *step += 1;
}

// ------------------------------------------------------------- NS input prep
constexpr int kPrepChunk = kThreads * 16;

__global__ void __launch_bounds__(kThreads) k_norm_partial(long long mn, const void* X, int xdt,
                                                            int nparts, double* part) {
  const int b = blockIdx.y;
  __shared__ double red[kThreads / 32];
  const long long base = (long long)b * mn;
  double acc = 0.0;
  for (long long e = (long long)blockIdx.x * kPrepChunk + threadIdx.x;
       e < min(mn, (long long)(blockIdx.x + 1) * kPrepChunk); e += kThreads) {
    const double v = load_as_float(X, base + e, xdt);
    acc += v * v;
  }
  const double s = block_sum_d(acc, red);
  if (threadIdx.x == 0) part[(long long)b * nparts + blockIdx.x] = s;
}

__global__ void k_norm_finalize(int nparts, const double* part, float eps, float* scale) {
  const int b = blockIdx.x;
  if (threadIdx.x != 0) return;
  double s = 0.0;
  for (int p = 0; p < nparts; ++p) s += part[(long long)b * nparts + p];
  scale[b] = (float)(1.0 / (sqrt(s) + (double)eps));
}

// 32 x 32 tiles through shared memory: Y (wide) = round16(scale * X).
__global__ void __launch_bounds__(kThreads) k_cast_wide(int m, int n, const void* X, int xdt,
                                                         const float* scale, uint16_t* Y, int f16) {
  const int b = blockIdx.z;
  const bool tall = m > n;
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const float sc = scale[b];
  const long long base = (long long)b * m * n;
  for (int r = ty; r < 32; r += 8) {
    const int gi = i0 + r, gj = j0 + tx;
    tile[r][tx] = (gi < m && gj < n) ? load_as_float(X, base + (long long)gi * n + gj, xdt) * sc : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    if (!tall) {
      const int gi = i0 + r, gj = j0 + tx;
      if (gi < m && gj < n) Y[base + (long long)gi * n + gj] = float_to_h16(tile[r][tx], f16);
    } else {
      const int gj = j0 + r, gi = i0 + tx;   // Y[j][i] = X[i][j]
      if (gi < m && gj < n) Y[base + (long long)gj * m + gi] = float_to_h16(tile[tx][r], f16);
    }
  }
}

template <int KP>
cudaError_t launch_backproject_t(int B, int m, int n, int k, const float* M, const uint32_t* PB,
                                 const float* scale, void* X16, bool f16, double* Rpart,
                                 float* R, uint32_t* RB, float* RT, unsigned* Rmax,
                                 const int32_t* skip, cudaStream_t s) {
  const int rs = backproject_row_splits(B, m, n);
  const size_t smem = (size_t)2 * 8 * 8 * 32 * sizeof(float4);
  static DeviceOnce attr_bf16, attr_f16;   // one latch per kernel instantiation
  {
    const cudaError_t e = f16 ? smem_attr_once(attr_f16, k_backproject<KP, true>, smem)
                              : smem_attr_once(attr_bf16, k_backproject<KP, false>, smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(cdiv(n, 64), rs, B);
  if (f16)
    k_backproject<KP, true><<<grid, kThreads, smem, s>>>(m, n, k, rs, M, PB, scale,
                                                         static_cast<uint16_t*>(X16), Rpart, skip);
  else
    k_backproject<KP, false><<<grid, kThreads, smem, s>>>(m, n, k, rs, M, PB, scale,
                                                          static_cast<uint16_t*>(X16), Rpart, skip);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((int)cdivll((long long)cdiv(n, 64) * 64 * KP, kThreads), B);
  k_finalize_r<<<g2, kThreads, 0, s>>>(n, k, rs, Rpart, R, RB, RT, Rmax, skip);
  return cudaGetLastError();
}

template <int KP, bool FR>
cudaError_t launch_residual_t(int B, int m, int n, int k, const float* X, const float* P,
                              const float* R, const uint32_t* PA, const uint32_t* RB,
                              uint8_t* codes4, float* rscale, float* cscale, const Quant8Out& q8,
                              const int32_t* skip, cudaStream_t s) {
  const size_t smem = (size_t)(2 * 8 * (KP / 8) * 2 * 128 + (FR ? 0 : 2 * kGrid * KP)) * sizeof(uint32_t);
  static DeviceOnce attr;
  if (smem > 0) {
    const cudaError_t e = smem_attr_once(attr, k_residual_quant4<KP, FR>, smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(cdiv(n, kGrid), cdiv(m, kGrid), B);
  k_residual_quant4<KP, FR><<<grid, kRT, smem, s>>>(m, n, k, X, P, R, PA, RB, codes4, rscale, cscale,
                                                    q8, skip);
  return cudaGetLastError();
}

}  // namespace

// ------------------------------------------------------------------ splits
int rebuild_row_blocks(int m) { return cdiv(m, kRB); }
int backproject_row_splits(int B, int m, int n) {
  const int ctas = cdiv(n, 64) * B;
  const int nchunks = cdiv(m, 128);
  const int need = cdiv(m, 1024);            // at most 1024 rows summed in fp32
  const int rs = max(need, cdiv(kTargetCtas, ctas));
  return max(1, min(rs, nchunks));
}
int gram_row_splits(int B, int m) {
  const int rs = cdiv(2 * kTargetCtas, B);   // about four CTAs per SM, 128 rows or more each
  return max(1, min(rs, cdiv(m, 128)));
}
int ns_prep_parts(int m, int n) { return (int)cdivll((long long)m * n, kPrepChunk); }

FactorFrags factor_frag_words(int B, int m, int n, int k) {
  const long long kp = factor_width(k), kb = kp < 16 ? 16 : kp;
  const long long np = (long long)cdiv(n, 64) * 64, bm = (long long)B * m, bn = (long long)B * np;
  FactorFrags f;
  f.QF = bn * kp * 2;
  f.RF = bn * kb / 2;
  f.PF = bm * kb * 3 / 2;
  f.PA = bm * kp * 2;
  f.RB = bn * kp * 2;
  f.PB = bm * kp * 2;
  return f;
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_warm_start(int B, int m, int n, int k, const int8_t* R8, const float* Rscale,
                              const int8_t* P8, const float* Pscale, const float* Rprev,
                              uint64_t seed, const int64_t* ids, float* Q, int* norm2_int,
                              uint32_t* QF, uint32_t* RF, uint32_t* PF, const int32_t* skip,
                              cudaStream_t s) {
  if (Rprev || !R8 || !norm2_int) {
    k_warm_start<<<B, kThreads, 0, s>>>(n, k, R8, Rscale, Rprev, seed, ids, Q, QF, skip);
    return cudaGetLastError();
  }
  cudaError_t e = cudaMemsetAsync(norm2_int, 0, sizeof(int) * (size_t)3 * B * k, s);
  if (e != cudaSuccess) return e;
  k_colnorm_int<<<dim3(cdiv(n, kThreads), B), kThreads, 0, s>>>(n, k, R8, norm2_int, skip);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int kb = kb16(factor_width(k));
  const int nbq = (int)cdivll((long long)cdiv(n, 64) * 64 * kb, kThreads * 4);
  const int nbp = (int)cdivll((long long)m * kb, kThreads * 4);
  k_warm_q<<<dim3(nbq + nbp, B), kThreads, 0, s>>>(m, n, k, nbq, R8, Rscale, P8, Pscale, norm2_int,
                                                   seed, ids, Q, QF, reinterpret_cast<uint16_t*>(RF),
                                                   reinterpret_cast<uint16_t*>(PF), skip);
  return cudaGetLastError();
}

template <int KP>
cudaError_t launch_dequant_t(int B, int m, int n, int k, const uint8_t* codes4, const float* rscale,
                             const float* cscale, const int8_t* P8, const float* Pscale,
                             const int8_t* R8, const float* Rscale, float* M, cudaStream_t s) {
  const size_t smem = (size_t)dequant_smem_words(KP) * sizeof(uint32_t);
  static DeviceOnce attr;
  {
    const cudaError_t e = smem_attr_once(attr, k_dequant_rebuild<KP>, smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(cdiv(n, kGrid), cdiv(m, kRB), B);
  k_dequant_rebuild<KP><<<grid, kRBT, smem, s>>>(m, n, k, codes4, rscale, cscale, P8, Pscale, R8, Rscale, M);
  return cudaGetLastError();
}

template <int SRC, int GDT, int KP>
cudaError_t launch_pipe_t(int B, int m, int n, cudaStream_t s, int k, const uint8_t* codes4,
                          const float* rscale, const float* cscale, const float* Mprev32, float mu,
                          const void* G, const uint32_t* QF, const uint32_t* RF, const uint32_t* PF,
                          float* M, double* norm2_part, float* Ppart, int32_t* status) {
  const size_t smem = (size_t)pipe_smem_words(SRC, GDT, KP) * sizeof(uint32_t);
  static DeviceOnce attr;
  {
    const cudaError_t e = smem_attr_once(attr, k_rebuild_pipe<SRC, GDT, KP>, smem);
    if (e != cudaSuccess) return e;
  }
  const int nb = cdiv(n, kGrid), nrb = cdiv(m, kRB);
  // tiles per CTA: up to kRebuildTiles while the grid keeps about four CTAs per SM
  const long long tiles = (long long)nb * nrb * B;
  const int per = (int)max(1LL, min((long long)kRebuildTiles, tiles / (4 * 148)));
  dim3 grid(nb, cdiv(nrb, per), B);
  k_rebuild_pipe<SRC, GDT, KP><<<grid, kRBT, smem, s>>>(m, n, k, codes4, rscale, cscale, Mprev32, mu, G,
                                                         QF, RF, PF, M, norm2_part, Ppart, status);
  return cudaGetLastError();
}

cudaError_t launch_rebuild(int B, int m, int n, int k, const uint8_t* codes4, const float* rscale,
                           const float* cscale, const int8_t* P8, const float* Pscale,
                           const int8_t* R8, const float* Rscale, const float* Mprev32, float mu,
                           const void* G, int gdt, const float* Q, const uint32_t* QF,
                           const uint32_t* RF, const uint32_t* PF, float* M, double* norm2_part,
                           float* Ppart, int32_t* status, cudaStream_t s) {
  const int kp = factor_width(k);
  const int src = codes4 ? SRC_STATE : (Mprev32 ? SRC_DENSE : SRC_ZERO);
  if (!G && !Q && src == SRC_STATE && !QF) {   // the rebuild alone, from the raw codes
    if (kp == 8) return launch_dequant_t<8>(B, m, n, k, codes4, rscale, cscale, P8, Pscale, R8, Rscale, M, s);
    if (kp == 16) return launch_dequant_t<16>(B, m, n, k, codes4, rscale, cscale, P8, Pscale, R8, Rscale, M, s);
    return launch_dequant_t<32>(B, m, n, k, codes4, rscale, cscale, P8, Pscale, R8, Rscale, M, s);
  }
  // the fused pass needs Q's fragments, and R's and P's for the stored state
  if (!Q || !QF || (src == SRC_STATE && (!RF || !PF))) return cudaErrorInvalidValue;
  const int gd = (G == nullptr) ? GM_F32 : gdt;
#define GM_RB(S, W, K) launch_pipe_t<S, W, K>(B, m, n, s, k, codes4, rscale, cscale, Mprev32, mu, G, QF, \
                                              RF, PF, M, norm2_part, Ppart, status)
#define GM_RBK(S, W) (kp == 8 ? GM_RB(S, W, 8) : (kp == 16 ? GM_RB(S, W, 16) : GM_RB(S, W, 32)))
#define GM_RBD(S) (gd == GM_F32 ? GM_RBK(S, GM_F32) : (gd == GM_BF16 ? GM_RBK(S, GM_BF16) : GM_RBK(S, GM_F16)))
  if (src == SRC_STATE) return GM_RBD(SRC_STATE);
  if (src == SRC_DENSE) return GM_RBD(SRC_DENSE);
  return GM_RBD(SRC_ZERO);
#undef GM_RBD
#undef GM_RBK
#undef GM_RB
}

cudaError_t launch_orth(int B, int m, int k, int csplit, const float* Ppart, double* Ptil,
                        double* gram_part, double* Lmat, const double* norm2_part, int ntiles,
                        float eps, float* scale, float* P, uint32_t* PB, uint32_t* PA, float* PT,
                        unsigned* Pmax, const int32_t* skip, cudaStream_t s) {
  const int rs = gram_row_splits(B, m);
  k_orth_gram<<<dim3(rs, B), kThreads, 0, s>>>(m, k, csplit, rs, Ppart, Ptil, gram_part, skip);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_orth_chol<<<B, kCholThreads, 0, s>>>(k, rs, gram_part, Lmat, norm2_part, ntiles, eps, scale, skip);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int kp = factor_width(k);
  const dim3 grid(cdiv(m, kThreads), B);
  if (kp == 8) k_orth_apply<8><<<grid, kThreads, 0, s>>>(m, k, Ptil, Lmat, P, PB, PA, PT, Pmax, skip);
  else if (kp == 16) k_orth_apply<16><<<grid, kThreads, 0, s>>>(m, k, Ptil, Lmat, P, PB, PA, PT, Pmax, skip);
  else k_orth_apply<32><<<grid, kThreads, 0, s>>>(m, k, Ptil, Lmat, P, PB, PA, PT, Pmax, skip);
  return cudaGetLastError();
}

cudaError_t launch_backproject(int B, int m, int n, int k, const float* M, const uint32_t* PB,
                               const float* scale, void* X16, bool f16, double* Rpart, float* R,
                               uint32_t* RB, float* RT, unsigned* Rmax, const int32_t* skip,
                               cudaStream_t s) {
  const int kp = factor_width(k);
  if (kp == 8) return launch_backproject_t<8>(B, m, n, k, M, PB, scale, X16, f16, Rpart, R, RB, RT, Rmax, skip, s);
  if (kp == 16) return launch_backproject_t<16>(B, m, n, k, M, PB, scale, X16, f16, Rpart, R, RB, RT, Rmax, skip, s);
  return launch_backproject_t<32>(B, m, n, k, M, PB, scale, X16, f16, Rpart, R, RB, RT, Rmax, skip, s);
}

cudaError_t launch_residual_quant4(int B, int m, int n, int k, const float* X, const float* P,
                                   const float* R, const uint32_t* PA, const uint32_t* RB,
                                   uint8_t* codes4, float* rscale, float* cscale,
                                   const unsigned* PRmax, int8_t* P8, float* Pscale, int8_t* R8,
                                   float* Rscale, int64_t* step, const int32_t* skip,
                                   cudaStream_t s) {
  const Quant8Out q8{PRmax, PRmax ? PRmax + (size_t)B * k : nullptr, P8, Pscale, R8, Rscale, step};
  if (k == 0 || !P || !R)
    return launch_residual_t<0, false>(B, m, n, 0, X, nullptr, nullptr, nullptr, nullptr, codes4,
                                       rscale, cscale, Quant8Out{}, skip, s);
  const int kp = factor_width(k);
#define GM_RQ(K, F) launch_residual_t<K, F>(B, m, n, k, X, P, R, PA, RB, codes4, rscale, cscale, q8, skip, s)
  if (PA && RB) return kp == 8 ? GM_RQ(8, true) : (kp == 16 ? GM_RQ(16, true) : GM_RQ(32, true));
  return kp == 8 ? GM_RQ(8, false) : (kp == 16 ? GM_RQ(16, false) : GM_RQ(32, false));
#undef GM_RQ
}

cudaError_t launch_codes_frags(int B, int m, int n, int k, const float* P, const float* R,
                               const unsigned* Pmax, const unsigned* Rmax, uint32_t* PA,
                               uint32_t* RB, float* PT, float* RT, const int32_t* skip,
                               cudaStream_t s) {
  const dim3 grid((unsigned)cdivll((long long)(m + n) * k, kThreads), B);
  const int kp = factor_width(k);
  if (kp == 8) k_codes_frags<8><<<grid, kThreads, 0, s>>>(m, n, k, P, R, Pmax, Rmax, PA, RB, PT, RT, skip);
  else if (kp == 16) k_codes_frags<16><<<grid, kThreads, 0, s>>>(m, n, k, P, R, Pmax, Rmax, PA, RB, PT, RT, skip);
  else k_codes_frags<32><<<grid, kThreads, 0, s>>>(m, n, k, P, R, Pmax, Rmax, PA, RB, PT, RT, skip);
  return cudaGetLastError();
}

// Tensor maps of the residual operand rows ([2][B][rows][32] fp32: hi then lo).
static bool tc_operand_maps(CUtensorMap* hi, CUtensorMap* lo, const float* base, int B, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)B};
  const cuuint64_t strides[2] = {32 * 4, (cuuint64_t)rows * 32 * 4};
  const cuuint32_t box[3] = {32, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  for (int h = 0; h < 2; ++h) {
    void* p = const_cast<float*>(base + (size_t)h * B * rows * 32);
    const CUresult r = fn(h ? lo : hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p, dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
  }
  return true;
}

cudaError_t launch_residual_ws(int B, int m, int n, int k, const float* X, const float* P,
                               const float* R, const float* PT, const float* RT, uint8_t* codes4,
                               float* rscale, float* cscale, const unsigned* PRmax, int8_t* P8,
                               float* Pscale, int8_t* R8, float* Rscale, int64_t* step,
                               const int32_t* skip, int32_t* status, cudaStream_t s) {
  ResidualWsMaps maps;
  if (!tc_operand_maps(&maps.P, &maps.Plo, PT, B, m) || !tc_operand_maps(&maps.R, &maps.Rlo, RT, B, n))
    return cudaErrorInvalidValue;
  {
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const cuuint64_t dims[3] = {(cuuint64_t)n, (cuuint64_t)m, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)n * 4, (cuuint64_t)m * n * 4};
    const cuuint32_t box[3] = {32, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&maps.M, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(X), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static DeviceOnce attr;
  {
    const cudaError_t e = smem_attr_once(attr, k_residual_ws, kWsSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const Quant8Out q8{PRmax, PRmax ? PRmax + (size_t)B * k : nullptr, P8, Pscale, R8, Rscale, step};
  const int nb = cdiv(n, kGrid), mb = cdiv(m, kGrid);
  const long long total = (long long)nb * mb * B;
  if (total > (1LL << 30)) return cudaErrorInvalidValue;
  const int grid = (int)min(total, (long long)sm_count());
  k_residual_ws<<<grid, kWsThreads, kWsSmemBytes, s>>>(maps, m, n, k, nb, mb, (int)total, P, R, codes4,
                                                       rscale, cscale, q8, skip, status);
  return cudaGetLastError();
}

cudaError_t launch_quant8(int B, int rows0, int rows1, int k, const float* X0, int8_t* c0,
                          float* s0, const float* X1, int8_t* c1, float* s1, int64_t* step,
                          const int32_t* skip, cudaStream_t s) {
  dim3 grid(X1 ? 2 : 1, B, kQuant8Split);
  k_quant8<<<grid, kThreads, 0, s>>>(rows0, rows1, k, X0, c0, s0, X1, c1, s1, step, skip);
  return cudaGetLastError();
}

cudaError_t launch_ns_prep(int B, int m, int n, const void* X, int xdt, float eps,
                           double* norm2_part, int nparts, float* scale, void* Y16, bool f16,
                           cudaStream_t s) {
  k_norm_partial<<<dim3(nparts, B), kThreads, 0, s>>>((long long)m * n, X, xdt, nparts, norm2_part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_norm_finalize<<<B, 32, 0, s>>>(nparts, norm2_part, eps, scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(n, 32), cdiv(m, 32), B);
  k_cast_wide<<<grid, kThreads, 0, s>>>(m, n, X, xdt, scale, static_cast<uint16_t*>(Y16), f16 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace gm
