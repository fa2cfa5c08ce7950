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

__device__ __forceinline__ int sext4(int v) { return (v & 0x8) ? (v | ~0xF) : (v & 0xF); }

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

// ------------------------------------------------------------------ S2
__global__ void __launch_bounds__(kThreads) k_warm_start(int n, int k, const int8_t* R8,
                                                          const float* Rscale, const float* Rprev,
                                                          uint64_t seed, float* Q,
                                                          const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.x, t = threadIdx.x;
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
  for (long long e = t; e < (long long)n * k; e += kThreads) {
    const int j = (int)(e / k), l = (int)(e % k);
    const double inv = nrm2[l];
    float q;
    if (inv == 0.0) {
      const uint64_t ctr = seed ^ ((uint64_t)b << 48) ^ ((uint64_t)j << 16) ^ (uint64_t)l;
      q = (splitmix64(ctr) >> 63) ? -rad : rad;
    } else {
      q = (float)((double)rhat(j, l) * inv);
    }
    Q[off + e] = q;
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

__global__ void __launch_bounds__(kThreads) k_warm_q(int n, int k, const int8_t* __restrict__ R8,
                                                      const float* __restrict__ Rscale,
                                                      const int* __restrict__ norm2, uint64_t seed,
                                                      float* __restrict__ Q, const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y, t = threadIdx.x;
  __shared__ double inv[kMaxK];
  if (t < k) {
    const int s2 = norm2[b * k + t];
    const float sc = Rscale[b * k + t];
    inv[t] = (s2 > 0 && sc != 0.f) ? (sc > 0.f ? 1.0 : -1.0) / sqrt((double)s2) : 0.0;
  }
  __syncthreads();
  const float rad = (float)(1.0 / sqrt((double)n));
  const long long base = (long long)blockIdx.x * kThreads * 4;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const long long e = base + u * kThreads + t;
    if (e >= (long long)n * k) break;
    const int j = (int)(e / k), l = (int)(e % k);
    const double iv = inv[l];
    float q;
    if (iv == 0.0) {
      const uint64_t ctr = seed ^ ((uint64_t)b << 48) ^ ((uint64_t)j << 16) ^ (uint64_t)l;
      q = (splitmix64(ctr) >> 63) ? -rad : rad;
    } else {
      q = (float)((double)R8[(long long)b * n * k + e] * iv);
    }
    Q[(long long)b * n * k + e] = q;
  }
}

// ------------------------------------------------------------------ S1
// One 128 x 128 grid block per CTA; thread (ty, tx) owns rows ty + 16 i and
// columns 4 tx + {0..3}, 64 + 4 tx + {0..3}.
__global__ void __launch_bounds__(kThreads) k_rebuild(
    int m, int n, int k, const uint8_t* __restrict__ codes4, const float* __restrict__ rscale,
    const float* __restrict__ cscale, const int8_t* __restrict__ P8,
    const float* __restrict__ Pscale, const int8_t* __restrict__ R8,
    const float* __restrict__ Rscale, const float* __restrict__ Mprev, float mu,
    const void* __restrict__ G, int gdt, float* __restrict__ M, double* __restrict__ norm2_part,
    int32_t* status) {
  const int bj = blockIdx.x, bi = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, mb = gridDim.y;
  const int r0 = bi * kGrid, c0 = bj * kGrid;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  __shared__ __align__(16) float Ps[kMaxK][kGrid];
  __shared__ __align__(16) float Rs[kMaxK][kGrid];
  __shared__ double red[kThreads / 32];
  const long long mn = (long long)m * n;
  const bool use_state = (codes4 != nullptr);
  const int kk = use_state ? k : 0;

  for (int e = t; e < kGrid * kk; e += kThreads) {
    const int rr = e / kk, l = e % kk;
    const int gi = r0 + rr, gj = c0 + rr;
    Ps[l][rr] = (gi < m) ? deq8(P8[((long long)b * m + gi) * kk + l], Pscale[b * kk + l]) : 0.f;
    Rs[l][rr] = (gj < n) ? deq8(R8[((long long)b * n + gj) * kk + l], Rscale[b * kk + l]) : 0.f;
  }
  __syncthreads();

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int l = 0; l < kk; ++l) {
    const float4 ra = *reinterpret_cast<const float4*>(&Rs[l][4 * tx]);
    const float4 rb = *reinterpret_cast<const float4*>(&Rs[l][64 + 4 * tx]);
    const float rv[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float p = Ps[l][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(p, rv[j], acc[i][j]);
    }
  }

  float cs[8];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int gj = c0 + 64 * h + 4 * tx + e;
      cs[4 * h + e] = (use_state && gj < n) ? cscale[((long long)b * mb + bi) * n + gj] : 0.f;
    }

  float nsq = 0.f;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gi = r0 + ty + 16 * i;
    if (gi >= m) continue;
    const float rsc = use_state ? rscale[((long long)b * m + gi) * nb + bj] : 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cb = c0 + 64 * h + 4 * tx;
      if (cb >= n) continue;
      const long long base = (long long)b * mn + (long long)gi * n + cb;
      float mp[4];
      if (use_state) {
        const uint16_t two = *reinterpret_cast<const uint16_t*>(
            codes4 + ((long long)b * m + gi) * (n / 2) + cb / 2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = sext4((two >> (4 * e)) & 0xF);
          const float s = fminf(rsc, cs[4 * h + e]);
          mp[e] = __fmul_rn(__fdiv_rn((float)q, 7.0f), s) + acc[i][4 * h + e];
        }
      } else if (Mprev) {
        const float4 v = *reinterpret_cast<const float4*>(Mprev + base);
        mp[0] = v.x; mp[1] = v.y; mp[2] = v.z; mp[3] = v.w;
      } else {
        mp[0] = mp[1] = mp[2] = mp[3] = 0.f;
      }
      float g[4] = {0.f, 0.f, 0.f, 0.f};
      if (G) {
        if (gdt == GM_F32) {
          const float4 v = *reinterpret_cast<const float4*>(static_cast<const float*>(G) + base);
          g[0] = v.x; g[1] = v.y; g[2] = v.z; g[3] = v.w;
        } else {
          const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(G) + base);
          const bool f16 = (gdt == GM_F16);
          g[0] = h16_to_float(raw.x & 0xFFFF, f16);
          g[1] = h16_to_float(raw.x >> 16, f16);
          g[2] = h16_to_float(raw.y & 0xFFFF, f16);
          g[3] = h16_to_float(raw.y >> 16, f16);
        }
      }
      float4 o;
      float* ov = &o.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v = __fadd_rn(__fmul_rn(mu, mp[e]), g[e]);
        ov[e] = v;
        bad |= !isfinite(v);
        nsq = fmaf(v, v, nsq);
      }
      *reinterpret_cast<float4*>(M + base) = o;
    }
  }
  const double tot = block_sum_d((double)nsq, red);
  if (t == 0 && norm2_part) norm2_part[((long long)b * mb + bi) * nb + bj] = tot;
  if (bad && status) atomicExch(status, GM_E_NONFINITE);
}

// ------------------------------------------------------------------ S3
// P~ = M Q. CTA: 64 rows x a contiguous range of 128-column chunks. Thread
// (rg, lg, jg) owns rows rg + 16 r (r < 4), columns l = 8 lg + {0..7} of P~
// and the j-slice jg of every chunk; fp32 within a chunk, fp64 across chunks.
template <int KP>
__global__ void __launch_bounds__(kThreads) k_project(int m, int n, int k, int csplit,
                                                       const float* __restrict__ M,
                                                       const float* __restrict__ Q,
                                                       double* __restrict__ Ppart,
                                                       const int32_t* skip) {
  if (skip && *skip) return;
  constexpr int RB = 64, CH = 128, LG = KP / 8, JG = kThreads / (16 * LG), JPER = CH / JG;
  constexpr int MS = CH + 1;   // odd row stride: conflict-free column reads
  extern __shared__ __align__(16) float smem[];   // RB * MS + CH * KP floats
  float* Ms = smem;
  float* Qs = smem + RB * MS;
  const int rb = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, rg = t & 15, lg = (t >> 4) % LG, jg = t / (16 * LG);
  const int r0 = rb * RB;
  const int nchunks = cdiv(n, CH);
  const int per = cdiv(nchunks, csplit);
  const int ch0 = split * per, ch1 = min(nchunks, ch0 + per);
  const float* Mb = M + (long long)b * m * n;
  const float* Qb = Q + (long long)b * n * k;

  double accd[4][8];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int l = 0; l < 8; ++l) accd[r][l] = 0.0;

  for (int ch = ch0; ch < ch1; ++ch) {
    const int c0 = ch * CH;
    for (int e = t; e < RB * (CH / 4); e += kThreads) {
      const int rr = e / (CH / 4), q4 = e % (CH / 4);
      const int gi = r0 + rr, gj = c0 + 4 * q4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gi < m && gj < n) v = *reinterpret_cast<const float4*>(Mb + (long long)gi * n + gj);
      float* d = Ms + rr * MS + 4 * q4;
      d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
    }
    for (int e = t; e < CH * KP; e += kThreads) {
      const int jj = e / KP, l = e % KP;
      const int gj = c0 + jj;
      Qs[e] = (gj < n && l < k) ? Qb[(long long)gj * k + l] : 0.f;
    }
    __syncthreads();
    float accf[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int l = 0; l < 8; ++l) accf[r][l] = 0.f;
#pragma unroll 4
    for (int jj = 0; jj < JPER; ++jj) {
      const int j = jg * JPER + jj;
      const float4 qa = *reinterpret_cast<const float4*>(Qs + j * KP + 8 * lg);
      const float4 qb = *reinterpret_cast<const float4*>(Qs + j * KP + 8 * lg + 4);
      const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float mv = Ms[(rg + 16 * r) * MS + j];
#pragma unroll
        for (int l = 0; l < 8; ++l) accf[r][l] = fmaf(mv, qv[l], accf[r][l]);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int l = 0; l < 8; ++l) accd[r][l] += (double)accf[r][l];
    __syncthreads();
  }
  // Ordered reduction over the j-groups, reusing the tile buffer.
  double* red = reinterpret_cast<double*>(smem);   // RB * KP doubles <= smem size
  for (int g = JG - 1; g >= 0; --g) {
    if (jg == g) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int l = 0; l < 8; ++l) {
          double* slot = red + (rg + 16 * r) * KP + 8 * lg + l;
          *slot = (g == JG - 1) ? accd[r][l] : (*slot + accd[r][l]);
        }
    }
    __syncthreads();
  }
  double* out = Ppart + ((long long)b * csplit + split) * m * k;
  for (int e = t; e < RB * k; e += kThreads) {
    const int rr = e / k, l = e % k;
    if (r0 + rr < m) out[(long long)(r0 + rr) * k + l] = red[rr * KP + l];
  }
}

// ------------------------------------------------------------------ S4
// (a) P~ = sum of column-split partials (fixed order); partial Gram P~^T P~.
__global__ void __launch_bounds__(kThreads) k_orth_gram(int m, int k, int csplit, int rsplit,
                                                         const double* __restrict__ Ppart,
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
        for (int s = 0; s < csplit; ++s) v += Ppart[(((long long)b * csplit + s) * m + gi) * k + l];
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

// (b) Cholesky of the Gram with dead-column exclusion; T = L^-T; NS scale.
__global__ void __launch_bounds__(32) k_orth_chol(int k, int rsplit, const double* __restrict__ gram_part,
                                                   double* __restrict__ Tmat,
                                                   const double* __restrict__ norm2_part, int ntiles,
                                                   float eps, float* __restrict__ scale,
                                                   const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.x, lane = threadIdx.x;
  __shared__ double G[kMaxK][kMaxK + 1];
  __shared__ double L[kMaxK][kMaxK + 1];
  __shared__ double Li[kMaxK][kMaxK + 1];
  __shared__ int live[kMaxK];
  for (int e = lane; e < k * k; e += 32) {
    double s = 0.0;
    for (int p = 0; p < rsplit; ++p) s += gram_part[((long long)b * rsplit + p) * k * k + e];
    G[e / k][e % k] = s;
    L[e / k][e % k] = 0.0;
    Li[e / k][e % k] = 0.0;
  }
  __syncwarp();
  double maxn2 = 0.0;
  for (int l = 0; l < k; ++l) maxn2 = fmax(maxn2, G[l][l]);
  const double tol2 = 1e-12 * maxn2;   // (1e-6 * max column norm)^2
  for (int j = 0; j < k; ++j) {
    double d = G[j][j];
    for (int l = 0; l < j; ++l) d -= L[j][l] * L[j][l];   // dead columns hold zeros
    const bool alive = (d > tol2) && (d > 0.0);
    const double ljj = alive ? sqrt(d) : 0.0;
    __syncwarp();
    if (lane == 0) { live[j] = alive; L[j][j] = ljj; }
    for (int i = j + 1 + lane; i < k; i += 32) {
      double v = 0.0;
      if (alive) {
        v = G[i][j];
        for (int l = 0; l < j; ++l) v -= L[i][l] * L[j][l];
        v /= ljj;
      }
      L[i][j] = v;
    }
    __syncwarp();
  }
  // Li = L^-1 on the live columns (forward substitution, one column per lane).
  for (int c = lane; c < k; c += 32) {
    if (!live[c]) continue;
    for (int i = c; i < k; ++i) {
      if (!live[i]) continue;
      double v = (i == c) ? 1.0 : 0.0;
      for (int l = c; l < i; ++l) v -= L[i][l] * Li[l][c];
      Li[i][c] = v / L[i][i];
    }
  }
  __syncwarp();
  for (int e = lane; e < k * k; e += 32) {
    const int a = e / k, c = e % k;
    Tmat[(long long)b * k * k + e] = Li[c][a];   // T = L^-T
  }
  if (lane == 0 && scale) {
    double s = 0.0;
    for (int p = 0; p < ntiles; ++p) s += norm2_part[(long long)b * ntiles + p];
    scale[b] = (float)(1.0 / (sqrt(s) + (double)eps));
  }
}

// (c) P = P~ T (fp64), stored fp32.
__global__ void __launch_bounds__(kThreads) k_orth_apply(int m, int k, const double* __restrict__ Ptil,
                                                          const double* __restrict__ Tmat,
                                                          float* __restrict__ P,
                                                          const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y, t = threadIdx.x;
  __shared__ double Ts[kMaxK][kMaxK];
  for (int e = t; e < k * k; e += kThreads) Ts[e / k][e % k] = Tmat[(long long)b * k * k + e];
  __syncthreads();
  const long long base = (long long)blockIdx.x * kThreads * 4;
  for (int s = 0; s < 4; ++s) {
    const long long e = base + s * kThreads + t;
    if (e >= (long long)m * k) break;
    const long long i = e / k;
    const int l = (int)(e % k);
    const double* row = Ptil + ((long long)b * m + i) * k;
    double v = 0.0;
    for (int a = 0; a <= l; ++a) v = fma(row[a], Ts[a][l], v);   // T upper triangular
    P[(long long)b * m * k + e] = (float)v;
  }
}

// ------------------------------------------------------------------ S5
// R = M^T P over row splits (fp64 partials), and the normalised wide-form NS
// input X = round16(scale * M) (X = M^T when m > n).
template <int KP>
__global__ void __launch_bounds__(kThreads) k_backproject(int m, int n, int k, int rsplit,
                                                           const float* __restrict__ M,
                                                           const float* __restrict__ P,
                                                           const float* __restrict__ scale,
                                                           uint16_t* __restrict__ X16, int f16,
                                                           double* __restrict__ Rpart,
                                                           const int32_t* skip) {
  if (skip && *skip) return;
  constexpr int CB = 64, CH = 128, LG = KP / 8, IG = kThreads / (16 * LG), IPER = CH / IG;
  constexpr int MS = CB + 1;
  extern __shared__ __align__(16) float smem[];   // CH * MS + CH * KP floats
  float* Ms = smem;
  float* Ps = smem + CH * MS;
  const int cbk = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, cg = t & 15, lg = (t >> 4) % LG, ig = t / (16 * LG);
  const int c0 = cbk * CB;
  const int nchunks = cdiv(m, CH);
  const int per = cdiv(nchunks, rsplit);
  const int ch0 = split * per, ch1 = min(nchunks, ch0 + per);
  const float* Mb = M + (long long)b * m * n;
  const float* Pb = P + (long long)b * m * k;
  const float sc = X16 ? scale[b] : 0.f;
  const bool tall = m > n;
  uint16_t* Xb = X16 ? X16 + (long long)b * m * n : nullptr;

  double accd[4][8];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int l = 0; l < 8; ++l) accd[c][l] = 0.0;

  for (int ch = ch0; ch < ch1; ++ch) {
    const int i0 = ch * CH;
    for (int e = t; e < CH * (CB / 4); e += kThreads) {
      const int ii = e / (CB / 4), q4 = e % (CB / 4);
      const int gi = i0 + ii, gj = c0 + 4 * q4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      const bool ok = gi < m && gj < n;
      if (ok) v = *reinterpret_cast<const float4*>(Mb + (long long)gi * n + gj);
      float* d = Ms + ii * MS + 4 * q4;
      d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
      if (Xb && ok && !tall) {
        const float xv[4] = {v.x * sc, v.y * sc, v.z * sc, v.w * sc};
        uint2 pk;
        pk.x = (uint32_t)float_to_h16(xv[0], f16) | ((uint32_t)float_to_h16(xv[1], f16) << 16);
        pk.y = (uint32_t)float_to_h16(xv[2], f16) | ((uint32_t)float_to_h16(xv[3], f16) << 16);
        *reinterpret_cast<uint2*>(Xb + (long long)gi * n + gj) = pk;
      }
    }
    for (int e = t; e < CH * KP; e += kThreads) {
      const int ii = e / KP, l = e % KP, gi = i0 + ii;
      Ps[e] = (gi < m && l < k) ? Pb[(long long)gi * k + l] : 0.f;
    }
    __syncthreads();
    if (Xb && tall) {
      // X[j][i] = M[i][j]: consecutive threads take consecutive i.
      for (int e = t; e < CH * CB; e += kThreads) {
        const int ii = e % CH, jj = e / CH;
        const int gi = i0 + ii, gj = c0 + jj;
        if (gi < m && gj < n)
          Xb[(long long)gj * m + gi] = float_to_h16(Ms[ii * MS + jj] * sc, f16);
      }
    }
    float accf[4][8];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int l = 0; l < 8; ++l) accf[c][l] = 0.f;
#pragma unroll 4
    for (int ii = 0; ii < IPER; ++ii) {
      const int i = ig * IPER + ii;
      const float4 pa = *reinterpret_cast<const float4*>(Ps + i * KP + 8 * lg);
      const float4 pb = *reinterpret_cast<const float4*>(Ps + i * KP + 8 * lg + 4);
      const float pv[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float mv = Ms[i * MS + cg + 16 * c];
#pragma unroll
        for (int l = 0; l < 8; ++l) accf[c][l] = fmaf(mv, pv[l], accf[c][l]);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int l = 0; l < 8; ++l) accd[c][l] += (double)accf[c][l];
    __syncthreads();
  }
  double* red = reinterpret_cast<double*>(smem);   // CB * KP doubles
  for (int g = IG - 1; g >= 0; --g) {
    if (ig == g) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int l = 0; l < 8; ++l) {
          double* slot = red + (cg + 16 * c) * KP + 8 * lg + l;
          *slot = (g == IG - 1) ? accd[c][l] : (*slot + accd[c][l]);
        }
    }
    __syncthreads();
  }
  double* out = Rpart + ((long long)b * rsplit + split) * n * k;
  for (int e = t; e < CB * k; e += kThreads) {
    const int cc = e / k, l = e % k;
    if (c0 + cc < n) out[(long long)(c0 + cc) * k + l] = red[cc * KP + l];
  }
}

__global__ void __launch_bounds__(kThreads) k_finalize_r(int n, int k, int rsplit,
                                                          const double* __restrict__ Rpart,
                                                          float* __restrict__ R,
                                                          const int32_t* skip) {
  if (skip && *skip) return;
  const int b = blockIdx.y;
  const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (e >= (long long)n * k) return;
  double s = 0.0;
  for (int p = 0; p < rsplit; ++p) s += Rpart[((long long)b * rsplit + p) * n * k + e];
  R[(long long)b * n * k + e] = (float)s;
}

// ------------------------------------------------------------------ S7
__global__ void __launch_bounds__(kThreads) k_residual_quant4(
    int m, int n, int k, const float* __restrict__ X, const float* __restrict__ P,
    const float* __restrict__ R, uint8_t* __restrict__ codes4, float* __restrict__ rscale,
    float* __restrict__ cscale, const int32_t* skip) {
  if (skip && *skip) return;
  const int bj = blockIdx.x, bi = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, mb = gridDim.y;
  const int r0 = bi * kGrid, c0 = bj * kGrid;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  __shared__ __align__(16) float Ps[kMaxK][kGrid];
  __shared__ __align__(16) float Rs[kMaxK][kGrid];
  __shared__ float cm[16][kGrid];
  __shared__ float cmax[kGrid];
  const int kk = (P && R) ? k : 0;
  for (int e = t; e < kGrid * kk; e += kThreads) {
    const int rr = e / kk, l = e % kk;
    const int gi = r0 + rr, gj = c0 + rr;
    Ps[l][rr] = (gi < m) ? P[((long long)b * m + gi) * kk + l] : 0.f;
    Rs[l][rr] = (gj < n) ? R[((long long)b * n + gj) * kk + l] : 0.f;
  }
  __syncthreads();
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int l = 0; l < kk; ++l) {
    const float4 ra = *reinterpret_cast<const float4*>(&Rs[l][4 * tx]);
    const float4 rb = *reinterpret_cast<const float4*>(&Rs[l][64 + 4 * tx]);
    const float rv[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float p = Ps[l][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(p, rv[j], acc[i][j]);
    }
  }
  // x = M - P R^T in registers (zero outside the matrix).
  float x[8][8];
  float cmx[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) cmx[j] = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gi = r0 + ty + 16 * i;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cb = c0 + 64 * h + 4 * tx;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gi < m && cb < n) v = *reinterpret_cast<const float4*>(X + ((long long)b * m + gi) * n + cb);
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float r = (gi < m && cb < n) ? __fsub_rn(vv[e], acc[i][4 * h + e]) : 0.f;
        x[i][4 * h + e] = r;
        cmx[4 * h + e] = fmaxf(cmx[4 * h + e], fabsf(r));
      }
    }
  }
  // column absmax: per-thread over its 8 rows, then over the 16 row groups
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) cm[ty][64 * h + 4 * tx + e] = cmx[4 * h + e];
  __syncthreads();
  if (t < kGrid) {
    float v = 0.f;
    for (int g = 0; g < 16; ++g) v = fmaxf(v, cm[g][t]);
    cmax[t] = v;
    if (c0 + t < n) cscale[((long long)b * mb + bi) * n + c0 + t] = v;
  }
  __syncthreads();
  float cs[8];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[4 * h + e] = cmax[64 * h + 4 * tx + e];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gi = r0 + ty + 16 * i;
    float rmx = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) rmx = fmaxf(rmx, fabsf(x[i][j]));
    // the 16 threads of a row are lanes 16*(ty&1) .. +15 of one warp
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) rmx = fmaxf(rmx, __shfl_xor_sync(0xffffffffu, rmx, o));
    if (gi >= m) continue;
    if (tx == 0) rscale[((long long)b * m + gi) * nb + bj] = rmx;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cb = c0 + 64 * h + 4 * tx;
      if (cb >= n) continue;
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float s = fminf(rmx, cs[4 * h + e]);
        int q = 0;
        if (s > 0.f) {
          const float r = __fmul_rn(__fdiv_rn(x[i][4 * h + e], s), 7.0f);
          q = (int)rintf(r);
          q = max(-7, min(7, q));
        }
        packed |= (uint32_t)(q & 0xF) << (4 * e);
      }
      *reinterpret_cast<uint16_t*>(codes4 + ((long long)b * m + gi) * (n / 2) + cb / 2) =
          (uint16_t)packed;
    }
  }
}

// ------------------------------------------------------------------ S6
// blockIdx.x selects the matrix (0: X0 with rows0 rows, 1: X1), blockIdx.y the batch.
__global__ void __launch_bounds__(kThreads) k_quant8(int rows0, int rows1, int k,
                                                      const float* __restrict__ X0,
                                                      int8_t* __restrict__ c0, float* __restrict__ s0,
                                                      const float* __restrict__ X1,
                                                      int8_t* __restrict__ c1, float* __restrict__ s1,
                                                      int64_t* step, const int32_t* skip) {
  if (skip && *skip) return;
  const int which = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int rows = which ? rows1 : rows0;
  const float* X = (which ? X1 : X0) + (long long)b * rows * k;
  int8_t* C = (which ? c1 : c0) + (long long)b * rows * k;
  float* S = (which ? s1 : s0) + (long long)b * k;
  __shared__ float red[kThreads];
  __shared__ float sc[kMaxK];
  const int groups = kThreads / k;
  float mx = 0.f;
  if (t < groups * k) {
    const int l = t % k, g = t / k;
    for (int i = g; i < rows; i += groups) mx = fmaxf(mx, fabsf(X[(long long)i * k + l]));
  }
  red[t] = mx;
  __syncthreads();
  if (t < k) {
    float v = 0.f;
    for (int g = 0; g < groups; ++g) v = fmaxf(v, red[g * k + t]);
    sc[t] = v;
    S[t] = v;
  }
  __syncthreads();
  for (long long e = t; e < (long long)rows * k; e += kThreads) {
    const int l = (int)(e % k);
    const float s = sc[l];
    int q = 0;
    if (s > 0.f) {
      q = (int)rintf(__fmul_rn(__fdiv_rn(X[e], s), 127.0f));
      q = max(-127, min(127, q));
    }
    C[e] = (int8_t)q;
  }
  if (step && which == 0 && b == 0 && t == 0) *step += 1;
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
cudaError_t launch_project_t(int B, int m, int n, int k, const float* M, const float* Q,
                             double* Ppart, const int32_t* skip, cudaStream_t s) {
  const int cs = project_col_splits(B, m, n);
  const size_t smem = (size_t)(64 * 129 + 128 * KP) * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_project<KP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid(cdiv(m, 64), cs, B);
  k_project<KP><<<grid, kThreads, smem, s>>>(m, n, k, cs, M, Q, Ppart, skip);
  return cudaGetLastError();
}

template <int KP>
cudaError_t launch_backproject_t(int B, int m, int n, int k, const float* M, const float* P,
                                 const float* scale, void* X16, bool f16, double* Rpart,
                                 float* R, const int32_t* skip, cudaStream_t s) {
  const int rs = backproject_row_splits(B, m, n);
  const size_t smem = (size_t)(128 * 65 + 128 * KP) * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_backproject<KP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid(cdiv(n, 64), rs, B);
  k_backproject<KP><<<grid, kThreads, smem, s>>>(m, n, k, rs, M, P, scale,
                                              static_cast<uint16_t*>(X16), f16 ? 1 : 0, Rpart,
                                              skip);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(cdiv(n * k, kThreads), B);
  k_finalize_r<<<g2, kThreads, 0, s>>>(n, k, rs, Rpart, R, skip);
  return cudaGetLastError();
}

}  // namespace

// ------------------------------------------------------------------ splits
int project_col_splits(int B, int m, int n) {
  const int ctas = cdiv(m, 64) * B;
  const int nchunks = cdiv(n, 128);
  int cs = cdiv(kTargetCtas, ctas);
  return max(1, min(cs, nchunks));
}
int backproject_row_splits(int B, int m, int n) {
  const int ctas = cdiv(n, 64) * B;
  const int nchunks = cdiv(m, 128);
  int rs = cdiv(kTargetCtas, ctas);
  return max(1, min(rs, nchunks));
}
int gram_row_splits(int B, int m) {
  int rs = cdiv(kTargetCtas, B);
  return max(1, min(rs, cdiv(m, 256)));
}
int ns_prep_parts(int m, int n) { return (int)cdivll((long long)m * n, kPrepChunk); }

// ---------------------------------------------------------------- launchers
cudaError_t launch_warm_start(int B, int n, int k, const int8_t* R8, const float* Rscale,
                              const float* Rprev, uint64_t seed, float* Q, int* norm2_int,
                              const int32_t* skip, cudaStream_t s) {
  if (Rprev || !R8 || !norm2_int) {
    k_warm_start<<<B, kThreads, 0, s>>>(n, k, R8, Rscale, Rprev, seed, Q, skip);
    return cudaGetLastError();
  }
  cudaError_t e = cudaMemsetAsync(norm2_int, 0, sizeof(int) * (size_t)B * k, s);
  if (e != cudaSuccess) return e;
  k_colnorm_int<<<dim3(cdiv(n, kThreads), B), kThreads, 0, s>>>(n, k, R8, norm2_int, skip);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_warm_q<<<dim3((int)cdivll((long long)n * k, kThreads * 4), B), kThreads, 0, s>>>(
      n, k, R8, Rscale, norm2_int, seed, Q, skip);
  return cudaGetLastError();
}

cudaError_t launch_rebuild(int B, int m, int n, int k, const uint8_t* codes4, const float* rscale,
                           const float* cscale, const int8_t* P8, const float* Pscale,
                           const int8_t* R8, const float* Rscale, const float* Mprev32, float mu,
                           const void* G, int gdt, float* M, double* norm2_part, int32_t* status,
                           cudaStream_t s) {
  dim3 grid(cdiv(n, kGrid), cdiv(m, kGrid), B);
  k_rebuild<<<grid, kThreads, 0, s>>>(m, n, k, codes4, rscale, cscale, P8, Pscale, R8, Rscale,
                                      Mprev32, mu, G, gdt, M, norm2_part, status);
  return cudaGetLastError();
}

cudaError_t launch_project(int B, int m, int n, int k, const float* M, const float* Q,
                           double* Ppart, const int32_t* skip, cudaStream_t s) {
  if (k <= 8) return launch_project_t<8>(B, m, n, k, M, Q, Ppart, skip, s);
  if (k <= 16) return launch_project_t<16>(B, m, n, k, M, Q, Ppart, skip, s);
  return launch_project_t<32>(B, m, n, k, M, Q, Ppart, skip, s);
}

cudaError_t launch_orth(int B, int m, int k, int csplit, const double* Ppart, double* Ptil,
                        double* gram_part, double* Tmat, const double* norm2_part, int ntiles,
                        float eps, float* scale, float* P, const int32_t* skip, cudaStream_t s) {
  const int rs = gram_row_splits(B, m);
  k_orth_gram<<<dim3(rs, B), kThreads, 0, s>>>(m, k, csplit, rs, Ppart, Ptil, gram_part, skip);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_orth_chol<<<B, 32, 0, s>>>(k, rs, gram_part, Tmat, norm2_part, ntiles, eps, scale, skip);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int blocks = (int)cdivll((long long)m * k, kThreads * 4);
  k_orth_apply<<<dim3(blocks, B), kThreads, 0, s>>>(m, k, Ptil, Tmat, P, skip);
  return cudaGetLastError();
}

cudaError_t launch_backproject(int B, int m, int n, int k, const float* M, const float* P,
                               const float* scale, void* X16, bool f16, double* Rpart, float* R,
                               const int32_t* skip, cudaStream_t s) {
  if (k <= 8) return launch_backproject_t<8>(B, m, n, k, M, P, scale, X16, f16, Rpart, R, skip, s);
  if (k <= 16) return launch_backproject_t<16>(B, m, n, k, M, P, scale, X16, f16, Rpart, R, skip, s);
  return launch_backproject_t<32>(B, m, n, k, M, P, scale, X16, f16, Rpart, R, skip, s);
}

cudaError_t launch_residual_quant4(int B, int m, int n, int k, const float* X, const float* P,
                                   const float* R, uint8_t* codes4, float* rscale, float* cscale,
                                   const int32_t* skip, cudaStream_t s) {
  dim3 grid(cdiv(n, kGrid), cdiv(m, kGrid), B);
  k_residual_quant4<<<grid, kThreads, 0, s>>>(m, n, k, X, P, R, codes4, rscale, cscale, skip);
  return cudaGetLastError();
}

cudaError_t launch_quant8(int B, int rows0, int rows1, int k, const float* X0, int8_t* c0,
                          float* s0, const float* X1, int8_t* c1, float* s1, int64_t* step,
                          const int32_t* skip, cudaStream_t s) {
  dim3 grid(X1 ? 2 : 1, B);
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
