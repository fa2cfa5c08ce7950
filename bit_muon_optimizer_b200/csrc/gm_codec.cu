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

// ------------------------------------------------------------------ S1 + S3
// Rebuild + momentum, fused with the projection P~ = M Q.
// CTA: 64 rows x 128 columns (half a grid block); thread (ty, tx) owns rows
// ty + 16 i (i < 4) and columns 4 tx + {0..3}, 64 + 4 tx + {0..3}.
// Global loads of the tile are issued before the rank-k product. The decoded
// nibble value q / 7 comes from a 16-entry table filled with IEEE divisions, so it
// is bit-identical to (float)q / 7.0f. P~ partials of the tile (sum over its 128
// columns, fp32) go to Ppart[b][bj][row][l]; the orthonormalisation sums the
// column blocks in fp64 in a fixed order.
constexpr int kRB = 64;   // rows per rebuild CTA

__device__ __forceinline__ void reduce_scatter16(float (&v)[16], int tx) {
  // After the four steps lane tx (of a 16-lane group) holds the group sum of v[tx].
#pragma unroll
  for (int s = 8; s >= 1; s >>= 1) {
    const bool up = (tx & s) != 0;
#pragma unroll
    for (int j = 0; j < s; ++j) {
      const float send = up ? v[j] : v[j + s];
      const float keep = up ? v[j + s] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
}

enum RebuildSrc { SRC_STATE = 0, SRC_DENSE = 1, SRC_ZERO = 2 };

// KP: the factor width k rounded up to 8, 16 or 32 (columns beyond k are zero).
template <int SRC, bool G32, int KP>
__global__ void __launch_bounds__(kThreads, 2) k_rebuild_proj(
    int m, int n, int k, const uint8_t* __restrict__ codes4, const float* __restrict__ rscale,
    const float* __restrict__ cscale, const int8_t* __restrict__ P8,
    const float* __restrict__ Pscale, const int8_t* __restrict__ R8,
    const float* __restrict__ Rscale, const float* __restrict__ Mprev, float mu,
    const void* __restrict__ G, int gdt, const float* __restrict__ Q, float* __restrict__ M,
    double* __restrict__ norm2_part, float* __restrict__ Ppart, int32_t* status) {
  const int bj = blockIdx.x, bh = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x;
  const int mb = cdiv(m, kGrid);
  const int r0 = bh * kRB, c0 = bj * kGrid, bi = r0 / kGrid;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  constexpr int KK = SRC == SRC_STATE ? KP : 0;
  extern __shared__ __align__(16) float sm[];
  float* Ps = sm;                  // [KK][64]
  float* Rs = Ps + KK * kRB;       // [KK][128]
  float* Qs = Rs + KK * kGrid;     // [KP][128] (with Q)
  __shared__ float deq4[16];
  __shared__ double red[kThreads / 32];
  const long long mn = (long long)m * n;
  const bool f16 = gdt == GM_F16;

  // 1. global loads of this thread's 32 elements, all issued up front
  uint32_t cw[4][2];      // four nibbles per (row, half)
  float4 mpv[4][2];       // dense M_prev
  uint2 gw[4][2];         // 16-bit gradient
  float4 gf[4][2];        // fp32 gradient
  float rsc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gi = r0 + ty + 16 * i;
    if (SRC == SRC_STATE) rsc[i] = gi < m ? rscale[((long long)b * m + gi) * nb + bj] : 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cb = c0 + 64 * h + 4 * tx;
      const bool ok = gi < m && cb < n;
      const long long base = (long long)b * mn + (long long)gi * n + cb;
      if (SRC == SRC_STATE)
        cw[i][h] = ok ? *reinterpret_cast<const uint16_t*>(codes4 + ((long long)b * m + gi) * (n / 2) + cb / 2) : 0u;
      if (SRC == SRC_DENSE)
        mpv[i][h] = ok ? *reinterpret_cast<const float4*>(Mprev + base) : make_float4(0.f, 0.f, 0.f, 0.f);
      if (G32) gf[i][h] = (ok && G) ? *reinterpret_cast<const float4*>(static_cast<const float*>(G) + base)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      else gw[i][h] = (ok && G) ? *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(G) + base)
                                : make_uint2(0u, 0u);
    }
  }
  float cs[8];
  if (SRC == SRC_STATE) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gj = c0 + 64 * h + 4 * tx + e;
        cs[4 * h + e] = gj < n ? cscale[((long long)b * mb + bi) * n + gj] : 0.f;
      }
  }

  // 2. factors of the tile into shared memory
  if (t < 16) deq4[t] = __fdiv_rn((float)((t & 8) ? t - 16 : t), 7.0f);
  if constexpr (SRC == SRC_STATE) {
#pragma unroll 4
    for (int e = t; e < kRB * KK; e += kThreads) {
      const int rr = e / KK, l = e % KK, gi = r0 + rr;
      Ps[l * kRB + rr] = (gi < m && l < k) ? deq8(P8[((long long)b * m + gi) * k + l], Pscale[b * k + l]) : 0.f;
    }
#pragma unroll 4
    for (int e = t; e < kGrid * KK; e += kThreads) {
      const int cc = e / KK, l = e % KK, gj = c0 + cc;
      Rs[l * kGrid + cc] = (gj < n && l < k) ? deq8(R8[((long long)b * n + gj) * k + l], Rscale[b * k + l]) : 0.f;
    }
  }
  if (Q) {
#pragma unroll 4
    for (int e = t; e < kGrid * KP; e += kThreads) {
      const int cc = e / KP, l = e % KP, gj = c0 + cc;
      Qs[l * kGrid + cc] = (gj < n && l < k) ? Q[((long long)b * n + gj) * k + l] : 0.f;
    }
  }
  __syncthreads();

  // 3. rank-k rebuild P^ R^T
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 4
  for (int l = 0; l < KK; ++l) {
    const float4 ra = *reinterpret_cast<const float4*>(Rs + l * kGrid + 4 * tx);
    const float4 rb = *reinterpret_cast<const float4*>(Rs + l * kGrid + 64 + 4 * tx);
    const float rv[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float pv = Ps[l * kRB + ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(pv, rv[j], acc[i][j]);
    }
  }

  // 4. M = mu M_prev + G, with M_prev = deq4 + P^R^T (state) or dense
  float nsq = 0.f;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gi = r0 + ty + 16 * i;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cb = c0 + 64 * h + 4 * tx;
      const bool ok = gi < m && cb < n;
      float g[4], mp[4];
      if (G32) {
        g[0] = gf[i][h].x; g[1] = gf[i][h].y; g[2] = gf[i][h].z; g[3] = gf[i][h].w;
      } else {
        g[0] = h16_to_float(gw[i][h].x & 0xFFFF, f16);
        g[1] = h16_to_float(gw[i][h].x >> 16, f16);
        g[2] = h16_to_float(gw[i][h].y & 0xFFFF, f16);
        g[3] = h16_to_float(gw[i][h].y >> 16, f16);
      }
      if (SRC == SRC_STATE) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float sc = fminf(rsc[i], cs[4 * h + e]);
          mp[e] = __fmul_rn(deq4[(cw[i][h] >> (4 * e)) & 0xF], sc) + acc[i][4 * h + e];
        }
      } else if (SRC == SRC_DENSE) {
        mp[0] = mpv[i][h].x; mp[1] = mpv[i][h].y; mp[2] = mpv[i][h].z; mp[3] = mpv[i][h].w;
      } else {
        mp[0] = mp[1] = mp[2] = mp[3] = 0.f;
      }
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        o[e] = ok ? __fadd_rn(__fmul_rn(mu, mp[e]), g[e]) : 0.f;
        acc[i][4 * h + e] = o[e];        // keep M for the projection
        bad |= !isfinite(o[e]);
        nsq = fmaf(o[e], o[e], nsq);
      }
      if (ok)
        *reinterpret_cast<float4*>(M + (long long)b * mn + (long long)gi * n + cb) =
            make_float4(o[0], o[1], o[2], o[3]);
    }
  }
  const double tot = block_sum_d((double)nsq, red);
  if (t == 0 && norm2_part) norm2_part[((long long)b * cdiv(m, kRB) + bh) * nb + bj] = tot;
  if (bad && status) atomicExch(status, GM_E_NONFINITE);

  // 5. projection partials: this tile's share of M Q, four columns of Q at a time
  if (Q) {
    for (int l0 = 0; l0 < KP; l0 += 4) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 qa = *reinterpret_cast<const float4*>(Qs + (l0 + j) * kGrid + 4 * tx);
        const float4 qb = *reinterpret_cast<const float4*>(Qs + (l0 + j) * kGrid + 64 + 4 * tx);
        const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float sacc = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) sacc = fmaf(acc[i][e], qv[e], sacc);
          v[i * 4 + j] = sacc;
        }
      }
      reduce_scatter16(v, tx);
      const int row = r0 + ty + 16 * (tx >> 2), l = l0 + (tx & 3);
      if (row < m && l < k) Ppart[(((long long)b * nb + bj) * m + row) * k + l] = v[0];
    }
  }
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
  {
    // element e = lane + 32 u of the k x k Gram, summed over the row splits in order;
    // the loads of all u are independent and issued together
    constexpr int U = kMaxK * kMaxK / 32;
    double acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u] = 0.0;
    const double* gp = gram_part + (long long)b * rsplit * k * k;
    for (int p = 0; p < rsplit; ++p) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int e = lane + 32 * u;
        if (e < k * k) acc[u] += gp[(long long)p * k * k + e];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int e = lane + 32 * u;
      if (e < k * k) {
        G[e / k][e % k] = acc[u];
        L[e / k][e % k] = 0.0;
        Li[e / k][e % k] = 0.0;
      }
    }
  }
  // |M_t|^2 from the rebuild's partials: lane-strided sums, then a fixed shuffle tree
  double ns2 = 0.0;
  for (int p = lane; p < ntiles; p += 32) ns2 += norm2_part[(long long)b * ntiles + p];
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ns2 += __shfl_xor_sync(0xffffffffu, ns2, off);
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
  if (lane == 0 && scale) scale[b] = (float)(1.0 / (sqrt(ns2) + (double)eps));
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
// R = M^T P over row splits, and the normalised wide-form NS input
// X = round16(scale * M) (X = M^T when m > n).
// CTA: 64 columns x the rows of its split, in chunks of 128 rows. Warp w owns
// rows 16 w .. 16 w + 15 of a chunk, lane c the columns 2c, 2c + 1, so every
// warp reads whole 256-byte row segments of M straight into registers; P rows
// are broadcast from shared memory. fp32 sums over at most 1024 rows per split,
// fp64 across splits.
template <int KP>
__global__ void __launch_bounds__(kThreads, 2) k_backproject(int m, int n, int k, int rsplit,
                                                              const float* __restrict__ M,
                                                              const float* __restrict__ P,
                                                              const float* __restrict__ scale,
                                                              uint16_t* __restrict__ X16, int f16,
                                                              double* __restrict__ Rpart,
                                                              const int32_t* skip) {
  if (skip && *skip) return;
  constexpr int CB = 64, CH = 128, RPW = 16, XS = CH + 2;
  extern __shared__ __align__(16) float smb[];
  float* Ps = smb;                                             // [CH][KP]
  uint16_t* Xt = reinterpret_cast<uint16_t*>(Ps + CH * KP);     // [CB][XS], tall staging
  const int cbk = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, cq = t & 31, rg = t >> 5;
  const int c0 = cbk * CB;
  const int col = c0 + 2 * cq;
  const int nchunks = cdiv(m, CH);
  const int per = cdiv(nchunks, rsplit);
  const int ch0 = split * per, ch1 = min(nchunks, ch0 + per);
  const float* Mb = M + (long long)b * m * n;
  const float* Pb = P + (long long)b * m * k;
  const bool tall = m > n;
  const float sc = X16 ? scale[b] : 0.f;
  uint16_t* Xb = X16 ? X16 + (long long)b * m * n : nullptr;

  float acc[2][KP];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int l = 0; l < KP; ++l) acc[c][l] = 0.f;

  for (int ch = ch0; ch < ch1; ++ch) {
    const int i0 = ch * CH;
    float2 mv[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int gi = i0 + rg * RPW + r;
      mv[r] = (gi < m && col < n) ? *reinterpret_cast<const float2*>(Mb + (long long)gi * n + col)
                                  : make_float2(0.f, 0.f);
    }
    for (int e = t; e < CH * KP; e += kThreads) {
      const int ii = e / KP, l = e % KP, gi = i0 + ii;
      Ps[e] = (gi < m && l < k) ? Pb[(long long)gi * k + l] : 0.f;
    }
    if (Xb) {
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const int gi = i0 + rg * RPW + r;
        const uint16_t x0 = float_to_h16(mv[r].x * sc, f16), x1 = float_to_h16(mv[r].y * sc, f16);
        if (!tall) {
          if (gi < m && col < n)
            *reinterpret_cast<uint32_t*>(Xb + (long long)gi * n + col) = (uint32_t)x0 | ((uint32_t)x1 << 16);
        } else {
          Xt[(2 * cq) * XS + rg * RPW + r] = x0;
          Xt[(2 * cq + 1) * XS + rg * RPW + r] = x1;
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const float* prow = Ps + (rg * RPW + r) * KP;
#pragma unroll
      for (int l = 0; l < KP; l += 4) {
        const float4 pv = *reinterpret_cast<const float4*>(prow + l);
        acc[0][l] = fmaf(mv[r].x, pv.x, acc[0][l]);
        acc[0][l + 1] = fmaf(mv[r].x, pv.y, acc[0][l + 1]);
        acc[0][l + 2] = fmaf(mv[r].x, pv.z, acc[0][l + 2]);
        acc[0][l + 3] = fmaf(mv[r].x, pv.w, acc[0][l + 3]);
        acc[1][l] = fmaf(mv[r].y, pv.x, acc[1][l]);
        acc[1][l + 1] = fmaf(mv[r].y, pv.y, acc[1][l + 1]);
        acc[1][l + 2] = fmaf(mv[r].y, pv.z, acc[1][l + 2]);
        acc[1][l + 3] = fmaf(mv[r].y, pv.w, acc[1][l + 3]);
      }
    }
    if (Xb && tall) {
      // X[j][i] = M[i][j]: rows of X are 256-byte runs of this chunk
      for (int idx = t; idx < CB * (CH / 2); idx += kThreads) {
        const int j = idx / (CH / 2), i2 = idx % (CH / 2);
        const int gj = c0 + j, gi = i0 + 2 * i2;
        if (gj < n && gi < m)
          *reinterpret_cast<uint32_t*>(Xb + (long long)gj * m + gi) =
              *reinterpret_cast<const uint32_t*>(Xt + j * XS + 2 * i2);
      }
    }
    __syncthreads();
  }
  // ordered reduction over the eight warps
  float* red = smb;   // [CB][KP]
  for (int w = (kThreads / 32) - 1; w >= 0; --w) {
    if (rg == w) {
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int l = 0; l < KP; ++l) {
          float* slot = red + (2 * cq + c) * KP + l;
          *slot = (w == (kThreads / 32) - 1) ? acc[c][l] : (*slot + acc[c][l]);
        }
    }
    __syncthreads();
  }
  double* out = Rpart + ((long long)b * rsplit + split) * n * k;
  for (int e = t; e < CB * k; e += kThreads) {
    const int cc = e / k, l = e % k;
    if (c0 + cc < n) out[(long long)(c0 + cc) * k + l] = (double)red[cc * KP + l];
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
// One 128 x 128 grid block per CTA of 512 threads; thread (ty, tx) owns rows
// ty + 32 i (i < 4) and columns 4 tx + {0..3}, 64 + 4 tx + {0..3}. The residual
// x = M - sum_l P_il R_jl is formed in place (fp32 FMA), then the block's row and
// column absolute maxima, then the codes q = rint(fp32(x / s) * 7).
__global__ void __launch_bounds__(512, 2) k_residual_quant4(
    int m, int n, int k, const float* __restrict__ X, const float* __restrict__ P,
    const float* __restrict__ R, uint8_t* __restrict__ codes4, float* __restrict__ rscale,
    float* __restrict__ cscale, const int32_t* skip) {
  if (skip && *skip) return;
  const int bj = blockIdx.x, bi = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, mb = gridDim.y;
  const int r0 = bi * kGrid, c0 = bj * kGrid;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  const int kk = (P && R) ? k : 0;
  extern __shared__ __align__(16) float smq[];
  float* Ps = smq;                 // [kk][128]
  float* Rs = Ps + kk * kGrid;     // [kk][128]
  __shared__ float cm[32][kGrid];
  __shared__ float cmax[kGrid];

  float x[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gi = r0 + ty + 32 * i;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cb = c0 + 64 * h + 4 * tx;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gi < m && cb < n) v = *reinterpret_cast<const float4*>(X + ((long long)b * m + gi) * n + cb);
      x[i][4 * h] = v.x; x[i][4 * h + 1] = v.y; x[i][4 * h + 2] = v.z; x[i][4 * h + 3] = v.w;
    }
  }
  for (int e = t; e < kGrid * kk; e += 512) {
    const int rr = e / kk, l = e % kk;
    const int gi = r0 + rr, gj = c0 + rr;
    Ps[l * kGrid + rr] = (gi < m) ? P[((long long)b * m + gi) * kk + l] : 0.f;
    Rs[l * kGrid + rr] = (gj < n) ? R[((long long)b * n + gj) * kk + l] : 0.f;
  }
  __syncthreads();
  for (int l = 0; l < kk; ++l) {
    const float4 ra = *reinterpret_cast<const float4*>(Rs + l * kGrid + 4 * tx);
    const float4 rb = *reinterpret_cast<const float4*>(Rs + l * kGrid + 64 + 4 * tx);
    const float rv[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float pv = -Ps[l * kGrid + ty + 32 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) x[i][j] = fmaf(pv, rv[j], x[i][j]);
    }
  }
  // rows and columns outside the matrix are 0 (loaded as 0; their P, R rows are 0)
  float cmx[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) v = fmaxf(v, fabsf(x[i][j]));
    cmx[j] = v;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) cm[ty][64 * h + 4 * tx + e] = cmx[4 * h + e];
  __syncthreads();
  if (t < kGrid) {
    float v = 0.f;
#pragma unroll 8
    for (int g = 0; g < 32; ++g) v = fmaxf(v, cm[g][t]);
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
  for (int i = 0; i < 4; ++i) {
    const int gi = r0 + ty + 32 * i;
    float rmx = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) rmx = fmaxf(rmx, fabsf(x[i][j]));
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
        const float sv = fminf(rmx, cs[4 * h + e]);
        int q = 0;
        if (sv > 0.f) {
          q = (int)rintf(__fmul_rn(__fdiv_rn(x[i][4 * h + e], sv), 7.0f));
          q = max(-7, min(7, q));
        }
        packed |= (uint32_t)(q & 0xF) << (4 * e);
      }
      *reinterpret_cast<uint16_t*>(codes4 + ((long long)b * m + gi) * (n / 2) + cb / 2) = (uint16_t)packed;
    }
  }
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
cudaError_t launch_backproject_t(int B, int m, int n, int k, const float* M, const float* P,
                                 const float* scale, void* X16, bool f16, double* Rpart,
                                 float* R, const int32_t* skip, cudaStream_t s) {
  const int rs = backproject_row_splits(B, m, n);
  const size_t smem = (size_t)128 * KP * sizeof(float) + (size_t)64 * 130 * sizeof(uint16_t);
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
int rebuild_row_blocks(int m) { return cdiv(m, kRB); }
int backproject_row_splits(int B, int m, int n) {
  const int ctas = cdiv(n, 64) * B;
  const int nchunks = cdiv(m, 128);
  const int need = cdiv(m, 1024);            // at most 1024 rows summed in fp32
  const int rs = max(need, cdiv(kTargetCtas, ctas));
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

template <int SRC, bool G32, int KP>
cudaError_t launch_rebuild_t(dim3 grid, size_t smem, cudaStream_t s, int m, int n, int k,
                             const uint8_t* codes4, const float* rscale, const float* cscale,
                             const int8_t* P8, const float* Pscale, const int8_t* R8,
                             const float* Rscale, const float* Mprev32, float mu, const void* G,
                             int gdt, const float* Q, float* M, double* norm2_part, float* Ppart,
                             int32_t* status) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_rebuild_proj<SRC, G32, KP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)((2 * kMaxK * kGrid + kMaxK * kRB) * sizeof(float)));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  k_rebuild_proj<SRC, G32, KP><<<grid, kThreads, smem, s>>>(m, n, k, codes4, rscale, cscale, P8, Pscale,
                                                        R8, Rscale, Mprev32, mu, G, gdt, Q, M,
                                                        norm2_part, Ppart, status);
  return cudaGetLastError();
}

cudaError_t launch_rebuild(int B, int m, int n, int k, const uint8_t* codes4, const float* rscale,
                           const float* cscale, const int8_t* P8, const float* Pscale,
                           const int8_t* R8, const float* Rscale, const float* Mprev32, float mu,
                           const void* G, int gdt, const float* Q, float* M, double* norm2_part,
                           float* Ppart, int32_t* status, cudaStream_t s) {
  dim3 grid(cdiv(n, kGrid), cdiv(m, kRB), B);
  const int kp = k <= 8 ? 8 : (k <= 16 ? 16 : 32);
  const int kk = codes4 ? kp : 0;
  const int kq = Q ? kp : 0;
  const size_t smem = (size_t)(kk * kRB + kk * kGrid + kq * kGrid) * sizeof(float);
  const bool g32 = (G == nullptr) || gdt == GM_F32;
  const int src = codes4 ? SRC_STATE : (Mprev32 ? SRC_DENSE : SRC_ZERO);
#define GM_RB(S, W, K) launch_rebuild_t<S, W, K>(grid, smem, s, m, n, k, codes4, rscale, cscale, P8, Pscale, \
                                                 R8, Rscale, Mprev32, mu, G, gdt, Q, M, norm2_part, Ppart, status)
#define GM_RBK(S, W) (kp == 8 ? GM_RB(S, W, 8) : (kp == 16 ? GM_RB(S, W, 16) : GM_RB(S, W, 32)))
  if (src == SRC_STATE) return g32 ? GM_RBK(SRC_STATE, true) : GM_RBK(SRC_STATE, false);
  if (src == SRC_DENSE) return g32 ? GM_RBK(SRC_DENSE, true) : GM_RBK(SRC_DENSE, false);
  return g32 ? GM_RBK(SRC_ZERO, true) : GM_RBK(SRC_ZERO, false);
#undef GM_RBK
#undef GM_RB
}

cudaError_t launch_orth(int B, int m, int k, int csplit, const float* Ppart, double* Ptil,
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
  const size_t smem = (size_t)2 * k * kGrid * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_residual_quant4, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(2 * kMaxK * kGrid * sizeof(float)));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  k_residual_quant4<<<grid, 512, smem, s>>>(m, n, k, X, P, R, codes4, rscale, cscale, skip);
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
