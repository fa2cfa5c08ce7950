// Tensor-core Newton-Schulz chains for sm_100a: tcgen05.mma with the
// accumulator in TMEM, operands staged in shared memory by TMA.
//
// Standard NS ("优化器 (3)（Gram Newton-Schulz）", §1.2 eq. (2)) and the
// stabilized Gram NS (same page, Algorithm 2) reduce to three product shapes
// on the wide-form iterate X (N x M', row-major, 16-bit):
//   XX^T      : C = X X^T                     (both operands K-major rows of X)
//   sym       : C = S1 S2 for symmetric N x N S1, S2 (both operands K-major rows)
//   left      : C = S X (S symmetric N x N)   (B operand MN-major: rows of X are K)
// The first two produce symmetric results: only the lower-triangle tiles are
// computed and each off-diagonal tile is stored twice (the triangular
// scheduler of the page's §4). Epilogues apply C = alpha acc + beta Cin +
// gamma I in fp32 (a_t enters here, never as an explicit identity).
//
// Kernel anatomy (one 128 x BN output tile per CTA, 6 warps):
//   warp 0 lane 0 : TMA producer over a STAGES-deep shared-memory ring
//   warp 1        : allocates TMEM; lane 0 issues tcgen05.mma (M=128, N=BN, K=16)
//   warps 2..5    : epilogue, tcgen05.ld 32 lanes x 32 columns at a time
// Every mbarrier wait is bounded (~2 s of %globaltimer); on timeout the
// kernel records GM_E_TIMEOUT in an error word and unwinds.

#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "gm_common.cuh"
#include "gm_internal.h"

namespace gm {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 x 16-bit = 128 B = one swizzle row
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ int32_t g_device_error = 0;

enum EpiMode : int { EPI_STORE = 0, EPI_OUT = 1, EPI_WUPDATE = 2 };

struct GemmParams {
  int M, N, K;                 // output M x N; reduction K
  int batch;
  int tiles_m, tiles_n;
  int sym;                     // lower-triangle schedule + mirrored store
  int f16;                     // operand / 16-bit output type: 1 fp16, 0 bf16
  float alpha, beta, gamma;    // v = alpha acc + beta Cin + gamma [r == c]
  const uint16_t* C; long long c_bs; int ldc;
  uint16_t* D; long long d_bs; int ldd;
  uint16_t* D2; float gamma2;  // optional D2 = v + gamma2 [r == c]
  int mode;
  int transpose_out;           // EPI_OUT / EPI_WUPDATE: natural = transpose of the tile
  void* O; int odt; long long o_bs; int ldo;
  float* W; long long w_bs; int ldw; float eta, wd;
  const int32_t* skip;
  int32_t* err;
};

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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
// Bounded wait: false (and the error word set) once ~2 s have passed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && globaltimer() - t0 > kWaitLimitNs) {
      if (err) atomicExch(err, (int32_t)GM_E_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// UMMA shared-memory descriptor: SWIZZLE_128B, version 1 (sm_100).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor, kind::f16: D f32, A/B bf16 or f16, A K-major.
__host__ __device__ constexpr uint32_t idesc_f16(bool f16, bool b_mn_major, int n) {
  return (1u << 4) | ((f16 ? 0u : 1u) << 7) | ((f16 ? 0u : 1u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tri_tile(int x, int& ti, int& tj) {
  int i = (int)((sqrtf(8.0f * (float)x + 1.0f) - 1.0f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= x) ++i;
  while (i * (i + 1) / 2 > x) --i;
  ti = i;
  tj = x - i * (i + 1) / 2;
}

// ------------------------------------------------------------------ epilogue
// Staging buffers (separate from the operand ring, which keeps streaming the
// next tile while this one is written out), one 32-column slab at a time:
//   EPI_STORE : sC [BM][SP] 16-bit (C slab in, output out, in place)
//               sT [32][TP] 16-bit (transposed output, for mirrored stores)
//   otherwise : sF [BM][FP] fp32, or its transpose [32][FT] for transposed output
#ifndef GM_EPI_WARPS
#define GM_EPI_WARPS 8
#endif
constexpr int kEpiWarps = GM_EPI_WARPS;   // 8 or 16: two or four warps per TMEM lane quarter
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kGemmThreadsP = 64 + kEpiThreads;
#ifndef GM_EPI_SLAB
#define GM_EPI_SLAB 64
#endif
#ifndef GM_PREFETCH_DIST
#define GM_PREFETCH_DIST 0
#endif
#ifndef GM_LEFT_BN
#define GM_LEFT_BN 256
#endif
constexpr int SLAB = GM_EPI_SLAB;      // epilogue columns staged at a time (32, 64 or 128)
constexpr int SP = SLAB + 8;
constexpr int TP = BM + 8;
constexpr int FP = SLAB + 4;
constexpr int FT = BM + 4;
constexpr uint32_t cmax_u(uint32_t a, uint32_t b) { return a > b ? a : b; }
constexpr uint32_t kStagingBytes =
    cmax_u(cmax_u(BM * SP * 2 + SLAB * TP * 2, BM * FP * 4), SLAB * FT * 4);
constexpr int kPrefetchDist = GM_PREFETCH_DIST;  // k-blocks prefetched into L2 ahead (0: none)

template <int BN, int STAGES>
__host__ __device__ constexpr uint32_t gemm_smem_bytes() {
  return STAGES * (BM * BK * 2 + BN * BK * 2) + kStagingBytes + 256 /* barriers etc. */ +
         BM * 2 /* second-output diagonal */ + 1024 /* alignment slack */;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

__device__ __forceinline__ bool epi_any(bool pred) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(res)
      : "r"((uint32_t)pred), "n"(kEpiThreads)
      : "memory");
  return res != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
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

__device__ __forceinline__ void unpack8(const uint4 w, bool f16, float* o) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    o[2 * e] = h16_to_float(u[e] & 0xFFFF, f16);
    o[2 * e + 1] = h16_to_float(u[e] >> 16, f16);
  }
}
__device__ __forceinline__ uint4 pack8(const float* v, bool f16) {
  uint32_t u[4];
#pragma unroll
  for (int e = 0; e < 4; ++e)
    u[e] = (uint32_t)float_to_h16(v[2 * e], f16) | ((uint32_t)float_to_h16(v[2 * e + 1], f16) << 16);
  return make_uint4(u[0], u[1], u[2], u[3]);
}

// A tile of the flattened (batch, tile) list. r0 / c0 are the global row /
// column origins of this CTA's part of the output tile (a CTA owns 128 rows).
struct TileCoord {
  int bz, ti, tj, r0, c0;
};
__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int T, int tiles_per,
                                                 int tile_m, int tile_n, int row_off) {
  TileCoord c;
  c.bz = T / tiles_per;
  const int x = T - c.bz * tiles_per;
  if (p.sym) tri_tile(x, c.ti, c.tj);
  else { c.ti = x % p.tiles_m; c.tj = x / p.tiles_m; }
  c.r0 = c.ti * tile_m + row_off;
  c.c0 = c.tj * tile_n;
  return c;
}

// C values of one slab, fetched into registers one slab ahead of their use.
// Store mode: thread et holds the sC fill chunks idx = et + u * 256. Output
// modes: the thread's own row, its SLAB/2-column half of the slab.
constexpr int kWarpsPerQuarter = kEpiWarps / 4;
constexpr int CPW = SLAB / kWarpsPerQuarter;          // slab columns per epilogue warp
constexpr int NCH = BM * SLAB / 8 / kEpiThreads;      // 16-byte C chunks per thread per slab
static_assert(CPW % 16 == 0 && NCH >= 1, "slab too narrow for the epilogue warp count");

template <int BN>
__device__ __forceinline__ void c_prefetch(const GemmParams& p, const TileCoord& tc, int slab,
                                           int warp, int lane, uint4 (&cpre)[NCH]) {
#pragma unroll
  for (int u = 0; u < NCH; ++u) cpre[u] = make_uint4(0, 0, 0, 0);
  if (!p.C || p.beta == 0.f) return;
  const int r0 = tc.r0;
  const int c0 = tc.c0 + slab * SLAB;
  const long long cbs = (long long)tc.bz * p.c_bs;
  if (p.mode == EPI_STORE) {
    const int et = threadIdx.x - 64;
#pragma unroll
    for (int u = 0; u < NCH; ++u) {
      const int idx = et + u * kEpiThreads;
      const int row = idx / (SLAB / 8), cc = idx % (SLAB / 8);
      if (r0 + row < p.M && c0 + cc * 8 < p.N)
        cpre[u] = *reinterpret_cast<const uint4*>(p.C + cbs + (long long)(r0 + row) * p.ldc + c0 + cc * 8);
    }
  } else {
    const int r = r0 + (warp & 3) * 32 + lane;
    const int cl = ((warp - 2) >> 2) * CPW;
#pragma unroll
    for (int g = 0; g < NCH; ++g)
      if (r < p.M && c0 + cl + g * 8 < p.N)
        cpre[g] = *reinterpret_cast<const uint4*>(p.C + cbs + (long long)r * p.ldc + c0 + cl + g * 8);
  }
}

__device__ __forceinline__ uint32_t pack2(float a, float b, bool f16) {
  if (f16) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// One SLAB-column slab of the tile: TMEM -> registers -> staging -> global.
template <int BN>
__device__ __forceinline__ void epilogue_slab(const GemmParams& p, uint8_t* stg, uint32_t tacc,
                                              const TileCoord& tc, int slab, int warp, int lane,
                                              uint16_t* d2diag, bool last_slab, uint32_t acc_empty_bar,
                                              uint4 (&cpre)[NCH], bool cluster_arrive = false) {
  const int et = threadIdx.x - 64;          // 0..255
  const int q = warp & 3;                   // TMEM lane quarter of this warp
  const int sub = (warp - 2) >> 2;          // column part of the slab
  const int rr = q * 32 + lane;             // tile row owned by this thread
  const int r0 = tc.r0;
  const int cs0 = slab * SLAB;              // slab column offset inside the tile
  const int c0 = tc.c0 + cs0;               // global column of the slab
  const int dlt = tc.r0 - tc.c0;            // element (row, tile col j) lies below the
                                            // diagonal iff dlt + row - j > 0
  const int r = r0 + rr;
  const bool f16 = p.f16 != 0;
  const bool store_mode = p.mode == EPI_STORE;
  const bool tr = p.transpose_out != 0;
  uint16_t* sC = reinterpret_cast<uint16_t*>(stg);
  uint16_t* sT = sC + BM * SP;
  float* sF = reinterpret_cast<float*>(stg);
  const int rows_valid = min(BM, p.M - r0);
  const int cols_valid = min(SLAB, p.N - c0);   // may be <= 0 for a ragged tile
  const bool use_c = p.C && p.beta != 0.f;
  const float alpha = p.alpha, beta = p.beta;

  // 1. C slab (fetched one slab ahead) -> sC; start fetching the next slab
  uint4 cnow[NCH];
#pragma unroll
  for (int u = 0; u < NCH; ++u) cnow[u] = cpre[u];
  if (store_mode && use_c) {
#pragma unroll
    for (int u = 0; u < NCH; ++u) {
      const int idx = et + u * kEpiThreads;
      *reinterpret_cast<uint4*>(sC + (idx / (SLAB / 8)) * SP + (idx % (SLAB / 8)) * 8) = cnow[u];
    }
  }
  if (!last_slab) c_prefetch<BN>(p, tc, slab + 1, warp, lane, cpre);
  epi_bar();

  // 2. TMEM -> registers -> epilogue math -> staging
#pragma unroll
  for (int h = 0; h < CPW / 16; ++h) {
    const int cl = sub * CPW + h * 16;   // column inside the slab
    float v[16];
    tmem_ld16(tacc + ((uint32_t)(q * 32) << 16) + (uint32_t)(cs0 + cl), v);
    const bool has_diag = r >= c0 + cl && r < c0 + cl + 16;
    if (store_mode) {
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        float x[8];
        if (use_c) {
          float cin[8];
          unpack8(*reinterpret_cast<const uint4*>(sC + rr * SP + cl + g * 8), f16, cin);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = fmaf(beta, cin[e], alpha * v[g * 8 + e]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = alpha * v[g * 8 + e];
        }
        if (has_diag) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (c0 + cl + g * 8 + e == r) {
              x[e] += p.gamma;
              if (p.D2) d2diag[rr] = float_to_h16(x[e] + p.gamma2, f16);
            }
          }
        }
        uint4 w;
        w.x = pack2(x[0], x[1], f16);
        w.y = pack2(x[2], x[3], f16);
        w.z = pack2(x[4], x[5], f16);
        w.w = pack2(x[6], x[7], f16);
        *reinterpret_cast<uint4*>(sC + rr * SP + cl + g * 8) = w;
        if (p.sym) {
          const uint32_t u4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sT[(cl + g * 8 + 2 * e) * TP + rr] = (uint16_t)(u4[e] & 0xFFFF);
            sT[(cl + g * 8 + 2 * e + 1) * TP + rr] = (uint16_t)(u4[e] >> 16);
          }
        }
      }
    } else {
      // O = alpha acc + beta C (this thread's C values were fetched a slab ahead)
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        float cin[8];
        unpack8(cnow[h * 2 + g], f16, cin);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float val = fmaf(beta, cin[e], alpha * v[g * 8 + e]);
          if (!tr) sF[rr * FP + cl + g * 8 + e] = val;
          else sF[(cl + g * 8 + e) * FT + rr] = val;
        }
      }
    }
  }
  if (last_slab) {
    // every TMEM read of this accumulator is done: hand it back to the MMA warp
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (cluster_arrive) asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(acc_empty_bar) : "memory");
      else mbar_arrive(acc_empty_bar);
    }
  }
  epi_bar();

  // 3. staging -> global (coalesced)
  if (cols_valid > 0) {
    if (store_mode) {
      uint16_t* dbase = p.D + (long long)tc.bz * p.d_bs;
      uint16_t* d2base = p.D2 ? p.D2 + (long long)tc.bz * p.d_bs : nullptr;
      // direct pass; for symmetric products only positions on or below the diagonal
#pragma unroll
      for (int u = 0; u < NCH; ++u) {
        const int idx = et + u * kEpiThreads;
        const int row = idx / (SLAB / 8), cc = idx % (SLAB / 8);
        if (row >= rows_valid || cc * 8 >= cols_valid) continue;
        const int rel0 = dlt + row - (cs0 + cc * 8);   // for the chunk's first column
        if (p.sym && rel0 < 0) continue;
        const uint4 w = *reinterpret_cast<const uint4*>(sC + row * SP + cc * 8);
        const long long goff = (long long)(r0 + row) * p.ldd + c0 + cc * 8;
        if (p.sym && rel0 < 8) {
          uint16_t hv[8];
          *reinterpret_cast<uint4*>(hv) = w;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (rel0 - e >= 0) {
              dbase[goff + e] = hv[e];
              if (d2base) d2base[goff + e] = (rel0 == e) ? d2diag[row] : hv[e];
            }
          }
        } else {
          *reinterpret_cast<uint4*>(dbase + goff) = w;
          if (d2base) *reinterpret_cast<uint4*>(d2base + goff) = w;
        }
      }
      if (p.sym) {
        // mirror pass: D[c0 + j][r0 + i] = value(i, j) for i strictly below the diagonal
#pragma unroll
        for (int u = 0; u < NCH; ++u) {
          const int idx = et + u * kEpiThreads;
          const int row = idx >> 4, cc = idx & 15;   // row: slab column j; cc: chunk of tile rows
          if (row >= cols_valid || cc * 8 >= rows_valid) continue;
          const int relf = dlt + cc * 8 - (cs0 + row);   // for the chunk's first tile row
          if (relf + 7 <= 0) continue;
          const uint4 w = *reinterpret_cast<const uint4*>(sT + row * TP + cc * 8);
          const long long goff = (long long)(c0 + row) * p.ldd + r0 + cc * 8;
          if (relf <= 0) {
            uint16_t hv[8];
            *reinterpret_cast<uint4*>(hv) = w;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              if (relf + e > 0) {
                dbase[goff + e] = hv[e];
                if (d2base) d2base[goff + e] = hv[e];
              }
            }
          } else {
            *reinterpret_cast<uint4*>(dbase + goff) = w;
            if (d2base) *reinterpret_cast<uint4*>(d2base + goff) = w;
          }
        }
      }
    } else {
      // fp32 values -> O (any dtype) or W -= eta (O + wd W), natural orientation;
      // four 16-byte accesses per thread in flight at a time
      const int ld = p.mode == EPI_OUT ? p.ldo : p.ldw;
      constexpr int NB = 4;
      constexpr int kQ = BM * SLAB / 4;   // float4 chunks per slab
#pragma unroll 1
      for (int b0 = 0; b0 < kQ; b0 += kEpiThreads * NB) {
        float4 val[NB], wv[NB];
        long long off[NB];
        bool okc[NB];
#pragma unroll
        for (int u = 0; u < NB; ++u) {
          const int idx = b0 + et + u * kEpiThreads;
          if (!tr) {
            const int row = idx / (SLAB / 4), col = (idx % (SLAB / 4)) * 4;
            okc[u] = row < rows_valid && col < cols_valid;
            off[u] = (long long)(r0 + row) * ld + c0 + col;
            if (okc[u]) val[u] = *reinterpret_cast<const float4*>(sF + row * FP + col);
          } else {
            const int col = idx >> 5, row = (idx & 31) * 4;   // slab column = natural row
            okc[u] = col < cols_valid && row < rows_valid;
            off[u] = (long long)(c0 + col) * ld + r0 + row;
            if (okc[u]) val[u] = *reinterpret_cast<const float4*>(sF + col * FT + row);
          }
          if (p.mode == EPI_WUPDATE && okc[u])
            wv[u] = *reinterpret_cast<const float4*>(p.W + (long long)tc.bz * p.w_bs + off[u]);
        }
#pragma unroll
        for (int u = 0; u < NB; ++u) {
          if (!okc[u]) continue;
          if (p.mode == EPI_OUT) {
            store4_from_float(p.O, (long long)tc.bz * p.o_bs + off[u], p.odt, val[u]);
          } else {
            float4 w = wv[u];
            w.x -= p.eta * (val[u].x + p.wd * w.x);
            w.y -= p.eta * (val[u].y + p.wd * w.y);
            w.z -= p.eta * (val[u].z + p.wd * w.z);
            w.w -= p.eta * (val[u].w + p.wd * w.w);
            *reinterpret_cast<float4*>(p.W + (long long)tc.bz * p.w_bs + off[u]) = w;
          }
        }
      }
    }
  }
  epi_bar();   // staging free for the next slab
}

// ------------------------------------------------------------------ kernel
// Persistent: one CTA per SM walks the flattened (batch, tile) list with a
// stride of gridDim.x. Warp 0 streams operand k-blocks through a STAGES-deep
// ring, continuously across tiles; warp 1 accumulates each tile into one of two
// TMEM accumulators; warps 2..9 drain the other accumulator meanwhile.
template <int BN, bool B_MN, int STAGES>
__global__ void __launch_bounds__(kGemmThreadsP, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const GemmParams p) {
  if (p.skip && *p.skip) return;
  constexpr uint32_t kABytes = BM * BK * 2;
  constexpr uint32_t kBBytes = BN * BK * 2;
  constexpr uint32_t kStageBytes = kABytes + kBBytes;
  constexpr uint32_t kTmemCols = 2 * BN;   // two accumulators (power of two, <= 512)

  extern __shared__ __align__(1024) uint8_t dsm[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stg = base + STAGES * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + kStagingBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;     // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* consumed = abort_flag + 1;
  uint16_t* d2diag = reinterpret_cast<uint16_t*>(consumed + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_per = p.sym ? p.tiles_m * (p.tiles_m + 1) / 2 : p.tiles_m * p.tiles_n;
  const int total = p.batch * tiles_per;
  const int nk = cdiv(p.K, BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), kEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    *consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_map(&tmA);
    prefetch_map(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;   // producer only
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      uint32_t g = 0;
      bool ok = true;
      // L2 prefetch cursor (tile pT, k-block pkb), kPrefetchDist k-blocks ahead of the loads
      int pT = blockIdx.x, pkb = 0;
      TileCoord pc = decode_tile(p, pT, tiles_per, BM, BN, 0);
      auto prefetch_next = [&]() {
        if (pT >= total) return;
        tma_prefetch_3d(&tmA, pkb * BK, pc.r0, pc.bz);
        if (!B_MN) {
          tma_prefetch_3d(&tmB, pkb * BK, pc.c0, pc.bz);
        } else {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) tma_prefetch_3d(&tmB, pc.c0 + c * 64, pkb * BK, pc.bz);
        }
        if (++pkb == nk) {
          pkb = 0;
          pT += gridDim.x;
          if (pT < total) pc = decode_tile(p, pT, tiles_per, BM, BN, 0);
        }
      };
      for (int i = 0; i < kPrefetchDist; ++i) prefetch_next();
      const bool do_prefetch = kPrefetchDist > 0;
      for (int T = blockIdx.x; T < total && ok; T += gridDim.x) {
        const TileCoord tc = decode_tile(p, T, tiles_per, BM, BN, 0);
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          const uint32_t ph = (g / STAGES) & 1u;
          if (do_prefetch) prefetch_next();
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, p.err)) { ok = false; break; }
          const uint32_t a_dst = smem_u32(base + s * kStageBytes);
          const uint32_t b_dst = a_dst + kABytes;
          const uint32_t bar = smem_u32(&full[s]);
          mbar_expect_tx(bar, kStageBytes);
          tma_load_3d(a_dst, &tmA, bar, kb * BK, tc.r0, tc.bz);
          if (!B_MN) {
            tma_load_3d(b_dst, &tmB, bar, kb * BK, tc.c0, tc.bz);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_3d(b_dst + c * (BK * 128), &tmB, bar, tc.c0 + c * 64, kb * BK, tc.bz);
          }
        }
      }
      if (!ok) *abort_flag = 1;
      issued = (int)g;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = idesc_f16(p.f16 != 0, B_MN, BN);
      uint32_t g = 0;
      bool ok = true;
      int it = 0;
      for (int T = blockIdx.x; T < total && ok; T += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(smem_u32(&acc_empty[ab]), (use & 1u) ^ 1u, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * BN);
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          const uint32_t ph = (g / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&full[s]), ph, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(base + s * kStageBytes);
          const uint32_t b_base = a_base + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = sdesc(a_base + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc(b_base + kk * 2048, BK * 128, 1024)
                                     : sdesc(b_base + kk * 32, 16, 1024);
            umma(d, ad, bd, idesc, (kb | kk) ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty[s]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&acc_full[ab]));
      }
      *consumed = (int)g;
      if (!ok) *abort_flag = 1;
      // every MMA issued above has completed once this barrier fires
      umma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, p.err);
    }
  } else {
    // ---------------- epilogue warps
    int it = 0;
    for (int T = blockIdx.x; T < total; T += gridDim.x, ++it) {
      const int ab = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      const TileCoord tc = decode_tile(p, T, tiles_per, BM, BN, 0);
      uint4 cpre[NCH];
      c_prefetch<BN>(p, tc, 0, warp, lane, cpre);   // overlaps the MMAs of this tile
      const bool ok = mbar_wait(smem_u32(&acc_full[ab]), use & 1u, p.err);
      tc_fence_after();
      // the eight epilogue warps share named barriers: leave together or not at all
      if (epi_any(!ok || *abort_flag)) break;
      const uint32_t tacc = tmem + (uint32_t)(ab * BN);
#pragma unroll 1
      for (int slab = 0; slab < BN / SLAB; ++slab)
        epilogue_slab<BN>(p, stg, tacc, tc, slab, warp, lane, d2diag, slab == BN / SLAB - 1,
                          smem_u32(&acc_empty[ab]), cpre);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0) {
    // after an abort, let the copies still in flight land before the CTA exits
    for (int g = *consumed; g < issued; ++g)
      mbar_wait(smem_u32(&full[g % STAGES]), (uint32_t)(g / STAGES) & 1u, p.err);
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------ 2-SM kernel
// A CTA pair (cluster of 2) computes 256 x 256 output tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256): each CTA stages its own 128 rows
// of A and 128 of the 256 B rows (columns, for an MN-major B) per k-block, so a
// pair moves 32 KB per SM for 4.2 MFLOP per SM -- half the operand traffic per
// FLOP of a 128 x 128 tile. Both CTAs' TMA loads complete on the leader's
// (rank 0) full barrier; the leader's MMA thread commits to both CTAs' empty
// and accumulator barriers; each CTA drains its own 128 TMEM lanes. No load uses
// multicast.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs once the issued MMAs finish.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  const uint16_t both = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(both)
      : "memory");
}

template <bool B_MN, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreadsP, 1)
    k_gemm2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const GemmParams p) {
  constexpr int BN = 256;                     // tile columns (per CTA accumulator width)
  constexpr uint32_t kABytes = BM * BK * 2;   // 128 rows of A
  constexpr uint32_t kBBytes = 128 * BK * 2;  // this CTA's half of B
  constexpr uint32_t kStageBytes = kABytes + kBBytes;
  constexpr uint32_t kTmemCols = 2 * BN;      // two 256-column accumulators

  // The skip flag is read by both CTAs of a pair before any cluster-level
  // operation, so they return together.
  if (p.skip && *p.skip) return;

  extern __shared__ __align__(1024) uint8_t dsm[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stg = base + STAGES * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + kStagingBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;     // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* consumed = abort_flag + 1;
  uint16_t* d2diag = reinterpret_cast<uint16_t*>(consumed + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t cr = cluster_rank();
  const bool leader = cr == 0;
  const int pid = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int tiles_per = p.sym ? p.tiles_m * (p.tiles_m + 1) / 2 : p.tiles_m * p.tiles_n;
  const int total = p.batch * tiles_per;
  const int nk = cdiv(p.K, BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    *consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_map(&tmA);
    prefetch_map(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      uint32_t g = 0;
      bool ok = true;
      for (int T = pid; T < total && ok; T += npairs) {
        const TileCoord tc = decode_tile(p, T, tiles_per, 2 * BM, BN, (int)cr * BM);
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          const uint32_t ph = (g / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, p.err)) { ok = false; break; }
          const uint32_t a_dst = smem_u32(base + s * kStageBytes);
          const uint32_t b_dst = a_dst + kABytes;
          const uint32_t bar = map_to_rank(smem_u32(&full[s]), 0);   // the leader's barrier
          if (leader) mbar_expect_tx(smem_u32(&full[s]), 2 * kStageBytes);
          tma_load_3d_pair(a_dst, &tmA, bar, kb * BK, tc.r0, tc.bz);
          if (!B_MN) {
            tma_load_3d_pair(b_dst, &tmB, bar, kb * BK, tc.c0 + (int)cr * 128, tc.bz);
          } else {
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tma_load_3d_pair(b_dst + c * (BK * 128), &tmB, bar, tc.c0 + (int)cr * 128 + c * 64,
                               kb * BK, tc.bz);
          }
        }
      }
      if (!ok) *abort_flag = 1;
      issued = (int)g;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader CTA only)
      // M = 256 across the pair: replace the descriptor's M field (bits 24..28)
      const uint32_t idesc = (idesc_f16(p.f16 != 0, B_MN, BN) & ~(0x1Fu << 24)) |
                             ((uint32_t)((2 * BM) >> 4) << 24);
      uint32_t g = 0;
      bool ok = true;
      int it = 0;
      for (int T = pid; T < total && ok; T += npairs, ++it) {
        const int ab = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(smem_u32(&acc_empty[ab]), (use & 1u) ^ 1u, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * BN);
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          const uint32_t ph = (g / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&full[s]), ph, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(base + s * kStageBytes);
          const uint32_t b_base = a_base + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = sdesc(a_base + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc(b_base + kk * 2048, BK * 128, 1024)
                                     : sdesc(b_base + kk * 32, 16, 1024);
            umma_pair(d, ad, bd, idesc, (kb | kk) ? 1u : 0u);
          }
          umma_commit_pair(smem_u32(&empty[s]));
        }
        if (!ok) break;
        umma_commit_pair(smem_u32(&acc_full[ab]));
      }
      *consumed = (int)g;
      if (!ok) *abort_flag = 1;
      umma_commit_pair(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, p.err);
    }
  } else {
    // ---------------- epilogue warps (both CTAs, 128 TMEM lanes each)
    const uint32_t empty_remote0 = map_to_rank(smem_u32(&acc_empty[0]), 0);
    const uint32_t empty_remote1 = map_to_rank(smem_u32(&acc_empty[1]), 0);
    int it = 0;
    for (int T = pid; T < total; T += npairs, ++it) {
      const int ab = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      const TileCoord tc = decode_tile(p, T, tiles_per, 2 * BM, BN, (int)cr * BM);
      uint4 cpre[NCH];
      c_prefetch<BN>(p, tc, 0, warp, lane, cpre);
      const bool ok = mbar_wait(smem_u32(&acc_full[ab]), use & 1u, p.err);
      tc_fence_after();
      if (epi_any(!ok || *abort_flag)) break;
      const uint32_t tacc = tmem + (uint32_t)(ab * BN);
#pragma unroll 1
      for (int slab = 0; slab < BN / SLAB; ++slab)
        epilogue_slab<BN>(p, stg, tacc, tc, slab, warp, lane, d2diag, slab == BN / SLAB - 1,
                          ab ? empty_remote1 : empty_remote0, cpre, true);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && leader) {
    // after an abort, let the copies still in flight (from both CTAs) land
    for (int g = *consumed; g < issued; ++g)
      mbar_wait(smem_u32(&full[g % STAGES]), (uint32_t)(g / STAGES) & 1u, p.err);
  }
  cluster_sync_all();   // neither CTA leaves while the other may still signal it
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 3-D map over [batch][rows][cols] of 16-bit elements with a {64, box_rows, 1}
// box and the 128-byte swizzle the UMMA descriptors above expect.
bool make_map(CUtensorMap* map, const void* base, bool f16, int rows, int cols, int ld,
              int batch, long long batch_stride, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)batch_stride * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int BN, bool B_MN, int STAGES>
cudaError_t launch_gemm_t(const CUtensorMap& a, const CUtensorMap& b, GemmParams p, int batch,
                          cudaStream_t s) {
  constexpr int smem = (int)gemm_smem_bytes<BN, STAGES>();
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm<BN, B_MN, STAGES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  p.batch = batch;
  const int tiles = p.sym ? p.tiles_m * (p.tiles_m + 1) / 2 : p.tiles_m * p.tiles_n;
  const int total = tiles * batch;
  const int grid = total < num_sms() ? total : num_sms();
  k_gemm<BN, B_MN, STAGES><<<grid, kGemmThreadsP, smem, s>>>(a, b, p);
  return cudaGetLastError();
}

#ifndef GM_PAIR
#define GM_PAIR 1
#endif
constexpr bool kPair = GM_PAIR != 0;   // 2-SM (cta_group::2) 256 x 256 tiles

template <bool B_MN>
cudaError_t launch_gemm_pair(const CUtensorMap& a, const CUtensorMap& b, GemmParams p, int batch,
                             cudaStream_t s) {
  constexpr uint32_t kBudget = 227 * 1024 - 2048 - kStagingBytes;
  constexpr int kStagesFit = (int)(kBudget / (2 * BM * BK * 2));
  constexpr int STAGES = kStagesFit > 8 ? 8 : kStagesFit;
  constexpr int smem = (int)gemm_smem_bytes<128, STAGES>();
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm2<B_MN, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  p.batch = batch;
  const int tiles = p.sym ? p.tiles_m * (p.tiles_m + 1) / 2 : p.tiles_m * p.tiles_n;
  const int total = tiles * batch;
  const int pairs = total < num_sms() / 2 ? total : num_sms() / 2;
  k_gemm2<B_MN, STAGES><<<2 * pairs, kGemmThreadsP, smem, s>>>(a, b, p);
  return cudaGetLastError();
}

template <int BN, bool B_MN>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, int batch,
                        cudaStream_t s) {
  constexpr uint32_t kBudget = 227 * 1024 - 2048 - kStagingBytes;   // ring budget per CTA
  constexpr int kStagesFit = (int)(kBudget / (BM * BK * 2 + BN * BK * 2));
  constexpr int kStagesUse = kStagesFit > 8 ? 8 : kStagesFit;
  return launch_gemm_t<BN, B_MN, kStagesUse>(a, b, p, batch, s);
}

constexpr int kLeftBN = GM_LEFT_BN;   // output tile width of the S X products

GemmParams base_params(int M, int N, int K, bool f16, const int32_t* skip, int32_t* err) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M; p.N = N; p.K = K;
  p.f16 = f16 ? 1 : 0;
  p.alpha = 1.f;
  p.skip = skip;
  p.err = err;
  return p;
}

struct Ns {
  int B, N, Mp;     // wide form N x M'
  bool f16;
  bool tall;        // natural = transpose of the wide form
  const int32_t* skip;
  int32_t* err;
  cudaStream_t s;
};

// C (N x N, symmetric) = X X^T (+ epilogue), X: N x M'.
cudaError_t xxt(const Ns& c, const uint16_t* X, uint16_t* D) {
  CUtensorMap ma;
  if (!make_map(&ma, X, c.f16, c.N, c.Mp, c.Mp, c.B, (long long)c.N * c.Mp, BM)) return cudaErrorInvalidValue;
  GemmParams p = base_params(c.N, c.N, c.Mp, c.f16, c.skip, c.err);
  p.tiles_m = p.tiles_n = cdiv(c.N, kPair ? 2 * BM : BM);
  p.sym = 1;
  p.D = D; p.d_bs = (long long)c.N * c.N; p.ldd = c.N;
  if (kPair) return launch_gemm_pair<false>(ma, ma, p, c.B, c.s);
  return launch_gemm<128, false>(ma, ma, p, c.B, c.s);
}

// D = alpha S1 S2 + beta Cin + gamma I (symmetric N x N operands); D2 optional.
cudaError_t symmul(const Ns& c, const uint16_t* S1, const uint16_t* S2, float alpha, float beta,
                   const uint16_t* Cin, float gamma, uint16_t* D, uint16_t* D2 = nullptr,
                   float gamma2 = 0.f) {
  CUtensorMap ma, mb;
  const long long bs = (long long)c.N * c.N;
  if (!make_map(&ma, S1, c.f16, c.N, c.N, c.N, c.B, bs, BM)) return cudaErrorInvalidValue;
  if (!make_map(&mb, S2, c.f16, c.N, c.N, c.N, c.B, bs, 128)) return cudaErrorInvalidValue;
  GemmParams p = base_params(c.N, c.N, c.N, c.f16, c.skip, c.err);
  p.tiles_m = p.tiles_n = cdiv(c.N, kPair ? 2 * BM : BM);
  p.sym = 1;
  p.alpha = alpha; p.beta = beta; p.gamma = gamma;
  p.C = Cin; p.c_bs = bs; p.ldc = c.N;
  p.D = D; p.d_bs = bs; p.ldd = c.N;
  p.D2 = D2; p.gamma2 = gamma2;
  if (kPair) return launch_gemm_pair<false>(ma, mb, p, c.B, c.s);
  return launch_gemm<128, false>(ma, mb, p, c.B, c.s);
}

// Y = alpha S X + beta X  (S symmetric N x N, X N x M'); either stored as a new
// iterate (D) or written out in natural orientation (final step).
cudaError_t leftmul(const Ns& c, const uint16_t* S, const uint16_t* X, float alpha, float beta,
                    uint16_t* D, const NsOutput* out) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, S, c.f16, c.N, c.N, c.N, c.B, (long long)c.N * c.N, BM)) return cudaErrorInvalidValue;
  // MN-major B operand: rows of X are the K index, columns the N index.
  if (!make_map(&mb, X, c.f16, c.N, c.Mp, c.Mp, c.B, (long long)c.N * c.Mp, BK)) return cudaErrorInvalidValue;
  GemmParams p = base_params(c.N, c.Mp, c.N, c.f16, c.skip, c.err);
  p.tiles_m = cdiv(c.N, kPair ? 2 * BM : BM);
  p.tiles_n = cdiv(c.Mp, kPair ? 256 : kLeftBN);
  p.alpha = alpha; p.beta = beta;
  p.C = X; p.c_bs = (long long)c.N * c.Mp; p.ldc = c.Mp;
  if (!out) {
    p.mode = EPI_STORE;
    p.D = D; p.d_bs = (long long)c.N * c.Mp; p.ldd = c.Mp;
  } else {
    p.transpose_out = c.tall ? 1 : 0;
    const int ld = c.tall ? c.N : c.Mp;   // natural row length
    if (out->mode == 0) {
      p.mode = EPI_OUT;
      p.O = out->O; p.odt = out->odt; p.o_bs = (long long)c.N * c.Mp; p.ldo = ld;
    } else {
      p.mode = EPI_WUPDATE;
      p.W = out->W; p.w_bs = (long long)c.N * c.Mp; p.ldw = ld;
      p.eta = out->eta; p.wd = out->wd;
    }
  }
  if (kPair) return launch_gemm_pair<true>(ma, mb, p, c.B, c.s);
  return launch_gemm<kLeftBN, true>(ma, mb, p, c.B, c.s);
}

#define GM_TRY(x)                          \
  do {                                     \
    cudaError_t e_ = (x);                  \
    if (e_ != cudaSuccess) return e_;      \
  } while (0)

uint8_t* carve(uint8_t*& cur, size_t bytes) {
  uint8_t* p = cur;
  cur += (bytes + 255) & ~size_t(255);
  return p;
}

}  // namespace

size_t ns_standard_ws_bytes(int B, int m, int n) {
  const size_t N = (size_t)(m < n ? m : n), Mp = (size_t)(m < n ? n : m);
  auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
  return al(B * N * Mp * 2) + 2 * al(B * N * N * 2);
}
size_t ns_gram_ws_bytes(int B, int m, int n) {
  const size_t N = (size_t)(m < n ? m : n), Mp = (size_t)(m < n ? n : m);
  auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
  return al(B * N * Mp * 2) + 6 * al(B * N * N * 2);
}

cudaError_t run_ns_standard(int B, int m, int n, uint16_t* X16, const float* abc, int T,
                            const NsOutput& out, void* ws, const int32_t* skip, int32_t* err,
                            cudaStream_t s) {
  Ns c{B, m < n ? m : n, m < n ? n : m, false, m > n, skip, err ? err : device_error_word(), s};
  uint8_t* cur = static_cast<uint8_t*>(ws);
  uint16_t* Xb = reinterpret_cast<uint16_t*>(carve(cur, (size_t)B * c.N * c.Mp * 2));
  uint16_t* A = reinterpret_cast<uint16_t*>(carve(cur, (size_t)B * c.N * c.N * 2));
  uint16_t* Bm = reinterpret_cast<uint16_t*>(carve(cur, (size_t)B * c.N * c.N * 2));
  uint16_t* X = X16;
  uint16_t* Xn = Xb;
  for (int t = 0; t < T; ++t) {
    const float a = abc[3 * t], b = abc[3 * t + 1], cc = abc[3 * t + 2];
    GM_TRY(xxt(c, X, A));                                  // A = X X^T
    GM_TRY(symmul(c, A, A, cc, b, A, 0.f, Bm));            // B = c A^2 + b A
    const bool last = (t == T - 1);
    GM_TRY(leftmul(c, Bm, X, 1.f, a, Xn, last ? &out : nullptr));   // X = B X + a X
    uint16_t* tmp = X; X = Xn; Xn = tmp;
  }
  return cudaSuccess;
}

cudaError_t run_ns_gram(int B, int m, int n, uint16_t* X16, const float* abc, int T,
                        const int* restart_after, int n_restart, const NsOutput& out, void* ws,
                        const int32_t* skip, int32_t* err, cudaStream_t s) {
  Ns c{B, m < n ? m : n, m < n ? n : m, true, m > n, skip, err ? err : device_error_word(), s};
  uint8_t* cur = static_cast<uint8_t*>(ws);
  const size_t nn = (size_t)B * c.N * c.N * 2;
  uint16_t* Xb = reinterpret_cast<uint16_t*>(carve(cur, (size_t)B * c.N * c.Mp * 2));
  uint16_t* R = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Rn = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Z = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Q = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Qn = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* RZ = reinterpret_cast<uint16_t*>(carve(cur, nn));
  bool restart_at[GM_MAX_T + 1] = {false};
  for (int i = 0; i < n_restart; ++i)
    if (restart_after[i] >= 1 && restart_after[i] < T) restart_at[restart_after[i]] = true;
  uint16_t* X = X16;
  uint16_t* Xn = Xb;
  GM_TRY(xxt(c, X, R));                                    // R = X X^T
  bool q_is_identity = true;
  for (int t = 1; t <= T; ++t) {
    const float a = abc[3 * (t - 1)], b = abc[3 * (t - 1) + 1], cc = abc[3 * (t - 1) + 2];
    const bool block_end = restart_at[t] || t == T;
    if (q_is_identity) {
      // Z = c R^2 + b R, and Q = Z + a I from the same epilogue
      GM_TRY(symmul(c, R, R, cc, b, R, 0.f, Z, Q, a));
      q_is_identity = false;
    } else {
      GM_TRY(symmul(c, R, R, cc, b, R, 0.f, Z));
      GM_TRY(symmul(c, Q, Z, 1.f, a, Q, 0.f, Qn));          // Q = Q Z + a Q
      uint16_t* tq = Q; Q = Qn; Qn = tq;
    }
    if (!block_end) {
      GM_TRY(symmul(c, R, Z, 1.f, a, R, 0.f, RZ));          // RZ = R Z + a R
      GM_TRY(symmul(c, Z, RZ, 1.f, a, RZ, 0.f, Rn));        // R = Z RZ + a RZ
      uint16_t* tr = R; R = Rn; Rn = tr;
    } else if (t < T) {
      GM_TRY(leftmul(c, Q, X, 1.f, 0.f, Xn, nullptr));      // restart: X = Q X
      uint16_t* tx = X; X = Xn; Xn = tx;
      GM_TRY(xxt(c, X, R));
      q_is_identity = true;
    } else {
      GM_TRY(leftmul(c, Q, X, 1.f, 0.f, nullptr, &out));    // O = Q X
    }
  }
  return cudaSuccess;
}

void ns_schedule_flops(int ns_mode, int m, int n, int T, const int* restart_after, int n_restart,
                       double* flops, int* products) {
  const double N = (double)(m < n ? m : n), Mp = (double)(m < n ? n : m);
  const double xxt_f = Mp * N * N, sym_f = N * N * N, left_f = 2.0 * Mp * N * N;
  double f = 0.0;
  int cnt = 0;
  if (ns_mode == GM_NS_STANDARD) {
    f = T * (xxt_f + sym_f + left_f);
    cnt = 3 * T;
  } else {
    bool restart_at[GM_MAX_T + 1] = {false};
    for (int i = 0; i < n_restart; ++i)
      if (restart_after[i] >= 1 && restart_after[i] < T) restart_at[restart_after[i]] = true;
    f += xxt_f; cnt += 1;
    bool qi = true;
    for (int t = 1; t <= T; ++t) {
      const bool block_end = restart_at[t] || t == T;
      f += sym_f; cnt += 1;                  // R^2 (Q = Z + aI rides in its epilogue)
      if (!qi) { f += sym_f; cnt += 1; }     // Q Z
      qi = false;
      if (!block_end) { f += 2 * sym_f; cnt += 2; }
      else {
        f += left_f; cnt += 1;
        if (t < T) { f += xxt_f; cnt += 1; qi = true; }
      }
    }
  }
  if (flops) *flops = f;
  if (products) *products = cnt;
}

int32_t* device_error_word() {
  static int32_t* ptr = nullptr;
  if (!ptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) ptr = static_cast<int32_t*>(p);
  }
  return ptr;
}

}  // namespace gm
