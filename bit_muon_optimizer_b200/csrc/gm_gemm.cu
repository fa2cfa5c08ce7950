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
// computed and each off-diagonal block is stored twice (the triangular
// scheduler of the page's §4). Epilogues apply C = alpha acc + beta Cin +
// gamma I in fp32 (a_t enters here, never as an explicit identity).
//
// One persistent kernel of CTA pairs (clusters of two, one pair per two SMs)
// computes 256 x 256 output tiles with tcgen05.mma.cta_group::2 (M = 256,
// N = 256, K = 16); each CTA of a pair owns 128 rows of every tile.
//   warp 0      : TMA producer of A     (one 32 KB box per stage: 128 rows x two k-blocks)
//   warp 1      : allocates TMEM; lane 0 of the leader CTA issues the MMAs into one
//                 of two 256-column accumulators while the epilogue drains the other
//   warp 2      : TMA producer of B     (this CTA's 128 of the 256 B rows or columns)
//   warp 3      : TMA bulk stores of the staged 16-bit results
//   warps 4..19 : epilogue: tcgen05.ld (32 lanes x 16 columns), fp32 math, staging
// A thread's bulk-tensor copies are processed one after another, so operand
// loads come from two threads and each copy moves two k-blocks (32 KB). Loads
// take ~1.4 us under load, so the ring keeps three 64 KB stages in flight and
// the epilogue makes do with two 16 KB staging buffers.
// Every wait is bounded (~2 s of %globaltimer) and also gives up once another
// role has flagged an abort; a timeout records GM_E_TIMEOUT in an error word
// and every role unwinds.
//
// All product dimensions are multiples of 64 (the chains zero-pad otherwise;
// zero rows and columns stay zero through every product of both chains).

#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "gm_common.cuh"
#include "gm_internal.h"

namespace gm {

namespace {

constexpr int BM = 128;                // output rows per CTA
constexpr int BN = 256;                // output columns per tile
constexpr int BK = 64;                 // 64 x 16-bit = 128 B = one swizzle row
// The operand ring holds kRingKBlocks k-blocks of A and B per CTA, cut into
// stages of KPS k-blocks (a kernel template parameter): 3 stages of 2 k-blocks
// (32 KB copies) for deep products, 6 stages of 1 for short ones, where finer
// stages keep the MMAs fed across the more frequent tile changes.
constexpr int kRingKBlocks = 6;
constexpr uint32_t kKBlockBytes = 128 * BK * 2;          // 128 rows (or columns) x one k-block
constexpr uint32_t kRingBytes = 2 * kRingKBlocks * kKBlockBytes;   // A and B: 192 KB per CTA
constexpr uint64_t kWaitLimitNs = 2000000000ull;


constexpr int kEpiWarp0 = 4;
constexpr int kEpiWarps = 16;                            // four per TMEM lane quarter
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
constexpr int SLAB = 64;                                 // accumulator columns per slab
constexpr int kSlabs = BN / SLAB;
constexpr int CPW = SLAB / (kEpiWarps / 4);              // slab columns per epilogue thread
constexpr int NCH = CPW / 8;                             // 16-byte C chunks per thread per slab
static_assert(CPW == 16, "one tcgen05.ld x16 per thread per slab");

constexpr uint32_t kBoxBytes = 64 * 128;                 // 64 x 64 16-bit values
constexpr uint32_t kOutBufBytes = 2 * kBoxBytes;         // rows 0..63 and 64..127 of a slab
static_assert(BM * SLAB * 4 <= 2 * kOutBufBytes, "fp32 staging (output modes) fits the slab buffers");
constexpr uint32_t kSmemBytes = kRingBytes + 2 * kOutBufBytes + 1024 /* barriers */ + 1024 /* align */;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

__device__ int32_t g_device_error = 0;

enum EpiMode : int { EPI_STORE = 0, EPI_OUT = 1, EPI_WUPDATE = 2 };

struct GemmParams {
  int M, N, K;                 // output M x N; reduction K (multiples of 64)
  int vm, vn;                  // EPI_OUT / EPI_WUPDATE: valid rows / columns of the output
  int batch;
  int tiles_m, tiles_n;
  int sym;                     // lower-triangle schedule + mirrored store
  int f16;                     // operand / 16-bit output type: 1 fp16, 0 bf16
  float alpha, beta, gamma;    // v = alpha acc + beta Cin + gamma [r == c]
  const uint16_t* C; long long c_bs; int ldc;
  uint16_t* D; uint16_t* D2; long long d_bs; int ldd;   // 16-bit outputs (EPI_STORE)
  int has_d2; float gamma2;    // symmetric products: D2 = v + gamma2 [r == c]
  int mode;
  int transpose_out;           // EPI_OUT / EPI_WUPDATE: natural = transpose of the tile
  void* O; int odt; long long o_bs; int ldo;
  int npeers; void* peer[kMaxPeers]; const int64_t* dst_index;   // EPI_OUT to several destinations
  float* W; long long w_bs; int ldw; float eta, wd;
  const int32_t* skip;
  int32_t* err;
  uint64_t wait_ns;            // limit of every bounded wait
  int stall;                   // test hook: the operand producers issue no copies
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
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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
// Bounded wait: false once limit_ns have passed (error word and abort flag
// set), or as soon as the abort flag is seen.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int32_t* err,
                                          volatile int* abort_flag, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (abort_flag && *abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        if (err) atomicExch(err, (int32_t)GM_E_TIMEOUT);
        if (abort_flag) *abort_flag = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 4-D tile load into this CTA's shared memory, completing on the pair
// leader's barrier (`bar` is a cluster shared-memory address).
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// Bulk tensor stores of one shared-memory box; completion tracked by bulk groups.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Bulk stores committed so far have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Bulk stores committed so far have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Generic-proxy shared-memory writes become visible to the bulk-copy (async) proxy.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
// Instruction descriptor, kind::f16: D f32, A/B bf16 or f16, A K-major, M = 256.
__host__ __device__ constexpr uint32_t idesc_f16(bool f16, bool b_mn_major, int n) {
  return (1u << 4) | ((f16 ? 0u : 1u) << 7) | ((f16 ? 0u : 1u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)((2 * BM) >> 4) << 24);
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
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

__device__ __forceinline__ void tri_tile(int x, int& ti, int& tj) {
  int i = (int)((sqrtf(8.0f * (float)x + 1.0f) - 1.0f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= x) ++i;
  while (i * (i + 1) / 2 > x) --i;
  ti = i;
  tj = x - i * (i + 1) / 2;
}

// A tile of the flattened (batch, tile) list. r0 / c0 are the global row /
// column origins of this CTA's 128 rows of the 256 x 256 tile.
struct TileCoord {
  int bz, r0, c0;
};
__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int T, int tiles_per, int cr) {
  TileCoord c;
  c.bz = T / tiles_per;
  const int x = T - c.bz * tiles_per;
  int ti, tj;
  if (p.sym) tri_tile(x, ti, tj);
  else { ti = x % p.tiles_m; tj = x / p.tiles_m; }
  c.r0 = ti * 2 * BM + cr * BM;
  c.c0 = tj * BN;
  return c;
}

// ------------------------------------------------------------------ epilogue
// 16-bit results (EPI_STORE) leave through two 64 x 64 boxes per slab (rows
// 0..63 and 64..127 of the tile, the slab's 64 columns) in the 128-byte
// swizzled layout, two slab buffers alternating, written out by bulk tensor
// stores from one thread. For a symmetric product every 64 x 64 box strictly
// below the diagonal is stored as is and, from the epilogue threads'
// registers, transposed into the upper triangle (coalesced 2-byte stores: the
// 32 lanes of a warp hold 32 consecutive rows); a box on the diagonal is made
// exactly symmetric in shared memory (each lower value written at (i, j) and
// (j, i)) and stored once; boxes strictly above are not stored. The C input of
// a slab is fetched into registers one slab ahead. The epilogue warps never
// wait for one another: slab_full (all epilogue warps staged a slab) and
// buf_free (the stores of a buffer have read it) order them against the storer.
//
// fp32 results (EPI_OUT, EPI_WUPDATE: the last product of a chain) go through
// an fp32 staging tile and per-thread coalesced stores.

__device__ __forceinline__ void unpack8(const uint4 w, bool f16, float* o) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    o[2 * e] = h16_to_float(u[e] & 0xFFFF, f16);
    o[2 * e + 1] = h16_to_float(u[e] >> 16, f16);
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

// Byte offset of element (row, col) in a 64 x 64 16-bit box with the 128-byte
// swizzle (16-byte chunk index XOR row mod 8), the layout a SWIZZLE_128B
// tensor map reads from or writes to a 1024-byte aligned box.
__device__ __forceinline__ uint32_t swz(int row, int col) {
  return (uint32_t)(row * 128 + ((((col >> 3) ^ row) & 7) << 4) + (col & 7) * 2);
}

// Hand an accumulator back to the leader's MMA thread once this warp's TMEM
// reads are done (tcgen05.wait::ld has returned for all of them). The arrive is
// relaxed: a release at cluster scope waits for the SM's outstanding memory
// traffic (the operand TMA loads among it) and costs about a microsecond.
__device__ __forceinline__ void release_acc(uint32_t leader_bar, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0)
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(leader_bar)
                 : "memory");
}

// One slab of a 16-bit result, one warp: TMEM -> registers -> swizzled boxes.
// `cin` holds this thread's C values for the slab; `d2diag` the D2 values on
// the diagonal of this slab buffer. Returns true when the box lies strictly
// below the diagonal of a symmetric product: its transpose, packed in `w`,
// still has to be written (mirror_slab, after the slab is handed over).
__device__ __forceinline__ bool stage_slab(const GemmParams& p, uint8_t* buf, const uint4 (&cin)[NCH],
                                           uint32_t tacc, const TileCoord& tc, int slab, int q,
                                           int sub, int lane, uint16_t* d2diag, uint32_t (&w)[8]) {
  const int h = q >> 1;                     // 64-row box of this warp
  const int a = (q & 1) * 32 + lane;        // row inside the box
  const int cs0 = slab * SLAB;
  const int cl = sub * CPW;                 // column inside the slab
  // element (a, b) of the box lies on the global diagonal iff b == a + rel
  const int rel = tc.r0 - tc.c0 + 64 * h - cs0;
  const bool sym = p.sym != 0;
  const bool f16 = p.f16 != 0;
  uint8_t* bC = buf + h * kBoxBytes;
  float v[16];
  tmem_ld16(tacc + (uint32_t)(cs0 + cl), v);
  float x[16];
  if (p.C && p.beta != 0.f) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float c8[8];
      unpack8(cin[g], f16, c8);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[g * 8 + e] = fmaf(p.beta, c8[e], p.alpha * v[g * 8 + e]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) x[e] = p.alpha * v[e];
  }
  if (rel == 0) {
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if (cl + e == a) {
        x[e] += p.gamma;
        if (p.has_d2) d2diag[a] = float_to_h16(x[e] + p.gamma2, f16);
      }
  }
  if (sym && rel == 0) {
    // diagonal box: lower values at (a, b) and (b, a)
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int b = cl + e;
      if (b > a) continue;
      const uint16_t hv = float_to_h16(x[e], f16);
      *reinterpret_cast<uint16_t*>(bC + swz(a, b)) = hv;
      if (b < a) *reinterpret_cast<uint16_t*>(bC + swz(b, a)) = hv;
    }
    return false;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) w[e] = pack2(x[2 * e], x[2 * e + 1], f16);
  *reinterpret_cast<uint4*>(bC + swz(a, cl)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(bC + swz(a, cl + 8)) = make_uint4(w[4], w[5], w[6], w[7]);
  return sym;
}

// The transposed copy of a box strictly below the diagonal: D[c][r] = value
// (r, c) for the upper triangle, straight from registers (the 32 lanes of a
// warp hold 32 consecutive rows, so each 2-byte store instruction is coalesced).
__device__ __forceinline__ void mirror_slab(const GemmParams& p, const TileCoord& tc, int slab, int q,
                                            int sub, int lane, const uint32_t (&w)[8]) {
  const int mrow = tc.c0 + slab * SLAB + sub * CPW;       // mirror row of column cl
  const int mcol = tc.r0 + 64 * (q >> 1) + (q & 1) * 32 + lane;   // mirror column of this row
  if (mcol >= p.N) return;
  const long long off = (long long)tc.bz * p.d_bs + (long long)mrow * p.ldd + mcol;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    if (mrow + e >= p.M) break;
    const uint16_t hv = (uint16_t)(w[e >> 1] >> (16 * (e & 1)));
    p.D[off + (long long)e * p.ldd] = hv;
    if (p.has_d2) p.D2[off + (long long)e * p.ldd] = hv;
  }
}

// Stores of one staged slab (storer thread): D (and D2) with 64 x 128 boxes
// (both row boxes of the slab) or 64 x 64 boxes (one). D2 differs from D on the
// diagonal only: its diagonal box is stored from the same staging and its
// diagonal then rewritten once that copy has completed.
struct StoreMaps {
  const CUtensorMap *D, *Ds, *D2, *D2s;
};
__device__ __forceinline__ void store_slab(const GemmParams& p, const StoreMaps& m, uint8_t* buf,
                                           const TileCoord& tc, int slab, const uint16_t* d2diag) {
  const int xcol = tc.c0 + slab * SLAB;
  if (xcol >= p.N || tc.r0 >= p.M) return;
  const uint32_t s0 = smem_u32(buf), s1 = s0 + kBoxBytes;
  const bool d2 = p.has_d2 != 0;
  const int rel0 = tc.r0 - tc.c0 - slab * SLAB;   // box 0; box 1 is rel0 + 64
  int diag_row = -1;                              // first row of a diagonal box
  if (!p.sym || rel0 >= 0) {
    // both boxes on or below the diagonal
    tma_store_3d(m.D, s0, xcol, tc.r0, tc.bz);
    if (d2) tma_store_3d(m.D2, s0, xcol, tc.r0, tc.bz);
    if (p.sym && rel0 == 0) diag_row = tc.r0;
  } else if (rel0 == -64 && tc.r0 + 64 < p.M) {
    // box 0 above the diagonal, box 1 on it
    tma_store_3d(m.Ds, s1, xcol, tc.r0 + 64, tc.bz);
    if (d2) tma_store_3d(m.D2s, s1, xcol, tc.r0 + 64, tc.bz);
    diag_row = tc.r0 + 64;
  }
  if (d2 && diag_row >= 0) {
    bulk_commit();
    bulk_wait_all();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    uint16_t* dst = p.D2 + (long long)tc.bz * p.d_bs;
    for (int i = 0; i < 64 && diag_row + i < p.M && xcol + i < p.N; ++i)
      dst[(long long)(diag_row + i) * p.ldd + xcol + i] = d2diag[i];
  }
}

// One slab of an fp32 result: O = alpha acc + beta C (any output dtype) or
// W -= eta (O + wd W), in natural orientation (transposed for a tall matrix).
// C values of a slab are fetched into registers one slab ahead of their use.
__device__ __forceinline__ void c_prefetch(const GemmParams& p, const TileCoord& tc, int slab,
                                           int q, int sub, int lane, uint4 (&cpre)[NCH]) {
#pragma unroll
  for (int u = 0; u < NCH; ++u) cpre[u] = make_uint4(0, 0, 0, 0);
  if (!p.C || p.beta == 0.f) return;
  const int c0 = tc.c0 + slab * SLAB;
  if (p.sym && tc.r0 + 64 * (q >> 1) < c0) return;   // box strictly above the diagonal
  const int r = tc.r0 + q * 32 + lane;
  const int cl = sub * CPW;
  const long long cbs = (long long)tc.bz * p.c_bs;
#pragma unroll
  for (int g = 0; g < NCH; ++g)
    if (r < p.M && c0 + cl + g * 8 < p.N)
      cpre[g] = *reinterpret_cast<const uint4*>(p.C + cbs + (long long)r * p.ldc + c0 + cl + g * 8);
}

__device__ __forceinline__ void epilogue_out_slab(const GemmParams& p, uint8_t* stg, uint32_t tacc,
                                                  const TileCoord& tc, int slab, int q, int sub,
                                                  int lane, bool last_slab, uint32_t leader_bar,
                                                  uint4 (&cpre)[NCH]) {
  const int et = threadIdx.x - kEpiWarp0 * 32;
  const int rr = q * 32 + lane;             // tile row owned by this thread
  const int r0 = tc.r0;
  const int cs0 = slab * SLAB;
  const int c0 = tc.c0 + cs0;
  const bool f16 = p.f16 != 0;
  const bool tr = p.transpose_out != 0;
  float* sF = reinterpret_cast<float*>(stg);
  const int rows_valid = min(BM, p.vm - r0);
  const int cols_valid = min(SLAB, p.vn - c0);   // may be <= 0 for a ragged tile
  const float alpha = p.alpha, beta = p.beta;
  // natural layout: row-major 128 x 64 with 16-byte chunk c of row r at c ^ (r mod 16);
  // transposed: column-major (64 x 128), no padding needed
  auto fidx = [](int r, int c) { return r * SLAB + ((((c >> 2) ^ r) & 15) << 2) + (c & 3); };

  uint4 cnow[NCH];
#pragma unroll
  for (int u = 0; u < NCH; ++u) cnow[u] = cpre[u];
  if (!last_slab) c_prefetch(p, tc, slab + 1, q, sub, lane, cpre);

  // 1. TMEM -> registers -> fp32 staging
  {
    const int cl = sub * CPW;
    float v[16];
    tmem_ld16(tacc + (uint32_t)(cs0 + cl), v);
    float val[16];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float cin[8];
      unpack8(cnow[g], f16, cin);
#pragma unroll
      for (int e = 0; e < 8; ++e) val[g * 8 + e] = fmaf(beta, cin[e], alpha * v[g * 8 + e]);
    }
    if (!tr) {
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        *reinterpret_cast<float4*>(sF + fidx(rr, cl + 4 * c4)) =
            make_float4(val[4 * c4], val[4 * c4 + 1], val[4 * c4 + 2], val[4 * c4 + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) sF[(cl + e) * BM + rr] = val[e];
    }
  }
  if (last_slab) release_acc(leader_bar, lane);
  epi_bar();

  // 2. staging -> global (coalesced); two 16-byte accesses per thread in flight
  if (cols_valid > 0 && rows_valid > 0) {
    const int ld = p.mode == EPI_OUT ? p.ldo : p.ldw;
    constexpr int NB = 2;
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
          if (okc[u]) val[u] = *reinterpret_cast<const float4*>(sF + fidx(row, col));
        } else {
          const int col = idx >> 5, row = (idx & 31) * 4;   // slab column = natural row
          okc[u] = col < cols_valid && row < rows_valid;
          off[u] = (long long)(c0 + col) * ld + r0 + row;
          if (okc[u]) val[u] = *reinterpret_cast<const float4*>(sF + col * BM + row);
        }
        if (p.mode == EPI_WUPDATE && okc[u])
          wv[u] = *reinterpret_cast<const float4*>(p.W + (long long)tc.bz * p.w_bs + off[u]);
      }
#pragma unroll
      for (int u = 0; u < NB; ++u) {
        if (!okc[u]) continue;
        if (p.mode == EPI_OUT) {
          if (p.npeers == 0) {
            store4_from_float(p.O, (long long)tc.bz * p.o_bs + off[u], p.odt, val[u]);
          } else {   // every rank's receive buffer, peers' over NVLink (plain stores)
            const long long mb = p.dst_index ? p.dst_index[tc.bz] : tc.bz;
#pragma unroll
            for (int r = 0; r < kMaxPeers; ++r)
              if (r < p.npeers) store4_from_float(p.peer[r], mb * p.o_bs + off[u], p.odt, val[u]);
          }
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
  epi_bar();   // staging free for the next slab
}

// ------------------------------------------------------------------ kernel
template <bool B_MN, int KPS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmDs,
           const __grid_constant__ CUtensorMap tmD2, const __grid_constant__ CUtensorMap tmD2s,
           const GemmParams p) {
  // The skip flag is read by both CTAs of a pair before any cluster-level
  // operation, so they return together.
  if (p.skip && *p.skip) return;
  constexpr int STAGES = kRingKBlocks / KPS;
  constexpr uint32_t kABytes = KPS * kKBlockBytes;       // A and B per stage and CTA
  constexpr uint32_t kStageBytes = 2 * kABytes;
  static_assert(STAGES * KPS == kRingKBlocks, "the ring holds whole stages");

  extern __shared__ __align__(1024) uint8_t dsm[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* outbuf = base + STAGES * kStageBytes;            // [2] slab buffers
  uint64_t* full = reinterpret_cast<uint64_t*>(outbuf + 2 * kOutBufBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;     // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2] (the leader's are used)
  uint64_t* slab_full = acc_empty + 2;     // [2]
  uint64_t* buf_free = slab_full + 2;      // [2]
  uint64_t* drain = buf_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* flags = reinterpret_cast<int*>(tmem_slot + 1);
  uint16_t* d2diag = reinterpret_cast<uint16_t*>(flags + 4);   // [2][64]
  volatile int* abort_flag = flags;
  int* consumed = flags + 1;
  int* issued = flags + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t cr = cluster_rank();
  const bool leader = cr == 0;
  const int pid = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int tiles_per = p.sym ? p.tiles_m * (p.tiles_m + 1) / 2 : p.tiles_m * p.tiles_n;
  const int total = p.batch * tiles_per;
  const int nkb = p.K / BK;
  const int nst = cdiv(nkb, KPS);
  const bool store_mode = p.mode == EPI_STORE;
  constexpr uint32_t kTmemCols = 2 * BN;   // two 256-column accumulators

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 2 * kEpiWarps);
      mbar_init(smem_u32(&slab_full[a]), kEpiWarps);
      mbar_init(smem_u32(&buf_free[a]), 1);
    }
    mbar_init(smem_u32(drain), 1);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_map(&tmA);
    prefetch_map(&tmB);
    if (store_mode) {
      prefetch_map(&tmD);
      if (p.sym) prefetch_map(&tmDs);
    }
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
  // Products of a chain are launched as programmatic dependents: a CTA of the
  // next product may start (and run the prologue above) on an SM this launch
  // has left once every CTA here has finished its work; no thread touches
  // global memory before the previous product has completed and its writes are
  // visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Role dispatch by warp; within a role warp only the lanes named below work,
  // the others go straight to the final barrier.
  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // ---------------- TMA producers: warp 0 loads A, warp 2 loads B (both CTAs)
      const bool isA = warp == 0;
      uint32_t g = 0;
      bool ok = !p.stall;
      for (int T = pid; T < total && ok; T += npairs) {
        const TileCoord tc = decode_tile(p, T, tiles_per, (int)cr);
        for (int st = 0; st < nst; ++st, ++g) {
          const int s = (int)(g % STAGES);
          const uint32_t ph = (g / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, p.err, abort_flag, p.wait_ns)) { ok = false; break; }
          const uint32_t bar = map_to_rank(smem_u32(&full[s]), 0);   // the leader's barrier
          const uint32_t dst = smem_u32(base + s * kStageBytes) + (isA ? 0u : kABytes);
          if (isA) {
            if (leader) mbar_expect_tx(smem_u32(&full[s]), 2 * kStageBytes);
            tma_load_4d_pair(dst, &tmA, bar, 0, tc.r0, st * KPS, tc.bz);
          } else if (!B_MN) {
            tma_load_4d_pair(dst, &tmB, bar, 0, tc.c0 + (int)cr * 128, st * KPS, tc.bz);
          } else {
            tma_load_4d_pair(dst, &tmB, bar, 0, st * KPS * BK, (tc.c0 + (int)cr * 128) / 64, tc.bz);
          }
        }
      }
      atomicMax(issued, (int)g);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader CTA only)
      const uint32_t idesc = idesc_f16(p.f16 != 0, B_MN, BN);
      uint32_t g = 0;
      bool ok = true;
      int it = 0;
      for (int T = pid; T < total && ok; T += npairs, ++it) {
        const int ab = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(smem_u32(&acc_empty[ab]), (use & 1u) ^ 1u, p.err, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * BN);
        for (int st = 0; st < nst; ++st, ++g) {
          const int s = (int)(g % STAGES);
          const uint32_t ph = (g / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&full[s]), ph, p.err, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(base + s * kStageBytes);
          const uint32_t b_base = a_base + kABytes;
          for (int j = 0; j < KPS; ++j) {
            const int kb = st * KPS + j;
            if (kb >= nkb) break;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = sdesc(a_base + j * kKBlockBytes + kk * 32, 16, 1024);
              // MN-major B: [64-column chunk][KPS * BK rows of K][64]
              const uint64_t bd = B_MN ? sdesc(b_base + j * (BK * 128) + kk * 2048, KPS * BK * 128, 1024)
                                       : sdesc(b_base + j * kKBlockBytes + kk * 32, 16, 1024);
              umma_pair(d, ad, bd, idesc, (kb | kk) ? 1u : 0u);
            }
          }
          umma_commit_pair(smem_u32(&empty[s]));
        }
        if (!ok) break;
        umma_commit_pair(smem_u32(&acc_full[ab]));
      }
      *consumed = (int)g;
      if (!ok) *abort_flag = 1;
      // every MMA issued above has completed once this barrier fires
      umma_commit_pair(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, p.err, nullptr, p.wait_ns);
    }
  } else if (warp == 3) {
    if (lane == 0 && store_mode) {
      // ---------------- storer: bulk tensor stores of each staged slab
      const StoreMaps maps{&tmD, &tmDs, &tmD2, &tmD2s};
      uint32_t g = 0;
      bool ok = true;
      for (int T = pid; T < total && ok; T += npairs) {
        const TileCoord tc = decode_tile(p, T, tiles_per, (int)cr);
        for (int slab = 0; slab < kSlabs; ++slab, ++g) {
          const int b = (int)(g & 1u);
          const uint32_t n = g >> 1;
          if (!mbar_wait(smem_u32(&slab_full[b]), n & 1u, p.err, abort_flag, p.wait_ns)) { ok = false; break; }
          store_slab(p, maps, outbuf + b * kOutBufBytes, tc, slab, d2diag + b * 64);
          bulk_commit();
          bulk_wait_read_all();
          mbar_arrive(smem_u32(&buf_free[b]));
        }
      }
      // every slab's bulk store has read its staging by now (waited above); the
      // writes themselves complete with the grid, before any dependent launch reads them
    }
  } else {
    // ---------------- epilogue warps (both CTAs, 128 TMEM lanes each)
    const int q = warp & 3;                    // TMEM lane quarter of this warp
    const int sub = (warp - kEpiWarp0) >> 2;   // column part of each slab
    const uint32_t leader_empty0 = map_to_rank(smem_u32(&acc_empty[0]), 0);
    const uint32_t leader_empty1 = map_to_rank(smem_u32(&acc_empty[1]), 0);
    int it = 0;
    if (store_mode) {
      uint32_t g = 0;
      bool ok = true;
      for (int T = pid; T < total && ok; T += npairs, ++it) {
        const int ab = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        const TileCoord tc = decode_tile(p, T, tiles_per, (int)cr);
        uint4 cpre[NCH];
        c_prefetch(p, tc, 0, q, sub, lane, cpre);   // overlaps the MMAs of this tile
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[ab]), use & 1u, p.err, abort_flag, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tacc = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * BN);
#pragma unroll 1
        for (int slab = 0; slab < kSlabs; ++slab, ++g) {
          const int b = (int)(g & 1u);
          const uint32_t n = g >> 1;
          uint4 cnow[NCH];
#pragma unroll
          for (int u = 0; u < NCH; ++u) cnow[u] = cpre[u];
          if (n >= 1) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&buf_free[b]), (n - 1) & 1u, p.err, abort_flag, p.wait_ns));
            if (!ok) break;
          }
          // a box strictly above the diagonal of a symmetric product is never stored
          const bool skip = p.sym && tc.r0 - tc.c0 + 64 * (q >> 1) - slab * SLAB < 0;
          uint32_t w[8];
          const bool mirror =
              !skip && stage_slab(p, outbuf + b * kOutBufBytes, cnow, tacc, tc, slab, q, sub, lane,
                                  d2diag + b * 64, w);
          if (slab == kSlabs - 1) release_acc(ab ? leader_empty1 : leader_empty0, lane);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&slab_full[b]));
          // global stores and the next slab's C loads only after the hand-over, so
          // that neither the proxy fence nor the (releasing) arrive waits for them
          if (mirror) mirror_slab(p, tc, slab, q, sub, lane, w);
          if (slab + 1 < kSlabs) c_prefetch(p, tc, slab + 1, q, sub, lane, cpre);
        }
      }
    } else {
      for (int T = pid; T < total; T += npairs, ++it) {
        const int ab = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        const TileCoord tc = decode_tile(p, T, tiles_per, (int)cr);
        uint4 cpre[NCH];
        c_prefetch(p, tc, 0, q, sub, lane, cpre);
        const bool ok = mbar_wait(smem_u32(&acc_full[ab]), use & 1u, p.err, abort_flag, p.wait_ns);
        tc_fence_after();
        // the epilogue warps share named barriers here: leave together or not at all
        if (epi_any(!ok || *abort_flag)) break;
        const uint32_t tacc = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * BN);
#pragma unroll 1
        for (int slab = 0; slab < kSlabs; ++slab)
          epilogue_out_slab(p, outbuf, tacc, tc, slab, q, sub, lane, slab == kSlabs - 1,
                            ab ? leader_empty1 : leader_empty0, cpre);
      }
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && leader) {
    // after an abort, let the copies still in flight (from both CTAs) land
    for (int g = *consumed; g < *issued; ++g)
      mbar_wait(smem_u32(&full[g % STAGES]), (uint32_t)(g / STAGES) & 1u, p.err, nullptr, p.wait_ns);
  }
  cluster_sync_all();   // neither CTA leaves while the other may still signal it
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// Zero-padded copy of a batch of 16-bit matrices: Y[b][i][j] = X[b][i][j]
// inside rows x cols, 0 elsewhere in prow x pcol.
__global__ void k_pad16(int B, int rows, int cols, int prow, int pcol, const uint16_t* __restrict__ X,
                        uint16_t* __restrict__ Y) {
  const long long total = (long long)B * prow * pcol;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long b = i / ((long long)prow * pcol);
    const int r = (int)((i / pcol) % prow), c = (int)(i % pcol);
    Y[i] = (r < rows && c < cols) ? X[(b * rows + r) * cols + c] : (uint16_t)0;
  }
}

// ------------------------------------------------------------------ host side
}  // namespace

// The driver's tensor-map encoder (one function for every device of the process).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
  if (!f) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

namespace {

// Map over 16-bit elements with the 128-byte swizzle (innermost box extent 64).
bool encode(CUtensorMap* map, const void* base, bool f16, int rank, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
// [batch][rows][cols] with {64, box_rows, 1} boxes (C loads, direct and single stores).
bool map_tile(CUtensorMap* m, const void* base, bool f16, int rows, int cols, int ld, int batch,
              long long bs, int box_rows) {
  const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  const cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)bs * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  return encode(m, base, f16, 3, dims, strides, box);
}
// The same matrix viewed as [batch][cols / 64][rows][64] (64-column chunks as a
// dimension) with {64, box_rows, box_chunks, 1} boxes: box_rows rows of
// box_chunks consecutive chunks in one copy, each chunk landing as its own
// box_rows x 128 B block. Used for K-major operands (rows x K: 128 rows, one
// chunk per k-block of a stage) and the MN-major B (K rows x N: the stage's
// k-blocks of rows, two chunks = 128 columns). Requires cols % 64 == 0.
bool map_chunks(CUtensorMap* m, const void* base, bool f16, int rows, int cols, int ld, int batch,
                long long bs, int box_rows, int box_chunks) {
  const cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64), (cuuint64_t)batch};
  const cuuint64_t strides[3] = {(cuuint64_t)ld * 2, 128, (cuuint64_t)bs * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_chunks, 1};
  return encode(m, base, f16, 4, dims, strides, box);
}
// A K-major operand: 128 rows x the kps k-blocks of one stage per copy.
bool map_kmajor(CUtensorMap* m, const void* base, bool f16, int rows, int cols, int ld, int batch,
                long long bs, int kps) {
  return map_chunks(m, base, f16, rows, cols, ld, batch, bs, 128, kps);
}
// The MN-major B operand: the kps * 64 rows of K of one stage x 128 columns
// (two 64-column chunks) per copy.
bool map_mnmajor(CUtensorMap* m, const void* base, bool f16, int rows, int cols, int ld, int batch,
                 long long bs, int kps) {
  return map_chunks(m, base, f16, rows, cols, ld, batch, bs, kps * BK, 2);
}
// k-blocks per pipeline stage for a product of reduction depth K (see kRingKBlocks)
constexpr int kShortK = 1024;
int stage_kblocks(int K) { return K <= kShortK ? 1 : 2; }

// SM count of the current device (cached per device).
int num_sms() {
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

struct Maps {
  CUtensorMap A, B, D, Ds, D2, D2s;
};

template <bool B_MN, int KPS>
cudaError_t launch_gemm_t(const Maps& m, const GemmParams& p, cudaStream_t s) {
  static DeviceOnce attr;
  {
    const cudaError_t e = smem_attr_once(attr, k_gemm<B_MN, KPS>, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const int tiles = p.sym ? p.tiles_m * (p.tiles_m + 1) / 2 : p.tiles_m * p.tiles_n;
  const int total = tiles * p.batch;
  const int pairs = total < num_sms() / 2 ? total : num_sms() / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_gemm<B_MN, KPS>, m.A, m.B, m.D, m.Ds, m.D2, m.D2s, p);
}
// The operand maps must have been encoded for stage_kblocks(p.K).
template <bool B_MN>
cudaError_t launch_gemm(const Maps& m, const GemmParams& p, cudaStream_t s) {
  return stage_kblocks(p.K) == 1 ? launch_gemm_t<B_MN, 1>(m, p, s) : launch_gemm_t<B_MN, 2>(m, p, s);
}

GemmParams base_params(int M, int N, int K, int batch, bool f16, const int32_t* skip, int32_t* err) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M; p.N = N; p.K = K;
  p.vm = M; p.vn = N;
  p.batch = batch;
  p.f16 = f16 ? 1 : 0;
  p.alpha = 1.f;
  p.skip = skip;
  p.err = err;
  p.wait_ns = kWaitLimitNs;
  return p;
}

struct Ns {
  int B, N, Mp;     // padded wide form N x M' (multiples of 64)
  int vN, vMp;      // the true wide form
  bool f16;
  bool tall;        // natural = transpose of the wide form
  const int32_t* skip;
  int32_t* err;
  cudaStream_t s;
};

// Output maps and pointers of a symmetric N x N result.
bool sym_out(Maps& m, GemmParams& p, const Ns& c, uint16_t* D, uint16_t* D2) {
  const long long bs = (long long)c.N * c.N;
  if (!map_tile(&m.D, D, c.f16, c.N, c.N, c.N, c.B, bs, 128) ||
      !map_tile(&m.Ds, D, c.f16, c.N, c.N, c.N, c.B, bs, 64))
    return false;
  if (D2 && (!map_tile(&m.D2, D2, c.f16, c.N, c.N, c.N, c.B, bs, 128) ||
             !map_tile(&m.D2s, D2, c.f16, c.N, c.N, c.N, c.B, bs, 64)))
    return false;
  p.D = D; p.D2 = D2; p.d_bs = bs; p.ldd = c.N;
  p.has_d2 = D2 ? 1 : 0;
  return true;
}

// C (N x N, symmetric) = X X^T (+ epilogue), X: N x M'.
cudaError_t xxt(const Ns& c, const uint16_t* X, uint16_t* D) {
  Maps m;
  memset(&m, 0, sizeof(m));
  const long long xbs = (long long)c.N * c.Mp;
  if (!map_kmajor(&m.A, X, c.f16, c.N, c.Mp, c.Mp, c.B, xbs, stage_kblocks(c.Mp)))
    return cudaErrorInvalidValue;
  m.B = m.A;
  GemmParams p = base_params(c.N, c.N, c.Mp, c.B, c.f16, c.skip, c.err);
  if (!sym_out(m, p, c, D, nullptr)) return cudaErrorInvalidValue;
  p.tiles_m = p.tiles_n = cdiv(c.N, 2 * BM);
  p.sym = 1;
  return launch_gemm<false>(m, p, c.s);
}

// D = alpha S1 S2 + beta Cin + gamma I (symmetric N x N operands); D2 optional.
cudaError_t symmul(const Ns& c, const uint16_t* S1, const uint16_t* S2, float alpha, float beta,
                   const uint16_t* Cin, float gamma, uint16_t* D, uint16_t* D2 = nullptr,
                   float gamma2 = 0.f) {
  Maps m;
  memset(&m, 0, sizeof(m));
  const long long bs = (long long)c.N * c.N;
  const int kps = stage_kblocks(c.N);
  if (!map_kmajor(&m.A, S1, c.f16, c.N, c.N, c.N, c.B, bs, kps) ||
      !map_kmajor(&m.B, S2, c.f16, c.N, c.N, c.N, c.B, bs, kps))
    return cudaErrorInvalidValue;
  GemmParams p = base_params(c.N, c.N, c.N, c.B, c.f16, c.skip, c.err);
  if (!sym_out(m, p, c, D, D2)) return cudaErrorInvalidValue;
  p.tiles_m = p.tiles_n = cdiv(c.N, 2 * BM);
  p.sym = 1;
  p.alpha = alpha; p.beta = beta; p.gamma = gamma;
  p.C = (Cin && beta != 0.f) ? Cin : nullptr; p.c_bs = bs; p.ldc = c.N;
  p.gamma2 = gamma2;
  return launch_gemm<false>(m, p, c.s);
}

// Y = alpha S X + beta X  (S symmetric N x N, X N x M'); either stored as a new
// iterate (D) or written out in natural orientation (final step).
cudaError_t leftmul(const Ns& c, const uint16_t* S, const uint16_t* X, float alpha, float beta,
                    uint16_t* D, const NsOutput* out) {
  Maps m;
  memset(&m, 0, sizeof(m));
  const long long xbs = (long long)c.N * c.Mp;
  const int kps = stage_kblocks(c.N);
  if (!map_kmajor(&m.A, S, c.f16, c.N, c.N, c.N, c.B, (long long)c.N * c.N, kps) ||
      // MN-major B operand: rows of X are the K index, 64-column chunks the N index
      !map_mnmajor(&m.B, X, c.f16, c.N, c.Mp, c.Mp, c.B, xbs, kps))
    return cudaErrorInvalidValue;
  GemmParams p = base_params(c.N, c.Mp, c.N, c.B, c.f16, c.skip, c.err);
  p.tiles_m = cdiv(c.N, 2 * BM);
  p.tiles_n = cdiv(c.Mp, BN);
  p.alpha = alpha; p.beta = beta;
  p.C = beta != 0.f ? X : nullptr; p.c_bs = xbs; p.ldc = c.Mp;
  if (!out) {
    p.mode = EPI_STORE;
    if (!map_tile(&m.D, D, c.f16, c.N, c.Mp, c.Mp, c.B, xbs, 128)) return cudaErrorInvalidValue;
    p.D = D; p.d_bs = xbs; p.ldd = c.Mp;
  } else {
    p.vm = c.vN; p.vn = c.vMp;
    p.transpose_out = c.tall ? 1 : 0;
    const int ld = c.tall ? c.vN : c.vMp;   // natural row length
    if (out->mode == 0) {
      p.mode = EPI_OUT;
      p.O = out->O; p.odt = out->odt; p.o_bs = (long long)c.vN * c.vMp; p.ldo = ld;
      p.npeers = out->npeers;
      for (int r = 0; r < kMaxPeers; ++r) p.peer[r] = r < out->npeers ? out->peer[r] : nullptr;
      p.dst_index = out->dst_index;
    } else {
      p.mode = EPI_WUPDATE;
      p.W = out->W; p.w_bs = (long long)c.vN * c.vMp; p.ldw = ld;
      p.eta = out->eta; p.wd = out->wd;
    }
  }
  return launch_gemm<true>(m, p, c.s);
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

size_t al256(size_t b) { return (b + 255) & ~size_t(255); }
int pad64(int x) { return (x + 63) & ~63; }

struct NsDims {
  int N, Mp, Np, Mpp;
  bool padded;
};
NsDims ns_dims(int m, int n) {
  NsDims d;
  d.N = m < n ? m : n;
  d.Mp = m < n ? n : m;
  d.Np = pad64(d.N);
  d.Mpp = pad64(d.Mp);
  d.padded = d.Np != d.N || d.Mpp != d.Mp;
  return d;
}

// The chain's iterate starts in X16 (true shape) or, when a dimension is not
// a multiple of 64, in a zero-padded copy.
cudaError_t ns_setup(const NsDims& d, int B, uint16_t* X16, uint8_t*& cur, uint16_t** X,
                     uint16_t** Xn, cudaStream_t s) {
  const size_t xbytes = (size_t)B * d.Np * d.Mpp * 2;
  *Xn = reinterpret_cast<uint16_t*>(carve(cur, xbytes));
  if (!d.padded) {
    *X = X16;
    return cudaSuccess;
  }
  *X = reinterpret_cast<uint16_t*>(carve(cur, xbytes));
  const long long total = (long long)B * d.Np * d.Mpp;
  const int blocks = (int)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  k_pad16<<<blocks, 256, 0, s>>>(B, d.N, d.Mp, d.Np, d.Mpp, X16, *X);
  return cudaGetLastError();
}

}  // namespace

size_t ns_standard_ws_bytes(int B, int m, int n) {
  const NsDims d = ns_dims(m, n);
  return (d.padded ? 2 : 1) * al256((size_t)B * d.Np * d.Mpp * 2) + 2 * al256((size_t)B * d.Np * d.Np * 2);
}
size_t ns_gram_ws_bytes(int B, int m, int n) {
  const NsDims d = ns_dims(m, n);
  return (d.padded ? 2 : 1) * al256((size_t)B * d.Np * d.Mpp * 2) + 6 * al256((size_t)B * d.Np * d.Np * 2);
}

cudaError_t run_ns_standard(int B, int m, int n, uint16_t* X16, const float* abc, int T,
                            const NsOutput& out, void* ws, const int32_t* skip, int32_t* err,
                            cudaStream_t s) {
  const NsDims d = ns_dims(m, n);
  Ns c{B, d.Np, d.Mpp, d.N, d.Mp, false, m > n, skip, err ? err : device_error_word(), s};
  uint8_t* cur = static_cast<uint8_t*>(ws);
  uint16_t *X, *Xn;
  GM_TRY(ns_setup(d, B, X16, cur, &X, &Xn, s));
  uint16_t* A = reinterpret_cast<uint16_t*>(carve(cur, (size_t)B * c.N * c.N * 2));
  uint16_t* Bm = reinterpret_cast<uint16_t*>(carve(cur, (size_t)B * c.N * c.N * 2));
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
                        const int32_t* skip, int32_t* err, cudaStream_t s, uint16_t* Rtrace,
                        uint16_t* Qtrace) {
  const NsDims d = ns_dims(m, n);
  Ns c{B, d.Np, d.Mpp, d.N, d.Mp, true, m > n, skip, err ? err : device_error_word(), s};
  uint8_t* cur = static_cast<uint8_t*>(ws);
  uint16_t *X, *Xn;
  GM_TRY(ns_setup(d, B, X16, cur, &X, &Xn, s));
  const size_t nn = (size_t)B * c.N * c.N * 2;
  uint16_t* R = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Rn = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Z = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Q = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* Qn = reinterpret_cast<uint16_t*>(carve(cur, nn));
  uint16_t* RZ = reinterpret_cast<uint16_t*>(carve(cur, nn));
  bool restart_at[GM_MAX_T + 1] = {false};
  for (int i = 0; i < n_restart; ++i)
    if (restart_after[i] >= 1 && restart_after[i] < T) restart_at[restart_after[i]] = true;
  GM_TRY(xxt(c, X, R));                                    // R = X X^T
  bool q_is_identity = true;
  // optional per-step copies of R_t and Q_t (padded N x N blocks of the batch)
  auto dump = [&](uint16_t* trace, const uint16_t* src, int t) -> cudaError_t {
    if (!trace) return cudaSuccess;
    return cudaMemcpyAsync(trace + (size_t)(t - 1) * B * c.N * c.N, src, nn, cudaMemcpyDeviceToDevice, s);
  };
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
    GM_TRY(dump(Qtrace, Q, t));
    if (!block_end) {
      GM_TRY(symmul(c, R, Z, 1.f, a, R, 0.f, RZ));          // RZ = R Z + a R
      GM_TRY(symmul(c, Z, RZ, 1.f, a, RZ, 0.f, Rn));        // R = Z RZ + a RZ
      uint16_t* tr = R; R = Rn; Rn = tr;
      GM_TRY(dump(Rtrace, R, t));
    } else if (t < T) {
      GM_TRY(leftmul(c, Q, X, 1.f, 0.f, Xn, nullptr));      // restart: X = Q X
      uint16_t* tx = X; X = Xn; Xn = tx;
      GM_TRY(xxt(c, X, R));
      GM_TRY(dump(Rtrace, R, t));
      q_is_identity = true;
    } else {
      GM_TRY(leftmul(c, Q, X, 1.f, 0.f, nullptr, &out));    // O = Q X
    }
  }
  return cudaSuccess;
}

cudaError_t run_wait_timeout_probe(const uint16_t* X, uint16_t* D, uint64_t limit_ns, cudaStream_t s) {
  // one 256 x 256 bf16 X X^T tile whose operand producers issue nothing: the MMA
  // issuer's wait for the first stage runs out after limit_ns, records
  // GM_E_TIMEOUT in the error word and every role unwinds
  Ns c{1, 256, 256, 256, 256, false, false, nullptr, device_error_word(), s};
  Maps m;
  memset(&m, 0, sizeof(m));
  if (!c.err) return cudaErrorInvalidValue;
  if (!map_kmajor(&m.A, X, false, 256, 256, 256, 1, 256 * 256, stage_kblocks(256)))
    return cudaErrorInvalidValue;
  m.B = m.A;
  GemmParams p = base_params(256, 256, 256, 1, false, nullptr, c.err);
  if (!sym_out(m, p, c, D, nullptr)) return cudaErrorInvalidValue;
  p.tiles_m = p.tiles_n = 1;
  p.sym = 1;
  p.wait_ns = limit_ns;
  p.stall = 1;
  return launch_gemm<false>(m, p, s);
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

// Device address of the error word on the current device (looked up with that
// device current, cached per device).
int32_t* device_error_word() {
  static std::atomic<int32_t*> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  int32_t* ptr = cache[dev].load(std::memory_order_acquire);
  if (!ptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptr = static_cast<int32_t*>(p);
    cache[dev].store(ptr, std::memory_order_release);
  }
  return ptr;
}

}  // namespace gm
