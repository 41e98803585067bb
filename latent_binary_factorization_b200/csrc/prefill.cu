// Prefill forward (batch M >= 128, multiple of 128) of the LittleBit layer on
// the sm_100a tensor cores (tcgen05.mma, fp32 accumulators in tensor memory).
//
//   y = sum_p h_p (.) ( U_p ( l_p (.) ( V_p^T ( g_p (.) x ) ) ) )
// (Samsung LittleBit article, section 2) as two thin matrix products:
//   GEMM1  T  = X * B1^T,  B1 = [V_1 (.) g_1 | V_2 (.) g_2]^T   (P*Sp x d_in)
//          T' = l (.) T   (fp16)
//   GEMM2  Y  = T' * B2^T, B2 = [U_1 (.) h_1 | U_2 (.) h_2]      (d_out x P*Sp)
// The scales ride in the +-1 operands: V[i][j] * g[i] and U[o][j] * h[o] are
// exactly +-g[i] and +-h[o] in fp16, so both products are exact, and putting
// the two residual paths side by side along N (GEMM1) and along K (GEMM2)
// makes the path sum part of the accumulation.  x is taken to fp16 (exact for
// bf16 values in fp16's normal range); t' is rounded once to fp16; y is
// rounded once to its output type.
//
// Operand layout ("core-matrix tiles"): an R x K fp16 operand (K contraction,
// R a multiple of 8, K of 64) is stored K-block major: for each 64-wide
// K-block, row-groups of 8 rows, each 1 KB = eight 8x8 core matrices (8 rows
// x 16 bytes) along K.  Element (r, k) is at byte
//   ((k/64) * (R/8) + r/8) * 1024 + ((k%64)/8) * 128 + (r%8) * 16 + (k%8) * 2.
// So the rows r0..r0+T-1 of one K-block are T/8 contiguous KB: one bulk copy
// brings a whole stage, and in shared memory it is the canonical K-major
// no-swizzle UMMA layout (core matrices 128 B apart along K, row-groups 1 KB
// apart).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <array>
#include <cstring>
#include <functional>
#include <map>
#include <queue>
#include <utility>
#include <vector>

#include "lb_internal.h"

namespace lb {
namespace {

constexpr int kBM = 128;          // rows per tile (UMMA M)
constexpr int kBN = 256;          // max columns per tile (UMMA N)
constexpr int kBK = 64;           // K per stage
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kYPitch = 144;             // y staging row: 64 outputs (128 B) + 16 B against bank conflicts

__host__ __device__ __forceinline__ size_t tiled_off(int r, int k, int R) {
  return ((size_t)(k >> 6) * (R >> 3) + (r >> 3)) * 1024 + ((k & 63) >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2;
}

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t su(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su(b)), "r"(parity), "r"(1000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
  for (int i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(b, parity)) return true;
  return false;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(su(dst)),
      "l"(src), "r"(bytes), "r"(su(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// shared-memory matrix descriptor: K-major, no swizzle; LBO = distance between
// core matrices along K, SBO = distance between 8-row groups
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version
  return d;                 // base offset 0, relative LBO, no swizzle
}

// instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 D, M x N
__device__ __forceinline__ uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4)                           // D = F32
         | (0u << 7) | (0u << 10)            // A, B = F16
         | ((uint32_t)(N >> 3) << 17)        // N / 8
         | ((uint32_t)(M >> 4) << 24);       // M / 16
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on `bar` once every tcgen05.mma issued so far by this thread is done
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su(bar))
               : "memory");
}

// 32 lanes x 16 fp32 columns: this thread's TMEM lane, columns col..col+15
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  // the registers are valid only after wait::ld: thread them through it so
  // that no use can be scheduled before the wait
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------------ operand preparation

// x (M x K, fp16 or bf16, row-major) -> fp16 core-matrix tiles.  Work unit =
// one 16-byte chunk of the output; eight consecutive units read one 128-byte
// run of a row.  Each thread takes kXUnroll units spaced a grid apart and
// issues all their loads before converting, so several loads are in flight.
constexpr int kXUnroll = 4;
// Preparation blocks (256 threads, <= 40 registers) per SM in one launch: three
// leave room for a GEMM CTA beside them.
constexpr int kPrepBlocksPerSm = 3;

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  uint32_t* w = &v.x;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
    const __half2 h = __floats2half2_rn(__bfloat162float(b.x), __bfloat162float(b.y));
    w[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return v;
}

// The three preparation steps below each run as one grouped launch over all
// layers of a chunk: a layer owns a contiguous range of blocks (PrepJob) and
// its step runs with block `bid` of `nblk` in place of blockIdx/gridDim.
// An fp16 value that is inf or NaN after the conversion (a bf16 input beyond
// fp16's finite range, or a non-finite input) raises LB_ERR_RANGE in *status.
__device__ __forceinline__ void prep_x(const uint16_t* __restrict__ x, int is_bf16, int M, int K,
                                       unsigned char* __restrict__ out, unsigned bid, unsigned nblk,
                                       unsigned int* status) {
  unsigned bad = 0;
  const unsigned n16 = (unsigned)((size_t)M * K / 8);   // < 2^32 for the shapes accepted
  const unsigned rgs = (unsigned)M >> 3;
  const unsigned stride = nblk * blockDim.x;
  for (unsigned t0 = bid * blockDim.x + threadIdx.x; t0 < n16; t0 += stride * kXUnroll) {
    uint4 v[kXUnroll];
    unsigned dst[kXUnroll];
#pragma unroll
    for (int u = 0; u < kXUnroll; ++u) {
      const unsigned t = t0 + u * stride;
      if (t < n16) {
        const unsigned kc = t & 7, rr = (t >> 3) & 7, blk = t >> 6;   // blk: (K-block, row-group) KB
        const unsigned kb = blk / rgs, rg = blk - kb * rgs;
        v[u] = *reinterpret_cast<const uint4*>(x + (size_t)(8 * rg + rr) * K + 64 * kb + 8 * kc);
        dst[u] = blk * 1024 + kc * 128 + rr * 16;
      }
    }
#pragma unroll
    for (int u = 0; u < kXUnroll; ++u) {
      if (t0 + u * stride < n16) {
        const uint4 h = is_bf16 ? bf16x8_to_f16x8(v[u]) : v[u];
        bad |= half2_nonfinite(h.x) | half2_nonfinite(h.y) | half2_nonfinite(h.z) | half2_nonfinite(h.w);
        *reinterpret_cast<uint4*>(out + dst[u]) = h;
      }
    }
  }
  if (bad) atomicOr(status, kStatusRange);
}

// The bit of word w (of a packed tile's 16-byte lane) for product q, as the
// fp16 sign bits of four consecutive elements: byte m of (w >> q) & 0x01010101
// is element m's sign.
__device__ __forceinline__ uint2 sign_bits4(uint32_t w, int q) {
  const uint32_t bits = (w >> q) & 0x01010101u;
  return make_uint2(((bits & 1u) << 15) | (((bits >> 8) & 1u) << 31),
                    (((bits >> 16) & 1u) << 15) | (((bits >> 24) & 1u) << 31));
}

// B1 (P*Sp rows x d_in): row p*Sp + j holds V_p[i][j] * g_p[i].  One warp per
// packed role-V tile (16 rows j x 256 inputs i): each lane loads its 16-byte
// lane of the tile once; word r, product q gives four consecutive i of one row,
// i.e. one 8-byte piece of B1, for 32 pieces per lane.  For each (q, r) the
// warp's pieces cover two whole 128-byte core-matrix rows.  g is read through
// L1 (8 bytes per lane and q, shared by the tile's rows).  Rows j >= s inside
// the packed tiles get +-g (finite; GEMM1's epilogue zeroes them through l);
// rows from the tiles' end up to Sp are zero, written by the same threads in
// 16-byte pieces after the tiles.
__device__ __forceinline__ void prep_b1(const LayerDesc& L, int Sp, unsigned char* __restrict__ out, unsigned bid,
                                        unsigned nblk) {
  const int R = L.npaths * Sp, K = L.d_in;
  const int n_kt = K / kVTileK, n_rb = (L.s + 15) >> 4;
  const unsigned tiles_p = (unsigned)(n_rb * n_kt);
  const unsigned tiles = (unsigned)L.npaths * tiles_p;
  const int lane = threadIdx.x & 31, gg = lane >> 2, c = lane & 3;
  const unsigned nwarps = nblk * (blockDim.x >> 5);
  for (unsigned tile = bid * (blockDim.x >> 5) + (threadIdx.x >> 5); tile < tiles; tile += nwarps) {
    const int p = tile >= tiles_p ? 1 : 0;
    const int tt = (int)(tile - p * tiles_p);
    const int rb = tt / n_kt, kt = tt - rb * n_kt;
    const uint4 wv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned char*>(L.p[p].V) +
                                                          (size_t)tt * kTileBytes) + lane);
    const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
    const uint16_t* g = L.p[p].g;
    const int j0 = p * Sp + 16 * rb + gg;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
        const int i0 = 256 * kt + 32 * q + 16 * rh + 4 * c;
        const uint2 gv = __ldg(reinterpret_cast<const uint2*>(g + i0));
#pragma unroll
        for (int rl = 0; rl < 2; ++rl) {
          const uint2 sg = sign_bits4(w[2 * rh + rl], q);
          *reinterpret_cast<uint2*>(out + tiled_off(j0 + 8 * rl, i0, R)) = make_uint2(gv.x ^ sg.x, gv.y ^ sg.y);
        }
      }
    }
  }
  const unsigned zrow16 = (unsigned)(K / 8);                    // 16-byte pieces per zero row
  const int per = Sp - 16 * n_rb;
  const unsigned zeros = (unsigned)(L.npaths * per) * zrow16;
  for (unsigned z = bid * blockDim.x + threadIdx.x; z < zeros; z += nblk * blockDim.x) {
    const unsigned row_i = z / zrow16;
    const int k = (int)(z - row_i * zrow16) * 8;
    const int p = (int)row_i / per, jr = p * Sp + 16 * n_rb + ((int)row_i - p * per);
    *reinterpret_cast<uint4*>(out + tiled_off(jr, k, R)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// B2 (d_out rows x P*Sp): row o, column p*Sp + j holds U_p[o][j] * h_p[o].  One
// warp per packed role-U tile (128 rows o x 32 latent j), as prep_b1: word r,
// product q of a lane gives four consecutive j of row o = 128*ob + 16*q + gg +
// 8*(r&1).  Columns from the tiles' end up to Sp are zero.
__device__ __forceinline__ void prep_b2(const LayerDesc& L, int Sp, unsigned char* __restrict__ out, unsigned bid,
                                        unsigned nblk) {
  const int R = L.d_out;
  const int n_kt = (L.s + 31) >> 5, n_ob = R / kUTileRows;
  const unsigned tiles_p = (unsigned)(n_ob * n_kt);
  const unsigned tiles = (unsigned)L.npaths * tiles_p;
  const int lane = threadIdx.x & 31, gg = lane >> 2, c = lane & 3;
  const unsigned nwarps = nblk * (blockDim.x >> 5);
  for (unsigned tile = bid * (blockDim.x >> 5) + (threadIdx.x >> 5); tile < tiles; tile += nwarps) {
    const int p = tile >= tiles_p ? 1 : 0;
    const int tt = (int)(tile - p * tiles_p);
    const int ob = tt / n_kt, kt = tt - ob * n_kt;
    const uint4 wv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned char*>(L.p[p].U) +
                                                          (size_t)tt * kTileBytes) + lane);
    const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
    const uint16_t* h = L.p[p].h;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
#pragma unroll
      for (int rl = 0; rl < 2; ++rl) {
        const int o = kUTileRows * ob + 16 * q + gg + 8 * rl;
        const uint32_t hv = (uint32_t)__ldg(h + o) * 0x00010001u;
#pragma unroll
        for (int rh = 0; rh < 2; ++rh) {
          const int j0 = p * Sp + 32 * kt + 16 * rh + 4 * c;
          const uint2 sg = sign_bits4(w[2 * rh + rl], q);
          *reinterpret_cast<uint2*>(out + tiled_off(o, j0, R)) = make_uint2(hv ^ sg.x, hv ^ sg.y);
        }
      }
    }
  }
  const int zc8 = (Sp - 32 * n_kt) / 8;                    // zero 16-byte pieces per row and path
  const unsigned per = (unsigned)(R * zc8);
  const unsigned zeros = (unsigned)L.npaths * per;
  for (unsigned z = bid * blockDim.x + threadIdx.x; z < zeros; z += nblk * blockDim.x) {
    const int p = (int)(z / per);
    const int zz = (int)(z - (unsigned)p * per);
    const int o = zz / zc8, j = p * Sp + 32 * n_kt + (zz - o * zc8) * 8;
    *reinterpret_cast<uint4*>(out + tiled_off(o, j, R)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// One layer of a chunk in the grouped preparation launches: its arguments and
// the first block it owns in each of the three launches (blocks first[k] up to
// the next layer's first[k], or the grid's end, belong to it).
struct PrepJob {
  LayerDesc L;
  const uint16_t* x;        // the activations, or (expand calls) the cache rows
  unsigned char *X16, *B1, *B2, *T;
  int M, x_bf16, Sp;
  int first[kPrepKinds];    // 0: x, 1: B1, 2: B2, 3: T' from cache rows
};

// T' (M x npaths*Sp core-matrix tiles, the A operand of GEMM2) from the
// caller's cache rows: element (r, p*Sp + j) = cache[r * t_ld + p*s + j] for
// j < s, else 0.  Work unit = one 16-byte piece (8 consecutive columns of one
// row) of the tiles; the cache offsets need not be 16-byte aligned, so the
// piece is gathered element by element.
__device__ __forceinline__ void prep_t(const uint16_t* __restrict__ tc, const LayerDesc& L, int M, int Sp,
                                       unsigned char* __restrict__ out, unsigned bid, unsigned nblk) {
  const int NK = L.npaths * Sp;
  const unsigned pieces = (unsigned)M * (unsigned)(NK / 8);
  for (unsigned t = bid * blockDim.x + threadIdx.x; t < pieces; t += nblk * blockDim.x) {
    const int r = (int)(t / (unsigned)(NK / 8)), k0 = (int)(t - (unsigned)r * (NK / 8)) * 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      uint32_t lo = 0, hi = 0;
      const int k = k0 + e;
      const int p0 = k / Sp, j0 = k - p0 * Sp, p1 = (k + 1) / Sp, j1 = k + 1 - p1 * Sp;
      if (j0 < L.s) lo = tc[(size_t)r * L.t_ld + p0 * L.s + j0];
      if (j1 < L.s) hi = tc[(size_t)r * L.t_ld + p1 * L.s + j1];
      w[e >> 1] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(out + tiled_off(r, k0, M)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// The job that owns block b of launch k: the last one whose first[k] <= b.
__device__ __forceinline__ int prep_job_of(const PrepJob* jobs, int n, int k, unsigned b) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((unsigned)jobs[mid].first[k] <= b) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int KIND>
__global__ void __launch_bounds__(256) prep_group_kernel(const PrepJob* __restrict__ jobs, int n,
                                                         unsigned int* status) {
  const int j = prep_job_of(jobs, n, KIND, blockIdx.x);
  const PrepJob& J = jobs[j];
  const unsigned b0 = (unsigned)J.first[KIND];
  const unsigned b1 = j + 1 < n ? (unsigned)jobs[j + 1].first[KIND] : gridDim.x;
  const unsigned bid = blockIdx.x - b0, nblk = b1 - b0;
  if (KIND == 0) prep_x(J.x, J.x_bf16, J.M, J.L.d_in, J.X16, bid, nblk, status);
  else if (KIND == 1) prep_b1(J.L, J.Sp, J.B1, bid, nblk);
  else if (KIND == 2) prep_b2(J.L, J.Sp, J.B2, bid, nblk);
  else prep_t(J.x, J.L, J.M, J.Sp, J.T, bid, nblk);
}

// ------------------------------------------------------------------ grouped persistent tcgen05 GEMM
//
// One launch computes every tile of a list of problems D = A * B^T (M x N,
// fp32 in tensor memory).  Warp 0 lane 0 streams A/B stages with bulk copies,
// warp 1 lane 0 issues tcgen05.mma, warps 2..5 drain the accumulator; two
// 256-column accumulators alternate so a tile's epilogue overlaps the next
// tile's products.

struct GemmProblem {
  const unsigned char* A;   // core-matrix tiles, M rows x K
  const unsigned char* B;   // core-matrix tiles, N rows x K
  int M, N, K, mode;        // mode 0: T' = l * acc -> fp16 tiles; 1: y = acc -> row-major;
                            // 2: T' = l * acc -> fp16 cache rows (latent-only calls)
  const uint16_t* l0;
  const uint16_t* l1;
  int s, Sp;
  unsigned char* T;         // mode 0 output, core-matrix tiles M x N
  void* Y;                  // mode 1 output, row-major M x N; mode 2: cache rows, t_ld apart
  int y_bf16, t_ld;
  int tiles_n, tile_w;      // N is cut into tiles_n column tiles of tile_w (the last may be narrower)
  int tile_begin;
};

// Tiles of CTA b: sched[begin[b] .. begin[b+1]), built on the host (longest
// first, each to the least-loaded CTA).
struct GroupArgs {
  const GemmProblem* probs;
  const int* sched;
  const int* begin;
  int n_probs, total_tiles;
  unsigned int* status;
};

constexpr int kGroupThreads = 192;

// The pair kernel (below): 256-row tiles, each CTA of the pair holding 128
// rows of A and half of B's rows per stage.
constexpr int kPairStages = 6;
constexpr int kPairBBytes = kBN / 2 * kBK * 2;   // 16 KB

struct TileInfo {
  const GemmProblem* P;
  int m0, n0, n_len, nk;
};

// Tile `tile` of the problem list; m-tiles are `rows` high (128, or 256 for
// a pair of CTAs).
__device__ __forceinline__ TileInfo tile_info(const GroupArgs& ga, int tile, int rows) {
  int lo = 0, hi = ga.n_probs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ga.probs[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  TileInfo ti;
  ti.P = ga.probs + lo;
  const int local = tile - ti.P->tile_begin;
  const int mt = local / ti.P->tiles_n, nt = local - mt * ti.P->tiles_n;
  ti.m0 = mt * rows;
  ti.n0 = nt * ti.P->tile_w;
  ti.n_len = min(ti.P->tile_w, ti.P->N - ti.n0);
  ti.nk = ti.P->K / kBK;
  return ti;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su(b)) : "memory");
}

// Drains one accumulator into the tile's output.  The calling warp reads TMEM
// lanes 32*quarter .. +31 from taddr on, which hold output rows
// row0 + 32*quarter + lane; `bad` collects fp16 values beyond range.
__device__ __forceinline__ void epilogue_tile(const TileInfo& ti, uint32_t taddr, int row0, int quarter, int lane,
                                              unsigned char* ystage, unsigned& bad) {
  const GemmProblem& P = *ti.P;
  const int row = row0 + 32 * quarter + lane;
  if (P.mode == 1) {
    // y: 64 columns at a time through shared memory, so that eight lanes
    // write one row's 128 contiguous bytes
    unsigned char* sy = ystage + (size_t)quarter * 32 * kYPitch;
    for (int c0 = 0; c0 < ti.n_len; c0 += 64) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float v[16];
        tmem_ld16(taddr + (uint32_t)(c0 + 16 * h), v);
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          if (P.y_bf16) {
            const __nv_bfloat162 bb = __floats2bfloat162_rn(v[e], v[e + 1]);
            w[e >> 1] = *reinterpret_cast<const uint32_t*>(&bb);
          } else {
            const __half2 hh = __floats2half2_rn(v[e], v[e + 1]);
            w[e >> 1] = *reinterpret_cast<const uint32_t*>(&hh);
            bad |= half2_nonfinite(w[e >> 1]);
          }
        }
        *reinterpret_cast<uint4*>(sy + lane * kYPitch + 32 * h) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(sy + lane * kYPitch + 32 * h + 16) = make_uint4(w[4], w[5], w[6], w[7]);
      }
      __syncwarp();
      const int cb = lane & 7;
#pragma unroll
      for (int r4 = 0; r4 < 32; r4 += 4) {
        const int r = r4 + (lane >> 3);
        const uint4 val = *reinterpret_cast<const uint4*>(sy + r * kYPitch + cb * 16);
        uint16_t* yr = static_cast<uint16_t*>(P.Y) + (size_t)(row0 + 32 * quarter + r) * P.N + ti.n0 + c0;
        *reinterpret_cast<uint4*>(yr + 8 * cb) = val;
      }
      __syncwarp();
    }
    return;
  }
  for (int c0 = 0; c0 < ti.n_len; c0 += 16) {
    float v[16];
    tmem_ld16(taddr + (uint32_t)c0, v);
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      float lv[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int n = ti.n0 + c0 + e + u;
        const int p = n / P.Sp, j = n - p * P.Sp;
        const uint16_t* l = p == 0 ? P.l0 : P.l1;
        lv[u] = j < P.s ? __half2float(__ushort_as_half(l[j])) : 0.f;
      }
      const __half2 hh = __floats2half2_rn(lv[0] * v[e], lv[1] * v[e + 1]);
      w[e >> 1] = *reinterpret_cast<const uint32_t*>(&hh);
      bad |= half2_nonfinite(w[e >> 1]);
    }
    if (P.mode == 0) {
      *reinterpret_cast<uint4*>(P.T + tiled_off(row, ti.n0 + c0, P.M)) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(P.T + tiled_off(row, ti.n0 + c0 + 8, P.M)) = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
      // cache row: path p's t'_j at column p*s + j, j < s
      uint16_t* yr = static_cast<uint16_t*>(P.Y) + (size_t)row * P.t_ld;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int n = ti.n0 + c0 + e;
        const int p = n / P.Sp, j = n - p * P.Sp;
        if (j < P.s) yr[p * P.s + j] = (uint16_t)(w[e >> 1] >> (16 * (e & 1)));
      }
    }
  }
}

__global__ void __launch_bounds__(kGroupThreads, 1) umma_group_kernel(const GroupArgs ga) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* sA = smem;
  unsigned char* sB = smem + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
  // y staging of the epilogue warps: [4 warps][32 rows][kYPitch bytes]
  unsigned char* ystage = smem + kStages * (kABytes + kBBytes) + 1024;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su(tmem_slot)),
                 "r"(2 * kBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool dead = false;

  if (threadIdx.x == 0) {
    // ---- producer
    uint32_t it = 0;
    for (int k = ga.begin[blockIdx.x]; k < ga.begin[blockIdx.x + 1]; ++k) {
      const TileInfo ti = tile_info(ga, ga.sched[k], kBM);
      const uint32_t bbytes = (uint32_t)ti.n_len * kBK * 2;
      const int Mg = ti.P->M >> 3, Ng = ti.P->N >> 3;
      for (int kb = 0; kb < ti.nk; ++kb, ++it) {
        const int st = it % kStages;
        if (it >= kStages && !dead && !mbar_wait(&empty[st], ((it / kStages) - 1) & 1)) dead = true;
        mbar_expect_tx(&full[st], kABytes + bbytes);
        bulk_g2s(sA + st * kABytes, ti.P->A + ((size_t)kb * Mg + (ti.m0 >> 3)) * 1024, kABytes, &full[st]);
        bulk_g2s(sB + st * kBBytes, ti.P->B + ((size_t)kb * Ng + (ti.n0 >> 3)) * 1024, bbytes, &full[st]);
      }
    }
  } else if (threadIdx.x == 32) {
    // ---- MMA issuer
    uint32_t it = 0, nt = 0;
    for (int k = ga.begin[blockIdx.x]; k < ga.begin[blockIdx.x + 1]; ++k, ++nt) {
      const TileInfo ti = tile_info(ga, ga.sched[k], kBM);
      const int ab = nt & 1;
      if (nt >= 2 && !dead && !mbar_wait(&acce[ab], ((nt >> 1) - 1) & 1)) dead = true;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(ab * kBN);
      const uint32_t idesc = umma_idesc_f16(kBM, ti.n_len);
      for (int kb = 0; kb < ti.nk; ++kb, ++it) {
        const int st = it % kStages;
        if (!dead && !mbar_wait(&full[st], (it / kStages) & 1)) dead = true;
        tc_fence_after();
        const uint32_t a0 = su(sA + st * kABytes), b0 = su(sB + st * kBBytes);
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks)
          umma_f16(d, umma_desc(a0 + ks * 256, 128, 1024), umma_desc(b0 + ks * 256, 128, 1024), idesc,
                   (kb > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&empty[st]);
      }
      umma_commit(&accf[ab]);
    }
  } else if (warp >= 2) {
    // ---- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
    const int quarter = warp & 3;
    uint32_t nt = 0;
    unsigned bad = 0;   // a t' (or fp16 y) beyond fp16's range: LB_ERR_RANGE
    for (int k = ga.begin[blockIdx.x]; k < ga.begin[blockIdx.x + 1]; ++k, ++nt) {
      const TileInfo ti = tile_info(ga, ga.sched[k], kBM);
      const int ab = nt & 1;
      if (!dead && !mbar_wait(&accf[ab], (nt >> 1) & 1)) dead = true;
      dead = __any_sync(0xffffffffu, dead);
      tc_fence_after();
      epilogue_tile(ti, tmem + (uint32_t)(ab * kBN) + ((uint32_t)(32 * quarter) << 16), ti.m0, quarter, lane,
                    ystage, bad);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[ab]);
    }
    if (dead && lane == 0) atomicOr(ga.status, kStatusTimeout);
    if (__any_sync(0xffffffffu, bad != 0) && lane == 0) atomicOr(ga.status, kStatusRange);
  }
  if ((threadIdx.x == 0 || threadIdx.x == 32) && dead) atomicOr(ga.status, kStatusTimeout);
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kBN) : "memory");
  }
}

// ---- helpers of the pair kernel

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of this CTA's variable p in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(su(p)), "r"(rank));
  return a;
}
// arrive on a barrier of another CTA of the cluster (or this one), given its
// shared::cluster address
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// every thread of both CTAs
__device__ __forceinline__ void pair_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void umma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on `bar` of both CTAs of the pair once every pair product issued so
// far by this thread is done
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  const uint16_t both = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          su(bar)),
      "h"(both)
      : "memory");
}

// The grouped GEMM on pairs of SMs (clusters of two CTAs).  A tile is 256 rows:
// CTA r of the pair holds rows 128r .. 128r+127 of A and rows
// r*n_len/2 .. (r+1)*n_len/2 - 1 of B in its shared memory, and the even CTA
// issues tcgen05.mma.cta_group::2 (M = 256), which reads both CTAs' operands
// and writes each CTA's 128 accumulator rows into that CTA's tensor memory.
// A K-block stage is 32 KB per CTA instead of 48, so shared memory moves a
// third fewer bytes per product and each B tile leaves L2 once per pair.
//
// Synchronisation.  Each CTA's copies complete on its own full barrier; in the
// odd CTA, warp 1 relays every completed stage to the even CTA's full barrier
// (which counts two arrivals: its own copies' and the relay's).  The pair's
// commits arrive on the empty and accumulator-full barriers of both CTAs.  The
// epilogue warps of both CTAs free an accumulator on the even CTA's barrier
// (eight arrivals).  Producers wait for the commits of their last stages, and
// a cluster barrier precedes the exit, so nothing arrives on a CTA that has
// left.  Every wait is bounded, as in the single-CTA kernel.
__global__ void __launch_bounds__(kGroupThreads, 1) umma_pair_kernel(const GroupArgs ga) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* sA = smem;
  unsigned char* sB = smem + kPairStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kPairStages * kPairBBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* accf = empty + kPairStages;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
  unsigned char* ystage = smem + kPairStages * (kABytes + kPairBBytes) + 1024;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su(tmem_slot)),
                 "r"(2 * kBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < kPairStages; ++i) {
      mbar_init(&full[i], rank == 0 ? 2 : 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 8);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  pair_sync();   // both CTAs' barriers and tensor memory are set up before either uses the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int t_begin = ga.begin[pair], t_end = ga.begin[pair + 1];
  bool dead = false;

  if (threadIdx.x == 0) {
    // ---- producer: this CTA's half of every stage
    uint32_t it = 0;
    for (int k = t_begin; k < t_end; ++k) {
      const TileInfo ti = tile_info(ga, ga.sched[k], 2 * kBM);
      const int half = ti.n_len >> 1;
      const uint32_t bbytes = (uint32_t)half * kBK * 2;
      const int Mg = ti.P->M >> 3, Ng = ti.P->N >> 3;
      const int ag = (ti.m0 + kBM * (int)rank) >> 3, bg = (ti.n0 + half * (int)rank) >> 3;
      for (int kb = 0; kb < ti.nk; ++kb, ++it) {
        const int st = it % kPairStages;
        if (it >= kPairStages && !dead && !mbar_wait(&empty[st], ((it / kPairStages) - 1) & 1)) dead = true;
        mbar_expect_tx(&full[st], kABytes + bbytes);
        bulk_g2s(sA + st * kABytes, ti.P->A + ((size_t)kb * Mg + ag) * 1024, kABytes, &full[st]);
        bulk_g2s(sB + st * kPairBBytes, ti.P->B + ((size_t)kb * Ng + bg) * 1024, bbytes, &full[st]);
      }
    }
    // the commits that free the last stages
    for (uint32_t i = it > kPairStages ? it - kPairStages : 0; i < it && !dead; ++i)
      if (!mbar_wait(&empty[i % kPairStages], (i / kPairStages) & 1)) dead = true;
  } else if (threadIdx.x == 32 && rank == 0) {
    // ---- MMA issuer (even CTA)
    uint32_t it = 0, nt = 0;
    for (int k = t_begin; k < t_end; ++k, ++nt) {
      const TileInfo ti = tile_info(ga, ga.sched[k], 2 * kBM);
      const int ab = nt & 1;
      if (nt >= 2 && !dead && !mbar_wait(&acce[ab], ((nt >> 1) - 1) & 1)) dead = true;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(ab * kBN);
      const uint32_t idesc = umma_idesc_f16(2 * kBM, ti.n_len);
      for (int kb = 0; kb < ti.nk; ++kb, ++it) {
        const int st = it % kPairStages;
        if (!dead && !mbar_wait(&full[st], (it / kPairStages) & 1)) dead = true;
        tc_fence_after();
        const uint32_t a0 = su(sA + st * kABytes), b0 = su(sB + st * kPairBBytes);
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks)
          umma_f16_pair(d, umma_desc(a0 + ks * 256, 128, 1024), umma_desc(b0 + ks * 256, 128, 1024), idesc,
                        (kb > 0 || ks > 0) ? 1u : 0u);
        umma_commit_pair(&empty[st]);
      }
      umma_commit_pair(&accf[ab]);
    }
  } else if (threadIdx.x == 32) {
    // ---- relay (odd CTA): each stage of this CTA, once landed, to the even CTA
    uint32_t it = 0;
    for (int k = t_begin; k < t_end; ++k) {
      const TileInfo ti = tile_info(ga, ga.sched[k], 2 * kBM);
      for (int kb = 0; kb < ti.nk; ++kb, ++it) {
        const int st = it % kPairStages;
        if (!dead && !mbar_wait(&full[st], (it / kPairStages) & 1)) dead = true;
        if (!dead) mbar_arrive_remote(cluster_addr(&full[st], 0));
      }
    }
  } else if (warp >= 2) {
    // ---- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 of this CTA
    const int quarter = warp & 3;
    const uint32_t acce_even0 = cluster_addr(&acce[0], 0), acce_even1 = cluster_addr(&acce[1], 0);
    uint32_t nt = 0;
    unsigned bad = 0;
    for (int k = t_begin; k < t_end; ++k, ++nt) {
      const TileInfo ti = tile_info(ga, ga.sched[k], 2 * kBM);
      const int ab = nt & 1;
      if (!dead && !mbar_wait(&accf[ab], (nt >> 1) & 1)) dead = true;
      dead = __any_sync(0xffffffffu, dead);
      tc_fence_after();
      epilogue_tile(ti, tmem + (uint32_t)(ab * kBN) + ((uint32_t)(32 * quarter) << 16), ti.m0 + kBM * (int)rank,
                    quarter, lane, ystage, bad);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(ab ? acce_even1 : acce_even0);
    }
    if (dead && lane == 0) atomicOr(ga.status, kStatusTimeout);
    if (__any_sync(0xffffffffu, bad != 0) && lane == 0) atomicOr(ga.status, kStatusRange);
  }
  if ((threadIdx.x == 0 || threadIdx.x == 32) && dead) atomicOr(ga.status, kStatusTimeout);
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  pair_sync();   // neither CTA leaves while the pair's products or arrivals may still reach it
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kBN) : "memory");
  }
}

size_t group_smem() { return (size_t)kStages * (kABytes + kBBytes) + 1024 + (size_t)4 * 32 * kYPitch; }
size_t pair_smem() { return (size_t)kPairStages * (kABytes + kPairBBytes) + 1024 + (size_t)4 * 32 * kYPitch; }

cudaLaunchConfig_t pair_config(int clusters, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kGroupThreads, 1, 1);
  cfg.dynamicSmemBytes = pair_smem();
  cfg.stream = st;
  attr->id = cudaLaunchAttributeClusterDimension;
  attr->val.clusterDim.x = 2;
  attr->val.clusterDim.y = 1;
  attr->val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// `clusters` pairs of CTAs over the tile lists of ga
cudaError_t launch_pair(const GroupArgs& ga, int clusters, cudaStream_t st) {
  cudaLaunchAttribute attr;
  const cudaLaunchConfig_t cfg = pair_config(clusters, st, &attr);
  return cudaLaunchKernelEx(&cfg, umma_pair_kernel, ga);
}

int grid_for(long long work, int per_block) {
  long long b = (work + per_block - 1) / per_block;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace

// Pairs of CTAs of the pair kernel that can be resident at once on the
// current device (its shared-memory attribute set on first use); 0 when the
// device runs none.  Returns a CUDA error code, 0 on success.
int prefill_pair_slots(int* slots) {
  static PerDevice cache;
  int v = 0;
  const int err = cache.get(current_device(), v, [](int& out) -> int {
    cudaError_t e = cudaFuncSetAttribute(umma_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)pair_smem());
    if (e != cudaSuccess) return (int)e;
    cudaLaunchAttribute attr;
    const cudaLaunchConfig_t cfg = pair_config(1, nullptr, &attr);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, umma_pair_kernel, &cfg);
    if (e != cudaSuccess) return (int)e;
    out = n > 0 ? n : -1;   // -1: cached "none"
    return 0;
  });
  if (err != 0) return err;
  *slots = v > 0 ? v : 0;
  return 0;
}

int prefill_sp(int s, int npaths) { return npaths == 2 ? s32(s) : ceil_div(s, 64) * 64; }

size_t prefill_layer_bytes(int M, int d_in, int d_out, int s, int npaths) {
  const size_t NK = (size_t)npaths * prefill_sp(s, npaths);
  auto a1k = [](size_t v) { return (v + 1023) & ~(size_t)1023; };
  return a1k((size_t)M * d_in * 2) + a1k(NK * d_in * 2) + a1k((size_t)d_out * NK * 2) + a1k((size_t)M * NK * 2);
}

constexpr int kMaxGemmGrid = 1024;

long long prefill_layer_tiles(int M, int d_out, int s, int npaths) {
  const int NK = npaths * prefill_sp(s, npaths);
  return (long long)(M / kBM) * (ceil_div(NK, kBN) + ceil_div(d_out, kBN));
}

// Offset of the PrepJob array inside a chunk's table (after the problems,
// the two CTA offset arrays and the tile lists), 16-byte aligned.
static size_t prep_jobs_off(int n_layers, long long tiles) {
  const size_t b = (size_t)2 * n_layers * sizeof(GemmProblem) + (size_t)2 * (kMaxGemmGrid + 1) * sizeof(int) +
                   (size_t)tiles * sizeof(int);
  return (b + 15) & ~(size_t)15;
}

size_t prefill_table_bytes(int n_layers, long long tiles) {
  const size_t b = prep_jobs_off(n_layers, tiles) + (size_t)n_layers * sizeof(PrepJob);
  return (b + 1023) & ~(size_t)1023;
}

static long long group_tiles(const LayerDesc* Ls, int n, int M) {
  long long t = 0;
  for (int i = 0; i < n; ++i) t += prefill_layer_tiles(M, Ls[i].d_out, Ls[i].s, Ls[i].npaths);
  return t;
}

// Buffers of one chunk of layers: each layer's X16 | B1 | B2 | T
// (prefill_layer_bytes), from `bufs` on.
struct LayerBufs {
  unsigned char *X16, *B1, *B2, *T;
};

static LayerBufs layer_bufs(unsigned char*& buf, const LayerDesc& L, int M) {
  const int P = L.npaths, NK = P * prefill_sp(L.s, P);
  auto a1k = [](size_t v) { return (v + 1023) & ~(size_t)1023; };
  LayerBufs b;
  b.X16 = buf;
  b.B1 = b.X16 + a1k((size_t)M * L.d_in * 2);
  b.B2 = b.B1 + a1k((size_t)NK * L.d_in * 2);
  b.T = b.B2 + a1k((size_t)L.d_out * NK * 2);
  buf = b.T + a1k((size_t)M * NK * 2);
  return b;
}

// Blocks of one layer's preparation steps (x, B1, B2), as for a launch of its own.
static void prep_blocks(const LayerDesc& L, int M, int Sp, int mode, std::array<int, kPrepKinds>& blocks) {
  const int P = L.npaths;
  blocks[3] = grid_for((long long)M * P * Sp / 8, 256);
  blocks[0] = grid_for((long long)M * L.d_in / 8 / kXUnroll, 256);
  // B1, B2: a warp per packed tile, then a thread per zero 16-byte piece
  const long long v_tiles = (long long)P * ((L.s + 15) >> 4) * (L.d_in / kVTileK);
  const long long v_zeros = (long long)P * (Sp - 16 * ((L.s + 15) >> 4)) * (L.d_in / 8);
  blocks[1] = grid_for(std::max(v_tiles * 32, v_zeros), 256);
  const long long u_tiles = (long long)P * (L.d_out / kUTileRows) * ((L.s + 31) >> 5);
  const long long u_zeros = (long long)P * L.d_out * ((Sp - 32 * ((L.s + 31) >> 5)) / 8);
  blocks[2] = grid_for(std::max(u_tiles * 32, u_zeros), 256);
  // forward: x, B1, B2; latent-only: x, B1; expand: B2 and T' from the cache
  if (mode == kModeLatent) blocks[2] = 0;
  if (mode == kModeExpand) blocks[0] = blocks[1] = 0;
  if (mode != kModeExpand) blocks[3] = 0;
}

// Operand preparation of a planned chunk: three grouped launches (x, B1, B2)
// over all its layers, arguments in the chunk's table at table_dev.
cudaError_t launch_prefill_prep(const PrefillPlan& plan, const unsigned char* table_dev, unsigned int* status,
                                cudaStream_t st) {
  const PrepJob* jobs = reinterpret_cast<const PrepJob*>(table_dev + plan.table_off + plan.jobs_off);
  // the kinds a call's mode needs (a kind with no blocks is not launched)
  if (plan.prep_grid[0]) prep_group_kernel<0><<<plan.prep_grid[0], 256, 0, st>>>(jobs, plan.n, status);
  if (plan.prep_grid[1]) prep_group_kernel<1><<<plan.prep_grid[1], 256, 0, st>>>(jobs, plan.n, status);
  if (plan.prep_grid[2]) prep_group_kernel<2><<<plan.prep_grid[2], 256, 0, st>>>(jobs, plan.n, status);
  if (plan.prep_grid[3]) prep_group_kernel<3><<<plan.prep_grid[3], 256, 0, st>>>(jobs, plan.n, status);
  return cudaGetLastError();
}

// Longest-first schedule of `cost` over `grid` CTAs: every tile goes to the
// CTA with the least work so far.  Tiles are taken in order of decreasing
// `key`, ties in list order; the key is the cost of the tile's row panel (its
// first tile), so the tiles of one panel stay together and run at about the
// same time.  Writes the CTA lists to sched (tile indices) and their offsets
// to begin[0..grid].
static void lpt_schedule(const std::vector<double>& cost, const std::vector<double>& key, int grid, int* sched,
                         int* begin) {
  const int T = (int)cost.size();
  std::vector<int> order(T);
  for (int i = 0; i < T; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return key[a] > key[b]; });
  using Slot = std::pair<double, int>;   // (load, cta)
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int b = 0; b < grid; ++b) heap.push({0.0, b});
  std::vector<std::vector<int>> lists(grid);
  for (int t : order) {
    Slot sl = heap.top();
    heap.pop();
    lists[sl.second].push_back(t);
    heap.push({sl.first + cost[t], sl.second});
  }
  int k = 0;
  for (int b = 0; b < grid; ++b) {
    begin[b] = k;
    for (int t : lists[b]) sched[k++] = t;
  }
  begin[grid] = k;
}

// Column tiles of an N-wide product: as few as UMMA's N <= 256 allows, of
// equal width rounded up to `gran` (16; 64 for GEMM2, whose epilogue stores
// 64 columns at a time).  Equal widths keep a row panel's tiles in one cost
// class of the schedule, so they run at about the same time and the panel
// leaves DRAM once; a narrow last tile would be scheduled much later and read
// it again.
static void split_n(int N, int gran, int& tiles, int& width) {
  tiles = ceil_div(N, kBN);
  width = ceil_div(ceil_div(N, tiles), gran) * gran;
  tiles = ceil_div(N, width);
}

// Tile cost for the schedule: K-blocks times the tile's share of a full-width
// product, plus about one K-block of fixed per-tile work.
static double tile_cost(int K, int n_len) { return (double)(K / kBK) * (double)max(n_len, 64) / kBN + 1.0; }

// Host image of a chunk's table, appended to `img` at a 1 KB boundary:
// 2n problems | begin1 | begin2 | sched1 | sched2.  Device pointers in it refer
// to the chunk's buffers at `bufs` and to the image's own place at
// table_dev + plan.table_off.
void plan_prefill_chunk(const LayerDesc* Ls, const void* const* xs, void* const* ys, int n, int M, int x_bf16,
                        int mode, unsigned char* bufs, int num_sms, int pair_slots, std::vector<unsigned char>& img,
                        PrefillPlan& plan) {
  const long long tiles_all = group_tiles(Ls, n, M);
  plan.n = n;
  // 256-row tiles on pairs of SMs when M allows them and pairs can be resident
  plan.pair = (M % (2 * kBM) == 0 && pair_slots > 0) ? 1 : 0;
  const int rows = plan.pair ? 2 * kBM : kBM;
  plan.table_off = (img.size() + 1023) & ~(size_t)1023;
  plan.table_bytes = prefill_table_bytes(n, tiles_all);
  plan.jobs_off = prep_jobs_off(n, tiles_all);
  img.resize(plan.table_off + plan.table_bytes, 0);
  unsigned char* base = img.data() + plan.table_off;
  PrepJob* jobs = reinterpret_cast<PrepJob*>(base + plan.jobs_off);
  for (int k = 0; k < kPrepKinds; ++k) plan.prep_grid[k] = 0;
  const size_t prob_b = (size_t)2 * n * sizeof(GemmProblem);
  GemmProblem* probs = reinterpret_cast<GemmProblem*>(base);
  int* begin1 = reinterpret_cast<int*>(base + prob_b);
  int* begin2 = begin1 + kMaxGemmGrid + 1;
  int* sched1 = begin2 + kMaxGemmGrid + 1;
  std::vector<double> cost1, cost2, key1, key2;
  int tiles1 = 0, tiles2 = 0;
  unsigned char* buf = bufs;
  std::vector<std::array<int, kPrepKinds>> blocks(n);
  // layers of the chunk that read the same x (same pointer and width; a
  // block's q, k and v projections, gate and up) share one converted X16
  std::map<std::pair<const void*, int>, unsigned char*> x16_of;
  for (int i = 0; i < n; ++i) {
    const LayerDesc& L = Ls[i];
    const int P = L.npaths, Sp = prefill_sp(L.s, P), NK = P * Sp;
    LayerBufs b = layer_bufs(buf, L, M);
    PrepJob& J = jobs[i];
    std::memset(&J, 0, sizeof(J));
    J.L = L;
    J.x = static_cast<const uint16_t*>(xs[i]);
    prep_blocks(L, M, Sp, mode, blocks[i]);
    if (mode != kModeExpand) {
      const auto key = std::make_pair(xs[i], L.d_in);
      const auto it = x16_of.find(key);
      if (it == x16_of.end()) {
        x16_of.emplace(key, b.X16);
      } else {
        b.X16 = it->second;   // converted by the first layer that reads this x
        blocks[i][0] = 0;
      }
    }
    J.X16 = b.X16; J.B1 = b.B1; J.B2 = b.B2; J.T = b.T;
    J.M = M; J.x_bf16 = x_bf16; J.Sp = Sp;
    GemmProblem& g1 = probs[i];
    g1 = GemmProblem{};
    g1.A = b.X16; g1.B = b.B1; g1.M = M; g1.N = NK; g1.K = L.d_in; g1.mode = mode == kModeLatent ? 2 : 0;
    g1.l0 = L.p[0].l; g1.l1 = P == 2 ? L.p[1].l : L.p[0].l; g1.s = L.s; g1.Sp = Sp; g1.T = b.T;
    g1.Y = mode == kModeLatent ? ys[i] : nullptr; g1.t_ld = L.t_ld;
    split_n(NK, 16, g1.tiles_n, g1.tile_w);
    g1.tile_begin = tiles1;
    if (mode != kModeExpand) {
      tiles1 += (M / rows) * g1.tiles_n;
      for (int mt = 0; mt < M / rows; ++mt)
        for (int nt = 0; nt < g1.tiles_n; ++nt) {
          cost1.push_back(tile_cost(g1.K, min(g1.tile_w, NK - nt * g1.tile_w)));
          key1.push_back(tile_cost(g1.K, g1.tile_w));
        }
    }
    GemmProblem& g2 = probs[n + i];
    g2 = GemmProblem{};
    g2.A = b.T; g2.B = b.B2; g2.M = M; g2.N = L.d_out; g2.K = NK; g2.mode = 1; g2.Y = ys[i]; g2.y_bf16 = x_bf16;
    split_n(L.d_out, 64, g2.tiles_n, g2.tile_w);
    g2.tile_begin = tiles2;
    if (mode != kModeLatent) {
      tiles2 += (M / rows) * g2.tiles_n;
      for (int mt = 0; mt < M / rows; ++mt)
        for (int nt = 0; nt < g2.tiles_n; ++nt) {
          cost2.push_back(tile_cost(g2.K, min(g2.tile_w, L.d_out - nt * g2.tile_w)));
          key2.push_back(tile_cost(g2.K, g2.tile_w));
        }
    }
  }
  // The preparation of the next chunk runs beside this chunk's GEMM (one CTA
  // per SM, 192 threads x 128 registers).  Each preparation launch is
  // therefore held to kPrepBlocksPerSm blocks per SM in total, so that a GEMM
  // CTA still fits on an SM next to them; a layer's share stays proportional
  // to its work.
  for (int k = 0; k < kPrepKinds; ++k) {
    long long total = 0;
    for (int i = 0; i < n; ++i) total += blocks[i][k];
    const long long cap = (long long)kPrepBlocksPerSm * num_sms;
    for (int i = 0; i < n; ++i) {
      int b = blocks[i][k];
      if (total > cap && b > 0) b = (int)std::max<long long>(1, (long long)b * cap / total);
      jobs[i].first[k] = plan.prep_grid[k];
      plan.prep_grid[k] += b;
    }
  }
  int* sched2 = sched1 + tiles1;
  plan.tiles1 = tiles1;
  plan.tiles2 = tiles2;
  // CTAs (or, for pairs, clusters) of the persistent launches
  const int slots = plan.pair ? min(pair_slots, kMaxGemmGrid / 2) : min(num_sms, kMaxGemmGrid);
  plan.grid1 = min(tiles1, slots);
  plan.grid2 = min(tiles2, slots);
  if (plan.grid1 > 0) lpt_schedule(cost1, key1, plan.grid1, sched1, begin1);
  if (plan.grid2 > 0) lpt_schedule(cost2, key2, plan.grid2, sched2, begin2);
}

// GEMM1 and GEMM2 of a planned chunk (table uploaded at table_dev +
// plan.table_off, operands prepared by launch_prefill_prep): one grouped
// launch each.
cudaError_t launch_prefill_gemms(const PrefillPlan& plan, const unsigned char* table_dev, unsigned int* status,
                                 cudaStream_t st) {
  // the shared-memory attribute, once per device
  static PerDevice cache;
  int done = 0;
  const int err = cache.get(current_device(), done, [](int& v) -> int {
    v = 1;
    return (int)cudaFuncSetAttribute(umma_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)group_smem());
  });
  if (err != 0) return (cudaError_t)err;
  if (plan.pair) {
    const int perr = prefill_pair_slots(&done);
    if (perr != 0) return (cudaError_t)perr;
  }
  const unsigned char* base = table_dev + plan.table_off;
  const size_t prob_b = (size_t)2 * plan.n * sizeof(GemmProblem);
  const GemmProblem* probs = reinterpret_cast<const GemmProblem*>(base);
  const int* begin_dev = reinterpret_cast<const int*>(base + prob_b);
  const int* sched_dev = begin_dev + 2 * (kMaxGemmGrid + 1);
  // GEMM1 (not in expand calls) and GEMM2 (not in latent-only calls)
  GroupArgs g1a{probs, sched_dev, begin_dev, plan.n, plan.tiles1, status};
  GroupArgs g2a{probs + plan.n, sched_dev + plan.tiles1, begin_dev + kMaxGemmGrid + 1, plan.n, plan.tiles2, status};
  if (!plan.pair) {
    if (plan.grid1 > 0) umma_group_kernel<<<plan.grid1, kGroupThreads, group_smem(), st>>>(g1a);
    if (plan.grid2 > 0) umma_group_kernel<<<plan.grid2, kGroupThreads, group_smem(), st>>>(g2a);
    return cudaGetLastError();
  }
  cudaError_t e = cudaSuccess;
  if (plan.grid1 > 0) e = launch_pair(g1a, plan.grid1, st);
  if (e == cudaSuccess && plan.grid2 > 0) e = launch_pair(g2a, plan.grid2, st);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace lb
