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

#include "lb_internal.h"

namespace lb {
namespace {

constexpr int kBM = 128;          // rows per tile (UMMA M)
constexpr int kBN = 256;          // max columns per tile (UMMA N)
constexpr int kBK = 64;           // K per stage
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kGemmThreads = 128;

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

// x (M x K, fp16 or bf16, row-major, leading dimension K) -> fp16 core-matrix tiles
__global__ void __launch_bounds__(256) prep_x_kernel(const uint16_t* __restrict__ x, int is_bf16, int M, int K,
                                                     unsigned char* __restrict__ out) {
  const long long n16 = (long long)M * K / 8;   // 16-byte chunks
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n16;
       t += (long long)gridDim.x * blockDim.x) {
    // chunk t covers row r, columns 8c .. 8c+7 in row-major order
    const int r = (int)(t / (K / 8));
    const int k = (int)(t % (K / 8)) * 8;
    uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)r * K + k);
    if (is_bf16) {
      uint32_t* w = &v.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
        const __half2 h = __floats2half2_rn(__bfloat162float(b.x), __bfloat162float(b.y));
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
    }
    *reinterpret_cast<uint4*>(out + tiled_off(r, k, M)) = v;
  }
}

// B1 (P*Sp rows x d_in): row j' = p*Sp + j holds V_p[i][j] * g_p[i] (0 for j >= s)
__global__ void __launch_bounds__(256) prep_b1_kernel(const LayerDesc L, int Sp, unsigned char* __restrict__ out) {
  const int R = L.npaths * Sp, K = L.d_in;
  const int n_kt = K / kVTileK;
  const long long n16 = (long long)R * K / 8;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n16;
       t += (long long)gridDim.x * blockDim.x) {
    const int jr = (int)(t / (K / 8));
    const int i0 = (int)(t % (K / 8)) * 8;
    const int p = jr / Sp, j = jr - p * Sp;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (j < L.s) {
      const unsigned char* V = reinterpret_cast<const unsigned char*>(L.p[p].V);
      const uint16_t* g = L.p[p].g;
      const int rb = j >> 4, jj = j & 15, gg = jj & 7, rlo = jj >> 3;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = i0 + e;
        const int kk = i & 255, q = kk >> 5, rem = kk & 31;
        const int rhi = rem >> 4, c = (rem & 15) >> 2, m = rem & 3;
        const int lane = 4 * gg + c, r = 2 * rhi + rlo;
        const unsigned char byte = V[((size_t)rb * n_kt + (i >> 8)) * kTileBytes + 16 * lane + 4 * r + m];
        const uint32_t bit = (byte >> q) & 1u;
        const uint32_t val = (uint32_t)g[i] ^ (bit << 15);
        w[e >> 1] |= val << (16 * (e & 1));
      }
    }
    *reinterpret_cast<uint4*>(out + tiled_off(jr, i0, R)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// B2 (d_out rows x P*Sp): column j' = p*Sp + j of row o holds U_p[o][j] * h_p[o]
__global__ void __launch_bounds__(256) prep_b2_kernel(const LayerDesc L, int Sp, unsigned char* __restrict__ out) {
  const int R = L.d_out, K = L.npaths * Sp;
  const int n_kt = (L.s + 31) >> 5;
  const long long n16 = (long long)R * K / 8;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n16;
       t += (long long)gridDim.x * blockDim.x) {
    const int o = (int)(t / (K / 8));
    const int j0 = (int)(t % (K / 8)) * 8;
    const int ob = o >> 7, oo = o & 127, q = oo >> 4, rr = oo & 15, gg = rr & 7, rlo = rr >> 3;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int jr = j0 + e, p = jr / Sp, j = jr - p * Sp;
      if (j < L.s) {
        const unsigned char* U = reinterpret_cast<const unsigned char*>(L.p[p].U);
        const int kk = j & 31, rhi = kk >> 4, c = (kk & 15) >> 2, m = kk & 3;
        const int lane = 4 * gg + c, r = 2 * rhi + rlo;
        const unsigned char byte = U[((size_t)ob * n_kt + (j >> 5)) * kTileBytes + 16 * lane + 4 * r + m];
        const uint32_t bit = (byte >> q) & 1u;
        const uint32_t val = (uint32_t)L.p[p].h[o] ^ (bit << 15);
        w[e >> 1] |= val << (16 * (e & 1));
      }
    }
    *reinterpret_cast<uint4*>(out + tiled_off(o, j0, R)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------------------ tcgen05 GEMM

struct GemmArgs {
  const unsigned char* A;   // core-matrix tiles, M rows x K
  const unsigned char* B;   // core-matrix tiles, N rows x K
  int M, N, K;
  int mode;                 // 0: T' = l * acc -> fp16 tiles; 1: y = acc -> row-major
  // mode 0
  const uint16_t* l0;
  const uint16_t* l1;
  int s, Sp;
  unsigned char* T;         // core-matrix tiles, M rows x N (N = P*Sp)
  // mode 1
  void* Y;                  // row-major M x N
  int y_bf16;
  unsigned int* status;
};

__global__ void __launch_bounds__(kGemmThreads, 1) umma_gemm_kernel(const GemmArgs g) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* sA = smem;                                   // [stages][16 KB]
  unsigned char* sB = smem + kStages * kABytes;               // [stages][32 KB]
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN;
  const int n_len = min(kBN, g.N - n0);   // multiple of 16
  const int nk = g.K / kBK;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su(tmem_slot)),
                 "r"(kBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (threadIdx.x == 0) {
    // ---- producer: one bulk copy per operand per stage
    const uint32_t bbytes = (uint32_t)n_len * kBK * 2;
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int st = kb % kStages;
      if (kb >= kStages) ok = mbar_wait(&empty[st], ((kb / kStages) - 1) & 1);
      if (!ok) break;
      mbar_expect_tx(&full[st], kABytes + bbytes);
      bulk_g2s(sA + st * kABytes, g.A + ((size_t)kb * (g.M >> 3) + (m0 >> 3)) * 1024, kABytes, &full[st]);
      bulk_g2s(sB + st * kBBytes, g.B + ((size_t)kb * (g.N >> 3) + (n0 >> 3)) * 1024, bbytes, &full[st]);
    }
  } else if (threadIdx.x == 32) {
    // ---- MMA issuer: 4 x (M=128, N=n_len, K=16) per stage
    const uint32_t idesc = umma_idesc_f16(kBM, n_len);
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int st = kb % kStages;
      ok = mbar_wait(&full[st], (kb / kStages) & 1);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a0 = su(sA + st * kABytes), b0 = su(sB + st * kBBytes);
#pragma unroll
      for (int ks = 0; ks < kBK / 16; ++ks) {
        const uint64_t ad = umma_desc(a0 + ks * 256, 128, 1024);
        const uint64_t bd = umma_desc(b0 + ks * 256, 128, 1024);
        umma_f16(tmem, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(&empty[st]);   // stage free once these products are done
    }
    umma_commit(done);
  }
  __syncwarp();

  // ---- epilogue: warp w owns TMEM lanes 32w..32w+31 = tile rows
  if (!mbar_wait(done, 0)) ok = false;
  ok = __all_sync(0xffffffffu, ok);   // tcgen05.ld below needs the whole warp
  if (!ok) {
    if (lane == 0) atomicOr(g.status, 1u << LB_ERR_TIMEOUT);
  } else {
    tc_fence_after();
    const int row = m0 + warp * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < n_len; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + (uint32_t)c0, v);
      if (g.mode == 0) {
        // T'[row][n] = l(n) * acc, n = n0 + c0 + e; two fp16 x 8 chunks
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float lv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int n = n0 + c0 + e + u;
            const int p = n / g.Sp, j = n - p * g.Sp;
            const uint16_t* l = p == 0 ? g.l0 : g.l1;
            lv[u] = j < g.s ? __half2float(__ushort_as_half(l[j])) : 0.f;
          }
          const __half2 h = __floats2half2_rn(lv[0] * v[e], lv[1] * v[e + 1]);
          w[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(g.T + tiled_off(row, n0 + c0, g.M)) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(g.T + tiled_off(row, n0 + c0 + 8, g.M)) = make_uint4(w[4], w[5], w[6], w[7]);
      } else {
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          if (g.y_bf16) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(v[e], v[e + 1]);
            w[e >> 1] = *reinterpret_cast<const uint32_t*>(&b);
          } else {
            const __half2 h = __floats2half2_rn(v[e], v[e + 1]);
            w[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
          }
        }
        uint16_t* yr = static_cast<uint16_t*>(g.Y) + (size_t)row * g.N + n0 + c0;
        *reinterpret_cast<uint4*>(yr) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(yr + 8) = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kBN) : "memory");
  }
}

size_t gemm_smem() { return (size_t)kStages * (kABytes + kBBytes) + (2 * kStages + 1) * 8 + 16; }

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(umma_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem());
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid(g.M / kBM, (g.N + kBN - 1) / kBN);
  umma_gemm_kernel<<<grid, kGemmThreads, gemm_smem(), st>>>(g);
  return cudaGetLastError();
}

int grid_for(long long work, int per_block) {
  long long b = (work + per_block - 1) / per_block;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace

// One layer, M rows: prepare the three operands, then GEMM1 and GEMM2.
// ws must hold prefill_workspace_bytes(...) bytes, 1 KB aligned.
size_t prefill_workspace_bytes(int M, int d_in, int d_out, int s, int npaths) {
  const int Sp = npaths == 2 ? s32(s) : ceil_div(s, 64) * 64;
  const size_t NK = (size_t)npaths * Sp;
  const size_t x16 = (size_t)M * d_in * 2, b1 = NK * d_in * 2, b2 = (size_t)d_out * NK * 2, t = (size_t)M * NK * 2;
  return ((x16 + 1023) & ~1023ull) + ((b1 + 1023) & ~1023ull) + ((b2 + 1023) & ~1023ull) + ((t + 1023) & ~1023ull);
}

cudaError_t launch_prefill(const LayerDesc& L, int M, const void* x, int x_bf16, void* y, unsigned char* ws,
                           unsigned int* status, cudaStream_t st) {
  const int P = L.npaths;
  const int Sp = P == 2 ? s32(L.s) : ceil_div(L.s, 64) * 64;
  const int NK = P * Sp;
  unsigned char* X16 = ws;
  unsigned char* B1 = X16 + (((size_t)M * L.d_in * 2 + 1023) & ~1023ull);
  unsigned char* B2 = B1 + (((size_t)NK * L.d_in * 2 + 1023) & ~1023ull);
  unsigned char* T = B2 + (((size_t)L.d_out * NK * 2 + 1023) & ~1023ull);

  prep_x_kernel<<<grid_for((long long)M * L.d_in / 8, 256), 256, 0, st>>>(static_cast<const uint16_t*>(x), x_bf16, M,
                                                                          L.d_in, X16);
  prep_b1_kernel<<<grid_for((long long)NK * L.d_in / 8, 256), 256, 0, st>>>(L, Sp, B1);
  prep_b2_kernel<<<grid_for((long long)L.d_out * NK / 8, 256), 256, 0, st>>>(L, Sp, B2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  GemmArgs g1 = {};
  g1.A = X16;
  g1.B = B1;
  g1.M = M;
  g1.N = NK;
  g1.K = L.d_in;
  g1.mode = 0;
  g1.l0 = L.p[0].l;
  g1.l1 = P == 2 ? L.p[1].l : L.p[0].l;
  g1.s = L.s;
  g1.Sp = Sp;
  g1.T = T;
  g1.status = status;
  e = launch_gemm(g1, st);
  if (e != cudaSuccess) return e;

  GemmArgs g2 = {};
  g2.A = T;
  g2.B = B2;
  g2.M = M;
  g2.N = L.d_out;
  g2.K = NK;
  g2.mode = 1;
  g2.Y = y;
  g2.y_bf16 = x_bf16;
  g2.status = status;
  return launch_gemm(g2, st);
}

}  // namespace lb
