// Initialisation of LittleBit factors on the GPU: Dual-SVID and Joint-ITQ.
//
// Dual-SVID (Samsung LittleBit article, section 2, the Dual-SVID bullet):
// from the real factors of a truncated SVD, U' (d_out x s) and V' (d_in x s),
// the binary factors are their signs and the scales come from rank-1 fits of
// their magnitudes: |U'| ~ a_U b_U^T, |V'| ~ a_V b_V^T, giving
//   h = a_U / mean(a_U),  g = a_V / mean(a_V),
//   l = (mean(a_U) b_U) (.) (mean(a_V) b_V)
// so that h_o l_j g_i = a_U[o] b_U[j] a_V[i] b_V[j] (the split between the
// row or column scale and l is a gauge; h and g are normalised to mean 1).
// The best rank-1 fit of a non-negative matrix is its top singular pair; it
// is found here by power iteration from the all-ones vector (which keeps both
// vectors non-negative), with deterministic fixed-order reductions.
//
// Joint-ITQ (LittleBit-2 column, chapter 2, "solution 1"): the stacked
// factors X = [U'; V'] ((d_out + d_in) x s) are rotated by an orthogonal R
// found by alternating B = sign(X R) and R = argmax tr(B^T X R), the polar
// factor of M = X^T B; then U' <- U' R and V' <- V' R, which leaves U' V'^T
// unchanged.  The products run as fp32 tiled GEMMs on the CUDA cores; the
// polar factor is taken by Newton-Schulz steps Y <- Y (3 I - Y^T Y) / 2 from
// Y = M / ||M||_F, which converge to it for any M of full rank.
#include <cuda_fp16.h>

#include <cmath>
#include <vector>

#include "lb_internal.h"

namespace lb {
namespace {

constexpr int kRedThreads = 256;

// ---------------------------------------------------------------- reductions

// Sum of a block's values (every thread gets it); fixed order, so deterministic.
__device__ __forceinline__ float block_sum(float v, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh[w];
  return t;
}

// partial[blk][j] = sum over the block's rows i of |A[i][j]| a[i]  (A: n x s row-major)
__global__ void __launch_bounds__(kRedThreads) abs_colsum_kernel(const float* __restrict__ A, const float* __restrict__ a,
                                                                 int n, int s, int rows_per_blk, float* __restrict__ partial) {
  const int i0 = blockIdx.x * rows_per_blk, i1 = min(n, i0 + rows_per_blk);
  for (int j = threadIdx.x; j < s; j += blockDim.x) {
    float acc = 0.f;
    for (int i = i0; i < i1; ++i) acc += fabsf(A[(size_t)i * s + j]) * a[i];
    partial[(size_t)blockIdx.x * s + j] = acc;
  }
}

// b[j] = sum_blk partial[blk][j], in block order
__global__ void reduce_rows_kernel(const float* __restrict__ partial, int nblk, int s, float* __restrict__ b) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= s) return;
  float acc = 0.f;
  for (int k = 0; k < nblk; ++k) acc += partial[(size_t)k * s + j];
  b[j] = acc;
}

// a[i] = sum_j |A[i][j]| b[j]: one warp per row
__global__ void abs_rowdot_kernel(const float* __restrict__ A, const float* __restrict__ b, int n, int s,
                                  float* __restrict__ a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= n) return;
  const float* row = A + (size_t)warp * s;
  float acc = 0.f;
  for (int j = lane; j < s; j += 32) acc += fabsf(row[j]) * b[j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) a[warp] = acc;
}

// v /= ||v||; *norm_out = ||v|| (one block)
__global__ void __launch_bounds__(1024) normalize_kernel(float* __restrict__ v, int n, float* __restrict__ norm_out) {
  __shared__ float sh[32];
  float acc = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) acc += v[i] * v[i];
  const float nrm = sqrtf(block_sum(acc, sh));
  const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) v[i] *= inv;
  if (threadIdx.x == 0) *norm_out = nrm;
}

__global__ void fill_kernel(float* __restrict__ v, int n, float value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] = value;
}

// From the unit rank-1 vectors (a, b) and sigma of |U'| and |V'|:
// h = a_U / mean(a_U), g = a_V / mean(a_V), l = (sig_U mean(a_U) b_U) (.) (sig_V mean(a_V) b_V), in fp16.
__global__ void __launch_bounds__(1024) dual_svid_scales_kernel(const float* __restrict__ au, const float* __restrict__ bu,
                                                                const float* __restrict__ sig_u, int d_out,
                                                                const float* __restrict__ av, const float* __restrict__ bv,
                                                                const float* __restrict__ sig_v, int d_in, int s,
                                                                uint16_t* __restrict__ h, uint16_t* __restrict__ g,
                                                                uint16_t* __restrict__ l) {
  __shared__ float sh[32];
  float su = 0.f, sv = 0.f;
  for (int i = threadIdx.x; i < d_out; i += blockDim.x) su += au[i];
  const float mu = block_sum(su, sh) / (float)d_out;
  for (int i = threadIdx.x; i < d_in; i += blockDim.x) sv += av[i];
  const float mv = block_sum(sv, sh) / (float)d_in;
  const float iu = mu > 0.f ? 1.f / mu : 0.f, iv = mv > 0.f ? 1.f / mv : 0.f;
  for (int i = threadIdx.x; i < d_out; i += blockDim.x) h[i] = __half_as_ushort(__float2half_rn(au[i] * iu));
  for (int i = threadIdx.x; i < d_in; i += blockDim.x) g[i] = __half_as_ushort(__float2half_rn(av[i] * iv));
  const float cu = *sig_u * mu, cv = *sig_v * mv;
  for (int j = threadIdx.x; j < s; j += blockDim.x)
    l[j] = __half_as_ushort(__float2half_rn((cu * bu[j]) * (cv * bv[j])));
}

// ---------------------------------------------------------------- fp32 GEMM
//
// C = alpha * op(A) * B + beta * Cin  (row-major; op(A) = A, M x K, or A^T
// with A stored K x M), or C = sign(op(A) * B) as +-1 (sign(0) = +1).  Tile
// 64 x 64 x 16, 256 threads, 4 x 4 outputs per thread; bounds-checked loads
// (zero fill) and stores.  With gridDim.z > 1 each z takes a K range and
// writes its own M x N partial at C + z * M * N (alpha 1, no Cin).
constexpr int kGT = 64, kGK = 16;
enum GemmEpi { kEpiLinear = 0, kEpiSign = 1 };

template <bool TA, int EPI>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, const float* __restrict__ B,
                                                       float* __restrict__ C, const float* __restrict__ Cin, int M,
                                                       int N, int K, float alpha, float beta) {
  __shared__ float As[kGK][kGT + 4];
  __shared__ float Bs[kGK][kGT + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * kGT, n0 = blockIdx.x * kGT;
  const int ksplit = (K + gridDim.z - 1) / gridDim.z;
  const int kb = blockIdx.z * ksplit, ke = min(K, kb + ksplit);
  float acc[4][4] = {};
  for (int k0 = kb; k0 < ke; k0 += kGK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = threadIdx.x + 256 * r;   // 0..1023
      if (TA) {
        const int kk = e >> 6, mm = e & 63;   // A stored K x M
        const int gk = k0 + kk, gm = m0 + mm;
        As[kk][mm] = (gk < ke && gm < M) ? A[(size_t)gk * M + gm] : 0.f;
      } else {
        const int mm = e >> 4, kk = e & 15;   // A stored M x K
        const int gk = k0 + kk, gm = m0 + mm;
        As[kk][mm] = (gk < ke && gm < M) ? A[(size_t)gm * K + gk] : 0.f;
      }
      const int kk = e >> 6, nn = e & 63;
      const int gk = k0 + kk, gn = n0 + nn;
      Bs[kk][nn] = (gk < ke && gn < N) ? B[(size_t)gk * N + gn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* Cz = C + (size_t)blockIdx.z * M * N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      const size_t o = (size_t)gm * N + gn;
      if (EPI == kEpiSign) Cz[o] = acc[i][j] < 0.f ? -1.f : 1.f;
      else if (gridDim.z > 1) Cz[o] = acc[i][j];
      else Cz[o] = alpha * acc[i][j] + (beta != 0.f ? beta * Cin[o] : 0.f);
    }
  }
}

// out[e] = sum_z partial[z][e] in z order (deterministic split-K reduction)
__global__ void reduce_splits_kernel(const float* __restrict__ partial, int splits, size_t n, float* __restrict__ out) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  float acc = 0.f;
  for (int z = 0; z < splits; ++z) acc += partial[(size_t)z * n + e];
  out[e] = acc;
}

// v *= 1 / ||v||_F (one block; v has n elements)
__global__ void __launch_bounds__(1024) frob_normalize_kernel(float* __restrict__ v, size_t n) {
  __shared__ float sh[32];
  float acc = 0.f;
  for (size_t i = threadIdx.x; i < n; i += blockDim.x) acc += v[i] * v[i];
  const float nrm = sqrtf(block_sum(acc, sh));
  const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
  for (size_t i = threadIdx.x; i < n; i += blockDim.x) v[i] *= inv;
}

__global__ void identity_kernel(float* __restrict__ R, int s) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < s * s) R[e] = (e / s == e % s) ? 1.f : 0.f;
}

__global__ void copy_kernel(const float* __restrict__ src, float* __restrict__ dst, size_t n) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < n) dst[e] = src[e];
}

inline unsigned blocks_for(size_t n, int per) { return (unsigned)((n + per - 1) / per); }

template <bool TA, int EPI>
cudaError_t gemm(const float* A, const float* B, float* C, const float* Cin, int M, int N, int K, float alpha,
                 float beta, int splits, cudaStream_t st) {
  dim3 grid(blocks_for(N, kGT), blocks_for(M, kGT), splits);
  gemm_f32_kernel<TA, EPI><<<grid, 256, 0, st>>>(A, B, C, Cin, M, N, K, alpha, beta);
  return cudaGetLastError();
}

}  // namespace

// ---------------------------------------------------------------- Dual-SVID

// The rank-1 fit |A| ~ sigma a b^T (a, b unit, non-negative) by `iters` power
// steps from a = 1/sqrt(n); scratch: partial (>= nblk * s floats).
static cudaError_t rank1_power(const float* A, int n, int s, int iters, float* a, float* b, float* sig_b,
                               float* sig_a, float* partial, cudaStream_t st) {
  const int rows_per_blk = 64;
  const int nblk = (n + rows_per_blk - 1) / rows_per_blk;
  fill_kernel<<<blocks_for(n, 256), 256, 0, st>>>(a, n, 1.f / sqrtf((float)n));
  for (int it = 0; it < iters; ++it) {
    abs_colsum_kernel<<<nblk, kRedThreads, 0, st>>>(A, a, n, s, rows_per_blk, partial);
    reduce_rows_kernel<<<blocks_for(s, 256), 256, 0, st>>>(partial, nblk, s, b);
    normalize_kernel<<<1, 1024, 0, st>>>(b, s, sig_b);
    abs_rowdot_kernel<<<blocks_for((size_t)n * 32, 256), 256, 0, st>>>(A, b, n, s, a);
    normalize_kernel<<<1, 1024, 0, st>>>(a, n, sig_a);
  }
  return cudaGetLastError();
}

size_t dual_svid_scratch_floats(int d_out, int d_in, int s) {
  const int n = d_out > d_in ? d_out : d_in;
  return (size_t)((n + 63) / 64) * s + (size_t)d_out + d_in + 2 * (size_t)s + 8;
}

cudaError_t launch_dual_svid(const float* Uf, const float* Vf, int d_out, int d_in, int s, int iters, void* U_bits,
                             void* V_bits, uint16_t* h, uint16_t* g, uint16_t* l, float* scratch, cudaStream_t st) {
  const int n = d_out > d_in ? d_out : d_in;
  float* partial = scratch;
  float* au = partial + (size_t)((n + 63) / 64) * s;
  float* av = au + d_out;
  float* bu = av + d_in;
  float* bv = bu + s;
  float* sc = bv + s;   // [sig_b_U, sig_U, sig_b_V, sig_V]
  cudaError_t e = launch_pack(Uf, LB_F32, d_out, s, s, 1, LB_ROLE_U, U_bits, st);
  if (e == cudaSuccess) e = launch_pack(Vf, LB_F32, d_in, s, s, 1, LB_ROLE_V, V_bits, st);
  if (e == cudaSuccess) e = rank1_power(Uf, d_out, s, iters, au, bu, sc + 0, sc + 1, partial, st);
  if (e == cudaSuccess) e = rank1_power(Vf, d_in, s, iters, av, bv, sc + 2, sc + 3, partial, st);
  if (e != cudaSuccess) return e;
  // |A| ~ sigma_a a b^T with a, b unit: the product of the pair is sig_a
  dual_svid_scales_kernel<<<1, 1024, 0, st>>>(au, bu, sc + 1, d_out, av, bv, sc + 3, d_in, s, h, g, l);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- Joint-ITQ

size_t itq_scratch_floats(int n_rows, int s) {
  const int splits = 16;
  return 2 * (size_t)n_rows * s + (size_t)splits * s * s + 4 * (size_t)s * s;
}

cudaError_t launch_joint_itq(float* X, int n_rows, int s, int iters, int ns_steps, float* R, int r_given,
                             float* scratch, cudaStream_t st) {
  const int splits = 16;
  const size_t ss = (size_t)s * s;
  float* Z = scratch;                      // n_rows x s: X R, then its signs
  float* Xr = Z + (size_t)n_rows * s;      // n_rows x s: the rotated factors
  float* part = Xr + (size_t)n_rows * s;   // splits x s x s
  float* Mx = part + (size_t)splits * ss;  // s x s: X^T B, then the Newton-Schulz iterate
  float* G = Mx + ss;                      // s x s: Y^T Y
  float* Y2 = G + ss;                      // s x s
  cudaError_t e = cudaSuccess;
  if (!r_given) identity_kernel<<<blocks_for(ss, 256), 256, 0, st>>>(R, s);
  for (int it = 0; it < iters && e == cudaSuccess; ++it) {
    // B = sign(X R)
    e = gemm<false, kEpiSign>(X, R, Z, nullptr, n_rows, s, s, 1.f, 0.f, 1, st);
    // M = X^T B, split over the long dimension and reduced in a fixed order
    if (e == cudaSuccess) e = gemm<true, kEpiLinear>(X, Z, part, nullptr, s, s, n_rows, 1.f, 0.f, splits, st);
    if (e != cudaSuccess) break;
    reduce_splits_kernel<<<blocks_for(ss, 256), 256, 0, st>>>(part, splits, ss, Mx);
    frob_normalize_kernel<<<1, 1024, 0, st>>>(Mx, ss);
    // polar factor of M: Y <- 1.5 Y - 0.5 Y (Y^T Y)
    float* Yc = Mx;
    float* Yn = Y2;
    for (int k = 0; k < ns_steps && e == cudaSuccess; ++k) {
      e = gemm<true, kEpiLinear>(Yc, Yc, G, nullptr, s, s, s, 1.f, 0.f, 1, st);
      if (e == cudaSuccess) e = gemm<false, kEpiLinear>(Yc, G, Yn, Yc, s, s, s, -0.5f, 1.5f, 1, st);
      float* t = Yc;
      Yc = Yn;
      Yn = t;
    }
    if (e == cudaSuccess) {
      copy_kernel<<<blocks_for(ss, 256), 256, 0, st>>>(Yc, R, ss);
      e = cudaGetLastError();
    }
  }
  // U' <- U' R, V' <- V' R (the stacked rows of X), written back in place
  if (e == cudaSuccess) e = gemm<false, kEpiLinear>(X, R, Xr, nullptr, n_rows, s, s, 1.f, 0.f, 1, st);
  if (e == cudaSuccess) {
    copy_kernel<<<blocks_for((size_t)n_rows * s, 256), 256, 0, st>>>(Xr, X, (size_t)n_rows * s);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace lb

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Newton-Schulz steps per polar factor: from Y = M / ||M||_F every singular
// value of Y is in (0, 1] and grows by up to 1.5x per step until it nears 1,
// then converges quadratically; 30 steps cover condition numbers of M up to
// about 1e3 / sqrt(s).
constexpr int kPolarSteps = 30;

}  // namespace

extern "C" {

lb_status littlebit_init_dual_svid(const float* Uf_dev, const float* Vf_dev, int d_out, int d_in, int s, int iters,
                                   void* U_bits_dev, void* V_bits_dev, uint16_t* h_dev, uint16_t* g_dev,
                                   uint16_t* l_dev, void* stream) {
  if (!Uf_dev || !Vf_dev || !U_bits_dev || !V_bits_dev || !h_dev || !g_dev || !l_dev) return LB_ERR_ARG;
  if (d_in < 256 || d_in % 256 != 0 || d_out < 128 || d_out % 128 != 0) return LB_ERR_SHAPE;
  if (s < 1 || s > lb::kMaxRank || iters < 1 || iters > 1000) return LB_ERR_SHAPE;
  if (!aligned16(Uf_dev) || !aligned16(Vf_dev) || !aligned16(U_bits_dev) || !aligned16(V_bits_dev)) return LB_ERR_ALIGN;
  if (!aligned16(h_dev) || !aligned16(g_dev) || (reinterpret_cast<uintptr_t>(l_dev) & 1)) return LB_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, lb::dual_svid_scratch_floats(d_out, d_in, s) * sizeof(float), st);
  if (e != cudaSuccess) return lb::cuda_fail(e);
  e = lb::launch_dual_svid(Uf_dev, Vf_dev, d_out, d_in, s, iters, U_bits_dev, V_bits_dev, h_dev, g_dev, l_dev, scratch,
                           st);
  const cudaError_t f = cudaFreeAsync(scratch, st);
  if (e == cudaSuccess) e = f;
  return e == cudaSuccess ? LB_OK : lb::cuda_fail(e);
}

lb_status littlebit_joint_itq(float* X_dev, int n_rows, int s, int iters, float* R_dev, int r_given, void* stream) {
  if (!X_dev || !R_dev) return LB_ERR_ARG;
  if (n_rows < 1 || s < 1 || s > lb::kMaxRank || iters < 0 || iters > 1000) return LB_ERR_SHAPE;
  if ((size_t)n_rows * s > ((size_t)1 << 31)) return LB_ERR_SHAPE;
  if (r_given != 0 && r_given != 1) return LB_ERR_ARG;
  if (!aligned16(X_dev) || !aligned16(R_dev)) return LB_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, lb::itq_scratch_floats(n_rows, s) * sizeof(float), st);
  if (e != cudaSuccess) return lb::cuda_fail(e);
  e = lb::launch_joint_itq(X_dev, n_rows, s, iters, kPolarSteps, R_dev, r_given, scratch, st);
  const cudaError_t f = cudaFreeAsync(scratch, st);
  if (e == cudaSuccess) e = f;
  return e == cudaSuccess ? LB_OK : lb::cuda_fail(e);
}

}  // extern "C"
