// Sign packing: real (or +-1) factor -> sign-plane tiles (layout in littlebit.h).
//
// The pages binarise the latent factors with sign() (LittleBit-2 column,
// chapter 2: "sign(U), sign(V)"; Samsung LittleBit article, section 2: factors
// binarised to +-1) and store one bit per entry (the s(a+b) term of the
// effective-bit formula).  Bit = [value < 0], so +0, -0 and NaN pack as +1.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lb_internal.h"

namespace lb {
namespace {

template <lb_dtype DT>
__device__ __forceinline__ bool is_negative(const void* src, int64_t idx) {
  if constexpr (DT == LB_F16) {
    return __half2float(static_cast<const __half*>(src)[idx]) < 0.f;
  } else if constexpr (DT == LB_BF16) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(src)[idx]) < 0.f;
  } else if constexpr (DT == LB_F32) {
    return static_cast<const float*>(src)[idx] < 0.f;
  } else {
    return static_cast<const int8_t*>(src)[idx] < 0;
  }
}

// One thread builds the 16 bytes of one lane of one tile.
template <lb_dtype DT, lb_role ROLE>
__global__ void __launch_bounds__(256) pack_kernel(const void* __restrict__ src, int n_long, int s,
                                                   int64_t stride_long, int64_t stride_s, int n_kt,
                                                   long long n_lanes, uint4* __restrict__ dst) {
  // logical matrix F: R x K ; role V: R = s, K = n_long ; role U: R = n_long, K = s
  const int R = (ROLE == LB_ROLE_V) ? s : n_long;
  const int K = (ROLE == LB_ROLE_V) ? n_long : s;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n_lanes;
       t += (long long)gridDim.x * blockDim.x) {
    const long long tile = t >> 5;
    const int lane = (int)(t & 31);
    const int rb = (int)(tile / n_kt), kt = (int)(tile % n_kt);
    const int g = lane >> 2, c = lane & 3;
    uint32_t w[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      uint32_t word = 0;
#pragma unroll
      for (int n = 0; n < 32; ++n) {
        const int m = n >> 3, q = n & 7;
        int row, k;
        if (ROLE == LB_ROLE_V) {
          row = 16 * rb + g + 8 * (r & 1);
          k = 256 * kt + 32 * q + 16 * (r >> 1) + 4 * c + m;
        } else {
          row = 128 * rb + 16 * q + g + 8 * (r & 1);
          k = 32 * kt + 16 * (r >> 1) + 4 * c + m;
        }
        if (row < R && k < K) {
          // role V: F[j][i] = V[i][j] -> natural element (a = i = k, j = row)
          // role U: F[o][j] = U[o][j] -> natural element (a = o = row, j = k)
          const int64_t a = (ROLE == LB_ROLE_V) ? k : row;
          const int64_t j = (ROLE == LB_ROLE_V) ? row : k;
          if (is_negative<DT>(src, a * stride_long + j * stride_s)) word |= 1u << n;
        }
      }
      w[r] = word;
    }
    dst[t] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <lb_dtype DT>
cudaError_t launch_dt(const void* src, int n_long, int s, int64_t sl, int64_t ss, lb_role role,
                      void* dst, cudaStream_t st) {
  const int R = (role == LB_ROLE_V) ? s : n_long;
  const int K = (role == LB_ROLE_V) ? n_long : s;
  const int tr = (role == LB_ROLE_V) ? kVTileRows : kUTileRows;
  const int tk = (role == LB_ROLE_V) ? kVTileK : kUTileK;
  const int n_rb = ceil_div(R, tr), n_kt = ceil_div(K, tk);
  const long long n_lanes = (long long)n_rb * n_kt * 32;
  const int threads = 256;
  long long blocks = (n_lanes + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (role == LB_ROLE_V)
    pack_kernel<DT, LB_ROLE_V><<<(int)blocks, threads, 0, st>>>(src, n_long, s, sl, ss, n_kt, n_lanes,
                                                                  static_cast<uint4*>(dst));
  else
    pack_kernel<DT, LB_ROLE_U><<<(int)blocks, threads, 0, st>>>(src, n_long, s, sl, ss, n_kt, n_lanes,
                                                                  static_cast<uint4*>(dst));
  return cudaGetLastError();
}

// Inverse of pack_kernel: one thread per element (a, j) of the natural
// n_long x s factor, written row-major as +-1 int8.  The (row, k) of the
// element in F gives its tile, lane, word and bit by inverting the layout.
template <lb_role ROLE>
__global__ void __launch_bounds__(256) unpack_kernel(const unsigned char* __restrict__ src, int n_long, int s,
                                                     int n_kt, int8_t* __restrict__ dst) {
  const long long total = (long long)n_long * s;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(t / s), j = (int)(t - (long long)a * s);
    const int row = (ROLE == LB_ROLE_V) ? j : a, k = (ROLE == LB_ROLE_V) ? a : j;
    int rb, kt, g, c, m, q, rlo, rhi;
    if (ROLE == LB_ROLE_V) {
      // row = 16 rb + g + 8 (r % 2),  k = 256 kt + 32 q + 16 (r / 2) + 4 c + m
      rb = row >> 4;
      g = row & 7;
      rlo = (row >> 3) & 1;
      kt = k >> 8;
      q = (k >> 5) & 7;
      rhi = (k >> 4) & 1;
      c = (k >> 2) & 3;
      m = k & 3;
    } else {
      // row = 128 rb + 16 q + g + 8 (r % 2),  k = 32 kt + 16 (r / 2) + 4 c + m
      rb = row >> 7;
      q = (row >> 4) & 7;
      g = row & 7;
      rlo = (row >> 3) & 1;
      kt = k >> 5;
      rhi = (k >> 4) & 1;
      c = (k >> 2) & 3;
      m = k & 3;
    }
    const int r = 2 * rhi + rlo, lane = 4 * g + c;
    const uint32_t word =
        *reinterpret_cast<const uint32_t*>(src + 512 * ((size_t)rb * n_kt + kt) + 16 * lane + 4 * r);
    dst[t] = ((word >> (8 * m + q)) & 1u) ? (int8_t)-1 : (int8_t)1;
  }
}

}  // namespace

cudaError_t launch_unpack(const void* src, int n_long, int s, lb_role role, int8_t* dst, cudaStream_t st) {
  const int K = (role == LB_ROLE_V) ? n_long : s;
  const int n_kt = ceil_div(K, (role == LB_ROLE_V) ? kVTileK : kUTileK);
  const long long total = (long long)n_long * s;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  const unsigned char* p = static_cast<const unsigned char*>(src);
  if (role == LB_ROLE_V) unpack_kernel<LB_ROLE_V><<<(int)blocks, 256, 0, st>>>(p, n_long, s, n_kt, dst);
  else unpack_kernel<LB_ROLE_U><<<(int)blocks, 256, 0, st>>>(p, n_long, s, n_kt, dst);
  return cudaGetLastError();
}

cudaError_t launch_pack(const void* src, lb_dtype dt, int n_long, int s, int64_t stride_long,
                        int64_t stride_s, lb_role role, void* dst, cudaStream_t st) {
  switch (dt) {
    case LB_F16: return launch_dt<LB_F16>(src, n_long, s, stride_long, stride_s, role, dst, st);
    case LB_BF16: return launch_dt<LB_BF16>(src, n_long, s, stride_long, stride_s, role, dst, st);
    case LB_F32: return launch_dt<LB_F32>(src, n_long, s, stride_long, stride_s, role, dst, st);
    case LB_I8: return launch_dt<LB_I8>(src, n_long, s, stride_long, stride_s, role, dst, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lb
