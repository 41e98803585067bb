// Decode forward (batch 1..16) of the LittleBit layer on sm_100a.
//
//   y = sum_p h_p (.) ( U_p ( l_p (.) ( V_p^T ( g_p (.) x ) ) ) )
// (Samsung LittleBit article, section 2: two binary matrix products plus
// elementwise scaling, residual paths added).
//
// Both binary products run on the int8 tensor cores (mma.sync m16n8k32,
// u8 x s8 -> s32) without unpacking the signs.  The packed layout stores, for
// each lane of a 512-byte tile, the four 32-bit A-fragment registers of eight
// m16n8k32 products at once: bit q of every byte belongs to product q.  So
// `word & (0x01010101 << q)` is that product's A register with entries
// {0, 2^q}; one logic op per four signs, and the product's sum carries a known
// factor 2^q that is shifted out once per output (exact integer arithmetic).
// The B operand is the vector (g*x for the latent pass, t' = l*t for the
// output pass) quantised to 16 bits, v = scale * (256*hi + lo), hi and lo being
// two int8 columns; for a +-1 sign b = 1 - 2*bit,
//     sum_k sign_k v_k = sum_k v_k - 2 * sum_k bit_k v_k.
// Columns 2r and 2r+1 of the 8-column product hold batch row r's hi and lo
// bytes, so one product serves four batch rows.
//
// Latent pass: CTA = (layer, path, 4096-input slice); each warp owns 4 tiles of
// the slice and walks all 16-row latent blocks; the slice's exact integer sums
// are combined in shared memory and written as one fp32 partial per latent
// row.  The CTA that finishes a path's last slice (atomic ticket, no waiting)
// sums the partials in slice order, multiplies by l and quantises t'.
// Output pass: warp = (layer, 128 output rows); walks the role-U tiles of both
// paths, scales by the quantisation step and h, adds the paths, writes fp16.
#include <cuda_fp16.h>

#include "lb_internal.h"

namespace lb {
namespace {

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float h2f(uint16_t v) { return __half2float(__ushort_as_half(v)); }
__device__ __forceinline__ uint16_t f2h(float v) { return __half_as_ushort(__float2half_rn(v)); }

__device__ __forceinline__ const LayerDesc& find_layer(const DecodeArgs& a, int item, bool latent) {
  int lo = 0, hi = a.n_layers - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int begin = latent ? a.layers[mid].v_begin : a.layers[mid].u_begin;
    if (begin <= item) lo = mid; else hi = mid - 1;
  }
  return a.layers[lo];
}

// quantise to v = 256*hi + lo; returns v and writes the two int8 bytes
__device__ __forceinline__ int quantise(float u, float inv, int8_t& hi, int8_t& lo) {
  int v = __float2int_rn(u * inv);
  v = max(-32639, min(32639, v));
  const int h = (v + 128) >> 8;   // floor((v + 128) / 256) in [-127, 127]
  hi = (int8_t)h;
  lo = (int8_t)(v - 256 * h);     // in [-128, 127]
  return v;
}

template <int NB>
__device__ __forceinline__ void block_reduce_max_sum(float (&mx)[4 * NB], int (&sm)[4 * NB],
                                                     float (*s_mx)[16], int (*s_sm)[16], int B) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < 4 * NB; ++b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx[b] = fmaxf(mx[b], __shfl_xor_sync(0xffffffffu, mx[b], o));
      sm[b] += __shfl_xor_sync(0xffffffffu, sm[b], o);
    }
    if (lane == 0 && b < B) { s_mx[warp][b] = mx[b]; s_sm[warp][b] = sm[b]; }
  }
  __syncthreads();
#pragma unroll
  for (int b = 0; b < 4 * NB; ++b) {
    if (b < B) {
      float m = s_mx[0][b];
      int ssum = s_sm[0][b];
#pragma unroll
      for (int w = 1; w < kVWarps; ++w) { m = fmaxf(m, s_mx[w][b]); ssum += s_sm[w][b]; }
      mx[b] = m;
      sm[b] = ssum;
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// latent pass:  t_j (partial over one slice) = sum_i V[i][j] g_i x_i
// ---------------------------------------------------------------------------
template <int NB>
__global__ void __launch_bounds__(kVWarps * 32) latent_pass_kernel(const DecodeArgs a) {
  constexpr int NCOL = 8 * NB;
  extern __shared__ __align__(16) unsigned char smem[];
  int8_t* bpl = reinterpret_cast<int8_t*>(smem);                         // [kVSlice/32][NCOL][32]
  int* acc = reinterpret_cast<int*>(smem + (size_t)kVSlice * NCOL);      // [B][S16] (or fp32 t')
  __shared__ float s_mx[kVWarps][16];
  __shared__ int s_sm[kVWarps][16];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int B = a.batch;

  for (int item = blockIdx.x; item < a.v_items; item += gridDim.x) {
    const LayerDesc& L = find_layer(a, item, true);
    const int rel = item - L.v_begin;
    const int p = rel / L.n_slices, sl = rel - p * L.n_slices;
    const PathDesc& P = L.p[p];
    const int d_in = L.d_in, s = L.s;
    const int S16 = (s + 15) & ~15;
    const int k0 = sl * kVSlice;
    const int klen = min(kVSlice, d_in - k0);          // multiple of 256
    const int n_kt_all = d_in / kVTileK;

    // ---- 1. u = g * x on the slice: per-row max |u| and the quantisation step
    float mx[4 * NB];
    int vs[4 * NB];
#pragma unroll
    for (int b = 0; b < 4 * NB; ++b) { mx[b] = 0.f; vs[b] = 0; }
    for (int k = tid; k < klen; k += kVWarps * 32) {
      const float gk = h2f(P.g[k0 + k]);
#pragma unroll
      for (int b = 0; b < 4 * NB; ++b)
        if (b < B) mx[b] = fmaxf(mx[b], fabsf(gk * h2f(L.x[(size_t)b * d_in + k0 + k])));
    }
    block_reduce_max_sum<NB>(mx, vs, s_mx, s_sm, B);
    float inv[4 * NB], step[4 * NB];
#pragma unroll
    for (int b = 0; b < 4 * NB; ++b) {
      inv[b] = mx[b] > 0.f ? kQMax / mx[b] : 0.f;
      step[b] = mx[b] > 0.f ? mx[b] / kQMax : 0.f;
    }
    // ---- 2. quantised planes into the B-operand staging area; sum of v
    for (int k = tid; k < klen; k += kVWarps * 32) {
      const float gk = h2f(P.g[k0 + k]);
      int8_t* col = bpl + (size_t)(k >> 5) * NCOL * 32 + (k & 31);
#pragma unroll
      for (int b = 0; b < 4 * NB; ++b) {
        int8_t hi = 0, lo = 0;
        if (b < B) vs[b] += quantise(gk * h2f(L.x[(size_t)b * d_in + k0 + k]), inv[b], hi, lo);
        const int n = (b >> 2) * 8 + (b & 3) * 2;   // column of (row b, hi); lo is n + 1
        col[n * 32] = hi;
        col[(n + 1) * 32] = lo;
      }
    }
    block_reduce_max_sum<NB>(mx, vs, s_mx, s_sm, B);   // mx unchanged; vs = slice sum of v
    for (int i = tid; i < B * S16; i += kVWarps * 32) acc[i] = 0;
    __syncthreads();

    // ---- 3. warp w: tiles 4w..4w+3 of the slice, all 16-row latent blocks
    const int nt = max(0, min(kVTilesPerWarp, klen / kVTileK - kVTilesPerWarp * warp));
    const int kt0 = k0 / kVTileK + kVTilesPerWarp * warp;   // first global K-tile of this warp
    uint32_t bf[NB == 1 ? kVTilesPerWarp * 8 : 1][2];
    if constexpr (NB == 1) {
#pragma unroll
      for (int t = 0; t < kVTilesPerWarp; ++t)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int kb = (kVTilesPerWarp * warp + t) * 8 + q;
          const int8_t* base = bpl + ((size_t)kb * NCOL + g) * 32 + 4 * c;
          bf[t * 8 + q][0] = *reinterpret_cast<const uint32_t*>(base);
          bf[t * 8 + q][1] = *reinterpret_cast<const uint32_t*>(base + 16);
        }
    }
    const int n_rb = S16 / 16;
    const uint4* vt = P.V + (size_t)lane;
    uint4 cur[kVTilesPerWarp], nxt[kVTilesPerWarp];
#pragma unroll
    for (int t = 0; t < kVTilesPerWarp; ++t)
      cur[t] = (t < nt) ? ld_stream(vt + ((size_t)0 * n_kt_all + kt0 + t) * 32) : make_uint4(0, 0, 0, 0);
    for (int rb = 0; rb < n_rb; ++rb) {
      if (rb + 1 < n_rb) {
#pragma unroll
        for (int t = 0; t < kVTilesPerWarp; ++t)
          nxt[t] = (t < nt) ? ld_stream(vt + ((size_t)(rb + 1) * n_kt_all + kt0 + t) * 32)
                            : make_uint4(0, 0, 0, 0);
      }
      int d[8][NB][4];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) d[q][nb][0] = d[q][nb][1] = d[q][nb][2] = d[q][nb][3] = 0;
#pragma unroll
      for (int t = 0; t < kVTilesPerWarp; ++t) {
        if (t < nt) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t m = 0x01010101u << q;
            const uint32_t a0 = cur[t].x & m, a1 = cur[t].y & m, a2 = cur[t].z & m, a3 = cur[t].w & m;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              uint32_t b0, b1;
              if constexpr (NB == 1) {
                b0 = bf[t * 8 + q][0];
                b1 = bf[t * 8 + q][1];
              } else {
                const int kb = (kVTilesPerWarp * warp + t) * 8 + q;
                const int8_t* base = bpl + ((size_t)kb * NCOL + nb * 8 + g) * 32 + 4 * c;
                b0 = *reinterpret_cast<const uint32_t*>(base);
                b1 = *reinterpret_cast<const uint32_t*>(base + 16);
              }
              mma_u8s8(d[q][nb], a0, a1, a2, a3, b0, b1);
            }
          }
        }
      }
      // fold: sum_q (256*D_hi + D_lo) / 2^q, Horner from q = 7 down (exact)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        int r0 = 256 * d[7][nb][0] + d[7][nb][1];
        int r1 = 256 * d[7][nb][2] + d[7][nb][3];
#pragma unroll
        for (int q = 6; q >= 0; --q) {
          r0 = (r0 >> 1) + 256 * d[q][nb][0] + d[q][nb][1];
          r1 = (r1 >> 1) + 256 * d[q][nb][2] + d[q][nb][3];
        }
        const int b = 4 * nb + c;
        if (b < B && nt > 0) {
          atomicAdd(&acc[b * S16 + 16 * rb + g], r0);
          atomicAdd(&acc[b * S16 + 16 * rb + g + 8], r1);
        }
      }
#pragma unroll
      for (int t = 0; t < kVTilesPerWarp; ++t) cur[t] = nxt[t];
    }
    __syncthreads();

    // ---- 4. slice partial: step * (sum v - 2 * sum bit*v)
    float* part = P.ws.partial + (size_t)sl * B * S16;
    for (int i = tid; i < B * S16; i += kVWarps * 32) {
      const int b = i / S16;
      float st = 0.f;
      int vsum = 0;
#pragma unroll
      for (int bb = 0; bb < 4 * NB; ++bb)
        if (bb == b) { st = step[bb]; vsum = vs[bb]; }
      part[i] = st * (float)(vsum - 2 * acc[i]);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(P.ws.counter, 1u) == (unsigned)(L.n_slices - 1));
    __syncthreads();

    if (s_last) {
      // ---- 5. last slice of this path: t' = l * sum of partials, quantised
      __threadfence();
      float* tp = reinterpret_cast<float*>(acc);
      float mt[4 * NB];
      int ts[4 * NB];
#pragma unroll
      for (int b = 0; b < 4 * NB; ++b) { mt[b] = 0.f; ts[b] = 0; }
      for (int i = tid; i < B * S16; i += kVWarps * 32) {
        const int b = i / S16, j = i - b * S16;
        float t = 0.f;
        if (j < s) {
          for (int q = 0; q < L.n_slices; ++q) t += __ldcg(P.ws.partial + ((size_t)q * B) * S16 + i);
          t *= h2f(P.l[j]);
        }
        tp[i] = t;
#pragma unroll
        for (int bb = 0; bb < 4 * NB; ++bb)
          if (bb == b) mt[bb] = fmaxf(mt[bb], fabsf(t));
      }
      block_reduce_max_sum<NB>(mt, ts, s_mx, s_sm, B);
      const int S32 = (s + 31) & ~31;
      for (int i = tid; i < B * S32; i += kVWarps * 32) {
        const int b = i / S32, j = i - b * S32;
        float tinv = 0.f;
#pragma unroll
        for (int bb = 0; bb < 4 * NB; ++bb)
          if (bb == b) tinv = mt[bb] > 0.f ? kQMax / mt[bb] : 0.f;
        int8_t hi = 0, lo = 0;
        if (j < s) {
          const int v = quantise(tp[b * S16 + j], tinv, hi, lo);
#pragma unroll
          for (int bb = 0; bb < 4 * NB; ++bb)
            if (bb == b) ts[bb] += v;
        }
        P.ws.planes[(size_t)(b * 2) * S32 + j] = hi;
        P.ws.planes[(size_t)(b * 2 + 1) * S32 + j] = lo;
      }
      block_reduce_max_sum<NB>(mt, ts, s_mx, s_sm, B);
      if (tid < B) {
        float m = 0.f;
        int sum = 0;
#pragma unroll
        for (int bb = 0; bb < 4 * NB; ++bb)
          if (bb == tid) { m = mt[bb]; sum = ts[bb]; }
        P.ws.tscale[tid] = m > 0.f ? m / kQMax : 0.f;
        P.ws.tsum[tid] = sum;
      }
      if (tid == 0) *P.ws.counter = 0u;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// output pass:  y_o = sum_p h_p[o] * sum_j U_p[o][j] t'_p[j]
// ---------------------------------------------------------------------------
template <int NB>
__global__ void __launch_bounds__(kUWarps * 32) output_pass_kernel(const DecodeArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int B = a.batch;
  for (int item = blockIdx.x * kUWarps + warp; item < a.u_items; item += gridDim.x * kUWarps) {
    const LayerDesc& L = find_layer(a, item, false);
    const int ob = item - L.u_begin;
    const int s = L.s, S32 = (s + 31) & ~31, n_kt = S32 / kUTileK;
    float yacc[8][2][NB];
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) yacc[q][0][nb] = yacc[q][1][nb] = 0.f;

    for (int p = 0; p < L.npaths; ++p) {
      const PathDesc& P = L.p[p];
      int d[8][NB][4];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) d[q][nb][0] = d[q][nb][1] = d[q][nb][2] = d[q][nb][3] = 0;
      const uint4* ut = P.U + (size_t)ob * n_kt * 32 + lane;
      uint4 w = ld_stream(ut);
      for (int kt = 0; kt < n_kt; ++kt) {
        const uint4 cur = w;
        if (kt + 1 < n_kt) w = ld_stream(ut + (size_t)(kt + 1) * 32);
        uint32_t b0[NB], b1[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const int b = 4 * nb + (g >> 1);
          if (b < B) {
            const int8_t* pl = P.ws.planes + (size_t)(b * 2 + (g & 1)) * S32 + kt * 32 + 4 * c;
            b0[nb] = *reinterpret_cast<const uint32_t*>(pl);
            b1[nb] = *reinterpret_cast<const uint32_t*>(pl + 16);
          } else {
            b0[nb] = b1[nb] = 0u;
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t m = 0x01010101u << q;
          const uint32_t a0 = cur.x & m, a1 = cur.y & m, a2 = cur.z & m, a3 = cur.w & m;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) mma_u8s8(d[q][nb], a0, a1, a2, a3, b0[nb], b1[nb]);
        }
      }
      // epilogue of this path: rows 128ob + 16q + g (+8), batch row 4nb + c
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int b = 4 * nb + c;
        if (b < B) {
          const float st = P.ws.tscale[b];
          const int tsum = P.ws.tsum[b];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int c0 = ((d[q][nb][0] >> q) << 8) + (d[q][nb][1] >> q);
            const int c1 = ((d[q][nb][2] >> q) << 8) + (d[q][nb][3] >> q);
            const int o0 = ob * kUTileRows + 16 * q + g;
            yacc[q][0][nb] += h2f(P.h[o0]) * (st * (float)(tsum - 2 * c0));
            yacc[q][1][nb] += h2f(P.h[o0 + 8]) * (st * (float)(tsum - 2 * c1));
          }
        }
      }
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int b = 4 * nb + c;
      if (b < B) {
        uint16_t* yr = L.y + (size_t)b * L.d_out + ob * kUTileRows + g;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          yr[16 * q] = f2h(yacc[q][0][nb]);
          yr[16 * q + 8] = f2h(yacc[q][1][nb]);
        }
      }
    }
  }
}

template <int NB>
size_t smem_bytes(int batch, int max_s16) {
  return (size_t)kVSlice * 8 * NB + (size_t)batch * max_s16 * 4;
}

template <int NB>
cudaError_t launch_latent(const DecodeArgs& a, int max_s16, int num_sms, cudaStream_t st) {
  const size_t smem = smem_bytes<NB>(a.batch, max_s16);
  cudaError_t e = cudaFuncSetAttribute(latent_pass_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, latent_pass_kernel<NB>, kVWarps * 32, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int grid = max(1, min(a.v_items, per_sm * num_sms));
  latent_pass_kernel<NB><<<grid, kVWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

template <int NB>
cudaError_t launch_output(const DecodeArgs& a, int num_sms, cudaStream_t st) {
  int per_sm = 0;
  cudaError_t e =
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, output_pass_kernel<NB>, kUWarps * 32, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int grid = max(1, min((a.u_items + kUWarps - 1) / kUWarps, per_sm * num_sms));
  output_pass_kernel<NB><<<grid, kUWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t latent_pass_smem(int batch, int max_s16) {
  const int nb = (batch + 3) / 4;
  return (size_t)kVSlice * 8 * nb + (size_t)batch * max_s16 * 4;
}

cudaError_t launch_latent_pass(const DecodeArgs& a, int max_s16, int num_sms, cudaStream_t st) {
  switch ((a.batch + 3) / 4) {
    case 1: return launch_latent<1>(a, max_s16, num_sms, st);
    case 2: return launch_latent<2>(a, max_s16, num_sms, st);
    case 3: return launch_latent<3>(a, max_s16, num_sms, st);
    case 4: return launch_latent<4>(a, max_s16, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_output_pass(const DecodeArgs& a, int num_sms, cudaStream_t st) {
  switch ((a.batch + 3) / 4) {
    case 1: return launch_output<1>(a, num_sms, st);
    case 2: return launch_output<2>(a, num_sms, st);
    case 3: return launch_output<3>(a, num_sms, st);
    case 4: return launch_output<4>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lb
