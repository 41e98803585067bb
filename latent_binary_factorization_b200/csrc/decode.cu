// Decode forward (batch 1..16) of the LittleBit layer on sm_100a.
//
//   y = sum_p h_p (.) ( U_p ( l_p (.) ( V_p^T ( g_p (.) x ) ) ) )
// (Samsung LittleBit article, section 2: two binary matrix products plus
// elementwise scaling, residual paths added).
//
// Arithmetic.  Both binary products run on the int8 tensor cores
// (mma.sync m16n8k32, u8 x s8 -> s32) without unpacking the signs.  The packed
// layout stores, for each lane of a 512-byte tile, the four 32-bit A-fragment
// registers of eight m16n8k32 products at once: bit q of every byte belongs to
// product q.  So `word & (0x01010101 << q)` is that product's A register with
// entries {0, 2^q}; one logic op per four signs, and the product's sum carries
// a known factor 2^q that is shifted out exactly in integer arithmetic.  The B
// operand is the vector (g*x for the latent pass, t' = l*t for the output
// pass) quantised to 16 bits, v = step * (256*hi + lo), hi and lo being two
// int8 columns; for a +-1 sign s = 1 - 2*bit,
//     sum_k s_k v_k = sum_k v_k - 2 * sum_k bit_k v_k.
// Columns 2r and 2r+1 of an 8-column product hold batch row r's hi and lo
// bytes, so one product serves four batch rows.
//
// Data movement.  Sign tiles stream from HBM into a per-warp ring of shared
// memory stages with bulk async copies (cp.async.bulk, completion counted on
// an mbarrier per stage); the warp issues the copy for chunk c + stages as soon
// as it has read chunk c, so a few KB per warp stay in flight without holding
// registers.  Every wait is bounded: after kSpinLimit polls the kernel sets
// LB_ERR_TIMEOUT in the status word and stops waiting.
//
// Four launches, in stream order, chained by programmatic dependent launch
// (each later kernel starts early and waits for its predecessor's output):
// quantise: warp per (layer, path, 2048-input slice) quantises u = g*x per
//   batch row and stores it as int8 B fragments with the step and sum per row.
// latent:   CTA item = (layer, path, slice, 2W latent 16-row blocks) for a
//   CTA of W = 3 or 4 warps; the slice's B fragments arrive by one bulk copy
//   into a double buffer, warp w streams row blocks 2w, 2w+1 over the slice
//   and writes one fp32 partial sum per latent row and slice.
// finalize: CTA per (layer, path) sums the partials in slice order, multiplies
//   by l and quantises t' to int8 hi/lo planes with a step per batch row.
// output:   warp item = (layer, 128 output rows); each warp owns a contiguous
//   item range and streams it as chunks of up to 8 K-tiles, across path, item
//   and layer boundaries; the bulk copies also bring the chunk's t' bytes and,
//   for the last chunk of a path, the 128 h values and the quantisation step.
//   Paths are added in fp32 and y is written in fp16.  At batch 1 with
//   residual layers the two paths share one accumulator (packed form).
#include <cuda_fp16.h>

#include "lb_internal.h"

namespace lb {
namespace {

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// global -> shared bulk copy (no multicast); 16-byte aligned, size % 16 == 0
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// try_wait may suspend the warp for up to this long before reporting "not yet"
constexpr uint32_t kWaitHintNs = 1000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitHintNs)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity` of `bar`.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Plain arrival (no transaction bytes) on `bar`.
__device__ __forceinline__ void mbar_arrive_one(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait for phase `parity` of `bar`; false after kSpinLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (int i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Programmatic dependent launch: a kernel launched with the programmatic
// stream serialization attribute may start before the previous kernel in the
// stream has finished; grid_dep_wait() returns once that kernel has completed
// and its writes are visible.  grid_dep_launch() lets the next such kernel
// start launching.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint4 ld_nc(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A*B (accumulator starts at zero)
__device__ __forceinline__ void mma_u8s8_zc(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ float2 h2x2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}
__device__ __forceinline__ float h2f(uint16_t v) { return __half2float(__ushort_as_half(v)); }
__device__ __forceinline__ uint16_t f2h(float v) { return __half_as_ushort(__float2half_rn(v)); }

// Layer of a work item: one load from the item's map (no map with one layer).
__device__ __forceinline__ int layer_of(const int* map, int n_layers, int item) {
  return n_layers == 1 ? 0 : __ldg(map + item);
}

// ---------------------------------------------------------------------------
// quantise pass:  u = g_p (.) x on one 2048-input slice of one layer, for each
// path p, quantised per batch row to 16 bits, v = step * (256*hi + lo), and
// stored as the latent pass's int8 B fragments (slice block layout in
// lb_internal.h).  One warp per (group of layers reading one x, slice, up to
// kQRows batch rows): lane i holds the 8-input chunks i + 32j (j < 8) of one
// batch row at a time; max and sum are warp reductions, so the kernel has no
// CTA barrier.
//
// Arithmetic per value: u = g*x in fp32 (exact for fp16 operands); v =
// round(u * 32639 / max|u|) by adding 1.5*2^23 in fp32, which leaves v in the
// low bits of the float's encoding: its low byte is the int8 lo byte of
// v = 256*hi + lo, and byte 1 of (encoding + 128) is hi.  |v| <= 32639 holds
// because max|u| is taken over the same fp32 values.
// ---------------------------------------------------------------------------
constexpr int kQWarps = 4;                          // warps (slices) per CTA
constexpr int kQChunks = kVSlice / 8 / 32;          // 8-input chunks per lane
constexpr float kRoundMagic = 12582912.f;           // 1.5 * 2^23

// byte b (0 or 1) of a, c, d, e packed low to high
__device__ __forceinline__ uint32_t pack_byte(uint32_t a, uint32_t c, uint32_t d, uint32_t e, int b) {
  const uint32_t sel = b == 0 ? 0x0040u : 0x0051u;   // {a.b, c.b} into the low half
  const uint32_t lo = __byte_perm(a, c, sel), hi = __byte_perm(d, e, sel);
  return __byte_perm(lo, hi, 0x5410);
}

// One (layer, path): u = g (.) x for one batch row from the lane's x chunks,
// quantised and stored in the slice block at `blk`.
__device__ __forceinline__ void quantise_row(const uint4 (&xq)[kQChunks], const uint16_t* __restrict__ g, int k0,
                                             int nchunk, int row, int NC, int lane, unsigned char* blk, int B) {
  uint32_t* frag = reinterpret_cast<uint32_t*>(blk + xq_stats_bytes(B));
  // u = g * x is formed twice (for the max, then for the codes) rather than
  // held: 64 more live registers would halve the resident warps
  float mx = 0.f;
#pragma unroll
  for (int j = 0; j < kQChunks; ++j) {
    const int ch = lane + 32 * j;
    const uint4 gq = ch < nchunk ? ld_nc(g + k0 + 8 * ch) : make_uint4(0, 0, 0, 0);
    const uint32_t* xw = &xq[j].x;
    const uint32_t* gw = &gq.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 xf = h2x2(xw[e]), gf = h2x2(gw[e]);
      mx = fmaxf(mx, fmaxf(fabsf(xf.x * gf.x), fabsf(xf.y * gf.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float inv = mx > 0.f ? kQMax / mx : 0.f;
  int sum_hi = 0, sum_lo = 0;
#pragma unroll
  for (int j = 0; j < kQChunks; ++j) {
    const int ch = lane + 32 * j;
    const uint4 gq = ch < nchunk ? ld_nc(g + k0 + 8 * ch) : make_uint4(0, 0, 0, 0);
    const uint32_t* xw = &xq[j].x;
    const uint32_t* gw = &gq.x;
    uint32_t fb[8], fh[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 xf = h2x2(xw[e]), gf = h2x2(gw[e]);
      fb[2 * e] = __float_as_uint(fmaf(xf.x * gf.x, inv, kRoundMagic));
      fb[2 * e + 1] = __float_as_uint(fmaf(xf.y * gf.y, inv, kRoundMagic));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) fh[e] = fb[e] + 128u;
    const uint32_t lw0 = pack_byte(fb[0], fb[1], fb[2], fb[3], 0), lw1 = pack_byte(fb[4], fb[5], fb[6], fb[7], 0);
    const uint32_t hw0 = pack_byte(fh[0], fh[1], fh[2], fh[3], 1), hw1 = pack_byte(fh[4], fh[5], fh[6], fh[7], 1);
    sum_hi = __dp4a((int)hw0, 0x01010101, __dp4a((int)hw1, 0x01010101, sum_hi));
    sum_lo = __dp4a((int)lw0, 0x01010101, __dp4a((int)lw1, 0x01010101, sum_lo));
    if (ch < nchunk) {
      // inputs 8ch..8ch+7: K-block kb, offset kk0 (0, 8, 16, 24) inside it;
      // kk < 16 -> b0 words of threads c = kk/4, else b1 words of c = (kk-16)/4
      const int kb = ch >> 2, kk0 = (ch & 3) * 8;
      const int cc = (kk0 & 15) >> 2, half = kk0 >> 4;
      uint32_t* fhp = frag + ((size_t)kb * NC + 2 * row) * 8;   // column 2*row: 4 threads x (b0, b1)
      uint32_t* flp = fhp + 8;                                  // column 2*row + 1
      fhp[2 * cc + half] = hw0;
      fhp[2 * (cc + 1) + half] = hw1;
      flp[2 * cc + half] = lw0;
      flp[2 * (cc + 1) + half] = lw1;
    }
  }
  int vsum = 256 * sum_hi + sum_lo;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vsum += __shfl_xor_sync(0xffffffffu, vsum, o);
  if (lane == 0) {
    TStat st;
    st.step = mx > 0.f ? mx / kQMax : 0.f;
    st.sum = vsum;
    st.pad[0] = st.pad[1] = 0;
    reinterpret_cast<TStat*>(blk)[row] = st;
  }
}

// Work item = (group of layers that read the same x, 2048-input slice, group
// of kQRows batch rows): the item reads each of its batch rows' x slice once
// and quantises g (.) x for every path of every layer of the group (layers
// chained by x_next from the group's first layer, whose x_begin numbers the
// group's items, slice-major).
__global__ void __launch_bounds__(kQWarps * 32) quantise_input_kernel(const DecodeArgs a) {
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * kQWarps + (threadIdx.x >> 5);
  if (item >= a.x_items) return;
  const int B = a.batch, NC = 2 * xq_rows(B);
  const int first = layer_of(a.item_layer.x, a.n_layers, item);
  const LayerDesc& L0 = a.layers[first];
  const int n_rg = (B + kQRows - 1) / kQRows, rel = item - L0.x_begin;
  const int sl = rel / n_rg, rg = rel - sl * n_rg;
  const int d_in = L0.d_in, k0 = sl * kVSlice;
  const int nchunk = min(kVSlice, d_in - k0) / 8;
  const size_t blk_off = (size_t)sl * xq_slice_bytes(B);

  unsigned bad = 0;   // an input x that is inf or NaN (LB_ERR_RANGE)
  // rows B .. 4*nb-1 of a block are never read: their product columns are
  // independent of the batch rows' and their sums are discarded
  const int row_end = min(B, kQRows * (rg + 1));
#pragma unroll 1
  for (int row = kQRows * rg; row < row_end; ++row) {
    uint4 xq[kQChunks];
#pragma unroll
    for (int j = 0; j < kQChunks; ++j) {
      const int ch = lane + 32 * j;
      xq[j] = ch < nchunk ? ld_nc(L0.x + (size_t)row * d_in + k0 + 8 * ch) : make_uint4(0, 0, 0, 0);
      bad |= half2_nonfinite(xq[j].x) | half2_nonfinite(xq[j].y) | half2_nonfinite(xq[j].z) |
             half2_nonfinite(xq[j].w);
    }
#pragma unroll 1
    for (int li = first; li >= 0; li = a.layers[li].x_next) {
      const LayerDesc& L = a.layers[li];
#pragma unroll 1
      for (int p = 0; p < L.npaths; ++p)
        quantise_row(xq, L.p[p].g, k0, nchunk, row, NC, lane, L.p[p].ws.xq + blk_off, B);
    }
  }
  if (__any_sync(0xffffffffu, bad != 0) && lane == 0) atomicOr(a.status, kStatusRange);
}

// ---------------------------------------------------------------------------
// latent pass:  t_j (partial over one slice) = sum_i V[i][j] g_i x_i
// ---------------------------------------------------------------------------
// CTA item = (layer, path, 2048-input slice, 8 latent row blocks; 6 with three
// warps).  The slice's quantised input (B fragments and per-row step) arrives
// by one bulk copy into one of two shared buffers; warp w takes row blocks 2w,
// 2w+1 (w alone in the eight-warp CTAs of batches 9-16) and accumulates their
// eight products per K-block over the whole slice (at batch 1-4 one B fragment
// load feeds both blocks), then folds the 2^q factors once and writes one fp32
// partial per latent row.
//
// Buffer hand-over without CTA barriers: the CTA's items are walked by every
// warp in the same order, so each warp sees the same sequence of distinct
// slices.  Slice n uses buffer n % 2.  A warp that moves on from slice n - 1
// counts itself done on that buffer (shared atomic); the warp that completes
// the count issues the copy of slice n + 1 into it.  Every warp then waits for
// slice n's copy (bounded).

struct VItem {
  int li, p, sl, rc;
};

// decode `item` into (layer, path, slice, row chunk); li walks forward
__device__ __forceinline__ VItem decode_v(const DecodeArgs& a, int item, int& li) {
  while (li + 1 < a.n_layers && a.layers[li + 1].v_begin <= item) ++li;
  const LayerDesc& L = a.layers[li];
  int rel = item - L.v_begin;
  const int per_path = L.n_slices * L.n_rchunks;
  VItem it;
  it.li = li;
  it.p = rel / per_path;
  rel -= it.p * per_path;
  it.sl = rel / L.n_rchunks;
  it.rc = rel - it.sl * L.n_rchunks;
  return it;
}

// A latent-pass item's coordinates and its layer's constants, advanced one
// item at a time by comparisons only (items run path-major, then slice, then
// row chunk, layer after layer).
struct VPos {
  int item, li, p, sl, rc;
  const LayerDesc* L;   // the layer's counts are read from its (cached) descriptor

  __device__ __forceinline__ void load(const DecodeArgs& a) { L = a.layers + li; }
  // position at `it`, whose layer is li0 or a later one
  __device__ __forceinline__ void start(const DecodeArgs& a, int it, int li0) {
    int l = li0;
    const VItem v = decode_v(a, it, l);
    item = it;
    li = l;
    p = v.p;
    sl = v.sl;
    rc = v.rc;
    load(a);
  }
  __device__ __forceinline__ void next(const DecodeArgs& a) {
    ++item;
    if (++rc < L->n_rchunks) return;
    rc = 0;
    if (++sl < L->n_slices) return;
    sl = 0;
    if (++p < L->npaths) return;
    p = 0;
    if (li + 1 < a.n_layers) {
      ++li;
      load(a);
    }
  }
};

// Row blocks a warp processes at once: two share each B-fragment load; with
// more than four batch rows the accumulators would not fit, so one.
template <int NB>
struct VCfg {
  static constexpr int kRPW = NB == 1 ? 2 : 1;
};

// Row blocks of a latent-pass item per warp: an item is 8 row blocks (6 with
// three warps), two per warp, or one per warp in the eight-warp CTAs.
__host__ __device__ constexpr int latent_rows_per_warp(int W) { return W == 8 ? 1 : 2; }

// Bytes of one quantised input slice buffer (shared memory and global stride).
__host__ __device__ constexpr int xq_buf_bytes(int nb, int rb) { return (64 * nb + kVSlice * 2 * rb + 127) & ~127; }

// Copy the quantised slice of `item` (from its first byte to the end of its
// last K-block) into `dst`, completion on `bar`.
template <int NB, int RB>
__device__ __forceinline__ void x_issue(const DecodeArgs& a, int item, int li, unsigned char* dst, uint64_t* bar) {
  const VItem it = decode_v(a, item, li);
  const LayerDesc& L = a.layers[it.li];
  const int klen = min(kVSlice, L.d_in - it.sl * kVSlice);
  const uint32_t bytes = 64 * NB + klen * 2 * RB;
  mbar_expect_tx(bar, bytes);
  bulk_g2s(dst, L.p[it.p].ws.xq + (size_t)it.sl * xq_buf_bytes(NB, RB), bytes, bar);
}

// One warp's sequence of bulk-copy chunks: per item, per group of kRPW row
// blocks, per 4 K-tiles of the slice.
template <int NB, int W>
struct VFeed {
  static constexpr int RPW = VCfg<NB>::kRPW;
  static constexpr int kRW = latent_rows_per_warp(W);
  VPos pos;
  int item, grp, kc;
  int rb0, n_rb, n_kt_all, kt0, nkt;   // current item
  const unsigned char* V;

  // the current item's chunk parameters (from pos; no divisions)
  __device__ __forceinline__ void set(int warp) {
    static_assert(W == 3 || W == 4 || W == 8, "latent-pass CTA width");
    item = pos.item;
    const int k0 = pos.sl * kVSlice, d_in = pos.L->d_in;
    nkt = min(kVSliceTiles, (d_in - k0) / kVTileK);
    n_kt_all = d_in / kVTileK;
    kt0 = k0 / kVTileK;
    n_rb = (pos.L->s + 15) >> 4;
    rb0 = pos.rc * (W * kRW) + kRW * warp;
    V = reinterpret_cast<const unsigned char*>(pos.L->p[pos.p].V);
    grp = 0;
    kc = 0;
  }
  __device__ __forceinline__ void start(const DecodeArgs& a, int warp, int it, int li0) {
    pos.start(a, it, li0);
    set(warp);
  }
  __device__ __forceinline__ int rb() const { return rb0 + grp * RPW; }
  __device__ __forceinline__ bool valid() const { return rb() < n_rb; }
  __device__ __forceinline__ void normalize(const DecodeArgs& a, int warp, int end) {
    while (item < end && !valid()) {
      pos.next(a);
      if (pos.item < end) set(warp);
      else item = pos.item;
    }
  }
  __device__ __forceinline__ void advance(const DecodeArgs& a, int warp, int end) {
    if (++kc * kChunkTiles >= nkt) {
      kc = 0;
      if (++grp * RPW >= kRW) {
        pos.next(a);
        if (pos.item < end) set(warp);
        else item = pos.item;
      }
    }
    normalize(a, warp, end);
  }
  // issue this chunk: up to RPW row blocks x ntile K-tiles into `stage`
  __device__ __forceinline__ void issue(unsigned char* stage, uint64_t* bar) const {
    const int ntile = min(kChunkTiles, nkt - kc * kChunkTiles);
    const uint32_t bytes = (uint32_t)ntile * kTileBytes;
    int nrb = 0;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
      if (rb() + r < n_rb) ++nrb;
    mbar_expect_tx(bar, bytes * nrb);
#pragma unroll
    for (int r = 0; r < RPW; ++r)
      if (rb() + r < n_rb)
        bulk_g2s(stage + r * kChunkBytes,
                 V + ((size_t)(rb() + r) * n_kt_all + kt0 + kc * kChunkTiles) * kTileBytes, bytes, bar);
  }
};

template <int NB, int RB, int W>
__global__ void __launch_bounds__(W * 32, NB == 1 ? 3 : 1) latent_pass_kernel(const DecodeArgs a) {
  constexpr int NC = 2 * RB;                      // B-fragment columns stored per K-block
  constexpr int RPW = VCfg<NB>::kRPW;
  constexpr int kRW = latent_rows_per_warp(W);    // row blocks of an item per warp
  constexpr int kStageBytes = RPW * kChunkBytes;
  constexpr int kXBuf = xq_buf_bytes(NB, RB);
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* ring = smem;                                        // [warps][stages][RPW x 2 KB]
  unsigned char* xbuf = smem + W * kVStages * kStageBytes;           // [2][kXBuf]
  uint64_t* mbar = reinterpret_cast<uint64_t*>(xbuf + 2 * kXBuf);    // [warps][stages]
  uint64_t* xfull = mbar + W * kVStages;                             // [2]
  __shared__ int s_done[2];   // warps done with each buffer, accumulated over its uses

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int B = a.batch;
  const int i_begin = (int)((long long)a.v_items * blockIdx.x / gridDim.x);
  const int i_end = (int)((long long)a.v_items * (blockIdx.x + 1) / gridDim.x);
  if (i_begin >= i_end) return;   // uniform over the CTA

  unsigned char* my_ring = ring + (size_t)warp * kVStages * kStageBytes;
  uint64_t* my_bar = mbar + warp * kVStages;
  if (lane == 0) {
    for (int st = 0; st < kVStages; ++st) mbar_init(&my_bar[st], 1);
  }
  if (tid == 0) {
    mbar_init(&xfull[0], 1);
    mbar_init(&xfull[1], 1);
    s_done[0] = s_done[1] = 0;
  }
  if (lane == 0) fence_mbar_init();
  __syncthreads();   // the only CTA barrier: barriers and counters initialised

  grid_dep_launch();
  const int li0 = layer_of(a.item_layer.v, a.n_layers, i_begin);
  VFeed<NB, W> feed;
  feed.start(a, warp, i_begin, li0);
  feed.normalize(a, warp, i_end);
#pragma unroll 1
  for (int st = 0; st < kVStages; ++st) {
    if (feed.item < i_end) {
      if (lane == 0) feed.issue(my_ring + st * kStageBytes, &my_bar[st]);
      feed.advance(a, warp, i_end);
    }
  }
  // the sign tiles above are weights; the quantised slices are the quantise
  // pass's output
  grid_dep_wait();
  if (tid == 0) {
    // slices 0 and 1 of this CTA's sequence
    int lj = li0;
    const VItem it = decode_v(a, i_begin, lj);
    x_issue<NB, RB>(a, i_begin, li0, xbuf, &xfull[0]);
    const int nxt = i_begin - it.rc + a.layers[it.li].n_rchunks;
    if (nxt < i_end) x_issue<NB, RB>(a, nxt, it.li, xbuf + kXBuf, &xfull[1]);
  }
  uint32_t consumed = 0;
  int slot = 0;
  bool dead = false;

  // this thread's B column in K-block 0 (uint2 units): column (8nb + g) mod NC
  int boff[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) boff[nb] = ((8 * nb + g) % NC) * 4 + c;

  int prev_li = -1, prev_p = -1, prev_sl = -1;
  int seq = -1;   // index of the current slice in this CTA's sequence

  VPos cur;
  cur.start(a, i_begin, li0);
  for (; cur.item < i_end; cur.next(a)) {
    const int item = cur.item, li = cur.li;
    const VItem it{cur.li, cur.p, cur.sl, cur.rc};
    const LayerDesc& L = *cur.L;
    const PathDesc& P = L.p[it.p];
    const int s = L.s;
    const int S16 = (s + 15) & ~15, n_rb = S16 >> 4;
    const int nkt = min(kVSlice, L.d_in - it.sl * kVSlice) / kVTileK;

    if (it.li != prev_li || it.p != prev_p || it.sl != prev_sl) {
      ++seq;
      if (seq > 0) {
        // done with slice seq - 1: the last warp out refills its buffer with slice seq + 1
        __syncwarp();
        if (lane == 0) {
          const int b = (seq - 1) & 1;
          __threadfence_block();
          const int old = atomicAdd(&s_done[b], 1);
          if (old == W * (((seq - 1) >> 1) + 1) - 1) {
            __threadfence_block();
            const int nxt = item - it.rc + L.n_rchunks;   // first item of the following slice
            if (nxt < i_end) x_issue<NB, RB>(a, nxt, li, xbuf + b * kXBuf, &xfull[b]);
          }
        }
      }
      if (!dead && !mbar_wait(&xfull[seq & 1], (seq >> 1) & 1)) {
        dead = true;
        atomicOr(a.status, 1u << LB_ERR_TIMEOUT);
      }
      prev_li = it.li;
      prev_p = it.p;
      prev_sl = it.sl;
    }
    const unsigned char* xb = xbuf + (seq & 1) * kXBuf;
    const uint2* frag = reinterpret_cast<const uint2*>(xb + 64 * NB);
    const TStat* xst = reinterpret_cast<const TStat*>(xb);

    // ---- this warp's row blocks over the slice, RPW at once.  A block past the
    //      last one (odd count) still runs its products on whatever its stage
    //      half holds, so that the product loop has no branches; its sums are
    //      not written.
    const int ns4 = (L.n_slices + 3) & ~3;
    float* part = P.ws.partial + it.sl;
#pragma unroll 1
    for (int grp = 0; grp * RPW < kRW; ++grp) {
      const int rbA = it.rc * (W * kRW) + kRW * warp + grp * RPW;
      if (rbA >= n_rb) break;
      const int nvalid = min(RPW, n_rb - rbA);
      constexpr int R = RPW;
      int d[R][8][NB][4];
#pragma unroll 1
      for (int kc = 0; kc * kChunkTiles < nkt; ++kc) {
        if (!dead && !mbar_wait(&my_bar[slot], (consumed / kVStages) & 1)) {
          dead = true;
          atomicOr(a.status, 1u << LB_ERR_TIMEOUT);
        }
        const unsigned char* stage = my_ring + slot * kStageBytes + lane * 16;
        const uint2* fc = frag + (size_t)kc * kChunkTiles * 8 * NC * 4;
        const int ntile = min(kChunkTiles, nkt - kc * kChunkTiles);
        // one K-tile of the chunk for the R row blocks
        auto ktile = [&](int t, bool first) {
          uint4 cur[R];
#pragma unroll
          for (int r = 0; r < R; ++r)
            cur[r] = *reinterpret_cast<const uint4*>(stage + r * kChunkBytes + t * kTileBytes);
          const uint2* fk = fc + t * 8 * NC * 4;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t m = 0x01010101u << q;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              const uint2 bb = fk[q * NC * 4 + boff[nb]];
#pragma unroll
              for (int r = 0; r < R; ++r) {
                const uint32_t a0 = cur[r].x & m, a1 = cur[r].y & m, a2 = cur[r].z & m, a3 = cur[r].w & m;
                if (first) mma_u8s8_zc(d[r][q][nb], a0, a1, a2, a3, bb.x, bb.y);
                else mma_u8s8(d[r][q][nb], a0, a1, a2, a3, bb.x, bb.y);
              }
            }
          }
        };
        if (kc == 0) ktile(0, true); else ktile(0, false);
        if (ntile == kChunkTiles) {
#pragma unroll
          for (int t = 1; t < kChunkTiles; ++t) ktile(t, false);
        } else {
#pragma unroll 1
          for (int t = 1; t < ntile; ++t) ktile(t, false);
        }
        // the stage has been read: refill it
        __syncwarp();
        if (feed.item < i_end) {
          if (lane == 0) feed.issue(my_ring + slot * kStageBytes, &my_bar[slot]);
          feed.advance(a, warp, i_end);
        }
        ++consumed;
        if (++slot == kVStages) slot = 0;
      }
      // fold: sum_q D_q / 2^q per plane = 2^-7 * sum_q D_q * 2^(7-q) (each term a
      // multiple of 2^7), then 256*hi + lo; slice partial = step*(sum v - 2*that)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r >= nvalid) break;
        const int row = 16 * (rbA + r) + g;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          int h0 = d[r][0][nb][0], l0 = d[r][0][nb][1], h1 = d[r][0][nb][2], l1 = d[r][0][nb][3];
#pragma unroll
          for (int q = 1; q < 8; ++q) {
            h0 = 2 * h0 + d[r][q][nb][0];
            l0 = 2 * l0 + d[r][q][nb][1];
            h1 = 2 * h1 + d[r][q][nb][2];
            l1 = 2 * l1 + d[r][q][nb][3];
          }
          const int b = 4 * nb + c;
          if (b < B) {
            const float st = xst[b].step;
            const int vsum = xst[b].sum;
            part[((size_t)b * S16 + row) * ns4] = st * (float)(vsum - 2 * (2 * h0 + (l0 >> 7)));
            part[((size_t)b * S16 + row + 8) * ns4] = st * (float)(vsum - 2 * (2 * h1 + (l1 >> 7)));
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// finalize:  t'_j = l_j * sum over slices of the partials, quantised per batch
// row to the int8 hi/lo planes and the step the output pass reads.  In a
// packed call (batch 1 with a residual layer) the planes of a layer's paths
// form one K range (packed output pass): path
// p's K-tiles come after path p-1's, with its t' in row p of each tile and
// zeros in the other path's row.  One CTA
// per (layer, path), in a launch between the two passes: warp w takes the
// 32-row groups k = w, w+4, ...; the max and the sum over the path are combined
// with integer atomics in shared memory (order-independent, so deterministic).
// Plane bytes of rows >= batch are not written: the output pass's product
// columns for them are independent of the batch rows' and their sums are
// discarded.
// ---------------------------------------------------------------------------
constexpr int kFWarps = 4;

template <int NB>
__global__ void __launch_bounds__(kFWarps * 32) finalize_kernel(const DecodeArgs a) {
  __shared__ float s_t[kMaxRank];   // t' of this path, one batch row at a time
  __shared__ unsigned s_mx;         // max |t'| (non-negative float bits order as unsigned)
  __shared__ int s_sum;
  grid_dep_launch();
  grid_dep_wait();   // the latent pass's partials
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int item = blockIdx.x;
  const int B = a.batch;
  const LayerDesc& L = a.layers[layer_of(a.item_layer.p, a.n_layers, item)];
  const int pi = item - L.p_begin;
  const PathDesc& P = L.p[pi];
  const int s = L.s, S16 = (s + 15) & ~15, nkt = (s + 31) >> 5;
  const int ns = L.n_slices, ng = (ns + 3) >> 2;
  const bool packed = a.packed != 0;   // the output pass takes both paths as one K range
  const int mode = a.mode;
#pragma unroll 1
  for (int b = 0; b < B; ++b) {
    if (tid == 0) {
      s_mx = 0u;
      s_sum = 0;
    }
    __syncthreads();
    float mx = 0.f;
#pragma unroll 2
    for (int k = warp; k < nkt; k += kFWarps) {
      const int j = lane + 32 * k;
      float v;
      if (mode == kModeExpand) {
        // t' from the caller's cache row (l already applied)
        v = j < s ? h2f(L.x[(size_t)b * L.t_ld + pi * s + j]) : 0.f;
      } else {
        // a latent row's slice partials are contiguous float4s, summed in slice order
        const int jc = min(j, S16 - 1);   // rows past S16 clamp (finite; zeroed below)
        const float4* pp = reinterpret_cast<const float4*>(P.ws.partial) + ((size_t)b * S16 + jc) * ng;
        float t = 0.f;
#pragma unroll 4
        for (int q4 = 0; q4 < ng; ++q4) {
          const float4 f = pp[q4];
          const int q = 4 * q4;
          t += f.x;
          if (q + 1 < ns) t += f.y;
          if (q + 2 < ns) t += f.z;
          if (q + 3 < ns) t += f.w;
        }
        const float l = h2f(P.l[min(j, s - 1)]);
        v = j < s ? t * l : 0.f;
        if (mode == kModeLatent && j < s) L.y[(size_t)b * L.t_ld + pi * s + j] = f2h(v);
      }
      s_t[j] = v;
      mx = fmaxf(mx, fabsf(v));
    }
    if (mode == kModeLatent) continue;   // the cache row is the result (mode is uniform over the CTA)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) atomicMax(&s_mx, __float_as_uint(mx));
    __syncthreads();
    mx = __uint_as_float(s_mx);
    const float inv = mx > 0.f ? kQMax / mx : 0.f;
    int vsum = 0;
#pragma unroll 2
    for (int k = warp; k < nkt; k += kFWarps) {
      // v = round(t' * inv) in the low bits of the float's encoding (see the
      // quantise pass); lo = its low byte, hi = byte 1 of v + 128
      const uint32_t fb = __float_as_uint(fmaf(s_t[lane + 32 * k], inv, kRoundMagic));
      vsum += (int)(fb - 0x4B400000u);
      if (packed) {
        // K-tile pi*nkt + k of the layer's combined planes: row pi holds this
        // path's t', the other path's row is zero
        int8_t* pl = L.p[0].ws.planes + ((size_t)(pi * nkt + k) * 4 * 2) * 32 + lane;
        pl[pi * 64] = (int8_t)((fb + 128u) >> 8);
        pl[pi * 64 + 32] = (int8_t)fb;
        if (L.npaths == 2) {
          pl[(1 - pi) * 64] = 0;
          pl[(1 - pi) * 64 + 32] = 0;
        }
      } else {
        // RS rows per K-tile: 1 at batch 1 (only row 0 is read), else 4*NB
        const int RS = B == 1 ? 1 : 4 * NB;
        int8_t* pl = P.ws.planes + ((size_t)(k * RS + b) * 2) * 32 + lane;
        pl[0] = (int8_t)((fb + 128u) >> 8);
        pl[32] = (int8_t)fb;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vsum += __shfl_xor_sync(0xffffffffu, vsum, o);
    if (lane == 0) atomicAdd(&s_sum, vsum);
    __syncthreads();
    if (tid == 0) {
      TStat st;
      st.step = mx > 0.f ? mx / kQMax : 0.f;
      st.sum = s_sum;
      st.pad[0] = st.pad[1] = 0;
      P.ws.tstat[b] = st;
    }
    __syncthreads();   // s_mx, s_sum and s_t are reset for the next batch row
  }
}

// ---------------------------------------------------------------------------
// output pass:  y_o = sum_p h_p[o] * sum_j U_p[o][j] t'_p[j]
// ---------------------------------------------------------------------------

constexpr int kUChunkTiles = 8;                           // K-tiles per bulk copy
constexpr int kUChunkBytes = kUChunkTiles * kTileBytes;   // 4 KB

template <int NB>
struct OutCfg {
  static constexpr int kStages = 2;
};

// stage: [8 tiles: 4 KB][t' bytes: 8 K-tiles x RS x 64][h: 256][tstat: 16 B x RS]
// (B below is RS, the batch rows stored per K-tile of the t' planes: 1 at
// batch 1, else 4*NB; at batch 1 the product's columns for rows 1..3 are
// never read, so their zero planes are not stored or copied)
__host__ __device__ __forceinline__ int out_planes_off() { return kUChunkBytes; }
__host__ __device__ __forceinline__ int out_h_off(int B) { return kUChunkBytes + kUChunkTiles * B * 64; }
__host__ __device__ __forceinline__ int out_tstat_off(int B) { return out_h_off(B) + kUTileRows * 2; }
__host__ __device__ __forceinline__ int out_stage_bytes(int B) {
  return (out_tstat_off(B) + 16 * B + 127) & ~127;
}

// Position in a warp's stream of output-pass chunks (up to 8 K-tiles of one
// (item, path)), with the current layer's fields and the path's base
// pointers cached so that issuing a chunk needs no descriptor loads.
struct OutCursor {
  int li, item, p, kt0;
  int n_kt, npaths, u_begin, u_end;
  const unsigned char* U;   // path p's tiles
  const int8_t* planes;     // path p's t' bytes
  const uint16_t* h;
  const TStat* tstat;

  __device__ __forceinline__ void set_path(const DecodeArgs& a) {
    const PathDesc& P = a.layers[li].p[p];
    U = reinterpret_cast<const unsigned char*>(P.U);
    planes = P.ws.planes;
    h = P.h;
    tstat = P.ws.tstat;
  }
  __device__ __forceinline__ void enter(const DecodeArgs& a, int l) {
    li = l;
    const LayerDesc& L = a.layers[l];
    n_kt = (L.s + 31) >> 5;
    npaths = L.npaths;
    u_begin = L.u_begin;
    u_end = (l + 1 < a.n_layers) ? a.layers[l + 1].u_begin : a.u_items;
  }
  __device__ __forceinline__ int ntile() const { return min(kUChunkTiles, n_kt - kt0); }
  __device__ __forceinline__ bool path_end() const { return kt0 + kUChunkTiles >= n_kt; }
  __device__ __forceinline__ void advance(const DecodeArgs& a) {
    kt0 += kUChunkTiles;
    if (kt0 >= n_kt) {
      kt0 = 0;
      if (++p == npaths) {
        p = 0;
        if (++item == u_end && item < a.u_items) enter(a, li + 1);
      }
      set_path(a);
    }
  }
};

__device__ __forceinline__ void out_issue(const OutCursor& cu, unsigned char* stage, uint64_t* bar, int B) {
  const int ob = cu.item - cu.u_begin;
  const int nt = cu.ntile();
  const uint32_t tb = (uint32_t)nt * kTileBytes, pb = (uint32_t)nt * B * 64;
  const bool last = cu.path_end();
  mbar_expect_tx(bar, tb + pb + (last ? kUTileRows * 2 + 16 * B : 0));
  bulk_g2s(stage, cu.U + ((size_t)ob * cu.n_kt + cu.kt0) * kTileBytes, tb, bar);
  bulk_g2s(stage + out_planes_off(), cu.planes + (size_t)cu.kt0 * B * 64, pb, bar);
  if (last) {
    bulk_g2s(stage + out_h_off(B), cu.h + (size_t)ob * kUTileRows, kUTileRows * 2, bar);
    bulk_g2s(stage + out_tstat_off(B), cu.tstat, 16 * B, bar);
  }
}

// One K-tile of one path: eight m16n8k32 products (row block q = 0..7).
// `pl` points at this thread's t' bytes of tile 0 (batch row 4nb + g/2,
// plane g%2); RS * 64 bytes separate one tile's t' bytes from the next.
template <int NB, int RS, bool kFirst = false>
__device__ __forceinline__ void out_tile(int (&d)[8][NB][4], const unsigned char* stage, int t, int lane,
                                         const unsigned char* pl) {
  const uint4 cur = *reinterpret_cast<const uint4*>(stage + t * kTileBytes + lane * 16);
  uint32_t b0[NB], b1[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    b0[nb] = *reinterpret_cast<const uint32_t*>(pl + t * (64 * RS) + nb * 256);
    b1[nb] = *reinterpret_cast<const uint32_t*>(pl + t * (64 * RS) + nb * 256 + 16);
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t m = 0x01010101u << q;
    const uint32_t a0 = cur.x & m, a1 = cur.y & m, a2 = cur.z & m, a3 = cur.w & m;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      if (kFirst) mma_u8s8_zc(d[q][nb], a0, a1, a2, a3, b0[nb], b1[nb]);   // a path's first K-tile
      else mma_u8s8(d[q][nb], a0, a1, a2, a3, b0[nb], b1[nb]);
    }
  }
}

template <int NB, int RS>
__global__ void __launch_bounds__(kUWarps * 32) output_pass_kernel(const DecodeArgs a) {
  static_assert(RS == 4 * NB || (NB == 1 && RS == 1), "t' rows stored: 1 at batch 1, else 4 per n-block");
  constexpr int S = OutCfg<NB>::kStages;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int B = a.batch;            // rows stored
  constexpr int BP = RS;            // rows in the t' planes and stats
  const int sb = out_stage_bytes(BP);
  unsigned char* my_ring = smem + (size_t)warp * S * sb;
  uint64_t* my_bar = reinterpret_cast<uint64_t*>(smem + (size_t)kUWarps * S * sb) + warp * S;

  const long long W = (long long)gridDim.x * kUWarps, gw = (long long)blockIdx.x * kUWarps + warp;
  const int i_begin = (int)(a.u_items * gw / W), i_end = (int)(a.u_items * (gw + 1) / W);
  if (i_begin >= i_end) return;   // no CTA-wide barriers in this kernel

  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init(&my_bar[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  grid_dep_wait();   // finalize's t' planes and steps

  OutCursor fd;
  fd.enter(a, layer_of(a.item_layer.u, a.n_layers, i_begin));
  fd.item = i_begin;
  fd.p = 0;
  fd.kt0 = 0;
  fd.set_path(a);
  OutCursor cs = fd;
#pragma unroll 1
  for (int st = 0; st < S; ++st) {
    if (fd.item < i_end) {
      if (lane == 0) out_issue(fd, my_ring + st * sb, &my_bar[st], BP);
      fd.advance(a);
    }
  }

  // d starts at a path's first K-tile (zero-accumulator product); yacc at its
  // first path (assigned, not added)
  float yacc[8][2][NB];
  int d[8][NB][4];
  uint32_t consumed = 0;
  int slot = 0;
  bool dead = false;
  // this thread's B-operand column: batch row 4nb + g/2, plane g%2 (at batch
  // 1, columns of rows 1..3 read row 0's bytes; their sums are not used)
  const int pl_off = out_planes_off() + (RS == 1 ? (g & 1) : g) * 32 + 4 * c;

  while (cs.item < i_end) {
    if (!dead && !mbar_wait(&my_bar[slot], (consumed / S) & 1)) {
      dead = true;
      atomicOr(a.status, 1u << LB_ERR_TIMEOUT);
    }
    const unsigned char* stage = my_ring + slot * sb;
    const int nt = cs.ntile();
    const unsigned char* pl = stage + pl_off;
    if (cs.kt0 == 0) out_tile<NB, RS, true>(d, stage, 0, lane, pl);
    else out_tile<NB, RS>(d, stage, 0, lane, pl);
    if (nt == kUChunkTiles) {
#pragma unroll
      for (int t = 1; t < kUChunkTiles; ++t) out_tile<NB, RS>(d, stage, t, lane, pl);
    } else {
#pragma unroll 1
      for (int t = 1; t < nt; ++t) out_tile<NB, RS>(d, stage, t, lane, pl);
    }
    if (cs.path_end()) {
      // path finished: rows 128*ob + 16q + g (+8), batch row 4nb + c
      const uint16_t* hs = reinterpret_cast<const uint16_t*>(stage + out_h_off(BP));
      const TStat* tst = reinterpret_cast<const TStat*>(stage + out_tstat_off(BP));
      const bool first_path = cs.p == 0;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int b = 4 * nb + c;
        if (b < B) {
          const float st = tst[b].step;
          const float base = st * (float)tst[b].sum;
          const float m2 = -2.f * st;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int c0 = ((d[q][nb][0] >> q) << 8) + (d[q][nb][1] >> q);
            const int c1 = ((d[q][nb][2] >> q) << 8) + (d[q][nb][3] >> q);
            const float y0 = first_path ? 0.f : yacc[q][0][nb], y1 = first_path ? 0.f : yacc[q][1][nb];
            yacc[q][0][nb] = fmaf(h2f(hs[16 * q + g]), fmaf(m2, (float)c0, base), y0);
            yacc[q][1][nb] = fmaf(h2f(hs[16 * q + g + 8]), fmaf(m2, (float)c1, base), y1);
          }
        }
      }
      if (cs.p == cs.npaths - 1) {
        const LayerDesc& L = a.layers[cs.li];
        const int ob = cs.item - cs.u_begin;
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
    // the stage has been read: refill it with the chunk `S` ahead
    __syncwarp();
    if (fd.item < i_end) {
      if (lane == 0) out_issue(fd, my_ring + slot * sb, &my_bar[slot], BP);
      fd.advance(a);
    }
    ++consumed;
    if (++slot == S) slot = 0;
    cs.advance(a);
  }
}

// ---------------------------------------------------------------------------
// output pass with a producer warp ("fed"): the same products and epilogue as
// output_pass_kernel, but the bulk copies are issued by a ninth warp, so that
// the eight consumer warps only wait, compute and release.  Lane w < 8 of the
// producer warp runs consumer w's stream: its items are the CTA's items
// w, w + 8, ..., each cut into chunks of up to 8 K-tiles per path; it writes
// a 16-byte header into the stage (output pointer, tile count, flags) before
// the stage's copies, and a final header that ends the stream.  A consumer
// has kFedSlots stages; the lane refills a stage once its consumer has
// released it (polled with test_wait, so a lane whose consumer is behind
// does not hold up the others).
// ---------------------------------------------------------------------------
constexpr int kFedCons = 8;     // consumer warps per CTA
constexpr int kFedSlots = 2;    // stages per consumer warp

// stage: the per-warp pass's stage layout (out_*_off(RS)), then the header
__host__ __device__ __forceinline__ int fed_hdr_off(int RS) { return out_tstat_off(RS) + 16 * RS; }
__host__ __device__ __forceinline__ int fed_stage_bytes(int RS) { return (fed_hdr_off(RS) + 16 + 127) & ~127; }
__host__ __device__ __forceinline__ size_t fed_smem(int RS) {
  return (size_t)kFedCons * kFedSlots * fed_stage_bytes(RS) + (size_t)2 * kFedCons * kFedSlots * 8;
}

// header flags
constexpr uint32_t kFedFirstTile = 1;   // the chunk starts a path: zero the accumulators
constexpr uint32_t kFedPathEnd = 2;     // the chunk ends a path: scale it into the output
constexpr uint32_t kFedFirstPath = 4;   // that path is the item's first (assign, not add)
constexpr uint32_t kFedItemEnd = 8;     // store the item's 128 outputs
constexpr uint32_t kFedEnd = 16;        // no more chunks for this consumer

// A producer lane's position: item, path, first K-tile, and what it needs
// to issue the chunk without further descriptor loads.
struct FedCursor {
  int item, p, kt0, n_kt, npaths, ob;
  const LayerDesc* L;
  const unsigned char* U;
  const int8_t* planes;
  const uint16_t* h;
  const TStat* tstat;

  __device__ __forceinline__ void set_path() {
    const PathDesc& P = L->p[p];
    U = reinterpret_cast<const unsigned char*>(P.U);
    planes = P.ws.planes;
    h = P.h;
    tstat = P.ws.tstat;
  }
  __device__ __forceinline__ void enter(const DecodeArgs& a, int it) {
    item = it;
    L = a.layers + layer_of(a.item_layer.u, a.n_layers, it);
    n_kt = (L->s + 31) >> 5;
    npaths = L->npaths;
    ob = it - L->u_begin;
    p = 0;
    kt0 = 0;
    set_path();
  }
};

template <int NB, int RS>
__global__ void __launch_bounds__((kFedCons + 1) * 32, NB == 1 ? 2 : 1) output_fed_kernel(const DecodeArgs a) {
  static_assert(RS == 4 * NB || (NB == 1 && RS == 1), "t' rows stored: 1 at batch 1, else 4 per n-block");
  extern __shared__ __align__(1024) unsigned char smem[];
  const int sb = fed_stage_bytes(RS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kFedCons * kFedSlots * sb);
  uint64_t* empty = full + kFedCons * kFedSlots;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int i_begin = (int)((long long)a.u_items * blockIdx.x / gridDim.x);
  const int i_end = (int)((long long)a.u_items * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kFedCons * kFedSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();   // the only CTA barrier

  if (warp == kFedCons) {
    // ---- producer: lane w feeds consumer w.  The first kFedSlots chunks'
    //      sign tiles and h (weights) are issued before the wait for
    //      finalize; their t' bytes and step records after it.
    if (lane >= kFedCons) return;
    FedCursor cu;
    if (i_begin + lane < i_end) cu.enter(a, i_begin + lane);
    else cu.item = i_end;
    struct TCopy {
      unsigned char* stage;
      const int8_t* planes;
      const TStat* tstat;
      uint32_t pb;
      bool path_end;
      uint64_t* bar;
    };
    auto issue = [&](int s, TCopy& tc) -> bool {
      unsigned char* stage = smem + (size_t)s * sb;
      uint4* hdr = reinterpret_cast<uint4*>(stage + fed_hdr_off(RS));
      if (cu.item >= i_end) {
        *hdr = make_uint4(0u, 0u, kFedEnd << 8, 0u);
        mbar_arrive_one(&full[s]);
        tc.pb = 0;
        return true;
      }
      const int nt = min(kUChunkTiles, cu.n_kt - cu.kt0);
      const bool path_end = cu.kt0 + kUChunkTiles >= cu.n_kt;
      const uint32_t flags = (cu.kt0 == 0 ? kFedFirstTile : 0u) | (path_end ? kFedPathEnd : 0u) |
                             (cu.p == 0 ? kFedFirstPath : 0u) |
                             (path_end && cu.p == cu.npaths - 1 ? kFedItemEnd : 0u);
      const unsigned long long y = reinterpret_cast<unsigned long long>(cu.L->y + (size_t)cu.ob * kUTileRows);
      *hdr = make_uint4((uint32_t)y, (uint32_t)(y >> 32), (uint32_t)nt | (flags << 8), (uint32_t)cu.L->d_out);
      const uint32_t tb = (uint32_t)nt * kTileBytes, pb = (uint32_t)nt * RS * 64;
      mbar_expect_tx(&full[s], tb + pb + (path_end ? kUTileRows * 2 + 16 * RS : 0));
      bulk_g2s(stage, cu.U + ((size_t)cu.ob * cu.n_kt + cu.kt0) * kTileBytes, tb, &full[s]);
      if (path_end) bulk_g2s(stage + out_h_off(RS), cu.h + (size_t)cu.ob * kUTileRows, kUTileRows * 2, &full[s]);
      tc.stage = stage;
      tc.planes = cu.planes + (size_t)cu.kt0 * RS * 64;
      tc.tstat = cu.tstat;
      tc.pb = pb;
      tc.path_end = path_end;
      tc.bar = &full[s];
      // next chunk of this consumer's stream
      cu.kt0 += kUChunkTiles;
      if (cu.kt0 >= cu.n_kt) {
        cu.kt0 = 0;
        if (++cu.p == cu.npaths) {
          if (cu.item + kFedCons < i_end) cu.enter(a, cu.item + kFedCons);
          else cu.item = i_end;
        } else {
          cu.set_path();
        }
      }
      return false;
    };
    auto issue_t = [&](const TCopy& tc) {
      if (!tc.pb) return;
      bulk_g2s(tc.stage + out_planes_off(), tc.planes, tc.pb, tc.bar);
      if (tc.path_end) bulk_g2s(tc.stage + out_tstat_off(RS), tc.tstat, 16 * RS, tc.bar);
    };
    bool done = false, dead = false;
    uint32_t n = 0, idle = 0;
    TCopy pre[kFedSlots];
    for (int k = 0; k < kFedSlots; ++k) pre[k].pb = 0;
    for (; n < (uint32_t)kFedSlots && !done; ++n) done = issue(lane * kFedSlots + (int)n, pre[n]);
    grid_dep_wait();   // finalize's t' planes and steps
    for (int k = 0; k < kFedSlots; ++k) issue_t(pre[k]);
    while (!done) {
      const int s = lane * kFedSlots + (int)(n % kFedSlots);
      if (!mbar_test_wait(&empty[s], ((n / kFedSlots) - 1) & 1)) {
        if (++idle > (uint32_t)kSpinLimit) {   // the consumer stopped releasing stages
          dead = true;
          break;
        }
        __nanosleep(64);
        continue;
      }
      idle = 0;
      TCopy tc;
      done = issue(s, tc);
      issue_t(tc);
      ++n;
    }
    if (dead) atomicOr(a.status, kStatusTimeout);
    return;
  }

  // ---- consumer warp
  const int B = a.batch;
  float yacc[8][2][NB];
  int d[8][NB][4];
  bool dead = false;
  const int pl_off = out_planes_off() + (RS == 1 ? (g & 1) : g) * 32 + 4 * c;
#pragma unroll 1
  for (uint32_t n = 0;; ++n) {
    const int s = warp * kFedSlots + (int)(n % kFedSlots);
    if (!mbar_wait(&full[s], (n / kFedSlots) & 1)) {
      dead = true;
      break;
    }
    const unsigned char* stage = smem + (size_t)s * sb;
    const uint4 hdr = *reinterpret_cast<const uint4*>(stage + fed_hdr_off(RS));
    const uint32_t flags = hdr.z >> 8;
    if (flags & kFedEnd) break;
    const int nt = (int)(hdr.z & 0xff);
    const unsigned char* pl = stage + pl_off;
    if (flags & kFedFirstTile) out_tile<NB, RS, true>(d, stage, 0, lane, pl);
    else out_tile<NB, RS>(d, stage, 0, lane, pl);
    if (nt == kUChunkTiles) {
#pragma unroll
      for (int t = 1; t < kUChunkTiles; ++t) out_tile<NB, RS>(d, stage, t, lane, pl);
    } else {
#pragma unroll 1
      for (int t = 1; t < nt; ++t) out_tile<NB, RS>(d, stage, t, lane, pl);
    }
    if (flags & kFedPathEnd) {
      // rows 16q + g (+8) of the item, batch row 4nb + c
      const uint16_t* hs = reinterpret_cast<const uint16_t*>(stage + out_h_off(RS));
      const TStat* tst = reinterpret_cast<const TStat*>(stage + out_tstat_off(RS));
      const bool first_path = (flags & kFedFirstPath) != 0;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int b = 4 * nb + c;
        if (b < B) {
          const float st = tst[b].step;
          const float base = st * (float)tst[b].sum;
          const float m2 = -2.f * st;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int c0 = ((d[q][nb][0] >> q) << 8) + (d[q][nb][1] >> q);
            const int c1 = ((d[q][nb][2] >> q) << 8) + (d[q][nb][3] >> q);
            const float y0 = first_path ? 0.f : yacc[q][0][nb], y1 = first_path ? 0.f : yacc[q][1][nb];
            yacc[q][0][nb] = fmaf(h2f(hs[16 * q + g]), fmaf(m2, (float)c0, base), y0);
            yacc[q][1][nb] = fmaf(h2f(hs[16 * q + g + 8]), fmaf(m2, (float)c1, base), y1);
          }
        }
      }
      if (flags & kFedItemEnd) {
        uint16_t* y = reinterpret_cast<uint16_t*>((unsigned long long)hdr.x | ((unsigned long long)hdr.y << 32));
        const int d_out = (int)hdr.w;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const int b = 4 * nb + c;
          if (b < B) {
            uint16_t* yr = y + (size_t)b * d_out + g;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              yr[16 * q] = f2h(yacc[q][0][nb]);
              yr[16 * q + 8] = f2h(yacc[q][1][nb]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_one(&empty[s]);
  }
  if (dead && lane == 0) atomicOr(a.status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// output pass, batch 1 with residual layers ("packed"): the product's 8
// columns hold 4 batch rows, of which batch 1 uses one, so the paths take the
// spare ones instead.  Both
// paths' K-tiles form one K range (path 1's after path 0's); the t' operand
// of path p's tiles sits in column pair p with zeros in the other path's pair,
// so one accumulator holds both paths' sums, in different columns.  Lanes with
// c = 0 and c = 1 scale their path's rows (h_p, step_p) and one shuffle adds
// the paths.  One chunk carries up to 8 K-tiles of the range, so a small-rank
// residual layer's 128-row item is one chunk and one epilogue.
// ---------------------------------------------------------------------------
// stage: [8 tiles: 4 KB][t' bytes: 8 x 256][h of path 0, 1: 2 x 256][TStat of path 0, 1]
constexpr int kPkPlanesOff = kUChunkBytes;
constexpr int kPkHOff = kPkPlanesOff + kUChunkTiles * 256;
constexpr int kPkTsOff = kPkHOff + 2 * kUTileRows * 2;
constexpr int kPkStageBytes = (kPkTsOff + 2 * 16 + 127) & ~127;
constexpr int kPkStages = 2;

struct PkCursor {
  int li, item, kv0;                 // item, first K-tile of the chunk in the packed range
  int n_kt, npaths, u_begin, u_end;
  const unsigned char *U0, *U1;      // path 1 = path 0 for a single-path layer
  const int8_t* planes;              // the layer's combined t' bytes
  const uint16_t *h0, *h1;
  const TStat *ts0, *ts1;

  __device__ __forceinline__ void enter(const DecodeArgs& a, int l) {
    li = l;
    const LayerDesc& L = a.layers[l];
    n_kt = (L.s + 31) >> 5;
    npaths = L.npaths;
    u_begin = L.u_begin;
    u_end = (l + 1 < a.n_layers) ? a.layers[l + 1].u_begin : a.u_items;
    const PathDesc& P0 = L.p[0];
    const PathDesc& P1 = L.p[npaths - 1];
    U0 = reinterpret_cast<const unsigned char*>(P0.U);
    U1 = reinterpret_cast<const unsigned char*>(P1.U);
    h0 = P0.h;
    h1 = P1.h;
    ts0 = P0.ws.tstat;
    ts1 = P1.ws.tstat;
    planes = P0.ws.planes;
  }
  __device__ __forceinline__ int n_kv() const { return npaths * n_kt; }
  __device__ __forceinline__ int ntile() const { return min(kUChunkTiles, n_kv() - kv0); }
  __device__ __forceinline__ bool item_end() const { return kv0 + kUChunkTiles >= n_kv(); }
  __device__ __forceinline__ void advance(const DecodeArgs& a) {
    kv0 += kUChunkTiles;
    if (kv0 >= n_kv()) {
      kv0 = 0;
      if (++item == u_end && item < a.u_items) enter(a, li + 1);
    }
  }
};

__device__ __forceinline__ void pk_issue(const PkCursor& cu, unsigned char* stage, uint64_t* bar) {
  const int ob = cu.item - cu.u_begin;
  const int nt = cu.ntile();
  const int t0 = max(0, min(nt, cu.n_kt - cu.kv0));   // tiles of path 0 in this chunk
  const int t1 = nt - t0;                              // tiles of path 1
  const bool last = cu.item_end();
  mbar_expect_tx(bar, (uint32_t)nt * (kTileBytes + 256) + (last ? cu.npaths * (kUTileRows * 2 + 16) : 0));
  if (t0 > 0)
    bulk_g2s(stage, cu.U0 + ((size_t)ob * cu.n_kt + cu.kv0) * kTileBytes, (uint32_t)t0 * kTileBytes, bar);
  if (t1 > 0)
    bulk_g2s(stage + t0 * kTileBytes, cu.U1 + ((size_t)ob * cu.n_kt + (cu.kv0 + t0 - cu.n_kt)) * kTileBytes,
             (uint32_t)t1 * kTileBytes, bar);
  bulk_g2s(stage + kPkPlanesOff, cu.planes + (size_t)cu.kv0 * 256, (uint32_t)nt * 256, bar);
  if (last) {
    bulk_g2s(stage + kPkHOff, cu.h0 + (size_t)ob * kUTileRows, kUTileRows * 2, bar);
    bulk_g2s(stage + kPkTsOff, cu.ts0, 16, bar);
    if (cu.npaths == 2) {
      bulk_g2s(stage + kPkHOff + kUTileRows * 2, cu.h1 + (size_t)ob * kUTileRows, kUTileRows * 2, bar);
      bulk_g2s(stage + kPkTsOff + 16, cu.ts1, 16, bar);
    }
  }
}

__global__ void __launch_bounds__(kUWarps * 32) output_packed_kernel(const DecodeArgs a) {
  constexpr int S = kPkStages;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  unsigned char* my_ring = smem + (size_t)warp * S * kPkStageBytes;
  uint64_t* my_bar = reinterpret_cast<uint64_t*>(smem + (size_t)kUWarps * S * kPkStageBytes) + warp * S;

  const long long W = (long long)gridDim.x * kUWarps, gw = (long long)blockIdx.x * kUWarps + warp;
  const int i_begin = (int)(a.u_items * gw / W), i_end = (int)(a.u_items * (gw + 1) / W);
  if (i_begin >= i_end) return;   // no CTA-wide barriers in this kernel

  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init(&my_bar[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  grid_dep_wait();   // finalize's t' planes and steps

  PkCursor fd;
  fd.enter(a, layer_of(a.item_layer.u, a.n_layers, i_begin));
  fd.item = i_begin;
  fd.kv0 = 0;
  PkCursor cs = fd;
#pragma unroll 1
  for (int st = 0; st < S; ++st) {
    if (fd.item < i_end) {
      if (lane == 0) pk_issue(fd, my_ring + st * kPkStageBytes, &my_bar[st]);
      fd.advance(a);
    }
  }

  int d[8][1][4];   // starts at an item's first K-tile (zero-accumulator product)
  uint32_t consumed = 0;
  int slot = 0;
  bool dead = false;
  // this thread's B-operand column: row g/2 (path g/2 for g < 4), plane g%2
  const int pl_off = kPkPlanesOff + g * 32 + 4 * c;
  const int pc = min(c, 1);   // path whose sums this lane's columns 2c, 2c+1 hold (c < 2)

  while (cs.item < i_end) {
    if (!dead && !mbar_wait(&my_bar[slot], (consumed / S) & 1)) {
      dead = true;
      atomicOr(a.status, 1u << LB_ERR_TIMEOUT);
    }
    const unsigned char* stage = my_ring + slot * kPkStageBytes;
    const int nt = cs.ntile();
    const unsigned char* pl = stage + pl_off;
    if (cs.kv0 == 0) out_tile<1, 4, true>(d, stage, 0, lane, pl);
    else out_tile<1, 4>(d, stage, 0, lane, pl);
    if (nt == kUChunkTiles) {
#pragma unroll
      for (int t = 1; t < kUChunkTiles; ++t) out_tile<1, 4>(d, stage, t, lane, pl);
    } else {
#pragma unroll 1
      for (int t = 1; t < nt; ++t) out_tile<1, 4>(d, stage, t, lane, pl);
    }
    if (cs.item_end()) {
      // rows 128*ob + 16q + g (+8); lane c < npaths scales path c, then c = 0
      // adds c = 1's value and stores
      const bool live = c < cs.npaths;
      const uint16_t* hs = reinterpret_cast<const uint16_t*>(stage + kPkHOff + pc * kUTileRows * 2);
      const TStat tsp = reinterpret_cast<const TStat*>(stage + kPkTsOff)[pc];
      const float base = tsp.step * (float)tsp.sum, m2 = -2.f * tsp.step;
      const LayerDesc& L = a.layers[cs.li];
      uint16_t* yr = L.y + (cs.item - cs.u_begin) * kUTileRows + g;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int c0 = ((d[q][0][0] >> q) << 8) + (d[q][0][1] >> q);
        const int c1 = ((d[q][0][2] >> q) << 8) + (d[q][0][3] >> q);
        float v0 = live ? h2f(hs[16 * q + g]) * fmaf(m2, (float)c0, base) : 0.f;
        float v1 = live ? h2f(hs[16 * q + g + 8]) * fmaf(m2, (float)c1, base) : 0.f;
        v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
        if (c == 0) {
          yr[16 * q] = f2h(v0);
          yr[16 * q + 8] = f2h(v1);
        }
      }
    }
    // the stage has been read: refill it with the chunk `S` ahead
    __syncwarp();
    if (fd.item < i_end) {
      if (lane == 0) pk_issue(fd, my_ring + slot * kPkStageBytes, &my_bar[slot]);
      fd.advance(a);
    }
    ++consumed;
    if (++slot == S) slot = 0;
    cs.advance(a);
  }
}

// ------------------------------------------------------------------ launchers

// Launch `kern` on `st` with programmatic stream serialization: it may start
// while the previous kernel of the stream finishes, and waits for it with
// grid_dep_wait() before reading its output.
template <class K>
cudaError_t launch_dependent(K kern, int grid, int block, size_t smem, cudaStream_t st, const DecodeArgs& a) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int NB, int RB, int W>
constexpr size_t latent_smem() {
  return (size_t)W * kVStages * VCfg<NB>::kRPW * kChunkBytes + 2 * (size_t)xq_buf_bytes(NB, RB) +
         ((size_t)W * kVStages + 2) * 8;
}


template <int NB>
cudaError_t launch_finalize(const DecodeArgs& a, int, cudaStream_t st) {
  return launch_dependent(finalize_kernel<NB>, a.p_items, kFWarps * 32, 0, st, a);
}

// The non-packed output pass runs as the producer-fed kernel (true; up to 8
// batch rows) or as the per-warp kernel that issues its own copies (false).
constexpr bool kOutputFed = true;

template <int NB, int RS>
size_t output_smem() {
  return (size_t)kUWarps * OutCfg<NB>::kStages * out_stage_bytes(RS) + (size_t)kUWarps * OutCfg<NB>::kStages * 8;
}

template <int NB, int RB, int W>
cudaError_t launch_latent(const DecodeArgs& a, int num_sms, cudaStream_t st) {
  static_assert(RB == 4 * NB || (NB == 1 && RB == 1), "stored rows: 1 at batch 1, else 4 per n-block");
  constexpr size_t smem = latent_smem<NB, RB, W>();
  static_assert(smem <= 227 * 1024, "latent pass shared memory");
  auto kern = latent_pass_kernel<NB, RB, W>;
  // the shared-memory attribute and the occupancy it allows, once per device
  static PerDevice cache;
  int per_sm = 0;
  const int err = cache.get(current_device(), per_sm, [&](int& v) -> int {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, W * 32, smem);
    if (e == cudaSuccess && v < 1) e = cudaErrorInvalidConfiguration;
    return (int)e;
  });
  if (err != 0) return (cudaError_t)err;
  const int grid = max(1, min(a.v_items, per_sm * num_sms));
  return launch_dependent(kern, grid, W * 32, smem, st, a);
}

template <int NB, int RS>
cudaError_t launch_output_fed(const DecodeArgs& a, int num_sms, cudaStream_t st) {
  const size_t smem = fed_smem(RS);
  auto kern = output_fed_kernel<NB, RS>;
  // the shared-memory attribute and the occupancy it allows, once per device
  static PerDevice cache;
  int per_sm = 0;
  const int err = cache.get(current_device(), per_sm, [&](int& v) -> int {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, (kFedCons + 1) * 32, smem);
    if (e == cudaSuccess && v < 1) e = cudaErrorInvalidConfiguration;
    return (int)e;
  });
  if (err != 0) return (cudaError_t)err;
  // at least two items per consumer warp where there are enough
  const int grid = max(1, min((a.u_items + 2 * kFedCons - 1) / (2 * kFedCons), per_sm * num_sms));
  return launch_dependent(kern, grid, (kFedCons + 1) * 32, smem, st, a);
}

template <int NB, int RS>
cudaError_t launch_output(const DecodeArgs& a, int num_sms, cudaStream_t st) {
  // (at three or four n-blocks the fed kernel's 288 threads leave too few
  // registers for the accumulators; those batches keep the per-warp kernel)
  if constexpr (kOutputFed && NB <= 2) return launch_output_fed<NB, RS>(a, num_sms, st);
  const size_t smem = output_smem<NB, RS>();
  auto kern = output_pass_kernel<NB, RS>;
  // the shared-memory attribute and the occupancy it allows, once per device
  static PerDevice cache;
  int per_sm = 0;
  const int err = cache.get(current_device(), per_sm, [&](int& v) -> int {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, kUWarps * 32, smem);
    if (e == cudaSuccess && v < 1) e = cudaErrorInvalidConfiguration;
    return (int)e;
  });
  if (err != 0) return (cudaError_t)err;
  const int grid = max(1, min((a.u_items + kUWarps - 1) / kUWarps, per_sm * num_sms));
  return launch_dependent(kern, grid, kUWarps * 32, smem, st, a);
}

}  // namespace

cudaError_t launch_quantise_pass(const DecodeArgs& a, cudaStream_t st) {
  if (a.x_items < 1) return cudaErrorInvalidValue;
  quantise_input_kernel<<<(a.x_items + kQWarps - 1) / kQWarps, kQWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_latent_pass(const DecodeArgs& a, int, int num_sms, cudaStream_t st) {
  if (a.batch == 1) {
    if (a.v_warps == 3) return launch_latent<1, 1, 3>(a, num_sms, st);
    if (a.v_warps == 4) return launch_latent<1, 1, 4>(a, num_sms, st);
    return cudaErrorInvalidValue;
  }
  if (a.v_warps != 4) return cudaErrorInvalidValue;
  switch ((a.batch + 3) / 4) {
    case 1: return launch_latent<1, 4, 4>(a, num_sms, st);
    case 2: return launch_latent<2, 8, 4>(a, num_sms, st);
    // 9-16 rows: the two slice buffers fill most of shared memory, so one CTA
    // per SM runs; eight warps of one row block each (instead of four of two)
    // keep the same items with twice the resident warps
    case 3: return launch_latent<3, 12, 8>(a, num_sms, st);
    case 4: return launch_latent<4, 16, 8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_finalize_pass(const DecodeArgs& a, int max_s16, cudaStream_t st) {
  switch ((a.batch + 3) / 4) {
    case 1: return launch_finalize<1>(a, max_s16, st);
    case 2: return launch_finalize<2>(a, max_s16, st);
    case 3: return launch_finalize<3>(a, max_s16, st);
    case 4: return launch_finalize<4>(a, max_s16, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_output_packed(const DecodeArgs& a, int num_sms, cudaStream_t st) {
  const size_t smem = (size_t)kUWarps * kPkStages * kPkStageBytes + (size_t)kUWarps * kPkStages * 8;
  // the shared-memory attribute and the occupancy it allows, once per device
  static PerDevice cache;
  int per_sm = 0;
  const int err = cache.get(current_device(), per_sm, [&](int& v) -> int {
    cudaError_t e = cudaFuncSetAttribute(output_packed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, output_packed_kernel, kUWarps * 32, smem);
    if (e == cudaSuccess && v < 1) e = cudaErrorInvalidConfiguration;
    return (int)e;
  });
  if (err != 0) return (cudaError_t)err;
  const int grid = max(1, min((a.u_items + kUWarps - 1) / kUWarps, per_sm * num_sms));
  return launch_dependent(output_packed_kernel, grid, kUWarps * 32, smem, st, a);
}

cudaError_t launch_output_pass(const DecodeArgs& a, int num_sms, cudaStream_t st) {
  if (a.packed) return launch_output_packed(a, num_sms, st);
  if (a.batch == 1) return launch_output<1, 1>(a, num_sms, st);
  switch ((a.batch + 3) / 4) {
    case 1: return launch_output<1, 4>(a, num_sms, st);
    case 2: return launch_output<2, 8>(a, num_sms, st);
    case 3: return launch_output<3, 12>(a, num_sms, st);
    case 4: return launch_output<4, 16>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lb
