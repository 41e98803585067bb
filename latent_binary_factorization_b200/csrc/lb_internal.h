// Internal declarations shared by the CUDA translation units of the library.
// Nothing here is part of the C ABI (see include/littlebit.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "littlebit.h"
#include "per_device.h"

namespace lb {

// The device ordinal that is current on this thread (-1 if it cannot be read).
inline int current_device() {
  int d = -1;
  return cudaGetDevice(&d) == cudaSuccess ? d : -1;
}

constexpr int kMaxBatchDecode = 16;   // decode kernels: 1..16 rows
constexpr int kMaxRank = 1024;        // latent rank s accepted by the kernels
constexpr int kVTileRows = 16, kVTileK = 256;   // role-V tile
constexpr int kUTileRows = 128, kUTileK = 32;   // role-U tile
constexpr int kTileBytes = 512;

// Latent pass (V^T) work item: (layer, path, input slice, row chunk).  One CTA
// of W warps (latent_warps: 3 or 4) covers kVSlice inputs (kVSliceTiles
// K-tiles) for 2*W 16-row latent blocks; warp w owns row blocks 2w and 2w+1 of
// the chunk over the whole slice and streams their tiles in chunks of
// kChunkTiles K-tiles.  (Shorter slices for larger batches would shrink the
// quantised-input buffers and raise occupancy, but each slice change costs a
// buffer copy and wait, and finalize sums more partials: at batch 16 on a
// 28672-input layer, 512-input slices ran 4x slower.)
constexpr int kVSliceTiles = 8;
// Batch rows per quantise-pass item: a batch of B rows is quantised by
// ceil(B / kQRows) warps per input slice.
constexpr int kQRows = 4;
inline int q_row_groups(int batch) { return (batch + kQRows - 1) / kQRows; }
constexpr int kVSlice = kVSliceTiles * kVTileK;          // 2048 inputs
constexpr int kVStages = 2;                              // bulk-copy ring per warp

// Latent-pass CTA width for a call: at batch 1, 3 or 4 warps, whichever leaves
// fewer row-block slots of the items idle (a chunk is 2*W row blocks), weighted
// by each layer's V bits and with 3-warp CTAs discounted for their occupancy
// (15 against 16 resident warps per SM); else 4.  rb_work(i, n_rb, w) gives
// layer i's 16-row block count and weight.
template <class F>
inline int latent_warps(int n, int batch, F rb_work) {
  if (batch != 1) return 4;
  double sc3 = 0.0, sc4 = 0.0;
  for (int i = 0; i < n; ++i) {
    int n_rb = 1;
    double w = 0.0;
    rb_work(i, n_rb, w);
    sc3 += w * n_rb / (double)(((n_rb + 5) / 6) * 6) * (15.0 / 16.0);
    sc4 += w * n_rb / (double)(((n_rb + 7) / 8) * 8);
  }
  return sc3 > sc4 ? 3 : 4;
}
constexpr int kChunkTiles = 4;                           // K-tiles per bulk copy
constexpr int kChunkBytes = kChunkTiles * kTileBytes;    // 2048

// Quantised input slice (u = g * x on kVSlice inputs, per batch row), written by
// the quantise pass and copied whole into the latent pass's shared memory:
//   [TStat x 4*nb]  step and sum of v per batch row (rows >= batch are zero)
//   [K-block kb][column n][thread c] (b0, b1) B-fragment pairs of the int8
//       mma: b0 = inputs 32kb + 4c .. +3, b1 = inputs 32kb + 16 + 4c .. +3;
//       column 2r holds batch row r's hi bytes, 2r + 1 its lo bytes.
// xq_rows(batch) rows are stored: one at batch 1 (the product's other columns
// then repeat row 0 and their sums are ignored), else 4*nb.
__host__ __device__ inline int xq_nb(int batch) { return (batch + 3) / 4; }
__host__ __device__ inline int xq_rows(int batch) { return batch == 1 ? 1 : 4 * xq_nb(batch); }
__host__ __device__ inline int xq_stats_bytes(int batch) { return 64 * xq_nb(batch); }
__host__ __device__ inline int xq_slice_bytes(int batch) {
  return (xq_stats_bytes(batch) + kVSlice * 2 * xq_rows(batch) + 127) & ~127;
}

// Output pass (U) work item: (layer, 128 output rows), one warp.
constexpr int kUWarps = 4;

// Quantisation of the int8 B operand: v = 256*hi + lo with hi, lo in [-128, 127]
// needs |v| <= 32639.
constexpr float kQMax = 32639.f;

// Device status word bits raised by the kernels (littlebit_device_status).
constexpr unsigned kStatusTimeout = 1u << LB_ERR_TIMEOUT;
constexpr unsigned kStatusRange = 1u << LB_ERR_RANGE;

// Non-zero when either fp16 of the pair in `w` is inf or NaN (exponent field
// all ones): adding 1 to an all-ones exponent carries into the sign position.
__host__ __device__ inline unsigned half2_nonfinite(unsigned w) {
  return ((w & 0x7c007c00u) + 0x04000400u) & 0x80008000u;
}

// Bounded waits: polls of mbarrier.try_wait (each may suspend up to ~1 us)
// before a wait gives up (a few seconds in total).
constexpr int kSpinLimit = 1 << 22;

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
inline int s16(int s) { return ceil_div(s, 16) * 16; }
inline int s32(int s) { return ceil_div(s, 32) * 32; }

// Quantised t' of one path, per batch row b: t'_j ~= step_b * (256*hi + lo).
struct TStat {
  float step;   // quantisation step
  int sum;      // sum over j < s of (256*hi + lo)
  int pad[2];
};

// Per-path scratch of the decode passes.
//   xq      : [n_slices][xq_slice_bytes]        quantised input slices (quantise pass)
//   partial : [batch][s16][ns4] fp32             latent sums per input slice (latent pass;
//                                                ns4 = n_slices rounded up to 4, pad unused)
//   planes  : [s32/32][4*nb][2][32] int8         hi and lo bytes of t', K-tile major
//                                                (nb = ceil(batch/4); rows >= batch are zero)
//   tstat   : [4*nb] TStat                        (planes and tstat: finalize pass)
struct PathScratch {
  unsigned char* xq;
  float* partial;
  int8_t* planes;
  TStat* tstat;
};

struct PathDesc {
  const uint4* V;     // role-V tiles
  const uint4* U;     // role-U tiles
  const uint16_t* h;
  const uint16_t* g;
  const uint16_t* l;
  PathScratch ws;
};

// What a forward call computes (Samsung LittleBit article, section 4, the
// KV-cache bullet: a factorised K/V projection can be cached as its latent):
//   kModeForward: y = layer(x)                       (all passes)
//   kModeLatent:  t = [t'_1 | t'_2] cache rows of x    (no output pass; the
//                 latent rows are written where y would go)
//   kModeExpand:  y = sum_p h_p (.) U_p t'_p from cache rows (no input or
//                 latent pass; the cache rows are read where x would be)
// A cache row holds npaths*s fp16 values, path p at columns p*s .. p*s+s-1,
// rows latent_row_elems(s, npaths) elements apart.
enum CallMode { kModeForward = 0, kModeLatent = 1, kModeExpand = 2 };
inline int latent_row_elems(int s, int npaths) { return (npaths * s + 7) / 8 * 8; }

struct LayerDesc {
  PathDesc p[2];
  const uint16_t* x;  // [batch][d_in] fp16; kModeExpand: the cache rows [batch][t_ld]
  uint16_t* y;        // [batch][d_out] fp16; kModeLatent: the cache rows [batch][t_ld]
  int t_ld;           // elements between cache rows (latent_row_elems)
  int d_in, d_out, s, npaths;
  int n_slices;       // ceil(d_in / kVSlice)
  int n_rchunks;      // ceil(s16 / 16 / (2 * latent-pass warps))
  int v_begin;        // first latent-pass work item of this layer
  int u_begin;        // first output-pass work item of this layer
  int p_begin;        // first (layer, path) index of this layer
  int x_begin;        // first quantise-pass item (x group, input slice, row group) of this layer's x group
                      // (set on the group's first layer)
  int x_next;         // next layer of the call that reads the same x (same pointer and d_in), or -1
};

// Layer index of every work item of each pass (device arrays built with the
// table; null when the call has one layer, whose index is 0).
struct ItemLayers {
  const int* x;   // quantise items
  const int* v;   // latent items
  const int* p;   // (layer, path) items
  const int* u;   // output items
};

struct DecodeArgs {
  const LayerDesc* layers;  // device table
  ItemLayers item_layer;
  unsigned int* status;     // device error word (LB_ERR_TIMEOUT bit on a wait timeout)
  int n_layers;
  int batch;
  int v_items;              // total latent-pass items
  int u_items;              // total output-pass items (layer, 128-row block)
  int p_items;              // total (layer, path) pairs
  int x_items;              // total quantise-pass items (group of layers sharing x, input slice, row group)
  int v_warps;              // latent-pass CTA width (3 or 4; latent_warps)
  int packed;               // batch 1 with a residual layer: paths share the output pass's product
  int mode;                 // CallMode
};

// Launchers (decode.cu), in stream order quantise -> latent -> finalize ->
// output.  The batch selects the template (4 rows per n-block).
cudaError_t launch_quantise_pass(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_latent_pass(const DecodeArgs& a, int max_s16, int num_sms, cudaStream_t st);
cudaError_t launch_finalize_pass(const DecodeArgs& a, int max_s16, cudaStream_t st);
cudaError_t launch_output_pass(const DecodeArgs& a, int num_sms, cudaStream_t st);
// selfcheck.cu: one warp polls `polls` times (1..kSpinLimit) an mbarrier that
// nothing completes and raises LB_ERR_TIMEOUT in *status, as every bounded
// wait of the forward kernels does when it gives up.
cudaError_t launch_wait_timeout_probe(unsigned int* status, int polls, cudaStream_t st);

// prefill.cu: layers of M rows (multiple of 128), x fp16 or bf16 (y the same)
int prefill_sp(int s, int npaths);
size_t prefill_layer_bytes(int M, int d_in, int d_out, int s, int npaths);
long long prefill_layer_tiles(int M, int d_out, int s, int npaths);   // GEMM1 + GEMM2 tiles
size_t prefill_table_bytes(int n_layers, long long tiles);
constexpr int kPrefillMaxGroup = 4096;   // layers per chunk
constexpr int kPrepKinds = 4;            // preparation steps: x, B1, B2, T' from cache rows
// A chunk of layers: its table's place in the call's table image and the two
// GEMMs' tile counts and grids.
struct PrefillPlan {
  int n;
  int pair;                      // 1: 256-row tiles on pairs of SMs (M a multiple of 256)
  int tiles1, tiles2, grid1, grid2;
  int prep_grid[kPrepKinds];     // blocks of the grouped x, B1, B2 and cache-to-T' preparation launches
  size_t table_off, table_bytes;
  size_t jobs_off;               // preparation jobs, from table_off
};
// Append the chunk's table image (GEMM problems, tile schedules and the
// per-layer preparation jobs) to img; its device pointers refer to the
// chunk's operand buffers at `bufs`, the inputs xs and the outputs ys.
void plan_prefill_chunk(const LayerDesc* Ls, const void* const* xs, void* const* ys, int n, int M, int x_bf16,
                        int mode, unsigned char* bufs, int num_sms, int pair_slots, std::vector<unsigned char>& img,
                        PrefillPlan& plan);
// Clusters of two CTAs of the 256-row GEMM that the current device holds at
// once (0: none); a CUDA error code, 0 on success.
int prefill_pair_slots(int* slots);
// A chunk's operand preparation (three grouped launches), then its two
// grouped GEMM launches; both read the table image uploaded at table_dev.
cudaError_t launch_prefill_prep(const PrefillPlan& plan, const unsigned char* table_dev, unsigned int* status,
                                cudaStream_t st);
cudaError_t launch_prefill_gemms(const PrefillPlan& plan, const unsigned char* table_dev, unsigned int* status,
                                 cudaStream_t st);

// littlebit_capi.cu: helpers shared by the entry points.
// Records `e` as this thread's last CUDA error text and returns LB_ERR_CUDA.
lb_status cuda_fail(cudaError_t e);
// Shape, pointer and alignment checks of one layer (not of x and y).
lb_status check_layer(const lb_layer& L);
// Bytes of each per-path decode scratch region of a layer at this batch
// (every region a multiple of 256 bytes; PathScratch order).
size_t xq_bytes(const lb_layer& L, int batch);
size_t partial_bytes(const lb_layer& L, int batch);
size_t planes_bytes(const lb_layer& L, int batch);
size_t tstat_bytes(int batch);
size_t path_scratch_bytes(const lb_layer& L, int batch);

// noalloc.cu: device address of the allocation-free forward's status word on
// device `dev`, or null before that entry point's first call on the device.
unsigned int* noalloc_status_word(int dev);

// init.cu: Dual-SVID and Joint-ITQ (scratch sizes in floats)
size_t dual_svid_scratch_floats(int d_out, int d_in, int s);
cudaError_t launch_dual_svid(const float* Uf, const float* Vf, int d_out, int d_in, int s, int iters, void* U_bits,
                             void* V_bits, uint16_t* h, uint16_t* g, uint16_t* l, float* scratch, cudaStream_t st);
size_t itq_scratch_floats(int n_rows, int s);
cudaError_t launch_joint_itq(float* X, int n_rows, int s, int iters, int ns_steps, float* R, int r_given,
                             float* scratch, cudaStream_t st);

// pack.cu
cudaError_t launch_unpack(const void* src, int n_long, int s, lb_role role, int8_t* dst, cudaStream_t st);
cudaError_t launch_pack(const void* src, lb_dtype dt, int n_long, int s, int64_t stride_long,
                        int64_t stride_s, lb_role role, void* dst, cudaStream_t st);

}  // namespace lb
