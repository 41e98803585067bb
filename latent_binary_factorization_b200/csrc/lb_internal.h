// Internal declarations shared by the CUDA translation units of the library.
// Nothing here is part of the C ABI (see include/littlebit.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "littlebit.h"

namespace lb {

constexpr int kMaxBatchDecode = 16;   // decode kernels: 1..16 rows
constexpr int kMaxRank = 1024;        // latent rank s accepted by the kernels
constexpr int kVTileRows = 16, kVTileK = 256;   // role-V tile
constexpr int kUTileRows = 128, kUTileK = 32;   // role-U tile
constexpr int kTileBytes = 512;

// Latent pass (V^T) work unit: one CTA reduces kVSliceTiles role-V K-tiles
// (kVSlice inputs) for every latent row of one path; warp w owns tiles
// kVTilesPerWarp*w .. kVTilesPerWarp*w + kVTilesPerWarp - 1 of the slice.
constexpr int kVWarps = 4;
constexpr int kVTilesPerWarp = 4;
constexpr int kVSliceTiles = kVWarps * kVTilesPerWarp;   // 16 tiles
constexpr int kVSlice = kVSliceTiles * kVTileK;          // 4096 inputs
// Output pass (U) work unit: one warp owns one 128-row block of one layer.
constexpr int kUWarps = 4;
// Quantisation of the int8 B operand: v = 256*hi + lo with hi, lo in [-128, 127]
// needs |v| <= 32639.
constexpr float kQMax = 32639.f;

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
inline int s16(int s) { return ceil_div(s, 16) * 16; }
inline int s32(int s) { return ceil_div(s, 32) * 32; }

// Per-path scratch written by the latent pass and read by the output pass.
//   partial : [n_slices][batch][s16] fp32  sums of one input slice
//   planes  : [batch][2][s32] int8          t' = l*t quantised, hi and lo bytes
//   tscale  : [batch] fp32                  t' ~= tscale * (256*hi + lo)
//   tsum    : [batch] int32                 sum over j of (256*hi + lo)
//   counter : slices of this path finished (reset to 0 by the last one)
struct PathScratch {
  float* partial;
  int8_t* planes;
  float* tscale;
  int32_t* tsum;
  unsigned int* counter;
};

struct PathDesc {
  const uint4* V;     // role-V tiles
  const uint4* U;     // role-U tiles
  const uint16_t* h;
  const uint16_t* g;
  const uint16_t* l;
  PathScratch ws;
};

struct LayerDesc {
  PathDesc p[2];
  const uint16_t* x;  // [batch][d_in] fp16
  uint16_t* y;        // [batch][d_out] fp16
  int d_in, d_out, s, npaths;
  int n_slices;       // ceil(d_in / kVSlice)
  int v_begin;        // first latent-pass work item of this layer
  int u_begin;        // first output-pass work item of this layer
  int pad;
};

struct DecodeArgs {
  const LayerDesc* layers;  // device table
  int n_layers;
  int batch;
  int v_items;              // total latent-pass items (layer, path, slice)
  int u_items;              // total output-pass items (layer, 128-row block)
};

// Launchers (decode.cu).  The batch selects the template (4 rows per n-block).
size_t latent_pass_smem(int batch, int max_s16);
cudaError_t launch_latent_pass(const DecodeArgs& a, int max_s16, int num_sms, cudaStream_t st);
cudaError_t launch_output_pass(const DecodeArgs& a, int num_sms, cudaStream_t st);

// pack.cu
cudaError_t launch_pack(const void* src, lb_dtype dt, int n_long, int s, int64_t stride_long,
                        int64_t stride_s, lb_role role, void* dst, cudaStream_t st);

}  // namespace lb
