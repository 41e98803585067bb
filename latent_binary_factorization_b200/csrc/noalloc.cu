// littlebit_linear_forward_noalloc: the decode forward of one layer with its
// scratch in a fixed device array instead of a cudaMalloc'ed workspace.
//
// Some callers cannot let a library allocate device memory: a process whose
// device memory is reserved up front by its own allocator (so a cudaMalloc
// behind its back can fail or fragment the pool), or a latency-critical loop
// that cannot afford the device-wide synchronisation that cudaMalloc and
// cudaFree imply.  This entry point never allocates: the latent-vector scratch
// lives in the file-scope array below, which every GPU that loads the library
// holds until the process exits.
#include <cuda_runtime.h>

#include <cstring>

#include "lb_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 1u << 20;   // 1 MiB per device

// The shared scratch.  In host code this name is only a stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Layout inside the array: [status word][one LayerDesc][per path: xq | partial
// | planes | tstat], each region 256-byte aligned.
constexpr size_t kStatusOff = 0;
constexpr size_t kTableOff = 256;
constexpr size_t kPathOff = 512;
static_assert(sizeof(lb::LayerDesc) <= kPathOff - kTableOff, "layer descriptor must fit its slot");

constexpr int kMaxDevices = 64;
unsigned char* g_scratch_dev[kMaxDevices] = {nullptr};   // device address per device, set once

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

lb_status check(const lb_layer& L, const void* x, const void* y, int batch, lb_dtype xdt) {
  if (!x || !y) return LB_ERR_ARG;
  if (L.d_in < 256 || L.d_in % 256 != 0 || L.d_out < 128 || L.d_out % 128 != 0) return LB_ERR_SHAPE;
  if (L.s < 1 || L.s > lb::kMaxRank) return LB_ERR_SHAPE;
  if (L.residual != 0 && L.residual != 1) return LB_ERR_ARG;
  if (batch < 1 || batch > lb::kMaxBatchDecode) return batch < 1 ? LB_ERR_SHAPE : LB_ERR_UNSUPPORTED;
  if (xdt != LB_F16) return LB_ERR_UNSUPPORTED;
  if (!aligned_to(x, 16) || !aligned_to(y, 16)) return LB_ERR_ALIGN;
  for (int p = 0; p <= L.residual; ++p) {
    const lb_path& P = L.path[p];
    if (!P.V_bits || !P.U_bits || !P.h || !P.g || !P.l) return LB_ERR_ARG;
    if (!aligned_to(P.V_bits, 16) || !aligned_to(P.U_bits, 16)) return LB_ERR_ALIGN;
    if (!aligned_to(P.h, 16) || !aligned_to(P.g, 16) || !aligned_to(P.l, 2)) return LB_ERR_ALIGN;
  }
  return LB_OK;
}

}  // namespace

extern "C" {

lb_status littlebit_linear_forward_noalloc(const lb_layer* layer, const void* x_dev, void* y_dev, int batch,
                                           lb_dtype xdt, void* stream) {
  if (!layer) return LB_ERR_ARG;
  const lb_layer& L = *layer;
  lb_status chk = check(L, x_dev, y_dev, batch, xdt);
  if (chk != LB_OK) return chk;

  // scratch needed by this layer at this batch
  const int n_slices = lb::ceil_div(L.d_in, lb::kVSlice);
  const int S16 = lb::s16(L.s), S32 = lb::s32(L.s);
  const size_t xq_b = round256((size_t)n_slices * lb::xq_slice_bytes(batch));
  const size_t part_b = round256((size_t)lb::ceil_div(n_slices, 4) * 4 * batch * S16 * sizeof(float));
  const int bpad = lb::ceil_div(batch, 4) * 4;   // t' planes and stats padded to groups of 4 rows
  // at batch 1 path 0's planes hold the combined K range of both paths
  const size_t planes_b = round256((size_t)bpad * 2 * S32 * (batch == 1 ? 2 : 1));
  const size_t tstat_b = round256((size_t)bpad * sizeof(lb::TStat));
  const int npaths = L.residual + 1;
  if (kPathOff + (size_t)npaths * (xq_b + part_b + planes_b + tstat_b) > kNoAllocScratchBytes) return LB_ERR_SHAPE;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LB_ERR_CUDA;
  if (!g_scratch_dev[dev]) {
    // once per device, with that device current
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) return LB_ERR_CUDA;
    g_scratch_dev[dev] = static_cast<unsigned char*>(ptr);
  }
  unsigned char* base = g_scratch_dev[dev];
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  lb::LayerDesc D;
  std::memset(&D, 0, sizeof(D));
  D.x = static_cast<const uint16_t*>(x_dev);
  D.y = static_cast<uint16_t*>(y_dev);
  D.d_in = L.d_in;
  D.d_out = L.d_out;
  D.s = L.s;
  D.npaths = npaths;
  D.n_slices = n_slices;
  const int vw = lb::latent_warps(1, batch, [&](int, int& n_rb, double& w) {
    n_rb = S16 / 16;
    w = 1.0;
  });
  D.n_rchunks = lb::ceil_div(S16 / 16, 2 * vw);
  D.v_begin = 0;
  D.u_begin = 0;
  D.p_begin = 0;
  D.x_begin = 0;
  size_t off = kPathOff;
  for (int p = 0; p < npaths; ++p) {
    lb::PathDesc& P = D.p[p];
    P.V = static_cast<const uint4*>(L.path[p].V_bits);
    P.U = static_cast<const uint4*>(L.path[p].U_bits);
    P.h = L.path[p].h;
    P.g = L.path[p].g;
    P.l = L.path[p].l;
    P.ws.xq = base + off;
    off += xq_b;
    P.ws.partial = reinterpret_cast<float*>(base + off);
    off += part_b;
    P.ws.planes = reinterpret_cast<int8_t*>(base + off);
    off += planes_b;
    P.ws.tstat = reinterpret_cast<lb::TStat*>(base + off);
    off += tstat_b;
  }
  // every call shares the array: the status word must start at zero, whatever
  // the previous call left there (every other region is written before it is read)
  e = cudaMemsetAsync(base + kStatusOff, 0, kTableOff - kStatusOff, st);
  if (e != cudaSuccess) return LB_ERR_CUDA;
  e = cudaMemcpyAsync(base + kTableOff, &D, sizeof(D), cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return LB_ERR_CUDA;

  lb::DecodeArgs a;
  a.layers = reinterpret_cast<const lb::LayerDesc*>(base + kTableOff);
  a.item_layer = lb::ItemLayers{nullptr, nullptr, nullptr, nullptr};   // one layer: index 0
  a.status = reinterpret_cast<unsigned int*>(base + kStatusOff);
  a.n_layers = 1;
  a.batch = batch;
  a.v_items = npaths * D.n_slices * D.n_rchunks;
  a.u_items = L.d_out / lb::kUTileRows;
  a.p_items = npaths;
  a.x_items = npaths * D.n_slices;
  a.v_warps = vw;
  a.packed = batch == 1 && L.residual ? 1 : 0;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess || sms <= 0) return LB_ERR_CUDA;
  e = lb::launch_quantise_pass(a, st);
  if (e != cudaSuccess) return LB_ERR_CUDA;
  e = lb::launch_latent_pass(a, S16, sms, st);
  if (e != cudaSuccess) return LB_ERR_CUDA;
  e = lb::launch_finalize_pass(a, S16, st);
  if (e != cudaSuccess) return LB_ERR_CUDA;
  e = lb::launch_output_pass(a, sms, st);
  if (e != cudaSuccess) return LB_ERR_CUDA;
  return LB_OK;
}

}  // extern "C"
