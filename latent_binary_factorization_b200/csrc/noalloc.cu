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

#include <atomic>
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

// Device address of the array per device, set once by the first call on that
// device (with the device current); read by littlebit_device_status too.
std::atomic<unsigned char*> g_scratch_dev[lb::kMaxDevices];

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Writes the call's layer descriptor into the array.  The descriptor travels
// as a kernel argument, so no host buffer has to outlive the call.
__global__ void write_desc_kernel(const lb::LayerDesc d, lb::LayerDesc* dst) { *dst = d; }

// The array's device address on the current device `dev`, looked up (and its
// status word zeroed on `st`) by the first call on that device.
lb_status scratch_base(int dev, cudaStream_t st, unsigned char** base) {
  unsigned char* b = g_scratch_dev[dev].load(std::memory_order_acquire);
  if (!b) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return lb::cuda_fail(e);
    if (!ptr) return lb::cuda_fail(cudaErrorInvalidSymbol);
    e = cudaMemsetAsync(static_cast<unsigned char*>(ptr) + kStatusOff, 0, kTableOff - kStatusOff, st);
    if (e != cudaSuccess) return lb::cuda_fail(e);
    b = static_cast<unsigned char*>(ptr);
    g_scratch_dev[dev].store(b, std::memory_order_release);
  }
  *base = b;
  return LB_OK;
}

}  // namespace

namespace lb {

unsigned int* noalloc_status_word(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned char* b = g_scratch_dev[dev].load(std::memory_order_acquire);
  return b ? reinterpret_cast<unsigned int*>(b + kStatusOff) : nullptr;
}

}  // namespace lb

extern "C" {

lb_status littlebit_linear_forward_noalloc(const lb_layer* layer, const void* x_dev, void* y_dev, int batch,
                                           lb_dtype xdt, void* stream) {
  if (!layer || !x_dev || !y_dev) return LB_ERR_ARG;
  const lb_layer& L = *layer;
  lb_status chk = lb::check_layer(L);
  if (chk != LB_OK) return chk;
  if (batch < 1) return LB_ERR_SHAPE;
  if (batch > lb::kMaxBatchDecode || xdt != LB_F16) return LB_ERR_UNSUPPORTED;
  if (!aligned_to(x_dev, 16) || !aligned_to(y_dev, 16)) return LB_ERR_ALIGN;

  // scratch needed by this layer at this batch (the regular workspace's sizes)
  const int npaths = L.residual + 1;
  const size_t xq_b = lb::xq_bytes(L, batch), part_b = lb::partial_bytes(L, batch);
  const size_t planes_b = lb::planes_bytes(L, batch), tstat_b = lb::tstat_bytes(batch);
  if (kPathOff + (size_t)npaths * (xq_b + part_b + planes_b + tstat_b) > kNoAllocScratchBytes) return LB_ERR_SHAPE;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return lb::cuda_fail(e);
  if (dev < 0 || dev >= lb::kMaxDevices) return LB_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* base = nullptr;
  lb_status r = scratch_base(dev, st, &base);
  if (r != LB_OK) return r;

  const int n_slices = lb::ceil_div(L.d_in, lb::kVSlice);
  const int S16 = lb::s16(L.s);
  lb::LayerDesc D;
  std::memset(&D, 0, sizeof(D));
  D.x = static_cast<const uint16_t*>(x_dev);
  D.y = static_cast<uint16_t*>(y_dev);
  D.d_in = L.d_in;
  D.d_out = L.d_out;
  D.s = L.s;
  D.npaths = npaths;
  D.t_ld = lb::latent_row_elems(L.s, npaths);
  D.n_slices = n_slices;
  D.x_next = -1;
  const int vw = lb::latent_warps(1, batch, [&](int, int& n_rb, double& w) {
    n_rb = S16 / 16;
    w = 1.0;
  });
  D.n_rchunks = lb::ceil_div(S16 / 16, 2 * vw);
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
  // every region the kernels read is written earlier in the same call; the
  // status word keeps its bits until littlebit_device_status reads them
  write_desc_kernel<<<1, 1, 0, st>>>(D, reinterpret_cast<lb::LayerDesc*>(base + kTableOff));
  e = cudaGetLastError();
  if (e != cudaSuccess) return lb::cuda_fail(e);

  lb::DecodeArgs a;
  a.layers = reinterpret_cast<const lb::LayerDesc*>(base + kTableOff);
  a.item_layer = lb::ItemLayers{nullptr, nullptr, nullptr, nullptr};   // one layer: index 0
  a.status = reinterpret_cast<unsigned int*>(base + kStatusOff);
  a.n_layers = 1;
  a.batch = batch;
  a.v_items = npaths * D.n_slices * D.n_rchunks;
  a.u_items = L.d_out / lb::kUTileRows;
  a.p_items = npaths;
  a.x_items = D.n_slices * lb::q_row_groups(batch);
  a.v_warps = vw;
  a.packed = batch == 1 && L.residual ? 1 : 0;
  a.mode = lb::kModeForward;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return lb::cuda_fail(e);
  if (sms <= 0) return lb::cuda_fail(cudaErrorInvalidDevice);
  e = lb::launch_quantise_pass(a, st);
  if (e == cudaSuccess) e = lb::launch_latent_pass(a, S16, sms, st);
  if (e == cudaSuccess) e = lb::launch_finalize_pass(a, S16, st);
  if (e == cudaSuccess) e = lb::launch_output_pass(a, sms, st);
  return e == cudaSuccess ? LB_OK : lb::cuda_fail(e);
}

}  // extern "C"
