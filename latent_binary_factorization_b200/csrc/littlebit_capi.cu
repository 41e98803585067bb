// Host side of the C ABI declared in include/littlebit.h: argument checks,
// per-(device, stream) workspaces, the device descriptor table and launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "lb_internal.h"

namespace {

thread_local char g_last_cuda_error[256] = "";

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

namespace lb {

lb_status cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return LB_ERR_CUDA;
}

lb_status check_layer(const lb_layer& L) {
  if (L.d_in < 256 || L.d_in % 256 != 0) return LB_ERR_SHAPE;
  if (L.d_out < 128 || L.d_out % 128 != 0) return LB_ERR_SHAPE;
  if (L.s < 1 || L.s > kMaxRank) return LB_ERR_SHAPE;
  if (L.residual != 0 && L.residual != 1) return LB_ERR_ARG;
  for (int p = 0; p <= L.residual; ++p) {
    const lb_path& P = L.path[p];
    if (!P.V_bits || !P.U_bits || !P.h || !P.g || !P.l) return LB_ERR_ARG;
    if (!aligned(P.V_bits, 16) || !aligned(P.U_bits, 16)) return LB_ERR_ALIGN;
    if (!aligned(P.h, 16) || !aligned(P.g, 16) || !aligned(P.l, 2)) return LB_ERR_ALIGN;
  }
  return LB_OK;
}

size_t xq_bytes(const lb_layer& L, int batch) {
  return align_up((size_t)ceil_div(L.d_in, kVSlice) * xq_slice_bytes(batch), 256);
}
size_t partial_bytes(const lb_layer& L, int batch) {
  const size_t ns4 = (size_t)ceil_div(ceil_div(L.d_in, kVSlice), 4) * 4;
  return align_up(ns4 * batch * s16(L.s) * sizeof(float), 256);
}
// t' planes and stats are padded to whole groups of four batch rows; at batch
// 1 path 0's planes hold the combined K range of both paths (packed output pass)
size_t planes_bytes(const lb_layer& L, int batch) {
  return align_up((size_t)ceil_div(batch, 4) * 4 * 2 * s32(L.s) * (batch == 1 ? 2 : 1), 256);
}
size_t tstat_bytes(int batch) { return align_up((size_t)ceil_div(batch, 4) * 4 * sizeof(TStat), 256); }
size_t path_scratch_bytes(const lb_layer& L, int batch) {
  return xq_bytes(L, batch) + partial_bytes(L, batch) + planes_bytes(L, batch) + tstat_bytes(batch);
}

}  // namespace lb

namespace {

using lb::check_layer;
using lb::cuda_fail;
using lb::partial_bytes;
using lb::path_scratch_bytes;
using lb::planes_bytes;
using lb::tstat_bytes;
using lb::xq_bytes;

struct Workspace {
  void* buf = nullptr;
  size_t cap = 0;
  std::vector<unsigned char> table;   // last descriptor table uploaded
  // prefill: side stream for operand preparation and the events that order it
  // against the caller's stream (created on first use)
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr, prep_done[2] = {nullptr, nullptr}, gemm_done[2] = {nullptr, nullptr};
  // the last call's arguments and what was derived from them: a call with the
  // same arguments (a serving loop's every step) reuses them and enqueues
  // kernels and events only
  std::vector<unsigned char> key;
  lb::DecodeArgs dargs{};
  int d_max_s16 = 16;
  std::vector<lb::PrefillPlan> p_plans;
};

// Call arguments that determine a forward's tables and plans.
std::vector<unsigned char> call_key(char mode, const lb_layer* layers, int n, const void* const* xs,
                                    void* const* ys, int batch, int x_bf16) {
  std::vector<unsigned char> k;
  const size_t lb = (size_t)n * sizeof(lb_layer), pb = (size_t)n * sizeof(void*);
  k.resize(16 + lb + 2 * pb);
  k[0] = (unsigned char)mode;
  std::memcpy(k.data() + 4, &batch, 4);
  std::memcpy(k.data() + 8, &x_bf16, 4);
  std::memcpy(k.data() + 12, &n, 4);
  std::memcpy(k.data() + 16, layers, lb);
  std::memcpy(k.data() + 16 + lb, xs, pb);
  std::memcpy(k.data() + 16 + lb + pb, ys, pb);
  return k;
}

void release_workspace(Workspace& w) {
  if (w.buf) cudaFree(w.buf);
  cudaEvent_t* evs[] = {&w.fork, &w.join, &w.prep_done[0], &w.prep_done[1], &w.gemm_done[0], &w.gemm_done[1]};
  for (cudaEvent_t* ev : evs)
    if (*ev) cudaEventDestroy(*ev);
  if (w.side) cudaStreamDestroy(w.side);
  w = Workspace();
}

// Workspaces are keyed by (device, stream, tag).  The tag separates calls
// that alternate on one stream, so that each keeps its cached tables: the
// prefill part and each 16-row decode group of a mixed batch, and each chunk
// of a host-buffer stack call (ws_tag below).
std::mutex g_mu;
using WsKey = std::tuple<int, cudaStream_t, int>;
std::map<WsKey, Workspace> g_ws;

// tag = (base << 8) | part; base 0 is the device-pointer API, base c+1 chunk c
// of littlebit_linear_forward_many_host; part 0 is prefill, 1 + g decode group g.
int ws_tag(int base, int part) { return (base << 8) | part; }
int g_num_sms[64] = {0};

int num_sms(int dev) {
  if (dev < 0 || dev >= 64) return 148;
  if (g_num_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}


constexpr size_t kStatusBytes = 256;   // device status word at the start of a workspace
constexpr int kMaxHostChunks = 64;     // chunks of one host-buffer stack call

// Replaces the workspace buffer with a zeroed one of `cap` bytes.  The old
// buffer is freed once `st` has drained; its status word is carried over, so
// bits raised before the growth are still reported by littlebit_device_status.
lb_status grow_workspace(Workspace& ws, size_t cap, cudaStream_t st) {
  unsigned int status = 0;
  cudaError_t e;
  if (ws.buf) {
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemcpy(&status, ws.buf, sizeof(status), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    cudaFree(ws.buf);
    ws.buf = nullptr;
    ws.cap = 0;
  }
  e = cudaMalloc(&ws.buf, cap);
  if (e != cudaSuccess) return cuda_fail(e);
  ws.cap = cap;
  ws.table.clear();
  e = cudaMemsetAsync(ws.buf, 0, cap, st);
  // pageable source: staged before cudaMemcpyAsync returns
  if (e == cudaSuccess && status) e = cudaMemcpyAsync(ws.buf, &status, sizeof(status), cudaMemcpyHostToDevice, st);
  return e == cudaSuccess ? LB_OK : cuda_fail(e);
}

// The four decode launches of a prepared call; events[i] (if given) is
// recorded right after launch i.
// The launches of a prepared call: all four for a forward, the first three
// for a latent-only call, finalize and output for an expand call.
lb_status decode_launch(const lb::DecodeArgs& a, int max_s16, int sms, cudaStream_t st, const cudaEvent_t* events,
                        int n_events) {
  auto mark = [&](int i) { return i < n_events && events[i] ? cudaEventRecord(events[i], st) : cudaSuccess; };
  cudaError_t e = cudaSuccess;
  if (a.mode != lb::kModeExpand) {
    e = lb::launch_quantise_pass(a, st);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess) e = lb::launch_latent_pass(a, max_s16, sms, st);
    if (e == cudaSuccess) e = mark(1);
  }
  if (e == cudaSuccess) e = lb::launch_finalize_pass(a, max_s16, st);
  if (e == cudaSuccess) e = mark(2);
  if (e == cudaSuccess && a.mode != lb::kModeLatent) e = lb::launch_output_pass(a, sms, st);
  return e == cudaSuccess ? LB_OK : cuda_fail(e);
}

lb_status decode_forward(const lb_layer* layers, int n, const void* const* xs, void* const* ys, int batch,
                         int mode, cudaStream_t st, const cudaEvent_t* events, int n_events, int tag) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& ws = g_ws[{dev, st, tag}];
  std::vector<unsigned char> key = call_key((char)('D' + 16 * mode), layers, n, xs, ys, batch, 0);
  if (ws.buf && ws.key == key) return decode_launch(ws.dargs, ws.d_max_s16, num_sms(dev), st, events, n_events);
  ws.key.clear();

  // ---- work items of each pass, per layer
  const int vw = lb::latent_warps(n, batch, [&](int i, int& n_rb, double& w) {
    n_rb = lb::s16(layers[i].s) / 16;
    w = (double)(layers[i].residual + 1) * n_rb * layers[i].d_in;
  });
  // layers that read the same x (same pointer and width) form one quantise
  // group: x_lead[i] is the group's first layer, x_next[i] the next member
  std::vector<int> x_lead(n), x_next(n, -1);
  {
    std::map<std::pair<const void*, int>, int> last;   // (x, d_in) -> latest member
    for (int i = 0; i < n; ++i) {
      auto it = last.find({xs[i], layers[i].d_in});
      if (it == last.end()) {
        x_lead[i] = i;
      } else {
        x_lead[i] = x_lead[it->second];
        x_next[it->second] = i;
      }
      last[{xs[i], layers[i].d_in}] = i;
    }
  }
  int x_items = 0, v_items = 0, p_items = 0, u_items = 0;
  int max_s16 = 16;
  size_t scratch = 0;
  for (int i = 0; i < n; ++i) {
    const lb_layer& L = layers[i];
    const int npaths = L.residual + 1, n_slices = lb::ceil_div(L.d_in, lb::kVSlice);
    if (x_lead[i] == i) x_items += n_slices * lb::q_row_groups(batch);
    v_items += npaths * n_slices * lb::ceil_div(lb::s16(L.s) / 16, 2 * vw);
    p_items += npaths;
    u_items += L.d_out / lb::kUTileRows;
    scratch += (size_t)npaths * path_scratch_bytes(L, batch);
    max_s16 = std::max(max_s16, lb::s16(L.s));
  }
  const int n_items = x_items + v_items + p_items + u_items;

  // ---- sizes: [status][table][item -> layer maps][per-path scratch...]
  const size_t table_bytes = align_up((size_t)n * sizeof(lb::LayerDesc), 256);
  const size_t map_bytes = align_up((size_t)n_items * sizeof(int), 256);
  const size_t total = kStatusBytes + table_bytes + map_bytes + scratch;

  if (ws.cap < total) {
    const lb_status r = grow_workspace(ws, align_up(total + total / 4, 1 << 20), st);
    if (r != LB_OK) return r;
  }

  // ---- descriptor table and item maps
  unsigned char* base = static_cast<unsigned char*>(ws.buf);
  lb::LayerDesc* table = reinterpret_cast<lb::LayerDesc*>(base + kStatusBytes);
  int* maps = reinterpret_cast<int*>(base + kStatusBytes + table_bytes);
  size_t off = kStatusBytes + table_bytes + map_bytes;
  // the table and the maps are one host block, compared and uploaded together
  const size_t tb = (size_t)n * sizeof(lb::LayerDesc);
  std::vector<unsigned char> host(tb + (size_t)n_items * sizeof(int));
  lb::LayerDesc* tab = reinterpret_cast<lb::LayerDesc*>(host.data());
  int* xm = reinterpret_cast<int*>(host.data() + tb);
  int* vm = xm + x_items;
  int* pm = vm + v_items;
  int* um = pm + p_items;
  int xi = 0, vi = 0, pi = 0, ui = 0;
  for (int i = 0; i < n; ++i) {
    const lb_layer& L = layers[i];
    lb::LayerDesc& D = tab[i];
    std::memset(&D, 0, sizeof(D));
    D.x = static_cast<const uint16_t*>(xs[i]);
    D.y = static_cast<uint16_t*>(ys[i]);
    D.d_in = L.d_in;
    D.d_out = L.d_out;
    D.s = L.s;
    D.npaths = L.residual + 1;
    D.t_ld = lb::latent_row_elems(L.s, D.npaths);
    D.n_slices = lb::ceil_div(L.d_in, lb::kVSlice);
    D.n_rchunks = lb::ceil_div(lb::s16(L.s) / 16, 2 * vw);
    D.x_begin = x_lead[i] == i ? xi : -1;
    D.x_next = x_next[i];
    D.v_begin = vi;
    D.p_begin = pi;
    D.u_begin = ui;
    if (x_lead[i] == i)
      for (int k = 0; k < D.n_slices * lb::q_row_groups(batch); ++k) xm[xi++] = i;
    for (int k = 0; k < D.npaths * D.n_slices * D.n_rchunks; ++k) vm[vi++] = i;
    for (int k = 0; k < D.npaths; ++k) pm[pi++] = i;
    for (int k = 0; k < L.d_out / lb::kUTileRows; ++k) um[ui++] = i;
    for (int p = 0; p < D.npaths; ++p) {
      lb::PathDesc& P = D.p[p];
      P.V = static_cast<const uint4*>(L.path[p].V_bits);
      P.U = static_cast<const uint4*>(L.path[p].U_bits);
      P.h = L.path[p].h;
      P.g = L.path[p].g;
      P.l = L.path[p].l;
      P.ws.xq = base + off;
      off += xq_bytes(L, batch);
      P.ws.partial = reinterpret_cast<float*>(base + off);
      off += partial_bytes(L, batch);
      P.ws.planes = reinterpret_cast<int8_t*>(base + off);
      off += planes_bytes(L, batch);
      P.ws.tstat = reinterpret_cast<lb::TStat*>(base + off);
      off += tstat_bytes(batch);
    }
  }
  if (ws.table.size() != host.size() || std::memcmp(ws.table.data(), host.data(), host.size()) != 0) {
    // pageable source: the calls return once the bytes are staged, so `host`
    // may go out of scope; stream order protects kernels still reading them
    e = cudaMemcpyAsync(table, host.data(), tb, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e);
    if (n_items > 0) {
      e = cudaMemcpyAsync(maps, host.data() + tb, (size_t)n_items * sizeof(int), cudaMemcpyHostToDevice, st);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    ws.table.swap(host);
  }

  lb::DecodeArgs a;
  a.layers = table;
  a.item_layer.x = maps;
  a.item_layer.v = maps + x_items;
  a.item_layer.p = maps + x_items + v_items;
  a.item_layer.u = maps + x_items + v_items + p_items;
  a.status = reinterpret_cast<unsigned int*>(base);
  a.n_layers = n;
  a.batch = batch;
  a.v_items = v_items;
  a.u_items = u_items;
  a.p_items = p_items;
  a.x_items = x_items;
  a.v_warps = vw;
  a.mode = mode;
  a.packed = 0;
  if (batch == 1)
    for (int i = 0; i < n; ++i) a.packed |= layers[i].residual;
  ws.key.swap(key);
  ws.dargs = a;
  ws.d_max_s16 = max_s16;
  return decode_launch(a, max_s16, num_sms(dev), st, events, n_events);
}

// Prefill (batch a multiple of 128): the tensor-core path.  Layers are taken
// in chunks whose operand buffers fit kPrefillChunkBytes; each chunk is one set
// of operand preparations plus two grouped GEMM launches.  Chunks alternate
// between two halves of the workspace, and the preparation of chunk c + 1 runs
// on a side stream while the GEMMs of chunk c run on the caller's stream:
// preparation is memory-bound and needs no shared memory, so its CTAs run
// beside the GEMM's.  Events fork the side stream from the caller's stream and
// join it back before the call returns, so stream order (and graph capture)
// hold as for a single stream.
constexpr size_t kPrefillChunkBytes = (size_t)512 << 20;

cudaError_t ensure_side(Workspace& ws) {
  if (ws.side) return cudaSuccess;
  cudaError_t e = cudaStreamCreateWithFlags(&ws.side, cudaStreamNonBlocking);
  if (e != cudaSuccess) return e;
  cudaEvent_t* evs[] = {&ws.fork, &ws.join, &ws.prep_done[0], &ws.prep_done[1], &ws.gemm_done[0], &ws.gemm_done[1]};
  for (cudaEvent_t* ev : evs) {
    e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

lb_status prefill_launch(Workspace& ws, cudaStream_t st);

lb_status prefill_forward(const lb_layer* layers, int n, const void* const* xs, void* const* ys, int batch,
                          int x_bf16, int mode, cudaStream_t st, int tag) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& ws = g_ws[{dev, st, tag}];
  std::vector<unsigned char> key = call_key((char)('P' + 16 * mode), layers, n, xs, ys, batch, x_bf16);
  if (ws.buf && ws.key == key) return prefill_launch(ws, st);
  ws.key.clear();
  // plan the chunks: operand bytes per chunk (a workspace half) and table bytes
  std::vector<int> starts;
  size_t half = 0, cur = 0, tables = 0;
  long long tiles = 0;
  int cnt = 0;
  for (int i = 0; i < n; ++i) {
    const lb_layer& L = layers[i];
    const size_t b = lb::prefill_layer_bytes(batch, L.d_in, L.d_out, L.s, L.residual + 1);
    if (cnt == 0 || cur + b > kPrefillChunkBytes || cnt == lb::kPrefillMaxGroup) {
      if (cnt) {
        half = std::max(half, cur);
        tables += align_up(lb::prefill_table_bytes(cnt, tiles), 1024);
      }
      starts.push_back(i);
      cur = 0;
      cnt = 0;
      tiles = 0;
    }
    cur += b;
    tiles += lb::prefill_layer_tiles(batch, L.d_out, L.s, L.residual + 1);
    ++cnt;
  }
  half = align_up(std::max(half, cur), 1024);
  tables = align_up(tables + align_up(lb::prefill_table_bytes(cnt, tiles), 1024), 1024);
  starts.push_back(n);
  const int n_chunks = (int)starts.size() - 1;
  // workspace: [status][tables of all chunks][half 0][half 1]
  const size_t need = kStatusBytes + tables + (n_chunks > 1 ? 2 : 1) * half;

  if (ws.cap < need) {
    // the side stream always joins `st`, so waiting for `st` covers it
    const lb_status r = grow_workspace(ws, align_up(need + need / 8, 1 << 20), st);
    if (r != LB_OK) return r;
  }
  unsigned char* base = static_cast<unsigned char*>(ws.buf);
  unsigned char* table_dev = base + kStatusBytes;
  auto chunk_bufs = [&](int c) { return base + kStatusBytes + tables + (size_t)(c & 1) * half; };
  std::vector<lb::LayerDesc> descs(n);
  for (int i = 0; i < n; ++i) {
    const lb_layer& L = layers[i];
    lb::LayerDesc& D = descs[i];
    std::memset(&D, 0, sizeof(D));
    D.d_in = L.d_in;
    D.d_out = L.d_out;
    D.s = L.s;
    D.npaths = L.residual + 1;
    D.t_ld = lb::latent_row_elems(L.s, D.npaths);
    for (int p = 0; p < D.npaths; ++p) {
      D.p[p].V = static_cast<const uint4*>(L.path[p].V_bits);
      D.p[p].U = static_cast<const uint4*>(L.path[p].U_bits);
      D.p[p].h = L.path[p].h;
      D.p[p].g = L.path[p].g;
      D.p[p].l = L.path[p].l;
    }
  }
  // the tables of every chunk, uploaded only when they change (as the decode
  // table), so that a repeated call enqueues kernels and events only and can
  // be captured into a CUDA graph
  const int sms = num_sms(dev);
  int pair_slots = 0;
  const int perr = lb::prefill_pair_slots(&pair_slots);
  if (perr != 0) return cuda_fail((cudaError_t)perr);
  std::vector<unsigned char> img;
  std::vector<lb::PrefillPlan> plans(n_chunks);
  for (int c = 0; c < n_chunks; ++c)
    lb::plan_prefill_chunk(descs.data() + starts[c], xs + starts[c], ys + starts[c], starts[c + 1] - starts[c],
                           batch, x_bf16, mode, chunk_bufs(c), sms, pair_slots, img, plans[c]);
  if (img.size() > tables) return LB_ERR_SHAPE;   // the plan above sized the tables
  if (ws.table.size() != img.size() || std::memcmp(ws.table.data(), img.data(), img.size()) != 0) {
    // pageable source: the copy is staged before the call returns
    e = cudaMemcpyAsync(table_dev, img.data(), img.size(), cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e);
    ws.table.swap(img);
  }
  ws.p_plans.swap(plans);
  ws.key.swap(key);
  return prefill_launch(ws, st);
}

// The launches of a planned prefill call (plans and tables in ws).
lb_status prefill_launch(Workspace& ws, cudaStream_t st) {
  unsigned char* base = static_cast<unsigned char*>(ws.buf);
  unsigned int* status = reinterpret_cast<unsigned int*>(base);
  unsigned char* table_dev = base + kStatusBytes;
  const int n_chunks = (int)ws.p_plans.size();
  cudaError_t e;
  if (n_chunks == 1) {
    e = lb::launch_prefill_prep(ws.p_plans[0], table_dev, status, st);
    if (e != cudaSuccess) return cuda_fail(e);
    e = lb::launch_prefill_gemms(ws.p_plans[0], table_dev, status, st);
    return e == cudaSuccess ? LB_OK : cuda_fail(e);
  }
  e = ensure_side(ws);
  if (e != cudaSuccess) return cuda_fail(e);
  // fork: the side stream starts after everything already enqueued on `st`
  e = cudaEventRecord(ws.fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ws.side, ws.fork, 0);
  if (e != cudaSuccess) return cuda_fail(e);
  for (int c = 0; c < n_chunks && e == cudaSuccess; ++c) {
    const int h = c & 1;
    // the half was last used by chunk c - 2's GEMMs
    if (c >= 2) e = cudaStreamWaitEvent(ws.side, ws.gemm_done[h], 0);
    if (e == cudaSuccess) e = lb::launch_prefill_prep(ws.p_plans[c], table_dev, status, ws.side);
    if (e == cudaSuccess) e = cudaEventRecord(ws.prep_done[h], ws.side);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ws.prep_done[h], 0);
    if (e == cudaSuccess) e = lb::launch_prefill_gemms(ws.p_plans[c], table_dev, status, st);
    if (e == cudaSuccess) e = cudaEventRecord(ws.gemm_done[h], st);
  }
  // join, also after an error, so that no side-stream work outlives the call's stream order
  cudaError_t j = cudaEventRecord(ws.join, ws.side);
  if (j == cudaSuccess) j = cudaStreamWaitEvent(st, ws.join, 0);
  if (e == cudaSuccess) e = j;
  return e == cudaSuccess ? LB_OK : cuda_fail(e);
}


// State of littlebit_linear_forward_many_host per (device, stream): device
// copies of the whole stack's x and y, the two copy streams and the events
// that chain copy-in -> forward -> copy-out chunk by chunk.
struct HostPipe {
  unsigned char* x_dev = nullptr;
  unsigned char* y_dev = nullptr;
  size_t x_cap = 0, y_cap = 0;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t fork = nullptr, join_in = nullptr, join_out = nullptr;
  std::vector<cudaEvent_t> in_done, fwd_done;   // per chunk
  // the last call's plan (layers, batch, dtype, chunk count) and what follows
  std::vector<unsigned char> key;
  std::vector<int> starts;             // chunk c = layers starts[c] .. starts[c+1]-1
  std::vector<size_t> xo, yo;          // byte offsets of each layer's x and y; [n] = totals
  std::vector<const void*> xs;         // device views into x_dev / y_dev
  std::vector<void*> ys;
  // the pipeline of the last call, captured as a CUDA graph and replayed while
  // the calls repeat (same plan and host buffers): one launch per call
  // instead of a few dozen copy, event and kernel calls
  cudaGraphExec_t graph = nullptr;
  const void* g_x = nullptr;           // host buffers the graph copies from / to
  void* g_y = nullptr;
  int repeats = 0;                     // consecutive calls with this plan and these buffers
  bool no_graph = false;               // capture failed for this plan: enqueue eagerly
  bool key_changed_this_call = false;  // the plan was rebuilt by this call
};

std::mutex g_host_mu;   // taken before g_mu, never after it
std::map<std::pair<int, cudaStream_t>, HostPipe> g_pipes;

void drop_graph(HostPipe& hp) {
  if (hp.graph) cudaGraphExecDestroy(hp.graph);
  hp.graph = nullptr;
  hp.repeats = 0;
  hp.no_graph = false;
}

void release_pipe(HostPipe& hp) {
  drop_graph(hp);
  if (hp.x_dev) cudaFree(hp.x_dev);
  if (hp.y_dev) cudaFree(hp.y_dev);
  for (cudaEvent_t ev : {hp.fork, hp.join_in, hp.join_out})
    if (ev) cudaEventDestroy(ev);
  for (cudaEvent_t ev : hp.in_done) cudaEventDestroy(ev);
  for (cudaEvent_t ev : hp.fwd_done) cudaEventDestroy(ev);
  if (hp.h2d) cudaStreamDestroy(hp.h2d);
  if (hp.d2h) cudaStreamDestroy(hp.d2h);
  hp = HostPipe();
}

cudaError_t ensure_pipe_objects(HostPipe& hp, int n_chunks) {
  cudaError_t e = cudaSuccess;
  if (!hp.h2d) e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess && !hp.d2h) e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
  for (cudaEvent_t* ev : {&hp.fork, &hp.join_in, &hp.join_out})
    if (e == cudaSuccess && !*ev) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  while (e == cudaSuccess && (int)hp.in_done.size() < n_chunks) {
    cudaEvent_t a = nullptr, b = nullptr;
    e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      if (a) cudaEventDestroy(a);
      break;
    }
    hp.in_done.push_back(a);
    hp.fwd_done.push_back(b);
  }
  return e;
}

// Cut layers 0..n-1 into `chunks` consecutive groups of about equal x + y bytes.
std::vector<int> chunk_starts(const std::vector<size_t>& xo, const std::vector<size_t>& yo, int n, int chunks) {
  std::vector<int> starts{0};
  const double total = (double)(xo[n] + yo[n]);
  for (int c = 1; c < chunks; ++c) {
    const double target = total * c / chunks;
    int i = starts.back() + 1;
    while (i < n && (double)(xo[i] + yo[i]) < target) ++i;
    if (i >= n) break;
    starts.push_back(i);
  }
  starts.push_back(n);
  return starts;
}

// Host-checkable conditions of a forward call, before any device work.
lb_status check_call(const lb_layer* layers, int n, int batch, lb_dtype xdt) {
  if (batch < 1) return LB_ERR_SHAPE;
  for (int i = 0; i < n; ++i) {
    const lb_status st = check_layer(layers[i]);
    if (st != LB_OK) return st;
  }
  if (batch <= lb::kMaxBatchDecode) return xdt == LB_F16 ? LB_OK : LB_ERR_UNSUPPORTED;
  if (xdt != LB_F16 && xdt != LB_BF16) return LB_ERR_UNSUPPORTED;
  // operand preparation indexes one layer's fp16 copy of x with 32-bit offsets
  for (int i = 0; i < n; ++i)
    if ((size_t)batch * layers[i].d_in > ((size_t)1 << 30)) return LB_ERR_SHAPE;
  if (batch % 128 != 0 && xdt != LB_F16) return LB_ERR_UNSUPPORTED;
  return LB_OK;
}

// The forward of a checked call on `st`, with the workspaces of tag base
// `base`: batch <= 16 on the decode path, a multiple of 128 on the prefill
// path, any other batch (fp16) the leading multiple of 128 rows through the
// prefill path and the rest through the decode path in groups of at most 16
// rows (rows are contiguous in the inputs and outputs, so a group is an
// offset view).  `mode` (CallMode) selects the whole forward or one of its
// halves around the latent cache rows.
lb_status forward_dispatch(const lb_layer* layers, int n, const void* const* xs, void* const* ys, int batch,
                           lb_dtype xdt, int mode, cudaStream_t st, const cudaEvent_t* evs, int n_events,
                           int base) {
  if (batch <= lb::kMaxBatchDecode)
    return decode_forward(layers, n, xs, ys, batch, mode, st, evs, n_events, ws_tag(base, 1));
  if (batch % 128 == 0)
    return prefill_forward(layers, n, xs, ys, batch, xdt == LB_BF16 ? 1 : 0, mode, st, ws_tag(base, 0));
  std::vector<const void*> xv(n);
  std::vector<void*> yv(n);
  // bytes per row of each layer's input and output (2-byte elements)
  auto in_row = [&](int i) -> size_t {
    return 2 * (size_t)(mode == lb::kModeExpand ? lb::latent_row_elems(layers[i].s, layers[i].residual + 1)
                                                : layers[i].d_in);
  };
  auto out_row = [&](int i) -> size_t {
    return 2 * (size_t)(mode == lb::kModeLatent ? lb::latent_row_elems(layers[i].s, layers[i].residual + 1)
                                                : layers[i].d_out);
  };
  auto views = [&](int r0) {
    for (int i = 0; i < n; ++i) {
      xv[i] = static_cast<const unsigned char*>(xs[i]) + (size_t)r0 * in_row(i);
      yv[i] = static_cast<unsigned char*>(ys[i]) + (size_t)r0 * out_row(i);
    }
  };
  const int m128 = batch / 128 * 128;
  if (m128 > 0) {
    const lb_status r = prefill_forward(layers, n, xs, ys, m128, 0, mode, st, ws_tag(base, 0));
    if (r != LB_OK) return r;
  }
  for (int r0 = m128, grp = 0; r0 < batch; r0 += lb::kMaxBatchDecode, ++grp) {
    views(r0);
    const int rows = std::min(lb::kMaxBatchDecode, batch - r0);
    const lb_status r = decode_forward(layers, n, xv.data(), yv.data(), rows, mode, st,
                                       r0 == m128 ? evs : nullptr, r0 == m128 ? n_events : 0, ws_tag(base, 1 + grp));
    if (r != LB_OK) return r;
  }
  return LB_OK;
}

// Checks of a device-pointer call's buffers, then the dispatch.
lb_status checked_forward(const lb_layer* layers, int n, const void* const* xs, void* const* ys, int batch,
                          lb_dtype xdt, int mode, void* stream, const cudaEvent_t* evs, int n_events) {
  if (!layers || !xs || !ys || n < 1) return LB_ERR_ARG;
  const lb_status chk = check_call(layers, n, batch, xdt);
  if (chk != LB_OK) return chk;
  for (int i = 0; i < n; ++i) {
    if (!xs[i] || !ys[i]) return LB_ERR_ARG;
    if (!aligned(xs[i], 16) || !aligned(ys[i], 16)) return LB_ERR_ALIGN;
  }
  return forward_dispatch(layers, n, xs, ys, batch, xdt, mode, static_cast<cudaStream_t>(stream), evs, n_events,
                          0);
}

// Page-locked host memory (cudaHostAlloc or cudaHostRegister): the copies of a
// captured graph need it.
bool pinned(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost;
}

// The copies and forwards of a planned host-buffer call on `st`: both copy
// streams start after everything already on `st` (so x_dev, y_dev and the
// host buffers are free), and `st` ends after both.
lb_status enqueue_pipe(HostPipe& hp, const lb_layer* layers, int batch, lb_dtype xdt, const void* x_host,
                       void* y_host, cudaStream_t st) {
  const int chunks = (int)hp.starts.size() - 1;
  cudaError_t e;
  e = cudaEventRecord(hp.fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.h2d, hp.fork, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.d2h, hp.fork, 0);
  if (e != cudaSuccess) return cuda_fail(e);
  const unsigned char* xh = static_cast<const unsigned char*>(x_host);
  unsigned char* yh = static_cast<unsigned char*>(y_host);
  lb_status r = LB_OK;
  for (int c = 0; c < chunks && r == LB_OK; ++c) {
    const int i0 = hp.starts[c], i1 = hp.starts[c + 1];
    e = cudaMemcpyAsync(hp.x_dev + hp.xo[i0], xh + hp.xo[i0], hp.xo[i1] - hp.xo[i0], cudaMemcpyHostToDevice,
                        hp.h2d);
    if (e == cudaSuccess) e = cudaEventRecord(hp.in_done[c], hp.h2d);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, hp.in_done[c], 0);
    if (e != cudaSuccess) {
      r = cuda_fail(e);
      break;
    }
    r = forward_dispatch(layers + i0, i1 - i0, hp.xs.data() + i0, hp.ys.data() + i0, batch, xdt, lb::kModeForward,
                         st, nullptr, 0, c + 1);
    if (r != LB_OK) break;
    e = cudaEventRecord(hp.fwd_done[c], st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.d2h, hp.fwd_done[c], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(yh + hp.yo[i0], hp.y_dev + hp.yo[i0], hp.yo[i1] - hp.yo[i0], cudaMemcpyDeviceToHost,
                          hp.d2h);
    if (e != cudaSuccess) r = cuda_fail(e);
  }
  // join on every path, so that `st` always covers the copies it started
  e = cudaEventRecord(hp.join_in, hp.h2d);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, hp.join_in, 0);
  if (e == cudaSuccess) e = cudaEventRecord(hp.join_out, hp.d2h);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, hp.join_out, 0);
  if (e != cudaSuccess && r == LB_OK) r = cuda_fail(e);
  return r;
}


}  // namespace

extern "C" {

size_t littlebit_packed_bytes(lb_role role, int rows, int cols) {
  if (rows < 1 || cols < 1) return 0;
  const int tr = (role == LB_ROLE_V) ? lb::kVTileRows : lb::kUTileRows;
  const int tk = (role == LB_ROLE_V) ? lb::kVTileK : lb::kUTileK;
  return (size_t)lb::ceil_div(rows, tr) * lb::ceil_div(cols, tk) * lb::kTileBytes;
}

double littlebit_eff_bits(int d_in, int d_out, int s, int residual) {
  const double a = d_in, b = d_out;
  const double num = residual ? 2.0 * s * (a + b + 16) + 32.0 * (a + b) : (double)s * (a + b + 16) + 16.0 * (a + b);
  return num / (a * b);
}

lb_status littlebit_pack_signs(const void* src_dev, lb_dtype dt, int n_long, int s, int64_t stride_long,
                               int64_t stride_s, lb_role role, void* dst_dev, void* stream) {
  if (!src_dev || !dst_dev) return LB_ERR_ARG;
  if (dt != LB_F16 && dt != LB_BF16 && dt != LB_F32 && dt != LB_I8) return LB_ERR_ARG;
  if (role != LB_ROLE_V && role != LB_ROLE_U) return LB_ERR_ARG;
  if (n_long < 1 || s < 1) return LB_ERR_SHAPE;
  if (!aligned(dst_dev, 16)) return LB_ERR_ALIGN;
  cudaError_t e = lb::launch_pack(src_dev, dt, n_long, s, stride_long, stride_s, role, dst_dev,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LB_OK : cuda_fail(e);
}

lb_status littlebit_unpack_signs(const void* src_dev, lb_role role, int n_long, int s, int8_t* dst_dev,
                                 void* stream) {
  if (!src_dev || !dst_dev) return LB_ERR_ARG;
  if (role != LB_ROLE_V && role != LB_ROLE_U) return LB_ERR_ARG;
  if (n_long < 1 || s < 1) return LB_ERR_SHAPE;
  if (!aligned(src_dev, 16)) return LB_ERR_ALIGN;
  cudaError_t e = lb::launch_unpack(src_dev, n_long, s, role, dst_dev, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LB_OK : cuda_fail(e);
}

lb_status littlebit_linear_forward_many_timed(const lb_layer* layers, int n, const void* const* xs,
                                              void* const* ys, int batch, lb_dtype xdt, void* stream,
                                              void* const* events, int n_events) {
  return checked_forward(layers, n, xs, ys, batch, xdt, lb::kModeForward, stream,
                         reinterpret_cast<const cudaEvent_t*>(events), n_events);
}

int littlebit_latent_row_elems(int s, int residual) {
  if (s < 1 || s > lb::kMaxRank || (residual != 0 && residual != 1)) return 0;
  return lb::latent_row_elems(s, residual + 1);
}

lb_status littlebit_latent_forward(const lb_layer* layers, int n, const void* const* xs, void* const* ts,
                                   int batch, lb_dtype xdt, void* stream) {
  return checked_forward(layers, n, xs, ts, batch, xdt, lb::kModeLatent, stream, nullptr, 0);
}

lb_status littlebit_latent_expand(const lb_layer* layers, int n, const void* const* ts, void* const* ys, int rows,
                                  lb_dtype ydt, void* stream) {
  return checked_forward(layers, n, ts, ys, rows, ydt, lb::kModeExpand, stream, nullptr, 0);
}

lb_status littlebit_linear_forward_many(const lb_layer* layers, int n, const void* const* xs, void* const* ys,
                                        int batch, lb_dtype xdt, void* stream) {
  return littlebit_linear_forward_many_timed(layers, n, xs, ys, batch, xdt, stream, nullptr, 0);
}

lb_status littlebit_linear_forward(const lb_layer* layer, const void* x_dev, void* y_dev, int batch,
                                   lb_dtype xdt, void* stream) {
  return littlebit_linear_forward_many(layer, 1, &x_dev, &y_dev, batch, xdt, stream);
}

lb_status littlebit_device_status(void* stream, unsigned int* status) {
  if (!status) return LB_ERR_ARG;
  *status = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_mu);
  // every workspace of this stream (all tags): their status words, OR-ed
  for (auto it = g_ws.lower_bound({dev, st, INT_MIN}); it != g_ws.end(); ++it) {
    if (std::get<0>(it->first) != dev || std::get<1>(it->first) != st) break;
    if (!it->second.buf) continue;
    unsigned int bits = 0;
    e = cudaMemcpy(&bits, it->second.buf, sizeof(bits), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (bits) {
      e = cudaMemset(it->second.buf, 0, sizeof(unsigned int));
      if (e != cudaSuccess) return cuda_fail(e);
    }
    *status |= bits;
  }
  // the allocation-free forward's word on this device (any stream)
  unsigned int* word = lb::noalloc_status_word(dev);
  if (word) {
    unsigned int bits = 0;
    e = cudaMemcpy(&bits, word, sizeof(bits), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (bits) {
      e = cudaMemset(word, 0, sizeof(unsigned int));
      if (e != cudaSuccess) return cuda_fail(e);
    }
    *status |= bits;
  }
  return LB_OK;
}

lb_status littlebit_check_wait_timeout(void* stream, int polls) {
  if (polls < 1 || polls > lb::kSpinLimit) return LB_ERR_ARG;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& ws = g_ws[{dev, st, ws_tag(0, 1)}];   // the decode workspace of the device API
  if (!ws.buf) {
    // just the status word; a later forward grows the workspace
    const lb_status r = grow_workspace(ws, kStatusBytes, st);
    if (r != LB_OK) return r;
  }
  e = lb::launch_wait_timeout_probe(static_cast<unsigned int*>(ws.buf), polls, st);
  return e == cudaSuccess ? LB_OK : cuda_fail(e);
}

lb_status littlebit_linear_forward_many_host(const lb_layer* layers, int n, const void* x_host, void* y_host,
                                             int batch, lb_dtype xdt, int n_chunks, void* stream) {
  if (!layers || n < 1 || !x_host || !y_host || n_chunks < 1) return LB_ERR_ARG;
  const lb_status chk = check_call(layers, n, batch, xdt);
  if (chk != LB_OK) return chk;
  n_chunks = std::min(std::min(n_chunks, n), kMaxHostChunks);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostPipe& hp = g_pipes[{dev, st}];

  // ---- plan: offsets, chunks, device views (reused while the call repeats)
  std::vector<unsigned char> key((size_t)n * sizeof(lb_layer) + 12);
  std::memcpy(key.data(), &batch, 4);
  std::memcpy(key.data() + 4, &xdt, 4);
  std::memcpy(key.data() + 8, &n_chunks, 4);
  std::memcpy(key.data() + 12, layers, (size_t)n * sizeof(lb_layer));
  if (hp.key != key) {
    hp.key.clear();
    hp.xo.assign(n + 1, 0);
    hp.yo.assign(n + 1, 0);
    for (int i = 0; i < n; ++i) {   // 2-byte elements; d_in % 256 == 0 and d_out % 128 == 0 keep 256-byte steps
      hp.xo[i + 1] = hp.xo[i] + (size_t)batch * layers[i].d_in * 2;
      hp.yo[i + 1] = hp.yo[i] + (size_t)batch * layers[i].d_out * 2;
    }
    if (hp.x_cap < hp.xo[n] || hp.y_cap < hp.yo[n]) {
      e = cudaStreamSynchronize(st);   // every earlier call on `st` joined its copies into `st`
      if (e != cudaSuccess) return cuda_fail(e);
      if (hp.x_cap < hp.xo[n]) {
        if (hp.x_dev) cudaFree(hp.x_dev);
        hp.x_dev = nullptr;
        hp.x_cap = 0;
        e = cudaMalloc(&hp.x_dev, hp.xo[n]);
        if (e != cudaSuccess) return cuda_fail(e);
        hp.x_cap = hp.xo[n];
      }
      if (hp.y_cap < hp.yo[n]) {
        if (hp.y_dev) cudaFree(hp.y_dev);
        hp.y_dev = nullptr;
        hp.y_cap = 0;
        e = cudaMalloc(&hp.y_dev, hp.yo[n]);
        if (e != cudaSuccess) return cuda_fail(e);
        hp.y_cap = hp.yo[n];
      }
    }
    hp.xs.resize(n);
    hp.ys.resize(n);
    for (int i = 0; i < n; ++i) {
      hp.xs[i] = hp.x_dev + hp.xo[i];
      hp.ys[i] = hp.y_dev + hp.yo[i];
    }
    hp.starts = chunk_starts(hp.xo, hp.yo, n, n_chunks);
    hp.key = key;
    hp.key_changed_this_call = true;
  }
  const int chunks = (int)hp.starts.size() - 1;
  e = ensure_pipe_objects(hp, chunks);
  if (e != cudaSuccess) return cuda_fail(e);

  // the graph's copies need the same, still page-locked, host buffers
  const bool locked = pinned(x_host) && pinned(y_host);
  if (hp.key_changed_this_call || hp.g_x != x_host || hp.g_y != y_host || !locked) {
    drop_graph(hp);
    hp.g_x = x_host;
    hp.g_y = y_host;
  }
  hp.key_changed_this_call = false;
  if (hp.graph) {
    e = cudaGraphLaunch(hp.graph, st);
    return e == cudaSuccess ? LB_OK : cuda_fail(e);
  }
  // capture from the second identical call on (the first has settled every
  // workspace and table, so the enqueue allocates and uploads nothing), with
  // page-locked buffers and a stream that is not already being captured
  ++hp.repeats;
  if (hp.repeats >= 2 && !hp.no_graph && locked) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cs);
    if (e == cudaSuccess && cs == cudaStreamCaptureStatusNone) {
      e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
      lb_status r = e == cudaSuccess ? enqueue_pipe(hp, layers, batch, xdt, x_host, y_host, st) : LB_ERR_CUDA;
      cudaGraph_t g = nullptr;
      const cudaError_t ee = e == cudaSuccess ? cudaStreamEndCapture(st, &g) : e;
      cudaGraphExec_t ex = nullptr;
      if (r == LB_OK && ee == cudaSuccess && g && cudaGraphInstantiate(&ex, g, 0) == cudaSuccess) {
        hp.graph = ex;
      } else {
        hp.no_graph = true;
      }
      if (g) cudaGraphDestroy(g);
      (void)cudaGetLastError();   // a refused capture leaves no sticky error
      if (hp.graph) {
        e = cudaGraphLaunch(hp.graph, st);
        return e == cudaSuccess ? LB_OK : cuda_fail(e);
      }
    } else {
      (void)cudaGetLastError();
    }
  }
  return enqueue_pipe(hp, layers, batch, xdt, x_host, y_host, st);
}

void littlebit_release(void) {
  std::lock_guard<std::mutex> host_lock(g_host_mu);
  for (auto& kv : g_pipes) release_pipe(kv.second);
  g_pipes.clear();
  std::lock_guard<std::mutex> lock(g_mu);
  for (auto& kv : g_ws) release_workspace(kv.second);
  g_ws.clear();
}

const char* littlebit_status_string(lb_status st) {
  switch (st) {
    case LB_OK: return "LB_OK";
    case LB_ERR_ARG: return "LB_ERR_ARG: invalid argument";
    case LB_ERR_ALIGN: return "LB_ERR_ALIGN: pointer misaligned";
    case LB_ERR_SHAPE: return "LB_ERR_SHAPE: unsupported shape";
    case LB_ERR_CUDA: return "LB_ERR_CUDA: CUDA runtime error";
    case LB_ERR_TIMEOUT: return "LB_ERR_TIMEOUT: device wait timed out";
    case LB_ERR_UNSUPPORTED: return "LB_ERR_UNSUPPORTED: not implemented for these arguments";
    case LB_ERR_RANGE: return "LB_ERR_RANGE: a value left the range of its format";
  }
  return "unknown lb_status";
}

const char* littlebit_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
