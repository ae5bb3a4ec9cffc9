// api_host.cu -- the host-buffer layer of the C ABI (include/moe.h): token
// chunks whose copies in and out run on two library-owned copy streams while
// the layer runs on the neighbouring chunk.
#include <algorithm>
#include <mutex>

#include "api_detail.h"

namespace moe {
namespace api {

// ---- host-buffer layer: token chunks pipelined over two copy streams
//
// Without a capacity limit a token's output depends on that token alone, so
// the batch is cut into n token chunks: the copy of chunk i+1 to the device
// and of chunk i-1 back to the host overlap the layer on chunk i.  Staging buffers are double-buffered in the workspace.  With a capacity
// limit the drops depend on every token's rank, so the batch is one chunk.
constexpr int kDefaultHostChunks = 3;  // measured best on the Mixtral-shaped layer (2..8 tried)

struct HostPipe {
  bool made = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, h2d_done[2] = {nullptr, nullptr}, comp_done[2] = {nullptr, nullptr},
              d2h_done[2] = {nullptr, nullptr};
};
std::mutex g_pipe_mutex[kMaxDevices];
HostPipe g_pipe[kMaxDevices];

bool make_pipe(HostPipe& p) {
  if (p.made) return true;
  bool ok = cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess;
  for (int b = 0; ok && b < 2; ++b)
    ok = cudaEventCreateWithFlags(&p.h2d_done[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.comp_done[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.d2h_done[b], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return false;
  }
  p.made = true;
  return true;
}

constexpr int kMaxHostChunks = 64;

struct HostLayout {
  int n;                         // chunks
  int64_t start[kMaxHostChunks + 1];  // token offsets of the chunks
  int64_t tc;                    // tokens of the largest chunk
  size_t layer;                  // bytes of the per-chunk layer workspace (at offset 0)
  size_t xs[2], os[2], total;
};

// Chunk sizes in the ratio 1 : 4 : ... : 4 : 1: only the first chunk's copy
// in and the last chunk's copy out are not hidden behind compute, so those two
// are small; a middle chunk's copy (4 units) then takes about as long as an
// end chunk's compute.  Measured on the Mixtral-shaped layer with 3 chunks:
// 1:2:1 10.74 ms, 1:3:1 10.87 ms, 1:4:1 10.42 ms end to end.
HostLayout host_layout_of(const moe_config_t& c, int n_chunks) {
  HostLayout H{};
  int n = n_chunks > 0 ? n_chunks : kDefaultHostChunks;
  if (capacity_of(c) >= 0) n = 1;          // capacity ranks span the whole batch
  if (n > kMaxHostChunks) n = kMaxHostChunks;
  if (n > c.T) n = c.T > 0 ? c.T : 1;
  const int64_t wsum = n <= 2 ? n : 4 * (n - 2) + 2;
  int64_t acc = 0;
  H.start[0] = 0;
  for (int i = 0; i < n; ++i) {
    acc += (n <= 2 || i == 0 || i == n - 1) ? 1 : 4;
    H.start[i + 1] = (static_cast<int64_t>(c.T) * acc) / wsum;
  }
  for (int i = 1; i < n; ++i)  // no empty chunk (n <= T leaves room for one token each)
    H.start[i] = std::min<int64_t>(std::max<int64_t>(H.start[i], H.start[i - 1] + 1), c.T - (n - i));
  H.n = n;
  H.tc = 0;
  for (int i = 0; i < n; ++i) H.tc = std::max<int64_t>(H.tc, H.start[i + 1] - H.start[i]);
  moe_config_t cc = c;
  cc.T = static_cast<int32_t>(H.tc);
  H.layer = align_up(layout_of(cc).total, 1024);
  const size_t chunk_bytes = align_up(static_cast<size_t>(H.tc) * c.d_model * 2, 1024);
  size_t off = H.layer;
  for (int b = 0; b < 2; ++b) { H.xs[b] = off; off += chunk_bytes; }
  for (int b = 0; b < 2; ++b) { H.os[b] = off; off += chunk_bytes; }
  H.total = off;
  return H;
}

}  // namespace api
}  // namespace moe

using namespace moe;
using namespace moe::api;

extern "C" {

size_t moe_host_workspace_size(const moe_config_t* cfg, int32_t n_chunks) {
  if (validate(cfg) != MOE_OK) return 0;
  return host_layout_of(*cfg, n_chunks).total;
}

int32_t moe_host_chunks(const moe_config_t* cfg, int32_t n_chunks) {
  if (validate(cfg) != MOE_OK) return -1;
  return host_layout_of(*cfg, n_chunks).n;
}

moe_status_t moe_layer_fwd_host(const moe_config_t* cfg, const moe_bf16_t* x_host, const moe_bf16_t* gamma,
                                const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                                const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out_host,
                                int32_t n_chunks, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T == 0) return MOE_OK;
  if (!x_host || !gamma || !Wr || !W1 || !W3 || !W2 || !out_host) return MOE_ERR_INVALID_ARG;
  if (!aligned(gamma, 16) || !aligned(Wr, 2) || !aligned(bias, 4) || !aligned(W1, 16) || !aligned(W3, 16) ||
      !aligned(W2, 16) || !aligned(x_host, 2) || !aligned(out_host, 2))
    return MOE_ERR_ALIGNMENT;
  const HostLayout H = host_layout_of(c, n_chunks);
  if (ws == nullptr || ws_bytes < H.total) return MOE_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_pipe_mutex[dev]);
  HostPipe& P = g_pipe[dev];
  if (!make_pipe(P)) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = static_cast<size_t>(c.d_model) * 2;
  const char* xh = reinterpret_cast<const char*>(x_host);
  char* oh = reinterpret_cast<char*>(out_host);
  cudaError_t e = cudaEventRecord(P.start, s);  // copies start after earlier work on `stream`
  if (e == cudaSuccess) e = cudaStreamWaitEvent(P.h2d, P.start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(P.d2h, P.start, 0);
  if (e != cudaSuccess) return cuda_status(e);
  for (int i = 0; i < H.n; ++i) {
    const int b = i & 1;
    const int64_t t0 = H.start[i];
    const int64_t ti = H.start[i + 1] - t0;  // >= 1: n <= T
    moe_config_t ci = c;
    ci.T = static_cast<int32_t>(ti);
    const Layout Li = layout_of(ci);
    moe_bf16_t* xs = at<moe_bf16_t>(ws, H.xs[b]);
    moe_bf16_t* os = at<moe_bf16_t>(ws, H.os[b]);
    const size_t bytes = static_cast<size_t>(ti) * row_bytes;
    if (i >= 2) e = cudaStreamWaitEvent(P.h2d, P.comp_done[b], 0);  // xs[b] read by chunk i-2
    if (e == cudaSuccess) e = cudaMemcpyAsync(xs, xh + t0 * row_bytes, bytes, cudaMemcpyHostToDevice, P.h2d);
    if (e == cudaSuccess) e = cudaEventRecord(P.h2d_done[b], P.h2d);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, P.h2d_done[b], 0);
    if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(s, P.d2h_done[b], 0);  // os[b] copied out
    if (e != cudaSuccess) return cuda_status(e);
    // the chunk's layer workspace: the error word lives in its header (offset 0)
    if ((st = run_layer(ci, Li, ws, xs, gamma, Wr, bias, W1, W3, W2, os, nullptr, nullptr, nullptr, nullptr,
                        nullptr, nullptr, sms, s)) != MOE_OK)
      return st;
    e = cudaEventRecord(P.comp_done[b], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(P.d2h, P.comp_done[b], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(oh + t0 * row_bytes, os, bytes, cudaMemcpyDeviceToHost, P.d2h);
    if (e == cudaSuccess) e = cudaEventRecord(P.d2h_done[b], P.d2h);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // the caller's stream completes after the last copies out
  e = cudaStreamWaitEvent(s, P.d2h_done[(H.n - 1) & 1], 0);
  if (e == cudaSuccess && H.n >= 2) e = cudaStreamWaitEvent(s, P.d2h_done[H.n & 1], 0);
  return cuda_status(e);
}

}  // extern "C"
