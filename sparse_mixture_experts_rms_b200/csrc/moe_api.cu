// moe_api.cu -- the C ABI declared in include/moe.h: argument validation,
// workspace layout, TMA descriptor encoding and launch sequencing on one
// stream.  Allocates nothing; never synchronises except in
// moe_get_device_error.
#include <cmath>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;
constexpr size_t kHeaderBytes = 256;

struct DeviceState {
  bool ready = false;
  bool ok = false;
  int sms = 0;
  int gemm_grid = 0;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;
bool g_encode_tried = false;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Layout {
  size_t err, ticket, rw, prob_partial, prob_mean, tile_counts, r, idx, gate, counts, offsets, perm,
      inv_perm, x_perm, H, y, total;
  // training workspace only
  size_t logits, U, V, yu, dY, dS, dS3, drp, dXp, dgate, rdl, dr, dbias_part, dgamma_part, dWr_part;
  // MXFP8 workspace only
  size_t x8, xsf, h8, hsf;
  int64_t max_kept;  // rows of the permuted buffers (padded in the training layout)
  int ldh;
  int ld_drp, chunks, chunk_tokens, route_blocks;
  bool train;
  bool mx;
};

constexpr int kTrainRowAlign = 64;  // row-segment padding of the training layout
constexpr int kMxRowAlign = 128;    // MX path: a CTA's 128 rows are one scale block

int64_t capacity_of(const moe_config_t& c) {
  if (!(c.capacity_factor > 0.0f)) return -1;
  const double v = static_cast<double>(c.T) * c.k / c.E * static_cast<double>(c.capacity_factor);
  const double tk = static_cast<double>(c.T) * c.k;
  return static_cast<int64_t>(std::floor(v < tk ? v : tk));
}

int64_t max_kept_of(const moe_config_t& c) {
  const int64_t tk = static_cast<int64_t>(c.T) * c.k;
  const int64_t cap = capacity_of(c);
  if (cap < 0) return tk;
  const int64_t ec = cap * c.E;
  return ec < tk ? ec : tk;
}

moe_status_t validate(const moe_config_t* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d_model <= 0 || c->E <= 0 || c->k <= 0 || c->k > c->E) return MOE_ERR_INVALID_ARG;
  if (c->d_model % 128 != 0) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(c->eps) || c->eps < 0.0f) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(c->capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (c->ffn_offsets == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(c->T) * c->k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (c->ffn_offsets[0] != 0) return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < c->E; ++e) {
    const int64_t w = static_cast<int64_t>(c->ffn_offsets[e + 1]) - c->ffn_offsets[e];
    if (w <= 0 || w % kBlockN != 0) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

Layout layout_of(const moe_config_t& c, bool train = false, bool mx = false) {
  Layout L{};
  L.train = train;
  L.mx = mx;
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes > 0 ? bytes : 1, 1024);
    return o;
  };
  const size_t tk = static_cast<size_t>(c.T) * c.k;
  const size_t ntiles = (tk + kDispatchTile - 1) / kDispatchTile;
  int fmax = 0;
  for (int e = 0; e < c.E; ++e) {
    const int w = c.ffn_offsets[e + 1] - c.ffn_offsets[e];
    fmax = w > fmax ? w : fmax;
  }
  L.max_kept = max_kept_of(c) + (train ? static_cast<int64_t>(c.E) * (kTrainRowAlign - 1) : 0);
  if (mx) L.max_kept = (max_kept_of(c) + static_cast<int64_t>(c.E) * (kMxRowAlign - 1) + 127) / 128 * 128;
  L.ldh = fmax;
  const size_t mk = static_cast<size_t>(L.max_kept);
  L.err = 0;
  L.ticket = 4;  // second word of the header
  L.rw = take(static_cast<size_t>(c.d_model) * kRouterPadE * 4);
  L.prob_partial = take(static_cast<size_t>((c.T + kRouteTok - 1) / kRouteTok) * c.E * 4);
  L.prob_mean = take(static_cast<size_t>(c.E) * 4);
  L.tile_counts = take(ntiles * c.E * 4);
  L.r = take(static_cast<size_t>(c.T) * 4);
  L.idx = take(tk * 4);
  L.gate = take(tk * 4);
  L.counts = take(static_cast<size_t>(c.E) * 4);
  L.offsets = take(static_cast<size_t>(c.E + 1) * 4);
  L.perm = take(mk * 4);
  L.inv_perm = take(tk * 4);
  if (mx) {
    const size_t d = static_cast<size_t>(c.d_model);
    L.x8 = take(mk * d);
    L.xsf = take((mk / 128) * (d / 128) * 512);
    L.h8 = take(mk * static_cast<size_t>(fmax));
    L.hsf = take((mk / 128) * (static_cast<size_t>(fmax) / 128) * 512);
  } else {
    L.x_perm = take(mk * c.d_model * 2);
    L.H = take(mk * static_cast<size_t>(fmax) * 2);
  }
  L.y = take(mk * c.d_model * 2);
  if (train) {
    const size_t T = static_cast<size_t>(c.T), d = static_cast<size_t>(c.d_model);
    const size_t E = static_cast<size_t>(c.E);
    L.ld_drp = fmax / kBlockN;  // one dr partial per N tile of the dS GEMM
    L.route_blocks = (c.T + kBwdRouteTokens - 1) / kBwdRouteTokens;
    // bwd_norm grid: d/128 column slices x chunks, about 1024 CTAs
    const int slices = c.d_model / kBwdNormCols;
    int chunks = (1024 + slices - 1) / slices;
    const int max_chunks = (c.T + 31) / 32;
    chunks = chunks < max_chunks ? chunks : max_chunks;
    L.chunks = chunks > 0 ? chunks : 1;
    L.chunk_tokens = (c.T + L.chunks - 1) / L.chunks;
    L.logits = take(T * E * 4);
    L.U = take(mk * static_cast<size_t>(fmax) * 2);
    L.V = take(mk * static_cast<size_t>(fmax) * 2);
    L.yu = take(mk * d * 2);
    L.dY = take(mk * d * 2);
    L.dS = take(mk * static_cast<size_t>(fmax) * 2);
    L.dS3 = take(mk * static_cast<size_t>(fmax) * 2);
    L.drp = take(mk * static_cast<size_t>(L.ld_drp) * 4);
    L.dXp = take(mk * d * 4);
    L.dgate = take(tk * 4);
    L.rdl = take(T * E * 4);
    L.dr = take(T * 4);
    L.dbias_part = take(static_cast<size_t>(L.route_blocks) * E * 4);
    L.dgamma_part = take(static_cast<size_t>(L.chunks) * d * 4);
    L.dWr_part = take(static_cast<size_t>(L.chunks) * d * E * 4);
  }
  L.total = off;
  return L;
}

moe_status_t check_ws(const moe_config_t& c, void* ws, size_t ws_bytes, Layout* L, bool train = false,
                      bool mx = false) {
  *L = layout_of(c, train, mx);
  if (ws == nullptr || ws_bytes < L->total) return MOE_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

moe_status_t device_ready(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    st.ready = true;
    st.ok = false;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_NO_DEVICE;
    }
    if (prop.major != 10) return MOE_ERR_NO_DEVICE;
    if (prepare_grouped_gemm() != cudaSuccess || prepare_grouped_gemm_mx() != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    if (!g_encode_tried) {
      g_encode_tried = true;
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
              cudaSuccess &&
          q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      cudaGetLastError();
    }
    if (g_encode == nullptr) return MOE_ERR_CUDA;
    st.sms = prop.multiProcessorCount;
    st.gemm_grid = grouped_gemm_max_grid(st.sms);
    if (st.gemm_grid < 2) return MOE_ERR_CUDA;
    st.ok = true;
  }
  if (!st.ok) return MOE_ERR_NO_DEVICE;
  *sms = st.sms;
  return MOE_OK;
}

int gemm_grid_of_current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_mutex);
  return g_dev[dev].gemm_grid;
}

// 2-D bf16 tensor map with 128-byte swizzle: `inner` contiguous elements per
// row, `outer` rows, `row_elems` elements between rows; box inner x outer.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_elems,
              uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_elems * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D E4M3 (byte) tensor map, 128-byte swizzle, box inner x outer.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MX scale blocks as a [nblocks, 128] array of 32-bit words; one block per box.
bool make_map_sf(CUtensorMap* m, const void* base, uint64_t nblocks) {
  const cuuint64_t dims[2] = {128, nblocks};
  const cuuint64_t strides[1] = {512};
  const cuuint32_t box[2] = {128, 1};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

moe_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  cudaGetLastError();
  return MOE_ERR_CUDA;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status_t run_route(const moe_config_t& c, const moe_bf16_t* x, const moe_bf16_t* gamma,
                       const moe_bf16_t* Wr, const float* bias, int32_t* idx, float* gate, float* r,
                       float* logits, float* prob_mean, const Layout& L, void* ws, cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  RouteArgs a{};
  a.wprime = at<float>(ws, L.rw);
  a.err = at<uint32_t>(ws, L.err);
  a.prob_mean = prob_mean;
  a.prob_partial = at<float>(ws, L.prob_partial);
  a.ticket = at<unsigned>(ws, L.ticket);
  if (prob_mean != nullptr) {
    cudaError_t e = cudaMemsetAsync(a.ticket, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return cuda_status(e);
  }
  a.x = reinterpret_cast<const __nv_bfloat16*>(x);
  a.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  a.Wr = reinterpret_cast<const __nv_bfloat16*>(Wr);
  a.bias = bias;
  a.idx = idx;
  a.gate = gate;
  a.r = r;
  a.logits = logits;
  a.T = c.T;
  a.d = c.d_model;
  a.E = c.E;
  a.k = c.k;
  a.eps = c.eps;
  a.renormalize = c.renormalize ? 1 : 0;
  CUtensorMap xmap;
  // x [T, d]: tiles of 64 tokens x 64 elements
  if (!make_map(&xmap, x, static_cast<uint64_t>(c.d_model), static_cast<uint64_t>(c.T),
                static_cast<uint64_t>(c.d_model), 64, 64))
    return MOE_ERR_CUDA;
  return cuda_status(launch_route(a, xmap, s));
}

moe_status_t run_dispatch(const moe_config_t& c, const Layout& L, void* ws, const int32_t* idx,
                          const moe_bf16_t* x, const moe_bf16_t* gamma, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv_perm, moe_bf16_t* x_perm,
                          int sms, cudaStream_t s, int row_align = 1, uint8_t* x8 = nullptr,
                          uint8_t* xsf = nullptr) {
  DispatchArgs a{};
  a.x8 = x8;
  a.xsf = xsf;
  a.idx = idx;
  a.x = reinterpret_cast<const __nv_bfloat16*>(x);
  a.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  a.tile_counts = at<int32_t>(ws, L.tile_counts);
  a.counts = counts;
  a.offsets = offsets;
  a.perm = perm;
  a.inv_perm = inv_perm;
  a.x_perm = reinterpret_cast<__nv_bfloat16*>(x_perm);
  a.err = at<uint32_t>(ws, L.err);
  a.T = c.T;
  a.d = c.d_model;
  a.E = c.E;
  a.k = c.k;
  const int64_t cap = capacity_of(c);
  a.capacity = static_cast<int>(cap);
  a.max_kept = static_cast<int>(L.max_kept);
  a.row_align = row_align;
  if (c.T == 0) {
    // nothing routed: offsets and counts are still defined
    cudaError_t e = cudaMemsetAsync(offsets, 0, (c.E + 1) * sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, c.E * sizeof(int32_t), s);
    return cuda_status(e);
  }
  return cuda_status(launch_dispatch(a, sms, s));
}

void fill_gemm_common(GemmArgs& g, const moe_config_t& c, const Layout& L, void* ws,
                      const int32_t* perm, const int32_t* offsets) {
  g.E = c.E;
  g.k = c.k;
  g.d = c.d_model;
  g.rows = static_cast<int>(L.max_kept);
  g.offsets = offsets;
  g.perm = perm;
  g.err = at<uint32_t>(ws, L.err);
  for (int e = 0; e <= c.E; ++e) g.ffn.off[e] = c.ffn_offsets[e];
}

// GEMM 1: x_perm [rows, d] x (W1 | W3) [d, F] -> SwiGLU -> H [rows, ldh] (workspace)
moe_status_t run_up(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x_perm,
                    const float* r, const int32_t* perm, const int32_t* offsets,
                    const moe_bf16_t* W1, const moe_bf16_t* W3, int sms, cudaStream_t s,
                    moe_bf16_t* U = nullptr, moe_bf16_t* V = nullptr) {
  if (L.max_kept == 0) return MOE_OK;
  const uint64_t rows = static_cast<uint64_t>(L.max_kept);
  const uint64_t d = static_cast<uint64_t>(c.d_model);
  const uint64_t F = static_cast<uint64_t>(c.ffn_offsets[c.E]);
  GemmArgs g{};
  fill_gemm_common(g, c, L, ws, perm, offsets);
  CUtensorMap mA, mB0, mB1;
  if (!make_map(&mA, x_perm, d, rows, d, 64, 128) || !make_map(&mB0, W1, F, d, F, 64, 64) ||
      !make_map(&mB1, W3, F, d, F, 64, 64))
    return MOE_ERR_CUDA;
  g.mode = kGemmUp;
  g.bn = 2 * kBlockN;
  g.scale = r;
  g.out = at<__nv_bfloat16>(ws, L.H);
  g.ld_out = L.ldh;
  g.out_u = reinterpret_cast<__nv_bfloat16*>(U);
  g.out_v = reinterpret_cast<__nv_bfloat16*>(V);
  (void)sms;
  return cuda_status(launch_grouped_gemm(g, mA, mA, mB0, mB1, gemm_grid_of_current_device(), s));
}

// GEMM 2: H [rows, f_e] (workspace) x W2 [F, d] -> y [rows, d], gate in the epilogue
moe_status_t run_down(const moe_config_t& c, const Layout& L, void* ws, const float* gate,
                      const int32_t* perm, const int32_t* offsets, const moe_bf16_t* W2,
                      moe_bf16_t* y, int sms, cudaStream_t s, moe_bf16_t* yu = nullptr) {
  if (L.max_kept == 0) return MOE_OK;
  const uint64_t rows = static_cast<uint64_t>(L.max_kept);
  const uint64_t d = static_cast<uint64_t>(c.d_model);
  const uint64_t F = static_cast<uint64_t>(c.ffn_offsets[c.E]);
  GemmArgs g{};
  fill_gemm_common(g, c, L, ws, perm, offsets);
  CUtensorMap mA, mB;
  if (!make_map(&mA, at<void>(ws, L.H), static_cast<uint64_t>(L.ldh), rows,
                static_cast<uint64_t>(L.ldh), 64, 128) ||
      !make_map(&mB, W2, d, F, d, 64, 64))
    return MOE_ERR_CUDA;
  g.mode = kGemmDown;
  g.bn = (c.d_model % 256 == 0) ? 256 : 128;
  g.scale = gate;
  g.out = reinterpret_cast<__nv_bfloat16*>(y);
  g.ld_out = c.d_model;
  g.out_yu = reinterpret_cast<__nv_bfloat16*>(yu);
  (void)sms;
  return cuda_status(launch_grouped_gemm(g, mA, mA, mB, mB, gemm_grid_of_current_device(), s));
}

moe_status_t run_experts(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x_perm,
                         const float* r, const float* gate, const int32_t* perm,
                         const int32_t* offsets, const moe_bf16_t* W1, const moe_bf16_t* W3,
                         const moe_bf16_t* W2, moe_bf16_t* y, int sms, cudaStream_t s) {
  moe_status_t st = run_up(c, L, ws, x_perm, r, perm, offsets, W1, W3, sms, s);
  if (st != MOE_OK) return st;
  return run_down(c, L, ws, gate, perm, offsets, W2, y, sms, s);
}

moe_status_t run_combine(const moe_config_t& c, const moe_bf16_t* y, const int32_t* inv_perm,
                         moe_bf16_t* out, int sms, cudaStream_t s) {
  CombineArgs a{};
  a.y = reinterpret_cast<const __nv_bfloat16*>(y);
  a.inv_perm = inv_perm;
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.T = c.T;
  a.d = c.d_model;
  a.k = c.k;
  return cuda_status(launch_combine(a, sms, s));
}

// ---- scratch of moe_dispatch_noalloc: a fixed device array instead of a workspace
constexpr int64_t kNoallocMaxAssignments = int64_t(1) << 20;
constexpr size_t kNoallocHeaderInts = 64;  // 256 B: the error word, then padding
constexpr size_t kNoallocCountInts =
    static_cast<size_t>(kNoallocMaxAssignments / kDispatchTile) * kMaxExperts;  // 256 KiB
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocHeaderInts + kNoallocCountInts];

int32_t* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per
// device; in host code the symbol itself is only a host-side stand-in).
moe_status_t noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

// ---- the layer on device buffers (cfg validated, T > 0, pointers checked)
moe_status_t run_layer(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x,
                       const moe_bf16_t* gamma, const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                       const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out, int32_t* expert_idx,
                       float* gate, float* r, int32_t* counts, float* prob_mean, float* stats, int sms,
                       cudaStream_t s) {
  moe_status_t st;
  int32_t* idx_ = expert_idx ? expert_idx : at<int32_t>(ws, L.idx);
  float* gate_ = gate ? gate : at<float>(ws, L.gate);
  float* r_ = r ? r : at<float>(ws, L.r);
  int32_t* counts_ = counts ? counts : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  moe_bf16_t* x_perm = at<moe_bf16_t>(ws, L.x_perm);
  moe_bf16_t* y = at<moe_bf16_t>(ws, L.y);
  float* pm = prob_mean ? prob_mean : (stats ? at<float>(ws, L.prob_mean) : nullptr);
  if ((st = run_route(c, x, gamma, Wr, bias, idx_, gate_, r_, nullptr, pm, L, ws, s)) != MOE_OK) return st;
  if ((st = run_dispatch(c, L, ws, idx_, x, gamma, counts_, offsets, perm, inv_perm, x_perm, sms, s)) != MOE_OK)
    return st;
  if ((st = run_experts(c, L, ws, x_perm, r_, gate_, perm, offsets, W1, W3, W2, y, sms, s)) != MOE_OK)
    return st;
  if ((st = run_combine(c, y, inv_perm, out, sms, s)) != MOE_OK) return st;
  if (stats != nullptr)
    return cuda_status(launch_router_stats(pm, counts_, offsets, stats, c.T, c.E, c.k, s));
  return MOE_OK;
}

// ---- the layer with MXFP8 expert GEMMs (cfg validated, T > 0, pointers checked)
moe_status_t run_layer_mx(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x,
                          const moe_bf16_t* gamma, const moe_bf16_t* Wr, const float* bias, const MxWeights& q,
                          moe_bf16_t* out, int sms, cudaStream_t s) {
  moe_status_t st;
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* gate = at<float>(ws, L.gate);
  float* r = at<float>(ws, L.r);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  moe_bf16_t* y = at<moe_bf16_t>(ws, L.y);
  if ((st = run_route(c, x, gamma, Wr, bias, idx, gate, r, nullptr, nullptr, L, ws, s)) != MOE_OK) return st;
  if ((st = run_dispatch(c, L, ws, idx, x, gamma, at<int32_t>(ws, L.counts), offsets, perm, inv_perm, nullptr,
                         sms, s, kMxRowAlign, at<uint8_t>(ws, L.x8), at<uint8_t>(ws, L.xsf))) != MOE_OK)
    return st;
  const uint64_t rows = static_cast<uint64_t>(L.max_kept);
  const uint64_t d = static_cast<uint64_t>(c.d_model);
  const uint64_t F = static_cast<uint64_t>(c.ffn_offsets[c.E]);
  const uint64_t ldh = static_cast<uint64_t>(L.ldh);
  MxGemmArgs g{};
  g.E = c.E; g.k = c.k; g.d = c.d_model; g.F = static_cast<int>(F);
  g.rows = static_cast<int>(L.max_kept);
  g.ldh = L.ldh;
  g.offsets = offsets;
  g.perm = perm;
  g.err = at<uint32_t>(ws, L.err);
  for (int e = 0; e <= c.E; ++e) g.ffn.off[e] = c.ffn_offsets[e];
  const int grid = gemm_grid_of_current_device();
  CUtensorMap mA, mB0, mB1, mSA, mSB0, mSB1;
  g.up = 1;
  g.bn = 256;
  g.scale = r;
  g.h8 = at<uint8_t>(ws, L.h8);
  g.hsf = at<uint8_t>(ws, L.hsf);
  if (!make_map_u8(&mA, at<void>(ws, L.x8), d, rows, d, 128, 128) || !make_map_u8(&mB0, q.w1, d, F, d, 128, 128) ||
      !make_map_u8(&mB1, q.w3, d, F, d, 128, 128) ||
      !make_map_sf(&mSA, at<void>(ws, L.xsf), (rows / 128) * (d / 128)) ||
      !make_map_sf(&mSB0, q.sf1, (F / 128) * (d / 128)) || !make_map_sf(&mSB1, q.sf3, (F / 128) * (d / 128)))
    return MOE_ERR_CUDA;
  if ((st = cuda_status(launch_grouped_gemm_mx(g, mA, mB0, mB1, mSA, mSB0, mSB1, grid, s))) != MOE_OK) return st;
  g.up = 0;
  g.bn = (c.d_model % 256 == 0) ? 256 : 128;
  g.scale = gate;
  g.y = reinterpret_cast<__nv_bfloat16*>(y);
  if (!make_map_u8(&mA, at<void>(ws, L.h8), ldh, rows, ldh, 128, 128) ||
      !make_map_u8(&mB0, q.w2, F, d, F, 128, static_cast<uint32_t>(g.bn / 2)) ||
      !make_map_sf(&mSA, at<void>(ws, L.hsf), (rows / 128) * (ldh / 128)) ||
      !make_map_sf(&mSB0, q.sf2, (d / 128) * (F / 128)))
    return MOE_ERR_CUDA;
  if ((st = cuda_status(launch_grouped_gemm_mx(g, mA, mB0, mB0, mSA, mSB0, mSB0, grid, s))) != MOE_OK) return st;
  return run_combine(c, y, inv_perm, out, sms, s);
}

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

// Chunk sizes in the ratio 1 : 2 : ... : 2 : 1: only the first chunk's copy
// in and the last chunk's copy out are not hidden behind compute, so those two
// are half the size of the others.
HostLayout host_layout_of(const moe_config_t& c, int n_chunks) {
  HostLayout H{};
  int n = n_chunks > 0 ? n_chunks : kDefaultHostChunks;
  if (capacity_of(c) >= 0) n = 1;          // capacity ranks span the whole batch
  if (n > kMaxHostChunks) n = kMaxHostChunks;
  if (n > c.T) n = c.T > 0 ? c.T : 1;
  const int64_t wsum = n <= 2 ? n : 2 * n - 2;
  int64_t acc = 0;
  H.start[0] = 0;
  for (int i = 0; i < n; ++i) {
    acc += (n <= 2 || i == 0 || i == n - 1) ? 1 : 2;
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

// ---- training backward: gather -> bwd_h -> bwd_x -> weight gradients ->
// router/statistic backward -> norm backward -> reductions, on one stream.
moe_status_t run_backward(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x,
                          const moe_bf16_t* gamma, const moe_bf16_t* Wr, const float* bias,
                          const moe_bf16_t* W1, const moe_bf16_t* W3, const moe_bf16_t* W2,
                          const moe_bf16_t* dout, float* dx, float* dgamma, float* dWr, float* dbias,
                          float* dW1, float* dW3, float* dW2, int sms, cudaStream_t s) {
  const uint64_t rows = static_cast<uint64_t>(L.max_kept);
  const uint64_t d = static_cast<uint64_t>(c.d_model);
  const uint64_t F = static_cast<uint64_t>(c.ffn_offsets[c.E]);
  const uint64_t ldh = static_cast<uint64_t>(L.ldh);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  bool all256 = true;
  for (int e = 0; e < c.E; ++e) all256 = all256 && ((c.ffn_offsets[e + 1] - c.ffn_offsets[e]) % 256 == 0);
  const int bn_h = all256 ? 256 : 128;
  const int bn_d = (c.d_model % 256 == 0) ? 256 : 128;
  const int grid = gemm_grid_of_current_device();

  BwdArgs b{};
  b.T = c.T; b.d = c.d_model; b.E = c.E; b.k = c.k; b.renormalize = c.renormalize;
  b.rows = static_cast<int>(L.max_kept);
  b.x = reinterpret_cast<const __nv_bfloat16*>(x);
  b.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  b.Wr = reinterpret_cast<const __nv_bfloat16*>(Wr);
  b.bias = bias;
  b.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
  b.r = at<float>(ws, L.r);
  b.idx = at<int32_t>(ws, L.idx);
  b.gate = at<float>(ws, L.gate);
  b.logits = at<float>(ws, L.logits);
  b.offsets = offsets;
  b.perm = perm;
  b.inv_perm = at<int32_t>(ws, L.inv_perm);
  b.yu = at<__nv_bfloat16>(ws, L.yu);
  b.dY = at<__nv_bfloat16>(ws, L.dY);
  b.dgate = at<float>(ws, L.dgate);
  b.drp = at<float>(ws, L.drp);
  b.ld_drp = L.ld_drp;
  b.bn_h = bn_h;
  b.dXp = at<float>(ws, L.dXp);
  b.rdl = at<float>(ws, L.rdl);
  b.dr = at<float>(ws, L.dr);
  b.dbias_part = at<float>(ws, L.dbias_part);
  b.route_blocks = L.route_blocks;
  b.dx = dx;
  b.dgamma_part = at<float>(ws, L.dgamma_part);
  b.dWr_part = at<float>(ws, L.dWr_part);
  b.chunks = L.chunks;
  b.chunk_tokens = L.chunk_tokens;
  b.dgamma = dgamma;
  b.dWr = dWr;
  b.dbias = dbias;
  b.err = at<uint32_t>(ws, L.err);
  for (int e = 0; e <= c.E; ++e) b.ffn.off[e] = c.ffn_offsets[e];

  moe_status_t st = cuda_status(launch_bwd_gather(b, sms, s));
  if (st != MOE_OK) return st;
  void* dY = at<void>(ws, L.dY);
  void* dS = at<void>(ws, L.dS);
  void* dS3 = at<void>(ws, L.dS3);
  CUtensorMap mA0, mA1, mB0, mB1;
  {  // dS, dS3, dr partials: dY [rows, d] x W2 rows (K-major)
    GemmArgs g{};
    fill_gemm_common(g, c, L, ws, perm, offsets);
    g.mode = kGemmBwdH;
    g.bn = bn_h;
    g.scale = b.r;
    g.ld_out = L.ldh;
    g.in_u = at<__nv_bfloat16>(ws, L.U);
    g.in_v = at<__nv_bfloat16>(ws, L.V);
    g.out_ds = static_cast<__nv_bfloat16*>(dS);
    g.out_ds3 = static_cast<__nv_bfloat16*>(dS3);
    g.drp = at<float>(ws, L.drp);
    g.ld_drp = L.ld_drp;
    if (!make_map(&mA0, dY, d, rows, d, 64, 128) || !make_map(&mB0, W2, d, F, d, 64, bn_h / 2))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA0, mB0, mB0, grid, s))) != MOE_OK) return st;
  }
  {  // dX per kept row: [dS | dS3] x [W1 | W3]^T (W rows, K-major)
    GemmArgs g{};
    fill_gemm_common(g, c, L, ws, perm, offsets);
    g.mode = kGemmBwdX;
    g.bn = bn_d;
    g.out_f0 = at<float>(ws, L.dXp);
    g.ld_f = c.d_model;
    if (!make_map(&mA0, dS, ldh, rows, ldh, 64, 128) || !make_map(&mA1, dS3, ldh, rows, ldh, 64, 128) ||
        !make_map(&mB0, W1, F, d, F, 64, bn_d / 2) || !make_map(&mB1, W3, F, d, F, 64, bn_d / 2))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA1, mB0, mB1, grid, s))) != MOE_OK) return st;
  }
  {  // dW1 | dW3 = x_perm^T [dS | dS3]  (both operands MN-major, K = rows)
    GemmArgs g{};
    fill_gemm_common(g, c, L, ws, perm, offsets);
    g.mode = kGemmWgradX;
    g.bn = 256;
    g.out_f0 = dW1;
    g.out_f1 = dW3;
    g.ld_f = static_cast<int>(F);
    if (!make_map(&mA0, at<void>(ws, L.x_perm), d, rows, d, 64, 64) ||
        !make_map(&mB0, dS, ldh, rows, ldh, 64, 64) || !make_map(&mB1, dS3, ldh, rows, ldh, 64, 64))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA0, mB0, mB1, grid, s))) != MOE_OK) return st;
  }
  {  // dW2 = H^T dY
    GemmArgs g{};
    fill_gemm_common(g, c, L, ws, perm, offsets);
    g.mode = kGemmWgradH;
    g.bn = bn_d;
    g.out_f0 = dW2;
    g.ld_f = c.d_model;
    if (!make_map(&mA0, at<void>(ws, L.H), ldh, rows, ldh, 64, 64) || !make_map(&mB0, dY, d, rows, d, 64, 64))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA0, mB0, mB0, grid, s))) != MOE_OK) return st;
  }
  if ((st = cuda_status(launch_bwd_route(b, s))) != MOE_OK) return st;
  if ((st = cuda_status(launch_bwd_norm(b, s))) != MOE_OK) return st;
  return cuda_status(launch_bwd_reduce(b, s));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT: pointer not aligned as required";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: outside this build's limits";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE: the device error word is set";
    case MOE_ERR_NO_DEVICE: return "MOE_ERR_NO_DEVICE: no usable sm_100 device";
  }
  return "MOE_ERR_UNKNOWN";
}

int64_t moe_capacity(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return -1;
  return capacity_of(*cfg);
}

int64_t moe_max_kept(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return -1;
  return max_kept_of(*cfg);
}

size_t moe_workspace_size(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return layout_of(*cfg).total;
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < kHeaderBytes) return MOE_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  int sms;
  moe_status_t st = device_ready(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(cudaMemsetAsync(ws, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_get_device_error(void* ws, size_t ws_bytes, void* stream, uint32_t* code) {
  if (code == nullptr) return MOE_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < kHeaderBytes) return MOE_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  int sms;
  moe_status_t st = device_ready(&sms);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(v), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  *code = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

moe_status_t moe_route(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                       const moe_bf16_t* Wr, const float* bias, int32_t* expert_idx, float* gate,
                       float* r, float* logits, float* prob_mean, void* ws, size_t ws_bytes,
                       void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;  // no tokens: nothing to do (pointers may be null)
  if (!x || !gamma || !Wr || !expert_idx || !gate || !r) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(gamma, 16) || !aligned(Wr, 2) || !aligned(bias, 4) ||
      !aligned(expert_idx, 4) || !aligned(gate, 4) || !aligned(r, 4) || !aligned(logits, 4) ||
      !aligned(prob_mean, 4))
    return MOE_ERR_ALIGNMENT;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L)) != MOE_OK) return st;
  return run_route(*cfg, x, gamma, Wr, bias, expert_idx, gate, r, logits, prob_mean, L, ws,
                   static_cast<cudaStream_t>(stream));
}

moe_status_t moe_dispatch(const moe_config_t* cfg, const int32_t* expert_idx, const moe_bf16_t* x,
                          const moe_bf16_t* gamma, int32_t* counts, int32_t* expert_offsets,
                          int32_t* perm, int32_t* inv_perm, moe_bf16_t* x_perm, void* ws,
                          size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) {  // no tokens: counts and offsets are zero, nothing else is touched
    if (!counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (!aligned(counts, 4) || !aligned(expert_offsets, 4)) return MOE_ERR_ALIGNMENT;
    int sms;
    if ((st = device_ready(&sms)) != MOE_OK) return st;
    cudaStream_t s0 = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(expert_offsets, 0, (cfg->E + 1) * sizeof(int32_t), s0);
    if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, cfg->E * sizeof(int32_t), s0);
    return cuda_status(e);
  }
  if (!expert_idx || !x || !gamma || !counts || !expert_offsets || !perm || !inv_perm || !x_perm)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(expert_idx, 4) || !aligned(counts, 4) || !aligned(expert_offsets, 4) ||
      !aligned(perm, 4) || !aligned(inv_perm, 4) || !aligned(x, 16) || !aligned(gamma, 16) ||
      !aligned(x_perm, 16))
    return MOE_ERR_ALIGNMENT;
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L)) != MOE_OK) return st;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_dispatch(*cfg, L, ws, expert_idx, x, gamma, counts, expert_offsets, perm, inv_perm,
                      x_perm, sms, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_dispatch_noalloc(const moe_config_t* cfg, const int32_t* expert_idx,
                                  const moe_bf16_t* x, const moe_bf16_t* gamma, int32_t* counts,
                                  int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                                  moe_bf16_t* x_perm, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  const int64_t tk = static_cast<int64_t>(cfg->T) * cfg->k;
  if (tk > kNoallocMaxAssignments) return MOE_ERR_UNSUPPORTED;
  if (!counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!expert_idx || !x || !gamma || !perm || !inv_perm || !x_perm))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(expert_idx, 4) || !aligned(counts, 4) || !aligned(expert_offsets, 4) ||
      !aligned(perm, 4) || !aligned(inv_perm, 4) || !aligned(x, 16) || !aligned(gamma, 16) ||
      !aligned(x_perm, 16))
    return MOE_ERR_ALIGNMENT;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  int32_t* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->T == 0) {
    cudaError_t e = cudaMemsetAsync(expert_offsets, 0, (cfg->E + 1) * sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, cfg->E * sizeof(int32_t), s);
    return cuda_status(e);
  }
  // the error word must start at zero; the tile counts are fully rewritten
  cudaError_t e = cudaMemsetAsync(scratch, 0, kNoallocHeaderInts * sizeof(int32_t), s);
  if (e != cudaSuccess) return cuda_status(e);
  DispatchArgs a{};
  a.idx = expert_idx;
  a.x = reinterpret_cast<const __nv_bfloat16*>(x);
  a.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  a.tile_counts = scratch + kNoallocHeaderInts;
  a.counts = counts;
  a.offsets = expert_offsets;
  a.perm = perm;
  a.inv_perm = inv_perm;
  a.x_perm = reinterpret_cast<__nv_bfloat16*>(x_perm);
  a.err = reinterpret_cast<uint32_t*>(scratch);
  a.T = cfg->T;
  a.d = cfg->d_model;
  a.E = cfg->E;
  a.k = cfg->k;
  a.capacity = static_cast<int>(capacity_of(*cfg));
  a.max_kept = static_cast<int>(max_kept_of(*cfg));
  a.row_align = 1;
  return cuda_status(launch_dispatch(a, sms, s));
}

moe_status_t moe_experts_fwd(const moe_config_t* cfg, const moe_bf16_t* x_perm, const float* r,
                             const float* gate, const int32_t* perm,
                             const int32_t* expert_offsets, const moe_bf16_t* W1,
                             const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* y, void* ws,
                             size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x_perm || !r || !gate || !perm || !expert_offsets || !W1 || !W3 || !W2 || !y)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x_perm, 16) || !aligned(W1, 16) || !aligned(W3, 16) || !aligned(W2, 16) ||
      !aligned(y, 16) || !aligned(r, 4) || !aligned(gate, 4) || !aligned(perm, 4) ||
      !aligned(expert_offsets, 4))
    return MOE_ERR_ALIGNMENT;
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L)) != MOE_OK) return st;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_experts(*cfg, L, ws, x_perm, r, gate, perm, expert_offsets, W1, W3, W2, y, sms,
                     static_cast<cudaStream_t>(stream));
}

moe_status_t moe_experts_up(const moe_config_t* cfg, const moe_bf16_t* x_perm, const float* r,
                            const int32_t* perm, const int32_t* expert_offsets, const moe_bf16_t* W1,
                            const moe_bf16_t* W3, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x_perm || !r || !perm || !expert_offsets || !W1 || !W3) return MOE_ERR_INVALID_ARG;
  if (!aligned(x_perm, 16) || !aligned(W1, 16) || !aligned(W3, 16) || !aligned(r, 4) ||
      !aligned(perm, 4) || !aligned(expert_offsets, 4))
    return MOE_ERR_ALIGNMENT;
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L)) != MOE_OK) return st;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_up(*cfg, L, ws, x_perm, r, perm, expert_offsets, W1, W3, sms,
                static_cast<cudaStream_t>(stream));
}

moe_status_t moe_experts_down(const moe_config_t* cfg, const float* gate, const int32_t* perm,
                              const int32_t* expert_offsets, const moe_bf16_t* W2, moe_bf16_t* y,
                              void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!gate || !perm || !expert_offsets || !W2 || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned(W2, 16) || !aligned(y, 16) || !aligned(gate, 4) || !aligned(perm, 4) ||
      !aligned(expert_offsets, 4))
    return MOE_ERR_ALIGNMENT;
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L)) != MOE_OK) return st;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_down(*cfg, L, ws, gate, perm, expert_offsets, W2, y, sms,
                  static_cast<cudaStream_t>(stream));
}

moe_status_t moe_combine(const moe_config_t* cfg, const moe_bf16_t* y, const int32_t* inv_perm,
                         moe_bf16_t* out, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!y || !inv_perm || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(out, 16) || !aligned(inv_perm, 4)) return MOE_ERR_ALIGNMENT;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_combine(*cfg, y, inv_perm, out, sms, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_layer_fwd(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                           const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                           const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out,
                           int32_t* expert_idx, float* gate, float* r, int32_t* counts,
                           float* prob_mean, float* stats, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) {  // no tokens: only the optional counts are written (zeros)
    if (counts == nullptr) return MOE_OK;
    if (!aligned(counts, 4)) return MOE_ERR_ALIGNMENT;
    int sms;
    if ((st = device_ready(&sms)) != MOE_OK) return st;
    return cuda_status(cudaMemsetAsync(counts, 0, cfg->E * sizeof(int32_t), static_cast<cudaStream_t>(stream)));
  }
  if (!aligned(prob_mean, 4) || !aligned(stats, 4)) return MOE_ERR_ALIGNMENT;
  if (!x || !gamma || !Wr || !W1 || !W3 || !W2 || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(gamma, 16) || !aligned(Wr, 2) || !aligned(bias, 4) ||
      !aligned(W1, 16) || !aligned(W3, 16) || !aligned(W2, 16) || !aligned(out, 16) ||
      !aligned(expert_idx, 4) || !aligned(gate, 4) || !aligned(r, 4) || !aligned(counts, 4))
    return MOE_ERR_ALIGNMENT;
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L)) != MOE_OK) return st;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_layer(*cfg, L, ws, x, gamma, Wr, bias, W1, W3, W2, out, expert_idx, gate, r, counts, prob_mean,
                   stats, sms, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_router_stats(const moe_config_t* cfg, const float* prob_mean, const int32_t* counts,
                              const int32_t* expert_offsets, float* stats, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!prob_mean || !counts || !expert_offsets || !stats) return MOE_ERR_INVALID_ARG;
  if (!aligned(prob_mean, 4) || !aligned(counts, 4) || !aligned(expert_offsets, 4) || !aligned(stats, 4))
    return MOE_ERR_ALIGNMENT;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return cuda_status(launch_router_stats(prob_mean, counts, expert_offsets, stats, cfg->T, cfg->E, cfg->k,
                                         static_cast<cudaStream_t>(stream)));
}

size_t moe_mx_weights_size(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return mx_weights_bytes(cfg->d_model, cfg->ffn_offsets[cfg->E]);
}

moe_status_t moe_quantize_weights_mx(const moe_config_t* cfg, const moe_bf16_t* W1, const moe_bf16_t* W3,
                                     const moe_bf16_t* W2, void* wq, size_t wq_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (!W1 || !W3 || !W2 || !wq) return MOE_ERR_INVALID_ARG;
  if (!aligned(W1, 16) || !aligned(W3, 16) || !aligned(W2, 16) || !aligned(wq, 256)) return MOE_ERR_ALIGNMENT;
  const int d = cfg->d_model, F = cfg->ffn_offsets[cfg->E];
  if (wq_bytes < mx_weights_bytes(d, F)) return MOE_ERR_WORKSPACE;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return cuda_status(launch_quantize_weights_mx(reinterpret_cast<const __nv_bfloat16*>(W1),
                                                reinterpret_cast<const __nv_bfloat16*>(W3),
                                                reinterpret_cast<const __nv_bfloat16*>(W2), mx_weights_at(wq, d, F),
                                                d, F, static_cast<cudaStream_t>(stream)));
}

size_t moe_mx_workspace_size(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return layout_of(*cfg, false, true).total;
}

int64_t moe_mx_rows(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return -1;
  return layout_of(*cfg, false, true).max_kept;
}

moe_status_t moe_layer_fwd_mx(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                              const moe_bf16_t* Wr, const float* bias, const void* wq, size_t wq_bytes,
                              moe_bf16_t* out, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !gamma || !Wr || !wq || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(gamma, 16) || !aligned(Wr, 2) || !aligned(bias, 4) || !aligned(wq, 256) ||
      !aligned(out, 16))
    return MOE_ERR_ALIGNMENT;
  const int d = cfg->d_model, F = cfg->ffn_offsets[cfg->E];
  if (wq_bytes < mx_weights_bytes(d, F)) return MOE_ERR_WORKSPACE;
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L, false, true)) != MOE_OK) return st;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_layer_mx(*cfg, L, ws, x, gamma, Wr, bias, mx_weights_at(const_cast<void*>(wq), d, F), out, sms,
                      static_cast<cudaStream_t>(stream));
}

moe_status_t moe_mx_part(const moe_config_t* cfg, void* wq, void* ws, size_t ws_bytes, int32_t which,
                         void** ptr) {
  if (ptr == nullptr) return MOE_ERR_INVALID_ARG;
  *ptr = nullptr;
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (which < 0) return MOE_ERR_INVALID_ARG;
  if (which <= MOE_MX_SF2) {
    if (wq == nullptr) return MOE_ERR_INVALID_ARG;
    const MxWeights q = mx_weights_at(wq, cfg->d_model, cfg->ffn_offsets[cfg->E]);
    uint8_t* parts[] = {q.w1, q.w3, q.w2, q.sf1, q.sf3, q.sf2};
    *ptr = parts[which];
    return MOE_OK;
  }
  Layout L;
  if ((st = check_ws(*cfg, ws, ws_bytes, &L, false, true)) != MOE_OK) return st;
  size_t off;
  switch (which) {
    case MOE_MX_X8: off = L.x8; break;
    case MOE_MX_XSF: off = L.xsf; break;
    case MOE_MX_H8: off = L.h8; break;
    case MOE_MX_HSF: off = L.hsf; break;
    case MOE_MX_PERM: off = L.perm; break;
    case MOE_MX_OFFSETS: off = L.offsets; break;
    case MOE_MX_IDX: off = L.idx; break;
    case MOE_MX_GATE: off = L.gate; break;
    case MOE_MX_R: off = L.r; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  *ptr = at<void>(ws, off);
  return MOE_OK;
}

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

size_t moe_train_workspace_size(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return layout_of(*cfg, true).total;
}

int64_t moe_train_rows(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return -1;
  return layout_of(*cfg, true).max_kept;
}

moe_status_t moe_train_saved(const moe_config_t* cfg, void* tws, size_t tws_bytes, int32_t which,
                             void** ptr) {
  if (ptr == nullptr) return MOE_ERR_INVALID_ARG;
  *ptr = nullptr;
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  Layout L;
  if ((st = check_ws(*cfg, tws, tws_bytes, &L, true)) != MOE_OK) return st;
  size_t off;
  switch (which) {
    case MOE_SAVED_R: off = L.r; break;
    case MOE_SAVED_IDX: off = L.idx; break;
    case MOE_SAVED_GATE: off = L.gate; break;
    case MOE_SAVED_LOGITS: off = L.logits; break;
    case MOE_SAVED_OFFSETS: off = L.offsets; break;
    case MOE_SAVED_PERM: off = L.perm; break;
    case MOE_SAVED_INV_PERM: off = L.inv_perm; break;
    case MOE_SAVED_U: off = L.U; break;
    case MOE_SAVED_V: off = L.V; break;
    case MOE_SAVED_H: off = L.H; break;
    case MOE_SAVED_Y: off = L.yu; break;
    case MOE_SAVED_DGATE: off = L.dgate; break;
    case MOE_SAVED_DR: off = L.dr; break;
    case MOE_SAVED_COUNTS: off = L.counts; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  *ptr = at<void>(tws, off);
  return MOE_OK;
}

moe_status_t moe_layer_fwd_train(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                                 const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                                 const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out, void* tws,
                                 size_t tws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !gamma || !Wr || !W1 || !W3 || !W2 || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(gamma, 16) || !aligned(Wr, 2) || !aligned(bias, 4) ||
      !aligned(W1, 16) || !aligned(W3, 16) || !aligned(W2, 16) || !aligned(out, 16))
    return MOE_ERR_ALIGNMENT;
  Layout L;
  if ((st = check_ws(*cfg, tws, tws_bytes, &L, true)) != MOE_OK) return st;
  int sms;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const moe_config_t& c = *cfg;
  void* ws = tws;
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* gate = at<float>(ws, L.gate);
  float* r = at<float>(ws, L.r);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  moe_bf16_t* x_perm = at<moe_bf16_t>(ws, L.x_perm);
  moe_bf16_t* y = at<moe_bf16_t>(ws, L.y);
  if ((st = run_route(c, x, gamma, Wr, bias, idx, gate, r, at<float>(ws, L.logits), nullptr, L, ws, s)) !=
      MOE_OK)
    return st;
  if ((st = run_dispatch(c, L, ws, idx, x, gamma, at<int32_t>(ws, L.counts), offsets, perm, inv_perm, x_perm,
                         sms, s, kTrainRowAlign)) != MOE_OK)
    return st;
  if ((st = run_up(c, L, ws, x_perm, r, perm, offsets, W1, W3, sms, s, at<moe_bf16_t>(ws, L.U),
                   at<moe_bf16_t>(ws, L.V))) != MOE_OK)
    return st;
  if ((st = run_down(c, L, ws, gate, perm, offsets, W2, y, sms, s, at<moe_bf16_t>(ws, L.yu))) != MOE_OK)
    return st;
  return run_combine(c, y, inv_perm, out, sms, s);
}

moe_status_t moe_layer_bwd(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                           const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                           const moe_bf16_t* W3, const moe_bf16_t* W2, const moe_bf16_t* dout, float* dx,
                           float* dgamma, float* dWr, float* dbias, float* dW1, float* dW3, float* dW2,
                           void* tws, size_t tws_bytes, void* stream) {
  moe_status_t st = validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (!dgamma || !dWr || !dbias || !dW1 || !dW3 || !dW2) return MOE_ERR_INVALID_ARG;
  if (!aligned(dgamma, 4) || !aligned(dWr, 16) || !aligned(dbias, 4) || !aligned(dW1, 16) ||
      !aligned(dW3, 16) || !aligned(dW2, 16))
    return MOE_ERR_ALIGNMENT;
  int sms;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t d = static_cast<size_t>(c.d_model), F = static_cast<size_t>(c.ffn_offsets[c.E]);
  if (c.T == 0) {  // no tokens: every parameter gradient is zero
    if ((st = device_ready(&sms)) != MOE_OK) return st;
    cudaError_t e = cudaMemsetAsync(dgamma, 0, d * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dWr, 0, d * c.E * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dbias, 0, static_cast<size_t>(c.E) * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW1, 0, d * F * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW3, 0, d * F * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW2, 0, d * F * 4, s);
    return cuda_status(e);
  }
  if (!x || !gamma || !Wr || !W1 || !W3 || !W2 || !dout || !dx) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(gamma, 16) || !aligned(Wr, 2) || !aligned(bias, 4) ||
      !aligned(W1, 16) || !aligned(W3, 16) || !aligned(W2, 16) || !aligned(dout, 16) || !aligned(dx, 16))
    return MOE_ERR_ALIGNMENT;
  Layout L;
  if ((st = check_ws(c, tws, tws_bytes, &L, true)) != MOE_OK) return st;
  if ((st = device_ready(&sms)) != MOE_OK) return st;
  return run_backward(c, L, tws, x, gamma, Wr, bias, W1, W3, W2, dout, dx, dgamma, dWr, dbias, dW1, dW3, dW2,
                      sms, s);
}

}  // extern "C"
