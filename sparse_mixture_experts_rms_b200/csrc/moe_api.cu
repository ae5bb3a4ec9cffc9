// moe_api.cu -- the C ABI declared in include/moe.h (the forward layer and
// its stages; training in api_train.cu, MXFP8 in api_mx.cu, host buffers in
// api_host.cu): argument validation, workspace layout, TMA descriptor
// encoding and launch sequencing on one stream.  Allocates nothing; never synchronises except in
// moe_get_device_error.
#include <cmath>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "api_detail.h"

namespace moe {
namespace api {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);


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

Layout layout_of(const moe_config_t& c, bool train, bool mx) {
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
  L.rw = take(static_cast<size_t>(c.d_model) * 2 * kRouterPadE * 2);  // router hi/lo B [2 EP, d] bf16
  L.prob_partial = take(static_cast<size_t>((c.T + kRouteTok - 1) / kRouteTok) * c.E * 4);
  L.prob_mean = take(static_cast<size_t>(c.E) * 4);
  L.scan = take(dispatch_scan_ints(static_cast<int>(ntiles), c.E) * 4);
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
    // x_perm, or the gathering layer's xg [T, d] (token order) in the same buffer
    L.x_perm = take(std::max<size_t>(mk, static_cast<size_t>(c.T)) * c.d_model * 2);
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

moe_status_t check_ws(const moe_config_t& c, void* ws, size_t ws_bytes, Layout* L, bool train,
                      bool mx) {
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
              uint32_t box_inner, uint32_t box_outer, bool swizzle64) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_elems * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor map, 128-byte swizzle, box inner x outer.
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_elems,
                  uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_elems * 4};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

// The MX weights' paired scale regions (4 KB each) as a [4 * nregions, 256]
// array of 32-bit words; one region (4 rows) per box.
bool make_map_sfp(CUtensorMap* m, const void* base, uint64_t nregions) {
  const cuuint64_t dims[2] = {256, 4 * nregions};
  const cuuint64_t strides[1] = {1024};
  const cuuint32_t box[2] = {256, 4};
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


moe_status_t run_route(const moe_config_t& c, const moe_bf16_t* x, const moe_bf16_t* gamma,
                       const moe_bf16_t* Wr, const float* bias, int32_t* idx, float* gate, float* r,
                       float* logits, float* prob_mean, const Layout& L, void* ws, cudaStream_t s,
                       moe_bf16_t* xg) {
  if (c.T == 0) return MOE_OK;
  RouteArgs a{};
  a.wprime = at<__nv_bfloat16>(ws, L.rw);
  a.err = at<uint32_t>(ws, L.err);
  a.wait_ctl = at<uint32_t>(ws, kWaitCtlOffset);
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
  CUtensorMap xmap, wmap, xgmap;
  // x [T, d]: tiles of 128 tokens x 64 elements; the router's hi/lo B [2 EP, d]: 2 EP x 64;
  // xg [T, d] (optional): 32-token boxes, one per epilogue lane quarter
  const uint32_t ep2 = static_cast<uint32_t>(2 * route_padded_experts(c.E));
  const uint64_t d = static_cast<uint64_t>(c.d_model), T = static_cast<uint64_t>(c.T);
  if (!make_map(&xmap, x, d, T, d, 64, kRouteTok) || !make_map(&wmap, a.wprime, d, ep2, d, 64, ep2) ||
      (xg != nullptr && !make_map(&xgmap, xg, d, T, d, 64, 32)))
    return MOE_ERR_CUDA;
  return cuda_status(launch_route(a, xmap, wmap, xg != nullptr ? &xgmap : nullptr, s));
}

moe_status_t run_dispatch(const moe_config_t& c, const Layout& L, void* ws, const int32_t* idx,
                          const moe_bf16_t* x, const moe_bf16_t* gamma, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv_perm, moe_bf16_t* x_perm,
                          int sms, cudaStream_t s, int row_align, uint8_t* x8,
                          uint8_t* xsf) {
  DispatchArgs a{};
  a.x8 = x8;
  a.xsf = xsf;
  a.idx = idx;
  a.x = reinterpret_cast<const __nv_bfloat16*>(x);
  a.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  a.scan = at<int32_t>(ws, L.scan);
  a.wait_ctl = at<uint32_t>(ws, kWaitCtlOffset);
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
  g.wait_ctl = at<uint32_t>(ws, kWaitCtlOffset);
  for (int e = 0; e <= c.E; ++e) g.ffn.off[e] = c.ffn_offsets[e];
}

// GEMM 1: x_perm [rows, d] x (W1 | W3) [d, F] -> SwiGLU -> H [rows, ldh] (workspace)
moe_status_t run_up(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x_perm,
                    const float* r, const int32_t* perm, const int32_t* offsets,
                    const moe_bf16_t* W1, const moe_bf16_t* W3, int sms, cudaStream_t s,
                    moe_bf16_t* U, moe_bf16_t* V, bool gather) {
  if (L.max_kept == 0) return MOE_OK;
  const uint64_t rows = static_cast<uint64_t>(L.max_kept);
  const uint64_t d = static_cast<uint64_t>(c.d_model);
  const uint64_t F = static_cast<uint64_t>(c.ffn_offsets[c.E]);
  GemmArgs g{};
  fill_gemm_common(g, c, L, ws, perm, offsets);
  CUtensorMap mA, mB0, mB1;
  // A: x_perm [rows, d] in 128-row boxes, or (gather) xg [T, d] in one-row boxes, row p = token perm[p] / k
  const bool a_ok = gather ? make_map(&mA, x_perm, d, static_cast<uint64_t>(c.T), d, 64, 1)
                           : make_map(&mA, x_perm, d, rows, d, 64, 128);
  if (!a_ok || !make_map(&mB0, W1, F, d, F, 64, 64) ||
      !make_map(&mB1, W3, F, d, F, 64, 64))
    return MOE_ERR_CUDA;
  g.mode = kGemmUp;
  g.gather = gather ? 1 : 0;
  g.bn = 2 * kBlockN;
  g.scale = r;
  g.out = at<__nv_bfloat16>(ws, L.H);
  g.ld_out = L.ldh;
  g.out_u = reinterpret_cast<__nv_bfloat16*>(U);
  g.out_v = reinterpret_cast<__nv_bfloat16*>(V);
  // short reduction: a tile's MMAs take about as long as its epilogue, so run 8 epilogue
  // warps (the training up keeps 4: its three output boxes per chunk need a warp's 8 KB)
  g.epi8 = (c.d_model <= kEpi8MaxK && U == nullptr) ? 1 : 0;
  const uint64_t ldh = static_cast<uint64_t>(L.ldh);
  EpiMaps em{};
  if (!make_map(&em.m[0], g.out, ldh, rows, ldh, 32, 32, true) ||
      (U != nullptr && (!make_map(&em.m[1], U, ldh, rows, ldh, 32, 32, true) ||
                        !make_map(&em.m[2], V, ldh, rows, ldh, 32, 32, true))))
    return MOE_ERR_CUDA;
  (void)sms;
  return cuda_status(launch_grouped_gemm(g, mA, mA, mB0, mB1, gemm_grid_of_current_device(), s, &em));
}

// GEMM 2: H [rows, f_e] (workspace) x W2 [F, d] -> y [rows, d], gate in the epilogue;
// to_token (k = 1): y is the layer output [T, d] and row p goes to row perm[p]
moe_status_t run_down(const moe_config_t& c, const Layout& L, void* ws, const float* gate,
                      const int32_t* perm, const int32_t* offsets, const moe_bf16_t* W2,
                      moe_bf16_t* y, int sms, cudaStream_t s, moe_bf16_t* yu, bool to_token) {
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
  g.epi8 = L.ldh <= kEpi8MaxK ? 1 : 0;  // the down GEMM reduces over the expert width
  (void)sms;
  if (to_token && c.k == 1 && yu == nullptr) {  // scattered rows: stored row by row
    g.to_token = 1;
    return cuda_status(launch_grouped_gemm(g, mA, mA, mB, mB, gemm_grid_of_current_device(), s, nullptr));
  }
  EpiMaps em{};
  if (!make_map(&em.m[0], y, d, rows, d, 32, 32, true) ||
      (yu != nullptr && !make_map(&em.m[1], yu, d, rows, d, 32, 32, true)))
    return MOE_ERR_CUDA;
  return cuda_status(launch_grouped_gemm(g, mA, mA, mB, mB, gemm_grid_of_current_device(), s, &em));
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
// the look-back scan of 1024 tiles of 1024 assignments, up to 64 experts: 516 KiB
constexpr size_t kNoallocScanInts =
    dispatch_scan_ints(static_cast<int>(kNoallocMaxAssignments / kDispatchTile), kMaxExperts);
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocHeaderInts + kNoallocScanInts];

static int32_t* g_noalloc_ptr[kMaxDevices] = {};

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
                       cudaStream_t s, bool gather) {
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
  // k = 1: nothing to sum per token -- the down GEMM writes each kept row
  // straight to its token's row of out; with a capacity limit the rows of
  // dropped tokens are cleared first, by one memset of out (the dispatch
  // clearing them row by row, in its few CTAs, was measured 22 us slower on
  // the Switch config than a combine launch)
  const bool direct = c.k == 1;
  if (direct && capacity_of(c) >= 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, static_cast<size_t>(c.T) * c.d_model * sizeof(moe_bf16_t), s);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // gather: the router also writes xg = bf16(x * gamma) in token order (into
  // the x_perm buffer, which holds T rows), no permuted copy is made, and the
  // up GEMM gathers its A rows from xg by perm as it loads them
  if ((st = run_route(c, x, gamma, Wr, bias, idx_, gate_, r_, nullptr, pm, L, ws, s, gather ? x_perm : nullptr)) !=
      MOE_OK)
    return st;
  if ((st = run_dispatch(c, L, ws, idx_, x, gamma, counts_, offsets, perm, inv_perm, gather ? nullptr : x_perm, sms,
                         s)) != MOE_OK)
    return st;
  if ((st = run_up(c, L, ws, x_perm, r_, perm, offsets, W1, W3, sms, s, nullptr, nullptr, gather)) != MOE_OK)
    return st;
  if ((st = run_down(c, L, ws, gate_, perm, offsets, W2, direct ? out : y, sms, s, nullptr, direct)) != MOE_OK)
    return st;
  if (!direct && (st = run_combine(c, y, inv_perm, out, sms, s)) != MOE_OK) return st;
  if (stats != nullptr)
    return cuda_status(launch_router_stats(pm, counts_, offsets, stats, c.T, c.E, c.k, s));
  return MOE_OK;
}

}  // namespace api
}  // namespace moe

using namespace moe;
using namespace moe::api;

namespace {
// moe_layer_fwd and moe_layer_fwd_gather: argument checks, then the layer.
moe_status_t layer_fwd_entry(bool gather, const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                             const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1, const moe_bf16_t* W3,
                             const moe_bf16_t* W2, moe_bf16_t* out, int32_t* expert_idx, float* gate, float* r,
                             int32_t* counts, float* prob_mean, float* stats, void* ws, size_t ws_bytes,
                             void* stream) {
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
                   stats, sms, static_cast<cudaStream_t>(stream), gather);
}
}  // namespace

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

int32_t moe_expert_offsets(const int32_t* counts, const int32_t* sizes, int32_t n_groups, int32_t* offsets,
                           int32_t max_experts) {
  if (counts == nullptr || sizes == nullptr || offsets == nullptr || n_groups < 0 || max_experts < 0) return -1;
  int64_t E = 0, total = 0;
  for (int32_t g = 0; g < n_groups; ++g) {
    if (counts[g] < 0 || sizes[g] < 1) return -1;
    const int64_t width = (static_cast<int64_t>(sizes[g]) + kBlockN - 1) / kBlockN * kBlockN;
    E += counts[g];
    total += width * counts[g];
    if (E > max_experts || total > INT32_MAX) return -1;
  }
  int32_t e = 0;
  offsets[0] = 0;
  for (int32_t g = 0; g < n_groups; ++g) {
    const int32_t width = static_cast<int32_t>((static_cast<int64_t>(sizes[g]) + kBlockN - 1) / kBlockN * kBlockN);
    for (int32_t c = 0; c < counts[g]; ++c, ++e) offsets[e + 1] = offsets[e] + width;
  }
  return e;
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

moe_status_t moe_set_wait_limit(void* ws, size_t ws_bytes, uint32_t limit_ns, void* stream) {
  if (ws == nullptr || ws_bytes < kHeaderBytes) return MOE_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  int sms;
  moe_status_t st = device_ready(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(launch_set_words(at<uint32_t>(ws, kWaitCtlOffset), limit_ns != 0 ? kWaitCtlTag : 0u,
                                      limit_ns, static_cast<cudaStream_t>(stream)));
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
  // the error word must start at zero (the dispatch clears its scan's status words itself;
  // the scan's count vectors are written before they are read)
  cudaError_t e = cudaMemsetAsync(scratch, 0, kNoallocHeaderInts * sizeof(int32_t), s);
  if (e != cudaSuccess) return cuda_status(e);
  DispatchArgs a{};
  a.idx = expert_idx;
  a.x = reinterpret_cast<const __nv_bfloat16*>(x);
  a.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  a.scan = scratch + kNoallocHeaderInts;
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
  return layer_fwd_entry(false, cfg, x, gamma, Wr, bias, W1, W3, W2, out, expert_idx, gate, r, counts, prob_mean,
                         stats, ws, ws_bytes, stream);
}

moe_status_t moe_layer_fwd_gather(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                                  const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                                  const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out,
                                  int32_t* expert_idx, float* gate, float* r, int32_t* counts,
                                  float* prob_mean, float* stats, void* ws, size_t ws_bytes, void* stream) {
  return layer_fwd_entry(true, cfg, x, gamma, Wr, bias, W1, W3, W2, out, expert_idx, gate, r, counts, prob_mean,
                         stats, ws, ws_bytes, stream);
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

}  // extern "C"
