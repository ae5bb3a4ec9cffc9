// api_mx.cu -- the MXFP8 entry points of the C ABI (include/moe.h): weight
// quantisation, the layer with block-scaled E4M3 expert GEMMs
// (grouped_gemm_mx.cu) and the inspection of its buffers.
#include <algorithm>
#include <mutex>

#include "api_detail.h"

namespace moe {
namespace api {

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
  g.wait_ctl = at<uint32_t>(ws, kWaitCtlOffset);
  for (int e = 0; e <= c.E; ++e) g.ffn.off[e] = c.ffn_offsets[e];
  const int grid = gemm_grid_of_current_device();
  CUtensorMap mA, mB0, mB1, mSA, mSB0;
  g.up = 1;
  g.bn = 256;
  g.scale = r;
  g.h8 = at<uint8_t>(ws, L.h8);
  g.hsf = at<uint8_t>(ws, L.hsf);
  if (!make_map_u8(&mA, at<void>(ws, L.x8), d, rows, d, 128, 128) || !make_map_u8(&mB0, q.w1, d, F, d, 128, 128) ||
      !make_map_u8(&mB1, q.w3, d, F, d, 128, 128) ||
      !make_map_sf(&mSA, at<void>(ws, L.xsf), (rows / 128) * (d / 128)) ||
      !make_map_sfp(&mSB0, q.sfp13, (F / 128) * (d / 128)))
    return MOE_ERR_CUDA;
  if ((st = cuda_status(launch_grouped_gemm_mx(g, mA, mB0, mB1, mSA, mSB0, mSB0, grid, s))) != MOE_OK) return st;
  g.up = 0;
  g.bn = (c.d_model % 256 == 0) ? 256 : 128;
  g.scale = gate;
  g.y = reinterpret_cast<__nv_bfloat16*>(y);
  if (!make_map_u8(&mA, at<void>(ws, L.h8), ldh, rows, ldh, 128, 128) ||
      !make_map_u8(&mB0, q.w2, F, d, F, 128, static_cast<uint32_t>(g.bn / 2)) ||
      !make_map_sf(&mSA, at<void>(ws, L.hsf), (rows / 128) * (ldh / 128)) ||
      !make_map_sfp(&mSB0, q.sfp2, ((d / 128 + 1) / 2) * (F / 128)))
    return MOE_ERR_CUDA;
  if ((st = cuda_status(launch_grouped_gemm_mx(g, mA, mB0, mB0, mSA, mSB0, mSB0, grid, s))) != MOE_OK) return st;
  return run_combine(c, y, inv_perm, out, sms, s);
}

}  // namespace api
}  // namespace moe

using namespace moe;
using namespace moe::api;

extern "C" {

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

}  // extern "C"
