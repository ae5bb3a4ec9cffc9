// api_train.cu -- the training entry points of the C ABI (include/moe.h):
// the forward that saves the backward's inputs and the layer backward, whose
// contractions are modes of the grouped GEMM and whose bandwidth-bound stages
// are in backward.cu.
#include <algorithm>
#include <mutex>

#include "api_detail.h"

namespace moe {
namespace api {

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
    EpiMaps em{};
    if (!make_map(&mA0, dY, d, rows, d, 64, 128) || !make_map(&mB0, W2, d, F, d, 64, bn_h / 2) ||
        !make_map(&em.m[0], g.in_u, ldh, rows, ldh, 32, 32, true) ||
        !make_map(&em.m[1], g.in_v, ldh, rows, ldh, 32, 32, true) ||
        !make_map(&em.m[2], dS, ldh, rows, ldh, 32, 32, true) ||
        !make_map(&em.m[3], dS3, ldh, rows, ldh, 32, 32, true))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA0, mB0, mB0, grid, s, &em))) != MOE_OK) return st;
  }
  {  // dX per kept row: [dS | dS3] x [W1 | W3]^T (W rows, K-major)
    GemmArgs g{};
    fill_gemm_common(g, c, L, ws, perm, offsets);
    g.mode = kGemmBwdX;
    g.bn = bn_d;
    g.out_f0 = at<float>(ws, L.dXp);
    g.ld_f = c.d_model;
    EpiMaps em{};
    if (!make_map(&mA0, dS, ldh, rows, ldh, 64, 128) || !make_map(&mA1, dS3, ldh, rows, ldh, 64, 128) ||
        !make_map(&mB0, W1, F, d, F, 64, bn_d / 2) || !make_map(&mB1, W3, F, d, F, 64, bn_d / 2) ||
        !make_map_f32(&em.m[0], g.out_f0, d, rows, d, 32, 32))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA1, mB0, mB1, grid, s, &em))) != MOE_OK) return st;
  }
  {  // dW1 | dW3 = x_perm^T [dS | dS3]  (both operands MN-major, K = rows)
    GemmArgs g{};
    fill_gemm_common(g, c, L, ws, perm, offsets);
    g.mode = kGemmWgradX;
    g.bn = 256;
    g.out_f0 = dW1;
    g.out_f1 = dW3;
    g.ld_f = static_cast<int>(F);
    EpiMaps em{};
    if (!make_map(&mA0, at<void>(ws, L.x_perm), d, rows, d, 64, 64) ||
        !make_map(&mB0, dS, ldh, rows, ldh, 64, 64) || !make_map(&mB1, dS3, ldh, rows, ldh, 64, 64) ||
        !make_map_f32(&em.m[0], dW1, F, d, F, 32, 32) || !make_map_f32(&em.m[1], dW3, F, d, F, 32, 32))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA0, mB0, mB1, grid, s, &em))) != MOE_OK) return st;
  }
  {  // dW2 = H^T dY
    GemmArgs g{};
    fill_gemm_common(g, c, L, ws, perm, offsets);
    g.mode = kGemmWgradH;
    g.bn = bn_d;
    g.out_f0 = dW2;
    g.ld_f = c.d_model;
    EpiMaps em{};
    if (!make_map(&mA0, at<void>(ws, L.H), ldh, rows, ldh, 64, 64) || !make_map(&mB0, dY, d, rows, d, 64, 64) ||
        !make_map_f32(&em.m[0], dW2, d, F, d, 32, 32))
      return MOE_ERR_CUDA;
    if ((st = cuda_status(launch_grouped_gemm(g, mA0, mA0, mB0, mB0, grid, s, &em))) != MOE_OK) return st;
  }
  if ((st = cuda_status(launch_bwd_route(b, s))) != MOE_OK) return st;
  if ((st = cuda_status(launch_bwd_norm(b, s))) != MOE_OK) return st;
  return cuda_status(launch_bwd_reduce(b, s));
}

}  // namespace api
}  // namespace moe

using namespace moe;
using namespace moe::api;

extern "C" {

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
