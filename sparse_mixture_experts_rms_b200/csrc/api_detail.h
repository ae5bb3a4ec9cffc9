// api_detail.h -- internals shared by the C-ABI translation units (moe_api.cu,
// api_train.cu, api_mx.cu, api_host.cu): workspace layouts, validation,
// tensor-map encoding, per-device state and the launch sequences of the
// layer's stages.  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>

#include "moe_internal.h"

namespace moe {
namespace api {

constexpr int kMaxDevices = 64;
constexpr size_t kHeaderBytes = 256;  // workspace header: the device error word, the ticket

struct Layout {
  size_t err, ticket, rw, prob_partial, prob_mean, scan, r, idx, gate, counts, offsets, perm,
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

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
template <typename T>
inline T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int64_t capacity_of(const moe_config_t& c);
int64_t max_kept_of(const moe_config_t& c);
moe_status_t validate(const moe_config_t* c);
// Offsets of every buffer in a workspace: inference (default), training
// (segments padded to 64 rows, saved state and backward scratch) or MXFP8
// (segments padded to 128 rows, E4M3 activations and scale blocks).
Layout layout_of(const moe_config_t& c, bool train = false, bool mx = false);
moe_status_t check_ws(const moe_config_t& c, void* ws, size_t ws_bytes, Layout* L, bool train = false,
                      bool mx = false);
// Per-device set-up on first use (kernel attributes, the TMA encoder, the GEMM
// grid); the SM count of the current device.
moe_status_t device_ready(int* sms);
int gemm_grid_of_current_device();
moe_status_t cuda_status(cudaError_t e);

// 2-D tensor maps with 128-byte swizzle (make_map: 64-byte when asked): bf16
// (make_map), fp32 (make_map_f32) or bytes (make_map_u8), `inner` contiguous
// elements per row,
// `outer` rows; and the MX scale blocks as a [nblocks, 128] array of 32-bit
// words (make_map_sf).
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_elems,
              uint32_t box_inner, uint32_t box_outer, bool swizzle64 = false);
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_elems,
                  uint32_t box_inner, uint32_t box_outer);
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer);
bool make_map_sf(CUtensorMap* m, const void* base, uint64_t nblocks);
bool make_map_sfp(CUtensorMap* m, const void* base, uint64_t nregions);

// The layer's stages on one stream (cfg validated, pointers checked).
moe_status_t run_route(const moe_config_t& c, const moe_bf16_t* x, const moe_bf16_t* gamma,
                       const moe_bf16_t* Wr, const float* bias, int32_t* idx, float* gate, float* r,
                       float* logits, float* prob_mean, const Layout& L, void* ws, cudaStream_t s,
                       moe_bf16_t* xg = nullptr);
moe_status_t run_dispatch(const moe_config_t& c, const Layout& L, void* ws, const int32_t* idx,
                          const moe_bf16_t* x, const moe_bf16_t* gamma, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv_perm, moe_bf16_t* x_perm,
                          int sms, cudaStream_t s, int row_align = 1, uint8_t* x8 = nullptr,
                          uint8_t* xsf = nullptr);
void fill_gemm_common(GemmArgs& g, const moe_config_t& c, const Layout& L, void* ws,
                      const int32_t* perm, const int32_t* offsets);
moe_status_t run_up(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x_perm,
                    const float* r, const int32_t* perm, const int32_t* offsets,
                    const moe_bf16_t* W1, const moe_bf16_t* W3, int sms, cudaStream_t s,
                    moe_bf16_t* U = nullptr, moe_bf16_t* V = nullptr, bool gather = false);
moe_status_t run_down(const moe_config_t& c, const Layout& L, void* ws, const float* gate,
                      const int32_t* perm, const int32_t* offsets, const moe_bf16_t* W2,
                      moe_bf16_t* y, int sms, cudaStream_t s, moe_bf16_t* yu = nullptr,
                      bool to_token = false);
moe_status_t run_experts(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x_perm,
                         const float* r, const float* gate, const int32_t* perm,
                         const int32_t* offsets, const moe_bf16_t* W1, const moe_bf16_t* W3,
                         const moe_bf16_t* W2, moe_bf16_t* y, int sms, cudaStream_t s);
moe_status_t run_combine(const moe_config_t& c, const moe_bf16_t* y, const int32_t* inv_perm,
                         moe_bf16_t* out, int sms, cudaStream_t s);
moe_status_t run_layer(const moe_config_t& c, const Layout& L, void* ws, const moe_bf16_t* x,
                       const moe_bf16_t* gamma, const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                       const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out, int32_t* expert_idx,
                       float* gate, float* r, int32_t* counts, float* prob_mean, float* stats, int sms,
                       cudaStream_t s, bool gather = false);

}  // namespace api
}  // namespace moe
