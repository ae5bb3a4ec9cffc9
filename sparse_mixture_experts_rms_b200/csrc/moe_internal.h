// moe_internal.h -- launchers shared between the C ABI (moe_api.cu) and the
// kernel translation units.  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe.h"

#include <utility>

namespace moe {

constexpr int kMaxExperts = 64;
constexpr int kRouterPadE = 64;         // w' scratch is sized for the widest router variant
constexpr int kBlockN = 128;            // expert width granule (and G1's N per projection)
constexpr int kDispatchTile = 1024;     // assignments per dispatch CTA
constexpr uint64_t kWaitTimeoutNs = 4000000000ull;  // bounded pipeline waits: 4 s (default)

// Workspace header (256 bytes at offset 0 of every workspace): word 0 = the
// device error word, word 1 = a CTA ticket, words 2-3 = the wait-limit
// control: the tag kWaitCtlTag and a limit in ns for the pipeline waits of
// the kernels that run on this workspace (moe_set_wait_limit).  Any other
// tag, or a zero limit, means the default kWaitTimeoutNs.
constexpr size_t kWaitCtlOffset = 8;
constexpr uint32_t kWaitCtlTag = 0x544D494Cu;
__device__ __forceinline__ uint64_t wait_limit_ns(const uint32_t* ctl) {
  if (ctl != nullptr) {
    const uint32_t tag = ctl[0], ns = ctl[1];
    if (tag == kWaitCtlTag && ns != 0) return ns;
  }
  return kWaitTimeoutNs;
}

// Expert widths passed by value to the GEMM kernels (no device copy needed).
struct ExpertTable {
  int32_t off[kMaxExperts + 1];
};

struct RouteArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* gamma;
  const __nv_bfloat16* Wr;
  const float* bias;  // may be null
  int32_t* idx;
  float* gate;
  float* r;
  float* logits;      // may be null
  uint32_t* err;      // device error word, may be null
  const uint32_t* wait_ctl;  // wait-limit control of the workspace header, may be null
  __nv_bfloat16* wprime;  // [2 EP, d] scratch: (gamma * Wr)^T split into bf16 hi rows, then lo rows
  float* prob_mean;     // [E] out: mean softmax probability per expert, may be null
  float* prob_partial;  // scratch [gridDim, E]: per-CTA probability sums
  unsigned* ticket;     // scratch: CTAs done (zeroed before the launch)
  int T, d, E, k;
  float eps;
  int renormalize;
};

struct DispatchArgs {
  const int32_t* idx;       // [T*k]
  const __nv_bfloat16* x;   // [T, d]
  const __nv_bfloat16* gamma;
  int32_t* scan;            // scratch of the look-back scan (dispatch_scan_ints)
  int32_t* counts;          // [E]
  int32_t* offsets;         // [E+1]
  int32_t* perm;            // [T*k]
  int32_t* inv_perm;        // [T*k]
  __nv_bfloat16* x_perm;    // [max_kept, d]
  uint32_t* err;
  int T, d, E, k;
  int capacity;             // -1: dropless
  int max_kept;             // rows of x_perm
  int row_align;            // 1: dense segments; 64 / 128: each expert's segment
                            // padded to that multiple (perm = -1, zero rows there)
  uint8_t* x8;              // MX mode (x_perm == null): E4M3 codes [max_kept, d]
  uint8_t* xsf;             // MX mode: E8M0 scale blocks of x8 (see mx_sf_offset)
  const uint32_t* wait_ctl; // wait-limit control of the workspace header, may be null
};

// Scratch of the dispatch's look-back scan over tiles of kDispatchTile
// assignments: per tile a status word, then its aggregate and its inclusive
// prefix as E-wide count vectors.
__host__ __device__ constexpr int dispatch_status_ints(int ntiles) { return (ntiles + 63) / 64 * 64; }
__host__ __device__ constexpr size_t dispatch_scan_ints(int ntiles, int E) {
  return static_cast<size_t>(dispatch_status_ints(ntiles)) + 2 * static_cast<size_t>(ntiles) * E;
}

// ---- MXFP8 (OCP MX: 32-element blocks along K, E4M3 codes, E8M0 scales)
//
// Scale factors of an operand with rows r and reduction index k are stored in
// 512-byte blocks of 128 rows x 128 k (4 scales per row), the layout the
// tensor memory expects: block (r / 128, k / 128) of a [rows, K] operand sits
// at block index (r / 128) * (K / 128) + k / 128, and inside a block the scale
// of (r, k) is byte 16 * (r % 32) + 4 * ((r % 128) / 32) + (k % 128) / 32.
__host__ __device__ inline size_t mx_sf_offset(int64_t r, int64_t k, int64_t K) {
  return static_cast<size_t>(((r >> 7) * (K >> 7) + (k >> 7)) * 512 + 16 * (r & 31) + 4 * ((r & 127) >> 5) +
                             ((k & 127) >> 5));
}

// Quantised expert weights: K-major E4M3 copies and their scale blocks.
//   w1, w3 [F, d]   (row n = column n of W1 / W3)      w2 [d, F] (row c = column c of W2)
//   sf1, sf3, sf2: the standard scale blocks of those [rows, K] operands
// sf1 / sf3 / sf2: the weights' scales in the standard blocks (mx_sf_offset).
// sfp13 / sfp2: the same scales as the MX GEMM loads them for its B operand:
// 4 KB regions of two 2 KB halves, each half one 512-byte block written four
// times over, which one tcgen05.cp.128x256b copies into the TMEM image of two
// 32x128b.warpx4 copies.  sfp13 region (nb, kb) = [W1 block | W3 block] of
// column block nb and K block kb (index nb * d/128 + kb); sfp2 region (q, kb)
// = [W2 column block 2q | 2q + 1] (index q * F/128 + kb).
struct MxWeights {
  uint8_t *w1, *w3, *w2, *sf1, *sf3, *sf2, *sfp13, *sfp2;
};
constexpr int kMxPairRegion = 4096;
size_t mx_weights_bytes(int d, int F);
MxWeights mx_weights_at(void* base, int d, int F);
cudaError_t launch_quantize_weights_mx(const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                                       const __nv_bfloat16* W2, MxWeights q, int d, int F, cudaStream_t s);

struct MxGemmArgs {
  int up;                   // 1: x8 x (W1|W3) -> SwiGLU -> H8 (+ scales); 0: H8 x W2 -> gate * y
  int bn;                   // pair MMA N: 256 (the down GEMM: 128 when d % 256 != 0)
  int E, k, d, F;
  int rows;                 // rows of the permuted buffers (a multiple of 128)
  int ldh;                  // row stride of H8 (max expert width)
  const int32_t* offsets;   // [E+1] row segments, multiples of 128
  const int32_t* perm;      // [rows]; -1 = padding
  const float* scale;       // up: r [T]; down: gate [T*k]
  uint8_t* h8;              // up: E4M3 H [rows, ldh]
  uint8_t* hsf;             // up: scale blocks of h8 (K = ldh)
  __nv_bfloat16* y;         // down: [rows, d]
  uint32_t* err;
  const uint32_t* wait_ctl;  // wait-limit control of the workspace header
  ExpertTable ffn;
};
// up: mapSFB0 / mapSFB1 = scales of W1 / W3; down: both the scales of W2.
cudaError_t launch_grouped_gemm_mx(const MxGemmArgs& a, const CUtensorMap& mapA, const CUtensorMap& mapB0,
                                   const CUtensorMap& mapB1, const CUtensorMap& mapSFA,
                                   const CUtensorMap& mapSFB0, const CUtensorMap& mapSFB1, int grid,
                                   cudaStream_t s);
cudaError_t prepare_grouped_gemm_mx();

// Modes of the grouped GEMM (one kernel template, one instantiation each).
enum GemmMode : int {
  kGemmUp = 0,      // x_perm x (W1|W3) -> SwiGLU -> H            (forward GEMM 1)
  kGemmDown = 1,    // H x W2 -> gate * y                         (forward GEMM 2)
  kGemmBwdH = 2,    // dY x W2^T -> SwiGLU/statistic backward -> dS, dS3, dr partials
  kGemmBwdX = 3,    // [dS | dS3] x [W1 | W3]^T -> dX per kept row (fp32)
  kGemmWgradX = 4,  // x_perm^T x [dS | dS3] -> dW1 | dW3 (fp32), K = expert rows
  kGemmWgradH = 5,  // H^T x dY -> dW2 (fp32), K = expert rows
};

struct GemmArgs {
  int mode;
  int E, k, d;
  int bn;                   // N tile of the pair MMA: 128 or 256
  int rows;                 // rows of the permuted buffers
  const int32_t* offsets;   // [E+1] row-segment offsets (device)
  const int32_t* perm;      // [rows]; -1 marks a padding row
  const float* scale;       // up, bwd_h: r [T] (by token); down: gate [T*k] (by assignment)
  __nv_bfloat16* out;       // up: H [rows, ld_out]; down: y [rows, d]
  int ld_out;               // row stride of H-shaped buffers (max expert width)
  __nv_bfloat16* out_u;     // up, training: U = r*(x W1) [rows, ld_out] (may be null)
  __nv_bfloat16* out_v;     // up, training: V = r*(x W3)
  __nv_bfloat16* out_yu;    // down, training: ungated y [rows, d] (may be null)
  const __nv_bfloat16* in_u;  // bwd_h: U, V saved by the forward
  const __nv_bfloat16* in_v;
  __nv_bfloat16* out_ds;    // bwd_h: dS = r*du, dS3 = r*dv [rows, ld_out]
  __nv_bfloat16* out_ds3;
  float* drp;               // bwd_h: [rows, ld_drp] partials of dr, one per N tile
  int ld_drp;
  float* out_f0;            // bwd_x: dX [rows, d]; wgrad_x: dW1 [d, F]; wgrad_h: dW2 [F, d]
  float* out_f1;            // wgrad_x: dW3 [d, F]
  int ld_f;
  uint32_t* err;
  const uint32_t* wait_ctl;  // wait-limit control of the workspace header
  ExpertTable ffn;
  int to_token;             // down, k = 1: row p goes to row perm[p] (its token) of out [T, d]
  int staged;               // set by the launcher: epilogue tensor maps were given
  int epi8;                 // up / down: 8 epilogue warps (short reductions)
  int gather;               // up: A rows gathered from xg [T, d] (mapA0, one-row box) by perm[p] / k
};

struct CombineArgs {
  const __nv_bfloat16* y;
  const int32_t* inv_perm;
  __nv_bfloat16* out;
  int T, d, k;
};

// Backward elementwise / reduction stages (backward.cu).
struct BwdArgs {
  int T, d, E, k, renormalize;
  int rows;                       // rows of the padded permuted buffers
  const __nv_bfloat16* x;         // [T, d]
  const __nv_bfloat16* gamma;     // [d]
  const __nv_bfloat16* Wr;        // [d, E]
  const float* bias;              // [E] or null
  const __nv_bfloat16* dout;      // [T, d] upstream gradient
  const float* r;                 // [T] saved statistic
  const int32_t* idx;             // [T, k] saved routing
  const float* gate;              // [T, k]
  const float* logits;            // [T, E] saved fp32 logits (bias included)
  const int32_t* offsets;         // [E+1] padded row segments
  const int32_t* perm;            // [rows], -1 = padding
  const int32_t* inv_perm;        // [T*k], -1 = dropped
  const __nv_bfloat16* yu;        // [rows, d] saved ungated expert outputs
  __nv_bfloat16* dY;              // [rows, d] out: gate * dout of the row's token
  float* dgate;                   // [T*k] out: <dout_t, y_a> (kept slots only)
  const float* drp;               // [rows, ld_drp] dr partials of the bwd_h GEMM
  int ld_drp, bn_h;               // bn_h: N tile of that GEMM (partials per row = f_e / bn_h)
  const float* dXp;               // [rows, d] expert part of d(x*gamma) per kept row
  float* rdl;                     // [T, E] out: r_t * dl_t
  float* dr;                      // [T] out: dL/dr_t
  float* dbias_part;              // [route_blocks, E]
  int route_blocks;
  float* dx;                      // [T, d] out
  float* dgamma_part;             // [chunks, d]
  float* dWr_part;                // [chunks, d, E]
  int chunks, chunk_tokens;
  float* dgamma;                  // [d] out
  float* dWr;                     // [d, E] out
  float* dbias;                   // [E] out
  uint32_t* err;
  ExpertTable ffn;
};

cudaError_t launch_bwd_gather(const BwdArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_bwd_route(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_norm(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_reduce(const BwdArgs& a, cudaStream_t s);
constexpr int kBwdRouteTokens = 64;   // tokens per bwd_route CTA (8 warps x 8)
constexpr int kBwdNormCols = 128;     // columns per bwd_norm CTA
// Up / down GEMMs whose reduction is at most this long run 8 epilogue warps.
constexpr int kEpi8MaxK = 1024;

// Launchers (return the launch error, if any).
// xmap: x [T, d], boxes of 64 x 128 tokens; wmap: the [2 EP, d] hi/lo scratch,
// boxes of 64 x 2 EP (both 128-byte swizzled).
// With `xgmap` (may be null; box 64 x 32, 128-byte swizzle over a [T, d] bf16
// buffer) the router also writes xg = bf16(x * gamma) in token order.
cudaError_t launch_route(const RouteArgs& a, const CUtensorMap& xmap, const CUtensorMap& wmap,
                         const CUtensorMap* xgmap, cudaStream_t s);
int route_padded_experts(int E);  // EP: E rounded up to 8, 16, 32 or 64
cudaError_t launch_dispatch(const DispatchArgs& a, int num_sms, cudaStream_t s);
// Tensor maps of the epilogues that move their bf16 rows through shared
// memory by TMA (64-byte swizzle, 32 x 32 boxes over [rows, columns]):
//   up:    m[0] = H, m[1] = U, m[2] = V (U, V when kept)   [rows, ld_out]
//   down:  m[0] = y, m[1] = ungated y (when kept)          [rows, d]
//   bwd_h: m[0] = U, m[1] = V (loaded), m[2] = dS, m[3] = dS3 (stored)
//   bwd_x: m[0] = dX rows [rows, d];  wgrad_x: m[0] = dW1, m[1] = dW3 [d, F];
//   wgrad_h: m[0] = dW2 [F, d]  (these three fp32, 128-byte swizzle)
// Required by bwd_h; without them the other modes store row by row.
struct EpiMaps {
  CUtensorMap m[4];
};

// mapA1 is the second A operand (bwd_x: dS3); mapB1 the second B operand
// (up: W3; bwd_x: W3; wgrad_x: dS3).  Unused maps may repeat another.  `em`:
// see EpiMaps.
cudaError_t launch_grouped_gemm(const GemmArgs& a, const CUtensorMap& mapA0, const CUtensorMap& mapA1,
                                const CUtensorMap& mapB0, const CUtensorMap& mapB1, int grid,
                                cudaStream_t s, const EpiMaps* em = nullptr);
cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s);
// dst[0] = w0, dst[1] = w1 on the device, in stream order (one thread).
cudaError_t launch_set_words(uint32_t* dst, uint32_t w0, uint32_t w1, cudaStream_t s);
// stats[4] = {E*sum_e f_e*P_e, CV^2(P), CV^2(counts), dropped fraction}
cudaError_t launch_router_stats(const float* prob_mean, const int32_t* counts, const int32_t* offsets,
                                float* stats, int T, int E, int k, cudaStream_t s);
constexpr int kRouteTok = 128;  // tokens per router CTA

// One-time per-device kernel attributes (dynamic shared memory opt-in).
cudaError_t prepare_grouped_gemm();
// Persistent grid of the grouped GEMM: an even number of CTAs (pairs), at most
// the number of co-resident 2-CTA clusters times 2.
int grouped_gemm_max_grid(int num_sms);
size_t grouped_gemm_smem_bytes();

// Launch with programmatic stream serialization: the kernel's CTAs may start
// (and run their prologue up to griddep_wait, which every such kernel calls
// before touching global memory another kernel uses) while the previous
// kernel of the stream drains.  Used between the layer's consecutive kernels.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moe
