// moe_internal.h -- launchers shared between the C ABI (moe_api.cu) and the
// kernel translation units.  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

constexpr int kMaxExperts = 64;
constexpr int kRouterPadE = 64;         // w' scratch is sized for the widest router variant
constexpr int kBlockN = 128;            // expert width granule (and G1's N per projection)
constexpr int kDispatchTile = 1024;     // assignments per dispatch CTA
constexpr uint64_t kWaitTimeoutNs = 4000000000ull;  // bounded pipeline waits: 4 s

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
  float* wprime;      // [d, EP] fp32 scratch: gamma * Wr, zero-padded
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
  int32_t* tile_counts;     // [ntiles, E] scratch
  int32_t* counts;          // [E]
  int32_t* offsets;         // [E+1]
  int32_t* perm;            // [T*k]
  int32_t* inv_perm;        // [T*k]
  __nv_bfloat16* x_perm;    // [max_kept, d]
  uint32_t* err;
  int T, d, E, k;
  int capacity;             // -1: dropless
  int max_kept;             // rows of x_perm
};

struct GemmArgs {
  int up;                   // 1: x_perm x (W1|W3) -> SwiGLU -> H; 0: H x W2 -> y
  int E, k, d;
  int bn;                   // N tile: 256 for up (128 of W1 + 128 of W3); 128/256 for down
  int rows;                 // rows of the A operand buffer (max kept)
  const int32_t* offsets;   // [E+1] kept-row offsets (device)
  const int32_t* perm;      // [max_kept]
  const float* scale;       // up: r [T] (indexed by token); down: gate [T*k] (by assignment)
  __nv_bfloat16* out;       // up: H [rows, ld_out]; down: y [rows, d]
  int ld_out;
  uint32_t* err;
  ExpertTable ffn;
};

struct CombineArgs {
  const __nv_bfloat16* y;
  const int32_t* inv_perm;
  __nv_bfloat16* out;
  int T, d, k;
};

// Launchers (return the launch error, if any).
cudaError_t launch_route(const RouteArgs& a, const CUtensorMap& xmap, cudaStream_t s);
cudaError_t launch_dispatch(const DispatchArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_grouped_gemm(const GemmArgs& a, const CUtensorMap& mapA,
                                const CUtensorMap& mapB0, const CUtensorMap& mapB1, int grid,
                                cudaStream_t s);
cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s);
// stats[4] = {E*sum_e f_e*P_e, CV^2(P), CV^2(counts), dropped fraction}
cudaError_t launch_router_stats(const float* prob_mean, const int32_t* counts, const int32_t* offsets,
                                float* stats, int T, int E, int k, cudaStream_t s);
constexpr int kRouteTok = 64;  // tokens per router CTA

// One-time per-device kernel attributes (dynamic shared memory opt-in).
cudaError_t prepare_grouped_gemm();
// Persistent grid of the grouped GEMM: an even number of CTAs (pairs), at most
// the number of co-resident 2-CTA clusters times 2.
int grouped_gemm_max_grid(int num_sms);
size_t grouped_gemm_smem_bytes();

}  // namespace moe
