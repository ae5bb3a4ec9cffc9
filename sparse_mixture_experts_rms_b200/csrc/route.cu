// route.cu -- RMS statistic + router GEMM + fp32 softmax / top-k, one pass over x.
//
// CODA sparse-MoE thread (digg.com), RMSNorm paragraphs: the router is a plain
// GEMM right after the RMSNorm, and the scale by the statistic r commutes
// across it, so it is applied in the GEMM's epilogue right before the top-k:
//     l_te = r_t * sum_i x_ti * (gamma_i * Wr_ie) + b_e .
// MoE glossary (inferensys.com), "Top-k Gating" / "Switch Routing": the k
// largest router scores pick the experts; their softmax probabilities weight
// the expert outputs.
//
// One thread owns one token.  The token's row streams through L1 in 16-byte
// loads (the only pass over x); gamma*Wr is staged in shared memory in fp32
// chunks of 128 rows.  gamma_i*Wr_ie (two bf16) is exact in fp32, and so is
// x_ti times it, so the only rounding is the fp32 accumulation, done per
// 128-element chunk and then across chunks.  Sum of squares likewise.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRouteChunk = 128;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int EP, int TPB>
__global__ void __launch_bounds__(TPB) route_kernel(const RouteArgs a) {
  extern __shared__ __align__(16) float w_s[];  // [kRouteChunk][EP]
  const int t = blockIdx.x * TPB + threadIdx.x;
  const bool valid = t < a.T;
  const uint4* xrow = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(valid ? t : 0) * a.d);
  const uint16_t* gam = reinterpret_cast<const uint16_t*>(a.gamma);
  const uint16_t* wr = reinterpret_cast<const uint16_t*>(a.Wr);

  float acc[EP];
#pragma unroll
  for (int e = 0; e < EP; ++e) acc[e] = 0.f;
  float ss = 0.f;

  for (int c0 = 0; c0 < a.d; c0 += kRouteChunk) {
    __syncthreads();
    for (int i = threadIdx.x; i < kRouteChunk * EP; i += TPB) {
      const int row = i / EP, e = i % EP;
      float w = 0.f;
      if (e < a.E) {
        const float g = __uint_as_float(static_cast<uint32_t>(gam[c0 + row]) << 16);
        const float v = __uint_as_float(static_cast<uint32_t>(wr[static_cast<size_t>(c0 + row) * a.E + e]) << 16);
        w = g * v;  // exact: two 8-bit significands
      }
      w_s[i] = w;
    }
    __syncthreads();
    float part[EP];
#pragma unroll
    for (int e = 0; e < EP; ++e) part[e] = 0.f;
    float ssp = 0.f;
#pragma unroll 2
    for (int i = 0; i < kRouteChunk; i += 8) {
      float xv[8];
      bf16x8_to_f32(__ldg(xrow + (c0 + i) / 8), xv);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ssp = fmaf(xv[j], xv[j], ssp);
        const float4* wrow = reinterpret_cast<const float4*>(w_s + (i + j) * EP);
#pragma unroll
        for (int q = 0; q < EP / 4; ++q) {
          const float4 w = wrow[q];
          part[4 * q + 0] = fmaf(xv[j], w.x, part[4 * q + 0]);
          part[4 * q + 1] = fmaf(xv[j], w.y, part[4 * q + 1]);
          part[4 * q + 2] = fmaf(xv[j], w.z, part[4 * q + 2]);
          part[4 * q + 3] = fmaf(xv[j], w.w, part[4 * q + 3]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[e] += part[e];
    ss += ssp;
  }
  if (!valid) return;

  const float r = 1.0f / sqrtf(ss / static_cast<float>(a.d) + a.eps);
  float l[EP];
  float m = -INFINITY;
#pragma unroll
  for (int e = 0; e < EP; ++e) {
    if (e < a.E) {
      l[e] = fmaf(r, acc[e], a.bias ? a.bias[e] : 0.f);
      m = fmaxf(m, l[e]);
    } else {
      l[e] = -INFINITY;
    }
  }
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < EP; ++e)
    if (e < a.E) s += expf(l[e] - m);
  const float inv_s = 1.0f / s;

  if (a.logits) {
#pragma unroll
    for (int e = 0; e < EP; ++e)
      if (e < a.E) a.logits[static_cast<size_t>(t) * a.E + e] = l[e];
  }
  a.r[t] = r;

  // top-k: k rounds of a first-maximum scan (strict '>' keeps the lower index on ties)
  uint64_t used = 0;
  float gsum = 0.f;
  const size_t base = static_cast<size_t>(t) * a.k;
  for (int j = 0; j < a.k; ++j) {
    float best = -INFINITY;
    int bi = -1;
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      const bool free_e = e < a.E && !((used >> e) & 1ull);
      if (free_e && (bi < 0 || l[e] > best)) {
        best = l[e];
        bi = e;
      }
    }
    used |= 1ull << bi;
    const float g = expf(best - m) * inv_s;
    a.idx[base + j] = bi;
    a.gate[base + j] = g;
    gsum += g;
  }
  if (a.renormalize) {
    const float inv = 1.0f / gsum;
    for (int j = 0; j < a.k; ++j) a.gate[base + j] *= inv;
  }
}

template <int EP, int TPB>
cudaError_t launch_route_t(const RouteArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(kRouteChunk) * EP * sizeof(float);
  const int grid = (a.T + TPB - 1) / TPB;
  route_kernel<EP, TPB><<<grid, TPB, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  if (a.E <= 8) return launch_route_t<8, 64>(a, s);
  if (a.E <= 16) return launch_route_t<16, 64>(a, s);
  if (a.E <= 32) return launch_route_t<32, 64>(a, s);
  return launch_route_t<64, 64>(a, s);
}

}  // namespace moe
