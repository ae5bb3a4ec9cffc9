// route.cu -- RMS statistic + router GEMM + fp32 softmax / top-k, one pass over x.
//
// CODA sparse-MoE thread (digg.com), RMSNorm paragraphs: the router is a plain
// GEMM right after the RMSNorm, and the scale by the statistic r commutes
// across it, so it is applied in the GEMM's epilogue right before the top-k:
//     l_te = r_t * sum_i x_ti * w'_ie + b_e ,   w'_ie = gamma_i * Wr_ie .
// MoE glossary (inferensys.com), "Top-k Gating" / "Switch Routing": the k
// largest router scores pick the experts; their softmax probabilities weight
// the expert outputs.
//
// The contraction runs on the tensor cores (warp-level mma.sync m16n8k16,
// bf16 in, fp32 out) without losing the exactness routing needs:
//  - w' (two bf16 multiplied: 16 significant bits) is split exactly into
//    w' = hi + lo with hi, lo bf16 (8 bits each), so x*w' = x*hi + x*lo and
//    every product the tensor core forms is exact;
//  - each 64-element chunk is accumulated by the MMAs from zero (4 k-steps),
//    and the chunk partials are summed in fp64; r and l = r*acc + b are
//    formed in fp64 and each logit is rounded once to fp32.
// A near-tie between the k-th and (k+1)-th logit can therefore only flip when
// the two fp32 logits differ by about one ulp.
//
// Layout: a CTA (4 warps) owns 64 tokens, a warp 16.  x streams through a ring
// of stages, each a TMA tile [64 tokens x 64 elements] (128-byte swizzle;
// ldmatrix reads it conflict-free) plus the chunk's B fragments of hi/lo
// (precomputed once per call into the workspace, in the per-lane order the
// MMA wants, and fetched with one bulk copy).  The sum of squares for r comes
// from the same A fragments.  Logits meet in shared memory (rows padded to an
// odd word stride, so the per-token threads read them without bank conflicts),
// where one thread per token does the softmax and the top-k.
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kTok = kRouteTok;                // tokens per CTA
constexpr int kWarps = kTok / 16;              // a warp owns 16 tokens (MMA rows)
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 64;                     // elements of d per stage (4 k-steps)
constexpr int kTileBytes = kTok * kChunk * 2;  // 8 KB of x per stage

template <int EP>
struct RouteCfg {
  static constexpr int NT = EP / 8;                            // MMA n-tiles
  static constexpr int kFragBytes = 4 * NT * 2 * 32 * 8;       // k-steps x tiles x {hi,lo} x lanes x 8 B
  static constexpr int kStageBytes = kTileBytes + kFragBytes;  // a multiple of 1024
  static constexpr int kRing = EP <= 16 ? 6 : (EP == 32 ? 5 : 4);
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kRing) * kStageBytes + 64;
};

__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h));
}

// B fragments of hi(w') and lo(w') for every (k-step, n-tile, lane):
// b0 = {w'[k0][n], w'[k0+1][n]}, b1 = {w'[k0+8][n], w'[k0+9][n]},
// k0 = 16*ks + 2*(lane%4), n = 8*nt + lane/4 (zero for n >= E).
__global__ void router_weight_kernel(const RouteArgs a, int nt_count) {
  const int ksteps = a.d / 16;
  const int n = ksteps * nt_count * 2 * 32;
  const uint16_t* gam = reinterpret_cast<const uint16_t*>(a.gamma);
  const uint16_t* wr = reinterpret_cast<const uint16_t*>(a.Wr);
  uint2* out = reinterpret_cast<uint2*>(a.wprime);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int lane = i % 32;
    const int hl = (i / 32) % 2;
    const int nt = (i / 64) % nt_count;
    const int ks = i / (64 * nt_count);
    const int col = nt * 8 + lane / 4;
    const int k0 = ks * 16 + 2 * (lane % 4);
    uint32_t h16[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int kk = k0 + (j & 1) + (j >> 1) * 8;
      float w = 0.f;
      if (col < a.E) {
        const float g = __uint_as_float(static_cast<uint32_t>(gam[kk]) << 16);
        const float v = __uint_as_float(static_cast<uint32_t>(wr[static_cast<size_t>(kk) * a.E + col]) << 16);
        w = g * v;  // exact
      }
      const uint32_t hi = bf16_bits_rn(w);
      const float hif = __uint_as_float(hi << 16);
      h16[j] = hl == 0 ? hi : bf16_bits_rn(w - hif);  // w - hi is exact and fits in bf16
    }
    out[i] = make_uint2(h16[0] | (h16[1] << 16), h16[2] | (h16[3] << 16));
  }
}

template <int EP>
__device__ __forceinline__ void route_token(const RouteArgs& a, float* lg, float rtok, int t,
                                            bool keep_probs);

template <int EP>
__global__ void __launch_bounds__(kThreads) route_kernel(const __grid_constant__ CUtensorMap xmap,
                                                         const RouteArgs a) {
  using Cfg = RouteCfg<EP>;
  constexpr int NT = Cfg::NT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + Cfg::kRing * Cfg::kStageBytes);
  int* abort_flag = reinterpret_cast<int*>(full + Cfg::kRing);
  uint32_t* dummy_err = reinterpret_cast<uint32_t*>(abort_flag + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kTok;
  uint32_t* err = a.err ? a.err : dummy_err;
  const int nchunks = a.d / kChunk;
  const uint64_t wait_ns = wait_limit_ns(a.wait_ctl);  // the stage waits' limit (workspace header)
  const uint8_t* frag_src = reinterpret_cast<const uint8_t*>(a.wprime);

  auto issue = [&](int c, int s) {
    uint8_t* st = ring + s * Cfg::kStageBytes;
    mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
    tma_load_2d(st, &xmap, &full[s], c * kChunk, t0);
    bulk_load(st + kTileBytes, frag_src + static_cast<size_t>(c) * Cfg::kFragBytes, Cfg::kFragBytes, &full[s]);
  };

  if (tid == 0) {
    for (int s = 0; s < Cfg::kRing; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    *dummy_err = 0;
    fence_mbar_init();
    tma_prefetch_map(&xmap);
  }
  __syncthreads();
  if (tid == 0)
    for (int c = 0; c < Cfg::kRing && c < nchunks; ++c) issue(c, c);

  // accumulators: this lane's C elements (rows g, g+8; columns 2t, 2t+1 of each n-tile)
  double acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0;
  double ss_g = 0.0, ss_g8 = 0.0;
  bool ok = true;

  // ldmatrix row address of this lane: matrix m = lane/8 -> rows +8*(m&1), k piece +(m>>1)
  const int lrow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int lpiece = lane >> 4;

  int stop = nchunks;  // chunks consumed
  for (int c = 0; c < nchunks; ++c) {
    const int s = c % Cfg::kRing;
    const uint32_t ph = (c / Cfg::kRing) & 1u;
    ok = mbar_wait(&full[s], ph, abort_flag, err, MOE_DEVERR_TIMEOUT, wait_ns);
    if (ok) {
      const uint8_t* st = ring + s * Cfg::kStageBytes;
      const uint2* frag = reinterpret_cast<const uint2*>(st + kTileBytes);
      const uint32_t tile = smem_addr(st);
      float chi[NT][4], clo[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) chi[nt][i] = clo[nt][i] = 0.f;
      float sg = 0.f, sg8 = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int piece = 2 * kk + lpiece;
        uint32_t av[4];
        ldmatrix_x4(tile + lrow * 128 + ((piece ^ (lrow & 7)) << 4), av);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(av[i] << 16), hi = __uint_as_float(av[i] & 0xFFFF0000u);
          if (i & 1) {
            sg8 = fmaf(lo, lo, sg8);
            sg8 = fmaf(hi, hi, sg8);
          } else {
            sg = fmaf(lo, lo, sg);
            sg = fmaf(hi, hi, sg);
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint2 bh = frag[((kk * NT + nt) * 2 + 0) * 32 + lane];
          const uint2 bl = frag[((kk * NT + nt) * 2 + 1) * 32 + lane];
          mma_bf16_16816(chi[nt], av, bh.x, bh.y);
          mma_bf16_16816(clo[nt], av, bl.x, bl.y);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] += static_cast<double>(chi[nt][i]) + static_cast<double>(clo[nt][i]);
      ss_g += static_cast<double>(sg);
      ss_g8 += static_cast<double>(sg8);
    }
    // every warp is done with stage s; a wait that gave up anywhere stops the CTA
    ok = __syncthreads_and(ok) != 0;
    if (!ok) {
      stop = c;
      break;
    }
    if (tid == 0 && c + Cfg::kRing < nchunks) issue(c + Cfg::kRing, s);
  }
  if (!ok) {
    // chunks [stop, stop + ring) were issued but not consumed: let them land
    // (default limit: issued copies always finish) before exiting
    if (tid == 0) {
      volatile int no_abort = 0;
      for (int c = stop; c < nchunks && c < stop + Cfg::kRing; ++c)
        mbar_wait(&full[c % Cfg::kRing], (c / Cfg::kRing) & 1u, &no_abort, err, MOE_DEVERR_TIMEOUT,
                  kWaitTimeoutNs);
    }
    return;
  }

  // sum of squares of rows g and g+8 over the quad's columns
#pragma unroll
  for (int m = 1; m <= 2; m <<= 1) {
    ss_g += __shfl_xor_sync(0xFFFFFFFFu, ss_g, m);
    ss_g8 += __shfl_xor_sync(0xFFFFFFFFu, ss_g8, m);
  }
  const int g = lane >> 2, tq = lane & 3;
  const int row_g = warp * 16 + g, row_g8 = row_g + 8;
  const double inv_d = 1.0 / static_cast<double>(a.d);
  const double r_g = 1.0 / sqrt(ss_g * inv_d + static_cast<double>(a.eps));
  const double r_g8 = 1.0 / sqrt(ss_g8 * inv_d + static_cast<double>(a.eps));

  // logits of the CTA's 64 tokens meet in shared memory (the ring is idle now)
  float* lg = reinterpret_cast<float*>(ring);
  constexpr int LS = EP + 1;  // logit row stride in words: odd, so one token per bank
  static_assert((kTok * LS + kTok) * 4 <= Cfg::kRing * Cfg::kStageBytes, "logits exceed the idle ring");
  float* rr = lg + kTok * LS;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = nt * 8 + 2 * tq + (i & 1);
      const int row = (i < 2) ? row_g : row_g8;
      const double rv = (i < 2) ? r_g : r_g8;
      const double b = (a.bias != nullptr && e < a.E) ? static_cast<double>(a.bias[e]) : 0.0;
      lg[row * LS + e] = e < a.E ? static_cast<float>(fma(rv, acc[nt][i], b)) : -INFINITY;
    }
  }
  if (tq == 0) {
    rr[row_g] = static_cast<float>(r_g);
    rr[row_g8] = static_cast<float>(r_g8);
  }
  __syncthreads();
  const int t = t0 + tid;
  if (tid < kTok && t < a.T) route_token<EP>(a, lg + tid * LS, rr[tid], t, a.prob_mean != nullptr);
  else if (tid < kTok && a.prob_mean != nullptr)
    for (int e = 0; e < EP; ++e) lg[tid * LS + e] = 0.f;  // rows past T add nothing
  if (a.prob_mean == nullptr) return;

  // Router metric in the epilogue: this CTA's probability sums, then the last
  // CTA to finish sums every CTA's partials in CTA order (deterministic).
  __shared__ int is_last;
  __syncthreads();
  if (tid < a.E) {
    float sum = 0.f;
    for (int i = 0; i < kTok; ++i) sum += lg[i * LS + tid];
    a.prob_partial[static_cast<size_t>(blockIdx.x) * a.E + tid] = sum;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (tid < a.E) {
    double sum = 0.0;
    for (unsigned c = 0; c < gridDim.x; ++c)
      sum += static_cast<double>(__ldcg(a.prob_partial + static_cast<size_t>(c) * a.E + tid));
    a.prob_mean[tid] = static_cast<float>(sum / static_cast<double>(a.T));
  }
}

// Softmax and top-k of one token from its fp32 logits (row of `lg`).  With
// `keep_probs`, the row is overwritten with the token's softmax probabilities.
template <int EP>
__device__ __forceinline__ void route_token(const RouteArgs& a, float* lg, float rtok, int t,
                                            bool keep_probs) {
  float l[EP];
  float m = -INFINITY;
#pragma unroll
  for (int e = 0; e < EP; ++e) {
    l[e] = lg[e];
    if (e < a.E) m = fmaxf(m, l[e]);
  }
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < EP; ++e)
    if (e < a.E) sum += expf(l[e] - m);
  const float inv_s = 1.0f / sum;

  if (a.logits) {
#pragma unroll
    for (int e = 0; e < EP; ++e)
      if (e < a.E) a.logits[static_cast<size_t>(t) * a.E + e] = l[e];
  }
  a.r[t] = rtok;
  if (keep_probs) {
#pragma unroll
    for (int e = 0; e < EP; ++e) lg[e] = e < a.E ? expf(l[e] - m) * inv_s : 0.f;
  }

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
    const float gt = expf(best - m) * inv_s;
    a.idx[base + j] = bi;
    a.gate[base + j] = gt;
    gsum += gt;
  }
  if (a.renormalize) {
    const float inv = 1.0f / gsum;
    for (int j = 0; j < a.k; ++j) a.gate[base + j] *= inv;
  }
}

template <int EP>
cudaError_t launch_route_t(const RouteArgs& a, const CUtensorMap& xmap, cudaStream_t s) {
  const size_t smem = RouteCfg<EP>::kSmem;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<EP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int n = (a.d / 16) * RouteCfg<EP>::NT * 64;
  router_weight_kernel<<<(n + 255) / 256, 256, 0, s>>>(a, RouteCfg<EP>::NT);
  const int grid = (a.T + kTok - 1) / kTok;
  route_kernel<EP><<<grid, kThreads, smem, s>>>(xmap, a);
  return cudaGetLastError();
}

// Load-balance metrics from the router's prob_mean and the dispatch counts:
// stats = {E * sum_e f_e * P_e, CV^2(P), CV^2(counts), dropped fraction},
// f_e = counts_e / (T*k), CV^2 with the population variance, in fp64.
__global__ void router_stats_kernel(const float* P, const int32_t* counts, const int32_t* offsets,
                                    float* stats, int T, int E, int k) {
  __shared__ double sp[kMaxExperts], sc[kMaxExperts];
  const int e = threadIdx.x;
  if (e < E) {
    sp[e] = static_cast<double>(P[e]);
    sc[e] = static_cast<double>(counts[e]);
  }
  __syncthreads();
  if (e != 0) return;
  const double tk = static_cast<double>(T) * k;
  double aux = 0.0, mp = 0.0, mc = 0.0;
  for (int i = 0; i < E; ++i) {
    aux += (sc[i] / tk) * sp[i];
    mp += sp[i];
    mc += sc[i];
  }
  mp /= E;
  mc /= E;
  double vp = 0.0, vc = 0.0;
  for (int i = 0; i < E; ++i) {
    vp += (sp[i] - mp) * (sp[i] - mp);
    vc += (sc[i] - mc) * (sc[i] - mc);
  }
  vp /= E;
  vc /= E;
  stats[0] = static_cast<float>(E * aux);
  stats[1] = static_cast<float>(mp != 0.0 ? vp / (mp * mp) : 0.0);
  stats[2] = static_cast<float>(mc != 0.0 ? vc / (mc * mc) : 0.0);
  stats[3] = static_cast<float>(1.0 - static_cast<double>(offsets[E]) / tk);
}

}  // namespace

cudaError_t launch_router_stats(const float* prob_mean, const int32_t* counts, const int32_t* offsets,
                                float* stats, int T, int E, int k, cudaStream_t s) {
  router_stats_kernel<<<1, kMaxExperts, 0, s>>>(prob_mean, counts, offsets, stats, T, E, k);
  return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& a, const CUtensorMap& xmap, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  if (a.E <= 8) return launch_route_t<8>(a, xmap, s);
  if (a.E <= 16) return launch_route_t<16>(a, xmap, s);
  if (a.E <= 32) return launch_route_t<32>(a, xmap, s);
  return launch_route_t<64>(a, xmap, s);
}

}  // namespace moe
