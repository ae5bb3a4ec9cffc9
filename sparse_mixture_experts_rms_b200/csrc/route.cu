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
// The contraction runs on the 5th-generation tensor cores (tcgen05.mma,
// cta_group::1, M = 128 tokens, N = 2 EP, bf16 in, fp32 in TMEM) without
// losing the exactness routing needs:
//  - w' (two bf16 multiplied: 16 significant bits) is split exactly into
//    w' = hi + lo with hi, lo bf16 (8 bits each), so x*w' = x*hi + x*lo and
//    every product the tensor core forms is exact; B = [hi | lo] holds the
//    two halves as 2 EP columns (EP = E rounded up to 8, 16, 32 or 64);
//  - each 64-element chunk of d is accumulated by 4 MMAs from zero into its
//    own TMEM buffer, so no fp32 sum runs over more than 64 products; the
//    epilogue adds the hi and lo partials of a stage's 2-4 chunks in fp32
//    and the stage sums in fp64; r and l = r*acc + b are formed in fp64 and
//    each logit is rounded once to fp32.
// The logit's error is a few fp32 roundings of 64-product partial sums, far
// below the 1e-5 margin within which a near-tie of the k-th and (k+1)-th
// logit is treated as either order.
//
// Layout: a CTA owns 128 tokens.  Warp 0 streams x through a ring of stages
// by TMA, each [128 tokens x 64 elements] (128-byte swizzle) plus the chunk's
// B tile [2 EP x 64] of hi/lo (precomputed once per call into the workspace,
// K-major); warp 1 issues the MMAs; warps 2-5 (one per TMEM lane quarter, a
// thread per token) read each chunk's partials from TMEM, add the sum of
// squares of their token's 64 elements from the staged x tile (for r), and
// release the stage.  After the last chunk each thread has its token's fp64
// logit sums and sum of squares; logits meet in shared memory (rows padded to
// an odd word stride, so per-token threads read them without bank conflicts),
// where each thread does its token's softmax and top-k.
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kTok = kRouteTok;                // tokens per CTA (the MMA's M)
constexpr int kChunk = 64;                     // elements of d per fp32 partial (4 MMAs of K = 16)
constexpr int kTileBytes = kTok * kChunk * 2;  // 16 KB of x per chunk
constexpr int kGroups = 2;                     // TMEM buffer groups (one stage's chunks each)
constexpr int kMaxStages = 8;

template <int EP>
struct RouteCfg {
  static constexpr int N = 2 * EP;                             // MMA N: hi and lo columns
  // epilogue warps: one per TMEM lane quarter, or two (each on half of the
  // experts and half of the row's sum of squares) when the fp64 chunk sums of
  // 32 or 64 experts would bound the kernel
  static constexpr int kEpi = EP >= 32 ? 8 : 4;
  static constexpr int kEP = EP / (kEpi / 4);                  // experts per epilogue thread
  static constexpr int kThreads = 64 + 32 * kEpi;
  static constexpr int kBBytes = N * kChunk * 2;               // B tile of a chunk: a multiple of 1024
  // A stage carries several chunks (their x tiles side by side along d, so a
  // row's 256-512 contiguous bytes are fetched together, and one MMA commit /
  // epilogue hand-off per stage); each chunk still gets its own TMEM buffer.
  static constexpr int kCps = EP <= 8 ? 4 : 2;                 // chunks per stage
  static constexpr int kStageBytes = kCps * (kTileBytes + kBBytes);
  static constexpr int kStages = (220 * 1024) / kStageBytes < kMaxStages ? (220 * 1024) / kStageBytes : kMaxStages;
  static constexpr uint32_t kTmemCols = kGroups * kCps * N < 32 ? 32u : static_cast<uint32_t>(kGroups * kCps * N);
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kStages) * kStageBytes + 512;
};

struct __align__(8) RouteShared {
  uint64_t full[kMaxStages];   // the stage's x and B tiles landed
  uint64_t empty[kMaxStages];  // the MMAs and the epilogue's sums of squares are done with the stage
  uint64_t tfull[kGroups];     // a stage's chunk partials are in the TMEM buffer group
  uint64_t tempty[kGroups];    // the epilogue read the group
  uint64_t drain;
  uint64_t xg_ready[4];        // with xg and 8 epilogue warps: both warps of a lane quarter rewrote their pieces
  uint32_t tmem_base;
  int abort_flag;
  uint32_t dummy_err;
  int is_last;
};

__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h));
}

// B = (gamma * Wr)^T split exactly into bf16 hi (rows [0, EP)) and lo (rows
// [EP, 2 EP)), K-major [2 EP, d]; experts n >= E are zero rows.
__global__ void router_weight_kernel(const RouteArgs a, int ep) {
  griddep_launch_dependents();  // the router may launch and set up meanwhile
  const int n = 2 * ep * a.d;
  const uint16_t* gam = reinterpret_cast<const uint16_t*>(a.gamma);
  const uint16_t* wr = reinterpret_cast<const uint16_t*>(a.Wr);
  uint16_t* out = reinterpret_cast<uint16_t*>(a.wprime);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int row = i / a.d, kk = i - row * a.d;
    const int col = row < ep ? row : row - ep;
    float w = 0.f;
    if (col < a.E) {
      const float g = __uint_as_float(static_cast<uint32_t>(gam[kk]) << 16);
      const float v = __uint_as_float(static_cast<uint32_t>(wr[static_cast<size_t>(kk) * a.E + col]) << 16);
      w = g * v;  // exact
    }
    const uint32_t hi = bf16_bits_rn(w);
    out[i] = static_cast<uint16_t>(row < ep ? hi : bf16_bits_rn(w - __uint_as_float(hi << 16)));  // w - hi is exact
  }
}

// 32 lanes x 16 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

// 32 lanes x 8 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}

template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[NC]) {
  if constexpr (NC == 8) tmem_ld_32x32b_x8(taddr, v);
  else if constexpr (NC == 16) tmem_ld_32x32b_x16(taddr, v);
  else tmem_ld_32x32b_x32(taddr, v);
}

// sum[e] += hi_e + lo_e (fp32) for NE experts whose chunk partials sit in
// TMEM columns [thi, thi + NE) (hi) and [tlo, tlo + NE) (lo) of this warp's
// lane quarter.
template <int NE>
__device__ __forceinline__ void add_chunk(uint32_t thi, uint32_t tlo, float (&sum)[NE]) {
  static_assert(NE == 8 || NE == 16 || NE == 32, "8, 16 or 32 experts per epilogue thread");
  constexpr int P = NE < 16 ? NE : 16;  // columns per load (bounds the registers in flight)
#pragma unroll
  for (int e0 = 0; e0 < NE; e0 += P) {
    uint32_t h[P], l[P];
    tmem_ld_cols<P>(thi + e0, h);
    tmem_ld_cols<P>(tlo + e0, l);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < P; ++e) sum[e0 + e] += __uint_as_float(h[e]) + __uint_as_float(l[e]);
  }
}

template <int EP>
__device__ __forceinline__ void route_token(const RouteArgs& a, float* lg, float rtok, int t,
                                            bool keep_probs);

template <int EP, bool XG>
__global__ void __launch_bounds__(RouteCfg<EP>::kThreads, 1)
    route_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                 const __grid_constant__ CUtensorMap xgmap, const RouteArgs a) {
  using Cfg = RouteCfg<EP>;
  constexpr int N = Cfg::N;
  constexpr int EPI = Cfg::kEpi;
  constexpr int NE = Cfg::kEP;          // experts per epilogue thread
  constexpr int NJ = 8 / (EPI / 4);     // 16-byte pieces of a row's 64 elements per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RouteShared& sh = *reinterpret_cast<RouteShared*>(ring + Cfg::kStages * Cfg::kStageBytes);
  static_assert(Cfg::kStages >= 2 && Cfg::kStages <= kMaxStages, "stage count");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kTok;
  const int nchunks = a.d / kChunk;
  const uint64_t wait_ns = wait_limit_ns(a.wait_ctl);  // the pipeline waits' limit (workspace header)

  if (tid == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1 + EPI);  // MMA commit + the epilogue warps
    }
    for (int g = 0; g < kGroups; ++g) {
      mbar_init(&sh.tfull[g], 1);
      mbar_init(&sh.tempty[g], EPI);
    }
    mbar_init(&sh.drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&sh.xg_ready[i], 2);
    sh.abort_flag = 0;
    sh.dummy_err = 0;
    fence_mbar_init();
    tma_prefetch_map(&xmap);
    tma_prefetch_map(&wmap);
    if (XG) tma_prefetch_map(&xgmap);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the split router weights come from router_weight_kernel
  uint32_t* err = a.err ? a.err : &sh.dummy_err;
  volatile int* abort_flag = &sh.abort_flag;
  const uint32_t tmem_base = sh.tmem_base;

  double acc[NE];
#pragma unroll
  for (int e = 0; e < NE; ++e) acc[e] = 0.0;
  double ss = 0.0;
  bool ok = true;
  const int q = warp & 3;                     // TMEM lane quarter of an epilogue warp
  const int half = warp >= 2 ? (warp - 2) / 4 : 0;  // which half of the experts (8 epilogue warps)
  const int row = q * 32 + lane;              // token row of an epilogue thread

  constexpr int S = Cfg::kStages, CPS = Cfg::kCps;
  const int nst = (nchunks + CPS - 1) / CPS;  // stages; the last one may hold fewer chunks
  auto chunks_of = [&](int st) { return nchunks - st * CPS < CPS ? nchunks - st * CPS : CPS; };
  if (warp == 0) {
    // ================= TMA producer
    if (lane == 0) {
      int st = 0;
      for (; st < nst; ++st) {
        const int s = st % S, nc = chunks_of(st);
        if (!mbar_wait(&sh.empty[s], ((st / S) & 1u) ^ 1u, abort_flag, err, MOE_DEVERR_TIMEOUT, wait_ns)) break;
        uint8_t* xs = ring + s * Cfg::kStageBytes;
        uint8_t* bs = xs + CPS * kTileBytes;
        mbar_arrive_expect_tx(&sh.full[s], static_cast<uint32_t>(nc * (kTileBytes + Cfg::kBBytes)));
        for (int i = 0; i < nc; ++i) {
          const int kx = (st * CPS + i) * kChunk;
          tma_load_2d(xs + i * kTileBytes, &xmap, &sh.full[s], kx, t0);
          tma_load_2d(bs + i * Cfg::kBBytes, &wmap, &sh.full[s], kx, 0);
        }
      }
      // the copies still in flight land before the CTA goes on (default limit)
      volatile int no_abort = 0;
      for (int j = st > S ? st - S : 0; j < st; ++j)
        mbar_wait(&sh.full[j % S], (j / S) & 1u, &no_abort, err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
    }
  } else if (warp == 1) {
    // ================= MMA issuer: chunk i of a stage goes to TMEM buffer g*CPS + i
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kTok, N, 0u, 0u);  // A and B K-major
      for (int st = 0; st < nst; ++st) {
        const int s = st % S, g = st % kGroups, nc = chunks_of(st);
        if (!mbar_wait(&sh.full[s], (st / S) & 1u, abort_flag, err, MOE_DEVERR_TIMEOUT, wait_ns) ||
            !mbar_wait(&sh.tempty[g], ((st / kGroups) & 1u) ^ 1u, abort_flag, err, MOE_DEVERR_TIMEOUT, wait_ns))
          break;
        tc_fence_after();
        const uint32_t aX = smem_addr(ring + s * Cfg::kStageBytes);
        const uint32_t aB = aX + CPS * kTileBytes;
        for (int i = 0; i < nc; ++i) {
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((g * CPS + i) * N);
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk)
            umma_bf16(d_tmem, smem_desc_sw128(aX + i * kTileBytes + kk * 32, 16, 1024),
                      smem_desc_sw128(aB + i * Cfg::kBBytes + kk * 32, 16, 1024), idesc, kk != 0 ? 1u : 0u);
        }
        umma_commit(&sh.empty[s]);
        umma_commit(&sh.tfull[g]);
      }
      umma_commit(&sh.drain);
      volatile int no_abort = 0;
      mbar_wait(&sh.drain, 0, &no_abort, err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
    }
  } else {
    // ================= epilogue: thread = token row (TMEM lane q*32 + lane);
    // experts [half*NE, half*NE + NE) and pieces [half*NJ, half*NJ + NJ) of each chunk's row
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + half * NE;
    for (int st = 0; st < nst; ++st) {
      const int s = st % S, g = st % kGroups, nc = chunks_of(st);
      ok = mbar_wait(&sh.full[s], (st / S) & 1u, abort_flag, err, MOE_DEVERR_TIMEOUT, wait_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      // sum of squares of this thread's pieces of its token's elements
      // (128-byte swizzled rows), one independent accumulator per piece
      float sq[CPS * NJ];
#pragma unroll
      for (int i = 0; i < CPS; ++i) {
        const uint8_t* xr = ring + s * Cfg::kStageBytes + i * kTileBytes + row * 128;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          float acc_j = 0.f;
          if (i < nc) {
            const int jj = half * NJ + j;
            const uint4 v = *reinterpret_cast<const uint4*>(xr + ((jj ^ (row & 7)) << 4));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float lo = __uint_as_float(w4[u] << 16), hi = __uint_as_float(w4[u] & 0xFFFF0000u);
              acc_j = fmaf(lo, lo, acc_j);
              acc_j = fmaf(hi, hi, acc_j);
            }
          }
          sq[i * NJ + j] = acc_j;
        }
      }
      ok = mbar_wait(&sh.tfull[g], (st / kGroups) & 1u, abort_flag, err, MOE_DEVERR_TIMEOUT, wait_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      // the stage's 2 * nc partials of each logit meet in fp32 (a few fp32
      // roundings of the partials' size, like the MMA's own accumulation),
      // and the stage sum goes into the fp64 accumulator: one fp64 conversion
      // per expert and stage, not two per chunk
      float stage_sum[NE];
#pragma unroll
      for (int e = 0; e < NE; ++e) stage_sum[e] = 0.f;
      for (int i = 0; i < nc; ++i) {
        const uint32_t tb = tq + static_cast<uint32_t>((g * CPS + i) * N);
        add_chunk<NE>(tb, tb + EP, stage_sum);
      }
#pragma unroll
      for (int e = 0; e < NE; ++e) acc[e] += static_cast<double>(stage_sum[e]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tempty[g]);
      if constexpr (XG) {
        // The stage's MMAs are complete (tfull), so its x tiles may change:
        // this thread's pieces become bf16(x * gamma) in place, and one warp
        // of the lane quarter stores the quarter's 32 rows of every chunk to
        // xg by TMA before the stage goes back to the producer.
        uint8_t* xs = ring + s * Cfg::kStageBytes;
        const uint4* g4 = reinterpret_cast<const uint4*>(a.gamma);
        for (int i = 0; i < nc; ++i) {
          uint8_t* xr = xs + i * kTileBytes + row * 128;
          const int kx8 = (st * CPS + i) * (kChunk / 8);
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const int jj = half * NJ + j;
            uint4* pv = reinterpret_cast<uint4*>(xr + ((jj ^ (row & 7)) << 4));
            const uint4 v = *pv, gv = __ldg(g4 + kx8 + jj);
            const uint32_t xw[4] = {v.x, v.y, v.z, v.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t o[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float lo = __uint_as_float(xw[u] << 16) * __uint_as_float(gw[u] << 16);
              const float hi = __uint_as_float(xw[u] & 0xFFFF0000u) * __uint_as_float(gw[u] & 0xFFFF0000u);
              const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
              o[u] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *pv = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        bool stored = true;
        if (EPI == 8) {
          // the other warp of the quarter holds the rest of each row
          if (lane == 0) mbar_arrive(&sh.xg_ready[q]);
          if (half == 0) {
            int got = 1;
            if (lane == 0)
              got = mbar_wait(&sh.xg_ready[q], st & 1u, abort_flag, err, MOE_DEVERR_TIMEOUT, wait_ns) ? 1 : 0;
            stored = __shfl_sync(0xFFFFFFFFu, got, 0) != 0;
          }
        }
        if (stored && half == 0 && lane == 0 && t0 + q * 32 < a.T) {
          for (int i = 0; i < nc; ++i)
            tma_store_2d(&xgmap, xs + i * kTileBytes + q * 32 * 128, (st * CPS + i) * kChunk, t0 + q * 32);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
        __syncwarp();
        if (!stored) {
          ok = false;
          break;
        }
      }
      if (lane == 0) mbar_arrive(&sh.empty[s]);
      float sqs = 0.f;
#pragma unroll
      for (int j = 0; j < CPS * NJ; ++j) sqs += sq[j];
      ss += static_cast<double>(sqs);
    }
    if (XG && half == 0 && lane == 0) bulk_wait_group0();  // xg written before the kernel ends
  }
  ok = __syncthreads_and(ok && !*abort_flag) != 0;
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
  if (!ok) return;  // a wait gave up: the error word says so, outputs are undefined

  // logits of the CTA's tokens meet in shared memory (the ring is idle now)
  float* lg = reinterpret_cast<float*>(ring);
  constexpr int LS = EP + 1;  // logit row stride in words: odd, so one token per bank
  static_assert((kTok * LS + 1 + 4 * kTok) * 4 <= Cfg::kStages * Cfg::kStageBytes, "logits exceed the idle ring");
  double* ssp = reinterpret_cast<double*>(lg + kTok * LS + (kTok * LS) % 2);  // [2][kTok] partial sums of squares
  const bool keep_probs = a.prob_mean != nullptr;
  if (warp >= 2) ssp[half * kTok + row] = ss;
  __syncthreads();
  if (warp >= 2) {
    const double sst = EPI == 8 ? ssp[row] + ssp[kTok + row] : ssp[row];
    const double rv = 1.0 / sqrt(sst / static_cast<double>(a.d) + static_cast<double>(a.eps));
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      const int ex = half * NE + e;
      const double bb = (a.bias != nullptr && ex < a.E) ? static_cast<double>(a.bias[ex]) : 0.0;
      lg[row * LS + ex] = ex < a.E ? static_cast<float>(fma(rv, acc[e], bb)) : -INFINITY;
    }
  }
  __syncthreads();
  if (warp >= 2 && half == 0) {
    const double sst = EPI == 8 ? ssp[row] + ssp[kTok + row] : ssp[row];
    const float rv = static_cast<float>(1.0 / sqrt(sst / static_cast<double>(a.d) + static_cast<double>(a.eps)));
    const int t = t0 + row;
    if (t < a.T) route_token<EP>(a, lg + row * LS, rv, t, keep_probs);
    else if (keep_probs)
      for (int e = 0; e < EP; ++e) lg[row * LS + e] = 0.f;  // rows past T add nothing
  }
  if (!keep_probs) return;

  // Router metric in the epilogue: this CTA's probability sums, then the last
  // CTA to finish sums every CTA's partials in CTA order (deterministic).
  __syncthreads();
  if (tid < a.E) {
    float sum = 0.f;
    for (int i = 0; i < kTok; ++i) sum += lg[i * LS + tid];
    a.prob_partial[static_cast<size_t>(blockIdx.x) * a.E + tid] = sum;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.is_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!sh.is_last) return;
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

template <int EP, bool XG>
cudaError_t launch_route_t(const RouteArgs& a, const CUtensorMap& xmap, const CUtensorMap& wmap,
                           const CUtensorMap& xgmap, cudaStream_t s) {
  const size_t smem = RouteCfg<EP>::kSmem;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<EP, XG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int n = 2 * EP * a.d;
  router_weight_kernel<<<(n + 255) / 256, 256, 0, s>>>(a, EP);
  const int grid = (a.T + kTok - 1) / kTok;
  return launch_pdl(route_kernel<EP, XG>, dim3(grid), dim3(RouteCfg<EP>::kThreads), smem, s, xmap, wmap, xgmap, a);
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

int route_padded_experts(int E) { return E <= 8 ? 8 : (E <= 16 ? 16 : (E <= 32 ? 32 : 64)); }

cudaError_t launch_route(const RouteArgs& a, const CUtensorMap& xmap, const CUtensorMap& wmap,
                         const CUtensorMap* xgmap, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  if (xgmap != nullptr) {
    switch (route_padded_experts(a.E)) {
      case 8: return launch_route_t<8, true>(a, xmap, wmap, *xgmap, s);
      case 16: return launch_route_t<16, true>(a, xmap, wmap, *xgmap, s);
      case 32: return launch_route_t<32, true>(a, xmap, wmap, *xgmap, s);
      default: return launch_route_t<64, true>(a, xmap, wmap, *xgmap, s);
    }
  }
  switch (route_padded_experts(a.E)) {
    case 8: return launch_route_t<8, false>(a, xmap, wmap, xmap, s);
    case 16: return launch_route_t<16, false>(a, xmap, wmap, xmap, s);
    case 32: return launch_route_t<32, false>(a, xmap, wmap, xmap, s);
    default: return launch_route_t<64, false>(a, xmap, wmap, xmap, s);
  }
}

}  // namespace moe
