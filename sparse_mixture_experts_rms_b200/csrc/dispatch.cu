// dispatch.cu -- histogram, capacity, stable expert-centric permutation, and
// the permuted gamma-scaled activations.
//
// OmniMoE summary (gist.science), section 2.2 "Expert-Centric Scheduling":
// the routing decisions of a batch are flattened into a task list, grouped by
// expert and ordered by token id inside each group, so each expert's weights
// are read once for a contiguous block of rows.  MoE glossary (inferensys.com),
// "Expert Capacity": an expert keeps at most C = (T*k)/E * capacity_factor
// assignments; the rest are dropped (here: the first C in token order stay).
// CODA sparse-MoE thread: the statistic travels with the dispatched token to
// the first expert GEMM (the expert GEMM reads r through perm).
//
// One launch for the index work, no host synchronisation:
//   The assignments a = t*k + j are cut into tiles of 1024.  A CTA counts a
//   tile's experts with warp-aggregated shared-memory atomics and publishes
//   the tile's E-wide count vector (status "aggregate"), then looks back over
//   the tiles before it -- a warp reads 32 predecessors' statuses at a time --
//   summing aggregates until it meets a tile that has published its inclusive
//   prefix; it publishes its own inclusive prefix (status "inclusive").  This
//   is a single-pass scan with decoupled look-back: each tile waits only for
//   its predecessors' counts, never for their scans.  The last tile's
//   inclusive prefix is the histogram; every CTA waits for it, derives the
//   capacity-clipped segment offsets, and scatters its tiles: the rank of an
//   assignment inside its expert is the tile's exclusive prefix plus its rank
//   inside the tile (warp match + per-warp counts), which keeps token order.
//   The launch is cooperative (all CTAs resident), so the wait for the last
//   tile cannot starve it; every spin is bounded by the workspace's wait limit
//   and gives up into MOE_DEVERR_TIMEOUT.
//   permute (a second launch, when the permuted activations are wanted):
//   x_perm[p] = bf16(x_t * gamma), t = perm[p] / k, one warp per row.
#include "moe_internal.h"
#include "mx.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kDispThreads = 256;
constexpr int kDispWarps = kDispThreads / 32;
constexpr uint32_t kStAggregate = 1u, kStInclusive = 2u;

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

struct ScanView {
  uint32_t* status;  // [ntiles]
  int32_t* agg;      // [ntiles, E]
  int32_t* inc;      // [ntiles, E]
};

__device__ __forceinline__ ScanView scan_view(int32_t* scan, int ntiles, int E) {
  ScanView v;
  v.status = reinterpret_cast<uint32_t*>(scan);
  v.agg = scan + dispatch_status_ints(ntiles);
  v.inc = v.agg + static_cast<size_t>(ntiles) * E;
  return v;
}

// Warp 0 looks back from tile b: returns (in *stop) the nearest predecessor
// that has published its inclusive prefix (-1: none needed -- the sum starts
// at zero before tile 0), once every tile between it and b has published at
// least its aggregate.  False if the wait ran out (lane 0's clock decides, so
// the warp agrees).
__device__ bool look_back(const ScanView& v, int b, int lane, uint64_t wait_ns, volatile int* abort, int* stop) {
  int j0 = b - 1;  // the window is tiles j0, j0 - 1, ..., j0 - 31 (lane i: j0 - i)
  uint32_t polls = 0;
  uint64_t t0 = 0;
  while (true) {
    const int j = j0 - lane;
    const uint32_t st = j >= 0 ? ld_acquire_gpu(&v.status[j]) : kStInclusive;
    const unsigned inc_mask = __ballot_sync(0xFFFFFFFFu, st == kStInclusive);
    const unsigned none_mask = __ballot_sync(0xFFFFFFFFu, st == 0u);
    const unsigned nearer = inc_mask ? ((inc_mask & (0u - inc_mask)) - 1u) : 0xFFFFFFFFu;
    if ((none_mask & nearer) == 0u) {
      if (inc_mask) {  // tiles j0 .. (nearest inclusive) have all published
        *stop = j0 - (__ffs(inc_mask) - 1);
        return true;
      }
      j0 -= 32;  // the whole window holds aggregates: continue further back
      polls = 0;
      continue;
    }
    if (polls == 0) {
      t0 = global_timer_ns();
    } else if ((polls & 15u) == 0u) {
      const int give_up = lane == 0 ? ((*abort != 0) || (global_timer_ns() - t0 > wait_ns)) : 0;
      if (__shfl_sync(0xFFFFFFFFu, give_up, 0)) return false;
    }
    ++polls;
  }
}

// One cooperative launch over a persistent grid; CTA c handles tiles c, c + G, ...
__global__ void __launch_bounds__(kDispThreads) dispatch_kernel(const DispatchArgs a, int ntiles) {
  griddep_launch_dependents();  // the permute may launch; it waits for this grid to finish
  __shared__ int hist[kMaxExperts];      // this tile's counts
  __shared__ int excl[kMaxExperts];      // assignments to e in the tiles before this one
  __shared__ int offs[kMaxExperts + 1];  // row-segment offsets (kept rows + padding)
  __shared__ int kept[kMaxExperts];      // kept rows per expert
  __shared__ int run[kMaxExperts];       // running count inside this tile
  __shared__ int wcnt[kDispWarps][kMaxExperts];
  __shared__ int stop_s;
  __shared__ int abort_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E;
  const int cap = a.capacity;
  const int n = a.T * a.k;
  const uint64_t wait_ns = wait_limit_ns(a.wait_ctl);
  const ScanView v = scan_view(a.scan, ntiles, E);
  if (tid == 0) abort_s = 0;

  // ---- count, publish, look back, publish (tiles in increasing order per CTA)
  for (int b = blockIdx.x; b < ntiles; b += gridDim.x) {
    for (int e = tid; e < E; e += kDispThreads) hist[e] = 0;
    __syncthreads();
    const int base = b * kDispatchTile;
    for (int i = 0; i < kDispatchTile; i += kDispThreads) {
      const int asg = base + i + tid;
      int e = asg < n ? a.idx[asg] : -1;
      if (e >= E || (asg < n && e < 0)) {
        atomicOr(a.err, MOE_DEVERR_EXPERT_ID);
        e = -1;
      }
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      const int leader = __ffs(peers) - 1;
      if (e >= 0 && lane == leader) atomicAdd(&hist[e], __popc(peers));
    }
    __syncthreads();
    if (tid < E) v.agg[static_cast<size_t>(b) * E + tid] = hist[tid];
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release_gpu(&v.status[b], kStAggregate);
    if (warp == 0) {
      int stop = -1;
      const bool ok = b == 0 || look_back(v, b, lane, wait_ns, &abort_s, &stop);
      if (lane == 0) {
        stop_s = stop;
        if (!ok) {
          abort_s = 1;
          atomicOr(a.err, MOE_DEVERR_TIMEOUT);
        }
      }
    }
    __syncthreads();
    if (abort_s) break;
    if (tid < E) {
      const int stop = stop_s;
      int acc = stop >= 0 ? __ldcg(&v.inc[static_cast<size_t>(stop) * E + tid]) : 0;
      for (int j = stop + 1; j < b; ++j) acc += __ldcg(&v.agg[static_cast<size_t>(j) * E + tid]);
      v.inc[static_cast<size_t>(b) * E + tid] = acc + hist[tid];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release_gpu(&v.status[b], kStInclusive);
  }

  // ---- the histogram: the last tile's inclusive prefix
  if (tid == 0 && !abort_s) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t k = 0; ld_acquire_gpu(&v.status[ntiles - 1]) != kStInclusive; ++k) {
      if ((k & 15u) == 15u && global_timer_ns() - t0 > wait_ns) {
        abort_s = 1;
        atomicOr(a.err, MOE_DEVERR_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
  if (abort_s) return;  // outputs undefined; the error word says why
  if (tid < E) {
    const int tot = __ldcg(&v.inc[static_cast<size_t>(ntiles - 1) * E + tid]);
    const int align = a.row_align > 1 ? a.row_align : 1;
    kept[tid] = (cap < 0) ? tot : min(tot, cap);
    offs[tid + 1] = (kept[tid] + align - 1) / align * align;
    if (blockIdx.x == 0) a.counts[tid] = tot;
  }
  __syncthreads();
  if (tid == 0) {
    offs[0] = 0;
    for (int e = 0; e < E; ++e) offs[e + 1] += offs[e];
    if (offs[E] > a.max_kept) atomicOr(a.err, MOE_DEVERR_TILE_TABLE);
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e <= E; e += kDispThreads) a.offsets[e] = offs[e];
  // padding rows of the training layout (fewer than row_align per expert): expert e by CTA e % G
  for (int e = blockIdx.x; e < E; e += gridDim.x)
    for (int i = offs[e] + kept[e] + tid; i < offs[e + 1] && i < a.max_kept; i += kDispThreads) a.perm[i] = -1;

  // ---- scatter: stable ranks inside each expert, capacity, perm / inv_perm
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int b = blockIdx.x; b < ntiles; b += gridDim.x) {
    if (tid < E) {
      const size_t o = static_cast<size_t>(b) * E + tid;
      excl[tid] = __ldcg(&v.inc[o]) - __ldcg(&v.agg[o]);
      run[tid] = 0;
    }
    for (int i = tid; i < kDispWarps * kMaxExperts; i += kDispThreads) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int base = b * kDispatchTile;
    for (int i = 0; i < kDispatchTile; i += kDispThreads) {
      const int asg = base + i + tid;
      int e = asg < n ? a.idx[asg] : -1;
      if (e < 0 || e >= E) e = -1;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      const int leader = __ffs(peers) - 1;
      if (e >= 0 && lane == leader) wcnt[warp][e] = __popc(peers);
      __syncthreads();
      bool dropped = asg < n;
      if (e >= 0) {
        int rank = excl[e] + run[e] + __popc(peers & lt_mask);
        for (int w = 0; w < warp; ++w) rank += wcnt[w][e];
        const bool keep = (cap < 0) || (rank < cap);
        const int pos = offs[e] + rank;
        if (keep && pos < a.max_kept) {
          a.perm[pos] = asg;
          a.inv_perm[asg] = pos;
          dropped = false;
        }
      }
      if (dropped) a.inv_perm[asg] = -1;
      __syncthreads();
      if (tid < E) {
        int s2 = 0;
        for (int w = 0; w < kDispWarps; ++w) s2 += wcnt[w][tid];
        run[tid] += s2;
      }
      __syncthreads();
      if (e >= 0 && lane == leader) wcnt[warp][e] = 0;
      __syncthreads();
    }
  }
}

// x_perm[p] = bf16(x[perm[p]/k] * gamma) for p < offsets[E]; zero rows where
// perm[p] = -1 (padding).
__global__ void __launch_bounds__(256) permute_rows_kernel(const DispatchArgs a) {
  griddep_wait();                 // perm and offsets come from dispatch_kernel
  griddep_launch_dependents();    // the up GEMM may launch and set up meanwhile
  const int n_kept = min(a.offsets[a.E], a.max_kept);
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int chunks = a.d / 8;
  const uint4* g4 = reinterpret_cast<const uint4*>(a.gamma);
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < n_kept; p += warps) {
    const int asg = a.perm[p];
    if (asg < 0) {
      uint4* dst = reinterpret_cast<uint4*>(a.x_perm + static_cast<size_t>(p) * a.d);
      for (int c = lane; c < chunks; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const int t = asg / a.k;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.d);
    uint4* dst = reinterpret_cast<uint4*>(a.x_perm + static_cast<size_t>(p) * a.d);
    // four 16-byte loads per lane in flight before any store
    for (int c0 = lane; c0 < chunks; c0 += 128) {
      uint4 xv[4], gv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c < chunks) {
          xv[u] = __ldg(src + c);
          gv[u] = __ldg(g4 + c);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c >= chunks) break;
        const uint32_t xw[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
        const uint32_t gw[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(xw[i] << 16) * __uint_as_float(gw[i] << 16);
          const float hi = __uint_as_float(xw[i] & 0xFFFF0000u) * __uint_as_float(gw[i] & 0xFFFF0000u);
          const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
          o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// MX variant: x8[p] = E4M3 codes of x[perm[p]/k] * gamma in 32-column
// blocks (the product of two bf16 values is exact in fp32), one scale byte
// per block; zero codes and scales at padding rows.  One warp per row, one
// block per lane at a time.
__global__ void __launch_bounds__(256) permute_rows_mx_kernel(const DispatchArgs a) {
  const int n_rows = min(a.offsets[a.E], a.max_kept);
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nblk = a.d / 32;
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < n_rows; p += warps) {
    const int asg = a.perm[p];
    uint4* dst = reinterpret_cast<uint4*>(a.x8 + static_cast<size_t>(p) * a.d);
    for (int b = lane; b < nblk; b += 32) {
      uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      uint32_t sb = 0u;
      if (asg >= 0) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(asg / a.k) * a.d + b * 32);
        const uint4* g4 = reinterpret_cast<const uint4*>(a.gamma + b * 32);
        float v[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 xv = __ldg(src + j), gv = __ldg(g4 + j);
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[8 * j + 2 * i] = __uint_as_float(xw[i] << 16) * __uint_as_float(gw[i] << 16);
            v[8 * j + 2 * i + 1] = __uint_as_float(xw[i] & 0xFFFF0000u) * __uint_as_float(gw[i] & 0xFFFF0000u);
          }
        }
        sb = mx_quantize32(v, w);
      }
      dst[2 * b] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[2 * b + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      a.xsf[mx_sf_offset(p, b * 32, a.d)] = static_cast<uint8_t>(sb);
    }
  }
}

}  // namespace

// CTAs of dispatch_kernel that fit on the device at once (once per device).
int dispatch_resident_ctas(int num_sms) {
  static int per_sm[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return num_sms;
  if (per_sm[dev] == 0) {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, dispatch_kernel, kDispThreads, 0) != cudaSuccess || b < 1) {
      cudaGetLastError();
      b = 1;
    }
    per_sm[dev] = b;
  }
  return per_sm[dev] * num_sms;
}

cudaError_t launch_dispatch(const DispatchArgs& a, int num_sms, cudaStream_t s) {
  const int n = a.T * a.k;
  if (n == 0) return cudaSuccess;
  const int ntiles = (n + kDispatchTile - 1) / kDispatchTile;
  cudaError_t e = cudaMemsetAsync(a.scan, 0, static_cast<size_t>(ntiles) * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  const int resident = dispatch_resident_ctas(num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ntiles < resident ? ntiles : resident), 1, 1);
  cfg.blockDim = dim3(kDispThreads, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, dispatch_kernel, a, ntiles);
  if (e != cudaSuccess) return e;
  if ((a.x_perm != nullptr || a.x8 != nullptr) && a.max_kept > 0) {
    int grid = (a.max_kept + 7) / 8;
    grid = grid < num_sms * 8 ? grid : num_sms * 8;
    if (a.x8 != nullptr)
      permute_rows_mx_kernel<<<grid, 256, 0, s>>>(a);
    else
      return launch_pdl(permute_rows_kernel, dim3(grid), dim3(256), 0, s, a);
  }
  return cudaGetLastError();
}

}  // namespace moe
