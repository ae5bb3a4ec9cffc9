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
// Three launches, no host synchronisation and no inter-CTA waiting:
//   count:    CTA b counts the experts of assignments [b*1024, (b+1)*1024)
//             with warp-aggregated shared-memory atomics -> tile_counts[b][E].
//   scatter:  CTA b sums the count vectors of tiles < b (its exclusive
//             prefix) and of all tiles (the histogram), derives capacity-
//             clipped offsets, ranks its assignments stably (warp match +
//             per-warp prefix), and writes perm / inv_perm.  CTA 0 also
//             writes counts and offsets.
//   permute:  x_perm[p] = bf16(x_t * gamma), t = perm[p] / k, one warp per row,
//             16-byte loads and stores.
#include "moe_internal.h"
#include "mx.cuh"

namespace moe {
namespace {

constexpr int kDispThreads = 256;
constexpr int kDispWarps = kDispThreads / 32;

__global__ void __launch_bounds__(kDispThreads) dispatch_count_kernel(const DispatchArgs a) {
  __shared__ int hist[kMaxExperts];
  const int tid = threadIdx.x;
  for (int e = tid; e < a.E; e += kDispThreads) hist[e] = 0;
  __syncthreads();
  const int n = a.T * a.k;
  const int base = blockIdx.x * kDispatchTile;
  const int lane = tid & 31;
  for (int i = 0; i < kDispatchTile; i += kDispThreads) {
    const int asg = base + i + tid;
    int e = asg < n ? a.idx[asg] : -1;
    if (e >= a.E || (asg < n && e < 0)) {
      atomicOr(a.err, MOE_DEVERR_EXPERT_ID);
      e = -1;
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    const int leader = __ffs(peers) - 1;
    if (e >= 0 && lane == leader) atomicAdd(&hist[e], __popc(peers));
  }
  __syncthreads();
  for (int e = tid; e < a.E; e += kDispThreads)
    a.tile_counts[static_cast<size_t>(blockIdx.x) * a.E + e] = hist[e];
}

__global__ void __launch_bounds__(kDispThreads) dispatch_scatter_kernel(const DispatchArgs a,
                                                                        int ntiles) {
  __shared__ int before[kMaxExperts];   // assignments to e in tiles < this one
  __shared__ int offs[kMaxExperts + 1];  // row-segment offsets (kept rows + padding)
  __shared__ int kept[kMaxExperts];      // kept rows per expert
  __shared__ int run[kMaxExperts];       // running count inside this tile
  __shared__ int wcnt[kDispWarps][kMaxExperts];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E;
  const int cap = a.capacity;

  if (tid < E) {
    int b = 0, tot = 0;
    for (int j = 0; j < ntiles; ++j) {
      const int c = a.tile_counts[static_cast<size_t>(j) * E + tid];
      if (j < static_cast<int>(blockIdx.x)) b += c;
      tot += c;
    }
    before[tid] = b;
    run[tid] = 0;
    const int align = a.row_align > 1 ? a.row_align : 1;
    kept[tid] = (cap < 0) ? tot : min(tot, cap);
    offs[tid + 1] = (kept[tid] + align - 1) / align * align;
    if (blockIdx.x == 0) a.counts[tid] = tot;
  }
  for (int i = tid; i < kDispWarps * kMaxExperts; i += kDispThreads) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  if (tid == 0) {
    offs[0] = 0;
    for (int e = 0; e < E; ++e) offs[e + 1] += offs[e];
    if (offs[E] > a.max_kept) atomicOr(a.err, MOE_DEVERR_TILE_TABLE);
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int e = tid; e <= E; e += kDispThreads) a.offsets[e] = offs[e];
    // padding rows of the training layout (fewer than row_align per expert)
    for (int e = 0; e < E; ++e)
      for (int i = offs[e] + kept[e] + tid; i < offs[e + 1] && i < a.max_kept; i += kDispThreads)
        a.perm[i] = -1;
  }

  const int n = a.T * a.k;
  const int base = blockIdx.x * kDispatchTile;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int i = 0; i < kDispatchTile; i += kDispThreads) {
    const int asg = base + i + tid;
    int e = asg < n ? a.idx[asg] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    const int leader = __ffs(peers) - 1;
    if (e >= 0 && lane == leader) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int rank = before[e] + run[e] + __popc(peers & lt_mask);
      for (int w = 0; w < warp; ++w) rank += wcnt[w][e];
      const bool kept = (cap < 0) || (rank < cap);
      const int pos = offs[e] + rank;
      if (kept && pos < a.max_kept) {
        a.perm[pos] = asg;
        a.inv_perm[asg] = pos;
      } else {
        a.inv_perm[asg] = -1;
      }
    } else if (asg < n) {
      a.inv_perm[asg] = -1;
    }
    __syncthreads();
    if (tid < E) {
      int s = 0;
      for (int w = 0; w < kDispWarps; ++w) s += wcnt[w][tid];
      run[tid] += s;
    }
    __syncthreads();
    if (e >= 0 && lane == leader) wcnt[warp][e] = 0;
    __syncthreads();
  }
}

// x_perm[p] = bf16(x[perm[p]/k] * gamma) for p < offsets[E]; zero rows where
// perm[p] = -1 (padding).
__global__ void __launch_bounds__(256) permute_rows_kernel(const DispatchArgs a) {
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

cudaError_t launch_dispatch(const DispatchArgs& a, int num_sms, cudaStream_t s) {
  const int n = a.T * a.k;
  if (n == 0) return cudaSuccess;
  const int ntiles = (n + kDispatchTile - 1) / kDispatchTile;
  dispatch_count_kernel<<<ntiles, kDispThreads, 0, s>>>(a);
  dispatch_scatter_kernel<<<ntiles, kDispThreads, 0, s>>>(a, ntiles);
  if ((a.x_perm != nullptr || a.x8 != nullptr) && a.max_kept > 0) {
    int grid = (a.max_kept + 7) / 8;
    grid = grid < num_sms * 8 ? grid : num_sms * 8;
    if (a.x8 != nullptr)
      permute_rows_mx_kernel<<<grid, 256, 0, s>>>(a);
    else
      permute_rows_kernel<<<grid, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace moe
