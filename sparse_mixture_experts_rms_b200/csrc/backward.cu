// backward.cu -- the bandwidth-bound stages of the layer backward (the
// contractions run in grouped_gemm.cu).
//
// CODA sparse-MoE thread (digg.com): the RMSNorm backward is fused into the
// backward of the linears that consume the normalised token -- the expert's
// first linear and the router -- and it needs each token's statistic r.
// With l_t = r_t (x_t*gamma) Wr + b and u = r_t (x_t*gamma) W1_e, the
// statistic's gradient is a per-row dot product of each linear's output
// gradient with its pre-statistic output; the first expert GEMM's backward
// epilogue forms the expert part (dr partials), bwd_route the router part.
//
//   gather  dY[p] = bf16(gate_a * dout_t), dgate_a = <dout_t, y_a> for the kept
//           row p = position of assignment a (y ungated, saved by the forward);
//           zero rows at padding.
//   route   per token: softmax of the saved logits, gate -> q -> p -> logits
//           backward (with the optional renormalisation over the k chosen),
//           dr_t = sum of the expert partials + <dl_t, z_t>, z_t = (l_t - b)/r_t;
//           writes r_t * dl_t and per-CTA partial sums of dl (the bias gradient).
//   norm    per (column slice, token chunk):
//           dxg_t = sum_j dX[p_j] + (r_t dl_t) Wr^T,
//           dx_t  = gamma * dxg_t - (r_t^3 / d) dr_t x_t,
//           partial sums of dgamma = dxg_t * x_t and dWr = (x_t*gamma)^T (r_t dl_t).
//   reduce  the partial sums, in a fixed order (deterministic).
#include <cfloat>

#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// One warp per padded row; 16-byte loads and stores.
__global__ void __launch_bounds__(256) bwd_gather_kernel(const BwdArgs a) {
  const int n_rows = min(a.offsets[a.E], a.rows);
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int chunks = a.d / 8;
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < n_rows; p += warps) {
    uint4* dst = reinterpret_cast<uint4*>(a.dY + static_cast<size_t>(p) * a.d);
    const int asg = a.perm[p];
    if (asg < 0) {
      for (int c = lane; c < chunks; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const int t = asg / a.k;
    const float gt = a.gate[asg];
    const uint4* g4 = reinterpret_cast<const uint4*>(a.dout + static_cast<size_t>(t) * a.d);
    const uint4* y4 = reinterpret_cast<const uint4*>(a.yu + static_cast<size_t>(p) * a.d);
    float acc = 0.f;
    for (int c = lane; c < chunks; c += 32) {
      const uint4 gv = __ldg(g4 + c), yv = y4[c];
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
      const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float g0 = __uint_as_float(gw[i] << 16), g1 = __uint_as_float(gw[i] & 0xFFFF0000u);
        acc += g0 * __uint_as_float(yw[i] << 16) + g1 * __uint_as_float(yw[i] & 0xFFFF0000u);
        const __nv_bfloat162 h = __floats2bfloat162_rn(gt * g0, gt * g1);
        o[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    acc = warp_sum(acc);
    if (lane == 0) a.dgate[asg] = acc;
  }
}

// One warp per token, lanes over experts (e = lane, lane + 32).
__global__ void __launch_bounds__(256) bwd_route_kernel(const BwdArgs a) {
  __shared__ int s_idx[8][kMaxExperts];
  __shared__ float s_dq[8][kMaxExperts];
  __shared__ float s_red[8][kMaxExperts];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int E = a.E, k = a.k;
  const int e0 = lane, e1 = lane + 32;
  float db0 = 0.f, db1 = 0.f;
  const int t_begin = blockIdx.x * kBwdRouteTokens;
  const int t_end = min(a.T, t_begin + kBwdRouteTokens);
  for (int t = t_begin + warp; t < t_end; t += 8) {
    const float* lt = a.logits + static_cast<size_t>(t) * E;
    const float l0 = e0 < E ? lt[e0] : -FLT_MAX, l1 = e1 < E ? lt[e1] : -FLT_MAX;
    const float m = warp_max(fmaxf(l0, l1));
    const float x0 = e0 < E ? expf(l0 - m) : 0.f, x1 = e1 < E ? expf(l1 - m) : 0.f;
    const float inv_s = 1.0f / warp_sum(x0 + x1);
    const float p0 = x0 * inv_s, p1 = x1 * inv_s;
    // the k chosen: id, gradient of the gate (0 if dropped), q = p[id]
    const float r = a.r[t];
    float qsum = 0.f, gq = 0.f, dr_exp = 0.f;
    for (int j = lane; j < k; j += 32) {
      const int aidx = t * k + j;
      const int e = a.idx[aidx];
      const int pos = a.inv_perm[aidx];
      const float dg = pos >= 0 ? a.dgate[aidx] : 0.f;
      s_idx[warp][j] = e;
      s_dq[warp][j] = dg;
      if (pos >= 0) {
        const int nt = (a.ffn.off[e + 1] - a.ffn.off[e]) / a.bn_h;
        const float* dp = a.drp + static_cast<size_t>(pos) * a.ld_drp;
        for (int n = 0; n < nt; ++n) dr_exp += dp[n];
      }
    }
    __syncwarp();
    dr_exp = warp_sum(dr_exp);
    if (a.renormalize) {
      // gate_j = q_j / S: dq_j = (dgate_j - sum_i dgate_i gate_i) / S
      for (int jj = 0; jj < 2; ++jj) {  // k <= 64: slots lane and lane + 32
        const int j = lane + 32 * jj;
        const int e = j < k ? s_idx[warp][j] : 0;
        const float pe_lo = __shfl_sync(0xFFFFFFFFu, p0, e & 31);  // every lane shuffles
        const float pe_hi = __shfl_sync(0xFFFFFFFFu, p1, e & 31);
        const float q = j < k ? (e < 32 ? pe_lo : pe_hi) : 0.f;
        qsum += q;
        gq += (j < k ? s_dq[warp][j] : 0.f) * q;
      }
      const float S = warp_sum(qsum);
      const float G = warp_sum(gq) / S;
      __syncwarp();
      for (int j = lane; j < k; j += 32) s_dq[warp][j] = (s_dq[warp][j] - G) / S;
      __syncwarp();
    }
    float dp0 = 0.f, dp1 = 0.f;
    for (int j = 0; j < k; ++j) {
      const int e = s_idx[warp][j];
      if (e == e0) dp0 += s_dq[warp][j];
      if (e == e1) dp1 += s_dq[warp][j];
    }
    const float pd = warp_sum(dp0 * p0 + dp1 * p1);
    const float dl0 = p0 * (dp0 - pd), dl1 = p1 * (dp1 - pd);
    const float b0 = (a.bias != nullptr && e0 < E) ? a.bias[e0] : 0.f;
    const float b1 = (a.bias != nullptr && e1 < E) ? a.bias[e1] : 0.f;
    const float z0 = e0 < E ? (l0 - b0) / r : 0.f, z1 = e1 < E ? (l1 - b1) / r : 0.f;
    const float dr_router = warp_sum(dl0 * z0 + dl1 * z1);
    float* rdl = a.rdl + static_cast<size_t>(t) * E;
    if (e0 < E) rdl[e0] = r * dl0;
    if (e1 < E) rdl[e1] = r * dl1;
    if (lane == 0) a.dr[t] = dr_exp + dr_router;
    db0 += dl0;
    db1 += dl1;
    __syncwarp();
  }
  s_red[warp][e0] = db0;
  s_red[warp][e1] = db1;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += s_red[w][e];
    a.dbias_part[static_cast<size_t>(blockIdx.x) * E + e] = s;
  }
}

// One thread per column c of a 128-column slice, tokens of one chunk in
// batches of 32 staged in shared memory.  Wr[c, :] sits in registers.
template <int EMAX>
__global__ void __launch_bounds__(kBwdNormCols) bwd_norm_kernel(const BwdArgs a) {
  constexpr int kBatch = 32;
  __shared__ float s_rdl[kBatch][EMAX];
  __shared__ int s_pos[kBatch][EMAX];
  __shared__ float s_coef[kBatch];
  const int tid = threadIdx.x;
  const int E = a.E, k = a.k, d = a.d;
  const int c = blockIdx.x * kBwdNormCols + tid;
  const int t0 = blockIdx.y * a.chunk_tokens;
  const int t1 = min(a.T, t0 + a.chunk_tokens);
  float wr[EMAX], acc_w[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    wr[e] = e < E ? __bfloat162float(a.Wr[static_cast<size_t>(c) * E + e]) : 0.f;
    acc_w[e] = 0.f;
  }
  const float gam = __bfloat162float(a.gamma[c]);
  float acc_g = 0.f;
  for (int tb = t0; tb < t1; tb += kBatch) {
    const int nt = min(kBatch, t1 - tb);
    __syncthreads();
    for (int i = tid; i < nt * E; i += kBwdNormCols) s_rdl[i / E][i % E] = a.rdl[static_cast<size_t>(tb) * E + i];
    for (int i = tid; i < nt * k; i += kBwdNormCols) s_pos[i / k][i % k] = a.inv_perm[static_cast<size_t>(tb) * k + i];
    for (int i = tid; i < nt; i += kBwdNormCols) {
      const float r = a.r[tb + i];
      s_coef[i] = r * r * r / static_cast<float>(d) * a.dr[tb + i];
    }
    __syncthreads();
    // 8 tokens at a time: per slot, the 8 tokens' loads are all issued before any
    // is used, so they are in flight together
    for (int i0 = 0; i0 < nt; i0 += 8) {
      float xv[8], dxg[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u;
        xv[u] = i < nt ? __bfloat162float(__ldg(a.x + static_cast<size_t>(tb + i) * d + c)) : 0.f;
        dxg[u] = 0.f;
      }
      for (int j = 0; j < k; ++j) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u;
          const int p = i < nt ? s_pos[i][j] : -1;
          v[u] = p >= 0 ? __ldg(a.dXp + static_cast<size_t>(p) * d + c) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) dxg[u] += v[u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u;
        if (i >= nt) break;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) dxg[u] += s_rdl[i][e < E ? e : 0] * (e < E ? wr[e] : 0.f);
        a.dx[static_cast<size_t>(tb + i) * d + c] = gam * dxg[u] - s_coef[i] * xv[u];
        acc_g += dxg[u] * xv[u];
        const float xg = xv[u] * gam;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) acc_w[e] += xg * (e < E ? s_rdl[i][e] : 0.f);
      }
    }
  }
  a.dgamma_part[static_cast<size_t>(blockIdx.y) * d + c] = acc_g;
  float* wp = a.dWr_part + (static_cast<size_t>(blockIdx.y) * d + c) * E;
#pragma unroll
  for (int e = 0; e < EMAX; ++e)
    if (e < E) wp[e] = acc_w[e];
}

// dWr [d*E], dgamma [d], dbias [E] from their partial sums, in chunk order.
__global__ void __launch_bounds__(256) bwd_reduce_kernel(const BwdArgs a) {
  const int nw = a.d * a.E;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < nw) {
    float s = 0.f;
    for (int ch = 0; ch < a.chunks; ++ch) s += a.dWr_part[static_cast<size_t>(ch) * nw + i];
    a.dWr[i] = s;
  } else if (i < nw + a.d) {
    const int c = i - nw;
    float s = 0.f;
    for (int ch = 0; ch < a.chunks; ++ch) s += a.dgamma_part[static_cast<size_t>(ch) * a.d + c];
    a.dgamma[c] = s;
  } else if (i < nw + a.d + a.E) {
    const int e = i - nw - a.d;
    float s = 0.f;
    for (int b = 0; b < a.route_blocks; ++b) s += a.dbias_part[static_cast<size_t>(b) * a.E + e];
    a.dbias[e] = s;
  }
}

}  // namespace

cudaError_t launch_bwd_gather(const BwdArgs& a, int num_sms, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  int grid = (a.rows + 7) / 8;
  grid = grid < num_sms * 8 ? grid : num_sms * 8;
  bwd_gather_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_route(const BwdArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  bwd_route_kernel<<<a.route_blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_norm(const BwdArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(a.d / kBwdNormCols), static_cast<unsigned>(a.chunks));
  if (a.E <= 8)
    bwd_norm_kernel<8><<<grid, kBwdNormCols, 0, s>>>(a);
  else if (a.E <= 16)
    bwd_norm_kernel<16><<<grid, kBwdNormCols, 0, s>>>(a);
  else if (a.E <= 32)
    bwd_norm_kernel<32><<<grid, kBwdNormCols, 0, s>>>(a);
  else
    bwd_norm_kernel<64><<<grid, kBwdNormCols, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_reduce(const BwdArgs& a, cudaStream_t s) {
  const int n = a.d * a.E + a.d + a.E;
  bwd_reduce_kernel<<<(n + 255) / 256, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
