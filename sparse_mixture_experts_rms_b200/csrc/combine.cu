// combine.cu -- gate-weighted combine back to token order.
//
// MoE glossary (inferensys.com), "Top-k Gating": the outputs of a token's k
// experts are combined by a weighted sum of their scores; "Expert Capacity":
// an assignment dropped by the capacity limit contributes nothing.  The gate
// weighting already happened in the second expert GEMM's epilogue, so here
//     out_t = bf16( sum_{j : inv_perm[t*k+j] >= 0} y[inv_perm[t*k+j]] ),
// accumulated in fp32 in slot order j = 0..k-1 (no atomics: one warp owns a
// token row).  A token whose slots were all dropped gets a zero row.
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const CombineArgs a) {
  griddep_wait();  // y and inv_perm come from the kernels before
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int chunks = a.d / 8;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < a.T; t += warps) {
    uint4* dst = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(t) * a.d);
    for (int c0 = 0; c0 < chunks; c0 += 32) {
      const int c = c0 + lane;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int jb = 0; jb < a.k; jb += 32) {
        const int j = jb + lane;
        const int mine = j < a.k ? a.inv_perm[static_cast<size_t>(t) * a.k + j] : -1;
        const int nj = min(32, a.k - jb);
        for (int jj = 0; jj < nj; ++jj) {
          const int pos = __shfl_sync(0xFFFFFFFFu, mine, jj);
          if (pos >= 0 && c < chunks) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.y + static_cast<size_t>(pos) * a.d) + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[2 * i] += __uint_as_float(w[i] << 16);
              acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
            }
          }
        }
      }
      if (c < chunks) {
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
          o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

}  // namespace

__global__ void set_words_kernel(uint32_t* dst, uint32_t w0, uint32_t w1) {
  dst[0] = w0;
  dst[1] = w1;
}

cudaError_t launch_set_words(uint32_t* dst, uint32_t w0, uint32_t w1, cudaStream_t s) {
  set_words_kernel<<<1, 1, 0, s>>>(dst, w0, w1);
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  int grid = (a.T + 7) / 8;
  grid = grid < num_sms * 8 ? grid : num_sms * 8;
  return launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, s, a);
}

}  // namespace moe
