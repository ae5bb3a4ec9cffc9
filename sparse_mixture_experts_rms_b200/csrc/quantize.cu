// quantize.cu -- MXFP8 copies of the expert weights for the MX expert GEMMs
// (done once per set of weights, outside the layer).
//
// Each weight is a K x N row-major bf16 matrix whose GEMM reduces over K
// (W1, W3: K = d, N = F; W2: K = F, N = d).  The copy is K-major: row n holds
// the E4M3 codes of column n, blocked by 32 along K (see mx.cuh), so the GEMM
// loads it like its activations.  Expert boundaries (multiples of 128 in F)
// never cut a block.
#include "moe_internal.h"
#include "mx.cuh"

namespace moe {
namespace {

size_t al(size_t v) { return (v + 1023) / 1024 * 1024; }

// One thread per (column n, 32-block of K); consecutive threads take
// consecutive n, so the reads of a K row are coalesced.  Scales go to the
// standard blocks of the [N, K] copy.
//
// The scale byte also goes, four times, into the pair copy `sfp`: column block
// nb = n / 128 and K block kb = k / 128 select region (nb >> pair_shift) *
// (K / 128) + kb, and half `half` (W1 / W3: fixed 0 / 1; W2: nb & 1).
__global__ void __launch_bounds__(128) quantize_kn_mx_kernel(const __nv_bfloat16* W, int K, int N, uint8_t* q,
                                                             uint8_t* sf, uint8_t* sfp, int half, int pair_shift) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int k0 = blockIdx.y * 32;
  if (n >= N) return;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(W[static_cast<size_t>(k0 + i) * N + n]);
  uint32_t w[8];
  const uint32_t sb = mx_quantize32(v, w);
  uint4* dst = reinterpret_cast<uint4*>(q + static_cast<size_t>(n) * K + k0);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  sf[mx_sf_offset(n, k0, K)] = static_cast<uint8_t>(sb);
  const int nb = n >> 7, kb = k0 >> 7;
  const int h = half >= 0 ? half : (nb & 1);
  uint8_t* region = sfp + (static_cast<size_t>(nb >> pair_shift) * (K >> 7) + kb) * kMxPairRegion + h * 2048;
  const int inner = 16 * (n & 31) + 4 * ((n & 127) >> 5) + ((k0 & 127) >> 5);
#pragma unroll
  for (int rep = 0; rep < 4; ++rep) region[rep * 512 + inner] = static_cast<uint8_t>(sb);
}

}  // namespace

size_t mx_weights_bytes(int d, int F) {
  const size_t dd = static_cast<size_t>(d), ff = static_cast<size_t>(F);
  const size_t sf = al((ff / 128) * (dd / 128) * 512);  // each of sf1, sf3, sf2
  const size_t p13 = al((ff / 128) * (dd / 128) * kMxPairRegion);
  const size_t p2 = al(((dd / 128 + 1) / 2) * (ff / 128) * kMxPairRegion);
  return 3 * al(dd * ff) + 3 * sf + p13 + p2;
}

MxWeights mx_weights_at(void* base, int d, int F) {
  const size_t dd = static_cast<size_t>(d), ff = static_cast<size_t>(F);
  const size_t sf = al((ff / 128) * (dd / 128) * 512);
  uint8_t* p = static_cast<uint8_t*>(base);
  MxWeights m;
  m.w1 = p;
  m.w3 = m.w1 + al(dd * ff);
  m.w2 = m.w3 + al(dd * ff);
  m.sf1 = m.w2 + al(dd * ff);
  m.sf3 = m.sf1 + sf;
  m.sf2 = m.sf3 + sf;
  m.sfp13 = m.sf2 + sf;
  m.sfp2 = m.sfp13 + al((ff / 128) * (dd / 128) * kMxPairRegion);
  return m;
}

cudaError_t launch_quantize_weights_mx(const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                                       const __nv_bfloat16* W2, MxWeights q, int d, int F, cudaStream_t s) {
  const dim3 g13((F + 127) / 128, d / 32), g2((d + 127) / 128, F / 32);
  quantize_kn_mx_kernel<<<g13, 128, 0, s>>>(W1, d, F, q.w1, q.sf1, q.sfp13, 0, 0);
  quantize_kn_mx_kernel<<<g13, 128, 0, s>>>(W3, d, F, q.w3, q.sf3, q.sfp13, 1, 0);
  quantize_kn_mx_kernel<<<g2, 128, 0, s>>>(W2, F, d, q.w2, q.sf2, q.sfp2, -1, 1);
  return cudaGetLastError();
}

}  // namespace moe
