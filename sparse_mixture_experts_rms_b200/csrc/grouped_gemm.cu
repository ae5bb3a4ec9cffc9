// grouped_gemm.cu -- the expert FFN as two persistent grouped GEMMs on the
// 5th-generation tensor cores (tcgen05.mma, fp32 accumulators in TMEM,
// operands staged by TMA into 128-byte-swizzled shared memory).
//
// OmniMoE summary (gist.science), section 2.2 "Expert-Centric Scheduling":
// with the rows grouped by expert, each expert's weight block is loaded once
// and reused over a batch of its tokens -- a grouped GEMM.  nanoMOE
// variable-size-experts notes (hbfreed.com): experts have different widths
// f_e (multiples of 128) inside concatenated W1 [d, F] / W2 [F, d], addressed
// through cumulative offsets; the work decomposition uses running sums of
// per-expert tile counts, never index * size ("Critical Bug Fix").
// CODA sparse-MoE thread (digg.com): the RMS statistic r of each token is
// applied in the epilogue of the first expert GEMM.
//
//   up   (GEMM 1): for the kept rows p of expert e (t = perm[p] / k),
//        H[p, n] = bf16( silu(r_t * acc1[p, n]) * (r_t * acc3[p, n]) ),
//        acc1 = x_perm[p] . W1[:, o_e + n], acc3 = x_perm[p] . W3[:, o_e + n].
//        One 128 x 256 x 16 MMA covers 128 columns of W1 and the same 128
//        columns of W3, so both SwiGLU inputs of a tile sit in one accumulator.
//   down (GEMM 2): y[p, n] = bf16( gate[perm[p]] * (H[p, :f_e] . W2[o_e + :, n]) ).
//
// Tiles: BM = 128 rows of one expert x BN columns, K in blocks of 64.  The
// tile list is built on the device from the kept-row offsets (no host sync):
// expert e contributes ceil(n_e/128) * (N_e/BN) tiles, enumerated M-fastest
// so that CTAs running together share a weight column block in L2.
// Persistent CTAs (one per SM) stride through the list.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = MMA issuer (and
// TMEM owner), warps 2..5 = epilogue (TMEM -> registers -> global).
// Smem ring of 4 stages (A 16 KB + B 32 KB); two TMEM accumulators of 256
// fp32 columns so the epilogue of tile i overlaps the mainloop of tile i+1.
// Every wait is bounded (4 s) and sets a device error bit instead of hanging.
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;          // 16 KB
constexpr int kBBytes = BK * 256 * 2;         // 32 KB (BN up to 256)
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;                 // columns per accumulator buffer
constexpr int kAtomBytes = BK * 64 * 2;       // one 64(n) x 64(k) B box: 8 KB

struct __align__(8) GemmShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int total_tiles;
  int tile_start[kMaxExperts + 1];
  int m_tiles[kMaxExperts];
  int seg[kMaxExperts + 1];
};

constexpr size_t kSmemBytes = 1024 /* alignment slack */ + kStages * kStageBytes + sizeof(GemmShared);

struct TileCoord {
  int e, nt, mt;
};

__device__ __forceinline__ TileCoord decode_tile(const GemmShared& sh, int E, int tile) {
  int e = 0;
  while (e + 1 < E && tile >= sh.tile_start[e + 1]) ++e;
  const int local = tile - sh.tile_start[e];
  const int mt_count = sh.m_tiles[e];
  return TileCoord{e, local / mt_count, local % mt_count};
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                        const __grid_constant__ CUtensorMap mapB0,
                        const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmShared& sh = *reinterpret_cast<GemmShared*>(smem + kStages * kStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;

  // ---- prologue: barriers, TMEM, tile table
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.tfull[b], 1);
      mbar_init(&sh.tempty[b], 4);
    }
    mbar_init(&sh.drain, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapA);
    tma_prefetch_map(&mapB0);
    tma_prefetch_map(&mapB1);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid < E + 1) sh.seg[tid] = a.offsets[tid];
  __syncthreads();
  if (tid < E) {
    const int rows = sh.seg[tid + 1] - sh.seg[tid];
    const int ncols = a.up ? (a.ffn.off[tid + 1] - a.ffn.off[tid]) : a.d;
    const int nt = a.up ? ncols / kBlockN : ncols / a.bn;
    const int mt = (rows + BM - 1) / BM;
    sh.m_tiles[tid] = mt > 0 ? mt : 1;
    sh.tile_start[tid + 1] = mt * nt;  // count for now
  }
  __syncthreads();
  if (tid == 0) {
    sh.tile_start[0] = 0;
    for (int e = 0; e < E; ++e) sh.tile_start[e + 1] += sh.tile_start[e];
    sh.total_tiles = sh.tile_start[E];
    if (sh.seg[E] > a.rows) {  // more kept rows than the buffers hold: do nothing
      atomicOr(a.err, MOE_DEVERR_TILE_TABLE);
      sh.total_tiles = 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  const int total = sh.total_tiles;
  volatile int* abort_flag = &sh.abort_flag;

  if (warp == 0) {
    // ================= TMA producer (one lane)
    if (lane == 0) {
      uint32_t it = 0;
      const uint32_t tx = kABytes + a.bn * BK * 2;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int row0 = sh.seg[c.e] + c.mt * BM;
        const int o_e = a.ffn.off[c.e];
        const int kblocks = a.up ? a.d / BK : (a.ffn.off[c.e + 1] - o_e) / BK;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&sh.empty[s], ph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + s * kStageBytes;
          uint8_t* sB = sA + kABytes;
          mbar_arrive_expect_tx(&sh.full[s], tx);
          tma_load_2d(sA, &mapA, &sh.full[s], kb * BK, row0);
          if (a.up) {
            const int n0 = o_e + c.nt * kBlockN;
            tma_load_2d(sB + 0 * kAtomBytes, &mapB0, &sh.full[s], n0, kb * BK);
            tma_load_2d(sB + 1 * kAtomBytes, &mapB0, &sh.full[s], n0 + 64, kb * BK);
            tma_load_2d(sB + 2 * kAtomBytes, &mapB1, &sh.full[s], n0, kb * BK);
            tma_load_2d(sB + 3 * kAtomBytes, &mapB1, &sh.full[s], n0 + 64, kb * BK);
          } else {
            const int n0 = c.nt * a.bn;
            for (int j = 0; j < a.bn / 64; ++j)
              tma_load_2d(sB + j * kAtomBytes, &mapB0, &sh.full[s], n0 + j * 64, o_e + kb * BK);
          }
        }
      }
      // Drain: wait until every load issued into the ring has landed, so no
      // copy is in flight when the CTA exits (normally already true).
      const uint32_t n_issued = it;
      for (uint32_t j = (n_issued > kStages ? n_issued - kStages : 0); j < n_issued; ++j) {
        const int s = j % kStages;
        const uint32_t ph = (j / kStages) & 1u;
        volatile int no_abort = 0;
        mbar_wait(&sh.full[s], ph, &no_abort, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (one lane)
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(BM, a.bn, 1);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++tcount) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int o_e = a.ffn.off[c.e];
        const int kblocks = a.up ? a.d / BK : (a.ffn.off[c.e + 1] - o_e) / BK;
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
        if (!mbar_wait(&sh.tempty[buf], aph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kAccCols;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&sh.full[s], ph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aA = smem_addr(smem + s * kStageBytes);
          const uint32_t aB = aA + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(aA + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(aB + kk * 2048, kAtomBytes, 1024);
            umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&sh.empty[s]);  // frees the stage once these MMAs finish
        }
        if (!ok) break;
        umma_commit(&sh.tfull[buf]);  // accumulator ready for the epilogue
      }
      umma_commit(&sh.drain);
      volatile int no_abort = 0;
      mbar_wait(&sh.drain, 0, &no_abort, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
    }
  } else {
    // ================= epilogue (warps 2..5, one TMEM lane quarter each)
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
      const TileCoord c = decode_tile(sh, E, tile);
      const uint32_t buf = tcount & 1u;
      const uint32_t aph = (tcount >> 1) & 1u;
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait(&sh.tfull[buf], aph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const int p = sh.seg[c.e] + c.mt * BM + row_in_tile;
      const bool valid = p < sh.seg[c.e + 1];
      float scale = 0.f;
      if (valid) {
        const int asg = a.perm[p];
        scale = a.up ? a.scale[asg / a.k] : a.scale[asg];
      }
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kAccCols;
      if (a.up) {
        __nv_bfloat16* dst = a.out + static_cast<size_t>(valid ? p : 0) * a.ld_out + c.nt * kBlockN;
#pragma unroll 1
        for (int cc = 0; cc < kBlockN; cc += 32) {
          uint32_t u[32], v[32];
          tmem_ld_32x32b_x32(taddr + cc, u);
          tmem_ld_32x32b_x32(taddr + kBlockN + cc, v);
          tmem_ld_wait();
          if (valid) {
            uint32_t o[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float h0 = silu(scale * __uint_as_float(u[2 * j])) * (scale * __uint_as_float(v[2 * j]));
              const float h1 = silu(scale * __uint_as_float(u[2 * j + 1])) * (scale * __uint_as_float(v[2 * j + 1]));
              o[j] = pack_bf16(h0, h1);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
            for (int j = 0; j < 4; ++j) d4[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        }
      } else {
        __nv_bfloat16* dst = a.out + static_cast<size_t>(valid ? p : 0) * a.ld_out + c.nt * a.bn;
#pragma unroll 1
        for (int cc = 0; cc < a.bn; cc += 32) {
          uint32_t u[32];
          tmem_ld_32x32b_x32(taddr + cc, u);
          tmem_ld_wait();
          if (valid) {
            uint32_t o[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              o[j] = pack_bf16(scale * __uint_as_float(u[2 * j]), scale * __uint_as_float(u[2 * j + 1]));
            uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
            for (int j = 0; j < 4; ++j) d4[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tempty[buf]);
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace

size_t grouped_gemm_smem_bytes() { return kSmemBytes; }

cudaError_t prepare_grouped_gemm() {
  return cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

cudaError_t launch_grouped_gemm(const GemmArgs& a, const CUtensorMap& mapA, const CUtensorMap& mapB0,
                                const CUtensorMap& mapB1, int grid, cudaStream_t s) {
  grouped_gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(mapA, mapB0, mapB1, a);
  return cudaGetLastError();
}

}  // namespace moe
