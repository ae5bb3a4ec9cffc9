// grouped_gemm.cu -- the expert FFN as two persistent grouped GEMMs on the
// 5th-generation tensor cores: 2-CTA (cta_group::2) tcgen05.mma with fp32
// accumulators in TMEM, operands staged by TMA into 128-byte-swizzled shared
// memory.
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
//        One 256 x 256 x 16 pair MMA covers 128 columns of W1 and the same 128
//        columns of W3, so both SwiGLU inputs of a row sit in one accumulator.
//   down (GEMM 2): y[p, n] = bf16( gate[perm[p]] * (H[p, :f_e] . W2[o_e + :, n]) ).
//
// CTA pairs (clusters of 2): a pair owns a 256-row x BN tile.  Each CTA loads
// its own 128 rows of A and its half of the BN columns of B (so B crosses L2
// once per pair, not once per CTA); the leader CTA issues the pair MMA, which
// reads both CTAs' shared memory and writes each CTA's 128 rows of D into that
// CTA's TMEM.  Both CTAs' loads complete on the leader's "full" barrier; the
// MMA commit arrives on both CTAs' "empty" and "accumulator full" barriers;
// both CTAs' epilogues arrive on the leader's "accumulator empty" barrier.
//
// Tiles: expert e contributes ceil(n_e/256) * (N_e/BN) pair tiles, listed on
// the device from the kept-row offsets (no host sync) in raster groups of
// M tiles whose A rows fit a 48 MB L2 budget (M fastest inside a group), so
// pairs running together share A rows and weight column blocks in L2.
// Persistent pairs stride through the list.
//
// Warp roles (192 threads per CTA): warp 0 = TMA producer, warp 1 = MMA issuer
// (leader only) and TMEM owner, warps 2..5 = epilogue (TMEM -> registers ->
// global).  Ring of 6 stages x (A 16 KB + B 16 KB) per CTA; two TMEM
// accumulators of 256 fp32 columns, so the epilogue of tile i overlaps the
// mainloop of tile i+1.  Every wait is bounded (4 s) and sets a device error
// bit instead of hanging.
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 256;                       // rows per pair tile (128 per CTA)
constexpr int BM_CTA = 128;
constexpr int BK = 64;
constexpr int kStages = 6;
constexpr int kABytes = BM_CTA * BK * 2;      // 16 KB
constexpr int kBBytes = BK * 128 * 2;         // 16 KB: this CTA's half of BN <= 256
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;                 // columns per accumulator buffer
constexpr int kAtomBytes = BK * 64 * 2;       // one 64(n) x 64(k) B box: 8 KB
constexpr int kEpiWarps = 4;
constexpr long long kL2GroupBudget = 48ll << 20;  // A bytes of one raster group

struct __align__(8) GemmShared {
  uint64_t full[kStages];    // leader: both CTAs' loads of a stage landed
  uint64_t empty[kStages];   // each CTA: the MMAs reading its stage finished
  uint64_t tfull[2];         // each CTA: accumulator buffer ready
  uint64_t tempty[2];        // leader: both CTAs' epilogues drained the buffer
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int total_tiles;
  int tile_start[kMaxExperts + 1];
  int m_tiles[kMaxExperts];
  int n_tiles[kMaxExperts];
  int group_m[kMaxExperts];  // m tiles per raster group (see decode_tile)
  int seg[kMaxExperts + 1];
};

constexpr size_t kSmemBytes = 1024 /* alignment slack */ + kStages * kStageBytes + sizeof(GemmShared);

struct TileCoord {
  int e, nt, mt;
};

// Tiles of expert e are rastered in groups of group_m[e] M tiles: inside a
// group, M is fastest and N next, so the pairs running together share the
// group's A rows (kept in L2) and a few B column blocks.  group_m is chosen so
// that a group's A rows fit an L2 budget; when the whole expert fits, the
// order is plain M-fastest.
__device__ __forceinline__ TileCoord decode_tile(const GemmShared& sh, int E, int tile) {
  int e = 0;
  while (e + 1 < E && tile >= sh.tile_start[e + 1]) ++e;
  const int local = tile - sh.tile_start[e];
  const int mt_count = sh.m_tiles[e], nt_count = sh.n_tiles[e], gm = sh.group_m[e];
  const int g = local / (gm * nt_count);
  const int rem = local - g * gm * nt_count;
  const int gm_g = min(gm, mt_count - g * gm);  // the last group may be short
  return TileCoord{e, rem / gm_g, g * gm + rem % gm_g};
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                        const __grid_constant__ CUtensorMap mapB0,
                        const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmShared& sh = *reinterpret_cast<GemmShared*>(smem + kStages * kStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;
  const uint32_t rank = cluster_ctarank();      // 0 = leader, 1 = peer
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  // ---- prologue: barriers, TMEM, tile table
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.tfull[b], 1);
      mbar_init(&sh.tempty[b], 2 * kEpiWarps);
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
    tmem_alloc_pair(&sh.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (tid < E + 1) sh.seg[tid] = a.offsets[tid];
  __syncthreads();
  if (tid < E) {
    const int rows = sh.seg[tid + 1] - sh.seg[tid];
    const int ncols = a.up ? (a.ffn.off[tid + 1] - a.ffn.off[tid]) : a.d;
    const int nt = a.up ? ncols / kBlockN : ncols / a.bn;
    const int mt = (rows + BM - 1) / BM;
    // A bytes of one M tile: 256 rows x the reduction length (d up, f_e down)
    const long long a_rows_bytes =
        static_cast<long long>(BM) * (a.up ? a.d : (a.ffn.off[tid + 1] - a.ffn.off[tid])) * 2;
    int gm = static_cast<int>(kL2GroupBudget / (a_rows_bytes > 0 ? a_rows_bytes : 1));
    gm = gm < 1 ? 1 : gm;
    sh.m_tiles[tid] = mt > 0 ? mt : 1;
    sh.n_tiles[tid] = nt > 0 ? nt : 1;
    sh.group_m[tid] = gm < sh.m_tiles[tid] ? gm : sh.m_tiles[tid];
    sh.tile_start[tid + 1] = mt * nt;  // count for now
  }
  __syncthreads();
  if (tid == 0) {
    sh.tile_start[0] = 0;
    for (int e = 0; e < E; ++e) sh.tile_start[e + 1] += sh.tile_start[e];
    sh.total_tiles = sh.tile_start[E];
    if (sh.seg[E] > a.rows) {  // more kept rows than the buffers hold: do nothing
      if (rank == 0) atomicOr(a.err, MOE_DEVERR_TILE_TABLE);
      sh.total_tiles = 0;
    }
  }
  tc_fence_before();
  cluster_sync();  // barrier inits and the TMEM allocation are visible pair-wide
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  const int total = sh.total_tiles;
  volatile int* abort_flag = &sh.abort_flag;
  const int half_bn = a.bn / 2;

  if (warp == 0) {
    // ================= TMA producer (one lane per CTA)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to_cta(smem_addr(&sh.full[0]), 0);
      const uint32_t tx_pair = 2u * (kABytes + static_cast<uint32_t>(half_bn) * BK * 2u);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int row0 = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA;
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
          const uint32_t bar = full_leader0 + static_cast<uint32_t>(s) * 8u;
          if (rank == 0) mbar_arrive_expect_tx(&sh.full[s], tx_pair);
          tma_load_2d_pair(sA, &mapA, bar, kb * BK, row0);
          if (a.up) {
            // leader: 128 columns of W1; peer: the same 128 columns of W3
            const CUtensorMap* mB = rank == 0 ? &mapB0 : &mapB1;
            const int n0 = o_e + c.nt * kBlockN;
            tma_load_2d_pair(sB, mB, bar, n0, kb * BK);
            tma_load_2d_pair(sB + kAtomBytes, mB, bar, n0 + 64, kb * BK);
          } else {
            const int n0 = c.nt * a.bn + static_cast<int>(rank) * half_bn;
            for (int j = 0; j < half_bn / 64; ++j)
              tma_load_2d_pair(sB + j * kAtomBytes, &mapB0, bar, n0 + j * 64, o_e + kb * BK);
          }
        }
      }
      // Drain: the last stages issued are released by the MMA (normally already
      // true), so no copy into this CTA is in flight when it exits.
      const uint32_t n_issued = it;
      for (uint32_t j = (n_issued > kStages ? n_issued - kStages : 0); j < n_issued; ++j) {
        volatile int no_abort = 0;
        mbar_wait(&sh.empty[j % kStages], (j / kStages) & 1u, &no_abort, a.err, MOE_DEVERR_TIMEOUT,
                  kWaitTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (leader CTA, one lane)
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(BM, a.bn, 1);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs, ++tcount) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int o_e = a.ffn.off[c.e];
        const int kblocks = a.up ? a.d / BK : (a.ffn.off[c.e + 1] - o_e) / BK;
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
        // both CTAs' epilogues release the buffer (the peer's arrival is remote)
        if (!mbar_wait(&sh.tempty[buf], aph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs,
                       true)) {
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
            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(&sh.empty[s], 0x3);  // frees the stage in both CTAs
        }
        if (!ok) break;
        umma_commit_pair_mc(&sh.tfull[buf], 0x3);  // both CTAs' accumulators ready
      }
      umma_commit_pair(&sh.drain);
      volatile int no_abort = 0;
      mbar_wait(&sh.drain, 0, &no_abort, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
    }
  } else {
    // ================= epilogue (warps 2..5, one TMEM lane quarter each)
    const int q = warp & 3;
    const int row_in_cta = q * 32 + lane;
    const uint32_t tempty_leader0 = map_to_cta(smem_addr(&sh.tempty[0]), 0);
    uint32_t tcount = 0;
    for (int tile = pair; tile < total; tile += npairs, ++tcount) {
      const TileCoord c = decode_tile(sh, E, tile);
      const uint32_t buf = tcount & 1u;
      const uint32_t aph = (tcount >> 1) & 1u;
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait(&sh.tfull[buf], aph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const int p = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA + row_in_cta;
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
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + buf * 8u);
    }
  }

  // ---- teardown: neither CTA leaves while its pair may still touch its memory
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace

size_t grouped_gemm_smem_bytes() { return kSmemBytes; }

cudaError_t prepare_grouped_gemm() {
  return cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

int grouped_gemm_max_grid(int num_sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_kernel, &cfg) != cudaSuccess || clusters <= 0) {
    cudaGetLastError();
    return num_sms & ~1;
  }
  const int grid = 2 * clusters;
  return grid < (num_sms & ~1) ? grid : (num_sms & ~1);
}

cudaError_t launch_grouped_gemm(const GemmArgs& a, const CUtensorMap& mapA, const CUtensorMap& mapB0,
                                const CUtensorMap& mapB1, int grid, cudaStream_t s) {
  grouped_gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(mapA, mapB0, mapB1, a);
  return cudaGetLastError();
}

}  // namespace moe
