// grouped_gemm_mx.cu -- the expert GEMMs with MXFP8 operands: 2-CTA
// (cta_group::2) block-scaled tcgen05.mma (kind::mxf8f6f4, E4M3 x E4M3 with
// E8M0 scales per 32 K, fp32 accumulators in TMEM).
//
// CODA sparse-MoE thread (digg.com): in a low-precision pipeline the
// conversions sit in epilogues -- here the permute writes the E4M3 codes and
// scales of x*gamma, and the up GEMM's epilogue quantises the SwiGLU output H
// (one thread holds 32 consecutive columns of a row: exactly one MX block) for
// the down GEMM.  OmniMoE summary, section 2.2: expert-centric grouped GEMM;
// nanoMOE notes: variable widths through cumulative offsets.
//
//   up    H8[p, n] = MX( silu(r_t * acc1) * (r_t * acc3) ),  acc1 = x8[p] . W1[:, o_e+n] ...
//         a pair tile is 256 rows x 128 columns: 64 columns of W1 (leader's B
//         half) and the same 64 of W3 (peer's half)
//   down  y[p, n] = bf16( gate * (H8[p, :f_e] . W2[o_e + :, n]) ), 128 columns per tile
//
// Per pipeline stage each CTA holds 128 rows x 128 K of A (16 KB), 64 rows of
// B (8 KB), and the scale blocks of its A rows and of all 128 B columns
// (512 B each, the layout tcgen05.cp takes).  The MMA thread copies both
// scale blocks into TMEM (columns 256..263) and then issues the stage's four
// K=32 MMAs, naming the scale byte of each; tcgen05 operations of one thread
// run in order, so the next stage's copy cannot overtake them.  Row segments
// are padded to 128 rows, so a CTA's 128 rows are one scale block.
#include "moe_internal.h"
#include "mx.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 256;
constexpr int BM_CTA = 128;
constexpr int BN = 128;                          // pair MMA N
constexpr int BK = 128;                          // K per stage (E4M3 bytes per row)
constexpr int kStages = 8;
constexpr int kABytes = BM_CTA * BK;             // 16 KB
constexpr int kBBytes = (BN / 2) * BK;           // 8 KB
constexpr int kSfBytes = 512;
constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;  // 25 KB, a multiple of 1024
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccCols = BN;                     // two accumulators: columns 0 and 128
constexpr uint32_t kSfaCol = 256, kSfbCol = 260;
constexpr int kEpiWarps = 4;
constexpr long long kL2GroupBudget = 48ll << 20;
static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned (128-byte swizzle)");

struct __align__(8) MxShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int bad_segment;
  int total_tiles;
  int tile_start[kMaxExperts + 1];
  int m_tiles[kMaxExperts];
  int n_tiles[kMaxExperts];
  int k_blocks[kMaxExperts];
  int group_m[kMaxExperts];
  int seg[kMaxExperts + 1];
};

constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + sizeof(MxShared);

struct TileCoord {
  int e, nt, mt;
};

__device__ __forceinline__ TileCoord decode_tile(const MxShared& sh, int E, int tile) {
  int e = 0;
  while (e + 1 < E && tile >= sh.tile_start[e + 1]) ++e;
  const int local = tile - sh.tile_start[e];
  const int mt_count = sh.m_tiles[e], nt_count = sh.n_tiles[e], gm = sh.group_m[e];
  const int g = local / (gm * nt_count);
  const int rem = local - g * gm * nt_count;
  const int gm_g = min(gm, mt_count - g * gm);
  return TileCoord{e, rem / gm_g, g * gm + rem % gm_g};
}

__device__ __forceinline__ float sigmoid(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// TMA loads of K block kb of tile c into one stage (this CTA's half); every
// x coordinate is a multiple of 128 bytes.
__device__ __forceinline__ void issue_loads(const MxGemmArgs& a, const CUtensorMap* mA, const CUtensorMap* mB0,
                                            const CUtensorMap* mB1, const CUtensorMap* mSFA,
                                            const CUtensorMap* mSFB, const TileCoord& c, int kb, uint8_t* stage,
                                            uint32_t bar, int seg_e, int o_e, uint32_t rank) {
  uint8_t* sA = stage;
  uint8_t* sB = stage + kABytes;
  uint8_t* sSFA = sB + kBBytes;
  uint8_t* sSFB = sSFA + kSfBytes;
  const int row0 = seg_e + c.mt * BM + static_cast<int>(rank) * BM_CTA;  // a multiple of 128
  const int KA = a.up ? a.d : a.ldh;                                      // A's reduction length
  tma_load_2d_pair(sA, mA, bar, kb * BK, row0);
  tma_load_2d_pair(sSFA, mSFA, bar, 0, (row0 >> 7) * (KA >> 7) + kb);
  if (a.up) {
    // leader: 64 columns of W1 (w1 rows), peer: the same 64 of W3
    tma_load_2d_pair(sB, rank == 0 ? mB0 : mB1, bar, kb * BK, o_e + c.nt * (BN / 2));
    tma_load_2d_pair(sSFB, mSFB, bar, 0, ((o_e >> 6) + c.nt) * (a.d >> 7) + kb);
  } else {
    tma_load_2d_pair(sB, mB0, bar, o_e + kb * BK, c.nt * BN + static_cast<int>(rank) * (BN / 2));
    tma_load_2d_pair(sSFB, mSFB, bar, 0, c.nt * (a.F >> 7) + (o_e >> 7) + kb);
  }
}

// One thread per accumulator row (TMEM lane); tcgen05.ld is warp-wide, so
// every lane loads and only the stores are predicated.
__device__ __forceinline__ void epilogue(const MxGemmArgs& a, const MxShared& sh, const TileCoord& c,
                                         uint32_t taddr, int row_in_cta, uint32_t rank) {
  const int p = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA + row_in_cta;
  const bool valid = p < sh.seg[c.e + 1];
  const int asg = valid ? a.perm[p] : -1;
  const size_t prow = static_cast<size_t>(valid ? p : 0);
  if (a.up) {
    const float r = asg >= 0 ? a.scale[asg / a.k] : 0.f;  // padding rows: r = 0 -> H = 0
#pragma unroll 1
    for (int cc = 0; cc < BN / 2; cc += 32) {
      uint32_t u[32], v[32];
      tmem_ld_32x32b_x32(taddr + cc, u);
      tmem_ld_32x32b_x32(taddr + BN / 2 + cc, v);
      tmem_ld_wait();
      if (!valid) continue;
      float h[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float uu = r * __uint_as_float(u[j]);
        h[j] = uu * sigmoid(uu) * (r * __uint_as_float(v[j]));
      }
      uint32_t q[8];
      const uint32_t sb = mx_quantize32(h, q);
      const int n = c.nt * (BN / 2) + cc;  // column of H within the expert
      uint4* dst = reinterpret_cast<uint4*>(a.h8 + prow * a.ldh + n);
      dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
      dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
      a.hsf[mx_sf_offset(p, n, a.ldh)] = static_cast<uint8_t>(sb);
    }
  } else {
    const float g = asg >= 0 ? a.scale[asg] : 0.f;
    __nv_bfloat16* dst = a.y + prow * a.d + c.nt * BN;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      uint32_t u[32];
      tmem_ld_32x32b_x32(taddr + cc, u);
      tmem_ld_wait();
      if (!valid) continue;
      uint32_t o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = pack_bf16(g * __uint_as_float(u[2 * j]), g * __uint_as_float(u[2 * j + 1]));
      uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
      for (int j = 0; j < 4; ++j) d4[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
    }
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                           const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ CUtensorMap mapSFA,
                           const __grid_constant__ CUtensorMap mapSFB, const __grid_constant__ MxGemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  MxShared& sh = *reinterpret_cast<MxShared*>(smem + kStages * kStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

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
    sh.bad_segment = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapA);
    tma_prefetch_map(&mapB0);
    tma_prefetch_map(&mapB1);
    tma_prefetch_map(&mapSFA);
    tma_prefetch_map(&mapSFB);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sh.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (tid < E + 1) sh.seg[tid] = a.offsets[tid];
  __syncthreads();
  if (tid < E) {
    const int rows = sh.seg[tid + 1] - sh.seg[tid];
    const int f = a.ffn.off[tid + 1] - a.ffn.off[tid];
    if ((sh.seg[tid] & 127) != 0 || rows < 0) sh.bad_segment = 1;  // scale blocks need 128-row segments
    const int nt = a.up ? f / (BN / 2) : a.d / BN;
    const int kb = a.up ? a.d / BK : f / BK;
    const int mt = (rows + BM - 1) / BM;
    const long long a_rows_bytes = static_cast<long long>(BM) * kb * BK;
    int gm = static_cast<int>(kL2GroupBudget / (a_rows_bytes > 0 ? a_rows_bytes : 1));
    gm = gm < 1 ? 1 : gm;
    sh.m_tiles[tid] = mt > 0 ? mt : 1;
    sh.n_tiles[tid] = nt > 0 ? nt : 1;
    sh.k_blocks[tid] = kb;
    sh.group_m[tid] = gm < sh.m_tiles[tid] ? gm : sh.m_tiles[tid];
    sh.tile_start[tid + 1] = (mt > 0 && nt > 0) ? mt * nt : 0;
  }
  __syncthreads();
  if (tid == 0) {
    sh.tile_start[0] = 0;
    for (int e = 0; e < E; ++e) sh.tile_start[e + 1] += sh.tile_start[e];
    sh.total_tiles = sh.tile_start[E];
    if (sh.seg[E] > a.rows || sh.bad_segment) {
      if (rank == 0) atomicOr(a.err, MOE_DEVERR_TILE_TABLE);
      sh.total_tiles = 0;
    }
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  const int total = sh.total_tiles;
  volatile int* abort_flag = &sh.abort_flag;

  if (warp == 0) {
    // ================= TMA producer (one lane per CTA)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to_cta(smem_addr(&sh.full[0]), 0);
      const uint32_t tx_pair = 2u * static_cast<uint32_t>(kStageBytes);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int o_e = a.ffn.off[c.e];
        const int kblocks = sh.k_blocks[c.e];
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&sh.empty[s], ph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          const uint32_t bar = full_leader0 + static_cast<uint32_t>(s) * 8u;
          if (rank == 0) mbar_arrive_expect_tx(&sh.full[s], tx_pair);
          issue_loads(a, &mapA, &mapB0, &mapB1, &mapSFA, &mapSFB, c, kb, smem + s * kStageBytes, bar, sh.seg[c.e],
                      o_e, rank);
        }
      }
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
      const uint32_t sfa_t = tmem_base + kSfaCol, sfb_t = tmem_base + kSfbCol;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs, ++tcount) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int kblocks = sh.k_blocks[c.e];
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
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
          const uint32_t aSFA = aB + kBBytes, aSFB = aSFA + kSfBytes;
          // scale blocks: 32 lines x 16 bytes = four 8 x 16-byte core matrices, 128 bytes apart
          tmem_cp_pair_32x128b_warpx4(sfa_t, smem_desc_noswz(aSFA, 0, 128));
          tmem_cp_pair_32x128b_warpx4(sfb_t, smem_desc_noswz(aSFB, 0, 128));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t adesc = smem_desc_sw128(aA + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(aB + kk * 32, 16, 1024);
            const uint32_t idesc = umma_idesc_mxf8(BM, BN, kk, kk);
            umma_mxf8_pair(d_tmem, adesc, bdesc, idesc, sfa_t | (static_cast<uint32_t>(kk) << 30),
                           sfb_t | (static_cast<uint32_t>(kk) << 30), (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(&sh.empty[s], 0x3);
        }
        if (!ok) break;
        umma_commit_pair_mc(&sh.tfull[buf], 0x3);
      }
      umma_commit_pair(&sh.drain);
      volatile int no_abort = 0;
      mbar_wait(&sh.drain, 0, &no_abort, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
    }
  } else {
    // ================= epilogue (warps 2..5, TMEM lane quarter warp % 4)
    const int q = warp & 3;
    const int row_in_cta = q * 32 + lane;
    const uint32_t tempty_leader0 = map_to_cta(smem_addr(&sh.tempty[0]), 0);
    uint32_t tcount = 0;
    for (int tile = pair; tile < total; tile += npairs, ++tcount) {
      const TileCoord c = decode_tile(sh, E, tile);
      const uint32_t buf = tcount & 1u;
      const uint32_t aph = (tcount >> 1) & 1u;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&sh.tfull[buf], aph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      epilogue(a, sh, c, tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kAccCols, row_in_cta, rank);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + buf * 8u);
    }
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace

cudaError_t prepare_grouped_gemm_mx() {
  return cudaFuncSetAttribute(grouped_gemm_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

cudaError_t launch_grouped_gemm_mx(const MxGemmArgs& a, const CUtensorMap& mapA, const CUtensorMap& mapB0,
                                   const CUtensorMap& mapB1, const CUtensorMap& mapSFA,
                                   const CUtensorMap& mapSFB, int grid, cudaStream_t s) {
  grouped_gemm_mx_kernel<<<grid, kThreads, kSmemBytes, s>>>(mapA, mapB0, mapB1, mapSFA, mapSFB, a);
  return cudaGetLastError();
}

}  // namespace moe
