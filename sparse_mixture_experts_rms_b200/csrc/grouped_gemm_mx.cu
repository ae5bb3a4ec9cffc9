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
//         a pair tile is 256 rows x 256 columns: 128 columns of W1 (leader's B
//         half) and the same 128 of W3 (peer's half)
//   down  y[p, n] = bf16( gate * (H8[p, :f_e] . W2[o_e + :, n]) ), 256 columns per tile
//         (128 when d is not a multiple of 256)
//
// Per pipeline stage each CTA holds 128 rows x 128 K of A (16 KB), its 128
// rows of B (16 KB), the scale block of its A rows (512 B, the layout
// tcgen05.cp.32x128b.warpx4 replicates into the four TMEM lane quarters) and
// the scales of all 256 B columns as one 4 KB paired region (both 512-B
// blocks, each stored four times over by the weight quantiser), which a
// single tcgen05.cp.128x256b turns into the same TMEM image: each copy
// instruction costs the MMA thread about as much as the next, so one copy of
// the region beats two of the blocks (measured -2.5 % up, -3 % down).  The
// MMA thread copies the scales into TMEM (columns 480..491) and then issues
// the stage's four K=32 MMAs, naming the scale byte of each; tcgen05
// operations of one thread run in order, so the next stage's copy cannot
// overtake them.  Row segments are padded to 128 rows, so a CTA's 128 rows
// are one scale block.
//
// N = 256 keeps the shared-memory operand traffic at 12 KB per 64 tensor
// cycles (N = 128 would need 8 KB per 32 and saturate shared memory).  Two
// 256-column accumulators and the scales exceed TMEM's 512 columns, so the
// accumulators overlap by 32 columns: buffer 0 = [0, 256), buffer 1 =
// [224, 480).  Each epilogue reads the shared 32 columns first and arrives on
// an "overlap drained" barrier; the next tile's MMAs wait for that (short)
// and for the full drain of the tile before it in their own buffer.
#include "moe_internal.h"
#include "mx.cuh"
#include "pair_pipe.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 256;
constexpr int BM_CTA = 128;
constexpr int BN = 256;                          // pair MMA N (the down GEMM may use 128)
constexpr int BK = 128;                          // K per stage (E4M3 bytes per row)
constexpr int kStages = 6;
constexpr int kABytes = BM_CTA * BK;             // 16 KB
constexpr int kBBytes = (BN / 2) * BK;           // 16 KB
constexpr int kSfBytes = 512;                    // one scale block: 128 rows x 4 scales
// stage: [B scales: one 4 KB paired region | A 16 KB | B 16 KB | A scales 512 B]
constexpr int kLoadBytes = kMxPairRegion + kABytes + kBBytes + kSfBytes;
constexpr int kStageBytes = (kLoadBytes + 1023) / 1024 * 1024;  // 1024-byte aligned stages
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr uint32_t kBuf1Col = 224;              // accumulators [0, 256) and [224, 480) overlap in [224, 256)
__device__ __forceinline__ uint32_t buf_col(uint32_t b) { return b ? kBuf1Col : 0u; }
constexpr uint32_t kSfaCol = 480, kSfbCol = 484; // 4 + 8 scale columns
constexpr int kEpiWarps = 4;
constexpr long long kL2GroupBudget = 48ll << 20;

struct __align__(8) MxShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t ovl[2];           // leader: both CTAs' epilogues read the buffer's overlap columns
  uint64_t drain;
  PairDrain pd;              // the producers' end-of-pipeline handshake
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
static_assert(kSmemBytes <= 232448, "shared memory above the per-block opt-in limit");

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
// x coordinate is a multiple of 128 bytes.  Both CTAs load the scales of all
// the tile's B columns.
__device__ __forceinline__ void issue_loads(const MxGemmArgs& a, const CUtensorMap* mA, const CUtensorMap* mB0,
                                            const CUtensorMap* mB1, const CUtensorMap* mSFA,
                                            const CUtensorMap* mSFB0, const CUtensorMap* mSFB1, const TileCoord& c,
                                            int kb, uint8_t* stage, uint32_t bar, int seg_e, int o_e,
                                            uint32_t rank, int bn) {
  uint8_t* sSFB = stage;
  uint8_t* sA = stage + kMxPairRegion;
  uint8_t* sB = sA + kABytes;
  uint8_t* sSFA = sB + kBBytes;
  const int row0 = seg_e + c.mt * BM + static_cast<int>(rank) * BM_CTA;  // a multiple of 128
  const int KA = a.up ? a.d : a.ldh;                                      // A's reduction length
  tma_load_2d_pair(sA, mA, bar, kb * BK, row0);
  tma_load_2d_pair(sSFA, mSFA, bar, 0, (row0 >> 7) * (KA >> 7) + kb);
  // B scales: one paired region (a box of 4 rows of 1 KB)
  if (a.up) {
    // leader: 128 columns of W1 (w1 rows), peer: the same 128 of W3; the region
    // holds both blocks of scales
    const int n0 = o_e + c.nt * 128;
    tma_load_2d_pair(sB, rank == 0 ? mB0 : mB1, bar, kb * BK, n0);
    tma_load_2d_pair(sSFB, mSFB0, bar, 0, 4 * ((n0 >> 7) * (a.d >> 7) + kb));
  } else {
    // the region of column blocks (2q, 2q + 1) holding this tile's n0
    const int n0 = c.nt * bn;
    tma_load_2d_pair(sB, mB0, bar, o_e + kb * BK, n0 + static_cast<int>(rank) * (bn / 2));
    tma_load_2d_pair(sSFB, mSFB0, bar, 0, 4 * ((n0 >> 8) * (a.F >> 7) + (o_e >> 7) + kb));
  }
}

// Arrive (once per warp) on the leader's overlap barrier of the buffer just
// read: the TMEM loads of the overlapping columns have completed.
__device__ __forceinline__ void signal_overlap(uint32_t ovl_leader, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(ovl_leader);
}

// One thread per accumulator row (TMEM lane); tcgen05.ld is warp-wide, so
// every lane loads and only the stores are predicated.  Chunks of 32 columns;
// the chunk holding the buffer's overlap columns (the last for buffer 0, the
// first for buffer 1) goes first, and the overlap barrier is signalled as
// soon as it has been read.
__device__ __forceinline__ void epilogue(const MxGemmArgs& a, const MxShared& sh, const TileCoord& c,
                                         uint32_t taddr, int row_in_cta, uint32_t rank, uint32_t buf, int bn,
                                         uint32_t ovl_leader, int lane) {
  const int p = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA + row_in_cta;
  const bool valid = p < sh.seg[c.e + 1];
  const int asg = valid ? a.perm[p] : -1;
  const size_t prow = static_cast<size_t>(valid ? p : 0);
  if (a.up) {
    const float r = asg >= 0 ? a.scale[asg / a.k] : 0.f;  // padding rows: r = 0 -> H = 0
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
      const int j = buf == 0 ? (i + 3) & 3 : i;  // buffer 0: v of chunk 3 is the overlap
      uint32_t u[32], v[32];
      tmem_ld_32x32b_x32(taddr + 32 * j, u);
      tmem_ld_32x32b_x32(taddr + 128 + 32 * j, v);
      tmem_ld_wait();
      if (i == 0) signal_overlap(ovl_leader, lane);
      if (!valid) continue;
      float h[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float uu = r * __uint_as_float(u[t]);
        h[t] = uu * sigmoid(uu) * (r * __uint_as_float(v[t]));
      }
      uint32_t q[8];
      const uint32_t sb = mx_quantize32(h, q);
      const int n = c.nt * 128 + 32 * j;  // column of H within the expert
      uint4* dst = reinterpret_cast<uint4*>(a.h8 + prow * a.ldh + n);
      dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
      dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
      a.hsf[mx_sf_offset(p, n, a.ldh)] = static_cast<uint8_t>(sb);
    }
  } else {
    const float g = asg >= 0 ? a.scale[asg] : 0.f;
    const int nchunk = bn / 32;
    __nv_bfloat16* dst = a.y + prow * a.d + c.nt * bn;
#pragma unroll 1
    for (int i = 0; i < nchunk; ++i) {
      const int j = buf == 0 ? (i + nchunk - 1) % nchunk : i;
      uint32_t u[32];
      tmem_ld_32x32b_x32(taddr + 32 * j, u);
      tmem_ld_wait();
      if (i == 0) signal_overlap(ovl_leader, lane);
      if (!valid) continue;
      uint32_t o[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) o[t] = pack_bf16(g * __uint_as_float(u[2 * t]), g * __uint_as_float(u[2 * t + 1]));
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * j);
#pragma unroll
      for (int t = 0; t < 4; ++t) d4[t] = make_uint4(o[4 * t], o[4 * t + 1], o[4 * t + 2], o[4 * t + 3]);
    }
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                           const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ CUtensorMap mapSFA,
                           const __grid_constant__ CUtensorMap mapSFB0, const __grid_constant__ CUtensorMap mapSFB1,
                           const __grid_constant__ MxGemmArgs a) {
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
      mbar_init(&sh.ovl[b], 2 * kEpiWarps);
    }
    mbar_init(&sh.drain, 1);
    pair_drain_init(sh.pd);
    sh.abort_flag = 0;
    sh.bad_segment = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapA);
    tma_prefetch_map(&mapB0);
    tma_prefetch_map(&mapB1);
    tma_prefetch_map(&mapSFA);
    tma_prefetch_map(&mapSFB0);
    tma_prefetch_map(&mapSFB1);
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
    const int nt = a.up ? f / 128 : a.d / a.bn;
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
  // main-loop waits: the workspace's limit; a wait that gives up also stops the other CTA
  const uint64_t wait_ns = wait_limit_ns(a.wait_ctl);
  const uint32_t peer_abort = map_to_cta(smem_addr(&sh.abort_flag), rank ^ 1u);

  if (warp == 0) {
    // ================= TMA producer (one lane per CTA)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to_cta(smem_addr(&sh.full[0]), 0);
      const uint32_t tx_pair = 2u * static_cast<uint32_t>(kABytes + (a.bn / 2) * BK + kSfBytes + kMxPairRegion);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int o_e = a.ffn.off[c.e];
        const int kblocks = sh.k_blocks[c.e];
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&sh.empty[s], ph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, false,
                         peer_abort)) {
            ok = false;
            break;
          }
          const uint32_t bar = full_leader0 + static_cast<uint32_t>(s) * 8u;
          if (rank == 0) mbar_arrive_expect_tx(&sh.full[s], tx_pair);
          issue_loads(a, &mapA, &mapB0, &mapB1, &mapSFA, &mapSFB0, &mapSFB1, c, kb, smem + s * kStageBytes, bar,
                      sh.seg[c.e], o_e, rank, a.bn);
        }
      }
      // no copy into either CTA is in flight when it exits, whatever stopped the loop
      pair_producer_drain<kStages>(sh.pd, sh.full, it, rank, tx_pair / 2u, a.err);
    }
  } else if (warp == 1) {
    // ================= MMA issuer (leader CTA, one lane)
    if (rank == 0 && lane == 0) {
      const uint32_t sfa_t = tmem_base + kSfaCol, sfb_t = tmem_base + kSfbCol;
      const uint32_t idesc_n = static_cast<uint32_t>(a.bn);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs, ++tcount) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int kblocks = sh.k_blocks[c.e];
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
        if (!mbar_wait(&sh.tempty[buf], aph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, true,
                       peer_abort)) {
          ok = false;
          break;
        }
        // the previous tile's epilogues have read the columns both buffers share
        if (tcount >= 1 && !mbar_wait(&sh.ovl[buf ^ 1u], ((tcount - 1) >> 1) & 1u, abort_flag, a.err,
                                      MOE_DEVERR_TIMEOUT, wait_ns, true, peer_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf_col(buf);
        // a 128-column down tile of an odd column block reads the region's second half
        const uint32_t sfb_k = sfb_t + ((!a.up && a.bn == 128 && (c.nt & 1)) ? 4u : 0u);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&sh.full[s], ph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, false, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aSFB = smem_addr(smem + s * kStageBytes);
          const uint32_t aA = aSFB + kMxPairRegion;
          const uint32_t aB = aA + kABytes;
          const uint32_t aSFA = aB + kBBytes;
          // A scale block: 32 lines x 16 bytes = four 8 x 16-byte core matrices, 128 bytes
          // apart; B: the paired region, 128 rows of 2 x 16 bytes, halves 2 KB apart
          tmem_cp_pair_32x128b_warpx4(sfa_t, smem_desc_noswz(aSFA, 0, 128));
          tmem_cp_pair_128x256b(sfb_t, smem_desc_noswz(aSFB, kMxPairRegion / 2, 128));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t adesc = smem_desc_sw128(aA + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(aB + kk * 32, 16, 1024);
            const uint32_t idesc = umma_idesc_mxf8(BM, idesc_n, kk, kk);
            umma_mxf8_pair(d_tmem, adesc, bdesc, idesc, sfa_t | (static_cast<uint32_t>(kk) << 30),
                           sfb_k | (static_cast<uint32_t>(kk) << 30), (kb | kk) != 0 ? 1u : 0u);
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
    const uint32_t ovl_leader0 = map_to_cta(smem_addr(&sh.ovl[0]), 0);
    uint32_t tcount = 0;
    for (int tile = pair; tile < total; tile += npairs, ++tcount) {
      const TileCoord c = decode_tile(sh, E, tile);
      const uint32_t buf = tcount & 1u;
      const uint32_t aph = (tcount >> 1) & 1u;
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait(&sh.tfull[buf], aph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, false, peer_abort);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      epilogue(a, sh, c, tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf_col(buf), row_in_cta, rank, buf,
               a.bn, ovl_leader0 + buf * 8u, lane);
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
                                   const CUtensorMap& mapSFB0, const CUtensorMap& mapSFB1, int grid,
                                   cudaStream_t s) {
  if (a.bn != 256 && !(a.bn == 128 && !a.up)) return cudaErrorInvalidValue;
  grouped_gemm_mx_kernel<<<grid, kThreads, kSmemBytes, s>>>(mapA, mapB0, mapB1, mapSFA, mapSFB0, mapSFB1, a);
  return cudaGetLastError();
}

}  // namespace moe
