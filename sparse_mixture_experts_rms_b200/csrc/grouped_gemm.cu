// grouped_gemm.cu -- the expert FFN's contractions, forward and backward, as
// persistent grouped GEMMs on the 5th-generation tensor cores: 2-CTA
// (cta_group::2) tcgen05.mma with fp32 accumulators in TMEM, operands staged
// by TMA into 128-byte-swizzled shared memory.
//
// OmniMoE summary (gist.science), section 2.2 "Expert-Centric Scheduling":
// with the rows grouped by expert, each expert's weight block is loaded once
// and reused over a batch of its tokens -- a grouped GEMM.  nanoMOE
// variable-size-experts notes (hbfreed.com): experts have different widths
// f_e (multiples of 128) inside concatenated W1 [d, F] / W2 [F, d], addressed
// through cumulative offsets; the work decomposition uses running sums of
// per-expert tile counts, never index * size ("Critical Bug Fix").
// CODA sparse-MoE thread (digg.com): the RMS statistic r of each token is
// applied in the epilogue of the first expert GEMM, and the RMSNorm backward
// is fused into that linear's backward, which is why r travels with the token.
//
// Modes (p = kept row of expert e, t = perm[p] / k; -1 in perm marks a
// padding row, whose outputs are zero):
//   up     H[p, n] = bf16( silu(r_t * acc1) * (r_t * acc3) ), acc1 = x_perm[p] . W1[:, o_e+n],
//          acc3 = x_perm[p] . W3[:, o_e+n].  One 256 x 256 x 16 pair MMA covers 128 columns
//          of W1 and the same 128 of W3.  Training also stores U = r*acc1, V = r*acc3.
//   down   y[p, n] = bf16( gate[perm[p]] * (H[p, :f_e] . W2[o_e + :, n]) ); training also
//          stores the ungated bf16(acc).  With k = 1 the layer has nothing to sum, so
//          the row goes straight to its token's row of the layer output (to_token).
//   bwd_h  G = dY[p] . W2[o_e + n, :]  (dY = gate * dout of the row's token), then
//          du = G * v * silu'(u), dv = G * silu(u) from the saved U, V, and
//          dS = bf16(r_t du), dS3 = bf16(r_t dv), plus the dr partial sum_n (du u + dv v) / r_t
//          of this N tile.
//   bwd_x  dX[p, c] = dS[p] . W1[c, o_e + :] + dS3[p] . W3[c, o_e + :]   (fp32 out)
//   wgrad_x dW1[c, o_e+n] = sum_p x_perm[p, c] dS[p, n], dW3 likewise with dS3 (fp32 out)
//   wgrad_h dW2[o_e+m, c] = sum_p H[p, m] dY[p, c]                          (fp32 out)
// The weight-gradient modes reduce over an expert's rows, so their K range is
// the expert's row segment; the training layout pads every segment to a
// multiple of 64 rows with zero rows so that K blocks never cross segments.
//
// CTA pairs (clusters of 2): a pair owns a 256-row x BN tile.  Each CTA loads
// its own 128 rows (M) of A and half of the BN columns of B; the leader CTA
// issues the pair MMA, which reads both CTAs' shared memory and writes each
// CTA's 128 rows of D into that CTA's TMEM.  Both CTAs' loads complete on the
// leader's "full" barrier; the MMA commit arrives on both CTAs' "empty" and
// "accumulator full" barriers; both CTAs' epilogues arrive on the leader's
// "accumulator empty" barrier.
//
// Tiles: expert e contributes ceil(M_e/256) * (N_e/BN) pair tiles, listed on
// the device from the row offsets (no host sync) in raster groups of M tiles
// whose A bytes fit a 48 MB L2 budget (M fastest inside a group).  Persistent
// pairs stride through the list.
//
// Warp roles (192 threads per CTA): warp 0 = TMA producer, warp 1 = MMA issuer
// (leader only) and TMEM owner, warps 2..5 = epilogue (TMEM -> registers ->
// shared -> TMA store), one per TMEM lane quarter.  Ring of 6 stages x (A 16
// KB + B 16 KB) per CTA; two TMEM accumulators of 256 fp32 columns, so the
// epilogue of tile i overlaps the mainloop of tile i+1 -- as long as it is
// shorter.  With a reduction of at most 1024 (up: d, down: the widest
// expert) a tile's MMAs take about as long as its epilogue, so up and down
// then run 8 epilogue warps (320 threads), two per lane quarter on the two
// halves of the tile's columns: measured -17 % (up, d = 1024), -27 % (up, d =
// 768), -14 % (down, f = 512).  At d = 2048 and above the extra warps cost
// 1-2 %, as they did (2.5-5 %) on every mode of the Mixtral shape: they share
// sub-partitions with the producer and MMA warps.
//
// Epilogue output: a thread holds one accumulator row, so storing rows
// directly makes every warp-wide store touch 32 rows in 16-byte pieces, which
// costs the load/store path 8x the wavefronts of whole-row segments and slows
// the MMAs sharing it (measured 5-7% on the training up, dS and weight-
// gradient GEMMs).  Instead each epilogue warp writes its 32 rows of a
// 32-column chunk into a swizzled 32 x 32 box in shared memory (conflict-free:
// lane = row) and one lane stores the box by TMA; 8 KB of boxes per warp form
// a ring.  The dS GEMM also loads its saved U, V chunks as boxes by TMA.  A
// box is used when the warp's 32 rows all belong to the expert (always in the
// 64-row-padded training layout); otherwise the threads store their rows.
// Every wait is bounded (4 s by default; the workspace header can set another
// limit) and sets a device error bit instead of hanging; a wait that gives up
// stops both CTAs of the pair, which still let every copy and MMA in flight
// finish before they exit (pair_pipe.cuh).
#include "moe_internal.h"
#include "pair_pipe.cuh"
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
constexpr int kEpiWarps = 4;                  // one per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer, MMA, epilogue
// up and down with a short reduction may run 8 epilogue warps, two per TMEM
// lane quarter on the two halves of the tile's columns
__host__ __device__ constexpr int threads_of(int epi) { return 64 + 32 * epi; }
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;                 // columns per accumulator buffer
constexpr int kAtomBytes = BK * 64 * 2;       // one 64(mn) x 64(k) MN-major box: 8 KB
constexpr long long kL2GroupBudget = 48ll << 20;  // A bytes of one raster group
// Epilogue staging: per epilogue warp four 32-row x 32-column bf16 boxes
// (2 KB each, 64-byte swizzle) through which up, down and bwd_h move their
// rows by TMA
constexpr int kEpiBoxBytes = 32 * 32 * 2;
constexpr int kEpiBytes = kEpiWarps * 4 * kEpiBoxBytes;  // 32 KB

struct __align__(8) GemmShared {
  uint64_t full[kStages];    // leader: both CTAs' loads of a stage landed
  uint64_t empty[kStages];   // each CTA: the MMAs reading its stage finished
  uint64_t tfull[2];         // each CTA: accumulator buffer ready
  uint64_t tempty[2];        // leader: both CTAs' epilogues drained the buffer
  uint64_t drain;
  uint64_t ebar[kEpiWarps][2];  // bwd_h: an epilogue warp's U, V box pair landed
  PairDrain pd;                 // the producers' end-of-pipeline handshake
  uint32_t tmem_base;
  int abort_flag;
  int bad_segment;
  int total_tiles;
  int tile_start[kMaxExperts + 1];
  int m_tiles[kMaxExperts];
  int n_tiles[kMaxExperts];
  int k_blocks[kMaxExperts];
  int group_m[kMaxExperts];  // raster block: group_m x group_n tiles (see decode_tile)
  int group_n[kMaxExperts];
  int seg[kMaxExperts + 1];
};

// [stages | bwd_h epilogue staging | GemmShared]
constexpr size_t kSmemBytes = 1024 /* alignment slack */ + kStages * kStageBytes + kEpiBytes + sizeof(GemmShared);
static_assert(kSmemBytes <= 232448, "shared memory above the per-block opt-in limit");

struct TileCoord {
  int e, nt, mt;
};

// Tiles of expert e are rastered in blocks of group_m[e] x group_n[e] (M x N)
// tiles, M fastest inside a block, blocks N-fastest along a row of blocks, so
// the pairs running together share a few A row panels and B column panels in
// L2.  When all of an expert's A panels fit an L2 budget the block spans the
// expert (plain M-fastest order: every B panel is read once); when they do
// not (a long reduction), blocks are about as square as the resident pairs
// allow, so a wave touches about 2 sqrt(pairs) panels instead of
// group_m + every N panel.
__device__ __forceinline__ TileCoord decode_tile(const GemmShared& sh, int E, int tile) {
  int e = 0;
  while (e + 1 < E && tile >= sh.tile_start[e + 1]) ++e;
  const int local = tile - sh.tile_start[e];
  const int mt_count = sh.m_tiles[e], nt_count = sh.n_tiles[e];
  const int gm = sh.group_m[e], gn = sh.group_n[e];
  const int bm = local / (gm * nt_count);            // row of blocks
  const int rem = local - bm * gm * nt_count;
  const int gm_b = min(gm, mt_count - bm * gm);      // the last row may be short
  const int bn = rem / (gm_b * gn);                  // block in the row
  const int rem2 = rem - bn * gm_b * gn;
  return TileCoord{e, bn * gn + rem2 / gm_b, bm * gm + rem2 % gm_b};
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float sigmoid(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }
__device__ __forceinline__ float silu(float z) { return z * sigmoid(z); }

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&o)[16]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) d4[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

__device__ __forceinline__ void store_row_f32(float* dst, const uint32_t (&u)[32], bool zero) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    d4[j] = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                 : make_float4(__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                               __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3]));
}

template <int MODE>
struct Traits {
  static constexpr bool a_mn = (MODE == kGemmWgradX || MODE == kGemmWgradH);
  static constexpr bool b_mn = (MODE == kGemmUp || MODE == kGemmDown || MODE == kGemmWgradX ||
                                MODE == kGemmWgradH);
  static constexpr bool row_tiles = !a_mn;  // M runs over an expert's rows
};

// Extent of the tile space of expert e: M extent (rows of D), N tiles, K blocks.
template <int MODE>
__device__ __forceinline__ void geometry(int rows, int f, int d, int bn, int& mext, int& nt, int& kb) {
  if (MODE == kGemmUp) {
    mext = rows; nt = f / kBlockN; kb = d / BK;
  } else if (MODE == kGemmDown) {
    mext = rows; nt = d / bn; kb = f / BK;
  } else if (MODE == kGemmBwdH) {
    mext = rows; nt = f / bn; kb = d / BK;
  } else if (MODE == kGemmBwdX) {
    mext = rows; nt = d / bn; kb = 2 * f / BK;
  } else if (MODE == kGemmWgradX) {
    mext = d; nt = 2 * f / bn; kb = rows / BK;
  } else {  // kGemmWgradH
    mext = f; nt = d / bn; kb = rows / BK;
  }
}

struct Maps {
  const CUtensorMap* a0;
  const CUtensorMap* a1;
  const CUtensorMap* b0;
  const CUtensorMap* b1;
};

// TMA loads of K block kb of tile c into one stage (this CTA's half).
// Every x coordinate is a multiple of 64 elements (128 B).
template <int MODE>
__device__ __forceinline__ void issue_loads(const Maps& m, const TileCoord& c, int kb, uint8_t* sA,
                                            uint8_t* sB, uint32_t bar, int seg_e, int o_e, int f,
                                            uint32_t rank, int bn) {
  const int half_bn = bn / 2;
  if (Traits<MODE>::row_tiles) {
    const int row0 = seg_e + c.mt * BM + static_cast<int>(rank) * BM_CTA;
    if (MODE == kGemmUp) {
      // leader: 128 columns of W1; peer: the same 128 columns of W3 (MN-major)
      tma_load_2d_pair(sA, m.a0, bar, kb * BK, row0);
      const CUtensorMap* mB = rank == 0 ? m.b0 : m.b1;
      const int n0 = o_e + c.nt * kBlockN;
      tma_load_2d_pair(sB, mB, bar, n0, kb * BK);
      tma_load_2d_pair(sB + kAtomBytes, mB, bar, n0 + 64, kb * BK);
    } else if (MODE == kGemmDown) {
      tma_load_2d_pair(sA, m.a0, bar, kb * BK, row0);
      const int n0 = c.nt * bn + static_cast<int>(rank) * half_bn;
      for (int j = 0; j < half_bn / 64; ++j)
        tma_load_2d_pair(sB + j * kAtomBytes, m.b0, bar, n0 + j * 64, o_e + kb * BK);
    } else if (MODE == kGemmBwdH) {
      // B = rows o_e + n of W2 [F, d], K-major (box 64 k x half_bn rows)
      tma_load_2d_pair(sA, m.a0, bar, kb * BK, row0);
      tma_load_2d_pair(sB, m.b0, bar, kb * BK, o_e + c.nt * bn + static_cast<int>(rank) * half_bn);
    } else {  // kGemmBwdX: K runs over f_e columns of dS (x W1^T), then of dS3 (x W3^T)
      const int kf = f / BK;
      const bool second = kb >= kf;
      const int kk = second ? kb - kf : kb;
      tma_load_2d_pair(sA, second ? m.a1 : m.a0, bar, kk * BK, row0);
      tma_load_2d_pair(sB, second ? m.b1 : m.b0, bar, o_e + kk * BK,
                       c.nt * bn + static_cast<int>(rank) * half_bn);
    }
  } else {
    // weight gradients: A^T and B both MN-major, K = rows seg_e + kb*64 ...
    const int m0 = c.mt * BM + static_cast<int>(rank) * BM_CTA;
    const int k0 = seg_e + kb * BK;
    tma_load_2d_pair(sA, m.a0, bar, m0, k0);
    tma_load_2d_pair(sA + kAtomBytes, m.a0, bar, m0 + 64, k0);
    int n0 = c.nt * bn + static_cast<int>(rank) * half_bn;
    const CUtensorMap* mB = m.b0;
    if (MODE == kGemmWgradX && n0 >= f) {  // dW3 half of the [dW1 | dW3] N range
      n0 -= f;
      mB = m.b1;
    }
    for (int j = 0; j < half_bn / 64; ++j) tma_load_2d_pair(sB + j * kAtomBytes, mB, bar, n0 + j * 64, k0);
  }
}

// ---- epilogues: one thread per accumulator row (TMEM lane), 32 columns per load
// Byte offset of 16-byte unit `unit` (0..3) of row `row` in a box of 64-byte
// rows under TMA's 64-byte swizzle (unit bits [4,6) ^= address bits [7,9)).
__device__ __forceinline__ uint32_t sw64(int row, int unit) {
  return static_cast<uint32_t>(row * 64 + ((unit ^ ((row >> 1) & 3)) << 4));
}

// One lane's row (32 bf16 = 16 words) into a staged 32 x 32 box.
__device__ __forceinline__ void box_put_row(uint8_t* box, int lane, const uint32_t (&o)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(box + sw64(lane, j)) = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

// One lane's row (32 fp32) into a staged 32 x 32 fp32 box of 128-byte rows
// under TMA's 128-byte swizzle (unit bits [4,7) ^= address bits [7,10)).
__device__ __forceinline__ void box_put_row_f32(uint8_t* box, int lane, const uint32_t (&u)[32], bool zero) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) =
        zero ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(u[4 * j], u[4 * j + 1], u[4 * j + 2], u[4 * j + 3]);
}

// Staged output of a warp: `nbox` boxes per 32-column chunk in a ring of
// bpw / nbox slots (the warp's bpw boxes).  Before a slot is rewritten, lane 0
// waits until at most (slots - 1) of its bulk-store groups -- one per chunk --
// are still reading shared memory.
__device__ __forceinline__ uint8_t* box_slot_acquire(uint8_t* boxes, int nbox, uint32_t n, int lane, int bpw) {
  const int slots = bpw / nbox;
  if (lane == 0) bulk_wait_group_read_allow(slots - 1);
  __syncwarp();
  return boxes + (n % static_cast<uint32_t>(slots)) * nbox * kEpiBoxBytes;
}

// After every lane wrote its rows of the slot's boxes: lane 0 stores box b
// with map m[b] at (x, p0), one bulk group for the chunk.
__device__ __forceinline__ void box_slot_store(const EpiMaps& em, uint8_t* slot, int nbox, int x, int p0,
                                               int lane) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    for (int b = 0; b < nbox; ++b) tma_store_2d(&em.m[b], slot + b * kEpiBoxBytes, x, p0);
    bulk_commit_group();
  }
}

// A row-tile epilogue thread's assignment (perm entry of its row, -1 past the
// expert's rows or at padding) and scale (up: r of the token; down: the
// gate), read before the thread waits for the tile's accumulator so that the
// two dependent loads overlap the tile's MMAs.
struct RowPre {
  int asg;
  float scale;
};

template <int MODE>
__device__ __forceinline__ RowPre row_pre(const GemmArgs& a, const GemmShared& sh, const TileCoord& c, int q,
                                          int lane, uint32_t rank) {
  const int p = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA + q * 32 + lane;
  const int asg = p < sh.seg[c.e + 1] ? a.perm[p] : -1;
  float scale = 0.f;
  if (MODE == kGemmUp && asg >= 0) scale = a.scale[asg / a.k];
  if (MODE == kGemmDown && asg >= 0) scale = a.scale[asg];
  return RowPre{asg, scale};
}

// Row-tile epilogues (up, down, bwd_x); one thread per accumulator row
// (TMEM lane), 32-column chunks.  The outputs leave through shared memory by
// TMA when the warp's 32 rows all belong to the expert (`staged`); otherwise
// each thread stores its own row.  Padding rows of the training layout
// (perm = -1) get zeros.
template <int MODE>
__device__ __forceinline__ void epilogue_rows(const GemmArgs& a, const GemmShared& sh, const EpiMaps& em,
                                              const TileCoord& c, uint32_t taddr, int q, int lane,
                                              uint32_t rank, uint8_t* boxes, int bpw, uint32_t& n, int c_lo,
                                              int c_hi, const RowPre& pre) {
  const int p0 = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA + q * 32;
  const int p = p0 + lane;
  const bool valid = p < sh.seg[c.e + 1];
  const int nbox_max = MODE == kGemmUp ? (a.out_u != nullptr ? 3 : 1) : (MODE == kGemmDown && a.out_yu != nullptr ? 2 : 1);
  // rows sent to their tokens (down, k = 1) are not contiguous: no boxes
  const bool staged = a.staged != 0 && a.to_token == 0 && nbox_max <= bpw && p0 + 32 <= sh.seg[c.e + 1];
  const int asg = pre.asg;
  const bool pad = valid && asg < 0;
  const size_t prow = static_cast<size_t>(valid ? p : 0);
  if (MODE == kGemmUp) {
    const float scale = pre.scale;
    const size_t off = prow * a.ld_out + c.nt * kBlockN;
    const bool keep_uv = a.out_u != nullptr;
    const int nbox = keep_uv ? 3 : 1;
#pragma unroll 1
    for (int cc = c_lo; cc < c_hi; cc += 32) {
      uint32_t u[32], v[32];
      tmem_ld_32x32b_x32(taddr + cc, u);
      tmem_ld_32x32b_x32(taddr + kBlockN + cc, v);
      tmem_ld_wait();
      if (!valid) continue;  // never taken when staged
      uint32_t o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float h0 = silu(scale * __uint_as_float(u[2 * j])) * (scale * __uint_as_float(v[2 * j]));
        const float h1 = silu(scale * __uint_as_float(u[2 * j + 1])) * (scale * __uint_as_float(v[2 * j + 1]));
        o[j] = pad ? 0u : pack_bf16(h0, h1);
      }
      uint8_t* slot = nullptr;
      if (staged) {
        slot = box_slot_acquire(boxes, nbox, n++, lane, bpw);
        box_put_row(slot, lane, o);
      } else {
        store_row_bf16(a.out + off + cc, o);
      }
      if (keep_uv) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          o[j] = pad ? 0u : pack_bf16(scale * __uint_as_float(u[2 * j]), scale * __uint_as_float(u[2 * j + 1]));
        if (staged) box_put_row(slot + kEpiBoxBytes, lane, o);
        else store_row_bf16(a.out_u + off + cc, o);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          o[j] = pad ? 0u : pack_bf16(scale * __uint_as_float(v[2 * j]), scale * __uint_as_float(v[2 * j + 1]));
        if (staged) box_put_row(slot + 2 * kEpiBoxBytes, lane, o);
        else store_row_bf16(a.out_v + off + cc, o);
      }
      if (staged) box_slot_store(em, slot, nbox, c.nt * kBlockN + cc, p0, lane);
    }
  } else if (MODE == kGemmDown) {
    const float scale = pre.scale;
    const size_t orow = a.to_token ? static_cast<size_t>(asg >= 0 ? asg : 0) : prow;
    const size_t off = orow * a.ld_out + c.nt * a.bn;
    const bool keep_yu = a.out_yu != nullptr;
    const int nbox = keep_yu ? 2 : 1;
    // one 32-column chunk: gate scale, bf16 pack, out through the staged boxes or row stores
    auto chunk = [&](const uint32_t (&u)[32], int cc) {
      if (!valid || (a.to_token && asg < 0)) return;  // never taken when staged
      uint32_t o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        o[j] = pad ? 0u : pack_bf16(scale * __uint_as_float(u[2 * j]), scale * __uint_as_float(u[2 * j + 1]));
      uint8_t* slot = nullptr;
      if (staged) {
        slot = box_slot_acquire(boxes, nbox, n++, lane, bpw);
        box_put_row(slot, lane, o);
      } else {
        store_row_bf16(a.out + off + cc, o);
      }
      if (keep_yu) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          o[j] = pad ? 0u : pack_bf16(__uint_as_float(u[2 * j]), __uint_as_float(u[2 * j + 1]));
        if (staged) box_put_row(slot + kEpiBoxBytes, lane, o);
        else store_row_bf16(a.out_yu + off + cc, o);
      }
      if (staged) box_slot_store(em, slot, nbox, c.nt * a.bn + cc, p0, lane);
    };
    // the next chunk's TMEM load is in flight while this one is scaled,
    // packed, fenced and stored (two 32-column register sets)
    uint32_t ua[32], ub[32];
    tmem_ld_32x32b_x32(taddr + c_lo, ua);
#pragma unroll 1
    for (int cc = c_lo; cc < c_hi; cc += 64) {
      tmem_ld_wait();  // ua
      if (cc + 32 < c_hi) tmem_ld_32x32b_x32(taddr + cc + 32, ub);
      chunk(ua, cc);
      if (cc + 32 >= c_hi) break;
      tmem_ld_wait();  // ub
      if (cc + 64 < c_hi) tmem_ld_32x32b_x32(taddr + cc + 64, ua);
      chunk(ub, cc + 32);
    }
  } else {  // kGemmBwdX: fp32 rows, staged as 32 x 32 fp32 boxes (128-byte swizzle, two per warp)
    float* dst = a.out_f0 + prow * a.ld_f + c.nt * a.bn;
#pragma unroll 1
    for (int cc = 0; cc < a.bn; cc += 32) {
      uint32_t u[32];
      tmem_ld_32x32b_x32(taddr + cc, u);
      tmem_ld_wait();
      if (!valid) continue;  // never taken when staged
      if (staged) {
        uint8_t* box = boxes + (n++ & 1u) * 2 * kEpiBoxBytes;
        if (lane == 0) bulk_wait_group_read_allow(1);
        __syncwarp();
        box_put_row_f32(box, lane, u, pad);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&em.m[0], box, c.nt * a.bn + cc, p0);
          bulk_commit_group();
        }
      } else {
        store_row_f32(dst + cc, u, pad);
      }
    }
  }
}

// bwd_h epilogue of one warp: its 32 accumulator rows (TMEM lane quarter q)
// in 32-column chunks.  The saved U, V chunks come in and dS, dS3 go out as
// whole 32 x 32 boxes through shared memory by TMA, so global memory sees
// contiguous row segments; each lane reads and writes its own row of the
// boxes, conflict-free under the swizzle.  Two box pairs per warp form a
// ring: chunk n reads U, V from pair n % 2, overwrites them with dS, dS3 and
// stores them from there, while chunk n + 1's U, V load into the other pair
// (once that pair's previous store has read it out).  The training layout
// pads every expert segment to a multiple of 64 rows, so a box lies entirely
// inside or entirely past the expert's rows.  `n` counts this warp's chunks
// across tiles.  Returns false when a wait gave up.
__device__ __forceinline__ bool epilogue_dsh(const GemmArgs& a, const GemmShared& sh, const EpiMaps& em,
                                             const TileCoord& c, uint32_t taddr, int q, int lane, uint32_t rank,
                                             uint8_t* boxes, uint64_t* bars, uint32_t& n, volatile int* abort_flag,
                                             uint64_t wait_ns, uint32_t peer_abort) {
  const int p0 = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA + q * 32;
  if (p0 >= sh.seg[c.e + 1]) return true;
  const int p = p0 + lane;
  const int asg = a.perm[p];
  const bool pad = asg < 0;  // padding row: zeros out
  const float r = pad ? 0.f : a.scale[asg / a.k];
  const int col0 = c.nt * a.bn;
  auto load_uv = [&](uint32_t slot, int col) {  // lane 0
    uint8_t* bx = boxes + slot * 2 * kEpiBoxBytes;
    bulk_wait_group_read0();  // the slot's previous store has read it
    mbar_arrive_expect_tx(&bars[slot], 2 * kEpiBoxBytes);
    tma_load_2d(bx, &em.m[0], &bars[slot], col, p0);
    tma_load_2d(bx + kEpiBoxBytes, &em.m[1], &bars[slot], col, p0);
  };
  if (lane == 0) load_uv(n & 1u, col0);
  float dr = 0.f;
#pragma unroll 1
  for (int cc = 0; cc < a.bn; cc += 32, ++n) {
    const uint32_t slot = n & 1u;
    uint8_t* s_u = boxes + slot * 2 * kEpiBoxBytes;
    uint8_t* s_v = s_u + kEpiBoxBytes;
    uint32_t g[32];
    tmem_ld_32x32b_x32(taddr + cc, g);
    if (lane == 0 && cc + 32 < a.bn) load_uv(slot ^ 1u, col0 + cc + 32);
    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars[slot], (n >> 1) & 1u, abort_flag, a.err,
                                                     MOE_DEVERR_TIMEOUT, wait_ns, false, peer_abort));
    tmem_ld_wait();
    if (!ok) {
      if (lane == 0) {  // let the loads in flight land (bounded) before giving up
        volatile int no_abort = 0;
        mbar_wait(&bars[slot], (n >> 1) & 1u, &no_abort, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
        if (cc + 32 < a.bn)
          mbar_wait(&bars[slot ^ 1u], ((n + 1) >> 1) & 1u, &no_abort, a.err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
      }
      return false;
    }
    uint32_t uw[16], vw[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 u4 = *reinterpret_cast<const uint4*>(s_u + sw64(lane, j));
      const uint4 v4 = *reinterpret_cast<const uint4*>(s_v + sw64(lane, j));
      uw[4 * j] = u4.x; uw[4 * j + 1] = u4.y; uw[4 * j + 2] = u4.z; uw[4 * j + 3] = u4.w;
      vw[4 * j] = v4.x; vw[4 * j + 1] = v4.y; vw[4 * j + 2] = v4.z; vw[4 * j + 3] = v4.w;
    }
    uint32_t o1[16], o3[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float du[2], dv[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float uu = h ? bf16_hi(uw[j]) : bf16_lo(uw[j]);
        const float vv = h ? bf16_hi(vw[j]) : bf16_lo(vw[j]);
        const float gg = __uint_as_float(g[2 * j + h]);
        const float sg = sigmoid(uu);
        du[h] = gg * vv * (sg * (1.0f + uu * (1.0f - sg)));
        dv[h] = gg * (uu * sg);
        dr += du[h] * uu + dv[h] * vv;
      }
      o1[j] = pad ? 0u : pack_bf16(r * du[0], r * du[1]);
      o3[j] = pad ? 0u : pack_bf16(r * dv[0], r * dv[1]);
    }
    // each lane overwrites only its own row of the boxes it has just read
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      *reinterpret_cast<uint4*>(s_u + sw64(lane, j)) = make_uint4(o1[4 * j], o1[4 * j + 1], o1[4 * j + 2], o1[4 * j + 3]);
      *reinterpret_cast<uint4*>(s_v + sw64(lane, j)) = make_uint4(o3[4 * j], o3[4 * j + 1], o3[4 * j + 2], o3[4 * j + 3]);
    }
    fence_proxy_async_smem();  // the boxes' writes are visible to the TMA stores
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&em.m[2], s_u, col0 + cc, p0);
      tma_store_2d(&em.m[3], s_v, col0 + cc, p0);
      bulk_commit_group();
    }
  }
  a.drp[static_cast<size_t>(p) * a.ld_drp + c.nt] = pad ? 0.f : dr / r;
  return true;
}

// Weight gradients: the accumulator row is an output row of dW (a column of
// x_perm or H); an expert with no rows gets zeros.  The fp32 rows leave
// through shared memory by TMA (32 x 32 fp32 boxes, 128-byte swizzle, a ring
// of two per warp) when tensor maps were given; every box is whole, since d
// and the expert widths are multiples of 128.
template <int MODE>
__device__ __forceinline__ void epilogue_wgrad(const GemmArgs& a, const GemmShared& sh, const EpiMaps& em,
                                               const TileCoord& c, uint32_t taddr, int q, int lane,
                                               uint32_t rank, uint8_t* boxes, uint32_t& n) {
  const int o_e = a.ffn.off[c.e];
  const int f = a.ffn.off[c.e + 1] - o_e;
  const int m0 = c.mt * BM + static_cast<int>(rank) * BM_CTA + q * 32;
  const int m = m0 + lane;
  const bool zero = sh.k_blocks[c.e] == 0;
  const int m_end = MODE == kGemmWgradX ? a.d : f;
  const bool valid = m < m_end;
  const bool staged = a.staged != 0 && m0 + 32 <= m_end;
#pragma unroll 1
  for (int cc = 0; cc < a.bn; cc += 32) {
    uint32_t u[32];
    if (!zero) {
      tmem_ld_32x32b_x32(taddr + cc, u);
      tmem_ld_wait();
    }
    if (!valid) continue;  // never taken when staged
    const int nn = c.nt * a.bn + cc;
    if (staged) {
      uint8_t* box = boxes + (n++ & 1u) * 2 * kEpiBoxBytes;  // 4 KB fp32 box
      if (lane == 0) bulk_wait_group_read_allow(1);
      __syncwarp();
      box_put_row_f32(box, lane, u, zero);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (MODE == kGemmWgradX)
          tma_store_2d(&em.m[nn < f ? 0 : 1], box, o_e + (nn < f ? nn : nn - f), m0);
        else
          tma_store_2d(&em.m[0], box, nn, o_e + m0);
        bulk_commit_group();
      }
      continue;
    }
    float* dst;
    if (MODE == kGemmWgradX)
      dst = (nn < f ? a.out_f0 + static_cast<size_t>(m) * a.ld_f + o_e + nn
                    : a.out_f1 + static_cast<size_t>(m) * a.ld_f + o_e + (nn - f));
    else
      dst = a.out_f0 + static_cast<size_t>(o_e + m) * a.ld_f + nn;
    store_row_f32(dst, u, zero);
  }
}

template <int MODE, int EPI, int AG = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_of(EPI), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mapA0, const __grid_constant__ CUtensorMap mapA1,
                        const __grid_constant__ CUtensorMap mapB0, const __grid_constant__ CUtensorMap mapB1,
                        const __grid_constant__ GemmArgs a, const __grid_constant__ EpiMaps em) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_boxes = smem + kStages * kStageBytes;
  GemmShared& sh = *reinterpret_cast<GemmShared*>(epi_boxes + kEpiBytes);
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
      mbar_init(&sh.tempty[b], 2 * EPI);
    }
    mbar_init(&sh.drain, 1);
    for (int w = 0; w < kEpiWarps; ++w) {
      mbar_init(&sh.ebar[w][0], 1);
      mbar_init(&sh.ebar[w][1], 1);
    }
    pair_drain_init(sh.pd);
    sh.abort_flag = 0;
    sh.bad_segment = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapA0);
    tma_prefetch_map(&mapB0);
    if (MODE == kGemmBwdX) tma_prefetch_map(&mapA1);
    if (MODE == kGemmUp || MODE == kGemmBwdX || MODE == kGemmWgradX) tma_prefetch_map(&mapB1);
    if (MODE == kGemmBwdH)
      for (int i = 0; i < 4; ++i) tma_prefetch_map(&em.m[i]);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sh.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  // barriers, TMEM and descriptors are set up while the kernel before drains;
  // the row offsets and every operand come from the kernels before
  griddep_wait();
  if (tid < E + 1) sh.seg[tid] = a.offsets[tid];
  __syncthreads();
  if (tid < E) {
    const int rows = sh.seg[tid + 1] - sh.seg[tid];
    const int f = a.ffn.off[tid + 1] - a.ffn.off[tid];
    int mext, nt, kb;
    geometry<MODE>(rows, f, a.d, a.bn, mext, nt, kb);
    // K of the weight gradients is a row segment: it must be whole K blocks
    if (!Traits<MODE>::row_tiles && (rows < 0 || rows % BK != 0)) sh.bad_segment = 1;
    // bwd_h moves 32-row boxes: segments must start and end on 32-row boundaries
    if (MODE == kGemmBwdH && (sh.seg[tid] % 32 != 0 || rows < 0 || rows % 32 != 0)) sh.bad_segment = 1;
    const int mt = (mext + BM - 1) / BM;
    const long long a_panel = static_cast<long long>(BM) * kb * BK * 2;  // one M tile's A over all K
    const long long b_panel = static_cast<long long>(a.bn) * kb * BK * 2;  // one N tile's B over all K
    const int mtc = mt > 0 ? mt : 1, ntc = nt > 0 ? nt : 1;
    int gm = mtc, gn = ntc;
    if (a_panel > 0 && static_cast<long long>(mtc) * a_panel > kL2GroupBudget) {
      // square-ish blocks of about one wave of pairs
      const int pairs = static_cast<int>(gridDim.x >> 1);
      gm = static_cast<int>(sqrtf(static_cast<float>(pairs) * static_cast<float>(b_panel) /
                                  static_cast<float>(a_panel)));
      gm = gm < 1 ? 1 : (gm > mtc ? mtc : gm);
      gn = pairs / gm;
      gn = gn < 1 ? 1 : (gn > ntc ? ntc : gn);
    }
    sh.m_tiles[tid] = mtc;
    sh.n_tiles[tid] = ntc;
    sh.k_blocks[tid] = kb;
    sh.group_m[tid] = gm;
    sh.group_n[tid] = gn;
    sh.tile_start[tid + 1] = (mt > 0 && nt > 0) ? mt * nt : 0;  // count for now
  }
  __syncthreads();
  if (tid == 0) {
    sh.tile_start[0] = 0;
    for (int e = 0; e < E; ++e) sh.tile_start[e + 1] += sh.tile_start[e];
    sh.total_tiles = sh.tile_start[E];
    if (sh.seg[E] > a.rows || sh.bad_segment) {  // rows the buffers do not hold: do nothing
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
  const Maps maps{&mapA0, &mapA1, &mapB0, &mapB1};
  // main-loop waits: the workspace's limit; a wait that gives up also stops the other CTA
  const uint64_t wait_ns = wait_limit_ns(a.wait_ctl);
  const uint32_t peer_abort = map_to_cta(smem_addr(&sh.abort_flag), rank ^ 1u);

  static_assert(MODE == kGemmUp || !AG, "the row gather feeds the up GEMM only");
  if (AG && warp == 0) {
    // ================= TMA producer, row gather (the whole warp): A rows are
    // the tokens' rows of xg = x * gamma [T, d] (mapA0, one-row box), row p
    // of the tile being token perm[p] / k.  Lane l gathers the CTA's rows
    // 4l .. 4l+3 with one four-row gather per K block; lane 0 waits for the
    // stage, arms the leader's barrier and loads the stage's B.
    const uint32_t full_leader0 = map_to_cta(smem_addr(&sh.full[0]), 0);
    const uint32_t tx_pair = 2u * (kABytes + static_cast<uint32_t>(a.bn / 2) * BK * 2u);
    const int kept = sh.seg[E];
    uint32_t it = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < total; tile += npairs) {
      const TileCoord c = decode_tile(sh, E, tile);
      const int o_e = a.ffn.off[c.e];
      const int kblocks = sh.k_blocks[c.e];
      // rows past the last kept row (their results are discarded) read token 0
      const int p0 = sh.seg[c.e] + c.mt * BM + static_cast<int>(rank) * BM_CTA + 4 * lane;
      int tok[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int asg = p0 + j < kept ? a.perm[p0 + j] : -1;
        tok[j] = asg >= 0 ? asg / a.k : 0;
      }
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        int got = 1;
        if (lane == 0)
          got = mbar_wait(&sh.empty[s], ph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, false, peer_abort)
                    ? 1 : 0;
        if (!__shfl_sync(0xFFFFFFFFu, got, 0)) {
          ok = false;
          break;
        }
        uint8_t* sA = smem + s * kStageBytes;
        const uint32_t bar = full_leader0 + static_cast<uint32_t>(s) * 8u;
        if (lane == 0) {
          if (rank == 0) mbar_arrive_expect_tx(&sh.full[s], tx_pair);
          // leader: 128 columns of W1; peer: the same 128 columns of W3 (MN-major)
          const CUtensorMap* mB = rank == 0 ? maps.b0 : maps.b1;
          const int n0 = o_e + c.nt * kBlockN;
          tma_load_2d_pair(sA + kABytes, mB, bar, n0, kb * BK);
          tma_load_2d_pair(sA + kABytes + kAtomBytes, mB, bar, n0 + 64, kb * BK);
        }
        tma_gather4_pair(sA + lane * 4 * 128, maps.a0, bar, kb * BK, tok[0], tok[1], tok[2], tok[3]);
      }
    }
    // no copy into either CTA is in flight when it exits, whatever stopped the loop
    if (lane == 0) pair_producer_drain<kStages>(sh.pd, sh.full, it, rank, tx_pair / 2u, a.err);
  } else if (warp == 0) {
    // ================= TMA producer (one lane per CTA)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to_cta(smem_addr(&sh.full[0]), 0);
      const uint32_t tx_pair = 2u * (kABytes + static_cast<uint32_t>(a.bn / 2) * BK * 2u);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int o_e = a.ffn.off[c.e];
        const int f = a.ffn.off[c.e + 1] - o_e;
        const int kblocks = sh.k_blocks[c.e];
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&sh.empty[s], ph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, false,
                         peer_abort)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + s * kStageBytes;
          const uint32_t bar = full_leader0 + static_cast<uint32_t>(s) * 8u;
          if (rank == 0) mbar_arrive_expect_tx(&sh.full[s], tx_pair);
          issue_loads<MODE>(maps, c, kb, sA, sA + kABytes, bar, sh.seg[c.e], o_e, f, rank, a.bn);
        }
      }
      // no copy into either CTA is in flight when it exits, whatever stopped the loop
      pair_producer_drain<kStages>(sh.pd, sh.full, it, rank, tx_pair / 2u, a.err);
    }
  } else if (warp == 1) {
    // ================= MMA issuer (leader CTA, one lane)
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(BM, a.bn, Traits<MODE>::b_mn ? 1u : 0u, Traits<MODE>::a_mn ? 1u : 0u);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs, ++tcount) {
        const TileCoord c = decode_tile(sh, E, tile);
        const int kblocks = sh.k_blocks[c.e];
        const uint32_t buf = tcount & 1u;
        const uint32_t aph = (tcount >> 1) & 1u;
        // both CTAs' epilogues release the buffer (the peer's arrival is remote)
        if (!mbar_wait(&sh.tempty[buf], aph ^ 1u, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, true,
                       peer_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kAccCols;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&sh.full[s], ph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, false, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aA = smem_addr(smem + s * kStageBytes);
          const uint32_t aB = aA + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = Traits<MODE>::a_mn ? smem_desc_sw128(aA + kk * 2048, kAtomBytes, 1024)
                                                      : smem_desc_sw128(aA + kk * 32, 16, 1024);
            const uint64_t bdesc = Traits<MODE>::b_mn ? smem_desc_sw128(aB + kk * 2048, kAtomBytes, 1024)
                                                      : smem_desc_sw128(aB + kk * 32, 16, 1024);
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
    // ================= epilogue (warps 2 .. 1 + EPI): a warp reads TMEM lane quarter
    // warp % 4; with 8 warps the second four take the second half of the columns
    static_assert(EPI == 4 || MODE == kGemmUp || MODE == kGemmDown, "8 epilogue warps: up and down only");
    const int q = warp & 3;
    const int w = warp - 2;
    const int bpw = kEpiBytes / EPI / kEpiBoxBytes;  // staging boxes of this warp
    uint8_t* my_boxes = epi_boxes + w * (kEpiBytes / EPI);
    int c_lo = 0, c_hi = MODE == kGemmUp ? kBlockN : a.bn;
    if (EPI == 8) {
      const int span = c_hi / 2;
      c_lo = (w >> 2) * span;
      c_hi = c_lo + span;
    }
    const uint32_t tempty_leader0 = map_to_cta(smem_addr(&sh.tempty[0]), 0);
    uint32_t tcount = 0, eit = 0;
    for (int tile = pair; tile < total; tile += npairs, ++tcount) {
      const TileCoord c = decode_tile(sh, E, tile);
      const uint32_t buf = tcount & 1u;
      const uint32_t aph = (tcount >> 1) & 1u;
      RowPre pre{-1, 0.f};
      if (Traits<MODE>::row_tiles && MODE != kGemmBwdH) pre = row_pre<MODE>(a, sh, c, q, lane, rank);
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait(&sh.tfull[buf], aph, abort_flag, a.err, MOE_DEVERR_TIMEOUT, wait_ns, false, peer_abort);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kAccCols;
      if (MODE == kGemmBwdH)
        ok = epilogue_dsh(a, sh, em, c, taddr, q, lane, rank, my_boxes, sh.ebar[w], eit, abort_flag, wait_ns,
                          peer_abort);
      else if (Traits<MODE>::row_tiles)
        epilogue_rows<MODE>(a, sh, em, c, taddr, q, lane, rank, my_boxes, bpw, eit, c_lo, c_hi, pre);
      else
        epilogue_wgrad<MODE>(a, sh, em, c, taddr, q, lane, rank, my_boxes, eit);
      tc_fence_before();
      __syncwarp();
      if (!ok) break;
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + buf * 8u);
    }
    // the staged stores have completed before the CTA's shared memory goes away
    if (lane == 0) bulk_wait_group0();
  }

  // ---- teardown: neither CTA leaves while its pair may still touch its memory
  griddep_launch_dependents();  // the next kernel may launch and set up meanwhile
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

template <int MODE, int EPI = 4, int AG = 0>
cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<MODE, EPI, AG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

}  // namespace

size_t grouped_gemm_smem_bytes() { return kSmemBytes; }

cudaError_t prepare_grouped_gemm() {
  cudaError_t e = set_smem_attr<kGemmUp>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmDown>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmBwdH>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmBwdX>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmWgradX>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmWgradH>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmUp, 8>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmDown, 8>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmUp, 4, 1>();
  if (e == cudaSuccess) e = set_smem_attr<kGemmUp, 8, 1>();
  return e;
}

// All modes share the launch shape (192 threads, the same shared memory), so
// the co-resident cluster count of one instantiation holds for all.
int grouped_gemm_max_grid(int num_sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_kernel<kGemmUp, 4>, &cfg) != cudaSuccess ||
      clusters <= 0) {
    cudaGetLastError();
    return num_sms & ~1;
  }
  const int grid = 2 * clusters;
  return grid < (num_sms & ~1) ? grid : (num_sms & ~1);
}

cudaError_t launch_grouped_gemm(const GemmArgs& a, const CUtensorMap& mapA0, const CUtensorMap& mapA1,
                                const CUtensorMap& mapB0, const CUtensorMap& mapB1, int grid,
                                cudaStream_t s, const EpiMaps* em_opt) {
  if (a.bn != 128 && a.bn != 256) return cudaErrorInvalidValue;
  if (a.mode == kGemmBwdH && em_opt == nullptr) return cudaErrorInvalidValue;
  static const EpiMaps kNoMaps{};
  const EpiMaps& em = em_opt != nullptr ? *em_opt : kNoMaps;
  if (a.epi8 && a.mode != kGemmUp && a.mode != kGemmDown) return cudaErrorInvalidValue;
  if (a.gather && a.mode != kGemmUp) return cudaErrorInvalidValue;
  GemmArgs ga = a;
  ga.staged = em_opt != nullptr ? 1 : 0;
  cudaError_t e = cudaSuccess;
  switch (a.mode) {
    case kGemmUp:
      if (ga.gather && ga.epi8)
        e = launch_pdl(grouped_gemm_kernel<kGemmUp, 8, 1>, dim3(grid), dim3(threads_of(8)), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      else if (ga.gather)
        e = launch_pdl(grouped_gemm_kernel<kGemmUp, 4, 1>, dim3(grid), dim3(kThreads), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      else if (ga.epi8)
        e = launch_pdl(grouped_gemm_kernel<kGemmUp, 8>, dim3(grid), dim3(threads_of(8)), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      else
        e = launch_pdl(grouped_gemm_kernel<kGemmUp, 4>, dim3(grid), dim3(kThreads), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      break;
    case kGemmDown:
      if (ga.epi8)
        e = launch_pdl(grouped_gemm_kernel<kGemmDown, 8>, dim3(grid), dim3(threads_of(8)), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      else
        e = launch_pdl(grouped_gemm_kernel<kGemmDown, 4>, dim3(grid), dim3(kThreads), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      break;
    case kGemmBwdH:
      e = launch_pdl(grouped_gemm_kernel<kGemmBwdH, 4>, dim3(grid), dim3(kThreads), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      break;
    case kGemmBwdX:
      e = launch_pdl(grouped_gemm_kernel<kGemmBwdX, 4>, dim3(grid), dim3(kThreads), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      break;
    case kGemmWgradX:
      e = launch_pdl(grouped_gemm_kernel<kGemmWgradX, 4>, dim3(grid), dim3(kThreads), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      break;
    case kGemmWgradH:
      e = launch_pdl(grouped_gemm_kernel<kGemmWgradH, 4>, dim3(grid), dim3(kThreads), kSmemBytes, s, mapA0, mapA1, mapB0, mapB1, ga, em);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return e;
}

}  // namespace moe
