// The Newton-Schulz products on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// One persistent kernel runs one stage of one Newton-Schulz iteration for every
// matrix of the parameter set (all shape groups in one launch):
//   Gram    A = s * X X^T          (s = 1/(||U||+eps)^2 on the first iteration)
//   Poly    B' = a I + b A + c A A (A symmetric, so A A = A A^T)
//   Update  X' = s * (B' X)        (s = 1/(||U||+eps) on the first iteration)
// which together are one step of the Newton-Schulz orthogonalisation the pages
// name for Muon's matrix parameters (aiproducthub "开发者千美元训3.8B模型 击败GPT-2",
// 影响 paragraph).  B' carries the a X term of the update (a X + B X =
// (a I + B) X), which also keeps the cancellation a + b s^2 + c s^4 inside one
// fp32 sum before rounding.
//
// CTA pairs.  The kernel runs as clusters of two CTAs (one per SM of a TPC).
// A pair computes one 256 x 256 output tile with tcgen05.mma.cta_group::2
// (M = 256, N = 256, K = 16): CTA r holds rows 128r..128r+127 of the A operand
// and half of the B operand (tile columns 128r..128r+127) in its own shared
// memory, and rows 128r..128r+127 of the fp32 accumulator in its TMEM.  Each
// CTA loads only its own halves (TMA, no multicast), so per k slice a CTA moves
// 32 KB for 128 x 256 x 64 multiply-adds, two thirds of what a single-CTA
// 128 x 256 tile needs.  The even CTA issues the MMAs; its commits are
// multicast to the barriers of both CTAs.
//
// Gram and Poly outputs are symmetric: only the 256 x 256 blocks on or above the
// diagonal are computed and stored (diagonal blocks in full).  Whoever needs a
// block below the diagonal (Poly reading A, Update reading B') TMA-loads the
// stored block above it and feeds it to the tensor core as an MN-major operand,
// so the lower halves of A and B' are never written or read.
//
// Wide Update tiles.  When every group's padded width is a multiple of 512, the
// Updates that do not write the parameters use 256 x 512 pair tiles: two N = 256
// MMAs per k step share each k slice of B', so 25 % fewer operand bytes cross from
// L2 per multiply-add, at the price of one 512-column accumulator (the epilogue
// of a tile no longer overlaps the main loop of the next).
//
// Roles in each CTA (320 threads, 576 for Poly; one CTA per SM,
// persistent over a static round-robin list of pair tiles):
//   warp 0      TMA producer, one TMA per operand tile and k slice (a 64 x 128
//               box for K-major tiles, a 4-D box of two 64-wide chunks for
//               MN-major ones, 128-byte swizzle) into a ring of as many stages
//               as shared memory holds (6 x 32 KB for Gram, 5 x 32 KB for Poly
//               and the 256-wide Update, 4 x 48 KB for 512-wide tiles); the even
//               CTA's full
//               barrier counts the bytes of both CTAs
//   warp 1      TMEM allocation (512 columns: two 256-column accumulators, so
//               the epilogue of one tile overlaps the main loop of the next, or
//               one 512-column accumulator for wide tiles); in the even CTA,
//               lane 0 issues the MMAs
//   warps 2..    epilogue: 8 warps, two per TMEM lane quadrant, each on half of the
//               tile's columns; Poly 16, four per quadrant, each on a quarter (its
//               epilogue reads A as well and its k loop is short): tcgen05.ld 32
//               columns at a time, the fp32
//               combination (Poly: c A A + b A + a I), bf16 pack into a
//               64B-swizzled 32 x 32 staging tile, one TMA store per chunk
//               (upper blocks only for Gram/Poly).  In the last Update the
//               epilogue writes the parameters directly:
//               W = (1 - lr wd) W - lr sqrt(max(1, r/c)) X_k, transposed back for
//               tall matrices, from X_k rounded to bf16 exactly as the separate
//               write kernel reads it from the workspace.
// Operand B of Update is X itself in its row-major layout, i.e. MN-major, and so
// is every transposed block of A or B'; the other operands are K-major.  The
// instruction descriptor's major bits are set per k slice.  All waits are
// bounded (see muon_device.cuh).
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "muon_device.cuh"
#include "muon_internal.h"

namespace muon {
namespace {

constexpr int BM = kTcBM, BN = kTcBN, BK = kTcBK;
constexpr int TILE = 256;                               // pair tile: 256 x 256
constexpr uint32_t A_STAGE = BM * BK * 2;               // 16 KB: this CTA's 128 rows of A
constexpr uint32_t B_STAGE = (BN / 2) * BK * 2;         // 16 KB: this CTA's half of B
constexpr uint32_t TMEM_COLS = 512;                     // 2 accumulators x 256 fp32 columns
constexpr uint32_t BAR_BYTES = 512;
constexpr int F32_PITCH = 36;                            // staged fp32 row: 32 + 4 pad (144 B, 16-B aligned)
constexpr uint32_t EPI_OUT_BYTES = 2048;
constexpr uint32_t EPI_AUX_BYTES = 2048;
constexpr uint32_t EPI_F32_BYTES = 32 * F32_PITCH * 4;
constexpr uint32_t SMEM_LIMIT = 232448;                 // 227 KB per CTA

// Shared memory of one stage's kernel: the operand ring, then per epilogue warp two 32 x 32 bf16
// store tiles (2 KB each, 64-byte swizzle).  Poly's epilogue loads each 32 x 32 chunk of its
// input A by TMA into the store tile that chunk's result will leave from (same swizzle); the
// fused parameter write of the last Update stages fp32 chunks in the epilogue region instead.
// The ring gets as many stages as fit (at most 6): 6 x 32 KB for Gram, 5 x 32 KB for Poly and
// the 256-wide Update, 4 x 48 KB for the 256 x 512 Update tiles (ring depths from 4 to 6
// measured the same).
template <int KIND, bool WIDE>
struct Layout {
  // Epilogue warps: 8 (two per TMEM lane quadrant), 16 for Poly (four per quadrant, each on a
  // quarter of the tile's columns), whose epilogue does the most work per multiply-add.
  static constexpr int EW = KIND == kPoly ? 2 * kTcEpiWarps : kTcEpiWarps;
  static constexpr int THREADS = 64 + 32 * EW;
  static constexpr int NSUB = WIDE ? 2 : 1;
  static constexpr uint32_t SB = A_STAGE + NSUB * B_STAGE;  // bytes of one stage in one CTA
  // Poly loads each chunk of its input A into the store tile the chunk's result leaves from.
  static constexpr uint32_t EPI = EW * 2 * EPI_OUT_BYTES;
  static constexpr uint32_t F32 = (KIND == kUpdate && !WIDE) ? EW * EPI_F32_BYTES : 0;
  static constexpr uint32_t EPI_REGION = EPI > F32 ? EPI : F32;
  static constexpr int FIT = static_cast<int>((SMEM_LIMIT - 1024 - BAR_BYTES - EPI_REGION) / SB);
  static constexpr int NST = FIT < 6 ? FIT : 6;
  static constexpr uint32_t EPI_OFFSET = NST * SB;          // 16 KB multiples: 1024-byte aligned
  static constexpr uint32_t EPI_AUX_OFFSET = EPI_OFFSET;   // shares the store tiles
  static_assert(EPI_AUX_BYTES == EPI_OUT_BYTES, "an A chunk and a result chunk share a tile");
  static constexpr uint32_t BAR_OFFSET = EPI_OFFSET + EPI_REGION;
  static constexpr size_t SMEM_BYTES = 1024 + BAR_OFFSET + BAR_BYTES;
  static_assert(NST >= 3, "at least three operand stages");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory per CTA");
  // barriers: full[NST], empty[NST], accf[2], acce[2], the TMEM slot word, two per epilogue warp
  static_assert((2 * NST + 5 + 2 * EW) * 8 <= BAR_BYTES, "barriers must fit their region");
};

struct Tile {
  int g, mat, row0, col0;
};

template <int KIND, int TW>
__device__ __forceinline__ Tile decode_tile(const TcParams& p, int t) {
  int g = 0;
  while (g + 1 < p.ngroups && p.g[g + 1].tile_begin <= t) ++g;
  const TcGroup& G = p.g[g];
  const int local = t - G.tile_begin;
  const int mat = local / G.tiles_per_mat;
  const int r = local - mat * G.tiles_per_mat;
  Tile ti;
  ti.g = g;
  ti.mat = mat;
  if (KIND == kUpdate) {
    const int tm = r / G.tdim;
    ti.row0 = tm * TILE;
    ti.col0 = (r - tm * G.tdim) * TW;
  } else {
    // upper-triangle tile q = (I, J), I <= J, row-major over the triangle
    int q = r, I = 0;
    while (q >= G.tdim - I) {
      q -= G.tdim - I;
      ++I;
    }
    ti.row0 = I * TILE;
    ti.col0 = (I + q) * TILE;
  }
  return ti;
}

__device__ __forceinline__ void unpack8(const uint4& q, float* v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  return q;
}

template <int KIND, bool WIDE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Layout<KIND, WIDE>::THREADS, 1)
    ns_gemm_tc_kernel(const __grid_constant__ TcParams p) {
  // WIDE (Update only): the pair tile is 256 x 512, two N = 256 MMAs per k step into one
  // 512-column accumulator, so every k slice of A feeds twice the columns.
  using LY = Layout<KIND, WIDE>;
  constexpr int EPI_WARPS = LY::EW;
  constexpr int NSUB = LY::NSUB;
  constexpr int TW = TILE * NSUB;                   // pair tile width
  constexpr int NST = LY::NST;
  constexpr uint32_t SB = LY::SB;                   // bytes of one stage in one CTA
  constexpr uint32_t EPI_OFFSET = LY::EPI_OFFSET, EPI_AUX_OFFSET = LY::EPI_AUX_OFFSET, BAR_OFFSET = LY::BAR_OFFSET;
  constexpr int NACC = WIDE ? 1 : 2;                 // accumulators in TMEM
  static_assert(!WIDE || KIND == kUpdate, "wide tiles are for the Update only");
  static_assert(NACC * TW <= TMEM_COLS, "accumulators must fit TMEM");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t smem_base = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFFSET);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (NST + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * NST + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * NST + 2 + a); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NST + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto aux_bar = [&](int w, int j) { return bar0 + 8u * (2 * NST + 5 + 2 * w + j); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();           // 0: issues the MMAs; 1: its peer
  const int cl = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full_bar(s), 1);   // the even CTA's arrive.expect_tx (bytes of both CTAs)
      mbar_init(empty_bar(s), 1);  // one multicast commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf_bar(a), 1);   // one multicast commit
      mbar_init(acce_bar(a), 2 * EPI_WARPS);   // one arrival per epilogue warp of both CTAs
    }
    for (int w = 0; w < EPI_WARPS; ++w)
      for (int j = 0; j < 2; ++j) mbar_init(aux_bar(w, j), 1);  // the warp's arrive.expect_tx
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.ngroups; ++g) {
      tma_prefetch_desc(&p.g[g].tm_a);
      tma_prefetch_desc(&p.g[g].tm_at);
      tma_prefetch_desc(&p.g[g].tm_b);
      tma_prefetch_desc(&p.g[g].tm_bt);
      if (KIND == kPoly) tma_prefetch_desc(&p.g[g].tm_aux);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_arrive_wait();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      const int half = static_cast<int>(rank) * (BN / 2);
      constexpr bool sym_a = KIND != kGram;         // A (Poly) and B' (Update) are stored as upper blocks
      constexpr bool sym_b = KIND == kPoly;
      constexpr bool ta_update_b = KIND == kUpdate;  // X is always read MN-major by Update
      for (int t = cl; t < p.total_tiles; t += ncl) {
        const Tile ti = decode_tile<KIND, TW>(p, t);
        const TcGroup& G = p.g[ti.g];
        const int arow = ti.row0 + static_cast<int>(rank) * BM;
        const int ia = ti.row0 / TILE, jb = ti.col0 / TILE;
        bool ok = true;
        for (int kb = 0; kb < G.kblocks; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, tmo, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * SB);
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          const uint32_t sa = smem_base + stage * SB, sb = sa + A_STAGE;
          const int k0 = kb * BK;
          // Blocks of A / B' below the diagonal are not stored: load the transposed block
          // above it instead (the MMA reads it MN-major).
          const bool ta = sym_a && k0 / TILE < ia;
          const bool tb = sym_b && k0 / TILE < jb;
          const bool mnb = ta_update_b || tb;
          // One TMA per operand tile: 128 rows x 64 k (K-major), or 64 k rows x two 64-wide
          // chunks of the M/N dimension (MN-major), 16 KB each.  A wide tile has two B
          // tiles, for tile columns [0, 256) and [256, 512); each CTA holds its half of both.
          if (!ta)
            tma_load_3d_pair(sa, &G.tm_a, fb, k0, arow, ti.mat);
          else
            tma_load_4d_pair(sa, &G.tm_at, fb, 0, k0, arow / 64, ti.mat);
#pragma unroll
          for (int u = 0; u < NSUB; ++u) {
            const int bcol = ti.col0 + u * TILE + half;
            if (!mnb)
              tma_load_3d_pair(sb + u * B_STAGE, &G.tm_b, fb, k0, bcol, ti.mat);
            else
              tma_load_4d_pair(sb + u * B_STAGE, &G.tm_bt, fb, 0, k0, bcol / 64, ti.mat);
          }
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // Do not leave while loads or MMAs may still touch this CTA's shared memory:
      // wait (bounded) until the last use of every stage has been released.
      for (int i = 0; i < NST; ++i) {
        if (*abort_flag) break;
        (void)mbar_wait_bounded(empty_bar(stage), phase ^ 1u, tmo, abort_flag, p.status);
        if (++stage == NST) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------- MMA issuer (even CTA)
      constexpr bool sym_a = KIND != kGram;
      constexpr bool sym_b = KIND == kPoly;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = cl; t < p.total_tiles && ok; t += ncl) {
        const Tile ti = decode_tile<KIND, TW>(p, t);
        const TcGroup& G = p.g[ti.g];
        if (!mbar_wait_bounded(acce_bar(acc), acc_phase ^ 1u, tmo, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * TW);
        const int ia = ti.row0 / TILE, jb = ti.col0 / TILE;
        for (int kb = 0; kb < G.kblocks; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, tmo, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * SB, sb = sa + A_STAGE;
          const int kk = kb * BK / TILE;
          const bool mna = sym_a && kk < ia;                        // transposed block of A / B'
          const bool mnb = (KIND == kUpdate) || (sym_b && kk < jb);
          const uint32_t idesc = idesc_bf16_f32(2 * BM, BN, mna ? 1 : 0, mnb ? 1 : 0);
          // K-major: 16 k per step = 32 bytes along the swizzled row; MN-major: 16 k rows
          // = 2 KB, with the two 64-wide M/N chunks 8 KB apart.  The start address sits
          // in the low bits of the descriptor (16-byte units), so a step is a plain add.
          const uint64_t adesc0 = mna ? smem_desc_sw128(sa, 8192, 1024) : smem_desc_sw128(sa, 16, 1024);
          const uint64_t bdesc0 = mnb ? smem_desc_sw128(sb, 8192, 1024) : smem_desc_sw128(sb, 16, 1024);
          const uint64_t astep = mna ? (2048u >> 4) : (32u >> 4);
          const uint64_t bstep = mnb ? (2048u >> 4) : (32u >> 4);
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
#pragma unroll
            for (int u = 0; u < NSUB; ++u)
              tc_mma_bf16_pair(d_tmem + u * TILE, adesc0 + astep * j, bdesc0 + ((u * B_STAGE) >> 4) + bstep * j, idesc,
                               (kb | j) != 0 ? 1u : 0u);
          tc_commit_pair_mc(empty_bar(stage), 0x3);  // frees the stage in both CTAs
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(accf_bar(acc), 0x3);  // accumulator ready for both epilogues
        if (++acc == NACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // EPI_WARPS warps, EPI_WARPS / 4 per TMEM lane quadrant: each owns 32 rows of the CTA's 128
    // and its share of the tile's columns, which it walks in 32 x 32 chunks.  A finished chunk is packed
    // to bf16 into one of the warp's two 32 x 32 staging tiles (64-byte rows, 64-byte
    // swizzle, so the row-per-lane writes are free of bank conflicts) and written to global
    // memory by one TMA store.  The fused parameter write goes through an fp32 staging tile
    // and plain stores instead, since W is the caller's memory.
    const int e = warp - 2;                 // epilogue warp 0 .. EPI_WARPS-1
    const int quad = warp & 3;              // TMEM lanes 32*quad .. 32*quad+31
    constexpr int NW = TW / (8 * EPI_WARPS);  // chunks per warp and tile (32 columns each)
    static_assert(KIND != kPoly || NW % 2 == 0, "A chunk naux + c and result chunk c share tile c & 1");
    const int ch0 = (e >> 2) * NW;          // this warp's first chunk
    uint8_t* otile = smem + EPI_OFFSET + e * 2 * EPI_OUT_BYTES;
    const uint32_t otile_u32 = smem_u32(otile);
    const uint8_t* abuf = smem + EPI_AUX_OFFSET + e * 2 * EPI_AUX_BYTES;  // = otile: A in, B' out
    const uint32_t abuf_u32 = smem_u32(abuf);
    float* st32 = reinterpret_cast<float*>(smem + EPI_OFFSET + e * EPI_F32_BYTES);
    const int sub_r = lane >> 2, sub_c = (lane & 3) * 8;
    const int swz = (lane >> 1) & 3;  // 64-byte swizzle of this lane's staging row
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t naux = 0;                // A chunks this warp has consumed (their buffers alternate)
    uint32_t nissued = 0;             // A chunks lane 0 has requested
    bool aux_ok = true;
    for (int t = cl; t < p.total_tiles && aux_ok; t += ncl) {
      const Tile ti = decode_tile<KIND, TW>(p, t);
      const TcGroup& G = p.g[ti.g];
      const bool aux = KIND == kPoly;   // the polynomial's b A + a I reads A
      const int gr0 = ti.row0 + static_cast<int>(rank) * BM + quad * 32;  // first row of this warp
      const int gr = gr0 + lane;
      // Fused parameter write (last Update): the caller's matrix of this tile.
      const bool fw = KIND == kUpdate && p.fuse_write != 0;
      __nv_bfloat16* W = nullptr;
      float cw = 0.0f;
      bool tr = false;
      int ldw = 0;
      if (fw) {
        const int slot = G.scal_base + ti.mat;
        W = static_cast<__nv_bfloat16*>(p.wptr[slot]);
        cw = p.wcoef[slot];
        tr = p.wtrans[slot] != 0;
        ldw = tr ? G.m_real : G.n_real;
      }
      const bool wread = fw && p.w_decay != 0.0f && gr0 < G.m_real;
      // element (row rr, 8 columns from sub_c) of the chunk at column gc in W's own layout
      auto woff = [&](int gc, int rr) -> size_t {
        return tr ? static_cast<size_t>(gc + rr) * ldw + gr0 + sub_c : static_cast<size_t>(gr0 + rr) * ldw + gc + sub_c;
      };
      // The auxiliary inputs do not depend on the accumulator, so they are fetched before
      // waiting for it: the polynomial's chunks of A by TMA into the warp's two A buffers (the
      // first two now, each later one as soon as the buffer two chunks back is read), the W of
      // the fused parameter write into registers one chunk ahead.
      auto aux_issue = [&](int c) {  // lane 0: chunk c of this warp into buffer (naux + c) & 1
        const uint32_t n = naux + static_cast<uint32_t>(c);
        ++nissued;
        mbar_arrive_expect_tx(aux_bar(e, n & 1), EPI_AUX_BYTES);
        tma_load_3d(abuf_u32 + (n & 1) * EPI_AUX_BYTES, &G.tm_aux, aux_bar(e, n & 1), ti.col0 + (ch0 + c) * 32, gr0,
                    ti.mat);
      };
      if (aux && lane == 0) {
        bulk_wait_read<0>();  // the previous tile's last stores have left both tiles
        aux_issue(0);
        if (NW > 1) aux_issue(1);
      }
      uint4 pf[4];
      auto pre_load = [&](int ch, uint4 (&dst)[4]) {
        const int gc = ti.col0 + ch * 32;
        if (wread && gc < G.n_real) {
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = __ldcs(reinterpret_cast<const uint4*>(W + woff(gc, q * 8 + sub_r)));
        }
      };
      const bool has_pre = wread && !WIDE;  // (the wide path loads W after reading the accumulator)
      if (has_pre) pre_load(ch0, pf);
      if (WIDE && wread && (lane & 3) == 0) {
        // The wide path writes W only after the accumulator is back: pull this warp's rows of
        // W for the whole tile into L2 now, while the tile's MMAs run (no registers held).
#pragma unroll 1
        for (int c = 0; c < NW; ++c) {
          const int gc = ti.col0 + (ch0 + c) * 32;
          if (gc < G.n_real) {
#pragma unroll
            for (int q = 0; q < 4; ++q) prefetch_l2(W + woff(gc, q * 8 + sub_r));
          }
        }
      }
      if (!mbar_wait_bounded(accf_bar(acc), acc_phase, tmo, abort_flag, p.status)) break;
      tc_fence_after();
      float s = 1.0f;
      if (p.use_scal) {
        const float al = p.scal[2 * (G.scal_base + ti.mat) + 1];
        s = (KIND == kGram) ? al * al : al;
      }
      const float cdiag = (KIND == kPoly && gr < G.m_real) ? p.c_diag : 0.0f;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * TW);
      const uint32_t acce_leader = map_to_rank(acce_bar(acc), 0);
      if constexpr (WIDE) {
        // One accumulator, so the MMA issuer waits for it: read this warp's whole part (32 rows
        // x 256 columns) into registers as bf16 (the X_k the workspace would hold), hand the
        // accumulator back, and only then stage and store the chunks.  (Chunk by chunk, the
        // stores of the first seven chunks would sit between the issuer and its next tile.)
        // When the launch writes the parameters, each chunk goes through a padded row-major
        // staging tile (read column-wise for tall parameters) into W = w_decay W + coef X_k, the
        // arithmetic of param_write_kernel on the same bf16 X_k.
        uint32_t pk[NW][16];
#pragma unroll
        for (int c = 0; c < NW; ++c) {
          float v[32];
          tmem_ld_32cols(taddr + (ch0 + c) * 32, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(s * p.c_acc * v[2 * i], s * p.c_acc * v[2 * i + 1]);
            pk[c][i] = *reinterpret_cast<const uint32_t*>(&h);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acce_leader);
        if (fw) {
          constexpr int PITCH = 80;  // bytes per staged row: 32 bf16 + 16 (16-byte aligned, conflict-free)
          static_assert(32 * PITCH <= 2 * EPI_OUT_BYTES, "the staging tile fits the warp's two store tiles");
          uint8_t* stg = otile;
#pragma unroll
          for (int c = 0; c < NW; ++c) {
            const int gc0 = ti.col0 + (ch0 + c) * 32;
            if (gr0 < G.m_real && gc0 < G.n_real) {  // the padding has no parameters
              uint4 w4[4];
              if (wread) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  w4[q] = __ldcs(reinterpret_cast<const uint4*>(W + woff(gc0, q * 8 + sub_r)));
              }
              __syncwarp();  // the previous chunk's staged rows have been read
              // row r of the staged tile = row r of this chunk of X_k
#pragma unroll
              for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(stg + lane * PITCH + q * 16) =
                    make_uint4(pk[c][4 * q], pk[c][4 * q + 1], pk[c][4 * q + 2], pk[c][4 * q + 3]);
              __syncwarp();
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int rr = q * 8 + sub_r;
                float x8[8], r8[8];
                if (!tr) {
                  unpack8(*reinterpret_cast<const uint4*>(stg + rr * PITCH + sub_c * 2), x8);
                } else {
                  // W row gc0 + rr, columns gr0 + sub_c .. +7: column rr of staged rows sub_c ..
#pragma unroll
                  for (int j = 0; j < 8; ++j)
                    x8[j] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(stg + (sub_c + j) * PITCH + rr * 2));
                }
                if (wread) {
                  float w8[8];
                  unpack8(w4[q], w8);
#pragma unroll
                  for (int i = 0; i < 8; ++i) r8[i] = fmaf(p.w_decay, w8[i], cw * x8[i]);
                } else {
#pragma unroll
                  for (int i = 0; i < 8; ++i) r8[i] = cw * x8[i];
                }
                __stcs(reinterpret_cast<uint4*>(W + woff(gc0, rr)), pack8(r8));
              }
            }
          }
        } else {
#pragma unroll
        for (int c = 0; c < NW; ++c) {
          const uint32_t ob = (c & 1) * EPI_OUT_BYTES;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(otile + ob + lane * 64 + ((q ^ swz) << 4)) =
                make_uint4(pk[c][4 * q], pk[c][4 * q + 1], pk[c][4 * q + 2], pk[c][4 * q + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&G.tm_out, otile_u32 + ob, ti.col0 + (ch0 + c) * 32, gr0, ti.mat);
            bulk_commit();
          }
        }
        }
      } else {
#pragma unroll 1
      for (int c = 0; c < NW; ++c) {
        const int ch = ch0 + c;
        const int gc0 = ti.col0 + ch * 32;
        float v[32];
        __syncwarp();
        tmem_ld_32cols(taddr + ch * 32, v);
        if (c == NW - 1) {
          // all of this warp's part of the accumulator has been read: tell the MMA issuer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(acce_leader);
        }
        uint4 nx[4];
        if (has_pre && c + 1 < NW) pre_load(ch + 1, nx);
        if (fw) {
          // Last Update: write the parameters instead of X_k.  Chunks in the zero padding
          // of the workspace have no parameters (real dimensions are multiples of 32).
          if (gr0 < G.m_real && gc0 < G.n_real) {
            // stage X_k = s * acc as its bf16 store would hold it (so the write is exactly
            // param_write_kernel's on the stored X_k), row-major or transposed for tall parameters
            if (!tr) {
#pragma unroll
              for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(st32 + lane * F32_PITCH + i) =
                    make_float4(bf16_round(s * v[i]), bf16_round(s * v[i + 1]), bf16_round(s * v[i + 2]),
                                bf16_round(s * v[i + 3]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) st32[i * F32_PITCH + lane] = bf16_round(s * v[i]);
            }
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int rr = q * 8 + sub_r;
              const float4 o0 = *reinterpret_cast<const float4*>(st32 + rr * F32_PITCH + sub_c);
              const float4 o1 = *reinterpret_cast<const float4*>(st32 + rr * F32_PITCH + sub_c + 4);
              float r8[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
              if (wread) {
                float w8[8];
                unpack8(pf[q], w8);
#pragma unroll
                for (int i = 0; i < 8; ++i) r8[i] = fmaf(p.w_decay, w8[i], cw * r8[i]);
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) r8[i] = cw * r8[i];
              }
              __stcs(reinterpret_cast<uint4*>(W + woff(gc0, rr)), pack8(r8));
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) pf[q] = nx[q];
          continue;
        }
        if (aux) {
          // this lane's row of the chunk of A (64-byte rows, 64-byte swizzle, as TMA wrote them)
          const uint32_t n = naux + static_cast<uint32_t>(c);
          if (!mbar_wait_bounded(aux_bar(e, n & 1), (n >> 1) & 1u, tmo, abort_flag, p.status)) {
            aux_ok = false;
            break;
          }
          const uint8_t* arow = abuf + (n & 1) * EPI_AUX_BYTES + lane * 64;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float a8[8];
            unpack8(*reinterpret_cast<const uint4*>(arow + ((q ^ swz) << 4)), a8);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[8 * q + i] = s * fmaf(p.c_acc, v[8 * q + i], p.c_aux * a8[i]);
          }
          __syncwarp();  // every lane has read its row of A: the tile takes the result next
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = s * p.c_acc * v[i];
        }
        if (gc0 == gr0) {
          // the chunk on the diagonal: Poly adds a on the real diagonal (B' = a I + ...)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (gc0 + i == gr) v[i] += cdiag;
        }
        // The store issued two chunks ago used this staging tile: wait until it has been read.
        const uint32_t ob = (c & 1) * EPI_OUT_BYTES;
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(otile + ob + lane * 64 + ((q ^ swz) << 4)) = pack8(v + 8 * q);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&G.tm_out, otile_u32 + ob, gc0, gr0, ti.mat);
          bulk_commit();
          if (aux && c + 2 < NW) {
            // the tile takes the chunk of A two ahead once this store has read it
            bulk_wait_read<0>();
            aux_issue(c + 2);
          }
        }
      }
      if (aux) naux += NW;  // (an early exit leaves naux behind nissued; see the drain below)
      }
      if (++acc == NACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // every TMA store of this warp has finished (its shared memory read, its global write)
    if (lane == 0) bulk_wait_all();
    // after an early exit, A chunks may still be on their way into this warp's buffers: wait
    // (bounded) for them before the CTA leaves
    if (KIND == kPoly && lane == 0) {
      for (uint32_t n = naux; n < nissued; ++n)
        (void)mbar_wait_bounded(aux_bar(e, n & 1), (n >> 1) & 1u, tmo, nullptr, p.status);
    }
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  cluster_arrive_wait();  // neither CTA frees TMEM or leaves while the pair may still use it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <int KIND, bool WIDE>
cudaError_t launch_kind(const TcParams& p, int grid, cudaStream_t s) {
  // The shared-memory limit is a property of the function on each device: set it once per device.
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if ((attr_set.load() & bit) == 0) {
    e = cudaFuncSetAttribute(ns_gemm_tc_kernel<KIND, WIDE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Layout<KIND, WIDE>::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  ns_gemm_tc_kernel<KIND, WIDE><<<grid, Layout<KIND, WIDE>::THREADS, Layout<KIND, WIDE>::SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t tc_smem_bytes() { return Layout<kUpdate, true>::SMEM_BYTES; }

cudaError_t launch_tc_gemm(const TcParams& p, int num_sms, cudaStream_t s) {
  if (p.total_tiles <= 0) return cudaSuccess;
  if (p.wide && p.kind != kUpdate) return cudaErrorInvalidValue;  // 256-wide only
  // one CTA pair per TPC, at most one pair per tile
  const int grid = 2 * std::min(num_sms / 2, p.total_tiles);
  if (p.kind == kGram) return launch_kind<kGram, false>(p, grid, s);
  if (p.kind == kPoly) return launch_kind<kPoly, false>(p, grid, s);
  if (p.wide) return launch_kind<kUpdate, true>(p, grid, s);
  return launch_kind<kUpdate, false>(p, grid, s);
}

}  // namespace muon
