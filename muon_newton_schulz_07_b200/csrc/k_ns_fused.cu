// Every Newton-Schulz iteration of a parameter set in one persistent launch (sm_100a).
//
// The orthogonalisation the pages name for Muon's matrix parameters (aiproducthub
// "开发者千美元训3.8B模型 击败GPT-2", 影响 paragraph) is k rounds of
//   Gram    A  = s X X^T             (s = 1/(||U||+eps)^2 in the first round)
//   Poly    B' = a I + b A + c A A
//   Update  X  = s B' X              (s = 1/(||U||+eps) in the first round)
// The staged schedule (k_ns_gemm_tc.cu) launches each of the 3k stages separately; between two
// launches the machine drains and refills, which costs most for sets of small matrices (the
// GPT-2-small set, m = 768: each stage is only tens of microseconds of tensor work).  Here one
// launch runs all 3k stages.  The tiles of all stages form one list, stage after stage, dealt
// round-robin to the CTA pairs; a pair only waits for the stage its next tile reads, and only
// for that tile's own matrix:
//   * every epilogue warp that has stored its part of a tile (its TMA stores complete) adds 1 to
//     a completion counter of (stage, matrix) in the workspace (release);
//   * before loading a tile's operands, the producer of each CTA waits (acquire, bounded) until
//     the counter of the stage it reads has every arrival of that matrix;
//   * the polynomial's epilogue reads A itself (b A + a I), so it waits for the same counter and
//     then loads its chunks of A by TMA (through L2, never the non-coherent L1).
// A stage that waits for every tile of its matrix's previous stage also orders all
// write-after-read reuse of the buffers (A, B', the two X buffers).  Since a pair works through
// its tiles in list order and a tile only waits for tiles earlier in the list, the earliest
// unfinished tile can always proceed: with every pair resident (the grid never exceeds the
// clusters that fit at once) the launch cannot deadlock, and every wait is bounded anyway.
//
// The per-tile machinery is that of the staged kernel (CTA pairs with tcgen05.mma.cta_group::2,
// TMA operand ring without multicast, upper blocks only for the symmetric A and B', MN-major
// reads of the transposed blocks, eight epilogue warps, fused parameter write in the last
// Update), with the stage a run-time property of the tile.  Update tiles may be 256 x 512
// (when every group's padded width allows it); TMEM holds two 256-column accumulator slots:
// a 256-wide tile takes one slot (alternating), a 512-wide tile takes both, and its epilogue
// drains the first half, hands that slot back, then drains the second, while the MMA issuer
// already accumulates the next tile's first k slices into the freed half.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <vector>

#include "muon_device.cuh"
#include "muon_internal.h"

namespace muon {
namespace {

constexpr int BM = kTcBM, BN = kTcBN, BK = kTcBK;
constexpr int TILE = 256;
constexpr uint32_t A_STAGE = BM * BK * 2;           // 16 KB: this CTA's 128 rows of A
constexpr uint32_t B_STAGE = (BN / 2) * BK * 2;     // 16 KB: this CTA's half of one 256-column B tile
constexpr uint32_t TMEM_COLS = 512;                 // two 256-column accumulator slots
constexpr int EPI_WARPS = kTcEpiWarps;
constexpr int F32_PITCH = 36;                        // staged fp32 row: 32 + 4 pad
constexpr uint32_t EPI_OUT_BYTES = 2048;
constexpr uint32_t EPI_AUX_BYTES = 2048;              // one 32 x 32 bf16 chunk of A (64B swizzle)
constexpr uint32_t EPI_F32_BYTES = 32 * F32_PITCH * 4;
constexpr uint32_t BAR_BYTES = 256;

// The operand ring: stages of 48 KB (three) when the list holds 512-wide tiles, else stages of
// 32 KB (five), after which come the epilogue's store tiles and A chunks and the barriers.
template <bool WR>
struct FLayout {
  static constexpr int NST = WR ? 3 : 5;
  static constexpr uint32_t SB = A_STAGE + (WR ? 2 : 1) * B_STAGE;
  // Each epilogue warp owns one 8 KB block: its two store tiles, then its two A chunks.  The
  // fp32 staging of the fused parameter write overlays the warp's own block only (a warp on a
  // parameter-writing tile has no store or A load of its own in flight), never another warp's:
  // the warps of a pair drift apart by up to two tiles, and a neighbour may still be reading
  // its A chunks of an earlier polynomial tile.
  static constexpr uint32_t EPI_OFFSET = NST * SB;
  static constexpr uint32_t EPI_WARP_BYTES = 2 * EPI_OUT_BYTES + 2 * EPI_AUX_BYTES;
  static constexpr uint32_t BAR_OFFSET = EPI_OFFSET + EPI_WARPS * EPI_WARP_BYTES;
  static constexpr size_t SMEM_BYTES = 1024 + BAR_OFFSET + BAR_BYTES;
  static_assert(EPI_F32_BYTES <= EPI_WARP_BYTES, "fp32 staging must fit the warp's own block");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(2 * NST + 5 + 2 * EPI_WARPS <= BAR_BYTES / 8, "barriers must fit their region");
};
constexpr unsigned int ARRIVALS_PER_TILE = 2 * EPI_WARPS;   // epilogue warps of both CTAs
static_assert(sizeof(NsParams) <= 32764, "kernel parameters are limited to 32764 bytes");

struct FTile {
  int it, kind, g, mat, row0, col0, tw;
  bool last;
};

__host__ __device__ __forceinline__ FTile decode(const NsParams& p, int t) {
  FTile f;
  int it = t / p.tiles_iter;
  if (it > p.k - 1) it = p.k - 1;  // the last iteration may hold more tiles (256-wide Update)
  const int r = t - it * p.tiles_iter;
  const int L = (it == p.k - 1) ? 1 : 0;
  int kind = 0;
  while (kind < 2 && r >= p.begin[L][kind + 1][0]) ++kind;
  int g = 0;
  while (g + 1 < p.ngroups && r >= p.begin[L][kind][g + 1]) ++g;
  const NsGroup& G = p.g[g];
  const int local = r - p.begin[L][kind][g];
  const int T = G.tdim;
  f.it = it;
  f.kind = kind;
  f.g = g;
  f.last = L != 0;
  if (kind == kUpdate) {
    f.tw = p.upd_tw[L];
    const int tc = G.np / f.tw;
    const int tpm = T * tc;
    f.mat = local / tpm;
    const int q = local - f.mat * tpm;
    const int tm = q / tc;
    f.row0 = tm * TILE;
    f.col0 = (q - tm * tc) * f.tw;
  } else if (p.sym_wide) {
    // block row I of the upper triangle holds blocks J = I .. T-1, taken two at a time
    // (256 x 512 tiles) with a 256-wide tile for an odd one out at the end of the row
    const int tpm = sym_tiles(T, true);
    f.mat = local / tpm;
    int q = local - f.mat * tpm, I = 0;
    while (q >= (T - I + 1) / 2) {
      q -= (T - I + 1) / 2;
      ++I;
    }
    const int J = I + 2 * q;
    f.row0 = I * TILE;
    f.col0 = J * TILE;
    f.tw = (J + 1 < T) ? 2 * TILE : TILE;
  } else {
    // upper-triangle block (I, J), I <= J, row-major over the triangle
    const int tpm = sym_tiles(T, false);
    f.mat = local / tpm;
    int q = local - f.mat * tpm, I = 0;
    while (q >= T - I) {
      q -= T - I;
      ++I;
    }
    f.row0 = I * TILE;
    f.col0 = (I + q) * TILE;
    f.tw = TILE;
  }
  return f;
}

// Index of the completion counter of (stage s, matrix of f).
__host__ __device__ __forceinline__ size_t counter_index(const NsParams& p, int s, const FTile& f) {
  return static_cast<size_t>(s) * p.nslots + p.g[f.g].scal_base + f.mat;
}
__device__ __forceinline__ unsigned int* counter(const NsParams& p, int s, const FTile& f) {
  return p.deps + counter_index(p, s, f);
}

// The stage a tile reads (the stage index and the tiles per matrix that mean "complete");
// false for the first Gram, which reads the momentum kernel's X0 (an earlier launch).
__host__ __device__ __forceinline__ bool dependency_stage(const NsParams& p, const FTile& f, int* stage,
                                                          unsigned int* tiles) {
  const NsGroup& G = p.g[f.g];
  const int T = G.tdim;
  if (f.kind == kGram) {
    if (f.it == 0) return false;
    *stage = 3 * (f.it - 1) + kUpdate;
    *tiles = static_cast<unsigned int>(T * (G.np / p.upd_tw[0]));  // that iteration is not the last
  } else {
    *stage = 3 * f.it + f.kind - 1;
    *tiles = static_cast<unsigned int>(sym_tiles(T, p.sym_wide != 0));
  }
  return true;
}
__device__ __forceinline__ bool dependency(const NsParams& p, const FTile& f, const unsigned int** ctr,
                                           unsigned int* target) {
  int s;
  unsigned int tiles;
  if (!dependency_stage(p, f, &s, &tiles)) return false;
  *ctr = counter(p, s, f);
  *target = tiles * ARRIVALS_PER_TILE;
  return true;
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

// Issue the four K = 16 MMAs of one 64-deep k slice into the 256 columns at d_tmem.
__device__ __forceinline__ void mma_slice(uint32_t d_tmem, uint32_t sa, uint32_t sb, bool mna, bool mnb,
                                          bool first) {
  const uint32_t idesc = idesc_bf16_f32(2 * BM, BN, mna ? 1 : 0, mnb ? 1 : 0);
  // K-major: 16 k per step = 32 bytes along the swizzled row; MN-major: 16 k rows = 2 KB, the
  // two 64-wide M/N chunks 8 KB apart.
  const uint64_t adesc0 = mna ? smem_desc_sw128(sa, 8192, 1024) : smem_desc_sw128(sa, 16, 1024);
  const uint64_t bdesc0 = mnb ? smem_desc_sw128(sb, 8192, 1024) : smem_desc_sw128(sb, 16, 1024);
  const uint64_t astep = mna ? (2048u >> 4) : (32u >> 4);
  const uint64_t bstep = mnb ? (2048u >> 4) : (32u >> 4);
#pragma unroll
  for (int j = 0; j < BK / 16; ++j)
    tc_mma_bf16_pair(d_tmem, adesc0 + astep * j, bdesc0 + bstep * j, idesc, (!first || j != 0) ? 1u : 0u);
}

template <bool WR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
    ns_fused_kernel(const __grid_constant__ NsParams p) {
  constexpr int NST = FLayout<WR>::NST;
  constexpr uint32_t SB = FLayout<WR>::SB;
  constexpr uint32_t EPI_OFFSET = FLayout<WR>::EPI_OFFSET, EPI_WARP_BYTES = FLayout<WR>::EPI_WARP_BYTES,
                     BAR_OFFSET = FLayout<WR>::BAR_OFFSET;
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
      mbar_init(accf_bar(a), 1);                    // one multicast commit
      mbar_init(acce_bar(a), ARRIVALS_PER_TILE);    // every epilogue warp of both CTAs
    }
    for (int w = 0; w < EPI_WARPS; ++w)
      for (int j = 0; j < 2; ++j) mbar_init(aux_bar(w, j), 1);  // the warp's arrive.expect_tx
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.ngroups; ++g) {
      const NsGroup& G = p.g[g];
      for (int b = 0; b < 2; ++b) {
        tma_prefetch_desc(&G.x_row[b]);
        tma_prefetch_desc(&G.x_chk[b]);
      }
      tma_prefetch_desc(&G.a_row);
      tma_prefetch_desc(&G.a_chk);
      tma_prefetch_desc(&G.b_row);
      tma_prefetch_desc(&G.b_chk);
      tma_prefetch_desc(&G.a_st);
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
      bool ok = true;
      for (int t = p.t_begin + cl; t < p.t_end && ok; t += ncl) {
        const FTile f = decode(p, t);
        const NsGroup& G = p.g[f.g];
        const unsigned int* dep;
        unsigned int target;
        if (dependency(p, f, &dep, &target)) {
          if (!wait_counter_bounded(dep, target, tmo, abort_flag, p.status)) break;
          fence_proxy_async_global();  // the TMA loads below read what the acquire made visible
        }
        const int cur = f.it & 1;
        const CUtensorMap* ma_row = f.kind == kGram ? &G.x_row[cur] : f.kind == kPoly ? &G.a_row : &G.b_row;
        const CUtensorMap* ma_chk = f.kind == kGram ? &G.x_chk[cur] : f.kind == kPoly ? &G.a_chk : &G.b_chk;
        const CUtensorMap* mb_row = f.kind == kGram ? &G.x_row[cur] : f.kind == kPoly ? &G.a_row : &G.x_row[cur];
        const CUtensorMap* mb_chk = f.kind == kGram ? &G.x_chk[cur] : f.kind == kPoly ? &G.a_chk : &G.x_chk[cur];
        const bool sym_a = f.kind != kGram, sym_b = f.kind == kPoly, upd = f.kind == kUpdate;
        const int nsub = f.tw / TILE;
        if (!WR && nsub > 1) {  // a 512-wide tile does not fit this ring's stages (host plan error)
          record_status(p.status, kDevFault);
          *abort_flag = 1;
          break;
        }
        const uint32_t bytes = 2 * (A_STAGE + nsub * B_STAGE);
        const int kblocks = (f.kind == kGram ? G.np : G.mp) / BK;
        const int arow = f.row0 + static_cast<int>(rank) * BM;
        const int ia = f.row0 / TILE, jb = f.col0 / TILE;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, tmo, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), bytes);
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          const uint32_t sa = smem_base + stage * SB, sb = sa + A_STAGE;
          const int k0 = kb * BK;
          // blocks of A / B' below the diagonal are not stored: load the transposed block above
          const bool ta = sym_a && k0 / TILE < ia;
          const bool tb = sym_b && k0 / TILE < jb;
          if (!ta)
            tma_load_3d_pair(sa, ma_row, fb, k0, arow, f.mat);
          else
            tma_load_4d_pair(sa, ma_chk, fb, 0, k0, arow / 64, f.mat);
          for (int u = 0; u < nsub; ++u) {
            const int bcol = f.col0 + u * TILE + half;
            const bool tbu = tb || (sym_b && k0 / TILE < jb + u);
            if (!(upd || tbu))
              tma_load_3d_pair(sb + u * B_STAGE, mb_row, fb, k0, bcol, f.mat);
            else
              tma_load_4d_pair(sb + u * B_STAGE, mb_chk, fb, 0, k0, bcol / 64, f.mat);
          }
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Do not leave while loads or MMAs may still touch this CTA's shared memory.
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
      int stage = 0;
      uint32_t phase = 0;
      uint32_t uses[2] = {0u, 0u};  // completed uses of each accumulator slot
      int next_slot = 0;
      bool ok = true;
      for (int t = p.t_begin + cl; t < p.t_end && ok; t += ncl) {
        const FTile f = decode(p, t);
        const NsGroup& G = p.g[f.g];
        const int kblocks = (f.kind == kGram ? G.np : G.mp) / BK;
        const bool sym_a = f.kind != kGram, sym_b = f.kind == kPoly, upd = f.kind == kUpdate;
        const int ia = f.row0 / TILE, jb = f.col0 / TILE;
        auto major_a = [&](int kb) { return sym_a && (kb * BK) / TILE < ia; };
        // the B operand of half u covers block column jb + u
        auto major_b = [&](int kb, int u) { return upd || (sym_b && (kb * BK) / TILE < jb + u); };
        if (f.tw == TILE) {
          const int sl = next_slot;
          next_slot ^= 1;
          if (!mbar_wait_bounded(acce_bar(sl), (uses[sl] & 1u) ^ 1u, tmo, abort_flag, p.status)) break;
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(sl * TILE);
          for (int kb = 0; kb < kblocks; ++kb) {
            if (!mbar_wait_bounded(full_bar(stage), phase, tmo, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_base + stage * SB;
            mma_slice(d, sa, sa + A_STAGE, major_a(kb), major_b(kb, 0), kb == 0);
            tc_commit_pair_mc(empty_bar(stage), 0x3);  // frees the stage in both CTAs
            if (++stage == NST) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          tc_commit_pair_mc(accf_bar(sl), 0x3);
          ++uses[sl];
        } else {
          // 512-wide tile: slot 0 holds columns 0..255, slot 1 columns 256..511.  The first D
          // k slices go into the first half as soon as slot 0 is free; the second half joins
          // once the epilogue has handed slot 1 back.
          if (!mbar_wait_bounded(acce_bar(0), (uses[0] & 1u) ^ 1u, tmo, abort_flag, p.status)) break;
          tc_fence_after();
          const int D = kblocks < 2 ? kblocks : 2;   // at most NST - 1 stages held
          int held[2] = {0, 0};
          for (int kb = 0; kb < D; ++kb) {
            if (!mbar_wait_bounded(full_bar(stage), phase, tmo, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_base + stage * SB;
            mma_slice(tmem_base, sa, sa + A_STAGE, major_a(kb), major_b(kb, 0), kb == 0);
            held[kb] = stage;
            if (++stage == NST) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          if (!mbar_wait_bounded(acce_bar(1), (uses[1] & 1u) ^ 1u, tmo, abort_flag, p.status)) break;
          tc_fence_after();
          for (int kb = 0; kb < D; ++kb) {
            const uint32_t sa = smem_base + held[kb] * SB;
            mma_slice(tmem_base + TILE, sa, sa + A_STAGE + B_STAGE, major_a(kb), major_b(kb, 1), kb == 0);
            tc_commit_pair_mc(empty_bar(held[kb]), 0x3);
          }
          for (int kb = D; kb < kblocks; ++kb) {
            if (!mbar_wait_bounded(full_bar(stage), phase, tmo, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_base + stage * SB;
            mma_slice(tmem_base, sa, sa + A_STAGE, major_a(kb), major_b(kb, 0), false);
            mma_slice(tmem_base + TILE, sa, sa + A_STAGE + B_STAGE, major_a(kb), major_b(kb, 1), false);
            tc_commit_pair_mc(empty_bar(stage), 0x3);
            if (++stage == NST) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          tc_commit_pair_mc(accf_bar(0), 0x3);
          tc_commit_pair_mc(accf_bar(1), 0x3);
          ++uses[0];
          ++uses[1];
          next_slot = 0;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Eight warps, two per TMEM lane quadrant; in each 256-column half of a tile a warp owns 32
    // rows and 128 columns (four 32 x 32 chunks).  Chunks go out as bf16 through a 64B-swizzled
    // staging tile and one TMA store each; the fused parameter write uses fp32 staging and
    // plain stores into the caller's W.
    const int e = warp - 2;                 // epilogue warp 0..7
    const int quad = warp & 3;              // TMEM lanes 32*quad .. 32*quad+31
    const int cbase = (e >> 2) * 128;       // this warp's first column within each half
    uint8_t* wblock = smem + EPI_OFFSET + e * EPI_WARP_BYTES;  // this warp's own epilogue block
    uint8_t* otile = wblock;
    const uint32_t otile_u32 = smem_u32(otile);
    const uint8_t* abuf = wblock + 2 * EPI_OUT_BYTES;  // this warp's two A chunks
    const uint32_t abuf_u32 = smem_u32(abuf);
    uint32_t naux = 0, nissued = 0;   // A chunks consumed / requested (their buffers alternate)
    float* st32 = reinterpret_cast<float*>(wblock);
    const int sub_r = lane >> 2, sub_c = (lane & 3) * 8;
    const int swz = (lane >> 1) & 3;  // 64-byte swizzle of this lane's staging row
    uint32_t uses[2] = {0u, 0u};
    int next_slot = 0;
    int nchunk = 0;                   // chunks stored so far (alternates the staging tiles)
    bool ok = true;
    for (int t = p.t_begin + cl; t < p.t_end && ok; t += ncl) {
      const FTile f = decode(p, t);
      const NsGroup& G = p.g[f.g];
      const int nsub = f.tw / TILE;
      const bool fw = p.fuse_write != 0 && f.kind == kUpdate && f.last;
      const bool aux = f.kind == kPoly;   // the polynomial's b A + a I reads A
      const CUtensorMap* out_map =
          f.kind == kGram ? &G.a_st : f.kind == kPoly ? &G.b_st : &G.x_st[(f.it + 1) & 1];
      const int gr0 = f.row0 + static_cast<int>(rank) * BM + quad * 32;  // first row of this warp
      const int gr = gr0 + lane;
      __nv_bfloat16* W = nullptr;
      float cw = 0.0f;
      bool tr = false;
      int ldw = 0;
      if (fw) {
        const int slot = G.scal_base + f.mat;
        W = static_cast<__nv_bfloat16*>(p.wptr[slot]);
        cw = p.wcoef[slot];
        tr = p.wtrans[slot] != 0;
        ldw = tr ? G.m_real : G.n_real;
      }
      const bool wread = fw && p.w_decay != 0.0f && gr0 < G.m_real;
      if (fw) {
        // the fp32 staging overlays this warp's store tiles: no store of its may still read them
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      auto woff = [&](int gc, int rr) -> size_t {
        return tr ? static_cast<size_t>(gc + rr) * ldw + gr0 + sub_c : static_cast<size_t>(gr0 + rr) * ldw + gc + sub_c;
      };
      // column (within the tile) of chunk c of half h for this warp
      auto chunk_col = [&](int h, int c) { return h * TILE + cbase + c * 32; };
      const int nchunks = 4 * nsub;     // this warp's chunks of the tile, j = 4 h + c
      auto aux_issue = [&](int j) {     // lane 0: chunk j of this warp into buffer (naux + j) & 1
        const uint32_t n = naux + static_cast<uint32_t>(j);
        ++nissued;
        mbar_arrive_expect_tx(aux_bar(e, n & 1), EPI_AUX_BYTES);
        tma_load_3d(abuf_u32 + (n & 1) * EPI_AUX_BYTES, &G.a_st, aux_bar(e, n & 1), f.col0 + chunk_col(j >> 2, j & 3),
                    gr0, f.mat);
      };
      if (aux) {
        // A is this round's Gram output, written by other pairs: wait for it as the producer
        // does, then fetch the first two chunks by TMA
        const unsigned int* dep;
        unsigned int target;
        bool dok = true;
        if (lane == 0) {
          if (dependency(p, f, &dep, &target)) dok = wait_counter_bounded(dep, target, tmo, abort_flag, p.status);
          if (dok) {
            fence_proxy_async_global();
            aux_issue(0);
            aux_issue(1);
          }
        }
        ok = __shfl_sync(0xffffffffu, dok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      uint4 pf[4];
      auto pre_load = [&](int colw, uint4 (&dst)[4]) {
        const int gc = f.col0 + colw;
        if (wread && gc < G.n_real) {
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = __ldcs(reinterpret_cast<const uint4*>(W + woff(gc, q * 8 + sub_r)));
        }
      };
      const bool has_pre = wread;
      if (has_pre) pre_load(chunk_col(0, 0), pf);
      int sl = 0;
      if (nsub == 1) {
        sl = next_slot;
        next_slot ^= 1;
        if (!mbar_wait_bounded(accf_bar(sl), uses[sl] & 1u, tmo, abort_flag, p.status)) break;
      } else {
        if (!mbar_wait_bounded(accf_bar(0), uses[0] & 1u, tmo, abort_flag, p.status)) break;
        if (!mbar_wait_bounded(accf_bar(1), uses[1] & 1u, tmo, abort_flag, p.status)) break;
      }
      tc_fence_after();
      float s = 1.0f;
      if (f.it == 0 && f.kind != kPoly) {
        const float al = p.scal[2 * (G.scal_base + f.mat) + 1];
        s = (f.kind == kGram) ? al * al : al;
      }
      const float c_acc = f.kind == kPoly ? p.c : 1.0f;
      const float c_aux = f.kind == kPoly ? p.b : 0.0f;
      const float cdiag = (f.kind == kPoly && gr < G.m_real) ? p.a : 0.0f;
      const uint32_t tlane = static_cast<uint32_t>(quad * 32) << 16;
      const uint32_t tcol0 = nsub == 1 ? static_cast<uint32_t>(sl * TILE) : 0u;
#pragma unroll 1
      for (int h = 0; h < nsub; ++h) {
        const int slot = nsub == 1 ? sl : h;
        const uint32_t acce_leader = map_to_rank(acce_bar(slot), 0);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int colw = chunk_col(h, c);
          const int gc0 = f.col0 + colw;
          float v[32];
          __syncwarp();
          tmem_ld_32cols(tmem_base + tlane + tcol0 + static_cast<uint32_t>(colw), v);
          if (c == 3) {
            // this warp's part of the slot has been read: hand it back to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acce_leader);
          }
          uint4 nx[4];
          if (has_pre) {
            if (c + 1 < 4)
              pre_load(chunk_col(h, c + 1), nx);
            else if (h + 1 < nsub)
              pre_load(chunk_col(h + 1, 0), nx);
          }
          if (fw) {
            // Last Update: write the parameters instead of X_k (no chunk straddles the padding:
            // real dimensions are multiples of 32), from X_k as its bf16 store would hold it, so
            // the write is exactly param_write_kernel's on the stored X_k.
            if (gr0 < G.m_real && gc0 < G.n_real) {
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
              __syncwarp();
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) pf[q] = nx[q];
            continue;
          }
          if (aux) {
            // this lane's row of the chunk of A (64-byte rows, 64-byte swizzle, as TMA wrote them)
            const int j = 4 * h + c;
            const uint32_t n = naux + static_cast<uint32_t>(j);
            if (!mbar_wait_bounded(aux_bar(e, n & 1), (n >> 1) & 1u, tmo, abort_flag, p.status)) {
              ok = false;
              break;
            }
            const uint8_t* arow = abuf + (n & 1) * EPI_AUX_BYTES + lane * 64;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float a8[8];
              unpack8(*reinterpret_cast<const uint4*>(arow + ((q ^ swz) << 4)), a8);
#pragma unroll
              for (int i = 0; i < 8; ++i) v[8 * q + i] = s * fmaf(c_acc, v[8 * q + i], c_aux * a8[i]);
            }
            // every lane has used its row: the buffer may take the chunk two ahead
            __syncwarp();
            if (lane == 0 && j + 2 < nchunks) {
              fence_async_smem();
              aux_issue(j + 2);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = s * c_acc * v[i];
          }
          if (gc0 == gr0) {
            // the chunk on the diagonal: the polynomial adds a on the real diagonal (B' = a I + ...)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (gc0 + i == gr) v[i] += cdiag;
          }
          // the store issued two chunks ago used this staging tile: wait until it has been read
          const uint32_t ob = (nchunk & 1) * EPI_OUT_BYTES;
          ++nchunk;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(otile + ob + lane * 64 + ((q ^ swz) << 4)) = pack8(v + 8 * q);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(out_map, otile_u32 + ob, gc0, gr0, f.mat);
            bulk_commit();
          }
        }
        if (!ok) break;
      }
      if (!ok) break;
      if (aux) naux += static_cast<uint32_t>(nchunks);
      if (nsub == 1) {
        ++uses[sl];
      } else {
        ++uses[0];
        ++uses[1];
        next_slot = 0;
      }
      // Publish this warp's part of the tile to the stages that read it (the last round's
      // Update has no reader inside this launch).
      if (!(f.kind == kUpdate && f.last)) {
        if (lane == 0) {
          bulk_wait_all();             // this warp's TMA stores of the tile are complete
          fence_proxy_async_global();  // ... and ordered before the release below
          red_release_gpu_add(counter(p, 3 * f.it + f.kind, f), 1u);
        }
        __syncwarp();
      }
    }
    // every TMA store of this warp has finished (its shared memory read, its global write)
    if (lane == 0) bulk_wait_all();
    // after an early exit, A chunks may still be on their way into this warp's buffers: wait
    // (bounded) for them before the CTA leaves
    if (lane == 0) {
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

}  // namespace

size_t fused_smem_bytes() { return FLayout<true>::SMEM_BYTES; }

long long check_fused_tiles(const NsParams& p) {
  // Walk the tile list with the kernel's own decoding: every tile in range, every stored block of
  // every (stage, matrix) covered exactly once, each stage's tiles all listed before any tile
  // that reads them (so the earliest unfinished tile never waits), and every wait's target equal
  // to the tiles the read stage actually has for that matrix.
  long long bad = 0;
  if (p.k < 1 || p.ngroups < 1 || p.ngroups > kTcMaxGroups || p.total_tiles < 1 || p.tiles_iter < 1) return 1;
  const int nst = 3 * p.k;
  std::vector<int> count(static_cast<size_t>(nst) * p.nslots, 0), last(count.size(), -1);
  std::vector<std::vector<unsigned char>> cover(count.size());
  for (int g = 0; g < p.ngroups; ++g) {
    const NsGroup& G = p.g[g];
    if (G.tdim * TILE != G.mp || G.mp < TILE || G.np < G.mp || G.np % TILE != 0) ++bad;
  }
  for (int t = 0; t < p.total_tiles; ++t) {
    const FTile f = decode(p, t);
    if (f.g < 0 || f.g >= p.ngroups || f.it < 0 || f.it >= p.k || f.kind < kGram || f.kind > kUpdate) {
      ++bad;
      continue;
    }
    const NsGroup& G = p.g[f.g];
    const int T = G.tdim;
    if (f.mat < 0 || f.mat >= G.cnt || f.row0 % TILE != 0 || f.col0 % TILE != 0 || f.row0 < 0 ||
        f.row0 + TILE > G.mp || (f.tw != TILE && f.tw != 2 * TILE)) {
      ++bad;
      continue;
    }
    const int width = f.kind == kUpdate ? G.np : G.mp;
    if (f.col0 + f.tw > width || (f.kind != kUpdate && f.col0 < f.row0)) {
      ++bad;
      continue;
    }
    if (f.kind == kUpdate && f.last && p.fuse_write && f.tw != TILE) ++bad;
    const size_t ci = counter_index(p, 3 * f.it + f.kind, f);
    if (ci >= count.size()) {
      ++bad;
      continue;
    }
    ++count[ci];
    last[ci] = t;
    std::vector<unsigned char>& cv = cover[ci];
    const int nb = (width / TILE) * T;
    if (cv.empty()) cv.assign(nb, 0);
    for (int c = f.col0; c < f.col0 + f.tw; c += TILE) ++cv[(f.row0 / TILE) * (width / TILE) + c / TILE];
    int s;
    unsigned int tiles;
    if (dependency_stage(p, f, &s, &tiles)) {
      const size_t di = counter_index(p, s, f);
      // the read stage must be complete, and listed entirely, before this tile
      if (di >= count.size() || count[di] != static_cast<int>(tiles) || last[di] >= t) ++bad;
    }
  }
  for (int g = 0; g < p.ngroups; ++g) {
    const NsGroup& G = p.g[g];
    const int T = G.tdim;
    for (int it = 0; it < p.k; ++it)
      for (int kind = kGram; kind <= kUpdate; ++kind)
        for (int m = 0; m < G.cnt; ++m) {
          const size_t ci = static_cast<size_t>(3 * it + kind) * p.nslots + G.scal_base + m;
          if (ci >= cover.size() || cover[ci].empty()) {
            ++bad;
            continue;
          }
          const int cols = (kind == kUpdate ? G.np : G.mp) / TILE;
          for (int I = 0; I < T; ++I)
            for (int J = 0; J < cols; ++J) {
              const int want = (kind == kUpdate || J >= I) ? 1 : 0;  // upper blocks only for A, B'
              if (cover[ci][I * cols + J] != want) ++bad;
            }
        }
  }
  return bad;
}

namespace {

template <bool WR>
cudaError_t launch_fused_kind(const NsParams& p, int num_sms, cudaStream_t s) {
  static std::atomic<unsigned long long> attr_set{0};
  static std::atomic<int> max_clusters[64];
  constexpr size_t smem = FLayout<WR>::SMEM_BYTES;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << dev;
  if ((attr_set.load() & bit) == 0) {
    e = cudaFuncSetAttribute(ns_fused_kernel<WR>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // Every pair must be resident at once (a tile may wait for a tile of any other pair): the
    // grid never exceeds the clusters of two that fit on the device together.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, ns_fused_kernel<WR>, &cfg);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    max_clusters[dev].store(n);
    attr_set.fetch_or(bit);
  }
  const int pairs = std::min({num_sms / 2, max_clusters[dev].load(), p.t_end - p.t_begin});
  ns_fused_kernel<WR><<<2 * pairs, kTcThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ns_fused(const NsParams& p, int num_sms, cudaStream_t s) {
  if (p.t_end <= p.t_begin) return cudaSuccess;
  const bool wide = p.upd_tw[0] > TILE || p.upd_tw[1] > TILE || p.sym_wide != 0;
  return wide ? launch_fused_kind<true>(p, num_sms, s) : launch_fused_kind<false>(p, num_sms, s);
}

}  // namespace muon
