// Newton-Schulz for small matrices: all k iterations of one matrix in one CTA pair.
//
// The orthogonalisation the pages name for Muon's matrix parameters (aiproducthub
// "开发者千美元训3.8B模型 击败GPT-2", 影响 paragraph) iterates A = X X^T, B = b A + c A A,
// X = a X + B X.  When every matrix of the set fits one 256 x 256 tile (max(rows, cols)
// <= 256, zero-padded to 256 x 256 in the workspace), the per-stage launches of the
// general path are mostly latency.  Here one CTA pair keeps the whole iteration on chip:
//
//   shared memory of CTA r (r = 0, 1):
//     XROW  64 KB  rows 128r..128r+127 of X, K-major (4 chunks of 64 columns), 128B swizzle:
//                  the A and B operand of the Gram product
//     XCOL  64 KB  columns 128r..128r+127 of X for all 256 rows, MN-major (4 blocks of 64
//                  rows, two 64-wide column chunks each), 128B swizzle: the B operand of
//                  the update
//     ABUF  64 KB  rows 128r.. of A (the operand of A A), then of B' = a I + b A + c A A
//                  (the A operand of the update), K-major
//   TMEM of CTA r (512 columns, rows 128r.. of each product):
//     columns   0..255  A, then X'
//     columns 256..511  A A
//
// Every product is one tcgen05.mma.cta_group::2 sequence (M = 256, N = 256, K = 256) issued
// by the even CTA: A and B' are symmetric, so A A = A A^T and each CTA's own rows serve as
// its half of the B operand.  After the update, each CTA writes its rows of X' into its own
// XROW and, through distributed shared memory, into the XCOL of the CTA that owns each
// column half.  The normalisation is folded into the first iteration (the Gram product
// scaled by 1/(||U||+eps)^2, the update by 1/(||U||+eps)), as in the general path; the
// result X_k goes to the workspace, where the parameter write reads it.
//
// All waits are bounded.  A CTA whose wait runs out records the timeout and stops its own
// work, but still takes every cluster barrier of the schedule, so its peer cannot hang.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "muon_device.cuh"
#include "muon_internal.h"

namespace muon {
namespace {

constexpr uint32_t XROW_OFF = 0;
constexpr uint32_t XCOL_OFF = 65536;
constexpr uint32_t ABUF_OFF = 131072;
constexpr uint32_t BAR_OFF = 196608;
constexpr uint32_t CHUNK = 16384;  // one 64-deep slice of a 128-row (or 128-column) operand
constexpr size_t SMEM_BYTES = 1024 + BAR_OFF + 64;
constexpr int THREADS = 256;        // 8 warps, two per TMEM lane quadrant

__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  return q;
}

// 32 values of row r (0..127), columns 32 ch .. 32 ch + 31, into a K-major 128-row operand.
__device__ __forceinline__ void put_kmajor(uint8_t* buf, int r, int ch, const float* v) {
  const int kc = ch >> 1, u0 = (ch & 1) * 4;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(buf + kc * CHUNK + r * 128 + (((u0 + q) ^ (r & 7)) << 4)) = pack8(v + 8 * q);
}

// Issue one 256 x 256 x 256 product into TMEM columns d_col (even CTA, one thread).
__device__ __forceinline__ void issue_product(uint32_t tmem, uint32_t d_col, uint32_t a_addr, bool a_mn,
                                              uint32_t b_addr, bool b_mn, uint32_t bar) {
  tc_fence_after();
  const uint32_t idesc = idesc_bf16_f32(256, 256, a_mn ? 1 : 0, b_mn ? 1 : 0);
#pragma unroll 1
  for (int kb = 0; kb < 4; ++kb) {
    // K-major: 16 k per step = 32 bytes along the swizzled row; MN-major: 16 k rows = 2 KB,
    // with the two 64-wide M/N chunks 8 KB apart.
    const uint64_t ad = a_mn ? smem_desc_sw128(a_addr + kb * CHUNK, 8192, 1024)
                             : smem_desc_sw128(a_addr + kb * CHUNK, 16, 1024);
    const uint64_t bd = b_mn ? smem_desc_sw128(b_addr + kb * CHUNK, 8192, 1024)
                             : smem_desc_sw128(b_addr + kb * CHUNK, 16, 1024);
    const uint64_t as = a_mn ? (2048u >> 4) : (32u >> 4), bs = b_mn ? (2048u >> 4) : (32u >> 4);
#pragma unroll
    for (int j = 0; j < 4; ++j) tc_mma_bf16_pair(tmem + d_col, ad + as * j, bd + bs * j, idesc, (kb | j) != 0 ? 1u : 0u);
  }
  tc_commit_pair_mc(bar, 0x3);  // both CTAs learn that the product is in TMEM
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    ns_small_kernel(const __grid_constant__ SmallParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  const uint32_t ld_bar = smem_u32(bars), mma_bar = smem_u32(bars + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int cl = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    mbar_init(ld_bar, 1);
    mbar_init(mma_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_arrive_wait();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;
  const bool issuer = rank == 0 && threadIdx.x == 32;

  const int quad = warp & 3;          // TMEM lanes 32*quad .. 32*quad+31
  const int half = warp >> 2;         // this warp's column half: chunks 4*half .. 4*half+3
  const int r = quad * 32 + lane;     // row within this CTA's 128
  const int gr = static_cast<int>(rank) * 128 + r;  // row within the 256 x 256 tile
  const uint32_t t_row = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  // The update's columns of this warp belong to the XCOL of CTA `half`.
  const uint32_t xcol_base = (static_cast<uint32_t>(half) == rank) ? sbase + XCOL_OFF
                                                                   : map_to_rank(sbase + XCOL_OFF, peer);
  const int kb_r = gr >> 6, rr = gr & 63;  // this row's place in an MN-major operand
  bool ok = true;
  uint32_t ld_par = 0, mma_par = 0;
  auto wait_product = [&]() {
    if (ok) ok = mbar_wait_bounded(mma_bar, mma_par, tmo, nullptr, p.status);
    mma_par ^= 1u;
    ok = __all_sync(0xffffffffu, ok);  // warp-uniform: the TMEM reads below are warp-wide
    tc_fence_after();
  };
  auto sync_pair = [&]() {
    tc_fence_before();
    cluster_arrive_wait();
  };

#pragma unroll 1
  for (int m = cl; m < p.total; m += ncl) {
    int g = 0;
    while (g + 1 < p.ngroups && p.g[g + 1].mat_begin <= m) ++g;
    const SmGroup& G = p.g[g];
    const int mat = m - G.mat_begin;
    const float alpha = p.scal[2 * (G.scal_base + mat) + 1];

    // X0: this CTA's rows (K-major) and columns (MN-major), each CTA from its own barrier.
    if (threadIdx.x == 0 && ok) {
      mbar_arrive_expect_tx(ld_bar, 8 * CHUNK);
#pragma unroll 1
      for (int kc = 0; kc < 4; ++kc) tma_load_3d(sbase + XROW_OFF + kc * CHUNK, &G.tm_row, ld_bar, kc * 64,
                                                 static_cast<int>(rank) * 128, mat);
#pragma unroll 1
      for (int kb = 0; kb < 4; ++kb) tma_load_4d(sbase + XCOL_OFF + kb * CHUNK, &G.tm_col, ld_bar, 0, kb * 64,
                                                 static_cast<int>(rank) * 2, mat);
    }
    if (ok) ok = mbar_wait_bounded(ld_bar, ld_par, tmo, nullptr, p.status);
    ld_par ^= 1u;
    ok = __all_sync(0xffffffffu, ok);
    sync_pair();  // both CTAs' operands are in place before the even CTA multiplies

#pragma unroll 1
    for (int it = 1; it <= p.k; ++it) {
      const bool first = it == 1, last = it == p.k;
      // ---------------------------------------------------------------- A = s X X^T
      if (issuer && ok) issue_product(tmem, 0, sbase + XROW_OFF, false, sbase + XROW_OFF, false, mma_bar);
      wait_product();
      const float sg = first ? alpha * alpha : 1.0f;
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int ch = half * 4 + c;
          float v[32];
          tmem_ld_32cols(t_row + ch * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= sg;
          put_kmajor(smem + ABUF_OFF, r, ch, v);
        }
      }
      fence_async_smem();
      sync_pair();
      // ---------------------------------------------------------------- B' = a I + b A + c A A
      if (issuer && ok) issue_product(tmem, 256, sbase + ABUF_OFF, false, sbase + ABUF_OFF, false, mma_bar);
      wait_product();
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int ch = half * 4 + c;
          float aa[32], av[32];
          tmem_ld_32cols(t_row + 256 + ch * 32, aa);
          tmem_ld_32cols(t_row + ch * 32, av);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            // b A uses the bf16 A that A A was formed from, so that B' is the polynomial of one
            // matrix (the rounded A); mixing the unrounded A in spoils the quintic's cancellation.
            const float ar = __bfloat162float(__float2bfloat16_rn(sg * av[i]));
            const int col = ch * 32 + i;
            aa[i] = p.c * aa[i] + p.b * ar + ((col == gr && gr < G.m_real) ? p.a : 0.0f);
          }
          put_kmajor(smem + ABUF_OFF, r, ch, aa);  // the products reading ABUF have completed
        }
      }
      fence_async_smem();
      sync_pair();
      // ---------------------------------------------------------------- X' = s B' X
      if (issuer && ok) issue_product(tmem, 0, sbase + ABUF_OFF, false, sbase + XCOL_OFF, true, mma_bar);
      wait_product();
      const float su = first ? alpha : 1.0f;
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int ch = half * 4 + c;
          float v[32];
          tmem_ld_32cols(t_row + ch * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= su;
          if (!last) {
            put_kmajor(smem + XROW_OFF, r, ch, v);
            // columns 32 ch.. of row gr, in the XCOL of CTA `half`
            const int cw = ch * 32 - half * 128;
            const int cc = cw >> 6, u0 = (cw & 63) >> 3;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t off = kb_r * CHUNK + cc * 8192 + rr * 128 + (((u0 + q) ^ (rr & 7)) << 4);
              st_cluster_v4(xcol_base + off, pack8(v + 8 * q));
            }
          } else {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(G.out) +
                                 static_cast<size_t>(mat) * kSmallTile * kSmallTile +
                                 static_cast<size_t>(gr) * kSmallTile + ch * 32;
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(out)[q] = pack8(v + 8 * q);
          }
        }
      }
      fence_async_all();  // XROW here and XCOL here or in the peer feed the next products
      sync_pair();
    }
  }

  // ------------------------------------------------------------ teardown
  sync_pair();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

size_t small_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_ns_small(const SmallParams& p, int num_sms, cudaStream_t s) {
  if (p.total <= 0) return cudaSuccess;
  // The shared-memory limit is a property of the function on each device: set it once per device.
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if ((attr_set.load() & bit) == 0) {
    e = cudaFuncSetAttribute(ns_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(SMEM_BYTES));
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  const int grid = 2 * std::min(num_sms / 2, p.total);
  ns_small_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

}  // namespace muon
