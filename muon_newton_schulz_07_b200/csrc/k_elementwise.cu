// Bandwidth-bound kernels of the Muon step:
//
//  * momentum_norm_kernel — momentum lerp, Nesterov blend, orientation and the
//    Frobenius norm in one pass over G and M (the first three steps of the
//    orthogonalised-momentum update the pages name: magicnetworld glossary
//    table, row "Muon"; aiproducthub "开发者千美元训3.8B模型 击败GPT-2",
//    影响 paragraph).  It reads G and M once, writes M1 in place and U (cast to
//    the Newton-Schulz operand type) into the zero-padded, oriented workspace
//    buffer X0.  Tall matrices are transposed through shared memory so X0 is
//    always min x max.  Each CTA handles two tiles.  The sum of squares is
//    reduced warp -> CTA -> 8-CTA cluster (each CTA stores its partial into the
//    rank-0 CTA's shared memory, one cluster barrier) -> one partial per
//    cluster; the last cluster of a matrix to finish (acquire-release arrival
//    counter) adds the partials in a fixed order, so the norm is
//    deterministic, and stores ||U|| and 1/(||U|| + eps).  The normalisation itself is folded into the first
//    Newton-Schulz products.
//
//  * param_write_kernel — the parameter write
//    W1 = (1 - lr*wd) W - lr*sqrt(max(1, rows/cols)) O, O the final X oriented
//    back (transposed through shared memory for tall matrices), or O itself for
//    the orthogonaliser-only entry point.
//
// Both work on 64 x 128 tiles of the oriented matrix with 16-byte vector
// accesses whenever a row segment is aligned and complete, and element-wise
// accesses on ragged edges.
#include <cuda_bf16.h>

#include "muon_device.cuh"
#include "muon_internal.h"

namespace muon {
namespace {

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  // Load that may alias a later store by the same thread (no read-only path).
  static __device__ __forceinline__ void load_rw(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 q = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 q;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = q;
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void load_rw(const float* p, float (&v)[8]) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <typename Mats>
__device__ __forceinline__ int find_matrix(const Mats* mats, int nmat, int cta) {
  int lo = 0, hi = nmat - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (mats[mid].tile_begin <= cta) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Raw 16/32-byte vectors of 8 elements, loaded with the streaming (evict-first)
// hint: G, M and W are each touched once per step.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 q;
  __device__ __forceinline__ void load_cs(const __nv_bfloat16* p) { q = __ldcs(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void to_f32x8(float (&v)[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store_cs(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 q;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    __stcs(reinterpret_cast<uint4*>(p), q);
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load_cs(const float* p) {
    a = __ldcs(reinterpret_cast<const float4*>(p));
    b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void to_f32x8(float (&v)[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store_cs(float* p, const float (&v)[8]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
  }
};

// The four 8-element chunks a thread handles in one tile: every vector load of
// the tile is issued before any arithmetic or store, so each thread keeps eight
// 16-byte loads in flight.
template <typename T>
struct MomentumChunks {
  Raw8<T> g[4], m[4];
  bool vec[4];
};

template <typename T>
__device__ __forceinline__ void momentum_load(const EwMat& mt, const EwParams& p, int q, int row, int col,
                                              MomentumChunks<T>& c) {
  c.vec[q] = row < mt.rows && p.vec_ok && col + 8 <= mt.cols;
  if (c.vec[q]) {
    const size_t base = static_cast<size_t>(row) * mt.cols + col;
    c.g[q].load_cs(static_cast<const T*>(mt.src) + base);
    if (mt.mom != nullptr) c.m[q].load_cs(static_cast<const T*>(mt.mom) + base);
  }
}

// Momentum + Nesterov on 8 consecutive elements of row `row`, columns col..col+7
// of the caller's matrix (chunk q, loaded by momentum_load when it is a full
// aligned vector).  Writes M1 back, returns U (0 outside the matrix).
template <typename T>
__device__ __forceinline__ void momentum_chunk(const EwMat& mt, const EwParams& p, int row, int col,
                                               const MomentumChunks<T>& c, int q, float (&u)[8], float& ss) {
  const bool in_row = row < mt.rows;
  const T* src = static_cast<const T*>(mt.src);
  T* mom = static_cast<T*>(mt.mom);
  const size_t base = static_cast<size_t>(row) * mt.cols + col;
  const float beta = p.beta, omb = 1.0f - p.beta;
  if (c.vec[q]) {
    float g[8];
    c.g[q].to_f32x8(g);
    if (mom != nullptr) {
      float m[8];
      c.m[q].to_f32x8(m);
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmaf(beta, m[i], omb * g[i]);
      Raw8<T>::store_cs(mom + base, m);
#pragma unroll
      for (int i = 0; i < 8; ++i) u[i] = p.nesterov ? fmaf(beta, m[i], omb * g[i]) : m[i];
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) u[i] = g[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      u[i] = 0.0f;
      if (in_row && col + i < mt.cols) {
        float g = to_f32(src[base + i]);
        if (mom != nullptr) {
          float m = fmaf(beta, to_f32(mom[base + i]), omb * g);
          mom[base + i] = from_f32<T>(m);
          u[i] = p.nesterov ? fmaf(beta, m, omb * g) : m;
        } else {
          u[i] = g;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(u[i], u[i], ss);
}

// One 64 x 128 tile of the oriented X0: momentum/Nesterov on the matching source
// elements, U stored to X0 (transposed through shared memory for tall matrices);
// returns this thread's sum of squares.
template <typename T, typename XT, int LD>
__device__ __forceinline__ float momentum_tile(const EwMat& mt, const EwParams& p, int t, XT (*stage)[LD]) {
  float ss = 0.0f;
  const int xr0 = (t / mt.tiles_c) * kEwTileR;
  const int xc0 = (t % mt.tiles_c) * kEwTileC;
  XT* x = static_cast<XT*>(mt.x);
  MomentumChunks<T> ch;
  if (!mt.trans) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      momentum_load<T>(mt, p, q, xr0 + (c >> 4), xc0 + (c & 15) * 8, ch);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int r = c >> 4, cc = (c & 15) * 8;
      float u[8];
      momentum_chunk<T>(mt, p, xr0 + r, xc0 + cc, ch, q, u, ss);
      Vec8<XT>::store(x + static_cast<size_t>(xr0 + r) * mt.np + xc0 + cc, u);
    }
  } else {
    // source tile in the caller's layout: rows xc0.., cols xr0..
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      momentum_load<T>(mt, p, q, xc0 + (c >> 3), xr0 + (c & 7) * 8, ch);
    }
    __syncthreads();  // the previous tile's staged values have been read out
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int sr = c >> 3, sc = (c & 7) * 8;
      float u[8];
      momentum_chunk<T>(mt, p, xc0 + sr, xr0 + sc, ch, q, u, ss);
#pragma unroll
      for (int i = 0; i < 8; ++i) stage[sc + i][sr] = from_f32<XT>(u[i]);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int r = c >> 4, cc = (c & 15) * 8;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = to_f32(stage[r][cc + i]);
      Vec8<XT>::store(x + static_cast<size_t>(xr0 + r) * mt.np + xc0 + cc, v);
    }
  }
  return ss;
}

template <typename T, typename XT>
__global__ void __cluster_dims__(kEwCluster, 1, 1) __launch_bounds__(kEwThreads, 3)
    momentum_norm_kernel(const __grid_constant__ EwParams p) {
  constexpr int LD = kEwTileC + (sizeof(XT) == 2 ? 2 : 1);
  __shared__ XT stage[kEwTileR][LD];
  __shared__ float red[kEwThreads / 32];
  __shared__ float slots[kEwCluster];  // used in the cluster's rank-0 CTA: one partial per CTA

  const int cta = blockIdx.x;
  const EwMat& mt = p.mat[find_matrix(p.mat, p.nmat, cta)];
  const int local = cta - mt.tile_begin;  // CTA index within the matrix
  float ss = 0.0f;
#pragma unroll 1
  for (int j = 0; j < kEwTilesPerCta; ++j) {
    const int t = local * kEwTilesPerCta + j;
    if (t < mt.ntiles) ss += momentum_tile<T, XT, LD>(mt, p, t, stage);
  }

  // CTA reduction (fixed order)
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kEwThreads / 32; ++w) s += red[w];
    // push this CTA's partial into its slot in the rank-0 CTA's shared memory
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(remote) : "r"(smem_u32(&slots[rank])));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(s) : "memory");
  }
  // One cluster barrier: every partial has landed in rank 0 before it reads them, and no
  // CTA touches another CTA's shared memory afterwards.
  cluster_sync_all();
  if (rank == 0 && threadIdx.x < 32) {
    unsigned int prev = 0;
    if (threadIdx.x == 0) {
      float s = 0.0f;
#pragma unroll
      for (int r = 0; r < kEwCluster; ++r) s += slots[r];
      p.partials[mt.part_begin + local / kEwCluster] = s;
      // release the partial, acquire the others' if this cluster is the matrix's last
      asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                   : "=r"(prev)
                   : "l"(p.counters + mt.scal_idx)
                   : "memory");
    }
    __syncwarp();
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev == static_cast<unsigned int>(mt.nclusters - 1)) {
      float s = 0.0f;
      for (int i = threadIdx.x; i < mt.nclusters; i += 32) s += __ldcg(&p.partials[mt.part_begin + i]);
      s = warp_sum(s);
      if (threadIdx.x == 0) {
        const float nrm = sqrtf(s);
        p.scal[2 * mt.scal_idx] = nrm;
        p.scal[2 * mt.scal_idx + 1] = 1.0f / (nrm + p.eps);
        p.norms[mt.caller_idx] = nrm;
        p.counters[mt.scal_idx] = 0u;
      }
    }
  }
}

template <typename T>
struct WriteChunks {
  Raw8<T> w[4];
  bool vec[4];
};

template <typename T>
__device__ __forceinline__ void write_load(const WrMat& mt, const WrParams& p, int q, int row, int col,
                                           WriteChunks<T>& c) {
  c.vec[q] = row < mt.rows && p.vec_ok && col + 8 <= mt.cols;
  if (c.vec[q] && !p.store_only) c.w[q].load_cs(static_cast<const T*>(mt.w) + static_cast<size_t>(row) * mt.cols + col);
}

template <typename T>
__device__ __forceinline__ void write_chunk(const WrMat& mt, const WrParams& p, int row, int col,
                                            const WriteChunks<T>& c, int q, const float (&o)[8], float coef_w,
                                            float coef_o) {
  if (row >= mt.rows) return;
  T* w = static_cast<T*>(mt.w);
  const size_t base = static_cast<size_t>(row) * mt.cols + col;
  if (c.vec[q]) {
    float v[8];
    if (p.store_only) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = coef_o * o[i];
    } else {
      c.w[q].to_f32x8(v);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = fmaf(coef_w, v[i], coef_o * o[i]);
    }
    Raw8<T>::store_cs(w + base, v);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (col + i < mt.cols) {
        const float prev = p.store_only ? 0.0f : to_f32(w[base + i]);
        w[base + i] = from_f32<T>(p.store_only ? coef_o * o[i] : fmaf(coef_w, prev, coef_o * o[i]));
      }
    }
  }
}

template <typename T, typename XT>
__global__ void __launch_bounds__(kEwThreads, 3) param_write_kernel(const __grid_constant__ WrParams p) {
  __shared__ float stage[kEwTileR][kEwTileC + 1];
  const int cta = blockIdx.x;
  const WrMat& mt = p.mat[find_matrix(p.mat, p.nmat, cta)];
  const int t = cta - mt.tile_begin;
  const int xr0 = (t / mt.tiles_c) * kEwTileR;
  const int xc0 = (t % mt.tiles_c) * kEwTileC;
  const XT* x = static_cast<const XT*>(mt.x);
  const float alpha = p.use_alpha ? p.scal[2 * mt.scal_idx + 1] : 1.0f;
  const float coef_o = p.store_only ? alpha : -p.lr * mt.shape_scale * alpha;
  const float coef_w = 1.0f - p.lr * p.wd;
  WriteChunks<T> wc4;
  if (!mt.trans) {
    float o[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int r = c >> 4, cc = (c & 15) * 8;
      write_load<T>(mt, p, q, xr0 + r, xc0 + cc, wc4);
      if (xr0 + r < mt.rows) Vec8<XT>::load(x + static_cast<size_t>(xr0 + r) * mt.np + xc0 + cc, o[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      write_chunk<T>(mt, p, xr0 + (c >> 4), xc0 + (c & 15) * 8, wc4, q, o[q], coef_w, coef_o);
    }
  } else {
    // The X tile (rows xr0.. = W columns, columns xc0.. = W rows) goes through shared
    // memory and comes out transposed; the W loads are issued before the barrier.
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      write_load<T>(mt, p, q, xc0 + (c >> 3), xr0 + (c & 7) * 8, wc4);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int r = c >> 4, cc = (c & 15) * 8;
      float o[8];
      Vec8<XT>::load(x + static_cast<size_t>(xr0 + r) * mt.np + xc0 + cc, o);
#pragma unroll
      for (int i = 0; i < 8; ++i) stage[r][cc + i] = o[i];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int wr = c >> 3, wc = (c & 7) * 8;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = stage[wc + i][wr];
      write_chunk<T>(mt, p, xc0 + wr, xr0 + wc, wc4, q, o, coef_w, coef_o);
    }
  }
}

template <typename T, typename XT>
cudaError_t launch_mn(const EwParams& p, cudaStream_t s) {
  momentum_norm_kernel<T, XT><<<p.total_ctas, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
template <typename T, typename XT>
cudaError_t launch_wr(const WrParams& p, cudaStream_t s) {
  param_write_kernel<T, XT><<<p.total_ctas, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_momentum_norm(const EwParams& p, Dtype io, Dtype xt, cudaStream_t s) {
  if (p.total_ctas <= 0) return cudaSuccess;
  if (io == kBF16 && xt == kBF16) return launch_mn<__nv_bfloat16, __nv_bfloat16>(p, s);
  if (io == kF32 && xt == kBF16) return launch_mn<float, __nv_bfloat16>(p, s);
  if (io == kBF16 && xt == kF32) return launch_mn<__nv_bfloat16, float>(p, s);
  return launch_mn<float, float>(p, s);
}

cudaError_t launch_param_write(const WrParams& p, Dtype io, Dtype xt, cudaStream_t s) {
  if (p.total_ctas <= 0) return cudaSuccess;
  if (io == kBF16 && xt == kBF16) return launch_wr<__nv_bfloat16, __nv_bfloat16>(p, s);
  if (io == kF32 && xt == kBF16) return launch_wr<float, __nv_bfloat16>(p, s);
  if (io == kBF16 && xt == kF32) return launch_wr<__nv_bfloat16, float>(p, s);
  return launch_wr<float, float>(p, s);
}

}  // namespace muon
