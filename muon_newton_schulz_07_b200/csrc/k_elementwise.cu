// Bandwidth-bound kernels of the Muon step:
//
//  * momentum_norm_kernel — momentum lerp, Nesterov blend, orientation and the
//    Frobenius norm in one pass over G and M (the first three steps of the
//    orthogonalised-momentum update the pages name: magicnetworld glossary
//    table, row "Muon"; aiproducthub "开发者千美元训3.8B模型 击败GPT-2",
//    影响 paragraph).  It reads G and M once, writes M1 in place and U (cast to
//    the Newton-Schulz operand type) into the zero-padded, oriented workspace
//    buffer X0.  Tall matrices are transposed through shared memory so X0 is
//    always min x max.  One CTA per 64 x 128 tile, four CTAs per SM.  The sum
//    of squares goes warp -> one partial per (CTA, warp)
//    in the workspace; norm_finish_kernel, the next launch, adds each matrix's
//    partials in a fixed order, so the norm is
//    deterministic, and stores ||U|| and 1/(||U|| + eps) (0 when both are 0: a
//    zero direction gives a zero update).  The normalisation itself is folded
//    into the first Newton-Schulz products.
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

#include <algorithm>
#include <vector>

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
      // the same fp32 products and fused multiply-adds as the scalar path, two lanes per
      // instruction (f32x2: each lane rounds exactly like fmaf / a * b)
      float m[8];
      c.m[q].to_f32x8(m);
      const float2 b2 = make_float2(beta, beta), o2 = make_float2(omb, omb);
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float2 og = __fmul2_rn(o2, make_float2(g[i], g[i + 1]));
        const float2 m1 = __ffma2_rn(b2, make_float2(m[i], m[i + 1]), og);
        const float2 u1 = p.nesterov ? __ffma2_rn(b2, m1, og) : m1;
        m[i] = m1.x;
        m[i + 1] = m1.y;
        u[i] = u1.x;
        u[i + 1] = u1.y;
      }
      Raw8<T>::store_cs(mom + base, m);
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

// The loads of one 64 x 128 tile of the oriented X0 (the matching source elements of G and M,
// whole aligned 8-element vectors only; ragged edges are read by momentum_chunk itself).
template <typename T>
__device__ __forceinline__ void momentum_tile_load(const EwMat& mt, const EwParams& p, int t, MomentumChunks<T>& ch) {
  const int xr0 = (t / mt.tiles_c) * kEwTileR;
  const int xc0 = (t % mt.tiles_c) * kEwTileC;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = threadIdx.x + q * kEwThreads;
    if (!mt.trans)
      momentum_load<T>(mt, p, q, xr0 + (c >> 4), xc0 + (c & 15) * 8, ch);
    else  // source tile in the caller's layout: rows xc0.., cols xr0..
      momentum_load<T>(mt, p, q, xc0 + (c >> 3), xr0 + (c & 7) * 8, ch);
  }
}

// The rest of the tile once its loads are in `ch`: momentum/Nesterov, M1 stored, U stored to X0
// (transposed through shared memory for tall matrices); returns this thread's sum of squares.
// A barrier over the kEwThreads threads that compute (named barrier 1: the bulk-copy kernel's
// producer warp does not take part), or the whole CTA.
template <bool NAMED>
__device__ __forceinline__ void compute_sync() {
  if (NAMED)
    asm volatile("bar.sync 1, %0;" ::"n"(kEwThreads) : "memory");
  else
    __syncthreads();
}

template <typename T, typename XT, int LD, bool NAMED = false>
__device__ __forceinline__ float momentum_tile_store(const EwMat& mt, const EwParams& p, int t,
                                                     const MomentumChunks<T>& ch, XT (*stage)[LD]) {
  float ss = 0.0f;
  const int xr0 = (t / mt.tiles_c) * kEwTileR;
  const int xc0 = (t % mt.tiles_c) * kEwTileC;
  XT* x = static_cast<XT*>(mt.x);
  if (!mt.trans) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int r = c >> 4, cc = (c & 15) * 8;
      float u[8];
      momentum_chunk<T>(mt, p, xr0 + r, xc0 + cc, ch, q, u, ss);
      Vec8<XT>::store(x + static_cast<size_t>(xr0 + r) * mt.np + xc0 + cc, u);
    }
  } else {
    compute_sync<NAMED>();  // the previous tile's staged values have been read out
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = threadIdx.x + q * kEwThreads;
      const int sr = c >> 3, sc = (c & 7) * 8;
      float u[8];
      momentum_chunk<T>(mt, p, xc0 + sr, xr0 + sc, ch, q, u, ss);
#pragma unroll
      for (int i = 0; i < 8; ++i) stage[sc + i][sr] = from_f32<XT>(u[i]);
    }
    compute_sync<NAMED>();
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

// This warp's part of its matrix's sum of squares: one plain store into slot (CTA, warp), which
// no other warp writes.  No atomics and no fences: the sums are added by norm_finish_kernel, the
// next launch on the stream.
__device__ __forceinline__ void momentum_flush(const EwParams& p, float ss) {
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0)
    p.partials[static_cast<size_t>(blockIdx.x) * (kEwThreads / 32) + (threadIdx.x >> 5)] = ss;
}

// One CTA per 64 x 128 tile: CTA c works on tile c of the launch (matrix j owns CTAs part_begin ..
// part_begin + nparts - 1, one per tile).  Each thread issues all eight of its 16-byte loads (G and
// M of four 8-element chunks) before any arithmetic, and four CTAs share an SM, so 32 KB per CTA
// (128 KB per SM) are in flight.  Short-lived CTAs rather than a persistent grid or several tiles
// per CTA: the block scheduler starts a new tile the moment one ends, which kept DRAM busier than
// every longer-lived form measured.
template <typename T, typename XT>
__global__ void __launch_bounds__(kEwThreads, sizeof(T) == 2 ? kEwMinCtasPerSm : 2)
    momentum_norm_kernel(const __grid_constant__ EwParams p) {
  constexpr int LD = kEwTileC + (sizeof(XT) == 2 ? 2 : 1);
  __shared__ XT stage[kEwTileR][LD];
  const int cta = static_cast<int>(blockIdx.x);
  int lo = 0, hi = p.nmat - 1;  // the matrix whose CTA range holds this CTA
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.mat[mid].part_begin <= cta) lo = mid; else hi = mid - 1;
  }
  const EwMat& mt = p.mat[lo];
  const int t = cta - mt.part_begin;
  MomentumChunks<T> ch;
  momentum_tile_load<T>(mt, p, t, ch);
  momentum_flush(p, momentum_tile_store<T, XT, LD>(mt, p, t, ch, stage));
}

// The norms of one momentum/norm launch's matrices: CTA j adds matrix j's per-warp partial sums
// in a fixed order (so the norm is the same on every run), and stores ||U|| and 1/(||U|| + eps)
// (0 when both are 0: a zero direction gives a zero update).
__global__ void __launch_bounds__(kEwThreads) norm_finish_kernel(const __grid_constant__ EwParams p) {
  __shared__ float red[kEwThreads / 32];
  const EwMat& mt = p.mat[blockIdx.x];
  const int n = mt.nparts * (kEwThreads / 32);
  const float* src = p.partials + static_cast<size_t>(mt.part_begin) * (kEwThreads / 32);
  float s = 0.0f;
  for (int i = threadIdx.x; i < n; i += kEwThreads) s += src[i];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < kEwThreads / 32; ++w) t += red[w];
    const float nrm = sqrtf(t);
    const float den = nrm + p.eps;
    p.scal[2 * mt.scal_idx] = nrm;
    p.scal[2 * mt.scal_idx + 1] = den > 0.0f ? 1.0f / den : 0.0f;
    p.norms[mt.caller_idx] = nrm;
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
  momentum_norm_kernel<T, XT><<<p.grid, kEwThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  norm_finish_kernel<<<p.nmat, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
template <typename T, typename XT>
cudaError_t launch_wr(const WrParams& p, cudaStream_t s) {
  param_write_kernel<T, XT><<<p.total_ctas, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

long long check_front_tables(const EwParams& p) {
  // The matrices' tile ranges back to back, one CTA (one partial-sum slot per warp) per tile, so
  // each matrix's CTA range is its tile range; the grid is the launch's tile count.
  long long bad = 0;
  if (p.nmat < 1 || p.nmat > kEwMatsPerLaunch) return 1;
  long long tiles = 0;
  for (int j = 0; j < p.nmat; ++j) {
    const EwMat& m = p.mat[j];
    if (m.tile_begin != tiles || m.ntiles < 1 || m.part_begin != m.tile_begin || m.nparts != m.ntiles ||
        m.tiles_c * kEwTileC != m.np ||
        static_cast<long long>(m.ntiles) * kEwTileR * kEwTileC != static_cast<long long>(m.mp) * m.np)
      ++bad;
    tiles += m.ntiles;
  }
  if (tiles != p.total_tiles || tiles != p.grid || p.grid < 1) ++bad;
  return bad;
}

cudaError_t launch_momentum_norm(const EwParams& p, Dtype io, Dtype xt, cudaStream_t s) {
  if (p.total_tiles <= 0 || p.grid <= 0) return cudaSuccess;
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
