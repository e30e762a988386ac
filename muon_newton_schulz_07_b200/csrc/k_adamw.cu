// AdamW for the parameters that are not 2-D matrices (embeddings, heads, gains,
// scalars): the other half of the hybrid optimizer ("开发者千美元训3.8B模型
// 击败GPT-2", aiproducthub, 影响 paragraph: Newton-Schulz for the matrix
// parameters, AdamW for the rest).  Per element, with bias corrections
// bc1 = 1 - beta1^t and bc2 = 1 - beta2^t computed on the host in double:
//   m1 = beta1 m + (1 - beta1) g
//   v1 = beta2 v + (1 - beta2) g^2
//   p1 = (1 - lr wd) p - (lr / bc1) m1 / (sqrt(v1) / sqrt(bc2) + eps)
// which is (1 - lr wd) p - lr mh / (sqrt(vh) + eps) with mh = m1/bc1, vh = v1/bc2.
//
// One multi-tensor launch covers up to 256 tensors: every CTA handles a chunk of
// 2048 elements of one tensor, each thread 8 consecutive elements, all loads of
// a thread issued before its arithmetic (16-byte vectors when the tensor's
// pointers are aligned, element-wise on a ragged tail).  p and g are bf16 or
// fp32; the moments m and v are always fp32.  Purely bandwidth-bound.
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>

#include "muon.h"
#include "muon_device.cuh"

namespace muon {
namespace {

constexpr int kAdamThreads = 256;
constexpr int kAdamPerThread = 8;
constexpr int kAdamChunk = kAdamThreads * kAdamPerThread;  // 2048
constexpr int kAdamMaxTensors = 256;

struct AdamTensor {
  void* p;
  const void* g;
  float* m;
  float* v;
  long long n;
  long long chunk_begin;
  int vec_ok;
  int pad_;
};

struct AdamParams {
  AdamTensor t[kAdamMaxTensors];
  int ntensors;
  float beta1, beta2, eps;
  float decay;          // 1 - lr * wd
  float step_size;      // lr / bc1
  float inv_sqrt_bc2;   // 1 / sqrt(bc2)
};

template <typename T> __device__ __forceinline__ void ld8(const T* p, float (&v)[8]);
template <> __device__ __forceinline__ void ld8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = __ldcs(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
template <> __device__ __forceinline__ void ld8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(p)), b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <typename T> __device__ __forceinline__ void st8(T* p, const float (&v)[8]);
template <> __device__ __forceinline__ void st8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  __stcs(reinterpret_cast<uint4*>(p), q);
}
template <> __device__ __forceinline__ void st8<float>(float* p, const float (&v)[8]) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

__device__ __forceinline__ float adam_update(float& m, float& v, float p, float g, const AdamParams& a) {
  m = fmaf(a.beta1, m, (1.0f - a.beta1) * g);
  v = fmaf(a.beta2, v, (1.0f - a.beta2) * g * g);
  const float denom = fmaf(sqrtf(v), a.inv_sqrt_bc2, a.eps);
  return fmaf(a.decay, p, -a.step_size * (m / denom));
}

template <typename T>
__global__ void __launch_bounds__(kAdamThreads) adamw_kernel(const __grid_constant__ AdamParams a) {
  const long long chunk = blockIdx.x;
  int lo = 0, hi = a.ntensors - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.t[mid].chunk_begin <= chunk) lo = mid; else hi = mid - 1;
  }
  const AdamTensor& tt = a.t[lo];
  const long long e = (chunk - tt.chunk_begin) * kAdamChunk + static_cast<long long>(threadIdx.x) * kAdamPerThread;
  if (e >= tt.n) return;
  T* p = static_cast<T*>(tt.p) + e;
  const T* g = static_cast<const T*>(tt.g) + e;
  float* m = tt.m + e;
  float* v = tt.v + e;
  if (tt.vec_ok && e + kAdamPerThread <= tt.n) {
    float pv[8], gv[8], mv[8], vv[8];
    ld8<T>(p, pv);
    ld8<T>(g, gv);
    ld8<float>(m, mv);
    ld8<float>(v, vv);
#pragma unroll
    for (int i = 0; i < 8; ++i) pv[i] = adam_update(mv[i], vv[i], pv[i], gv[i], a);
    st8<T>(p, pv);
    st8<float>(m, mv);
    st8<float>(v, vv);
  } else {
    const int cnt = static_cast<int>(min(static_cast<long long>(kAdamPerThread), tt.n - e));
    for (int i = 0; i < cnt; ++i) {
      float mi = m[i], vi = v[i];
      const float pi = adam_update(mi, vi, to_f32(p[i]), to_f32(g[i]), a);
      p[i] = from_f32<T>(pi);
      m[i] = mi;
      v[i] = vi;
    }
  }
}

}  // namespace
}  // namespace muon

extern "C" MUON_API muon_status_t muon_adamw_step(void* const* P, const void* const* G, float* const* M,
                                                  float* const* V, const int64_t* numel, int n, muon_dtype_t dtype,
                                                  const muon_adamw_hparams_t* hp, cudaStream_t stream) {
  using namespace muon;
  if (n < 0 || hp == nullptr) return MUON_ERR_INVALID_ARG;
  if (n == 0) return MUON_OK;
  if (P == nullptr || G == nullptr || M == nullptr || V == nullptr || numel == nullptr) return MUON_ERR_INVALID_ARG;
  if (dtype != MUON_BF16 && dtype != MUON_FP32) return MUON_ERR_INVALID_ARG;
  if (hp->step < 1 || !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) ||
      !(hp->eps >= 0.0f) || !std::isfinite(hp->lr) || !std::isfinite(hp->weight_decay))
    return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (numel[i] < 0) return MUON_ERR_INVALID_ARG;
    if (numel[i] > 0 && (P[i] == nullptr || G[i] == nullptr || M[i] == nullptr || V[i] == nullptr))
      return MUON_ERR_INVALID_ARG;
  }
  const double bc1 = 1.0 - std::pow(static_cast<double>(hp->beta1), hp->step);
  const double bc2 = 1.0 - std::pow(static_cast<double>(hp->beta2), hp->step);
  static thread_local AdamParams prm;  // ~12 KB: kept off the stack
  int i = 0;
  while (i < n) {
    std::memset(&prm, 0, sizeof(prm));
    prm.beta1 = hp->beta1;
    prm.beta2 = hp->beta2;
    prm.eps = hp->eps;
    prm.decay = static_cast<float>(1.0 - static_cast<double>(hp->lr) * hp->weight_decay);
    prm.step_size = static_cast<float>(hp->lr / bc1);
    prm.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
    long long chunks = 0;
    int cnt = 0;
    for (; i < n && cnt < kAdamMaxTensors; ++i) {
      if (numel[i] == 0) continue;
      AdamTensor& t = prm.t[cnt++];
      t.p = P[i];
      t.g = G[i];
      t.m = M[i];
      t.v = V[i];
      t.n = numel[i];
      t.chunk_begin = chunks;
      const uintptr_t al = reinterpret_cast<uintptr_t>(P[i]) | reinterpret_cast<uintptr_t>(G[i]) |
                           reinterpret_cast<uintptr_t>(M[i]) | reinterpret_cast<uintptr_t>(V[i]);
      t.vec_ok = (al & 15u) == 0 ? 1 : 0;
      chunks += (numel[i] + kAdamChunk - 1) / kAdamChunk;
    }
    if (cnt == 0) break;
    if (chunks > 0x7fffffffll) return MUON_ERR_UNSUPPORTED;
    prm.ntensors = cnt;
    if (dtype == MUON_BF16)
      adamw_kernel<__nv_bfloat16><<<static_cast<unsigned>(chunks), kAdamThreads, 0, stream>>>(prm);
    else
      adamw_kernel<float><<<static_cast<unsigned>(chunks), kAdamThreads, 0, stream>>>(prm);
    if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  }
  return MUON_OK;
}
