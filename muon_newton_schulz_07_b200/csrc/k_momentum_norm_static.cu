// Momentum + Nesterov + Frobenius norm of one matrix without any caller-provided
// workspace (muon_momentum_norm_static in include/muon.h).
//
// Some callers cannot hand this library device memory for scratch: code that
// runs while another component owns every allocation on the device (a
// framework's caching allocator, a fixed memory pool), or code that must not
// call cudaMalloc at all.  For them this entry point keeps the reduction
// scratch of the norm (one partial sum per 8-CTA cluster and one arrival
// counter) in a file-scope __device__ array of fixed size, which every GPU that
// loads the library holds until the process exits.  The caller passes only the
// inputs and outputs.
//
// Set-up: the first call on a device (with that device current) looks up the
// array's device address with cudaGetSymbolAddress and caches it; make that
// first call before capturing any stream.  A first call made on a stream that
// is being captured returns MUON_ERR_UNSUPPORTED and leaves the capture intact.  Every call shares the one array and
// leaves its last contents behind; the counter is cleared at the start of each
// call, so calls in sequence are independent, but calls that overlap on the GPU
// (different streams, or graphs replayed concurrently) race on the array.
#include <cuda_bf16.h>

#include <mutex>

#include "muon.h"
#include "muon_device.cuh"

namespace muon {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 32;                        // 4 vectors of 8 elements
constexpr int kPerCta = kThreads * kPerThread;        // 8192 elements
constexpr int kCluster = 8;
constexpr int kMaxClusters = static_cast<int>(MUON_STATIC_MAX_ELEMENTS / (kPerCta * kCluster));
constexpr size_t kScratchBytes = 256 + sizeof(float) * kMaxClusters;   // counter block + partials

// The scratch.  In host code this name is only a host-side stand-in for the
// device array: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_norm_scratch[kScratchBytes];

template <typename T> __device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
template <> __device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <typename T> __device__ __forceinline__ void store8(T* p, const float (&v)[8]);
template <> __device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = q;
}
template <> __device__ __forceinline__ void store8<float>(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

template <typename T>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads)
    momentum_norm_static_kernel(const T* __restrict__ g, T* m, T* __restrict__ u, long long n, float beta,
                                int nesterov, int vec_ok, float* norm_out, unsigned char* scratch) {
  __shared__ float red[kThreads / 32];
  __shared__ float cta_part;
  unsigned int* counter = reinterpret_cast<unsigned int*>(scratch);
  float* partials = reinterpret_cast<float*>(scratch + 256);
  const float omb = 1.0f - beta;
  const long long base = static_cast<long long>(blockIdx.x) * kPerCta;
  float ss = 0.0f;
#pragma unroll
  for (int q = 0; q < kPerThread / 8; ++q) {
    const long long e = base + (static_cast<long long>(q) * kThreads + threadIdx.x) * 8;
    if (e >= n) continue;
    float gv[8], mv[8], uv[8];
    if (vec_ok && e + 8 <= n) {
      load8<T>(g + e, gv);
      load8<T>(m + e, mv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        mv[i] = fmaf(beta, mv[i], omb * gv[i]);
        uv[i] = nesterov ? fmaf(beta, mv[i], omb * gv[i]) : mv[i];
        ss = fmaf(uv[i], uv[i], ss);
      }
      store8<T>(m + e, mv);
      store8<T>(u + e, uv);
    } else {
      for (int i = 0; i < 8 && e + i < n; ++i) {
        const float gi = to_f32(g[e + i]);
        const float mi = fmaf(beta, to_f32(m[e + i]), omb * gi);
        const float ui = nesterov ? fmaf(beta, mi, omb * gi) : mi;
        m[e + i] = from_f32<T>(mi);
        u[e + i] = from_f32<T>(ui);
        ss = fmaf(ui, ui, ss);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) s += red[w];
    cta_part = s;
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  if (rank == 0 && threadIdx.x < 32) {
    int last = 0;
    if (threadIdx.x == 0) {
      float s = 0.0f;
      for (uint32_t r = 0; r < kCluster; ++r) {
        uint32_t remote;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(&cta_part)), "r"(r));
        float v;
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
        s += v;
      }
      partials[blockIdx.x / kCluster] = s;
      __threadfence();
      const unsigned int nclusters = gridDim.x / kCluster;
      last = (atomicAdd(counter, 1u) == nclusters - 1);
      if (last) __threadfence();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      const int nclusters = static_cast<int>(gridDim.x / kCluster);
      float s = 0.0f;
      for (int i = threadIdx.x; i < nclusters; i += 32) s += __ldcg(&partials[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (threadIdx.x == 0) {
        *norm_out = sqrtf(s);
        *counter = 0u;
      }
    }
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Device address of the scratch array, looked up once per device.
constexpr int kMaxDevices = 64;
unsigned char* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Returns MUON_OK, MUON_ERR_UNSUPPORTED when the address is not known yet and `stream` is being
// captured (the look-up would break the capture), or MUON_ERR_CUDA.
muon_status_t scratch_for_current_device(cudaStream_t stream, unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MUON_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return MUON_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return MUON_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_norm_scratch) != cudaSuccess) return MUON_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_scratch_addr[dev];
  return MUON_OK;
}

}  // namespace
}  // namespace muon

extern "C" MUON_API muon_status_t muon_momentum_norm_static(const void* G, void* M, void* U, int64_t rows,
                                                            int64_t cols, muon_dtype_t dtype, float beta,
                                                            int32_t nesterov, float* norm, cudaStream_t stream) {
  using namespace muon;
  if (G == nullptr || M == nullptr || U == nullptr || norm == nullptr) return MUON_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1 || !(beta >= 0.0f && beta <= 1.0f)) return MUON_ERR_INVALID_ARG;
  if (dtype != MUON_BF16 && dtype != MUON_FP32) return MUON_ERR_INVALID_ARG;
  if (rows > MUON_STATIC_MAX_ELEMENTS / cols) return MUON_ERR_UNSUPPORTED;  // beyond the fixed scratch
  const long long n = rows * cols;
  unsigned char* scratch = nullptr;
  const muon_status_t st = scratch_for_current_device(stream, &scratch);
  if (st != MUON_OK) {
    cudaGetLastError();
    return st;
  }
  const long long ctas = (n + kPerCta - 1) / kPerCta;
  const int grid = static_cast<int>((ctas + kCluster - 1) / kCluster * kCluster);
  const uintptr_t all = reinterpret_cast<uintptr_t>(G) | reinterpret_cast<uintptr_t>(M) |
                        reinterpret_cast<uintptr_t>(U);
  const int vec_ok = (all & 15u) == 0 ? 1 : 0;
  // The arrival counter must start at zero; the partials are all rewritten.
  if (cudaMemsetAsync(scratch, 0, sizeof(unsigned int), stream) != cudaSuccess) return MUON_ERR_CUDA;
  if (dtype == MUON_BF16) {
    momentum_norm_static_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(G), static_cast<__nv_bfloat16*>(M), static_cast<__nv_bfloat16*>(U), n,
        beta, nesterov ? 1 : 0, vec_ok, norm, scratch);
  } else {
    momentum_norm_static_kernel<float><<<grid, kThreads, 0, stream>>>(
        static_cast<const float*>(G), static_cast<float*>(M), static_cast<float*>(U), n, beta, nesterov ? 1 : 0,
        vec_ok, norm, scratch);
  }
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}
