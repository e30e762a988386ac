// FP32 reference-mode products of the Newton-Schulz iteration on the CUDA
// cores, one batched launch per shape group and stage.  Operands and results are
// fp32; the products of fp32 numbers are exact in fp64 and are summed in fp64
// (DFMA) and combined in fp64, so the only roundings are the fp32 stores of X, A
// and B'.  (Summing in
// fp32 along K = 8192 loses enough that ten Newton-Schulz steps, which amplify
// small singular directions by up to a^10, miss 1e-4 on condition-1e6 inputs.)
//   Gram:    C = s * (X X^T)           (b_trans = 1, second operand X itself)
//   Poly:    C = c * (A A) + b * A + a * I   (A symmetric; B' carries the a X term)
//   Update:  C = s * (B' X)
// 64 x 64 output tiles, 16-deep k slices through shared memory, 4 x 4 outputs per
// thread.  Every dimension is a multiple of 64 (the workspace is zero-padded), so
// the kernel has no edge predicates; the host checks this before launching.
// Also here: the failure-detection self-test kernel.
#include "muon_device.cuh"
#include "muon_internal.h"

namespace muon {
namespace {

constexpr int SB = 64, SK = 16;

template <int BT>
__global__ void __launch_bounds__(256) sgemm_kernel(const SgParams p) {
  __shared__ float As[SK][SB + 4];
  __shared__ float Bs[SK][SB + 4];
  const int z = blockIdx.z;
  const float* A = p.a + z * p.sa;
  const float* B = p.b + z * p.sb;
  float* C = p.c + z * p.sc;
  const int m0 = blockIdx.y * SB, n0 = blockIdx.x * SB;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;

  for (int k0 = 0; k0 < p.K; k0 += SK) {
#pragma unroll
    for (int e = threadIdx.x; e < SB * SK; e += 256) {
      const int r = e / SK, kk = e % SK;
      As[kk][r] = A[static_cast<size_t>(m0 + r) * p.lda + k0 + kk];
      if (BT) {
        Bs[kk][r] = B[static_cast<size_t>(n0 + r) * p.ldb + k0 + kk];
      } else {
        const int kr = e / SB, c = e % SB;
        Bs[kr][c] = B[static_cast<size_t>(k0 + kr) * p.ldb + n0 + c];
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  // The epilogue works in fp64 as well, so each stored element is rounded to fp32 once.
  double s = 1.0;
  if (p.scal_mode != 0) {
    const double al = p.scal[2 * (p.scal_base + z) + 1];
    s = (p.scal_mode == 1) ? al * al : al;
  }
  const float* aux = p.aux ? p.aux + z * p.sc : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const size_t row = static_cast<size_t>(m0 + ty * 4 + i) * p.ldc;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      double v = static_cast<double>(p.c_acc) * acc[i][j];
      if (aux) v = fma(static_cast<double>(p.c_aux), static_cast<double>(aux[row + col]), v);
      if (col == m0 + ty * 4 + i && col < p.diag_n) v += p.c_diag;
      C[row + col] = static_cast<float>(s * v);
    }
  }
}

__global__ void timeout_selftest_kernel(unsigned int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_barrier_init();
    // Nothing ever arrives on this barrier: the bounded wait must give up,
    // record the timeout and return.
    (void)mbar_wait_bounded(b, 0, timeout_ns, nullptr, status);
  }
}

}  // namespace

cudaError_t launch_sgemm(const SgParams& p, cudaStream_t s) {
  if (p.M % SB || p.N % SB || p.K % SK || p.cnt <= 0) return cudaErrorInvalidValue;
  dim3 grid(p.N / SB, p.M / SB, p.cnt);
  if (p.b_trans) sgemm_kernel<1><<<grid, 256, 0, s>>>(p);
  else sgemm_kernel<0><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_timeout_selftest(unsigned int* status, unsigned long long timeout_ns, cudaStream_t s) {
  timeout_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace muon
