// Internal launch interfaces between the C ABI (muon_api.cu) and the kernels.
// Nothing here is exported from libmuon.so.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime_api.h>

namespace muon {

// Device status codes (written to the workspace status word; match muon_status_t).
constexpr unsigned int kDevTimeout = 5;
constexpr unsigned int kDevFault = 6;

// Every workspace buffer is padded to multiples of this many rows/columns.
constexpr int kPad = 256;

// ------------------------------------------------------------------ elementwise
// Elementwise kernels work on X-coordinate tiles of 64 x 128 (X is the oriented
// matrix, min(rows,cols) x max(rows,cols), padded to multiples of kPad).
constexpr int kEwTileR = 64;
constexpr int kEwTileC = 128;
constexpr int kEwThreads = 256;
constexpr int kEwMinCtasPerSm = 4;  // resident momentum/norm CTAs per SM the register budget allows (bf16 sources)
constexpr int kEwMatsPerLaunch = 192;

enum Dtype : int { kBF16 = 0, kF32 = 1 };

struct EwMat {
  const void* src;   // G (step) or X (orthogonalize), rows x cols, caller's layout
  void* mom;         // M, updated in place; nullptr: no momentum (U = src)
  void* x;           // workspace X buffer of this matrix, mp x np, row stride np
  int rows, cols;    // caller's shape
  int mp, np;        // padded oriented shape
  int trans;         // rows > cols: X = U^T
  int tile_begin;    // first tile of this matrix in the launch's tile list
  int tiles_c;       // X tiles along np
  int ntiles;        // X tiles of the padded matrix (mp/64 * np/128)
  int scal_idx;      // slot of this matrix in the scalar / counter tables
  int caller_idx;    // position in the caller's matrix list
  int part_begin;    // first CTA of this matrix in the launch (= tile_begin: one CTA per tile)
  int nparts;        // CTAs of this matrix, each with one partial-sum slot per warp (= ntiles)
};

// The momentum/norm launch: one CTA per tile, matrix j's CTAs part_begin .. part_begin + nparts - 1.
struct EwParams {
  EwMat mat[kEwMatsPerLaunch];
  int nmat;
  int total_tiles;
  int grid;                // CTAs of the launch: the sum of the matrices' nparts
  float beta;
  float eps;
  int nesterov;
  int vec_ok;              // every row of every matrix starts 16-byte aligned
  float* partials;         // per (CTA, warp) sums of squares
  float* scal;             // per matrix: {||U||_F, 1/(||U||_F + eps)}
  float* norms;            // ||U||_F per matrix, caller order
  unsigned int* status;    // device status word (a bounded wait that ran out)
};

struct WrMat {
  void* w;           // W (updated in place) or O (written)
  const void* x;     // final X of this matrix, mp x np, row stride np
  int rows, cols, mp, np, trans;
  int tile_begin;    // first CTA of this matrix
  int tiles_c;       // tiles along the real n
  int scal_idx;
  float shape_scale; // sqrt(max(1, rows/cols))
};

struct WrParams {
  WrMat mat[kEwMatsPerLaunch];
  int nmat;
  int total_ctas;
  float lr, wd;
  int store_only;   // 1: O = X (orthogonalize); 0: W = (1 - lr*wd) W - lr*s*X
  int use_alpha;    // 1: X still unnormalised (k = 0), multiply by 1/(||U||+eps)
  int vec_ok;
  const float* scal;
};

cudaError_t launch_momentum_norm(const EwParams& p, Dtype io, Dtype xt, cudaStream_t s);
cudaError_t launch_param_write(const WrParams& p, Dtype io, Dtype xt, cudaStream_t s);

// ------------------------------------------------------------------ tcgen05 GEMMs
constexpr int kTcBM = 128;
constexpr int kTcBN = 256;
constexpr int kTcBK = 64;
constexpr int kTcMaxGroups = 6;
constexpr int kTcEpiWarps = 8;     // two per TMEM lane quadrant, each on half of the tile's columns
constexpr int kTcThreads = 64 + 32 * kTcEpiWarps;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue

enum TcKind : int { kGram = 0, kPoly = 1, kUpdate = 2 };

struct alignas(64) TcGroup {
  CUtensorMap tm_a;     // operand A source, row view: box 64 (k) x 128 (rows) x 1, 128B swizzle
  CUtensorMap tm_at;    // the same buffer, chunked view for MN-major reads: box 64 x 64 (k) x 2 chunks x 1
  CUtensorMap tm_b;     // operand B source, row view
  CUtensorMap tm_bt;    // operand B source, chunked view
  CUtensorMap tm_out;   // output, store view: box 32 x 32 x 1, 64B swizzle
  CUtensorMap tm_aux;   // Poly's epilogue input A, store view (box 32 x 32, 64B swizzle), loaded by TMA
  void* out;            // [cnt][rows][ld] bf16
  int cnt, mp, np;
  int tiles_per_mat;
  int tile_begin;
  int kblocks;
  int scal_base;
  int tdim;             // Gram/Poly: mp/256 (triangle side); Update: np/256
  int out_ld;
  int m_real;           // real (unpadded) rows: Poly adds its diagonal term only there
  int n_real;           // real (unpadded) columns of X
  int pad_;
};

// Largest number of matrices whose parameter write can be fused into the last
// Update launch (their pointers travel in the kernel parameters).
constexpr int kTcMaxFused = 1024;

struct TcParams {
  TcGroup g[kTcMaxGroups];
  int ngroups;
  int total_tiles;
  int kind;
  int wide;              // Update with 256 x 512 pair tiles (every group's np a multiple of 512)
  int use_scal;          // first iteration: fold the normalisation in
  float c_acc, c_aux;    // out = s * (c_acc * acc + c_aux * aux) (+ c_diag on the real diagonal)
  float c_diag;
  const float* scal;
  unsigned int* status;
  unsigned long long timeout_ns;
  // Fused parameter write (last Update only).  Instead of storing X_k, the epilogue
  // writes W = w_decay * W + wcoef[slot] * X_k into the caller's bf16 matrix of each
  // slot (the scalar-table index), transposed back when wtrans[slot] is set.  With
  // w_decay == 0 it stores wcoef * X_k without reading W (the orthogonaliser output).
  int fuse_write;
  float w_decay;
  void* wptr[kTcMaxFused];
  float wcoef[kTcMaxFused];
  unsigned char wtrans[kTcMaxFused];
};

size_t tc_smem_bytes();
cudaError_t launch_tc_gemm(const TcParams& p, int num_sms, cudaStream_t s);

// ------------------------------------------------------------------ every iteration in one launch
// One persistent launch runs all k x {Gram, Poly, Update} stages of every matrix of up to
// kTcMaxGroups shape groups.  Tiles are listed stage after stage (iteration-major, then
// Gram / Poly / Update, then group, matrix and tile) and dealt round-robin to the CTA pairs;
// before loading a tile, a pair waits (bounded) until the stage the tile reads is complete for
// its matrix: every epilogue warp that finishes a tile adds 1 to a per (stage, matrix)
// completion counter in the workspace.
struct alignas(64) NsGroup {
  CUtensorMap x_row[2], x_chk[2], x_st[2];  // X0 / X1: row, chunked and store views
  CUtensorMap a_row, a_chk, a_st;           // A
  CUtensorMap b_row, b_chk, b_st;           // B'
  int cnt, mp, np;
  int m_real, n_real;
  int scal_base;        // first slot of the group in the scalar / counter tables
  int tdim;             // mp / 256
  int pad_[7];
};

struct NsParams {
  NsGroup g[kTcMaxGroups];
  int ngroups;
  int k;                 // iterations, >= 1
  int nslots;            // matrices of the launch (the counter table's row length)
  int tiles_iter;        // tiles of an iteration other than the last
  int total_tiles;
  int t_begin, t_end;    // the tiles this launch runs: [0, total_tiles), or one stage of them
  int upd_tw[2];         // Update tile width (256 or 512) of [other, last] iterations
  int sym_wide;          // Gram and Poly take two neighbouring upper blocks per tile (256 x 512)
  int fuse_write;        // the last Update writes the parameters (see TcParams)
  // first tile of (stage, group) within an iteration, [other, last][stage][group];
  // [..][stage][ngroups] is the end of the stage
  int begin[2][3][kTcMaxGroups + 1];
  float a, b, c;
  const float* scal;
  unsigned int* status;
  unsigned int* deps;    // [3 k][nslots] completion counters, zero before the launch
  unsigned long long timeout_ns;
  float w_decay;
  void* wptr[kTcMaxFused];
  float wcoef[kTcMaxFused];
  unsigned char wtrans[kTcMaxFused];
};

// Tiles per matrix of a symmetric stage (Gram, Poly) over the T x T blocks of the upper
// triangle: one per block, or (wide) one per pair of neighbouring blocks of a block row, with a
// 256-wide tile for the odd block at the end of a row.
__host__ __device__ inline int sym_tiles(int T, bool wide) {
  if (!wide) return T * (T + 1) / 2;
  int n = 0;
  for (int I = 0; I < T; ++I) n += (T - I + 1) / 2;
  return n;
}

size_t fused_smem_bytes();
cudaError_t launch_ns_fused(const NsParams& p, int num_sms, cudaStream_t s);
// Host-side consistency check of a single-launch tile list (number of problems found).
long long check_fused_tiles(const NsParams& p);
// Host-side consistency check of one momentum/norm launch's tables (number of problems found).
long long check_front_tables(const EwParams& p);

// ------------------------------------------------------------------ small matrices, all iterations in one kernel
// Every matrix of the set fits one 256 x 256 tile (max(rows, cols) <= 256; the workspace
// pads it to 256 x 256).  One CTA pair runs all k Newton-Schulz iterations of a matrix.
constexpr int kSmallTile = 256;

struct alignas(64) SmGroup {
  CUtensorMap tm_row;   // X0, row view (box 64 x 128 x 1): this CTA's 128 rows, one 64-wide k chunk
  CUtensorMap tm_col;   // X0, chunked view (box 64 x 64 x 2 x 1): 64 rows of this CTA's 128 columns
  void* out;            // [cnt][256][256] bf16: X_k
  int mat_begin;        // first matrix of the group in the launch's numbering
  int cnt;
  int scal_base;
  int m_real;           // real rows of the Gram matrix (the polynomial's a I stops there)
};

struct SmallParams {
  SmGroup g[kTcMaxGroups];
  int ngroups;
  int total;            // matrices in the launch
  int k;                // Newton-Schulz iterations, >= 1
  float a, b, c;
  const float* scal;    // per matrix {||U||, 1/(||U||+eps)}
  unsigned int* status;
  unsigned long long timeout_ns;
};

size_t small_smem_bytes();
cudaError_t launch_ns_small(const SmallParams& p, int num_sms, cudaStream_t s);

// ------------------------------------------------------------------ fp32 reference GEMMs
struct SgParams {
  const float* a; const float* b; float* c; const float* aux;
  int M, N, K;
  int lda, ldb, ldc;
  long long sa, sb, sc;   // batch strides (elements)
  int cnt;
  int b_trans;            // 1: second operand is b^T (b row-major N x K)
  float c_acc, c_aux;
  const float* scal; int scal_base; int scal_mode;  // 0: none, 1: alpha^2, 2: alpha
  float c_diag; int diag_n;  // add c_diag to C[i][i] for i < diag_n
};
cudaError_t launch_sgemm(const SgParams& p, cudaStream_t s);

// ------------------------------------------------------------------ self-test
cudaError_t launch_timeout_selftest(unsigned int* status, unsigned long long timeout_ns, cudaStream_t s);

}  // namespace muon
