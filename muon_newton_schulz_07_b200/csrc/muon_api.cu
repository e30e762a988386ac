// C ABI of libmuon.so (declared in include/muon.h): argument checks, the shape
// grouping and workspace plan, TMA descriptors, and the launch sequence of one
// Muon step.  All arithmetic runs in the kernels; this file only plans and
// enqueues.
//
// One step enqueues, on the caller's stream and without any host sync:
//   memset of the per-matrix arrival counters
//   momentum_norm_kernel   (one launch per <= 192 matrices)
//   k x { Gram, Poly, Update }   tcgen05 kernels, every shape group in one launch
//                                (or fp32 CUDA-core kernels, one per group, in
//                                the reference mode); the last Update writes the
//                                parameters itself when the shapes allow it.  When
//                                every matrix fits one 256 x 256 tile, one
//                                ns_small_kernel launch runs all k iterations instead.
//   param_write_kernel     (one launch per <= 192 matrices, only when not fused)
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <new>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "muon.h"
#include "muon_internal.h"

using namespace muon;

namespace {

constexpr unsigned long long kTimeoutNs = 4000000000ull;  // bounded waits give up after 4 s

// An NVTX range around the host-side enqueue of a call or a stage: it names the stages on a
// profiler's timeline and costs nothing when no profiler is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int round_up(long long x, int a) { return static_cast<int>((x + a - 1) / a * a); }

struct GroupPlan {
  int m, n, mp, np, cnt;
  std::vector<int> mats;      // caller indices, in caller order
  size_t off_x[2], off_a, off_b;
  int scal_base;
  CUtensorMap tm_x[2], tm_a, tm_b;   // row views (K-major operand tiles)
  CUtensorMap tt_x[2], tt_a, tt_b;   // chunked views (MN-major operand tiles)
  CUtensorMap ts_x[2], ts_a, ts_b;   // store views (32 x 32 epilogue tiles)
};

struct Plan {
  std::vector<GroupPlan> groups;
  std::vector<int> mat_group, mat_slot, scal_idx;
  std::vector<int> ew_ntiles;
  size_t off_status, off_deps, off_scal, off_norms, off_partials;
  size_t total;
};

bool shapes_ok(const muon_shape_t* shapes, int n) {
  if (shapes == nullptr || n < 1 || n > MUON_MAX_MATRICES) return false;
  for (int i = 0; i < n; ++i) {
    if (shapes[i].rows < 1 || shapes[i].cols < 1) return false;
    if (shapes[i].rows > (1 << 20) || shapes[i].cols > (1 << 20)) return false;
  }
  return true;
}

void make_plan(const muon_shape_t* shapes, int n, muon_mode_t mode, Plan* P) {
  const size_t elem = (mode == MUON_MODE_FAST) ? 2 : 4;
  std::map<std::pair<long long, long long>, int> key_to_group;
  P->groups.clear();
  P->mat_group.assign(n, 0);
  P->mat_slot.assign(n, 0);
  for (int i = 0; i < n; ++i) {
    const long long r = shapes[i].rows, c = shapes[i].cols;
    const long long m = std::min(r, c), nn = std::max(r, c);
    auto key = std::make_pair(m, nn);
    auto it = key_to_group.find(key);
    int g;
    if (it == key_to_group.end()) {
      g = static_cast<int>(P->groups.size());
      key_to_group[key] = g;
      GroupPlan gp{};
      gp.m = static_cast<int>(m);
      gp.n = static_cast<int>(nn);
      gp.mp = round_up(m, kPad);
      gp.np = round_up(nn, kPad);
      gp.cnt = 0;
      P->groups.push_back(gp);
    } else {
      g = it->second;
    }
    P->groups[g].mats.push_back(i);
    P->groups[g].cnt++;
  }
  // Larger per-matrix work first: the round-robin tile list then ends on the
  // cheaper tiles, which evens out the tail of each launch.
  std::stable_sort(P->groups.begin(), P->groups.end(), [](const GroupPlan& a, const GroupPlan& b) {
    return static_cast<long long>(a.mp) * a.np > static_cast<long long>(b.mp) * b.np;
  });
  P->scal_idx.assign(n, 0);
  int base = 0;
  for (size_t g = 0; g < P->groups.size(); ++g) {
    GroupPlan& gp = P->groups[g];
    gp.scal_base = base;
    for (int s = 0; s < gp.cnt; ++s) {
      P->mat_group[gp.mats[s]] = static_cast<int>(g);
      P->mat_slot[gp.mats[s]] = s;
      P->scal_idx[gp.mats[s]] = base + s;
    }
    base += gp.cnt;
  }
  P->ew_ntiles.assign(n, 0);
  for (int i = 0; i < n; ++i) {
    const GroupPlan& gp = P->groups[P->mat_group[i]];
    P->ew_ntiles[i] = (gp.mp / kEwTileR) * (gp.np / kEwTileC);
  }
  // One partial sum per (CTA, warp) of the momentum/norm kernel, one CTA per tile; launches in
  // sequence reuse the buffer, so the whole set bounds it.
  size_t parts = 0;
  for (int i = 0; i < n; ++i) parts += static_cast<size_t>(P->ew_ntiles[i]) * (kEwThreads / 32);
  size_t off = 0;
  P->off_status = off;
  off = align_up(off + 64, 1024);
  // the single-launch schedule's completion counters, [3 k][n] for k up to 64
  P->off_deps = off;
  off = align_up(P->off_deps + sizeof(unsigned int) * 3 * 64 * static_cast<size_t>(n), 1024);
  P->off_scal = off;
  off = align_up(off + sizeof(float) * 2 * n, 1024);
  P->off_norms = off;
  off = align_up(off + sizeof(float) * n, 1024);
  P->off_partials = off;
  off = align_up(off + sizeof(float) * parts, 1024);
  for (GroupPlan& gp : P->groups) {
    const size_t xb = static_cast<size_t>(gp.cnt) * gp.mp * gp.np * elem;
    const size_t ab = static_cast<size_t>(gp.cnt) * gp.mp * gp.mp * elem;
    gp.off_x[0] = off; off = align_up(off + xb, 1024);
    gp.off_x[1] = off; off = align_up(off + xb, 1024);
    gp.off_a = off;    off = align_up(off + ab, 1024);
    gp.off_b = off;    off = align_up(off + ab, 1024);
  }
  P->total = off;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row view of a [cnt][rows][cols] bf16 buffer: one box is 64 columns x 128 rows of one
// matrix (16 KB, 128-byte swizzle), the K-major operand tile of one CTA and k slice.
bool encode_rows(CUtensorMap* map, void* base, int cols, int rows, int cnt) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(cnt)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(cols) * rows * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Store view of a [cnt][rows][cols] bf16 buffer: one box is a 32 x 32 tile of one matrix
// (64-byte rows, 64-byte swizzle), one epilogue chunk.
bool encode_store(CUtensorMap* map, void* base, int cols, int rows, int cnt) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(cnt)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(cols) * rows * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Chunked view of the same buffer, [cnt][cols/64][rows][64]: one box is 64 rows (the k
// slice) of two neighbouring 64-column chunks, stored chunk after chunk (2 x 8 KB), the
// MN-major operand tile of one CTA and k slice.
bool encode_chunks(CUtensorMap* map, void* base, int cols, int rows, int cnt) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(cols / 64),
                        static_cast<cuuint64_t>(cnt)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(cols) * 2, 128, static_cast<cuuint64_t>(cols) * rows * 2};
  cuuint32_t box[4] = {64, 64, 2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev_) == cudaSuccess && prev_ != dev) {
      if (cudaSetDevice(dev) == cudaSuccess) switched_ = true;
    }
  }
  ~DeviceGuard() {
    if (switched_) cudaSetDevice(prev_);
  }

 private:
  int prev_ = -1;
  bool switched_ = false;
};

bool hp_ok(const muon_hparams_t* hp, bool need_momentum) {
  if (hp == nullptr) return false;
  if (hp->ns_steps < 0 || hp->ns_steps > 64) return false;
  if (!std::isfinite(hp->eps) || hp->eps < 0.0f) return false;
  if (!std::isfinite(hp->a) || !std::isfinite(hp->b) || !std::isfinite(hp->c)) return false;
  if (need_momentum) {
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->weight_decay)) return false;
    if (!std::isfinite(hp->beta) || hp->beta < 0.0f || hp->beta > 1.0f) return false;
  }
  return true;
}

}  // namespace

struct muon_ctx {
  int device = 0;
  int num_sms = 0;
  muon_dtype_t dtype = MUON_BF16;
  muon_mode_t mode = MUON_MODE_FAST;
  int n = 0;
  std::vector<muon_shape_t> shapes;
  Plan plan;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  unsigned int* d_status = nullptr;
  float* d_scal = nullptr;
  float* d_partials = nullptr;
  float* d_norms = nullptr;   // ||U_i||_F in caller order
  bool fuse_shapes_ok = false;  // every group's real dimensions are multiples of 32, n <= kTcMaxFused
  int schedule = MUON_SCHEDULE_AUTO;
  // launch parameter blocks (tens of KB), reused by every call on this handle
  EwParams ew;
  WrParams wr;
  TcParams tc;
  SmallParams sm;
  NsParams ns;
  // tracing (muon_profile_begin / muon_profile_end)
  int prof_steps_left = 0;
  std::vector<std::pair<int, cudaEvent_t>> prof_events;  // kind (-1: start of a call), event
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Record a tracing event after a launch of `kind` (or at the start of a call, kind -1).
void trace(muon_ctx* h, int kind, cudaStream_t st) {
  if (h->prof_steps_left <= 0) return;
  cudaEvent_t ev;
  if (cudaEventCreate(&ev) != cudaSuccess) return;
  if (cudaEventRecord(ev, st) != cudaSuccess) {
    cudaEventDestroy(ev);
    return;
  }
  h->prof_events.emplace_back(kind, ev);
}

void trace_call_end(muon_ctx* h) {
  if (h->prof_steps_left > 0) --h->prof_steps_left;
}

bool small_path(const muon_ctx* h, int k);

// Whether the k iterations run as one launch (all stages, per-matrix completion counters)
// rather than one launch per stage: FAST mode, at most kTcMaxGroups shape groups, not the
// small-matrix kernel's sets, and the handle's schedule allows it.
bool fused_possible(const muon_ctx* h, int k) {
  return h->mode == MUON_MODE_FAST && k >= 1 && !h->plan.groups.empty() &&
         h->plan.groups.size() <= static_cast<size_t>(kTcMaxGroups) && !small_path(h, k);
}
bool fused_schedule(const muon_ctx* h, int k) {
  if (!fused_possible(h, k)) return false;
  if (h->schedule == MUON_SCHEDULE_AUTO) {
    // AUTO takes the single launch for sets whose every shape group is at most 768 wide, whose
    // short stages spend the largest share of their time at launch boundaries: on the
    // GPT-2-small set it runs within 1 % of the staged schedule (faster in short runs, slower in
    // sustained ones) with one launch per step instead of 3 k.  Wider sets (d24's 1536) measured
    // faster staged.
    for (const GroupPlan& gp : h->plan.groups)
      if (gp.mp > 768) return false;
    return true;
  }
  return h->schedule == MUON_SCHEDULE_FUSED || h->schedule == MUON_SCHEDULE_SPLIT;
}

// Tile tables of one momentum/norm launch (matrices b .. b+cnt-1), without the pointers and the
// hyper-parameters: one CTA per tile, the matrices' tiles back to back.
void front_tables(const Plan& P, const std::vector<muon_shape_t>& shapes, int b, int cnt, EwParams* prm) {
  std::memset(prm, 0, sizeof(*prm));
  prm->nmat = cnt;
  int tiles = 0, parts = 0;
  for (int j = 0; j < cnt; ++j) {
    const int i = b + j;
    const GroupPlan& gp = P.groups[P.mat_group[i]];
    EwMat& m = prm->mat[j];
    m.rows = static_cast<int>(shapes[i].rows);
    m.cols = static_cast<int>(shapes[i].cols);
    m.mp = gp.mp;
    m.np = gp.np;
    m.trans = shapes[i].rows > shapes[i].cols ? 1 : 0;
    m.tile_begin = tiles;
    m.tiles_c = gp.np / kEwTileC;
    m.ntiles = P.ew_ntiles[i];
    m.scal_idx = P.scal_idx[i];
    m.caller_idx = i;
    m.nparts = m.ntiles;
    m.part_begin = parts;
    parts += m.nparts;
    tiles += m.ntiles;
  }
  prm->total_tiles = tiles;
  prm->grid = parts;
}

// The elementwise front end (momentum + norm + orientation) over all matrices.
cudaError_t enqueue_front(muon_ctx* h, const void* const* src, void* const* mom, const muon_hparams_t* hp,
                          cudaStream_t st, int* launches) {
  NvtxRange range("muon: momentum + norm");
  const Plan& P = h->plan;
  const Dtype io = (h->dtype == MUON_BF16) ? kBF16 : kF32;
  const Dtype xt = (h->mode == MUON_MODE_FAST) ? kBF16 : kF32;
  cudaError_t e = cudaSuccess;
  if (fused_schedule(h, hp->ns_steps)) {
    // the single-launch schedule's stage completion counters start at zero
    e = cudaMemsetAsync(h->ws + P.off_deps, 0, sizeof(unsigned int) * 3 * hp->ns_steps * static_cast<size_t>(h->n), st);
    if (e != cudaSuccess) return e;
  }
  trace(h, -1, st);  // start of the traced kernel sequence of this call
  EwParams& prm = h->ew;
  for (int b = 0; b < h->n; b += kEwMatsPerLaunch) {
    const int cnt = std::min(kEwMatsPerLaunch, h->n - b);
    // 16-byte aligned rows everywhere: vector accesses (else element by element)
    int vec_ok = 1;
    for (int j = 0; j < cnt; ++j) {
      const int i = b + j;
      const int vmul = (h->dtype == MUON_BF16) ? 8 : 4;
      if (!aligned16(src[i]) || (mom && !aligned16(mom[i])) || (h->shapes[i].cols % vmul) != 0) vec_ok = 0;
    }
    front_tables(P, h->shapes, b, cnt, &prm);
    prm.beta = hp->beta;
    prm.eps = hp->eps;
    prm.nesterov = hp->nesterov ? 1 : 0;
    prm.partials = h->d_partials;
    prm.scal = h->d_scal;
    prm.norms = h->d_norms;
    prm.status = h->d_status;
    for (int j = 0; j < cnt; ++j) {
      const int i = b + j;
      const GroupPlan& gp = P.groups[P.mat_group[i]];
      const size_t elem = (h->mode == MUON_MODE_FAST) ? 2 : 4;
      EwMat& m = prm.mat[j];
      m.src = src[i];
      m.mom = mom ? mom[i] : nullptr;
      m.x = h->ws + gp.off_x[0] + static_cast<size_t>(P.mat_slot[i]) * gp.mp * gp.np * elem;
    }
    prm.vec_ok = vec_ok;
    e = launch_momentum_norm(prm, io, xt, st);
    if (e != cudaSuccess) return e;
    ++*launches;
    trace(h, MUON_KERNEL_MOMENTUM_NORM, st);
  }
  return cudaSuccess;
}

// Tile tables of the single-launch schedule (everything but the tensor maps, pointers and
// hyper-parameters): Update tiles 256 x 512 when every group's padded width allows it (except in
// the iteration that writes W), Gram and Poly two upper blocks per tile, and the first tile of
// each (stage, group) within an iteration.
void fused_tables(const Plan& P, int nslots, int k, bool fuse_write, NsParams* q) {
  std::memset(q, 0, sizeof(*q));
  const int ng = static_cast<int>(P.groups.size());
  bool wide = true;
  for (const GroupPlan& gp : P.groups) wide = wide && gp.np % 512 == 0;
  q->upd_tw[0] = wide ? 512 : 256;
  q->upd_tw[1] = (wide && !fuse_write) ? 512 : 256;  // the Update that writes W keeps 256-wide tiles
  // Gram and Poly keep one 256 x 256 block per tile: two blocks per tile (256 x 512, one
  // accumulator, half of the epilogue exposed) measured 13 % (Gram) and 20 % (Poly) slower on d24
  q->sym_wide = 0;
  for (int g = 0; g < ng; ++g) {
    const GroupPlan& gp = P.groups[g];
    NsGroup& G = q->g[g];
    G.cnt = gp.cnt;
    G.mp = gp.mp;
    G.np = gp.np;
    G.m_real = gp.m;
    G.n_real = gp.n;
    G.scal_base = gp.scal_base;
    G.tdim = gp.mp / 256;
  }
  int iter_tiles[2] = {0, 0};
  for (int L = 0; L < 2; ++L) {
    int off = 0;
    for (int kind = kGram; kind <= kUpdate; ++kind) {
      for (int g = 0; g < ng; ++g) {
        const GroupPlan& gp = P.groups[g];
        const int T = gp.mp / 256;
        const int tpm = kind == kUpdate ? T * (gp.np / q->upd_tw[L]) : sym_tiles(T, q->sym_wide != 0);
        q->begin[L][kind][g] = off;
        off += tpm * gp.cnt;
      }
      q->begin[L][kind][ng] = off;
    }
    iter_tiles[L] = off;
  }
  q->fuse_write = fuse_write ? 1 : 0;
  q->ngroups = ng;
  q->k = k;
  q->nslots = nslots;
  q->tiles_iter = k > 1 ? iter_tiles[0] : iter_tiles[1];
  q->total_tiles = (k - 1) * iter_tiles[0] + iter_tiles[1];
}

// The parameter write can ride on the last Update launch when the parameters are bf16,
// every real dimension is a multiple of 32 (epilogue chunks are all real or all padding),
// the pointers fit the launch parameters and every destination is 16-byte aligned.
// All k >= 1 iterations in one kernel when every group pads to one 256 x 256 tile.
bool small_path(const muon_ctx* h, int k) {
  if (h->mode != MUON_MODE_FAST || k < 1 || h->plan.groups.empty() ||
      h->plan.groups.size() > static_cast<size_t>(kTcMaxGroups))
    return false;
  for (const GroupPlan& gp : h->plan.groups)
    if (gp.mp != kSmallTile || gp.np != kSmallTile) return false;
  return true;
}

bool write_fusable(const muon_ctx* h, void* const* dst, int k) {
  if (h->mode != MUON_MODE_FAST || h->dtype != MUON_BF16 || k < 1 || !h->fuse_shapes_ok) return false;
  for (int i = 0; i < h->n; ++i)
    if ((reinterpret_cast<uintptr_t>(dst[i]) & 15u) != 0) return false;
  return true;
}

// k Newton-Schulz iterations.  When *fused comes back true, the last Update has also
// written dst (the parameter update, or O itself when store_only) and the separate
// write kernel must not run.
cudaError_t enqueue_ns(muon_ctx* h, const muon_hparams_t* hp, cudaStream_t st, int* launches, void* const* dst,
                       bool store_only, bool* fused) {
  const Plan& P = h->plan;
  const int k = hp->ns_steps;
  if (small_path(h, k)) {
    // every matrix fits one 256 x 256 tile: all k iterations in one launch, X_k into X[k & 1]
    NvtxRange range("muon: Newton-Schulz, all iterations (small matrices)");
    *fused = false;
    SmallParams& sp = h->sm;
    std::memset(&sp, 0, sizeof(sp));
    int mats = 0;
    for (size_t g = 0; g < P.groups.size(); ++g) {
      const GroupPlan& gp = P.groups[g];
      SmGroup& G = sp.g[g];
      G.tm_row = gp.tm_x[0];
      G.tm_col = gp.tt_x[0];
      G.out = h->ws + gp.off_x[k & 1];
      G.mat_begin = mats;
      G.cnt = gp.cnt;
      G.scal_base = gp.scal_base;
      G.m_real = gp.m;
      mats += gp.cnt;
    }
    sp.ngroups = static_cast<int>(P.groups.size());
    sp.total = mats;
    sp.k = k;
    sp.a = hp->a;
    sp.b = hp->b;
    sp.c = hp->c;
    sp.scal = h->d_scal;
    sp.status = h->d_status;
    sp.timeout_ns = kTimeoutNs;
    cudaError_t e = launch_ns_small(sp, h->num_sms, st);
    if (e != cudaSuccess) return e;
    ++*launches;
    trace(h, MUON_KERNEL_NS_SMALL, st);
    return cudaSuccess;
  }
  const bool fuse = write_fusable(h, dst, k);
  *fused = fuse;
  if (fused_schedule(h, k)) {
    // every iteration in one launch: tiles of all 3k stages in one list, per-matrix counters
    NvtxRange range("muon: Newton-Schulz, every iteration in one launch");
    NsParams& q = h->ns;
    fused_tables(P, h->n, k, fuse, &q);
    const int ng = static_cast<int>(P.groups.size());
    for (int g = 0; g < ng; ++g) {
      const GroupPlan& gp = P.groups[g];
      NsGroup& G = q.g[g];
      for (int b = 0; b < 2; ++b) {
        G.x_row[b] = gp.tm_x[b];
        G.x_chk[b] = gp.tt_x[b];
        G.x_st[b] = gp.ts_x[b];
      }
      G.a_row = gp.tm_a;
      G.a_chk = gp.tt_a;
      G.a_st = gp.ts_a;
      G.b_row = gp.tm_b;
      G.b_chk = gp.tt_b;
      G.b_st = gp.ts_b;
    }
    q.a = hp->a;
    q.b = hp->b;
    q.c = hp->c;
    q.scal = h->d_scal;
    q.status = h->d_status;
    q.deps = reinterpret_cast<unsigned int*>(h->ws + P.off_deps);
    q.timeout_ns = kTimeoutNs;
    if (fuse) {
      q.w_decay = store_only ? 0.0f : 1.0f - hp->lr * hp->weight_decay;
      for (const GroupPlan& gp : P.groups) {
        for (int sl = 0; sl < gp.cnt; ++sl) {
          const int i = gp.mats[sl], slot = gp.scal_base + sl;
          const float r = static_cast<float>(h->shapes[i].rows), c = static_cast<float>(h->shapes[i].cols);
          q.wptr[slot] = dst[i];
          q.wcoef[slot] = store_only ? 1.0f : -hp->lr * std::sqrt(std::max(1.0f, r / c));
          q.wtrans[slot] = h->shapes[i].rows > h->shapes[i].cols ? 1 : 0;
        }
      }
    }
    if (h->schedule != MUON_SCHEDULE_SPLIT) {
      q.t_begin = 0;
      q.t_end = q.total_tiles;
      cudaError_t e = launch_ns_fused(q, h->num_sms, st);
      if (e != cudaSuccess) return e;
      ++*launches;
      trace(h, MUON_KERNEL_NS_FUSED, st);
      return cudaSuccess;
    }
    // the same tiles, one launch per stage (the stage boundaries then come from stream order)
    for (int s = 0; s < 3 * k; ++s) {
      const int it = s / 3, kind = s % 3, L = (it == k - 1) ? 1 : 0;
      const int base = it * q.tiles_iter;
      q.t_begin = base + q.begin[L][kind][0];
      q.t_end = base + q.begin[L][kind][q.ngroups];
      cudaError_t e = launch_ns_fused(q, h->num_sms, st);
      if (e != cudaSuccess) return e;
      ++*launches;
      trace(h, MUON_KERNEL_GRAM + kind, st);
    }
    return cudaSuccess;
  }
  for (int t = 1; t <= k; ++t) {
    const int cur = (t - 1) & 1, nxt = t & 1;
    if (h->mode == MUON_MODE_FAST) {
      for (int kind = kGram; kind <= kUpdate; ++kind) {
        NvtxRange range(kind == kGram ? "muon: Gram" : kind == kPoly ? "muon: polynomial" : "muon: update");
        for (size_t g0 = 0; g0 < P.groups.size(); g0 += kTcMaxGroups) {
          TcParams& prm = h->tc;
          std::memset(&prm, 0, sizeof(prm));
          const int ng = static_cast<int>(std::min<size_t>(kTcMaxGroups, P.groups.size() - g0));
          prm.ngroups = ng;
          prm.kind = kind;
          // Update takes 256 x 512 pair tiles when every group's padded width allows them:
          // each k slice of B' then feeds 512 output columns instead of 256.  Its epilogue reads
          // the single accumulator into registers before any store.  The Update that writes the
          // parameters does so only when its k loops are long (the flop-weighted mean of m at
          // least 2048): the parameter write of one tile (W read from and written to HBM) then
          // finishes inside the next tile's MMAs, where at m = 1536 it does not (measured: 3.4 %
          // faster on the l38b set, mean m 3028; 2.5 % slower on d24).
          bool wide = kind == kUpdate;
          double wsum = 0.0, wm = 0.0;
          for (int gi = 0; gi < ng; ++gi) {
            const GroupPlan& gp = P.groups[g0 + gi];
            wide = wide && gp.np % 512 == 0;
            const double f = static_cast<double>(gp.cnt) * gp.mp * gp.mp * gp.np;
            wsum += f;
            wm += f * gp.mp;
          }
          if (t == k && fuse) wide = wide && wm >= 2048.0 * wsum;
          prm.wide = wide ? 1 : 0;
          const int tw = wide ? 512 : 256;
          // The first iteration reads the unnormalised U: Gram scales by 1/(||U||+eps)^2 and
          // Update by 1/(||U||+eps); Poly works on the already normalised A.
          prm.use_scal = (t == 1 && kind != kPoly) ? 1 : 0;
          prm.scal = h->d_scal;
          prm.status = h->d_status;
          prm.timeout_ns = kTimeoutNs;
          if (kind == kGram) { prm.c_acc = 1.0f; prm.c_aux = 0.0f; }
          // Poly writes B' = a I + b A + c A A (the a X term of the update folded into B'),
          // so Update is the plain product X' = s * (B' X).
          if (kind == kPoly) { prm.c_acc = hp->c; prm.c_aux = hp->b; prm.c_diag = hp->a; }
          if (kind == kUpdate) { prm.c_acc = 1.0f; prm.c_aux = 0.0f; }
          if (kind == kUpdate && t == k && fuse) {
            prm.fuse_write = 1;
            prm.w_decay = store_only ? 0.0f : 1.0f - hp->lr * hp->weight_decay;
            for (const GroupPlan& gp : P.groups) {
              for (int sl = 0; sl < gp.cnt; ++sl) {
                const int i = gp.mats[sl], slot = gp.scal_base + sl;
                const float r = static_cast<float>(h->shapes[i].rows), c = static_cast<float>(h->shapes[i].cols);
                prm.wptr[slot] = dst[i];
                prm.wcoef[slot] = store_only ? 1.0f : -hp->lr * std::sqrt(std::max(1.0f, r / c));
                prm.wtrans[slot] = h->shapes[i].rows > h->shapes[i].cols ? 1 : 0;
              }
            }
          }
          int tiles = 0;
          for (int gi = 0; gi < ng; ++gi) {
            const GroupPlan& gp = P.groups[g0 + gi];
            TcGroup& G = prm.g[gi];
            G.cnt = gp.cnt;
            G.mp = gp.mp;
            G.np = gp.np;
            G.scal_base = gp.scal_base;
            G.tile_begin = tiles;
            const int T = gp.mp / 256;
            if (kind == kGram) {
              G.tm_a = gp.tm_x[cur];
              G.tm_at = gp.tt_x[cur];
              G.tm_b = gp.tm_x[cur];
              G.tm_bt = gp.tt_x[cur];
              G.tm_out = gp.ts_a;
              G.out = h->ws + gp.off_a;
              G.tiles_per_mat = T * (T + 1) / 2;  // 256 x 256 pair tiles on or above the diagonal
              G.kblocks = gp.np / kTcBK;
              G.tdim = T;
              G.out_ld = gp.mp;
              G.m_real = gp.m;
            } else if (kind == kPoly) {
              G.tm_a = gp.tm_a;
              G.tm_at = gp.tt_a;
              G.tm_b = gp.tm_a;
              G.tm_bt = gp.tt_a;
              G.tm_out = gp.ts_b;
              G.out = h->ws + gp.off_b;
              G.tm_aux = gp.ts_a;
              G.tiles_per_mat = T * (T + 1) / 2;
              G.m_real = gp.m;
              G.kblocks = gp.mp / kTcBK;
              G.tdim = T;
              G.out_ld = gp.mp;
            } else {
              G.tm_a = gp.tm_b;
              G.tm_at = gp.tt_b;
              G.tm_b = gp.tm_x[cur];
              G.tm_bt = gp.tt_x[cur];
              G.tm_out = gp.ts_x[nxt];
              G.out = h->ws + gp.off_x[nxt];
              G.tiles_per_mat = (gp.mp / 256) * (gp.np / tw);  // 256 x tw pair tiles
              G.kblocks = gp.mp / kTcBK;
              G.tdim = gp.np / tw;
              G.out_ld = gp.np;
              G.m_real = gp.m;
              G.n_real = gp.n;
            }
            tiles += G.tiles_per_mat * gp.cnt;
          }
          prm.total_tiles = tiles;
          cudaError_t e = launch_tc_gemm(prm, h->num_sms, st);
          if (e != cudaSuccess) return e;
          ++*launches;
          trace(h, MUON_KERNEL_GRAM + kind, st);
        }
      }
    } else {
      for (int kind = kGram; kind <= kUpdate; ++kind) {
        NvtxRange range(kind == kGram ? "muon: Gram" : kind == kPoly ? "muon: polynomial" : "muon: update");
        for (const GroupPlan& gp : P.groups) {
          SgParams s{};
          const float* x = reinterpret_cast<const float*>(h->ws + gp.off_x[cur]);
          float* xn = reinterpret_cast<float*>(h->ws + gp.off_x[nxt]);
          float* A = reinterpret_cast<float*>(h->ws + gp.off_a);
          float* B = reinterpret_cast<float*>(h->ws + gp.off_b);
          s.cnt = gp.cnt;
          s.scal = h->d_scal;
          s.scal_base = gp.scal_base;
          const long long xs = static_cast<long long>(gp.mp) * gp.np, as = static_cast<long long>(gp.mp) * gp.mp;
          if (kind == kGram) {
            s.a = x; s.b = x; s.c = A; s.aux = nullptr;
            s.M = gp.mp; s.N = gp.mp; s.K = gp.np;
            s.lda = gp.np; s.ldb = gp.np; s.ldc = gp.mp;
            s.sa = xs; s.sb = xs; s.sc = as;
            s.b_trans = 1; s.c_acc = 1.0f; s.c_aux = 0.0f;
            s.scal_mode = (t == 1) ? 1 : 0;
          } else if (kind == kPoly) {
            s.a = A; s.b = A; s.c = B; s.aux = A;
            s.M = gp.mp; s.N = gp.mp; s.K = gp.mp;
            s.lda = gp.mp; s.ldb = gp.mp; s.ldc = gp.mp;
            s.sa = as; s.sb = as; s.sc = as;
            s.b_trans = 0; s.c_acc = hp->c; s.c_aux = hp->b;
            s.c_diag = hp->a; s.diag_n = gp.m;  // B' = a I + b A + c A A
            s.scal_mode = 0;
          } else {
            s.a = B; s.b = x; s.c = xn; s.aux = nullptr;
            s.M = gp.mp; s.N = gp.np; s.K = gp.mp;
            s.lda = gp.mp; s.ldb = gp.np; s.ldc = gp.np;
            s.sa = as; s.sb = xs; s.sc = xs;
            s.b_trans = 0; s.c_acc = 1.0f; s.c_aux = 0.0f;
            s.scal_mode = (t == 1) ? 2 : 0;
          }
          cudaError_t e = launch_sgemm(s, st);
          if (e != cudaSuccess) return e;
          ++*launches;
          trace(h, MUON_KERNEL_SGEMM, st);
        }
      }
    }
  }
  return cudaSuccess;
}

cudaError_t enqueue_back(muon_ctx* h, void* const* dst, const muon_hparams_t* hp, bool store_only, cudaStream_t st,
                         int* launches) {
  NvtxRange range("muon: parameter write");
  const Plan& P = h->plan;
  const Dtype io = (h->dtype == MUON_BF16) ? kBF16 : kF32;
  const Dtype xt = (h->mode == MUON_MODE_FAST) ? kBF16 : kF32;
  const size_t elem = (h->mode == MUON_MODE_FAST) ? 2 : 4;
  const int fin = hp->ns_steps & 1;
  WrParams& prm = h->wr;
  for (int b = 0; b < h->n; b += kEwMatsPerLaunch) {
    const int cnt = std::min(kEwMatsPerLaunch, h->n - b);
    std::memset(&prm, 0, sizeof(prm));
    prm.nmat = cnt;
    prm.lr = hp->lr;
    prm.wd = hp->weight_decay;
    prm.store_only = store_only ? 1 : 0;
    prm.use_alpha = (hp->ns_steps == 0) ? 1 : 0;
    prm.scal = h->d_scal;
    int vec_ok = 1, tiles = 0;
    for (int j = 0; j < cnt; ++j) {
      const int i = b + j;
      const GroupPlan& gp = P.groups[P.mat_group[i]];
      WrMat& m = prm.mat[j];
      m.w = dst[i];
      m.x = h->ws + gp.off_x[fin] + static_cast<size_t>(P.mat_slot[i]) * gp.mp * gp.np * elem;
      m.rows = static_cast<int>(h->shapes[i].rows);
      m.cols = static_cast<int>(h->shapes[i].cols);
      m.mp = gp.mp;
      m.np = gp.np;
      m.trans = m.rows > m.cols ? 1 : 0;
      m.tile_begin = tiles;
      m.tiles_c = (gp.n + kEwTileC - 1) / kEwTileC;
      m.scal_idx = P.scal_idx[i];
      m.shape_scale = std::sqrt(std::max(1.0f, static_cast<float>(m.rows) / static_cast<float>(m.cols)));
      tiles += ((gp.m + kEwTileR - 1) / kEwTileR) * m.tiles_c;
      const int vmul = (h->dtype == MUON_BF16) ? 8 : 4;
      if (!aligned16(m.w) || (m.cols % vmul) != 0) vec_ok = 0;
    }
    prm.vec_ok = vec_ok;
    prm.total_ctas = tiles;
    cudaError_t e = launch_param_write(prm, io, xt, st);
    if (e != cudaSuccess) return e;
    ++*launches;
    trace(h, MUON_KERNEL_WRITE, st);
  }
  return cudaSuccess;
}

int launches_for(const muon_ctx* h, int k) {
  const int chunks = (h->n + kEwMatsPerLaunch - 1) / kEwMatsPerLaunch;
  const int front = 2 * chunks;  // momentum/norm and the norms' finishing pass, per 192 matrices
  if (small_path(h, k)) return front + 1 + chunks;
  const bool fused_write = h->mode == MUON_MODE_FAST && h->dtype == MUON_BF16 && k >= 1 && h->fuse_shapes_ok;
  if (fused_schedule(h, k))
    return front + (h->schedule == MUON_SCHEDULE_SPLIT ? 3 * k : 1) + (fused_write ? 0 : chunks);
  const int ng = static_cast<int>(h->plan.groups.size());
  const int per_stage = (h->mode == MUON_MODE_FAST) ? (ng + kTcMaxGroups - 1) / kTcMaxGroups : ng;
  return front + 3 * k * per_stage + (fused_write ? 0 : chunks);
}

}  // namespace

extern "C" {

const char* muon_status_string(muon_status_t s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_INVALID_ARG: return "MUON_ERR_INVALID_ARG";
    case MUON_ERR_UNSUPPORTED: return "MUON_ERR_UNSUPPORTED";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA";
    case MUON_ERR_WORKSPACE: return "MUON_ERR_WORKSPACE";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT";
    case MUON_ERR_DEVICE_STATUS: return "MUON_ERR_DEVICE_STATUS";
    case MUON_ERR_NO_DEVICE: return "MUON_ERR_NO_DEVICE";
  }
  return "MUON_ERR_UNKNOWN";
}

muon_status_t muon_workspace_size(const muon_shape_t* shapes, int n, muon_dtype_t dtype, muon_mode_t mode,
                                  size_t* bytes) {
  if (bytes == nullptr || !shapes_ok(shapes, n)) return MUON_ERR_INVALID_ARG;
  if ((dtype != MUON_BF16 && dtype != MUON_FP32) || (mode != MUON_MODE_FAST && mode != MUON_MODE_FP32_REF))
    return MUON_ERR_INVALID_ARG;
  Plan P;
  make_plan(shapes, n, mode, &P);
  *bytes = P.total;
  return MUON_OK;
}

muon_status_t muon_create(muon_handle_t* handle, const muon_shape_t* shapes, int n, muon_dtype_t dtype,
                          muon_mode_t mode, void* workspace, size_t ws_bytes) {
  if (handle == nullptr) return MUON_ERR_INVALID_ARG;
  *handle = nullptr;
  if (!shapes_ok(shapes, n)) return MUON_ERR_INVALID_ARG;
  if ((dtype != MUON_BF16 && dtype != MUON_FP32) || (mode != MUON_MODE_FAST && mode != MUON_MODE_FP32_REF))
    return MUON_ERR_INVALID_ARG;
  int dev = -1, ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev < 1 || cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_NO_DEVICE;
  }
  int major = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10) return MUON_ERR_UNSUPPORTED;
  muon_ctx* h = new (std::nothrow) muon_ctx();
  if (h == nullptr) return MUON_ERR_INVALID_ARG;
  h->device = dev;
  h->num_sms = sms;
  h->dtype = dtype;
  h->mode = mode;
  h->n = n;
  h->shapes.assign(shapes, shapes + n);
  make_plan(shapes, n, mode, &h->plan);
  h->fuse_shapes_ok = n <= kTcMaxFused;
  for (const GroupPlan& gp : h->plan.groups)
    if (gp.m % 32 != 0 || gp.n % 32 != 0) h->fuse_shapes_ok = false;
  if (workspace == nullptr || ws_bytes < h->plan.total || (reinterpret_cast<uintptr_t>(workspace) & 1023u) != 0) {
    delete h;
    return MUON_ERR_WORKSPACE;
  }
  h->ws = static_cast<char*>(workspace);
  h->ws_bytes = ws_bytes;
  h->d_status = reinterpret_cast<unsigned int*>(h->ws + h->plan.off_status);
  h->d_scal = reinterpret_cast<float*>(h->ws + h->plan.off_scal);
  h->d_partials = reinterpret_cast<float*>(h->ws + h->plan.off_partials);
  h->d_norms = reinterpret_cast<float*>(h->ws + h->plan.off_norms);
  if (cudaMemset(workspace, 0, h->plan.total) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MUON_ERR_CUDA;
  }
  if (mode == MUON_MODE_FAST) {
    for (GroupPlan& gp : h->plan.groups) {
      bool ok = true;
      for (int b = 0; b < 2; ++b)
        ok = ok && encode_rows(&gp.tm_x[b], h->ws + gp.off_x[b], gp.np, gp.mp, gp.cnt) &&
             encode_chunks(&gp.tt_x[b], h->ws + gp.off_x[b], gp.np, gp.mp, gp.cnt) &&
             encode_store(&gp.ts_x[b], h->ws + gp.off_x[b], gp.np, gp.mp, gp.cnt);
      ok = ok && encode_rows(&gp.tm_a, h->ws + gp.off_a, gp.mp, gp.mp, gp.cnt) &&
           encode_chunks(&gp.tt_a, h->ws + gp.off_a, gp.mp, gp.mp, gp.cnt) &&
           encode_store(&gp.ts_a, h->ws + gp.off_a, gp.mp, gp.mp, gp.cnt) &&
           encode_rows(&gp.tm_b, h->ws + gp.off_b, gp.mp, gp.mp, gp.cnt) &&
           encode_chunks(&gp.tt_b, h->ws + gp.off_b, gp.mp, gp.mp, gp.cnt) &&
           encode_store(&gp.ts_b, h->ws + gp.off_b, gp.mp, gp.mp, gp.cnt);
      if (!ok) {
        delete h;
        return MUON_ERR_CUDA;
      }
    }
  }
  if (std::getenv("MUON_DEBUG") != nullptr) {
    std::fprintf(stderr, "[muon] %d matrices, %zu groups, workspace %zu bytes\n", n, h->plan.groups.size(),
                 h->plan.total);
    for (const GroupPlan& gp : h->plan.groups)
      std::fprintf(stderr, "[muon]   group %dx%d (padded %dx%d) x %d\n", gp.m, gp.n, gp.mp, gp.np, gp.cnt);
  }
  *handle = h;
  return MUON_OK;
}

muon_status_t muon_step(muon_handle_t h, void* const* W, const void* const* G, void* const* M,
                        const muon_hparams_t* hp, cudaStream_t stream) {
  if (h == nullptr || W == nullptr || G == nullptr || M == nullptr || !hp_ok(hp, true)) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < h->n; ++i)
    if (W[i] == nullptr || G[i] == nullptr || M[i] == nullptr) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  NvtxRange range("muon_step");
  int launches = 0;
  bool fused = false;
  cudaError_t e = enqueue_front(h, G, M, hp, stream, &launches);
  if (e == cudaSuccess) e = enqueue_ns(h, hp, stream, &launches, W, false, &fused);
  if (e == cudaSuccess && !fused) e = enqueue_back(h, W, hp, false, stream, &launches);
  trace_call_end(h);
  return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

muon_status_t muon_orthogonalize(muon_handle_t h, const void* const* X, void* const* O, const muon_hparams_t* hp,
                                 cudaStream_t stream) {
  if (h == nullptr || X == nullptr || O == nullptr || !hp_ok(hp, false)) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < h->n; ++i)
    if (X[i] == nullptr || O[i] == nullptr) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  NvtxRange range("muon_orthogonalize");
  muon_hparams_t q = *hp;
  q.beta = 0.0f;
  q.nesterov = 0;
  q.lr = 0.0f;
  q.weight_decay = 0.0f;
  int launches = 0;
  cudaError_t e = enqueue_front(h, X, nullptr, &q, stream, &launches);
  bool fused = false;
  if (e == cudaSuccess) e = enqueue_ns(h, &q, stream, &launches, O, true, &fused);
  if (e == cudaSuccess && !fused) e = enqueue_back(h, O, &q, true, stream, &launches);
  trace_call_end(h);
  return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

muon_status_t muon_get_norms(muon_handle_t h, float* dst, cudaStream_t stream) {
  if (h == nullptr || dst == nullptr) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  return cudaMemcpyAsync(dst, h->d_norms, sizeof(float) * h->n, cudaMemcpyDefault, stream) == cudaSuccess
             ? MUON_OK
             : MUON_ERR_CUDA;
}

muon_status_t muon_get_status(muon_handle_t h, cudaStream_t stream) {
  if (h == nullptr) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MUON_ERR_CUDA;
  unsigned int code = 0;
  if (cudaMemcpy(&code, h->d_status, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess) return MUON_ERR_CUDA;
  if (code == 0) return MUON_OK;
  if (cudaMemset(h->d_status, 0, sizeof(code)) != cudaSuccess) return MUON_ERR_CUDA;
  return code == kDevTimeout ? MUON_ERR_TIMEOUT : MUON_ERR_DEVICE_STATUS;
}

muon_status_t muon_selftest_timeout(muon_handle_t h, uint64_t timeout_ns, cudaStream_t stream) {
  if (h == nullptr || timeout_ns < 1000ull || timeout_ns > 10000000000ull) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  return launch_timeout_selftest(h->d_status, timeout_ns, stream) == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

muon_status_t muon_get_plan(muon_handle_t h, int ns_steps, int* n_groups, int* launches_per_step) {
  if (h == nullptr || ns_steps < 0 || ns_steps > 64) return MUON_ERR_INVALID_ARG;
  if (n_groups) *n_groups = static_cast<int>(h->plan.groups.size());
  if (launches_per_step) *launches_per_step = launches_for(h, ns_steps);
  return MUON_OK;
}

muon_status_t muon_check_plan(const muon_shape_t* shapes, int n, int ns_steps, int num_sms, int64_t* problems) {
  if (problems == nullptr || !shapes_ok(shapes, n) || ns_steps < 0 || ns_steps > 64 || num_sms < 2 ||
      num_sms > 4096)
    return MUON_ERR_INVALID_ARG;
  Plan P;
  make_plan(shapes, n, MUON_MODE_FAST, &P);
  std::vector<muon_shape_t> sh(shapes, shapes + n);
  long long bad = 0;
  EwParams* ew = new (std::nothrow) EwParams;
  NsParams* ns = new (std::nothrow) NsParams;
  if (ew == nullptr || ns == nullptr) {
    delete ew;
    delete ns;
    return MUON_ERR_INVALID_ARG;
  }
  for (int b = 0; b < n; b += kEwMatsPerLaunch) {
    front_tables(P, sh, b, std::min(kEwMatsPerLaunch, n - b), ew);
    bad += check_front_tables(*ew);
  }
  if (ns_steps >= 1 && P.groups.size() <= static_cast<size_t>(kTcMaxGroups)) {
    for (int fw = 0; fw < 2; ++fw) {
      fused_tables(P, n, ns_steps, fw != 0, ns);
      bad += check_fused_tiles(*ns);
    }
  }
  delete ew;
  delete ns;
  *problems = bad;
  return MUON_OK;
}

muon_status_t muon_set_schedule(muon_handle_t h, int schedule) {
  if (h == nullptr) return MUON_ERR_INVALID_ARG;
  if (schedule != MUON_SCHEDULE_AUTO && schedule != MUON_SCHEDULE_STAGED && schedule != MUON_SCHEDULE_FUSED &&
      schedule != MUON_SCHEDULE_SPLIT)
    return MUON_ERR_INVALID_ARG;
  if ((schedule == MUON_SCHEDULE_FUSED || schedule == MUON_SCHEDULE_SPLIT) && !fused_possible(h, 1))
    return MUON_ERR_UNSUPPORTED;
  h->schedule = schedule;
  return MUON_OK;
}

muon_status_t muon_get_matrix_slot(muon_handle_t h, int i, int* group, int* slot) {
  if (h == nullptr || i < 0 || i >= h->n) return MUON_ERR_INVALID_ARG;
  if (group) *group = h->plan.mat_group[i];
  if (slot) *slot = h->plan.mat_slot[i];
  return MUON_OK;
}

muon_status_t muon_get_group_buffers(muon_handle_t h, int group, int* mp, int* np, int* count, void** x0, void** x1,
                                     void** a, void** b) {
  if (h == nullptr || group < 0 || group >= static_cast<int>(h->plan.groups.size())) return MUON_ERR_INVALID_ARG;
  const GroupPlan& gp = h->plan.groups[group];
  if (mp) *mp = gp.mp;
  if (np) *np = gp.np;
  if (count) *count = gp.cnt;
  if (x0) *x0 = h->ws + gp.off_x[0];
  if (x1) *x1 = h->ws + gp.off_x[1];
  if (a) *a = h->ws + gp.off_a;
  if (b) *b = h->ws + gp.off_b;
  return MUON_OK;
}

muon_status_t muon_profile_begin(muon_handle_t h, int max_steps) {
  if (h == nullptr || max_steps < 1 || max_steps > 100000) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  for (auto& pe : h->prof_events) cudaEventDestroy(pe.second);
  h->prof_events.clear();
  h->prof_events.reserve(static_cast<size_t>(max_steps) * 64);
  h->prof_steps_left = max_steps;
  return MUON_OK;
}

muon_status_t muon_profile_end(muon_handle_t h, double* ms, int* launches, int n_kinds) {
  if (h == nullptr || ms == nullptr || launches == nullptr || n_kinds < 1) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  for (int k = 0; k < n_kinds; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  muon_status_t st = MUON_OK;
  for (size_t i = 0; i < h->prof_events.size(); ++i) {
    if (cudaEventSynchronize(h->prof_events[i].second) != cudaSuccess) st = MUON_ERR_CUDA;
  }
  for (size_t i = 1; i < h->prof_events.size() && st == MUON_OK; ++i) {
    const int kind = h->prof_events[i].first;
    if (kind < 0 || kind >= n_kinds) continue;
    float t = 0.0f;
    if (cudaEventElapsedTime(&t, h->prof_events[i - 1].second, h->prof_events[i].second) != cudaSuccess) {
      st = MUON_ERR_CUDA;
      break;
    }
    ms[kind] += t;
    launches[kind] += 1;
  }
  for (auto& pe : h->prof_events) cudaEventDestroy(pe.second);
  h->prof_events.clear();
  h->prof_steps_left = 0;
  return st;
}

muon_status_t muon_destroy(muon_handle_t h) {
  if (h == nullptr) return MUON_ERR_INVALID_ARG;
  {
    DeviceGuard guard(h->device);
    for (auto& pe : h->prof_events) cudaEventDestroy(pe.second);
  }
  delete h;
  return MUON_OK;
}

}  // extern "C"
