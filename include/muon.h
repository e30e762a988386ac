/*
 * muon.h — C ABI of libmuon.so: the Muon optimizer step for 2-D weight
 * matrices on NVIDIA B200 (sm_100a).
 *
 * The method.  Muon is the orthogonalised-momentum optimizer for matrix
 * parameters ("把 GPT-2 的训练租金估算从 4.3 万美元压到 40 美元 ...",
 * magicnetworld, glossary table, row "Muon"); the hybrid recipe orthogonalises
 * the matrix parameters by Newton-Schulz and leaves the rest to AdamW
 * ("开发者千美元训3.8B模型 击败GPT-2", aiproducthub, 影响 paragraph).  The pages
 * print no formula; the step implemented here, per matrix W, G, M of shape
 * rows x cols, is
 *
 *   M1 = beta*M + (1-beta)*G                         (momentum, lerp form)
 *   U  = (1-beta)*G + beta*M1  if nesterov, else M1  (Nesterov blend)
 *   X  = U, or U^T if rows > cols;  X = X / (||X||_F + eps)
 *   k times:  A = X X^T;  B = b*A + c*A A;  X = a*X + B X
 *   O  = X, or X^T if rows > cols
 *   W1 = (1 - lr*weight_decay)*W - lr*sqrt(max(1, rows/cols))*O
 *
 * Memory.  The caller owns every byte of device memory: W, G, M and one
 * workspace buffer sized by muon_workspace_size().  The library never calls
 * cudaMalloc/cudaFree.  A handle owns only host-side tables (the shape
 * grouping and the TMA descriptors of the workspace).
 *
 * Streams.  muon_step and muon_orthogonalize only enqueue work on the given
 * stream and return; they never synchronise the device, so they can be
 * captured into a CUDA graph.  Pointers must stay valid until the enqueued
 * work has finished.  Calls on one handle must not overlap on the device
 * (they share the workspace).
 *
 * Kernels.  A step enqueues the momentum/norm kernel, then the Newton-Schulz
 * iterations, then the parameter write.  In MUON_MODE_FAST the iterations run
 * as three tensor-core launches each (Gram, polynomial, update) over every
 * matrix of the handle, with the parameter write fused into the last update
 * for bf16 sets whose dimensions are multiples of 32 and whose parameters are
 * 16-byte aligned (the fused write and the separate write kernel compute the
 * same W, bit for bit, from X_k rounded to bf16).  When every matrix fits
 * one 256 x 256 tile (max(rows, cols) <= 256, at most six distinct shapes),
 * all k iterations run in one launch instead (MUON_KERNEL_NS_SMALL).
 * Results are the same function of the inputs on either path, within the
 * bf16 rounding described under muon_mode_t.
 *
 * Errors.  Every entry point returns a muon_status_t and never throws.
 * Argument errors are detected on the host before anything is enqueued.
 * Launch failures return MUON_ERR_CUDA.  Faults the kernels detect on the
 * device (a bounded wait that ran out) are recorded in a status word in the
 * workspace and reported by muon_get_status().
 */
#ifndef MUON_H_
#define MUON_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,    /* null pointer, bad size or count, bad hyper-parameter */
  MUON_ERR_UNSUPPORTED = 2,    /* dtype/mode combination or shape this build does not run */
  MUON_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed (launch, descriptor encode) */
  MUON_ERR_WORKSPACE = 4,      /* workspace null, too small or not 1024-byte aligned */
  MUON_ERR_TIMEOUT = 5,        /* a device-side bounded wait ran out (see muon_get_status) */
  MUON_ERR_DEVICE_STATUS = 6,  /* any other fault recorded by a kernel */
  MUON_ERR_NO_DEVICE = 7       /* no sm_100 device current */
} muon_status_t;

/* Storage type of W, G, M (and of the X/O buffers of muon_orthogonalize). */
typedef enum { MUON_BF16 = 0, MUON_FP32 = 1 } muon_dtype_t;

/* Arithmetic of the Newton-Schulz products.
 * FAST:     bf16 operands on the tcgen05 tensor cores, fp32 accumulation in
 *           TMEM, fp32 epilogue math, one bf16 rounding per stored intermediate
 *           (X, A, and B' = a I + b A + c A A, every term of B' taken from the
 *           rounded A).
 * FP32_REF: fp32 operands and intermediates, products accumulated in fp64 on
 *           the CUDA cores (no TF32): a slow, accurate mode for checking. */
typedef enum { MUON_MODE_FAST = 0, MUON_MODE_FP32_REF = 1 } muon_mode_t;

typedef struct { int64_t rows, cols; } muon_shape_t;

typedef struct {
  float lr;            /* learning rate */
  float beta;          /* momentum coefficient, 0 <= beta <= 1 */
  float weight_decay;  /* decoupled weight decay, applied to the pre-update W */
  float eps;           /* added to ||X||_F before dividing, >= 0; an all-zero X with
                          eps = 0 is taken as the zero direction (zero update) */
  float a, b, c;       /* Newton-Schulz polynomial a x + b x^3 + c x^5 */
  int32_t nesterov;    /* nonzero: Nesterov blend */
  int32_t ns_steps;    /* iterations k, 0 <= k <= 64 */
} muon_hparams_t;

typedef struct muon_ctx* muon_handle_t;

/* Largest number of matrices one handle accepts. */
#define MUON_MAX_MATRICES 4096

/*
 * Bytes of device workspace a handle for these shapes needs.  Matrices of one
 * orientation-free shape (min(rows,cols), max(rows,cols)) form one group and
 * share one batched buffer set; each group holds two X buffers, A and B, all
 * padded with zeros to multiples of 256.
 *   shapes: host array of n shapes, rows >= 1, cols >= 1.
 *   bytes:  host out-pointer.
 * Returns MUON_ERR_INVALID_ARG on a null pointer, n < 1 or n > MUON_MAX_MATRICES,
 * or a non-positive dimension.
 */
MUON_API muon_status_t muon_workspace_size(const muon_shape_t* shapes, int n, muon_dtype_t dtype,
                                  muon_mode_t mode, size_t* bytes);

/*
 * Build a handle for a fixed parameter set.
 *   shapes:    host array of n shapes (copied).
 *   workspace: device pointer, 1024-byte aligned, ws_bytes >= muon_workspace_size().
 *              It is zero-filled here (synchronously, on the legacy default stream
 *              semantics of cudaMemset) and must outlive the handle.
 * Uses the current CUDA device, which must be sm_100 (B200).  The handle is
 * bound to that device.
 */
MUON_API muon_status_t muon_create(muon_handle_t* handle, const muon_shape_t* shapes, int n, muon_dtype_t dtype,
                          muon_mode_t mode, void* workspace, size_t ws_bytes);

/*
 * One Muon step for every matrix of the handle, enqueued on `stream`.
 *   W, G, M: host arrays of n device pointers, in the order of the shapes given to
 *            muon_create; matrix i is rows_i x cols_i, row-major, contiguous, of the
 *            handle's dtype.  W and M are updated in place; G is only read.  Any
 *            alignment is accepted; 16-byte aligned rows take the vector path.
 *   hp:      host pointer, read before returning.
 * Returns MUON_ERR_INVALID_ARG for null arrays/pointers or bad hyper-parameters.
 */
MUON_API muon_status_t muon_step(muon_handle_t handle, void* const* W, const void* const* G, void* const* M,
                        const muon_hparams_t* hp, cudaStream_t stream);

/*
 * The orthogonaliser alone: O_i = NS_k(X_i) (normalise, k iterations, orient back),
 * with no momentum and no parameter write.  X and O are host arrays of n device
 * pointers of the handle's dtype and shapes; X is only read.  Only hp->eps, a, b, c
 * and ns_steps are used.
 */
MUON_API muon_status_t muon_orthogonalize(muon_handle_t handle, const void* const* X, void* const* O,
                                 const muon_hparams_t* hp, cudaStream_t stream);

/*
 * AdamW for the parameters that are not matrices: the other half of the hybrid
 * optimizer ("开发者千美元训3.8B模型 击败GPT-2", aiproducthub, 影响 paragraph:
 * Newton-Schulz orthogonalisation for the matrix parameters, AdamW for the rest).
 * The pages print no formula; per element, with t = hp->step >= 1:
 *   m1 = beta1 m + (1-beta1) g;  v1 = beta2 v + (1-beta2) g^2
 *   p1 = (1 - lr wd) p - lr (m1 / (1-beta1^t)) / (sqrt(v1 / (1-beta2^t)) + eps)
 *   P, G: host arrays of n device pointers to tensors of numel[i] elements of
 *         `dtype` (any shape, contiguous); P is updated in place, G only read.
 *   M, V: host arrays of n device pointers to numel[i] fp32 moments each,
 *         updated in place.
 * No handle and no workspace: the call is stateless (the step count is the
 * caller's).  16-byte-aligned tensors take the vector path.  Returns
 * MUON_ERR_INVALID_ARG for null pointers, negative sizes, step < 1, betas
 * outside [0, 1), eps < 0 or non-finite lr/wd; n == 0 is a no-op.
 */
typedef struct {
  float lr, beta1, beta2, eps, weight_decay;
  int32_t step;
} muon_adamw_hparams_t;
MUON_API muon_status_t muon_adamw_step(void* const* P, const void* const* G, float* const* M, float* const* V,
                                       const int64_t* numel, int n, muon_dtype_t dtype,
                                       const muon_adamw_hparams_t* hp, cudaStream_t stream);

/*
 * Copy the n per-matrix Frobenius norms ||U_i||_F of the last step (fp32) into
 * `dst` (host or device memory, n floats), enqueued on `stream`.  Host memory
 * should be pinned for the copy to stay asynchronous.
 */
MUON_API muon_status_t muon_get_norms(muon_handle_t handle, float* dst, cudaStream_t stream);

/*
 * Synchronise `stream`, read the device status word of the handle and clear it.
 * Returns MUON_OK, MUON_ERR_TIMEOUT or MUON_ERR_DEVICE_STATUS (device fault
 * recorded since the last call), or MUON_ERR_CUDA if the stream reported an error.
 */
MUON_API muon_status_t muon_get_status(muon_handle_t handle, cudaStream_t stream);

/*
 * Failure-detection self-test: enqueue one kernel whose only work is a wait on a
 * shared-memory barrier that nothing signals, bounded by `timeout_ns`
 * (1e3 .. 1e10).  The kernel gives up, records MUON_ERR_TIMEOUT in the status
 * word and returns; muon_get_status() then reports it.  Uses the same bounded
 * wait as the GEMM pipelines.
 */
MUON_API muon_status_t muon_selftest_timeout(muon_handle_t handle, uint64_t timeout_ns, cudaStream_t stream);

/* Release the handle (host memory only; the workspace stays the caller's). */
MUON_API muon_status_t muon_destroy(muon_handle_t handle);

/* Static, human-readable name of a status code. */
MUON_API const char* muon_status_string(muon_status_t status);

/*
 * Plan introspection: the number of shape groups the handle formed, and the
 * number of kernel launches one muon_step with `ns_steps` iterations enqueues
 * (the memset of the arrival counters is not a kernel and is not counted).
 */
MUON_API muon_status_t muon_get_plan(muon_handle_t handle, int ns_steps, int* n_groups, int* launches_per_step);

/*
 * How the k Newton-Schulz iterations of a MUON_MODE_FAST handle are launched.
 *   MUON_SCHEDULE_STAGED  one tensor-core launch per stage and iteration (3 k
 *                         launches: Gram, polynomial, update), each over every
 *                         matrix of the handle.
 *   MUON_SCHEDULE_FUSED   all 3 k stages in one persistent launch: the tiles of
 *                         every stage form one list, and a tile waits (on the
 *                         device, bounded) only until the stage it reads is
 *                         complete for its own matrix, so the stages of different
 *                         matrices overlap and no launch boundary drains the GPU.
 *                         Same arithmetic and rounding as STAGED (results are
 *                         bitwise equal).  Needs at most 6 distinct shape groups.
 *   MUON_SCHEDULE_SPLIT   the tiles of FUSED, one launch per stage (3 k launches):
 *                         separates the single-launch kernel's tile machinery
 *                         from its scheduling, for measurements.
 *   MUON_SCHEDULE_AUTO    (default) FUSED when every shape group's smaller
 *                         dimension is at most 768 (there it measured within 1 %
 *                         of STAGED with one launch per step instead of 3 k),
 *                         else STAGED.
 * The small-matrix kernel (MUON_KERNEL_NS_SMALL) keeps precedence when its
 * conditions hold; FP32_REF handles always run staged.  Returns
 * MUON_ERR_UNSUPPORTED if FUSED is asked of a handle that cannot run it.
 * The setting applies to later calls; it must not change while a captured graph
 * of the handle is replayed.
 */
/*
 * Host-only consistency check of the launch tables muon_step would build for
 * these shapes on a device with num_sms SMs (no device needed): the persistent
 * momentum/norm kernel's tile ranges and partial-sum slots, and the single-launch
 * schedule's tile list for ns_steps iterations (every stage of every matrix
 * covered once, stages listed before the tiles that wait for them, wait targets
 * equal to the stages' tile counts), with and without the fused parameter
 * write.  *problems receives the number of inconsistencies (0 when sound).  For
 * tests and tools.
 */
MUON_API muon_status_t muon_check_plan(const muon_shape_t* shapes, int n, int ns_steps, int num_sms,
                                       int64_t* problems);

#define MUON_SCHEDULE_AUTO 0
#define MUON_SCHEDULE_STAGED 1
#define MUON_SCHEDULE_FUSED 2
#define MUON_SCHEDULE_SPLIT 3
MUON_API muon_status_t muon_set_schedule(muon_handle_t handle, int schedule);

/*
 * Momentum, Nesterov blend and Frobenius norm of ONE matrix, with no workspace.
 * The pages have no counterpart for this entry point: it exists for callers that
 * cannot give this library device memory (a framework whose allocator must own
 * every device allocation, a fixed memory pool, code that may not call
 * cudaMalloc).  It computes, for the rows x cols row-major matrix of `dtype`,
 *   M <- beta*M + (1-beta)*G   (in place),
 *   U <- (1-beta)*G + beta*M   if nesterov, else U <- M   (U: same shape/dtype),
 *   *norm <- ||U||_F           (fp32; `norm` is a device pointer to one float),
 * the same arithmetic as the first stage of muon_step (U in the caller's layout,
 * not transposed).  The norm's reduction scratch is a fixed array of device
 * memory inside libmuon.so (about 16 KB, held by every GPU that loads the
 * library until the process exits); the call allocates nothing.
 *   - rows * cols may be at most MUON_STATIC_MAX_ELEMENTS, else
 *     MUON_ERR_UNSUPPORTED is returned and nothing is enqueued.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address; make it before capturing any stream.  A first
 *     call on a stream that is being captured returns MUON_ERR_UNSUPPORTED
 *     without touching the capture.
 *   - All calls share the array.  Calls in sequence on one stream are
 *     independent (the arrival counter is cleared at the start of each call);
 *     calls that overlap on the GPU race and give wrong norms.
 */
#define MUON_STATIC_MAX_ELEMENTS (1ll << 28)
MUON_API muon_status_t muon_momentum_norm_static(const void* G, void* M, void* U, int64_t rows, int64_t cols,
                                                 muon_dtype_t dtype, float beta, int32_t nesterov, float* norm,
                                                 cudaStream_t stream);

/*
 * Workspace introspection, for tests and tools.  muon_get_matrix_slot gives the
 * shape group of matrix i and its slot inside the group's batched buffers;
 * muon_get_group_buffers gives a group's padded oriented shape (mp x np, both
 * multiples of 256), its matrix count and the device addresses of its buffers
 * inside the workspace: X0 and X1 ([count][mp][np]) and A and B
 * ([count][mp][mp]), elements bf16 in FAST mode and fp32 in FP32_REF mode.
 * After muon_orthogonalize/muon_step with k iterations, X0 holds U (oriented,
 * unnormalised), A and B hold the last iteration's Gram and polynomial
 * matrices, and X(k mod 2) the final iterate.  Any output pointer may be NULL.
 */
MUON_API muon_status_t muon_get_matrix_slot(muon_handle_t handle, int i, int* group, int* slot);
MUON_API muon_status_t muon_get_group_buffers(muon_handle_t handle, int group, int* mp, int* np, int* count,
                                              void** x0, void** x1, void** a, void** b);

/*
 * Kernel tracing with CUDA events (no device memory).  After
 * muon_profile_begin(h, max_steps), each of the next max_steps calls of
 * muon_step / muon_orthogonalize records one event before its first kernel and
 * one after every kernel, on the caller's stream.  muon_profile_end()
 * synchronises those events, writes for each kernel kind k (MUON_KERNEL_*) the
 * summed device milliseconds ms[k] and the number of launches launches[k]
 * (arrays of n_kinds entries, host memory), destroys the events and stops
 * recording.  The time of a kernel is the gap between the events around it.
 */
#define MUON_KERNEL_MOMENTUM_NORM 0
#define MUON_KERNEL_GRAM 1
#define MUON_KERNEL_POLY 2
#define MUON_KERNEL_UPDATE 3
#define MUON_KERNEL_WRITE 4
#define MUON_KERNEL_SGEMM 5
#define MUON_KERNEL_NS_SMALL 6 /* all iterations of a set of matrices of at most 256 x 256 */
#define MUON_KERNEL_NS_FUSED 7 /* all iterations of a set in one launch (MUON_SCHEDULE_FUSED) */
#define MUON_KERNEL_KINDS 8
MUON_API muon_status_t muon_profile_begin(muon_handle_t handle, int max_steps);
MUON_API muon_status_t muon_profile_end(muon_handle_t handle, double* ms, int* launches, int n_kinds);

#ifdef __cplusplus
}
#endif

#endif /* MUON_H_ */
