/*
 * nshb.h -- C ABI of the B200 (sm_100a) Muon / Hyperball optimizer step.
 *
 * One call performs one optimizer step for a set of 2-D weight matrices:
 *
 *   1. momentum   M <- beta M + (1 - beta) G;  U = (1 - beta) G + beta M  (Nesterov)
 *                 ("Muon: the orthogonalized optimizer explained", momentum recap note
 *                  and the Muon.step code);
 *   2. msgn       O = NS_K(U): X = U / (||U||_F + eps) on the wide side, then K times
 *                 A = X X^T, B = b A + c A^2, X <- a X + B X
 *                 (same page, Newton-Schulz section and newton_schulz5);
 *   3. a weight-update rule:
 *        muon_step          W <- (1 - lr wd) W - lr max(1, m/n)^0.5 O    (Muon.step code)
 *        hyperball_step     W <- rho (W - eta O/||O||) / ||W - eta O/||O|| ||
 *                           ("Fantastic Pretraining Optimizers ... II: Hyperball
 *                            Optimization", Method)
 *        radial_brake_step  plain Muon step, then ||w|| <- ||w_prev|| + s (||w|| - ||w_prev||)
 *                           ("Refactor of pre/post weight update hook functions", PR #224,
 *                            RadialBrake description)
 *        relative_update_step  Muon step of length lr ||W||_F along O (same PR, RelativeUpdate)
 *      and two variants of step 2:
 *        himuon_step        NS run independently on every T x T tile, then Hyperball
 *                           ("Hierarchical Muon: Tiled Newton-Schulz Updates", abstract)
 *        newton_muon_step   NS of U (Z Z^T + lambda I)^-1, then Hyperball
 *                           ("The Newton-Muon Optimizer", abstract)
 *      and one step without NS:
 *        adamh_step         Adam's bias-corrected direction in place of O, then Hyperball
 *                           (Hyperball paper, Method)
 *
 * Conventions shared by every entry point:
 *   - Every data pointer (W, G, M, O_out, rho, Z, workspace, norms) is a DEVICE pointer
 *     owned by the caller.  The library allocates no device or host memory.
 *   - Matrices are row-major with leading dimension `ld` (elements, ld >= cols) shared by
 *     W, G and M.  O_out, when given, is row-major with leading dimension `cols`.
 *   - All work is enqueued on `stream`; no call synchronises with the host except
 *     nshb_device_status.  Concurrent calls that share a workspace race.
 *   - Argument errors are returned synchronously and nothing is enqueued.  Conditions met
 *     on the device (fallbacks, non-finite values, bounded waits that ran out) set bits in a
 *     status word kept in the workspace; each step clears it first and
 *     nshb_device_status reads it.  Nothing aborts or traps.
 */
#ifndef NSHB_H
#define NSHB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nshb_stream; /* a cudaStream_t; NULL = legacy default stream */

typedef enum { NSHB_BF16 = 0, NSHB_F32 = 1 } nshb_dtype;

typedef enum {
  NSHB_OK = 0,
  NSHB_ERR_NULL = 1,           /* a required pointer is NULL                                 */
  NSHB_ERR_SHAPE = 2,          /* rows/cols <= 0, ld < cols, a pointer not element-aligned  */
  NSHB_ERR_DTYPE = 3,          /* unknown dtype or unsupported dtype combination              */
  NSHB_ERR_PARAM = 4,          /* a scalar parameter out of range                             */
  NSHB_ERR_WORKSPACE = 5,      /* workspace smaller than nshb_workspace_size or misaligned    */
  NSHB_ERR_CUDA = 6,           /* a CUDA runtime call or a kernel launch failed               */
  NSHB_ERR_DEVICE_TIMEOUT = 7, /* (device status) a bounded wait inside a kernel ran out      */
  NSHB_ERR_NONFINITE = 8,      /* (device status) a NaN/Inf norm was met                      */
  NSHB_ERR_ZERO_NORM = 9,      /* (device status) radius taken from a zero weight norm        */
  NSHB_ERR_UNSUPPORTED = 10    /* operation/size not supported by the library                */
} nshb_status;

/* Bits of the device status word (nshb_device_status). */
#define NSHB_DEV_ZERO_NORM_FALLBACK 0x1u /* ||W - eta U_hat|| < hb_eps: step skipped, W kept on its sphere */
#define NSHB_DEV_NONFINITE 0x2u          /* a momentum, update or weight norm was NaN/Inf                  */
#define NSHB_DEV_TIMEOUT 0x4u            /* a bounded device wait ran out; results are not valid           */
#define NSHB_DEV_ZERO_RADIUS 0x8u        /* rho <= 0 asked for the current norm, which was < hb_eps        */
#define NSHB_DEV_NOT_SPD 0x10u           /* Newton-Muon: Z Z^T + lambda I not positive definite in fp32    */

typedef enum {
  NSHB_OP_MUON = 0,
  NSHB_OP_HYPERBALL = 1,
  NSHB_OP_RADIAL_BRAKE = 2,
  NSHB_OP_HIMUON = 3,
  NSHB_OP_NEWTON_MUON = 4,
  NSHB_OP_RELATIVE_UPDATE = 5,
  NSHB_OP_ADAMH = 6
} nshb_op;

/* One weight matrix (rows x cols).  W is updated in place, G is read, M is the fp32
 * momentum buffer (zero before the first step; the only state a step keeps).
 * W and G share w_dtype.  Rows are read and written with 16-byte vector accesses when
 * W, G and M are 16-byte aligned and ld * sizeof(element) and ld * 4 are multiples of 16;
 * other layouts take a slower element-wise path.  W, G and O_out must be aligned to their
 * element size and M (and AdamH's V) to 4 bytes, else NSHB_ERR_SHAPE.
 * O_out (optional, may be NULL) receives the orthogonalised update O = NS_K(U)
 * (before any step-length or shape scaling), dtype w_dtype, leading dimension cols.
 * z_index picks the layer input Z of newton_muon_step (ignored elsewhere).
 * Sizes: rows and cols up to 2^20 and ld up to 2^30; larger ones return
 * NSHB_ERR_UNSUPPORTED. */
typedef struct {
  int64_t rows, cols, ld;
  int32_t w_dtype; /* nshb_dtype */
  int32_t z_index;
  void *W;
  const void *G;
  float *M;
  void *O_out;
} nshb_matrix;

/* Step parameters.  Defaults (nshb_default_params): beta 0.95, Nesterov, K = 5 with
 * (a, b, c) = (3.4445, -4.7750, 2.0315), ns_eps 1e-7, bf16 tensor-core NS, lr 0.02,
 * wd 0, eta 0.02, rho NULL, hb_eps 1e-8, brake 0.5 / 1.0, tile 256, ridge_rel 1e-3,
 * ns_compensated 2. */
typedef struct {
  float beta;            /* momentum coefficient, [0, 1)                                    */
  int32_t nesterov;      /* 1: U = (1-beta) G + beta M; 0: U = M                             */
  int32_t ns_steps;      /* K >= 1 (<= 32)                                                   */
  int32_t ns_precision;  /* NSHB_BF16: bf16 tensor cores, fp32 accumulate; NSHB_F32: fp32     */
  const float *coeffs;   /* HOST pointer to ns_steps x 3 (a, b, c) rows, or NULL for the      */
                         /* constant quintic (3.4445, -4.7750, 2.0315)                        */
  float ns_eps;          /* additive eps of the NS normalisation, > 0                         */
  float lr;              /* muon_step / radial_brake_step learning rate                       */
  float weight_decay;    /* muon_step decoupled weight decay                                  */
  float eta;             /* Hyperball step length (absolute Frobenius length), >= 0           */
  const float *rho;      /* DEVICE array [n_mats] of radii; entry <= 0, or rho == NULL, means */
                         /* "use the current ||W||_F" (radius=None in the hook); 4-byte       */
                         /* aligned, else NSHB_ERR_PARAM                                      */
  float hb_eps;          /* numerical-zero threshold for norms, > 0                           */
  float brake_out;       /* RadialBrake outward factor in [0, 1]                              */
  float brake_in;        /* RadialBrake inward factor in [0, 1]                               */
  int32_t tile;          /* HiMuon tile size T: 128, 256 or 512                               */
  float ridge_rel;       /* Newton-Muon: lambda = ridge_rel * tr(Z Z^T) / d_in, >= 0          */
  int32_t ns_compensated;/* bf16 NS: leading iterations whose a*X term reads X as a bf16 hi/lo */
                         /* pair (about fp32 accuracy); 0 = plain bf16 chain; default 2;      */
                         /* values above ns_steps act as ns_steps; range [0, 32]             */
  uint32_t debug_flags;  /* 0 in normal use.  Tests only: bit 0 shortens every device wait    */
                         /* limit to ~1 ms; bit 1 makes the tensor-core GEMM withhold one     */
                         /* accumulator hand-off so that a bounded wait runs out and the step */
                         /* reports NSHB_DEV_TIMEOUT (results then are not valid)             */
} nshb_params;

/* Fills *p with the defaults listed above.  Returns NSHB_ERR_NULL if p is NULL. */
nshb_status nshb_default_params(nshb_params *p);

/* Bytes of device workspace that a step of kind `op` on these matrices needs.
 * z_rows (HOST array of n_z), n_z and n_tokens matter only for NSHB_OP_NEWTON_MUON
 * (pass NULL / 0 / 0 otherwise).  Host-only: touches no device memory.  The workspace must
 * be 256-byte aligned. */
nshb_status nshb_workspace_size(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p,
                                int32_t op, const int64_t *z_rows, int32_t n_z, int64_t n_tokens,
                                size_t *bytes);

/* Muon step (Muon.step code): momentum, NS, W <- (1 - lr wd) W - lr max(1, m/n)^0.5 O. */
nshb_status muon_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                      size_t ws_bytes, nshb_stream stream);

/* Muon step wrapped by Hyperball (Hyperball paper, Method):
 * W <- rho (W - eta U_hat) / ||W - eta U_hat||_F with U_hat = O / max(||O||_F, hb_eps).
 * If ||W - eta U_hat|| < hb_eps the step is skipped and W <- rho W / ||W||
 * (NSHB_DEV_ZERO_NORM_FALLBACK).  Shape scaling and weight decay do not apply. */
nshb_status hyperball_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                           size_t ws_bytes, nshb_stream stream);

/* Muon step followed by the RadialBrake hook (PR #224): w = w_prev - lr max(1,m/n)^0.5 O,
 * then w <- w (||w_prev|| + s (||w|| - ||w_prev||)) / ||w||, s = brake_out if the norm grew,
 * else brake_in; w is left as is when ||w|| < hb_eps.  weight_decay must be 0. */
nshb_status radial_brake_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p,
                              void *ws, size_t ws_bytes, nshb_stream stream);

/* Hierarchical Muon wrapped by Hyperball: U is cut into T x T tiles anchored at (0, 0)
 * (edge tiles are the remainder), every tile gets its own normalisation and NS map,
 * then the Hyperball rule acts on the whole matrix.  bf16 NS only. */
nshb_status himuon_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                        size_t ws_bytes, nshb_stream stream);

/* Newton-Muon wrapped by Hyperball: P = U (Z Z^T + lambda I)^-1 with
 * lambda = ridge_rel tr(Z Z^T) / d_in, solved through a blocked Cholesky factorisation (the
 * 256 x 256 diagonal blocks factored and inverted in fp32; every other product on the tensor
 * cores with each operand split into two bf16 parts, three products per output, fp32
 * accumulation), then O = NS_K(P) and the Hyperball rule (U is the Nesterov momentum update).  Z[j] is a
 * DEVICE pointer to a bf16 row-major z_rows[j] x n_tokens matrix (leading dimension
 * n_tokens, 16-byte aligned); n_tokens (up to 2^24) and every z_rows[j] (up to 16384) must be
 * multiples of 64, else NSHB_ERR_SHAPE; matrix i uses Z[mats[i].z_index] (an index outside
 * [0, n_z) is NSHB_ERR_PARAM), which needs z_rows == cols (else NSHB_ERR_SHAPE).  Z and z_rows
 * are HOST arrays of n_z entries (1 <= n_z <= 224).  A pivot that is not positive in fp32 sets
 * NSHB_DEV_NOT_SPD.  bf16 NS only.  The tensor cores read every Z in place during the call
 * (no copy in the workspace), so Z must stay unchanged until the step has run on the stream. */
nshb_status newton_muon_step(const nshb_matrix *mats, int32_t n_mats, const void *const *Z,
                             const int64_t *z_rows, int32_t n_z, int64_t n_tokens,
                             const nshb_params *p, void *ws, size_t ws_bytes, nshb_stream stream);

/* Muon step followed by the RelativeUpdate hook (PR #224 file list: a pre-update scaling that
 * matches the update's norm to the current weight norm):
 *   W <- (1 - lr wd) W - lr ||W||_F O / max(||O||_F, hb_eps)
 * (the shape factor of the Muon update cancels in the rescaling; a zero O leaves W scaled by
 * 1 - lr wd).  Same momentum, NS options and workspace as muon_step (op
 * NSHB_OP_RELATIVE_UPDATE in nshb_workspace_size). */
nshb_status relative_update_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                                 size_t ws_bytes, nshb_stream stream);

/* Adam options of adamh_step.  Defaults (nshb_default_adam_params): the values of "Adam: A
 * Method for Stochastic Optimization", beta1 0.9, beta2 0.999, eps 1e-8, step 1. */
typedef struct {
  float beta1;   /* first-moment coefficient, [0, 1)                                      */
  float beta2;   /* second-moment coefficient, [0, 1)                                     */
  float eps;     /* added to sqrt(v_hat), > 0                                             */
  int32_t step;  /* t >= 1, the step being taken (bias corrections 1 - beta^t)            */
} nshb_adam_params;

/* Fills *a with the defaults listed above.  Returns NSHB_ERR_NULL if a is NULL. */
nshb_status nshb_default_adam_params(nshb_adam_params *a);

/* AdamH (Hyperball paper, Method: Hyperball around Adam's preconditioned update):
 *   M <- beta1 M + (1 - beta1) G;  V <- beta2 V + (1 - beta2) G^2;
 *   U~ = (M / (1 - beta1^t)) / (sqrt(V / (1 - beta2^t)) + eps);
 *   W <- rho (W - eta U_hat) / ||W - eta U_hat||_F,  U_hat = U~ / max(||U~||_F, hb_eps),
 * with the zero-norm fallback and status bits of hyperball_step.  mats[i].M is the fp32 first
 * moment; V is a HOST array of n_mats DEVICE pointers to the fp32 second moments (same rows,
 * cols and ld as W, zero before step 1).  U~ is formed in fp32 and kept in w_dtype for the
 * Hyperball rule.  p supplies eta, rho and hb_eps (the NS fields are not used); O_out, when
 * set, receives U~.  Workspace: nshb_workspace_size(..., NSHB_OP_ADAMH, ...). */
nshb_status adamh_step(const nshb_matrix *mats, int32_t n_mats, float *const *V, const nshb_adam_params *a,
                       const nshb_params *p, void *ws, size_t ws_bytes, nshb_stream stream);

/* Memory-bounded steps (Hierarchical Muon's scaling note: the work is independent per tile, so
 * it can be processed in pieces).  nshb_step_chunked runs the step of kind `op` (NSHB_OP_MUON,
 * _HYPERBALL, _RADIAL_BRAKE, _HIMUON or _RELATIVE_UPDATE) over mats[0..n_mats) in consecutive
 * chunks, each as long as fits in ws_bytes, one after the other on `stream`; p->rho (when set)
 * is indexed like mats.  Every matrix's result is the one the unchunked call computes, and
 * the device status word holds the flags of every chunk (the call clears it once, before
 * the first).  *n_chunks (optional) receives the number of chunks.
 * nshb_workspace_size_min gives the smallest workspace it accepts (the largest single-matrix
 * need); a smaller one returns NSHB_ERR_WORKSPACE before anything is queued. */
nshb_status nshb_workspace_size_min(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, int32_t op,
                                    size_t *bytes);
nshb_status nshb_step_chunked(int32_t op, const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                              size_t ws_bytes, nshb_stream stream, int32_t *n_chunks);

/* out[i] = ||W_i||_F (fp32) into the DEVICE array out (n_mats floats, 4-byte aligned, else
 * NSHB_ERR_SHAPE), e.g. rho = ||W0||.
 * Needs a workspace of nshb_workspace_size(..., NSHB_OP_MUON, ...) bytes. */
nshb_status nshb_fro_norms(const nshb_matrix *mats, int32_t n_mats, float *out, void *ws,
                           size_t ws_bytes, nshb_stream stream);

/* No counterpart in the papers: an allocation-free variant of nshb_fro_norms for callers
 * that cannot allocate device memory (e.g. a hook running inside a framework whose caching
 * allocator owns the device memory, or a C tool with no allocator) and so cannot pass a
 * workspace.  out[i] = ||W_i||_F (fp32, DEVICE array of n_mats floats); only W, rows, cols,
 * ld and w_dtype of each matrix are read.  Scratch is a fixed NSHB_STATIC_SCRATCH_BYTES
 * device array inside the library, held by every GPU that loads it until exit.  The first
 * call on a device looks up that array's address (make it before any stream capture).
 * Limits: n_mats <= 192 and sum over matrices of ceil(rows/64) * ceil(cols/64) <= 174,240
 * (about 7.1e8 elements); larger requests return NSHB_ERR_WORKSPACE before any work is
 * queued.  Calls share the array, so calls that overlap on the GPU race.  The array's
 * address is looked up once per device and kept, so resetting a device (cudaDeviceReset)
 * after the first call on it is not supported.  There is no status word to read: a
 * non-finite norm shows only as NaN or Inf in out.  A failed launch returns NSHB_ERR_CUDA
 * and records the CUDA error for nshb_last_cuda_error. */
#define NSHB_STATIC_SCRATCH_BYTES (4u << 20)
nshb_status nshb_fro_norms_static(const nshb_matrix *mats, int32_t n_mats, float *out, nshb_stream stream);

/* Synchronises `stream`, then copies the device status word of the last step that used
 * this workspace into *flags (NSHB_DEV_* bits).  The one call that blocks the host. */
nshb_status nshb_device_status(const void *ws, nshb_stream stream, uint32_t *flags);

/* Static, NUL-terminated name of a status code. */
const char *nshb_status_string(int32_t status);

/* Measurement aid.  While enabled (process-wide switch), every kernel launch of a step is
 * bracketed by two CUDA events recorded on the step's stream.  nshb_profile_read waits for
 * the recorded events, writes the summed kernel time (ms) and the launch count of each
 * kind (NSHB_PROF_*) into ms[0..n_kinds) / launches[0..n_kinds), and clears the record.
 * The events are created by the library on first use and reused afterwards. */
#define NSHB_PROF_MOMENTUM 0 /* momentum + U + norm partials                  */
#define NSHB_PROF_NORM 1     /* per-matrix / per-tile normalisation scales    */
#define NSHB_PROF_GRAM 2     /* tensor-core A = s^2 X X^T                      */
#define NSHB_PROF_POLY 3     /* tensor-core B = b A + c A^2                    */
#define NSHB_PROF_UPDATE 4   /* tensor-core X' = s (a X + B X)                 */
#define NSHB_PROF_REDUCE 5   /* ||O||^2, <W,O>, ||W||^2 partials               */
#define NSHB_PROF_FINALIZE 6 /* per-matrix update coefficients                 */
#define NSHB_PROF_EXACT 7    /* element-wise ||W - tO||^2 for cancelling steps */
#define NSHB_PROF_APPLY 8    /* W <- alpha W + beta O                          */
#define NSHB_PROF_F32GEMM 9  /* fp32 NS GEMMs (all three phases)               */
#define NSHB_PROF_NEWTON 10  /* Newton-Muon Gram, Cholesky and solves          */
#define NSHB_PROF_ADAM 11    /* AdamH moments, direction and partials         */
#define NSHB_PROF_KINDS 12
nshb_status nshb_profile_enable(int32_t on);
nshb_status nshb_profile_read(int32_t n_kinds, float *ms, int32_t *launches);

/* The cudaError_t value behind the last NSHB_ERR_CUDA returned to this host thread
 * (0 if none): a diagnostic for failed launches or runtime calls. */
int32_t nshb_last_cuda_error(void);

/* ABI version (major * 10000 + minor * 100 + patch). */
int32_t nshb_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NSHB_H */
