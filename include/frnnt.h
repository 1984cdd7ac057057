/*
 * frnnt -- fused RNN-T joint network + transducer loss, forward and backward,
 * for NVIDIA B200 (sm_100a).  C ABI.
 *
 * What one call computes ("Flash RNN-T: Memory-Efficient Joint Network and
 * Transducer Loss Computation", abstract: a joint and loss implementation with
 * optional tiled recomputation over the full alignment space and vocabulary;
 * the transducer of "Sequence Transduction with Recurrent Neural Networks",
 * abstract; the feed-forward joint of "Transformer Transducer", abstract):
 *
 *   h[b,t,u,:] = tanh(f[b,t,:] W_f + g[b,u,:] W_g)          (H)
 *   z[b,t,u,:] = W_o h[b,t,u,:] + b_o                        (V)
 *   blank_lp = z_blank - logsumexp(z), label_lp = z_{y_u} - logsumexp(z)
 *   loss[b]  = -log sum over all alignments of the (T_len, U_len+1) lattice
 *   and the gradients of sum_b w_b loss[b] for f, g, W_f, W_g, W_o and b_o.
 *
 * Shapes (all row-major, contiguous, element strides only):
 *   f [B, T, D_enc]      g [B, U+1, D_pred]     (g[b,u] = prediction output
 *                                                after u labels)
 *   W_f [D_enc, H]       W_g [D_pred, H]
 *   W_o [V, H]           b_o [V]
 *   labels [B, U] int32  T_len [B] int32        U_len [B] int32
 * Valid lattice cells of utterance b: 0 <= t < T_len[b], 0 <= u <= U_len[b].
 * Frames t >= T_len[b], positions u > U_len[b] and labels[b, u >= U_len[b]]
 * are padding: never read into the result; their gradient rows are 0.
 *
 * Modes:
 *   FRNNT_UNTILED  the logits z are materialised (bf16 for FRNNT_BF16, fp32
 *                  for FRNNT_F32) in the workspace by the forward joint and
 *                  re-read by the backward -- fastest, memory ~ cells * V.
 *   FRNNT_TILED    only per-cell log-sum-exp / blank / label log-probs are
 *                  kept; the backward recomputes z tile by tile, and the
 *                  logit gradient lives in a bounded chunk of the workspace
 *                  (chunk_cells) -- memory independent of the batch's cells*V.
 * Both modes return the same result up to floating-point rounding.
 *
 * Precision: FRNNT_BF16 takes bf16 inputs/weights (raw uint16 bit patterns),
 * multiplies in bf16 on the tensor cores with fp32 accumulation, keeps every
 * reduction, log-sum-exp and lattice value in fp32, and returns bf16
 * gradients (round-to-nearest-even).  FRNNT_F32 computes in fp32 throughout
 * (CUDA-core FMA) and returns fp32 gradients.
 */
#ifndef FRNNT_H
#define FRNNT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FRNNT_API __attribute__((visibility("default")))
#else
#define FRNNT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FRNNT_UNTILED = 0, FRNNT_TILED = 1 } frnnt_mode;
typedef enum { FRNNT_F32 = 0, FRNNT_BF16 = 1 } frnnt_dtype;
/* Kernel family.  AUTO picks the tcgen05 tensor-core kernels for FRNNT_BF16
 * when the shape allows them (H, D_enc, D_pred multiples of 64 and V a
 * multiple of 128) and the CUDA-core kernels otherwise; SIMT forces the
 * CUDA-core kernels (fp32 arithmetic on bf16 or fp32 inputs). */
typedef enum { FRNNT_PATH_AUTO = 0, FRNNT_PATH_SIMT = 1 } frnnt_path;
/* Training criterion.  MARGINAL: -log of the probability summed over every
 * alignment ("Sequence Transduction with Recurrent Neural Networks",
 * abstract).  VITERBI: the maximum approximation, -log of the probability of
 * the single best alignment ("Daily Papers" page, CTC/RNN-T architecture
 * search, the RNN-transducer abstract comparing full marginalisation with the
 * maximum approximation): the same lattice with max in place of log-add-exp,
 * ties broken towards the blank edge, and the gradient taken along that one
 * alignment (0/1 edge posteriors). */
typedef enum { FRNNT_LOSS_MARGINAL = 0, FRNNT_LOSS_VITERBI = 1 } frnnt_loss;

/* Token-and-duration transducer limits: at most 8 durations, none above 8 frames. */
#define FRNNT_MAX_DURATIONS 8
#define FRNNT_MAX_DURATION 8

typedef struct {
  int B, T, U;            /* batch, max frames, max labels (g has U+1 rows) */
  int D_enc, D_pred;      /* encoder / prediction feature sizes              */
  int H, V;               /* joint hidden size, vocabulary size (incl. blank)*/
  int blank;              /* blank id, 0 <= blank < V                         */
  frnnt_dtype dtype;
  frnnt_mode mode;
  frnnt_path path;
  int chunk_cells;        /* FRNNT_TILED: lattice cells per backward chunk;
                             0 = default (75776 = 592 tiles of 128 cells, four
                             waves over 148 SMs, on the tensor-core kernels;
                             65536 on the CUDA-core kernels).  Rounded up to
                             whole tiles (whole frame rows on the CUDA-core
                             kernels). */
  frnnt_loss loss;        /* training criterion (MARGINAL unless set)         */
  int prune_S;            /* 0: the whole lattice.  S > 0 (S <= 32): pruned
                             lattice, frame t of utterance b keeps only the S
                             label positions bounds[b,t] <= u < bounds[b,t]+S
                             ("Pruned RNN-T for fast, memory-efficient ASR
                             training", abstract: the non-linear joiner is
                             evaluated only within pruning bounds, which are
                             an input here).  Call frnnt_fwd_bwd_pruned.
                             Needs FRNNT_BF16 on the tensor-core kernels
                             (FRNNT_ERR_UNSUPPORTED otherwise).               */
  int n_dur;              /* 0: the transducer.  n_dur > 0: the token-and-
                             duration transducer with the n_dur durations
                             below (call frnnt_fwd_bwd_tdt).                  */
  int durations[FRNNT_MAX_DURATIONS];
                          /* strictly increasing frame counts, durations[0] = 0,
                             durations[1] = 1, durations[n_dur-1] <=
                             FRNNT_MAX_DURATION; entries past n_dur unused    */
  int wgrad_f32;          /* 0: every gradient in the input dtype.  1: the
                             weight gradients dW_f, dW_g, dW_o, db_o (and the
                             duration head's dW_d, db_d) are written as fp32
                             arrays -- the library's fp32 accumulators, never
                             rounded -- also for FRNNT_BF16; df and dg stay in
                             the input dtype.  For data parallelism: partial
                             weight gradients of several devices are summed in
                             fp32 and rounded once (the loss is a sum over
                             utterances, "Sequence Transduction with Recurrent
                             Neural Networks", abstract).                     */
} frnnt_dims;

/* Host return codes. */
enum {
  FRNNT_OK = 0,
  FRNNT_ERR_NULL = 1,          /* a required pointer is NULL                  */
  FRNNT_ERR_DIMS = 2,          /* a size <= 0, blank outside [0,V), U+1 > 1024, or dims that break
                                  the pruned / duration rules or go to the wrong entry point */
  FRNNT_ERR_WORKSPACE = 3,     /* workspace_bytes smaller than required       */
  FRNNT_ERR_UNSUPPORTED = 4,   /* unknown dtype / mode / path value            */
  FRNNT_ERR_CUDA = 5,          /* a CUDA launch or query failed                */
  FRNNT_ERR_ALIGN = 6          /* a pointer is not 16-byte aligned             */
};

/* Device status bits written to *status (0 = all inputs valid). */
enum {
  FRNNT_STATUS_LENGTH = 1,     /* T_len[b] outside [1,T] or U_len[b] outside [0,U] */
  FRNNT_STATUS_LABEL = 2,      /* labels[b,u] (u < U_len[b]) outside [0,V) or == blank */
  FRNNT_STATUS_TIMEOUT = 4,    /* a bounded device-side wait gave up           */
  FRNNT_STATUS_BOUNDS = 8      /* pruned: bounds[b,0] != 0, a start outside [0,U_len[b]],
                                  bounds[b,t+1] outside [bounds[b,t], bounds[b,t]+S-1],
                                  or bounds[b,T_len[b]-1]+S-1 < U_len[b] (t < T_len[b]) */
};

/* Bytes of device workspace frnnt_fwd_bwd needs for these dims.  Host-only:
 * makes no CUDA call.  Returns FRNNT_OK or FRNNT_ERR_NULL / _DIMS / _UNSUPPORTED. */
FRNNT_API int frnnt_workspace_size(const frnnt_dims* d, size_t* bytes);

/* One forward + backward pass over one batch (one call per batch).
 *
 * All pointers are DEVICE pointers on the current device, 16-byte aligned,
 * owned by the caller; the library allocates no device memory and keeps no
 * data between calls.  Host-side it caches, per device, kernel attributes and
 * one internal stream with its events (created by the first call on that
 * device, outside any stream capture), on which part of the work runs beside
 * the caller's stream.  Calls may come from several host threads at once, on
 * one device or several, on any streams: a per-device lock serialises the
 * host-side queuing of the calls that use the internal stream (each holds it
 * from its first fork to its last join), so every call's joins wait for its
 * own side work; on the GPU the calls still overlap, except that their side
 * work runs in queue order on the one internal stream.  Float tensors are
 * fp32 (FRNNT_F32) or bf16 bit patterns (FRNNT_BF16); b_o and all gradients
 * have that same element type (weight gradients: fp32 with d->wgrad_f32).
 *   grad_loss   [B] fp32 weights w_b of d(sum_b w_b loss_b), or NULL (= 1)
 *   loss        [B] fp32 output, -log P(y_b | x_b) per utterance
 *   df, dg, dW_f, dW_g, dW_o, db_o   outputs, overwritten (not accumulated),
 *               same shapes as f, g, W_f, W_g, W_o, b_o (dW_* and db_o fp32
 *               when d->wgrad_f32 is 1)
 *   workspace   >= frnnt_workspace_size bytes, contents undefined on entry
 *   status      [1] int32 output: 0, or an OR of FRNNT_STATUS_* bits found by
 *               the device-side validation; when non-zero every other output
 *               is unspecified (no out-of-bounds access happens either way:
 *               lengths and labels are clamped before use)
 *   stream      cudaStream_t the work is queued on (NULL = legacy stream)
 * The call is stream-ordered and returns without synchronising.  Host-side
 * errors (return value != FRNNT_OK) are detected before any launch.  Its
 * consecutive kernels on `stream` are chained by programmatic dependent launch
 * (each is launched as the previous one's last CTA exits and waits for that
 * grid's results before touching memory); FRNNT_CHAIN=0 in the environment
 * turns that off, for tools that do not follow such launches. */
FRNNT_API int frnnt_fwd_bwd(const frnnt_dims* d,
                  const void* f, const void* g, const void* W_f, const void* W_g,
                  const void* W_o, const void* b_o,
                  const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                  const float* grad_loss, float* loss,
                  void* df, void* dg, void* dW_f, void* dW_g, void* dW_o, void* db_o,
                  void* workspace, size_t workspace_bytes,
                  int32_t* status, void* stream);

/* frnnt_fwd_bwd on the pruned lattice of d->prune_S > 0 (frnnt_fwd_bwd itself
 * returns FRNNT_ERR_DIMS for such dims, and this call for d->prune_S == 0).
 *   bounds      [B, T] int32 device array: first label position of frame t's
 *               band; rows past T_len[b] are padding and not read.
 * The loss sums over the alignments that stay inside the band (maximum over
 * them with FRNNT_LOSS_VITERBI); cells outside it have no logits and no
 * gradient.  Invalid bounds set FRNNT_STATUS_BOUNDS.  Everything else as
 * frnnt_fwd_bwd (same workspace size query: frnnt_workspace_size(d)). */
FRNNT_API int frnnt_fwd_bwd_pruned(const frnnt_dims* d,
                  const void* f, const void* g, const void* W_f, const void* W_g,
                  const void* W_o, const void* b_o,
                  const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                  const int32_t* bounds,
                  const float* grad_loss, float* loss,
                  void* df, void* dg, void* dW_f, void* dW_g, void* dW_o, void* db_o,
                  void* workspace, size_t workspace_bytes,
                  int32_t* status, void* stream);

/* The token-and-duration transducer (TDT) of "Efficient Sequence Transduction
 * by Jointly Predicting Tokens and Durations" (abstract: the joint network has
 * two outputs, normalised independently, one over the labels and one over
 * durations, a duration being the number of input frames the emitted symbol
 * covers).  With the hidden h of every cell as above:
 *   z  = W_o h + b_o   (V label logits, blank included)
 *   zd = W_d h + b_d   (n_dur duration logits)
 * A label y_u emitted at (t,u) with duration durations[i] moves to
 * (t + durations[i], u+1); a blank with a duration >= 1 moves to
 * (t + durations[i], u) (a zero-frame blank would be a self-loop); each edge
 * weighs P(symbol) * P(duration).  An alignment starts at (0,0) and ends with
 * a blank from (t, U_len) that lands exactly on frame T_len; loss[b] = -log of
 * the summed weight of all alignments.  The gradients of sum_b w_b loss[b]
 * come back for f, g, W_f, W_g, W_o, b_o and the duration head:
 *   W_d [n_dur, H], b_d [n_dur]  inputs;  dW_d, db_d  outputs, same shapes.
 * Needs d->n_dur in [2, FRNNT_MAX_DURATIONS] with valid durations (else
 * FRNNT_ERR_DIMS; frnnt_fwd_bwd returns FRNNT_ERR_DIMS for n_dur != 0),
 * FRNNT_BF16 on the tensor-core kernels, the marginal loss and the whole
 * lattice (FRNNT_ERR_UNSUPPORTED otherwise).  Workspace:
 * frnnt_workspace_size(d).  Everything else as frnnt_fwd_bwd. */
FRNNT_API int frnnt_fwd_bwd_tdt(const frnnt_dims* d,
                  const void* f, const void* g, const void* W_f, const void* W_g,
                  const void* W_o, const void* b_o, const void* W_d, const void* b_d,
                  const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                  const float* grad_loss, float* loss,
                  void* df, void* dg, void* dW_f, void* dW_g, void* dW_o, void* db_o,
                  void* dW_d, void* db_d,
                  void* workspace, size_t workspace_bytes,
                  int32_t* status, void* stream);

/* Size of the library-owned scratch array used by frnnt_fwd_bwd_noalloc. */
#define FRNNT_NOALLOC_MAX_BYTES (64u * 1024u * 1024u)

/* frnnt_fwd_bwd without caller-provided workspace, for callers that cannot
 * allocate device memory when they run the loss (their framework's allocator
 * owns all device memory, or an allocation could synchronise the device).
 * Not from the pages: the paper has no counterpart; this is a deployment
 * convenience of this library.
 *
 * Same arguments, semantics and return codes as frnnt_fwd_bwd, minus the
 * workspace.  The scratch is one FRNNT_NOALLOC_MAX_BYTES __device__ array in
 * the library, reserved on every GPU that loads the library until the process
 * exits; dims whose frnnt_workspace_size exceeds it return FRNNT_ERR_WORKSPACE
 * before any launch (a smaller chunk_cells lowers the need in tiled mode).
 * Allocates nothing itself: no cudaMalloc, cudaFree or allocating library
 * call.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    outside any stream capture.  Under lazy module loading (the CUDA 12
 *    default) that lookup is also when the driver loads the array's module
 *    and reserves its FRNNT_NOALLOC_MAX_BYTES on the device: if the device's
 *    memory is already taken by then, that first call fails with
 *    FRNNT_ERR_CUDA (the CUDA error state is cleared).  So make one call
 *    during start-up, before a framework allocator takes the device's memory
 *    (or load modules eagerly, CUDA_MODULE_LOADING=EAGER).
 *  - Two host threads making their first calls on different devices at once
 *    are safe (each device's address is stored atomically).
 *  - All calls share the one array, which keeps the previous call's
 *    contents; each call clears on its stream what must start at zero.
 *    Calls that can overlap on the GPU (different streams, or different
 *    host threads on one device) race on the array: serialise them. */
FRNNT_API int frnnt_fwd_bwd_noalloc(const frnnt_dims* d,
                  const void* f, const void* g, const void* W_f, const void* W_g,
                  const void* W_o, const void* b_o,
                  const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                  const float* grad_loss, float* loss,
                  void* df, void* dg, void* dW_f, void* dW_g, void* dW_o, void* db_o,
                  int32_t* status, void* stream);

/* Static description of a return code or status bit set. */
FRNNT_API const char* frnnt_error_string(int code);

/* Per-stage statistics (tracing).  A stage is one step of the path (for
 * example the forward joint) and may be one or several kernel launches. */
typedef struct {
  char name[32];
  int launches;       /* kernel launches issued by this stage since the last read */
  int calls;          /* times the stage ran since the last read                  */
  double ms;          /* summed device time between the stage's CUDA events, or 0
                         when timing was off                                       */
} frnnt_stage_stat;

/* Turns per-stage device timing on (1) or off (0) for subsequent calls.
 * When on, each stage is bracketed by two CUDA events on the call's stream
 * (events are created on first use and reused).  Launch counting is always
 * on.  Host-only; not thread-safe.  Returns FRNNT_OK. */
FRNNT_API int frnnt_profile(int enable);

/* Copies up to `capacity` stage statistics accumulated since the previous
 * read into `out`, sets *count to the number of stages, then resets them.
 * Waits for the recorded events to complete.  Returns FRNNT_OK, or
 * FRNNT_ERR_CUDA if an event query failed. */
FRNNT_API int frnnt_profile_read(frnnt_stage_stat* out, int capacity, int* count);

/* Library version, "MAJOR.MINOR.PATCH". */
FRNNT_API const char* frnnt_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FRNNT_H */
