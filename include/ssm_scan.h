/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective-scan library (Mamba-1 S6).
 *
 * The operation (per batch element b, channel d, state n, time t):
 *
 *   u_t      = SiLU(conv_b[d] + sum_{k<K} conv_w[d][k] * x_{t-k})      (x_{t<0} = 0)
 *   Delta_t  = softplus(dt_t + dt_bias[d])          (or dt_t + dt_bias[d] when delta_softplus = 0)
 *   A        = -exp(A_log[d][n])
 *   A_bar    = exp(Delta_t * A),   B_bar = (A_bar - 1) / A * B_t[n]      (exact zero-order hold)
 *   h_t[n]   = A_bar * h_{t-1}[n] + B_bar * u_t,                         h_{-1} = 0
 *   y_t      = sum_n C_t[n] * h_t[n] + D[d] * u_t
 *   out_t    = y_t * SiLU(z_t)
 *
 * Sources (page title, section):
 *  - "Sequence and state-space models" (docs.algenta.ai), `state_space_models`: the exact ZOH
 *    pair ssm_discretize_zoh / ssm_discretize_b, ssm_recurrence_step, ssm_output_step and
 *    mamba_delta_softplus.
 *  - "state-space models" (aarnphm.xyz): "From continuous time to tokens", "One recurrence, one
 *    convolution" (h_{-1} = 0), "Mamba" (token-dependent Delta_t, B_t, C_t; fixed diagonal A).
 *  - "State-Space Models & Long-Context Sequence Architectures (Mamba)" (glossary),
 *    "Mathematical Formulation" (the D feed-through) and Lab 3 (associative scan).
 *  - "Selective Mamba" (TorchLean Runtime.Autograd.Model.Mamba): Parameters (convKernel rows
 *    newest-first, convBias before the SiLU, logA, dSkip on the activated feature, the SiLU
 *    gate; B and C shared by the expanded channels), Options.validate (empty axes rejected),
 *    runArray (an empty chunk changes nothing).
 *  - rustytorch commit log: the real S6 forward order and the hand-written VJP (reverse-time
 *    recurrence; dA_log = dA * A).
 *
 * Conventions for every entry point:
 *  - Pointers named "device" are CUDA device (or managed) memory on the current device. The
 *    caller owns every buffer; the entry points allocate no device memory. Library state is
 *    limited to a per-thread last-CUDA-error word (ssm_last_cuda_error) and, for
 *    ssm_scan_bwd_noalloc only, one built-in scratch array per device with a per-device address
 *    cache behind a mutex. Calls from several host threads on different streams are safe, except
 *    that ssm_scan_bwd_noalloc calls must not overlap on one device (they share that array).
 *  - Layouts are dense, row-major, innermost axis last: activations (Bt, Dn, L) with L
 *    contiguous; B and C (Bt, N, L) with L contiguous; per-channel parameters fp32.
 *    conv_w is [Dn, K] (each channel's taps contiguous, tap 0 = the current token), i.e. the
 *    transpose of the page's [kernelWidth, innerWidth] orientation.
 *  - Validation is synchronous on the host and happens before any launch; on an error nothing
 *    is launched. Execution is asynchronous on `stream` (a cudaStream_t passed as void*; NULL =
 *    the legacy default stream). A returned SSM_OK means the launches were enqueued; later
 *    device faults surface on the stream as usual.
 *  - Sizes: Dn, N and (with a conv) K must be >= 1 (SSM_ERR_SHAPE otherwise); Bt = 0 or L = 0 is
 *    a valid empty problem and returns SSM_OK without launching anything.
 *  - Alignment: every tensor pointer must be aligned to its element size (SSM_ERR_ALIGN).
 *    Inputs whose rows are also 16-byte aligned (L * element size a multiple of 16 and 16-byte
 *    aligned bases) take the 128-bit cp.async path; others take a scalar-load path.
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ssm_status {
  SSM_OK = 0,
  SSM_ERR_NULL = 1,        /* a required pointer is NULL */
  SSM_ERR_SHAPE = 2,       /* negative size, empty internal axis, or size overflow */
  SSM_ERR_ALIGN = 3,       /* a pointer is not aligned to its element type */
  SSM_ERR_DTYPE = 4,       /* unknown dtype code */
  SSM_ERR_UNSUPPORTED = 5, /* d_state > 64 or K > 4 */
  SSM_ERR_CUDA = 6,        /* a CUDA call or launch failed; see ssm_last_cuda_error() */
  SSM_ERR_WORKSPACE = 7,   /* workspace NULL or smaller than ssm_*_workspace_size() */
  SSM_ERR_TIMEOUT = 8      /* a bounded device-side wait ran out (ssm_ssd_check,
                              ssm_wait_selftest); the CUDA context stays usable */
} ssm_status;

typedef enum ssm_dtype { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

/* Input discretisation. SSM_ZOH: B_bar = (A_bar - 1)/A * B, the exact zero-order hold
 * ("Sequence and state-space models", ssm_discretize_b). SSM_EULER: B_bar = Delta * B, Mamba's
 * first-order simplification ("Sequence and state-space models", mamba_selective_scan_step;
 * "Selective Mamba", step). A_bar = exp(Delta * A) in both. */
typedef enum ssm_discretization { SSM_ZOH = 0, SSM_EULER = 1 } ssm_discretization;

/* How the forward's one-pass scan is laid out on the GPU (both compute the same outputs; fp32
 * rounding differs). SSM_SCAN_LANES: a channel's states are spread over lanes that each walk the
 * whole sequence in time order. SSM_SCAN_CHUNKED: lanes own consecutive time steps; each 64-step
 * chunk of a channel is scanned in parallel -- every lane runs its 8 steps from a zero state, an
 * associative warp-shuffle scan of the (product of A_bar, end state) pairs gives every lane the
 * state entering its steps ("State-Space Models & Long-Context Sequence Architectures (Mamba)",
 * Lab 3; "state-space models", "One recurrence, one convolution"), and the chunk's end state is
 * carried into the next chunk. Split-L calls (ssm_fwd_args.n_segments) use the lane layout. */
typedef enum ssm_scan_form { SSM_SCAN_LANES = 0, SSM_SCAN_CHUNKED = 1 } ssm_scan_form;

/* Time steps between saved states (chunk_states) and of the backward's recompute blocks. */
#define SSM_STATE_CHUNK 16

/* Number of saved states per channel for a sequence of length L: ceil(L / SSM_STATE_CHUNK). */
int64_t ssm_num_state_chunks(int64_t L);

/*
 * Forward arguments. The activations x, dt, z, B, C share one dtype (in_dtype); out and u_out
 * share out_dtype. fp32 inputs select the accurate math path (library expf/expm1f/log1pf);
 * bf16 inputs select the fast path (hardware ex2/lg2/rcp approximations).
 */
typedef struct ssm_fwd_args {
  const void *x;         /* device (Bt, Dn, L): pre-conv input when conv_w != NULL, else u itself */
  const void *dt;        /* device (Bt, Dn, L): time-step input before dt_bias / softplus */
  const float *dt_bias;  /* device [Dn] or NULL (= 0) */
  const float *A_log;    /* device [Dn, N]: A = -exp(A_log) */
  const void *B;         /* device (Bt, N, L): input state vectors, shared by all channels */
  const void *C;         /* device (Bt, N, L): readout state vectors, shared by all channels */
  const float *D;        /* device [Dn] or NULL (= 0): skip coefficient on u */
  const void *z;         /* device (Bt, Dn, L) or NULL: no SiLU(z) gate */
  const float *conv_w;   /* device [Dn, K] newest-first taps, or NULL: no conv (x is u) */
  const float *conv_b;   /* device [Dn] or NULL (= 0); ignored without conv_w */
  void *out;             /* device (Bt, Dn, L), out_dtype: the gated output */
  float *chunk_states;   /* device (Bt, Dn, ssm_num_state_chunks(L), N) fp32 or NULL: h after
                            every SSM_STATE_CHUNK-th step (the last entry after step L-1);
                            ssm_scan_bwd consumes them */
  void *u_out;           /* device (Bt, Dn, L), out_dtype, or NULL: the scan input u */
  int64_t Bt, Dn, N, L;  /* batch, channels (d_inner), states (d_state), sequence length */
  int32_t K;             /* conv taps, 1..4 (ignored without conv_w) */
  int32_t in_dtype;      /* ssm_dtype of x, dt, z, B, C */
  int32_t out_dtype;     /* ssm_dtype of out and u_out */
  int32_t delta_softplus;/* 1: Delta = softplus(dt + dt_bias); 0: Delta = dt + dt_bias */
  /* State carried between calls ("Selective Mamba", State / runArray): a sequence processed as
   * consecutive chunks, each call given the previous call's h_last and conv_hist_out, produces
   * exactly the outputs of one call over the whole sequence. */
  const float *h0;       /* device (Bt, Dn, N) fp32 or NULL (= 0): the state before step 0 */
  const void *conv_hist; /* device (Bt, Dn, K-1) in_dtype or NULL (= 0): the K-1 pre-conv inputs
                            before step 0, newest-first (ignored without conv_w) */
  float *h_last;         /* device (Bt, Dn, N) fp32 or NULL: the state after step L-1 */
  void *conv_hist_out;   /* device (Bt, Dn, K-1) in_dtype or NULL: the K-1 newest pre-conv inputs
                            after this call, newest-first (may alias conv_hist) */
  int32_t discretization;/* ssm_discretization */
  /* Split-L, for long sequences with few channels ("Sequence and state-space models", the
   * chunked scan of affine pairs; "Selective Mamba", runArray over consecutive chunks): the
   * sequence is cut into segments that run in parallel -- (1) every segment but the last runs
   * from a zero state and keeps its end state and its sum of Delta, (2) the start state of every
   * segment follows from those in one pass over the segments (the product of a segment's A_bar
   * is exp(A * its sum of Delta)), (3) every segment runs from its start state, its conv prefix
   * read from x. The results equal one pass up to fp32 rounding; the arithmetic is about 1.6x,
   * for up to n_segments times the parallelism. ssm_scan_bwd splits the same way, from the end:
   * (1) every segment but the first runs the adjoint backwards from a zero arrival (it needs
   * only Delta, dy and C) and keeps A_bar_ts lambda_ts, (2) the gradient arriving at every
   * segment's last state follows in one pass from the end, (3) every segment runs the full
   * backward from its arrival; then each segment's conv-history gradient is added into the
   * previous segment's last K-1 steps of dx. The backward reads n_segments from its fwd
   * block; its scratch comes from the backward workspace (workspace / workspace_bytes below are
   * the forward's only). */
  int32_t n_segments;    /* 0 or 1: one pass. >= 2: up to that many segments, each a multiple of
                            64 steps long. -1: chosen from the current device's SM count and the
                            shape (one pass when the one-pass grid fills the SMs once; else enough
                            segments for one wave (very few channels) or about two). */
  void *workspace;       /* device scratch of at least ssm_fwd_workspace_size() bytes, 256-byte
                            aligned, when the call splits L; may be NULL otherwise */
  size_t workspace_bytes;
  int32_t scan_form;     /* ssm_scan_form of a one-pass call (0 = SSM_SCAN_LANES) */
} ssm_fwd_args;

/*
 * Forward selective scan with the causal depthwise conv1d + SiLU fused in front and the SiLU(z)
 * gate fused behind: computes every output listed in ssm_fwd_args on `stream`.
 * Errors: SSM_ERR_NULL (x, dt, A_log, B, C or out NULL), SSM_ERR_SHAPE (also n_segments < -1),
 * SSM_ERR_ALIGN, SSM_ERR_DTYPE, SSM_ERR_UNSUPPORTED (N > 64, K outside 1..4, an unknown
 * discretization or scan_form), SSM_ERR_WORKSPACE
 * (a split-L call whose workspace is NULL, too small or not 256-byte aligned), SSM_ERR_CUDA.
 */
ssm_status ssm_scan_fwd(const ssm_fwd_args *args, void *stream);

/*
 * Mamba-2 state-space duality (SSD) forward ("state-space models", "Mamba-2 and state-space
 * duality"). Within a head h the transition is a scalar multiple of the identity, A_bar_t = a_t I:
 *
 *   Delta_t = softplus(dt_t + dt_bias[h])   (or dt_t + dt_bias[h] when delta_softplus = 0, which
 *             must then be >= 0: a step size; a negative one makes a_t > 1 and the chunk-local
 *             decay factors e^{cum_t - cum_s} can overflow fp32)
 *   a_t     = exp(Delta_t A_h),  A_h = -exp(A_log[h])
 *   B_bar_t = beta_t B_t,  beta_t = (a_t - 1) / A_h (exact ZOH) or Delta_t (SSM_EULER)
 *   h_t     = a_t h_{t-1} + B_bar_t x_t^T       (N x P per head; h_{-1} = h0 or 0)
 *   y_t     = h_t^T C_t + D[h] x_t
 *
 * i.e. y_t = sum_{s<=t} (C_t . B_bar_s) (prod_{k=s+1..t} a_k) x_s + D x_t = (L o C B_bar^T) X.
 * Computed in chunks of 128 steps: matrix products within a chunk on the tensor cores (bf16
 * operands, fp32 accumulation), the N x P state carried between chunks in fp32. B and C are
 * shared by all heads of a batch element (one group). Supported: bf16 inputs, P (head dim) 64 or
 * 128, N (state) 64 or 128 (SSM_ERR_UNSUPPORTED otherwise).
 */
/* How ssm_ssd_fwd schedules the chunks.
 *   SSM_SSD_AUTO       the fused form where it applies (P = 64), else the three-pass form.
 *   SSM_SSD_THREE_PASS three launches: every chunk's state product in parallel, the carry of the
 *                      states over the chunks (fp32, through the workspace), every chunk's output
 *                      in parallel.
 *   SSM_SSD_FUSED      one launch: one CTA per (batch, head) walks the chunks in order with the
 *                      state in tensor memory, tiles loaded by TMA; P = 64 only
 *                      (SSM_ERR_UNSUPPORTED otherwise). */
typedef enum ssm_ssd_form { SSM_SSD_AUTO = 0, SSM_SSD_THREE_PASS = 1, SSM_SSD_FUSED = 2 } ssm_ssd_form;

typedef struct ssm_ssd_args {
  const void *x;         /* device (Bt, H, L, P) bf16, 16-byte aligned */
  const void *dt;        /* device (Bt, H, L) bf16 */
  const float *dt_bias;  /* device [H] or NULL (= 0) */
  const float *A_log;    /* device [H] */
  const void *B;         /* device (Bt, L, N) bf16, 16-byte aligned */
  const void *C;         /* device (Bt, L, N) bf16, 16-byte aligned */
  const float *D;        /* device [H] or NULL (= 0) */
  const float *h0;       /* device (Bt, H, N, P) fp32, 16-byte aligned, or NULL (= 0) */
  void *y;               /* device (Bt, H, L, P) out_dtype, 16-byte aligned */
  float *h_last;         /* device (Bt, H, N, P) fp32, 16-byte aligned, or NULL: the state after
                            step L-1 */
  int64_t Bt, H, L, P, N;
  int32_t in_dtype;      /* must be SSM_BF16 */
  int32_t out_dtype;     /* SSM_BF16 or SSM_F32 */
  int32_t delta_softplus;
  int32_t discretization;/* ssm_discretization */
  void *workspace;       /* device scratch of ssm_ssd_workspace_size() bytes, 256-byte aligned */
  size_t workspace_bytes;
  void *const *timing_events; /* NULL, or 2 caller-created cudaEvent_t recorded on `stream`: with
                                 the fused form [0] just before its one launch and [1] just after;
                                 with the three-pass form around the output kernel (the last of the
                                 three launches). Recording does not synchronise. */
  int32_t form;          /* ssm_ssd_form: how the chunks are scheduled */
} ssm_ssd_args;

/* Scratch bytes ssm_ssd_fwd needs: the chunk states (fp32), the state entering every chunk
 * (bf16), one log-decay per chunk, and an error word; 0 for an empty or invalid problem. */
size_t ssm_ssd_workspace_size(const ssm_ssd_args *args);

/* Errors: SSM_ERR_NULL, SSM_ERR_SHAPE (negative sizes, H/P/N = 0), SSM_ERR_ALIGN,
 * SSM_ERR_DTYPE (codes), SSM_ERR_UNSUPPORTED (in_dtype not bf16, P not 64/128, N not 64/128, an
 * unknown form, SSM_SSD_FUSED with P != 64),
 * SSM_ERR_WORKSPACE, SSM_ERR_CUDA. Bt = 0 or L = 0: nothing to do (h_last = h0 or 0). */
ssm_status ssm_ssd_fwd(const ssm_ssd_args *args, void *stream);

/* Failure detection for ssm_ssd_fwd. Its kernels wait for every tensor-core product through an
 * mbarrier, polling a bounded number of times (2^18, about one second on B200, where a failed poll
 * takes about 4 us); a wait that runs out sets an error word in
 * the workspace (zeroed at the start of every ssm_ssd_fwd), and the kernel still releases its
 * tensor memory and exits, so the context stays usable. This call SYNCHRONISES `stream`, reads the
 * word of the latest ssm_ssd_fwd that used args->workspace, and returns SSM_ERR_TIMEOUT when it is
 * set, SSM_OK otherwise. Same argument checks as ssm_ssd_fwd (plus SSM_ERR_WORKSPACE); SSM_ERR_CUDA
 * when the copy or the synchronisation fails. */
ssm_status ssm_ssd_check(const ssm_ssd_args *args, void *stream);

/* Self-test of that timeout path on the current device: one CTA of 128 threads waits, polling at
 * most `polls` times (1..2^22), on a shared-memory mbarrier that expects one arrival. With arrive
 * != 0 one thread arrives first and the wait succeeds (SSM_OK); with arrive = 0 nothing arrives, the
 * wait runs out and the kernel sets *error_word (device int32, 4-byte aligned, zeroed here first)
 * through the same bounded wait the SSD kernels use; the call then returns SSM_ERR_TIMEOUT.
 * Synchronises `stream`. Errors: SSM_ERR_NULL, SSM_ERR_ALIGN, SSM_ERR_SHAPE (polls out of range),
 * SSM_ERR_CUDA. */
ssm_status ssm_wait_selftest(int32_t arrive, int32_t polls, int32_t *error_word, void *stream);

/* Bytes of workspace ssm_scan_fwd needs for these arguments: 0 when the call runs in one pass
 * (n_segments 0 or 1, or a split that would leave a single segment), else 2 (n Bt Dn N) + n Bt Dn
 * floats for n segments (each array rounded up to 256 bytes). With n_segments = -1 the answer
 * depends on the current device (its SM count is read). Returns 0 for invalid arguments. */
size_t ssm_fwd_workspace_size(const ssm_fwd_args *args);

/*
 * Backward arguments: the forward's inputs (same meaning and dtypes; out/u_out unused) plus the
 * upstream gradient and the gradient outputs. Every gradient output is fp32, caller-allocated,
 * OVERWRITTEN (never accumulated into) and may be NULL when not wanted.
 */
typedef struct ssm_bwd_args {
  ssm_fwd_args fwd;            /* forward inputs; fwd.out and fwd.u_out are ignored */
  const void *dout;            /* device (Bt, Dn, L), fwd.in_dtype: dLoss/dout */
  const float *chunk_states;   /* device states saved by ssm_scan_fwd, or NULL: recomputed into
                                  the workspace */
  float *dx;      /* (Bt, Dn, L): w.r.t. the pre-conv x, or w.r.t. u when there is no conv */
  float *ddt;     /* (Bt, Dn, L): w.r.t. dt (before dt_bias / softplus) */
  float *dz;      /* (Bt, Dn, L): w.r.t. z (ignored without a gate) */
  float *dA_log;  /* [Dn, N] */
  float *dB;      /* (Bt, N, L) */
  float *dC;      /* (Bt, N, L) */
  float *dD;      /* [Dn] */
  float *ddt_bias;/* [Dn] */
  float *dconv_w; /* [Dn, K] (ignored without a conv) */
  float *dconv_b; /* [Dn]    (ignored without a conv) */
  void *workspace;          /* device scratch of at least ssm_bwd_workspace_size() bytes,
                               256-byte aligned; contents need not be initialised */
  size_t workspace_bytes;
  void *const *timing_events; /* NULL, or 2 caller-created cudaEvent_t: [0] is recorded on
                                 `stream` just before the main backward kernel, [1] just after it
                                 (before the cross-tile reductions); lets a caller time the
                                 kernel alone. Recording does not synchronise. */
  const float *dh_last;  /* (Bt, Dn, N) or NULL: gradient arriving at fwd.h_last (the next
                            chunk's dh0 when chunks are chained) */
  float *dh0;            /* (Bt, Dn, N) or NULL: gradient w.r.t. fwd.h0 */
  float *dconv_hist;     /* (Bt, Dn, K-1) or NULL: gradient w.r.t. fwd.conv_hist. When chunks are
                            chained, add it to the previous chunk's dx over its last K-1 steps
                            (entry j belongs to step L-1-j). */
} ssm_bwd_args;

/* Bytes of device scratch ssm_scan_bwd needs for these arguments (0 for an empty problem). */
size_t ssm_bwd_workspace_size(const ssm_bwd_args *args);

/*
 * Workspace bytes from the forward arguments alone: for_bwd = 0 gives ssm_fwd_workspace_size(args);
 * for_bwd != 0 gives ssm_bwd_workspace_size() of a backward whose fwd block is *args and which is
 * handed saved states exactly when args->chunk_states is not NULL (the forward that saved them).
 * The caller allocates the answer (256-byte aligned) and passes it as `workspace`. 0 when nothing
 * is needed or the arguments are invalid.
 */
size_t ssm_workspace_size(const ssm_fwd_args *args, int32_t for_bwd);

/*
 * Backward (vector-Jacobian product) of ssm_scan_fwd against `dout`: the reverse-time adjoint
 * recurrence lambda_t = C_t * dy_t + A_bar_{t+1} * lambda_{t+1} over the states recomputed from
 * chunk_states, with all parameter gradients. Always deterministic -- there is no switch for it,
 * and no faster non-deterministic variant: every cross-channel and cross-batch sum (dB, dC and the
 * per-channel parameter gradients) is reduced in a fixed order without atomics, so the same
 * inputs on the same device give bit-identical gradients on every run. Errors as ssm_scan_fwd,
 * plus SSM_ERR_WORKSPACE.
 */
ssm_status ssm_scan_bwd(const ssm_bwd_args *args, void *stream);

/*
 * Single-token decode step ("Selective Mamba", step): advance every channel by one token, reading
 * and updating the carried state in place. Same arithmetic as ssm_scan_fwd with L = 1, h0 =
 * h_last = h and conv_hist = conv_hist_out = conv_hist, without the scan machinery.
 */
typedef struct ssm_step_args {
  const void *x;        /* device (Bt, Dn) in_dtype: this token's pre-conv input (u without conv) */
  const void *dt;       /* device (Bt, Dn) in_dtype */
  const float *dt_bias; /* device [Dn] or NULL */
  const float *A_log;   /* device [Dn, N] */
  const void *B;        /* device (Bt, N) in_dtype */
  const void *C;        /* device (Bt, N) in_dtype */
  const float *D;       /* device [Dn] or NULL */
  const void *z;        /* device (Bt, Dn) in_dtype or NULL */
  const float *conv_w;  /* device [Dn, K] or NULL */
  const float *conv_b;  /* device [Dn] or NULL */
  float *h;             /* device (Bt, Dn, N) fp32: state, read then overwritten */
  void *conv_hist;      /* device (Bt, Dn, K-1) in_dtype: history, read then overwritten (with a
                           conv; may be NULL without one) */
  void *out;            /* device (Bt, Dn) out_dtype */
  int64_t Bt, Dn, N;
  int32_t K, in_dtype, out_dtype, delta_softplus, discretization;
} ssm_step_args;

/* One decode step. Errors: SSM_ERR_NULL, SSM_ERR_SHAPE, SSM_ERR_ALIGN, SSM_ERR_DTYPE,
 * SSM_ERR_UNSUPPORTED, SSM_ERR_CUDA. Bt = 0 is a no-op. */
ssm_status ssm_scan_step(const ssm_step_args *args, void *stream);

/* Size of the scratch array built into the library for ssm_scan_bwd_noalloc (72 MiB). */
#define SSM_NOALLOC_SCRATCH_BYTES (72u << 20)

/*
 * ssm_scan_bwd_noalloc -- the same backward as ssm_scan_bwd for callers that cannot allocate device
 * memory (a host program or plugin that only receives device pointers and has no allocator, or
 * code running where allocating is not permitted). The pages describe no such entry point: it has
 * no counterpart there and exists only for these callers.
 *
 * Arguments are those of ssm_scan_bwd; args->workspace and args->workspace_bytes are ignored.
 * Scratch comes from one library-owned device array of SSM_NOALLOC_SCRATCH_BYTES per GPU, held
 * until the process exits. When ssm_bwd_workspace_size() exceeds that size, the call runs with
 * thread-block clusters of 4 or 8 CTAs that add their dB / dC partial sums on chip, dividing that
 * part of the scratch by 4 or 8 (measured on B200: 6% slower with 4, 1.6x with 8; the results
 * stay deterministic and agree with ssm_scan_bwd up to fp32 summation order): e.g. 4 x 4096 x 16
 * x 4096 with saved states needs 257 MiB regularly and 65 MiB with clusters of 4. Problems that do not fit even so are rejected with SSM_ERR_WORKSPACE before
 * anything runs (pass chunk_states from the forward to keep the requirement small). The first call on a device looks up the array's device address (a runtime
 * API call): make it before any stream capture on that device. All calls on a device share the
 * array, so calls that overlap on the GPU race; order them (one stream, or events). The call
 * allocates nothing (no cudaMalloc / cudaFree). Errors: as ssm_scan_bwd; SSM_ERR_CUDA also when
 * the current device or the array's address cannot be read (ssm_last_cuda_error() says why), and
 * SSM_ERR_UNSUPPORTED on a device index of 64 or more.
 */
ssm_status ssm_scan_bwd_noalloc(const ssm_bwd_args *args, void *stream);

/*
 * Standalone causal depthwise conv1d + SiLU: u = SiLU(b + sum_k w[k] * x_{t-k}).
 * x: device (Bt, Dn, L) in_dtype; u: device (Bt, Dn, L) out_dtype; w: device [Dn, K] fp32,
 * newest-first; b: device [Dn] fp32 or NULL. K in 1..4.
 * Errors: SSM_ERR_NULL, SSM_ERR_SHAPE, SSM_ERR_ALIGN, SSM_ERR_DTYPE, SSM_ERR_UNSUPPORTED,
 * SSM_ERR_CUDA.
 */
ssm_status ssm_conv1d_silu(const void *x, void *u, const float *w, const float *b, int64_t Bt,
                           int64_t Dn, int64_t L, int32_t K, int32_t in_dtype, int32_t out_dtype,
                           void *stream);

/* Static description of a status code (never NULL). */
const char *ssm_status_string(ssm_status s);

/* The cudaError_t (as int) behind the calling thread's most recent SSM_ERR_CUDA, or 0. */
int ssm_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
