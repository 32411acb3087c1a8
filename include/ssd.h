/*
 * ssd.h -- C ABI of libssd_b200: the forward pass of the chunked SSD scan
 * (the state-space-duality layer of Mamba-2) on NVIDIA B200 (sm_100a).
 *
 * What is computed ("Transformers are SSMs: Generalized Models and Efficient
 * Algorithms Through Structured State Space Duality", paperlayer.ai summary):
 * the selective SSM with scalar-times-identity transitions (§2.4), per head h
 * and token t of a document, with g = h / (H/G) the B/C group of the head
 * (shared B, C across heads, §7.1-§7.2):
 *
 *     delta_t = softplus(dt[t,h] + dt_bias[h])
 *     S_t     = exp(delta_t A[h]) S_{t-1} + delta_t B[t,g,:]^T x[t,h,:]      (N x P)
 *     y[t,h]  = C[t,g,:] S_t + D[h] x[t,h,:]
 *
 * with S_{start-1} the document's initial state, evaluated by the block
 * decomposition of §6: quadratic (masked attention) form on the diagonal
 * blocks (§6.1), chunk states from the right factors, a scalar scan of states
 * across chunks and outputs from the left factors (§6.2).  Documents never
 * exchange information (§8.3 Variable Length); the final state of each
 * document is returned so that a later call can continue from it (§8.2
 * Sequence Parallelism: each worker starts from an initial state and passes
 * its final state on).
 *
 * Conventions for every entry point:
 *  - Return value: SSD_OK (0) or a negative SSD_ERR_* code.  No C++ exception
 *    crosses this boundary.  ssd_error_string() names a code.
 *  - Device pointers are CUDA global-memory pointers on the handle's device,
 *    contiguous, row-major (last index fastest), 16-byte aligned.  The caller
 *    owns every buffer it passes; the library only reads inputs and writes
 *    outputs during the work it enqueues.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous: ssd_forward never synchronises.  Buffers
 *    must stay valid until that work completes.
 *  - A handle is not thread-safe: concurrent ssd_forward calls on one handle
 *    share its workspace and race.  Use one handle per stream.
 *  - Device-side failures (an invalid cu_seqlens array, a bounded wait that
 *    gave up) are recorded in a status word read by ssd_get_status().
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

typedef struct CUstream_st* ssd_stream_t; /* same type as cudaStream_t */

/* element types */
enum { SSD_F32 = 0, SSD_BF16 = 1 };

/* return codes */
enum {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = -1, /* null required pointer, bad size, misaligned pointer */
  SSD_ERR_UNSUPPORTED = -2, /* shape or dtype outside what the library implements */
  SSD_ERR_CUDA = -3,        /* a CUDA runtime call or kernel launch failed */
  SSD_ERR_TIMEOUT = -4,     /* a device-side bounded wait gave up (status word) */
  SSD_ERR_OOM = -5,         /* device allocation failed */
  SSD_ERR_BAD_SEQLENS = -6, /* cu_seqlens not 0 = c[0] <= ... <= c[n] = tokens (status word) */
  SSD_ERR_SCRATCH_TOO_SMALL = -7, /* ssd_forward_noalloc: problem needs more than its fixed scratch */
  SSD_ERR_DEBUG_CHECK = -8  /* debug builds only (SSD_DEBUG): a device-side bounds or barrier-phase
                             * check failed (status word; the offending source line is in the
                             * word after it) */
};

/* kernel paths (ssd_plan_t.path, SSD_OPT_FORCE_PATH) */
enum {
  SSD_PATH_AUTO = -1,
  SSD_PATH_SIMT = 0, /* chunk-parallel CUDA-core kernels, fp32 arithmetic (any shape, f32 or bf16) */
  SSD_PATH_TC = 1    /* fused persistent tcgen05/TMEM kernel (bf16 inputs, fp32 accumulate) */
};

/* handle options (ssd_set_option) */
enum {
  SSD_OPT_FORCE_PATH = 1, /* value: SSD_PATH_AUTO (default), SSD_PATH_SIMT or SSD_PATH_TC */
  /* value: 64 (default) or 128, the column width of the tensor-core kernel's work
   * units.  128-column units pair two heads of P = 64 that share a B/C group (or
   * take 128 columns of one head with P = 128 or 256), computing C B^T once for
   * the pair and the state update and left factors as N = 128 products; they need
   * dstate <= 128.  On a shape they do not cover, ssd_forward returns
   * SSD_ERR_UNSUPPORTED.  Both widths compute the same result. */
  SSD_OPT_TC_UNIT_COLUMNS = 2,
  /* value: 1 .. 60,000,000 microseconds (default 2,000,000), the bound of every
   * device-side wait of the tensor-core forward.  A value other than the default
   * selects the tensor-core kernel with the register-resident state chain for every
   * N <= 256 (it is the default kernel for N > 128; the one for N <= 128 bounds its
   * waits at the default).  A wait that runs out records SSD_ERR_TIMEOUT in the
   * status word (ssd_get_status) and the kernel unwinds, leaving the outputs of
   * that call undefined and the handle and context usable. */
  SSD_OPT_WAIT_LIMIT_US = 3,
  /* value: 0 (default) or 1.  Failure-path test: with 1, every following
   * ssd_forward on the tensor-core path (64-column units) first waits on
   * a device barrier that nothing completes, so that wait runs out after the
   * SSD_OPT_WAIT_LIMIT_US bound and the call reports SSD_ERR_TIMEOUT through the
   * status word.  No GPU fault is involved.  Set it back to 0 to compute again. */
  SSD_OPT_TEST_FORCE_TIMEOUT = 4
};

/*
 * Problem description, fixed for the life of a handle.
 *   batch, seqlen   sequences of `seqlen` tokens each; tokens = batch * seqlen.
 *   nheads H, headdim P, dstate N, ngroups G (H % G == 0; head h reads group
 *                   h / (H/G)).  Typical head dimensions are 64 and 128 (§2.4).
 *   in_dtype        SSD_F32 or SSD_BF16: the type of x, dt, B and C.
 *   out_dtype       SSD_F32 or SSD_BF16: the type of y.
 *   max_docs        0: sequences are the batch rows.  > 0: ssd_forward may be
 *                   given cu_seqlens with up to max_docs documents packed into
 *                   one row (then batch must be 1; §8.3 padding-free packing).
 *   flags           reserved, must be 0.
 */
typedef struct {
  int64_t batch;
  int64_t seqlen;
  int32_t nheads;
  int32_t headdim;
  int32_t dstate;
  int32_t ngroups;
  int32_t in_dtype;
  int32_t out_dtype;
  int32_t max_docs;
  int32_t flags;
} ssd_desc_t;

typedef struct ssd_handle_s* ssd_handle_t;

/* What ssd_forward would run for a given call (host-only query, no GPU needed). */
typedef struct {
  int32_t path;            /* SSD_PATH_SIMT or SSD_PATH_TC */
  int32_t num_docs;        /* documents of the call */
  int64_t num_chunks_max;  /* upper bound on chunks (SIMT path) */
  int64_t workspace_bytes; /* device workspace the call needs */
  int32_t units;           /* work units of the TC path (document x head x P-slice), else 0 */
  int32_t kernels;         /* kernel launches one ssd_forward call makes */
} ssd_plan_t;

/*
 * ssd_validate_desc: checks a description without touching the GPU.
 * Returns SSD_OK, SSD_ERR_INVALID_ARG (non-positive sizes, bad dtype, flags != 0,
 * max_docs > 0 with batch != 1) or SSD_ERR_UNSUPPORTED (H % G != 0,
 * P or N outside [1, 256]).
 */
SSD_API int ssd_validate_desc(const ssd_desc_t* desc);

/*
 * ssd_plan: the kernel path and workspace a call with this chunk size and
 * document count would use (num_docs = 0 for batch mode).  Host only.
 * chunk_size must be in [1, 256] (the chunk length Q of §6).
 */
SSD_API int ssd_plan(const ssd_desc_t* desc, int chunk_size, int num_docs, ssd_plan_t* out);

/*
 * ssd_create: validates `desc`, selects the current CUDA device, allocates a
 * small device status word and returns a handle in *out.  Workspace for the
 * chunk-parallel path is allocated on first use by ssd_forward, stream-ordered
 * (cudaMallocAsync on the call's stream), and grown when a later call needs
 * more.  Errors: those of ssd_validate_desc, SSD_ERR_CUDA, SSD_ERR_OOM.
 */
SSD_API int ssd_create(const ssd_desc_t* desc, ssd_handle_t* out);

/* ssd_set_option: see SSD_OPT_*.  SSD_ERR_INVALID_ARG for an unknown option or value. */
SSD_API int ssd_set_option(ssd_handle_t h, int option, int value);

/*
 * ssd_forward: y, final_states = SSD(x, dt, A, B, C, D, dt_bias, initial_states).
 *
 *   x        [batch, seqlen, H, P]  in_dtype     (device)
 *   dt       [batch, seqlen, H]     in_dtype     (device) raw step before softplus
 *   A        [H] float32, negative               (device) scalar-times-identity A (§2.4)
 *   B, C     [batch, seqlen, G, N]  in_dtype     (device)
 *   D        [H] float32 or NULL (no skip term)  (device)
 *   dt_bias  [H] float32 or NULL (zero bias)     (device)
 *   chunk_size  Q in [1, 256]: the chunk length of the block decomposition.
 *               The result does not depend on Q except through rounding.
 *   initial_states  [ndocs, H, N, P] float32 or NULL (zero)  (device)
 *   cu_seqlens  NULL (documents = batch rows, ndocs = batch) or int32
 *               [num_docs + 1] on the device with 0 = c[0] <= c[1] <= ... <=
 *               c[num_docs] = batch*seqlen (empty documents allowed); needs
 *               batch == 1 and 1 <= num_docs <= max_docs.  A violation found on
 *               the device sets SSD_ERR_BAD_SEQLENS in the status word and the
 *               call then writes no output.
 *   num_docs    documents in cu_seqlens (ignored when cu_seqlens is NULL).
 *   y        [batch, seqlen, H, P] out_dtype (device, written)
 *   final_states [ndocs, H, N, P] float32 or NULL (device, written): the state
 *               after each document's last token (its initial state if empty).
 * Errors (before anything is enqueued): SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED
 * (a forced path that cannot run this shape), SSD_ERR_OOM; SSD_ERR_CUDA if a
 * launch fails.
 */
SSD_API int ssd_forward(ssd_handle_t h, const void* x, const void* dt, const float* A,
                const void* B, const void* C, const float* D, const float* dt_bias,
                int chunk_size, const float* initial_states, const int32_t* cu_seqlens,
                int num_docs, void* y, float* final_states, ssd_stream_t stream);

/*
 * ssd_forward_host: the same computation with every array in HOST memory
 * (pageable or pinned; cu_seqlens too, then num_docs is read from the caller).
 * Copies the inputs to handle-owned device buffers on `stream`, runs
 * ssd_forward, copies y and final_states back, and synchronises `stream`
 * before returning.  The device buffers are allocated on first use and kept.
 */
SSD_API int ssd_forward_host(ssd_handle_t h, const void* x, const void* dt, const float* A,
                     const void* B, const void* C, const float* D, const float* dt_bias,
                     int chunk_size, const float* initial_states, const int32_t* cu_seqlens,
                     int num_docs, void* y, float* final_states, ssd_stream_t stream);

/*
 * ssd_backward: the gradient of the forward pass.  The pages give only its cost
 * ("Transformers are SSMs", paperlayer.ai summary: training FLOPs of the SSD layer,
 * §6); what it computes is the derivative of the same recurrence, taken through
 * the block decomposition of §6 one chunk at a time.  For the loss
 *
 *   sum over tokens, heads of <dy, y>  +  sum over documents, heads of <dfinal_states, final_states>
 *
 * it writes the gradient with respect to every input of ssd_forward.  The handle,
 * the problem (desc, cu_seqlens, num_docs) and the inputs x, dt, A, B, C, D,
 * dt_bias, initial_states are exactly those of the forward call being
 * differentiated; the forward's outputs are not needed (the states are recomputed).
 *   dy              [batch, seqlen, H, P] out_dtype (the cotangent of y; required)
 *   dfinal_states   [docs, H, N, P] fp32 or NULL (zero)
 * Outputs, fp32, device, owned by the caller, overwritten:
 *   dx [batch, seqlen, H, P]; ddt [batch, seqlen, H]; dB, dC [batch, seqlen, G, N]
 *   (summed over the heads of each group); dA [H]; dD [H] and ddt_bias [H]
 *   (either may be NULL: not computed); dinitial_states [docs, H, N, P] or NULL.
 * The chunk size is the backward's own, whatever the forward used (the chunking
 * changes only rounding).  bf16 inputs and outputs with headdim a multiple of 64
 * (up to 256), dstate 64 or 128 and 16-byte aligned x, B, C, dy, dx, dB and dC run
 * on the tensor cores with 128-token chunks, one slice of 64 head-dimension columns
 * per block: bf16 operands, the in-chunk weighted matrices and the cotangent as
 * hi + lo bf16 pairs, fp32 accumulation.  Everything else runs on the CUDA cores in
 * fp32 with 64-token chunks.  dB, dC, dA, dD and ddt_bias (and ddt, when the head
 * dimension has more than one slice) are sums of fp32 atomic additions, so their
 * last bits can differ from run to run.  Workspace grows in the handle as for ssd_forward.  Errors as for
 * ssd_forward; inputs need only element alignment.
 */
SSD_API int ssd_backward(ssd_handle_t h, const void* x, const void* dt, const float* A,
                         const void* B, const void* C, const float* D, const float* dt_bias,
                         const float* initial_states, const int32_t* cu_seqlens, int num_docs,
                         const void* dy, const float* dfinal_states, float* dx, float* ddt,
                         float* dA, float* dB, float* dC, float* dD, float* ddt_bias,
                         float* dinitial_states, ssd_stream_t stream);

/*
 * Feature maps and denominator normalisation ("Transformers are SSMs", paperlayer.ai
 * summary: §7.3, SSD extensions taken from linear attention; the kernel
 * approximations of §9.4.3 and App. D.4).  A feature map phi is applied to each
 * (token, group) row of B and of C before the scan:
 *   SSD_FMAP_SILU     phi(x) = x sigmoid(x), elementwise (the default of §7.3)
 *   SSD_FMAP_RELU     phi(x) = max(x, 0), elementwise
 *   SSD_FMAP_BASED    phi(x) = [1, x, (x outer x) / sqrt(2)] (second-order Taylor
 *                     expansion of exp(<a, b>)): dstate N becomes 1 + N + N^2
 *   SSD_FMAP_REBASED  phi(x) = x outer x (row-major flattening): N becomes N^2
 * With normalisation, y = num / den + D x, where num is the scan's output on x and
 * den the same scan on a column of ones (§7.3: X augmented with ones); phi should
 * be positive so that den is (ReLU, Based and ReBased are non-negative; SiLU is not).
 */
enum {
  SSD_FMAP_NONE = 0,
  SSD_FMAP_SILU = 1,
  SSD_FMAP_RELU = 2,
  SSD_FMAP_BASED = 3,
  SSD_FMAP_REBASED = 4
};

/* dstate of the scan after feature map `kind` on an input of dstate N; -1 if unknown. */
SSD_API int ssd_feature_map_dim(int kind, int dstate);

/*
 * ssd_forward_ext: ssd_forward with a feature map on B and C and optional
 * normalisation.  The handle's desc gives the input dstate N of B and C; the scan
 * runs with N' = ssd_feature_map_dim(feature_map, N) (which the tensor-core path
 * takes when N' is a multiple of 16 up to 256, else the CUDA-core path).  Arguments
 * as for ssd_forward, except:
 *   no initial states (the denominator's state would need one of its own);
 *   final_states [docs, H, N', P] fp32 or NULL: the numerator's final states;
 *   normalize 0 or 1.
 * The mapped B and C and the denominator live in the handle's workspace.  The
 * denominator is its own single-column scan in 64-token chunks and takes N' up to
 * 1024.  With normalisation the call takes one of two orders:
 *   - the denominator on a second CUDA stream that the handle creates on first use
 *     (non-blocking, destroyed by ssd_destroy), forked from `stream` after the feature
 *     maps and joined back into it before the division, so every result is still
 *     ordered on `stream` (a graph captured from `stream` takes both branches); used
 *     when the numerator leaves at least a quarter of the SMs idle;
 *   - otherwise everything on `stream`: the denominator first, then the numerator
 *     kernel with the division in its epilogue (tensor-core path, N' <= 128).
 * Calls on one handle must not overlap (they share the workspace and the second
 * stream).  Errors as for ssd_forward; SSD_ERR_INVALID_ARG for an unknown map,
 * SSD_ERR_UNSUPPORTED for a normalised N' over 1024.
 */
SSD_API int ssd_forward_ext(ssd_handle_t h, const void* x, const void* dt, const float* A,
                            const void* B, const void* C, const float* D, const float* dt_bias,
                            int chunk_size, const int32_t* cu_seqlens, int num_docs,
                            int feature_map, int normalize, void* y, float* final_states,
                            ssd_stream_t stream);

/*
 * ssd_get_status: synchronises `stream`, returns the first device-side error
 * recorded since the last call (SSD_OK if none) and clears it.
 */
SSD_API int ssd_get_status(ssd_handle_t h, ssd_stream_t stream);

/* ssd_destroy: synchronises the device and frees everything the handle owns. NULL is a no-op. */
SSD_API int ssd_destroy(ssd_handle_t h);

/*
 * ssd_step: one token of the recurrence for every sequence of a decode batch
 * ("Transformers are SSMs", paperlayer.ai summary: the recurrent, linear-time
 * mode of the selective SSM, §3.4.1, used to generate one token at a time; A is
 * a scalar times the identity, §2.4):
 *
 *   delta = softplus(dt + dt_bias[h]);  S <- exp(delta A[h]) S + delta B^T x;  y = C S + D[h] x
 *
 *   desc      batch = number of sequences, seqlen = 1, max_docs = 0; nheads,
 *             headdim (a multiple of 4, at most 1024), dstate, ngroups and the
 *             dtypes as for ssd_forward.
 *   x         [batch, H, P]  in_dtype      dt    [batch, H]  in_dtype
 *   A         [H] fp32 (required)          D, dt_bias [H] fp32, nullable (zero)
 *   B, C      [batch, G, N]  in_dtype (head h reads group h / (H/G))
 *   state     [batch, H, N, P] fp32, 16-byte aligned; read and updated in place:
 *             on return (in stream order) it holds the state after this token, so
 *             a prefill's final_states can be passed straight in
 *   y         [batch, H, P]  out_dtype
 * Device pointers, owned by the caller; asynchronous on `stream`; no handle and
 * no workspace.  SSD_ERR_INVALID_ARG for bad sizes, pointers or alignment,
 * SSD_ERR_UNSUPPORTED for a headdim the kernel does not take.  The step moves
 * 8 N P bytes of state per (sequence, head) and is bound by HBM bandwidth.
 */
SSD_API int ssd_step(const ssd_desc_t* desc, const void* x, const void* dt, const float* A,
                     const void* B, const void* C, const float* D, const float* dt_bias,
                     float* state, void* y, ssd_stream_t stream);

/*
 * Context-parallel forward: the three device steps of one rank.
 *
 * A batch of sequences is cut along the tokens into consecutive slices, one per
 * rank ("Transformers are SSMs", paperlayer.ai summary, §8.2: a worker hands its
 * final state to the next; the state-passing scan of §6.2, across workers).  Rank
 * r runs ssd_forward on its slice with no initial state, then:
 *   1. ssd_cp_logdecay: cs[b, t, h] = sum over the slice up to t of delta A, and
 *      logdecay[b, h] = cs at the slice's last token;
 *   2. (the caller all-gathers every rank's final state and logdecay)
 *   3. ssd_cp_combine: H_in = the state entering the slice, by the scan
 *      H_in(0) = init, H_in(k+1) = exp(logdecay_k) H_in(k) + S_k over ranks k < r;
 *      and the slice's true final state exp(logdecay_r) H_in + S_r;
 *   4. ssd_cp_correct: y[b, t, h, :] += exp(cs[b, t, h]) C[b, t, g, :] H_in[b, h]
 *      (the left factors of the entering state, §6.2).
 * desc describes the rank's slice in batch mode: batch rows of seqlen tokens,
 * max_docs = 0.  Device pointers owned by the caller, fp32 unless stated,
 * asynchronous on `stream`:
 *   dt [batch, L, H], C [batch, L, G, N] in_dtype;  A, dt_bias [H] (dt_bias nullable)
 *   cs [batch, L, H], logdecay [batch, H]
 *   local_final_all [nranks, batch, H, N, P], logdecay_all [nranks, batch, H]
 *   initial_states [batch, H, N, P] (nullable: zero), h_in and final_states
 *   [batch, H, N, P] (either may be NULL, not both), 16-byte aligned
 *   y [batch, L, H, P] out_dtype, read and updated (headdim a multiple of 4)
 *   status: one device int32 (nullable), set to SSD_ERR_TIMEOUT if a wait inside the
 *   tensor-core correction ran out (then y is incomplete); 0 is left untouched
 * ssd_cp_correct runs on the tensor cores for bf16 C with headdim and dstate
 * multiples of 64 up to 256, slices of at least 128 tokens and 16-byte aligned C
 * and y, else on the CUDA cores.
 * Errors: SSD_ERR_INVALID_ARG for bad sizes, ranks or pointers,
 * SSD_ERR_UNSUPPORTED for shapes the kernels do not take.
 */
SSD_API int ssd_cp_logdecay(const ssd_desc_t* desc, const void* dt, const float* A,
                            const float* dt_bias, float* cs, float* logdecay, ssd_stream_t stream);
SSD_API int ssd_cp_combine(const ssd_desc_t* desc, int rank, int nranks,
                           const float* local_final_all, const float* logdecay_all,
                           const float* initial_states, float* h_in, float* final_states,
                           ssd_stream_t stream);
SSD_API int ssd_cp_correct(const ssd_desc_t* desc, const void* C, const float* cs,
                           const float* h_in, void* y, int* status, ssd_stream_t stream);

/*
 * ssd_forward_noalloc: ssd_forward for callers that may not allocate device memory.
 * The paper has no counterpart to this entry point; it exists for deployment.
 *
 * Some callers cannot call cudaMalloc on the path that runs the layer: an
 * application that budgets all device memory up front through its own allocator,
 * or code that cannot afford the device-wide synchronisation an allocation may
 * cause.  This entry point takes no handle and allocates nothing.  The caller
 * passes every input and output exactly as for ssd_forward (same layouts,
 * alignment and stream semantics; `desc` describes the problem).  The computation
 * is the chunk-parallel CUDA-core path (the kernels ssd_forward runs with
 * SSD_PATH_SIMT) and gives its results.
 *
 * Its scratch memory is one fixed device array of SSD_NOALLOC_SCRATCH_BYTES
 * (32 MiB) inside the library, reserved on every device where the library's
 * kernels are loaded and held until the process exits.  A problem whose scratch
 * would exceed it (about chunks x H x N x P x 4 bytes plus 8 bytes per token and
 * head) is refused with SSD_ERR_SCRATCH_TOO_SMALL before any work is enqueued.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture.  The address is kept for the life of the process, so a
 * device reset (cudaDeviceReset) between calls is not supported.  All calls on a device share the one array and the previous
 * call's contents stay in it (nothing needs to start at zero), so calls whose GPU
 * work overlaps -- on different streams without ordering -- race and must be
 * serialised by the caller.
 *
 *   status   optional device int (NULL: none).  Set to 0 on `stream` at the start
 *            of the call; a device-side error (an invalid cu_seqlens array,
 *            SSD_ERR_BAD_SEQLENS) is written there, and then no output is written.
 * Returns SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED,
 * SSD_ERR_SCRATCH_TOO_SMALL or SSD_ERR_CUDA (launch failure).
 */
#define SSD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
SSD_API int ssd_forward_noalloc(const ssd_desc_t* desc, const void* x, const void* dt,
                                const float* A, const void* B, const void* C, const float* D,
                                const float* dt_bias, int chunk_size, const float* initial_states,
                                const int32_t* cu_seqlens, int num_docs, void* y,
                                float* final_states, int* status, ssd_stream_t stream);

/* Debug builds: the source line of the first failed device-side check recorded in
 * the handle's status word since the handle was created (0: none).  Synchronises
 * the device.  Release builds record nothing and return 0. */
SSD_API int ssd_debug_line(ssd_handle_t h);

/* 1 for a library built with device-side checks (`build.py --debug`), 0 otherwise. */
SSD_API int ssd_debug_build(void);

/* Static string naming a return code. */
SSD_API const char* ssd_error_string(int code);

/* Library version string. */
SSD_API const char* ssd_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SSD_B200_H */
