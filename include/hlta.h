/*
 * hlta.h -- C ABI of the Hybrid Linear Temporal Attention (HLTA) forward pass
 * for NVIDIA B200 (sm_100a).
 *
 * The layer is the temporal mixer of "Kairos: A Regret-Aware Native
 * World-Action Model Stack for Physical AI" (arXiv 2606.16533), section 2.2:
 *
 *   SWA   sliding-window softmax attention, Eq. (7). Causal reading: query i
 *         attends to the w most recent keys, i - w < j <= i.
 *   DSWA  dilated sliding-window attention, Eq. (8): SWA after rearranging the
 *         frames into d residue classes (f mod d); token t = f*P + s sits at
 *         rearranged position r(t) = floor(f/d)*P + s, and query i attends to key j
 *         iff f_i = f_j (mod d) and 0 <= r(i) - r(j) < w.
 *   GDN   the gated delta memory of section 2.2.1 (Eq. (1)-(6), step 4):
 *           S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *           o_t = S_t q_t,
 *         i.e. the retrieval of Eq. (2) reads the decayed state alpha_t S_{t-1}.
 *
 *   out[b,t,h,:] = g[h,0]*SWA + g[h,1]*DSWA + g[h,2]*GDN   (per-head gates;
 *   the paper leaves the branch combination open, this weighted sum is fixed
 *   here).  The softmax scale is 1/sqrt(d_k).
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, with no padding:
 *       q, k      [B, L, H, d_k]  element type = cfg.dtype
 *       v, out    [B, L, H, d_v]  element type = cfg.dtype
 *       alpha     [B, L, H] float32, each in (0, 1]
 *       beta      [B, L, H] float32, each in [0, 1]
 *       gates     [H, 3]    float32 (SWA, DSWA, GDN weight of head h)
 *       S         [B, H, d_v, d_k] float32 (S maps keys to values: v ~ S k)
 *   - Pointers are DEVICE pointers on the handle's device unless stated;
 *     every pointer must be 16-byte aligned.  The caller owns them; the library
 *     never frees or retains them past the call.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on it: they return once the work is enqueued.
 *   - Host-side argument checks run before anything is enqueued.  On error
 *     nothing is enqueued and hlta_last_error() describes the failure.
 *   - No exception crosses this boundary.  The library is not thread-safe per
 *     handle (one thread per handle at a time); distinct handles are
 *     independent.
 *   - The calls of one handle share its device workspace: enqueue them on one
 *     stream, or order the streams (events) so that they do not overlap.
 */
#ifndef HLTA_H
#define HLTA_H

#if defined(__GNUC__)
#define HLTA_API __attribute__((visibility("default")))
#else
#define HLTA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HLTA_OK = 0,
    HLTA_ERR_INVALID_ARG = 1,    /* a null/misaligned pointer, a size out of range */
    HLTA_ERR_UNSUPPORTED = 2,    /* a valid request this build does not run */
    HLTA_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed */
    HLTA_ERR_OOM = 4,            /* device allocation failed (hlta_create only) */
    HLTA_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up a bounded wait (see hlta_device_status) */
    HLTA_ERR_INJECTED = 6        /* failure injected by HLTA_INJECT_FAIL (tests) */
} hlta_status;

typedef enum { HLTA_BF16 = 0, HLTA_FP32 = 1 } hlta_dtype;

/* Branch selection bits for hlta_forward / hlta_stream_step.  A branch that is
 * not selected is not computed and contributes nothing (as if its gate were 0);
 * the memory state is advanced whenever the GDN bit is set. */
enum {
    HLTA_BRANCH_SWA = 1,
    HLTA_BRANCH_DSWA = 2,
    HLTA_BRANCH_GDN = 4,
    HLTA_BRANCH_ALL = 7
};

/* Form of the memory update (hlta_config.gdn_form).  Both share
 *   S_t = alpha_t S_{t-1} + u_t k_t^T,  o_t = S_t q_t  (section 2.2.1, Eq. (5), step 4)
 * and differ in what the retrieval of Eq. (2) reads:
 *   HLTA_GDN_DECAYED  u_t = beta_t (v_t - alpha_t S_{t-1} k_t): the decayed state, i.e.
 *                     S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 *                     The layer's fixed form and the default.
 *   HLTA_GDN_PAGES    u_t = beta_t (v_t - S_{t-1} k_t): Eq. (2) and Eq. (6) as printed.
 *                     Contractive as well, with factor max(alpha, |alpha - beta|) < 1 along
 *                     a unit k_t. */
enum { HLTA_GDN_DECAYED = 0, HLTA_GDN_PAGES = 1 };

/* Attention window (hlta_config.window_mode), in (rearranged, for DSWA) token
 * positions r, with w the branch's window:
 *   HLTA_WINDOW_CAUSAL   keys r - w < r_k <= r: the w most recent keys (default).
 *   HLTA_WINDOW_CENTRED  keys |r_k - r| <= floor(w/2): the centred window Eq. (7)
 *                        prints, for in-clip (bidirectional) use.  One-shot
 *                        hlta_forward only: not with streaming. */
enum { HLTA_WINDOW_CAUSAL = 0, HLTA_WINDOW_CENTRED = 1 };

/* Layer configuration, fixed for the life of a handle. */
typedef struct {
    int B;                 /* batch, >= 1 */
    int H;                 /* heads, >= 1 */
    int d_k;               /* key/query head dim: 64 or 128 */
    int d_v;               /* value head dim: 64 or 128 */
    int tokens_per_frame;  /* P >= 1: tokens of one latent frame (section 2.2.2) */
    int swa_window;        /* w of SWA in tokens, >= 1 (w = P x window_size on the pages) */
    int dswa_window;       /* w of DSWA in rearranged tokens, >= 1 */
    int dswa_dilation;     /* d of DSWA, >= 1 (d = 1 makes DSWA equal SWA) */
    int chunk;             /* GDN chunk length; must be 64 */
    int dtype;             /* hlta_dtype of q, k, v and out */
    int max_seq_len;       /* largest L accepted by hlta_forward (>= 1) */
    int max_stream_tokens; /* largest n of hlta_stream_step; 0 disables streaming */
    int gdn_form;          /* HLTA_GDN_DECAYED (0) or HLTA_GDN_PAGES (1) */
    int window_mode;       /* HLTA_WINDOW_CAUSAL (0) or HLTA_WINDOW_CENTRED (1) */
    float rope_base;       /* > 0: rotary embedding of q and k for SWA/DSWA (the pages name
                              RoPE for these blocks; reading: channel pair (2m, 2m+1) of the
                              token at position t turns by t * rope_base^(-2m/d_k)); 0: none.
                              Centred windows only.  The memory branch never rotates. */
    int attn_fp8;          /* 1: the SWA/DSWA logits Q K^T run in FP8 (e4m3, one scale per
                              128-row tile of q and of k, the pages' FP8 attention
                              quantization) on the tensor cores; P V stays bf16.  Needs
                              dtype HLTA_BF16 and d_k = d_v = 128; applies where the
                              tensor-core kernel takes the branch (full frames), elsewhere
                              the branch runs unquantized.  hlta_backward does not use it. */
} hlta_config;

typedef struct hlta_handle hlta_handle;

/*
 * hlta_create: validate `cfg` and allocate, on the CURRENT CUDA device, the
 * handle's workspace (sized by max_seq_len), the streaming memory state S
 * (zeroed) and the streaming key/value ring (empty).  *out receives the handle.
 * Errors: INVALID_ARG (null pointer, field out of range), UNSUPPORTED
 * (d_k/d_v/chunk not supported), CUDA (no usable sm_100 device), OOM.
 */
HLTA_API hlta_status hlta_create(const hlta_config *cfg, hlta_handle **out);

/* hlta_destroy: synchronise the device and free everything the handle owns.
 * NULL is accepted (no-op). */
HLTA_API hlta_status hlta_destroy(hlta_handle *h);

/*
 * hlta_forward: the whole layer over a full sequence of L tokens
 * (1 <= L <= max_seq_len), section 2.2.
 *   q, k, v, alpha, beta, gates: inputs, layouts above, token t of batch b at
 *     row b*L + t.
 *   S0:    initial memory state [B,H,d_v,d_k] float32, or NULL for zeros.
 *   S_out: receives the state after token L-1, or NULL.  May alias S0.  Written
 *          only when the GDN branch is selected.
 *   out:   [B,L,H,d_v] of cfg.dtype.
 *   branches: OR of HLTA_BRANCH_* (0 means all).
 * Does not touch the streaming state.  Enqueued on `stream`.
 */
HLTA_API hlta_status hlta_forward(hlta_handle *h, int L, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, const float *gates,
                         const float *S0, float *S_out, void *out, unsigned branches,
                         void *stream);

/*
 * hlta_backward: gradients of hlta_forward (the same L, inputs, S0 and branch
 * selection) for training.  The pages train the layer but print no backward;
 * this is the chain rule through section 2.2.1's recurrence (memory branch,
 * chunk form), section 2.2.2's Eq. (7)/(8) softmax windows and the per-head
 * gated sum.
 *   dout:     [B,L,H,d_v] cfg.dtype, the gradient of the layer output.
 *   dS_final: [B,H,d_v,d_k] float32 gradient of the final memory state, or NULL
 *             (zero).
 *   dq, dk:   [B,L,H,d_k] cfg.dtype, dv: [B,L,H,d_v] cfg.dtype (written).
 *   dalpha, dbeta: [B,L,H] float32 (written; zero without the memory branch).
 *   dgates:   [H,3] float32 (written; zero in unselected columns).
 *   dS0:      [B,H,d_v,d_k] float32 gradient of the initial state, or NULL.
 * The forward is recomputed inside (nothing is kept from hlta_forward).
 * Scratch (about 7 x B*max_seq_len*H*128 floats plus 4 states per 64-token
 * chunk) is allocated at the first call and kept until hlta_destroy
 * (HLTA_ERR_OOM when it cannot be).  The memory branch's backward covers
 * gdn_form = HLTA_GDN_DECAYED (HLTA_ERR_UNSUPPORTED otherwise).  Centred
 * windows and rotary embedding are covered.  Enqueued on `stream`.
 */
HLTA_API hlta_status hlta_backward(hlta_handle *h, int L, const void *q, const void *k, const void *v,
                                   const float *alpha, const float *beta, const float *gates,
                                   const float *S0, const void *dout, const float *dS_final, void *dq,
                                   void *dk, void *dv, float *dalpha, float *dbeta, float *dgates,
                                   float *dS0, unsigned branches, void *stream);

/*
 * hlta_forward_host: hlta_forward on HOST buffers (pinned memory recommended):
 * copies the inputs to device staging owned by the handle (allocated at the
 * first call, kept until hlta_destroy), runs the layer, copies `out` (and
 * S_out when non-NULL) back, and synchronises `stream` before returning.
 * S0 / S_out are host pointers or NULL.
 */
HLTA_API hlta_status hlta_forward_host(hlta_handle *h, int L, const void *q, const void *k, const void *v,
                              const float *alpha, const float *beta, const float *gates,
                              const float *S0, float *S_out, void *out, unsigned branches,
                              void *stream);

/*
 * hlta_stream_step: append n new tokens (1 <= n <= max_stream_tokens) to the
 * handle's stream and compute their outputs: the constant-memory rollout that
 * carries the recurrent state from step to step (section 2.2.2, Long-Horizon
 * Generation).
 * q, k, v: [B,n,H,d]; alpha, beta: [B,n,H]; out: [B,n,H,d_v].  Positions are
 * absolute: the tokens take positions pos .. pos+n-1 where pos counts every
 * token appended since creation or the last reset, so frame membership
 * (t = f*P + s) is stable across steps.  Keys and values needed by later windows
 * are kept in the handle's ring; the memory state S is carried in the handle.
 * Outputs equal hlta_forward over the concatenated sequence.
 * branches: as for hlta_forward; GDN's state advances only when its bit is set,
 * the ring and the position always advance.
 */
HLTA_API hlta_status hlta_stream_step(hlta_handle *h, int n, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const float *gates,
                             void *out, unsigned branches, void *stream);

/* hlta_state_get: copy the streaming memory state S [B,H,d_v,d_k] float32 to
 * the device buffer S_dst (enqueued on `stream`) and write the number of tokens
 * appended so far to *pos_out (host, may be NULL). */
HLTA_API hlta_status hlta_state_get(hlta_handle *h, float *S_dst, long long *pos_out, void *stream);

/* hlta_stream_reset: position 0, S = 0, ring emptied (enqueued on `stream`). */
HLTA_API hlta_status hlta_stream_reset(hlta_handle *h, void *stream);

/* Checkpoint of the whole streaming state (S, ring, position) as an opaque
 * device blob of hlta_stream_checkpoint_bytes(h) bytes.  Restoring it into a
 * handle created with the same config resumes the stream bit-for-bit. */
HLTA_API long long hlta_stream_checkpoint_bytes(const hlta_handle *h);
HLTA_API hlta_status hlta_stream_save(hlta_handle *h, void *dst, void *stream);
HLTA_API hlta_status hlta_stream_load(hlta_handle *h, const void *src, void *stream);

/* hlta_device_status: synchronise the handle's device and report a device-side
 * error recorded since the last call (HLTA_ERR_DEVICE_TIMEOUT when a kernel
 * gave up a bounded wait; the flag is then cleared), or HLTA_OK. */
HLTA_API hlta_status hlta_device_status(hlta_handle *h);

/* Per-branch device timing.  While enabled, every branch of every pass is
 * bracketed by CUDA events recorded on the caller's stream (the stream its
 * kernels run on), so the times are those of the real launches inside the
 * caller's timed region.  Enabling clears earlier records. */
typedef struct {
    int count;                 /* number of valid slots (3: swa, dswa, gdn) */
    char name[4][16];          /* branch names */
    double total_ms[4];        /* summed device time of the branch's kernels */
    long long passes[4];       /* passes in which the branch ran */
    long long kernel_launches; /* kernels launched by all recorded passes */
} hlta_profile_data;

HLTA_API hlta_status hlta_profile_enable(hlta_handle *h, int enable);
/* Synchronise the handle's device and report the records since enabling. */
HLTA_API hlta_status hlta_profile_read(hlta_handle *h, hlta_profile_data *out);

/*
 * hlta_gdn_forward_noalloc: the memory branch alone (the chunked gated delta
 * memory of hlta_forward with branches = HLTA_BRANCH_GDN) for callers that must
 * not allocate device memory once running -- a control loop with a fixed memory
 * budget reserved at start-up, or code under an allocator that forbids
 * cudaMalloc -- and therefore cannot create a handle.  It has no counterpart on
 * the pages; it exists only so that such callers can run the layer's memory.
 *   Sizes come as arguments; head dims are fixed at d_k = d_v = 128, dtype bf16,
 *   chunk 64.  q, k, v: [B,L,H,128] bf16; alpha, beta: [B,L,H] f32; gates: [H,3]
 *   f32 (only g[h,2] is used); S0, S_out: [B,H,128,128] f32 or NULL; out:
 *   [B,L,H,128] bf16 receives g[h,2] * o_t.  Device pointers, 16-byte aligned,
 *   owned by the caller.  Requires L >= 64 and B*H*ceil(L/64) <= 1110.
 * It allocates nothing: its scratch is a 96 MiB array in the library image,
 * which every GPU that loads the library holds until the process exits.  The
 * first call on a device looks up that array's device address and sets kernel
 * attributes; make that first call before any stream capture.  All calls share
 * the array: calls that overlap on the GPU race and must be ordered by the
 * caller.  Enqueued on `stream`; INVALID_ARG / UNSUPPORTED (too large) / CUDA.
 */
HLTA_API hlta_status hlta_gdn_forward_noalloc(int B, int L, int H, const void *q, const void *k, const void *v,
                                              const float *alpha, const float *beta, const float *gates,
                                              const float *S0, float *S_out, void *out, void *stream);

/* Thread-local message describing the last failed call ("" if none). */
HLTA_API const char *hlta_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
HLTA_API int hlta_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HLTA_H */
