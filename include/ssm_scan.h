/*
 * ssm_scan.h -- C ABI of the B200 selective state space (S6) scan library.
 *
 * The library computes the forward pass of the selective scan of Mamba
 * ("Mamba: linear-time sequence modelling with selective state spaces",
 * summary page on azimuth.plus) and its one-token recurrent form:
 *
 *   Delta_t = softplus(dt_t + dt_bias)        selectivity paragraph: Delta_t = softplus(Linear(x_t))
 *   Abar_t  = exp(Delta_t * A)                zero-order hold (SSM glossary, yapayzekasozluk.tr,
 *   Bbar_t  = Delta_t * B_t                     "Temel Matematiksel Cerceve": ZOH discretisation)
 *   h_t     = Abar_t (.) h_{t-1} + Bbar_t x_t  hardware-aware algorithm paragraph (the recurrence)
 *   y_t     = (C_t . h_t + D x_t) * silu(z_t)  glossary output equation y = C h + D x; block
 *                                              paragraph: gate branch SiLU, multiplied in
 *
 * A is diagonal per channel ([D, N]); B_t and C_t are per token and shared by all
 * channels of a sequence ([B, L, N]); Delta is per token and channel. The state
 * h is float32 and never leaves the chip during a scan: only y (and optionally
 * the final state) is written.
 *
 * Conventions for every call:
 *  - All pointers are device pointers into memory the caller owns (the library
 *    allocates nothing). All arrays are contiguous and row-major. Alignment: the
 *    scan's x, dt, z, y and workspace start on 16 bytes (they are moved by TMA);
 *    ssm_step's h starts on 16 bytes when dstate == 16; every other pointer on
 *    its element size.
 *  - dim is a multiple of 8 for bfloat16 tokens and of 4 for float32 tokens;
 *    1 <= dstate <= 16. Other shapes or alignments return SSM_ERR_UNSUPPORTED
 *    before any launch.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream) and runs asynchronously. A returned SSM_OK means the
 *    launch was accepted; device-side problems are reported by
 *    ssm_workspace_status().
 *  - Nothing aborts, throws or traps. Invalid arguments return SSM_ERR_INVALID,
 *    with nothing launched. A failed launch returns SSM_ERR_CUDA.
 *  - Outputs must not alias inputs, except ssm_step's in-place state h.
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID = 1,     /* null required pointer, negative size, bad dtype/flags, short workspace */
    SSM_ERR_UNSUPPORTED = 2, /* valid but not handled: dstate > 16, misaligned pointer or dim */
    SSM_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    SSM_ERR_TIMEOUT = 4      /* a bounded device-side wait for a carry gave up (see ssm_workspace_status) */
} ssm_status;

typedef enum {
    SSM_F32 = 0,  /* x, dt, z, B, C and y are float32 */
    SSM_BF16 = 1  /* x, dt, z, B, C and y are bfloat16; A, D, dt_bias, states stay float32 */
} ssm_dtype;

enum {
    SSM_DELTA_SOFTPLUS = 1u, /* Delta = softplus(dt + dt_bias); without it Delta = dt + dt_bias */
    SSM_A_GENERAL = 2u,      /* evaluate every exp(Delta A[d,n]) on its own, even where a row of A
                                is an arithmetic progression in n (see ssm_scan_fwd) */
    SSM_EXACT_ZOH = 4u,      /* exact zero-order hold for the input: Bbar = (exp(Delta A) - 1) / A * B
                                (Delta B where A[d,n] = 0) instead of Delta B; the form under which
                                the Mamba summary's Theorem 1 (a gated RNN for N = 1) is exact. The
                                kernels evaluate (exp(z) - 1) / z, z = Delta A, by a series for
                                |z| < 1/16, where the subtraction would lose relative precision */
    SSM_SEQ_PARALLEL = 8u,   /* evaluate the sequence in parallel segments: a local pass runs every
                                segment from a zero state, a combine pass chains the segments'
                                carries, a main pass runs every segment from its true start; about
                                twice the work, used automatically when the channel groups (B x
                                D / 32) fill at most a quarter of the GPU's block slots and L >=
                                2048, and asked for by this flag; taken when the workspace is the
                                one ssm_scan_workspace_size() gives, the sequence spans at least
                                two segments of 16 tiles (or, under SSM_TEST_SHORT_SEGMENTS, of
                                one) and groups x segments <= 1024; otherwise the hand-off */
    SSM_SEQ_HANDOFF = 16u,   /* never the sequence-parallel evaluation (with SSM_SEQ_PARALLEL:
                                SSM_ERR_INVALID) */
    SSM_TEST_SHORT_SEGMENTS = 0x40000000u, /* test hook: time segments of one 32-step tile each,
                                so that every tile boundary is a carry between segments (the
                                result is the same; it runs slower) */
    SSM_TEST_DROP_HANDOFF = 0x80000000u /* fault-injection hook for tests: the first time segment of
                                channel group 0 does not publish its state, so its successor's
                                bounded wait runs out; ssm_workspace_status() then reports
                                SSM_ERR_TIMEOUT and that call's outputs are not valid */
};

/* Arguments of one full-sequence scan. Shapes: B = batch, L = seqlen, D = dim, N = dstate. */
typedef struct {
    int64_t batch, seqlen, dim, dstate;
    ssm_dtype dtype;
    uint32_t flags;          /* SSM_DELTA_SOFTPLUS | SSM_A_GENERAL */
    const void *x;           /* [B, L, D] input tokens                               */
    const void *dt;          /* [B, L, D] raw step size (before bias and softplus)   */
    const void *z;           /* [B, L, D] gate input, or NULL for no gate            */
    const void *Bm;          /* [B, L, N] input projection B_t                       */
    const void *Cm;          /* [B, L, N] output projection C_t                      */
    const float *A;          /* [D, N] diagonal state matrix (float32)               */
    const float *Dskip;      /* [D] skip weight D, or NULL for 0                      */
    const float *dt_bias;    /* [D] step-size bias, or NULL for 0                     */
    const float *h0;         /* [B, D, N] initial state, or NULL for zero            */
    void *y;                 /* [B, L, D] output, same dtype as x                    */
    float *h_last;           /* [B, D, N] final state out (float32), or NULL         */
    void *workspace;         /* device scratch of ssm_scan_workspace_size() bytes    */
    size_t workspace_bytes;
    /* The block's short causal convolution in front of the scan (optional, see ssm_scan_fwd) */
    const float *conv_w;     /* [D, 4] depthwise taps, oldest token first, float32 on 16 bytes; NULL: none */
    const float *conv_b;     /* [D] convolution bias, or NULL for 0 (needs conv_w)    */
    const void *conv_x0;     /* [B, 3, D] the three tokens before t = 0, oldest first, dtype of x;
                                NULL for zeros (needs conv_w)                         */
} ssm_scan_args;

/*
 * Bytes of device workspace ssm_scan_fwd needs for these shapes (0 for invalid
 * arguments, for B = 0 or D = 0, which need none, and for more than 2^40 channel slots
 * B x round_up(D, 32), which ssm_scan_fwd refuses with SSM_ERR_UNSUPPORTED). The workspace
 * holds a status word, the hand-over of the running state between consecutive time
 * segments of a channel group (B x round_up(D, 32) x 64 bytes and a little more: about
 * 330 KB for B=1, D=5120), and after it a fixed 4.5 MiB area for the sequence-parallel
 * evaluation (SSM_SEQ_PARALLEL: the segments' local end states, start states and sums). A
 * workspace with the hand-over part only (4.5 MiB less) is accepted and never takes the
 * sequence-parallel evaluation. The library clears what it needs at the start of each
 * call, on the call's stream; one workspace must not be shared by calls that can overlap
 * on the GPU.
 */
size_t ssm_scan_workspace_size(const ssm_scan_args *args);

/*
 * Full-sequence selective scan: writes y for every (b, t, d) and, if h_last is
 * not NULL, the state after the last token. L == 0 writes h_last = h0 (or 0).
 * B or D == 0 does nothing.
 *
 * Sequence parallelism: the sequence of every group of channels is cut into
 * time segments; a segment starts from the state its predecessor hands over
 * (a bounded wait on a flag in the workspace), so no exponential is evaluated
 * twice. With few groups (B x D / 32 at most half the SMs) and a long sequence, or
 * with SSM_SEQ_PARALLEL, the segments run concurrently instead: a local pass from zero
 * states, a combine of the segments' affine maps h -> a h + l, and a main pass from
 * the combined start states, all on the call's stream. The chunked form is exact: the
 * recurrence is associative (Mamba summary, hardware-aware algorithm paragraph:
 * parallel scan).
 *
 * Where every row of A used by a thread block is an exact arithmetic progression
 * in n (A[d,n] = A[d,0] + n * (A[d,1] - A[d,0]) in float32; the S4D-real
 * initialisation A[d,n] = -(n+1) is one), a thread's four factors exp(Delta A[d,n])
 * for n = 4w .. 4w+3 follow from two exponentials, exp(Delta A[d,4w]) and the
 * ratio r = exp(Delta (A[d,1] - A[d,0])), by multiplication. SSM_A_GENERAL turns
 * this off (one exponential per state and step).
 *
 * Short convolution (conv_w not NULL): the Mamba block's main branch runs a causal
 * 1-D convolution of kernel size 4 and SiLU before the selective SSM (Mamba summary,
 * block-architecture paragraph). The scan then reads, per channel d,
 *   u_t = silu(conv_b[d] + sum_{k=0..3} conv_w[d,k] x_{t-3+k})
 * (x_{t} for t < 0 from conv_x0, or 0) and uses u_t wherever x_t appears above (Bbar_t
 * u_t and D u_t). The convolution runs inside the scan kernel on the tiles it loads
 * anyway, in float32: x crosses HBM once and u is never stored. The y, h_last and
 * chunking rules are unchanged; to continue a sequence in a later call, pass its last
 * three tokens as conv_x0 and its h_last as h0. Errors: SSM_ERR_INVALID for conv_b or
 * conv_x0 without conv_w; SSM_ERR_UNSUPPORTED for conv_w not on 16 bytes.
 */
ssm_status ssm_scan_fwd(const ssm_scan_args *args, void *stream);

/*
 * One recurrent decode step for every sequence b and channel d (the scan with
 * L = 1, state carried in place; SSM blog on shakilmahmud.com, section 3: the
 * recurrent form at inference, constant memory per token):
 *   x, dt, z : [B, D] (z may be NULL);  Bm, Cm : [B, N];  A : [D, N];
 *   Dskip, dt_bias : [D] or NULL;  h : [B, D, N] float32, read and overwritten;
 *   y : [B, D] output. No workspace. flags as for the scan.
 * With dstate == 16, A on 16 bytes and Bm, Cm on four elements, two threads
 * share a channel (two float4 of h each); otherwise one thread per channel.
 */
ssm_status ssm_step(int64_t batch, int64_t dim, int64_t dstate, ssm_dtype dtype, uint32_t flags,
                    const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                    const float *A, const float *Dskip, const float *dt_bias, float *h, void *y,
                    void *stream);

/*
 * ssm_step behind the Mamba block's short causal convolution (kernel size 4) and SiLU
 * (Mamba summary, block-architecture paragraph), the decode form of the scan's conv_w:
 * the SSM's input is u = silu(conv_b[d] + conv_w[d,0] s0 + conv_w[d,1] s1 +
 * conv_w[d,2] s2 + conv_w[d,3] x), where s0, s1, s2 are the three previous tokens of
 * the window conv_state ([B, 3, D], dtype of x, oldest first: the layout of the scan's
 * conv_x0, so the last three tokens of a prefill start the decode). conv_state is then
 * moved on by one token in place, to (s1, s2, x). conv_w [D, 4] float32 on 16 bytes;
 * conv_b [D] or NULL; conv_state must not alias any other argument. Errors as
 * ssm_step; SSM_ERR_INVALID if conv_w or conv_state is NULL.
 */
ssm_status ssm_step_conv(int64_t batch, int64_t dim, int64_t dstate, ssm_dtype dtype, uint32_t flags,
                         const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                         const float *A, const float *Dskip, const float *dt_bias, const float *conv_w,
                         const float *conv_b, void *conv_state, float *h, void *y, void *stream);

/*
 * Synchronises `stream` and returns the device-side status of the last scan
 * that used `workspace`: SSM_OK, or SSM_ERR_TIMEOUT if a segment gave up
 * waiting for its predecessor's state (its outputs are then incomplete).
 */
ssm_status ssm_workspace_status(const void *workspace, void *stream);

/*
 * The scan for callers that must not allocate device memory: a host runtime
 * whose memory pool owns all of the GPU's memory (a cudaMalloc there fails or
 * fragments the pool), or a real-time loop that cannot accept the device-wide
 * synchronisation cudaMalloc/cudaFree may imply. It computes exactly what
 * ssm_scan_fwd computes and takes the same arguments, but ignores
 * args->workspace: its scratch is a fixed 2 MiB array in the library's device
 * memory, which every GPU that loads the library keeps until the process
 * exits. It holds the hand-over part of the workspace only, so the evaluation is
 * always the hand-off (never sequence-parallel); shapes whose hand-over part exceeds
 * 2 MiB (a little over 32,000 channels B x D) return SSM_ERR_UNSUPPORTED, with
 * nothing launched. The
 * caller still provides all inputs
 * and outputs. Nothing is allocated: no cudaMalloc, cudaFree or allocating
 * library routine is called.
 *  - The first call on each device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *  - All calls share the one array and the library clears what must start at
 *    zero at each call, so calls that can overlap on the GPU (other streams,
 *    other host threads) race and must be serialised by the caller.
 *  - Its device-side status word also lives in that array: ssm_noalloc_status()
 *    reads it back.
 * Errors: those of ssm_scan_fwd (shapes, pointers and alignment are checked before
 * the size bound), SSM_ERR_UNSUPPORTED for shapes beyond the array.
 * The pages have no counterpart: this entry point exists only for such callers.
 */
ssm_status ssm_scan_fwd_noalloc(const ssm_scan_args *args, void *stream);

/*
 * Synchronises `stream` and returns the device-side status of the last
 * ssm_scan_fwd_noalloc on the current device: SSM_OK, or SSM_ERR_TIMEOUT if a bounded
 * wait for a carried state gave up (the y of that call is then not valid), as
 * ssm_workspace_status does for a caller's workspace. It copies four bytes to a host
 * variable and allocates nothing; SSM_ERR_CUDA if the copy or the synchronisation
 * fails. Like the entry point above, it has no counterpart on the pages.
 */
ssm_status ssm_noalloc_status(void *stream);

/*
 * The scan with its token tensors in HOST memory, for callers whose inputs arrive from
 * and whose outputs go back to the host. args->x, dt, z, Bm, Cm and y are host
 * pointers (page-locked memory lets the copies run asynchronously and overlap; with
 * pageable memory the copies still work but serialise); A, Dskip, dt_bias, h0, h_last
 * and workspace are device pointers, as for ssm_scan_fwd. The sequence is processed in
 * chunks of chunk_len steps through `staging`, caller-owned device memory of at least
 * ssm_scan_host_staging_size(args, chunk_len) bytes starting on 256 bytes: while chunk
 * c is scanned on `stream`, chunk c+1 is copied in and the y of chunk c-1 copied out
 * on two copy streams of the library, so both transfer directions overlap each other
 * and the kernels. The state passes from chunk to chunk through h0/h_last in the
 * staging memory, so the result equals ssm_scan_fwd over the whole sequence bit for
 * bit where both take the hand-off evaluation (SSM_SEQ_HANDOFF makes sure of it; the
 * sequence-parallel one differs from it by float32 rounding only). Batch rows are strided in host memory ([B, L, ...]); each chunk moves them with
 * one two-dimensional copy per tensor. With the short convolution (conv_w, conv_b and
 * conv_x0 device pointers), every chunk after the first also copies in the three host
 * tokens before it as its prefix; the staging size then includes room for them.
 *
 * Ordering: the call enqueues and returns; all of its work is ordered after the work
 * already on `stream` and before the work enqueued on `stream` later. The host buffers
 * must stay valid, and y unread, until then. The copy streams and their events are
 * created on the first call on each device and kept until the process exits (make the
 * first call before any stream capture); calls from several host threads are
 * serialised while they enqueue.
 * Errors: as ssm_scan_fwd; SSM_ERR_INVALID if chunk_len < 1 or staging is NULL or too
 * small; SSM_ERR_UNSUPPORTED if staging is not 256-byte aligned. When a call fails
 * after it has queued copies, it waits for the library's copy streams before it
 * returns, so the host buffers may be reused at once. There is no
 * counterpart on the pages: this is the host side of the layer's input and output.
 */
size_t ssm_scan_host_staging_size(const ssm_scan_args *args, int64_t chunk_len);
ssm_status ssm_scan_fwd_host(const ssm_scan_args *args, int64_t chunk_len, void *staging, size_t staging_bytes,
                             void *stream);

/*
 * Backward of ssm_scan_fwd: the gradients of a loss with respect to every input, given
 * dy = dL/dy and optionally dh_last = dL/dh_L. The pages print no backward formulas;
 * this is the derivative of the forward above, with the states recomputed rather than
 * stored (Mamba summary, hardware-aware algorithm paragraph: recomputation in the
 * backward pass). The sequence of every group of 32 channels is cut into segments
 * (about 1,800 (group, segment) items in all), each a thread block: a first pass gives
 * each segment's end state from a zero start and its adjoint at the start from a zero
 * end, a short combine pass chains them into every segment's true start state and end
 * adjoint (both recurrences are linear). The first pass also keeps, in the workspace,
 * the zero-start state at every 32 steps and the sum of Delta up to there, from which
 * the main pass rebuilds the true state at those points; it then walks each segment
 * backwards, recomputing each 16 steps' states from them.
 *
 * Shapes and types as for ssm_scan_fwd; x, dt, z, Bm, Cm, A, Dskip, dt_bias, h0 are the
 * forward's inputs. Outputs (all overwritten; device memory the caller owns):
 *   dx, ddt, dz : [B, L, D], dtype of x (dz is required exactly when z is given);
 *                 ddt is dL/d(dt), the raw step size before bias and softplus
 *   dB, dC      : [B, L, N] float32 (B_t and C_t are shared by the channels of a
 *                 sequence: their gradients sum over the channels)
 *   dA          : [D, N] float32;  dD, ddt_bias : [D] float32, or NULL to skip
 *   dh0         : [B, D, N] float32 dL/dh0, or NULL to skip
 * dB, dC, dA, dD and ddt_bias are sums accumulated with float atomics: their last bits
 * can vary from run to run with the order of the additions. SSM_DELTA_SOFTPLUS and
 * SSM_EXACT_ZOH as in the forward call (SSM_A_GENERAL changes nothing here). With the
 * short convolution (conv_w, conv_b, conv_x0 as in the forward) dx is the gradient of
 * the raw tokens before it, and dconv_w, dconv_b, dconv_x0 those of its taps, bias and
 * prefix tokens (dconv_w and dconv_b also accumulate with atomics): a first kernel writes
 * the convolution's output u into the workspace, the passes run on it and write dL/du in
 * float32 there, and a last kernel takes dL/du back through SiLU and the taps. The
 * workspace holds the checkpoints (68 bytes per channel and 32 steps: about one [B, L, D]
 * bfloat16 tensor), 8.3 KB per item and, with the convolution, u and dL/du:
 * ssm_scan_bwd_workspace_size() bytes, 16-byte aligned.
 * Errors: as ssm_scan_fwd (x, dt, z, dy and workspace on 16 bytes).
 */
typedef struct {
    int64_t batch, seqlen, dim, dstate;
    ssm_dtype dtype;
    uint32_t flags;          /* SSM_DELTA_SOFTPLUS as in the forward call */
    const void *x, *dt, *z, *Bm, *Cm;          /* the forward's tokens (z may be NULL) */
    const float *A, *Dskip, *dt_bias, *h0;     /* the forward's parameters (NULL as there) */
    const void *dy;          /* [B, L, D] dL/dy, dtype of x                          */
    const float *dh_last;    /* [B, D, N] dL/dh_L, or NULL for 0                       */
    void *dx, *ddt, *dz;     /* [B, L, D] outputs, dtype of x (dz NULL iff z NULL)    */
    float *dB, *dC;          /* [B, L, N] float32 outputs                            */
    float *dA;               /* [D, N] float32 output                                */
    float *dD, *ddt_bias;    /* [D] float32 outputs, or NULL                          */
    float *dh0;              /* [B, D, N] float32 output, or NULL                     */
    void *workspace;         /* ssm_scan_bwd_workspace_size() bytes                  */
    size_t workspace_bytes;
    /* The short convolution of the forward call (conv_w NULL: none), and its gradients:
       dconv_w [D, 4] and dconv_b [D] float32 (required with conv_w; dconv_b also when
       conv_b is NULL), dconv_x0 [B, 3, D] dtype of x (exactly when conv_x0 is given). */
    const float *conv_w, *conv_b;
    const void *conv_x0;
    float *dconv_w, *dconv_b;
    void *dconv_x0;
} ssm_scan_bwd_args;

size_t ssm_scan_bwd_workspace_size(const ssm_scan_bwd_args *args);
ssm_status ssm_scan_bwd(const ssm_scan_bwd_args *args, void *stream);

/*
 * The state space model in its chunked matrix form (structured state space duality;
 * Mamba-2 article, mugbit.ir, "Mamba-2 / SSD" section: the recurrence is a product with a
 * lower-triangular semiseparable matrix, computed by matrix multiplications on tensor
 * cores). It is the same model as ssm_scan_fwd restricted the Mamba-2 way: H heads of P
 * channels each; the P channels of a head share one step size dt[b, t, h] and one scalar
 * A[h] (A[d, n] = A[h] for all n), and D[h], dt_bias[h] per head; B_t, C_t [N] shared by
 * all heads, as in ssm_scan_fwd. Per head h and channel p (d = h P + p):
 *   Delta_t = softplus(dt[b, t, h] + dt_bias[h])  (or dt + dt_bias without the flag)
 *   state[p, n] <- exp(Delta_t A[h]) state[p, n] + Delta_t B_t[n] x_t[d]
 *   y_t[d] = (sum_n C_t[n] state[p, n] + D[h] x_t[d]) * silu(z_t[d])   (no gate if z NULL)
 * Evaluated per chunk of 128 steps as four tcgen05 matrix products with float32
 * accumulation: C B^T, the decay-masked matrix times x, C times the chunk's starting
 * state, and the decay-weighted B^T times x for the next state; the skip D x is added in
 * float32. The operands of the products are bfloat16 (the decay matrix rounded to it; the
 * state entering C S as two bfloat16 parts, high and low, to keep its float32
 * precision); the state is carried between chunks in float32.
 * Shapes: x, z, y [B, L, H, P]; dt [B, L, H]; Bm, Cm [B, L, N]; A, Dskip, dt_bias [H];
 * h0, h_last [B, H, P, N] float32 (state[p, n] of head h), NULL for 0 / not wanted.
 * Supported: dtype SSM_BF16, headdim P = 64, dstate N = 128 (the Mamba-2 head shape);
 * anything else returns SSM_ERR_UNSUPPORTED (ssm_scan_fwd computes the same model for
 * other shapes and float32, one exponential per state). Alignment: x, z, y, Bm, Cm, h0,
 * h_last and the workspace on 16 bytes, A, Dskip, dt_bias on 4. flags: SSM_DELTA_SOFTPLUS
 * and the test hook SSM_TEST_DROP_HANDOFF (the first time segment of sequence 0, head 0
 * does not publish its state: its successor's bounded wait runs out, the status word then
 * reads SSM_ERR_TIMEOUT and that call's outputs are not valid). The workspace (ssm_ssd_workspace_size bytes, caller-owned device memory, one
 * per concurrently running call) holds a counter, a status word (ssm_workspace_status
 * reads it: SSM_ERR_TIMEOUT if a bounded device wait gave up), a flag per (sequence,
 * head) and the float32 state handed between the time segments of each (B x H x 32 KB).
 * L == 0 writes h_last = h0 (or 0). The call enqueues work on `stream` and returns.
 */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate;  /* B, L, H, P, N */
    ssm_dtype dtype;
    uint32_t flags;          /* SSM_DELTA_SOFTPLUS                                     */
    const void *x;           /* [B, L, H, P] input tokens                             */
    const void *dt;          /* [B, L, H] raw step sizes                              */
    const void *z;           /* [B, L, H, P] gate, or NULL                            */
    const void *Bm, *Cm;     /* [B, L, N]                                             */
    const float *A;          /* [H] one scalar per head                               */
    const float *Dskip;      /* [H] or NULL                                           */
    const float *dt_bias;    /* [H] or NULL                                           */
    const float *h0;         /* [B, H, P, N] or NULL                                  */
    void *y;                 /* [B, L, H, P] output                                   */
    float *h_last;           /* [B, H, P, N] output or NULL                           */
    void *workspace;         /* ssm_ssd_workspace_size() bytes                         */
    size_t workspace_bytes;
} ssm_ssd_args;

size_t ssm_ssd_workspace_size(const ssm_ssd_args *args);  /* 0 for invalid shapes */
ssm_status ssm_ssd_fwd(const ssm_ssd_args *args, void *stream);

/* Human-readable name of a status code (static storage). */
const char *ssm_status_string(ssm_status status);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
