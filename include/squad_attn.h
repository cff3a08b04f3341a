/*
 * squad_attn.h -- C ABI of the SQuad-Attention CUDA library (sm_100a, one GPU).
 *
 * SQuad-Attention ("SQuad: Sub-Quadratic Attention Distillation for Efficient Video Generation")
 * replaces full softmax self-attention over a T x H x W latent token grid by a sequence of two plain
 * softmax attentions, the second fed by the first (paper §3.2; agihunt.info digest, the paragraph that
 * defines the operator):
 *
 *   local pass  Attn_L: every token attends to the w = tw*hw*ww tokens of its window. A window spans
 *                       every frame (tw = T) and an hw x ww block of space (agihunt.info digest,
 *                       the paragraph on the window size: 21x2x4 = 168 at n = 18480).
 *   global pass Attn_G: the n/w tokens that occupy the same slot (t, y mod hw, x mod ww) in every
 *                       window attend to one another; the pass-1 output is its value stream (paper
 *                       appendix "Reachability": the two-hop path (c',j') -> (c',j) -> (c,j)).
 *
 * The passes are joined by re-indexing alone, with no arithmetic (paper appendix "Cost of the two
 * passes"); this library never materialises a permuted copy: both views are strided boxes of the
 * caller's [B, h, n, d] tensors.
 *
 * When hw does not divide H or ww does not divide W, the grid is reflect-padded (paper appendix,
 * "Conformance to the theoretical curves is quantitative"): each frame is padded at the bottom and
 * right up to multiples of hw and ww, reflecting about the edge (the edge token is not repeated);
 * both passes run on the padded grid (padded copies of q, k, v live in the forward workspace) and o
 * is cropped back. The backward is that composition's gradient: zero upstream gradient on the padded
 * tokens, and each input token's gradient summed over its padded copies. squad_window_solve picks a
 * window.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout:     every tensor is contiguous [B, h, n, d] (d fastest), n = T*H*W tokens ordered
 *             (t, y, x) row-major: token = (t*H + y)*W + x. LSE buffers are contiguous [B, h, n] fp32.
 * Dtypes:     SQUAD_BF16: q, k, v, o, dout, dq, dk, dv are bfloat16; accumulation and softmax in
 *             fp32 (tcgen05 tensor cores). SQUAD_FP32: all of them are float32, computed with fp32
 *             FMA on the CUDA cores (exact fp32 path).
 * Pointers:   device pointers, 16-byte aligned, caller-owned. The library allocates no device
 *             memory; scratch comes from the caller's workspace (size from the *_workspace_bytes
 *             query). Workspace pointers must be 256-byte aligned.
 * Streams:    every call is asynchronous on `stream` (0 = legacy default stream); buffers must stay
 *             valid until the stream reaches the call.
 * Errors:     argument errors are detected on the host before anything is launched and returned
 *             synchronously (SQUAD_ERR_INVALID_ARG / SQUAD_ERR_UNSUPPORTED); a failed launch returns
 *             SQUAD_ERR_CUDA. Device-side waits are bounded: a wait that gives up records
 *             SQUAD_ERR_TIMEOUT in the workspace status word, which squad_attn_fwd_status() reads.
 *             No C++ exception crosses this interface.
 */
#ifndef SQUAD_ATTN_H
#define SQUAD_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SQUAD_API __attribute__((visibility("default")))
#else
#define SQUAD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA runtime stream (cudaStream_t); declared opaquely so this header needs no CUDA headers. */
typedef struct CUstream_st* squad_stream_t;

typedef enum {
  SQUAD_OK = 0,
  SQUAD_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, n != T*H*W, ...            */
  SQUAD_ERR_UNSUPPORTED = 2,  /* well-formed but outside what the kernels implement           */
  SQUAD_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, tensor map, ...)   */
  SQUAD_ERR_TIMEOUT = 4       /* a bounded device-side wait gave up (read via *_status)        */
} squad_status_t;

typedef enum { SQUAD_BF16 = 0, SQUAD_FP32 = 1 } squad_dtype_t;

/* Pass order. LOCAL_THEN_GLOBAL is the paper's chosen order; GLOBAL_THEN_LOCAL the ablated reverse
 * (paper §4.4 "The need for and the order of the two passes"; appendix "On the ordering").
 * LOCAL_ONLY and GLOBAL_ONLY run one pass alone (o = pass(q, k, v)), the single-pass variants the
 * same section ablates; chaining them reproduces either two-pass order. */
typedef enum {
  SQUAD_LOCAL_THEN_GLOBAL = 0,
  SQUAD_GLOBAL_THEN_LOCAL = 1,
  SQUAD_LOCAL_ONLY = 2,
  SQUAD_GLOBAL_ONLY = 3
} squad_order_t;

typedef struct {
  int B, h, d;      /* batch, heads, head dim (d in {64, 128}; bf16 tensor-core path: d == 128)  */
  int T, H, W;      /* latent grid; n = T*H*W                                                     */
  int tw, hw, ww;   /* window; tw must equal T (the window spans all frames), 1 <= hw <= H, 1 <= ww <= W;
                       hw not dividing H or ww not dividing W is handled by reflect padding        */
  int order;        /* squad_order_t                                                              */
  int dtype;        /* squad_dtype_t                                                              */
  float scale;      /* softmax scale; 0 selects 1/sqrt(d) (paper eq. 5)                           */
} squad_params_t;

/* Bytes of forward workspace: the pass-1 output O1 ([B,h,n,d] in the tensor dtype), both passes'
 * LSE ([B,h,n] fp32 each) and a small control block; for a padded grid these are sized for the
 * padded n, plus the padded q, k, v and output. Keep the workspace unchanged between
 * squad_attn_fwd and squad_attn_bwd: the backward reads O1 and the LSEs from it. Returns 0 for
 * invalid parameters. */
SQUAD_API size_t squad_attn_fwd_workspace_bytes(const squad_params_t* p);

/* SQuad-Attention forward: o = pass2(q, k, pass1(q, k, v)) with the passes in `order` (or one pass,
 * o = pass(q, k, v), for the single-pass orders).
 * q, k, v: inputs [B,h,n,d]; o: output [B,h,n,d]; workspace: >= squad_attn_fwd_workspace_bytes. */
SQUAD_API squad_status_t squad_attn_fwd(const squad_params_t* p, const void* q, const void* k, const void* v,
                              void* o, void* workspace, squad_stream_t stream);

/* Device status recorded by the last forward/backward call on `workspace`: SQUAD_OK or
 * SQUAD_ERR_TIMEOUT. Synchronises `stream` first. */
SQUAD_API squad_status_t squad_attn_fwd_status(const squad_params_t* p, const void* workspace,
                                     squad_stream_t stream);

/* Bytes of backward workspace: fp32 partial dQ and dK, the gradient of the pass-1 output, the per-row
 * softmax-Jacobian terms of each pass, and a control block (for a padded grid: sized for the padded n,
 * plus the zero-padded dout and the gradients on the padded grid); when a pass has sequences of 129 to
 * 208 tokens, also the bf16 P and dS of one sequence per resident CTA (160 slots of at most 208 KB,
 * independent of n). Returns 0 for invalid params. */
SQUAD_API size_t squad_attn_bwd_workspace_bytes(const squad_params_t* p);

/* SQuad-Attention backward (the pages print no formula; it is the chain rule through both passes).
 * Gradients of <dout, o> with respect to q, k, v. Inputs: q, k, v and o as given to / returned by
 * squad_attn_fwd, dout [B,h,n,d], and fwd_workspace as left by that forward call. Outputs dq, dk,
 * dv [B,h,n,d] (overwritten). q and k are used by both passes, so dq and dk sum two terms. */
SQUAD_API squad_status_t squad_attn_bwd(const squad_params_t* p, const void* q, const void* k, const void* v,
                              const void* o, const void* dout, const void* fwd_workspace,
                              void* dq, void* dk, void* dv, void* bwd_workspace,
                              squad_stream_t stream);

/* The kernel each pass of squad_attn_bwd(p, ...) runs on, in execution order of the forward:
 * kernels[0] for the first pass, kernels[1] for the second (0 when the order has one pass). The
 * choice depends only on p (on the padded grid where the window does not divide it):
 *   SQUAD_BWD_TC_WHOLE    tensor cores, whole sequences, one per work item (several per 128-row
 *                         tile when they have at most 64 tokens) (bf16, d = 128, sequences of at
 *                         most 208 tokens, whatever fits its shared-memory plan);
 *   SQUAD_BWD_TC_CHUNKED  tensor cores, sequences cut into chunks of whole lines of at most 128 rows
 *                         (bf16, d = 128, lines of at most 128 tokens): any sequence length;
 *   SQUAD_BWD_CUDA_CORE   the fp32 CUDA-core kernels (fp32 inputs, other d).
 * Enqueues nothing. SQUAD_ERR_INVALID_ARG / SQUAD_ERR_UNSUPPORTED as squad_attn_bwd would return. */
#define SQUAD_BWD_TC_WHOLE 1
#define SQUAD_BWD_TC_CHUNKED 2
#define SQUAD_BWD_CUDA_CORE 3
SQUAD_API squad_status_t squad_attn_bwd_kernels(const squad_params_t* p, int kernels[2]);

/* Full softmax self-attention softmax(q k^T * scale) v over all n tokens per head (paper eq. 5),
 * the operator SQuad replaces. The window fields and `order` of *p are ignored (grid still gives n).
 * lse_or_null: optional [B,h,n] fp32 output of the natural-log log-sum-exp per query. This call has
 * no workspace and so no status word: its device-side waits are bounded too, but a wait that gives
 * up (leaving o incomplete) is not reported. */
SQUAD_API squad_status_t full_attn_fwd(const squad_params_t* p, const void* q, const void* k, const void* v,
                             void* o, float* lse_or_null, squad_stream_t stream);

/* Largest workspace squad_attn_fwd_noalloc can provide: 128 MiB (one Wan-2.2-5B-shaped block,
 * B = 1, h = 24, n = 18480, d = 128 in bf16, needs about 117 MB). */
#define SQUAD_NOALLOC_MAX_WORKSPACE_BYTES (128u * 1024u * 1024u)

/* squad_attn_fwd without a caller-provided workspace, for callers that cannot allocate device memory:
 * code running inside a framework or engine that owns the whole device memory pool (a cudaMalloc
 * there fails or fragments the pool), latency-critical loops where an allocation's synchronisation
 * is not acceptable, and plugins that only receive the input and output tensors. The paper has no
 * counterpart: this is a deployment variant of squad_attn_fwd with the same arguments minus the
 * workspace, and the same results.
 *
 * The scratch is a file-scope device array of SQUAD_NOALLOC_MAX_WORKSPACE_BYTES in this library,
 * which every GPU that loads the library holds until the process exits. It is shared by every call:
 * calls that may overlap on the GPU (different streams, or different host threads, without ordering
 * between them) race on it and must be serialised by the caller. Each call zeroes what must start at
 * zero. Every call looks up the array's device address on the current device (a host-side query
 * with no stream work); make the first call on a device before any stream capture on it. q, k, v
 * and o must be device memory of the current device (SQUAD_ERR_INVALID_ARG otherwise: the scratch
 * used is the current device's). The LSEs and the device status word of this entry point stay inside
 * the scratch and are not exposed: a bounded device-side wait that gives up leaves o incomplete and
 * is not reported to the caller (the workspace entry point reports it through squad_attn_fwd_status).
 * Returns SQUAD_ERR_UNSUPPORTED, before launching anything, when squad_attn_fwd_workspace_bytes(p)
 * exceeds SQUAD_NOALLOC_MAX_WORKSPACE_BYTES. It allocates nothing (no cudaMalloc or cudaFree). */
SQUAD_API squad_status_t squad_attn_fwd_noalloc(const squad_params_t* p, const void* q, const void* k,
                                                const void* v, void* o, squad_stream_t stream);

/* squad_attn_fwd from host memory, end to end: q, k, v are copied from host to the device buffers, the
 * forward runs, and o is copied back to host memory. The B*h (batch, head) pairs are split into
 * `groups` runs of consecutive pairs; every pair is independent in both passes (each pass folds the
 * axis it does not attend over into the batch of heads: agihunt.info digest, the paragraph that
 * defines the operator), so each run is a forward of its own on contiguous slices of the tensors. The
 * run's host-to-device copies go on copy_in, its forward on compute and its device-to-host copy on
 * copy_out, ordered by events: the input copies of one run overlap the forward of the previous run
 * and the output copy of the one before (the three streams may be the same stream, which serialises
 * everything). The call only enqueues work: q_host, k_host, v_host must stay unchanged until copy_in
 * has passed this call, and o_host is complete once copy_out has. Host buffers should be pinned
 * (cudaHostAlloc / cudaHostRegister) for the copies to be asynchronous.
 * q_dev, k_dev, v_dev, o_dev: device buffers of the full [B,h,n,d] size (16-byte aligned);
 * workspace: >= squad_attn_fwd_host_workspace_bytes(p, groups) (256-byte aligned), reused by the runs
 * one after another on `compute`. Work already queued on `compute` or `copy_out` when the call is made
 * is finished before this call's copies overwrite the device buffers. 1 <= groups <= min(64, B*h).
 * The library creates 130 CUDA events per device on the first call there and keeps them until the
 * process exits; calls on one device enqueue one at a time. Argument errors return
 * SQUAD_ERR_INVALID_ARG before anything is enqueued; a failed copy or launch returns SQUAD_ERR_CUDA (or
 * the forward's own status) with the runs before it enqueued. */
SQUAD_API size_t squad_attn_fwd_host_workspace_bytes(const squad_params_t* p, int groups);
SQUAD_API squad_status_t squad_attn_fwd_host(const squad_params_t* p, const void* q_host, const void* k_host,
                                             const void* v_host, void* o_host, void* q_dev, void* k_dev,
                                             void* v_dev, void* o_dev, void* workspace, int groups,
                                             squad_stream_t copy_in, squad_stream_t compute,
                                             squad_stream_t copy_out);

/* FLOPs of one call, from the paper's cost model (appendix "Conformance to the theoretical curves
 * is quantitative"): 4 B h d (n w + n^2/w) for SQuad (one of the two terms for a single-pass order;
 * n = the padded token count when the window does not divide the grid, the cost of the window
 * actually used), 4 B h d n^2 for full attention. */
SQUAD_API double squad_attn_flops(const squad_params_t* p);
SQUAD_API double full_attn_flops(const squad_params_t* p);

/* The window for a T x H x W grid, chosen anew at each resolution as the paper's appendix describes
 * ("What is measured" for the rule; "Conformance to the theoretical curves is quantitative" for the
 * cost of the window actually used): tw = T; for each hw the ww whose ratio hw:ww is
 * closest to H:W (in log ratio, the smaller ww on a tie); and, among those, the hw whose cost
 * n'm + n'^2/m is least, m = T*hw*ww the window size and n' the reflect-padded token count (ties: the
 * smaller hw). Recovers 21x2x4 at 21x22x40 and at 21x30x52. Writes *tw, *hw, *ww; SQUAD_ERR_INVALID_ARG
 * for non-positive extents or null outputs. Host-only; launches nothing. */
SQUAD_API squad_status_t squad_window_solve(int T, int H, int W, int* tw, int* hw, int* ww);

/* Self-test of the bounded device-side waits (no counterpart in the paper): launches one small kernel
 * that waits, with the library's bounded wait, on a barrier that nothing completes. After timeout_ns
 * (1 ns .. 1 s) the wait gives up, writes SQUAD_ERR_TIMEOUT into *status (a device word the caller
 * zeroed) and the kernel returns, leaving the context usable. status: 4-byte aligned device pointer. */
SQUAD_API squad_status_t squad_wait_selftest(uint32_t* status, unsigned long long timeout_ns, squad_stream_t stream);

/* ------------------------------------------------------------------------------------------------
 * k composed passes over nested windows
 *
 * The paper names composing more than two passes as an open direction (§5 "Limitations and future
 * work") and defines no partition for them. This library's reading, the plainest generalisation of
 * the two passes: each spatial axis is factored into k levels, H = h_1 h_2 ... h_k and
 * W = w_1 w_2 ... w_k, so that a token's row and column are mixed-radix numbers with level 1 least
 * significant, y = a_1 + h_1 (a_2 + h_2 (a_3 + ...)) and x = b_1 + w_1 (b_2 + ...). Pass p attends
 * among the tokens that agree on every digit except (a_p, b_p); pass 1 also spans all frames (as the
 * two-pass window does), the others keep the frame. Every pass takes the same q and k; its values are
 * the previous pass's output. k = 2 is SQuad with window (T, h_1, w_1); k = 1 is full attention.
 * Cost: 4 B h d n (m_1 + ... + m_k) with m_1 = T h_1 w_1 and m_p = h_p w_p.
 *
 * Each pass is one single-pass problem of this library on a reinterpretation of the same contiguous
 * [B, h, n, d] buffers (no copy): pass 1 is SQUAD_LOCAL_ONLY with window (T, h_1, w_1); pass p >= 2 is
 * SQUAD_GLOBAL_ONLY on B' = B h T H/(h_1...h_p) sequences-of-heads of the grid
 * (1, (h_1...h_p) W/(w_1...w_p), w_1...w_p) with window (1, (h_1...h_{p-1}) W/(w_1...w_p), w_1...w_{p-1}).
 * squad_kpass_pass_params reports that problem. Layout, dtypes, pointers, streams and errors follow
 * the conventions above; the levels must factor the grid exactly (no padding).
 * ------------------------------------------------------------------------------------------------ */
#define SQUAD_KPASS_MAX_LEVELS 4

typedef enum {
  SQUAD_KPASS_FORWARD = 0,   /* level 1 first (the analogue of local -> global) */
  SQUAD_KPASS_REVERSE = 1    /* level k first                                   */
} squad_kpass_order_t;

typedef struct {
  int B, h, d;                              /* as in squad_params_t                                   */
  int T, H, W;                              /* latent grid; n = T*H*W                                 */
  int k;                                    /* passes, 1 .. SQUAD_KPASS_MAX_LEVELS                     */
  int level_h[SQUAD_KPASS_MAX_LEVELS];      /* h_1 .. h_k (first k used), product H                    */
  int level_w[SQUAD_KPASS_MAX_LEVELS];      /* w_1 .. w_k, product W; every pass attends over at least
                                               two tokens (T h_1 w_1 >= 2 and h_p w_p >= 2)             */
  int order;                                /* squad_kpass_order_t                                     */
  int dtype;                                /* squad_dtype_t                                           */
  float scale;                              /* softmax scale of every pass; 0 selects 1/sqrt(d)        */
} squad_kpass_params_t;

/* The single-pass problem that level `level` (0-based: 0 is the innermost window) runs, written to
 * *out (its order is SQUAD_LOCAL_ONLY or SQUAD_GLOBAL_ONLY). Host-only; launches nothing.
 * SQUAD_ERR_INVALID_ARG for invalid parameters or level; SQUAD_ERR_UNSUPPORTED where a pass is not
 * supported (as for squad_attn_fwd, or a level past the first of one token). */
SQUAD_API squad_status_t squad_kpass_pass_params(const squad_kpass_params_t* p, int level, squad_params_t* out);

/* Bytes of forward workspace: a control block, the k - 1 intermediate outputs (input dtype) and the
 * k per-pass log-sum-exps (fp32, [B, h, n] each). 0 for invalid parameters. */
SQUAD_API size_t squad_kpass_fwd_workspace_bytes(const squad_kpass_params_t* p);

/* Forward: o = pass_k(q, k, ... pass_1(q, k, v)) in the given order. q, k, v, o: [B, h, n, d];
 * workspace: >= squad_kpass_fwd_workspace_bytes, kept for the backward. */
SQUAD_API squad_status_t squad_kpass_fwd(const squad_kpass_params_t* p, const void* q, const void* k,
                                         const void* v, void* o, void* workspace, squad_stream_t stream);

/* Bytes of backward workspace: a control block, fp32 dQ and dK shares, per-row softmax-Jacobian terms
 * and up to two intermediate value gradients (input dtype), plus, when a level has sequences of 129 to
 * 208 tokens, the bf16 P and dS of one sequence per resident CTA (as for squad_attn_bwd). 0 for
 * invalid parameters. */
SQUAD_API size_t squad_kpass_bwd_workspace_bytes(const squad_kpass_params_t* p);

/* Backward (the chain rule through the k passes, last executed first): gradients of <dout, o> with
 * respect to q, k, v; dq and dk sum the k passes' shares (in fp32, rounded once). Inputs as given to /
 * left by squad_kpass_fwd; dq, dk, dv [B, h, n, d] are overwritten. */
SQUAD_API squad_status_t squad_kpass_bwd(const squad_kpass_params_t* p, const void* q, const void* k,
                                         const void* v, const void* o, const void* dout,
                                         const void* fwd_workspace, void* dq, void* dk, void* dv,
                                         void* bwd_workspace, squad_stream_t stream);

/* Device status recorded by the last squad_kpass_fwd or squad_kpass_bwd on `workspace`: SQUAD_OK or
 * SQUAD_ERR_TIMEOUT. Synchronises `stream` first. */
SQUAD_API squad_status_t squad_kpass_status(const squad_kpass_params_t* p, const void* workspace,
                                            squad_stream_t stream);

/* FLOPs of one k-pass forward: 4 B h d n (m_1 + ... + m_k); 0 for invalid parameters. */
SQUAD_API double squad_kpass_flops(const squad_kpass_params_t* p);

/* ------------------------------------------------------------------------------------------------
 * Sequence split over R ranks: the reorderings around its all-to-all exchanges
 *
 * Each pass folds the axis it does not attend over into the batch of heads (agihunt.info digest, the
 * paragraph that defines the operator), so the tokens of a block can be split over R ranks with one
 * exchange between the passes: a rank holds a band of latent rows of every frame for the local pass,
 * and a group of frames with every row for the global pass. A tensor of the split is a stack of
 * blocks of Hb*W*d contiguous elements (Hb = H/R rows of one frame of one head), indexed by
 * (b, head, r, tg) with r < R and tg < Tg = T/R, in one of three layouts:
 *   SQUAD_SP_BAND    [B, h, R, Tg]  a rank's band: its Hb rows of frame t = r*Tg + tg ([B,h,T*Hb*W,d])
 *   SQUAD_SP_FRAMES  [B, h, Tg, R]  a rank's frame group: row band r of its frame tg ([B,h,Tg*H*W,d])
 *   SQUAD_SP_CHUNKS  [R, B, h, Tg]  an all-to-all buffer: chunk r goes to, or came from, rank r
 * squad_seqpar_reorder writes y (layout `to`) from x (layout `from`), moving whole blocks; with add
 * (layout `to`) not NULL, each element of y is the moved value plus add's element, summed in fp32 and
 * rounded once to the dtype (the two passes' shares of dq and dk). p gives B, h, d, T, H, W and dtype
 * (window fields and order are ignored); T and H must be multiples of R. x, add, y: device buffers
 * of one rank's share, B*h*T*(H/R)*W*d elements, 16-byte aligned, caller-owned; y must not overlap
 * x or add. Asynchronous on `stream`; argument errors return SQUAD_ERR_INVALID_ARG before anything is
 * launched, a failed launch SQUAD_ERR_CUDA. */
#define SQUAD_SP_BAND 0
#define SQUAD_SP_FRAMES 1
#define SQUAD_SP_CHUNKS 2
SQUAD_API squad_status_t squad_seqpar_reorder(const squad_params_t* p, int R, int from, int to, const void* x,
                                              const void* add, void* y, squad_stream_t stream);

/* Static string for a status code (never NULL). */
SQUAD_API const char* squad_status_string(squad_status_t s);

/* Library ABI version (incremented on any incompatible change of this header). */
SQUAD_API int squad_attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SQUAD_ATTN_H */
