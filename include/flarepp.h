/*
 * flarepp.h -- C ABI of the B200 (sm_100a) FLARE++ token mixer: forward and backward.
 *
 * The operation (FLARE.py README, "FLARE++" code block, flarepp_multihead_mixer;
 * shapes from its docstring):
 *
 *     q_dyn = SDPA(q0, k0, k0)          synthesis: M latent seeds read the N tokens
 *     q     = q_fixed + gate * q_dyn    routing queries (physicsnemo issue #2024,
 *                                       "Fixed reference and gate")
 *     z     = SDPA(q, k, v)             encode:  N tokens -> M latents
 *     y     = SDPA(k, q, z)             decode:  M latents -> N tokens
 *
 * SDPA(Q, K, V)_i = sum_j softmax_j(scale * <Q_i, K_j>) V_j, no mask, no dropout,
 * not causal; scale = 1/sqrt(D) unless an options struct says otherwise.  With
 * the gate closed the mixer is FLARE (FLARE.py README, "FLARE" code block,
 * flare_multihead_mixer): z = SDPA(q_fixed, k, v), y = SDPA(k, q_fixed, z).
 *
 * Layout and ownership (every entry point):
 *   - All tensor pointers are caller-owned DEVICE pointers (except the *_host
 *     entry), row-major and contiguous, 16-byte aligned:
 *       q0, q_fixed   [H, M, D]     shared by every batch element
 *       k0, k, v, y   [B, H, N, D]  (or [B, N, H, D] with
 *                                    flarepp_options_t.layout = FLAREPP_LAYOUT_BNHD:
 *                                    the heads of one token adjacent, as a
 *                                    [B, N, H*D] projection output viewed per head)
 *     in the I/O dtype (FLAREPP_F32 = fp32, FLAREPP_BF16 = bf16, FLAREPP_F16 =
 *     fp16; the last for the fp16 forward that physicsnemo issue #1150, the
 *     author's reply, "3. Scaling to 1 M points", calls essential at 1M points).
 *   - gate: DEVICE float[H], the gate value sigmoid(g) per head (never the
 *     logit; the library applies no sigmoid).  gate == NULL closes the gate:
 *     the synthesis is skipped and the result is FLARE with q = q_fixed
 *     (q0 and k0 may then be NULL).  A gate of zeros still runs the synthesis
 *     and gives the same y.
 *   - y must not overlap any input.
 *   - stream is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Every call is asynchronous on it except the *_host entry and
 *     flarepp_check_device_status, which synchronise the stream.
 *   - Accumulation is fp32 for every dtype.  16-bit I/O (bf16 or fp16) rounds
 *     q, z and the softmax weights to the I/O dtype where they feed the tensor
 *     cores; y is rounded to the I/O dtype once, at the end.  With fp16 the
 *     weights are taken relative to (running row max - 7 log2 units), so they
 *     stay below 2^15 (fp16's largest finite value is 65504); weights below
 *     about 2^-31 of the row's largest round to zero.
 *
 * Errors: every entry returns a flarepp_status_t and never throws or aborts.
 * Arguments are checked before any CUDA call or launch; a failed check
 * launches nothing.  Launch failures are reported as FLAREPP_ERR_CUDA.  A
 * kernel whose bounded wait runs out records FLAREPP_ERR_TIMEOUT in a device
 * status word, returns early (its output is then undefined) and leaves the
 * context usable; flarepp_check_device_status() reads and clears that word.
 *
 * Limits: 1 <= B*H <= 65535, 1 <= N <= 2^31-1, 1 <= M <= 4096,
 * D in {16, 32, 64, 128}; other values give FLAREPP_ERR_UNSUPPORTED.
 */
#ifndef FLAREPP_H_
#define FLAREPP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLAREPP_ABI_VERSION 5

typedef enum flarepp_dtype {
    FLAREPP_F32 = 0,
    FLAREPP_BF16 = 1,
    FLAREPP_F16 = 2
} flarepp_dtype_t;

typedef enum flarepp_status {
    FLAREPP_OK = 0,
    FLAREPP_ERR_INVALID_ARG = 1,   /* NULL pointer, misaligned pointer, overlap, bad size */
    FLAREPP_ERR_UNSUPPORTED = 2,   /* valid but outside the limits above (e.g. D = 48) */
    FLAREPP_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    FLAREPP_ERR_WORKSPACE = 4,     /* caller workspace too small, or allocation failed */
    FLAREPP_ERR_TIMEOUT = 5        /* a kernel's bounded wait ran out (device status word) */
} flarepp_status_t;

/* Kernel family.  AUTO picks the tcgen05 tensor-core kernels for 16-bit I/O
 * (bf16 or fp16, every supported D) and the SIMT (FFMA) kernels for fp32 I/O
 * (TF32 products would not meet fp32 accuracy). */
typedef enum flarepp_path {
    FLAREPP_PATH_AUTO = 0,
    FLAREPP_PATH_SIMT = 1,
    FLAREPP_PATH_TCGEN05 = 2
} flarepp_path_t;

/* Memory layout of the token tensors k0, k, v and y (q0, q_fixed are always
 * [H, M, D]; q_out and z_out always [B, H, M, D]). */
typedef enum flarepp_layout {
    FLAREPP_LAYOUT_BHND = 0,   /* [B, H, N, D]: one head's tokens contiguous           */
    FLAREPP_LAYOUT_BNHD = 1    /* [B, N, H, D]: one token's heads contiguous; read and
                                  written in place, no transpose pass                 */
} flarepp_layout_t;

/* Optional controls for the _ex entry.  Zero-initialise and set what you need. */
typedef struct flarepp_options {
    float scale;             /* softmax scale; <= 0 selects 1/sqrt(D)                        */
    int path;                /* flarepp_path_t; TCGEN05 on an unsupported shape -> UNSUPPORTED */
    int force_chunks;        /* 0 = planned; > 0 forces the number of token chunks per (b,h)
                                in the synthesis and encode passes (clamped to the tile count) */
    int n_stage_events;      /* length of stage_events (0 = none)                            */
    float* q_out;            /* optional DEVICE fp32 [B,H,M,D]: the routing queries q        */
    float* z_out;            /* optional DEVICE fp32 [B,H,M,D]: the latents z                */
    void* workspace;         /* optional DEVICE scratch, 256-byte aligned; NULL = the library
                                allocates stream-ordered (cudaMallocAsync/cudaFreeAsync)      */
    size_t workspace_bytes;  /* size of `workspace`; must be >= flarepp_workspace_bytes()    */
    void* const* stage_events; /* optional caller-created cudaEvent_t handles (as void*):
                                  [0] is recorded on `stream` before the first kernel launch
                                  and [i] after the i-th launch, for i < n_stage_events; lets a
                                  caller time each kernel on the stream it runs on            */
    int layout;              /* flarepp_layout_t of k0, k, v, y; other values -> INVALID_ARG  */
    int norm_synthesis;      /* 1: head-wise RMS normalisation of the synthesis seeds and
                                keys/values, q0 and k0 rows -> x / sqrt(mean_d x^2 + 1e-6)
                                (no learned scale; physicsnemo issue #2024, FLARE++ list,
                                "Normalizing the synthesis call"): one extra launch writes
                                normalised copies into the workspace (which grows by the
                                sizes of q0 and k0) and the synthesis reads them.  In
                                flarepp_cp_partials it applies to that call, which must then
                                be the synthesis (q_shared = 1, v == k).  Ignored with the
                                gate closed.  0: none.  Other values -> INVALID_ARG          */
} flarepp_options_t;

/* Kernel launches one forward call makes (gated = 0: closed gate / FLARE).
 * Launch order: gated -> split partial (synthesis), merge (q), split partial
 * (encode), merge (z), decode; closed gate -> the last three.  A gated call
 * with norm_synthesis makes one more, first: the normalisation of q0, k0. */
int flarepp_launches_per_call(int gated);

/* FLARE++ mixer forward (see the top of this file).  gate == NULL -> FLARE. */
int flarepp_mixer_fwd(const void* q0, const void* q_fixed, const float* gate,
                      const void* k0, const void* k, const void* v, void* y,
                      int B, int H, int N, int M, int D, int dtype, void* stream);

/* FLARE (closed gate): z = SDPA(q, k, v), y = SDPA(k, q, z), q [H,M,D] shared over B.
 * Same result as flarepp_mixer_fwd(NULL, q, NULL, NULL, k, v, y, ...). */
int flare_fwd(const void* q, const void* k, const void* v, void* y,
              int B, int H, int N, int M, int D, int dtype, void* stream);

/* flarepp_mixer_fwd with options (opts may be NULL = all defaults). */
int flarepp_mixer_fwd_ex(const void* q0, const void* q_fixed, const float* gate,
                         const void* k0, const void* k, const void* v, void* y,
                         int B, int H, int N, int M, int D, int dtype,
                         const flarepp_options_t* opts, void* stream);

/* Bytes of device scratch one call needs (partial softmax triples per token
 * chunk, and q, z in fp32 and in the 16-bit I/O dtype).  gated = 0 for the closed-gate form.
 * opts (may be NULL) is the call's options: force_chunks, layout and
 * norm_synthesis change the size.  Returns 0 for arguments the forward
 * entries would reject. */
size_t flarepp_workspace_bytes(int B, int H, int N, int M, int D, int dtype, int gated,
                               const flarepp_options_t* opts);

/* Registers a caller-owned DEVICE scratch buffer for the current device
 * (256-byte aligned; dev_ptr = NULL unregisters).  The forward entries that
 * get no workspace through their options (flarepp_mixer_fwd, flare_fwd,
 * flarepp_mixer_fwd_debug, flarepp_mixer_fwd_ex with opts->workspace = NULL)
 * use it when it holds at least flarepp_workspace_bytes(...) bytes for the
 * call, and allocate stream-ordered otherwise.  The caller keeps the buffer
 * alive while it is registered; forward calls whose kernels overlap on the GPU
 * (other streams, other host threads) race on a shared registered buffer.
 * The per-call flarepp_options_t.workspace needs no shared state and takes
 * precedence.  Misaligned dev_ptr -> FLAREPP_ERR_INVALID_ARG. */
int flarepp_set_workspace(void* dev_ptr, size_t bytes);

/* flarepp_mixer_fwd that also returns the intermediates for debugging and
 * parity checks: q_out and z_out, optional DEVICE fp32 [B,H,M,D] (either may
 * be NULL; 16-byte aligned), the routing queries q and the latents z; and
 * force_chunks > 0 forces the number of token chunks of the synthesis and
 * encode passes (0 = planned; < 0 -> FLAREPP_ERR_INVALID_ARG).  The same as
 * flarepp_mixer_fwd_ex with those three options set. */
int flarepp_mixer_fwd_debug(const void* q0, const void* q_fixed, const float* gate,
                            const void* k0, const void* k, const void* v, void* y,
                            int B, int H, int N, int M, int D, int dtype,
                            float* q_out, float* z_out, int force_chunks, void* stream);

/* Same operation with HOST buffers (end-to-end form): streams the (b, h)
 * slices through the GPU -- the copy-in of one slice, the forward of the
 * previous one (on `stream`) and the copy-out of the one before overlap, on two
 * library-owned copy streams -- and synchronises `stream` before returning.
 * Device staging (two slices of inputs and output, the latent inputs, scratch)
 * comes from a library-owned memory pool that keeps it reserved between calls.
 * Pinned host memory lets the copies run at full speed; pageable memory works
 * but is slower.  gate is a HOST float[H] here (NULL = FLARE).  The result is
 * identical to flarepp_mixer_fwd's up to the token-chunk split, which is
 * planned per slice here. */
int flarepp_mixer_fwd_host(const void* q0, const void* q_fixed, const float* gate,
                           const void* k0, const void* k, const void* v, void* y,
                           int B, int H, int N, int M, int D, int dtype, void* stream);

/* FLARE++ mixer forward that allocates no memory: the same operation, arguments
 * and result as flarepp_mixer_fwd (up to rounding: it may split the token axis
 * into fewer chunks), with its scratch taken from a fixed device array inside
 * the library instead of cudaMallocAsync.  (This entry has no counterpart in
 * the FLARE++ paper or pages; it serves callers that cannot allocate device
 * memory during the call: code whose memory belongs to another allocator,
 * such as a framework's caching allocator or a pre-reserved arena that may
 * not be bypassed, and code that must not run the implicit synchronisation a
 * cudaMalloc/cudaFree can bring.)
 *   - The array holds FLAREPP_NOALLOC_SCRATCH_BYTES and every GPU that loads
 *     the library keeps it until the process exits.  A problem whose scratch
 *     does not fit even with one token chunk returns FLAREPP_ERR_WORKSPACE and
 *     launches nothing.
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress) and caches it; make that first call before
 *     any stream capture.
 *   - All calls share the array.  Calls whose kernels overlap on the GPU
 *     (different streams, or different host threads on one device) race on
 *     it and give undefined results: serialise them.
 *   - No cudaMalloc, cudaFree or allocating library routine is called. */
#define FLAREPP_NOALLOC_SCRATCH_BYTES (32u << 20)
int flarepp_mixer_fwd_noalloc(const void* q0, const void* q_fixed, const float* gate,
                              const void* k0, const void* k, const void* v, void* y,
                              int B, int H, int N, int M, int D, int dtype, void* stream);

/* Which kernel family AUTO would run for this shape (flarepp_path_t), or 0 for
 * arguments the forward entries would reject. */
int flarepp_selected_path(int B, int H, int N, int M, int D, int dtype);

/* Diagnostic for the failure path: launches on `stream` one thread that waits,
 * with the kernels' bounded wait and a limit of limit_us microseconds
 * (1 .. 1e6), on an mbarrier nothing ever arrives at.  The wait gives up and
 * records FLAREPP_ERR_TIMEOUT in the device status word, which the next
 * flarepp_check_device_status returns (and clears); the context stays usable.
 * Returns the launch status. */
int flarepp_selftest_wait_timeout(void* stream, unsigned int limit_us);

/* Synchronises `stream`, then returns and clears the device status word
 * (FLAREPP_OK when no kernel recorded a failure on the current device). */
int flarepp_check_device_status(void* stream);

/* Static text for a status code. */
const char* flarepp_status_string(int status);

/* ---------------------------------------------------------------------------
 * Token-sharded (context-parallel) form, physicsnemo issue #2024, section 2:
 * the N tokens are split across ranks and no rank holds the whole sequence.
 * (An extension beyond the single-GPU forward that the library's benchmark
 * measures; the single-GPU entries above do not depend on it.)
 * Each rank runs the split softmax passes on its own tokens and reduces them
 * to one unnormalised triple (row max in log2 units, row sum, weighted sum of
 * the value rows) per latent row; the ranks' triples are all-gathered (by the
 * caller, e.g. NCCL) and merged by log-sum-exp, which rebuilds the globally
 * normalised attention exactly up to rounding; the decode stays local.  Per
 * rank, for the gated form:
 *     flarepp_cp_partials(q0, 1, k0, k0, T)   all-gather T -> Tg
 *     flarepp_cp_merge(Tg, G, q_fixed, gate, Q)            routing queries q
 *     flarepp_cp_partials(Q, 0, k, v, T)      all-gather T -> Tg
 *     flarepp_cp_merge(Tg, G, NULL, NULL, Z)               latents z
 *     flarepp_cp_decode(Q, 0, Z, k, y)
 * and for the closed gate (FLARE) the encode and decode take q_fixed with
 * q_shared = 1.  N is this rank's token count (>= 1); k0, k, v, y hold this
 * rank's tokens in the layout of opts->layout.  Every rank must use the same
 * B, H, M, D, dtype, scale and rank order.  Arguments, ownership, alignment,
 * errors and asynchrony are as for flarepp_mixer_fwd_ex; opts (may be NULL)
 * supplies scale, path, force_chunks, workspace and layout.
 * ------------------------------------------------------------------------ */

/* Bytes of one rank's triple buffer T: B*H*M*(D+2) fp32 -- the O rows
 * [B,H,M,D] followed by (max, sum) pairs [B,H,M,2].  The all-gathered buffer
 * Tg is G such buffers back to back in rank order.  0 for invalid sizes. */
size_t flarepp_cp_triple_bytes(int B, int H, int M, int D);

/* Bytes of a latent state Q or Z: [B,H,M,D] fp32, then (16-bit I/O) the same
 * rows in the I/O dtype at a 256-byte-aligned offset.  0 for invalid sizes. */
size_t flarepp_cp_latent_bytes(int B, int H, int M, int D, int dtype);

/* One split pass over this rank's N tokens into `triple` (DEVICE, 16-byte
 * aligned, flarepp_cp_triple_bytes).  q: q_shared = 1 -> [H,M,D] in the I/O
 * dtype (q0 for the synthesis, q_fixed for the closed-gate encode);
 * q_shared = 0 -> a latent state from flarepp_cp_merge.  v == k reads each key
 * tile once and uses it as the value tile (the synthesis, V = K = k0). */
int flarepp_cp_partials(const void* q, int q_shared, const void* k, const void* v, float* triple,
                        int B, int H, int N, int M, int D, int dtype,
                        const flarepp_options_t* opts, void* stream);

/* Log-sum-exp merge of `ranks` gathered triples into the latent state `state`
 * (DEVICE, flarepp_cp_latent_bytes).  gate != NULL: synthesis, state = q =
 * q_fixed + gate * merged (q_fixed [H,M,D] in the I/O dtype, gate fp32 [H]);
 * gate == NULL: encode, state = z = merged (q_fixed ignored). */
int flarepp_cp_merge(const float* gathered, int ranks, const void* q_fixed, const float* gate, void* state,
                     int B, int H, int M, int D, int dtype, void* stream);

/* Decode of this rank's N tokens: y = SDPA(k, q, z) with q as in
 * flarepp_cp_partials (the routing-query state, or q_fixed with q_shared = 1)
 * and z_state from the encode merge; y in the token layout of opts. */
int flarepp_cp_decode(const void* q, int q_shared, const void* z_state, const void* k, void* y,
                      int B, int H, int N, int M, int D, int dtype,
                      const flarepp_options_t* opts, void* stream);

/* Log-sum-exp merge as flarepp_cp_merge that also writes, for the backward,
 * lse_out: fp32 [B,H,M], each latent row's log-sum-exp over all ranks' tokens
 * (log2 units, of the scores times scale*log2(e)), and (gate != NULL)
 * pregate_out: fp32 [B,H,M,D], the merged value before the gate.  Either may
 * be NULL; neither may overlap the state or the gathered triples. */
int flarepp_cp_merge_ex(const float* gathered, int ranks, const void* q_fixed, const float* gate, void* state,
                        float* lse_out, float* pregate_out, int B, int H, int M, int D, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * Backward: the gradients of a scalar loss L with respect to every input of
 * the mixer, given dy = dL/dy.  By the chain rule through each softmax
 * attention O = softmax(scale Q K^T) V of the FLARE++ block (FLARE.py
 * README, "FLARE++" code block; the same algebra as FlashAttention's backward,
 * applied to the decode, the encode, the gate q = q_fixed + gate * q_dyn and
 * the synthesis in that order).  The forward is not saved: the call runs the
 * forward's synthesis and encode passes again, on the forward's own kernel
 * family, and recomputes the decode's per-token softmax inside the backward.
 * The physicsnemo issue #2024 speaks of the encoder's custom backward; the
 * pages state no formulas for it, so this is the plain chain rule.
 *
 * Arguments (same conventions, limits and checks as flarepp_mixer_fwd_ex):
 *   q0, q_fixed, gate, k0, k, v   the forward's inputs (gate == NULL: FLARE,
 *                                 then q0, k0, dq0, dgate, dk0 are ignored)
 *   dy        [B,H,N,D] token layout, I/O dtype: the gradient of y
 *   dq0, dq_fixed   DEVICE fp32 [H,M,D] (sums over the batch)
 *   dgate     DEVICE fp32 [H]: dL/d(gate value), not of the logit
 *   dk0, dk, dv     [B,H,N,D] token layout, I/O dtype
 * No output may overlap an input or another output.  opts (may be NULL):
 * scale, path (the kernel family: with 16-bit I/O the tcgen05 forward and the
 * tcgen05 backward kernel, whose score and gradient products take bf16/fp16
 * operands -- P and dS rounded to the I/O type -- with fp32 accumulation;
 * with fp32 I/O, or path = SIMT, fp32 SIMT kernels throughout), force_chunks
 * (the token chunks of both the recomputed passes and the backward's token sums),
 * workspace / workspace_bytes (>= flarepp_mixer_bwd_workspace_bytes),
 * stage_events (recorded before the first and after every launch), layout,
 * norm_synthesis (the synthesis reads RMS-normalised q0 and k0 rows as in the
 * forward, and dq0, dk0 are taken through that step: dx = r (g - xh <g, xh>/D)
 * per row, xh = x r, r = (mean x^2 + 1e-6)^(-1/2); three more launches).
 * q_out, z_out are ignored.
 * Sums over tokens are taken per token chunk and added in a fixed order
 * (deterministic); the 16-bit gradients are rounded once, at the end.
 * Asynchronous on `stream`. */
int flarepp_mixer_bwd(const void* q0, const void* q_fixed, const float* gate,
                      const void* k0, const void* k, const void* v, const void* dy,
                      float* dq0, float* dq_fixed, float* dgate,
                      void* dk0, void* dk, void* dv,
                      int B, int H, int N, int M, int D, int dtype,
                      const flarepp_options_t* opts, void* stream);

/* Bytes of device scratch one backward call needs (the forward's scratch,
 * the log-sum-exps, fp32 latent gradients, per-chunk partial sums and an
 * fp32 [B,H,N,D] buffer for the decode's share of dk).  0 for arguments the
 * backward would reject. */
size_t flarepp_mixer_bwd_workspace_bytes(int B, int H, int N, int M, int D, int dtype,
                                         const flarepp_options_t* opts);

/* Kernel launches one backward call makes, for the kernel family `path`
 * (flarepp_path_t, as flarepp_selected_path reports it) of its recomputed
 * forward: SIMT, gated 14 (4 recomputed forward passes, 3 per attention, 1
 * batch reduce), closed gate 9; TCGEN05, also gated 14 and closed gate 9 (the
 * forward's decode runs too, for the per-token statistics, and the token
 * sides of the decode and the encode are one launch).  A gated call with
 * norm_synthesis makes three more: the normalisation of q0, k0 first, and the
 * gradients of k0 and q0 through it last. */
int flarepp_mixer_bwd_launches(int gated, int path);

/* ---------------------------------------------------------------------------
 * Training step with saved forward state.  (A convenience of this library for
 * a forward followed by its backward; the pages have no counterpart.)
 * flarepp_mixer_fwd_train is flarepp_mixer_fwd_ex (same arguments, checks and
 * result y, bitwise) that also writes into the caller-owned DEVICE buffer ctx
 * (256-byte aligned, >= flarepp_train_context_bytes) what the backward would
 * otherwise recompute: q and z (fp32 [B,H,M,D]), the synthesis output before
 * the gate, the per-latent log-sum-exps of the synthesis and the encode, and
 * (tcgen05 path) the decode's per-token log-sum-exp -- latent-sized except the
 * last, B*H*N*8 bytes.  opts->q_out and opts->z_out are ignored (the context
 * holds q and z).  ctx must not overlap any tensor argument.
 * flarepp_mixer_bwd_ctx is flarepp_mixer_bwd given that context and the
 * forward's output y (token layout, I/O dtype): it skips the recomputed
 * forward passes (on the tcgen05 path it rounds q and z to the I/O dtype for
 * the tensor cores and takes <dy, y> per token from y).  The inputs, shape,
 * dtype and options must be those of the forward call that filled ctx;
 * nothing checks this.  Results equal flarepp_mixer_bwd's up to rounding (the
 * per-token <dy, y> uses the rounded y).  Launches: the backward's minus the
 * recomputed forward passes, plus two (q/z rounding, <dy, y>) on the tcgen05
 * path.  Errors: ctx NULL or misaligned, y NULL -> FLAREPP_ERR_INVALID_ARG;
 * ctx_bytes too small -> FLAREPP_ERR_WORKSPACE. */
size_t flarepp_train_context_bytes(int B, int H, int N, int M, int D, int dtype);
int flarepp_mixer_fwd_train(const void* q0, const void* q_fixed, const float* gate,
                            const void* k0, const void* k, const void* v, void* y,
                            int B, int H, int N, int M, int D, int dtype,
                            const flarepp_options_t* opts, void* ctx, size_t ctx_bytes, void* stream);
int flarepp_mixer_bwd_ctx(const void* q0, const void* q_fixed, const float* gate,
                          const void* k0, const void* k, const void* v, const void* y, const void* dy,
                          float* dq0, float* dq_fixed, float* dgate,
                          void* dk0, void* dk, void* dv,
                          int B, int H, int N, int M, int D, int dtype,
                          const flarepp_options_t* opts, const void* ctx, size_t ctx_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Token-sharded backward (physicsnemo issue #2024, section 2: the distributed
 * encoder and its backward).  Every sum over tokens in the backward is a sum
 * of per-rank sums, every sum over latents is local; so each rank runs the
 * backward's steps on its own tokens in four stages, and after stages 1, 2
 * and 3 the caller sums one fp32 region of every rank's state over the ranks,
 * in place (an all-reduce, e.g. NCCL), before the next stage:
 *   stage 1: per-token decode statistics; the decode's latent side -> region 0
 *   stage 2: dz, the token sides of decode and encode (dk, dv of this rank's
 *            tokens), the encode's latent side                  -> region 1
 *   stage 3: dq, dq_dyn; the synthesis' token side (dk0), its latent side
 *                                                               -> region 2
 *   stage 4: dq_fixed, dq0, dgate (the same on every rank).
 * Arguments: the latent inputs and gate as for flarepp_mixer_bwd; q_state and
 * z_state: the merged states of the forward's token-sharded passes
 * (flarepp_cp_merge; q_state is ignored with the gate closed); lse_syn,
 * lse_enc, qdyn: from flarepp_cp_merge_ex of the synthesis and the encode
 * merges (lse_syn and qdyn ignored with the gate closed); k0, k, v, dy and
 * dk0, dk, dv: this rank's N tokens in the layout of opts; dq0, dq_fixed,
 * dgate as for flarepp_mixer_bwd.  Pass the same arguments to every stage and
 * the same sizes, dtype and options on every rank.  state: DEVICE, 256-byte
 * aligned, flarepp_cp_bwd_layout().bytes, kept by the caller across the four
 * stages.  opts: as for flarepp_mixer_bwd (q_out, z_out must be NULL).
 * Errors and asynchrony as for flarepp_mixer_bwd; stage outside 1..4 ->
 * FLAREPP_ERR_INVALID_ARG. */
typedef struct flarepp_cp_bwd_layout {
    size_t bytes;               /* the per-rank state */
    size_t reduce_offset[3];    /* byte offset in the state of the region stage 1, 2, 3 leaves to sum */
    size_t reduce_bytes[3];     /* its size (fp32 values) */
} flarepp_cp_bwd_layout_t;

int flarepp_cp_bwd_layout(int B, int H, int N, int M, int D, int dtype, const flarepp_options_t* opts,
                          flarepp_cp_bwd_layout_t* out);

int flarepp_cp_bwd_stage(int stage, const void* q0, const void* q_fixed, const float* gate,
                         const void* q_state, const void* z_state,
                         const float* lse_syn, const float* lse_enc, const float* qdyn,
                         const void* k0, const void* k, const void* v, const void* dy,
                         float* dq0, float* dq_fixed, float* dgate, void* dk0, void* dk, void* dv,
                         void* state, int B, int H, int N, int M, int D, int dtype,
                         const flarepp_options_t* opts, void* stream);

/* FLAREPP_ABI_VERSION of the loaded library. */
int flarepp_abi_version(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* FLAREPP_H_ */
