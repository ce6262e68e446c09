/*
 * moe.h -- C ABI of libmoe: one DeepSeek-V3-style MoE layer forward on one
 * B200 (sm_100a).
 *
 * The layer (sources are the pages' titles and sections):
 *   route     s_i = sigmoid(x . e_i [+ o_i]); b_i = s_i + bias_i picks experts
 *             only ("MoE + Expert-Parallel Overlap (Exp08)", Implemented:
 *             top-k gating, per-expert bias balancing); node-limited top-K:
 *             the E experts form G contiguous groups standing in for nodes
 *             ("moe-node-limited-routing", opening definition; deepnotes
 *             "The real cluster, and the mesh DeepSeek actually disclosed":
 *             four experts per GPU), the M groups with the largest sum of
 *             their top-(K/M) b are kept, the top-K b inside them are chosen
 *             (ties to the lower index), gates w_j = s_j / sum s over the K
 *             chosen UNBIASED affinities.
 *   dispatch  the token copies are sorted by expert into expert-contiguous
 *             rows (stable: tokens ascending inside a segment) with counts,
 *             offsets and the group-to-group send matrices (the dispatch
 *             all-to-all of "moe-node-limited-routing", "Why all to all
 *             dominates MoE step time", becomes a local permutation; "send
 *             matrices", shivam2003 "5. Tail latency controls step time").
 *   expert    y = W_d (SiLU(W_g x) * (W_u x)) per expert on its rows, plus
 *             the always-on shared experts on every token (Exp08,
 *             Implemented: shared + fine-grained routed experts).
 *   combine   out_t = shared_t + sum_j w_j y_(t,j) back in token order (the
 *             combine all-to-all, same section).
 * Variants (same passage of Exp08, Implemented): the V4 affinity
 * sqrt(softplus(L)) in place of the sigmoid, a hash router for early layers,
 * and the per-expert bias update that balances the load without an
 * auxiliary loss (moe_config.router, moe_route_hash, moe_bias_update).
 *
 * Conventions for every entry point:
 *   - Tensors are DEVICE pointers to dense row-major arrays; bf16 data is
 *     passed as `void *` (IEEE bfloat16 bit patterns).  The caller owns every
 *     buffer; the library never allocates, frees, or keeps a pointer after
 *     the call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     compute entry point only enqueues kernels: it returns before they run,
 *     performs no host<->device copy and no synchronisation.
 *   - A nonzero moe_status means nothing was enqueued (argument errors) or a
 *     launch failed (MOE_ERR_CUDA).  Faults found by the kernels themselves
 *     (an expert id out of range, a bounded wait that ran out) are written to
 *     the status word at the start of the workspace; read it with
 *     moe_read_device_status() after the stream has run.
 *   - Buffers must be 16-byte aligned; the workspace 256-byte aligned.
 *   - Sizes supported: E % G == 0, K % M == 0, K/M <= E/G, M <= G, K <= 32,
 *     E <= 1024, G <= 64, T % G == 0, d % 64 == 0, d_ff % 64 == 0,
 *     d_ff_shared % 64 == 0, T*K < 2^31, T >= 0 (T == 0 is a no-op).
 *     Anything else returns MOE_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Router of the layer (moe_config.router). */
typedef enum moe_router {
    MOE_ROUTER_SIGMOID = 0,       /* s = sigmoid(L) (DeepSeek-V3); the default */
    MOE_ROUTER_SQRT_SOFTPLUS = 1, /* s = sqrt(log(1 + e^L)) (the V4 form)      */
    MOE_ROUTER_HASH = 2           /* experts from a hash of the token id       */
} moe_router;

/* Element type of the dispatched (routed) copies of x (moe_config.payload). */
typedef enum moe_payload {
    MOE_PAYLOAD_BF16 = 0, /* x_perm in bf16; the default                       */
    MOE_PAYLOAD_FP8 = 1   /* FP8 E4M3 codes + one fp32 scale per 128 channels   */
} moe_payload;

/* Layer sizes, router and payload.  Zero-initialised `router` and `payload`
 * are the sigmoid router and the bf16 payload. */
typedef struct moe_config {
    int32_t T;           /* tokens in the batch                               */
    int32_t d;           /* hidden size                                       */
    int32_t E;           /* routed experts                                    */
    int32_t G;           /* expert groups (emulated nodes), E/G experts each  */
    int32_t K;           /* routed experts per token                          */
    int32_t M;           /* max groups a token may use                        */
    int32_t d_ff;        /* routed expert intermediate size                   */
    int32_t n_shared;    /* always-on shared experts (0 allowed)              */
    int32_t d_ff_shared; /* shared expert intermediate size                   */
    int32_t router;      /* moe_router; other values: UNSUPPORTED_SHAPE       */
    int32_t payload;     /* moe_payload; FP8 needs d % 128 == 0               */
} moe_config;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,         /* NULL required pointer, bad alignment   */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* sizes outside the supported set above  */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < moe_workspace_size(cfg)     */
    MOE_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed      */
    MOE_ERR_DEVICE_TIMEOUT = 5,      /* device status: a bounded wait ran out  */
    MOE_ERR_DEVICE_FAULT = 6,        /* device status: bad index in the inputs */
    MOE_ERR_NO_DEVICE = 7            /* no sm_100 device is current            */
} moe_status;

/* Validates sizes only (no CUDA call).  MOE_OK or MOE_ERR_UNSUPPORTED_SHAPE /
 * MOE_ERR_INVALID_ARG (cfg == NULL). */
MOE_API moe_status moe_check_config(const moe_config *cfg);

/* Bytes of device workspace every entry point that takes `ws` may use for
 * this configuration; 0 if the configuration is unsupported.  Monotone in T. */
MOE_API size_t moe_workspace_size(const moe_config *cfg);

/* Static English text for a status code (never NULL). */
MOE_API const char *moe_status_string(int status);

/* Number of kernels this library has launched in this process (all devices,
 * all streams).  For accounting; not synchronised with the GPU. */
MOE_API uint64_t moe_launch_count(void);

/* Copies the workspace status word to *host_status after synchronising
 * `stream` (the only entry point that synchronises).  MOE_OK if no kernel
 * recorded a fault since the last moe_clear_device_status(). */
MOE_API moe_status moe_read_device_status(const void *ws, int32_t *host_status, void *stream);

/* The same read, returning the device status word itself: MOE_OK, or the
 * MOE_ERR_DEVICE_* code a kernel recorded; a host-side failure of the read
 * (ws NULL, no device, a CUDA error) is returned in its place. */
MOE_API moe_status moe_last_device_status(const void *ws, void *stream);

/* Enqueues a reset of the workspace status word to MOE_OK. */
MOE_API moe_status moe_clear_device_status(void *ws, void *stream);

/*
 * Router (affinity + node-limited top-K) for cfg->router SIGMOID or
 * SQRT_SOFTPLUS (HASH: MOE_ERR_INVALID_ARG; use moe_route_hash).
 *   x            [T, d]   bf16
 *   router_w     [E, d]   fp32  (e_i rows)
 *   logit_offset [E]      fp32 or NULL: added to x . e_i before the affinity
 *   bias         [E]      fp32: selection-only balance bias (NULL = zeros)
 *   topk_idx     [T, K]   int32 out: chosen experts, descending b_i then
 *                               ascending index
 *   topk_w       [T, K]   fp32 out: gates, sum to 1 over the K slots
 *   scores       [T, E]   fp32 out or NULL (then kept in the workspace):
 *                               the affinities s
 *   ws, ws_bytes          workspace of moe_workspace_size(cfg) bytes (required)
 * L = x . e_i on the tensor cores: e_i is split into three bf16 parts whose
 * sum reproduces the fp32 value to ~2^-27 relative, the products are exact,
 * and the accumulation is fp32; s = 1 / (1 + expf(-L)), or for SQRT_SOFTPLUS
 * s = sqrtf(softplus(L)) with softplus(L) = L + log1pf(expf(-L)) for L > 0,
 * log1pf(expf(L)) otherwise (no overflow on either side).
 */
MOE_API moe_status moe_route(const moe_config *cfg, const void *x, const float *router_w,
                     const float *logit_offset, const float *bias,
                     int32_t *topk_idx, float *topk_w, float *scores,
                     void *ws, size_t ws_bytes, void *stream);

/* Selection only, from given fp32 affinities scores[T, E]: exactly the
 * selection and gate steps of moe_route.  Same fp32 operations in the same
 * order as the written-out definition, so equal inputs give equal bits. */
MOE_API moe_status moe_route_select(const moe_config *cfg, const float *scores, const float *bias,
                            int32_t *topk_idx, float *topk_w, void *stream);

/*
 * Hash router ("a hash router for early-layer emulation", Exp08,
 * Implemented; the page gives no formula, this is the library's reading):
 * the node limit is kept -- a token takes M of the G groups and K/M experts
 * in each, drawn without replacement by a partial Fisher-Yates shuffle driven
 * by the lowbias32 integer hash of its 64-bit id; every gate is 1/K.
 *   token_ids  [T]     int64, or NULL: the row index t is the id
 *   topk_idx   [T, K]  int32 out: slots grouped by group in draw order
 *   topk_w     [T, K]  fp32 out: 1/K
 * Deterministic: equal ids give equal routes, on any batch position.
 * cfg->router is not consulted.
 */
MOE_API moe_status moe_route_hash(const moe_config *cfg, const int64_t *token_ids,
                                  int32_t *topk_idx, float *topk_w, void *stream);

/*
 * Per-expert bias update of auxiliary-loss-free balancing ("per-expert bias
 * updates", Exp08, Implemented; the sign rule of DeepSeek-V3, its step size a
 * parameter): every expert above the mean load T*K/E moves its bias down by
 * gamma, every expert below it moves up, one exactly at the mean keeps it:
 *   bias[i] = bias[i] + gamma * sign(T*K/E - counts[i])   (one fp32 add)
 * The comparison is exact (counts[i] * E against T * K in 64-bit integers).
 *   counts  [E]  int32: copies per expert, as moe_dispatch / moe_forward write
 *   gamma        fp32 step (finite)
 *   bias    [E]  fp32 in/out
 */
MOE_API moe_status moe_bias_update(const moe_config *cfg, const int32_t *counts, float gamma,
                                   float *bias, void *stream);

/*
 * Dispatch: stable counting sort of the T*K token copies by expert.
 *   topk_idx   [T, K]   int32 in (distinct experts per token, each < E)
 *   counts     [E]      int32 out: copies per expert
 *   offsets    [E+1]    int32 out: exclusive prefix sum of counts
 *   send       [G, G]   int32 out: copies from source group (t / (T/G)) to
 *                               expert group (e / (E/G)); sums to T*K
 *   send_tok   [G, G]   int32 out (or NULL): tokens from source group to
 *                               expert group, one per token and group
 *   perm_token [T*K]    int32 out: token of each permuted row
 *   inv_perm   [T, K]   int32 out: permuted row of copy (t, j)
 *   x_perm     [T*K, d] bf16 out (or NULL): x_perm[row] = x[perm_token[row]]
 * Bad ids are skipped and flagged MOE_ERR_DEVICE_FAULT in the status word.
 */
MOE_API moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                        int32_t *counts, int32_t *offsets, int32_t *send, int32_t *send_tok,
                        int32_t *perm_token, int32_t *inv_perm, void *x_perm,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * The gather-permute step of moe_dispatch alone: x_perm[inv_perm[t][j]] = x[t]
 * for every copy (t, j), 16-byte vector copies reading each x row once.
 *   x         [T, d]     bf16
 *   inv_perm  [T, K]     int32 from moe_dispatch (rows outside [0, T*K) are
 *                        skipped)
 *   x_perm    [T*K, d]   bf16 out
 * moe_dispatch(x_perm = NULL) followed by moe_permute equals moe_dispatch
 * with x_perm, bit for bit.
 */
MOE_API moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *inv_perm,
                               void *x_perm, void *stream);

/*
 * moe_dispatch for callers that cannot allocate device memory.  No passage of
 * the pages has a counterpart: this entry point exists for deployment only.
 * Callers such as a serving runtime that owns the whole HBM budget through
 * its own pool, or a latency-critical path that cannot afford cudaMalloc's
 * implicit device synchronisation, get the same results as moe_dispatch
 * (same kernels, bit for bit) without passing a workspace.
 *   Arguments are those of moe_dispatch, without ws / ws_bytes, plus
 *   device_status: a device int32 (or NULL) that receives the first fault a
 *   kernel finds (MOE_ERR_DEVICE_FAULT for a bad expert id); the caller
 *   clears it.  With NULL, faults are not reported.
 *   Scratch: a fixed 4 MiB static device array, held by every GPU that loads
 *   the library until the process exits.  This call needs
 *   256 + 2 * r(4 E n) + 2 * r(4 n G^2) bytes of it, n = ceil(T / 256) and
 *   r() rounding up to 256; larger sizes return MOE_ERR_WORKSPACE_TOO_SMALL
 *   before anything is launched (the five named workloads need at most
 *   0.3 MiB).  It allocates and frees nothing.
 *   First call on a device: it looks up the array's device address with
 *   cudaGetSymbolAddress (with that device current) and keeps it once the
 *   lookup has succeeded; make that first call before any stream capture.  A
 *   lookup that fails returns MOE_ERR_CUDA and is not kept, so a later call
 *   on that device tries again.
 *   Every call uses the same array: nothing in it has to start at zero
 *   (each call writes every scratch word before reading it), but calls whose
 *   kernels overlap on the GPU -- on two streams, or from two threads --
 *   race on it and give wrong results.  Serialise them.
 */
MOE_API moe_status moe_dispatch_noalloc(const moe_config *cfg, const void *x,
                                        const int32_t *topk_idx, int32_t *counts,
                                        int32_t *offsets, int32_t *send, int32_t *send_tok,
                                        int32_t *perm_token, int32_t *inv_perm, void *x_perm,
                                        int32_t *device_status, void *stream);

/*
 * FP8 dispatch payload ("sending fewer bytes through lower-precision
 * activations", "DeepSeek 8.7 - communication", section 4; the format is the
 * library's reading, DeepSeek-V3's recipe): the dispatch of moe_dispatch, but
 * the permuted copies of x are written as OCP FP8 E4M3 codes with one fp32
 * scale per token and 128-channel block:
 *   s = amax / 448 over the block (fp32),  q = E4M3(x / s) (fp32 division,
 *   nearest-even, saturating to +-448);  an all-zero block has s = 0, q = 0.
 *   x_perm_q  [T*K, d]      uint8 out (codes)
 *   x_scale   [T*K, d/128]  fp32 out
 *   other arguments as moe_dispatch.  Needs d % 128 == 0 (else
 *   MOE_ERR_UNSUPPORTED_SHAPE); half the bytes of a bf16 x_perm plus 1/64.
 */
MOE_API moe_status moe_dispatch_fp8(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                                    int32_t *counts, int32_t *offsets, int32_t *send,
                                    int32_t *send_tok, int32_t *perm_token, int32_t *inv_perm,
                                    uint8_t *x_perm_q, float *x_scale, void *ws, size_t ws_bytes,
                                    void *stream);

/*
 * Expert FFN on the FP8 payload: as moe_expert_ffn, with the routed rows given
 * as x_perm_q / x_scale (moe_dispatch_fp8).  The gate/up GEMM widens each row
 * to x_hat = bf16(float(E4M3^-1(q)) * s) (one fp32 multiply, bf16 nearest-even)
 * in shared memory before the tensor cores read it, so the results equal
 * moe_expert_ffn on x_perm = x_hat bit for bit.  The shared experts read x.
 */
MOE_API moe_status moe_expert_ffn_fp8(const moe_config *cfg, const uint8_t *x_perm_q,
                                      const float *x_scale, const int32_t *offsets,
                                      const void *w_gate, const void *w_up, const void *w_down,
                                      void *y_perm, const void *x, const void *ws_gate,
                                      const void *ws_up, const void *ws_down, void *y_shared,
                                      void *ws, size_t ws_bytes, void *stream);

/*
 * Expert FFN: grouped SwiGLU over the expert segments plus the shared experts.
 *   x_perm    [T*K, d]             bf16 expert-contiguous rows
 *   offsets   [E+1]                int32 segment starts (offsets[E] == T*K)
 *   w_gate    [E, d_ff, d]         bf16     w_up [E, d_ff, d]   bf16
 *   w_down    [E, d, d_ff]         bf16
 *   y_perm    [T*K, d]             bf16 out: y_perm[r] = FFN_e(x_perm[r])
 *   x         [T, d]               bf16 (shared-expert input; may be NULL
 *                                  only when n_shared == 0)
 *   ws_gate   [n_shared, d_ff_shared, d]   ws_up same   bf16
 *   ws_down   [n_shared, d, d_ff_shared]   bf16
 *   y_shared  [T, d]               bf16 out: sum of the shared FFNs
 * tcgen05 tensor cores, fp32 accumulation; the intermediate h = SiLU(gate) *
 * up is rounded to bf16 (nearest even) before the down projection.
 * Passage: "MoE + Expert-Parallel Overlap (Exp08)", Implemented: shared
 * (always active) plus fine-grained routed experts; its overlap simulator
 * counts 6*d*d_ff FLOPs per token-expert pair, the work this call does.
 * No counts argument: a segment's length is offsets[e+1] - offsets[e].
 * Errors: MOE_ERR_INVALID_ARG (a required pointer NULL or not 16-byte
 * aligned, ws not 256-byte aligned), MOE_ERR_WORKSPACE_TOO_SMALL,
 * MOE_ERR_UNSUPPORTED_SHAPE (d or d_ff not a multiple of 64); offsets that
 * are not monotone or leave [0, T*K] are skipped on the device and flagged
 * MOE_ERR_DEVICE_FAULT in the status word.
 */
MOE_API moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                          const void *w_gate, const void *w_up, const void *w_down,
                          void *y_perm, const void *x, const void *ws_gate,
                          const void *ws_up, const void *ws_down, void *y_shared,
                          void *ws, size_t ws_bytes, void *stream);

/*
 * Expert FFN fused with the dispatch gather: as moe_expert_ffn, but the routed
 * rows are read straight from x -- row r of expert segment e is
 * x[perm_token[r]] -- by gatherer warps of the gate/up GEMM (16-byte
 * asynchronous copies into the swizzled operand stage), so the permuted copy
 * x_perm is never written or read (the gather-permute step of
 * the dispatch, "moe-node-limited-routing", "Why all to all dominates MoE step
 * time", folded into the expert GEMM).
 *   x           [T, d]     bf16
 *   perm_token  [T*K]      int32 from moe_dispatch (values in [0, T))
 *   other arguments as moe_expert_ffn (x also feeds the shared experts).
 * Results are bit-identical to moe_dispatch(x_perm) + moe_expert_ffn.
 * A perm_token value outside [0, T) is read as row 0 and flagged
 * MOE_ERR_DEVICE_FAULT in the status word.
 */
MOE_API moe_status moe_expert_ffn_gather(const moe_config *cfg, const void *x,
                                         const int32_t *perm_token, const int32_t *offsets,
                                         const void *w_gate, const void *w_up, const void *w_down,
                                         void *y_perm, const void *ws_gate, const void *ws_up,
                                         const void *ws_down, void *y_shared, void *ws,
                                         size_t ws_bytes, void *stream);

/*
 * Combine: out[t] = y_shared[t] + sum_j topk_w[t,j] * y_perm[inv_perm[t,j]],
 * fp32 accumulation, rounded to bf16.  y_shared may be NULL (treated as 0).
 * Passage: "moe-node-limited-routing", "Why all to all dominates MoE step
 * time": the combine all-to-all that returns each expert output to its
 * token, here a local gather in token order, weighted by the gates.
 *   y_perm   [T*K, d] bf16, inv_perm [T, K] int32 (row of copy (t, j), -1 for
 *            none), topk_w [T, K] fp32, out [T, d] bf16; all caller-owned.
 * Errors: MOE_ERR_INVALID_ARG (a required pointer NULL or not 16-byte
 * aligned); rows of inv_perm outside [0, T*K) count as 0.
 */
MOE_API moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *inv_perm,
                       const float *topk_w, const void *y_shared, void *out, void *stream);

/*
 * The whole layer: route -> dispatch -> expert FFN -> combine on `stream`.
 *   out [T, d] bf16 out.  topk_idx [T,K], topk_w [T,K], counts [E],
 *   offsets [E+1], send [G,G], send_tok [G,G] are optional outputs (NULL:
 *   kept in the workspace).  Intermediates live in the workspace.
 *   The dispatch writes x_perm into the workspace and the expert FFN reads it
 *   (moe_expert_ffn); moe_expert_ffn_gather gives the same bits without
 *   x_perm but runs slower.  With cfg->payload == MOE_PAYLOAD_FP8 the copies
 *   travel as FP8 (moe_dispatch_fp8 + moe_expert_ffn_fp8); the router and the
 *   shared experts still read x.
 *   The route is cfg->router's: moe_route's for SIGMOID and SQRT_SOFTPLUS
 *   (router_w required, token_ids ignored), moe_route_hash's for HASH
 *   (token_ids [T] int64 or NULL; router_w, logit_offset, bias ignored).
 */
MOE_API moe_status moe_forward(const moe_config *cfg, const void *x, const float *router_w,
                       const float *logit_offset, const float *bias, const int64_t *token_ids,
                       const void *w_gate, const void *w_up, const void *w_down,
                       const void *ws_gate, const void *ws_up, const void *ws_down,
                       void *out, int32_t *topk_idx, float *topk_w, int32_t *counts,
                       int32_t *offsets, int32_t *send, int32_t *send_tok,
                       void *ws, size_t ws_bytes, void *stream);

/*
 * Packed expert weights.  The grouped GEMMs stream every expert weight from
 * HBM about once per step (6 d d_ff FLOPs per token-expert against 3 d d_ff
 * weight elements, "MoE + Expert-Parallel Overlap (Exp08)", Implemented /
 * overlap simulator: at V3 sizes each weight byte feeds only ~2.5 tiles of
 * 128 token rows), so their speed follows the weights' DRAM access pattern.
 * moe_pack_weights rewrites the routed and shared expert weights once (at
 * model load) as contiguous, pre-swizzled 32 KB tiles in the order the GEMMs
 * read them; moe_expert_ffn_packed and moe_forward_packed then fetch each
 * tile with one bulk copy.  The arithmetic is unchanged: the packed entry
 * points return the same bits as moe_expert_ffn / moe_forward.
 *   moe_packed_weights_size  bytes of the packed buffer (0: unsupported cfg);
 *                            about the bytes of the six weight tensors
 *   moe_pack_weights         w_gate, w_up [E, d_ff, d], w_down [E, d, d_ff],
 *                            ws_gate, ws_up [n_shared, d_ff_shared, d],
 *                            ws_down [n_shared, d, d_ff_shared] (bf16, the
 *                            layouts of moe_expert_ffn) -> packed (device,
 *                            moe_packed_weights_size bytes, 16-byte aligned).
 *                            Enqueued on `stream`; the inputs are not modified
 *                            and may be freed once the stream has run it.
 *   moe_expert_ffn_packed    moe_expert_ffn with `packed` in place of the six
 *                            weight pointers (bf16 payload only).
 *   moe_forward_packed       moe_forward likewise; cfg->payload must be bf16
 *                            (MOE_ERR_UNSUPPORTED_SHAPE otherwise).
 * The packed buffer depends on E, d, d_ff, n_shared and d_ff_shared only.
 */
MOE_API size_t moe_packed_weights_size(const moe_config *cfg);
MOE_API moe_status moe_pack_weights(const moe_config *cfg, const void *w_gate, const void *w_up,
                                    const void *w_down, const void *ws_gate, const void *ws_up,
                                    const void *ws_down, void *packed, void *stream);
MOE_API moe_status moe_expert_ffn_packed(const moe_config *cfg, const void *x_perm,
                                         const int32_t *offsets, const void *packed, void *y_perm,
                                         const void *x, void *y_shared, void *ws, size_t ws_bytes,
                                         void *stream);
MOE_API moe_status moe_forward_packed(const moe_config *cfg, const void *x, const float *router_w,
                                      const float *logit_offset, const float *bias,
                                      const int64_t *token_ids, const void *packed, void *out,
                                      int32_t *topk_idx, float *topk_w, int32_t *counts,
                                      int32_t *offsets, int32_t *send, int32_t *send_tok,
                                      void *ws, size_t ws_bytes, void *stream);

/*
 * Expert parallelism over `world` ranks, one GPU each (the dispatch and
 * combine all-to-alls of "moe-node-limited-routing", "Why all to all
 * dominates MoE step time", and the expert placement of deepnotes "The real
 * cluster, and the mesh DeepSeek actually disclosed").  Rank r owns experts
 * [r*E/world, (r+1)*E/world) and routes its own T tokens (cfg is the
 * per-rank configuration, cfg->T its token count; E % world == 0, world <= 64,
 * world * T * K < 2^31; otherwise MOE_ERR_UNSUPPORTED_SHAPE).
 * A rank's step: moe_route and moe_dispatch(x_perm = NULL) on its tokens; an
 * all-gather of the dispatch counts into counts_all [world, E] (the caller's
 * collective); moe_ep_plan; moe_ep_dispatch; a barrier (every rank's stores
 * done); moe_ep_expert_ffn; a barrier; moe_ep_combine.
 * Receive buffers: recv_x and recv_y of every rank hold world * T * K rows of
 * d bf16 (every copy of every rank could go to one owner, and no copy is
 * dropped).  Per-rank footprint of the exchange, in bytes:
 *   recv_x + recv_y          2 * (2 * world * T * K * d)
 *   moe_ep_workspace_size    about 2 * world * T * K * (2 d + d_ff) more
 *                            (the expert FFN's x_perm / h / y_perm slots)
 * so it grows linearly with world: at V3 sizes (T = 8192 per rank, K = 8,
 * d = 7168, d_ff = 2048) and world = 8, recv_x and recv_y are 7.5 GB each.
 * The kernels reach
 * the other ranks' buffers through device arrays of `world` device pointers
 * (this rank's own and peers' buffers mapped with moe_ipc_open_handle), with
 * plain peer stores (dispatch) and peer loads (combine): the transfer is the
 * gather / reduce itself, with no staging copy.
 * Row layout at owner o: its experts in order; inside an expert's segment the
 * copies of rank 0, then rank 1, ..., each in its token order.  With a batch
 * split into equal contiguous rank chunks this is the single-GPU x_perm
 * restricted to o's experts, so the layer equals moe_forward bit for bit.
 */
/* Workspace bytes for moe_ep_expert_ffn: moe_workspace_size of the global
 * batch (cfg with T * world); 0 if unsupported. */
MOE_API size_t moe_ep_workspace_size(const moe_config *cfg, int32_t world);

/* From counts_all [world, E] int32 (counts_all[r][e] = copies of rank r's
 * tokens to expert e): base [E] int32 out, the first row of this rank's copies
 * for expert e in owner(e)'s receive buffer; local_offsets [E/world + 1]
 * int32 out, the segment starts of this rank's experts in its own receive
 * buffer (the last entry = rows received). */
MOE_API moe_status moe_ep_plan(const moe_config *cfg, int32_t world, int32_t rank,
                               const int32_t *counts_all, int32_t *base, int32_t *local_offsets,
                               void *stream);

/* Dispatch fused with its all-to-all: x [T, d] bf16, topk_idx [T, K],
 * offsets [E+1] and inv_perm [T, K] from this rank's moe_dispatch, base from
 * moe_ep_plan; recv_x: device array of `world` device pointers to the ranks'
 * receive buffers.  Copy (t, j) of expert e lands in row base[e] + (inv_perm
 * [t][j] - offsets[e]) of recv_x[e / (E/world)].  Rows outside the buffer are
 * skipped and flagged MOE_ERR_DEVICE_FAULT in *device_status (may be NULL). */
MOE_API moe_status moe_ep_dispatch(const moe_config *cfg, int32_t world, const void *x,
                                   const int32_t *topk_idx, const int32_t *offsets,
                                   const int32_t *inv_perm, const int32_t *base,
                                   void *const *recv_x, int32_t *device_status, void *stream);

/* The expert FFN of this rank: its E/world experts (w_gate / w_up
 * [E/world, d_ff, d], w_down [E/world, d, d_ff]) over recv_x with
 * local_offsets, into recv_y (same capacity); the shared experts on this
 * rank's x [T, d] into y_shared [T, d].  ws: moe_ep_workspace_size bytes. */
MOE_API moe_status moe_ep_expert_ffn(const moe_config *cfg, int32_t world, int32_t rank,
                                     const void *recv_x, const int32_t *local_offsets,
                                     const void *w_gate, const void *w_up, const void *w_down,
                                     void *recv_y, const void *x, const void *ws_gate,
                                     const void *ws_up, const void *ws_down, void *y_shared,
                                     void *ws, size_t ws_bytes, void *stream);

/* FP8 payload variant of moe_ep_dispatch (moe_dispatch_fp8's format, d % 128
 * == 0): each copy travels as d E4M3 codes into recv_q[owner] ([world*T*K, d]
 * bytes) and one fp32 scale per 128-channel block into recv_scale[owner]
 * ([world*T*K, d/128]), both device arrays of `world` device pointers.  The
 * quantization is moe_dispatch_fp8's, done once per token at the source: the
 * codes equal those moe_dispatch_fp8 writes for the same token.  Halves the
 * bytes of the dispatch exchange ("DeepSeek 8.7 -- communication", section 4). */
MOE_API moe_status moe_ep_dispatch_fp8(const moe_config *cfg, int32_t world, const void *x,
                                       const int32_t *topk_idx, const int32_t *offsets,
                                       const int32_t *inv_perm, const int32_t *base,
                                       void *const *recv_q, void *const *recv_scale,
                                       int32_t *device_status, void *stream);

/* moe_ep_expert_ffn over the FP8 payload: recv_q / recv_scale of this rank
 * (moe_expert_ffn_fp8's operands); x [T, d] is required (shared experts and
 * the GEMM's operand map). */
MOE_API moe_status moe_ep_expert_ffn_fp8(const moe_config *cfg, int32_t world, int32_t rank,
                                         const uint8_t *recv_q, const float *recv_scale,
                                         const int32_t *local_offsets, const void *w_gate,
                                         const void *w_up, const void *w_down, void *recv_y,
                                         const void *x, const void *ws_gate, const void *ws_up,
                                         const void *ws_down, void *y_shared, void *ws,
                                         size_t ws_bytes, void *stream);

/* Deduplicated dispatch: with node-limited routing a token's row needs to
 * reach each owner holding one of its experts once ("moe-node-limited-
 * routing": the node limit bounds the nodes a token's activations reach; the
 * single-GPU send_tok matrix counts these pairs), then fans out to its
 * experts there.  Steps of a rank, replacing moe_ep_dispatch:
 *   moe_ep_token_plan  (local)  tok_slot [T, world] int32 out: position of
 *                      token t among this rank's tokens with an expert at
 *                      owner o (token order), -1 if none; tok_counts [world]
 *                      int32 out: this rank's tokens per owner
 *   (caller) all-gather tok_counts into tok_counts_all [world, world]
 *   moe_ep_token_base  tok_base [world + 1] int32 out: this rank's first row
 *                      in each owner's token buffer (sum over lower ranks);
 *                      tok_base[world] = token rows this rank receives
 *   moe_ep_dispatch_dedup  one store of each token row per owner into
 *                      recv_tok[o] (rows: rank 0's tokens, then rank 1's,
 *                      each in token order; capacity world * T rows of d
 *                      bf16) and, per copy (t, j), the 4-byte token row into
 *                      recv_idx[o][copy row] (capacity world * T * K int32);
 *                      recv_tok / recv_idx: device arrays of `world` pointers
 *   barrier, then at every owner: moe_ep_fanout  recv_x[r] = recv_tok
 *                      [recv_idx[r]] for its local_offsets[E/world] rows
 * recv_x then holds exactly what moe_ep_dispatch writes, so the rest of the
 * step (moe_ep_expert_ffn, moe_ep_combine) is unchanged and the layer's
 * output is the same bit for bit.  Rows or slots outside the buffers are
 * skipped and flagged MOE_ERR_DEVICE_FAULT in *device_status (may be NULL). */
MOE_API moe_status moe_ep_token_plan(const moe_config *cfg, int32_t world,
                                     const int32_t *topk_idx, int32_t *tok_slot,
                                     int32_t *tok_counts, void *stream);
MOE_API moe_status moe_ep_token_base(const moe_config *cfg, int32_t world, int32_t rank,
                                     const int32_t *tok_counts_all, int32_t *tok_base,
                                     void *stream);
MOE_API moe_status moe_ep_dispatch_dedup(const moe_config *cfg, int32_t world, const void *x,
                                         const int32_t *topk_idx, const int32_t *offsets,
                                         const int32_t *inv_perm, const int32_t *base,
                                         const int32_t *tok_slot, const int32_t *tok_base,
                                         void *const *recv_tok, int32_t *const *recv_idx,
                                         int32_t *device_status, void *stream);
MOE_API moe_status moe_ep_fanout(const moe_config *cfg, int32_t world, const void *recv_tok,
                                 const int32_t *recv_idx, const int32_t *local_offsets,
                                 void *recv_x, int32_t *device_status, void *stream);

/* moe_ep_dispatch_dedup and moe_ep_combine_plan (below) in one launch: the
 * same recv_tok / recv_idx and the same list / lw / lcnt, bit for bit.  The
 * lane that writes copy (t, j)'s fan-out index already holds its owner, token
 * row and copy row, which are what the combine's list entry needs, so the
 * lists cost no second pass over the copies.  Arguments as in the two calls;
 * all pointers are required when T > 0; errors as moe_ep_dispatch_dedup. */
MOE_API moe_status moe_ep_dispatch_dedup_plan(const moe_config *cfg, int32_t world,
                                              const void *x, const int32_t *topk_idx,
                                              const float *topk_w, const int32_t *offsets,
                                              const int32_t *inv_perm, const int32_t *base,
                                              const int32_t *tok_slot, const int32_t *tok_base,
                                              void *const *recv_tok, int32_t *const *recv_idx,
                                              int32_t *const *list, float *const *lw,
                                              int32_t *const *lcnt, int32_t *device_status,
                                              void *stream);

/* The deduplicated dispatch of the FP8 payload (d % 128 == 0): codes and
 * scales of a token go once to each owner, recv_tq[o] ([world*T, d] bytes)
 * and recv_ts[o] ([world*T, d/128] fp32), quantized once at the source as by
 * moe_dispatch_fp8, plus the fan-out index per copy into recv_idx[o];
 * moe_ep_fanout_fp8 then builds the owner's recv_q / recv_scale (the operands
 * of moe_ep_expert_ffn_fp8), byte for byte what moe_ep_dispatch_fp8 writes. */
MOE_API moe_status moe_ep_dispatch_dedup_fp8(const moe_config *cfg, int32_t world, const void *x,
                                             const int32_t *topk_idx, const int32_t *offsets,
                                             const int32_t *inv_perm, const int32_t *base,
                                             const int32_t *tok_slot, const int32_t *tok_base,
                                             void *const *recv_tq, void *const *recv_ts,
                                             int32_t *const *recv_idx, int32_t *device_status,
                                             void *stream);
MOE_API moe_status moe_ep_fanout_fp8(const moe_config *cfg, int32_t world, const uint8_t *recv_tq,
                                     const float *recv_ts, const int32_t *recv_idx,
                                     const int32_t *local_offsets, uint8_t *recv_q,
                                     float *recv_scale, int32_t *device_status, void *stream);

/* Deduplicated combine (with the deduplicated dispatch): each owner sums the
 * gate-weighted outputs of its copies of a token into one bf16 partial row,
 * and only that row crosses back.
 *   moe_ep_combine_plan  (source, before the dispatch barrier) for every token
 *                      t and owner o holding cnt of its copies: the copy rows
 *                      and gates in slot order into list[o] / lw[o]
 *                      ([world*T*K] int32 / fp32, entry trow*K + k) and cnt
 *                      into lcnt[o] ([world*T] int32), trow = t's token row
 *                      at o; list / lw / lcnt: device arrays of `world`
 *                      pointers
 *   moe_ep_precombine    (owner, after its expert FFN) partial [world*T, d]
 *                      bf16: partial[trow] = bf16(sum_k lw[k] * recv_y
 *                      [list[k]]), fp32 multiply-adds in slot order, for its
 *                      tok_base[world] token rows
 *   barrier, then moe_ep_combine_dedup (source) out[t] = bf16(y_shared[t] +
 *                      the partial rows of t's owners in the order of their
 *                      first slots, fp32), partial: device array of `world`
 *                      pointers
 * The partial sums are rounded to bf16 once more than in moe_ep_combine, so
 * the output equals the single-GPU layer within its tolerances, not bit for
 * bit. */
MOE_API moe_status moe_ep_combine_plan(const moe_config *cfg, int32_t world,
                                       const int32_t *topk_idx, const float *topk_w,
                                       const int32_t *offsets, const int32_t *inv_perm,
                                       const int32_t *base, const int32_t *tok_slot,
                                       const int32_t *tok_base, int32_t *const *list,
                                       float *const *lw, int32_t *const *lcnt,
                                       int32_t *device_status, void *stream);
MOE_API moe_status moe_ep_precombine(const moe_config *cfg, int32_t world, const void *recv_y,
                                     const int32_t *list, const float *lw, const int32_t *lcnt,
                                     const int32_t *tok_base, void *partial,
                                     int32_t *device_status, void *stream);
MOE_API moe_status moe_ep_combine_dedup(const moe_config *cfg, int32_t world,
                                        const int32_t *topk_idx, const int32_t *tok_slot,
                                        const int32_t *tok_base, const void *const *partial,
                                        const void *y_shared, void *out, int32_t *device_status,
                                        void *stream);

/* Combine fused with its all-to-all: out[t] = y_shared[t] + sum_j topk_w[t][j]
 * * (row of copy (t, j) in recv_y[owner]), fp32 multiply-adds in slot order,
 * bf16 out [T, d].  recv_y: device array of `world` device pointers. */
MOE_API moe_status moe_ep_combine(const moe_config *cfg, int32_t world, const int32_t *topk_idx,
                                  const float *topk_w, const int32_t *offsets,
                                  const int32_t *inv_perm, const int32_t *base,
                                  const void *const *recv_y, const void *y_shared, void *out,
                                  int32_t *device_status, void *stream);

/* CUDA IPC of a device buffer for the peer pointer tables.  get_handle writes
 * MOE_IPC_HANDLE_BYTES opaque bytes (the CUDA IPC handle of the allocation
 * that holds dev_ptr, and dev_ptr's offset inside it: a caching allocator may
 * place the buffer inside a larger allocation) to send to the other ranks.
 * open_handle, in another process, maps that allocation into this GPU's
 * address space (peer access enabled) and returns the buffer's address in
 * it; close_handle takes that address and unmaps the allocation
 * (MOE_ERR_INVALID_ARG for an address open_handle did not return).  A process
 * cannot open its own handles. */
#define MOE_IPC_HANDLE_BYTES 72
MOE_API moe_status moe_ipc_get_handle(const void *dev_ptr, void *handle);
MOE_API moe_status moe_ipc_open_handle(const void *handle, void **dev_ptr);
MOE_API moe_status moe_ipc_close_handle(void *dev_ptr);

/*
 * Self-test of the bounded device waits: launches one kernel that waits on
 * an mbarrier no thread ever arrives on, with a limit of `timeout_ns`
 * nanoseconds (1e3 .. 1e10).  The kernel must give up, record
 * MOE_ERR_DEVICE_TIMEOUT in the status word and return; the context stays
 * usable.  Uses only the status word of `ws` (>= 256 bytes).
 */
MOE_API moe_status moe_selftest_bounded_wait(int64_t timeout_ns, void *ws, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
