/*
 * hymba.h -- C ABI of the B200 (sm_100a) library for the forward (prefill) pass
 * of Hymba's fused hybrid-head layer.
 *
 * What the layer computes (sources: the blog.outta.ai review of arXiv
 * 2411.13676 "Hymba: A Hybrid-head Architecture for Small Language Models",
 * section "Design formulation"; the metaphor-xennon page, sections
 * "混合头模块" and "PyTorch伪代码"; the networkstorageforum summary, section
 * "Key Components of Hymba"):
 *
 *   X~      = [meta; X]                                  (meta tokens prepended)
 *   [Q K V X_ssm G_raw] = X~ W_in^T                      (one fused in_proj)
 *   Y_attn  = softmax(Q K^T / sqrt(dh) + mask) V         (causal / SWA, meta always visible, GQA)
 *   [dt_low B C] = X_ssm W_x^T,  dt = softplus(dt_low W_dt^T + b_dt),  A = -exp(A_log)
 *   h_t     = exp(A dt_t) h_{t-1} + dt_t B_t x_t,  y_t = C_t . h_t     (selective scan)
 *   Y_ssm   = SiLU(G_raw) * y
 *   out     = W_out [ beta1 * rms(Y_attn) || beta2 * rms(Y_ssm) ]
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; row-major;
 *     the library allocates no memory.  Calls are asynchronous on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - Per device the library keeps a few handles it makes on first use (kernel
 *     attributes, the second streams of hymba_layer_fwd, the address of the
 *     hymba_layer_fwd_noalloc block); none of them survives a reset of the device or of
 *     its primary context, so no call may follow cudaDeviceReset in the same process.
 *   - "dtype" tensors (activations and projection weights) are bf16 when
 *     cfg.dtype == HYMBA_BF16 (fp32 accumulation, fp32 scan state) and fp32
 *     when cfg.dtype == HYMBA_F32.  a_log, b_dt, beta1, beta2 are always fp32.
 *   - Arguments are validated before anything is launched; a bad argument
 *     returns an error status with no side effect.  HYMBA_ERR_CUDA is returned
 *     only for a failed launch or CUDA call.
 *   - Every kernel bounds its internal waits.  A wait that runs out records
 *     HYMBA_ERR_TIMEOUT in the status word at the start of the workspace and
 *     the kernel returns early; hymba_workspace_status() reads it.
 */
#ifndef HYMBA_H_
#define HYMBA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HYMBA_API __attribute__((visibility("default")))
#else
#define HYMBA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HYMBA_OK = 0,
  HYMBA_ERR_INVALID_ARG = 1,  /* null pointer, negative or inconsistent size */
  HYMBA_ERR_UNSUPPORTED = 2,  /* well-formed but outside what the kernels implement */
  HYMBA_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than hymba_*workspace_size() */
  HYMBA_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  HYMBA_ERR_TIMEOUT = 5       /* a kernel's bounded wait ran out (reported by hymba_workspace_status) */
} hymba_status_t;

typedef enum { HYMBA_F32 = 0, HYMBA_BF16 = 1 } hymba_dtype_t;

/* Cross-layer KV sharing ("Cross-layer KV sharing" in the blog.outta.ai
 * review: two consecutive layers share one KV cache).  The even layer of a
 * pair produces K/V, the odd one consumes it and has no W_K / W_V rows. */
typedef enum {
  HYMBA_KV_OWN = 0,      /* compute K/V for this layer only (kept in the workspace) */
  HYMBA_KV_PRODUCE = 1,  /* compute K/V and write them to kv_out for the partner layer */
  HYMBA_KV_CONSUME = 2   /* no K/V projection: read the partner's K/V from kv_in */
} hymba_kv_mode_t;

typedef struct {
  int batch;        /* B >= 1 */
  int seq_len;      /* L >= 1: user tokens per sequence */
  int n_meta;       /* M >= 0: meta tokens; T = L + M rows per sequence */
  int d_model;      /* d */
  int n_q_heads;    /* Hq */
  int n_kv_heads;   /* Hkv, divides Hq (GQA) */
  int head_dim;     /* dh: 128 for bf16; <= 128 for fp32 */
  int window;       /* W: -1 = global causal; >= 0: query i sees key j iff j <= i and
                       (i - j <= W or j < M) -- meta tokens always visible */
  int d_inner;      /* Di: SSM channels */
  int d_state;      /* N: 16, 32, 64, 128 or 256 */
  int n_ssm_heads;  /* recorded only: the per-channel scan does not depend on it */
  int dt_rank;      /* R: width of dt_low */
  int a_per_state;  /* 0: A_log [Di] (one decay per channel); 1: A_log [Di, N] (one per channel and state) */
  int kv_mode;      /* hymba_kv_mode_t */
  int ffn_dim;      /* F: SwiGLU FFN width for hymba_stack_fwd; 0 = no FFN */
  float rms_eps;    /* RMSNorm epsilon (1e-6) */
  hymba_dtype_t dtype;
  /* Options beyond the pages' formula (0 = off; the five workloads use none):           */
  int conv_width;   /* 1..4: Mamba's causal depthwise conv + SiLU on X_ssm before x_proj
                       and the scan (weights w_conv, b_conv); prefill/decode and the
                       meta-prefix calls return HYMBA_ERR_UNSUPPORTED with it */
  int norm_group;   /* 64, 128 or 256: the branch norm per group of this many features
                       (per head); 0 = over each branch's full width */
  int fusion;       /* 0: out = W_out,a(b1 n(Y_a)) + W_out,s(b2 n(Y_s)); 1: difference, the SSM
                       branch subtracted (the intra-layer hybrid study, gist.science page) */
} hymba_cfg_t;

/* Weights of one layer; device pointers, nn.Linear layout [out_features, in_features]. */
typedef struct {
  const void* w_in;       /* [Hq*dh + 2*Hkv*dh + 2*Di, d] rows W_Q, W_K, W_V, W_SSM, W_G
                             (a HYMBA_KV_CONSUME layer has no W_K, W_V rows) */
  const void* w_x;        /* [R + 2N, Di]   rows dt_low, B, C */
  const void* w_dt;       /* [Di, R] */
  const void* w_out;      /* [d, Hq*dh + Di] */
  const float* a_log;     /* [Di]   A = -exp(A_log) */
  const float* b_dt;      /* [Di] */
  const float* beta1;     /* [Hq*dh] */
  const float* beta2;     /* [Di] */
  const void* w_gate_up;  /* [2F, d] gate rows then up rows (stack with ffn_dim > 0), else NULL */
  const void* w_down;     /* [d, F] (stack with ffn_dim > 0), else NULL */
  const float* norm1;     /* [d] fp32 gain of the block's pre-norm before the mixer (stack only);
                             NULL = unit gain; ignored by the single-layer entry points */
  const float* norm2;     /* [d] fp32 gain of the pre-norm before the FFN (stack only); NULL = unit gain */
  const void* w_conv;     /* [Di, conv_width] dtype: the causal conv taps (tap conv_width-1 = current row) */
  const float* b_conv;    /* [Di] fp32 conv bias (required with conv_width) */
  const float* d_skip;    /* [Di] fp32: Mamba's D, Y_ssm = gate * (y + D x); NULL = no skip */
} hymba_weights_t;

/* Human-readable name of a status code (static string). */
HYMBA_API const char* hymba_status_string(hymba_status_t s);

/* Workspace bytes needed by hymba_layer_fwd for `cfg` (0 if cfg is invalid). */
HYMBA_API size_t hymba_workspace_size(const hymba_cfg_t* cfg);

/* Workspace bytes needed by hymba_stack_fwd for `n_layers` configs (0 if invalid). */
HYMBA_API size_t hymba_stack_workspace_size(const hymba_cfg_t* cfgs, int n_layers);

/*
 * One hybrid-head layer, forward (prefill): the fused hybrid-head module of the
 * blog.outta.ai review, section "Design formulation" -- X~ = [meta; X], the one input
 * projection W_in_proj = [W_Q, W_K, W_V, W_SSM, W_G], attention heads and SSM heads in
 * parallel (the SSM head's mixing matrix alpha_ij = C_i (prod_{k=j+1..i} exp(A dt_k)) B_j dt_j,
 * gated by G), each branch normalised and scaled by beta1 / beta2, summed through W_out
 * ("total fusion formulation"); sliding-window attention with the meta tokens always
 * visible ("Combine global and local attention", "Meta Tokens"); cross-layer KV sharing
 * through kv_out / kv_in ("Cross-layer KV sharing").
 *   x       [B, L, d] dtype when meta != NULL; [B, T, d] (rows already X~) when meta == NULL
 *   meta    [M, d] dtype, the learnable meta tokens shared by the batch, or NULL
 *   kv_in   [2, B, T, Hkv*dh] dtype (K then V, token-major, head h at columns
 *           [h*dh, (h+1)*dh)) -- required iff kv_mode == HYMBA_KV_CONSUME
 *   kv_out  same layout -- required iff kv_mode == HYMBA_KV_PRODUCE
 *   out     [B, T, d] dtype; meta rows are kept so the next layer sees [meta; X] state
 *   workspace >= hymba_workspace_size(cfg) bytes, 256-byte aligned; its first 256
 *           bytes hold the status word (reset by this call)
 * Streams: all work is ordered on `stream`.  The attention heads run on a second,
 * non-blocking stream of the library's (forked from `stream` after the input projection
 * with an event and joined back before the branch norm), so the call behaves as one
 * stream-ordered operation.  There is one such second stream (and its two events) per
 * host thread, device and stream priority, made on that thread's first call with the
 * caller stream's priority: calls from different threads never share one; calls one
 * thread makes on several streams do (their attention launches are then ordered among
 * themselves).  The call can be captured into a CUDA graph once the calling thread has
 * made one call on the device outside the capture.
 */
HYMBA_API hymba_status_t hymba_layer_fwd(const void* x, const void* meta, const hymba_weights_t* w,
                               const hymba_cfg_t* cfg, const void* kv_in, void* kv_out,
                               void* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * A stack of hybrid-head blocks ("Key Components of Hymba", networkstorageforum:
 * blocks stacked with SWA and cross-layer KV sharing; the blog.outta.ai review,
 * "Cross-layer KV sharing": two consecutive layers share one KV cache).  For each block i:
 *   h += layer_i(RMSNorm_1(h));  if cfgs[i].ffn_dim: h += W_down(SiLU(W_gate u) * W_up u), u = RMSNorm_2(h)
 * with RMSNorm_k(v) = norm_k * v / sqrt(mean(v^2) + eps) (w[i].norm1 / norm2; NULL = unit
 * gain); h starts as [meta; x].  K/V flow from a HYMBA_KV_PRODUCE block to the
 * HYMBA_KV_CONSUME block after it through the workspace.  x, meta as in hymba_layer_fwd;
 * out [B, T, d] dtype = final h.  All cfgs must share batch, seq_len, n_meta, d_model, dtype.
 * Precision (bf16): the residual stream h is carried in fp32 in the workspace and rounded
 * to bf16 once, into `out`; each pre-norm's output is the bf16 operand of the next GEMM,
 * and the part of it that the bf16 rounding drops is carried into the SSM heads' B and C
 * (x_proj adds it through W_x W_SSM, formed per call in the workspace), because a block's
 * output at early positions depends on those two projections with a large condition number.
 */
HYMBA_API hymba_status_t hymba_stack_fwd(const void* x, const void* meta, const hymba_weights_t* w,
                               const hymba_cfg_t* cfgs, int n_layers, void* out,
                               void* workspace, size_t ws_bytes, void* stream);

/*
 * Whether the layer of `cfg` computes its dt projection ("Design formulation", the
 * SSM head's dt = softplus(dt_low W_dt^T + b_dt)) inside the selective-scan kernel
 * instead of as a separate GEMM: 1 for bf16 with d_state 16, dt_rank 64 and one decay
 * per channel (a_per_state 0), given 16-byte aligned weights; 0 otherwise (also for an
 * invalid cfg).
 * With 1, stage 2 of hymba_layer_fwd_events launches nothing and its work is part of
 * stage 4.
 */
HYMBA_API int hymba_layer_fuses_dt_proj(const hymba_cfg_t* cfg);

/*
 * hymba_layer_fwd with stage timing (tracing hook).  `events` holds 8 cudaEvent_t
 * (created by the caller, passed as void*): events[i] is recorded on `stream`
 * right before stage i and events[7] after the last one.  Stages:
 * 0 in_proj, 1 x_proj, 2 dt_proj, 3 attention, 4 selective scan, 5 branch
 * norm, 6 out_proj.  events == NULL behaves exactly like hymba_layer_fwd; a NULL
 * entry in a non-NULL `events` returns HYMBA_ERR_INVALID_ARG before any launch.
 */
HYMBA_API hymba_status_t hymba_layer_fwd_events(const void* x, const void* meta, const hymba_weights_t* w,
                               const hymba_cfg_t* cfg, const void* kv_in, void* kv_out,
                               void* out, void* workspace, size_t ws_bytes, void* stream,
                               void* const* events);

/*
 * hymba_layer_fwd without a caller-provided workspace.  The paper has no
 * counterpart to this entry point: it exists for callers that cannot allocate
 * device memory when they run the layer -- code inside a host framework that owns
 * every device allocation (a plugin or custom-op execute step that must not call
 * cudaMalloc), or latency-critical paths where cudaMalloc/cudaFree would
 * synchronise the device.  Such a caller passes only inputs and outputs.
 *
 * Scratch: the layer's intermediates live in one block of HYMBA_NOALLOC_SCRATCH_BYTES
 * bytes that the library reserves statically on every GPU that loads it; the
 * block is held until the process exits.  Nothing is allocated by this call (no
 * cudaMalloc, cudaFree or allocating library routine).
 *   - A cfg whose hymba_workspace_size(cfg) exceeds HYMBA_NOALLOC_SCRATCH_BYTES
 *     returns HYMBA_ERR_WORKSPACE before anything runs; use hymba_layer_fwd there.
 *   - The first call on a device looks up the block's device address (once per
 *     device, with that device current) and creates the layer's second stream (see
 *     hymba_layer_fwd).  Make that first call before any stream capture on the device.
 *   - Every call on a device shares the block, which keeps the last call's
 *     contents; the call clears its status word and overwrites every intermediate
 *     before reading it.  Calls whose execution overlaps on the GPU (different
 *     streams, or several host threads) race on the block: serialise them.
 *   - A kernel wait that runs out is recorded in the block's status word, which
 *     the caller cannot read; callers that need HYMBA_ERR_TIMEOUT reports use
 *     hymba_layer_fwd with their own workspace.
 * Arguments, layouts, validation and results are those of hymba_layer_fwd.
 */
#define HYMBA_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB per GPU */
HYMBA_API hymba_status_t hymba_layer_fwd_noalloc(const void* x, const void* meta, const hymba_weights_t* w,
                               const hymba_cfg_t* cfg, const void* kv_in, void* kv_out,
                               void* out, void* stream);

/* Synchronises `stream`, reads and clears the status word at the start of
 * `workspace`: HYMBA_OK, or HYMBA_ERR_TIMEOUT if a kernel's bounded wait ran out. */
HYMBA_API hymba_status_t hymba_workspace_status(void* workspace, void* stream);

/* ---------------- generation: prefill with state, then one token per step ----------------
 * The attention heads keep a K/V cache that grows with the sequence; the SSM heads keep a
 * fixed-size state (the blog.outta.ai review, "Efficiency and KV cache optimization").
 * A KV-sharing pair keeps one cache (the review, "Cross-layer KV sharing"): the producer's.
 *
 * Layouts (dtype unless noted):
 *   kv_cache   [2, B, cache_rows, Hkv*dh]: K then V; sequence b's row t at (b*cache_rows + t)
 *   ssm_state  [B, Di, N] fp32: the state after the last row processed
 * Workspace for both calls: hymba_decode_workspace_size(cfg) bytes, 256-byte aligned, its
 * first 256 bytes the status word.  Both calls are asynchronous on `stream`; the head_dim
 * must be a multiple of 32, at most 8 query heads per KV head, d_state a multiple of 8.
 */
HYMBA_API size_t hymba_decode_workspace_size(const hymba_cfg_t* cfg);

/*
 * hymba_layer_fwd over the T = L + M prompt rows (cfg.seq_len = L) that also leaves what
 * the next token needs: rows [0, T) of each sequence's K/V in kv_cache (cache_rows >= T;
 * for a HYMBA_KV_CONSUME layer kv_cache is the producer's cache, read only) and the SSM
 * state after row T - 1 in ssm_state.  x, meta, out as in hymba_layer_fwd (meta NULL: x
 * already holds the T rows of X~, e.g. the previous layer's output).
 */
HYMBA_API hymba_status_t hymba_layer_prefill(const void* x, const void* meta, const hymba_weights_t* w,
                                   const hymba_cfg_t* cfg, void* kv_cache, int cache_rows,
                                   float* ssm_state, void* out, void* workspace, size_t ws_bytes,
                                   void* stream);

/*
 * One new token per sequence at row `pos` (rows [0, pos) are in the cache, meta rows
 * included; 0 <= pos < cache_rows): x_t [B, d] -> out_t [B, d].  The same definitions as
 * hymba_layer_fwd applied to row pos: its query attends over the cached rows it sees
 * (causal, window W, meta rows always visible) and its own; the SSM heads advance one
 * step, h <- exp(A dt) h + dt x B, y = C . h (the review, "Design formulation").  A layer
 * with its own K/V (HYMBA_KV_OWN / HYMBA_KV_PRODUCE) writes the token's K, V into row pos
 * of kv_cache first; a HYMBA_KV_CONSUME layer reads the producer's cache, which must
 * already hold row pos.  ssm_state is read and updated in place.  cfg.seq_len is not used.
 */
HYMBA_API hymba_status_t hymba_layer_decode(const void* x_t, const hymba_weights_t* w, const hymba_cfg_t* cfg,
                                  void* kv_cache, int cache_rows, int pos, float* ssm_state,
                                  void* out_t, void* workspace, size_t ws_bytes, void* stream);

/* ---------------- meta-prefix precompute ----------------
 * The meta tokens are the same learned rows in front of every sequence (the review,
 * "Meta Tokens"; the networkstorageforum page, "Key Components of Hymba": a learned
 * initialisation of the caches).  Under the causal mask a meta row sees only meta rows,
 * so everything the layer computes for them -- their K/V, the SSM state after them, their
 * output rows -- is the same for every sequence and every call with the same weights.
 * hymba_meta_prefix computes that once into a record; hymba_layer_fwd_prefixed then runs
 * only the user rows.
 *
 * Record (caller-owned device memory of hymba_meta_prefix_size(cfg) bytes, 256-byte
 * aligned): the M meta rows' outputs [M, d] (dtype), their K then V [2, M, Hkv*dh]
 * (dtype; absent for a HYMBA_KV_CONSUME layer), the SSM state after them [Di, N] fp32.
 */
HYMBA_API size_t hymba_meta_prefix_size(const hymba_cfg_t* cfg);  /* 0 if cfg invalid or n_meta = 0 */

/*
 * Fills `prefix` for the layer of `cfg` (n_meta >= 1; batch and seq_len are not used).
 *   meta_in       [M, d] dtype: the layer's input meta rows -- the meta tokens for the first
 *                 layer, or the previous layer's prefix output rows (the first M rows of the
 *                 record) for a layer that takes another layer's output
 *   kv_prefix_in  the producer's record, for a HYMBA_KV_CONSUME layer; else NULL
 *   workspace     >= hymba_workspace_size(cfg) bytes (the full layer's; 256-byte aligned)
 */
HYMBA_API hymba_status_t hymba_meta_prefix(const void* meta_in, const hymba_weights_t* w, const hymba_cfg_t* cfg,
                                 const void* kv_prefix_in, void* prefix, void* workspace, size_t ws_bytes,
                                 void* stream);

/*
 * hymba_layer_fwd with the meta rows taken from a record of hymba_meta_prefix: x holds
 * the user rows only, [B, L, d]; the input projection, attention queries and scan run on
 * rows [M, T) of each sequence (the scan from the record's state), the meta rows' K/V are
 * copied into each sequence's K/V (kv_out for a producing layer), and out [B, T, d]
 * receives the record's meta rows and the computed user rows.  Other arguments as in
 * hymba_layer_fwd (kv_in for a consuming layer: the producer's kv_out of its prefixed call).
 * With d_state 128 the scan of such a call runs on the CUDA cores after a separate dt_proj
 * GEMM, not in the tensor-core scan with the fused dt projection (that kernel, started from
 * a stored state, was seen to write a few wrong rows of its first block intermittently).
 */
HYMBA_API hymba_status_t hymba_layer_fwd_prefixed(const void* x, const void* prefix, const hymba_weights_t* w,
                                        const hymba_cfg_t* cfg, const void* kv_in, void* kv_out, void* out,
                                        void* workspace, size_t ws_bytes, void* stream);

/*
 * Check of the failure-detection path (no counterpart in the pages).  Every kernel of this
 * library bounds its waits on mbarriers; a wait that runs out records HYMBA_ERR_TIMEOUT
 * in the status word and the kernel returns instead of hanging.  This call runs one
 * kernel whose single waiting thread waits on an mbarrier that nothing arrives on, with
 * a limit of limit_us microseconds (1 .. 1000000): the wait runs out, the status word at
 * the start of `workspace` (>= 256 bytes; cleared first) becomes HYMBA_ERR_TIMEOUT, and
 * the kernel returns.  Read it with hymba_workspace_status().
 */
HYMBA_API hymba_status_t hymba_check_wait_timeout(void* workspace, size_t ws_bytes, unsigned limit_us,
                                                  void* stream);

/* ---------------- stage entry points (each one kernel family) ---------------- */

/* C[M, N] = A[M, K] W[N, K]^T (dtype in and out, fp32 accumulation); bf16 runs on the
 * tcgen05 tensor-core GEMM, or for M <= 8 (K a multiple of 8, 16-byte aligned A and W) on
 * the CUDA cores as a stream over W.  workspace: >= 256 bytes (status word). */
HYMBA_API hymba_status_t hymba_gemm(const void* a, const void* w, void* c, int M, int N, int K,
                          hymba_dtype_t dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * Selective scan fused with the output gate ("Design formulation": SSM head
 * alpha_ij and Y_ssm = G . alpha W_SSM X~):
 *   for each sequence b and channel c, from h = 0:
 *     h_t = exp(A_c dt_t) h_{t-1} + dt_t x_t B_t,   y_t = gate_t * (C_t . h_t),   A_c = -exp(a_log[c])
 *   a_per_state = 0: a_log [d_inner];  1: a_log [d_inner, d_state] and the state component n
 *     decays by exp(A_{c,n} dt_t), A_{c,n} = -exp(a_log[c, n]) (the Mamba variant with a
 *     diagonal A per channel)
 *   x, dt, gate [batch*T, d_inner] dtype (dt > 0 already discretised; gate = SiLU(G_raw))
 *   bc   [batch*T, 2*d_state] fp32, B_t then C_t
 *   y    written at y + row*y_ld, dtype
 *   workspace >= 256 bytes (status word)
 */
HYMBA_API hymba_status_t hymba_selective_scan(const void* x, const void* dt, const float* bc,
                                    const void* gate, const float* a_log, void* y, int y_ld,
                                    int batch, int T, int d_inner, int d_state, int a_per_state,
                                    hymba_dtype_t dtype, void* workspace, size_t ws_bytes,
                                    void* stream);

/*
 * The selective scan with the SSM heads' dt projection in front of it: the same scan
 * as hymba_selective_scan with
 *   dt = softplus(dt_low W_dt^T + b_dt)          (Mamba's discretisation step, per row and channel)
 *   dt_low [batch*T, dt_rank] dtype (row stride dt_rank);  w_dt [d_inner, dt_rank] dtype;
 *   b_dt [d_inner] fp32;  one decay rate per channel (a_log [d_inner]).
 * Where a tensor-core kernel takes the configuration (bf16; d_state 16 with dt_rank 64,
 * or d_state 128 with dt_rank a multiple of 8 up to 128; 16-byte aligned operands and
 * row strides) dt is formed block by block inside the scan and never stored; otherwise
 * it is computed into the workspace first.
 * hymba_selective_scan_dtproj_workspace_size gives the bytes needed (for the fused
 * kernels the 256-byte status word, plus for d_state 128 36 KB per sequence and 32 rows
 * for the operands every channel shares: C B^T, B^T and C of each block); HYMBA_ERR_WORKSPACE
 * when ws_bytes is smaller.
 */
HYMBA_API size_t hymba_selective_scan_dtproj_workspace_size(int batch, int T, int d_inner, int d_state,
                                                            int dt_rank, hymba_dtype_t dtype);
HYMBA_API hymba_status_t hymba_selective_scan_dtproj(const void* x, const void* dt_low, const void* w_dt,
                                           const float* b_dt, int dt_rank, const float* bc,
                                           const void* gate, const float* a_log, void* y, int y_ld,
                                           int batch, int T, int d_inner, int d_state,
                                           hymba_dtype_t dtype, void* workspace, size_t ws_bytes,
                                           void* stream);

/*
 * Attention heads ("Design formulation", attention head; "Combine global and local
 * attention"): per sequence and query head h (KV head h / (Hq/Hkv)),
 *   out_i = sum_j softmax_j(q_i . k_j / sqrt(dh)) v_j  over visible j (see hymba_cfg_t.window)
 *   q   [batch*T, Hq*dh] dtype;  kv [2, batch*T, Hkv*dh] dtype (K then V)
 *   out written at out + row*out_ld + h*dh, dtype
 */
HYMBA_API hymba_status_t hymba_attention(const void* q, const void* kv, void* out, int out_ld, int batch,
                               int T, int n_q_heads, int n_kv_heads, int head_dim, int n_meta,
                               int window, hymba_dtype_t dtype, void* workspace,
                               size_t ws_bytes, void* stream);

/*
 * Per-branch RMSNorm and beta scale, in place ("Design formulation", total fusion):
 *   z [rows, w_attn + w_ssm] dtype;  z[:, :w_attn] = beta1 * rms(z[:, :w_attn]),
 *   z[:, w_attn:] = beta2 * rms(z[:, w_attn:]),   rms(v) = v / sqrt(mean(v^2) + eps)
 */
HYMBA_API hymba_status_t hymba_branch_norm(void* z, const float* beta1, const float* beta2, int rows,
                                 int w_attn, int w_ssm, float eps, hymba_dtype_t dtype,
                                 void* stream);

/* y[rows, d] = x / sqrt(mean(x^2) + eps) row-wise (unit gain); x and y may alias. */
HYMBA_API hymba_status_t hymba_rmsnorm(const void* x, void* y, int rows, int d, float eps,
                             hymba_dtype_t dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HYMBA_H_ */
