/*
 * gla.h -- C ABI of the B200 (sm_100a) chunkwise gated linear attention library.
 *
 * The operation (recurrent form; talk summary "Hardware-Efficient Training of Linear
 * Attention Models", sections 4:04 and 7:36; data-dependent gates from the GLA
 * abstract, Yang et al.): per (batch b, head h), with a Dk x Dv matrix state S,
 *
 *     S_t = diag(alpha_t) S_{t-1} + k'_t^T v_t,    o_t = scale * q_t S_t,
 *     alpha_t = exp(g_t),  k'_t = i_t k_t (input gate, optional, else k'_t = k_t),
 *     S_{-1} = h0 (or 0),  hT = S_{L-1}.
 *
 * The readout uses the updated state S_t. The library evaluates it with the chunkwise
 * ("trunk-wise") algorithm of the same talk, section 11:58: the sequence is cut into
 * chunks of C tokens, states are formed only at chunk boundaries with K^T V matrix
 * products, and each chunk's output is the inter-chunk term (q_t decayed) S plus a
 * masked intra-chunk product. Large chunks are tiled inside the chunk (Tiled Flash
 * Linear Attention abstract).
 *
 * Conventions for every entry point:
 *  - Layout BHLD, contiguous: q,k [B,H,L,Dk]; v,o,dO [B,H,L,Dv]; per-key gates
 *    g,dg [B,H,L,Dk]; per-head gates g,dg [B,H,L]; input gate i,di [B,H,L];
 *    states h0,hT,dhT,dh0 [B,H,Dk,Dv] (row = key dim).
 *  - q,k,v,o,dO,dq,dk,dv have the I/O dtype of the problem (GLA_F32 or GLA_BF16);
 *    g, i, h0, hT and all their gradients are always float32. Accumulation is fp32.
 *  - g is the log of the decay (g <= 0 for a decay in (0,1]); the library applies no
 *    activation to it. It must be finite. The tensor-core forward and backward factor each
 *    64-token tile's in-tile decays into exponentials about one reference row, which must stay
 *    inside the fp32 range: a tile whose total log-decay in some key dim is below -70 sets the
 *    device status word, so that gla_check_device_status returns GLA_ERR_RANGE (the results of
 *    that call are then not valid; nothing faults). GLA_PLAN_SIMT evaluates any finite gate
 *    (log-space sub-tiles), and the state-only passes (gla_shard_state, gla_shard_state_grad)
 *    any gate on the tensor cores.
 *  - Every pointer is a DEVICE pointer owned by the caller, 16-byte aligned. The
 *    library allocates nothing; scratch memory is the caller's workspace `ws` of at
 *    least gla_workspace_bytes() bytes (16-byte aligned, contents need not be zeroed).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL means
 *    the legacy default stream). Argument errors are detected on the host before any
 *    launch; launch failures map to GLA_ERR_CUDA. No exception crosses the ABI.
 *    The tensor-core backward runs its state-gradient pass on a second stream of its own
 *    (one per device, created on first use), forked from `stream` by an event after all
 *    work enqueued before the call and joined back by an event before its last kernel, so
 *    the call still orders like a single launch sequence on `stream`.
 *  - Thread safety: concurrent calls are safe when they use distinct workspaces.
 */
#ifndef GLA_B200_H
#define GLA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GLA_API __attribute__((visibility("default")))
#else
#define GLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GLA_OK = 0,
    GLA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, bad enum */
    GLA_ERR_UNSUPPORTED = 2,  /* valid request this build cannot run (shape, plan) */
    GLA_ERR_WORKSPACE = 3,    /* ws_bytes smaller than gla_workspace_bytes() */
    GLA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    GLA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (see below) */
    GLA_ERR_RANGE = 6         /* log-gate decay too strong for the tensor-core plan (see below) */
} gla_status;

typedef enum { GLA_F32 = 0, GLA_BF16 = 1 } gla_dtype;

typedef enum {
    GLA_GATE_NONE = 0,     /* alpha = 1: plain causal linear attention */
    GLA_GATE_PER_KEY = 1,  /* g [B,H,L,Dk]: one log-decay per key dim (GLA) */
    GLA_GATE_PER_HEAD = 2  /* g [B,H,L]: one scalar log-decay per head (mLSTM-style) */
} gla_gate_mode;

typedef enum {
    GLA_PLAN_AUTO = 0,     /* library picks from shape, dtype and SM count */
    GLA_PLAN_SIMT = 1,     /* CUDA-core chunk-parallel kernels: any supported shape,
                              fp32 or bf16 I/O; the only plan for fp32 I/O */
    GLA_PLAN_TC = 2        /* tcgen05/TMEM tensor-core kernels; bf16 I/O only */
} gla_plan;

typedef struct {
    int B, H, L;          /* batch, heads, tokens (L >= 0; L = 0 gives hT = h0) */
    int Dk, Dv;           /* head dims: each one of 64, 128, 256 */
    int chunk;            /* chunk size C: a multiple of 16 in [16, 1024] */
    float scale;          /* output scale (typically Dk^-1/2) */
    gla_dtype io;         /* dtype of q, k, v, o, dO, dq, dk, dv */
    gla_gate_mode gate;
    int plan;             /* a gla_plan value */
} gla_problem;

/* Bytes of caller-provided workspace needed by gla_fwd (for_backward = 0) or gla_bwd
 * (for_backward = 1) for this problem; 0 when the problem is invalid. The size depends
 * only on the problem (sizes, dtype, gate mode, plan), never on the data. */
GLA_API size_t gla_workspace_bytes(const gla_problem* p, int for_backward);

/* Forward pass.
 *   q,k,v  : inputs (I/O dtype);  g: log-decays (NULL iff gate == GLA_GATE_NONE)
 *   igate  : input gate [B,H,L] f32 or NULL;  h0: initial state f32 or NULL (= 0)
 *   o      : output [B,H,L,Dv] (I/O dtype), written completely
 *   hT     : final state f32 or NULL (not written)
 *   ws     : workspace, ws_bytes >= gla_workspace_bytes(p, 0)
 * Errors: GLA_ERR_INVALID_ARG, GLA_ERR_UNSUPPORTED, GLA_ERR_WORKSPACE, GLA_ERR_CUDA. */
GLA_API gla_status gla_fwd(const gla_problem* p, const void* q, const void* k, const void* v,
                   const float* g, const float* igate, const float* h0,
                   void* o, float* hT, void* ws, size_t ws_bytes, void* stream);

/* Backward pass. Recomputes the chunk states from its inputs (it does not need the
 * forward's workspace). Inputs as for gla_fwd plus
 *   dO  : upstream gradient of o (I/O dtype);  dhT: upstream gradient of hT or NULL (= 0)
 * Outputs (written completely):
 *   dq, dk, dv (I/O dtype);  dg (like g, f32; must be NULL iff gate == GLA_GATE_NONE)
 *   di [B,H,L] f32 (non-NULL only with igate);  dh0 f32 or NULL (not written)
 * dg is the reverse cumulative sum over the whole sequence of q*dq - k'*dk' (plus the
 * final-state term sum_e dhT*hT); for GLA_GATE_PER_HEAD it is summed over key dims.
 * Errors as for gla_fwd. */
GLA_API gla_status gla_bwd(const gla_problem* p, const void* q, const void* k, const void* v,
                   const float* g, const float* igate, const float* h0,
                   const void* dO, const float* dhT,
                   void* dq, void* dk, void* dv, float* dg, float* di, float* dh0,
                   void* ws, size_t ws_bytes, void* stream);

/* Saved states: the training pair forward -> backward without recomputation.
 * gla_saved_states_bytes: bytes of the f32 buffer in which gla_fwd_save leaves, for
 *   gla_bwd_saved, the states at the segment boundaries of the backward's tensor-core plan
 *   (layout [B*H][nseg][Dk][Dv], entry 0 unused); 0 when that backward needs none (CUDA-core
 *   plan, one segment) or the problem is invalid.
 * gla_fwd_save: gla_fwd that also writes those states into `saved` (NULL, or a buffer of
 *   gla_saved_states_bytes(p) bytes owned by the caller; ignored when that is 0). They come
 *   from the tensor-core forward: GLA_ERR_UNSUPPORTED if the forward's plan is the CUDA-core
 *   one while the backward needs saved states.
 * gla_bwd_saved: gla_bwd that takes them instead of recomputing (skips one pass over k, v, g
 *   and a scan). `saved` must come from gla_fwd_save with the same problem and the same q, k,
 *   v, g, igate, h0; NULL means recompute (the same as gla_bwd).
 * Other arguments, results and errors as for gla_fwd / gla_bwd. */
GLA_API size_t gla_saved_states_bytes(const gla_problem* p);
GLA_API gla_status gla_fwd_save(const gla_problem* p, const void* q, const void* k, const void* v,
                                const float* g, const float* igate, const float* h0,
                                void* o, float* hT, float* saved, void* ws, size_t ws_bytes, void* stream);
GLA_API gla_status gla_bwd_saved(const gla_problem* p, const void* q, const void* k, const void* v,
                                 const float* g, const float* igate, const float* h0,
                                 const void* dO, const float* dhT, const float* saved,
                                 void* dq, void* dk, void* dv, float* dg, float* di, float* dh0,
                                 void* ws, size_t ws_bytes, void* stream);

/* Recurrent single-token step from a given state (the inference use of the same state):
 *     S <- diag(alpha) S + k'^T v,   o = scale * q S   (alpha = e^g, k' = i k, S updated first),
 * per (b, h), with the state updated in place. p->L must be 1 (one token per (b, h));
 * p->chunk and p->plan are ignored. q,k [B,H,1,Dk]; v,o [B,H,1,Dv] (I/O dtype); g as for
 * gla_fwd with L = 1 ([B,H,1,Dk] or [B,H,1]) or NULL iff gate == GLA_GATE_NONE; igate [B,H,1]
 * or NULL; state [B,H,Dk,Dv] f32, read and overwritten (must not alias the other buffers).
 * The result equals gla_fwd over the one token with h0 = state: o, and hT into state. Needs
 * no workspace; bound by HBM bandwidth (the state is read and written once).
 * Errors: GLA_ERR_INVALID_ARG (null or misaligned pointer, L != 1, bad enum),
 * GLA_ERR_UNSUPPORTED (head dims), GLA_ERR_CUDA. */
GLA_API gla_status gla_decode(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                              const float* igate, float* state, void* o, void* stream);

/* Sequence sharding (one exchange step per pass). A sequence cut into contiguous shards, one per
 * rank, runs as: each rank calls gla_shard_state on its shard; the (state, gamma) pairs of all
 * ranks are all-gathered (rank order); each rank calls gla_state_fold with count = its rank to
 * get its shard's initial state, and gla_fwd on its shard from that state. The outputs are
 * those of one gla_fwd over the whole sequence; the last rank's hT is the sequence's.
 * gla_shard_state: the shard's end state from a zero initial state, state [B,H,Dk,Dv] f32, and
 *   its total log-decay per key dim, gamma [B,H,Dk] f32 (per-head gates: the head's total in
 *   every key slot). p describes the shard (L = its tokens; L = 0 gives zeros). Tensor-core
 *   state pass: bf16 I/O, chunk a multiple of 64; otherwise GLA_ERR_UNSUPPORTED. The pass runs
 *   in as many segments of the shard as fill the GPU, whose (state, log-decay) pairs one small
 *   kernel then folds. ws: at least gla_shard_workspace_bytes(p) bytes (the device status word,
 *   as for gla_fwd, then the segments' pairs), caller-owned device memory. q is not read.
 * gla_state_fold: out = S after S <- h0 (or 0), then for i = 0 .. count-1:
 *   S <- diag(e^{gammas[i]}) S + states[i], with states [count][B,H,Dk,Dv] and gammas
 *   [count][B,H,Dk] f32 as all-gathered; p gives B, H, Dk, Dv. out may not alias the inputs.
 * Errors: GLA_ERR_INVALID_ARG, GLA_ERR_UNSUPPORTED, GLA_ERR_WORKSPACE, GLA_ERR_CUDA. */
GLA_API size_t gla_shard_workspace_bytes(const gla_problem* p);   /* 0 when p is invalid */
GLA_API gla_status gla_shard_state(const gla_problem* p, const void* k, const void* v, const float* g,
                                   const float* igate, float* state, float* gamma, void* ws, size_t ws_bytes,
                                   void* stream);
GLA_API gla_status gla_state_fold(const gla_problem* p, int count, const float* states, const float* gammas,
                                  const float* h0, float* out, void* stream);

/* Sequence-sharded backward (same single exchange step). A shard's state gradient obeys the
 * reverse recurrence dS_{t-1} = diag(alpha_t) dS_t + scale q_t^T dO_t, so the gradient w.r.t.
 * the state at a shard's end is a fold of the LATER shards in reverse order: each rank calls
 * gla_shard_state and gla_shard_state_grad on its shard; the triples (state, state_grad, gamma)
 * of all ranks are all-gathered; rank r folds states 0..r-1 from h0 (its initial state, as in
 * the forward) and state_grads P-1 .. r+1 (reverse order, with their gammas) from dhT (the
 * gradient at its end); then gla_bwd on its shard with those two gives its dq, dk, dv, dg, di,
 * and on rank 0 the sequence's dh0.
 * gla_shard_state_grad: the gradient w.r.t. the state before the shard's first token from the
 *   shard's own outputs alone (a zero gradient at its end), state_grad [B,H,Dk,Dv] f32, and the
 *   same total log-decay as gla_shard_state, gamma [B,H,Dk] f32. q [B,H,L,Dk] and dO
 *   [B,H,L,Dv] bf16, g as for gla_fwd; the input gate does not enter it. p->scale is the output
 *   scale. Same support, workspace and errors as gla_shard_state; L = 0 gives zeros. */
GLA_API gla_status gla_shard_state_grad(const gla_problem* p, const void* q, const void* dO, const float* g,
                                        float* state_grad, float* gamma, void* ws, size_t ws_bytes, void* stream);

/* Chunkwise DeltaNet (delta-rule) forward, after the talk summary "Hardware-Efficient Training of
 * Linear Attention Models", sections 22:36 and 31:16 (writing strength beta_t; one gradient step
 * per token on the key-to-value regression loss; the WY representation for the chunk form):
 *   S_t = (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t,   o_t = scale q_t S_t.
 * p: B, H, L >= 0 with B*H at most 65535; Dk 64 or 128; Dv a multiple of 64 up to 4096;
 *   chunk = 64; scale; io bf16 or f32; gate must be GLA_GATE_NONE (no decay gates); plan is
 *   ignored. The backward accepts exactly the problems the forward accepts.
 * q, k [B,H,L,Dk] and v [B,H,L,Dv] in io dtype; beta [B,H,L] f32; h0 [B,H,Dk,Dv] f32 or NULL
 *   (zero); o [B,H,L,Dv] io dtype (written); hT [B,H,Dk,Dv] f32 or NULL (final state, written).
 *   Keys are used as given (unit-norm keys with beta in [0, 1] keep each transition's
 *   eigenvalues in [1 - beta, 1]). All pointers 16-byte aligned, device memory, owned by the
 *   caller; no workspace. L = 0 copies h0 (or zero) to hT.
 * bf16 I/O runs on the tensor cores (chunk products as tcgen05 MMAs with fp32 accumulation,
 * the chunk's triangular solve in fp32); fp32 I/O on the CUDA cores in fp32. Asynchronous on
 * `stream`. There is no device status word: the tensor-core kernels' waits on their own copies
 * and products are bounded, and one that gave up (a fault elsewhere on the device) leaves the
 * outputs unwritten rather than hanging.
 * Errors: GLA_ERR_INVALID_ARG (null or misaligned pointer, bad enum, a gate mode),
 *   GLA_ERR_UNSUPPORTED (head dims, chunk, B*H), GLA_ERR_CUDA (gla_last_error_detail says
 *   which call failed). */
GLA_API gla_status gla_deltanet_fwd(const gla_problem* p, const void* q, const void* k, const void* v,
                                    const float* beta, const float* h0, void* o, float* hT, void* stream);

/* DeltaNet backward: gradients of sum(dO * o) + sum(dhT * hT) for gla_deltanet_fwd's inputs.
 * The chunk form runs in reverse: dX = scale P^T dO + K dS', dR = T^T dX, dV = diag(beta) dR,
 * dS <- dS' + scale Q^T dO - K^T diag(beta) dR (P = lower(Q K^T), T, X as in the forward, dS'
 * the gradient at the chunk's end), then per chunk dQ, dK, dbeta from those products.
 * Same p and inputs as gla_deltanet_fwd; dO [B,H,L,Dv] io dtype; dhT [B,H,Dk,Dv] f32 or NULL.
 * Outputs (written): dq, dk [B,H,L,Dk] and dv [B,H,L,Dv] io dtype; dbeta [B,H,L] f32; dh0
 * [B,H,Dk,Dv] f32 or NULL. ws: device workspace of gla_deltanet_bwd_workspace_bytes(p) bytes,
 * caller-owned: the chunk start states and end gradients (bf16 for bf16 I/O, fp32 for fp32 I/O)
 * and dR; fp32 I/O also X and per-slice sums. Three launches on `stream` (the forward's state
 * walk, the reverse walk, the per-chunk gradients); bf16 I/O runs them on the tensor cores.
 * Errors: as gla_deltanet_fwd, plus GLA_ERR_WORKSPACE. */
GLA_API size_t gla_deltanet_bwd_workspace_bytes(const gla_problem* p);
GLA_API gla_status gla_deltanet_bwd(const gla_problem* p, const void* q, const void* k, const void* v,
                                    const float* beta, const float* h0, const void* dO, const float* dhT,
                                    void* dq, void* dk, void* dv, float* dbeta, float* dh0, void* ws,
                                    size_t ws_bytes, void* stream);

/* DeltaNet training pair without the backward's state walk.
 * gla_deltanet_saved_bytes: bytes of the buffer in which gla_deltanet_fwd_save leaves the state
 *   entering every 64-token chunk, layout [B*H][ceil(L/64)][Dk][Dv], bf16 for bf16 I/O and f32
 *   for f32 I/O (the values the backward's own state walk would write); 0 for an invalid
 *   problem or L = 0.
 * gla_deltanet_fwd_save: gla_deltanet_fwd that also writes those states into `saved` (NULL, or
 *   a caller-owned device buffer of gla_deltanet_saved_bytes(p) bytes, 16-byte aligned).
 * gla_deltanet_bwd_saved: gla_deltanet_bwd that reads them from `saved` instead of walking the
 *   forward's recurrence again (two launches instead of three). `saved` must come from
 *   gla_deltanet_fwd_save with the same problem and the same q, k, v, beta, h0; NULL means
 *   recompute (the same as gla_deltanet_bwd). The workspace is gla_deltanet_bwd_workspace_bytes.
 * Other arguments, results and errors as for gla_deltanet_fwd / gla_deltanet_bwd. */
GLA_API size_t gla_deltanet_saved_bytes(const gla_problem* p);
GLA_API gla_status gla_deltanet_fwd_save(const gla_problem* p, const void* q, const void* k, const void* v,
                                         const float* beta, const float* h0, void* o, float* hT, void* saved,
                                         void* stream);
GLA_API gla_status gla_deltanet_bwd_saved(const gla_problem* p, const void* q, const void* k, const void* v,
                                          const float* beta, const float* h0, const void* dO, const float* dhT,
                                          const void* saved, void* dq, void* dk, void* dv, float* dbeta,
                                          float* dh0, void* ws, size_t ws_bytes, void* stream);

/* mLSTM cell: matrix memory with an exponential input gate, a normaliser state and a
 * max-stabiliser (named by the Tiled Flash Linear Attention abstract as the xLSTM cell its kernels
 * speed up; the cell is the published xLSTM one). Per (batch, head), with g_t the log forget gate
 * (<= 0) and i~_t the log of the exponential input gate (any finite real), from zero states:
 *     C_t = e^{g_t} C_{t-1} + e^{i~_t} k_t^T v_t,   n_t = e^{g_t} n_{t-1} + e^{i~_t} k_t,
 *     h_t = (scale q_t) C_t / max(|(scale q_t) . n_t|, 1).
 * The stabilised recurrence (running max m_t of the log weights, states kept times e^{-m_t}, bound
 * e^{-m_t}) gives the same h_t; here both sums use the input gate e^{i~ - c}, c the head's largest
 * i~, so no gate exceeds 1. The numerator is a gated linear attention pass with values v; the
 * normaliser n_t (a Dk-vector) is an fp32 recurrence on the CUDA cores, because h divides by
 * |den| and an error proportional to den's terms would be amplified where |den| is near the bound.
 * p: as for gla_fwd with gate = GLA_GATE_PER_HEAD (g [B,H,L] f32 is the log forget gate). plan:
 *   GLA_PLAN_AUTO and GLA_PLAN_SIMT run the numerator on the CUDA cores in fp32 (bf16 inputs are
 *   converted in the workspace, gradients cast back); GLA_PLAN_TC (bf16 I/O) runs it on the tensor
 *   cores in bf16: much faster, with the bf16 pass's error carried into h and, where the
 *   numerator's and normaliser's gradients nearly cancel, amplified in dq and dk.
 *   itil [B,H,L] f32: i~.
 * gla_mlstm_fwd: h [B,H,L,Dv] (I/O dtype, written).
 * gla_mlstm_bwd: gradients of sum(dh * h): dq, dk [B,H,L,Dk], dv [B,H,L,Dv] (I/O dtype), dg and
 *   ditil [B,H,L] f32 (all written). dh [B,H,L,Dv] I/O dtype.
 * ws: caller-owned device workspace of gla_mlstm_workspace_bytes(p, for_backward) bytes (0 when p
 *   is invalid or unsupported); gla_check_device_status(ws, stream) reports both passes.
 * Asynchronous on `stream`: the gated linear attention launches of both passes plus a few small
 * kernels. Errors: as gla_fwd / gla_bwd; GLA_ERR_INVALID_ARG also for another gate mode. */
GLA_API size_t gla_mlstm_workspace_bytes(const gla_problem* p, int for_backward);
GLA_API gla_status gla_mlstm_fwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                                 const float* itil, void* h, void* ws, size_t ws_bytes, void* stream);
GLA_API gla_status gla_mlstm_bwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                                 const float* itil, const void* dh, void* dq, void* dk, void* dv, float* dg,
                                 float* ditil, void* ws, size_t ws_bytes, void* stream);

/* mLSTM training pair without the backward's forward passes.
 * gla_mlstm_saved_bytes: bytes of the caller-owned device buffer in which gla_mlstm_fwd_save
 *   leaves, for gla_mlstm_bwd_saved, the forward's results the backward reads: the input gate and
 *   per-head shift, the numerator and the normaliser term of every token, the normaliser
 *   recurrence's segment decays and start states, and the value pass's saved states
 *   (gla_saved_states_bytes of that pass); 0 for an invalid problem or an empty one.
 * gla_mlstm_fwd_save: gla_mlstm_fwd that keeps those results in `saved` (NULL: in the workspace,
 *   the same as gla_mlstm_fwd).
 * gla_mlstm_bwd_saved: gla_mlstm_bwd that reads them from `saved` instead of running the forward
 *   passes again, and hands the value pass's saved states to gla_bwd_saved. `saved` must come
 *   from gla_mlstm_fwd_save with the same problem (plan included) and the same q, k, v, g, itil;
 *   NULL means recompute (the same as gla_mlstm_bwd). The workspace is
 *   gla_mlstm_workspace_bytes(p, 1) bytes.
 * `saved` 16-byte aligned; other arguments, results and errors as for gla_mlstm_fwd /
 * gla_mlstm_bwd. */
GLA_API size_t gla_mlstm_saved_bytes(const gla_problem* p);
GLA_API gla_status gla_mlstm_fwd_save(const gla_problem* p, const void* q, const void* k, const void* v,
                                      const float* g, const float* itil, void* h, void* saved, void* ws,
                                      size_t ws_bytes, void* stream);
GLA_API gla_status gla_mlstm_bwd_saved(const gla_problem* p, const void* q, const void* k, const void* v,
                                       const float* g, const float* itil, const void* dh, const void* saved,
                                       void* dq, void* dk, void* dv, float* dg, float* ditil, void* ws,
                                       size_t ws_bytes, void* stream);

/* Static description of a status code (never NULL). */
GLA_API const char* gla_status_string(gla_status s);

/* Synchronises `stream`, then reads the device status word kept at the start of the
 * workspace of the last call that used `ws`: GLA_OK; GLA_ERR_TIMEOUT when a bounded
 * device-side wait gave up; GLA_ERR_RANGE when the tensor-core plan met a 64-token tile whose
 * total log-decay in some key dim is below -70 (its in-tile factors e^-b would leave the fp32
 * range, so that call's results are not valid; GLA_PLAN_SIMT evaluates such gates in log-space
 * sub-tiles); GLA_ERR_CUDA if the synchronisation itself failed. */
GLA_API gla_status gla_check_device_status(void* ws, void* stream);

/* Text of the CUDA error behind the calling thread's last GLA_ERR_CUDA (where it happened,
 * the CUDA error name and description); "no error" if there was none. Never NULL. */
GLA_API const char* gla_last_error_detail(void);

/* Library version as 10000*major + 100*minor + patch. */
GLA_API int gla_version(void);

/* How gla_fwd (for_backward = 0) or gla_bwd (1) would run `p`, for measurement and
 * capacity planning: *plan_out = the resolved GLA_PLAN_SIMT or GLA_PLAN_TC; *nseg_out =
 * sequence segments processed in parallel (1 = one pass over the whole sequence);
 * *tiles_out = 64-token tiles per segment (the chunk count for the SIMT plan). Any output
 * pointer may be NULL. Returns the same status that gla_fwd / gla_bwd would return for an
 * invalid or unsupported problem, else GLA_OK. Launches nothing. */
GLA_API gla_status gla_plan_info(const gla_problem* p, int for_backward, int* plan_out, int* nseg_out,
                                 int* tiles_out);

/* Forward pass that allocates nothing, for callers that cannot allocate device memory
 * themselves (for example a host whose device memory is all owned by another allocator
 * under a fixed budget, or code that must not call cudaMalloc because it synchronises the
 * device). The pages describe no such call; it is an addition of this library.
 * Same arguments and results as gla_fwd, without the workspace: the scratch memory of the
 * CUDA-core forward (GLA_PLAN_SIMT, any supported shape, fp32 or bf16 I/O) comes from one
 * array of 16 MiB compiled into the library, which every GPU that loads the library holds
 * until the process exits. The caller still provides inputs and outputs.
 *  - Problems whose scratch exceeds 16 MiB (gla_workspace_bytes of the same problem with
 *    plan GLA_PLAN_SIMT and for_backward = 0) return GLA_ERR_WORKSPACE before any launch.
 *  - The first call on a device looks up that device's address of the array
 *    (cudaGetSymbolAddress with the device current), and so does the first call after the
 *    device's CUDA context was replaced (cudaDeviceReset); make those calls before any
 *    stream capture.
 *  - All calls share the array and it keeps the last call's contents; calls whose work
 *    overlaps on the GPU (other streams, other host threads) race on it.
 *  - The CUDA-core forward has no device-side waits or range checks, so it reports every
 *    failure through the return value (GLA_ERR_CUDA with gla_last_error_detail); there is no
 *    device status word to read for this call.
 *  - No cudaMalloc, cudaFree or allocating library routine is called. */
GLA_API gla_status gla_fwd_static_scratch(const gla_problem* p, const void* q, const void* k, const void* v,
                                          const float* g, const float* igate, const float* h0,
                                          void* o, float* hT, void* stream);

/* Diagnostics of the device-side failure path (not needed for computing): launches one small
 * kernel on `stream` whose bounded mbarrier wait is never completed, so that it gives up after
 * `polls` polls (1 .. 2^20; each poll suspends the thread for at most a system-dependent time)
 * and sets the timeout bit of the device status word in `ws` (at least 256 bytes, 16-byte
 * aligned, device memory owned by the caller), as a timed-out wait inside gla_fwd / gla_bwd
 * does. gla_check_device_status(ws, stream) then returns GLA_ERR_TIMEOUT and the CUDA context
 * stays usable. Nothing faults, traps or hangs. Errors: GLA_ERR_INVALID_ARG (before any
 * launch), GLA_ERR_CUDA. */
GLA_API gla_status gla_debug_wait_timeout(void* ws, unsigned polls, void* stream);

/* Measurement support (not needed for computing).
 * gla_launch_count: number of kernels this process has launched through the library.
 * gla_profiler_enable(1): from now on every kernel launch is bracketed by two CUDA events
 *   recorded on the launching stream (host cost: a few microseconds per launch).
 * gla_profiler_read: synchronises on the recorded events, aggregates them by kernel name
 *   into up to max_kernels entries (name copied into names + i*name_stride, NUL-terminated;
 *   launches[i]; total_ms[i] = summed event time), forgets them, and returns the number of
 *   distinct kernels seen (-1 on a CUDA error). Any output pointer may be NULL.
 * Not meant for concurrent use from several host threads while enabled. */
GLA_API unsigned long long gla_launch_count(void);
GLA_API gla_status gla_profiler_enable(int enable);
GLA_API int gla_profiler_read(char* names, int name_stride, int* launches, double* total_ms, int max_kernels);

#ifdef __cplusplus
}
#endif

#endif /* GLA_B200_H */
