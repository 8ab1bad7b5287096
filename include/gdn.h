/*
 * gdn.h — C ABI of the gated delta-rule recurrence library (libgdn.so, CUDA for sm_100a).
 *
 * The operation (Gated DeltaNet-2 summary, gist.science, «Méthodologie» §1 «Règle Delta
 * Portée-2»; restated in the zubnet.ai news item on Gated DeltaNet-2):
 *
 *     S_t = (I - k_t e_t^T) Diag(alpha_t) S_{t-1} + k_t z_t^T,   e_t = b_t .* k_t,  z_t = w_t .* v_t
 *     o_t = scale * S_t^T q_t
 *
 * with S_t in R^{dk x dv} (dk rows, dv contiguous columns), the erase gate b_t in [0,1]^dk on the
 * key axis, the write gate w_t in [0,1]^dv on the value axis and the channel decay alpha_t in
 * (0,1)^dk.  Erase gates (b or the scalar beta) up to 2 are accepted as well: the negative-
 * eigenvalue variant of the Gated DeltaNet explainer's note under «Réunir les deux» (for a unit
 * key the transition's eigenvalue along k is 1 - beta in [-1, 1]); every kernel is unchanged.  With b = w = beta (one scalar per token and head) and a scalar alpha this is Gated
 * DeltaNet (Gated DeltaNet explainer, docsaid.org, «Réunir les deux»); with alpha = 1 as well it
 * is DeltaNet («DeltaNet : ne corriger que l'entrée visée»).  Channel alpha with scalar beta is
 * the KDA case named on the same GDN-2 page.
 *
 * Conventions shared by every call
 *  - Ownership: the caller owns every buffer.  The library allocates no device memory; scratch
 *    memory is a caller workspace whose size the *_workspace_size() calls return (the workspace
 *    may be reused across calls on the same stream; its contents on entry do not matter).
 *  - Pointers: every tensor pointer is a device pointer (cudaMalloc'd or equivalent) to a dense,
 *    contiguous array in the layout stated; all must be 16-byte aligned.  Token-major inputs
 *    may instead be given with a token stride (gdn_strides below).  Outputs must not overlap
 *    inputs (a strided input spans its first to its last element) or each other (in-place
 *    arguments say so explicitly).
 *  - Execution: every call is asynchronous on the given stream and never synchronises.
 *    Outputs are valid once the stream reaches the end of the call.
 *  - Layouts: token-major.  q, k: [B,T,Hk,dk]; v, o, z: [B,T,Hv,dv]; channel gates alpha, b:
 *    [B,T,Hv,dk], w: [B,T,Hv,dv]; scalar gates alpha, beta: [B,T,Hv]; states: [B,Hv,dk,dv] fp32.
 *  - GQA: value head hv reads key head head_map[hv] (int32 device array of Hv entries).  NULL
 *    means contiguous groups hv / (Hv / Hk) (Hv must then be a multiple of Hk).  Every entry
 *    must lie in [0, Hk); the map lives on the device, so the host cannot check it: kernels clamp
 *    an entry outside that range into it (no read falls outside q or k) and the results are then
 *    unspecified.  The Python binding checks the map before uploading it.  Several value
 *    heads share each key head in the 16-key / 128-value layer of the mkdocs chapter «Gated
 *    DeltaNet», «Les projections d'entrée».
 *  - Sizes: dk, dv in {64, 128}; B, T, Hk, Hv >= 1 (T = 0 is accepted and does nothing but copy
 *    h0 to ht).  T need not be a multiple of the chunk length 64.
 *  - Dtypes: q, k, v, o, z in `dtype`; alpha, b, w, beta in `gate_dtype`; states are fp32;
 *    gradients are fp32 by default (they leave the fp32 accumulators unrounded: several of them
 *    are heavy-tailed, and a bf16 store alone would cost up to half an ulp of their largest
 *    entry), or in the inputs' dtypes with gdn_chunk_bwd's grads_in_dtype.
 *  - Range: every alpha in [0, 1] is supported.  The chunked kernels carry the decay inside a
 *    chunk of 64 tokens as a ratio Gamma_r / Gamma_s of running products of alpha, which fp32
 *    holds while the product over a chunk stays at or above 2^-100 (~7.9e-31) on every channel.
 *    Each chunk kernel checks that bound on every chunk; a (sequence, head) pair with a chunk
 *    below it is recomputed by an exact sequential kernel in the same call (token by token, no
 *    ratio of decays), which overwrites that pair's results.  Such pairs cost several times more
 *    than the chunk form.  The single-token decode step has no ratio and no such bound.
 *  - Gates as logits (optional, gate_logits = 1 in the args): alpha, b, w, beta are then given as
 *    logits x (same layouts and gate_dtype) and every kernel applies, where it reads a gate,
 *        alpha = exp(-alpha_scale[hv] * softplus(x)),   b, w, beta = sigmoid(x)
 *    with alpha_scale [Hv] fp32 > 0 (explainer «Architecture et versions hybrides», Figure 1
 *    caption: alpha takes the Mamba-2 parametrisation exp(-A dt), dt = softplus(x), A = alpha_scale;
 *    the zubnet.ai news item: the erase and write gates are two sigmoids).  The backward then
 *    returns the gradients of the logits in grad_alpha, grad_b, grad_w, and (if not NULL) that of
 *    alpha_scale in grad_alpha_scale [Hv] (summed over batch, tokens and channels in a fixed order).
 *  - Errors: every call returns a gdn_status.  Invalid arguments are detected on the host before
 *    any launch and nothing is written.  gdn_last_error() returns a thread-local message about
 *    the last failure of the calling thread.  No C++ exception crosses this interface.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int gdn_status;
#define GDN_OK 0
#define GDN_ERR_INVALID_ARG 1 /* null required pointer, bad size, misaligned or overlapping buffer */
#define GDN_ERR_UNSUPPORTED 2 /* valid but not implemented here: dk/dv outside {64,128}, dtype */
#define GDN_ERR_CUDA 3        /* a CUDA call or kernel launch failed (message has the CUDA error) */
#define GDN_ERR_WORKSPACE 4   /* workspace NULL or smaller than *_workspace_size() */
#define GDN_ERR_TIMEOUT 5     /* a bounded wait inside a kernel expired (see gdn_workspace_status) */

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

/* Opaque stream handle: a cudaStream_t (NULL = the legacy default stream). */
typedef void* gdn_stream;

/* Token strides of the token-major inputs of a call, in elements (every field optional).
 *  - 0: the tensor is dense in the layout stated for it.
 *  - s > 0: token t of sequence b starts at element (b * T + t) * s (the decode step: sequence n
 *    at n * s), and that token's heads and channels follow it densely.  This lets a caller pass
 *    the slices of one fused projection buffer ([B, T, C] with the q, k, v, gate columns side by
 *    side) without copying them first.  s must be at least the token's own element count (H * d,
 *    or H for a scalar gate) and at most 2^31; a tensor given with s > that count needs only the
 *    alignment of its element type.
 *  - Chunk forward, backward, segment map and layer calls copy every tensor whose stride is not
 *    its dense one into a dense part of the workspace first (one copy kernel per tensor; the
 *    bytes are part of *_workspace_size()).  The decode step reads strided tensors in place.
 *  - The layer calls read q, k, v as the strides of xq, xk, xv.  A field whose tensor the call
 *    does not take (z of gdn_chunk_bwd) must be 0. */
typedef struct gdn_strides {
    int64_t q, k, v, alpha, b, w, z;
} gdn_strides;

/* ------------------------------------------------------------------------------------------
 * Chunkwise forward.  Chunkwise-parallel form with chunk length 64: inside a chunk the decay is
 * absorbed into the erase and write factors and the lower-triangular system (I + A)^-1 is solved
 * for the erase-side and write-side auxiliaries (GDN-2 summary, «Entraînement Parallèle
 * Efficace par Blocs»; explainer «Rendre l'entraînement parallèle»); the state is carried from
 * chunk to chunk in fp32.
 * ------------------------------------------------------------------------------------------ */
typedef struct gdn_fwd_args {
    const void* q;        /* [B,T,Hk,dk]  dtype */
    const void* k;        /* [B,T,Hk,dk]  dtype */
    const void* v;        /* [B,T,Hv,dv]  dtype */
    const void* alpha;    /* [B,T,Hv,dk] if alpha_per_channel else [B,T,Hv]; gate_dtype, in (0,1] */
    const void* b;        /* erase gate [B,T,Hv,dk] if gates_per_channel, else beta [B,T,Hv] */
    const void* w;        /* write gate [B,T,Hv,dv] if gates_per_channel, else must be NULL */
    const float* h0;      /* [B,Hv,dk,dv] initial state, NULL = zeros */
    const void* z;        /* optional swish output gate [B,T,Hv,dv] dtype: o <- o * z * sigmoid(z) */
    void* o;              /* out [B,T,Hv,dv] dtype (fp32 if out_f32) */
    float* ht;            /* out [B,Hv,dk,dv] final state, may be NULL */
    const int32_t* head_map; /* [Hv] value head -> key head, NULL = contiguous groups */
    int64_t B, T, Hk, Hv, dk, dv;
    float scale;          /* readout scale (the pages use 1) */
    int32_t alpha_per_channel; /* 1: alpha in (0,1)^dk; 0: one scalar per token and value head */
    int32_t gates_per_channel; /* 1: separate b (dk) and w (dv); 0: scalar beta, b = w = beta */
    int32_t dtype;        /* gdn_dtype of q, k, v, z, o */
    int32_t gate_dtype;   /* gdn_dtype of alpha, b, w */
    int32_t out_f32;      /* 1: o is written in fp32 (unrounded accumulator) instead of dtype */
    /* Optional cache for a later gdn_chunk_bwd over the same inputs (training): when not NULL the
     * forward also writes the state entering every chunk, the final state and V' = T (Z - Ehat S0)
     * of every token into this caller buffer, and a backward given it skips recomputing them.
     * Needs bwd_cache_bytes >= gdn_chunk_fwd_cache_size(args) and a 256-byte-aligned start; only
     * the tensor-core path (bf16 q/k/v, dk = dv = 128) keeps a cache: elsewhere the size is 0 and
     * bwd_cache must be NULL.  The cache is independent of z. */
    void* bwd_cache;
    size_t bwd_cache_bytes;
    int32_t gate_logits;       /* 1: alpha, b, w are logits (see the conventions above) */
    const float* alpha_scale;  /* [Hv] fp32, with gate_logits */
    gdn_strides strides;       /* token strides of q, k, v, alpha, b, w, z (all 0: dense) */
} gdn_fwd_args;

/* Bytes of the optional forward cache (0 where the problem cannot keep one). */
GDN_API size_t gdn_chunk_fwd_cache_size(const gdn_fwd_args* args);
GDN_API size_t gdn_chunk_fwd_workspace_size(const gdn_fwd_args* args);
GDN_API gdn_status gdn_chunk_fwd(const gdn_fwd_args* args, void* workspace, size_t workspace_bytes,
                         gdn_stream stream);

/* Chunkwise forward without a caller workspace.  The source pages have no counterpart: this is a
 * convenience of the library for callers that cannot hand out device memory.  Arguments, results,
 * validation and errors are those of gdn_chunk_fwd; the scratch memory is a fixed 16 MiB device
 * array inside the library (one per device), used as gdn_chunk_fwd's workspace.
 *  - Limit: a problem whose gdn_chunk_fwd_workspace_size() exceeds 16 MiB is rejected with
 *    GDN_ERR_WORKSPACE before anything is launched (the tensor-core path needs 256 bytes plus
 *    4 bytes per (sequence, value head), so bf16 problems with dk = dv = 128 fit up to ~4 million
 *    pairs; the CUDA-core path needs per-chunk factors; strided inputs add their dense copies).
 *  - Set-up: every call looks up the array's address on the current device with
 *    cudaGetSymbolAddress (so a device reset between calls is harmless).  The first call on a
 *    device may load the library's device code there; make it before any stream capture.  Later
 *    lookups are host-side; each call then launches work on `stream` only.
 *  - Nothing is allocated (no cudaMalloc, no host or device allocation by any library).  The
 *    status word at the start of the scratch is cleared on `stream` at the start of every call;
 *    nothing else in the scratch needs to start at zero.  An expired bounded wait inside a kernel
 *    is not reported by this call (it returns before the kernels run); gdn_chunk_fwd_noalloc_status
 *    reads the status word afterwards.
 *  - Concurrency: every call on a device uses the same scratch array.  Calls whose execution can
 *    overlap (different streams, or different host threads without ordering) race on it; the
 *    caller must order them, e.g. by issuing them all on one stream. */
GDN_API gdn_status gdn_chunk_fwd_noalloc(const gdn_fwd_args* args, gdn_stream stream);
/* The status word of the current device's scratch, as gdn_workspace_status reads a workspace's:
 * synchronises `stream`, then GDN_OK, or GDN_ERR_TIMEOUT if a bounded wait of the last
 * gdn_chunk_fwd_noalloc call on this device expired. */
GDN_API gdn_status gdn_chunk_fwd_noalloc_status(gdn_stream stream);

/* ------------------------------------------------------------------------------------------
 * Chunkwise backward.  Reverse mode of gdn_chunk_fwd (without z): the chunk-boundary states are
 * recomputed, the state gradient is scanned from the last chunk to the first, and per chunk the
 * gradients of the auxiliary matrices carry the channel gates b and w inside their accumulation
 * (GDN-2 summary, «Passage Arrière Conscient des Portes»).
 * grad_alpha is the gradient with respect to alpha itself (not log alpha).  grad_q and grad_k are summed
 * over the value heads that share a key head, in a fixed order (deterministic).
 * Gradient dtype: fp32 by default.  With grads_in_dtype = 1 they are returned in the inputs' dtypes:
 * grad_q, grad_k, grad_v in `dtype`, grad_alpha, grad_b, grad_w in `gate_dtype`, each rounded once
 * from its fp32 value (accumulation stays fp32; sums over value heads are taken in fp32 before the
 * rounding).  grad_h0 and grad_alpha_scale are fp32 always.  grads_in_dtype = 1 with dtype BF16 is
 * served by the tensor-core backward only (dk = dv = 128, bf16 gates with channel gates); other
 * bf16 problems return GDN_ERR_UNSUPPORTED.  With dtype F32 the two settings are the same.
 * ------------------------------------------------------------------------------------------ */
typedef struct gdn_bwd_args {
    const void* q;        /* forward inputs, same layouts and dtypes as gdn_fwd_args */
    const void* k;
    const void* v;
    const void* alpha;
    const void* b;
    const void* w;
    const float* h0;      /* NULL = zeros */
    const int32_t* head_map;
    const void* grad_o;   /* [B,T,Hv,dv] dtype, gradient of o */
    const float* grad_ht; /* [B,Hv,dk,dv] gradient of the final state, NULL = zeros */
    void* grad_q;         /* out [B,T,Hk,dk] fp32 (dtype with grads_in_dtype) */
    void* grad_k;         /* out [B,T,Hk,dk] fp32 (dtype with grads_in_dtype) */
    void* grad_v;         /* out [B,T,Hv,dv] fp32 (dtype with grads_in_dtype) */
    void* grad_alpha;     /* out, shape of alpha, fp32 (gate_dtype with grads_in_dtype) */
    void* grad_b;         /* out, shape of b (grad of beta [B,T,Hv] when gates are scalar), fp32 (gate_dtype
                           * with grads_in_dtype) */
    void* grad_w;         /* out, shape of w, fp32 (gate_dtype with grads_in_dtype); NULL for scalar gates */
    float* grad_h0;       /* out [B,Hv,dk,dv] fp32, may be NULL */
    int64_t B, T, Hk, Hv, dk, dv;
    float scale;
    int32_t alpha_per_channel;
    int32_t gates_per_channel;
    int32_t dtype;
    int32_t gate_dtype;
    /* Optional: the cache a gdn_chunk_fwd call wrote with exactly these inputs (q, k, v, alpha, b,
     * w, h0, head_map, scale, sizes).  The backward then reads the saved chunk states and V' instead
     * of recomputing the forward.  The library cannot check that the cache belongs to these
     * inputs: a stale cache gives wrong gradients.  NULL: the forward is recomputed. */
    const void* fwd_cache;
    size_t fwd_cache_bytes;
    int32_t gate_logits;       /* 1: alpha, b, w are logits; the gradients returned are those of the logits */
    const float* alpha_scale;  /* [Hv] fp32, with gate_logits */
    float* grad_alpha_scale;   /* out [Hv] fp32, may be NULL (must be NULL without gate_logits) */
    int32_t grads_in_dtype;    /* 1: gradients in the inputs' dtypes (see above); 0: fp32 */
    gdn_strides strides;       /* token strides of q, k, v, alpha, b, w (z: 0); gradients are dense */
} gdn_bwd_args;

GDN_API size_t gdn_chunk_bwd_workspace_size(const gdn_bwd_args* args);
GDN_API gdn_status gdn_chunk_bwd(const gdn_bwd_args* args, void* workspace, size_t workspace_bytes,
                         gdn_stream stream);

/* ------------------------------------------------------------------------------------------
 * Sequence split along time (several GPUs, one segment of every sequence each).  The recurrent
 * state has a fixed size whatever the context length (mkdocs chapter «Gated DeltaNet», «L'état,
 * en mémoire»), and each token's update is affine in it (GDN-2 summary, «Méthodologie» §1):
 * S_t = A_t S_{t-1} + k_t z_t^T with A_t = (I - k_t e_t^T) Diag(alpha_t).  A segment therefore
 * maps the state entering it to M S + N, with M = A_T ... A_1 (dk x dk) and N the state after the
 * segment entered with zeros (dk x dv).  The state entering segment r is the composition of the
 * maps of segments 0 .. r-1 applied to h0; a state gradient crosses a segment backwards as
 * M^T dS (+ the segment's own contribution, which a backward with zero dht gives as dh0).
 *
 * gdn_segment_map: for one segment of every (sequence, value head), M [B,Hv,dk,dk] fp32 and
 * N = args->ht [B,Hv,dk,dv] fp32 (required).  args is read as by gdn_chunk_fwd, except that h0, z
 * and bwd_cache must be NULL and o may be NULL (if given, it receives the segment's output from a
 * zero entering state).  Needs dk == dv.  It runs the chunk forward twice: from a zero state (N),
 * and from the identity with the writes zeroed (M), so the decay-range handling of
 * gdn_chunk_fwd applies.  Workspace: gdn_segment_map_workspace_size(args) bytes, 256-byte aligned.
 * ------------------------------------------------------------------------------------------ */
GDN_API size_t gdn_segment_map_workspace_size(const gdn_fwd_args* args);
GDN_API gdn_status gdn_segment_map(const gdn_fwd_args* args, float* M, void* workspace, size_t workspace_bytes,
                                   gdn_stream stream);

/* S_out = M S_in + N (transpose = 0) or M^T S_in + N (transpose = 1, needs dk == dv) for `pairs`
 * independent (sequence, head) pairs, fp32: M [pairs,dk,dk], N and S_in and S_out [pairs,dk,dv].
 * S_in or N may be NULL (taken as zero).  S_out must not overlap M, N or S_in.  dk, dv in
 * {64, 128}.  The composition step of the sequence split above, on the device. */
GDN_API gdn_status gdn_state_compose(const float* M, const float* N, const float* S_in, float* S_out, int64_t pairs,
                                     int64_t dk, int64_t dv, int32_t transpose, gdn_stream stream);

/* ------------------------------------------------------------------------------------------
 * Single-token decode step for N sequences: the recurrence applied once, with the fp32 state
 * read, updated and written back in place (constant memory per sequence; mkdocs chapter «Gated
 * DeltaNet», «L'état, en mémoire»).
 * Optional fusions (mkdocs chapter «La convolution causale», «La porte de sortie»; explainer
 * Figure 1 caption):
 *  - conv_state != NULL: q, k, v are the raw projections of the new token; each of the
 *    Cch = 2*Hk*dk + Hv*dv channels (ordered q, k, v) is convolved with its 4 taps over the
 *    3 stored previous inputs and the new one (conv_w[ch][3] weights the new token), passed
 *    through SiLU, and q, k are L2-normalised (x / sqrt(sum x^2 + 1e-6)); conv_state
 *    [N, Cch, 3] (dtype, oldest first) is then shifted to hold the last 3 inputs.
 *  - z != NULL: o <- o * z * sigmoid(z).
 * ------------------------------------------------------------------------------------------ */
typedef struct gdn_decode_args {
    const void* q;        /* [N,Hk,dk] dtype */
    const void* k;        /* [N,Hk,dk] dtype */
    const void* v;        /* [N,Hv,dv] dtype */
    const void* alpha;    /* [N,Hv,dk] or [N,Hv], gate_dtype */
    const void* b;        /* [N,Hv,dk] or beta [N,Hv] */
    const void* w;        /* [N,Hv,dv] or NULL */
    float* state;         /* in/out [N,Hv,dk,dv] fp32, updated in place */
    void* o;              /* out [N,Hv,dv] dtype */
    const int32_t* head_map;
    void* conv_state;     /* optional in/out [N, 2*Hk*dk + Hv*dv, 3] dtype */
    const void* conv_w;   /* [2*Hk*dk + Hv*dv, 4] dtype, required with conv_state */
    const void* z;        /* optional [N,Hv,dv] dtype */
    int64_t N, Hk, Hv, dk, dv;
    float scale;
    int32_t alpha_per_channel;
    int32_t gates_per_channel;
    int32_t dtype;
    int32_t gate_dtype;
    int32_t out_f32;      /* 1: o is written in fp32 instead of dtype */
    int32_t gate_logits;       /* 1: alpha, b, w are logits */
    const float* alpha_scale;  /* [Hv] fp32, with gate_logits */
    gdn_strides strides;       /* per-sequence strides of q, k, v, alpha, b, w, z, read in place */
} gdn_decode_args;

GDN_API gdn_status gdn_decode_step(const gdn_decode_args* args, gdn_stream stream);

/* ------------------------------------------------------------------------------------------
 * GQA layer core (forward): causal depthwise convolution (kernel 4, no bias, zero history)
 * + SiLU on the q, k, v projections, L2 normalisation of q and k, the chunkwise recurrence, and
 * the swish(z) output gate.  Explainer «Architecture et versions hybrides» (Figure 1 caption);
 * mkdocs chapter «Gated DeltaNet» (16 key heads, 128 value heads, kernel 4, swish gate).
 * Convolution channels are ordered q (Hk*dk), k (Hk*dk), v (Hv*dv); conv_w is [Cch, 4] with
 * conv_w[ch][3] weighting the current token.  conv_state_out, if not NULL, receives the last
 * three raw inputs of every channel ([B, Cch, 3], dtype) so that decoding can continue.
 * The convolution outputs are fp32 values kept in the workspace.  With bf16 tensors, dk = dv =
 * 128 and scalar gates they are stored as bf16 hi/lo pairs (x = hi + lo to 16 mantissa bits) and
 * the tensor-core chunk forward consumes them; otherwise they stay fp32 for the CUDA-core forward.
 * ------------------------------------------------------------------------------------------ */
typedef struct gdn_layer_args {
    const void* xq;       /* [B,T,Hk,dk] dtype (pre-convolution projections) */
    const void* xk;       /* [B,T,Hk,dk] */
    const void* xv;       /* [B,T,Hv,dv] */
    const void* conv_w;   /* [Cch, 4] dtype */
    const void* alpha;    /* as gdn_fwd_args */
    const void* b;
    const void* w;
    const void* z;        /* [B,T,Hv,dv] swish gate, required */
    const float* h0;      /* NULL = zeros */
    void* y;              /* out [B,T,Hv,dv] dtype */
    float* ht;            /* out, may be NULL */
    void* conv_state_out; /* out, may be NULL */
    const int32_t* head_map;
    int64_t B, T, Hk, Hv, dk, dv;
    float scale;
    int32_t alpha_per_channel;
    int32_t gates_per_channel;
    int32_t dtype;
    int32_t gate_dtype;
    int32_t out_f32;      /* 1: y is written in fp32 instead of dtype */
    /* Optional cache for a later gdn_layer_core_bwd over the same inputs (training): when not NULL
     * the forward also keeps its conv results (bf16 hi/lo pairs), the recurrence's output before
     * the gate (fp32), the state entering every chunk and V' of every token in this caller
     * buffer, and a backward given it skips recomputing them.  Needs bwd_cache_bytes >=
     * gdn_layer_core_fwd_cache_size(args) and a 256-byte-aligned start.  Only the layer's
     * tensor-core backward form keeps one (bf16 tensors, dk = dv = 128, scalar gates, no h0):
     * elsewhere the size is 0 and bwd_cache must be NULL. */
    void* bwd_cache;
    size_t bwd_cache_bytes;
    /* Optional output norm before the gate (explainer «Architecture et versions hybrides», Figure 1
     * caption: the output is normalised, then multiplied by a gate; mkdocs chapter «Gated
     * DeltaNet», «Le décompte»: dv norm weights shared by the heads).  When norm_w [dv] (dtype) is
     * not NULL: y = o / sqrt(mean_j o_j^2 + norm_eps) * norm_w * z * sigmoid(z) for every
     * (token, value head) row o of dv values.  NULL: y = o * z * sigmoid(z).  The cache keeps o
     * before the norm. */
    const void* norm_w;
    float norm_eps;
    int32_t gate_logits;       /* 1: alpha, b, w are logits */
    const float* alpha_scale;  /* [Hv] fp32, with gate_logits */
    gdn_strides strides;       /* token strides of xq, xk, xv (fields q, k, v), alpha, b, w, z */
} gdn_layer_args;

/* Bytes of the optional layer forward cache (0 where the layer backward cannot use one). */
GDN_API size_t gdn_layer_core_fwd_cache_size(const gdn_layer_args* args);
GDN_API size_t gdn_layer_core_fwd_workspace_size(const gdn_layer_args* args);
GDN_API gdn_status gdn_layer_core_fwd(const gdn_layer_args* args, void* workspace, size_t workspace_bytes,
                              gdn_stream stream);

/* ------------------------------------------------------------------------------------------
 * GQA layer core (backward): the reverse mode of gdn_layer_core_fwd for the gradients dy of y
 * and (optionally) dht of the final state.  The explainer's «Architecture et versions hybrides»
 * (Figure 1 caption) and the mkdocs chapter «Gated DeltaNet» give the layer; each reverse step is
 * the derivative of its forward step:
 *   swish gate  y = o * z * sigmoid(z):  do = dy * z s,  dz = dy * o * (s + z s (1 - s)), s = sigmoid(z)
 *   recurrence  the chunk backward (gdn_chunk_bwd) on the fp32 conv results, with do and dht
 *   L2 norm     q = a / sqrt(|a|^2 + 1e-6):  da = (dq - q (q . dq)) / sqrt(|a|^2 + 1e-6)
 *   SiLU        a = u sigmoid(u):  du = da * (s + u s (1 - s))
 *   conv        u_t = sum_tap w[tap] x_{t-3+tap}:  dx_s = sum_tap w[tap] du_{s+3-tap},
 *               dconv_w[ch][tap] = sum over tokens of du_t x_{t-3+tap}
 * The forward parts it needs (conv results, the recurrence's output o) are recomputed in the
 * workspace.  With bf16 tensors, d = 128, scalar gates and no h0 the recurrence runs on the
 * tensor cores: the conv results as bf16 hi/lo pairs, do as bf16 hi/lo pairs, the backward once
 * per half of do (it is linear in do and dht) with the two sets of gradients added.  Otherwise
 * (h0 given, channel gates, d = 64, fp32 tensors) it runs on the fp32 CUDA-core chunk kernels,
 * whose workspace is large.  gdn_layer_core_bwd_workspace_size() says how large; dk must equal
 * dv.  With h0 the first tokens' dxk reaches tens of times its RMS, where the tensor-core path's
 * ~1e-3 relative error would exceed the 2e-2-of-RMS budget: hence the fp32 kernels there.
 * ------------------------------------------------------------------------------------------ */
typedef struct gdn_layer_bwd_args {
    const void* xq;       /* the forward's inputs, as in gdn_layer_args */
    const void* xk;
    const void* xv;
    const void* conv_w;
    const void* alpha;
    const void* b;
    const void* w;
    const void* z;
    const float* h0;      /* NULL = zeros */
    const int32_t* head_map;
    const void* grad_y;   /* [B,T,Hv,dv] dtype, required */
    const float* grad_ht; /* [B,Hv,dk,dv] fp32, NULL = zeros */
    float* grad_xq;       /* out [B,T,Hk,dk] fp32 */
    float* grad_xk;       /* out [B,T,Hk,dk] fp32 */
    float* grad_xv;       /* out [B,T,Hv,dv] fp32 */
    float* grad_conv_w;   /* out [Cch, 4] fp32 */
    float* grad_alpha;    /* out, shape of alpha, fp32 */
    float* grad_b;        /* out, shape of b (grad of beta [B,T,Hv] when gates are scalar), fp32 */
    float* grad_w;        /* out, shape of w with channel gates; NULL otherwise */
    float* grad_z;        /* out [B,T,Hv,dv] fp32 */
    float* grad_h0;       /* out [B,Hv,dk,dv] fp32, may be NULL */
    int64_t B, T, Hk, Hv, dk, dv;
    float scale;
    int32_t alpha_per_channel;
    int32_t gates_per_channel;
    int32_t dtype;
    int32_t gate_dtype;
    /* Optional: the cache a gdn_layer_core_fwd call wrote with exactly these inputs.  The backward
     * then reads the conv results, o, the chunk states and V' from it instead of recomputing them.
     * The library cannot check that the cache belongs to these inputs: a stale cache gives wrong
     * gradients.  NULL: the forward parts are recomputed. */
    const void* fwd_cache;
    size_t fwd_cache_bytes;
    /* The output norm of gdn_layer_args (NULL: none).  With it, grad_norm_w [dv] fp32 is required and
     * receives the norm weights' gradient, summed over tokens and heads in a fixed order. */
    const void* norm_w;
    float norm_eps;
    float* grad_norm_w;
    int32_t gate_logits;       /* 1: alpha, b, w are logits; the gradients returned are those of the logits */
    const float* alpha_scale;  /* [Hv] fp32, with gate_logits */
    float* grad_alpha_scale;   /* out [Hv] fp32, may be NULL (must be NULL without gate_logits) */
    gdn_strides strides;       /* token strides of xq, xk, xv (fields q, k, v), alpha, b, w, z */
} gdn_layer_bwd_args;

GDN_API size_t gdn_layer_core_bwd_workspace_size(const gdn_layer_bwd_args* args);
GDN_API gdn_status gdn_layer_core_bwd(const gdn_layer_bwd_args* args, void* workspace, size_t workspace_bytes,
                                      gdn_stream stream);

/* Device-side status of the last call that used `workspace` (a chunk forward, backward or layer
 * core).  The tensor-core kernels bound every internal wait; when one expires the kernel records
 * it in the workspace, stops issuing work, releases its tensor memory and returns.  This call
 * synchronises `stream`, returns GDN_ERR_TIMEOUT if such an expiry was recorded (GDN_OK
 * otherwise) and does not clear the record (the next call on the workspace does). */
GDN_API gdn_status gdn_workspace_status(const void* workspace, gdn_stream stream);

/* Thread-local description of the calling thread's last failure ("" if none). */
GDN_API const char* gdn_last_error(void);

/* Number of CUDA kernels this library has launched in the calling process so far (all
 * devices and threads).  For benchmarking and diagnostics; it never resets. */
GDN_API long long gdn_kernel_launches(void);

/* Library version, major * 10000 + minor * 100 + patch. */
GDN_API int gdn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN_H */
