// Host-side launch interface between the C ABI (gdn_api.cu) and the per-dtype kernel
// instantiation units (inst_*.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "simt_chunk.cuh"
#include "decode.cuh"
#include "conv.cuh"

namespace gdn {

// Process-wide count of kernel launches issued by the library (gdn_kernel_launches()).
void count_launch();

struct Flags {
    bool apc;   // alpha per channel
    bool gpc;   // b, w per channel (else scalar beta)
    bool gate;  // swish(z) output gate in the forward
    // CUDA-core path, a forward and a backward on one workspace: the forward also saves what the
    // backward needs (chunk states, Kt, G), and the backward does not run the forward again.
    bool paired = false;
};

// Workspace carving.  Every array is 256-byte aligned.
struct WsPlan {
    size_t bytes = 0;
    size_t T, P, Eh, Qh, Kb, Kt, Gm, gam, S0, dSC, V, Y, dV, dY, dbw, dq_v, dk_v;
    size_t flags, sbuf;  // pairs outside the chunk form's decay range; the sequential backward's states
};
WsPlan plan_chunk_ws(const Problem& pb, bool bwd, bool gqa_partials);
ChunkWs carve_chunk_ws(const WsPlan& plan, void* base);

// Per (TIn, TG) instantiation units define these (TIn: q/k/v dtype, TG: gate dtype).
#define GDN_DECLARE_LAUNCHERS(NAME)                                                           \
    cudaError_t NAME##_chunk_fwd(const Problem&, const ChunkIO&, const ChunkWs&, Flags,       \
                                 cudaStream_t);                                              \
    cudaError_t NAME##_chunk_bwd(const Problem&, const ChunkIO&, const ChunkWs&, Flags, bool, \
                                 cudaStream_t);                                              \
    cudaError_t NAME##_decode(const DecodeParams&, Flags, cudaStream_t);                       \
    cudaError_t NAME##_conv(const ConvParams&, cudaStream_t);

// Tensor-core chunk forward (tc_fwd.cu): bf16 q/k/v with dk = dv = 128.  With `save`, the state
// entering every chunk and V' of every token are written for the backward (o and ht may be NULL).
struct TcFwdSave {
    float* s0;               // [B*Hv][NT + 1][dv/8][dk][8]
    __nv_bfloat16* vp_hi;    // [B*Hv][NT][dv][64 tokens]: chunk-major, a column's tokens contiguous
    __nv_bfloat16* vp_lo;
    float* o_raw;            // with the swish gate, may be NULL: the output before the gate (fp32)
    uint8_t* t;              // [B*Hv][NT] 8 KB images of each chunk's bf16 T tile (swizzled), or NULL
};
bool tc_fwd_eligible(const Problem& pb, bool bf16_inputs, bool bf16_gates, Flags f);
// flags: [B*Hv] ints, zero on entry (or NULL): the kernel marks the pairs whose decay leaves the
// chunk form's range, and the exact sequential kernel then recomputes their outputs.
cudaError_t tc_chunk_fwd(const Problem& pb, const ChunkIO& io, Flags f, bool bf16_gates, int* err,
                         cudaStream_t st, const TcFwdSave* save = nullptr, int* flags = nullptr);

// Exact sequential recurrence (seq.cu) for the pairs marked in flags: the forward (o, the output
// before the gate, ht) and the backward (every gradient; ck: per pair ck_stride floats for the
// states entering chunks 1..NT-1, sbuf: seq_sbuf_floats()).  dq, dk are per key head when direct
// (in the gradients' type, io.grad_type), else per value head (fp32 partials).
size_t seq_sbuf_floats(const Problem& pb);
cudaError_t seq_fwd(const Problem& pb, const ChunkIO& io, Flags f, bool tin_f32, bool tg_f32, const int* flags,
                    float* o_raw, cudaStream_t st);
cudaError_t seq_bwd(const Problem& pb, const ChunkIO& io, Flags f, bool tin_f32, bool tg_f32, const int* flags,
                    void* dq, void* dk, bool direct, float* ck, long ck_stride, float* sbuf, cudaStream_t st);

// Gates as logits (gates.cu): after a backward, the gates' gradients become those of their logits
// (in place, fp32 or, with grad_bf16, bf16), and alpha's scale gets its gradient (dalpha_scale [Hv]
// fp32, may be NULL).
cudaError_t gate_logit_grads(const Problem& pb, Flags f, bool tg_f32, const void* x_alpha, const void* x_b,
                             const void* x_w, void* dalpha, void* db, void* dw, bool grad_bf16, float* dalpha_scale,
                             cudaStream_t st);

// Sequence split along time (seqpar.cu): S = I for `pairs` states of d x d; S_out = op(M) S_in + N
// per pair (op = transpose or not; S_in or N may be NULL: taken as zero).
cudaError_t identity_states(float* S, long pairs, int d, cudaStream_t st);
cudaError_t compose_states(const float* M, const float* N, const float* S_in, float* S_out, long pairs, int dk,
                           int dv, bool transpose, cudaStream_t st);

// Strided inputs (strides.cu): `rows` rows of row_bytes bytes, stride_bytes apart in src, copied
// back to back into dst (256-byte aligned).  cudaErrorMisalignedAddress if src is odd.
cudaError_t pack_rows(const void* src, void* dst, long rows, long row_bytes, long stride_bytes, cudaStream_t st);

// Tensor-core chunk backward (tc_bwd.cu): same eligibility as the forward, without z.
// The forward cache (what the backward needs from the forward): byte offsets from its start.
struct TcCache {
    size_t bytes = 0;
    size_t s0, vp_hi, vp_lo;  // states [B*Hv][NT+1][dv/8][dk][8] fp32; V' hi, lo [B*Hv][NT][dv][64] bf16
    size_t t;                 // T tiles [B*Hv][NT][8 KB]: bf16, 64 rows of 128 swizzled bytes
};
TcCache plan_tc_cache(const Problem& pb);
// The forward's save targets inside a cache laid out by plan_tc_cache.
TcFwdSave tc_save_in(void* cache, const Problem& pb, float* o_raw);
struct TcBwdWs {
    size_t bytes = 0;  // total, including the 256-byte status word at offset 0
    size_t cache;      // a forward cache inside the workspace (~0 when the caller passes one)
    size_t dsc, ny_hi, ny_lo, dq_v, dk_v;  // byte offsets (dq_v, dk_v: GQA only)
    size_t flags, sbuf;                    // pairs outside the decay range; sequential backward states
};
TcBwdWs plan_tc_bwd_ws(const Problem& pb, bool gqa_partials, bool caller_cache);
// cache: the caller's forward cache (the forward is not recomputed), or NULL.
cudaError_t tc_chunk_bwd(const Problem& pb, const ChunkIO& io, Flags f, bool bf16_gates, bool direct,
                         const TcBwdWs& plan, void* ws, const void* cache, cudaStream_t st);

// Layer-core backward pieces (layer_bwd.cu).
struct LayerBwdIO {
    const void *xq, *xk, *xv, *conv_w;  // layer inputs (dtype)
    const void *z, *dy;                 // [B,T,Hv,d] (dtype)
    const float* o;                     // [B,T,Hv,d] the recurrence's output, before the gate
    const float *gq, *gk, *gv;          // gradients of the L2-normalised q, k and of v
    float *dout, *dz;                   // out: gradient of o (fp32), of z
    __nv_bfloat16 *dout16, *dout16_lo;  // out instead of dout when set: the gradient of o as bf16 hi/lo
    float *dxq, *dxk, *dxv;             // out: gradients of the conv inputs
    float *wpart, *dconv_w;             // per-tile partial sums of the conv-weight gradient; out
    int B, T, Hk, Hv, d;
    // the output norm (y = RMSNorm(o) * norm_w * swish(z)), or norm_w NULL: y = o * swish(z)
    const void* norm_w;
    int norm_w_f32;
    float norm_eps;
    float *npart, *dnorm_w;             // per-warp partials of the norm weights' gradient; out [d]
};
size_t layer_bwd_wpart_floats(int B, int T, int Hk, int Hv, int d);
size_t layer_norm_partials_floats(int d);
// y = RMSNorm(o) * norm_w * swish(z) over rows of d values (o fp32; z, y in the layer dtype, or y fp32)
cudaError_t layer_norm_gate_fwd(const float* o, const void* z, const void* norm_w, int norm_w_f32, float eps,
                                void* y, int y_f32, bool bf16, long rows, int d, cudaStream_t st);
cudaError_t layer_gate_bwd(const LayerBwdIO& io, bool bf16, cudaStream_t st);
cudaError_t layer_conv_bwd(const LayerBwdIO& io, bool bf16, cudaStream_t st);

GDN_DECLARE_LAUNCHERS(bf16)       // bf16 tensors, bf16 gates
GDN_DECLARE_LAUNCHERS(bf16_f32g)  // bf16 tensors, fp32 gates
GDN_DECLARE_LAUNCHERS(f32)        // fp32 tensors, fp32 gates
GDN_DECLARE_LAUNCHERS(f32_bf16g)  // fp32 tensors, bf16 gates (layer-core intermediates)

}  // namespace gdn
