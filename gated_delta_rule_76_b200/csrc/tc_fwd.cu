// Host side of the tensor-core chunk forward: TMA descriptors and parameters; the launches of
// each gate form are in tc_fwd_gates.cu and tc_fwd_logits.cu.
#include <cuda.h>

#include <type_traits>

#include "launch.h"
#include "tc_fwd_launch.cuh"
#include "tma_host.h"

namespace gdn {

bool tc_fwd_eligible(const Problem& pb, bool bf16_inputs, bool bf16_gates, Flags f) {
    if (!bf16_inputs || pb.dk != 128 || pb.dv != 128 || pb.T < 1) return false;
    if ((f.apc || f.gpc) && !bf16_gates) return false;  // channel gates are loaded by TMA as bf16 tiles
    return encode_fn() != nullptr;
}

namespace {
cudaError_t tc_chunk_fwd_kernel(const Problem& pb, const ChunkIO& io, Flags f, bool bf16_gates, int* err,
                                cudaStream_t st, const TcFwdSave* save, int* flags) {
    CUtensorMap maps[7];
    const bool split = io.q_lo != nullptr;
    if (split && (f.apc || f.gpc || !io.k_lo || !io.v_lo)) return cudaErrorInvalidValue;
    bool ok = make_map(&maps[0], io.q, pb.B, pb.T, pb.Hk) && make_map(&maps[1], io.k, pb.B, pb.T, pb.Hk) &&
              make_map(&maps[2], io.v, pb.B, pb.T, pb.Hv);
    // Unused maps are copies of a valid one (never dereferenced).
    maps[3] = maps[2];
    maps[4] = maps[2];
    maps[5] = maps[2];
    maps[6] = maps[2];
    if (ok && f.gate) ok = make_map(&maps[6], io.z, pb.B, pb.T, pb.Hv);  // z [B,T,Hv,dv] bf16
    if (ok && f.apc) ok = make_map(&maps[3], io.alpha, pb.B, pb.T, pb.Hv);
    if (ok && f.gpc) ok = make_map(&maps[4], io.b, pb.B, pb.T, pb.Hv) && make_map(&maps[5], io.w, pb.B, pb.T, pb.Hv);
    // Split inputs: the lo halves take the gate slots (k lo: alpha, q lo: b, v lo: w).
    if (ok && split)
        ok = make_map(&maps[3], io.k_lo, pb.B, pb.T, pb.Hk) && make_map(&maps[4], io.q_lo, pb.B, pb.T, pb.Hk) &&
             make_map(&maps[5], io.v_lo, pb.B, pb.T, pb.Hv);
    if (!ok) return cudaErrorInvalidValue;
    tcfwd::Params p{};
    p.pb = pb;
    p.alpha = io.alpha;
    p.b = io.b;
    p.z = io.z;
    p.h0 = io.h0;
    p.o = io.o;
    p.o_type = io.o_type == 1 ? 1 : 0;
    p.ht = io.ht;
    p.err = err;
    p.flags = flags;
    p.norm_w = f.gate ? io.norm_w : nullptr;
    p.norm_w_f32 = io.norm_w_f32;
    p.norm_eps = io.norm_eps;
    if (save) {
        p.s0_out = save->s0;
        p.vp_hi = save->vp_hi;
        p.vp_lo = save->vp_lo;
        p.t_out = save->t;
        p.o_raw = save->o_raw;
    }
    return pb.gate_logits ? tc_fwd_dispatch<true>(maps, p, f, split, bf16_gates, st)
                          : tc_fwd_dispatch<false>(maps, p, f, split, bf16_gates, st);
}
}  // namespace

cudaError_t tc_chunk_fwd(const Problem& pb, const ChunkIO& io, Flags f, bool bf16_gates, int* err,
                         cudaStream_t st, const TcFwdSave* save, int* flags) {
    cudaError_t e = tc_chunk_fwd_kernel(pb, io, f, bf16_gates, err, st, save, flags);
    if (e != cudaSuccess || !flags) return e;
    // Pairs whose decay left the factors' range: their outputs again, exactly (the backward's
    // saving-only forward asks for no output, and its backward recomputes such pairs itself).
    float* o_raw = save ? save->o_raw : nullptr;
    if (!io.o && !io.ht && !o_raw) return cudaSuccess;
    return seq_fwd(pb, io, f, false, !bf16_gates, flags, o_raw, st);
}

}  // namespace gdn
