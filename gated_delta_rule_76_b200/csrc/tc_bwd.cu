// Host side of the tensor-core chunk backward: workspace plan, TMA descriptors, launches.
// One call runs the forward kernel in saving mode, the reverse state-gradient scan, the
// chunk-parallel gradient kernel, the exact sequential backward for the pairs outside the decay
// range (a launch that returns at once for the others) and, when value heads share key heads, the
// GQA reduction.
#include <cuda.h>

#include "launch.cuh"
#include "tc_bwd_launch.cuh"
#include "tma_host.h"

namespace gdn {

namespace {

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

TcCache plan_tc_cache(const Problem& pb) {
    TcCache c;
    const size_t st1 = (size_t)pb.B * pb.Hv * (pb.NT + 1) * pb.dk * pb.dv * sizeof(float);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = al256(off + bytes);
        return o;
    };
    c.s0 = take(st1);  // entering state of every chunk, then the final state
    const size_t vtile = (size_t)pb.B * pb.Hv * pb.NT * pb.dv * 64 * 2;  // chunk-major, padded to 64 tokens
    c.vp_hi = take(vtile);
    c.vp_lo = take(vtile);
    c.t = take((size_t)pb.B * pb.Hv * pb.NT * 8192);
    c.bytes = off;
    return c;
}

TcFwdSave tc_save_in(void* cache, const Problem& pb, float* o_raw) {
    const TcCache c = plan_tc_cache(pb);
    char* cb = static_cast<char*>(cache);
    TcFwdSave s{};
    s.s0 = reinterpret_cast<float*>(cb + c.s0);
    s.vp_hi = reinterpret_cast<__nv_bfloat16*>(cb + c.vp_hi);
    s.vp_lo = reinterpret_cast<__nv_bfloat16*>(cb + c.vp_lo);
    s.o_raw = o_raw;
    s.t = reinterpret_cast<uint8_t*>(cb + c.t);
    return s;
}

TcBwdWs plan_tc_bwd_ws(const Problem& pb, bool gqa_partials, bool caller_cache) {
    TcBwdWs w;
    const size_t nch = (size_t)pb.B * pb.Hv * pb.NT;
    const size_t st = nch * pb.dk * pb.dv * sizeof(float);
    const size_t tok = (size_t)pb.B * pb.T * pb.Hv * pb.dv * 2;
    const size_t part = (size_t)pb.B * pb.T * pb.Hv * pb.dk * sizeof(float);
    size_t off = 256;  // bytes [0, 256): device status word
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = al256(off + bytes);
        return o;
    };
    w.cache = caller_cache ? ~size_t(0) : take(plan_tc_cache(pb).bytes);
    w.dsc = take(st);
    w.ny_hi = take(tok);
    w.ny_lo = take(tok);
    w.dq_v = gqa_partials ? take(part) : ~size_t(0);
    w.dk_v = gqa_partials ? take(part) : ~size_t(0);
    w.flags = take((size_t)pb.B * pb.Hv * sizeof(int));
    w.sbuf = take(seq_sbuf_floats(pb) * sizeof(float));
    w.bytes = off;
    return w;
}

cudaError_t tc_chunk_bwd(const Problem& pb, const ChunkIO& io, Flags f, bool bf16_gates, bool direct,
                         const TcBwdWs& plan, void* ws, const void* cache, cudaStream_t st) {
    char* base = static_cast<char*>(ws);
    int* err = static_cast<int*>(ws);
    char* cb = cache ? static_cast<char*>(const_cast<void*>(cache)) : base + plan.cache;
    const TcFwdSave save = tc_save_in(cb, pb, nullptr);
    float* s0 = save.s0;
    auto* vph = save.vp_hi;
    auto* vpl = save.vp_lo;
    float* dsc = reinterpret_cast<float*>(base + plan.dsc);
    auto* nyh = reinterpret_cast<__nv_bfloat16*>(base + plan.ny_hi);
    auto* nyl = reinterpret_cast<__nv_bfloat16*>(base + plan.ny_lo);
    // dq, dk: the outputs when value heads map one to one on key heads, else per-value-head fp32
    // partials in the workspace, summed at the end
    void* dq_v = direct ? io.dq : base + plan.dq_v;
    void* dk_v = direct ? io.dk : base + plan.dk_v;
    const bool gbf = io.grad_type == 1;  // gradients returned in bf16
    int* flags = reinterpret_cast<int*>(base + plan.flags);  // zeroed by the caller

    const bool split = io.q_lo != nullptr;
    if (split && (f.apc || f.gpc || !io.k_lo || !io.v_lo)) return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (!cache) {
        // 1. forward in saving mode (no output, no final state)
        ChunkIO fio = io;
        fio.o = nullptr;
        fio.ht = nullptr;
        fio.z = nullptr;
        Flags ff = f;
        ff.gate = false;
        e = tc_chunk_fwd(pb, fio, ff, bf16_gates, err, st, &save, flags);
        if (e != cudaSuccess) return e;
    }

    // 2. maps: q, k, alpha, b, dO, -dY hi/lo, V' hi/lo (unused gate maps copy a valid one)
    CUtensorMap m[10];
    bool ok = make_map(&m[0], io.q, pb.B, pb.T, pb.Hk) && make_map(&m[1], io.k, pb.B, pb.T, pb.Hk) &&
              make_map(&m[4], io.dout, pb.B, pb.T, pb.Hv) && make_map(&m[5], nyh, pb.B, pb.T, pb.Hv) &&
              make_map(&m[6], nyl, pb.B, pb.T, pb.Hv) &&
              make_chunk_map(&m[7], vph, (long)pb.B * pb.Hv * pb.NT) &&
              make_chunk_map(&m[8], vpl, (long)pb.B * pb.Hv * pb.NT);
    m[2] = m[4];
    m[3] = m[4];
    if (ok && f.apc) ok = make_map(&m[2], io.alpha, pb.B, pb.T, pb.Hv);
    if (ok && f.gpc) ok = make_map(&m[3], io.b, pb.B, pb.T, pb.Hv);
    // split inputs: the lo halves of k and q take the alpha and b slots
    if (ok && split) ok = make_map(&m[2], io.k_lo, pb.B, pb.T, pb.Hk) && make_map(&m[3], io.q_lo, pb.B, pb.T, pb.Hk);
    if (!ok) return cudaErrorInvalidValue;
    // dO lo (the layer core's gradient of o as a bf16 hi/lo pair), else a copy of the dO map
    m[9] = m[4];
    if (io.dout_lo && !make_map(&m[9], io.dout_lo, pb.B, pb.T, pb.Hv)) return cudaErrorInvalidValue;
    const CUtensorMap ms[6] = {m[0], m[1], m[2], m[3], m[4], m[9]};

    tcbwd::scan::Params sp{};
    sp.pb = pb;
    sp.alpha = io.alpha;
    sp.b = io.b;
    sp.dht = io.dht;
    sp.dh0 = io.dh0;
    sp.dsc = dsc;
    sp.ny_hi = nyh;
    sp.ny_lo = nyl;
    sp.err = err;
    sp.flags = flags;
    sp.t_in = save.t;
    sp.do_lo = io.dout_lo ? 1 : 0;

    tcbwd::grad::Params gp{};
    gp.pb = pb;
    gp.alpha = io.alpha;
    gp.b = io.b;
    gp.w = io.w;
    gp.q = static_cast<const __nv_bfloat16*>(io.q);
    gp.k = static_cast<const __nv_bfloat16*>(io.k);
    gp.v = static_cast<const __nv_bfloat16*>(io.v);
    gp.q_lo = static_cast<const __nv_bfloat16*>(io.q_lo);
    gp.k_lo = static_cast<const __nv_bfloat16*>(io.k_lo);
    gp.v_lo = static_cast<const __nv_bfloat16*>(io.v_lo);
    gp.s0 = s0;
    gp.dsc = dsc;
    gp.dq = dq_v;
    gp.dk = dk_v;
    gp.dv = io.dv;
    gp.dalpha = io.dalpha;
    gp.db = io.db;
    gp.dw = io.dw;
    gp.direct = direct ? 1 : 0;
    gp.do_lo = io.dout_lo ? 1 : 0;
    gp.err = err;

    if (split && gbf) return cudaErrorInvalidValue;  // the layer core's form returns fp32 gradients
    e = pb.gate_logits ? tc_scan_dispatch<true>(ms, sp, f, split, bf16_gates, st)
                       : tc_scan_dispatch<false>(ms, sp, f, split, bf16_gates, st);
    if (e != cudaSuccess) return e;
    if (!gbf)
        e = pb.gate_logits ? tc_grad_dispatch<true, float, float>(m, gp, f, split, bf16_gates, st)
                           : tc_grad_dispatch<false, float, float>(m, gp, f, split, bf16_gates, st);
    else if (direct)
        e = pb.gate_logits ? tc_grad_dispatch<true, __nv_bfloat16, __nv_bfloat16>(m, gp, f, split, bf16_gates, st)
                           : tc_grad_dispatch<false, __nv_bfloat16, __nv_bfloat16>(m, gp, f, split, bf16_gates, st);
    else
        e = pb.gate_logits ? tc_grad_dispatch<true, __nv_bfloat16, float>(m, gp, f, split, bf16_gates, st)
                           : tc_grad_dispatch<false, __nv_bfloat16, float>(m, gp, f, split, bf16_gates, st);
    if (e != cudaSuccess) return e;
    // 3. pairs whose decay left the factors' range (marked by the scan): every gradient again,
    //    exactly; the pair's slice of the dS array holds its checkpoints
    e = seq_bwd(pb, io, f, false, !bf16_gates, flags, dq_v, dk_v, direct, dsc, (long)pb.NT * pb.dk * pb.dv,
                reinterpret_cast<float*>(base + plan.sbuf), st);
    if (e != cudaSuccess || direct) return e;

    // 4. GQA: sum the per-value-head dq, dk over the value heads of each key head
    GDN_TRY(gqa_reduce(pb, static_cast<const float*>(dq_v), io.dq, gbf, st));
    return gqa_reduce(pb, static_cast<const float*>(dk_v), io.dk, gbf, st);
}

}  // namespace gdn
