// C ABI of libgdn (see include/gdn.h): argument validation on the host, workspace carving and
// dispatch to the kernels.  No device memory is allocated here and nothing synchronises.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "gdn.h"
#include "launch.h"

namespace gdn {

namespace {
std::atomic<long long> g_launches{0};
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

thread_local std::string g_last_error;

gdn_status fail(gdn_status code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

gdn_status cuda_fail(cudaError_t e, const char* where) {
    return fail(GDN_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t elem_size(int dtype) { return dtype == GDN_F32 ? 4 : 2; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Buf {
    const void* p;
    size_t bytes;
    const char* name;
    size_t align = 16;  // required alignment of p (a strided input: its element size)
};

bool overlaps(const Buf& a, const Buf& b) {
    if (!a.p || !b.p || !a.bytes || !b.bytes) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

// Every output against every input and every other output.
gdn_status check_buffers(const Buf* in, int nin, const Buf* out, int nout) {
    for (int i = 0; i < nin; ++i)
        if (in[i].p && (reinterpret_cast<uintptr_t>(in[i].p) & (in[i].align - 1)))
            return fail(GDN_ERR_INVALID_ARG, "%s is not %zu-byte aligned", in[i].name, in[i].align);
    for (int i = 0; i < nout; ++i) {
        if (out[i].p && !aligned16(out[i].p))
            return fail(GDN_ERR_INVALID_ARG, "%s is not 16-byte aligned", out[i].name);
        for (int j = 0; j < nin; ++j)
            if (overlaps(out[i], in[j]))
                return fail(GDN_ERR_INVALID_ARG, "output %s overlaps input %s", out[i].name, in[j].name);
        for (int j = 0; j < i; ++j)
            if (overlaps(out[i], out[j]))
                return fail(GDN_ERR_INVALID_ARG, "outputs %s and %s overlap", out[i].name, out[j].name);
    }
    return GDN_OK;
}

// Shared checks of sizes, modes and dtypes.
gdn_status check_common(int64_t B, int64_t T, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                        const int32_t* head_map, int32_t apc, int32_t gpc, int32_t dtype,
                        int32_t gate_dtype) {
    if (B < 1 || T < 0 || Hk < 1 || Hv < 1)
        return fail(GDN_ERR_INVALID_ARG, "bad sizes B=%lld T=%lld Hk=%lld Hv=%lld", (long long)B,
                    (long long)T, (long long)Hk, (long long)Hv);
    if (dk != dv || (dk != 64 && dk != 128))
        return fail(GDN_ERR_UNSUPPORTED, "dk=%lld dv=%lld: supported are dk = dv in {64, 128}",
                    (long long)dk, (long long)dv);
    if (!head_map && Hv % Hk != 0)
        return fail(GDN_ERR_INVALID_ARG, "Hv=%lld is not a multiple of Hk=%lld and no head_map given",
                    (long long)Hv, (long long)Hk);
    if ((apc != 0 && apc != 1) || (gpc != 0 && gpc != 1))
        return fail(GDN_ERR_INVALID_ARG, "alpha_per_channel and gates_per_channel must be 0 or 1");
    if ((dtype != GDN_BF16 && dtype != GDN_F32) || (gate_dtype != GDN_BF16 && gate_dtype != GDN_F32))
        return fail(GDN_ERR_INVALID_ARG, "unknown dtype %d / gate_dtype %d", dtype, gate_dtype);
    if (dtype == GDN_F32 && gate_dtype != GDN_F32)
        return fail(GDN_ERR_UNSUPPORTED, "fp32 tensors need fp32 gates");
    if (B * T * (Hk > Hv ? Hk : Hv) * dk >= (int64_t(1) << 40) || B * T >= (int64_t(1) << 30))
        return fail(GDN_ERR_UNSUPPORTED, "problem too large for 32-bit token indices");
    return GDN_OK;
}

Problem make_problem(int64_t B, int64_t T, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                     float scale, const int32_t* head_map) {
    Problem pb{};
    pb.B = (int)B; pb.T = (int)T; pb.Hk = (int)Hk; pb.Hv = (int)Hv; pb.dk = (int)dk; pb.dv = (int)dv;
    pb.NT = (int)((T + kChunk - 1) / kChunk);
    pb.scale = scale;
    pb.head_map = head_map;
    return pb;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---- token strides (gdn_strides) ---------------------------------------------------------
// A token-major input of `rows` tokens of `row` elements whose tokens are `stride` elements apart
// (0: dense).  One that is not dense is copied into the workspace before the call's kernels run.
bool strided(int64_t stride, int64_t row) { return stride != 0 && stride != row; }

// The input as a buffer: from its first to its last element; a strided one needs only the
// alignment of its element type.
Buf tok(const void* p, size_t rows, int64_t row, int64_t stride, size_t es, const char* name) {
    const size_t step = (size_t)(stride ? stride : row);
    return Buf{p, p && rows ? ((rows - 1) * step + (size_t)row) * es : 0, name, strided(stride, row) ? es : 16};
}

gdn_status check_stride(int64_t stride, int64_t row, const char* name) {
    if (stride != 0 && (stride < row || stride > (int64_t(1) << 31)))
        return fail(GDN_ERR_INVALID_ARG, "token stride of %s is %lld: it must be 0 or in [%lld, 2^31]", name,
                    (long long)stride, (long long)row);
    return GDN_OK;
}

// One input of a call, for the copies: where the call reads its pointer, its row and stride.
struct StridedIn {
    const void** slot;
    int64_t row, stride;
    size_t es;
};

// Bytes of the dense copies of the strided inputs (each 256-byte aligned).
size_t pack_bytes(const StridedIn* in, int n, size_t rows) {
    size_t bytes = 0;
    for (int i = 0; i < n; ++i)
        if (*in[i].slot && strided(in[i].stride, in[i].row)) bytes += align256(rows * (size_t)in[i].row * in[i].es);
    return bytes;
}

// Copies every strided input into `dst` (the workspace past the call's own part) and points its
// slot at the copy.
cudaError_t pack_inputs(const StridedIn* in, int n, size_t rows, char* dst, cudaStream_t st) {
    for (int i = 0; i < n; ++i) {
        if (!*in[i].slot || !strided(in[i].stride, in[i].row)) continue;
        const long row_bytes = (long)(in[i].row * (int64_t)in[i].es);
        cudaError_t e = pack_rows(*in[i].slot, dst, (long)rows, row_bytes, (long)(in[i].stride * (int64_t)in[i].es), st);
        if (e != cudaSuccess) return e;
        *in[i].slot = dst;
        dst += align256(rows * (size_t)row_bytes);
    }
    return cudaSuccess;
}

// Gates as logits: the flag and alpha's per-head scale (grad: the scale's gradient, optional).
gdn_status check_logits(int32_t gate_logits, const float* alpha_scale, const float* grad_alpha_scale = nullptr) {
    if (gate_logits != 0 && gate_logits != 1) return fail(GDN_ERR_INVALID_ARG, "gate_logits must be 0 or 1");
    if (gate_logits && !alpha_scale) return fail(GDN_ERR_INVALID_ARG, "alpha_scale is required with gate_logits");
    if (!gate_logits && (alpha_scale || grad_alpha_scale))
        return fail(GDN_ERR_INVALID_ARG, "alpha_scale and grad_alpha_scale must be NULL without gate_logits");
    return GDN_OK;
}
void apply_logits(Problem& pb, int32_t gate_logits, const float* alpha_scale) {
    pb.gate_logits = gate_logits;
    pb.alpha_scale = gate_logits ? alpha_scale : nullptr;
}

int variant(int32_t dtype, int32_t gate_dtype) {
    if (dtype == GDN_F32) return 2;
    return gate_dtype == GDN_F32 ? 1 : 0;
}

bool identity_heads(const Problem& pb) { return pb.Hk == pb.Hv && pb.head_map == nullptr; }

}  // namespace

WsPlan plan_chunk_ws(const Problem& pb, bool bwd, bool gqa_partials) {
    WsPlan w{};
    const size_t nch = (size_t)pb.B * pb.Hv * pb.NT, C = kChunk, dk = pb.dk, dv = pb.dv;
    size_t off = 256;  // bytes [0, 256): device status word
    auto take = [&](size_t floats) {
        size_t o = off;
        off = align256(off + floats * sizeof(float));
        return o;
    };
    const size_t none = ~size_t(0);
    w.T = take(nch * C * C);
    w.P = take(nch * C * C);
    w.Eh = take(nch * C * dk);
    w.Qh = take(nch * C * dk);
    w.Kb = take(nch * C * dk);
    w.gam = take(nch * dk);
    w.Kt = bwd ? take(nch * C * dk) : none;
    w.Gm = bwd ? take(nch * C * dk) : none;
    w.S0 = bwd ? take(nch * dk * dv) : none;
    w.dSC = bwd ? take(nch * dk * dv) : none;
    w.V = bwd ? take(nch * C * dv) : none;
    w.Y = bwd ? take(nch * C * dv) : none;
    w.dV = bwd ? take(nch * C * dv) : none;
    w.dY = bwd ? take(nch * C * dv) : none;
    w.dbw = bwd ? take(nch * (dv / kDvTile) * C) : none;
    const size_t part = (size_t)pb.B * pb.T * pb.Hv * dk;
    w.dq_v = (bwd && gqa_partials) ? take(part) : none;
    w.dk_v = (bwd && gqa_partials) ? take(part) : none;
    w.flags = take((size_t)pb.B * pb.Hv);  // ints: pairs outside the decay range
    w.sbuf = bwd ? take(seq_sbuf_floats(pb)) : none;
    w.bytes = off;
    return w;
}

ChunkWs carve_chunk_ws(const WsPlan& w, void* base) {
    const size_t none = ~size_t(0);
    char* b = static_cast<char*>(base);
    auto at = [&](size_t o) { return o == none ? nullptr : reinterpret_cast<float*>(b + o); };
    ChunkWs ws;
    ws.T = at(w.T); ws.P = at(w.P); ws.Eh = at(w.Eh); ws.Qh = at(w.Qh); ws.Kb = at(w.Kb);
    ws.Kt = at(w.Kt); ws.Gm = at(w.Gm); ws.gam = at(w.gam); ws.S0 = at(w.S0); ws.dSC = at(w.dSC);
    ws.V = at(w.V); ws.Y = at(w.Y); ws.dV = at(w.dV); ws.dY = at(w.dY); ws.dbw = at(w.dbw);
    ws.dq_v = at(w.dq_v); ws.dk_v = at(w.dk_v);
    ws.flags = reinterpret_cast<int*>(at(w.flags));
    ws.sbuf = at(w.sbuf);
    return ws;
}

}  // namespace gdn

using namespace gdn;

namespace {

gdn_status check_fwd(const gdn_fwd_args* a, bool need_o = true) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    gdn_status s = check_common(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->head_map,
                                a->alpha_per_channel, a->gates_per_channel, a->dtype, a->gate_dtype);
    if (s) return s;
    if (a->T > 0 && (!a->q || !a->k || !a->v || !a->alpha || !a->b || (need_o && !a->o)))
        return fail(GDN_ERR_INVALID_ARG, need_o ? "q, k, v, alpha, b and o are required"
                                                : "q, k, v, alpha and b are required");
    if (a->gates_per_channel && a->T > 0 && !a->w)
        return fail(GDN_ERR_INVALID_ARG, "w is required when gates_per_channel = 1");
    if (!a->gates_per_channel && a->w)
        return fail(GDN_ERR_INVALID_ARG, "w must be NULL for scalar gates (b holds beta)");
    const size_t es = elem_size(a->dtype), gs = elem_size(a->gate_dtype);
    const size_t BT = (size_t)(a->B * a->T);
    const gdn_strides& sd = a->strides;
    const int64_t ra = a->Hv * (a->alpha_per_channel ? a->dk : 1), rb = a->Hv * (a->gates_per_channel ? a->dk : 1);
    if ((s = check_stride(sd.q, a->Hk * a->dk, "q")) || (s = check_stride(sd.k, a->Hk * a->dk, "k")) ||
        (s = check_stride(sd.v, a->Hv * a->dv, "v")) || (s = check_stride(sd.alpha, ra, "alpha")) ||
        (s = check_stride(sd.b, rb, "b")) || (s = check_stride(sd.w, a->Hv * a->dv, "w")) ||
        (s = check_stride(sd.z, a->Hv * a->dv, "z")))
        return s;
    const Buf in[] = {
        tok(a->q, BT, a->Hk * a->dk, sd.q, es, "q"),
        tok(a->k, BT, a->Hk * a->dk, sd.k, es, "k"),
        tok(a->v, BT, a->Hv * a->dv, sd.v, es, "v"),
        tok(a->alpha, BT, ra, sd.alpha, gs, "alpha"),
        tok(a->b, BT, rb, sd.b, gs, "b"),
        tok(a->w, BT, a->Hv * a->dv, sd.w, gs, "w"),
        {a->h0, (size_t)(a->B * a->Hv * a->dk * a->dv) * 4, "h0"},
        tok(a->z, BT, a->Hv * a->dv, sd.z, es, "z"),
        {a->head_map, (size_t)a->Hv * 4, "head_map"},
        {a->alpha_scale, (size_t)a->Hv * 4, "alpha_scale"},
    };
    if (a->out_f32 != 0 && a->out_f32 != 1) return fail(GDN_ERR_INVALID_ARG, "out_f32 must be 0 or 1");
    if ((s = check_logits(a->gate_logits, a->alpha_scale))) return s;
    const Buf out[] = {
        {a->o, BT * a->Hv * a->dv * (a->out_f32 ? 4 : es), "o"},
        {a->ht, (size_t)(a->B * a->Hv * a->dk * a->dv) * 4, "ht"},
        {a->bwd_cache, a->bwd_cache ? a->bwd_cache_bytes : 0, "bwd_cache"},
    };
    if (a->bwd_cache && (reinterpret_cast<uintptr_t>(a->bwd_cache) & 255u))
        return fail(GDN_ERR_INVALID_ARG, "bwd_cache is not 256-byte aligned");
    return check_buffers(in, 10, out, 3);
}

gdn_status check_bwd(const gdn_bwd_args* a) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    gdn_status s = check_common(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->head_map,
                                a->alpha_per_channel, a->gates_per_channel, a->dtype, a->gate_dtype);
    if (s) return s;
    if (a->T > 0 && (!a->q || !a->k || !a->v || !a->alpha || !a->b || !a->grad_o || !a->grad_q ||
                     !a->grad_k || !a->grad_v || !a->grad_alpha || !a->grad_b))
        return fail(GDN_ERR_INVALID_ARG, "q, k, v, alpha, b, grad_o and grad_q/k/v/alpha/b are required");
    if (a->gates_per_channel && a->T > 0 && (!a->w || !a->grad_w))
        return fail(GDN_ERR_INVALID_ARG, "w and grad_w are required when gates_per_channel = 1");
    if (!a->gates_per_channel && (a->w || a->grad_w))
        return fail(GDN_ERR_INVALID_ARG, "w and grad_w must be NULL for scalar gates");
    const size_t es = elem_size(a->dtype), gs = elem_size(a->gate_dtype);
    const size_t BT = (size_t)(a->B * a->T);
    const size_t st = (size_t)(a->B * a->Hv * a->dk * a->dv) * 4;
    const size_t na = BT * a->Hv * (a->alpha_per_channel ? a->dk : 1) * gs;
    const size_t nb = BT * a->Hv * (a->gates_per_channel ? a->dk : 1) * gs;
    const gdn_strides& sd = a->strides;
    const int64_t ra = a->Hv * (a->alpha_per_channel ? a->dk : 1), rb = a->Hv * (a->gates_per_channel ? a->dk : 1);
    if ((s = check_stride(sd.q, a->Hk * a->dk, "q")) || (s = check_stride(sd.k, a->Hk * a->dk, "k")) ||
        (s = check_stride(sd.v, a->Hv * a->dv, "v")) || (s = check_stride(sd.alpha, ra, "alpha")) ||
        (s = check_stride(sd.b, rb, "b")) || (s = check_stride(sd.w, a->Hv * a->dv, "w")))
        return s;
    if (sd.z != 0) return fail(GDN_ERR_INVALID_ARG, "strides.z must be 0: the backward takes no z");
    const Buf in[] = {
        tok(a->q, BT, a->Hk * a->dk, sd.q, es, "q"), tok(a->k, BT, a->Hk * a->dk, sd.k, es, "k"),
        tok(a->v, BT, a->Hv * a->dv, sd.v, es, "v"), tok(a->alpha, BT, ra, sd.alpha, gs, "alpha"),
        tok(a->b, BT, rb, sd.b, gs, "b"), tok(a->w, BT, a->Hv * a->dv, sd.w, gs, "w"), {a->h0, st, "h0"},
        {a->head_map, (size_t)a->Hv * 4, "head_map"},
        {a->grad_o, BT * a->Hv * a->dv * es, "grad_o"}, {a->grad_ht, st, "grad_ht"},
        {a->fwd_cache, a->fwd_cache ? a->fwd_cache_bytes : 0, "fwd_cache"},
        {a->alpha_scale, (size_t)a->Hv * 4, "alpha_scale"},
    };
    if ((s = check_logits(a->gate_logits, a->alpha_scale, a->grad_alpha_scale))) return s;
    if (a->fwd_cache && (reinterpret_cast<uintptr_t>(a->fwd_cache) & 255u))
        return fail(GDN_ERR_INVALID_ARG, "fwd_cache is not 256-byte aligned");
    if (a->grads_in_dtype != 0 && a->grads_in_dtype != 1)
        return fail(GDN_ERR_INVALID_ARG, "grads_in_dtype must be 0 or 1");
    // element sizes of the gradients: fp32, or the inputs' dtypes
    const size_t ge = a->grads_in_dtype ? es : 4, gg = a->grads_in_dtype ? gs : 4;
    const size_t nag = na / gs * gg, nbg = nb / gs * gg;
    const Buf out[] = {
        {a->grad_q, BT * a->Hk * a->dk * ge, "grad_q"}, {a->grad_k, BT * a->Hk * a->dk * ge, "grad_k"},
        {a->grad_v, BT * a->Hv * a->dv * ge, "grad_v"}, {a->grad_alpha, nag, "grad_alpha"},
        {a->grad_b, nbg, "grad_b"}, {a->grad_w, BT * a->Hv * a->dv * gg, "grad_w"}, {a->grad_h0, st, "grad_h0"},
        {a->grad_alpha_scale, (size_t)a->Hv * 4, "grad_alpha_scale"},
    };
    return check_buffers(in, 12, out, 8);
}

gdn_status check_workspace(void* ws, size_t have, size_t need) {
    if (need == 0) return GDN_OK;
    if (!ws) return fail(GDN_ERR_WORKSPACE, "workspace is NULL, %zu bytes needed", need);
    if (have < need) return fail(GDN_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", have, need);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(GDN_ERR_WORKSPACE, "workspace is not 256-byte aligned");
    return GDN_OK;
}

ChunkIO io_from(const gdn_fwd_args* a) {
    ChunkIO io{};
    io.q = a->q; io.k = a->k; io.v = a->v; io.alpha = a->alpha; io.b = a->b; io.w = a->w;
    io.z = a->z; io.h0 = a->h0; io.o = a->o; io.ht = a->ht; io.o_type = a->out_f32 ? 1 : 0;
    io.z_bf16 = 0;
    return io;
}

// The token-major inputs of a forward, a backward and a layer call, for the copies of the strided
// ones; `p` is the call's own copy of its arguments, whose pointers the copies replace.
int fwd_inputs(gdn_fwd_args* p, StridedIn* in) {
    const size_t es = elem_size(p->dtype), gs = elem_size(p->gate_dtype);
    const int64_t ra = p->Hv * (p->alpha_per_channel ? p->dk : 1), rb = p->Hv * (p->gates_per_channel ? p->dk : 1);
    in[0] = {&p->q, p->Hk * p->dk, p->strides.q, es};
    in[1] = {&p->k, p->Hk * p->dk, p->strides.k, es};
    in[2] = {&p->v, p->Hv * p->dv, p->strides.v, es};
    in[3] = {&p->alpha, ra, p->strides.alpha, gs};
    in[4] = {&p->b, rb, p->strides.b, gs};
    in[5] = {&p->w, p->Hv * p->dv, p->strides.w, gs};
    in[6] = {&p->z, p->Hv * p->dv, p->strides.z, es};
    return 7;
}
int bwd_inputs(gdn_bwd_args* p, StridedIn* in) {
    const size_t es = elem_size(p->dtype), gs = elem_size(p->gate_dtype);
    const int64_t ra = p->Hv * (p->alpha_per_channel ? p->dk : 1), rb = p->Hv * (p->gates_per_channel ? p->dk : 1);
    in[0] = {&p->q, p->Hk * p->dk, p->strides.q, es};
    in[1] = {&p->k, p->Hk * p->dk, p->strides.k, es};
    in[2] = {&p->v, p->Hv * p->dv, p->strides.v, es};
    in[3] = {&p->alpha, ra, p->strides.alpha, gs};
    in[4] = {&p->b, rb, p->strides.b, gs};
    in[5] = {&p->w, p->Hv * p->dv, p->strides.w, gs};
    return 6;
}
template <class LA>
int layer_inputs(LA* p, StridedIn* in) {
    const size_t es = elem_size(p->dtype), gs = elem_size(p->gate_dtype);
    const int64_t ra = p->Hv * (p->alpha_per_channel ? p->dk : 1), rb = p->Hv * (p->gates_per_channel ? p->dk : 1);
    in[0] = {&p->xq, p->Hk * p->dk, p->strides.q, es};
    in[1] = {&p->xk, p->Hk * p->dk, p->strides.k, es};
    in[2] = {&p->xv, p->Hv * p->dv, p->strides.v, es};
    in[3] = {&p->alpha, ra, p->strides.alpha, gs};
    in[4] = {&p->b, rb, p->strides.b, gs};
    in[5] = {&p->w, p->Hv * p->dv, p->strides.w, gs};
    in[6] = {&p->z, p->Hv * p->dv, p->strides.z, es};
    return 7;
}
template <class A, int (*LIST)(A*, StridedIn*)>
size_t args_pack_bytes(const A* a) {
    A p = *a;
    StridedIn in[7];
    const int n = LIST(&p, in);
    return pack_bytes(in, n, (size_t)(a->B * a->T));
}
// Workspace of a call's own part plus the copies of its strided inputs after it.
size_t with_copies(size_t own, size_t copies) { return copies ? align256(own) + copies : own; }

// Validates the workspace for a call's own part and its copies, then copies the strided inputs
// of *a past its own part and points *a (the call's copy of its arguments) at them.
template <class A>
gdn_status copy_strided(A* p, int (*list)(A*, StridedIn*), void* ws, size_t ws_bytes, size_t own, cudaStream_t st,
                        const char* who) {
    StridedIn in[7];
    const int n = list(p, in);
    const size_t rows = (size_t)(p->B * p->T), copies = pack_bytes(in, n, rows);
    gdn_status s = check_workspace(ws, ws_bytes, with_copies(own, copies));
    if (s || !copies) return s;
    cudaError_t e = pack_inputs(in, n, rows, static_cast<char*>(ws) + align256(own), st);
    if (e != cudaSuccess) return cuda_fail(e, who);
    p->strides = gdn_strides{};
    return GDN_OK;
}

// Status word at the start of every workspace, cleared at the start of each call.
int* ws_status(void* ws) { return static_cast<int*>(ws); }

// The flag array of the pairs outside the chunk form's decay range, cleared at the start of a call.
cudaError_t clear_flags(int* flags, const Problem& pb, cudaStream_t st) {
    return cudaMemsetAsync(flags, 0, (size_t)pb.B * pb.Hv * sizeof(int), st);
}

// The tensor-core forward's workspace: the status word, then the flag array.
size_t tc_fwd_ws_bytes(const Problem& pb) { return 256 + align256((size_t)pb.B * pb.Hv * sizeof(int)); }
int* tc_fwd_flags(void* ws) { return reinterpret_cast<int*>(static_cast<char*>(ws) + 256); }

cudaError_t run_fwd(int var, const Problem& pb, const ChunkIO& io, const ChunkWs& ws, Flags f,
                    cudaStream_t st) {
    switch (var) {
        case 0: return bf16_chunk_fwd(pb, io, ws, f, st);
        case 1: return bf16_f32g_chunk_fwd(pb, io, ws, f, st);
        case 3: return f32_bf16g_chunk_fwd(pb, io, ws, f, st);
        default: return f32_chunk_fwd(pb, io, ws, f, st);
    }
}

// ht = h0 (or zeros) when there is no token to process.
gdn_status copy_state(float* dst, const float* src, size_t bytes, cudaStream_t st, const char* what) {
    if (!dst) return GDN_OK;
    cudaError_t e = src ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st)
                        : cudaMemsetAsync(dst, 0, bytes, st);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e, what);
}

}  // namespace

namespace gdn {
// For the other translation units of the C ABI.
gdn_status check_fwd_args(const gdn_fwd_args* a) { return check_fwd(a); }
gdn_status record_error(gdn_status code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace gdn

extern "C" {

static bool fwd_uses_tensor_cores(const gdn_fwd_args* a, const Problem& pb) {
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, a->z != nullptr};
    return tc_fwd_eligible(pb, a->dtype == GDN_BF16, a->gate_dtype == GDN_BF16, f);
}

size_t gdn_chunk_fwd_cache_size(const gdn_fwd_args* a) {
    if (!a || a->B < 1 || a->T < 1 || a->Hv < 1 || a->dk < 1 || a->dv < 1) return 0;
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    return fwd_uses_tensor_cores(a, pb) ? plan_tc_cache(pb).bytes : 0;
}

// The forward's own workspace (without the copies of strided inputs).
static size_t fwd_own_ws(const gdn_fwd_args* a) {
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    if (fwd_uses_tensor_cores(a, pb)) return tc_fwd_ws_bytes(pb);
    return plan_chunk_ws(pb, false, false).bytes;
}

size_t gdn_chunk_fwd_workspace_size(const gdn_fwd_args* a) {
    if (!a || a->B < 1 || a->T < 1 || a->Hv < 1 || a->dk < 1 || a->dv < 1) return 0;
    return with_copies(fwd_own_ws(a), args_pack_bytes<gdn_fwd_args, fwd_inputs>(a));
}

}  // extern "C"

// The chunk forward on validated arguments (o may be NULL: no output is written).
static gdn_status chunk_fwd_core(const gdn_fwd_args* a, void* workspace, size_t workspace_bytes,
                                 gdn_stream stream) {
    gdn_status s = GDN_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t sbytes = (size_t)(a->B * a->Hv * a->dk * a->dv) * 4;
    if (a->T == 0) return copy_state(a->ht, a->h0, sbytes, st, "gdn_chunk_fwd");
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    apply_logits(pb, a->gate_logits, a->alpha_scale);
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, a->z != nullptr};
    const bool tc = fwd_uses_tensor_cores(a, pb);
    if (a->bwd_cache) {
        if (!tc)
            return fail(GDN_ERR_UNSUPPORTED, "bwd_cache: only the tensor-core path (bf16, dk = dv = 128) keeps a cache");
        if (a->bwd_cache_bytes < plan_tc_cache(pb).bytes)
            return fail(GDN_ERR_WORKSPACE, "bwd_cache has %zu bytes, %zu needed", a->bwd_cache_bytes,
                        plan_tc_cache(pb).bytes);
    }
    WsPlan plan = plan_chunk_ws(pb, false, false);
    // the workspace, then the dense copies of strided inputs, which the rest reads instead
    gdn_fwd_args pa = *a;
    if ((s = copy_strided(&pa, fwd_inputs, workspace, workspace_bytes, tc ? tc_fwd_ws_bytes(pb) : plan.bytes, st,
                          "gdn_chunk_fwd (strided inputs)")))
        return s;
    a = &pa;
    int* flags = tc ? tc_fwd_flags(workspace) : carve_chunk_ws(plan, workspace).flags;
    cudaError_t e = cudaMemsetAsync(ws_status(workspace), 0, sizeof(int), st);
    if (e == cudaSuccess) e = clear_flags(flags, pb, st);
    if (e == cudaSuccess) {
        TcFwdSave save{};
        if (a->bwd_cache) save = tc_save_in(a->bwd_cache, pb, nullptr);
        if (tc)
            e = tc_chunk_fwd(pb, io_from(a), f, a->gate_dtype == GDN_BF16, ws_status(workspace), st,
                             a->bwd_cache ? &save : nullptr, flags);
        else e = run_fwd(variant(a->dtype, a->gate_dtype), pb, io_from(a), carve_chunk_ws(plan, workspace), f, st);
    }
    return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_chunk_fwd");
}

extern "C" {

gdn_status gdn_chunk_fwd(const gdn_fwd_args* a, void* workspace, size_t workspace_bytes,
                         gdn_stream stream) {
    gdn_status s = check_fwd(a);
    if (s) return s;
    return chunk_fwd_core(a, workspace, workspace_bytes, stream);
}

// Segment map: the forward from a zero state (N = ht, o optional), then the forward from the
// identity with the writes zeroed (v = 0), whose final state is M.
// Its own part: the forward's workspace, the identity states, the zero v; then the copies.
static size_t segment_map_own_ws(const gdn_fwd_args* a) {
    const size_t es = elem_size(a->dtype);
    return align256(fwd_own_ws(a)) + align256((size_t)(a->B * a->Hv * a->dk * a->dk) * 4) +
           align256((size_t)(a->B * a->T * a->Hv * a->dv) * es);
}

size_t gdn_segment_map_workspace_size(const gdn_fwd_args* a) {
    if (!a || a->B < 1 || a->T < 1 || a->Hv < 1 || a->dk < 1 || a->dv < 1) return 0;
    return with_copies(segment_map_own_ws(a), args_pack_bytes<gdn_fwd_args, fwd_inputs>(a));
}

gdn_status gdn_segment_map(const gdn_fwd_args* a, float* M, void* workspace, size_t workspace_bytes,
                           gdn_stream stream) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    if (a->h0 || a->z || a->bwd_cache)
        return fail(GDN_ERR_INVALID_ARG, "gdn_segment_map: h0, z and bwd_cache must be NULL");
    if (!a->ht || !M) return fail(GDN_ERR_INVALID_ARG, "gdn_segment_map: ht (receives N) and M are required");
    // validated as a forward whose o is optional; M must not overlap any input or output
    gdn_status s = check_fwd(a, false);
    if (s) return s;
    gdn_fwd_args x = *a;
    const size_t es = elem_size(a->dtype), gs = elem_size(a->gate_dtype), BT = (size_t)(a->B * a->T);
    const size_t mbytes = (size_t)(a->B * a->Hv * a->dk * a->dk) * 4;
    const gdn_strides& sd = a->strides;
    const Buf in[] = {tok(a->q, BT, a->Hk * a->dk, sd.q, es, "q"), tok(a->k, BT, a->Hk * a->dk, sd.k, es, "k"),
                      tok(a->v, BT, a->Hv * a->dv, sd.v, es, "v"),
                      tok(a->alpha, BT, a->Hv * (a->alpha_per_channel ? a->dk : 1), sd.alpha, gs, "alpha"),
                      tok(a->b, BT, a->Hv * (a->gates_per_channel ? a->dk : 1), sd.b, gs, "b"),
                      tok(a->w, BT, a->Hv * a->dv, sd.w, gs, "w"), {a->head_map, (size_t)a->Hv * 4, "head_map"}};
    const Buf out[] = {{M, mbytes, "M"}, {a->ht, (size_t)(a->B * a->Hv * a->dk * a->dv) * 4, "ht"},
                       {a->o, a->o ? BT * a->Hv * a->dv * (a->out_f32 ? 4 : es) : 0, "o"}};
    if ((s = check_buffers(in, 7, out, 3))) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (a->T > 0 && (s = copy_strided(&x, fwd_inputs, workspace, workspace_bytes, segment_map_own_ws(a), st,
                                      "gdn_segment_map (strided inputs)")))
        return s;
    if (a->T == 0) {
        cudaError_t e = cudaMemsetAsync(a->ht, 0, (size_t)(a->B * a->Hv * a->dk * a->dv) * 4, st);
        if (e == cudaSuccess) e = identity_states(M, a->B * a->Hv, (int)a->dk, st);
        return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_segment_map");
    }
    char* base = static_cast<char*>(workspace);
    const size_t fw = align256(fwd_own_ws(a));
    float* ident = reinterpret_cast<float*>(base + fw);
    void* zero_v = base + fw + align256(mbytes);
    // N: the segment from a zero state
    if ((s = chunk_fwd_core(&x, workspace, fw, stream))) return s;
    // M: from the identity, with nothing written (z = w .* v = 0)
    cudaError_t e = identity_states(ident, a->B * a->Hv, (int)a->dk, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(zero_v, 0, BT * a->Hv * a->dv * es, st);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_segment_map");
    gdn_fwd_args y = x;
    y.v = zero_v;
    y.h0 = ident;
    y.ht = M;
    y.o = nullptr;
    return chunk_fwd_core(&y, workspace, fw, stream);
}

gdn_status gdn_state_compose(const float* M, const float* N, const float* S_in, float* S_out, int64_t pairs,
                             int64_t dk, int64_t dv, int32_t transpose, gdn_stream stream) {
    if (!M || !S_out) return fail(GDN_ERR_INVALID_ARG, "gdn_state_compose: M and S_out are required");
    if (pairs < 1) return fail(GDN_ERR_INVALID_ARG, "gdn_state_compose: pairs must be >= 1");
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128))
        return fail(GDN_ERR_UNSUPPORTED, "gdn_state_compose: dk, dv must be 64 or 128");
    if (transpose != 0 && transpose != 1) return fail(GDN_ERR_INVALID_ARG, "transpose must be 0 or 1");
    if (transpose && dk != dv) return fail(GDN_ERR_INVALID_ARG, "gdn_state_compose: M^T needs dk == dv");
    const size_t st = (size_t)(pairs * dk * dv) * 4;
    const Buf in[] = {{M, (size_t)(pairs * dk * dk) * 4, "M"}, {N, N ? st : 0, "N"}, {S_in, S_in ? st : 0, "S_in"}};
    const Buf out[] = {{S_out, st, "S_out"}};
    gdn_status s = check_buffers(in, 3, out, 1);
    if (s) return s;
    cudaError_t e = compose_states(M, N, S_in, S_out, (long)pairs, (int)dk, (int)dv, transpose != 0,
                                   static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_state_compose");
}

static bool bwd_uses_tensor_cores(const gdn_bwd_args* a, const Problem& pb) {
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, false};
    return tc_fwd_eligible(pb, a->dtype == GDN_BF16, a->gate_dtype == GDN_BF16, f);
}

size_t gdn_chunk_bwd_workspace_size(const gdn_bwd_args* a) {
    if (!a || a->B < 1 || a->T < 1 || a->Hv < 1 || a->dk < 1 || a->dv < 1) return 0;
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    const size_t own = bwd_uses_tensor_cores(a, pb) ? plan_tc_bwd_ws(pb, !identity_heads(pb), a->fwd_cache != nullptr).bytes
                                                    : plan_chunk_ws(pb, true, !identity_heads(pb)).bytes;
    return with_copies(own, args_pack_bytes<gdn_bwd_args, bwd_inputs>(a));
}

gdn_status gdn_chunk_bwd(const gdn_bwd_args* a, void* workspace, size_t workspace_bytes,
                         gdn_stream stream) {
    gdn_status s = check_bwd(a);
    if (s) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t sbytes = (size_t)(a->B * a->Hv * a->dk * a->dv) * 4;
    if (a->T == 0) {
        if (a->grad_alpha_scale) {
            cudaError_t e = cudaMemsetAsync(a->grad_alpha_scale, 0, (size_t)a->Hv * 4, st);
            if (e != cudaSuccess) return cuda_fail(e, "gdn_chunk_bwd");
        }
        return copy_state(a->grad_h0, a->grad_ht, sbytes, st, "gdn_chunk_bwd");
    }
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    apply_logits(pb, a->gate_logits, a->alpha_scale);
    const bool direct = identity_heads(pb);
    const bool tc = bwd_uses_tensor_cores(a, pb);
    WsPlan plan = plan_chunk_ws(pb, true, !direct);
    if (a->fwd_cache) {
        if (!tc) return fail(GDN_ERR_UNSUPPORTED, "fwd_cache: only the tensor-core path keeps a forward cache");
        if (a->fwd_cache_bytes < plan_tc_cache(pb).bytes)
            return fail(GDN_ERR_INVALID_ARG, "fwd_cache has %zu bytes, %zu needed", a->fwd_cache_bytes,
                        plan_tc_cache(pb).bytes);
    }
    // gradients in bf16: written by the tensor-core kernels (the CUDA-core backward writes fp32)
    const bool grad_bf16 = a->grads_in_dtype && a->dtype == GDN_BF16;
    if (grad_bf16 && !tc)
        return fail(GDN_ERR_UNSUPPORTED, "grads_in_dtype with bf16 inputs: only the tensor-core backward (dk = dv = "
                                         "128, bf16 channel gates) returns bf16 gradients");
    TcBwdWs tplan = tc ? plan_tc_bwd_ws(pb, !direct, a->fwd_cache != nullptr) : TcBwdWs{};
    // the workspace, then the dense copies of strided inputs, which the rest reads instead
    gdn_bwd_args pa = *a;
    if ((s = copy_strided(&pa, bwd_inputs, workspace, workspace_bytes, tc ? tplan.bytes : plan.bytes, st,
                          "gdn_chunk_bwd (strided inputs)")))
        return s;
    a = &pa;
    ChunkIO io{};
    io.q = a->q; io.k = a->k; io.v = a->v; io.alpha = a->alpha; io.b = a->b; io.w = a->w;
    io.h0 = a->h0; io.dout = a->grad_o; io.dht = a->grad_ht; io.dq = a->grad_q; io.dk = a->grad_k;
    io.dv = a->grad_v; io.dalpha = a->grad_alpha; io.db = a->grad_b; io.dw = a->grad_w;
    io.dh0 = a->grad_h0;
    io.grad_type = grad_bf16 ? 1 : 0;
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, false};
    cudaError_t e = cudaMemsetAsync(ws_status(workspace), 0, sizeof(int), st);
    if (e == cudaSuccess)
        e = clear_flags(tc ? reinterpret_cast<int*>(static_cast<char*>(workspace) + tplan.flags)
                           : carve_chunk_ws(plan, workspace).flags, pb, st);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_chunk_bwd");
    if (tc) {
        e = tc_chunk_bwd(pb, io, f, a->gate_dtype == GDN_BF16, direct, tplan, workspace, a->fwd_cache, st);
    } else {
        ChunkWs ws = carve_chunk_ws(plan, workspace);
        switch (variant(a->dtype, a->gate_dtype)) {
            case 0: e = bf16_chunk_bwd(pb, io, ws, f, direct, st); break;
            case 1: e = bf16_f32g_chunk_bwd(pb, io, ws, f, direct, st); break;
            default: e = f32_chunk_bwd(pb, io, ws, f, direct, st); break;
        }
    }
    // gates as logits: the gradients of the gates become those of their logits
    if (e == cudaSuccess && pb.gate_logits)
        e = gate_logit_grads(pb, f, a->gate_dtype == GDN_F32, a->alpha, a->b, a->w, a->grad_alpha, a->grad_b,
                             a->grad_w, grad_bf16 && a->gate_dtype == GDN_BF16, a->grad_alpha_scale, st);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_chunk_bwd");
}

gdn_status gdn_decode_step(const gdn_decode_args* a, gdn_stream stream) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    gdn_status s = check_common(a->N, 1, a->Hk, a->Hv, a->dk, a->dv, a->head_map,
                                a->alpha_per_channel, a->gates_per_channel, a->dtype, a->gate_dtype);
    if (s) return s;
    if (!a->q || !a->k || !a->v || !a->alpha || !a->b || !a->state || !a->o)
        return fail(GDN_ERR_INVALID_ARG, "q, k, v, alpha, b, state and o are required");
    if (a->gates_per_channel ? !a->w : a->w != nullptr)
        return fail(GDN_ERR_INVALID_ARG, "w is required with channel gates and must be NULL otherwise");
    if (a->conv_state && !a->conv_w)
        return fail(GDN_ERR_INVALID_ARG, "conv_w is required with conv_state");
    const size_t es = elem_size(a->dtype), gs = elem_size(a->gate_dtype), N = (size_t)a->N;
    const size_t cch = (size_t)(2 * a->Hk * a->dk + a->Hv * a->dv);
    const size_t st = N * a->Hv * a->dk * a->dv * 4;
    // per-sequence strides (read in place; the kernels load one element at a time)
    const gdn_strides& sd = a->strides;
    const int64_t rq = a->Hk * a->dk, rv = a->Hv * a->dv;
    const int64_t ra = a->Hv * (a->alpha_per_channel ? a->dk : 1), rb = a->Hv * (a->gates_per_channel ? a->dk : 1);
    if ((s = check_stride(sd.q, rq, "q")) || (s = check_stride(sd.k, rq, "k")) || (s = check_stride(sd.v, rv, "v")) ||
        (s = check_stride(sd.alpha, ra, "alpha")) || (s = check_stride(sd.b, rb, "b")) ||
        (s = check_stride(sd.w, rv, "w")) || (s = check_stride(sd.z, rv, "z")))
        return s;
    const Buf in[] = {
        tok(a->q, N, rq, sd.q, es, "q"), tok(a->k, N, rq, sd.k, es, "k"), tok(a->v, N, rv, sd.v, es, "v"),
        tok(a->alpha, N, ra, sd.alpha, gs, "alpha"), tok(a->b, N, rb, sd.b, gs, "b"),
        tok(a->w, N, rv, sd.w, gs, "w"), {a->head_map, (size_t)a->Hv * 4, "head_map"},
        {a->conv_w, cch * 4 * es, "conv_w"}, tok(a->z, N, rv, sd.z, es, "z"),
    };
    if (a->out_f32 != 0 && a->out_f32 != 1) return fail(GDN_ERR_INVALID_ARG, "out_f32 must be 0 or 1");
    const Buf out[] = {
        {a->o, N * a->Hv * a->dv * (a->out_f32 ? 4 : es), "o"}, {a->state, st, "state"},
        {a->conv_state, a->conv_state ? N * cch * 3 * es : 0, "conv_state"},
    };
    if ((s = check_buffers(in, 9, out, 3))) return s;
    DecodeParams p{};
    p.q = a->q; p.k = a->k; p.v = a->v; p.alpha = a->alpha; p.b = a->b; p.w = a->w;
    p.state = a->state; p.o = a->o; p.o_f32 = a->out_f32; p.head_map = a->head_map; p.conv_state = a->conv_state;
    p.conv_w = a->conv_w; p.z = a->z;
    p.sq = sd.q ? sd.q : rq; p.sk = sd.k ? sd.k : rq; p.sv = sd.v ? sd.v : rv;
    p.sa = sd.alpha ? sd.alpha : ra; p.sb = sd.b ? sd.b : rb; p.sw = sd.w ? sd.w : rv; p.sz = sd.z ? sd.z : rv;
    p.N = (int)a->N; p.Hk = (int)a->Hk; p.Hv = (int)a->Hv; p.dk = (int)a->dk; p.dv = (int)a->dv;
    p.scale = a->scale;
    if ((s = check_logits(a->gate_logits, a->alpha_scale))) return s;
    p.gate_logits = a->gate_logits;
    p.alpha_scale = a->gate_logits ? a->alpha_scale : nullptr;
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, a->z != nullptr};
    cudaStream_t sm = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch (variant(a->dtype, a->gate_dtype)) {
        case 0: e = bf16_decode(p, f, sm); break;
        case 1: e = bf16_f32g_decode(p, f, sm); break;
        default: e = f32_decode(p, f, sm); break;
    }
    return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_decode_step");
}

// The layer backward's tensor-core form: bf16 tensors, d = 128, scalar gates, no initial state.
// With an initial state h0 the first tokens' dxk is tens of times its RMS (the conv sees one tap
// there, and the L2 norm's backward divides by a small norm): the tensor-core backward's ~1e-3
// relative error there exceeds the 2e-2-of-RMS budget, so such calls keep the fp32 CUDA-core form.
static bool layer_tc_form(int32_t dtype, int64_t dk, int64_t dv, int32_t apc, int32_t gpc, const float* h0) {
    return dtype == GDN_BF16 && dk == 128 && dv == 128 && !apc && !gpc && h0 == nullptr;
}

// The layer forward's backward cache (tensor-core form only), byte offsets from its start: the
// conv results as bf16 hi/lo pairs (q, k, v), the recurrence's output before the gate (fp32),
// then the chunk forward cache (states, V').
struct LayerCache {
    size_t q, k, v, o, tc, bytes;
};
static LayerCache plan_layer_cache(const Problem& pb) {
    LayerCache c{};
    const size_t BT = (size_t)pb.B * pb.T, qn = BT * pb.Hk * pb.dk, vn = BT * pb.Hv * pb.dv;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    c.q = take(qn * 4); c.k = take(qn * 4); c.v = take(vn * 4); c.o = take(vn * 4);
    c.tc = take(plan_tc_cache(pb).bytes);
    c.bytes = off;
    return c;
}

size_t gdn_layer_core_fwd_cache_size(const gdn_layer_args* a) {
    if (!a || a->B < 1 || a->T < 1 || a->Hk < 1 || a->Hv < 1 || a->dk < 1 || a->dv < 1) return 0;
    if (!layer_tc_form(a->dtype, a->dk, a->dv, a->alpha_per_channel, a->gates_per_channel, a->h0)) return 0;
    return plan_layer_cache(make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map)).bytes;
}

// The layer forward hands its conv results to the tensor-core forward as bf16 hi/lo pairs (bf16
// tensors, scalar gates, d = 128); otherwise they stay fp32 for the CUDA-core forward.
static bool layer_fwd_split(const gdn_layer_args* a, const Problem& pb) {
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, true};
    return a->dtype == GDN_BF16 && !f.apc && !f.gpc && tc_fwd_eligible(pb, true, a->gate_dtype == GDN_BF16, f);
}

static size_t layer_fwd_own_ws(const gdn_layer_args* a) {
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    // q, k, v after the convolution are kept in fp32 between the two kernels.
    const size_t conv = align256((size_t)(a->B * a->T) * (2 * a->Hk * a->dk + a->Hv * a->dv) * 4);
    // the CUDA-core form with the output norm keeps o (fp32) for the norm + gate kernel
    const size_t onorm = a->norm_w && !layer_fwd_split(a, pb) ? align256((size_t)(a->B * a->T * a->Hv * a->dv) * 4) : 0;
    return 256 + conv + plan_chunk_ws(pb, false, false).bytes + onorm;
}

size_t gdn_layer_core_fwd_workspace_size(const gdn_layer_args* a) {
    if (!a || a->B < 1 || a->T < 1 || a->Hv < 1 || a->dk < 1 || a->dv < 1) return 0;
    return with_copies(layer_fwd_own_ws(a), args_pack_bytes<gdn_layer_args, layer_inputs<gdn_layer_args>>(a));
}

gdn_status gdn_layer_core_fwd(const gdn_layer_args* a, void* workspace, size_t workspace_bytes,
                              gdn_stream stream) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    gdn_status s = check_common(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->head_map,
                                a->alpha_per_channel, a->gates_per_channel, a->dtype, a->gate_dtype);
    if (s) return s;
    if (a->T > 0 && (!a->xq || !a->xk || !a->xv || !a->conv_w || !a->alpha || !a->b || !a->z || !a->y))
        return fail(GDN_ERR_INVALID_ARG, "xq, xk, xv, conv_w, alpha, b, z and y are required");
    if (a->gates_per_channel ? (a->T > 0 && !a->w) : a->w != nullptr)
        return fail(GDN_ERR_INVALID_ARG, "w is required with channel gates and must be NULL otherwise");
    const size_t es = elem_size(a->dtype), gs = elem_size(a->gate_dtype);
    const size_t BT = (size_t)(a->B * a->T);
    const size_t cch = (size_t)(2 * a->Hk * a->dk + a->Hv * a->dv);
    const size_t st = (size_t)(a->B * a->Hv * a->dk * a->dv) * 4;
    const gdn_strides& sd = a->strides;
    const int64_t ra = a->Hv * (a->alpha_per_channel ? a->dk : 1), rb = a->Hv * (a->gates_per_channel ? a->dk : 1);
    if ((s = check_stride(sd.q, a->Hk * a->dk, "xq")) || (s = check_stride(sd.k, a->Hk * a->dk, "xk")) ||
        (s = check_stride(sd.v, a->Hv * a->dv, "xv")) || (s = check_stride(sd.alpha, ra, "alpha")) ||
        (s = check_stride(sd.b, rb, "b")) || (s = check_stride(sd.w, a->Hv * a->dv, "w")) ||
        (s = check_stride(sd.z, a->Hv * a->dv, "z")))
        return s;
    const Buf in[] = {
        tok(a->xq, BT, a->Hk * a->dk, sd.q, es, "xq"), tok(a->xk, BT, a->Hk * a->dk, sd.k, es, "xk"),
        tok(a->xv, BT, a->Hv * a->dv, sd.v, es, "xv"), {a->conv_w, cch * 4 * es, "conv_w"},
        tok(a->alpha, BT, ra, sd.alpha, gs, "alpha"), tok(a->b, BT, rb, sd.b, gs, "b"),
        tok(a->w, BT, a->Hv * a->dv, sd.w, gs, "w"), tok(a->z, BT, a->Hv * a->dv, sd.z, es, "z"),
        {a->h0, st, "h0"}, {a->head_map, (size_t)a->Hv * 4, "head_map"},
        {a->norm_w, (size_t)a->dv * es, "norm_w"},
    };
    if (a->out_f32 != 0 && a->out_f32 != 1) return fail(GDN_ERR_INVALID_ARG, "out_f32 must be 0 or 1");
    if (a->norm_w && !(a->norm_eps >= 0.f && a->norm_eps < 1e30f))
        return fail(GDN_ERR_INVALID_ARG, "norm_eps must be a finite number >= 0");
    if ((s = check_logits(a->gate_logits, a->alpha_scale))) return s;
    const Buf out[] = {
        {a->y, BT * a->Hv * a->dv * (a->out_f32 ? 4 : es), "y"}, {a->ht, st, "ht"},
        {a->conv_state_out, (size_t)a->B * cch * 3 * es, "conv_state_out"},
        {a->bwd_cache, a->bwd_cache ? a->bwd_cache_bytes : 0, "bwd_cache"},
    };
    if ((s = check_buffers(in, 11, out, 4))) return s;
    if (a->bwd_cache) {
        if (!layer_tc_form(a->dtype, a->dk, a->dv, a->alpha_per_channel, a->gates_per_channel, a->h0))
            return fail(GDN_ERR_UNSUPPORTED, "bwd_cache: only the tensor-core form (bf16, d = 128, scalar gates, no h0) "
                                             "keeps a layer cache");
        if (reinterpret_cast<uintptr_t>(a->bwd_cache) & 255u)
            return fail(GDN_ERR_INVALID_ARG, "bwd_cache is not 256-byte aligned");
        if (a->bwd_cache_bytes < gdn_layer_core_fwd_cache_size(a))
            return fail(GDN_ERR_WORKSPACE, "bwd_cache has %zu bytes, %zu needed", a->bwd_cache_bytes,
                        gdn_layer_core_fwd_cache_size(a));
    }
    cudaStream_t sm = static_cast<cudaStream_t>(stream);
    if (a->T == 0) {
        if (a->conv_state_out) {
            cudaError_t e = cudaMemsetAsync(a->conv_state_out, 0, (size_t)a->B * cch * 3 * es, sm);
            if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_fwd");
        }
        return copy_state(a->ht, a->h0, st, sm, "gdn_layer_core_fwd");
    }
    // the workspace, then the dense copies of strided inputs, which the rest reads instead
    gdn_layer_args pa = *a;
    if ((s = copy_strided(&pa, layer_inputs<gdn_layer_args>, workspace, workspace_bytes, layer_fwd_own_ws(a), sm,
                          "gdn_layer_core_fwd (strided inputs)")))
        return s;
    a = &pa;
    char* base = static_cast<char*>(workspace) + 256;
    const size_t conv_bytes = align256(BT * cch * 4);
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    // the chunk part of the workspace (after the conv results) holds the flag array in both forms
    apply_logits(pb, a->gate_logits, a->alpha_scale);
    const WsPlan chunk_plan = plan_chunk_ws(pb, false, false);
    int* flags = carve_chunk_ws(chunk_plan, base + conv_bytes).flags;
    cudaError_t e0 = cudaMemsetAsync(ws_status(workspace), 0, sizeof(int), sm);
    if (e0 == cudaSuccess) e0 = clear_flags(flags, pb, sm);
    if (e0 != cudaSuccess) return cuda_fail(e0, "gdn_layer_core_fwd");
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, true};
    // The conv outputs are fp32 values.  With scalar gates and bf16 tensors they go to the
    // tensor-core forward as bf16 hi/lo pairs (same bytes); otherwise they stay fp32 for the
    // CUDA-core forward.
    const bool split = layer_fwd_split(a, pb);
    if (a->bwd_cache && !split)
        return fail(GDN_ERR_UNSUPPORTED, "bwd_cache: the tensor-map encoder of the CUDA driver is unavailable");
    const size_t qn = BT * a->Hk * a->dk, vn = BT * a->Hv * a->dv;
    const LayerCache lc = a->bwd_cache ? plan_layer_cache(pb) : LayerCache{};
    char* cache = static_cast<char*>(a->bwd_cache);
    if (cache) base = cache;  // the conv results are kept in the cache (same layout as below)
    ConvParams cp{};
    cp.xq = a->xq; cp.xk = a->xk; cp.xv = a->xv; cp.conv_w = a->conv_w;
    if (split) {
        cp.q = base; cp.q_lo = base + qn * 2;
        cp.k = base + qn * 4; cp.k_lo = base + qn * 6;
        cp.v = base + qn * 8; cp.v_lo = base + qn * 8 + vn * 2;
    } else {
        cp.q = base; cp.k = base + qn * 4; cp.v = base + qn * 8;
    }
    cp.conv_state_out = a->conv_state_out;
    cp.B = (int)a->B; cp.T = (int)a->T; cp.Hk = (int)a->Hk; cp.Hv = (int)a->Hv; cp.d = (int)a->dk;
    const int var = variant(a->dtype, a->gate_dtype);
    cudaError_t e = var == 2 ? f32_conv(cp, sm) : bf16_conv(cp, sm);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_fwd (conv)");
    ChunkIO io{};
    io.q = cp.q; io.k = cp.k; io.v = cp.v; io.alpha = a->alpha; io.b = a->b; io.w = a->w; io.z = a->z;
    io.h0 = a->h0; io.o = a->y; io.ht = a->ht;
    // y is written in dtype (bf16 -> o_type 2) unless out_f32.
    io.o_type = a->out_f32 || a->dtype == GDN_F32 ? 1 : 2;
    io.z_bf16 = a->dtype == GDN_BF16;
    io.norm_w = a->norm_w;
    io.norm_w_f32 = a->dtype == GDN_F32;
    io.norm_eps = a->norm_eps;
    if (split) {
        io.q_lo = cp.q_lo; io.k_lo = cp.k_lo; io.v_lo = cp.v_lo;
        if (cache) {
            const TcFwdSave save = tc_save_in(cache + lc.tc, pb, reinterpret_cast<float*>(cache + lc.o));
            e = tc_chunk_fwd(pb, io, f, a->gate_dtype == GDN_BF16, ws_status(workspace), sm, &save, flags);
        } else {
            e = tc_chunk_fwd(pb, io, f, a->gate_dtype == GDN_BF16, ws_status(workspace), sm, nullptr, flags);
        }
    } else if (a->norm_w) {
        // the CUDA-core chunk kernels split a row's columns over blocks: o (fp32, no gate) first, then
        // the norm and the gate row by row
        float* onorm = reinterpret_cast<float*>(static_cast<char*>(workspace) + 256 + conv_bytes + chunk_plan.bytes);
        io.o = onorm;
        io.o_type = 1;
        Flags fo = f;
        fo.gate = false;
        e = run_fwd(a->gate_dtype == GDN_F32 ? 2 : 3, pb, io, carve_chunk_ws(chunk_plan, base + conv_bytes), fo, sm);
        if (e == cudaSuccess)
            e = layer_norm_gate_fwd(onorm, a->z, a->norm_w, a->dtype == GDN_F32, a->norm_eps, a->y,
                                    a->out_f32 || a->dtype == GDN_F32, a->dtype == GDN_BF16, (long)BT * a->Hv,
                                    (int)a->dv, sm);
    } else {
        e = run_fwd(a->gate_dtype == GDN_F32 ? 2 : 3, pb, io, carve_chunk_ws(chunk_plan, base + conv_bytes), f, sm);
    }
    return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_layer_core_fwd");
}

// Workspace of the layer backward, offsets from its start, 256-byte aligned.
// Tensor-core form (bf16 tensors, d = 128, scalar gates, no initial state): the tensor-core
// backward's own workspace
// first (its status word is the call's, at offset 0), then the conv results as bf16 hi/lo pairs,
// the recurrence's output o, the gradient of o (bf16 hi/lo), the q, k, v gradients from the
// recurrence, the conv-weight partials and the forward cache (states, V', T tiles).
// CUDA-core form (everything else): the status word, the fp32 conv results, o, the gradient of o
// (fp32), the q, k, v gradients, the conv-weight partials, then the CUDA-core chunk workspace.
struct LayerBwdPlan {
    bool tc;
    size_t q, k, v, o, dout, npart, gq, gk, gv, wpart, cache, chunk, bytes;
};
static bool layer_bwd_tc_form(const gdn_layer_bwd_args* a) {
    return layer_tc_form(a->dtype, a->dk, a->dv, a->alpha_per_channel, a->gates_per_channel, a->h0);
}
static LayerBwdPlan plan_layer_bwd(const gdn_layer_bwd_args* a, const Problem& pb) {
    LayerBwdPlan w{};
    w.tc = layer_bwd_tc_form(a);
    const size_t BT = (size_t)(a->B * a->T), qn = BT * a->Hk * a->dk, vn = BT * a->Hv * a->dv;
    size_t off = w.tc ? align256(plan_tc_bwd_ws(pb, !identity_heads(pb), true).bytes) : 256;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    w.chunk = w.tc ? 0 : ~size_t(0);
    // with the forward's cache the conv results, o, the states and V' are read from it
    const bool cached = w.tc && a->fwd_cache != nullptr;
    if (!cached) {
        w.q = take(qn * 4); w.k = take(qn * 4); w.v = take(vn * 4); w.o = take(vn * 4);
    }
    w.dout = take(vn * 4);  // fp32, or bf16 hi then lo
    w.npart = a->norm_w ? take(layer_norm_partials_floats((int)a->dv) * 4) : ~size_t(0);
    w.gq = take(qn * 4); w.gk = take(qn * 4); w.gv = take(vn * 4);
    w.wpart = take(layer_bwd_wpart_floats((int)a->B, (int)a->T, (int)a->Hk, (int)a->Hv, (int)a->dk) * 4);
    if (w.tc) {
        w.cache = cached ? ~size_t(0) : take(plan_tc_cache(pb).bytes);
    } else {
        w.cache = ~size_t(0);
        w.chunk = off;
        off += plan_chunk_ws(pb, true, !identity_heads(pb)).bytes;
    }
    w.bytes = off;
    return w;
}

size_t gdn_layer_core_bwd_workspace_size(const gdn_layer_bwd_args* a) {
    if (!a || a->B < 1 || a->T < 1 || a->Hv < 1 || a->dk < 1 || a->dv < 1) return 0;
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    return with_copies(plan_layer_bwd(a, pb).bytes,
                       args_pack_bytes<gdn_layer_bwd_args, layer_inputs<gdn_layer_bwd_args>>(a));
}

gdn_status gdn_layer_core_bwd(const gdn_layer_bwd_args* a, void* workspace, size_t workspace_bytes,
                              gdn_stream stream) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    gdn_status s = check_common(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->head_map,
                                a->alpha_per_channel, a->gates_per_channel, a->dtype, a->gate_dtype);
    if (s) return s;
    if (a->dk != a->dv) return fail(GDN_ERR_UNSUPPORTED, "the layer core needs dk == dv");
    if (a->T > 0 && (!a->xq || !a->xk || !a->xv || !a->conv_w || !a->alpha || !a->b || !a->z || !a->grad_y ||
                     !a->grad_xq || !a->grad_xk || !a->grad_xv || !a->grad_alpha || !a->grad_b || !a->grad_z))
        return fail(GDN_ERR_INVALID_ARG, "inputs, grad_y and the gradients of xq, xk, xv, alpha, b, z are required");
    if (!a->grad_conv_w) return fail(GDN_ERR_INVALID_ARG, "grad_conv_w is required");
    if (a->norm_w && !a->grad_norm_w) return fail(GDN_ERR_INVALID_ARG, "grad_norm_w is required with norm_w");
    if (!a->norm_w && a->grad_norm_w) return fail(GDN_ERR_INVALID_ARG, "grad_norm_w must be NULL without norm_w");
    if (a->norm_w && !(a->norm_eps >= 0.f && a->norm_eps < 1e30f))
        return fail(GDN_ERR_INVALID_ARG, "norm_eps must be a finite number >= 0");
    if ((s = check_logits(a->gate_logits, a->alpha_scale, a->grad_alpha_scale))) return s;
    if (a->gates_per_channel ? (a->T > 0 && (!a->w || !a->grad_w)) : (a->w != nullptr || a->grad_w != nullptr))
        return fail(GDN_ERR_INVALID_ARG, "w and grad_w are required with channel gates and must be NULL otherwise");
    const size_t es = elem_size(a->dtype), gs = elem_size(a->gate_dtype);
    const size_t BT = (size_t)(a->B * a->T);
    const size_t cch = (size_t)(2 * a->Hk * a->dk + a->Hv * a->dv);
    const size_t st = (size_t)(a->B * a->Hv * a->dk * a->dv) * 4;
    const size_t na = BT * a->Hv * (a->alpha_per_channel ? a->dk : 1), nb = BT * a->Hv * (a->gates_per_channel ? a->dk : 1);
    const size_t nw = a->gates_per_channel ? BT * a->Hv * a->dv : 0;
    const gdn_strides& sd = a->strides;
    const int64_t ra = a->Hv * (a->alpha_per_channel ? a->dk : 1), rb = a->Hv * (a->gates_per_channel ? a->dk : 1);
    if ((s = check_stride(sd.q, a->Hk * a->dk, "xq")) || (s = check_stride(sd.k, a->Hk * a->dk, "xk")) ||
        (s = check_stride(sd.v, a->Hv * a->dv, "xv")) || (s = check_stride(sd.alpha, ra, "alpha")) ||
        (s = check_stride(sd.b, rb, "b")) || (s = check_stride(sd.w, a->Hv * a->dv, "w")) ||
        (s = check_stride(sd.z, a->Hv * a->dv, "z")))
        return s;
    const Buf in[] = {
        tok(a->xq, BT, a->Hk * a->dk, sd.q, es, "xq"), tok(a->xk, BT, a->Hk * a->dk, sd.k, es, "xk"),
        tok(a->xv, BT, a->Hv * a->dv, sd.v, es, "xv"), {a->conv_w, cch * 4 * es, "conv_w"},
        tok(a->alpha, BT, ra, sd.alpha, gs, "alpha"), tok(a->b, BT, rb, sd.b, gs, "b"),
        tok(a->w, BT, a->Hv * a->dv, sd.w, gs, "w"), tok(a->z, BT, a->Hv * a->dv, sd.z, es, "z"), {a->h0, st, "h0"},
        {a->head_map, (size_t)a->Hv * 4, "head_map"},
        {a->grad_y, BT * a->Hv * a->dv * es, "grad_y"}, {a->grad_ht, st, "grad_ht"},
        {a->fwd_cache, a->fwd_cache ? a->fwd_cache_bytes : 0, "fwd_cache"},
        {a->norm_w, (size_t)a->dv * es, "norm_w"},
    };
    const Buf out[] = {
        {a->grad_xq, BT * a->Hk * a->dk * 4, "grad_xq"}, {a->grad_xk, BT * a->Hk * a->dk * 4, "grad_xk"},
        {a->grad_xv, BT * a->Hv * a->dv * 4, "grad_xv"}, {a->grad_conv_w, cch * 4 * 4, "grad_conv_w"},
        {a->grad_alpha, na * 4, "grad_alpha"}, {a->grad_b, nb * 4, "grad_b"}, {a->grad_w, nw * 4, "grad_w"},
        {a->grad_z, BT * a->Hv * a->dv * 4, "grad_z"}, {a->grad_h0, st, "grad_h0"},
        {a->grad_norm_w, (size_t)a->dv * 4, "grad_norm_w"},
    };
    if ((s = check_buffers(in, 14, out, 10))) return s;
    if (a->fwd_cache) {
        if (!layer_bwd_tc_form(a))
            return fail(GDN_ERR_UNSUPPORTED, "fwd_cache: only the tensor-core form (bf16, d = 128, scalar gates, no h0) "
                                             "keeps a layer cache");
        if (reinterpret_cast<uintptr_t>(a->fwd_cache) & 255u)
            return fail(GDN_ERR_INVALID_ARG, "fwd_cache is not 256-byte aligned");
        const size_t need = plan_layer_cache(make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale,
                                                          a->head_map)).bytes;
        if (a->fwd_cache_bytes < need)
            return fail(GDN_ERR_INVALID_ARG, "fwd_cache has %zu bytes, %zu needed", a->fwd_cache_bytes, need);
    }
    cudaStream_t sm = static_cast<cudaStream_t>(stream);
    if (a->T == 0) {
        cudaError_t e = cudaMemsetAsync(a->grad_conv_w, 0, cch * 4 * 4, sm);
        if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd");
        return copy_state(a->grad_h0, a->grad_ht, st, sm, "gdn_layer_core_bwd");
    }
    Problem pb = make_problem(a->B, a->T, a->Hk, a->Hv, a->dk, a->dv, a->scale, a->head_map);
    apply_logits(pb, a->gate_logits, a->alpha_scale);
    const LayerBwdPlan plan = plan_layer_bwd(a, pb);
    // the workspace, then the dense copies of strided inputs, which the rest reads instead
    gdn_layer_bwd_args pa = *a;
    if ((s = copy_strided(&pa, layer_inputs<gdn_layer_bwd_args>, workspace, workspace_bytes, plan.bytes, sm,
                          "gdn_layer_core_bwd (strided inputs)")))
        return s;
    a = &pa;
    char* wsb = static_cast<char*>(workspace);
    auto at = [&](size_t o) { return reinterpret_cast<float*>(wsb + o); };
    const bool bf16 = a->dtype == GDN_BF16, bf16g = a->gate_dtype == GDN_BF16;
    const bool direct = identity_heads(pb);
    // the flag array of the pairs outside the decay range: in the tensor-core backward's workspace
    // (at offset 0) or in the CUDA-core chunk workspace
    int* flags = plan.tc ? reinterpret_cast<int*>(wsb + plan_tc_bwd_ws(pb, !direct, true).flags)
                         : carve_chunk_ws(plan_chunk_ws(pb, true, !direct), wsb + plan.chunk).flags;
    cudaError_t e = cudaMemsetAsync(ws_status(workspace), 0, sizeof(int), sm);
    if (e == cudaSuccess) e = clear_flags(flags, pb, sm);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd");
    Flags f{a->alpha_per_channel != 0, a->gates_per_channel != 0, false};
    ConvParams cp{};
    cp.xq = a->xq; cp.xk = a->xk; cp.xv = a->xv; cp.conv_w = a->conv_w;
    cp.B = (int)a->B; cp.T = (int)a->T; cp.Hk = (int)a->Hk; cp.Hv = (int)a->Hv; cp.d = (int)a->dk;
    LayerBwdIO lio{};
    lio.xq = a->xq; lio.xk = a->xk; lio.xv = a->xv; lio.conv_w = a->conv_w; lio.z = a->z; lio.dy = a->grad_y;
    lio.o = at(plan.o); lio.gq = at(plan.gq); lio.gk = at(plan.gk); lio.gv = at(plan.gv);
    lio.dz = a->grad_z;
    lio.dxq = a->grad_xq; lio.dxk = a->grad_xk; lio.dxv = a->grad_xv;
    lio.wpart = at(plan.wpart); lio.dconv_w = a->grad_conv_w;
    lio.B = (int)a->B; lio.T = (int)a->T; lio.Hk = (int)a->Hk; lio.Hv = (int)a->Hv; lio.d = (int)a->dk;
    lio.norm_w = a->norm_w;
    lio.norm_w_f32 = a->dtype == GDN_F32;
    lio.norm_eps = a->norm_eps;
    lio.npart = a->norm_w ? at(plan.npart) : nullptr;
    lio.dnorm_w = a->grad_norm_w;
    ChunkIO io{};
    io.alpha = a->alpha; io.b = a->b; io.w = a->w; io.h0 = a->h0;
    if (plan.tc) {
        if (!tc_fwd_eligible(pb, true, bf16g, f))
            return fail(GDN_ERR_UNSUPPORTED, "the tensor-map encoder of the CUDA driver is unavailable");
        // 1. conv + SiLU + L2, fp32 results stored as bf16 hi/lo pairs; 2. the tensor-core forward
        //    in saving mode: o (fp32, no gate), the chunk states and V'.  Both come from the
        //    forward's cache when the caller passes one.
        const size_t qn = BT * a->Hk * a->dk, vn = BT * a->Hv * a->dv;
        char* fc = static_cast<char*>(const_cast<void*>(a->fwd_cache));
        const LayerCache lc = fc ? plan_layer_cache(pb) : LayerCache{};
        char* q = fc ? fc + lc.q : wsb + plan.q;
        char* k = fc ? fc + lc.k : wsb + plan.k;
        char* v = fc ? fc + lc.v : wsb + plan.v;
        float* o = fc ? reinterpret_cast<float*>(fc + lc.o) : at(plan.o);
        char* cb = fc ? fc + lc.tc : wsb + plan.cache;
        cp.q = q; cp.q_lo = q + qn * 2; cp.k = k; cp.k_lo = k + qn * 2; cp.v = v; cp.v_lo = v + vn * 2;
        io.q = cp.q; io.k = cp.k; io.v = cp.v; io.q_lo = cp.q_lo; io.k_lo = cp.k_lo; io.v_lo = cp.v_lo;
        lio.o = o;
        if (!fc) {
            e = bf16_conv(cp, sm);
            if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (conv)");
            io.o = o; io.o_type = 1;
            const TcFwdSave save = tc_save_in(cb, pb, nullptr);
            e = tc_chunk_fwd(pb, io, f, bf16g, ws_status(workspace), sm, &save, flags);
            if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (forward)");
        }
        // 3. swish gate; the gradient of o as bf16 hi/lo pairs (tensor-core operands)
        lio.dout16 = reinterpret_cast<__nv_bfloat16*>(wsb + plan.dout);
        lio.dout16_lo = lio.dout16 + vn;
        e = layer_gate_bwd(lio, bf16, sm);
        if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (gate)");
        // 4. the tensor-core backward from the cache, with do as its bf16 hi/lo pair: the scan and
        //    the gradient kernel take the lo tiles as a third operand of their dO products (a
        //    single bf16 do would move dq by ~5% of its RMS on this layer).
        const TcBwdWs tplan = plan_tc_bwd_ws(pb, !direct, true);
        io.o = nullptr;
        io.dout = lio.dout16; io.dout_lo = lio.dout16_lo; io.dht = a->grad_ht;
        io.dq = at(plan.gq); io.dk = at(plan.gk); io.dv = at(plan.gv);
        io.dalpha = a->grad_alpha; io.db = a->grad_b; io.dw = nullptr; io.dh0 = a->grad_h0;
        e = tc_chunk_bwd(pb, io, f, bf16g, direct, tplan, workspace, cb, sm);
        if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (recurrence)");
    } else {
        // 1. conv + SiLU + L2, fp32 results
        cp.q = at(plan.q); cp.k = at(plan.k); cp.v = at(plan.v);
        e = bf16 ? bf16_conv(cp, sm) : f32_conv(cp, sm);
        if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (conv)");
        // 2. o (fp32, no gate) on the CUDA-core forward, which also keeps the chunk states for step 4
        //    (paired: the backward does not run the forward again)
        f.paired = true;
        const ChunkWs cws = carve_chunk_ws(plan_chunk_ws(pb, true, !direct), wsb + plan.chunk);
        io.q = cp.q; io.k = cp.k; io.v = cp.v;
        io.o = at(plan.o); io.o_type = 1;
        const int var = a->gate_dtype == GDN_F32 ? 2 : 3;
        e = run_fwd(var, pb, io, cws, f, sm);
        if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (forward)");
        // 3. swish gate
        lio.dout = at(plan.dout);
        e = layer_gate_bwd(lio, bf16, sm);
        if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (gate)");
        // 4. the recurrence's backward on the fp32 conv results
        io.o = nullptr;
        io.dout = at(plan.dout); io.dht = a->grad_ht;
        io.dq = at(plan.gq); io.dk = at(plan.gk); io.dv = at(plan.gv);
        io.dalpha = a->grad_alpha; io.db = a->grad_b; io.dw = a->grad_w; io.dh0 = a->grad_h0;
        e = var == 2 ? f32_chunk_bwd(pb, io, cws, f, direct, sm) : f32_bf16g_chunk_bwd(pb, io, cws, f, direct, sm);
        if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (recurrence)");
    }
    // 5. L2 norm, SiLU and conv backward, conv-weight gradient
    e = layer_conv_bwd(lio, bf16, sm);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_layer_core_bwd (conv)");
    // 6. gates as logits: the gradients of the gates become those of their logits
    if (pb.gate_logits)
        e = gate_logit_grads(pb, f, a->gate_dtype == GDN_F32, a->alpha, a->b, a->w, a->grad_alpha, a->grad_b,
                             a->grad_w, false, a->grad_alpha_scale, sm);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_layer_core_bwd (gate logits)");
}

gdn_status gdn_workspace_status(const void* workspace, gdn_stream stream) {
    if (!workspace) return fail(GDN_ERR_INVALID_ARG, "workspace is NULL");
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost,
                                    static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gdn_workspace_status");
    if (word != 0) return fail(GDN_ERR_TIMEOUT, "a bounded wait inside a kernel expired (status %d)", word);
    return GDN_OK;
}

const char* gdn_last_error(void) { return g_last_error.c_str(); }

int gdn_version(void) { return 100; }

long long gdn_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
