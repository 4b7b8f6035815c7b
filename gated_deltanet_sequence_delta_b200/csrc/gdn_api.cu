// gdn_api.cu -- the C ABI declared in gdn.h: host-side validation, then launches.
// Nothing is launched unless every check passes; nothing is allocated or freed.
#include <cuda_runtime.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.cuh"

namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_stall_site{0};   // gdn_testing_stall

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    const void* p;
    size_t bytes;
};

bool overlap(Range a, Range b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

size_t esize(gdn_dtype d) { return d == GDN_BF16 ? 2 : 4; }
bool dtype_ok(gdn_dtype d) { return d == GDN_F32 || d == GDN_BF16; }
bool head_dim_ok(int32_t d) { return d == 64 || d == 128; }

gdn_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return GDN_OK;
    g_last_cuda_error = (int)e;
    return GDN_ERR_CUDA;
}

}  // namespace

namespace gdn {
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
int testing_stall_site() { return g_stall_site.load(std::memory_order_relaxed); }
}  // namespace gdn

extern "C" {

uint64_t gdn_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_NULL: return "GDN_ERR_NULL: a required pointer is NULL";
        case GDN_ERR_SHAPE: return "GDN_ERR_SHAPE: a size is out of range or inconsistent";
        case GDN_ERR_ALIGN: return "GDN_ERR_ALIGN: a pointer is not 16-byte aligned";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: head dim, chunk size or dtype not implemented";
        case GDN_ERR_ALIAS: return "GDN_ERR_ALIAS: an output overlaps an input or another output";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing or too small";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a CUDA call or launch failed";
        case GDN_ERR_DEVICE: return "GDN_ERR_DEVICE: a device-side check failed";
        default: return "GDN: unknown status";
    }
}

int gdn_abi_version(void) { return GDN_ABI_VERSION; }

gdn_status gdn_testing_stall(int32_t site) {
    if (site < GDN_STALL_NONE || site > GDN_STALL_PREFILL_PREP) return GDN_ERR_SHAPE;
    g_stall_site.store(site, std::memory_order_relaxed);
    return GDN_OK;
}

int gdn_last_cuda_error(void) { return g_last_cuda_error; }

gdn_status gdn_gates(const void* a, const void* b, gdn_dtype ab_dtype, const float* A_log,
                     const float* dt_bias, int64_t n_tokens, int32_t HV, float* g, float* beta,
                     void* stream) {
    if (!A_log || !dt_bias) return GDN_ERR_NULL;
    if (HV <= 0 || n_tokens < 0) return GDN_ERR_SHAPE;
    if (!dtype_ok(ab_dtype)) return GDN_ERR_UNSUPPORTED;
    if (n_tokens == 0) return GDN_OK;
    if (!a || !b || !g || !beta) return GDN_ERR_NULL;
    if (!aligned16(a) || !aligned16(b) || !aligned16(g) || !aligned16(beta) || !aligned16(A_log) ||
        !aligned16(dt_bias))
        return GDN_ERR_ALIGN;
    const size_t n = (size_t)n_tokens * (size_t)HV;
    const Range ra{a, n * esize(ab_dtype)}, rb{b, n * esize(ab_dtype)};
    const Range rA{A_log, (size_t)HV * 4}, rd{dt_bias, (size_t)HV * 4};
    const Range rg{g, n * 4}, rbeta{beta, n * 4};
    for (Range out : {rg, rbeta})
        for (Range in : {ra, rb, rA, rd})
            if (overlap(out, in)) return GDN_ERR_ALIAS;
    if (overlap(rg, rbeta)) return GDN_ERR_ALIAS;
    return cuda_status(gdn::launch_gates(a, b, ab_dtype == GDN_BF16, A_log, dt_bias, n_tokens, HV,
                                         g, beta, (cudaStream_t)stream));
}

size_t gdn_chunk_prefill_workspace_bytes(int64_t n_tokens, int32_t n_seqs, int32_t HK, int32_t HV,
                                         int32_t Dk, int32_t Dv, int32_t BT, gdn_dtype io_dtype) {
    if (n_tokens < 0 || n_tokens > INT32_MAX || n_seqs < 0 || HK <= 0 || HV <= 0 || HV % HK != 0) return 0;
    if (!head_dim_ok(Dk) || !head_dim_ok(Dv) || !dtype_ok(io_dtype)) return 0;
    if (!(BT == 16 || BT == 32 || BT == 64)) return 0;
    if (io_dtype == GDN_BF16 && gdn::prefill_tc_supported(Dk, Dv, HK, HV, BT))
        return gdn::prefill_tc_workspace_bytes(n_tokens, n_seqs, HK, HV);
    return gdn::kStatusBytes;
}

}  // extern "C"

namespace gdn {
// The size checks of gdn_chunk_prefill, in its order: SHAPE for sizes out of range or
// inconsistent with the layout, UNSUPPORTED for head dims, chunk sizes or dtypes that no
// kernel takes (including sizes past the tile-copy coordinates); GDN_OK otherwise.
gdn_status prefill_check_sizes(gdn_dtype io_dtype, bool packed, int32_t B, int64_t T, int32_t n_seqs, int32_t HK,
                               int32_t HV, int32_t Dk, int32_t Dv, int32_t BT) {
    if (B < 0 || T < 0 || n_seqs < 0 || HK <= 0 || HV <= 0 || Dk <= 0 || Dv <= 0 || BT <= 0)
        return GDN_ERR_SHAPE;
    if (HV % HK != 0) return GDN_ERR_SHAPE;
    if (packed) {
        if (B != 1) return GDN_ERR_SHAPE;
        if (T > INT32_MAX) return GDN_ERR_SHAPE;
    } else if (n_seqs != B) {
        return GDN_ERR_SHAPE;
    }
    if (!dtype_ok(io_dtype) || !head_dim_ok(Dk) || !head_dim_ok(Dv)) return GDN_ERR_UNSUPPORTED;
    if (gdn_chunk_prefill_workspace_bytes((int64_t)B * T, n_seqs, HK, HV, Dk, Dv, BT, io_dtype) == 0)
        return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}
}  // namespace gdn

namespace {
// Raw gate inputs of gdn_chunk_prefill_gated (all null for the entry points that take g, beta).
struct RawGates {
    const void* a;
    const void* b;
    gdn_dtype ab_dtype;
    const float* A_log;
    const float* dt_bias;
};

// gdn_chunk_prefill, with the output epilogue when z is given (tensor-core path only) and the
// gates formed in the kernel when g is null and gin.a is given (tensor-core path only)
gdn_status prefill_impl(const void* q, const void* k, const void* v, gdn_dtype io_dtype, const float* g,
                        const float* beta, const RawGates& gin, const float* initial_state,
                        const int32_t* cu_seqlens, int32_t B,
                        int64_t T, int32_t n_seqs, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t BT,
                        float scale, int32_t qk_l2norm, const void* z, const float* norm_w, float eps, void* o,
                        float* final_state, void* o_tr, float* final_tr, void* workspace, size_t workspace_bytes,
                        void* stream) {
    // ---- sizes -----------------------------------------------------------------
    const gdn_status sz =
        gdn::prefill_check_sizes(io_dtype, cu_seqlens != nullptr, B, T, n_seqs, HK, HV, Dk, Dv, BT);
    if (sz != GDN_OK) return sz;
    const size_t need = gdn_chunk_prefill_workspace_bytes((int64_t)B * T, n_seqs, HK, HV, Dk, Dv,
                                                          BT, io_dtype);
    const int64_t n_tok = (int64_t)B * T;
    if (n_seqs == 0) return GDN_OK;
    // ---- pointers ----------------------------------------------------------------
    if (!workspace) return GDN_ERR_WORKSPACE;
    if (workspace_bytes < need) return GDN_ERR_WORKSPACE;
    const bool raw = gin.a != nullptr || gin.b != nullptr;
    if (raw && !(io_dtype == GDN_BF16 && gdn::prefill_tc_supported(Dk, Dv, HK, HV, BT))) return GDN_ERR_UNSUPPORTED;
    if (raw && !dtype_ok(gin.ab_dtype)) return GDN_ERR_UNSUPPORTED;
    if (n_tok > 0 && (!q || !k || !v || !o)) return GDN_ERR_NULL;
    if (n_tok > 0 && (raw ? (!gin.a || !gin.b || !gin.A_log || !gin.dt_bias) : (!g || !beta))) return GDN_ERR_NULL;
    if (z && (!norm_w || !(eps >= 0.f))) return norm_w ? GDN_ERR_SHAPE : GDN_ERR_NULL;
    if ((z || o_tr) && !(io_dtype == GDN_BF16 && gdn::prefill_tc_supported(Dk, Dv, HK, HV, BT)))
        return GDN_ERR_UNSUPPORTED;
    if (o_tr && n_tok > 0 && !final_tr) return GDN_ERR_NULL;
    if (cu_seqlens == nullptr && n_tok == 0 && final_state == nullptr) return GDN_OK;
    const void* ptrs[] = {q, k, v, g, beta, initial_state, cu_seqlens, o, final_state, workspace, z, norm_w,
                          o_tr, final_tr, gin.a, gin.b, gin.A_log, gin.dt_bias};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    // ---- aliasing ----------------------------------------------------------------
    const size_t es = esize(io_dtype);
    const size_t state_bytes = (size_t)n_seqs * HV * Dk * Dv * 4;
    const Range rq{q, (size_t)n_tok * HK * Dk * es}, rk{k, (size_t)n_tok * HK * Dk * es};
    const Range rv{v, (size_t)n_tok * HV * Dv * es};
    const Range rg{g, (size_t)n_tok * HV * 4}, rb{beta, (size_t)n_tok * HV * 4};
    const Range rh0{initial_state, state_bytes}, rcu{cu_seqlens, cu_seqlens ? (size_t)(n_seqs + 1) * 4 : 0};
    const Range ro{o, (size_t)n_tok * HV * Dv * es}, rhT{final_state, state_bytes};
    const Range rws{workspace, workspace_bytes};
    const Range rz{z, z ? (size_t)n_tok * HV * Dv * es : 0}, rnw{norm_w, z ? (size_t)Dv * 4 : 0};
    const Range rotr{o_tr, o_tr ? (size_t)n_tok * HV * Dv * es : 0}, rhtr{final_tr, o_tr ? state_bytes : 0};
    const size_t eab = raw ? esize(gin.ab_dtype) : 0;
    const Range rra{gin.a, (size_t)n_tok * HV * eab}, rrb{gin.b, (size_t)n_tok * HV * eab};
    const Range rAl{gin.A_log, raw ? (size_t)HV * 4 : 0}, rdb{gin.dt_bias, raw ? (size_t)HV * 4 : 0};
    for (Range out : {ro, rhT, rws, rotr, rhtr}) {
        for (Range in : {rq, rk, rv, rg, rb, rcu, rz, rnw, rra, rrb, rAl, rdb})
            if (overlap(out, in)) return GDN_ERR_ALIAS;
    }
    for (Range tr : {rotr, rhtr})
        for (Range other : {ro, rhT, rws, rh0})
            if (overlap(tr, other)) return GDN_ERR_ALIAS;
    if (overlap(rotr, rhtr)) return GDN_ERR_ALIAS;
    if (overlap(ro, rhT) || overlap(ro, rws) || overlap(rhT, rws) || overlap(ro, rh0) ||
        overlap(rws, rh0))
        return GDN_ERR_ALIAS;
    // final_state may be exactly initial_state (in-place carry), nothing else
    if (overlap(rhT, rh0) && final_state != initial_state) return GDN_ERR_ALIAS;

    cudaStream_t s = (cudaStream_t)stream;
    int32_t* status = reinterpret_cast<int32_t*>(workspace);
    const bool use_tc = io_dtype == GDN_BF16 && gdn::prefill_tc_supported(Dk, Dv, HK, HV, BT);
    if (!use_tc) {
        gdn_status st = cuda_status(gdn::launch_check_cu_seqlens(cu_seqlens, n_seqs, T, status, s));
        if (st != GDN_OK) return st;
    }

    gdn::PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.bf16 = io_dtype == GDN_BF16;
    a.g = raw ? nullptr : g; a.beta = raw ? nullptr : beta; a.h0 = initial_state; a.cu = cu_seqlens;
    a.gates = raw ? gdn::DecodeGates{nullptr, nullptr, gin.a, gin.b, gin.ab_dtype == GDN_BF16, gin.A_log, gin.dt_bias}
                  : gdn::DecodeGates{g, beta, nullptr, nullptr, false, nullptr, nullptr};
    a.T = T; a.n_seqs = n_seqs; a.HK = HK; a.HV = HV; a.Dk = Dk; a.Dv = Dv; a.BT = BT;
    a.scale = scale; a.l2norm = qk_l2norm ? 1 : 0; a.o = o; a.hT = final_state;
    a.z = z; a.norm_w = norm_w; a.eps = eps;
    a.o_tr = o_tr; a.hT_tr = o_tr ? final_tr : nullptr;
    a.status = status;
    a.scratch = static_cast<char*>(workspace) + gdn::kStatusBytes;
    a.scratch_bytes = workspace_bytes - gdn::kStatusBytes;
    if (use_tc) return cuda_status(gdn::launch_prefill_tc(a, workspace, s));
    return cuda_status(gdn::launch_prefill_cudacore(a, s));
}
}  // namespace

extern "C" {

gdn_status gdn_chunk_prefill(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                             const float* g, const float* beta, const float* initial_state,
                             const int32_t* cu_seqlens, int32_t B, int64_t T, int32_t n_seqs,
                             int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t BT,
                             float scale, int32_t qk_l2norm, void* o, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream) {
    return prefill_impl(q, k, v, io_dtype, g, beta, RawGates{}, initial_state, cu_seqlens, B, T, n_seqs, HK, HV, Dk,
                        Dv, BT, scale, qk_l2norm, nullptr, nullptr, 0.f, o, final_state, nullptr, nullptr, workspace,
                        workspace_bytes, stream);
}

gdn_status gdn_chunk_prefill_gated(const void* q, const void* k, const void* v, gdn_dtype io_dtype, const void* a,
                                   const void* b, gdn_dtype ab_dtype, const float* A_log, const float* dt_bias,
                                   const float* initial_state, const int32_t* cu_seqlens, int32_t B, int64_t T,
                                   int32_t n_seqs, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t BT,
                                   float scale, int32_t qk_l2norm, void* o, float* final_state, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    if (!a || !b) return GDN_ERR_NULL;
    return prefill_impl(q, k, v, io_dtype, nullptr, nullptr, RawGates{a, b, ab_dtype, A_log, dt_bias}, initial_state,
                        cu_seqlens, B, T, n_seqs, HK, HV, Dk, Dv, BT, scale, qk_l2norm, nullptr, nullptr, 0.f, o,
                        final_state, nullptr, nullptr, workspace, workspace_bytes, stream);
}

gdn_status gdn_chunk_prefill_outgate(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                                     const float* g, const float* beta, const float* initial_state,
                                     const int32_t* cu_seqlens, int32_t B, int64_t T, int32_t n_seqs,
                                     int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t BT, float scale,
                                     int32_t qk_l2norm, const void* z, const float* norm_w, float eps, void* o,
                                     float* final_state, void* workspace, size_t workspace_bytes, void* stream) {
    if (!z) return GDN_ERR_NULL;
    return prefill_impl(q, k, v, io_dtype, g, beta, RawGates{}, initial_state, cu_seqlens, B, T, n_seqs, HK, HV, Dk,
                        Dv, BT, scale, qk_l2norm, z, norm_w, eps, o, final_state, nullptr, nullptr, workspace,
                        workspace_bytes, stream);
}

gdn_status gdn_cp_segment(const void* q, const void* k, const void* v, gdn_dtype io_dtype, const float* g,
                          const float* beta, const float* initial_state, const int32_t* cu_seqlens, int32_t B,
                          int64_t T, int32_t n_seqs, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t BT,
                          float scale, int32_t qk_l2norm, void* o, float* final_state, void* c, float* transition,
                          void* workspace, size_t workspace_bytes, void* stream) {
    if (!c) return GDN_ERR_NULL;
    if (Dk != Dv) return GDN_ERR_UNSUPPORTED;
    return prefill_impl(q, k, v, io_dtype, g, beta, RawGates{}, initial_state, cu_seqlens, B, T, n_seqs, HK, HV, Dk,
                        Dv, BT, scale, qk_l2norm, nullptr, nullptr, 0.f, o, final_state, c, transition, workspace,
                        workspace_bytes, stream);
}

gdn_status gdn_chunk_prefill_status(const void* workspace, void* stream, int32_t* device_error) {
    if (!workspace || !device_error) return GDN_ERR_NULL;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    int32_t word = 0;
    e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    *device_error = word;
    return word ? GDN_ERR_DEVICE : GDN_OK;
}

gdn_status gdn_decode_step(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                           const float* g, const float* beta, float* state, int32_t B, int32_t HK,
                           int32_t HV, int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm,
                           void* o, void* stream) {
    if (B < 0 || HK <= 0 || HV <= 0 || Dk <= 0 || Dv <= 0 || HV % HK != 0) return GDN_ERR_SHAPE;
    if (!dtype_ok(io_dtype) || !head_dim_ok(Dk) || !head_dim_ok(Dv)) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_NULL;
    const void* ptrs[] = {q, k, v, g, beta, state, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return GDN_ERR_ALIGN;
    const size_t es = esize(io_dtype);
    const Range rq{q, (size_t)B * HK * Dk * es}, rk{k, (size_t)B * HK * Dk * es};
    const Range rv{v, (size_t)B * HV * Dv * es}, rg{g, (size_t)B * HV * 4}, rb{beta, (size_t)B * HV * 4};
    const Range rs{state, (size_t)B * HV * Dk * Dv * 4}, ro{o, (size_t)B * HV * Dv * es};
    for (Range out : {rs, ro})
        for (Range in : {rq, rk, rv, rg, rb})
            if (overlap(out, in)) return GDN_ERR_ALIAS;
    if (overlap(rs, ro)) return GDN_ERR_ALIAS;
    const gdn::DecodeGates gates{g, beta, nullptr, nullptr, false, nullptr, nullptr};
    return cuda_status(gdn::launch_decode(q, k, v, io_dtype == GDN_BF16, gates, state, B, HK, HV, Dk, Dv, scale,
                                          qk_l2norm ? 1 : 0, o, (cudaStream_t)stream));
}

gdn_status gdn_decode_step_gated(const void* q, const void* k, const void* v, gdn_dtype io_dtype, const void* a,
                                 const void* b, gdn_dtype ab_dtype, const float* A_log, const float* dt_bias,
                                 float* state, int32_t B, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                                 float scale, int32_t qk_l2norm, void* o, void* stream) {
    if (B < 0 || HK <= 0 || HV <= 0 || Dk <= 0 || Dv <= 0 || HV % HK != 0) return GDN_ERR_SHAPE;
    if (!dtype_ok(io_dtype) || !dtype_ok(ab_dtype) || !head_dim_ok(Dk) || !head_dim_ok(Dv))
        return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !o) return GDN_ERR_NULL;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, state, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return GDN_ERR_ALIGN;
    const size_t es = esize(io_dtype), eab = esize(ab_dtype);
    const Range rq{q, (size_t)B * HK * Dk * es}, rk{k, (size_t)B * HK * Dk * es};
    const Range rv{v, (size_t)B * HV * Dv * es}, ra{a, (size_t)B * HV * eab}, rb{b, (size_t)B * HV * eab};
    const Range rA{A_log, (size_t)HV * 4}, rd{dt_bias, (size_t)HV * 4};
    const Range rs{state, (size_t)B * HV * Dk * Dv * 4}, ro{o, (size_t)B * HV * Dv * es};
    for (Range out : {rs, ro})
        for (Range in : {rq, rk, rv, ra, rb, rA, rd})
            if (overlap(out, in)) return GDN_ERR_ALIAS;
    if (overlap(rs, ro)) return GDN_ERR_ALIAS;
    const gdn::DecodeGates gates{nullptr, nullptr, a, b, ab_dtype == GDN_BF16, A_log, dt_bias};
    return cuda_status(gdn::launch_decode(q, k, v, io_dtype == GDN_BF16, gates, state, B, HK, HV, Dk, Dv, scale,
                                          qk_l2norm ? 1 : 0, o, (cudaStream_t)stream));
}

}  // extern "C"

namespace {
// gdn_decode_step_fused, with the output epilogue when og.z is given
gdn_status decode_fused_impl(const void* x, gdn_dtype io_dtype, const float* conv_w, const float* conv_state_in,
                             float* conv_state_out, int32_t conv_act, const void* a, const void* b,
                             gdn_dtype ab_dtype, const float* A_log, const float* dt_bias, float* state, int32_t B,
                             int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm,
                             const gdn::DecodeOutGate& og, void* o, void* stream) {
    if (B < 0 || HK <= 0 || HV <= 0 || Dk <= 0 || Dv <= 0 || HV % HK != 0) return GDN_ERR_SHAPE;
    if (!dtype_ok(io_dtype) || !dtype_ok(ab_dtype) || Dk != 128 || Dv != 128 || (conv_act != 0 && conv_act != 1))
        return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!x || !conv_w || !conv_state_in || !conv_state_out || !a || !b || !A_log || !dt_bias || !state || !o)
        return GDN_ERR_NULL;
    const void* ptrs[] = {x, conv_w, conv_state_in, conv_state_out, a, b, A_log, dt_bias, state, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return GDN_ERR_ALIGN;
    const size_t C = (size_t)2 * HK * Dk + (size_t)HV * Dv;
    const size_t es = esize(io_dtype), eab = esize(ab_dtype);
    const Range rx{x, (size_t)B * C * es}, rw{conv_w, C * 16}, rci{conv_state_in, (size_t)B * C * 12};
    const Range rco{conv_state_out, (size_t)B * C * 12};
    const Range ra{a, (size_t)B * HV * eab}, rb{b, (size_t)B * HV * eab};
    const Range rA{A_log, (size_t)HV * 4}, rd{dt_bias, (size_t)HV * 4};
    const Range rs{state, (size_t)B * HV * Dk * Dv * 4}, ro{o, (size_t)B * HV * Dv * es};
    for (Range out : {rs, ro, rco})
        for (Range in : {rx, rw, rci, ra, rb, rA, rd})
            if (overlap(out, in)) return GDN_ERR_ALIAS;
    if (overlap(rs, ro) || overlap(rs, rco) || overlap(ro, rco)) return GDN_ERR_ALIAS;
    if (og.z) {   // the output epilogue's inputs
        if (!og.w) return GDN_ERR_NULL;
        if (!(og.eps >= 0.f)) return GDN_ERR_SHAPE;
        if (!aligned16(og.z) || !aligned16(og.w)) return GDN_ERR_ALIGN;
        const Range rz{og.z, (size_t)B * HV * Dv * es}, rw2{og.w, (size_t)Dv * 4};
        for (Range out : {rs, ro, rco})
            for (Range in : {rz, rw2})
                if (overlap(out, in)) return GDN_ERR_ALIAS;
    }
    const gdn::DecodeGates gates{nullptr, nullptr, a, b, ab_dtype == GDN_BF16, A_log, dt_bias};
    const gdn::DecodeConv conv{x, conv_w, conv_state_in, conv_state_out, conv_act};
    return cuda_status(gdn::launch_decode_conv(io_dtype == GDN_BF16, conv, gates, state, B, HK, HV, scale,
                                               qk_l2norm ? 1 : 0, o, og, (cudaStream_t)stream));
}
}  // namespace

extern "C" {

gdn_status gdn_decode_step_fused(const void* x, gdn_dtype io_dtype, const float* conv_w, const float* conv_state_in,
                                 float* conv_state_out, int32_t conv_act, const void* a, const void* b,
                                 gdn_dtype ab_dtype, const float* A_log, const float* dt_bias, float* state,
                                 int32_t B, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, float scale,
                                 int32_t qk_l2norm, void* o, void* stream) {
    return decode_fused_impl(x, io_dtype, conv_w, conv_state_in, conv_state_out, conv_act, a, b, ab_dtype, A_log,
                             dt_bias, state, B, HK, HV, Dk, Dv, scale, qk_l2norm, gdn::DecodeOutGate{}, o, stream);
}

gdn_status gdn_decode_step_fused_outgate(const void* x, gdn_dtype io_dtype, const float* conv_w,
                                         const float* conv_state_in, float* conv_state_out, int32_t conv_act,
                                         const void* a, const void* b, gdn_dtype ab_dtype, const float* A_log,
                                         const float* dt_bias, float* state, int32_t B, int32_t HK, int32_t HV,
                                         int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm, const void* z,
                                         const float* norm_w, float eps, void* o, void* stream) {
    if (!z) return GDN_ERR_NULL;
    return decode_fused_impl(x, io_dtype, conv_w, conv_state_in, conv_state_out, conv_act, a, b, ab_dtype, A_log,
                             dt_bias, state, B, HK, HV, Dk, Dv, scale, qk_l2norm, gdn::DecodeOutGate{z, norm_w, eps},
                             o, stream);
}

gdn_status gdn_conv_prefill(const void* x, gdn_dtype io_dtype, const float* conv_w, const float* conv_state_in,
                            const int32_t* cu_seqlens, int32_t B, int64_t T, int32_t n_seqs, int32_t HK,
                            int32_t HV, int32_t Dk, int32_t Dv, int32_t conv_act, void* q, void* k, void* v,
                            float* conv_state_out, void* stream) {
    if (B < 0 || T < 0 || n_seqs < 0 || HK <= 0 || HV <= 0) return GDN_ERR_SHAPE;
    if (cu_seqlens ? B != 1 : n_seqs != B) return GDN_ERR_SHAPE;
    if (!dtype_ok(io_dtype) || !head_dim_ok(Dk) || !head_dim_ok(Dv) || (conv_act != 0 && conv_act != 1))
        return GDN_ERR_UNSUPPORTED;
    const int64_t n_tok = (int64_t)B * T;
    const size_t C = (size_t)2 * HK * Dk + (size_t)HV * Dv;
    if (C > (size_t)INT32_MAX || (n_tok > 0 && (size_t)n_tok > SIZE_MAX / (C * 4))) return GDN_ERR_SHAPE;
    if (n_seqs == 0) return GDN_OK;
    if (!conv_w || (n_tok > 0 && (!x || !q || !k || !v))) return GDN_ERR_NULL;
    const void* ptrs[] = {x, conv_w, conv_state_in, cu_seqlens, q, k, v, conv_state_out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    const size_t es = esize(io_dtype), qk = (size_t)HK * Dk;
    const Range rx{x, (size_t)n_tok * C * es}, rw{conv_w, C * 16};
    const Range rci{conv_state_in, conv_state_in ? (size_t)n_seqs * C * 12 : 0};
    const Range rcu{cu_seqlens, cu_seqlens ? (size_t)(n_seqs + 1) * 4 : 0};
    const Range rq{q, (size_t)n_tok * qk * es}, rk{k, (size_t)n_tok * qk * es};
    const Range rv{v, (size_t)n_tok * HV * Dv * es};
    const Range rco{conv_state_out, conv_state_out ? (size_t)n_seqs * C * 12 : 0};
    for (Range out : {rq, rk, rv, rco})
        for (Range in : {rx, rw, rci, rcu})
            if (overlap(out, in)) return GDN_ERR_ALIAS;
    if (overlap(rq, rk) || overlap(rq, rv) || overlap(rk, rv) || overlap(rq, rco) || overlap(rk, rco) ||
        overlap(rv, rco))
        return GDN_ERR_ALIAS;
    return cuda_status(gdn::launch_conv_prefill(x, io_dtype == GDN_BF16, conv_w, conv_state_in, cu_seqlens, n_tok,
                                                T, n_seqs, (int)C, (int)qk, conv_act, q, k, v, conv_state_out,
                                                (cudaStream_t)stream));
}

gdn_status gdn_cp_combine(const float* A_all, const float* B_all, const float* initial_state, int32_t R,
                          int32_t rank, int32_t n_seqs, int64_t T_seg, int32_t HV, int32_t Dk, int32_t Dv,
                          gdn_dtype io_dtype, void* o, const void* c, float* start_state, float* final_state,
                          void* stream) {
    if (R < 1 || rank < 0 || rank >= R || n_seqs < 0 || T_seg < 0 || HV <= 0) return GDN_ERR_SHAPE;
    if (!dtype_ok(io_dtype) || Dk != 128 || Dv != 128) return GDN_ERR_UNSUPPORTED;
    // sizes the correction kernels address: 128-token tiles as a grid row (fp32), 32-bit tile
    // coordinates (bf16)
    if (io_dtype == GDN_F32 ? (T_seg + 127) / 128 > 65535 : (int64_t)n_seqs * T_seg > INT32_MAX - 128)
        return GDN_ERR_UNSUPPORTED;
    if (n_seqs == 0) return GDN_OK;
    if (!A_all || !B_all || !start_state || (T_seg > 0 && (!o || !c))) return GDN_ERR_NULL;
    const void* ptrs[] = {A_all, B_all, initial_state, o, c, start_state, final_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    const size_t nh = (size_t)n_seqs * HV, mat = (size_t)Dk * Dv * 4, es = esize(io_dtype);
    const Range rA{A_all, (size_t)R * nh * mat}, rB{B_all, (size_t)R * nh * mat};
    const Range rh{initial_state, initial_state ? nh * mat : 0};
    const Range ro{o, (size_t)T_seg * nh * Dv * es}, rc{c, (size_t)T_seg * nh * Dk * es};
    const Range rs{start_state, nh * mat}, rf{final_state, final_state ? nh * mat : 0};
    for (Range out : {ro, rs, rf})
        for (Range in : {rA, rB, rh, rc})
            if (overlap(out, in)) return GDN_ERR_ALIAS;
    if (overlap(ro, rs) || overlap(ro, rf) || overlap(rs, rf)) return GDN_ERR_ALIAS;
    return cuda_status(gdn::launch_cp_combine(A_all, B_all, initial_state, R, rank, n_seqs, T_seg, HV,
                                              io_dtype == GDN_BF16, o, c, start_state, final_state,
                                              (cudaStream_t)stream));
}

gdn_status gdn_cp_status(int32_t* device_error) {
    if (!device_error) return GDN_ERR_NULL;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    int32_t word = 0;
    e = gdn::read_cp_error(&word, true);
    if (e != cudaSuccess) return cuda_status(e);
    *device_error = word;
    return word ? GDN_ERR_DEVICE : GDN_OK;
}

gdn_status gdn_conv_status(int32_t* device_error) {
    if (!device_error) return GDN_ERR_NULL;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    int32_t word = 0;
    e = gdn::read_conv_error(&word, true);
    if (e != cudaSuccess) return cuda_status(e);
    *device_error = word;
    return word ? GDN_ERR_DEVICE : GDN_OK;
}

gdn_status gdn_decode_status(int32_t* device_error) {
    if (!device_error) return GDN_ERR_NULL;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    int32_t word = 0;
    e = gdn::read_decode_error(&word, true);
    if (e != cudaSuccess) return cuda_status(e);
    *device_error = word;
    return word ? GDN_ERR_DEVICE : GDN_OK;
}

}  // extern "C"
