// host_pipeline.cu -- gdn_chunk_prefill_host: the gates + chunked prefill of sequences held
// in host memory, streamed through the GPU in pieces of whole chunks so that the
// host -> device copies, the kernels and the device -> host copies of different pieces
// overlap (three internal streams, two buffer slots per direction).
//
// The state is carried from piece to piece in place in a device buffer (the prefill's
// initial_state == final_state form), which is exactly the chunk recurrence: a piece
// boundary is a chunk boundary because every piece but the last is a whole number of
// chunks.  The arithmetic of each piece is that of gdn_chunk_prefill; only the power-of-
// two data scale of the fp16 intermediates is chosen per piece instead of per sequence.
#include <cuda_runtime.h>

#include <mutex>

#include "gdn.h"
#include "gdn_internal.cuh"

namespace {

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
size_t esz(gdn_dtype d) { return d == GDN_BF16 ? 2 : 4; }

// Device workspace of one call, all offsets 256-byte aligned.
struct HostLayout {
    int64_t P;          // tokens per piece
    size_t state, A_log, dt_bias, g, beta, prefill_ws, prefill_ws_bytes;
    size_t q[2], k[2], v[2], a[2], b[2], o[2];
    size_t total;
};

bool host_layout(int32_t B, int64_t T, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t BT,
                 gdn_dtype io, gdn_dtype ab, int64_t piece_tokens, HostLayout* L) {
    if (B <= 0 || T < 0 || HK <= 0 || HV <= 0 || HV % HK != 0 || BT <= 0) return false;
    if (piece_tokens <= 0 || piece_tokens % BT != 0) return false;
    const int64_t P = T < piece_tokens ? (T > 0 ? T : BT) : piece_tokens;
    const size_t pws = gdn_chunk_prefill_workspace_bytes((int64_t)B * P, B, HK, HV, Dk, Dv, BT, io);
    if (pws == 0) return false;
    const size_t es = esz(io), eab = esz(ab);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = round_up(off + bytes, 256);
        return at;
    };
    L->P = P;
    L->state = take((size_t)B * HV * Dk * Dv * 4);
    L->A_log = take((size_t)HV * 4);
    L->dt_bias = take((size_t)HV * 4);
    L->g = take((size_t)B * P * HV * 4);
    L->beta = take((size_t)B * P * HV * 4);
    for (int s = 0; s < 2; ++s) {
        L->q[s] = take((size_t)B * P * HK * Dk * es);
        L->k[s] = take((size_t)B * P * HK * Dk * es);
        L->v[s] = take((size_t)B * P * HV * Dv * es);
        L->a[s] = take((size_t)B * P * HV * eab);
        L->b[s] = take((size_t)B * P * HV * eab);
        L->o[s] = take((size_t)B * P * HV * Dv * es);
    }
    L->prefill_ws_bytes = pws;
    L->prefill_ws = take(pws);
    L->total = off;
    return true;
}

// Streams and events of one device, created on first use and kept for the process.
struct Pipe {
    cudaStream_t in = nullptr, run = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr, run_done = nullptr;
    cudaEvent_t in_ready[2] = {}, in_free[2] = {}, out_ready[2] = {}, out_free[2] = {};
    bool used = false;   // `done` has been recorded by an earlier call
};
constexpr int kMaxDevices = 64;
std::mutex g_pipe_mu[kMaxDevices];
Pipe g_pipe[kMaxDevices];

cudaError_t pipe_init(Pipe& p) {
    if (p.in) return cudaSuccess;
    cudaError_t e = cudaSuccess;
    auto ev = [&](cudaEvent_t* x) {
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(x, cudaEventDisableTiming);
    };
    auto st = [&](cudaStream_t* x) {
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(x, cudaStreamNonBlocking);
    };
    st(&p.in);
    st(&p.run);
    st(&p.out);
    ev(&p.start);
    ev(&p.done);
    ev(&p.run_done);
    for (int s = 0; s < 2; ++s) {
        ev(&p.in_ready[s]);
        ev(&p.in_free[s]);
        ev(&p.out_ready[s]);
        ev(&p.out_free[s]);
    }
    return e;
}

// rows of `row_bytes` per token: tokens [t0, t0 + n) of each of B sequences of T tokens
cudaError_t copy_piece(void* dst, const void* src, size_t row_bytes, int B, int64_t T, int64_t t0, int64_t n,
                       cudaMemcpyKind kind, cudaStream_t s, bool to_device) {
    const size_t w = (size_t)n * row_bytes, full = (size_t)T * row_bytes;
    if (to_device)
        return cudaMemcpy2DAsync(dst, w, static_cast<const char*>(src) + (size_t)t0 * row_bytes, full, w, B, kind,
                                 s);
    return cudaMemcpy2DAsync(static_cast<char*>(dst) + (size_t)t0 * row_bytes, full, src, w, w, B, kind, s);
}

}  // namespace

extern "C" {

size_t gdn_chunk_prefill_host_workspace_bytes(int32_t B, int64_t T, int32_t HK, int32_t HV, int32_t Dk,
                                              int32_t Dv, int32_t BT, gdn_dtype io_dtype, gdn_dtype ab_dtype,
                                              int64_t piece_tokens) {
    if ((io_dtype != GDN_F32 && io_dtype != GDN_BF16) || (ab_dtype != GDN_F32 && ab_dtype != GDN_BF16)) return 0;
    HostLayout L;
    if (!host_layout(B, T, HK, HV, Dk, Dv, BT, io_dtype, ab_dtype, piece_tokens, &L)) return 0;
    return L.total;
}

gdn_status gdn_chunk_prefill_host(const void* q, const void* k, const void* v, gdn_dtype io_dtype, const void* a,
                                  const void* b, gdn_dtype ab_dtype, const float* A_log, const float* dt_bias,
                                  const float* initial_state, int32_t B, int64_t T, int32_t HK, int32_t HV,
                                  int32_t Dk, int32_t Dv, int32_t BT, float scale, int32_t qk_l2norm,
                                  int64_t piece_tokens, void* o, float* final_state, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    if (B < 0 || T < 0 || HK <= 0 || HV <= 0 || Dk <= 0 || Dv <= 0 || BT <= 0 || HV % HK != 0)
        return GDN_ERR_SHAPE;
    if (piece_tokens <= 0 || piece_tokens % BT != 0) return GDN_ERR_SHAPE;
    const size_t need =
        gdn_chunk_prefill_host_workspace_bytes(B > 0 ? B : 1, T, HK, HV, Dk, Dv, BT, io_dtype, ab_dtype, piece_tokens);
    if (need == 0) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || (T == 0 && final_state == nullptr)) return GDN_OK;
    if (!A_log || !dt_bias) return GDN_ERR_NULL;
    if (T > 0 && (!q || !k || !v || !a || !b || !o)) return GDN_ERR_NULL;
    if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_ALIGN;

    HostLayout L;
    host_layout(B, T, HK, HV, Dk, Dv, BT, io_dtype, ab_dtype, piece_tokens, &L);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_pipe_mu[dev]);   // one call's work is enqueued as a unit
    Pipe& p = g_pipe[dev];
    if ((e = pipe_init(p)) != cudaSuccess) return GDN_ERR_CUDA;

    char* ws = static_cast<char*>(workspace);
    float* d_state = reinterpret_cast<float*>(ws + L.state);
    float* d_Alog = reinterpret_cast<float*>(ws + L.A_log);
    float* d_dtb = reinterpret_cast<float*>(ws + L.dt_bias);
    float* d_g = reinterpret_cast<float*>(ws + L.g);
    float* d_beta = reinterpret_cast<float*>(ws + L.beta);
    const size_t es = esz(io_dtype), eab = esz(ab_dtype);
    const size_t rq = (size_t)HK * Dk * es, rv = (size_t)HV * Dv * es, rab = (size_t)HV * eab;
    const size_t state_bytes = (size_t)B * HV * Dk * Dv * 4;
    cudaStream_t user = (cudaStream_t)stream;

#define GDN_TRY(x)                               \
    do {                                         \
        if ((e = (x)) != cudaSuccess) return GDN_ERR_CUDA; \
    } while (0)
    // order after the caller's stream and after any earlier call on these streams
    GDN_TRY(cudaEventRecord(p.start, user));
    for (cudaStream_t s : {p.in, p.run, p.out}) {
        GDN_TRY(cudaStreamWaitEvent(s, p.start, 0));
        if (p.used) GDN_TRY(cudaStreamWaitEvent(s, p.done, 0));
    }
    GDN_TRY(cudaMemcpyAsync(d_Alog, A_log, (size_t)HV * 4, cudaMemcpyHostToDevice, p.run));
    GDN_TRY(cudaMemcpyAsync(d_dtb, dt_bias, (size_t)HV * 4, cudaMemcpyHostToDevice, p.run));
    if (initial_state) GDN_TRY(cudaMemcpyAsync(d_state, initial_state, state_bytes, cudaMemcpyHostToDevice, p.run));

    const bool fused_gates = io_dtype == GDN_BF16 && gdn::prefill_tc_supported(Dk, Dv, HK, HV, BT);
    const int64_t n_pieces = T > 0 ? (T + L.P - 1) / L.P : 0;
    for (int64_t i = 0; i < n_pieces; ++i) {
        const int sl = (int)(i & 1);
        const int64_t t0 = i * L.P, n = (T - t0) < L.P ? (T - t0) : L.P;
        // inputs of piece i into slot sl, once piece i - 2 has consumed it
        if (i >= 2) GDN_TRY(cudaStreamWaitEvent(p.in, p.in_free[sl], 0));
        GDN_TRY(copy_piece(ws + L.q[sl], q, rq, B, T, t0, n, cudaMemcpyHostToDevice, p.in, true));
        GDN_TRY(copy_piece(ws + L.k[sl], k, rq, B, T, t0, n, cudaMemcpyHostToDevice, p.in, true));
        GDN_TRY(copy_piece(ws + L.v[sl], v, rv, B, T, t0, n, cudaMemcpyHostToDevice, p.in, true));
        GDN_TRY(copy_piece(ws + L.a[sl], a, rab, B, T, t0, n, cudaMemcpyHostToDevice, p.in, true));
        GDN_TRY(copy_piece(ws + L.b[sl], b, rab, B, T, t0, n, cudaMemcpyHostToDevice, p.in, true));
        GDN_TRY(cudaEventRecord(p.in_ready[sl], p.in));
        // gates + prefill of piece i, the state carried in place
        GDN_TRY(cudaStreamWaitEvent(p.run, p.in_ready[sl], 0));
        if (i >= 2) GDN_TRY(cudaStreamWaitEvent(p.run, p.out_free[sl], 0));
        const float* h_in = (i > 0 || initial_state) ? d_state : nullptr;
        gdn_status st;
        if (fused_gates) {   // the tensor-core shapes form the gates inside the prefill
            st = gdn_chunk_prefill_gated(ws + L.q[sl], ws + L.k[sl], ws + L.v[sl], io_dtype, ws + L.a[sl],
                                         ws + L.b[sl], ab_dtype, d_Alog, d_dtb, h_in, nullptr, B, n, B, HK, HV, Dk,
                                         Dv, BT, scale, qk_l2norm, ws + L.o[sl], d_state, ws + L.prefill_ws,
                                         L.prefill_ws_bytes, p.run);
        } else {
            st = gdn_gates(ws + L.a[sl], ws + L.b[sl], ab_dtype, d_Alog, d_dtb, (int64_t)B * n, HV, d_g, d_beta, p.run);
            if (st != GDN_OK) return st;
            st = gdn_chunk_prefill(ws + L.q[sl], ws + L.k[sl], ws + L.v[sl], io_dtype, d_g, d_beta, h_in, nullptr, B, n,
                                   B, HK, HV, Dk, Dv, BT, scale, qk_l2norm, ws + L.o[sl], d_state, ws + L.prefill_ws,
                                   L.prefill_ws_bytes, p.run);
        }
        if (st != GDN_OK) return st;
        GDN_TRY(cudaEventRecord(p.in_free[sl], p.run));
        GDN_TRY(cudaEventRecord(p.out_ready[sl], p.run));
        // output of piece i back to the host
        GDN_TRY(cudaStreamWaitEvent(p.out, p.out_ready[sl], 0));
        GDN_TRY(copy_piece(o, ws + L.o[sl], rv, B, T, t0, n, cudaMemcpyDeviceToHost, p.out, false));
        GDN_TRY(cudaEventRecord(p.out_free[sl], p.out));
    }
    GDN_TRY(cudaEventRecord(p.run_done, p.run));
    GDN_TRY(cudaStreamWaitEvent(p.out, p.run_done, 0));
    if (final_state) {
        if (n_pieces == 0 && !initial_state) GDN_TRY(cudaMemsetAsync(d_state, 0, state_bytes, p.out));
        GDN_TRY(cudaMemcpyAsync(final_state, d_state, state_bytes, cudaMemcpyDeviceToHost, p.out));
    }
    GDN_TRY(cudaEventRecord(p.done, p.out));
    p.used = true;
    GDN_TRY(cudaStreamWaitEvent(user, p.done, 0));
#undef GDN_TRY
    return GDN_OK;
}

}  // extern "C"
