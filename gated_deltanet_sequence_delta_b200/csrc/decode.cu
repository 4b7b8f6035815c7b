// decode.cu -- one recurrent step of the gated delta rule per sequence, state updated
// in place (the incremental update of the "QWEN3.5" Q&A page, question 2a).
//
// With H = S^T (Dk x Dv, fp32) the pre-update state, unit-normalised k, q:
//     u     = H^T k                      (the current read along k)
//     delta = beta (v - alpha u)         (decay first, then the beta write)
//     H'    = alpha H + k delta^T
//     o     = scale H'^T q = scale (alpha H^T q + delta (k . q))
// so a single pass over H gives both reductions, and H' is written from the same
// registers: the state crosses HBM exactly once each way (2 x Dk x Dv x 4 bytes).
//
// One CTA per (sequence, value head).  Warp w owns rows 8w .. 8w+7 of H; lane l owns
// Dv/32 contiguous columns, so every warp load/store is a contiguous 8 x 512-byte
// (Dv = 128) burst of 128-bit accesses.  The Dk reduction is a per-thread sum over
// 8 rows, then a cross-warp sum through shared memory.
//
// For Dk = Dv = 128 a persistent variant streams the slices through shared memory: one CTA
// per SM, a producer warp keeps a ring of three slices in flight with bulk copies
// (64 KB of state plus the q, k, v rows per slice), sixteen warps update each slice in
// shared memory with the same arithmetic and mapping, and one thread writes it back with
// a bulk store.  HBM then sees a steady stream of loads and stores instead of the gaps
// between short-lived CTAs.
#include <mutex>
#include <type_traits>

#include "gdn_internal.cuh"
#include "tc_ptx.cuh"

namespace gdn {

// set (to GDN_DEVERR_TIMEOUT) by a staged decode launch whose bounded wait expired
__device__ int32_t g_decode_error = 0;

namespace {

template <int CPL>
struct VecF;
template <>
struct VecF<4> {
    using T = float4;
    static __device__ __forceinline__ void get(const T& x, float* f) {
        f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
    }
    static __device__ __forceinline__ T make(const float* f) { return make_float4(f[0], f[1], f[2], f[3]); }
};
template <>
struct VecF<2> {
    using T = float2;
    static __device__ __forceinline__ void get(const T& x, float* f) { f[0] = x.x; f[1] = x.y; }
    static __device__ __forceinline__ T make(const float* f) { return make_float2(f[0], f[1]); }
};

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(DK * 4, (DK == 128 ? 2 : 4))
decode_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
              const DecodeGates gates, float* __restrict__ state, int HK, int HV, float scale, int l2norm,
              IO* __restrict__ o) {
    constexpr int NW = DK / 8;      // warps; 8 state rows each
    constexpr int CPL = DV / 32;    // state columns per lane
    using V = VecF<CPL>;
    __shared__ float s_q[DK], s_k[DK];
    __shared__ float s_red_u[NW][DV], s_red_q[NW][DV];
    __shared__ float s_dot[3];

    const int bh = blockIdx.x;                 // b * HV + h
    const int b = bh / HV;
    const int h = bh - b * HV;
    const int hk = h / (HV / HK);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* Hp = state + (size_t)bh * DK * DV;

    // 1. the state slice, issued first so its latency overlaps the rest
    typename V::T hv[8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
        hv[r] = *reinterpret_cast<const typename V::T*>(Hp + (size_t)(warp * 8 + r) * DV + lane * CPL);

    // 2. q, k to shared memory; norms and k.q by three warps
    const int64_t qk_off = ((int64_t)b * HK + hk) * DK;
    for (int i = threadIdx.x; i < DK; i += blockDim.x) {
        s_q[i] = load_elem(q, qk_off + i);
        s_k[i] = load_elem(k, qk_off + i);
    }
    __syncthreads();
    if (warp < 3) {
        float acc = 0.f;
        for (int i = lane; i < DK; i += 32) {
            const float x = warp == 1 ? s_k[i] : s_q[i];
            const float y = warp == 0 ? s_q[i] : s_k[i];
            acc += x * y;   // warp 0: q.q, warp 1: k.k, warp 2: q.k
        }
        acc = warp_sum(acc);
        if (lane == 0) s_dot[warp] = acc;
    }

    // 3. per-thread partial reductions over its 8 rows (raw q, k; norms applied later)
    float pu[CPL], pq[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) pu[c] = pq[c] = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        float hf[CPL];
        V::get(hv[r], hf);
        const float kr = s_k[warp * 8 + r], qr = s_q[warp * 8 + r];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            pu[c] = fmaf(kr, hf[c], pu[c]);
            pq[c] = fmaf(qr, hf[c], pq[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        s_red_u[warp][lane * CPL + c] = pu[c];
        s_red_q[warp][lane * CPL + c] = pq[c];
    }
    __syncthreads();

    const float rq = l2_inv(s_dot[0], l2norm);
    const float rk = l2_inv(s_dot[1], l2norm);
    const float kq = s_dot[2] * rq * rk;
    float gv, bt;
    decode_gates(gates, bh, h, gv, bt);
    const float alpha = expf(gv);

    // 4. column sums, delta and the output (threads 0 .. DV-1); delta -> shared
    float* s_delta = &s_red_u[0][0];   // row 0 reused after its value is consumed
    if (threadIdx.x < DV) {
        const int j = threadIdx.x;
        float su = 0.f, sq = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            su += s_red_u[w][j];
            sq += s_red_q[w][j];
        }
        const float u = su * rk;
        const float vj = load_elem(v, (int64_t)bh * DV + j);
        const float delta = bt * (vj - alpha * u);
        store_elem(o, (int64_t)bh * DV + j, scale * (alpha * (sq * rq) + delta * kq));
        s_delta[j] = delta;   // each thread overwrites only the entry it has read
    }
    __syncthreads();

    // 5. H' = alpha H + k_hat delta^T, stored from registers
    float dl[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) dl[c] = s_delta[lane * CPL + c];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        float hf[CPL];
        V::get(hv[r], hf);
        const float kr = s_k[warp * 8 + r] * rk;
#pragma unroll
        for (int c = 0; c < CPL; ++c) hf[c] = fmaf(alpha, hf[c], kr * dl[c]);
        *reinterpret_cast<typename V::T*>(Hp + (size_t)(warp * 8 + r) * DV + lane * CPL) = V::make(hf);
    }
}

// ---- persistent, shared-memory staged variant (Dk = Dv = 128) --------------------------
constexpr int kSD = 128;                   // Dk = Dv of this variant
constexpr int kSStages = 3;
constexpr int kSWarps = 16;                // compute warps: rows 8w .. 8w+7 each
constexpr int kSThreads = kSWarps * 32 + 32;   // + producer warp
struct StagedSlot {
    float H[kSD * kSD];                    // the state slice, row-major as in global memory
    __align__(16) uint8_t q[kSD * 4], k[kSD * 4], v[kSD * 4];   // rows (io dtype, or fp32 with CONV)
};
struct ConvSlot {                          // CONV: this item's convolution inputs
    __align__(16) uint8_t x[3][kSD * 4];   // raw q, k, v channel rows (io dtype)
    float s[3][3][kSD];                    // state taps (oldest first) x (q, k, v) x channel
};
template <bool CONV>
struct StagedSmem {
    StagedSlot st[kSStages];
    // column partial sums: their own arrays, or (CONV, for room) the slot's state tile,
    // which is free between the reads of the old rows and the writes of the new ones
    float red[CONV ? 1 : 2][CONV ? 1 : kSWarps][CONV ? 1 : kSD];
    ConvSlot cv[CONV ? kSStages : 1];
    float delta[kSD];
    float dot[4];
    float osq[4];   // output epilogue: per warp of the row, its part of sum(o^2)
    uint64_t full[kSStages], empty[kSStages];
};
template <bool CONV>
constexpr size_t staged_smem_bytes() { return sizeof(StagedSmem<CONV>) + 128; }

template <typename IO>
__device__ __forceinline__ float ld_raw(const uint8_t* p, int i) {
    return load_elem(reinterpret_cast<const IO*>(p), i);
}

// CONV: q, k, v are not read from memory but formed from the raw projections by the
// convolution prologue (threads 0-383, one channel each: q, k, v rows of this item), kept
// in the slot as fp32.
// sigmoid(x) = (1 + tanh(x / 2)) / 2 from the hardware tanh (one special-function op, about
// 2^-11 relative error): an absolute gate error below 2^-12
__device__ __forceinline__ float sigmoid_tanh(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}

// OUTG (with CONV only): the output epilogue of the Qwen3-next page (section 3.2: a
// zero-centred RMSNorm, weight stored as w with the scale 1 + w) and the sigmoid output gate of
// the GDN resource-allocation page, on each output row before the store.
template <typename IO, bool CONV, bool OUTG = false>
__global__ void __launch_bounds__(kSThreads, 1)
decode_staged_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                     const DecodeConv conv, const DecodeGates gates, float* __restrict__ state, int n_items,
                     int HK, int HV, float scale, int l2norm, IO* __restrict__ o, int stall,
                     const DecodeOutGate og) {
    using QT = typename std::conditional<CONV, float, IO>::type;   // element type of the q, k, v rows
    constexpr int CPL = kSD / 32;   // 4 columns per lane
    constexpr uint32_t kRowBytes = kSD * sizeof(IO);
    constexpr uint32_t kTx = kSD * kSD * 4 + 3 * kRowBytes + (CONV ? 9 * kSD * 4 : 0);
    extern __shared__ uint8_t smem_raw[];
    StagedSmem<CONV>& S = *reinterpret_cast<StagedSmem<CONV>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int n_mine = blockIdx.x < n_items ? (n_items - 1 - blockIdx.x) / G + 1 : 0;
    if (tid == 0) {
        for (int i = 0; i < kSStages; ++i) {
            tc::mbar_init(&S.full[i], 1);
            tc::mbar_init(&S.empty[i], 1);
        }
        tc::fence_mbar_init();
    }
    __syncthreads();
    // launched with programmatic stream serialisation: the next step's CTAs take each SM as
    // this grid's CTA there exits (tc::grid_dependency_sync)
    tc::grid_dependency_sync();

    if (warp == kSWarps) {
        // ---------------- producer ----------------------------------------------------
        if (lane == 0) {
            for (int i = 0; i < n_mine; ++i) {
                const int st = i % kSStages, r = i / kSStages;
                if (r > 0 && !tc::mbar_wait(&S.empty[st], (r - 1) & 1)) {
                    atomicExch(&g_decode_error, GDN_DEVERR_TIMEOUT);
                    break;
                }
                // test hook (gdn_testing_stall): the first CTA's first item gets no copies, so
                // the compute warps' wait for it runs out
                if (stall && blockIdx.x == 0 && i == 0) continue;
                const int bh = blockIdx.x + i * G;
                const int b = bh / HV, h = bh - b * HV, hk = h / (HV / HK);
                StagedSlot& B = S.st[st];
                tc::mbar_expect_tx(&S.full[st], kTx);
                const float* src = state + (size_t)bh * kSD * kSD;
#pragma unroll
                for (int p = 0; p < 4; ++p) tc::bulk_load(B.H + p * 4096, src + p * 4096, 16384, &S.full[st]);
                if (!CONV) {
                    tc::bulk_load(B.q, q + ((size_t)b * HK + hk) * kSD, kRowBytes, &S.full[st]);
                    tc::bulk_load(B.k, k + ((size_t)b * HK + hk) * kSD, kRowBytes, &S.full[st]);
                    tc::bulk_load(B.v, v + (size_t)bh * kSD, kRowBytes, &S.full[st]);
                } else {   // x rows and state taps of the item's q, k, v channels
                    const int64_t C = (int64_t)2 * HK * kSD + (int64_t)HV * kSD;
                    const int64_t c0[3] = {(int64_t)hk * kSD, (int64_t)HK * kSD + (int64_t)hk * kSD,
                                           (int64_t)2 * HK * kSD + (int64_t)h * kSD};
                    ConvSlot& V = S.cv[st];
                    const IO* xb = reinterpret_cast<const IO*>(conv.x) + (int64_t)b * C;
#pragma unroll
                    for (int sg = 0; sg < 3; ++sg) {
                        tc::bulk_load(V.x[sg], xb + c0[sg], kRowBytes, &S.full[st]);
#pragma unroll
                        for (int tp = 0; tp < 3; ++tp)
                            tc::bulk_load(V.s[tp][sg], conv.state_in + ((int64_t)b * 3 + tp) * C + c0[sg], kSD * 4,
                                          &S.full[st]);
                    }
                }
            }
        }
        return;   // the producer takes part in no later barrier
    }

    // ---------------- 512 compute threads (named barrier 1) ------------------------------
    // convolution channel of this thread (CONV): seg 0 / 1 / 2 = q / k / v, d its index
    const int cseg = tid >> 7, cd = tid & (kSD - 1);
    const int64_t C = (int64_t)2 * HK * kSD + (int64_t)HV * kSD;
    auto conv_channel = [&](int item) -> int64_t {
        const int bh_ = item, b_ = bh_ / HV, h_ = bh_ - b_ * HV, hk_ = h_ / (HV / HK);
        return cseg < 2 ? (int64_t)cseg * HK * kSD + (int64_t)hk_ * kSD + cd : (int64_t)2 * HK * kSD + (int64_t)h_ * kSD + cd;
    };
    const float wj = OUTG && tid < kSD ? 1.f + og.w[tid] : 1.f;   // (1 + w) of output column tid
    float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);   // this item's taps (weights), an item ahead
    if (CONV && tid < 3 * kSD && n_mine > 0) cw = *reinterpret_cast<const float4*>(conv.w + conv_channel(blockIdx.x) * 4);
    for (int i = 0; i < n_mine; ++i) {
        const int st = i % kSStages, r = i / kSStages;
        const int bh = blockIdx.x + i * G;
        StagedSlot& B = S.st[st];
        float gv, bt;
        decode_gates(gates, bh, bh % HV, gv, bt);   // issued before the wait
        float zj = 0.f;   // the gate input of output column tid, also issued before the wait
        if (OUTG && tid < kSD) zj = load_elem(reinterpret_cast<const IO*>(og.z), (int64_t)bh * kSD + tid);
        const float alpha = expf(gv);
        const bool ok = tc::mbar_wait(&S.full[st], r & 1);
        if (tc::named_bar_any(1, kSWarps * 32, !ok)) {   // uniform decision to stop
            if (tid == 0) atomicExch(&g_decode_error, GDN_DEVERR_TIMEOUT);
            break;
        }
        if (CONV) {
            if (tid < 3 * kSD) {
                // y = w . (x_{t-3}, x_{t-2}, x_{t-1}, x_t), then the activation; the three
                // newest inputs go to state_out (q, k channels by the group's first value head)
                const ConvSlot& V = S.cv[st];
                const float s0 = V.s[0][cseg][cd], s1 = V.s[1][cseg][cd], s2 = V.s[2][cseg][cd];
                const float xc = ld_raw<IO>(V.x[cseg], cd);
                float y = cw.x * s0 + cw.y * s1 + cw.z * s2 + cw.w * xc;
                if (conv.act == 1) y = y / (1.f + expf(-y));
                float* row = reinterpret_cast<float*>(cseg == 0 ? B.q : cseg == 1 ? B.k : B.v);
                row[cd] = y;
                const int h = bh % HV;
                if (cseg == 2 || h % (HV / HK) == 0) {
                    float* so = conv.state_out + (int64_t)(bh / HV) * 3 * C + conv_channel(bh);
                    so[0] = s1;
                    so[C] = s2;
                    so[2 * C] = xc;
                }
                if (i + 1 < n_mine) cw = *reinterpret_cast<const float4*>(conv.w + conv_channel(bh + G) * 4);
            }
            tc::named_bar(1, kSWarps * 32);   // q, k, v of this item are in the slot
        }
        // norms and k.q (warps 0-2), partial column sums over this warp's 8 rows
        if (warp < 3) {
            float acc = 0.f;
            for (int e = lane; e < kSD; e += 32) {
                const float x = warp == 1 ? ld_raw<QT>(B.k, e) : ld_raw<QT>(B.q, e);
                const float y = warp == 0 ? ld_raw<QT>(B.q, e) : ld_raw<QT>(B.k, e);
                acc += x * y;   // warp 0: q.q, warp 1: k.k, warp 2: q.k
            }
            acc = warp_sum(acc);
            if (lane == 0) S.dot[warp] = acc;
        }
        float4 hv[8];
        float pu[CPL] = {}, pq[CPL] = {};
        float o_keep = 0.f;   // OUTG: this thread's output value, kept for the epilogue
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const int row = warp * 8 + rr;
            hv[rr] = *reinterpret_cast<const float4*>(B.H + row * kSD + lane * CPL);
            const float kr = ld_raw<QT>(B.k, row), qr = ld_raw<QT>(B.q, row);
            const float hf[4] = {hv[rr].x, hv[rr].y, hv[rr].z, hv[rr].w};
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                pu[c] = fmaf(kr, hf[c], pu[c]);
                pq[c] = fmaf(qr, hf[c], pq[c]);
            }
        }
        float* red_u = CONV ? B.H : &S.red[0][0][0];
        float* red_q = CONV ? B.H + kSWarps * kSD : &S.red[CONV ? 0 : 1][0][0];
        if (CONV) tc::named_bar(1, kSWarps * 32);   // every old row is in registers: the tile is scratch
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            red_u[warp * kSD + lane * CPL + c] = pu[c];
            red_q[warp * kSD + lane * CPL + c] = pq[c];
        }
        tc::named_bar(1, kSWarps * 32);
        const float rq = l2_inv(S.dot[0], l2norm);
        const float rk = l2_inv(S.dot[1], l2norm);
        const float kq = S.dot[2] * rq * rk;
        if (tid < kSD) {   // column sums, delta and the output
            const int j = tid;
            float su = 0.f, sq = 0.f;
#pragma unroll
            for (int w = 0; w < kSWarps; ++w) {
                su += red_u[w * kSD + j];
                sq += red_q[w * kSD + j];
            }
            const float delta = bt * (ld_raw<QT>(B.v, j) - alpha * su * rk);
            const float oj = scale * (alpha * (sq * rq) + delta * kq);
            S.delta[j] = delta;
            if (!OUTG) store_elem(o, (int64_t)bh * kSD + j, oj);
            else o_keep = oj;   // the output epilogue runs after the state update is under way
        }
        tc::named_bar(1, kSWarps * 32);
        // H' = alpha H + k_hat delta^T, written back in place
        const float4 dl = *reinterpret_cast<const float4*>(&S.delta[lane * CPL]);
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const int row = warp * 8 + rr;
            const float kr = ld_raw<QT>(B.k, row) * rk;
            float4 x = hv[rr];
            x.x = fmaf(alpha, x.x, kr * dl.x);
            x.y = fmaf(alpha, x.y, kr * dl.y);
            x.z = fmaf(alpha, x.z, kr * dl.z);
            x.w = fmaf(alpha, x.w, kr * dl.w);
            *reinterpret_cast<float4*>(B.H + row * kSD + lane * CPL) = x;
        }
        tc::fence_async_smem();
        tc::named_bar(1, kSWarps * 32);
        if (tid == 0) {
            float* dst = state + (size_t)bh * kSD * kSD;
#pragma unroll
            for (int p = 0; p < 4; ++p) tc::bulk_store(dst + p * 4096, B.H + p * 4096, 16384);
            tc::bulk_commit();
            tc::bulk_wait_read<1>();   // the previous slice's store has read its slot
            if (i > 0) tc::mbar_arrive(&S.empty[(i - 1) % kSStages]);
        }
        if (OUTG && tid < kSD) {
            // the output epilogue, behind the state update and its store: the row's mean square
            // over its 128 values from these four warps (one barrier among them), then the
            // norm, (1 + w) and the gate.  osq is rewritten only after the next item's CTA-wide
            // barrier, which every reader here has passed first.
            const float ss = warp_sum(o_keep * o_keep);
            if (lane == 0) S.osq[warp] = ss;
            tc::named_bar(2, kSD);
            const float ms = (S.osq[0] + S.osq[1] + S.osq[2] + S.osq[3]) * (1.f / kSD);
            store_elem(o, (int64_t)bh * kSD + tid, o_keep * rsqrtf(ms + og.eps) * wj * sigmoid_tanh(zj));
        }
    }
    if (tid == 0) tc::bulk_wait<0>();   // every store complete before the CTA exits
}

int staged_grid() {
    static std::mutex mu;
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        sms[dev] = n;
    }
    return sms[dev];
}

template <typename IO, bool CONV, bool OUTG = false>
cudaError_t launch_decode_staged(const void* q, const void* k, const void* v, const DecodeConv& conv,
                                 const DecodeGates& gates, float* state, int B, int HK, int HV, float scale,
                                 int l2norm, void* o, cudaStream_t s, const DecodeOutGate& og = DecodeOutGate{}) {
    const int n_items = B * HV;
    const int sms = staged_grid();
    if (sms <= 0) return cudaErrorInvalidDevice;
    constexpr size_t smem = staged_smem_bytes<CONV>();
    static_assert(smem <= 227 * 1024, "staged decode: shared memory over the per-block limit");
    cudaError_t e = cudaFuncSetAttribute(decode_staged_kernel<IO, CONV, OUTG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = n_items < sms ? n_items : sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kSThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddepcontrol in the kernel
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_staged_kernel<IO, CONV, OUTG>, (const IO*)q, (const IO*)k, (const IO*)v, conv,
                           gates, state, n_items, HK, HV, scale, l2norm, (IO*)o,
                           testing_stall_site() == GDN_STALL_DECODE ? 1 : 0, og);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

template <int DK, int DV, typename IO>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const DecodeGates& gates,
                            float* state, int B, int HK, int HV, float scale, int l2norm, void* o,
                            cudaStream_t s) {
    const unsigned blocks = (unsigned)B * (unsigned)HV;
    decode_kernel<DK, DV, IO><<<blocks, DK * 4, 0, s>>>(
        (const IO*)q, (const IO*)k, (const IO*)v, gates, state, HK, HV, scale, l2norm, (IO*)o);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, bool bf16, const DecodeGates& gates,
                          float* state, int B, int HK, int HV, int Dk, int Dv, float scale, int l2norm, void* o,
                          cudaStream_t s) {
    if (B == 0) return cudaSuccess;
    const DecodeConv none{nullptr, nullptr, nullptr, nullptr, 0};
    if (Dk == kSD && Dv == kSD)   // the API guarantees 16-byte aligned pointers
        return bf16 ? launch_decode_staged<__nv_bfloat16, false>(q, k, v, none, gates, state, B, HK, HV, scale,
                                                                 l2norm, o, s)
                    : launch_decode_staged<float, false>(q, k, v, none, gates, state, B, HK, HV, scale, l2norm, o, s);
#define GDN_DECODE_CASE(DK_, DV_)                                                                  \
    if (Dk == DK_ && Dv == DV_)                                                                    \
        return bf16 ? launch_decode_t<DK_, DV_, __nv_bfloat16>(q, k, v, gates, state, B, HK, HV, scale, \
                                                               l2norm, o, s)                       \
                    : launch_decode_t<DK_, DV_, float>(q, k, v, gates, state, B, HK, HV, scale, l2norm, o, s);
    GDN_DECODE_CASE(128, 64)
    GDN_DECODE_CASE(64, 128)
    GDN_DECODE_CASE(64, 64)
#undef GDN_DECODE_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_conv(bool bf16, const DecodeConv& conv, const DecodeGates& gates, float* state, int B,
                               int HK, int HV, float scale, int l2norm, void* o, const DecodeOutGate& og,
                               cudaStream_t s) {
    if (B == 0) return cudaSuccess;
    if (og.z)
        return bf16 ? launch_decode_staged<__nv_bfloat16, true, true>(nullptr, nullptr, nullptr, conv, gates, state, B,
                                                                      HK, HV, scale, l2norm, o, s, og)
                    : launch_decode_staged<float, true, true>(nullptr, nullptr, nullptr, conv, gates, state, B, HK, HV,
                                                              scale, l2norm, o, s, og);
    return bf16 ? launch_decode_staged<__nv_bfloat16, true>(nullptr, nullptr, nullptr, conv, gates, state, B, HK, HV,
                                                            scale, l2norm, o, s)
                : launch_decode_staged<float, true>(nullptr, nullptr, nullptr, conv, gates, state, B, HK, HV, scale,
                                                    l2norm, o, s);
}

cudaError_t read_decode_error(int32_t* out, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_decode_error, sizeof(int32_t));
    if (e == cudaSuccess && reset && *out != 0) {
        const int32_t zero = 0;
        e = cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(int32_t));
    }
    return e;
}

}  // namespace gdn
