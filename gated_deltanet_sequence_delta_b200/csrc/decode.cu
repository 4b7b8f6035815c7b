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
#include "gdn_internal.cuh"

namespace gdn {
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
              const float* __restrict__ g, const float* __restrict__ beta,
              float* __restrict__ state, int HK, int HV, float scale, int l2norm,
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
    const float alpha = expf(g[bh]);
    const float bt = beta[bh];

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

template <int DK, int DV, typename IO>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, float* state, int B, int HK, int HV, float scale,
                            int l2norm, void* o, cudaStream_t s) {
    const unsigned blocks = (unsigned)B * (unsigned)HV;
    decode_kernel<DK, DV, IO><<<blocks, DK * 4, 0, s>>>(
        (const IO*)q, (const IO*)k, (const IO*)v, g, beta, state, HK, HV, scale, l2norm, (IO*)o);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, bool bf16,
                          const float* g, const float* beta, float* state, int B, int HK,
                          int HV, int Dk, int Dv, float scale, int l2norm, void* o,
                          cudaStream_t s) {
    if (B == 0) return cudaSuccess;
#define GDN_DECODE_CASE(DK_, DV_)                                                                \
    if (Dk == DK_ && Dv == DV_)                                                                  \
        return bf16 ? launch_decode_t<DK_, DV_, __nv_bfloat16>(q, k, v, g, beta, state, B, HK,   \
                                                               HV, scale, l2norm, o, s)          \
                    : launch_decode_t<DK_, DV_, float>(q, k, v, g, beta, state, B, HK, HV,       \
                                                       scale, l2norm, o, s);
    GDN_DECODE_CASE(128, 128)
    GDN_DECODE_CASE(128, 64)
    GDN_DECODE_CASE(64, 128)
    GDN_DECODE_CASE(64, 64)
#undef GDN_DECODE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace gdn
