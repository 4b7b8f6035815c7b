// cp_combine.cu -- the exchange step of a context-parallel prefill.  One sequence is cut
// into R consecutive segments, one per rank.  Over a segment the gated delta rule is affine
// in the state it starts from (the product form of the "Gated DeltaNet" research log's
// update rule; with H = S^T):
//     H_end = A H_start + B,     o_t = o0_t + H_start^T c_t
// where B and o0 come from running the segment from a zero state, and A and c from running
// it with v = 0 from H_start = I (A = the product of the segment's transitions, c_t =
// scale A_{<=t}^T q_t).  Given every segment's (A, B), each rank finds its own H_start by
// the scan H_start(0) = h0, H_start(r + 1) = A_r H_start(r) + B_r and corrects its outputs.
// All matrices are 128 x 128 fp32 per (sequence, value head); the products run on CUDA
// cores in fp32 (the state's precision), staged through shared memory.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int DD = 128;           // Dk = Dv of this path
constexpr int THREADS = 256;      // thread t: row t / 2, columns 64 (t % 2) .. +63
// Shared-memory layouts of the 128 x 128 fp32 operands, free of bank conflicts for the
// reads below: Y rows padded to 129 floats (a warp's 16 rows fall in 16 banks); X rows of
// 136 floats with the second 64-column half shifted by 4 (the two halves' broadcast reads
// fall in different banks)
constexpr int YS = DD + 1, XS = DD + 8;
__device__ __forceinline__ int yidx(int i, int k) { return i * YS + k; }
__device__ __forceinline__ int xidx(int k, int j) { return k * XS + j + ((j >> 6) << 2); }

// out[jj] (+)= sum_k Y[i][k] X[k][64 h + jj] for this thread's row i and column half h
__device__ __forceinline__ void row_times(const float* Y, const float* X, int i, int h, float* out) {
#pragma unroll 4
    for (int k = 0; k < DD; ++k) {
        const float y = Y[yidx(i, k)];
        const float4* xr = reinterpret_cast<const float4*>(X + xidx(k, 64 * h));
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float4 x = xr[q];
            out[4 * q] = fmaf(y, x.x, out[4 * q]);
            out[4 * q + 1] = fmaf(y, x.y, out[4 * q + 1]);
            out[4 * q + 2] = fmaf(y, x.z, out[4 * q + 2]);
            out[4 * q + 3] = fmaf(y, x.w, out[4 * q + 3]);
        }
    }
}

struct ScanSmem {
    float Y[DD * YS];            // A_r
    float X[DD * XS];            // the running state H
};

// One CTA per (sequence, value head): H = h0; for r = 0 .. R-1: (r == rank: H is this rank's
// start state) H = A_r H + B_r; finally H is the sequence's end state.
__global__ void __launch_bounds__(THREADS) cp_scan_kernel(const float* __restrict__ A_all,
                                                          const float* __restrict__ B_all,
                                                          const float* __restrict__ h0, int R, int rank,
                                                          int64_t nh, float* __restrict__ start_state,
                                                          float* __restrict__ final_state) {
    extern __shared__ uint8_t smem_raw[];
    ScanSmem& S = *reinterpret_cast<ScanSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, i = tid >> 1, h = tid & 1;
    const int64_t m = blockIdx.x;   // (sequence, value head)
    for (int e = tid; e < DD * DD; e += THREADS) S.X[xidx(e / DD, e % DD)] = h0 ? h0[m * DD * DD + e] : 0.f;
    __syncthreads();
    for (int r = 0; r < R; ++r) {
        const float* A = A_all + ((int64_t)r * nh + m) * DD * DD;
        const float* Bm = B_all + ((int64_t)r * nh + m) * DD * DD;
        if (r == rank && start_state)
            for (int e = tid; e < DD * DD; e += THREADS) start_state[m * DD * DD + e] = S.X[xidx(e / DD, e % DD)];
        for (int e = tid; e < DD * DD; e += THREADS) S.Y[yidx(e / DD, e % DD)] = A[e];
        __syncthreads();
        float out[64];
        const float4* br = reinterpret_cast<const float4*>(Bm + i * DD + 64 * h);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float4 b = br[q];
            out[4 * q] = b.x;
            out[4 * q + 1] = b.y;
            out[4 * q + 2] = b.z;
            out[4 * q + 3] = b.w;
        }
        row_times(S.Y, S.X, i, h, out);
        __syncthreads();   // every read of H precedes its overwrite
        float4* xr = reinterpret_cast<float4*>(S.X + xidx(i, 64 * h));
#pragma unroll
        for (int q = 0; q < 16; ++q) xr[q] = make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
        __syncthreads();
    }
    if (final_state)
        for (int e = tid; e < DD * DD; e += THREADS) final_state[m * DD * DD + e] = S.X[xidx(e / DD, e % DD)];
}

struct CorrSmem {
    float Y[DD * YS];            // c rows of 128 tokens (rows past the segment zero)
    float X[DD * XS];            // H_start
};

template <typename IO>
__device__ __forceinline__ float io_to_f(IO x);
template <> __device__ __forceinline__ float io_to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float io_to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename IO>
__device__ __forceinline__ IO f_to_io(float x);
template <> __device__ __forceinline__ float f_to_io<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 f_to_io<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// o[n, t, h, :] += H_start[n, h]^T c[n, t, h, :] for 128 tokens t of the segment per CTA;
// grid (n_seqs * HV, token tiles).  o and c: [n_seqs, T_seg, HV, 128].
template <typename IO>
__global__ void __launch_bounds__(THREADS) cp_correct_kernel(const float* __restrict__ start, const IO* __restrict__ c,
                                                             IO* __restrict__ o, int64_t T_seg, int HV) {
    extern __shared__ uint8_t smem_raw[];
    CorrSmem& S = *reinterpret_cast<CorrSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, i = tid >> 1, h = tid & 1;
    const int64_t m = blockIdx.x;          // (sequence, value head)
    const int64_t n = m / HV, hv = m % HV;
    const int64_t t0 = (int64_t)blockIdx.y * DD;
    for (int e = tid; e < DD * DD; e += THREADS) {
        S.X[xidx(e / DD, e % DD)] = start[m * DD * DD + e];
        const int64_t t = t0 + e / DD;
        S.Y[yidx(e / DD, e % DD)] = t < T_seg ? io_to_f<IO>(c[((n * T_seg + t) * HV + hv) * DD + e % DD]) : 0.f;
    }
    __syncthreads();
    const int64_t t = t0 + i;
    if (t >= T_seg) return;
    IO* orow = o + ((n * T_seg + t) * HV + hv) * DD + 64 * h;
    float out[64];
#pragma unroll
    for (int jj = 0; jj < 64; ++jj) out[jj] = io_to_f<IO>(orow[jj]);
    row_times(S.Y, S.X, i, h, out);
#pragma unroll
    for (int jj = 0; jj < 64; ++jj) orow[jj] = f_to_io<IO>(out[jj]);
}

}  // namespace

cudaError_t launch_cp_combine(const float* A_all, const float* B_all, const float* h0, int R, int rank, int n_seqs,
                              int64_t T_seg, int HV, bool bf16, void* o, const void* c, float* start_state,
                              float* final_state, cudaStream_t s) {
    const int64_t nh = (int64_t)n_seqs * HV;
    if (nh == 0) return cudaSuccess;
    const size_t smem = sizeof(ScanSmem) + 16;
    static_assert(sizeof(ScanSmem) == sizeof(CorrSmem), "one shared-memory size for both kernels");
    cudaError_t e = cudaFuncSetAttribute(cp_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cp_scan_kernel<<<(unsigned)nh, THREADS, smem, s>>>(A_all, B_all, h0, R, rank, nh, start_state, final_state);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    if (T_seg == 0) return cudaSuccess;
    const dim3 grid((unsigned)nh, (unsigned)((T_seg + DD - 1) / DD));
    if (bf16) {
        e = cudaFuncSetAttribute(cp_correct_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        cp_correct_kernel<__nv_bfloat16><<<grid, THREADS, smem, s>>>(start_state, (const __nv_bfloat16*)c,
                                                                      (__nv_bfloat16*)o, T_seg, HV);
    } else {
        e = cudaFuncSetAttribute(cp_correct_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        cp_correct_kernel<float><<<grid, THREADS, smem, s>>>(start_state, (const float*)c, (float*)o, T_seg, HV);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace gdn
