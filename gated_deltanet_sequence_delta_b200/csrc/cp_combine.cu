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
#include "tc_ptx.cuh"

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

template <typename IO>
__device__ __forceinline__ float io_to_f(IO x);
template <> __device__ __forceinline__ float io_to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float io_to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename IO>
__device__ __forceinline__ IO f_to_io(float x);
template <> __device__ __forceinline__ float f_to_io<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 f_to_io<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// The correction O (+)= C H_start for 128 tokens of one (sequence, value head): thread
// (ty, tx) of a 16 x 16 grid owns tokens 8 ty .. 8 ty + 7 and values 8 tx .. 8 tx + 7, so that
// per k it reads 8 + 8 operands (four 16-byte loads) for 64 FMAs.  C sits transposed in
// shared memory (k-major, rows of 132 floats), H_start row-major.
constexpr int CTS = DD + 4;
struct CorrSmem {
    float Ct[DD * CTS];          // Ct[k][t] = c of token t, component k (tokens past the segment zero)
    float H[DD * DD];            // H_start[k][j]
};

template <typename IO>
__global__ void __launch_bounds__(THREADS) cp_correct_kernel(const float* __restrict__ start, const IO* __restrict__ c,
                                                             IO* __restrict__ o, int64_t T_seg, int HV) {
    extern __shared__ uint8_t smem_raw[];
    CorrSmem& S = *reinterpret_cast<CorrSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int64_t m = blockIdx.x;          // (sequence, value head)
    const int64_t n = m / HV, hv = m % HV;
    const int64_t t0 = (int64_t)blockIdx.y * DD;
    for (int e = tid * 4; e < DD * DD; e += THREADS * 4)
        *reinterpret_cast<float4*>(S.H + e) = *reinterpret_cast<const float4*>(start + m * DD * DD + e);
    for (int e = tid; e < DD * DD; e += THREADS) {   // consecutive threads: consecutive k of a token
        const int tt = e / DD, kk = e % DD;
        const int64_t t = t0 + tt;
        S.Ct[kk * CTS + tt] = t < T_seg ? io_to_f<IO>(c[((n * T_seg + t) * HV + hv) * DD + kk]) : 0.f;
    }
    __syncthreads();
    float acc[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[r][j] = 0.f;
#pragma unroll 2
    for (int k = 0; k < DD; ++k) {
        const float4 a0 = *reinterpret_cast<const float4*>(S.Ct + k * CTS + 8 * ty);
        const float4 a1 = *reinterpret_cast<const float4*>(S.Ct + k * CTS + 8 * ty + 4);
        const float4 b0 = *reinterpret_cast<const float4*>(S.H + k * DD + 8 * tx);
        const float4 b1 = *reinterpret_cast<const float4*>(S.H + k * DD + 8 * tx + 4);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[r][j] = fmaf(a[r], b[j], acc[r][j]);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int64_t t = t0 + 8 * ty + r;
        if (t >= T_seg) break;
        IO* orow = o + ((n * T_seg + t) * HV + hv) * DD + 8 * tx;
#pragma unroll
        for (int j = 0; j < 8; ++j) orow[j] = f_to_io<IO>(io_to_f<IO>(orow[j]) + acc[r][j]);
    }
}

// ---- bf16: the correction on the tensor cores ---------------------------------------------
// Per 128-token tile, D[128 tokens x 128 values] = C[128 x 128] H_start as eight tcgen05 MMAs
// (bf16, M = N = 128, K = 16 each) into 128 TMEM columns; the epilogue adds o0 and stores.
// A CTA owns one (sequence, value head) and walks token tiles b, b + per_head, ...: it writes
// H_start^T once as bf16 in the 128B-swizzled K-major layout (thread t: row t, i.e. column t
// of H_start, read with coalesced loads across the warp) and streams the c tiles by TMA
// through two stages, the next tile loading while the current one is multiplied and
// written.  H_start in bf16 is the one rounding beyond the output's own.
struct CorrTcSmem {
    uint8_t A[2][2][128 * 128];  // c tiles by stage, halves k 0-63 / 64-127: 128 rows x 128 bytes
    uint8_t Bt[2][128 * 128];    // H_start^T, same layout (row n = value column)
    uint64_t full[2], bar_mma;
    uint32_t tmem_base;
};
constexpr size_t kCorrTcSmemBytes = sizeof(CorrTcSmem) + 1024;

__device__ int32_t g_cp_error = 0;

__global__ void __launch_bounds__(128) cp_correct_tc_kernel(const __grid_constant__ CUtensorMap tm_c,
                                                            const float* __restrict__ start,
                                                            __nv_bfloat16* __restrict__ o, int64_t T_seg, int HV,
                                                            int per_head) {
    extern __shared__ uint8_t smem_raw[];
    CorrTcSmem& S = *reinterpret_cast<CorrTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t m = blockIdx.x / per_head, n = m / HV, hv = m % HV;
    const int j0 = blockIdx.x % per_head;
    const int n_tiles = (int)((T_seg + DD - 1) / DD);
    const int mine = j0 < n_tiles ? (n_tiles - 1 - j0) / per_head + 1 : 0;
    if (warp == 0) {
        tc::tmem_alloc(&S.tmem_base, 128);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        tc::mbar_init(&S.full[0], 1);
        tc::mbar_init(&S.full[1], 1);
        tc::mbar_init(&S.bar_mma, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    auto load_tile = [&](int i) {   // this CTA's i-th tile into stage i % 2 (thread 0)
        const int st = i & 1;
        const int64_t row = n * T_seg + (int64_t)(j0 + i * per_head) * DD;
        tc::mbar_expect_tx(&S.full[st], 2 * 128 * 128);
        tc::tma_load_3d(S.A[st][0], &tm_c, &S.full[st], 0, (int)hv, (int)row);
        tc::tma_load_3d(S.A[st][1], &tm_c, &S.full[st], 64, (int)hv, (int)row);
    };
    if (tid == 0)
        for (int i = 0; i < 2 && i < mine; ++i) load_tile(i);
    {   // H_start^T, row tid: for each 8 k, one 16-byte piece of bf16
        const float* H = start + m * DD * DD + tid;
#pragma unroll 4
        for (int kc = 0; kc < 16; ++kc) {
            __align__(16) __nv_bfloat162 h[4];
#pragma unroll
            for (int p = 0; p < 4; ++p)
                h[p] = __floats2bfloat162_rn(H[(kc * 8 + 2 * p) * DD], H[(kc * 8 + 2 * p + 1) * DD]);
            *reinterpret_cast<uint4*>(S.Bt[kc >> 3] + tc::sw128_off(tid, (kc & 7) * 8)) =
                *reinterpret_cast<const uint4*>(h);
        }
    }
    tc::fence_async_smem();
    int issued = mine < 2 ? mine : 2;   // tiles whose copies thread 0 has started
    int landed = 0;                     // tiles whose copies completed and were waited for
    int products = 0;                   // MMA groups thread 0 has committed to bar_mma
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int i = 0; i < mine; ++i) {
        const int st = i & 1;
        bool ok = tc::mbar_wait(&S.full[st], (uint32_t)((i >> 1) & 1));
        tc::tc_fence_before();
        if (__syncthreads_or(!ok)) {   // (also orders every thread's H_start^T writes before the MMA)
            if (tid == 0) atomicExch(&g_cp_error, GDN_DEVERR_TIMEOUT);
            break;
        }
        landed = i + 1;
        if (tid == 0) {
            tc::tc_fence_after();
            const uint32_t a0 = tc::smem_u32(S.A[st][0]), b0 = tc::smem_u32(S.Bt[0]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                tc::mma_bf16(tmem, tc::desc_sw128(a0 + off, 16, 1024), tc::desc_sw128(b0 + off, 16, 1024),
                             tc::idesc_bf16(128, 128, 0, 0), kk > 0);
            }
            tc::mma_commit(&S.bar_mma);
            ++products;
        }
        ok = tc::mbar_wait(&S.bar_mma, (uint32_t)(i & 1));
        tc::tc_fence_after();
        if (tid == 0 && ok && i + 2 < mine) {   // the stage's tile is consumed: tile i + 2
            load_tile(i + 2);
            ++issued;
        }
        // epilogue: thread t <-> TMEM lane t <-> token row t of the tile
        const int64_t t = (int64_t)(j0 + i * per_head) * DD + tid;
        __nv_bfloat16* orow = o + ((n * T_seg + t) * HV + hv) * DD;
#pragma unroll
        for (int part = 0; part < 4; ++part) {
            float acc[32];
            tc::tmem_ld32(tmem + lane_base + part * 32, acc);   // the whole warp, every row
            tc::tmem_wait_ld();
            if (ok && t < T_seg) {
                uint4* dst = reinterpret_cast<uint4*>(orow + part * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 u = dst[q];
                    __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float2 f = __bfloat1622float2(e[p]);
                        e[p] = __floats2bfloat162_rn(f.x + acc[q * 8 + 2 * p], f.y + acc[q * 8 + 2 * p + 1]);
                    }
                    dst[q] = u;
                }
            }
        }
        tc::tc_fence_before();
        if (__syncthreads_or(!ok)) {   // TMEM read out before the next tile's MMA overwrites it
            if (tid == 0) atomicExch(&g_cp_error, GDN_DEVERR_TIMEOUT);
            break;
        }
    }
    if (tid == 0) {   // copies started but never waited for (a wait gave up) land before the CTA leaves;
                      // each is the latest use of its stage, so its parity is the one still pending
        for (int i = landed; i < issued; ++i) (void)tc::mbar_wait(&S.full[i & 1], (uint32_t)((i >> 1) & 1), 50000000ull);
        // so does the latest MMA group, which may still read the tiles and write TMEM (at once
        // if it completed)
        if (products > 0) (void)tc::mbar_wait(&S.bar_mma, (uint32_t)((products - 1) & 1), 50000000ull);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

}  // namespace

cudaError_t read_cp_error(int32_t* out, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_cp_error, sizeof(int32_t));
    if (e == cudaSuccess && reset) {
        const int32_t zero = 0;
        e = cudaMemcpyToSymbol(g_cp_error, &zero, sizeof(int32_t));
    }
    return e;
}

cudaError_t launch_cp_combine(const float* A_all, const float* B_all, const float* h0, int R, int rank, int n_seqs,
                              int64_t T_seg, int HV, bool bf16, void* o, const void* c, float* start_state,
                              float* final_state, cudaStream_t s) {
    const int64_t nh = (int64_t)n_seqs * HV;
    if (nh == 0) return cudaSuccess;
    const size_t smem = sizeof(ScanSmem) + 16;
    static_assert(sizeof(CorrSmem) <= sizeof(ScanSmem), "one shared-memory size for both kernels");
    cudaError_t e = cudaFuncSetAttribute(cp_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cp_scan_kernel<<<(unsigned)nh, THREADS, smem, s>>>(A_all, B_all, h0, R, rank, nh, start_state, final_state);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    if (T_seg == 0) return cudaSuccess;
    const dim3 grid((unsigned)nh, (unsigned)((T_seg + DD - 1) / DD));
    CUtensorMap tm;
    if (bf16 && (int64_t)n_seqs * T_seg <= INT32_MAX - DD) {
        // c [n_seqs * T_seg, HV, 128] bf16 in boxes of 64 columns x 128 tokens of one head
        const cuuint64_t dims[3] = {(cuuint64_t)DD, (cuuint64_t)HV, (cuuint64_t)(n_seqs * T_seg)};
        const cuuint64_t str[2] = {(cuuint64_t)DD * 2, (cuuint64_t)HV * DD * 2};
        const cuuint32_t box[3] = {64, 1, DD};
        if (make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) {
            e = cudaFuncSetAttribute(cp_correct_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kCorrTcSmemBytes);
            if (e != cudaSuccess) return e;
            // per (sequence, value head) a share of about two CTAs per SM in all
            int dev = 0, sms = 148;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            const int64_t n_tiles = (T_seg + DD - 1) / DD;
            int64_t per_head = 2 * (int64_t)sms / nh;
            if (per_head < 1) per_head = 1;
            if (per_head > n_tiles) per_head = n_tiles;
            cp_correct_tc_kernel<<<(unsigned)(nh * per_head), 128, kCorrTcSmemBytes, s>>>(
                tm, start_state, (__nv_bfloat16*)o, T_seg, HV, (int)per_head);
            e = cudaGetLastError();
            if (e == cudaSuccess) count_launch();
            return e;
        }
    }
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
