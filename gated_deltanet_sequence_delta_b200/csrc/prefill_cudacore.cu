// prefill_cudacore.cu -- chunked prefill of the gated delta rule on CUDA cores (fp32
// arithmetic throughout, no tensor cores, no TF32).  It is the fp32-mode kernel.
//
// Time is cut into chunks of BT tokens; inside a chunk the work is parallel and the
// state is carried serially from chunk to chunk ("QWEN3.5" Q&A page, question 1).
// The chunk equations follow from the recurrence alone.  With H0 = S^T (Dk x Dv) the
// state at the chunk start, rows k_i, q_i (L2-normalised), v_i, and G_i the running
// sum of g inside the chunk (gamma_i = exp(G_i)):
//     (I + L) Delta = diag(beta) V - diag(beta gamma) K H0,
//         L_ij = beta_i exp(G_i - G_j) k_i . k_j           (i > j)
//     O   = scale (diag(gamma) Q H0 + P Delta),  P_ij = exp(G_i - G_j) q_i . k_j   (i >= j)
//     H_C = gamma_C H0 + (diag(exp(G_C - G)) K)^T Delta
// Every exponent evaluated is <= 0.  The value columns of H evolve independently (k,
// alpha, beta are shared), so each CTA owns one 32-column slice of one value head of
// one sequence and needs no communication.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int VS = 32;        // value columns per CTA
constexpr int NT = 256;       // threads per CTA
constexpr int NWARP = NT / 32;

template <int DK, int BT>
struct CCSmem {
    // floats
    static constexpr int kKT = 0;                       // [DK][BT]  normalised k, transposed
    static constexpr int kQT = kKT + DK * BT;           // [DK][BT]  normalised q, transposed
    static constexpr int kV = kQT + DK * BT;            // [BT][VS]
    static constexpr int kH = kV + BT * VS;             // [DK][VS]  state slice
    static constexpr int kL = kH + DK * VS;             // [BT][BT+1]
    static constexpr int kP = kL + BT * (BT + 1);       // [BT][BT+1]
    static constexpr int kR = kP + BT * (BT + 1);       // [BT][VS]  right-hand side, then Delta
    static constexpr int kG = kR + BT * VS;             // [BT] cumulative log-decay
    static constexpr int kBeta = kG + BT;               // [BT]
    static constexpr int kNorm = kBeta + BT;            // [2][BT] inverse norms of q, k
    static constexpr int kTotal = kNorm + 2 * BT;
    static constexpr size_t bytes = sizeof(float) * kTotal;
};

template <int DK, int BT, typename IO>
__global__ void __launch_bounds__(NT, 1)
prefill_cudacore_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                        const IO* __restrict__ v, const float* __restrict__ g,
                        const float* __restrict__ beta, const float* __restrict__ h0,
                        const int32_t* __restrict__ cu, int64_t T, int n_seqs, int HK, int HV,
                        int Dv, float scale, int l2norm, IO* __restrict__ o,
                        float* __restrict__ hT, const int32_t* __restrict__ status) {
    using SM = CCSmem<DK, BT>;
    extern __shared__ float smem[];
    float* sKT = smem + SM::kKT;
    float* sQT = smem + SM::kQT;
    float* sV = smem + SM::kV;
    float* sH = smem + SM::kH;
    float* sL = smem + SM::kL;
    float* sP = smem + SM::kP;
    float* sR = smem + SM::kR;
    float* sG = smem + SM::kG;
    float* sB = smem + SM::kBeta;
    constexpr int LD = BT + 1;

    if (*status != 0) return;   // a bad cu_seqlens table was found: write nothing

    const int nvs = Dv / VS;
    int idx = blockIdx.x;
    const int vs = idx % nvs;  idx /= nvs;
    const int h = idx % HV;    idx /= HV;
    const int n = idx;
    const int hk = h / (HV / HK);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    int64_t bos, eos;
    if (cu) { bos = cu[n]; eos = cu[n + 1]; }
    else    { bos = (int64_t)n * T; eos = bos + T; }
    // the table was validated by the check kernel; stay in bounds regardless
    if (bos < 0 || eos < bos || (cu && eos > T)) return;

    const int col0 = vs * VS;
    const size_t hoff = ((size_t)n * HV + h) * DK * Dv;
    for (int i = tid; i < DK * VS; i += NT) {
        const int c = i / VS, j = i % VS;
        sH[i] = h0 ? h0[hoff + (size_t)c * Dv + col0 + j] : 0.f;
    }

    for (int64_t s = bos; s < eos; s += BT) {
        const int Cn = (int)((eos - s) < BT ? (eos - s) : BT);
        __syncthreads();   // previous chunk fully consumed

        // ---- load the chunk: q, k rows (warp per row), v slice, g, beta -------------
        for (int i = warp; i < BT; i += NWARP) {
            float kr[DK / 32], qr[DK / 32];
            float ssk = 0.f, ssq = 0.f;
            const int64_t t = s + i;
#pragma unroll
            for (int m = 0; m < DK / 32; ++m) {
                const int c = lane + 32 * m;
                kr[m] = i < Cn ? load_elem(k, (t * HK + hk) * DK + c) : 0.f;
                qr[m] = i < Cn ? load_elem(q, (t * HK + hk) * DK + c) : 0.f;
                ssk += kr[m] * kr[m];
                ssq += qr[m] * qr[m];
            }
            const float rk = l2_inv(warp_sum(ssk), l2norm);
            const float rq = l2_inv(warp_sum(ssq), l2norm);
#pragma unroll
            for (int m = 0; m < DK / 32; ++m) {
                const int c = lane + 32 * m;
                sKT[c * BT + i] = kr[m] * rk;
                sQT[c * BT + i] = qr[m] * rq;
            }
        }
        for (int e = tid; e < BT * VS; e += NT) {
            const int i = e / VS, j = e % VS;
            sV[e] = i < Cn ? load_elem(v, ((s + i) * HV + h) * Dv + col0 + j) : 0.f;
        }
        if (tid < BT) {
            sG[tid] = tid < Cn ? g[(s + tid) * HV + h] : 0.f;
            sB[tid] = tid < Cn ? beta[(s + tid) * HV + h] : 0.f;
        }
        __syncthreads();
        if (tid == 0) {   // inclusive running sum of the log-decays (padding adds 0)
            float acc = 0.f;
            for (int i = 0; i < BT; ++i) { acc += sG[i]; sG[i] = acc; }
        }
        __syncthreads();

        // ---- L (strictly lower) and P (lower incl. diagonal) -------------------------
        {
            constexpr int JN = (BT + 31) / 32;   // columns j per lane
            float accA[BT / NWARP][JN], accP[BT / NWARP][JN];
#pragma unroll
            for (int m = 0; m < BT / NWARP; ++m)
#pragma unroll
                for (int jj = 0; jj < JN; ++jj) accA[m][jj] = accP[m][jj] = 0.f;
            for (int c = 0; c < DK; ++c) {
                float kj[JN];
#pragma unroll
                for (int jj = 0; jj < JN; ++jj)
                    kj[jj] = (lane + 32 * jj < BT) ? sKT[c * BT + lane + 32 * jj] : 0.f;
#pragma unroll
                for (int m = 0; m < BT / NWARP; ++m) {
                    const int i = warp + NWARP * m;
                    const float ki = sKT[c * BT + i], qi = sQT[c * BT + i];
#pragma unroll
                    for (int jj = 0; jj < JN; ++jj) {
                        accA[m][jj] = fmaf(ki, kj[jj], accA[m][jj]);
                        accP[m][jj] = fmaf(qi, kj[jj], accP[m][jj]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < BT / NWARP; ++m) {
                const int i = warp + NWARP * m;
#pragma unroll
                for (int jj = 0; jj < JN; ++jj) {
                    const int j = lane + 32 * jj;
                    if (j >= BT) continue;
                    const float decay = i >= j ? expf(sG[i] - sG[j]) : 0.f;
                    sL[i * LD + j] = i > j ? sB[i] * decay * accA[m][jj] : 0.f;
                    sP[i * LD + j] = decay * accP[m][jj];
                }
            }
        }

        // ---- right-hand side beta (v - gamma k H0) and Q H0 (kept in registers) -----
        float qh[BT / NWARP];
        {
            float kh[BT / NWARP];
#pragma unroll
            for (int m = 0; m < BT / NWARP; ++m) kh[m] = qh[m] = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float hc = sH[c * VS + lane];
#pragma unroll
                for (int m = 0; m < BT / NWARP; ++m) {
                    const int i = warp + NWARP * m;
                    kh[m] = fmaf(sKT[c * BT + i], hc, kh[m]);
                    qh[m] = fmaf(sQT[c * BT + i], hc, qh[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < BT / NWARP; ++m) {
                const int i = warp + NWARP * m;
                sR[i * VS + lane] = sB[i] * (sV[i * VS + lane] - expf(sG[i]) * kh[m]);
            }
        }
        __syncthreads();

        // ---- forward substitution (I + L) Delta = R, one column per lane of warp 0 ---
        if (warp == 0) {
            for (int i = 1; i < Cn; ++i) {
                float d = sR[i * VS + lane];
                for (int j = 0; j < i; ++j) d = fmaf(-sL[i * LD + j], sR[j * VS + lane], d);
                sR[i * VS + lane] = d;
                __syncwarp();
            }
        }
        __syncthreads();

        // ---- output rows: scale (gamma_i (Q H0)_i + sum_j P_ij Delta_j) ---------------
        {
            float acc[BT / NWARP];
#pragma unroll
            for (int m = 0; m < BT / NWARP; ++m) acc[m] = 0.f;
            for (int j = 0; j < BT; ++j) {
                const float dj = sR[j * VS + lane];
#pragma unroll
                for (int m = 0; m < BT / NWARP; ++m)
                    acc[m] = fmaf(sP[(warp + NWARP * m) * LD + j], dj, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < BT / NWARP; ++m) {
                const int i = warp + NWARP * m;
                if (i < Cn)
                    store_elem(o, ((s + i) * HV + h) * Dv + col0 + lane,
                               scale * (expf(sG[i]) * qh[m] + acc[m]));
            }
        }

        // ---- state: H = gamma_C H + (diag(exp(G_C - G)) K)^T Delta ------------------
        {
            const float GC = sG[BT - 1];
            const float gC = expf(GC);
            float acc[DK / NWARP];
#pragma unroll
            for (int m = 0; m < DK / NWARP; ++m) acc[m] = 0.f;
            for (int i = 0; i < Cn; ++i) {
                const float di = sR[i * VS + lane] * expf(GC - sG[i]);
#pragma unroll
                for (int m = 0; m < DK / NWARP; ++m)
                    acc[m] = fmaf(sKT[(warp + NWARP * m) * BT + i], di, acc[m]);
            }
            __syncthreads();   // every reader of the old H (Q H0, K H0) is done
#pragma unroll
            for (int m = 0; m < DK / NWARP; ++m) {
                const int c = warp + NWARP * m;
                sH[c * VS + lane] = fmaf(gC, sH[c * VS + lane], acc[m]);
            }
        }
    }
    __syncthreads();
    if (hT)
        for (int i = tid; i < DK * VS; i += NT) {
            const int c = i / VS, j = i % VS;
            hT[hoff + (size_t)c * Dv + col0 + j] = sH[i];
        }
}

template <int DK, int BT, typename IO>
cudaError_t launch_cc(const PrefillArgs& a, cudaStream_t s) {
    const size_t smem = CCSmem<DK, BT>::bytes;
    auto kern = prefill_cudacore_kernel<DK, BT, IO>;
    const cudaError_t ea = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (ea != cudaSuccess) return ea;
    const unsigned blocks = (unsigned)a.n_seqs * (unsigned)a.HV * (unsigned)(a.Dv / VS);
    if (blocks == 0) return cudaSuccess;
    kern<<<blocks, NT, smem, s>>>((const IO*)a.q, (const IO*)a.k, (const IO*)a.v, a.g, a.beta,
                                  a.h0, a.cu, a.T, a.n_seqs, a.HK, a.HV, a.Dv, a.scale, a.l2norm,
                                  (IO*)a.o, a.hT, a.status);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

template <int DK, typename IO>
cudaError_t launch_cc_bt(const PrefillArgs& a, cudaStream_t s) {
    switch (a.BT) {
        case 16: return launch_cc<DK, 16, IO>(a, s);
        case 32: return launch_cc<DK, 32, IO>(a, s);
        case 64: return launch_cc<DK, 64, IO>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

// Single CTA: status = error if cu[0] != 0, any cu[n+1] < cu[n], or cu[n_seqs] != T;
// with no table (dense layout) it just clears the status word.
__global__ void check_cu_kernel(const int32_t* __restrict__ cu, int n_seqs, int64_t T,
                                int32_t* __restrict__ status) {
    if (!cu) {
        if (threadIdx.x == 0) *status = GDN_DEVERR_NONE;
        return;
    }
    int bad = 0;
    for (int n = threadIdx.x; n < n_seqs; n += blockDim.x)
        if (cu[n + 1] < cu[n]) bad = 1;
    if (threadIdx.x == 0 && (cu[0] != 0 || (int64_t)cu[n_seqs] != T)) bad = 1;
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) *status = bad ? GDN_DEVERR_CU_SEQLENS : GDN_DEVERR_NONE;
}

}  // namespace

cudaError_t launch_check_cu_seqlens(const int32_t* cu, int n_seqs, int64_t T, int32_t* status,
                                    cudaStream_t s) {
    check_cu_kernel<<<1, 256, 0, s>>>(cu, n_seqs, T, status);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

cudaError_t launch_prefill_cudacore(const PrefillArgs& a, cudaStream_t s) {
    if (a.Dk == 128) return a.bf16 ? launch_cc_bt<128, __nv_bfloat16>(a, s) : launch_cc_bt<128, float>(a, s);
    if (a.Dk == 64) return a.bf16 ? launch_cc_bt<64, __nv_bfloat16>(a, s) : launch_cc_bt<64, float>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace gdn
