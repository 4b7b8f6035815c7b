// prefill_tc.cu -- chunked prefill of the gated delta rule on the 5th-generation tensor
// cores (tcgen05, TMA, TMEM), bf16 operands with fp32 accumulation and fp32 state.
//
// The chunk scheme ("QWEN3.5" Q&A page, question 1): time is cut into chunks of C = 64
// tokens; inside a chunk the work is parallel, across chunks the state is carried
// serially.  The chunk equations follow from the recurrence alone.  For one chunk of one
// value head, with H0 = S^T (Dk x Dv) the state at the chunk start, raw (not yet
// normalised) rows k_i, q_i, inverse norms rk_i, rq_i, write strengths b_i, and G_i the
// running sum of the log-decays inside the chunk (gamma_i = exp(G_i)):
//     L_ij = b_i exp(G_i - G_j) rk_i rk_j k_i.k_j   (i > j)      T = (I + L)^-1
//     W    = T diag(b gamma rk) K,   U = T diag(b) V                     (chunk-local)
//     P_ij = scale exp(G_i - G_j) rq_i rk_j q_i.k_j  (i >= j)
//     Delta = U - W H0
//     O     = diag(scale gamma rq) Q H0 + P Delta
//     H_C   = gamma_C H0 + K^T diag(exp(G_C - G) rk) Delta
// (with K_hat = diag(rk) K and Q_hat = diag(rq) Q the same reads diag(gamma) Q_hat H0 and
// K_hat^T diag(exp(G_C - G)) Delta).
// Every exponent evaluated is <= 0.
//
// Precision.  The output is a sum of terms much larger than itself (U - W H0 cancels, so
// does P Delta against the decayed Q H0 part), so bf16 rounding of the intermediates
// alone costs 3-5% of RMS(o).  Hence every intermediate operand is fp16 (10-bit
// mantissa): the normalised K_hat, Q_hat, the T diag(.) factors and V of the chunk-local
// products, and W, U, P, Delta and the state copy of the serial stage.  Data-dependent
// operands (V, U, Delta, state) carry a power-of-two scale so fp16 range is never at issue.
//
// Two kernels:
//  * chunk_prep (one CTA per chunk and q/k head, fully parallel, four CTAs per SM): the
//    Gram tiles [K;Q] K^T on tcgen05 (M=128), norms, gates, the unit-lower-triangular
//    inverse T in fp32 (16x16 diagonal blocks by substitution, off-diagonal blocks by
//    mma.sync block products), then W^T = K_hat^T (T diag(b gamma))^T and
//    U^T = V^T (T diag(b))^T on tcgen05 (M=128: Dk or Dv rows), read out of TMEM straight
//    to global memory.  Writes fp16 W, U (scaled), P, the normalised fp16 K_hat, Q_hat
//    tiles and per-row scalars.
//  * chunk_carry (one CTA per sequence, value head and 32-column slice of Dv; the value
//    columns of the state evolve independently): walks the chunks in order.  Per chunk:
//    [W;Q_hat] H0 (M=128) -> Delta on CUDA cores -> K_hat^T Delta~ and [0;P] Delta (M=128),
//    state kept in fp32 registers, its scaled fp16 copy in shared memory as the next MMA
//    operand.  A producer warp streams the operands through a 2-stage TMA ring.
// All waits on mbarriers are bounded: on expiry the kernel records GDN_DEVERR_TIMEOUT in
// the workspace status word and exits cleanly (TMEM freed).
#include <cudaTypedefs.h>

#include "gdn_internal.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace {

using bf16 = __nv_bfloat16;
using f16 = __half;
constexpr int C = 64;      // chunk length
constexpr int D = 128;     // head dim (Dk = Dv) of this path
constexpr int NS = 32;     // value columns per carry CTA
constexpr int NSTAGE = 2;  // TMA ring depth of the carry kernel
constexpr int SC_FLOATS = 256;   // per (chunk, value head): a[64], d[64], scalars below
constexpr int MS = 68;           // row stride (floats) of the chunk-local L / T buffer: rows
                                 //   start on 16-byte boundaries for vector accesses
constexpr int SC_GC = 128;       //   gamma_C = exp(G at the chunk's last token)
constexpr int SC_UINV = 129;     //   U is stored as fp16(U * 2^-e); this holds 2^e
constexpr int SC_VMAX = 130;     //   max |v| over the chunk's tile of this value head

// power of two 2^e with max_abs * 2^-e in [0.5, 1) (1 for max_abs == 0 or non-finite)
__device__ __forceinline__ float pow2_above(float max_abs) {
    if (!(max_abs > 0.f) || !isfinite(max_abs)) return 1.f;
    int e;
    frexpf(max_abs, &e);
    return ldexpf(1.f, e);
}

// sigmoid(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh (one special-function op, about
// 2^-11 relative error): an absolute gate error below 2^-12, under the bf16 rounding of the
// output for gates above 1/8 and a negligible absolute error below; saturates to 0 and 1
__device__ __forceinline__ float sigmoid_fast(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void record_timeout(int32_t* status) {
    atomicCAS(status, GDN_DEVERR_NONE, GDN_DEVERR_TIMEOUT);
}

// Locate chunk `chunk` of the flattened chunk list: its sequence n, first token s and
// length cn.  chunk_off[n] is the first chunk of sequence n (chunk_off[N] = total).
__device__ __forceinline__ bool locate_chunk(int chunk, const int32_t* __restrict__ chunk_off,
                                             const int32_t* __restrict__ cu, int64_t T, int n_seqs,
                                             int& n, int64_t& s, int& cn) {
    if (chunk >= chunk_off[n_seqs]) return false;
    int lo = 0, hi = n_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= chunk) lo = mid; else hi = mid - 1;
    }
    n = lo;
    const int64_t bos = cu ? (int64_t)cu[n] : (int64_t)n * T;
    const int64_t len = cu ? (int64_t)cu[n + 1] - cu[n] : T;
    const int j = chunk - chunk_off[n];
    s = bos + (int64_t)C * j;
    const int64_t rem = len - (int64_t)C * j;
    cn = (int)(rem < C ? rem : C);
    return cn > 0;
}

// ======================================================================================
// chunk table: validate cu_seqlens (if any) and write chunk_off[0..N] (one CTA)
// ======================================================================================
__global__ void __launch_bounds__(1024) chunk_table_kernel(const int32_t* __restrict__ cu, int n_seqs,
                                                           int64_t T, int32_t* __restrict__ chunk_off,
                                                           int32_t* __restrict__ status) {
    __shared__ int s_part[1024];
    __shared__ int s_bad;
    const int tid = threadIdx.x;
    if (tid == 0) s_bad = 0;
    __syncthreads();
    const int per = (n_seqs + 1023) / 1024;
    const int n0 = tid * per, n1 = min(n_seqs, n0 + per);
    int local = 0;
    for (int n = n0; n < n1; ++n) {
        int64_t len = T;
        if (cu) {
            len = (int64_t)cu[n + 1] - cu[n];
            if (len < 0) s_bad = 1;
        }
        if (len > 0) local += (int)((len + C - 1) / C);
    }
    if (cu && tid == 0 && (cu[0] != 0 || (int64_t)cu[n_seqs] != T)) s_bad = 1;
    s_part[tid] = local;
    __syncthreads();
    // inclusive scan of the 1024 partial counts (Hillis-Steele)
    for (int o = 1; o < 1024; o <<= 1) {
        const int v = tid >= o ? s_part[tid - o] : 0;
        __syncthreads();
        s_part[tid] += v;
        __syncthreads();
    }
    int off = s_part[tid] - local;
    for (int n = n0; n < n1; ++n) {
        chunk_off[n] = off;
        int64_t len = cu ? (int64_t)cu[n + 1] - cu[n] : T;
        if (len > 0) off += (int)((len + C - 1) / C);
    }
    if (tid == 1023) chunk_off[n_seqs] = s_part[1023];
    __syncthreads();
    if (tid == 0) *status = s_bad ? GDN_DEVERR_CU_SEQLENS : GDN_DEVERR_NONE;
}

// ======================================================================================
// In-place T = (I + L)^-1 for a 64 x 64 strictly lower L held in M (fp32, row stride MS),
// 128 threads.  On return the strictly lower triangle of M holds T (its unit diagonal is
// implied); entries on and above the diagonal are untouched.  With 16 x 16 blocks (b, b')
// and the 32 x 32 halves A (blocks 0, 1) and B (blocks 2, 3):
//  * the four diagonal blocks T_bb = (I + L_bb)^-1 by right-looking column substitution
//    (one thread per column; every finished x_j updates all later rows at once, so the
//    dependent chain is one FMA per row);
//  * inside each half, T_10 = -T_11 L_10 T_00 and T_32 = -T_33 L_32 T_22, one warp each;
//  * the lower-left half T_BA = -T_B (L_BA T_A): first the four blocks of Y = L_BA T_A, then
//    the four of -T_B Y, one warp per block.
// The block products run on mma.sync with fp16 operands and fp32 accumulation (the T
// entries are rounded to fp16 for the W / U operands anyway); the intermediate products go
// through shared memory as fp16, transposed so that a B fragment is one 32-bit load.  Five
// CTA barriers.
// ======================================================================================
// Warp-level 16x16x16 products on the legacy tensor-core path (mma.sync m16n8k16, fp16
// operands, fp32 accumulation); fragment layouts of that instruction: g = lane / 4,
// q = lane % 4; A (16 x 16): rows g, g+8 x columns 2q, 2q+1, 2q+8, 2q+9; B (16 x 8):
// rows 2q, 2q+1, 2q+8, 2q+9 x column g; D (16 x 8): rows g, g+8 x columns 2q, 2q+1.
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// Element (r, c) of a 16 x 16 block of M at (r0, c0); UNIT: the block is a diagonal block
// of T (unit diagonal implied, zero above it).
template <bool UNIT>
__device__ __forceinline__ float blk(const float (*M)[MS], int r0, int c0, int r, int c) {
    if (UNIT) return r == c ? 1.f : (r > c ? M[r0 + r][c0 + c] : 0.f);
    return M[r0 + r][c0 + c];
}
template <bool UNIT>
__device__ __forceinline__ void frag_a(uint32_t* a, const float (*M)[MS], int r0, int c0, int g, int q) {
    a[0] = pack_h2(blk<UNIT>(M, r0, c0, g, 2 * q), blk<UNIT>(M, r0, c0, g, 2 * q + 1));
    a[1] = pack_h2(blk<UNIT>(M, r0, c0, g + 8, 2 * q), blk<UNIT>(M, r0, c0, g + 8, 2 * q + 1));
    a[2] = pack_h2(blk<UNIT>(M, r0, c0, g, 2 * q + 8), blk<UNIT>(M, r0, c0, g, 2 * q + 9));
    a[3] = pack_h2(blk<UNIT>(M, r0, c0, g + 8, 2 * q + 8), blk<UNIT>(M, r0, c0, g + 8, 2 * q + 9));
}
// B fragment of the 16 x 8 slice (all 16 rows, columns n0 .. n0+7) of a block
template <bool UNIT>
__device__ __forceinline__ void frag_b(uint32_t* b, const float (*M)[MS], int r0, int c0, int n0, int g, int q) {
    b[0] = pack_h2(blk<UNIT>(M, r0, c0, 2 * q, n0 + g), blk<UNIT>(M, r0, c0, 2 * q + 1, n0 + g));
    b[1] = pack_h2(blk<UNIT>(M, r0, c0, 2 * q + 8, n0 + g), blk<UNIT>(M, r0, c0, 2 * q + 9, n0 + g));
}

// B fragment (rows 2q, 2q+1, 2q+8, 2q+9 of column n0 + g) of a 16 x 16 block held
// transposed in fp16 (Yt[n][k] = Y[k][n])
__device__ __forceinline__ void frag_b_t(uint32_t* b, const __half (*Yt)[18], int n0, int g, int q) {
    b[0] = *reinterpret_cast<const uint32_t*>(&Yt[n0 + g][2 * q]);
    b[1] = *reinterpret_cast<const uint32_t*>(&Yt[n0 + g][2 * q + 8]);
}
// a 16 x 16 product (the accumulators of two 16 x 8 tiles), transposed, as fp16
__device__ __forceinline__ void store_d_t(__half (*Yt)[18], const float (*acc)[4], int g, int q) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        Yt[8 * nt + 2 * q][g] = __float2half_rn(acc[nt][0]);
        Yt[8 * nt + 2 * q + 1][g] = __float2half_rn(acc[nt][1]);
        Yt[8 * nt + 2 * q][g + 8] = __float2half_rn(acc[nt][2]);
        Yt[8 * nt + 2 * q + 1][g + 8] = __float2half_rn(acc[nt][3]);
    }
}
// -(a 16 x 16 product) into block (bi, bj) of M
__device__ __forceinline__ void store_neg_block(float (*M)[MS], const float (*acc)[4], int bi, int bj, int g, int q) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        M[16 * bi + g][16 * bj + 8 * nt + 2 * q] = -acc[nt][0];
        M[16 * bi + g][16 * bj + 8 * nt + 2 * q + 1] = -acc[nt][1];
        M[16 * bi + g + 8][16 * bj + 8 * nt + 2 * q] = -acc[nt][2];
        M[16 * bi + g + 8][16 * bj + 8 * nt + 2 * q + 1] = -acc[nt][3];
    }
}

__device__ __forceinline__ void tinv64_inplace(float (*M)[MS], __half (*Y)[16][18], int tid) {
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    {   // ---- diagonal blocks -----------------------------------------------------------
        float col[16];
        const int b = tid >> 4, c = tid & 15, o = 16 * b;
        if (tid < 64) {
#pragma unroll
            for (int i = 0; i < 16; ++i) col[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < 15; ++j) {
                const float xj = col[j];
#pragma unroll
                for (int i = j + 1; i < 16; ++i) col[i] = fmaf(-M[o + i][o + j], xj, col[i]);
            }
        }
        __syncthreads();   // all reads of the diagonal blocks of L precede their overwrite
        if (tid < 64) {
#pragma unroll
            for (int i = 1; i < 16; ++i)
                if (i > c) M[o + i][o + c] = col[i];
        }
        __syncthreads();
    }
    uint32_t a[4], bb[2];
    if (warp < 2) {   // ---- T_10 (warp 0) and T_32 (warp 1): -T_ii (L_ij T_jj) ------------------
        const int i = 2 * warp + 1, j = i - 1;
        float acc[2][4] = {};
        frag_a<false>(a, M, 16 * i, 16 * j, g, q);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            frag_b<true>(bb, M, 16 * j, 16 * j, 8 * nt, g, q);
            mma16816(acc[nt], a, bb);
        }
        store_d_t(Y[warp], acc, g, q);
        __syncwarp();
        float acc2[2][4] = {};
        frag_a<true>(a, M, 16 * i, 16 * i, g, q);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            frag_b_t(bb, Y[warp], 8 * nt, g, q);
            mma16816(acc2[nt], a, bb);
        }
        store_neg_block(M, acc2, i, j, g, q);
    }
    __syncthreads();
    const int bi = 2 + (warp >> 1), bj = warp & 1;   // this warp's block of the lower-left half
    {   // ---- Y_ij = sum_{m >= j} L_im T_mj (T_A is lower) ----------------------------------
        float acc[2][4] = {};
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            if (m < bj) continue;
            frag_a<false>(a, M, 16 * bi, 16 * m, g, q);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                if (m == bj) frag_b<true>(bb, M, 16 * m, 16 * bj, 8 * nt, g, q);
                else frag_b<false>(bb, M, 16 * m, 16 * bj, 8 * nt, g, q);
                mma16816(acc[nt], a, bb);
            }
        }
        store_d_t(Y[warp], acc, g, q);
    }
    __syncthreads();   // Y complete, and every read of L_BA done before T_BA overwrites it
    {   // ---- T_ij = -sum_{k <= i} T_ik Y_kj (T_B is lower) -----------------------------------
        float acc[2][4] = {};
#pragma unroll
        for (int k = 2; k < 4; ++k) {
            if (k > bi) continue;
            if (k == bi) frag_a<true>(a, M, 16 * bi, 16 * bi, g, q);
            else frag_a<false>(a, M, 16 * bi, 16 * k, g, q);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                frag_b_t(bb, Y[(k - 2) * 2 + bj], 8 * nt, g, q);
                mma16816(acc[nt], a, bb);
            }
        }
        store_neg_block(M, acc, bi, bj, g, q);
    }
    __syncthreads();
}

// ======================================================================================
// chunk_prep
// ======================================================================================
struct PrepSmem {
    // [K; Q] in two 64-column halves (rows 0-63 K, 64-127 Q), 16 KB each.  Rows 0-63 are
    // rewritten in place as fp16 K_hat; rows 64-127 are reused for V (bf16 from TMA, then
    // fp16 V * sv in place) once Q_hat has been written out.
    uint16_t KQ[2][128 * 64];
    // L, then T in place (fp32, row stride MS); then, in the same bytes, the fp16 MMA
    // operands T diag(b gamma) (bytes 0-8191) and T diag(b) (8192-16383), K-major 128B-swizzled
    float M[64][MS];
    __half Y[4][16][18];   // the inverse's intermediate 16 x 16 products, transposed, fp16
    float rk[64], rq[64], G[64], bt[64], bgr[64], red[8];
    alignas(16) float eu[64];   // rk_j exp(G_r - G_j), the token factor of the separated decays
    float ga[2][64], ba[2][64];   // g, beta of value head gi in slot gi % 2, loaded ahead
    uint64_t bar_load, bar_v, bar_mma;
    uint32_t tmem_base;
    uint32_t nv;   // V tile copies issued so far (thread 96)
};
static_assert(offsetof(PrepSmem, M) % 1024 == 0, "the swizzled operands in M need 1024-byte alignment");
constexpr size_t kPrepSmemBytes = sizeof(PrepSmem) + 1024;
static_assert(4 * (kPrepSmemBytes + 1024) <= 228 * 1024, "four chunk_prep CTAs per SM (1 KB reserved each)");
constexpr uint32_t kPrepTmemCols = 128;   // 4 resident CTAs fill the 512 columns

// Column t = tid of a 64 x 128 fp16 tile from TMEM lane t (64 fp32 columns = the tile's 64
// rows), stored straight to global memory.  Lane pairs swap one value so that each thread
// writes 4-byte pairs: per warp and row, 64 contiguous bytes.
__device__ __forceinline__ void store_tile_from_tmem(f16* __restrict__ dst, uint32_t taddr, int tid) {
    const bool odd = (tid & 1) != 0;
    const int col = tid - (odd ? 1 : 0);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        float w[32];
        tc::tmem_ld32(taddr + part * 32, w);
        tc::tmem_wait_ld();
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const float send = odd ? w[2 * p] : w[2 * p + 1];
            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
            const int row = part * 32 + 2 * p + (odd ? 1 : 0);
            const __half2 h = odd ? __floats2half2_rn(recv, w[2 * p + 1]) : __floats2half2_rn(w[2 * p], recv);
            *reinterpret_cast<__half2*>(dst + (size_t)row * D + col) = h;
        }
    }
}

template <int G>
__global__ void __launch_bounds__(128, 4)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const DecodeGates gs, const int32_t* __restrict__ cu,
                  const int32_t* __restrict__ chunk_off, int64_t T, int n_seqs, int HV, float scale,
                  int l2norm, int HK, f16* __restrict__ Wg, f16* __restrict__ Ug,
                  const __grid_constant__ CUtensorMap tm_p_st, const __grid_constant__ CUtensorMap tm_qk_st,
                  float* __restrict__ SCg, int32_t* __restrict__ status, int stall) {
    extern __shared__ uint8_t smem_raw[];
    PrepSmem& S = *reinterpret_cast<PrepSmem*>(align1024(smem_raw));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int chunk = blockIdx.x, hk = blockIdx.y;
    if (*reinterpret_cast<volatile int32_t*>(status) != 0) return;
    int n, cn;
    int64_t s;
    if (!locate_chunk(chunk, chunk_off, cu, T, n_seqs, n, s, cn)) return;

    if (warp == 0) {
        tc::tmem_alloc(&S.tmem_base, kPrepTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        tc::mbar_init(&S.bar_load, 1);
        tc::mbar_init(&S.bar_v, 1);
        tc::mbar_init(&S.bar_mma, 1);
        tc::fence_mbar_init();
        S.nv = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // TMEM: columns 0-63 the Gram tiles (kept for every value head), 64-127 W^T; U^T goes
    // to 64-127 after W^T is read out, except for the last value head, whose U^T takes the
    // Gram columns (no longer needed) so both products run back to back.
    const uint32_t tG = tmem, tW = tmem + 64;
    const int si = (int)s;
    uint8_t* kq = reinterpret_cast<uint8_t*>(&S.KQ[0][0]);
    uint32_t mma_phase = 0;

    if (tid == 0) {
        tc::mbar_expect_tx(&S.bar_load, 4 * 64 * 64 * 2);
        tc::tma_load_3d(kq, &tm_k, &S.bar_load, 0, hk, si);
        tc::tma_load_3d(kq + 16384, &tm_k, &S.bar_load, 64, hk, si);
        tc::tma_load_3d(kq + 8192, &tm_q, &S.bar_load, 0, hk, si);
        tc::tma_load_3d(kq + 16384 + 8192, &tm_q, &S.bar_load, 64, hk, si);
    }
    // gates of token s + tid, value head h: read, or formed from the raw inputs (the formula of
    // gdn_gates, so the two are bit-identical)
    auto gate_of = [&](int h, float& gv, float& bv) {
        gv = 0.f;
        bv = 0.f;
        if (tid < cn) decode_gates(gs, (s + tid) * HV + h, h, gv, bv);
    };
    if (tid < 64) {   // gates of the group's first two value heads, under the TMA latency
#pragma unroll
        for (int gi = 0; gi < (G < 2 ? G : 2); ++gi) gate_of(hk * G + gi, S.ga[gi][tid], S.ba[gi][tid]);
    }
    bool ok = tc::mbar_wait(&S.bar_load, 0);
    if (__syncthreads_or(!ok)) goto abort;

    // ---- Gram tiles: D_G[0:64] = K K^T, D_G[64:128] = Q K^T (bf16, M=128, N=64, K=Dk) ----
    if (tid == 0) {
        tc::tc_fence_after();
        const uint32_t base = tc::smem_u32(kq);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = tc::desc_sw128(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            tc::mma_bf16(tG, d, d, tc::idesc_bf16(128, 64, 0, 0), kk > 0);
        }
        tc::mma_commit(&S.bar_mma);
    }
    {   // inverse norms of the k (tid < 64) and q rows, under the Gram MMA (order inside a
        // row is irrelevant)
        float ss = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint4* row = reinterpret_cast<const uint4*>(kq + half * 16384 + tid * 128);
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {   // chunk order c16 ^ (row % 8): conflict-free
                const uint4 u = row[c16 ^ (tid & 7)];
                const bf16* e = reinterpret_cast<const bf16*>(&u);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const float x = __bfloat162float(e[t]);
                    ss = fmaf(x, x, ss);
                }
            }
        }
        if (tid < 64) S.rk[tid] = l2_inv(ss, l2norm);
        else S.rq[tid - 64] = l2_inv(ss, l2norm);
    }
    ok = tc::mbar_wait(&S.bar_mma, mma_phase);
    mma_phase ^= 1;
    if (__syncthreads_or(!ok)) goto abort;
    tc::tc_fence_after();
    {
        const float rki = tid < 64 ? S.rk[tid] : 0.f;
        const float rqi = tid >= 64 ? S.rq[tid - 64] : 0.f;
        {   // K_hat (tid < 64) / Q_hat row: fp16 in place (K_hat feeds the W MMA, and both go
            // out from there by tensor-map stores); rows past the chunk are zeroed
            const float rr = tid < cn || (tid >= 64 && tid - 64 < cn) ? (tid < 64 ? rki : rqi) : 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint4* row = reinterpret_cast<uint4*>(kq + half * 16384 + tid * 128);
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                    const int pc = c16 ^ (tid & 7);   // logical chunk c16 sits at c16 ^ (row % 8)
                    const uint4 u = row[pc];
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                    uint32_t hv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {   // bf16 pair -> two floats (exact) -> fp16 pair
                        const __half2 h2 = __floats2half2_rn(__uint_as_float(w[q] << 16) * rr,
                                                             __uint_as_float(w[q] & 0xffff0000u) * rr);
                        hv[q] = *reinterpret_cast<const uint32_t*>(&h2);
                    }
                    row[pc] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                }
            }
        }
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {   // [K_hat; Q_hat] of the (chunk, q/k head), 128 rows
            const int qkrow = (chunk * HK + hk) * 128;
            tc::tma_store_2d(&tm_qk_st, kq, 0, qkrow);
            tc::tma_store_2d(&tm_qk_st, kq + 16384, 64, qkrow);
            tc::tma_store_2d(&tm_qk_st, kq + 8192, 0, qkrow + 64);
            tc::tma_store_2d(&tm_qk_st, kq + 16384 + 8192, 64, qkrow + 64);
            tc::bulk_commit();
        }
        // From here the Q rows of the first half stage each value head's P (written by
        // threads 64-127, stored by thread 96), then take that head's V tile; the second
        // half's Q rows take the rest of V.

        for (int gi = 0; gi < G; ++gi) {
            const int h = hk * G + gi;
            const size_t ch = (size_t)chunk * HV + h;
            const bool last = gi == G - 1;
            if (gi == 0 && tid == 0) tc::bulk_wait_read<0>();   // Q_hat has left the staging rows
            // ---- running sum of the log-decays, write strengths -------------------------
            if (tid < 64) {
                float gv = S.ga[gi & 1][tid];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, gv, o);
                    if ((tid & 31) >= o) gv += y;
                }
                S.G[tid] = gv;
                S.bt[tid] = S.ba[gi & 1][tid];
            }
            __syncthreads();
            if (G > 2 && gi + 2 < G && tid < 64)   // slot gi % 2 is read: value head gi + 2's gates
                gate_of(h + 2, S.ga[gi & 1][tid], S.ba[gi & 1][tid]);
            if (tid >= 32 && tid < 64) S.G[tid] += S.G[31];
            __syncthreads();
            if (tid < 64) S.bgr[tid] = S.bt[tid] * expf(S.G[tid]);
            const float Gl = S.G[63];   // padding adds 0, so this is G at the last token
            // exp(G_i - G_j) = exp(G_i - G_r) exp(G_r - G_j) with G_r = G_last / 2: both
            // factors stay inside fp32 range while G_last >= -160, and the row loops below
            // then need no exponential per pair; deeper decays take exp(G_i - G_j) directly
            const bool sep = Gl >= -160.f;
            const float Gr = 0.5f * Gl;
            if (sep) {
                if (tid < 64) S.eu[tid] = S.rk[tid] * __expf(Gr - S.G[tid]);
                __syncthreads();
            }
            // ---- L (strictly lower) into M, P (lower incl. diagonal) out, scalars; the
            //      Gram row of this thread is read back from TMEM --------------------------
            {
                float row[64];
                tc::tmem_ld32(tG + lane_base, row);
                tc::tmem_ld32(tG + lane_base + 32, row + 32);
                tc::tmem_wait_ld();
                if (tid < 64) {
                    const int i = tid;
                    const float Gi = S.G[i], bi = S.bt[i] * rki;
                    if (sep) {
                        const float ai = i < cn ? bi * __expf(Gi - Gr) : 0.f;
                        float4* mrow = reinterpret_cast<float4*>(&S.M[i][0]);
                        const float4* eu4 = reinterpret_cast<const float4*>(S.eu);
#pragma unroll
                        for (int j4 = 0; j4 < 16; ++j4) {
                            const float4 e = eu4[j4];
                            const int j = 4 * j4;
                            float4 l;
                            l.x = j < i ? ai * e.x * row[j] : 0.f;
                            l.y = j + 1 < i ? ai * e.y * row[j + 1] : 0.f;
                            l.z = j + 2 < i ? ai * e.z * row[j + 2] : 0.f;
                            l.w = j + 3 < i ? ai * e.w * row[j + 3] : 0.f;
                            mrow[j4] = l;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            float v = 0.f;
                            if (j < i && i < cn) v = bi * __expf(Gi - S.G[j]) * S.rk[j] * row[j];
                            S.M[i][j] = v;
                        }
                    }
                    SCg[ch * SC_FLOATS + 64 + i] = i < cn ? expf(Gl - Gi) : 0.f;
                } else {
                    const int i = tid - 64;
                    const float Gi = S.G[i], qi = scale * rqi;
                    SCg[ch * SC_FLOATS + i] = i < cn ? scale * expf(Gi) : 0.f;
                    if (i == 0) SCg[ch * SC_FLOATS + SC_GC] = expf(Gl);
                    uint8_t* prow = kq + 8192 + i * 128;   // 128B-swizzled like the tensor map
                    const float ai = sep && i < cn ? qi * __expf(Gi - Gr) : 0.f;
                    const float4* eu4 = reinterpret_cast<const float4*>(S.eu);
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        __align__(16) f16 e[8];
                        const float4 ea = eu4[2 * c8], eb = eu4[2 * c8 + 1];
                        const float ev[8] = {ea.x, ea.y, ea.z, ea.w, eb.x, eb.y, eb.z, eb.w};
                        float pv[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int j = c8 * 8 + t;
                            float v = 0.f;
                            if (sep) v = j <= i ? ai * ev[t] * row[j] : 0.f;
                            else if (j <= i && i < cn) v = qi * __expf(Gi - S.G[j]) * S.rk[j] * row[j];
                            pv[t] = v;
                        }
#pragma unroll
                        for (int t = 0; t < 4; ++t) reinterpret_cast<__half2*>(e)[t] = __floats2half2_rn(pv[2 * t], pv[2 * t + 1]);
                        *reinterpret_cast<uint4*>(prow + ((c8 ^ (i & 7)) << 4)) = *reinterpret_cast<const uint4*>(e);
                    }
                }
            }
            tc::fence_async_smem();
            __syncthreads();
            if (tid == 96) {
                // warp 3 has no part in the inverse's first phase: P out, then this head's V
                // into the staging rows once the store has read them (test hook,
                // gdn_testing_stall: no V for the first CTA's first head, whose wait then runs out)
                tc::tma_store_2d(&tm_p_st, kq + 8192, 0, (int)(ch * 64));
                tc::bulk_commit();
                tc::bulk_wait_read<0>();
                if (!(stall && chunk == 0 && hk == 0 && gi == 0)) {
                    tc::mbar_expect_tx(&S.bar_v, 2 * 64 * 64 * 2);
                    ++S.nv;
                    tc::tma_load_3d(kq + 8192, &tm_v, &S.bar_v, 0, h, si);
                    tc::tma_load_3d(kq + 16384 + 8192, &tm_v, &S.bar_v, 64, h, si);
                }
            }
            tinv64_inplace(S.M, S.Y, tid);
            // ---- fp16 MMA operands T diag(b gamma) and T diag(b), 128B-swizzled, written
            //      over M once every thread holds its part of T -----------------------------
            {
                const int i = tid >> 1, c0 = (tid & 1) * 32;
                float tv[32];
                const float4* mrow = reinterpret_cast<const float4*>(&S.M[i][c0]);
#pragma unroll
                for (int t4 = 0; t4 < 8; ++t4) {
                    const float4 m4 = mrow[t4];
                    const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = c0 + 4 * t4 + e;
                        tv[4 * t4 + e] = j < i ? mv[e] : (j == i ? 1.f : 0.f);
                    }
                }
                __syncthreads();
                uint8_t* aw = reinterpret_cast<uint8_t*>(&S.M[0][0]);
                uint8_t* au = aw + 8192;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    __align__(16) f16 w8[8], u8[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        const int j = c0 + cc * 8 + t;
                        w8[t] = __float2half_rn(tv[cc * 8 + t] * S.bgr[j]);
                        u8[t] = __float2half_rn(tv[cc * 8 + t] * S.bt[j]);
                    }
                    const uint32_t off = tc::sw128_off(i, c0 + cc * 8);
                    *reinterpret_cast<uint4*>(aw + off) = *reinterpret_cast<const uint4*>(w8);
                    *reinterpret_cast<uint4*>(au + off) = *reinterpret_cast<const uint4*>(u8);
                }
            }
            // ---- V tile of this head: max |v|, then fp16(v * sv) in place, rows past the
            //      chunk zeroed -----------------------------------------------------------
            ok = tc::mbar_wait(&S.bar_v, gi & 1);
            if (__syncthreads_or(!ok)) goto abort;
            {
                const int r = tid >> 1, half = tid & 1;
                uint4* vr = reinterpret_cast<uint4*>(kq + half * 16384 + 8192 + r * 128);
                // max |v| from the bf16 bit patterns: with the sign bit cleared, their order as
                // 16-bit integers is the order of the magnitudes (a NaN pattern exceeds them all
                // and turns the scale off, as an infinite value does)
                uint32_t m2 = 0;
                if (r < cn) {
#pragma unroll
                    for (int c16 = 0; c16 < 8; ++c16) {
                        const uint4 u = vr[c16 ^ (r & 7)];
                        m2 = __vmaxu2(m2, u.x & 0x7fff7fffu);
                        m2 = __vmaxu2(m2, u.y & 0x7fff7fffu);
                        m2 = __vmaxu2(m2, u.z & 0x7fff7fffu);
                        m2 = __vmaxu2(m2, u.w & 0x7fff7fffu);
                    }
                }
                const uint32_t mw = __reduce_max_sync(0xffffffffu, max(m2 & 0xffffu, m2 >> 16));
                if ((tid & 31) == 0) S.red[warp] = __uint_as_float(mw << 16);
                __syncthreads();
                const float vmax = fmaxf(fmaxf(S.red[0], S.red[1]), fmaxf(S.red[2], S.red[3]));
                const float uinv = pow2_above(vmax), sv = r < cn ? 1.f / uinv : 0.f;
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {   // bf16 pair -> two floats (exact) -> fp16 pair
                    const int pc = c16 ^ (r & 7);
                    const uint4 u = vr[pc];
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                    uint32_t hv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const __half2 h2 = __floats2half2_rn(__uint_as_float(w[q] << 16) * sv,
                                                             __uint_as_float(w[q] & 0xffff0000u) * sv);
                        hv[q] = *reinterpret_cast<const uint32_t*>(&h2);
                    }
                    vr[pc] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                }
                if (tid == 0) {
                    SCg[ch * SC_FLOATS + SC_UINV] = uinv;
                    SCg[ch * SC_FLOATS + SC_VMAX] = vmax;
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            __syncthreads();
            // ---- W^T = K_hat^T AW^T and (V sv)^T AU^T (fp16, M=128, N=64, K=64 tokens) ----
            const uint32_t kb = tc::smem_u32(kq), vb = kb + 8192;
            const uint32_t awb = tc::smem_u32(&S.M[0][0]), aub = awb + 8192;
            constexpr uint32_t idx = tc::idesc_f16(128, 64, 1, 0);
            if (tid == 0) {
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tW, tc::desc_sw128(kb + kk * 2048, 16384, 1024),
                                 tc::desc_sw128(awb + kk * 32, 16, 1024), idx, kk > 0);
                if (last) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(tG, tc::desc_sw128(vb + kk * 2048, 16384, 1024),
                                     tc::desc_sw128(aub + kk * 32, 16, 1024), idx, kk > 0);
                }
                tc::mma_commit(&S.bar_mma);
            }
            ok = tc::mbar_wait(&S.bar_mma, mma_phase);
            mma_phase ^= 1;
            if (__syncthreads_or(!ok)) goto abort;
            tc::tc_fence_after();
            // ---- epilogue: lane t of D_W / D_U is column t of W / U -----------------------
            store_tile_from_tmem(Wg + ch * 64 * D, tW + lane_base, tid);
            if (!last) {   // U^T into the W^T columns once they are read
                tc::tc_fence_before();
                __syncthreads();
                if (tid == 0) {
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(tW, tc::desc_sw128(vb + kk * 2048, 16384, 1024),
                                     tc::desc_sw128(aub + kk * 32, 16, 1024), idx, kk > 0);
                    tc::mma_commit(&S.bar_mma);
                }
                ok = tc::mbar_wait(&S.bar_mma, mma_phase);
                mma_phase ^= 1;
                if (__syncthreads_or(!ok)) goto abort;
                tc::tc_fence_after();
            }
            store_tile_from_tmem(Ug + ch * 64 * D, (last ? tG : tW) + lane_base, tid);
            tc::tc_fence_before();
            __syncthreads();   // TMEM reads done; M (the operands) free for the next head
        }
    }
    if (tid == 0 || tid == 96) tc::bulk_wait<0>();   // this thread's tensor-map stores are done
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kPrepTmemCols);
    return;
abort:
    if (tid == 0 || tid == 96) tc::bulk_wait<0>();
    if (tid == 0) {
        record_timeout(status);
        // the copies and products still in flight land before the shared memory and TMEM are
        // released; each wait is for the latest phase of its barrier (at once if complete)
        (void)tc::mbar_wait(&S.bar_load, 0, 50000000ull);
        const uint32_t nv = S.nv;
        if (nv > 0) (void)tc::mbar_wait(&S.bar_v, (nv - 1u) & 1u, 50000000ull);
        (void)tc::mbar_wait(&S.bar_mma, mma_phase ^ 1u, 50000000ull);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kPrepTmemCols);
}
// ======================================================================================
// chunk_carry
// ======================================================================================
struct CarryStage {
    f16 A[2][128 * 64];    // [W; Q_hat] in two 64-column halves (32 KB), K-major 128B-swizzled
    f16 K[2][64 * 64];     // K_hat in two 64-column halves (16 KB)
    f16 P[128 * 64];       // rows 0-63 zero, rows 64-127 P (16 KB)
    f16 U[64 * NS];        // scaled U columns of this slice, row-major (4 KB)
    float SC[SC_FLOATS];   // a[64], d[64], gamma_C, U scale, max |v|
};
constexpr int NZ = 4;   // ring of gate-input tiles (output epilogue)
struct ZSlot {
    bf16 z[C * NS];    // z of the chunk's rows, this slice's values, row-major (4 KB)
    float a[C];        // the chunk's per-row output scalars
};
struct CarrySmem {
    CarryStage st[NSTAGE];
    f16 H0[2][D * NS];     // scaled fp16 state slice: MN-major unswizzled B operand (K = Dk),
                           //   by chunk parity
    f16 Dl[C * NS];        // scaled Delta, same layout (K = tokens)
    f16 Dt[C * NS];        // scaled Delta~ = diag(exp(G_C - G)) Delta
    alignas(128) ZSlot zr[NZ];   // output epilogue: z tiles and scalars, chunk c in slot c % NZ
                                 //   (tensor-map copy targets: 128-byte aligned)
    float red[4];
    // output epilogue: per chunk parity, this CTA's per-row sums of squares and those
    // received from the other slices (bulk-copy source and target: 16-byte aligned)
    alignas(16) float oloc[2][C];
    alignas(16) float opart[2][D / NS][C];
    float onw[NS];   // 1 + w of this slice's values
    float inv_sc;    // the data scale, for the output warps
    // bar_o: one per output buffer, so that a deferred wait can never fall two phases behind;
    // ofree: the output warps are done with an output buffer; zfull / zempty: the z ring
    uint64_t full[NSTAGE], empty[NSTAGE], bar_a, bar_b, bar_o[3], h0_ready, d_ready, obar[2];
    uint64_t ofree[3], zfull[NZ], zempty[NZ];
    uint32_t tmem_base;
    volatile int abort;
};
constexpr size_t kCarrySmemBytes = sizeof(CarrySmem) + 1024;
// targets and sources of TMA and bulk copies sit on 16-byte (swizzled tiles: 1024-byte) boundaries
static_assert(sizeof(CarryStage) % 1024 == 0 && offsetof(CarryStage, K) % 1024 == 0 &&
                  offsetof(CarryStage, P) % 1024 == 0 && offsetof(CarryStage, U) % 16 == 0 &&
                  offsetof(CarryStage, SC) % 16 == 0,
              "carry stage layout");
static_assert(offsetof(CarrySmem, zr) % 128 == 0 && sizeof(ZSlot) % 128 == 0 && offsetof(ZSlot, a) % 16 == 0 &&
                  offsetof(CarrySmem, oloc) % 16 == 0 && offsetof(CarrySmem, opart) % 16 == 0 &&
                  offsetof(CarrySmem, H0) % 16 == 0 && offsetof(CarrySmem, Dl) % 16 == 0 &&
                  offsetof(CarrySmem, Dt) % 16 == 0,
              "carry shared-memory layout");
constexpr uint32_t kCarryTmemCols = 256;
constexpr uint32_t kStageTxBytes = 2 * 128 * 64 * 2 + 2 * 64 * 64 * 2 + 64 * 64 * 2 + 64 * NS * 2 + SC_FLOATS * 4;
constexpr uint32_t kZTxBytes = C * NS * 2 + C * 4;
// warps 0-3 epilogues, warp 4 TMA producer, warp 5 MMA issuer; with the output epilogue,
// warps 6-7 write the output rows (TMEM lanes 64-127, as warps 2-3)
__host__ __device__ constexpr int carry_threads(bool outg) { return outg ? 256 : 192; }

// MN-major, unswizzled B operand with N = NS (32) columns: 8 x 8 core matrices of 128 bytes
// (8 K-rows of 16 bytes); the NS / 8 core matrices of one group of 8 K-rows sit 128 bytes
// apart (stride between N blocks, SBO), consecutive K groups 512 bytes apart (LBO).
constexpr uint32_t kOpSBO = 128, kOpLBO = 128 * (NS / 8);
__device__ __forceinline__ uint32_t op_off(int k, int nb) {   // 16-byte chunk of row k, N block nb
    return (uint32_t)((k & 7) * 16 + nb * kOpSBO + (k >> 3) * kOpLBO);
}
__device__ __forceinline__ uint64_t desc_noswz(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version; layout bits 61-63 = 0: no swizzle
    return d;
}
// write NS values of row k (scaled, fp16) into an MN-major operand
__device__ __forceinline__ void store_op_row(f16* op, int k, const float* v, float sc) {
    uint8_t* base = reinterpret_cast<uint8_t*>(op);
#pragma unroll
    for (int nb = 0; nb < NS / 8; ++nb) {
        __align__(16) f16 h8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) h8[e] = __float2half_rn(v[nb * 8 + e] * sc);
        *reinterpret_cast<uint4*>(base + op_off(k, nb)) = *reinterpret_cast<const uint4*>(h8);
    }
}

// Per chunk c, the MMA warp issues (each group committed to its own mbarrier):
//   a: [W; Q_hat] H0     (M=128, 8 MMAs)  -> D_a[c % nb]  rows 0-63 W H0, rows 64-127 Q_hat H0
//   b: K_hat^T Delta~    (M=128, 4 MMAs)  -> D_b          state update
//   c: [0; P] Delta      (M=128, 4 MMAs)  -> D_c[c % nb]  rows 64-127 P Delta
// Epilogue threads 0-63 turn D_a rows into Delta, Delta~; all 128 update the state rows
// from D_b; without OUTG, threads 64-127 write the output rows of chunk c while chunk
// c+1's MMAs run.
// The two sides meet only through mbarriers (h0_ready, d_ready: one arrival per epilogue
// warp, after its threads' shared-memory writes and proxy fences; the output warps
// arrive on d_ready as soon as they have read the chunk's scalars, then
// write the previous chunk's output rows while Delta and the state MMA proceed; the
// stage is released only after every thread's reads of it).
//
// OUTG adds the output epilogue out = o rsqrt(mean(o^2) + eps) (1 + w) sigmoid(z) over the
// 128 values of a head, which live in the head's four slice CTAs: those run as one
// thread-block cluster (cluster rank = slice), and each output row's four partial sums of
// squares cross over distributed shared memory by bulk copies.  Two extra warps (6-7, on
// TMEM lanes 64-127 like warps 2-3) do all of the output work, so that none of it sits
// on the serial chain: the producer streams each chunk's z tile and row scalars into a
// ring of NZ slots, D_a and D_c rotate over three buffers, and the MMA warp reuses a
// buffer only after the output warps release it (ofree).
// TR: the transition run of a context-parallel segment: U taken as zero (v = 0) and the
// identity as the initial state (Dk = Dv), on the chunk-local operands of the same call.
template <bool OUTG, bool TR = false>
__global__ void __launch_bounds__(carry_threads(OUTG), 1)
chunk_carry_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_qk,
                   const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_u,
                   const __grid_constant__ CUtensorMap tm_z,
                   const float* __restrict__ SCg, const int32_t* __restrict__ cu,
                   const int32_t* __restrict__ chunk_off, int64_t T, int n_seqs, int HK, int HV,
                   const float* __restrict__ h0, float* __restrict__ hT, bf16* __restrict__ o,
                   const bf16* __restrict__ zg, const float* __restrict__ norm_w, float eps,
                   int32_t* __restrict__ status) {
    constexpr int nb = OUTG ? 3 : 2;   // buffers of D_a and D_c
    extern __shared__ uint8_t smem_raw[];
    CarrySmem& S = *reinterpret_cast<CarrySmem*>(align1024(smem_raw));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int nslices = D / NS;
    int idx = blockIdx.x;
    const int vs = idx % nslices; idx /= nslices;
    const int h = idx % HV;       idx /= HV;
    const int n = idx;
    const int hk = h / (HV / HK);
    // Without clusters a CTA may leave at once; with them every CTA must reach both cluster
    // barriers, so a failed earlier stage only empties the work.
    const bool failed = *reinterpret_cast<volatile int32_t*>(status) != 0;
    if (!OUTG && failed) return;
    const int64_t bos = cu ? (int64_t)cu[n] : (int64_t)n * T;
    const int64_t len = cu ? (int64_t)cu[n + 1] - cu[n] : T;
    const int c0 = chunk_off[n];
    const int nch = failed ? 0 : chunk_off[n + 1] - c0;

    if (warp == 0) {
        tc::tmem_alloc(&S.tmem_base, kCarryTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        for (int i = 0; i < NSTAGE; ++i) {
            tc::mbar_init(&S.full[i], 1);
            tc::mbar_init(&S.empty[i], 1);
        }
        tc::mbar_init(&S.bar_a, 1);
        tc::mbar_init(&S.bar_b, 1);
        for (int i = 0; i < 3; ++i) tc::mbar_init(&S.bar_o[i], 1);
        tc::mbar_init(&S.h0_ready, 4);   // one arrival per epilogue warp
        tc::mbar_init(&S.d_ready, 4);
        if (OUTG) {   // one local arrival per use, plus the peers' bulk copies as transactions
            tc::mbar_init(&S.obar[0], 1);
            tc::mbar_init(&S.obar[1], 1);
            for (int i = 0; i < 3; ++i) tc::mbar_init(&S.ofree[i], 2);   // one per output warp
            for (int i = 0; i < NZ; ++i) {
                tc::mbar_init(&S.zfull[i], 1);
                tc::mbar_init(&S.zempty[i], 2);
            }
        }
        tc::fence_mbar_init();
        S.abort = 0;
    }
    if (OUTG && tid < NS) S.onw[tid] = 1.f + norm_w[vs * NS + tid];   // the (1 + w) factor
    // zero rows 0-63 of the P operands (the producer only ever writes rows 64-127)
    for (int e = tid; e < NSTAGE * 64 * 64 / 8; e += carry_threads(OUTG)) {
        const int st = e / (64 * 64 / 8), r = e % (64 * 64 / 8);
        reinterpret_cast<uint4*>(S.st[st].P)[r] = make_uint4(0, 0, 0, 0);
    }
    tc::fence_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    if (OUTG) tc::cluster_sync();   // every slice CTA's barriers exist before any remote arrival
    tc::tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t tA = tmem, tB = tmem + nb * 32, tC = tmem + nb * 32 + 32;   // tA, tC: +32 per buffer

    if (warp == 4) {
        // ---------------- producer: stream the chunks through the ring ----------------
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const int st = c % NSTAGE, r = c / NSTAGE;
                if (r > 0 && !tc::mbar_wait(&S.empty[st], (r - 1) & 1)) {
                    record_timeout(status);
                    S.abort = 1;
                }
                if (S.abort) break;
                CarryStage& B = S.st[st];
                const int cid = c0 + c;
                const int row = (cid * HV + h) * 64;
                const int qkrow = (cid * HK + hk) * 128;
                tc::mbar_expect_tx(&S.full[st], kStageTxBytes);
                tc::tma_load_2d(&B.A[0][0], &tm_w, &S.full[st], 0, row);
                tc::tma_load_2d(&B.A[1][0], &tm_w, &S.full[st], 64, row);
                tc::tma_load_2d(&B.A[0][64 * 64], &tm_qk, &S.full[st], 0, qkrow + 64);
                tc::tma_load_2d(&B.A[1][64 * 64], &tm_qk, &S.full[st], 64, qkrow + 64);
                tc::tma_load_2d(&B.K[0][0], &tm_qk, &S.full[st], 0, qkrow);
                tc::tma_load_2d(&B.K[1][0], &tm_qk, &S.full[st], 64, qkrow);
                tc::tma_load_2d(&B.P[64 * 64], &tm_p, &S.full[st], 0, row);
                tc::tma_load_2d(B.U, &tm_u, &S.full[st], vs * NS, row);
                tc::bulk_load(B.SC, SCg + ((size_t)cid * HV + h) * SC_FLOATS, SC_FLOATS * 4, &S.full[st]);
                if (OUTG) {   // the chunk's z tile and per-row scalars, for the output warps
                    const int k = c % NZ;
                    if (c >= NZ && !tc::mbar_wait(&S.zempty[k], (uint32_t)(((c / NZ) - 1) & 1))) {
                        record_timeout(status);
                        S.abort = 1;
                    }
                    if (S.abort) break;
                    tc::mbar_expect_tx(&S.zfull[k], kZTxBytes);
                    tc::tma_load_3d(S.zr[k].z, &tm_z, &S.zfull[k], vs * NS, h, (int)(bos + (int64_t)C * c));
                    tc::bulk_load(S.zr[k].a, SCg + ((size_t)cid * HV + h) * SC_FLOATS, C * 4, &S.zfull[k]);
                }
            }
        }
    } else if (warp == 5) {
        // ---------------- MMA issuer ---------------------------------------------------------
        if (lane == 0) {
            constexpr uint32_t idA = tc::idesc_f16(128, NS, 0, 1);   // K-major A, MN-major B
            constexpr uint32_t idB = tc::idesc_f16(128, NS, 1, 1);   // MN-major A and B
            const uint64_t ddl = desc_noswz(tc::smem_u32(S.Dl), kOpLBO, kOpSBO);
            const uint64_t ddt = desc_noswz(tc::smem_u32(S.Dt), kOpLBO, kOpSBO);
            for (int c = 0; c < nch; ++c) {
                const int st = c % NSTAGE, r = c / NSTAGE;
                const CarryStage& B = S.st[st];
                bool ok = tc::mbar_wait(&S.full[st], r & 1);
                ok = ok && tc::mbar_wait_spin(&S.h0_ready, c & 1);
                if (!ok || S.abort) {
                    if (!ok) record_timeout(status);
                    S.abort = 1;
                    break;
                }
                if (OUTG && c >= nb && !tc::mbar_wait_spin(&S.ofree[c % nb], (uint32_t)(((c / nb) - 1) & 1))) {
                    record_timeout(status);
                    S.abort = 1;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t par = (uint32_t)(c % nb) * 32;
                // descriptors built once; a k-step only advances the start-address field
                const uint64_t da = tc::desc_sw128(tc::smem_u32(&B.A[0][0]), 16, 1024);
                const uint64_t dh = desc_noswz(tc::smem_u32(S.H0[c & 1]), kOpLBO, kOpSBO);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tA + par, da + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                                 dh + (uint64_t)((kk * 2 * kOpLBO) >> 4), idA, kk > 0);
                tc::mma_commit(&S.bar_a);
                if (!tc::mbar_wait_spin(&S.d_ready, c & 1) || S.abort) {
                    record_timeout(status);
                    S.abort = 1;
                    break;
                }
                tc::tc_fence_after();
                const uint64_t dk = tc::desc_sw128(tc::smem_u32(&B.K[0][0]), 8192, 1024);
                const uint64_t dp = tc::desc_sw128(tc::smem_u32(B.P), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tB, dk + (uint64_t)((kk * 2048) >> 4), ddt + (uint64_t)((kk * 2 * kOpLBO) >> 4),
                                 idB, kk > 0);
                tc::mma_commit(&S.bar_b);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tC + par, dp + (uint64_t)((kk * 32) >> 4), ddl + (uint64_t)((kk * 2 * kOpLBO) >> 4),
                                 idA, kk > 0);
                tc::mma_commit(&S.bar_o[c % nb]);
                tc::mma_commit(&S.empty[st]);   // the stage's operands are consumed
            }
        }
    } else if (warp < 4) {
        // ---------------- epilogues: 128 threads, thread t <-> TMEM lane t ------------------
        const int t = tid;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        float Hr[NS];
        const size_t hrow = (((size_t)n * HV + h) * D + t) * D + vs * NS;
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < NS; ++j) {   // the initial state (TR: the identity)
            Hr[j] = TR ? (t == vs * NS + j ? 1.f : 0.f) : (h0 ? h0[hrow + j] : 0.f);
            m = fmaxf(m, fabsf(Hr[j]));
        }
        // data scale: fp16 operands carry x * sc with sc = 2^-e, max(|h0|, |v|) * sc < 1
        for (int c = t; c < nch; c += 128) m = fmaxf(m, SCg[((size_t)(c0 + c) * HV + h) * SC_FLOATS + SC_VMAX]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) S.red[warp] = m;
        tc::named_bar(1, 128);
        const float inv_sc = pow2_above(fmaxf(fmaxf(S.red[0], S.red[1]), fmaxf(S.red[2], S.red[3])));
        const float sc = 1.f / inv_sc;
        if (OUTG) {   // publish the scale to the output warps
            if (t == 0) S.inv_sc = inv_sc;
            tc::named_bar_arrive(3, 128 + 64);
        }
        store_op_row(S.H0[0], t, Hr, sc);
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.h0_ready);   // phase 0: the initial state operand

        bool ok = true;
        float a_prev = 0.f;          // plain: per-row scalar, length and first token of the
        int cn_prev = 0;             //   previous chunk, whose output rows are written next
        int64_t tok_prev = 0;
        // plain: output rows of chunk cc (threads 64-127, row t - 64), from D_a and D_c
        // buffer cc % nb, written under the next chunk's Delta epilogue and state MMA
        auto write_output = [&](int cc) -> bool {
            const int i = t - 64;
            const bool good = tc::mbar_wait(&S.bar_o[cc % nb], (uint32_t)((cc / nb) & 1));
            tc::tc_fence_after();
            const uint32_t par = (uint32_t)(cc % nb) * 32;
            float q[NS], z[NS];
            tc::tmem_ld32(tA + par + lane_base, q);
            tc::tmem_ld32(tC + par + lane_base, z);
            tc::tmem_wait_ld();
            if (i < cn_prev) {
                __align__(16) bf16 ob[NS];
#pragma unroll
                for (int j = 0; j < NS; ++j) ob[j] = __float2bfloat16_rn(fmaf(a_prev, q[j], z[j]) * inv_sc);
                uint4* dst = reinterpret_cast<uint4*>(o + ((tok_prev + i) * HV + h) * D + vs * NS);
#pragma unroll
                for (int qq = 0; qq < NS / 8; ++qq) dst[qq] = reinterpret_cast<const uint4*>(ob)[qq];
            }
            return good;
        };
        for (int c = 0; c < nch && ok; ++c) {
            const int st = c % NSTAGE, rr = c / NSTAGE;
            const CarryStage& B = S.st[st];
            const int64_t tok = bos + (int64_t)C * c;
            const int64_t rem = len - (int64_t)C * c;
            const int cn = (int)(rem < C ? rem : C);
            ok = tc::mbar_wait(&S.full[st], rr & 1);
            const float gC = B.SC[SC_GC];
            if (warp < 2) {
                // ---- Delta rows (threads 0-63) ----------------------------------------------
                ok = tc::mbar_wait(&S.bar_a, c & 1) && ok;
                tc::tc_fence_after();
                float x[NS];
                tc::tmem_ld32(tA + (uint32_t)(c % nb) * 32 + lane_base, x);
                tc::tmem_wait_ld();
                const float dr = B.SC[64 + t], uinv = TR ? 0.f : B.SC[SC_UINV];   // TR: v = 0
                const uint4* urow = reinterpret_cast<const uint4*>(B.U + t * NS);
                float dv[NS];
#pragma unroll
                for (int nb8 = 0; nb8 < NS / 8; ++nb8) {   // 16-byte pieces of the row
                    const uint4 u = urow[nb8];
                    const f16* e = reinterpret_cast<const f16*>(&u);
#pragma unroll
                    for (int q = 0; q < 8; ++q) dv[nb8 * 8 + q] = __half2float(e[q]) * uinv;
                }
#pragma unroll
                for (int j = 0; j < NS; ++j) dv[j] -= x[j] * inv_sc;
                store_op_row(S.Dl, t, dv, sc);
                store_op_row(S.Dt, t, dv, dr * sc);
                tc::fence_async_smem();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&S.d_ready);
            } else {
                // ---- warps 2-3: the chunk's scalars; plain, then the previous chunk's output
                //      rows under this chunk's Delta epilogue and state MMA --------------------
                const float a_cur = OUTG ? 0.f : B.SC[t - 64];
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&S.d_ready);   // the stage's scalars are read
                if (!OUTG) {
                    if (c > 0) ok = write_output(c - 1) && ok;
                    a_prev = a_cur;
                    cn_prev = cn;
                    tok_prev = tok;
                }
            }
            // ---- state rows (all 128) ---------------------------------------------------------
            ok = tc::mbar_wait(&S.bar_b, c & 1) && ok;
            tc::tc_fence_after();
            {
                float y[NS];
                tc::tmem_ld32(tB + lane_base, y);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < NS; ++j) Hr[j] = fmaf(gC, Hr[j], y[j] * inv_sc);
            }
            store_op_row(S.H0[(c + 1) & 1], t, Hr, sc);
            tc::fence_async_smem();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.h0_ready);
            if (S.abort) ok = false;
        }
        if (!OUTG && warp >= 2 && ok && nch > 0) ok = write_output(nch - 1);   // the last chunk's rows
        if (!ok) {
            record_timeout(status);
            S.abort = 1;
        } else if (hT) {
#pragma unroll
            for (int j = 0; j < NS; ++j) hT[hrow + j] = Hr[j];
        }
    } else if (OUTG) {
        // ---------------- output warps 6-7: row i = TMEM lane 64 + i of D_a and D_c ----------
        // out = o rsqrt(mean(o^2) + eps) (1 + w) sigmoid(z) per row over the head's 128
        // values: this slice's sum of squares goes to the other three slice CTAs of the
        // cluster in one bulk copy per peer, completing on their barrier obar[chunk parity]
        const int i = tid - 192;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        tc::named_bar(3, 128 + 64);   // the state warps have published the data scale
        const float inv_sc = S.inv_sc;
        float wn[NS];   // 1 + w
#pragma unroll
        for (int j = 0; j < NS; ++j) wn[j] = S.onw[j];
        for (int cc = 0; cc < nch; ++cc) {
            const int k = cc % NZ, p = cc & 1;
            const int64_t tok = bos + (int64_t)C * cc;
            const int64_t rem = len - (int64_t)C * cc;
            const int cn = (int)(rem < C ? rem : C);
            bool good = tc::mbar_wait(&S.zfull[k], (uint32_t)((cc / NZ) & 1));
            good = tc::mbar_wait(&S.bar_o[cc % nb], (uint32_t)((cc / nb) & 1)) && good;
            tc::tc_fence_after();
            const uint32_t par = (uint32_t)(cc % nb) * 32;
            float q[NS], zc[NS];
            tc::tmem_ld32(tA + par + lane_base, q);
            tc::tmem_ld32(tC + par + lane_base, zc);
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.ofree[cc % nb]);   // the buffer may take chunk cc + nb
            const float a = S.zr[k].a[i];
            float ps = 0.f;
#pragma unroll
            for (int j = 0; j < NS; ++j) {   // the core output, then its sum of squares
                q[j] = fmaf(a, q[j], zc[j]) * inv_sc;
                ps = fmaf(q[j], q[j], ps);
            }
            S.oloc[p][i] = ps;
            tc::fence_async_smem();
            tc::named_bar(2, 64);   // the 64 rows are in oloc
            if (i == 0) {
                tc::mbar_expect_tx(&S.obar[p], (nslices - 1) * C * 4);
#pragma unroll
                for (int rk = 0; rk < nslices; ++rk)
                    if (rk != vs)
                        tc::bulk_copy_to_peer(tc::cluster_map(tc::smem_u32(&S.opart[p][vs][0]), rk), S.oloc[p], C * 4,
                                              tc::cluster_map(tc::smem_u32(&S.obar[p]), rk));
            }
            good = tc::mbar_wait_cluster(&S.obar[p], (uint32_t)((cc >> 1) & 1)) && good;
            float ss = ps;
#pragma unroll
            for (int rk = 0; rk < nslices; ++rk)
                if (rk != vs) ss += S.opart[p][rk][i];
            const float inv_rms = rsqrtf(ss * (1.f / D) + eps);
            if (i < cn) {
                const uint4* zrow = reinterpret_cast<const uint4*>(S.zr[k].z + i * NS);
                __align__(16) bf16 ob[NS];
#pragma unroll
                for (int qq = 0; qq < NS / 8; ++qq) {
                    const uint4 u = zrow[qq];
                    const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 zz = __bfloat1622float2(e[e2]);
                        const int j = qq * 8 + e2 * 2;
                        ob[j] = __float2bfloat16_rn(q[j] * inv_rms * wn[j] * sigmoid_fast(zz.x));
                        ob[j + 1] = __float2bfloat16_rn(q[j + 1] * inv_rms * wn[j + 1] * sigmoid_fast(zz.y));
                    }
                }
                uint4* dst = reinterpret_cast<uint4*>(o + ((tok + i) * HV + h) * D + vs * NS);
#pragma unroll
                for (int qq = 0; qq < NS / 8; ++qq) dst[qq] = reinterpret_cast<const uint4*>(ob)[qq];
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.zempty[k]);   // the slot may take chunk cc + NZ
            // both output warps leave together: a failed wait or an abort elsewhere
            if (tc::named_bar_any(2, 64, !good || S.abort)) {
                if (i == 0) record_timeout(status);
                S.abort = 1;
                break;
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (S.abort && tid == 0) {
        // let copies already issued land before the shared memory is released
        for (int i = 0; i < NSTAGE; ++i) (void)tc::mbar_wait(&S.full[i], 0, 50000000ull);
        if (OUTG)
            for (int i = 0; i < NZ; ++i) (void)tc::mbar_wait(&S.zfull[i], 0, 50000000ull);
    }
    __syncthreads();
    if (OUTG) tc::cluster_sync();   // no CTA leaves while a peer may still write its shared memory
    if (warp == 0) tc::tmem_dealloc(tmem, kCarryTmemCols);
}

// ======================================================================================
// host side
// ======================================================================================
struct TcLayout {
    int64_t max_chunks;
    size_t off_chunk, off_w, off_u, off_p, off_qk, off_sc, total;
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Upper bound on the chunk count of any split of n_tokens into n_seqs sequences (each
// sequence adds at most one partial chunk); used for dense and packed layouts alike.
TcLayout tc_layout(int64_t n_tokens, int n_seqs, int HK, int HV) {
    TcLayout L;
    L.max_chunks = (n_tokens + C - 1) / C + n_seqs;
    const size_t rows = (size_t)L.max_chunks * HV * 64;
    L.off_chunk = kStatusBytes;
    L.off_w = round_up(L.off_chunk + (size_t)(n_seqs + 1) * 4, 1024);
    L.off_u = round_up(L.off_w + rows * D * 2, 1024);
    L.off_p = round_up(L.off_u + rows * D * 2, 1024);
    L.off_qk = round_up(L.off_p + rows * 64 * 2, 1024);
    L.off_sc = round_up(L.off_qk + (size_t)L.max_chunks * HK * 128 * D * 2, 1024);
    L.total = round_up(L.off_sc + (size_t)L.max_chunks * HV * SC_FLOATS * 4, 1024);
    return L;
}

}  // namespace

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool prefill_tc_supported(int Dk, int Dv, int HK, int HV, int BT) {
    return Dk == D && Dv == D && BT == C && HV % HK == 0 && (HV / HK == 1 || HV / HK == 2 || HV / HK == 4);
}

size_t prefill_tc_workspace_bytes(int64_t n_tokens, int n_seqs, int HK, int HV) {
    // TMA coordinates are 32-bit: token index, tile rows (chunk, head) * 64 and * 128
    const int64_t max_chunks = (n_tokens + C - 1) / C + n_seqs;
    if (n_tokens > INT32_MAX || max_chunks * HV * 64 > INT32_MAX || max_chunks * HK * 128 > INT32_MAX) return 0;
    return tc_layout(n_tokens, n_seqs, HK, HV).total;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, void* workspace, cudaStream_t s) {
    const bool packed = a.cu != nullptr;
    const int64_t n_tokens = packed ? a.T : (int64_t)a.n_seqs * a.T;
    const TcLayout L = tc_layout(n_tokens, a.n_seqs, a.HK, a.HV);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* chunk_off = reinterpret_cast<int32_t*>(ws + L.off_chunk);
    f16* W = reinterpret_cast<f16*>(ws + L.off_w);
    f16* U = reinterpret_cast<f16*>(ws + L.off_u);
    f16* P = reinterpret_cast<f16*>(ws + L.off_p);
    f16* QK = reinterpret_cast<f16*>(ws + L.off_qk);
    float* SC = reinterpret_cast<float*>(ws + L.off_sc);

    chunk_table_kernel<<<1, 1024, 0, s>>>(a.cu, a.n_seqs, a.T, chunk_off, a.status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    if (n_tokens == 0 && a.hT == nullptr) return cudaSuccess;

    // tensor maps: bf16 inputs for the chunk-local stage, fp16 intermediates for the carry
    CUtensorMap tq, tk, tv, tw, tu, tp, tqk;
    const cuuint64_t tok = (cuuint64_t)(n_tokens > 0 ? n_tokens : 1);
    {
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.HK, tok};
        cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.HK * D * 2};
        cuuint32_t box[3] = {64, 1, 64};
        const void* qb = a.q ? a.q : workspace;
        const void* kb = a.k ? a.k : workspace;
        if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qb, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        if (!make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kb, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.HV, tok};
        cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.HV * D * 2};
        cuuint32_t box[3] = {64, 1, 64};
        const void* vb = a.v ? a.v : workspace;
        if (!make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, vb, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    const cuuint64_t mc = (cuuint64_t)(L.max_chunks > 0 ? L.max_chunks : 1);
    const cuuint64_t rows = mc * a.HV * 64;
    {
        cuuint64_t dims[2] = {(cuuint64_t)D, rows};
        cuuint64_t str[1] = {(cuuint64_t)D * 2};
        cuuint32_t box[2] = {64, 64};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, W, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        cuuint32_t boxu[2] = {NS, 64};
        if (!make_map(&tu, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, U, 2, dims, str, boxu, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {64, rows};
        cuuint64_t str[1] = {64 * 2};
        cuuint32_t box[2] = {64, 64};
        if (!make_map(&tp, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, P, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)D, mc * a.HK * 128};
        cuuint64_t str[1] = {(cuuint64_t)D * 2};
        cuuint32_t box[2] = {64, 64};
        if (!make_map(&tqk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, QK, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }

    const int G = a.HV / a.HK;
    if (n_tokens > 0 && L.max_chunks > 0) {
        dim3 grid((unsigned)L.max_chunks, (unsigned)a.HK);
        auto launch_prep = [&](auto kern) -> cudaError_t {
            cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)kPrepSmemBytes);
            if (err == cudaSuccess)   // four CTAs per SM need the largest shared-memory carveout
                err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                           (int)cudaSharedmemCarveoutMaxShared);
            if (err != cudaSuccess) return err;
            kern<<<grid, 128, kPrepSmemBytes, s>>>(tq, tk, tv, a.gates, a.cu, chunk_off, a.T, a.n_seqs, a.HV,
                                                   a.scale, a.l2norm, a.HK, W, U, tp, tqk, SC, a.status,
                                                   testing_stall_site() == GDN_STALL_PREFILL_PREP ? 1 : 0);
            return cudaSuccess;
        };
        e = G == 1 ? launch_prep(chunk_prep_kernel<1>) : G == 2 ? launch_prep(chunk_prep_kernel<2>)
                                                                 : launch_prep(chunk_prep_kernel<4>);
        if (e != cudaSuccess) return e;
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        count_launch();
    }
    const unsigned blocks = (unsigned)a.n_seqs * (unsigned)a.HV * (unsigned)(D / NS);
    if (!a.z) {
        e = cudaFuncSetAttribute(chunk_carry_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kCarrySmemBytes);
        if (e != cudaSuccess) return e;
        chunk_carry_kernel<false><<<blocks, carry_threads(false), kCarrySmemBytes, s>>>(
            tw, tqk, tp, tu, tw, SC, a.cu, chunk_off, a.T, a.n_seqs, a.HK, a.HV, a.h0, a.hT, (bf16*)a.o, nullptr,
            nullptr, 0.f, a.status);
        if (a.o_tr) {   // the transition run on the same chunk-local operands: v = 0 from the identity
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            count_launch();
            e = cudaFuncSetAttribute(chunk_carry_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kCarrySmemBytes);
            if (e != cudaSuccess) return e;
            chunk_carry_kernel<false, true><<<blocks, carry_threads(false), kCarrySmemBytes, s>>>(
                tw, tqk, tp, tu, tw, SC, a.cu, chunk_off, a.T, a.n_seqs, a.HK, a.HV, nullptr, a.hT_tr,
                (bf16*)a.o_tr, nullptr, nullptr, 0.f, a.status);
        }
    } else {   // the head's four column slices as one cluster (output epilogue)
        // z [tokens, HV, Dv] bf16: one slice's 32 values of one head for 64 tokens per tile
        CUtensorMap tz;
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.HV, tok};
        cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.HV * D * 2};
        cuuint32_t box[3] = {NS, 1, 64};
        if (!make_map(&tz, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.z, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
        e = cudaFuncSetAttribute(chunk_carry_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kCarrySmemBytes);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(blocks);
        cfg.blockDim = dim3(carry_threads(true));
        cfg.dynamicSmemBytes = kCarrySmemBytes;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = D / NS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, chunk_carry_kernel<true>, tw, tqk, tp, tu, tz, (const float*)SC, a.cu,
                               (const int32_t*)chunk_off, a.T, a.n_seqs, a.HK, a.HV, a.h0, a.hT, (bf16*)a.o,
                               (const bf16*)a.z, a.norm_w, a.eps, a.status);
        if (e != cudaSuccess) return e;
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    return cudaSuccess;
}

}  // namespace gdn
