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
                                                           int32_t* __restrict__ status,
                                                           int32_t* __restrict__ flags, int64_t n_flags) {
    __shared__ int s_part[1024];
    __shared__ int s_bad;
    const int tid = threadIdx.x;
    for (int64_t i = tid; i < n_flags; i += 1024) flags[i] = 0;   // ready flags of the fused launch
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
// In-place T = (I + L)^-1 for a 64 x 64 strictly lower L held in M (fp32, row stride 65),
// 128 threads.  On return the strictly lower triangle of M holds T (its unit diagonal is
// implied); entries on and above the diagonal are untouched.  Blocks of 16:
//  * diagonal blocks T_bb = (I + L_bb)^-1 by right-looking column substitution: every
//    finished x_j updates all later rows at once, so the dependent chain is one FMA per row;
//  * block rows I = 1, 2, 3: T_Ij = -T_II sum_{k=j}^{I-1} L_Ik T_kj for all j < I at once,
//    one warp per j, the 16 x 16 block products on mma.sync with fp16 operands (the T
//    entries are rounded to fp16 for the W / U operands anyway).  Row block I of L is
//    read only while row block I of T is formed, so T overwrites it.
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
__device__ __forceinline__ float blk(const float (*M)[65], int r0, int c0, int r, int c) {
    if (UNIT) return r == c ? 1.f : (r > c ? M[r0 + r][c0 + c] : 0.f);
    return M[r0 + r][c0 + c];
}
template <bool UNIT>
__device__ __forceinline__ void frag_a(uint32_t* a, const float (*M)[65], int r0, int c0, int g, int q) {
    a[0] = pack_h2(blk<UNIT>(M, r0, c0, g, 2 * q), blk<UNIT>(M, r0, c0, g, 2 * q + 1));
    a[1] = pack_h2(blk<UNIT>(M, r0, c0, g + 8, 2 * q), blk<UNIT>(M, r0, c0, g + 8, 2 * q + 1));
    a[2] = pack_h2(blk<UNIT>(M, r0, c0, g, 2 * q + 8), blk<UNIT>(M, r0, c0, g, 2 * q + 9));
    a[3] = pack_h2(blk<UNIT>(M, r0, c0, g + 8, 2 * q + 8), blk<UNIT>(M, r0, c0, g + 8, 2 * q + 9));
}
// B fragment of the 16 x 8 slice (all 16 rows, columns n0 .. n0+7) of a block
template <bool UNIT>
__device__ __forceinline__ void frag_b(uint32_t* b, const float (*M)[65], int r0, int c0, int n0, int g, int q) {
    b[0] = pack_h2(blk<UNIT>(M, r0, c0, 2 * q, n0 + g), blk<UNIT>(M, r0, c0, 2 * q + 1, n0 + g));
    b[1] = pack_h2(blk<UNIT>(M, r0, c0, 2 * q + 8, n0 + g), blk<UNIT>(M, r0, c0, 2 * q + 9, n0 + g));
}

// Block row I of T: warp j (< I) forms X_j = sum_{k=j}^{I-1} L_Ik T_kj, then T_Ij = -T_II X_j.
template <int I>
__device__ __forceinline__ void tinv_row_block(float (*M)[65], float (*X)[16][17], int tid, int bar) {
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const float(*Xc)[17] = nullptr;
    if (warp < I) {
        const int j = warp;
        float acc[2][4] = {};
#pragma unroll
        for (int k = 0; k < I; ++k) {
            if (k < j) continue;
            uint32_t a[4], b[2];
            frag_a<false>(a, M, 16 * I, 16 * k, g, q);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                if (k == j) frag_b<true>(b, M, 16 * k, 16 * j, 8 * nt, g, q);
                else frag_b<false>(b, M, 16 * k, 16 * j, 8 * nt, g, q);
                mma16816(acc[nt], a, b);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            X[j][g][8 * nt + 2 * q] = acc[nt][0];
            X[j][g][8 * nt + 2 * q + 1] = acc[nt][1];
            X[j][g + 8][8 * nt + 2 * q] = acc[nt][2];
            X[j][g + 8][8 * nt + 2 * q + 1] = acc[nt][3];
        }
    }
    tc::named_bar(bar, 128);   // every read of row block I of L is done before it is overwritten
    if (warp < I) {
        const int j = warp;
        Xc = X[j];
        float acc[2][4] = {};
        uint32_t a[4], b[2];
        frag_a<true>(a, M, 16 * I, 16 * I, g, q);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            b[0] = pack_h2(Xc[2 * q][8 * nt + g], Xc[2 * q + 1][8 * nt + g]);
            b[1] = pack_h2(Xc[2 * q + 8][8 * nt + g], Xc[2 * q + 9][8 * nt + g]);
            mma16816(acc[nt], a, b);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            M[16 * I + g][16 * j + 8 * nt + 2 * q] = -acc[nt][0];
            M[16 * I + g][16 * j + 8 * nt + 2 * q + 1] = -acc[nt][1];
            M[16 * I + g + 8][16 * j + 8 * nt + 2 * q] = -acc[nt][2];
            M[16 * I + g + 8][16 * j + 8 * nt + 2 * q + 1] = -acc[nt][3];
        }
    }
    tc::named_bar(bar, 128);
}

// The 128 threads of one worker run it; `bar` is their named barrier (0 when they are the
// whole CTA).
__device__ __forceinline__ void tinv64_inplace(float (*M)[65], float (*X)[16][17], int tid, int bar) {
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
    tc::named_bar(bar, 128);   // all reads of the diagonal blocks of L precede their overwrite
    if (tid < 64) {
#pragma unroll
        for (int i = 1; i < 16; ++i)
            if (i > c) M[o + i][o + c] = col[i];
    }
    tc::named_bar(bar, 128);
    tinv_row_block<1>(M, X, tid, bar);
    tinv_row_block<2>(M, X, tid, bar);
    tinv_row_block<3>(M, X, tid, bar);
}

// ======================================================================================
// chunk_prep
// ======================================================================================
struct PrepSmem {
    // [K; Q] in two 64-column halves (rows 0-63 K, 64-127 Q), 16 KB each.  Rows 0-63 are
    // rewritten in place as fp16 K_hat; rows 64-127 are reused for V (bf16 from TMA, then
    // fp16 V * sv in place) once Q_hat has been written out.
    uint16_t KQ[2][128 * 64];
    // L, then T in place (fp32, row stride 65); then, in the same bytes, the fp16 MMA
    // operands T diag(b gamma) (bytes 0-8191) and T diag(b) (8192-16383), K-major 128B-swizzled
    float M[64][65];
    float X[3][16][17];
    float rk[64], rq[64], G[64], bt[64], bgr[64], red[8];
    float eu[64];   // rk_j exp(G_r - G_j), the token factor of the separated decays
    float dd[64];   // exp(G_C - G_j): the decay from token j to the chunk's end (K_tilde rows)
    float ga[2][64], ba[2][64];   // g, beta of value head gi in slot gi % 2, loaded ahead
    uint64_t bar_load, bar_v, bar_mma;
    uint32_t tmem_base;
};
static_assert(offsetof(PrepSmem, M) % 1024 == 0, "the swizzled operands in M need 1024-byte alignment");
constexpr size_t kPrepSmemBytes = sizeof(PrepSmem) + 1024;
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

// Row t = tid of a 128 x 64 fp16 tile from TMEM lane t (64 fp32 columns), stored as one
// contiguous 128-byte row: the tile's transpose in the layout the MMA produced it.
__device__ __forceinline__ void store_rows_from_tmem(f16* __restrict__ dst, uint32_t taddr, int tid) {
    uint4* d = reinterpret_cast<uint4*>(dst + (size_t)tid * 64);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        float w[32];
        tc::tmem_ld32(taddr + part * 32, w);
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint4 u;
            u.x = pack_h2(w[8 * c + 0], w[8 * c + 1]);
            u.y = pack_h2(w[8 * c + 2], w[8 * c + 3]);
            u.z = pack_h2(w[8 * c + 4], w[8 * c + 5]);
            u.w = pack_h2(w[8 * c + 6], w[8 * c + 7]);
            d[part * 4 + c] = u;
        }
    }
}

// Where one worker's chunk-local results go.
struct PrepOut {
    f16* W;          // [rows, 128]: W of each (chunk, value head), 64 rows
    f16* U;          // two-kernel path: [rows, 128] U * 2^-e (e per chunk and value head); fused: its
                     //   transpose, [(chunk, value head) * 128 + value, 64 tokens]
    f16* P;          // [rows, 64]: P (two-kernel path) or P^T (fused path)
    f16* QK;         // two-kernel path: [K_hat; Q_hat] per (chunk, q/k head), 128 rows; fused: Q_hat, 64 rows
    float* SC;       // [chunks * HV, SC_FLOATS] per-row scalars
    f16* Kt;         // fused: K_tilde = diag(exp(G_C - G)) K_hat per (chunk, value head), 64 rows
    int32_t* flags;  // fused: per (chunk, q/k head) ready flag, set once all of the above are written
};

// Barrier phases a worker carries from one item to the next.
struct PrepPhases {
    uint32_t load = 0;     // parity of the next K / Q tile wait
    uint32_t mma = 0;      // parity of the next product wait
    uint32_t vcount = 0;   // V tile copies issued so far
};

// The chunk-local stage for one (chunk, q/k head) item, run by 128 threads (tid 0-127, their
// TMEM lanes 0-127 at column base `tmem`, named barrier `bar`).  Returns false if a bounded
// wait gave up (recorded in `status`; what was issued has landed again on return).
// FUSED writes P^T, Q_hat alone and K_tilde per value head (the operands of the fused
// carry), then raises the item's ready flag.
// issue the K and Q tile copies of item (chunk at token s, q/k head hk) on bar_load (one thread)
__device__ __forceinline__ void prep_load_kq(PrepSmem& S, const CUtensorMap* tm_q, const CUtensorMap* tm_k, int hk,
                                             int si) {
    uint8_t* kq = reinterpret_cast<uint8_t*>(&S.KQ[0][0]);
    tc::mbar_expect_tx(&S.bar_load, 4 * 64 * 64 * 2);
    tc::tma_load_3d(kq, tm_k, &S.bar_load, 0, hk, si);
    tc::tma_load_3d(kq + 16384, tm_k, &S.bar_load, 64, hk, si);
    tc::tma_load_3d(kq + 8192, tm_q, &S.bar_load, 0, hk, si);
    tc::tma_load_3d(kq + 16384 + 8192, tm_q, &S.bar_load, 64, hk, si);
}

// FUSED: `loaded` says this item's K, Q copies were issued by the item before; next_hk >= 0 asks
// for the next item's copies (q/k head next_hk at token next_s) to be issued at the end, before
// the release of this item's flag, so that their latency overlaps it.
template <int G, bool FUSED>
__device__ bool prep_item(PrepSmem& S, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                          const float* __restrict__ g, const float* __restrict__ beta, int chunk, int hk, int64_t s,
                          int cn, int HV, int HK, float scale, int l2norm, const PrepOut& out,
                          int32_t* __restrict__ status, bool stall, uint32_t tmem, int tid, int bar, PrepPhases& ph,
                          bool loaded = false, int next_hk = -1, int64_t next_s = 0) {
    const int warp = tid >> 5;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // TMEM: columns 0-63 the Gram tiles (kept for every value head), 64-127 W^T; U^T goes
    // to 64-127 after W^T is read out, except for the last value head, whose U^T takes the
    // Gram columns (no longer needed) so both products run back to back.
    const uint32_t tG = tmem, tW = tmem + 64;
    const int si = (int)s;
    uint8_t* kq = reinterpret_cast<uint8_t*>(&S.KQ[0][0]);
    const uint32_t load_par = ph.load;
    ph.load ^= 1u;
    const uint32_t vbase = ph.vcount;   // V copies of earlier items
    bool ok;

    if (tid == 0 && !loaded) prep_load_kq(S, tm_q, tm_k, hk, si);
    if (tid < 64) {   // gates of the group's first two value heads, under the TMA latency
#pragma unroll
        for (int gi = 0; gi < (G < 2 ? G : 2); ++gi) {
            const int h = hk * G + gi;
            S.ga[gi][tid] = tid < cn ? g[(s + tid) * HV + h] : 0.f;
            S.ba[gi][tid] = tid < cn ? beta[(s + tid) * HV + h] : 0.f;
        }
    }
    ok = tc::mbar_wait(&S.bar_load, load_par);
    if (tc::named_bar_any(bar, 128, !ok)) goto abort;

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
    ok = tc::mbar_wait(&S.bar_mma, ph.mma);
    ph.mma ^= 1u;
    if (tc::named_bar_any(bar, 128, !ok)) goto abort;
    tc::tc_fence_after();
    {
        const float rki = tid < 64 ? S.rk[tid] : 0.f;
        const float rqi = tid >= 64 ? S.rq[tid - 64] : 0.f;
        {   // K_hat (tid < 64) / Q_hat row: fp16 in place (K_hat feeds the W MMA) and out to
            // global in natural column order; rows past the chunk are zeroed
            const float rr = tid < cn || (tid >= 64 && tid - 64 < cn) ? (tid < 64 ? rki : rqi) : 0.f;
            uint4* dst = nullptr;
            if (!FUSED) dst = reinterpret_cast<uint4*>(out.QK + (((size_t)chunk * HK + hk) * 128 + tid) * D);
            else if (tid >= 64) dst = reinterpret_cast<uint4*>(out.QK + (((size_t)chunk * HK + hk) * 64 + tid - 64) * D);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint4* row = reinterpret_cast<uint4*>(kq + half * 16384 + tid * 128);
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                    const int pc = c16 ^ (tid & 7);   // logical chunk c16 sits at c16 ^ (row % 8)
                    const uint4 u = row[pc];
                    const bf16* e = reinterpret_cast<const bf16*>(&u);
                    __align__(16) f16 hx[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) hx[t] = __float2half_rn(__bfloat162float(e[t]) * rr);
                    const uint4 hv = *reinterpret_cast<const uint4*>(hx);
                    row[pc] = hv;
                    if (dst) dst[half * 8 + c16] = hv;
                }
            }
        }
        tc::fence_async_smem();
        tc::named_bar(bar, 128);
        // Q is consumed: its rows now receive V of the first value head (test hook,
        // gdn_testing_stall: not for the first item, whose wait for it then runs out)
        if (!FUSED && !stall) {
            ++ph.vcount;   // every thread counts the copies: the parity of each V wait follows from it
            if (tid == 0) {
                tc::mbar_expect_tx(&S.bar_v, 2 * 64 * 64 * 2);
                tc::tma_load_3d(kq + 8192, tm_v, &S.bar_v, 0, hk * G, si);
                tc::tma_load_3d(kq + 16384 + 8192, tm_v, &S.bar_v, 64, hk * G, si);
            }
        }

        for (int gi = 0; gi < G; ++gi) {
            const int h = hk * G + gi;
            const size_t ch = (size_t)chunk * HV + h;
            const bool last = gi == G - 1;
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
            tc::named_bar(bar, 128);
            if (G > 2 && gi + 2 < G && tid < 64) {   // slot gi % 2 is read: value head gi + 2's gates
                S.ga[gi & 1][tid] = tid < cn ? g[(s + tid) * HV + h + 2] : 0.f;
                S.ba[gi & 1][tid] = tid < cn ? beta[(s + tid) * HV + h + 2] : 0.f;
            }
            if (tid >= 32 && tid < 64) S.G[tid] += S.G[31];
            tc::named_bar(bar, 128);
            if (tid < 64) S.bgr[tid] = S.bt[tid] * expf(S.G[tid]);
            const float Gl = S.G[63];   // padding adds 0, so this is G at the last token
            // exp(G_i - G_j) = exp(G_i - G_r) exp(G_r - G_j) with G_r = G_last / 2: both
            // factors stay inside fp32 range while G_last >= -160, and the row loops below
            // then need no exponential per pair; deeper decays take exp(G_i - G_j) directly
            const bool sep = Gl >= -160.f;
            const float Gr = 0.5f * Gl;
            if (sep) {
                if (tid < 64) S.eu[tid] = S.rk[tid] * __expf(Gr - S.G[tid]);
                tc::named_bar(bar, 128);
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
#pragma unroll
                        for (int j = 0; j < 64; ++j) S.M[i][j] = j < i ? ai * S.eu[j] * row[j] : 0.f;
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            float v = 0.f;
                            if (j < i && i < cn) v = bi * __expf(Gi - S.G[j]) * S.rk[j] * row[j];
                            S.M[i][j] = v;
                        }
                    }
                    const float di = i < cn ? expf(Gl - Gi) : 0.f;
                    out.SC[ch * SC_FLOATS + 64 + i] = di;
                    if (FUSED) S.dd[i] = di;
                } else {
                    const int i = tid - 64;
                    const float Gi = S.G[i], qi = scale * rqi;
                    out.SC[ch * SC_FLOATS + i] = i < cn ? scale * expf(Gi) : 0.f;
                    if (i == 0) out.SC[ch * SC_FLOATS + SC_GC] = expf(Gl);
                    const float ai = sep && i < cn ? qi * __expf(Gi - Gr) : 0.f;
                    if (!FUSED) {
                        uint4* prow = reinterpret_cast<uint4*>(out.P + (ch * 64 + i) * 64);
#pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8) {
                            __align__(16) f16 e[8];
#pragma unroll
                            for (int t = 0; t < 8; ++t) {
                                const int j = c8 * 8 + t;
                                float v = 0.f;
                                if (sep) v = j <= i ? ai * S.eu[j] * row[j] : 0.f;
                                else if (j <= i && i < cn) v = qi * __expf(Gi - S.G[j]) * S.rk[j] * row[j];
                                e[t] = __float2half_rn(v);
                            }
                            prow[c8] = *reinterpret_cast<const uint4*>(e);
                        }
                    } else {   // P^T: P[i][j] at row j, column i of a staging tile (the V rows of K / Q
                               // half 0, free until this head's V is loaded); a warp writes 64
                               // contiguous bytes per j
                        f16* pst = reinterpret_cast<f16*>(kq + 8192) + i;
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            float v = 0.f;
                            if (sep) v = j <= i ? ai * S.eu[j] * row[j] : 0.f;
                            else if (j <= i && i < cn) v = qi * __expf(Gi - S.G[j]) * S.rk[j] * row[j];
                            pst[j * 64] = __float2half_rn(v);
                        }
                    }
                }
            }
            tc::named_bar(bar, 128);
            if (FUSED) {
                // K_tilde = diag(d) K_hat and P^T out, 16 bytes per thread and copy, 16 consecutive
                // threads on one row: every store instruction covers whole rows
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int m = tid + 128 * r, krow = m >> 4, c16 = m & 15;
                    const uint4 u = *reinterpret_cast<const uint4*>(kq + (c16 >> 3) * 16384 + krow * 128 +
                                                                    (((c16 & 7) ^ (krow & 7)) << 4));
                    const __half2* e = reinterpret_cast<const __half2*>(&u);
                    const __half2 dd = __float2half2_rn(S.dd[krow]);
                    uint4 o4;
                    __half2* oh = reinterpret_cast<__half2*>(&o4);
#pragma unroll
                    for (int t = 0; t < 4; ++t) oh[t] = __hmul2(e[t], dd);
                    reinterpret_cast<uint4*>(out.Kt + (ch * 64 + krow) * D)[c16] = o4;
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int m = tid + 128 * r;   // 16-byte piece m of the 8 KB P^T tile
                    reinterpret_cast<uint4*>(out.P + ch * 64 * 64)[m] = reinterpret_cast<const uint4*>(kq + 8192)[m];
                }
                // the staging tile is read: this head's V may now overwrite it (the copies run
                // under the inverse below)
                tc::fence_async_smem();
                tc::named_bar(bar, 128);
                if (!(stall && gi == 0)) {
                    ++ph.vcount;
                    if (tid == 0) {
                        tc::mbar_expect_tx(&S.bar_v, 2 * 64 * 64 * 2);
                        tc::tma_load_3d(kq + 8192, tm_v, &S.bar_v, 0, h, si);
                        tc::tma_load_3d(kq + 16384 + 8192, tm_v, &S.bar_v, 64, h, si);
                    }
                }
            }
            tinv64_inplace(S.M, S.X, tid, bar);
            // ---- fp16 MMA operands T diag(b gamma) and T diag(b), 128B-swizzled, written
            //      over M once every thread holds its part of T -----------------------------
            {
                const int i = tid >> 1, c0 = (tid & 1) * 32;
                float tv[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const int j = c0 + t;
                    tv[t] = j < i ? S.M[i][j] : (j == i ? 1.f : 0.f);
                }
                tc::named_bar(bar, 128);
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
            ok = tc::mbar_wait(&S.bar_v, (vbase + (uint32_t)gi) & 1u);
            if (tc::named_bar_any(bar, 128, !ok)) goto abort;
            {
                const int r = tid >> 1, half = tid & 1;
                uint4* vr = reinterpret_cast<uint4*>(kq + half * 16384 + 8192 + r * 128);
                float vmax = 0.f;
                if (r < cn) {
#pragma unroll
                    for (int c16 = 0; c16 < 8; ++c16) {
                        const uint4 u = vr[c16 ^ (r & 7)];
                        const bf16* e = reinterpret_cast<const bf16*>(&u);
#pragma unroll
                        for (int t = 0; t < 8; ++t) vmax = fmaxf(vmax, fabsf(__bfloat162float(e[t])));
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
                if ((tid & 31) == 0) S.red[warp] = vmax;
                tc::named_bar(bar, 128);
                vmax = fmaxf(fmaxf(S.red[0], S.red[1]), fmaxf(S.red[2], S.red[3]));
                const float uinv = pow2_above(vmax), sv = r < cn ? 1.f / uinv : 0.f;
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                    const int pc = c16 ^ (r & 7);
                    const uint4 u = vr[pc];
                    const bf16* e = reinterpret_cast<const bf16*>(&u);
                    __align__(16) f16 hx[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) hx[t] = __float2half_rn(__bfloat162float(e[t]) * sv);
                    vr[pc] = *reinterpret_cast<const uint4*>(hx);
                }
                if (tid == 0) {
                    out.SC[ch * SC_FLOATS + SC_UINV] = uinv;
                    out.SC[ch * SC_FLOATS + SC_VMAX] = vmax;
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::named_bar(bar, 128);
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
            ok = tc::mbar_wait(&S.bar_mma, ph.mma);
            ph.mma ^= 1u;
            if (tc::named_bar_any(bar, 128, !ok)) goto abort;
            tc::tc_fence_after();
            // ---- epilogue: lane t of D_W / D_U is column t of W / U -----------------------
            store_tile_from_tmem(out.W + ch * 64 * D, tW + lane_base, tid);
            if (!last) {   // U^T into the W^T columns once they are read
                tc::tc_fence_before();
                tc::named_bar(bar, 128);
                if (tid == 0) {
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(tW, tc::desc_sw128(vb + kk * 2048, 16384, 1024),
                                     tc::desc_sw128(aub + kk * 32, 16, 1024), idx, kk > 0);
                    tc::mma_commit(&S.bar_mma);
                }
                ok = tc::mbar_wait(&S.bar_mma, ph.mma);
                ph.mma ^= 1u;
                if (tc::named_bar_any(bar, 128, !ok)) goto abort;
                tc::tc_fence_after();
                if (!FUSED) {
                    ++ph.vcount;
                    if (tid == 0) {   // the V rows are free again: next head's V
                        tc::mbar_expect_tx(&S.bar_v, 2 * 64 * 64 * 2);
                        tc::tma_load_3d(kq + 8192, tm_v, &S.bar_v, 0, h + 1, si);
                        tc::tma_load_3d(kq + 16384 + 8192, tm_v, &S.bar_v, 64, h + 1, si);
                    }
                }
            }
            if (FUSED) store_rows_from_tmem(out.U + ch * 128 * 64, (last ? tG : tW) + lane_base, tid);
            else store_tile_from_tmem(out.U + ch * 64 * D, (last ? tG : tW) + lane_base, tid);
            tc::tc_fence_before();
            tc::named_bar(bar, 128);   // TMEM reads done; M (the operands) free for the next head
        }
    }
    // the next item's tile copies overwrite what this one wrote to the tiles with generic stores
    tc::fence_async_smem();
    tc::tc_fence_before();
    tc::named_bar(bar, 128);
    if (FUSED) {
        if (tid == 0 && next_hk >= 0) prep_load_kq(S, tm_q, tm_k, next_hk, (int)next_s);
        // every thread's writes of this item, then the flag (release, GPU scope)
        __threadfence();
        tc::named_bar(bar, 128);
        if (tid == 0) {
            asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(out.flags + (size_t)chunk * HK + hk), "r"(1)
                         : "memory");
        }
    }
    return true;
abort:
    if (tid == 0) {
        record_timeout(status);
        // the copies and products still in flight land before the shared memory and TMEM are
        // released or reused; each wait is for the latest phase of its barrier (at once if
        // complete)
        (void)tc::mbar_wait(&S.bar_load, load_par, 50000000ull);
        if (ph.vcount > vbase) (void)tc::mbar_wait(&S.bar_v, (ph.vcount - 1u) & 1u, 50000000ull);
        (void)tc::mbar_wait(&S.bar_mma, ph.mma ^ 1u, 50000000ull);
    }
    tc::tc_fence_before();
    tc::named_bar(bar, 128);
    return false;
}

// The chunk-local stage of the two-kernel path: one CTA per (chunk, q/k head), four per SM.
template <int G>
__global__ void __launch_bounds__(128, 4)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ g,
                  const float* __restrict__ beta, const int32_t* __restrict__ cu,
                  const int32_t* __restrict__ chunk_off, int64_t T, int n_seqs, int HV, float scale,
                  int l2norm, int HK, PrepOut out, int32_t* __restrict__ status, int stall) {
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
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    PrepPhases ph;
    (void)prep_item<G, false>(S, &tm_q, &tm_k, &tm_v, g, beta, chunk, hk, s, cn, HV, HK, scale, l2norm, out, status,
                              stall && chunk == 0 && hk == 0, tmem, tid, 0, ph);
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
    ZSlot zr[NZ];          // output epilogue: z tiles and scalars, chunk c in slot c % NZ
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
static_assert(offsetof(CarrySmem, zr) % 16 == 0 && sizeof(ZSlot) % 16 == 0 && offsetof(ZSlot, a) % 16 == 0 &&
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
// Fused prefill: one cooperative launch, one CTA per SM.  CTAs [0, n_carry) carry the state
// of the (sequence, value head) chains; the others each hold four chunk-local workers
// (prep_item, FUSED) that run through the (chunk, q/k head) items in chunk order and raise a
// ready flag per item.  The carry waits on those flags, so the chunk-local work of later
// chunks runs while the state is carried through earlier ones; no worker ever waits on the
// carry, so neither side can block the other.
//
// Carry CTA, per chain (sequence n, value head h) and chunk (64 tokens), with the state
// held transposed in TMEM (lane v = value column v, H^T[v][k] = H[k][v]):
//   D1 = H^T [W; Q_hat]^T          A = H^T (fp16, TMEM), B = [W; Q_hat] (K-major)   8 MMAs, N = 128
//        -> columns 0-63: (W H)^T, columns 64-127: (Q_hat H)^T
//   Delta^T = U^T - (W H)^T        (epilogue, into TMEM as the next A operand)
//   D2 += Delta^T [K_tilde | P^T]  A = Delta^T (TMEM),  B MN-major                   4 MMAs, N = 192
//        -> columns 0-127 accumulate onto gamma_C H^T: the new state H^T (fp32, never leaves
//           TMEM but for its fp16 operand copy); columns 128-191: (P Delta)^T
//   O = diag(a) Q_hat H + P Delta  (output warps)
// so 12 tensor-core instructions per chunk and head (the instruction count, not the FLOPs,
// sets a tensor-core step's time).  The fp16 operands carry a data scale sc = 2^-e chosen per
// chunk from the exact max |H| of the state and max |v| of the chunk, so a quiet stretch that
// follows a loud one keeps its precision.
// Warps: 0 producer (flags, TMA), 1 MMA issue, 4-11 state epilogue (lane group w % 4, value
// column v; half (w - 4) / 4 of the K or token columns), 12-15 outputs.
// ======================================================================================
constexpr int kFcThreads = 512;
struct FcStage {
    uint8_t B1[2][128 * 128];   // [W; Q_hat]: rows 0-63 W, 64-127 Q_hat; K-major 128B-swizzled K halves
    uint8_t B2[3][64 * 128];    // K_tilde (two 64-column halves) and P^T: MN-major 128B-swizzled
    uint8_t U[128 * 128];       // U^T * 2^-e: [128 values][64 tokens], 128B-swizzled rows
    float SC[SC_FLOATS];
};
struct FcSmem {
    FcStage st[2];
    float red[2][8];            // max |H| per epilogue warp, alternating buffers
    float scale[4];             // data scale sc of step it, at it % 4
    float nxt[4][2];            // gamma_C and max |v| of step it, at it % 4, ahead of its stage
    uint64_t full[2], empty[2], d1, d2, h_ready, d_ready, ofree1, ofree2, scal[4];
    volatile int abort;
    int issued;                 // steps whose copies the producer has started
};
constexpr uint32_t kFcTx = (uint32_t)sizeof(FcStage);
static_assert(sizeof(FcStage) % 1024 == 0 && offsetof(FcStage, B2) % 1024 == 0 && offsetof(FcStage, U) % 1024 == 0 &&
                  offsetof(FcStage, SC) % 16 == 0,
              "fused carry stage layout");
constexpr size_t kPrepSlot = (sizeof(PrepSmem) + 1023) / 1024 * 1024;
constexpr size_t kFusedSmemBytes = (4 * kPrepSlot > sizeof(FcSmem) ? 4 * kPrepSlot : sizeof(FcSmem)) + 1024;
static_assert(kFusedSmemBytes <= 227 * 1024, "fused prefill: shared memory over the per-block limit");
// TMEM columns of a carry CTA
constexpr uint32_t kFcD1 = 0, kFcD2 = 128, kFcA1 = 320, kFcA2 = 384;

struct FusedArgs {
    const float* g;
    const float* beta;
    const int32_t* cu;
    const int32_t* chunk_off;
    int64_t T;
    int n_seqs, HK, HV;
    float scale;
    int l2norm;
    PrepOut out;
    const float* h0;
    float* hT;
    bf16* o;
    int32_t* status;
    int n_carry;
    int stall;
};

// Bounded wait on a barrier of the carry CTA that also gives up at once when another role
// has aborted.  Polls without suspending first (hand-offs on the serial chain are short).
__device__ __forceinline__ bool fc_wait(uint64_t* bar, uint32_t parity, const volatile int* abort,
                                        uint64_t timeout_ns = 2000000000ull) {
    const uint32_t addr = tc::smem_u32(bar);
    for (int i = 0; i < 2048; ++i)
        if (tc::mbar_test_wait(addr, parity)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (tc::mbar_try_wait(addr, parity)) return true;
        if (*abort) return false;
        const uint64_t dt = tc::globaltimer_ns() - t0;
        if (dt > timeout_ns) return false;
        if (dt > 20000) __nanosleep(128);
    }
}

// Wait (bounded) until a worker has published chunk-local item `flag`; gives up early if the
// device status word reports a failure or the CTA aborted.
__device__ __forceinline__ bool wait_flag(const int32_t* flag, const int32_t* status, const volatile int* abort) {
    if (tc::ld_acquire_gpu(flag)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    while (true) {
        for (int i = 0; i < 16; ++i)
            if (tc::ld_acquire_gpu(flag)) return true;
        if (*reinterpret_cast<const volatile int32_t*>(status) != 0 || *abort) return false;
        const uint64_t dt = tc::globaltimer_ns() - t0;
        if (dt > 2000000000ull) return false;
        if (dt > 20000) __nanosleep(256);
    }
}

__device__ __forceinline__ uint32_t pack_h2u(float lo, float hi) { return pack_h2(lo, hi); }

// Walk the chains of carry CTA `cta` in order; f(n, h, bos, len, c0, nch) per chain.
template <typename F>
__device__ __forceinline__ void for_each_chain(const FusedArgs& fa, F&& f) {
    const int n_chains = fa.n_seqs * fa.HV;
    for (int j = blockIdx.x; j < n_chains; j += fa.n_carry) {
        const int n = j / fa.HV, h = j - n * fa.HV;
        const int64_t bos = fa.cu ? (int64_t)fa.cu[n] : (int64_t)n * fa.T;
        const int64_t len = fa.cu ? (int64_t)fa.cu[n + 1] - fa.cu[n] : fa.T;
        const int c0 = fa.chunk_off[n];
        const int nch = fa.chunk_off[n + 1] - c0;
        if (!f(n, h, bos, len, c0, nch)) break;
    }
}

template <int G>
__device__ void fused_carry(FcSmem& S, const CUtensorMap* tm_w, const CUtensorMap* tm_qh, const CUtensorMap* tm_kt,
                            const CUtensorMap* tm_pt, const CUtensorMap* tm_u, const FusedArgs& fa, uint32_t tmem,
                            int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    const int HV = fa.HV, HK = fa.HK;
    const uint32_t tD1 = tmem + kFcD1, tD2 = tmem + kFcD2, tA1 = tmem + kFcA1, tA2 = tmem + kFcA2;
    const volatile int* abort = &S.abort;

    if (warp == 0) {
        // ---------------- producer: flags, then the chunk's operands by TMA ----------------
        if (lane != 0) return;
        int it = 0;
        for_each_chain(fa, [&](int n, int h, int64_t, int64_t, int c0, int nch) -> bool {
            const int hk = h / G;
            for (int c = 0; c < nch; ++c, ++it) {
                const int st = it & 1, r = it >> 1;
                FcStage& B = S.st[st];
                const int cid = c0 + c;
                // the step's two scalars first: the state epilogue of the step before needs them
                // (entry it % 4 is free again: its reader finished step it - 3 before the stage
                // this producer filled last was released)
                bool ok = wait_flag(fa.out.flags + (size_t)cid * HK + hk, fa.status, abort);
                if (ok) {
                    const float* scg = fa.out.SC + ((size_t)cid * HV + h) * SC_FLOATS;
                    S.nxt[it & 3][0] = scg[SC_GC];
                    S.nxt[it & 3][1] = scg[SC_VMAX];
                    tc::mbar_arrive(&S.scal[it & 3]);
                }
                ok = ok && (r == 0 || fc_wait(&S.empty[st], (uint32_t)((r - 1) & 1), abort));
                if (!ok) {
                    record_timeout(fa.status);
                    S.abort = 1;
                    return false;
                }
                tc::fence_async_global();   // the worker's stores, acquired above, before the copies
                const int row = (cid * HV + h) * 64, qrow = (cid * HK + hk) * 64;
                tc::mbar_expect_tx(&S.full[st], kFcTx);
                tc::tma_load_2d(B.B1[0], tm_w, &S.full[st], 0, row);
                tc::tma_load_2d(B.B1[1], tm_w, &S.full[st], 64, row);
                tc::tma_load_2d(B.B1[0] + 8192, tm_qh, &S.full[st], 0, qrow);
                tc::tma_load_2d(B.B1[1] + 8192, tm_qh, &S.full[st], 64, qrow);
                tc::tma_load_2d(B.B2[0], tm_kt, &S.full[st], 0, row);
                tc::tma_load_2d(B.B2[1], tm_kt, &S.full[st], 64, row);
                tc::tma_load_2d(B.B2[2], tm_pt, &S.full[st], 0, row);
                tc::tma_load_2d(B.U, tm_u, &S.full[st], 0, row * 2);   // U^T rows (chunk, head) * 128
                tc::bulk_load(B.SC, fa.out.SC + ((size_t)cid * HV + h) * SC_FLOATS, SC_FLOATS * 4, &S.full[st]);
                S.issued = it + 1;
            }
            return true;
        });
        return;
    }
    if (warp == 1) {
        // ---------------- MMA issue ------------------------------------------------------------
        if (lane != 0) return;
        constexpr uint32_t idD1 = tc::idesc_f16(128, 128, 0, 0);   // B K-major
        constexpr uint32_t idD2 = tc::idesc_f16(128, 192, 0, 1);   // B MN-major
        int it = 0, d1_issued = 0, d2_issued = 0;
        for_each_chain(fa, [&](int, int, int64_t, int64_t, int, int nch) -> bool {
            for (int c = 0; c < nch; ++c, ++it) {
                const int st = it & 1, r = it >> 1;
                const FcStage& B = S.st[st];
                bool ok = fc_wait(&S.full[st], (uint32_t)(r & 1), abort) &&
                          fc_wait(&S.h_ready, (uint32_t)(it & 1), abort) &&
                          fc_wait(&S.ofree1, (uint32_t)(it & 1), abort);
                if (!ok) {
                    record_timeout(fa.status);
                    S.abort = 1;
                    return false;
                }
                tc::tc_fence_after();
                const uint32_t b1 = tc::smem_u32(B.B1[0]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ts(tD1, tA1 + kk * 8, tc::desc_sw128(b1 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                                   idD1, kk > 0);
                tc::mma_commit(&S.d1);
                ++d1_issued;
                ok = fc_wait(&S.d_ready, (uint32_t)(it & 1), abort) && fc_wait(&S.ofree2, (uint32_t)(it & 1), abort);
                if (!ok) {
                    record_timeout(fa.status);
                    S.abort = 1;
                    return false;
                }
                tc::tc_fence_after();
                const uint64_t b2 = tc::desc_sw128(tc::smem_u32(B.B2[0]), 8192, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ts(tD2, tA2 + kk * 8, b2 + (uint64_t)((kk * 2048) >> 4), idD2, kk > 0);
                tc::mma_commit(&S.d2);
                tc::mma_commit(&S.empty[st]);
                ++d2_issued;
            }
            return true;
        });
        if (S.abort) {   // products still running land before TMEM is released (at once if done)
            if (d1_issued > 0) (void)tc::mbar_wait(&S.d1, (uint32_t)((d1_issued - 1) & 1), 50000000ull);
            if (d2_issued > 0) (void)tc::mbar_wait(&S.d2, (uint32_t)((d2_issued - 1) & 1), 50000000ull);
        }
        return;
    }
    if (warp >= 4 && warp < 12) {
        // ---------------- state epilogues: thread <-> (value column v, half hf) ------------------
        // The fp32 state stays in registers: this thread holds H[k][v] for k in [64 hf, 64 hf + 64).
        const int grp = warp & 3, v = grp * 32 + lane, hf = (warp - 4) >> 2;
        const uint32_t lb = (uint32_t)(grp * 32) << 16;
        const int wi = warp - 4;   // 0..7
        int it = 0, ruse = 0;
        bool ok = true;
        float sc = 1.f, inv_sc = 1.f;
        float H[64];
        // max |H| over the 8 epilogue warps (one bar.red per call keeps the warps' decisions
        // uniform: every warp learns whether any of them saw a failed wait)
        auto block_max = [&](float m, bool& good) -> float {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float* red = S.red[ruse & 1];
            ++ruse;
            if (lane == 0) red[wi] = m;
            good = !tc::named_bar_any(2, 256, !good || S.abort);
            float r = red[0];
#pragma unroll
            for (int i = 1; i < 8; ++i) r = fmaxf(r, red[i]);
            return r;
        };
        // the data scale of step `in` from max |H| and that step's max |v|, then the fp16 operand
        // H^T * sc into A1; returns with the operand complete in TMEM
        auto publish_state = [&](int in, bool& good) {
            float m = 0.f;
#pragma unroll
            for (int k = 0; k < 64; ++k) m = fmaxf(m, fabsf(H[k]));
            good = fc_wait(&S.scal[in & 3], (uint32_t)((in >> 2) & 1), abort) && good;
            m = block_max(m, good);
            if (!good) return;
            inv_sc = pow2_above(fmaxf(m, S.nxt[in & 3][1]));
            sc = 1.f / inv_sc;
            if (wi == 0 && lane == 0) S.scale[in & 3] = sc;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) pk[j] = pack_h2u(H[32 * part + 2 * j] * sc, H[32 * part + 2 * j + 1] * sc);
                tc::tmem_st16(tA1 + lb + 32 * hf + 16 * part, pk);
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.h_ready);
        };
        for_each_chain(fa, [&](int n, int h, int64_t, int64_t, int, int nch) -> bool {
            const size_t hrow = ((size_t)n * HV + h) * D * D;
#pragma unroll
            for (int k = 0; k < 64; ++k) H[k] = fa.h0 ? fa.h0[hrow + (size_t)(64 * hf + k) * D + v] : 0.f;
            if (nch == 0) {   // nothing to carry: the final state is the initial one
                if (fa.hT)
#pragma unroll
                    for (int k = 0; k < 64; ++k) fa.hT[hrow + (size_t)(64 * hf + k) * D + v] = H[k];
                return true;
            }
            publish_state(it, ok);   // the chain's first operand, with the scale of its first chunk
            if (!ok) return false;
            for (int c = 0; c < nch; ++c, ++it) {
                const int st = it & 1;
                const FcStage& B = S.st[st];
                // ---- Delta^T = U^T uinv - (W H)^T / sc, 32 tokens of this half -> A2 ----
                ok = fc_wait(&S.full[st], (uint32_t)((it >> 1) & 1), abort) && ok;
                ok = fc_wait(&S.d1, (uint32_t)(it & 1), abort) && ok;
                tc::tc_fence_after();
                const float gC = B.SC[SC_GC];
                {
                    float x[32];
                    tc::tmem_ld32(tD1 + lb + 32 * hf, x);
                    const float uinv = B.SC[SC_UINV];
                    // row v of U^T, tokens 32 hf .. 32 hf + 31: 16-byte chunks 4 hf .. 4 hf + 3 of
                    // the 128-byte row, at chunk ^ (v % 8) in the swizzled tile
                    const uint4* urow = reinterpret_cast<const uint4*>(B.U + v * 128);
                    uint4 u4[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) u4[q] = urow[(4 * hf + q) ^ (v & 7)];
                    tc::tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const __half2* e = reinterpret_cast<const __half2*>(&u4[q]);
#pragma unroll
                        for (int p2 = 0; p2 < 4; ++p2) {
                            const float2 uf = __half22float2(e[p2]);
                            const int j = q * 4 + p2;
                            const float d0 = uf.x * uinv - x[2 * j] * inv_sc;
                            const float d1 = uf.y * uinv - x[2 * j + 1] * inv_sc;
                            pk[j] = pack_h2u(d0 * sc, d1 * sc);
                        }
                    }
                    tc::tmem_st16(tA2 + lb + 16 * hf, pk);
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                }
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(&S.d_ready);
                    tc::mbar_arrive(&S.empty[st]);   // this warp has read the stage's U and scalars
                }
                // ---- the new state H = gamma_C H + (K_tilde^T Delta) from D2 columns 0-127 ----
                ok = fc_wait(&S.d2, (uint32_t)(it & 1), abort) && ok;
                tc::tc_fence_after();
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float y[32];
                    tc::tmem_ld32(tD2 + lb + 64 * hf + 32 * part, y);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) H[32 * part + j] = fmaf(gC, H[32 * part + j], y[j] * inv_sc);
                }
                if (c == nch - 1) {   // chain done: the final state (no further step of this chain)
                    // the step's one barrier, as in the other steps: every warp takes the same decision
                    if (tc::named_bar_any(2, 256, !ok || S.abort)) {
                        ok = false;
                        return false;
                    }
                    if (fa.hT)
#pragma unroll
                        for (int k = 0; k < 64; ++k) fa.hT[hrow + (size_t)(64 * hf + k) * D + v] = H[k];
                    continue;
                }
                publish_state(it + 1, ok);
                if (!ok) return false;
            }
            return true;
        });
        if (!ok) {
            record_timeout(fa.status);
            S.abort = 1;
        }
        return;
    }
    if (warp >= 12) {
        // ---------------- outputs: thread <-> value column v, all 64 tokens ------------------
        const int grp = warp & 3, v = grp * 32 + lane;
        const uint32_t lb = (uint32_t)(grp * 32) << 16;
        if (lane == 0) {   // the output columns of D1 and D2 are free before the first step
            tc::mbar_arrive(&S.ofree1);
            tc::mbar_arrive(&S.ofree2);
        }
        int it = 0;
        bool ok = true;
        for_each_chain(fa, [&](int, int h, int64_t bos, int64_t len, int, int nch) -> bool {
            for (int c = 0; c < nch; ++c, ++it) {
                const int st = it & 1;
                const FcStage& B = S.st[st];
                const int64_t tok0 = bos + (int64_t)C * c;
                const int64_t rem = len - (int64_t)C * c;
                const int cn = (int)(rem < C ? rem : C);
                ok = fc_wait(&S.full[st], (uint32_t)((it >> 1) & 1), abort) && ok;
                ok = fc_wait(&S.d1, (uint32_t)(it & 1), abort) && ok;
                tc::tc_fence_after();
                float q[64];
                tc::tmem_ld32(tD1 + lb + 64, q);
                tc::tmem_ld32(tD1 + lb + 96, q + 32);
                tc::tmem_wait_ld();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&S.ofree1);
                // (Q_hat H)^T * a: the row scalar a_t of each token, read now (the stage may go)
#pragma unroll
                for (int t = 0; t < 64; ++t) q[t] *= B.SC[t];
                const float inv = 1.f / S.scale[it & 3];
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&S.empty[st]);   // this warp has read the stage's scalars
                ok = fc_wait(&S.d2, (uint32_t)(it & 1), abort) && ok;
                tc::tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float pd[32];
                    tc::tmem_ld32(tD2 + lb + 128 + 32 * half, pd);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) q[32 * half + i] += pd[i];
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&S.ofree2);   // D2's output columns are read
                bf16* ocol = fa.o + (size_t)(tok0 * HV + h) * D + v;
#pragma unroll
                for (int t = 0; t < 64; ++t)
                    if (t < cn) ocol[(size_t)t * HV * D] = __float2bfloat16_rn(q[t] * inv);
                if (!ok || S.abort) return false;
            }
            return true;
        });
        if (!ok) {
            record_timeout(fa.status);
            S.abort = 1;
        }
    }
}

template <int G>
__global__ void __launch_bounds__(kFcThreads, 1)
prefill_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_kt,
                     const __grid_constant__ CUtensorMap tm_pt, const __grid_constant__ CUtensorMap tm_u,
                     const FusedArgs fa) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_failed;
    uint8_t* base = align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool carry = (int)blockIdx.x < fa.n_carry;
    // an earlier stage of the call (the cu_seqlens check) failed: write nothing (read once, so
    // that every thread of the CTA takes the same branch)
    if (tid == 0) s_failed = *reinterpret_cast<volatile int32_t*>(fa.status) != 0;
    if (warp == 0) {
        tc::tmem_alloc(&s_tmem, 512);
        tc::tmem_relinquish();
    }
    if (carry) {
        FcSmem& S = *reinterpret_cast<FcSmem*>(base);
        if (tid == 32) {
            for (int i = 0; i < 2; ++i) {
                tc::mbar_init(&S.full[i], 1);
                tc::mbar_init(&S.empty[i], 1 + 8 + 4);   // MMA commit, 8 state warps (U), 4 output warps (scalars)
            }
            tc::mbar_init(&S.d1, 1);
            tc::mbar_init(&S.d2, 1);
            tc::mbar_init(&S.h_ready, 8);
            tc::mbar_init(&S.d_ready, 8);
            tc::mbar_init(&S.ofree1, 4);
            tc::mbar_init(&S.ofree2, 4);
            for (int i = 0; i < 4; ++i) tc::mbar_init(&S.scal[i], 1);
            tc::fence_mbar_init();
            S.abort = 0;
            S.issued = 0;
        }
    } else if ((tid & 127) == 32) {
        PrepSmem& S = *reinterpret_cast<PrepSmem*>(base + (tid >> 7) * kPrepSlot);
        tc::mbar_init(&S.bar_load, 1);
        tc::mbar_init(&S.bar_v, 1);
        tc::mbar_init(&S.bar_mma, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = s_tmem;
    if (s_failed) {
    } else if (carry) {
        fused_carry<G>(*reinterpret_cast<FcSmem*>(base), &tm_w, &tm_qh, &tm_kt, &tm_pt, &tm_u, fa, tmem, tid);
    } else {
        // ---------------- chunk-local workers: four per CTA, items in chunk order ----------------
        const int wg = tid >> 7, wt = tid & 127;
        PrepSmem& S = *reinterpret_cast<PrepSmem*>(base + wg * kPrepSlot);
        const int worker = ((int)blockIdx.x - fa.n_carry) * 4 + wg;
        const int n_workers = ((int)gridDim.x - fa.n_carry) * 4;
        const int total = fa.chunk_off[fa.n_seqs] * fa.HK;
        PrepPhases ph;
        bool loaded = false;   // this item's K, Q copies were issued by the item before
        for (int item = worker; item < total; item += n_workers) {
            const bool failed = *reinterpret_cast<volatile int32_t*>(fa.status) != 0;
            if (tc::named_bar_any(1 + wg, 128, failed)) break;   // every thread of the worker agrees
            const int chunk = item / fa.HK, hk = item - chunk * fa.HK;
            int n, cn, nn, ncn, nhk = -1;
            int64_t s, ns = 0;
            if (!locate_chunk(chunk, fa.chunk_off, fa.cu, fa.T, fa.n_seqs, n, s, cn)) break;
            const int nitem = item + n_workers;
            if (nitem < total) {
                const int nchunk = nitem / fa.HK;
                if (locate_chunk(nchunk, fa.chunk_off, fa.cu, fa.T, fa.n_seqs, nn, ns, ncn)) nhk = nitem - nchunk * fa.HK;
            }
            const bool ok = prep_item<G, true>(S, &tm_q, &tm_k, &tm_v, fa.g, fa.beta, chunk, hk, s, cn, fa.HV, fa.HK,
                                               fa.scale, fa.l2norm, fa.out, fa.status,
                                               fa.stall && chunk == 0 && hk == 0, tmem + 128 * wg, wt, 1 + wg, ph,
                                               loaded, nhk, ns);
            loaded = nhk >= 0;
            if (!ok) {
                loaded = false;
                break;
            }
        }
        // copies issued for an item that will not run land before the CTA leaves
        if (loaded && wt == 0) (void)tc::mbar_wait(&S.bar_load, ph.load, 50000000ull);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (carry && tid == 0) {   // copies still in flight after an abort land before the CTA leaves:
        FcSmem& S = *reinterpret_cast<FcSmem*>(base);   // the latest step issued on each stage
        if (S.abort)
            for (int k = S.issued - 2; k < S.issued; ++k)
                if (k >= 0) (void)tc::mbar_wait(&S.full[k & 1], (uint32_t)((k >> 1) & 1), 50000000ull);
    }
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
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

// Workspace of the fused launch: per (chunk, value head) W, U, P^T, K_tilde and scalars, per
// (chunk, q/k head) Q_hat and a ready flag.
struct FusedLayout {
    int64_t max_chunks;
    size_t off_chunk, off_flags, off_w, off_u, off_p, off_kt, off_q, off_sc, total;
};

FusedLayout fused_layout(int64_t n_tokens, int n_seqs, int HK, int HV) {
    FusedLayout L;
    L.max_chunks = (n_tokens + C - 1) / C + n_seqs;
    const size_t rows = (size_t)L.max_chunks * HV * 64;
    L.off_chunk = kStatusBytes;
    L.off_flags = round_up(L.off_chunk + (size_t)(n_seqs + 1) * 4, 256);
    L.off_w = round_up(L.off_flags + (size_t)L.max_chunks * HK * 4, 1024);
    L.off_u = round_up(L.off_w + rows * D * 2, 1024);
    L.off_p = round_up(L.off_u + rows * D * 2, 1024);
    L.off_kt = round_up(L.off_p + rows * 64 * 2, 1024);
    L.off_q = round_up(L.off_kt + rows * D * 2, 1024);
    L.off_sc = round_up(L.off_q + (size_t)L.max_chunks * HK * 64 * D * 2, 1024);
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
    // one size for both launch forms (the fused one for the plain prefill, the two-kernel one
    // for the output epilogue and the context-parallel segment)
    const size_t a = tc_layout(n_tokens, n_seqs, HK, HV).total, b = fused_layout(n_tokens, n_seqs, HK, HV).total;
    return a > b ? a : b;
}

namespace {
int sm_count() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

// The plain prefill (no output epilogue, no transition run) as one cooperative launch.
cudaError_t launch_prefill_fused(const PrefillArgs& a, void* workspace, cudaStream_t s) {
    const bool packed = a.cu != nullptr;
    const int64_t n_tokens = packed ? a.T : (int64_t)a.n_seqs * a.T;
    const FusedLayout L = fused_layout(n_tokens, a.n_seqs, a.HK, a.HV);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* chunk_off = reinterpret_cast<int32_t*>(ws + L.off_chunk);
    int32_t* flags = reinterpret_cast<int32_t*>(ws + L.off_flags);
    f16* W = reinterpret_cast<f16*>(ws + L.off_w);
    f16* U = reinterpret_cast<f16*>(ws + L.off_u);
    f16* P = reinterpret_cast<f16*>(ws + L.off_p);
    f16* Kt = reinterpret_cast<f16*>(ws + L.off_kt);
    f16* Q = reinterpret_cast<f16*>(ws + L.off_q);
    float* SC = reinterpret_cast<float*>(ws + L.off_sc);

    chunk_table_kernel<<<1, 1024, 0, s>>>(a.cu, a.n_seqs, a.T, chunk_off, a.status, flags,
                                          (int64_t)L.max_chunks * a.HK);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();

    CUtensorMap tq, tk, tv, tw, tqh, tkt, tpt, tu;
    const cuuint64_t tok = (cuuint64_t)(n_tokens > 0 ? n_tokens : 1);
    {
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.HK, tok};
        cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.HK * D * 2};
        cuuint32_t box[3] = {64, 1, 64};
        const void* qb = a.q ? a.q : workspace;
        const void* kb = a.k ? a.k : workspace;
        if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qb, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kb, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
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
    {
        const cuuint64_t rows = mc * a.HV * 64;
        cuuint64_t dims[2] = {(cuuint64_t)D, rows};
        cuuint64_t str[1] = {(cuuint64_t)D * 2};
        cuuint32_t box[2] = {64, 64};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, W, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tkt, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Kt, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        // U^T: rows (chunk, value head) * 128 + value, 64 tokens each; one box is a whole tile
        cuuint64_t udims[2] = {64, rows * 2};
        cuuint64_t ustr[1] = {64 * 2};
        cuuint32_t ubox[2] = {64, 128};
        if (!make_map(&tu, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, U, 2, udims, ustr, ubox, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        cuuint64_t pdims[2] = {64, rows};
        cuuint64_t pstr[1] = {64 * 2};
        if (!make_map(&tpt, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, P, 2, pdims, pstr, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        cuuint64_t qdims[2] = {(cuuint64_t)D, mc * a.HK * 64};
        if (!make_map(&tqh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Q, 2, qdims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }

    const int sms = sm_count();
    if (sms < 2) return cudaErrorInvalidDevice;
    const int n_chains = a.n_seqs * a.HV;
    // carry CTAs: one per chain up to a quarter of the SMs (the chunk-local workers take the rest)
    int n_carry = n_chains < sms / 4 ? n_chains : sms / 4;
    if (n_carry < 1) n_carry = 1;
    FusedArgs fa;
    fa.g = a.g; fa.beta = a.beta; fa.cu = a.cu; fa.chunk_off = chunk_off; fa.T = a.T;
    fa.n_seqs = a.n_seqs; fa.HK = a.HK; fa.HV = a.HV; fa.scale = a.scale; fa.l2norm = a.l2norm;
    fa.out = PrepOut{W, U, P, Q, SC, Kt, flags};
    fa.h0 = a.h0; fa.hT = a.hT; fa.o = (bf16*)a.o; fa.status = a.status; fa.n_carry = n_carry;
    fa.stall = testing_stall_site() == GDN_STALL_PREFILL_PREP ? 1 : 0;

    auto launch = [&](auto kern) -> cudaError_t {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedSmemBytes);
        if (err != cudaSuccess) return err;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)sms);
        cfg.blockDim = dim3(kFcThreads);
        cfg.dynamicSmemBytes = kFusedSmemBytes;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident at once: carry and workers meet
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, tw, tqh, tkt, tpt, tu, fa);
    };
    const int G = a.HV / a.HK;
    e = G == 1 ? launch(prefill_fused_kernel<1>) : G == 2 ? launch(prefill_fused_kernel<2>)
                                                          : launch(prefill_fused_kernel<4>);
    if (e != cudaSuccess) return e;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    return cudaSuccess;
}
}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, void* workspace, cudaStream_t s) {
    if (!a.z && !a.o_tr) return launch_prefill_fused(a, workspace, s);
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

    chunk_table_kernel<<<1, 1024, 0, s>>>(a.cu, a.n_seqs, a.T, chunk_off, a.status, nullptr, 0);
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
            const PrepOut po{W, U, P, QK, SC, nullptr, nullptr};
            kern<<<grid, 128, kPrepSmemBytes, s>>>(tq, tk, tv, a.g, a.beta, a.cu, chunk_off, a.T, a.n_seqs, a.HV,
                                                   a.scale, a.l2norm, a.HK, po, a.status,
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
