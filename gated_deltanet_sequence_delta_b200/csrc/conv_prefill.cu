// conv_prefill.cu -- the causal depthwise convolution of kernel 4 that the "Gated DeltaNet
// ... Qwen3-next" page (section 3.1) places before the gated update (kernel size from the
// tutorial page, section 6, linear_conv_kernel_dim = 4), over whole sequences, dense or
// packed, with the rolling state of the three previous inputs carried in and out:
//   y_t = w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t   (per channel, then identity or SiLU)
// SiLU here uses the hardware exponential and reciprocal approximations (a few ulp); the
// fused decode step uses the full-precision functions: both far below the bf16 rounding of
// the outputs.
// The input is the raw q | k | v projection rows [tokens, C]; the output goes straight to the
// q, k, v tensors the chunked prefill reads.  HBM-bound: each input and output element
// crosses HBM once; the three previous inputs of a channel ride along in registers.
#include "gdn_internal.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace {

constexpr int CV = 8;         // channels per thread (16 bytes of bf16)
constexpr int RUN = 32;       // tokens per thread
constexpr int BATCH16 = 4;    // input rows per pipeline step (bf16; fp32: 2); the next step's
                              //   rows load meanwhile
constexpr int THREADS = 256;

struct Vec8 {
    float v[CV];
};

// eight channels as loaded (kept packed while in flight) and as floats
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
};
template <> struct Raw8<float> {
    float4 a, b;
};
__device__ __forceinline__ Raw8<__nv_bfloat16> load_raw(const __nv_bfloat16* p) {
    return {__ldg(reinterpret_cast<const uint4*>(p))};
}
__device__ __forceinline__ Raw8<float> load_raw(const float* p) {
    return {__ldg(reinterpret_cast<const float4*>(p)), __ldg(reinterpret_cast<const float4*>(p) + 1)};
}
__device__ __forceinline__ Vec8 unpack(const Raw8<__nv_bfloat16>& r) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.u);
    Vec8 o;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        o.v[2 * i] = f.x;
        o.v[2 * i + 1] = f.y;
    }
    return o;
}
__device__ __forceinline__ Vec8 unpack(const Raw8<float>& r) {
    Vec8 o;
    o.v[0] = r.a.x; o.v[1] = r.a.y; o.v[2] = r.a.z; o.v[3] = r.a.w;
    o.v[4] = r.b.x; o.v[5] = r.b.y; o.v[6] = r.b.z; o.v[7] = r.b.w;
    return o;
}
template <typename T>
__device__ __forceinline__ Vec8 load8(const T* p) { return unpack(load_raw(p)); }
__device__ __forceinline__ Vec8 load8_smem(const __nv_bfloat16* p) {
    return unpack(Raw8<__nv_bfloat16>{*reinterpret_cast<const uint4*>(p)});
}

// SiLU y * sigmoid(y) = y / (1 + 2^(-y log2 e)) from the hardware base-2 exponential and
// reciprocal approximations (PTX ex2.approx, rcp.approx: a few ulp of fp32, two special-function
// ops); y -> -inf gives 0 (the reciprocal of +inf), y -> +inf gives y
__device__ __forceinline__ float silu_fast(float y) {
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * y));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
    return y * r;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* y) {
    __align__(16) __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(h);
}
__device__ __forceinline__ void store8(float* p, const float* y) {
    reinterpret_cast<float4*>(p)[0] = make_float4(y[0], y[1], y[2], y[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(y[4], y[5], y[6], y[7]);
}

// One thread: channels c0 .. c0+7 for tokens t0 .. t0+RUN-1 of the packed token range.
// Sequence n holds tokens [cu[n], cu[n+1]) (dense: [n T, (n+1) T)).  A bad table gives
// undefined values, but every index below is clamped to its buffer.
template <typename T>
__global__ void __launch_bounds__(THREADS, 2) conv_prefill_kernel(
    const T* __restrict__ x, const float* __restrict__ w, const float* __restrict__ state_in,
    const int32_t* __restrict__ cu, int64_t n_tokens, int64_t Tlen, int n_seqs, int C, int qk, int act,
    T* __restrict__ q, T* __restrict__ k, T* __restrict__ v, float* __restrict__ state_out) {
    const int c0 = (blockIdx.y * THREADS + threadIdx.x) * CV;
    if (c0 >= C) return;
    auto seq_start = [&](int n) -> int64_t { return cu ? (int64_t)__ldg(cu + n) : (int64_t)n * Tlen; };

    // sequences of length zero: the state passes through unchanged
    if (blockIdx.x == 0 && state_out) {
        for (int n = 0; n < n_seqs; ++n) {
            if (seq_start(n + 1) != seq_start(n)) continue;
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const size_t off = ((size_t)n * 3 + i) * C + c0;
                float s[CV];
#pragma unroll
                for (int j = 0; j < CV; ++j) s[j] = state_in ? state_in[off + j] : 0.f;
                store8(state_out + off, s);
            }
        }
    }
    const int64_t t0 = (int64_t)blockIdx.x * RUN;
    if (t0 >= n_tokens) return;
    const int64_t t1 = t0 + RUN < n_tokens ? t0 + RUN : n_tokens;

    // the sequence holding t0: the last n with start <= t0
    int n = 0;
    if (cu) {
        int lo = 0, hi = n_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (seq_start(mid) <= t0) lo = mid;
            else hi = mid - 1;
        }
        n = lo;
    } else {
        n = (int)(t0 / Tlen);
        if (n > n_seqs - 1) n = n_seqs - 1;
    }
    int64_t s = seq_start(n), e = seq_start(n + 1);

    Vec8 wt[4];   // tap i of the 8 channels
    {
        const float4* wp = reinterpret_cast<const float4*>(w + (size_t)c0 * 4);
#pragma unroll
        for (int j = 0; j < CV; ++j) {
            const float4 t4 = __ldg(wp + j);
            wt[0].v[j] = t4.x;
            wt[1].v[j] = t4.y;
            wt[2].v[j] = t4.z;
            wt[3].v[j] = t4.w;
        }
    }
    // the window x_{t-3}, x_{t-2}, x_{t-1} of sequence n at token t: earlier tokens of the
    // sequence, else the carried state (tap 3 + r for r = position - start < 0)
    Vec8 win[3];
    auto fill_window = [&](int64_t t) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int64_t pos = t - 3 + i, r = pos - s;
            if (r >= 0 && pos >= 0 && pos < n_tokens) {
                win[i] = load8(x + pos * C + c0);
            } else {
                const int tap = (int)(r < -3 ? 0 : 3 + (r >= 0 ? -1 : r));
#pragma unroll
                for (int j = 0; j < CV; ++j)
                    win[i].v[j] = state_in ? state_in[((size_t)n * 3 + tap) * C + c0 + j] : 0.f;
            }
        }
    };
    fill_window(t0);

    T* dst;
    int64_t dstride;
    int dc;
    if (c0 < qk) {
        dst = q; dstride = qk; dc = c0;
    } else if (c0 < 2 * qk) {
        dst = k; dstride = qk; dc = c0 - qk;
    } else {
        dst = v; dstride = C - 2 * qk; dc = c0 - 2 * qk;
    }

    constexpr int BATCH = sizeof(T) == 2 ? BATCH16 : BATCH16 / 2;
    Raw8<T> xb[BATCH], xn[BATCH];   // this step's rows, the next step's (in flight)
#pragma unroll
    for (int b = 0; b < BATCH; ++b)
        if (t0 + b < t1) xb[b] = load_raw(x + (t0 + b) * C + c0);
    for (int64_t tb = t0; tb < t1; tb += BATCH) {
#pragma unroll
        for (int b = 0; b < BATCH; ++b)
            if (tb + BATCH + b < t1) xn[b] = load_raw(x + (tb + BATCH + b) * C + c0);
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int64_t t = tb + b;
            if (t >= t1) break;
            if (t >= e) {   // the next non-empty sequence starts here
                while (n < n_seqs - 1 && seq_start(n + 1) <= t) ++n;
                s = seq_start(n);
                e = seq_start(n + 1);
                fill_window(t);
            }
            const Vec8 xt = unpack(xb[b]);
            float y[CV];
#pragma unroll
            for (int j = 0; j < CV; ++j) {
                float a = wt[0].v[j] * win[0].v[j];
                a = fmaf(wt[1].v[j], win[1].v[j], a);
                a = fmaf(wt[2].v[j], win[2].v[j], a);
                a = fmaf(wt[3].v[j], xt.v[j], a);
                y[j] = act == 1 ? silu_fast(a) : a;
            }
            store8(dst + t * dstride + dc, y);
            win[0] = win[1];
            win[1] = win[2];
            win[2] = xt;
            if (t == e - 1 && state_out) {   // the sequence's last token: its three newest inputs
#pragma unroll
                for (int i = 0; i < 3; ++i) store8(state_out + ((size_t)n * 3 + i) * C + c0, win[i].v);
            }
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b) xb[b] = xn[b];
    }
}

// ---- bf16: a persistent kernel fed by TMA ----------------------------------------------
// Each CTA owns one block of TC channels (its weights stay in registers) and walks token
// tiles of TT: CTA b takes channel block b % n_cb and tiles b / n_cb, + per_cb, ...  A
// producer warp streams each tile's TT + 3 rows (three halo tokens before it, zero-filled
// before token 0) into a ring of NSTG shared-memory stages; eight consumer warps take
// TT / 8 tokens each, read their rows conflict-free (one 512-byte row per warp access) and
// store coalesced rows.
constexpr int TT = 64;                 // tokens per tile
constexpr int TC = 256;                // channels per tile: 32 lanes x 8
constexpr int TROWS = TT + 3;
constexpr int NSTG = 3;
constexpr int CWARPS = 8;              // consumer warps; warp 8 is the producer
constexpr int TPW = TT / CWARPS;       // tokens per consumer warp and tile
constexpr uint32_t kTileBytes = TROWS * TC * 2;

struct ConvSmem {
    __nv_bfloat16 tile[NSTG][TROWS * TC];
    uint64_t full[NSTG], empty[NSTG];
};
constexpr size_t kConvSmemBytes = sizeof(ConvSmem) + 128;

__device__ int32_t g_conv_error = 0;

__global__ void __launch_bounds__((CWARPS + 1) * 32, 2) conv_prefill_tma_kernel(
    const __grid_constant__ CUtensorMap tm_x, const float* __restrict__ w, const float* __restrict__ state_in,
    const int32_t* __restrict__ cu, int64_t n_tokens, int64_t Tlen, int n_seqs, int C, int qk, int act,
    __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v,
    float* __restrict__ state_out) {
    extern __shared__ uint8_t smem_raw[];
    ConvSmem& S = *reinterpret_cast<ConvSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t n_tt = (n_tokens + TT - 1) / TT;
    const int n_cb = (C + TC - 1) / TC;
    const int cb = (int)(blockIdx.x % n_cb);
    const int64_t per_cb = gridDim.x / n_cb;   // CTAs per channel block (the grid is a multiple of n_cb)
    const int64_t tt0 = blockIdx.x / n_cb;
    auto seq_start = [&](int n) -> int64_t { return cu ? (int64_t)__ldg(cu + n) : (int64_t)n * Tlen; };
    if (tid == 0) {
        for (int i = 0; i < NSTG; ++i) {
            tc::mbar_init(&S.full[i], 1);
            tc::mbar_init(&S.empty[i], CWARPS);
        }
        tc::fence_mbar_init();
    }
    __syncthreads();

    if (warp == CWARPS) {
        // ---------------- producer ----------------------------------------------------
        if (lane == 0) {
            int j = 0;
            for (int64_t tt = tt0; tt < n_tt; tt += per_cb, ++j) {
                const int st = j % NSTG, r = j / NSTG;
                if (r > 0 && !tc::mbar_wait(&S.empty[st], (uint32_t)((r - 1) & 1))) {
                    atomicExch(&g_conv_error, GDN_DEVERR_TIMEOUT);
                    break;
                }
                tc::mbar_expect_tx(&S.full[st], kTileBytes);
                tc::tma_load_2d(S.tile[st], &tm_x, &S.full[st], cb * TC, (int)(tt * TT) - 3);
            }
            // loads issued but not consumed (a consumer gave up) land before the CTA leaves
            for (int i = 0; i < NSTG && i < j; ++i) {
                const int jj = j - 1 - i, st = jj % NSTG;
                (void)tc::mbar_wait(&S.full[st], (uint32_t)((jj / NSTG) & 1), 50000000ull);
            }
        }
        return;
    }

    // sequences of length zero: the state passes through unchanged
    if (blockIdx.x == 0 && state_out) {
        for (int n = 0; n < n_seqs; ++n) {
            if (seq_start(n + 1) != seq_start(n)) continue;
            for (int cg = tid; cg < C / CV; cg += CWARPS * 32)
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const size_t off = ((size_t)n * 3 + i) * C + (size_t)cg * CV;
                    float sv[CV];
#pragma unroll
                    for (int jj = 0; jj < CV; ++jj) sv[jj] = state_in ? state_in[off + jj] : 0.f;
                    store8(state_out + off, sv);
                }
        }
    }

    // ---------------- consumers: warp w takes tokens TPW w .. TPW w + TPW - 1 of each tile ------
    const int c0 = cb * TC + lane * CV;
    Vec8 wt[4];   // tap i of this lane's 8 channels, for every tile of the CTA
    if (c0 < C) {
        const float4* wp = reinterpret_cast<const float4*>(w + (size_t)c0 * 4);
#pragma unroll
        for (int jj = 0; jj < CV; ++jj) {
            const float4 t4 = __ldg(wp + jj);
            wt[0].v[jj] = t4.x;
            wt[1].v[jj] = t4.y;
            wt[2].v[jj] = t4.z;
            wt[3].v[jj] = t4.w;
        }
    }
    int j = 0;
    for (int64_t tt = tt0; tt < n_tt; tt += per_cb, ++j) {
        const int st = j % NSTG, r = j / NSTG;
        const int64_t tf = tt * TT + (int64_t)warp * TPW;   // this warp's first token
        // the sequence bounds, before the wait for the tile
        int n = 0;
        int64_t s0 = 0, e0 = 0;
        const bool active = c0 < C && tf < n_tokens;
        if (active) {
            if (cu) {
                int lo = 0, hi = n_seqs - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (seq_start(mid) <= tf) lo = mid;
                    else hi = mid - 1;
                }
                n = lo;
            } else {
                n = (int)(tf / Tlen);
                if (n > n_seqs - 1) n = n_seqs - 1;
            }
            s0 = seq_start(n);
            e0 = seq_start(n + 1);
        }
        if (!tc::mbar_wait(&S.full[st], (uint32_t)(r & 1))) {
            if (lane == 0) atomicExch(&g_conv_error, GDN_DEVERR_TIMEOUT);
            break;
        }
        if (active) {
            const __nv_bfloat16* tile = S.tile[st] + lane * CV;   // row rr of the tile: + rr * TC
            const int64_t row0 = tt * TT - 3;                     // token of tile row 0
            Vec8 win[3];
            auto fill_window = [&](int64_t t) {
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int64_t pos = t - 3 + i, rel = pos - s0;
                    if (rel >= 0) {
                        win[i] = load8_smem(tile + (pos - row0) * TC);
                    } else {
                        const int tap = (int)(rel < -3 ? 0 : 3 + rel);
#pragma unroll
                        for (int jj = 0; jj < CV; ++jj)
                            win[i].v[jj] = state_in ? state_in[((size_t)n * 3 + tap) * C + c0 + jj] : 0.f;
                    }
                }
            };
            fill_window(tf);
            __nv_bfloat16* dst;
            int64_t dstride;
            int dc;
            if (c0 < qk) {
                dst = q; dstride = qk; dc = c0;
            } else if (c0 < 2 * qk) {
                dst = k; dstride = qk; dc = c0 - qk;
            } else {
                dst = v; dstride = C - 2 * qk; dc = c0 - 2 * qk;
            }
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
                const int64_t t = tf + i;
                if (t >= n_tokens) break;
                if (t >= e0) {   // the next non-empty sequence starts here
                    while (n < n_seqs - 1 && seq_start(n + 1) <= t) ++n;
                    s0 = seq_start(n);
                    e0 = seq_start(n + 1);
                    fill_window(t);
                }
                const Vec8 xt = load8_smem(tile + (t - row0) * TC);
                float y[CV];
#pragma unroll
                for (int jj = 0; jj < CV; ++jj) {
                    float a = wt[0].v[jj] * win[0].v[jj];
                    a = fmaf(wt[1].v[jj], win[1].v[jj], a);
                    a = fmaf(wt[2].v[jj], win[2].v[jj], a);
                    a = fmaf(wt[3].v[jj], xt.v[jj], a);
                    y[jj] = act == 1 ? silu_fast(a) : a;
                }
                store8(dst + t * dstride + dc, y);
                win[0] = win[1];
                win[1] = win[2];
                win[2] = xt;
                if (t == e0 - 1 && state_out) {
#pragma unroll
                    for (int ii = 0; ii < 3; ++ii) store8(state_out + ((size_t)n * 3 + ii) * C + c0, win[ii].v);
                }
            }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.empty[st]);   // this warp is done with the stage
    }
}

}  // namespace

cudaError_t read_conv_error(int32_t* out, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_conv_error, sizeof(int32_t));
    if (e == cudaSuccess && reset) {
        const int32_t zero = 0;
        e = cudaMemcpyToSymbol(g_conv_error, &zero, sizeof(int32_t));
    }
    return e;
}

cudaError_t launch_conv_prefill(const void* x, bool bf16, const float* w, const float* state_in,
                                const int32_t* cu, int64_t n_tokens, int64_t T, int n_seqs, int C, int qk,
                                int act, void* q, void* k, void* v, float* state_out, cudaStream_t s) {
    if (n_seqs == 0) return cudaSuccess;
    CUtensorMap tm;
    if (bf16 && n_tokens > 0 && n_tokens <= INT32_MAX - TT) {
        // x [n_tokens, C] bf16 in tiles of TC channels x (TT + 3) tokens
        const cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)n_tokens};
        const cuuint64_t str[1] = {(cuuint64_t)C * 2};
        const cuuint32_t box[2] = {TC, TROWS};
        if (make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE)) {
            cudaError_t e = cudaFuncSetAttribute(conv_prefill_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kConvSmemBytes);
            if (e != cudaSuccess) return e;
            int dev = 0, sms = 148;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            // whole multiples of the channel-block count, about two CTAs per SM in all
            const int64_t n_cb = (C + TC - 1) / TC, n_tt = (n_tokens + TT - 1) / TT;
            int64_t per_cb = 2 * (int64_t)sms / n_cb;
            if (per_cb < 1) per_cb = 1;
            if (per_cb > n_tt) per_cb = n_tt;
            const unsigned grid = (unsigned)(per_cb * n_cb);
            conv_prefill_tma_kernel<<<grid, (CWARPS + 1) * 32, kConvSmemBytes, s>>>(
                tm, w, state_in, cu, n_tokens, T, n_seqs, C, qk, act, (__nv_bfloat16*)q, (__nv_bfloat16*)k,
                (__nv_bfloat16*)v, state_out);
            e = cudaGetLastError();
            if (e == cudaSuccess) count_launch();
            return e;
        }
    }
    // x: runs of RUN tokens (at least one, for the state of empty sequences); y: channel blocks
    const int64_t runs = n_tokens > 0 ? (n_tokens + RUN - 1) / RUN : 1;
    const dim3 grid((unsigned)runs, (unsigned)((C / CV + THREADS - 1) / THREADS));
    if (bf16)
        conv_prefill_kernel<__nv_bfloat16><<<grid, THREADS, 0, s>>>(
            (const __nv_bfloat16*)x, w, state_in, cu, n_tokens, T, n_seqs, C, qk, act, (__nv_bfloat16*)q,
            (__nv_bfloat16*)k, (__nv_bfloat16*)v, state_out);
    else
        conv_prefill_kernel<float><<<grid, THREADS, 0, s>>>((const float*)x, w, state_in, cu, n_tokens, T, n_seqs,
                                                             C, qk, act, (float*)q, (float*)k, (float*)v,
                                                             state_out);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace gdn
