// gdn_internal.cuh -- private declarations shared by the library's .cu files.
#pragma once

#include <cuda_bf16.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// ---- element access ------------------------------------------------------
__device__ __forceinline__ float load_elem(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float* p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// softplus(x) = log(1 + e^x) in the overflow-free form max(x,0) + log1p(e^{-|x|}).
__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

// The gates ("Gated DeltaNet ... Qwen3-next" page, section 2.1) of one (token, value head):
// g = -exp(A_log) * softplus(a + dt_bias), beta = sigmoid(b).  Every kernel that forms
// gates calls this, so a fused gate prologue is bit-identical to gdn_gates.
__device__ __forceinline__ void gate_pair(float a, float b, float A_log, float dt_bias, float& g, float& beta) {
    g = -expf(A_log) * softplus_f(a + dt_bias);
    beta = 1.0f / (1.0f + expf(-b));
}

// L2-normalisation factor 1 / sqrt(sum x^2 + 1e-6) (flag off: 1).
__device__ __forceinline__ float l2_inv(float sumsq, int enabled) {
    return enabled ? 1.0f / sqrtf(sumsq + 1e-6f) : 1.0f;
}

// Launch accounting: every launcher calls count_launch() after a successful launch.
void count_launch(int n = 1);

// The site gdn_testing_stall selected (GDN_STALL_NONE normally); launchers read it on the
// host and pass the kernels a flag.
int testing_stall_site();

// Workspace layout: [0, 256) status words; then kernel-specific scratch.
constexpr size_t kStatusBytes = 256;

// ---- launchers (return cudaError_t of the launch) -------------------------
cudaError_t launch_gates(const void* a, const void* b, bool ab_bf16, const float* A_log,
                         const float* dt_bias, int64_t n_tokens, int HV, float* g, float* beta,
                         cudaStream_t s);

// Where a kernel takes its gates from: g, beta [rows, HV] as given, or (g == nullptr) formed
// in the kernel from a, b [rows, HV] (bf16 or fp32) and A_log, dt_bias [HV] (rows are the
// decode step's sequences or the prefill's tokens).
struct DecodeGates {
    const float* g;
    const float* beta;
    const void* a;
    const void* b;
    bool ab_bf16;
    const float* A_log;
    const float* dt_bias;
};
__device__ __forceinline__ void decode_gates(const DecodeGates& G, int64_t bh, int h, float& g, float& beta) {
    if (G.g) {
        g = G.g[bh];
        beta = G.beta[bh];
    } else if (G.ab_bf16) {
        gate_pair(load_elem((const __nv_bfloat16*)G.a, bh), load_elem((const __nv_bfloat16*)G.b, bh), G.A_log[h],
                  G.dt_bias[h], g, beta);
    } else {
        gate_pair(((const float*)G.a)[bh], ((const float*)G.b)[bh], G.A_log[h], G.dt_bias[h], g, beta);
    }
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, bool bf16, const DecodeGates& gates,
                          float* state, int B, int HK, int HV, int Dk, int Dv, float scale, int l2norm, void* o,
                          cudaStream_t s);

// The convolution prologue of a decode step: q, k, v are formed in the kernel from the raw
// projections x = [q | k | v] per sequence (C = 2 HK Dk + HV Dv channels) by a causal
// depthwise convolution of kernel 4, taps oldest first, over the three previous inputs
// held in state_in and the current one; state_out receives the three newest inputs.  The
// states are tap-major, [B, 3, C], so that a warp's channels are contiguous.
struct DecodeConv {
    const void* x;            // [B, C] io dtype
    const float* w;           // [C, 4]
    const float* state_in;    // [B, 3, C]
    float* state_out;         // [B, 3, C]
    int act;                  // 0 identity, 1 SiLU
};
// The output epilogue of a decode step: out = o rsqrt(mean(o^2) + eps) (1 + w) sigmoid(z) over
// each (sequence, value head) row of Dv values, before the store (z == nullptr: none).
struct DecodeOutGate {
    const void* z;            // [B, HV, Dv] io dtype
    const float* w;           // [Dv]
    float eps;
};
// Dk = Dv = 128 only.
cudaError_t launch_decode_conv(bool bf16, const DecodeConv& conv, const DecodeGates& gates, float* state, int B,
                               int HK, int HV, float scale, int l2norm, void* o, const DecodeOutGate& og,
                               cudaStream_t s);

// Tiled tensor map (element strides 1, no interleave, zero fill out of range); false if the
// driver entry point is missing or the encoder rejects the arguments.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw);

// Causal depthwise convolution of kernel 4 over whole sequences (dense when cu is null:
// n_seqs sequences of T tokens): x [n_tokens, C] with C = 2 qk + (v channels), written to
// q, k [n_tokens, qk] and v [n_tokens, C - 2 qk]; states [n_seqs, 3, C] fp32 tap-major.
cudaError_t launch_conv_prefill(const void* x, bool bf16, const float* w, const float* state_in,
                                const int32_t* cu, int64_t n_tokens, int64_t T, int n_seqs, int C, int qk,
                                int act, void* q, void* k, void* v, float* state_out, cudaStream_t s);

// Context-parallel prefill, the exchange step: A_all, B_all [R, n_seqs, HV, 128, 128] (every
// segment's transition and zero-start final state), h0 the sequence's initial states (may be
// null); writes this rank's start states, the sequences' final states (may be null) and adds
// H_start^T c_t to o in place (o, c [n_seqs, T_seg, HV, 128]).
cudaError_t launch_cp_combine(const float* A_all, const float* B_all, const float* h0, int R, int rank, int n_seqs,
                              int64_t T_seg, int HV, bool bf16, void* o, const void* c, float* start_state,
                              float* final_state, cudaStream_t s);

// Read (and on request clear) the device word the tensor-core correction of gdn_cp_combine sets
// on a timeout.
cudaError_t read_cp_error(int32_t* out, bool reset);

// Read (and on request clear) the device word the bf16 convolution kernel sets on a timeout.
cudaError_t read_conv_error(int32_t* out, bool reset);

// Read (and on request clear) the device word a staged decode launch sets on a timeout.
cudaError_t read_decode_error(int32_t* out, bool reset);

struct PrefillArgs {
    const void* q;
    const void* k;
    const void* v;
    bool bf16;
    const float* g;           // [tokens, HV], or null: gates formed in the kernel from `gates`
    const float* beta;
    DecodeGates gates;        // the gate source (g, beta as above, or raw a, b with A_log, dt_bias)
    const float* h0;          // may be null
    const int32_t* cu;        // may be null (dense)
    int64_t T;                // tokens per sequence (dense) or total (packed)
    int n_seqs, HK, HV, Dk, Dv, BT;
    float scale;
    int l2norm;
    void* o;
    float* hT;                // may be null
    const void* z;            // output epilogue gate inputs [.., HV, Dv] io dtype, or null (none)
    const float* norm_w;      // output epilogue norm weights [Dv] (with z)
    float eps;                // output epilogue norm epsilon (with z)
    void* o_tr;               // with hT_tr: the transition run's outputs (v = 0 from the identity;
    float* hT_tr;             //   tensor-core path only), or null
    int32_t* status;          // device status word (workspace)
    void* scratch;            // workspace after the status words
    size_t scratch_bytes;
};

// The size checks of gdn_chunk_prefill (GDN_OK, GDN_ERR_SHAPE or GDN_ERR_UNSUPPORTED), shared
// by every prefill entry point so that they reject the same sizes with the same status.
gdn_status prefill_check_sizes(gdn_dtype io_dtype, bool packed, int32_t B, int64_t T, int32_t n_seqs, int32_t HK,
                               int32_t HV, int32_t Dk, int32_t Dv, int32_t BT);

cudaError_t launch_check_cu_seqlens(const int32_t* cu, int n_seqs, int64_t T, int32_t* status,
                                    cudaStream_t s);
cudaError_t launch_prefill_cudacore(const PrefillArgs& a, cudaStream_t s);

// Tensor-core (tcgen05) prefill: bf16, Dk = Dv = 128, BT = 64, HV / HK in {1, 2, 4}.
bool prefill_tc_supported(int Dk, int Dv, int HK, int HV, int BT);
size_t prefill_tc_workspace_bytes(int64_t n_tokens, int n_seqs, int HK, int HV);
cudaError_t launch_prefill_tc(const PrefillArgs& a, void* workspace, cudaStream_t s);

}  // namespace gdn
