// gates.cu -- the gate computation ("Gated DeltaNet ... Qwen3-next" page, section 2.1):
//   beta = sigmoid(b),  g = -exp(A_log) * softplus(a + dt_bias).
// Elementwise and HBM-bound: 8 (or 4) bytes in and 8 bytes out per (token, value head).
#include "gdn_internal.cuh"

namespace gdn {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) gates_kernel(const T* __restrict__ a, const T* __restrict__ b,
                                                    const float* __restrict__ A_log,
                                                    const float* __restrict__ dt_bias,
                                                    int64_t n, int HV, float* __restrict__ g,
                                                    float* __restrict__ beta) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int h = (int)(i % HV);
        float gv, bv;
        gate_pair(load_elem(a, i), load_elem(b, i), __ldg(A_log + h), __ldg(dt_bias + h), gv, bv);
        g[i] = gv;
        beta[i] = bv;
    }
}

}  // namespace

cudaError_t launch_gates(const void* a, const void* b, bool ab_bf16, const float* A_log,
                         const float* dt_bias, int64_t n_tokens, int HV, float* g, float* beta,
                         cudaStream_t s) {
    const int64_t n = n_tokens * HV;
    if (n == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)sms * 8;
    if (blocks > cap) blocks = cap;
    if (ab_bf16)
        gates_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            (const __nv_bfloat16*)a, (const __nv_bfloat16*)b, A_log, dt_bias, n, HV, g, beta);
    else
        gates_kernel<float><<<(unsigned)blocks, 256, 0, s>>>((const float*)a, (const float*)b, A_log,
                                                             dt_bias, n, HV, g, beta);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace gdn
