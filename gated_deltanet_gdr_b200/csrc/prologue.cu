// prologue.cu -- the layer's pre-processing materialised as tensors.
//
// q_hat = q / sqrt(sum q^2 + eps), k_hat likewise (deltanet.rs l2norm, eps inside the
// square root; the transformers fallback normalises q and k with eps 1e-6),
// beta = sigmoid(b) and g = -exp(A_log[h]) * softplus(a + dt_bias[h]) (the beta and g
// lines of the transformers GatedDeltaNet forward).  One warp per row for the norms,
// one thread per element for beta and g.  The same arithmetic is fused into the load
// stage of the chunk and decode kernels; this kernel exists for callers that want the
// normalised tensors themselves.
#include "common.cuh"
#include "kernels.h"

namespace gdr {

template <typename T>
__global__ void l2norm_rows_kernel(const T *x, T *y, long long rows, int D, float eps) {
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const T *xr = x + row * D;
    float ss = 0.f;
    for (int i = lane; i < D; i += 32) {
        float f = to_f32(xr[i]);
        ss += f * f;
    }
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss + eps);
    T *yr = y + row * D;
    for (int i = lane; i < D; i += 32) yr[i] = from_f32<T>(to_f32(xr[i]) * inv);
}

template <typename T>
__global__ void beta_gate_kernel(const T *b, T *beta, const float *a, float *g, const float *A_log,
                                 const float *dt_bias, long long n, int Nv, int S) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    if (b) beta[i] = from_f32<T>(sigmoid_f32(to_f32(b[i])));
    if (a) {
        const int h = (int)((i / S) % Nv);
        g[i] = gate_from_raw(a[i], A_log[h], dt_bias[h]);
    }
}

template <typename T>
static cudaError_t launch_prologue_t(const void *q, const void *k, const void *b, const float *a,
                                     const float *A_log, const float *dt_bias, float eps, int B, int Nk, int Nv,
                                     int S, int Dk, void *q_hat, void *k_hat, void *beta, float *g,
                                     cudaStream_t stream) {
    const long long rows = (long long)B * Nk * S;
    const int wpb = 8;
    if (rows > 0) {
        const unsigned grid = (unsigned)((rows + wpb - 1) / wpb);
        if (q) l2norm_rows_kernel<T><<<grid, 32 * wpb, 0, stream>>>((const T *)q, (T *)q_hat, rows, Dk, eps);
        if (k) l2norm_rows_kernel<T><<<grid, 32 * wpb, 0, stream>>>((const T *)k, (T *)k_hat, rows, Dk, eps);
    }
    const long long n = (long long)B * Nv * S;
    if (n > 0 && (b || a)) {
        beta_gate_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, stream>>>((const T *)b, (T *)beta, a, g, A_log,
                                                                             dt_bias, n, Nv, S);
    }
    return cudaGetLastError();
}

cudaError_t launch_prologue(const void *q, const void *k, const void *b, const float *a, const float *A_log,
                            const float *dt_bias, float eps, int B, int Nk, int Nv, int S, int Dk, gdr_dtype dt,
                            void *q_hat, void *k_hat, void *beta, float *g, cudaStream_t stream) {
    if (dt == GDR_BF16)
        return launch_prologue_t<__nv_bfloat16>(q, k, b, a, A_log, dt_bias, eps, B, Nk, Nv, S, Dk, q_hat, k_hat,
                                                beta, g, stream);
    if (dt == GDR_F16)
        return launch_prologue_t<__half>(q, k, b, a, A_log, dt_bias, eps, B, Nk, Nv, S, Dk, q_hat, k_hat, beta, g,
                                         stream);
    return launch_prologue_t<float>(q, k, b, a, A_log, dt_bias, eps, B, Nk, Nv, S, Dk, q_hat, k_hat, beta, g,
                                    stream);
}

}  // namespace gdr
