// epilogue.cu -- the gated RMSNorm output epilogue as one pass over the stored out rows, for the paths that
// do not fuse it (decode, whose rows are few, and the CUDA-core prefill, whose CTAs each hold only a slab of
// a row).
//
// Per head and valid token, out row o (length Dv) becomes o / sqrt(mean_j o_j^2 + eps) * norm_w * silu(z)
// (the per-head gated RMSNorm of deltanet.rs and of its WGSL core shader), in fp32, written back in place.
#include "common.cuh"
#include "kernels.h"

namespace gdr {
namespace {

constexpr int kRowsPerBlock = 8;  // one warp per row

// silu(x) = x / (1 + e^{-x}); for very negative x the quotient goes to -0, as it should
__device__ __forceinline__ float silu_f32(float x) { return x / (1.f + __expf(-x)); }

template <typename T, int DV>
__global__ void __launch_bounds__(32 * kRowsPerBlock) gated_rmsnorm_kernel(T *out, const T *z, const float *w,
                                                                           float eps, const int32_t *lengths,
                                                                           int Nv, int S, long long rows) {
    constexpr int PER = DV >= 32 ? DV / 32 : 1;
    const long long r = (long long)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const int t = (int)(r % S);
    const int b = (int)(r / S / Nv);
    int L = lengths ? lengths[b] : S;
    if (L < 0 || L > S) L = 0;  // the main kernel skipped such a sequence and flagged it
    if (t >= L) return;         // padding rows stay zero
    T *o = out + r * DV;
    const T *zr = z + r * DV;
    float x[PER];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int j = i * 32 + lane;
        x[i] = j < DV ? to_f32(o[j]) : 0.f;
        ss = fmaf(x[i], x[i], ss);
    }
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss * (1.f / DV) + eps);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int j = i * 32 + lane;
        if (j < DV) o[j] = from_f32<T>(x[i] * inv * w[j] * silu_f32(to_f32(zr[j])));
    }
}

template <typename T>
cudaError_t launch_t(T *out, const T *z, const float *w, float eps, const int32_t *lengths, int B, int Nv, int S,
                     int Dv, cudaStream_t s) {
    const long long rows = (long long)B * Nv * S;
    if (rows == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
    const dim3 block(32 * kRowsPerBlock);
    switch (Dv) {
        case 16: gated_rmsnorm_kernel<T, 16><<<blocks, block, 0, s>>>(out, z, w, eps, lengths, Nv, S, rows); break;
        case 32: gated_rmsnorm_kernel<T, 32><<<blocks, block, 0, s>>>(out, z, w, eps, lengths, Nv, S, rows); break;
        case 64: gated_rmsnorm_kernel<T, 64><<<blocks, block, 0, s>>>(out, z, w, eps, lengths, Nv, S, rows); break;
        case 128: gated_rmsnorm_kernel<T, 128><<<blocks, block, 0, s>>>(out, z, w, eps, lengths, Nv, S, rows); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_rmsnorm(void *out, const void *z, const float *norm_w, float eps, const int32_t *lengths,
                                 int B, int Nv, int S, int Dv, gdr_dtype dt, cudaStream_t s) {
    if (dt == GDR_BF16)
        return launch_t(static_cast<__nv_bfloat16 *>(out), static_cast<const __nv_bfloat16 *>(z), norm_w, eps,
                        lengths, B, Nv, S, Dv, s);
    if (dt == GDR_F16)
        return launch_t(static_cast<__half *>(out), static_cast<const __half *>(z), norm_w, eps, lengths, B, Nv, S,
                        Dv, s);
    return launch_t(static_cast<float *>(out), static_cast<const float *>(z), norm_w, eps, lengths, B, Nv, S, Dv, s);
}

}  // namespace gdr
