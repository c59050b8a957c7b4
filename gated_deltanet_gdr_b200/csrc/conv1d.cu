// conv1d.cu -- the depthwise causal conv1d + SiLU over the fused q/k/v channels, the step before the rule
// (the layer's causal_conv1d_fn / causal_conv1d_update on the blog "gated-delta-net" page; the per-channel
// ring of the last K inputs of deltanet.rs).
//
// y[t, c] = silu(bias[c] + sum_j w[c, j] x[t - K + 1 + j, c]), the positions before 0 taken from the state
// (the last K inputs, newest last).  The output goes straight into the rule's q, k and v layouts.
//
// One thread owns V = 4 channels (one 8- or 16-byte access, always inside one head) and walks a
// tile of kTile time steps with the K taps and the window in registers; a warp's loads and stores at one
// time step are contiguous.  HBM-bound: per valid position it reads C inputs and writes C outputs.
#include "common.cuh"
#include "kernels.h"

namespace gdr {
namespace {

constexpr int kThreads = 128;
constexpr int kTile = 64;

constexpr int kBatch = 4;  // time steps whose inputs a thread loads before it computes any of them
// CTAs per SM the register budget is capped for: 6 (80 registers a thread) up to the layer's K = 4, 4 beyond
// (the taps and window then need more registers)
__host__ __device__ constexpr int min_blocks(int K) { return K <= 4 ? 6 : 4; }

// silu(x) = x / (1 + e^{-x}) with the fast division (relative error ~1e-6; for x < -88 the quotient is 0,
// where silu is below 1e-36)
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// V = 4 channels per thread (one 8-byte access for bf16, 16 bytes for fp32), loaded raw through the read-only
// path and unpacked to fp32
template <typename T> struct ConvV;
template <> struct ConvV<__nv_bfloat16> {
    static constexpr int V = 4;
    using Raw = uint2;
    static __device__ __forceinline__ Raw zero() { return make_uint2(0, 0); }
    static __device__ __forceinline__ void unpack(uint2 u, float (&x)[4]) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
        const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
        x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&x)[4]) {
        __nv_bfloat162 h[2] = {__floats2bfloat162_rn(x[0], x[1]), __floats2bfloat162_rn(x[2], x[3])};
        *reinterpret_cast<uint2 *>(p) = *reinterpret_cast<const uint2 *>(h);
    }
};
template <> struct ConvV<__half> {
    static constexpr int V = 4;
    using Raw = uint2;
    static __device__ __forceinline__ Raw zero() { return make_uint2(0, 0); }
    static __device__ __forceinline__ void unpack(uint2 u, float (&x)[4]) {
        const __half2 *h = reinterpret_cast<const __half2 *>(&u);
        const float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]);
        x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
    }
    static __device__ __forceinline__ void store(__half *p, const float (&x)[4]) {
        __half2 h[2] = {__floats2half2_rn(x[0], x[1]), __floats2half2_rn(x[2], x[3])};
        *reinterpret_cast<uint2 *>(p) = *reinterpret_cast<const uint2 *>(h);
    }
};
template <> struct ConvV<float> {
    static constexpr int V = 4;
    using Raw = uint4;
    static __device__ __forceinline__ Raw zero() { return make_uint4(0, 0, 0, 0); }
    static __device__ __forceinline__ void unpack(uint4 u, float (&x)[4]) {
        x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y); x[2] = __uint_as_float(u.z);
        x[3] = __uint_as_float(u.w);
    }
    static __device__ __forceinline__ void store(float *p, const float (&x)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

struct ConvK {
    const void *x, *w, *bias, *state_in;
    const int32_t *lengths;
    void *q, *k, *v, *state_out;
    int S, C, Nk, Nv, Dk, Dv;
    unsigned int *err;
};

// First element of channel group c0 of sequence b in q, k or v (time 0), and that tensor's row length
template <typename T>
__device__ __forceinline__ T *out_base(const ConvK &a, int b, int c0, int &row) {
    const int qk = a.Nk * a.Dk;
    if (c0 < qk) {
        row = a.Dk;
        return static_cast<T *>(a.q) + ((size_t)b * a.Nk + c0 / a.Dk) * a.S * a.Dk + c0 % a.Dk;
    }
    if (c0 < 2 * qk) {
        c0 -= qk;
        row = a.Dk;
        return static_cast<T *>(a.k) + ((size_t)b * a.Nk + c0 / a.Dk) * a.S * a.Dk + c0 % a.Dk;
    }
    c0 -= 2 * qk;
    row = a.Dv;
    return static_cast<T *>(a.v) + ((size_t)b * a.Nv + c0 / a.Dv) * a.S * a.Dv + c0 % a.Dv;
}

// length of sequence b, or -1 for one outside [0, S] (skipped and flagged)
__device__ __forceinline__ int seq_len(const ConvK &a, int b) {
    const int L = a.lengths ? a.lengths[b] : a.S;
    return (L < 0 || L > a.S) ? -1 : L;
}

// value of the history (state followed by x) at index i of sequence b, channel c: i < K from the state
template <typename T, int K>
__device__ __forceinline__ float hist_at(const ConvK &a, int b, int c, int i) {
    if (i < K) return a.state_in ? to_f32(static_cast<const T *>(a.state_in)[((size_t)b * a.C + c) * K + i]) : 0.f;
    return to_f32(static_cast<const T *>(a.x)[((size_t)b * a.S + (i - K)) * a.C + c]);
}

// the state after the sequence: the last K entries of the history, read completely before any is written
// (the output may alias the input state)
template <typename T, int K, int V>
__device__ __forceinline__ void write_state(const ConvK &a, int b, int c0, int L) {
    float nv[V][K];
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) nv[i][j] = hist_at<T, K>(a, b, c0 + i, L + j);
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j)
            static_cast<T *>(a.state_out)[((size_t)b * a.C + c0 + i) * K + j] = from_f32<T>(nv[i][j]);
}

template <typename T, int K>
__global__ void __launch_bounds__(kThreads, min_blocks(K)) conv1d_kernel(const ConvK a, int state_here) {
    constexpr int V = ConvV<T>::V;
    const int b = blockIdx.z;
    const int c0 = (blockIdx.x * kThreads + threadIdx.x) * V;
    if (c0 >= a.C) return;
    const int t0 = blockIdx.y * kTile, t1 = min(t0 + kTile, a.S);
    const int Lr = seq_len(a, b);
    if (Lr < 0 && c0 == 0 && blockIdx.y == 0) raise_device_error(a.err, GDR_DEVERR_LENGTH);
    const int L = Lr < 0 ? 0 : Lr;
    int row;
    T *op = out_base<T>(a, b, c0, row);

    // taps, bias and the window as channel pairs (f32x2 arithmetic)
    constexpr int V2 = V / 2;
    f2_t w2[K][V2], b2[V2];
#pragma unroll
    for (int p = 0; p < V2; ++p) {
        const T *b_ = static_cast<const T *>(a.bias);
        b2[p] = pk2(b_ ? to_f32(b_[c0 + 2 * p]) : 0.f, b_ ? to_f32(b_[c0 + 2 * p + 1]) : 0.f);
#pragma unroll
        for (int j = 0; j < K; ++j)
            w2[j][p] = pk2(to_f32(static_cast<const T *>(a.w)[(size_t)(c0 + 2 * p) * K + j]),
                           to_f32(static_cast<const T *>(a.w)[(size_t)(c0 + 2 * p + 1) * K + j]));
    }
    // window: win[j] holds position t - K + 1 + j for the step at t; the K - 1 positions before the tile
    f2_t win[K][V2];
#pragma unroll
    for (int j = 0; j < K - 1; ++j)
#pragma unroll
        for (int p = 0; p < V2; ++p)  // history index = position + K
            win[j][p] = t0 < L ? pk2(hist_at<T, K>(a, b, c0 + 2 * p, t0 + 1 + j),
                                     hist_at<T, K>(a, b, c0 + 2 * p + 1, t0 + 1 + j))
                               : pk2(0.f, 0.f);

    using Raw = typename ConvV<T>::Raw;
    const unsigned xstep = (unsigned)((size_t)a.C * sizeof(T) / sizeof(Raw));  // one time step, in access units
    const Raw *xq = reinterpret_cast<const Raw *>(static_cast<const T *>(a.x) + ((size_t)b * a.S + t0) * a.C + c0);
    T *oq = op + (size_t)t0 * row;
    const int nv = min(t1, L) - t0;  // valid steps of this tile (may be <= 0)
    const int nt = t1 - t0;          // steps of this tile
    // (unrolling the whole tile, so that the window shifts become register renames, measured slower: the
    // batch loop stays rolled)
#pragma unroll 1
    for (int tb = 0; tb < kTile; tb += kBatch) {
        if (tb >= nt) break;
        // the batch's inputs first (read-only path, so they need not wait for this thread's earlier stores)
        Raw raw[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) raw[u] = tb + u < nv ? __ldg(xq + u * xstep) : ConvV<T>::zero();
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (tb + u >= nt) break;
            float y[V];
            if (tb + u < nv) {
                float x[V];
                ConvV<T>::unpack(raw[u], x);
#pragma unroll
                for (int p = 0; p < V2; ++p) win[K - 1][p] = pk2(x[2 * p], x[2 * p + 1]);
#pragma unroll
                for (int p = 0; p < V2; ++p) {
                    f2_t acc = b2[p];
#pragma unroll
                    for (int j = 0; j < K; ++j) acc = fma2(w2[j][p], win[j][p], acc);
                    up2(acc, y[2 * p], y[2 * p + 1]);
                }
#pragma unroll
                for (int i = 0; i < V; ++i) y[i] = silu_fast(y[i]);
#pragma unroll
                for (int j = 0; j < K - 1; ++j)
#pragma unroll
                    for (int p = 0; p < V2; ++p) win[j][p] = win[j + 1][p];
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) y[i] = 0.f;
            }
            ConvV<T>::store(oq + u * row, y);
        }
        xq += kBatch * xstep;
        oq += kBatch * row;
    }
    if (state_here && a.state_out && Lr >= 0) write_state<T, K, V>(a, b, c0, L);
}

// the state after the sequence, for launches with several time tiles (whose first tile reads the input
// state, which the output state may alias): one thread per channel group, after the conv kernel
template <typename T, int K>
__global__ void __launch_bounds__(kThreads) conv1d_state_kernel(const ConvK a) {
    constexpr int V = ConvV<T>::V;
    const int b = blockIdx.z;
    const int c0 = (blockIdx.x * kThreads + threadIdx.x) * V;
    if (c0 >= a.C) return;
    const int L = seq_len(a, b);
    if (L >= 0) write_state<T, K, V>(a, b, c0, L);
}

template <typename T, int K>
cudaError_t launch_tk(const ConvK &a, int B, cudaStream_t s) {
    constexpr int V = ConvV<T>::V;
    const unsigned gx = (unsigned)((a.C / V + kThreads - 1) / kThreads);
    const unsigned gy = (unsigned)((a.S + kTile - 1) / kTile);
    if (gy > 0) {
        conv1d_kernel<T, K><<<dim3(gx, gy, B), kThreads, 0, s>>>(a, gy == 1);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.state_out && gy != 1) conv1d_state_kernel<T, K><<<dim3(gx, 1, B), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const ConvK &a, int B, int K, cudaStream_t s) {
    switch (K) {
        case 1: return launch_tk<T, 1>(a, B, s);
        case 2: return launch_tk<T, 2>(a, B, s);
        case 3: return launch_tk<T, 3>(a, B, s);
        case 4: return launch_tk<T, 4>(a, B, s);
        case 5: return launch_tk<T, 5>(a, B, s);
        case 6: return launch_tk<T, 6>(a, B, s);
        case 7: return launch_tk<T, 7>(a, B, s);
        case 8: return launch_tk<T, 8>(a, B, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_conv1d(const void *x, const void *weight, const void *bias, const void *state_in,
                          const int32_t *lengths, int B, int S, int Nk, int Nv, int Dk, int Dv, int K, gdr_dtype dt,
                          void *q, void *k, void *v, void *state_out, unsigned int *err, cudaStream_t s) {
    ConvK a{};
    a.x = x; a.w = weight; a.bias = bias; a.state_in = state_in; a.lengths = lengths;
    a.q = q; a.k = k; a.v = v; a.state_out = state_out;
    a.S = S; a.C = 2 * Nk * Dk + Nv * Dv; a.Nk = Nk; a.Nv = Nv; a.Dk = Dk; a.Dv = Dv; a.err = err;
    if (B == 0) return cudaSuccess;
    if (dt == GDR_BF16) return launch_t<__nv_bfloat16>(a, B, K, s);
    if (dt == GDR_F16) return launch_t<__half>(a, B, K, s);
    return launch_t<float>(a, B, K, s);
}

}  // namespace gdr
