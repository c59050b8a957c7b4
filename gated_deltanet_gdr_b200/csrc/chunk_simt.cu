// chunk_simt.cu -- chunked prefill of the gated delta rule on the CUDA cores, in fp32.
//
// This is the path for fp32 inputs (whose 1e-4 max-abs parity a bf16 tensor-core
// product cannot meet) and for head sizes the tensor-core kernel is not built for.
// It follows the chunked (WY / UT transform) form of torch_chunk_gated_delta_rule
// (blog "gated-delta-net" page, steps 1-8), chunk C = 64, per CTA one
// (b, value head h, slab of VC state columns) -- state columns evolve independently,
// so slabs need no communication:
//   a1  G_t = cumulative log-gate inside the chunk (tokens past the length count 0)
//   a2  A[t][s] = beta_t (k_t . k_s) exp(G_t - G_s) for s < t;
//       P[t][s] = (x_t . k_s) exp(G_t - G_s) for s <= t, x = scale * q
//   a3+a4  W = (I + A)^{-1} diag(beta e^G) K and U = (I + A)^{-1} diag(beta) V by forward
//       substitution (one column per thread, no barrier inside the solve)
//   a5  v_new = U - W S;  o = diag(e^G) X S + P v_new;  S = e^{G_last} S + (e^{G_last - G} K)^T v_new
//   a6  out rows t >= L are zero; the slab of the final state is written once.
// Everything is staged in shared memory as fp32 (rows padded by one word against bank
// conflicts); HBM sees each input once and each output once.
#include "common.cuh"
#include "kernels.h"

namespace gdr {

template <int DK, int VC> struct SimtLayout {
    static constexpr int C = kChunk;
    static constexpr int KP = DK + 1, VP = VC + 1, CP = C + 1;
    static constexpr int oK = 0;
    static constexpr int oQ = oK + C * KP;
    static constexpr int oW = oQ + C * KP;
    static constexpr int oU = oW + C * KP;
    static constexpr int oS = oU + C * VP;
    static constexpr int oA = oS + DK * VP;
    static constexpr int oP = oA + C * CP;
    static constexpr int oVec = oP + C * CP;      // beta, G, e^G, e^{G_last - G}
    static constexpr int floats = oVec + 4 * C;
    static constexpr size_t bytes = (size_t)floats * sizeof(float);
};

template <int DK, int VC, typename TI>
__global__ void __launch_bounds__(256, 1) chunk_simt_kernel(const ChunkArgs a, const int DV) {
    using Ly = SimtLayout<DK, VC>;
    constexpr int C = Ly::C, KP = Ly::KP, VP = Ly::VP, CP = Ly::CP, NT = 256;
    extern __shared__ float sm[];
    float *sK = sm + Ly::oK, *sQ = sm + Ly::oQ, *sW = sm + Ly::oW, *sU = sm + Ly::oU;
    float *sS = sm + Ly::oS, *sA = sm + Ly::oA, *sP = sm + Ly::oP;
    float *sBeta = sm + Ly::oVec, *sG = sBeta + C, *sEG = sG + C, *sTail = sEG + C;

    const int nsplit = DV / VC;
    const int split = blockIdx.x % nsplit;
    const int bh = blockIdx.x / nsplit;
    const int h = bh % a.Nv, b = bh / a.Nv, kh = h / (a.Nv / a.Nk);
    const int S = a.S, col0 = split * VC;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    int L = a.lengths ? a.lengths[b] : S;
    if (L < 0 || L > S) {
        if (tid == 0) raise_device_error(a.err, GDR_DEVERR_LENGTH);
        L = 0;  // skipped: zero output, final state = initial state
    }
    const TI *qg = reinterpret_cast<const TI *>(a.q) + (((size_t)b * a.Nk + kh) * S) * DK;
    const TI *kg = reinterpret_cast<const TI *>(a.k) + (((size_t)b * a.Nk + kh) * S) * DK;
    const TI *vg = reinterpret_cast<const TI *>(a.v) + ((size_t)bh * S) * DV + col0;
    const TI *bg = reinterpret_cast<const TI *>(a.beta) + (size_t)bh * S;
    const float *gg = a.g ? a.g + (size_t)bh * S : nullptr;
    TI *og = reinterpret_cast<TI *>(a.out) + ((size_t)bh * S) * DV + col0;
    const size_t st_off = (size_t)bh * DK * DV + col0;

    // initial state slab
    for (int e = tid; e < DK * VC; e += NT) {
        int i = e / VC, j = e % VC;
        sS[i * VP + j] = a.initial_state ? to_f32(reinterpret_cast<const TI *>(a.initial_state)[st_off + (size_t)i * DV + j]) : 0.f;
    }
    // padding rows
    for (size_t e = tid; e < (size_t)(S - L) * VC; e += NT) og[(size_t)(L + e / VC) * DV + e % VC] = from_f32<TI>(0.f);

    const float gA = (a.A_log && a.g) ? a.A_log[h] : 0.f, gB = (a.A_log && a.g) ? a.dt_bias[h] : 0.f;
    for (int t0 = 0; t0 < L; t0 += C) {
        const int n = min(C, L - t0);  // valid tokens in this chunk
        __syncthreads();
        // ---- stage K, Q (normalised, scaled), V slab, beta, gate ----
        for (int r = warp; r < C; r += NT / 32) {
            float ks = 0.f, qs = 0.f;
            for (int i = lane; i < DK; i += 32) {
                float xk = 0.f, xq = 0.f;
                if (r < n) {
                    xk = to_f32(kg[(size_t)(t0 + r) * DK + i]);
                    xq = to_f32(qg[(size_t)(t0 + r) * DK + i]);
                }
                sK[r * KP + i] = xk;
                sQ[r * KP + i] = xq;
                ks += xk * xk;
                qs += xq * xq;
            }
            float kn = 1.f, qn = a.scale;
            if (a.l2norm) {
                ks = warp_sum(ks);
                qs = warp_sum(qs);
                kn = rsqrtf(ks + a.eps);
                qn = a.scale * rsqrtf(qs + a.eps);
            }
            for (int i = lane; i < DK; i += 32) {
                sK[r * KP + i] *= kn;
                sQ[r * KP + i] *= qn;
            }
            if (lane == 0) {
                float bt = 0.f, gt = 0.f;
                if (r < n) {
                    bt = to_f32(bg[t0 + r]);
                    if (a.beta_logits) bt = sigmoid_f32(bt);
                    if (gg) gt = a.A_log ? gate_from_raw(gg[t0 + r], gA, gB) : gg[t0 + r];
                }
                sBeta[r] = bt;
                sG[r] = gt;
            }
        }
        for (int e = tid; e < C * VC; e += NT) {
            int r = e / VC, j = e % VC;
            sU[r * VP + j] = r < n ? to_f32(vg[(size_t)(t0 + r) * DV + j]) : 0.f;
        }
        __syncthreads();
        if (tid == 0) {  // a1: cumulative gate
            float acc = 0.f;
            for (int r = 0; r < C; ++r) {
                acc += sG[r];
                sG[r] = acc;
            }
        }
        __syncthreads();
        if (tid < C) {
            sEG[tid] = expf(sG[tid]);
            sTail[tid] = expf(sG[C - 1] - sG[tid]);
        }
        // ---- a2: A (strict lower) and P (lower incl. diagonal) ----
        for (int e = tid; e < C * C; e += NT) {
            int t = e / C, s = e % C;
            float av = 0.f, pv = 0.f;
            if (s <= t) {
                float dk = 0.f, dq = 0.f;
                const float *kt = sK + t * KP, *ks = sK + s * KP, *qt = sQ + t * KP;
#pragma unroll 8
                for (int i = 0; i < DK; ++i) {
                    dk = fmaf(kt[i], ks[i], dk);
                    dq = fmaf(qt[i], ks[i], dq);
                }
                float dec = expf(sG[t] - sG[s]);
                pv = dq * dec;
                if (s < t) av = sBeta[t] * dk * dec;
            }
            sA[t * CP + s] = av;
            sP[t * CP + s] = pv;
        }
        __syncthreads();
        // ---- a3/a4: forward substitution, W (DK columns) and U (VC columns) in place ----
        if (tid < DK + VC) {
            const bool isW = tid < DK;
            const int c = isW ? tid : tid - DK;
            float *X = isW ? sW : sU;
            const int XP = isW ? KP : VP;
            for (int t = 0; t < C; ++t) {
                float rhs = isW ? sBeta[t] * sEG[t] * sK[t * KP + c] : sBeta[t] * sU[t * VP + c];
                const float *arow = sA + t * CP;
                for (int s = 0; s < t; ++s) rhs = fmaf(-arow[s], X[s * XP + c], rhs);
                X[t * XP + c] = rhs;
            }
        }
        __syncthreads();
        // ---- a5: v_new = U - W S (in place in sU) ----
        for (int e = tid; e < C * VC; e += NT) {
            int t = e / VC, j = e % VC;
            float acc = sU[t * VP + j];
            const float *wt = sW + t * KP;
#pragma unroll 8
            for (int i = 0; i < DK; ++i) acc = fmaf(-wt[i], sS[i * VP + j], acc);
            sU[t * VP + j] = acc;
        }
        __syncthreads();
        // ---- a5: o = diag(e^G) X S + P v_new ----
        for (int e = tid; e < C * VC; e += NT) {
            int t = e / VC, j = e % VC;
            if (t >= n) continue;
            float acc = 0.f;
            const float *qt = sQ + t * KP;
#pragma unroll 8
            for (int i = 0; i < DK; ++i) acc = fmaf(qt[i], sS[i * VP + j], acc);
            acc *= sEG[t];
            const float *pt = sP + t * CP;
            for (int s = 0; s <= t; ++s) acc = fmaf(pt[s], sU[s * VP + j], acc);
            og[(size_t)(t0 + t) * DV + j] = from_f32<TI>(acc);
        }
        __syncthreads();
        // ---- a5: S = e^{G_last} S + (e^{G_last - G} K)^T v_new ----
        const float eL = sEG[C - 1];
        for (int e = tid; e < DK * VC; e += NT) {
            int i = e / VC, j = e % VC;
            float acc = eL * sS[i * VP + j];
            for (int t = 0; t < C; ++t) acc = fmaf(sTail[t] * sK[t * KP + i], sU[t * VP + j], acc);
            sS[i * VP + j] = acc;
        }
    }
    __syncthreads();
    if (a.final_state) {
        TI *fs = reinterpret_cast<TI *>(a.final_state) + st_off;
        for (int e = tid; e < DK * VC; e += NT) {
            int i = e / VC, j = e % VC;
            fs[(size_t)i * DV + j] = from_f32<TI>(sS[i * VP + j]);
        }
    }
}

template <int DK, int VC, typename TI>
static cudaError_t launch_simt_t(const ChunkArgs &a, int DV, cudaStream_t stream) {
    using Ly = SimtLayout<DK, VC>;
    const long long blocks = (long long)a.B * a.Nv * (DV / VC);
    if (blocks == 0) return cudaSuccess;
    auto kern = chunk_simt_kernel<DK, VC, TI>;
    static LaunchCache cache(reinterpret_cast<const void *>(kern));
    cudaError_t e = cache.allow_smem((int)Ly::bytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)blocks, 256, Ly::bytes, stream>>>(a, DV);
    return cudaGetLastError();
}

template <int DK, typename TI>
static cudaError_t launch_simt_k(const ChunkArgs &a, int DV, cudaStream_t s) {
    switch (DV) {
        case 16: return launch_simt_t<DK, 16, TI>(a, DV, s);
        case 32: return launch_simt_t<DK, 32, TI>(a, DV, s);
        default: return launch_simt_t<DK, 64, TI>(a, DV, s);  // 64 and 128: slabs of 64 columns
    }
}

cudaError_t launch_chunk_simt(const ChunkArgs &a, int Dk, int Dv, gdr_dtype dt, cudaStream_t s) {
    if (dt == GDR_F16) {
        switch (Dk) {
            case 16: return launch_simt_k<16, __half>(a, Dv, s);
            case 32: return launch_simt_k<32, __half>(a, Dv, s);
            case 64: return launch_simt_k<64, __half>(a, Dv, s);
            default: return launch_simt_k<128, __half>(a, Dv, s);
        }
    }
    if (dt == GDR_BF16) {
        switch (Dk) {
            case 16: return launch_simt_k<16, __nv_bfloat16>(a, Dv, s);
            case 32: return launch_simt_k<32, __nv_bfloat16>(a, Dv, s);
            case 64: return launch_simt_k<64, __nv_bfloat16>(a, Dv, s);
            default: return launch_simt_k<128, __nv_bfloat16>(a, Dv, s);
        }
    }
    switch (Dk) {
        case 16: return launch_simt_k<16, float>(a, Dv, s);
        case 32: return launch_simt_k<32, float>(a, Dv, s);
        case 64: return launch_simt_k<64, float>(a, Dv, s);
        default: return launch_simt_k<128, float>(a, Dv, s);
    }
}

}  // namespace gdr
