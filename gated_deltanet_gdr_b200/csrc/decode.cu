// decode.cu -- recurrent decode step of the gated delta rule over a slot pool.
//
// Operation (lite_boost recurrent_gated_delta_rule; torch_recurrent_gated_delta_rule
// token loop; deltanet.rs delta_step): per (sequence b, value head h) the state
// S = pool[idx[b*S]][h] (Dk x Dv) is read ONCE from HBM, the L_b tokens of the
// call are applied in fp32 registers (decay by exp(g) * exp(gk[i]) per row, readout
// k^T S, delta, rank-1 write, output q^T S), and the state is written back ONCE per
// commit (normally once per call).
//
// The work is memory bound: ~7 flops per state element per token against 2 (bf16)
// or 4 (fp32) bytes read and written.  Mapping (one CTA per (b, h, 64-column slab)):
//   - a warp owns 16 state columns; lane = (row group rg in 0..15, column vector cv in 0..1),
//     each lane holds rows rg, rg+16, ... of 8 consecutive columns in registers;
//   - every state access is a 16-byte vector (8 bf16 or 2 x 4 fp32), and a lane pair
//     covers a full 32-byte sector of one row;
//   - the two column reductions of a token (k^T S' and q^T S' of the decayed state S')
//     are taken in one pass and finished by a 4-step xor butterfly inside the warp, so
//     no shared memory or block barrier sits in the token loop;
//   - the output uses o = q^T S' + (q . k) d, which needs no second pass over S.
#include "common.cuh"
#include "kernels.h"

namespace gdr {

template <int DK, int DV> struct DecodeShape {
    static constexpr int DVC = DV < 64 ? DV : 64;  // state columns per CTA
    static constexpr int NSPLIT = DV / DVC;        // CTAs per (b, h)
    static constexpr int NW = DVC / 16;            // warps per CTA, 16 columns each
    static constexpr int NT = NW * 32;
    static constexpr int RPT = DK / 16;            // state rows per lane
    static_assert(DK % 16 == 0 && DV % 16 == 0, "head sizes must be multiples of 16");
};

template <int DK, int DV, typename TI, typename TS>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
decode_kernel(const DecodeArgs a) {
    using Sh = DecodeShape<DK, DV>;
    constexpr int DVC = Sh::DVC, NW = Sh::NW, NT = Sh::NT, RPT = Sh::RPT;
    constexpr int T = kDecodeMaxTokens;

    __shared__ float s_x[T][DK];    // scale * q_hat
    __shared__ float s_k[T][DK];    // k_hat
    __shared__ float s_dec[T][DK];  // exp(g) * exp(gk[i])
    __shared__ float s_v[T][DVC];
    __shared__ float s_beta[T], s_qk[T];
    __shared__ int s_idx[T];
    __shared__ int s_state;  // 0 ok, 1 skip (bad args)

    const int split = blockIdx.x % Sh::NSPLIT;
    const int bh = blockIdx.x / Sh::NSPLIT;
    const int h = bh % a.Nv, b = bh / a.Nv;
    const int kh = h / (a.Nv / a.Nk);
    const int S = a.S;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int col_cta = split * DVC;

    const int L = a.lengths[b];
    int A = a.accepted ? a.accepted[b] : L;
    TI *out = reinterpret_cast<TI *>(a.out) + ((size_t)bh * S) * DV + col_cta;

    if (tid == 0) {
        int bad = 0;
        if (L < 0 || L > S) {
            bad = 1;
            raise_device_error(a.err, GDR_DEVERR_LENGTH);
        } else {
            int nref = L < A ? L : A;
            if (nref < 1) nref = L > 0 ? 1 : 0;
            for (int t = 0; t < nref; ++t) {
                int s = a.idx[(size_t)b * S + t];
                if (s < 0 || s >= a.slots) bad = 1;
            }
            if (bad) raise_device_error(a.err, GDR_DEVERR_SLOT_INDEX);
        }
        s_state = bad;
    }
    __syncthreads();
    const bool skip = s_state != 0;
    const int Lv = skip ? 0 : L;
    if (A > Lv) A = Lv;

    // zero the padding rows t >= L (all rows when the sequence is skipped)
    for (int e = tid; e < (S - Lv) * (DVC / 8); e += NT) {
        int t = Lv + e / (DVC / 8), c = (e % (DVC / 8)) * 8;
        float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        Vec8<TI>::store(out + (size_t)t * DV + c, z);
    }
    if (Lv == 0) return;

    // ---- stage the per-token vectors (with the optional prologue) ----
    const TI *qg = reinterpret_cast<const TI *>(a.q) + (((size_t)b * a.Nk + kh) * S) * DK;
    const TI *kg = reinterpret_cast<const TI *>(a.k) + (((size_t)b * a.Nk + kh) * S) * DK;
    for (int t = warp; t < Lv; t += NW) {
        float xs = 0.f, ks = 0.f;
        for (int i = lane; i < DK; i += 32) {
            float xq = to_f32(qg[(size_t)t * DK + i]), xk = to_f32(kg[(size_t)t * DK + i]);
            s_x[t][i] = xq;
            s_k[t][i] = xk;
            xs += xq * xq;
            ks += xk * xk;
        }
        float qs = a.scale, kn = 1.f;
        if (a.l2norm) {
            xs = warp_sum(xs);
            ks = warp_sum(ks);
            qs = a.scale * rsqrtf(xs + a.eps);
            kn = rsqrtf(ks + a.eps);
        }
        float dot = 0.f;
        for (int i = lane; i < DK; i += 32) {
            float xq = s_x[t][i] * qs, xk = s_k[t][i] * kn;
            s_x[t][i] = xq;
            s_k[t][i] = xk;
            dot += xq * xk;
        }
        dot = warp_sum(dot);
        const size_t gi = ((size_t)bh * S) + t;
        float gt = 0.f;
        if (a.g) gt = a.A_log ? gate_from_raw(a.g[gi], a.A_log[h], a.dt_bias[h]) : a.g[gi];
        const float ag = expf(gt);
        for (int i = lane; i < DK; i += 32) s_dec[t][i] = a.gk ? ag * expf(a.gk[gi * DK + i]) : ag;
        if (lane == 0) {
            float bt = to_f32(reinterpret_cast<const TI *>(a.beta)[gi]);
            s_beta[t] = a.beta_logits ? sigmoid_f32(bt) : bt;
            s_qk[t] = dot;
            s_idx[t] = a.idx[(size_t)b * S + t];
        }
    }
    const TI *vg = reinterpret_cast<const TI *>(a.v) + ((size_t)bh * S) * DV + col_cta;
    for (int e = tid; e < Lv * DVC; e += NT) s_v[e / DVC][e % DVC] = to_f32(vg[(size_t)(e / DVC) * DV + e % DVC]);
    __syncthreads();

    // ---- read the state tile once ----
    const int cv = lane & 1, rg = lane >> 1;
    const int col = warp * 16 + cv * 8;  // column within the CTA slab
    const size_t head_off = (size_t)h * DK * DV + col_cta + col;
    const TS *src = reinterpret_cast<const TS *>(a.pool) + (size_t)s_idx[0] * a.Nv * DK * DV + head_off;
    float st[RPT][8];
#pragma unroll
    for (int m = 0; m < RPT; ++m) Vec8<TS>::load(src + (size_t)(rg + 16 * m) * DV, st[m]);

    for (int t = 0; t < Lv; ++t) {
        float mk[8], mq[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mk[c] = mq[c] = 0.f;
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int r = rg + 16 * m;
            const float dec = s_dec[t][r], kr = s_k[t][r], xr = s_x[t][r];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float s = st[m][c] * dec;
                st[m][c] = s;
                mk[c] = fmaf(kr, s, mk[c]);
                mq[c] = fmaf(xr, s, mq[c]);
            }
        }
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                mk[c] += __shfl_xor_sync(0xffffffffu, mk[c], o);
                mq[c] += __shfl_xor_sync(0xffffffffu, mq[c], o);
            }
        }
        const float bt = s_beta[t], qk = s_qk[t];
        float d[8], o8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            d[c] = bt * (s_v[t][col + c] - mk[c]);
            o8[c] = fmaf(qk, d[c], mq[c]);
        }
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float kr = s_k[t][rg + 16 * m];
#pragma unroll
            for (int c = 0; c < 8; ++c) st[m][c] = fmaf(kr, d[c], st[m][c]);
        }
        if (rg == 0) Vec8<TI>::store(out + (size_t)t * DV + col, o8);
        if (t < A && (t == A - 1 || s_idx[t + 1] != s_idx[t])) {
            TS *dst = reinterpret_cast<TS *>(a.pool) + (size_t)s_idx[t] * a.Nv * DK * DV + head_off;
#pragma unroll
            for (int m = 0; m < RPT; ++m) Vec8<TS>::store(dst + (size_t)(rg + 16 * m) * DV, st[m]);
        }
    }
}

template <int DK, int DV, typename TI, typename TS>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t stream) {
    using Sh = DecodeShape<DK, DV>;
    const long long blocks = (long long)a.B * a.Nv * Sh::NSPLIT;
    if (blocks == 0) return cudaSuccess;
    decode_kernel<DK, DV, TI, TS><<<(unsigned)blocks, Sh::NT, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int DK, int DV>
static cudaError_t launch_decode_d(const DecodeArgs &a, gdr_dtype dt, gdr_dtype st, cudaStream_t stream) {
    if (dt == GDR_BF16 && st == GDR_BF16) return launch_decode_t<DK, DV, __nv_bfloat16, __nv_bfloat16>(a, stream);
    if (dt == GDR_BF16 && st == GDR_F32) return launch_decode_t<DK, DV, __nv_bfloat16, float>(a, stream);
    if (dt == GDR_F32 && st == GDR_BF16) return launch_decode_t<DK, DV, float, __nv_bfloat16>(a, stream);
    return launch_decode_t<DK, DV, float, float>(a, stream);
}

template <int DK>
static cudaError_t launch_decode_k(const DecodeArgs &a, int Dv, gdr_dtype dt, gdr_dtype st, cudaStream_t s) {
    switch (Dv) {
        case 16: return launch_decode_d<DK, 16>(a, dt, st, s);
        case 32: return launch_decode_d<DK, 32>(a, dt, st, s);
        case 64: return launch_decode_d<DK, 64>(a, dt, st, s);
        default: return launch_decode_d<DK, 128>(a, dt, st, s);
    }
}

cudaError_t launch_decode(const DecodeArgs &a, int Dk, int Dv, gdr_dtype dt, gdr_dtype st, cudaStream_t s) {
    switch (Dk) {
        case 16: return launch_decode_k<16>(a, Dv, dt, st, s);
        case 32: return launch_decode_k<32>(a, Dv, dt, st, s);
        case 64: return launch_decode_k<64>(a, Dv, dt, st, s);
        default: return launch_decode_k<128>(a, Dv, dt, st, s);
    }
}

}  // namespace gdr
