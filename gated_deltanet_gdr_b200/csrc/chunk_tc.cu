// chunk_tc.cu -- chunked prefill of the gated delta rule on the sm_100a tensor cores.
//
// The chunked (WY / UT transform) form of torch_chunk_gated_delta_rule (blog
// "gated-delta-net" page, steps 1-8), chunk C = 64, head size Dk = Dv = 128, bf16 in
// and out, fp32 accumulation and an fp32 state.  One CTA owns one (b, value head)
// chain and walks its chunks in order; per chunk:
//
//   a1  G_t = cumulative log-gate (tokens past the length count 0).
//   a2  [G; P] = [K; Q] K^T                 tcgen05.mma  M=128 N=64  K=128
//   a3  A = strictLower(beta_t k_t.k_s e^{G_t-G_s}),  T = (I + A)^{-1}  (fp32, CUDA cores:
//       16x16 diagonal blocks by forward substitution, merged 16 -> 32 -> 64 with
//       T21 = -T22 A21 T11)
//   a4  W = T diag(beta e^G) K,  U = T diag(beta) V   tcgen05.mma  M=128 N=128 K=64 (x2)
//   a5  R = [W; diag(e^G) X] S              tcgen05.mma  M=128 N=128 K=128
//       v_new = U - R[0:64]
//       dS = (diag(e^{G_last-G}) K)^T v_new tcgen05.mma  M=128 N=128 K=64
//       R[64:128] += Pm v_new, Pm = (X K^T) * e^{G_t-G_s} (causal)  -> o
//       S = e^{G_last} S + dS               (fp32, in registers)
//   a6  o -> bf16 -> TMA store; padding rows and chunks zero; final state once.
//
// X = scale * q / |q| (the fused l2norm and the 1/|k| factors are folded into the
// row/column scalings above, so raw q/k tiles feed the tensor cores directly).
// Operands are staged by TMA with 128-byte swizzle; accumulators live in TMEM
// (448 of 512 columns); the MMA is issued by one thread and completion is signalled
// through tcgen05.commit on an mbarrier.  Every wait is bounded: on a timeout the
// CTA sets GDR_DEVERR_TIMEOUT, releases TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdr {
using namespace sm100;

namespace {

constexpr int C = 64, D = 128, NT = 256;
constexpr uint32_t kTimeoutBit = 0x4u;

// ---- shared memory map (bytes from a 1024-aligned base) ----
// input stage: [K_b0 | Q_b0 | K_b1 | Q_b1 | V_b0 | V_b1], each 64 rows x 128 B (64 bf16)
constexpr uint32_t OFF_K0 = 0, OFF_Q0 = 8192, OFF_K1 = 16384, OFF_Q1 = 24576, OFF_V0 = 32768, OFF_V1 = 40960;
constexpr uint32_t STAGE_BYTES = 49152;
constexpr uint32_t OFF_A1 = 49152;   // [W; X_g] K-major 128 x 128: dk blocks at +0, +16K
constexpr uint32_t OFF_S = 81920;    // S bf16, MN-major (K = dk rows, N = dv): dv blocks at +0, +16K
constexpr uint32_t OFF_KT = 114688;  // K~ MN-major (M = dk, K = tok): dk blocks at +0, +8K
constexpr uint32_t OFF_TT = 131072;  // [T diag(beta); T diag(c_W)] K-major 128 x 64
constexpr uint32_t OFF_PM = 147456;  // [0; Pm] K-major 128 x 64
constexpr uint32_t OFF_O = 163840;   // out tile [tok][dv]: dv blocks at +0, +8K (TMA store source)
constexpr uint32_t OFF_R1 = 180224;  // solve workspace, aliased later in the chunk by VN
constexpr uint32_t OFF_VN = OFF_R1;  // v_new MN-major (K = tok, N = dv): dv blocks at +0, +8K
constexpr int FP = 65;               // padded fp32 row stride of the solve matrices
constexpr uint32_t OFF_AF = OFF_R1;
constexpr uint32_t OFF_TF = OFF_AF + 64 * FP * 4;
constexpr uint32_t OFF_X = OFF_TF + 64 * FP * 4;  // 32 x 33 fp32 scratch
constexpr uint32_t OFF_VEC = OFF_X + 32 * 33 * 4;
constexpr uint32_t OFF_BAR = OFF_VEC + 8 * 64 * 4;
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t TM_GP = 0, TM_WD = 64, TM_U = 192, TM_R = 320, TM_COLS = 512;

struct TcArgs {
    const void *beta;
    const float *g;
    const void *initial_state;
    const int32_t *lengths;
    float scale;
    int B, Nk, Nv, S;
    void *final_state;
    int l2norm;
    float eps;
    int beta_logits;
    const float *A_log, *dt_bias;
    unsigned int *err;
};

__device__ __forceinline__ uint32_t blk_off(uint32_t row, uint32_t col) {  // within a 128-B-row block
    return (row >> 3) * 1024u + sw128_offset(row & 7u, col);
}

// 16 bytes of 8 bf16 <-> 8 floats
__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ uint4 pack8(const float *f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

// T = (I + A)^{-1} for a strictly lower 64 x 64 A (fp32, row stride FP), 256 threads.
__device__ void solve_unit_lower(const float *sA, float *sT, float *sX, int tid) {
    // 16 x 16 diagonal blocks, one column per thread (64 threads)
    if (tid < 64) {
        const int base = (tid >> 4) * 16, j = tid & 15;
        float x[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) x[t] = (t == j) ? 1.f : 0.f;
#pragma unroll
        for (int t = 1; t < 16; ++t) {
            const float *ar = sA + (base + t) * FP + base;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int s = 0; s < t; ++s) {
                if (s & 1) a1 = fmaf(ar[s], x[s], a1);
                else a0 = fmaf(ar[s], x[s], a0);
            }
            if (t > j) x[t] = -(a0 + a1);
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) sT[(base + t) * FP + base + j] = x[t];
    }
    __syncthreads();
    // 16 -> 32: for p in {0,1}: T[r0.., c0..] = -T22 (A21 T11), r0 = 32p + 16, c0 = 32p
    for (int e = tid; e < 512; e += NT) {
        const int p = e >> 8, r = (e >> 4) & 15, c = e & 15, r0 = 32 * p + 16, c0 = 32 * p;
        float acc = 0.f;
        for (int k = c; k < 16; ++k) acc = fmaf(sA[(r0 + r) * FP + c0 + k], sT[(c0 + k) * FP + c0 + c], acc);
        sX[e] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 512; e += NT) {
        const int p = e >> 8, r = (e >> 4) & 15, c = e & 15, r0 = 32 * p + 16, c0 = 32 * p;
        float acc = 0.f;
        for (int k = 0; k <= r; ++k) acc = fmaf(sT[(r0 + r) * FP + r0 + k], sX[(p << 8) + (k << 4) + c], acc);
        sT[(r0 + r) * FP + c0 + c] = -acc;
    }
    __syncthreads();
    // 32 -> 64: T[32.., 0..32] = -T22 (A21 T11)
    for (int e = tid; e < 1024; e += NT) {
        const int r = e >> 5, c = e & 31;
        float acc = 0.f;
        for (int k = c; k < 32; ++k) acc = fmaf(sA[(32 + r) * FP + k], sT[k * FP + c], acc);
        sX[r * 33 + c] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 1024; e += NT) {
        const int r = e >> 5, c = e & 31;
        float acc = 0.f;
        for (int k = 0; k <= r; ++k) acc = fmaf(sT[(32 + r) * FP + 32 + k], sX[k * 33 + c], acc);
        sT[(32 + r) * FP + c] = -acc;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const TcArgs a) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_VEC);
    float *sGam = sBeta + 64, *sEG = sGam + 64, *sTail = sEG + 64, *sRk = sTail + 64, *sRq = sRk + 64;
    float *sCw = sRq + 64;
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_mma = bar_ld + 1;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar_ld + 2);
    float *sA = reinterpret_cast<float *>(sm + OFF_AF), *sT = reinterpret_cast<float *>(sm + OFF_TF);
    float *sX = reinterpret_cast<float *>(sm + OFF_X);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, hf = warp >> 2;
    const int bh = blockIdx.x, h = bh % a.Nv, b = bh / a.Nv, kh = h / (a.Nv / a.Nk);
    const int S = a.S;
    int L = a.lengths ? a.lengths[b] : S;
    const bool bad_len = (L < 0 || L > S);
    if (bad_len) L = 0;
    const int nvalid = (L + C - 1) / C, ntotal = (S + C - 1) / C;
    const int zq = b * a.Nk + kh;  // TMA z coordinate of q/k rows
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;

    if (tid == 0) {
        if (bad_len) raise_device_error(a.err, GDR_DEVERR_LENGTH);
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
    }
    if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
    // rows 0..63 of the [0; Pm] operand stay zero
    for (int e = tid; e < 8192 / 16; e += NT) reinterpret_cast<uint4 *>(sm + OFF_PM)[e] = make_uint4(0, 0, 0, 0);

    // ---- initial state: thread owns dk row i, dv columns [64 hf, 64 hf + 64) ----
    const int srow = q4 * 32 + lane;
    float st[64];
    {
        const __nv_bfloat16 *s0 = reinterpret_cast<const __nv_bfloat16 *>(a.initial_state);
        const size_t off = ((size_t)bh * D + srow) * D + 64 * hf;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            float f[8];
            if (s0) {
                unpack8(*reinterpret_cast<const uint4 *>(s0 + off + 8 * c8), f);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) st[8 * c8 + i] = f[i];
            *reinterpret_cast<uint4 *>(sm + OFF_S + hf * 16384 + blk_off(srow, 8 * c8)) = pack8(&st[8 * c8]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    uint32_t ph_ld = 0, ph_mma = 0;
    bool ok = true;
    auto issue_loads = [&](int chunk) {
        const int y = chunk * C;
        mbar_arrive_expect_tx(bar_ld, STAGE_BYTES);
        tma_load_3d(sm + OFF_K0, &tm_k, bar_ld, 0, y, zq);
        tma_load_3d(sm + OFF_K1, &tm_k, bar_ld, 64, y, zq);
        tma_load_3d(sm + OFF_Q0, &tm_q, bar_ld, 0, y, zq);
        tma_load_3d(sm + OFF_Q1, &tm_q, bar_ld, 64, y, zq);
        tma_load_3d(sm + OFF_V0, &tm_v, bar_ld, 0, y, bh);
        tma_load_3d(sm + OFF_V1, &tm_v, bar_ld, 64, y, bh);
    };
    auto mma_wait = [&]() {
        bool w = mbar_wait(bar_mma, ph_mma);
        ph_mma ^= 1u;
        tc_fence_after();
        return w;
    };
    if (tid == 0 && nvalid > 0) issue_loads(0);

    const float gA = (a.A_log && a.g) ? a.A_log[h] : 0.f, gB = (a.A_log && a.g) ? a.dt_bias[h] : 0.f;
    const __nv_bfloat16 *bg = reinterpret_cast<const __nv_bfloat16 *>(a.beta) + (size_t)bh * S;
    const float *gg = a.g ? a.g + (size_t)bh * S : nullptr;

    for (int c = 0; c < nvalid; ++c) {
        const int t0 = c * C, n = min(C, L - t0);
        // ---- a1: per-token scalars ----
        if (tid < C) {
            float bt = 0.f, gt = 0.f;
            if (tid < n) {
                bt = __bfloat162float(bg[t0 + tid]);
                if (a.beta_logits) bt = sigmoid_f32(bt);
                if (gg) gt = a.A_log ? gate_from_raw(gg[t0 + tid], gA, gB) : gg[t0 + tid];
            }
            sBeta[tid] = bt;
            sGam[tid] = gt;
        }
        bool w = mbar_wait(bar_ld, ph_ld);
        ph_ld ^= 1u;
        if (!__syncthreads_and(w)) { ok = false; break; }
        if (n < C) {  // padding rows of the last chunk: zero them so no padding value reaches a product
            for (int e = tid; e < (C - n) * 48; e += NT) {
                const int r = n + e / 48, k = e % 48, blk = k >> 3, ch = k & 7;
                const uint32_t base = blk == 0 ? OFF_K0 : blk == 1 ? OFF_Q0 : blk == 2 ? OFF_K1 : blk == 3 ? OFF_Q1
                                      : blk == 4 ? OFF_V0 : OFF_V1;
                *reinterpret_cast<uint4 *>(sm + base + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
            }
        }
        if (warp == 0) {  // inclusive scan of the gate over the chunk
            float x0 = sGam[2 * lane], x1 = sGam[2 * lane + 1];
            x1 += x0;
            float s = x1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                float y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            const float excl = s - x1;
            sGam[2 * lane] = excl + x0;
            sGam[2 * lane + 1] = excl + x1;
        }
        if (tid >= 64 && tid < 192) {  // row norms of k (tid 64..127) and q (tid 128..191)
            const int r = tid & 63;
            const bool isq = tid >= 128;
            float ss = 0.f;
            if (r < n) {
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
                    const uint8_t *rowp = sm + (isq ? (blk ? OFF_Q1 : OFF_Q0) : (blk ? OFF_K1 : OFF_K0)) + r * 128;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        float f[8];
                        unpack8(*reinterpret_cast<const uint4 *>(rowp + ch * 16), f);
#pragma unroll
                        for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
                    }
                }
            }
            const float rn = r < n ? (a.l2norm ? rsqrtf(ss + a.eps) : 1.f) : 0.f;
            if (isq) sRq[r] = a.scale * rn;
            else sRk[r] = rn;
        }
        __syncthreads();
        if (tid < C) {
            const float gl = sGam[C - 1], gt = sGam[tid];
            sEG[tid] = __expf(gt);
            sTail[tid] = __expf(gl - gt) * sRk[tid];
            sCw[tid] = sBeta[tid] * __expf(gt) * sRk[tid];
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- a2: [G; P] = [K; Q] K^T ----
        if (tid == 0) {
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t addr = sbase + OFF_K0 + (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16(tmem + TM_GP, sdesc_sw128(addr, 16, 1024), sdesc_sw128(addr, 16, 1024), id, k > 0);
            }
            mma_commit(bar_mma);
        }
        if (!__syncthreads_and(mma_wait())) { ok = false; break; }
        {
            float v[32];
            tmem_ld32(tmem + TM_GP + lane_base + 32 * hf, v);
            tmem_ld_wait();
            const int t = (q4 & 1) * 32 + lane;  // token (row of G or P)
            const float gt = sGam[t];
            if (q4 < 2) {  // A row t
                const float rb = sBeta[t] * sRk[t];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = 32 * hf + j;
                    sA[t * FP + s] = (s < t && t < n) ? rb * sRk[s] * v[j] * __expf(gt - sGam[s]) : 0.f;
                }
            } else {  // Pm row t -> rows 64 + t of the [0; Pm] operand
                const float rq = sRq[t];
                float pm[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = 32 * hf + j;
                    pm[j] = (s <= t && t < n) ? rq * sRk[s] * v[j] * __expf(gt - sGam[s]) : 0.f;
                }
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(sm + OFF_PM + blk_off(64 + t, 32 * hf + 8 * c8)) = pack8(&pm[8 * c8]);
            }
        }
        tc_fence_before();
        __syncthreads();
        // ---- a3: T = (I + A)^{-1}, then [T diag(beta); T diag(c_W)] as a bf16 operand ----
        solve_unit_lower(sA, sT, sX, tid);
        for (int e = tid; e < 128 * 8; e += NT) {
            const int R = e >> 3, j = e & 7, t = R & 63;
            const float *scl = R < 64 ? sBeta : sCw;
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int s = 8 * j + i;
                f[i] = s <= t ? sT[t * FP + s] * scl[s] : 0.f;
            }
            *reinterpret_cast<uint4 *>(sm + OFF_TT + blk_off(R, 8 * j)) = pack8(f);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- a4: W (rows 64..127 of T'K) and U (rows 0..63 of T'V) ----
        if (tid == 0) {
            const uint32_t id = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_TT + k * 32, 16, 1024);
                mma_bf16(tmem + TM_WD, ad, sdesc_sw128(sbase + OFF_K0 + k * 2048, 16384, 1024), id, k > 0);
                mma_bf16(tmem + TM_U, ad, sdesc_sw128(sbase + OFF_V0 + k * 2048, 8192, 1024), id, k > 0);
            }
            mma_commit(bar_mma);
        }
        // meanwhile: X_g rows (64..127 of A1) and K~ from the staged q/k tiles
        for (int e = tid; e < 2 * 64 * 16; e += NT) {
            const int isk = e >> 10, r = (e >> 4) & 63, blk = (e >> 3) & 1, ch = e & 7;
            const uint32_t rb = (r >> 3) * 1024u + (r & 7) * 128u + ch * 16u;  // same swizzle phase (row % 8)
            float f[8];
            if (isk) {
                unpack8(*reinterpret_cast<const uint4 *>(sm + (blk ? OFF_K1 : OFF_K0) + rb), f);
                const float sc = r < n ? sTail[r] : 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] *= sc;
                *reinterpret_cast<uint4 *>(sm + OFF_KT + blk * 8192 + rb) = pack8(f);
            } else {
                unpack8(*reinterpret_cast<const uint4 *>(sm + (blk ? OFF_Q1 : OFF_Q0) + rb), f);
                const float sc = r < n ? sEG[r] * sRq[r] : 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] *= sc;
                *reinterpret_cast<uint4 *>(sm + OFF_A1 + blk * 16384 + 8192 + rb) = pack8(f);
            }
        }
        fence_proxy_async_smem();
        if (!__syncthreads_and(mma_wait())) { ok = false; break; }
        if (q4 >= 2) {  // W rows -> rows 0..63 of A1
            const int t = (q4 - 2) * 32 + lane;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(tmem + TM_WD + lane_base + 64 * hf + 32 * half, v);
                tmem_ld_wait();
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(sm + OFF_A1 + hf * 16384 + blk_off(t, 32 * half + 8 * c8)) =
                        pack8(&v[8 * c8]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- a5: R = [W; X_g] S; the staged tiles are free: prefetch the next chunk ----
        if (tid == 0) {
            if (c + 1 < nvalid) issue_loads(c + 1);
            const uint32_t id = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_A1 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(sbase + OFF_S + k * 2048, 16384, 1024);
                mma_bf16(tmem + TM_R, ad, bd, id, k > 0);
            }
            mma_commit(bar_mma);
        }
        if (!__syncthreads_and(mma_wait())) { ok = false; break; }
        if (q4 < 2) {  // v_new = U - W S for token t, dv columns [64 hf, +64)
            const int t = q4 * 32 + lane;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float u[32], r[32];
                tmem_ld32(tmem + TM_U + lane_base + 64 * hf + 32 * half, u);
                tmem_ld32(tmem + TM_R + lane_base + 64 * hf + 32 * half, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) u[j] = t < n ? u[j] - r[j] : 0.f;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(sm + OFF_VN + hf * 8192 + blk_off(t, 32 * half + 8 * c8)) =
                        pack8(&u[8 * c8]);
            }
        }
        if (tid == 0) bulk_wait_read0();  // the previous out tile has been read by its store
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- dS = K~^T v_new ;  R[64:128] += Pm v_new ----
        if (tid == 0) {
            const uint32_t id_s = idesc_bf16(128, 128, true, true);
            const uint32_t id_o = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t bd = sdesc_sw128(sbase + OFF_VN + k * 2048, 8192, 1024);
                mma_bf16(tmem + TM_WD, sdesc_sw128(sbase + OFF_KT + k * 2048, 8192, 1024), bd, id_s, k > 0);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t bd = sdesc_sw128(sbase + OFF_VN + k * 2048, 8192, 1024);
                mma_bf16(tmem + TM_R, sdesc_sw128(sbase + OFF_PM + k * 32, 16, 1024), bd, id_o, 1);
            }
            mma_commit(bar_mma);
        }
        if (!__syncthreads_and(mma_wait())) { ok = false; break; }
        {
            const float eL = sEG[C - 1];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float d[32];
                tmem_ld32(tmem + TM_WD + lane_base + 64 * hf + 32 * half, d);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) st[32 * half + j] = fmaf(eL, st[32 * half + j], d[j]);
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(sm + OFF_S + hf * 16384 + blk_off(srow, 32 * half + 8 * c8)) =
                        pack8(&st[32 * half + 8 * c8]);
            }
            if (q4 >= 2) {  // o rows -> out tile
                const int t = (q4 - 2) * 32 + lane;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tmem_ld32(tmem + TM_R + lane_base + 64 * hf + 32 * half, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = t < n ? o[j] : 0.f;
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(sm + OFF_O + hf * 8192 + blk_off(t, 32 * half + 8 * c8)) =
                            pack8(&o[8 * c8]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            tma_store_3d(&tm_o, sm + OFF_O, 0, t0, bh);
            tma_store_3d(&tm_o, sm + OFF_O + 8192, 64, t0, bh);
            bulk_commit();
        }
    }
    if (!ok) {
        if (tid == 0) raise_device_error(a.err, kTimeoutBit);
    } else {
        // chunks past the length: zero rows
        if (nvalid < ntotal) {
            if (tid == 0) bulk_wait_read0();
            __syncthreads();
            for (int e = tid; e < 16384 / 16; e += NT) reinterpret_cast<uint4 *>(sm + OFF_O)[e] = make_uint4(0, 0, 0, 0);
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                for (int c = nvalid; c < ntotal; ++c) {
                    tma_store_3d(&tm_o, sm + OFF_O, 0, c * C, bh);
                    tma_store_3d(&tm_o, sm + OFF_O + 8192, 64, c * C, bh);
                }
                bulk_commit();
            }
        }
        if (a.final_state) {
            __nv_bfloat16 *fs = reinterpret_cast<__nv_bfloat16 *>(a.final_state) + ((size_t)bh * D + srow) * D + 64 * hf;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) *reinterpret_cast<uint4 *>(fs + 8 * c8) = pack8(&st[8 * c8]);
        }
    }
    if (tid == 0) bulk_wait0();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    }
    return fn;
}

// (D, S, Z) bf16 tensor, 64 x 64 boxes, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int S, long long Z) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)Z};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
    cuuint32_t box[3] = {64, 64, 1}, es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(int Dk, int Dv, gdr_dtype dt, int S) { return dt == GDR_BF16 && Dk == D && Dv == D && S > 0; }

cudaError_t launch_chunk_tc(const ChunkArgs &ca, cudaStream_t stream) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, ca.q, ca.S, (long long)ca.B * ca.Nk) || !make_map(&mk, ca.k, ca.S, (long long)ca.B * ca.Nk) ||
        !make_map(&mv, ca.v, ca.S, (long long)ca.B * ca.Nv) || !make_map(&mo, ca.out, ca.S, (long long)ca.B * ca.Nv))
        return cudaErrorInvalidValue;
    TcArgs a{};
    a.beta = ca.beta; a.g = ca.g; a.initial_state = ca.initial_state; a.lengths = ca.lengths; a.scale = ca.scale;
    a.B = ca.B; a.Nk = ca.Nk; a.Nv = ca.Nv; a.S = ca.S; a.final_state = ca.final_state;
    a.l2norm = ca.l2norm; a.eps = ca.eps; a.beta_logits = ca.beta_logits; a.A_log = ca.A_log;
    a.dt_bias = ca.dt_bias; a.err = ca.err;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const long long blocks = (long long)ca.B * ca.Nv;
    if (blocks == 0) return cudaSuccess;
    chunk_tc_kernel<<<(unsigned)blocks, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, a);
    return cudaGetLastError();
}

}  // namespace gdr
