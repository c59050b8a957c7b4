// chunk_tc.cu -- chunked prefill of the gated delta rule on the sm_100a tensor cores.
//
// The chunked (WY / UT transform) form of torch_chunk_gated_delta_rule (blog
// "gated-delta-net" page, steps 1-8), chunk C = 64, head size Dk = Dv = 128, bf16 in
// and out, fp32 accumulation and an fp32 state.  One CTA owns one (b, value head)
// chain.  Per chunk:
//
//   a1  G_t = cumulative log-gate (tokens past the length count 0).
//   a2  [G; P] = [K; Q] K^T                       tcgen05.mma  M=128 N=64  K=128
//   a3  A = strictLower(beta_t k_t.k_s e^{G_t-G_s});  T = (I + A)^{-1} in fp32 on the CUDA
//       cores: 16x16 diagonal blocks by forward substitution, merged 16 -> 32 -> 64 with
//       T21 = -T22 A21 T11 (register-blocked, fully unrolled).
//   a4  W = T diag(beta e^G) K,  U = T diag(beta) V        tcgen05.mma  M=128 N=128 K=64
//   a5  R = [W; diag(e^G) X] S                    tcgen05.mma  M=128 N=128 K=128
//       v_new = U - R[0:64]
//       S <- e^{G_last} S  (in TMEM, while R is computed)
//       S += (diag(e^{G_last-G}) K)^T v_new       tcgen05.mma  accumulate into the TMEM state
//       R[64:128] += Pm v_new,  Pm = (X K^T) e^{G_t-G_s} (causal)  -> o
//   a6  o -> bf16 -> TMA store; padding rows and chunks are zero; the final state is
//       written once from TMEM.
//
// X = scale * q / |q| (the fused l2norm and the 1/|k| factors are folded into row and
// column scalings, so the raw q/k tiles feed the tensor cores directly).
//
// Warp roles: warps 0-7 ("carry") run the serial chain of chunk c -- the three MMAs that
// touch the state and their epilogues; warps 8-15 ("prep") meanwhile prepare chunk c+1
// (tile loads, norms, gate scan, [G; P], the solve, W and U, the X_g and K~ operands).
// They hand over through mbarriers: a1_ready (prep -> carry: operands of chunk c are in
// place) and mma2_done (carry -> prep: the MMAs of chunk c-1 that read the shared
// operand buffers have completed).  Every wait is bounded: on a timeout the CTA sets
// the timeout bit of the device error word, releases TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdr {
using namespace sm100;

#ifdef GDR_PHASE_TIMERS
// Development aid, compiled only with -DGDR_PHASE_TIMERS: clock64() cycles per phase, summed
// in shared memory (so that taking a time stalls nothing) and added to g_phase by CTA 0 at
// the end; slots 0..15 prep group, 16..31 carry group; read by gdr_phase_timers_read.
__device__ unsigned long long g_phase[64];
#define PHASE(slot)                                                            \
    do {                                                                       \
        if (tid == 0 || tid == NGRP) {                                         \
            const unsigned long long now_ = clock64();                         \
            s_phase_[(slot)] += now_ - t_prev_;                                \
            t_prev_ = now_;                                                    \
        }                                                                      \
    } while (0)
// cycles one thread spends in the statements, accumulated into `slot`
#define TIMED(slot, ...)                                                       \
    do {                                                                       \
        const unsigned long long t0_ = clock64();                              \
        __VA_ARGS__;                                                           \
        s_phase_[(slot)] += clock64() - t0_;                                   \
    } while (0)
#define SOLVE_TIMER_ARGS , unsigned long long &t_prev_, int tid, unsigned long long *s_phase_
#define SOLVE_TIMER_PASS , t_prev_, tid, s_phase_
#else
#define PHASE(slot) \
    do {            \
    } while (0)
#define TIMED(slot, ...) \
    do {                 \
        __VA_ARGS__;     \
    } while (0)
#define SOLVE_TIMER_ARGS
#define SOLVE_TIMER_PASS
#endif

namespace {

// warps 0-7 carry, 8-15 prep, 16 control (TMA loads and the prep MMAs)
constexpr int C = 64, D = 128, NGRP = 256, NT = 2 * NGRP + 32, NPC = NGRP + 32;
constexpr int CTL_WARP = 16;
// BAR_PCTL: the prep warps and the control warp, at the hand-offs between them
constexpr int BAR_CARRY = 1, BAR_PREP = 2, BAR_PCTL = 3;
constexpr uint32_t kTimeoutBit = 0x4u;
// carry thread that issues the out-tile TMA stores (thread 0 issues the carry's MMAs)
constexpr int kStorer = 32;

// ---- shared memory map (bytes from a 1024-aligned base) ----
// input stage: [K_b0 | Q_b0 | K_b1 | Q_b1 | V_b0 | V_b1], each 64 rows x 128 B (64 bf16)
constexpr uint32_t OFF_K0 = 0, OFF_Q0 = 8192, OFF_K1 = 16384, OFF_Q1 = 24576, OFF_V0 = 32768;
constexpr uint32_t STAGE_BYTES = 49152;
constexpr uint32_t OFF_A1 = 49152;   // [W; X_g] K-major 128 x 128: dk blocks at +0, +16K
constexpr uint32_t OFF_S = 81920;    // S bf16, MN-major (K = dk rows, N = dv): dv blocks at +0, +16K
constexpr uint32_t OFF_KT = 114688;  // K~ MN-major (M = dk, K = tok): dk blocks at +0, +8K
constexpr uint32_t OFF_PM = 131072;  // [0; Pm] K-major 128 x 64
constexpr uint32_t OFF_VO = 147456;  // v_new (MN-major, K = tok, N = dv) then the out tile: dv blocks +0, +8K
constexpr int FP = 68;               // row stride (floats) of T: 16-byte aligned rows for float4 access
constexpr int FA = 68;               // row stride of A: each quarter-warp's 16-byte row stores hit distinct banks
constexpr int XP = 36;               // row stride of the merge scratch
constexpr uint32_t OFF_AF = 163840;  // A (fp32); after the solve it holds TT = [T diag(beta); T diag(c_W)]
constexpr uint32_t OFF_TT = OFF_AF;
constexpr uint32_t OFF_TF = OFF_AF + 64 * FA * 4;  // T (fp32)
constexpr uint32_t OFF_X = OFF_TF + 64 * FP * 4;
constexpr int NVEC = 10;             // per-chunk vectors of 64 floats (enum below)
constexpr uint32_t OFF_VEC = OFF_X + 32 * XP * 4;  // 2 sets x NVEC vectors x 64 floats
constexpr uint32_t OFF_BAR = OFF_VEC + 2 * NVEC * 64 * 4;
constexpr uint32_t SMEM_USED = OFF_BAR + 128;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_TF % 16 == 0 && OFF_X % 16 == 0, "float4 alignment");
static_assert(OFF_TF >= OFF_TT + 16384, "TT must fit inside the A matrix area");

// TMEM columns (all 128 lanes): [G;P] then W, U, R = [W S; o], the fp32 state S
constexpr uint32_t TM_GPW = 0, TM_U = 128, TM_R = 256, TM_S = 384, TM_COLS = 512;

// V_G2 = G log2(e); V_LAM = V_G2 - log2(1/|k|), so that e^{G_t - G_s} / |k_s| = 2^{V_G2[t] - V_LAM[s]};
// V_N holds the chunk's valid-token count in its first entry.
enum { V_BETA = 0, V_GAM, V_EG, V_TAIL, V_RK, V_RQ, V_CW, V_G2, V_LAM, V_N };
static_assert(V_N < NVEC, "vector slots");

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

// 2^x and log2(x) on the special-function unit (PTX ex2.approx / lg2.approx, flush to zero)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

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

// T = (I + A)^{-1} for a strictly lower 64 x 64 A (fp32, row stride FA; T row stride FP), by the 256 prep
// threads (p = 0..255).  Writes the lower triangle of T and zeros in the upper 16 x 16
// blocks that the merges read.
__device__ __forceinline__ void solve_unit_lower(const float *sA, float *sT, float *sX, int p SOLVE_TIMER_ARGS) {
    if (p < 64) {  // 16 x 16 diagonal blocks, one column per thread
        const int base = (p >> 4) * 16, j = p & 15;
        float x[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) x[t] = (t == j) ? 1.f : 0.f;
#pragma unroll
        for (int t = 1; t < 16; ++t) {
            const float *ar = sA + (base + t) * FA + base;
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
    } else {  // zero the upper 16 x 16 blocks inside the two 32 x 32 diagonal blocks
        for (int e = p - 64; e < 512; e += NGRP - 64) {
            const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
            sT[(32 * blk + r) * FP + 32 * blk + 16 + c] = 0.f;
        }
    }
    named_sync(BAR_PREP, NGRP);
    PHASE(13);
    // 16 -> 32: X_b = A21 T11, then T21 = -T22 X_b, for the blocks at rows 32b+16, cols 32b
    {
        const int blk = p >> 7, r = (p >> 3) & 15, c2 = (p & 7) * 2, r0 = 32 * blk + 16, c0 = 32 * blk;
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = sA[(r0 + r) * FA + c0 + k];
            const float2 t = *reinterpret_cast<const float2 *>(sT + (c0 + k) * FP + c0 + c2);
            x0 = fmaf(a, t.x, x0);
            x1 = fmaf(a, t.y, x1);
        }
        *reinterpret_cast<float2 *>(sX + (blk * 16 + r) * XP + c2) = make_float2(x0, x1);
        named_sync(BAR_PREP, NGRP);
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float t = sT[(r0 + r) * FP + r0 + k];
            const float2 xx = *reinterpret_cast<const float2 *>(sX + (blk * 16 + k) * XP + c2);
            y0 = fmaf(t, xx.x, y0);
            y1 = fmaf(t, xx.y, y1);
        }
        *reinterpret_cast<float2 *>(sT + (r0 + r) * FP + c0 + c2) = make_float2(-y0, -y1);
    }
    named_sync(BAR_PREP, NGRP);
    PHASE(14);
    // 32 -> 64: X = A21 T11, T21 = -T22 X with 32 x 32 blocks; one row x 4 columns per thread
    {
        const int r = p >> 3, c4 = (p & 7) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float a = sA[(32 + r) * FA + k];
            const float4 t = *reinterpret_cast<const float4 *>(sT + k * FP + c4);
            x.x = fmaf(a, t.x, x.x);
            x.y = fmaf(a, t.y, x.y);
            x.z = fmaf(a, t.z, x.z);
            x.w = fmaf(a, t.w, x.w);
        }
        *reinterpret_cast<float4 *>(sX + r * XP + c4) = x;
        named_sync(BAR_PREP, NGRP);
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float t = sT[(32 + r) * FP + 32 + k];
            const float4 xx = *reinterpret_cast<const float4 *>(sX + k * XP + c4);
            y.x = fmaf(t, xx.x, y.x);
            y.y = fmaf(t, xx.y, y.y);
            y.z = fmaf(t, xx.z, y.z);
            y.w = fmaf(t, xx.w, y.w);
        }
        *reinterpret_cast<float4 *>(sT + (32 + r) * FP + c4) = make_float4(-y.x, -y.y, -y.z, -y.w);
    }
    named_sync(BAR_PREP, NGRP);
}

__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smraw[];
    // 1024-byte aligned base, derived from smraw by pointer arithmetic (not through an
    // integer) so that the compiler keeps every access below in the shared address space
    uint8_t *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    float *vecs = reinterpret_cast<float *>(sm + OFF_VEC);
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_gp = bar_ld + 1, *bar_wu = bar_ld + 2, *bar_m1 = bar_ld + 3, *bar_m2 = bar_ld + 4;
    uint64_t *bar_a1 = bar_ld + 5;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar_ld + 8);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
    float *sA = reinterpret_cast<float *>(sm + OFF_AF), *sT = reinterpret_cast<float *>(sm + OFF_TF);
    float *sX = reinterpret_cast<float *>(sm + OFF_X);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, hf = (warp >> 2) & 1;
    const bool carry = warp < 8, control = warp == CTL_WARP;
    const int bh = blockIdx.x, h = bh % a.Nv, b = bh / a.Nv, kh = h / (a.Nv / a.Nk);
    const int S = a.S;
    int L = a.lengths ? a.lengths[b] : S;
    const bool bad_len = (L < 0 || L > S);
    if (bad_len) L = 0;
    const int nvalid = (L + C - 1) / C, ntotal = (S + C - 1) / C;
    const int zq = b * a.Nk + kh;  // TMA z coordinate of q/k rows
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const int row = q4 * 32 + lane;  // TMEM lane of this thread

    if (tid == 0) {
        if (bad_len) raise_device_error(a.err, GDR_DEVERR_LENGTH);
        for (int i = 0; i < 6; ++i) mbar_init(bar_ld + i, 1);
        *s_abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
    }
    if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
    for (int e = tid; e < 8192 / 16; e += NT) reinterpret_cast<uint4 *>(sm + OFF_PM)[e] = make_uint4(0, 0, 0, 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (carry) {
        // ---- initial state into TMEM (fp32) and the bf16 operand tile ----
        const __nv_bfloat16 *s0 = reinterpret_cast<const __nv_bfloat16 *>(a.initial_state);
        const size_t off = ((size_t)bh * D + row) * D + 64 * hf;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[32];
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float f[8];
                if (s0) {
                    unpack8(*reinterpret_cast<const uint4 *>(s0 + off + 32 * half + 8 * c8), f);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) v[8 * c8 + i] = f[i];
                *reinterpret_cast<uint4 *>(sm + OFF_S + hf * 16384 + blk_off(row, 32 * half + 8 * c8)) =
                    pack8(&v[8 * c8]);
            }
            tmem_st32(tmem + TM_S + lane_base + 64 * hf + 32 * half, v);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

#ifdef GDR_PHASE_TIMERS
    unsigned long long t_prev_ = clock64();
    __shared__ unsigned long long s_phase_[64];
    if (tid < 64) s_phase_[tid] = 0;
    __syncthreads();
#endif
    if (control) {
        // ============================== control warp ==============================
        // Lane 0 issues the prep MMAs and nothing else, lane 1 the TMA loads and L2 prefetches
        // (an MMA issued by a thread with copies of its own outstanding was seen to wait for
        // them).  Having a warp of its own, neither blocks a prep warp while the tensor pipe is
        // busy.  The warp follows the prep group's hand-off barriers (BAR_PCTL) and leaves
        // at the same barrier as the prep group when a wait timed out.
        auto prefetch_l2 = [&](int chunk) {
            const int y = chunk * C;
            tma_prefetch_3d(&tm_k, 0, y, zq);
            tma_prefetch_3d(&tm_k, 64, y, zq);
            tma_prefetch_3d(&tm_q, 0, y, zq);
            tma_prefetch_3d(&tm_q, 64, y, zq);
            tma_prefetch_3d(&tm_v, 0, y, bh);
            tma_prefetch_3d(&tm_v, 64, y, bh);
        };
        auto issue_loads = [&](int chunk) {
            const int y = chunk * C;
            mbar_arrive_expect_tx(bar_ld, STAGE_BYTES);
            tma_load_3d(sm + OFF_K0, &tm_k, bar_ld, 0, y, zq);
            tma_load_3d(sm + OFF_K1, &tm_k, bar_ld, 64, y, zq);
            tma_load_3d(sm + OFF_Q0, &tm_q, bar_ld, 0, y, zq);
            tma_load_3d(sm + OFF_Q1, &tm_q, bar_ld, 64, y, zq);
            tma_load_3d(sm + OFF_V0, &tm_v, bar_ld, 0, y, bh);
            tma_load_3d(sm + OFF_V0 + 8192, &tm_v, bar_ld, 64, y, bh);
        };
        if (lane == 1 && nvalid > 0) {
            issue_loads(0);
            if (nvalid > 1) prefetch_l2(1);
        }
        for (int c = 0; c < nvalid; ++c) {
            if (named_sync_or(BAR_PCTL, NPC, false)) break;  // H0: chunk c staged (or a timeout)
            if (lane == 1 && c + 2 < nvalid) prefetch_l2(c + 2);
            named_sync(BAR_PCTL, NPC);  // H1: padding rows zeroed
            if (lane == 0) {  // a2: [G; P] = [K; Q] K^T
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t addr = sbase + OFF_K0 + (k >> 2) * 16384 + (k & 3) * 32;
                    mma_bf16(tmem + TM_GPW, sdesc_sw128(addr, 16, 1024), sdesc_sw128(addr, 16, 1024), id, k > 0);
                }
                mma_commit(bar_gp);
            }
            if (named_sync_or(BAR_PCTL, NPC, false)) break;  // H2: TT operand and Pm in place
            if (lane == 0) {  // a4: W (rows 64..127 of TT K) and U (rows 0..63 of TT V)
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 128, false, true);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ad = sdesc_sw128(sbase + OFF_TT + k * 32, 16, 1024);
                    mma_bf16(tmem + TM_GPW, ad, sdesc_sw128(sbase + OFF_K0 + k * 2048, 16384, 1024), id, k > 0);
                    mma_bf16(tmem + TM_U, ad, sdesc_sw128(sbase + OFF_V0 + k * 2048, 8192, 1024), id, k > 0);
                }
                mma_commit(bar_wu);
            }
            if (named_sync_or(BAR_PCTL, NPC, false)) break;  // H3: staged tiles fully consumed
            if (lane == 1 && c + 1 < nvalid) issue_loads(c + 1);
        }
    } else if (!carry) {
        // =============================== prep group ===============================
        const int p = tid - NGRP;
        const float gA = (a.A_log && a.g) ? a.A_log[h] : 0.f, gB = (a.A_log && a.g) ? a.dt_bias[h] : 0.f;
        const __nv_bfloat16 *bg = reinterpret_cast<const __nv_bfloat16 *>(a.beta) + (size_t)bh * S;
        const float *gg = a.g ? a.g + (size_t)bh * S : nullptr;
        float nb = 0.f, ng = 0.f;  // prefetched raw beta / gate of the next chunk (threads p < 64)
        auto fetch = [&](int chunk) {
            nb = 0.f;
            ng = 0.f;
            const int t = chunk * C + p;
            if (p < C && chunk < nvalid && t < L) {
                nb = __bfloat162float(bg[t]);
                if (gg) ng = gg[t];
            }
        };
        bool to = false;  // a wait of this thread timed out
        auto wait_ok = [&](uint64_t *bar, uint32_t parity) {
            if (!mbar_wait(bar, parity)) to = true;
        };
        fetch(0);
        for (int c = 0; c < nvalid; ++c) {
            const uint32_t par = c & 1;
            float *vec = vecs + (c & 1) * NVEC * 64;
            float *vBeta = vec + V_BETA * 64, *vGam = vec + V_GAM * 64, *vEG = vec + V_EG * 64;
            float *vTail = vec + V_TAIL * 64, *vRk = vec + V_RK * 64, *vRq = vec + V_RQ * 64, *vCw = vec + V_CW * 64;
            const int n = min(C, L - c * C);
            if (p < C) {
                const bool valid = p < n;
                vBeta[p] = valid ? (a.beta_logits ? sigmoid_f32(nb) : nb) : 0.f;
                vGam[p] = valid ? (a.A_log ? gate_from_raw(ng, gA, gB) : ng) : 0.f;
            }
            fetch(c + 1);
            wait_ok(bar_ld, par);
            if (named_sync_or(BAR_PCTL, NPC, to)) break;  // H0
            PHASE(0);
            if (n < C) {  // padding rows of the last chunk: zero them so no padding value reaches a product
                for (int e = p; e < (C - n) * 48; e += NGRP) {
                    const int r = n + e / 48, k = e % 48;
                    *reinterpret_cast<uint4 *>(sm + (k >> 3) * 8192 + r * 128 + (k & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            named_sync(BAR_PCTL, NPC);  // H1: the control warp issues [G; P] = [K; Q] K^T
            PHASE(10);
            if (p < 32) {  // inclusive scan of the gate over the chunk (warp 8)
                float x0 = vGam[2 * p], x1 = vGam[2 * p + 1];
                x1 += x0;
                float s = x1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, o);
                    if (p >= o) s += y;
                }
                const float excl = s - x1;
                vGam[2 * p] = excl + x0;
                vGam[2 * p + 1] = excl + x1;
            }
#ifdef GDR_PHASE_TIMERS
            const unsigned long long tn0_ = clock64();
#endif
            {  // row norms of k and q: 4 threads per row, 32 elements each
                const int r = p >> 2, part = p & 3;
                const uint32_t off = (part >> 1) * 16384 + r * 128 + (part & 1) * 64;
                float sk = 0.f, sq = 0.f;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    // the order of the row's chunks does not matter for the sum; rotating it by
                    // the row spreads the warp's 8 rows over all banks
                    const uint32_t o = off + ((ch + r) & 3) * 16;
                    float fk[8], fq[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_K0 + o), fk);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_Q0 + o), fq);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        sk = fmaf(fk[i], fk[i], sk);
                        sq = fmaf(fq[i], fq[i], sq);
                    }
                }
                sk += __shfl_xor_sync(0xffffffffu, sk, 1);
                sq += __shfl_xor_sync(0xffffffffu, sq, 1);
                sk += __shfl_xor_sync(0xffffffffu, sk, 2);
                sq += __shfl_xor_sync(0xffffffffu, sq, 2);
                if (part == 0) {
                    vRk[r] = r < n ? (a.l2norm ? rsqrtf(sk + a.eps) : 1.f) : 0.f;
                    vRq[r] = r < n ? a.scale * (a.l2norm ? rsqrtf(sq + a.eps) : 1.f) : 0.f;
                }
            }
#ifdef GDR_PHASE_TIMERS
            if (lane == 0) s_phase_[40 + warp - 8] += clock64() - tn0_;
#endif
            named_sync(BAR_PREP, NGRP);
            PHASE(11);
            if (p < C) {
                const float gl = vGam[C - 1], gt = vGam[p];
                vEG[p] = __expf(gt);
                vTail[p] = __expf(gl - gt) * vRk[p];
                vCw[p] = vBeta[p] * __expf(gt) * vRk[p];
                const float g2 = gt * 1.4426950408889634f;
                vec[V_G2 * 64 + p] = g2;
                // padding rows have 1/|k| = 0, so their lambda is +inf and their entries vanish
                vec[V_LAM * 64 + p] = g2 - lg2_approx(vRk[p]);
                if (p == 0) vec[V_N * 64] = (float)n;
            }
            named_sync(BAR_PREP, NGRP);
            PHASE(1);
            wait_ok(bar_gp, par);
            tc_fence_after();
            PHASE(2);
            // A rows (from G, lanes 0..63) and Pm rows (from P, lanes 64..127; parked in TMEM as
            // fp32), with the decay e^{G_t - G_s} taken per entry.  Columns s > t are never read
            // (the solve reads the strict lower triangle, the Pm conversion masks), so the warps
            // whose 32 x 32 block lies wholly above the diagonal skip it.
#ifdef GDR_PHASE_TIMERS
            const unsigned long long tb0_ = clock64();
#endif
            if (!((q4 & 1) == 0 && hf == 1)) {
                float v[32];
                const uint32_t ta = tmem + TM_GPW + lane_base + 32 * hf;
                tmem_ld32(ta, v);
                const int t = row & 63;
                const float g2t = vec[V_G2 * 64 + t];
                // row factor: beta_t / |k_t| for A, scale / |q_t| for Pm (zero past the length)
                const float rf = t < n ? (q4 < 2 ? vBeta[t] * vRk[t] : vRq[t]) : 0.f;
                const float4 *lam4 = reinterpret_cast<const float4 *>(vec + V_LAM * 64 + 32 * hf);
                tmem_ld_wait();
                PHASE(12);
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 l = lam4[j4];
                    v[4 * j4 + 0] *= rf * ex2_approx(g2t - l.x);
                    v[4 * j4 + 1] *= rf * ex2_approx(g2t - l.y);
                    v[4 * j4 + 2] *= rf * ex2_approx(g2t - l.z);
                    v[4 * j4 + 3] *= rf * ex2_approx(g2t - l.w);
                }
                if (q4 < 2) {
                    // entries on or above the diagonal are never read by the solve
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4)
                        *reinterpret_cast<float4 *>(sA + t * FA + 32 * hf + 4 * j4) =
                            make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
                } else {
                    // entries above the diagonal are masked when Pm is converted to bf16
                    tmem_st32(ta, v);
                    tmem_st_wait();
                }
            }
#ifdef GDR_PHASE_TIMERS
            if (lane == 0) s_phase_[32 + warp - 8] += clock64() - tb0_;
#endif
            tc_fence_before();
            // a timed-out wait is carried to the next hand-off barrier, where the control warp
            // learns of it too
            named_sync(BAR_PREP, NGRP);
            PHASE(3);
            // ---- a3: T = (I + A)^{-1} and the bf16 operand [T diag(beta); T diag(c_W)] ----
            solve_unit_lower(sA, sT, sX, p SOLVE_TIMER_PASS);
            PHASE(4);
            for (int e = p; e < 128 * 8; e += NGRP) {
                const int R = e >> 3, j = e & 7, t = R & 63;
                const float *scl = (R < 64 ? vBeta : vCw) + 8 * j;
                const float4 t0 = *reinterpret_cast<const float4 *>(sT + t * FP + 8 * j);
                const float4 t1 = *reinterpret_cast<const float4 *>(sT + t * FP + 8 * j + 4);
                const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = (8 * j + i <= t) ? tv[i] * scl[i] : 0.f;
                *reinterpret_cast<uint4 *>(sm + OFF_TT + blk_off(R, 8 * j)) = pack8(f);
            }
            PHASE(5);
            // the carry group must be done with chunk c-1's MMAs before PM, K~, A1, U are rewritten
            if (c > 0 && !mbar_wait_sleep(bar_m2, (c - 1) & 1)) to = true;
            tc_fence_after();
            PHASE(6);
            if (q4 >= 2) {  // Pm rows (TMEM, fp32) -> rows 64 + t of the bf16 [0; Pm] operand
                float v[32];
                tmem_ld32(tmem + TM_GPW + lane_base + 32 * hf, v);
                tmem_ld_wait();
                const int t = row - 64;
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = (32 * hf + j <= t) ? v[j] : 0.f;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(sm + OFF_PM + blk_off(64 + t, 32 * hf + 8 * c8)) = pack8(&v[8 * c8]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            // H2: the control warp issues W and U (rows 64..127 of TT K, rows 0..63 of TT V)
            if (named_sync_or(BAR_PCTL, NPC, to)) break;
            tc_fence_after();
            PHASE(7);
            // meanwhile: X_g rows (64..127 of A1) and K~ from the staged q/k tiles
            for (int e = p; e < 2 * 64 * 16; e += NGRP) {
                const int isk = e >> 10, r = (e >> 4) & 63, blk = (e >> 3) & 1, ch = e & 7;
                const uint32_t rb = (r >> 3) * 1024u + (r & 7) * 128u + ch * 16u;  // same swizzle phase (row % 8)
                float f[8];
                if (isk) {
                    unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_K0 + blk * 16384 + rb), f);
                    const float sc = vTail[r];
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] *= sc;
                    *reinterpret_cast<uint4 *>(sm + OFF_KT + blk * 8192 + rb) = pack8(f);
                } else {
                    unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_Q0 + blk * 16384 + rb), f);
                    const float sc = vEG[r] * vRq[r];
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] *= sc;
                    *reinterpret_cast<uint4 *>(sm + OFF_A1 + blk * 16384 + 8192 + rb) = pack8(f);
                }
            }
            wait_ok(bar_wu, par);
            tc_fence_after();
            if (named_sync_or(BAR_PCTL, NPC, to)) break;  // H3: staged tiles fully consumed
            PHASE(8);
            if (q4 >= 2) {  // W rows -> rows 0..63 of A1
                const int t = row - 64;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(tmem + TM_GPW + lane_base + 64 * hf + 32 * half, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(sm + OFF_A1 + hf * 16384 + blk_off(t, 32 * half + 8 * c8)) =
                            pack8(&v[8 * c8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_PREP, NGRP);
            if (p == 0) mbar_arrive(bar_a1);
            PHASE(9);
        }
        if (to && p == 0) *s_abort = 1;
    } else {
        // =============================== carry group ==============================
        bool to = false;  // a wait of this thread timed out
        bool stop = false;
        auto wait_ok = [&](uint64_t *bar, uint32_t parity) {
            if (!mbar_wait(bar, parity)) to = true;
        };
        for (int c = 0; c < nvalid; ++c) {
            const uint32_t par = c & 1;
            const float *vec = vecs + (c & 1) * NVEC * 64;
            if (!mbar_wait_sleep(bar_a1, par)) to = true;
            if (named_sync_or(BAR_CARRY, NGRP, to)) { stop = true; break; }
            tc_fence_after();
            PHASE(16);
            const int n = (int)vec[V_N * 64];
            const float eL = vec[V_EG * 64 + C - 1];
            // ---- R = [W; X_g] S ----
            if (tid == 0) {
                const uint32_t id = idesc_bf16(128, 128, false, true);
                TIMED(23, {
                    _Pragma("unroll")
                    for (int k = 0; k < 8; ++k) {
                        const uint64_t ad = sdesc_sw128(sbase + OFF_A1 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(sbase + OFF_S + k * 2048, 16384, 1024);
                        mma_bf16(tmem + TM_R, ad, bd, id, k > 0);
                    }
                    mma_commit(bar_m1);
                });
            }
            // meanwhile: S <- e^{G_last} S in TMEM (MMA2 accumulates onto it)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                const uint32_t ta = tmem + TM_S + lane_base + 64 * hf + 32 * half;
                tmem_ld32(ta, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= eL;
                tmem_st32(ta, v);
            }
            tmem_st_wait();
            wait_ok(bar_m1, par);
            if (tid == kStorer) bulk_wait_read0();  // the previous out tile (same buffer as v_new) is read
            tc_fence_before();
            if (named_sync_or(BAR_CARRY, NGRP, to)) { stop = true; break; }
            tc_fence_after();
            PHASE(17);
            if (q4 < 2) {  // v_new = U - W S for token t, dv columns [64 hf, +64)
                const int t = row;
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
                        *reinterpret_cast<uint4 *>(sm + OFF_VO + hf * 8192 + blk_off(t, 32 * half + 8 * c8)) =
                            pack8(&u[8 * c8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_CARRY, NGRP);
            tc_fence_after();
            PHASE(18);
            // ---- S += K~^T v_new ;  R[64:128] += Pm v_new ----
            if (tid == 0) {
                const uint32_t id_s = idesc_bf16(128, 128, true, true);
                const uint32_t id_o = idesc_bf16(128, 128, false, true);
                TIMED(24, {
                    _Pragma("unroll")
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t bd = sdesc_sw128(sbase + OFF_VO + k * 2048, 8192, 1024);
                        mma_bf16(tmem + TM_S, sdesc_sw128(sbase + OFF_KT + k * 2048, 8192, 1024), bd, id_s, 1);
                    }
                    _Pragma("unroll")
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t bd = sdesc_sw128(sbase + OFF_VO + k * 2048, 8192, 1024);
                        mma_bf16(tmem + TM_R, sdesc_sw128(sbase + OFF_PM + k * 32, 16, 1024), bd, id_o, 1);
                    }
                    mma_commit(bar_m2);
                });
            }
            wait_ok(bar_m2, par);
            tc_fence_after();
            if (named_sync_or(BAR_CARRY, NGRP, to)) { stop = true; break; }
            PHASE(19);
            // ---- S (fp32, TMEM) -> bf16 operand tile;  o rows -> out tile ----
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(tmem + TM_S + lane_base + 64 * hf + 32 * half, v);
                tmem_ld_wait();
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(sm + OFF_S + hf * 16384 + blk_off(row, 32 * half + 8 * c8)) =
                        pack8(&v[8 * c8]);
            }
            if (q4 >= 2) {
                const int t = row - 64;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tmem_ld32(tmem + TM_R + lane_base + 64 * hf + 32 * half, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = t < n ? o[j] : 0.f;
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(sm + OFF_VO + hf * 8192 + blk_off(t, 32 * half + 8 * c8)) =
                            pack8(&o[8 * c8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_CARRY, NGRP);
            tc_fence_after();
            if (tid == kStorer) {
                tma_store_3d(&tm_o, sm + OFF_VO, 0, c * C, bh);
                tma_store_3d(&tm_o, sm + OFF_VO + 8192, 64, c * C, bh);
                bulk_commit();
            }
            PHASE(20);
        }
        if (stop && tid == 0) *s_abort = 1;
        if (!stop) {
            // chunks past the length: zero rows
            if (nvalid < ntotal) {
                if (tid == kStorer) bulk_wait_read0();
                named_sync(BAR_CARRY, NGRP);
                for (int e = tid; e < 16384 / 16; e += NGRP)
                    reinterpret_cast<uint4 *>(sm + OFF_VO)[e] = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
                named_sync(BAR_CARRY, NGRP);
                if (tid == kStorer) {
                    for (int c = nvalid; c < ntotal; ++c) {
                        tma_store_3d(&tm_o, sm + OFF_VO, 0, c * C, bh);
                        tma_store_3d(&tm_o, sm + OFF_VO + 8192, 64, c * C, bh);
                    }
                    bulk_commit();
                }
            }
            if (a.final_state) {
                __nv_bfloat16 *fs =
                    reinterpret_cast<__nv_bfloat16 *>(a.final_state) + ((size_t)bh * D + row) * D + 64 * hf;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(tmem + TM_S + lane_base + 64 * hf + 32 * half, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(fs + 32 * half + 8 * c8) = pack8(&v[8 * c8]);
                }
            }
        }
        if (tid == kStorer) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *s_abort) raise_device_error(a.err, kTimeoutBit);
#ifdef GDR_PHASE_TIMERS
    if (blockIdx.x == 0 && tid < 64) g_phase[tid] += s_phase_[tid];
#endif
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

#ifdef GDR_PHASE_TIMERS
extern "C" int gdr_phase_timers_read(unsigned long long *out) {
    cudaDeviceSynchronize();
    cudaMemcpyFromSymbol(out, g_phase, sizeof(unsigned long long) * 64);
    unsigned long long z[64] = {0};
    cudaMemcpyToSymbol(g_phase, z, sizeof(z));
    return 0;
}
#endif

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
