// chunk_tc.cu -- chunked prefill of the gated delta rule on the sm_100a tensor cores.
//
// The chunked (WY / UT transform) form of torch_chunk_gated_delta_rule (blog
// "gated-delta-net" page, steps 1-8), chunk C = 64, head size Dk = Dv = 128, bf16 or fp16
// in and out (the MMA operand copies in the same type), fp32 accumulation and an fp32 state.  One CTA owns one (b, value head)
// chain.  Per chunk:
//
//   a1  G_t = cumulative log-gate (tokens past the length count 0).
//   a2  [G; P] = [K; Q] K^T                       tcgen05.mma  M=128 N=64  K=128
//   a3  A = strictLower(beta_t k_t.k_s e^{G_t-G_s});  T = (I + A)^{-1}: 16x16 diagonal blocks by
//       forward substitution and the 16 -> 32 merges T21 = -T22 A21 T11 in fp32 on the CUDA
//       cores, the 32 -> 64 merge with warp-level tf32 tensor-core MMAs (mma.sync m16n8k8,
//       operands and products in registers).
//   a4  W = T diag(beta e^G) K,  U = T diag(beta) V        tcgen05.mma  M=128 N=128 K=64
//   a5  R = [W; diag(e^G) X] S                    tcgen05.mma  M=128 N=128 K=128
//       v_new = U - R[0:64]
//       S <- e^{G_last} S  (in TMEM, while R is computed)
//       S += (diag(e^{G_last-G}) K)^T v_new       tcgen05.mma  accumulate into the TMEM state
//       R[64:128] += Pm v_new,  Pm = (X K^T) e^{G_t-G_s} (causal)  -> o
//   a6  o -> bf16 -> TMA store; padding rows and chunks are zero; the final state is
//       written once from TMEM.  With the optional epilogue each o row first becomes
//       o / sqrt(mean o^2 + eps) * norm_w * silu(z) in fp32 (the layer's gated RMSNorm).
//
// X = scale * q / |q| (the fused l2norm and the 1/|k| factors are folded into row and
// column scalings, so the raw q/k tiles feed the tensor cores directly).
//
// Warp roles: warps 0-7 ("carry") run the serial chain of chunk c -- the three MMAs that
// touch the state and their epilogues; warps 8-15 ("prep") meanwhile prepare chunk c+1
// (tile loads, norms, gate scan, [G; P], the solve, W and U, the X_g and K~ operands).
// They hand over through mbarriers: a1_ready (prep -> carry: operands of chunk c are in
// place) and mma2_done (carry -> prep: the MMAs of chunk c-1 that read the shared
// operand buffers have completed).  Every wait is bounded by elapsed time and gives up early once another group
// has stopped; then the CTA waits for its own copies and MMAs still in flight, sets the timeout bit of the device
// error word, releases TMEM and returns.  Stop decisions inside a group are collective (bar.red.or at the group's
// hand-offs), so every member leaves its loop at the same barrier.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdr {
using namespace sm100;

namespace {
// The first bounded wait of the one-kernel schedule that ran out since the word was last read (0: none): bit 31
// set, the warp in bits 24-29, the barrier in bits 16-23, its phase parity in bit 15, the CTA in bits 0-14.
__device__ unsigned int g_timeout_site = 0;
constexpr uint64_t kDefaultWaitNs = 1000000000ull;  // a bounded wait gives up after 1 s
constexpr uint64_t kDrainWaitNs = 1000000000ull;    // waits for the CTA's own copies and MMAs at the exit
unsigned long long g_wait_ns = 0;                   // 0: the default limit (a test may shorten it)
}  // namespace

void chunk_tc_set_wait_ns(unsigned long long ns) { g_wait_ns = ns; }
unsigned long long chunk_wait_ns() { return g_wait_ns ? g_wait_ns : kDefaultWaitNs; }
cudaError_t chunk_tc_take_timeout_site(unsigned int *site) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(site, g_timeout_site, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_timeout_site, &zero, sizeof(unsigned int));
    return e;
}

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

// warps 0-7 carry, 8-15 prep, 16 control (TMA loads and the prep MMAs), 17-19 helpers (the K~ operand).  The
// register file is allocated to warps in groups of four, so the helpers cost no registers per thread.
constexpr int C = 64, D = 128, NGRP = 256, NHELP = 96, NT = 2 * NGRP + 32 + NHELP, NPC = NGRP + 32;
constexpr int CTL_WARP = 16;
// BAR_PCTL: the prep warps and the control warp, at the hand-offs between them; BAR_HELP: the helper warps
// BAR_EPI: the carry warps that hold o rows (TMEM lanes 64..127), at the epilogue's row-norm exchange
constexpr int BAR_CARRY = 1, BAR_PREP = 2, BAR_PCTL = 3, BAR_HELP = 4, BAR_EPI = 5;
// carry thread that issues the out-tile TMA stores (thread 0 issues the carry's MMAs)
constexpr int kStorer = 32;

// ---- shared memory map (bytes from a 1024-aligned base) ----
// input tiles of the prep group, 64 rows x 128 B (64 bf16) each, per dk block b (b = 0, 1) at 24 KB b:
// [K even chunk | Q | K odd chunk], so that [K; Q] (even chunks) and [Q; K] (odd chunks) are each one
// 128-row operand for the Gram; the K tile is double-buffered so that the next chunk's K and Q can land
// during the current chunk.  V (dv blocks at +0, +8K) is single-buffered: it is needed late.
constexpr uint32_t KQ_BLK = 24576, OFF_V = 49152;
__host__ __device__ constexpr uint32_t off_k(int par, int blk) { return blk * KQ_BLK + (par ? 16384u : 0u); }
__host__ __device__ constexpr uint32_t off_q(int blk) { return blk * KQ_BLK + 8192u; }
__host__ __device__ constexpr uint32_t off_gram(int par, int blk) { return blk * KQ_BLK + (par ? 8192u : 0u); }
// operands of the carry group for the chunk it runs
constexpr uint32_t OFF_A1 = 65536;   // [W; Q] K-major 128 x 128: dk blocks at +0, +16K (Q rows by TMA)
constexpr uint32_t OFF_KT = 98304;   // K tile by TMA, scaled in place to diag(tail) K: MN-major (M = dk,
                                     // K = tok), dk blocks at +0, +8K
constexpr uint32_t OFF_S = 114688;   // S bf16, MN-major (K = dk rows, N = dv): dv blocks at +0, +16K
// Pm (K-major 64 x 64), two buffers; the o MMA reads 128 rows starting 8 KB before the buffer so that
// Pm forms rows 64..127 (rows 0..63 are whatever precedes it and land in dead accumulator lanes)
constexpr uint32_t OFF_PM0 = 147456, OFF_PM1 = 155648;
constexpr uint32_t OFF_VO = 163840;  // v_new (MN-major, K = tok, N = dv), then the out tile: dv blocks +0, +8K
// the solve T = (I + A)^{-1} (see solve_diag16_merge and the prep group's a3 step)
constexpr int SP = 36;                 // row stride (floats) of the plain 32 x 32 blocks: 16-byte aligned rows
constexpr uint32_t OFF_TT = 180224;   // TT = [T diag(beta); T diag(c_W)], bf16, K-major 128 x 64; until it is
                                      // written it holds the diagonal blocks of A (plain) and the merge scratch
constexpr uint32_t OFF_AP = OFF_TT;              // A11, A22 (plain, 2 x 32 rows of SP floats)
constexpr uint32_t OFF_XP = OFF_TT + 64 * SP * 4;  // 16 x 16 merge scratch (2 x 16 rows of SP floats)
constexpr uint32_t OFF_TP = 196608;   // T11, T22 (plain, 2 x 32 rows of SP floats)
constexpr uint32_t OFF_A21 = 205824;  // A rows 32..63, columns 0..31 (plain, 32 rows of SP floats)
constexpr uint32_t OFF_XM = 210432;   // X = A21 T11 of the 32 -> 64 merge (plain, 32 rows of SP floats)
static_assert(OFF_XP + 32 * SP * 4 <= OFF_TT + 16384, "plain A and the merge scratch fit in the TT area");
static_assert(OFF_TP + 64 * SP * 4 <= OFF_A21 && OFF_A21 + 32 * SP * 4 <= OFF_XM, "plain T, A21");
constexpr int NVEC = 11;             // per-chunk vectors of 64 floats (enum below)
constexpr uint32_t OFF_VEC = 215040;  // 2 sets x NVEC vectors x 64 floats
static_assert(OFF_XM + 32 * SP * 4 <= OFF_VEC, "merge product");
constexpr uint32_t OFF_BAR = OFF_VEC + 2 * NVEC * 64 * 4;
constexpr uint32_t OFF_EPI = OFF_BAR + 256;  // epilogue: partial squared norms of the o rows (2 x 64 floats)
// the order of the chains (see order_chain): the B lengths, then the selected sequence
constexpr int kRankMaxB = 256;
constexpr uint32_t OFF_LEN = OFF_EPI + 512;
constexpr uint32_t SMEM_USED = OFF_LEN + kRankMaxB * 4 + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_TT % 1024 == 0, "swizzle atoms");
static_assert(OFF_PM0 >= 8192 && OFF_PM1 == OFF_PM0 + 8192, "Pm buffers");

// TMEM columns (all 128 lanes): the Gram [K; Q][K; Q]^T (then the solve's merge products); U (lanes
// 0..63; with the epilogue, lanes 64..127 take the chunk's gate factors norm_w * silu(z) once the U product
// has completed); R: first W of the chunk (lanes 64..127, written while R is otherwise free), then [W S; o]
// (lanes 0..63 / 64..127); the fp32 state S
constexpr uint32_t TM_GPW = 0, TM_U = 128, TM_R = 256, TM_S = 384, TM_COLS = 512;

// V_G2 = G log2(e); V_LAM = V_G2 - log2(1/|k|), so that e^{G_t - G_s} / |k_s| = 2^{V_G2[t] - V_LAM[s]};
// V_XS = e^G scale / |q| (row factor of Q S); V_N holds the chunk's valid-token count in its first entry.
// V_ET = e^{G_last - G}; V_TAIL = V_ET / |k|.
enum { V_BETA = 0, V_EG, V_TAIL, V_RK, V_RQ, V_CW, V_G2, V_LAM, V_XS, V_ET, V_N };
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
    const void *epi_z;  // NULL: no epilogue
    const float *epi_w;
    float epi_eps;
    uint64_t wait_ns;  // limit of each bounded wait
};

__device__ __forceinline__ uint32_t blk_off(uint32_t row, uint32_t col) {  // within a 128-B-row block
    return (row >> 3) * 1024u + sw128_offset(row & 7u, col);
}

// silu(x) = x sigmoid(x).  For bf16 outputs sigmoid(x) = (1 + tanh(x / 2)) / 2 with tanh on the special-function
// unit (PTX tanh.approx, relative error about 2^-11, below the bf16 rounding of 2^-9 that follows): one
// special-function operation per element.  For fp16 outputs (rounding 2^-11) x / (1 + e^{-x}) with the fast
// division (about 1e-6).
template <typename T> __device__ __forceinline__ float silu_out(float x);
template <> __device__ __forceinline__ float silu_out<__nv_bfloat16>(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return x * fmaf(0.5f, t, 0.5f);
}
template <> __device__ __forceinline__ float silu_out<__half>(float x) { return __fdividef(x, 1.f + __expf(-x)); }

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

// The element type of the inputs, the operand copies and the outputs: bf16 or fp16 (tcgen05 kind::f16 takes
// either, A and B of the same type).  TMA data type, descriptor operand format, and pairs packed / unpacked.
template <typename T> struct TcT;
template <> struct TcT<__nv_bfloat16> {
    static constexpr CUtensorMapDataType kMap = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static constexpr uint32_t kFmt = 1;
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }
    static __device__ __forceinline__ float2 unpack2(uint32_t u) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
    }
};
template <> struct TcT<__half> {
    static constexpr CUtensorMapDataType kMap = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    static constexpr uint32_t kFmt = 0;
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
    static __device__ __forceinline__ float2 unpack2(uint32_t u) {
        return __half22float2(*reinterpret_cast<const __half2 *>(&u));
    }
};
template <typename T> __host__ __device__ constexpr uint32_t idesc_t(int M, int N, bool a_mn_major, bool b_mn_major) {
    return idesc_f16kind(M, N, a_mn_major, b_mn_major, TcT<T>::kFmt);
}

template <typename T> __device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = TcT<T>::unpack2(w[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
template <typename T> __device__ __forceinline__ uint4 pack8(const float *f) {
    return make_uint4(TcT<T>::pack2(f[0], f[1]), TcT<T>::pack2(f[2], f[3]), TcT<T>::pack2(f[4], f[5]),
                      TcT<T>::pack2(f[6], f[7]));
}

// D (16 x 8) += A (16 x 8) B (8 x 8) with tf32 operands and fp32 accumulation: one warp-level tensor-core MMA.
// Thread l of the warp (g = l / 4, i = l % 4) holds a = {A[g][i], A[g+8][i], A[g][i+4], A[g+8][i+4]},
// b = {B[i][g], B[i+4][g]} and d = {D[g][2i], D[g][2i+1], D[g+8][2i], D[g+8][2i+1]}.
__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// fp32 -> tf32, rounded to nearest (ties away from zero)
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
    return y;
}

// One 16 x 8 tile of D = A B (32 x 32 operands, plain layouts with row stride SP floats) for k-steps
// [ks0, ks1): thread fragments as in mma_16x8x8_tf32.
__device__ __forceinline__ void gemm32_tile(float (&d)[4], const float *A, const float *B, int rt, int ct, int ks0,
                                            int ks1, int lane) {
    const int g = lane >> 2, i = lane & 3;
    d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        if (ks < ks0 || ks >= ks1) continue;
        const float *ar = A + (16 * rt + g) * SP + 8 * ks + i;
        const float *br = B + (8 * ks + i) * SP + 8 * ct + g;
        const uint32_t a[4] = {to_tf32(ar[0]), to_tf32(ar[8 * SP]), to_tf32(ar[4]), to_tf32(ar[8 * SP + 4])};
        const uint32_t b[2] = {to_tf32(br[0]), to_tf32(br[4 * SP])};
        mma_16x8x8_tf32(d, a, b);
    }
}

// Element (r, c) of a 32 x 32 diagonal block (r and c in the same 32-block) in the plain layout.
__device__ __forceinline__ int pl(int r, int c) { return ((r >> 5) * 32 + (r & 31)) * SP + (c & 31); }

// T = (I + A)^{-1}, first part, by the 256 prep threads p: the two 32 x 32 diagonal blocks T11 and T22
// (A strictly lower; its diagonal blocks plain in sA).  The four 16 x 16 diagonal blocks by forward
// substitution (one column per thread, zeros above the diagonal), then for each 32-block the lower-left
// 16 x 16 block T21 = -T22 (A21 T11) with the CUDA cores.
__device__ __forceinline__ void solve_diag16_merge(const float *sA, float *sT, float *sX, int p) {
    if (p < 64) {
        const int base = (p >> 4) * 16, j = p & 15;
        float x[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) x[t] = (t == j) ? 1.f : 0.f;
        const float *a0p = sA + pl(base, base);
#pragma unroll
        for (int t = 1; t < 16; ++t) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int sv = 0; sv < t; ++sv) {
                if (sv & 1) a1 = fmaf(a0p[t * SP + sv], x[sv], a1);
                else a0 = fmaf(a0p[t * SP + sv], x[sv], a0);
            }
            if (t > j) x[t] = -(a0 + a1);
        }
        float *t0p = sT + pl(base, base) + j;
#pragma unroll
        for (int t = 0; t < 16; ++t) t0p[t * SP] = x[t];
    } else {  // zero the upper 16 x 16 block inside each 32 x 32 diagonal block
        for (int e = p - 64; e < 512; e += 192) {
            const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
            sT[(32 * blk + r) * SP + 16 + c] = 0.f;
        }
    }
    named_sync(BAR_PREP, NGRP);
    // 16 -> 32: X = A21 T11, then T21 = -T22 X, for the blocks at rows 32 b + 16, columns 32 b
    const int blk = p >> 7, r = (p >> 3) & 15, c2 = (p & 7) * 2;
    const float *ab = sA + blk * 32 * SP;
    float *tb = sT + blk * 32 * SP;
    float x0 = 0.f, x1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float a = ab[(16 + r) * SP + k];
        const float2 t = *reinterpret_cast<const float2 *>(tb + k * SP + c2);
        x0 = fmaf(a, t.x, x0);
        x1 = fmaf(a, t.y, x1);
    }
    *reinterpret_cast<float2 *>(sX + (blk * 16 + r) * SP + c2) = make_float2(x0, x1);
    named_sync(BAR_PREP, NGRP);
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float t = tb[(16 + r) * SP + 16 + k];
        const float2 xx = *reinterpret_cast<const float2 *>(sX + (blk * 16 + k) * SP + c2);
        y0 = fmaf(t, xx.x, y0);
        y1 = fmaf(t, xx.y, y1);
    }
    *reinterpret_cast<float2 *>(tb + (16 + r) * SP + c2) = make_float2(-y0, -y1);
    named_sync(BAR_PREP, NGRP);
}

// The sequence a CTA runs, longest first.  A CTA holds an SM for its whole chain and CTAs start in index
// order as SMs free up, so with more chains than SMs a long chain that starts late sets the end of the launch
// (longest-processing-time-first list scheduling).  CTA i takes the sequence whose valid length ranks
// i / Nv-th (longest first, ties by index; an invalid length counts as 0); its value head stays i % Nv.
// Without lengths, or with more than kRankMaxB sequences, the order is the index order.  Called by all
// threads of the CTA before anything else touches shared memory.  The kernel's ordered instantiation runs
// it, and the host launches that one only when the chains outnumber the resident CTAs: its sequence index
// lives in a register, where the index order's is recomputed from blockIdx, and in one wave order is moot.
__device__ __forceinline__ int order_chain(const TcArgs &a, int tid, uint8_t *sm) {
    const int seq = blockIdx.x / a.Nv;
    if (!a.lengths || a.B <= 1 || a.B > kRankMaxB) return seq;
    int *s_len = reinterpret_cast<int *>(sm + OFF_LEN);
    volatile int *s_sel = s_len + kRankMaxB;
    for (int i = tid; i < a.B; i += NT) {
        const int L = a.lengths[i];
        s_len[i] = (L < 0 || L > a.S) ? 0 : L;
    }
    __syncthreads();
    for (int i = tid; i < a.B; i += NT) {  // the ranks are a permutation of 0..B-1: one i matches
        const int Li = s_len[i];
        int r = 0;
        for (int j = 0; j < a.B; ++j) {
            const int Lj = s_len[j];
            r += (Lj > Li) || (Lj == Li && j < i);
        }
        if (r == seq) *s_sel = i;
    }
    __syncthreads();
    return *s_sel;
}

// kGate = false: the build for g = NULL (no decay): no gate scan, the A and Pm entries take the column factor
// 1/|k_s| without an exponential, and the state is never rescaled in TMEM.
// The part of a bounded wait after its first test failed, out of line: one copy of the polling loop and the
// timeout record instead of one per call site.  The kernel's code is large (every role's loop is hot at once),
// and with a CTA on most SMs its instruction fetches contend: the warps' stalls for instructions doubled from
// 32 to 128 CTAs.  This, with the loops over 32-column halves kept rolled, took 12 % off a launch of 128 chains.
__device__ __noinline__ bool wait_slow(uint64_t *bar, uint32_t parity, uint64_t limit_ns, volatile int *abort,
                                       uint32_t bar_index) {
    if (mbar_wait_ns(bar, parity, limit_ns, abort)) return true;
    if (!*abort)
        atomicCAS(&g_timeout_site, 0u,
                  0x80000000u | ((threadIdx.x >> 5) << 24) | (bar_index << 16) | (parity << 15) |
                      (blockIdx.x & 0x7fffu));
    return false;
}

template <typename T, bool kGate, bool kOrdered>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smraw[];
    // 1024-byte aligned base, derived from smraw by pointer arithmetic (not through an
    // integer) so that the compiler keeps every access below in the shared address space
    uint8_t *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    float *vecs = reinterpret_cast<float *>(sm + OFF_VEC);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    // bar_ld: K and Q of the chunk landed (bar_ldv: V); bar_gp / bar_wu: the prep MMAs completed; bar_m1 / bar_m2: the carry MMAs
    // completed; bar_a1: the prep group handed chunk c to the carry group; bar_cq / bar_ck: the raw Q rows
    // of A1 / the raw K tile landed; bar_pf[i]: the carry group is done with Pm buffer i and vector set i
    uint64_t *bar_ld = bars, *bar_gp = bars + 1, *bar_wu = bars + 2, *bar_m1 = bars + 3, *bar_m2 = bars + 4;
    uint64_t *bar_a1 = bars + 5, *bar_cq = bars + 6, *bar_ck = bars + 7, *bar_pf = bars + 8;
    // bar_vr: the control warp has written the gate vectors of the next chunk (one phase per chunk)
    uint64_t *bar_vr = bars + 10, *bar_ldv = bars + 11;
    // bar_go: the carry group has taken chunk c over (its tail factors are in place); bar_kt: the helper warps
    // have scaled chunk c's K tile into K~ (one phase per chunk each)
    uint64_t *bar_go = bars + 12, *bar_kt = bars + 13;
    // bar_dr: two commits, every MMA of the control warp and of the carry group completed (exit); bar_gf: the
    // two helper warps of TMEM lanes 64..127 have written chunk c's epilogue gate factors (one phase per chunk)
    uint64_t *bar_dr = bars + 14, *bar_gf = bars + 15;
    constexpr int kNumBars = 16;
    static_assert(kNumBars * 8 + 8 <= OFF_EPI - OFF_BAR, "barriers, TMEM base and abort flag before the epilogue scratch");
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + kNumBars);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, hf = (warp >> 2) & 1;
    const bool carry = warp < 8, control = warp == CTL_WARP, helper = warp > CTL_WARP;
    const int h = blockIdx.x % a.Nv;
    const int b = kOrdered ? order_chain(a, tid, sm) : (int)blockIdx.x / a.Nv;
    const int bh = kOrdered ? b * a.Nv + h : (int)blockIdx.x, kh = h / (a.Nv / a.Nk);
    const int S = a.S;
    int L = a.lengths ? a.lengths[b] : S;
    const bool bad_len = (L < 0 || L > S);
    if (bad_len) L = 0;
    const int nvalid = (L + C - 1) / C, ntotal = (S + C - 1) / C;
    const int zq = b * a.Nk + kh;  // TMA z coordinate of q/k rows
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const int row = q4 * 32 + lane;  // TMEM lane of this thread

    // a bounded wait: false when it ran out (the first such wait of the launch is recorded) or another group stopped
    auto bw = [&](uint64_t *bar, uint32_t parity) -> bool {
        if (mbar_test(bar, parity)) return true;
        return wait_slow(bar, parity, a.wait_ns, s_abort, (uint32_t)(bar - bars));
    };
    // loads issued per barrier by the thread that issues them (one phase each), for the drain at the exit
    int n_ld = 0, n_ldv = 0, n_cq = 0, n_ck = 0;

    // raw Q rows of A1 and the raw K tile of chunk c, for the carry group (issued by carry thread 0)
    auto load_carry_q = [&](int chunk) {
        ++n_cq;
        mbar_arrive_expect_tx(bar_cq, 16384);
        tma_load_3d(sm + OFF_A1 + 8192, &tm_q, bar_cq, 0, chunk * C, zq);
        tma_load_3d(sm + OFF_A1 + 16384 + 8192, &tm_q, bar_cq, 64, chunk * C, zq);
    };
    auto load_carry_k = [&](int chunk) {
        ++n_ck;
        mbar_arrive_expect_tx(bar_ck, 16384);
        tma_load_3d(sm + OFF_KT, &tm_k, bar_ck, 0, chunk * C, zq);
        tma_load_3d(sm + OFF_KT + 8192, &tm_k, bar_ck, 64, chunk * C, zq);
    };

    if (tid == 0) {
        if (bad_len) raise_device_error(a.err, GDR_DEVERR_LENGTH);
        for (int i = 0; i < kNumBars; ++i) mbar_init(bars + i, i >= 14 ? 2 : 1);
        *s_abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
        if (nvalid > 0) {
            load_carry_q(0);
            load_carry_k(0);
        }
    }
    if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (carry) {
        // ---- initial state into TMEM (fp32) and the bf16 operand tile ----
        const T *s0 = reinterpret_cast<const T *>(a.initial_state);
        const size_t off = ((size_t)bh * D + row) * D + 64 * hf;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            float v[32];
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float f[8];
                if (s0) {
                    unpack8<T>(*reinterpret_cast<const uint4 *>(s0 + off + 32 * half + 8 * c8), f);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) v[8 * c8 + i] = f[i];
                *reinterpret_cast<uint4 *>(sm + OFF_S + hf * 16384 + blk_off(row, 32 * half + 8 * c8)) =
                    pack8<T>(&v[8 * c8]);
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
        // Lane 0 issues the prep MMAs and nothing else, lane 1 the input-stage TMA loads and L2
        // prefetches (an MMA issued by a thread with copies of its own outstanding was seen to wait
        // for them).  Having a warp of its own, neither blocks a prep warp while the tensor pipe is
        // busy.  The warp follows the prep group's hand-off barriers (BAR_PCTL) and leaves at the
        // same barrier as the prep group when a wait timed out.
        auto prefetch_l2 = [&](int chunk) {
            const int y = chunk * C;
            tma_prefetch_3d(&tm_k, 0, y, zq);
            tma_prefetch_3d(&tm_k, 64, y, zq);
            tma_prefetch_3d(&tm_q, 0, y, zq);
            tma_prefetch_3d(&tm_q, 64, y, zq);
            tma_prefetch_3d(&tm_v, 0, y, bh);
            tma_prefetch_3d(&tm_v, 64, y, bh);
            if (a.epi_z) {  // the chunk's z rows of the epilogue: one contiguous block of valid rows
                const int rows = min(C, L - y);
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                             ::"l"(static_cast<const T *>(a.epi_z) + ((size_t)bh * S + y) * D),
                             "r"((uint32_t)(rows * D * 2))
                             : "memory");
            }
        };
        // K of a chunk into its buffer (this also arms the chunk's K/Q barrier), Q into the single Q buffer,
        // V into the single V buffer
        auto issue_k = [&](int chunk) {
            const int y = chunk * C, pc = chunk & 1;
            ++n_ld;
            mbar_arrive_expect_tx(bar_ld, 32768);
            tma_load_3d(sm + off_k(pc, 0), &tm_k, bar_ld, 0, y, zq);
            tma_load_3d(sm + off_k(pc, 1), &tm_k, bar_ld, 64, y, zq);
        };
        auto issue_q = [&](int chunk) {
            const int y = chunk * C;
            tma_load_3d(sm + off_q(0), &tm_q, bar_ld, 0, y, zq);
            tma_load_3d(sm + off_q(1), &tm_q, bar_ld, 64, y, zq);
        };
        auto issue_v = [&](int chunk) {
            const int y = chunk * C;
            ++n_ldv;
            mbar_arrive_expect_tx(bar_ldv, 16384);
            tma_load_3d(sm + OFF_V, &tm_v, bar_ldv, 0, y, bh);
            tma_load_3d(sm + OFF_V + 8192, &tm_v, bar_ldv, 64, y, bh);
        };
        // The gate and beta vectors of a chunk, which need no Gram: beta (from logits), the cumulative
        // gate G (from the raw gate), e^G, G log2(e), e^{G_last - G} and the valid-token count; two
        // tokens per lane, the scan over the chunk by warp shuffles.
        const float gA = (a.A_log && a.g) ? a.A_log[h] : 0.f, gB = (a.A_log && a.g) ? a.dt_bias[h] : 0.f;
        const T *bg = reinterpret_cast<const T *>(a.beta) + (size_t)bh * S;
        const float *gg = (kGate && a.g) ? a.g + (size_t)bh * S : nullptr;
        // raw beta and gate values of a chunk's tokens (two per lane), loaded a chunk before they are used so
        // that their memory latency stays off the hand-offs
        auto load_raw = [&](int chunk, float (&rb)[2], float (&rg)[2]) {
            const int n = min(C, L - chunk * C);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int tt = 2 * lane + i, t = chunk * C + tt;
                rb[i] = tt < n ? to_f32(bg[t]) : 0.f;
                rg[i] = (tt < n && gg) ? gg[t] : 0.f;
            }
        };
        auto chunk_vectors = [&](int chunk, const float (&rb)[2], const float (&rg)[2]) {
            float *vec = vecs + (chunk & 1) * NVEC * 64;
            const int n = min(C, L - chunk * C);
            float bv[2], gv[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int tt = 2 * lane + i;
                bv[i] = tt < n ? (a.beta_logits ? sigmoid_f32(rb[i]) : rb[i]) : 0.f;
                gv[i] = (kGate && tt < n) ? (a.A_log ? gate_from_raw(rg[i], gA, gB) : rg[i]) : 0.f;
            }
            if (!kGate) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int tt = 2 * lane + i;
                    vec[V_BETA * 64 + tt] = bv[i];
                    vec[V_EG * 64 + tt] = 1.f;
                    vec[V_G2 * 64 + tt] = 0.f;
                    vec[V_ET * 64 + tt] = 1.f;
                }
                if (lane == 0) vec[V_N * 64] = (float)n;
                return;
            }
            const float x1 = gv[0] + gv[1];
            float sc = x1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, sc, o);
                if (lane >= o) sc += y;
            }
            const float gl = __shfl_sync(0xffffffffu, sc, 31);
            const float G[2] = {sc - x1 + gv[0], sc};
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int tt = 2 * lane + i;
                vec[V_BETA * 64 + tt] = bv[i];
                vec[V_EG * 64 + tt] = __expf(G[i]);
                vec[V_G2 * 64 + tt] = G[i] * 1.4426950408889634f;
                vec[V_ET * 64 + tt] = __expf(gl - G[i]);
            }
            if (lane == 0) vec[V_N * 64] = (float)n;
        };
        bool to = false;
        float rbN[2] = {0.f, 0.f}, rgN[2] = {0.f, 0.f};
        if (nvalid > 0) {
            load_raw(0, rbN, rgN);
            chunk_vectors(0, rbN, rgN);
        }
        if (lane == 1 && nvalid > 0) {
            issue_k(0);
            issue_q(0);
            issue_v(0);
            if (nvalid > 1) prefetch_l2(1);
        }
        __syncwarp();
        for (int c = 0; c < nvalid; ++c) {
            const uint32_t par = c & 1;
            if (c + 1 < nvalid) load_raw(c + 1, rbN, rgN);
            // H0: the prep group is at chunk c (and, for a last partial chunk, has zeroed its padding rows)
            if (named_sync_or(BAR_PCTL, NPC, to)) break;
            if (lane == 0) {  // a2: the Gram [K; Q][K; Q]^T ([Q; K][Q; K]^T for odd chunks); its diagonal gives
                              // the row norms
                if (!bw(bar_ld, par)) to = true;
                tc_fence_after();
                const uint32_t id = idesc_t<T>(128, 128, false, false);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t addr = sbase + off_gram(par, k >> 2) + (k & 3) * 32;
                    mma_bf16(tmem + TM_GPW, sdesc_sw128(addr, 16, 1024), sdesc_sw128(addr, 16, 1024), id, k > 0);
                }
                mma_commit(bar_gp);
            }
            if (lane == 1) {
                // V and the other K buffer were last read by the W/U MMAs of chunk c-1, issued a whole chunk
                // ago; V of this chunk is needed only at its own W/U MMAs, K and Q of the next chunk at its
                // Gram.  Q is free once this chunk's Gram has read it.
                if (c > 0 && !bw(bar_wu, (c - 1) & 1)) to = true;
                if (c > 0) issue_v(c);
                if (c + 1 < nvalid) {
                    // the K/Q barrier is armed for chunk c+1 only after its phase for chunk c has completed (an
                    // arrival on a phase still pending would count towards that phase)
                    if (!bw(bar_ld, par)) to = true;
                    issue_k(c + 1);
                    if (bw(bar_gp, par)) issue_q(c + 1);
                    else to = true;
                    if (c + 2 < nvalid) prefetch_l2(c + 2);
                }
            }
            __syncwarp();
            // while the prep group solves chunk c: the vectors of chunk c+1, into the set that chunk c-1
            // used (free once the carry's MMA2 of chunk c-1 completed)
            if (c + 1 < nvalid) {
                if (c >= 1 && !bw(bar_pf + ((c + 1) & 1), ((c - 1) >> 1) & 1)) to = true;
                chunk_vectors(c + 1, rbN, rgN);
            }
            __syncwarp();
            if (lane == 0 && c + 1 < nvalid) mbar_arrive(bar_vr);
        }
    } else if (helper) {
        // ============================== helper warps ==============================
        // K~ = diag(e^{G_last - G} / |k|) K of each chunk, in place in the carry's raw K tile (rows past the
        // length, whatever they hold, become zero): the A operand of the state update, made off the carry's
        // serial chain.  The tile of chunk c lands after MMA2 of chunk c-1 and is needed at MMA2 of chunk c.
        // With the epilogue, the two helper warps of TMEM lanes 64..127 (the lanes of the o rows) then write
        // the chunk's gate factors w silu(z) for their row, all 128 columns, into columns TM_U.. of those
        // lanes: the U product leaves them unused (its rows 64..127 are never read), they are free from the
        // completion of the chunk's W/U products until the carry's epilogue has read them, and the next W/U
        // products are issued only after that.
        const int hp = tid - (CTL_WARP + 1) * 32;
        const bool gf_rows = a.epi_z != nullptr && q4 >= 2;  // warps 18 and 19
        bool to = false;
        for (int c = 0; c < nvalid; ++c) {
            const uint32_t par = c & 1;
            const float *vec = vecs + par * NVEC * 64;
            const int t_gf = row - 64, n_gf = min(C, L - c * C);
            const T *z_row = gf_rows && t_gf < n_gf
                                 ? static_cast<const T *>(a.epi_z) + ((size_t)bh * S + (size_t)c * C + t_gf) * D
                                 : nullptr;
            if (z_row) {  // the row's 256 bytes of z into L1 while the K~ tile is scaled
                asm volatile("prefetch.global.L1 [%0];" ::"l"(z_row));
                asm volatile("prefetch.global.L1 [%0];" ::"l"(z_row + 64));
            }
            // bar_go of chunk c+1 follows bar_kt of chunk c, and the K tile of chunk c+1 is loaded after MMA2 of
            // chunk c, which waits for bar_kt of chunk c: neither wait can be a phase behind
            if (!bw(bar_go, par)) to = true;
            if (!bw(bar_ck, par)) to = true;
            if (!to) {
                const int n = (int)vec[V_N * 64];
                const float *vtail = vec + V_TAIL * 64;
                for (int e = hp; e < 1024; e += NHELP) {
                    const int t = (e >> 3) & 63;
                    uint4 *pk = reinterpret_cast<uint4 *>(sm + OFF_KT + (e >> 9) * 8192 + t * 128 + (e & 7) * 16);
                    float f[8];
                    unpack8<T>(*pk, f);
                    const float sc = vtail[t];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f[j] = t < n ? f[j] * sc : 0.f;
                    *pk = pack8<T>(f);
                }
            }
            fence_proxy_async_smem();
            if (named_sync_or(BAR_HELP, NHELP, to)) break;
            if (hp == 0) mbar_arrive(bar_kt);
            if (gf_rows) {
                // the chunk's W/U products (which also write these lanes of TM_U) have completed: bar_wu of
                // chunk c+1 needs the carry's epilogue of chunk c, which waits for this warp's bar_gf
                // (one verdict per warp: the TMEM stores below are warp-collective)
                if (!__all_sync(0xffffffffu, bw(bar_wu, par))) to = true;
                tc_fence_after();
                if (!to) {
#pragma unroll 1
                    for (int blk = 0; blk < 4; ++blk) {
                        float f[32];
#pragma unroll
                        for (int c8 = 0; c8 < 4; ++c8) {
                            float zf[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                            if (z_row) unpack8<T>(*reinterpret_cast<const uint4 *>(z_row + 32 * blk + 8 * c8), zf);
                            const float4 *wp = reinterpret_cast<const float4 *>(a.epi_w + 32 * blk + 8 * c8);
                            const float4 w0 = wp[0], w1 = wp[1];
                            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i) f[8 * c8 + i] = wv[i] * silu_out<T>(zf[i]);
                        }
                        tmem_st32(tmem + TM_U + lane_base + 32 * blk, f);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_gf);
            }
        }
        if (to && hp == 0) *s_abort = 1;
    } else if (!carry) {
        // =============================== prep group ===============================
        const int p = tid - NGRP;
        bool to = false;  // a wait of this thread timed out
        auto wait_ok = [&](uint64_t *bar, uint32_t parity) {
            if (!bw(bar, parity)) to = true;
        };
        for (int c = 0; c < nvalid; ++c) {
            const uint32_t par = c & 1;
            float *vec = vecs + par * NVEC * 64;
            float *vBeta = vec + V_BETA * 64, *vEG = vec + V_EG * 64;
            float *vRk = vec + V_RK * 64, *vRq = vec + V_RQ * 64, *vCw = vec + V_CW * 64;
            uint8_t *pm = sm + (par ? OFF_PM1 : OFF_PM0);
            const int n = min(C, L - c * C);
            // Pm buffer `par` and the norm vectors of set `par` were last read for chunk c-2, before its MMA2
            // Pm buffer `par` and the norm vectors of set `par` were last read for chunk c-2, before its MMA2;
            // the control warp waited for that MMA2 before it wrote chunk c's gate vectors, ahead of H0.
            PHASE(26);
            if (n < C) {  // padding rows of the last chunk's K and Q: zero them so no padding value reaches a product
                wait_ok(bar_ld, par);
                for (int e = p; e < (C - n) * 32; e += NGRP) {
                    const int r = n + e / 32, k = e % 32, tile = k >> 3;
                    const uint32_t base = (tile & 1) ? off_q(tile >> 1) : off_k(par, tile >> 1);
                    *reinterpret_cast<uint4 *>(sm + base + r * 128 + (k & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            // H0: the control warp (which wrote chunk c's gate vectors during chunk c-1) issues the Gram
            if (named_sync_or(BAR_PCTL, NPC, to)) break;
            PHASE(0);
            wait_ok(bar_gp, par);
            tc_fence_after();
            PHASE(3);
            // Each thread takes its Gram row's 32 columns of [K; Q] K^T (lanes 0..63: k_t.k_s, lanes
            // 64..127: q_t.k_s); the blocks wholly above the diagonal are never read.  The diagonal
            // gives |k_t|^2 and (from the q_t.q_s columns) |q_t|^2.
            // Even chunks: TMEM lanes 0..63 hold the k rows and 64..127 the q rows, columns 0..63 the k
            // columns; odd chunks ([Q; K]) swap both.  A warp of the "k role" builds rows of A, one of the
            // "q role" rows of Pm; qa is the 32-row block of the chunk its lanes cover.
            const bool krole = (q4 >> 1) == (int)par;
            const int qa = q4 & 1, kcol = par ? 64 : 0, qcol = par ? 0 : 64;
            const bool need = !(qa == 0 && hf == 1);
            if (qa == hf) {
                // |k_t|^2 / |q_t|^2 is the diagonal entry of this thread's row: entry `lane` of the 32 columns
                // its warp loads
                float d32[32];
                tmem_ld32(tmem + TM_GPW + lane_base + (krole ? kcol : qcol) + 32 * hf, d32);
                tmem_ld_wait();
                float d = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) d = (j == lane) ? d32[j] : d;
                const int t = row & 63;
                const float r = t < n ? (a.l2norm ? rsqrtf(d + a.eps) : 1.f) : 0.f;
                if (krole) {
                    vRk[t] = r;
                    vec[V_TAIL * 64 + t] = vec[V_ET * 64 + t] * r;
                    vCw[t] = vBeta[t] * vEG[t] * r;
                    // padding rows have 1/|k| = 0, so their lambda is +inf and their entries vanish
                    vec[V_LAM * 64 + t] = vec[V_G2 * 64 + t] - lg2_approx(r);
                } else {
                    vRq[t] = a.scale * r;
                    vec[V_XS * 64 + t] = vEG[t] * a.scale * r;
                }
            }
            // the TT area (which takes plain A next) is free once the W/U MMAs of chunk c-1 completed
            if (p == 0 && c > 0) wait_ok(bar_wu, (c - 1) & 1);
            named_sync(BAR_PREP, NGRP);
            PHASE(4);
            // A rows (k role, fp32 for the solve) and Pm rows (q role, bf16 operand of the carry's o MMA), with
            // the decay e^{G_t - G_s} taken per entry
            {
                const int t = row & 63;
                if (need) {
                    float v[32];
                    tmem_ld32(tmem + TM_GPW + lane_base + kcol + 32 * hf, v);
                    const float g2t = vec[V_G2 * 64 + t];
                    // row factor: beta_t / |k_t| for A, scale / |q_t| for Pm (zero past the length)
                    const float rf = t < n ? (krole ? vBeta[t] * vRk[t] : vRq[t]) : 0.f;
                    const float4 *lam4 = reinterpret_cast<const float4 *>(vec + V_LAM * 64 + 32 * hf);
                    tmem_ld_wait();
                    if (kGate) {
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 l = lam4[j4];
                            v[4 * j4 + 0] *= rf * ex2_approx(g2t - l.x);
                            v[4 * j4 + 1] *= rf * ex2_approx(g2t - l.y);
                            v[4 * j4 + 2] *= rf * ex2_approx(g2t - l.z);
                            v[4 * j4 + 3] *= rf * ex2_approx(g2t - l.w);
                        }
                    } else {  // no decay: the column factor 1/|k_s| alone (0 past the length)
                        const float4 *rk4 = reinterpret_cast<const float4 *>(vRk + 32 * hf);
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 l = rk4[j4];
                            v[4 * j4 + 0] *= rf * l.x;
                            v[4 * j4 + 1] *= rf * l.y;
                            v[4 * j4 + 2] *= rf * l.z;
                            v[4 * j4 + 3] *= rf * l.w;
                        }
                    }
                    if (krole && hf == qa) {
                        // a diagonal 32 x 32 block, plain (entries on or above the diagonal are never read)
                        float *ap = reinterpret_cast<float *>(sm + OFF_AP) + pl(t, 0);
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4)
                            *reinterpret_cast<float4 *>(ap + 4 * j4) =
                                make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
                    } else if (krole) {  // A21 (rows 32..63, columns 0..31), operand of the 32 -> 64 merge
                        float *ap = reinterpret_cast<float *>(sm + OFF_A21) + (t - 32) * SP;
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4)
                            *reinterpret_cast<float4 *>(ap + 4 * j4) =
                                make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = (32 * hf + j <= t) ? v[j] : 0.f;
#pragma unroll
                        for (int c8 = 0; c8 < 4; ++c8)
                            *reinterpret_cast<uint4 *>(pm + blk_off(t, 32 * hf + 8 * c8)) = pack8<T>(&v[8 * c8]);
                    }
                } else if (!krole) {  // Pm rows 0..31, columns 32..63: above the diagonal
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(pm + blk_off(t, 32 + 8 * c8)) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_PREP, NGRP);
            PHASE(5);
            // ---- a3: T = (I + A)^{-1} and the bf16 operand TT = [T diag(beta); T diag(c_W)] ----
            // T = [[T11, 0], [T21, T22]]: the diagonal 32 x 32 blocks on the CUDA cores (solve_diag16_merge), then
            // T21 = -T22 (A21 T11) by the eight prep warps, one 16 x 8 tile each of X = A21 T11 and then of T21,
            // on warp-level tf32 MMAs; the diagonal blocks go into TT meanwhile.
            solve_diag16_merge(reinterpret_cast<const float *>(sm + OFF_AP), reinterpret_cast<float *>(sm + OFF_TP),
                               reinterpret_cast<float *>(sm + OFF_XP), p);
            PHASE(12);
            const float *tpl = reinterpret_cast<const float *>(sm + OFF_TP);
            float *xm = reinterpret_cast<float *>(sm + OFF_XM);
            const int pw = p >> 5, rt = pw >> 2, ct = pw & 3, gq = lane >> 2, iq = lane & 3;
            {
                // X tile (rows 16 rt.., columns 8 ct..); T11 is lower triangular, so k-steps before ct add nothing
                float d[4];
                gemm32_tile(d, reinterpret_cast<const float *>(sm + OFF_A21), tpl, rt, ct, ct, 4, lane);
                *reinterpret_cast<float2 *>(xm + (16 * rt + gq) * SP + 8 * ct + 2 * iq) = make_float2(d[0], d[1]);
                *reinterpret_cast<float2 *>(xm + (16 * rt + gq + 8) * SP + 8 * ct + 2 * iq) = make_float2(d[2], d[3]);
            }
            {
                // TT rows of the diagonal blocks (and zeros above them), while other warps finish X
                const int blk = p >> 7, t = (p >> 2) & 31, c8 = p & 3, R = 32 * blk + t, col = 32 * blk + 8 * c8;
                const float *tp = tpl + pl(R, col);
                const float4 u0 = *reinterpret_cast<const float4 *>(tp), u1 = *reinterpret_cast<const float4 *>(tp + 4);
                const float tv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                float fb[8], fw[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    fb[i] = tv[i] * vBeta[col + i];
                    fw[i] = tv[i] * vCw[col + i];
                }
                *reinterpret_cast<uint4 *>(sm + OFF_TT + blk_off(R, col)) = pack8<T>(fb);
                *reinterpret_cast<uint4 *>(sm + OFF_TT + blk_off(64 + R, col)) = pack8<T>(fw);
                // zeros: TT rows 0..31 and 64..95, columns 32..63 (above the diagonal)
                const int Rz = (p >> 2) + ((p >> 7) << 5), cz = 4 + (p & 3);
                *reinterpret_cast<uint4 *>(sm + OFF_TT + blk_off(Rz, 8 * cz)) = make_uint4(0, 0, 0, 0);
            }
            named_sync(BAR_PREP, NGRP);
            PHASE(13);
            {
                // T21 tile = -(T22 X): T22 is lower triangular, so rows 16 rt.. need k-steps up to 2 rt + 1 only;
                // straight into TT rows 32 + r (times beta_s) and 96 + r (times c_W,s), columns s < 32
                float d[4];
                gemm32_tile(d, tpl + 32 * SP, xm, rt, ct, 0, 2 * rt + 2, lane);
                const int s0 = 8 * ct + 2 * iq;
                const float b0 = vBeta[s0], b1 = vBeta[s0 + 1], w0 = vCw[s0], w1 = vCw[s0 + 1];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = 16 * rt + gq + 8 * hh;
                    const float t0 = -d[2 * hh], t1 = -d[2 * hh + 1];
                    *reinterpret_cast<uint32_t *>(sm + OFF_TT + blk_off(32 + r, s0)) = TcT<T>::pack2(t0 * b0, t1 * b1);
                    *reinterpret_cast<uint32_t *>(sm + OFF_TT + blk_off(96 + r, s0)) = TcT<T>::pack2(t0 * w0, t1 * w1);
                }
            }
            PHASE(14);
            PHASE(6);
            PHASE(7);
            if (n < C) {  // padding rows of the last chunk's V, once it has landed
                wait_ok(bar_ldv, par);
                for (int e = p; e < (C - n) * 16; e += NGRP) {
                    const int r = n + e / 16, k = e % 16;
                    *reinterpret_cast<uint4 *>(sm + OFF_V + (k >> 3) * 8192 + r * 128 + (k & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            // hand the chunk over: the carry group issues W and U from TT (it owns TMEM R and U, so they are
            // free in its own program order), waits for them and moves W into A1
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_PREP, NGRP);
            if (p == 0) mbar_arrive(bar_a1);
            PHASE(8);
        }
        if (to && p == 0) *s_abort = 1;
    } else {
        // =============================== carry group ==============================
        bool to = false;  // a wait of this thread timed out
        bool stop = false;
        auto wait_ok = [&](uint64_t *bar, uint32_t parity) {
            if (!bw(bar, parity)) to = true;
        };
        // warp 0 issues the carry's MMAs as a whole warp, one elected lane issuing, with warp-uniform operand
        // addresses (a lone divergent lane issues several times slower)
        const uint32_t tmu = __shfl_sync(0xffffffffu, tmem, 0), sbu = __shfl_sync(0xffffffffu, sbase, 0);
        for (int c = 0; c < nvalid; ++c) {
            const uint32_t par = c & 1;
            const float *vec = vecs + par * NVEC * 64;
            if (!bw(bar_a1, par)) to = true;
            wait_ok(bar_cq, par);
            if (named_sync_or(BAR_CARRY, NGRP, to)) { stop = true; break; }
            PHASE(21);
            if (tid == 0) mbar_arrive(bar_go);
            if (warp == 0) {  // a4: W (rows 64..127 of TT K, into TMEM R) and U (rows 0..63 of TT V)
                if (!__all_sync(0xffffffffu, bw(bar_ldv, par))) to = true;
                tc_fence_after();
                const uint32_t id = idesc_t<T>(128, 128, false, true);
                if (elect_one_sync()) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t ad = sdesc_sw128(sbu + OFF_TT + k * 32, 16, 1024);
                        mma_bf16(tmu + TM_R, ad, sdesc_sw128(sbu + off_k(par, 0) + k * 2048, KQ_BLK, 1024), id, k > 0);
                        mma_bf16(tmu + TM_U, ad, sdesc_sw128(sbu + OFF_V + k * 2048, 8192, 1024), id, k > 0);
                    }
                    mma_commit(bar_wu);
                }
                __syncwarp();
            }
            wait_ok(bar_wu, par);
            tc_fence_after();
            PHASE(22);
            if (q4 >= 2) {  // W rows (TMEM lanes 64..127 of R) -> rows 0..63 of A1
                const int t = row - 64;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float w[32];
                    tmem_ld32(tmem + TM_R + lane_base + 64 * hf + 32 * half, w);
                    tmem_ld_wait();
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(sm + OFF_A1 + hf * 16384 + blk_off(t, 32 * half + 8 * c8)) =
                            pack8<T>(&w[8 * c8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_CARRY, NGRP);
            tc_fence_after();
            PHASE(16);
            const int n = (int)vec[V_N * 64];
            const float eL = vec[V_EG * 64 + C - 1];
            // ---- R = [W; Q] S ----
            if (warp == 0) {
                const uint32_t id = idesc_t<T>(128, 128, false, true);
                if (elect_one_sync()) {
                    TIMED(23, {
                        _Pragma("unroll")
                        for (int k = 0; k < 8; ++k) {
                            const uint64_t ad = sdesc_sw128(sbu + OFF_A1 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(sbu + OFF_S + k * 2048, 16384, 1024);
                            mma_bf16(tmu + TM_R, ad, bd, id, k > 0);
                        }
                        mma_commit(bar_m1);
                    });
                }
                __syncwarp();
            }
            // S <- e^{G_last} S in TMEM, onto which MMA2 accumulates (for c > 0 the previous chunk's
            // epilogue already wrote the scaled state back)
            if (kGate && c == 0) {
#pragma unroll 1
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
            }
            wait_ok(bar_m1, par);
            if (tid == 0 && c + 1 < nvalid) load_carry_q(c + 1);  // the Q rows of A1 are read
            if (tid == kStorer) bulk_wait_read0();  // the previous out tile (same buffer as v_new) is read
            tc_fence_before();
            if (named_sync_or(BAR_CARRY, NGRP, to)) { stop = true; break; }
            tc_fence_after();
            PHASE(17);
            if (q4 < 2) {  // v_new = U - W S for token t, dv columns [64 hf, +64)
                const int t = row;
#pragma unroll 1
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
                            pack8<T>(&u[8 * c8]);
                }
            } else {  // rows of Q S: scale by e^{G_t} scale / |q_t| before Pm v_new accumulates onto them
                const float xs = vec[V_XS * 64 + row - 64];
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float r[32];
                    const uint32_t ta = tmem + TM_R + lane_base + 64 * hf + 32 * half;
                    tmem_ld32(ta, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] *= xs;
                    tmem_st32(ta, r);
                }
                tmem_st_wait();
            }
            // e^{G_last} of the next chunk (for the state written back after MMA2), read before this chunk's MMA2:
            // the control warp cannot get two chunks ahead of it then
            const bool more = c + 1 < nvalid;
            float eLn = 1.f;
            if (more) {
                wait_ok(bar_vr, par);
                eLn = vecs[(par ^ 1) * NVEC * 64 + V_EG * 64 + C - 1];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_sync_or(BAR_CARRY, NGRP, to)) { stop = true; break; }
            tc_fence_after();
            PHASE(18);
            // ---- S += K~^T v_new ;  R[64:128] += Pm v_new ----
            if (warp == 0) {
                if (!__all_sync(0xffffffffu, bw(bar_kt, par))) to = true;  // K~ of this chunk (helper warps)
                tc_fence_after();
                const uint32_t id_s = idesc_t<T>(128, 128, true, true);
                const uint32_t id_o = idesc_t<T>(128, 128, false, true);
                const uint32_t pm_rows = sbu + (par ? OFF_PM1 : OFF_PM0) - 8192;
                if (elect_one_sync()) {
                    TIMED(24, {
                        _Pragma("unroll")
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t bd = sdesc_sw128(sbu + OFF_VO + k * 2048, 8192, 1024);
                            mma_bf16(tmu + TM_S, sdesc_sw128(sbu + OFF_KT + k * 2048, 8192, 1024), bd, id_s, 1);
                        }
                        _Pragma("unroll")
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t bd = sdesc_sw128(sbu + OFF_VO + k * 2048, 8192, 1024);
                            mma_bf16(tmu + TM_R, sdesc_sw128(pm_rows + k * 32, 16, 1024), bd, id_o, 1);
                        }
                        mma_commit(bar_m2);
                        mma_commit(bar_pf + par);
                    });
                }
                __syncwarp();
            }
            wait_ok(bar_m2, par);
            if (tid == 0 && c + 1 < nvalid) load_carry_k(c + 1);  // the raw K tile is read
            tc_fence_after();
            if (named_sync_or(BAR_CARRY, NGRP, to)) { stop = true; break; }
            PHASE(19);
            // ---- S (fp32, TMEM) -> bf16 operand tile, and back to TMEM scaled by e^{G_last} of the next
            // chunk (its gate vectors were written before this chunk was handed over);  o rows -> out tile ----
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float v[32];
                const uint32_t ta = tmem + TM_S + lane_base + 64 * hf + 32 * half;
                tmem_ld32(ta, v);
                tmem_ld_wait();
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(sm + OFF_S + hf * 16384 + blk_off(row, 32 * half + 8 * c8)) =
                        pack8<T>(&v[8 * c8]);
                if (kGate && more) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] *= eLn;
                    tmem_st32(ta, v);
                }
            }
            if (kGate && more) tmem_st_wait();
            if (q4 >= 2) {
                const int t = row - 64;
                // epilogue: the row's squared norm from its two halves (this thread and the one of the other hf
                // warp with the same lane), then o * inv * (norm_w * silu(z)) for this thread's 64 columns, the
                // gate factors read from TMEM where the helper warps put them
                const bool epi = a.epi_z != nullptr;
                float inv = 1.f;
                if (epi) {
                    float ss = 0.f;
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        float o[32];
                        tmem_ld32(tmem + TM_R + lane_base + 64 * hf + 32 * half, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) ss = fmaf(o[j], o[j], ss);
                    }
                    float *eps2 = reinterpret_cast<float *>(sm + OFF_EPI);
                    eps2[hf * 64 + t] = ss;
                    named_sync(BAR_EPI, 128);
                    inv = rsqrtf((eps2[t] + eps2[64 + t]) * (1.f / D) + a.epi_eps);
                    wait_ok(bar_gf, par);  // the gate factors w silu(z) of this chunk's rows (helper warps)
                    tc_fence_after();
                }
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tmem_ld32(tmem + TM_R + lane_base + 64 * hf + 32 * half, o);
                    tmem_ld_wait();
                    if (epi) {
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            float gfv[16];
                            tmem_ld16(tmem + TM_U + lane_base + 64 * hf + 32 * half + 16 * q, gfv);
                            tmem_ld_wait();
#pragma unroll
                            for (int j = 0; j < 16; ++j) o[16 * q + j] *= inv * gfv[j];
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = t < n ? o[j] : 0.f;
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(sm + OFF_VO + hf * 8192 + blk_off(t, 32 * half + 8 * c8)) =
                            pack8<T>(&o[8 * c8]);
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
                T *fs = reinterpret_cast<T *>(a.final_state) + ((size_t)bh * D + row) * D + 64 * hf;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(tmem + TM_S + lane_base + 64 * hf + 32 * half, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(fs + 32 * half + 8 * c8) = pack8<T>(&v[8 * c8]);
                }
            }
        }
        if (tid == kStorer) bulk_wait0();
    }
    // drain: every copy and MMA the CTA issued has completed before its shared memory and TMEM are released
    // (normally each was consumed already; after a stop some may still be in flight)
    if (control && lane == 1) {
        if (n_ld) mbar_wait_ns(bar_ld, (n_ld - 1) & 1, kDrainWaitNs);
        if (n_ldv) mbar_wait_ns(bar_ldv, (n_ldv - 1) & 1, kDrainWaitNs);
    }
    if (tid == 0) {
        if (n_cq) mbar_wait_ns(bar_cq, (n_cq - 1) & 1, kDrainWaitNs);
        if (n_ck) mbar_wait_ns(bar_ck, (n_ck - 1) & 1, kDrainWaitNs);
    }
    if (control && lane == 0) {
        mma_commit(bar_dr);
        mbar_wait_ns(bar_dr, 0, kDrainWaitNs);
    }
    if (warp == 0) {  // the carry's MMAs were issued by the lane of warp 0 that elect.sync picks
        if (elect_one_sync()) mma_commit(bar_dr);
        __syncwarp();
        mbar_wait_ns(bar_dr, 0, kDrainWaitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *s_abort) raise_device_error(a.err, GDR_DEVERR_TIMEOUT);
#ifdef GDR_PHASE_TIMERS
    if (blockIdx.x == 0 && tid < 64) g_phase[tid] += s_phase_[tid];
#endif
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// (D, S, Z) tensor of 2-byte elements (bf16 or fp16), 64 x 64 boxes, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int S, long long Z, CUtensorMapDataType type) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)Z};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
    cuuint32_t box[3] = {64, 64, 1}, es[3] = {1, 1, 1};
    return enc(m, type, 3, const_cast<void *>(base), dims, strides, box, es,
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

bool chunk_tc_supported(int Dk, int Dv, gdr_dtype dt, int S) {
    return (dt == GDR_BF16 || dt == GDR_F16) && Dk == D && Dv == D && S > 0;
}

namespace {
template <typename T, bool kGate>
cudaError_t launch_tc_t(const ChunkArgs &ca, cudaStream_t stream) {
    constexpr CUtensorMapDataType ty = TcT<T>::kMap;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, ca.q, ca.S, (long long)ca.B * ca.Nk, ty) ||
        !make_map(&mk, ca.k, ca.S, (long long)ca.B * ca.Nk, ty) ||
        !make_map(&mv, ca.v, ca.S, (long long)ca.B * ca.Nv, ty) ||
        !make_map(&mo, ca.out, ca.S, (long long)ca.B * ca.Nv, ty))
        return cudaErrorInvalidValue;
    TcArgs a{};
    a.beta = ca.beta; a.g = ca.g; a.initial_state = ca.initial_state; a.lengths = ca.lengths; a.scale = ca.scale;
    a.B = ca.B; a.Nk = ca.Nk; a.Nv = ca.Nv; a.S = ca.S; a.final_state = ca.final_state;
    a.l2norm = ca.l2norm; a.eps = ca.eps; a.beta_logits = ca.beta_logits; a.A_log = ca.A_log;
    a.dt_bias = ca.dt_bias; a.err = ca.err;
    a.epi_z = ca.epi_z; a.epi_w = ca.epi_w; a.epi_eps = ca.epi_eps;
    a.wait_ns = chunk_wait_ns();
    static LaunchCache plain(reinterpret_cast<const void *>(chunk_tc_kernel<T, kGate, false>));
    static LaunchCache ordered(reinterpret_cast<const void *>(chunk_tc_kernel<T, kGate, true>));
    const long long blocks = (long long)ca.B * ca.Nv;
    if (blocks == 0) return cudaSuccess;
    // longest sequences first only when the chains do not all start at once
    bool order = false;
    if (ca.lengths && ca.B > 1 && ca.B <= kRankMaxB) {
        int resident = 0;
        cudaError_t e = ordered.resident_grid(NT, (int)SMEM_BYTES, &resident);
        if (e != cudaSuccess) return e;
        order = blocks > resident;
    }
    cudaError_t e = (order ? ordered : plain).allow_smem((int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (order)
        chunk_tc_kernel<T, kGate, true><<<(unsigned)blocks, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, a);
    else
        chunk_tc_kernel<T, kGate, false><<<(unsigned)blocks, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, a);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_chunk_tc(const ChunkArgs &ca, gdr_dtype dt, cudaStream_t stream) {
    const bool gate = ca.g != nullptr;
    if (dt == GDR_F16) return gate ? launch_tc_t<__half, true>(ca, stream) : launch_tc_t<__half, false>(ca, stream);
    return gate ? launch_tc_t<__nv_bfloat16, true>(ca, stream) : launch_tc_t<__nv_bfloat16, false>(ca, stream);
}

}  // namespace gdr
