// chunk_wy.cu -- chunked prefill of the gated delta rule on the sm_100a tensor cores (bf16 or fp16 in and out,
// Dk = Dv = 128, chunk C = 64), in two kernels: the schedule for few chains (fewer (b, value head) pairs than a
// third of the SMs), where the one-kernel schedule of chunk_tc.cu would leave most SMs idle while its chains
// solve each chunk's WY system serially.
//
// The chunked (WY / UT transform) form of torch_chunk_gated_delta_rule (blog "gated-delta-net" page, steps
// 1-8).  Everything that does not depend on the state is independent per chunk, so it runs first, over all
// chunks at once; only the state carry is serial.
//
//   wy_kernel (one CTA per (sequence, key head, chunk), every SM, several CTAs per SM):
//     a0  the fused prologue: beta = sigmoid(b), g = -e^{A_log} softplus(a + dt_bias), 1/|k| (eps inside the
//         root, from the diagonal of the Gram)
//     a1  G_t = cumulative log-gate inside the chunk (tokens past the length count 0)
//     a2  Gram K K^T of the raw keys (warp-level bf16/fp16 tensor-core MMAs, fp32 accumulation)
//     a3  A = strictLower(beta_t k_t.k_s e^{G_t-G_s}) with unit keys;  T = (I + A)^{-1}: 16 x 16 diagonal
//         blocks by forward substitution, the 16 -> 32 merges on the CUDA cores, the 32 -> 64 merge on tf32
//         warp MMAs
//     and writes, per (b, value head, chunk), into the caller's workspace: T' = T diag(beta) (16-bit,
//     row-major 64 x 64) and six vectors of 64 floats (e^G, e^G/|k|, e^{G_last-G}/|k|, G log2 e,
//     G log2 e - log2(1/|k|), and [e^{G_last}, valid count]).
//
//   chain_kernel (one CTA per (b, value head) chain): per chunk, with the state held TRANSPOSED in tensor
//   memory (lane = value column j, columns = key row i, fp32) so that the state and v_new are the A operand
//   of the tensor core straight from TMEM:
//     a4  U^T = V^T T'^T                                     tcgen05 M=128 (dv) N=64 (t) K=64
//         W^T = K^T (T' diag(e^G/|k|))^T                     tcgen05 M=128 (dk) N=64 K=64
//     a5  v_new^T = U^T - S^T W^T                            tcgen05, A = S^T (bf16 copy in TMEM)
//         o^T     = S^T Q~^T + v_new^T Pm^T                  Q~ = diag(e^G) Q, Pm = causal
//                                                            q_t.k_s/|k_s| e^{G_t-G_s}; the row factor
//                                                            scale/|q_t| is applied to o afterwards
//         S^T     = e^{G_last} S^T + (v_new diag(c))^T K     c_t = e^{G_last-G_t}/|k_t| folded into the
//                                                            16-bit copy of v_new (A from TMEM), K raw
//     a6  o -> dtype -> TMA store (padding rows and chunks zero); the final state written once from TMEM.
//   The serial chain per chunk is MMA -> v_new (TMEM -> registers -> TMEM) -> MMA -> S (TMEM -> registers ->
//   TMEM): no shared-memory round trip and no proxy fence on it.  The other products run on the tensor pipe
//   while the carry warps convert.
//
// Warp roles of chain_kernel: warps 0-7 carry (the two conversions of the chain, the initial and final
// state), 8-11 out (1/|q| and Q~ of the next chunk; o rows -> out tile, the optional gated RMSNorm epilogue,
// TMA stores), 12-15 prep (W^T, Pm and T' diag(e^G/|k|) of the next chunk, padding rows), 16 MMA issue (one
// thread issues every tcgen05.mma; the products of the next chunk go in when their operands are ready, never
// ahead of the chain's own), 17 TMA loads.  Hand-offs are mbarriers; every wait is bounded by elapsed time and gives up
// when another group has stopped, after which the CTA drains its own copies and MMAs, sets the timeout bit
// of the device error word, releases TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdr {
using namespace sm100;

// The first bounded wait of the chain kernel that ran out since the word was last read (0: none): bit 31 set,
// the warp in bits 24-29, the barrier in bits 16-23, its phase parity in bit 15, the CTA in bits 0-14.
namespace {
__device__ unsigned int g_timeout_site = 0;
}

#ifdef GDR_PHASE_TIMERS
// Development aid, compiled only with -DGDR_PHASE_TIMERS (never in the library the package builds): cycles the
// first thread of each role of CTA 0 spends blocked in each barrier wait, [role][barrier] with roles carry, out,
// prep, MMA, TMA; then the CTA's total cycles and its chunk count.  Read by gdr_phase_timers_read.
constexpr int kTimerSlots = 5 * 36 + 2;
__device__ unsigned long long g_phase[kTimerSlots];
// and a timeline of chunks kEvC0 .. kEvC0 + kEvN - 1 of CTA 0: clock64 at 16 hand-off / issue events per chunk
constexpr int kEvC0 = 8, kEvN = 8, kEvK = 16;
__device__ long long g_events[kEvN * kEvK];
__device__ long long g_seen[kEvN * 16];  // when the MMA thread first saw each hand-off of a round (bit index)
#define EVENT(chunk, k)                                                                       \
    do {                                                                                      \
        if (blockIdx.x == 0 && (chunk) >= kEvC0 && (chunk) < kEvC0 + kEvN)                    \
            g_events[((chunk) - kEvC0) * kEvK + (k)] = clock64();                             \
    } while (0)
#else
#define EVENT(chunk, k) \
    do {                \
    } while (0)
#endif
#ifdef GDR_PHASE_TIMERS
#define SEEN_EVENT(chunk, bitv)                                                                   \
    do {                                                                                           \
        if (blockIdx.x == 0 && (chunk) >= kEvC0 && (chunk) < kEvC0 + kEvN)                         \
            g_seen[((chunk) - kEvC0) * 16 + (31 - __clz(bitv))] = clock64();                       \
    } while (0)
#else
#define SEEN_EVENT(chunk, bitv) \
    do {                        \
    } while (0)
#endif

namespace {

constexpr int C = 64, D = 128;
constexpr uint64_t kDrainWaitNs = 1000000000ull;    // waits for the CTA's own copies and MMAs when it stops

// ---- workspace (per (b, value head, chunk): T' then, in a second region, the vectors) ----
constexpr size_t kTpBytes = (size_t)C * C * 2;
constexpr int kNumVec = 6;
constexpr size_t kVecBytes = (size_t)kNumVec * C * 4;
// V_EG = e^{G_t}; V_CW = e^{G_t}/|k_t| (column factor of T' for W); V_CT = e^{G_last - G_t}/|k_t| (row factor
// of K~); V_G2 = G_t log2 e; V_LAM = V_G2 - log2(1/|k_t|) (so that e^{G_t - G_s}/|k_s| = 2^{V_G2[t] - V_LAM[s]});
// V_MISC[0] = e^{G_last}, V_MISC[1] = the chunk's valid-token count.  Entries past the length: 1/|k| = 0.
enum { V_EG = 0, V_CW, V_CT, V_G2, V_LAM, V_MISC };

__host__ __device__ constexpr size_t vec_offset(size_t nch) { return nch * kTpBytes; }

__device__ __forceinline__ uint32_t blk_off(uint32_t row, uint32_t col) {  // within a 128-B-row swizzled block
    return (row >> 3) * 1024u + sw128_offset(row & 7u, col);
}

// silu(x) = x sigmoid(x).  For bf16 outputs sigmoid(x) = (1 + tanh(x / 2)) / 2 with tanh on the special-function
// unit (PTX tanh.approx, relative error about 2^-11, below the bf16 rounding of 2^-9 that follows); for fp16
// outputs (rounding 2^-11) x / (1 + e^{-x}) with the fast division (about 1e-6).
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
// either, A and B of the same type).  TMA data type, descriptor operand format, pairs packed / unpacked, and the
// warp-level MMA of the Gram.
template <typename T> struct TcT;
template <> struct TcT<__nv_bfloat16> {
    static constexpr CUtensorMapDataType kMap = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static constexpr uint32_t kFmt = 1;
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }
    static __device__ __forceinline__ float2 unpack2(uint32_t u) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
    }
    // D (16 x 8, fp32) += A (16 x 16) B (16 x 8): m16n8k16, operands in the mma.sync fragment layout
    static __device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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
    static __device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

// four 8 x 8 16-bit matrices from shared memory into the mma.sync fragment layout (lane l supplies the address of
// row l % 8 of matrix l / 8)
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// ============================================================================================================
// The WY solve T = (I + A)^{-1} (A strictly lower triangular, 64 x 64, fp32), by 256 threads.
// ============================================================================================================

constexpr int SP = 36;  // row stride (floats) of the plain 32 x 32 blocks: 16-byte aligned rows
constexpr int BAR_SOLVE = 1;

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

// T = (I + A)^{-1}, first part, by 256 threads p: the two 32 x 32 diagonal blocks T11 and T22 (A strictly lower;
// its diagonal blocks plain in sA).  The four 16 x 16 diagonal blocks by forward substitution (one column per
// thread, zeros above the diagonal), then for each 32-block the lower-left 16 x 16 block T21 = -T22 (A21 T11)
// with the CUDA cores.
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
    named_sync(BAR_SOLVE, 256);
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
    named_sync(BAR_SOLVE, 256);
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float t = tb[(16 + r) * SP + 16 + k];
        const float2 xx = *reinterpret_cast<const float2 *>(sX + (blk * 16 + k) * SP + c2);
        y0 = fmaf(t, xx.x, y0);
        y1 = fmaf(t, xx.y, y1);
    }
    *reinterpret_cast<float2 *>(tb + (16 + r) * SP + c2) = make_float2(-y0, -y1);
    named_sync(BAR_SOLVE, 256);
}

// ============================================================================================================
// wy_kernel: per (b, key head, chunk), for each value head of the group: T' = (I + A)^{-1} diag(beta) and the
// chunk's vectors, into the workspace.
// ============================================================================================================

struct WyArgs {
    const void *k;
    const void *beta;
    const float *g;
    const int32_t *lengths;
    int B, Nk, Nv, S, NC;
    int l2norm;
    float eps;
    int beta_logits;
    const float *A_log, *dt_bias;
    void *tp;    // workspace: T' (16-bit), (B Nv NC) x 64 x 64
    float *vec;  // workspace: vectors, (B Nv NC) x kNumVec x 64
};

constexpr int WY_THREADS = 256;
constexpr int KST = 136;  // K tile row stride in elements (272 B: the 8 rows of an ldmatrix hit distinct banks)
constexpr int GST = 65;   // Gram row stride (floats)
constexpr uint32_t WY_OFF_K = 0;                             // 64 x KST 16-bit; after the Gram: A (diag blocks), X
constexpr uint32_t WY_OFF_G = 17408;                         // Gram, 64 x GST fp32
constexpr uint32_t WY_OFF_TP = WY_OFF_G + 64 * GST * 4;      // T diagonal blocks, 64 x SP
constexpr uint32_t WY_OFF_A21 = WY_OFF_TP + 64 * SP * 4;     // A21, then T21: 32 x SP
constexpr uint32_t WY_OFF_XM = WY_OFF_A21 + 32 * SP * 4;     // X = A21 T11 of the 32 -> 64 merge: 32 x SP
constexpr uint32_t WY_OFF_VEC = WY_OFF_XM + 32 * SP * 4;     // kNumVec vectors, then beta, then 1/|k|
constexpr uint32_t WY_SMEM = WY_OFF_VEC + (kNumVec + 2) * 64 * 4;
static_assert(64 * KST * 2 <= WY_OFF_G, "K tile");
static_assert(64 * SP * 4 + 32 * SP * 4 <= WY_OFF_G, "A diagonal blocks and the merge scratch fit in the K tile");
constexpr int WV_BETA = kNumVec, WV_RK = kNumVec + 1;

template <typename T, bool kGate>
__global__ void __launch_bounds__(WY_THREADS, 4) wy_kernel(const WyArgs a) {
    extern __shared__ __align__(16) uint8_t wsm[];
    T *Ks = reinterpret_cast<T *>(wsm + WY_OFF_K);
    float *sAP = reinterpret_cast<float *>(wsm + WY_OFF_K);  // reuses the K tile after the Gram
    float *sXP = sAP + 64 * SP;
    float *Gs = reinterpret_cast<float *>(wsm + WY_OFF_G);
    float *sTP = reinterpret_cast<float *>(wsm + WY_OFF_TP);
    float *sA21 = reinterpret_cast<float *>(wsm + WY_OFF_A21);
    float *sXM = reinterpret_cast<float *>(wsm + WY_OFF_XM);
    float *sv = reinterpret_cast<float *>(wsm + WY_OFF_VEC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x % a.NC;
    const int rest = blockIdx.x / a.NC;
    const int kh = rest % a.Nk, b = rest / a.Nk;
    int L = a.lengths ? a.lengths[b] : a.S;
    if (L < 0 || L > a.S) L = 0;  // the chain kernel reports the bad length
    const int n = min(C, L - c * C);
    if (n <= 0) return;

    // ---- the raw K tile (rows past the length zero) ----
    const T *kp = static_cast<const T *>(a.k) + ((size_t)(b * a.Nk + kh) * a.S + (size_t)c * C) * D;
    for (int e = tid; e < C * (D / 8); e += WY_THREADS) {
        const int t = e >> 4, c8 = e & 15;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (t < n) u = __ldg(reinterpret_cast<const uint4 *>(kp + (size_t)t * D + 8 * c8));
        *reinterpret_cast<uint4 *>(Ks + t * KST + 8 * c8) = u;
    }
    __syncthreads();

    // ---- a2: the Gram K K^T, lower 16 x 16 blocks (bi >= bj), warp-level MMAs ----
    {
        const int g = lane >> 2, i4 = lane & 3;
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8, cofs = (lane >> 4) * 8;
        for (int blk = warp; blk < 10; blk += WY_THREADS / 32) {
            const int bi = blk < 1 ? 0 : blk < 3 ? 1 : blk < 6 ? 2 : 3;
            const int bj = blk - bi * (bi + 1) / 2;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const uint32_t abase = smem_u32(Ks + (16 * bi + r) * KST + cofs);
            const uint32_t bbase = smem_u32(Ks + (16 * bj + r) * KST + cofs);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t af[4], bf[4];
                ldsm_x4(af, abase + kk * 32);
                ldsm_x4(bf, bbase + kk * 32);
                TcT<T>::mma16816(acc[0], af, bf[0], bf[2]);
                TcT<T>::mma16816(acc[1], af, bf[1], bf[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int col = 16 * bj + 8 * nt + 2 * i4;
                float *g0 = Gs + (16 * bi + g) * GST + col;
                g0[0] = acc[nt][0];
                g0[1] = acc[nt][1];
                g0[8 * GST] = acc[nt][2];
                g0[8 * GST + 1] = acc[nt][3];
            }
        }
    }
    __syncthreads();
    if (tid < C) {  // 1/|k_t| from the Gram diagonal (0 past the length)
        const float d = Gs[tid * GST + tid];
        sv[WV_RK * 64 + tid] = tid < n ? (a.l2norm ? rsqrtf(d + a.eps) : 1.f) : 0.f;
    }

    const int grp = a.Nv / a.Nk;
    for (int hh = 0; hh < grp; ++hh) {
        const int h = kh * grp + hh;
        const size_t bh = (size_t)b * a.Nv + h;
        const size_t ch = bh * a.NC + c;
        __syncthreads();  // the previous head's solve and stores are done with the shared buffers
        // ---- a0/a1: beta, the gate, the cumulative gate and the vectors (warp 0, two tokens per lane) ----
        if (warp == 0) {
            const T *bp = static_cast<const T *>(a.beta) + bh * a.S + (size_t)c * C;
            const float *gp = a.g ? a.g + bh * a.S + (size_t)c * C : nullptr;
            const float gA = (kGate && a.A_log) ? a.A_log[h] : 0.f, gB = (kGate && a.A_log) ? a.dt_bias[h] : 0.f;
            float bv[2], gv[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int t = 2 * lane + i;
                const float rb = t < n ? to_f32(bp[t]) : 0.f;
                bv[i] = t < n ? (a.beta_logits ? sigmoid_f32(rb) : rb) : 0.f;
                gv[i] = 0.f;
                if (kGate && t < n) gv[i] = a.A_log ? gate_from_raw(gp[t], gA, gB) : gp[t];
            }
            float G[2] = {0.f, 0.f}, gl = 0.f;
            if (kGate) {
                const float x1 = gv[0] + gv[1];
                float sc = x1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, sc, o);
                    if (lane >= o) sc += y;
                }
                gl = __shfl_sync(0xffffffffu, sc, 31);
                G[0] = sc - x1 + gv[0];
                G[1] = sc;
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int t = 2 * lane + i;
                const float rk = sv[WV_RK * 64 + t];
                const float eg = kGate ? __expf(G[i]) : 1.f;
                const float g2 = G[i] * 1.4426950408889634f;
                sv[V_EG * 64 + t] = eg;
                sv[V_CW * 64 + t] = eg * rk;
                sv[V_CT * 64 + t] = (kGate ? __expf(gl - G[i]) : 1.f) * rk;
                sv[V_G2 * 64 + t] = g2;
                sv[V_LAM * 64 + t] = g2 - lg2_approx(rk);  // +inf past the length: those entries vanish
                sv[V_MISC * 64 + t] = t == 0 ? (kGate ? __expf(gl) : 1.f) : (t == 1 ? (float)n : 0.f);
                sv[WV_BETA * 64 + t] = bv[i];
            }
            __syncwarp();
            float4 *vo = reinterpret_cast<float4 *>(a.vec + ch * (kVecBytes / 4));
            const float4 *vi = reinterpret_cast<const float4 *>(sv);
#pragma unroll
            for (int e = 0; e < 3; ++e) vo[lane + 32 * e] = vi[lane + 32 * e];
        }
        __syncthreads();
        // ---- a3: A (strictly lower) into the solve's plain layouts ----
        {
            const int t = tid >> 2, s0 = (tid & 3) * 16;
            if (s0 < t) {
                const float rowf = sv[WV_BETA * 64 + t] * sv[WV_RK * 64 + t];
                const float g2t = sv[V_G2 * 64 + t];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int s = s0 + j;
                    float v = 0.f;
                    if (s < t)
                        v = Gs[t * GST + s] * rowf *
                            (kGate ? ex2_approx(g2t - sv[V_LAM * 64 + s]) : sv[WV_RK * 64 + s]);
                    if ((t >> 5) == (s >> 5)) sAP[pl(t, s)] = v;
                    else sA21[(t - 32) * SP + s] = v;
                }
            }
        }
        __syncthreads();
        solve_diag16_merge(sAP, sTP, sXP, tid);
        {
            // 32 -> 64: X = A21 T11 (T11 lower triangular: k-steps before ct add nothing), then T21 = -(T22 X)
            // (T22 lower triangular: rows 16 rt.. need k-steps up to 2 rt + 1), written over A21
            const int rt = warp >> 2, ct = warp & 3, gq = lane >> 2, iq = lane & 3;
            float d[4];
            gemm32_tile(d, sA21, sTP, rt, ct, ct, 4, lane);
            *reinterpret_cast<float2 *>(sXM + (16 * rt + gq) * SP + 8 * ct + 2 * iq) = make_float2(d[0], d[1]);
            *reinterpret_cast<float2 *>(sXM + (16 * rt + gq + 8) * SP + 8 * ct + 2 * iq) = make_float2(d[2], d[3]);
            __syncthreads();
            gemm32_tile(d, sTP + 32 * SP, sXM, rt, ct, 0, 2 * rt + 2, lane);
            *reinterpret_cast<float2 *>(sA21 + (16 * rt + gq) * SP + 8 * ct + 2 * iq) = make_float2(-d[0], -d[1]);
            *reinterpret_cast<float2 *>(sA21 + (16 * rt + gq + 8) * SP + 8 * ct + 2 * iq) = make_float2(-d[2], -d[3]);
        }
        __syncthreads();
        // ---- T' = T diag(beta), 16-bit, row-major, coalesced ----
        T *tpo = static_cast<T *>(a.tp) + ch * (C * C);
        for (int e = tid; e < C * C / 8; e += WY_THREADS) {
            const int t = e >> 3, s8 = (e & 7) * 8;
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int s = s8 + j;
                float tv = 0.f;
                if (s <= t) tv = ((t >> 5) == (s >> 5)) ? sTP[pl(t, s)] : sA21[(t - 32) * SP + s];
                f[j] = tv * sv[WV_BETA * 64 + s];
            }
            *reinterpret_cast<uint4 *>(tpo + t * C + s8) = pack8<T>(f);
        }
    }
}

// ============================================================================================================
// chain_kernel: the serial carry of one (b, value head) chain.
// ============================================================================================================

constexpr int NCARRY = 256, NOUTW = 128, NPREP = 128;
constexpr int W_OUT0 = 8, W_PREP0 = 12, W_MMA = 16, W_TMA = 17, W_VLD = 18, W_SIDE = 19;
constexpr int CH_THREADS = 20 * 32;
constexpr int BAR_CARRY = 1, BAR_OUT = 2, BAR_PREP = 3;

// ---- shared memory map (bytes from a 1024-aligned base); tiles of 64 rows x 128 B, 128-byte swizzle ----
constexpr int NKQ = 3, NAX = 2;
constexpr uint32_t KQ_STAGE = 32768;                      // [Q dk 0-63 | K dk 0-63 | Q dk 64-127 | K dk 64-127]
constexpr uint32_t OFF_KQ = 0;
constexpr uint32_t OFF_V = OFF_KQ + NKQ * KQ_STAGE;       // V of one chunk: [dv 0-63 | dv 64-127]
constexpr uint32_t OFF_TPS = OFF_V + 16384;               // T' stages (K-major [t][s])
constexpr uint32_t OFF_TW = OFF_TPS + NAX * 8192;         // T' diag(e^G/|k|): B operand of the W product
// B operands of the v_new / o product, MN-major [dk][t], one 64-token block each: -W^T of even chunks, Q~^T, -W^T of
// odd chunks, so that [-W^T | Q~^T] (even) and [Q~^T | -W^T] (odd) are each one N = 128 operand.  -W^T has a buffer
// per parity (W of the next chunk is ready long before the state is); Q~^T has one, rewritten once the product that
// read it has completed.
constexpr uint32_t OFF_WT0 = OFF_TW + 8192;
constexpr uint32_t OFF_QT = OFF_WT0 + 16384;
constexpr uint32_t OFF_WT1 = OFF_QT + 16384;
constexpr uint32_t OFF_PM = OFF_WT1 + 16384;              // Pm, two buffers, K-major [t][s]
constexpr uint32_t OFF_OUT = OFF_PM + 2 * 8192;           // out tile [t][dv] (two 64-column boxes); at the start,
                                                          // the lengths of the longest-first order
constexpr uint32_t OFF_VECS = OFF_OUT + 16384;            // vector stages
constexpr uint32_t OFF_RED = OFF_VECS + NAX * kVecBytes;  // epilogue: 4 x 64 partial sums, then 64 factors
constexpr uint32_t OFF_RQ = OFF_RED + 5 * 64 * 4;         // scale / |q_t|, two chunks (out warps)
constexpr uint32_t OFF_BARS = OFF_RQ + 2 * 64 * 4;
constexpr int kNumBars = 40;
constexpr uint32_t OFF_MISC = OFF_BARS + kNumBars * 8;    // TMEM base, abort flag, selected sequence
constexpr uint32_t CH_SMEM_USED = OFF_MISC + 16;
constexpr uint32_t CH_SMEM = CH_SMEM_USED + 1024;         // + alignment slack
constexpr int kRankMaxB = 256;
static_assert(CH_SMEM <= 232448, "shared memory budget");
static_assert(kRankMaxB * 4 + 16 <= 16384, "the ordering scratch fits in the out tile");
static_assert(OFF_TPS % 1024 == 0 && OFF_TW % 1024 == 0 && OFF_WT0 % 1024 == 0 && OFF_QT % 1024 == 0 &&
                  OFF_WT1 % 1024 == 0 && OFF_PM % 1024 == 0 && OFF_OUT % 1024 == 0,
              "swizzle atoms");

// TMEM columns (128 lanes, lane = value column j of S^T, v_new^T and o^T; key row of W^T; token row of the Gram):
// [o^T of odd chunks | v_new^T | o^T of even chunks] (so that the v_new / o product writes 128 adjacent columns),
// S^T fp32, its 16-bit copy, W^T, the Gram [Q; K] K^T.  v_new^T's two 16-bit copies (plain for o, scaled by c_t for
// the state) are packed over its fp32 columns once those are read.
constexpr uint32_t TM_O1 = 0, TM_V = 64, TM_O0 = 128, TM_S = 192, TM_SA = 320, TM_W = 384, TM_P = 448, TM_COLS = 512;

// barrier indices
enum {
    B_FULL_KQ = 0,                  // [3] K, Q of a chunk landed (TMA)
    B_EMPTY_KQ = 3,                 // [3] 2 commits: the chunk's state product and its Gram have read K, Q
    B_FULL_V = 6, B_EMPTY_V = 7,    // V of a chunk landed; the U product read it
    B_FULL_AX = 8,                  // [2] T' and the vectors landed
    B_EMPTY_AX = 10,                // [2] 11 arrivals: the U product read T'; prep, the 8 carry warps and out read the vectors
    B_KQ_OK = 12, B_V_OK,           // prep: the raw K, Q of the chunk may be read (padding rows zeroed); V of the last
                                    // chunk, when partial, has its padding rows zeroed (one phase)
    B_TW, B_W_DONE, B_WT,           // T' diag(cw) written; W^T in TMEM; -W^T in shared memory
    B_P_DONE, B_PM,                 // Gram in TMEM; Pm written (and the Gram read)
    B_V_DONE, B_VA,                 // v_new^T (and o^T's first part) in TMEM; its 16-bit copies written (8 warps)
    B_S_DONE, B_SA, B_SD,           // state updated; its 16-bit copy written; the decayed fp32 state written (8 warps)
    B_O_DONE,                       // [2] o^T of a chunk complete, per TMEM buffer
    B_O_READ = B_O_DONE + 2,        // [2] per TMEM buffer: zeroed at the start (phase 0), then o^T of each chunk
                                    // using it read and the buffer zeroed again
    B_KQO = B_O_READ + 2,           // [2] prep -> out: the raw Q rows of a chunk may be read (alternating per chunk)
    B_QK = B_KQO + 2,               // [2] out -> MMA: Q~^T of a chunk written (alternating per chunk)
    B_U_DONE = B_QK + 2,            // U^T of a chunk in TMEM (and every earlier product of the side issuer done)
    B_DRAIN,                        // 2 commits: the last MMAs of both issuers completed (exit)
    B_COUNT
};
static_assert(B_COUNT <= kNumBars, "barriers");
constexpr int kCarryWarps = NCARRY / 32;

struct ChainArgs {
    const void *initial_state;
    void *final_state;
    const int32_t *lengths;
    float scale;
    int B, Nk, Nv, S, NC;
    int l2norm;
    float eps;
    const float *vec;  // workspace vectors
    unsigned int *err;
    const void *epi_z;  // NULL: no epilogue
    const float *epi_w;
    float epi_eps;
    unsigned long long wait_ns;
};

// The sequence a CTA runs, longest first.  A CTA holds an SM for its whole chain and CTAs start in index order as
// SMs free up, so with more chains than SMs a long chain that starts late sets the end of the launch (longest-
// processing-time-first list scheduling).  CTA i takes the sequence whose valid length ranks i / Nv-th (longest
// first, ties by index; an invalid length counts as 0); its value head stays i % Nv.  Without lengths, or with more
// than kRankMaxB sequences, the order is the index order.  Called by all threads before anything else.
__device__ __forceinline__ int order_chain(const ChainArgs &a, int tid, uint8_t *sm) {
    const int seq = blockIdx.x / a.Nv;
    if (!a.lengths || a.B <= 1 || a.B > kRankMaxB) return seq;
    int *s_len = reinterpret_cast<int *>(sm + OFF_OUT);
    volatile int *s_sel = reinterpret_cast<volatile int *>(sm + OFF_OUT + kRankMaxB * 4);
    for (int i = tid; i < a.B; i += CH_THREADS) {
        const int L = a.lengths[i];
        s_len[i] = (L < 0 || L > a.S) ? 0 : L;
    }
    __syncthreads();
    for (int i = tid; i < a.B; i += CH_THREADS) {  // the ranks are a permutation of 0..B-1: one i matches
        const int Li = s_len[i];
        int r = 0;
        for (int j = 0; j < a.B; ++j) {
            const int Lj = s_len[j];
            r += (Lj > Li) || (Lj == Li && j < i);
        }
        if (r == seq) *s_sel = i;
    }
    __syncthreads();
    const int sel = *s_sel;
    __syncthreads();  // everyone has read it before the tile is reused
    return sel;
}

// Pairs of 16-bit values across neighbouring lanes: lane l holds x[k] = M[k][col] for its column col = base + l and
// rows k = 0..63; after this, even lanes hold the word (M[2i][col], M[2i][col+1]) of row 2i and odd lanes the word
// (M[2i+1][col-1], M[2i+1][col]) of row 2i+1, i = 0..31 (one shuffle per pair of rows).
template <typename T> __device__ __forceinline__ uint32_t pair_word(float x0, float x1, int lane) {
    const bool odd = lane & 1;
    const float send = odd ? x0 : x1;
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    return odd ? TcT<T>::pack2(recv, x1) : TcT<T>::pack2(x0, recv);
}

// four 8 x 8 16-bit matrices from registers (mma.sync fragment layout) into shared memory, each transposed (lane l
// supplies the address of row l % 8 of destination matrix l / 8)
__device__ __forceinline__ void stsm_x4_trans(uint32_t addr, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

// The part of a bounded wait after its first test failed, out of line: one copy of the polling loop and the
// timeout record instead of one per call site.  The kernel's code is large (every role's loop is hot at once),
// and with a CTA on most SMs its instruction fetches contend: the warps' stalls for instructions doubled from
// 32 to 128 CTAs.  This, with the loops over 32-column halves kept rolled, took 12 % off a launch of 128 chains.
__device__ __noinline__ bool wait_slow(uint64_t *bar, uint32_t parity, uint64_t limit_ns, volatile int *abort,
                                       uint32_t bar_index) {
    if (mbar_wait_ns(bar, parity, limit_ns, abort)) return true;
    if (!*abort)  // this wait ran out (rather than seeing another group stop): record where
        atomicCAS(&g_timeout_site, 0u,
                  0x80000000u | ((threadIdx.x >> 5) << 24) | (bar_index << 16) | (parity << 15) |
                      (blockIdx.x & 0x7fffu));
    return false;
}

template <typename T, bool kGate, bool kOrdered>
__global__ void __launch_bounds__(CH_THREADS, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const __grid_constant__ CUtensorMap tm_tp, const __grid_constant__ CUtensorMap tm_fs, const ChainArgs a) {
    extern __shared__ __align__(1024) uint8_t smraw[];
    uint8_t *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BARS);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const float *vecs = reinterpret_cast<const float *>(sm + OFF_VECS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3;
    const int h = blockIdx.x % a.Nv;
    const int b = kOrdered ? order_chain(a, tid, sm) : (int)blockIdx.x / a.Nv;
    const int bh = b * a.Nv + h, kh = h / (a.Nv / a.Nk);
    const int S = a.S;
    int L = a.lengths ? a.lengths[b] : S;
    const bool bad_len = (L < 0 || L > S);
    if (bad_len) L = 0;
    const int nvalid = (L + C - 1) / C, ntotal = (S + C - 1) / C;
    const int zq = b * a.Nk + kh;  // TMA z coordinate of q/k rows
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint64_t wait_ns = a.wait_ns;
    const size_t ch0 = (size_t)bh * a.NC;  // workspace index of chunk 0

    if (tid == 0) {
        if (bad_len) raise_device_error(a.err, GDR_DEVERR_LENGTH);
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t cnt = 1;
            if (i == B_EMPTY_AX || i == B_EMPTY_AX + 1) cnt = 3 + kCarryWarps;
            if (i == B_VA || i == B_SA || i == B_SD) cnt = kCarryWarps;
            if (i == B_EMPTY_KQ || i == B_EMPTY_KQ + 1 || i == B_EMPTY_KQ + 2 || i == B_DRAIN) cnt = 2;
            mbar_init(bars + i, cnt);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    auto vec_of = [&](int j) { return vecs + (j % NAX) * (kVecBytes / 4); };
    auto chunk_n = [&](int j) { return min(C, L - j * C); };
    auto stop = [&]() { *s_abort = 1; };

#ifdef GDR_PHASE_TIMERS
    __shared__ unsigned long long s_wcyc[kTimerSlots];
    for (int i = tid; i < kTimerSlots; i += CH_THREADS) s_wcyc[i] = 0;
    __syncthreads();
    const long long t_start = clock64();
    const int role = warp < 8 ? 0 : warp < W_PREP0 ? 1 : warp < W_MMA ? 2 : warp == W_MMA ? 3 : 4;  // 4: loaders, side
    const bool rep_thread = tid == 0 || tid == W_OUT0 * 32 || tid == W_PREP0 * 32 || tid == W_MMA * 32 ||
                            tid == W_SIDE * 32;  // role 4: the side issuer
#endif
    auto wait = [&](int idx, uint32_t parity) {
#ifdef GDR_PHASE_TIMERS
        const long long t0 = clock64();
        const bool ok = mbar_wait_ns(bars + idx, parity, wait_ns, s_abort);
        if (rep_thread) s_wcyc[role * 36 + idx] += (unsigned long long)(clock64() - t0);
        if (ok) return true;
        if (!*s_abort)  // this wait ran out (rather than seeing another group stop): record where
            atomicCAS(&g_timeout_site, 0u,
                      0x80000000u | ((uint32_t)warp << 24) | ((uint32_t)idx << 16) | (parity << 15) |
                          (blockIdx.x & 0x7fffu));
        return false;
#else
        if (mbar_test(bars + idx, parity)) return true;
        return wait_slow(bars + idx, parity, wait_ns, s_abort, (uint32_t)idx);
#endif
    };

    if (warp == W_VLD) {
        // ===================== V loads (a warp of their own: a suspended wait of the other loader's thread must not
        // hold them back) =====================
        int issued_v = 0;
        if (lane == 0) {
            // V, one chunk at a time into its single buffer once the U product of the chunk before has read it (from
            // L2: the other loader prefetches V two chunks ahead)
            for (int j = 0; j < nvalid; ++j) {
                if (j >= 1 && !wait(B_EMPTY_V, (j - 1) & 1)) { stop(); break; }
                mbar_arrive_expect_tx(bars + B_FULL_V, 16384);
                tma_load_3d(sm + OFF_V, &tm_v, bars + B_FULL_V, 0, j * C, bh);
                tma_load_3d(sm + OFF_V + 8192, &tm_v, bars + B_FULL_V, 64, j * C, bh);
                ++issued_v;
            }
            if (issued_v) mbar_wait_ns(bars + B_FULL_V, (issued_v - 1) & 1, kDrainWaitNs);
        }
    } else if (warp == W_TMA) {
        // ================================ TMA loads ================================
        int issued_kq[NKQ] = {0, 0, 0}, issued_ax[NAX] = {0, 0};
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_tp);
            auto prefetch_l2 = [&](int j) {  // V and the epilogue's z rows of chunk j, ahead of their loads
                tma_prefetch_3d(&tm_v, 0, j * C, bh);
                tma_prefetch_3d(&tm_v, 64, j * C, bh);
                if (a.epi_z) {
                    const int rows = min(C, L - j * C);
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                                     static_cast<const T *>(a.epi_z) + ((size_t)bh * S + (size_t)j * C) * D),
                                 "r"((uint32_t)(rows * D * 2))
                                 : "memory");
                }
            };
            for (int j = 0; j < min(nvalid, 2); ++j) prefetch_l2(j);
            for (int j = 0; j < nvalid; ++j) {
                const int y = j * C;
                const int sk = j % NKQ, sa = j % NAX;
                if (j >= NKQ && !wait(B_EMPTY_KQ + sk, ((j / NKQ) - 1) & 1)) { stop(); break; }
                mbar_arrive_expect_tx(bars + B_FULL_KQ + sk, 32768);
                uint8_t *st = sm + OFF_KQ + sk * KQ_STAGE;
                tma_load_3d(st, &tm_q, bars + B_FULL_KQ + sk, 0, y, zq);
                tma_load_3d(st + 8192, &tm_k, bars + B_FULL_KQ + sk, 0, y, zq);
                tma_load_3d(st + 16384, &tm_q, bars + B_FULL_KQ + sk, 64, y, zq);
                tma_load_3d(st + 24576, &tm_k, bars + B_FULL_KQ + sk, 64, y, zq);
                ++issued_kq[sk];
                if (j >= NAX && !wait(B_EMPTY_AX + sa, ((j / NAX) - 1) & 1)) { stop(); break; }
                mbar_arrive_expect_tx(bars + B_FULL_AX + sa, (uint32_t)(kTpBytes + kVecBytes));
                tma_load_3d(sm + OFF_TPS + sa * 8192, &tm_tp, bars + B_FULL_AX + sa, 0, 0, (int)(ch0 + j));
                bulk_load(sm + OFF_VECS + sa * kVecBytes, a.vec + (ch0 + j) * (kVecBytes / 4), (uint32_t)kVecBytes,
                          bars + B_FULL_AX + sa);
                ++issued_ax[sa];
                if (j + 2 < nvalid) prefetch_l2(j + 2);
            }
            // drain: every load this lane issued has landed before the CTA leaves
            for (int s = 0; s < NKQ; ++s)
                if (issued_kq[s]) mbar_wait_ns(bars + B_FULL_KQ + s, (issued_kq[s] - 1) & 1, kDrainWaitNs);
            for (int s = 0; s < NAX; ++s)
                if (issued_ax[s]) mbar_wait_ns(bars + B_FULL_AX + s, (issued_ax[s] - 1) & 1, kDrainWaitNs);
        }
    } else if (warp == W_MMA || warp == W_SIDE) {
        // ============================== MMA issue ==============================
        // Two issuing warps.  Each runs its branch as a whole warp, so every operand address is warp-uniform, and one
        // elected lane issues (a lone divergent lane costs several times more per instruction).
        //   chain warp: per chunk c only the two products that depend on the state, each issued the moment its
        //     operands are in place: [v_new^T | o^T] of c, then the state product of c.
        //   side warp: the products that do not depend on the state, placed where the carry warps convert and the
        //     tensor pipe would otherwise idle: W and the Gram of c+1 while v_new of c is converted, o's Pm term of c
        //     and U of c+1 while the state is converted.
        // Products of different warps are ordered only through barriers: U of c+1 is issued after the state product
        // of c completed (both read or write v_new^T's columns), and the chain warp waits for U of c before the
        // [v_new^T | o^T] product that accumulates onto it.  Each hand-off phase is waited for once, before this
        // warp's own step that lets its producer reach the next phase of the same barrier.
        if (nvalid > 0) {
            const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
            const uint32_t sb = __shfl_sync(0xffffffffu, sbase, 0);
            const uint32_t idSS = idesc_t<T>(128, 64, true, false);    // A MN-major smem, B K-major
            const uint32_t idP = idesc_t<T>(128, 64, false, false);    // A, B K-major smem
            const uint32_t id1 = idesc_t<T>(128, 128, false, true);    // A TMEM, B MN-major, N = 128
            const uint32_t idO = idesc_t<T>(128, 64, false, false);    // A TMEM, B K-major
            auto kq_base = [&](int j) { return sb + OFF_KQ + (uint32_t)(j % NKQ) * KQ_STAGE; };
            // v_new^T's 16-bit copies over its fp32 columns: tokens 16 kk .. 16 kk + 15, plain and scaled by c_t
            auto va_col = [&](int kk) { return tm + TM_V + 32 * (kk >> 1) + 8 * (kk & 1); };
            auto vs_col = [&](int kk) { return tm + TM_V + 32 * (kk >> 1) + 16 + 8 * (kk & 1); };
            auto uwait = [&](int idx, uint32_t parity) { return __all_sync(0xffffffffu, wait(idx, parity)); };
#ifdef GDR_PHASE_TIMERS
            // cycles spent issuing each kind of product: 1, 2, W, Gram, O2, U
            long long t_iss[6] = {0, 0, 0, 0, 0, 0};
#define ISSUE_T(kind, ...)                      \
    do {                                        \
        const long long t0_ = clock64();        \
        if (elect_one_sync()) {                 \
            __VA_ARGS__;                        \
        }                                       \
        __syncwarp();                           \
        t_iss[kind] += clock64() - t0_;         \
    } while (0)
#else
#define ISSUE_T(kind, ...)         \
    do {                           \
        if (elect_one_sync()) {    \
            __VA_ARGS__;           \
        }                          \
        __syncwarp();              \
    } while (0)
#endif
            bool to = false;
            if (warp == W_MMA) {
                auto issue_1 = [&](int c) {  // [v_new^T | o^T] = [U^T | 0] + S^T [-W^T | Q~^T]  (odd c: [o^T | v_new^T])
                    const uint32_t bb = sb + ((c & 1) ? OFF_QT : OFF_WT0);
                    const uint32_t d = tm + ((c & 1) ? TM_O1 : TM_V);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(d, tm + TM_SA + 8 * kk, sdesc_sw128(bb + kk * 2048, 16384, 1024), id1, 1);
                };
                auto issue_2 = [&](int c) {  // S^T = e^{G_last} S^T + (v_new diag(c))^T K
                    const uint32_t kb = kq_base(c) + 8192;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tm + TM_S, vs_col(kk), sdesc_sw128(kb + kk * 2048, 16384, 1024), id1, 1);
                };
                for (int c = 0; c < nvalid; ++c) {
                    const uint32_t par = c & 1;
                    if (!(uwait(B_U_DONE, par) && uwait(B_SA, par) && uwait(B_WT, par) &&
                          uwait(B_QK + par, (c >> 1) & 1) && uwait(B_O_READ + par, (c >> 1) & 1))) {
                        to = true;
                        break;
                    }
                    tc_fence_after();
                    ISSUE_T(0, issue_1(c); mma_commit(bars + B_V_DONE));
                    EVENT(c, 1);
                    // v_new's copies written; each carry warp wrote its decayed fp32 state before them
                    if (!uwait(B_VA, par)) {
                        to = true;
                        break;
                    }
                    tc_fence_after();
                    ISSUE_T(1, issue_2(c); mma_commit(bars + B_S_DONE); mma_commit(bars + B_EMPTY_KQ + c % NKQ));
                    EVENT(c, 4);
                }
            } else {
                auto issue_W = [&](int j) {  // W^T = K^T (T' diag(cw))^T
                    const uint32_t kb = kq_base(j) + 8192;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tm + TM_W, sdesc_sw128(kb + kk * 2048, 16384, 1024),
                                 sdesc_sw128(sb + OFF_TW + kk * 32, 16, 1024), idSS, kk > 0);
                };
                auto issue_P = [&](int j) {  // [Q; K] K^T
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t ad = kq_base(j) + (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_bf16(tm + TM_P, sdesc_sw128(ad, 16, 1024), sdesc_sw128(ad + 8192, 16, 1024), idP,
                                 kk > 0);
                    }
                };
                auto issue_U = [&](int j) {  // U^T = V^T T'^T
                    const uint32_t tb = sb + OFF_TPS + (uint32_t)(j % NAX) * 8192;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tm + TM_V, sdesc_sw128(sb + OFF_V + kk * 2048, 8192, 1024),
                                 sdesc_sw128(tb + kk * 32, 16, 1024), idSS, kk > 0);
                };
                auto issue_O2 = [&](int c) {  // o^T += v_new^T Pm^T
                    const uint32_t pb = sb + OFF_PM + (uint32_t)(c & 1) * 8192;
                    const uint32_t d = tm + ((c & 1) ? TM_O1 : TM_O0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(d, va_col(kk), sdesc_sw128(pb + kk * 32, 16, 1024), idO, 1);
                };
                const bool vpad = chunk_n(nvalid - 1) < C;  // the last chunk's V needs its padding rows zeroed
                // chunk 0's W, Gram and U
                if (uwait(B_TW, 0) && uwait(B_KQ_OK, 0) && uwait(B_FULL_KQ, 0) && uwait(B_FULL_AX, 0) &&
                    uwait(B_FULL_V, 0) && (!(vpad && nvalid == 1) || uwait(B_V_OK, 0))) {
                    tc_fence_after();
                    ISSUE_T(2, issue_W(0); mma_commit(bars + B_W_DONE); issue_P(0); mma_commit(bars + B_P_DONE);
                            mma_commit(bars + B_EMPTY_KQ); issue_U(0); mma_commit(bars + B_EMPTY_V);
                            mma_commit(bars + B_EMPTY_AX); mma_commit(bars + B_U_DONE));
                } else {
                    to = true;
                }
                for (int c = 0; !to && c < nvalid; ++c) {
                    const uint32_t par = c & 1;
                    const int j = c + 1;
                    const bool more = j < nvalid;
                    if (more) {
                        // W of c+1 once prep has read W^T of c out of TMEM
                        if (!(uwait(B_WT, par) && uwait(B_TW, j & 1) && uwait(B_KQ_OK, j & 1) &&
                              uwait(B_FULL_KQ + j % NKQ, (j / NKQ) & 1))) {
                            to = true;
                            break;
                        }
                        tc_fence_after();
                        ISSUE_T(2, issue_W(j); mma_commit(bars + B_W_DONE));
                        EVENT(c, 6);
                    }
                    // Pm of c written (the Gram of c read out of TMEM)
                    if (!uwait(B_PM, par)) {
                        to = true;
                        break;
                    }
                    if (more) {
                        tc_fence_after();
                        ISSUE_T(3, issue_P(j); mma_commit(bars + B_P_DONE); mma_commit(bars + B_EMPTY_KQ + j % NKQ));
                        EVENT(c, 7);
                    }
                    // the state product of c done: v_new^T's copies are written and no longer read by it
                    if (!uwait(B_S_DONE, par)) {
                        to = true;
                        break;
                    }
                    tc_fence_after();
                    ISSUE_T(4, issue_O2(c); mma_commit(bars + B_O_DONE + par));
                    EVENT(c, 9);
                    if (more) {
                        if (!(uwait(B_FULL_V, j & 1) && uwait(B_FULL_AX + j % NAX, (j / NAX) & 1) &&
                              (!(vpad && j == nvalid - 1) || uwait(B_V_OK, 0)))) {
                            to = true;
                            break;
                        }
                        tc_fence_after();
                        ISSUE_T(5, issue_U(j); mma_commit(bars + B_EMPTY_V); mma_commit(bars + B_EMPTY_AX + j % NAX);
                                mma_commit(bars + B_U_DONE));
                        EVENT(c, 10);
                    }
                }
            }
#undef ISSUE_T
#ifdef GDR_PHASE_TIMERS
            if (blockIdx.x == 0 && lane == 0)
                for (int i = (warp == W_MMA ? 0 : 2); i < (warp == W_MMA ? 2 : 6); ++i)
                    g_events[kEvN * kEvK - 6 + i] = t_iss[i];
#endif
            if (to) stop();
            // drain: every MMA of both issuers has completed before TMEM is released
            if (elect_one_sync()) mma_commit(bars + B_DRAIN);
            __syncwarp();
            mbar_wait_ns(bars + B_DRAIN, 0, kDrainWaitNs);
        }
    } else if (warp >= W_PREP0) {
        // ================================ prep ================================
        const int p = tid - W_PREP0 * 32;
        bool to = false;
        // padding rows of chunk j's raw K and Q (zeroed so that no padding value reaches a product), then the
        // hand-offs that let the MMA and out warps read them; then T' diag(e^G/|k|) of chunk j
        auto stage_in = [&](int j) -> bool {
            const int n = chunk_n(j);
            bool t2 = !(wait(B_FULL_KQ + j % NKQ, (j / NKQ) & 1) && wait(B_FULL_AX + j % NAX, (j / NAX) & 1));
            if (named_sync_or(BAR_PREP, NPREP, t2)) return false;
            if (n < C) {
                uint8_t *kq = sm + OFF_KQ + (j % NKQ) * KQ_STAGE;
                for (int e = p; e < (C - n) * 8 * 4; e += NPREP) {  // 4 tiles x (C - n) rows x 8 chunks
                    const int tile = e / ((C - n) * 8), r = n + (e / 8) % (C - n), c8 = e & 7;
                    *reinterpret_cast<uint4 *>(kq + tile * 8192 + r * 128 + c8 * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            named_sync(BAR_PREP, NPREP);
            if (p == 0) {
                mbar_arrive(bars + B_KQ_OK);
                mbar_arrive(bars + B_KQO + (j & 1));
            }
            // T' diag(cw): column factors of T' (the B operand of W^T = K^T (T' diag(cw))^T)
            const uint8_t *tp = sm + OFF_TPS + (j % NAX) * 8192;
            const float *cw = vec_of(j) + V_CW * 64;
            for (int e = p; e < 512; e += NPREP) {
                const int t = e >> 3, pos = e & 7, s0 = ((pos ^ (t & 7)) * 8);
                float f[8];
                unpack8<T>(*reinterpret_cast<const uint4 *>(tp + t * 128 + pos * 16), f);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] *= cw[s0 + i];
                *reinterpret_cast<uint4 *>(sm + OFF_TW + t * 128 + pos * 16) = pack8<T>(f);
            }
            fence_proxy_async_smem();
            named_sync(BAR_PREP, NPREP);
            if (p == 0) mbar_arrive(bars + B_TW);
            return true;
        };
        // V of the last chunk, if partial: padding rows zeroed once it has landed (its U product waits for this)
        const int vlast = nvalid - 1;
        auto pad_v = [&]() -> bool {
            bool t2 = !wait(B_FULL_V, vlast & 1);
            if (named_sync_or(BAR_PREP, NPREP, t2)) return false;
            const int n = chunk_n(vlast);
            for (int e = p; e < (C - n) * 8 * 2; e += NPREP) {
                const int tile = e / ((C - n) * 8), r = n + (e / 8) % (C - n), c8 = e & 7;
                *reinterpret_cast<uint4 *>(sm + OFF_V + tile * 8192 + r * 128 + c8 * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            named_sync(BAR_PREP, NPREP);
            if (p == 0) mbar_arrive(bars + B_V_OK);
            return true;
        };
        const bool vpad = nvalid > 0 && chunk_n(vlast) < C;
        if (nvalid > 0 && !stage_in(0)) to = true;
        if (!to && vpad && vlast == 0 && !pad_v()) to = true;
        for (int c = 0; !to && c < nvalid; ++c) {
            const uint32_t par = c & 1;
            const int n = chunk_n(c);
            const float *vc = vec_of(c);
            // ---- -W^T of chunk c into its parity's MN-major B tile [dk][t] (last read by the [v_new^T | o^T]
            // product of c - 2, complete before the side issuer started W of c) ----
            bool t2 = !wait(B_W_DONE, par);
            if (named_sync_or(BAR_PREP, NPREP, t2)) { to = true; break; }
            tc_fence_after();
            {
                const int dk = q4 * 32 + lane;
#pragma unroll 1
                for (int hv = 0; hv < 2; ++hv) {
                    float w[32];
                    tmem_ld32(tmem + TM_W + lane_base + 32 * hv, w);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) w[i] = -w[i];
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(sm + OFF_WT0 + par * 32768 + blk_off(dk, 32 * hv + 8 * c8)) =
                            pack8<T>(&w[8 * c8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_PREP, NPREP);
            if (p == 0) mbar_arrive(bars + B_WT);
            // ---- the next chunk's raw tiles and T' diag(cw), early: the W product and Q~^T of chunk c + 1 wait on them
            if (c + 1 < nvalid && !stage_in(c + 1)) { to = true; break; }
            // ---- the Gram of chunk c has landed: Pm (rows t of lanes 0..63; the row factor scale/|q_t| is applied
            // to o by the out warps) ----
            t2 = !wait(B_P_DONE, par);
            if (named_sync_or(BAR_PREP, NPREP, t2)) { to = true; break; }
            tc_fence_after();
            if (q4 < 2) {
                const int t = q4 * 32 + lane;
                const bool valid = t < n;
                const float g2t = vc[V_G2 * 64 + t];
                uint8_t *pm = sm + OFF_PM + par * 8192;
#pragma unroll 1
                for (int hv = 0; hv < 2; ++hv) {
                    float v[32];
                    if (hv == 1 && q4 == 0) {  // rows 0..31, columns 32..63: above the diagonal
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0.f;
                    } else {
                        tmem_ld32(tmem + TM_P + lane_base + 32 * hv, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int s = 32 * hv + i;
                            const float dec = kGate ? ex2_approx(g2t - vc[V_LAM * 64 + s]) : vc[V_CT * 64 + s];
                            v[i] = (valid && s <= t) ? v[i] * dec : 0.f;
                        }
                    }
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(pm + blk_off(t, 32 * hv + 8 * c8)) = pack8<T>(&v[8 * c8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(BAR_PREP, NPREP);
            if (p == 0) {
                EVENT(c, 12);
                mbar_arrive(bars + B_PM);
                mbar_arrive(bars + B_EMPTY_AX + c % NAX);  // done with chunk c's vectors
            }
            if (vpad && c + 1 == vlast && !pad_v()) { to = true; break; }
        }
        if (to && p == 0) stop();
    } else if (warp >= W_OUT0) {
        // ================================ out ================================
        const int p = tid - W_OUT0 * 32, dv = q4 * 32 + lane;
        const bool storer = p == 0;
        const bool epi = a.epi_z != nullptr;
        float *red = reinterpret_cast<float *>(sm + OFF_RED);
        float *rqs = reinterpret_cast<float *>(sm + OFF_RQ);  // scale / |q_t| of chunks j (set j % 2)
        bool to = false;
        float wdv = 1.f;
        if (epi) wdv = a.epi_w[dv];
        // Once the raw Q rows of chunk j are in place (padding rows zeroed): scale / |q_t| (eps inside the root; 0 past
        // the length), and Q~^T = (diag(e^{G_t}) Q)^T as the MN-major B tile [dk][t] of chunk j's v_new / o product,
        // transposed in 8 x 8 blocks with ldmatrix / stmatrix.  Its single buffer was last read by the v_new / o
        // product of chunk j - 1, waited for first.
        auto make_q = [&](int j) -> bool {
            const int n = chunk_n(j);
            bool t2 = !((j == 0 || wait(B_V_DONE, (j - 1) & 1)) && wait(B_KQO + (j & 1), (j >> 1) & 1) &&
                        wait(B_FULL_KQ + j % NKQ, (j / NKQ) & 1) && wait(B_FULL_AX + j % NAX, (j / NAX) & 1));
            if (named_sync_or(BAR_OUT, NOUTW, t2)) return false;
            if (storer) EVENT(j, 15);
            const uint8_t *qt = sm + OFF_KQ + (j % NKQ) * KQ_STAGE;  // raw Q: dk blocks at +0, +16384
            {
                // thread p: half p & 1 of row p / 2; its 8 chunks in a rotated order (no two threads of a quarter warp
                // on the same bank group)
                const int t = p >> 1, hb = p & 1;
                const uint4 *qrow = reinterpret_cast<const uint4 *>(qt + hb * 16384 + t * 128);
                float ss = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float f[8];
                    unpack8<T>(qrow[(i + p) & 7], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                if (hb == 0) rqs[(j & 1) * 64 + t] = t < n ? a.scale * (a.l2norm ? rsqrtf(ss + a.eps) : 1.f) : 0.f;
            }
            {
                // warp w transposes token blocks 2w, 2w + 1 (16 rows) for all 128 key columns: four 8 x 8 blocks per
                // ldmatrix / stmatrix
                const uint32_t dst = sbase + OFF_QT;
                const float *eg = vec_of(j) + V_EG * 64;
                const int r = lane & 7, mi = lane >> 3;
#pragma unroll
                for (int tbi = 0; tbi < 2; ++tbi) {
                    const int tb = 2 * q4 + tbi;
                    const float e0 = kGate ? eg[8 * tb + (lane >> 2)] : 1.f;
#pragma unroll
                    for (int dq = 0; dq < 4; ++dq) {
                        const int db = 4 * dq + mi;  // the 8-column key block this lane addresses
                        const uint32_t src = smem_u32(qt) + (db >> 3) * 16384 + (8 * tb + r) * 128 +
                                             ((((db & 7) ^ r)) << 4);
                        uint32_t f[4];
                        ldsm_x4(f, src);
                        if (kGate) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float2 x = TcT<T>::unpack2(f[i]);
                                f[i] = TcT<T>::pack2(x.x * e0, x.y * e0);
                            }
                        }
                        const int dk = 8 * db + r;  // destination row of this lane's address
                        stsm_x4_trans(dst + dk * 128 + (((tb ^ r)) << 4), f);
                    }
                }
            }
            fence_proxy_async_smem();
            named_sync(BAR_OUT, NOUTW);
            if (storer) {
                EVENT(j, 13);
                mbar_arrive(bars + B_QK + (j & 1));
                mbar_arrive(bars + B_EMPTY_AX + j % NAX);  // done with chunk j's vectors
            }
            return true;
        };
        if (nvalid > 0) {  // both o buffers start from zero (TMEM holds no defined value after allocation)
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0.f;
            tmem_st32(tmem + lane_base + TM_O0, z);
            tmem_st32(tmem + lane_base + TM_O0 + 32, z);
            tmem_st32(tmem + lane_base + TM_O1, z);
            tmem_st32(tmem + lane_base + TM_O1 + 32, z);
            tmem_st_wait();
            tc_fence_before();
            named_sync(BAR_OUT, NOUTW);
            if (storer) {
                mbar_arrive(bars + B_O_READ);
                mbar_arrive(bars + B_O_READ + 1);
            }
        }
        if (nvalid > 0 && !make_q(0)) to = true;
        for (int c = 0; !to && c < nvalid; ++c) {
            const uint32_t par = c & 1;
            const int n = chunk_n(c);
            if (c + 1 < nvalid && !make_q(c + 1)) { to = true; break; }
            bool t2 = !wait(B_O_DONE + (c & 1), (c >> 1) & 1);
            if (named_sync_or(BAR_OUT, NOUTW, t2)) { to = true; break; }
            if (storer) EVENT(c, 8);
            tc_fence_after();
            float o[2][32];  // o[hv][i]: token 32 hv + i of this lane's value column
            const uint32_t ocol = tmem + lane_base + (par ? TM_O1 : TM_O0);
            tmem_ld32(ocol, o[0]);
            tmem_ld32(ocol + 32, o[1]);
            tmem_ld_wait();
            {  // the buffer starts from zero for the chunk after next
                float z[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) z[i] = 0.f;
                tmem_st32(ocol, z);
                tmem_st32(ocol + 32, z);
                tmem_st_wait();
            }
            tc_fence_before();
            if (storer) bulk_wait_read0();  // the previous out tile has been read by its store
            named_sync(BAR_OUT, NOUTW);
            if (storer) mbar_arrive(bars + B_O_READ + (c & 1));
            {
                const float *rq = rqs + par * 64;
#pragma unroll
                for (int t = 0; t < 64; ++t) o[t >> 5][t & 31] *= rq[t];
            }
            if (epi) {
                // sum over the head's Dv outputs of o^2 for each token: reduce-scatter inside the warp (per half of
                // the tokens, lane l ends with token 32 hv + l), then over the four warps through shared memory
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {
                    float x[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = o[hv][i] * o[hv][i];
#pragma unroll
                    for (int w = 16, off = 16; off >= 1; w >>= 1, off >>= 1) {
                        const bool up = lane & off;
#pragma unroll
                        for (int i = 0; i < w; ++i) {
                            const float send = up ? x[i] : x[i + w];
                            const float keep = up ? x[i + w] : x[i];
                            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                        }
                    }
                    red[q4 * 64 + 32 * hv + lane] = x[0];
                }
                named_sync(BAR_OUT, NOUTW);
                if (p < C) {
                    const float ssq = red[p] + red[64 + p] + red[128 + p] + red[192 + p];
                    red[256 + p] = rsqrtf(ssq * (1.f / D) + a.epi_eps);
                }
                named_sync(BAR_OUT, NOUTW);
                // z of this lane's column for the valid tokens, from global memory (prefetched into L2 two chunks
                // ahead): even lanes load the words of even tokens, odd lanes of odd tokens, then swap halves
                const T *zr = static_cast<const T *>(a.epi_z) + ((size_t)bh * S + (size_t)c * C) * D + (dv & ~1);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = 2 * i + (lane & 1);
                    const uint32_t wz = t < n ? *reinterpret_cast<const uint32_t *>(zr + (size_t)t * D) : 0u;
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, wz, 1);
                    // even lane: own word (t even) low half; other's (t odd) low half.  odd lane: mirror.
                    const float2 mine = TcT<T>::unpack2(wz), oth = TcT<T>::unpack2(other);
                    const float z0 = (lane & 1) ? oth.y : mine.x;  // token 2i
                    const float z1 = (lane & 1) ? mine.y : oth.x;  // token 2i + 1
                    o[(2 * i) >> 5][(2 * i) & 31] *= red[256 + 2 * i] * wdv * silu_out<T>(z0);
                    o[(2 * i + 1) >> 5][(2 * i + 1) & 31] *= red[256 + 2 * i + 1] * wdv * silu_out<T>(z1);
                }
            }
            // out rows t < n; zero past the length.  Neighbouring lanes exchange values so that each stores
            // 32-bit words of one row.
            uint8_t *ot = sm + OFF_OUT + (dv >> 6) * 8192;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float x0 = 2 * i < n ? o[i >> 4][(2 * i) & 31] : 0.f;
                const float x1 = 2 * i + 1 < n ? o[i >> 4][(2 * i + 1) & 31] : 0.f;
                const uint32_t wv = pair_word<T>(x0, x1, lane);
                const int row = 2 * i + (lane & 1), col = (dv & 63) & ~1;
                *reinterpret_cast<uint32_t *>(ot + blk_off(row, col)) = wv;
            }
            fence_proxy_async_smem();
            named_sync(BAR_OUT, NOUTW);
            if (storer) {
                tma_store_3d(&tm_o, sm + OFF_OUT, 0, c * C, bh);
                tma_store_3d(&tm_o, sm + OFF_OUT + 8192, 64, c * C, bh);
                bulk_commit();
                EVENT(c, 11);
            }
        }
        if (!to && nvalid < ntotal) {  // chunks past the length: zero rows
            if (storer) bulk_wait_read0();
            named_sync(BAR_OUT, NOUTW);
            for (int e = p; e < 16384 / 16; e += NOUTW) reinterpret_cast<uint4 *>(sm + OFF_OUT)[e] = make_uint4(0, 0, 0, 0);
            fence_proxy_async_smem();
            named_sync(BAR_OUT, NOUTW);
            if (storer) {
                for (int c = nvalid; c < ntotal; ++c) {
                    tma_store_3d(&tm_o, sm + OFF_OUT, 0, c * C, bh);
                    tma_store_3d(&tm_o, sm + OFF_OUT + 8192, 64, c * C, bh);
                }
                bulk_commit();
            }
        }
        if (storer) bulk_wait0();
        if (to && storer) stop();
    } else {
        // ================================ carry ================================
        const int hf = warp >> 2;          // key rows [64 hf, 64 hf + 64)
        const int dv = q4 * 32 + lane;     // this thread's value column = TMEM lane
        bool to = false;
        // a wait whose outcome the whole warp shares (the hand-offs below are per warp)
        auto wwait = [&](int idx, uint32_t parity) { return __all_sync(0xffffffffu, wait(idx, parity)); };
        // per-warp hand-offs (the barriers count the 8 carry warps)
        auto warp_arrive = [&](int idx) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + idx);
        };
        // S^T of chunk j (in v): its 16-bit copy (the A operand of chunk j's v_new / o product), then the fp32 state
        // decayed by the chunk's e^{G_last}, onto which the chunk's state update accumulates (without a gate the fp32
        // state in TMEM is already the state, except before chunk 0)
        auto put_state = [&](int j, float (&v)[2][32]) -> bool {
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = TcT<T>::pack2(v[hv][2 * i], v[hv][2 * i + 1]);
                tmem_st16(tmem + TM_SA + lane_base + 32 * hf + 16 * hv, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            warp_arrive(B_SA);
            if (lane == 0) EVENT(j, 0);
            if (!wwait(B_FULL_AX + j % NAX, (j / NAX) & 1)) return false;  // chunk j's vectors
            if (kGate) {
                const float eL = vec_of(j)[V_MISC * 64];
                float w[32];
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) w[i] = v[hv][i] * eL;
                    tmem_st32(tmem + TM_S + lane_base + 64 * hf + 32 * hv, w);
                }
                tmem_st_wait();
            } else if (j == 0) {
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) tmem_st32(tmem + TM_S + lane_base + 64 * hf + 32 * hv, v[hv]);
                tmem_st_wait();
            }
            tc_fence_before();
            warp_arrive(B_SD);
            if (lane == 0) EVENT(j, 14);
            return true;
        };
        if (nvalid > 0) {
            // the initial state column dv, rows 64 hf.. (fp32), straight from global memory (64 B per row per warp)
            float v[2][32];
            const T *s0 = static_cast<const T *>(a.initial_state);
#pragma unroll
            for (int i = 0; i < 64; ++i)
                v[i >> 5][i & 31] = s0 ? to_f32(s0[((size_t)bh * D + 64 * hf + i) * D + dv]) : 0.f;
            if (!put_state(0, v)) to = true;
        }
        for (int c = 0; !to && c < nvalid; ++c) {
            const uint32_t par = c & 1;
            // ---- v_new^T (fp32, 32 of this lane's token columns) -> its two 16-bit copies over the same columns ----
            if (!wwait(B_V_DONE, par)) { to = true; break; }
            if (tid == 0) EVENT(c, 2);
            tc_fence_after();
            {
                // tokens 32 hf .. 32 hf + 31: the plain copy (for o) and the copy scaled by
                // c_t = e^{G_last - G_t}/|k_t| (for the state update)
                const float *ct = vec_of(c) + V_CT * 64 + 32 * hf;
                float u[32];
                tmem_ld32(tmem + TM_V + lane_base + 32 * hf, u);
                tmem_ld_wait();
                uint32_t pk[16], ps[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    pk[i] = TcT<T>::pack2(u[2 * i], u[2 * i + 1]);
                    ps[i] = TcT<T>::pack2(u[2 * i] * ct[2 * i], u[2 * i + 1] * ct[2 * i + 1]);
                }
                tmem_st16(tmem + TM_V + lane_base + 32 * hf, pk);
                tmem_st16(tmem + TM_V + lane_base + 32 * hf + 16, ps);
                tmem_st_wait();
            }
            tc_fence_before();
            warp_arrive(B_VA);
            if (tid == 0) EVENT(c, 3);
            warp_arrive(B_EMPTY_AX + c % NAX);  // done with chunk c's vectors
            // ---- the updated state: 16-bit copy for the next chunk, decayed fp32 back ----
            if (!wwait(B_S_DONE, par)) { to = true; break; }
            if (tid == 0) EVENT(c, 5);
            if (c + 1 == nvalid) break;  // the final state stays in TMEM
            tc_fence_after();
            float sv[2][32];
            tmem_ld32(tmem + TM_S + lane_base + 64 * hf, sv[0]);
            tmem_ld32(tmem + TM_S + lane_base + 64 * hf + 32, sv[1]);
            tmem_ld_wait();
            if (!put_state(c + 1, sv)) { to = true; break; }
        }
        // the warps agree on whether to write the final state (a named barrier below must see all of them)
        to = named_sync_or(BAR_CARRY, NCARRY, to);
        // ---- the final state (or the initial one, for an empty sequence) ----
        if (!to && a.final_state) {
            // staging: a K/Q stage no load or MMA uses any more
            uint8_t *st = sm + OFF_KQ + (nvalid % NKQ) * KQ_STAGE;
            float fv[2][32];
            if (nvalid > 0) {  // S^T after the last chunk, fp32 in TMEM
                tc_fence_after();
                tmem_ld32(tmem + TM_S + lane_base + 64 * hf, fv[0]);
                tmem_ld32(tmem + TM_S + lane_base + 64 * hf + 32, fv[1]);
                tmem_ld_wait();
            } else {
                const T *s0 = static_cast<const T *>(a.initial_state);
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    fv[i >> 5][i & 31] = s0 ? to_f32(s0[((size_t)bh * D + 64 * hf + i) * D + dv]) : 0.f;
            }
            uint8_t *bx = st + ((dv >> 6) * 2 + hf) * 8192;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t wv = pair_word<T>(fv[i >> 4][(2 * i) & 31], fv[i >> 4][(2 * i + 1) & 31], lane);
                const int row = 2 * i + (lane & 1), col = (dv & 63) & ~1;
                *reinterpret_cast<uint32_t *>(bx + blk_off(row, col)) = wv;
            }
            fence_proxy_async_smem();
            named_sync(BAR_CARRY, NCARRY);
            if (tid == 0) {
                for (int bxi = 0; bxi < 4; ++bxi)
                    tma_store_3d(&tm_fs, st + bxi * 8192, 64 * (bxi >> 1), 64 * (bxi & 1), bh);
                bulk_commit();
                bulk_wait0();
            }
        }
        if (to && tid == 0) stop();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *s_abort) raise_device_error(a.err, GDR_DEVERR_TIMEOUT);
#ifdef GDR_PHASE_TIMERS
    if (blockIdx.x == 0) {
        if (tid == 0) {
            s_wcyc[5 * 36] = (unsigned long long)(clock64() - t_start);
            s_wcyc[5 * 36 + 1] = (unsigned long long)nvalid;
        }
        __syncthreads();
        for (int i = tid; i < kTimerSlots; i += CH_THREADS) g_phase[i] += s_wcyc[i];
    }
#endif
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// (inner, rows, Z) tensor of 2-byte elements (bf16 or fp16), 64 x 64 boxes, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int inner, long long rows, long long Z, CUtensorMapDataType type) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)Z};
    cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)rows * inner * 2};
    cuuint32_t box[3] = {64, 64, 1}, es[3] = {1, 1, 1};
    return enc(m, type, 3, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t chunk_wy_workspace(int B, int Nv, int S) {
    const size_t nch = (size_t)B * Nv * (size_t)((S + C - 1) / C);
    return nch * (kTpBytes + kVecBytes);
}

namespace {
template <typename T, bool kGate>
cudaError_t launch_tc_t(const ChunkArgs &ca, cudaStream_t stream) {
    constexpr CUtensorMapDataType ty = TcT<T>::kMap;
    const int NC = (ca.S + C - 1) / C;
    const size_t nch = (size_t)ca.B * ca.Nv * NC;
    if (nch == 0) return cudaSuccess;
    uint8_t *ws = static_cast<uint8_t *>(ca.workspace);
    float *vec = reinterpret_cast<float *>(ws + vec_offset(nch));

    // ---- the WY pass over every chunk ----
    WyArgs w{};
    w.k = ca.k; w.beta = ca.beta; w.g = ca.g; w.lengths = ca.lengths;
    w.B = ca.B; w.Nk = ca.Nk; w.Nv = ca.Nv; w.S = ca.S; w.NC = NC;
    w.l2norm = ca.l2norm; w.eps = ca.eps; w.beta_logits = ca.beta_logits; w.A_log = ca.A_log; w.dt_bias = ca.dt_bias;
    w.tp = ws;
    w.vec = vec;
    static LaunchCache wyc(reinterpret_cast<const void *>(wy_kernel<T, kGate>));
    cudaError_t e = wyc.allow_smem((int)WY_SMEM);
    if (e != cudaSuccess) return e;
    const long long wy_blocks = (long long)ca.B * ca.Nk * NC;
    if (wy_blocks >= (1LL << 31)) return cudaErrorInvalidValue;
    wy_kernel<T, kGate><<<(unsigned)wy_blocks, WY_THREADS, WY_SMEM, stream>>>(w);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // ---- the chains ----
    CUtensorMap mq, mk, mv, mo, mtp, mfs;
    memset(&mfs, 0, sizeof(mfs));
    if (!make_map(&mq, ca.q, D, ca.S, (long long)ca.B * ca.Nk, ty) ||
        !make_map(&mk, ca.k, D, ca.S, (long long)ca.B * ca.Nk, ty) ||
        !make_map(&mv, ca.v, D, ca.S, (long long)ca.B * ca.Nv, ty) ||
        !make_map(&mo, ca.out, D, ca.S, (long long)ca.B * ca.Nv, ty) ||
        !make_map(&mtp, ws, C, C, (long long)nch, ty))
        return cudaErrorInvalidValue;
    if (ca.final_state && !make_map(&mfs, ca.final_state, D, D, (long long)ca.B * ca.Nv, ty))
        return cudaErrorInvalidValue;
    ChainArgs a{};
    a.initial_state = ca.initial_state; a.final_state = ca.final_state; a.lengths = ca.lengths; a.scale = ca.scale;
    a.B = ca.B; a.Nk = ca.Nk; a.Nv = ca.Nv; a.S = ca.S; a.NC = NC;
    a.l2norm = ca.l2norm; a.eps = ca.eps; a.vec = vec; a.err = ca.err;
    a.epi_z = ca.epi_z; a.epi_w = ca.epi_w; a.epi_eps = ca.epi_eps;
    a.wait_ns = chunk_wait_ns();
    static LaunchCache plain(reinterpret_cast<const void *>(chain_kernel<T, kGate, false>));
    static LaunchCache ordered(reinterpret_cast<const void *>(chain_kernel<T, kGate, true>));
    const long long blocks = (long long)ca.B * ca.Nv;
    // longest sequences first only when the chains do not all start at once
    bool order = false;
    if (ca.lengths && ca.B > 1 && ca.B <= kRankMaxB) {
        int resident = 0;
        if ((e = ordered.resident_grid(CH_THREADS, (int)CH_SMEM, &resident)) != cudaSuccess) return e;
        order = blocks > resident;
    }
    if ((e = (order ? ordered : plain).allow_smem((int)CH_SMEM)) != cudaSuccess) return e;
    if (order)
        chain_kernel<T, kGate, true><<<(unsigned)blocks, CH_THREADS, CH_SMEM, stream>>>(mq, mk, mv, mo, mtp, mfs, a);
    else
        chain_kernel<T, kGate, false><<<(unsigned)blocks, CH_THREADS, CH_SMEM, stream>>>(mq, mk, mv, mo, mtp, mfs, a);
    return cudaGetLastError();
}
}  // namespace

#ifdef GDR_PHASE_TIMERS
extern "C" int gdr_phase_events_read(long long *out) {
    cudaDeviceSynchronize();
    cudaMemcpyFromSymbol(out, g_events, sizeof(long long) * kEvN * kEvK);
    cudaMemcpyFromSymbol(out + kEvN * kEvK, g_seen, sizeof(long long) * kEvN * 16);
    return kEvN * kEvK;
}
extern "C" int gdr_phase_timers_read(unsigned long long *out) {
    cudaDeviceSynchronize();
    cudaMemcpyFromSymbol(out, g_phase, sizeof(unsigned long long) * kTimerSlots);
    static unsigned long long z[kTimerSlots];
    cudaMemcpyToSymbol(g_phase, z, sizeof(z));
    return kTimerSlots;
}
#endif

cudaError_t chunk_wy_take_timeout_site(unsigned int *site) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(site, g_timeout_site, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_timeout_site, &zero, sizeof(unsigned int));
    return e;
}

cudaError_t launch_chunk_wy(const ChunkArgs &ca, gdr_dtype dt, cudaStream_t stream) {
    const bool gate = ca.g != nullptr;
    if (dt == GDR_F16) return gate ? launch_tc_t<__half, true>(ca, stream) : launch_tc_t<__half, false>(ca, stream);
    return gate ? launch_tc_t<__nv_bfloat16, true>(ca, stream) : launch_tc_t<__nv_bfloat16, false>(ca, stream);
}

}  // namespace gdr
