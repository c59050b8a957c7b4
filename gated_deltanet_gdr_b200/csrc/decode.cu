// decode.cu -- recurrent decode step of the gated delta rule over a slot pool.
//
// Operation (lite_boost recurrent_gated_delta_rule; torch_recurrent_gated_delta_rule
// token loop; deltanet.rs delta_step): per (sequence b, value head h) the state
// S = pool[idx[b*S]][h] (Dk x Dv) is read ONCE from HBM, the L_b tokens of the call are
// applied in fp32 registers (decay by exp(g) * exp(gk[i]) per row, readout k^T S, delta,
// rank-1 write, output q^T S), and the state is written back once per commit (normally
// once per call).
//
// The step is bound by HBM bandwidth: ~7 flops per state element per token against 2
// (bf16) or 4 (fp32) bytes read and written.  Design:
//   - a tile is (b, h, 64-column slab) of the state; a persistent CTA walks tiles
//     blockIdx.x, +gridDim.x, ... and keeps the NEXT tile's state and per-token rows in
//     flight (cp.async, 16-byte pieces, two shared-memory stages) while it computes the
//     current one, so HBM sees a continuous stream instead of load/compute/store waves;
//   - every thread fetches exactly the 16-byte pieces it will later use ("private slots"),
//     so the shared-memory reads back are conflict-free;
//   - the slot indices, lengths and per-token scalars of the tile after next are
//     prefetched into registers (no branch on a loaded value), and the next tile's are
//     checked before any of its state is requested;
//   - a warp owns 16 state columns, lane = (row group rg 0..15, column vector cv 0..1);
//     each warp prepares its own per-token vectors (norms of q and k, decay factors, v) in
//     registers with shuffle reductions, so the only block barriers are the two stage
//     hand-offs per tile;
//   - the column reductions k^T S' and q^T S' of the decayed state are taken in one pass
//     and finished by a 4-step xor butterfly inside the warp, and the output uses
//     o = q^T S' + (q . k) d, so no second pass over S is needed.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdr {

namespace {

constexpr int T = kDecodeMaxTokens;
constexpr uint64_t kDecodeDrainNs = 1000000000ull;  // bound of the drain after a timed-out wait

// explicit shared-memory loads (32-bit shared addresses), so that every operand read of the decode loop
// is a shared-memory access
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float lds_bf16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return __uint_as_float((uint32_t)v << 16);
}
__device__ __forceinline__ float lds_f16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return __half2float(__ushort_as_half(v));
}
template <typename T> __device__ __forceinline__ float lds_elem(uint32_t a);
template <> __device__ __forceinline__ float lds_elem<float>(uint32_t a) { return lds_f32(a); }
template <> __device__ __forceinline__ float lds_elem<__nv_bfloat16>(uint32_t a) { return lds_bf16(a); }
template <> __device__ __forceinline__ float lds_elem<__half>(uint32_t a) { return lds_f16(a); }
// the two 16-bit values packed in w (low half first) as floats
template <typename T> __device__ __forceinline__ void unpack2(uint32_t w, float &lo, float &hi);
template <> __device__ __forceinline__ void unpack2<__nv_bfloat16>(uint32_t w, float &lo, float &hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}
template <> __device__ __forceinline__ void unpack2<__half>(uint32_t w, float &lo, float &hi) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w));
    lo = f.x;
    hi = f.y;
}
template <> __device__ __forceinline__ void unpack2<float>(uint32_t, float &, float &) {}

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32)
__device__ __forceinline__ float exp2f_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <int DK, int DV, typename TI, typename TS> struct DecodeCfg {
    static constexpr int DVC = DV < 64 ? DV : 64;  // state columns per tile
    static constexpr int NSPLIT = DV / DVC;        // tiles per (b, h)
    static constexpr int NW = DVC / 16;            // warps per CTA, 16 columns each
    static constexpr int NT = NW * 32;
    static constexpr int RPT = DK / 16;            // state rows per lane
    static constexpr int PPS = 8 * (int)sizeof(TS) / 16;  // 16-byte pieces per 8 state columns
    // The state slab is staged row-major with rows padded by 32 bytes: copies between HBM and
    // shared memory move whole 128-byte lines (a warp covers 512 contiguous bytes per
    // instruction), while the per-thread reads in compute order (16 rows x 2 pieces per warp)
    // land on distinct banks.
    static constexpr int ROWB = DVC * (int)sizeof(TS);  // bytes of one slab row
    static constexpr int RS = ROWB + 32;                // padded row stride in shared memory
    static constexpr int CPR = ROWB / 16;               // 16-byte pieces per slab row
    static constexpr int SB_STATE = DK * RS;
    static constexpr int COPY_ITERS = DK * CPR / NT;    // pieces per thread per slab copy
    static_assert(DK % 16 == 0 && DV % 16 == 0, "head sizes must be multiples of 16");
    static_assert((DK * CPR) % NT == 0, "slab copy must split evenly");
    // per-token rows of a stage, sized by the call's S (and gk present or not)
    struct Layout {
        int off_q, off_k, off_v, off_gk, stage, off_meta, smem;
    };
    static __host__ __device__ Layout layout(int S, bool gk) {
        Layout l;
        l.off_q = SB_STATE;
        l.off_k = l.off_q + S * DK * (int)sizeof(TI);
        l.off_v = l.off_k + S * DK * (int)sizeof(TI);
        l.off_gk = l.off_v + S * DVC * (int)sizeof(TI);
        l.stage = l.off_gk + (gk ? S * DK * 4 : 0);
        l.stage = (l.stage + 127) & ~127;
        l.off_meta = 2 * l.stage;
        l.smem = l.off_meta + 3 * (2 + 3 * kDecodeMaxTokens) * 4;  // three scalar sets (see the kernel)
        return l;
    }
};

// Per-tile scalars live in shared memory: meta[0] = L, meta[1] = A, then idx[T], beta[T], g[T]
// (beta and g as raw bits).  Threads 0..T+1 prefetch them one tile ahead into registers
// (thread t < T: token t's idx, beta, g; thread T: L; thread T+1: A), with no branch on any
// loaded value, so the loads never stall the thread that issues them.
constexpr int META_INTS = 2 + 3 * T;

template <typename TI>
__device__ __forceinline__ void prefetch_meta(const DecodeArgs &a, int tile, int nsplit, int tid, int (&r)[3]) {
    const int bh = tile / nsplit, b = bh / a.Nv, S = a.S;
    r[0] = r[1] = r[2] = 0;
    if (tid < T) {
        if (tid < S) {
            r[0] = a.idx[(size_t)b * S + tid];
            r[1] = __float_as_int(to_f32(reinterpret_cast<const TI *>(a.beta)[(size_t)bh * S + tid]));
            if (a.g) r[2] = __float_as_int(a.g[(size_t)bh * S + tid]);
        }
    } else if (tid == T) {
        r[0] = a.lengths[b];
    } else if (tid == T + 1) {
        r[0] = a.accepted ? a.accepted[b] : (a.per_token ? 1 : a.lengths[b]);
    }
}
__device__ __forceinline__ void put_meta(int *mm, int tid, const int (&r)[3]) {
    if (tid < T) {
        mm[2 + tid] = r[0];
        mm[2 + T + tid] = r[1];
        mm[2 + 2 * T + tid] = r[2];
    } else if (tid == T) {
        mm[0] = r[0];
    } else if (tid == T + 1) {
        mm[1] = r[0];
    }
}
// 0 = process, 1 = bad length (or, per-token reading, an accepted count outside [1, S]), 2 = a referenced slot
// index out of range (same answer in every thread).  mm = (L, A, idx[T], ...).
__device__ __forceinline__ int tile_status(const int *mm, int S, int slots, int per_token) {
    const int L = mm[0], A = mm[1];
    if (L < 0 || L > S) return 1;
    if (per_token && L > 0) {  // the start slot is that of token A - 1; every processed token commits
        if (A < 1 || A > S) return 1;
        if (mm[2 + A - 1] < 0 || mm[2 + A - 1] >= slots) return 2;
        for (int t = 0; t < L; ++t)
            if (mm[2 + t] < 0 || mm[2 + t] >= slots) return 2;
        return 0;
    }
    int nref = min(L, A);
    if (L > 0 && nref < 1) nref = 1;
    for (int t = 0; t < nref; ++t)
        if (mm[2 + t] < 0 || mm[2 + t] >= slots) return 2;
    return 0;
}
// slot the chain starts from, and the number of leading tokens whose states are committed (a valid tile)
__device__ __forceinline__ int start_slot(const int *mm, int per_token) { return mm[2 + (per_token ? mm[1] - 1 : 0)]; }
__device__ __forceinline__ int commit_count(const int *mm, int Lv, int per_token) {
    return per_token ? Lv : min(mm[1], Lv);
}

template <int DK, int DV, typename TI, typename TS>
__global__ void __launch_bounds__(DecodeCfg<DK, DV, TI, TS>::NT)
decode_kernel(const DecodeArgs a, const int ntiles) {
    using Cf = DecodeCfg<DK, DV, TI, TS>;
    constexpr int DVC = Cf::DVC, NT = Cf::NT, RPT = Cf::RPT, PPS = Cf::PPS, RS = Cf::RS, CPR = Cf::CPR;
    extern __shared__ __align__(128) uint8_t smem[];
    const typename Cf::Layout ly = Cf::layout(a.S, a.gk != nullptr);
    int *s_meta = reinterpret_cast<int *>(smem + ly.off_meta);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cv = lane & 1, rg = lane >> 1;
    const int col = warp * 16 + cv * 8;  // first state column of this lane within the tile
    const int S = a.S;
    const size_t tile_elems = (size_t)DK * DV;

    // asynchronous copies of one tile into a stage, after its scalars were checked
    auto issue = [&](int tile, const int *mm, int stage) {
        uint8_t *st = smem + stage * ly.stage;
        const int split = tile % Cf::NSPLIT, bh = tile / Cf::NSPLIT, h = bh % a.Nv, b = bh / a.Nv;
        const int kh = h / (a.Nv / a.Nk), col0 = split * DVC;
        const int Lc = tile_status(mm, S, a.slots, a.per_token) ? 0 : mm[0];
        if (Lc > 0) {
            const uint8_t *src = reinterpret_cast<const uint8_t *>(
                reinterpret_cast<const TS *>(a.pool) + ((size_t)start_slot(mm, a.per_token) * a.Nv + h) * tile_elems +
                col0);
#pragma unroll
            for (int i = 0; i < Cf::COPY_ITERS; ++i) {
                const int e = i * NT + tid, row = e / CPR, pc = e % CPR;
                cp_async16(st + row * RS + pc * 16, src + (size_t)row * DV * sizeof(TS) + pc * 16);
            }
            const TI *qg = reinterpret_cast<const TI *>(a.q) + ((size_t)b * a.Nk + kh) * S * DK;
            const TI *kg = reinterpret_cast<const TI *>(a.k) + ((size_t)b * a.Nk + kh) * S * DK;
            const TI *vg = reinterpret_cast<const TI *>(a.v) + (size_t)bh * S * DV + col0;
            constexpr int QP = DK * (int)sizeof(TI) / 16, VP = DVC * (int)sizeof(TI) / 16, GP = DK * 4 / 16;
            for (int e = tid; e < Lc * QP; e += NT) {
                const int t = e / QP, pc = e % QP;
                cp_async16(st + ly.off_q + t * DK * sizeof(TI) + pc * 16,
                           reinterpret_cast<const uint8_t *>(qg + (size_t)t * DK) + pc * 16);
                cp_async16(st + ly.off_k + t * DK * sizeof(TI) + pc * 16,
                           reinterpret_cast<const uint8_t *>(kg + (size_t)t * DK) + pc * 16);
            }
            for (int e = tid; e < Lc * VP; e += NT) {
                const int t = e / VP, pc = e % VP;
                cp_async16(st + ly.off_v + t * DVC * sizeof(TI) + pc * 16,
                           reinterpret_cast<const uint8_t *>(vg + (size_t)t * DV) + pc * 16);
            }
            if (a.gk) {
                const float *gkg = a.gk + (size_t)bh * S * DK;
                for (int e = tid; e < Lc * GP; e += NT) {
                    const int t = e / GP, pc = e % GP;
                    cp_async16(st + ly.off_gk + t * DK * 4 + pc * 16,
                               reinterpret_cast<const uint8_t *>(gkg + (size_t)t * DK) + pc * 16);
                }
            }
        }
        cp_async_commit();
    };

    int tile = blockIdx.x;
    if (tile >= ntiles) return;
    int pre[3];
    prefetch_meta<TI>(a, tile, Cf::NSPLIT, tid, pre);
    put_meta(s_meta, tid, pre);
    __syncthreads();
    issue(tile, s_meta, 0);
    if (tile + (int)gridDim.x < ntiles) prefetch_meta<TI>(a, tile + gridDim.x, Cf::NSPLIT, tid, pre);

    // Stages alternate between two buffers; the scalar sets rotate over three, so a warp that has
    // finished tile j can already publish the scalars of tile j+1's successor while slower warps
    // still read tile j's: the only block barrier per tile is the one that makes the copies visible.
    for (int j = 0; tile < ntiles; ++j, tile += gridDim.x) {
        const int stg = j & 1;
        const int nxt = tile + gridDim.x;
        int *mn = s_meta + ((j + 1) % 3) * META_INTS;
        if (nxt < ntiles) put_meta(mn, tid, pre);
        cp_async_wait0();  // the current tile's copies (the only ones in flight)
        __syncthreads();
        if (nxt < ntiles) {
            issue(nxt, mn, stg ^ 1);
            if (nxt + (int)gridDim.x < ntiles) prefetch_meta<TI>(a, nxt + gridDim.x, Cf::NSPLIT, tid, pre);
        }

        // ---------------- process the current tile (each warp independently) ----------------
        const int *mm = s_meta + (j % 3) * META_INTS;
        const int split = tile % Cf::NSPLIT, bh = tile / Cf::NSPLIT, h = bh % a.Nv;
        const int col0 = split * DVC;
        const int status = tile_status(mm, S, a.slots, a.per_token);
        const int Lv = status ? 0 : mm[0];
        const int A = commit_count(mm, Lv, a.per_token);
        if (tid == 0 && status) raise_device_error(a.err, status == 1 ? GDR_DEVERR_LENGTH : GDR_DEVERR_SLOT_INDEX);
        TI *out = reinterpret_cast<TI *>(a.out) + (size_t)bh * S * DV + col0;
        for (int e = tid; e < (S - Lv) * (DVC / 8); e += NT) {
            const int t = Lv + e / (DVC / 8), c = (e % (DVC / 8)) * 8;
            float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            Vec8<TI>::store(out + (size_t)t * DV + c, z);
        }
        if (Lv > 0) {
            uint8_t *st = smem + stg * ly.stage;
            // this thread's rows rg + 16 r, columns col .. col + 7 of the padded slab
            auto slot = [&](int r) { return st + (rg + 16 * r) * RS + col * (int)sizeof(TS); };
            f2_t sv[RPT][4];  // the state as column pairs
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                float f[8];
                Vec8<TS>::load(reinterpret_cast<const TS *>(slot(r)), f);
#pragma unroll
                for (int p = 0; p < 4; ++p) sv[r][p] = pk2(f[2 * p], f[2 * p + 1]);
            }
            const float gA = a.A_log ? a.A_log[h] : 0.f, gB = a.A_log ? a.dt_bias[h] : 0.f;
            const int own_c = rg >> 1;          // after the reduce-scatter this lane owns column own_c
            const bool own_q = (rg & 1) != 0;   // ... of q^T S' (true) or of k^T S' (false)
            for (int t = 0; t < Lv; ++t) {
                // this lane's rows of q, k (and gk) for token t
                const TI *qr = reinterpret_cast<const TI *>(st + ly.off_q) + t * DK;
                const TI *kr = reinterpret_cast<const TI *>(st + ly.off_k) + t * DK;
                float xq[RPT], xk[RPT], dec[RPT];
                float ss_q = 0.f, ss_k = 0.f, qk = 0.f;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    xq[r] = to_f32(qr[rg + 16 * r]);
                    xk[r] = to_f32(kr[rg + 16 * r]);
                    ss_q = fmaf(xq[r], xq[r], ss_q);
                    ss_k = fmaf(xk[r], xk[r], ss_k);
                    qk = fmaf(xq[r], xk[r], qk);
                }
#pragma unroll
                for (int o = 2; o < 32; o <<= 1) {  // sums over all DK rows (the 16 row groups)
                    ss_q += __shfl_xor_sync(0xffffffffu, ss_q, o);
                    ss_k += __shfl_xor_sync(0xffffffffu, ss_k, o);
                    qk += __shfl_xor_sync(0xffffffffu, qk, o);
                }
                float qs = a.scale, kn = 1.f;
                if (a.l2norm) {
                    qs = a.scale * rsqrtf(ss_q + a.eps);
                    kn = rsqrtf(ss_k + a.eps);
                }
                qk *= qs * kn;
                const float graw = __int_as_float(mm[2 + 2 * T + t]);
                const float ag = a.g ? expf(a.A_log ? gate_from_raw(graw, gA, gB) : graw) : 1.f;
                const float *gkr = reinterpret_cast<const float *>(st + ly.off_gk) + t * DK;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    xq[r] *= qs;
                    xk[r] *= kn;
                    dec[r] = a.gk ? ag * expf(gkr[rg + 16 * r]) : ag;
                }
                const float braw = __int_as_float(mm[2 + T + t]);
                const float bt = a.beta_logits ? sigmoid_f32(braw) : braw;

                // decay, and both column readouts of the decayed state, two columns per op
                f2_t mk[4], mq[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) mk[p] = mq[p] = 0ull;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const f2_t d2 = pk2(dec[r], dec[r]), k2 = pk2(xk[r], xk[r]), q2 = pk2(xq[r], xq[r]);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const f2_t sd = mul2(sv[r][p], d2);
                        sv[r][p] = sd;
                        mk[p] = fma2(k2, sd, mk[p]);
                        mq[p] = fma2(q2, sd, mq[p]);
                    }
                }
                // reduce-scatter over the 16 row groups: value j = 2c + w (w = 0: k^T S', 1: q^T S')
                // ends fully summed in the lane with row group rg = j
                float v[16];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    up2(mk[p], v[4 * p], v[4 * p + 2]);
                    up2(mq[p], v[4 * p + 1], v[4 * p + 3]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const bool hi = lane & 16;
                    const float send = hi ? v[i] : v[8 + i], keep = hi ? v[8 + i] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool hi = lane & 8;
                    const float send = hi ? v[i] : v[4 + i], keep = hi ? v[4 + i] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const bool hi = lane & 4;
                    const float send = hi ? v[i] : v[2 + i], keep = hi ? v[2 + i] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                {
                    const bool hi = lane & 2;
                    const float send = hi ? v[0] : v[1], keep = hi ? v[1] : v[0];
                    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                }
                const float other = __shfl_xor_sync(0xffffffffu, v[0], 2);
                const float rk = own_q ? other : v[0], rq = own_q ? v[0] : other;
                const float vc = to_f32(reinterpret_cast<const TI *>(st + ly.off_v)[t * DVC + col + own_c]);
                const float dc = bt * (vc - rk);
                if (!own_q) out[(size_t)t * DV + col + own_c] = from_f32<TI>(fmaf(qk, dc, rq));
                float d[8];  // delta for this lane's 8 columns, from the lanes that own them
#pragma unroll
                for (int c = 0; c < 8; ++c) d[c] = __shfl_sync(0xffffffffu, dc, 4 * c + cv);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const f2_t k2 = pk2(xk[r], xk[r]);
#pragma unroll
                    for (int p = 0; p < 4; ++p) sv[r][p] = fma2(k2, pk2(d[2 * p], d[2 * p + 1]), sv[r][p]);
                }
                if (t < A && (t == A - 1 || mm[2 + t + 1] != mm[2 + t])) {
                    // commit straight from registers (each store covers 16 rows x 32 bytes per warp)
                    TS *dst = reinterpret_cast<TS *>(a.pool) + ((size_t)mm[2 + t] * a.Nv + h) * tile_elems + col0 + col;
#pragma unroll
                    for (int r = 0; r < RPT; ++r) {
                        float f[8];
#pragma unroll
                        for (int p = 0; p < 4; ++p) up2(sv[r][p], f[2 * p], f[2 * p + 1]);
                        Vec8<TS>::store(dst + (size_t)(rg + 16 * r) * DV, f);
                    }
                }
            }
        }
    }
    cp_async_wait0();
}

// ------------------------------------------------------------------------------------------------
// Dk = Dv = 128: one tile is a whole (sequence, value head) state.  A persistent CTA of four warps
// keeps up to NSTAGE tiles in flight (one TMA copy of the state slab plus one bulk copy per token
// array, on the stage's mbarrier) and computes one; warp w owns state columns [32 w, 32 w + 32),
// lane (rg = lane / 4, cv = lane % 4) rows rg + 8 r (r = 0..15) and columns 32 w + 8 cv .. + 7, so a
// thread holds 128 state values and the per-token work (norms, gate, reductions) is spread over twice
// as many elements as in the general kernel.  The gate e^g and beta are computed once per tile by
// the scalar threads.  After the three-level reduce-scatter over the row groups, lane (rg, cv) holds
// both readouts k^T S' and q^T S' of column 32 w + 8 cv + rg, so it computes that column's delta and
// output directly.
template <typename TI, typename TS, int NW, int NSTG> struct D128 {
    static constexpr int D = 128, NT = 32 * NW;
    static constexpr int NCV = 16 / NW;           // 8-column vectors per warp (lanes per row group)
    static constexpr int NRG = 32 / NCV;          // row groups per warp
    static constexpr int RPT = D / NRG;           // state rows per thread (16 or 8)
    static constexpr int NSTAGE = NSTG;
    static constexpr int BOXC = 128 / (int)sizeof(TS);  // state columns per 128-byte box row
    static constexpr int NBOX = D / BOXC;                // boxes per state slab (2 for bf16, 4 for fp32)
    static constexpr int STATE_BYTES = D * D * (int)sizeof(TS);
    struct Layout {
        int off_q, off_k, off_v, off_gk, stage, off_bar, off_meta, smem;
    };
    static __host__ __device__ Layout layout(int S, bool gk) {
        Layout l;
        l.off_q = STATE_BYTES;
        l.off_k = l.off_q + S * D * (int)sizeof(TI);
        l.off_v = l.off_k + S * D * (int)sizeof(TI);
        l.off_gk = l.off_v + S * D * (int)sizeof(TI);
        const int end = l.off_gk + (gk ? S * D * 4 : 0);
        l.stage = (end + 1023) & ~1023;  // the TMA destinations stay 1024-byte aligned
        l.off_bar = NSTAGE * l.stage;     // NSTAGE "full" then NSTAGE "empty" mbarriers
        l.off_meta = l.off_bar + 64;
        l.smem = l.off_meta + 4 * META_INTS * 4 + 1024;  // four scalar sets, + alignment slack
        return l;
    }
};

// Raw per-tile scalars, prefetched one tile ahead into registers by threads 0..T+1 (no branch on a
// loaded value): thread t < T: idx[b S + t], raw beta, raw gate, A_log[h], dt_bias[h]; thread T: L;
// thread T+1: A.
template <typename TI>
__device__ __forceinline__ void prefetch_meta128(const DecodeArgs &a, int bh, int tid, int (&r)[5]) {
    const int b = bh / a.Nv, h = bh % a.Nv, S = a.S;
    r[0] = r[1] = r[2] = r[3] = r[4] = 0;
    if (tid < T) {
        if (tid < S) {
            r[0] = a.idx[(size_t)b * S + tid];
            r[1] = __float_as_int(to_f32(reinterpret_cast<const TI *>(a.beta)[(size_t)bh * S + tid]));
            if (a.g) r[2] = __float_as_int(a.g[(size_t)bh * S + tid]);
            if (a.A_log) {
                r[3] = __float_as_int(a.A_log[h]);
                r[4] = __float_as_int(a.dt_bias[h]);
            }
        }
    } else if (tid == T) {
        r[0] = a.lengths[b];
    } else if (tid == T + 1) {
        r[0] = a.accepted ? a.accepted[b] : (a.per_token ? 1 : a.lengths[b]);
    }
}
// The set layout of put_meta (L, A, idx[T], beta[T], g[T]), with beta and the decay e^g final.
__device__ __forceinline__ void put_meta128(const DecodeArgs &a, int *mm, int tid, const int (&r)[5]) {
    if (tid < T) {
        mm[2 + tid] = r[0];
        const float braw = __int_as_float(r[1]), graw = __int_as_float(r[2]);
        mm[2 + T + tid] = __float_as_int(a.beta_logits ? sigmoid_f32(braw) : braw);
        const float g = a.A_log ? gate_from_raw(graw, __int_as_float(r[3]), __int_as_float(r[4])) : graw;
        mm[2 + 2 * T + tid] = __float_as_int(a.g ? expf(g) : 1.f);
    } else if (tid == T) {
        mm[0] = r[0];
    } else if (tid == T + 1) {
        mm[1] = r[0];
    }
}

// kDecay = false: the build for g = NULL and gk = NULL (no decay), which never rescales the state.
template <typename TI, typename TS, int NW, int NSTG, int MINB, bool kDecay>
__global__ void __launch_bounds__(32 * NW, MINB)
decode128_kernel(const __grid_constant__ CUtensorMap tm_pool, const DecodeArgs a, const int ntiles) {
    using Cf = D128<TI, TS, NW, NSTG>;
    constexpr int NCV = Cf::NCV, NRG = Cf::NRG, RPT = Cf::RPT;
    constexpr int D = Cf::D, NS = Cf::NSTAGE;
    extern __shared__ __align__(1024) uint8_t smraw[];
    uint8_t *smem = smraw + ((1024u - (sm100::smem_u32(smraw) & 1023u)) & 1023u);
    const typename Cf::Layout ly = Cf::layout(a.S, a.gk != nullptr);
    // full[s]: stage s holds its tile (TMA / bulk transactions); empty[s]: the four warps are done with it
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + ly.off_bar), *empty = full + NS;
    int *s_meta = reinterpret_cast<int *>(smem + ly.off_meta);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = lane / NCV, cv = lane % NCV;
    const int c0 = 8 * NCV * warp + 8 * cv;  // first state column of this thread
    const int S = a.S;
    // byte offset of this thread's 8 columns of row rg (row rg + NRG r is 128 NRG r further): the 128-byte
    // swizzle XORs the 16-byte chunk index with the row index modulo 8, which is rg % 8 for every row here
    const int box = c0 / Cf::BOXC, ch0 = (c0 % Cf::BOXC) * (int)sizeof(TS) / 16, sw = rg & 7;
    const int soff = box * (D * 128) + rg * 128 + ((ch0 ^ sw) << 4);
    const int soff2 = box * (D * 128) + rg * 128 + (((ch0 + 1) ^ sw) << 4);  // second chunk (fp32 state)

    // tiles thread 0 has issued; the i-th went to stage i % NS (for the drain after a timeout)
    int n_issued = 0;
    // checked copies of a tile into stage `st` (thread 0): the state slab by TMA, the token rows by bulk copies
    auto issue = [&](int tile, const int *mm, int st) {
        uint64_t *bar = full + st;
        ++n_issued;
        uint8_t *base = smem + st * ly.stage;
        const int status = tile_status(mm, S, a.slots, a.per_token);
        const int Lc = status ? 0 : mm[0];
        if (Lc <= 0) {
            sm100::mbar_arrive(bar);
            return;
        }
        const int h = tile % a.Nv, b = tile / a.Nv, kh = h / (a.Nv / a.Nk);
        const uint32_t tok = (uint32_t)Lc * D * (uint32_t)sizeof(TI);
        sm100::mbar_arrive_expect_tx(bar, Cf::STATE_BYTES + 3 * tok + (a.gk ? (uint32_t)Lc * D * 4 : 0));
        const int z = start_slot(mm, a.per_token) * a.Nv + h;
#pragma unroll
        for (int x = 0; x < Cf::NBOX; ++x) sm100::tma_load_3d(base + x * (D * 128), &tm_pool, bar, x * Cf::BOXC, 0, z);
        const size_t qk_off = ((size_t)b * a.Nk + kh) * S * D, v_off = (size_t)tile * S * D;
        sm100::bulk_load(base + ly.off_q, reinterpret_cast<const TI *>(a.q) + qk_off, tok, bar);
        sm100::bulk_load(base + ly.off_k, reinterpret_cast<const TI *>(a.k) + qk_off, tok, bar);
        sm100::bulk_load(base + ly.off_v, reinterpret_cast<const TI *>(a.v) + v_off, tok, bar);
        if (a.gk) sm100::bulk_load(base + ly.off_gk, a.gk + v_off, (uint32_t)Lc * D * 4, bar);
    };

    int tile = blockIdx.x;
    if (tile >= ntiles) return;
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            sm100::mbar_init(full + i, 1);
            sm100::mbar_init(empty + i, Cf::NT / 32);
        }
        sm100::fence_mbar_init();
        sm100::prefetch_tmap(&tm_pool);
    }
    // prologue: scalars of the first NS + 1 tiles, copies of the first NS
    int pre[5];
    for (int i = 0; i <= NS; ++i) {
        const int ti = tile + i * (int)gridDim.x;
        if (ti < ntiles) {
            prefetch_meta128<TI>(a, ti, tid, pre);
            put_meta128(a, s_meta + (i & 3) * META_INTS, tid, pre);
        }
    }
    __syncthreads();
    if (tid == 0)
        for (int i = 0; i < NS; ++i) {
            const int ti = tile + i * (int)gridDim.x;
            if (ti < ntiles) issue(ti, s_meta + (i & 3) * META_INTS, i);
        }
    // raw scalars of the next two tiles to publish (tiles j + NS + 1 and j + NS + 2 at iteration j), so
    // that their global loads have a whole tile of time to land before they are used
    int pre2[5] = {0, 0, 0, 0, 0};
    {
        const int ti = tile + (NS + 1) * (int)gridDim.x, ti2 = ti + (int)gridDim.x;
        if (ti < ntiles) prefetch_meta128<TI>(a, ti, tid, pre);
        if (ti2 < ntiles) prefetch_meta128<TI>(a, ti2, tid, pre2);
    }
    bool timed_out = false;

    for (int j = 0; tile < ntiles; ++j, tile += gridDim.x) {
        const int st = j % NS;
        const int *mm = s_meta + (j & 3) * META_INTS;
        const int h = tile % a.Nv;
        const int status = tile_status(mm, S, a.slots, a.per_token);
        const int Lv = status ? 0 : mm[0];
        const int A = commit_count(mm, Lv, a.per_token);
        if (tid == 0 && status) raise_device_error(a.err, status == 1 ? GDR_DEVERR_LENGTH : GDR_DEVERR_SLOT_INDEX);
        TI *out = reinterpret_cast<TI *>(a.out) + (size_t)tile * S * D;
        for (int e = tid; e < (S - Lv) * (D / 8); e += Cf::NT) {
            const int t = Lv + e / (D / 8), c = (e % (D / 8)) * 8;
            float zz[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            Vec8<TI>::store(out + (size_t)t * D + c, zz);
        }
        if (!sm100::mbar_wait_ns(full + st, (uint32_t)(j / NS) & 1u, a.wait_ns)) timed_out = true;
        if (Lv > 0 && !timed_out) {
            const uint8_t *base = smem + st * ly.stage;
            const uint32_t sb = sm100::smem_u32(base);
            f2_t sv[RPT][4];
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                float f[8];
                if (sizeof(TS) == 2) {
                    const uint4 u = lds128(sb + soff + r * NRG * 128);
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) unpack2<TS>(w4[i], f[2 * i], f[2 * i + 1]);
                } else {
                    const uint4 u0 = lds128(sb + soff + r * NRG * 128), u1 = lds128(sb + soff2 + r * NRG * 128);
                    f[0] = __uint_as_float(u0.x); f[1] = __uint_as_float(u0.y);
                    f[2] = __uint_as_float(u0.z); f[3] = __uint_as_float(u0.w);
                    f[4] = __uint_as_float(u1.x); f[5] = __uint_as_float(u1.y);
                    f[6] = __uint_as_float(u1.z); f[7] = __uint_as_float(u1.w);
                }
#pragma unroll
                for (int p = 0; p < 4; ++p) sv[r][p] = pk2(f[2 * p], f[2 * p + 1]);
            }
            const uint32_t sq = sb + ly.off_q + rg * (int)sizeof(TI), sk = sb + ly.off_k + rg * (int)sizeof(TI);
            const uint32_t sgk = sb + ly.off_gk + rg * 4, svv = sb + ly.off_v;
            // the column whose readouts this lane ends up with (with 16 row groups, lanes rg and rg ^ 1 share
            // a column: rg even holds k^T S', rg odd q^T S', exchanged below)
            const int own = c0 + (NRG == 8 ? rg : rg >> 1);
            for (int t = 0; t < Lv; ++t) {
                const uint32_t qrow = sq + t * D * (int)sizeof(TI), krow = sk + t * D * (int)sizeof(TI);
                float xq[RPT], xk[RPT];
                float ss_q = 0.f, ss_k = 0.f, qk = 0.f;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    xq[r] = lds_elem<TI>(qrow + NRG * r * (int)sizeof(TI));
                    xk[r] = lds_elem<TI>(krow + NRG * r * (int)sizeof(TI));
                    ss_q = fmaf(xq[r], xq[r], ss_q);
                    ss_k = fmaf(xk[r], xk[r], ss_k);
                    qk = fmaf(xq[r], xk[r], qk);
                }
#pragma unroll
                for (int o = NCV; o < 32; o <<= 1) {  // sums over the row groups
                    ss_q += __shfl_xor_sync(0xffffffffu, ss_q, o);
                    ss_k += __shfl_xor_sync(0xffffffffu, ss_k, o);
                    qk += __shfl_xor_sync(0xffffffffu, qk, o);
                }
                float qs = a.scale, kn = 1.f;
                if (a.l2norm) {
                    qs = a.scale * rsqrtf(ss_q + a.eps);
                    kn = rsqrtf(ss_k + a.eps);
                }
                qk *= qs * kn;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    xq[r] *= qs;
                    xk[r] *= kn;
                }
                const float ag = __int_as_float(mm[2 + 2 * T + t]), bt = __int_as_float(mm[2 + T + t]);
                // decay (and, with gk, the per-row factor e^{gk} = 2^{gk log2 e} on the special-function
                // unit), and both column readouts of the decayed state
                f2_t mk[4], mq[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) mk[p] = mq[p] = 0ull;
                const uint32_t gkrow = sgk + t * D * 4;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const f2_t k2 = pk2(xk[r], xk[r]), q2 = pk2(xq[r], xq[r]);
                    if (kDecay) {
                        const float dr =
                            a.gk ? ag * exp2f_approx(lds_f32(gkrow + NRG * r * 4) * 1.4426950408889634f) : ag;
                        const f2_t d2 = pk2(dr, dr);
#pragma unroll
                        for (int p = 0; p < 4; ++p) sv[r][p] = mul2(sv[r][p], d2);
                    }
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        mk[p] = fma2(k2, sv[r][p], mk[p]);
                        mq[p] = fma2(q2, sv[r][p], mq[p]);
                    }
                }
                // reduce-scatter over the row groups (lane bits 2..4): value i = 2c + w (column c of the 8,
                // w = 0: k^T S', 1: q^T S') ends summed in the lane with rg = c
                float v[16];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    up2(mk[p], v[4 * p], v[4 * p + 2]);
                    up2(mq[p], v[4 * p + 1], v[4 * p + 3]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const bool hi = lane & 16;
                    const float send = hi ? v[i] : v[8 + i], keep = hi ? v[8 + i] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool hi = lane & 8;
                    const float send = hi ? v[i] : v[4 + i], keep = hi ? v[4 + i] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const bool hi = lane & 4;
                    const float send = hi ? v[i] : v[2 + i], keep = hi ? v[2 + i] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                float rk, rq;
                if (NRG == 8) {
                    rk = v[0];
                    rq = v[1];
                } else {  // one more level (lane bit 1), then the two halves of the column swap
                    const bool hi = lane & 2;
                    const float send = hi ? v[0] : v[1], keep = hi ? v[1] : v[0];
                    const float mine = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    const float other = __shfl_xor_sync(0xffffffffu, mine, 2);
                    rk = hi ? other : mine;
                    rq = hi ? mine : other;
                }
                const float vc = lds_elem<TI>(svv + (t * D + own) * (int)sizeof(TI));
                const float dc = bt * (vc - rk);
                if (NRG == 8 || !(lane & 2)) out[(size_t)t * D + own] = from_f32<TI>(fmaf(qk, dc, rq));
                float d[8];  // delta for this thread's 8 columns, from the lanes that own them
#pragma unroll
                for (int c = 0; c < 8; ++c) d[c] = __shfl_sync(0xffffffffu, dc, 4 * c + cv);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const f2_t k2 = pk2(xk[r], xk[r]);
#pragma unroll
                    for (int p = 0; p < 4; ++p) sv[r][p] = fma2(k2, pk2(d[2 * p], d[2 * p + 1]), sv[r][p]);
                }
                if (t < A && (t == A - 1 || mm[2 + t + 1] != mm[2 + t])) {
                    // commit straight from registers
                    TS *dst = reinterpret_cast<TS *>(a.pool) + ((size_t)mm[2 + t] * a.Nv + h) * (D * D) + c0;
#pragma unroll
                    for (int r = 0; r < RPT; ++r) {
                        float f[8];
#pragma unroll
                        for (int p = 0; p < 4; ++p) up2(sv[r][p], f[2 * p], f[2 * p + 1]);
                        Vec8<TS>::store(dst + (size_t)(rg + NRG * r) * D, f);
                    }
                }
            }
        }
        // Each warp releases the stage (and the tile's scalar set) on its own; only warp 0 waits until all
        // four are done, then refills the stage with tile j + NS (whose scalars it published an iteration
        // ago) and publishes the scalars of tile j + NS + 1 into the freed set (four sets: tiles j .. j + NS
        // are live).  The other warps go straight on to their next tile.
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(empty + st);
        if (timed_out) break;
        if (warp == 0) {
            const int nxt = tile + NS * (int)gridDim.x;
            if (!sm100::mbar_wait_ns(empty + st, (uint32_t)(j / NS) & 1u, a.wait_ns)) {
                timed_out = true;
                break;
            }
            if (nxt + (int)gridDim.x < ntiles) put_meta128(a, s_meta + ((j + NS + 1) & 3) * META_INTS, tid, pre);
            __syncwarp();
            if (tid == 0 && nxt < ntiles) issue(nxt, s_meta + ((j + NS) & 3) * META_INTS, st);
#pragma unroll
            for (int i = 0; i < 5; ++i) pre[i] = pre2[i];
            if (nxt + 3 * (int)gridDim.x < ntiles) prefetch_meta128<TI>(a, nxt + 3 * gridDim.x, tid, pre2);
        }
    }
    if (timed_out && tid == 0) {
        // drain: each stage's last armed phase (the only one that can still be in flight) has landed before the
        // CTA leaves, so no copy writes into the shared memory of a later CTA
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int phases = n_issued > i ? (n_issued - 1 - i) / NS + 1 : 0;  // issues that went to stage i
            if (phases) sm100::mbar_wait_ns(full + i, (uint32_t)(phases - 1) & 1u, kDecodeDrainNs);
        }
        raise_device_error(a.err, GDR_DEVERR_TIMEOUT);
    }
}

template <typename TI, typename TS>
cudaError_t launch_decode128(const DecodeArgs &a, cudaStream_t stream) {
#ifndef GDR_DEC_NSTG
#define GDR_DEC_NSTG 3
#define GDR_DEC_MINB 2
#endif
    constexpr int NW = 4, NSTG = sizeof(TS) == 2 ? GDR_DEC_NSTG : 2, MINB = GDR_DEC_MINB;
    using Cf = D128<TI, TS, NW, NSTG>;
    const long long ntiles = (long long)a.B * a.Nv;
    if (ntiles == 0) return cudaSuccess;
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap tm;
    const cuuint64_t dims[3] = {(cuuint64_t)Cf::D, (cuuint64_t)Cf::D, (cuuint64_t)a.slots * (cuuint64_t)a.Nv};
    const cuuint64_t strides[2] = {(cuuint64_t)Cf::D * sizeof(TS), (cuuint64_t)Cf::D * Cf::D * sizeof(TS)};
    const cuuint32_t box[3] = {(cuuint32_t)Cf::BOXC, (cuuint32_t)Cf::D, 1}, es[3] = {1, 1, 1};
    const CUtensorMapDataType tmt = sizeof(TS) == 4                        ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                    : std::is_same<TS, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (enc(&tm, tmt, 3, a.pool, dims,
            strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kern = (a.g || a.gk) ? decode128_kernel<TI, TS, NW, NSTG, MINB, true>
                              : decode128_kernel<TI, TS, NW, NSTG, MINB, false>;
    const int smem = Cf::layout(a.S, a.gk != nullptr).smem;
    static LaunchCache cache_decay(reinterpret_cast<const void *>(decode128_kernel<TI, TS, NW, NSTG, MINB, true>));
    static LaunchCache cache_plain(reinterpret_cast<const void *>(decode128_kernel<TI, TS, NW, NSTG, MINB, false>));
    LaunchCache &cache = (a.g || a.gk) ? cache_decay : cache_plain;
    cudaError_t e = cache.allow_smem(smem);
    if (e != cudaSuccess) return e;
    int grid_cap = 1;
    e = cache.resident_grid(Cf::NT, smem, &grid_cap);
    if (e != cudaSuccess) return e;
    const int grid = (int)(ntiles < grid_cap ? ntiles : grid_cap);
    kern<<<grid, Cf::NT, smem, stream>>>(tm, a, (int)ntiles);
    return cudaGetLastError();
}

template <int DK, int DV, typename TI, typename TS>
cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t stream) {
    using Cf = DecodeCfg<DK, DV, TI, TS>;
    const long long ntiles = (long long)a.B * a.Nv * Cf::NSPLIT;
    if (ntiles == 0) return cudaSuccess;
    auto kern = decode_kernel<DK, DV, TI, TS>;
    const int smem = Cf::layout(a.S, a.gk != nullptr).smem;
    // a persistent grid of the CTAs resident at once for this shared-memory size (tiles are independent, so
    // an overestimate would only queue extra CTAs)
    static LaunchCache cache(reinterpret_cast<const void *>(kern));
    cudaError_t e = cache.allow_smem(smem);
    if (e != cudaSuccess) return e;
    int grid_cap = 1;
    e = cache.resident_grid(Cf::NT, smem, &grid_cap);
    if (e != cudaSuccess) return e;
    const int grid = (int)(ntiles < grid_cap ? ntiles : grid_cap);
    kern<<<grid, Cf::NT, smem, stream>>>(a, (int)ntiles);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_decode_d(const DecodeArgs &a, gdr_dtype dt, gdr_dtype st, cudaStream_t stream) {
    // fp16 inputs take an fp16 or fp32 state
    if (dt == GDR_F16 && st != GDR_F16 && st != GDR_F32) return cudaErrorInvalidValue;
    if (DK == 128 && DV == 128) {
        if (dt == GDR_F16 && st == GDR_F16) return launch_decode128<__half, __half>(a, stream);
        if (dt == GDR_F16) return launch_decode128<__half, float>(a, stream);
        if (dt == GDR_BF16 && st == GDR_BF16) return launch_decode128<__nv_bfloat16, __nv_bfloat16>(a, stream);
        if (dt == GDR_BF16 && st == GDR_F32) return launch_decode128<__nv_bfloat16, float>(a, stream);
        if (dt == GDR_F32 && st == GDR_BF16) return launch_decode128<float, __nv_bfloat16>(a, stream);
        return launch_decode128<float, float>(a, stream);
    }
    if (dt == GDR_F16 && st == GDR_F16) return launch_decode_t<DK, DV, __half, __half>(a, stream);
    if (dt == GDR_F16) return launch_decode_t<DK, DV, __half, float>(a, stream);
    if (dt == GDR_BF16 && st == GDR_BF16) return launch_decode_t<DK, DV, __nv_bfloat16, __nv_bfloat16>(a, stream);
    if (dt == GDR_BF16 && st == GDR_F32) return launch_decode_t<DK, DV, __nv_bfloat16, float>(a, stream);
    if (dt == GDR_F32 && st == GDR_BF16) return launch_decode_t<DK, DV, float, __nv_bfloat16>(a, stream);
    return launch_decode_t<DK, DV, float, float>(a, stream);
}

template <int DK>
cudaError_t launch_decode_k(const DecodeArgs &a, int Dv, gdr_dtype dt, gdr_dtype st, cudaStream_t s) {
    switch (Dv) {
        case 16: return launch_decode_d<DK, 16>(a, dt, st, s);
        case 32: return launch_decode_d<DK, 32>(a, dt, st, s);
        case 64: return launch_decode_d<DK, 64>(a, dt, st, s);
        default: return launch_decode_d<DK, 128>(a, dt, st, s);
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, int Dk, int Dv, gdr_dtype dt, gdr_dtype st, cudaStream_t s) {
    switch (Dk) {
        case 16: return launch_decode_k<16>(a, Dv, dt, st, s);
        case 32: return launch_decode_k<32>(a, Dv, dt, st, s);
        case 64: return launch_decode_k<64>(a, Dv, dt, st, s);
        default: return launch_decode_k<128>(a, Dv, dt, st, s);
    }
}

}  // namespace gdr
