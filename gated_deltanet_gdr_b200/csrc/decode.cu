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
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdr {

namespace {

constexpr int T = kDecodeMaxTokens;

// packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction updates two state columns
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t pk2(float lo, float hi) {
    f2_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ void up2(f2_t v, float &lo, float &hi) { asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v)); }
__device__ __forceinline__ f2_t mul2(f2_t a, f2_t b) {
    f2_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2_t fma2(f2_t a, f2_t b, f2_t c) {
    f2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
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
        r[0] = a.accepted ? a.accepted[b] : a.lengths[b];
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
// 0 = process, 1 = bad length, 2 = a referenced slot index out of range (same answer in every thread)
__device__ __forceinline__ int tile_status(const int *mm, int S, int slots) {
    const int L = mm[0], A = mm[1];
    if (L < 0 || L > S) return 1;
    int nref = min(L, A);
    if (L > 0 && nref < 1) nref = 1;
    for (int t = 0; t < nref; ++t)
        if (mm[2 + t] < 0 || mm[2 + t] >= slots) return 2;
    return 0;
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
        const int Lc = tile_status(mm, S, a.slots) ? 0 : mm[0];
        if (Lc > 0) {
            const uint8_t *src = reinterpret_cast<const uint8_t *>(
                reinterpret_cast<const TS *>(a.pool) + ((size_t)mm[2] * a.Nv + h) * tile_elems + col0);
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
        const int status = tile_status(mm, S, a.slots);
        const int Lv = status ? 0 : mm[0];
        const int A = min(mm[1], Lv);
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

template <int DK, int DV, typename TI, typename TS>
cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t stream) {
    using Cf = DecodeCfg<DK, DV, TI, TS>;
    const long long ntiles = (long long)a.B * a.Nv * Cf::NSPLIT;
    if (ntiles == 0) return cudaSuccess;
    auto kern = decode_kernel<DK, DV, TI, TS>;
    const int smem = Cf::layout(a.S, a.gk != nullptr).smem;
    // resident CTAs on the device for this shared-memory size (all B200s have the same count),
    // cached per instantiation and size; an overestimate would only queue extra CTAs, since
    // tiles are independent
    static int attr_smem = 0, cached_smem = -1, grid_cap = 1;
    if (smem > attr_smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_smem = smem;
    }
    if (smem != cached_smem) {
        int dev = 0, nsm = 0, per_sm = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cf::NT, smem);
        grid_cap = max(1, nsm * max(1, per_sm));
        cached_smem = smem;
    }
    const int grid = (int)(ntiles < grid_cap ? ntiles : grid_cap);
    kern<<<grid, Cf::NT, smem, stream>>>(a, (int)ntiles);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_decode_d(const DecodeArgs &a, gdr_dtype dt, gdr_dtype st, cudaStream_t stream) {
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
