// api.cu -- the C ABI of libgdr.so: argument checks, dispatch, device error word.
//
// Every entry point validates its arguments on the host before touching the GPU; on a
// non-zero status nothing has been launched.  The library allocates no device memory.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/gdr.h"
#include "kernels.h"

namespace gdr {

// The device error word (GDR_DEVERR_* bits) of this library, one per device.
__device__ unsigned int g_device_error = 0;
// Snapshots of the error word taken by gdr_get_error, one slot per concurrent call (a call takes the next slot
// round-robin, so calls on different streams or host threads do not share one).
constexpr int kErrSlots = 64;
__device__ unsigned int g_error_snapshot[kErrSlots];

// Reads and clears the error word in one atomic step, so no bit raised meanwhile by another stream's kernel is lost.
__global__ void take_error_kernel(unsigned int *err, unsigned int *slot) { *slot = atomicExch(err, 0u); }

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_dev_checked[kMaxDevices];        // 0 unknown, 1 sm_100, -1 unusable
unsigned int *g_err_ptr[kMaxDevices];  // device address of g_device_error per device
unsigned int *g_snap_ptr[kMaxDevices]; // device address of g_error_snapshot per device
unsigned int g_snap_next = 0;          // next snapshot slot (under g_mu)

int g_sm_count[kMaxDevices];           // multiprocessors per device (0 until first asked)
int g_chunk_schedule = 0;              // tensor-core prefill schedule: 0 by shape, 1 one kernel, 2 two kernels

bool supported_head(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// Multiprocessors of the current device; 148 (a full B200) when no device can be asked, so that the workspace
// query answers the same on a machine without a GPU.
int sm_count() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 148;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            return 148;
        }
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

// The tensor-core prefill's two-kernel schedule (a WY pass over every chunk on every SM, then the chains) pays
// off when the (b, value head) chains occupy at most a third of the SMs: the one-kernel schedule would leave the
// rest idle while each chain solves its chunks' WY systems in turn.  With more chains the one-kernel schedule,
// which needs no workspace, is faster.
bool two_kernel_schedule(int B, int Nv) {
    if (g_chunk_schedule == 1) return false;
    if (g_chunk_schedule == 2) return true;
    return (long long)B * Nv * 3 <= sm_count();
}
bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks the current device once (sm_100 family) and fetches the address of the error
// word on it.  Returns GDR_OK, GDR_ERR_DEVICE or GDR_ERR_LAUNCH.
int device_setup(unsigned int **err) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return GDR_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_dev_checked[dev] == 0) {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return GDR_ERR_DEVICE;
        }
        if (major != 10) {
            g_dev_checked[dev] = -1;
            return GDR_ERR_DEVICE;
        }
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) {
            cudaGetLastError();
            return GDR_ERR_LAUNCH;
        }
        g_err_ptr[dev] = static_cast<unsigned int *>(p);
        if (cudaGetSymbolAddress(&p, g_error_snapshot) != cudaSuccess) {
            cudaGetLastError();
            return GDR_ERR_LAUNCH;
        }
        g_snap_ptr[dev] = static_cast<unsigned int *>(p);
        g_dev_checked[dev] = 1;
    }
    if (g_dev_checked[dev] < 0) return GDR_ERR_DEVICE;
    *err = g_err_ptr[dev];
    return GDR_OK;
}

int check_common(int B, int Nk, int Nv, int S, int Dk, int Dv, int dtype) {
    if (dtype != GDR_F32 && dtype != GDR_BF16 && dtype != GDR_F16) return GDR_ERR_DTYPE;
    if (B < 0 || S < 0 || Nk < 1 || Nv < 1 || Dk < 1 || Dv < 1) return GDR_ERR_SHAPE;
    if (Nv % Nk != 0) return GDR_ERR_SHAPE;
    if (!supported_head(Dk) || !supported_head(Dv)) return GDR_ERR_UNSUPPORTED;
    // grids are one-dimensional: B * Nv * (column slabs) blocks
    if ((long long)B * Nv * 8 >= (1LL << 31)) return GDR_ERR_SHAPE;
    return GDR_OK;
}

int check_prologue(const gdr_prologue *p, const float *g) {
    if (!p) return GDR_OK;
    if (p->A_log && (!p->dt_bias || !g)) return GDR_ERR_NULL;
    if (p->l2norm_qk && !(p->eps >= 0.f)) return GDR_ERR_SHAPE;
    return GDR_OK;
}

// ---- checked mode (environment variable GDR_CHECKS=1): host-side validation of the index and length arrays ----
// The kernels never trap on bad lengths or slots (they skip the sequence and flag the error word), and two
// sequences that share a slot race silently.  In checked mode the library copies the arrays to the host before
// launching (a synchronisation on the caller's stream, so for debugging only) and rejects such calls with
// GDR_ERR_SHAPE.
bool checks_enabled() {
    const char *v = std::getenv("GDR_CHECKS");
    return v && v[0] && std::strcmp(v, "0") != 0;
}

bool copy_i32(std::vector<int32_t> &h, const int32_t *d, size_t n, cudaStream_t s) {
    h.assign(n, 0);
    if (n == 0 || !d) return true;
    if (cudaMemcpyAsync(h.data(), d, n * sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess) return false;
    return cudaStreamSynchronize(s) == cudaSuccess;
}

// lengths within [0, S]
int check_lengths_host(const int32_t *lengths, int B, int S, cudaStream_t s) {
    if (!lengths) return GDR_OK;
    std::vector<int32_t> L;
    if (!copy_i32(L, lengths, (size_t)B, s)) return GDR_ERR_LAUNCH;
    for (int b = 0; b < B; ++b)
        if (L[b] < 0 || L[b] > S) return GDR_ERR_SHAPE;
    return GDR_OK;
}

// Decode: lengths in [0, S], accepted counts in range, every slot a sequence reads or writes in [0, slots), and
// no slot touched by two sequences.  per_token selects the speculative-decoding reading (the chain starts at token
// A - 1's slot and every processed token's state goes to its own slot); otherwise the chain starts at token 0's
// slot and the first min(A, L) states are committed.
int check_decode_host(const int32_t *idx, const int32_t *lengths, const int32_t *accepted, int B, int S, int slots,
                      int per_token, cudaStream_t s) {
    std::vector<int32_t> I, L, A;
    if (!copy_i32(I, idx, (size_t)B * S, s) || !copy_i32(L, lengths, (size_t)B, s) ||
        !copy_i32(A, accepted, accepted ? (size_t)B : 0, s))
        return GDR_ERR_LAUNCH;
    std::unordered_map<int32_t, int> owner;
    for (int b = 0; b < B; ++b) {
        const int Lb = L[b];
        if (Lb < 0 || Lb > S) return GDR_ERR_SHAPE;
        if (Lb == 0) continue;
        int Ab = accepted ? A[b] : (per_token ? 1 : Lb);
        std::vector<int32_t> touched;
        if (per_token) {
            if (Ab < 1 || Ab > S) return GDR_ERR_SHAPE;
            touched.push_back(I[(size_t)b * S + Ab - 1]);
            for (int t = 0; t < Lb; ++t) touched.push_back(I[(size_t)b * S + t]);
        } else {
            if (Ab < 0) return GDR_ERR_SHAPE;
            touched.push_back(I[(size_t)b * S]);
            for (int t = 0; t < (Ab < Lb ? Ab : Lb); ++t) touched.push_back(I[(size_t)b * S + t]);
        }
        for (int32_t x : touched) {
            if (x < 0 || x >= slots) return GDR_ERR_SHAPE;
            auto it = owner.find(x);
            if (it != owner.end() && it->second != b) return GDR_ERR_SHAPE;
            owner[x] = b;
        }
    }
    return GDR_OK;
}

int check_epilogue(const gdr_epilogue *e) {
    if (!e) return GDR_OK;
    if (!e->z || !e->norm_w) return GDR_ERR_NULL;
    if (!(e->eps >= 0.f)) return GDR_ERR_SHAPE;
    if (!aligned16(e->z) || !aligned16(e->norm_w)) return GDR_ERR_ALIGN;
    return GDR_OK;
}

}  // namespace
}  // namespace gdr

using namespace gdr;

extern "C" size_t gdr_chunk_fwd_workspace(int B, int Nk, int Nv, int S, int Dk, int Dv, gdr_dtype dtype) {
    if (check_common(B, Nk, Nv, S, Dk, Dv, dtype) != GDR_OK) return 0;
    if ((long long)B * S == 0 || !chunk_tc_supported(Dk, Dv, dtype, S)) return 0;
    return two_kernel_schedule(B, Nv) ? chunk_wy_workspace(B, Nv, S) : 0;
}

extern "C" int gdr_chunk_fwd(const void *q, const void *k, const void *v, const void *beta, const float *g,
                             const void *initial_state, const int32_t *actual_seq_lengths, float scale, int B,
                             int Nk, int Nv, int S, int Dk, int Dv, gdr_dtype dtype, const gdr_prologue *prologue,
                             const gdr_epilogue *epilogue, void *out, void *final_state, void *workspace,
                             size_t ws_bytes, gdr_stream_t stream) {
    int st = check_common(B, Nk, Nv, S, Dk, Dv, dtype);
    if (st) return st;
    if ((st = check_prologue(prologue, g))) return st;
    if ((st = check_epilogue(epilogue))) return st;
    if ((long long)B * S > 0 && (!q || !k || !v || !beta || !out)) return GDR_ERR_NULL;
    const void *ptrs[] = {q, k, v, beta, g, initial_state, actual_seq_lengths, out, final_state, workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGN;
    // a workspace of at least the queried size selects the two-kernel schedule where the query asks for one; no
    // workspace runs the one-kernel schedule, which needs none
    const size_t need = gdr_chunk_fwd_workspace(B, Nk, Nv, S, Dk, Dv, dtype);
    if (workspace && ws_bytes < need) return GDR_ERR_WORKSPACE;
    if (B == 0 || (S == 0 && !final_state)) return GDR_OK;
    unsigned int *err = nullptr;
    if ((st = device_setup(&err))) return st;

    ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g;
    a.initial_state = initial_state;
    a.lengths = actual_seq_lengths;
    a.scale = scale;
    a.B = B; a.Nk = Nk; a.Nv = Nv; a.S = S;
    a.out = out; a.final_state = final_state;
    a.l2norm = prologue ? prologue->l2norm_qk : 0;
    a.eps = prologue ? prologue->eps : 0.f;
    a.beta_logits = prologue ? prologue->beta_logits : 0;
    a.A_log = prologue ? prologue->A_log : nullptr;
    a.dt_bias = prologue ? prologue->dt_bias : nullptr;
    a.err = err;
    a.workspace = workspace;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (checks_enabled() && (st = check_lengths_host(actual_seq_lengths, B, S, cs))) return st;
    cudaError_t e;
    if (chunk_tc_supported(Dk, Dv, dtype, S)) {
        if (epilogue) {  // fused into the tensor-core kernel's out epilogue
            a.epi_z = epilogue->z;
            a.epi_w = epilogue->norm_w;
            a.epi_eps = epilogue->eps;
        }
        e = (need > 0 && workspace) ? launch_chunk_wy(a, dtype, cs) : launch_chunk_tc(a, dtype, cs);
    } else {
        e = launch_chunk_simt(a, Dk, Dv, dtype, cs);
        if (e == cudaSuccess && epilogue && S > 0)
            e = launch_gated_rmsnorm(out, epilogue->z, epilogue->norm_w, epilogue->eps, actual_seq_lengths, B, Nv,
                                     S, Dv, dtype, cs);
    }
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}

namespace {
int recurrent_step(const void *q, const void *k, const void *v, const void *beta, const float *g, const float *gk,
                   void *state_pool, int slots, const int32_t *ssm_state_indices, const int32_t *actual_seq_lengths,
                   const int32_t *num_accepted_tokens, float scale, int B, int Nk, int Nv, int S, int Dk, int Dv,
                   gdr_dtype dtype, gdr_dtype state_dtype, const gdr_prologue *prologue, const gdr_epilogue *epilogue,
                   void *out, gdr_stream_t stream, int per_token) {
    int st = check_common(B, Nk, Nv, S, Dk, Dv, dtype);
    if (st) return st;
    if (state_dtype != GDR_F32 && state_dtype != GDR_BF16 && state_dtype != GDR_F16) return GDR_ERR_DTYPE;
    // fp16 inputs take an fp16 or fp32 state; an fp16 state takes fp16 inputs
    if ((dtype == GDR_F16 && state_dtype == GDR_BF16) || (state_dtype == GDR_F16 && dtype != GDR_F16))
        return GDR_ERR_DTYPE;
    if (S < 1 || S > kDecodeMaxTokens || slots < 1) return GDR_ERR_SHAPE;
    // the kernels address the pool by (slot, head) tile in 32-bit arithmetic
    if ((long long)slots * Nv >= (1LL << 31)) return GDR_ERR_SHAPE;
    if ((st = check_prologue(prologue, g))) return st;
    if ((st = check_epilogue(epilogue))) return st;
    if (B > 0 && (!q || !k || !v || !beta || !out || !state_pool || !ssm_state_indices || !actual_seq_lengths))
        return GDR_ERR_NULL;
    const void *ptrs[] = {q, k, v, beta, g, gk, state_pool, ssm_state_indices, actual_seq_lengths,
                          num_accepted_tokens, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGN;
    if (B == 0) return GDR_OK;
    unsigned int *err = nullptr;
    if ((st = device_setup(&err))) return st;

    DecodeArgs a{};
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.gk = gk;
    a.pool = state_pool; a.slots = slots;
    a.idx = ssm_state_indices; a.lengths = actual_seq_lengths; a.accepted = num_accepted_tokens;
    a.scale = scale;
    a.B = B; a.Nk = Nk; a.Nv = Nv; a.S = S;
    a.out = out;
    a.l2norm = prologue ? prologue->l2norm_qk : 0;
    a.eps = prologue ? prologue->eps : 0.f;
    a.beta_logits = prologue ? prologue->beta_logits : 0;
    a.A_log = prologue ? prologue->A_log : nullptr;
    a.dt_bias = prologue ? prologue->dt_bias : nullptr;
    a.err = err;
    a.per_token = per_token;
    a.wait_ns = chunk_wait_ns();
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (checks_enabled() &&
        (st = check_decode_host(ssm_state_indices, actual_seq_lengths, num_accepted_tokens, B, S, slots, per_token,
                                cs)))
        return st;
    cudaError_t e = launch_decode(a, Dk, Dv, dtype, state_dtype, cs);
    if (e == cudaSuccess && epilogue)
        e = launch_gated_rmsnorm(out, epilogue->z, epilogue->norm_w, epilogue->eps, actual_seq_lengths, B, Nv, S, Dv,
                                 dtype, cs);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}
}  // namespace

extern "C" int gdr_recurrent_step(const void *q, const void *k, const void *v, const void *beta, const float *g,
                                  const float *gk, void *state_pool, int slots, const int32_t *ssm_state_indices,
                                  const int32_t *actual_seq_lengths, const int32_t *num_accepted_tokens,
                                  float scale, int B, int Nk, int Nv, int S, int Dk, int Dv, gdr_dtype dtype,
                                  gdr_dtype state_dtype, const gdr_prologue *prologue,
                                  const gdr_epilogue *epilogue, void *out, gdr_stream_t stream) {
    return recurrent_step(q, k, v, beta, g, gk, state_pool, slots, ssm_state_indices, actual_seq_lengths,
                          num_accepted_tokens, scale, B, Nk, Nv, S, Dk, Dv, dtype, state_dtype, prologue, epilogue,
                          out, stream, 0);
}

extern "C" int gdr_recurrent_step_spec(const void *q, const void *k, const void *v, const void *beta,
                                       const float *g, const float *gk, void *state_pool, int slots,
                                       const int32_t *ssm_state_indices, const int32_t *actual_seq_lengths,
                                       const int32_t *num_accepted_tokens, float scale, int B, int Nk, int Nv, int S,
                                       int Dk, int Dv, gdr_dtype dtype, gdr_dtype state_dtype,
                                       const gdr_prologue *prologue, const gdr_epilogue *epilogue, void *out,
                                       gdr_stream_t stream) {
    return recurrent_step(q, k, v, beta, g, gk, state_pool, slots, ssm_state_indices, actual_seq_lengths,
                          num_accepted_tokens, scale, B, Nk, Nv, S, Dk, Dv, dtype, state_dtype, prologue, epilogue,
                          out, stream, 1);
}

extern "C" int gdr_conv1d(const void *x, const void *weight, const void *bias, const void *conv_state_in,
                          const int32_t *actual_seq_lengths, int B, int S, int Nk, int Nv, int Dk, int Dv, int K,
                          gdr_dtype dtype, void *q, void *k, void *v, void *conv_state_out, gdr_stream_t stream) {
    int st = check_common(B, Nk, Nv, S, Dk, Dv, dtype);
    if (st) return st;
    if (K < 1 || K > 8) return GDR_ERR_SHAPE;
    // grid: (channel groups, 64-step time tiles, B)
    if (B > 65535 || (long long)S > 65535LL * 64) return GDR_ERR_SHAPE;
    if ((long long)B * S > 0 && (!x || !weight || !q || !k || !v)) return GDR_ERR_NULL;
    if (B > 0 && conv_state_out && !weight) return GDR_ERR_NULL;
    const void *ptrs[] = {x, weight, bias, conv_state_in, actual_seq_lengths, q, k, v, conv_state_out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGN;
    if (B == 0 || (S == 0 && !conv_state_out)) return GDR_OK;
    unsigned int *err = nullptr;
    if ((st = device_setup(&err))) return st;
    cudaError_t e = launch_conv1d(x, weight, bias, conv_state_in, actual_seq_lengths, B, S, Nk, Nv, Dk, Dv, K, dtype,
                                  q, k, v, conv_state_out, err, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}

extern "C" int gdr_prologue_apply(const void *q, const void *k, const void *b, const float *a, const float *A_log,
                                  const float *dt_bias, float eps, int B, int Nk, int Nv, int S, int Dk,
                                  gdr_dtype dtype, void *q_hat, void *k_hat, void *beta, float *g,
                                  gdr_stream_t stream) {
    if (dtype != GDR_F32 && dtype != GDR_BF16 && dtype != GDR_F16) return GDR_ERR_DTYPE;
    if (B < 0 || S < 0 || Nk < 1 || Nv < 1 || Dk < 1) return GDR_ERR_SHAPE;
    if (!(eps >= 0.f)) return GDR_ERR_SHAPE;
    if ((q && !q_hat) || (k && !k_hat) || (b && !beta) || (a && (!g || !A_log || !dt_bias))) return GDR_ERR_NULL;
    const void *ptrs[] = {q, k, b, a, A_log, dt_bias, q_hat, k_hat, beta, g};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGN;
    if ((long long)B * S == 0 || (!q && !k && !b && !a)) return GDR_OK;
    unsigned int *err = nullptr;
    int st = device_setup(&err);
    if (st) return st;
    cudaError_t e = launch_prologue(q, k, b, a, A_log, dt_bias, eps, B, Nk, Nv, S, Dk, dtype, q_hat, k_hat, beta, g,
                                    reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}

extern "C" int gdr_get_error(gdr_stream_t stream, int *device_error) {
    if (!device_error) return GDR_ERR_NULL;
    *device_error = 0;
    unsigned int *err = nullptr;
    int st = device_setup(&err);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned int *slot = nullptr;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        std::lock_guard<std::mutex> lk(g_mu);
        slot = g_snap_ptr[dev] + (g_snap_next++ % kErrSlots);
    }
    unsigned int host = 0;
    take_error_kernel<<<1, 1, 0, s>>>(err, slot);
    if (cudaGetLastError() != cudaSuccess) return GDR_ERR_LAUNCH;
    if (cudaMemcpyAsync(&host, slot, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return GDR_ERR_LAUNCH;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDR_ERR_LAUNCH;
    *device_error = (int)host;
    return GDR_OK;
}

extern "C" const char *gdr_status_string(int status) {
    switch (status) {
        case GDR_OK: return "ok";
        case GDR_ERR_SHAPE: return "invalid shape or size argument";
        case GDR_ERR_DTYPE: return "unsupported dtype";
        case GDR_ERR_NULL: return "a required pointer is NULL";
        case GDR_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case GDR_ERR_UNSUPPORTED: return "head size not built (Dk and Dv must be 16, 32, 64 or 128)";
        case GDR_ERR_DEVICE: return "no usable sm_100 CUDA device";
        case GDR_ERR_LAUNCH: return "a CUDA call or kernel launch failed";
        case GDR_ERR_WORKSPACE: return "workspace smaller than gdr_chunk_fwd_workspace() returns";
        default: return "unknown status";
    }
}

extern "C" int gdr_version(void) { return 200; }

extern "C" int gdr_debug_set_wait_limit(unsigned long long ns) {
    chunk_tc_set_wait_ns(ns);
    return GDR_OK;
}

extern "C" int gdr_debug_timeout_site(unsigned int *site) {
    if (!site) return GDR_ERR_NULL;
    *site = 0;
    unsigned int *err = nullptr;
    int st = device_setup(&err);
    if (st) return st;
    unsigned int one = 0, two = 0;
    if (chunk_tc_take_timeout_site(&one) != cudaSuccess || chunk_wy_take_timeout_site(&two) != cudaSuccess)
        return GDR_ERR_LAUNCH;
    *site = one ? one : two;
    return GDR_OK;
}

extern "C" int gdr_debug_set_chunk_schedule(int schedule) {
    if (schedule < 0 || schedule > 2) return GDR_ERR_SHAPE;
    g_chunk_schedule = schedule;
    return GDR_OK;
}
