// noalloc.cu -- gdr_chunk_fwd_noalloc: the chunked prefill with its scratch in a fixed array compiled into the
// library, for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs where allocation is not allowed or not
// available -- inside a framework hook or plug-in that only receives the tensors of one operation, a serving loop
// whose device memory is all reserved up front by its own pool, a runtime with no allocator of its own -- cannot call
// cudaMalloc (or a torch allocation) on the path that calls the prefill.  For them the scratch the tensor-core path
// needs lives in g_noalloc_scratch below: one array of kNoAllocScratchBytes per GPU that loads the library, held
// until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/gdr.h"
#include "kernels.h"

namespace gdr {
namespace {

// 16 MiB: per (b, value head, 64-token chunk) the prefill needs 9728 bytes, so B * Nv * ceil(S / 64) <= 1724
// (for example one sequence of 3392 tokens with 32 value heads).
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];  // device address of the array on each device (NULL until that device's first call)

// The array's device address on the current device.  In host code the name g_noalloc_scratch only stands for the
// symbol, so it is looked up once per device, with that device current, and the result is cached.
int noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return GDR_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return GDR_ERR_LAUNCH;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return GDR_OK;
}

}  // namespace
}  // namespace gdr

// The same call as gdr_chunk_fwd, with the library's own fixed scratch in place of a caller workspace.  Nothing here
// allocates: the size check, the one-time address lookup and then gdr_chunk_fwd's own checks and launches.  The
// workspace's contents on entry never matter to the prefill (every entry it reads is written earlier in the same
// call), so nothing needs clearing between calls.
extern "C" int gdr_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *beta, const float *g,
                                     const void *initial_state, const int32_t *actual_seq_lengths, float scale, int B,
                                     int Nk, int Nv, int S, int Dk, int Dv, gdr_dtype dtype,
                                     const gdr_prologue *prologue, const gdr_epilogue *epilogue, void *out,
                                     void *final_state, gdr_stream_t stream) {
    const size_t need = gdr_chunk_fwd_workspace(B, Nk, Nv, S, Dk, Dv, dtype);
    if (need > gdr::kNoAllocScratchBytes) return GDR_ERR_WORKSPACE;
    void *ws = nullptr;
    if (need > 0) {
        const int st = gdr::noalloc_scratch(&ws);
        if (st != GDR_OK) return st;
    }
    return gdr_chunk_fwd(q, k, v, beta, g, initial_state, actual_seq_lengths, scale, B, Nk, Nv, S, Dk, Dv, dtype,
                         prologue, epilogue, out, final_state, ws, need, stream);
}
