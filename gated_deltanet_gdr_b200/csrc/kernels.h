// kernels.h -- argument blocks and launchers of the device kernels (internal to libgdr.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/gdr.h"

namespace gdr {

constexpr int kChunk = 64;            // tokens per chunk of the prefill kernels
constexpr int kDecodeMaxTokens = 8;   // decode tokens per call (the operator is decode-only)

struct DecodeArgs {
    const void *q, *k, *v, *beta;
    const float *g, *gk;
    void *pool;
    int slots;
    const int32_t *idx, *lengths, *accepted;
    float scale;
    int B, Nk, Nv, S;
    void *out;
    int l2norm;
    float eps;
    int beta_logits;
    const float *A_log, *dt_bias;
    unsigned int *err;
    int per_token;  // num_accepted_tokens read per token (speculative decoding): see gdr_recurrent_step_spec
    uint64_t wait_ns;  // limit of each bounded wait of the D = 128 kernel (its stage pipeline)
};

struct ChunkArgs {
    const void *q, *k, *v, *beta;
    const float *g;
    const void *initial_state;
    const int32_t *lengths;
    float scale;
    int B, Nk, Nv, S;
    void *out, *final_state;
    int l2norm;
    float eps;
    int beta_logits;
    const float *A_log, *dt_bias;
    unsigned int *err;
    // fused gated RMSNorm epilogue (tensor-core path only): z (B, Nv, S, Dv) in the input dtype, norm_w (Dv)
    const void *epi_z;
    const float *epi_w;
    float epi_eps;
    // caller-owned scratch of the two-kernel tensor-core schedule (chunk_wy_workspace bytes, 16-byte aligned)
    void *workspace;
};

// cuTensorMapEncodeTiled, obtained once through the runtime's driver entry point (NULL if unavailable).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Launch facts of one kernel, kept per device: the dynamic shared-memory size its attribute allows, and the number
// of CTAs resident at once for a block shape.  Function attributes and occupancy belong to a device, so a process
// that drives several devices sets and asks them on each; the record is guarded for use from several host threads.
class LaunchCache {
  public:
    explicit LaunchCache(const void *func) : func_(func) {}
    // make `smem` bytes of dynamic shared memory launchable on the current device
    cudaError_t allow_smem(int smem);
    // CTAs of `threads` threads with `smem` bytes that the current device holds at once (at least 1)
    cudaError_t resident_grid(int threads, int smem, int *grid);

  private:
    static constexpr int kMaxDevices = 64;  // devices past this count are served without a record
    const void *func_;
    std::mutex mu_;
    int smem_[kMaxDevices] = {};
    int grid_key_[kMaxDevices] = {};  // (threads << 20) | smem of the recorded grid, 0 = none
    int grid_[kMaxDevices] = {};
};

cudaError_t launch_decode(const DecodeArgs &a, int Dk, int Dv, gdr_dtype dt, gdr_dtype st, cudaStream_t s);
// The tensor-core prefill (bf16 / fp16, Dk = Dv = 128) has two schedules:
//   chunk_tc.cu  one kernel, one CTA per (b, value head) chain that also solves each chunk's WY system; needs no
//                workspace;
//   chunk_wy.cu  a WY pass over every chunk on every SM into a caller workspace, then a chain kernel that only
//                carries the state; for few chains (B Nv at most a third of the SMs).
bool chunk_tc_supported(int Dk, int Dv, gdr_dtype dt, int S);
cudaError_t launch_chunk_tc(const ChunkArgs &a, gdr_dtype dt, cudaStream_t s);
// bytes of workspace the two-kernel schedule needs: per (b, value head, 64-token chunk) the 64 x 64 16-bit T' and
// six vectors of 64 floats
size_t chunk_wy_workspace(int B, int Nv, int S);
cudaError_t launch_chunk_wy(const ChunkArgs &a, gdr_dtype dt, cudaStream_t s);
// limit of the tensor-core prefill's bounded waits, in ns (0: the default of one second); the value in force
void chunk_tc_set_wait_ns(unsigned long long ns);
unsigned long long chunk_wait_ns();
// read and clear the record of the first bounded wait of each schedule that ran out (synchronous)
cudaError_t chunk_tc_take_timeout_site(unsigned int *site);
cudaError_t chunk_wy_take_timeout_site(unsigned int *site);
cudaError_t launch_chunk_simt(const ChunkArgs &a, int Dk, int Dv, gdr_dtype dt, cudaStream_t s);
// out rows t < L_b <- rmsnorm(out row) * norm_w * silu(z row), in place (the unfused epilogue)
cudaError_t launch_gated_rmsnorm(void *out, const void *z, const float *norm_w, float eps, const int32_t *lengths,
                                 int B, int Nv, int S, int Dv, gdr_dtype dt, cudaStream_t s);
// depthwise causal conv1d + SiLU over the fused q/k/v channels into q, k, v, and its state (gdr_conv1d)
cudaError_t launch_conv1d(const void *x, const void *weight, const void *bias, const void *state_in,
                          const int32_t *lengths, int B, int S, int Nk, int Nv, int Dk, int Dv, int K, gdr_dtype dt,
                          void *q, void *k, void *v, void *state_out, unsigned int *err, cudaStream_t s);
cudaError_t launch_prologue(const void *q, const void *k, const void *b, const float *a, const float *A_log,
                            const float *dt_bias, float eps, int B, int Nk, int Nv, int S, int Dk, gdr_dtype dt,
                            void *q_hat, void *k_hat, void *beta, float *g, cudaStream_t stream);

}  // namespace gdr
