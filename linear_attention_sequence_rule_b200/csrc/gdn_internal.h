// gdn_internal.h -- declarations shared by the host-side dispatcher and the kernel files of
// libgdn.  Nothing here is part of the public C-ABI (that is include/gdn.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

// Records a one-line reason for the calling host thread (read back by gdn_last_error()).
void set_error(const char *fmt, ...);

// Every argument check of the plain chunk forward except the workspace's (sizes, dtype, required
// and aligned pointers, S0 / S_final overlap), on the host only: GDN_OK, or the error code with
// the reason recorded under the name fn.
int chunk_fwd_check(const char *fn, const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, const float *S0, const void *out, const float *S_final, int B, int T,
                    int H, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype);

// Launchers (defined in the kernel .cu files).  They assume the arguments were validated by the
// C-ABI layer and return the cudaError_t of the launch.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, void *out, int N, int H, int dk, int dv,
                          int dtype, cudaStream_t stream, int G = 1, int prologue = 0, float a_scale = 0.f,
                          float b_scale = 0.f);

struct ChunkArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    void *out;
    float *S_final;
    const int32_t *cu_seqlens;  // NULL: dense [B,T,...]
    int B, T, H, dk, dv, dtype;
    void *workspace;
    size_t workspace_bytes;
    // fused prologue (bf16 only): q, k unnormalised, log_alpha / beta hold the raw projections a, b
    int prologue = 0;
    float a_scale = 0.f, b_scale = 0.f;
    // grouped value heads: H value heads, H / G q/k heads; value head h reads q/k head h / G
    int G = 1;
};

// Chunk forward on CUDA cores, fp32 arithmetic throughout (fp32 inputs).
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream);

// Chunk forward on the tcgen05 tensor cores (bf16 inputs).  Dense inputs with few (sequence,
// head) chains for the SM count run as a segment scan, which needs a workspace of
// chunk_tc_workspace_bytes(...) bytes (0 when not).
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream);
size_t chunk_tc_workspace_bytes(int B, int T, int H, int dk, int dv, int varlen, int dtype);

// Chunk forward for key head size 256 and chunk 128 (gdn_chunk_general.cu): fp32 on CUDA cores in
// two launches (per-chunk factors, then the state chain) through a workspace of
// chunk_general_workspace_bytes(...) bytes.
bool chunk_general_needed(int dk, int dv, int chunk);
size_t chunk_general_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen);
cudaError_t launch_chunk_general(const ChunkArgs &a, int chunk, cudaStream_t stream);

// Device error word of the tensor-core kernels (bounded waits that ran out); read and cleared
// after synchronising the device.  Returns -1 when the read itself failed.
int read_and_clear_tc_error();

// Self-test of the bounded waits: a kernel whose wait on an mbarrier nothing arrives on runs out
// after limit_ms and records it in that error word (see gdn_selftest_wait_timeout).
cudaError_t launch_wait_probe(int limit_ms, cudaStream_t stream);

// Gradients of the chunk forward (fp32-level accuracy, dk = 64, dv = 64 VS); see gdn_chunk_bwd.cu.
struct BwdArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    const void *dout;
    const float *dS_final;
    float *dq, *dk, *dv, *dlog_alpha, *dbeta, *dS0;
    const int32_t *cu_seqlens;
    int B, T, H, dtype;  // H value heads
    void *workspace;
    int G = 1;   // grouped value heads: H / G q/k heads, value head h reads q/k head h / G
    int VS = 1;  // value splits: dv = 64 VS, each value head run as VS heads of 64 columns
    int KB = 1;  // key blocks: dk = 64 KB
};
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int varlen, int G = 1, int VS = 1, int KB = 1);
cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t stream);

// Complex-phase memory with one decay per value channel (gdn_phase_rowdecay.cu): K, Q, M0,
// M_final as (re, im) fp32 pairs; V and out bf16 (bf16 != 0) or fp32.
// The complex-phase memory at dk = 32 complex, dv = 64 with its prologue in the chunk kernel: K, Q
// fp32 (re, im) pairs [tokens, H, 32, 2], V bf16, raw log_lam and beta; S0 / S_final the real
// state [B, H, 64, 64] ([Re | Im] rows).  phase_fused_ok: the sizes run as one launch (no
// segment scan), which the fused form requires.
bool phase_fused_ok(int B, int T, int H, int varlen);
cudaError_t launch_phase_chunk(const float *K, const float *Q, const void *V, const float *log_lam,
                               const float *beta, const float *S0, void *out, float *S_final, const int32_t *cu,
                               int B, int T, int H, cudaStream_t stream);

cudaError_t launch_phase_rowdecay(const float *K, const float *Q, const void *V, const float *log_r,
                                  const float *beta, const float *M0, void *out, float *M_final,
                                  const int32_t *cu_seqlens, int nseq, int T, int H, int dk, int dv, int bf16,
                                  cudaStream_t stream);
// The row-decay kernel's device error record (bounded MMA waits that ran out), read and cleared.
int read_and_clear_rowdecay_error();

}  // namespace gdn
