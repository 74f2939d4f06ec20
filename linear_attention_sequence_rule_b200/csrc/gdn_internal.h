// gdn_internal.h -- declarations shared by the host-side dispatcher and the kernel files of
// libgdn.  Nothing here is part of the public C-ABI (that is include/gdn.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

// Records a one-line reason for the calling host thread (read back by gdn_last_error()).
void set_error(const char *fmt, ...);

// Launchers (defined in the kernel .cu files).  They assume the arguments were validated by the
// C-ABI layer and return the cudaError_t of the launch.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, void *out, int N, int H, int dk, int dv,
                          int dtype, cudaStream_t stream);

struct ChunkArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    void *out;
    float *S_final;
    const int32_t *cu_seqlens;  // NULL: dense [B,T,...]
    int B, T, H, dk, dv, dtype;
    void *workspace;
    size_t workspace_bytes;
};

// Chunk forward on CUDA cores, fp32 arithmetic throughout (any supported dtype).
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream);

}  // namespace gdn
