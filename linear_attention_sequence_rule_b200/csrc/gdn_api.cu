// gdn_api.cu -- the C-ABI of libgdn (declared in include/gdn.h): argument validation on the
// host, choice of kernel, and launch on the caller's stream.  No call allocates device memory.
// The one fixed device footprint of the library is the 32 MiB scratch array of
// gdn_chunk_fwd_noalloc (gdn_noalloc.cu), held on each device where its module is loaded (with
// CUDA's default lazy loading: from that entry point's first call on the device).
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {

static thread_local char g_last_error[512];

void set_error(const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return code;
}

static int cuda_fail(cudaError_t e, const char *where)
{
    return fail(GDN_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

static bool head_dim_ok(int d) { return d == 64 || d == 128; }

// Shapes of the chunk forward: the fused tensor-core kernel (bf16; dk, dv in {64, 128}, dv 256 as
// two column blocks; chunk 64) and the fp32 CUDA-core kernel (fp32; dk, dv in {64, 128}; chunk
// 64) cover the common sizes; key head size 256 and chunk 128 (and fp32 at dv 256) take the
// general two-launch path of gdn_chunk_general.cu.
static bool general_path(int dk, int dv, int chunk, int dtype)
{
    return chunk_general_needed(dk, dv, chunk) || (dv == 256 && dtype == GDN_DTYPE_F32);
}

// Shared shape/type checks of the chunk forward (and, with fwd = false, of the backward, which
// keeps chunk 64 and its own head sizes); returns GDN_OK or an error code.
static int check_chunk_shape(int B, int T, int H, int dk, int dv, int chunk, int varlen, int dtype,
                             bool fwd = true)
{
    if (dtype != GDN_DTYPE_BF16 && dtype != GDN_DTYPE_F32)
        return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_fwd: unknown dtype %d", dtype);
    if (fwd && (!(head_dim_ok(dk) || dk == 256) || !(head_dim_ok(dv) || dv == 256)))
        return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_fwd: dk=%d dv=%d, supported: dk and dv in {64, 128, 256}", dk, dv);
    if (fwd ? (chunk != 64 && chunk != 128) : chunk != 64)
        return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_fwd: chunk=%d, supported: %s", chunk, fwd ? "64 or 128" : "64");
    if (B < 1 || H < 1)
        return fail(GDN_ERR_INVALID_ARGUMENT, "gdn_chunk_fwd: B=%d H=%d must be >= 1", B, H);
    if (T < 0 || (!varlen && T < 1))
        return fail(GDN_ERR_INVALID_ARGUMENT, "gdn_chunk_fwd: T=%d (dense needs T >= 1)", T);
    const long long tokens = varlen ? (long long)T : (long long)B * T;
    if (tokens * H * (dk > dv ? dk : dv) >= (1LL << 40))
        return fail(GDN_ERR_INVALID_ARGUMENT, "gdn_chunk_fwd: problem too large");
    if ((long long)B * H > (1LL << 30))
        return fail(GDN_ERR_INVALID_ARGUMENT, "gdn_chunk_fwd: B*H too large");
    return GDN_OK;
}

int chunk_fwd_check(const char *fn, const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, const float *S0, const void *out, const float *S_final, int B, int T,
                    int H, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype)
{
    const int varlen = cu_seqlens != nullptr;
    int rc = check_chunk_shape(B, T, H, dk, dv, chunk, varlen, dtype);
    if (rc != GDN_OK) return rc;
    if (!q || !k || !v || !log_alpha || !beta || !out)
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: q, k, v, the two gate arrays and out are required", fn);
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, out, S_final, cu_seqlens};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(GDN_ERR_INVALID_ARGUMENT, "%s: pointer %p is not 16-byte aligned", fn, p);
    if (S_final && S_final != S0 && S0) {
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        const char *a0 = (const char *)S0, *b0 = (const char *)S_final;
        if (a0 < b0 + bytes && b0 < a0 + bytes)
            return fail(GDN_ERR_INVALID_ARGUMENT, "%s: S0 and S_final overlap partially", fn);
    }
    return GDN_OK;
}

static size_t chunk_workspace(int B, int T, int H, int dk, int dv, int chunk, int varlen, int dtype)
{
    if (general_path(dk, dv, chunk, dtype)) return chunk_general_workspace_bytes(B, T, H, dk, dv, chunk, varlen);
    if (dtype != GDN_DTYPE_BF16) return 0;
    return chunk_tc_workspace_bytes(B, T, H, dk, dv, varlen, dtype);
}

}  // namespace gdn

using namespace gdn;

extern "C" {

const char *gdn_version(void) { return "gdn-b200 0.1"; }

const char *gdn_last_error(void) { return g_last_error; }

const char *gdn_status_string(int status)
{
    switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARGUMENT: return "GDN_ERR_INVALID_ARGUMENT";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    default: return "GDN_ERR_UNKNOWN";
    }
}

size_t gdn_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen,
                                     int dtype)
{
    if (check_chunk_shape(B, T, H, dk, dv, chunk, varlen, dtype) != GDN_OK) return (size_t)-1;
    return chunk_workspace(B, T, H, dk, dv, chunk, varlen, dtype);
}

namespace gdn {

// Validation and launch shared by the plain and the fused-prologue chunk forward.
static int chunk_fwd_common(const char *fn, const void *q, const void *k, const void *v,
                            const float *log_alpha, const float *beta, const float *S0, void *out,
                            float *S_final, int B, int T, int H, int dk, int dv, int chunk,
                            const int32_t *cu_seqlens, int dtype, int prologue, float a_scale,
                            float b_scale, void *workspace, size_t workspace_bytes, void *stream,
                            int G = 1)
{
    const int varlen = cu_seqlens != nullptr;
    const int rc = chunk_fwd_check(fn, q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk,
                                   cu_seqlens, dtype);
    if (rc != GDN_OK) return rc;
    if (prologue && general_path(dk, dv, chunk, dtype))
        return fail(GDN_ERR_UNSUPPORTED, "%s: the fused prologue takes dk, dv in {64, 128} (dv 256) and chunk 64",
                    fn);
    const size_t need = chunk_workspace(B, T, H, dk, dv, chunk, varlen, dtype);
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(GDN_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                        workspace ? workspace_bytes : (size_t)0);
        if (reinterpret_cast<uintptr_t>(workspace) & 255u)
            return fail(GDN_ERR_INVALID_ARGUMENT, "%s: workspace must be 256-byte aligned", fn);
    }
    ChunkArgs a{q, k, v, log_alpha, beta, S0, out, S_final, cu_seqlens, B, T, H, dk, dv, dtype,
                workspace, workspace_bytes, prologue, a_scale, b_scale, G};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = general_path(dk, dv, chunk, dtype) ? launch_chunk_general(a, chunk, st)
                    : dtype == GDN_DTYPE_BF16                ? launch_chunk_tc(a, st)
                                                             : launch_chunk_simt(a, st);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDN_OK;
}

}  // namespace gdn

int gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, void *out, float *S_final, int B, int T,
                  int H, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype,
                  void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    return chunk_fwd_common("gdn_chunk_fwd", q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv,
                            chunk, cu_seqlens, dtype, 0, 0.f, 0.f, workspace, workspace_bytes, stream);
}

int gdn_chunk_fwd_fused(const void *q_raw, const void *k_raw, const void *v, const float *a_raw,
                        const float *b_raw, const float *S0, void *out, float *S_final, int B, int T,
                        int H, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype,
                        float a_scale, float b_scale, void *workspace, size_t workspace_bytes,
                        void *stream)
{
    g_last_error[0] = 0;
    if (dtype != GDN_DTYPE_BF16)
        return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_fwd_fused: dtype %d, supported: bf16", dtype);
    if (!(a_scale >= 0.f) || !(a_scale < INFINITY))
        return fail(GDN_ERR_INVALID_ARGUMENT, "gdn_chunk_fwd_fused: a_scale %g, must be finite and >= 0",
                    (double)a_scale);
    if (!(b_scale >= 0.f && b_scale <= 2.f))
        return fail(GDN_ERR_INVALID_ARGUMENT, "gdn_chunk_fwd_fused: b_scale %g, must lie in [0, 2]",
                    (double)b_scale);
    return chunk_fwd_common("gdn_chunk_fwd_fused", q_raw, k_raw, v, a_raw, b_raw, S0, out, S_final, B, T, H,
                            dk, dv, chunk, cu_seqlens, dtype, 1, a_scale, b_scale, workspace,
                            workspace_bytes, stream);
}

namespace gdn {

static int decode_common(const char *fn, const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, float *S_inout, void *out, int N, int H, int G, int dk, int dv,
                         int dtype, void *stream, int prologue = 0, float a_scale = 0.f, float b_scale = 0.f)
{
    if (dtype != GDN_DTYPE_BF16 && dtype != GDN_DTYPE_F32)
        return fail(GDN_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, dtype);
    if (!(head_dim_ok(dk) || dk == 256) || !(head_dim_ok(dv) || dv == 256))
        return fail(GDN_ERR_UNSUPPORTED, "%s: dk=%d dv=%d, supported: dk and dv in {64, 128, 256}", fn, dk, dv);
    if (N < 1 || H < 1 || (long long)N * H > (1LL << 30))
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: N=%d H=%d out of range", fn, N, H);
    if (!q || !k || !v || !log_alpha || !beta || !S_inout || !out)
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: every pointer is required", fn);
    const void *ptrs[] = {q, k, v, log_alpha, beta, S_inout, out};
    for (const void *p : ptrs)
        if (!aligned16(p))
            return fail(GDN_ERR_INVALID_ARGUMENT, "%s: pointer %p is not 16-byte aligned", fn, p);
    if (prologue && (!(a_scale >= 0.f) || !(a_scale < INFINITY) || !(b_scale >= 0.f && b_scale <= 2.f)))
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: a_scale %g (finite, >= 0) or b_scale %g (in [0, 2]) out of range",
                    fn, (double)a_scale, (double)b_scale);
    cudaError_t e = launch_decode(q, k, v, log_alpha, beta, S_inout, out, N, H, dk, dv, dtype,
                                  static_cast<cudaStream_t>(stream), G, prologue, a_scale, b_scale);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDN_OK;
}

// Head counts of the grouped-value-head entries: Hv value heads share Hk q/k heads.
static int check_groups(const char *fn, int Hk, int Hv)
{
    if (Hk < 1 || Hv < 1 || Hv % Hk != 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: Hk=%d Hv=%d, need Hk >= 1 and Hv a multiple of Hk", fn, Hk,
                    Hv);
    return GDN_OK;
}

}  // namespace gdn

int gdn_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, float *S_inout, void *out, int N, int H, int dk, int dv,
                    int dtype, void *stream)
{
    g_last_error[0] = 0;
    return decode_common("gdn_decode_step", q, k, v, log_alpha, beta, S_inout, out, N, H, 1, dk, dv, dtype,
                         stream);
}

int gdn_decode_step_fused(const void *q_raw, const void *k_raw, const void *v, const float *a_raw,
                          const float *b_raw, float *S_inout, void *out, int N, int H, int dk, int dv, int dtype,
                          float a_scale, float b_scale, void *stream)
{
    g_last_error[0] = 0;
    return decode_common("gdn_decode_step_fused", q_raw, k_raw, v, a_raw, b_raw, S_inout, out, N, H, 1, dk, dv,
                         dtype, stream, 1, a_scale, b_scale);
}

int gdn_decode_step_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                        const float *beta, float *S_inout, void *out, int N, int Hk, int Hv, int dk,
                        int dv, int dtype, void *stream)
{
    g_last_error[0] = 0;
    const int rc = check_groups("gdn_decode_step_gva", Hk, Hv);
    if (rc != GDN_OK) return rc;
    return decode_common("gdn_decode_step_gva", q, k, v, log_alpha, beta, S_inout, out, N, Hv, Hv / Hk, dk,
                         dv, dtype, stream);
}

int gdn_chunk_fwd_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                      const float *beta, const float *S0, void *out, float *S_final, int B, int T,
                      int Hk, int Hv, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    const int rc = check_groups("gdn_chunk_fwd_gva", Hk, Hv);
    if (rc != GDN_OK) return rc;
    return chunk_fwd_common("gdn_chunk_fwd_gva", q, k, v, log_alpha, beta, S0, out, S_final, B, T, Hv, dk, dv,
                            chunk, cu_seqlens, dtype, 0, 0.f, 0.f, workspace, workspace_bytes, stream,
                            Hv / Hk);
}

int gdn_phase_rowdecay_fwd(const float *K, const float *Q, const void *v, const float *log_r, const float *beta,
                           const float *M0, void *out, float *M_final, int B, int T, int H, int dk, int dv,
                           const int32_t *cu_seqlens, int dtype, void *stream)
{
    g_last_error[0] = 0;
    const char *fn = "gdn_phase_rowdecay_fwd";
    if (dtype != GDN_DTYPE_BF16 && dtype != GDN_DTYPE_F32) return fail(GDN_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, dtype);
    if (dk != 32 && dk != 64) return fail(GDN_ERR_UNSUPPORTED, "%s: dk=%d, supported: 32 or 64 (complex)", fn, dk);
    if (dv < 1 || dv > 4096) return fail(GDN_ERR_UNSUPPORTED, "%s: dv=%d, supported: 1 .. 4096", fn, dv);
    const int varlen = cu_seqlens != nullptr;
    if (B < 1 || H < 1 || T < 0 || (!varlen && T < 1))
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: B=%d T=%d H=%d (B, H >= 1; dense T >= 1)", fn, B, T, H);
    const long long tokens = varlen ? (long long)T : (long long)B * T;
    if (tokens * H * (dv > 2 * dk ? dv : 2 * dk) >= (1LL << 40) || (long long)B * H * dv >= (1LL << 31) ||
        B > 65535 || H > 65535)
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: problem too large (B and H at most 65535)", fn);
    if (!K || !Q || !v || !log_r || !beta || !out)
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: K, Q, v, log_r, beta and out are required", fn);
    const void *ptrs[] = {K, Q, v, log_r, beta, M0, out, M_final, cu_seqlens};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(GDN_ERR_INVALID_ARGUMENT, "%s: pointer %p is not 16-byte aligned", fn, p);
    if (M0 && M_final && M0 != M_final) {
        const size_t bytes = (size_t)B * H * dv * dk * 2 * sizeof(float);
        const char *a0 = (const char *)M0, *b0 = (const char *)M_final;
        if (a0 < b0 + bytes && b0 < a0 + bytes)
            return fail(GDN_ERR_INVALID_ARGUMENT, "%s: M0 and M_final overlap partially", fn);
    }
    cudaError_t e = launch_phase_rowdecay(K, Q, v, log_r, beta, M0, out, M_final, cu_seqlens, B, T, H, dk, dv,
                                          dtype == GDN_DTYPE_BF16, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDN_OK;
}

int gdn_selftest_wait_timeout(int limit_ms, void *stream)
{
    g_last_error[0] = 0;
    if (limit_ms < 1 || limit_ms > 2000)
        return fail(GDN_ERR_INVALID_ARGUMENT, "gdn_selftest_wait_timeout: limit_ms=%d, must lie in [1, 2000]",
                    limit_ms);
    cudaError_t e = launch_wait_probe(limit_ms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gdn_selftest_wait_timeout");
    return GDN_OK;
}

int gdn_device_status(void *stream)
{
    g_last_error[0] = 0;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gdn_device_status");
    const int v1 = read_and_clear_tc_error(), v2 = read_and_clear_rowdecay_error();
    if (v1 < 0 || v2 < 0) return fail(GDN_ERR_CUDA, "gdn_device_status: reading the device record failed");
    const int v = v1 | v2;
    if (v) return fail(GDN_ERR_TIMEOUT, "a device-side wait ran out (record 0x%x)", v);
    return GDN_OK;
}

}  // extern "C"

// Head sizes of the backward: dk = 64 KB with KB in {1, 2} (key blocks), dv = 64 VS with VS in
// {1, 2, 4} (value splits).
static bool bwd_heads_ok(int dk, int dv) { return (dk == 64 || dk == 128) && (dv == 64 || dv == 128 || dv == 256); }

size_t gdn_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen)
{
    if (!bwd_heads_ok(dk, dv) || chunk != 64 || B < 1 || H < 1 || T < 0 || (!varlen && T < 1)) return (size_t)-1;
    return chunk_bwd_workspace_bytes(B, T, H, varlen, 1, dv / 64, dk / 64);
}

size_t gdn_chunk_bwd_gva_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk, int varlen)
{
    if (Hk < 1 || Hv < 1 || Hv % Hk != 0) return (size_t)-1;
    if (!bwd_heads_ok(dk, dv) || chunk != 64 || B < 1 || T < 0 || (!varlen && T < 1)) return (size_t)-1;
    return chunk_bwd_workspace_bytes(B, T, Hv, varlen, Hv / Hk, dv / 64, dk / 64);
}

namespace gdn {

// Validation and launch shared by the plain (G = 1) and the grouped-value-head backward.
static int chunk_bwd_common(const char *fn, const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *S0, const void *dout, const float *dS_final, float *dq,
                            float *dk, float *dv, float *dlog_alpha, float *dbeta, float *dS0, int B, int T, int H,
                            int G, int dk_, int dv_, int chunk, const int32_t *cu_seqlens, int dtype,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    const int varlen = cu_seqlens != nullptr;
    if (!bwd_heads_ok(dk_, dv_))
        return fail(GDN_ERR_UNSUPPORTED, "%s: dk=%d dv=%d, supported: dk 64 or 128, dv 64, 128 or 256", fn, dk_,
                    dv_);
    int rc = check_chunk_shape(B, T, H, dk_, dv_, chunk, varlen, dtype, false);
    if (rc != GDN_OK) return rc;
    if (!q || !k || !v || !log_alpha || !beta || !dout || !dq || !dk || !dv || !dlog_alpha || !dbeta)
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: inputs, dout and every gradient output except dS0 are required",
                    fn);
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta, dS0,
                          cu_seqlens};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(GDN_ERR_INVALID_ARGUMENT, "%s: pointer %p is not 16-byte aligned", fn, p);
    const int VS = dv_ / 64, KB = dk_ / 64;
    const size_t need = chunk_bwd_workspace_bytes(B, T, H, varlen, G, VS, KB);
    if (!workspace || workspace_bytes < need)
        return fail(GDN_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                    workspace ? workspace_bytes : (size_t)0);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(GDN_ERR_INVALID_ARGUMENT, "%s: workspace must be 256-byte aligned", fn);
    BwdArgs a{q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta, dS0, cu_seqlens,
              B, T, H, dtype, workspace, G, VS, KB};
    cudaError_t e = launch_chunk_bwd(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDN_OK;
}

}  // namespace gdn

int gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                  const float *S0, const void *dout, const float *dS_final, float *dq, float *dk, float *dv,
                  float *dlog_alpha, float *dbeta, float *dS0, int B, int T, int H, int dk_, int dv_, int chunk,
                  const int32_t *cu_seqlens, int dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    return chunk_bwd_common("gdn_chunk_bwd", q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv, dlog_alpha,
                            dbeta, dS0, B, T, H, 1, dk_, dv_, chunk, cu_seqlens, dtype, workspace, workspace_bytes,
                            stream);
}

int gdn_chunk_bwd_gva(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                      const float *S0, const void *dout, const float *dS_final, float *dq, float *dk, float *dv,
                      float *dlog_alpha, float *dbeta, float *dS0, int B, int T, int Hk, int Hv, int dk_, int dv_,
                      int chunk, const int32_t *cu_seqlens, int dtype, void *workspace, size_t workspace_bytes,
                      void *stream)
{
    g_last_error[0] = 0;
    const int rc = check_groups("gdn_chunk_bwd_gva", Hk, Hv);
    if (rc != GDN_OK) return rc;
    return chunk_bwd_common("gdn_chunk_bwd_gva", q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv,
                            dlog_alpha, dbeta, dS0, B, T, Hv, Hv / Hk, dk_, dv_, chunk, cu_seqlens, dtype, workspace,
                            workspace_bytes, stream);
}
