// gdn_bwd_fused.cu -- gdn_chunk_bwd_fused: gradients of gdn_chunk_fwd_fused (the chunk forward from
// raw projections) with respect to the raw inputs.  The forward's prologue (q and k rows divided
// by sqrt(|x|^2 + 1e-6), log alpha = -a_scale softplus(a), beta = b_scale sigmoid(b); DeltaPhase
// README section 1 for beta = 2 sigmoid(W_beta x)) is formed again here in fp32, the fp32 backward
// of the recurrence runs on it, and the chain rule through the prologue is applied elementwise:
//   q = x / n:                       dx = (dq - q (q . dq)) / n
//   log alpha = -a_scale softplus(a): da = -a_scale sigmoid(a) dlog_alpha      (0 at a = +inf)
//   beta = b_scale sigmoid(b):        db = b_scale sigmoid(b) (1 - sigmoid(b)) dbeta
// The backward runs in fp32 whatever the input type (normalised rows in bf16 would cost the
// gradients their fp32-level accuracy), so v and dout are widened to fp32 as well.
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

constexpr int D = 64;              // key head size (the backward supports dk = 64, dv = 64, 128, 256)
constexpr float kEps = 1e-6f;      // the forward prologue's normalisation epsilon

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float sigmoidf_(float x)
{
    const float e = expf(-fabsf(x));
    return x >= 0.f ? 1.f / (1.f + e) : e / (1.f + e);
}

__device__ __forceinline__ float softplusf_(float x) { return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x)); }

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// One warp per (token, head): normalised q and k rows, v and dout (dv values) widened to fp32, the
// gates.
template <typename TIn>
__global__ void __launch_bounds__(256) fused_bwd_prologue(const TIn *__restrict__ q_raw, const TIn *__restrict__ k_raw,
                                                          const TIn *__restrict__ v, const TIn *__restrict__ dout,
                                                          const float *__restrict__ a_raw,
                                                          const float *__restrict__ b_raw, float a_scale,
                                                          float b_scale, long rows, int dv, float *__restrict__ qn,
                                                          float *__restrict__ kn, float *__restrict__ v32,
                                                          float *__restrict__ d32, float *__restrict__ la,
                                                          float *__restrict__ be)
{
    const long row = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const size_t o = (size_t)row * D;
    const float q0 = to_f(q_raw[o + lane]), q1 = to_f(q_raw[o + lane + 32]);
    const float k0 = to_f(k_raw[o + lane]), k1 = to_f(k_raw[o + lane + 32]);
    const float rq = 1.f / sqrtf(warp_sum(q0 * q0 + q1 * q1) + kEps);
    const float rk = 1.f / sqrtf(warp_sum(k0 * k0 + k1 * k1) + kEps);
    qn[o + lane] = q0 * rq;
    qn[o + lane + 32] = q1 * rq;
    kn[o + lane] = k0 * rk;
    kn[o + lane + 32] = k1 * rk;
    const size_t ov = (size_t)row * dv;
    for (int j = lane; j < dv; j += 32) {
        v32[ov + j] = to_f(v[ov + j]);
        d32[ov + j] = to_f(dout[ov + j]);
    }
    if (lane == 0) {
        const float a = a_raw[row];
        la[row] = a == INFINITY ? -INFINITY : -a_scale * softplusf_(a);
        be[row] = b_scale * sigmoidf_(b_raw[row]);
    }
}

// One warp per (token, head): dq, dk (in place, from the recurrence's gradients) to the raw rows,
// and the gate gradients to the raw projections.
template <typename TIn>
__global__ void __launch_bounds__(256) fused_bwd_epilogue(const TIn *__restrict__ q_raw, const TIn *__restrict__ k_raw,
                                                          const float *__restrict__ qn, const float *__restrict__ kn,
                                                          const float *__restrict__ a_raw,
                                                          const float *__restrict__ b_raw, float a_scale,
                                                          float b_scale, const float *__restrict__ dla,
                                                          const float *__restrict__ dbe, long rows,
                                                          float *__restrict__ dq, float *__restrict__ dk,
                                                          float *__restrict__ da, float *__restrict__ db)
{
    const long row = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const size_t o = (size_t)row * D;
    {
        const float x0 = to_f(q_raw[o + lane]), x1 = to_f(q_raw[o + lane + 32]);
        const float y0 = qn[o + lane], y1 = qn[o + lane + 32], g0 = dq[o + lane], g1 = dq[o + lane + 32];
        const float rn = 1.f / sqrtf(warp_sum(x0 * x0 + x1 * x1) + kEps), yg = warp_sum(y0 * g0 + y1 * g1);
        dq[o + lane] = (g0 - y0 * yg) * rn;
        dq[o + lane + 32] = (g1 - y1 * yg) * rn;
    }
    {
        const float x0 = to_f(k_raw[o + lane]), x1 = to_f(k_raw[o + lane + 32]);
        const float y0 = kn[o + lane], y1 = kn[o + lane + 32], g0 = dk[o + lane], g1 = dk[o + lane + 32];
        const float rn = 1.f / sqrtf(warp_sum(x0 * x0 + x1 * x1) + kEps), yg = warp_sum(y0 * g0 + y1 * g1);
        dk[o + lane] = (g0 - y0 * yg) * rn;
        dk[o + lane + 32] = (g1 - y1 * yg) * rn;
    }
    if (lane == 0) {
        const float a = a_raw[row];
        da[row] = a == INFINITY ? 0.f : -a_scale * sigmoidf_(a) * dla[row];
        const float sb = sigmoidf_(b_raw[row]);
        db[row] = b_scale * sb * (1.f - sb) * dbe[row];
    }
}

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct FusedBwdPlan {
    size_t qn, kn, v32, d32, la, be, dla, dbe, ws, ws_bytes, total;
};

bool fused_bwd_plan(FusedBwdPlan &p, int B, int T, int H, int dv, int varlen)
{
    const size_t ws = gdn_chunk_bwd_workspace_bytes(B, T, H, D, dv, 64, varlen);
    if (ws == (size_t)-1) return false;
    const size_t rows = (varlen ? (size_t)T : (size_t)B * T) * H;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += al256(bytes);
        return at;
    };
    p.qn = take(rows * D * 4);
    p.kn = take(rows * D * 4);
    p.v32 = take(rows * dv * 4);
    p.d32 = take(rows * dv * 4);
    p.la = take(rows * 4);
    p.be = take(rows * 4);
    p.dla = take(rows * 4);
    p.dbe = take(rows * 4);
    p.ws_bytes = ws;
    p.ws = take(ws);
    p.total = o;
    return true;
}

template <typename TIn>
int run_fused_bwd(const void *q_raw, const void *k_raw, const void *v, const float *a_raw, const float *b_raw,
                  const float *S0, const void *dout, const float *dS_final, float *dq_raw, float *dk_raw, float *dv,
                  float *da_raw, float *db_raw, float *dS0, int B, int T, int H, int dv_, const int32_t *cu_seqlens,
                  float a_scale, float b_scale, char *w, const FusedBwdPlan &p, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long rows = (cu_seqlens ? (long)T : (long)B * T) * H;
    const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
    float *qn = reinterpret_cast<float *>(w + p.qn), *kn = reinterpret_cast<float *>(w + p.kn);
    float *dla = reinterpret_cast<float *>(w + p.dla), *dbe = reinterpret_cast<float *>(w + p.dbe);
    if (blocks)
        fused_bwd_prologue<TIn><<<blocks, 256, 0, st>>>(
            static_cast<const TIn *>(q_raw), static_cast<const TIn *>(k_raw), static_cast<const TIn *>(v),
            static_cast<const TIn *>(dout), a_raw, b_raw, a_scale, b_scale, rows, dv_, qn, kn,
            reinterpret_cast<float *>(w + p.v32), reinterpret_cast<float *>(w + p.d32),
            reinterpret_cast<float *>(w + p.la), reinterpret_cast<float *>(w + p.be));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("gdn_chunk_bwd_fused: launch: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    const int rc = gdn_chunk_bwd(qn, kn, w + p.v32, reinterpret_cast<const float *>(w + p.la),
                                 reinterpret_cast<const float *>(w + p.be), S0, w + p.d32, dS_final, dq_raw, dk_raw,
                                 dv, dla, dbe, dS0, B, T, H, D, dv_, 64, cu_seqlens, GDN_DTYPE_F32, w + p.ws,
                                 p.ws_bytes, stream);
    if (rc != GDN_OK) return rc;
    if (blocks)
        fused_bwd_epilogue<TIn><<<blocks, 256, 0, st>>>(static_cast<const TIn *>(q_raw),
                                                        static_cast<const TIn *>(k_raw), qn, kn, a_raw, b_raw,
                                                        a_scale, b_scale, dla, dbe, rows, dq_raw, dk_raw, da_raw,
                                                        db_raw);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("gdn_chunk_bwd_fused: launch: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" {

size_t gdn_chunk_bwd_fused_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen)
{
    if (dk != D || (dv != 64 && dv != 128 && dv != 256) || chunk != 64) return (size_t)-1;
    FusedBwdPlan p;
    if (!fused_bwd_plan(p, B, T, H, dv, varlen)) return (size_t)-1;
    return p.total;
}

int gdn_chunk_bwd_fused(const void *q_raw, const void *k_raw, const void *v, const float *a_raw, const float *b_raw,
                        const float *S0, const void *dout, const float *dS_final, float *dq_raw, float *dk_raw,
                        float *dv, float *da_raw, float *db_raw, float *dS0, int B, int T, int H, int dk, int dv_,
                        int chunk, const int32_t *cu_seqlens, int dtype, float a_scale, float b_scale,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    const int varlen = cu_seqlens != nullptr;
    if (dtype != GDN_DTYPE_BF16 && dtype != GDN_DTYPE_F32) {
        set_error("gdn_chunk_bwd_fused: unknown dtype %d", dtype);
        return GDN_ERR_UNSUPPORTED;
    }
    if (dk != D || (dv_ != 64 && dv_ != 128 && dv_ != 256) || chunk != 64) {
        set_error("gdn_chunk_bwd_fused: dk=%d dv=%d chunk=%d, supported: dk 64, dv 64, 128 or 256, chunk 64", dk,
                  dv_, chunk);
        return GDN_ERR_UNSUPPORTED;
    }
    if (!(a_scale >= 0.f) || !(a_scale < INFINITY) || !(b_scale >= 0.f && b_scale <= 2.f)) {
        set_error("gdn_chunk_bwd_fused: a_scale %g (finite, >= 0) or b_scale %g (in [0, 2]) out of range",
                  (double)a_scale, (double)b_scale);
        return GDN_ERR_INVALID_ARGUMENT;
    }
    FusedBwdPlan p;
    if (!fused_bwd_plan(p, B, T, H, dv_, varlen))  // the backward's own checks give the reason
        return gdn_chunk_bwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, B, T, H, dk, dv_, chunk, cu_seqlens,
                             GDN_DTYPE_F32, nullptr, 0, stream);
    if (!q_raw || !k_raw || !v || !a_raw || !b_raw || !dout || !dq_raw || !dk_raw || !dv || !da_raw || !db_raw) {
        set_error("gdn_chunk_bwd_fused: inputs, dout and every gradient output except dS0 are required");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    const void *ptrs[] = {q_raw, k_raw, v, a_raw, b_raw, S0, dout, dS_final, dq_raw, dk_raw, dv, da_raw, db_raw,
                          dS0, cu_seqlens};
    for (const void *ptr : ptrs)
        if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u)) {
            set_error("gdn_chunk_bwd_fused: pointer %p is not 16-byte aligned", ptr);
            return GDN_ERR_INVALID_ARGUMENT;
        }
    if (!workspace || workspace_bytes < p.total) {
        set_error("gdn_chunk_bwd_fused: workspace of %zu bytes needed, %zu given", p.total,
                  workspace ? workspace_bytes : (size_t)0);
        return GDN_ERR_WORKSPACE;
    }
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) {
        set_error("gdn_chunk_bwd_fused: workspace must be 256-byte aligned");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    char *w = static_cast<char *>(workspace);
    return dtype == GDN_DTYPE_BF16
               ? run_fused_bwd<__nv_bfloat16>(q_raw, k_raw, v, a_raw, b_raw, S0, dout, dS_final, dq_raw, dk_raw,
                                              dv, da_raw, db_raw, dS0, B, T, H, dv_, cu_seqlens, a_scale, b_scale, w,
                                              p, stream)
               : run_fused_bwd<float>(q_raw, k_raw, v, a_raw, b_raw, S0, dout, dS_final, dq_raw, dk_raw, dv,
                                      da_raw, db_raw, dS0, B, T, H, dv_, cu_seqlens, a_scale, b_scale, w, p, stream);
}

}  // extern "C"
