// gdn_phase.cu -- gdn_phase_fwd: the complex-phase delta memory (DeltaPhase README, section 2
// "Complex Phase Matrix Delta Memory", gated-decay form; section 5 for keys e^{s dt}) on the
// chunk kernels of the real gated delta rule.
//
// Per (sequence, head) the state is M in C^{dv x dk}; per token
//     e_t = V_t - (1/dk) Re(M_{t-1} conj K_t),   M_t = lam_t M_{t-1} + beta_t e_t K_t^T,
//     o_t = (1/dk) Re(M_t conj Q_t).
// Written over the real vector space C^dk = R^{2dk} with S = [Re M | Im M]^T (2dk x dv), this is
//     S_t = lam_t S_{t-1} - (beta_t/dk) k~ k~^T S_{t-1} + beta_t k~ V_t^T,   o_t = (1/dk) S_t^T q~
// with k~ = (Re K, Im K), q~ = (Re Q, Im Q): the real gated delta rule
//     S_t = a_t (I - b_t k k^T) S_{t-1} + b_t k v^T,   o_t = S_t^T q
// at head size 2dk with a = lam, b = beta / lam, k = k~ / sqrt(dk), v = lam sqrt(dk) V, q = q~ / dk
// (lam > 0).  At dk = 32, dv = 64 with bf16 values the chunk kernel forms those inputs itself
// (kFlagPhase: K and Q converted in shared memory, b v = beta sqrt(dk) V folded into its U~
// product); otherwise one prologue kernel writes them and the chunk kernel runs unchanged.  The
// complex state is converted on the way in and out.
#include <cuda_bf16.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// 1 / sqrt(DK) and sqrt(DK) for the two key sizes
template <int DK> struct KeyScale;
template <> struct KeyScale<32> {
    static constexpr float inv_sqrt = 0.17677669529663688f, sqrt = 5.656854249492381f;
};
template <> struct KeyScale<64> {
    static constexpr float inv_sqrt = 0.125f, sqrt = 8.0f;
};

// The real recurrence's inputs of token-head th, written by DK / 4 threads, thread i taking key
// elements 4i .. 4i + 3 (two 16-byte loads each of K and Q) and value elements i DV' .. (i + 1) DV'
// - 1, DV' = 4 DV / DK:
//   k[th] = (Re K, Im K) / sqrt(DK),  q[th] = (Re Q, Im Q) / DK     (2 DK elements each)
//   v[th] = lam sqrt(DK) V[th],  b[th] = beta / lam
template <typename TV> struct Pack4;  // four elements as one store
template <> struct Pack4<float> {
    using type = float4;
    __device__ static float4 make(float a, float b, float c, float d) { return make_float4(a, b, c, d); }
};
template <> struct Pack4<__nv_bfloat16> {
    using type = uint2;
    __device__ static uint2 make(float a, float b, float c, float d)
    {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
        return make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
    }
};

template <int DK, int DV, typename TV, typename TO>
__global__ void __launch_bounds__(256) phase_prologue(const float4 *__restrict__ K, const float4 *__restrict__ Q,
                                                      const TV *__restrict__ V, const float *__restrict__ log_lam,
                                                      const float *__restrict__ beta, long token_heads,
                                                      TO *__restrict__ kr, TO *__restrict__ qr, TO *__restrict__ vr,
                                                      float *__restrict__ br)
{
    constexpr int TPT = DK / 4;       // threads per token-head
    constexpr int VPT = DV / TPT;     // value elements per thread
    using P = Pack4<TO>;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long th = idx / TPT;
    const int i = (int)(idx % TPT);
    if (th >= token_heads) return;
    const float ll = log_lam[th];
    // complex elements 4i .. 4i + 3 = float4 pieces 2i, 2i + 1 of the token-head's (re, im) row
    const float4 k0 = K[th * (DK / 2) + 2 * i], k1 = K[th * (DK / 2) + 2 * i + 1];
    const float4 q0 = Q[th * (DK / 2) + 2 * i], q1 = Q[th * (DK / 2) + 2 * i + 1];
    TV vin[VPT];
#pragma unroll
    for (int e = 0; e < VPT; ++e) vin[e] = V[th * DV + i * VPT + e];
    const float lam = expf(ll);
    constexpr float ks = KeyScale<DK>::inv_sqrt, qs = 1.0f / DK;
    using S = typename P::type;
    reinterpret_cast<S *>(kr + th * 2 * DK)[i] = P::make(k0.x * ks, k0.z * ks, k1.x * ks, k1.z * ks);
    reinterpret_cast<S *>(kr + th * 2 * DK + DK)[i] = P::make(k0.y * ks, k0.w * ks, k1.y * ks, k1.w * ks);
    reinterpret_cast<S *>(qr + th * 2 * DK)[i] = P::make(q0.x * qs, q0.z * qs, q1.x * qs, q1.z * qs);
    reinterpret_cast<S *>(qr + th * 2 * DK + DK)[i] = P::make(q0.y * qs, q0.w * qs, q1.y * qs, q1.w * qs);
    const float vs = lam * KeyScale<DK>::sqrt;
#pragma unroll
    for (int e = 0; e < VPT; e += 4)
        reinterpret_cast<S *>(vr + th * DV + i * VPT + e)[0] =
            P::make(vs * to_f(vin[e]), vs * to_f(vin[e + 1]), vs * to_f(vin[e + 2]), vs * to_f(vin[e + 3]));
    if (i == 0) br[th] = beta[th] * expf(-ll);
}

// Complex state [n, dv, dk] (re, im pairs) -> real state [n, 2dk, dv]: S[a][j] = Re M[j][a] (a < dk),
// Im M[j][a - dk] (a >= dk); one thread per element of S.
__global__ void phase_state_in(const float2 *__restrict__ M, float *__restrict__ S, int dk, int dv, long states)
{
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long per = 2L * dk * dv;
    if (idx >= states * per) return;
    const long n = idx / per;
    const int a = (int)((idx % per) / dv), j = (int)(idx % dv);
    const float2 m = M[n * dk * dv + (long)j * dk + (a < dk ? a : a - dk)];
    S[idx] = a < dk ? m.x : m.y;
}

// The reverse: one thread per complex element of M.
__global__ void phase_state_out(const float *__restrict__ S, float2 *__restrict__ M, int dk, int dv, long states)
{
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long per = (long)dk * dv;
    if (idx >= states * per) return;
    const long n = idx / per;
    const int j = (int)((idx % per) / dk), a = (int)(idx % dk);
    const float *s = S + n * 2 * per;
    M[idx] = make_float2(s[(long)a * dv + j], s[(long)(a + dk) * dv + j]);
}

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct PhasePlan {
    size_t kr, qr, vr, br, s0, sf, ws, total, ws_bytes;
};

// Workspace: the real recurrence's k, q, v (element type of v), b (fp32), its states, and the
// chunk forward's own scratch.
bool phase_plan(PhasePlan &p, int B, int T, int H, int dk, int dv, int varlen, int dtype)
{
    if (dv == 256 && dtype != GDN_DTYPE_BF16) return false;  // the prologue's fp32 forms stop at 128
    const size_t ws = gdn_chunk_fwd_workspace_bytes(B, T, H, 2 * dk, dv, 64, varlen, dtype);
    if (ws == (size_t)-1) return false;
    const size_t es = dtype == GDN_DTYPE_BF16 ? 2 : 4;
    const size_t th = (varlen ? (size_t)T : (size_t)B * T) * H;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += al256(bytes);
        return at;
    };
    p.kr = take(th * 2 * dk * es);
    p.qr = take(th * 2 * dk * es);
    p.vr = take(th * dv * es);
    p.br = take(th * 4);
    p.s0 = take((size_t)B * H * 2 * dk * dv * 4);
    p.sf = take((size_t)B * H * 2 * dk * dv * 4);
    p.ws_bytes = ws;
    p.ws = take(ws);
    p.total = o;
    return true;
}

// The prologue into the workspace regions p.kr, p.qr, p.vr, p.br; v read as TV, written as TO.
template <int DK, int DV, typename TV, typename TO = TV>
cudaError_t launch_prologue(const float *K, const float *Q, const void *V, const float *log_lam, const float *beta,
                            long token_heads, char *w, const PhasePlan &p, cudaStream_t st)
{
    const long threads = token_heads * (DK / 4);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    if (blocks)
        phase_prologue<DK, DV, TV, TO><<<blocks, 256, 0, st>>>(
            reinterpret_cast<const float4 *>(K), reinterpret_cast<const float4 *>(Q), static_cast<const TV *>(V),
            log_lam, beta, token_heads, reinterpret_cast<TO *>(w + p.kr), reinterpret_cast<TO *>(w + p.qr),
            reinterpret_cast<TO *>(w + p.vr), reinterpret_cast<float *>(w + p.br));
    return cudaGetLastError();
}

template <typename TV>
cudaError_t prologue_for(int dk, int dv, const float *K, const float *Q, const void *V, const float *log_lam,
                         const float *beta, long token_heads, char *w, const PhasePlan &p, cudaStream_t st)
{
    if (dk == 64)
        return dv == 256   ? launch_prologue<64, 256, TV>(K, Q, V, log_lam, beta, token_heads, w, p, st)
               : dv == 128 ? launch_prologue<64, 128, TV>(K, Q, V, log_lam, beta, token_heads, w, p, st)
                           : launch_prologue<64, 64, TV>(K, Q, V, log_lam, beta, token_heads, w, p, st);
    return dv == 256   ? launch_prologue<32, 256, TV>(K, Q, V, log_lam, beta, token_heads, w, p, st)
           : dv == 128 ? launch_prologue<32, 128, TV>(K, Q, V, log_lam, beta, token_heads, w, p, st)
                       : launch_prologue<32, 64, TV>(K, Q, V, log_lam, beta, token_heads, w, p, st);
}

// ---- backward ---------------------------------------------------------------------------------
// gdn_phase_bwd runs the fp32 backward of the real recurrence (head size 2 dk = 64, dv = 64) on the
// same map and applies its chain rule: dK = dk_r / sqrt(dk), dQ = dq_r / dk, dV = lam sqrt(dk) dv_r,
// dbeta = db_r / lam, dlog_lam = dlog_a + sum_j dv_r,j v_r,j - db_r b_r, dM0 from the real dS0.

// dout in fp32 (a copy when it arrives in bf16); one thread per element.
template <typename TV>
__global__ void phase_widen(const TV *__restrict__ x, float *__restrict__ y, long n)
{
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = to_f(x[i]);
}

// One warp per token-head (DK = 32 complex key elements: one per lane; DV / 32 values per lane).
template <int DV>
__global__ void __launch_bounds__(256) phase_bwd_epilogue(const float *__restrict__ dq_r,
                                                          const float *__restrict__ dk_r,
                                                          const float *__restrict__ dv_r,
                                                          const float *__restrict__ v_r, const float *__restrict__ dla,
                                                          const float *__restrict__ db_r,
                                                          const float *__restrict__ b_r,
                                                          const float *__restrict__ log_lam, long token_heads,
                                                          float2 *__restrict__ dK, float2 *__restrict__ dQ,
                                                          float *__restrict__ dV, float *__restrict__ dlog_lam,
                                                          float *__restrict__ dbeta)
{
    constexpr int DK = 32;
    const long th = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (th >= token_heads) return;
    const float lam = expf(log_lam[th]);
    dK[th * DK + lane] = make_float2(dk_r[th * 2 * DK + lane] * KeyScale<DK>::inv_sqrt,
                                     dk_r[th * 2 * DK + DK + lane] * KeyScale<DK>::inv_sqrt);
    dQ[th * DK + lane] = make_float2(dq_r[th * 2 * DK + lane] * (1.0f / DK), dq_r[th * 2 * DK + DK + lane] * (1.0f / DK));
    const float vs = lam * KeyScale<DK>::sqrt;
    float dot = 0.f;
#pragma unroll
    for (int j = lane; j < DV; j += 32) {
        const float gj = dv_r[th * DV + j];
        dV[th * DV + j] = vs * gj;
        dot = fmaf(gj, v_r[th * DV + j], dot);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) {
        dlog_lam[th] = dla[th] + dot - db_r[th] * b_r[th];
        dbeta[th] = db_r[th] / lam;
    }
}

struct PhaseBwdPlan {
    size_t kr, qr, vr, br, d32, s0, sf, dq, dk, dv, dla, db, ds0, ws, ws_bytes, total;
};

bool phase_bwd_plan(PhaseBwdPlan &p, int B, int T, int H, int DV, int varlen)
{
    constexpr int DK = 32;
    const size_t ws = gdn_chunk_bwd_workspace_bytes(B, T, H, 2 * DK, DV, 64, varlen);
    if (ws == (size_t)-1) return false;
    const size_t th = (varlen ? (size_t)T : (size_t)B * T) * H, st = (size_t)B * H * 2 * DK * DV * 4;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += al256(bytes);
        return at;
    };
    p.kr = take(th * 2 * DK * 4);
    p.qr = take(th * 2 * DK * 4);
    p.vr = take(th * DV * 4);
    p.br = take(th * 4);
    p.d32 = take(th * DV * 4);
    p.s0 = take(st);
    p.sf = take(st);
    p.dq = take(th * 2 * DK * 4);
    p.dk = take(th * 2 * DK * 4);
    p.dv = take(th * DV * 4);
    p.dla = take(th * 4);
    p.db = take(th * 4);
    p.ds0 = take(st);
    p.ws_bytes = ws;
    p.ws = take(ws);
    p.total = o;
    return true;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" {

size_t gdn_phase_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int varlen, int dtype)
{
    if ((dk != 32 && dk != 64) || (dv != 64 && dv != 128 && dv != 256)) return (size_t)-1;
    PhasePlan p;
    if (!phase_plan(p, B, T, H, dk, dv, varlen, dtype)) return (size_t)-1;
    return p.total;
}

int gdn_phase_fwd(const float *K, const float *Q, const void *v, const float *log_lam, const float *beta,
                  const float *M0, void *out, float *M_final, int B, int T, int H, int dk, int dv,
                  const int32_t *cu_seqlens, int dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    const int varlen = cu_seqlens != nullptr;
    if ((dk != 32 && dk != 64) || (dv != 64 && dv != 128 && dv != 256) || (dv == 256 && dtype != GDN_DTYPE_BF16)) {
        set_error("gdn_phase_fwd: dk=%d dv=%d, supported: dk 32 or 64 (the real recurrence runs at 2 dk), dv 64, "
                  "128 or 256 (256 with bf16)", dk, dv);
        return GDN_ERR_UNSUPPORTED;
    }
    PhasePlan p;
    if (!phase_plan(p, B, T, H, dk, dv, varlen, dtype))  // the chunk forward's shape check gives the reason
        return gdn_chunk_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, T, H, 2 * dk,
                             dv, 64, cu_seqlens, dtype, nullptr, 0, stream);
    if (!K || !Q || !v || !log_lam || !beta || !out) {
        set_error("gdn_phase_fwd: K, Q, v, log_lam, beta and out are required");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    const void *ptrs[] = {K, Q, v, log_lam, beta, M0, out, M_final, cu_seqlens};
    for (const void *ptr : ptrs)
        if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u)) {
            set_error("gdn_phase_fwd: pointer %p is not 16-byte aligned", ptr);
            return GDN_ERR_INVALID_ARGUMENT;
        }
    if (!workspace || workspace_bytes < p.total) {
        set_error("gdn_phase_fwd: workspace of %zu bytes needed, %zu given", p.total,
                  workspace ? workspace_bytes : (size_t)0);
        return GDN_ERR_WORKSPACE;
    }
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) {
        set_error("gdn_phase_fwd: workspace must be 256-byte aligned");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(workspace);
    const long token_heads = (varlen ? (long)T : (long)B * T) * H;
    const long states = (long)B * H;
    cudaError_t e;
    // dk = 32, dv = 64, bf16 in one launch: the chunk kernel reads K, Q, V, log_lam and beta as
    // given and forms the real recurrence's inputs itself (no prologue pass)
    if (dtype == GDN_DTYPE_BF16 && dk == 32 && dv == 64 && phase_fused_ok(B, T, H, varlen)) {
        if (M0) {
            const long n = states * 2 * dk * dv;
            phase_state_in<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float2 *>(M0),
                                                                         reinterpret_cast<float *>(w + p.s0), dk, dv,
                                                                         states);
        }
        e = cudaGetLastError();
        if (e == cudaSuccess)
            e = launch_phase_chunk(K, Q, v, log_lam, beta, M0 ? reinterpret_cast<const float *>(w + p.s0) : nullptr,
                                   out, M_final ? reinterpret_cast<float *>(w + p.sf) : nullptr, cu_seqlens, B, T, H,
                                   st);
        if (e == cudaSuccess && M_final) {
            const long n = states * dk * dv;
            phase_state_out<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float *>(w + p.sf),
                                                                          reinterpret_cast<float2 *>(M_final), dk, dv,
                                                                          states);
            e = cudaGetLastError();
        }
        if (e != cudaSuccess) {
            set_error("gdn_phase_fwd: launch: %s", cudaGetErrorString(e));
            return GDN_ERR_CUDA;
        }
        return GDN_OK;
    }
    e = dtype == GDN_DTYPE_BF16
            ? prologue_for<__nv_bfloat16>(dk, dv, K, Q, v, log_lam, beta, token_heads, w, p, st)
            : prologue_for<float>(dk, dv, K, Q, v, log_lam, beta, token_heads, w, p, st);
    if (e == cudaSuccess && M0) {
        const long n = states * 2 * dk * dv;
        phase_state_in<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float2 *>(M0),
                                                                     reinterpret_cast<float *>(w + p.s0), dk, dv,
                                                                     states);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        set_error("gdn_phase_fwd: launch: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    const int rc = gdn_chunk_fwd(w + p.qr, w + p.kr, w + p.vr, log_lam, reinterpret_cast<const float *>(w + p.br),
                                 M0 ? reinterpret_cast<const float *>(w + p.s0) : nullptr, out,
                                 M_final ? reinterpret_cast<float *>(w + p.sf) : nullptr, B, T, H, 2 * dk, dv, 64,
                                 cu_seqlens, dtype, p.ws_bytes ? w + p.ws : nullptr, p.ws_bytes, stream);
    if (rc != GDN_OK) return rc;
    if (M_final) {
        const long n = states * dk * dv;
        phase_state_out<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float *>(w + p.sf),
                                                                      reinterpret_cast<float2 *>(M_final), dk, dv,
                                                                      states);
        e = cudaGetLastError();
        if (e != cudaSuccess) {
            set_error("gdn_phase_fwd: launch: %s", cudaGetErrorString(e));
            return GDN_ERR_CUDA;
        }
    }
    return GDN_OK;
}


size_t gdn_phase_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int varlen)
{
    if (dk != 32 || (dv != 64 && dv != 128 && dv != 256)) return (size_t)-1;
    PhaseBwdPlan p;
    if (!phase_bwd_plan(p, B, T, H, dv, varlen)) return (size_t)-1;
    return p.total;
}

int gdn_phase_bwd(const float *K, const float *Q, const void *v, const float *log_lam, const float *beta,
                  const float *M0, const void *dout, const float *dM_final, float *dK, float *dQ, float *dv_out,
                  float *dlog_lam, float *dbeta, float *dM0, int B, int T, int H, int dk, int dv,
                  const int32_t *cu_seqlens, int dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    const int varlen = cu_seqlens != nullptr;
    if (dk != 32 || (dv != 64 && dv != 128 && dv != 256) || (dtype != GDN_DTYPE_BF16 && dtype != GDN_DTYPE_F32)) {
        set_error("gdn_phase_bwd: dk=%d dv=%d dtype=%d, supported: dk 32 (64 real), dv 64, 128 or 256, bf16 or fp32",
                  dk, dv, dtype);
        return GDN_ERR_UNSUPPORTED;
    }
    PhaseBwdPlan p;
    if (!phase_bwd_plan(p, B, T, H, dv, varlen))  // the backward's own checks give the reason
        return gdn_chunk_bwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, B, T, H, 2 * dk, dv, 64, cu_seqlens,
                             GDN_DTYPE_F32, nullptr, 0, stream);
    if (!K || !Q || !v || !log_lam || !beta || !dout || !dK || !dQ || !dv_out || !dlog_lam || !dbeta) {
        set_error("gdn_phase_bwd: inputs, dout and every gradient output except dM0 are required");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    const void *ptrs[] = {K, Q, v, log_lam, beta, M0, dout, dM_final, dK, dQ, dv_out, dlog_lam, dbeta, dM0,
                          cu_seqlens};
    for (const void *ptr : ptrs)
        if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u)) {
            set_error("gdn_phase_bwd: pointer %p is not 16-byte aligned", ptr);
            return GDN_ERR_INVALID_ARGUMENT;
        }
    if (!workspace || workspace_bytes < p.total) {
        set_error("gdn_phase_bwd: workspace of %zu bytes needed, %zu given", p.total,
                  workspace ? workspace_bytes : (size_t)0);
        return GDN_ERR_WORKSPACE;
    }
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) {
        set_error("gdn_phase_bwd: workspace must be 256-byte aligned");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(workspace);
    const long th = (varlen ? (long)T : (long)B * T) * H, states = (long)B * H;
    auto fail_launch = [](cudaError_t err) {
        set_error("gdn_phase_bwd: launch: %s", cudaGetErrorString(err));
        return GDN_ERR_CUDA;
    };
    // the forward's prologue, written in fp32: k, q, v, b of the real recurrence
    PhasePlan fp{};
    fp.kr = p.kr;
    fp.qr = p.qr;
    fp.vr = p.vr;
    fp.br = p.br;
    cudaError_t e;
    if (dv == 64)
        e = dtype == GDN_DTYPE_BF16 ? launch_prologue<32, 64, __nv_bfloat16, float>(K, Q, v, log_lam, beta, th, w, fp, st)
                                    : launch_prologue<32, 64, float, float>(K, Q, v, log_lam, beta, th, w, fp, st);
    else if (dv == 128)
        e = dtype == GDN_DTYPE_BF16 ? launch_prologue<32, 128, __nv_bfloat16, float>(K, Q, v, log_lam, beta, th, w, fp, st)
                                    : launch_prologue<32, 128, float, float>(K, Q, v, log_lam, beta, th, w, fp, st);
    else
        e = dtype == GDN_DTYPE_BF16 ? launch_prologue<32, 256, __nv_bfloat16, float>(K, Q, v, log_lam, beta, th, w, fp, st)
                                    : launch_prologue<32, 256, float, float>(K, Q, v, log_lam, beta, th, w, fp, st);
    if (e != cudaSuccess) return fail_launch(e);
    const long nv = th * dv;
    float *d32 = reinterpret_cast<float *>(w + p.d32);
    if (dtype == GDN_DTYPE_BF16) {
        if (nv) phase_widen<__nv_bfloat16><<<(unsigned)((nv + 255) / 256), 256, 0, st>>>(
                static_cast<const __nv_bfloat16 *>(dout), d32, nv);
        e = cudaGetLastError();
    } else if (nv) {
        e = cudaMemcpyAsync(d32, dout, (size_t)nv * 4, cudaMemcpyDeviceToDevice, st);
    }
    if (e != cudaSuccess) return fail_launch(e);
    const long ns = states * 2 * dk * dv;
    if (M0) phase_state_in<<<(unsigned)((ns + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float2 *>(M0),
                                                                          reinterpret_cast<float *>(w + p.s0), dk, dv,
                                                                          states);
    if (dM_final)
        phase_state_in<<<(unsigned)((ns + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float2 *>(dM_final),
                                                                     reinterpret_cast<float *>(w + p.sf), dk, dv,
                                                                     states);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail_launch(e);
    float *dq = reinterpret_cast<float *>(w + p.dq), *dkr = reinterpret_cast<float *>(w + p.dk),
          *dvr = reinterpret_cast<float *>(w + p.dv), *dla = reinterpret_cast<float *>(w + p.dla),
          *dbr = reinterpret_cast<float *>(w + p.db);
    const int rc = gdn_chunk_bwd(w + p.qr, w + p.kr, w + p.vr, log_lam, reinterpret_cast<const float *>(w + p.br),
                                 M0 ? reinterpret_cast<const float *>(w + p.s0) : nullptr, d32,
                                 dM_final ? reinterpret_cast<const float *>(w + p.sf) : nullptr, dq, dkr, dvr, dla,
                                 dbr, dM0 ? reinterpret_cast<float *>(w + p.ds0) : nullptr, B, T, H, 2 * dk, dv, 64,
                                 cu_seqlens, GDN_DTYPE_F32, w + p.ws, p.ws_bytes, stream);
    if (rc != GDN_OK) return rc;
    if (th) {
        auto epi = dv == 64 ? phase_bwd_epilogue<64> : dv == 128 ? phase_bwd_epilogue<128> : phase_bwd_epilogue<256>;
        epi<<<(unsigned)((th * 32 + 255) / 256), 256, 0, st>>>(
            dq, dkr, dvr, reinterpret_cast<const float *>(w + p.vr), dla, dbr,
            reinterpret_cast<const float *>(w + p.br), log_lam, th, reinterpret_cast<float2 *>(dK),
            reinterpret_cast<float2 *>(dQ), dv_out, dlog_lam, dbeta);
    }
    if (dM0) {
        const long nm = states * dk * dv;
        phase_state_out<<<(unsigned)((nm + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float *>(w + p.ds0),
                                                                       reinterpret_cast<float2 *>(dM0), dk, dv,
                                                                       states);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail_launch(e);
    return GDN_OK;
}

}  // extern "C"
