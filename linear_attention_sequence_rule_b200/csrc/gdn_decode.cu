// gdn_decode.cu -- one-token decode step of the gated delta rule, streamed at HBM speed.
//
// Source: Sykra README, "Architectural Highlights" (generation updates a fixed d x d state per
// token) and "Computational Complexity" (O(d^2) per decode step).  With r = S^T k and s = S^T q
// taken from the state before the step:
//     u = b (v - a r),   out = a s + (k . q) u,   S <- a S + k u^T
// which is S_t = a (I - b k k^T) S + b k v^T followed by out = S_t^T q, regrouped so that the
// state is read once and written once.
//
// Design: one CTA of 256 threads per (n, h) state.  Thread t owns four adjacent value columns
// (one float4) of every (256 / (dv/4))-th row: a warp covers whole 512-byte rows, so every load
// and store is a coalesced 16-byte access.  The whole state is loaded into registers before any
// arithmetic (dk*dv*4 bytes in flight per CTA), the two column sums S^T k and S^T q are reduced
// across row groups through shared memory, and the updated state is written back with
// streaming stores.  The state is touched by no other CTA, so there is no inter-CTA traffic.
// A value head of VB x DV columns runs as VB CTAs per state (blockIdx.y = column block): value
// columns do not interact in the step, so each CTA updates its own columns of every row.
// PRO (gdn_decode_step_fused): q, k are raw rows and log_alpha, beta hold the raw gate projections
// a, b; the kernel forms k / sqrt(|k|^2 + 1e-6), q likewise, log alpha = -a_scale softplus(a)
// (a = +inf: an exact reset) and beta = b_scale sigmoid(b).  The norms come out of the same
// block reduction as k . q, and the scales are applied to the reduced sums, so the state is still
// read and written once.
#include <cuda_bf16.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

__device__ __forceinline__ float sigmoid_f(float x)
{
    const float e = expf(-fabsf(x));
    return x >= 0.f ? 1.f / (1.f + e) : e / (1.f + e);
}

__device__ __forceinline__ float softplus_f(float x) { return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x)); }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

constexpr int kThreads = 256;

template <int DK, int DV, int VB, typename TIn, bool PRO>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ S, TIn *__restrict__ out, int H, int G, float a_scale, float b_scale)
{
    constexpr int TPR = DV / 4;          // threads per state row (one float4 each)
    constexpr int RPP = kThreads / TPR;  // rows covered per pass
    constexpr int R = DK / RPP;          // rows per thread
    static_assert(R * RPP == DK, "row split");
    constexpr int LDV = VB * DV;         // row length of v, out and the state

    __shared__ float4 red_r[RPP][TPR];
    __shared__ float4 red_s[RPP][TPR];
    __shared__ float red_kq[RPP];
    __shared__ float red_kk[PRO ? RPP : 1], red_qq[PRO ? RPP : 1];

    const size_t u = blockIdx.x;  // state index n * H + h
    const int tid = threadIdx.x;
    const int c4 = tid % TPR;
    const int rg = tid / TPR;  // row group: rows rg, rg + RPP, ...
    const int col0 = VB == 1 ? 0 : (int)blockIdx.y * DV;

    float4 *Sp = reinterpret_cast<float4 *>(S + u * (size_t)(DK * LDV) + col0);
    float4 s[R];
#pragma unroll
    for (int p = 0; p < R; ++p) s[p] = __ldcs(&Sp[(rg + p * RPP) * (LDV / 4) + c4]);

    // q/k of state (n, h) live at (n, h / G) among the H / G q/k heads (grouped value heads)
    const size_t uq = G == 1 ? u : (size_t)((unsigned)u / (unsigned)H) * (unsigned)(H / G) + ((unsigned)u % (unsigned)H) / (unsigned)G;
    const TIn *kp = k + uq * DK;
    const TIn *qp = q + uq * DK;
    float kr[R], qr[R];
#pragma unroll
    for (int p = 0; p < R; ++p) {
        kr[p] = to_f32(kp[rg + p * RPP]);
        qr[p] = to_f32(qp[rg + p * RPP]);
    }
    float a, b;
    if constexpr (PRO) {
        const float ar = log_alpha[u];
        a = ar == INFINITY ? 0.f : expf(-a_scale * softplus_f(ar));
        b = b_scale * sigmoid_f(beta[u]);
    } else {
        a = expf(log_alpha[u]);
        b = beta[u];
    }
    float vv[4];
    {
        const TIn *vp = v + u * LDV + col0 + 4 * c4;
#pragma unroll
        for (int j = 0; j < 4; ++j) vv[j] = to_f32(vp[j]);
    }

    // partial column sums over this thread's rows
    float4 pr = make_float4(0.f, 0.f, 0.f, 0.f), ps = pr;
    float pkq = 0.f, pkk = 0.f, pqq = 0.f;
#pragma unroll
    for (int p = 0; p < R; ++p) {
        if constexpr (PRO) {
            pkk = fmaf(kr[p], kr[p], pkk);
            pqq = fmaf(qr[p], qr[p], pqq);
        }
        pr.x = fmaf(s[p].x, kr[p], pr.x); pr.y = fmaf(s[p].y, kr[p], pr.y);
        pr.z = fmaf(s[p].z, kr[p], pr.z); pr.w = fmaf(s[p].w, kr[p], pr.w);
        ps.x = fmaf(s[p].x, qr[p], ps.x); ps.y = fmaf(s[p].y, qr[p], ps.y);
        ps.z = fmaf(s[p].z, qr[p], ps.z); ps.w = fmaf(s[p].w, qr[p], ps.w);
        pkq = fmaf(kr[p], qr[p], pkq);
    }
    red_r[rg][c4] = pr;
    red_s[rg][c4] = ps;
    if (c4 == 0) {
        red_kq[rg] = pkq;
        if constexpr (PRO) {
            red_kk[rg] = pkk;
            red_qq[rg] = pqq;
        }
    }
    __syncthreads();

    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), sq = r;
    float kq = 0.f;
#pragma unroll
    for (int g = 0; g < RPP; ++g) {
        const float4 x = red_r[g][c4], y = red_s[g][c4];
        r.x += x.x; r.y += x.y; r.z += x.z; r.w += x.w;
        sq.x += y.x; sq.y += y.y; sq.z += y.z; sq.w += y.w;
        kq += red_kq[g];
    }
    if constexpr (PRO) {  // S^T k, S^T q and k . q of the normalised rows from the raw sums
        float kk = 0.f, qq = 0.f;
#pragma unroll
        for (int g = 0; g < RPP; ++g) {
            kk += red_kk[g];
            qq += red_qq[g];
        }
        const float rk = 1.f / sqrtf(kk + 1e-6f), rq = 1.f / sqrtf(qq + 1e-6f);
        r.x *= rk; r.y *= rk; r.z *= rk; r.w *= rk;
        sq.x *= rq; sq.y *= rq; sq.z *= rq; sq.w *= rq;
        kq *= rk * rq;
#pragma unroll
        for (int p = 0; p < R; ++p) kr[p] *= rk;
    }
    // u = b (v - a r)
    const float u0 = b * (vv[0] - a * r.x), u1 = b * (vv[1] - a * r.y);
    const float u2 = b * (vv[2] - a * r.z), u3 = b * (vv[3] - a * r.w);

#pragma unroll
    for (int p = 0; p < R; ++p) {
        float4 t;
        t.x = fmaf(a, s[p].x, kr[p] * u0);
        t.y = fmaf(a, s[p].y, kr[p] * u1);
        t.z = fmaf(a, s[p].z, kr[p] * u2);
        t.w = fmaf(a, s[p].w, kr[p] * u3);
        __stcs(&Sp[(rg + p * RPP) * (LDV / 4) + c4], t);
    }
    if (rg == 0) {
        TIn *op = out + u * LDV + col0 + 4 * c4;
        op[0] = from_f32<TIn>(fmaf(a, sq.x, kq * u0));
        op[1] = from_f32<TIn>(fmaf(a, sq.y, kq * u1));
        op[2] = from_f32<TIn>(fmaf(a, sq.z, kq * u2));
        op[3] = from_f32<TIn>(fmaf(a, sq.w, kq * u3));
    }
}

template <typename TIn, bool PRO>
cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *la,
                         const float *be, float *S, void *out, int NH, int H, int G, int dk, int dv,
                         float as, float bs, cudaStream_t st)
{
    const dim3 grid(NH), block(kThreads);
    const TIn *Q = static_cast<const TIn *>(q), *K = static_cast<const TIn *>(k),
              *V = static_cast<const TIn *>(v);
    TIn *O = static_cast<TIn *>(out);
    const dim3 grid2(NH, 2);  // dv = 256: two 128-column blocks per state
    if (dk == 256) {
        // key head size 256: 64-column blocks (a thread then holds 16 float4 of the state, as at
        // dk = dv = 128), dv / 64 CTAs per state
        const dim3 gridk(NH, dv / 64);
        if (dv == 64) decode_kernel<256, 64, 1, TIn, PRO><<<gridk, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
        else if (dv == 128) decode_kernel<256, 64, 2, TIn, PRO><<<gridk, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
        else decode_kernel<256, 64, 4, TIn, PRO><<<gridk, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
    } else if (dk == 128 && dv == 256) decode_kernel<128, 128, 2, TIn, PRO><<<grid2, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
    else if (dk == 64 && dv == 256) decode_kernel<64, 128, 2, TIn, PRO><<<grid2, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
    else if (dk == 128 && dv == 128) decode_kernel<128, 128, 1, TIn, PRO><<<grid, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
    else if (dk == 128 && dv == 64) decode_kernel<128, 64, 1, TIn, PRO><<<grid, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
    else if (dk == 64 && dv == 128) decode_kernel<64, 128, 1, TIn, PRO><<<grid, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
    else decode_kernel<64, 64, 1, TIn, PRO><<<grid, block, 0, st>>>(Q, K, V, la, be, S, O, H, G, as, bs);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, void *out, int N, int H, int dk, int dv,
                          int dtype, cudaStream_t stream, int G, int prologue, float a_scale, float b_scale)
{
    const int NH = N * H;
    if (prologue)
        return dtype == GDN_DTYPE_BF16
                   ? launch_typed<__nv_bfloat16, true>(q, k, v, log_alpha, beta, S, out, NH, H, G, dk, dv, a_scale,
                                                       b_scale, stream)
                   : launch_typed<float, true>(q, k, v, log_alpha, beta, S, out, NH, H, G, dk, dv, a_scale, b_scale,
                                               stream);
    if (dtype == GDN_DTYPE_BF16)
        return launch_typed<__nv_bfloat16, false>(q, k, v, log_alpha, beta, S, out, NH, H, G, dk, dv, 0.f, 0.f,
                                                  stream);
    return launch_typed<float, false>(q, k, v, log_alpha, beta, S, out, NH, H, G, dk, dv, 0.f, 0.f, stream);
}

}  // namespace gdn
