// gdn_chunk_simt.cu -- chunkwise (WY / UT-transform) forward of the gated delta rule on CUDA
// cores, fp32 arithmetic throughout.  This is the library's path for fp32 inputs, where the
// fp32 tolerance rules out bf16 tensor-core operands.
//
// Sources: Sykra README, "Architectural Highlights" (chunk-parallel training via the WY / unit
// triangular transform, a triangular solve per chunk); DeltaPhase README, section 1 ("Fast
// Triangular Solve": exact O(C^2) per-chunk transition solve).  For a chunk of C = 64 tokens
// entered with state S (dk x dv):
//   A  = strictly_lower(diag(b) (Gam o K K^T))      T = (I + A)^{-1}
//   W  = T diag(b gam) K                            U = T diag(b) V - W S
//   O  = diag(gam) Q S + lower_incl(Gam o Q K^T) U
//   S' = gam_C S + (diag(lam) K)^T U
// Gam[r][i] = prod_{j=i+1..r} a_j, gam[r] = prod_{j<=r} a_j, lam[i] = Gam[C-1][i].
//
// Gates: the decays are exp of sums of log_alpha taken from the last exact reset
// (log_alpha = -inf) inside the chunk, so a reset gives exact zeros and never 0 * inf or
// inf - inf.  A partial last chunk is padded with k = v = q = 0, b = 0, log_alpha = 0, which
// leaves the state unchanged on the padded rows.
//
// Grid: one CTA per (value block of 64 columns, head, sequence); the CTA walks its sequence
// chunk by chunk with the state block in shared memory.  Value columns are independent in the
// recurrence (column j of S and O depends only on column j of V and S0), so the blocks need
// no communication.
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

constexpr int C = 64;         // chunk length
constexpr int VB = 64;        // value columns per CTA
constexpr int kThreads = 256;

__device__ __forceinline__ float ld_f32(const float *p) { return *p; }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <int DK>
struct SimtSmem {
    float Q[C][DK + 1];
    float K[C][DK + 1];
    float W[C][DK + 1];
    float S[DK][VB + 1];
    float V[C][VB + 1];
    float U[C][VB + 1];
    float T[C][C + 1];
    float P[C][C + 1];
    float G[C];    // log-decay sums from the last reset (or the chunk start)
    int last[C];   // index of the last reset at or before row r, -1 if none
    float gam[C];
    float lam[C];
    float bet[C];
};

template <int DK, typename TIn>
__global__ void __launch_bounds__(kThreads)
chunk_simt_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                  const float *__restrict__ log_alpha, const float *__restrict__ beta,
                  const float *__restrict__ S0, TIn *__restrict__ out, float *__restrict__ S_final,
                  const int32_t *__restrict__ cu_seqlens, int T, int H, int DV, int G)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem<DK> &sm = *reinterpret_cast<SimtSmem<DK> *>(smem_raw);

    const int vb = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x;
    long tok0, len;
    if (cu_seqlens) {
        tok0 = cu_seqlens[s];
        len = (long)cu_seqlens[s + 1] - tok0;
    } else {
        tok0 = (long)s * T;
        len = T;
    }
    const size_t state_off = ((size_t)s * H + h) * (size_t)DK * DV + (size_t)vb * VB;

    // initial state block
    for (int idx = tid; idx < DK * VB; idx += kThreads) {
        const int i = idx / VB, j = idx % VB;
        sm.S[i][j] = S0 ? S0[state_off + (size_t)i * DV + j] : 0.f;
    }

    for (long c0 = 0; c0 < len; c0 += C) {
        const int n = (int)min((long)C, len - c0);
        __syncthreads();  // previous chunk fully consumed
        // ---- load the chunk (zero padding past the sequence end) ----
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int r = idx / DK, c = idx % DK;
            float qv = 0.f, kv = 0.f;
            if (r < n) {
                const size_t off = ((size_t)(tok0 + c0 + r) * (H / G) + h / G) * DK + c;  // q/k head h / G
                qv = ld_f32(q + off);
                kv = ld_f32(k + off);
            }
            sm.Q[r][c] = qv;
            sm.K[r][c] = kv;
        }
        for (int idx = tid; idx < C * VB; idx += kThreads) {
            const int r = idx / VB, c = idx % VB;
            float x = 0.f;
            if (r < n) x = ld_f32(v + ((size_t)(tok0 + c0 + r) * H + h) * DV + vb * VB + c);
            sm.V[r][c] = x;
        }
        if (tid < C) {
            const int r = tid;
            float g = 0.f, b = 0.f;
            if (r < n) {
                const size_t off = (size_t)(tok0 + c0 + r) * H + h;
                g = log_alpha[off];
                b = beta[off];
            }
            sm.G[r] = g;  // raw log-gate for now
            sm.bet[r] = b;
        }
        __syncthreads();
        // ---- gate sums from the last reset (one thread; 64 steps) ----
        if (tid == 0) {
            float acc = 0.f;
            int last = -1;
            for (int r = 0; r < C; ++r) {
                const float g = sm.G[r];
                if (g == -INFINITY) {
                    last = r;
                    acc = 0.f;
                } else {
                    acc += g;
                }
                sm.G[r] = acc;
                sm.last[r] = last;
            }
        }
        __syncthreads();
        if (tid < C) {
            const int r = tid;
            sm.gam[r] = sm.last[r] >= 0 ? 0.f : expf(sm.G[r]);
            // lam[i] = Gam[C-1][i]
            sm.lam[r] = sm.last[C - 1] > r ? 0.f : expf(sm.G[C - 1] - sm.G[r]);
        }
        // ---- A (into T's storage for now) and P ----
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int r = idx / C, i = idx % C;
            float a = 0.f, p = 0.f;
            if (i <= r) {
                const float gm = sm.last[r] > i ? 0.f : expf(sm.G[r] - sm.G[i]);
                float kk = 0.f, qk = 0.f;
                for (int c = 0; c < DK; ++c) {
                    kk = fmaf(sm.K[r][c], sm.K[i][c], kk);
                    qk = fmaf(sm.Q[r][c], sm.K[i][c], qk);
                }
                if (i < r) a = sm.bet[r] * gm * kk;
                p = gm * qk;
            }
            sm.U[r][i] = a;  // A staged in U (64 x 64) until T is formed
            sm.P[r][i] = p;
        }
        __syncthreads();
        // ---- T = (I + A)^{-1} by forward substitution, one column per thread ----
        if (tid < C) {
            const int c = tid;
            for (int r = 0; r < C; ++r) {
                float x;
                if (r < c) x = 0.f;
                else if (r == c) x = 1.f;
                else {
                    x = 0.f;
                    for (int i = c; i < r; ++i) x = fmaf(sm.U[r][i], sm.T[i][c], x);
                    x = -x;
                }
                sm.T[r][c] = x;
            }
        }
        __syncthreads();
        // ---- W = T diag(b gam) K ----
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int r = idx / DK, c = idx % DK;
            float w = 0.f;
            for (int i = 0; i <= r; ++i) w = fmaf(sm.T[r][i] * (sm.bet[i] * sm.gam[i]), sm.K[i][c], w);
            sm.W[r][c] = w;
        }
        __syncthreads();
        // ---- U = T diag(b) V - W S ----
        for (int idx = tid; idx < C * VB; idx += kThreads) {
            const int r = idx / VB, j = idx % VB;
            float x = 0.f;
            for (int i = 0; i <= r; ++i) x = fmaf(sm.T[r][i] * sm.bet[i], sm.V[i][j], x);
            float ws = 0.f;
            for (int c = 0; c < DK; ++c) ws = fmaf(sm.W[r][c], sm.S[c][j], ws);
            sm.U[r][j] = x - ws;
        }
        __syncthreads();
        // ---- O = diag(gam) Q S + P U  (rows past the sequence end are not stored) ----
        for (int idx = tid; idx < C * VB; idx += kThreads) {
            const int r = idx / VB, j = idx % VB;
            if (r >= n) continue;
            float qs = 0.f;
            for (int c = 0; c < DK; ++c) qs = fmaf(sm.Q[r][c], sm.S[c][j], qs);
            float pu = 0.f;
            for (int i = 0; i <= r; ++i) pu = fmaf(sm.P[r][i], sm.U[i][j], pu);
            st_out(out + ((size_t)(tok0 + c0 + r) * H + h) * DV + vb * VB + j,
                   fmaf(sm.gam[r], qs, pu));
        }
        __syncthreads();
        // ---- S' = gam_C S + K^T diag(lam) U ----
        const float gC = sm.gam[C - 1];
        for (int idx = tid; idx < DK * VB; idx += kThreads) {
            const int c = idx / VB, j = idx % VB;
            float x = 0.f;
            for (int r = 0; r < C; ++r) x = fmaf(sm.K[r][c] * sm.lam[r], sm.U[r][j], x);
            sm.S[c][j] = fmaf(gC, sm.S[c][j], x);
        }
    }
    __syncthreads();
    if (S_final) {
        for (int idx = tid; idx < DK * VB; idx += kThreads) {
            const int i = idx / VB, j = idx % VB;
            S_final[state_off + (size_t)i * DV + j] = sm.S[i][j];
        }
    }
}

template <int DK, typename TIn>
cudaError_t launch_dk(const ChunkArgs &a, cudaStream_t st)
{
    const size_t smem = sizeof(SimtSmem<DK>);
    auto kern = chunk_simt_kernel<DK, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.dv / VB, a.H, a.B);
    kern<<<grid, kThreads, smem, st>>>(
        static_cast<const TIn *>(a.q), static_cast<const TIn *>(a.k), static_cast<const TIn *>(a.v),
        a.log_alpha, a.beta, a.S0, static_cast<TIn *>(a.out), a.S_final, a.cu_seqlens, a.T, a.H,
        a.dv, a.G);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream)
{
    if (a.dtype == GDN_DTYPE_BF16)
        return a.dk == 128 ? launch_dk<128, __nv_bfloat16>(a, stream) : launch_dk<64, __nv_bfloat16>(a, stream);
    return a.dk == 128 ? launch_dk<128, float>(a, stream) : launch_dk<64, float>(a, stream);
}

}  // namespace gdn
