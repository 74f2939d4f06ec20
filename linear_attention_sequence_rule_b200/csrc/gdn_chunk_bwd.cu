// gdn_chunk_bwd.cu -- gradients of the chunk forward (dq, dk, dv, dlog_alpha, dbeta, dS0) on the
// CUDA cores in fp32, for dk = dv = 64 (the training path; Sykra README, "Architectural
// Highlights": chunk-parallel training through the WY / UT transform).
//
// Per chunk of C = 64 tokens with entry state S (the forward's chunk form):
//   A = strictly_lower(diag(b) (Gam o K K^T)),  T = (I + A)^{-1}
//   W = T diag(b gam) K,  U~ = T diag(b) V,  U = U~ - W S,  P = lower_incl(Gam o Q K^T)
//   O = diag(gam) Q S + P U,   S' = gam_C S + K^T diag(lam) U
// so the chunk maps states and state gradients affinely:
//   S'  = M S + Bm,              M  = gam_C I - K^T diag(lam) W,   Bm = K^T diag(lam) U~
//   dS  = M^T dS' + R,           R  = (Q^T diag(gam) - W^T P^T) dO
// Four kernels:
//   bwd_prep   (chunk x head, parallel)  : T, W, U~, P  ->  M, Bm, R
//   bwd_fscan  (sequence x head)         : S_c for every chunk, from S0
//   bwd_bscan  (sequence x head, reverse): dS at every chunk's end, from dS_final; dS0
//   bwd_grads  (chunk x head, parallel)  : with S_c and dS_{c+1}, every input gradient of the chunk
// All matrices are 64 x 64 fp32 in shared memory (row stride 65); 256 threads; a matrix product
// gives each thread a 4 x 4 block of the result.
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

constexpr int N = 64;          // chunk length = dk = dv
constexpr int LD = 65;         // shared-memory row stride
constexpr int MAT = N * LD;    // floats per matrix
constexpr int kThreads = 256;

__device__ __forceinline__ float ld_in(const float *p) { return *p; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// One chunk's place: sequence, first token, valid rows, chunk index inside the sequence.
struct ChunkRef {
    int seq, chunk, n;
    long tok;
};

// Chunk table entry e of `nseq` sequences (dense: T tokens each; varlen: cu offsets), or n = 0
// when e lies past the last chunk.  `off` (varlen) holds the first chunk index of every
// sequence, off[nseq] = total.
__device__ ChunkRef chunk_ref(int e, const int32_t *cu, const int32_t *off, int nseq, int T)
{
    ChunkRef r{0, 0, 0, 0};
    if (!cu) {
        const int per = (T + N - 1) / N;
        if (e >= nseq * per) return r;
        r.seq = e / per;
        r.chunk = e % per;
        r.tok = (long)r.seq * T + (long)r.chunk * N;
        r.n = min(N, T - r.chunk * N);
        return r;
    }
    if (e >= off[nseq]) return r;
    int lo = 0, hi = nseq - 1;  // last sequence with off[s] <= e
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= e) lo = mid;
        else hi = mid - 1;
    }
    r.seq = lo;
    r.chunk = e - off[lo];
    r.tok = (long)cu[lo] + (long)r.chunk * N;
    r.n = (int)min((long)N, (long)cu[lo + 1] - r.tok);
    return r;
}

// C(r, c) = sum_k opA(r, k) ks[k] opB(k, c) for 64 x 64 operands (ks: optional diagonal, NULL = 1);
// thread t gets rows 4 (t / 16) .. +3 and columns 4 (t % 16) .. +3 and hands each result to
// emit(r, c, value).
template <bool TA, bool TB, typename F>
__device__ __forceinline__ void mm(const float *A, const float *B, int t, F &&emit, const float *ks = nullptr)
{
    const int r0 = (t >> 4) * 4, c0 = (t & 15) * 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < N; ++k) {
        float a[4], b[4];
        const float sk = ks ? ks[k] : 1.f;  // optional scale of the summation index (a diagonal)
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = (TA ? A[k * LD + r0 + i] : A[(r0 + i) * LD + k]) * sk;
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = TB ? B[(c0 + j) * LD + k] : B[k * LD + c0 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) emit(r0 + i, c0 + j, acc[i][j]);
}

// Gate vectors of one chunk (thread 0 computes them; the caller synchronises):
// G[r] = sum of log_alpha over (last reset, r], last[r] = last exact reset at or before r (-1:
// none), gam[r] = exp(G[r]) (0 after a reset), lam[i] = exp(G[63] - G[i]) (0 when a reset lies in
// (i, 63]), bet[r]; padded rows get log_alpha = 0, beta = 0.
struct Gates {
    float G[N], gam[N], lam[N], bet[N];
    int last[N];
};

template <typename TIn>
__device__ void chunk_gates(Gates &g, const float *log_alpha, const float *beta, const ChunkRef &c, int H, int h,
                            int t)
{
    if (t == 0) {
        float acc = 0.f;
        int lst = -1;
        for (int r = 0; r < N; ++r) {
            const size_t off = (size_t)(c.tok + r) * H + h;
            const float la = r < c.n ? log_alpha[off] : 0.f;
            g.bet[r] = r < c.n ? beta[off] : 0.f;
            if (la == -INFINITY) {
                lst = r;
                acc = 0.f;
            } else {
                acc += la;
            }
            g.G[r] = acc;
            g.last[r] = lst;
        }
        for (int r = 0; r < N; ++r) {
            g.gam[r] = g.last[r] >= 0 ? 0.f : expf(g.G[r]);
            g.lam[r] = g.last[N - 1] > r ? 0.f : expf(g.G[N - 1] - g.G[r]);
        }
    }
}

// Decay between token i and a later token r of the chunk (zero across a reset or for i > r).
__device__ __forceinline__ float decay(const Gates &g, int r, int i)
{
    return (i <= r && g.last[r] <= i) ? expf(g.G[r] - g.G[i]) : 0.f;
}

// Rows of a [tokens, H, 64] tensor into a 64 x LD shared matrix (zero past the chunk end).
template <typename TIn>
__device__ void load_rows(float *M, const TIn *x, const ChunkRef &c, int H, int h, int t)
{
    for (int e = t; e < N * N; e += kThreads) {
        const int r = e >> 6, j = e & 63;
        M[r * LD + j] = r < c.n ? ld_in(x + ((size_t)(c.tok + r) * H + h) * N + j) : 0.f;
    }
}

// T = (I + A)^{-1} for strictly lower A (only entries below the diagonal are read): column c by
// forward substitution on thread c (threads 0..63); every entry of T is written.
__device__ void unit_lower_inverse(const float *A, float *Tm, int t)
{
    if (t < N) {
        const int c = t;
        float x[N];
#pragma unroll
        for (int r = 0; r < N; ++r) {
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) s = fmaf(A[r * LD + i], x[i], s);
            x[r] = r < c ? 0.f : (r == c ? 1.f : -s);
        }
#pragma unroll
        for (int r = 0; r < N; ++r) Tm[r * LD + c] = x[r];
    }
}

// ---- bwd_prep: per (chunk, head) the forward map (M, Bm) and the output term R ----------------
template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_prep(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
             const float *__restrict__ log_alpha, const float *__restrict__ beta, const TIn *__restrict__ dout,
             const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int nseq, int T, int H,
             float *__restrict__ Mo, float *__restrict__ Bo, float *__restrict__ Ro)
{
    extern __shared__ float smf[];
    float *K = smf, *Q = K + MAT, *V = Q + MAT, *dO = V + MAT, *A = dO + MAT, *Tm = A + MAT, *W = Tm + MAT,
          *Ut = W + MAT, *P = Ut + MAT;
    Gates &g = *reinterpret_cast<Gates *>(P + MAT);
    float *bg = reinterpret_cast<float *>(&g + 1);  // beta gam
    const int t = threadIdx.x, h = blockIdx.y, e = blockIdx.x;
    const ChunkRef c = chunk_ref(e, cu, off, nseq, T);
    if (c.n == 0) return;
    load_rows(K, k, c, H, h, t);
    load_rows(Q, q, c, H, h, t);
    load_rows(V, v, c, H, h, t);
    load_rows(dO, dout, c, H, h, t);
    chunk_gates<TIn>(g, log_alpha, beta, c, H, h, t);
    __syncthreads();
    if (t < N) bg[t] = g.bet[t] * g.gam[t];
    mm<false, true>(K, K, t, [&](int r, int i, float x) { A[r * LD + i] = i < r ? g.bet[r] * decay(g, r, i) * x : 0.f; });
    mm<false, true>(Q, K, t, [&](int r, int i, float x) { P[r * LD + i] = decay(g, r, i) * x; });
    __syncthreads();
    unit_lower_inverse(A, Tm, t);
    __syncthreads();
    mm<false, false>(Tm, K, t, [&](int r, int m, float x) { W[r * LD + m] = x; }, bg);
    mm<false, false>(Tm, V, t, [&](int r, int j, float x) { Ut[r * LD + j] = x; }, g.bet);
    mm<true, false>(P, dO, t, [&](int i, int j, float x) { A[i * LD + j] = x; });  // Y = P^T dO (A is free)
    __syncthreads();
    const size_t base = ((size_t)e * H + h) * (size_t)(N * N);
    const float gC = g.gam[N - 1];
    mm<true, false>(K, W, t, [&](int m, int n2, float x) { Mo[base + m * N + n2] = (m == n2 ? gC : 0.f) - x; }, g.lam);
    mm<true, false>(K, Ut, t, [&](int m, int j, float x) { Bo[base + m * N + j] = x; }, g.lam);
    mm<true, false>(Q, dO, t, [&](int m, int j, float x) { Tm[m * LD + j] = x; }, g.gam);  // T is free
    __syncthreads();
    mm<true, false>(W, A, t, [&](int m, int j, float x) { Ro[base + m * N + j] = Tm[m * LD + j] - x; });
}

// Number of chunks of sequence s and the table index of its first chunk.
__device__ __forceinline__ void seq_chunks(int s, const int32_t *cu, const int32_t *off, int T, int &first, int &count)
{
    if (cu) {
        first = off[s];
        count = off[s + 1] - off[s];
    } else {
        count = (T + N - 1) / N;
        first = s * count;
    }
}

// ---- bwd_fscan: S_c for every chunk of one (sequence, head), from S0 ------------------------
__global__ void __launch_bounds__(kThreads, 1)
    bwd_fscan(const float *__restrict__ Mo, const float *__restrict__ Bo, const float *__restrict__ S0,
              const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int T, int H, float *__restrict__ Sc)
{
    extern __shared__ float smf[];
    float *S = smf, *Mm = S + MAT;
    const int t = threadIdx.x, h = blockIdx.x, s = blockIdx.y;
    int first, count;
    seq_chunks(s, cu, off, T, first, count);
    const size_t st0 = ((size_t)s * H + h) * (size_t)(N * N);
    for (int i = t; i < N * N; i += kThreads) S[(i >> 6) * LD + (i & 63)] = S0 ? S0[st0 + i] : 0.f;
    __syncthreads();
    for (int cc = 0; cc < count; ++cc) {
        const size_t base = ((size_t)(first + cc) * H + h) * (size_t)(N * N);
        for (int i = t; i < N * N; i += kThreads) {
            Sc[base + i] = S[(i >> 6) * LD + (i & 63)];
            Mm[(i >> 6) * LD + (i & 63)] = Mo[base + i];
        }
        __syncthreads();
        float nx[16];
        int idx = 0;
        mm<false, false>(Mm, S, t, [&](int r, int j, float x) { nx[idx++] = x + Bo[base + r * N + j]; });
        __syncthreads();
        idx = 0;
        mm<false, false>(Mm, S, t, [&](int r, int j, float) { S[r * LD + j] = nx[idx++]; });
        __syncthreads();
    }
}

// ---- bwd_bscan: dL/dS at the end of every chunk (reverse), and dS0 ---------------------------
__global__ void __launch_bounds__(kThreads, 1)
    bwd_bscan(const float *__restrict__ Mo, const float *__restrict__ Ro, const float *__restrict__ dS_final,
              const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int T, int H, float *__restrict__ dSn,
              float *__restrict__ dS0)
{
    extern __shared__ float smf[];
    float *D = smf, *Mm = D + MAT;
    const int t = threadIdx.x, h = blockIdx.x, s = blockIdx.y;
    int first, count;
    seq_chunks(s, cu, off, T, first, count);
    const size_t st0 = ((size_t)s * H + h) * (size_t)(N * N);
    for (int i = t; i < N * N; i += kThreads) D[(i >> 6) * LD + (i & 63)] = dS_final ? dS_final[st0 + i] : 0.f;
    __syncthreads();
    for (int cc = count - 1; cc >= 0; --cc) {
        const size_t base = ((size_t)(first + cc) * H + h) * (size_t)(N * N);
        for (int i = t; i < N * N; i += kThreads) {
            dSn[base + i] = D[(i >> 6) * LD + (i & 63)];
            Mm[(i >> 6) * LD + (i & 63)] = Mo[base + i];
        }
        __syncthreads();
        float nx[16];
        int idx = 0;
        mm<true, false>(Mm, D, t, [&](int r, int j, float x) { nx[idx++] = x + Ro[base + r * N + j]; });
        __syncthreads();
        idx = 0;
        mm<true, false>(Mm, D, t, [&](int r, int j, float) { D[r * LD + j] = nx[idx++]; });
        __syncthreads();
    }
    if (dS0)
        for (int i = t; i < N * N; i += kThreads) dS0[st0 + i] = D[(i >> 6) * LD + (i & 63)];
}

// ---- bwd_grads: every input gradient of one (chunk, head) --------------------------------------
// With S = S_c and dS' = dL/dS_{c+1}:
//   dU = P^T dO + diag(lam) K dS'          dW = -dU S^T            dP = dO U^T (lower incl.)
//   dV = diag(b) T^T dU                    dT = dU (diag(b) V)^T + dW (diag(b gam) K)^T
//   dA = -T^T dT T^T (strictly lower)      D = diag(b) dA o Gam    D2 = dP o Gam
//   dQ = diag(gam) dO S^T + D2 K
//   dK = (D + D^T) K + D2^T Q + diag(b gam) T^T dW + diag(lam) U dS'^T
//   dbeta = rows of (dA o Gam o KK^T) + rows of (T^T dU o V) + gam rows of (T^T dW o K)
//   d gam (O1, W), d lam, d gam_C, d Gam (A, P) -> dG -> dlog_alpha by segmented suffix sums.
template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_grads(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta, const TIn *__restrict__ dout,
              const float *__restrict__ Sc, const float *__restrict__ dSn, const int32_t *__restrict__ cu,
              const int32_t *__restrict__ off, int nseq, int T, int H, float *__restrict__ dq,
              float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dla, float *__restrict__ dbe)
{
    extern __shared__ float smf[];
    float *K = smf, *Q = K + MAT, *V = Q + MAT, *dO = V + MAT, *S = dO + MAT, *dSp = S + MAT, *KK = dSp + MAT,
          *Tm = KK + MAT, *X1 = Tm + MAT, *U = X1 + MAT, *QK = U + MAT, *dU = QK + MAT, *X2 = dU + MAT;
    Gates &g = *reinterpret_cast<Gates *>(X2 + MAT);
    float *vec = reinterpret_cast<float *>(&g + 1);
    float *bg = vec, *dG = vec + N, *dgam = vec + 2 * N, *dlam = vec + 3 * N, *dbet = vec + 4 * N, *dgC = vec + 5 * N;
    const int t = threadIdx.x, h = blockIdx.y, e = blockIdx.x;
    const ChunkRef c = chunk_ref(e, cu, off, nseq, T);
    if (c.n == 0) return;
    const size_t base = ((size_t)e * H + h) * (size_t)(N * N);
    load_rows(K, k, c, H, h, t);
    load_rows(Q, q, c, H, h, t);
    load_rows(V, v, c, H, h, t);
    load_rows(dO, dout, c, H, h, t);
    for (int i = t; i < N * N; i += kThreads) {
        S[(i >> 6) * LD + (i & 63)] = Sc[base + i];
        dSp[(i >> 6) * LD + (i & 63)] = dSn[base + i];
    }
    vec[N + t] = 0.f;  // dG, dgam, dlam, dbet
    if (t == 0) dgC[0] = 0.f;
    chunk_gates<TIn>(g, log_alpha, beta, c, H, h, t);
    __syncthreads();
    if (t < N) bg[t] = g.bet[t] * g.gam[t];
    float aq[16], ak[16], av[16];  // this thread's 4 x 4 blocks of dQ, dK, dV
#pragma unroll
    for (int i = 0; i < 16; ++i) aq[i] = ak[i] = av[i] = 0.f;
    int id;
    mm<false, true>(K, K, t, [&](int r, int i, float x) { KK[r * LD + i] = x; });
    mm<false, true>(Q, K, t, [&](int r, int i, float x) { QK[r * LD + i] = x; });
    mm<false, false>(K, dSp, t, [&](int i, int m, float x) { X2[i * LD + m] = x; });  // K dS'
    __syncthreads();
    // A (strictly lower) in dU for the solve; P in X1; d gam_C = <S, dS'>
    {
        float part = 0.f;
        for (int idx = t; idx < N * N; idx += kThreads) {
            const int r = idx >> 6, i = idx & 63;
            const float gm = decay(g, r, i);
            dU[r * LD + i] = i < r ? g.bet[r] * gm * KK[r * LD + i] : 0.f;
            X1[r * LD + i] = gm * QK[r * LD + i];
            part = fmaf(S[r * LD + i], dSp[r * LD + i], part);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((t & 31) == 0) atomicAdd(dgC, part);
    }
    __syncthreads();
    unit_lower_inverse(dU, Tm, t);
    __syncthreads();
    // U~ into U, W into dU (A is no longer needed)
    mm<false, false>(Tm, V, t, [&](int r, int j, float x) { U[r * LD + j] = x; }, g.bet);
    mm<false, false>(Tm, K, t, [&](int r, int m, float x) { dU[r * LD + m] = x; }, bg);
    __syncthreads();
    // U = U~ - W S
    mm<false, false>(dU, S, t, [&](int r, int j, float x) { U[r * LD + j] -= x; });
    __syncthreads();
    // dU = P^T dO + diag(lam) K dS'; d lam_i = sum_j (K dS')_ij U_ij
    mm<true, false>(X1, dO, t, [&](int i, int j, float x) {
        dU[i * LD + j] = x + g.lam[i] * X2[i * LD + j];
        atomicAdd(&dlam[i], X2[i * LD + j] * U[i * LD + j]);
    });
    __syncthreads();
    // dP = dO U^T (lower incl.) over P; dK += diag(lam) U dS'^T; d gam (O1) and dQ += diag(gam) dO S^T
    mm<false, true>(dO, U, t, [&](int r, int i, float x) { X1[r * LD + i] = i <= r ? x : 0.f; });
    id = 0;
    mm<false, true>(U, dSp, t, [&](int i, int m, float x) { ak[id++] += g.lam[i] * x; });
    id = 0;
    mm<false, true>(dO, S, t, [&](int r, int m, float x) { aq[id++] += g.gam[r] * x; });
    mm<false, false>(Q, S, t, [&](int r, int j, float x) { atomicAdd(&dgam[r], dO[r * LD + j] * x); });
    __syncthreads();
    // dW = -dU S^T into U (U is no longer needed)
    mm<false, true>(dU, S, t, [&](int r, int m, float x) { U[r * LD + m] = -x; });
    __syncthreads();
    // Y = T^T dU: dV, dbeta;  X = T^T dW: dK, dbeta, d gam
    id = 0;
    mm<true, false>(Tm, dU, t, [&](int i, int j, float x) {
        av[id++] += g.bet[i] * x;
        atomicAdd(&dbet[i], x * V[i * LD + j]);
    });
    id = 0;
    mm<true, false>(Tm, U, t, [&](int i, int m, float x) {
        ak[id++] += bg[i] * x;
        const float xk = x * K[i * LD + m];
        atomicAdd(&dbet[i], g.gam[i] * xk);
        atomicAdd(&dgam[i], g.bet[i] * xk);
    });
    // dT = dU (diag(b) V)^T + dW (diag(b gam) K)^T into X2 (K dS' is no longer needed); the
    // diagonals scale the result's column index
    mm<false, true>(dU, V, t, [&](int r, int i, float x) { X2[r * LD + i] = g.bet[i] * x; });
    mm<false, true>(U, K, t, [&](int r, int i, float x) { X2[r * LD + i] += bg[i] * x; });
    __syncthreads();
    // Z = dT T^T into dU
    mm<false, true>(X2, Tm, t, [&](int r, int i, float x) { dU[r * LD + i] = x; });
    __syncthreads();
    // dA = -T^T Z (strictly lower) -> D into U; dbeta (A); dG from Gam (A)
    mm<true, false>(Tm, dU, t, [&](int r, int i, float x) {
        float d = 0.f;
        if (i < r) {
            const float dA = -x, gm = decay(g, r, i);
            const float dAbar = g.bet[r] * dA;
            d = dAbar * gm;
            atomicAdd(&dbet[r], dA * gm * KK[r * LD + i]);
            const float E = dAbar * KK[r * LD + i] * gm;
            atomicAdd(&dG[r], E);
            atomicAdd(&dG[i], -E);
        }
        U[r * LD + i] = d;
    });
    // D2 = dP o Gam in X1; dG from Gam (P)
    for (int idx = t; idx < N * N; idx += kThreads) {
        const int r = idx >> 6, i = idx & 63;
        const float gm = decay(g, r, i), dp = X1[r * LD + i];
        X1[r * LD + i] = dp * gm;
        const float E = dp * QK[r * LD + i] * gm;
        if (E != 0.f) {
            atomicAdd(&dG[r], E);
            atomicAdd(&dG[i], -E);
        }
    }
    __syncthreads();
    // dK += D K + D^T K + D2^T Q;  dQ += D2 K
    id = 0;
    mm<false, false>(U, K, t, [&](int r, int m, float x) { ak[id++] += x; });
    id = 0;
    mm<true, false>(U, K, t, [&](int i, int m, float x) { ak[id++] += x; });
    id = 0;
    mm<true, false>(X1, Q, t, [&](int i, int m, float x) { ak[id++] += x; });
    id = 0;
    mm<false, false>(X1, K, t, [&](int r, int m, float x) { aq[id++] += x; });
    __syncthreads();
    // gate gradients: gam_r = exp(G_r), lam_i = exp(G_63 - G_i), gam_C = gam_63; then dlog_alpha_j =
    // sum of dG_r over the rows r >= j of j's reset segment (0 at a reset itself)
    if (t == 0) {
        for (int r = 0; r < N; ++r) dG[r] += dgam[r] * g.gam[r];
        float s63 = dgC[0] * g.gam[N - 1];
        for (int i = 0; i < N; ++i) {
            const float li = dlam[i] * g.lam[i];
            s63 += li;
            dG[i] -= li;
        }
        dG[N - 1] += s63;
        float acc = 0.f;
        for (int j = N - 1; j >= 0; --j) {
            acc += dG[j];
            const bool reset = g.last[j] == j;
            dlam[j] = reset ? 0.f : acc;  // reuse as dlog_alpha
            if (reset) acc = 0.f;
        }
    }
    __syncthreads();
    const int r0 = (t >> 4) * 4, c0 = (t & 15) * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + i;
        if (r >= c.n) continue;
        const size_t row = ((size_t)(c.tok + r) * H + h) * N + c0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            dq[row + j] = aq[i * 4 + j];
            dk[row + j] = ak[i * 4 + j];
            dv[row + j] = av[i * 4 + j];
        }
    }
    if (t < c.n) {
        const size_t o = (size_t)(c.tok + t) * H + h;
        dla[o] = dlam[t];
        dbe[o] = dbet[t];
    }
}

// chunk offsets of varlen sequences: off[s] = sum over s' < s of ceil(len / 64); off[nseq] = total
__global__ void bwd_offsets(const int32_t *__restrict__ cu, int nseq, int32_t *__restrict__ off)
{
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        int acc = 0;
        for (int s = 0; s < nseq; ++s) {
            off[s] = acc;
            acc += (cu[s + 1] - cu[s] + N - 1) / N;
        }
        off[nseq] = acc;
    }
}

}  // namespace

// ---- host side -------------------------------------------------------------------------------

namespace {

size_t align256b(size_t x) { return (x + 255) & ~(size_t)255; }

// Upper bound on the chunk count (varlen: every sequence adds at most one partial chunk).
long bwd_chunks(int B, int T, int varlen)
{
    return varlen ? (long)(T + N - 1) / N + B : (long)B * ((T + N - 1) / N);
}

template <typename TIn>
cudaError_t run_bwd(const BwdArgs &a, cudaStream_t st)
{
    const int varlen = a.cu_seqlens != nullptr;
    const long chunks = bwd_chunks(a.B, a.T, varlen);
    const size_t mats = (size_t)chunks * a.H * N * N * sizeof(float);
    char *w = static_cast<char *>(a.workspace);
    int32_t *off = reinterpret_cast<int32_t *>(w);
    w += align256b((size_t)(a.B + 1) * sizeof(int32_t));
    float *Mo = reinterpret_cast<float *>(w);
    float *Bo = reinterpret_cast<float *>(w + align256b(mats));
    float *Ro = reinterpret_cast<float *>(w + 2 * align256b(mats));
    float *Sc = reinterpret_cast<float *>(w + 3 * align256b(mats));
    float *dSn = reinterpret_cast<float *>(w + 4 * align256b(mats));
    const int32_t *offp = varlen ? off : nullptr;
    if (varlen) {
        bwd_offsets<<<1, 1, 0, st>>>(a.cu_seqlens, a.B, off);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const TIn *q = static_cast<const TIn *>(a.q), *k = static_cast<const TIn *>(a.k),
              *v = static_cast<const TIn *>(a.v), *dout = static_cast<const TIn *>(a.dout);
    const int smem_prep = (9 * MAT) * (int)sizeof(float) + (int)sizeof(Gates) + N * (int)sizeof(float);
    const int smem_grads = (13 * MAT) * (int)sizeof(float) + (int)sizeof(Gates) + 6 * N * (int)sizeof(float);
    const int smem_scan = 2 * MAT * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_prep<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_grads<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_grads);
    if (e != cudaSuccess) return e;
    const dim3 gc((unsigned)chunks, a.H), gs(a.H, a.B);
    bwd_prep<TIn><<<gc, kThreads, smem_prep, st>>>(q, k, v, a.log_alpha, a.beta, dout, a.cu_seqlens, offp, a.B, a.T,
                                                   a.H, Mo, Bo, Ro);
    bwd_fscan<<<gs, kThreads, smem_scan, st>>>(Mo, Bo, a.S0, a.cu_seqlens, offp, a.T, a.H, Sc);
    bwd_bscan<<<gs, kThreads, smem_scan, st>>>(Mo, Ro, a.dS_final, a.cu_seqlens, offp, a.T, a.H, dSn, a.dS0);
    bwd_grads<TIn><<<gc, kThreads, smem_grads, st>>>(q, k, v, a.log_alpha, a.beta, dout, Sc, dSn, a.cu_seqlens, offp,
                                                     a.B, a.T, a.H, a.dq, a.dk, a.dv, a.dlog_alpha, a.dbeta);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int varlen)
{
    const size_t mats = (size_t)bwd_chunks(B, T, varlen) * H * N * N * sizeof(float);
    return align256b((size_t)(B + 1) * sizeof(int32_t)) + 5 * align256b(mats);
}

cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t stream)
{
    return a.dtype == GDN_DTYPE_BF16 ? run_bwd<__nv_bfloat16>(a, stream) : run_bwd<float>(a, stream);
}

}  // namespace gdn
