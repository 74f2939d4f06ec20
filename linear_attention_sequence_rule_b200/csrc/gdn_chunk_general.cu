// gdn_chunk_general.cu -- the chunkwise (WY / UT-transform) forward for shapes outside the fused
// tensor-core kernel's on-chip plan: key head size 256 and chunk length 128 (any of dk in
// {64, 128, 256}, dv in {64, 128, 256}, C in {64, 128}), fp32 arithmetic on CUDA cores.
//
// Sources: Sykra README, "Architectural Highlights" (chunk-parallel training through the WY /
// unit triangular transform; `chunk_size` of SykraConfig) and DeltaPhase README, section 1
// ("Fast Triangular Solve"; head size 256 in section 5).  Per chunk of C tokens entered with
// state S (dk x dv):
//   A  = strictly_lower(diag(b) (Gam o K K^T)),   T = (I + A)^{-1}
//   W  = T diag(b gam) K,   U~ = T diag(b) V,   P = lower_incl(Gam o Q K^T)
//   U  = U~ - W S,   O = diag(gam) Q S + P U,   S' = gam_C S + K^T diag(lam) U
// The fused kernel keeps every per-chunk factor on chip next to a state held in TMEM; at
// dk = 256 the fp32 state alone takes half of TMEM and the K/Q tiles of a stage 64 KB, and a
// chunk of 128 doubles every C x C factor, so neither fits its plan.  Here the work is split in
// two launches with the chunk factors passing through a workspace:
//   gen_prep_kernel  -- one CTA per (chunk, value head), all chunks at once: gate sums, the two
//                       Gram matrices, A, P, the triangular inverse T, then W and U~ (dk and dv
//                       in 64-column tiles); writes W, U~, P and the decay vectors.
//   gen_chain_kernel -- one CTA per (sequence, value head, 64 value columns), chunk after
//                       chunk: U, the outputs and the state update, with the 64 x dk block of S
//                       in shared memory.
// A table kernel first lists every chunk as (sequence, first token, length); chunks never cross
// a sequence start and the last one of a sequence may be partial.  Gates follow the fused
// kernel's rules: sums of log_alpha since the last exact reset (log_alpha = -inf), padded rows
// with b = 0 and log_alpha = 0.
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int TILE = 64;  // key / value columns per tile

__device__ __forceinline__ float ldf(const float *p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float *p, float x) { *p = x; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct GenWork {
    int32_t *table;      // [max_chunks][3]: sequence, first token, length (0: unused entry)
    int32_t *first;      // [nseq + 1]: first chunk of each sequence
    float *W, *U, *P;    // per (chunk, head): C x dk, C x dv, C x C
    float *gam, *lam;    // per (chunk, head): C each
    size_t bytes;
};

GenWork gen_layout(void *base, long max_chunks, int nseq, int H, int dk, int dv, int C)
{
    GenWork w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += al256(b);
        return o;
    };
    const size_t ch = (size_t)max_chunks * H;
    const size_t o_t = take((size_t)max_chunks * 3 * sizeof(int32_t));
    const size_t o_f = take((size_t)(nseq + 1) * sizeof(int32_t));
    const size_t o_w = take(ch * C * dk * sizeof(float));
    const size_t o_u = take(ch * C * dv * sizeof(float));
    const size_t o_p = take(ch * C * C * sizeof(float));
    const size_t o_g = take(ch * C * sizeof(float));
    const size_t o_l = take(ch * C * sizeof(float));
    w.bytes = off;
    if (base) {
        char *b = static_cast<char *>(base);
        w.table = reinterpret_cast<int32_t *>(b + o_t);
        w.first = reinterpret_cast<int32_t *>(b + o_f);
        w.W = reinterpret_cast<float *>(b + o_w);
        w.U = reinterpret_cast<float *>(b + o_u);
        w.P = reinterpret_cast<float *>(b + o_p);
        w.gam = reinterpret_cast<float *>(b + o_g);
        w.lam = reinterpret_cast<float *>(b + o_l);
    }
    return w;
}

long gen_max_chunks(int B, int T, int C, bool varlen)
{
    return varlen ? (long)T / C + B : (long)B * ((T + C - 1) / C);
}

// The chunk table, one CTA: each thread counts the chunks of a contiguous range of sequences, a
// block scan gives every range its first chunk, then each thread writes its entries; entries
// past the last chunk are marked empty.
__global__ void __launch_bounds__(1024) gen_table_kernel(const int32_t *__restrict__ cu, int nseq, int T, int C,
                                                         long max_chunks, int32_t *__restrict__ table,
                                                         int32_t *__restrict__ first)
{
    __shared__ long part[1024];
    const int t = threadIdx.x;
    const int per = (nseq + 1023) / 1024;
    const int s0 = min(nseq, t * per), s1 = min(nseq, s0 + per);
    auto bounds = [&](int s, long &a, long &n) {
        if (cu) {
            a = cu[s];
            n = (long)cu[s + 1] - a;
        } else {
            a = (long)s * T;
            n = T;
        }
    };
    long cnt = 0;
    for (int s = s0; s < s1; ++s) {
        long a, n;
        bounds(s, a, n);
        cnt += (n + C - 1) / C;
    }
    part[t] = cnt;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan
        const long x = t >= o ? part[t - o] : 0;
        __syncthreads();
        part[t] += x;
        __syncthreads();
    }
    long off = part[t] - cnt;
    for (int s = s0; s < s1; ++s) {
        long a, n;
        bounds(s, a, n);
        first[s] = (int32_t)off;
        for (long c = 0; c * C < n; ++c, ++off) {
            table[3 * off + 0] = s;
            table[3 * off + 1] = (int32_t)(a + c * C);
            table[3 * off + 2] = (int32_t)min((long)C, n - c * C);
        }
    }
    const long total = part[1023];
    if (t == 0) first[nseq] = (int32_t)total;
    for (long e = total + t; e < max_chunks; e += 1024) table[3 * e + 2] = 0;
}

// Gate vectors of one chunk (thread 0, sequential over the C rows): G[r] = sum of log_alpha since
// the last exact reset at or before r (0 at a reset), last[r] = that reset's row or -1.
__device__ void gate_sums(const float *graw, float *G, int *last, int C)
{
    float g = 0.f;
    int l = -1;
    for (int r = 0; r < C; ++r) {
        const float x = graw[r];
        if (x == -INFINITY) {
            g = 0.f;
            l = r;
        } else {
            g += x;
        }
        G[r] = g;
        last[r] = l;
    }
}

__device__ __forceinline__ float decay(const float *G, const int *last, int r, int i)
{
    return (i <= r && last[r] <= i) ? expf(G[r] - G[i]) : 0.f;
}

// Prep: one CTA per (chunk cid, value head h).  Shared memory (fp32, row stride +1 against bank
// conflicts): A and then T's workspace, T, two C x TILE tiles, and the gate vectors.
template <int C, typename TIn>
__global__ void __launch_bounds__(kThreads)
    gen_prep_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                    const float *__restrict__ log_alpha, const float *__restrict__ beta, GenWork w, int H, int G,
                    int dk, int dv)
{
    extern __shared__ __align__(16) float shf[];
    float *A = shf;                      // [C][C + 1]: Gram K K^T, then A
    float *Pm = A + C * (C + 1);         // [C][C + 1]: Gram Q K^T, then P, then T
    float *X = Pm + C * (C + 1);         // [C][TILE + 1]: K tile (or V tile)
    float *Y = X + C * (TILE + 1);       // [C][TILE + 1]: Q tile
    float *Gs = Y + C * (TILE + 1);      // [C] each: Gs, gam, lam, bet, graw, last
    float *gam = Gs + C, *lam = gam + C, *bet = lam + C, *graw = bet + C;
    int *last = reinterpret_cast<int *>(graw + C);
    const long cid = blockIdx.x;
    const int h = blockIdx.y, hq = h / G, Hk = H / G, tid = threadIdx.x;
    const int n = w.table[3 * cid + 2];
    if (n == 0) return;
    const long tok0 = w.table[3 * cid + 1];
    const size_t ch = (size_t)cid * H + h;

    for (int r = tid; r < C; r += kThreads) {
        const bool ok = r < n;
        graw[r] = ok ? log_alpha[(size_t)(tok0 + r) * H + h] : 0.f;
        bet[r] = ok ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
    }
    for (int i = tid; i < C * (C + 1); i += kThreads) {
        A[i] = 0.f;
        Pm[i] = 0.f;
    }
    __syncthreads();
    if (tid == 0) gate_sums(graw, Gs, last, C);
    // ---- Gram matrices over key tiles: A = K K^T, Pm = Q K^T (lower triangles) ----
    for (int f0 = 0; f0 < dk; f0 += TILE) {
        __syncthreads();
        for (int i = tid; i < C * TILE; i += kThreads) {
            const int r = i / TILE, f = i % TILE;
            const bool ok = r < n;
            const size_t off = ((size_t)(tok0 + r) * Hk + hq) * dk + f0 + f;
            X[r * (TILE + 1) + f] = ok ? ldf(k + off) : 0.f;
            Y[r * (TILE + 1) + f] = ok ? ldf(q + off) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * C; e += kThreads) {
            const int r = e / C, i = e % C;
            if (i > r) continue;
            float a = 0.f, p = 0.f;
            const float *kr = X + r * (TILE + 1), *ki = X + i * (TILE + 1), *qr = Y + r * (TILE + 1);
#pragma unroll 8
            for (int f = 0; f < TILE; ++f) {
                a = fmaf(kr[f], ki[f], a);
                p = fmaf(qr[f], ki[f], p);
            }
            A[r * (C + 1) + i] += a;
            Pm[r * (C + 1) + i] += p;
        }
    }
    __syncthreads();
    // ---- decays: A = diag(b)(Gam o K K^T) strictly lower, P = Gam o Q K^T lower inclusive ----
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, i = e % C;
        const float d = decay(Gs, last, r, i);
        A[r * (C + 1) + i] = i < r ? bet[r] * d * A[r * (C + 1) + i] : 0.f;
        const float p = i <= r ? d * Pm[r * (C + 1) + i] : 0.f;
        w.P[ch * C * C + (size_t)r * C + i] = p;
    }
    for (int r = tid; r < C; r += kThreads) {
        gam[r] = last[r] >= 0 ? 0.f : expf(Gs[r]);
        lam[r] = decay(Gs, last, C - 1, r);
        w.gam[ch * C + r] = gam[r];
        w.lam[ch * C + r] = lam[r];
    }
    __syncthreads();
    // ---- T = (I + A)^{-1} into Pm, column j by thread j (forward substitution) ----
    float *Tm = Pm;
    for (int j = tid; j < C; j += kThreads) {
        for (int r = 0; r < C; ++r) {
            float x = 0.f;
            if (r == j) {
                x = 1.f;
            } else if (r > j) {
                for (int i = j; i < r; ++i) x = fmaf(-A[r * (C + 1) + i], Tm[i * (C + 1) + j], x);
            }
            Tm[r * (C + 1) + j] = x;
        }
    }
    __syncthreads();
    // ---- W = T diag(b gam) K over key tiles ----
    for (int f0 = 0; f0 < dk; f0 += TILE) {
        for (int i = tid; i < C * TILE; i += kThreads) {
            const int r = i / TILE, f = i % TILE;
            const size_t off = ((size_t)(tok0 + r) * Hk + hq) * dk + f0 + f;
            X[r * (TILE + 1) + f] = r < n ? bet[r] * gam[r] * ldf(k + off) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * TILE; e += kThreads) {
            const int r = e / TILE, f = e % TILE;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * (C + 1) + i], X[i * (TILE + 1) + f], acc);
            w.W[(ch * C + r) * dk + f0 + f] = acc;
        }
        __syncthreads();
    }
    // ---- U~ = T diag(b) V over value tiles ----
    for (int c0 = 0; c0 < dv; c0 += TILE) {
        for (int i = tid; i < C * TILE; i += kThreads) {
            const int r = i / TILE, c = i % TILE;
            X[r * (TILE + 1) + c] = r < n ? bet[r] * ldf(v + ((size_t)(tok0 + r) * H + h) * dv + c0 + c) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * TILE; e += kThreads) {
            const int r = e / TILE, c = e % TILE;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * (C + 1) + i], X[i * (TILE + 1) + c], acc);
            w.U[(ch * C + r) * dv + c0 + c] = acc;
        }
        __syncthreads();
    }
}

// Chain: one CTA per (64 value columns, value head, sequence), chunk after chunk.  S holds the
// block's dk x 64 state (fp32); per chunk, over key tiles: U = U~ - W S, then O = diag(gam) Q S
// + P U and S <- gam_C S + (diag(lam) K)^T U.
template <int C, typename TIn>
__global__ void __launch_bounds__(kThreads)
    gen_chain_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const float *__restrict__ S0,
                     TIn *__restrict__ out, float *__restrict__ S_final, GenWork w, int H, int G, int dk, int dv)
{
    extern __shared__ __align__(16) float shf[];
    constexpr int LD = TILE + 1;
    float *S = shf;                 // [dk][LD]
    float *X = S + dk * LD;         // [C][LD]: W, Q, K or P tile
    float *Us = X + C * LD;         // [C][LD]: U of the chunk
    float *Os = Us + C * LD;        // [C][LD]: output accumulator
    const int vb = blockIdx.x, h = blockIdx.y, s = blockIdx.z, tid = threadIdx.x;
    const int hq = h / G, Hk = H / G;
    const int c0 = vb * TILE;
    const size_t sbase = ((size_t)s * H + h) * (size_t)dk * dv + c0;
    for (int i = tid; i < dk * TILE; i += kThreads) {
        const int f = i / TILE, j = i % TILE;
        S[f * LD + j] = S0 ? S0[sbase + (size_t)f * dv + j] : 0.f;
    }
    const int cid0 = w.first[s], cid1 = w.first[s + 1];
    for (int cid = cid0; cid < cid1; ++cid) {
        const int n = w.table[3 * cid + 2];
        const long tok0 = w.table[3 * cid + 1];
        const size_t ch = (size_t)cid * H + h;
        const float *gam = w.gam + ch * C, *lam = w.lam + ch * C;
        __syncthreads();
        // Us = U~ (this block's columns), Os = 0
        for (int i = tid; i < C * TILE; i += kThreads) {
            const int r = i / TILE, j = i % TILE;
            Us[r * LD + j] = w.U[(ch * C + r) * dv + c0 + j];
            Os[r * LD + j] = 0.f;
        }
        // over key tiles: Us -= W S, Os += Q S
        for (int f0 = 0; f0 < dk; f0 += TILE) {
            __syncthreads();
            for (int i = tid; i < C * TILE; i += kThreads) {
                const int r = i / TILE, f = i % TILE;
                X[r * LD + f] = w.W[(ch * C + r) * dk + f0 + f];
            }
            __syncthreads();
            for (int e = tid; e < C * TILE; e += kThreads) {
                const int r = e / TILE, j = e % TILE;
                float acc = 0.f;
#pragma unroll 8
                for (int f = 0; f < TILE; ++f) acc = fmaf(X[r * LD + f], S[(f0 + f) * LD + j], acc);
                Us[r * LD + j] -= acc;
            }
            __syncthreads();
            for (int i = tid; i < C * TILE; i += kThreads) {
                const int r = i / TILE, f = i % TILE;
                X[r * LD + f] = r < n ? ldf(q + ((size_t)(tok0 + r) * Hk + hq) * dk + f0 + f) : 0.f;
            }
            __syncthreads();
            for (int e = tid; e < C * TILE; e += kThreads) {
                const int r = e / TILE, j = e % TILE;
                float acc = 0.f;
#pragma unroll 8
                for (int f = 0; f < TILE; ++f) acc = fmaf(X[r * LD + f], S[(f0 + f) * LD + j], acc);
                Os[r * LD + j] += acc;
            }
        }
        __syncthreads();
        // Os = diag(gam) Os + P U (P in C x TILE column tiles)
        for (int e = tid; e < C * TILE; e += kThreads) {
            const int r = e / TILE, j = e % TILE;
            Os[r * LD + j] *= gam[r];
        }
        for (int i0 = 0; i0 < C; i0 += TILE) {
            __syncthreads();
            for (int i = tid; i < C * TILE; i += kThreads) {
                const int r = i / TILE, c = i % TILE;
                X[r * LD + c] = w.P[ch * C * C + (size_t)r * C + i0 + c];
            }
            __syncthreads();
            for (int e = tid; e < C * TILE; e += kThreads) {
                const int r = e / TILE, j = e % TILE;
                float acc = 0.f;
#pragma unroll 8
                for (int c = 0; c < TILE; ++c) acc = fmaf(X[r * LD + c], Us[(i0 + c) * LD + j], acc);
                Os[r * LD + j] += acc;
            }
        }
        __syncthreads();
        for (int e = tid; e < n * TILE; e += kThreads) {
            const int r = e / TILE, j = e % TILE;
            stf(out + ((size_t)(tok0 + r) * H + h) * dv + c0 + j, Os[r * LD + j]);
        }
        // S <- gam_C S + (diag(lam) K)^T U over key tiles
        const float gC = gam[C - 1];
        for (int f0 = 0; f0 < dk; f0 += TILE) {
            __syncthreads();
            for (int i = tid; i < C * TILE; i += kThreads) {
                const int r = i / TILE, f = i % TILE;
                X[r * LD + f] = r < n ? lam[r] * ldf(k + ((size_t)(tok0 + r) * Hk + hq) * dk + f0 + f) : 0.f;
            }
            __syncthreads();
            for (int e = tid; e < TILE * TILE; e += kThreads) {
                const int f = e / TILE, j = e % TILE;
                float acc = 0.f;
#pragma unroll 8
                for (int r = 0; r < C; ++r) acc = fmaf(X[r * LD + f], Us[r * LD + j], acc);
                S[(f0 + f) * LD + j] = fmaf(gC, S[(f0 + f) * LD + j], acc);
            }
        }
    }
    __syncthreads();
    if (S_final) {
        for (int i = tid; i < dk * TILE; i += kThreads) {
            const int f = i / TILE, j = i % TILE;
            S_final[sbase + (size_t)f * dv + j] = S[f * LD + j];
        }
    }
}

template <int C, typename TIn>
cudaError_t run_general(const ChunkArgs &a, int C_, cudaStream_t st)
{
    (void)C_;
    const bool varlen = a.cu_seqlens != nullptr;
    const long mc = gen_max_chunks(a.B, a.T, C, varlen);
    GenWork w = gen_layout(a.workspace, mc, a.B, a.H, a.dk, a.dv, C);
    gen_table_kernel<<<1, 1024, 0, st>>>(a.cu_seqlens, a.B, a.T, C, mc, w.table, w.first);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t prep_smem = (size_t)(2 * C * (C + 1) + 2 * C * (TILE + 1) + 6 * C) * sizeof(float);
    e = cudaFuncSetAttribute(gen_prep_kernel<C, TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
    if (e != cudaSuccess) return e;
    if (mc > 0) {
        gen_prep_kernel<C, TIn><<<dim3((unsigned)mc, a.H), kThreads, prep_smem, st>>>(
            static_cast<const TIn *>(a.q), static_cast<const TIn *>(a.k), static_cast<const TIn *>(a.v), a.log_alpha,
            a.beta, w, a.H, a.G, a.dk, a.dv);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const size_t chain_smem = (size_t)(a.dk * (TILE + 1) + 3 * C * (TILE + 1)) * sizeof(float);
    e = cudaFuncSetAttribute(gen_chain_kernel<C, TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain_smem);
    if (e != cudaSuccess) return e;
    gen_chain_kernel<C, TIn><<<dim3(a.dv / TILE, a.H, a.B), kThreads, chain_smem, st>>>(
        static_cast<const TIn *>(a.q), static_cast<const TIn *>(a.k), a.S0, static_cast<TIn *>(a.out), a.S_final, w,
        a.H, a.G, a.dk, a.dv);
    return cudaGetLastError();
}

}  // namespace

bool chunk_general_needed(int dk, int dv, int chunk)
{
    return chunk == 128 || dk == 256;
}

size_t chunk_general_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen)
{
    return gen_layout(nullptr, gen_max_chunks(B, T, chunk, varlen != 0), B, H, dk, dv, chunk).bytes;
}

cudaError_t launch_chunk_general(const ChunkArgs &a, int chunk, cudaStream_t stream)
{
    const bool bf = a.dtype == GDN_DTYPE_BF16;
    if (chunk == 128)
        return bf ? run_general<128, __nv_bfloat16>(a, chunk, stream) : run_general<128, float>(a, chunk, stream);
    return bf ? run_general<64, __nv_bfloat16>(a, chunk, stream) : run_general<64, float>(a, chunk, stream);
}

}  // namespace gdn
