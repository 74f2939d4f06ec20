// gdn_chunk_bwd.cu -- gradients of the chunk forward (dq, dk, dv, dlog_alpha, dbeta, dS0) with
// fp32-level accuracy, for dk = 64 and dv = 64 VS, VS in {1, 2, 4} (the training path; Sykra
// README, "Architectural Highlights": chunk-parallel training through the WY / UT transform).
// The 64 x 64 products run on the tensor cores as three tf32 products each; the rest is fp32 on
// the CUDA cores.
//
// Per chunk of C = 64 tokens with entry state S (the forward's chunk form):
//   A = strictly_lower(diag(b) (Gam o K K^T)),  T = (I + A)^{-1}
//   W = T diag(b gam) K,  U~ = T diag(b) V,  U = U~ - W S,  P = lower_incl(Gam o Q K^T)
//   O = diag(gam) Q S + P U,   S' = gam_C S + K^T diag(lam) U
// so the chunk maps states and state gradients affinely:
//   S'  = M S + Bm,              M  = gam_C I - K^T diag(lam) W,   Bm = K^T diag(lam) U~
//   dS  = M^T dS' + R,           R  = (Q^T diag(gam) - W^T P^T) dO
// Three kernels (plus the varlen chunk offsets and, when gradients are partial, their sums):
//   bwd_prep   (chunk x head, parallel)  : T, W, U~, P  ->  M, Bm, R, and T, W, U~ for bwd_grads
//   bwd_scans  (sequence x head x 2)     : forward, S_c for every chunk from S0; reverse, dS at every
//                                          chunk's end from dS_final, and dS0 (one launch, both at once)
//   bwd_grads  (chunk x head, parallel)  : with S_c and dS_{c+1}, every input gradient of the chunk
// All matrices are 64 x 64 fp32 in shared memory (XOR-swizzled rows); 256 threads; a product
// leaves each thread 16 results in the tensor cores' fragment layout (see mm_core).
// Value splits: the recurrence never mixes value columns (column j of S, O and dS follows from
// column j of V, S0 and dO alone), so a value head of 64 VS columns runs as VS virtual heads of 64
// columns, hx = h VS + block, that share q, k and the gates.  Their dv and dS0 are disjoint column
// blocks of the outputs; their dq, dk, dbeta and dlog_alpha are partial sums, added up at the end
// (with the grouped-value-head sums when value heads also share q/k heads).
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

constexpr int N = 64;          // chunk length = dk = dv
constexpr int MAT = N * N;     // floats per matrix
constexpr int kThreads = 256;               // 8 warps (16 measured slower: 4.5 against 4.1 ms)
constexpr int kColBlocks = kThreads / 128;  // a product's warps: 4 row blocks of 16 x this many column blocks
constexpr int kNT = N / (8 * kColBlocks);   // 8-column MMA tiles per warp
constexpr int kFrag = 4 * kNT;              // results per thread of a product
constexpr int kColSlots = 2 * kNT;          // distinct columns among them
constexpr int kSolveLanes = kThreads / N;   // threads per column in the triangular solve
constexpr int kSolveRows = N / kSolveLanes; // rows per thread there
static_assert(kNT >= 1 && 8 * kNT * kColBlocks == N && kSolveLanes * N == kThreads, "thread layout");

// Shared matrices are 64 x 64 fp32 with 64-float rows; column c of row r is stored at position
// c ^ 4 sigma(r mod 8), sigma = (0 2 4 6 1 3 5 7), which moves whole 16-byte groups.  Both access
// patterns of the tensor-core fragments -- 8 rows x 4 columns and 4 rows x 8 columns -- then fall
// on 32 different banks, and so do whole rows.  Element (r, c) lives at sw(r, c).
__device__ __forceinline__ int sw(int r, int c)
{
    return r * N + (c ^ (((r & 3) << 3) | (((r >> 2) & 1) << 2)));
}

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

// fp32 x fp32 on the tensor cores: x = hi + lo with hi, lo tf32 (11 significant bits each), and
// a b ~ hi_a hi_b + hi_a lo_b + lo_a hi_b (the dropped lo_a lo_b is below 2^-22 |a b|).
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo)
{
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(x - __uint_as_float(hi)));
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The dynamic shared memory of every kernel in this file.
extern __shared__ __align__(16) float smf[];

// One thread's 16 results of a product, index u (see mm).
struct Frag {
    float v[kFrag];
};

// C(r, c) = sum_k opA(r, k) ks[k] opB(k, c) for 64 x 64 operands (opA = A or A^T, opB = B or B^T;
// ks: optional diagonal), on the tensor cores with the three-term tf32 split.  Warp w computes
// rows 16 (w mod 4) .. +15 and the W = 8 kNT columns from W (w / 4); lane l holds rows
// 16 (w mod 4) + l / 4 + {0, 8} and columns W (w / 4) + 8 n + 2 (l mod 4) + {0, 1}, n < kNT, as
// element u = 4 n + 2 (row half) + (column parity) of its Frag -- the same u for the same (r, c)
// in every product, so per-thread accumulators can be indexed by it.  The operands are given as offsets
// into the shared memory.  Kept out of line: a kernel runs this loop some twenty times, and one
// shared copy of it stays in the instruction cache.
template <bool TA, bool TB, bool KS>
__device__ __noinline__ Frag mm_core(int a_off, int b_off, int ks_off)
{
    const float *A = smf + a_off, *B = smf + b_off, *ks = smf + ks_off;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5, g = lane >> 2, q = lane & 3;
    const int m0 = (w & 3) * 16, n0 = (w >> 2) * 8 * kNT;
    float acc[kNT][4], cor[kNT][4];  // hi x hi, and the two cross terms (independent chains)
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[n][j] = cor[n][j] = 0.f;
#pragma unroll 2
    for (int k0 = 0; k0 < N; k0 += 8) {
        float a[4];  // opA at (m0 + g, k0 + q), (m0 + g + 8, k0 + q), (m0 + g, k0 + q + 4), (m0 + g + 8, k0 + q + 4)
        a[0] = TA ? A[sw(k0 + q, m0 + g)] : A[sw(m0 + g, k0 + q)];
        a[1] = TA ? A[sw(k0 + q, m0 + g + 8)] : A[sw(m0 + g + 8, k0 + q)];
        a[2] = TA ? A[sw(k0 + q + 4, m0 + g)] : A[sw(m0 + g, k0 + q + 4)];
        a[3] = TA ? A[sw(k0 + q + 4, m0 + g + 8)] : A[sw(m0 + g + 8, k0 + q + 4)];
        if (KS) {
            const float s0 = ks[k0 + q], s1 = ks[k0 + q + 4];
            a[0] *= s0;
            a[1] *= s0;
            a[2] *= s1;
            a[3] *= s1;
        }
        uint32_t ah[4], al[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) split_tf32(a[j], ah[j], al[j]);
#pragma unroll
        for (int n = 0; n < kNT; ++n) {
            const int col = n0 + 8 * n + g;  // opB at (k0 + q, col), (k0 + q + 4, col)
            const float b0 = TB ? B[sw(col, k0 + q)] : B[sw(k0 + q, col)];
            const float b1 = TB ? B[sw(col, k0 + q + 4)] : B[sw(k0 + q + 4, col)];
            uint32_t bh0, bl0, bh1, bl1;
            split_tf32(b0, bh0, bl0);
            split_tf32(b1, bh1, bl1);
            mma_tf32(cor[n], al, bh0, bh1);
            mma_tf32(acc[n], ah, bh0, bh1);
            mma_tf32(cor[n], ah, bl0, bl1);
        }
    }
    Frag f;
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int j = 0; j < 4; ++j) f.v[4 * n + j] = acc[n][j] + cor[n][j];
    return f;
}

// The product of mm_core, handed element by element to emit(r, c, value, u).  A, B and ks (NULL:
// no diagonal) point into the shared memory.
template <bool TA, bool TB, typename F>
__device__ __forceinline__ void mm(const float *A, const float *B, int t, F &&emit, const float *ks = nullptr)
{
    const int lane = t & 31, w = t >> 5, g = lane >> 2, q = lane & 3;
    const int m0 = (w & 3) * 16, n0 = (w >> 2) * 8 * kNT;
    const Frag f = ks ? mm_core<TA, TB, true>((int)(A - smf), (int)(B - smf), (int)(ks - smf))
                      : mm_core<TA, TB, false>((int)(A - smf), (int)(B - smf), 0);
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                emit(m0 + g + 8 * hh, n0 + 8 * n + 2 * q + e, f.v[4 * n + 2 * hh + e], 4 * n + 2 * hh + e);
}

// Per-thread partial sums over the rows and columns a thread holds in mm's layout, completed over
// the block in two steps: *_put writes a thread's share to scratch shared memory (rows: two per
// thread, u bit 1, summed over the 4 lanes of a row, kColBlocks x 64 floats of scratch; columns:
// kColSlots per thread, u / 4 and u bit 0, summed over the 8 row groups of a warp, 4 x 64 floats),
// and after a barrier *_get(j) returns the total of row or column j.
__device__ __forceinline__ void row_put(const float (&p)[2], float *buf, int t)
{
    const int lane = t & 31, w = t >> 5, r = (w & 3) * 16 + (lane >> 2);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float x = p[hh];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        if ((lane & 3) == 0) buf[(w >> 2) * N + r + 8 * hh] = x;
    }
}

__device__ __forceinline__ float row_get(const float *buf, int j)
{
    float x = 0.f;
#pragma unroll
    for (int b = 0; b < kColBlocks; ++b) x += buf[b * N + j];
    return x;
}

__device__ __forceinline__ void col_put(const float (&p)[kColSlots], float *buf, int t)
{
    const int lane = t & 31, w = t >> 5;
#pragma unroll
    for (int j = 0; j < kColSlots; ++j) {
        float x = p[j];
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        if (lane < 4) buf[(w & 3) * N + (w >> 2) * 8 * kNT + 8 * (j >> 1) + 2 * lane + (j & 1)] = x;
    }
}

__device__ __forceinline__ float col_get(const float *buf, int j)
{
    return buf[j] + buf[N + j] + buf[2 * N + j] + buf[3 * N + j];
}

// Row half (0, 1) and column slot (0..7) of mm's element index u.
__device__ __forceinline__ constexpr int u_row(int u) { return (u >> 1) & 1; }
__device__ __forceinline__ constexpr int u_col(int u) { return ((u >> 2) << 1) | (u & 1); }

// Inclusive sums of x over the 32 lanes of a warp, restarted at every lane whose f is set (f on
// return: a restart lies at or before this lane).
__device__ __forceinline__ void seg_scan32(float &x, int &f, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float xo = __shfl_up_sync(0xffffffffu, x, o);
        const int fo = __shfl_up_sync(0xffffffffu, f, o);
        if (lane >= o) {
            if (!f) x += xo;
            f |= fo;
        }
    }
}

// The same over 64 positions, lane l holding positions l (x0, f0) and l + 32 (x1, f1).
__device__ __forceinline__ void seg_scan64(float &x0, int f0, float &x1, int f1, int lane)
{
    seg_scan32(x0, f0, lane);
    seg_scan32(x1, f1, lane);
    const float carry = __shfl_sync(0xffffffffu, x0, 31);
    if (!f1) x1 += carry;
}

// Gate vectors of one chunk (every thread of the block calls this; the caller synchronises after):
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
    if (t < N) {
        const size_t off = (size_t)(c.tok + t) * H + h;
        g.G[t] = t < c.n ? log_alpha[off] : 0.f;
        g.bet[t] = t < c.n ? beta[off] : 0.f;
    }
    __syncthreads();
    if (t < 32) {
        const float la0 = g.G[t], la1 = g.G[t + 32];
        const int r0 = la0 == -INFINITY, r1 = la1 == -INFINITY;
        float x0 = r0 ? 0.f : la0, x1 = r1 ? 0.f : la1;
        seg_scan64(x0, r0, x1, r1, t);
        int l0 = r0 ? t : -1, l1 = r1 ? t + 32 : -1;  // prefix maxima of the reset positions
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, l0, o), b = __shfl_up_sync(0xffffffffu, l1, o);
            if (t >= o) {
                l0 = max(l0, a);
                l1 = max(l1, b);
            }
        }
        l1 = max(l1, __shfl_sync(0xffffffffu, l0, 31));
        g.G[t] = x0;
        g.G[t + 32] = x1;
        g.last[t] = l0;
        g.last[t + 32] = l1;
    }
    __syncthreads();
    if (t < N) {
        g.gam[t] = g.last[t] >= 0 ? 0.f : expf(g.G[t]);
        g.lam[t] = g.last[N - 1] > t ? 0.f : expf(g.G[N - 1] - g.G[t]);
    }
}

// Decay between token i and a later token r of the chunk (zero across a reset or for i > r).
__device__ __forceinline__ float decay(const Gates &g, int r, int i)
{
    return (i <= r && g.last[r] <= i) ? expf(g.G[r] - g.G[i]) : 0.f;
}

// One chunk's rows of a [tokens, H, 64] tensor in registers, as 16-byte pieces (zero past the
// chunk end): fetch() issues every load, put() converts to fp32 into a shared matrix, so that the
// loads of several tensors are in flight at once.
template <typename TIn>
struct RowTile {
    static constexpr int V = 16 / (int)sizeof(TIn);      // elements per piece
    static constexpr int PER_ROW = N / V;
    static constexpr int ITER = N * PER_ROW / kThreads;  // pieces per thread
    uint4 b[ITER];

    __device__ __forceinline__ void fetch(const TIn *x, const ChunkRef &c, int H, int h, int t)
    {
#pragma unroll
        for (int u = 0; u < ITER; ++u) {
            const int e = t + u * kThreads, r = e / PER_ROW, j = (e % PER_ROW) * V;
            b[u] = r < c.n ? __ldg(reinterpret_cast<const uint4 *>(x + ((size_t)(c.tok + r) * H + h) * N + j))
                           : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    __device__ __forceinline__ void put(float *M, int t) const
    {
#pragma unroll
        for (int u = 0; u < ITER; ++u) {
            const int e = t + u * kThreads, r = e / PER_ROW, j = (e % PER_ROW) * V;
            if constexpr (sizeof(TIn) == 4) {
                *reinterpret_cast<float4 *>(&M[sw(r, j)]) = *reinterpret_cast<const float4 *>(&b[u]);
            } else {
                const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&b[u]);
                const float2 a0 = __bfloat1622float2(p[0]), a1 = __bfloat1622float2(p[1]),
                             a2 = __bfloat1622float2(p[2]), a3 = __bfloat1622float2(p[3]);
                *reinterpret_cast<float4 *>(&M[sw(r, j)]) = make_float4(a0.x, a0.y, a1.x, a1.y);
                *reinterpret_cast<float4 *>(&M[sw(r, j + 4)]) = make_float4(a2.x, a2.y, a3.x, a3.y);
            }
        }
    }
};

// A dense 64 x 64 fp32 matrix from global memory (row-major) into a shared matrix, and back.
__device__ __forceinline__ void mat_to_shared(float *M, const float *src, int t)
{
    constexpr int PER = MAT / 4 / kThreads;  // float4 pieces per thread
    float4 b[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) b[u] = __ldg(reinterpret_cast<const float4 *>(src) + t + u * kThreads);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = (t + u * kThreads) * 4;
        *reinterpret_cast<float4 *>(&M[sw(e >> 6, e & 63)]) = b[u];
    }
}

__device__ __forceinline__ void mat_from_shared(float *dst, const float *M, int t)
{
#pragma unroll
    for (int u = 0; u < MAT / 4 / kThreads; ++u) {
        const int e = (t + u * kThreads) * 4;
        reinterpret_cast<float4 *>(dst)[t + u * kThreads] = *reinterpret_cast<const float4 *>(&M[sw(e >> 6, e & 63)]);
    }
}

// A 64 x 64 block of a row-major fp32 matrix whose rows are `ld` floats apart, to and from a
// shared matrix (ld = 64: the dense forms above).
__device__ __forceinline__ void mat_to_shared_ld(float *M, const float *src, int ld, int t)
{
    constexpr int PER = MAT / 4 / kThreads;
    float4 b[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = (t + u * kThreads) * 4;
        b[u] = __ldg(reinterpret_cast<const float4 *>(src + (size_t)(e >> 6) * ld + (e & 63)));
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = (t + u * kThreads) * 4;
        *reinterpret_cast<float4 *>(&M[sw(e >> 6, e & 63)]) = b[u];
    }
}

__device__ __forceinline__ void mat_from_shared_ld(float *dst, const float *M, int ld, int t)
{
#pragma unroll
    for (int u = 0; u < MAT / 4 / kThreads; ++u) {
        const int e = (t + u * kThreads) * 4;
        *reinterpret_cast<float4 *>(dst + (size_t)(e >> 6) * ld + (e & 63)) =
            *reinterpret_cast<const float4 *>(&M[sw(e >> 6, e & 63)]);
    }
}

// T = (I + A)^{-1} for strictly lower A, given transposed (At(i, r) = A(r, i); only i < r is read).
// Column c of T is found by forward substitution on the kSolveLanes = L threads Lc .. Lc + L - 1,
// thread Lc + q holding rows q, q + L, q + 2L, ...: once row j is final it is passed among the L
// and subtracted from every later row, so one multiply-add lies between row j and row j + 1.  Every warp runs all 64
// steps (a column's rows above its diagonal stay zero; skipping them per warp would put a branch
// between the steps and keep the next step's loads from being issued early).  Every entry of T is
// written.
__device__ void unit_lower_inverse(const float *At, float *Tm, int t)
{
    constexpr int L = kSolveLanes;
    const int c = t / L, q = t % L;
    float s[kSolveRows];
#pragma unroll
    for (int m = 0; m < kSolveRows; ++m) s[m] = (L * m + q == c) ? 1.f : 0.f;
#pragma unroll
    for (int j = 0; j < N; ++j) {
        const float xj = __shfl_sync(0xffffffffu, s[j / L], j % L, L);
#pragma unroll
        for (int m = j / L; m < kSolveRows; ++m)
            if (L * m + q > j) s[m] = fmaf(-At[sw(j, L * m + q)], xj, s[m]);
    }
#pragma unroll
    for (int m = 0; m < kSolveRows; ++m) Tm[sw(L * m + q, c)] = s[m];
}

// ---- bwd_prep: per (chunk, head) the forward map (M, Bm) and the output term R ----------------
// Six shared matrices, reused as their contents die, so that two CTAs share an SM:
//   B0 K | B1 Q, then V, then Q again | B2 A^T, then W | B3 P | B4 T, then dO | B5 U~, then X.
template <typename TIn>
__global__ void __launch_bounds__(kThreads, 2)
    bwd_prep(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
             const float *__restrict__ log_alpha, const float *__restrict__ beta, const TIn *__restrict__ dout,
             const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int nseq, int T, int H, int G, int VS,
             float *__restrict__ Mo, float *__restrict__ Bo, float *__restrict__ Ro, float *__restrict__ Tw,
             float *__restrict__ Ww, float *__restrict__ Uw)
{
    float *K = smf, *B1 = K + MAT, *B2 = B1 + MAT, *P = B2 + MAT, *B4 = P + MAT, *B5 = B4 + MAT;
    Gates &g = *reinterpret_cast<Gates *>(B5 + MAT);
    float *bg = reinterpret_cast<float *>(&g + 1);  // beta gam
    // virtual head hx = h VS + value block; v, dout are [tokens, H VS, 64] in these terms
    const int t = threadIdx.x, hx = blockIdx.y, Hx = H * VS, h = VS == 1 ? hx : hx / VS, e = blockIdx.x;
    const ChunkRef c = chunk_ref(e, cu, off, nseq, T);
    if (c.n == 0) return;
    // grouped value heads: value head h reads q/k head h / G of H / G
    const int Hq = G == 1 ? H : H / G, hq = G == 1 ? h : h / G;
    RowTile<TIn> tv;
    {
        RowTile<TIn> tk, tq;
        tk.fetch(k, c, Hq, hq, t);
        tq.fetch(q, c, Hq, hq, t);
        tv.fetch(v, c, Hx, hx, t);
        tk.put(K, t);
        tq.put(B1, t);  // Q
    }
    chunk_gates<TIn>(g, log_alpha, beta, c, H, h, t);
    __syncthreads();
    if (t < N) bg[t] = g.bet[t] * g.gam[t];
    // A transposed: At(i, r) = b_r Gam_ri (K K^T)_ri for i < r (K K^T is symmetric)
    mm<false, true>(K, K, t, [&](int i, int r, float x, int) { B2[sw(i, r)] = i < r ? g.bet[r] * decay(g, r, i) * x : 0.f; });
    mm<false, true>(B1, K, t, [&](int r, int i, float x, int) { P[sw(r, i)] = decay(g, r, i) * x; });
    __syncthreads();
    tv.put(B1, t);  // V over Q (Q comes back for X)
    unit_lower_inverse(B2, B4, t);  // T in B4
    __syncthreads();
    const size_t base = ((size_t)e * Hx + hx) * (size_t)(N * N);
    mat_from_shared(Tw + base, B4, t);  // T for the gradient kernel
    mm<false, false>(B4, K, t, [&](int r, int m, float x, int) { B2[sw(r, m)] = x; }, bg);       // W over A^T
    mm<false, false>(B4, B1, t, [&](int r, int j, float x, int) { B5[sw(r, j)] = x; }, g.bet);   // U~
    __syncthreads();
    {
        RowTile<TIn> tq, td;
        tq.fetch(q, c, Hq, hq, t);
        td.fetch(dout, c, Hx, hx, t);
        mat_from_shared(Ww + base, B2, t);  // W and U~ for the gradient kernel
        mat_from_shared(Uw + base, B5, t);
        tq.put(B1, t);  // Q again, over V
        td.put(B4, t);  // dO over T
    }
    const float gC = g.gam[N - 1];
    mm<true, false>(K, B2, t, [&](int m, int n2, float x, int) { Mo[base + m * N + n2] = (m == n2 ? gC : 0.f) - x; }, g.lam);
    mm<true, false>(K, B5, t, [&](int m, int j, float x, int) { Bo[base + m * N + j] = x; }, g.lam);
    __syncthreads();
    // R = (Q^T diag(gam) - W^T P^T) dO = X^T dO with X = diag(gam) Q - P W (over U~)
    mm<false, false>(P, B2, t, [&](int r, int m, float x, int) { B5[sw(r, m)] = g.gam[r] * B1[sw(r, m)] - x; });
    __syncthreads();
    mm<true, false>(B5, B4, t, [&](int m, int j, float x, int) { Ro[base + m * N + j] = x; });
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

// ---- the scans: the chunk maps along one (sequence, head) ---------------------------------------
// Forward (REV = false): X = S0, then X <- M_c X + Bm_c; Xc[c] = the state entering chunk c.
// Reverse (REV = true):  X = dS_final, then X <- M_c^T X + R_c over the chunks from the last;
// Xc[c] = dL/dS at the end of chunk c, Xend = dS0.
// X is double-buffered in shared memory, and so is M_c; chunk c + 2's M and additive term are
// loaded into registers while chunk c is multiplied, so one barrier per chunk remains.
// X0 and Xend are [B, H, 64, 64 VS] (the caller's states); this chain takes the 64 columns of
// value block hx mod VS.
template <bool REV>
__device__ __forceinline__ void scan_body(const float *__restrict__ Mo, const float *__restrict__ Add,
                                          const float *__restrict__ X0, const int32_t *__restrict__ cu,
                                          const int32_t *__restrict__ off, int T, int H, int VS,
                                          float *__restrict__ Xc, float *__restrict__ Xend)
{
    // shared memory: X[2], then M[2]
    const int t = threadIdx.x, hx = blockIdx.x, s = blockIdx.y, Hx = H * VS;
    const int g = (t & 31) >> 2, q = t & 3, m0 = ((t >> 5) & 3) * 16, n0 = (t >> 7) * 8 * kNT;
    constexpr int PER = MAT / 4 / kThreads;  // float4 pieces of a matrix per thread
    int first, count;
    seq_chunks(s, cu, off, T, first, count);
    const int ld = N * VS;  // row stride of the caller's states
    const size_t st0 = ((size_t)s * H + hx / VS) * (size_t)N * ld + (size_t)(hx % VS) * N;
    auto chunk_base = [&](int i) { return ((size_t)(first + (REV ? count - 1 - i : i)) * Hx + hx) * (size_t)MAT; };
    auto fetch_m = [&](int i, float4 (&m)[PER]) {
        const float4 *src = reinterpret_cast<const float4 *>(Mo + chunk_base(i));
#pragma unroll
        for (int u = 0; u < PER; ++u) m[u] = __ldg(src + t + u * kThreads);
    };
    auto fetch_a = [&](int i, float2 (&a)[2 * kNT]) {  // the additive term in mm's layout
        const float *src = Add + chunk_base(i);
#pragma unroll
        for (int n = 0; n < kNT; ++n)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                a[2 * n + hh] = __ldg(reinterpret_cast<const float2 *>(src + (m0 + g + 8 * hh) * N + n0 + 8 * n + 2 * q));
    };
    auto put_m = [&](float *M, const float4 (&m)[PER]) {
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = (t + u * kThreads) * 4;
            *reinterpret_cast<float4 *>(&M[sw(e >> 6, e & 63)]) = m[u];
        }
    };
    float4 pm[PER];
    float2 pa[2 * kNT], pa2[2 * kNT];
    if (X0) {
        mat_to_shared_ld(smf, X0 + st0, ld, t);
    } else {
#pragma unroll
        for (int u = 0; u < PER; ++u) reinterpret_cast<float4 *>(smf)[t + u * kThreads] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (count > 0) {
        fetch_m(0, pm);
        fetch_a(0, pa);
        put_m(smf + 2 * MAT, pm);
    }
    if (count > 1) {
        fetch_m(1, pm);
        fetch_a(1, pa2);
    }
    __syncthreads();
    for (int i = 0; i < count; ++i) {
        const int cur = i & 1;
        float *Xcur = smf + cur * MAT, *Xnxt = smf + (cur ^ 1) * MAT, *Mcur = smf + (2 + cur) * MAT,
              *Mnxt = smf + (3 - cur) * MAT;
        mat_from_shared(Xc + chunk_base(i), Xcur, t);
        mm<REV, false>(Mcur, Xcur, t, [&](int r, int c, float x, int u) {
            const float2 a = pa[2 * (u >> 2) + u_row(u)];
            Xnxt[sw(r, c)] = x + ((u & 1) ? a.y : a.x);
        });
        if (i + 1 < count) {
            put_m(Mnxt, pm);
#pragma unroll
            for (int u = 0; u < 2 * kNT; ++u) pa[u] = pa2[u];
        }
        if (i + 2 < count) {
            fetch_m(i + 2, pm);
            fetch_a(i + 2, pa2);
        }
        __syncthreads();
    }
    if (Xend) mat_from_shared_ld(Xend + st0, smf + (count & 1) * MAT, ld, t);
}

// Both scans in one launch, blockIdx.z = 0 forward and 1 reverse: they are independent, and with
// 64 KB of shared memory two CTAs share an SM, so all 2 B H chains run at once.
__global__ void __launch_bounds__(kThreads, 2)
    bwd_scans(const float *__restrict__ Mo, const float *__restrict__ Bo, const float *__restrict__ Ro,
              const float *__restrict__ S0, const float *__restrict__ dS_final, const int32_t *__restrict__ cu,
              const int32_t *__restrict__ off, int T, int H, int VS, float *__restrict__ Sc,
              float *__restrict__ dSn, float *__restrict__ dS0)
{
    if (blockIdx.z == 0) scan_body<false>(Mo, Bo, S0, cu, off, T, H, VS, Sc, nullptr);
    else scan_body<true>(Mo, Ro, dS_final, cu, off, T, H, VS, dSn, dS0);
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
              const float *__restrict__ Sc, const float *__restrict__ dSn, const float *__restrict__ Tw,
              const float *__restrict__ Ww, const float *__restrict__ Uw, const int32_t *__restrict__ cu,
              const int32_t *__restrict__ off, int nseq, int T, int H, int G, int VS, float *__restrict__ dq,
              float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dla, float *__restrict__ dbe)
{
    float *K = smf, *Q = K + MAT, *V = Q + MAT, *dO = V + MAT, *S = dO + MAT, *dSp = S + MAT, *KK = dSp + MAT,
          *Tm = KK + MAT, *X1 = Tm + MAT, *U = X1 + MAT, *QK = U + MAT, *dU = QK + MAT, *X2 = dU + MAT;
    Gates &g = *reinterpret_cast<Gates *>(X2 + MAT);
    float *vec = reinterpret_cast<float *>(&g + 1);
    float *bg = vec, *dG = vec + N, *dgam = vec + 2 * N, *dlam = vec + 3 * N, *dbet = vec + 4 * N, *dgC = vec + 5 * N;
    // virtual head hx = h VS + value block (see the file's head); dq, dk, dv are written as
    // [tokens, H VS, 64] and dlog_alpha, dbeta as [tokens, H VS]
    const int t = threadIdx.x, hx = blockIdx.y, Hx = H * VS, h = VS == 1 ? hx : hx / VS, e = blockIdx.x;
    const ChunkRef c = chunk_ref(e, cu, off, nseq, T);
    if (c.n == 0) return;
    const size_t base = ((size_t)e * Hx + hx) * (size_t)(N * N);
    {
        // grouped value heads: value head h reads q/k head h / G of H / G (dq, dk per value head)
        const int Hq = G == 1 ? H : H / G, hq = G == 1 ? h : h / G;
        RowTile<TIn> tk, tq, tv, td;
        tk.fetch(k, c, Hq, hq, t);
        tq.fetch(q, c, Hq, hq, t);
        tv.fetch(v, c, Hx, hx, t);
        td.fetch(dout, c, Hx, hx, t);
        mat_to_shared(S, Sc + base, t);
        mat_to_shared(dSp, dSn + base, t);
        mat_to_shared(Tm, Tw + base, t);  // T = (I + A)^{-1}, W and U~ from the prep kernel
        mat_to_shared(dU, Ww + base, t);
        mat_to_shared(U, Uw + base, t);
        tk.put(K, t);
        tq.put(Q, t);
        tv.put(V, t);
        td.put(dO, t);
    }
    chunk_gates<TIn>(g, log_alpha, beta, c, H, h, t);
    __syncthreads();
    if (t < N) bg[t] = g.bet[t] * g.gam[t];
    // per thread, in mm's layout (index u): the dQ, dK, dV accumulators; partial d beta, d gam, dG
    // and d lam over its two rows; partial dG over its columns
    float aq[kFrag], ak[kFrag], av[kFrag];
    float pb[2] = {0.f, 0.f}, pg[2] = {0.f, 0.f}, pG[2] = {0.f, 0.f}, pl[2] = {0.f, 0.f};
    float pc[kColSlots];
#pragma unroll
    for (int i = 0; i < kFrag; ++i) aq[i] = ak[i] = av[i] = 0.f;
#pragma unroll
    for (int i = 0; i < kColSlots; ++i) pc[i] = 0.f;
    mm<false, true>(K, K, t, [&](int r, int i, float x, int) { KK[sw(r, i)] = x; });
    mm<false, true>(Q, K, t, [&](int r, int i, float x, int) { QK[sw(r, i)] = x; });
    mm<false, false>(K, dSp, t, [&](int i, int m, float x, int) { X2[sw(i, m)] = x; });  // K dS'
    __syncthreads();
    // P in X1; d gam_C = <S, dS'>
    {
        float part = 0.f;
        for (int idx = t; idx < N * N; idx += kThreads) {
            const int r = idx >> 6, i = idx & 63;
            X1[sw(r, i)] = decay(g, r, i) * QK[sw(r, i)];
            part = fmaf(S[sw(r, i)], dSp[sw(r, i)], part);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((t & 31) == 0) dgC[t >> 5] = part;  // per warp, summed in warp order below (reproducible)
    }
    __syncthreads();
    // U = U~ - W S (U~ in U, W in dU, both loaded)
    mm<false, false>(dU, S, t, [&](int r, int j, float x, int) { U[sw(r, j)] -= x; });
    __syncthreads();
    // dU = P^T dO + diag(lam) K dS'; d lam_i = sum_j (K dS')_ij U_ij (the only term of d lam)
    mm<true, false>(X1, dO, t, [&](int i, int j, float x, int u) {
        const float kd = X2[sw(i, j)];
        dU[sw(i, j)] = x + g.lam[i] * kd;
        pl[u_row(u)] = fmaf(kd, U[sw(i, j)], pl[u_row(u)]);
    });
    __syncthreads();
    // dP = dO U^T (lower incl.), and at once D2 = dP o Gam into X1 (P is no longer needed) with the
    // dG terms of Gam (P); dK += diag(lam) U dS'^T; d gam (O1) and dQ += diag(gam) dO S^T
    mm<false, true>(dO, U, t, [&](int r, int i, float x, int u) {
        const float gm = decay(g, r, i), dp = i <= r ? x : 0.f;
        X1[sw(r, i)] = dp * gm;
        const float E = dp * QK[sw(r, i)] * gm;
        pG[u_row(u)] += E;
        pc[u_col(u)] -= E;
    });
    mm<false, true>(U, dSp, t, [&](int i, int m, float x, int u) { ak[u] += g.lam[i] * x; });
    // dQ += diag(gam) dO S^T, and d gam_r (O1) = sum_j dO_rj (Q S)_rj = sum_m Q_rm (dO S^T)_rm
    mm<false, true>(dO, S, t, [&](int r, int m, float x, int u) {
        aq[u] += g.gam[r] * x;
        pg[u_row(u)] = fmaf(Q[sw(r, m)], x, pg[u_row(u)]);
    });
    __syncthreads();
    // dW = -dU S^T into U (U is no longer needed)
    mm<false, true>(dU, S, t, [&](int r, int m, float x, int) { U[sw(r, m)] = -x; });
    __syncthreads();
    // Y = T^T dU: dV, dbeta;  X = T^T dW: dK, dbeta, d gam
    mm<true, false>(Tm, dU, t, [&](int i, int j, float x, int u) {
        av[u] += g.bet[i] * x;
        pb[u_row(u)] = fmaf(x, V[sw(i, j)], pb[u_row(u)]);
    });
    mm<true, false>(Tm, U, t, [&](int i, int m, float x, int u) {
        ak[u] += bg[i] * x;
        const float xk = x * K[sw(i, m)];
        pb[u_row(u)] = fmaf(g.gam[i], xk, pb[u_row(u)]);
        pg[u_row(u)] = fmaf(g.bet[i], xk, pg[u_row(u)]);
    });
    // dT = dU (diag(b) V)^T + dW (diag(b gam) K)^T into X2 (K dS' is no longer needed); the
    // diagonals scale the result's column index
    mm<false, true>(dU, V, t, [&](int r, int i, float x, int) { X2[sw(r, i)] = g.bet[i] * x; });
    mm<false, true>(U, K, t, [&](int r, int i, float x, int) { X2[sw(r, i)] += bg[i] * x; });
    __syncthreads();
    // Z = dT T^T into dU
    mm<false, true>(X2, Tm, t, [&](int r, int i, float x, int) { dU[sw(r, i)] = x; });
    __syncthreads();
    // dA = -T^T Z (strictly lower) -> D into U; dbeta (A); dG from Gam (A)
    mm<true, false>(Tm, dU, t, [&](int r, int i, float x, int u) {
        float d = 0.f;
        if (i < r) {
            const float gm = decay(g, r, i), kk = KK[sw(r, i)];
            const float dAg = -x * gm;  // dA o Gam
            d = g.bet[r] * dAg;
            pb[u_row(u)] = fmaf(dAg, kk, pb[u_row(u)]);
            const float E = d * kk;
            pG[u_row(u)] += E;
            pc[u_col(u)] -= E;
        }
        U[sw(r, i)] = d;
    });
    __syncthreads();
    // D + D^T into dU (Z is no longer needed), so that D K + D^T K is one product
    for (int idx = t; idx < N * N; idx += kThreads) {
        const int r = idx >> 6, i = idx & 63;
        dU[sw(r, i)] = U[sw(r, i)] + U[sw(i, r)];
    }
    __syncthreads();
    // dK += (D + D^T) K + D2^T Q;  dQ += D2 K
    mm<false, false>(dU, K, t, [&](int, int, float x, int u) { ak[u] += x; });
    mm<true, false>(X1, Q, t, [&](int, int, float x, int u) { ak[u] += x; });
    mm<false, false>(X1, K, t, [&](int, int, float x, int u) { aq[u] += x; });
    // the partial sums over the block (X2 is free scratch now: its last reader is two barriers back)
    constexpr int RB = kColBlocks * N;  // scratch of one row sum
    row_put(pb, X2, t);
    row_put(pg, X2 + RB, t);
    row_put(pG, X2 + 2 * RB, t);
    row_put(pl, X2 + 3 * RB, t);
    col_put(pc, X2 + 4 * RB, t);
    __syncthreads();
    if (t < N) {
        dbet[t] = row_get(X2, t);
        dgam[t] = row_get(X2 + RB, t);
        dG[t] = row_get(X2 + 2 * RB, t) + col_get(X2 + 4 * RB, t);
        dlam[t] = row_get(X2 + 3 * RB, t);
    }
    __syncthreads();
    // gate gradients: gam_r = exp(G_r), lam_i = exp(G_63 - G_i), gam_C = gam_63; then dlog_alpha_j =
    // sum of dG_r over the rows r >= j of j's reset segment (0 at a reset itself): a segmented sum
    // over the reversed rows, restarting below every reset
    if (t < 32) {
        float x[2], li[2];
        int f[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = N - 1 - (t + 32 * u);
            li[u] = dlam[j] * g.lam[j];
            x[u] = dG[j] + dgam[j] * g.gam[j] - li[u];
            f[u] = j < N - 1 && g.last[j + 1] == j + 1;
        }
        float s63 = li[0] + li[1];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s63 += __shfl_xor_sync(0xffffffffu, s63, o);
        if (t == 0) {  // row 63
            float dgc = 0.f;
            for (int w = 0; w < kThreads / 32; ++w) dgc += dgC[w];
            x[0] += s63 + dgc * g.gam[N - 1];
        }
        seg_scan64(x[0], f[0], x[1], f[1], t);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = N - 1 - (t + 32 * u);
            dlam[j] = g.last[j] == j ? 0.f : x[u];  // reuse as dlog_alpha
        }
    }
    __syncthreads();
    {
        const int lane = t & 31, w = t >> 5, gq = lane >> 2, qq = lane & 3;
        const int m0 = (w & 3) * 16, n0 = (w >> 2) * 8 * kNT;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = m0 + gq + 8 * hh;
            if (r >= c.n) continue;
            const size_t row = ((size_t)(c.tok + r) * Hx + hx) * N + n0 + 2 * qq;
#pragma unroll
            for (int n = 0; n < kNT; ++n) {
                const int u = 4 * n + 2 * hh;
                *reinterpret_cast<float2 *>(dq + row + 8 * n) = make_float2(aq[u], aq[u + 1]);
                *reinterpret_cast<float2 *>(dk + row + 8 * n) = make_float2(ak[u], ak[u + 1]);
                *reinterpret_cast<float2 *>(dv + row + 8 * n) = make_float2(av[u], av[u + 1]);
            }
        }
    }
    if (t < c.n) {
        const size_t o = (size_t)(c.tok + t) * Hx + hx;
        dla[o] = dlam[t];
        dbe[o] = dbet[t];
    }
}

// Grouped value heads: dq, dk of q/k head j = the sum over its G value heads (rows of 64 fp32,
// [rows, Hv, 64] -> [rows, Hv / G, 64]); one thread per output element.
__global__ void bwd_group_sum(const float *__restrict__ gq, const float *__restrict__ gk, float *__restrict__ dq,
                              float *__restrict__ dk, long out_elems, int G)
{
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= out_elems) return;
    const long row = i / N, col = i % N;  // row = token * Hk + j
    const float *a = gq + row * G * N + col, *b = gk + row * G * N + col;
    float sq = 0.f, sk = 0.f;
    for (int u = 0; u < G; ++u) {
        sq += a[u * N];
        sk += b[u * N];
    }
    dq[i] = sq;
    dk[i] = sk;
}

// Value splits: dlog_alpha, dbeta of value head i = the sum over its VS virtual heads
// ([rows, H VS] -> [rows, H]); one thread per output element.
__global__ void bwd_gate_sum(const float *__restrict__ pla, const float *__restrict__ pbe, float *__restrict__ dla,
                             float *__restrict__ dbe, long out_elems, int VS)
{
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= out_elems) return;
    float sa = 0.f, sb = 0.f;
    for (int u = 0; u < VS; ++u) {
        sa += pla[i * VS + u];
        sb += pbe[i * VS + u];
    }
    dla[i] = sa;
    dbe[i] = sb;
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


// ==== dk = 128: the key dimension as two 64-column blocks (KB = 2) ==============================
// Every formula of the dk = 64 kernels with the key dimension split into blocks a in {0, 1}: q and
// k rows of 128 are read as two heads of 64 ([tokens, 2 Hq, 64]); K K^T, Q K^T, K dS' and
// sum_a W_a S_a are sums of two products; M is four tiles (M_ab = gam_C delta_ab I -
// K_a^T diag(lam) W_b), Bm, R, W, S_c and dS are two.  Value splits apply unchanged (VS heads of
// 64 value columns).

// The sum of two products of mm_core, handed out as mm does.
template <bool TA, bool TB, typename F>
__device__ __forceinline__ void mm2(const float *A0, const float *B0, const float *A1, const float *B1, int t,
                                    F &&emit)
{
    const int lane = t & 31, w = t >> 5, g = lane >> 2, q = lane & 3;
    const int m0 = (w & 3) * 16, n0 = (w >> 2) * 8 * kNT;
    Frag f = mm_core<TA, TB, false>((int)(A0 - smf), (int)(B0 - smf), 0);
    const Frag f1 = mm_core<TA, TB, false>((int)(A1 - smf), (int)(B1 - smf), 0);
#pragma unroll
    for (int i = 0; i < kFrag; ++i) f.v[i] += f1.v[i];
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                emit(m0 + g + 8 * hh, n0 + 8 * n + 2 * q + e, f.v[4 * n + 2 * hh + e], 4 * n + 2 * hh + e);
}

// Per (chunk, virtual head) unit u: T and U~ one matrix each at u; W, Bm, R, S_c, dS two at 2u + a;
// M four at 4u + 2a + b.
// Ten shared matrices: K0 K1 | Q0 Q1 (then X0 X1) | A^T (then V, then dO) | P | T | U~ | W0 W1.
template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_prep2(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta, const TIn *__restrict__ dout,
              const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int nseq, int T, int H, int G, int VS,
              float *__restrict__ Mo, float *__restrict__ Bo, float *__restrict__ Ro, float *__restrict__ Tw,
              float *__restrict__ Ww, float *__restrict__ Uw)
{
    float *K0 = smf, *K1 = K0 + MAT, *Q0 = K1 + MAT, *Q1 = Q0 + MAT, *AT = Q1 + MAT, *P = AT + MAT, *Tm = P + MAT,
          *Ub = Tm + MAT, *W0 = Ub + MAT, *W1 = W0 + MAT;
    Gates &g = *reinterpret_cast<Gates *>(W1 + MAT);
    float *bg = reinterpret_cast<float *>(&g + 1);
    const int t = threadIdx.x, hx = blockIdx.y, Hx = H * VS, h = VS == 1 ? hx : hx / VS, e = blockIdx.x;
    const ChunkRef c = chunk_ref(e, cu, off, nseq, T);
    if (c.n == 0) return;
    const int Hq = G == 1 ? H : H / G, hq = G == 1 ? h : h / G;
    RowTile<TIn> tv;
    {
        RowTile<TIn> tk0, tk1, tq0, tq1;
        tk0.fetch(k, c, 2 * Hq, 2 * hq, t);
        tk1.fetch(k, c, 2 * Hq, 2 * hq + 1, t);
        tq0.fetch(q, c, 2 * Hq, 2 * hq, t);
        tq1.fetch(q, c, 2 * Hq, 2 * hq + 1, t);
        tv.fetch(v, c, Hx, hx, t);
        tk0.put(K0, t);
        tk1.put(K1, t);
        tq0.put(Q0, t);
        tq1.put(Q1, t);
    }
    chunk_gates<TIn>(g, log_alpha, beta, c, H, h, t);
    __syncthreads();
    if (t < N) bg[t] = g.bet[t] * g.gam[t];
    mm2<false, true>(K0, K0, K1, K1, t,
                     [&](int i, int r, float x, int) { AT[sw(i, r)] = i < r ? g.bet[r] * decay(g, r, i) * x : 0.f; });
    mm2<false, true>(Q0, K0, Q1, K1, t, [&](int r, int i, float x, int) { P[sw(r, i)] = decay(g, r, i) * x; });
    __syncthreads();
    unit_lower_inverse(AT, Tm, t);
    __syncthreads();
    tv.put(AT, t);  // V over A^T
    const size_t u = (size_t)e * Hx + hx;
    mat_from_shared(Tw + u * MAT, Tm, t);
    __syncthreads();
    mm<false, false>(Tm, K0, t, [&](int r, int m, float x, int) { W0[sw(r, m)] = x; }, bg);
    mm<false, false>(Tm, K1, t, [&](int r, int m, float x, int) { W1[sw(r, m)] = x; }, bg);
    mm<false, false>(Tm, AT, t, [&](int r, int j, float x, int) { Ub[sw(r, j)] = x; }, g.bet);
    __syncthreads();
    RowTile<TIn> td;
    td.fetch(dout, c, Hx, hx, t);
    mat_from_shared(Ww + (2 * u) * MAT, W0, t);
    mat_from_shared(Ww + (2 * u + 1) * MAT, W1, t);
    mat_from_shared(Uw + u * MAT, Ub, t);
    const float gC = g.gam[N - 1];
    float *Mb = Mo + 4 * u * MAT;
    mm<true, false>(K0, W0, t, [&](int m, int n2, float x, int) { Mb[m * N + n2] = (m == n2 ? gC : 0.f) - x; }, g.lam);
    mm<true, false>(K0, W1, t, [&](int m, int n2, float x, int) { Mb[MAT + m * N + n2] = -x; }, g.lam);
    mm<true, false>(K1, W0, t, [&](int m, int n2, float x, int) { Mb[2 * MAT + m * N + n2] = -x; }, g.lam);
    mm<true, false>(K1, W1, t,
                    [&](int m, int n2, float x, int) { Mb[3 * MAT + m * N + n2] = (m == n2 ? gC : 0.f) - x; }, g.lam);
    mm<true, false>(K0, Ub, t, [&](int m, int j, float x, int) { Bo[(2 * u) * MAT + m * N + j] = x; }, g.lam);
    mm<true, false>(K1, Ub, t, [&](int m, int j, float x, int) { Bo[(2 * u + 1) * MAT + m * N + j] = x; }, g.lam);
    // X_a = diag(gam) Q_a - P W_a in place over Q_a (each element read and written by one thread)
    mm<false, false>(P, W0, t, [&](int r, int m, float x, int) { Q0[sw(r, m)] = g.gam[r] * Q0[sw(r, m)] - x; });
    mm<false, false>(P, W1, t, [&](int r, int m, float x, int) { Q1[sw(r, m)] = g.gam[r] * Q1[sw(r, m)] - x; });
    td.put(AT, t);  // dO over V (its last reader, the U~ product, is behind the barrier above)
    __syncthreads();
    // R_a = X_a^T dO
    mm<true, false>(Q0, AT, t, [&](int m, int j, float x, int) { Ro[(2 * u) * MAT + m * N + j] = x; });
    mm<true, false>(Q1, AT, t, [&](int m, int j, float x, int) { Ro[(2 * u + 1) * MAT + m * N + j] = x; });
}

// The scans for KB = 2: the state is two 64 x 64 blocks (rows 0..63 and 64..127 of the 128-row
// state); forward X_a <- sum_b M_ab X_b + Bm_a, reverse X_a <- sum_b M_ba^T X_b + R_a.  Shared
// memory: X[2][2], then M[2][4] (192 KB, one CTA per SM).
template <bool REV>
__device__ __forceinline__ void scan_body2(const float *__restrict__ Mo, const float *__restrict__ Add,
                                           const float *__restrict__ X0, const int32_t *__restrict__ cu,
                                           const int32_t *__restrict__ off, int T, int H, int VS,
                                           float *__restrict__ Xc, float *__restrict__ Xend)
{
    const int t = threadIdx.x, hx = blockIdx.x, s = blockIdx.y, Hx = H * VS;
    const int g = (t & 31) >> 2, q = t & 3, m0 = ((t >> 5) & 3) * 16, n0 = (t >> 7) * 8 * kNT;
    constexpr int PER = MAT / 4 / kThreads;
    int first, count;
    seq_chunks(s, cu, off, T, first, count);
    const int ld = N * VS;  // row stride of the caller's states [B, H, 128, 64 VS]
    const size_t st0 = ((size_t)s * H + hx / VS) * (size_t)(2 * N) * ld + (size_t)(hx % VS) * N;
    auto unit = [&](int i) { return (size_t)(first + (REV ? count - 1 - i : i)) * Hx + hx; };
    auto fetch_m = [&](int i, float4 (&m)[4][PER]) {
        const float4 *src = reinterpret_cast<const float4 *>(Mo + 4 * unit(i) * MAT);
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
#pragma unroll
            for (int uu = 0; uu < PER; ++uu) m[bb][uu] = __ldg(src + bb * (MAT / 4) + t + uu * kThreads);
    };
    auto fetch_a = [&](int i, float2 (&a)[2][2 * kNT]) {
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            const float *src = Add + (2 * unit(i) + blk) * MAT;
#pragma unroll
            for (int n = 0; n < kNT; ++n)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    a[blk][2 * n + hh] =
                        __ldg(reinterpret_cast<const float2 *>(src + (m0 + g + 8 * hh) * N + n0 + 8 * n + 2 * q));
        }
    };
    auto put_m = [&](float *M, const float4 (&m)[4][PER]) {
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
#pragma unroll
            for (int uu = 0; uu < PER; ++uu) {
                const int e = (t + uu * kThreads) * 4;
                *reinterpret_cast<float4 *>(&M[bb * MAT + sw(e >> 6, e & 63)]) = m[bb][uu];
            }
    };
    float *Xs = smf, *Ms = smf + 4 * MAT;
    float4 pm[4][PER];
    float2 pa[2][2 * kNT], pa2[2][2 * kNT];
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
        if (X0) {
            mat_to_shared_ld(Xs + blk * MAT, X0 + st0 + (size_t)blk * N * ld, ld, t);
        } else {
#pragma unroll
            for (int uu = 0; uu < PER; ++uu)
                reinterpret_cast<float4 *>(Xs + blk * MAT)[t + uu * kThreads] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    if (count > 0) {
        fetch_m(0, pm);
        fetch_a(0, pa);
        put_m(Ms, pm);
    }
    if (count > 1) {
        fetch_m(1, pm);
        fetch_a(1, pa2);
    }
    __syncthreads();
    for (int i = 0; i < count; ++i) {
        const int cur = i & 1;
        float *Xcur = Xs + cur * 2 * MAT, *Xnxt = Xs + (cur ^ 1) * 2 * MAT, *Mcur = Ms + cur * 4 * MAT,
              *Mnxt = Ms + (cur ^ 1) * 4 * MAT;
        mat_from_shared(Xc + (2 * unit(i)) * MAT, Xcur, t);
        mat_from_shared(Xc + (2 * unit(i) + 1) * MAT, Xcur + MAT, t);
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            const float *A0 = Mcur + (REV ? a : 2 * a) * MAT;      // M_0a (reverse) or M_a0
            const float *A1 = Mcur + (REV ? 2 + a : 2 * a + 1) * MAT;  // M_1a (reverse) or M_a1
            mm2<REV, false>(A0, Xcur, A1, Xcur + MAT, t, [&](int r, int cc, float x, int uu) {
                const float2 av = pa[a][2 * (uu >> 2) + u_row(uu)];
                Xnxt[a * MAT + sw(r, cc)] = x + ((uu & 1) ? av.y : av.x);
            });
        }
        if (i + 1 < count) {
            put_m(Mnxt, pm);
#pragma unroll
            for (int blk = 0; blk < 2; ++blk)
#pragma unroll
                for (int uu = 0; uu < 2 * kNT; ++uu) pa[blk][uu] = pa2[blk][uu];
        }
        if (i + 2 < count) {
            fetch_m(i + 2, pm);
            fetch_a(i + 2, pa2);
        }
        __syncthreads();
    }
    if (Xend) {
#pragma unroll
        for (int blk = 0; blk < 2; ++blk)
            mat_from_shared_ld(Xend + st0 + (size_t)blk * N * ld, Xs + (count & 1) * 2 * MAT + blk * MAT, ld, t);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    bwd_scans2(const float *__restrict__ Mo, const float *__restrict__ Bo, const float *__restrict__ Ro,
               const float *__restrict__ S0, const float *__restrict__ dS_final, const int32_t *__restrict__ cu,
               const int32_t *__restrict__ off, int T, int H, int VS, float *__restrict__ Sc,
               float *__restrict__ dSn, float *__restrict__ dS0)
{
    if (blockIdx.z == 0) scan_body2<false>(Mo, Bo, S0, cu, off, T, H, VS, Sc, nullptr);
    else scan_body2<true>(Mo, Ro, dS_final, cu, off, T, H, VS, dSn, dS0);
}

// Gradients for KB = 2.  Thirteen shared matrices, reused as their contents die:
//   K0 K1 | B0 B1: Q, then W, then dW, then Q again | S0 S1: S, then dT (S0), Z (S1), D + D^T (S0) |
//   D0 D1: dS', then T (D0), V (D1) | KK | X1: P, then D2 | Ub: U~, then U, then D | X2: K dS', then dU,
//   then scratch | dO.
template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_grads2(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
               const float *__restrict__ log_alpha, const float *__restrict__ beta, const TIn *__restrict__ dout,
               const float *__restrict__ Sc, const float *__restrict__ dSn, const float *__restrict__ Tw,
               const float *__restrict__ Ww, const float *__restrict__ Uw, const int32_t *__restrict__ cu,
               const int32_t *__restrict__ off, int nseq, int T, int H, int G, int VS, float *__restrict__ dq,
               float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dla, float *__restrict__ dbe)
{
    float *K0 = smf, *K1 = K0 + MAT, *B0 = K1 + MAT, *B1 = B0 + MAT, *S0s = B1 + MAT, *S1s = S0s + MAT,
          *D0 = S1s + MAT, *D1 = D0 + MAT, *KK = D1 + MAT, *X1 = KK + MAT, *Ub = X1 + MAT, *X2 = Ub + MAT,
          *dO = X2 + MAT;
    Gates &g = *reinterpret_cast<Gates *>(dO + MAT);
    float *vec = reinterpret_cast<float *>(&g + 1);
    float *bg = vec, *dG = vec + N, *dgam = vec + 2 * N, *dlam = vec + 3 * N, *dbet = vec + 4 * N, *dgC = vec + 5 * N;
    const int t = threadIdx.x, hx = blockIdx.y, Hx = H * VS, h = VS == 1 ? hx : hx / VS, e = blockIdx.x;
    const ChunkRef c = chunk_ref(e, cu, off, nseq, T);
    if (c.n == 0) return;
    const size_t u1 = (size_t)e * Hx + hx;
    const int Hq = G == 1 ? H : H / G, hq = G == 1 ? h : h / G;
    {
        RowTile<TIn> tk0, tk1, tq0, tq1, td;
        tk0.fetch(k, c, 2 * Hq, 2 * hq, t);
        tk1.fetch(k, c, 2 * Hq, 2 * hq + 1, t);
        tq0.fetch(q, c, 2 * Hq, 2 * hq, t);
        tq1.fetch(q, c, 2 * Hq, 2 * hq + 1, t);
        td.fetch(dout, c, Hx, hx, t);
        mat_to_shared(S0s, Sc + (2 * u1) * MAT, t);
        mat_to_shared(S1s, Sc + (2 * u1 + 1) * MAT, t);
        mat_to_shared(D0, dSn + (2 * u1) * MAT, t);
        mat_to_shared(D1, dSn + (2 * u1 + 1) * MAT, t);
        mat_to_shared(Ub, Uw + u1 * MAT, t);
        tk0.put(K0, t);
        tk1.put(K1, t);
        tq0.put(B0, t);
        tq1.put(B1, t);
        td.put(dO, t);
    }
    chunk_gates<TIn>(g, log_alpha, beta, c, H, h, t);
    __syncthreads();
    if (t < N) bg[t] = g.bet[t] * g.gam[t];
    float aq0[kFrag], aq1[kFrag], ak0[kFrag], ak1[kFrag], av[kFrag];
    float pb[2] = {0.f, 0.f}, pg[2] = {0.f, 0.f}, pG[2] = {0.f, 0.f}, pl[2] = {0.f, 0.f};
    float pc[kColSlots];
#pragma unroll
    for (int i = 0; i < kFrag; ++i) aq0[i] = aq1[i] = ak0[i] = ak1[i] = av[i] = 0.f;
#pragma unroll
    for (int i = 0; i < kColSlots; ++i) pc[i] = 0.f;
    // K K^T; P = Gam o Q K^T; K dS'
    mm2<false, true>(K0, K0, K1, K1, t, [&](int r, int i, float x, int) { KK[sw(r, i)] = x; });
    mm2<false, true>(B0, K0, B1, K1, t, [&](int r, int i, float x, int) { X1[sw(r, i)] = decay(g, r, i) * x; });
    mm2<false, false>(K0, D0, K1, D1, t, [&](int i, int m, float x, int) { X2[sw(i, m)] = x; });
    // dQ_a += diag(gam) dO S_a^T, and d gam_r (O1) = sum_a sum_m Q_a(r, m) (dO S_a^T)(r, m)
    mm<false, true>(dO, S0s, t, [&](int r, int m, float x, int uu) {
        aq0[uu] += g.gam[r] * x;
        pg[u_row(uu)] = fmaf(B0[sw(r, m)], x, pg[u_row(uu)]);
    });
    mm<false, true>(dO, S1s, t, [&](int r, int m, float x, int uu) {
        aq1[uu] += g.gam[r] * x;
        pg[u_row(uu)] = fmaf(B1[sw(r, m)], x, pg[u_row(uu)]);
    });
    // d gam_C = <S, dS'>, per warp (summed in warp order with the gate gradients)
    {
        float part = 0.f;
        for (int idx = t; idx < N * N; idx += kThreads) {
            const int r = idx >> 6, i = idx & 63;
            part = fmaf(S0s[sw(r, i)], D0[sw(r, i)], part);
            part = fmaf(S1s[sw(r, i)], D1[sw(r, i)], part);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((t & 31) == 0) dgC[t >> 5] = part;
    }
    __syncthreads();
    mat_to_shared(B0, Ww + (2 * u1) * MAT, t);  // W over Q
    mat_to_shared(B1, Ww + (2 * u1 + 1) * MAT, t);
    __syncthreads();
    // U = U~ - sum_a W_a S_a
    mm2<false, false>(B0, S0s, B1, S1s, t, [&](int r, int j, float x, int) { Ub[sw(r, j)] -= x; });
    __syncthreads();
    // dU = P^T dO + diag(lam) K dS' over K dS'; d lam_i = sum_j (K dS')_ij U_ij
    mm<true, false>(X1, dO, t, [&](int i, int j, float x, int uu) {
        const float kd = X2[sw(i, j)];
        X2[sw(i, j)] = x + g.lam[i] * kd;
        pl[u_row(uu)] = fmaf(kd, Ub[sw(i, j)], pl[u_row(uu)]);
    });
    __syncthreads();
    // dP = dO U^T (lower incl.) -> D2 = dP o Gam over P, with the dG terms of Gam (P): E = dP o P
    mm<false, true>(dO, Ub, t, [&](int r, int i, float x, int uu) {
        const float gm = decay(g, r, i), dp = i <= r ? x : 0.f;
        const float E = dp * X1[sw(r, i)];
        X1[sw(r, i)] = dp * gm;
        pG[u_row(uu)] += E;
        pc[u_col(uu)] -= E;
    });
    // dK_a += diag(lam) U dS'_a^T
    mm<false, true>(Ub, D0, t, [&](int i, int, float x, int uu) { ak0[uu] += g.lam[i] * x; });
    mm<false, true>(Ub, D1, t, [&](int i, int, float x, int uu) { ak1[uu] += g.lam[i] * x; });
    __syncthreads();
    {
        RowTile<TIn> tv;
        tv.fetch(v, c, Hx, hx, t);
        mat_to_shared(D0, Tw + u1 * MAT, t);  // T over dS'_0
        tv.put(D1, t);                         // V over dS'_1
    }
    // dW_a = -dU S_a^T over W_a
    mm<false, true>(X2, S0s, t, [&](int r, int m, float x, int) { B0[sw(r, m)] = -x; });
    mm<false, true>(X2, S1s, t, [&](int r, int m, float x, int) { B1[sw(r, m)] = -x; });
    __syncthreads();
    // Y = T^T dU: dV, dbeta;  X_a = T^T dW_a: dK_a, dbeta, d gam
    mm<true, false>(D0, X2, t, [&](int i, int j, float x, int uu) {
        av[uu] += g.bet[i] * x;
        pb[u_row(uu)] = fmaf(x, D1[sw(i, j)], pb[u_row(uu)]);
    });
    mm<true, false>(D0, B0, t, [&](int i, int m, float x, int uu) {
        ak0[uu] += bg[i] * x;
        const float xk = x * K0[sw(i, m)];
        pb[u_row(uu)] = fmaf(g.gam[i], xk, pb[u_row(uu)]);
        pg[u_row(uu)] = fmaf(g.bet[i], xk, pg[u_row(uu)]);
    });
    mm<true, false>(D0, B1, t, [&](int i, int m, float x, int uu) {
        ak1[uu] += bg[i] * x;
        const float xk = x * K1[sw(i, m)];
        pb[u_row(uu)] = fmaf(g.gam[i], xk, pb[u_row(uu)]);
        pg[u_row(uu)] = fmaf(g.bet[i], xk, pg[u_row(uu)]);
    });
    // dT = dU (diag(b) V)^T + sum_a dW_a (diag(b gam) K_a)^T over S_0; the diagonals scale the
    // result's column index
    mm<false, true>(X2, D1, t, [&](int r, int i, float x, int) { S0s[sw(r, i)] = g.bet[i] * x; });
    mm2<false, true>(B0, K0, B1, K1, t, [&](int r, int i, float x, int) { S0s[sw(r, i)] += bg[i] * x; });
    __syncthreads();
    // Z = dT T^T over S_1
    mm<false, true>(S0s, D0, t, [&](int r, int i, float x, int) { S1s[sw(r, i)] = x; });
    __syncthreads();
    // dA = -T^T Z (strictly lower) -> D over U; dbeta (A); dG from Gam (A)
    mm<true, false>(D0, S1s, t, [&](int r, int i, float x, int uu) {
        float d = 0.f;
        if (i < r) {
            const float gm = decay(g, r, i), kk = KK[sw(r, i)];
            const float dAg = -x * gm;
            d = g.bet[r] * dAg;
            pb[u_row(uu)] = fmaf(dAg, kk, pb[u_row(uu)]);
            const float E = d * kk;
            pG[u_row(uu)] += E;
            pc[u_col(uu)] -= E;
        }
        Ub[sw(r, i)] = d;
    });
    __syncthreads();
    // D + D^T over dT, and Q again over dW
    {
        RowTile<TIn> tq0, tq1;
        tq0.fetch(q, c, 2 * Hq, 2 * hq, t);
        tq1.fetch(q, c, 2 * Hq, 2 * hq + 1, t);
        for (int idx = t; idx < N * N; idx += kThreads) {
            const int r = idx >> 6, i = idx & 63;
            S0s[sw(r, i)] = Ub[sw(r, i)] + Ub[sw(i, r)];
        }
        tq0.put(B0, t);
        tq1.put(B1, t);
    }
    __syncthreads();
    // dK_a += (D + D^T) K_a + D2^T Q_a;  dQ_a += D2 K_a
    mm<false, false>(S0s, K0, t, [&](int, int, float x, int uu) { ak0[uu] += x; });
    mm<false, false>(S0s, K1, t, [&](int, int, float x, int uu) { ak1[uu] += x; });
    mm<true, false>(X1, B0, t, [&](int, int, float x, int uu) { ak0[uu] += x; });
    mm<true, false>(X1, B1, t, [&](int, int, float x, int uu) { ak1[uu] += x; });
    mm<false, false>(X1, K0, t, [&](int, int, float x, int uu) { aq0[uu] += x; });
    mm<false, false>(X1, K1, t, [&](int, int, float x, int uu) { aq1[uu] += x; });
    // the partial sums over the block (X2 is free scratch: its last reader is behind two barriers)
    constexpr int RB = kColBlocks * N;
    row_put(pb, X2, t);
    row_put(pg, X2 + RB, t);
    row_put(pG, X2 + 2 * RB, t);
    row_put(pl, X2 + 3 * RB, t);
    col_put(pc, X2 + 4 * RB, t);
    __syncthreads();
    if (t < N) {
        dbet[t] = row_get(X2, t);
        dgam[t] = row_get(X2 + RB, t);
        dG[t] = row_get(X2 + 2 * RB, t) + col_get(X2 + 4 * RB, t);
        dlam[t] = row_get(X2 + 3 * RB, t);
    }
    __syncthreads();
    if (t < 32) {
        float x[2], li[2];
        int f[2];
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) {
            const int j = N - 1 - (t + 32 * w2);
            li[w2] = dlam[j] * g.lam[j];
            x[w2] = dG[j] + dgam[j] * g.gam[j] - li[w2];
            f[w2] = j < N - 1 && g.last[j + 1] == j + 1;
        }
        float s63 = li[0] + li[1];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s63 += __shfl_xor_sync(0xffffffffu, s63, o);
        if (t == 0) {  // row 63
            float dgc = 0.f;
            for (int w2 = 0; w2 < kThreads / 32; ++w2) dgc += dgC[w2];
            x[0] += s63 + dgc * g.gam[N - 1];
        }
        seg_scan64(x[0], f[0], x[1], f[1], t);
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) {
            const int j = N - 1 - (t + 32 * w2);
            dlam[j] = g.last[j] == j ? 0.f : x[w2];  // reuse as dlog_alpha
        }
    }
    __syncthreads();
    {
        const int lane = t & 31, w = t >> 5, gq = lane >> 2, qq = lane & 3;
        const int m0 = (w & 3) * 16, n0 = (w >> 2) * 8 * kNT;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = m0 + gq + 8 * hh;
            if (r >= c.n) continue;
            const size_t rowk = ((size_t)(c.tok + r) * Hx + hx) * (2 * N) + n0 + 2 * qq;  // dq, dk rows of 128
            const size_t rowv = ((size_t)(c.tok + r) * Hx + hx) * N + n0 + 2 * qq;
#pragma unroll
            for (int n = 0; n < kNT; ++n) {
                const int uu = 4 * n + 2 * hh;
                *reinterpret_cast<float2 *>(dq + rowk + 8 * n) = make_float2(aq0[uu], aq0[uu + 1]);
                *reinterpret_cast<float2 *>(dq + rowk + N + 8 * n) = make_float2(aq1[uu], aq1[uu + 1]);
                *reinterpret_cast<float2 *>(dk + rowk + 8 * n) = make_float2(ak0[uu], ak0[uu + 1]);
                *reinterpret_cast<float2 *>(dk + rowk + N + 8 * n) = make_float2(ak1[uu], ak1[uu + 1]);
                *reinterpret_cast<float2 *>(dv + rowv + 8 * n) = make_float2(av[uu], av[uu + 1]);
            }
        }
    }
    if (t < c.n) {
        const size_t o = (size_t)(c.tok + t) * Hx + hx;
        dla[o] = dlam[t];
        dbe[o] = dbet[t];
    }
}

// Grouped sums over rows of width W (dq, dk of KB = 2 have rows of 128): out[row][col] =
// sum_u in[row G + u][col]; one thread per output element.
__global__ void bwd_group_sum_w(const float *__restrict__ gq, const float *__restrict__ gk, float *__restrict__ dq,
                                float *__restrict__ dk, long out_elems, int G, int W)
{
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= out_elems) return;
    const long row = i / W, col = i % W;
    const float *a = gq + row * G * W + col, *b = gk + row * G * W + col;
    float sq = 0.f, sk = 0.f;
    for (int u = 0; u < G; ++u) {
        sq += a[u * W];
        sk += b[u * W];
    }
    dq[i] = sq;
    dk[i] = sk;
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

// Workspace: chunk offsets, then eight matrices per (chunk, virtual head) -- M, Bm, R, S_c, dS_{c+1},
// T, W, U~ -- then, when the q/k gradients are partial (G VS > 1), per-virtual-head dq and dk, and
// when the gate gradients are partial (VS > 1), per-virtual-head dlog_alpha and dbeta.
struct BwdLayout {
    size_t off, mats, qk, gates, bytes;
};

BwdLayout bwd_layout(int B, int T, int H, int varlen, int G, int VS, int KB = 1)
{
    BwdLayout l;
    const size_t Hx = (size_t)H * VS, tokens = varlen ? (size_t)T : (size_t)B * T;
    l.off = align256b((size_t)(B + 1) * sizeof(int32_t));
    l.mats = align256b((size_t)bwd_chunks(B, T, varlen) * Hx * N * N * sizeof(float));
    l.qk = G * VS > 1 ? align256b(tokens * Hx * N * KB * sizeof(float)) : 0;
    l.gates = VS > 1 ? align256b(tokens * Hx * sizeof(float)) : 0;
    // KB = 1: M, Bm, R, S_c, dS, T, W, U~; KB = 2: M four, Bm, R, S_c, dS, W two, T and U~ one
    l.bytes = l.off + (KB == 1 ? 8 : 16) * l.mats + 2 * l.qk + 2 * l.gates;
    return l;
}

// dk = 128: the same plan with the KB = 2 kernels.
template <typename TIn>
cudaError_t run_bwd2(const BwdArgs &a, cudaStream_t st)
{
    const int varlen = a.cu_seqlens != nullptr;
    const long chunks = bwd_chunks(a.B, a.T, varlen);
    const int VS = a.VS, Hx = a.H * VS;
    const BwdLayout l = bwd_layout(a.B, a.T, a.H, varlen, a.G, VS, 2);
    const size_t mats = l.mats;
    char *w = static_cast<char *>(a.workspace);
    int32_t *off = reinterpret_cast<int32_t *>(w);
    w += l.off;
    float *Mo = reinterpret_cast<float *>(w);
    float *Bo = reinterpret_cast<float *>(w + 4 * mats);
    float *Ro = reinterpret_cast<float *>(w + 6 * mats);
    float *Sc = reinterpret_cast<float *>(w + 8 * mats);
    float *dSn = reinterpret_cast<float *>(w + 10 * mats);
    float *Tw = reinterpret_cast<float *>(w + 12 * mats);
    float *Ww = reinterpret_cast<float *>(w + 13 * mats);
    float *Uw = reinterpret_cast<float *>(w + 15 * mats);
    const size_t tokens = varlen ? (size_t)a.T : (size_t)a.B * a.T;
    const int GQ = a.G * VS;
    char *pw = w + 16 * mats;
    float *gq = GQ > 1 ? reinterpret_cast<float *>(pw) : a.dq;
    float *gk = GQ > 1 ? reinterpret_cast<float *>(pw + l.qk) : a.dk;
    float *gla = VS > 1 ? reinterpret_cast<float *>(pw + 2 * l.qk) : a.dlog_alpha;
    float *gbe = VS > 1 ? reinterpret_cast<float *>(pw + 2 * l.qk + l.gates) : a.dbeta;
    const int32_t *offp = varlen ? off : nullptr;
    if (varlen) {
        bwd_offsets<<<1, 1, 0, st>>>(a.cu_seqlens, a.B, off);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const TIn *q = static_cast<const TIn *>(a.q), *k = static_cast<const TIn *>(a.k),
              *v = static_cast<const TIn *>(a.v), *dout = static_cast<const TIn *>(a.dout);
    const int smem_prep = (10 * MAT) * (int)sizeof(float) + (int)sizeof(Gates) + N * (int)sizeof(float);
    const int smem_grads = (13 * MAT) * (int)sizeof(float) + (int)sizeof(Gates) + 6 * N * (int)sizeof(float);
    const int smem_scan = 12 * MAT * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_prep2<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_grads2<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_grads);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_scans2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_scan);
    if (e != cudaSuccess) return e;
    const dim3 gc((unsigned)chunks, Hx);
    bwd_prep2<TIn><<<gc, kThreads, smem_prep, st>>>(q, k, v, a.log_alpha, a.beta, dout, a.cu_seqlens, offp, a.B, a.T,
                                                    a.H, a.G, VS, Mo, Bo, Ro, Tw, Ww, Uw);
    bwd_scans2<<<dim3(Hx, a.B, 2), kThreads, smem_scan, st>>>(Mo, Bo, Ro, a.S0, a.dS_final, a.cu_seqlens, offp, a.T,
                                                             a.H, VS, Sc, dSn, a.dS0);
    bwd_grads2<TIn><<<gc, kThreads, smem_grads, st>>>(q, k, v, a.log_alpha, a.beta, dout, Sc, dSn, Tw, Ww, Uw,
                                                      a.cu_seqlens, offp, a.B, a.T, a.H, a.G, VS, gq, gk, a.dv, gla,
                                                      gbe);
    if (GQ > 1) {
        const long out_elems = (long)(tokens * (a.H / a.G)) * 2 * N;
        if (out_elems > 0)
            bwd_group_sum_w<<<(unsigned)((out_elems + 255) / 256), 256, 0, st>>>(gq, gk, a.dq, a.dk, out_elems, GQ,
                                                                                 2 * N);
    }
    if (VS > 1) {
        const long out_elems = (long)(tokens * a.H);
        if (out_elems > 0)
            bwd_gate_sum<<<(unsigned)((out_elems + 255) / 256), 256, 0, st>>>(gla, gbe, a.dlog_alpha, a.dbeta,
                                                                              out_elems, VS);
    }
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t run_bwd(const BwdArgs &a, cudaStream_t st)
{
    const int varlen = a.cu_seqlens != nullptr;
    const long chunks = bwd_chunks(a.B, a.T, varlen);
    const int VS = a.VS, Hx = a.H * VS;
    const BwdLayout l = bwd_layout(a.B, a.T, a.H, varlen, a.G, VS);
    const size_t mats = l.mats;
    char *w = static_cast<char *>(a.workspace);
    int32_t *off = reinterpret_cast<int32_t *>(w);
    w += l.off;
    float *Mo = reinterpret_cast<float *>(w);
    float *Bo = reinterpret_cast<float *>(w + mats);
    float *Ro = reinterpret_cast<float *>(w + 2 * mats);
    float *Sc = reinterpret_cast<float *>(w + 3 * mats);
    float *dSn = reinterpret_cast<float *>(w + 4 * mats);
    float *Tw = reinterpret_cast<float *>(w + 5 * mats);
    float *Ww = reinterpret_cast<float *>(w + 6 * mats);
    float *Uw = reinterpret_cast<float *>(w + 7 * mats);
    // grouped value heads and value splits: per-virtual-head dq, dk (and dlog_alpha, dbeta) here,
    // summed at the end
    const size_t tokens = varlen ? (size_t)a.T : (size_t)a.B * a.T;
    const int GQ = a.G * VS;  // virtual heads per q/k head
    char *pw = w + 8 * mats;
    float *gq = GQ > 1 ? reinterpret_cast<float *>(pw) : a.dq;
    float *gk = GQ > 1 ? reinterpret_cast<float *>(pw + l.qk) : a.dk;
    float *gla = VS > 1 ? reinterpret_cast<float *>(pw + 2 * l.qk) : a.dlog_alpha;
    float *gbe = VS > 1 ? reinterpret_cast<float *>(pw + 2 * l.qk + l.gates) : a.dbeta;
    const int32_t *offp = varlen ? off : nullptr;
    if (varlen) {
        bwd_offsets<<<1, 1, 0, st>>>(a.cu_seqlens, a.B, off);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const TIn *q = static_cast<const TIn *>(a.q), *k = static_cast<const TIn *>(a.k),
              *v = static_cast<const TIn *>(a.v), *dout = static_cast<const TIn *>(a.dout);
    const int smem_prep = (6 * MAT) * (int)sizeof(float) + (int)sizeof(Gates) + N * (int)sizeof(float);
    const int smem_grads = (13 * MAT) * (int)sizeof(float) + (int)sizeof(Gates) + 6 * N * (int)sizeof(float);
    const int smem_scan = 4 * MAT * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_prep<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_grads<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_grads);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_scans, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_scan);
    if (e != cudaSuccess) return e;
    const dim3 gc((unsigned)chunks, Hx);
    bwd_prep<TIn><<<gc, kThreads, smem_prep, st>>>(q, k, v, a.log_alpha, a.beta, dout, a.cu_seqlens, offp, a.B, a.T,
                                                   a.H, a.G, VS, Mo, Bo, Ro, Tw, Ww, Uw);
    bwd_scans<<<dim3(Hx, a.B, 2), kThreads, smem_scan, st>>>(Mo, Bo, Ro, a.S0, a.dS_final, a.cu_seqlens, offp, a.T,
                                                            a.H, VS, Sc, dSn, a.dS0);
    bwd_grads<TIn><<<gc, kThreads, smem_grads, st>>>(q, k, v, a.log_alpha, a.beta, dout, Sc, dSn, Tw, Ww, Uw,
                                                     a.cu_seqlens, offp, a.B, a.T, a.H, a.G, VS, gq, gk, a.dv, gla,
                                                     gbe);
    if (GQ > 1) {
        const long out_elems = (long)(tokens * (a.H / a.G)) * N;
        if (out_elems > 0)
            bwd_group_sum<<<(unsigned)((out_elems + 255) / 256), 256, 0, st>>>(gq, gk, a.dq, a.dk, out_elems, GQ);
    }
    if (VS > 1) {
        const long out_elems = (long)(tokens * a.H);
        if (out_elems > 0)
            bwd_gate_sum<<<(unsigned)((out_elems + 255) / 256), 256, 0, st>>>(gla, gbe, a.dlog_alpha, a.dbeta,
                                                                              out_elems, VS);
    }
    return cudaGetLastError();
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int varlen, int G, int VS, int KB)
{
    return bwd_layout(B, T, H, varlen, G, VS, KB).bytes;
}

cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t stream)
{
    if (a.KB == 2)
        return a.dtype == GDN_DTYPE_BF16 ? run_bwd2<__nv_bfloat16>(a, stream) : run_bwd2<float>(a, stream);
    return a.dtype == GDN_DTYPE_BF16 ? run_bwd<__nv_bfloat16>(a, stream) : run_bwd<float>(a, stream);
}

}  // namespace gdn
