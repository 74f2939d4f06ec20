// gdn_chunk_tc.cu -- chunkwise (WY / UT-transform) forward of the gated delta rule for bf16
// q/k/v on the 5th-generation tensor cores (tcgen05, accumulators in TMEM, tiles fed by TMA).
//
// Sources: Sykra README, "Architectural Highlights" (chunk-parallel training through the WY /
// unit triangular transform: one triangular solve per chunk, the rest matrix products; the
// data-dependent forget gate) and DeltaPhase README, section 1 ("Fast Triangular Solve": an
// exact O(C^2) per-chunk transition solve; beta in (0, 2)).  Per chunk of C = 64 tokens entered
// with state S (dk x dv):
//   A  = strictly_lower(diag(b) (Gam o K K^T)),   T = (I + A)^{-1}
//   W  = T diag(b gam) K,   U~ = T diag(b) V,   U = U~ - W S
//   O  = diag(gam) Q S + lower_incl(Gam o Q K^T) U
//   S' = gam_C S + K^T diag(lam) U
//
// One CTA of 384 threads per (sequence, head, value-column block); three warpgroups work
// concurrently:
//   two intra warpgroups (warps 4-7 and 8-11) take alternate chunks, ahead of the state chain:
//       gate sums (warp-shuffle segmented scan), Gram matrices [K;Q] K^T (tcgen05, M=128),
//       decays, A = diag(b)(Gam o K K^T) and P = Gam o Q K^T, T = (I+A)^{-1} (8x8 diagonal
//       blocks by substitution on CUDA cores, 16->32->64 merges on mma.sync TF32), written as
//       T diag(b) and T diag(b gam) in bf16, then the WY products U~^T = V^T (T diag b)^T and
//       W^T = K^T (T diag(b gam))^T (tcgen05) and W^T to shared memory.
//   chain warpgroup (warps 0-3), thread j = value column j, for chunk c:
//       U^T   = U~^T - S^T W^T           (accumulated onto U~^T)
//       O     = (gam Q) S + P U          (value head 64: M = 64 token rows, 16-byte row stores)
//       S'^T  = gam_C S^T + U^T (lam K)  (accumulated onto the pre-scaled fp32 state in TMEM)
//   At value head 128 the chain's A operands (the bf16 copy of S^T, U^T as hi + lo parts) stay in
//   tensor memory, the intra side writes -W^T, and the outputs are formed transposed (O^T) and
//   leave through shared memory (transposing stmatrix, then 16-byte row stores).
//   Loads: K/Q through a TMA stage ring (NS stages, reissued as soon as a stage's last MMA
//   completes), V through NB buffers, gates by cp.async onto an mbarrier.
// The state chain's critical path per chunk is two MMA round trips plus their epilogues.  The
// three roles run different code on the same SM sub-partitions, so loops whose bodies hold no
// register arrays are kept rolled where that measured faster (instruction-cache misses).
//
// Gates: decays are exp of log_alpha sums taken from the last exact reset (log_alpha = -inf)
// inside the chunk.  Padded rows of a partial chunk get b = 0 and log_alpha = 0, which makes
// their (finite) K/Q/V contents contribute nothing.
//
// Every mbarrier wait is bounded (2 s).  On timeout the kernel records an error word, stops
// issuing work and skips all later waits; at the end each MMA-issuing thread waits (bounded) for
// the MMAs it had issued before TMEM is freed.  The call's outputs are then undefined.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"
#include "sm100_ptx.cuh"
#include "../../include/gdn.h"

namespace gdn {

__device__ int g_tc_device_error = 0;

namespace {

using namespace sm100;

constexpr int CH = 64;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int LDF = 68;  // fp32 row stride of the 64 x 64 solve matrices
// Kernel flags (used by the segment scan): V is taken as zero (nothing of V is loaded), and the
// initial state is the identity (dv must equal dk).  With out == nullptr no output is formed.
constexpr int kFlagVZero = 1;
constexpr int kFlagS0Identity = 2;
// Fused prologue: q and k arrive unnormalised and the gate arrays hold raw projections a, b;
// rows are divided by sqrt(|x|^2 + kNormEps) and log alpha = -a_scale softplus(a),
// beta = b_scale sigmoid(b) (DeltaPhase README, section 1: beta = 2 sigmoid(W_beta x)).
constexpr int kFlagPrologue = 4;
constexpr float kNormEps = 1e-6f;
// Longest sequence first (varlen launches of at most THREADS sequences): CTA z takes the sequence
// of rank z by length (ties by index), so that the longest chains, which set the launch's length,
// start in the first wave instead of wherever the packing put them.
constexpr int kFlagLongestFirst = 8;
// Complex-phase memory with its prologue fused (dk = 32 complex, the real recurrence at head size
// 64): K and Q arrive as fp32 (re, im) pairs and are scaled (1 / sqrt(dk), 1 / dk), real parts
// first, into the bf16 tiles in shared memory; beta arrives raw, b = beta / lam is formed in the
// gate scan, and V enters unscaled with lam sqrt(dk) folded into T diag(.) of the U~ product
// (b v = beta sqrt(dk) V); see gdn_phase.cu for the algebra.
constexpr int kFlagPhase = 16;
constexpr float kPhaseSqrtDk = 5.656854249492381f;  // sqrt(32)
#ifndef GDN_U_SPLIT
#define GDN_U_SPLIT 1
#endif

template <int DK, int DV, bool PH = false>
struct TcCfg {
    static_assert(!PH || (DK == 64 && DV == 64), "the fused phase prologue is built for dk = 32 complex, dv = 64");
    // Two intra warpgroups take alternate chunks.
    static constexpr int NI = 2;
    static constexpr int THREADS = 128 * (1 + NI);
    // TA (value head 128): the chain keeps its MMA A operands -- the bf16 copy of S^T and U^T --
    // in tensor memory and forms the outputs transposed (O^T, value columns on the TMEM lanes),
    // which frees the shared S^T and U^T copies for a third K/Q stage.
    static constexpr bool TA = DV == 128;
    static constexpr int NS = TA ? 3 : ((DK == 128 || DV == 128) ? 2 : 3);  // K/Q stages
    // U~^T / U^T slots in TMEM: one per intra warpgroup (TA) or per stage
    static constexpr int NU = TA ? NI : NS;
    // O buffers in TMEM (two: the output epilogue of a chunk overlaps the next state MMA); O^T
    // takes 64 columns (TA), O (M = 64 token rows) DV columns
    static constexpr int O_COLS = TA ? 64 : DV;
    static constexpr int SB_COLS = TA ? DK / 2 : 0;  // bf16 S^T, two per column (TA)
    static constexpr int NBO = (2 * O_COLS + DK + SB_COLS + NI * 64 + NU * 64 <= 512) ? 2 : 1;
    // V buffers (two: the V load of a chunk starts two chunks ahead)
    // (one with the fused phase prologue, whose K/Q stages are twice as large)
    static constexpr int NB = PH ? 1 : (TA ? (DK == 64 ? 2 : 1) : NBO);
    // shared memory byte offsets (swizzled tiles first, all 1024-aligned)
    static constexpr int KQ = 0;                                 // per stage: per 64-feature block K (8K) | Q (8K)
    // PH: a stage first holds the fp32 K and Q rows (two 32-float blocks each), which the intra
    // warpgroup turns into the bf16 tiles in place
    static constexpr int KQ_STAGE = (DK / 64) * 16384 * (PH ? 2 : 1);
    static constexpr int V = KQ + NS * KQ_STAGE;                 // per buffer: per 64-column block 8 KB
    static constexpr int V_BUF = (DV / 64) * 8192;
    static constexpr int PM = V + NB * V_BUF;                    // per stage: P bf16, 64 x 128 B
    static constexpr int ST = PM + NS * 8192;                    // S^T bf16, per 64-feature block DV x 128 B
    // one S^T copy: the copy of chunk c + 1 is written once the state MMA of chunk c has
    // completed, and that MMA's commit also covers the U and O1 MMAs that read the copy of chunk c
    static constexpr int ST_BYTES = TA ? 0 : (DK / 64) * DV * 128;
    static constexpr int UT = ST + ST_BYTES;                     // U^T bf16, DV x 128 B
    static constexpr int WG0 = UT + (TA ? 0 : DV * 128);         // per intra warpgroup:
    static constexpr int W_TB = 0;                               //   T diag(b)      bf16 64 x 128 B
    static constexpr int W_TG = 8192;                            //   T diag(b gam)  bf16 64 x 128 B
    // W^T (DK rows x 128 B bf16) is written over T diag(b gam) (dk = 64) or over both T tiles
    // (dk = 128) once the WY MMAs have read them
    static constexpr int W_WT = DK == 64 ? W_TG : W_TB;
    static constexpr int W_AT = 16384;                           //   decays, then A, then T: fp32 [64][LDF]
    static constexpr int W_XS = W_AT + CH * LDF * 4;             //   merge scratch, 4 x 256 fp32
    static constexpr int WG_BYTES = (W_XS + 4 * 256 * 4 + 1023) & ~1023;
    // TA with two O buffers: a bf16 tile [64 tokens][DV] through which the outputs leave (one
    // O buffer: the chunk's own K/Q stage serves, once its state MMA has completed)
    static constexpr int OT = WG0 + NI * WG_BYTES;
    static constexpr int OT_BYTES = (TA && NBO == 2) ? CH * DV * 2 : 0;
    static constexpr int GT = OT + OT_BYTES;                     // per stage: gate vectors
    static constexpr int GT_STAGE = (PH ? 8 : 7) * CH * 4;       //   graw, G2, gam, lam, bet, last, (gC), (PH: bv)
    static constexpr int BAR = GT + NS * GT_STAGE;
    static constexpr int NBAR = 5 * NS + NB + NBO + 2 + 4 * NI + 1 + NI;
    static constexpr int MISC = BAR + NBAR * 8;                  // TMEM slot, abort flag
    static constexpr int TOTAL = MISC + 16;
    // TMEM columns
    static constexpr uint32_t T_O = 0;                            // NBO x O_COLS: outputs
    static constexpr uint32_t T_S = NBO * O_COLS;                 // DK: fp32 state (transposed)
    static constexpr uint32_t T_SB = T_S + DK;                    // SB_COLS: bf16 S^T (TA)
    static constexpr uint32_t T_G = T_SB + SB_COLS;               // NI x 64: Gram, then W^T (intra)
    static constexpr uint32_t T_U = T_G + NI * 64;                // NU x 64: U~^T, then U^T
    static_assert(T_U + NU * 64 <= 512, "TMEM budget");
    static_assert(TOTAL + 1024 <= 232448, "shared memory budget");
};

// barrier indices
template <int NS, int NI, int NB, int NBO> struct Bars {
    static constexpr int kq_full = 0;            // [NS] K/Q tiles of a stage landed (TMA)
    static constexpr int gfull = NS;             // [NS] gates landed, 32 arrivals (cp.async of chain warp 0)
    static constexpr int gready = 2 * NS;        // [NS] gate vectors (gam, lam, gam_C) computed
    static constexpr int tready = 3 * NS;        // [NS] intra -> chain: P, U~^T, W^T, gam Q, lam K ready
    static constexpr int cdone = 4 * NS;         // [NS] chain -> intra: the output MMA has read the stage's P
    static constexpr int v_full = 5 * NS;        // [NB] V tile landed
    static constexpr int u = 5 * NS + NB;
    static constexpr int s = 5 * NS + NB + 1;
    static constexpr int o = 5 * NS + NB + 2;    // [NBO] output MMAs of a chunk done
    static constexpr int gram = 5 * NS + NB + NBO + 2;  // [NI] Gram MMA done
    static constexpr int uw = gram + NI;               // [NI] WY MMAs done
    static constexpr int tfree = uw + NI;              // [NI] chain -> intra: the U MMA has read W^T
    static constexpr int ufree = tfree + NI;           // [NI] chain -> intra: the U slot has been read (TA)
    static constexpr int drain = ufree + NI;           // [1 + NI] after a timeout: the MMAs of each issuer done
};

// Thread roles inside an intra warpgroup (t = 0..127): the gate scan runs on warp scan_warp(wg)
// and the MMAs are issued by thread kIssuer, away from SM sub-partition 0, which holds the
// chain's issuing thread (thread 0).
__device__ __forceinline__ int scan_warp(int wg) { return wg == 0 ? 1 : 2; }
constexpr int kIssuer = 96;

// The bounded wait past a first unsuccessful try, out of line: one copy serves every wait site.
__device__ __noinline__ void wait_slow(uint64_t *b, uint32_t parity, int *abort)
{
    if (!mbar_wait_bounded(b, parity, kWaitLimitNs)) {
        atomicOr(&g_tc_device_error, 1);
        *(volatile int *)abort = 1;
    }
}

struct Ctl {
    uint64_t *bar;
    int *abort;
    __device__ void wait(int i, uint32_t parity) const
    {
        if (*(volatile int *)abort) return;
        if (mbar_try_wait(&bar[i], parity)) return;
        wait_slow(&bar[i], parity, abort);
    }
    __device__ bool aborted() const { return *(volatile int *)abort != 0; }
    __device__ void arrive(int i) const
    {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar[i])) : "memory");
    }
};

__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Final value v of T[r][c]: written as the bf16 entries of T diag(b) and T diag(b gam)
// (128B-swizzled rows, the B operands of the WY products) and, where later merges read it, in fp32.
struct TOut {
    float *Tm;
    unsigned char *TB, *TG;
    const float *bet, *gam;
    // the column factors of T diag(.) for the U~ product: bet, or (fused phase prologue) the
    // per-token factor that also carries the scale of V
    const float *bv;
    __device__ __forceinline__ float vfac(int c, float bc) const { return bv ? bv[c] : bc; }
    // (vc, bc, gc) = factors of column c, loaded once by the caller
    __device__ __forceinline__ void put(int r, int c, float v, float vc, float bc, float gc) const
    {
        Tm[r * LDF + c] = v;
        const float b = v * bc;
        *reinterpret_cast<__nv_bfloat16 *>(TB + sw128_off(r, c)) = __float2bfloat16_rn(v * vc);
        *reinterpret_cast<__nv_bfloat16 *>(TG + sw128_off(r, c)) = __float2bfloat16_rn(b * gc);
    }
    // c even; (u0, u1, b0, b1, g0, g1) = factors of columns c, c+1; keep: also store the fp32 values
    __device__ __forceinline__ void put2(int r, int c, float v0, float v1, float u0, float u1, float b0, float b1,
                                         float g0, float g1, bool keep) const
    {
        if (keep) *reinterpret_cast<float2 *>(&Tm[r * LDF + c]) = make_float2(v0, v1);
        const float x0 = v0 * b0, x1 = v1 * b1;
        *reinterpret_cast<uint32_t *>(TB + sw128_off(r, c)) = pack_bf16x2(v0 * u0, v1 * u1);
        *reinterpret_cast<uint32_t *>(TG + sw128_off(r, c)) = pack_bf16x2(x0 * g0, x1 * g1);
    }
};

// fp32 bits used as a TF32 operand: the tensor core ignores the low 13 mantissa bits.
__device__ __forceinline__ uint32_t tf(float x) { return __float_as_uint(x); }

// T = (I + A)^{-1} for strictly lower triangular A (64 x 64 fp32, row stride LDF; only entries
// below the diagonal are read), executed by the 128 threads of the intra warpgroup (t = 0..127).
// T is written over A in place (out.Tm == A): every block of A is read before T's block at the
// same place is written (registers, __syncwarp, or the barrier inside the 16 -> 32 step), and the
// last step's lower-left block goes to the bf16 tiles only.
// Warp w owns the 16 x 16 diagonal block w: its two 8 x 8 diagonal sub-blocks are inverted by
// column-parallel forward substitution (lane = column, running sums, 7 dependent steps), then one
// doubling step T_ba = -T_bb (A_ba T_aa) joins them.  The 16 -> 32 and 32 -> 64 merges run the
// same step on mma.sync TF32 (T is rounded to bf16 afterwards, so TF32 products stay below that
// rounding).  Every entry of the lower triangle is written exactly once, through `out`; entries
// above the diagonal are never written (the caller keeps them zero in the bf16 copies).
__device__ void solve_unit_lower(const float *A, const TOut &out, float *__restrict__ XS, int t, int bar_id)
{
    float *Tm = out.Tm;
    const int w = t >> 5, lane = t & 31, g = lane >> 2, tq = lane & 3;
    float *xs = XS + w * 256;
    {
        const int o = 16 * w;
        if (lane < 16) {
            const int sb = o + 8 * (lane >> 3), c = lane & 7;
            const float bc = out.bet[sb + c], gc = out.gam[sb + c], vc = out.vfac(sb + c, bc);
            float a[8][8];  // the block's strictly lower part, read before any lane writes T there
#pragma unroll
            for (int r = 1; r < 8; ++r)
#pragma unroll
                for (int i = 0; i < r; ++i) a[r][i] = A[(sb + r) * LDF + sb + i];
            float p[8], x[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) p[r] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                x[i] = (i < c) ? 0.f : (i == c ? 1.f : -p[i]);
#pragma unroll
                for (int r = i + 1; r < 8; ++r) p[r] = fmaf(a[r][i], x[i], p[r]);
            }
            __syncwarp(0xffffu);
#pragma unroll
            for (int r = 0; r < 8; ++r)
                if (r >= c) out.put(sb + r, sb + c, x[r], vc, bc, gc);
        }
        __syncwarp();
#pragma unroll
        for (int q0 = 0; q0 < 64; q0 += 32) {
            const int q = q0 + lane, i = q >> 3, j = q & 7;
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k >= j) acc = fmaf(A[(o + 8 + i) * LDF + o + k], Tm[(o + k) * LDF + o + j], acc);
            xs[i * 8 + j] = acc;
        }
        __syncwarp();
        const float bj = out.bet[o + (lane & 7)], gj = out.gam[o + (lane & 7)], vj = out.vfac(o + (lane & 7), bj);
#pragma unroll
        for (int q0 = 0; q0 < 64; q0 += 32) {
            const int q = q0 + lane, i = q >> 3, j = q & 7;
            float acc = xs[i * 8 + j];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < i) acc = fmaf(Tm[(o + 8 + i) * LDF + o + 8 + k], xs[k * 8 + j], acc);
            out.put(o + 8 + i, o + j, -acc, vj, bj, gj);
        }
    }
    named_bar(bar_id, 128);
    // ---- 16 -> 32: pair p = w/2 (blocks 2p, 2p+1), output column tile nt = w%2 ----
    {
        const int p = w >> 1, nt = w & 1, oa = 32 * p, ob = oa + 16, n = oa + 8 * nt + g;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            if (kk < nt) continue;
            const int k0 = oa + 8 * kk + tq, k1 = k0 + 4;
            mma_tf32(d, tf(A[(ob + g) * LDF + k0]), tf(A[(ob + g + 8) * LDF + k0]),
                     tf(A[(ob + g) * LDF + k1]), tf(A[(ob + g + 8) * LDF + k1]),
                     tf(k0 >= n ? Tm[k0 * LDF + n] : 0.f), tf(k1 >= n ? Tm[k1 * LDF + n] : 0.f));
        }
        xs[g * 8 + 2 * tq] = d[0];
        xs[g * 8 + 2 * tq + 1] = d[1];
        xs[(g + 8) * 8 + 2 * tq] = d[2];
        xs[(g + 8) * 8 + 2 * tq + 1] = d[3];
        // both warps of the pair have read A's block before T's block replaces it
        named_bar(bar_id, 128);
        float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int k0 = 8 * kk + tq, k1 = k0 + 4;
            mma_tf32(e, tf(k0 <= g ? Tm[(ob + g) * LDF + ob + k0] : 0.f),
                     tf(k0 <= g + 8 ? Tm[(ob + g + 8) * LDF + ob + k0] : 0.f),
                     tf(k1 <= g ? Tm[(ob + g) * LDF + ob + k1] : 0.f),
                     tf(k1 <= g + 8 ? Tm[(ob + g + 8) * LDF + ob + k1] : 0.f),
                     tf(xs[k0 * 8 + g]), tf(xs[k1 * 8 + g]));
        }
        const int c0 = oa + 8 * nt + 2 * tq;
        const float b0 = out.bet[c0], b1 = out.bet[c0 + 1], g0 = out.gam[c0], g1 = out.gam[c0 + 1];
        const float u0 = out.vfac(c0, b0), u1 = out.vfac(c0 + 1, b1);
        out.put2(ob + g, c0, -e[0], -e[1], u0, u1, b0, b1, g0, g1, true);
        out.put2(ob + g + 8, c0, -e[2], -e[3], u0, u1, b0, b1, g0, g1, true);
    }
    named_bar(bar_id, 128);
    // ---- 32 -> 64: warp w takes output column tile wt = 3 - w ----
    {
        const int wt = 3 - w;
        const int n = 8 * wt + g;
        float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk < wt) continue;
            const int k0 = 8 * kk + tq, k1 = k0 + 4;
            const uint32_t b0 = tf(k0 >= n ? Tm[k0 * LDF + n] : 0.f);
            const uint32_t b1 = tf(k1 >= n ? Tm[k1 * LDF + n] : 0.f);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int r = 32 + 16 * mt + g;
                mma_tf32(d[mt], tf(A[r * LDF + k0]), tf(A[(r + 8) * LDF + k0]), tf(A[r * LDF + k1]),
                         tf(A[(r + 8) * LDF + k1]), b0, b1);
            }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            xs[(16 * mt + g) * 8 + 2 * tq] = d[mt][0];
            xs[(16 * mt + g) * 8 + 2 * tq + 1] = d[mt][1];
            xs[(16 * mt + g + 8) * 8 + 2 * tq] = d[mt][2];
            xs[(16 * mt + g + 8) * 8 + 2 * tq + 1] = d[mt][3];
        }
        __syncwarp();
        const int c0 = 8 * wt + 2 * tq;
        const float bb0 = out.bet[c0], bb1 = out.bet[c0 + 1], gg0 = out.gam[c0], gg1 = out.gam[c0 + 1];
        const float uu0 = out.vfac(c0, bb0), uu1 = out.vfac(c0 + 1, bb1);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float e[4] = {0.f, 0.f, 0.f, 0.f};
            const int rl = 16 * mt + g, rh = rl + 8;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                if (kk > 2 * mt + 1) continue;
                const int k0 = 8 * kk + tq, k1 = k0 + 4;
                mma_tf32(e, tf(k0 <= rl ? Tm[(32 + rl) * LDF + 32 + k0] : 0.f),
                         tf(k0 <= rh ? Tm[(32 + rh) * LDF + 32 + k0] : 0.f),
                         tf(k1 <= rl ? Tm[(32 + rl) * LDF + 32 + k1] : 0.f),
                         tf(k1 <= rh ? Tm[(32 + rh) * LDF + 32 + k1] : 0.f),
                         tf(xs[k0 * 8 + g]), tf(xs[k1 * 8 + g]));
            }
            out.put2(32 + rl, c0, -e[0], -e[1], uu0, uu1, bb0, bb1, gg0, gg1, false);
            out.put2(32 + rh, c0, -e[2], -e[3], uu0, uu1, bb0, bb1, gg0, gg1, false);
        }
    }
}

// Gate forms of the fused prologue (valid = the row lies inside the sequence; padded rows keep the
// exact zeros of log alpha and beta that make them contribute nothing).
__device__ __forceinline__ float prologue_log_alpha(float a, bool valid, float a_scale)
{
    if (!valid) return 0.f;
    if (a == INFINITY) return -INFINITY;  // an exact reset
    const float sp = a > 0.f ? a + log1pf(expf(-a)) : log1pf(expf(a));
    return -a_scale * sp;
}
__device__ __forceinline__ float prologue_beta(float b, bool valid, float b_scale)
{
    return valid ? b_scale / (1.f + expf(-b)) : 0.f;
}

// Divide bf16 row `row` of a swizzled tile (NBLK blocks of 64 features at a 16 KB stride) by
// sqrt(sum of squares + kNormEps), in fp32, rounding back to bf16.
template <int NBLK>
__device__ __forceinline__ void normalize_row_bf16(unsigned char *tile, int row)
{
    uint4 w[NBLK * 8];
    float ss = 0.f;
#pragma unroll
    for (int b = 0; b < NBLK; ++b)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            w[b * 8 + c] = *reinterpret_cast<const uint4 *>(tile + b * 16384 + row * 128 + ((c ^ (row & 7)) << 4));
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w[b * 8 + c]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
            }
        }
    const float sc = rsqrtf(ss + kNormEps);
#pragma unroll
    for (int b = 0; b < NBLK; ++b)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&w[b * 8 + c]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                h[e] = __floats2bfloat162_rn(f.x * sc, f.y * sc);
            }
            *reinterpret_cast<uint4 *>(tile + b * 16384 + row * 128 + ((c ^ (row & 7)) << 4)) = w[b * 8 + c];
        }
}

// Scale row r (64 bf16 = 128 swizzled bytes, 8 chunks of 16 B) of a tile by s: the caller owns
// chunks [c0, c1) counted from position row % 8, so that the threads of a warp (consecutive rows)
// touch 8 different bank groups at every step.  Packed bf16x2 multiplies (s rounded to bf16).
__device__ __forceinline__ void scale_row_bf16(unsigned char *tile, int row, float s, int c0, int c1)
{
    const __nv_bfloat162 s2 = __float2bfloat162_rn(s);
#pragma unroll 2
    for (int c = c0; c < c1; ++c) {
        uint4 *p = reinterpret_cast<uint4 *>(tile + row * 128 + (((c + row) & 7) << 4));
        uint4 w = *p;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __hmul2(h[e], s2);
        *p = w;
    }
}

// PRO: fused prologue (kFlagPrologue), PH: fused complex-phase prologue (kFlagPhase), separate
// instantiations so that the plain path carries none of their code.
template <int DK, int DV, bool PRO, bool PH = false>
__global__ void __launch_bounds__(TcCfg<DK, DV, PH>::THREADS, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const float *__restrict__ log_alpha,
                    const float *__restrict__ beta, const float *__restrict__ S0,
                    __nv_bfloat16 *__restrict__ out, float *__restrict__ S_final,
                    const int32_t *__restrict__ cu_seqlens, int T, int H, int flags, float a_scale,
                    float b_scale, int G)
{
    using L = TcCfg<DK, DV, PH>;
    constexpr int NS = L::NS;
    constexpr int NI = L::NI;
    constexpr int NB = L::NB;
    constexpr int NBO = L::NBO;
    constexpr bool TA = L::TA;
    // TA: U^T enters the state and output MMAs as two bf16 parts (hi + lo)
    constexpr bool kUSplit = GDN_U_SPLIT;
    using B = Bars<NS, NI, NB, NBO>;
    // gam Q and lam K are formed in place by the intra side, which runs ahead of the chain
    constexpr bool kChainScales = false;
    // Unrolling of the intra side's MMA issue loops: rolled at value head 128, where the smaller
    // code (fewer instruction-cache misses among the three roles) measured faster, unrolled at 64,
    // where it did not
    constexpr int kIssueUnroll = TA ? 1 : 8;
    extern __shared__ unsigned char smem_raw[];
    // 1024-aligned base by pointer arithmetic on the shared array, so that the compiler keeps
    // every access below in the shared address space
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC);
    int *abort_flag = reinterpret_cast<int *>(sm + L::MISC + 4);
    const Ctl ctl{bars, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    int s = blockIdx.z;
    if (flags & kFlagLongestFirst) {  // gridDim.z <= THREADS sequences: thread i ranks sequence i
        int *pick = reinterpret_cast<int *>(sm + L::MISC + 8);
        const int nseq = (int)gridDim.z;
        if (tid < nseq) {
            const int mine = cu_seqlens[tid + 1] - cu_seqlens[tid];
            int rank = 0;
            for (int o = 0; o < nseq; ++o) {
                const int other = cu_seqlens[o + 1] - cu_seqlens[o];
                rank += (other > mine) || (other == mine && o < tid);
            }
            if (rank == (int)blockIdx.z) *pick = tid;
        }
        __syncthreads();
        s = *pick;
    }
    const int hq = G == 1 ? h : h / G;  // q/k head of value head h (G value heads share one q/k head)
    long tok0, len;
    if (cu_seqlens) {
        tok0 = cu_seqlens[s];
        len = (long)cu_seqlens[s + 1] - tok0;
    } else {
        tok0 = (long)s * T;
        len = T;
    }
    const int nchunks = (int)((len + CH - 1) / CH);
    // value columns col0 .. col0 + DV - 1 of a row of ldv: a wider value head runs as gridDim.x
    // column blocks, one CTA each (value columns do not interact in the recurrence)
    const int col0 = (int)blockIdx.x * DV;
    const size_t ldv = (size_t)gridDim.x * DV;
    const size_t sbase = ((size_t)s * H + h) * (size_t)DK * ldv + col0;

    if (tid == 0) {
        for (int i = 0; i < L::NBAR; ++i) mbar_init(&bars[i], (i >= B::gfull && i < B::gfull + NS) ? 32 : 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto gates = [&](int stage) { return reinterpret_cast<float *>(sm + L::GT + stage * L::GT_STAGE); };
    // Loads of chunk c into K/Q stage c % NS: gates by cp.async from the 32 lanes of warp 0
    // (rows past the sequence end are zero-filled), K and Q tiles by TMA from thread 0.
    auto load_kq = [&](int c) {
        const int st = c % NS;
        const long tk = tok0 + (long)c * CH;
        const int n = (int)min((long)CH, len - (long)c * CH);
        float *gv = gates(st);
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
            const int r = lane + 32 * k2;
            const size_t off = (size_t)(tk + min(r, n - 1)) * H + h;
            cp_async_4(&gv[r], log_alpha + off, r < n ? 4u : 0u);
            cp_async_4(&gv[4 * CH + r], beta + off, r < n ? 4u : 0u);
        }
        cp_async_mbar_arrive(&bars[B::gfull + st]);
        if (lane == 0 && !ctl.aborted()) {
            mbar_arrive_expect_tx(&bars[B::kq_full + st], L::KQ_STAGE);
            unsigned char *kq = sm + L::KQ + st * L::KQ_STAGE;
            if constexpr (PH) {
                // fp32 rows of 64 (32 complex pairs) as two 32-float blocks: K at +0, Q at +16 KB
                for (int hb = 0; hb < 2; ++hb) {
                    tma_load_3d(kq + hb * 8192, &tmK, &bars[B::kq_full + st], hb * 32, hq, (int)tk);
                    tma_load_3d(kq + 16384 + hb * 8192, &tmQ, &bars[B::kq_full + st], hb * 32, hq, (int)tk);
                }
            } else {
                for (int kb = 0; kb < DK / 64; ++kb) {
                    tma_load_3d(kq + kb * 16384, &tmK, &bars[B::kq_full + st], kb * 64, hq, (int)tk);
                    tma_load_3d(kq + kb * 16384 + 8192, &tmQ, &bars[B::kq_full + st], kb * 64, hq, (int)tk);
                }
            }
        }
    };
    const bool v_zero = (flags & kFlagVZero) != 0;
    const bool want_out = out != nullptr;
    // V tile of chunk c into buffer c % NB (issued once the U~ MMA of chunk c - NB has read it)
    auto load_v = [&](int c) {
        if (ctl.aborted() || v_zero) return;
        const int tk = (int)(tok0 + (long)c * CH);
        uint64_t *vb_bar = &bars[B::v_full + c % NB];
        mbar_arrive_expect_tx(vb_bar, L::V_BUF);
        for (int vb = 0; vb < DV / 64; ++vb)
            tma_load_3d(sm + L::V + (c % NB) * L::V_BUF + vb * 8192, &tmV, vb_bar, col0 + vb * 64, h, tk);
    };
    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
        }
        for (int c = 0; c < min(nchunks, NS); ++c) load_kq(c);
    }
    if (tid == 0)
        for (int c = 0; c < min(nchunks, NB); ++c) load_v(c);

    if (warp >= 4) {
        // ======================= intra warpgroup(s): chunks wg, wg + NI, ... =======================
        const int wg = (warp - 4) >> 2;
        const int t = tid - 128 * (1 + wg), wi = t >> 5;
        const int bar_id = 2 + wg;
        const uint32_t tl = tmem + ((uint32_t)(wi * 32) << 16);
        const uint32_t tG = L::T_G + wg * 64;  // Gram accumulator, then W^T
        unsigned char *wsm = sm + L::WG0 + wg * L::WG_BYTES;
        unsigned char *TBs = wsm + L::W_TB, *TGs = wsm + L::W_TG, *WTs = wsm + L::W_WT;
        float *AT = reinterpret_cast<float *>(wsm + L::W_AT);  // decays, then A, then T (in place)
        float *XSm = reinterpret_cast<float *>(wsm + L::W_XS);
        // entries above the diagonal of T diag(b..) stay zero (the solve writes the lower part)
        for (int i = t; i < 2 * 8192 / 16; i += 128)
            reinterpret_cast<uint4 *>(TBs)[i] = make_uint4(0u, 0u, 0u, 0u);
        for (int c = wg; c < nchunks; c += NI) {
            const int st = c % NS;
            const int kc = c / NI;  // this warpgroup's chunk count
            float *gv = gates(st);
            float *graw = gv, *Gs = gv + CH, *gam = gv + 2 * CH, *lam = gv + 3 * CH, *bet = gv + 4 * CH;
            int *last = reinterpret_cast<int *>(gv + 5 * CH);
            float *gC = gv + 6 * CH;
            unsigned char *Kt = sm + L::KQ + st * L::KQ_STAGE;  // K at +0, Q at +8192 per block
            // ---- Gram matrices [K; Q] K^T (issued first: they need no gates, so the scan below
            //      runs while they are in flight) ----
            ctl.wait(B::kq_full + st, (c / NS) & 1);
            if (PH) {
                // fp32 (re, im) rows -> bf16 rows of k~ / sqrt(dk) (threads 0-63) and q~ / dk
                // (threads 64-127), real parts in columns 0-31 and imaginary parts in 32-63,
                // written over the fp32 rows once all of them have been read
                const int r = t & 63;
                const bool isq = t >= 64;
                const unsigned char *src = Kt + (isq ? 16384 : 0);
                const float sc = isq ? 1.f / 32.f : 1.f / kPhaseSqrtDk;
                float x[64];
#pragma unroll
                for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float4 f = *reinterpret_cast<const float4 *>(src + hb * 8192 + r * 128 +
                                                                            (((u ^ r) & 7) << 4));
                        const int i = 16 * hb + 2 * u;  // complex index of f.x, f.y
                        x[i] = f.x * sc;
                        x[32 + i] = f.y * sc;
                        x[i + 1] = f.z * sc;
                        x[33 + i] = f.w * sc;
                    }
                named_bar(bar_id, 128);
                st_row_bf16_sw128(Kt + (isq ? 8192 : 0), r, x);
                fence_proxy_async_smem();
                named_bar(bar_id, 128);
            }
            if (PRO) {
                // fused prologue: unit rows of K (threads 0-63) and Q (threads 64-127)
                normalize_row_bf16<DK / 64>(Kt + (t >= 64 ? 8192 : 0), t & 63);
                fence_proxy_async_smem();
                named_bar(bar_id, 128);
            }
            if (t == kIssuer && !ctl.aborted()) {
                tc_fence_after();
                constexpr uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll(kIssueUnroll)
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t a = smem_u32(Kt + (kk >> 2) * 16384 + (kk & 3) * 32);
                    mma_bf16(tmem + tG, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), id, kk > 0);
                }
                mma_commit(&bars[B::gram + wg]);
            }
            // ---- gates: segmented scan of log_alpha (restarts at exact resets) ----
            if (wi == scan_warp(wg)) {
                ctl.wait(B::gfull + st, (c / NS) & 1);
                const int r0 = 2 * lane, r1 = r0 + 1;
                float g0 = graw[r0], g1 = graw[r1];
                if (PRO) {
                    const int n = (int)min((long)CH, len - (long)c * CH);
                    g0 = prologue_log_alpha(g0, r0 < n, a_scale);
                    g1 = prologue_log_alpha(g1, r1 < n, a_scale);
                    bet[r0] = prologue_beta(bet[r0], r0 < n, b_scale);
                    bet[r1] = prologue_beta(bet[r1], r1 < n, b_scale);
                }
                if (PH) {
                    // U~ factor beta sqrt(dk) (= b v / V), then b = beta / lam (lam > 0; padded rows
                    // hold beta = 0 and log lam = 0)
                    float *bv = gv + 7 * CH;
                    bv[r0] = bet[r0] * kPhaseSqrtDk;
                    bv[r1] = bet[r1] * kPhaseSqrtDk;
                    bet[r0] *= expf(-g0);
                    bet[r1] *= expf(-g1);
                }
                const bool f0 = (g0 == -INFINITY), f1 = (g1 == -INFINITY);
                const float v0 = f0 ? 0.f : g0, v1 = f1 ? 0.f : g1;
                // inclusive pair value and reset flag, then a segmented warp scan over lanes
                float a = f1 ? v1 : v0 + v1;
                int fa = (f0 || f1) ? 1 : 0;
                int li = f1 ? r1 : (f0 ? r0 : -1);
#pragma unroll 1
                for (int off = 1; off < 32; off <<= 1) {
                    const float ab = __shfl_up_sync(0xffffffffu, a, off);
                    const int fb = __shfl_up_sync(0xffffffffu, fa, off);
                    const int lb = __shfl_up_sync(0xffffffffu, li, off);
                    if (lane >= off) {
                        a = fa ? a : ab + a;
                        fa |= fb;
                        li = max(li, lb);
                    }
                }
                float ex = __shfl_up_sync(0xffffffffu, a, 1);
                int lex = __shfl_up_sync(0xffffffffu, li, 1);
                if (lane == 0) { ex = 0.f; lex = -1; }
                // sums in the log2 domain, so every decay below is a single exp2
                constexpr float kLog2e = 1.4426950408889634f;
                const float G0 = f0 ? 0.f : ex + v0;
                const float G1 = f1 ? 0.f : G0 + v1;
                const float H0 = G0 * kLog2e, H1 = G1 * kLog2e;
                const int L0 = f0 ? r0 : lex;
                const int L1 = f1 ? r1 : L0;
                Gs[r0] = H0; Gs[r1] = H1;
                last[r0] = L0; last[r1] = L1;
                __syncwarp();
                const int l63 = last[CH - 1];
                const float G63 = Gs[CH - 1];
                gam[r0] = L0 >= 0 ? 0.f : exp2f(H0);
                gam[r1] = L1 >= 0 ? 0.f : exp2f(H1);
                lam[r0] = l63 > r0 ? 0.f : exp2f(G63 - H0);
                lam[r1] = l63 > r1 ? 0.f : exp2f(G63 - H1);
                __syncwarp();
                if (lane == 0) {
                    gC[0] = gam[CH - 1];
                    ctl.arrive(B::gready + st);
                }
            }
            named_bar(bar_id, 128);
            // ---- decays Gam[r][i] (lower triangle; zero across a reset) into the A/T buffer ----
            {
                const int r = t & 63, c0 = (t >> 6) * 32;
                const float Gr = Gs[r];
                const int lr = last[r];
                float *gm = AT + r * LDF + c0;
#pragma unroll 2
                for (int j4 = 0; j4 < 32; j4 += 4) {
                    const float4 g4 = *reinterpret_cast<const float4 *>(&Gs[c0 + j4]);
                    const float gi[4] = {g4.x, g4.y, g4.z, g4.w};
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = c0 + j4 + e;
                        const float ex = ex2_approx(Gr - gi[e]);
                        v[e] = (i <= r && lr <= i) ? ex : 0.f;
                    }
                    *reinterpret_cast<float4 *>(gm + j4) = make_float4(v[0], v[1], v[2], v[3]);
                }
            }
            ctl.wait(B::gram + wg, kc & 1);
            // the stage's P tile is free once the output MMA of chunk c - NS has read it
            if (c >= NS) ctl.wait(B::cdone + st, ((c / NS) - 1) & 1);
            tc_fence_after();
            named_bar(bar_id, 128);
            {
                // A = diag(b) (Gam o K K^T) (fp32; its diagonal and upper part are never read),
                // P = Gam o Q K^T (bf16) and, unless the chain does it, gam Q in place (no MMA
                // reads Q unscaled any more)
                float x[64];
                tmem_ld32(tl + tG, *reinterpret_cast<float(*)[32]>(&x[0]));
                tmem_ld32(tl + tG + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
                tmem_wait_ld();
                const int r = t & 63;
                const bool isq = t >= 64;
                const float sc = isq ? 1.f : bet[r];
#pragma unroll
                for (int i4 = 0; i4 < CH; i4 += 4) {
                    const float4 gm = *reinterpret_cast<const float4 *>(&AT[r * LDF + i4]);
                    x[i4] *= gm.x * sc;
                    x[i4 + 1] *= gm.y * sc;
                    x[i4 + 2] *= gm.z * sc;
                    x[i4 + 3] *= gm.w * sc;
                }
                // both threads of row r have read its decays before A overwrites them
                named_bar(bar_id, 128);
                if (isq) {
                    st_row_bf16_sw128(sm + L::PM + st * 8192, r, x);
                } else {
#pragma unroll
                    for (int i = 0; i < CH; i += 4)
                        *reinterpret_cast<float4 *>(&AT[r * LDF + i]) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
                }
                if (!kChainScales) {
                    if (DK == 64) scale_row_bf16(Kt + 8192, r, gam[r], (t >> 6) * 4, (t >> 6) * 4 + 4);
                    else scale_row_bf16(Kt + (t >> 6) * 16384 + 8192, r, gam[r], 0, 8);
                }
            }
            tc_fence_before();
            // this warpgroup's previous chunk: its W^T and T diag(b..) tiles must have been read
            if (kc >= 1) ctl.wait(B::tfree + wg, (kc - 1) & 1);
            if (kc >= 1) {
                // W^T of the previous chunk sits in T diag(b gam) (dk = 64) or in both T tiles
                // (dk = 128): clear every 16-byte chunk from the diagonal block rightwards (the
                // solve then writes the lower part)
                constexpr int kTiles = DK / 64;
#pragma unroll 1
                for (int i = t; i < kTiles * 64 * 8; i += 128) {
                    const int r = (i >> 3) & 63, cb = i & 7;
                    unsigned char *tile = (kTiles == 2 && i >= 64 * 8) ? TGs : (kTiles == 2 ? TBs : TGs);
                    if (cb >= (r >> 3))
                        *reinterpret_cast<uint4 *>(tile + r * 128 + ((cb ^ (r & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            named_bar(bar_id, 128);
            // ---- T = (I + A)^{-1}, written with the bf16 rows of T diag(b), T diag(b gam) ----
            solve_unit_lower(AT, TOut{AT, TBs, TGs, bet, gam, PH ? gv + 7 * CH : nullptr}, XSm, t, bar_id);
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(bar_id, 128);
            // ---- WY products: U~^T = V^T (T diag b)^T into the chunk's U slot and
            //      W^T = K^T (T diag(b gam))^T over the Gram accumulator ----
            if (t == kIssuer) {
                if (!v_zero) ctl.wait(B::v_full + c % NB, (c / NB) & 1);
                // TA: the slot is this warpgroup's; the chain's state and output MMAs of its
                // previous chunk read U^T from it
                if (TA && kc >= 1) ctl.wait(B::ufree + wg, (kc - 1) & 1);
                if (!ctl.aborted()) {
                    tc_fence_after();
                    constexpr uint32_t idU = idesc_bf16(DV, 64, 1, 0);
                    // TA: -W^T (A operand negated), so that the chain's U MMA (A operand in tensor
                    // memory) adds S^T (-W^T) onto U~^T without negating its A operand
                    constexpr uint32_t idW = idesc_bf16(DK, 64, 1, 0, TA ? 1 : 0);
                    if (!v_zero) {
#pragma unroll(kIssueUnroll)
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16(tmem + L::T_U + (TA ? wg : st) * 64,
                                     sdesc_sw128(smem_u32(sm + L::V + (c % NB) * L::V_BUF + kk * 2048), 8192, 1024),
                                     sdesc_sw128(smem_u32(TBs + kk * 32), 16, 1024), idU, kk > 0);
                    }
#pragma unroll(kIssueUnroll)
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + tG, sdesc_sw128(smem_u32(Kt + kk * 2048), 16384, 1024),
                                 sdesc_sw128(smem_u32(TGs + kk * 32), 16, 1024), idW, kk > 0);
                    mma_commit(&bars[B::uw + wg]);
                }
            }
            ctl.wait(B::uw + wg, kc & 1);
            tc_fence_after();
            if (t == kIssuer && c + NB < nchunks) load_v(c + NB);  // the U~ MMA has read V
            {
                // W^T rows (one per feature; -W^T with TA) to shared memory in bf16, then (unless the
                // chain does it) lam K in place: the W MMA has read K unscaled
                if (DK == 128) {
                    float x[64];
                    tmem_ld32(tl + tG, *reinterpret_cast<float(*)[32]>(&x[0]));
                    tmem_ld32(tl + tG + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
                    tmem_wait_ld();
                    st_row_bf16_sw128(WTs, t, x);
                } else {
                    // M = 64 layout: threads lane and lane + 16 take the two halves of a row
                    float x[32];
                    tmem_ld16x2_32<32>(tl + tG, x);
                    tmem_wait_ld();
                    st_half_row_bf16_sw128(WTs, wi * 16 + (t & 15), (t >> 4) & 1, x);
                }
                if (!kChainScales) {
                    if (DK == 64) scale_row_bf16(Kt, t & 63, lam[t & 63], (t >> 6) * 4, (t >> 6) * 4 + 4);
                    else scale_row_bf16(Kt + (t >> 6) * 16384, t & 63, lam[t & 63], 0, 8);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(bar_id, 128);
            if (t == 0) ctl.arrive(B::tready + st);
        }
    } else {
        // ======================= chain warpgroup =======================
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        // dv = 64 puts S^T and U^T in the M = 64 accumulator layout (rows at lanes r % 16 of each
        // warp quadrant); every row is then split between threads `lane` and `lane + 16`, which
        // take the first and the second half of its columns (16x32bx2 TMEM accesses)
        constexpr bool kHalf = DV == 64;
        const int j = kHalf ? warp * 16 + (lane & 15) : tid;  // value column = S^T row
        const int hh = kHalf ? (lane >> 4) : 0;               // column half of that row
        // 32-feature blocks cb of S^T row j held by this thread, as the k-th of its loads
        constexpr int kSB = kHalf ? DK / 64 : DK / 32;
        auto s_block = [&](int k) { return kHalf ? k + hh * (DK / 64) : k; };
        auto ld_state = [&](int k, float (&x)[32]) {
            if (kHalf) tmem_ld16x2_32<DK / 2>(tl + L::T_S + 32 * k, x);
            else tmem_ld32(tl + L::T_S + 32 * k, x);
        };
        auto st_state = [&](int k, const float (&x)[32]) {
            if (kHalf) tmem_st16x2_32<DK / 2>(tl + L::T_S + 32 * k, x);
            else tmem_st32(tl + L::T_S + 32 * k, x);
        };
        // bf16 copy of S^T row j, features 32cb .. 32cb+31
        auto store_state_bf16 = [&](int cb, const float (&x)[32]) {
            unsigned char *stt = sm + L::ST + (cb >> 1) * (DV * 128);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int chunk = (cb & 1) * 4 + cc;
                uint4 w;
                w.x = pack_bf16x2(x[8 * cc + 0], x[8 * cc + 1]);
                w.y = pack_bf16x2(x[8 * cc + 2], x[8 * cc + 3]);
                w.z = pack_bf16x2(x[8 * cc + 4], x[8 * cc + 5]);
                w.w = pack_bf16x2(x[8 * cc + 6], x[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(stt + j * 128 + (((chunk ^ (j & 7)) & 7) << 4)) = w;
            }
        };
        // Output rows of chunk c: O (M = 64 tokens, N = DV) sits in lanes 0..15 of each warp
        // quadrant, row 16w + lane % 16; threads lane and lane + 16 store the two halves of a row.
        // The chunk's P tile is released to the intra side as soon as the output MMA has completed.
        auto out_epilogue = [&](int c) {
            const long tk = tok0 + (long)c * CH;
            const int n = (int)min((long)CH, len - (long)c * CH);
            if (want_out) {
                ctl.wait(B::o + c % NBO, (c / NBO) & 1);
                tc_fence_after();
                if (tid == 0) ctl.arrive(B::cdone + (c % NS));
                const int r = 16 * warp + (lane & 15);
                __nv_bfloat16 *op = out + ((size_t)(tk + r) * H + h) * ldv + col0 + (lane >> 4) * (DV / 2);
#pragma unroll 1
                for (int cb = 0; cb < DV / 64; ++cb) {
                    float o[32];
                    tmem_ld16x2_32<DV / 2>(tl + L::T_O + (c % NBO) * DV + cb * 32, o);
                    tmem_wait_ld();
                    if (r < n) {
                        uint4 *dst = reinterpret_cast<uint4 *>(op + cb * 32);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 w;
                            w.x = pack_bf16x2(o[8 * q + 0], o[8 * q + 1]);
                            w.y = pack_bf16x2(o[8 * q + 2], o[8 * q + 3]);
                            w.z = pack_bf16x2(o[8 * q + 4], o[8 * q + 5]);
                            w.w = pack_bf16x2(o[8 * q + 6], o[8 * q + 7]);
                            dst[q] = w;
                        }
                    }
                }
                tc_fence_before();
            } else if (tid == 0) {
                ctl.arrive(B::cdone + (c % NS));
            }
            named_bar(1, 128);
        };
        if constexpr (TA) {
            // ---- value head 128: thread j = value column = TMEM lane j.  The bf16 copy of S^T
            //      and U^T are the A operands of the chain's MMAs, read from tensor memory; the
            //      outputs are formed as O^T (64 token columns) ----
            // S^T row j (64 features) as 32 packed bf16 pairs into the copy at column 32 kb
            auto st_state_bf16 = [&](int kb, const float *x) {
                float p[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) p[i] = __uint_as_float(pack_bf16x2(x[2 * i], x[2 * i + 1]));
                tmem_st32(tl + L::T_SB + 32 * kb, *reinterpret_cast<const float(*)[32]>(p));
            };
            // Outputs of chunk c: O^T row j holds column j of the chunk's 64 token rows.  They
            // leave through a bf16 tile in shared memory -- thread j writes column j (16-byte
            // units XOR-swizzled by row), then each thread stores half a row with 16-byte stores
            // -- the chunk's own K/Q stage with one O buffer (free from its state MMA's
            // completion until the next load is issued into it), a tile of its own with two.
            auto out_epilogue_staged = [&](int c, unsigned char *buf) {
                if (!want_out) return;
                const long tk = tok0 + (long)c * CH;
                const int n = (int)min((long)CH, len - (long)c * CH);
                // per warp: its 32 lanes as two halves of 16, the 64 token columns as four groups
                // of 16; a 16 x 16 block is loaded in fragments and stored transposed as four
                // 8 x 8 bf16 matrices (rows = tokens), thread `lane` addressing row lane % 8 of
                // matrix lane / 8
                const int mi = lane >> 3, mrow = lane & 7;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t f[4][8];  // the four loads first, then one wait
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        tmem_ld16x256b_x2(tmem + ((uint32_t)(warp * 32 + 16 * hf) << 16) + L::T_O + (c % NBO) * 64 + 16 * g,
                                          f[g]);
                    tmem_wait_ld();
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int r = 16 * g + 8 * (mi >> 1) + mrow;        // token row of this address
                        const int col = warp * 32 + 16 * hf + 8 * (mi & 1);  // first value column
                        stmatrix_x4_trans(smem_u32(buf + r * 256 + (((col >> 3) ^ (r & 15)) << 4)),
                                          pack_bf16x2(__uint_as_float(f[g][0]), __uint_as_float(f[g][1])),
                                          pack_bf16x2(__uint_as_float(f[g][2]), __uint_as_float(f[g][3])),
                                          pack_bf16x2(__uint_as_float(f[g][4]), __uint_as_float(f[g][5])),
                                          pack_bf16x2(__uint_as_float(f[g][6]), __uint_as_float(f[g][7])));
                    }
                }
                named_bar(1, 128);
                // rows to global memory: eight threads per 256-byte row, each taking 16-byte units
                // (tid & 7) and (tid & 7) + 8, so a warp stores four rows with full 128-byte runs
#pragma unroll 1
                for (int p = 0; p < 4; ++p) {
                    const int r = 16 * p + (tid >> 3);
                    if (r < n) {
                        uint4 *dst = reinterpret_cast<uint4 *>(out + ((size_t)(tk + r) * H + h) * ldv + col0);
#pragma unroll
                        for (int s8 = 0; s8 < 2; ++s8) {
                            const int u = (tid & 7) + 8 * s8;
                            dst[u] = *reinterpret_cast<const uint4 *>(buf + r * 256 + ((u ^ (r & 15)) << 4));
                        }
                    }
                }
            };
            if (nchunks > 0) {
                // initial state: fp32 S^T row j pre-scaled by gam_C of chunk 0, and its bf16 copy
                ctl.wait(B::gready + 0, 0);
                const float g0 = gates(0)[6 * CH];
#pragma unroll 1
                for (int kb = 0; kb < DK / 64; ++kb) {
                    float x[64];
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        const int f = kb * 64 + i;
                        x[i] = (flags & kFlagS0Identity) ? (f == j ? 1.f : 0.f)
                                                         : (S0 ? S0[sbase + (size_t)f * ldv + j] : 0.f);
                    }
                    st_state_bf16(kb, x);
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] *= g0;
                    tmem_st32(tl + L::T_S + 64 * kb, *reinterpret_cast<const float(*)[32]>(&x[0]));
                    tmem_st32(tl + L::T_S + 64 * kb + 32, *reinterpret_cast<const float(*)[32]>(&x[32]));
                }
                tmem_wait_st();
                tc_fence_before();
                named_bar(1, 128);
            }
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % NS, wu = c % NI;
                const uint32_t tO = tmem + L::T_O + (c % NBO) * 64;
                const uint32_t tU = tmem + L::T_U + wu * 64;  // lane 0: the MMAs' operand address
                unsigned char *Kt = sm + L::KQ + st * L::KQ_STAGE;
                const unsigned char *WTc = sm + L::WG0 + wu * L::WG_BYTES + L::W_WT;
                constexpr uint32_t idU = idesc_bf16(128, 64, 0, 1);   // B = -W^T rows (MN-major)
                constexpr uint32_t idO = idesc_bf16(128, 64, 0, 0);   // O^T: B = gam Q or P rows (K-major)
                constexpr uint32_t idS = idesc_bf16(128, DK, 0, 1);   // B = lam K (MN-major)
                ctl.wait(B::tready + st, (c / NS) & 1);
                if (tid == 0 && !ctl.aborted()) {
                    tc_fence_after();
                    // U^T = U~^T + S^T (-W^T), accumulated onto U~^T
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        mma_bf16_ta(tU, tmem + L::T_SB + 8 * kk, sdesc_sw128(smem_u32(WTc + kk * 2048), 16, 1024), idU,
                                    v_zero ? (kk > 0) : 1);
                    mma_commit(&bars[B::u]);
                    // O^T = S^T (gam Q)^T; its completion is covered by the state MMA's commit
                    if (want_out) {
#pragma unroll 1
                        for (int kk = 0; kk < DK / 16; ++kk)
                            mma_bf16_ta(tO, tmem + L::T_SB + 8 * kk,
                                        sdesc_sw128(smem_u32(Kt + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32), 16, 1024),
                                        idO, kk > 0);
                    }
                }
                ctl.wait(B::u, c & 1);
                tc_fence_after();
                if (tid == 0) ctl.arrive(B::tfree + wu);  // W^T of this chunk has been read
                {
                    // U^T row j: 64 fp32 -> 32 packed bf16 pairs, over the slot's first 32 columns
                    float x[64];
                    tmem_ld32(tl + L::T_U + wu * 64, *reinterpret_cast<float(*)[32]>(&x[0]));
                    tmem_ld32(tl + L::T_U + wu * 64 + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
                    tmem_wait_ld();
                    // U^T = hi + lo in two bf16 parts (hi over columns 0-31, lo over 32-63): the
                    // state and output MMAs then see U to about 16 bits instead of 8
                    float p[32], pl[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const uint32_t hi = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                        p[i] = __uint_as_float(hi);
                        const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
                        pl[i] = __uint_as_float(pack_bf16x2(x[2 * i] - h0, x[2 * i + 1] - h1));
                    }
                    tmem_st32(tl + L::T_U + wu * 64, *reinterpret_cast<const float(*)[32]>(p));
                    if (kUSplit) tmem_st32(tl + L::T_U + wu * 64 + 32, *reinterpret_cast<const float(*)[32]>(pl));
                    tmem_wait_st();
                }
                tc_fence_before();
                named_bar(1, 128);
                if (tid == 0 && !ctl.aborted()) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < (kUSplit ? 8 : 4); ++kk)  // S^T += (U_hi + U_lo)^T (lam K)
                        mma_bf16_ta(tmem + L::T_S, tU + 8 * kk,
                                    sdesc_sw128(smem_u32(Kt + (kk & 3) * 2048), 16384, 1024), idS, 1);
                    if (want_out) {
#pragma unroll 1
                        for (int kk = 0; kk < (kUSplit ? 8 : 4); ++kk)  // O^T += (U_hi + U_lo)^T P^T
                            mma_bf16_ta(tO, tU + 8 * kk,
                                        sdesc_sw128(smem_u32(sm + L::PM + st * 8192 + (kk & 3) * 32), 16, 1024), idO, 1);
                    }
                    mma_commit(&bars[B::s]);
                    if (NBO == 2) mma_commit(&bars[B::o + c % NBO]);
                }
                // two O buffers: the previous chunk's outputs leave while the state MMA runs
                if (NBO == 2 && c >= 1) {
                    ctl.wait(B::o + (c - 1) % NBO, ((c - 1) / NBO) & 1);
                    tc_fence_after();
                    out_epilogue_staged(c - 1, sm + L::OT);
                }
                ctl.wait(B::s, c & 1);
                tc_fence_after();
                if (tid == 0) {
                    ctl.arrive(B::cdone + st);  // P of this stage has been read
                    ctl.arrive(B::ufree + wu);  // the U slot has been read
                }
                if (NBO == 1) {
                    out_epilogue_staged(c, Kt);
                    // every thread has read the tile before the stage is reloaded by TMA
                    fence_proxy_async_smem();
                    named_bar(1, 128);
                }
                if (warp == 0 && c + NS < nchunks) load_kq(c + NS);
                {
                    // S_{c+1} = gam_C(c) S_c + increment is in TMEM: its bf16 copy, and the fp32
                    // state pre-scaled by gam_C of the next chunk
                    const bool more = c + 1 < nchunks;
                    float gn = 1.f;
                    if (more) {
                        ctl.wait(B::gready + (c + 1) % NS, ((c + 1) / NS) & 1);
                        gn = gates((c + 1) % NS)[6 * CH];
                    }
#pragma unroll 1
                    for (int kb = 0; kb < DK / 64; ++kb) {
                        float x[64];
                        tmem_ld32(tl + L::T_S + 64 * kb, *reinterpret_cast<float(*)[32]>(&x[0]));
                        tmem_ld32(tl + L::T_S + 64 * kb + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
                        tmem_wait_ld();
                        st_state_bf16(kb, x);
                        if (more) {
#pragma unroll
                            for (int i = 0; i < 64; ++i) x[i] *= gn;
                            tmem_st32(tl + L::T_S + 64 * kb, *reinterpret_cast<const float(*)[32]>(&x[0]));
                            tmem_st32(tl + L::T_S + 64 * kb + 32, *reinterpret_cast<const float(*)[32]>(&x[32]));
                        }
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                named_bar(1, 128);
            }
            if (NBO == 2 && nchunks > 0) {
                ctl.wait(B::o + (nchunks - 1) % NBO, ((nchunks - 1) / NBO) & 1);
                tc_fence_after();
                out_epilogue_staged(nchunks - 1, sm + L::OT);
            }
        } else {
            if (nchunks > 0) {
                // initial state: S^T row j (fp32, pre-scaled by gam_C of chunk 0) and its bf16 copy
                ctl.wait(B::gready + 0, 0);
                const float g0 = gates(0)[6 * CH];
    #pragma unroll 1
                for (int k = 0; k < kSB; ++k) {
                    const int cb = s_block(k);
                    float x[32];
    #pragma unroll
                    for (int i = 0; i < 32; ++i)
                        x[i] = (flags & kFlagS0Identity) ? ((cb * 32 + i == j) ? 1.f : 0.f)
                                                         : (S0 ? S0[sbase + (size_t)(cb * 32 + i) * ldv + j] : 0.f);
                    store_state_bf16(cb, x);
    #pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] *= g0;
                    st_state(k, x);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(1, 128);
            }
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % NS;
                const uint32_t tO = tmem + L::T_O + (c % NBO) * DV;
                const uint32_t stc = smem_u32(sm + L::ST);  // S_c^T, bf16
                unsigned char *Kt = sm + L::KQ + st * L::KQ_STAGE;
                const unsigned char *WTc = sm + L::WG0 + (c % NI) * L::WG_BYTES + L::W_WT;
                // O = (gam Q) S: A = gam-scaled Q tile (K-major), B = S^T rows (K-major)
                auto issue_o1 = [&]() {
                    constexpr uint32_t idQ = idesc_bf16(64, DV, 0, 0);
    #pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t a = smem_u32(Kt + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32);
                        mma_bf16(tO, sdesc_sw128(a, 16, 1024), sdesc_sw128(stc + (kk >> 2) * (DV * 128) + (kk & 3) * 32, 16, 1024),
                                 idQ, kk > 0);
                    }
                };
                ctl.wait(B::tready + st, (c / NS) & 1);
                if (tid == 0 && !ctl.aborted()) {
                    // U^T = U~^T - S^T W^T, accumulated onto U~^T (A operand negated)
                    tc_fence_after();
                    constexpr uint32_t idN = idesc_bf16(DV, 64, 0, 1, 1);
    #pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint64_t a = sdesc_sw128(stc + (kk >> 2) * (DV * 128) + (kk & 3) * 32, 16, 1024);
                        mma_bf16(tmem + L::T_U + st * 64, a, sdesc_sw128(smem_u32(WTc + kk * 2048), 16, 1024), idN,
                                 v_zero ? (kk > 0) : 1);
                    }
                    mma_commit(&bars[B::u]);
                }
                if (kChainScales) {
                    // while the U MMA runs: gam Q and lam K in place for O1 and the state MMA (every
                    // MMA that reads them unscaled, Gram and W, completed before the chunk was ready)
                    const float *gv = gates(st);
                    const int r = tid & 63;
                    scale_row_bf16(Kt + (tid >> 6) * 16384 + 8192, r, gv[2 * CH + r], 0, 8);
                    scale_row_bf16(Kt + (tid >> 6) * 16384, r, gv[3 * CH + r], 0, 8);
                    fence_proxy_async_smem();
                }
                // O1 goes before the state MMA's commit, so that its completion also covers O1's reads
                // of the Q tile (reloaded right after) and of the S_c copy.  One O buffer: the previous
                // chunk's outputs leave first, while the U MMA runs.
                if (NBO == 1 && c >= 1) out_epilogue(c - 1);
                if (kChainScales) named_bar(1, 128);  // the scaled tiles are complete
                if (tid == 0 && want_out && !ctl.aborted()) {
                    tc_fence_after();
                    issue_o1();
                }
                ctl.wait(B::u, c & 1);
                tc_fence_after();
                if (tid == 0) ctl.arrive(B::tfree + (c % NI));  // W^T of this chunk has been read
                if (kHalf) {
                    float x[32];
                    tmem_ld16x2_32<32>(tl + L::T_U + st * 64, x);
                    tmem_wait_ld();
                    st_half_row_bf16_sw128(sm + L::UT, j, hh, x);
                } else {
                    float x[64];
                    tmem_ld32(tl + L::T_U + st * 64, *reinterpret_cast<float(*)[32]>(&x[0]));
                    tmem_ld32(tl + L::T_U + st * 64 + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
                    tmem_wait_ld();
                    st_row_bf16_sw128(sm + L::UT, j, x);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(1, 128);
                if (tid == 0 && !ctl.aborted()) {
                    tc_fence_after();
                    constexpr uint32_t idS = idesc_bf16(DV, DK, 0, 1);
    #pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // S^T += U^T (lam K)
                        mma_bf16(tmem + L::T_S, sdesc_sw128(smem_u32(sm + L::UT + kk * 32), 16, 1024),
                                 sdesc_sw128(smem_u32(Kt + kk * 2048), 16384, 1024), idS, 1);
                    mma_commit(&bars[B::s]);
                    if (want_out) {
                        constexpr uint32_t idP = idesc_bf16(64, DV, 0, 0);
    #pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // O += P U: A = P rows (K-major), B = U^T rows (K-major)
                            mma_bf16(tO, sdesc_sw128(smem_u32(sm + L::PM + st * 8192 + kk * 32), 16, 1024),
                                     sdesc_sw128(smem_u32(sm + L::UT + kk * 32), 16, 1024), idP, 1);
                        mma_commit(&bars[B::o + c % NBO]);
                    }
                }
                // two O buffers: the previous chunk's outputs leave while the state MMA runs
                if (NBO == 2 && c >= 1) out_epilogue(c - 1);
                ctl.wait(B::s, c & 1);
                tc_fence_after();
                if (warp == 0 && c + NS < nchunks) load_kq(c + NS);
                {
                    // S_{c+1} = gam_C(c) S_c + increment is in TMEM; keep a bf16 copy
                    // and pre-scale the fp32 state by gam_C of the next chunk
                    const bool more = c + 1 < nchunks;
                    float gn = 1.f;
                    if (more) {
                        ctl.wait(B::gready + (c + 1) % NS, ((c + 1) / NS) & 1);
                        gn = gates((c + 1) % NS)[6 * CH];
                    }
    #pragma unroll 1
                    for (int k = 0; k < kSB; ++k) {
                        float x[32];
                        ld_state(k, x);
                        tmem_wait_ld();
                        store_state_bf16(s_block(k), x);
                        if (more) {
    #pragma unroll
                            for (int i = 0; i < 32; ++i) x[i] *= gn;
                            st_state(k, x);
                        }
                    }
                    tmem_wait_st();
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(1, 128);
            }
            if (nchunks > 0) out_epilogue(nchunks - 1);
        }
        // final state
        if (S_final) {
            if (nchunks > 0) {
#pragma unroll 1
                for (int k = 0; k < kSB; ++k) {
                    const int cb = s_block(k);
                    float x[32];
                    ld_state(k, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) S_final[sbase + (size_t)(cb * 32 + i) * ldv + j] = x[i];
                }
            } else if (hh == 0) {
                for (int c2 = 0; c2 < DK; ++c2)
                    S_final[sbase + (size_t)c2 * ldv + j] =
                        (flags & kFlagS0Identity) ? (c2 == j ? 1.f : 0.f) : (S0 ? S0[sbase + (size_t)c2 * ldv + j] : 0.f);
            }
        }
    }
    // After a wait ran out, MMAs already issued may still be running: each issuing thread (the
    // chain's thread 0 and each intra warpgroup's issuer) commits once more and waits, bounded,
    // for its MMAs to complete before the tensor memory is freed.
    if (ctl.aborted()) {
        const int who = tid == 0 ? 0 : (tid >= 128 && (tid - 128) % 128 == kIssuer ? 1 + (tid - 128) / 128 : -1);
        if (who >= 0) {
            mma_commit(&bars[B::drain + who]);
            mbar_wait_bounded(&bars[B::drain + who], 0, 100000000ull);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- host side -------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3-D view [tokens][H][d] of a bf16 tensor; box = 64 features x 1 head x 64 tokens, 128B swizzle.
// A box row is 128 bytes of one head; L2 promotion is kept at 128 bytes so that a fetch does not
// pull in the neighbouring head's row.
bool make_map(CUtensorMap *m, const void *base, long tokens, int H, int d)
{
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D view [tokens][H][d] of an fp32 tensor (the phase memory's (re, im) pairs, d = 2 dk); box =
// 32 floats (128 bytes, the swizzle span) x 1 head x 64 tokens, 128-byte swizzle.
bool make_map_f32(CUtensorMap *m, const void *base, long tokens, int H, int d)
{
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4};
    cuuint32_t box[3] = {32, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// One launch of the chunk kernel over `nseq` sequences given either densely (cu == nullptr:
// sequence s owns tokens s*T .. s*T+T-1) or by offsets cu[0..nseq].
struct TcLaunch {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    void *out;
    float *S_final;
    const int32_t *cu;
    int nseq, T, H;  // H value heads; H / G q/k heads
    long tokens;  // rows of the q/k/v tensors
    int flags;
    float a_scale, b_scale;  // fused prologue (kFlagPrologue)
    int G;                   // value heads per q/k head
    int vblocks = 1;         // value head size = vblocks x DV, one CTA per column block
};

template <int DK, int DV>
cudaError_t launch_tc(const TcLaunch &a, cudaStream_t st)
{
    using L = TcCfg<DK, DV>;
    CUtensorMap mq, mk, mv;
    // a zero-token varlen call still launches so that S_final = S0 is written
    const long map_tokens = a.tokens > 0 ? a.tokens : 1;
    // with V taken as zero nothing is loaded through the V map; any valid map will do
    // with V taken as zero the V map is never read: the k map (H / G heads) serves as a stand-in
    const void *vsrc = (a.flags & kFlagVZero) ? a.k : a.v;
    const int vdim = (a.flags & kFlagVZero) ? DK : DV * a.vblocks;
    const int vheads = (a.flags & kFlagVZero) ? a.H / a.G : a.H;
    const bool ph = (a.flags & kFlagPhase) != 0;
    const bool qk_ok = ph ? make_map_f32(&mq, a.q, map_tokens, a.H / a.G, DK) &&
                                make_map_f32(&mk, a.k, map_tokens, a.H / a.G, DK)
                          : make_map(&mq, a.q, map_tokens, a.H / a.G, DK) &&
                                make_map(&mk, a.k, map_tokens, a.H / a.G, DK);
    if (!qk_ok || !make_map(&mv, vsrc, map_tokens, vheads, vdim)) {
        set_error("cuTensorMapEncodeTiled failed");
        return cudaErrorInvalidValue;
    }
    int smem = L::TOTAL + 1024;
    auto kern = (a.flags & kFlagPrologue) ? chunk_tc_kernel<DK, DV, true> : chunk_tc_kernel<DK, DV, false>;
    if constexpr (DK == 64 && DV == 64) {
        if (ph) {
            kern = chunk_tc_kernel<DK, DV, false, true>;
            smem = TcCfg<DK, DV, true>::TOTAL + 1024;
        }
    } else if (ph) {
        set_error("the fused phase prologue runs at head size 64, value head 64 only");
        return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.vblocks, a.H, a.nseq);
    kern<<<grid, L::THREADS, smem, st>>>(mq, mk, mv, a.log_alpha, a.beta, a.S0,
                                       static_cast<__nv_bfloat16 *>(a.out), a.S_final, a.cu, a.T, a.H,
                                       a.flags, a.a_scale, a.b_scale, a.G);
    return cudaGetLastError();
}

// ---- segment scan for long sequences with few (sequence, head) chains ------------------------
//
// The state map over a stretch of tokens is affine, S_end = M S_in + S_loc, with M the
// transition of the stretch (the recurrence started from S = I with V = 0) and S_loc the state
// it reaches from S = 0.  A sequence is cut into G segments of L chunks:
//   pass A: per segment, S_loc (value chains from zero) and M (transition chains from the
//           identity with V = 0), both by the chunk kernel with outputs off, all segments at once;
//   pass B: per (sequence, head), the scan S_in,g+1 = M_g S_in,g + S_loc,g in fp32, ending with
//           S_final = M_{G-1} S_in,G-1 + S_loc,G-1;
//   pass C: the chunk kernel over every segment from its S_in, writing the outputs.

struct SegPlan {
    int G = 1, L = 0;  // segments per sequence, chunks per segment
};

SegPlan plan_segments(int B, int T, int H, int varlen, int dtype)
{
    SegPlan p;
    if (varlen || dtype != GDN_DTYPE_BF16) return p;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return p;
    }
    const long nchunks = ((long)T + CH - 1) / CH;
    const long chains = (long)B * H;
    long G = sms / chains;     // pass C then fills the SMs
    G = min(G, nchunks / 16);  // at least 16 chunks per segment
    if (G < 2) return p;
    const long L = (nchunks + G - 1) / G;
    p.L = (int)L;
    p.G = (int)((nchunks + L - 1) / L);
    return p;
}

struct SegWork {
    int32_t *cu;
    float *Sloc, *M, *Sin;
    size_t bytes;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

SegWork seg_layout(void *base, int B, int H, int dk, int dv, const SegPlan &p)
{
    SegWork w{};
    const size_t nseg = (size_t)B * p.G;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t o_cu = take((nseg + 1) * sizeof(int32_t));
    const size_t o_sloc = take(nseg * H * (size_t)dk * dv * sizeof(float));
    const size_t o_m = take(nseg * H * (size_t)dk * dk * sizeof(float));
    const size_t o_sin = take(nseg * H * (size_t)dk * dv * sizeof(float));
    w.bytes = off;
    char *b = static_cast<char *>(base);
    if (b) {
        w.cu = reinterpret_cast<int32_t *>(b + o_cu);
        w.Sloc = reinterpret_cast<float *>(b + o_sloc);
        w.M = reinterpret_cast<float *>(b + o_m);
        w.Sin = reinterpret_cast<float *>(b + o_sin);
    }
    return w;
}

// cu[b*G + g] = first token of segment g of sequence b; cu[B*G] = B*T.
__global__ void seg_table_kernel(int32_t *cu, int B, int T, int G, int L)
{
    const int n = B * G;
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s <= n; s += gridDim.x * blockDim.x) {
        if (s == n) {
            cu[s] = B * T;
        } else {
            const int b = s / G, g = s % G;
            const long start = min((long)g * L * CH, (long)T);
            cu[s] = (int32_t)((long)b * T + start);
        }
    }
}

// Pass B: one CTA of 256 threads per (32 value columns, head, sequence).  S (DK x 32, fp32) is
// kept in shared memory; S_in of every segment is written out, then S <- M_g S + S_loc,g with M_g
// staged in shared memory first (coalesced 8-byte loads; row stride DK + 2 so that the rows the
// threads of a warp read at one k fall on different banks).
template <int DK>
__global__ void __launch_bounds__(256) seg_combine_kernel(const float *__restrict__ M, const float *__restrict__ Sloc,
                                                          const float *__restrict__ S0, float *__restrict__ Sin,
                                                          float *__restrict__ S_final, int G, int H, int dv)
{
    constexpr int LDM = DK + 2;
    constexpr int PER = DK * 32 / 256;  // outputs per thread, all in one row: 8 (DK = 64) or 16 (DK = 128)
    extern __shared__ float sh[];       // M_g [DK][LDM], then two DK x 32 state buffers
    float *Ms = sh, *cur = sh + DK * LDM, *nxt = cur + DK * 32;
    const int cb = blockIdx.x, h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    const int c0 = cb * 32;
    const size_t st0 = ((size_t)b * H + h) * DK * dv;
    for (int i = t; i < DK * 32; i += 256) {
        const int r = i / 32, c = i % 32;
        cur[i] = S0 ? S0[st0 + (size_t)r * dv + c0 + c] : 0.f;
    }
    const int first = t * PER, r = first / 32, cc = first % 32;
    for (int g = 0; g < G; ++g) {
        const size_t seg = (size_t)b * G + g;
        const size_t sv = (seg * H + h) * (size_t)DK * dv;
        const float2 *mg = reinterpret_cast<const float2 *>(M + (seg * H + h) * (size_t)DK * DK);
        for (int i = t; i < DK * DK / 2; i += 256) {
            const int rr = (2 * i) / DK, k = (2 * i) % DK;
            *reinterpret_cast<float2 *>(&Ms[rr * LDM + k]) = mg[i];
        }
        __syncthreads();  // M_g staged; cur complete (previous step or the initial load)
        for (int i = t; i < DK * 32; i += 256) {
            const int rr = i / 32, c = i % 32;
            Sin[sv + (size_t)rr * dv + c0 + c] = cur[i];
        }
        float acc[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.f;
#pragma unroll 8
        for (int k = 0; k < DK; ++k) {
            const float m = Ms[r * LDM + k];
#pragma unroll
            for (int e = 0; e < PER; ++e) acc[e] = fmaf(m, cur[k * 32 + cc + e], acc[e]);
        }
#pragma unroll
        for (int e = 0; e < PER; ++e) nxt[r * 32 + cc + e] = acc[e] + Sloc[sv + (size_t)r * dv + c0 + cc + e];
        __syncthreads();  // every read of Ms and cur done
        float *tmp = cur;
        cur = nxt;
        nxt = tmp;
    }
    if (S_final) {
        for (int i = t; i < DK * 32; i += 256) {
            const int rr = i / 32, c = i % 32;
            S_final[st0 + (size_t)rr * dv + c0 + c] = cur[i];
        }
    }
}

// vblocks > 1: a value head of vblocks x DV columns, one CTA per column block in every pass (the
// transitions of the segment scan do not depend on V and run once per chain)
template <int DK, int DV>
cudaError_t run_chunk(const ChunkArgs &a, cudaStream_t st, int vblocks = 1)
{
    const long tokens = a.cu_seqlens ? (long)a.T : (long)a.B * a.T;
    const int dv = DV * vblocks;
    const SegPlan p = plan_segments(a.B, a.T, a.H * vblocks, a.cu_seqlens != nullptr, a.dtype);
    const int pf = a.prologue ? kFlagPrologue : 0;
    const float as = a.a_scale, bs = a.b_scale;
    if (p.G <= 1) {
        const int lf = (a.cu_seqlens && a.B <= TcCfg<DK, DV>::THREADS) ? kFlagLongestFirst : 0;
        TcLaunch t{a.q, a.k, a.v, a.log_alpha, a.beta, a.S0, a.out, a.S_final,
                   a.cu_seqlens, a.B, a.T, a.H, tokens, pf | lf, as, bs, a.G};
        t.vblocks = vblocks;
        return launch_tc<DK, DV>(t, st);
    }
    const SegWork w = seg_layout(a.workspace, a.B, a.H, DK, dv, p);
    const int nseg = a.B * p.G;
    seg_table_kernel<<<(nseg + 256) / 256, 256, 0, st>>>(w.cu, a.B, a.T, p.G, p.L);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // pass A: local states from zero, and transitions from the identity with V = 0
    TcLaunch ta{a.q, a.k, a.v, a.log_alpha, a.beta, nullptr, nullptr, w.Sloc, w.cu, nseg, a.T, a.H, tokens, pf, as, bs,
                a.G};
    ta.vblocks = vblocks;
    e = launch_tc<DK, DV>(ta, st);
    if (e != cudaSuccess) return e;
    e = launch_tc<DK, DK>(TcLaunch{a.q, a.k, nullptr, a.log_alpha, a.beta, nullptr, nullptr, w.M, w.cu, nseg,
                                   a.T, a.H, tokens, kFlagVZero | kFlagS0Identity | pf, as, bs, a.G},
                          st);
    if (e != cudaSuccess) return e;
    // pass B: segment scan of the states
    const int shm = (DK * (DK + 2) + 2 * DK * 32) * (int)sizeof(float);
    e = cudaFuncSetAttribute(seg_combine_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, shm);
    if (e != cudaSuccess) return e;
    seg_combine_kernel<DK><<<dim3(dv / 32, a.H, a.B), 256, shm, st>>>(w.M, w.Sloc, a.S0, w.Sin, a.S_final, p.G,
                                                                      a.H, dv);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // pass C: outputs of every segment from its entry state
    TcLaunch tc{a.q, a.k, a.v, a.log_alpha, a.beta, w.Sin, a.out, nullptr, w.cu, nseg, a.T, a.H, tokens, pf, as, bs,
                a.G};
    tc.vblocks = vblocks;
    return launch_tc<DK, DV>(tc, st);
}

}  // namespace

size_t chunk_tc_workspace_bytes(int B, int T, int H, int dk, int dv, int varlen, int dtype)
{
    const SegPlan p = plan_segments(B, T, H * (dv > 128 ? dv / 128 : 1), varlen, dtype);
    if (p.G <= 1) return 0;
    return seg_layout(nullptr, B, H, dk, dv, p).bytes;
}

bool phase_fused_ok(int B, int T, int H, int varlen)
{
    return plan_segments(B, T, H, varlen, GDN_DTYPE_BF16).G <= 1;
}

cudaError_t launch_phase_chunk(const float *K, const float *Q, const void *V, const float *log_lam,
                               const float *beta, const float *S0, void *out, float *S_final, const int32_t *cu,
                               int B, int T, int H, cudaStream_t stream)
{
    const long tokens = cu ? (long)T : (long)B * T;
    const int lf = (cu && B <= TcCfg<64, 64>::THREADS) ? kFlagLongestFirst : 0;
    TcLaunch t{Q, K, V, log_lam, beta, S0, out, S_final, cu, B, T, H, tokens, kFlagPhase | lf, 0.f, 0.f, 1};
    return launch_tc<64, 64>(t, stream);
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream)
{
    if (a.dv == 256) return a.dk == 128 ? run_chunk<128, 128>(a, stream, 2) : run_chunk<64, 128>(a, stream, 2);
    if (a.dk == 128 && a.dv == 128) return run_chunk<128, 128>(a, stream);
    if (a.dk == 128 && a.dv == 64) return run_chunk<128, 64>(a, stream);
    if (a.dk == 64 && a.dv == 128) return run_chunk<64, 128>(a, stream);
    return run_chunk<64, 64>(a, stream);
}

// Self-test of the failure path: one thread waits, bounded by limit_ns, on an mbarrier that nothing
// arrives on; the wait runs out, the thread records it in the same device error word the kernels
// use, and the kernel returns (it holds no TMEM and has no copies in flight).
__global__ void wait_probe_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(&g_tc_device_error, 2);
    }
}

cudaError_t launch_wait_probe(int limit_ms, cudaStream_t stream)
{
    wait_probe_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_ms * 1000000ull);
    return cudaGetLastError();
}

int read_and_clear_tc_error()
{
    int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(g_tc_device_error, &z, sizeof(int));
    return v;
}

}  // namespace gdn
