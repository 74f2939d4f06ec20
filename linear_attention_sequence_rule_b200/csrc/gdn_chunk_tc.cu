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
// Data flow in one CTA per (sequence, head); 4 warps; thread j owns value column j.
//   TMA  : K, Q (64 tokens x dk) and V (64 x dv) tiles, 128-byte swizzled, into shared memory.
//   MMA 1: [K; Q] K^T                   -> TMEM (M=128, N=64)   Gram matrices of the chunk
//   CUDA : A and P = lower_incl(Gam o Q K^T) with the decays; T = (I + A)^{-1} (fp32 blocked
//          forward substitution in shared memory); T diag(b), T diag(b gam) in bf16
//   MMA 2: V^T (T diag b)^T  -> U~^T      K^T (T diag(b gam))^T -> W^T
//   MMA 3: U^T = U~^T - S^T W^T   (accumulated onto U~^T, A operand negated)
//          S^T Q^T -> first output term
//   MMA 4: U^T P^T -> second output term;   (U^T diag lam) K -> state increment
//   CUDA : S^T <- gam_C S^T + increment (fp32 state kept in TMEM), bf16 copy for the next
//          chunk's MMAs; outputs o[r][j] = gam_r (S^T Q^T)[j][r] + (U^T P^T)[j][r].
// Everything after MMA 3 is transposed (value column = TMEM lane), so the chain MMAs have
// M = dv and each thread handles one value column end to end.
//
// Gates: decays are exp of log_alpha sums taken from the last exact reset (log_alpha = -inf)
// inside the chunk.  Padded rows of a partial chunk get b = 0 and log_alpha = 0, which makes
// their (finite) K/Q/V contents contribute nothing.
//
// Every wait on an mbarrier is bounded (2 s); on timeout the kernel records an error word and
// stops issuing work, then frees its TMEM and returns.
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
constexpr int kThreads = 128;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int LDF = 65;  // padded fp32 row stride of the 64 x 64 scratch matrices

template <int DK, int DV>
struct TcLayout {
    static constexpr int KQ = 0;                             // per 64-feature block: K (8 KB) | Q (8 KB)
    static constexpr int V = KQ + (DK / 64) * 16384;         // per 64-column block: 8 KB
    static constexpr int ST = V + (DV / 64) * 8192;          // S^T bf16, per 64-feature block DV x 128 B
    static constexpr int WT = ST + (DK / 64) * DV * 128;     // W^T bf16, DK rows x 128 B
    static constexpr int PM = WT + DK * 128;                 // P bf16, 64 x 128 B
    static constexpr int TB = PM + 8192;                     // T diag(b)
    static constexpr int TG = TB + 8192;                     // T diag(b gam)
    static constexpr int UT = TG + 8192;                     // U^T bf16, DV x 128 B
    static constexpr int UL = UT + DV * 128;                 // (U^T diag lam) bf16
    static constexpr int AF = UL + DV * 128;                 // A fp32 [64][65]
    static constexpr int TF = AF + CH * LDF * 4;             // T fp32 [64][65]
    static constexpr int XF = TF + CH * LDF * 4;             // merge scratch fp32 [64][65]
    static constexpr int GT = XF + CH * LDF * 4;             // gate vectors (8 x 64 x 4 B)
    static constexpr int BAR = GT + 8 * CH * 4;              // mbarriers + TMEM slot
    static constexpr int TOTAL = BAR + 64;
};

__device__ __forceinline__ void record_error(int code, int *abort_flag)
{
    atomicOr(&g_tc_device_error, code);
    *abort_flag = 1;
}

// T = (I + A)^{-1} for strictly lower triangular A (64 x 64 fp32, row stride LDF), by blocked
// forward substitution: the four 16 x 16 diagonal blocks by substitution, then the 16 -> 32
// and 32 -> 64 merges T_ba = -T_bb A_ba T_aa.  Only the lower triangle of Tm is written.
// Called by all 128 threads; contains __syncthreads.
__device__ void solve_unit_lower(const float *A, float *Tm, float *X, int tid)
{
    if (tid < 64) {
        const int o = (tid >> 4) * 16, c = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float v = 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i)
                if (i >= c) v = fmaf(A[(o + r) * LDF + o + i], x[i], v);
            x[r] = (r < c) ? 0.f : (r == c ? 1.f : -v);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r)
            if (r >= c) Tm[(o + r) * LDF + o + c] = x[r];
    }
    __syncthreads();
    // 16 -> 32: pairs (blocks 0,1) and (2,3).  X = A_ba T_aa, then T_ba = -T_bb X.
    {
        const int p = tid >> 6, rem = tid & 63, r = rem >> 2, c0 = (rem & 3) * 4;
        const int oa = 32 * p, ob = oa + 16;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = A[(ob + r) * LDF + oa + i];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (i >= c0 + q) acc[q] = fmaf(a, Tm[(oa + i) * LDF + oa + c0 + q], acc[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) X[(ob + r) * LDF + oa + c0 + q] = acc[q];
        __syncthreads();
        float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i <= r) {
                const float b = Tm[(ob + r) * LDF + ob + i];
#pragma unroll
                for (int q = 0; q < 4; ++q) t[q] = fmaf(b, X[(ob + i) * LDF + oa + c0 + q], t[q]);
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) Tm[(ob + r) * LDF + oa + c0 + q] = -t[q];
    }
    __syncthreads();
    // 32 -> 64: X = A_ba T_aa with a = [0,32), b = [32,64); then T_ba = -T_bb X.
    {
        const int r = tid >> 2, c0 = (tid & 3) * 8;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const float a = A[(32 + r) * LDF + i];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (i >= c0 + q) acc[q] = fmaf(a, Tm[i * LDF + c0 + q], acc[q]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) X[(32 + r) * LDF + c0 + q] = acc[q];
        __syncthreads();
        float t[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) t[q] = 0.f;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            if (i <= r) {
                const float b = Tm[(32 + r) * LDF + 32 + i];
#pragma unroll
                for (int q = 0; q < 8; ++q) t[q] = fmaf(b, X[(32 + i) * LDF + c0 + q], t[q]);
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) Tm[(32 + r) * LDF + c0 + q] = -t[q];
    }
    __syncthreads();
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const float *__restrict__ log_alpha,
                const float *__restrict__ beta, const float *__restrict__ S0,
                __nv_bfloat16 *__restrict__ out, float *__restrict__ S_final,
                const int32_t *__restrict__ cu_seqlens, int T, int H)
{
    using L = TcLayout<DK, DV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *Af = reinterpret_cast<float *>(sm + L::AF);
    float *Tf = reinterpret_cast<float *>(sm + L::TF);
    float *Xf = reinterpret_cast<float *>(sm + L::XF);
    float *graw = reinterpret_cast<float *>(sm + L::GT);
    float *Gs = graw + CH;
    float *gam = graw + 2 * CH;
    float *lam = graw + 3 * CH;
    float *bet = graw + 4 * CH;
    int *last = reinterpret_cast<int *>(graw + 5 * CH);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);  // [0] TMA, [1] MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::BAR + 16);
    int *abort_flag = reinterpret_cast<int *>(sm + L::BAR + 20);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, s = blockIdx.z;
    long tok0, len;
    if (cu_seqlens) {
        tok0 = cu_seqlens[s];
        len = (long)cu_seqlens[s + 1] - tok0;
    } else {
        tok0 = (long)s * T;
        len = T;
    }
    const size_t sbase = ((size_t)s * H + h) * (size_t)DK * DV;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lanes
    constexpr uint32_t C_G = 0, C_O1 = 0, C_W = 64, C_O2 = 64, C_U = 128, C_DS = 192,
                       C_S = 192 + DK;
    // Rows owned in accumulators with M = DV (value columns) and M = DK (key features).
    // M = 128: row = thread; M = 64: rows 16w..16w+15 sit in lanes 0..15 of warp w.
    const int jrow = (DV == 128) ? tid : (lane < 16 ? warp * 16 + lane : -1);
    const int crow = (DK == 128) ? tid : (lane < 16 ? warp * 16 + lane : -1);

    // ---- initial state: thread jrow holds column jrow of S as a row of S^T ----
#pragma unroll 1
    for (int cb = 0; cb < DK / 32; ++cb) {
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            x[i] = (jrow >= 0 && S0) ? S0[sbase + (size_t)(cb * 32 + i) * DV + jrow] : 0.f;
        tmem_st32(tl + C_S + cb * 32, x);
        if (jrow >= 0) {
            unsigned char *st = sm + L::ST + (cb >> 1) * (DV * 128);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int chunk = (cb & 1) * 4 + c;
                uint4 w;
                w.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
                w.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
                w.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
                w.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
                *reinterpret_cast<uint4 *>(st + jrow * 128 + (((chunk ^ (jrow & 7)) & 7) << 4)) = w;
            }
        }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    uint32_t ph_tma = 0, ph_mma = 0;
    auto wait_mma = [&]() {
        if (!*abort_flag && !mbar_wait_bounded(&bars[1], ph_mma, kWaitLimitNs)) record_error(1, abort_flag);
        ph_mma ^= 1;
        tc_fence_after();
    };

#pragma unroll 1
    for (long c0 = 0; c0 < len; c0 += CH) {
        if (*abort_flag) break;
        const int n = (int)min((long)CH, len - c0);
        const long tk = tok0 + c0;
        if (tid == 0) {
            mbar_arrive_expect_tx(&bars[0], (2 * (DK / 64) + DV / 64) * 8192);
#pragma unroll
            for (int kb = 0; kb < DK / 64; ++kb) {
                tma_load_3d(sm + L::KQ + kb * 16384, &tmK, &bars[0], kb * 64, h, (int)tk);
                tma_load_3d(sm + L::KQ + kb * 16384 + 8192, &tmQ, &bars[0], kb * 64, h, (int)tk);
            }
#pragma unroll
            for (int vb = 0; vb < DV / 64; ++vb)
                tma_load_3d(sm + L::V + vb * 8192, &tmV, &bars[0], vb * 64, h, (int)tk);
        }
        // ---- gates: sums of log_alpha from the last reset (or the chunk start) ----
        if (tid < CH) {
            const bool ok = tid < n;
            graw[tid] = ok ? log_alpha[(size_t)(tk + tid) * H + h] : 0.f;
            bet[tid] = ok ? beta[(size_t)(tk + tid) * H + h] : 0.f;
        }
        __syncthreads();
        if (tid < CH) {
            float acc = 0.f;
            int lst = -1;
            for (int j = 0; j <= tid; ++j) {
                const float g = graw[j];
                if (g == -INFINITY) {
                    lst = j;
                    acc = 0.f;
                } else {
                    acc += g;
                }
            }
            Gs[tid] = acc;
            last[tid] = lst;
        }
        __syncthreads();
        if (tid < CH) {
            gam[tid] = last[tid] >= 0 ? 0.f : expf(Gs[tid]);
            lam[tid] = last[CH - 1] > tid ? 0.f : expf(Gs[CH - 1] - Gs[tid]);
        }
        if (!*abort_flag && !mbar_wait_bounded(&bars[0], ph_tma, kWaitLimitNs)) record_error(2, abort_flag);
        ph_tma ^= 1;
        __syncthreads();

        // ---- MMA 1: Gram matrices [K; Q] K^T ----
        if (tid == 0 && !*abort_flag) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t a = smem_u32(sm + L::KQ + (kk >> 2) * 16384 + (kk & 3) * 32);
                mma_bf16(tmem + C_G, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), id, kk > 0);
            }
            mma_commit(&bars[1]);
        }
        wait_mma();
        {
            float x[64];
            tmem_ld32(tl + C_G, *reinterpret_cast<float(*)[32]>(&x[0]));
            tmem_ld32(tl + C_G + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
            tmem_wait_ld();
            const int r = tid & 63;
            const bool isq = tid >= 64;
            const float Gr = Gs[r], br = bet[r];
            const int lr = last[r];
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const float gm = (i <= r && lr <= i) ? expf(Gr - Gs[i]) : 0.f;
                x[i] = isq ? gm * x[i] : (i < r ? br * gm * x[i] : 0.f);
            }
            if (isq) {
                st_row_bf16_sw128(sm + L::PM, r, x);
            } else {
#pragma unroll
                for (int i = 0; i < CH; ++i) Af[r * LDF + i] = x[i];
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^{-1}; rows of T diag(b) and T diag(b gam) in bf16 ----
        solve_unit_lower(Af, Tf, Xf, tid);
        if (tid < CH) {
            const int r = tid;
            float a[64], b[64];
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const float t = (i <= r) ? Tf[r * LDF + i] : 0.f;
                a[i] = t * bet[i];
                b[i] = a[i] * gam[i];
            }
            st_row_bf16_sw128(sm + L::TB, r, a);
            st_row_bf16_sw128(sm + L::TG, r, b);
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- MMA 2: U~^T = V^T (T diag b)^T ;  W^T = K^T (T diag(b gam))^T ----
        if (tid == 0 && !*abort_flag) {
            tc_fence_after();
            constexpr uint32_t idU = idesc_bf16(DV, 64, 1, 0);
            constexpr uint32_t idW = idesc_bf16(DK, 64, 1, 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16(tmem + C_U, sdesc_sw128(smem_u32(sm + L::V + kk * 2048), 8192, 1024),
                         sdesc_sw128(smem_u32(sm + L::TB + kk * 32), 16, 1024), idU, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16(tmem + C_W, sdesc_sw128(smem_u32(sm + L::KQ + kk * 2048), 16384, 1024),
                         sdesc_sw128(smem_u32(sm + L::TG + kk * 32), 16, 1024), idW, kk > 0);
            }
            mma_commit(&bars[1]);
        }
        wait_mma();
        {
            float x[64];
            tmem_ld32(tl + C_W, *reinterpret_cast<float(*)[32]>(&x[0]));
            tmem_ld32(tl + C_W + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
            tmem_wait_ld();
            if (crow >= 0) st_row_bf16_sw128(sm + L::WT, crow, x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA 3: U^T = U~^T - S^T W^T ;  O1 = S^T Q^T ----
        if (tid == 0 && !*abort_flag) {
            tc_fence_after();
            constexpr uint32_t idN = idesc_bf16(DV, 64, 0, 1, 1);
            constexpr uint32_t idQ = idesc_bf16(DV, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint64_t a = sdesc_sw128(smem_u32(sm + L::ST + (kk >> 2) * (DV * 128) + (kk & 3) * 32), 16, 1024);
                mma_bf16(tmem + C_U, a, sdesc_sw128(smem_u32(sm + L::WT + kk * 2048), 16, 1024), idN, 1);
            }
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint64_t a = sdesc_sw128(smem_u32(sm + L::ST + (kk >> 2) * (DV * 128) + (kk & 3) * 32), 16, 1024);
                const uint32_t b = smem_u32(sm + L::KQ + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32);
                mma_bf16(tmem + C_O1, a, sdesc_sw128(b, 16, 1024), idQ, kk > 0);
            }
            mma_commit(&bars[1]);
        }
        wait_mma();
        {
            float x[64];
            tmem_ld32(tl + C_U, *reinterpret_cast<float(*)[32]>(&x[0]));
            tmem_ld32(tl + C_U + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
            tmem_wait_ld();
            if (jrow >= 0) {
                st_row_bf16_sw128(sm + L::UT, jrow, x);
#pragma unroll
                for (int r = 0; r < CH; ++r) x[r] *= lam[r];
                st_row_bf16_sw128(sm + L::UL, jrow, x);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA 4: O2 = U^T P^T ;  dS^T = (U^T diag lam) K ----
        if (tid == 0 && !*abort_flag) {
            tc_fence_after();
            constexpr uint32_t idP = idesc_bf16(DV, 64, 0, 0);
            constexpr uint32_t idS = idesc_bf16(DV, DK, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + C_O2, sdesc_sw128(smem_u32(sm + L::UT + kk * 32), 16, 1024),
                         sdesc_sw128(smem_u32(sm + L::PM + kk * 32), 16, 1024), idP, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + C_DS, sdesc_sw128(smem_u32(sm + L::UL + kk * 32), 16, 1024),
                         sdesc_sw128(smem_u32(sm + L::KQ + kk * 2048), 16384, 1024), idS, kk > 0);
            mma_commit(&bars[1]);
        }
        wait_mma();
        // ---- state: S^T <- gam_C S^T + dS^T (fp32 in TMEM), bf16 copy for the next chunk ----
        {
            const float gC = gam[CH - 1];
#pragma unroll 1
            for (int cb = 0; cb < DK / 32; ++cb) {
                float x[32], d[32];
                tmem_ld32(tl + C_S + cb * 32, x);
                tmem_ld32(tl + C_DS + cb * 32, d);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = fmaf(gC, x[i], d[i]);
                tmem_st32(tl + C_S + cb * 32, x);
                if (jrow >= 0) {
                    unsigned char *st = sm + L::ST + (cb >> 1) * (DV * 128);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int chunk = (cb & 1) * 4 + c;
                        uint4 w;
                        w.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
                        w.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
                        w.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
                        w.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
                        *reinterpret_cast<uint4 *>(st + jrow * 128 + (((chunk ^ (jrow & 7)) & 7) << 4)) = w;
                    }
                }
            }
            tmem_wait_st();
        }
        // ---- outputs: o[r][j] = gam_r O1[j][r] + O2[j][r] ----
        {
            float o1[32], o2[32];
#pragma unroll 1
            for (int hb = 0; hb < 2; ++hb) {
                tmem_ld32(tl + C_O1 + hb * 32, o1);
                tmem_ld32(tl + C_O2 + hb * 32, o2);
                tmem_wait_ld();
                if (jrow >= 0) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int r = hb * 32 + i;
                        if (r < n)
                            out[((size_t)(tk + r) * H + h) * DV + jrow] =
                                __float2bfloat16_rn(fmaf(gam[r], o1[i], o2[i]));
                    }
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    // ---- final state ----
    if (S_final) {
#pragma unroll 1
        for (int cb = 0; cb < DK / 32; ++cb) {
            float x[32];
            tmem_ld32(tl + C_S + cb * 32, x);
            tmem_wait_ld();
            if (jrow >= 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) S_final[sbase + (size_t)(cb * 32 + i) * DV + jrow] = x[i];
            }
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
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int DK, int DV>
cudaError_t launch_tc(const ChunkArgs &a, cudaStream_t st)
{
    using L = TcLayout<DK, DV>;
    const long tokens = a.cu_seqlens ? (long)a.T : (long)a.B * a.T;
    CUtensorMap mq, mk, mv;
    if (tokens <= 0) return cudaSuccess;
    if (!make_map(&mq, a.q, tokens, a.H, DK) || !make_map(&mk, a.k, tokens, a.H, DK) ||
        !make_map(&mv, a.v, tokens, a.H, DV)) {
        set_error("cuTensorMapEncodeTiled failed");
        return cudaErrorInvalidValue;
    }
    // at least 116 KB so that two CTAs (each holding 512 TMEM columns) never share an SM
    const int smem = (L::TOTAL + 1024) > 118784 ? (L::TOTAL + 1024) : 118784;
    auto kern = chunk_tc_kernel<DK, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(1, a.H, a.B);
    kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, a.log_alpha, a.beta, a.S0,
                                       static_cast<__nv_bfloat16 *>(a.out), a.S_final, a.cu_seqlens,
                                       a.T, a.H);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream)
{
    if (a.dk == 128 && a.dv == 128) return launch_tc<128, 128>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_tc<128, 64>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_tc<64, 128>(a, stream);
    return launch_tc<64, 64>(a, stream);
}

int read_and_clear_tc_error()
{
    int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(g_tc_device_error, &z, sizeof(int));
    return v;
}

}  // namespace gdn
