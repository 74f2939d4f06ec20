// gdn_phase_rowdecay.cu -- the complex-phase delta memory with one decay per output row of the
// state (value channel): the Delta-Laplace core's diag(r_t) (DeltaPhase README, section 5,
// "Delta-Laplace Phase Memory Core", "Exact Chunkwise-Parallel Scan"; the delta steps of section 2,
// "Complex Phase Matrix Delta Memory").  Per (sequence, head) the state M is dv x dk complex; for
// channel j (row j of M, written m_j) and token t:
//     e_t,j = V_t,j - (1/dk) Re(m_j . conj K_t)          read-out with the previous row
//     m_j  <- r_t,j m_j + beta_t e_t,j K_t                the row's own decay, then the correction
//     o_t,j = (1/dk) Re(m_j . conj Q_t)
// Re(m . conj k) is the real dot product of the interleaved (re, im) pairs, so with the real
// state S = [m_0 .. m_{dv-1}] (2 dk x dv, column j = row j of M as pairs) and real keys k~, q~
// (the pairs as stored) every product below is real.
//
// Chunk form (C tokens, entry state S; g_t,j = sum of log r over the chunk's tokens up to t,
// gp_t,j = g_{t-1},j, gp_0 = 0): unrolling the token steps inside the chunk,
//     e_t,j = v_t,j - e^{gp_t,j} (k~_t . S_j)/dk - sum_{s<t} e^{gp_t,j - g_s,j} b_s e_s,j (k~_s . k~_t)/dk
//     o_t,j = e^{g_t,j} (q~_t . S_j)/dk + sum_{s<=t} e^{g_t,j - g_s,j} b_s e_s,j (k~_s . q~_t)/dk
//     S_j  <- e^{g_{C-1},j} S_j + sum_s e^{g_{C-1},j - g_s,j} b_s e_s,j k~_s
// The products shared by all channels -- R = [K; Q] S, the Grams [K; Q] K^T and the state
// increment K^T W -- run on the tensor cores (tcgen05, kind::tf32, accumulators in tensor memory)
// with every fp32 operand split as x = hi + lo (hi: x with its 13 low mantissa bits cleared, so
// exact in tf32; lo = x - hi) and each product formed as hi hi + hi lo + lo hi, which keeps it to
// about 2^-21 relative (fp32 level).  Only the decay weights differ per channel, so each channel
// solves its own unit-lower system by forward substitution (the batched triangular solve per
// output channel of the page), one thread per channel, with the weights e^{gp_t - g_s} =
// r_{s+1} .. r_{t-1} kept as running products (none is formed from a ratio, none can overflow).
//
// A CTA of 256 threads takes CB channels (64 at dk = 32, 32 at dk = 64) of one (sequence, head)
// and walks its chunks of C = 32 tokens; the state stays in shared memory (hi and lo parts, as
// the MMAs read it), the next chunk's keys, queries, decays and values are fetched while the
// current one is computed.  Per chunk:
//   1. the staged [K; Q] split into hi (in place) and lo; cumulative decays per channel (shuffle
//      scan) and the factors 2^{gp}, 2^{g}, r, 2^{g_end - g}; one thread issues R and the Grams
//   2. R and the Grams from tensor memory to shared memory; the substitution, one thread per
//      channel: per token a sum over the known sources, then e_t, the output o_t and the state
//      weight w_t = 2^{g_end - g_t} b_t e_t (hi and lo); one thread issues K^T W
//   3. the outputs to global memory; S <- diag(2^{g_end}) S + K^T W.
// Every wait on the MMAs is bounded: after a timeout the CTA records the error, issues nothing
// more, and drains what it issued before the tensor memory is freed.
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"
#include "sm100_ptx.cuh"

namespace gdn {

__device__ int g_rd_device_error = 0;

namespace {

using namespace sm100;

constexpr int C = 32;      // tokens per chunk
constexpr int NT = 256;    // threads per CTA
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kTmemCols = 256;  // R at column 0, the Grams at 64, the state increment at 128

// Shared memory plan (byte offsets from a 1024-byte aligned base).  The MMA operand tiles are
// fp32 with 128-byte rows (32 elements) whose 16-byte units are XOR-swizzled by row % 8, in
// column blocks of 32 elements, every operand K-major (the contracted index along the rows): the
// state is kept transposed (S^T, rows = channels), the weights as W^T (rows = channels) and the
// keys also as K^T (rows = features) for the state increment.
template <int DK> struct Plan {
    static constexpr int D = 2 * DK;                  // real size of a key
    static constexpr int CB = DK == 32 ? 64 : 32;     // channels per CTA
    static constexpr int LPC = NT / CB;               // lanes per channel in the decay scan
    static constexpr int SPL = C / LPC;               // tokens per lane there
    static constexpr int LDC = CB + 1;                // row stride of the per-(token, channel) arrays
    static constexpr int LDR = CB + 4;                // row stride of R
    static constexpr int KQ_BYTES = (D / 32) * (2 * C) * 128;  // [K; Q]: 2C rows, D / 32 blocks
    static constexpr int KT_BYTES = D * 128;                   // K^T: D rows of C = 32
    static constexpr int S_BYTES = (D / 32) * CB * 128;        // S^T: CB rows, D / 32 blocks
    static constexpr int W_BYTES = CB * 128;                   // W^T: CB rows of C = 32
    static constexpr int KQH = 0;                     // [2] staged [K; Q], hi parts after the split
    static constexpr int KQL = KQH + 2 * KQ_BYTES;    // lo parts of the current chunk
    static constexpr int KTH = KQL + KQ_BYTES;        // K^T of the current chunk, hi and lo
    static constexpr int KTL = KTH + KT_BYTES;
    static constexpr int SH = KTL + KT_BYTES;         // S^T, hi and lo
    static constexpr int SL = SH + S_BYTES;
    static constexpr int WH = SL + S_BYTES;           // W^T, hi and lo
    static constexpr int WL = WH + W_BYTES;
    static constexpr int LR = WL + W_BYTES;           // [2][C][LDC] log r
    static constexpr int BE = LR + 2 * C * LDC * 4;   // [2][C] beta
    static constexpr int R = BE + 2 * C * 4;          // [2C][LDR] K S / dk, Q S / dk
    static constexpr int GK = R + 2 * C * LDR * 4;    // [C][C] (k_t . k_s) / dk
    static constexpr int GQ = GK + C * C * 4;         // [C][C] (q_t . k_s) / dk
    static constexpr int GQD = GQ + C * C * 4;        // [C] (q_t . k_t) / dk
    static constexpr int EGP = GQD + C * 4;           // [C][LDC] 2^{gp}
    static constexpr int EG = EGP + C * LDC * 4;      // [C][LDC] 2^{g}
    static constexpr int ER = EG + C * LDC * 4;       // [C][LDC] r
    static constexpr int EW = ER + C * LDC * 4;       // [C][LDC] 2^{g_end - g}
    static constexpr int VF = EW + C * LDC * 4;       // [C][CB] values
    static constexpr int O = VF + C * CB * 4;         // [C][CB] outputs
    static constexpr int BAR = O + C * CB * 4;        // two mbarriers: MMAs done, drain
    static constexpr int MISC = BAR + 16;             // TMEM address, abort flag
    static constexpr int TOTAL = MISC + 16;
    static_assert(KQ_BYTES % 1024 == 0 && S_BYTES % 1024 == 0 && W_BYTES % 1024 == 0, "1024-byte tiles");
    static_assert(R % 16 == 0 && GK % 16 == 0 && GQ % 16 == 0 && EGP % 16 == 0 && VF % 16 == 0 && BAR % 8 == 0,
                  "alignment");
    static_assert(TOTAL + 1024 <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// x with its 13 low mantissa bits cleared: exact as a tf32 operand, and x - hi is exact in fp32.
__device__ __forceinline__ float hi_part(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// Byte offset of element e (0..31) of row `row` in a swizzled tile block.
__device__ __forceinline__ int swz(int row, int e)
{
    return row * 128 + ((((e >> 2) ^ row) & 7) << 4) + ((e & 3) << 2);
}

// cp.async with zero fill: ok == false copies no bytes and writes zeros.
__device__ __forceinline__ void cp16z(void *dst, const void *src, bool ok)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(ok ? 16u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp4z(void *dst, const void *src, bool ok)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(ok ? 4u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// K, Q [tokens, H, DK] complex (float2); V, out [tokens, H, dv] in TV; log_r [tokens, H, dv] fp32;
// beta [tokens, H] fp32; M0, Mf [nseq, H, dv, DK] complex (either may be null, or both the same);
// cu [nseq + 1] or null (dense: sequence s owns tokens s T .. s T + T - 1).  CTA (x, h, s) takes
// channels CB x .. CB x + CB - 1 of head h of sequence s.
template <int DK, typename TV>
__global__ void __launch_bounds__(NT, 1) rowdecay_chunk(const float2 *__restrict__ K, const float2 *__restrict__ Q,
                                                       const TV *__restrict__ V, const float *__restrict__ log_r,
                                                       const float *__restrict__ beta, const float2 *M0,
                                                       TV *__restrict__ out, float2 *Mf, const int *__restrict__ cu,
                                                       int T, int H, int dv)
{
    using L = Plan<DK>;
    constexpr int D = L::D, CB = L::CB, LPC = L::LPC, SPL = L::SPL, LDC = L::LDC, LDR = L::LDR;
    constexpr float inv_dk = 1.0f / DK;
    extern __shared__ __align__(16) unsigned char smraw[];
    unsigned char *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    auto F = [&](int off) { return reinterpret_cast<float *>(sm + off); };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, sq = blockIdx.z;
    const int cbase = blockIdx.x * CB;
    const int ncb = min(CB, dv - cbase);
    long t0, t1;
    if (cu) {
        t0 = cu[sq];
        t1 = cu[sq + 1];
    } else {
        t0 = (long)sq * T;
        t1 = t0 + T;
    }
    const int nch = (int)((t1 - t0 + C - 1) / C);
    const size_t mrow = ((size_t)sq * H + h) * dv + cbase;  // row of M of this CTA's channel 0
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::MISC);
    volatile int *abortp = reinterpret_cast<volatile int *>(sm + L::MISC + 4);
    // byte offset of state entry (d, j) in the S^T tiles, of weight entry (s, j) in the W^T tiles
    auto s_off = [](int d, int j) { return (d >> 5) * (CB * 128) + swz(j, d & 31); };
    auto w_off = [](int s, int j) { return swz(j, s); };

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
        *abortp = 0;
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    // entry state S[2i + (0, 1)][j] = (re, im) of entry i of row j (zero past the last channel)
    for (int e = tid; e < CB * DK; e += NT) {
        const int j = e / DK, i = e % DK;
        const float2 m = (M0 && j < ncb) ? M0[(mrow + j) * DK + i] : make_float2(0.f, 0.f);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const float x = p ? m.y : m.x, hx = hi_part(x);
            *F(L::SH + s_off(2 * i + p, j)) = hx;
            *F(L::SL + s_off(2 * i + p, j)) = x - hx;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    uint32_t mphase = 0;
    auto wait_mma = [&]() {
        if (!*abortp && !mbar_wait_bounded(&bar[0], mphase & 1, kWaitLimitNs)) {
            atomicOr(&g_rd_device_error, 4);
            *abortp = 1;
        }
        ++mphase;
        tc_fence_after();
    };
    // R = [K; Q] S (M = 2C, N = CB) at column 0 and the Grams [K; Q] K^T (N = C) at column 64
    auto issue_r_gram = [&](int b) {
        if (tid != 0 || *abortp) return;
        tc_fence_after();
        const uint32_t kqh = smem_u32(sm + L::KQH + b * L::KQ_BYTES), kql = smem_u32(sm + L::KQL);
        const uint32_t sh = smem_u32(sm + L::SH), sl = smem_u32(sm + L::SL);
        constexpr uint32_t idR = idesc_tf32(2 * C, CB, 0, 0), idG = idesc_tf32(2 * C, C, 0, 0);
#pragma unroll
        for (int term = 0; term < 3; ++term) {  // hi hi, hi lo, lo hi
            const uint32_t a = term == 2 ? kql : kqh, bs = term == 1 ? sl : sh, bk = term == 1 ? kql : kqh;
#pragma unroll
            for (int kk = 0; kk < D / 8; ++kk) {
                const uint32_t koff = (kk >> 2) * (2 * C * 128) + (kk & 3) * 32;
                const uint32_t soff = (kk >> 2) * (CB * 128) + (kk & 3) * 32;
                const uint64_t ad = sdesc_sw128(a + koff, 16, 1024);
                const uint32_t acc = (term > 0 || kk > 0) ? 1u : 0u;
                mma_tf32(tmem, ad, sdesc_sw128(bs + soff, 16, 1024), idR, acc);
                mma_tf32(tmem + 64, ad, sdesc_sw128(bk + koff, 16, 1024), idG, acc);
            }
        }
        mma_commit(&bar[0]);
    };
    // the state increment K^T W (M = D, N = CB) at column 128
    auto issue_update = [&]() {
        if (tid != 0 || *abortp) return;
        tc_fence_after();
        const uint32_t kth = smem_u32(sm + L::KTH), ktl = smem_u32(sm + L::KTL);
        const uint32_t wh = smem_u32(sm + L::WH), wl = smem_u32(sm + L::WL);
        constexpr uint32_t idS = idesc_tf32(D, CB, 0, 0);
#pragma unroll
        for (int term = 0; term < 3; ++term) {
            const uint32_t a = term == 2 ? ktl : kth, bw = term == 1 ? wl : wh;
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk)
                mma_tf32(tmem + 128, sdesc_sw128(a + kk * 32, 16, 1024), sdesc_sw128(bw + kk * 32, 16, 1024), idS,
                         (term > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar[0]);
    };

    // chunk c's keys, queries, decays and beta into buffer b (zero past the sequence end and past
    // the last channel); [K; Q] rows of D floats go as 16-byte pieces into the swizzled tile
    auto stage = [&](int c, int b) {
        const long tb = t0 + (long)c * C;
        const int n = (int)min((long)C, t1 - tb);
        unsigned char *kq = sm + L::KQH + b * L::KQ_BYTES;
        for (int p = tid; p < 2 * C * (D / 4); p += NT) {
            const int r = p / (D / 4), o = (p % (D / 4)) * 4;
            const int t = r % C;
            const bool ok = t < n;
            const float2 *src = (r >= C ? Q : K) + ((size_t)(ok ? tb + t : t0) * H + h) * DK + o / 2;
            cp16z(kq + (o >> 5) * (2 * C * 128) + swz(r, o & 31), src, ok);
        }
        float *lr = F(L::LR) + b * C * LDC;
        for (int p = tid; p < C * CB; p += NT) {
            const int t = p / CB, j = p % CB;
            const bool ok = t < n && j < ncb;
            cp4z(lr + t * LDC + j, log_r + ((size_t)(ok ? tb + t : t0) * H + h) * dv + cbase + (ok ? j : 0), ok);
        }
        if (tid < C) {
            const bool ok = tid < n;
            cp4z(F(L::BE) + b * C + tid, beta + (size_t)(ok ? tb + tid : t0) * H + h, ok);
        }
    };
    // values (any element type) go through registers: loaded for the next chunk while the
    // current one is computed, written to shared memory at the top of the next iteration
    constexpr int VPT = C * CB / NT;
    float vreg[VPT];
    auto load_v = [&](int c) {
        const long tb = t0 + (long)c * C;
        const int n = (int)min((long)C, t1 - tb);
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
            const int p = tid + u * NT, t = p / CB, j = p % CB;
            vreg[u] = (t < n && j < ncb) ? to_f(V[((size_t)(tb + t) * H + h) * dv + cbase + j]) : 0.f;
        }
    };

    if (nch > 0) {
        stage(0, 0);
        load_v(0);
    }
    cp_commit();
    for (int c = 0; c < nch; ++c) {
        const int b = c & 1;
#pragma unroll
        for (int u = 0; u < VPT; ++u) F(L::VF)[tid + u * NT] = vreg[u];
        if (c + 1 < nch) stage(c + 1, b ^ 1);
        cp_commit();
        if (c + 1 < nch) load_v(c + 1);
        cp_wait_one();  // chunk c's copies (this thread's) have landed
        __syncthreads();
        const float *bet = F(L::BE) + b * C;

        // ---- 1. the hi / lo split of [K; Q] (and of K^T); decays; R and the Grams issued ----
        {
            unsigned char *kqh = sm + L::KQH + b * L::KQ_BYTES, *kql = sm + L::KQL;
            for (int p = tid; p < L::KQ_BYTES / 16; p += NT) {
                const float4 x = *reinterpret_cast<const float4 *>(kqh + 16 * p);
                const float4 hx = make_float4(hi_part(x.x), hi_part(x.y), hi_part(x.z), hi_part(x.w));
                const float4 lx = make_float4(x.x - hx.x, x.y - hx.y, x.z - hx.z, x.w - hx.w);
                *reinterpret_cast<float4 *>(kqh + 16 * p) = hx;
                *reinterpret_cast<float4 *>(kql + 16 * p) = lx;
                // piece p: block p / (2C * 8), row (p / 8) % 2C, 16-byte unit (p % 8) ^ (row % 8)
                const int r = (p >> 3) % (2 * C);
                if (r < C) {
                    const int d = (p / (2 * C * 8)) * 32 + 4 * ((p & 7) ^ (r & 7));
                    const float hv[4] = {hx.x, hx.y, hx.z, hx.w}, lv[4] = {lx.x, lx.y, lx.z, lx.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        *F(L::KTH + swz(d + u, r)) = hv[u];
                        *F(L::KTL + swz(d + u, r)) = lv[u];
                    }
                }
            }
        }
        {
            // cumulative decays (log2 domain): LPC lanes per channel, SPL consecutive tokens each
            const float *lr = F(L::LR) + b * C * LDC;
            const int j = tid / LPC, l = tid % LPC;
            float x[SPL], inc[SPL], run = 0.f;
#pragma unroll
            for (int i = 0; i < SPL; ++i) {
                x[i] = lr[(SPL * l + i) * LDC + j] * kLog2e;
                run += x[i];
                inc[i] = run;
            }
            float pre = run;  // inclusive scan of the lane totals over the channel's lanes
#pragma unroll
            for (int o = 1; o < LPC; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, pre, o, LPC);
                if (l >= o) pre += y;
            }
            const float excl = pre - run;
            const float gend = __shfl_sync(0xffffffffu, pre, LPC - 1, LPC);
            float gprev = excl;
#pragma unroll
            for (int i = 0; i < SPL; ++i) {
                const int t = SPL * l + i;
                const float g2 = excl + inc[i];
                F(L::EGP)[t * LDC + j] = ex2_approx(gprev);
                F(L::EG)[t * LDC + j] = ex2_approx(g2);
                F(L::ER)[t * LDC + j] = ex2_approx(x[i]);
                F(L::EW)[t * LDC + j] = ex2_approx(gend - g2);
                gprev = g2;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        issue_r_gram(b);

        // ---- 2. R and the Grams to shared memory (M = 64 layout: row r at lane r % 16 of
        //      quadrant r / 16; threads l and l + 16 take the two column halves) ----
        wait_mma();
        {
            const int q = warp & 3, hf = lane >> 4, r = 16 * q + (lane & 15);
            const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
            if (warp < 4) {
                if constexpr (CB == 64) {
                    float x[32];
                    tmem_ld16x2_32<32>(tq, x);
                    tmem_wait_ld();
                    float *dst = F(L::R) + r * LDR + 32 * hf;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(dst + i) =
                            make_float4(x[i] * inv_dk, x[i + 1] * inv_dk, x[i + 2] * inv_dk, x[i + 3] * inv_dk);
                } else {
                    float x[16];
                    tmem_ld16x2_16<16>(tq, x);
                    tmem_wait_ld();
                    float *dst = F(L::R) + r * LDR + 16 * hf;
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        *reinterpret_cast<float4 *>(dst + i) =
                            make_float4(x[i] * inv_dk, x[i + 1] * inv_dk, x[i + 2] * inv_dk, x[i + 3] * inv_dk);
                }
            } else {
                float x[16];
                tmem_ld16x2_16<16>(tq + 64, x);
                tmem_wait_ld();
                const int s0 = 16 * hf;
                float *dst = r < C ? F(L::GK) + r * C + s0 : F(L::GQ) + (r - C) * C + s0;
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4 *>(dst + i) =
                        make_float4(x[i] * inv_dk, x[i + 1] * inv_dk, x[i + 2] * inv_dk, x[i + 3] * inv_dk);
                if (r >= C) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (r - C == s0 + i) F(L::GQD)[r - C] = x[i] * inv_dk;
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- forward substitution, one thread per channel, with the outputs and weights ----
        // y_s = e^{gp_t - g_s} b e_s for the sources s < t of the current token t, as running
        // products: y_{t-1} = b e_{t-1} enters at step t, the older ones are scaled by r_{t-1}.
        if (tid < CB) {
            const int j = tid;
            float y[C];
            const float *Rk = F(L::R), *Rq = F(L::R) + C * LDR;
#pragma unroll
            for (int t = 0; t < C; ++t) {
                float pa = 0.f, pp = 0.f;
                if (t > 0) {
                    const float rprev = F(L::ER)[(t - 1) * LDC + j];
#pragma unroll
                    for (int u = 0; u + 1 < t; ++u) y[u] *= rprev;
                    const float *gk = F(L::GK) + t * C, *gq = F(L::GQ) + t * C;
                    float pa1 = 0.f, pp1 = 0.f;  // two partial sums each for shorter chains
#pragma unroll
                    for (int u = 0; u < t; u += 4) {
                        const float4 a = *reinterpret_cast<const float4 *>(gk + u);
                        const float4 q4 = *reinterpret_cast<const float4 *>(gq + u);
                        pa = fmaf(a.x, y[u], pa);
                        pp = fmaf(q4.x, y[u], pp);
                        if (u + 1 < t) {
                            pa1 = fmaf(a.y, y[u + 1], pa1);
                            pp1 = fmaf(q4.y, y[u + 1], pp1);
                        }
                        if (u + 2 < t) {
                            pa = fmaf(a.z, y[u + 2], pa);
                            pp = fmaf(q4.z, y[u + 2], pp);
                        }
                        if (u + 3 < t) {
                            pa1 = fmaf(a.w, y[u + 3], pa1);
                            pp1 = fmaf(q4.w, y[u + 3], pp1);
                        }
                    }
                    pa += pa1;
                    pp += pp1;
                }
                const float e = F(L::VF)[t * CB + j] - F(L::EGP)[t * LDC + j] * Rk[t * LDR + j] - pa;
                const float be = bet[t] * e;
                y[t] = be;
                F(L::O)[t * CB + j] =
                    F(L::EG)[t * LDC + j] * Rq[t * LDR + j] + F(L::ER)[t * LDC + j] * pp + F(L::GQD)[t] * be;
                const float w = F(L::EW)[t * LDC + j] * be, wh = hi_part(w);
                *F(L::WH + w_off(t, j)) = wh;
                *F(L::WL + w_off(t, j)) = w - wh;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        issue_update();

        // ---- 3. the chunk's outputs; then S <- diag(2^{g_end}) S + K^T W ----
        {
            const long tb = t0 + (long)c * C;
            const int n = (int)min((long)C, t1 - tb);
            for (int p = tid; p < C * CB; p += NT) {
                const int t = p / CB, j = p % CB;
                if (t < n && j < ncb) store_out(out + ((size_t)(tb + t) * H + h) * dv + cbase + j, F(L::O)[p]);
            }
        }
        wait_mma();
        {
            // each thread: 16 consecutive channels j0 .. j0 + 15 of state row d
            float x[16];
            int d, j0;
            const int q = warp & 3;
            const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + 128;
            if constexpr (D == 64) {  // M = 64 layout
                d = 16 * q + (lane & 15);
                j0 = 32 * (warp >> 2) + 16 * (lane >> 4);
                tmem_ld16x2_16<16>(tq + 32 * (warp >> 2), x);
            } else {  // M = 128: row d at lane d
                d = 32 * q + lane;
                j0 = 16 * (warp >> 2);
                tmem_ld32x32b_16(tq + j0, x);
            }
            tmem_wait_ld();
            const float *ge = F(L::EG) + (C - 1) * LDC;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int j = j0 + i, off = s_off(d, j);
                const float nv = fmaf(ge[j], *F(L::SH + off) + *F(L::SL + off), x[i]), nh = hi_part(nv);
                *F(L::SH + off) = nh;
                *F(L::SL + off) = nv - nh;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }
    if (Mf) {
        for (int e = tid; e < CB * DK; e += NT) {
            const int j = e / DK, i = e % DK;
            if (j < ncb)
                Mf[(mrow + j) * DK + i] = make_float2(*F(L::SH + s_off(2 * i, j)) + *F(L::SL + s_off(2 * i, j)),
                                                      *F(L::SH + s_off(2 * i + 1, j)) + *F(L::SL + s_off(2 * i + 1, j)));
        }
    }
    // after a timeout, MMAs issued before may still run: drain them (bounded) before the free
    if (*abortp && tid == 0) {
        mma_commit(&bar[1]);
        mbar_wait_bounded(&bar[1], 0, kWaitLimitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int DK, typename TV>
cudaError_t launch_dk(const float2 *K, const float2 *Q, const TV *V, const float *log_r, const float *beta,
                      const float2 *M0, TV *out, float2 *Mf, const int32_t *cu, int nseq, int T, int H, int dv,
                      cudaStream_t st)
{
    const int smem = Plan<DK>::TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(rowdecay_chunk<DK, TV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((dv + Plan<DK>::CB - 1) / Plan<DK>::CB), (unsigned)H, (unsigned)nseq);
    rowdecay_chunk<DK, TV><<<grid, NT, smem, st>>>(K, Q, V, log_r, beta, M0, out, Mf, cu, T, H, dv);
    return cudaGetLastError();
}

template <typename TV>
cudaError_t launch_typed(const float *K, const float *Q, const void *V, const float *log_r, const float *beta,
                         const float *M0, void *out, float *Mf, const int32_t *cu, int nseq, int T, int H, int dk,
                         int dv, cudaStream_t st)
{
    const float2 *k2 = reinterpret_cast<const float2 *>(K), *q2 = reinterpret_cast<const float2 *>(Q);
    const float2 *m0 = reinterpret_cast<const float2 *>(M0);
    float2 *mf = reinterpret_cast<float2 *>(Mf);
    const TV *v = static_cast<const TV *>(V);
    TV *o = static_cast<TV *>(out);
    if (dk == 64) return launch_dk<64, TV>(k2, q2, v, log_r, beta, m0, o, mf, cu, nseq, T, H, dv, st);
    return launch_dk<32, TV>(k2, q2, v, log_r, beta, m0, o, mf, cu, nseq, T, H, dv, st);
}

}  // namespace

cudaError_t launch_phase_rowdecay(const float *K, const float *Q, const void *V, const float *log_r,
                                  const float *beta, const float *M0, void *out, float *M_final,
                                  const int32_t *cu_seqlens, int nseq, int T, int H, int dk, int dv, int bf16,
                                  cudaStream_t stream)
{
    return bf16 ? launch_typed<__nv_bfloat16>(K, Q, V, log_r, beta, M0, out, M_final, cu_seqlens, nseq, T, H, dk,
                                              dv, stream)
                : launch_typed<float>(K, Q, V, log_r, beta, M0, out, M_final, cu_seqlens, nseq, T, H, dk, dv,
                                      stream);
}

int read_and_clear_rowdecay_error()
{
    int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_rd_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(g_rd_device_error, &z, sizeof(int));
    return v;
}

}  // namespace gdn
