// gdn_phase_rowdecay.cu -- the complex-phase delta memory with one decay per output row of the
// state (value channel): the Delta-Laplace core's diag(r_t) (DeltaPhase README, section 5,
// "Delta-Laplace Phase Memory Core", "Exact Chunkwise-Parallel Scan"; the delta steps of section 2,
// "Complex Phase Matrix Delta Memory").  Per (sequence, head) the state M is dv x dk complex; for
// channel j (row j of M, written m_j) and token t:
//     e_t,j = V_t,j - (1/dk) Re(m_j . conj K_t)          read-out with the previous row
//     m_j  <- r_t,j m_j + beta_t e_t,j K_t                the row's own decay, then the correction
//     o_t,j = (1/dk) Re(m_j . conj Q_t)
// The rows never interact: each channel is the scalar-decay phase memory with its own decay, so
// its chunk form needs a triangular system of its own per chunk (a 64 x 64 solve and the decay
// weights of 2 x 2016 token pairs per channel, where the scalar memory shares one solve among all
// channels).  Per token a channel costs O(dk), so the channels run here as independent sequential
// scans instead: LPC lanes per channel, each lane holding DK / LPC complex entries of m_j in
// registers; per token two reductions over the LPC lanes (log2 LPC shuffles) and a rank-one
// update.  A CTA takes CB channels of one (sequence, head): its threads stage the inputs of TT
// tokens at a time in shared memory by cp.async (K and Q rows once for all the CTA's channels,
// the channels' values and decays, the decays turned into factors once per tile), double
// buffered, so the scans read every input from shared memory while the next tile is in flight.
#include <cuda_bf16.h>
#include <math.h>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int LPC = 4;              // lanes per channel
constexpr int CPW = 32 / LPC;       // channels per warp
constexpr int WARPS = 4;
constexpr int CB = CPW * WARPS;     // channels per CTA
constexpr int TT = 32;              // tokens per staged tile

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Sum over the LPC lanes of a channel group (xor butterfly inside groups of LPC lanes).
__device__ __forceinline__ float group_sum(float x)
{
#pragma unroll
    for (int o = LPC / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o, LPC);
    return x;
}

__device__ __forceinline__ void cp4(void *dst, const void *src, bool ok)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(ok ? 4u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Shared tile of TT tokens: K, Q rows [TT][DK] complex; values, decays [TT][CB]; beta [TT].
template <int DK> struct Tile {
    float2 k[TT][DK];
    float2 q[TT][DK];
    float v[TT][CB];
    float lr[TT][CB];
    float b[TT];
};

// K, Q [tokens, H, DK] complex (float2); V, out [tokens, H, dv] in TV; log_r [tokens, H, dv] fp32;
// beta [tokens, H] fp32; M0, Mf [nseq, H, dv, DK] complex (either may be null); cu [nseq + 1] or
// null (dense: sequence s owns tokens s T .. s T + T - 1).  CTA (cb, h, s) takes channels
// CB cb .. CB cb + CB - 1 of head h of sequence s; warp w channels CPW w .. of those.
template <int DK, typename TV>
__global__ void __launch_bounds__(32 * WARPS) rowdecay_scan(const float2 *__restrict__ K, const float2 *__restrict__ Q,
                                                           const TV *__restrict__ V, const float *__restrict__ log_r,
                                                           const float *__restrict__ beta,
                                                           const float2 *__restrict__ M0, TV *__restrict__ out,
                                                           float2 *__restrict__ Mf, const int *__restrict__ cu, int T,
                                                           int H, int dv)
{
    constexpr int E = DK / LPC;  // complex entries per lane: i, i + LPC, i + 2 LPC, ...
    extern __shared__ __align__(16) unsigned char smraw[];
    Tile<DK> *tiles = reinterpret_cast<Tile<DK> *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, i = lane % LPC;
    const int h = blockIdx.y, s = blockIdx.z;
    const int cbase = blockIdx.x * CB;
    const int jl = warp * CPW + lane / LPC;  // channel within the CTA
    const bool valid = cbase + jl < dv;
    const int j = valid ? cbase + jl : dv - 1;  // lanes past the last channel compute a copy, store nothing
    long t0, t1;
    if (cu) {
        t0 = cu[s];
        t1 = cu[s + 1];
    } else {
        t0 = (long)s * T;
        t1 = t0 + T;
    }
    const size_t mrow = (((size_t)s * H + h) * dv + j) * DK;
    float2 m[E];
#pragma unroll
    for (int e = 0; e < E; ++e) m[e] = M0 ? M0[mrow + i + LPC * e] : make_float2(0.f, 0.f);
    constexpr float inv_dk = 1.0f / DK;
    const int ncb = min(CB, dv - cbase);  // channels of this CTA

    // stage tokens tb .. tb + TT - 1 by cp.async (rows past the end: not loaded, never read)
    auto stage = [&](long tb, Tile<DK> &tl) {
        const int nt = (int)min((long)TT, t1 - tb);
        // K and Q rows: DK float2 = DK / 2 chunks of 16 bytes per row
        for (int c = tid; c < nt * (DK / 2); c += 32 * WARPS) {
            const int r = c / (DK / 2), o = (c % (DK / 2)) * 2;
            const size_t g = ((size_t)(tb + r) * H + h) * DK + o;
            cp16(&tl.k[r][o], K + g);
            cp16(&tl.q[r][o], Q + g);
        }
        for (int c = tid; c < nt * CB; c += 32 * WARPS) {
            const int r = c / CB, ch = c % CB;
            const bool ok = ch < ncb;
            cp4(&tl.lr[r][ch], log_r + ((size_t)(tb + r) * H + h) * dv + cbase + (ok ? ch : 0), ok);
        }
        if (tid < nt) cp4(&tl.b[tid], beta + (size_t)(tb + tid) * H + h, true);
    };
    // values (any element type) go through registers: loaded at the start of a tile's scan for
    // the next tile, written to shared memory after the scan
    constexpr int VPT = TT * CB / (32 * WARPS);  // values per thread and tile
    float vreg[VPT];
    auto load_v = [&](long tb) {
        const int nt = (int)min((long)TT, t1 - tb);
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
            const int c = tid + u * 32 * WARPS, r = c / CB, ch = c % CB;
            vreg[u] = (r < nt && ch < ncb) ? to_f(V[((size_t)(tb + r) * H + h) * dv + cbase + ch]) : 0.f;
        }
    };
    auto store_v = [&](Tile<DK> &tl) {
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
            const int c = tid + u * 32 * WARPS;
            tl.v[c / CB][c % CB] = vreg[u];
        }
    };
    if (t0 < t1) {
        stage(t0, tiles[0]);
        load_v(t0);
        store_v(tiles[0]);
    }
    cp_commit();
    int buf = 0;
    for (long tb = t0; tb < t1; tb += TT, buf ^= 1) {
        const bool more = tb + TT < t1;
        if (more) {
            stage(tb + TT, tiles[buf ^ 1]);
            load_v(tb + TT);
        }
        cp_commit();
        cp_wait_one();  // this tile's copies have landed (the next tile's may still be in flight)
        __syncthreads();
        Tile<DK> &tl = tiles[buf];
        const int nt = (int)min((long)TT, t1 - tb);
        // the decay factors r = exp(log r), once per (token, channel) instead of in every lane
        for (int c = tid; c < TT * CB; c += 32 * WARPS) {
            float &x = (&tl.lr[0][0])[c];
            x = expf(x);
        }
        __syncthreads();
#pragma unroll 2
        for (int r = 0; r < nt; ++r) {
            const long t = tb + r;
            float2 k[E], q[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                k[e] = tl.k[r][i + LPC * e];
                q[e] = tl.q[r][i + LPC * e];
            }
            const float v = tl.v[r][jl];
            const float rr = tl.lr[r][jl], b = tl.b[r];
            // e = v - (1/dk) Re(m . conj k), Re(m conj k) = Re m Re k + Im m Im k
            float rd0 = 0.f, rd1 = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                rd0 = fmaf(m[e].x, k[e].x, rd0);
                rd1 = fmaf(m[e].y, k[e].y, rd1);
            }
            const float err = v - group_sum(rd0 + rd1) * inv_dk;
            const float be = b * err;
            float od0 = 0.f, od1 = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                m[e].x = fmaf(rr, m[e].x, be * k[e].x);
                m[e].y = fmaf(rr, m[e].y, be * k[e].y);
                od0 = fmaf(m[e].x, q[e].x, od0);
                od1 = fmaf(m[e].y, q[e].y, od1);
            }
            const float od = group_sum(od0 + od1);
            if (valid && i == 0) store_out(out + ((size_t)t * H + h) * dv + j, od * inv_dk);
        }
        if (more) store_v(tiles[buf ^ 1]);
        __syncthreads();  // every scan has read this tile before it is staged again
    }
    if (Mf && valid) {
#pragma unroll
        for (int e = 0; e < E; ++e) Mf[mrow + i + LPC * e] = m[e];
    }
}

template <typename TV>
cudaError_t launch_typed(const float *K, const float *Q, const void *V, const float *log_r, const float *beta,
                         const float *M0, void *out, float *Mf, const int32_t *cu, int nseq, int T, int H, int dk,
                         int dv, cudaStream_t st)
{
    const dim3 grid((unsigned)((dv + CB - 1) / CB), (unsigned)H, (unsigned)nseq);
    const float2 *k2 = reinterpret_cast<const float2 *>(K), *q2 = reinterpret_cast<const float2 *>(Q);
    const float2 *m0 = reinterpret_cast<const float2 *>(M0);
    float2 *mf = reinterpret_cast<float2 *>(Mf);
    const TV *v = static_cast<const TV *>(V);
    TV *o = static_cast<TV *>(out);
    if (dk == 64) {
        const int smem = 2 * (int)sizeof(Tile<64>);
        cudaError_t e = cudaFuncSetAttribute(rowdecay_scan<64, TV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        rowdecay_scan<64, TV><<<grid, 32 * WARPS, smem, st>>>(k2, q2, v, log_r, beta, m0, o, mf, cu, T, H, dv);
    } else {
        const int smem = 2 * (int)sizeof(Tile<32>);
        cudaError_t e = cudaFuncSetAttribute(rowdecay_scan<32, TV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        rowdecay_scan<32, TV><<<grid, 32 * WARPS, smem, st>>>(k2, q2, v, log_r, beta, m0, o, mf, cu, T, H, dv);
    }
    return cudaGetLastError();
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

}  // namespace gdn
