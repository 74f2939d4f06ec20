// gdn_chunk_fwd_host: the chunk forward from and to HOST buffers.  The batch is cut into up to
// four parts of whole sequences; part p's inputs go up on one side stream, part p runs
// on the caller's stream once they have arrived, and its outputs come down on a second side
// stream, so the copies of one part overlap the other parts' copies in the other direction and
// their compute.  Device memory is the caller's workspace; the side streams and events are created
// once per device and kept.
#include <mutex>

#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace gdn {
namespace {

// Parts per call.  The host-to-device copy is the bound (PCIe); more parts shorten the tail after
// the last upload only down to one part's compute, which stays near 0.2 ms however few sequences
// a part holds (its chains are latency-bound), and each part adds launches: four measured best
// on the hybrid-LM batch (3.42 ms per call, against 3.52 ms with eight and 3.92 ms serial).
constexpr int kMaxParts = 4;
constexpr int kMaxDevices = 64;

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace layout and the cut into parts.  Dense: parts of equal sequence counts.  Varlen: runs
// of whole sequences holding about the same number of tokens (known only from the host cu_seqlens).
struct HostPlan {
    int parts = 0;
    int first[kMaxParts + 1] = {};  // first sequence of part p; first[parts] = B
    size_t q = 0, k = 0, v = 0, la = 0, be = 0, s0 = 0, out = 0, sf = 0, cu = 0, cu_stride = 0, ws = 0, total = 0;
    size_t ws_bytes = 0;
};

int part_count(int B) { return B < kMaxParts ? B : kMaxParts; }

void layout(HostPlan &p, int B, int T, int H, int dk, int dv, int chunk, int varlen, int dtype)
{
    const size_t es = dtype == GDN_DTYPE_BF16 ? 2 : 4;
    const size_t tokens = varlen ? (size_t)T : (size_t)B * T;
    // dense parts get a 256-byte aligned sub-buffer each (their token rows start anywhere), so
    // every token-indexed region has room for one alignment gap per part
    const size_t gaps = varlen ? 0 : (size_t)part_count(B) * 256;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += al256(bytes + gaps);
        return at;
    };
    p.q = take(tokens * H * dk * es);
    p.k = take(tokens * H * dk * es);
    p.v = take(tokens * H * dv * es);
    p.la = take(tokens * H * 4);
    p.be = take(tokens * H * 4);
    p.s0 = take((size_t)B * H * dk * dv * 4);
    p.out = take(tokens * H * dv * es);
    p.sf = take((size_t)B * H * dk * dv * 4);
    // varlen: each part gets its own slice of cu_seqlens (absolute offsets), 256-byte aligned
    p.cu_stride = varlen ? al256((size_t)(B + 1) * 4) : 0;
    p.cu = take(p.cu_stride * part_count(B));
    // the parts run one after another on the caller's stream, so one chunk workspace serves all.
    // Dense parts hold floor(B / P) or ceil(B / P) sequences, and the larger need of the two sizes
    // is kept; a varlen part indexes the whole packed buffer (T tokens) with at most B sequences,
    // so the need of the whole batch bounds every part's
    size_t ws = 0;
    if (!varlen) {
        const int P = part_count(B);
        for (int bp : {B / P, (B + P - 1) / P}) {
            const size_t need = gdn_chunk_fwd_workspace_bytes(bp, T, H, dk, dv, chunk, 0, dtype);
            if (need != (size_t)-1 && need > ws) ws = need;
        }
    } else {
        const size_t need = gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, 1, dtype);
        if (need != (size_t)-1) ws = need;
    }
    p.ws_bytes = ws;
    p.ws = take(ws);
    p.total = o;
}

void cut_dense(HostPlan &p, int B)
{
    p.parts = part_count(B);
    for (int i = 0; i <= p.parts; ++i) p.first[i] = (int)((long long)B * i / p.parts);
}

void cut_varlen(HostPlan &p, int B, const int32_t *cu)
{
    const int P = part_count(B);
    const long long total = cu[B];
    int n = 0;
    p.first[0] = 0;
    for (int i = 1; i < P; ++i) {
        const long long target = total * i / P;
        int e = p.first[n] + 1;  // at least one sequence per part
        while (e < B && cu[e] < target) ++e;
        if (e >= B) break;
        p.first[++n] = e;
    }
    p.first[++n] = B;
    p.parts = n;
}

// Side streams and events of one device, made on first use.
struct DeviceRes {
    bool ready = false;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, done = nullptr, in[kMaxParts] = {}, comp[kMaxParts] = {};
};

std::mutex g_mu;
DeviceRes g_res[kMaxDevices];

cudaError_t get_res(DeviceRes *&r)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    r = &g_res[dev];
    if (r->ready) return cudaSuccess;
    const unsigned ef = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&r->up, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&r->down, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r->start, ef)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r->done, ef)) != cudaSuccess) return e;
    for (int i = 0; i < kMaxParts; ++i) {
        if ((e = cudaEventCreateWithFlags(&r->in[i], ef)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&r->comp[i], ef)) != cudaSuccess) return e;
    }
    r->ready = true;
    return cudaSuccess;
}

int cuda_err(cudaError_t e, const char *what)
{
    set_error("gdn_chunk_fwd_host: %s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return GDN_ERR_CUDA;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" {

size_t gdn_chunk_fwd_host_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen, int dtype)
{
    if (gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, varlen, dtype) == (size_t)-1) return (size_t)-1;
    HostPlan p;
    layout(p, B, T, H, dk, dv, chunk, varlen, dtype);
    return p.total;
}

int gdn_chunk_fwd_host(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                       const float *S0, void *out, float *S_final, int B, int T, int H, int dk, int dv, int chunk,
                       const int32_t *cu_seqlens, int dtype, void *workspace, size_t workspace_bytes,
                       void *stream)
{
    const int varlen = cu_seqlens != nullptr;
    const size_t need = gdn_chunk_fwd_host_workspace_bytes(B, T, H, dk, dv, chunk, varlen, dtype);
    if (need == (size_t)-1)  // the device entry's shape check gives the reason and the code
        return gdn_chunk_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, T, H, dk, dv,
                             chunk, cu_seqlens, dtype, nullptr, 0, stream);
    if (!q || !k || !v || !log_alpha || !beta || !out) {
        set_error("gdn_chunk_fwd_host: q, k, v, the two gate arrays and out are required");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    if (!workspace || workspace_bytes < need) {
        set_error("gdn_chunk_fwd_host: workspace of %zu bytes needed, %zu given", need,
                  workspace ? workspace_bytes : (size_t)0);
        return GDN_ERR_WORKSPACE;
    }
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) {
        set_error("gdn_chunk_fwd_host: workspace must be 256-byte aligned");
        return GDN_ERR_INVALID_ARGUMENT;
    }
    if (varlen) {
        if (cu_seqlens[0] != 0 || cu_seqlens[B] != T) {
            set_error("gdn_chunk_fwd_host: cu_seqlens must run from 0 to T = %d", T);
            return GDN_ERR_INVALID_ARGUMENT;
        }
        for (int s = 0; s < B; ++s)
            if (cu_seqlens[s + 1] < cu_seqlens[s]) {
                set_error("gdn_chunk_fwd_host: cu_seqlens decreases at %d", s);
                return GDN_ERR_INVALID_ARGUMENT;
            }
    }
    HostPlan p;
    layout(p, B, T, H, dk, dv, chunk, varlen, dtype);
    if (varlen) cut_varlen(p, B, cu_seqlens);
    else cut_dense(p, B);

    std::lock_guard<std::mutex> lock(g_mu);
    DeviceRes *r = nullptr;
    cudaError_t e = get_res(r);
    if (e != cudaSuccess) return cuda_err(e, "creating the copy streams");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(workspace);
    const size_t es = dtype == GDN_DTYPE_BF16 ? 2 : 4;
    const size_t row_k = (size_t)H * dk * es, row_v = (size_t)H * dv * es, row_g = (size_t)H * 4;
    const size_t state = (size_t)H * dk * dv * 4;
    auto tok = [&](int s) -> size_t { return varlen ? (size_t)cu_seqlens[s] : (size_t)s * T; };
    // where part i's rows of a token-indexed tensor (row bytes per token) start in its device
    // region: varlen parts index the whole packed buffer by absolute offsets; dense parts sit in
    // 256-byte aligned sub-buffers of their own
    auto dev_off = [&](int i, size_t row) -> size_t {
        if (varlen) return tok(p.first[i]) * row;
        size_t o = 0;
        for (int j = 0; j < i; ++j) o += al256((tok(p.first[j + 1]) - tok(p.first[j])) * row);
        return o;
    };
    const char *qh = static_cast<const char *>(q), *kh = static_cast<const char *>(k),
               *vh = static_cast<const char *>(v), *lah = reinterpret_cast<const char *>(log_alpha),
               *beh = reinterpret_cast<const char *>(beta), *s0h = reinterpret_cast<const char *>(S0);
    char *outh = static_cast<char *>(out), *sfh = reinterpret_cast<char *>(S_final);
    // part i of a token-indexed tensor: host rows from t0 on, device rows at dev_off(i, row)
    auto up = [&](size_t region, const char *src, int i, size_t row, size_t t0, size_t nt) {
        return nt ? cudaMemcpyAsync(w + region + dev_off(i, row), src + t0 * row, nt * row, cudaMemcpyHostToDevice,
                                    r->up)
                  : cudaSuccess;
    };
    auto down = [&](char *dst, size_t region, int i, size_t row, size_t t0, size_t nt) {
        return nt ? cudaMemcpyAsync(dst + t0 * row, w + region + dev_off(i, row), nt * row, cudaMemcpyDeviceToHost,
                                    r->down)
                  : cudaSuccess;
    };

    // the workspace may still be in use by earlier work on the caller's stream
    if ((e = cudaEventRecord(r->start, st)) != cudaSuccess) return cuda_err(e, "event");
    if ((e = cudaStreamWaitEvent(r->up, r->start, 0)) != cudaSuccess) return cuda_err(e, "event");
    if ((e = cudaStreamWaitEvent(r->down, r->start, 0)) != cudaSuccess) return cuda_err(e, "event");
    int rc = GDN_OK;
    for (int i = 0; i < p.parts && e == cudaSuccess; ++i) {
        const int s0 = p.first[i], s1 = p.first[i + 1];
        const size_t t0 = tok(s0), nt = tok(s1) - t0;
        if (varlen)
            e = cudaMemcpyAsync(w + p.cu + i * p.cu_stride, cu_seqlens + s0, (size_t)(s1 - s0 + 1) * 4,
                                cudaMemcpyHostToDevice, r->up);
        // The kernel's 64-row K, Q, V tiles run past a sequence's end; those rows are multiplied
        // by exact zeros, so they only need finite values.  A dense part's tensor maps end with the
        // part (the tiles read zeros beyond it); varlen parts share the whole packed buffer, so
        // each also brings up the 64 rows after it (as the whole batch would hold them) instead of
        // leaving the next part's rows to whatever the workspace held before.
        const size_t halo = varlen ? (size_t)(T - tok(s1) < 64 ? T - tok(s1) : 64) : 0;
        if (e == cudaSuccess) e = up(p.q, qh, i, row_k, t0, nt + halo);
        if (e == cudaSuccess) e = up(p.k, kh, i, row_k, t0, nt + halo);
        if (e == cudaSuccess) e = up(p.v, vh, i, row_v, t0, nt + halo);
        if (e == cudaSuccess) e = up(p.la, lah, i, row_g, t0, nt);
        if (e == cudaSuccess) e = up(p.be, beh, i, row_g, t0, nt);
        if (e == cudaSuccess && S0 && s1 > s0)
            e = cudaMemcpyAsync(w + p.s0 + s0 * state, s0h + s0 * state, (size_t)(s1 - s0) * state,
                                cudaMemcpyHostToDevice, r->up);
        if (e == cudaSuccess) e = cudaEventRecord(r->in[i], r->up);
    }
    if (e != cudaSuccess) rc = cuda_err(e, "host-to-device copy");
    for (int i = 0; i < p.parts && rc == GDN_OK; ++i) {
        const int s0 = p.first[i], s1 = p.first[i + 1];
        const size_t t0 = tok(s0), nt = tok(s1) - t0;
        if ((e = cudaStreamWaitEvent(st, r->in[i], 0)) != cudaSuccess) {
            rc = cuda_err(e, "event");
            break;
        }
        // dense: the part's rows as a batch of its own; varlen: the absolute token offsets of the
        // part's sequences index the whole packed buffers
        const int b0 = varlen ? 0 : i;
        rc = gdn_chunk_fwd(w + p.q + dev_off(b0, row_k), w + p.k + dev_off(b0, row_k), w + p.v + dev_off(b0, row_v),
                           reinterpret_cast<const float *>(w + p.la + dev_off(b0, row_g)),
                           reinterpret_cast<const float *>(w + p.be + dev_off(b0, row_g)),
                           S0 ? reinterpret_cast<const float *>(w + p.s0 + s0 * state) : nullptr,
                           w + p.out + dev_off(b0, row_v),
                           S_final ? reinterpret_cast<float *>(w + p.sf + s0 * state) : nullptr,
                           s1 - s0, T, H, dk, dv, chunk,
                           varlen ? reinterpret_cast<const int32_t *>(w + p.cu + i * p.cu_stride) : nullptr, dtype,
                           p.ws_bytes ? w + p.ws : nullptr, p.ws_bytes, st);
        if (rc != GDN_OK) break;
        if ((e = cudaEventRecord(r->comp[i], st)) == cudaSuccess) e = cudaStreamWaitEvent(r->down, r->comp[i], 0);
        if (e == cudaSuccess) e = down(outh, p.out, i, row_v, t0, nt);
        if (e == cudaSuccess && S_final && s1 > s0)
            e = cudaMemcpyAsync(sfh + s0 * state, w + p.sf + s0 * state, (size_t)(s1 - s0) * state,
                                cudaMemcpyDeviceToHost, r->down);
        if (e != cudaSuccess) rc = cuda_err(e, "device-to-host copy");
    }
    // join both side streams back into the caller's stream, whatever happened above
    cudaError_t e2 = cudaEventRecord(r->done, r->down);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, r->done, 0);
    if (e2 == cudaSuccess) e2 = cudaEventRecord(r->done, r->up);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, r->done, 0);
    if (e2 != cudaSuccess && rc == GDN_OK) rc = cuda_err(e2, "joining the copy streams");
    return rc;
}

}  // extern "C"
