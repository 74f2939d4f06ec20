// gdn_noalloc.cu -- gdn_chunk_fwd_noalloc: the chunk forward with the scratch of its segment scan
// taken from a fixed array of device memory that belongs to this library, so that the caller
// passes no workspace and nothing is allocated at call time.
//
// Who needs it: callers that cannot hand over device scratch of their own.  A serving runtime
// that reserves nearly all device memory up front for its recurrent-state cache has no room
// left for a call-time cudaMalloc (it fails, or forces a device-wide synchronisation in the
// middle of a step), and a host program in plain C that drives this library has no device
// allocator to carve a workspace from.  Everything else goes through gdn_chunk_fwd unchanged.
//
// Limits: the scratch is one array per device, so calls on the same device must not overlap in
// time (on two streams, or from two host threads): they would share it and corrupt each other's
// results.  Calls whose scratch would exceed kScratchBytes are rejected with GDN_ERR_WORKSPACE.
// Nothing in the scratch has to start at zero: the segment scan writes every byte it reads
// (offset table, local states, transitions, entry states) earlier in the same call.
#include "gdn_internal.h"
#include "../../include/gdn.h"

namespace {

// 32 MiB.  The segment scan keeps per (segment, head) a local state and an entry state
// (dk x dv fp32) and a transition (dk x dk fp32), with segments x heads bounded by the SM count,
// plus a small offset table: 3 * 148 * 128 * 128 * 4 B = 29.1 MB for dk = dv = 128 on a 148-SM
// device, the largest case there (dv = 256 counts its two column blocks as chains, which halves
// segments x heads: 74 * (2 * 128 * 256 + 128 * 128) * 4 B = 24.2 MB).
constexpr size_t kScratchBytes = size_t(32) << 20;

}  // namespace

// The array takes 32 MiB on every device where the module that holds it is loaded: with CUDA's
// default lazy module loading that happens the first time gdn_chunk_fwd_noalloc needs scratch on
// the device; with CUDA_MODULE_LOADING=EAGER, when the CUDA runtime initialises the device.  It stays
// until the process exits (or the context is destroyed).
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch in the current context, looked up on every call with the target
// device current.  The lookup is cheap once the module is loaded, and taking it afresh each time
// keeps it valid when the context changes under the library (a cudaDeviceReset, or a driver-API
// context the caller made current), where a cached address could point at unmapped memory.  The
// first call on a device loads the module there, so make it before any stream capture.
static int scratch_on_current_device(void **ptr)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr) {
        gdn::set_error("gdn_chunk_fwd_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    *ptr = p;
    return GDN_OK;
}

int gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *S0, void *out, float *S_final, int B, int T,
                          int H, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype,
                          void *stream)
{
    gdn::set_error("%s", "");
    // every argument first, on the host, so that a rejected call touches no device state
    int rc = gdn::chunk_fwd_check("gdn_chunk_fwd_noalloc", q, k, v, log_alpha, beta, S0, out, S_final, B, T,
                                  H, dk, dv, chunk, cu_seqlens, dtype);
    if (rc != GDN_OK) return rc;
    const size_t need = gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, cu_seqlens != nullptr, dtype);
    if (need == 0)  // a plan without scratch: the array is not looked up (nor its module loaded)
        return gdn_chunk_fwd(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk, cu_seqlens,
                             dtype, nullptr, 0, stream);
    if (need > kScratchBytes) {
        gdn::set_error("gdn_chunk_fwd_noalloc: these sizes need %zu bytes of scratch; the static scratch "
                       "holds %zu (use gdn_chunk_fwd with a workspace)",
                       need, kScratchBytes);
        return GDN_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    rc = scratch_on_current_device(&scratch);
    if (rc != GDN_OK) return rc;
    return gdn_chunk_fwd(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk, cu_seqlens, dtype,
                         scratch, kScratchBytes, stream);
}
