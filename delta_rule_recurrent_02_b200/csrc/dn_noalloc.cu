// dn_noalloc.cu -- dn_chunk_fwd_noalloc: the chunked prefill for callers that
// must not allocate device memory.
//
// Some callers cannot call cudaMalloc (or let a library do it for them): a
// serving process that reserved the device's memory up front for its own
// pools, a framework whose allocator must account for every byte, or a
// latency-critical loop that cannot risk an allocation's cost or implicit
// synchronisation.  The tensor-core prefill needs a scratch workspace (W^T and
// u^T of every chunk); this entry point takes it from a fixed area compiled
// into the library instead of from an allocator.
//
// The area is a file-scope __device__ array: the driver creates it once per
// device when it loads this library's code there, and it stays until the
// process exits.  Host code cannot use the array's name as a device address,
// so every call looks the address up with cudaGetSymbolAddress, with the
// call's device current.  Nothing is cached: after a cudaDeviceReset or a
// primary-context teardown the library's code is loaded again and the array
// may move, and a kept address would then point at freed memory.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "../../include/dn.h"
#include "dn_kernels.h"

namespace {

constexpr size_t kScratchBytes = DN_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the current device's scratch area, looked up afresh.
cudaError_t scratch_for_current_device(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" {

int dn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* beta,
                         const float* g, const float* S0, void* o, float* S_T,
                         int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                         dn_dtype dtype, dn_gate gate, void* cuda_stream) {
    // the request's scratch need, checked against the fixed area before any CUDA call
    size_t need = 0;
    int st = dn_chunk_fwd_workspace_size(B, T, H, d_k, d_v, chunk, dtype, gate, DN_PATH_AUTO, &need);
    if (st != DN_OK) return st;
    char msg[256];
    if (need > kScratchBytes) {
        snprintf(msg, sizeof(msg),
                 "dn_chunk_fwd_noalloc: this request needs %zu bytes of scratch, more than the library's fixed "
                 "%zu-byte area (use dn_chunk_fwd_ex with a caller workspace)",
                 need, kScratchBytes);
        return dn::report_error(DN_ERR_UNSUPPORTED, msg);
    }
    void* scratch = nullptr;
    if (need > 0) {
        const cudaError_t e = scratch_for_current_device(&scratch);
        if (e != cudaSuccess) {
            snprintf(msg, sizeof(msg), "dn_chunk_fwd_noalloc: scratch address lookup failed: %s",
                     cudaGetErrorString(e));
            return dn::report_error(DN_ERR_CUDA, msg);
        }
    }
    return dn_chunk_fwd_ex(q, k, v, beta, g, S0, o, S_T, B, T, H, d_k, d_v, chunk, scale, dtype, gate,
                           DN_PATH_AUTO, scratch, need > 0 ? kScratchBytes : 0, cuda_stream);
}

}  // extern "C"
