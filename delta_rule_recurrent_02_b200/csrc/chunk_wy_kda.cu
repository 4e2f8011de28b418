// chunk_wy_kda.cu -- the state-independent part of every chunk with the
// per-key gate (see chunk_wy_kda.cuh), one CTA per (b, h, chunk), two CTAs per
// SM.  Used when the prefill runs as two launches (chunk_tc.cu).
#include "chunk_wy_kda.cuh"
#include "dn_kernels.h"

namespace dn {

using namespace sm100;
using namespace tc;

__global__ void __launch_bounds__(kda::kNT, 2)
chunk_wy_kda_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_u, __nv_bfloat16* __restrict__ p_out,
                    __nv_bfloat16* __restrict__ kt_out, __nv_bfloat16* __restrict__ qh_out,
                    float* __restrict__ gam_out, unsigned int* __restrict__ flags, int BH,
                    const float* __restrict__ beta, const float* __restrict__ g, int T, int n, float scale,
                    unsigned int* status, int test_flags) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kda::GROUP_BYTES - 16);
    const int tid = threadIdx.x, warp = tid >> 5;
    kda::Group x = kda::make_group(sm, 0u, 1u, tid);
    if (tid == 0) {
        kda::init_group(x);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kda::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = *tmem_slot;
    const kda::Args ar{&tm_q, &tm_k, &tm_v, &tm_w, &tm_u, p_out, kt_out, qh_out, gam_out, flags, beta, g,
                       T, n, scale, test_flags, nullptr, BH, 0};
    // chunk-major order: chunk 0 of every head first
    const int c = (int)(blockIdx.x / (unsigned)BH);
    const int64_t bh = blockIdx.x - (int64_t)c * BH;
    int64_t pending = -1;
    const bool ok = kda::kda_tile(x, ar, c, bh, pending);
    if (ok && tid == kda::kStoreTid) kda::publish_pending(ar, pending);
    tc_fence_before();
    __syncthreads();
    if (!ok && tid == 0) atomicOr(status, 1u);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(x.tmem, kda::TM_COLS);
    }
}

// ---- host side ---------------------------------------------------------------

cudaError_t launch_chunk_wy_kda(const ChunkArgs& a, const TcMaps& m, cudaStream_t st) {
    const int n = (int)((a.T + kC - 1) / kC);
    constexpr uint32_t kBytes = kda::GROUP_BYTES + 1024;
    auto kern = chunk_wy_kda_kernel;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.B * a.H * n), kda::kNT, kBytes, st>>>(
        m.q, m.k, m.v, m.w, m.u, m.p_ws, m.kt_ws, m.qh_ws, m.gam_ws, m.flags, (int)(a.B * a.H), a.beta, a.g,
        (int)a.T, n, a.scale, a.status, a.test_flags);
    return counted(cudaGetLastError());
}

}  // namespace dn
