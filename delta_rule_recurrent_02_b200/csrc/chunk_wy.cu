// chunk_wy.cu -- the state-independent part of every chunk (gram, A and P,
// the 64 x 64 unit-lower inverse, W and u; see chunk_wy.cuh), one CTA per
// (b, h, chunk), four CTAs per SM.  Used when the prefill runs as two launches
// (chunk_tc.cu); each tile's ready flag is set when it is written.
#include "chunk_wy.cuh"
#include "dn_kernels.h"

namespace dn {

using namespace sm100;
using namespace tc;
using namespace wy;

template <int GATE, bool PRO>
__global__ void __launch_bounds__(kNT, 4)
chunk_wy_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_u, __nv_bfloat16* __restrict__ p_out,
                unsigned int* __restrict__ flags, int BH, const float* __restrict__ beta,
                const float* __restrict__ g, int T, int n, float scale, unsigned int* status, int test_flags,
                Prologue pro, const int* vl, int vl_N) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the __shared__ array itself so that
    // every access below compiles to a shared-memory (not generic) instruction
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 16);
    const int tid = threadIdx.x, warp = tid >> 5;
    // a packed batch: the grid covers the most chunks its tokens can make; the
    // blocks past the batch's actual chunks have nothing to do
    if (vl && (int)(blockIdx.x / (unsigned)BH) >= VarlenTables{vl, vl_N}.coff()[vl_N]) return;
    Group x = make_group(sm, 0u, 1u, tid);
    if (tid == 0) {
        init_group(x);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = *tmem_slot;
    const Args ar{&tm_q, &tm_k, &tm_v, &tm_w, &tm_u, p_out, flags, beta, g, T, n, scale, test_flags, nullptr,
                  BH, 0, pro.on, pro.A_log, pro.dt_bias, pro.H, pro.rep, vl, vl_N, pro.rq};
    // chunk-major order: chunk 0 of every head first
    const int c = (int)(blockIdx.x / (unsigned)BH);
    const int64_t bh = blockIdx.x - (int64_t)c * BH;
    int64_t pending = -1;
    const bool ok = wy_tile<GATE, PRO>(x, ar, c, bh, pending);
    if (ok && tid == kStoreTid) publish_pending(ar, pending);
    tc_fence_before();
    __syncthreads();
    if (!ok && tid == 0) atomicOr(status, 1u);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(x.tmem, TM_COLS);
    }
}

// ---- host side ---------------------------------------------------------------

namespace {

constexpr uint32_t SMEM_BYTES = GROUP_BYTES + 1024;

template <int GATE, bool PRO>
cudaError_t launch_wy_gate(const ChunkArgs& a, const TcMaps& m, int n, cudaStream_t st) {
    auto kern = chunk_wy_kernel<GATE, PRO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // a packed batch: H heads x the most chunks its tokens can make (the blocks past
    // the actual chunks return at once)
    const int64_t chunks = a.cu_seqlens ? vl_chunks_max(a.T, a.N) : n;
    kern<<<(unsigned)(a.B * a.H * chunks), kNT, SMEM_BYTES, st>>>(
        m.q, m.k, m.v, m.w, m.u, m.p_ws, m.flags, (int)(a.B * a.H), a.beta, a.g, (int)a.T, n, a.scale, a.status,
        a.test_flags, prologue_of(a, m), m.vl, a.N);
    return counted(cudaGetLastError());
}

}  // namespace

cudaError_t launch_chunk_wy(const ChunkArgs& a, const TcMaps& m, cudaStream_t st) {
    const int n = (int)((a.T + kC - 1) / kC);
    if (a.prologue) return launch_wy_gate<kGateScalar, true>(a, m, n, st);
    return a.gate == kGateScalar ? launch_wy_gate<kGateScalar, false>(a, m, n, st)
                                 : launch_wy_gate<kGateNone, false>(a, m, n, st);
}

}  // namespace dn
