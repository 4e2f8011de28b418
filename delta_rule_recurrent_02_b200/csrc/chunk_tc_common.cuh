// chunk_tc_common.cuh -- pieces shared by the two tensor-core chunk kernels:
// chunk_wy.cu (the UT/WY transform of every chunk, in parallel) and
// chunk_tc.cu (the sequential state pass and the output).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "dn_common.cuh"
#include "dn_kernels.h"
#include "sm100.cuh"

namespace dn {
namespace tc {

using namespace sm100;

constexpr int kC = 64;                      // chunk
constexpr int kD = 128;                     // d_k = d_v
constexpr uint64_t kWaitNs = 1000000000ull; // every mbarrier wait gives up after 1 s

// Workspace per (b, h, chunk), written by chunk_wy.cu and read by chunk_tc.cu,
// three bf16 arrays one after another:
//   -W   [tiles * 64 rows (position)][128 (d_k)]
//   u^T  [tiles * 128 rows (d_v)][64 (position)]
//   P    [tiles * 64 rows (i)][64 (j)]
//   rq   [tiles][64]  1 / max(||q_i||, 1e-12) of the tile's rows (fp32; written
//        only with the layer's prologue, for the state pass's output rows)
constexpr size_t kWsWBytes = (size_t)kC * kD * 2;
constexpr size_t kWsUBytes = (size_t)kD * kC * 2;
constexpr size_t kWsPBytes = (size_t)kC * kC * 2;
constexpr size_t kWsRqBytes = (size_t)kC * 4;
constexpr size_t kWsTileBytes = kWsWBytes + kWsUBytes + kWsPBytes + kWsRqBytes;
// With the per-key gate (KDA) three more arrays follow, which the state pass
// reads in place of q and k and of the scalar decays:
//   K~   [tiles * 64 rows][128]  k (.) e^(Gamma_last - Gamma)      (bf16)
//   Qh   [tiles * 64 rows][128]  scale q (.) e^Gamma               (bf16)
//   gam  [tiles][128]            e^(Gamma_last), per key channel  (fp32)
constexpr size_t kWsKtBytes = (size_t)kC * kD * 2;
constexpr size_t kWsQhBytes = (size_t)kC * kD * 2;
constexpr size_t kWsGamBytes = (size_t)kD * 4;
constexpr size_t kWsKdaTileBytes = kWsTileBytes + kWsKtBytes + kWsQhBytes + kWsGamBytes;
static_assert(kWsKdaTileBytes % 256 == 0, "flags stay 256-byte aligned");
// ...then one 32-bit ready flag per tile, set (release) once the tile is
// written and awaited (acquire) before the state pass loads it, and one
// 32-bit counter from which the single-launch WY groups take their tiles after
// the first; all zeroed before each prefill.
inline size_t ws_flags_offset(uint64_t tiles, bool kda = false) {
    return (size_t)tiles * (kda ? kWsKdaTileBytes : kWsTileBytes);
}
inline size_t ws_flag_words(uint64_t tiles) { return (size_t)tiles + 1; }
inline size_t ws_total_bytes(uint64_t tiles, bool kda = false) {
    return ws_flags_offset(tiles, kda) + ((ws_flag_words(tiles) * 4 + 255) / 256) * 256;
}

// Tensor maps of the tensor-core path (128-byte swizzle, 64-column boxes):
// q, k, v as [B H T][128] with 64-row boxes; the workspace's -W as [tiles 64][128]
// with 64-row boxes, u^T as [tiles 128][64] with 128-row boxes, P as
// [tiles 64][64] with 64-row boxes.
struct TcMaps {
    CUtensorMap q, k, v, w, u, p;
    __nv_bfloat16* p_ws;     // the workspace's P array (written with plain stores)
    unsigned int* flags;     // the workspace's ready flags, zeroed before each prefill
    // per-key gate only: the workspace's K~ and Qh as [tiles 64][128] with 64-row
    // boxes, and its gam array
    CUtensorMap kt, qh;
    __nv_bfloat16* kt_ws;
    __nv_bfloat16* qh_ws;
    float* gam_ws;
    // a packed batch only: the workspace's chunk tables (VarlenTables), else null
    const int* vl = nullptr;
    float* rq_ws = nullptr;  // the workspace's rq array
    // the workspace itself (null unless 128-byte aligned) and its tile count
    uint8_t* scratch = nullptr;
    uint64_t tiles = 0;
};

// The Gated DeltaNet layer's prologue, fused into the prefill kernels (scalar
// gate): when `on`, the beta and g arrays hold the raw inputs b and a, and q
// and k are normalised per row inside the kernels.
struct Prologue {
    int on;                  // 0: off; else beta = on * sigmoid(b) (1, or 2 for the gate in (0, 2))
    const float* A_log;      // [H]
    const float* dt_bias;    // [H]
    int H;                   // heads per batch row (head of bh: bh % H)
    int rep = 1;             // value heads per key head (q and k have H / rep heads)
    // the gated RMSNorm on the output rows (0 none, 1 SiLU(z), 2 sigmoid(z)): z and the
    // output token-major [B][T][H][d_v]
    int norm = 0;
    const __nv_bfloat16* z = nullptr;
    const float* norm_w = nullptr;
    float eps = 0.f;
    float* rq = nullptr;     // the workspace's 1 / ||q_i|| per tile row (with the prologue)
    // the workspace and its tile count: the state pass drops each tile's lines from L2
    // once its loads have landed, so that they are never written back (null: kept)
    uint8_t* scratch = nullptr;
    long long scratch_tiles = 0;
};

// Chunk tables of a packed batch of N sequences, built on the device from
// cu_seqlens before the prefill kernels run (varlen_table_kernel), as ints:
//   cu      [N + 1]   the sequences' token offsets (a checked copy: all zero if
//                     cu_seqlens was not non-decreasing from 0 to the total)
//   coff    [N + 1]   the first global chunk of each sequence; coff[N] = chunks in all
//   seq_of  [nc_max]  the sequence of each global chunk
struct VarlenTables {
    const int* base;
    int N;
    __host__ __device__ const int* cu() const { return base; }
    __host__ __device__ const int* coff() const { return base + N + 1; }
    __host__ __device__ const int* seq_of() const { return base + 2 * (N + 1); }
};
// Global chunks of a packed batch of T tokens in N sequences: at most T / 64 + N.
inline int64_t vl_chunks_max(int64_t T, int N) { return T / kC + N; }
inline size_t vl_table_ints(int N, int64_t nc_max) { return 2 * (size_t)(N + 1) + (size_t)nc_max; }

// The workspace whose consumed tiles the state passes drop from L2 (null: none).
// Dropping pays when a tile is consumed soon after it is written, while its
// lines are still in L2 (126 MB): then they are never written back to memory
// (measured at 4096 tiles, 169 MB: 196 -> 87 MB of DRAM writes per launch, no
// time cost).  Where the WY side runs far ahead of the chains (long sequences
// on few heads, workspaces of a GB and more) the lines have been written back
// long before; dropping saves nothing there and costs about 1%, so it is done
// only up to 512 MB of tiles.  The discards need 128-byte aligned lines.
inline uint8_t* drop_scratch(uint8_t* ws, uint64_t tile_bytes) {
    constexpr uint64_t kDropMaxBytes = 512ull << 20;
    return (reinterpret_cast<uintptr_t>(ws) & 127u) == 0 && tile_bytes <= kDropMaxBytes ? ws : nullptr;
}

// The Prologue argument of the tensor-core kernels for a request.
inline Prologue prologue_of(const ChunkArgs& a, const TcMaps& m) {
    Prologue p{a.prologue, a.A_log, a.dt_bias, (int)a.H, a.rep};
    p.norm = a.norm;
    p.z = static_cast<const __nv_bfloat16*>(a.z);
    p.norm_w = a.norm_weight;
    p.eps = a.eps;
    if (a.prologue) p.rq = m.rq_ws;
    p.scratch = m.scratch;
    p.scratch_tiles = (long long)m.tiles;
    return p;
}

// Row block of q and k for value head bh (b * H + h): key head h / rep of batch row b.
__host__ __device__ __forceinline__ int64_t key_head(int64_t bh, int H, int rep) {
    return rep == 1 ? bh : (bh / H) * (H / rep) + (bh % H) / rep;
}

// Gate slot of one chunk (floats).  G_RQ / G_RK: 1 / ||q_i|| and 1 / ||k_i||
// when the layer's prologue normalises q and k inside the kernels, else 1.
constexpr int G_BETA = 0, G_G2 = 64, G_EG = 128, G_ET = 192, G_BEG = 256, G_GAMMA = 320, G_RQ = 384, G_RK = 448;
constexpr uint32_t GATE_FLOATS = 512;

// The layer's raw gates as gdn_raw_gates computes them, with the fast exponential,
// logarithm and division, for the tensor-core kernels (the WY tile and the state
// pass both use this one, so they see the same beta and g).  softplus(x) =
// log(1 + y), y = e^x: x above 20, the series y - y^2/2 + y^3/3 - y^4/4 for
// y < 1/16 (truncated after y^4: under 3.1e-6 of the value), else log(1 + y)
// (the rounding of 1 + y and the fast logarithm: under about 7e-6 of the value).
__device__ __forceinline__ void gdn_raw_gates_fast(float& b, float& a, float eA, float dt_bias, float bmul) {
    b = __fdividef(bmul, 1.f + __expf(-b));
    const float x = a + dt_bias;
    const float y = __expf(x);
    const float sp = x > 20.f ? x
                   : y < 0.0625f ? y * (1.f - y * (0.5f - y * (1.f / 3.f - 0.25f * y)))
                                 : __logf(1.f + y);
    a = -eA * sp;
}

// Gates of one chunk from beta and g at positions lane and lane + 32 (zero past
// the chunk's end, which makes those positions identity steps).  G is the
// inclusive prefix sum of g inside the chunk ("Linear attention and Gated
// DeltaNet", ch. 28, the chunked form: cumulative log-decay); the slot gets
// beta, G log2(e), e^G, e^(G_last - G), beta e^G and e^(G_last).  One warp.
__device__ __forceinline__ void chunk_gates(float* gs, float b0, float b1, float a0, float a1, int lane) {
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, a0, o2);
        const float y1 = __shfl_up_sync(0xffffffffu, a1, o2);
        if (lane >= o2) { a0 += y0; a1 += y1; }
    }
    a1 += __shfl_sync(0xffffffffu, a0, 31);
    const float Glast = __shfl_sync(0xffffffffu, a1, 31);
    const float L2E = 1.4426950408889634f;
    gs[G_BETA + lane] = b0; gs[G_BETA + lane + 32] = b1;
    gs[G_G2 + lane] = a0 * L2E; gs[G_G2 + lane + 32] = a1 * L2E;
    const float e0 = expf(a0), e1 = expf(a1);
    gs[G_EG + lane] = e0; gs[G_EG + lane + 32] = e1;
    gs[G_BEG + lane] = b0 * e0; gs[G_BEG + lane + 32] = b1 * e1;
    gs[G_ET + lane] = expf(Glast - a0); gs[G_ET + lane + 32] = expf(Glast - a1);
    if (lane == 0) gs[G_GAMMA] = expf(Glast);
}

// e^(G_i - G_j) = 2^(G2_i - G2_j) with G2 = G log2(e), for j <= i (the
// exponent is <= 0 for g <= 0; very old positions underflow to 0).  The SFU's
// 2^x is accurate to about 2^-22 relative, far inside the bf16 rounding of
// the tiles these factors enter.
__device__ __forceinline__ float decay2(float g2i, float g2j) { return ex2_approx(g2i - g2j); }

// Wait (bounded) for a ready flag set with release semantics by another CTA.
__device__ __forceinline__ bool wait_flag(const unsigned int* f, volatile int* abort) {
    if (ld_acquire_gpu(f)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(200);
        if (ld_acquire_gpu(f)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitNs) {
            *abort = 1;
            return false;
        }
    }
}

// Bounded mbarrier waits for a CTA whose roles share an abort flag in shared memory.
struct Ctl {
    uint32_t bar0;                 // address of barrier 0
    volatile int* abort;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
    // gives up after kWaitNs, or early once another role has aborted
    __device__ bool wait(int i, uint32_t parity) const {
        const uint32_t b = bar(i);
        if (mbar_try_wait(b, parity)) return true;
        const uint64_t t0 = globaltimer_ns();
        while (true) {
            if (mbar_try_wait_sleep(b, parity, 20000u)) return true;
            if (*abort) return false;
            if (globaltimer_ns() - t0 > kWaitNs) {
                *abort = 1;
                return false;
            }
        }
    }
};

// ---- host side ---------------------------------------------------------------

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D bf16 tensor [rows][cols] (row-major), boxes of 64 columns x box_rows
// rows, 128-byte swizzle, zero fill past the end.
inline bool make_tmap(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc

// The state-independent part of every chunk into the workspace (chunk_wy.cu;
// chunk_wy_kda.cu for the per-key gate).
cudaError_t launch_chunk_wy(const ChunkArgs& a, const tc::TcMaps& m, cudaStream_t st);
cudaError_t launch_chunk_wy_kda(const ChunkArgs& a, const tc::TcMaps& m, cudaStream_t st);

}  // namespace dn
