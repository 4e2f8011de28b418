// chunk_tc.cu -- the tensor-core prefill: the per-chunk WY transform
// (chunk_wy.cuh) and the sequential state pass (chunk_state.cuh).
//
// Two ways to run them, both with a ready flag per workspace tile:
//   * one cooperative launch (chunk_fused_kernel), one CTA per SM: CTAs
//     0 .. B H - 1 run the state pass of one head each, the others run four
//     groups of 8 warps that take the WY tiles chunk by chunk (chunk 0 of every
//     head first).  A cooperative launch guarantees that every CTA is resident,
//     so the state pass may wait for tiles that other CTAs are writing; the WY
//     work overlaps the latency-bound state pass and its tiles are read while
//     still in L2.  With many heads the WY work is the longer of the two, and
//     each state-pass CTA also hosts a WY group (HOSTED: two stages, one [O|U]
//     buffer).  Used while B H leaves a quarter of the SMs to the WY groups.
//   * otherwise two launches on the stream: chunk_wy_kernel over all tiles,
//     then chunk_state_kernel (whose flags are then all set).
// The per-key gate (KDA) works the same way with its own WY tile
// (chunk_wy_kda.cuh, 88 KiB): chunk_fused_kda_kernel has CTAs of 16 warps, the
// state pass of one head or two KDA WY groups; else chunk_wy_kda_kernel and
// chunk_state_kernel<per-key>.
#include "chunk_state.cuh"
#include "chunk_wy.cuh"
#include "chunk_wy_kda.cuh"
#include "dn_kernels.h"

namespace dn {

using namespace sm100;
using namespace tc;

template <int GATE, int PRO>
__global__ void __launch_bounds__(state::Roles<GATE, false, PRO>::kNT, 1)
chunk_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_u,
                   const __grid_constant__ CUtensorMap tm_p, const unsigned int* __restrict__ flags,
                   const float* __restrict__ beta, const float* __restrict__ g, const float* S0,
                   __nv_bfloat16* __restrict__ o, float* S_T, int T, float scale, unsigned int* status,
                   int test_flags, const float* __restrict__ gam, float* snaps, int snap_every, int n_snap,
                   Prologue pro, const int* vl, int vl_N) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the __shared__ array itself so that
    // every access below compiles to a shared-memory (not generic) instruction
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const state::Args ar{&tm_k, &tm_q, &tm_w, &tm_u, &tm_p, flags, beta, g, S0, o, S_T, T, scale, status, test_flags,
                         gam, snaps, snap_every, n_snap, pro.on, pro.A_log, pro.dt_bias, pro.H, pro.rep, vl, vl_N,
                         pro.norm, pro.z, pro.norm_w, pro.eps, pro.rq, pro.scratch, pro.scratch_tiles};
    state::state_pass<GATE, false, PRO>(sm, ar, blockIdx.x, 0u);
}

// The chunk tables of a packed batch (VarlenTables) from cu_seqlens [N + 1], by
// one CTA: a checked copy of the offsets, each sequence's first global chunk
// (an exclusive prefix sum of ceil(len / 64)) and each global chunk's sequence.
// If cu_seqlens does not rise from 0 to T (non-decreasing), every length is
// taken as zero (nothing runs, every S_T = S0) and bit 1 of the status word is
// set, which dn_device_status reports as DN_ERR_INVALID.
__global__ void __launch_bounds__(1024)
varlen_table_kernel(const int* __restrict__ cu_in, int N, int T, int* tables, unsigned int* status) {
    __shared__ int s_carry, s_bad;
    __shared__ int s_warp[32];
    const VarlenTables vt{tables, N};
    int* cu = tables;
    int* coff = tables + N + 1;
    int* seq_of = tables + 2 * (N + 1);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) { s_carry = 0; s_bad = (cu_in[0] != 0 || cu_in[N] != T) ? 1 : 0; }
    __syncthreads();
    for (int s = tid; s < N; s += blockDim.x)
        if (cu_in[s + 1] < cu_in[s]) s_bad = 1;
    __syncthreads();
    const bool bad = s_bad != 0;
    for (int s = tid; s <= N; s += blockDim.x) cu[s] = bad ? 0 : cu_in[s];
    if (bad && tid == 0) atomicOr(status, 2u);
    // coff = exclusive prefix sum of the chunk counts, 1024 sequences per round
    for (int s0 = 0; s0 <= N; s0 += blockDim.x) {
        const int s = s0 + tid;
        const int nch = (s < N && !bad) ? (cu_in[s + 1] - cu_in[s] + kC - 1) / kC : 0;
        int x = nch;                                          // inclusive scan in the warp
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o2);
            if (lane >= o2) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = s_warp[lane];
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o2);
                if (lane >= o2) w += y;
            }
            s_warp[lane] = w;                                 // inclusive over warps
        }
        __syncthreads();
        const int before = s_carry + (warp > 0 ? s_warp[warp - 1] : 0) + x - nch;
        if (s <= N) coff[s] = before;
        __syncthreads();
        if (tid == blockDim.x - 1) s_carry = before + nch;
        __syncthreads();
    }
    // seq_of: each sequence's chunks
    for (int s = warp; s < N; s += blockDim.x / 32)
        for (int c = coff[s] + lane; c < coff[s + 1]; c += 32) seq_of[c] = s;
    (void)vt;
}

namespace {
constexpr int kFusedThreads = 4 * wy::kNT;          // 32 warps: 4 WY groups, or the state pass + up to 16 more
static_assert(state::kHostedNT + wy::kNT <= kFusedThreads && state::Roles<kGateScalar, false, 2>::kNT <= kFusedThreads,
              "fused CTA size");
constexpr uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }
// a hosted WY group's shared memory starts past the hosted state pass's
constexpr uint32_t kHostedWyOff = align1k(state::Layout<true>::STATE_BYTES);
constexpr uint32_t cmax(uint32_t a, uint32_t b) { return a > b ? a : b; }
constexpr uint32_t kFusedBytes =
    cmax(cmax(state::Layout<false>::STATE_BYTES, 4 * wy::GROUP_BYTES), kHostedWyOff + wy::GROUP_BYTES) + 1024;
static_assert(state::Layout<true>::kCols + wy::TM_COLS <= state::TM_COLS, "hosted TMEM split");
constexpr uint32_t kHostBar = 6;                    // named barrier of the hosting CTA's state pass + WY group
}  // namespace

template <int GATE, bool HOSTED, int PRO>
__global__ void __launch_bounds__(kFusedThreads, 1)
chunk_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_p,
                   __nv_bfloat16* __restrict__ p_out, unsigned int* __restrict__ flags, int BH,
                   const float* __restrict__ beta, const float* __restrict__ g, const float* S0,
                   __nv_bfloat16* __restrict__ o, float* S_T, int T, int n, float scale, unsigned int* status,
                   int test_flags, float* snaps, int snap_every, int n_snap, Prologue pro) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t tiles = (int64_t)BH * n;
    // the tile counter follows the ready flags: each group's first tile is its index,
    // the later ones come from tickets, in order (chunk-major), to whichever group is free
    const int64_t G = (int64_t)(gridDim.x - BH) * 4 + (HOSTED ? BH : 0);   // WY groups in the grid
    const wy::Args wa{&tm_q, &tm_k, &tm_v, &tm_w, &tm_u, p_out, flags, beta, g, T, n, scale, test_flags,
                      flags + tiles, BH, (int)G, pro.on, pro.A_log, pro.dt_bias, pro.H, pro.rep, nullptr, 0,
                      pro.rq};
    if ((int)blockIdx.x < BH) {
        const state::Args ar{&tm_k, &tm_q, &tm_w, &tm_u, &tm_p, flags, beta, g, S0, o, S_T, T, scale, status,
                             test_flags, nullptr, snaps, snap_every, n_snap, pro.on, pro.A_log, pro.dt_bias, pro.H,
                             pro.rep, nullptr, 0, pro.norm, pro.z, pro.norm_w, pro.eps, pro.rq, pro.scratch, pro.scratch_tiles};
        if constexpr (!HOSTED) {
            // ---- state pass of head blockIdx.x --------------------------------------------
            if (warp >= state::Roles<GATE, false, PRO>::kNT / 32) return;
            state::state_pass<GATE, false, PRO>(sm, ar, blockIdx.x, 0u);
            return;
        } else {
        // ---- state pass (warps 0-23) and one WY group (warps 24-31) ------------------------
        constexpr int kStateNT = state::Roles<GATE, true, PRO>::kNT;
        constexpr int kHostThreads = kStateNT + wy::kNT;
        if (tid >= kHostThreads) return;
        uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kHostedWyOff + wy::GROUP_BYTES - 16);
        wy::Group x = wy::make_group(sm + kHostedWyOff, 0u, 4u, tid - kStateNT);
        if (tid == kStateNT) {
            wy::init_group(x);
            fence_mbar_init();
        }
        if (warp == 2) {
            tmem_alloc(smem_u32(tslot), state::TM_COLS);
            tmem_relinquish();
        }
        tc_fence_before();
        named_bar_sync(kHostBar, kHostThreads);
        tc_fence_after();
        const uint32_t tbase = *tslot;
        if (tid < kStateNT) {
            state::state_pass<GATE, true, PRO>(sm, ar, blockIdx.x, tbase);
        } else {
            x.tmem = tbase + state::Layout<true>::kCols;
            bool ok = true;
            int64_t pending = -1;
            for (int64_t t = (int64_t)(gridDim.x - BH) * 4 + blockIdx.x; ok && t < tiles;) {
                const int c = (int)(t / BH);
                ok = wy::wy_tile<GATE, (PRO != 0)>(x, wa, c, t - (int64_t)c * BH, pending);
                if (ok) t = G + (int64_t)wy::next_ticket(x);
            }
            if (ok && x.tid == wy::kStoreTid) wy::publish_pending(wa, pending);
            if (!ok && x.tid == 0) atomicOr(status, 1u);
        }
        tc_fence_before();
        named_bar_sync(kHostBar, kHostThreads);
        if (warp == 2) {
            tc_fence_after();
            tmem_dealloc(tbase, state::TM_COLS);
        }
        return;
        }
    }
    // ---- four WY groups, each taking every G-th tile in chunk-major order -----------------
    const int grp = warp >> 3;                       // 0..3
    const uint32_t* tmem_slot = reinterpret_cast<const uint32_t*>(sm + 4 * wy::GROUP_BYTES - 16);
    wy::Group x = wy::make_group(sm + grp * wy::GROUP_BYTES, 0u, 1u + (uint32_t)grp, tid - grp * wy::kNT);
    if (x.tid == 0) {
        wy::init_group(x);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 4 * wy::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = *tmem_slot + (uint32_t)grp * wy::TM_COLS;
    bool ok = true;
    int64_t pending = -1;
    for (int64_t t = (int64_t)(blockIdx.x - BH) * 4 + grp; ok && t < tiles;) {
        const int c = (int)(t / BH);
        ok = wy::wy_tile<GATE, (PRO != 0)>(x, wa, c, t - (int64_t)c * BH, pending);
        if (ok) t = G + (int64_t)wy::next_ticket(x);
    }
    if (ok && x.tid == wy::kStoreTid) wy::publish_pending(wa, pending);
    tc_fence_before();
    __syncthreads();
    if (!ok && x.tid == 0) atomicOr(status, 1u);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*tmem_slot, 4 * wy::TM_COLS);
    }
}

// ---- host side ---------------------------------------------------------------

constexpr int kFusedKdaThreads = 2 * kda::kNT;     // 16 warps: two KDA WY groups, or the state pass
static_assert(state::Roles<kGatePerKey>::kNT == kFusedKdaThreads, "fused KDA CTA size");
constexpr uint32_t kFusedKdaBytes =
    (state::Layout<false>::STATE_BYTES > 2 * kda::GROUP_BYTES ? state::Layout<false>::STATE_BYTES
                                                               : 2 * kda::GROUP_BYTES) + 1024;

// The per-key-gate prefill in one cooperative launch: CTAs 0 .. BH - 1 run the
// state pass of one head each (reading Qh, K~ and the decays from the
// workspace); the others run two KDA WY groups over the tiles, chunk-major.
__global__ void __launch_bounds__(kFusedKdaThreads, 1)
chunk_fused_kda_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_p,
                       const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_qh,
                       __nv_bfloat16* p_out, __nv_bfloat16* kt_out, __nv_bfloat16* qh_out, float* gam,
                       unsigned int* flags, int BH, const float* __restrict__ beta, const float* __restrict__ g,
                       const float* S0, __nv_bfloat16* __restrict__ o, float* S_T, int T, int n, float scale,
                       unsigned int* status, int test_flags, float* snaps, int snap_every, int n_snap,
                       uint8_t* scratch, long long scratch_tiles) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    if ((int)blockIdx.x < BH) {
        const state::Args ar{&tm_kt, &tm_qh, &tm_w, &tm_u, &tm_p, flags, beta, g, S0, o, S_T, T, scale, status,
                             test_flags, gam, snaps, snap_every, n_snap, 0, nullptr, nullptr, 1, 1, nullptr, 0, 0,
                             nullptr, nullptr, 0.f, nullptr, scratch, scratch_tiles};
        state::state_pass<kGatePerKey, false, 0>(sm, ar, blockIdx.x, 0u);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5;
    const int grp = warp >> 3;                       // 0, 1
    const uint32_t* tmem_slot = reinterpret_cast<const uint32_t*>(sm + 2 * kda::GROUP_BYTES - 16);
    kda::Group x = kda::make_group(sm + grp * kda::GROUP_BYTES, 0u, 1u + (uint32_t)grp, tid - grp * kda::kNT);
    if (x.tid == 0) {
        kda::init_group(x);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 2 * kda::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = *tmem_slot + (uint32_t)grp * kda::TM_COLS;
    const int64_t tiles = (int64_t)BH * n;
    // first tile by group index, then tickets from the counter after the flags
    const int64_t G = (int64_t)(gridDim.x - BH) * 2;      // WY groups in the grid
    const kda::Args wa{&tm_q, &tm_k, &tm_v, &tm_w, &tm_u, p_out, kt_out, qh_out, gam, flags, beta, g,
                       T, n, scale, test_flags, flags + tiles, BH, (int)G};
    bool ok = true;
    int64_t pending = -1;
    for (int64_t t = (int64_t)(blockIdx.x - BH) * 2 + grp; ok && t < tiles;) {
        const int c = (int)(t / BH);
        ok = kda::kda_tile(x, wa, c, t - (int64_t)c * BH, pending);
        if (ok) t = G + (int64_t)kda::next_ticket(x);
    }
    if (ok && x.tid == kda::kStoreTid) kda::publish_pending(wa, pending);
    tc_fence_before();
    __syncthreads();
    if (!ok && x.tid == 0) atomicOr(status, 1u);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*tmem_slot, 2 * kda::TM_COLS);
    }
}

namespace {

// The single-launch prefill needs one resident CTA per SM and leaves at least
// a quarter of them (and 16) to the WY groups.
bool fused_fits(int64_t BH, int num_sms) {
    return BH + 16 <= num_sms && BH * 4 <= (int64_t)num_sms * 3;
}

template <int GATE, int PRO>
cudaError_t launch_tc_gate(const ChunkArgs& a, cudaStream_t st) {
    const uint64_t rows = (uint64_t)(a.B * a.H * a.T);
    const uint64_t krows = rows / (uint64_t)a.rep;          // q and k: H / rep heads
    const int n = (int)((a.T + kC - 1) / kC);
    const bool packed = a.cu_seqlens != nullptr;
    // a packed batch: tiles of H heads x the most chunks its tokens can make
    const uint64_t tiles = (uint64_t)(a.B * a.H) * (uint64_t)(packed ? vl_chunks_max(a.T, a.N) : n);
    uint8_t* w_ws = static_cast<uint8_t*>(a.ws);
    uint8_t* u_ws = w_ws + tiles * kWsWBytes;
    uint8_t* p_ws = u_ws + tiles * kWsUBytes;
    TcMaps m;
    if (!make_tmap(&m.q, a.q, kD, krows, 64) || !make_tmap(&m.k, a.k, kD, krows, 64) ||
        !make_tmap(&m.v, a.v, kD, rows, 64) || !make_tmap(&m.w, w_ws, kD, tiles * kC, 64) ||
        !make_tmap(&m.u, u_ws, kC, tiles * kD, 128) || !make_tmap(&m.p, p_ws, kC, tiles * kC, 64))
        return cudaErrorInvalidValue;
    m.p_ws = reinterpret_cast<__nv_bfloat16*>(p_ws);
    m.rq_ws = reinterpret_cast<float*>(p_ws + tiles * kWsPBytes);
    m.scratch = drop_scratch(w_ws, tiles * kWsTileBytes);
    m.tiles = tiles;
    m.flags = reinterpret_cast<unsigned int*>(w_ws + ws_flags_offset(tiles));
    if (packed) {
        // the chunk tables, then all WY tiles, then one state pass per (sequence, head)
        int* vl = reinterpret_cast<int*>(w_ws + ws_total_bytes(tiles));
        m.vl = vl;
        varlen_table_kernel<<<1, 1024, 0, st>>>(a.cu_seqlens, a.N, (int)a.T, vl, a.status);
        cudaError_t e = counted(cudaGetLastError());
        if (e != cudaSuccess) return e;
        e = launch_chunk_wy(a, m, st);
        if (e != cudaSuccess) return e;
        auto kern = chunk_state_kernel<GATE, PRO>;
        const uint32_t bytes = state::Layout<false>::STATE_BYTES + 1024;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)(a.N * a.H), state::Roles<GATE, false, PRO>::kNT, bytes, st>>>(
            m.k, m.q, m.w, m.u, m.p, nullptr, a.beta, a.g, a.S0, static_cast<__nv_bfloat16*>(a.o), a.S_T, (int)a.T,
            a.scale, a.status, a.test_flags, nullptr, nullptr, 1, 0,
            prologue_of(a, m), vl, a.N);
        return counted(cudaGetLastError());
    }

    int dev = 0, num_sms = 0, coop = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (e != cudaSuccess) return e;
    const int64_t BH = a.B * a.H;
    if (coop && fused_fits(BH, num_sms)) {
        // with many heads the dedicated WY groups get scarce: the state-pass CTAs
        // host one each (measured: at 64 heads of 148 SMs hosting is not yet a gain);
        // the gated norm's state pass needs its SM's shared memory alone
        auto kern = chunk_fused_kernel<GATE, false, PRO>;
        if constexpr (PRO != 2)
            if (BH * 2 > (int64_t)num_sms + 12) kern = chunk_fused_kernel<GATE, true, PRO>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedBytes);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedThreads, kFusedBytes);
        if (e != cudaSuccess) return e;
        if (per_sm >= 1) {
            int bh_i = (int)BH, T_i = (int)a.T, n_i = n;
            float scale = a.scale;
            int test_flags = a.test_flags;
            __nv_bfloat16* p_out = m.p_ws;
            unsigned int* flags = m.flags;
            const float* beta = a.beta;
            const float* g = a.g;
            const float* S0 = a.S0;
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);
            float* S_T = a.S_T;
            unsigned int* status = a.status;
            float* snaps = a.snaps;
            int snap_every = a.snap_every, n_snap = a.n_snap;
            Prologue pro = prologue_of(a, m);
            void* args[] = {&m.q, &m.k, &m.v, &m.w, &m.u, &m.p, &p_out, &flags, &bh_i, &beta, &g, &S0, &o, &S_T,
                            &T_i, &n_i, &scale, &status, &test_flags, &snaps, &snap_every, &n_snap, &pro};
            // the flags are cleared on the same stream right before the launch
            e = cudaMemsetAsync(m.flags, 0, ws_flag_words(tiles) * 4, st);
            if (e != cudaSuccess) return e;
            return counted(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3((unsigned)num_sms),
                                                       dim3(kFusedThreads), args, kFusedBytes, st));
        }
    }
    e = launch_chunk_wy(a, m, st);
    if (e != cudaSuccess) return e;
    auto kern = chunk_state_kernel<GATE, PRO>;
    const uint32_t bytes = state::Layout<false>::STATE_BYTES + 1024;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    // the WY kernel has finished before this launch starts: no flags to wait for
    kern<<<(unsigned)BH, state::Roles<GATE, false, PRO>::kNT, bytes, st>>>(m.k, m.q, m.w, m.u, m.p, nullptr, a.beta, a.g, a.S0,
                                                  static_cast<__nv_bfloat16*>(a.o), a.S_T, (int)a.T, a.scale,
                                                  a.status, a.test_flags, nullptr, a.snaps, a.snap_every, a.n_snap,
                                                  prologue_of(a, m),
                                                  nullptr, 0);
    return counted(cudaGetLastError());
}

// Per-key gate (KDA): the WY kernel for it (chunk_wy_kda.cu) over all tiles,
// then the state pass, which reads Qh, K~ and the decays from the workspace.
cudaError_t launch_tc_kda(const ChunkArgs& a, cudaStream_t st) {
    const uint64_t rows = (uint64_t)(a.B * a.H * a.T);
    const int n = (int)((a.T + kC - 1) / kC);
    const uint64_t tiles = (uint64_t)(a.B * a.H) * (uint64_t)n;
    uint8_t* w_ws = static_cast<uint8_t*>(a.ws);
    uint8_t* u_ws = w_ws + tiles * kWsWBytes;
    uint8_t* p_ws = u_ws + tiles * kWsUBytes;
    uint8_t* kt_ws = p_ws + tiles * (kWsPBytes + kWsRqBytes);
    uint8_t* qh_ws = kt_ws + tiles * kWsKtBytes;
    uint8_t* gam_ws = qh_ws + tiles * kWsQhBytes;
    TcMaps m;
    if (!make_tmap(&m.q, a.q, kD, rows, 64) || !make_tmap(&m.k, a.k, kD, rows, 64) ||
        !make_tmap(&m.v, a.v, kD, rows, 64) || !make_tmap(&m.w, w_ws, kD, tiles * kC, 64) ||
        !make_tmap(&m.u, u_ws, kC, tiles * kD, 128) || !make_tmap(&m.p, p_ws, kC, tiles * kC, 64) ||
        !make_tmap(&m.kt, kt_ws, kD, tiles * kC, 64) || !make_tmap(&m.qh, qh_ws, kD, tiles * kC, 64))
        return cudaErrorInvalidValue;
    m.p_ws = reinterpret_cast<__nv_bfloat16*>(p_ws);
    m.kt_ws = reinterpret_cast<__nv_bfloat16*>(kt_ws);
    m.qh_ws = reinterpret_cast<__nv_bfloat16*>(qh_ws);
    m.gam_ws = reinterpret_cast<float*>(gam_ws);
    m.flags = reinterpret_cast<unsigned int*>(w_ws + ws_flags_offset(tiles, true));
    m.scratch = drop_scratch(w_ws, tiles * kWsKdaTileBytes);
    m.tiles = tiles;

    int dev = 0, num_sms = 0, coop = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (e != cudaSuccess) return e;
    const int64_t BH = a.B * a.H;
    if (coop && fused_fits(BH, num_sms)) {
        auto kern = chunk_fused_kda_kernel;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedKdaBytes);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedKdaThreads, kFusedKdaBytes);
        if (e != cudaSuccess) return e;
        if (per_sm >= 1) {
            int bh_i = (int)BH, T_i = (int)a.T, n_i = n;
            float scale = a.scale;
            int test_flags = a.test_flags;
            __nv_bfloat16* p_out = m.p_ws;
            __nv_bfloat16* kt_out = m.kt_ws;
            __nv_bfloat16* qh_out = m.qh_ws;
            float* gam = m.gam_ws;
            unsigned int* flags = m.flags;
            const float* beta = a.beta;
            const float* g = a.g;
            const float* S0 = a.S0;
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);
            float* S_T = a.S_T;
            unsigned int* status = a.status;
            float* snaps = a.snaps;
            int snap_every = a.snap_every, n_snap = a.n_snap;
            uint8_t* scratch = m.scratch;
            long long scratch_tiles = (long long)m.tiles;
            void* args[] = {&m.q, &m.k, &m.v, &m.w, &m.u, &m.p, &m.kt, &m.qh, &p_out, &kt_out, &qh_out, &gam,
                            &flags, &bh_i, &beta, &g, &S0, &o, &S_T, &T_i, &n_i, &scale, &status, &test_flags,
                            &snaps, &snap_every, &n_snap, &scratch, &scratch_tiles};
            // the flags are cleared on the same stream right before the launch
            e = cudaMemsetAsync(m.flags, 0, ws_flag_words(tiles) * 4, st);
            if (e != cudaSuccess) return e;
            return counted(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3((unsigned)num_sms),
                                                       dim3(kFusedKdaThreads), args, kFusedKdaBytes, st));
        }
    }
    e = launch_chunk_wy_kda(a, m, st);
    if (e != cudaSuccess) return e;
    auto kern = chunk_state_kernel<kGatePerKey, 0>;
    const uint32_t bytes = state::Layout<false>::STATE_BYTES + 1024;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.B * a.H), state::Roles<kGatePerKey>::kNT, bytes, st>>>(m.kt, m.qh, m.w, m.u, m.p, nullptr, a.beta, a.g, a.S0,
                                                          static_cast<__nv_bfloat16*>(a.o), a.S_T, (int)a.T,
                                                          a.scale, a.status, a.test_flags, m.gam_ws, a.snaps,
                                                          a.snap_every, a.n_snap, prologue_of(a, m), nullptr, 0);
    return counted(cudaGetLastError());
}

}  // namespace

bool tc_supports(const ChunkArgs& a) {
    const int64_t n = a.cu_seqlens ? vl_chunks_max(a.T, a.N) : (a.T + kC - 1) / kC;
    return a.bf16 && a.chunk == kC && a.dk == kD && a.dv == kD &&
           a.B * a.H * a.T < (int64_t(1) << 31) && a.B * a.H * n * kD < (int64_t(1) << 31);
}

size_t tc_workspace_bytes(const ChunkArgs& a) {
    if (a.cu_seqlens) {
        // a packed batch: tiles for the most chunks its tokens can make, then its chunk tables
        const int64_t nc = vl_chunks_max(a.T, a.N);
        return ws_total_bytes((uint64_t)(a.H * nc)) + ((vl_table_ints(a.N, nc) * 4 + 255) / 256) * 256;
    }
    const int64_t n = (a.T + kC - 1) / kC;
    return ws_total_bytes((uint64_t)(a.B * a.H * n), a.gate == kGatePerKey);
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t st) {
    if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    if (a.gate == kGatePerKey) return launch_tc_kda(a, st);
    // the layer prologue (scalar gate), with or without the gated RMSNorm on the output rows
    if (a.prologue) return a.norm ? launch_tc_gate<kGateScalar, 2>(a, st) : launch_tc_gate<kGateScalar, 1>(a, st);
    return a.gate == kGateScalar ? launch_tc_gate<kGateScalar, 0>(a, st) : launch_tc_gate<kGateNone, 0>(a, st);
}

}  // namespace dn
