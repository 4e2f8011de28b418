// layer_ops.cu -- the two Gated DeltaNet layer steps on either side of the rule
// ("Linear attention and Gated DeltaNet", ch. 28, "The full layer"):
//
//   step 2, the short causal convolution over time (one length-K filter per
//   channel, then SiLU) with the previous K-1 inputs carried as its state;
//   step 7, the gated RMSNorm of each head's output row.
//
// Both are streaming work bound by HBM: vector loads across channels (coalesced),
// fp32 arithmetic, one rounding at the store.
#include <cuda_bf16.h>
#include <stdint.h>

#include "dn_kernels.h"
#include "sm100.cuh"

namespace dn {
namespace {

// ---- element access: V consecutive channels as one vector (or scalar) access ----------

template <typename T, int V>
struct Vec;
template <>
struct Vec<float, 4> {
    using raw = float4;
    __device__ static void to_f(const raw& r, float* f) { f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w; }
    __device__ static raw from_f(const float* f) { return make_float4(f[0], f[1], f[2], f[3]); }
};
template <>
struct Vec<float, 1> {
    using raw = float;
    __device__ static void to_f(const raw& r, float* f) { f[0] = r; }
    __device__ static raw from_f(const float* f) { return f[0]; }
};
template <>
struct Vec<__nv_bfloat16, 8> {
    using raw = uint4;
    __device__ static void to_f(const raw& r, float* f) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 p = __bfloat1622float2(h[e]);
            f[2 * e] = p.x;
            f[2 * e + 1] = p.y;
        }
    }
    __device__ static raw from_f(const float* f) {
        raw r;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
        return r;
    }
};
template <>
struct Vec<__nv_bfloat16, 1> {
    using raw = __nv_bfloat16;
    __device__ static void to_f(const raw& r, float* f) { f[0] = __bfloat162float(r); }
    __device__ static raw from_f(const float* f) { return __float2bfloat16_rn(f[0]); }
};
template <>
struct Vec<__nv_bfloat16, 2> {
    using raw = __nv_bfloat162;
    __device__ static void to_f(const raw& r, float* f) {
        const float2 p = __bfloat1622float2(r);
        f[0] = p.x;
        f[1] = p.y;
    }
    __device__ static raw from_f(const float* f) { return __floats2bfloat162_rn(f[0], f[1]); }
};
template <>
struct Vec<__nv_bfloat16, 4> {
    using raw = uint2;
    __device__ static void to_f(const raw& r, float* f) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float2 p = __bfloat1622float2(h[e]);
            f[2 * e] = p.x;
            f[2 * e + 1] = p.y;
        }
    }
    __device__ static raw from_f(const float* f) {
        raw r;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
        h[0] = __floats2bfloat162_rn(f[0], f[1]);
        h[1] = __floats2bfloat162_rn(f[2], f[3]);
        return r;
    }
};
template <>
struct Vec<float, 2> {
    using raw = float2;
    __device__ static void to_f(const raw& r, float* f) { f[0] = r.x; f[1] = r.y; }
    __device__ static raw from_f(const float* f) { return make_float2(f[0], f[1]); }
};

// SiLU and the logistic sigmoid through the fast exp and the approximate reciprocal
// (a few ulp, far inside a bf16 rounding): for very negative x the exp overflows to
// inf and 1 / inf gives 0, the right limit
__device__ __forceinline__ float sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
__device__ __forceinline__ float silu(float x) { return x * sigmoid(x); }

// ---- causal conv ----------------------------------------------------------------------
//
// Thread = V consecutive channels of one sequence over kConvRows consecutive tokens.
// The block's filters are staged once in shared memory, tap-major, from coalesced
// reads.  A thread's rows, plus the K-1 before them (from x, or from the carried state
// before token 0), are loaded up front so that every load of the tile is in flight at
// once; the filter then slides over them in registers.  The block whose tile holds the
// last token also writes the new state (the last K-1 inputs of history-then-x).

constexpr int kConvRows = 16;
constexpr int kConvThreads = 128;

template <typename Tin, int V, int K, bool ACT>
__global__ void __launch_bounds__(kConvThreads)
causal_conv1d_kernel(const Tin* __restrict__ x, int64_t ld_x, const float* __restrict__ w, const Tin* s_in,
                     Tin* __restrict__ y, Tin* s_out, int T, int C, int hd) {
    using VT = Vec<Tin, V>;
    using raw = typename VT::raw;
    constexpr int kCh = kConvThreads * V;       // channels of the block
    constexpr int kRow = kCh + 4;               // padded tap row: 16-byte aligned, banks shifted
    constexpr int kPer = (kCh * K + kConvThreads - 1) / kConvThreads;   // filter values per thread
    __shared__ __align__(16) float ws[K][kRow];
    const int cb0 = blockIdx.x * kCh;
    const int nch = min(kCh, C - cb0);
    const int cl = threadIdx.x * V;
    const int c0 = cb0 + cl;
    const bool active = c0 < C;
    const int64_t b = blockIdx.z;
    const int t0 = blockIdx.y * kConvRows;

    // input row t of this thread's channels: x for t >= 0, the carried state before
    const Tin* xb = x + b * T * ld_x + c0;
    const Tin* sb = s_in ? s_in + b * (K - 1) * (int64_t)C + c0 : nullptr;
    auto load_row = [&](int t, float* f) {
        if (t >= 0) {
            VT::to_f(*reinterpret_cast<const raw*>(xb + (int64_t)t * ld_x), f);
        } else if (sb) {
            VT::to_f(*reinterpret_cast<const raw*>(sb + (int64_t)(t + K - 1) * C), f);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) f[v] = 0.f;
        }
    };

    // the tile's rows first, so that their loads overlap the filter staging
    raw rows[K - 1 + kConvRows];
    if (active) {
#pragma unroll
        for (int i = 0; i < K - 1 + kConvRows; ++i) {
            const int t = t0 - (K - 1) + i;
            if (t < 0) {
                float f[V];
                load_row(t, f);
                rows[i] = VT::from_f(f);
            } else if (t < T) {
                rows[i] = *reinterpret_cast<const raw*>(xb + (int64_t)t * ld_x);
            }
        }
    }
    // the block's filters, tap-major in shared memory: every load issued before any store
    {
        float wv[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int e = threadIdx.x + u * kConvThreads;
            wv[u] = e < nch * K ? w[(int64_t)cb0 * K + e] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int e = threadIdx.x + u * kConvThreads;
            if (e < nch * K) {
                const int ch = e / K;
                ws[e - ch * K][ch] = wv[u];
            }
        }
    }
    __syncthreads();
    if (!active) return;

    float wf[K][V];
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if constexpr (V % 4 == 0) {
#pragma unroll
            for (int v = 0; v < V; v += 4) {
                const float4 f = *reinterpret_cast<const float4*>(&ws[j][cl + v]);
                wf[j][v] = f.x; wf[j][v + 1] = f.y; wf[j][v + 2] = f.z; wf[j][v + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) wf[j][v] = ws[j][cl + v];
        }
    }
    // rows before token 0 were rounded back to Tin above; they are Tin values already
    // (the state has x's dtype), so the round trip is exact

    const int nh = C / hd;
    const int head = c0 / hd, jj = c0 - head * hd;
    Tin* yb = y + ((b * nh + head) * (int64_t)T) * hd + jj;
    // sliding window of the K input rows behind output t, as floats: each row is
    // converted once
    float win[K][V];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) VT::to_f(rows[j], win[j]);
#pragma unroll
    for (int i = 0; i < kConvRows; ++i) {
        const int t = t0 + i;
        if (t < T) {
            VT::to_f(rows[i + K - 1], win[K - 1]);
            float acc[V];
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = 0.f;
#pragma unroll
            for (int j = 0; j < K; ++j)
#pragma unroll
                for (int v = 0; v < V; ++v) acc[v] = fmaf(wf[j][v], win[j][v], acc[v]);
            if (ACT) {
#pragma unroll
                for (int v = 0; v < V; ++v) acc[v] = silu(acc[v]);
            }
            *reinterpret_cast<raw*>(yb + (int64_t)t * hd) = VT::from_f(acc);
#pragma unroll
            for (int j = 0; j < K - 1; ++j)
#pragma unroll
                for (int v = 0; v < V; ++v) win[j][v] = win[j + 1][v];
        }
    }

    if (s_out && K > 1 && t0 + kConvRows >= T) {
        // new state row j = input row T-K+1+j; read all of them before the first write
        // (s_out may be s_in itself when the whole sequence is this one tile)
        float sv[K > 1 ? K - 1 : 1][V];
#pragma unroll
        for (int j = 0; j < K - 1; ++j) load_row(T - (K - 1) + j, sv[j]);
        Tin* so = s_out + b * (K - 1) * (int64_t)C + c0;
#pragma unroll
        for (int j = 0; j < K - 1; ++j) *reinterpret_cast<raw*>(so + (int64_t)j * C) = VT::from_f(sv[j]);
    }
}

// Tiled form for layouts that allow 16-byte accesses.  A block owns 32 vectors of
// V = 16 / sizeof(Tin) channels of one sequence (their filters stay in registers)
// and a run of 32-token tiles of it.  Each tile and the K-1 rows before it (x, or
// the carried state before token 0, or zeros) are copied into shared memory by
// cp.async, the next tile while the current one is computed (two buffers); each
// thread slides its channels' filter over 8 consecutive rows from there and
// stores 16 bytes a row.  The block of the last tile also writes the new state
// from the same rows.
constexpr int kTileRows = 32;
constexpr int kConvStages = 2;                           // tiles in flight per block
constexpr int kConvWarps = 4;                            // each thread: 32 / kConvWarps rows of a tile

template <typename Tin, int K>
struct ConvTile {
    static constexpr int V = 16 / (int)sizeof(Tin);
    static constexpr int kCh = 32 * V;                   // channels of a block
    static constexpr int kRowsIn = kTileRows + K - 1;
    Tin rows[kConvStages][kRowsIn][kCh];
};

template <typename Tin, int K, bool ACT>
__global__ void __launch_bounds__(kConvWarps * 32)
causal_conv1d_tile_kernel(const Tin* __restrict__ x, int64_t ld_x, const float* __restrict__ w, const Tin* s_in,
                          Tin* __restrict__ y, Tin* s_out, int T, int C, int hd, int run) {
    using CT = ConvTile<Tin, K>;
    constexpr int V = CT::V, kCh = CT::kCh, kRowsIn = CT::kRowsIn;
    constexpr int kNT = kConvWarps * 32, kRPT = kTileRows / kConvWarps;   // threads; rows per thread
    using VT = Vec<Tin, V>;
    using raw = typename VT::raw;
    extern __shared__ __align__(16) unsigned char conv_smem[];
    CT& sm = *reinterpret_cast<CT*>(conv_smem);
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int cb0 = blockIdx.x * kCh;
    const int64_t b = blockIdx.z;
    const int n_tiles = T > 0 ? (T + kTileRows - 1) / kTileRows : 1;
    const int tile_beg = blockIdx.y * run, tile_end = min(n_tiles, tile_beg + run);
    if (tile_beg >= tile_end) return;
    // rows t0 - (K-1) .. t0 + 31 of the block's channels into buffer buf; zero past
    // the sequence or C
    auto fetch = [&](int tile, int buf) {
        const int t0 = tile * kTileRows;
        for (int idx = threadIdx.x; idx < kRowsIn * 32; idx += kNT) {
            const int r = idx >> 5, cv = idx & 31;
            const int t = t0 - (K - 1) + r, c = cb0 + cv * V;
            const Tin* src = nullptr;
            if (c < C) {
                if (t >= 0 && t < T) src = x + (b * T + t) * ld_x + c;
                else if (t < 0 && s_in) src = s_in + (b * (K - 1) + (t + K - 1)) * (int64_t)C + c;
            }
            if (src) sm100::cp_async16(sm100::smem_u32(&sm.rows[buf][r][cv * V]), src, 16);
            else *reinterpret_cast<uint4*>(&sm.rows[buf][r][cv * V]) = make_uint4(0u, 0u, 0u, 0u);
        }
        sm100::cp_async_commit();
    };
#pragma unroll
    for (int s = 0; s < kConvStages - 1; ++s)
        if (tile_beg + s < tile_end) fetch(tile_beg + s, s);
    // the thread's filters while the rows land: channels c0 .. c0 + V - 1, K taps each,
    // V K consecutive floats of w
    const int c0 = cb0 + tx * V;
    const bool active = c0 < C;
    float wf[K][V];
    {
        float wl[V * K];
#pragma unroll
        for (int u = 0; u < V * K / 4; ++u) {
            const float4 f = active ? reinterpret_cast<const float4*>(w + (int64_t)c0 * K)[u]
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            wl[4 * u] = f.x; wl[4 * u + 1] = f.y; wl[4 * u + 2] = f.z; wl[4 * u + 3] = f.w;
        }
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int j = 0; j < K; ++j) wf[j][v] = wl[v * K + j];
    }
    const int nh = C / hd;
    const int head = c0 / hd, jj = c0 - head * hd;
    Tin* yb = y + ((b * nh + (active ? head : 0)) * (int64_t)T) * hd + jj;
    const int r0 = ty * kRPT;                             // the thread's first output row of a tile
    for (int tile = tile_beg; tile < tile_end; ++tile) {
        const int buf = (tile - tile_beg) % kConvStages;
        // the tile kConvStages - 1 ahead into the buffer read one tile ago (the barrier at
        // the end of that tile is behind every thread), then wait for this tile's rows
        const int ahead = tile + kConvStages - 1;
        if (ahead < tile_end) fetch(ahead, (ahead - tile_beg) % kConvStages);
        const int later = min(tile_end - 1, ahead) - tile;     // groups committed after this tile's
        if (later >= 2) sm100::cp_async_wait_group<2>();
        else if (later == 1) sm100::cp_async_wait_group<1>();
        else sm100::cp_async_wait_group<0>();
        __syncthreads();
        const int t0 = tile * kTileRows;
        if (active) {
            float win[K][V];
#pragma unroll
            for (int j = 0; j < K - 1; ++j) VT::to_f(*reinterpret_cast<const raw*>(&sm.rows[buf][r0 + j][tx * V]), win[j]);
#pragma unroll
            for (int i = 0; i < kRPT; ++i) {
                const int t = t0 + r0 + i;
                VT::to_f(*reinterpret_cast<const raw*>(&sm.rows[buf][r0 + i + K - 1][tx * V]), win[K - 1]);
                float acc[V];
                if constexpr (V % 2 == 0) {
                    // channel pairs through packed fp32 (the kernel is bound by instruction issue)
#pragma unroll
                    for (int v = 0; v < V; v += 2) {
                        float2 a = make_float2(0.f, 0.f);
#pragma unroll
                        for (int j = 0; j < K; ++j)
                            a = sm100::fma2(make_float2(wf[j][v], wf[j][v + 1]), make_float2(win[j][v], win[j][v + 1]), a);
                        if (ACT) a = sm100::silu2(a);
                        acc[v] = a.x;
                        acc[v + 1] = a.y;
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        float a = 0.f;
#pragma unroll
                        for (int j = 0; j < K; ++j) a = fmaf(wf[j][v], win[j][v], a);
                        acc[v] = ACT ? silu(a) : a;
                    }
                }
                if (t < T) *reinterpret_cast<raw*>(yb + (int64_t)t * hd) = VT::from_f(acc);
#pragma unroll
                for (int j = 0; j < K - 1; ++j)
#pragma unroll
                    for (int v = 0; v < V; ++v) win[j][v] = win[j + 1][v];
            }
            if (s_out && K > 1 && ty == 0 && t0 + kTileRows >= T) {
                // new state row j = input row T - K + 1 + j, local row T - t0 + j (all read
                // into shared memory above, so s_out may be s_in itself when this is the
                // only tile)
#pragma unroll
                for (int j = 0; j < K - 1; ++j)
                    *reinterpret_cast<uint4*>(s_out + (b * (K - 1) + j) * (int64_t)C + c0) =
                        *reinterpret_cast<const uint4*>(&sm.rows[buf][T - t0 + j][tx * V]);
            }
        }
        __syncthreads();                                   // buf is refilled from the next tile on
    }
}

template <typename Tin, int K>
cudaError_t launch_conv_tile_k(const ConvArgs& a, cudaStream_t st) {
    constexpr int kCh = ConvTile<Tin, K>::kCh;
    const int n_tiles = a.T > 0 ? (a.T + kTileRows - 1) / kTileRows : 1;
    const int n_cb = (a.C + kCh - 1) / kCh;
    // about four blocks per SM, each a run of consecutive tiles of one (sequence, channel block)
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    constexpr int kBytes = (int)sizeof(ConvTile<Tin, K>);
    if (kBytes > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(a.activation ? causal_conv1d_tile_kernel<Tin, K, true>
                                                                : causal_conv1d_tile_kernel<Tin, K, false>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kBytes);
        if (e != cudaSuccess) return e;
    }
    const int64_t pairs = (int64_t)n_cb * a.B;
    const int64_t want = (4 * (int64_t)sms + pairs - 1) / pairs;
    const int splits = (int)(want < 1 ? 1 : want > n_tiles ? n_tiles : want);
    const int run = (n_tiles + splits - 1) / splits;
    const dim3 grid((unsigned)n_cb, (unsigned)((n_tiles + run - 1) / run), (unsigned)a.B);
    const Tin* x = static_cast<const Tin*>(a.x);
    const Tin* s_in = static_cast<const Tin*>(a.state_in);
    Tin* y = static_cast<Tin*>(a.y);
    Tin* s_out = static_cast<Tin*>(a.state_out);
    if (a.activation)
        causal_conv1d_tile_kernel<Tin, K, true><<<grid, kConvWarps * 32, kBytes, st>>>(
            x, a.ld_x, a.weight, s_in, y, s_out, a.T, a.C, a.head_dim, run);
    else
        causal_conv1d_tile_kernel<Tin, K, false><<<grid, kConvWarps * 32, kBytes, st>>>(
            x, a.ld_x, a.weight, s_in, y, s_out, a.T, a.C, a.head_dim, run);
    return counted(cudaGetLastError());
}

template <typename Tin>
cudaError_t launch_conv_tile(const ConvArgs& a, cudaStream_t st) {
    switch (a.K) {
        case 1: return launch_conv_tile_k<Tin, 1>(a, st);
        case 2: return launch_conv_tile_k<Tin, 2>(a, st);
        case 3: return launch_conv_tile_k<Tin, 3>(a, st);
        default: return launch_conv_tile_k<Tin, 4>(a, st);
    }
}

template <typename Tin, int V, int K>
cudaError_t launch_conv_k(const ConvArgs& a, cudaStream_t st) {
    const int n_cv = a.C / V;
    const int tiles = a.T > 0 ? (a.T + kConvRows - 1) / kConvRows : 1;
    const dim3 grid((unsigned)((n_cv + kConvThreads - 1) / kConvThreads), (unsigned)tiles, (unsigned)a.B);
    const Tin* x = static_cast<const Tin*>(a.x);
    const Tin* s_in = static_cast<const Tin*>(a.state_in);
    Tin* y = static_cast<Tin*>(a.y);
    Tin* s_out = static_cast<Tin*>(a.state_out);
    if (a.activation)
        causal_conv1d_kernel<Tin, V, K, true><<<grid, kConvThreads, 0, st>>>(x, a.ld_x, a.weight, s_in, y, s_out,
                                                                             a.T, a.C, a.head_dim);
    else
        causal_conv1d_kernel<Tin, V, K, false><<<grid, kConvThreads, 0, st>>>(x, a.ld_x, a.weight, s_in, y, s_out,
                                                                              a.T, a.C, a.head_dim);
    return counted(cudaGetLastError());
}

template <typename Tin, int V>
cudaError_t launch_conv_v(const ConvArgs& a, cudaStream_t st) {
    switch (a.K) {
        case 1: return launch_conv_k<Tin, V, 1>(a, st);
        case 2: return launch_conv_k<Tin, V, 2>(a, st);
        case 3: return launch_conv_k<Tin, V, 3>(a, st);
        default: return launch_conv_k<Tin, V, 4>(a, st);
    }
}

// ---- gated RMSNorm ------------------------------------------------------------------------
//
// One warp per output row (b, t, h) of D channels, D / 32 consecutive channels per lane.
// A warp may take kNormRows rows, loading all of them before reducing any; one row per
// warp measured faster on B200 than four (four halve the resident warps for a small
// gain in loads in flight).  x is read head-major [B, H, T, D] (the layout the rule
// writes o in) or token-major [B, T, H, D]; z and y are token-major, the layout the
// output projection reads.

constexpr int kNormWarps = 8;
constexpr int kNormRows = 1;

template <typename Tin, int D, bool SILU, bool X_HEAD_MAJOR>
__global__ void __launch_bounds__(kNormWarps * 32)
rms_norm_gated_kernel(const Tin* __restrict__ x, const Tin* __restrict__ z, const float* __restrict__ w,
                      Tin* __restrict__ y, int64_t rows, int T, int H, float eps) {
    constexpr int VE = 16 / (int)sizeof(Tin);                   // channels per 16-byte access
    constexpr int LPR = D / VE < 32 ? D / VE : 32;              // lanes per row
    constexpr int NV = D / (VE * LPR);                          // accesses per lane
    constexpr int RPW = 32 / LPR;                               // rows per warp
    static_assert(NV * VE * LPR == D && RPW * LPR == 32, "row split");
    using VT = Vec<Tin, VE>;
    using raw = typename VT::raw;
    const int lane = threadIdx.x & 31, l = lane % LPR;
    // the weight, shared by every row, into shared memory (16-byte aligned there; the
    // caller's array need only be 4-byte aligned)
    __shared__ __align__(16) float ws[D];
    for (int c = threadIdx.x; c < D; c += kNormWarps * 32) ws[c] = w[c];
    __syncthreads();
    const int64_t r0w = ((int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5)) * RPW;
    if (r0w >= rows) return;
    const int64_t r = r0w + lane / LPR;
    const bool valid = r < rows;
    int64_t xr = r;
    if (X_HEAD_MAJOR && valid) {
        const int64_t h = r % H, bt = r / H;
        const int64_t t = bt % T, b = bt / T;
        xr = (b * H + h) * T + t;
    }
    float xf[NV * VE], zf[NV * VE];
    float ss = 0.f;
    if (valid) {
#pragma unroll
        for (int a = 0; a < NV; ++a) {
            const int c = (a * LPR + l) * VE;
            VT::to_f(*reinterpret_cast<const raw*>(x + xr * D + c), xf + a * VE);
            VT::to_f(*reinterpret_cast<const raw*>(z + r * D + c), zf + a * VE);
        }
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < NV * VE; e += 2) {
            const float2 xv = make_float2(xf[e], xf[e + 1]);
            s2 = sm100::fma2(xv, xv, s2);
        }
        ss = s2.x + s2.y;
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (!valid) return;
    const float inv = rsqrtf(ss / (float)D + eps);
#pragma unroll
    for (int a = 0; a < NV; ++a) {
        const int c = (a * LPR + l) * VE;
        float out[VE];
        // channel pairs through packed fp32 (the kernel is bound by instruction issue)
#pragma unroll
        for (int e = 0; e < VE; e += 2) {
            const float2 zv = make_float2(zf[a * VE + e], zf[a * VE + e + 1]);
            const float2 gate = SILU ? sm100::silu2(zv) : sm100::sigmoid2(zv);
            const float2 xn = sm100::mul2(make_float2(xf[a * VE + e], xf[a * VE + e + 1]), make_float2(inv, inv));
            const float2 o2 = sm100::mul2(sm100::mul2(*reinterpret_cast<const float2*>(ws + c + e), xn), gate);
            out[e] = o2.x;
            out[e + 1] = o2.y;
        }
        *reinterpret_cast<raw*>(y + r * D + c) = VT::from_f(out);
    }
}

template <typename Tin, int D>
cudaError_t launch_norm_d(const NormArgs& a, cudaStream_t st) {
    const int64_t rows = a.B * a.T * a.H;
    const int64_t per_block = (int64_t)kNormWarps * (32 / (D * (int)sizeof(Tin) / 16 < 32 ? D * (int)sizeof(Tin) / 16 : 32));
    const dim3 grid((unsigned)((rows + per_block - 1) / per_block));
    const Tin* x = static_cast<const Tin*>(a.x);
    const Tin* z = static_cast<const Tin*>(a.z);
    Tin* y = static_cast<Tin*>(a.y);
    const int T = (int)a.T, H = (int)a.H;
    if (a.silu) {
        if (a.x_head_major)
            rms_norm_gated_kernel<Tin, D, true, true><<<grid, kNormWarps * 32, 0, st>>>(x, z, a.weight, y, rows, T, H, a.eps);
        else
            rms_norm_gated_kernel<Tin, D, true, false><<<grid, kNormWarps * 32, 0, st>>>(x, z, a.weight, y, rows, T, H, a.eps);
    } else {
        if (a.x_head_major)
            rms_norm_gated_kernel<Tin, D, false, true><<<grid, kNormWarps * 32, 0, st>>>(x, z, a.weight, y, rows, T, H, a.eps);
        else
            rms_norm_gated_kernel<Tin, D, false, false><<<grid, kNormWarps * 32, 0, st>>>(x, z, a.weight, y, rows, T, H, a.eps);
    }
    return counted(cudaGetLastError());
}

template <typename Tin>
cudaError_t launch_norm_t(const NormArgs& a, cudaStream_t st) {
    switch (a.D) {
        case 64: return launch_norm_d<Tin, 64>(a, st);
        case 128: return launch_norm_d<Tin, 128>(a, st);
        default: return launch_norm_d<Tin, 256>(a, st);
    }
}

}  // namespace

// The tiled kernel where the layout allows 16-byte accesses (a.vec16); else 8-byte
// accesses where it allows those (a.vec): 4 bf16 or 2 fp32 channels per thread
cudaError_t launch_causal_conv1d(const ConvArgs& a, cudaStream_t st) {
    if (a.vec16) return a.bf16 ? launch_conv_tile<__nv_bfloat16>(a, st) : launch_conv_tile<float>(a, st);
    if (a.bf16) return a.vec ? launch_conv_v<__nv_bfloat16, 4>(a, st) : launch_conv_v<__nv_bfloat16, 1>(a, st);
    return a.vec ? launch_conv_v<float, 2>(a, st) : launch_conv_v<float, 1>(a, st);
}

cudaError_t launch_rms_norm_gated(const NormArgs& a, cudaStream_t st) {
    return a.bf16 ? launch_norm_t<__nv_bfloat16>(a, st) : launch_norm_t<float>(a, st);
}

}  // namespace dn
