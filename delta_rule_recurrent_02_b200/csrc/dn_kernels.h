// dn_kernels.h -- launchers behind the C ABI (private to the library).
// Arguments arrive already validated by dn_api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dn {

struct ChunkArgs {
    const void* q; const void* k; const void* v;
    const float* beta; const float* g; const float* S0;
    void* o; float* S_T;
    int64_t B, T, H;
    int dk, dv, chunk;
    float scale;
    bool bf16;
    int gate;                 // Gate
    unsigned int* status;     // device status word of the current device
    int test_flags;           // 1: withhold the tensor-core kernels' input loads (failure-path self-test)
    void* ws;                 // tensor-core path: workspace of tc_workspace_bytes(), 256-byte aligned
    float* snaps;             // null, or [B, H, n_snap, d_k, d_v]: the state after every snap_every chunks
    int snap_every, n_snap;
    // the layer's prologue inside the kernels (scalar gate): beta and g hold the raw b and
    // a; q and k are normalised per row.  0: off; else beta = prologue * sigmoid(b)
    // (1, or 2 for the gate in (0, 2))
    int prologue;
    const float* A_log;       // [H]
    const float* dt_bias;     // [H]
    int rep = 1;              // value heads per key head: q and k have H / rep heads
    // a packed batch (tensor-core path): N sequences of the B = 1 row of T tokens,
    // sequence s at tokens cu_seqlens[s] .. cu_seqlens[s + 1] - 1 (device int32 [N + 1]);
    // S0 and S_T are then [N, H, d_k, d_v].  Null: B independent rows.
    const int* cu_seqlens = nullptr;
    int N = 0;
    // with the prologue (tensor-core path): the layer's gated RMSNorm on the output rows
    // (0 none, 1 SiLU(z), 2 sigmoid(z)); o then receives y token-major [B, T, H, d_v], as z
    int norm = 0;
    const void* z = nullptr;
    const float* norm_weight = nullptr;
    float eps = 0.f;
};

struct DecodeArgs {
    const void* q; const void* k; const void* v;
    const float* beta; const float* g;
    float* S; void* o;
    int64_t B, H;
    int dk, dv;
    float scale;
    bool bf16;
    int gate;
    // the layer's prologue (scalar gate): beta and g hold the raw b and a; q and k are
    // normalised inside.  0: off; else beta = prologue * sigmoid(b)
    int prologue;
    const float* A_log;       // [H]
    const float* dt_bias;     // [H]
    int rep = 1;              // value heads per key head
    // with the prologue: the gated RMSNorm on the output row (0 none, 1 SiLU(z), 2 sigmoid(z))
    int norm = 0;
    const void* z = nullptr;  // [B, H, d_v] dtype
    const float* norm_weight = nullptr;   // [d_v]
    float eps = 0.f;
};

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t st);

// The generalised delta rule of RWKV-7 in chunks, fp32 on CUDA cores (chunk_general.cu).
struct GeneralArgs {
    const void* q; const float* wlog; const void* kappa; const float* a; const void* k; const void* v;
    const float* S0;
    void* o; float* S_T;
    int64_t B, T, H;
    int dk, dv, chunk;
    float scale;
    bool bf16;
};
cudaError_t launch_chunk_general(const GeneralArgs& a, cudaStream_t st);
int general_max_chunk();

// The layer's causal conv over time (layer_ops.cu).
struct ConvArgs {
    const void* x;            // [B, T, ld_x], channels 0..C-1 of each row
    int64_t ld_x;
    const float* weight;      // [C, K]
    const void* state_in;     // [B, K-1, C] or null (zeros)
    void* y;                  // [B, C / head_dim, T, head_dim]
    void* state_out;          // [B, K-1, C] or null
    int64_t B;
    int T, C, K, head_dim;
    bool activation;          // SiLU
    bool bf16;
    bool vec;                 // 8-byte accesses (alignment checked by the caller)
    bool vec16 = false;       // 16-byte accesses (likewise)
};
cudaError_t launch_causal_conv1d(const ConvArgs& a, cudaStream_t st);

// The layer's gated RMSNorm of each head's output row (layer_ops.cu).
struct NormArgs {
    const void* x;            // [B, H, T, D] (x_head_major) or [B, T, H, D]
    const void* z;            // [B, T, H, D]
    const float* weight;      // [D]
    void* y;                  // [B, T, H, D]
    int64_t B, T, H;
    int D;                    // 64, 128 or 256
    float eps;
    bool silu;                // else the logistic sigmoid
    bool x_head_major;
    bool bf16;
};
cudaError_t launch_rms_norm_gated(const NormArgs& a, cudaStream_t st);
cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t st);

// Tensor-core (tcgen05) chunk path: the per-chunk UT/WY transform (chunk_wy.cu)
// then the state pass (chunk_tc.cu).  tc_supports() says whether the request
// is inside its coverage (bf16, chunk 64, d_k = d_v = 128, any gate);
// tc_workspace_bytes() is the size of a.ws it needs (W^T and u^T of every chunk).
bool tc_supports(const ChunkArgs& a);
size_t tc_workspace_bytes(const ChunkArgs& a);
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t st);

// Record `msg` as the calling thread's dn_last_error() and return `code`.
int report_error(int code, const char* msg);

// Count one kernel launch of this library (read by dn_kernel_launches()).
void count_launch();
// `e` is the result of one kernel launch: count it if it succeeded.
inline cudaError_t counted(cudaError_t e) {
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace dn
