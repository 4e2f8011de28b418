// dn_common.cuh -- small device helpers shared by the delta-rule kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dn {

enum Gate { kGateNone = 0, kGateScalar = 1, kGatePerKey = 2 };

// Load / store one element of the token dtype as fp32.
__device__ __forceinline__ float ld_elem(const float* p) { return *p; }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_elem(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_elem(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Load four consecutive elements (p 8-byte aligned for bf16, 16-byte for fp32).
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void st4(float* p, float4 x) { *reinterpret_cast<float4*>(p) = x; }
__device__ __forceinline__ void st4(__nv_bfloat16* p, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

// Streaming 128-bit global access issued exactly once where written (volatile
// asm is neither duplicated nor re-materialised by the compiler).
__device__ __forceinline__ float4 ld_stream_f4(const float* p) {
    float4 r;
    asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ void st_stream_f4(float* p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// The Gated DeltaNet layer's gates from its raw per-token inputs ("Linear
// attention and Gated DeltaNet", ch. 28, "The full layer", step 5): beta =
// bmul sigmoid(b), g = -exp(A_log) softplus(a + dt_bias), softplus(x) =
// log(1 + e^x) (x above 20 taken as x).  eA = exp(A_log) of the head; bmul is 1,
// or 2 for the gate 2 sigmoid(b) in (0, 2) that admits the negative eigenvalues
// of D2L 12.5, "The reflection hiding in the delta rule".
__device__ __forceinline__ void gdn_raw_gates(float& b, float& a, float eA, float dt_bias, float bmul) {
    b = bmul / (1.f + expf(-b));
    const float x = a + dt_bias;
    a = -eA * (x > 20.f ? x : log1pf(expf(x)));
}

}  // namespace dn
