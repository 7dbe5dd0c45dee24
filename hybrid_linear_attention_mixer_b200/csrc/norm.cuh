// Output gated RMSNorm of the Gated DeltaNet layer, one (chunk, value head)
// tile of 64 tokens x d_v per CTA, fully parallel:
//     out = o * rsqrt(mean_dv(o^2) + eps) * w_norm * SiLU(z)
// (rms_norm_eps = 1e-6, "Raw config fields" of "Qwen3.8-Flash-Next",
// llm-atlas-9r2; SiLU(z) = z * sigmoid(z)).  o comes from the state-chain kernel
// as [chunk][head][64][128] tiles; z and out are the layer's [T][H_v][d_v]
// tensors.  One warp per token row, 4 channels per lane: HBM-bound.
#pragma once
#include "device.cuh"

namespace gdn {
namespace norm {

constexpr int C = 64;
constexpr int NT = 256;

struct Args {
    const void* o;              // [chunks][Hv][64][128] out dtype
    const void* z;              // [T][Hv][dv] act dtype
    const float* norm_w;        // [dv]
    const int32_t* cu;          // [N+1]
    const int32_t* chunk_off;   // [N+1]
    void* out;                  // [T][Hv][dv] out dtype
    int n_seqs, Hv, dv;
    float eps;
};

template <typename T> struct Vec4;
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
        const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float4 v) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&b);
        __stcs(reinterpret_cast<uint2*>(p), u);
    }
};
template <> struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
    static __device__ __forceinline__ void store(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
};

template <typename TA, typename TO>
__global__ void __launch_bounds__(NT) gdn_gated_norm_kernel(Args p) {
    const int Hv = p.Hv, dv = p.dv;
    const int h = blockIdx.x % Hv, gc = blockIdx.x / Hv;
    if (gc >= p.chunk_off[p.n_seqs]) return;
    int lo = 0, hi = p.n_seqs - 1;   // sequence of this chunk: last s with chunk_off[s] <= gc
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.chunk_off[mid] <= gc) lo = mid; else hi = mid - 1;
    }
    const int64_t t0 = (int64_t)p.cu[lo] + (int64_t)(gc - p.chunk_off[lo]) * C;
    const int64_t rem = (int64_t)p.cu[lo + 1] - t0;
    const int n = (int)(rem < C ? rem : C);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = 4 * lane;
    if (col >= dv) return;   // d_v in {32, 64, 128}: whole lanes drop out, no shuffle partners lost
    const unsigned mask = dv >= 128 ? 0xffffffffu : (dv == 64 ? 0x0000ffffu : 0x000000ffu);
    const float4 w4 = *reinterpret_cast<const float4*>(p.norm_w + col);
    const TO* ot = static_cast<const TO*>(p.o) + ((int64_t)gc * Hv + h) * C * 128;
    const int64_t ldv = (int64_t)Hv * dv;
    for (int r = warp; r < n; r += NT / 32) {
        const float4 o = Vec4<TO>::load(ot + r * 128 + col);
        const float4 z = Vec4<TA>::load(static_cast<const TA*>(p.z) + (t0 + r) * ldv + (int64_t)h * dv + col);
        float ss = o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
        for (int off = 16; off >= 1; off >>= 1)
            if (off < dv / 4) ss += __shfl_xor_sync(mask, ss, off);
        const float rs = rsqrtf(ss / (float)dv + p.eps);
        float4 y;
        y.x = o.x * rs * w4.x * silu_f(z.x);
        y.y = o.y * rs * w4.y * silu_f(z.y);
        y.z = o.z * rs * w4.z * silu_f(z.z);
        y.w = o.w * rs * w4.w * silu_f(z.w);
        Vec4<TO>::store(static_cast<TO*>(p.out) + (t0 + r) * ldv + (int64_t)h * dv + col, y);
    }
}

}  // namespace norm
}  // namespace gdn
