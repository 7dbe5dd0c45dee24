// Short causal depthwise convolution (kernel 4) + SiLU over the q|k|v channels,
// with the per-key-head L2 norm of q and k fused into the same pass.
//
// Layer: "Qwen3.8-Flash-Next" (llm-architectures-explained), "Every architecture
// field": linear_conv_kernel_dim = 4 over q|k|v; SiLU is the model's hidden_act
// ("Raw config fields", llm-atlas-9r2).  Tap K-1 multiplies the current token;
// the K-1 inputs before a sequence start come from conv_state (oldest first).
//
// Output: q^, k^ (unit norm per key head) and v^ as fp16 in the workspace.  The
// chunked prefill kernel feeds them straight to the tensor cores.  HBM-bound:
// each CTA streams 16 tokens x 1024 channels with 16-byte loads and stores.
#pragma once
#include "device.cuh"

namespace gdn {

struct ConvArgs {
    const void* q;           // [T][Cq]   act dtype
    const void* k;           // [T][Cq]
    const void* v;           // [T][Cv]
    const float* conv_w;     // [Ctot][4]
    const void* conv_state;  // [N][Ctot][3] act dtype (read only here)
    const int32_t* cu;       // [N+1]
    int n_seqs;
    int64_t T;
    int Hk, Hv, dk, dv;
    float l2_eps;
    __half* qh;              // [T][Cq]
    __half* kh;              // [T][Cq]
    __half* vh;              // [T][Cv]
};

constexpr int kConvThreads = 128;   // 8 channels per thread
// tokens per CTA: every thread keeps TT + 3 rows of 8 inputs in registers
template <typename TA> __host__ __device__ constexpr int conv_tokens() { return sizeof(TA) == 2 ? 8 : 4; }

template <typename TA>
__device__ __forceinline__ const TA* __restrict__ conv_channel_ptr(const ConvArgs& p, int64_t t, int c, int Cq, int Cv) {
    if (c < Cq) return static_cast<const TA*>(p.q) + t * Cq + c;
    if (c < 2 * Cq) return static_cast<const TA*>(p.k) + t * Cq + (c - Cq);
    return static_cast<const TA*>(p.v) + t * Cv + (c - 2 * Cq);
}

// 8 consecutive activations of one token, kept packed until used.
template <typename TA> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* __restrict__ p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void get(float (&f)[8]) const {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* __restrict__ p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void get(float (&f)[8]) const {
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

template <typename TA>
__global__ void __launch_bounds__(kConvThreads) conv_silu_norm_kernel(ConvArgs p) {
    constexpr int TT = conv_tokens<TA>();
    const int Cq = p.Hk * p.dk, Cv = p.Hv * p.dv, Ctot = 2 * Cq + Cv;
    const int c = (blockIdx.y * kConvThreads + threadIdx.x) * 8;   // first of 8 channels
    const int64_t t_begin = (int64_t)blockIdx.x * TT;
    __shared__ int s_seq[TT];
    __shared__ long long s_start[TT];
    if (threadIdx.x < TT) {
        const int64_t t = t_begin + threadIdx.x;
        int lo = 0, hi = p.n_seqs - 1;              // last s with cu[s] <= t
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if ((int64_t)p.cu[mid] <= t) lo = mid; else hi = mid - 1;
        }
        s_seq[threadIdx.x] = lo;
        s_start[threadIdx.x] = p.cu[lo];
    }
    const bool active = c < Ctot;
    const bool is_qk = c < 2 * Cq;
    // All TT + 3 input rows of this thread's 8 channels are requested before any
    // is used, so their latencies overlap.
    Raw8<TA> raw[TT + 3];
#pragma unroll
    for (int s = 0; s < TT + 3; s++) {
        const int64_t t = t_begin - 3 + s;
        raw[s].zero();
        if (active && t >= 0 && t < p.T) raw[s].load(conv_channel_ptr<TA>(p, t, c, Cq, Cv));
    }
    float w[8][4];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (active) t4 = __ldg(reinterpret_cast<const float4*>(p.conv_w) + c + i);
        w[i][0] = t4.x; w[i][1] = t4.y; w[i][2] = t4.z; w[i][3] = t4.w;
    }
    __syncthreads();

    const int group = p.dk >> 3;                    // threads per key head (4, 8 or 16)
#pragma unroll
    for (int it = 0; it < TT; it++) {
        const int64_t t = t_begin + it;
        const bool valid = active && t < p.T;
        float x[8], tap[3][8];
        raw[it + 3].get(x);
        const int64_t s0 = s_start[it];
#pragma unroll
        for (int s = 0; s < 3; s++) {
            const int64_t u = t - 3 + s;
            if (valid && u < s0) {     // taps before the sequence start come from its conv_state
                const int slot = 3 - (int)(s0 - u);
                const TA* st = static_cast<const TA*>(p.conv_state) + ((int64_t)s_seq[it] * Ctot + c) * 3 + slot;
#pragma unroll
                for (int i = 0; i < 8; i++) tap[s][i] = to_f32(st[i * 3]);
            } else {
                raw[it + s].get(tap[s]);
            }
        }
        float y[8];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            float acc = w[i][0] * tap[0][i];
            acc = fmaf(w[i][1], tap[1][i], acc);
            acc = fmaf(w[i][2], tap[2][i], acc);
            acc = fmaf(w[i][3], x[i], acc);
            y[i] = silu_f(acc);
            ss = fmaf(y[i], y[i], ss);
        }
        // sum of squares over the key head's `group` threads (aligned lane groups)
        for (int off = 1; off < group; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (is_qk) {
            const float r = rsqrtf(ss + p.l2_eps);
#pragma unroll
            for (int i = 0; i < 8; i++) y[i] *= r;
        }
        if (valid) {
            uint4 o;
            o.x = pack_half2(y[0], y[1]);
            o.y = pack_half2(y[2], y[3]);
            o.z = pack_half2(y[4], y[5]);
            o.w = pack_half2(y[6], y[7]);
            __half* dst = c < Cq ? p.qh + t * Cq + c
                        : c < 2 * Cq ? p.kh + t * Cq + (c - Cq)
                                     : p.vh + t * Cv + (c - 2 * Cq);
            __stcs(reinterpret_cast<uint4*>(dst), o);
        }
    }
}

// conv_state <- the last 3 raw inputs of each sequence (oldest first), keeping
// old entries when the sequence is shorter than 3.  Runs after the conv kernel,
// which still reads the old state.
template <typename TA>
__global__ void __launch_bounds__(256) conv_state_update_kernel(ConvArgs p, void* conv_state) {
    const int Cq = p.Hk * p.dk, Cv = p.Hv * p.dv, Ctot = 2 * Cq + Cv;
    const int c = blockIdx.y * 256 + threadIdx.x;
    const int s = blockIdx.x;
    if (c >= Ctot) return;
    const int64_t t0 = p.cu[s], t1 = p.cu[s + 1];
    TA* st = static_cast<TA*>(conv_state) + ((int64_t)s * Ctot + c) * 3;
    TA old[3] = {st[0], st[1], st[2]};
    TA nw[3];
#pragma unroll
    for (int q = 0; q < 3; q++) {
        const int64_t t = t1 - 3 + q;
        nw[q] = (t >= t0) ? *conv_channel_ptr<TA>(p, t, c, Cq, Cv) : old[3 - (int)(t0 - t)];
    }
#pragma unroll
    for (int q = 0; q < 3; q++) st[q] = nw[q];
}

}  // namespace gdn
