// Output gated RMSNorm of the Gated DeltaNet layer, one (chunk, value head)
// tile of 64 tokens x d_v per CTA, fully parallel:
//     out = o * rsqrt(mean_dv(o^2) + eps) * w_norm * SiLU(z)
// (rms_norm_eps = 1e-6, "Raw config fields" of "Qwen3.8-Flash-Next",
// llm-atlas-9r2; SiLU(z) = z * sigmoid(z)).  o comes from the state-chain kernel
// as [chunk][head][64][128] tiles; z and out are the layer's [T][H_v][d_v]
// tensors.  HBM-bound: persistent CTAs walk the tiles; the next tile's o (one
// bulk copy) and z rows (one TMA box) land in shared memory while the current
// one is finished, 4 threads per row, and stored with 16-byte stores.
#pragma once
#include "device.cuh"

namespace gdn {
namespace norm {

constexpr int C = kChunk;
constexpr int NT = 256;             // 4 threads per row, d_v / 4 channels each

struct Args {
    const void* o;              // [chunks][Hv][64][128] out dtype
    const float* norm_w;        // [dv]
    const int32_t* cu;          // [N+1]
    const int32_t* chunk_off;   // [N+1]
    const int32_t* flags;       // nonzero: a device check of the call failed, write nothing
    void* out;                  // [T][Hv][dv] out dtype
    int n_seqs, Hv, dv;
    float eps;
    int32_t g_lo, g_hi;         // the tiles of global chunks [g_lo, g_hi)
};

template <typename TA, typename TO> __host__ __device__ constexpr uint32_t stage_bytes() {
    return C * 128 * sizeof(TO) + C * 128 * sizeof(TA);
}
constexpr int STAGES = 3;   // tiles in flight per CTA: the current one and the next two
template <typename TA, typename TO> __host__ __device__ constexpr uint32_t smem_bytes() {
    return STAGES * stage_bytes<TA, TO>() + 64 + 128;
}

template <typename T> __device__ __forceinline__ void load8(const uint8_t* p, float (&f)[8]);
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const uint8_t* p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <> __device__ __forceinline__ void load8<float>(const uint8_t* p, float (&f)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 16);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
template <typename T> __device__ __forceinline__ void store8(T* p, const float (&f)[8]);
template <> __device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&f)[8]) {
    uint4 u;
    uint32_t* w = &u.x;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    __stcs(reinterpret_cast<uint4*>(p), u);
}
template <> __device__ __forceinline__ void store8<float>(float* p, const float (&f)[8]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(f[0], f[1], f[2], f[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(f[4], f[5], f[6], f[7]));
}

// tm_z: 2-D map over z as [T][Hv * dv], boxes of d_v x 64 tokens (rows past T read as zero)
template <typename TA, typename TO>
__global__ void __launch_bounds__(NT) gdn_gated_norm_kernel(const __grid_constant__ CUtensorMap tm_z, Args p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 127u) & ~127u;
    uint8_t* smem = smem_raw + (sb - raw);
    constexpr uint32_t O_BYTES = C * 128 * sizeof(TO), STAGE = stage_bytes<TA, TO>();
    const uint32_t bar0 = sb + STAGES * STAGE;                                   // [STAGES]
    int* s_n = reinterpret_cast<int*>(smem + STAGES * STAGE + 24);               // [STAGES] rows of the tile
    long long* s_t0 = reinterpret_cast<long long*>(smem + STAGES * STAGE + 40);  // [STAGES] first token
    const int Hv = p.Hv, dv = p.dv;
    const int64_t g_end = p.chunk_off[p.n_seqs] < p.g_hi ? p.chunk_off[p.n_seqs] : p.g_hi;
    const int64_t tile0 = (int64_t)p.g_lo * Hv;
    const int64_t n_tiles = g_end > p.g_lo ? (g_end - p.g_lo) * Hv : 0;
    const uint32_t z_bytes = (uint32_t)(C * dv * sizeof(TA));
    // this CTA's tile i is (chunk, head) index tile0 + blockIdx.x + i * gridDim.x; thread 0 issues its loads
    auto issue = [&](int i) {
        const int64_t tile = tile0 + blockIdx.x + (int64_t)i * gridDim.x;
        const int st = i % STAGES;
        const int h = (int)(tile % Hv), gc = (int)(tile / Hv);
        int lo = 0, hi = p.n_seqs - 1;   // sequence of this chunk: last s with chunk_off[s] <= gc
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.chunk_off[mid] <= gc) lo = mid; else hi = mid - 1;
        }
        const int64_t t0 = (int64_t)p.cu[lo] + (int64_t)(gc - p.chunk_off[lo]) * C;
        const int64_t rem = (int64_t)p.cu[lo + 1] - t0;
        s_t0[st] = t0;
        s_n[st] = (int)(rem < C ? rem : C);
        const uint32_t bar = bar0 + 8 * st, dst = sb + st * STAGE;
        mbar_arrive_expect_tx(bar, O_BYTES + z_bytes);
        bulk_g2s(dst, static_cast<const uint8_t*>(p.o) + tile * O_BYTES, O_BYTES, bar);
        tma_load_2d(dst + O_BYTES, &tm_z, h * dv, (int)t0, bar);
    };
    const int count = n_tiles > blockIdx.x ? (int)((n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
    if (count <= 0 || *p.flags) return;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; i++) mbar_init(bar0 + 8 * i, 1);
        fence_mbar_init();
        for (int i = 0; i < STAGES - 1 && i < count; i++) issue(i);
    }
    __syncthreads();
    // thread (r, q): row r; at step k the row's 4 threads take channels 32k + 8q .. + 7, so every
    // store instruction writes whole 32-byte sectors
    const int r = threadIdx.x >> 2, q = threadIdx.x & 3;
    const int steps = dv >> 5;                               // 1, 2 or 4
    int i = 0;
    bool ok = true;
    for (; i < count; i++) {
        const int st = i % STAGES;
        const bool got = mbar_wait_bounded(bar0 + 8 * st, (i / STAGES) & 1);
        // every thread is done with tile i - 1, and all take the same way out
        if (__syncthreads_or(!got)) {
            ok = false;
            break;
        }
        if (threadIdx.x == 0 && i + STAGES - 1 < count) {   // into the stage of tile i - 1
            fence_async_smem();
            issue(i + STAGES - 1);
        }
        const int64_t tile = tile0 + blockIdx.x + (int64_t)i * gridDim.x;
        const int h = (int)(tile % Hv);
        const int64_t t0 = s_t0[st];
        const int n = s_n[st];
        const uint8_t* orow = smem + st * STAGE + r * 128 * sizeof(TO) + q * 8 * sizeof(TO);
        const uint8_t* zrow = smem + st * STAGE + O_BYTES + (r * dv + q * 8) * sizeof(TA);
        float ss = 0.f;
        for (int k = 0; k < steps; k++) {
            float o8[8];
            load8<TO>(orow + 32 * k * sizeof(TO), o8);
#pragma unroll
            for (int e = 0; e < 8; e++) ss = fmaf(o8[e], o8[e], ss);
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        const float rs = rsqrtf(ss / (float)dv + p.eps);
        if (r < n) {
            TO* yt = static_cast<TO*>(p.out) + (t0 + r) * ((int64_t)Hv * dv) + (int64_t)h * dv + q * 8;
            const float4* w4 = reinterpret_cast<const float4*>(p.norm_w + q * 8);
            for (int k = 0; k < steps; k++) {
                float o8[8], z8[8], y[8];
                load8<TO>(orow + 32 * k * sizeof(TO), o8);
                load8<TA>(zrow + 32 * k * sizeof(TA), z8);
                const float4 wa = __ldg(w4 + 8 * k), wb = __ldg(w4 + 8 * k + 1);
                const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                for (int e = 0; e < 8; e++) y[e] = o8[e] * rs * wv[e] * silu_f(z8[e]);
                store8<TO>(yt + 32 * k, y);
            }
        }
    }
    if (!ok && threadIdx.x == 0) {
        // a copy never arrived: report it (the tiles from here on are not written) and give
        // the copies still in flight one more bounded wait
        record_error(kErrCopyTimeout);
        const int issued = count < i + STAGES - 1 ? count : i + STAGES - 1;
        for (int j = i; j < issued; j++) mbar_wait_bounded(bar0 + 8 * (j % STAGES), (j / STAGES) & 1);
    }
}

}  // namespace norm
}  // namespace gdn
