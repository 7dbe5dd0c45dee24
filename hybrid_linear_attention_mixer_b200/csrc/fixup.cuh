// Second half of a prefill whose state chain was split in two (one sequence).
//
// Over a range of chunks the recurrence maps its start state affinely: with S_t
// the state after token t of the range, S_t = S0 M_t + S_t^loc, where M_t is the
// product of the range's transitions (d_k x d_k) and S^loc the states from a zero
// start.  So o_t = S_t q_t / sqrt(d_k) = o_t^loc + S0 o_t^P, with o^loc the
// outputs of the range scanned from zero and o^P = M_t q_t / sqrt(d_k) the outputs
// of the range scanned from S0 = I with V = 0 (the scan kernel run on the
// identity: its "state" is M).  Both come as o tiles ([chunk][head][64][128]);
// S0 is the end state of the first half, known only once that half is done.
//
// This kernel takes one head and two chunks of the second half per CTA: the
// correction o^P S0^T (M = 128 tokens, N = d_v, K = d_k, bf16 operands, fp32
// accumulation in TMEM, on the tensor cores) plus o^loc, then the gated RMSNorm
// of each token row straight from TMEM (thread r owns row r):
//     out = o * rsqrt(mean_dv(o^2) + eps) * w_norm * SiLU(z)
// The end state of the second half, S0 P + S_loc with P = M at the range's end,
// is folded by cp.cuh's fold kernel.
#pragma once
#include "device.cuh"
#include "gemm.cuh"

namespace gdn {
namespace fix {

constexpr int NT = 128;                           // 4 warps: one TMEM lane quadrant each
constexpr uint32_t OFF_A = 0;                     // o^P rows: [K half][128 rows][128 B], 32 KiB
constexpr uint32_t OFF_B = 32768;                 // S0 (bf16): [K half][128 rows][128 B], 32 KiB
constexpr uint32_t OFF_BAR = 65536;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
constexpr uint32_t TMEM_COLS = 128;

struct Args {
    const __nv_bfloat16* o_loc;   // [chunks][Hv][64][128] o tiles of the second half (first half's too)
    const __nv_bfloat16* z;       // [T][Hv][dv]
    const float* norm_w;          // [dv]
    __nv_bfloat16* out;           // [T][Hv][dv]
    const int32_t* flags;         // nonzero: a device check of the call failed, write nothing
    int64_t T;
    int Hv;
    int c_lo, c_hi;               // chunks of the second half: [c_lo, c_hi)
    float eps;
};

// tm_p: o^P tiles as [rows = chunks * Hv * 64][128] bf16, boxes of 64 x 64, 128-byte swizzle.
// tm_s: S0 (bf16) as [Hv * 128][128], boxes of 64 x 128, 128-byte swizzle.
__global__ void __launch_bounds__(NT) gdn_fixup_norm_kernel(const __grid_constant__ CUtensorMap tm_p,
                                                            const __grid_constant__ CUtensorMap tm_s, Args p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.x % p.Hv;
    const int c = p.c_lo + 2 * (blockIdx.x / p.Hv);   // chunks c and c + 1 (if < c_hi) of head h
    if (c >= p.c_hi || *p.flags) return;
    const bool two = c + 1 < p.c_hi;
    const uint32_t bar_ld = sb + OFF_BAR, bar_mma = sb + OFF_BAR + 8;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 16);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 20);

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *s_abort = 0;
        mbar_arrive_expect_tx(bar_ld, (two ? 4u : 2u) * 8192u + 2u * 16384u);
#pragma unroll
        for (int kh = 0; kh < 2; kh++) {
            tma_load_2d(sb + OFF_A + kh * 16384, &tm_p, 64 * kh, (int)(((int64_t)c * p.Hv + h) * 64), bar_ld);
            if (two)
                tma_load_2d(sb + OFF_A + kh * 16384 + 8192, &tm_p, 64 * kh, (int)(((int64_t)(c + 1) * p.Hv + h) * 64),
                            bar_ld);
            tma_load_2d(sb + OFF_B + kh * 16384, &tm_s, 64 * kh, h * 128, bar_ld);
        }
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_BAR + 16, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    if (tid == 0) {
        if (!mbar_wait_bounded(bar_ld, 0)) atomicOr((unsigned*)s_abort, 2u);
        if (*s_abort == 0) {
            tc_fence_after();
            constexpr uint32_t ID = gemm::idesc_bf16(128, 128);
#pragma unroll
            for (int ks = 0; ks < 8; ks++)
                mma_f16(tmem, sdesc(sb + OFF_A + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                        sdesc(sb + OFF_B + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), ID, ks > 0);
            mma_commit(bar_mma);
        }
    }
    if (*s_abort == 0 && !mbar_wait_bounded(bar_mma, 0)) atomicOr((unsigned*)s_abort, 1u);
    __syncthreads();
    const bool ok = *s_abort == 0;
    if (ok) {
        tc_fence_after();
        // row r = tid: token rr of chunk c + r / 64 (rows of a chunk past the sequence end are skipped)
        const int rr = tid & 63, gc = c + (tid >> 6);
        const int64_t t = (int64_t)gc * 64 + rr;
        const bool row_ok = (tid < 64 || two) && t < p.T;
        const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
        const uint4* orow = reinterpret_cast<const uint4*>(p.o_loc + (((int64_t)gc * p.Hv + h) * 64 + rr) * 128);
        auto bf = [](uint32_t w, int hi) { return __uint_as_float(hi ? (w & 0xffff0000u) : (w << 16)); };
        float ss = 0.f;
#pragma unroll 1
        for (int q = 0; q < 4; q++) {   // 32 columns at a time
            uint32_t d[32];
            tmem_ld32(tl + 32 * q, d);
            if (row_ok) {
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const uint4 o8 = orow[4 * q + u];
                    const uint32_t ow[4] = {o8.x, o8.y, o8.z, o8.w};
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        const float x = __uint_as_float(d[8 * u + e]) + bf(ow[e >> 1], e & 1);
                        ss = fmaf(x, x, ss);
                    }
                }
            }
        }
        const float rs = rsqrtf(ss / 128.f + p.eps);
        const uint4* zrow = reinterpret_cast<const uint4*>(p.z + (t * p.Hv + h) * 128);
        uint4* yrow = reinterpret_cast<uint4*>(p.out + (t * p.Hv + h) * 128);
#pragma unroll 1
        for (int q = 0; q < 4; q++) {
            uint32_t d[32];
            tmem_ld32(tl + 32 * q, d);
            if (row_ok) {
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const uint4 o8 = orow[4 * q + u], z8 = zrow[4 * q + u];
                    const uint32_t ow[4] = {o8.x, o8.y, o8.z, o8.w}, zw[4] = {z8.x, z8.y, z8.z, z8.w};
                    const float4 wa = __ldg(reinterpret_cast<const float4*>(p.norm_w) + 8 * q + 2 * u);
                    const float4 wb = __ldg(reinterpret_cast<const float4*>(p.norm_w) + 8 * q + 2 * u + 1);
                    const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                    uint32_t y[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; e2++) {
                        float v2[2];
#pragma unroll
                        for (int s = 0; s < 2; s++) {
                            const int e = 2 * e2 + s;
                            const float x = __uint_as_float(d[8 * u + e]) + bf(ow[e2], s);
                            v2[s] = x * rs * wv[e] * silu_f(bf(zw[e2], s));
                        }
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v2[0], v2[1]);
                        y[e2] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
                    yrow[4 * q + u] = make_uint4(y[0], y[1], y[2], y[3]);
                }
            }
        }
    } else if (tid == 0) {
        // a copy or the tensor-core commit never arrived: report it, and give whatever may
        // still be in flight one more bounded wait
        record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
        mbar_wait_bounded(bar_ld, 0);
        mbar_wait_bounded(bar_mma, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// S0 (fp32 [Hv][dv][dk]) -> bf16, the B operand of the correction.
__global__ void __launch_bounds__(256) state_to_bf16_kernel(const float* s, __nv_bfloat16* d, int64_t n,
                                                           const int32_t* flags) {
    if (*flags) return;
    for (int64_t i = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 4 * (int64_t)gridDim.x * blockDim.x) {
        const float4 v = *reinterpret_cast<const float4*>(s + i);
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        *reinterpret_cast<uint2*>(d + i) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
    }
}

// The start states of the second half's two scans: zero (for S_loc) and the
// identity per head (for the transitions M); x holds [P | S_loc] as [2][Hv][d][d].
__global__ void __launch_bounds__(256) split_init_kernel(float* x, int Hv, int d, const int32_t* flags) {
    if (*flags) return;
    const int64_t per = (int64_t)Hv * d * d;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * per; i += (int64_t)gridDim.x * blockDim.x)
        x[i] = (i < per && (i / d) % d == i % d) ? 1.f : 0.f;
}

}  // namespace fix
}  // namespace gdn
