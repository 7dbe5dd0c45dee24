// Dense projections around the mixer on the 5th-generation tensor cores:
//   y[M][N] = x[M][K] . w[N][K]^T     (bf16 operands, fp32 accumulation, bf16 y)
//
// The mixer's hidden width and its head shapes come from "Qwen3.8-Flash-Next",
// the model-parameter and config tables (hidden_size 2,560; 16 key / 48 value
// heads of 128).  The pages give no projection layout; the reading used here is
// one bias-free linear map on each side: hidden -> q | k | v | z | a | b
// (2,048 + 2,048 + 6,144 + 6,144 + 48 + 48 channels) and o (6,144) -> hidden.
//
// One persistent CTA per SM walks the output tiles (BM x BN) in column-major
// tile order, so the CTAs in flight share the same few weight tiles.
//   warp 0      TMA producer: one A tile (BM x 64) and one B tile (BN x 64) per
//               stage, 128-byte swizzle, into a ring of shared-memory stages
//   warp 1      MMA issuer: 4 tcgen05.mma (M = 128, N = BN, K = 16) per stage
//               into one of two TMEM accumulators; a commit frees the stage
//   warps 2..5  epilogue: tcgen05.ld of the other accumulator (lane quadrant =
//               warp % 4), fp32 -> bf16, 16-byte stores into the output
//               segments; overlaps the next tile's main loop
// Every wait is bounded; a wait that runs out records an error, the roles drain
// what they issued and the kernel returns.
#pragma once

#include "device.cuh"

namespace gdn {
namespace gemm {

constexpr int BM = 128;         // rows per tile (tokens) = MMA M
constexpr int BK = 64;          // 64 bf16 = one 128-byte swizzle row along K
constexpr int NT = 192;         // 6 warps
constexpr int kMaxSeg = 8;      // output segments per call

// Columns [n0, n0 + width) of y go to dst, a row-major [M][width] matrix.
struct Seg {
    __nv_bfloat16* dst;
    int n0, width;
};

struct Args {
    int64_t M;
    int N, K;
    int m_blocks, n_blocks;
    int64_t tiles;
    int n_segs;
    Seg seg[kMaxSeg];
};

// Instruction descriptor for kind::f16 with bf16 A/B (both K-major) and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)                      // D format: f32
           | (1u << 7) | (1u << 10)       // A, B format: bf16
           | ((uint32_t)(N >> 3) << 17)
           | ((uint32_t)(M >> 4) << 24);
}

template <int BN>
struct Shape {
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "MMA N for M = 128");
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;   // a multiple of 1024 (swizzle atoms)
    static constexpr int STAGES = (200 * 1024) / STAGE;
    static constexpr int OFF_BAR = STAGES * STAGE;
    // full[S], empty[S], acc_full[2], acc_empty[2], drain, then the TMEM slot and abort word
    static constexpr int N_BARS = 2 * STAGES + 5;
    static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 8;
    static constexpr int SMEM = SMEM_USED + 1024;      // slack to align the base to 1024
    static constexpr uint32_t TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
    static_assert(STAGE % 1024 == 0, "stage alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(uint32_t lo, uint32_t hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<uint32_t*>(&v);
}

template <int BN>
__global__ void __launch_bounds__(NT, 1)
linear_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, Args p) {
    using S = Shape<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    const uint32_t bar0 = sb + S::OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (S::STAGES + s); };
    auto acc_full = [&](int a) { return bar0 + 8u * (2 * S::STAGES + a); };
    auto acc_empty = [&](int a) { return bar0 + 8u * (2 * S::STAGES + 2 + a); };
    const uint32_t drain = bar0 + 8u * (2 * S::STAGES + 4);
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + S::OFF_BAR + S::N_BARS * 8);
    volatile uint32_t* s_abort = s_tmem + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full(a), 1);
            mbar_init(acc_empty(a), 4);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(const_cast<uint32_t*>(s_tmem)), S::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int kb_n = (p.K + BK - 1) / BK;

    if (warp == 0) {
        // ---- TMA producer (one thread) ----
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_w);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
                const int mb = (int)(t % p.m_blocks), nb = (int)(t / p.m_blocks);
                for (int kb = 0; kb < kb_n; ++kb, ++it) {
                    const int s = (int)(it % S::STAGES);
                    if (!mbar_wait_bounded(empty(s), ((it / S::STAGES) & 1u) ^ 1u) || *s_abort) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = sb + (uint32_t)s * S::STAGE;
                    mbar_arrive_expect_tx(full(s), S::STAGE);
                    tma_load_2d(a_dst, &tm_x, kb * BK, mb * BM, full(s));
                    tma_load_2d(a_dst + S::A_BYTES, &tm_w, kb * BK, nb * BN, full(s));
                }
            }
            if (!ok) {
                record_error(kErrCopyTimeout);
                *s_abort = 1;
            }
            // the last copy armed on each stage lands before the CTA may exit
            for (uint32_t s = 0; s < (uint32_t)S::STAGES && s < it; ++s) {
                const uint32_t last = s + (it - 1 - s) / S::STAGES * S::STAGES;
                mbar_wait_bounded(full(s), (last / S::STAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer (converged warp, elected lane issues) ----
        constexpr uint32_t ID = idesc_bf16(BM, BN);
        uint32_t it = 0, ti = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++ti) {
            const uint32_t a = ti & 1u;
            if (!mbar_wait_bounded(acc_empty(a), ((ti >> 1) & 1u) ^ 1u) || *s_abort) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem + a * BN;
            for (int kb = 0; kb < kb_n; ++kb, ++it) {
                const int s = (int)(it % S::STAGES);
                if (!mbar_wait_bounded(full(s), (it / S::STAGES) & 1u) || *s_abort) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_src = sb + (uint32_t)s * S::STAGE;
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    mma_f16_w(d, sdesc(a_src + k * 32, 16, 1024), sdesc(a_src + S::A_BYTES + k * 32, 16, 1024), ID,
                              (kb | k) != 0);
                mma_commit_w(empty(s));
            }
            if (!ok) break;
            mma_commit_w(acc_full(a));
        }
        if (!ok) {
            record_error(kErrMmaTimeout);
            *s_abort = 1;
        }
        // every MMA issued here completes before TMEM and shared memory are released
        mma_commit_w(drain);
        mbar_wait_bounded(drain, 0);
    } else {
        // ---- epilogue: TMEM -> bf16 -> global ----
        const int q = warp & 3;             // TMEM lane quadrant this warp may read
        const int row = q * 32 + lane;
        uint32_t ti = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++ti) {
            const uint32_t a = ti & 1u;
            if (!mbar_wait_bounded(acc_full(a), (ti >> 1) & 1u) || *s_abort) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int mb = (int)(t % p.m_blocks), nb = (int)(t / p.m_blocks);
            const int64_t m = (int64_t)mb * BM + row;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + a * BN + c * 32, r);
                const int n = nb * BN + c * 32;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int n8 = n + g * 8;
                    if (n8 >= p.N) break;
                    int j = 0;
                    while (j + 1 < p.n_segs && n8 >= p.seg[j + 1].n0) ++j;
                    const Seg sg = p.seg[j];
                    if (m < p.M) {
                        const uint4 v = make_uint4(pack_bf16(r[8 * g], r[8 * g + 1]), pack_bf16(r[8 * g + 2], r[8 * g + 3]),
                                                   pack_bf16(r[8 * g + 4], r[8 * g + 5]),
                                                   pack_bf16(r[8 * g + 6], r[8 * g + 7]));
                        *reinterpret_cast<uint4*>(sg.dst + m * sg.width + (n8 - sg.n0)) = v;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive(acc_empty(a));
        }
        if (!ok && lane == 0) {
            record_error(kErrMmaTimeout);
            *s_abort = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace gdn
