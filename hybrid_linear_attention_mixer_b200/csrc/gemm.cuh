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

// Eight consecutive output columns [n8, n8 + 8) of row m: into the segment that
// holds them (segments are multiples of 8 wide), skipped past M or N.
__device__ __forceinline__ void store8(const uint32_t* r, const Args& p, int64_t m, int n8) {
    if (n8 >= p.N || m >= p.M) return;
    int j = 0;
    while (j + 1 < p.n_segs && n8 >= p.seg[j + 1].n0) ++j;
    const Seg& sg = p.seg[j];
    const uint4 v = make_uint4(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]), pack_bf16(r[4], r[5]),
                               pack_bf16(r[6], r[7]));
    *reinterpret_cast<uint4*>(sg.dst + m * sg.width + (n8 - sg.n0)) = v;
}

// One accumulator row (this thread's TMEM lane) of BN columns -> bf16 row m of y,
// columns [n0, n0 + BN).  taddr: the row's first column (lane quadrant in bits 16+).
template <int BN>
__device__ __forceinline__ void store_row(uint32_t taddr, const Args& p, int64_t m, int n0) {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
#pragma unroll
        for (int g = 0; g < 4; ++g) store8(r + 8 * g, p, m, n0 + c * 32 + g * 8);
    }
    if constexpr (BN % 32 != 0) {
        uint32_t r[16];
        tmem_ld16(taddr + (BN / 32) * 32, r);
        store8(r, p, m, n0 + (BN / 32) * 32);
        store8(r + 8, p, m, n0 + (BN / 32) * 32 + 8);
    }
}

template <int BN>
__global__ void __launch_bounds__(NT, 1)
linear_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
              const __grid_constant__ Args p) {
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
            store_row<BN>(tmem + ((uint32_t)(q * 32) << 16) + a * BN, p, (int64_t)mb * BM + row, nb * BN);
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

// ---------------------------------------------------------------------------
// Pair form: a cluster of 2 CTAs on neighbouring SMs computes a 256 x BN tile
// with tcgen05.mma.cta_group::2 (M = 256).  CTA r of the pair loads rows
// [128r, 128r + 128) of the A tile and rows [r BN/2, (r+1) BN/2) of the B tile
// into its own shared memory; the MMA issued by CTA 0 reads both halves and
// leaves rows [128r, 128r + 128) x BN of the product in CTA r's tensor memory.
// Each SM thus loads 16 KiB + BN/2 x 128 B per k-block instead of
// 16 KiB + BN x 128 B.  Barriers:
//   full[s]      in CTA 0: CTA 0 arms it for both CTAs' bytes; both CTAs' TMA
//                loads complete on it (the .cta_group::2 form of the load)
//   empty[s]     in each CTA: one commit from CTA 0's MMA thread per CTA
//   acc_full[a]  in each CTA: one commit per CTA when a tile's MMAs are done
//   acc_empty[a] in CTA 0: 4 epilogue warps x 2 CTAs arrive (cluster scope)
// No load is multicast; every cross-CTA signal names one barrier.
// ---------------------------------------------------------------------------
template <int BN>
struct Shape2 {
    static_assert(BN % 16 == 0 && BN >= 64 && BN <= 256, "MMA N for M = 256");
    static constexpr int A_BYTES = BM * BK * 2;              // this CTA's 128 rows of A
    static constexpr int B_BYTES = (BN / 2) * BK * 2;        // this CTA's half of B
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = (200 * 1024) / STAGE < 8 ? (200 * 1024) / STAGE : 8;
    static constexpr int OFF_BAR = STAGES * STAGE;
    static constexpr int N_BARS = 2 * STAGES + 5;
    static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 8;
    static constexpr int SMEM = SMEM_USED + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
    static_assert(STAGE % 1024 == 0, "stage alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address, in the cluster window, of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool wait_cluster_bounded(uint32_t bar, uint32_t parity) {
    if (try_wait_cluster(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!try_wait_cluster(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}
// Tiled 2-D TMA load into this CTA's shared memory whose completion is counted
// on an mbarrier that may live in the peer CTA (bar: cluster-window address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                                 uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
#define GDN_ELECT2 "{\n\t.reg .pred e;\n\t.reg .b32 ex;\n\telect.sync ex|e, 0xffffffff;\n\t"
__device__ __forceinline__ void mma_pair_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(GDN_ELECT2 ".reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
// One arrive on the barrier at `bar` (cluster-window address: this CTA's or the
// peer's) once every pair MMA this thread issued so far has completed.
__device__ __forceinline__ void commit_pair_w(uint32_t bar) {
    asm volatile(GDN_ELECT2 "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
                 ::"r"(bar)
                 : "memory");
}
#undef GDN_ELECT2

template <int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NT, 1)
linear_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ Args p) {
    using S = Shape2<BN>;
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
    const uint32_t rank = cluster_rank();
    const int64_t pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full(a), 1);
            mbar_init(acc_empty(a), 8);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(const_cast<uint32_t*>(s_tmem))),
                     "r"(S::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();    // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int kb_n = (p.K + BK - 1) / BK;
    const int64_t m_pairs = (p.M + 2 * BM - 1) / (2 * BM);
    const int64_t tiles = m_pairs * p.n_blocks;

    if (warp == 0) {
        // ---- TMA producer of this CTA's halves ----
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_w);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = pair; t < tiles && ok; t += n_pairs) {
                const int mb = (int)(t % m_pairs), nb = (int)(t / m_pairs);
                const int row_a = mb * 2 * BM + (int)rank * BM;
                const int row_b = nb * BN + (int)rank * (BN / 2);
                for (int kb = 0; kb < kb_n; ++kb, ++it) {
                    const int s = (int)(it % S::STAGES);
                    if (!mbar_wait_bounded(empty(s), ((it / S::STAGES) & 1u) ^ 1u) || *s_abort) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = sb + (uint32_t)s * S::STAGE;
                    const uint32_t fb = map_to_rank(full(s), 0);
                    if (rank == 0) mbar_arrive_expect_tx(full(s), 2 * S::STAGE);
                    tma_load_2d_pair(dst, &tm_x, kb * BK, row_a, fb);
                    tma_load_2d_pair(dst + S::A_BYTES, &tm_w, kb * BK, row_b, fb);
                }
            }
            if (!ok) {
                record_error(kErrCopyTimeout);
                *s_abort = 1;
            }
            if (rank == 0) {
                // the last phase armed on each stage (both CTAs' bytes) lands before exit
                for (uint32_t s = 0; s < (uint32_t)S::STAGES && s < it; ++s) {
                    const uint32_t last = s + (it - 1 - s) / S::STAGES * S::STAGES;
                    mbar_wait_bounded(full(s), (last / S::STAGES) & 1u);
                }
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer: CTA 0 only ----
        if (rank == 0) {
            constexpr uint32_t ID = idesc_bf16(2 * BM, BN);
            const uint32_t peer = 1;
            uint32_t it = 0, ti = 0;
            bool ok = true;
            for (int64_t t = pair; t < tiles && ok; t += n_pairs, ++ti) {
                const uint32_t a = ti & 1u;
                if (!wait_cluster_bounded(acc_empty(a), ((ti >> 1) & 1u) ^ 1u) || *s_abort) {
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
                        mma_pair_w(d, sdesc(a_src + k * 32, 16, 1024), sdesc(a_src + S::A_BYTES + k * 32, 16, 1024),
                                   ID, (kb | k) != 0);
                    commit_pair_w(empty(s));
                    commit_pair_w(map_to_rank(empty(s), peer));
                }
                if (!ok) break;
                commit_pair_w(acc_full(a));
                commit_pair_w(map_to_rank(acc_full(a), peer));
            }
            if (!ok) {
                record_error(kErrMmaTimeout);
                *s_abort = 1;
            }
            commit_pair_w(drain);
            mbar_wait_bounded(drain, 0);
        }
    } else {
        // ---- epilogue: this CTA's 128 rows of the pair tile ----
        const int q = warp & 3;
        const int row = q * 32 + lane;
        uint32_t ti = 0;
        bool ok = true;
        for (int64_t t = pair; t < tiles; t += n_pairs, ++ti) {
            const uint32_t a = ti & 1u;
            if (!mbar_wait_bounded(acc_full(a), (ti >> 1) & 1u) || *s_abort) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int mb = (int)(t % m_pairs), nb = (int)(t / m_pairs);
            store_row<BN>(tmem + ((uint32_t)(q * 32) << 16) + a * BN, p,
                          (int64_t)mb * 2 * BM + (int64_t)rank * BM + row, nb * BN);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_cluster(map_to_rank(acc_empty(a), 0));
        }
        if (!ok && lane == 0) {
            record_error(kErrMmaTimeout);
            *s_abort = 1;
        }
    }

    tc_fence_before();
    cluster_sync();    // no CTA leaves while its peer may still signal or read it
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS)
                     : "memory");
    }
}

}  // namespace gemm
}  // namespace gdn
