// State chain of the chunked gated delta rule on the sm_100a tensor cores.
//
// One CTA (17 warps) walks one (sequence, value head) chain chunk by chunk
// (C = 64 tokens).  The state-independent factors of every chunk come from the
// intra-chunk kernel's records (intra.cuh: -W, T, P, g, Q~).  With S0 the state
// at the chunk start:
//     U   = T V - W S0^T                                    (exact per-token updates)
//     O   = (diag(e^g) Q S0^T + P U) / sqrt(d_k)
//     S_C = e^{g_C} S0 + U^T diag(e^{g_C - g}) K
// o goes out as [chunk][head][64][128] tiles; the gated RMSNorm that follows
// runs in norm.cuh, in parallel over all tiles.
//
// A tcgen05.mma costs about the same whatever its N up to 128, so products that
// share an A operand are fused into one wide-N MMA, and A operands live in TMEM:
//   (c)   V^T T^T,             N = 64  -> U2^T           [A: V, shared memory]
//   MMA1  (d,e) S [-W ; Q~]^T, N = 128 -> [U2^T | O^T] += [A: S, TMEM]
//   MMA2  (f,g) U^T [P ; K~^T]^T, N=192 -> [O^T | S]  += [A: U^T, TMEM; B MN-major]
// with Q~ = diag(e^g) Q and K~ = diag(e^{g_C - g}) K.  (c) does not depend on the
// state, so its k-steps are issued right after MMA1 and MMA2 of the previous
// chunk and run while U^T and the new state are converted.  The fp32 state S lives in TMEM as an
// accumulator: before MMA2 it holds e^{g_C} S0, so MMA2 leaves S_C.  The operand
// tiles and the U, O accumulators alternate with chunk parity so that O is
// double-buffered while both fused MMAs keep contiguous outputs:
//   parity 0: B1 = [-W ; Q~], B2 = [P^T | K~], TMEM [U2 | O0 | S]
//   parity 1: B1 = [Q~ ; -W], B2 = [K~ | P^T], TMEM [S | O1 | U2']
// Per chunk, the critical chain is MMA1 -> U^T to fp16 -> MMA2 -> the fp16 copy
// of the new state.  While MMA1 runs, the 16 worker warps write the decayed state
// accumulator, build K~ and prepare the next chunk's gate vectors; while MMA2
// runs, they write the previous chunk's o tile (and zero its accumulator for the
// chunk after next).  A 17th warp issues every MMA and every copy, so that its
// waits on the tensor pipe delay no other work.  Loads are double-buffered: k, v (TMA)
// and the record (bulk copies) two chunks ahead, P one chunk ahead.
#pragma once
#include "device.cuh"
#include "intra.cuh"

namespace gdn {
namespace scan {

constexpr int C = 64;
constexpr int NW = 512;               // 16 worker warps: 4 per TMEM lane quadrant
constexpr int NT = NW + 32;           // + the issuing warp
constexpr int ISSUER = NW;            // lane 0 of warp 16: every MMA, load and store

// Shared memory (bytes from a 1024-aligned base); pairs are indexed by chunk parity.
constexpr uint32_t OFF_B1 = 0;          // x2: per 64-wide d_k half (16 KiB), 64 + 64 rows of -W / Q~
constexpr uint32_t B1_STRIDE = 32768;
constexpr uint32_t OFF_K = OFF_B1 + 2 * B1_STRIDE;   // K x2: 64 token rows x d_k, halves of 8192
constexpr uint32_t OFF_V = OFF_K + 2 * 16384;        // V x2: 64 token rows x d_v, halves of 8192
constexpr uint32_t OFF_T = OFF_V + 2 * 16384;        // T x2: 64 x 64
constexpr uint32_t OFF_B2 = OFF_T + 2 * 8192;        // x2: three MN-major 8 KiB atoms of P^T and K~
constexpr uint32_t B2_STRIDE = 24576;
constexpr uint32_t OFF_OST = OFF_B2 + 2 * B2_STRIDE; // o tile staging: 2 x 16 KiB (or 1 x 32 KiB)
constexpr uint32_t OFF_G = OFF_OST + 32768;          // g [2][64]
constexpr uint32_t OFF_KS = OFF_G + 512;             // e^{g_C - g} [2][64]
constexpr uint32_t OFF_BAR = OFF_KS + 512;           // mbarriers, TMEM address, abort flag, counters
constexpr uint32_t SMEM_USED = OFF_BAR + 128;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// Tensor memory: U2 | O0 | S (128) | O1 | U2' | S fp16 A (64) | U^T fp16 A (32)
constexpr uint32_t ACC_U0 = 0, ACC_O0 = 64, ACC_S = 128, ACC_O1 = 256, ACC_U1 = 320;
constexpr uint32_t TA_S = 384, TA_U = 448, TMEM_COLS = 512;
__host__ __device__ constexpr uint32_t acc_u(int b) { return b ? ACC_U1 : ACC_U0; }
__host__ __device__ constexpr uint32_t acc_o(int b) { return b ? ACC_O1 : ACC_O0; }

constexpr uint32_t KV_BYTES = 4 * 8192;
constexpr uint32_t REC_BYTES_IN = 4 * 8192 + 8192 + 256;   // -W, Q~ (two halves each), T, g

struct Args {
    float* rec_state;           // [N][Hv][dv][dk] in/out
    const int32_t* cu;          // [N+1]
    const int32_t* chunk_off;   // [N+1]
    const uint8_t* rec;         // intra-chunk records
    void* o;                    // [chunks][Hv][64][128] out dtype: o before the gated norm
    int Hk, Hv, dk, dv;
};

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint4 scale8(uint4 v, float s) {
    const float2 a = unpack_half2(v.x), b = unpack_half2(v.y), c = unpack_half2(v.z), d = unpack_half2(v.w);
    return make_uint4(pack_half2(a.x * s, a.y * s), pack_half2(b.x * s, b.y * s),
                      pack_half2(c.x * s, c.y * s), pack_half2(d.x * s, d.y * s));
}

template <typename TO>
__global__ void __launch_bounds__(NT, 1)
gdn_scan_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Args p) {
    constexpr uint32_t O_BYTES = C * 128 * sizeof(TO);
    constexpr int kOBufs = O_BYTES <= 16384 ? 2 : 1;   // staging buffers for the o tiles
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    float* s_g = reinterpret_cast<float*>(smem + OFF_G);
    float* s_ks = reinterpret_cast<float*>(smem + OFF_KS);
    const uint32_t bar = sb + OFF_BAR;                    // tensor-core commits
    const uint32_t bar_kv0 = sb + OFF_BAR + 8;            // +8 per parity: k, v tiles
    const uint32_t bar_rec0 = sb + OFF_BAR + 24;          // +8 per parity: -W, Q~, T, g
    const uint32_t bar_p0 = sb + OFF_BAR + 40;            // +8 per parity: P into B2
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 56);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 60);
    // loads issued per barrier (kv x2, record x2, P x2): the abort path waits for the last phase of each
    volatile int* s_issued = reinterpret_cast<volatile int*>(smem + OFF_BAR + 64);
    const uint32_t bar_fin = sb + OFF_BAR + 96;           // abort path: every MMA issued so far

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool worker = tid < NW;
    const int qd = warp & 3;      // TMEM lane quadrant
    const int cs = warp >> 2;     // column slice 0..3 (worker warps)
    const int Hv = p.Hv, dk = p.dk, dv = p.dv;
    const int seq = blockIdx.x / Hv, h = blockIdx.x % Hv;
    const int j = h / (Hv / p.Hk);
    const int64_t s0 = p.cu[seq], s1 = p.cu[seq + 1];
    const int nchunks = (int)((s1 - s0 + C - 1) / C);
    if (nchunks <= 0) return;
    const int64_t first = (int64_t)p.chunk_off[seq] * Hv + h;   // (chunk, head) index of chunk 0
    const uint8_t* rec0 = p.rec + first * intra::REC_BYTES;
    const int64_t rec_stride = (int64_t)Hv * intra::REC_BYTES;
    uint8_t* otile0 = static_cast<uint8_t*>(p.o) + first * O_BYTES;
    const int64_t o_stride = (int64_t)Hv * O_BYTES;

    // k, v tiles and the record (-W, Q~, T, g) of chunk ci into buffer ci & 1
    auto issue_chunk = [&](int ci) {
        const int bb = ci & 1;
        const int t = (int)(s0 + (int64_t)ci * C);
        s_issued[bb]++;
        mbar_arrive_expect_tx(bar_kv0 + 8 * bb, KV_BYTES);
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
            tma_load_3d(sb + OFF_K + bb * 16384 + hf * 8192, &tm_k, 64 * hf, j, t, bar_kv0 + 8 * bb);
            tma_load_3d(sb + OFF_V + bb * 16384 + hf * 8192, &tm_v, 64 * hf, h, t, bar_kv0 + 8 * bb);
        }
        const uint8_t* r = rec0 + ci * rec_stride;
        const uint32_t b1 = sb + OFF_B1 + bb * B1_STRIDE;
        const uint32_t wslot = bb ? 8192 : 0, qslot = bb ? 0 : 8192;   // row order of B1 by parity
        s_issued[2 + bb]++;
        mbar_arrive_expect_tx(bar_rec0 + 8 * bb, REC_BYTES_IN);
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
            bulk_g2s(b1 + hf * 16384 + wslot, r + intra::REC_W + hf * 8192, 8192, bar_rec0 + 8 * bb);
            bulk_g2s(b1 + hf * 16384 + qslot, r + intra::REC_Q + hf * 8192, 8192, bar_rec0 + 8 * bb);
        }
        bulk_g2s(sb + OFF_T + bb * 8192, r + intra::REC_T, 8192, bar_rec0 + 8 * bb);
        bulk_g2s(sb + OFF_G + bb * 256, r + intra::REC_G, 256, bar_rec0 + 8 * bb);
    };
    auto issue_p = [&](int ci) {   // P^T of chunk ci into its B2 atom (first at parity 0, last at 1)
        const int bb = ci & 1;
        s_issued[4 + bb]++;
        mbar_arrive_expect_tx(bar_p0 + 8 * bb, 8192);
        bulk_g2s(sb + OFF_B2 + bb * B2_STRIDE + (bb ? 16384 : 0), rec0 + ci * rec_stride + intra::REC_P, 8192,
                 bar_p0 + 8 * bb);
    };
    auto wait_par = [&](uint32_t bar0, int ci) {
        if (!mbar_wait_bounded(bar0 + 8 * (ci & 1), (ci >> 1) & 1)) atomicOr((unsigned*)s_abort, 2u);
    };

    if (tid == ISSUER) {
        mbar_init(bar, 1);
#pragma unroll
        for (int i = 0; i < 6; i++) mbar_init(bar_kv0 + 8 * i, 1);   // kv x2, rec x2, P x2
        mbar_init(bar_fin, 1);
        fence_mbar_init();
        *s_abort = 0;
        for (int i = 0; i < 6; i++) s_issued[i] = 0;
        issue_chunk(0);
        if (nchunks > 1) issue_chunk(1);
        issue_p(0);
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_BAR + 56, TMEM_COLS);
        tmem_relinquish();
    }
    const int dv_r = 32 * qd + lane;   // this worker's state row; columns [32 cs, 32 cs + 32)
    float* gstate = p.rec_state + ((int64_t)seq * Hv + h) * dv * dk;
    float Sv[32];   // this worker's slice of the state at the start of the current chunk
    if (worker) {
#pragma unroll
        for (int i = 0; i < 32; i++) {
            const int col = 32 * cs + i;
            Sv[i] = (dv_r < dv && col < dk) ? gstate[(int64_t)dv_r * dk + col] : 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    const float inv_sqrt_dk = rsqrtf((float)dk);
    uint32_t mphase = 0;

    // Shared-memory descriptors; per-step offsets are added to the start-address field.
    const uint64_t dV0 = sdesc(sb + OFF_V, 8192, 1024);
    const uint64_t dT0 = sdesc(sb + OFF_T, 16, 1024);
    const uint64_t dB10 = sdesc(sb + OFF_B1, 16, 1024);
    const uint64_t dB20 = sdesc(sb + OFF_B2, 8192, 1024);
    constexpr uint32_t ID_C = idesc_f16(128, 64, 1, 0);      // (c)
    constexpr uint32_t ID_DE = idesc_f16(128, 128, 0, 0);    // (d,e)
    constexpr uint32_t ID_FG = idesc_f16(128, 192, 0, 1);    // (f,g)

    // (c) of chunk ce, k-steps [k0, k1): U2^T = V^T T^T into its U accumulator (issuer; the
    // steps run in the tensor pipe's idle windows and are committed with the next MMA)
    auto issue_c = [&](int ce, int k0, int k1) {
        wait_par(bar_rec0, ce);
        wait_par(bar_kv0, ce);
        tc_fence_after();
        const int bb = ce & 1;
        for (int ks = k0; ks < k1; ks++)
            mma_f16(tmem + acc_u(bb), dV0 + bb * 1024 + ks * 128, dT0 + bb * 512 + ks * 2, ID_C, ks > 0);
    };
    // e^{g_C - g} (zero past the chunk's end) of chunk ce, by threads r0..r0+63
    auto chunk_vectors = [&](int ce, int r0) {
        wait_par(bar_rec0, ce);
        const int r = tid - r0;
        const float* rg = s_g + 64 * (ce & 1);
        s_ks[64 * (ce & 1) + r] = s0 + (int64_t)ce * C + r < s1 ? __expf(rg[C - 1] - rg[r]) : 0.f;
    };
    // fp16 copy of the state: the A operand of MMA1
    auto put_state_a = [&]() {
        uint32_t h16[16];
#pragma unroll
        for (int i = 0; i < 16; i++) h16[i] = pack_half2(Sv[2 * i], Sv[2 * i + 1]);
        tmem_st16(tl + TA_S + 16 * cs, h16);
    };
    // decayed state e^{g_C} S: the accumulator that MMA2 completes
    auto put_state_acc = [&](float decay) {
        uint32_t d[32];
#pragma unroll
        for (int i = 0; i < 32; i++) d[i] = __float_as_uint(decay * Sv[i]);
        tmem_st32(tl + ACC_S + 32 * cs, d);
    };
    // K~ = diag(e^{g_C - g}) K of chunk ce into its two B2 atoms (last two at parity 0, first two at 1)
    auto build_kt = [&](int ce) {
        wait_par(bar_kv0, ce);
        const int bb = ce & 1;
        const float* ks = s_ks + 64 * bb;
        const uint32_t dst = sb + OFF_B2 + bb * B2_STRIDE + (bb ? 0 : 8192);
        for (int idx = tid; idx < C * 16; idx += NW) {
            const int c = idx >> 4, c16 = idx & 15;
            const uint32_t off = (c16 >> 3) * 8192 + swz128(c, c16 & 7);
            const uint4 x = scale8(lds128(sb + OFF_K + bb * 16384 + off), ks[c]);
            sts128(dst + off, x.x, x.y, x.z, x.w);
        }
        fence_async_smem();
    };
    // o = O / sqrt(d_k) of chunk ce -> staging, and its accumulator zeroed for chunk ce + 2;
    // the issuer stores the tile after the next barrier (its buffer is free: see bulk_wait_read)
    auto stage_o = [&](int ce) {
        uint32_t o[16];
        tmem_ld16(tl + acc_o(ce & 1) + 16 * cs, o);
        TO* st = reinterpret_cast<TO*>(smem + OFF_OST + (ce % kOBufs) * 16384);
#pragma unroll
        for (int i = 0; i < 16; i++) from_f32(__uint_as_float(o[i]) * inv_sqrt_dk, st + (16 * cs + i) * 128 + dv_r);
        fence_async_smem();
#pragma unroll
        for (int i = 0; i < 16; i++) o[i] = 0u;
        tmem_st16(tl + acc_o(ce & 1) + 16 * cs, o);
    };
    auto issue_o = [&](int ce) {
        bulk_s2g(otile0 + ce * o_stride, sb + OFF_OST + (ce % kOBufs) * 16384, O_BYTES);
        bulk_commit();
    };

    // ---- prologue: zero O accumulators, fp16 S0, (c) and e^{g_C - g} of chunk 0 ----
    if (tid == ISSUER) issue_c(0, 0, 4);
    if (worker) {
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; i++) z[i] = 0u;
        tmem_st16(tl + ACC_O0 + 16 * cs, z);
        tmem_st16(tl + ACC_O1 + 16 * cs, z);
        put_state_a();
        if (tid < C) chunk_vectors(0, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (*s_abort) goto abort_;

#define GDN_MMA_WAIT()                                                                               \
    do {                                                                                             \
        if (tid == ISSUER && !mbar_wait_bounded(bar, mphase)) atomicOr((unsigned*)s_abort, 1u);    \
        mphase ^= 1u;                                                                                \
        __syncthreads();                                                                             \
        if (*s_abort) goto abort_;                                                                   \
        tc_fence_after();                                                                            \
    } while (0)

    for (int ci = 0; ci < nchunks; ci++) {
        const int b = ci & 1;

        // ---- MMA1: (d,e) [U2^T | O^T] += S [-W ; Q~]^T ((c) and zeroed O are already there) ----
        if (tid == ISSUER) {
            wait_par(bar_rec0, ci);
            tc_fence_after();
            const uint32_t d1 = tmem + (b ? ACC_O1 : ACC_U0);
#pragma unroll
            for (int ks = 0; ks < 8; ks++)
                mma_f16_ta(d1, tmem + TA_S + ks * 8, dB10 + b * 2048 + (ks >> 2) * 1024 + (ks & 3) * 2, ID_DE, 1);
            mma_commit(bar);
            if (ci + 1 < nchunks) issue_c(ci + 1, 0, 2);   // runs while U^T is converted
        }
        // ---- workers, while MMA1 runs: decayed state, next e^{g_C - g}, K~ ----
        if (worker) {
            put_state_acc(__expf(s_g[64 * b + C - 1]));
            if (tid >= 64 && tid < 64 + C && ci + 1 < nchunks) chunk_vectors(ci + 1, 64);
            build_kt(ci);
        }
        GDN_MMA_WAIT();

        // ---- U^T -> fp16 A operand; the issuer queues loads ----
        if (tid == ISSUER) {
            if (ci + 1 < nchunks) issue_p(ci + 1);   // its B2 atom was freed by MMA2 of chunk ci - 1
            if (ci + 2 < nchunks) {   // MMA1, (c) and K~ of chunk ci are done with buffer b
                fence_async_smem();
                issue_chunk(ci + 2);
            }
            if (kOBufs == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();   // staging buffer of stage_o(ci - 1)
        }
        if (worker) {
            uint32_t r16[16], u[8];
            tmem_ld16(tl + acc_u(b) + 16 * cs, r16);
#pragma unroll
            for (int i = 0; i < 8; i++) u[i] = pack_half2(__uint_as_float(r16[2 * i]), __uint_as_float(r16[2 * i + 1]));
            tmem_st8(tl + TA_U + 8 * cs, u);
        }
        tc_fence_before();
        __syncthreads();

        // ---- MMA2: [O^T | S] (parity 0) or [S | O^T] (parity 1) += U^T [P ; K~^T]^T ----
        if (tid == ISSUER) {
            wait_par(bar_p0, ci);
            tc_fence_after();
            const uint32_t d2 = tmem + (b ? ACC_S : ACC_O0);
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
                mma_f16_ta(d2, tmem + TA_U + ks * 8, dB20 + b * (B2_STRIDE >> 4) + ks * 128, ID_FG, 1);
            mma_commit(bar);
            if (ci + 1 < nchunks) issue_c(ci + 1, 2, 4);   // runs while the new state is converted
        }
        // ---- workers, while MMA2 runs: the previous chunk's o tile ----
        if (worker && ci > 0) stage_o(ci - 1);
        GDN_MMA_WAIT();

        // ---- new state: its fp16 copy for the next MMA1, or the final state ----
        if (tid == ISSUER && ci > 0) issue_o(ci - 1);
        if (worker) {
            uint32_t r32[32];
            tmem_ld32(tl + ACC_S + 32 * cs, r32);
#pragma unroll
            for (int i = 0; i < 32; i++) Sv[i] = __uint_as_float(r32[i]);
            if (ci + 1 < nchunks) {
                put_state_a();
            } else {
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int col = 32 * cs + i;
                    if (dv_r < dv && col < dk) gstate[(int64_t)dv_r * dk + col] = Sv[i];
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (*s_abort) goto abort_;
    }
    if (tid == ISSUER) {
        if (kOBufs == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();
    }
    __syncthreads();
    if (worker) stage_o(nchunks - 1);
    tc_fence_before();
    __syncthreads();
    if (tid == ISSUER) {
        issue_o(nchunks - 1);
        bulk_wait<0>();   // every o tile has reached global memory
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    return;

abort_:
    // A tensor-core commit or a copy never arrived: report it, give whatever is
    // still in flight one more bounded wait, free tensor memory and return.  The
    // recurrent state is left as it was.
    if (tid == ISSUER) {
        record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
        mma_commit(bar_fin);   // tracks every MMA this thread has issued
        mbar_wait_bounded(bar_fin, 0);
        for (int i = 0; i < 6; i++)   // the last phase issued on each barrier (returns at once if complete)
            if (s_issued[i] > 0) mbar_wait_bounded(bar_kv0 + 8 * i, (uint32_t)(s_issued[i] - 1) & 1u);
        bulk_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
#undef GDN_MMA_WAIT
}

}  // namespace scan
}  // namespace gdn
