// State chain of the chunked gated delta rule on the sm_100a tensor cores.
//
// One CTA (512 threads) walks one (sequence, value head) chain chunk by chunk
// (C = 64 tokens) and carries the d_v x d_k fp32 state in registers (row = TMEM
// lane, a quarter of d_k per warp).  The state-independent factors of every
// chunk come from the intra-chunk kernel's records (intra.cuh: -W, T, P, g).
// With S0 the state at the chunk start:
//     U   = T V - W S0^T                                    (exact per-token updates)
//     O   = (diag(e^g) Q S0^T + P U) / sqrt(d_k)
//     S_C = e^{g_C} S0 + U^T diag(e^{g_C - g}) K
// o goes out as [chunk][head][64][128] tiles; the gated RMSNorm that follows
// runs in norm.cuh, in parallel over all tiles.
//
// Products (tcgen05.mma kind::f16, fp16 operands, fp32 accumulators in TMEM,
// M = 128 = d_v always, the chunk is the N side):
//   (c) V^T T^T           -> U1^T                    [A: V in shared memory, MN-major]
//   (d) S (-W)^T          -> U2^T, U^T = U1^T + U2^T [A: S in TMEM; B: -W, MN-major]
//   (e) S Q~^T            -> O^T (Q~ = diag(e^g) Q)  [A: S in TMEM]
//   (f) U^T P^T           accumulated into (e)       [A: U^T in TMEM]
//   (g) U^T K~            -> state increment, K~ = diag(e^{g_C - g}) K [A: U^T in TMEM]
// S and U^T live in TMEM as fp16 A operands (written with tcgen05.st), so the
// tensor cores read only B tiles from shared memory.  MMAs that accumulate into
// one TMEM accumulator run back to back; (c), (d), (e) and then (f), (g) are
// issued interleaved across separate accumulators so that they overlap.  The
// chain per chunk is (c,d,e) -> U^T to fp16 -> (f,g) -> state update -> S to
// fp16, with the next chunk's Q~ and K~ prepared beside the state update and
// the o tile of chunk c-1 (O double-buffered in TMEM) formed and stored (one
// bulk copy) while (c,d,e) of chunk c run.  q^, k^, v^ tiles (double-buffered)
// and a chunk's record (one bulk copy) are fetched two chunks ahead.  One thread
// issues every MMA and waits on the tensor-core mbarrier; the others meet it at
// the CTA barrier.
#pragma once
#include "device.cuh"
#include "intra.cuh"

namespace gdn {
namespace scan {

constexpr int C = 64;
constexpr int NT = 512;   // 16 warps: 4 per TMEM lane quadrant
constexpr uint32_t REC_COPY = intra::REC_G + 256;   // bytes of a record brought in

constexpr uint32_t OFF_REC = 0;                     // two record buffers of REC_BYTES
constexpr uint32_t OFF_QKV = 2 * intra::REC_BYTES;  // two buffers of QKV_STRIDE:
constexpr uint32_t QKV_STRIDE = 49152;              //   [Q;K] 128 rows x d_k (halves of 16384), V
constexpr uint32_t QKV_V = 32768;                   //   V: 64 rows x d_v, halves of 8192
constexpr uint32_t OFF_OST = OFF_QKV + 2 * QKV_STRIDE;   // o tile staging: 32 KiB
constexpr uint32_t OFF_KT = OFF_OST + 32768;        // K~: 64 rows x d_k, halves of 8192
constexpr uint32_t OFF_EG = OFF_KT + 16384;         // e^g [2][64]
constexpr uint32_t OFF_KS = OFF_EG + 512;           // e^{g_C - g} [2][64]
constexpr uint32_t OFF_BAR = OFF_KS + 512;          // mbarriers, TMEM address, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// Tensor memory: U1^T, U2^T (64 each), O^T x2 (128), increment (128), S fp16 A
// operand (64 columns of packed pairs), U^T fp16 A operand (32).
constexpr uint32_t ACC_U1 = 0, ACC_U2 = 64, ACC_O = 128, ACC_SI = 256, TA_S = 384, TA_U = 448, TMEM_COLS = 512;
constexpr uint32_t QKV_BYTES = 6 * 8192;

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
gdn_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, Args p) {
    constexpr uint32_t O_BYTES = C * 128 * sizeof(TO);
    constexpr int kOBufs = O_BYTES <= 16384 ? 2 : 1;   // staging buffers for the o tiles
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    float* s_eg = reinterpret_cast<float*>(smem + OFF_EG);
    float* s_ks = reinterpret_cast<float*>(smem + OFF_KS);
    const uint32_t bar = sb + OFF_BAR;
    const uint32_t bar_qkv0 = sb + OFF_BAR + 8, bar_qkv1 = sb + OFF_BAR + 16;
    const uint32_t bar_rec0 = sb + OFF_BAR + 24, bar_rec1 = sb + OFF_BAR + 32;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 40);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 44);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3;      // TMEM lane quadrant
    const int cs = warp >> 2;     // column slice 0..3
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

    // TMA / bulk loads issued (thread 0) and completed waits on them (each thread
    // counts its own), for the abort path
    int qkv_issued[2] = {0, 0}, qkv_ok[2] = {0, 0}, rec_issued[2] = {0, 0}, rec_ok[2] = {0, 0};
    auto issue_qkv = [&](int ci) {
        const int t = (int)(s0 + (int64_t)ci * C);
        const uint32_t bb = (ci & 1) ? bar_qkv1 : bar_qkv0;
        const uint32_t base = sb + OFF_QKV + (ci & 1) * QKV_STRIDE;
        if (ci & 1) qkv_issued[1]++; else qkv_issued[0]++;
        mbar_arrive_expect_tx(bb, QKV_BYTES);
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
            tma_load_3d(base + hf * 16384, &tm_q, 64 * hf, j, t, bb);
            tma_load_3d(base + hf * 16384 + C * 128, &tm_k, 64 * hf, j, t, bb);
            tma_load_3d(base + QKV_V + hf * 8192, &tm_v, 64 * hf, h, t, bb);
        }
    };
    auto issue_rec = [&](int ci) {
        const uint32_t bb = (ci & 1) ? bar_rec1 : bar_rec0;
        if (ci & 1) rec_issued[1]++; else rec_issued[0]++;
        mbar_arrive_expect_tx(bb, REC_COPY);
        bulk_g2s(sb + OFF_REC + (ci & 1) * intra::REC_BYTES, rec0 + ci * rec_stride, REC_COPY, bb);
    };
    auto wait_buf = [&](uint32_t b0, uint32_t b1, int (&ok)[2], int ci) {
        const uint32_t bb = (ci & 1) ? b1 : b0;
        if (mbar_wait_bounded(bb, (ci >> 1) & 1)) {
            if (ci & 1) ok[1]++; else ok[0]++;
        } else {
            atomicOr((unsigned*)s_abort, 2u);
        }
    };

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_qkv0, 1);
        mbar_init(bar_qkv1, 1);
        mbar_init(bar_rec0, 1);
        mbar_init(bar_rec1, 1);
        fence_mbar_init();
        *s_abort = 0;
        issue_qkv(0);
        issue_rec(0);
        if (nchunks > 1) {
            issue_qkv(1);
            issue_rec(1);
        }
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_BAR + 40, TMEM_COLS);
        tmem_relinquish();
    }

    // fp32 state: row dv_r, columns [32 cs, 32 cs + 32)
    const int dv_r = 32 * qd + lane;
    float S[32];
    float* gstate = p.rec_state + ((int64_t)seq * Hv + h) * dv * dk;
#pragma unroll
    for (int i = 0; i < 32; i++) {
        const int col = 32 * cs + i;
        S[i] = (dv_r < dv && col < dk) ? gstate[(int64_t)dv_r * dk + col] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    const float inv_sqrt_dk = rsqrtf((float)dk);
    uint32_t mphase = 0;

    // S -> fp16 A operand in TMEM: this thread's 32 columns of d_k = 16 packed columns
    auto write_sa = [&]() {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; i++) r[i] = pack_half2(S[2 * i], S[2 * i + 1]);
        tmem_st16(tl + TA_S + 16 * cs, r);
    };
    // o = O / sqrt(d_k) of chunk ce -> staging buffer; tid 0 stores it with one bulk
    // copy after the next CTA barrier (issue_o).
    auto stage_o = [&](int ce) {
        uint32_t o[16];
        tmem_ld16(tl + ACC_O + 64 * (ce & 1) + 16 * cs, o);
        TO* st = reinterpret_cast<TO*>(smem + OFF_OST + (ce % kOBufs) * 16384);
#pragma unroll
        for (int i = 0; i < 16; i++) from_f32(__uint_as_float(o[i]) * inv_sqrt_dk, st + (16 * cs + i) * 128 + dv_r);
        fence_async_smem();
    };
    auto issue_o = [&](int ce) {
        bulk_s2g(otile0 + ce * o_stride, sb + OFF_OST + (ce % kOBufs) * 16384, O_BYTES);
        bulk_commit();
    };
    // e^g and e^{g_C - g} (zero past the chunk's end) of chunk ce, threads 0..63
    auto chunk_vectors = [&](int ce) {
        wait_buf(bar_rec0, bar_rec1, rec_ok, ce);
        const float* rg = reinterpret_cast<const float*>(smem + OFF_REC + (ce & 1) * intra::REC_BYTES + intra::REC_G);
        const float g = rg[tid], gl = rg[C - 1];
        s_eg[64 * (ce & 1) + tid] = __expf(g);
        s_ks[64 * (ce & 1) + tid] = s0 + (int64_t)ce * C + tid < s1 ? __expf(gl - g) : 0.f;
    };
    // Q~ = diag(e^g) Q in place and K~ = diag(e^{g_C - g}) K of chunk ce (all threads)
    auto scale_qk = [&](int ce) {
        wait_buf(bar_qkv0, bar_qkv1, qkv_ok, ce);
        const uint32_t qkv = sb + OFF_QKV + (ce & 1) * QKV_STRIDE;
        const float* eg = s_eg + 64 * (ce & 1);
        const float* ks = s_ks + 64 * (ce & 1);
        for (int idx = tid; idx < 2 * C * 16; idx += NT) {
            const int isk = idx >= C * 16;
            const int r = (idx & (C * 16 - 1)) >> 4, c16 = idx & 15;
            const int hf = c16 >> 3, cc = c16 & 7;
            const uint32_t src = qkv + hf * 16384 + swz128(isk * C + r, cc);
            const uint4 x = scale8(lds128(src), isk ? ks[r] : eg[r]);
            const uint32_t dst = isk ? sb + OFF_KT + hf * 8192 + swz128(r, cc) : src;
            sts128(dst, x.x, x.y, x.z, x.w);
        }
        fence_async_smem();
    };

    // Shared-memory descriptors; per-step offsets are added to the start-address field.
    const uint64_t dV0 = sdesc(sb + OFF_QKV + QKV_V, 8192, 1024);
    const uint64_t dQ0 = sdesc(sb + OFF_QKV, 16, 1024);
    const uint64_t dKT = sdesc(sb + OFF_KT, 8192, 1024);
    const uint64_t dT0 = sdesc(sb + OFF_REC + intra::REC_T, 16, 1024);
    const uint64_t dW0 = sdesc(sb + OFF_REC + intra::REC_W, 8192, 1024);
    const uint64_t dP0 = sdesc(sb + OFF_REC + intra::REC_P, 16, 1024);
    constexpr uint64_t kRecStep = intra::REC_BYTES >> 4, kQkvStep = QKV_STRIDE >> 4;
    constexpr uint32_t ID_MK = idesc_f16(128, 64, 1, 0), ID_KM = idesc_f16(128, 64, 0, 1);
    constexpr uint32_t ID_KK = idesc_f16(128, 64, 0, 0), ID_KM128 = idesc_f16(128, 128, 0, 1);

    write_sa();
    if (tid < C) chunk_vectors(0);
    tc_fence_before();
    __syncthreads();
    if (*s_abort) goto abort_;
    scale_qk(0);
    __syncthreads();
    if (*s_abort) goto abort_;

#define GDN_MMA_WAIT()                                                                        \
    do {                                                                                      \
        if (tid == 0 && !mbar_wait_bounded(bar, mphase)) atomicOr((unsigned*)s_abort, 1u);  \
        mphase ^= 1u;                                                                         \
        __syncthreads();                                                                      \
        if (*s_abort) goto abort_;                                                            \
        tc_fence_after();                                                                     \
    } while (0)

    for (int ci = 0; ci < nchunks; ci++) {
        const int b = ci & 1;
        const uint64_t rs = b ? kRecStep : 0, qs = b ? kQkvStep : 0;

        // ---- (c) U1^T = V^T T^T, (d) U2^T = S (-W)^T, (e) O^T = S Q~^T, interleaved ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t dO = tmem + ACC_O + 64 * b;
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                if (ks < 4) mma_f16(tmem + ACC_U1, dV0 + qs + ks * 128, dT0 + rs + ks * 2, ID_MK, ks > 0);
                mma_f16_ta(tmem + ACC_U2, tmem + TA_S + ks * 8, dW0 + rs + ks * 128, ID_KM, ks > 0);
                mma_f16_ta(dO, tmem + TA_S + ks * 8, dQ0 + qs + (ks >> 2) * 1024 + (ks & 3) * 2, ID_KK, ks > 0);
            }
            mma_commit(bar);
        }
        // ---- while they run: the previous o tile; the next chunk's e^g, e^{g_C - g} ----
        if (ci > 0) stage_o(ci - 1);
        if (tid < C && ci + 1 < nchunks) chunk_vectors(ci + 1);
        GDN_MMA_WAIT();
        if (tid == 0 && ci > 0) issue_o(ci - 1);

        // ---- U^T = U1^T + U2^T -> fp16 A operand in TMEM ----
        {
            uint32_t r1[16], r2[16], u[8];
            tmem_ld16(tl + ACC_U1 + 16 * cs, r1);
            tmem_ld16(tl + ACC_U2 + 16 * cs, r2);
#pragma unroll
            for (int i = 0; i < 8; i++)
                u[i] = pack_half2(__uint_as_float(r1[2 * i]) + __uint_as_float(r2[2 * i]),
                                  __uint_as_float(r1[2 * i + 1]) + __uint_as_float(r2[2 * i + 1]));
            tmem_st8(tl + TA_U + 8 * cs, u);
        }
        tc_fence_before();
        __syncthreads();

        // ---- (f) O^T += U^T P^T, (g) increment = U^T K~, interleaved ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t dO = tmem + ACC_O + 64 * b;
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                mma_f16_ta(dO, tmem + TA_U + ks * 8, dP0 + rs + ks * 2, ID_KK, 1);
                mma_f16_ta(tmem + ACC_SI, tmem + TA_U + ks * 8, dKT + ks * 128, ID_KM128, ks > 0);
            }
            mma_commit(bar);
        }
        GDN_MMA_WAIT();
        if (tid == 0) {   // buffers of chunk ci consumed: fetch chunk ci + 2's tiles and record
            if (ci + 2 < nchunks) {
                fence_async_smem();
                issue_qkv(ci + 2);
                issue_rec(ci + 2);
            }
            if (kOBufs == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();   // next staging buffer read
        }

        // ---- S <- e^{g_C} S + U^T K~ and its fp16 A operand; the next chunk's Q~, K~ ----
        {
            const float eg = s_eg[64 * b + C - 1];
            uint32_t r32[32];
            tmem_ld32(tl + ACC_SI + 32 * cs, r32);
#pragma unroll
            for (int i = 0; i < 32; i++) S[i] = fmaf(eg, S[i], __uint_as_float(r32[i]));
            write_sa();
        }
        if (ci + 1 < nchunks) scale_qk(ci + 1);
        tc_fence_before();
        __syncthreads();
        if (*s_abort) goto abort_;
    }
    stage_o(nchunks - 1);
    tc_fence_before();
    __syncthreads();
    if (tid == 0) issue_o(nchunks - 1);

    // ---- final state ----
#pragma unroll
    for (int i = 0; i < 32; i++) {
        const int col = 32 * cs + i;
        if (dv_r < dv && col < dk) gstate[(int64_t)dv_r * dk + col] = S[i];
    }
    if (tid == 0) bulk_wait<0>();   // every o tile has reached global memory
    tc_fence_before();
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
    if (tid == 0) {
        record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
        for (int bb = 0; bb < 2; bb++) {
            for (int k = qkv_ok[bb]; k < qkv_issued[bb]; k++) mbar_wait_bounded(bb ? bar_qkv1 : bar_qkv0, k & 1);
            for (int k = rec_ok[bb]; k < rec_issued[bb]; k++) mbar_wait_bounded(bb ? bar_rec1 : bar_rec0, k & 1);
        }
        bulk_wait<0>();
    }
    if (warp == 0) {
        mbar_wait_bounded(bar, mphase ^ 1u);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
#undef GDN_MMA_WAIT
}

}  // namespace scan
}  // namespace gdn
