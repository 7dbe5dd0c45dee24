// State chain of the chunked gated delta rule on the sm_100a tensor cores.
//
// One CTA (18 warps) walks one (sequence, value head) chain chunk by chunk
// (C = 64 tokens).  The state-independent factors of every chunk come from the
// intra-chunk kernel's records (intra.cuh: -W, Q~, T, the decay factors, P^T),
// whose tiles are already the shared-memory images the tensor cores read; v^
// and k^ come from the conv outputs by TMA.  With S0 the state at the chunk
// start, D = diag(e^{g_C - g}) and Q~ = diag(e^g) Q:
//     U   = T V - W S0^T                                    (exact per-token updates)
//     O   = (Q~ S0^T + P U) / sqrt(d_k)
//     S_C = e^{g_C} S0 + (D U)^T K
// o goes out as [chunk][head][64][128] tiles; the gated RMSNorm that follows
// runs in norm.cuh, in parallel over all tiles.  A launch may walk only a range
// of global chunks (a pipelined prefill): the state then passes to the next
// launch in fp32 through a carry buffer, so the arithmetic is the same as in
// one launch, bit for bit.
//
// A tcgen05.mma costs about the same whatever its N up to 128, so products that
// share an A operand are fused into one wide-N MMA, and A operands live in TMEM:
//   (c)   V^T T^T,              N = 64  -> U2^T          [A: V, shared memory; T as fp16 hi + lo]
//   MMA1  S [-W ; Q~]^T,        N = 128 -> [U2^T | O^T] += [A: S, TMEM]
//   MMA2a (D U)^T K,            N = 128 -> S  +=          [A: (D U)^T, TMEM; B: k^, MN-major]
//   MMA2b U^T P^T,              N = 64  -> O^T +=         [A: U^T, TMEM; B: P^T, MN-major]
// The fp32 state S lives in TMEM as an accumulator: before MMA2a the workers
// store e^{g_C} S0 into it, so MMA2a leaves S_C.  The decay D rides on the fp16
// copy of U that the workers make anyway (a second, scaled copy), so the raw k^
// tile is MMA2a's operand as it arrives.  U and O accumulators alternate with
// chunk parity, O double-buffered.
//
// Per chunk, the critical chain is MMA1 -> U^T to fp16 -> MMA2a -> the fp16 copy
// of the new state.  A dedicated warp issues every MMA: right after MMA1 it
// queues the first half of (c) of the next chunk, which runs while U is
// converted, and right after MMA2a it queues MMA2b and then the second half of
// (c), which run while the state is converted; it waits for
// the next MMA's operands while the workers convert, so each conversion is
// followed by an immediate issue.  While MMA1 runs, the 16 worker warps write the
// decayed state accumulator and stage the previous chunk's o tile (once its MMA2b
// has completed; MMA1's first K step restarts each O accumulator); MMA2a, the
// shortest product, is left to run alone.  An 18th warp issues
// every copy: a bulk copy holds its issuing thread for about as long as the copy
// engine takes to walk its bytes, so copies stay off the MMA chain.  It meets
// the others only through mbarriers (buffer released, o tile staged, staging
// buffer free), never at a CTA barrier.  Loads run two chunks ahead: v (TMA) and
// the record's B1 image, T and decay factors (one bulk copy) on one barrier; k^
// (TMA) and P^T (one bulk copy) on another.
#pragma once
#include "device.cuh"
#include "intra.cuh"

namespace gdn {
namespace scan {

constexpr int C = kChunk;
constexpr int NW = 512;               // 16 worker warps: 4 per TMEM lane quadrant
constexpr int IW = NW / 32;           // the issuing warp: every MMA
constexpr int LW = IW + 1;            // the loading warp: every copy
constexpr int NMAIN = NW + 32;        // workers + issuer: they meet at named barrier 1
constexpr int NT = NMAIN + 32;

// Shared memory (bytes from a 1024-aligned base); pairs are indexed by chunk parity.
constexpr uint32_t OFF_R = 0;           // x2: the record's B1 image (32 KiB), T hi and lo (16 KiB), decay factors
constexpr uint32_t R_STRIDE = 50176;
constexpr uint32_t R_T = intra::REC_T - intra::REC_B1, R_G = intra::REC_G - intra::REC_B1;
constexpr uint32_t OFF_V = OFF_R + 2 * R_STRIDE;     // V x2: 64 token rows x d_v, halves of 8192
constexpr uint32_t OFF_B2 = OFF_V + 2 * 16384;       // x2: [K half 0 | K half 1 | P^T], MN-major atoms
constexpr uint32_t B2_STRIDE = 24576;
constexpr uint32_t OFF_OST = OFF_B2 + 2 * B2_STRIDE; // o tile staging: 2 x 16 KiB (or 1 x 32 KiB)
constexpr uint32_t OFF_BAR = OFF_OST + 32768;        // mbarriers, TMEM address, abort flag, counters
constexpr uint32_t SMEM_USED = OFF_BAR + 192;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(R_STRIDE % 1024 == 0 && R_STRIDE >= intra::REC_LD_BYTES, "record slot");

// Tensor memory: [U2 | O] for parity 0 and 1, S (128), S fp16 A (64), U^T fp16 A (32), (D U)^T fp16 A (32)
constexpr uint32_t ACC_S = 256, TA_S = 384, TA_U = 448, TA_UD = 480, TMEM_COLS = 512;
__host__ __device__ constexpr uint32_t acc_u(int b) { return b ? 128u : 0u; }
__host__ __device__ constexpr uint32_t acc_o(int b) { return acc_u(b) + 64u; }

constexpr uint32_t LD_BYTES = 2 * 8192 + intra::REC_LD_BYTES;   // v halves + B1, T, decay factors
constexpr uint32_t B2_BYTES = 2 * 8192 + 8192;                  // k^ halves + P^T

struct Args {
    void* rec_state;            // [N][Hv][dv][dk] state dtype (fp32 or bf16), in/out
    float* carry;               // [N][Hv][dv][dk] fp32: the state from one launch over a chunk range to the next
    int32_t g_lo, g_hi;         // this launch walks global chunks [g_lo, g_hi) of every chain
    int32_t final_launch;       // nonzero: the call's last launch, which writes the final states
    const int32_t* cu;          // [N+1]
    const int32_t* chunk_off;   // [N+1]
    const int32_t* flags;       // nonzero: a device check of the call failed, write nothing
    const uint8_t* rec;         // intra-chunk records
    void* o;                    // [chunks][Hv][64][128] out dtype: o before the gated norm
    int Hk, Hv, dk, dv;
};

// 4 consecutive state entries: fp32, or bf16 storage (read exactly, written
// round-to-nearest-even); the chain itself always runs in fp32
__device__ __forceinline__ float4 ld_state4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld_state4(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ void st_state4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void st_state4(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}

__device__ __forceinline__ void main_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NMAIN) : "memory"); }
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <typename TO, typename TS>
__global__ void __launch_bounds__(NT, 1)
gdn_scan_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k, Args p) {
    constexpr uint32_t O_BYTES = C * 128 * sizeof(TO);
    constexpr int kOBufs = O_BYTES <= 16384 ? 2 : 1;   // staging buffers for the o tiles
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    const uint32_t bar = sb + OFF_BAR;                    // tensor-core commits of MMA1 and MMA2a (issuer)
    const uint32_t bar_ld0 = sb + OFF_BAR + 8;            // [2] v, B1, T, decay factors arrived
    const uint32_t bar_b20 = sb + OFF_BAR + 24;           // [2] k^, P^T arrived
    const uint32_t bar_fin = sb + OFF_BAR + 40;           // abort path: every MMA issued so far
    const uint32_t ev10 = sb + OFF_BAR + 48;              // [2] MMA1 of a chunk done: its v/record buffer is free
    const uint32_t ev20 = sb + OFF_BAR + 64;              // [2] MMA2b of a chunk done (tensor-core arrive): B2 free
    const uint32_t evo = sb + OFF_BAR + 80;               // a staging buffer is free again
    const uint32_t ev_end = sb + OFF_BAR + 88;            // the last o tile is staged
    const uint32_t ev_st = sb + OFF_BAR + 96;             // [2] o tile of a chunk staged
    const uint32_t ev_ldone = sb + OFF_BAR + 120;         // the loading warp has drained everything
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 128);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 132);
    // loads issued per barrier (ld x2, B2 x2): the loader's drain waits for the last phase of each
    volatile int* s_issued = reinterpret_cast<volatile int*>(smem + OFF_BAR + 136);
    // the issuer has issued MMA1 (phase parity 0) or MMA2a (parity 1) of the current chunk: the
    // workers' TMEM traffic waits for it so that it does not slow the issue down
    const uint32_t ev_iss = sb + OFF_BAR + 152;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool worker = tid < NW;
    const int qd = warp & 3;      // TMEM lane quadrant
    const int cs = warp >> 2;     // column slice 0..3 (worker warps)
    const int Hv = p.Hv, dk = p.dk, dv = p.dv;
    const int seq = blockIdx.x / Hv, h = blockIdx.x % Hv;
    const int kh = h / (Hv / p.Hk);
    const int n_all = (int)((p.cu[seq + 1] - (int64_t)p.cu[seq] + C - 1) / C);   // chunks of the sequence
    if (n_all <= 0 || *p.flags) return;
    // This launch walks chunks [c0, c1) of the sequence.  Its start state is rec_state at the
    // sequence's first chunk, else the carry a launch before left; its end state goes to
    // rec_state after the sequence's last chunk in the call's last launch, else to the carry.
    const int cfirst = p.chunk_off[seq];
    const int c0 = p.g_lo > cfirst ? p.g_lo - cfirst : 0;
    const int c1 = p.g_hi - cfirst < n_all ? p.g_hi - cfirst : n_all;
    TS* gstate = static_cast<TS*>(p.rec_state) + ((int64_t)seq * Hv + h) * dv * dk;
    float* cstate = p.carry ? p.carry + ((int64_t)seq * Hv + h) * dv * dk : nullptr;
    if (c0 >= c1) {
        // a sequence that ended before this range: the last launch moves its end state from the carry
        if (p.final_launch && c0 >= n_all && p.g_lo > cfirst && cstate) {
            for (int i = 4 * threadIdx.x; i < dv * dk; i += 4 * NT)
                st_state4(gstate + i, ld_state4(cstate + i));
        }
        return;
    }
    const bool from_rec = c0 == 0, to_rec = c1 == n_all && p.final_launch;
    if ((!from_rec || !to_rec) && !cstate) return;   // (the host always passes a carry when it splits a chain)
    const int nchunks = c1 - c0;
    // tokens in this launch's last chunk: the rows after them are zeroed before the tensor cores
    // read them (they hold another sequence's tokens, or rows a later launch has yet to write)
    const int n_tail = c1 == n_all ? (int)(p.cu[seq + 1] - p.cu[seq] - (int64_t)(n_all - 1) * C) : C;
    const int64_t s0 = p.cu[seq] + (int64_t)c0 * C;
    const int64_t first = ((int64_t)cfirst + c0) * Hv + h;   // (chunk, head) index of chunk c0
    const uint8_t* rec0 = p.rec + first * intra::REC_BYTES;
    const int64_t rec_stride = (int64_t)Hv * intra::REC_BYTES;
    uint8_t* otile0 = static_cast<uint8_t*>(p.o) + first * O_BYTES;
    const int64_t o_stride = (int64_t)Hv * O_BYTES;

    // ---- the loading warp's copies ----
    auto issue_chunk = [&](int ci) {   // v tile and the record's B1 image, T and decay factors of chunk ci
        const int bb = ci & 1;
        if (lane == 0) s_issued[bb]++;
        mbar_arrive_expect_tx_w(bar_ld0 + 8 * bb, LD_BYTES);
#pragma unroll
        for (int hf = 0; hf < 2; hf++)
            tma_load_3d_w(sb + OFF_V + bb * 16384 + hf * 8192, &tm_v, 64 * hf, h, (int)(s0 + (int64_t)ci * C),
                          bar_ld0 + 8 * bb);
        bulk_g2s_w(sb + OFF_R + bb * R_STRIDE, rec0 + ci * rec_stride + intra::REC_B1, intra::REC_LD_BYTES,
                   bar_ld0 + 8 * bb);
    };
    auto issue_b2 = [&](int ci) {   // k^ tile and the record's P^T of chunk ci
        const int bb = ci & 1;
        if (lane == 0) s_issued[2 + bb]++;
        mbar_arrive_expect_tx_w(bar_b20 + 8 * bb, B2_BYTES);
#pragma unroll
        for (int hf = 0; hf < 2; hf++)
            tma_load_3d_w(sb + OFF_B2 + bb * B2_STRIDE + hf * 8192, &tm_k, 64 * hf, kh, (int)(s0 + (int64_t)ci * C),
                          bar_b20 + 8 * bb);
        bulk_g2s_w(sb + OFF_B2 + bb * B2_STRIDE + 16384, rec0 + ci * rec_stride + intra::REC_P, 8192,
                   bar_b20 + 8 * bb);
    };
    auto issue_o = [&](int ce) {
        bulk_s2g_commit_w(otile0 + ce * o_stride, sb + OFF_OST + (ce % kOBufs) * 16384, O_BYTES);
    };
    auto wait_par = [&](uint32_t bar0, int ci) {
        if (!mbar_wait_bounded(bar0 + 8 * (ci & 1), (ci >> 1) & 1)) atomicOr((unsigned*)s_abort, 2u);
    };

    if (warp == LW) {
        if (lane == 0) {
            mbar_init(bar, 1);
#pragma unroll
            for (int i = 0; i < 15; i++) mbar_init(bar_ld0 + 8 * i, 1);   // ld, B2, fin, ev1, ev2, evo, end, st, -, ldone
            mbar_init(ev_iss, 1);
            fence_mbar_init();
            *s_abort = 0;
            for (int i = 0; i < 4; i++) s_issued[i] = 0;
        }
        __syncwarp();
        issue_chunk(0);   // chunk 1's loads follow once the chain can start
        issue_b2(0);
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_BAR + 128, TMEM_COLS);
        tmem_relinquish();
    }
    const int dv_r = 32 * qd + lane;   // this worker's state row; columns [32 cs, 32 cs + 32)
    float Sv[32];   // this worker's slice of the state at the start of the current chunk
    if (worker) {
#pragma unroll
        for (int i4 = 0; i4 < 8; i4++) {   // 16-byte loads (d_k and the slice start are multiples of 4)
            const int col = 32 * cs + 4 * i4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (dv_r < dv && col < dk)
                v = from_rec ? ld_state4(gstate + (int64_t)dv_r * dk + col) : ld_state4(cstate + (int64_t)dv_r * dk + col);
            Sv[4 * i4] = v.x; Sv[4 * i4 + 1] = v.y; Sv[4 * i4 + 2] = v.z; Sv[4 * i4 + 3] = v.w;
        }
    }
    tc_fence_before();
    __syncthreads();   // every warp: barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == LW) {
        // Waits for an event of the other warps; gives up on their abort or after the time limit.
        auto lwait = [&](uint32_t b, uint32_t parity) -> bool {
            if (mbar_try_wait(b, parity)) return true;
            const unsigned long long t0 = global_ns();
            while (!mbar_try_wait(b, parity)) {
                if (*s_abort) return false;
                if (global_ns() - t0 > kWaitLimitNs) {
                    atomicOr((unsigned*)s_abort, 2u);
                    return false;
                }
            }
            return true;
        };
        if (nchunks > 1) {
            issue_chunk(1);
            issue_b2(1);
        }
        bool ok = true;
        for (int ci = 0; ci < nchunks && ok; ci++) {
            if (ci > 0) {   // o of chunk ci - 1 was staged while MMA1 of chunk ci ran
                ok = lwait(ev_st + 8 * ((ci - 1) & 1), ((ci - 1) >> 1) & 1);
                if (!ok) break;
                issue_o(ci - 1);
            }
            if (kOBufs == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();   // the staging buffer of o(ci) is free
            if (lane == 0) mbar_arrive(evo);
            if (ci + 2 < nchunks) {
                ok = lwait(ev10 + 8 * (ci & 1), (ci >> 1) & 1);     // MMA1 of chunk ci is done with buffer ci & 1
                if (!ok) break;
                fence_async_smem();
                issue_chunk(ci + 2);
                ok = lwait(ev20 + 8 * (ci & 1), (ci >> 1) & 1);     // MMA2b of chunk ci is done with B2 buffer ci & 1
                if (!ok) break;
                issue_b2(ci + 2);
            }
        }
        if (ok && lwait(ev_end, 0)) issue_o(nchunks - 1);
        // drain: every copy this warp issued completes before the CTA may exit
        bulk_wait<0>();
        if (lane == 0)
            for (int i = 0; i < 4; i++)   // the last phase issued on each load barrier (returns at once if complete)
                if (s_issued[i] > 0) mbar_wait_bounded(bar_ld0 + 8 * i, (uint32_t)(s_issued[i] - 1) & 1u);
        __syncwarp();
        if (lane == 0) mbar_arrive(ev_ldone);
        return;
    }

    // ---- workers and the issuer ----
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    const float inv_sqrt_dk = rsqrtf((float)dk);
    uint32_t mphase = 0;
    const uint64_t dB1 = sdesc(sb + OFF_R, 16, 1024);
    const uint64_t dK = sdesc(sb + OFF_B2, 8192, 1024);
    const uint64_t dP = sdesc(sb + OFF_B2 + 16384, 8192, 1024);
    const uint64_t dV0 = sdesc(sb + OFF_V, 8192, 1024);
    const uint64_t dT0 = sdesc(sb + OFF_R + R_T, 16, 1024);
    constexpr uint32_t ID_1 = idesc_f16(128, 128, 0, 0);    // MMA1
    constexpr uint32_t ID_1H = idesc_f16(128, 64, 0, 0);    // MMA1's first K step, one half at a time
    constexpr uint32_t ID_2A = idesc_f16(128, 128, 0, 1);   // MMA2a
    constexpr uint32_t ID_2B = idesc_f16(128, 64, 0, 1);    // MMA2b
    constexpr uint32_t ID_C = idesc_f16(128, 64, 1, 0);     // (c)
    // (c) of chunk ce: U2^T = V^T T^T into its U accumulator (MMA1 of chunk ce accumulates onto it;
    // the tensor pipe runs one thread's MMAs in order)
    // T = fp16(T) + its fp16 remainder: pass 0 over fp16(T) (which starts the accumulator), pass 1
    // over the remainder.  They are queued where the tensor pipe would otherwise idle: pass 0 of
    // the next chunk right after MMA1 (it runs while U is converted), pass 1 right after MMA2b
    // (while the state is converted); MMA1 of that chunk follows both in the pipe.
    auto issue_c = [&](int ce, int pass) {
        const int bb = ce & 1;
        if (pass == 0 && ce == nchunks - 1 && n_tail < C) {
            zero_tile_rows(sb + OFF_V + bb * 16384, 2, n_tail, lane, 32);
            fence_async_smem();
            __syncwarp();
        }
#pragma unroll
        for (int ks = 0; ks < 4; ks++)
            mma_f16_w(tmem + acc_u(bb), dV0 + bb * 1024 + ks * 128,
                      dT0 + bb * (R_STRIDE >> 4) + pass * (8192 >> 4) + ks * 2, ID_C, pass > 0 || ks > 0);
    };
    // fp16 copy of the state: the A operand of MMA1
    auto put_state_a = [&]() {
        uint32_t h16[16];
#pragma unroll
        for (int i = 0; i < 16; i++) h16[i] = pack_half2(Sv[2 * i], Sv[2 * i + 1]);
        tmem_st16(tl + TA_S + 16 * cs, h16);
    };
    // decayed state e^{g_C} S: the accumulator that MMA2a completes
    auto put_state_acc = [&](float decay) {
        uint32_t d[32];
#pragma unroll
        for (int i = 0; i < 32; i++) d[i] = __float_as_uint(decay * Sv[i]);
        tmem_st32(tl + ACC_S + 32 * cs, d);
    };
    // o = O / sqrt(d_k) of chunk ce -> staging (MMA1 of chunk ce + 2 restarts the accumulator)
    auto stage_o = [&](int ce) {
        uint32_t o[16];
        tmem_ld16(tl + acc_o(ce & 1) + 16 * cs, o);
        TO* st = reinterpret_cast<TO*>(smem + OFF_OST + (ce % kOBufs) * 16384);
#pragma unroll
        for (int i = 0; i < 16; i++) from_f32(__uint_as_float(o[i]) * inv_sqrt_dk, st + (16 * cs + i) * 128 + dv_r);
        fence_async_smem();
    };

    // ---- prologue: fp16 S0; (c) of chunk 0 ----
    if (worker) put_state_a();
    if (warp == IW) {
        wait_par(bar_ld0, 0);
        tc_fence_after();
        issue_c(0, 0);
        issue_c(0, 1);
    }
    tc_fence_before();
    main_sync();
    if (*s_abort) goto abort_;

// Every main thread waits for the tensor-core commit itself (no CTA barrier: the
// barriers that follow each window order everything else).  A wait that gives up
// raises the abort flag, which the next barrier's check turns into a uniform exit.
#define GDN_MMA_WAIT()                                                                               \
    do {                                                                                             \
        if (!mbar_wait_bounded(bar, mphase)) atomicOr((unsigned*)s_abort, 1u);                      \
        mphase ^= 1u;                                                                                \
        tc_fence_after();                                                                            \
    } while (0)

    for (int ci = 0; ci < nchunks; ci++) {
        const int b = ci & 1;
        float dU[16];   // e^{g_C - g_c} for this worker's 16 chunk positions c = 16 cs + i

        // ---- MMA1: U2^T += S (-W)^T onto (c)'s result, O^T = S Q~^T; the first K step in halves,
        // so that the O half starts its accumulator, the rest at N = 128 ----
        if (warp == IW) {
            tc_fence_after();
            mma_f16_ta_w(tmem + acc_u(b), tmem + TA_S, dB1 + b * (R_STRIDE >> 4), ID_1H, 1);
            mma_f16_ta_w(tmem + acc_o(b), tmem + TA_S, dB1 + b * (R_STRIDE >> 4) + (8192 >> 4), ID_1H, 0);
#pragma unroll
            for (int ks = 1; ks < 8; ks++)
                mma_f16_ta_w(tmem + acc_u(b), tmem + TA_S + ks * 8,
                             dB1 + b * (R_STRIDE >> 4) + (ks >> 2) * 1024 + (ks & 3) * 2, ID_1, 1);
            mma_commit_w(bar);
            if (lane == 0) mbar_arrive(ev_iss);
            if (ci + 1 < nchunks) {   // (c) of the next chunk, pass 0, runs while U is converted
                wait_par(bar_ld0, ci + 1);
                tc_fence_after();
                issue_c(ci + 1, 0);
            }
        }
        // ---- workers, while MMA1 runs: the decayed state accumulator and the U^T decay factors ----
        if (worker) {
            wait_par(bar_ld0, ci);
            const float* gf = reinterpret_cast<const float*>(smem + OFF_R + b * R_STRIDE + R_G);
            const float decay = gf[C];
#pragma unroll
            for (int i4 = 0; i4 < 4; i4++) {
                const float4 f = *reinterpret_cast<const float4*>(gf + 16 * cs + 4 * i4);
                dU[4 * i4] = f.x; dU[4 * i4 + 1] = f.y; dU[4 * i4 + 2] = f.z; dU[4 * i4 + 3] = f.w;
            }
            if (!mbar_wait_bounded(ev_iss, 0)) atomicOr((unsigned*)s_abort, 1u);
            put_state_acc(decay);
            if (ci > 0) {   // O of the previous chunk is final once its MMA2b has completed
                wait_par(ev20, ci - 1);
                stage_o(ci - 1);
            }
        }
        GDN_MMA_WAIT();

        // ---- U^T and (D U)^T -> fp16 A operands; the issuer meanwhile waits for MMA2's operands ----
        if (warp == IW) {
            wait_par(bar_b20, ci);
            if (ci == nchunks - 1 && n_tail < C) {
                zero_tile_rows(sb + OFF_B2 + b * B2_STRIDE, 2, n_tail, lane, 32);
                fence_async_smem();
                __syncwarp();
            }
        }
        if (worker) {
            uint32_t r16[16], u[8], ud[8];
            tmem_ld16(tl + acc_u(b) + 16 * cs, r16);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float u0 = __uint_as_float(r16[2 * i]), u1 = __uint_as_float(r16[2 * i + 1]);
                u[i] = pack_half2(u0, u1);
                ud[i] = pack_half2(u0 * dU[2 * i], u1 * dU[2 * i + 1]);
            }
            tmem_st8x2(tl + TA_U + 8 * cs, u, tl + TA_UD + 8 * cs, ud);
        }
        tc_fence_before();
        main_sync();
        if (*s_abort) goto abort_;

        // ---- MMA2a: S += (D U)^T K; then MMA2b: O^T += U^T P^T, which runs while S is converted ----
        if (warp == IW) {
            if (lane == 0) {
                mbar_arrive(ev10 + 8 * b);                                // MMA1 and (c) are done with buffer b
                if (ci > 0) mbar_arrive(ev_st + 8 * ((ci - 1) & 1));      // o(ci - 1) is staged
            }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
                mma_f16_ta_w(tmem + ACC_S, tmem + TA_UD + ks * 8, dK + b * (B2_STRIDE >> 4) + ks * 128, ID_2A, 1);
            mma_commit_w(bar);
            if (lane == 0) mbar_arrive(ev_iss);
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
                mma_f16_ta_w(tmem + acc_o(b), tmem + TA_U + ks * 8, dP + b * (B2_STRIDE >> 4) + ks * 128, ID_2B, 1);
            mma_commit_w(ev20 + 8 * b);   // B2 buffer b is free once MMA2b has read P^T
            if (ci + 1 < nchunks) issue_c(ci + 1, 1);   // (c) of the next chunk, pass 1, while S is converted
        }
        GDN_MMA_WAIT();

        // ---- new state: its fp16 copy for the next MMA1, or the final state; the issuer
        // meanwhile makes sure the staging buffer for o(ci) is free ----
        if (warp == IW && !mbar_wait_bounded(evo, ci & 1)) atomicOr((unsigned*)s_abort, 2u);
        if (worker) {
            uint32_t r32[32];
            tmem_ld32(tl + ACC_S + 32 * cs, r32);
#pragma unroll
            for (int i = 0; i < 32; i++) Sv[i] = __uint_as_float(r32[i]);
            if (ci + 1 < nchunks) {
                put_state_a();
            } else {
#pragma unroll
                for (int i4 = 0; i4 < 8; i4++) {
                    const int col = 32 * cs + 4 * i4;
                    const float4 x = make_float4(Sv[4 * i4], Sv[4 * i4 + 1], Sv[4 * i4 + 2], Sv[4 * i4 + 3]);
                    if (dv_r < dv && col < dk) {
                        if (to_rec) st_state4(gstate + (int64_t)dv_r * dk + col, x);
                        else st_state4(cstate + (int64_t)dv_r * dk + col, x);
                    }
                }
            }
        }
        tc_fence_before();
        main_sync();
        if (*s_abort) goto abort_;
    }
    // the last o tile (its staging buffer was checked in the last chunk's state window)
    if (worker) {
        wait_par(ev20, nchunks - 1);
        stage_o(nchunks - 1);
    }
    tc_fence_before();
    main_sync();
    if (warp == IW && lane == 0) mbar_arrive(ev_end);   // the loader stores the last tile
    if (warp == 0) {
        mbar_wait_bounded(ev_ldone, 0);   // the loading warp's copies are done
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    return;

abort_:
    // A tensor-core commit or a copy never arrived: report it, give the MMAs still in
    // flight one more bounded wait, free tensor memory and return (the loading warp
    // sees the flag and drains its own copies).  The recurrent state is left as it was.
    if (warp == IW) {
        if (lane == 0)
            record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
        mma_commit_w(bar_fin);   // tracks every MMA the issuing lane has issued
        mbar_wait_bounded(bar_fin, 0);
    }
    tc_fence_before();
    main_sync();
    if (warp == 0) {
        mbar_wait_bounded(ev_ldone, 0);   // the loading warp sees the flag and drains its copies
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
#undef GDN_MMA_WAIT
}

}  // namespace scan
}  // namespace gdn
