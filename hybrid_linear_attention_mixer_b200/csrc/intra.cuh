// Intra-chunk part of the chunked gated delta rule: everything inside a chunk
// that does not depend on the recurrent state, for every (chunk, key head) pair
// in parallel.
//
// For a chunk of C = 64 tokens of one sequence and one value head h (key head
// j = h / G), with g_r = sum_{i<=r} log alpha_i (the in-chunk gate prefix sum):
//     A_rj = beta_r e^{g_r - g_j} k_r.k_j   (j < r),   T = (I + A)^-1 diag(beta)
//     P_rj = q_r.k_j e^{g_r - g_j}          (j <= r)
//     W    = T diag(e^g) K
// These are the state-independent factors of the chunk's update (scan.cuh runs
// the state chain that consumes them).
//
// One CTA takes one (chunk, key head) and the value heads that read that key
// head, up to three at a time, one 4-warp group each.  The products K K^T and
// K Q^T depend on the key head only, so they are computed once: the chunk's k
// rows are stacked on its q rows and one tcgen05 MMA chain of the tile with
// itself puts row j of [K K^T | K Q^T] on TMEM lane j.  Each group turns it
// into column j of its head's A (gated, masked, beta-scaled, fp32, in shared
// memory) and row j of its head's P^T, inverts I + A in place in fp32 on the
// CUDA cores (16 x 16 diagonal blocks by substitution, then two doubling
// steps), and forms T and T' = T diag(e^g).  The T' tiles of two heads are
// stacked into one M = 128 operand, so W = T' K for three heads takes two MMA
// chains.  Two CTAs fit on an SM.
//
// The record of each (chunk, value head) holds the scan's operands, the tiles
// in the exact 128-byte-swizzled shared-memory images its tensor cores read,
// written straight from registers:
//     +0      B1   per 64-wide d_k half (16384 B): [-W rows | Q~ rows], K-major,
//                  64 + 64 rows c; Q~ = diag(e^g) Q                      fp16  32768 B
//     +32768  T    K-major [64 rows c][64 columns j], as fp16(T), then  fp16  2 x 8192 B
//                  fp16(T - fp16(T)): the pair carries T to about 22 bits
//     +49152  decay factors: e^{g_C - g_c} for c < 64, then e^{g_C}     fp32  (65 used of 1024 B)
//     +50176  P^T  MN-major atom: row j holds P[0..63][j]               fp16  8192 B
// (g rows past the sequence end repeat the last g, so their factors are 1.)
// The scan applies e^{g_C - g} to U rather than to K, so K needs no copy here.
#pragma once
#include "device.cuh"

namespace gdn {
namespace intra {

constexpr int C = kChunk;
constexpr int GH = 3;                      // value heads per round: one 4-warp group each
constexpr int NT = 128 * GH;
constexpr uint32_t REC_B1 = 0, REC_T = 32768, REC_G = 49152, REC_P = 50176;
constexpr uint32_t REC_BYTES = 58368;      // 57 x 1024: every tile of a record stays 1024-aligned
constexpr uint32_t REC_LD_BYTES = REC_G + 512 - REC_B1;   // B1, T and the decay factors: one copy

constexpr uint32_t OFF_QK = 0;             // [K;Q]: 128 token rows x d_k, halves of 16384 (k rows first)
constexpr int LDA = 68;                    // fp32 64 x 64 work matrix rows (16-byte aligned)
constexpr int LDY = 36;
constexpr uint32_t AX_BYTES = 64 * LDA * 4;          // 17408 = 17 x 1024
constexpr uint32_t OFF_AX = 32768;                   // [GH] A, inverted in place into X; then T' tiles
constexpr uint32_t Y_BYTES = 32 * LDY * 4;           // products of the doubling steps
constexpr uint32_t OFF_Y = OFF_AX + GH * AX_BYTES;   // [GH]
constexpr uint32_t OFF_GATE = OFF_Y + GH * Y_BYTES;  // g [GH][64], beta [GH][64], e^g [GH][64]
constexpr uint32_t OFF_BAR = OFF_GATE + 3 * GH * 256;
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
static_assert(OFF_AX % 1024 == 0 && AX_BYTES % 1024 == 0, "T' operand tiles are 1024-aligned");
// TMEM: [K K^T | K Q^T] in columns 0..127 (lanes 0..63); then W of the head pair
// (slots 0, 1) in columns 128..255 and W of slot 2 in 0..127
constexpr uint32_t TMEM_COLS = 256;

struct Args {
    const void* a;            // [T][Hv] act dtype
    const void* b;            // [T][Hv]
    const float* A_log;       // [Hv]
    const float* dt_bias;     // [Hv]
    const int32_t* cu;        // [N+1]
    const int32_t* chunk_off; // [N+1] first chunk of each sequence; chunk_off[N] = total
    const int32_t* flags;     // nonzero: a device check failed, write nothing
    int n_seqs;
    int Hk, Hv;
    uint8_t* rec;             // [total chunks][Hv][REC_BYTES]
    int32_t g_lo;             // CTA x takes global chunk g_lo + x / Hk
};

__device__ __forceinline__ void stg128(void* p, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    *reinterpret_cast<uint4*>(p) = make_uint4(x, y, z, w);
}

// chunk_off[s] = sum_{i<s} ceil(len_i / C) (one CTA, any number of sequences),
// and the check of cu_seqlens that the host cannot make (it is device memory):
// cu[0] = 0, non-decreasing, cu[N] = T_total, at most max_chunks chunks.  A
// malformed cu sets bit 0 of *flags (every later kernel of the call then writes
// nothing), zeroes the chunk table and records kErrSeqlens.  *flags is written
// here on every call; the conv kernel may OR bit 1 into it afterwards.
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int32_t* cu, int n_seqs, int64_t T_total,
                                                             int64_t max_chunks, int32_t* chunk_off,
                                                             int32_t* flags) {
    __shared__ int32_t s_sum[32];
    __shared__ long long s_carry;
    if (threadIdx.x == 0) s_carry = 0;
    int bad = threadIdx.x == 0 && (cu[0] != 0 || (int64_t)cu[n_seqs] != T_total);
    __syncthreads();
    for (int base = 0; base < n_seqs; base += 1024) {
        const int s = base + threadIdx.x;
        int32_t v = 0;
        if (s < n_seqs) {
            const int64_t len = (int64_t)cu[s + 1] - cu[s];   // 64-bit: any int32 pair subtracts safely
            bad |= len < 0;
            v = len > 0 ? (int32_t)((len + C - 1) / C) : 0;
        }
        int32_t x = v;   // inclusive scan within the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
            if ((threadIdx.x & 31) >= off) x += y;
        }
        if ((threadIdx.x & 31) == 31) s_sum[threadIdx.x >> 5] = x;
        __syncthreads();
        if (threadIdx.x < 32) {
            int32_t w = s_sum[threadIdx.x];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, w, off);
                if (threadIdx.x >= off) w += y;
            }
            s_sum[threadIdx.x] = w;   // inclusive warp totals
        }
        __syncthreads();
        const int32_t warp_base = (threadIdx.x >> 5) ? s_sum[(threadIdx.x >> 5) - 1] : 0;
        if (s < n_seqs) chunk_off[s] = (int32_t)(s_carry + warp_base + x - v);
        __syncthreads();
        if (threadIdx.x == 1023) s_carry += warp_base + x;
        __syncthreads();
    }
    bad |= s_carry > max_chunks;
    if (__syncthreads_or(bad)) {
        for (int s = threadIdx.x; s <= n_seqs; s += 1024) chunk_off[s] = 0;
        if (threadIdx.x == 0) {
            *flags = 1;
            record_error(kErrSeqlens);
        }
    } else if (threadIdx.x == 0) {
        chunk_off[n_seqs] = (int32_t)s_carry;
        *flags = 0;
    }
}

// C = sgn * L R for n x n blocks (n = 16 or 32; rows 16-byte aligned), 1 x 4
// register tiles: thread t of nt takes tiles t, t + nt, ...  LTRI_L / LTRI_R: L or
// R is lower triangular, so the products it zeroes are skipped.
template <bool LTRI_L, bool LTRI_R>
__device__ __forceinline__ void block_mm(const float* L, int ldl, const float* R, int ldr, float* Cm, int ldc,
                                         int n, float sgn, int t, int nt) {
    const int tpr = n >> 2;
    for (int tile = t; tile < n * tpr; tile += nt) {
        const int i = tile / tpr, j0 = (tile % tpr) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const int l_begin = LTRI_R ? j0 : 0;                 // R[l][j] = 0 for l < j
        const int l_end = LTRI_L ? ((i >> 2) + 1) * 4 : n;   // L[i][l] = 0 for l > i
        for (int l0 = l_begin; l0 < l_end; l0 += 4) {
            const float4 a = *reinterpret_cast<const float4*>(L + i * ldl + l0);
            const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const float4 r = *reinterpret_cast<const float4*>(R + (l0 + u) * ldr + j0);
                acc.x = fmaf(av[u], r.x, acc.x);
                acc.y = fmaf(av[u], r.y, acc.y);
                acc.z = fmaf(av[u], r.z, acc.z);
                acc.w = fmaf(av[u], r.w, acc.w);
            }
        }
        *reinterpret_cast<float4*>(Cm + i * ldc + j0) = make_float4(sgn * acc.x, sgn * acc.y, sgn * acc.z, sgn * acc.w);
    }
}


// Address of row 0 of value-head slot s among the T' operand tiles: slots 0 and
// 1 stack into the 128-row tile at OFF_AX, slot 2 takes rows 0..63 of the tile
// at OFF_AX + AX_BYTES (whose rows 64..127 feed only TMEM lanes never read).
__host__ __device__ constexpr uint32_t tp_tile(int s) {
    return OFF_AX + (s == 2 ? AX_BYTES : 0u) + (s == 1 ? 8192u : 0u);
}

template <typename TA>
__global__ void __launch_bounds__(NT, 2)
gdn_intra_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, Args p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = warp >> 2, qd = warp & 3, tg = tid & 127;   // value-head slot, TMEM lane quadrant
    const int Hk = p.Hk, Hv = p.Hv, G = Hv / Hk;
    const int kh = blockIdx.x % Hk;
    const int gc = p.g_lo + (int)(blockIdx.x / Hk);
    if (gc >= p.chunk_off[p.n_seqs] || *p.flags) return;
    int lo = 0, hi = p.n_seqs - 1;   // sequence of this chunk: last s with chunk_off[s] <= gc
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.chunk_off[mid] <= gc) lo = mid; else hi = mid - 1;
    }
    const int seq = lo;
    const int64_t t0 = (int64_t)p.cu[seq] + (int64_t)(gc - p.chunk_off[seq]) * C;
    const int64_t rem = (int64_t)p.cu[seq + 1] - t0;
    const int n = (int)(rem < C ? rem : C);

    float* AX = reinterpret_cast<float*>(smem + OFF_AX + grp * AX_BYTES);
    float* Ym = reinterpret_cast<float*>(smem + OFF_Y + grp * Y_BYTES);
    float* s_g = reinterpret_cast<float*>(smem + OFF_GATE) + grp * 64;
    float* s_b = s_g + GH * 64;
    float* s_eg = s_b + GH * 64;
    const uint32_t bar_ld = sb + OFF_BAR, bar_mma = sb + OFF_BAR + 8;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 16);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 20);
    // the 128 threads of this thread's value-head group
    auto gsync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory"); };

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *s_abort = 0;
        mbar_arrive_expect_tx(bar_ld, 4 * 8192);
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
            tma_load_3d(sb + OFF_QK + hf * 16384, &tm_k, 64 * hf, kh, (int)t0, bar_ld);
            tma_load_3d(sb + OFF_QK + hf * 16384 + C * 128, &tm_q, 64 * hf, kh, (int)t0, bar_ld);
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
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    uint32_t mphase = 0;   // bar_mma: one phase per commit
    bool ok = true;

    for (int h0 = 0; h0 < G && ok; h0 += GH) {
        const int nh = G - h0 < GH ? G - h0 : GH;   // value heads of this round
        const bool act = grp < nh;
        const int h = kh * G + h0 + grp;
        uint8_t* rec = p.rec + ((int64_t)gc * Hv + h) * REC_BYTES;

        // ---- gates: log alpha, beta and the in-chunk prefix sum g ----
        if (act && tg < C) {
            float la = 0.f, bt = 0.f;
            if (tg < n) {
                const float av = to_f32(static_cast<const TA*>(p.a)[(t0 + tg) * Hv + h]);
                const float bv = to_f32(static_cast<const TA*>(p.b)[(t0 + tg) * Hv + h]);
                la = -__expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]);
                bt = sigmoid_f(bv);
            }
            float g = la;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, g, off);
                if (lane >= off) g += o;
            }
            s_g[tg] = g;
            s_b[tg] = bt;
        }
        // ---- [K;Q] [K;Q]^T: lane j holds row j of [K K^T | K Q^T] (lanes 0..63) ----
        if (warp == 0) {
            if (h0 == 0) {
                if (!mbar_wait_bounded(bar_ld, 0)) atomicOr((unsigned*)s_abort, 2u);
                // rows past the sequence's end hold another sequence's tokens, or rows a later
                // launch has yet to write: zeros, so that only finite values meet the zero gates
                if (n < C) {
                    zero_tile_rows(sb + OFF_QK, 4, n, lane, 32);
                    fence_async_smem();
                }
                __syncwarp();
            }
            if (lane == 0 && *s_abort == 0) {
                tc_fence_after();
                constexpr uint32_t ID = idesc_f16(128, 128, 0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ks++) {
                    const uint64_t d = sdesc(sb + OFF_QK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    mma_f16(tmem, d, d, ID, ks > 0);
                }
                mma_commit(bar_mma);
            }
        }
        __syncthreads();
        if (act && tg >= 32 && tg < C) s_g[tg] += s_g[31];   // carry of the first 32 tokens
        if (*s_abort == 0 && !mbar_wait_bounded(bar_mma, mphase)) atomicOr((unsigned*)s_abort, 1u);
        mphase ^= 1u;
        __syncthreads();
        ok = *s_abort == 0;
        if (!ok) break;
        if (h0 == 0 && !mbar_wait_bounded(bar_ld, 0)) atomicOr((unsigned*)s_abort, 2u);   // (the q rows, below)
        if (act && tg < C) {
            const float g = s_g[tg], gC = s_g[C - 1];
            s_eg[tg] = __expf(g);
            reinterpret_cast<float*>(rec + REC_G)[tg] = __expf(gC - g);
            if (tg == 0) reinterpret_cast<float*>(rec + REC_G)[C] = __expf(gC);
        }
        if (act) {   // Q~ = diag(e^g) Q rows into the B1 image (packed half2 products: Q~ feeds only the output)
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int idx = tg + 128 * j, hf = idx >> 9, r = (idx >> 3) & 63, ch = idx & 7;
                const uint32_t off = hf * 16384 + 8192 + swz128(r, ch);
                const uint4 x = scale8_h2(lds128(sb + OFF_QK + off), __expf(s_g[r]));
                stg128(rec + REC_B1 + off, x.x, x.y, x.z, x.w);
            }
        }
        // ---- column j of A into shared memory, row j of P^T into the record ----
        if (act && qd < 2) {
            tc_fence_after();
            const int jr = 32 * qd + lane;   // chunk position j of this lane
            const float gj = s_g[jr];
#pragma unroll
            for (int c4 = 0; c4 < 4; c4++) {
                uint32_t kk[16], kq[16], w[8];
                tmem_ld16(tl + 16 * c4, kk);
                tmem_ld16(tl + 64 + 16 * c4, kq);
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int r0 = 16 * c4 + 2 * i, r1 = r0 + 1;
                    const float e0 = __expf(fminf(s_g[r0] - gj, 0.f)), e1 = __expf(fminf(s_g[r1] - gj, 0.f));
                    AX[r0 * LDA + jr] = r0 > jr ? s_b[r0] * __uint_as_float(kk[2 * i]) * e0 : 0.f;
                    AX[r1 * LDA + jr] = r1 > jr ? s_b[r1] * __uint_as_float(kk[2 * i + 1]) * e1 : 0.f;
                    w[i] = pack_half2(r0 >= jr ? __uint_as_float(kq[2 * i]) * e0 : 0.f,
                                      r1 >= jr ? __uint_as_float(kq[2 * i + 1]) * e1 : 0.f);
                }
#pragma unroll
                for (int q = 0; q < 2; q++)
                    stg128(rec + REC_P + swz128(jr, 2 * c4 + q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            }
        }

        // ---- X = (I + A)^-1 in place: unit lower triangular, fp32 ----
        // 16 x 16 diagonal blocks by substitution, then two doubling steps: for
        // diagonal blocks [[L1, 0], [A21, L2]] the inverse is [[X1, 0], [-X2 A21 X1, X2]].
        if (act) {
            gsync();
            float x[16];
            const int base = 16 * (tg >> 4), cc = tg & 15;
            if (tg < 64) {   // one column of one diagonal block per thread
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    float acc = (i == cc) ? 1.f : 0.f;
                    const float* arow = AX + (base + i) * LDA + base;
#pragma unroll
                    for (int m4 = 0; m4 < 16; m4 += 4) {
                        if (m4 < i) {
                            const float4 a = *reinterpret_cast<const float4*>(arow + m4);
                            if (m4 + 0 < i) acc = fmaf(-a.x, x[m4 + 0], acc);
                            if (m4 + 1 < i) acc = fmaf(-a.y, x[m4 + 1], acc);
                            if (m4 + 2 < i) acc = fmaf(-a.z, x[m4 + 2], acc);
                            if (m4 + 3 < i) acc = fmaf(-a.w, x[m4 + 3], acc);
                        }
                    }
                    x[i] = acc;
                }
            }
            gsync();   // every block has been read before any is overwritten
            if (tg < 64) {
#pragma unroll
                for (int i = 0; i < 16; i++) AX[(base + i) * LDA + base + cc] = x[i];
            }
            gsync();
            {   // size 16 -> 32 for the block pairs (0,1) and (2,3): Y = A21 X1, then X21 = -X2 Y over A21
                const int o1 = tg < 64 ? 0 : 32, o2 = o1 + 16;
                block_mm<false, true>(AX + o2 * LDA + o1, LDA, AX + o1 * LDA + o1, LDA, Ym + (o1 >> 1), LDY, 16, 1.f,
                                      tg & 63, 64);
                gsync();
                block_mm<true, false>(AX + o2 * LDA + o2, LDA, Ym + (o1 >> 1), LDY, AX + o2 * LDA + o1, LDA, 16, -1.f,
                                      tg & 63, 64);
            }
            gsync();   // size 32 -> 64
            block_mm<false, true>(AX + 32 * LDA, LDA, AX, LDA, Ym, LDY, 32, 1.f, tg, 128);
            gsync();
            block_mm<true, false>(AX + 32 * LDA + 32, LDA, Ym, LDY, AX + 32 * LDA, LDA, 32, -1.f, tg, 128);
            gsync();
        }
        // ---- T = X diag(beta) into the record; T' = T diag(e^g) for the W MMA ----
        uint32_t tq[16];
        const int c = tg >> 1, jq = (tg & 1) * 32;   // row c, columns jq .. jq + 31
        if (act) {
            uint32_t tp[16], tl[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const int jj = jq + 2 * i;
                const float x0 = jj <= c ? AX[c * LDA + jj] * s_b[jj] : 0.f;
                const float x1 = jj + 1 <= c ? AX[c * LDA + jj + 1] * s_b[jj + 1] : 0.f;
                tp[i] = pack_half2(x0, x1);
                const float2 hi = unpack_half2(tp[i]);
                tl[i] = pack_half2(x0 - hi.x, x1 - hi.y);   // (exact differences)
                tq[i] = pack_half2(x0 * s_eg[jj], x1 * s_eg[jj + 1]);
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) {
                const uint32_t o = swz128(c, jq / 8 + q4);
                stg128(rec + REC_T + o, tp[4 * q4], tp[4 * q4 + 1], tp[4 * q4 + 2], tp[4 * q4 + 3]);
                stg128(rec + REC_T + 8192 + o, tl[4 * q4], tl[4 * q4 + 1], tl[4 * q4 + 2], tl[4 * q4 + 3]);
            }
        }
        __syncthreads();   // every group is done with its X: the T' tiles overwrite the work matrices
        if (act) {
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++)
                sts128(sb + tp_tile(grp) + swz128(c, jq / 8 + q4), tq[4 * q4], tq[4 * q4 + 1], tq[4 * q4 + 2],
                       tq[4 * q4 + 3]);
            fence_async_smem();
        }
        tc_fence_before();
        __syncthreads();

        // ---- W = T' K: slots 0 and 1 in one M = 128 chain (columns 128..255), slot 2 in another (0..127) ----
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t ID = idesc_f16(128, 128, 0, 1);
            for (int pr = 0; pr < (nh > 2 ? 2 : 1); pr++) {
#pragma unroll
                for (int ks = 0; ks < 4; ks++)
                    mma_f16(tmem + (pr ? 0u : 128u), sdesc(sb + OFF_AX + pr * AX_BYTES + ks * 32, 16, 1024),
                            sdesc(sb + OFF_QK + ks * 2048, 16384, 1024), ID, ks > 0);
            }
            mma_commit(bar_mma);
        }
        if (!mbar_wait_bounded(bar_mma, mphase)) atomicOr((unsigned*)s_abort, 1u);
        mphase ^= 1u;
        __syncthreads();
        ok = *s_abort == 0;
        if (!ok) break;
        {   // rows of -W into the records: 32-column slices spread over the three warps of each quadrant
            tc_fence_after();
            const int n_units = qd < 2 ? (nh > 2 ? 8 : 4) : (nh > 1 ? 4 : 0);
            const int cr = 32 * (qd & 1) + lane;   // this lane's row (chunk position) in its head's W
            for (int u = grp; u < n_units; u += GH) {
                const int slot = qd < 2 ? (u < 4 ? 0 : 2) : 1, sl = u & 3;
                uint8_t* rw = p.rec + ((int64_t)gc * Hv + kh * G + h0 + slot) * REC_BYTES + REC_B1 + (sl >> 1) * 16384;
                uint32_t r32[32];
                tmem_ld32(tl + (slot == 2 ? 0u : 128u) + 32 * sl, r32);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; i++)
                    w[i] = pack_half2(-__uint_as_float(r32[2 * i]), -__uint_as_float(r32[2 * i + 1]));
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++)
                    stg128(rw + swz128(cr, 4 * (sl & 1) + q4), w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
            }
        }
        tc_fence_before();
        __syncthreads();   // the next round's product overwrites columns 0..127
    }
    if (!ok && tid == 0) {
        // a copy or a tensor-core commit never arrived: report it, and give whatever may
        // still be in flight one more bounded wait
        record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
        mbar_wait_bounded(bar_ld, 0);
        mbar_wait_bounded(bar_mma, mphase);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace intra
}  // namespace gdn
