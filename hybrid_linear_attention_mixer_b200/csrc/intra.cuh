// Intra-chunk part of the chunked gated delta rule: everything inside a chunk
// that does not depend on the recurrent state, for every (chunk, value head)
// pair in parallel.
//
// For a chunk of C = 64 tokens of one sequence and one value head h (key head
// j = h / G), with g_r = sum_{i<=r} log alpha_i (the in-chunk gate prefix sum):
//     A_rj = beta_r e^{g_r - g_j} k_r.k_j   (j < r),   T = (I + A)^-1 diag(beta)
//     P_rj = q_r.k_j e^{g_r - g_j}          (j <= r)
//     W    = T diag(e^g) K
// These are the state-independent factors of the chunk's update (see scan.cuh
// for the state chain that consumes them).  The chunk's k rows are stacked on
// its q rows, so one tcgen05 MMA chain of the tile with itself gives K K^T and
// K Q^T = P^T (before masks) with the chunk position j on the TMEM lanes: P^T
// rows and A columns come straight out of TMEM.  W = T diag(e^g) K is a second
// MMA with the chunk position on the lanes again.  fp16 operands, fp32
// accumulators in TMEM; the triangular solve runs in fp32 on the CUDA cores.
// Warps with nothing to take out of TMEM scale Q and K into Q~ and K~ in place.
//
// Each (chunk, value head) record written to the workspace holds the operand
// tiles exactly as the scan kernel's tensor cores read them (128-byte swizzled
// shared-memory images), so the scan brings a record in with two bulk copies.
// Q~ = diag(e^g) Q and K~ = diag(e^{g_C - g}) K (zero past the sequence end).
// The order of the tiles inside the two images alternates with the parity p of
// the chunk within its sequence, to match the scan's alternating TMEM layout:
//     +0      B1 image, two 64-wide d_k halves of 16384 B, each [X rows | Y rows]
//             (64 rows each, K-major): X, Y = -W, Q~ (p = 0) or Q~, -W (p = 1)
//     +32768  T    K-major  [64 rows c][64 columns j]    fp16    8192 B
//     +40960  g    [64] fp32 (rows past the sequence end repeat the last g)
//     +41984  B2 image, three MN-major atoms of 8192 B:
//             [P^T | K~ half 0 | K~ half 1] (p = 0) or [K~ half 0 | K~ half 1 | P^T] (p = 1)
//             (P^T: row j holds P[0..63][j]; K~: row c holds 64 d_k values)
// Every tile is built in shared memory and written with a bulk copy.
#pragma once
#include "device.cuh"

namespace gdn {
namespace intra {

constexpr int C = 64;
constexpr int NT = 256;
constexpr uint32_t REC_B1 = 0, REC_T = 32768, REC_G = 40960, REC_B2 = 41984;
constexpr uint32_t REC_B1_BYTES = REC_G + 256 - REC_B1;   // B1, T and g: one copy
constexpr uint32_t REC_B2_BYTES = 24576;
constexpr uint32_t REC_BYTES = 66560;   // 65 x 1024: keeps every tile of a record 1024-aligned
__host__ __device__ constexpr uint32_t rec_w(int par, int hf) { return REC_B1 + hf * 16384 + (par ? 8192 : 0); }
__host__ __device__ constexpr uint32_t rec_q(int par, int hf) { return REC_B1 + hf * 16384 + (par ? 0 : 8192); }
__host__ __device__ constexpr uint32_t rec_p(int par) { return REC_B2 + (par ? 16384 : 0); }
__host__ __device__ constexpr uint32_t rec_kt(int par, int hf) { return REC_B2 + (par ? 0 : 8192) + hf * 8192; }

constexpr uint32_t OFF_QK = 0;          // [K;Q]: 128 token rows x d_k, halves of 16384 (k rows first)
constexpr int LDA = 68;                 // fp32 64 x 64 work matrices: 16-byte aligned rows
constexpr int LDY = 36;
constexpr uint32_t OFF_A = 32768;       // A; after the solve, T' = T diag(e^g) (fp16 tile)
constexpr uint32_t OFF_TP = OFF_A;
constexpr uint32_t OFF_X = OFF_A + 64 * LDA * 4;   // X = (I + A)^-1
constexpr uint32_t OFF_Y = OFF_X + 64 * LDA * 4;   // products of the doubling steps [32][LDY]
constexpr uint32_t OFF_G = OFF_Y + 32 * LDY * 4;   // g[64]
constexpr uint32_t OFF_B = OFF_G + 256;            // beta[64]
constexpr uint32_t OFF_EG = OFF_B + 256;           // e^g [64]
constexpr uint32_t OFF_BAR = OFF_EG + 256;         // mbarriers, TMEM address, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(3 * SMEM_BYTES <= 232448, "three CTAs per SM");
static_assert(OFF_A % 1024 == 0, "T' tile alignment");
constexpr uint32_t ACC_D = 0, TMEM_COLS = 128;   // [K K^T | K Q^T], later W

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

template <typename TA>
__global__ void __launch_bounds__(NT, 3)
gdn_intra_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, Args p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    float* s_g = reinterpret_cast<float*>(smem + OFF_G);
    float* s_b = reinterpret_cast<float*>(smem + OFF_B);
    float* Am = reinterpret_cast<float*>(smem + OFF_A);
    float* Xm = reinterpret_cast<float*>(smem + OFF_X);
    float* Ym = reinterpret_cast<float*>(smem + OFF_Y);
    float* s_eg = reinterpret_cast<float*>(smem + OFF_EG);
    const uint32_t bar = sb + OFF_BAR, bar_ld = sb + OFF_BAR + 8;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 16);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 20);
    // staging of the record tiles in regions that are free by then
    const uint32_t st_p = sb + OFF_X;                   // P^T: X (written only from the solve on)
    const uint32_t st_t = sb + OFF_QK + 16384 + 8192;   // T: q rows of half 1 (Q~ is stored by then)
    const uint32_t st_w = sb + OFF_X;                   // -W: X (dead once T is formed), 16 KiB

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, half = warp >> 2;
    const int Hv = p.Hv;
    const int h = blockIdx.x % Hv;
    const int gc = blockIdx.x / Hv;
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
    const int j = h / (Hv / p.Hk);
    const int par = (gc - p.chunk_off[seq]) & 1;   // parity of the chunk within its sequence
    uint8_t* rec = p.rec + ((int64_t)gc * Hv + h) * REC_BYTES;

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_ld, 1);
        fence_mbar_init();
        *s_abort = 0;
        mbar_arrive_expect_tx(bar_ld, 4 * 8192);
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
            tma_load_3d(sb + OFF_QK + hf * 16384, &tm_k, 64 * hf, j, (int)t0, bar_ld);
            tma_load_3d(sb + OFF_QK + hf * 16384 + C * 128, &tm_q, 64 * hf, j, (int)t0, bar_ld);
        }
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_BAR + 16, TMEM_COLS);
        tmem_relinquish();
    }
    // gates: log alpha, beta and the in-chunk prefix sum g
    if (tid < C) {
        float la = 0.f, bt = 0.f;
        if (tid < n) {
            const float av = to_f32(static_cast<const TA*>(p.a)[(t0 + tid) * Hv + h]);
            const float bv = to_f32(static_cast<const TA*>(p.b)[(t0 + tid) * Hv + h]);
            la = -__expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]);
            bt = sigmoid_f(bv);
        }
        float g = la;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, g, off);
            if (lane >= off) g += o;
        }
        s_g[tid] = g;
        s_b[tid] = bt;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid >= 32 && tid < C) s_g[tid] += s_g[31];

    const uint32_t tmem = *s_tmem;
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    if (!mbar_wait_bounded(bar_ld, 0)) atomicOr((unsigned*)s_abort, 2u);
    __syncthreads();
    bool ok = *s_abort == 0;

    // ---- [K;Q] [K;Q]^T: lanes 0-63 hold row j of [K K^T | K Q^T] ----
    if (ok && tid == 0) {
        tc_fence_after();
        constexpr uint32_t ID = idesc_f16(128, 128, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ks++) {
            const uint64_t d = sdesc(sb + OFF_QK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
            mma_f16(tmem + ACC_D, d, d, ID, ks > 0);
        }
        mma_commit(bar);
    }
    if (tid < C) {
        reinterpret_cast<float*>(rec + REC_G)[tid] = s_g[tid];
        s_eg[tid] = __expf(s_g[tid]);
    }
    if (ok && !mbar_wait_bounded(bar, 0)) atomicOr((unsigned*)s_abort, 1u);
    __syncthreads();
    ok = *s_abort == 0;
    if (ok && qd < 2) {
        tc_fence_after();
        const int jr = 32 * qd + lane;     // chunk position j of this lane
        const float gj = s_g[jr];
        uint32_t r32[32];
        if (half == 0) {
            // column j of A: A[r][j] = beta_r e^{g_r - g_j} k_r.k_j for r > j
#pragma unroll
            for (int c2 = 0; c2 < 2; c2++) {
                tmem_ld32(tl + ACC_D + 32 * c2, r32);
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int r = 32 * c2 + i;
                    const float e = __expf(fminf(s_g[r] - gj, 0.f));
                    Am[r * LDA + jr] = r > jr ? s_b[r] * __uint_as_float(r32[i]) * e : 0.f;
                }
            }
        } else {
            // row j of P^T: P[r][j] = e^{g_r - g_j} q_r.k_j for r >= j -> fp16, MN-major image
#pragma unroll
            for (int c2 = 0; c2 < 2; c2++) {
                tmem_ld32(tl + ACC_D + 64 + 32 * c2, r32);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const int r = 32 * c2 + 2 * i;
                    const float e0 = __expf(fminf(s_g[r] - gj, 0.f)), e1 = __expf(fminf(s_g[r + 1] - gj, 0.f));
                    w[i] = pack_half2(r >= jr ? __uint_as_float(r32[2 * i]) * e0 : 0.f,
                                      r + 1 >= jr ? __uint_as_float(r32[2 * i + 1]) * e1 : 0.f);
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++)
                    sts128(st_p + swz128(jr, 4 * c2 + q4), w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
            }
            fence_async_smem();
        }
    } else if (ok) {   // Q~ = diag(e^g) Q in place (the q rows are dead after the first MMA); Q~ feeds
                       // only the output, so packed half2 products are precise enough
        const int t = tid - 64 * (tid >= 128 ? 1 : 0) - 64;   // 0..127 over warps 2, 3, 6, 7
        for (int idx = t; idx < 2 * C * 8; idx += 128) {
            const int hf = idx >> 9, r = (idx >> 3) & 63, ch = idx & 7;
            const uint32_t a = sb + OFF_QK + hf * 16384 + 8192 + swz128(r, ch);
            const uint4 x = scale8_h2(lds128(a), s_eg[r]);
            sts128(a, x.x, x.y, x.z, x.w);
        }
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (ok && tid == 0) {
        bulk_s2g(rec + rec_p(par), st_p, 8192);
        bulk_s2g(rec + rec_q(par, 0), sb + OFF_QK + 8192, 8192);
        bulk_s2g(rec + rec_q(par, 1), sb + OFF_QK + 16384 + 8192, 8192);
        bulk_commit();
        bulk_wait_read<0>();   // the solve writes X, where P^T was staged
    }
    __syncthreads();

    // ---- X = (I + A)^-1, unit lower triangular, fp32 ----
    // 16 x 16 diagonal blocks by substitution, then two doubling steps: for
    // diagonal blocks [[L1, 0], [A21, L2]] the inverse is [[X1, 0], [-X2 A21 X1, X2]].
    if (ok && tid < 64) {   // one column of one diagonal block per thread
        const int base = 16 * (tid >> 4), c = tid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            float acc = (i == c) ? 1.f : 0.f;
            const float* arow = Am + (base + i) * LDA + base;
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
#pragma unroll
        for (int i = 0; i < 16; i++) Xm[(base + i) * LDA + base + c] = x[i];
    }
    __syncthreads();
    if (ok && tid < 128) {   // size 16 -> 32: Y = A21 X1 for the block pairs (0,1) and (2,3)
        const int o1 = tid < 64 ? 0 : 32, o2 = o1 + 16;
        block_mm<false, true>(Am + o2 * LDA + o1, LDA, Xm + o1 * LDA + o1, LDA, Ym + (o1 >> 1), LDY, 16, 1.f,
                              tid & 63, 64);
    }
    __syncthreads();
    if (ok && tid < 128) {   // X21 = -X2 Y
        const int o1 = tid < 64 ? 0 : 32, o2 = o1 + 16;
        block_mm<true, false>(Xm + o2 * LDA + o2, LDA, Ym + (o1 >> 1), LDY, Xm + o2 * LDA + o1, LDA, 16, -1.f,
                              tid & 63, 64);
    }
    __syncthreads();
    if (ok) block_mm<false, true>(Am + 32 * LDA, LDA, Xm, LDA, Ym, LDY, 32, 1.f, tid, NT);   // size 32 -> 64
    __syncthreads();
    if (ok) block_mm<true, false>(Xm + 32 * LDA + 32, LDA, Ym, LDY, Xm + 32 * LDA, LDA, 32, -1.f, tid, NT);
    __syncthreads();
    if (ok) {   // T = X diag(beta) -> staged for the record; T' = T diag(e^g) -> the W MMA's operand
        const int c = tid >> 2, jq = (tid & 3) * 16;
        uint32_t tp[8], tq[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int jj = jq + 2 * i;
            const float x0 = jj <= c ? Xm[c * LDA + jj] * s_b[jj] : 0.f;
            const float x1 = jj + 1 <= c ? Xm[c * LDA + jj + 1] * s_b[jj + 1] : 0.f;
            tp[i] = pack_half2(x0, x1);
            tq[i] = pack_half2(x0 * s_eg[jj], x1 * s_eg[jj + 1]);
        }
#pragma unroll
        for (int c2 = 0; c2 < 2; c2++) {
            sts128(st_t + swz128(c, jq / 8 + c2), tp[4 * c2], tp[4 * c2 + 1], tp[4 * c2 + 2], tp[4 * c2 + 3]);
            sts128(sb + OFF_TP + swz128(c, jq / 8 + c2), tq[4 * c2], tq[4 * c2 + 1], tq[4 * c2 + 2], tq[4 * c2 + 3]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- W = T' K (M = 128 with the chunk's 64 rows first, N = d_k, K = 64 tokens) ----
    if (ok && tid == 0) {
        bulk_s2g(rec + REC_T, st_t, 8192);
        bulk_commit();
        tc_fence_after();
        constexpr uint32_t ID = idesc_f16(128, 128, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ks++)
            mma_f16(tmem + ACC_D, sdesc(sb + OFF_TP + ks * 32, 16, 1024), sdesc(sb + OFF_QK + ks * 2048, 16384, 1024),
                    ID, ks > 0);
        mma_commit(bar);
    }
    if (ok && !mbar_wait_bounded(bar, 1)) atomicOr((unsigned*)s_abort, 1u);
    __syncthreads();
    ok = *s_abort == 0;
    if (ok && qd < 2) {   // row c of -W, one 64-wide d_k half per warp half -> K-major image
        tc_fence_after();
        const int c = 32 * qd + lane;
        uint32_t r32[32];
#pragma unroll
        for (int c2 = 0; c2 < 2; c2++) {
            tmem_ld32(tl + ACC_D + 64 * half + 32 * c2, r32);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; i++)
                w[i] = pack_half2(-__uint_as_float(r32[2 * i]), -__uint_as_float(r32[2 * i + 1]));
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++)
                sts128(st_w + half * 8192 + swz128(c, 4 * c2 + q4), w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2],
                       w[4 * q4 + 3]);
        }
        fence_async_smem();
    } else if (ok) {   // K~ = diag(e^{g_C - g}) K in place (the W MMA is done with K); zero past the end
        const int t = tid - 64 * (tid >= 128 ? 1 : 0) - 64;
        const float gC = s_g[C - 1];
        for (int idx = t; idx < 2 * C * 8; idx += 128) {
            const int hf = idx >> 9, r = (idx >> 3) & 63, ch = idx & 7;
            const uint32_t a = sb + OFF_QK + hf * 16384 + swz128(r, ch);
            const uint4 x = scale8(lds128(a), r < n ? __expf(gC - s_g[r]) : 0.f);   // fp32: K~ feeds the state
            sts128(a, x.x, x.y, x.z, x.w);
        }
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        if (ok) {
            bulk_s2g(rec + rec_w(par, 0), st_w, 8192);
            bulk_s2g(rec + rec_w(par, 1), st_w + 8192, 8192);
            bulk_s2g(rec + rec_kt(par, 0), sb + OFF_QK, 8192);
            bulk_s2g(rec + rec_kt(par, 1), sb + OFF_QK + 16384, 8192);
            bulk_commit();
        } else {
            record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
            // one more bounded wait for whatever may still be in flight
            mbar_wait_bounded(bar_ld, 0);
            mbar_wait_bounded(bar, 0);
            mbar_wait_bounded(bar, 1);
        }
        bulk_wait<0>();   // the record's bulk stores have read their staging
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace intra
}  // namespace gdn
