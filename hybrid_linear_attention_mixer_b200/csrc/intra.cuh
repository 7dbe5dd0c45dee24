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
// for the state chain that consumes them).  [Q;K] K^T and K^T (T diag(e^g))^T
// run as tcgen05 MMAs (fp16 operands, fp32 accumulators in TMEM); the
// triangular solve runs in fp32 on the CUDA cores.
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

constexpr uint32_t OFF_QK = 0;          // [Q;K]: 128 token rows x d_k, halves of 16384
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
constexpr uint32_t ACC_QK = 0, ACC_W = 64, TMEM_COLS = 128;

struct Args {
    const void* a;            // [T][Hv] act dtype
    const void* b;            // [T][Hv]
    const float* A_log;       // [Hv]
    const float* dt_bias;     // [Hv]
    const int32_t* cu;        // [N+1]
    const int32_t* chunk_off; // [N+1] first chunk of each sequence; chunk_off[N] = total
    int n_seqs;
    int Hk, Hv;
    uint8_t* rec;             // [total chunks][Hv][REC_BYTES]
};

__device__ __forceinline__ void stg128(void* p, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    *reinterpret_cast<uint4*>(p) = make_uint4(x, y, z, w);
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}

// chunk_off[s] = sum_{i<s} ceil(len_i / C) (one CTA, any number of sequences)
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int32_t* cu, int n_seqs, int32_t* chunk_off) {
    __shared__ int32_t s_sum[32];
    __shared__ int32_t s_carry;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base < n_seqs; base += 1024) {
        const int s = base + threadIdx.x;
        int32_t v = 0;
        if (s < n_seqs) v = (cu[s + 1] - cu[s] + C - 1) / C;
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
        if (s < n_seqs) chunk_off[s] = s_carry + warp_base + x - v;
        __syncthreads();
        if (threadIdx.x == 1023) s_carry += warp_base + x;
        __syncthreads();
    }
    if (threadIdx.x == 0) chunk_off[n_seqs] = s_carry;
}

// C = sgn * L R for n x n blocks (n = 16 or 32; rows 16-byte aligned), 1 x 4
// register tiles: thread t of nt takes tiles t, t + nt, ...
__device__ __forceinline__ void block_mm(const float* L, int ldl, const float* R, int ldr, float* Cm, int ldc,
                                         int n, float sgn, int t, int nt) {
    const int tpr = n >> 2;
    for (int tile = t; tile < n * tpr; tile += nt) {
        const int i = tile / tpr, j0 = (tile % tpr) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int l0 = 0; l0 < n; l0 += 4) {
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

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, half = warp >> 2;
    const int Hv = p.Hv;
    const int h = blockIdx.x % Hv;
    const int gc = blockIdx.x / Hv;
    if (gc >= p.chunk_off[p.n_seqs]) return;
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
            tma_load_3d(sb + OFF_QK + hf * 16384, &tm_q, 64 * hf, j, (int)t0, bar_ld);
            tma_load_3d(sb + OFF_QK + hf * 16384 + C * 128, &tm_k, 64 * hf, j, (int)t0, bar_ld);
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

    // ---- [Q;K] K^T ----
    if (ok && tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ks++) {
            const uint32_t o = (ks >> 2) * 16384 + (ks & 3) * 32;
            mma_f16(tmem + ACC_QK, sdesc(sb + OFF_QK + o, 16, 1024), sdesc(sb + OFF_QK + o + C * 128, 16, 1024),
                    idesc_f16(128, 64, 0, 0), ks > 0);
        }
        mma_commit(bar);
    }
    if (tid < C) {
        reinterpret_cast<float*>(rec + REC_G)[tid] = s_g[tid];
        s_eg[tid] = __expf(s_g[tid]);
    }
    __syncthreads();   // e^g
    if (ok) {   // Q~ and K~ -> the record (same swizzled rows as the Q and K tiles here)
        const float gC = s_g[C - 1];
        for (int idx = tid; idx < 2 * C * 16; idx += NT) {
            const int kk = idx >= C * 16, r = (idx >> 4) & (C - 1), c16 = idx & 15, hf = c16 >> 3;
            const uint32_t sw = swz128(r, c16 & 7);
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(sb + OFF_QK + hf * 16384 + kk * (C * 128) + sw));
            const float e = kk ? (r < n ? __expf(gC - s_g[r]) : 0.f) : s_eg[r];
            const float2 a0 = unpack_half2(v.x), a1 = unpack_half2(v.y), a2 = unpack_half2(v.z), a3 = unpack_half2(v.w);
            stg128(rec + (kk ? rec_kt(par, hf) : rec_q(par, hf)) + sw, pack_half2(a0.x * e, a0.y * e),
                   pack_half2(a1.x * e, a1.y * e), pack_half2(a2.x * e, a2.y * e), pack_half2(a3.x * e, a3.y * e));
        }
    }
    if (ok && !mbar_wait_bounded(bar, 0)) atomicOr((unsigned*)s_abort, 1u);
    __syncthreads();
    ok = *s_abort == 0;
    if (ok) {
        tc_fence_after();
        uint32_t r32[32];
        tmem_ld32(tl + ACC_QK + 32 * half, r32);
        const int j0 = 32 * half;
        if (qd < 2) {   // P rows -> fp16 rows [r][j] in shared memory (the X region, 132-byte rows)
            const int r = 32 * qd + lane;
            const float gr = s_g[r];
            uint32_t* pr = reinterpret_cast<uint32_t*>(Xm) + r * 33 + j0 / 2;
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const int jj = j0 + 2 * i;
                const float e0 = __expf(fminf(gr - s_g[jj], 0.f));
                const float e1 = __expf(fminf(gr - s_g[jj + 1], 0.f));
                pr[i] = pack_half2(jj <= r ? __uint_as_float(r32[2 * i]) * e0 : 0.f,
                                   jj + 1 <= r ? __uint_as_float(r32[2 * i + 1]) * e1 : 0.f);
            }
        } else {        // A rows -> shared memory
            const int r = 32 * (qd - 2) + lane;
            const float gr = s_g[r], br = s_b[r];
#pragma unroll
            for (int i4 = 0; i4 < 8; i4++) {
                float a4[4];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int jj = j0 + 4 * i4 + u;
                    const float e = __expf(fminf(gr - s_g[jj], 0.f));
                    a4[u] = jj < r ? br * __uint_as_float(r32[4 * i4 + u]) * e : 0.f;
                }
                *reinterpret_cast<float4*>(Am + r * LDA + j0 + 4 * i4) = make_float4(a4[0], a4[1], a4[2], a4[3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    if (ok) {   // P^T -> the record (MN-major B image: row j holds P[0..63][j])
        const __half* pr = reinterpret_cast<const __half*>(Xm);
        for (int idx = tid; idx < C * 8; idx += NT) {
            const int jj = idx >> 3, q8 = idx & 7;
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const __half lo = pr[(8 * q8 + 2 * i) * 66 + jj], hi = pr[(8 * q8 + 2 * i + 1) * 66 + jj];
                w4[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
            }
            stg128(rec + rec_p(par) + swz128(jj, q8), w4[0], w4[1], w4[2], w4[3]);
        }
    }
    __syncthreads();
    for (int i = tid; i < 64 * LDA / 4; i += NT)   // X starts as zero above its diagonal blocks
        reinterpret_cast<float4*>(Xm)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
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
        block_mm(Am + o2 * LDA + o1, LDA, Xm + o1 * LDA + o1, LDA, Ym + (o1 >> 1), LDY, 16, 1.f, tid & 63, 64);
    }
    __syncthreads();
    if (ok && tid < 128) {   // X21 = -X2 Y
        const int o1 = tid < 64 ? 0 : 32, o2 = o1 + 16;
        block_mm(Xm + o2 * LDA + o2, LDA, Ym + (o1 >> 1), LDY, Xm + o2 * LDA + o1, LDA, 16, -1.f, tid & 63, 64);
    }
    __syncthreads();
    if (ok) block_mm(Am + 32 * LDA, LDA, Xm, LDA, Ym, LDY, 32, 1.f, tid, NT);   // size 32 -> 64
    __syncthreads();
    if (ok) block_mm(Xm + 32 * LDA + 32, LDA, Ym, LDY, Xm + 32 * LDA, LDA, 32, -1.f, tid, NT);
    __syncthreads();
    if (ok) {   // T = X diag(beta) -> the record; T' = T diag(e^g) -> shared memory
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
            stg128(rec + REC_T + swz128(c, jq / 8 + c2), tp[4 * c2], tp[4 * c2 + 1], tp[4 * c2 + 2], tp[4 * c2 + 3]);
            sts128(sb + OFF_TP + swz128(c, jq / 8 + c2), tq[4 * c2], tq[4 * c2 + 1], tq[4 * c2 + 2], tq[4 * c2 + 3]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- W^T = K^T T'^T (M = d_k, N = 64 chunk columns, K = 64 tokens) ----
    if (ok && tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ks++)
            mma_f16(tmem + ACC_W, sdesc(sb + OFF_QK + C * 128 + ks * 2048, 16384, 1024),
                    sdesc(sb + OFF_TP + ks * 32, 16, 1024), idesc_f16(128, 64, 1, 0), ks > 0);
        mma_commit(bar);
    }
    if (ok && !mbar_wait_bounded(bar, 1)) atomicOr((unsigned*)s_abort, 1u);
    __syncthreads();
    ok = *s_abort == 0;
    if (ok) {   // -W^T from TMEM -> fp16 rows [d_k][c] in shared memory (reusing A)
        tc_fence_after();
        uint32_t r32[32];
        tmem_ld32(tl + ACC_W + 32 * half, r32);
        const int row = 32 * qd + lane;
        uint32_t* wt = reinterpret_cast<uint32_t*>(smem + OFF_A) + row * 33 + 16 * half;   // 132-byte rows
#pragma unroll
        for (int i = 0; i < 16; i++)
            wt[i] = pack_half2(-__uint_as_float(r32[2 * i]), -__uint_as_float(r32[2 * i + 1]));
    }
    __syncthreads();
    if (ok) {   // -> the record, K-major: 16-byte piece (c, d_k 8q..8q+7) gathers 8 rows of -W^T
        const __half* wt = reinterpret_cast<const __half*>(smem + OFF_A);
        for (int idx = tid; idx < C * 16; idx += NT) {
            const int c = idx >> 4, q8 = idx & 15;
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const __half lo = wt[(8 * q8 + 2 * i) * 66 + c], hi = wt[(8 * q8 + 2 * i + 1) * 66 + c];
                w4[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
            }
            stg128(rec + rec_w(par, q8 >> 3) + swz128(c, q8 & 7), w4[0], w4[1], w4[2], w4[3]);
        }
    } else if (tid == 0) {
        record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
        // one more bounded wait for whatever may still be in flight
        mbar_wait_bounded(bar_ld, 0);
        mbar_wait_bounded(bar, 0);
        mbar_wait_bounded(bar, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace intra
}  // namespace gdn
