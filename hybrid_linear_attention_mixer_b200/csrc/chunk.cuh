// Chunked gated-delta-rule prefill on the sm_100a tensor cores (tcgen05 + TMEM).
//
// One CTA walks one (sequence, value head) chain chunk by chunk (C = 64 tokens)
// and carries the d_v x d_k fp32 state in registers across chunks.  Inside a
// chunk with start state S0, gate prefix sums g_r = sum_{i<=r} log alpha_i and
// per-token updates u_r = beta_r (v_r - alpha_r S_{r-1} k_r), the recurrence
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
// re-associates exactly into (WY / UT form):
//     A_rj = beta_r e^{g_r - g_j} k_r.k_j (j < r),   T = (I + A)^-1 diag(beta)
//     W = T diag(e^g) K,   U = T V - W S0^T
//     O = (diag(e^g) Q S0^T + (Q K^T o M) U) / sqrt(d_k),  M_rj = e^{g_r - g_j}, j <= r
//     S_C = e^{g_C} S0 + U^T diag(e^{g_C - g}) K
// and the layer's output gated RMSNorm o * rsqrt(mean(o^2) + eps) * w * SiLU(z)
// runs in the epilogue.  Only exponentials of non-positive arguments are formed.
//
// Every dense product runs as tcgen05.mma (kind::f16: fp16 operands in shared
// memory, fp32 accumulators in tensor memory) with M = 128 = d_v or d_k, so the
// chunk dimension is always N:
//   (a) [Q;K] K^T        M=128 (q rows | k rows), N=64, K=d_k
//   (e) S Q^T            M=d_v, N=64, K=d_k          -> O1^T
//   (b) K^T T'^T         M=d_k, N=64, K=64           -> W^T  (T' = T diag(e^g))
//   (c) V^T T^T          M=d_v, N=64, K=64           -> U^T accumulator
//   (d) S (-W)^T         accumulated into (c)        -> U^T
//   (f) U^T P^T          M=d_v, N=64, K=64           -> O2^T  (P = Q K^T o M)
//   (g) U^T K~           M=d_v, N=d_k, K=64          -> state increment (K~ = diag(e^{g_C-g}) K)
// The triangular solve (I + A)^-1 runs in fp32 on the CUDA cores (16 x 16
// diagonal blocks by substitution, then block substitution).
//
// fp16 rather than bf16 operands: the state must match an fp64 reference to
// 1e-3 of its largest entry; bf16's 8-bit significand misses that by ~5x, fp16's
// 11 bits (the precision of tf32 at twice its rate) meets it.
#pragma once
#include "device.cuh"

namespace gdn {
namespace chunk {

constexpr int C = 64;          // chunk length
constexpr int D = 128;         // padded head dim (d_k, d_v <= 128)
constexpr int NT = 256;        // threads per CTA: 8 warps, two per TMEM lane quadrant

// Shared-memory map (bytes from a 1024-aligned base).  Tiles use 128-byte rows
// with the 128-byte swizzle; a 128-wide tile is two 64-wide halves.
constexpr uint32_t OFF_QK = 0;          // [Q;K]: 128 token rows x d_k, halves of 16384
constexpr uint32_t OFF_KT = 32768;      // K~: 64 token rows x d_k, halves of 8192
constexpr uint32_t OFF_V = 49152;       // V: 64 token rows x d_v, halves of 8192
constexpr uint32_t OFF_T = 65536;       // T: 64 x 64 (row c, col j)
constexpr uint32_t OFF_TP = 73728;      // T' = T diag(e^g)
constexpr uint32_t OFF_W = 81920;       // -W^T: 128 d_k rows x 64 chunk columns
constexpr uint32_t OFF_S16 = 98304;     // S (fp16 copy): 128 d_v rows x d_k, halves of 16384
constexpr uint32_t OFF_UT = 131072;     // U^T: 128 d_v rows x 64 chunk columns
constexpr uint32_t OFF_P = 147456;      // P: 64 x 64 (row r, col j)
constexpr uint32_t OFF_ZT = 155648;    // z (bf16): 64 token rows x d_v, halves of 8192; the
                                        // gated output is staged in place before its store
constexpr int LDA = 65;                 // fp32 64 x 64 work matrices, padded rows
constexpr uint32_t OFF_A = 172032;
constexpr uint32_t OFF_X = OFF_A + 64 * LDA * 4;
constexpr uint32_t OFF_Z = OFF_X + 64 * LDA * 4;
constexpr uint32_t OFF_G = OFF_Z + 64 * LDA * 4;   // g[64]
constexpr uint32_t OFF_B = OFF_G + 256;            // beta[64]
constexpr uint32_t OFF_RED = OFF_B + 256;          // [4][64] partial sums of o^2
constexpr uint32_t OFF_RS = OFF_RED + 1024;        // rsqrt(mean o^2 + eps) [64]
constexpr uint32_t OFF_BAR = OFF_RS + 256;         // mbarriers, TMEM address, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for the 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// Bytes one chunk's TMA loads deliver: q, k, v halves (6 boxes) and z halves (2 boxes)
constexpr uint32_t QKV_BYTES = 6 * 8192, Z_BYTES = 2 * 8192;

// Tensor-memory columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t ACC_QK = 0, ACC_W = 64, ACC_U = 128, ACC_O1 = 192, ACC_O2 = 256, ACC_SI = 320;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_KK_64 = idesc_f16(128, 64, 0, 0);
constexpr uint32_t ID_MK_64 = idesc_f16(128, 64, 1, 0);
constexpr uint32_t ID_KM_64 = idesc_f16(128, 64, 0, 1);
constexpr uint32_t ID_KM_128 = idesc_f16(128, 128, 0, 1);

// The q^, k^ (unit norm, fp16), v^ (fp16) and z (bf16) tiles arrive through 3-D
// TMA tensor maps over [T][H][d] with boxes of 64 (d) x 1 (head) x 64 (tokens)
// and the 128-byte swizzle; columns past d and rows past T read as zero.
struct Args {
    const void* a;           // [T][Hv] act dtype
    const void* b;           // [T][Hv]
    const void* z;           // [T][Hv][dv]
    const float* A_log;      // [Hv]
    const float* dt_bias;    // [Hv]
    const float* norm_w;     // [dv]
    float* rec_state;        // [N][Hv][dv][dk] in/out
    const int32_t* cu;       // [N+1]
    void* out;               // [T][Hv][dv] out dtype
    int Hk, Hv, dk, dv;
    float norm_eps;
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

// Scale 8 packed fp16 values by s (in fp32) and repack.
__device__ __forceinline__ uint4 scale8(uint4 v, float s) {
    float2 a = unpack_half2(v.x), b = unpack_half2(v.y), c = unpack_half2(v.z), d = unpack_half2(v.w);
    return make_uint4(pack_half2(a.x * s, a.y * s), pack_half2(b.x * s, b.y * s),
                      pack_half2(c.x * s, c.y * s), pack_half2(d.x * s, d.y * s));
}

template <typename TA, typename TO>
__global__ void __launch_bounds__(NT, 1)
gdn_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_z, Args p) {
    constexpr bool kZTile = sizeof(TA) == 2;                  // z through TMA (bf16 activations)
    constexpr bool kOutStage = kZTile && sizeof(TO) == 2;     // out staged in the z tile
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    float* s_g = reinterpret_cast<float*>(smem + OFF_G);
    float* s_b = reinterpret_cast<float*>(smem + OFF_B);
    float* s_red = reinterpret_cast<float*>(smem + OFF_RED);
    float* s_rs = reinterpret_cast<float*>(smem + OFF_RS);
    float* Am = reinterpret_cast<float*>(smem + OFF_A);
    float* Xm = reinterpret_cast<float*>(smem + OFF_X);
    float* Zm = reinterpret_cast<float*>(smem + OFF_Z);
    const uint32_t bar = sb + OFF_BAR;          // tensor-core commits
    const uint32_t bar_ld = sb + OFF_BAR + 24;  // q, k, v tiles of a chunk
    const uint32_t bar_z = sb + OFF_BAR + 32;   // z tile of a chunk
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 8);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3;       // TMEM lane quadrant of this warp
    const int half = warp >> 2;    // which half of the columns this warp handles
    const int Hv = p.Hv, Hk = p.Hk, dk = p.dk, dv = p.dv;
    const int seq = blockIdx.x / Hv, h = blockIdx.x % Hv;
    const int j = h / (Hv / Hk);
    const int64_t s0 = p.cu[seq], s1 = p.cu[seq + 1];
    const TA* __restrict__ pa = static_cast<const TA*>(p.a);
    const TA* __restrict__ pb = static_cast<const TA*>(p.b);
    const TA* __restrict__ pz = static_cast<const TA*>(p.z);
    TO* __restrict__ pout = static_cast<TO*>(p.out);
    const int nchunks = (int)((s1 - s0 + C - 1) / C);
    if (nchunks <= 0) return;

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_ld, 1);
        mbar_init(bar_z, 1);
        fence_mbar_init();
        *s_abort = 0;
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        if (kZTile) prefetch_tmap(&tm_z);
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_BAR + 8, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);   // this warp's lane quadrant
    uint32_t phase = 0;

    int ld_issued = 0, z_issued = 0;   // TMA loads issued (thread 0) ...
    int ld_ok = 0, z_ok = 0;           // ... and completed waits on them
    auto issue_qkv = [&](int64_t t) {   // one thread: the q, k, v tiles of the chunk at token t
        ld_issued++;
        mbar_arrive_expect_tx(bar_ld, QKV_BYTES);
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
            tma_load_3d(sb + OFF_QK + hf * 16384, &tm_q, 64 * hf, j, (int)t, bar_ld);
            tma_load_3d(sb + OFF_QK + hf * 16384 + C * 128, &tm_k, 64 * hf, j, (int)t, bar_ld);
            tma_load_3d(sb + OFF_V + hf * 8192, &tm_v, 64 * hf, h, (int)t, bar_ld);
        }
    };
    auto issue_z = [&](int64_t t) {
        z_issued++;
        mbar_arrive_expect_tx(bar_z, Z_BYTES);
#pragma unroll
        for (int hf = 0; hf < 2; hf++) tma_load_3d(sb + OFF_ZT + hf * 8192, &tm_z, 64 * hf, h, (int)t, bar_z);
    };
    if (tid == 0) {
        issue_qkv(s0);
        if (kZTile) issue_z(s0);
    }
    // gate inputs of the next chunk, loaded one chunk ahead (threads 0..63)
    float a_nx = 0.f, b_nx = 0.f;
    if (tid < C && s0 + tid < s1) {
        a_nx = to_f32(pa[(s0 + tid) * Hv + h]);
        b_nx = to_f32(pb[(s0 + tid) * Hv + h]);
    }

    // fp32 state: this thread owns row dv_r, columns [64*half, 64*half + 64)
    const int dv_r = 32 * qd + lane;
    float S[64];
    float* gstate = p.rec_state + ((int64_t)seq * Hv + h) * dv * dk;
#pragma unroll
    for (int i = 0; i < 64; i++) {
        const int col = 64 * half + i;
        S[i] = (dv_r < dv && col < dk) ? gstate[(int64_t)dv_r * dk + col] : 0.f;
    }

    const float expA = __expf(p.A_log[h]);
    const float dtb = p.dt_bias[h];
    const float inv_sqrt_dk = rsqrtf((float)dk);
    const float wn = dv_r < dv ? p.norm_w[dv_r] : 0.f;
    const int64_t ldv = (int64_t)Hv * dv;

#define GDN_MMA_WAIT()                                        \
    do {                                                      \
        if (!mbar_wait_bounded(bar, phase)) atomicOr((unsigned*)s_abort, 1u); \
        phase ^= 1;                                           \
        __syncthreads();                                      \
        if (*s_abort) goto abort_;                            \
        tc_fence_after();                                     \
    } while (0)

    for (int ci = 0; ci < nchunks; ci++) {
        // ---- S (fp16) operand tile for (d) and (e): row dv_r, this half of d_k ----
#pragma unroll
        for (int c8 = 0; c8 < 8; c8++) {
            sts128(sb + OFF_S16 + half * 16384 + swz128(dv_r, c8),
                   pack_half2(S[8 * c8 + 0], S[8 * c8 + 1]), pack_half2(S[8 * c8 + 2], S[8 * c8 + 3]),
                   pack_half2(S[8 * c8 + 4], S[8 * c8 + 5]), pack_half2(S[8 * c8 + 6], S[8 * c8 + 7]));
        }
        const int64_t t0 = s0 + (int64_t)ci * C;
        const int n = (int)((s1 - t0) < (int64_t)C ? (s1 - t0) : (int64_t)C);

        // ---- gates: log alpha, beta, and the in-chunk prefix sum g ----
        if (tid < C) {
            float la = 0.f, bt = 0.f;
            if (tid < n) {
                la = -expA * softplus_f(a_nx + dtb);
                bt = sigmoid_f(b_nx);
            }
            const int64_t tn = t0 + C + tid;   // prefetch the next chunk's a, b
            a_nx = b_nx = 0.f;
            if (tn < s1) {
                a_nx = to_f32(pa[tn * Hv + h]);
                b_nx = to_f32(pb[tn * Hv + h]);
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
        __syncthreads();
        if (tid >= 32 && tid < C) s_g[tid] += s_g[31];
        __syncthreads();
        const float g_last = s_g[C - 1];

        // ---- wait for this chunk's q, k, v tiles; K~ = diag(e^{g_C - g}) K from the k rows ----
        if (mbar_wait_bounded(bar_ld, ci & 1)) ld_ok++; else atomicOr((unsigned*)s_abort, 2u);
        for (int idx = tid; idx < C * 16; idx += NT) {
            const int r = idx >> 4, c16 = idx & 15;
            const int hf = c16 >> 3, cc = c16 & 7;
            const uint4 kv = lds128(sb + OFF_QK + hf * 16384 + swz128(C + r, cc));
            const uint4 kt = scale8(kv, r < n ? __expf(g_last - s_g[r]) : 0.f);
            sts128(sb + OFF_KT + hf * 8192 + swz128(r, cc), kt.x, kt.y, kt.z, kt.w);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*s_abort) goto abort_;

        // ---- (a) [Q;K] K^T and (e) S Q^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const uint32_t o = (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_f16(tmem + ACC_QK, sdesc(sb + OFF_QK + o, 16, 1024),
                        sdesc(sb + OFF_QK + o + C * 128, 16, 1024), ID_KK_64, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const uint32_t o = (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_f16(tmem + ACC_O1, sdesc(sb + OFF_S16 + o, 16, 1024), sdesc(sb + OFF_QK + o, 16, 1024),
                        ID_KK_64, ks > 0);
            }
            mma_commit(bar);
        }
        GDN_MMA_WAIT();

        // ---- P = Q K^T o M (fp16 tile) and A (fp32) ----
        {
            uint32_t r32[32];
            tmem_ld32(tl + ACC_QK + 32 * half, r32);
            const int j0 = 32 * half;
            if (qd < 2) {
                const int r = 32 * qd + lane;
                const float gr = s_g[r];
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const int jj = j0 + 2 * i;
                    const float e0 = __expf(fminf(gr - s_g[jj], 0.f));
                    const float e1 = __expf(fminf(gr - s_g[jj + 1], 0.f));
                    const float v0 = jj <= r ? __uint_as_float(r32[2 * i]) * e0 : 0.f;
                    const float v1 = jj + 1 <= r ? __uint_as_float(r32[2 * i + 1]) * e1 : 0.f;
                    pk[i] = pack_half2(v0, v1);
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; c4++)
                    sts128(sb + OFF_P + swz128(r, j0 / 8 + c4), pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2],
                           pk[4 * c4 + 3]);
            } else {
                const int r = 32 * (qd - 2) + lane;
                const float gr = s_g[r], br = s_b[r];
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int jj = j0 + i;
                    const float e = __expf(fminf(gr - s_g[jj], 0.f));
                    Am[r * LDA + jj] = jj < r ? br * __uint_as_float(r32[i]) * e : 0.f;
                }
            }
        }
        fence_async_smem();
        __syncthreads();

        // ---- X = (I + A)^-1, unit lower triangular, fp32 ----
        if (tid < 64) {   // diagonal 16 x 16 blocks: one column per thread
            const int base = 16 * (tid >> 4), c = tid & 15;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                float acc = (i == c) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < i; m++) acc = fmaf(-Am[(base + i) * LDA + base + m], x[m], acc);
                x[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < 16; i++) Xm[(base + i) * LDA + base + c] = x[i];
        }
        __syncthreads();
        {   // Z_{bi,m} = X_{bi,bi} A_{bi,m} for the six blocks below the diagonal
            const int i = tid >> 4, jj = tid & 15;
#pragma unroll
            for (int blk = 0; blk < 6; blk++) {
                const int bi = blk < 1 ? 1 : blk < 3 ? 2 : 3;
                const int m = blk < 1 ? 0 : blk < 3 ? blk - 1 : blk - 3;
                float acc = 0.f;
#pragma unroll
                for (int l = 0; l < 16; l++)
                    acc = fmaf(Xm[(16 * bi + i) * LDA + 16 * bi + l], Am[(16 * bi + l) * LDA + 16 * m + jj], acc);
                Zm[(16 * bi + i) * LDA + 16 * m + jj] = acc;
            }
        }
        __syncthreads();
#pragma unroll
        for (int dd = 1; dd < 4; dd++) {   // X_{bi,bj} = -sum_{m=bj}^{bi-1} Z_{bi,m} X_{m,bj}
            const int i = tid >> 4, jj = tid & 15;
            for (int bj = 0; bj + dd < 4; bj++) {
                const int bi = bj + dd;
                float acc = 0.f;
                for (int m = bj; m < bi; m++) {
#pragma unroll
                    for (int l = 0; l < 16; l++)
                        acc = fmaf(Zm[(16 * bi + i) * LDA + 16 * m + l], Xm[(16 * m + l) * LDA + 16 * bj + jj], acc);
                }
                Xm[(16 * bi + i) * LDA + 16 * bj + jj] = -acc;
            }
            __syncthreads();
        }
        {   // T = X diag(beta), T' = T diag(e^g): fp16 tiles, row c, 16 columns per thread
            const int c = tid >> 2, jq = (tid & 3) * 16;
            uint32_t tp[8], tq[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int jj = jq + 2 * i;
                const float x0 = jj <= c ? Xm[c * LDA + jj] * s_b[jj] : 0.f;
                const float x1 = jj + 1 <= c ? Xm[c * LDA + jj + 1] * s_b[jj + 1] : 0.f;
                tp[i] = pack_half2(x0, x1);
                tq[i] = pack_half2(x0 * __expf(s_g[jj]), x1 * __expf(s_g[jj + 1]));
            }
#pragma unroll
            for (int c2 = 0; c2 < 2; c2++) {
                sts128(sb + OFF_T + swz128(c, jq / 8 + c2), tp[4 * c2], tp[4 * c2 + 1], tp[4 * c2 + 2], tp[4 * c2 + 3]);
                sts128(sb + OFF_TP + swz128(c, jq / 8 + c2), tq[4 * c2], tq[4 * c2 + 1], tq[4 * c2 + 2], tq[4 * c2 + 3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- (b) W^T = K^T T'^T and (c) U^T = V^T T^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
                mma_f16(tmem + ACC_W, sdesc(sb + OFF_QK + C * 128 + ks * 2048, 16384, 1024),
                        sdesc(sb + OFF_TP + ks * 32, 16, 1024), ID_MK_64, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
                mma_f16(tmem + ACC_U, sdesc(sb + OFF_V + ks * 2048, 8192, 1024),
                        sdesc(sb + OFF_T + ks * 32, 16, 1024), ID_MK_64, ks > 0);
            mma_commit(bar);
        }
        GDN_MMA_WAIT();
        // (a), (b), (c), (e) are done with the q, k, v tiles: fetch the next chunk's
        if (tid == 0 && ci + 1 < nchunks) {
            fence_async_smem();
            issue_qkv(t0 + C);
        }

        // ---- -W^T -> fp16 tile (row d_k, chunk columns) ----
        {
            uint32_t r32[32];
            tmem_ld32(tl + ACC_W + 32 * half, r32);
            const int row = 32 * qd + lane;
#pragma unroll
            for (int c4 = 0; c4 < 4; c4++) {
                uint32_t w4[4];
#pragma unroll
                for (int i = 0; i < 4; i++)
                    w4[i] = pack_half2(-__uint_as_float(r32[8 * c4 + 2 * i]), -__uint_as_float(r32[8 * c4 + 2 * i + 1]));
                sts128(sb + OFF_W + swz128(row, 4 * half + c4), w4[0], w4[1], w4[2], w4[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- (d) U^T += S (-W)^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ks++)
                mma_f16(tmem + ACC_U, sdesc(sb + OFF_S16 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                        sdesc(sb + OFF_W + ks * 2048, 8192, 1024), ID_KM_64, 1);
            mma_commit(bar);
        }
        GDN_MMA_WAIT();

        // ---- U^T -> fp16 tile (row d_v, chunk columns) ----
        {
            uint32_t r32[32];
            tmem_ld32(tl + ACC_U + 32 * half, r32);
#pragma unroll
            for (int c4 = 0; c4 < 4; c4++) {
                uint32_t u4[4];
#pragma unroll
                for (int i = 0; i < 4; i++)
                    u4[i] = pack_half2(__uint_as_float(r32[8 * c4 + 2 * i]), __uint_as_float(r32[8 * c4 + 2 * i + 1]));
                sts128(sb + OFF_UT + swz128(dv_r, 4 * half + c4), u4[0], u4[1], u4[2], u4[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- (f) O2^T = U^T P^T and (g) state increment U^T K~ ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
                mma_f16(tmem + ACC_O2, sdesc(sb + OFF_UT + ks * 32, 16, 1024), sdesc(sb + OFF_P + ks * 32, 16, 1024),
                        ID_KK_64, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
                mma_f16(tmem + ACC_SI, sdesc(sb + OFF_UT + ks * 32, 16, 1024),
                        sdesc(sb + OFF_KT + ks * 2048, 8192, 1024), ID_KM_128, ks > 0);
            mma_commit(bar);
        }
        GDN_MMA_WAIT();

        // ---- state: S <- e^{g_C} S + U^T K~ ----
        {
            const float eg = __expf(g_last);
#pragma unroll
            for (int c2 = 0; c2 < 2; c2++) {
                uint32_t r32[32];
                tmem_ld32(tl + ACC_SI + 64 * half + 32 * c2, r32);
#pragma unroll
                for (int i = 0; i < 32; i++) S[32 * c2 + i] = fmaf(eg, S[32 * c2 + i], __uint_as_float(r32[i]));
            }
        }
        // ---- output: o = (e^{g_r} O1 + O2) / sqrt(d_k), then gated RMSNorm ----
        {
            uint32_t o1[32], o2[32];
            tmem_ld32(tl + ACC_O1 + 32 * half, o1);
            tmem_ld32(tl + ACC_O2 + 32 * half, o2);
            float o[32], v[32];
#pragma unroll
            for (int i = 0; i < 32; i++) {
                const int r = 32 * half + i;
                o[i] = (__expf(s_g[r]) * __uint_as_float(o1[i]) + __uint_as_float(o2[i])) * inv_sqrt_dk;
                v[i] = o[i] * o[i];
            }
            // transpose-reduce: lane L ends with the warp's sum for column 32*half + L
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const bool upper = (lane & off) != 0;
#pragma unroll
                for (int i = 0; i < off; i++) {
                    const float send = upper ? v[i] : v[i + off];
                    const float keep = upper ? v[i + off] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            s_red[qd * 64 + 32 * half + lane] = v[0];
            tc_fence_before();
            __syncthreads();
            if (tid < C) {
                const float ss = s_red[tid] + s_red[64 + tid] + s_red[128 + tid] + s_red[192 + tid];
                s_rs[tid] = rsqrtf(ss / (float)dv + p.norm_eps);
            }
            __syncthreads();
            if constexpr (kZTile) {
                if (mbar_wait_bounded(bar_z, ci & 1)) z_ok++; else atomicOr((unsigned*)s_abort, 2u);
                // z[r][dv_r] from the swizzled tile; the result overwrites it in place
                const uint32_t zcol = (uint32_t)(dv_r >> 6) * 8192 + (uint32_t)(dv_r & 7) * 2;
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int r = 32 * half + i;
                    __nv_bfloat16* zp = reinterpret_cast<__nv_bfloat16*>(smem + OFF_ZT + zcol +
                                                                         swz128(r, (dv_r & 63) >> 3));
                    const float y = o[i] * s_rs[r] * wn * silu_f(__bfloat162float(*zp));
                    if constexpr (kOutStage) {
                        *zp = __float2bfloat16_rn(y);
                    } else {
                        if (r < n && dv_r < dv) from_f32(y, pout + (t0 + r) * ldv + (int64_t)h * dv + dv_r);
                    }
                }
                if constexpr (kOutStage) {
                    __syncthreads();
                    for (int idx = tid; idx < C * 16; idx += NT) {   // 16-byte row pieces
                        const int r = idx >> 4, c16 = idx & 15;
                        if (r < n && c16 * 8 < dv) {
                            const uint4 v4 = lds128(sb + OFF_ZT + (c16 >> 3) * 8192 + swz128(r, c16 & 7));
                            __stcs(reinterpret_cast<uint4*>(pout + (t0 + r) * ldv + (int64_t)h * dv + c16 * 8), v4);
                        }
                    }
                }
                __syncthreads();
                if (*s_abort) goto abort_;
                if (tid == 0 && ci + 1 < nchunks) {   // the z tile is free: fetch the next chunk's
                    fence_async_smem();
                    issue_z(t0 + C);
                }
            } else if (dv_r < dv) {
                float zz[32];
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int r = 32 * half + i;
                    zz[i] = r < n ? to_f32(pz[(t0 + r) * ldv + (int64_t)h * dv + dv_r]) : 0.f;
                }
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int r = 32 * half + i;
                    if (r < n) from_f32(o[i] * s_rs[r] * wn * silu_f(zz[i]), pout + (t0 + r) * ldv + (int64_t)h * dv + dv_r);
                }
            }
        }
    }

    // ---- final state ----
#pragma unroll
    for (int i = 0; i < 64; i++) {
        const int col = 64 * half + i;
        if (dv_r < dv && col < dk) gstate[(int64_t)dv_r * dk + col] = S[i];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    return;

abort_:
    // A tensor-core commit or a TMA load never arrived: report it, give whatever
    // is still in flight one more bounded wait, release tensor memory and return.
    // The recurrent state is left as it was.
    if (tid == 0) {
        record_error((*s_abort & 1u ? kErrMmaTimeout : 0u) | (*s_abort & 2u ? kErrCopyTimeout : 0u));
        for (int k = ld_ok; k < ld_issued; k++) mbar_wait_bounded(bar_ld, k & 1);
        for (int k = z_ok; k < z_issued; k++) mbar_wait_bounded(bar_z, k & 1);
    }
    if (warp == 0) {
        mbar_wait_bounded(bar, phase ^ 1u);   // the tensor-core phase that did not complete, if any
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
#undef GDN_MMA_WAIT
}

}  // namespace chunk
}  // namespace gdn
