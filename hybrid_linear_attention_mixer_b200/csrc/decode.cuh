// Fused one-token decode step of the Gated DeltaNet mixer.
//
// One CTA per (sequence, key head): it rolls the conv state of the key head's
// q/k channels and of its G value heads' v channels, runs conv + SiLU, the L2
// norm of q and k, the gates, and then streams the G value-head states
// (G x d_v rows of d_k fp32, one contiguous block) through registers once.
// Row r of S gives row r of S' and o_r with no other row involved:
//     u_r   = S_r . k,   p_r = S_r . q
//     d_r   = beta (v_r - alpha u_r)
//     S'_r  = alpha S_r + d_r k^T
//     o_r   = (alpha p_r + d_r (k . q)) / sqrt(d_k)         (= S'_r . q / sqrt(d_k))
// which is S' = alpha S (I - beta k k^T) + beta v k^T applied row by row.  The
// gated RMSNorm over the d_v entries of o follows.  HBM-bound: 2 x 64 KiB of
// state per value head per step against ~1 KiB of everything else.
#pragma once
#include "device.cuh"

namespace gdn {
namespace dec {

constexpr int NT = 256;
constexpr int NW = NT / 32;

// 4 consecutive state entries: fp32 as is, or bf16 storage (read exactly, written
// round-to-nearest-even); all arithmetic is fp32.  Streaming (evict-first) accesses.
template <typename TS> struct State4;
template <> struct State4<float> {
    static __device__ __forceinline__ float4 ld(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
    static __device__ __forceinline__ void st(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
};
template <> struct State4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 ld(const __nv_bfloat16* p) {
        const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
    }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float4 v) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&b);
        __stcs(reinterpret_cast<uint2*>(p), u);
    }
};

struct Args {
    const void *q, *k, *v, *a, *b, *z;   // act dtype; q,k [N][Hk*dk], v,z [N][Hv*dv], a,b [N][Hv]
    const float* conv_w;                 // [Ctot][4]
    const float* A_log;
    const float* dt_bias;
    const float* norm_w;
    void* conv_state;                    // [N][Ctot][3] act dtype, in/out
    void* rec_state;                     // [N][Hv][dv][dk] state dtype (fp32 or bf16), in/out
    void* out;                           // [N][Hv][dv] out dtype
    int Hk, Hv, dk, dv;
    float l2_eps, norm_eps;
};

__host__ __device__ constexpr size_t smem_floats(int dk, int G, int dv) {
    return (size_t)2 * dk + (size_t)2 * G * dv + 2 * G;
}

template <typename TA, typename TO, typename TS, int DK>
__global__ void __launch_bounds__(NT) gdn_decode_kernel(Args p) {
    constexpr int LPR = DK / 4;        // lanes per state row (4 fp32 each)
    constexpr int RPP = 32 / LPR;      // rows per warp pass
    constexpr int U = DK == 128 ? 8 : 4;   // passes in flight per warp
    extern __shared__ float sm[];
    const int Hk = p.Hk, Hv = p.Hv, dv = p.dv, G = Hv / Hk;
    const int Cq = Hk * DK, Cv = Hv * dv, Ctot = 2 * Cq + Cv;
    const int seq = blockIdx.x / Hk, j = blockIdx.x % Hk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* sq = sm;                 // [DK]
    float* sk = sq + DK;            // [DK]
    float* sv = sk + DK;            // [G*dv]
    float* so = sv + G * dv;        // [G*dv]
    float* s_al = so + G * dv;      // [G]
    float* s_be = s_al + G;         // [G]

    // ---- conv + SiLU with the conv-state roll (channels of this key-head group) ----
    const TA* pq = static_cast<const TA*>(p.q);
    const TA* pk = static_cast<const TA*>(p.k);
    const TA* pv = static_cast<const TA*>(p.v);
    TA* cst = static_cast<TA*>(p.conv_state);
    const int nch = 2 * DK + G * dv;
    for (int i = tid; i < nch; i += NT) {
        int ch;
        const TA* src;
        if (i < DK) {
            ch = j * DK + i;
            src = pq + (int64_t)seq * Cq + ch;
        } else if (i < 2 * DK) {
            ch = Cq + j * DK + (i - DK);
            src = pk + (int64_t)seq * Cq + (ch - Cq);
        } else {
            const int vi = j * G * dv + (i - 2 * DK);
            ch = 2 * Cq + vi;
            src = pv + (int64_t)seq * Cv + vi;
        }
        TA* st = cst + ((int64_t)seq * Ctot + ch) * 3;
        const TA xr = *src, h0 = st[0], h1 = st[1], h2 = st[2];
        const float4 w = reinterpret_cast<const float4*>(p.conv_w)[ch];
        float acc = w.x * to_f32(h0);
        acc = fmaf(w.y, to_f32(h1), acc);
        acc = fmaf(w.z, to_f32(h2), acc);
        acc = fmaf(w.w, to_f32(xr), acc);
        sm[i] = silu_f(acc);
        st[0] = h1;
        st[1] = h2;
        st[2] = xr;
    }
    if (tid < G) {
        const int h = j * G + tid;
        const float av = to_f32(static_cast<const TA*>(p.a)[(int64_t)seq * Hv + h]);
        const float bv = to_f32(static_cast<const TA*>(p.b)[(int64_t)seq * Hv + h]);
        s_al[tid] = __expf(-__expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]));
        s_be[tid] = sigmoid_f(bv);
    }
    __syncthreads();
    if (warp < 2) {   // L2 norm: warp 0 -> q, warp 1 -> k
        float* x = warp == 0 ? sq : sk;
        float ss = 0.f;
        for (int i = lane; i < DK; i += 32) ss = fmaf(x[i], x[i], ss);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float r = rsqrtf(ss + p.l2_eps);
        for (int i = lane; i < DK; i += 32) x[i] *= r;
    }
    __syncthreads();

    // ---- stream the state rows ----
    const int col = 4 * (lane % LPR);
    const int sub = lane / LPR;
    const float4 k4 = *reinterpret_cast<const float4*>(sk + col);
    const float4 q4 = *reinterpret_cast<const float4*>(sq + col);
    float kq = k4.x * q4.x + k4.y * q4.y + k4.z * q4.z + k4.w * q4.w;
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    const float inv_sqrt_dk = rsqrtf((float)DK);
    TS* Sb = static_cast<TS*>(p.rec_state) + ((int64_t)seq * Hv + (int64_t)j * G) * dv * DK;
    const int rows = G * dv;
    for (int R0 = warp * RPP * U; R0 < rows; R0 += NW * RPP * U) {
        float4 s[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int R = R0 + u * RPP + sub;
            s[u] = R < rows ? State4<TS>::ld(Sb + (int64_t)R * DK + col)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int R = R0 + u * RPP + sub;
            const int g = min(R, rows - 1) / dv;
            float uk = s[u].x * k4.x + s[u].y * k4.y + s[u].z * k4.z + s[u].w * k4.w;
            float up = s[u].x * q4.x + s[u].y * q4.y + s[u].z * q4.z + s[u].w * q4.w;
#pragma unroll
            for (int off = LPR / 2; off >= 1; off >>= 1) {
                uk += __shfl_xor_sync(0xffffffffu, uk, off);
                up += __shfl_xor_sync(0xffffffffu, up, off);
            }
            if (R < rows) {
                const float al = s_al[g], be = s_be[g];
                const float d = be * (sv[R] - al * uk);
                float4 o4;
                o4.x = fmaf(al, s[u].x, d * k4.x);
                o4.y = fmaf(al, s[u].y, d * k4.y);
                o4.z = fmaf(al, s[u].z, d * k4.z);
                o4.w = fmaf(al, s[u].w, d * k4.w);
                State4<TS>::st(Sb + (int64_t)R * DK + col, o4);
                if (lane % LPR == 0) so[R] = (al * up + d * kq) * inv_sqrt_dk;
            }
        }
    }
    __syncthreads();

    // ---- gated RMSNorm per value head ----
    const TA* pz = static_cast<const TA*>(p.z);
    TO* po = static_cast<TO*>(p.out);
    for (int g = warp; g < G; g += NW) {
        float ss = 0.f;
        for (int r = lane; r < dv; r += 32) ss = fmaf(so[g * dv + r], so[g * dv + r], ss);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float rs = rsqrtf(ss / (float)dv + p.norm_eps);
        const int h = j * G + g;
        for (int r = lane; r < dv; r += 32) {
            const int64_t off = ((int64_t)seq * Hv + h) * dv + r;
            const float zz = to_f32(pz[off]);
            from_f32(so[g * dv + r] * rs * p.norm_w[r] * silu_f(zz), po + off);
        }
    }
}

// Multi-token rows: a state row (d_k fp32) is spread over 8 lanes; lane l of the row
// holds the float4s at columns 4l + 32i, i < d_k/32, so each 16-byte access of the
// row's 8 lanes is one contiguous 128-byte piece, and a row's dot products take
// 3 butterfly steps instead of 5.  Dot products add in one fixed order (explicit fmaf,
// then the butterfly over the 8 lanes).
constexpr int MLPR = 8;     // lanes per state row
constexpr int MRPP = 32 / MLPR;
template <int NF4>
__device__ __forceinline__ float row_dot(const float4 (&s)[NF4], const float4 (&v)[NF4]) {
    float x = 0.f;
#pragma unroll
    for (int i = 0; i < NF4; i++) {
        x = fmaf(s[i].x, v[i].x, x);
        x = fmaf(s[i].y, v[i].y, x);
        x = fmaf(s[i].z, v[i].z, x);
        x = fmaf(s[i].w, v[i].w, x);
    }
#pragma unroll
    for (int off = MLPR / 2; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}
template <int NF4>
__device__ __forceinline__ void row_load(const float* base, int lane8, float4 (&v)[NF4]) {
#pragma unroll
    for (int i = 0; i < NF4; i++) v[i] = *reinterpret_cast<const float4*>(base + 4 * lane8 + 32 * i);
}
// S_r <- alpha S_r + d k
template <int NF4>
__device__ __forceinline__ void row_update(float4 (&s)[NF4], const float4 (&k)[NF4], float al, float d) {
#pragma unroll
    for (int i = 0; i < NF4; i++) {
        s[i].x = fmaf(al, s[i].x, d * k[i].x);
        s[i].y = fmaf(al, s[i].y, d * k[i].y);
        s[i].z = fmaf(al, s[i].z, d * k[i].z);
        s[i].w = fmaf(al, s[i].w, d * k[i].w);
    }
}

// ---------------------------------------------------------------------------
// Multi-token decode (draft verification): n_tok consecutive tokens of each
// sequence in one pass over its state.  Multi-token prediction drafts several
// future tokens ("Qwen3.8-Flash-Next", "Architecture concepts": Multi-Token
// Prediction; table "Every architecture field", row mtp_layers); checking a
// draft runs the recurrence over the drafted tokens.  Row r of S takes the
// n_tok updates one after another, as n_tok decode steps would (equal to them up
// to the order of fp32 additions inside a row's dot products), while the state is
// read and written once.
// Optionally the state after every token is written out (snapshots), so that
// a caller who accepts only the first j drafted tokens can restore the state
// after token j; the conv state after every token can be written out likewise.
// Inputs and outputs are token-major within each sequence: row seq*n_tok + t.
// ---------------------------------------------------------------------------
constexpr int kMaxTok = 16;

struct MultiArgs {
    Args a;
    int n_tok;
    void* state_snap;    // [n_tok][N][Hv][dv][dk] state dtype, or null
    void* conv_snap;     // [n_tok][N][Ctot][3] act dtype, or null
    int n_seqs;
    int stages;          // streamed kernel: slabs in flight (2 .. stream_stages<TS>())
};

__host__ __device__ constexpr size_t smem_floats_multi(int dk, int G, int dv, int n_tok) {
    return (size_t)n_tok * (2 * dk + 2 * G * dv + 2 * G + 1);
}

template <typename TA, typename TO, typename TS, int DK>
__global__ void __launch_bounds__(NT, 2) gdn_decode_multi_kernel(MultiArgs m) {
    const Args& p = m.a;
    const int NTK = m.n_tok;
    extern __shared__ float sm[];
    const int Hk = p.Hk, Hv = p.Hv, dv = p.dv, G = Hv / Hk;
    const int Cq = Hk * DK, Cv = Hv * dv, Ctot = 2 * Cq + Cv;
    const int seq = blockIdx.x / Hk, j = blockIdx.x % Hk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nch = 2 * DK + G * dv;   // this CTA's channels: q, k of key head j, v of its value heads
    float* sfeat = sm;                      // [NTK][nch]: q^ | k^ | v^ per token
    float* so = sfeat + NTK * nch;          // [NTK][G*dv]
    float* s_al = so + NTK * G * dv;        // [NTK][G]
    float* s_be = s_al + NTK * G;           // [NTK][G]
    float* s_kq = s_be + NTK * G;           // [NTK] k_t . q_t

    // ---- conv + SiLU of every token, with the conv-state roll ----
    const TA* pq = static_cast<const TA*>(p.q);
    const TA* pk = static_cast<const TA*>(p.k);
    const TA* pv = static_cast<const TA*>(p.v);
    TA* cst = static_cast<TA*>(p.conv_state);
    for (int i = tid; i < nch; i += NT) {
        int ch;
        const TA* src;
        int64_t ld;
        if (i < DK) {
            ch = j * DK + i;
            src = pq + ch;
            ld = Cq;
        } else if (i < 2 * DK) {
            ch = Cq + j * DK + (i - DK);
            src = pk + (ch - Cq);
            ld = Cq;
        } else {
            const int vi = j * G * dv + (i - 2 * DK);
            ch = 2 * Cq + vi;
            src = pv + vi;
            ld = Cv;
        }
        TA* st = cst + ((int64_t)seq * Ctot + ch) * 3;
        TA h0 = st[0], h1 = st[1], h2 = st[2];
        const float4 w = reinterpret_cast<const float4*>(p.conv_w)[ch];
        for (int t = 0; t < NTK; t++) {
            const TA xr = src[((int64_t)seq * NTK + t) * ld];
            float acc = w.x * to_f32(h0);
            acc = fmaf(w.y, to_f32(h1), acc);
            acc = fmaf(w.z, to_f32(h2), acc);
            acc = fmaf(w.w, to_f32(xr), acc);
            sfeat[t * nch + i] = silu_f(acc);
            h0 = h1;
            h1 = h2;
            h2 = xr;
            if (m.conv_snap) {
                TA* cs = static_cast<TA*>(m.conv_snap) + (((int64_t)t * m.n_seqs + seq) * Ctot + ch) * 3;
                cs[0] = h0;
                cs[1] = h1;
                cs[2] = h2;
            }
        }
        st[0] = h0;
        st[1] = h1;
        st[2] = h2;
    }
    for (int i = tid; i < NTK * G; i += NT) {
        const int t = i / G, g = i % G, h = j * G + g;
        const int64_t row = (int64_t)seq * NTK + t;
        const float av = to_f32(static_cast<const TA*>(p.a)[row * Hv + h]);
        const float bv = to_f32(static_cast<const TA*>(p.b)[row * Hv + h]);
        s_al[i] = __expf(-__expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]));
        s_be[i] = sigmoid_f(bv);
    }
    __syncthreads();
    for (int vi = warp; vi < 2 * NTK; vi += NW) {   // L2 norms: q^ and k^ of every token
        float* x = sfeat + (vi >> 1) * nch + (vi & 1) * DK;
        float ss = 0.f;
        for (int i = lane; i < DK; i += 32) ss = fmaf(x[i], x[i], ss);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float r = rsqrtf(ss + p.l2_eps);
        for (int i = lane; i < DK; i += 32) x[i] *= r;
    }
    __syncthreads();

    // ---- stream the state rows: n_tok updates per row ----
    constexpr int NF4 = DK / 32;
    constexpr int U = DK == 32 ? 4 : 2;   // passes of MRPP rows in flight per warp
    const int lane8 = lane % MLPR, sub = lane / MLPR;
    if (warp < NTK) {   // k_t . q_t, formed as the one-token kernel forms it
        const int t = warp;
        float4 k4[NF4], q4[NF4];
        row_load<NF4>(sfeat + t * nch + DK, lane8, k4);
        row_load<NF4>(sfeat + t * nch, lane8, q4);
        const float x = row_dot<NF4>(k4, q4);
        if (lane == 0) s_kq[t] = x;
    }
    for (int t = NW + warp; t < NTK; t += NW) {
        float4 k4[NF4], q4[NF4];
        row_load<NF4>(sfeat + t * nch + DK, lane8, k4);
        row_load<NF4>(sfeat + t * nch, lane8, q4);
        const float x = row_dot<NF4>(k4, q4);
        if (lane == 0) s_kq[t] = x;
    }
    __syncthreads();
    const float inv_sqrt_dk = rsqrtf((float)DK);
    const int64_t blk = ((int64_t)seq * Hv + (int64_t)j * G) * dv * DK;
    TS* Sb = static_cast<TS*>(p.rec_state) + blk;
    TS* snap0 = static_cast<TS*>(m.state_snap);
    const int64_t snap_stride = (int64_t)m.n_seqs * Hv * dv * DK;
    const int rows = G * dv;
    for (int R0 = warp * MRPP * U; R0 < rows; R0 += NW * MRPP * U) {
        float4 s[U][NF4];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int R = R0 + u * MRPP + sub;
#pragma unroll
            for (int i = 0; i < NF4; i++)
                s[u][i] = R < rows ? State4<TS>::ld(Sb + (int64_t)R * DK + 4 * lane8 + 32 * i)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int t = 0; t < kMaxTok; t++) {
            if (t >= NTK) break;
            float4 k4[NF4], q4[NF4];
            row_load<NF4>(sfeat + t * nch + DK, lane8, k4);
            row_load<NF4>(sfeat + t * nch, lane8, q4);
#pragma unroll
            for (int u = 0; u < U; u++) {
                const int R = R0 + u * MRPP + sub;
                const int g = min(R, rows - 1) / dv;
                const float uk = row_dot<NF4>(s[u], k4);
                const float up = row_dot<NF4>(s[u], q4);
                if (R < rows) {
                    const float al = s_al[t * G + g], be = s_be[t * G + g];
                    const float d = be * (sfeat[t * nch + 2 * DK + R] - al * uk);
                    row_update<NF4>(s[u], k4, al, d);
                    if (snap0) {
#pragma unroll
                        for (int i = 0; i < NF4; i++)
                            State4<TS>::st(snap0 + t * snap_stride + blk + (int64_t)R * DK + 4 * lane8 + 32 * i,
                                           s[u][i]);
                    }
                    if (lane8 == 0) so[t * rows + R] = (al * up + d * s_kq[t]) * inv_sqrt_dk;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int R = R0 + u * MRPP + sub;
            if (R < rows) {
#pragma unroll
                for (int i = 0; i < NF4; i++)
                    State4<TS>::st(Sb + (int64_t)R * DK + 4 * lane8 + 32 * i, s[u][i]);
            }
        }
    }
    __syncthreads();

    // ---- gated RMSNorm per token and value head ----
    const TA* pz = static_cast<const TA*>(p.z);
    TO* po = static_cast<TO*>(p.out);
    for (int tg = warp; tg < NTK * G; tg += NW) {
        const int t = tg / G, g = tg % G;
        const float* o = so + t * rows + g * dv;
        float ss = 0.f;
        for (int r = lane; r < dv; r += 32) ss = fmaf(o[r], o[r], ss);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float rs = rsqrtf(ss / (float)dv + p.norm_eps);
        const int h = j * G + g;
        for (int r = lane; r < dv; r += 32) {
            const int64_t off = (((int64_t)seq * NTK + t) * Hv + h) * dv + r;
            const float zz = to_f32(pz[off]);
            from_f32(o[r] * rs * p.norm_w[r] * silu_f(zz), po + off);
        }
    }
}


// ---------------------------------------------------------------------------
// Decode (one or several tokens per sequence) with the state streamed in
// through shared memory by a persistent, warp-specialised kernel.  The work is
// the same as above, in units of one (sequence, key head): the unit's G x d_v
// state rows are one contiguous block.  A CTA takes units u = blockIdx.x,
// blockIdx.x + gridDim.x, ...; its warps split the work so that the state
// stream never waits for the per-unit set-up:
//   producer (1 warp)  bulk-copies the state in as slabs of SR rows, across
//                      units without a break, keeping SSTAGES slabs in flight,
//                      and each unit's conv state and q, k, v, z rows one unit
//                      ahead into a ring of three input buffers;
//   state (8 warps)    update the rows of each slab that has landed (8 lanes
//                      per row, n_tok updates, token after token, with the
//                      same per-row arithmetic and order as the kernels above)
//                      and store the new rows from registers (coalesced 16-byte
//                      streaming stores);
//   aux (3 warps)      conv + SiLU, conv-state roll, gates and L2 norms of the
//                      next unit (from its input buffer) into one of two feature
//                      buffers, and the gated RMSNorm of the unit the state warps
//                      have just finished.
// They meet only on mbarriers.  A wait that runs out raises the abort word,
// after which every wait returns at once, so all warps run to the end (through
// the aux warps' named barriers) and the error word reports it.
// ---------------------------------------------------------------------------
constexpr int SNW = 8;                        // state warps
constexpr int ANW = 3;                        // aux warps
constexpr int SNT = 32 * (SNW + ANW + 1);     // + the producer warp
constexpr int PRODUCER = SNW + ANW;           // warp index of the producer
constexpr int SR = SNW * MRPP;                // state rows per slab: 4 per state warp

// at most this many slabs in flight per CTA (64 KiB of state at d_k = 128 in either
// storage type); the host takes fewer where that lets two CTAs share an SM
template <typename TS> __host__ __device__ constexpr int stream_stages() { return sizeof(TS) == 4 ? 4 : 8; }
template <typename TS, int DK> __host__ __device__ constexpr uint32_t slab_bytes() {
    return (uint32_t)(SR * DK * sizeof(TS));
}
// mbarriers: full and read per stage, feature-ready, feature-free, o-ready and
// o-free per buffer, input-full and input-free per input buffer; the abort word
constexpr uint32_t kStreamBarBytes = 256;
static_assert(8 * (2 * 8 + 4 * 2 + 2 * 3) + 4 <= kStreamBarBytes, "mbarriers and the abort word");
// one input buffer: the unit's conv state (its q, k and v channels, 3 each), then
// per token its q, k, v and z rows, as the activation type
template <typename TA>
__host__ __device__ constexpr size_t input_bytes(int dk, int G, int dv, int n_tok) {
    return ((size_t)(2 * dk + G * dv) * 3 * sizeof(TA) + (size_t)n_tok * (2 * dk + 2 * G * dv) * sizeof(TA) + 127) /
           128 * 128;
}
// one feature buffer: q^ | k^ | v^ per token, gates, k.q per token; one o buffer.
// Rounded up to 16 bytes: the second buffer's q^ and k^ rows are read as float4.
__host__ __device__ constexpr size_t feat_floats(int dk, int G, int dv, int n_tok) {
    return ((size_t)n_tok * (2 * dk + G * dv + 2 * G + 1) + 3) / 4 * 4;
}
template <typename TA, typename TS, int DK>
__host__ __device__ constexpr size_t stream_smem_bytes(int G, int dv, int n_tok, int stages) {
    return (size_t)stages * slab_bytes<TS, DK>() + kStreamBarBytes + 3 * input_bytes<TA>(DK, G, dv, n_tok) +
           2 * (feat_floats(DK, G, dv, n_tok) + (size_t)n_tok * G * dv) * sizeof(float) + 128;
}

// A row's dot product with four partial sums (one per float4 component), added
// pairwise, then the butterfly over the row's 8 lanes: one fixed order, and a
// chain of d_k / 32 FMAs instead of d_k / 8.
template <int NF4>
__device__ __forceinline__ float row_dot4(const float4 (&s)[NF4], const float4 (&v)[NF4]) {
    float x = 0.f, y = 0.f, z = 0.f, w = 0.f;
#pragma unroll
    for (int i = 0; i < NF4; i++) {
        x = fmaf(s[i].x, v[i].x, x);
        y = fmaf(s[i].y, v[i].y, y);
        z = fmaf(s[i].z, v[i].z, z);
        w = fmaf(s[i].w, v[i].w, w);
    }
    x = (x + y) + (z + w);
#pragma unroll
    for (int off = MLPR / 2; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Slab rows in shared memory -> registers: lane8 of a row owns columns 4 lane8 + 32 i.
template <typename TS, int NF4> struct Slab;
template <int NF4> struct Slab<float, NF4> {
    static __device__ __forceinline__ void ld(const uint8_t* row, int lane8, float4 (&s)[NF4]) {
#pragma unroll
        for (int i = 0; i < NF4; i++) s[i] = *reinterpret_cast<const float4*>(row + 16 * lane8 + 128 * i);
    }
};
template <int NF4> struct Slab<__nv_bfloat16, NF4> {
    static __device__ __forceinline__ void ld(const uint8_t* row, int lane8, float4 (&s)[NF4]) {
#pragma unroll
        for (int i = 0; i < NF4; i++) {
            const uint2 u = *reinterpret_cast<const uint2*>(row + 8 * lane8 + 64 * i);
            s[i] = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                               __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        }
    }
};

template <typename TA, typename TO, typename TS, int DK>
__global__ void __launch_bounds__(SNT, 2) gdn_decode_stream_kernel(MultiArgs m) {
    constexpr int NF4 = DK / 32;
    constexpr uint32_t SB = slab_bytes<TS, DK>();
    constexpr uint32_t ROWB = DK * sizeof(TS);
    static_assert(8 * (2 * stream_stages<TS>() + 14) + 4 <= kStreamBarBytes, "mbarrier area");
    const int SSTAGES = m.stages;
    const Args& p = m.a;
    const int NTK = m.n_tok;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 127u) & ~127u;
    uint8_t* smem = smem_raw + (sb - raw);
    const uint32_t bar_full = sb + SSTAGES * SB, bar_done = bar_full + 8 * SSTAGES;
    const uint32_t bar_fready = bar_done + 8 * SSTAGES, bar_ffree = bar_fready + 16;
    const uint32_t bar_oready = bar_ffree + 16, bar_ofree = bar_oready + 16;
    const uint32_t bar_ifull = bar_ofree + 16, bar_ifree = bar_ifull + 24;
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + SSTAGES * SB + 8 * (2 * SSTAGES + 14));
    const int Hk = p.Hk, Hv = p.Hv, dv = p.dv, G = Hv / Hk;
    const int Cq = Hk * DK, Cv = Hv * dv, Ctot = 2 * Cq + Cv;
    const int nch = 2 * DK + G * dv;        // a unit's channels: q, k of its key head, v of its value heads
    const int rows = G * dv;                // a multiple of SR (d_v is 32, 64 or 128)
    const int n_slabs = rows / SR;          // per unit
    const int n_units = m.n_seqs * Hk;
    const int my_units = blockIdx.x < n_units ? (n_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const size_t FF = feat_floats(DK, G, dv, NTK);
    const uint32_t IB = (uint32_t)input_bytes<TA>(DK, G, dv, NTK);
    const uint32_t CSB = (uint32_t)(nch * 3 * sizeof(TA));          // conv state of a unit
    const uint32_t TOKB = (uint32_t)((2 * DK + 2 * G * dv) * sizeof(TA));   // q, k, v, z rows of a token
    const uint32_t in0 = sb + SSTAGES * SB + kStreamBarBytes;                          // [3][IB]
    float* feat0 = reinterpret_cast<float*>(smem + SSTAGES * SB + kStreamBarBytes + 3 * IB);   // [2][FF]
    float* so0 = feat0 + 2 * FF;                                                        // [2][NTK][rows]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < SSTAGES; s++) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_done + 8 * s, SNW);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(bar_fready + 8 * b, 1);
            mbar_init(bar_ffree + 8 * b, SNW);
            mbar_init(bar_oready + 8 * b, SNW);
            mbar_init(bar_ofree + 8 * b, 1);
        }
        for (int b = 0; b < 3; b++) {
            mbar_init(bar_ifull + 8 * b, 1);
            mbar_init(bar_ifree + 8 * b, 1);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();   // (the only CTA-wide barrier)
    // a bounded wait that, once anything has run out, returns at once; the state
    // warps' waits for a slab spin, the others sleep between checks
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (*s_abort) return;
        if (!mbar_wait_idle(bar, parity)) {
            *s_abort = 1;
            record_error(kErrCopyTimeout);
        }
    };
    auto wait_spin = [&](uint32_t bar, uint32_t parity) {
        if (*s_abort) return;
        if (!mbar_wait_bounded(bar, parity)) {
            *s_abort = 1;
            record_error(kErrCopyTimeout);
        }
    };
    auto arrive = [&](uint32_t bar) { asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory"); };
    auto unit_seq = [&](int k) { return (int)((blockIdx.x + (int64_t)k * gridDim.x) / Hk); };
    auto unit_kh = [&](int k) { return (int)((blockIdx.x + (int64_t)k * gridDim.x) % Hk); };
    auto unit_state = [&](int k) {
        return static_cast<TS*>(p.rec_state) + ((int64_t)unit_seq(k) * Hv + (int64_t)unit_kh(k) * G) * dv * DK;
    };

    if (warp == PRODUCER) {
        // ---- producer: slab g of the CTA's stream goes to stage g % SSTAGES once slab g - SSTAGES is read ----
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            // unit k's conv state and token rows into input buffer k % 3, once unit k - 3 is done with it
            auto load_inputs = [&](int k) {
                const int b = k % 3;
                if (k >= 3) wait(bar_ifree + 8 * b, ((k - 3) / 3) & 1);
                if (*s_abort) return;
                const int seq = unit_seq(k), j = unit_kh(k);
                const uint32_t dst = in0 + b * IB, bar = bar_ifull + 8 * b;
                mbar_arrive_expect_tx(bar, CSB + NTK * TOKB);
                const uint8_t* cs = static_cast<const uint8_t*>(p.conv_state) + (int64_t)seq * Ctot * 3 * sizeof(TA);
                bulk_g2s(dst, cs + (int64_t)j * DK * 3 * sizeof(TA), DK * 3 * sizeof(TA), bar);
                bulk_g2s(dst + DK * 3 * sizeof(TA), cs + (int64_t)(Cq + j * DK) * 3 * sizeof(TA), DK * 3 * sizeof(TA),
                         bar);
                bulk_g2s(dst + 2 * DK * 3 * sizeof(TA), cs + (int64_t)(2 * Cq + j * G * dv) * 3 * sizeof(TA),
                         G * dv * 3 * sizeof(TA), bar);
                for (int t = 0; t < NTK; t++) {
                    const int64_t row = (int64_t)seq * NTK + t;
                    const uint32_t d = dst + CSB + t * TOKB;
                    bulk_g2s(d, static_cast<const TA*>(p.q) + row * Cq + j * DK, DK * sizeof(TA), bar);
                    bulk_g2s(d + DK * sizeof(TA), static_cast<const TA*>(p.k) + row * Cq + j * DK, DK * sizeof(TA), bar);
                    bulk_g2s(d + 2 * DK * sizeof(TA), static_cast<const TA*>(p.v) + row * Cv + j * G * dv,
                             G * dv * sizeof(TA), bar);
                    bulk_g2s(d + (2 * DK + G * dv) * sizeof(TA), static_cast<const TA*>(p.z) + row * Cv + j * G * dv,
                             G * dv * sizeof(TA), bar);
                }
            };
            int in_issued = 0;
            for (; in_issued < 2 && in_issued < my_units; in_issued++) load_inputs(in_issued);
            // slab (k, i) of the CTA's stream goes to stage s; the stage's previous slab was
            // released in phase ph (stage and phase kept as counters: SSTAGES is a runtime value)
            int issued = 0, s = 0;
            uint32_t ph = 0;
            for (int k = 0; k < my_units && !*s_abort; k++) {
                if (k + 1 == in_issued && in_issued < my_units) load_inputs(in_issued++);
                const uint8_t* src = reinterpret_cast<const uint8_t*>(unit_state(k));
                for (int i = 0; i < n_slabs; i++) {
                    if (issued >= SSTAGES) wait(bar_done + 8 * s, ph);
                    if (*s_abort) break;
                    mbar_arrive_expect_tx(bar_full + 8 * s, SB);
                    bulk_g2s_hint(sb + s * SB, src + (int64_t)i * SB, SB, bar_full + 8 * s, pol);
                    issued++;
                    if (++s == SSTAGES) {
                        s = 0;
                        if (issued > SSTAGES) ph ^= 1u;
                    }
                }
            }
            // every load issued completes before the CTA may exit (bounded)
            for (int g = issued - SSTAGES > 0 ? issued - SSTAGES : 0; g < issued; g++)
                mbar_wait_bounded(bar_full + 8 * (g % SSTAGES), (g / SSTAGES) & 1);
            for (int k = in_issued - 3 > 0 ? in_issued - 3 : 0; k < in_issued; k++)
                mbar_wait_bounded(bar_ifull + 8 * (k % 3), (k / 3) & 1);
        }
        return;
    }

    const float inv_sqrt_dk = rsqrtf((float)DK);
    if (warp < SNW) {
        // ---- state warps ----
        const int lane8 = lane % MLPR, sub = lane / MLPR;
        TS* snap0 = static_cast<TS*>(m.state_snap);
        const int64_t snap_stride = (int64_t)m.n_seqs * Hv * dv * DK;
        int s = 0;         // stage of the next slab of the CTA's stream
        uint32_t ph = 0;   // and the phase it completes in
        for (int k = 0; k < my_units; k++) {
            const int b = k & 1;
            const float* feat = feat0 + b * FF;
            const float* s_al = feat + NTK * nch;
            const float* s_be = s_al + NTK * G;
            const float* s_kq = s_be + NTK * G;
            float* so = so0 + b * NTK * rows;
            wait(bar_fready + 8 * b, (k >> 1) & 1);
            if (k >= 2) wait(bar_ofree + 8 * b, ((k - 2) >> 1) & 1);
            TS* Sb = unit_state(k);
            const int64_t blk = Sb - static_cast<TS*>(p.rec_state);
            for (int i = 0; i < n_slabs; i++) {
                wait_spin(bar_full + 8 * s, ph);
                const int rl = MRPP * warp + sub;   // row within the slab
                const int R = i * SR + rl;          // row within the unit
                float4 st4[NF4];
                Slab<TS, NF4>::ld(smem + s * SB + rl * ROWB, lane8, st4);
                __syncwarp();   // the warp's rows are in registers: the stage may be refilled
                if (lane == 0) arrive(bar_done + 8 * s);
                if (++s == SSTAGES) {
                    s = 0;
                    ph ^= 1u;
                }
                const int gh = R / dv;
#pragma unroll 1
                for (int t = 0; t < NTK; t++) {
                    float4 k4[NF4], q4[NF4];
                    row_load<NF4>(feat + t * nch + DK, lane8, k4);
                    row_load<NF4>(feat + t * nch, lane8, q4);
                    const float uk = row_dot4<NF4>(st4, k4);
                    const float up = row_dot4<NF4>(st4, q4);
                    const float al = s_al[t * G + gh], be = s_be[t * G + gh];
                    const float d = be * (feat[t * nch + 2 * DK + R] - al * uk);
                    row_update<NF4>(st4, k4, al, d);
                    if (snap0) {
#pragma unroll
                        for (int c = 0; c < NF4; c++)
                            State4<TS>::st(snap0 + t * snap_stride + blk + (int64_t)R * DK + 4 * lane8 + 32 * c,
                                           st4[c]);
                    }
                    if (lane8 == 0) so[t * rows + R] = (al * up + d * s_kq[t]) * inv_sqrt_dk;
                }
#pragma unroll
                for (int c = 0; c < NF4; c++) State4<TS>::st(Sb + (int64_t)R * DK + 4 * lane8 + 32 * c, st4[c]);
            }
            __syncwarp();
            if (lane == 0) {
                arrive(bar_ffree + 8 * b);    // the unit's features are no longer read
                arrive(bar_oready + 8 * b);   // its o rows are complete
            }
        }
        return;
    }

    // ---- aux warps: features of unit k, then the gated norm of unit k - 1 ----
    const int at = tid - 32 * SNW;   // 0 .. 32 ANW - 1
    const int aw = at >> 5;
    auto asyncb = [&]() { asm volatile("bar.sync 1, %0;" ::"n"(32 * ANW) : "memory"); };
    TA* cst = static_cast<TA*>(p.conv_state);
    TO* po = static_cast<TO*>(p.out);
    auto norm_unit = [&](int k) {
        const int b = k & 1, seq = unit_seq(k), j = unit_kh(k);
        wait(bar_oready + 8 * b, (k >> 1) & 1);
        const float* so = so0 + b * NTK * rows;
        const uint8_t* inb = smem + (in0 - sb) + (k % 3) * IB + CSB;
        for (int tg = aw; tg < NTK * G; tg += ANW) {
            const int t = tg / G, gq = tg % G;
            const float* o = so + t * rows + gq * dv;
            const TA* zr = reinterpret_cast<const TA*>(inb + t * TOKB) + 2 * DK + G * dv + gq * dv;
            float ss = 0.f;
            for (int r = lane; r < dv; r += 32) ss = fmaf(o[r], o[r], ss);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float rs = rsqrtf(ss / (float)dv + p.norm_eps);
            const int h = j * G + gq;
            for (int r = lane; r < dv; r += 32) {
                const int64_t off = (((int64_t)seq * NTK + t) * Hv + h) * dv + r;
                from_f32(o[r] * rs * p.norm_w[r] * silu_f(to_f32(zr[r])), po + off);
            }
        }
        asyncb();   // every aux thread has read the o rows and z
        if (at == 0) {
            arrive(bar_ofree + 8 * b);
            arrive(bar_ifree + 8 * (k % 3));
        }
    };
    for (int k = 0; k < my_units; k++) {
        const int b = k & 1, seq = unit_seq(k), j = unit_kh(k);
        float* feat = feat0 + b * FF;
        float* s_al = feat + NTK * nch;
        float* s_be = s_al + NTK * G;
        float* s_kq = s_be + NTK * G;
        if (k >= 2) wait(bar_ffree + 8 * b, ((k - 2) >> 1) & 1);
        wait(bar_ifull + 8 * (k % 3), (k / 3) & 1);
        const uint8_t* inb = smem + (in0 - sb) + (k % 3) * IB;
        const TA* in_cs = reinterpret_cast<const TA*>(inb);   // [nch][3], in the unit's channel order
        for (int i = at; i < nch; i += 32 * ANW) {
            const int ch = i < DK ? j * DK + i : i < 2 * DK ? Cq + j * DK + (i - DK) : 2 * Cq + j * G * dv + (i - 2 * DK);
            TA* st = cst + ((int64_t)seq * Ctot + ch) * 3;
            TA h0 = in_cs[3 * i], h1 = in_cs[3 * i + 1], h2 = in_cs[3 * i + 2];
            const float4 w = reinterpret_cast<const float4*>(p.conv_w)[ch];
            for (int t = 0; t < NTK; t++) {
                const TA xr = reinterpret_cast<const TA*>(inb + CSB + t * TOKB)[i];
                float acc = w.x * to_f32(h0);
                acc = fmaf(w.y, to_f32(h1), acc);
                acc = fmaf(w.z, to_f32(h2), acc);
                acc = fmaf(w.w, to_f32(xr), acc);
                feat[t * nch + i] = silu_f(acc);
                h0 = h1;
                h1 = h2;
                h2 = xr;
                if (m.conv_snap) {
                    TA* cs = static_cast<TA*>(m.conv_snap) + (((int64_t)t * m.n_seqs + seq) * Ctot + ch) * 3;
                    cs[0] = h0;
                    cs[1] = h1;
                    cs[2] = h2;
                }
            }
            st[0] = h0;
            st[1] = h1;
            st[2] = h2;
        }
        for (int i = at; i < NTK * G; i += 32 * ANW) {
            const int t = i / G, gq = i % G, h = j * G + gq;
            const int64_t row = (int64_t)seq * NTK + t;
            const float av = to_f32(static_cast<const TA*>(p.a)[row * Hv + h]);
            const float bv = to_f32(static_cast<const TA*>(p.b)[row * Hv + h]);
            s_al[i] = __expf(-__expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]));
            s_be[i] = sigmoid_f(bv);
        }
        asyncb();
        for (int vi = aw; vi < 2 * NTK; vi += ANW) {   // L2 norms: q^ and k^ of every token
            float* x = feat + (vi >> 1) * nch + (vi & 1) * DK;
            float ss = 0.f;
            for (int i = lane; i < DK; i += 32) ss = fmaf(x[i], x[i], ss);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float r = rsqrtf(ss + p.l2_eps);
            for (int i = lane; i < DK; i += 32) x[i] *= r;
        }
        asyncb();
        const int lane8 = lane % MLPR;
        for (int t = aw; t < NTK; t += ANW) {   // k_t . q_t, formed as the state rows form their dot products
            float4 k4[NF4], q4[NF4];
            row_load<NF4>(feat + t * nch + DK, lane8, k4);
            row_load<NF4>(feat + t * nch, lane8, q4);
            const float x = row_dot4<NF4>(k4, q4);
            if (lane == 0) s_kq[t] = x;
        }
        asyncb();
        if (at == 0) arrive(bar_fready + 8 * b);
        if (k >= 1) norm_unit(k - 1);
    }
    if (my_units >= 1) norm_unit(my_units - 1);
}

}  // namespace dec
}  // namespace gdn
