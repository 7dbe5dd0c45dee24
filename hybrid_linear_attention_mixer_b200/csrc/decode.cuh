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

}  // namespace dec
}  // namespace gdn
