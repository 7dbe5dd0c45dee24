// Short causal depthwise convolution (kernel 4) + SiLU over the q|k|v channels,
// with the per-key-head L2 norm of q and k fused into the same pass.
//
// Layer: "Qwen3.8-Flash-Next" (llm-architectures-explained), "Every architecture
// field": linear_conv_kernel_dim = 4 over q|k|v; SiLU is the model's hidden_act
// ("Raw config fields", llm-atlas-9r2).  Tap K-1 multiplies the current token;
// the K-1 inputs before a sequence start come from conv_state (oldest first).
//
// Output: q^, k^ (unit norm per key head) and v^ as fp16 in the workspace.  The
// chunked prefill kernels feed them straight to the tensor cores.  HBM-bound:
// each thread owns 8 channels and streams a run of tokens through a 3-row
// window of past inputs, with the next rows' 16-byte loads already in flight;
// a CTA covers 1024 channels, so every load and store of a token row is one
// contiguous 2 KiB piece.
#pragma once
#include "device.cuh"

namespace gdn {

struct ConvArgs {
    const void* q;           // [T][Cq]   act dtype
    const void* k;           // [T][Cq]
    const void* v;           // [T][Cv]
    const float* conv_w;     // [Ctot][4]
    const void* conv_state;  // [N][Ctot][3] act dtype (read only here)
    const int32_t* cu;       // [N+1]
    int n_seqs;
    int64_t T;
    int Hk, Hv, dk, dv;
    float l2_eps;
    __half* qh;              // [T][Cq]
    __half* kh;              // [T][Cq]
    __half* vh;              // [T][Cv]
    int32_t* flags;          // per-call check word: bit 0 (malformed cu_seqlens) is read here,
                             // bit 1 is set here when an output overflows fp16
    const int32_t* chunk_off;  // [N+1] first global chunk of each sequence (chunk_offsets_kernel)
    int64_t g_lo, g_hi;      // this launch convolves the tokens of global chunks [g_lo, g_hi)
};

// The 32-token tiles (or runs) a launch over global chunks [g_lo, g_hi) owns:
// those that start in its token range.  A tile that starts before the range
// and reaches into it belongs to the launch before, so the launches over
// consecutive chunk ranges write disjoint tiles, and the tokens of chunks
// [g_lo, g_hi) are all written once this launch and the ones before it are done.
__device__ __forceinline__ void conv_tile_range(const ConvArgs& p, int64_t& first, int64_t& count) {
    const int64_t t_lo = chunk_first_token(p.cu, p.chunk_off, p.n_seqs, p.T, p.g_lo);
    const int64_t t_hi = chunk_first_token(p.cu, p.chunk_off, p.n_seqs, p.T, p.g_hi);
    first = (t_lo + 31) / 32;
    count = (t_hi + 31) / 32 - first;
}

// fp16 keeps values below 65520 in magnitude; larger ones round to infinity.
constexpr float kHalfOverflow = 65520.f;

// The range check's outcome: v outputs are checked by magnitude (vmax), q and k
// rows by their squared norm, which must stay finite for the L2 norm.
__device__ __forceinline__ void report_range(const ConvArgs& p, float vmax, bool qk_bad) {
    if (!(vmax < kHalfOverflow) || qk_bad) {
        atomicOr(p.flags, 2);
        record_error(kErrRange);
    }
}

constexpr int kConvThreads = 128;   // 8 channels per thread
constexpr int kConvRun = 32;        // tokens per thread (one run per CTA)
static_assert(kConvRun == 32, "conv_tile_range counts 32-token runs");
// input rows in flight per thread
template <typename TA> __host__ __device__ constexpr int conv_depth() { return sizeof(TA) == 2 ? 8 : 4; }

template <typename TA>
__device__ __forceinline__ const TA* __restrict__ conv_channel_ptr(const ConvArgs& p, int64_t t, int c, int Cq, int Cv) {
    if (c < Cq) return static_cast<const TA*>(p.q) + t * Cq + c;
    if (c < 2 * Cq) return static_cast<const TA*>(p.k) + t * Cq + (c - Cq);
    return static_cast<const TA*>(p.v) + t * Cv + (c - 2 * Cq);
}

// 8 consecutive activations of one token, kept packed until used.
template <typename TA> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* __restrict__ p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void get(float (&f)[8]) const {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* __restrict__ p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void get(float (&f)[8]) const {
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

template <typename TA>
__global__ void __launch_bounds__(kConvThreads, 4) conv_silu_norm_kernel(ConvArgs p) {
    if (*p.flags) return;   // cu_seqlens failed its check: sequence starts are not to be trusted
    const int Cq = p.Hk * p.dk, Cv = p.Hv * p.dv, Ctot = 2 * Cq + Cv;
    const int c = (blockIdx.y * kConvThreads + threadIdx.x) * 8;   // first of 8 channels
    int64_t run0, n_runs;
    conv_tile_range(p, run0, n_runs);
    if (blockIdx.x >= n_runs) return;
    const int64_t t_begin = (run0 + blockIdx.x) * kConvRun;
    // sequence of each token of the run and its first token
    __shared__ int s_seq[kConvRun];
    __shared__ long long s_start[kConvRun];
    if (threadIdx.x < kConvRun) {
        const int64_t t = t_begin + threadIdx.x;
        int lo = 0, hi = p.n_seqs - 1;              // last s with cu[s] <= t
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if ((int64_t)p.cu[mid] <= t) lo = mid; else hi = mid - 1;
        }
        s_seq[threadIdx.x] = lo;
        s_start[threadIdx.x] = p.cu[lo];
    }
    const bool active = c < Ctot;
    const bool is_qk = c < 2 * Cq;
    const TA* src = c < Cq ? static_cast<const TA*>(p.q) + c
                  : c < 2 * Cq ? static_cast<const TA*>(p.k) + (c - Cq)
                               : static_cast<const TA*>(p.v) + (c - 2 * Cq);
    const int64_t ld = is_qk ? Cq : Cv;
    __half* dst = c < Cq ? p.qh + c : c < 2 * Cq ? p.kh + (c - Cq) : p.vh + (c - 2 * Cq);
    const int n_run = (int)(p.T - t_begin < kConvRun ? p.T - t_begin : kConvRun);

    // the first rows of the run go in flight before anything else
    constexpr int kConvDepth = conv_depth<TA>();
    Raw8<TA> q[kConvDepth];
#pragma unroll
    for (int i = 0; i < kConvDepth; i++) {
        q[i].zero();
        if (active && i < n_run) q[i].load(src + (t_begin + i) * ld);
    }
    float w[8][4];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (active) t4 = __ldg(reinterpret_cast<const float4*>(p.conv_w) + c + i);
        w[i][0] = t4.x; w[i][1] = t4.y; w[i][2] = t4.z; w[i][3] = t4.w;
    }
    __syncthreads();

    // window of the 3 inputs before the current token (oldest first)
    float win[3][8];
    auto state_row = [&](int seq, int slot, float (&f)[8]) {
        const TA* st = static_cast<const TA*>(p.conv_state) + ((int64_t)seq * Ctot + c) * 3 + slot;
#pragma unroll
        for (int i = 0; i < 8; i++) f[i] = active ? to_f32(st[i * 3]) : 0.f;
    };
    {
        const int64_t s0 = s_start[0];
#pragma unroll
        for (int k = 0; k < 3; k++) {
            const int64_t u = t_begin - 3 + k;
            if (u < s0) {
                state_row(s_seq[0], 3 - (int)(s0 - u), win[k]);
            } else {
                Raw8<TA> r;
                r.zero();
                if (active) r.load(src + u * ld);
                r.get(win[k]);
            }
        }
    }

    const int group = p.dk >> 3;                    // threads per key head (4, 8 or 16)
    float vmax = 0.f;
    bool qk_bad = false;
#pragma unroll
    for (int it = 0; it < kConvRun; it++) {
        if (it >= n_run) break;
        const int64_t t = t_begin + it;
        if (it > 0 && t == s_start[it]) {            // a sequence starts here: its conv_state is the window
#pragma unroll
            for (int k = 0; k < 3; k++) state_row(s_seq[it], k, win[k]);
        }
        float x[8];
        q[it % kConvDepth].get(x);
        if (active && it + kConvDepth < n_run) q[it % kConvDepth].load(src + (t + kConvDepth) * ld);
        float y[8];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            float acc = w[i][0] * win[0][i];
            acc = fmaf(w[i][1], win[1][i], acc);
            acc = fmaf(w[i][2], win[2][i], acc);
            acc = fmaf(w[i][3], x[i], acc);
            y[i] = silu_f(acc);
            ss = fmaf(y[i], y[i], ss);
            win[0][i] = win[1][i];
            win[1][i] = win[2][i];
            win[2][i] = x[i];
        }
        // sum of squares over the key head's `group` threads (aligned lane groups)
        for (int off = 1; off < group; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (is_qk) {
            qk_bad |= !(ss <= 3.4e38f);
            const float r = rsqrtf(ss + p.l2_eps);
#pragma unroll
            for (int i = 0; i < 8; i++) y[i] *= r;
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) vmax = fmaxf(vmax, fabsf(y[i]));
        }
        if (active) {
            uint4 o;
            o.x = pack_half2(y[0], y[1]);
            o.y = pack_half2(y[2], y[3]);
            o.z = pack_half2(y[4], y[5]);
            o.w = pack_half2(y[6], y[7]);
            __stcs(reinterpret_cast<uint4*>(dst + t * ld), o);
        }
    }
    if (active) report_range(p, vmax, qk_bad);
}

// Tiled form of the same pass for bf16 activations whose q, k and v widths are
// multiples of 512 channels: each CTA owns one 512-channel slice of one of q, k,
// v and walks the token axis in tiles of 32 tokens.  A tile (35 rows: 3 rows of
// history, then the 32 tokens) arrives by TMA as 8 boxes of 64 channels, three
// tiles in flight, so the bytes in flight do not depend on registers.  Thread
// (tg, cg) computes 8 channels (cg) of 8 consecutive tokens (tg).
namespace ctile {
constexpr int NT = 256;
constexpr int CH = 512, TOK = 32, ROWS = TOK + 3, BOXW = 64, BOXES = CH / BOXW;
static_assert(TOK == 32, "conv_tile_range counts 32-token tiles");
constexpr uint32_t BOX_BYTES = ROWS * BOXW * 2;          // 4480
constexpr uint32_t TILE_BYTES = BOXES * BOX_BYTES;        // 35840
constexpr int BUFS = 3;
constexpr uint32_t OFF_BAR = BUFS * TILE_BYTES;
constexpr uint32_t OFF_SEQ = OFF_BAR + 64;                // int [2][TOK]
constexpr uint32_t OFF_START = OFF_SEQ + 2 * TOK * 4;     // int64 [2][TOK]
constexpr uint32_t SMEM_BYTES = OFF_START + 2 * TOK * 8 + 128;

// 8 consecutive tokens of one thread's 8 channels: tb points at the tile row of
// the first token's oldest tap.  PATCH: some of the tokens (bits of `near`) lie
// within 3 of their sequence start, and their older taps come from conv_state
// (cst: this thread's channels of sequence 0, seq_stride elements per sequence).
template <int GROUP, bool PATCH>
__device__ __forceinline__ void rows(const uint8_t* tb, const float (&w)[8][4], uint32_t near, int n_here,
                                     int64_t t0, const int* sq, const long long* sst, const __nv_bfloat16* cst,
                                     int64_t seq_stride, __half* out, int64_t ld, bool is_qk, float l2_eps,
                                     float& vmax, bool& qk_bad) {
    auto row = [&](int r, float (&f)[8]) {
        const uint4 u = *reinterpret_cast<const uint4*>(tb + r * 128);
        const uint32_t v[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            f[2 * i] = __uint_as_float(v[i] << 16);
            f[2 * i + 1] = __uint_as_float(v[i] & 0xffff0000u);
        }
    };
    float win[3][8];
    row(0, win[0]);
    row(1, win[1]);
    row(2, win[2]);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        if (i >= n_here) break;
        if (PATCH && (near & (1u << i))) {
            // History before the sequence start comes from its conv_state.  Patching the
            // window in place also serves the next tokens of the sequence.
            const int64_t t = t0 + i, s0 = sst[i];
#pragma unroll
            for (int k = 0; k < 3; k++) {
                const int64_t u = t - 3 + k;
                if (u < s0) {
                    const __nv_bfloat16* st = cst + (int64_t)sq[i] * seq_stride + (3 - (int)(s0 - u));
#pragma unroll
                    for (int e = 0; e < 8; e++) win[k][e] = __bfloat162float(st[e * 3]);
                }
            }
        }
        float x[8];
        row(i + 3, x);
        float y[8];
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e++) {
            float acc = w[e][0] * win[0][e];
            acc = fmaf(w[e][1], win[1][e], acc);
            acc = fmaf(w[e][2], win[2][e], acc);
            acc = fmaf(w[e][3], x[e], acc);
            y[e] = silu_f(acc);
            ss = fmaf(y[e], y[e], ss);
            win[0][e] = win[1][e];
            win[1][e] = win[2][e];
            win[2][e] = x[e];
        }
#pragma unroll
        for (int off = 1; off < GROUP; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (is_qk) {
            qk_bad |= !(ss <= 3.4e38f);
            const float r = rsqrtf(ss + l2_eps);
#pragma unroll
            for (int e = 0; e < 8; e++) y[e] *= r;
        } else {
#pragma unroll
            for (int e = 0; e < 8; e++) vmax = fmaxf(vmax, fabsf(y[e]));
        }
        uint4 o;
        o.x = pack_half2(y[0], y[1]);
        o.y = pack_half2(y[2], y[3]);
        o.z = pack_half2(y[4], y[5]);
        o.w = pack_half2(y[6], y[7]);
        __stcs(reinterpret_cast<uint4*>(out), o);
        out += ld;
    }
}
}  // namespace ctile

template <int GROUP>   // threads per key head: d_k / 8
__global__ void __launch_bounds__(ctile::NT, 2)
conv_tile_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, ConvArgs p, int parts) {
    using namespace ctile;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 127u) & ~127u;
    uint8_t* smem = smem_raw + (sb - raw);
    int* s_seq = reinterpret_cast<int*>(smem + OFF_SEQ);
    long long* s_start = reinterpret_cast<long long*>(smem + OFF_START);
    uint32_t* s_near = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 40);   // [2] per-tile masks
    const uint32_t bar0 = sb + OFF_BAR;
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 32);

    const int Cq = p.Hk * p.dk, Cv = p.Hv * p.dv, Ctot = 2 * Cq + Cv;
    const int n_slices = Ctot / CH;
    const int slice = blockIdx.x % n_slices, part = blockIdx.x / n_slices;
    const int c0 = slice * CH;                       // first channel of the slice (q|k|v numbering)
    const int tensor = c0 < Cq ? 0 : c0 < 2 * Cq ? 1 : 2;
    const int cl0 = c0 - (tensor == 0 ? 0 : tensor == 1 ? Cq : 2 * Cq);
    const CUtensorMap* tm = tensor == 0 ? &tm_q : tensor == 1 ? &tm_k : &tm_v;
    const int64_t ld = tensor == 2 ? Cv : Cq;
    __half* dst0 = tensor == 0 ? p.qh : tensor == 1 ? p.kh : p.vh;
    int64_t tile0, n_tiles;
    conv_tile_range(p, tile0, n_tiles);
    const int count = part < n_tiles ? (int)((n_tiles - part + parts - 1) / parts) : 0;
    if (count == 0 || *p.flags) return;   // (flags: cu_seqlens failed its check)

    const int tid = threadIdx.x, lane = tid & 31;
    const int tg = tid >> 6, cg = tid & 63;
    const int c = c0 + cg * 8, cl = cl0 + cg * 8;
    const bool is_qk = tensor < 2;
    auto tile_t0 = [&](int jj) { return (tile0 + part + (int64_t)jj * parts) * TOK; };
    auto issue = [&](int jj) {
        const uint32_t buf = sb + (jj % BUFS) * TILE_BYTES, bar = bar0 + 8 * (jj % BUFS);
        mbar_arrive_expect_tx(bar, TILE_BYTES);
        const int y = (int)(tile_t0(jj) - 3);
#pragma unroll
        for (int bx = 0; bx < BOXES; bx++) tma_load_2d(buf + bx * BOX_BYTES, tm, cl0 + bx * BOXW, y, bar);
    };
    auto search = [&](int jj) {   // sequence and its first token, for each token of tile jj (warp 0)
        const int64_t t = tile_t0(jj) + lane;
        int lo = 0, hi = p.n_seqs - 1;               // last s with cu[s] <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((int64_t)p.cu[mid] <= t) lo = mid; else hi = mid - 1;
        }
        s_seq[(jj & 1) * TOK + lane] = lo;
        s_start[(jj & 1) * TOK + lane] = p.cu[lo];
        const unsigned near = __ballot_sync(0xffffffffu, t < p.T && t - (int64_t)p.cu[lo] < 3);
        if (lane == 0) s_near[jj & 1] = near;
    };

    int issued = 0;   // tiles issued (thread 0)
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < BUFS; i++) mbar_init(bar0 + 8 * i, 1);
        fence_mbar_init();
        *s_abort = 0;
        for (; issued < BUFS - 1 && issued < count; issued++) issue(issued);
    }
    if (tid < 32) search(0);
    float w[8][4];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float4 t4 = __ldg(reinterpret_cast<const float4*>(p.conv_w) + c + i);
        w[i][0] = t4.x; w[i][1] = t4.y; w[i][2] = t4.z; w[i][3] = t4.w;
    }
    __syncthreads();

    float vmax = 0.f;
    bool qk_bad = false;
    for (int jj = 0; jj < count; jj++) {
        if (!mbar_wait_bounded(bar0 + 8 * (jj % BUFS), (jj / BUFS) & 1)) atomicOr((unsigned*)s_abort, 1u);
        __syncthreads();   // every thread is done with tile jj - 1 (buffer, sequence table)
        if (*s_abort) break;
        if (tid == 0 && jj + BUFS - 1 < count) {     // into the buffer of tile jj - 1
            fence_async_smem();
            issue(jj + BUFS - 1);
            issued = jj + BUFS;
        }
        if (tid < 32 && jj + 1 < count) search(jj + 1);
        const uint8_t* tb = smem + (jj % BUFS) * TILE_BYTES + (cg >> 3) * BOX_BYTES + (cg & 7) * 16;
        const int64_t t0 = tile_t0(jj) + tg * 8;
        const int* sq = s_seq + (jj & 1) * TOK + tg * 8;
        const long long* sst = s_start + (jj & 1) * TOK + tg * 8;
        const uint32_t near = (s_near[jj & 1] >> (tg * 8)) & 0xffu;   // bit i: token i is within 3 of its sequence start
        __half* out = dst0 + t0 * ld + cl;
        const int n_here = p.T - t0 < 8 ? (int)(p.T - t0) : 8;
        const __nv_bfloat16* cst = static_cast<const __nv_bfloat16*>(p.conv_state) + (int64_t)c * 3;
        if (near)
            ctile::rows<GROUP, true>(tb + tg * 8 * 128, w, near, n_here, t0, sq, sst, cst, (int64_t)Ctot * 3, out, ld,
                                     is_qk, p.l2_eps, vmax, qk_bad);
        else
            ctile::rows<GROUP, false>(tb + tg * 8 * 128, w, 0u, n_here, t0, sq, sst, cst, (int64_t)Ctot * 3, out, ld,
                                      is_qk, p.l2_eps, vmax, qk_bad);
    }
    report_range(p, vmax, qk_bad);
    if (*s_abort && tid == 0) {
        // a tile never arrived: report it and give the copies still in flight one more bounded wait
        record_error(kErrCopyTimeout);
        for (int i = issued > BUFS ? issued - BUFS : 0; i < issued; i++)
            mbar_wait_bounded(bar0 + 8 * (i % BUFS), (i / BUFS) & 1);
    }
}

// conv_state <- the last 3 raw inputs of each sequence (oldest first), keeping
// old entries when the sequence is shorter than 3.  Runs after the conv kernel,
// which still reads the old state, and after the call's checks (*flags): a call
// whose checks failed leaves conv_state as it was.  A sequence with cu[s+1] <
// cu[s] (which the checks reject) would read no row outside [cu[s], cu[s+1]).
template <typename TA>
__global__ void __launch_bounds__(256) conv_state_update_kernel(ConvArgs p, void* conv_state) {
    const int Cq = p.Hk * p.dk, Cv = p.Hv * p.dv, Ctot = 2 * Cq + Cv;
    const int c = blockIdx.y * 256 + threadIdx.x;
    const int s = blockIdx.x;
    if (c >= Ctot || *p.flags) return;
    const int64_t t0 = p.cu[s], t1 = p.cu[s + 1];
    if (t1 <= t0) return;
    TA* st = static_cast<TA*>(conv_state) + ((int64_t)s * Ctot + c) * 3;
    TA old[3] = {st[0], st[1], st[2]};
    TA nw[3];
#pragma unroll
    for (int q = 0; q < 3; q++) {
        const int64_t t = t1 - 3 + q;   // t >= t0 - 3 since t1 > t0
        nw[q] = (t >= t0) ? *conv_channel_ptr<TA>(p, t, c, Cq, Cv) : old[3 - (int)(t0 - t)];
    }
#pragma unroll
    for (int q = 0; q < 3; q++) st[q] = nw[q];
}

}  // namespace gdn
