// C ABI of the Gated DeltaNet mixer (include/gdn.h): argument checks and
// kernel launches.  One translation unit holds every kernel.
#include "gdn.h"

#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "conv.cuh"
#include "cp.cuh"
#include "decode.cuh"
#include "device.cuh"
#include "fixup.cuh"
#include "gemm.cuh"
#include "intra.cuh"
#include "norm.cuh"
#include "scan.cuh"

namespace {

using gdn::ConvArgs;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

// The CUDA error behind this thread's most recent GDN_ERR_CUDA (gdn_last_cuda_error).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

// GDN_OK for cudaSuccess; otherwise remembers e for this thread and returns GDN_ERR_CUDA.
gdn_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return GDN_OK;
    t_last_cuda_error = e;
    return GDN_ERR_CUDA;
}

gdn_status check_config(const gdn_config* c) {
    if (!c) return GDN_ERR_INVALID_ARG;
    if (c->n_k_heads <= 0 || c->n_v_heads <= 0 || c->d_k <= 0 || c->d_v <= 0) return GDN_ERR_INVALID_ARG;
    if (!(c->l2_eps >= 0.f) || !(c->norm_eps >= 0.f) || !std::isfinite(c->l2_eps) ||
        !std::isfinite(c->norm_eps))
        return GDN_ERR_INVALID_ARG;
    if (c->act_dtype != GDN_BF16 && c->act_dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (c->out_dtype != GDN_BF16 && c->out_dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (c->state_dtype != GDN_BF16 && c->state_dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (c->n_v_heads % c->n_k_heads != 0) return GDN_ERR_UNSUPPORTED;
    if (!dim_ok(c->d_k) || !dim_ok(c->d_v)) return GDN_ERR_UNSUPPORTED;
    if (c->conv_kernel != 4 || c->chunk != gdn::intra::C) return GDN_ERR_UNSUPPORTED;
    if (c->prefill_segments < GDN_PREFILL_SPLIT || c->prefill_segments > GDN_PREFILL_MAX_SEGMENTS)
        return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status check_weights(const gdn_weights* w) {
    if (!w || !w->conv_weight || !w->A_log || !w->dt_bias || !w->norm_weight) return GDN_ERR_INVALID_ARG;
    if (!aligned(w->conv_weight, 16)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

// Split-chain prefill (fixup.cuh): one sequence's chain cut in two at its middle
// chunk, the second half scanned from zero and, at the same time, as the
// transition map from the identity; its outputs and end state are then
// corrected with the first half's end state.  Taken when asked for
// (GDN_PREFILL_SPLIT), for one sequence at the published head size with bf16
// activations and output and an fp32 state.  Not chosen automatically: at 4096
// tokens it measured 363 us against 333 us for two pipelined chunk ranges (the
// three concurrent scans read records, v and k at a rate that HBM does not
// sustain, so each runs well below half the chain's time).
bool split_mode(const gdn_config* c, int64_t T, int64_t n_seqs) {
    const int64_t chunks = (T + gdn::kChunk - 1) / gdn::kChunk;
    return c->prefill_segments == GDN_PREFILL_SPLIT && n_seqs == 1 && chunks >= 2 && c->d_k == 128 &&
           c->d_v == 128 && c->state_dtype == GDN_F32 && c->act_dtype == GDN_BF16 && c->out_dtype == GDN_BF16;
}

// Chunk ranges a prefill is pipelined over (gdn_config.prefill_segments): range
// s is global chunks [lo[s], lo[s+1]), the last one running to the end.  Range
// s's conv and intra-chunk kernels overlap the scan of range s - 1.  Range s is
// kRangeRatio^s times as long as the first: equal ranges (1) measured best on
// B200; ranges shrinking by 0.8 or 0.6 each (a long first range whose producers
// run alone, a short tail) measured the same at 4K tokens and 2-5% slower at
// 256K.
constexpr double kRangeRatio = 1.0;
struct SegPlan {
    int n;
    int32_t lo[GDN_PREFILL_MAX_SEGMENTS + 1];
};

SegPlan seg_plan(const gdn_config* c, int64_t T, int64_t n_seqs) {
    const int64_t chunks = (T + gdn::kChunk - 1) / gdn::kChunk;   // of one sequence of T tokens
    int64_t want = c->prefill_segments;
    if (want < 0 || split_mode(c, T, n_seqs)) want = 1;   // (the split chain is not range-pipelined)
    if (want == 0)   // automatic: chains too few to fill the GPU, in at most 8 ranges, 32 chunks a range on average
        want = n_seqs * c->n_v_heads <= 96 ? (chunks / 32 < 8 ? chunks / 32 : 8) : 1;
    if (want > GDN_PREFILL_MAX_SEGMENTS) want = GDN_PREFILL_MAX_SEGMENTS;
    if (want > chunks) want = chunks;
    SegPlan p;
    p.lo[0] = 0;
    if (want <= 1) {
        p.n = 1;
        p.lo[1] = 0x7fffffff;
        return p;
    }
    double tot = 0.0, w = 1.0;
    for (int s = 0; s < want; s++, w *= kRangeRatio) tot += w;
    double acc = 0.0;
    w = 1.0;
    for (int s = 1; s < want; s++, w *= kRangeRatio) {
        acc += w;
        int64_t b = (int64_t)(chunks * acc / tot + 0.5);
        const int64_t lo_min = p.lo[s - 1] + 1, hi_max = chunks - (want - s);   // every range non-empty
        b = b < lo_min ? lo_min : b > hi_max ? hi_max : b;
        p.lo[s] = (int32_t)b;
    }
    p.n = (int)want;
    p.lo[want] = 0x7fffffff;
    return p;
}

// Prefill workspace: fp16 q^, k^, v^ (conv output), the first chunk of each
// sequence followed by the call's check word (flags), one intra-chunk record
// per (chunk, value head), the o tile ([64][128], out dtype) of each (chunk,
// value head) before the gated norm, and, for a pipelined call, the fp32 state
// of every chain between the launches over consecutive chunk ranges.
struct Layout {
    size_t q_off, k_off, v_off, coff_off, flags_off, rec_off, o_off, carry_off, total;
    // split chain: [P | S_loc] fp32, S0 as bf16, the o^P tiles, a zeroed 64-row v block
    size_t summ_off = 0, s0b_off = 0, op_off = 0, zv_off = 0;
};

Layout workspace_layout(const gdn_config* c, int64_t T, int64_t n_seqs) {
    Layout L;
    const size_t qb = align_up((size_t)T * c->n_k_heads * c->d_k * sizeof(__half), 256);
    const size_t vb = align_up((size_t)T * c->n_v_heads * c->d_v * sizeof(__half), 256);
    const size_t cb = align_up((size_t)(n_seqs + 2) * sizeof(int32_t), 256);
    const size_t max_chunks = (size_t)((T + gdn::intra::C - 1) / gdn::intra::C) + (size_t)n_seqs;
    const size_t o_tile = (size_t)gdn::intra::C * 128 * (c->out_dtype == GDN_F32 ? 4 : 2);
    L.q_off = 0;
    L.k_off = qb;
    L.v_off = 2 * qb;
    L.coff_off = 2 * qb + vb;
    L.flags_off = L.coff_off + (size_t)(n_seqs + 1) * sizeof(int32_t);
    L.rec_off = L.coff_off + cb;
    L.o_off = L.rec_off + max_chunks * c->n_v_heads * gdn::intra::REC_BYTES;
    L.carry_off = align_up(L.o_off + max_chunks * c->n_v_heads * o_tile, 256);
    L.total = L.carry_off;
    const size_t st_f32 = (size_t)c->n_v_heads * c->d_v * c->d_k * sizeof(float);
    if (split_mode(c, T, n_seqs)) {   // carry: the first half's end state
        L.summ_off = L.carry_off + st_f32;
        L.s0b_off = L.summ_off + 2 * st_f32;
        L.op_off = align_up(L.s0b_off + st_f32 / 2, 256);
        L.zv_off = L.op_off + max_chunks * c->n_v_heads * o_tile;
        L.total = align_up(L.zv_off + (size_t)gdn::intra::C * c->n_v_heads * c->d_v * sizeof(__half), 256);
    } else if (seg_plan(c, T, n_seqs).n > 1) {
        L.total += (size_t)n_seqs * st_f32;
    }
    return L;
}

// Context-parallel workspace: the one-sequence prefill workspace of the segment,
// then its cu_seqlens {0, T_seg}, then a zeroed 64-row v^ block whose tensor map
// reads zeros for every later row (V = 0 for the transition's scan).
struct CpLayout {
    Layout pre;
    size_t o2_off, cu_off, zv_off, total;
};

// (after the prefill workspace: a second o-tile region, for the transition's
// scan, whose outputs are not used, so that it may run beside the other scan)
CpLayout cp_layout(const gdn_config* c, int64_t T_seg) {
    CpLayout L;
    L.pre = workspace_layout(c, T_seg, 1);
    L.o2_off = align_up(L.pre.total, 256);
    L.cu_off = align_up(L.o2_off + (L.pre.total - L.pre.o_off), 256);
    L.zv_off = L.cu_off + 256;
    L.total = L.zv_off + align_up((size_t)gdn::intra::C * c->n_v_heads * c->d_v * sizeof(__half), 256);
    return L;
}

// Prefill from host buffers: the tokens are cut into at most 8 segments of a
// multiple of 64 rows (at least 512), which run one after another on the
// caller's stream with the states carried on the device, while the next
// segment's inputs come in and the previous segment's output goes out on two
// copy streams.  Two staging slots; one prefill workspace.
struct HostPlan {
    int64_t seg_len;
    int n_seg;
};

HostPlan host_plan(int64_t T) {
    HostPlan h;
    int64_t n = (T + 511) / 512;
    n = n < 1 ? 1 : n > 8 ? 8 : n;
    h.seg_len = align_up((size_t)((T + n - 1) / n), 64);
    h.n_seg = (int)((T + h.seg_len - 1) / h.seg_len);
    return h;
}

struct HostLayout {
    HostPlan plan;
    size_t row_in[6];     // bytes per token of q, k, v, a, b, z
    size_t row_out;       // bytes per token of out
    size_t pre_off, cu_off, seg_cu_off[2], slot_off[2], in_off[6], out_off, slot_bytes, total;
};

HostLayout host_layout(const gdn_config* c, int64_t T, int32_t n_seqs) {
    HostLayout L;
    L.plan = host_plan(T);
    const size_t ab = c->act_dtype == GDN_F32 ? 4 : 2, ob = c->out_dtype == GDN_F32 ? 4 : 2;
    const size_t qk = (size_t)c->n_k_heads * c->d_k, vz = (size_t)c->n_v_heads * c->d_v, g = c->n_v_heads;
    const size_t widths[6] = {qk, qk, vz, g, g, vz};
    for (int i = 0; i < 6; ++i) L.row_in[i] = widths[i] * ab;
    L.row_out = vz * ob;
    const size_t rows = (size_t)L.plan.seg_len;
    size_t off = 0;
    for (int i = 0; i < 6; ++i) {
        L.in_off[i] = off;
        off = align_up(off + rows * L.row_in[i], 256);
    }
    L.out_off = off;
    off = align_up(off + rows * L.row_out, 256);
    L.slot_bytes = off;
    L.pre_off = 0;
    const size_t pre = workspace_layout(c, L.plan.seg_len, n_seqs).total;
    L.cu_off = align_up(pre, 256);
    L.seg_cu_off[0] = align_up(L.cu_off + ((size_t)n_seqs + 1) * 4, 256);
    L.seg_cu_off[1] = align_up(L.seg_cu_off[0] + ((size_t)n_seqs + 1) * 4, 256);
    L.slot_off[0] = align_up(L.seg_cu_off[1] + ((size_t)n_seqs + 1) * 4, 256);
    L.slot_off[1] = L.slot_off[0] + L.slot_bytes;
    L.total = L.slot_off[1] + L.slot_bytes;
    return L;
}

// Opt in to > 48 KiB of dynamic shared memory, once per device and kernel.
template <typename K>
cudaError_t ensure_smem(K kernel, int variant, size_t bytes) {
    static bool done[64][32];   // variants in use: 4-6, 8-20, 24-31
    if (variant < 0 || variant >= 32) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && done[dev][variant]) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev < 64) done[dev][variant] = true;
    return e;
}

// cuCtxGetCurrent, fetched once from the driver through the runtime.
PFN_cuCtxGetCurrent_v4000 ctx_getter() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    });
    return fn;
}

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime.  It
// is a driver call and needs a current context, which a host thread that has
// made no runtime call yet does not have: the current device's primary context
// is made current first in that case.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    CUcontext ctx = nullptr;
    auto get_ctx = ctx_getter();
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
    if (!ctx) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return nullptr;
    }
    return fn;
}

// 3-D map over a row-major [T][H][d] tensor: boxes of 64 (d) x 1 (head) x 64
// (tokens), 128-byte swizzle; elements past d or T read as zero.
bool head_tile_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int H,
                   int64_t T) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)d * elem_bytes, (cuuint64_t)H * d * elem_bytes};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)gdn::intra::C};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a row-major [T][C] bf16 activation: boxes of 64 channels x 35
// tokens (the conv tile), no swizzle; rows outside [0, T) read as zero.
bool conv_tile_map(CUtensorMap* m, const void* base, int C, int64_t T) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)C * 2};
    cuuint32_t box[2] = {(cuuint32_t)gdn::ctile::BOXW, (cuuint32_t)gdn::ctile::ROWS};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over z as [T][Hv * dv] (bf16 or fp32): boxes of d_v channels x 64
// tokens (one chunk of one head), no swizzle; rows past T read as zero.
bool z_rows_map(CUtensorMap* m, const void* base, bool bf16, int width, int dv, int64_t T) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const int eb = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)width * eb};
    cuuint32_t box[2] = {(cuuint32_t)dv, (cuuint32_t)gdn::norm::C};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Non-blocking streams for work that may overlap the caller's stream (forked
// from and joined back to it by events): 0 = the context-parallel transition
// scan, 1 = host-to-device copies, 2 = device-to-host copies, 3 = the prefill's
// conv-state update, 4 = a pipelined prefill's state chain (the device's
// greatest priority: when the kernel before it completes, its CTAs take the
// freed SMs ahead of the caller's next producer kernel), 5 = a pipelined
// prefill's gated norm.  They are kept per host thread and device, like the
// events below: a call in one thread never waits on another thread's side work,
// and a thread that captures a CUDA graph records only its own side work.
constexpr int kSideStreams = 6;
struct StreamPool {
    cudaStream_t s[64][kSideStreams] = {};
    ~StreamPool() {
        for (auto& per_dev : s)
            for (cudaStream_t x : per_dev)
                if (x) cudaStreamDestroy(x);
    }
};

cudaStream_t side_stream(int which = 0) {
    thread_local StreamPool pool;
    int dev = 0;
    if (which < 0 || which >= kSideStreams || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    cudaStream_t& st = pool.s[dev][which];
    if (!st) {
        int least = 0, greatest = 0;
        if (which != 4 || cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) greatest = 0;
        if (cudaStreamCreateWithPriority(&st, cudaStreamNonBlocking, greatest) != cudaSuccess) st = nullptr;
    }
    return st;
}

// Events for the forks and joins above, kept per host thread, device and use and
// reused from call to call: a stream wait refers to the record enqueued before
// it, so recording an event again in a later call leaves earlier waits intact,
// and no two threads share an event.
enum EventUse { kEvStageA = 0, kEvCp = 1, kEvHost = 2, kEvPipe = 3, kEvSplit = 4, kEvUses = 5 };

struct EventPool {
    std::vector<cudaEvent_t> ev[64][kEvUses];
    ~EventPool() {
        for (auto& per_dev : ev)
            for (auto& v : per_dev)
                for (cudaEvent_t e : v) cudaEventDestroy(e);
    }
};

// n events of the given use for this thread on the current device, or nullptr.
cudaEvent_t* thread_events(EventUse use, size_t n) {
    thread_local EventPool pool;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::vector<cudaEvent_t>& v = pool.ev[dev][use];
    while (v.size() < n) {
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        v.push_back(e);
    }
    return v.data();
}

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
    static int count[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 64 && count[dev]) return count[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) count[dev] = n;
    return n;
}

// 2-D map over a row-major [rows][K] bf16 matrix for the projections: boxes of
// 64 (K) x box_rows, 128-byte swizzle; elements past K or rows read as zero.
bool kmajor_map(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)gdn::gemm::BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch_linear(const void* x, const void* w, gdn::gemm::Args a, int variant, cudaStream_t st) {
    using S = gdn::gemm::Shape<BN>;
    CUtensorMap tm_x, tm_w;
    if (!kmajor_map(&tm_x, x, a.M, a.K, gdn::gemm::BM) || !kmajor_map(&tm_w, w, a.N, a.K, BN))
        return cudaErrorInvalidValue;
    a.n_blocks = (a.N + BN - 1) / BN;
    a.tiles = (int64_t)a.m_blocks * a.n_blocks;
    cudaError_t e = ensure_smem(gdn::gemm::linear_kernel<BN>, variant, S::SMEM);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(a.tiles, sm_count());
    gdn::gemm::linear_kernel<BN><<<grid, gdn::gemm::NT, S::SMEM, st>>>(tm_x, tm_w, a);
    return cudaGetLastError();
}

// Tile width of the one-CTA form: fewest (waves x (BN + a fixed per-tile cost));
// ties go to the wider tile.
int pick_bn(int64_t M, int N, int sms) {
    static const int cand[] = {256, 128};
    const int64_t mb = (M + gdn::gemm::BM - 1) / gdn::gemm::BM;
    int best = 256;
    int64_t best_cost = -1;
    for (int bn : cand) {
        const int64_t tiles = mb * ((N + bn - 1) / bn);
        const int64_t cost = (tiles + sms - 1) / sms * (bn + 32);
        if (best_cost < 0 || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

// Pair form (2-CTA clusters, M = 256 pair tiles).  The number of clusters that
// fit at once is asked of the runtime once per device and width.
template <int BN>
cudaError_t launch_linear_pair(const void* x, const void* w, gdn::gemm::Args a, int variant, cudaStream_t st) {
    using S = gdn::gemm::Shape2<BN>;
    CUtensorMap tm_x, tm_w;
    if (!kmajor_map(&tm_x, x, a.M, a.K, gdn::gemm::BM) || !kmajor_map(&tm_w, w, a.N, a.K, BN / 2))
        return cudaErrorInvalidValue;
    a.n_blocks = (a.N + BN - 1) / BN;
    const int64_t m_pairs = (a.M + 2 * gdn::gemm::BM - 1) / (2 * gdn::gemm::BM);
    a.tiles = m_pairs * a.n_blocks;
    cudaError_t e = ensure_smem(gdn::gemm::linear_pair_kernel<BN>, variant, S::SMEM);
    if (e != cudaSuccess) return e;
    static int clusters[64];
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    int n_cl = dev < 64 ? clusters[dev] : 0;
    if (n_cl <= 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)std::max(1, sm_count() / 2), 1, 1);
        cfg.blockDim = dim3(gdn::gemm::NT, 1, 1);
        cfg.dynamicSmemBytes = S::SMEM;
        if (cudaOccupancyMaxActiveClusters(&n_cl, gdn::gemm::linear_pair_kernel<BN>, &cfg) != cudaSuccess ||
            n_cl <= 0) {
            (void)cudaGetLastError();
            n_cl = std::max(1, sm_count() / 2);
        }
        if (dev < 64) clusters[dev] = n_cl;
    }
    const int pairs = (int)std::min<int64_t>(a.tiles, n_cl);
    gdn::gemm::linear_pair_kernel<BN><<<2 * pairs, gdn::gemm::NT, S::SMEM, st>>>(tm_x, tm_w, a);
    return cudaGetLastError();
}

// Pair tile width: fewest waves x (time of one k-block), over the MMA widths,
// with ~74 pairs in flight on 148 SMs.  Measured on B200 the pair kernel is
// bound by the operand bytes each SM loads from L2 per k-block (16 KiB of A plus
// BN/2 rows of 128 B of B, ~90 GB/s per SM), and at the widest tiles by the MMA
// rate (~2.1 x BN in the same units): time ~ max(256 + BN, 17 BN / 8).
int pick_bn_pair(int64_t M, int N, int pairs) {
    static const int cand[] = {256, 224, 208, 192, 160, 144, 128};
    const int64_t mp = (M + 2 * gdn::gemm::BM - 1) / (2 * gdn::gemm::BM);
    int best = 256;
    int64_t best_cost = -1;
    for (int bn : cand) {
        const int64_t tiles = mp * ((N + bn - 1) / bn);
        const int64_t cost = (tiles + pairs - 1) / pairs * std::max<int64_t>(256 + bn, 17 * bn / 8);
        if (best_cost < 0 || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

gdn_status run_linear(const void* x, const void* w, int64_t M, int32_t N, int32_t K, const gdn_out_segment* segs,
                      int32_t n_segs, void* stream) {
    if (M < 0 || N <= 0 || K <= 0 || !segs || n_segs <= 0) return GDN_ERR_INVALID_ARG;
    if (n_segs > GDN_LINEAR_MAX_SEGMENTS) return GDN_ERR_UNSUPPORTED;
    if (N % 8 != 0 || K % 8 != 0) return GDN_ERR_UNSUPPORTED;
    if (M == 0) return GDN_OK;
    if (!x || !w || !aligned(x, 16) || !aligned(w, 16)) return GDN_ERR_INVALID_ARG;
    if ((M + gdn::gemm::BM - 1) / gdn::gemm::BM > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    gdn::gemm::Args a;
    a.M = M;
    a.N = N;
    a.K = K;
    a.m_blocks = (int)((M + gdn::gemm::BM - 1) / gdn::gemm::BM);
    a.n_segs = n_segs;
    int n0 = 0;
    for (int i = 0; i < n_segs; ++i) {
        const gdn_out_segment& g = segs[i];
        if (!g.dst || !aligned(g.dst, 16) || g.width <= 0 || g.width % 8 != 0) return GDN_ERR_INVALID_ARG;
        a.seg[i].dst = static_cast<__nv_bfloat16*>(g.dst);
        a.seg[i].n0 = n0;
        a.seg[i].width = g.width;
        n0 += g.width;
        if (n0 > N) return GDN_ERR_INVALID_ARG;
    }
    if (n0 != N) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (M > gdn::gemm::BM) {
        // pairs of CTAs once there are two 128-row halves to give them
        switch (pick_bn_pair(M, N, std::max(1, sm_count() / 2))) {
            case 256: e = launch_linear_pair<256>(x, w, a, 25, st); break;
            case 224: e = launch_linear_pair<224>(x, w, a, 26, st); break;
            case 208: e = launch_linear_pair<208>(x, w, a, 27, st); break;
            case 192: e = launch_linear_pair<192>(x, w, a, 28, st); break;
            case 160: e = launch_linear_pair<160>(x, w, a, 29, st); break;
            case 144: e = launch_linear_pair<144>(x, w, a, 30, st); break;
            default: e = launch_linear_pair<128>(x, w, a, 31, st); break;
        }
        return cuda_status(e);
    }
    // one CTA per 128-row tile for short inputs (decode-sized batches)
    if (pick_bn(M, N, sm_count()) == 256) e = launch_linear<256>(x, w, a, 20, st);
    else e = launch_linear<128>(x, w, a, 24, st);
    return cuda_status(e);
}

// Prefill, split in its two stages so that context-parallel prefill can run the
// chunk scan more than once over one set of intra-chunk records.
//   stage A: chunk offsets and the check of cu_seqlens, conv + SiLU + L2 norm
//            into the workspace, conv-state update, intra-chunk records
//   stage B: the chunk scan from rec_state (in/out), then the gated norm into out
// Set-up first: nothing is launched unless the tensor maps encode and the
// kernels' shared-memory opt-ins succeed.  The conv, intra-chunk, scan and norm
// launches each take a range of global chunks, so that a pipelined call
// (launch_prefill) can run them range by range on three streams.
template <typename TA>
struct StageA {
    ConvArgs ca;
    gdn::intra::Args ia;
    CUtensorMap tm_q, tm_k, tm_cq, tm_ck, tm_cv;
    bool tiled;
    int n_slices, cblocks;
    int64_t max_chunks;
    decltype(&gdn::conv_tile_kernel<16>) k_conv;
};

template <typename TA>
cudaError_t prepare_stage_a(const gdn_config* c, const gdn_weights* w, const void* q, const void* k, const void* v,
                            const void* a, const void* b, void* conv_state, const int32_t* cu, int n_seqs,
                            int64_t T, void* ws, StageA<TA>* S) {
    const Layout L = workspace_layout(c, T, n_seqs);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    int32_t* flags = reinterpret_cast<int32_t*>(wsb + L.flags_off);
    int32_t* chunk_off = reinterpret_cast<int32_t*>(wsb + L.coff_off);
    ConvArgs& ca = S->ca;
    ca.q = q; ca.k = k; ca.v = v;
    ca.conv_w = w->conv_weight;
    ca.conv_state = conv_state;
    ca.cu = cu;
    ca.n_seqs = n_seqs;
    ca.T = T;
    ca.Hk = c->n_k_heads; ca.Hv = c->n_v_heads; ca.dk = c->d_k; ca.dv = c->d_v;
    ca.l2_eps = c->l2_eps;
    ca.qh = reinterpret_cast<__half*>(wsb + L.q_off);
    ca.kh = reinterpret_cast<__half*>(wsb + L.k_off);
    ca.vh = reinterpret_cast<__half*>(wsb + L.v_off);
    ca.flags = flags;
    ca.chunk_off = chunk_off;
    ca.g_lo = 0;
    ca.g_hi = 0x7fffffff;
    auto k_intra = gdn::intra::gdn_intra_kernel<TA>;
    cudaError_t e = ensure_smem(k_intra, 4 + (sizeof(TA) == 2 ? 0 : 1), gdn::intra::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int Hk = c->n_k_heads, Hv = c->n_v_heads;
    if (!head_tile_map(&S->tm_q, ca.qh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c->d_k, Hk, T) ||
        !head_tile_map(&S->tm_k, ca.kh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c->d_k, Hk, T))
        return cudaErrorInvalidValue;
    const int Ctot = 2 * c->n_k_heads * c->d_k + c->n_v_heads * c->d_v;
    S->cblocks = (Ctot / 8 + gdn::kConvThreads - 1) / gdn::kConvThreads;
    S->max_chunks = (T + gdn::intra::C - 1) / gdn::intra::C + n_seqs;
    if ((T + gdn::kConvRun - 1) / gdn::kConvRun > 0x7fffffff || S->max_chunks * Hk > 0x7fffffff)
        return cudaErrorInvalidValue;

    // the tiled conv for bf16 activations whose q, k and v widths are multiples of its slice
    const int Cq = c->n_k_heads * c->d_k, Cv = c->n_v_heads * c->d_v;
    S->tiled = sizeof(TA) == 2 && Cq % gdn::ctile::CH == 0 && Cv % gdn::ctile::CH == 0;
    S->n_slices = Ctot / gdn::ctile::CH;
    S->k_conv = c->d_k == 32 ? gdn::conv_tile_kernel<4> : c->d_k == 64 ? gdn::conv_tile_kernel<8>
                                                                        : gdn::conv_tile_kernel<16>;
    if (S->tiled) {
        S->tiled = conv_tile_map(&S->tm_cq, q, Cq, T) && conv_tile_map(&S->tm_ck, k, Cq, T) &&
                   conv_tile_map(&S->tm_cv, v, Cv, T);
        e = ensure_smem(S->k_conv, 12 + (c->d_k == 32 ? 0 : c->d_k == 64 ? 1 : 2), gdn::ctile::SMEM_BYTES);
        if (e != cudaSuccess) return e;
    }

    gdn::intra::Args& ia = S->ia;
    ia.a = a; ia.b = b;
    ia.A_log = w->A_log; ia.dt_bias = w->dt_bias;
    ia.cu = cu; ia.chunk_off = chunk_off; ia.flags = flags; ia.n_seqs = n_seqs;
    ia.Hk = Hk; ia.Hv = Hv;
    ia.rec = wsb + L.rec_off;
    ia.g_lo = 0;
    return cudaSuccess;
}

// The chunk table and the check of cu_seqlens: the first kernel of every prefill.
template <typename TA>
cudaError_t launch_chunk_offsets(const StageA<TA>& S, cudaStream_t st) {
    gdn::intra::chunk_offsets_kernel<<<1, 1024, 0, st>>>(S.ca.cu, S.ca.n_seqs, S.ca.T, S.max_chunks,
                                                         const_cast<int32_t*>(S.ia.chunk_off), S.ca.flags);
    return cudaGetLastError();
}

// Conv + SiLU + L2 norm of the tokens of global chunks [g_lo, g_hi) (see conv_tile_range).
template <typename TA>
cudaError_t launch_conv(const StageA<TA>& S, int64_t g_lo, int64_t g_hi, cudaStream_t st) {
    ConvArgs ca = S.ca;
    ca.g_lo = g_lo;
    ca.g_hi = g_hi;
    const int64_t chunks = (g_hi < S.max_chunks ? g_hi : S.max_chunks) - g_lo;
    const int64_t all_tiles = (S.ca.T + 31) / 32;
    int64_t tiles = 2 * chunks + 1;   // 32-token tiles that start in the range's tokens (<= 64 per chunk)
    tiles = tiles < all_tiles ? tiles : all_tiles;
    if (tiles <= 0) return cudaSuccess;
    if (S.tiled) {
        int64_t parts = (int64_t)2 * sm_count() / S.n_slices;
        parts = parts < 1 ? 1 : parts > tiles ? tiles : parts;
        S.k_conv<<<(unsigned)(S.n_slices * parts), gdn::ctile::NT, gdn::ctile::SMEM_BYTES, st>>>(
            S.tm_cq, S.tm_ck, S.tm_cv, ca, (int)parts);
    } else {
        gdn::conv_silu_norm_kernel<TA><<<dim3((unsigned)tiles, S.cblocks), gdn::kConvThreads, 0, st>>>(ca);
    }
    return cudaGetLastError();
}

// conv_state <- the last 3 inputs of each sequence: after every conv launch of the call.
template <typename TA>
cudaError_t launch_conv_state(const StageA<TA>& S, cudaStream_t st) {
    const int Ctot = 2 * S.ca.Hk * S.ca.dk + S.ca.Hv * S.ca.dv;
    gdn::conv_state_update_kernel<TA><<<dim3(S.ca.n_seqs, (Ctot + 255) / 256), 256, 0, st>>>(
        S.ca, const_cast<void*>(S.ca.conv_state));
    return cudaGetLastError();
}

// Intra-chunk records of global chunks [g_lo, g_hi).
template <typename TA>
cudaError_t launch_intra(const StageA<TA>& S, int64_t g_lo, int64_t g_hi, cudaStream_t st) {
    gdn::intra::Args ia = S.ia;
    ia.g_lo = (int32_t)g_lo;
    const int64_t n = (g_hi < S.max_chunks ? g_hi : S.max_chunks) - g_lo;
    if (n <= 0) return cudaSuccess;
    gdn::intra::gdn_intra_kernel<TA><<<(unsigned)(n * S.ia.Hk), gdn::intra::NT, gdn::intra::SMEM_BYTES, st>>>(
        S.tm_q, S.tm_k, ia);
    return cudaGetLastError();
}

// Stage A over every chunk on `st`.  The conv-state update (which must follow the
// conv's reads of the old state) runs on a side stream beside the intra kernel.
// Once the side stream has been forked, *join receives an event recorded after
// its work, on every path, error paths included; the caller's stream waits on
// it before the call ends.
template <typename TA>
cudaError_t launch_stage_a(const gdn_config* c, const gdn_weights* w, const void* q, const void* k, const void* v,
                           const void* a, const void* b, void* conv_state, const int32_t* cu, int n_seqs,
                           int64_t T, void* ws, cudaStream_t st, cudaEvent_t* join) {
    *join = nullptr;
    StageA<TA> S;
    cudaError_t e = prepare_stage_a<TA>(c, w, q, k, v, a, b, conv_state, cu, n_seqs, T, ws, &S);
    if (e != cudaSuccess) return e;
    cudaStream_t aux = side_stream(3);
    cudaEvent_t* ev = thread_events(kEvStageA, 2);   // conv done (fork), side work done (join)
    if (!aux || !ev) return cudaErrorNotReady;
    if ((e = launch_chunk_offsets(S, st)) != cudaSuccess) return e;
    if ((e = launch_conv(S, 0, S.max_chunks, st)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(ev[0], st)) != cudaSuccess || (e = cudaStreamWaitEvent(aux, ev[0], 0)) != cudaSuccess)
        return e;
    // aux is forked: from here on it is joined back whatever happens
    const cudaError_t e_side = launch_conv_state(S, aux);
    if ((e = cudaEventRecord(ev[1], aux)) != cudaSuccess) return e;
    *join = ev[1];
    if (e_side != cudaSuccess) return e_side;
    return launch_intra(S, 0, S.max_chunks, st);
}

// The caller's stream waits for stage A's side work.
cudaError_t join_side(cudaEvent_t join, cudaStream_t st, cudaError_t prior) {
    if (!join) return prior;
    const cudaError_t e = cudaStreamWaitEvent(st, join, 0);
    return prior != cudaSuccess ? prior : e;
}

// The chunk scan over the records of stage A, reading V through `v_src` (the
// workspace's v^, or a zero block whose map reads zeros past its 64 rows).
struct ScanSetup {
    CUtensorMap tm_v, tm_k;
    gdn::scan::Args sa;
    unsigned grid;
    decltype(&gdn::scan::gdn_scan_kernel<float, float>) kernel;   // (every instance has this signature)
};

template <typename TO>
cudaError_t prepare_scan(const gdn_config* c, const void* v_src, int64_t v_rows, void* rec_state, const int32_t* cu,
                         int n_seqs, int64_t T, void* ws, void* o_dst, ScanSetup* S) {
    const Layout L = workspace_layout(c, T, n_seqs);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    auto k_scan = c->state_dtype == GDN_BF16 ? gdn::scan::gdn_scan_kernel<TO, __nv_bfloat16>
                                             : gdn::scan::gdn_scan_kernel<TO, float>;
    cudaError_t e = ensure_smem(k_scan, 16 + (sizeof(TO) == 2 ? 0 : 1) + (c->state_dtype == GDN_BF16 ? 2 : 0),
                                gdn::scan::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    S->kernel = k_scan;
    if (!head_tile_map(&S->tm_v, v_src, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c->d_v, c->n_v_heads, v_rows) ||
        !head_tile_map(&S->tm_k, wsb + L.k_off, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c->d_k, c->n_k_heads, T))
        return cudaErrorInvalidValue;
    gdn::scan::Args& sa = S->sa;
    sa.rec_state = rec_state;
    sa.carry = L.total > L.carry_off ? reinterpret_cast<float*>(wsb + L.carry_off) : nullptr;
    sa.g_lo = 0;
    sa.g_hi = 0x7fffffff;
    sa.final_launch = 1;
    sa.cu = cu;
    sa.chunk_off = reinterpret_cast<int32_t*>(wsb + L.coff_off);
    sa.flags = reinterpret_cast<int32_t*>(wsb + L.flags_off);
    sa.rec = wsb + L.rec_off;
    sa.o = o_dst ? o_dst : wsb + L.o_off;
    sa.Hk = c->n_k_heads; sa.Hv = c->n_v_heads; sa.dk = c->d_k; sa.dv = c->d_v;
    S->grid = (unsigned)n_seqs * c->n_v_heads;
    return cudaSuccess;
}

// The scan over global chunks [g_lo, g_hi) of every chain; `final` for the call's
// last scan launch, which leaves the final states in rec_state.
cudaError_t launch_scan_range(const ScanSetup& S, int64_t g_lo, int64_t g_hi, bool final, cudaStream_t st) {
    gdn::scan::Args sa = S.sa;
    sa.g_lo = (int32_t)g_lo;
    sa.g_hi = (int32_t)(g_hi < 0x7fffffff ? g_hi : 0x7fffffff);
    sa.final_launch = final ? 1 : 0;
    S.kernel<<<S.grid, gdn::scan::NT, gdn::scan::SMEM_BYTES, st>>>(S.tm_v, S.tm_k, sa);
    return cudaGetLastError();
}

template <typename TO>
cudaError_t launch_scan(const gdn_config* c, const void* v_src, int64_t v_rows, void* rec_state, const int32_t* cu,
                        int n_seqs, int64_t T, void* ws, cudaStream_t st, void* o_dst = nullptr) {
    ScanSetup S;
    const cudaError_t e = prepare_scan<TO>(c, v_src, v_rows, rec_state, cu, n_seqs, T, ws, o_dst, &S);
    return e != cudaSuccess ? e : launch_scan_range(S, 0, 0x7fffffff, true, st);
}

struct NormSetup {
    CUtensorMap tm_z;
    gdn::norm::Args na;
    int64_t ctas, max_chunks;
};

template <typename TA, typename TO>
cudaError_t prepare_norm(const gdn_config* c, const gdn_weights* w, const void* z, const int32_t* cu, int n_seqs,
                         int64_t T, void* out, void* ws, NormSetup* S) {
    const Layout L = workspace_layout(c, T, n_seqs);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    cudaError_t e = ensure_smem(gdn::norm::gdn_gated_norm_kernel<TA, TO>,
                                8 + (sizeof(TA) == 4 ? 2 : 0) + (sizeof(TO) == 4 ? 1 : 0),
                                gdn::norm::smem_bytes<TA, TO>());
    if (e != cudaSuccess) return e;
    const int Hv = c->n_v_heads;
    if (!z_rows_map(&S->tm_z, z, sizeof(TA) == 2, Hv * c->d_v, c->d_v, T)) return cudaErrorInvalidValue;
    S->max_chunks = (T + gdn::intra::C - 1) / gdn::intra::C + n_seqs;
    gdn::norm::Args& na = S->na;
    na.o = wsb + L.o_off; na.norm_w = w->norm_weight;
    na.cu = cu; na.chunk_off = reinterpret_cast<int32_t*>(wsb + L.coff_off); na.out = out;
    na.flags = reinterpret_cast<int32_t*>(wsb + L.flags_off);
    na.n_seqs = n_seqs; na.Hv = Hv; na.dv = c->d_v; na.eps = c->norm_eps;
    na.g_lo = 0;
    na.g_hi = 0x7fffffff;
    S->ctas = (int64_t)sm_count() * (232448 / (int64_t)gdn::norm::smem_bytes<TA, TO>());
    return cudaSuccess;
}

// The gated norm of the tiles of global chunks [g_lo, g_hi).
template <typename TA, typename TO>
cudaError_t launch_norm_range(const NormSetup& S, int64_t g_lo, int64_t g_hi, cudaStream_t st) {
    gdn::norm::Args na = S.na;
    na.g_lo = (int32_t)g_lo;
    na.g_hi = (int32_t)(g_hi < 0x7fffffff ? g_hi : 0x7fffffff);
    const int64_t tiles = ((g_hi < S.max_chunks ? g_hi : S.max_chunks) - g_lo) * na.Hv;
    if (tiles <= 0) return cudaSuccess;
    const int64_t ctas = S.ctas < tiles ? S.ctas : tiles;
    gdn::norm::gdn_gated_norm_kernel<TA, TO>
        <<<(unsigned)ctas, gdn::norm::NT, gdn::norm::smem_bytes<TA, TO>(), st>>>(S.tm_z, na);
    return cudaGetLastError();
}

template <typename TA, typename TO>
cudaError_t launch_norm(const gdn_config* c, const gdn_weights* w, const void* z, const int32_t* cu, int n_seqs,
                        int64_t T, void* out, void* ws, cudaStream_t st) {
    NormSetup S;
    const cudaError_t e = prepare_norm<TA, TO>(c, w, z, cu, n_seqs, T, out, ws, &S);
    return e != cudaSuccess ? e : launch_norm_range<TA, TO>(S, 0, S.max_chunks, st);
}

// A whole prefill.  One range: stage A then stage B on `st`.  Several ranges
// (seg_plan): a pipeline over three streams, ordered by events only.
//   st (the caller's):   chunk offsets; for each range s: conv(s), intra(s)
//   side 4 (priority):   scan(s) after intra(s) and scan(s-1)
//   side 5:              norm(s) after scan(s) and after the last conv
//   side 3:              the conv-state update after the last conv
// Intra(s) needs the conv output of range s and of the tile that range s-1 ends
// with, both before it on `st`; scan(s) carries each chain's fp32 state to
// scan(s+1) through the workspace.  Nothing the caller sees is written before
// the last conv has checked its range: out is written by the norms, which wait
// for it; conv_state by the update, which waits for it; rec_state by the last
// scan, which follows the last intra on `st` (the carry holds the states of the
// chains that end earlier until then).  A call whose checks fail therefore
// leaves out and the states as they were.  Every side stream that has been
// forked is joined back to `st` on every path.
// 2-D tensor map over row-major [rows][128] bf16 with boxes of 64 columns x box_rows,
// 128-byte swizzle (the split chain's o^P tiles and bf16 start state).
bool rows128_map(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {128 * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The split chain (split_mode; one sequence, bf16 activations and output, fp32 state):
//   st:      stage A (conv-state update on its side stream), the start states of the
//            second half (zero and identity) and the zero v block, the first half's scan
//            (its end state into the carry), its end state to bf16, then (after the two
//            side scans) the second half's correction and gated norm (fixup.cuh), and the
//            fold of the end state into rec_state;
//   side 5:  the first half's gated norm, after its scan;
//   side 4:  the second half scanned from zero (S_loc; o^loc tiles);
//   side 0:  the second half scanned from the identity with V = 0 (the transition P;
//            o^P tiles).
// The three scans take 48 SMs each at the same time.  Nothing the caller sees is
// written before every device check has passed (every kernel reads the check word).
template <typename TA, typename TO>
cudaError_t launch_prefill_split(const gdn_config* c, const gdn_weights* w, const void* q, const void* k,
                                 const void* v, const void* a, const void* b, const void* z, void* conv_state,
                                 void* rec_state, const int32_t* cu, int64_t T, void* out, void* ws, cudaStream_t st) {
    const Layout L = workspace_layout(c, T, 1);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    const int Hv = c->n_v_heads, d = c->d_k;
    const int64_t chunks = (T + gdn::kChunk - 1) / gdn::kChunk, mid = chunks / 2;
    const int64_t per = (int64_t)Hv * d * d;
    float* C0 = reinterpret_cast<float*>(wsb + L.carry_off);
    float* summ = reinterpret_cast<float*>(wsb + L.summ_off);   // [P | S_loc]
    __nv_bfloat16* s0b = reinterpret_cast<__nv_bfloat16*>(wsb + L.s0b_off);
    const int32_t* flags = reinterpret_cast<const int32_t*>(wsb + L.flags_off);

    StageA<TA> A;
    ScanSetup B0, B1, B2;
    NormSetup N;
    CUtensorMap tm_p, tm_s;
    cudaError_t e = prepare_stage_a<TA>(c, w, q, k, v, a, b, conv_state, cu, 1, T, ws, &A);
    if (e == cudaSuccess)
        e = prepare_scan<TO>(c, wsb + L.v_off, T, rec_state, cu, 1, T, ws, nullptr, &B0);
    if (e == cudaSuccess) e = prepare_scan<TO>(c, wsb + L.v_off, T, summ + per, cu, 1, T, ws, nullptr, &B1);
    if (e == cudaSuccess) e = prepare_scan<TO>(c, wsb + L.zv_off, gdn::intra::C, summ, cu, 1, T, ws, wsb + L.op_off, &B2);
    if (e == cudaSuccess) e = prepare_norm<TA, TO>(c, w, z, cu, 1, T, out, ws, &N);
    if (e == cudaSuccess)
        e = ensure_smem(gdn::fix::gdn_fixup_norm_kernel, 6, gdn::fix::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (!rows128_map(&tm_p, wsb + L.op_off, (int64_t)A.max_chunks * Hv * 64, 64) ||
        !rows128_map(&tm_s, s0b, (int64_t)Hv * 128, 128))
        return cudaErrorInvalidValue;
    B0.sa.carry = C0;                        // the first half's end state
    B1.sa.carry = summ + per;                // S_loc: starts at zero, ends there
    B2.sa.carry = summ;                      // P: starts at the identity, ends there
    cudaStream_t side[3] = {side_stream(4), side_stream(0), side_stream(5)};
    // start states ready; the two side scans done; the first half's scan done; its norm done
    cudaEvent_t* ev = thread_events(kEvSplit, 5);
    if (!side[0] || !side[1] || !side[2] || !ev) return cudaErrorNotReady;

    cudaEvent_t join = nullptr;   // the conv-state update's side stream
    cudaStream_t aux = side_stream(3);
    cudaEvent_t* evA = thread_events(kEvStageA, 2);
    if (!aux || !evA) return cudaErrorNotReady;
    e = launch_chunk_offsets(A, st);
    if (e == cudaSuccess) e = launch_conv(A, 0, A.max_chunks, st);
    if (e == cudaSuccess && (e = cudaEventRecord(evA[0], st)) == cudaSuccess &&
        (e = cudaStreamWaitEvent(aux, evA[0], 0)) == cudaSuccess) {
        const cudaError_t e_side = launch_conv_state(A, aux);
        if ((e = cudaEventRecord(evA[1], aux)) == cudaSuccess) join = evA[1];
        if (e == cudaSuccess) e = e_side;
    }
    if (e == cudaSuccess) e = launch_intra(A, 0, A.max_chunks, st);
    if (e == cudaSuccess) {
        gdn::fix::split_init_kernel<<<(unsigned)std::min<int64_t>((2 * per + 255) / 256, 1024), 256, 0, st>>>(
            summ, Hv, d, flags);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess)
        e = cudaMemsetAsync(wsb + L.zv_off, 0, (size_t)gdn::intra::C * Hv * c->d_v * sizeof(__half), st);
    bool forked[3] = {false, false, false};
    if (e == cudaSuccess) e = cudaEventRecord(ev[0], st);
    for (int i = 0; i < 2 && e == cudaSuccess; i++) {
        if ((e = cudaStreamWaitEvent(side[i], ev[0], 0)) != cudaSuccess) break;
        forked[i] = true;
        e = launch_scan_range(i == 0 ? B1 : B2, mid, 0x7fffffff, false, side[i]);
        const cudaError_t r = cudaEventRecord(ev[1 + i], side[i]);
        if (e == cudaSuccess) e = r;
    }
    if (e == cudaSuccess) e = launch_scan_range(B0, 0, mid, false, st);
    // the first half's norm beside the second half's scans
    if (e == cudaSuccess && (e = cudaEventRecord(ev[3], st)) == cudaSuccess &&
        (e = cudaStreamWaitEvent(side[2], ev[3], 0)) == cudaSuccess) {
        forked[2] = true;
        e = launch_norm_range<TA, TO>(N, 0, mid, side[2]);
        const cudaError_t r = cudaEventRecord(ev[4], side[2]);
        if (e == cudaSuccess) e = r;
    }
    if (e == cudaSuccess) {
        gdn::fix::state_to_bf16_kernel<<<(unsigned)std::min<int64_t>((per / 4 + 255) / 256, 1024), 256, 0, st>>>(
            C0, s0b, per, flags);
        e = cudaGetLastError();
    }
    for (int i = 0; i < 2; i++) {   // join the side scans, whatever happened above
        if (!forked[i]) continue;
        const cudaError_t r = cudaStreamWaitEvent(st, ev[1 + i], 0);
        if (e == cudaSuccess) e = r;
    }
    if (e == cudaSuccess) {
        gdn::fix::Args fa;
        fa.o_loc = reinterpret_cast<const __nv_bfloat16*>(wsb + L.o_off);
        fa.z = static_cast<const __nv_bfloat16*>(z);
        fa.norm_w = w->norm_weight;
        fa.out = static_cast<__nv_bfloat16*>(out);
        fa.flags = flags;
        fa.T = T;
        fa.Hv = Hv;
        fa.c_lo = (int)mid;
        fa.c_hi = (int)chunks;
        fa.eps = c->norm_eps;
        const int64_t pairs = (chunks - mid + 1) / 2;
        gdn::fix::gdn_fixup_norm_kernel<<<(unsigned)(pairs * Hv), gdn::fix::NT, gdn::fix::SMEM_BYTES, st>>>(tm_p, tm_s,
                                                                                                         fa);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        gdn::cp::fold_kernel<<<(unsigned)(Hv * (d / gdn::cp::CR)), gdn::cp::CT, 0, st>>>(
            C0, summ, 1, Hv, d, static_cast<float*>(rec_state), flags);
        e = cudaGetLastError();
    }
    if (forked[2]) {   // the first half's norm
        const cudaError_t r = cudaStreamWaitEvent(st, ev[4], 0);
        if (e == cudaSuccess) e = r;
    }
    return join_side(join, st, e);
}

template <typename TA, typename TO>
cudaError_t launch_prefill(const gdn_config* c, const gdn_weights* w, const void* q, const void* k,
                           const void* v, const void* a, const void* b, const void* z, void* conv_state,
                           void* rec_state, const int32_t* cu, int n_seqs, int64_t T, void* out,
                           void* ws, cudaStream_t st) {
    if (sizeof(TA) == 2 && sizeof(TO) == 2 && split_mode(c, T, n_seqs))
        return launch_prefill_split<TA, TO>(c, w, q, k, v, a, b, z, conv_state, rec_state, cu, T, out, ws, st);
    const Layout L = workspace_layout(c, T, n_seqs);
    const SegPlan P = seg_plan(c, T, n_seqs);
    if (P.n == 1) {
        cudaEvent_t join = nullptr;
        cudaError_t e = launch_stage_a<TA>(c, w, q, k, v, a, b, conv_state, cu, n_seqs, T, ws, st, &join);
        if (e == cudaSuccess)
            e = launch_scan<TO>(c, static_cast<uint8_t*>(ws) + L.v_off, T, rec_state, cu, n_seqs, T, ws, st);
        if (e == cudaSuccess) e = launch_norm<TA, TO>(c, w, z, cu, n_seqs, T, out, ws, st);
        return join_side(join, st, e);
    }
    StageA<TA> A;
    ScanSetup B;
    NormSetup N;
    cudaError_t e = prepare_stage_a<TA>(c, w, q, k, v, a, b, conv_state, cu, n_seqs, T, ws, &A);
    if (e == cudaSuccess)
        e = prepare_scan<TO>(c, static_cast<uint8_t*>(ws) + L.v_off, T, rec_state, cu, n_seqs, T, ws, nullptr, &B);
    if (e == cudaSuccess) e = prepare_norm<TA, TO>(c, w, z, cu, n_seqs, T, out, ws, &N);
    if (e != cudaSuccess) return e;
    if (!B.sa.carry) return cudaErrorInvalidValue;
    cudaStream_t side[3] = {side_stream(4), side_stream(5), side_stream(3)};   // scan, norm, conv state
    // events: [0, n) intra(s) done; [n, 2n) scan(s) done; 2n: last conv done; 2n+1 .. 2n+3: joins
    const int n = P.n;
    cudaEvent_t* ev = thread_events(kEvPipe, 2 * (size_t)n + 4);
    if (!side[0] || !side[1] || !side[2] || !ev) return cudaErrorNotReady;
    bool forked[3] = {false, false, false};
    auto fork = [&](int i, cudaEvent_t after) -> cudaError_t {
        const cudaError_t r = cudaStreamWaitEvent(side[i], after, 0);
        if (r == cudaSuccess) forked[i] = true;
        return r;
    };
    auto range_lo = [&](int s) -> int64_t { return P.lo[s]; };
    auto range_hi = [&](int s) -> int64_t { return s == n - 1 ? A.max_chunks : (int64_t)P.lo[s + 1]; };

    e = launch_chunk_offsets(A, st);
    for (int s = 0; s < n && e == cudaSuccess; s++) {
        if ((e = launch_conv(A, range_lo(s), range_hi(s), st)) != cudaSuccess) break;
        if (s == n - 1 && (e = cudaEventRecord(ev[2 * n], st)) != cudaSuccess) break;
        if ((e = launch_intra(A, range_lo(s), range_hi(s), st)) != cudaSuccess) break;
        if ((e = cudaEventRecord(ev[s], st)) != cudaSuccess) break;
        if ((e = fork(0, ev[s])) != cudaSuccess) break;
        if ((e = launch_scan_range(B, range_lo(s), range_hi(s), s == n - 1, side[0])) != cudaSuccess) break;
        if ((e = cudaEventRecord(ev[n + s], side[0])) != cudaSuccess) break;
    }
    if (e == cudaSuccess && (e = fork(2, ev[2 * n])) == cudaSuccess) e = launch_conv_state(A, side[2]);
    if (e == cudaSuccess) e = fork(1, ev[2 * n]);
    for (int s = 0; s < n && e == cudaSuccess; s++) {
        if ((e = cudaStreamWaitEvent(side[1], ev[n + s], 0)) != cudaSuccess) break;
        e = launch_norm_range<TA, TO>(N, range_lo(s), range_hi(s), side[1]);
    }
    for (int i = 0; i < 3; i++) {   // join every forked stream, whatever happened above
        if (!forked[i]) continue;
        cudaError_t r = cudaEventRecord(ev[2 * n + 1 + i], side[i]);
        if (r == cudaSuccess) r = cudaStreamWaitEvent(st, ev[2 * n + 1 + i], 0);
        if (e == cudaSuccess) e = r;
    }
    return e;
}

template <typename TA, typename TO, typename TS, int DK>
cudaError_t launch_decode_dk(const gdn::dec::Args& a, int n_seqs, cudaStream_t st) {
    const int G = a.Hv / a.Hk;
    const size_t smem = gdn::dec::smem_floats(DK, G, a.dv) * sizeof(float);
    auto kern = gdn::dec::gdn_decode_kernel<TA, TO, TS, DK>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)n_seqs * a.Hk, gdn::dec::NT, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename TA, typename TO, typename TS, int DK>
cudaError_t launch_decode_multi_dk(const gdn::dec::MultiArgs& m, cudaStream_t st) {
    const int G = m.a.Hv / m.a.Hk;
    const size_t smem = gdn::dec::smem_floats_multi(DK, G, m.a.dv, m.n_tok) * sizeof(float);
    auto kern = gdn::dec::gdn_decode_multi_kernel<TA, TO, TS, DK>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)m.n_seqs * m.a.Hk, gdn::dec::NT, smem, st>>>(m);
    return cudaGetLastError();
}

// The decode with the state streamed through shared memory (one or several tokens).
// Persistent: as many CTAs as fit at once (at most one per unit); shapes whose
// buffers do not fit in shared memory take the multi-token kernel instead.
template <typename TA, typename TO, typename TS, int DK>
cudaError_t launch_decode_stream_dk(const gdn::dec::MultiArgs& m_in, cudaStream_t st) {
    const int G = m_in.a.Hv / m_in.a.Hk;
    gdn::dec::MultiArgs m = m_in;
    // the deepest ring that lets two CTAs share an SM (228 KiB, 1 KiB reserved per CTA), else one
    auto smem_of = [&](int ns) { return gdn::dec::stream_smem_bytes<TA, TS, DK>(G, m.a.dv, m.n_tok, ns); };
    m.stages = gdn::dec::stream_stages<TS>();
    while (m.stages > 2 && 2 * (smem_of(m.stages) + 1024) > 233472) m.stages--;
    const size_t smem = smem_of(m.stages);
    if (smem > 232448) return launch_decode_multi_dk<TA, TO, TS, DK>(m, st);
    auto kern = gdn::dec::gdn_decode_stream_kernel<TA, TO, TS, DK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, gdn::dec::SNT, smem);
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)m.n_seqs * m.a.Hk;
    int64_t grid = (int64_t)(per_sm > 0 ? per_sm : 1) * sm_count();
    grid = grid < units ? grid : units;
    kern<<<(unsigned)grid, gdn::dec::SNT, smem, st>>>(m);
    return cudaGetLastError();
}

template <typename TA, typename TO, typename TS>
cudaError_t launch_decode_multi_ts(const gdn::dec::MultiArgs& m, cudaStream_t st) {
    switch (m.a.dk) {
        case 32: return launch_decode_stream_dk<TA, TO, TS, 32>(m, st);
        case 64: return launch_decode_stream_dk<TA, TO, TS, 64>(m, st);
        default: return launch_decode_stream_dk<TA, TO, TS, 128>(m, st);
    }
}
template <typename TA, typename TO>
cudaError_t launch_decode_multi(const gdn::dec::MultiArgs& m, bool bf16_state, cudaStream_t st) {
    return bf16_state ? launch_decode_multi_ts<TA, TO, __nv_bfloat16>(m, st)
                      : launch_decode_multi_ts<TA, TO, float>(m, st);
}

// One token: the fp32 state streams best through registers (gdn_decode_kernel,
// measured about 0.9 of the HBM copy rate at batch 256); the bf16 state, whose
// rows cost as many instructions for half the bytes, through the warp-specialised
// streamed kernel.
template <typename TA, typename TO, typename TS>
cudaError_t launch_decode_ts(const gdn::dec::Args& a, int n_seqs, cudaStream_t st) {
    if (sizeof(TS) == 4) {
        switch (a.dk) {
            case 32: return launch_decode_dk<TA, TO, TS, 32>(a, n_seqs, st);
            case 64: return launch_decode_dk<TA, TO, TS, 64>(a, n_seqs, st);
            default: return launch_decode_dk<TA, TO, TS, 128>(a, n_seqs, st);
        }
    }
    gdn::dec::MultiArgs m;
    m.a = a;
    m.n_tok = 1;
    m.state_snap = nullptr;
    m.conv_snap = nullptr;
    m.n_seqs = n_seqs;
    m.stages = 0;   // (chosen at launch)
    return launch_decode_multi_ts<TA, TO, TS>(m, st);
}
template <typename TA, typename TO>
cudaError_t launch_decode(const gdn::dec::Args& a, int n_seqs, bool bf16_state, cudaStream_t st) {
    return bf16_state ? launch_decode_ts<TA, TO, __nv_bfloat16>(a, n_seqs, st)
                      : launch_decode_ts<TA, TO, float>(a, n_seqs, st);
}

}  // namespace

extern "C" {

void gdn_config_default(gdn_config* cfg) {
    if (!cfg) return;
    cfg->n_k_heads = 16;
    cfg->n_v_heads = 48;
    cfg->d_k = 128;
    cfg->d_v = 128;
    cfg->conv_kernel = 4;
    cfg->chunk = 64;
    cfg->l2_eps = 1e-6f;
    cfg->norm_eps = 1e-6f;
    cfg->act_dtype = GDN_BF16;
    cfg->out_dtype = GDN_BF16;
    cfg->state_dtype = GDN_F32;
    cfg->prefill_segments = 0;
}

size_t gdn_prefill_workspace_size(const gdn_config* cfg, int64_t T_total, int32_t n_seqs) {
    if (check_config(cfg) != GDN_OK || T_total < 0 || n_seqs < 0) return 0;
    return workspace_layout(cfg, T_total, n_seqs).total;
}

int32_t gdn_prefill_segments(const gdn_config* cfg, int64_t T_total, int32_t n_seqs) {
    if (check_config(cfg) != GDN_OK || T_total < 0 || n_seqs < 0) return 0;
    if (split_mode(cfg, T_total, n_seqs)) return GDN_PREFILL_SPLIT;
    return seg_plan(cfg, T_total, n_seqs).n;
}

gdn_status gdn_prefill(const gdn_config* cfg, const gdn_weights* w, const void* q, const void* k,
                       const void* v, const void* a, const void* b, const void* z, void* conv_state,
                       void* rec_state, const int32_t* cu_seqlens, int32_t n_seqs, int64_t T_total,
                       void* out, void* workspace, size_t workspace_bytes, void* stream) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if ((s = check_weights(w)) != GDN_OK) return s;
    if (n_seqs < 0 || T_total < 0) return GDN_ERR_INVALID_ARG;
    if (T_total == 0 || n_seqs == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !z || !conv_state || !rec_state || !cu_seqlens || !out || !workspace)
        return GDN_ERR_INVALID_ARG;
    const void* a16[] = {q, k, v, z, out, rec_state};
    for (const void* p : a16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)n_seqs * cfg->n_v_heads > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (T_total > 0x7fffffffLL - 64) return GDN_ERR_UNSUPPORTED;   // token coordinates are int32
    if (workspace_bytes < workspace_layout(cfg, T_total, n_seqs).total) return GDN_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    const bool abf = cfg->act_dtype == GDN_BF16, obf = cfg->out_dtype == GDN_BF16;
    if (abf && obf)
        e = launch_prefill<__nv_bfloat16, __nv_bfloat16>(cfg, w, q, k, v, a, b, z, conv_state, rec_state,
                                                          cu_seqlens, n_seqs, T_total, out, workspace, st);
    else if (abf)
        e = launch_prefill<__nv_bfloat16, float>(cfg, w, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens,
                                                 n_seqs, T_total, out, workspace, st);
    else if (obf)
        e = launch_prefill<float, __nv_bfloat16>(cfg, w, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens,
                                                 n_seqs, T_total, out, workspace, st);
    else
        e = launch_prefill<float, float>(cfg, w, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens, n_seqs,
                                         T_total, out, workspace, st);
    return cuda_status(e);
}

gdn_status gdn_decode(const gdn_config* cfg, const gdn_weights* w, const void* q, const void* k,
                      const void* v, const void* a, const void* b, const void* z, void* conv_state,
                      void* rec_state, int32_t n_seqs, void* out, void* stream) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if ((s = check_weights(w)) != GDN_OK) return s;
    if (n_seqs < 0) return GDN_ERR_INVALID_ARG;
    if (n_seqs == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !z || !conv_state || !rec_state || !out) return GDN_ERR_INVALID_ARG;
    const void* a16[] = {q, k, v, z, out, rec_state};
    for (const void* p : a16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)n_seqs * cfg->n_k_heads > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    gdn::dec::Args da;
    da.q = q; da.k = k; da.v = v; da.a = a; da.b = b; da.z = z;
    da.conv_w = w->conv_weight; da.A_log = w->A_log; da.dt_bias = w->dt_bias; da.norm_w = w->norm_weight;
    da.conv_state = conv_state;
    da.rec_state = rec_state;
    da.out = out;
    da.Hk = cfg->n_k_heads; da.Hv = cfg->n_v_heads; da.dk = cfg->d_k; da.dv = cfg->d_v;
    da.l2_eps = cfg->l2_eps; da.norm_eps = cfg->norm_eps;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    const bool abf = cfg->act_dtype == GDN_BF16, obf = cfg->out_dtype == GDN_BF16;
    const bool sbf = cfg->state_dtype == GDN_BF16;
    if (abf && obf) e = launch_decode<__nv_bfloat16, __nv_bfloat16>(da, n_seqs, sbf, st);
    else if (abf) e = launch_decode<__nv_bfloat16, float>(da, n_seqs, sbf, st);
    else if (obf) e = launch_decode<float, __nv_bfloat16>(da, n_seqs, sbf, st);
    else e = launch_decode<float, float>(da, n_seqs, sbf, st);
    return cuda_status(e);
}

static_assert(gdn::dec::kMaxTok == GDN_DECODE_MULTI_MAX_TOKENS, "multi-token limit");

gdn_status gdn_decode_multi(const gdn_config* cfg, const gdn_weights* w, const void* q, const void* k,
                            const void* v, const void* a, const void* b, const void* z, void* conv_state,
                            void* rec_state, int32_t n_seqs, int32_t n_tok, void* out, void* state_snapshots,
                            void* conv_snapshots, void* stream) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if ((s = check_weights(w)) != GDN_OK) return s;
    if (n_seqs < 0 || n_tok < 0) return GDN_ERR_INVALID_ARG;
    if (n_tok > GDN_DECODE_MULTI_MAX_TOKENS) return GDN_ERR_UNSUPPORTED;
    if (n_seqs == 0 || n_tok == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !z || !conv_state || !rec_state || !out) return GDN_ERR_INVALID_ARG;
    const void* a16[] = {q, k, v, z, out, rec_state, state_snapshots};
    for (const void* p : a16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;   // null snapshots pass
    if ((int64_t)n_seqs * cfg->n_k_heads > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    gdn::dec::MultiArgs m;
    gdn::dec::Args& da = m.a;
    da.q = q; da.k = k; da.v = v; da.a = a; da.b = b; da.z = z;
    da.conv_w = w->conv_weight; da.A_log = w->A_log; da.dt_bias = w->dt_bias; da.norm_w = w->norm_weight;
    da.conv_state = conv_state;
    da.rec_state = rec_state;
    da.out = out;
    da.Hk = cfg->n_k_heads; da.Hv = cfg->n_v_heads; da.dk = cfg->d_k; da.dv = cfg->d_v;
    da.l2_eps = cfg->l2_eps; da.norm_eps = cfg->norm_eps;
    m.stages = 0;   // (chosen at launch)
    m.n_tok = n_tok;
    m.state_snap = state_snapshots;
    m.conv_snap = conv_snapshots;
    m.n_seqs = n_seqs;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    const bool abf = cfg->act_dtype == GDN_BF16, obf = cfg->out_dtype == GDN_BF16;
    const bool sbf = cfg->state_dtype == GDN_BF16;
    if (abf && obf) e = launch_decode_multi<__nv_bfloat16, __nv_bfloat16>(m, sbf, st);
    else if (abf) e = launch_decode_multi<__nv_bfloat16, float>(m, sbf, st);
    else if (obf) e = launch_decode_multi<float, __nv_bfloat16>(m, sbf, st);
    else e = launch_decode_multi<float, float>(m, sbf, st);
    return cuda_status(e);
}

gdn_status gdn_linear(const void* x, const void* w, int64_t M, int32_t N, int32_t K, const gdn_out_segment* segs,
                      int32_t n_segs, void* stream) {
    return run_linear(x, w, M, N, K, segs, n_segs, stream);
}

gdn_status gdn_in_proj(const gdn_config* cfg, const void* hidden, const void* w_in, int64_t T, int32_t d_model,
                       void* q, void* k, void* v, void* z, void* a, void* b, void* stream) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if (T < 0 || d_model <= 0) return GDN_ERR_INVALID_ARG;
    const int qk = cfg->n_k_heads * cfg->d_k, vz = cfg->n_v_heads * cfg->d_v, ab = cfg->n_v_heads;
    if (ab % 8 != 0) return GDN_ERR_UNSUPPORTED;
    const gdn_out_segment segs[6] = {{q, qk}, {k, qk}, {v, vz}, {z, vz}, {a, ab}, {b, ab}};
    return run_linear(hidden, w_in, T, 2 * qk + 2 * vz + 2 * ab, d_model, segs, 6, stream);
}

gdn_status gdn_out_proj(const gdn_config* cfg, const void* o, const void* w_out, int64_t T, int32_t d_model, void* y,
                        void* stream) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if (T < 0 || d_model <= 0) return GDN_ERR_INVALID_ARG;
    const gdn_out_segment seg = {y, d_model};
    return run_linear(o, w_out, T, d_model, cfg->n_v_heads * cfg->d_v, &seg, 1, stream);
}

// ---------------------------------------------------------------------------
// Context-parallel prefill (see cp.cuh)
// ---------------------------------------------------------------------------
static gdn_status cp_check(const gdn_config* cfg, int64_t T_seg) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if (T_seg < 1) return GDN_ERR_INVALID_ARG;
    if (cfg->state_dtype != GDN_F32 || cfg->d_k != cfg->d_v) return GDN_ERR_UNSUPPORTED;
    if (T_seg > 0x7fffffffLL - 64) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

size_t gdn_cp_workspace_size(const gdn_config* cfg, int64_t T_seg) {
    if (cp_check(cfg, T_seg) != GDN_OK) return 0;
    return cp_layout(cfg, T_seg).total;
}

gdn_status gdn_cp_local(const gdn_config* cfg, const gdn_weights* w, const void* q, const void* k, const void* v,
                        const void* a, const void* b, void* conv_state, int64_t T_seg, void* summary,
                        void* workspace, size_t workspace_bytes, void* stream) {
    gdn_status s = cp_check(cfg, T_seg);
    if (s != GDN_OK) return s;
    if ((s = check_weights(w)) != GDN_OK) return s;
    if (!q || !k || !v || !a || !b || !conv_state || !summary || !workspace) return GDN_ERR_INVALID_ARG;
    const void* a16[] = {q, k, v, summary};
    for (const void* p : a16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return GDN_ERR_INVALID_ARG;
    const CpLayout L = cp_layout(cfg, T_seg);
    if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    int32_t* cu = reinterpret_cast<int32_t*>(wsb + L.cu_off);
    const int Hv = cfg->n_v_heads, d = cfg->d_k;
    float* P = static_cast<float*>(summary);
    float* S_loc = P + (size_t)Hv * d * d;
    const bool abf = cfg->act_dtype == GDN_BF16, obf = cfg->out_dtype == GDN_BF16;
    gdn::cp::segment_cu_kernel<<<1, 32, 0, st>>>(cu, (int32_t)T_seg);
    cudaEvent_t side_join = nullptr;
    cudaError_t e = abf ? launch_stage_a<__nv_bfloat16>(cfg, w, q, k, v, a, b, conv_state, cu, 1, T_seg, workspace, st,
                                                        &side_join)
                        : launch_stage_a<float>(cfg, w, q, k, v, a, b, conv_state, cu, 1, T_seg, workspace, st,
                                                &side_join);
    if ((e = join_side(side_join, st, e)) != cudaSuccess) return cuda_status(e);
    // starting states: S_loc from zero, P from I; V = 0 for P: a zero block of 64
    // rows whose map reads zeros past it
    if ((e = cudaMemsetAsync(S_loc, 0, (size_t)Hv * d * d * sizeof(float), st)) != cudaSuccess) return cuda_status(e);
    if ((e = cudaMemsetAsync(wsb + L.zv_off, 0, L.total - L.zv_off, st)) != cudaSuccess) return cuda_status(e);
    gdn::cp::identity_kernel<<<(unsigned)std::max<int64_t>(1, std::min<int64_t>((int64_t)Hv * d * d / 256, 1024)), 256, 0,
                               st>>>(P, Hv, d);
    // The two scans read the same records and are independent, one CTA per head
    // each: the transition's runs on a side stream, forked from and joined back
    // to the caller's stream by events.
    cudaStream_t side = side_stream(0);
    cudaEvent_t* fj = thread_events(kEvCp, 2);
    if (!side || !fj) return cuda_status(cudaErrorNotReady);
    cudaEvent_t fork = fj[0], join = fj[1];
    cudaError_t e2 = cudaEventRecord(fork, st);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(side, fork, 0);
    if (e2 == cudaSuccess)
        e2 = obf ? launch_scan<__nv_bfloat16>(cfg, wsb + L.zv_off, gdn::intra::C, P, cu, 1, T_seg, workspace, side,
                                              wsb + L.o2_off)
                 : launch_scan<float>(cfg, wsb + L.zv_off, gdn::intra::C, P, cu, 1, T_seg, workspace, side,
                                      wsb + L.o2_off);
    if (e2 == cudaSuccess) e2 = cudaEventRecord(join, side);
    const void* vh = wsb + L.pre.v_off;
    e = obf ? launch_scan<__nv_bfloat16>(cfg, vh, T_seg, S_loc, cu, 1, T_seg, workspace, st)
            : launch_scan<float>(cfg, vh, T_seg, S_loc, cu, 1, T_seg, workspace, st);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, join, 0);
    return cuda_status(e != cudaSuccess ? e : e2);
}

gdn_status gdn_cp_finish(const gdn_config* cfg, const gdn_weights* w, const void* z, const void* summaries,
                         int32_t n_ranks, int32_t rank, const void* state_in, int64_t T_seg, void* out,
                         void* state_out, void* workspace, size_t workspace_bytes, void* stream) {
    gdn_status s = cp_check(cfg, T_seg);
    if (s != GDN_OK) return s;
    if ((s = check_weights(w)) != GDN_OK) return s;
    if (n_ranks < 1 || rank < 0 || rank >= n_ranks) return GDN_ERR_INVALID_ARG;
    if (!z || !summaries || !state_in || !out || !state_out || !workspace) return GDN_ERR_INVALID_ARG;
    const void* a16[] = {z, summaries, state_in, out, state_out};
    for (const void* p : a16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return GDN_ERR_INVALID_ARG;
    const CpLayout L = cp_layout(cfg, T_seg);
    if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    const int32_t* cu = reinterpret_cast<const int32_t*>(wsb + L.cu_off);
    const int Hv = cfg->n_v_heads, d = cfg->d_k;
    gdn::cp::fold_kernel<<<(unsigned)(Hv * (d / gdn::cp::CR)), gdn::cp::CT, 0, st>>>(
        static_cast<const float*>(state_in), static_cast<const float*>(summaries), rank, Hv, d,
        static_cast<float*>(state_out));
    const bool abf = cfg->act_dtype == GDN_BF16, obf = cfg->out_dtype == GDN_BF16;
    const void* vh = wsb + L.pre.v_off;
    cudaError_t e = obf ? launch_scan<__nv_bfloat16>(cfg, vh, T_seg, state_out, cu, 1, T_seg, workspace, st)
                        : launch_scan<float>(cfg, vh, T_seg, state_out, cu, 1, T_seg, workspace, st);
    if (e != cudaSuccess) return cuda_status(e);
    if (abf && obf) e = launch_norm<__nv_bfloat16, __nv_bfloat16>(cfg, w, z, cu, 1, T_seg, out, workspace, st);
    else if (abf) e = launch_norm<__nv_bfloat16, float>(cfg, w, z, cu, 1, T_seg, out, workspace, st);
    else if (obf) e = launch_norm<float, __nv_bfloat16>(cfg, w, z, cu, 1, T_seg, out, workspace, st);
    else e = launch_norm<float, float>(cfg, w, z, cu, 1, T_seg, out, workspace, st);
    return cuda_status(e);
}

// ---------------------------------------------------------------------------
// Prefill from host buffers (see host_layout)
// ---------------------------------------------------------------------------
namespace {
// cu of one segment: sequences s_a .. s_a + n_s - 1 clipped to tokens [t0, t1)
__global__ void segment_seqlens_kernel(const int32_t* cu, int32_t s_a, int32_t n_s, int32_t t0, int32_t t1,
                                       int32_t* out) {
    for (int j = threadIdx.x; j <= n_s; j += blockDim.x) {
        const int32_t x = cu[s_a + j];
        out[j] = (x < t0 ? t0 : x > t1 ? t1 : x) - t0;
    }
}
}  // namespace

size_t gdn_prefill_host_workspace_size(const gdn_config* cfg, int64_t T_total, int32_t n_seqs) {
    if (check_config(cfg) != GDN_OK || T_total < 0 || n_seqs < 0) return 0;
    return host_layout(cfg, T_total, n_seqs).total;
}

gdn_status gdn_prefill_host(const gdn_config* cfg, const gdn_weights* w, const void* q, const void* k,
                            const void* v, const void* a, const void* b, const void* z, void* conv_state,
                            void* rec_state, const int32_t* cu_seqlens, int32_t n_seqs, int64_t T_total,
                            void* out, void* workspace, size_t workspace_bytes, void* stream) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if ((s = check_weights(w)) != GDN_OK) return s;
    if (n_seqs < 0 || T_total < 0) return GDN_ERR_INVALID_ARG;
    if (T_total == 0 || n_seqs == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !z || !conv_state || !rec_state || !cu_seqlens || !out || !workspace)
        return GDN_ERR_INVALID_ARG;
    if (!aligned(rec_state, 16) || !aligned(workspace, 256)) return GDN_ERR_INVALID_ARG;
    if (T_total > 0x7fffffffLL - 64) return GDN_ERR_UNSUPPORTED;
    // the sequence offsets are on the host: check them here
    if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T_total) return GDN_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_seqs; ++i)
        if (cu_seqlens[i + 1] < cu_seqlens[i]) return GDN_ERR_INVALID_ARG;
    const HostLayout L = host_layout(cfg, T_total, n_seqs);
    if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t sin = side_stream(1), sout = side_stream(2);
    if (!sin || !sout) return cuda_status(cudaErrorNotReady);
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    const void* hin[6] = {q, k, v, a, b, z};
    const size_t state_bytes = (size_t)cfg->n_v_heads * cfg->d_v * cfg->d_k * (cfg->state_dtype == GDN_BF16 ? 2 : 4);
    const size_t conv_bytes = (size_t)(2 * cfg->n_k_heads * cfg->d_k + cfg->n_v_heads * cfg->d_v) *
                              (cfg->conv_kernel - 1) * (cfg->act_dtype == GDN_F32 ? 4 : 2);
    const int n_seg = L.plan.n_seg;
    // fork, then per segment: in_ready, computed, out_done
    cudaEvent_t* ev = thread_events(kEvHost, 1 + 3 * (size_t)n_seg);
    if (!ev) return cuda_status(cudaErrorNotReady);
    gdn_status rc = GDN_OK;
    auto cu_err = [&](cudaError_t e) {
        if (e != cudaSuccess && rc == GDN_OK) rc = cuda_status(e);
        return e == cudaSuccess;
    };
    cudaEvent_t fork = ev[0];
    cudaEvent_t* in_ready = ev + 1;
    cudaEvent_t* computed = ev + 1 + n_seg;
    cudaEvent_t* out_done = ev + 1 + 2 * n_seg;
    int32_t* cu_dev = reinterpret_cast<int32_t*>(wsb + L.cu_off);
    // (cu_err records the first failure in rc, which ends the loop below)
    (void)(cu_err(cudaMemcpyAsync(cu_dev, cu_seqlens, ((size_t)n_seqs + 1) * 4, cudaMemcpyHostToDevice, st)) &&
           cu_err(cudaEventRecord(fork, st)) && cu_err(cudaStreamWaitEvent(sin, fork, 0)) &&
           cu_err(cudaStreamWaitEvent(sout, fork, 0)));
    int32_t s_a = 0;
    for (int i = 0; rc == GDN_OK && i < n_seg; ++i) {
        const int slot = i & 1;
        const int64_t t0 = (int64_t)i * L.plan.seg_len;
        const int64_t t1 = std::min<int64_t>(T_total, t0 + L.plan.seg_len);
        // sequences overlapping [t0, t1): from the one holding token t0 to the one holding t1 - 1
        while (s_a + 1 < n_seqs && cu_seqlens[s_a + 1] <= t0) ++s_a;
        int32_t s_b = s_a;
        while (s_b + 1 < n_seqs && cu_seqlens[s_b + 1] < t1) ++s_b;
        const int32_t n_s = s_b - s_a + 1;
        uint8_t* slot_p = wsb + L.slot_off[slot];
        // inputs in, once the segment two back has read this slot
        if (i >= 2 && !cu_err(cudaStreamWaitEvent(sin, computed[i - 2], 0))) break;
        for (int j = 0; j < 6; ++j)
            if (!cu_err(cudaMemcpyAsync(slot_p + L.in_off[j], static_cast<const uint8_t*>(hin[j]) + t0 * L.row_in[j],
                                        (size_t)(t1 - t0) * L.row_in[j], cudaMemcpyHostToDevice, sin)))
                break;
        if (rc != GDN_OK || !cu_err(cudaEventRecord(in_ready[i], sin))) break;
        // the segment, once its inputs are in and the segment two back has sent its output out
        if (!cu_err(cudaStreamWaitEvent(st, in_ready[i], 0))) break;
        if (i >= 2 && !cu_err(cudaStreamWaitEvent(st, out_done[i - 2], 0))) break;
        int32_t* seg_cu = reinterpret_cast<int32_t*>(wsb + L.seg_cu_off[slot]);
        segment_seqlens_kernel<<<1, 256, 0, st>>>(cu_dev, s_a, n_s, (int32_t)t0, (int32_t)t1, seg_cu);
        if (!cu_err(cudaGetLastError())) break;
        const gdn_status g = gdn_prefill(
            cfg, w, slot_p + L.in_off[0], slot_p + L.in_off[1], slot_p + L.in_off[2], slot_p + L.in_off[3],
            slot_p + L.in_off[4], slot_p + L.in_off[5], static_cast<uint8_t*>(conv_state) + (size_t)s_a * conv_bytes,
            static_cast<uint8_t*>(rec_state) + (size_t)s_a * state_bytes, seg_cu, n_s, t1 - t0, slot_p + L.out_off,
            wsb + L.pre_off, L.cu_off - L.pre_off, st);
        if (g != GDN_OK) {
            rc = g;
            break;
        }
        if (!cu_err(cudaEventRecord(computed[i], st))) break;
        // the output out
        if (!cu_err(cudaStreamWaitEvent(sout, computed[i], 0))) break;
        if (!cu_err(cudaMemcpyAsync(static_cast<uint8_t*>(out) + t0 * L.row_out, slot_p + L.out_off,
                                    (size_t)(t1 - t0) * L.row_out, cudaMemcpyDeviceToHost, sout)))
            break;
        if (!cu_err(cudaEventRecord(out_done[i], sout))) break;
    }
    // join: the caller's stream waits for the last output copy (the copy streams are in order)
    if (rc == GDN_OK) cu_err(cudaStreamWaitEvent(st, out_done[n_seg - 1], 0));
    return rc;
}

gdn_status gdn_check_device_error(void* stream) {
    cudaError_t e = cudaSuccess;
    const gdn_status s = gdn::take_device_error(static_cast<cudaStream_t>(stream), &e);
    if (e != cudaSuccess) cuda_status(e);
    return s;
}

const char* gdn_last_cuda_error(void) {
    thread_local char buf[256];
    const cudaError_t e = t_last_cuda_error;
    if (e == cudaSuccess) return "no CUDA error";
    snprintf(buf, sizeof buf, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return buf;
}

const char* gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case GDN_ERR_WORKSPACE: return "workspace too small";
        case GDN_ERR_SEQLENS: return "cu_seqlens malformed (device check)";
        case GDN_ERR_RANGE: return "conv output beyond the fp16 range of the workspace (device check)";
    }
    return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// gdn_prefill_noalloc: gdn_prefill with its workspace in a fixed device array,
// for callers that cannot allocate device memory (see gdn.h).
// ---------------------------------------------------------------------------
#include <mutex>

static __device__ __align__(256) uint8_t g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
// Device address of g_noalloc_scratch per device, with the context it was
// looked up in: a reset device gets a new context, and the address is looked
// up again there.
struct NoallocSlot {
    CUcontext ctx;
    void* addr;
};
NoallocSlot g_noalloc_slot[64];

}  // namespace

extern "C" gdn_status gdn_prefill_noalloc(const gdn_config* cfg, const gdn_weights* w, const void* q,
                                          const void* k, const void* v, const void* a, const void* b,
                                          const void* z, void* conv_state, void* rec_state,
                                          const int32_t* cu_seqlens, int32_t n_seqs, int64_t T_total,
                                          void* out, void* stream) {
    gdn_status s = check_config(cfg);
    if (s != GDN_OK) return s;
    if (n_seqs < 0 || T_total < 0) return GDN_ERR_INVALID_ARG;
    if (workspace_layout(cfg, T_total, n_seqs).total > GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (T_total > 0 && n_seqs > 0) {
        int dev = 0;
        const cudaError_t ed = cudaGetDevice(&dev);
        if (ed != cudaSuccess) return cuda_status(ed);
        if (dev < 0 || dev >= 64) return GDN_ERR_UNSUPPORTED;
        auto get_ctx = ctx_getter();
        CUcontext ctx = nullptr;   // null while this thread has no current context yet
        if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return cuda_status(cudaErrorInitializationError);
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        NoallocSlot& slot = g_noalloc_slot[dev];
        if (!slot.addr || !ctx || slot.ctx != ctx) {
            // The array's name is a host-side stand-in; the kernels need its device address.
            // The lookup also makes the device's context current, so it is read again after.
            void* p = nullptr;
            const cudaError_t es = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (es != cudaSuccess || !p) return cuda_status(es != cudaSuccess ? es : cudaErrorInvalidSymbol);
            if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return cuda_status(cudaErrorInitializationError);
            slot.ctx = ctx;
            slot.addr = p;
        }
        scratch = slot.addr;
    }
    return gdn_prefill(cfg, w, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens, n_seqs, T_total, out,
                       scratch, GDN_NOALLOC_SCRATCH_BYTES, stream);
}
