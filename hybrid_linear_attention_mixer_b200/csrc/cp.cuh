// Context-parallel prefill of one long sequence cut into contiguous segments,
// one per rank (GPU).
//
// Over one segment the state map of the gated delta rule is affine:
//     S_end = S_0 . P + S_loc,
// with S_loc the segment's final state from a zero start and P (d_k x d_k) the
// product of the per-chunk transitions M_c = e^{g_C} I - W_c^T K~_c.  Written as
// S_new = e^{g_C} S - (W S^T)^T K~ + (T V)^T K~, the chunk step is exactly the
// scan's state update, so P is the scan's final state from S_0 = I with V = 0
// (and S_loc the scan's final state from S_0 = 0 with the real V).  Both runs
// reuse one set of intra-chunk records, and P carries the scan's own relative
// precision (its fp16 operands round P's entries, not P + S_loc's).
//
// Each rank computes (P, S_loc) for its segment, the ranks exchange them, and
// rank r folds the maps of ranks 0 .. r-1 onto the sequence's initial state to
// get its own S_0; a last scan from that S_0 gives its outputs and end state.
#pragma once

#include "device.cuh"

namespace gdn {
namespace cp {

// cu_seqlens {0, T} of a segment run as one sequence.
__global__ void segment_cu_kernel(int32_t* cu, int32_t T) {
    if (threadIdx.x == 0) {
        cu[0] = 0;
        cu[1] = T;
    }
}

// x[h] = I (d x d) for every value head.
__global__ void identity_kernel(float* x, int Hv, int d) {
    const int64_t n = (int64_t)Hv * d * d;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        x[i] = ((i / d) % d == i % d) ? 1.f : 0.f;
}

constexpr int CR = 16;    // state rows per CTA of the fold
constexpr int CT = 128;   // threads: one per column (d <= 128)

// state_out = fold_{j < rank} (S <- S . P_j + S_loc_j) applied to state_in, in
// fp32.  summaries: [n_ranks][2][Hv][d][d] with [j][0] = P_j, [j][1] = S_loc_j.
// Rows are independent, so one CTA takes CR rows of one head through every
// step; thread k holds column k.  state_out may alias state_in.
__global__ void __launch_bounds__(CT) fold_kernel(const float* state_in, const float* summaries, int rank, int Hv,
                                                  int d, float* state_out, const int32_t* flags = nullptr) {
    if (flags && *flags) return;   // (a prefill whose device checks failed writes nothing)
    __shared__ float s[CR][CT];
    const int blocks_per_head = d / CR;
    const int h = blockIdx.x / blocks_per_head, r0 = (blockIdx.x % blocks_per_head) * CR;
    const int k = threadIdx.x;
    const bool on = k < d;
    const size_t hd = (size_t)h * d * d;
#pragma unroll
    for (int i = 0; i < CR; ++i) s[i][k] = on ? state_in[hd + (size_t)(r0 + i) * d + k] : 0.f;
    __syncthreads();
    for (int j = 0; j < rank; ++j) {
        const float* P = summaries + ((size_t)j * 2 * Hv) * d * d + hd;
        const float* B = summaries + ((size_t)(j * 2 + 1) * Hv) * d * d + hd;
        float acc[CR];
#pragma unroll
        for (int i = 0; i < CR; ++i) acc[i] = on ? B[(size_t)(r0 + i) * d + k] : 0.f;
#pragma unroll 8   // eight P rows' loads in flight (d is a multiple of 32)
        for (int m = 0; m < d; ++m) {
            const float pm = on ? P[(size_t)m * d + k] : 0.f;
#pragma unroll
            for (int i = 0; i < CR; ++i) acc[i] = fmaf(s[i][m], pm, acc[i]);
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < CR; ++i) s[i][k] = acc[i];
        __syncthreads();
    }
    if (on) {
#pragma unroll
        for (int i = 0; i < CR; ++i) state_out[hd + (size_t)(r0 + i) * d + k] = s[i][k];
    }
}

}  // namespace cp
}  // namespace gdn
