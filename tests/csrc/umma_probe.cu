// Test-only check of the tcgen05 operand layouts the prefill kernel uses: one
// 128 x N x K product D = A B^T per call, operands staged in shared memory with
// the kernel's 128-byte-swizzled tiles and descriptors, read back from tensor
// memory.  The test compares D with numpy.
//   variant 0: A K-major  (M=128, K=128), B K-major  (N=64,  K=128)
//   variant 1: A MN-major (M=128, K=64),  B K-major  (N=64,  K=64)
//   variant 2: A K-major  (M=128, K=128), B MN-major (N=64,  K=128)
//   variant 3: A K-major  (M=128, K=64),  B MN-major (N=128, K=64)
//   variant 4: A in TMEM  (M=128, K=128), B K-major  (N=64,  K=128)
//   variant 5: A in TMEM  (M=128, K=64),  B MN-major (N=128, K=64)
//   variant 6: A in TMEM  (M=128, K=128), B MN-major (N=64,  K=128)
// It also holds a test of the bounded wait: an mbarrier wait that nothing
// completes gives up after its limit, records its code in the error word, and
// the kernel returns; the host side maps the word to a status (the same
// device.cuh code as the library's kernels and gdn_check_device_error).
#include "../../hybrid_linear_attention_mixer_b200/csrc/device.cuh"

using namespace gdn;

namespace {
constexpr uint32_t A_OFF = 0, B_OFF = 32768, BAR_OFF = 65536;

__global__ void __launch_bounds__(128, 1) umma_probe_kernel(int variant, const float* A, const float* B, float* D) {
    extern __shared__ uint8_t raw[];
    const uint32_t r0 = smem_u32(raw);
    const uint32_t sb = (r0 + 1023u) & ~1023u;
    uint8_t* sm = raw + (sb - r0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = (variant == 0 || variant == 2 || variant == 4 || variant == 6) ? 128 : 64;
    const int N = (variant == 3 || variant == 5) ? 128 : 64;
    const int a_tm = variant >= 4;
    const int a_mn = variant == 1, b_mn = variant == 2 || variant == 3 || variant == 5 || variant == 6;
    const uint32_t lbo_a = 8192;            // MN-major A: 64 K-rows x 128 B per MN half
    const uint32_t lbo_b = (uint32_t)K * 128;  // MN-major B: K rows x 128 B per MN half
    const uint32_t half_b = (uint32_t)N * 128; // K-major B: N rows x 128 B per K half
    for (int idx = tid; idx < 128 * K && !a_tm; idx += 128) {
        const int m = idx / K, k = idx % K;
        const uint32_t off = a_mn ? (m / 64) * lbo_a + swz128(k, (m % 64) / 8) + (m % 8) * 2
                                  : (k / 64) * 16384 + swz128(m, (k % 64) / 8) + (k % 8) * 2;
        *reinterpret_cast<__half*>(sm + A_OFF + off) = __float2half_rn(A[idx]);
    }
    for (int idx = tid; idx < N * K; idx += 128) {
        const int n = idx / K, k = idx % K;
        const uint32_t off = b_mn ? (n / 64) * lbo_b + swz128(k, (n % 64) / 8) + (n % 8) * 2
                                  : (k / 64) * half_b + swz128(n, (k % 64) / 8) + (k % 8) * 2;
        *reinterpret_cast<__half*>(sm + B_OFF + off) = __float2half_rn(B[idx]);
    }
    const uint32_t bar = sb + BAR_OFF;
    volatile uint32_t* slot = reinterpret_cast<volatile uint32_t*>(sm + BAR_OFF + 8);
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sb + BAR_OFF + 8, 256);
        tmem_relinquish();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t a_col = 128;   // A operand columns start here when it lives in TMEM
    if (a_tm) {   // row m = lane m (thread m); columns hold fp16 pairs (k even in the low half)
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16) + a_col;
        const int row = 32 * warp + lane;
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t r[16];
            for (int i = 0; i < 16; i++)
                r[i] = pack_half2(A[row * K + 2 * (c0 + i)], A[row * K + 2 * (c0 + i) + 1]);
            tmem_st16(lane_addr + c0, r);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (tid == 0) {
        for (int ks = 0; ks < K / 16; ks++) {
            const uint32_t aa = a_mn ? sb + A_OFF + ks * 2048 : sb + A_OFF + (ks >> 2) * 16384 + (ks & 3) * 32;
            const uint32_t ba = b_mn ? sb + B_OFF + ks * 2048 : sb + B_OFF + (ks >> 2) * half_b + (ks & 3) * 32;
            if (a_tm)
                mma_f16_ta(tmem, tmem + a_col + ks * 8, sdesc(ba, b_mn ? lbo_b : 16, 1024),
                           idesc_f16(128, N, 0, b_mn), ks > 0);
            else
                mma_f16(tmem, sdesc(aa, a_mn ? lbo_a : 16, 1024), sdesc(ba, b_mn ? lbo_b : 16, 1024),
                        idesc_f16(128, N, a_mn, b_mn), ks > 0);
        }
        mma_commit(bar);
    }
    const bool ok = mbar_wait_bounded(bar, 0);
    tc_fence_after();
    if (ok) {
        const int row = 32 * warp + lane;
        for (int c = 0; c < N / 32; c++) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * c, r);
            for (int i = 0; i < 32; i++) D[row * N + 32 * c + i] = __uint_as_float(r[i]);
        }
    } else if (tid == 0) {
        record_error(kErrMmaTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}
// One mbarrier that nothing ever arrives on, waited on for at most limit_ns.
__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(unsigned long long limit_ns, int* gave_up) {
    __shared__ __align__(8) uint64_t bar_mem;
    const uint32_t bar = smem_u32(&bar_mem);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        const bool done = mbar_wait_bounded(bar, 0, limit_ns);
        if (!done) record_error(kErrCopyTimeout);
        *gave_up = done ? 0 : 1;
    }
}
}  // namespace

// Runs the wait above on `stream` and returns the status the error word maps to
// (read and cleared), with the kernel's duration in *ms and its outcome in
// *gave_up_dev (device int: 1 if the wait gave up).
extern "C" int probe_wait_timeout(unsigned long long limit_ns, int* gave_up_dev, float* ms, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return -1;
    cudaEventRecord(e0, st);
    wait_timeout_kernel<<<1, 32, 0, st>>>(limit_ns, gave_up_dev);
    const bool launched = cudaGetLastError() == cudaSuccess;
    cudaEventRecord(e1, st);
    const gdn_status s = take_device_error(st);
    cudaEventElapsedTime(ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    return launched ? (int)s : -2;
}

// The error word of this module, read and cleared (the library's check, in this module).
extern "C" int probe_check_device_error(void* stream) {
    return (int)take_device_error(static_cast<cudaStream_t>(stream));
}

extern "C" int umma_probe(int variant, const float* A, const float* B, float* D) {
    if (variant < 0 || variant > 6) return 1;
    const int smem = 65536 + 64 + 1024;
    if (cudaFuncSetAttribute(umma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 2;
    umma_probe_kernel<<<1, 128, smem>>>(variant, A, B, D);
    if (cudaGetLastError() != cudaSuccess) return 3;
    if (cudaDeviceSynchronize() != cudaSuccess) return 4;
    unsigned int err = 0;
    cudaMemcpyFromSymbol(&err, g_device_error, sizeof err);
    return err ? 5 : 0;
}
