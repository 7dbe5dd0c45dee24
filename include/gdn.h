/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet token mixer.
 *
 * The layer (one of the 36 linear-attention layers of the hybrid decoder
 * described in "Qwen3.8-Flash-Next" (llm-architectures-explained), "Every
 * architecture field": mixers.linear.type deltanet, 16 key heads, 48 value
 * heads, key/value head dim 128, conv kernel 4; "Qwen3.8-Flash-Next anatomy"
 * (frontier-model-atlas), "Decoder microscope"):
 *
 *   x_t   = [q_t | k_t | v_t]                      (2*H_k*d_k + H_v*d_v channels)
 *   y_t   = SiLU(sum_i w[c,i] x_{t-K+1+i}[c])      depthwise causal conv, no bias;
 *                                                  the K-1 inputs before a sequence
 *                                                  start come from conv_state
 *   q^,k^ = y_q / sqrt(|y_q|^2 + l2_eps), same for k, per key head
 *   alpha = exp(-exp(A_log[h]) * softplus(a_t + dt_bias[h])),  beta = sigmoid(b_t)
 *   S_t   = alpha S_{t-1} (I - beta k^ k^T) + beta v^ k^T    (S: d_v x d_k, fp32)
 *   o_t   = S_t q^ / sqrt(d_k)
 *   out_t = o_t * rsqrt(mean(o_t^2) + norm_eps) * norm_weight * SiLU(z_t)
 *
 * Value head h reads key head h / (H_v / H_k).  The recurrent state is kept in
 * float32 (mamba_ssm_dtype float32, "Qwen3.8-Flash-Next" (llm-atlas-9r2),
 * "Raw config fields"); norm_eps defaults to rms_norm_eps = 1e-6 from the same
 * table.  The pages name the gated delta rule without printing it; the
 * recurrence above is its standard statement.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers, contiguous, row-major, owned by
 *     the caller.  The library allocates no memory and never synchronises the
 *     stream (gdn_check_device_error excepted).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream).  conv_state and rec_state are read and
 *     updated in place.
 *   - Activation tensors q, k, v, a, b, z and conv_state are all of
 *     config->act_dtype; out is of config->out_dtype.  Parameters are float32.
 *   - Pointers q, k, v, z, out, rec_state, conv_state and workspace must be
 *     16-byte aligned.
 *   - Argument errors are returned synchronously and launch nothing.  Launch
 *     failures return GDN_ERR_CUDA.  Kernels never trap: a bounded wait that
 *     runs out records a device error word and the kernel returns;
 *     gdn_check_device_error reports it as GDN_ERR_DEVICE_TIMEOUT.  Checks of
 *     device-resident inputs (prefill's cu_seqlens, and the fp16 range of the
 *     conv outputs it keeps in its workspace) report through the same word
 *     (GDN_ERR_SEQLENS, GDN_ERR_RANGE).
 *   - No C++ exception crosses this interface.
 *
 * Supported shapes: d_k, d_v in {32, 64, 128}; n_v_heads a multiple of
 * n_k_heads; conv_kernel == 4; chunk == 64 (the chunk length never changes the
 * result, only how prefill is computed).  Anything else: GDN_ERR_UNSUPPORTED.
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misaligned pointer   */
    GDN_ERR_UNSUPPORTED = 2,     /* shape or dtype outside the supported set     */
    GDN_ERR_CUDA = 3,            /* a CUDA launch or runtime call failed          */
    GDN_ERR_DEVICE_TIMEOUT = 4,  /* a kernel's bounded wait ran out               */
    GDN_ERR_WORKSPACE = 5,       /* workspace smaller than gdn_prefill_workspace_size */
    GDN_ERR_SEQLENS = 6,         /* (device check) cu_seqlens malformed           */
    GDN_ERR_RANGE = 7            /* (device check) a conv output beyond the fp16 range
                                    of the prefill workspace                        */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

typedef struct {
    int32_t n_k_heads;    /* H_k, default 16  */
    int32_t n_v_heads;    /* H_v, default 48  */
    int32_t d_k;          /* default 128      */
    int32_t d_v;          /* default 128      */
    int32_t conv_kernel;  /* K, default 4     */
    int32_t chunk;        /* prefill chunk, default 64 */
    float l2_eps;         /* default 1e-6     */
    float norm_eps;       /* default 1e-6     */
    int32_t act_dtype;    /* gdn_dtype of q, k, v, a, b, z, conv_state; default GDN_BF16 */
    int32_t out_dtype;    /* gdn_dtype of out; default GDN_BF16 */
    int32_t state_dtype;  /* gdn_dtype of rec_state and of state snapshots; default GDN_F32
                             (the layer's fp32 state).  GDN_BF16 stores the state in bf16
                             (half the bytes a decode step moves); every step still
                             computes in fp32 and rounds the stored state to nearest even */
    int32_t prefill_segments; /* how a prefill overlaps its state chain with other work.
                             n >= 2: pipelined over n chunk ranges (at most
                             GDN_PREFILL_MAX_SEGMENTS): the ranges' conv and intra-chunk
                             kernels run on the caller's stream while the state chain walks
                             the ranges before them on a high-priority stream of the
                             library's own; the results are those of one range, bit for bit.
                             1: one range.  GDN_PREFILL_SPLIT (-1): for one sequence at
                             d_k = d_v = 128 with bf16 activations and output and an fp32
                             state, the chain is cut in two at its middle chunk and the
                             halves run at the same time (the second from a zero state and as
                             its transition map), then the second half's outputs and end state
                             are corrected with the first half's end state; other calls take
                             one range.  The results then differ from one range's within the
                             rounding of the bf16 correction (well inside the layer's
                             tolerances).  0 (the default): automatic, at most 8 ranges of at
                             least 32 chunks when the call has at most 96 chains
                             (n_seqs x H_v), else one range */
} gdn_config;

#define GDN_PREFILL_MAX_SEGMENTS 32
/* gdn_config.prefill_segments: split one sequence's state chain in two (see gdn_prefill) */
#define GDN_PREFILL_SPLIT (-1)

typedef struct {
    const float* conv_weight;  /* [2*H_k*d_k + H_v*d_v][K], channel order q | k | v;
                                  tap K-1 multiplies the current token            */
    const float* A_log;        /* [H_v]                                           */
    const float* dt_bias;      /* [H_v]                                           */
    const float* norm_weight;  /* [d_v], shared by all value heads               */
} gdn_weights;

/* Fills *cfg with the layer's published shape (16/48 heads of 128, K = 4,
 * chunk 64, eps 1e-6, bf16 activations and output, fp32 state). */
void gdn_config_default(gdn_config* cfg);

/* Bytes of device workspace gdn_prefill needs for T_total packed tokens.
 * Returns 0 for an invalid or unsupported config. */
size_t gdn_prefill_workspace_size(const gdn_config* cfg, int64_t T_total, int32_t n_seqs);

/* How gdn_prefill runs a call of this size (see gdn_config.prefill_segments): the
 * number of chunk ranges it is pipelined over (1 when it runs in one piece; with
 * n > 1 ranges a call launches 2 + 4 n kernels, else 6), or GDN_PREFILL_SPLIT when
 * it splits the chain (12 kernels and one memset).  Returns 0 for an invalid config. */
int32_t gdn_prefill_segments(const gdn_config* cfg, int64_t T_total, int32_t n_seqs);

/*
 * Packed variable-length prefill.
 *   q, k        [T_total][H_k][d_k]    act_dtype
 *   v, z        [T_total][H_v][d_v]    act_dtype
 *   a, b        [T_total][H_v]         act_dtype
 *   conv_state  [n_seqs][2*H_k*d_k + H_v*d_v][K-1]  act_dtype, in/out, oldest first
 *   rec_state   [n_seqs][H_v][d_v][d_k] state_dtype (float32 by default), in/out
 *   cu_seqlens  [n_seqs + 1] int32 device, cu_seqlens[0] = 0, non-decreasing,
 *               cu_seqlens[n_seqs] = T_total.  It is device memory, so the host
 *               cannot read it without synchronising: the first kernel checks it.
 *               A malformed cu_seqlens records GDN_ERR_SEQLENS in the device
 *               error word, and the call then writes neither out nor either
 *               state (the workspace is scratch).
 *   out         [T_total][H_v][d_v]    out_dtype
 *   workspace   >= gdn_prefill_workspace_size(cfg, T_total, n_seqs) bytes,
 *               256-byte aligned; contents need not be initialised
 * Sequences of length 0 leave their states unchanged.  T_total == 0 is a no-op.
 * Range: the conv outputs q^, k^, v^ are kept in fp16 in the workspace.  If a
 * conv output lies beyond the fp16 range (|v^| > 65504, or a q or k row whose
 * squared norm overflows fp32), the call records GDN_ERR_RANGE and likewise
 * writes neither out nor either state.
 * Both device checks are read by gdn_check_device_error.
 */
gdn_status gdn_prefill(const gdn_config* cfg, const gdn_weights* w,
                       const void* q, const void* k, const void* v,
                       const void* a, const void* b, const void* z,
                       void* conv_state, void* rec_state,
                       const int32_t* cu_seqlens, int32_t n_seqs, int64_t T_total,
                       void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode step: one new token for each of n_seqs sequences.
 *   q, k [n_seqs][H_k][d_k]; v, z [n_seqs][H_v][d_v]; a, b [n_seqs][H_v]  act_dtype
 *   conv_state [n_seqs][C][K-1] act_dtype in/out; rec_state [n_seqs][H_v][d_v][d_k]
 *   state_dtype in/out; out [n_seqs][H_v][d_v] out_dtype.  No workspace.
 * Equal to gdn_prefill with every sequence of length 1.
 */
gdn_status gdn_decode(const gdn_config* cfg, const gdn_weights* w,
                      const void* q, const void* k, const void* v,
                      const void* a, const void* b, const void* z,
                      void* conv_state, void* rec_state, int32_t n_seqs,
                      void* out, void* stream);

/* Largest number of tokens per sequence that gdn_decode_multi takes in one call. */
#define GDN_DECODE_MULTI_MAX_TOKENS 16

/*
 * Several decode steps at once: n_tok consecutive new tokens for each of n_seqs
 * sequences, for checking tokens that a multi-token-prediction head drafted
 * ("Qwen3.8-Flash-Next", section "Architecture concepts": Multi-Token
 * Prediction drafts tokens at inference; table "Every architecture field",
 * row mtp_layers).  The result equals n_tok consecutive gdn_decode calls (the
 * conv states bit for bit, the rest up to the order of fp32 additions inside a
 * state row's dot products), but each state is read and written once.
 *   q, k [n_seqs*n_tok][H_k][d_k]; v, z [n_seqs*n_tok][H_v][d_v];
 *   a, b [n_seqs*n_tok][H_v]  act_dtype, token-major within a sequence: row
 *   seq*n_tok + t holds token t of sequence seq
 *   conv_state [n_seqs][C][K-1] act_dtype in/out; rec_state
 *   [n_seqs][H_v][d_v][d_k] state_dtype in/out (the state after the last token)
 *   out [n_seqs*n_tok][H_v][d_v] out_dtype
 *   state_snapshots  optional (may be NULL), [n_tok][n_seqs][H_v][d_v][d_k]
 *                    state_dtype, 16-byte aligned: the state after each token, so
 *                    that a caller who accepts only the first j drafted tokens
 *                    can restore the state after token j
 *   conv_snapshots   optional (may be NULL), [n_tok][n_seqs][C][K-1] act_dtype:
 *                    the conv state after each token
 * 1 <= n_tok <= GDN_DECODE_MULTI_MAX_TOKENS (larger: GDN_ERR_UNSUPPORTED);
 * n_tok == 0 or n_seqs == 0 is a no-op.  No workspace.
 */
gdn_status gdn_decode_multi(const gdn_config* cfg, const gdn_weights* w,
                            const void* q, const void* k, const void* v,
                            const void* a, const void* b, const void* z,
                            void* conv_state, void* rec_state, int32_t n_seqs, int32_t n_tok,
                            void* out, void* state_snapshots, void* conv_snapshots, void* stream);

/* Largest number of output segments one gdn_linear call writes. */
#define GDN_LINEAR_MAX_SEGMENTS 8

/* One output segment of a projection: the next `width` columns of y go to
 * dst, a row-major [M][width] bf16 matrix (device pointer, 16-byte aligned,
 * width a multiple of 8). */
typedef struct {
    void* dst;
    int32_t width;
} gdn_out_segment;

/*
 * Dense projection on the tensor cores: y[M][N] = x[M][K] . w[N][K]^T, bf16
 * operands, fp32 accumulation, each output rounded once to bf16 (nearest even).
 * No bias.  w is laid out as a linear layer's weight (one row per output
 * column).  The columns of y are split, in order, over segs[0..n_segs): the
 * widths must add up to N.  This serves the projections around the mixer,
 * whose widths come from the hidden size 2,560 ("Qwen3.8-Flash-Next"
 * (llm-atlas-9r2), "Key facts"; (llm-architectures-explained), "Every
 * architecture field", row d_model) and the head shapes above.
 *   x  [M][K] bf16, 16-byte aligned; w [N][K] bf16, 16-byte aligned
 *   N, K multiples of 8 (else GDN_ERR_UNSUPPORTED); M == 0 is a no-op;
 *   1 <= n_segs <= GDN_LINEAR_MAX_SEGMENTS (more: GDN_ERR_UNSUPPORTED)
 * No workspace.  Asynchronous on `stream`.
 */
gdn_status gdn_linear(const void* x, const void* w, int64_t M, int32_t N, int32_t K,
                      const gdn_out_segment* segs, int32_t n_segs, void* stream);

/*
 * The mixer's input projection.  The pages do not print the projection layout;
 * the reading taken is one bias-free linear map from the hidden state to all of
 * the mixer's inputs, its output channels in the order
 *   q (H_k*d_k) | k (H_k*d_k) | v (H_v*d_v) | z (H_v*d_v) | a (H_v) | b (H_v)
 * (16,480 channels at the published shape).
 *   hidden [T][d_model] bf16; w_in [2*H_k*d_k + 2*H_v*d_v + 2*H_v][d_model] bf16
 *   q, k [T][H_k][d_k]; v, z [T][H_v][d_v]; a, b [T][H_v]: bf16 outputs, 16-byte
 *   aligned, ready for gdn_prefill / gdn_decode with act_dtype GDN_BF16.
 * H_v must be a multiple of 8 and d_model of 8 (else GDN_ERR_UNSUPPORTED).
 */
gdn_status gdn_in_proj(const gdn_config* cfg, const void* hidden, const void* w_in, int64_t T,
                       int32_t d_model, void* q, void* k, void* v, void* z, void* a, void* b,
                       void* stream);

/*
 * The mixer's output projection: y[T][d_model] = o[T][H_v*d_v] . w_out^T, with
 * o the bf16 output of gdn_prefill / gdn_decode and w_out [d_model][H_v*d_v]
 * bf16.  d_model must be a multiple of 8.
 */
gdn_status gdn_out_proj(const gdn_config* cfg, const void* o, const void* w_out, int64_t T,
                        int32_t d_model, void* y, void* stream);

/*
 * Context-parallel prefill: one long sequence (up to the 262,144-token context of
 * "Qwen3.8-Flash-Next" (llm-atlas-9r2), "Key facts") cut into contiguous
 * segments, one per rank, computing what one gdn_prefill over the whole
 * sequence computes.  Over a segment the state map is affine,
 * S_end = S_0 . P + S_loc, with P (d_k x d_k) the product of the segment's chunk
 * transitions and S_loc its end state from S_0 = 0.  Each rank:
 *   1. gdn_cp_local on its segment, with conv_state set to the K-1 input rows
 *      (q | k | v channels) before the segment (the previous rank's last rows,
 *      or the sequence's conv state on rank 0): writes summary = {P, S_loc};
 *   2. the ranks exchange their summaries (an all-gather, in rank order);
 *   3. gdn_cp_finish: folds the maps of ranks 0 .. rank-1 onto state_in (the
 *      state before the whole sequence) to get this segment's S_0, then runs the
 *      scan and the gated norm: out holds the segment's outputs and state_out the
 *      state after the segment (on the last rank: the sequence's final state).
 * The segment runs as one sequence; the caller keeps `workspace` (of
 * gdn_cp_workspace_size bytes, 256-byte aligned) between the two calls.
 * Requires state_dtype GDN_F32 and d_k == d_v (else GDN_ERR_UNSUPPORTED).
 *   q, k, v, a, b, z: this segment's rows, as for gdn_prefill (T_seg >= 1)
 *   conv_state [C][K-1] act_dtype in/out (out: the segment's last K-1 inputs)
 *   summary    [2][H_v][d_k][d_k] fp32 out: P, then S_loc
 *   summaries  [n_ranks][2][H_v][d_k][d_k] fp32: every rank's summary
 *   state_in, state_out [H_v][d_v][d_k] fp32; they may alias
 */
size_t gdn_cp_workspace_size(const gdn_config* cfg, int64_t T_seg);
gdn_status gdn_cp_local(const gdn_config* cfg, const gdn_weights* w,
                        const void* q, const void* k, const void* v, const void* a, const void* b,
                        void* conv_state, int64_t T_seg, void* summary,
                        void* workspace, size_t workspace_bytes, void* stream);
gdn_status gdn_cp_finish(const gdn_config* cfg, const gdn_weights* w, const void* z,
                         const void* summaries, int32_t n_ranks, int32_t rank,
                         const void* state_in, int64_t T_seg, void* out, void* state_out,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_prefill from HOST buffers, end to end: the inputs come from the host, the
 * result goes back to the host, and the transfers overlap the work.  The tokens
 * are cut into at most 8 segments (multiples of 64 rows, at least 512); segment
 * i runs on `stream` while segment i+1's inputs are copied in and segment i-1's
 * output is copied out on two internal copy streams (one cudaMemcpyAsync per
 * tensor and segment).  Sequences that cross a cut continue from the states the
 * previous segment left, so the result is gdn_prefill's (up to where the chunk
 * boundaries fall).
 *   q, k, v, a, b, z, out: HOST pointers, same layouts as gdn_prefill (page-locked
 *     memory lets the copies overlap; pageable memory is correct but serialises)
 *   cu_seqlens: HOST [n_seqs+1], 0 = cu[0] <= ... <= cu[n_seqs] = T_total (checked)
 *   conv_state, rec_state, workspace: DEVICE, as for gdn_prefill; workspace of
 *     gdn_prefill_host_workspace_size bytes, 256-byte aligned
 * When the call returns, the work is queued on `stream`; synchronising `stream`
 * waits for the last output copy too.
 */
size_t gdn_prefill_host_workspace_size(const gdn_config* cfg, int64_t T_total, int32_t n_seqs);
gdn_status gdn_prefill_host(const gdn_config* cfg, const gdn_weights* w,
                            const void* q, const void* k, const void* v,
                            const void* a, const void* b, const void* z,
                            void* conv_state, void* rec_state, const int32_t* cu_seqlens,
                            int32_t n_seqs, int64_t T_total, void* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Capacity, in bytes, of the fixed scratch array used by gdn_prefill_noalloc. */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * gdn_prefill_noalloc -- gdn_prefill for callers that cannot allocate device
 * memory.  The pages have no counterpart of this call; it exists only for such
 * callers.  Examples: a server whose device memory is all carved into its own
 * pool at start-up, or a latency-critical caller that cannot afford the
 * implicit device synchronisation of cudaMalloc/cudaFree.  Either way the caller
 * cannot provide a gdn_prefill workspace.
 *
 * Arguments and results are those of gdn_prefill without `workspace` /
 * `workspace_bytes`.  The caller still provides every input and output buffer.
 * The scratch is one file-scope device array of GDN_NOALLOC_SCRATCH_BYTES
 * (64 MiB).  It is allocated when the library's module is loaded on a GPU, and
 * every GPU that loads the library keeps it until the process exits.  This call
 * allocates nothing itself: no cudaMalloc, no cudaFree, no allocating library
 * routine.
 *
 *   - Size limit: a request needing more than GDN_NOALLOC_SCRATCH_BYTES of
 *     workspace is rejected with GDN_ERR_WORKSPACE, before any launch.  The
 *     needed size is gdn_prefill_workspace_size(cfg, T_total, n_seqs).  At the
 *     published shape that is 76,544 bytes per token plus about 3.6 MB per
 *     sequence, so up to 823 tokens in one sequence.  Longer prompts can be
 *     split into consecutive calls, since the states carry from one call to
 *     the next.
 *   - First call on a device: it looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current), then reuses it.  Make
 *     this first call before any stream capture.
 *   - Shared contents: all calls on a device share the one array, which keeps
 *     the last call's contents.  Nothing in it needs to start at zero: each
 *     call writes every scratch element it reads.
 *   - Races: calls whose work overlaps on the GPU (different streams, no
 *     ordering between them) race on the array.  Order them on one stream, or
 *     with events.
 *   - Device reset: the looked-up address belongs to the device's current
 *     context.  The call remembers that context and looks the address up
 *     again when a later call finds a different one (after cudaDeviceReset,
 *     for instance).
 */
gdn_status gdn_prefill_noalloc(const gdn_config* cfg, const gdn_weights* w,
                               const void* q, const void* k, const void* v,
                               const void* a, const void* b, const void* z,
                               void* conv_state, void* rec_state,
                               const int32_t* cu_seqlens, int32_t n_seqs, int64_t T_total,
                               void* out, void* stream);

/* Synchronises `stream`, then reads and clears the device error word that
 * bounded waits and the prefill's device checks write.  GDN_OK, or the most
 * serious error recorded since the last call: GDN_ERR_DEVICE_TIMEOUT, then
 * GDN_ERR_SEQLENS, then GDN_ERR_RANGE; GDN_ERR_CUDA if a CUDA call failed. */
gdn_status gdn_check_device_error(void* stream);

/* Static string for a status code. */
const char* gdn_status_string(gdn_status s);

/* The CUDA error behind the calling thread's most recent GDN_ERR_CUDA, as
 * "name: description" ("no CUDA error" if there was none).  The string belongs
 * to the calling thread and stays valid until its next call of this function. */
const char* gdn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_H */
