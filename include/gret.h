/*
 * libgret -- gated retention (gRet) mixer on NVIDIA B200 (sm_100a).
 *
 * C ABI: plain pointers and sizes, no C++ or framework types.  Every call is
 * asynchronous on the given stream, allocates nothing and never throws; errors
 * come back as a gret_status.  All tensor pointers are DEVICE pointers owned
 * by the caller unless stated otherwise.
 *
 * What the mixer computes (web pages on the YOCO decoder-decoder family):
 *  - "YOCO 深度技术分析", section 2.2 "Gated Retention (gRet)":
 *      gate            gamma_n = sigmoid(z_n)^(1/tau), z = x W_gamma, one scalar
 *                      per token and head ("head-wise gate")
 *      parallel form   Y = (Q K^T (.) D) V, D[n][m] = prod_{i=m+1..n} gamma_i
 *      recurrent form  S_n = gamma_n S_{n-1} + K_n^T V_n,  Y_n = Q_n S_n
 *      per-head output GroupNorm(Y) (.) swish(G)
 *  - same page, section 5.3.2: the chunkwise form (parallel inside a block of
 *    `chunk` tokens, recurrent between blocks) is exactly equivalent; prefill
 *    uses it, decode uses the recurrent form (section 5.3.7), and prefill hands
 *    its last state to decode.
 * No 1/sqrt(d_k) scale is applied (none appears in either form).  GroupNorm
 * normalises the d_v channels of one token of one head with the biased
 * variance and `eps`, without affine parameters; swish(g) = g * sigmoid(g).
 *
 * Layouts (row-major, contiguous, element strides only):
 *   Q, K        [B][N][H][dk]   io dtype
 *   V, G, O     [B][N][H][dv]   io dtype
 *   gate_logits [B][N][H]       fp32 (z; the gate stays fp32 in both paths)
 *   S           [B][H][dk][dv]  fp32, d_v fastest
 * The decode step uses the same layouts with N = 1 and B = num_seqs.
 */
#ifndef GRET_H
#define GRET_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st* gret_stream_t;

typedef enum {
    GRET_OK = 0,
    GRET_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, non-positive size, bad enum */
    GRET_ERR_UNSUPPORTED = 2,   /* valid arguments outside what the kernels implement */
    GRET_ERR_CUDA = 3,          /* a CUDA runtime/driver call or kernel launch failed */
    GRET_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up (see below) */
} gret_status;

typedef enum { GRET_F32 = 0, GRET_BF16 = 1 } gret_dtype;

typedef enum {
    GRET_EPI_GN_SWISH = 0,      /* O = GroupNorm(Y) (.) swish(G)                    */
    GRET_EPI_NONE = 1           /* O = Y (pre-norm output; G is ignored, may be NULL) */
} gret_epilogue;

/* Kernel a prefill call runs (see gret_prefill_path). */
typedef enum {
    GRET_PATH_NONE = 0,         /* arguments are unsupported                         */
    GRET_PATH_SIMT = 1,         /* fp32 CUDA-core chunkwise kernel (any io dtype)    */
    GRET_PATH_TC = 2            /* tcgen05/TMEM tensor-core chunkwise kernel (bf16)  */
} gret_path;

/*
 * gret_prefill -- chunkwise prefill of B x H independent (batch, head) units.
 *
 *   Q, K, V, gate_logits, G : inputs (layouts above).  G may be NULL when
 *                             epi == GRET_EPI_NONE.
 *   tau                     : gate temperature, > 0.
 *   chunk                   : block length of the chunkwise form.  Supported:
 *                             16, 32, 64, 128, 256 (TC path: 64 or 128; 256,
 *                             the pages' own block size (section 5.3.8), runs
 *                             on the CUDA-core kernel, which works through a
 *                             chunk in blocks of rows and columns when the
 *                             whole chunk does not fit in shared memory).
 *   O                       : output [B][N][H][dv] in io_dtype; must not alias an input.
 *   S_final                 : fp32 [B][H][dk][dv] state after the last token, or NULL.
 *   B, H, N, dk, dv         : > 0; dk, dv multiples of 16 and <= 256.
 *   eps                     : GroupNorm epsilon (>= 0); 1e-5 is the usual value.
 *   workspace, workspace_bytes : device scratch of at least
 *                             gret_prefill_workspace_size(...) bytes, 256-byte
 *                             aligned; may be NULL when that size is 0.  Its
 *                             contents on entry do not matter.
 * The prefill starts from the zero state.  Pointers must be 16-byte aligned.
 * Calls that share a workspace must not overlap on the GPU.
 */
gret_status gret_prefill(const void* Q, const void* K, const void* V, const float* gate_logits,
                         const void* G, float tau, int chunk, void* O, float* S_final,
                         int B, int H, int N, int dk, int dv, gret_dtype io_dtype, float eps,
                         gret_epilogue epi, void* workspace, size_t workspace_bytes,
                         gret_stream_t stream);

/*
 * gret_prefill_from_state -- gret_prefill that continues from a given state.
 *
 * "YOCO 深度技术分析", sections 5.3.2 and 5.3.3: between blocks, and between
 * the devices of Chunk Parallelism, the only thing carried forward is the
 * state S; a prefill that starts from S0 instead of zero is the step that
 * continues a sequence (the next piece of a chunked prefill, or the next
 * device's slice of a long one).  With S0 = S_prev the result equals one
 * gret_prefill over the concatenated tokens, up to rounding.
 *
 *   S0 : fp32 [B][H][dk][dv] state before the first token (DEVICE, read
 *        only), or NULL for the zero state (then this is gret_prefill).
 *        16-byte aligned; must not overlap S_final (units are split into
 *        segments that run concurrently, so S_final may be written before
 *        every segment has read S0): keep two state buffers and alternate.
 * Every other argument, the workspace size and the errors are those of
 * gret_prefill; an S0 that overlaps S_final returns GRET_ERR_INVALID_ARG.
 */
gret_status gret_prefill_from_state(const void* Q, const void* K, const void* V, const float* gate_logits,
                                    const void* G, const float* S0, float tau, int chunk, void* O,
                                    float* S_final, int B, int H, int N, int dk, int dv,
                                    gret_dtype io_dtype, float eps, gret_epilogue epi, void* workspace,
                                    size_t workspace_bytes, gret_stream_t stream);

/*
 * gret_prefill_varlen -- prefill of a packed batch of sequences of different
 * lengths (the layout a serving batch of prompts has), each from its own
 * initial state or zero.
 *
 *   Q, K        [total_tokens][H][dk]   io dtype
 *   V, G, O     [total_tokens][H][dv]   io dtype
 *   gate_logits [total_tokens][H]       fp32
 *   cu_seqlens  int32 [num_seqs + 1] (DEVICE): sequence b is token rows
 *               cu_seqlens[b] .. cu_seqlens[b + 1] - 1, so cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[num_seqs] = total_tokens; a sequence
 *               may be empty (its S_final is then S0, or zero).
 *   max_seqlen  the longest sequence (>= every length; sizes the work split).
 *   S0, S_final fp32 [num_seqs][H][dk][dv]; S0 may be NULL (zero state); the
 *               rule of gret_prefill_from_state on overlap applies.
 * Workspace: gret_prefill_varlen_workspace_size(num_seqs, total_tokens,
 * max_seqlen, H, dk, dv, chunk, io_dtype) bytes.  Every sequence gives what
 * gret_prefill_from_state gives for it alone; nothing is written outside its
 * rows.  Offsets outside [0, total_tokens] are clamped into it; tokens past
 * max_seqlen in a sequence are not processed.  cu_seqlens must be 4-byte
 * aligned; total_tokens > 0.
 *
 * On the tensor-core path the work is planned on the device from cu_seqlens
 * (no host synchronisation): a sequence longer than one and a half work
 * slots' share (a slot is an SM, or an SM pair for dv = 256) of the batch's
 * tokens and heads is cut into segments of equal length -- a state pass gives
 * each segment its initial state -- while the others stay whole, and the
 * segments start longest first, so that one long prompt among short ones does
 * not finish alone.  Where max_seqlen is within that bound no sequence is cut
 * and the state pass is not launched.  The call then makes
 * gret_prefill_varlen_launches(...) launches.
 */
gret_status gret_prefill_varlen(const void* Q, const void* K, const void* V, const float* gate_logits,
                                const void* G, const float* S0, const int* cu_seqlens, int num_seqs,
                                int total_tokens, int max_seqlen, float tau, int chunk, void* O,
                                float* S_final, int H, int dk, int dv, gret_dtype io_dtype, float eps,
                                gret_epilogue epi, void* workspace, size_t workspace_bytes,
                                gret_stream_t stream);
size_t gret_prefill_varlen_workspace_size(int num_seqs, int total_tokens, int max_seqlen, int H, int dk, int dv,
                                          int chunk, gret_dtype io_dtype);
int gret_prefill_varlen_launches(int num_seqs, int total_tokens, int max_seqlen, int H, int dk, int dv, int chunk,
                                 gret_dtype io_dtype);

/*
 * Sequence-parallel prefill ("YOCO 深度技术分析", section 5.3.3, Chunk
 * Parallelism: the devices holding consecutive slices of one sequence pass
 * only the state between them).  For P slices of the same B x H units:
 *
 *   1. each slice: gret_prefill_state -> its increment dS_p (the final state
 *      of a zero-state prefill of the slice alone) and its total log-decay
 *      a_p = sum of log gamma over the slice;
 *   2. exchange (dS_p, a_p) among the slices (an all-gather across devices);
 *   3. each slice: gret_state_fold -> S_in(p) = e^{a_{p-1}} S_in(p-1) + dS_{p-1},
 *      S_in(0) = S0 or zero (the state decomposition of the recurrence);
 *   4. each slice: gret_prefill_from_state(..., S0 = S_in(p), ...).
 *
 * gret_prefill_state -- step 1.  K [B][N][H][dk], V [B][N][H][dv] (io dtype),
 * gate_logits [B][N][H] fp32; dS fp32 [B][H][dk][dv]; decay fp32 [B][H].
 * Workspace: gret_prefill_state_workspace_size(...) bytes, 256-byte aligned.
 * Q, G and O play no part.
 */
size_t gret_prefill_state_workspace_size(int B, int H, int N, int dk, int dv, int chunk, gret_dtype io_dtype);
gret_status gret_prefill_state(const void* K, const void* V, const float* gate_logits, float tau, int chunk,
                               float* dS, float* decay, int B, int H, int N, int dk, int dv,
                               gret_dtype io_dtype, void* workspace, size_t workspace_bytes,
                               gret_stream_t stream);

/*
 * gret_prefill_resume -- step 4 of a rank that ran gret_prefill_state on the
 * same tokens: gret_prefill_from_state(Q, K, V, gate_logits, G, S0, ...) that
 * takes the decay sums and the state pass's pieces from `workspace`, where
 * gret_prefill_state left them, instead of computing them again.  The state
 * pass folded its pieces from the zero state; this call adds S0 carried
 * through each piece's decay (S(x || y) = e^{sum log gamma(y)} S(x) + S(y),
 * the state decomposition) and runs the fused chunk loop: K, V and the gate
 * are read once by the state pass and once here, as in a single-device
 * prefill.  Arguments as gret_prefill_from_state; `workspace` must be the one
 * gret_prefill_state was given (at least gret_prefill_state_workspace_size
 * bytes) with the same K, V, gate_logits, tau, chunk, B, H, N, dk, dv and io
 * dtype and nothing written to it in between (otherwise the result is
 * undefined).  gate_logits is not read again.  On the CUDA-core path the call
 * is gret_prefill_from_state.
 */
gret_status gret_prefill_resume(const void* Q, const void* K, const void* V, const float* gate_logits,
                                const void* G, const float* S0, float tau, int chunk, void* O, float* S_final, int B,
                                int H, int N, int dk, int dv, gret_dtype io_dtype, float eps, gret_epilogue epi,
                                void* workspace, size_t workspace_bytes, gret_stream_t stream);

/*
 * gret_state_fold -- step 3.  dS_all fp32 [num_slices][B][H][dk][dv] and
 * decay_all fp32 [num_slices][B][H] as gathered; writes S_in fp32
 * [B][H][dk][dv] for slice `slice` (0 <= slice <= num_slices; slice =
 * num_slices gives the state after the whole sequence).  S0 may be NULL (zero)
 * and may be S_in itself; dS_all/decay_all may be NULL when slice = 0.
 */
gret_status gret_state_fold(const float* dS_all, const float* decay_all, int num_slices, int slice,
                            const float* S0, float* S_in, int B, int H, int dk, int dv, gret_stream_t stream);

/*
 * gret_prefill_backward -- gradients of the prefill (for training).
 *
 * The pages give the forward; this is its exact derivative.  For an upstream
 * gradient dO of O (and optionally dS_final of S_final), returns the gradients
 * of <O, dO> + <S_final, dS_final> with respect to Q, K, V (io dtype, their
 * layouts), the gate logits dz (fp32 [B][N][H]), G (io dtype; GN_SWISH only)
 * and the initial state dS0 (fp32 [B][H][dk][dv]; may be NULL).  S0 and
 * dS_final may be NULL (zero).  Accumulation is fp32 throughout.
 *
 * bf16 inputs with dk = 128 and dv = 128 or 256 take the tensor-core path
 * (6 launches, chunks of 128 tokens, tcgen05 products with fp32 accumulation;
 * the per-chunk states, state gradients and dy enter the products as bf16
 * pairs hi + lo, about 16 mantissa bits).  Its workspace holds, per chunk, an
 * fp32 state-shaped buffer and a state as a bf16 pair (B*H*ceil(N/128)*
 * dk*dv*(4 + 4) bytes in all), dy as a bf16 pair (B*N*H*dv*4), two fp32 terms
 * per token and head, and per chunk dv + 641 fp32 values (among them the
 * decay sums of its 128 tokens).  Other head sizes
 * that are multiples of 32 with dk <= 128 and dv <= 256 take the chunk-parallel
 * path on CUDA cores in fp32 (5 launches; chunks of 64 tokens for bf16, 32 for
 * fp32), whose workspace holds the state before every chunk and the gradient
 * at every chunk's end (2 * B*H*ceil(N/chunk)*dk*dv*4 bytes), the gradient of
 * the pre-norm output (B*N*H*dv*4) and one decay per chunk.  Other head sizes
 * (multiples of 16 up to 256) take a serial path (2 launches) that keeps the
 * state at every 32-token block (B*H*ceil(N/32)*dk*dv*4 plus one state per
 * unit) and walks the blocks in reverse.  The size depends on io_dtype; 0 for
 * an unsupported shape.  Where the forward clamps a log-decay at -64 the gate
 * gradient is zero.  A bounded device wait that gives up on the tensor-core
 * path is reported by gret_last_device_status.
 */
size_t gret_prefill_backward_workspace_size(int B, int H, int N, int dk, int dv, gret_dtype io_dtype);
/* Kernel launches one gret_prefill_backward call makes for this shape (0 if unsupported). */
int gret_prefill_backward_launches(int B, int H, int N, int dk, int dv, gret_dtype io_dtype);
gret_status gret_prefill_backward(const void* Q, const void* K, const void* V, const float* gate_logits,
                                  const void* G, const float* S0, const void* dO, const float* dS_final,
                                  float tau, float eps, gret_epilogue epi, void* dQ, void* dK, void* dV,
                                  float* dz, void* dG, float* dS0, int B, int H, int N, int dk, int dv,
                                  gret_dtype io_dtype, void* workspace, size_t workspace_bytes,
                                  gret_stream_t stream);

/* Size of the device scratch array gret_prefill_noalloc draws on (32 MiB). */
#define GRET_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * gret_prefill_noalloc -- gret_prefill without a workspace argument, for
 * callers that cannot allocate device memory: plugins and custom-op hosts that
 * are handed only the tensors' device pointers and have no allocator of their
 * own to ask, and code paths where calling cudaMalloc is not allowed because
 * it can synchronise the device or take memory from a pool someone else owns.
 * The pages describe no such entry point; it is an addition of this library.
 *
 * Arguments, layouts and results are those of gret_prefill.  Instead of a
 * caller workspace the call uses a fixed array of GRET_NOALLOC_SCRATCH_BYTES
 * that the library reserves in device memory on every GPU that loads it, for
 * the life of the process.  Calls whose gret_prefill_workspace_size exceeds
 * that return GRET_ERR_UNSUPPORTED before touching the GPU.  The call
 * allocates nothing itself.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the one array, and nothing in
 * it needs clearing between calls (each call writes what it reads), but two
 * calls whose work overlaps on the GPU (different streams, or different host
 * threads on one device) race on it: serialise them.
 */
gret_status gret_prefill_noalloc(const void* Q, const void* K, const void* V, const float* gate_logits,
                                 const void* G, float tau, int chunk, void* O, float* S_final,
                                 int B, int H, int N, int dk, int dv, gret_dtype io_dtype, float eps,
                                 gret_epilogue epi, gret_stream_t stream);

/* Device scratch (bytes) gret_prefill needs for these arguments; 0 if none.
 * Returns 0 as well for unsupported arguments (gret_prefill then reports them). */
size_t gret_prefill_workspace_size(int B, int H, int N, int dk, int dv, int chunk,
                                   gret_dtype io_dtype);

/* How many kernels one gret_prefill call with these arguments launches on its
 * stream (gate scan, fused chunk loop, and for a split sequence the state pass
 * and, with many pieces, the combine pass); 0 for unsupported arguments. */
int gret_prefill_launches(int B, int H, int N, int dk, int dv, int chunk, gret_dtype io_dtype);

/* Which kernel gret_prefill would run for these arguments, and into how many
 * sequence segments it splits each unit (1 = no split).  segments may be NULL. */
gret_path gret_prefill_path(int B, int H, int N, int dk, int dv, int chunk, gret_dtype io_dtype,
                            int* segments);

/*
 * gret_decode_step -- one recurrent step for num_seqs x H units
 * ("YOCO 深度技术分析" sections 2.2 and 5.3.7):
 *     S <- gamma S + k^T v ;  y = q S ;  o = GroupNorm(y) (.) swish(g)
 *   q, k        [num_seqs][H][dk] io dtype
 *   v, g, o     [num_seqs][H][dv] io dtype (g may be NULL when epi == GRET_EPI_NONE)
 *   gate_logit  [num_seqs][H] fp32
 *   S_inout     [num_seqs][H][dk][dv] fp32, updated in place
 * o must not alias any input or S_inout.  Pointers must be 16-byte aligned;
 * dk, dv multiples of 16 and <= 256.
 */
gret_status gret_decode_step(const void* q, const void* k, const void* v, const float* gate_logit,
                             const void* g, float* S_inout, void* o, int num_seqs, int H, int dk,
                             int dv, float tau, gret_dtype io_dtype, float eps, gret_epilogue epi,
                             gret_stream_t stream);

/* Synchronises `stream`, then reports (and clears) the device status word that
 * kernels set when they give up: GRET_ERR_TIMEOUT when a bounded wait (an
 * mbarrier or tensor-memory wait) ran out; GRET_ERR_CUDA when a kernel found
 * its dynamic shared memory base too poorly aligned for its layout, or when the
 * stream reports an error; else GRET_OK.  Kernels never trap; a kernel that
 * gave up returns early and its outputs are undefined. */
gret_status gret_last_device_status(gret_stream_t stream);

/*
 * gret_prefill_projected -- gret_prefill whose gate logits come from the gate
 * projection itself.
 *
 * "YOCO 深度技术分析", section 2.2: gamma = sigmoid(X W_gamma)^(1/tau), with one
 * column of W_gamma per head, so z[b][n][h] = sum_i X[b][n][i] W_gamma[i][h].
 * On the tensor-core path (bf16, as gret_prefill_path reports) with H <= 128
 * and d_model a multiple of 8, z is a tcgen05 product inside the kernel that
 * scans the gate (W_gamma fed as two bf16 halves for fp32-level accuracy) and
 * never reaches memory; elsewhere a CUDA-core kernel writes z into the
 * workspace first.  Everything else is gret_prefill.
 *
 *   X         [B][N][d_model] in io_dtype, the mixer's input rows
 *   W_gamma   [d_model][H] fp32
 *   workspace at least gret_prefill_projected_workspace_size(...) bytes
 * Pointers must be 16-byte aligned.  Same errors as gret_prefill.
 */
gret_status gret_prefill_projected(const void* Q, const void* K, const void* V, const void* X,
                                   const float* W_gamma, int d_model, const void* G, float tau, int chunk,
                                   void* O, float* S_final, int B, int H, int N, int dk, int dv,
                                   gret_dtype io_dtype, float eps, gret_epilogue epi, void* workspace,
                                   size_t workspace_bytes, gret_stream_t stream);
size_t gret_prefill_projected_workspace_size(int B, int H, int N, int dk, int dv, int chunk, int d_model,
                                             gret_dtype io_dtype);

/* Test aid for the give-up path of the bounded device waits.  The next `calls`
 * prefill calls that run the tensor-core kernels (any gret_prefill* entry
 * point on that path, from any host thread) make the fused kernel's TMA warp,
 * before it issues any load, wait on an mbarrier that nothing ever arrives at,
 * with a budget of about 2^20 cycles.  The wait runs out, the kernel records
 * GRET_ERR_TIMEOUT in the device status word, every role of the CTA stops
 * issuing work, the work already issued is awaited, and the kernel returns.
 * The call's outputs are then undefined; gret_last_device_status reports
 * GRET_ERR_TIMEOUT once and clears it, and later calls run normally.  No GPU
 * fault, trap or hang is involved.  `calls` <= 0 cancels pending injections.
 * Not for production use. */
void gret_debug_inject_timeout(int calls);

/* Profiling aid.  While set (non-NULL), every gret_prefill call made from the
 * calling host thread records `start` on its stream just before the launch of
 * the fused chunk-loop kernel (the dominant kernel of a prefill) and `stop`
 * just after it, so that cudaEventElapsedTime gives that kernel's duration.
 * Both are cudaEvent_t handles owned by the caller; pass NULL, NULL to stop. */
void gret_set_profile_events(void* start, void* stop);

/* The same for the gate prologue of a prefill (the gate scan, or on the
 * tensor-core path of gret_prefill_projected the fused projection and scan;
 * the CUDA-core projection of the other paths). */
void gret_set_gate_profile_events(void* start, void* stop);

/* Static, human-readable name of a status code. */
const char* gret_status_string(gret_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int gret_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GRET_H */
