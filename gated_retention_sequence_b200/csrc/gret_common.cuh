// Shared device helpers and launch descriptors of libgret (internal header).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gret.h"

namespace gret {

// Status word values a kernel writes when it gives up: a bounded wait ran out
// (host: GRET_ERR_TIMEOUT), or the dynamic shared memory base was not aligned
// enough for the kernel's layout and it did nothing (host: GRET_ERR_CUDA).
// Kernels never trap.
enum : unsigned int { kDevOk = 0u, kDevTimeout = 1u, kDevSmemLayout = 2u };

// Token rows row0 .. row0 + len - 1 of sequence b in a packed batch of `total`
// rows, clamped into [0, total] so that malformed offsets can neither address
// memory outside the tensors nor give a negative row.
__device__ __forceinline__ void packed_range(const int* cu, int b, int total, int& row0, int& len) {
    int a0 = cu[b], a1 = cu[b + 1];
    a0 = a0 < 0 ? 0 : (a0 > total ? total : a0);
    a1 = a1 < a0 ? a0 : (a1 > total ? total : a1);
    row0 = a0;
    len = a1 - a0;
}

struct PrefillArgs {
    const void* Q;
    const void* K;
    const void* V;
    const float* z;
    const void* G;
    void* O;
    float* S_final;
    const float* S0;          // initial state [B][H][dk][dv] fp32, or null for zero
    // packed variable-length batch: B sequences, sequence b holds token rows
    // cu_seqlens[b] .. cu_seqlens[b + 1] - 1 of [total][H][d] tensors (device
    // array), N is the longest; null for the uniform [B][N][H][d] layout
    const int* cu_seqlens;
    int total;
    // state-only pass (sequence-parallel prefill): no outputs; the state
    // increment goes to S_final and the slice's total log-decay to decay_out
    int state_only;
    float* decay_out;
    int B, H, N, dk, dv, chunk;
    float inv_tau, eps;
    gret_dtype io;
    gret_epilogue epi;
    void* workspace;
    size_t workspace_bytes;
    unsigned int* status;     // device status word
    int segments;             // sequence segments per unit (TC path)
    int seg_len;              // tokens per segment (multiple of chunk)
    int pieces;               // state-pass pieces per segment (divides seg_len / chunk)
    int fault;                // test only: inject a timed-out wait (gret_debug_inject_timeout)
    // resumed prefill (gret_prefill_resume): the workspace already holds the
    // decay sums and the folded state-pass pieces of these tokens; pieces is
    // then the state pass's pieces per segment
    int resume;
    int num_sms;              // the device's SM count (plans of packed batches)
    // gate projection (gret_prefill_projected): when X is set, the gate logits
    // are z = X W_gamma, computed by the tensor-core path's gate prologue;
    // X [B][N][d_model] bf16, Wg [d_model][H] fp32
    const void* X;
    const float* Wg;
    int d_model;
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* z;
    const void* g;
    float* S;
    void* o;
    int num_units, H, dk, dv;
    float inv_tau, eps;
    gret_dtype io;
    gret_epilogue epi;
};

// Gate ("YOCO 深度技术分析", section 2.2): gamma = sigmoid(z)^(1/tau), kept in
// log space: log gamma = -softplus(-z) / tau with
// softplus(x) = max(x, 0) + log1p(exp(-|x|)).  Clamped at kMinLogGamma: a
// token with gamma below e^-64 (about 1.6e-28) is treated as gamma = e^-64.
// This keeps z = -inf (gamma = 0) from producing -inf - (-inf) in the
// chunk-local sums, and keeps those fp32 sums small enough that the decay
// between two later tokens (a difference of two sums) keeps its precision.
constexpr float kMinLogGamma = -64.0f;
__device__ __forceinline__ float log_gamma(float z, float inv_tau) {
    float x = -z;
    float sp = fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
    return fmaxf(-sp * inv_tau, kMinLogGamma);
}

// P-block factors of the tensor-core prefill.  The P step forms
// e^{b_t - b_s} as e^{b_t - b_{s0}} E_s with E_s = e^{b_{s0} - b_s}, s0 the
// first token of s's block of C/4 columns (16 or 32 tokens, within one warp).
// A block whose log-decay drops by more than kBlockMax gets E_{s0} = -1 (and
// 0 elsewhere) instead, so the P step takes the exponentials directly there.
// x is this lane's chunk-local decay sum b; every lane of the warp calls this.
constexpr float kBlockMax = 40.0f;
__device__ __forceinline__ float p_block_factor(float x, int lane, int bw) {
    const float x0 = __shfl_sync(0xffffffffu, x, lane & ~(bw - 1));
    const float xl = __shfl_sync(0xffffffffu, x, lane | (bw - 1));
    float e = expf(x0 - x);
    if (x0 - xl > kBlockMax) e = (lane & (bw - 1)) == 0 ? -1.f : 0.f;
    return e;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Events gret_set_profile_events armed for this host thread (null when off),
// and those of gret_set_gate_profile_events (around the gate prologue).
extern thread_local cudaEvent_t g_profile_start;
extern thread_local cudaEvent_t g_profile_stop;
extern thread_local cudaEvent_t g_profile_gate_start;
extern thread_local cudaEvent_t g_profile_gate_stop;

// Host-side launchers (one per kernel family).
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s);
size_t prefill_simt_smem_bytes(int dk, int dv, int chunk);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s);

// Backward of the prefill (CUDA cores, gret_backward.cu).
struct BackwardArgs {
    const void *Q, *K, *V, *G, *dO;
    const float *z, *S0, *dS_final;
    void *dQ, *dK, *dV, *dG;
    float *dz, *dS0;
    void* workspace;
    int B, H, N, dk, dv;
    float inv_tau, eps;
    int gn;
    gret_dtype io;
    unsigned int* status;     // device status word (tensor-core path)
};
size_t prefill_backward_workspace_bytes(int B, int H, int N, int dk, int dv, gret_dtype io);
bool prefill_backward_supported(int dk, int dv);
// launches one backward call makes (6 on the tensor-core path, 5 on the chunk-parallel
// CUDA-core path, 2 on the serial one)
int prefill_backward_launches(int B, int H, int N, int dk, int dv, gret_dtype io);
cudaError_t launch_prefill_backward(const BackwardArgs& a, cudaStream_t s);
// chunk-parallel backward (gret_backward_chunk.cu): head sizes multiples of 32,
// dk <= 128, dv <= 256
bool bwd_chunked_supported(int B, int H, int N, int dk, int dv, gret_dtype io);
size_t bwd_chunked_workspace_bytes(int B, int H, int N, int dk, int dv, gret_dtype io);
cudaError_t launch_bwd_chunked(const BackwardArgs& a, cudaStream_t s);
// tensor-core backward (gret_backward_tc.cu): bf16, dk = 128, dv of 128 or 256
bool bwd_tc_supported(int B, int H, int N, int dk, int dv, gret_dtype io);
size_t bwd_tc_workspace_bytes(int B, int H, int N, int dv);
cudaError_t launch_bwd_tc(const BackwardArgs& a, cudaStream_t s);
// state-only pass of the tensor-core path (a.state_only): workspace bytes and launch
size_t prefill_tc_state_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk, int num_sms);
int prefill_tc_state_pieces(int B, int H, int chunk, int num_sms, int segments, int seg_len);
cudaError_t launch_prefill_state_tc(const PrefillArgs& a, int num_sms, cudaStream_t s);
// S_in = fold over slices q < slice of (decay_q, dS_q), from S0 or zero
cudaError_t launch_state_fold(const float* dS_all, const float* decay_all, int num_slices, int slice,
                              const float* S0, float* S_in, int units, int elems, cudaStream_t s);
bool prefill_tc_supported(int dk, int dv, int chunk, gret_dtype io);
// gate projection (gret_gate_project.cu): the fused tensor-core prologue, which
// writes the decay sums and P-block factors, and a CUDA-core projection to z
int gate_project_heads_padded(int H);
bool gate_project_tc_supported(int H, int d_model);
size_t gate_project_tc_ws_bytes(int H, int d_model);
cudaError_t launch_gate_project_tc(const PrefillArgs& a, float* bcum, float* eblk, int Npad, void* wsplit,
                                   cudaStream_t s);
cudaError_t launch_gate_project_simt(const PrefillArgs& a, float* z, cudaStream_t s);
// ctas_per_item: CTAs that run one fused work item (2 for the d_v = 256 pair).
void prefill_tc_plan(int B, int H, int N, int chunk, int num_sms, int* segments, int* seg_len, int* pieces,
                     int ctas_per_item = 1);
int prefill_tc_ctas_per_item(int dv, int chunk);
size_t prefill_tc_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk, int segments, int pieces);
size_t prefill_tc_varlen_workspace_bytes(int S, int H, int max_seqlen, int total, int dk, int dv, int chunk,
                                         int num_sms);
// Launches of a packed batch on the tensor-core path: 3, or 5 where max_seqlen
// allows a sequence to be cut (state pass and combine).
int prefill_tc_varlen_launches(int S, int H, int max_seqlen, int total, int dk, int dv, int chunk, int num_sms);
int prefill_tc_launches(int segments, int pieces);

}  // namespace gret
