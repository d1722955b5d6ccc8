// libgret C ABI: argument validation, kernel selection and launch.
//
// Nothing here allocates device memory, copies tensors or touches data: every
// step of the mixer runs in the kernels.  Validation happens before any launch
// so that a bad call has no effect on the stream.
#include <math.h>
#include <string.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "gret_common.cuh"

namespace gret {

thread_local cudaEvent_t g_profile_start = nullptr;
thread_local cudaEvent_t g_profile_stop = nullptr;
thread_local cudaEvent_t g_profile_gate_start = nullptr;
thread_local cudaEvent_t g_profile_gate_stop = nullptr;

namespace {

__device__ unsigned int g_device_status;

constexpr int kMaxDevices = 64;
unsigned int* g_status_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
std::mutex g_mu;

// prefill calls on the tensor-core path still to carry an injected timeout
std::atomic<int> g_inject_timeouts{0};

// Take one pending injected timeout, if any.
int take_injected_timeout() {
    int n = g_inject_timeouts.load();
    while (n > 0 && !g_inject_timeouts.compare_exchange_weak(n, n - 1)) {
    }
    return n > 0 ? 1 : 0;
}

// Device status word and SM count of the current device (looked up once per
// device, with that device current).
bool device_info(unsigned int** status, int* num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return false;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        g_status_ptr[dev] = static_cast<unsigned int*>(p);
        g_num_sms[dev] = sms;
    }
    if (status) *status = g_status_ptr[dev];
    if (num_sms) *num_sms = g_num_sms[dev];
    return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_supported(int dk, int dv) {
    return dk % 16 == 0 && dv % 16 == 0 && dk <= 256 && dv <= 256;
}

bool chunk_supported(int chunk) {
    return chunk == 16 || chunk == 32 || chunk == 64 || chunk == 128 || chunk == 256;
}

constexpr size_t kMaxSmem = 227 * 1024;

// Chunk the tensor-core kernels run for a requested chunk.  The chunkwise form is
// the same function for every chunk length (only the rounding differs), so
// d_v = 256 runs 128-token chunks (the output-rows CTA pair), uniform or packed,
// whichever of 64 and 128 was asked.
int run_chunk(int dk, int dv, int chunk, gret_dtype io, bool packed) {
    (void)packed;
    if (io != GRET_BF16 || dk != 128 || dv != 256) return chunk;
    return chunk == 64 ? 128 : chunk;
}

// Kernel choice for a prefill; segments/seg_len describe the sequence split.
gret_path select_path(int B, int H, int N, int dk, int dv, int chunk, gret_dtype io, int num_sms,
                      int* segments, int* seg_len, int* pieces = nullptr) {
    if (segments) *segments = 1;
    if (seg_len) *seg_len = N;
    if (pieces) *pieces = 1;
    if (B <= 0 || H <= 0 || N <= 0 || dk <= 0 || dv <= 0) return GRET_PATH_NONE;
    if (io != GRET_F32 && io != GRET_BF16) return GRET_PATH_NONE;
    if (!shape_supported(dk, dv) || !chunk_supported(chunk)) return GRET_PATH_NONE;
    if (io == GRET_BF16 && prefill_tc_supported(dk, dv, chunk, io)) {
        int segs = 1, len = N, pcs = 1;
        prefill_tc_plan(B, H, N, chunk, num_sms, &segs, &len, &pcs, prefill_tc_ctas_per_item(dv, chunk));
        if (segments) *segments = segs;
        if (seg_len) *seg_len = len;
        if (pieces) *pieces = pcs;
        return GRET_PATH_TC;
    }
    if (prefill_simt_smem_bytes(dk, dv, chunk) <= kMaxSmem) return GRET_PATH_SIMT;
    return GRET_PATH_NONE;
}

}  // namespace
}  // namespace gret

using namespace gret;

extern "C" {

const char* gret_status_string(gret_status s) {
    switch (s) {
        case GRET_OK: return "GRET_OK";
        case GRET_ERR_INVALID_ARG: return "GRET_ERR_INVALID_ARG";
        case GRET_ERR_UNSUPPORTED: return "GRET_ERR_UNSUPPORTED";
        case GRET_ERR_CUDA: return "GRET_ERR_CUDA";
        case GRET_ERR_TIMEOUT: return "GRET_ERR_TIMEOUT";
    }
    return "GRET_ERR_UNKNOWN";
}

int gret_version(void) { return 10000; }

void gret_set_profile_events(void* start, void* stop) {
    g_profile_start = static_cast<cudaEvent_t>(start);
    g_profile_stop = static_cast<cudaEvent_t>(stop);
}

void gret_set_gate_profile_events(void* start, void* stop) {
    g_profile_gate_start = static_cast<cudaEvent_t>(start);
    g_profile_gate_stop = static_cast<cudaEvent_t>(stop);
}

gret_path gret_prefill_path(int B, int H, int N, int dk, int dv, int chunk, gret_dtype io_dtype,
                            int* segments) {
    chunk = run_chunk(dk, dv, chunk, io_dtype, false);
    int sms = 148;
    device_info(nullptr, &sms);
    return select_path(B, H, N, dk, dv, chunk, io_dtype, sms, segments, nullptr);
}

int gret_prefill_launches(int B, int H, int N, int dk, int dv, int chunk, gret_dtype io_dtype) {
    chunk = run_chunk(dk, dv, chunk, io_dtype, false);
    int sms = 148, segs = 1, pcs = 1;
    device_info(nullptr, &sms);
    gret_path p = select_path(B, H, N, dk, dv, chunk, io_dtype, sms, &segs, nullptr, &pcs);
    if (p == GRET_PATH_TC) return prefill_tc_launches(segs, pcs);
    return p == GRET_PATH_SIMT ? 1 : 0;
}

size_t gret_prefill_workspace_size(int B, int H, int N, int dk, int dv, int chunk,
                                   gret_dtype io_dtype) {
    chunk = run_chunk(dk, dv, chunk, io_dtype, false);
    int sms = 148, segs = 1, pcs = 1;
    device_info(nullptr, &sms);
    gret_path p = select_path(B, H, N, dk, dv, chunk, io_dtype, sms, &segs, nullptr, &pcs);
    if (p != GRET_PATH_TC) return 0;
    return prefill_tc_workspace_bytes(B, H, N, dk, dv, chunk, segs, pcs);
}

// Workspace of a projected prefill: the prefill's own, then the split gate
// weights (fused tensor-core prologue) or the gate logits (other paths).
static size_t projected_extra_bytes(gret_path path, int B, int H, int N, int d_model) {
    if (path == GRET_PATH_TC && gate_project_tc_supported(H, d_model)) return gate_project_tc_ws_bytes(H, d_model);
    return ((size_t)B * N * H * 4 + 255) & ~size_t(255);
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static gret_status prefill_impl(const void* Q, const void* K, const void* V, const float* gate_logits,
                                const void* G, const float* S0, const int* cu_seqlens, int total, float tau,
                                int chunk, void* O, float* S_final, int B, int H, int N, int dk, int dv,
                                gret_dtype io_dtype, float eps, gret_epilogue epi, void* workspace,
                                size_t workspace_bytes, gret_stream_t stream, const void* X = nullptr,
                                const float* W_gamma = nullptr, int d_model = 0, bool resume = false) {
    const bool projected = X != nullptr;
    if (projected) {
        if (!W_gamma || d_model <= 0 || !aligned16(X) || !aligned16(W_gamma) || cu_seqlens) return GRET_ERR_INVALID_ARG;
        gate_logits = static_cast<const float*>(X);     // validated below like the logits it replaces
    }
    if (!Q || !K || !V || !gate_logits || !O) return GRET_ERR_INVALID_ARG;
    if (epi != GRET_EPI_GN_SWISH && epi != GRET_EPI_NONE) return GRET_ERR_INVALID_ARG;
    if (epi == GRET_EPI_GN_SWISH && !G) return GRET_ERR_INVALID_ARG;
    if (io_dtype != GRET_F32 && io_dtype != GRET_BF16) return GRET_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || dk <= 0 || dv <= 0 || chunk <= 0) return GRET_ERR_INVALID_ARG;
    if (!(tau > 0.0f) || !isfinite(tau) || !(eps >= 0.0f) || !isfinite(eps)) return GRET_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(gate_logits) || !aligned16(O) ||
        (G && !aligned16(G)) || (S_final && !aligned16(S_final)) || (S0 && !aligned16(S0)))
        return GRET_ERR_INVALID_ARG;
    if ((long long)B * H > (1LL << 30) || (long long)B * N > (1LL << 40)) return GRET_ERR_UNSUPPORTED;
    if (cu_seqlens && ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0 || total <= 0)) return GRET_ERR_INVALID_ARG;
    if (S0 && S_final) {
        // segments of one unit run in different CTAs: S_final must not overwrite S0
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(S0), a1 = reinterpret_cast<uintptr_t>(S_final);
        if (a0 < a1 + bytes && a1 < a0 + bytes) return GRET_ERR_INVALID_ARG;
    }

    chunk = run_chunk(dk, dv, chunk, io_dtype, cu_seqlens != nullptr);
    unsigned int* status = nullptr;
    int sms = 0;
    if (!device_info(&status, &sms)) return GRET_ERR_CUDA;
    int segs = 1, seg_len = N, pcs = 1;
    gret_path path = select_path(B, H, N, dk, dv, chunk, io_dtype, sms, &segs, &seg_len, &pcs);
    if (path == GRET_PATH_NONE) return GRET_ERR_UNSUPPORTED;

    PrefillArgs a = {};
    a.Q = Q; a.K = K; a.V = V; a.z = gate_logits; a.G = G; a.O = O; a.S_final = S_final; a.S0 = S0;
    a.cu_seqlens = cu_seqlens; a.total = total;
    a.B = B; a.H = H; a.N = N; a.dk = dk; a.dv = dv; a.chunk = chunk;
    a.inv_tau = 1.0f / tau; a.eps = eps; a.io = io_dtype; a.epi = epi;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    a.status = status; a.segments = segs; a.seg_len = seg_len; a.pieces = pcs; a.num_sms = sms;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (resume && path == GRET_PATH_TC) {
        a.resume = 1;
        a.pieces = prefill_tc_state_pieces(B, H, chunk, sms, segs, seg_len);
    }
    const size_t base = path != GRET_PATH_TC ? 0
                        : cu_seqlens ? prefill_tc_varlen_workspace_bytes(B, H, N, total, dk, dv, chunk, sms)
                        : resume ? prefill_tc_state_workspace_bytes(B, H, N, dk, dv, chunk, sms)
                                 : prefill_tc_workspace_bytes(B, H, N, dk, dv, chunk, segs, pcs);
    const size_t need = align256(base) + (projected ? projected_extra_bytes(path, B, H, N, d_model) : 0);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return GRET_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GRET_ERR_INVALID_ARG;
    }
    if (projected) {
        a.X = X;
        a.Wg = W_gamma;
        a.d_model = d_model;
        if (!(path == GRET_PATH_TC && gate_project_tc_supported(H, d_model))) {
            // the gate logits first, into the workspace after the prefill's own
            float* z = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(base));
            err = launch_gate_project_simt(a, z, s);
            if (err != cudaSuccess) return GRET_ERR_CUDA;
            a.z = z;
            a.X = nullptr;
        }
    }
    if (path == GRET_PATH_TC) {
        a.fault = take_injected_timeout();
        err = launch_prefill_tc(a, s);
    } else {
        err = launch_prefill_simt(a, s);
    }
    return err == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

size_t gret_prefill_projected_workspace_size(int B, int H, int N, int dk, int dv, int chunk, int d_model,
                                             gret_dtype io_dtype) {
    if (d_model <= 0) return 0;
    chunk = run_chunk(dk, dv, chunk, io_dtype, false);
    int sms = 148, segs = 1, pcs = 1;
    device_info(nullptr, &sms);
    gret_path p = select_path(B, H, N, dk, dv, chunk, io_dtype, sms, &segs, nullptr, &pcs);
    if (p == GRET_PATH_NONE) return 0;
    const size_t base = p == GRET_PATH_TC ? prefill_tc_workspace_bytes(B, H, N, dk, dv, chunk, segs, pcs) : 0;
    return align256(base) + projected_extra_bytes(p, B, H, N, d_model);
}

gret_status gret_prefill_projected(const void* Q, const void* K, const void* V, const void* X,
                                   const float* W_gamma, int d_model, const void* G, float tau, int chunk,
                                   void* O, float* S_final, int B, int H, int N, int dk, int dv,
                                   gret_dtype io_dtype, float eps, gret_epilogue epi, void* workspace,
                                   size_t workspace_bytes, gret_stream_t stream) {
    if (!X) return GRET_ERR_INVALID_ARG;
    return prefill_impl(Q, K, V, nullptr, G, nullptr, nullptr, 0, tau, chunk, O, S_final, B, H, N, dk, dv,
                        io_dtype, eps, epi, workspace, workspace_bytes, stream, X, W_gamma, d_model);
}

void gret_debug_inject_timeout(int calls) { g_inject_timeouts.store(calls > 0 ? calls : 0); }

gret_status gret_prefill(const void* Q, const void* K, const void* V, const float* gate_logits,
                         const void* G, float tau, int chunk, void* O, float* S_final, int B, int H,
                         int N, int dk, int dv, gret_dtype io_dtype, float eps, gret_epilogue epi,
                         void* workspace, size_t workspace_bytes, gret_stream_t stream) {
    return prefill_impl(Q, K, V, gate_logits, G, nullptr, nullptr, 0, tau, chunk, O, S_final, B, H, N, dk, dv,
                        io_dtype, eps, epi, workspace, workspace_bytes, stream);
}

gret_status gret_prefill_from_state(const void* Q, const void* K, const void* V, const float* gate_logits,
                                    const void* G, const float* S0, float tau, int chunk, void* O,
                                    float* S_final, int B, int H, int N, int dk, int dv, gret_dtype io_dtype,
                                    float eps, gret_epilogue epi, void* workspace, size_t workspace_bytes,
                                    gret_stream_t stream) {
    return prefill_impl(Q, K, V, gate_logits, G, S0, nullptr, 0, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype,
                        eps, epi, workspace, workspace_bytes, stream);
}

gret_status gret_prefill_resume(const void* Q, const void* K, const void* V, const float* gate_logits,
                                const void* G, const float* S0, float tau, int chunk, void* O, float* S_final, int B,
                                int H, int N, int dk, int dv, gret_dtype io_dtype, float eps, gret_epilogue epi,
                                void* workspace, size_t workspace_bytes, gret_stream_t stream) {
    return prefill_impl(Q, K, V, gate_logits, G, S0, nullptr, 0, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype,
                        eps, epi, workspace, workspace_bytes, stream, nullptr, nullptr, 0, true);
}

size_t gret_prefill_varlen_workspace_size(int num_seqs, int total_tokens, int max_seqlen, int H, int dk, int dv,
                                          int chunk, gret_dtype io_dtype) {
    if (num_seqs <= 0 || total_tokens <= 0 || max_seqlen <= 0) return 0;
    chunk = run_chunk(dk, dv, chunk, io_dtype, true);
    int sms = 148;
    device_info(nullptr, &sms);
    if (select_path(num_seqs, H, max_seqlen, dk, dv, chunk, io_dtype, sms, nullptr, nullptr) != GRET_PATH_TC) return 0;
    return prefill_tc_varlen_workspace_bytes(num_seqs, H, max_seqlen, total_tokens, dk, dv, chunk, sms);
}

int gret_prefill_varlen_launches(int num_seqs, int total_tokens, int max_seqlen, int H, int dk, int dv, int chunk,
                                 gret_dtype io_dtype) {
    if (num_seqs <= 0 || total_tokens <= 0 || max_seqlen <= 0) return 0;
    chunk = run_chunk(dk, dv, chunk, io_dtype, true);
    int sms = 148;
    device_info(nullptr, &sms);
    const gret_path p = select_path(num_seqs, H, max_seqlen, dk, dv, chunk, io_dtype, sms, nullptr, nullptr);
    // tensor cores: gate scan, plan, (where a sequence may be cut) state pass
    // and combine, fused loop
    if (p == GRET_PATH_TC) return prefill_tc_varlen_launches(num_seqs, H, max_seqlen, total_tokens, dk, dv, chunk, sms);
    return p == GRET_PATH_SIMT ? 1 : 0;
}

gret_status gret_prefill_varlen(const void* Q, const void* K, const void* V, const float* gate_logits,
                                const void* G, const float* S0, const int* cu_seqlens, int num_seqs,
                                int total_tokens, int max_seqlen, float tau, int chunk, void* O, float* S_final,
                                int H, int dk, int dv, gret_dtype io_dtype, float eps, gret_epilogue epi,
                                void* workspace, size_t workspace_bytes, gret_stream_t stream) {
    if (!cu_seqlens) return GRET_ERR_INVALID_ARG;
    return prefill_impl(Q, K, V, gate_logits, G, S0, cu_seqlens, total_tokens, tau, chunk, O, S_final, num_seqs, H,
                        max_seqlen, dk, dv, io_dtype, eps, epi, workspace, workspace_bytes, stream);
}

gret_status gret_decode_step(const void* q, const void* k, const void* v, const float* gate_logit,
                             const void* g, float* S_inout, void* o, int num_seqs, int H, int dk,
                             int dv, float tau, gret_dtype io_dtype, float eps, gret_epilogue epi,
                             gret_stream_t stream) {
    if (!q || !k || !v || !gate_logit || !S_inout || !o) return GRET_ERR_INVALID_ARG;
    if (epi != GRET_EPI_GN_SWISH && epi != GRET_EPI_NONE) return GRET_ERR_INVALID_ARG;
    if (epi == GRET_EPI_GN_SWISH && !g) return GRET_ERR_INVALID_ARG;
    if (io_dtype != GRET_F32 && io_dtype != GRET_BF16) return GRET_ERR_INVALID_ARG;
    if (num_seqs <= 0 || H <= 0 || dk <= 0 || dv <= 0) return GRET_ERR_INVALID_ARG;
    if (!(tau > 0.0f) || !isfinite(tau) || !(eps >= 0.0f) || !isfinite(eps)) return GRET_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate_logit) ||
        !aligned16(S_inout) || !aligned16(o) || (g && !aligned16(g)))
        return GRET_ERR_INVALID_ARG;
    if (!shape_supported(dk, dv)) return GRET_ERR_UNSUPPORTED;
    if ((long long)num_seqs * H > (1LL << 31) - 1) return GRET_ERR_UNSUPPORTED;

    DecodeArgs a = {};
    a.q = q; a.k = k; a.v = v; a.z = gate_logit; a.g = g; a.S = S_inout; a.o = o;
    a.num_units = num_seqs * H; a.H = H; a.dk = dk; a.dv = dv;
    a.inv_tau = 1.0f / tau; a.eps = eps; a.io = io_dtype; a.epi = epi;
    cudaError_t err = launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

gret_status gret_last_device_status(gret_stream_t stream) {
    unsigned int* status = nullptr;
    if (!device_info(&status, nullptr)) return GRET_ERR_CUDA;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GRET_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpy(&word, status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return GRET_ERR_CUDA;
    if (word != kDevOk) {
        unsigned int zero = 0;
        if (cudaMemcpy(status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return GRET_ERR_CUDA;
        return word == kDevTimeout ? GRET_ERR_TIMEOUT : GRET_ERR_CUDA;
    }
    return GRET_OK;
}

size_t gret_prefill_state_workspace_size(int B, int H, int N, int dk, int dv, int chunk, gret_dtype io_dtype) {
    chunk = run_chunk(dk, dv, chunk, io_dtype, false);
    int sms = 148;
    device_info(nullptr, &sms);
    if (select_path(B, H, N, dk, dv, chunk, io_dtype, sms, nullptr, nullptr) != GRET_PATH_TC) return 0;
    return prefill_tc_state_workspace_bytes(B, H, N, dk, dv, chunk, sms);
}

gret_status gret_prefill_state(const void* K, const void* V, const float* gate_logits, float tau, int chunk,
                               float* dS, float* decay, int B, int H, int N, int dk, int dv, gret_dtype io_dtype,
                               void* workspace, size_t workspace_bytes, gret_stream_t stream) {
    if (!K || !V || !gate_logits || !dS || !decay) return GRET_ERR_INVALID_ARG;
    if (io_dtype != GRET_F32 && io_dtype != GRET_BF16) return GRET_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || dk <= 0 || dv <= 0 || chunk <= 0) return GRET_ERR_INVALID_ARG;
    if (!(tau > 0.0f) || !isfinite(tau)) return GRET_ERR_INVALID_ARG;
    if (!aligned16(K) || !aligned16(V) || !aligned16(gate_logits) || !aligned16(dS) ||
        (reinterpret_cast<uintptr_t>(decay) & 3u) != 0)
        return GRET_ERR_INVALID_ARG;
    if ((long long)B * H > (1LL << 30) || (long long)B * N > (1LL << 40)) return GRET_ERR_UNSUPPORTED;
    chunk = run_chunk(dk, dv, chunk, io_dtype, false);
    unsigned int* status = nullptr;
    int sms = 0;
    if (!device_info(&status, &sms)) return GRET_ERR_CUDA;
    gret_path path = select_path(B, H, N, dk, dv, chunk, io_dtype, sms, nullptr, nullptr);
    if (path == GRET_PATH_NONE) return GRET_ERR_UNSUPPORTED;
    PrefillArgs a = {};
    memset(&a, 0, sizeof(a));
    a.Q = K; a.K = K; a.V = V; a.z = gate_logits; a.S_final = dS; a.decay_out = decay; a.state_only = 1;
    a.B = B; a.H = H; a.N = N; a.dk = dk; a.dv = dv; a.chunk = chunk;
    a.inv_tau = 1.0f / tau; a.eps = 0.f; a.io = io_dtype; a.epi = GRET_EPI_NONE;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes; a.status = status;
    a.segments = 1; a.seg_len = N; a.pieces = 1;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (path == GRET_PATH_TC) {
        const size_t need = prefill_tc_state_workspace_bytes(B, H, N, dk, dv, chunk, sms);
        if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return GRET_ERR_INVALID_ARG;
        err = launch_prefill_state_tc(a, sms, s);
    } else {
        err = launch_prefill_simt(a, s);
    }
    return err == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

gret_status gret_state_fold(const float* dS_all, const float* decay_all, int num_slices, int slice,
                            const float* S0, float* S_in, int B, int H, int dk, int dv, gret_stream_t stream) {
    if (!S_in || (slice > 0 && (!dS_all || !decay_all))) return GRET_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0 || num_slices <= 0 || slice < 0 || slice > num_slices)
        return GRET_ERR_INVALID_ARG;
    if ((long long)B * H * dk * dv > (1LL << 40)) return GRET_ERR_UNSUPPORTED;
    const cudaError_t err = launch_state_fold(dS_all, decay_all, num_slices, slice, S0, S_in, B * H, dk * dv,
                                              reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

size_t gret_prefill_backward_workspace_size(int B, int H, int N, int dk, int dv, gret_dtype io_dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || !shape_supported(dk, dv) || !prefill_backward_supported(dk, dv)) return 0;
    if (io_dtype != GRET_F32 && io_dtype != GRET_BF16) return 0;
    return prefill_backward_workspace_bytes(B, H, N, dk, dv, io_dtype);
}

int gret_prefill_backward_launches(int B, int H, int N, int dk, int dv, gret_dtype io_dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || !shape_supported(dk, dv) || !prefill_backward_supported(dk, dv)) return 0;
    if (io_dtype != GRET_F32 && io_dtype != GRET_BF16) return 0;
    return prefill_backward_launches(B, H, N, dk, dv, io_dtype);
}

gret_status gret_prefill_backward(const void* Q, const void* K, const void* V, const float* gate_logits,
                                  const void* G, const float* S0, const void* dO, const float* dS_final, float tau,
                                  float eps, gret_epilogue epi, void* dQ, void* dK, void* dV, float* dz, void* dG,
                                  float* dS0, int B, int H, int N, int dk, int dv, gret_dtype io_dtype,
                                  void* workspace, size_t workspace_bytes, gret_stream_t stream) {
    if (!Q || !K || !V || !gate_logits || !dO || !dQ || !dK || !dV || !dz) return GRET_ERR_INVALID_ARG;
    if (epi != GRET_EPI_GN_SWISH && epi != GRET_EPI_NONE) return GRET_ERR_INVALID_ARG;
    if (epi == GRET_EPI_GN_SWISH && (!G || !dG)) return GRET_ERR_INVALID_ARG;
    if (io_dtype != GRET_F32 && io_dtype != GRET_BF16) return GRET_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || dk <= 0 || dv <= 0) return GRET_ERR_INVALID_ARG;
    if (!(tau > 0.0f) || !isfinite(tau) || !(eps >= 0.0f) || !isfinite(eps)) return GRET_ERR_INVALID_ARG;
    const void* ptrs[] = {Q, K, V, gate_logits, dO, dQ, dK, dV, dz, G, dG, S0, dS_final, dS0};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return GRET_ERR_INVALID_ARG;
    if ((long long)B * H > (1LL << 30) || (long long)B * N > (1LL << 40)) return GRET_ERR_UNSUPPORTED;
    if (!shape_supported(dk, dv) || !prefill_backward_supported(dk, dv)) return GRET_ERR_UNSUPPORTED;
    const size_t need = prefill_backward_workspace_bytes(B, H, N, dk, dv, io_dtype);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return GRET_ERR_INVALID_ARG;
    BackwardArgs a = {};
    a.Q = Q; a.K = K; a.V = V; a.G = G; a.dO = dO; a.z = gate_logits; a.S0 = S0; a.dS_final = dS_final;
    a.dQ = dQ; a.dK = dK; a.dV = dV; a.dG = dG; a.dz = dz; a.dS0 = dS0; a.workspace = workspace;
    a.B = B; a.H = H; a.N = N; a.dk = dk; a.dv = dv; a.inv_tau = 1.0f / tau; a.eps = eps;
    a.gn = epi == GRET_EPI_GN_SWISH ? 1 : 0; a.io = io_dtype;
    if (!device_info(&a.status, nullptr)) return GRET_ERR_CUDA;
    return launch_prefill_backward(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? GRET_OK
                                                                                        : GRET_ERR_CUDA;
}

}  // extern "C"
