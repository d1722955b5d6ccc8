// gret_prefill_noalloc: the prefill for callers that cannot allocate device
// memory themselves.  Its scratch is a fixed array compiled into this file;
// the call passes that array's device address to gret_prefill.
#include <mutex>

#include "gret_common.cuh"

namespace {

constexpr size_t kScratchBytes = GRET_NOALLOC_SCRATCH_BYTES;

// Device memory every GPU that loads the library reserves for as long as the
// process runs.  In host code this name is only a stand-in for the device
// array; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up the
// first time the current device asks for it.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gret_status gret_prefill_noalloc(const void* Q, const void* K, const void* V,
                                            const float* gate_logits, const void* G, float tau,
                                            int chunk, void* O, float* S_final, int B, int H, int N,
                                            int dk, int dv, gret_dtype io_dtype, float eps,
                                            gret_epilogue epi, gret_stream_t stream) {
    // Invalid or unsupported arguments report 0 here and are rejected by gret_prefill.
    const size_t need = gret_prefill_workspace_size(B, H, N, dk, dv, chunk, io_dtype);
    if (need > kScratchBytes) return GRET_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (need > 0 && scratch_address(&ws) != cudaSuccess) return GRET_ERR_CUDA;
    return gret_prefill(Q, K, V, gate_logits, G, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype,
                        eps, epi, ws, need, stream);
}
