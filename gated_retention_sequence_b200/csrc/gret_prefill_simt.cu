// Chunkwise prefill on CUDA cores, fp32 arithmetic throughout.
//
// "YOCO 深度技术分析", section 5.3.2 (chunkwise form: parallel inside a block,
// recurrent between blocks) and section 2.2 (gate, forms, GroupNorm + swish);
// the chunk state and its decay summary are the "R_i" and "beta" of the
// "分段递归表示" paragraph of the Medium-article translation.  With t, s local
// indices of one chunk and b_t the chunk-local cumulative log-decay:
//   Y_t    = sum_{s<=t} (Q_t . K_s) e^{b_t - b_s} V_s + e^{b_t} Q_t S
//   S     <- e^{b_L} S + sum_s e^{b_L - b_s} K_s^T V_s
// All exponents are <= 0, so nothing overflows whatever the gate values.
//
// This kernel serves the fp32 I/O path (where tensor-core operands would cost
// the 1e-4 tolerance) and any shape the tensor-core kernel does not take.
// One CTA runs one (batch, head) unit; the state S [dk][dv] stays in shared
// memory for the whole sequence.
#include "gret_common.cuh"

namespace gret {
namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads) prefill_simt_kernel(PrefillArgs a) {
    extern __shared__ float smem[];
    const int dk = a.dk, dv = a.dv, C = a.chunk, N = a.N, H = a.H;
    const int u = blockIdx.x, b = u / H, h = u % H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kThreads / 32;

    float* S = smem;                      // [dk][dv]
    float* Qs = S + (size_t)dk * dv;      // [C][dk]
    float* Ks = Qs + (size_t)C * dk;      // [C][dk]
    float* Vs = Ks + (size_t)C * dk;      // [C][dv]
    float* Ys = Vs + (size_t)C * dv;      // [C][dv]
    float* As = Ys + (size_t)C * dv;      // [C][C]
    float* bc = As + (size_t)C * C;       // [C] cumulative log-decay
    float* wl = bc + C;                   // [C] e^{b_L - b_s}

    const float* S0 = a.S0 ? a.S0 + (size_t)u * dk * dv : nullptr;
    for (int e = tid; e < dk * dv; e += kThreads) S[e] = S0 ? S0[e] : 0.f;

    const T* Qg = static_cast<const T*>(a.Q);
    const T* Kg = static_cast<const T*>(a.K);
    const T* Vg = static_cast<const T*>(a.V);
    const T* Gg = static_cast<const T*>(a.G);
    T* Og = static_cast<T*>(a.O);
    const size_t rowk = (size_t)H * dk, rowv = (size_t)H * dv;

    // this unit's tokens: rows base .. base + Nu - 1
    int row0 = 0, Nu = N;
    if (a.cu_seqlens) packed_range(a.cu_seqlens, b, a.total, row0, Nu);
    const size_t base = a.cu_seqlens ? (size_t)row0 : (size_t)b * N;
    float decay = 0.f;      // the unit's total log-decay (state-only pass)
    for (int c0 = 0; c0 < Nu; c0 += C) {
        const int L = min(C, Nu - c0);
        const size_t tok0 = base + c0;
        for (int e = tid; e < L * dk; e += kThreads) {
            int t = e / dk, i = e % dk;
            if (!a.state_only) Qs[e] = to_f32(Qg[(tok0 + t) * rowk + (size_t)h * dk + i]);
            Ks[e] = to_f32(Kg[(tok0 + t) * rowk + (size_t)h * dk + i]);
        }
        for (int e = tid; e < L * dv; e += kThreads) {
            int t = e / dv, j = e % dv;
            Vs[e] = to_f32(Vg[(tok0 + t) * rowv + (size_t)h * dv + j]);
        }
        if (warp == 0) {
            // inclusive scan of log gamma over the chunk, 32 tokens at a time
            float carry = 0.f;
            for (int t0 = 0; t0 < L; t0 += 32) {
                int t = t0 + lane;
                float x = (t < L) ? log_gamma(a.z[(tok0 + t) * H + h], a.inv_tau) : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                x += carry;
                if (t < L) bc[t] = x;
                carry = __shfl_sync(0xffffffffu, x, 31);
            }
        }
        __syncthreads();
        const float bL = bc[L - 1];
        decay += bL;
        for (int s = tid; s < L; s += kThreads) wl[s] = expf(bL - bc[s]);
        if (a.state_only) {
            // state increment only: S <- e^{b_L} S + sum_s e^{b_L - b_s} K_s^T V_s
            __syncthreads();
            const float eL = expf(bL);
            for (int e = tid; e < dk * dv; e += kThreads) {
                int i = e / dv, j = e % dv;
                float acc = 0.f;
                for (int s = 0; s < L; ++s) acc = fmaf(wl[s] * Ks[s * dk + i], Vs[s * dv + j], acc);
                S[e] = fmaf(eL, S[e], acc);
            }
            __syncthreads();
            continue;
        }
        // intra-chunk scores with the decay mask
        for (int e = tid; e < L * L; e += kThreads) {
            int t = e / L, s = e % L;
            float acc = 0.f;
            if (s <= t) {
                for (int i = 0; i < dk; ++i) acc = fmaf(Qs[t * dk + i], Ks[s * dk + i], acc);
                acc *= expf(bc[t] - bc[s]);
            }
            As[t * C + s] = acc;
        }
        __syncthreads();
        // outputs: intra (P V) + inter (e^{b_t} Q_t S)
        for (int e = tid; e < L * dv; e += kThreads) {
            int t = e / dv, j = e % dv;
            float intra = 0.f, inter = 0.f;
            for (int s = 0; s <= t; ++s) intra = fmaf(As[t * C + s], Vs[s * dv + j], intra);
            for (int i = 0; i < dk; ++i) inter = fmaf(Qs[t * dk + i], S[i * dv + j], inter);
            Ys[e] = intra + expf(bc[t]) * inter;
        }
        __syncthreads();
        // state carry
        const float eL = expf(bL);
        for (int e = tid; e < dk * dv; e += kThreads) {
            int i = e / dv, j = e % dv;
            float acc = 0.f;
            for (int s = 0; s < L; ++s) acc = fmaf(wl[s] * Ks[s * dk + i], Vs[s * dv + j], acc);
            S[e] = fmaf(eL, S[e], acc);
        }
        // epilogue: one warp per token
        for (int t = warp; t < L; t += kWarps) {
            const float* y = Ys + t * dv;
            T* o = Og + (tok0 + t) * rowv + (size_t)h * dv;
            if (a.epi == GRET_EPI_NONE) {
                for (int j = lane; j < dv; j += 32) o[j] = from_f32<T>(y[j]);
                continue;
            }
            float sum = 0.f;
            for (int j = lane; j < dv; j += 32) sum += y[j];
            const float mean = warp_sum(sum) / (float)dv;
            float sq = 0.f;
            for (int j = lane; j < dv; j += 32) {
                float d = y[j] - mean;
                sq += d * d;
            }
            const float rstd = rsqrtf(warp_sum(sq) / (float)dv + a.eps);
            const T* g = Gg + (tok0 + t) * rowv + (size_t)h * dv;
            for (int j = lane; j < dv; j += 32) {
                float gj = to_f32(g[j]);
                o[j] = from_f32<T>((y[j] - mean) * rstd * gj * sigmoidf_(gj));
            }
        }
        __syncthreads();
    }
    if (a.S_final) {
        float* Sf = a.S_final + (size_t)u * dk * dv;
        for (int e = tid; e < dk * dv; e += kThreads) Sf[e] = S[e];
    }
    if (a.state_only && a.decay_out && tid == 0) a.decay_out[u] = decay;
}

}  // namespace

size_t prefill_simt_smem_bytes(int dk, int dv, int chunk) {
    size_t C = chunk;
    return sizeof(float) * ((size_t)dk * dv + C * (2 * dk + 2 * dv + C) + 2 * C);
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s) {
    size_t smem = prefill_simt_smem_bytes(a.dk, a.dv, a.chunk);
    int units = a.B * a.H;
    if (g_profile_start) cudaEventRecord(g_profile_start, s);
    if (a.io == GRET_BF16) {
        auto k = prefill_simt_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<units, kThreads, smem, s>>>(a);
    } else {
        auto k = prefill_simt_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<units, kThreads, smem, s>>>(a);
    }
    if (g_profile_stop) cudaEventRecord(g_profile_stop, s);
    return cudaGetLastError();
}

}  // namespace gret
