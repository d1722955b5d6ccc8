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
// memory for the whole sequence.  A chunk is worked through in blocks of SB
// rows (tokens t) and SB columns (tokens s), SB = C whenever the whole chunk
// fits in shared memory: for a row block, the inter-chunk term against the
// state at the chunk's start, then the intra-chunk term block by block over
// the columns s <= t, then the epilogue; the state update follows once every
// row block of the chunk is done.  The decay sums b run over the whole chunk
// either way, so the blocks only reorder the sums of the chunk's formula.
#include "gret_common.cuh"

namespace gret {
namespace {

constexpr int kThreads = 256;
constexpr size_t kSmemLimit = 227 * 1024;

// Shared memory of a CTA that works through chunks of C tokens in blocks of SB.
size_t simt_smem(int dk, int dv, int C, int SB) {
    const size_t sb = SB;
    return sizeof(float) * ((size_t)dk * dv + sb * (2 * dk + 2 * dv + sb) + (size_t)C + sb);
}

// Largest block (the whole chunk if it fits, else 64, 32 or 16 tokens).
int simt_block(int dk, int dv, int C) {
    const int cand[4] = {C, 64, 32, 16};
    for (int SB : cand)
        if (SB <= C && simt_smem(dk, dv, C, SB) <= kSmemLimit) return SB;
    return 0;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) prefill_simt_kernel(PrefillArgs a, int SB) {
    extern __shared__ float smem[];
    const int dk = a.dk, dv = a.dv, C = a.chunk, N = a.N, H = a.H;
    const int u = blockIdx.x, b = u / H, h = u % H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kThreads / 32;

    float* S = smem;                      // [dk][dv]
    float* Qs = S + (size_t)dk * dv;      // [SB][dk]  rows of the current row block
    float* Ks = Qs + (size_t)SB * dk;     // [SB][dk]  rows of the current column block
    float* Vs = Ks + (size_t)SB * dk;     // [SB][dv]
    float* Ys = Vs + (size_t)SB * dv;     // [SB][dv]
    float* As = Ys + (size_t)SB * dv;     // [SB][SB]
    float* bc = As + (size_t)SB * SB;     // [C] cumulative log-decay over the chunk
    float* wl = bc + C;                   // [SB] e^{b_L - b_s}

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

    // K and V rows j0 .. j0 + Lj - 1 of the chunk starting at token tok0
    auto load_kv = [&](size_t tok0, int j0, int Lj) {
        for (int e = tid; e < Lj * dk; e += kThreads) {
            const int t = e / dk, i = e % dk;
            Ks[e] = to_f32(Kg[(tok0 + j0 + t) * rowk + (size_t)h * dk + i]);
        }
        for (int e = tid; e < Lj * dv; e += kThreads) {
            const int t = e / dv, j = e % dv;
            Vs[e] = to_f32(Vg[(tok0 + j0 + t) * rowv + (size_t)h * dv + j]);
        }
    };

    float decay = 0.f;      // the unit's total log-decay (state-only pass)
    for (int c0 = 0; c0 < Nu; c0 += C) {
        const int L = min(C, Nu - c0);
        const size_t tok0 = base + c0;
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
        int kv_block = -1;      // first row of the column block held in Ks / Vs
        if (!a.state_only) {
            for (int i0 = 0; i0 < L; i0 += SB) {
                const int Li = min(SB, L - i0);
                for (int e = tid; e < Li * dk; e += kThreads) {
                    const int t = e / dk, i = e % dk;
                    Qs[e] = to_f32(Qg[(tok0 + i0 + t) * rowk + (size_t)h * dk + i]);
                }
                __syncthreads();
                // inter-chunk term e^{b_t} Q_t S (S still holds the chunk's initial state)
                for (int e = tid; e < Li * dv; e += kThreads) {
                    const int t = e / dv, j = e % dv;
                    float inter = 0.f;
                    for (int i = 0; i < dk; ++i) inter = fmaf(Qs[t * dk + i], S[i * dv + j], inter);
                    Ys[e] = expf(bc[i0 + t]) * inter;
                }
                // intra-chunk term over the column blocks s <= t
                for (int j0 = 0; j0 <= i0; j0 += SB) {
                    const int Lj = min(SB, L - j0);
                    __syncthreads();
                    if (kv_block != j0) load_kv(tok0, j0, Lj);
                    kv_block = j0;
                    __syncthreads();
                    // scores with the decay mask
                    for (int e = tid; e < Li * Lj; e += kThreads) {
                        const int t = e / Lj, s = e % Lj;
                        float acc = 0.f;
                        if (j0 + s <= i0 + t) {
                            for (int i = 0; i < dk; ++i) acc = fmaf(Qs[t * dk + i], Ks[s * dk + i], acc);
                            acc *= expf(bc[i0 + t] - bc[j0 + s]);
                        }
                        As[t * SB + s] = acc;
                    }
                    __syncthreads();
                    for (int e = tid; e < Li * dv; e += kThreads) {
                        const int t = e / dv, j = e % dv;
                        float intra = 0.f;
                        for (int s = 0; s < Lj; ++s) intra = fmaf(As[t * SB + s], Vs[s * dv + j], intra);
                        Ys[e] += intra;
                    }
                }
                __syncthreads();
                // epilogue: one warp per token
                for (int t = warp; t < Li; t += kWarps) {
                    const float* y = Ys + t * dv;
                    T* o = Og + (tok0 + i0 + t) * rowv + (size_t)h * dv;
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
                    const T* g = Gg + (tok0 + i0 + t) * rowv + (size_t)h * dv;
                    for (int j = lane; j < dv; j += 32) {
                        float gj = to_f32(g[j]);
                        o[j] = from_f32<T>((y[j] - mean) * rstd * gj * sigmoidf_(gj));
                    }
                }
            }
        }
        // state carry S <- e^{b_L} S + sum_s e^{b_L - b_s} K_s^T V_s, column blocks
        // from the last one (which may still be in Ks / Vs) down to the first
        const float eL = expf(bL);
        const int last0 = ((L - 1) / SB) * SB;
        for (int j0 = last0; j0 >= 0; j0 -= SB) {
            const int Lj = min(SB, L - j0);
            __syncthreads();
            if (kv_block != j0) load_kv(tok0, j0, Lj);
            kv_block = j0;
            for (int s = tid; s < Lj; s += kThreads) wl[s] = expf(bL - bc[j0 + s]);
            __syncthreads();
            const bool first = j0 == last0;
            for (int e = tid; e < dk * dv; e += kThreads) {
                const int i = e / dv, j = e % dv;
                float acc = 0.f;
                for (int s = 0; s < Lj; ++s) acc = fmaf(wl[s] * Ks[s * dk + i], Vs[s * dv + j], acc);
                S[e] = first ? fmaf(eL, S[e], acc) : S[e] + acc;
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
    const int SB = simt_block(dk, dv, chunk);
    return SB > 0 ? simt_smem(dk, dv, chunk, SB) : simt_smem(dk, dv, chunk, 16);
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s) {
    const int SB = simt_block(a.dk, a.dv, a.chunk);
    if (SB <= 0) return cudaErrorInvalidConfiguration;
    size_t smem = simt_smem(a.dk, a.dv, a.chunk, SB);
    int units = a.B * a.H;
    if (g_profile_start) cudaEventRecord(g_profile_start, s);
    if (a.io == GRET_BF16) {
        auto k = prefill_simt_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<units, kThreads, smem, s>>>(a, SB);
    } else {
        auto k = prefill_simt_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<units, kThreads, smem, s>>>(a, SB);
    }
    if (g_profile_stop) cudaEventRecord(g_profile_stop, s);
    return cudaGetLastError();
}

}  // namespace gret
