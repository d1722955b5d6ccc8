// Backward of the gated-retention prefill: the host entry points (workspace
// size, launch count, dispatch) and the serial CUDA-core path, fp32 arithmetic,
// for head sizes the chunk-parallel kernels (gret_backward_chunk.cu) do not
// take.
//
// The forward is the chunkwise form of "YOCO 深度技术分析", sections 2.2 and
// 5.3.2; this file computes its exact derivative.  Per (batch, head) unit, a
// block of L tokens starting from state S (b_t the block-local cumulative log
// decay, b_L its total):
//   A_ts = (q_t . k_s) e^{b_t - b_s}  (s <= t)
//   y_t  = sum_s A_ts v_s + e^{b_t} q_t S
//   S'   = e^{b_L} S + sum_s e^{b_L - b_s} k_s^T v_s
// Given dy (from the GroupNorm * swish backward of dO) and dS' (the gradient
// reaching the block's end state), with D_ts = dy_t . v_s (s <= t):
//   dq_t = sum_s e^{b_t - b_s} D_ts k_s + e^{b_t} S dy_t
//   dk_s = sum_t e^{b_t - b_s} D_ts q_t + e^{b_L - b_s} dS' v_s
//   dv_s = sum_t A_ts dy_t           + e^{b_L - b_s} dS'^T k_s
//   dS   = e^{b_L} dS' + sum_t e^{b_t} q_t^T dy_t
// and for the log-decay of token j of the block (b_t - b_s depends on it when
// s < j <= t, b_t when j <= t, b_L always, b_L - b_s when s < j):
//   dlg_j = sum_{t>=j, s<j} A_ts D_ts + sum_{t>=j} e^{b_t} dy_t.(q_t S)
//         + e^{b_L} <dS', S> + sum_{s<j} e^{b_L - b_s} k_s.(dS' v_s)
//   dz_j  = dlg_j (1 - sigmoid(z_j)) / tau   (0 where the forward clamps log gamma)
//
// Blocks of kBlk tokens: the chunk length is a free parameter of the chunkwise
// form (the result does not depend on it), and 32 keeps every per-block tile of
// up to 256 x 256 heads in shared memory.  A first kernel stores the state at
// the start of every block (the checkpoints); the second walks the blocks in
// reverse with dS in global memory (one unit's worth stays in L2).
#include "gret_common.cuh"

namespace gret {
namespace {

constexpr int kBThreads = 256;
constexpr int kBlk = 32;

struct BwdArgs {
    const void *Q, *K, *V, *G, *dO;
    const float *z, *S0, *dS_final;
    void *dQ, *dK, *dV, *dG;
    float *dz, *dS0;
    float* ckpt;    // [units][nblk][dk][dv]
    float* dSw;     // [units][dk][dv]
    int B, H, N, dk, dv, nblk;
    float inv_tau, eps;
    int gn;
};

// Block-local inclusive sums of log gamma for L tokens (warp 0), plus the log
// gamma values themselves.
template <typename Tz>
__device__ __forceinline__ void block_decay(const Tz* z, size_t stride, int L, float inv_tau, float* lg, float* bc) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        float x = lane < L ? log_gamma(z[(size_t)lane * stride], inv_tau) : 0.f;
        if (lane < L) lg[lane] = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane < L) bc[lane] = x;
    }
}

// ---- checkpoints: ckpt[u][c] = state before block c
template <typename T>
__global__ void __launch_bounds__(kBThreads) bwd_checkpoint_kernel(BwdArgs a) {
    extern __shared__ float sm[];
    const int dk = a.dk, dv = a.dv, H = a.H, N = a.N;
    const int u = blockIdx.x, b = u / H, h = u % H, tid = threadIdx.x;
    float* Ks = sm;                       // [kBlk][dk]
    float* Vs = Ks + kBlk * dk;           // [kBlk][dv]
    float* lg = Vs + kBlk * dv;           // [kBlk]
    float* bc = lg + kBlk;                // [kBlk]
    float* wl = bc + kBlk;                // [kBlk] e^{b_L - b_s}
    const T* Kg = static_cast<const T*>(a.K);
    const T* Vg = static_cast<const T*>(a.V);
    const size_t E = (size_t)dk * dv;
    float* ck = a.ckpt + (size_t)u * a.nblk * E;
    for (size_t e = tid; e < E; e += kBThreads) ck[e] = a.S0 ? a.S0[(size_t)u * E + e] : 0.f;
    for (int c = 0; c + 1 < a.nblk; ++c) {
        const int n0 = c * kBlk, L = min(kBlk, N - n0);
        const size_t tok0 = (size_t)b * N + n0;
        for (int e = tid; e < L * dk; e += kBThreads)
            Ks[e] = to_f32(Kg[(tok0 + e / dk) * H * dk + (size_t)h * dk + e % dk]);
        for (int e = tid; e < L * dv; e += kBThreads)
            Vs[e] = to_f32(Vg[(tok0 + e / dv) * H * dv + (size_t)h * dv + e % dv]);
        block_decay(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc);
        __syncthreads();
        const float bL = bc[L - 1];
        for (int s = tid; s < L; s += kBThreads) wl[s] = expf(bL - bc[s]);
        __syncthreads();
        const float eL = expf(bL);
        const float* cur = ck + (size_t)c * E;
        float* nxt = ck + (size_t)(c + 1) * E;
        for (size_t e = tid; e < E; e += kBThreads) {
            const int i = (int)(e / dv), j = (int)(e % dv);
            float acc = 0.f;
            for (int s = 0; s < L; ++s) acc = fmaf(wl[s] * Ks[s * dk + i], Vs[s * dv + j], acc);
            nxt[e] = fmaf(eL, cur[e], acc);
        }
        __syncthreads();
    }
}

// ---- the reverse walk over blocks
template <typename T>
__global__ void __launch_bounds__(kBThreads) bwd_block_kernel(BwdArgs a) {
    extern __shared__ float sm[];
    const int dk = a.dk, dv = a.dv, H = a.H, N = a.N;
    const int u = blockIdx.x, b = u / H, h = u % H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kBThreads / 32;
    constexpr int B2 = kBlk * kBlk;
    float* Qs = sm;                      // [kBlk][dk]
    float* Ks = Qs + kBlk * dk;          // [kBlk][dk]
    float* Vs = Ks + kBlk * dk;          // [kBlk][dv]
    float* Ys = Vs + kBlk * dv;          // [kBlk][dv]  pre-norm output
    float* dYs = Ys + kBlk * dv;         // [kBlk][dv]  dO, then dy
    float* As = dYs + kBlk * dv;         // [kBlk][kBlk] A_ts (decayed, masked)
    float* Ds = As + B2;                 // [kBlk][kBlk] D_ts = dy_t . v_s (masked)
    float* Ex = Ds + B2;                 // [kBlk][kBlk] e^{b_t - b_s} (masked)
    float* Us = Ex + B2;                 // [kBlk][dk]  S dy_t
    float* Ws = Us + kBlk * dk;          // [kBlk][dk]  dS' v_s
    float* lg = Ws + kBlk * dk;          // [kBlk]
    float* bc = lg + kBlk;               // [kBlk]
    float* eb = bc + kBlk;               // [kBlk] e^{b_t}
    float* rr = eb + kBlk;               // [kBlk]
    float* ust = rr + kBlk;              // [kBlk]
    float* red = ust + kBlk;             // [kWarps]
    const T* Qg = static_cast<const T*>(a.Q);
    const T* Kg = static_cast<const T*>(a.K);
    const T* Vg = static_cast<const T*>(a.V);
    const T* Gg = static_cast<const T*>(a.G);
    const T* dOg = static_cast<const T*>(a.dO);
    T* dQg = static_cast<T*>(a.dQ);
    T* dKg = static_cast<T*>(a.dK);
    T* dVg = static_cast<T*>(a.dV);
    T* dGg = static_cast<T*>(a.dG);
    const size_t E = (size_t)dk * dv;
    const float* ck = a.ckpt + (size_t)u * a.nblk * E;
    float* dS = a.dSw + (size_t)u * E;
    for (size_t e = tid; e < E; e += kBThreads) dS[e] = a.dS_final ? a.dS_final[(size_t)u * E + e] : 0.f;
    __syncthreads();

    for (int c = a.nblk - 1; c >= 0; --c) {
        const int n0 = c * kBlk, L = min(kBlk, N - n0);
        const size_t tok0 = (size_t)b * N + n0;
        const float* Ss = ck + (size_t)c * E;    // state before the block
        // tiles, decay sums
        for (int e = tid; e < L * dk; e += kBThreads) {
            const size_t off = (tok0 + e / dk) * H * dk + (size_t)h * dk + e % dk;
            Qs[e] = to_f32(Qg[off]);
            Ks[e] = to_f32(Kg[off]);
        }
        for (int e = tid; e < L * dv; e += kBThreads) {
            const size_t off = (tok0 + e / dv) * H * dv + (size_t)h * dv + e % dv;
            Vs[e] = to_f32(Vg[off]);
            dYs[e] = to_f32(dOg[off]);
        }
        block_decay(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc);
        __syncthreads();
        const float bL = bc[L - 1];
        for (int t = tid; t < kBlk; t += kBThreads) eb[t] = t < L ? expf(bc[t]) : 0.f;
        // A and the decay matrix (rows and columns past L are zero)
        for (int e = tid; e < B2; e += kBThreads) {
            const int t = e / kBlk, s = e % kBlk;
            float ex = 0.f, av = 0.f;
            if (t < L && s <= t) {
                ex = expf(bc[t] - bc[s]);
                float dot = 0.f;
                for (int i = 0; i < dk; ++i) dot = fmaf(Qs[t * dk + i], Ks[s * dk + i], dot);
                av = dot * ex;
            }
            Ex[e] = ex;
            As[e] = av;
        }
        __syncthreads();
        // y = A V + e^{b_t} q_t S, one output column per thread
        for (int j = tid; j < dv; j += kBThreads) {
            float acc[kBlk];
#pragma unroll
            for (int t = 0; t < kBlk; ++t) acc[t] = 0.f;
            for (int i = 0; i < dk; ++i) {
                const float sv = Ss[(size_t)i * dv + j];
#pragma unroll
                for (int t = 0; t < kBlk; ++t) acc[t] = fmaf(t < L ? Qs[t * dk + i] : 0.f, sv, acc[t]);
            }
#pragma unroll
            for (int t = 0; t < kBlk; ++t) {
                if (t < L) {
                    float intra = 0.f;
                    for (int s = 0; s <= t; ++s) intra = fmaf(As[t * kBlk + s], Vs[s * dv + j], intra);
                    Ys[t * dv + j] = fmaf(eb[t], acc[t], intra);
                }
            }
        }
        __syncthreads();
        // GroupNorm * swish backward, one warp per token: dG, and dy over dO
        if (a.gn) {
            for (int t = warp; t < L; t += kWarps) {
                const float* y = Ys + t * dv;
                float* dy = dYs + t * dv;
                const size_t go = (tok0 + t) * H * dv + (size_t)h * dv;
                float s1 = 0.f;
                for (int j = lane; j < dv; j += 32) s1 += y[j];
                const float mean = warp_sum(s1) / (float)dv;
                float s2 = 0.f;
                for (int j = lane; j < dv; j += 32) {
                    const float d = y[j] - mean;
                    s2 += d * d;
                }
                const float rstd = rsqrtf(warp_sum(s2) / (float)dv + a.eps);
                float m1 = 0.f, m2 = 0.f;
                for (int j = lane; j < dv; j += 32) {
                    const float g = to_f32(Gg[go + j]);
                    const float sg = sigmoidf_(g);
                    const float n = (y[j] - mean) * rstd;
                    const float gout = dy[j];
                    // d/dg [g sigmoid(g)] = sigmoid(g) (1 + g (1 - sigmoid(g)))
                    dGg[go + j] = from_f32<T>(gout * n * sg * (1.f + g * (1.f - sg)));
                    const float dn = gout * g * sg;
                    dy[j] = dn;
                    m1 += dn;
                    m2 += dn * n;
                }
                m1 = warp_sum(m1) / (float)dv;
                m2 = warp_sum(m2) / (float)dv;
                for (int j = lane; j < dv; j += 32) dy[j] = rstd * (dy[j] - m1 - (y[j] - mean) * rstd * m2);
            }
        }
        __syncthreads();
        // D, U = S dy_t (per t), W = dS' v_s (per s)
        for (int e = tid; e < B2; e += kBThreads) {
            const int t = e / kBlk, s = e % kBlk;
            float dval = 0.f;
            if (t < L && s <= t)
                for (int j = 0; j < dv; ++j) dval = fmaf(dYs[t * dv + j], Vs[s * dv + j], dval);
            Ds[e] = dval;
        }
        for (int i = tid; i < dk; i += kBThreads) {
            float au[kBlk], aw[kBlk];
#pragma unroll
            for (int t = 0; t < kBlk; ++t) au[t] = aw[t] = 0.f;
            for (int j = 0; j < dv; ++j) {
                const float sv = Ss[(size_t)i * dv + j], dsv = dS[(size_t)i * dv + j];
#pragma unroll
                for (int t = 0; t < kBlk; ++t) {
                    au[t] = fmaf(t < L ? dYs[t * dv + j] : 0.f, sv, au[t]);
                    aw[t] = fmaf(t < L ? Vs[t * dv + j] : 0.f, dsv, aw[t]);
                }
            }
#pragma unroll
            for (int t = 0; t < kBlk; ++t) {
                Us[t * dk + i] = au[t];
                Ws[t * dk + i] = aw[t];
            }
        }
        __syncthreads();
        // dq, dk
        for (int e = tid; e < L * dk; e += kBThreads) {
            const int t = e / dk, i = e % dk;
            float dq = 0.f, dkk = 0.f;
            for (int s = 0; s <= t; ++s) dq = fmaf(Ex[t * kBlk + s] * Ds[t * kBlk + s], Ks[s * dk + i], dq);
            dq = fmaf(eb[t], Us[t * dk + i], dq);
            const int s = t;   // the same thread also forms dk of token s = t
            for (int tt = s; tt < L; ++tt) dkk = fmaf(Ex[tt * kBlk + s] * Ds[tt * kBlk + s], Qs[tt * dk + i], dkk);
            dkk = fmaf(expf(bL - bc[s]), Ws[s * dk + i], dkk);
            const size_t off = (tok0 + t) * H * dk + (size_t)h * dk + i;
            dQg[off] = from_f32<T>(dq);
            dKg[off] = from_f32<T>(dkk);
        }
        // dv, one column per thread: sum_{t>=s} A_ts dy_t + e^{b_L - b_s} dS'^T k_s
        for (int j = tid; j < dv; j += kBThreads) {
            float acc[kBlk];
#pragma unroll
            for (int s = 0; s < kBlk; ++s) acc[s] = 0.f;
            for (int i = 0; i < dk; ++i) {
                const float dsv = dS[(size_t)i * dv + j];
#pragma unroll
                for (int s = 0; s < kBlk; ++s) acc[s] = fmaf(s < L ? Ks[s * dk + i] : 0.f, dsv, acc[s]);
            }
#pragma unroll
            for (int s = 0; s < kBlk; ++s) {
                if (s < L) {
                    float v = 0.f;
                    for (int t = s; t < L; ++t) v = fmaf(As[t * kBlk + s], dYs[t * dv + j], v);
                    dVg[(tok0 + s) * H * dv + (size_t)h * dv + j] = from_f32<T>(fmaf(expf(bL - bc[s]), acc[s], v));
                }
            }
        }
        // gate: r_t = e^{b_t} dy_t.(q_t S), ust_s = e^{b_L - b_s} k_s.(dS' v_s), c0 = e^{b_L} <dS', S>
        for (int t = warp; t < L; t += kWarps) {
            float x = 0.f, w = 0.f;
            for (int i = lane; i < dk; i += 32) {
                x = fmaf(Qs[t * dk + i], Us[t * dk + i], x);
                w = fmaf(Ks[t * dk + i], Ws[t * dk + i], w);
            }
            x = warp_sum(x);
            w = warp_sum(w);
            if (lane == 0) {
                rr[t] = eb[t] * x;
                ust[t] = expf(bL - bc[t]) * w;
            }
        }
        float part = 0.f;
        for (size_t e = tid; e < E; e += kBThreads) part = fmaf(dS[e], Ss[e], part);
        part = warp_sum(part);
        if (lane == 0) red[warp] = part;
        __syncthreads();
        if (tid < L) {
            const int j = tid;
            float c0 = 0.f;
            for (int w = 0; w < kWarps; ++w) c0 += red[w];
            float f = 0.f, rsum = 0.f, usum = 0.f;
            for (int t = j; t < L; ++t) {
                for (int s = 0; s < j; ++s) f = fmaf(As[t * kBlk + s], Ds[t * kBlk + s], f);
                rsum += rr[t];
            }
            for (int s = 0; s < j; ++s) usum += ust[s];
            const float dlg = f + rsum + expf(bL) * c0 + usum;
            const size_t zo = (tok0 + j) * H + h;
            // d log gamma / dz = (1 - sigmoid(z)) / tau, and 0 where the forward clamps
            const float deriv = lg[j] > kMinLogGamma ? (1.f - sigmoidf_(a.z[zo])) * a.inv_tau : 0.f;
            a.dz[zo] = dlg * deriv;
        }
        __syncthreads();
        // dS <- e^{b_L} dS' + sum_t e^{b_t} q_t^T dy_t
        const float eL = expf(bL);
        for (size_t e = tid; e < E; e += kBThreads) {
            const int i = (int)(e / dv), j = (int)(e % dv);
            float acc = 0.f;
            for (int t = 0; t < L; ++t) acc = fmaf(eb[t] * Qs[t * dk + i], dYs[t * dv + j], acc);
            dS[e] = fmaf(eL, dS[e], acc);
        }
        __syncthreads();
    }
    if (a.dS0)
        for (size_t e = tid; e < E; e += kBThreads) a.dS0[(size_t)u * E + e] = dS[e];
}

size_t bwd_block_smem(int dk, int dv) {
    return sizeof(float) * ((size_t)4 * kBlk * dk + (size_t)3 * kBlk * dv + 3 * kBlk * kBlk + 5 * kBlk + kBThreads / 32);
}
size_t bwd_ckpt_smem(int dk, int dv) { return sizeof(float) * ((size_t)kBlk * (dk + dv) + 3 * kBlk); }

}  // namespace

size_t prefill_backward_workspace_bytes(int B, int H, int N, int dk, int dv, gret_dtype io) {
    if (bwd_tc_supported(B, H, N, dk, dv, io)) return bwd_tc_workspace_bytes(B, H, N, dv);
    if (bwd_chunked_supported(B, H, N, dk, dv, io)) return bwd_chunked_workspace_bytes(B, H, N, dk, dv, io);
    const size_t units = (size_t)B * H, nblk = (N + kBlk - 1) / kBlk, E = (size_t)dk * dv;
    const size_t ck = (units * nblk * E * 4 + 255) & ~size_t(255);
    return ck + units * E * 4;
}

bool prefill_backward_supported(int dk, int dv) { return bwd_block_smem(dk, dv) <= 227 * 1024; }

int prefill_backward_launches(int B, int H, int N, int dk, int dv, gret_dtype io) {
    if (bwd_tc_supported(B, H, N, dk, dv, io)) return 6;
    return bwd_chunked_supported(B, H, N, dk, dv, io) ? 5 : 2;
}

cudaError_t launch_prefill_backward(const BackwardArgs& in, cudaStream_t s) {
    if (bwd_tc_supported(in.B, in.H, in.N, in.dk, in.dv, in.io)) return launch_bwd_tc(in, s);
    if (bwd_chunked_supported(in.B, in.H, in.N, in.dk, in.dv, in.io)) return launch_bwd_chunked(in, s);
    BwdArgs a;
    a.Q = in.Q; a.K = in.K; a.V = in.V; a.G = in.G; a.dO = in.dO;
    a.z = in.z; a.S0 = in.S0; a.dS_final = in.dS_final;
    a.dQ = in.dQ; a.dK = in.dK; a.dV = in.dV; a.dG = in.dG; a.dz = in.dz; a.dS0 = in.dS0;
    a.B = in.B; a.H = in.H; a.N = in.N; a.dk = in.dk; a.dv = in.dv;
    a.nblk = (in.N + kBlk - 1) / kBlk;
    a.inv_tau = in.inv_tau; a.eps = in.eps; a.gn = in.gn;
    const size_t units = (size_t)in.B * in.H, E = (size_t)in.dk * in.dv;
    uint8_t* ws = static_cast<uint8_t*>(in.workspace);
    a.ckpt = reinterpret_cast<float*>(ws);
    a.dSw = reinterpret_cast<float*>(ws + ((units * a.nblk * E * 4 + 255) & ~size_t(255)));
    const size_t sc = bwd_ckpt_smem(in.dk, in.dv), sb = bwd_block_smem(in.dk, in.dv);
    if (in.io == GRET_BF16) {
        auto k1 = bwd_checkpoint_kernel<__nv_bfloat16>;
        auto k2 = bwd_block_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc);
        cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
        k1<<<(unsigned)units, kBThreads, sc, s>>>(a);
        k2<<<(unsigned)units, kBThreads, sb, s>>>(a);
    } else {
        auto k1 = bwd_checkpoint_kernel<float>;
        auto k2 = bwd_block_kernel<float>;
        cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc);
        cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
        k1<<<(unsigned)units, kBThreads, sc, s>>>(a);
        k2<<<(unsigned)units, kBThreads, sb, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace gret
