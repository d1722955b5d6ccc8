// Recurrent decode step of the gated-retention mixer.
//
// "YOCO 深度技术分析", section 2.2 (recurrent form) and section 5.3.7 (decode
// uses the recurrent form on the state prefill left behind); "YOCO"
// (zdszero.github.io), "Self-Decoder": S_t = gamma_t S_{t-1} + K_t^T V_t,
// y_t = Q_t S_t; multi-head output GroupNorm(y) (.) swish(g).
//
// One CTA per (sequence, head) unit.  The fp32 state S [dk][dv] (128 KiB for
// 128 x 256) is the only large operand: the kernel streams it once, reading
// and writing each element exactly once with 128-bit accesses, and forms
// y = q S_new on the fly.  Thread (c, r) owns the float4 column group c of rows
// r, r + R, r + 2R, ...; consecutive threads touch consecutive 16-byte words
// of a row, so every warp access is a fully coalesced 512-byte segment.  Loads
// are issued in batches of kBatch rows before any of them is used, so each
// thread keeps kBatch 16-byte loads in flight.  This step is HBM-bound:
// 2 * 4 * dk * dv bytes per unit against ~0.5 flop per byte.
#include "gret_common.cuh"

namespace gret {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;

template <typename T>
__global__ void __launch_bounds__(kThreads) decode_step_kernel(DecodeArgs a) {
    extern __shared__ float smem[];
    const int dk = a.dk, dv = a.dv;
    const int u = blockIdx.x;
    const int tid = threadIdx.x;
    float* sq = smem;                 // q [dk]
    float* sk = sq + dk;              // k [dk]
    float* red = sk + dk;             // partial y [R][dv]
    float* sy = red + (kThreads / (dv / 4)) * dv;  // y [dv]
    float* sst = sy + dv;             // block-reduction scratch [32]

    const T* q = static_cast<const T*>(a.q) + (size_t)u * dk;
    const T* k = static_cast<const T*>(a.k) + (size_t)u * dk;
    const T* v = static_cast<const T*>(a.v) + (size_t)u * dv;
    for (int i = tid; i < dk; i += kThreads) {
        sq[i] = to_f32(q[i]);
        sk[i] = to_f32(k[i]);
    }
    const float gamma = expf(log_gamma(a.z[u], a.inv_tau));
    __syncthreads();

    const int c4n = dv / 4;           // float4 groups per state row
    const int R = kThreads / c4n;     // rows processed side by side
    const int c4 = tid % c4n;
    const int r0 = tid / c4n;
    float4* S = reinterpret_cast<float4*>(a.S + (size_t)u * dk * dv);
    if (r0 < R) {
        float vv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) vv[e] = to_f32(v[c4 * 4 + e]);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int m0 = r0; m0 < dk; m0 += R * kBatch) {
            float4 s[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                int m = m0 + b * R;
                if (m < dk) s[b] = __ldcs(&S[(size_t)m * c4n + c4]);
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                int m = m0 + b * R;
                if (m < dk) {
                    const float km = sk[m], qm = sq[m];
                    float4 t = s[b];
                    t.x = fmaf(gamma, t.x, km * vv[0]);
                    t.y = fmaf(gamma, t.y, km * vv[1]);
                    t.z = fmaf(gamma, t.z, km * vv[2]);
                    t.w = fmaf(gamma, t.w, km * vv[3]);
                    __stcs(&S[(size_t)m * c4n + c4], t);
                    acc[0] = fmaf(qm, t.x, acc[0]);
                    acc[1] = fmaf(qm, t.y, acc[1]);
                    acc[2] = fmaf(qm, t.z, acc[2]);
                    acc[3] = fmaf(qm, t.w, acc[3]);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) red[r0 * dv + c4 * 4 + e] = acc[e];
    }
    __syncthreads();

    // y = q S_new: add the R partial sums of every column.
    float lsum = 0.f;
    for (int j = tid; j < dv; j += kThreads) {
        float y = 0.f;
        for (int r = 0; r < R; ++r) y += red[r * dv + j];
        sy[j] = y;
        lsum += y;
    }
    T* o = static_cast<T*>(a.o) + (size_t)u * dv;
    if (a.epi == GRET_EPI_NONE) {
        for (int j = tid; j < dv; j += kThreads) o[j] = from_f32<T>(sy[j]);
        return;
    }
    // GroupNorm over the dv channels of this head: mean, then biased variance.
    const int lane = tid & 31, warp = tid >> 5;
    lsum = warp_sum(lsum);
    if (lane == 0) sst[warp] = lsum;
    __syncthreads();
    float mean = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) mean += sst[w];
    mean /= (float)dv;
    float lsq = 0.f;
    for (int j = tid; j < dv; j += kThreads) {
        float d = sy[j] - mean;
        lsq += d * d;
    }
    lsq = warp_sum(lsq);
    __syncthreads();
    if (lane == 0) sst[warp] = lsq;
    __syncthreads();
    float var = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) var += sst[w];
    var /= (float)dv;
    const float rstd = rsqrtf(var + a.eps);
    const T* g = static_cast<const T*>(a.g) + (size_t)u * dv;
    for (int j = tid; j < dv; j += kThreads) {
        float gj = to_f32(g[j]);
        o[j] = from_f32<T>((sy[j] - mean) * rstd * gj * sigmoidf_(gj));
    }
}

size_t decode_smem_bytes(int dk, int dv) {
    int R = kThreads / (dv / 4);
    return sizeof(float) * ((size_t)2 * dk + (size_t)R * dv + dv + 32);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    size_t smem = decode_smem_bytes(a.dk, a.dv);
    if (a.io == GRET_BF16) {
        auto k = decode_step_kernel<__nv_bfloat16>;
        if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<a.num_units, kThreads, smem, s>>>(a);
    } else {
        auto k = decode_step_kernel<float>;
        if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<a.num_units, kThreads, smem, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace gret
