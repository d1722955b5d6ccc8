// Chunk-parallel backward of the gated-retention prefill on CUDA cores: every
// (batch, head, chunk) its own thread block, fp32 arithmetic, for head sizes
// that are multiples of 32 (bf16 inputs with d_k = 128 and d_v of 128 or 256
// take the tensor-core backward of gret_backward_tc.cu).
//
// The forward is the chunkwise form of "YOCO 深度技术分析" (sections 2.2 and
// 5.3.2).  Per unit and chunk of L <= C tokens starting from state S_c, with
// b_t the chunk-local inclusive sum of log gamma and b_L its total:
//   A_ts = (q_t . k_s) e^{b_t - b_s}                       (s <= t)
//   y_t  = sum_s A_ts v_s + e^{b_t} q_t S_c
//   S_{c+1} = e^{b_L} S_c + sum_s e^{b_L - b_s} k_s^T v_s
// Both the forward state and the gradient flowing back through it are linear
// recurrences over chunks, so the backward splits into five launches:
//   1. bwd_inc_kernel      per chunk: the state increment and e^{b_L}
//   2. bwd_fwd_scan_kernel per state element: S_c for every chunk
//   3. bwd_dy_kernel       per chunk: y, the GroupNorm * swish backward (dG,
//                          dy) and G_c = sum_t e^{b_t} q_t^T dy_t
//   4. bwd_rev_scan_kernel per state element: dS'_c, the gradient at each
//                          chunk's end (dS'_{c-1} = e^{b_L} dS'_c + G_c), dS0
//   5. bwd_grad_kernel     per chunk: dq, dk, dv and the gate gradient
// with, for D_ts = dy_t . v_s (s <= t):
//   dq_t = sum_s e^{b_t - b_s} D_ts k_s + e^{b_t} S_c dy_t
//   dk_s = sum_t e^{b_t - b_s} D_ts q_t + e^{b_L - b_s} dS' v_s
//   dv_s = sum_t A_ts dy_t            + e^{b_L - b_s} dS'^T k_s
//   dlg_j = sum_{t>=j, s<j} A_ts D_ts + sum_{t>=j} e^{b_t} dy_t.(q_t S_c)
//         + e^{b_L} <dS', S_c> + sum_{s<j} e^{b_L - b_s} k_s.(dS' v_s)
// All exponents are <= 0.  The chunk length is a free parameter of the
// chunkwise form: 64 for bf16 inputs, 32 for fp32 (shared-memory budget).
//
// On CUDA cores products are register-tiled: a warp owns rows (warp + 8 r) of
// an output, its lanes own columns (lane + 32 c), so the row operand is a
// shared-memory broadcast and the column operand a conflict-free row of 32
// words.  Tiles read across their rows ("n-major") are padded to an odd word
// pitch.  States stream through shared memory in 32-column or 32-row slabs.
#include <algorithm>

#include "gret_common.cuh"

namespace gret {
namespace {

constexpr int kCT = 256;   // threads per block
constexpr int kSW = 32;    // slab width
constexpr size_t kMaxSmemB = 227 * 1024;

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~size_t(15); }
__host__ __device__ inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ inline int row_pad(int tsz) { return tsz == 2 ? 2 : 1; }

struct ChunkArgs {
    const void *Q, *K, *V, *G, *dO;
    const float *z, *S0, *dS_final;
    void *dQ, *dK, *dV, *dG;
    float *dz, *dS0;
    float* Sst;     // [units][nc][dk][dv] state before each chunk
    float* dSt;     // [units][nc][dk][dv] G_c, then the gradient at each chunk's end
    float* dyw;     // [B][N][H][dv] gradient of the pre-norm output (GroupNorm epilogue)
    float* decay;   // [units][nc] e^{b_L} of each chunk
    int B, H, N, dk, dv, nc;
    float inv_tau, eps;
    int gn;
};

// Shared-memory layouts (byte offsets), one per kernel, used by host and device.
struct IncLayout {
    size_t k, v, total;
    __host__ __device__ IncLayout(int C, int tsz, int dk, int dv) {
        size_t o = al16(sizeof(float) * (3 * C + 4));
        k = o; o = al16(o + (size_t)C * dk * tsz);
        v = o; o = al16(o + (size_t)C * dv * tsz);
        total = o;
    }
};
struct DyLayout {
    size_t q, k, a, v, dy, sl, total;
    int pq, pv;
    __host__ __device__ DyLayout(int C, int tsz, int dk, int dv) {
        pq = dk + row_pad(tsz);
        pv = dv + row_pad(tsz);
        size_t o = al16(sizeof(float) * (3 * C + 4));
        q = o; o = al16(o + (size_t)C * pq * tsz);
        k = o; o = al16(o + (size_t)C * pq * tsz);
        a = o; o = al16(o + (size_t)C * (C + 1) * 4);
        v = o; o = al16(o + (size_t)C * pv * tsz);
        dy = o; o = al16(o + (size_t)C * (dv + 1) * 4);
        sl = o; o = al16(o + (size_t)2 * kSW * dv * 4);
        total = o;
    }
};
struct GradLayout {
    size_t q, k, v, dy, a, d, sl, total;
    int pq, pv;
    __host__ __device__ GradLayout(int C, int tsz, int dk, int dv) {
        pq = dk + row_pad(tsz);
        pv = dv + row_pad(tsz);
        size_t o = al16(sizeof(float) * (8 * C + 16));
        q = o; o = al16(o + (size_t)C * pq * tsz);
        k = o; o = al16(o + (size_t)C * pq * tsz);
        v = o; o = al16(o + (size_t)C * pv * tsz);
        dy = o; o = al16(o + (size_t)C * (dv + 1) * 4);
        a = o; o = al16(o + (size_t)C * (C + 1) * 4);
        d = o; o = al16(o + (size_t)C * (C + 1) * 4);
        const size_t slabs = (size_t)2 * dk * (kSW + 1) * 4, scratch = (size_t)C * (C + 1) * 4;
        sl = o; o = al16(o + (slabs > scratch ? slabs : scratch));
        total = o;
    }
};

// lg[t] = log gamma of token t of the chunk (0 past L) and bc[t] its inclusive
// sum within the chunk.  Threads 0..C-1 take part; the whole block syncs.
template <int C>
__device__ __forceinline__ void chunk_gate(const float* z, size_t zstride, int L, float inv_tau, float* lg,
                                           float* bc, float* wsum) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float x = 0.f;
    if (tid < C) {
        x = tid < L ? log_gamma(z[(size_t)tid * zstride], inv_tau) : 0.f;
        lg[tid] = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
    }
    __syncthreads();
    if (tid < C) {
        for (int w = 0; w < warp; ++w) x += wsum[w];
        bc[tid] = x;
    }
    __syncthreads();
}

// rows 0..rows-1 of a tile with `cols` elements per row (a multiple of 16 bytes):
// row r < L from src + r * rstride, zeros after; dst row pitch P elements.
template <typename T, int NTH = kCT>
__device__ __forceinline__ void stage_rows(T* dst, int P, const T* src, size_t rstride, int L, int rows, int cols) {
    constexpr int VE = 16 / sizeof(T);
    const int vpr = cols / VE;
    for (int e = threadIdx.x; e < rows * vpr; e += NTH) {
        const int r = e / vpr, cv = e - r * vpr;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (r < L) w = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * rstride) + cv);
        uint32_t* d = reinterpret_cast<uint32_t*>(dst + (size_t)r * P + cv * VE);
        d[0] = w.x;
        d[1] = w.y;
        d[2] = w.z;
        d[3] = w.w;
    }
}

// the same into an fp32 tile, converting element by element
template <typename T, int NTH = kCT>
__device__ __forceinline__ void stage_rows_f32(float* dst, int P, const T* src, size_t rstride, int L, int rows,
                                               int cols) {
    for (int e = threadIdx.x; e < rows * cols; e += NTH) {
        const int r = e / cols, cc = e - r * cols;
        dst[(size_t)r * P + cc] = r < L ? to_f32(src[(size_t)r * rstride + cc]) : 0.f;
    }
}

// As[t][s] = (q_t . k_s) e^{b_t - b_s} for s <= t, else 0; the block syncs after.
template <typename T, int C>
__device__ __forceinline__ void chunk_scores(const T* Qs, const T* Ks, int PQ, int dk, const float* bc, float* As) {
    constexpr int RA = C / 8, CB = C / 32, PA = C + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float acc[RA][CB];
#pragma unroll
    for (int r = 0; r < RA; ++r)
#pragma unroll
        for (int cb = 0; cb < CB; ++cb) acc[r][cb] = 0.f;
    for (int i = 0; i < dk; ++i) {
        float kb[CB];
#pragma unroll
        for (int cb = 0; cb < CB; ++cb) kb[cb] = to_f32(Ks[(lane + 32 * cb) * PQ + i]);
#pragma unroll
        for (int r = 0; r < RA; ++r) {
            const float qa = to_f32(Qs[(warp + 8 * r) * PQ + i]);
#pragma unroll
            for (int cb = 0; cb < CB; ++cb) acc[r][cb] = fmaf(qa, kb[cb], acc[r][cb]);
        }
    }
#pragma unroll
    for (int r = 0; r < RA; ++r)
#pragma unroll
        for (int cb = 0; cb < CB; ++cb) {
            const int t = warp + 8 * r, s = lane + 32 * cb;
            As[t * PA + s] = s <= t ? acc[r][cb] * expf(bc[t] - bc[s]) : 0.f;
        }
    __syncthreads();
}

// out[i][j] = sum_{s<C} X[s][i] w[s] Y[s][j] for i < M, j < Nc (an M x Nc fp32
// matrix, row pitch Nc).  Rows i = warp + 8 r (M <= 128), columns in passes of 128.
template <typename TX, typename TY, int C>
__device__ __forceinline__ void outer_sum(const TX* X, int PX, const TY* Y, int PY, const float* w, int M, int Nc,
                                          float* out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nr = M / 8;
    for (int j0 = 0; j0 < Nc; j0 += 128) {
        const int ncb = min(4, (Nc - j0) / 32);
        float acc[16][4];
#pragma unroll
        for (int r = 0; r < 16; ++r)
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) acc[r][cb] = 0.f;
        for (int s = 0; s < C; ++s) {
            const float ws = w[s];
            float yb[4];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb)
                yb[cb] = cb < ncb ? ws * to_f32(Y[(size_t)s * PY + j0 + lane + 32 * cb]) : 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                if (r < nr) {
                    const float xa = to_f32(X[(size_t)s * PX + warp + 8 * r]);
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) acc[r][cb] = fmaf(xa, yb[cb], acc[r][cb]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 16; ++r)
            if (r < nr)
#pragma unroll
                for (int cb = 0; cb < 4; ++cb)
                    if (cb < ncb) out[(size_t)(warp + 8 * r) * Nc + j0 + lane + 32 * cb] = acc[r][cb];
    }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- 1. per chunk: e^{b_L} and the increment sum_s e^{b_L - b_s} k_s^T v_s,
// written as slot c + 1 of Sst (the last chunk's increment is never needed)
template <typename T, int C>
__global__ void __launch_bounds__(kCT) bwd_inc_kernel(ChunkArgs a) {
    extern __shared__ __align__(16) unsigned char smraw[];
    const int dk = a.dk, dv = a.dv, H = a.H, N = a.N, nc = a.nc;
    const int u = blockIdx.x / nc, c = blockIdx.x - u * nc, b = u / H, h = u - b * H;
    const int tid = threadIdx.x;
    const int n0 = c * C, L = min(C, N - n0);
    const size_t tok0 = (size_t)b * N + n0;
    const IncLayout lay(C, sizeof(T), dk, dv);
    float* lg = reinterpret_cast<float*>(smraw);
    float* bc = lg + C;
    float* wl = bc + C;
    float* wsum = wl + C;
    T* Ks = reinterpret_cast<T*>(smraw + lay.k);
    T* Vs = reinterpret_cast<T*>(smraw + lay.v);
    chunk_gate<C>(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc, wsum);
    const float bL = bc[L - 1];
    if (tid == 0) a.decay[(size_t)u * nc + c] = expf(bL);
    if (c == nc - 1) return;
    if (tid < C) wl[tid] = tid < L ? expf(bL - bc[tid]) : 0.f;
    stage_rows(Ks, dk, static_cast<const T*>(a.K) + (tok0 * H + h) * dk, (size_t)H * dk, L, C, dk);
    stage_rows(Vs, dv, static_cast<const T*>(a.V) + (tok0 * H + h) * dv, (size_t)H * dv, L, C, dv);
    __syncthreads();
    outer_sum<T, T, C>(Ks, dk, Vs, dv, wl, dk, dv, a.Sst + ((size_t)u * nc + c + 1) * (size_t)dk * dv);
}

// ---- 2. per state element: S_0 = S0 (or 0), S_c = e^{b_L(c-1)} S_{c-1} + inc_{c-1}
__global__ void __launch_bounds__(kCT) bwd_fwd_scan_kernel(ChunkArgs a) {
    const size_t E4 = (size_t)a.dk * a.dv / 4, units = (size_t)a.B * a.H, total = units * E4;
    const int nc = a.nc;
    for (size_t idx = (size_t)blockIdx.x * kCT + threadIdx.x; idx < total; idx += (size_t)gridDim.x * kCT) {
        const size_t u = idx / E4, e4 = idx - u * E4;
        float4* st = reinterpret_cast<float4*>(a.Sst) + u * nc * E4 + e4;
        const float* dec = a.decay + u * nc;
        float4 s = a.S0 ? reinterpret_cast<const float4*>(a.S0)[u * E4 + e4] : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 nxt = nc > 1 ? st[E4] : s;
        st[0] = s;
        for (int c = 1; c < nc; ++c) {
            const float4 inc = nxt;
            if (c + 1 < nc) nxt = st[(size_t)(c + 1) * E4];
            const float g = dec[c - 1];
            s.x = fmaf(g, s.x, inc.x);
            s.y = fmaf(g, s.y, inc.y);
            s.z = fmaf(g, s.z, inc.z);
            s.w = fmaf(g, s.w, inc.w);
            st[(size_t)c * E4] = s;
        }
    }
}

// ---- 4. per state element, from the last chunk back: slot c of dSt holds G_c
// on entry and dS'_c (the gradient at chunk c's end) on exit; dS0 gets the
// gradient at the start of the sequence
__global__ void __launch_bounds__(kCT) bwd_rev_scan_kernel(ChunkArgs a) {
    const size_t E4 = (size_t)a.dk * a.dv / 4, units = (size_t)a.B * a.H, total = units * E4;
    const int nc = a.nc;
    for (size_t idx = (size_t)blockIdx.x * kCT + threadIdx.x; idx < total; idx += (size_t)gridDim.x * kCT) {
        const size_t u = idx / E4, e4 = idx - u * E4;
        float4* st = reinterpret_cast<float4*>(a.dSt) + u * nc * E4 + e4;
        const float* dec = a.decay + u * nc;
        float4 cur = a.dS_final ? reinterpret_cast<const float4*>(a.dS_final)[u * E4 + e4]
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 nxt = st[(size_t)(nc - 1) * E4];
        for (int c = nc - 1; c >= 0; --c) {
            const float4 g = nxt;
            if (c > 0) nxt = st[(size_t)(c - 1) * E4];
            st[(size_t)c * E4] = cur;
            const float d = dec[c];
            cur.x = fmaf(d, cur.x, g.x);
            cur.y = fmaf(d, cur.y, g.y);
            cur.z = fmaf(d, cur.z, g.z);
            cur.w = fmaf(d, cur.w, g.w);
        }
        if (a.dS0) reinterpret_cast<float4*>(a.dS0)[u * E4 + e4] = cur;
    }
}

// ---- 3. per chunk: y = A V + e^{b_t} Q S_c, the GroupNorm * swish backward
// (dG out, dy to the workspace), then G_c = sum_t e^{b_t} q_t^T dy_t into dSt.
// With the plain epilogue dy is dO and only G_c is formed.
template <typename T, int C>
__global__ void __launch_bounds__(kCT, 1) bwd_dy_kernel(ChunkArgs a) {
    constexpr int RA = C / 8;
    extern __shared__ __align__(16) unsigned char smraw[];
    const int dk = a.dk, dv = a.dv, H = a.H, N = a.N, nc = a.nc;
    const int u = blockIdx.x / nc, c = blockIdx.x - u * nc, b = u / H, h = u - b * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n0 = c * C, L = min(C, N - n0);
    const size_t tok0 = (size_t)b * N + n0;
    const DyLayout lay(C, sizeof(T), dk, dv);
    const int PQ = lay.pq, PV = lay.pv, PY = dv + 1, PA = C + 1;
    float* lg = reinterpret_cast<float*>(smraw);
    float* bc = lg + C;
    float* eb = bc + C;
    float* wsum = eb + C;
    T* Qs = reinterpret_cast<T*>(smraw + lay.q);
    T* Ks = reinterpret_cast<T*>(smraw + lay.k);
    float* As = reinterpret_cast<float*>(smraw + lay.a);
    T* Vs = reinterpret_cast<T*>(smraw + lay.v);
    float* dYs = reinterpret_cast<float*>(smraw + lay.dy);
    float* Sl = reinterpret_cast<float*>(smraw + lay.sl);
    const size_t qoff = (tok0 * H + h) * (size_t)dk, voff = (tok0 * H + h) * (size_t)dv;

    chunk_gate<C>(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc, wsum);
    if (tid < C) eb[tid] = tid < L ? expf(bc[tid]) : 0.f;
    stage_rows(Qs, PQ, static_cast<const T*>(a.Q) + qoff, (size_t)H * dk, L, C, dk);
    if (a.gn) {
        stage_rows(Ks, PQ, static_cast<const T*>(a.K) + qoff, (size_t)H * dk, L, C, dk);
        stage_rows(Vs, PV, static_cast<const T*>(a.V) + voff, (size_t)H * dv, L, C, dv);
    } else {
        stage_rows_f32(dYs, PY, static_cast<const T*>(a.dO) + voff, (size_t)H * dv, L, C, dv);
    }
    __syncthreads();

    if (a.gn) {
        chunk_scores<T, C>(Qs, Ks, PQ, dk, bc, As);
        const int NJ = dv / 32;   // <= 8 column groups of 32
        float y[RA][8];
#pragma unroll
        for (int r = 0; r < RA; ++r)
#pragma unroll
            for (int cb = 0; cb < 8; ++cb) y[r][cb] = 0.f;
        // Q S_c, S_c streamed in slabs of 32 rows (double-buffered async copies)
        const float* S = a.Sst + ((size_t)u * nc + c) * (size_t)dk * dv;
        const int nsl = dk / kSW, vec = kSW * dv / 4;
        for (int e = tid; e < vec; e += kCT) cp_async16(Sl + 4 * e, S + 4 * e);
        cp_async_commit();
        for (int sl = 0; sl < nsl; ++sl) {
            if (sl + 1 < nsl) {
                const float* src = S + (size_t)(sl + 1) * kSW * dv;
                float* dst = Sl + (size_t)((sl + 1) & 1) * kSW * dv;
                for (int e = tid; e < vec; e += kCT) cp_async16(dst + 4 * e, src + 4 * e);
                cp_async_commit();
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();
            const float* Sb = Sl + (size_t)(sl & 1) * kSW * dv;
            for (int ii = 0; ii < kSW; ++ii) {
                float sb[8];
#pragma unroll
                for (int cb = 0; cb < 8; ++cb) sb[cb] = cb < NJ ? Sb[ii * dv + lane + 32 * cb] : 0.f;
#pragma unroll
                for (int r = 0; r < RA; ++r) {
                    const float qa = to_f32(Qs[(warp + 8 * r) * PQ + sl * kSW + ii]);
#pragma unroll
                    for (int cb = 0; cb < 8; ++cb) y[r][cb] = fmaf(qa, sb[cb], y[r][cb]);
                }
            }
            __syncthreads();   // this buffer is refilled two slabs on
        }
#pragma unroll
        for (int r = 0; r < RA; ++r) {
            const float e = eb[warp + 8 * r];
#pragma unroll
            for (int cb = 0; cb < 8; ++cb) y[r][cb] *= e;
        }
        // + A V
        for (int s = 0; s < C; ++s) {
            float vb[8];
#pragma unroll
            for (int cb = 0; cb < 8; ++cb) vb[cb] = cb < NJ ? to_f32(Vs[s * PV + lane + 32 * cb]) : 0.f;
#pragma unroll
            for (int r = 0; r < RA; ++r) {
                const float aa = As[(warp + 8 * r) * PA + s];
#pragma unroll
                for (int cb = 0; cb < 8; ++cb) y[r][cb] = fmaf(aa, vb[cb], y[r][cb]);
            }
        }
        // GroupNorm (biased variance, no affine) * swish(G) backward, one row per warp
        const T* Gg = static_cast<const T*>(a.G) + voff;
        const T* dOg = static_cast<const T*>(a.dO) + voff;
        T* dGg = static_cast<T*>(a.dG) + voff;
        float* dyw = a.dyw + voff;
        const float inv_dv = 1.0f / (float)dv;
#pragma unroll
        for (int r = 0; r < RA; ++r) {
            const int t = warp + 8 * r;
            if (t < L) {
                const size_t ro = (size_t)t * H * dv;
                float s1 = 0.f;
#pragma unroll
                for (int cb = 0; cb < 8; ++cb) s1 += y[r][cb];
                const float mean = warp_sum(s1) * inv_dv;
                float s2 = 0.f;
#pragma unroll
                for (int cb = 0; cb < 8; ++cb)
                    if (cb < NJ) {
                        const float d = y[r][cb] - mean;
                        s2 = fmaf(d, d, s2);
                    }
                const float rstd = rsqrtf(warp_sum(s2) * inv_dv + a.eps);
                float m1 = 0.f, m2 = 0.f;
#pragma unroll
                for (int cb = 0; cb < 8; ++cb)
                    if (cb < NJ) {
                        const int j = lane + 32 * cb;
                        const float g = to_f32(Gg[ro + j]), go = to_f32(dOg[ro + j]);
                        const float sg = sigmoidf_(g), n = (y[r][cb] - mean) * rstd;
                        // d/dg [g sigmoid(g)] = sigmoid(g) (1 + g (1 - sigmoid(g)))
                        dGg[ro + j] = from_f32<T>(go * n * sg * (1.f + g * (1.f - sg)));
                        const float dn = go * g * sg;
                        dYs[t * PY + j] = dn;
                        y[r][cb] = n;
                        m1 += dn;
                        m2 = fmaf(dn, n, m2);
                    }
                m1 = warp_sum(m1) * inv_dv;
                m2 = warp_sum(m2) * inv_dv;
#pragma unroll
                for (int cb = 0; cb < 8; ++cb)
                    if (cb < NJ) {
                        const int j = lane + 32 * cb;
                        const float dy = rstd * (dYs[t * PY + j] - m1 - y[r][cb] * m2);
                        dYs[t * PY + j] = dy;
                        dyw[ro + j] = dy;
                    }
            } else {
#pragma unroll
                for (int cb = 0; cb < 8; ++cb)
                    if (cb < NJ) dYs[t * PY + lane + 32 * cb] = 0.f;
            }
        }
        __syncthreads();
    }
    outer_sum<T, float, C>(Qs, PQ, dYs, PY, eb, dk, dv, a.dSt + ((size_t)u * nc + c) * (size_t)dk * dv);
}

// state slab: rows i < dk, columns j0 .. j0 + 31 of a [dk][dv] fp32 state,
// dk * 8 16-byte vectors (at most 4 per thread, dk <= 128), kept in registers
// between the global load and the shared-memory store (row pitch kSW + 1)
__device__ __forceinline__ void slab_load(const float* src, int dk, int dv, int j0, uint4 (&pre)[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = threadIdx.x + q * kCT;
        if (e < dk * 8) pre[q] = *reinterpret_cast<const uint4*>(src + (size_t)(e >> 3) * dv + j0 + 4 * (e & 7));
    }
}
__device__ __forceinline__ void slab_store(float* dst, int dk, const uint4 (&pre)[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = threadIdx.x + q * kCT;
        if (e < dk * 8) {
            float* d = dst + (e >> 3) * (kSW + 1) + 4 * (e & 7);
            d[0] = __uint_as_float(pre[q].x);
            d[1] = __uint_as_float(pre[q].y);
            d[2] = __uint_as_float(pre[q].z);
            d[3] = __uint_as_float(pre[q].w);
        }
    }
}

// ---- 5. per chunk: dq, dk, dv and dz from S_c, dS'_c and dy
template <typename T, int C>
__global__ void __launch_bounds__(kCT, 1) bwd_grad_kernel(ChunkArgs a) {
    constexpr int RA = C / 8, CB = C / 32, PA = C + 1, PS = kSW + 1;
    extern __shared__ __align__(16) unsigned char smraw[];
    const int dk = a.dk, dv = a.dv, H = a.H, N = a.N, nc = a.nc;
    const int u = blockIdx.x / nc, c = blockIdx.x - u * nc, b = u / H, h = u - b * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n0 = c * C, L = min(C, N - n0);
    const size_t tok0 = (size_t)b * N + n0;
    const GradLayout lay(C, sizeof(T), dk, dv);
    const int PQ = lay.pq, PV = lay.pv, PY = dv + 1, NCB = dk / 32;
    float* lg = reinterpret_cast<float*>(smraw);
    float* bc = lg + C;
    float* eb = bc + C;        // e^{b_t}
    float* wl = eb + C;        // e^{b_L - b_s}
    float* rr = wl + C;        // e^{b_t} dy_t . (q_t S_c)
    float* us = rr + C;        // e^{b_L - b_s} k_s . (dS' v_s)
    float* Fj = us + C;        // sum_{t>=j, s<j} A_ts D_ts
    float* wsum = Fj + 2 * C;
    float* red = wsum + 4;
    T* Qs = reinterpret_cast<T*>(smraw + lay.q);
    T* Ks = reinterpret_cast<T*>(smraw + lay.k);
    T* Vs = reinterpret_cast<T*>(smraw + lay.v);
    float* dYs = reinterpret_cast<float*>(smraw + lay.dy);
    float* As = reinterpret_cast<float*>(smraw + lay.a);
    float* Ds = reinterpret_cast<float*>(smraw + lay.d);   // D_ts e^{b_t - b_s}
    float* SL = reinterpret_cast<float*>(smraw + lay.sl);
    const size_t E = (size_t)dk * dv;
    const float* S = a.Sst + ((size_t)u * nc + c) * E;
    const float* dSp = a.dSt + ((size_t)u * nc + c) * E;
    const size_t qoff = (tok0 * H + h) * (size_t)dk, voff = (tok0 * H + h) * (size_t)dv;

    chunk_gate<C>(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc, wsum);
    const float bL = bc[L - 1];
    if (tid < C) {
        eb[tid] = tid < L ? expf(bc[tid]) : 0.f;
        wl[tid] = tid < L ? expf(bL - bc[tid]) : 0.f;
    }
    stage_rows(Qs, PQ, static_cast<const T*>(a.Q) + qoff, (size_t)H * dk, L, C, dk);
    stage_rows(Ks, PQ, static_cast<const T*>(a.K) + qoff, (size_t)H * dk, L, C, dk);
    stage_rows(Vs, PV, static_cast<const T*>(a.V) + voff, (size_t)H * dv, L, C, dv);
    if (a.gn)
        stage_rows_f32(dYs, PY, static_cast<const float*>(a.dyw) + voff, (size_t)H * dv, L, C, dv);
    else
        stage_rows_f32(dYs, PY, static_cast<const T*>(a.dO) + voff, (size_t)H * dv, L, C, dv);
    __syncthreads();
    chunk_scores<T, C>(Qs, Ks, PQ, dk, bc, As);

    // D = dy V^T on s <= t: Ds = D e^{b_t - b_s}; M = A o D into the slab scratch
    {
        float acc[RA][CB];
#pragma unroll
        for (int r = 0; r < RA; ++r)
#pragma unroll
            for (int cb = 0; cb < CB; ++cb) acc[r][cb] = 0.f;
        for (int j = 0; j < dv; ++j) {
            float vb[CB];
#pragma unroll
            for (int cb = 0; cb < CB; ++cb) vb[cb] = to_f32(Vs[(lane + 32 * cb) * PV + j]);
#pragma unroll
            for (int r = 0; r < RA; ++r) {
                const float ya = dYs[(warp + 8 * r) * PY + j];
#pragma unroll
                for (int cb = 0; cb < CB; ++cb) acc[r][cb] = fmaf(ya, vb[cb], acc[r][cb]);
            }
        }
#pragma unroll
        for (int r = 0; r < RA; ++r)
#pragma unroll
            for (int cb = 0; cb < CB; ++cb) {
                const int t = warp + 8 * r, s = lane + 32 * cb;
                const bool in = s <= t;
                Ds[t * PA + s] = in ? acc[r][cb] * expf(bc[t] - bc[s]) : 0.f;
                SL[t * PA + s] = in ? As[t * PA + s] * acc[r][cb] : 0.f;
            }
    }
    // <dS'_c, S_c>
    {
        const float4* s4 = reinterpret_cast<const float4*>(S);
        const float4* d4 = reinterpret_cast<const float4*>(dSp);
        float part = 0.f;
        for (size_t e = tid; e < E / 4; e += kCT) {
            const float4 x = s4[e], y = d4[e];
            part = fmaf(x.x, y.x, part);
            part = fmaf(x.y, y.y, part);
            part = fmaf(x.z, y.z, part);
            part = fmaf(x.w, y.w, part);
        }
        part = warp_sum(part);
        if (lane == 0) red[warp] = part;
    }
    __syncthreads();
    // F_j = sum_{t >= j} sum_{s < j} M_ts: exclusive prefix along each row, then
    // a suffix sum down each column
    if (tid < C) {
        float* row = SL + tid * PA;
        float run = 0.f;
        for (int s = 0; s < C; ++s) {
            const float v = row[s];
            row[s] = run;
            run += v;
        }
    }
    __syncthreads();
    if (tid < C) {
        float f = 0.f;
        for (int t = tid; t < C; ++t) f += SL[t * PA + tid];
        Fj[tid] = f;
    }
    __syncthreads();

    float accY[RA][4], accW[RA][4];   // dy S_c^T and V dS'^T, columns i = lane + 32 cb
#pragma unroll
    for (int r = 0; r < RA; ++r)
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) accY[r][cb] = accW[r][cb] = 0.f;
    const int NS = dv / kSW;
    uint4 pre[4];

    // pass over S_c: dy S_c^T
    slab_load(S, dk, dv, 0, pre);
    slab_store(SL, dk, pre);
    __syncthreads();
    for (int sl = 0; sl < NS; ++sl) {
        const float* cur = SL + (size_t)(sl & 1) * dk * PS;
        if (sl + 1 < NS) slab_load(S, dk, dv, (sl + 1) * kSW, pre);
        const int j0 = sl * kSW;
        for (int jj = 0; jj < kSW; ++jj) {
            float sb[4];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) sb[cb] = cb < NCB ? cur[(lane + 32 * cb) * PS + jj] : 0.f;
#pragma unroll
            for (int r = 0; r < RA; ++r) {
                const float ya = dYs[(warp + 8 * r) * PY + j0 + jj];
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) accY[r][cb] = fmaf(ya, sb[cb], accY[r][cb]);
            }
        }
        if (sl + 1 < NS) slab_store(SL + (size_t)((sl + 1) & 1) * dk * PS, dk, pre);
        __syncthreads();
    }

    // pass over dS'_c: V dS'^T, and dv for the slab's 32 columns
    T* dVg = static_cast<T*>(a.dV) + voff;
    slab_load(dSp, dk, dv, 0, pre);
    slab_store(SL, dk, pre);
    __syncthreads();
    for (int sl = 0; sl < NS; ++sl) {
        const float* cur = SL + (size_t)(sl & 1) * dk * PS;
        if (sl + 1 < NS) slab_load(dSp, dk, dv, (sl + 1) * kSW, pre);
        const int j0 = sl * kSW;
        for (int jj = 0; jj < kSW; ++jj) {
            float sb[4];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) sb[cb] = cb < NCB ? cur[(lane + 32 * cb) * PS + jj] : 0.f;
#pragma unroll
            for (int r = 0; r < RA; ++r) {
                const float va = to_f32(Vs[(warp + 8 * r) * PV + j0 + jj]);
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) accW[r][cb] = fmaf(va, sb[cb], accW[r][cb]);
            }
        }
        // dv_s (columns j0 + lane) = e^{b_L - b_s} (K dS')_s + sum_t A_ts dy_t
        float dva[RA];
#pragma unroll
        for (int r = 0; r < RA; ++r) dva[r] = 0.f;
        for (int i = 0; i < dk; ++i) {
            const float db = cur[i * PS + lane];
#pragma unroll
            for (int r = 0; r < RA; ++r) dva[r] = fmaf(to_f32(Ks[(warp + 8 * r) * PQ + i]), db, dva[r]);
        }
#pragma unroll
        for (int r = 0; r < RA; ++r) dva[r] *= wl[warp + 8 * r];
        for (int t = 0; t < C; ++t) {
            const float yb = dYs[t * PY + j0 + lane];
#pragma unroll
            for (int r = 0; r < RA; ++r) dva[r] = fmaf(As[t * PA + warp + 8 * r], yb, dva[r]);
        }
#pragma unroll
        for (int r = 0; r < RA; ++r) {
            const int s = warp + 8 * r;
            if (s < L) dVg[(size_t)s * H * dv + j0 + lane] = from_f32<T>(dva[r]);
        }
        if (sl + 1 < NS) slab_store(SL + (size_t)((sl + 1) & 1) * dk * PS, dk, pre);
        __syncthreads();
    }

    // gate pieces r_t, us_s, then dq = Ds K + e^{b_t} dy S^T and dk = Ds^T Q + e^{b_L - b_s} V dS'^T
#pragma unroll
    for (int r = 0; r < RA; ++r) {
        const int t = warp + 8 * r;
        float pr = 0.f, pu = 0.f;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
            if (cb < NCB) {
                const int i = lane + 32 * cb;
                pr = fmaf(to_f32(Qs[t * PQ + i]), accY[r][cb], pr);
                pu = fmaf(to_f32(Ks[t * PQ + i]), accW[r][cb], pu);
            }
        pr = warp_sum(pr);
        pu = warp_sum(pu);
        if (lane == 0) {
            rr[t] = eb[t] * pr;
            us[t] = wl[t] * pu;
        }
        const float et = eb[t], wt = wl[t];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            accY[r][cb] *= et;
            accW[r][cb] *= wt;
        }
    }
    for (int s = 0; s < C; ++s) {
        float kb[4];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) kb[cb] = cb < NCB ? to_f32(Ks[s * PQ + lane + 32 * cb]) : 0.f;
#pragma unroll
        for (int r = 0; r < RA; ++r) {
            const float da = Ds[(warp + 8 * r) * PA + s];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) accY[r][cb] = fmaf(da, kb[cb], accY[r][cb]);
        }
    }
    for (int t = 0; t < C; ++t) {
        float qb[4];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) qb[cb] = cb < NCB ? to_f32(Qs[t * PQ + lane + 32 * cb]) : 0.f;
#pragma unroll
        for (int r = 0; r < RA; ++r) {
            const float da = Ds[t * PA + warp + 8 * r];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) accW[r][cb] = fmaf(da, qb[cb], accW[r][cb]);
        }
    }
    T* dQg = static_cast<T*>(a.dQ) + qoff;
    T* dKg = static_cast<T*>(a.dK) + qoff;
#pragma unroll
    for (int r = 0; r < RA; ++r) {
        const int t = warp + 8 * r;
        if (t < L)
#pragma unroll
            for (int cb = 0; cb < 4; ++cb)
                if (cb < NCB) {
                    const size_t o = (size_t)t * H * dk + lane + 32 * cb;
                    dQg[o] = from_f32<T>(accY[r][cb]);
                    dKg[o] = from_f32<T>(accW[r][cb]);
                }
    }
    __syncthreads();
    // dz_j = dlg_j (1 - sigmoid(z_j)) / tau, zero where the forward clamps log gamma
    if (tid < L) {
        const int j = tid;
        float c0 = 0.f;
        for (int w = 0; w < kCT / 32; ++w) c0 += red[w];
        float rs = 0.f, su = 0.f;
        for (int t = j; t < L; ++t) rs += rr[t];
        for (int s = 0; s < j; ++s) su += us[s];
        const float dlg = Fj[j] + rs + expf(bL) * c0 + su;
        const size_t zo = (tok0 + j) * H + h;
        const float deriv = lg[j] > kMinLogGamma ? (1.f - sigmoidf_(a.z[zo])) * a.inv_tau : 0.f;
        a.dz[zo] = dlg * deriv;
    }
}

}  // namespace
}  // namespace gret

namespace gret {

namespace {
int bwd_chunk_len(gret_dtype io) { return io == GRET_BF16 ? 64 : 32; }
int io_size(gret_dtype io) { return io == GRET_BF16 ? 2 : 4; }
}  // namespace

bool bwd_chunked_supported(int B, int H, int N, int dk, int dv, gret_dtype io) {
    if (dk % 32 != 0 || dv % 32 != 0 || dk > 128 || dv > 256 || B <= 0 || H <= 0 || N <= 0) return false;
    const int C = bwd_chunk_len(io), tsz = io_size(io);
    const long long blocks = (long long)B * H * ((N + C - 1) / C);
    if (blocks >= (1LL << 31)) return false;
    return IncLayout(C, tsz, dk, dv).total <= kMaxSmemB && DyLayout(C, tsz, dk, dv).total <= kMaxSmemB &&
           GradLayout(C, tsz, dk, dv).total <= kMaxSmemB;
}

size_t bwd_chunked_workspace_bytes(int B, int H, int N, int dk, int dv, gret_dtype io) {
    const int C = bwd_chunk_len(io);
    const size_t units = (size_t)B * H, nc = (size_t)(N + C - 1) / C, E = (size_t)dk * dv;
    return 2 * al256(units * nc * E * 4) + al256((size_t)B * N * H * dv * 4) + al256(units * nc * 4);
}

static unsigned scan_blocks(const ChunkArgs& a) {
    const size_t scan_threads = (size_t)a.B * a.H * a.dk * a.dv / 4;
    return (unsigned)std::min<size_t>((scan_threads + kCT - 1) / kCT, 148 * 16);
}

template <typename T, int C>
static cudaError_t run_bwd_chunked(const ChunkArgs& a, cudaStream_t s) {
    const int tsz = sizeof(T);
    const size_t s1 = IncLayout(C, tsz, a.dk, a.dv).total, s3 = DyLayout(C, tsz, a.dk, a.dv).total,
                 s5 = GradLayout(C, tsz, a.dk, a.dv).total;
    auto k1 = bwd_inc_kernel<T, C>;
    auto k3 = bwd_dy_kernel<T, C>;
    auto k5 = bwd_grad_kernel<T, C>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k5, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s5)) != cudaSuccess) return e;
    const unsigned blocks = (unsigned)((size_t)a.B * a.H * a.nc);
    k1<<<blocks, kCT, s1, s>>>(a);
    bwd_fwd_scan_kernel<<<scan_blocks(a), kCT, 0, s>>>(a);
    k3<<<blocks, kCT, s3, s>>>(a);
    bwd_rev_scan_kernel<<<scan_blocks(a), kCT, 0, s>>>(a);
    k5<<<blocks, kCT, s5, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_bwd_chunked(const BackwardArgs& in, cudaStream_t s) {
    ChunkArgs a = {};
    a.Q = in.Q; a.K = in.K; a.V = in.V; a.G = in.G; a.dO = in.dO;
    a.z = in.z; a.S0 = in.S0; a.dS_final = in.dS_final;
    a.dQ = in.dQ; a.dK = in.dK; a.dV = in.dV; a.dG = in.dG; a.dz = in.dz; a.dS0 = in.dS0;
    a.B = in.B; a.H = in.H; a.N = in.N; a.dk = in.dk; a.dv = in.dv;
    a.inv_tau = in.inv_tau; a.eps = in.eps; a.gn = in.gn;
    const int C = bwd_chunk_len(in.io);
    a.nc = (in.N + C - 1) / C;
    const size_t units = (size_t)in.B * in.H, E = (size_t)in.dk * in.dv;
    uint8_t* ws = static_cast<uint8_t*>(in.workspace);
    const size_t st = al256(units * a.nc * E * 4);
    a.Sst = reinterpret_cast<float*>(ws);
    a.dSt = reinterpret_cast<float*>(ws + st);
    a.dyw = reinterpret_cast<float*>(ws + 2 * st);
    a.decay = reinterpret_cast<float*>(ws + 2 * st + al256((size_t)in.B * in.N * in.H * in.dv * 4));
    if (in.io == GRET_BF16) return run_bwd_chunked<__nv_bfloat16, 64>(a, s);
    return run_bwd_chunked<float, 32>(a, s);
}

}  // namespace gret
