// Chunk-parallel backward of the gated-retention prefill: every (batch, head,
// chunk) its own thread block, fp32 accumulation.  Two variants of the
// per-chunk kernels: tensor cores (mma.sync tf32 tiles, bf16 inputs with
// d_k = 128 and d_v of 128 or 256; second half of this file) and CUDA cores
// (fp32 arithmetic, other head sizes that are multiples of 32).
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

// ===========================================================================
// Tensor-core variant for bf16 inputs with d_k = 128 and d_v of 128 or 256:
// the same five steps with chunks of 64 tokens, every product on warp-level
// mma.sync m16n8k8 tiles (tf32 operands, fp32 accumulation).  The bf16 inputs
// are exact in tf32.  Every other operand (states, dy, the score and gradient
// matrices, decay-weighted values) is split into its tf32 rounding and the
// tf32 rounding of the remainder, and a product takes the three partial
// products hi*hi + hi*lo + lo*hi, which keeps it at fp32-level accuracy.
// Shared-memory pitches are chosen so that the fragment loads of the common
// access patterns are bank-conflict free (at most two-way for the transposed
// ones).
constexpr int kDKm = 128;   // d_k of the tensor-core variant
constexpr int kCm = 64;     // its chunk length

__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <bool SPLIT>
__device__ __forceinline__ void tf32_parts(float x, uint32_t& hi, uint32_t& lo) {
    if (SPLIT) {
        hi = f2tf32(x);
        lo = f2tf32(x - __uint_as_float(hi));
    } else {
        hi = __float_as_uint(x);
        lo = 0u;
    }
}

// One warp: acc[nt] += A(0..15, 0..K-1) * B(0..K-1, 8 nt .. 8 nt + 7), with
// A(m, k) = A[m * am + k * ak] and B(k, n) = B[k * bk + n * bn] (K a multiple
// of 8).  Fragment element e of acc[nt] is row g + 8 (e >> 1), column
// 8 nt + 2 q + (e & 1), where g = lane / 4 and q = lane % 4.  SA / SB mark an
// operand that is not exact in tf32.
template <int NT, bool SA, bool SB, typename TA, typename TB>
__device__ __forceinline__ void warp_mma(float (&acc)[NT][4], const TA* A, int am, int ak, const TB* B, int bk,
                                         int bn, int K) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const TA* pa = A + g * am + q * ak;
    const TB* pb = B + q * bk + g * bn;
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t ah[4], al[4];
        tf32_parts<SA>(ldf(pa + k0 * ak), ah[0], al[0]);
        tf32_parts<SA>(ldf(pa + 8 * am + k0 * ak), ah[1], al[1]);
        tf32_parts<SA>(ldf(pa + (k0 + 4) * ak), ah[2], al[2]);
        tf32_parts<SA>(ldf(pa + 8 * am + (k0 + 4) * ak), ah[3], al[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const TB* p = pb + k0 * bk + 8 * nt * bn;
            uint32_t bh[2], bl[2];
            tf32_parts<SB>(ldf(p), bh[0], bl[0]);
            tf32_parts<SB>(ldf(p + 4 * bk), bh[1], bl[1]);
            if (SA) mma_tf32(acc[nt], al, bh);
            if (SB) mma_tf32(acc[nt], ah, bl);
            mma_tf32(acc[nt], ah, bh);
        }
    }
}

template <int NT>
__device__ __forceinline__ void frag_zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
}

// the fragment tile (16 rows x 8 NT columns) to fp32 memory with row pitch ld
template <int NT>
__device__ __forceinline__ void frag_store(const float (&acc)[NT][4], float* out, size_t ld) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        *reinterpret_cast<float2*>(out + g * ld + 8 * nt + 2 * q) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(out + (g + 8) * ld + 8 * nt + 2 * q) = make_float2(acc[nt][2], acc[nt][3]);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

constexpr int kCTm = 512;   // threads per block of the tensor-core kernels (16 warps)

struct IncMmaLayout {
    size_t k, v, total;
    int pk, pv;
    __host__ __device__ explicit IncMmaLayout(int dv) {
        pk = kDKm + 4;
        pv = dv + 8;
        size_t o = al16(sizeof(float) * (3 * kCm + 4));
        k = o; o = al16(o + (size_t)kCm * pk * 2);
        v = o; o = al16(o + (size_t)kCm * pv * 4);
        total = o;
    }
};

// ---- 1 (tensor cores): e^{b_L} and sum_s k_s^T (e^{b_L - b_s} v_s) into slot
// c + 1.  Warp w owns rows 16 (w % 8) .. + 15 of d_k and the column half w / 8.
template <int DV>
__global__ void __launch_bounds__(kCTm, 1) bwd_inc_mma_kernel(ChunkArgs a) {
    constexpr int C = kCm, NT = DV / 16;
    extern __shared__ __align__(16) unsigned char smraw[];
    const int H = a.H, N = a.N, nc = a.nc;
    const int u = blockIdx.x / nc, c = blockIdx.x - u * nc, b = u / H, h = u - b * H;
    const int tid = threadIdx.x, warp = tid >> 5, mi = warp & 7, nh = warp >> 3;
    const int n0 = c * C, L = min(C, N - n0);
    const size_t tok0 = (size_t)b * N + n0;
    const IncMmaLayout lay(DV);
    float* lg = reinterpret_cast<float*>(smraw);
    float* bc = lg + C;
    float* wl = bc + C;
    float* wsum = wl + C;
    __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smraw + lay.k);
    float* Vw = reinterpret_cast<float*>(smraw + lay.v);
    chunk_gate<C>(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc, wsum);
    const float bL = bc[L - 1];
    if (tid == 0) a.decay[(size_t)u * nc + c] = expf(bL);
    if (c == nc - 1) return;
    if (tid < C) wl[tid] = tid < L ? expf(bL - bc[tid]) : 0.f;
    stage_rows<__nv_bfloat16, kCTm>(Ks, lay.pk, static_cast<const __nv_bfloat16*>(a.K) + (tok0 * H + h) * kDKm,
                                    (size_t)H * kDKm, L, C, kDKm);
    __syncthreads();
    const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.V) + (tok0 * H + h) * DV;
    for (int e = tid; e < C * DV; e += kCTm) {
        const int s = e / DV, j = e - s * DV;
        Vw[s * lay.pv + j] = s < L ? wl[s] * __bfloat162float(Vg[(size_t)s * H * DV + j]) : 0.f;
    }
    __syncthreads();
    float* out = a.Sst + ((size_t)u * nc + c + 1) * (size_t)kDKm * DV;
    float acc[NT][4];
    frag_zero(acc);
    // A(i, s) = K[s][i], B(s, j) = wl[s] V[s][j]
    warp_mma<NT, false, true>(acc, Ks + 16 * mi, 1, lay.pk, Vw + nh * (DV / 2), lay.pv, 1, C);
    frag_store(acc, out + (size_t)(16 * mi) * DV + nh * (DV / 2), DV);
}

struct DyMmaLayout {
    size_t q, k, a, v, dy, sl, part, total;
    int pq, pv, py, ps;
    __host__ __device__ explicit DyMmaLayout(int dv) {
        pq = kDKm + 4;
        pv = dv + 16;
        py = dv + 8;
        ps = dv + 8;
        size_t o = al16(sizeof(float) * (3 * kCm + 4));
        q = o; o = al16(o + (size_t)kCm * pq * 2);
        k = o; o = al16(o + (size_t)kCm * pq * 2);
        a = o; o = al16(o + (size_t)kCm * (kCm + 4) * 4);
        v = o; o = al16(o + (size_t)kCm * pv * 2);
        dy = o; o = al16(o + (size_t)kCm * py * 4);
        sl = o; o = al16(o + (size_t)2 * kSW * ps * 4);
        part = o; o = al16(o + (size_t)8 * kCm * 4);
        total = o;
    }
};

// sum over the 4 lanes of a fragment row group (lanes 4 g .. 4 g + 3)
__device__ __forceinline__ float quad_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

// Sum over the four column-quarter warps of a row: each quad writes its partial
// to part[quarter][row]; after the barrier every lane reads the four.
__device__ __forceinline__ float rows_total(const float* part, int t) {
    return part[t] + part[kCm + t] + part[2 * kCm + t] + part[3 * kCm + t];
}

// ---- 3 (tensor cores): y, the GroupNorm * swish backward, G_c.  Warp w owns
// rows 16 (w % 4) .. + 15 and the column quarter w / 4 of the C x C and C x d_v
// products; G_c (d_k x d_v) is cut into 16-row slices and column halves.
template <int DV>
__global__ void __launch_bounds__(kCTm, 1) bwd_dy_mma_kernel(ChunkArgs a) {
    constexpr int C = kCm, PA = C + 4, NTQ = DV / 32, QUART = DV / 4;
    extern __shared__ __align__(16) unsigned char smraw[];
    const int H = a.H, N = a.N, nc = a.nc;
    const int u = blockIdx.x / nc, c = blockIdx.x - u * nc, b = u / H, h = u - b * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3, mb = warp & 3, nq = warp >> 2;
    const int n0 = c * C, L = min(C, N - n0);
    const size_t tok0 = (size_t)b * N + n0;
    const DyMmaLayout lay(DV);
    const int pq = lay.pq, pv = lay.pv, py = lay.py, ps = lay.ps;
    using bf = __nv_bfloat16;
    float* lg = reinterpret_cast<float*>(smraw);
    float* bc = lg + C;
    float* eb = bc + C;
    float* wsum = eb + C;
    bf* Qs = reinterpret_cast<bf*>(smraw + lay.q);
    bf* Ks = reinterpret_cast<bf*>(smraw + lay.k);
    float* As = reinterpret_cast<float*>(smraw + lay.a);
    bf* Vs = reinterpret_cast<bf*>(smraw + lay.v);
    float* dYs = reinterpret_cast<float*>(smraw + lay.dy);
    float* Sl = reinterpret_cast<float*>(smraw + lay.sl);
    float* part = reinterpret_cast<float*>(smraw + lay.part);   // [8][C] row partial sums
    const size_t qoff = (tok0 * H + h) * (size_t)kDKm, voff = (tok0 * H + h) * (size_t)DV;

    chunk_gate<C>(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc, wsum);
    if (tid < C) eb[tid] = tid < L ? expf(bc[tid]) : 0.f;
    stage_rows<bf, kCTm>(Qs, pq, static_cast<const bf*>(a.Q) + qoff, (size_t)H * kDKm, L, C, kDKm);
    if (a.gn) {
        stage_rows<bf, kCTm>(Ks, pq, static_cast<const bf*>(a.K) + qoff, (size_t)H * kDKm, L, C, kDKm);
        stage_rows<bf, kCTm>(Vs, pv, static_cast<const bf*>(a.V) + voff, (size_t)H * DV, L, C, DV);
    } else {
        stage_rows_f32<bf, kCTm>(dYs, py, static_cast<const bf*>(a.dO) + voff, (size_t)H * DV, L, C, DV);
    }
    __syncthreads();

    const int t0 = 16 * mb + g, t1 = t0 + 8;   // the two fragment rows of this lane
    if (a.gn) {
        // G and dO of this lane's fragment elements, fetched now and used after the products
        const bf* Gg = static_cast<const bf*>(a.G) + voff;
        const bf* dOg = static_cast<const bf*>(a.dO) + voff;
        uint32_t gpre[NTQ][2], opre[NTQ][2];
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int t = hf ? t1 : t0;
                const size_t o = (size_t)t * H * DV + nq * QUART + 8 * nt + 2 * q;
                gpre[nt][hf] = t < L ? *reinterpret_cast<const uint32_t*>(Gg + o) : 0u;
                opre[nt][hf] = t < L ? *reinterpret_cast<const uint32_t*>(dOg + o) : 0u;
            }
        // A = (Q K^T) o e^{b_t - b_s} on s <= t
        {
            float acc[2][4];
            frag_zero(acc);
            warp_mma<2, false, false>(acc, Qs + 16 * mb * pq, pq, 1, Ks + 16 * nq * pq, 1, pq, kDKm);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = e < 2 ? t0 : t1, s = 16 * nq + 8 * nt + 2 * q + (e & 1);
                    As[t * PA + s] = s <= t ? acc[nt][e] * expf(bc[t] - bc[s]) : 0.f;
                }
        }
        // y = e^{b_t} Q S_c + A V; S_c streams through shared memory in 32-row
        // slabs (async copies, two buffers)
        float y[NTQ][4];
        frag_zero(y);
        const float* S = a.Sst + ((size_t)u * nc + c) * (size_t)kDKm * DV;
        constexpr int NSL = kDKm / kSW, VPR = DV / 4;
        for (int e = tid; e < kSW * VPR; e += kCTm) {
            const int r = e / VPR, v = e - r * VPR;
            cp_async16(Sl + r * ps + 4 * v, S + (size_t)r * DV + 4 * v);
        }
        cp_async_commit();
        for (int sl = 0; sl < NSL; ++sl) {
            if (sl + 1 < NSL) {
                const float* src = S + (size_t)(sl + 1) * kSW * DV;
                float* dst = Sl + (size_t)((sl + 1) & 1) * kSW * ps;
                for (int e = tid; e < kSW * VPR; e += kCTm) {
                    const int r = e / VPR, v = e - r * VPR;
                    cp_async16(dst + r * ps + 4 * v, src + (size_t)r * DV + 4 * v);
                }
                cp_async_commit();
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();
            const float* Sb = Sl + (size_t)(sl & 1) * kSW * ps;
            warp_mma<NTQ, false, true>(y, Qs + 16 * mb * pq + sl * kSW, pq, 1, Sb + nq * QUART, ps, 1, kSW);
            __syncthreads();   // this buffer is refilled two slabs on
        }
        {
            const float e0 = eb[t0], e1 = eb[t1];
#pragma unroll
            for (int nt = 0; nt < NTQ; ++nt) {
                y[nt][0] *= e0;
                y[nt][1] *= e0;
                y[nt][2] *= e1;
                y[nt][3] *= e1;
            }
        }
        warp_mma<NTQ, true, false>(y, As + 16 * mb * PA, PA, 1, Vs + nq * QUART, pv, 1, C);

        // GroupNorm (biased variance, no affine) * swish(G) backward.  A row's
        // d_v values sit in the 4 lanes of a group in each of four warps: sums
        // go through the quad, then through `part`.
        const float inv_dv = 1.0f / (float)DV;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt) {
            s0 += y[nt][0] + y[nt][1];
            s1 += y[nt][2] + y[nt][3];
        }
        s0 = quad_sum(s0);
        s1 = quad_sum(s1);
        if (q == 0) {
            part[nq * C + t0] = s0;
            part[nq * C + t1] = s1;
        }
        __syncthreads();
        const float mean0 = rows_total(part, t0) * inv_dv, mean1 = rows_total(part, t1) * inv_dv;
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt) {
            float d = y[nt][0] - mean0;
            v0 = fmaf(d, d, v0);
            d = y[nt][1] - mean0;
            v0 = fmaf(d, d, v0);
            d = y[nt][2] - mean1;
            v1 = fmaf(d, d, v1);
            d = y[nt][3] - mean1;
            v1 = fmaf(d, d, v1);
        }
        v0 = quad_sum(v0);
        v1 = quad_sum(v1);
        if (q == 0) {
            part[4 * C + nq * C + t0] = v0;
            part[4 * C + nq * C + t1] = v1;
        }
        __syncthreads();
        const float rstd0 = rsqrtf(rows_total(part + 4 * C, t0) * inv_dv + a.eps);
        const float rstd1 = rsqrtf(rows_total(part + 4 * C, t1) * inv_dv + a.eps);
        __syncthreads();   // every lane has read `part`; it is reused below
        bf* dGg = static_cast<bf*>(a.dG) + voff;
        float m10 = 0.f, m11 = 0.f, m20 = 0.f, m21 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int t = hf ? t1 : t0, j = nq * QUART + 8 * nt + 2 * q;
                const float mean = hf ? mean1 : mean0, rstd = hf ? rstd1 : rstd0;
                float dn[2] = {0.f, 0.f}, nn[2] = {0.f, 0.f};
                if (t < L) {
                    const uint32_t gw = gpre[nt][hf], ow = opre[nt][hf];
                    const float gv[2] = {__uint_as_float(gw << 16), __uint_as_float(gw & 0xffff0000u)};
                    const float gov[2] = {__uint_as_float(ow << 16), __uint_as_float(ow & 0xffff0000u)};
                    float dg[2];
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const float sg = sigmoidf_(gv[k]);
                        nn[k] = (y[nt][2 * hf + k] - mean) * rstd;
                        // d/dg [g sigmoid(g)] = sigmoid(g) (1 + g (1 - sigmoid(g)))
                        dg[k] = gov[k] * nn[k] * sg * (1.f + gv[k] * (1.f - sg));
                        dn[k] = gov[k] * gv[k] * sg;
                    }
                    *reinterpret_cast<uint32_t*>(dGg + (size_t)t * H * DV + j) = pack_bf16x2_rn(dg[0], dg[1]);
                }
                *reinterpret_cast<float2*>(dYs + t * py + j) = make_float2(dn[0], dn[1]);
                y[nt][2 * hf] = nn[0];
                y[nt][2 * hf + 1] = nn[1];
                if (hf) {
                    m11 += dn[0] + dn[1];
                    m21 = fmaf(dn[0], nn[0], fmaf(dn[1], nn[1], m21));
                } else {
                    m10 += dn[0] + dn[1];
                    m20 = fmaf(dn[0], nn[0], fmaf(dn[1], nn[1], m20));
                }
            }
        m10 = quad_sum(m10);
        m11 = quad_sum(m11);
        m20 = quad_sum(m20);
        m21 = quad_sum(m21);
        if (q == 0) {
            part[nq * C + t0] = m10;
            part[nq * C + t1] = m11;
            part[4 * C + nq * C + t0] = m20;
            part[4 * C + nq * C + t1] = m21;
        }
        __syncthreads();
        const float m1a = rows_total(part, t0) * inv_dv, m1b = rows_total(part, t1) * inv_dv;
        const float m2a = rows_total(part + 4 * C, t0) * inv_dv, m2b = rows_total(part + 4 * C, t1) * inv_dv;
        float* dyw = a.dyw + voff;
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int t = hf ? t1 : t0, j = nq * QUART + 8 * nt + 2 * q;
                if (t < L) {
                    const float rstd = hf ? rstd1 : rstd0, m1 = hf ? m1b : m1a, m2 = hf ? m2b : m2a;
                    const float2 dn = *reinterpret_cast<const float2*>(dYs + t * py + j);
                    const float2 dy = make_float2(rstd * (dn.x - m1 - y[nt][2 * hf] * m2),
                                                  rstd * (dn.y - m1 - y[nt][2 * hf + 1] * m2));
                    *reinterpret_cast<float2*>(dYs + t * py + j) = dy;
                    *reinterpret_cast<float2*>(dyw + (size_t)t * H * DV + j) = dy;
                }
            }
        __syncthreads();
    }
    // G_c = sum_t q_t^T (e^{b_t} dy_t): scale the dy rows, then warp w takes
    // rows 16 (w % 8) .. + 15 of d_k and the column half w / 8
    for (int e = tid; e < C * DV; e += kCTm) {
        const int t = e / DV, j = e - t * DV;
        dYs[t * py + j] *= eb[t];
    }
    __syncthreads();
    float* Gc = a.dSt + ((size_t)u * nc + c) * (size_t)kDKm * DV;
    {
        constexpr int NT = DV / 16;
        const int mi = warp & 7, nh = warp >> 3;
        float acc[NT][4];
        frag_zero(acc);
        warp_mma<NT, false, true>(acc, Qs + 16 * mi, 1, pq, dYs + nh * (DV / 2), py, 1, C);
        frag_store(acc, Gc + (size_t)(16 * mi) * DV + nh * (DV / 2), DV);
    }
}

struct GradMmaLayout {
    size_t q, k, v, dy, a, d, sl, part, total;
    int pq, pv, py;
    __host__ __device__ explicit GradMmaLayout(int dv) {
        pq = kDKm + 4;
        pv = dv + 4;
        py = dv + 4;
        size_t o = al16(sizeof(float) * (8 * kCm + 32));
        q = o; o = al16(o + (size_t)kCm * pq * 2);
        k = o; o = al16(o + (size_t)kCm * pq * 2);
        v = o; o = al16(o + (size_t)kCm * pv * 2);
        dy = o; o = al16(o + (size_t)kCm * py * 4);
        a = o; o = al16(o + (size_t)kCm * (kCm + 4) * 4);
        d = o; o = al16(o + (size_t)kCm * (kCm + 4) * 4);
        const size_t slabs = (size_t)2 * kDKm * (kSW + 4) * 4, scratch = (size_t)kCm * (kCm + 4) * 4;
        sl = o; o = al16(o + (slabs > scratch ? slabs : scratch));
        part = o; o = al16(o + (size_t)8 * kCm * 4);
        total = o;
    }
};

// 32-column state slab (rows i < d_k = 128, columns j0 .. j0 + 31 of a [128][dv]
// fp32 state): 1024 16-byte vectors, two per thread of a 512-thread block, held
// in registers between the global load and the shared store (row pitch kSW + 4)
__device__ __forceinline__ void slab_load_m(const float* src, int dv, int j0, uint4 (&pre)[2]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int e = threadIdx.x + k * kCTm;
        pre[k] = *reinterpret_cast<const uint4*>(src + (size_t)(e >> 3) * dv + j0 + 4 * (e & 7));
    }
}
__device__ __forceinline__ void slab_store_m(float* dst, const uint4 (&pre)[2]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int e = threadIdx.x + k * kCTm;
        *reinterpret_cast<uint4*>(dst + (e >> 3) * (kSW + 4) + 4 * (e & 7)) = pre[k];
    }
}

// ---- 5 (tensor cores): dq, dk, dv, dz.  Warp w owns rows 16 (w % 4) .. + 15
// and the column quarter w / 4 of each product.
template <int DV>
__global__ void __launch_bounds__(kCTm, 1) bwd_grad_mma_kernel(ChunkArgs a) {
    constexpr int C = kCm, PA = C + 4, PS = kSW + 4, NS = DV / kSW, NW = kCTm / 32;
    extern __shared__ __align__(16) unsigned char smraw[];
    const int H = a.H, N = a.N, nc = a.nc;
    const int u = blockIdx.x / nc, c = blockIdx.x - u * nc, b = u / H, h = u - b * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3, mb = warp & 3, nq = warp >> 2;
    const int n0 = c * C, L = min(C, N - n0);
    const size_t tok0 = (size_t)b * N + n0;
    const GradMmaLayout lay(DV);
    const int pq = lay.pq, pv = lay.pv, py = lay.py;
    using bf = __nv_bfloat16;
    float* lg = reinterpret_cast<float*>(smraw);
    float* bc = lg + C;
    float* eb = bc + C;        // e^{b_t}
    float* wl = eb + C;        // e^{b_L - b_s}
    float* rr = wl + C;        // e^{b_t} dy_t . (q_t S_c)
    float* us = rr + C;        // e^{b_L - b_s} k_s . (dS' v_s)
    float* Fj = us + C;        // sum_{t>=j, s<j} A_ts D_ts
    float* wsum = Fj + 2 * C;
    float* red = wsum + 4;     // [NW]
    bf* Qs = reinterpret_cast<bf*>(smraw + lay.q);
    bf* Ks = reinterpret_cast<bf*>(smraw + lay.k);
    bf* Vs = reinterpret_cast<bf*>(smraw + lay.v);
    float* dYs = reinterpret_cast<float*>(smraw + lay.dy);
    float* As = reinterpret_cast<float*>(smraw + lay.a);
    float* Ds = reinterpret_cast<float*>(smraw + lay.d);   // D_ts e^{b_t - b_s}
    float* SL = reinterpret_cast<float*>(smraw + lay.sl);
    float* part = reinterpret_cast<float*>(smraw + lay.part);
    const size_t E = (size_t)kDKm * DV;
    const float* S = a.Sst + ((size_t)u * nc + c) * E;
    const float* dSp = a.dSt + ((size_t)u * nc + c) * E;
    const size_t qoff = (tok0 * H + h) * (size_t)kDKm, voff = (tok0 * H + h) * (size_t)DV;
    const int t0 = 16 * mb + g, t1 = t0 + 8;

    chunk_gate<C>(a.z + tok0 * H + h, (size_t)H, L, a.inv_tau, lg, bc, wsum);
    const float bL = bc[L - 1];
    if (tid < C) {
        eb[tid] = tid < L ? expf(bc[tid]) : 0.f;
        wl[tid] = tid < L ? expf(bL - bc[tid]) : 0.f;
    }
    stage_rows<bf, kCTm>(Qs, pq, static_cast<const bf*>(a.Q) + qoff, (size_t)H * kDKm, L, C, kDKm);
    stage_rows<bf, kCTm>(Ks, pq, static_cast<const bf*>(a.K) + qoff, (size_t)H * kDKm, L, C, kDKm);
    stage_rows<bf, kCTm>(Vs, pv, static_cast<const bf*>(a.V) + voff, (size_t)H * DV, L, C, DV);
    if (a.gn)
        stage_rows_f32<float, kCTm>(dYs, py, static_cast<const float*>(a.dyw) + voff, (size_t)H * DV, L, C, DV);
    else
        stage_rows_f32<bf, kCTm>(dYs, py, static_cast<const bf*>(a.dO) + voff, (size_t)H * DV, L, C, DV);
    __syncthreads();

    // A = (Q K^T) o e^{b_t - b_s} on s <= t
    {
        float acc[2][4];
        frag_zero(acc);
        warp_mma<2, false, false>(acc, Qs + 16 * mb * pq, pq, 1, Ks + 16 * nq * pq, 1, pq, kDKm);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = e < 2 ? t0 : t1, s = 16 * nq + 8 * nt + 2 * q + (e & 1);
                As[t * PA + s] = s <= t ? acc[nt][e] * expf(bc[t] - bc[s]) : 0.f;
            }
    }
    // D = dy V^T on s <= t: Ds = D e^{b_t - b_s}; M = A o D into the slab scratch
    {
        float acc[2][4];
        frag_zero(acc);
        warp_mma<2, true, false>(acc, dYs + 16 * mb * py, py, 1, Vs + 16 * nq * pv, 1, pv, DV);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = e < 2 ? t0 : t1, s = 16 * nq + 8 * nt + 2 * q + (e & 1);
                const bool in = s <= t;
                Ds[t * PA + s] = in ? acc[nt][e] * expf(bc[t] - bc[s]) : 0.f;
                SL[t * PA + s] = in ? As[t * PA + s] * acc[nt][e] : 0.f;
            }
    }
    // <dS'_c, S_c>
    {
        const float4* s4 = reinterpret_cast<const float4*>(S);
        const float4* d4 = reinterpret_cast<const float4*>(dSp);
        float acc = 0.f;
#pragma unroll 4
        for (int e = tid; e < (int)(E / 4); e += kCTm) {
            const float4 x = s4[e], y = d4[e];
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
            acc = fmaf(x.z, y.z, acc);
            acc = fmaf(x.w, y.w, acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) red[warp] = acc;
    }
    __syncthreads();
    // F_j = sum_{t >= j} sum_{s < j} M_ts
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

    float accY[4][4], accW[4][4];   // dy S_c^T and V dS'^T: rows t0/t1, columns 32 nq + ...
    frag_zero(accY);
    frag_zero(accW);
    uint4 pre[2];
    // pass over S_c
    slab_load_m(S, DV, 0, pre);
    slab_store_m(SL, pre);
    __syncthreads();
    for (int sl = 0; sl < NS; ++sl) {
        const float* cur = SL + (size_t)(sl & 1) * kDKm * PS;
        if (sl + 1 < NS) slab_load_m(S, DV, (sl + 1) * kSW, pre);
        // B(j, i) = S_c[i][j]
        warp_mma<4, true, true>(accY, dYs + 16 * mb * py + sl * kSW, py, 1, cur + 32 * nq * PS, 1, PS, kSW);
        if (sl + 1 < NS) slab_store_m(SL + (size_t)((sl + 1) & 1) * kDKm * PS, pre);
        __syncthreads();
    }
    // pass over dS'_c: V dS'^T, and dv for the slab's 32 columns
    bf* dVg = static_cast<bf*>(a.dV) + voff;
    slab_load_m(dSp, DV, 0, pre);
    slab_store_m(SL, pre);
    __syncthreads();
    for (int sl = 0; sl < NS; ++sl) {
        const float* cur = SL + (size_t)(sl & 1) * kDKm * PS;
        if (sl + 1 < NS) slab_load_m(dSp, DV, (sl + 1) * kSW, pre);
        const int j0 = sl * kSW;
        warp_mma<4, false, true>(accW, Vs + 16 * mb * pv + j0, pv, 1, cur + 32 * nq * PS, 1, PS, kSW);
        // dv_s = e^{b_L - b_s} (K dS')_s + sum_t A_ts dy_t over columns j0 + 8 nq .. + 7
        float dva[1][4];
        frag_zero(dva);
        warp_mma<1, false, true>(dva, Ks + 16 * mb * pq, pq, 1, cur + 8 * nq, PS, 1, kDKm);
        {
            const float w0 = wl[t0], w1 = wl[t1];
            dva[0][0] *= w0;
            dva[0][1] *= w0;
            dva[0][2] *= w1;
            dva[0][3] *= w1;
        }
        warp_mma<1, true, true>(dva, As + 16 * mb, 1, PA, dYs + j0 + 8 * nq, py, 1, C);
        {
            const int j = j0 + 8 * nq + 2 * q;
            if (t0 < L)
                *reinterpret_cast<uint32_t*>(dVg + (size_t)t0 * H * DV + j) = pack_bf16x2_rn(dva[0][0], dva[0][1]);
            if (t1 < L)
                *reinterpret_cast<uint32_t*>(dVg + (size_t)t1 * H * DV + j) = pack_bf16x2_rn(dva[0][2], dva[0][3]);
        }
        if (sl + 1 < NS) slab_store_m(SL + (size_t)((sl + 1) & 1) * kDKm * PS, pre);
        __syncthreads();
    }

    // row dots q_t . (S dy_t) and k_s . (dS' v_s) (quarters through `part`), then
    // dq = Ds K + e^{b_t} dy S^T and dk = Ds^T Q + e^{b_L - b_s} V dS'^T
    {
        float r0 = 0.f, r1 = 0.f, u0 = 0.f, u1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int i = 32 * nq + 8 * nt + 2 * q;
            r0 += ldf(Qs + t0 * pq + i) * accY[nt][0] + ldf(Qs + t0 * pq + i + 1) * accY[nt][1];
            r1 += ldf(Qs + t1 * pq + i) * accY[nt][2] + ldf(Qs + t1 * pq + i + 1) * accY[nt][3];
            u0 += ldf(Ks + t0 * pq + i) * accW[nt][0] + ldf(Ks + t0 * pq + i + 1) * accW[nt][1];
            u1 += ldf(Ks + t1 * pq + i) * accW[nt][2] + ldf(Ks + t1 * pq + i + 1) * accW[nt][3];
        }
        r0 = quad_sum(r0);
        r1 = quad_sum(r1);
        u0 = quad_sum(u0);
        u1 = quad_sum(u1);
        if (q == 0) {
            part[nq * C + t0] = r0;
            part[nq * C + t1] = r1;
            part[4 * C + nq * C + t0] = u0;
            part[4 * C + nq * C + t1] = u1;
        }
        const float e0 = eb[t0], e1 = eb[t1], w0 = wl[t0], w1 = wl[t1];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            accY[nt][0] *= e0;
            accY[nt][1] *= e0;
            accY[nt][2] *= e1;
            accY[nt][3] *= e1;
            accW[nt][0] *= w0;
            accW[nt][1] *= w0;
            accW[nt][2] *= w1;
            accW[nt][3] *= w1;
        }
    }
    // dq: A(t, s) = Ds[t][s], B(s, i) = K[s][i];  dk: A(s, t) = Ds[t][s], B(t, i) = Q[t][i]
    warp_mma<4, true, false>(accY, Ds + 16 * mb * PA, PA, 1, Ks + 32 * nq, pq, 1, C);
    warp_mma<4, true, false>(accW, Ds + 16 * mb, 1, PA, Qs + 32 * nq, pq, 1, C);
    {
        bf* dQg = static_cast<bf*>(a.dQ) + qoff;
        bf* dKg = static_cast<bf*>(a.dK) + qoff;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int i = 32 * nq + 8 * nt + 2 * q;
            if (t0 < L) {
                const size_t o = (size_t)t0 * H * kDKm + i;
                *reinterpret_cast<uint32_t*>(dQg + o) = pack_bf16x2_rn(accY[nt][0], accY[nt][1]);
                *reinterpret_cast<uint32_t*>(dKg + o) = pack_bf16x2_rn(accW[nt][0], accW[nt][1]);
            }
            if (t1 < L) {
                const size_t o = (size_t)t1 * H * kDKm + i;
                *reinterpret_cast<uint32_t*>(dQg + o) = pack_bf16x2_rn(accY[nt][2], accY[nt][3]);
                *reinterpret_cast<uint32_t*>(dKg + o) = pack_bf16x2_rn(accW[nt][2], accW[nt][3]);
            }
        }
    }
    __syncthreads();
    if (tid < C) {
        rr[tid] = eb[tid] * rows_total(part, tid);
        us[tid] = wl[tid] * rows_total(part + 4 * C, tid);
    }
    __syncthreads();
    // dz_j = dlg_j (1 - sigmoid(z_j)) / tau, zero where the forward clamps log gamma
    if (tid < L) {
        const int j = tid;
        float c0 = 0.f;
        for (int w = 0; w < NW; ++w) c0 += red[w];
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
    if (io == GRET_BF16 && dk == kDKm && (dv == 128 || dv == 256))
        return IncMmaLayout(dv).total <= kMaxSmemB && DyMmaLayout(dv).total <= kMaxSmemB &&
               GradMmaLayout(dv).total <= kMaxSmemB;
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

template <int DV>
static cudaError_t run_bwd_mma(const ChunkArgs& a, cudaStream_t s) {
    const size_t s1 = IncMmaLayout(DV).total, s3 = DyMmaLayout(DV).total, s5 = GradMmaLayout(DV).total;
    auto k1 = bwd_inc_mma_kernel<DV>;
    auto k3 = bwd_dy_mma_kernel<DV>;
    auto k5 = bwd_grad_mma_kernel<DV>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k5, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s5)) != cudaSuccess) return e;
    const unsigned blocks = (unsigned)((size_t)a.B * a.H * a.nc);
    k1<<<blocks, kCTm, s1, s>>>(a);
    bwd_fwd_scan_kernel<<<scan_blocks(a), kCT, 0, s>>>(a);
    k3<<<blocks, kCTm, s3, s>>>(a);
    bwd_rev_scan_kernel<<<scan_blocks(a), kCT, 0, s>>>(a);
    k5<<<blocks, kCTm, s5, s>>>(a);
    return cudaGetLastError();
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
    if (in.io == GRET_BF16 && in.dk == kDKm && in.dv == 256) return run_bwd_mma<256>(a, s);
    if (in.io == GRET_BF16 && in.dk == kDKm && in.dv == 128) return run_bwd_mma<128>(a, s);
    if (in.io == GRET_BF16) return run_bwd_chunked<__nv_bfloat16, 64>(a, s);
    return run_bwd_chunked<float, 32>(a, s);
}

}  // namespace gret
