// Tensor-core (tcgen05) backward of the gated-retention prefill for bf16 inputs
// with d_k = 128 and d_v of 128 or 256, on chunks of 128 tokens.
//
// The forward is the chunkwise form of "YOCO 深度技术分析" (sections 2.2 and
// 5.3.2).  Per unit and chunk c of L <= 128 tokens with state S_c before it,
// b_t the chunk-local inclusive sum of log gamma, b_L its total and
// E_ts = e^{b_t - b_s} on s <= t:
//   y_t     = sum_s (q_t . k_s) E_ts v_s + e^{b_t} q_t S_c
//   S_{c+1} = e^{b_L} S_c + sum_s e^{b_L - b_s} k_s^T v_s
// With dy the gradient of y (GroupNorm * swish backward), D_ts = dy_t . v_s,
// A_ts = q_t . k_s and dS'_c the gradient at chunk c's end
// (dS'_{c-1} = e^{b_L} dS'_c + sum_t e^{b_t} q_t^T dy_t):
//   dq_t = sum_s D_ts E_ts k_s + e^{b_t} dy_t S_c^T
//   dk_s = sum_t D_ts E_ts q_t + e^{b_L - b_s} v_s dS'_c^T
//   dv_s = sum_t A_ts E_ts dy_t + e^{b_L - b_s} k_s dS'_c
// and the gate gradient of token j as four sums over the (s, t) pairs that
// straddle it (s < j <= t), none of which cancels:
//   dlg_j = sum_{t>=j, s<j} A_ts D_ts E_ts           (F_j, within the chunk)
//         + sum_{t>=j} dy_t . (e^{b_t} q_t S_c)        (earlier chunks -> t)
//         + e^{b_L} <dS'_c, S_c>                       (earlier -> later chunks)
//         + sum_{s<j} e^{b_L - b_s} k_s . (dS'_c v_s)  (s -> later chunks)
// (the final state's gradient enters through dS' of the last chunk).
//
// Five launches:
//   1. bwd_inc_tc      per chunk and channel half: e^{b_L} and the increment
//                      K~^T V (tcgen05)
//   2. bwd_scan_fwd    per state element: S_c of every chunk as a bf16 pair
//                      (hi = bf16(S), lo = bf16(S - hi))
//   3. bwd_dyq_tc      per chunk: y, the GroupNorm * swish backward (dG, dy),
//                      G_c = sum_t e^{b_t} q_t^T dy_t and dq (tcgen05)
//   4. bwd_scan_rev    per state element: dS'_c as a bf16 pair, dS0 and the
//                      shares of e^{b_L} <dS'_c, S_c>
//   5. bwd_kv_tc       per chunk: dk, dv and dz (tcgen05)
// The products whose operands are not bf16 inputs take them as bf16 pairs:
// a product with one such operand costs two MMAs (x_hi, x_lo), with two of
// them three (hi hi, hi lo, lo hi), which keeps about 16 mantissa bits.  The
// decay factors of a row (e^{b_t}, e^{b_L - b_s}) are applied to fp32
// accumulator rows in tensor memory instead of being folded into an operand.
// The masked score matrices (P, D o E, A o E) are single bf16 operands, as in
// the forward.  With d_v = 256 a chunk runs on a cluster of two CTAs, each
// owning 128 of the output channels: the GroupNorm row sums cross the pair
// through distributed shared memory, and the partial dq (dk) of the two
// channel halves are added by the CTA that stores the row.
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <utility>

#include "gret_common.cuh"
#include "gret_sm100.cuh"

namespace gret {
namespace {

using namespace sm100;

constexpr int kC = 128;                  // chunk length
constexpr int kDK = 128;                 // d_k
constexpr int kBox = 128 * 128;          // bytes of one [128 rows][64 bf16] swizzled box
constexpr int kTile = 2 * kBox;          // [128 rows][128 bf16]
constexpr int kRowThreads = 256;         // eight warps: lane quarter q = w & 3, column half w >> 2
constexpr int kThreads = kRowThreads + 32;
constexpr int kNamedBar = 1;             // named barrier among the row warps
constexpr int kRowThreads16 = 512;       // sixteen row warps: lane quarter q = w & 3, column quarter w >> 2
constexpr int kThreads16 = kRowThreads16 + 32;

struct BwdTcParams {
    CUtensorMap tmQ, tmK, tmV, tmDyH, tmDyL, tmSH, tmSL;
    CUtensorMap tmInc;        // incg as [rows][dv] fp32, box (32, 128): stores of state-shaped rows
    const void *Q, *K, *V, *G, *dO;
    const float *z, *S0, *dS_final;
    void *dQ, *dK, *dV, *dG;
    float *dz, *dS0;
    float* incg;              // [units][nc][dk][dv] fp32: increments, then G_c
    __nv_bfloat16* sh;        // [units][nc][dk][dv]: S_c hi, then dS'_c hi
    __nv_bfloat16* sl;        // the lo halves
    __nv_bfloat16* dyh;       // [B][N][H][dv] dy hi
    __nv_bfloat16* dyl;       // dy lo
    float* rr;                // [2][B][N][H] per channel half: dy_t . (e^{b_t} q_t S_c)
    float* xs;                // [units][nc][dv]: e^{b_L} <dS'_c, S_c> in shares of 128 elements
    float* decay;             // [units][nc] e^{b_L}
    float* bcg;               // [units][nc][128] chunk-local decay sums b_t (flat past the sequence's end)
    float* fus;               // [units][nc][2][256]: F and us per channel half
    unsigned int* status;
    int B, H, N, dv, nc;
    float inv_tau, eps;
    int gn;
};

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

// logistic sigmoid with the fast exponential and divide (a few ulp)
__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

// 16-byte global load through the non-coherent path, issued where it is written
// (volatile), for data read once well after it is requested
__device__ __forceinline__ uint4 ldg_nc_v4(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }

// bf16 pair of x: hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Byte offset of element (row r, column x < 64) of a [rows][64 bf16] box in
// the 128-byte swizzle layout (16-byte chunk x / 8 of row r sits at chunk
// (x / 8) ^ (r % 8)); boxes are 1024-byte aligned.
__device__ __forceinline__ uint32_t sw128(int r, int x) {
    return (uint32_t)(r * 128 + ((((x >> 3) ^ (r & 7)) & 7) << 4) + (x & 7) * 2);
}

// Chunk-local decay sums b_t of the chunk's tokens (0 past L: b_t = b_{L-1})
// into bc[0..127]; threads 0..127 of the NRT row threads compute them, all
// row threads sync after.
template <int NRT = kRowThreads>
__device__ __forceinline__ void chunk_decay(const BwdTcParams& p, size_t tok0, int hh, int L, float* bc, float* wsum) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < kC) {
        float x = tid < L ? log_gamma(p.z[(tok0 + tid) * p.H + hh], p.inv_tau) : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        bc[tid] = x;
    }
    named_bar_sync(kNamedBar, NRT);
    if (tid < kC) {
        float add = 0.f;
        for (int w = 0; w < warp; ++w) add += wsum[w];
        bc[tid] += add;
    }
    named_bar_sync(kNamedBar, NRT);
}

// ---- 1. per chunk and 128-channel half of d_v: e^{b_L} and the increment
// inc_c = sum_s e^{b_L - b_s} k_s^T v_s into slot c of incg ([d][j] fp32).
// K~ = diag(e^{b_L - b}) K is formed in shared memory as a bf16 pair; the MMA
// is D[d][j] = K~^T V (A = K~ MN-major, B = V MN-major), two passes.  96 KB of
// shared memory and 128 tensor-memory columns: two CTAs share an SM.
struct IncCfg {
    static constexpr int OFF_K = 0;                    // K~ hi (in place of K)
    static constexpr int OFF_KL = kTile;               // K~ lo
    static constexpr int OFF_V = 2 * kTile;            // 128 channels of V
    static constexpr int OFF_BC = 3 * kTile;
    static constexpr int OFF_BAR = OFF_BC + kC * 4 + 64;
    static constexpr int OFF_MISC = OFF_BAR + 64;
    static constexpr int SMEM = OFF_MISC + 64 + 1024;  // + alignment slack
};

__global__ void __launch_bounds__(kThreads, 2) bwd_inc_tc(const __grid_constant__ BwdTcParams p) {
    using CF = IncCfg;
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int halves = p.dv / 128, item = blockIdx.x / halves, ch0 = 128 * (blockIdx.x - item * halves);
    const int nc = p.nc, u = item / nc, c = item - u * nc, b = u / p.H, hh = u - b * p.H;
    const int n0 = c * kC, L = min(kC, p.N - n0);
    const size_t tok0 = (size_t)b * p.N + n0;
    const bool need = c + 1 < nc;   // the last chunk's increment is never used
    float* bc = reinterpret_cast<float*>(sm + CF::OFF_BC);
    float* wsum = bc + kC;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);
    const uint32_t bar_ld = sb + CF::OFF_BAR, bar_mma = sb + CF::OFF_BAR + 8, bar_rdy = sb + CF::OFF_BAR + 16;
    if (tid == kRowThreads) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_rdy, kRowThreads / 32);
        *abort_flag = 0;
        fence_mbar_init();
        if (need) {
            mbar_arrive_expect_tx(bar_ld, 2 * kTile);
            for (int x = 0; x < 2; ++x) {
                tma_load_4d(sb + CF::OFF_K + x * kBox, &p.tmK, x * 64, hh, n0, b, bar_ld);
                tma_load_4d(sb + CF::OFF_V + x * kBox, &p.tmV, ch0 + x * 64, hh, n0, b, bar_ld);
            }
        }
    }
    if (warp == kRowThreads / 32) {
        tmem_alloc(smem_u32(tmem_slot), 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;

    if (tid < kRowThreads) {
        chunk_decay(p, tok0, hh, L, bc, wsum);
        const float bL = bc[kC - 1];
        if (tid == 0 && ch0 == 0) p.decay[(size_t)u * nc + c] = __expf(bL);
        // the gradient kernels load the chunk's sums instead of scanning again
        if (tid < kC && ch0 == 0) p.bcg[((size_t)u * nc + c) * kC + tid] = bc[tid];
        // K~ = e^{b_L - b_s} k_s as a bf16 pair: row s, 64 columns per thread
        const int s = tid & 127, xb = tid >> 7;
        const float w = s < L ? __expf(bL - bc[s]) : 0.f;
        if (need && mbar_wait(bar_ld, 0, p.status, abort_flag)) {
            uint8_t* row = sm + CF::OFF_K + xb * kBox + s * 128;
            uint8_t* rowl = sm + CF::OFF_KL + xb * kBox + s * 128;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 v = *reinterpret_cast<const uint4*>(row + ch * 16), hi, lo;
                const uint32_t* e = reinterpret_cast<const uint32_t*>(&v);
                uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
                uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    split2(u2f(e[k] << 16) * w, u2f(e[k] & 0xffff0000u) * w, h[k], l[k]);
                *reinterpret_cast<uint4*>(row + ch * 16) = hi;    // the swizzle permutes whole
                *reinterpret_cast<uint4*>(rowl + ch * 16) = lo;   // 16-byte chunks of one row
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_rdy);
    } else if (lane == 0) {
        // ============================================================ MMA issuer
        constexpr uint32_t id = idesc_bf16(128, 128, true, true);
        if (mbar_wait(bar_rdy, 0, p.status, abort_flag) && need) {
            tc_fence_after();
            for (int pass = 0; pass < 2; ++pass) {
                const uint32_t sK = sb + (pass ? CF::OFF_KL : CF::OFF_K);
#pragma unroll
                for (int k = 0; k < kC / 16; ++k)
                    mma_ss(tm, sdesc_sw128(sK + k * 2048, kBox, 1024), sdesc_sw128(sb + CF::OFF_V + k * 2048, kBox, 1024),
                           id, pass > 0 || k > 0);
            }
        }
        mma_commit(bar_mma);
    }
    // store: row d of the increment (TMEM lane d), 64 columns per thread, staged
    // in the dead K~ tiles as four [128][32] fp32 boxes in the 128-byte swizzle
    // layout and stored by TMA (rows of 512 bytes, written whole)
    const bool stored = mbar_wait(bar_mma, 0, p.status, abort_flag) && need;
    if (tid < kRowThreads) {
        const int q = warp & 3, half = warp >> 2, d = 32 * q + lane;
        if (stored) {
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                uint32_t r[32];
                tmem_ld_x32(tm + ((uint32_t)(32 * q) << 16) + 64 * half + cb * 32, r);
                tmem_wait_ld();
                uint8_t* box = sm + (2 * half + cb) * kBox;   // [128 rows][32 fp32] = 16 KB
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<uint4*>(box + d * 128 + ((k ^ (d & 7)) << 4)) =
                        make_uint4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]);
            }
            fence_proxy_async_smem();
        }
    } else if (lane == 0 && *abort_flag) {
        if (need) mbar_wait_drain(bar_ld, 0, kWaitCycles);
        mbar_wait_drain(bar_mma, 0, kWaitCycles);
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && stored) {
        const int row0 = (u * nc + c) * kDK;
        for (int x = 0; x < 4; ++x) tma_store_2d(&p.tmInc, sb + x * kBox, ch0 + 32 * x, row0);
        bulk_commit();
        bulk_wait<0>();
    }
    if (warp == kRowThreads / 32) tmem_dealloc(tm, 128);
}

// ---- 2. per state element (4 per thread): S_0 = S0 (or 0), S_{c+1} =
// e^{b_L(c)} S_c + inc_c; S_c of every chunk as a bf16 pair
constexpr int kScanThreads = 256;
__global__ void __launch_bounds__(kScanThreads) bwd_scan_fwd(const __grid_constant__ BwdTcParams p) {
    const size_t E4 = (size_t)kDK * p.dv / 4;
    const int nc = p.nc;
    const size_t u = blockIdx.y, e4 = (size_t)blockIdx.x * kScanThreads + threadIdx.x;
    const bool on = e4 < E4;
    const float4* inc = reinterpret_cast<const float4*>(p.incg) + u * nc * E4 + e4;
    uint2* hi = reinterpret_cast<uint2*>(p.sh) + u * nc * E4 + e4;
    uint2* lo = reinterpret_cast<uint2*>(p.sl) + u * nc * E4 + e4;
    const float* dec = p.decay + u * nc;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (on && p.S0) s = reinterpret_cast<const float4*>(p.S0)[u * E4 + e4];
    if (!on) return;
    float4 nxt = nc > 1 ? inc[0] : s;
    for (int c = 0; c < nc; ++c) {
        uint2 h, l;
        split2(s.x, s.y, h.x, l.x);
        split2(s.z, s.w, h.y, l.y);
        hi[(size_t)c * E4] = h;
        lo[(size_t)c * E4] = l;
        if (c + 1 == nc) break;
        const float4 d = nxt;
        if (c + 2 < nc) nxt = inc[(size_t)(c + 1) * E4];
        const float g = dec[c];
        s.x = fmaf(g, s.x, d.x);
        s.y = fmaf(g, s.y, d.y);
        s.z = fmaf(g, s.z, d.z);
        s.w = fmaf(g, s.w, d.w);
    }
}

// ---- 4. per state element, from the last chunk back: cur = dS_final (or 0);
// for c = nc-1 .. 0: slot c <- cur as a bf16 pair (S_c is read from the slot
// first), cur = e^{b_L} cur + G_c; dS0 = cur.  Each warp also writes its
// 128 elements' share of e^{b_L} <cur, S_c> to xs[u][c][warp]; the dk/dv
// kernel adds a chunk's d_v shares.
__global__ void __launch_bounds__(kScanThreads) bwd_scan_rev(const __grid_constant__ BwdTcParams p) {
    const size_t E4 = (size_t)kDK * p.dv / 4, W = E4 / 32;
    const int nc = p.nc;
    const size_t u = blockIdx.y, e4 = (size_t)blockIdx.x * kScanThreads + threadIdx.x;
    if (e4 >= E4) return;
    const float4* gc = reinterpret_cast<const float4*>(p.incg) + u * nc * E4 + e4;
    uint2* hi = reinterpret_cast<uint2*>(p.sh) + u * nc * E4 + e4;
    uint2* lo = reinterpret_cast<uint2*>(p.sl) + u * nc * E4 + e4;
    float* xw = p.xs + u * nc * W + (e4 >> 5);
    const float* dec = p.decay + u * nc;
    float4 cur = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.dS_final) cur = reinterpret_cast<const float4*>(p.dS_final)[u * E4 + e4];
    float4 gn = gc[(size_t)(nc - 1) * E4];
    uint2 hn = hi[(size_t)(nc - 1) * E4], ln = lo[(size_t)(nc - 1) * E4];
    for (int c = nc - 1; c >= 0; --c) {
        const float4 g = gn;
        const uint2 h = hn, l = ln;
        if (c > 0) {
            gn = gc[(size_t)(c - 1) * E4];
            hn = hi[(size_t)(c - 1) * E4];
            ln = lo[(size_t)(c - 1) * E4];
        }
        const float e = dec[c];
        const float s0 = u2f(h.x << 16) + u2f(l.x << 16), s1 = u2f(h.x & 0xffff0000u) + u2f(l.x & 0xffff0000u);
        const float s2 = u2f(h.y << 16) + u2f(l.y << 16), s3 = u2f(h.y & 0xffff0000u) + u2f(l.y & 0xffff0000u);
        float acc = e * (cur.x * s0 + cur.y * s1 + cur.z * s2 + cur.w * s3);
        uint2 nh, nl;
        split2(cur.x, cur.y, nh.x, nl.x);
        split2(cur.z, cur.w, nh.y, nl.y);
        hi[(size_t)c * E4] = nh;
        lo[(size_t)c * E4] = nl;
        cur.x = fmaf(e, cur.x, g.x);
        cur.y = fmaf(e, cur.y, g.y);
        cur.z = fmaf(e, cur.z, g.z);
        cur.w = fmaf(e, cur.w, g.w);
        acc = warp_sum(acc);
        if ((threadIdx.x & 31) == 0) xw[(size_t)c * W] = acc;
    }
    if (p.dS0) reinterpret_cast<float4*>(p.dS0)[u * E4 + e4] = cur;
}

// Shared-memory layout of the two per-chunk gradient kernels: seven
// [128][128] bf16 tiles (two 64-column swizzled boxes each), then small arrays.
struct GradCfg {
    static constexpr int OFF_BC = 7 * kTile;          // b_t [128] of the chunk (bulk-loaded), 16 B spare
    static constexpr int OFF_AUX = OFF_BC + 528;      // 2 KB: exchange buffers / row sums
    static constexpr int NUM_BARS = 24;
    static constexpr int OFF_BAR = OFF_AUX + 2048;
    static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
    static constexpr int SMEM = OFF_MISC + 16;
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// ---- 3. per chunk: y = P V + e^{b_t} Q S_c, the GroupNorm * swish backward
// (dG; dy as a bf16 pair to the workspace), G_c = sum_t e^{b_t} q_t^T dy_t into
// slot c of incg, rr_t = dy_t . (e^{b_t} q_t S_c), and
// dq = (D o E) K + e^{b_t} dy S_c^T.  With PAIR the CTA of cluster rank h owns
// channels 128 h .. 128 h + 127 and rows 64 h .. 64 h + 63 of dq.  Persistent
// like the dk/dv kernel: the issuer loads the next chunk's Q once the rows have
// built Q~^T, V after D, S after dy S^T and K after the last product.
//
// Tensor memory (512 columns): [0,128) scores A, then row-sum scratch, then D,
// then D o E (bf16); [128,256) Y = P V, then e^{b_t} dy S^T + (D o E) K;
// [256,384) Yi = Q S, then G_c; [384,512) P (bf16), then Q~^T as a bf16 pair.
// Shared memory tiles: Q, K, V (this CTA's channels), S_c hi, S_c lo, dy hi,
// dy lo; after the chunk's products the dy tiles carry the dq exchange of the
// pair (lo: the rows sent, hi: the rows received).
template <bool PAIR>
__global__ void __launch_bounds__(kThreads16, 1) bwd_dyq_tc(const __grid_constant__ BwdTcParams p) {
    using CF = GradCfg;
    constexpr int RT = kRowThreads16;
    constexpr int OFF_Q = 0, OFF_K = kTile, OFF_V = 2 * kTile, OFF_SH = 3 * kTile, OFF_SL = 4 * kTile,
                  OFF_DYH = 5 * kTile, OFF_DYL = 6 * kTile;
    constexpr uint32_t R_A = 0, R_Y = 128, R_YI = 256, R_P = 384;
    constexpr int BQ = 0, BK = 1, BV = 2, BS = 3, BA = 4, BYI = 5, BP = 6, BY = 7, BDY = 8, BD = 9, BQI = 10,
                  BQT = 11, BGC = 12, BDS = 13, BDQ = 14, BX0 = 15, BX1 = 16, BX2 = 17, BXQ = 18, BDYRD = 19,
                  BDRAIN = 20, BEND = 21, BPR = 22, BBC = 23;
    static_assert(BBC < CF::NUM_BARS, "barrier count");
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    if (sb & 1023u) {
        if (threadIdx.x == 0) atomicExch(p.status, kDevSmemLayout);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = PAIR ? (int)cluster_ctarank() : 0;
    const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int ncl = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int nc = p.nc, nitems = p.B * p.H * nc;
    const int niter = cid < nitems ? (nitems - 1 - cid) / ncl + 1 : 0;
    const int DV = p.dv, ch0 = 128 * rank;
    auto bar = [&](int i) -> uint32_t { return sb + CF::OFF_BAR + 8 * i; };
    float* bc = reinterpret_cast<float*>(sm + CF::OFF_BC);    // the chunk's decay sums (bulk-loaded)
    float* xch = reinterpret_cast<float*>(sm + CF::OFF_AUX);   // [128][2] round 0, [128][2] round 2
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);
    // one-shot-per-chunk exchange barriers, armed for the bytes the other CTA sends
    auto arm_exchange = [&]() {
        if (p.gn) {
            mbar_arrive_expect_tx(bar(BX0), kC * 8);
            mbar_arrive_expect_tx(bar(BX2), kC * 8);
        }
        mbar_arrive_expect_tx(bar(BXQ), 64 * 128 * 4);
    };

    if (tid == RT) {
        for (int i = 0; i < CF::NUM_BARS; ++i)
            mbar_init(bar(i), (i == BP || i == BDY || i == BQT || i == BDS || i == BEND) ? RT / 32 : 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (PAIR && niter > 0) arm_exchange();
        tma_prefetch_desc(&p.tmQ);
        tma_prefetch_desc(&p.tmK);
        tma_prefetch_desc(&p.tmV);
        tma_prefetch_desc(&p.tmSH);
        tma_prefetch_desc(&p.tmSL);
        tma_prefetch_desc(&p.tmDyH);
        tma_prefetch_desc(&p.tmDyL);
        tma_prefetch_desc(&p.tmInc);
    }
    if (warp == RT / 32) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if constexpr (PAIR) cluster_sync_all();
    const uint32_t tm = *tmem_slot;
    const uint32_t peer = (uint32_t)(rank ^ 1);

    if (tid < RT) {
        const int q = warp & 3, cq = warp >> 2, t = 32 * q + lane;
        const uint32_t lq = (uint32_t)(32 * q) << 16;
        auto warp_arrive = [&](int i) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(i));
        };
        for (int it = 0; it < niter; ++it) {
            const uint32_t par = it & 1;
            const int item = cid + it * ncl;
            const int u = item / nc, c = item - u * nc, b = u / p.H, hh = u - b * p.H;
            const int n0 = c * kC, L = min(kC, p.N - n0);
            const size_t tok0 = (size_t)b * p.N + n0;
            // G and dO of this thread's row and 32 channels, requested now
            // (volatile loads stay where they are written)
            const size_t rowoff = ((tok0 + t) * p.H + hh) * (size_t)DV + ch0 + 32 * cq;
            uint4 gv[4], ov[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                ov[k] = make_uint4(0u, 0u, 0u, 0u);
                gv[k] = make_uint4(0u, 0u, 0u, 0u);
            }
            if (t < L) {
                const uint4* og = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dO) + rowoff);
#pragma unroll
                for (int k = 0; k < 4; ++k) ov[k] = ldg_nc_v4(og + k);
                if (p.gn) {
                    const uint4* gg = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.G) + rowoff);
#pragma unroll
                    for (int k = 0; k < 4; ++k) gv[k] = ldg_nc_v4(gg + k);
                }
            }
            // the chunk's decay sums b_t (loaded with the tiles)
            mbar_wait(bar(BBC), par, p.status, abort_flag);
            const float bt = bc[t], ebt = __expf(bt);

            // ------------------------------------------------ P = A o E, masked
            if (mbar_wait(bar(BA), par, p.status, abort_flag)) {
                tc_fence_after();
                uint32_t r[32], pk[16];
                tmem_ld_x32(tm + lq + R_A + 32 * cq, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int s0 = 32 * cq + 2 * j;
                    const float v0 = s0 <= t ? u2f(r[2 * j]) * __expf(fminf(bt - bc[s0], 0.f)) : 0.f;
                    const float v1 = s0 + 1 <= t ? u2f(r[2 * j + 1]) * __expf(fminf(bt - bc[s0 + 1], 0.f)) : 0.f;
                    pk[j] = pack_bf16x2(v0, v1);
                }
                tmem_st_x16(tm + lq + R_P + 16 * cq, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            warp_arrive(BP);

            // ------------------------------------------------ GroupNorm * swish backward
            // Row sums over the d_v channels: the four column-quarter warps of a lane
            // quarter through tensor-memory columns 8 slot .. 8 slot + 7 (the scores'
            // columns, free after P), the pair through distributed shared memory.
            auto row_sum = [&](int slot, int xbar, float a, float bv, bool two, bool pair, float& ra, float& rb) {
                const uint32_t col = tm + lq + R_A + 8 * slot;
                const uint32_t w2[2] = {f2u(a), f2u(bv)};
                tmem_st_x2(col + 2 * cq, w2);
                tmem_wait_st();
                named_bar_sync(kNamedBar, RT);
                uint32_t r8[8];
                tmem_ld_x8(col, r8);
                tmem_wait_ld();
                ra = u2f(r8[0]) + u2f(r8[2]) + u2f(r8[4]) + u2f(r8[6]);
                rb = u2f(r8[1]) + u2f(r8[3]) + u2f(r8[5]) + u2f(r8[7]);
                if (PAIR && pair) {
                    const int off = slot == 0 ? 2 * t : 2 * kC + 2 * t;
                    if (cq == 0) {
                        const uint32_t remote = cluster_map(smem_u32(xch + off), peer);
                        const uint32_t rbar = cluster_map(bar(xbar), peer);
                        if (two)
                            st_async_f2(remote, rbar, ra, rb);
                        else
                            st_async_f1(remote, rbar, ra);
                    }
                    if (mbar_wait_cluster(bar(xbar), par, p.status, abort_flag)) {
                        ra += xch[off];
                        if (two) rb += xch[off + 1];
                    }
                }
            };
            float y[32];
            const bool ok_y =
                mbar_wait(bar(BY), par, p.status, abort_flag) && mbar_wait(bar(BYI), par, p.status, abort_flag);
            tc_fence_after();
            if (ok_y) {
                uint32_t r[32], ri[32];
                tmem_ld_x32(tm + lq + R_Y + 32 * cq, r);
                tmem_ld_x32(tm + lq + R_YI + 32 * cq, ri);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] = fmaf(ebt, u2f(ri[j]), u2f(r[j]));
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] = 0.f;
            }
            if (p.gn) {
                const float inv_dv = 1.0f / (float)DV;
                // mean and variance from the sums of y and y^2 in one exchange (as the
                // forward's epilogue forms them)
                float s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    s1 += y[j];
                    s2 = fmaf(y[j], y[j], s2);
                }
                row_sum(0, BX0, s1, s2, true, true, s1, s2);
                const float mean = s1 * inv_dv;
                const float var = fmaxf(s2 * inv_dv - mean * mean, 0.f);
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] -= mean;
                const float rstd = rsqrtf(var + p.eps);
                float m1 = 0.f, m2 = 0.f;
                __nv_bfloat16* dGg = static_cast<__nv_bfloat16*>(p.dG) + rowoff;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t* ge = reinterpret_cast<const uint32_t*>(&gv[k]);
                    const uint32_t* oe = reinterpret_cast<const uint32_t*>(&ov[k]);
                    uint4 dg;
                    uint32_t* dge = reinterpret_cast<uint32_t*>(&dg);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float out[2];
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int j = 8 * k + 2 * e + hf;
                            const float g = hf ? u2f(ge[e] & 0xffff0000u) : u2f(ge[e] << 16);
                            const float o = hf ? u2f(oe[e] & 0xffff0000u) : u2f(oe[e] << 16);
                            const float sg = sigmoid_fast(g);
                            const float n = y[j] * rstd;
                            y[j] = n;
                            // d/dg [g sigmoid(g)] = sigmoid(g) (1 + g (1 - sigmoid(g)))
                            out[hf] = o * n * sg * (1.f + g * (1.f - sg));
                            const float dn = o * g * sg;
                            m1 += dn;
                            m2 = fmaf(dn, n, m2);
                        }
                        dge[e] = pack_bf16x2(out[0], out[1]);
                    }
                    if (t < L) reinterpret_cast<uint4*>(dGg)[k] = dg;
                }
                row_sum(2, BX2, m1, m2, true, true, m1, m2);
                m1 *= inv_dv;
                m2 *= inv_dv;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t* ge = reinterpret_cast<const uint32_t*>(&gv[k]);
                    const uint32_t* oe = reinterpret_cast<const uint32_t*>(&ov[k]);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int j = 8 * k + 2 * e + hf;
                            const float g = hf ? u2f(ge[e] & 0xffff0000u) : u2f(ge[e] << 16);
                            const float o = hf ? u2f(oe[e] & 0xffff0000u) : u2f(oe[e] << 16);
                            const float dn = o * g * sigmoid_fast(g);
                            y[j] = rstd * (dn - m1 - y[j] * m2);
                        }
                }
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t* oe = reinterpret_cast<const uint32_t*>(&ov[k]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        y[8 * k + 2 * e] = u2f(oe[e] << 16);
                        y[8 * k + 2 * e + 1] = u2f(oe[e] & 0xffff0000u);
                    }
                }
            }
            // rr_t = dy_t . (e^{b_t} q_t S_c) over this CTA's channels (Yi is still in
            // tensor memory: G_c overwrites it only after every row warp arrived on BQT)
            {
                float rp = 0.f, dummy;
                if (ok_y) {
                    uint32_t ri[32];
                    tmem_ld_x32(tm + lq + R_YI + 32 * cq, ri);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) rp = fmaf(y[j], u2f(ri[j]), rp);
                }
                float rt;
                row_sum(3, 0, rp * ebt, 0.f, false, false, rt, dummy);
                if (cq == 0 && t < L) p.rr[(size_t)rank * p.B * p.N * p.H + (tok0 + t) * p.H + hh] = rt;
            }
            // dy as a bf16 pair into the shared-memory tiles (row t, box cq / 2); the
            // issuer stores the tiles to the workspace
            {
                uint8_t* rh = sm + OFF_DYH + (cq >> 1) * kBox;
                uint8_t* rl = sm + OFF_DYL + (cq >> 1) * kBox;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint4 h, l;
                    split2(y[8 * k], y[8 * k + 1], h.x, l.x);
                    split2(y[8 * k + 2], y[8 * k + 3], h.y, l.y);
                    split2(y[8 * k + 4], y[8 * k + 5], h.z, l.z);
                    split2(y[8 * k + 6], y[8 * k + 7], h.w, l.w);
                    *reinterpret_cast<uint4*>(rh + sw128(t, 32 * (cq & 1) + 8 * k)) = h;
                    *reinterpret_cast<uint4*>(rl + sw128(t, 32 * (cq & 1) + 8 * k)) = l;
                }
            }
            fence_proxy_async_smem();
            warp_arrive(BDY);

            // ------------------------------------------------ Q~^T = (diag(e^{b}) Q)^T as a bf16 pair
            if (ok_y) {
                const uint8_t* qb = sm + OFF_Q + (q >> 1) * kBox;
                const int xq = 32 * (q & 1) + lane;   // column d = 32 q + lane of Q
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t0 = 32 * cq + 2 * j;
                    const float x0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qb + sw128(t0, xq)));
                    const float x1 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qb + sw128(t0 + 1, xq)));
                    split2(x0 * __expf(bc[t0]), x1 * __expf(bc[t0 + 1]), hi[j], lo[j]);
                }
                tmem_st_x16(tm + lq + R_P + 16 * cq, hi);
                tmem_st_x16(tm + lq + R_P + 64 + 16 * cq, lo);
                tmem_wait_st();
            }
            tc_fence_before();
            warp_arrive(BQT);

            // ------------------------------------------------ D o E (bf16) and e^{b_t} dy S^T
            if (mbar_wait(bar(BD), par, p.status, abort_flag)) {
                tc_fence_after();
                uint32_t r[32], pk[16];
                tmem_ld_x32(tm + lq + R_A + 32 * cq, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int s0 = 32 * cq + 2 * j;
                    const float v0 = s0 <= t ? u2f(r[2 * j]) * __expf(fminf(bt - bc[s0], 0.f)) : 0.f;
                    const float v1 = s0 + 1 <= t ? u2f(r[2 * j + 1]) * __expf(fminf(bt - bc[s0 + 1], 0.f)) : 0.f;
                    pk[j] = pack_bf16x2(v0, v1);
                }
                // every row warp has read D before D o E overwrites its first 64 columns
                named_bar_sync(kNamedBar, RT);
                tmem_st_x16(tm + lq + R_A + 16 * cq, pk);
                if (mbar_wait(bar(BQI), par, p.status, abort_flag)) {
                    tc_fence_after();
                    uint32_t v[32];
                    tmem_ld_x32(tm + lq + R_Y + 32 * cq, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = f2u(u2f(v[j]) * ebt);
                    tmem_st_x32(tm + lq + R_Y + 32 * cq, v);
                }
                tmem_wait_st();
            } else {
                named_bar_sync(kNamedBar, RT);
            }
            tc_fence_before();
            warp_arrive(BDS);

            // ------------------------------------------------ G_c rows (lane = d_k row)
            // staged in the dy tiles (free once G_c and the dy store have read them) as
            // four [128][32] fp32 boxes in the 128-byte swizzle layout, stored by TMA
            if (mbar_wait(bar(BGC), par, p.status, abort_flag) && mbar_wait(bar(BDYRD), par, p.status, abort_flag)) {
                tc_fence_after();
                uint32_t v[32];
                tmem_ld_x32(tm + lq + R_YI + 32 * cq, v);
                tmem_wait_ld();
                uint8_t* box = sm + OFF_DYH + cq * kBox;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<uint4*>(box + t * 128 + ((k ^ (t & 7)) << 4)) =
                        make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            }
            fence_proxy_async_smem();
            named_bar_sync(kNamedBar, RT);
            if (tid == 0 && !*abort_flag) {
                for (int x = 0; x < 4; ++x)
                    tma_store_2d(&p.tmInc, sb + OFF_DYH + x * kBox, ch0 + 32 * x, (u * nc + c) * kDK);
                bulk_commit();
            }
            // ------------------------------------------------ dq (this CTA's channel half)
            float dq[32];
            if (mbar_wait(bar(BDQ), par, p.status, abort_flag)) {
                tc_fence_after();
                uint32_t v[32];
                tmem_ld_x32(tm + lq + R_Y + 32 * cq, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) dq[j] = u2f(v[j]);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) dq[j] = 0.f;
            }
            tc_fence_before();
            warp_arrive(BEND);   // this chunk's tensor memory has been read
            // the G_c store has read the dy tiles; the other CTA may send into dy hi
            if (tid == 0) {
                bulk_wait_read<0>();
                if (PAIR) mbar_arrive_remote(cluster_map(bar(BPR), peer));
            }
            named_bar_sync(kNamedBar, RT);
            bool mine = true;
            if constexpr (PAIR) {
                // rows of the other CTA's half leave in one bulk copy, staged in the dy
                // lo tile ([64 rows][128] fp32, 16-byte chunks swizzled by row) and
                // received in the other CTA's dy hi tile
                float* stage = reinterpret_cast<float*>(sm + OFF_DYL);
                const float* recv = reinterpret_cast<const float*>(sm + OFF_DYH);
                const int r = t & 63;
                mine = (t >> 6) == rank;
                if (!mine)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        reinterpret_cast<float4*>(stage + r * 128)[8 * cq + (k ^ (r & 7))] =
                            make_float4(dq[4 * k], dq[4 * k + 1], dq[4 * k + 2], dq[4 * k + 3]);
                fence_proxy_async_smem();
                named_bar_sync(kNamedBar, RT);
                // the other CTA's dy hi tile is free
                if (tid == 0 && mbar_wait_cluster(bar(BPR), par, p.status, abort_flag)) {
                    bulk_copy_to_cluster(cluster_map(sb + OFF_DYH, peer), sb + OFF_DYL, 64 * 128 * 4,
                                         cluster_map(bar(BXQ), peer));
                    bulk_commit();
                }
                if (mine && mbar_wait_cluster(bar(BXQ), par, p.status, abort_flag)) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float4 x = reinterpret_cast<const float4*>(recv + r * 128)[8 * cq + (k ^ (r & 7))];
                        dq[4 * k] += x.x;
                        dq[4 * k + 1] += x.y;
                        dq[4 * k + 2] += x.z;
                        dq[4 * k + 3] += x.w;
                    }
                }
                if (tid == 0) bulk_wait_read<0>();   // the staging tile is read before dy is written again
            }
            if (mine && t < L) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dQ) +
                                                      ((tok0 + t) * p.H + hh) * kDK + 32 * cq);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    dst[k] = make_uint4(pack_bf16x2(dq[8 * k], dq[8 * k + 1]), pack_bf16x2(dq[8 * k + 2], dq[8 * k + 3]),
                                        pack_bf16x2(dq[8 * k + 4], dq[8 * k + 5]),
                                        pack_bf16x2(dq[8 * k + 6], dq[8 * k + 7]));
            }
        }
    } else {
        // ============================================================ TMA + MMA issuer (lane 0)
        constexpr uint32_t id_kk = idesc_bf16(128, 128, false, false);
        constexpr uint32_t id_kn = idesc_bf16(128, 128, false, true);
        auto kmaj = [&](uint32_t base, int k) { return sdesc_sw128(base + (k >> 2) * kBox + (k & 3) * 32, 16, 1024); };
        auto mnmaj = [&](uint32_t base, int k) { return sdesc_sw128(base + k * 2048, kBox, 1024); };
        auto coords = [&](int it, int& n0, int& b, int& hh, int& srow) {
            const int item = cid + it * ncl, u = item / nc, c = item - u * nc;
            b = u / p.H;
            hh = u - b * p.H;
            n0 = c * kC;
            srow = (u * nc + c) * kDK;
        };
        auto load_tile = [&](int it, int bi, const CUtensorMap* m, uint32_t off, int x0) {
            int n0, b, hh, srow;
            coords(it, n0, b, hh, srow);
            mbar_arrive_expect_tx(bar(bi), kTile);
            for (int x = 0; x < 2; ++x) tma_load_4d(sb + off + x * kBox, m, x0 + x * 64, hh, n0, b, bar(bi));
        };
        auto load_s = [&](int it) {
            int n0, b, hh, srow;
            coords(it, n0, b, hh, srow);
            mbar_arrive_expect_tx(bar(BS), 2 * kTile);
            for (int x = 0; x < 2; ++x) {
                tma_load_2d(sb + OFF_SH + x * kBox, &p.tmSH, ch0 + x * 64, srow, bar(BS));
                tma_load_2d(sb + OFF_SL + x * kBox, &p.tmSL, ch0 + x * 64, srow, bar(BS));
            }
        };
        auto load_bc = [&](int it) {
            mbar_arrive_expect_tx(bar(BBC), kC * 4);
            bulk_load(sb + CF::OFF_BC, p.bcg + (size_t)(cid + it * ncl) * kC, kC * 4, bar(BBC));
        };
        if (lane == 0 && niter > 0) {
            load_bc(0);
            load_tile(0, BQ, &p.tmQ, OFF_Q, 0);
            load_tile(0, BK, &p.tmK, OFF_K, 0);
            load_tile(0, BV, &p.tmV, OFF_V, ch0);
            load_s(0);
        }
        for (int it = 0; it < niter; ++it) {
            const uint32_t par = it & 1;
            const bool more = it + 1 < niter;
            if (lane == 0) {
                bool ok = mbar_wait(bar(BQ), par, p.status, abort_flag) && mbar_wait(bar(BK), par, p.status, abort_flag);
                // the rows have read the previous chunk's tensor memory
                ok = ok && (it == 0 || mbar_wait(bar(BEND), par ^ 1, p.status, abort_flag));
                if (ok) {
                    tc_fence_after();
                    // scores A = Q K^T
#pragma unroll
                    for (int k = 0; k < 8; ++k) mma_ss(tm + R_A, kmaj(sb + OFF_Q, k), kmaj(sb + OFF_K, k), id_kk, k > 0);
                }
                mma_commit(bar(BA));
                ok = ok && mbar_wait(bar(BS), par, p.status, abort_flag);
                if (ok) {
                    tc_fence_after();
                    // Yi = Q S_c (S as a bf16 pair)
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ss(tm + R_YI, kmaj(sb + OFF_Q, k), mnmaj(sb + (pass ? OFF_SL : OFF_SH), k), id_kn,
                                   pass > 0 || k > 0);
                }
                mma_commit(bar(BYI));
                ok = ok && mbar_wait(bar(BP), par, p.status, abort_flag) && mbar_wait(bar(BV), par, p.status, abort_flag);
                if (ok) {
                    tc_fence_after();
                    // Y = P V
#pragma unroll
                    for (int k = 0; k < 8; ++k) mma_ts(tm + R_Y, tm + R_P + k * 8, mnmaj(sb + OFF_V, k), id_kn, k > 0);
                }
                mma_commit(bar(BY));
                ok = ok && mbar_wait(bar(BDY), par, p.status, abort_flag);
                if (ok) {
                    // dy (both halves of the pair) to the workspace; rows past the end of
                    // the sequence fall outside the tensor map and are not written
                    int n0, b, hh, srow;
                    coords(it, n0, b, hh, srow);
                    for (int x = 0; x < 2; ++x) {
                        tma_store_4d(&p.tmDyH, sb + OFF_DYH + x * kBox, ch0 + x * 64, hh, n0, b);
                        tma_store_4d(&p.tmDyL, sb + OFF_DYL + x * kBox, ch0 + x * 64, hh, n0, b);
                    }
                    bulk_commit();
                    tc_fence_after();
                    // D = dy V^T (dy as a bf16 pair)
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ss(tm + R_A, kmaj(sb + (pass ? OFF_DYL : OFF_DYH), k), kmaj(sb + OFF_V, k), id_kk,
                                   pass > 0 || k > 0);
                }
                mma_commit(bar(BD));
                if (ok) {
                    // dy S^T: hi hi + hi lo + lo hi
                    for (int pass = 0; pass < 3; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ss(tm + R_Y, kmaj(sb + (pass == 2 ? OFF_DYL : OFF_DYH), k),
                                   kmaj(sb + (pass == 1 ? OFF_SL : OFF_SH), k), id_kk, pass > 0 || k > 0);
                }
                mma_commit(bar(BQI));
                // V is free after D, S after dy S^T: the next chunk's tiles may load
                if (mbar_wait(bar(BD), par, p.status, abort_flag) && more) load_tile(it + 1, BV, &p.tmV, OFF_V, ch0);
                if (mbar_wait(bar(BQI), par, p.status, abort_flag) && more) load_s(it + 1);
                ok = ok && mbar_wait(bar(BQT), par, p.status, abort_flag);
                // Q is free once the rows have built Q~^T
                if (ok && more) load_tile(it + 1, BQ, &p.tmQ, OFF_Q, 0);
                if (ok) {
                    tc_fence_after();
                    // G_c = Q~^T dy: A = Q~^T from tensor memory (lane = d_k row), B = dy MN-major
                    for (int pass = 0; pass < 3; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tm + R_YI, tm + R_P + (pass == 2 ? 64 : 0) + k * 8,
                                   mnmaj(sb + (pass == 1 ? OFF_DYL : OFF_DYH), k), id_kn, pass > 0 || k > 0);
                }
                mma_commit(bar(BGC));
                bulk_wait_read<0>();   // the dy store has read its tiles
                mbar_arrive(bar(BDYRD));
                ok = ok && mbar_wait(bar(BDS), par, p.status, abort_flag);
                // the rows have read this chunk's decay sums
                if (ok && more) load_bc(it + 1);
                if (ok) {
                    tc_fence_after();
                    // dq += (D o E) K
#pragma unroll
                    for (int k = 0; k < 8; ++k) mma_ts(tm + R_Y, tm + R_A + k * 8, mnmaj(sb + OFF_K, k), id_kn, 1);
                }
                mma_commit(bar(BDQ));
                // K is free after the last product
                if (mbar_wait(bar(BDQ), par, p.status, abort_flag) && more) load_tile(it + 1, BK, &p.tmK, OFF_K, 0);
            }
            __syncwarp();
            if constexpr (PAIR) {
                // the next chunk's exchanges, once this chunk's dq has arrived
                if (lane == 0 && more && mbar_wait_cluster(bar(BXQ), par, p.status, abort_flag)) arm_exchange();
                __syncwarp();
            }
        }
        if (lane == 0) {
            mma_commit(bar(BDRAIN));
            mbar_wait_drain(bar(BDRAIN), 0, kWaitCycles);
            bulk_wait<0>();
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();   // no CTA leaves while the other still sends to it
    if (warp == RT / 32) tmem_dealloc(tm, 512);
}

// Sum of v[0..31] over the warp's lanes for each of the 32 columns at once:
// after the five halving steps lane l holds the sum of column l (31 shuffles).
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

// ---- 5. per chunk: dk = (D o E)^T Q + e^{b_L - b_s} V dS'^T,
// dv = (A o E)^T dy + e^{b_L - b_s} K dS' and the gate gradient
//   dz_j = (F_j + sum_{t>=j} rr_t + X_c + sum_{s<j} us_s) (1 - sigmoid(z_j)) / tau
// with F_j = sum_{s<j<=t} A_ts D_ts E_ts and us_s = e^{b_L - b_s} k_s . (dS' v_s).
// The products are taken transposed (tensor-memory lane = key token s), so
// that (A o E)^T and (D o E)^T serve as A operands from tensor memory.  With
// PAIR the CTA of cluster rank h owns channels 128 h .. + 127 (the dv columns,
// a partial dk, F and us) and rows 64 h .. 64 h + 63 of dk; rank 0 forms dz.
// Persistent: a CTA (pair) takes chunks cid, cid + ncl, ...; the issuer loads
// the next chunk's tiles as the current one releases them (V after its last
// product, K after the rows' last read, Q and dy after the last products, dS'
// after the dk exchange, whose buffer is the dS' lo tile).
//
// Tensor memory: [0,128) A^T, then (A o E)^T (bf16); [128,256) D^T, then
// (D o E)^T; [256,384) V dS'^T, scaled, + (D o E)^T Q; [384,512) K dS',
// scaled, + (A o E)^T dy.  Shared tiles: Q, K, V, dy hi, dy lo, dS' hi, dS' lo.
template <bool PAIR>
__global__ void __launch_bounds__(kThreads16, 1) bwd_kv_tc(const __grid_constant__ BwdTcParams p) {
    using CF = GradCfg;
    constexpr int RT = kRowThreads16;
    constexpr int OFF_Q = 0, OFF_K = kTile, OFF_V = 2 * kTile, OFF_DYH = 3 * kTile, OFF_DYL = 4 * kTile,
                  OFF_DSH = 5 * kTile, OFF_DSL = 6 * kTile;
    constexpr uint32_t R_AT = 0, R_DT = 128, R_DK = 256, R_DV = 384;
    constexpr int BQ = 0, BK = 1, BV = 2, BDY = 3, BS = 4, BADT = 5, BINTER = 6, BROWS = 7, BOUT = 8, BXK = 9,
                  BXDONE = 10, BDRAIN = 11, BPR = 12, BBC = 13;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    if (sb & 1023u) {
        if (threadIdx.x == 0) atomicExch(p.status, kDevSmemLayout);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = PAIR ? (int)cluster_ctarank() : 0;
    const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int ncl = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int nc = p.nc, nitems = p.B * p.H * nc;
    const int niter = cid < nitems ? (nitems - 1 - cid) / ncl + 1 : 0;
    const int DV = p.dv, ch0 = 128 * rank;
    auto bar = [&](int i) -> uint32_t { return sb + CF::OFF_BAR + 8 * i; };
    float* bc = reinterpret_cast<float*>(sm + CF::OFF_BC);    // the chunk's decay sums (bulk-loaded)
    float* Facc = reinterpret_cast<float*>(sm + CF::OFF_AUX);   // [128] F_j over this CTA's channels
    float* ush = Facc + kC;                                      // [128] us_s over this CTA's channels
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);

    if (tid == RT) {
        for (int i = 0; i < CF::NUM_BARS; ++i) mbar_init(bar(i), (i == BROWS || i == BXDONE) ? RT / 32 : 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (PAIR && niter > 0) mbar_arrive_expect_tx(bar(BXK), 64 * 128 * 4);
        tma_prefetch_desc(&p.tmQ);
        tma_prefetch_desc(&p.tmK);
        tma_prefetch_desc(&p.tmV);
        tma_prefetch_desc(&p.tmDyH);
        tma_prefetch_desc(&p.tmDyL);
        tma_prefetch_desc(&p.tmSH);
        tma_prefetch_desc(&p.tmSL);
    }
    if (warp == RT / 32) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if constexpr (PAIR) cluster_sync_all();
    const uint32_t tm = *tmem_slot;
    const uint32_t peer = (uint32_t)(rank ^ 1);

    if (tid < RT) {
        const int q = warp & 3, cq = warp >> 2, s = 32 * q + lane;
        const uint32_t lq = (uint32_t)(32 * q) << 16;
        auto warp_arrive = [&](int i) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(i));
        };
        for (int it = 0; it < niter; ++it) {
            const uint32_t par = it & 1;
            const int item = cid + it * ncl;
            const int u = item / nc, c = item - u * nc, b = u / p.H, hh = u - b * p.H;
            const int n0 = c * kC, L = min(kC, p.N - n0);
            const size_t tok0 = (size_t)b * p.N + n0;
            // the chunk's decay sums b_t (loaded with the tiles)
            mbar_wait(bar(BBC), par, p.status, abort_flag);
            if (tid < kC) {
                Facc[tid] = 0.f;
                ush[tid] = 0.f;
            }
            const float bs = bc[s], bL = bc[kC - 1];
            const float ws = s < L ? __expf(bL - bs) : 0.f;
            named_bar_sync(kNamedBar, RT);

            // ------------------------------------------------ (A o E)^T, (D o E)^T and F
            // thread (s, cq): key token s, query tokens t = 32 cq .. 32 cq + 31
            const bool ok = mbar_wait(bar(BADT), par, p.status, abort_flag);
            tc_fence_after();
            {
                float m[32];
                uint32_t pa[16], pd[16];
                if (ok) {
                    uint32_t ra[32], rd[32];
                    tmem_ld_x32(tm + lq + R_AT + 32 * cq, ra);
                    tmem_ld_x32(tm + lq + R_DT + 32 * cq, rd);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float av[2], dv2[2];
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int jj = 2 * j + hf, t = 32 * cq + jj;
                            const float e = (t >= s && t < L) ? __expf(fminf(bc[t] - bs, 0.f)) : 0.f;
                            const float a = u2f(ra[jj]), d = u2f(rd[jj]);
                            av[hf] = a * e;
                            dv2[hf] = d * e;
                            m[jj] = av[hf] * d;
                        }
                        pa[j] = pack_bf16x2(av[0], av[1]);
                        pd[j] = pack_bf16x2(dv2[0], dv2[1]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) m[j] = 0.f;
                }
                // C_s(j) = sum_{t >= j} M_ts: suffix within this column quarter, plus
                // the later quarters' row totals (exchanged through tensor-memory
                // columns 64..71, free once every warp has read A^T)
                float run = 0.f;
#pragma unroll
                for (int j = 31; j >= 0; --j) {
                    run += m[j];
                    m[j] = run;
                }
                named_bar_sync(kNamedBar, RT);   // every row warp has read A^T and D^T
                if (ok) {
                    tmem_st_x16(tm + lq + R_AT + 16 * cq, pa);
                    tmem_st_x16(tm + lq + R_DT + 16 * cq, pd);
                    const uint32_t tv[2] = {f2u(run), 0u};
                    tmem_st_x2(tm + lq + R_AT + 64 + 2 * cq, tv);
                    tmem_wait_st();
                }
                named_bar_sync(kNamedBar, RT);
                float add = 0.f;
                if (ok) {
                    uint32_t tr[8];
                    tmem_ld_x8(tm + lq + R_AT + 64, tr);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k > cq) add += u2f(tr[2 * k]);
                }
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = s < 32 * cq + i ? m[i] + add : 0.f;   // the token j of F_j
                atomicAdd(Facc + 32 * cq + lane, transpose_reduce32(v, lane));
            }
            // ------------------------------------------------ e^{b_L - b_s} on the dS' products, us_s
            float usp = 0.f;
            if (mbar_wait(bar(BINTER), par, p.status, abort_flag)) {
                tc_fence_after();
                const uint8_t* krow = sm + OFF_K + (cq >> 1) * kBox;
                uint32_t v[32];
                tmem_ld_x32(tm + lq + R_DK + 32 * cq, v);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint4 kw = *reinterpret_cast<const uint4*>(krow + sw128(s, 32 * (cq & 1) + 8 * k));
                    const uint32_t* ke = reinterpret_cast<const uint32_t*>(&kw);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = u2f(v[8 * k + 2 * e]) * ws, x1 = u2f(v[8 * k + 2 * e + 1]) * ws;
                        usp = fmaf(u2f(ke[e] << 16), x0, fmaf(u2f(ke[e] & 0xffff0000u), x1, usp));
                        v[8 * k + 2 * e] = f2u(x0);
                        v[8 * k + 2 * e + 1] = f2u(x1);
                    }
                }
                tmem_st_x32(tm + lq + R_DK + 32 * cq, v);
                tmem_ld_x32(tm + lq + R_DV + 32 * cq, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = f2u(u2f(v[j]) * ws);
                tmem_st_x32(tm + lq + R_DV + 32 * cq, v);
            }
            atomicAdd(ush + s, usp);
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(BROWS);

            // ------------------------------------------------ dv rows out, dk partial rows
            float dk[32];
            if (mbar_wait(bar(BOUT), par, p.status, abort_flag)) {
                tc_fence_after();
                // this CTA's dS' products are done: the other CTA may send into dS' lo
                if (PAIR && tid == 0) mbar_arrive_remote(cluster_map(bar(BPR), peer));
                uint32_t v[32];
                tmem_ld_x32(tm + lq + R_DV + 32 * cq, v);
                tmem_wait_ld();
                if (s < L) {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dV) +
                                                          ((tok0 + s) * p.H + hh) * DV + ch0 + 32 * cq);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        dst[k] = make_uint4(pack_bf16x2(u2f(v[8 * k]), u2f(v[8 * k + 1])),
                                            pack_bf16x2(u2f(v[8 * k + 2]), u2f(v[8 * k + 3])),
                                            pack_bf16x2(u2f(v[8 * k + 4]), u2f(v[8 * k + 5])),
                                            pack_bf16x2(u2f(v[8 * k + 6]), u2f(v[8 * k + 7])));
                }
                tmem_ld_x32(tm + lq + R_DK + 32 * cq, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) dk[j] = u2f(v[j]);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) dk[j] = 0.f;
            }
            tc_fence_before();
            named_bar_sync(kNamedBar, RT);   // F and us of this CTA are complete
            if (tid < kC) {
                float* dst = p.fus + ((size_t)item * 2 + rank) * 2 * kC;
                dst[tid] = Facc[tid];
                dst[kC + tid] = ush[tid];
            }
            // ------------------------------------------------ dk rows
            bool mine = true;
            if constexpr (PAIR) {
                // the rows of the other CTA's half go to it in one bulk copy: staged
                // in this CTA's dS' hi tile ([64 rows][128] fp32, 16-byte chunks
                // swizzled by row), received in its dS' lo tile
                float* stage = reinterpret_cast<float*>(sm + OFF_DSH);
                const float* recv = reinterpret_cast<const float*>(sm + OFF_DSL);
                const int r = s & 63;
                mine = (s >> 6) == rank;
                if (!mine)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        reinterpret_cast<float4*>(stage + r * 128)[8 * cq + (k ^ (r & 7))] =
                            make_float4(dk[4 * k], dk[4 * k + 1], dk[4 * k + 2], dk[4 * k + 3]);
                fence_proxy_async_smem();
                named_bar_sync(kNamedBar, RT);
                // the other CTA is past its dS' products: its dS' lo tile is free
                if (tid == 0 && mbar_wait_cluster(bar(BPR), par, p.status, abort_flag)) {
                    bulk_copy_to_cluster(cluster_map(sb + OFF_DSL, peer), sb + OFF_DSH, 64 * 128 * 4,
                                         cluster_map(bar(BXK), peer));
                    bulk_commit();
                }
                if (mine && mbar_wait_cluster(bar(BXK), par, p.status, abort_flag)) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float4 x = reinterpret_cast<const float4*>(recv + r * 128)[8 * cq + (k ^ (r & 7))];
                        dk[4 * k] += x.x;
                        dk[4 * k + 1] += x.y;
                        dk[4 * k + 2] += x.z;
                        dk[4 * k + 3] += x.w;
                    }
                }
                if (tid == 0) bulk_wait_read<0>();   // the staging tile is read before the next dS' loads
            }
            if (mine && s < L) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dK) +
                                                      ((tok0 + s) * p.H + hh) * kDK + 32 * cq);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    dst[k] = make_uint4(pack_bf16x2(dk[8 * k], dk[8 * k + 1]), pack_bf16x2(dk[8 * k + 2], dk[8 * k + 3]),
                                        pack_bf16x2(dk[8 * k + 4], dk[8 * k + 5]),
                                        pack_bf16x2(dk[8 * k + 6], dk[8 * k + 7]));
            }
            // the exchange tiles have been read: the issuer may load the next dS'
            warp_arrive(BXDONE);
        }
    } else {
        // ============================================================ TMA + MMA issuer (lane 0)
        constexpr uint32_t id_kk = idesc_bf16(128, 128, false, false);
        constexpr uint32_t id_kn = idesc_bf16(128, 128, false, true);
        auto kmaj = [&](uint32_t base, int k) { return sdesc_sw128(base + (k >> 2) * kBox + (k & 3) * 32, 16, 1024); };
        auto mnmaj = [&](uint32_t base, int k) { return sdesc_sw128(base + k * 2048, kBox, 1024); };
        // the tiles of chunk item (coordinates: token n0 of sequence b, head hh)
        auto coords = [&](int it, int& n0, int& b, int& hh, int& srow) {
            const int item = cid + it * ncl, u = item / nc, c = item - u * nc;
            b = u / p.H;
            hh = u - b * p.H;
            n0 = c * kC;
            srow = (u * nc + c) * kDK;
        };
        auto load_tok = [&](int it, int bi, const CUtensorMap* m0, const CUtensorMap* m1, uint32_t o0, uint32_t o1,
                            int x0) {
            int n0, b, hh, srow;
            coords(it, n0, b, hh, srow);
            mbar_arrive_expect_tx(bar(bi), (m1 ? 2 : 1) * kTile);
            for (int x = 0; x < 2; ++x) {
                tma_load_4d(sb + o0 + x * kBox, m0, x0 + x * 64, hh, n0, b, bar(bi));
                if (m1) tma_load_4d(sb + o1 + x * kBox, m1, x0 + x * 64, hh, n0, b, bar(bi));
            }
        };
        auto load_q = [&](int it) { load_tok(it, BQ, &p.tmQ, nullptr, OFF_Q, 0, 0); };
        auto load_k = [&](int it) { load_tok(it, BK, &p.tmK, nullptr, OFF_K, 0, 0); };
        auto load_v = [&](int it) { load_tok(it, BV, &p.tmV, nullptr, OFF_V, 0, ch0); };
        auto load_dy = [&](int it) { load_tok(it, BDY, &p.tmDyH, &p.tmDyL, OFF_DYH, OFF_DYL, ch0); };
        auto load_s = [&](int it) {
            int n0, b, hh, srow;
            coords(it, n0, b, hh, srow);
            mbar_arrive_expect_tx(bar(BS), 2 * kTile);
            for (int x = 0; x < 2; ++x) {
                tma_load_2d(sb + OFF_DSH + x * kBox, &p.tmSH, ch0 + x * 64, srow, bar(BS));
                tma_load_2d(sb + OFF_DSL + x * kBox, &p.tmSL, ch0 + x * 64, srow, bar(BS));
            }
        };
        auto load_bc = [&](int it) {
            mbar_arrive_expect_tx(bar(BBC), kC * 4);
            bulk_load(sb + CF::OFF_BC, p.bcg + (size_t)(cid + it * ncl) * kC, kC * 4, bar(BBC));
        };
        if (lane == 0 && niter > 0) {
            load_bc(0);
            load_q(0);
            load_k(0);
            load_v(0);
            load_dy(0);
            load_s(0);
        }
        for (int it = 0; it < niter; ++it) {
            const uint32_t par = it & 1;
            const bool more = it + 1 < niter;
            if (lane == 0) {
                bool ok = mbar_wait(bar(BQ), par, p.status, abort_flag) && mbar_wait(bar(BK), par, p.status, abort_flag);
                if (ok) {
                    tc_fence_after();
                    // A^T = K Q^T
#pragma unroll
                    for (int k = 0; k < 8; ++k) mma_ss(tm + R_AT, kmaj(sb + OFF_K, k), kmaj(sb + OFF_Q, k), id_kk, k > 0);
                }
                ok = ok && mbar_wait(bar(BV), par, p.status, abort_flag) && mbar_wait(bar(BDY), par, p.status, abort_flag);
                if (ok) {
                    tc_fence_after();
                    // D^T = V dy^T (dy as a bf16 pair)
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ss(tm + R_DT, kmaj(sb + OFF_V, k), kmaj(sb + (pass ? OFF_DYL : OFF_DYH), k), id_kk,
                                   pass > 0 || k > 0);
                }
                mma_commit(bar(BADT));
                ok = ok && mbar_wait(bar(BS), par, p.status, abort_flag);
                if (ok) {
                    tc_fence_after();
                    // V dS'^T and K dS' (dS' as a bf16 pair)
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ss(tm + R_DK, kmaj(sb + OFF_V, k), kmaj(sb + (pass ? OFF_DSL : OFF_DSH), k), id_kk,
                                   pass > 0 || k > 0);
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ss(tm + R_DV, kmaj(sb + OFF_K, k), mnmaj(sb + (pass ? OFF_DSL : OFF_DSH), k), id_kn,
                                   pass > 0 || k > 0);
                }
                mma_commit(bar(BINTER));
                // V is free once the dS' products have read it
                if (mbar_wait(bar(BINTER), par, p.status, abort_flag) && more) load_v(it + 1);
                ok = ok && mbar_wait(bar(BROWS), par, p.status, abort_flag);
                // K is free once the rows have read it (us) and the products above are done;
                // the rows have read the chunk's decay sums
                if (ok && more) {
                    load_k(it + 1);
                    load_bc(it + 1);
                }
                if (ok) {
                    tc_fence_after();
                    // dk += (D o E)^T Q, dv += (A o E)^T dy
#pragma unroll
                    for (int k = 0; k < 8; ++k) mma_ts(tm + R_DK, tm + R_DT + k * 8, mnmaj(sb + OFF_Q, k), id_kn, 1);
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tm + R_DV, tm + R_AT + k * 8, mnmaj(sb + (pass ? OFF_DYL : OFF_DYH), k), id_kn, 1);
                }
                mma_commit(bar(BOUT));
                if (mbar_wait(bar(BOUT), par, p.status, abort_flag) && more) {
                    load_q(it + 1);
                    load_dy(it + 1);
                }
            }
            __syncwarp();
            if (lane == 0) {
                // the dk exchange of this chunk has been read: the next dS' may load
                // into its buffer, and the exchange barrier is armed for the next chunk
                if (mbar_wait(bar(BXDONE), par, p.status, abort_flag) && more) {
                    if (PAIR) mbar_arrive_expect_tx(bar(BXK), 64 * 128 * 4);
                    load_s(it + 1);
                }
            }
            __syncwarp();
        }
        if (lane == 0) {
            mma_commit(bar(BDRAIN));
            mbar_wait_drain(bar(BDRAIN), 0, kWaitCycles);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();   // no CTA leaves while the other still sends to it
    if (warp == RT / 32) tmem_dealloc(tm, 512);
}

// ---- 6. per chunk, one thread per token: the gate gradient
//   dz_j = (F_j + sum_{t>=j} rr_t + X_c + sum_{s<j} us_s) (1 - sigmoid(z_j)) / tau
// from the F and us the dk/dv kernel left per channel half, the rr of the dy
// kernel and the d_v shares of X_c of the reverse scan; zero where the
// forward clamps log gamma
__global__ void __launch_bounds__(kC) bwd_dz(const __grid_constant__ BwdTcParams p) {
    __shared__ float tot[12];
    const int item = blockIdx.x, nc = p.nc, u = item / nc, c = item - u * nc, b = u / p.H, hh = u - b * p.H;
    const int n0 = c * kC, L = min(kC, p.N - n0), j = threadIdx.x, lane = j & 31, warp = j >> 5;
    const int halves = p.dv / 128, DV = p.dv;
    const size_t tk = ((size_t)b * p.N + n0 + j) * p.H + hh;
    float F = 0.f, us = 0.f, rr = 0.f, X = 0.f;
    for (int h = 0; h < halves; ++h) {
        const float* src = p.fus + ((size_t)item * 2 + h) * 2 * kC;
        F += src[j];
        us += src[kC + j];
        if (j < L) rr += p.rr[(size_t)h * p.B * p.N * p.H + tk];
    }
    for (int w = j; w < DV; w += kC) X += p.xs[((size_t)u * nc + c) * DV + w];
    X = warp_sum(X);
    // R_j = sum_{t >= j} rr_t (suffix), U_j = sum_{s < j} us_s (exclusive prefix)
    float R = rr, U = us;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float r2 = __shfl_down_sync(0xffffffffu, R, o);
        const float u2 = __shfl_up_sync(0xffffffffu, U, o);
        if (lane + o < 32) R += r2;
        if (lane >= o) U += u2;
    }
    U -= us;
    if (lane == 0) tot[warp] = R;
    if (lane == 31) tot[4 + warp] = U + us;
    if (lane == 0) tot[8 + warp] = X;
    __syncthreads();
    for (int w = warp + 1; w < 4; ++w) R += tot[w];
    for (int w = 0; w < warp; ++w) U += tot[4 + w];
    X = tot[8] + tot[9] + tot[10] + tot[11];
    if (j < L) {
        const float zj = p.z[tk];
        const float deriv = log_gamma(zj, p.inv_tau) > kMinLogGamma ? (1.f - sigmoidf_(zj)) * p.inv_tau : 0.f;
        p.dz[tk] = (F + R + X + U) * deriv;
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_bwd() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// tensor of `rank` dimensions (innermost first) of bf16 or fp32 elements,
// 128-byte swizzle
bool encode_tile(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint32_t* box,
                 bool f32) {
    EncodeTiledFn fn = encode_fn_bwd();
    if (!fn) return false;
    cuuint64_t strides[4];
    cuuint64_t st = f32 ? 4 : 2;
    for (int i = 0; i + 1 < rank; ++i) {
        st *= dims[i];
        strides[i] = st;
    }
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool encode_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint32_t* box) {
    return encode_tile(m, base, rank, dims, box, false);
}

// state-shaped fp32 rows [rows][dv], box (32, 128): 128-byte rows in the swizzle layout
bool map_state_rows_f32(CUtensorMap* m, const void* base, int dv, size_t rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)dv, (cuuint64_t)rows};
    const cuuint32_t box[2] = {32, 128};
    return encode_tile(m, base, 2, dims, box, true);
}

// [B][N][H][d] viewed as (d, H, N, B), box (64, 1, 128, 1)
bool map_tokens(CUtensorMap* m, const void* base, int d, int H, int N, int B) {
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
    return encode_bf16(m, base, 4, dims, box);
}

// per-chunk states [rows][dv] (rows = units * nc * 128), box (64, 128)
bool map_states(CUtensorMap* m, const void* base, int dv, size_t rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)dv, (cuuint64_t)rows};
    const cuuint32_t box[2] = {64, 128};
    return encode_bf16(m, base, 2, dims, box);
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdTcWs {
    size_t incg, sh, sl, dyh, dyl, rr, xs, decay, bcg, fus, total;
};

BwdTcWs bwd_tc_ws(int B, int H, int N, int dv) {
    const size_t units = (size_t)B * H, nc = (size_t)(N + kC - 1) / kC, E = (size_t)kDK * dv;
    const size_t tok = (size_t)B * N * H;
    BwdTcWs w;
    size_t o = 0;
    w.incg = o; o += a256(units * nc * E * 4);
    w.sh = o; o += a256(units * nc * E * 2);
    w.sl = o; o += a256(units * nc * E * 2);
    w.dyh = o; o += a256(tok * dv * 2);
    w.dyl = o; o += a256(tok * dv * 2);
    w.rr = o; o += a256(2 * tok * 4);
    w.xs = o; o += a256(units * nc * dv * 4);
    w.decay = o; o += a256(units * nc * 4);
    w.bcg = o; o += a256(units * nc * kC * 4);
    w.fus = o; o += a256(units * nc * 2 * 2 * kC * 4);
    w.total = o;
    return w;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kernel)(KArgs...), unsigned grid, int cluster, size_t smem, cudaStream_t s,
                           int threads, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cluster > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int DV>
cudaError_t run_bwd_tc(BwdTcParams& p, cudaStream_t s) {
    constexpr bool PAIR = DV == 256;
    const unsigned items = (unsigned)((size_t)p.B * p.H * p.nc);
    auto k1 = bwd_inc_tc;
    auto k3 = bwd_dyq_tc<PAIR>;
    auto k5 = bwd_kv_tc<PAIR>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, IncCfg::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, GradCfg::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k5, cudaFuncAttributeMaxDynamicSharedMemorySize, GradCfg::SMEM)) != cudaSuccess)
        return e;
    const dim3 sgrid((unsigned)((kDK * DV / 4 + kScanThreads - 1) / kScanThreads), (unsigned)(p.B * p.H));
    k1<<<items * (DV / 128), kThreads, IncCfg::SMEM, s>>>(p);
    bwd_scan_fwd<<<sgrid, kScanThreads, 0, s>>>(p);
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // the two gradient kernels are persistent: one CTA (pair) per SM (pair of SMs)
    const unsigned ncl = std::min<unsigned>(items, (unsigned)std::max(1, PAIR ? sms / 2 : sms));
    if ((e = launch_cluster(k3, ncl * (PAIR ? 2 : 1), PAIR ? 2 : 1, GradCfg::SMEM, s, kThreads16, p)) !=
        cudaSuccess)
        return e;
    bwd_scan_rev<<<sgrid, kScanThreads, 0, s>>>(p);
    if ((e = launch_cluster(k5, ncl * (PAIR ? 2 : 1), PAIR ? 2 : 1, GradCfg::SMEM, s, kThreads16, p)) !=
        cudaSuccess)
        return e;
    bwd_dz<<<items, kC, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool bwd_tc_supported(int B, int H, int N, int dk, int dv, gret_dtype io) {
    if (io != GRET_BF16 || dk != kDK || (dv != 128 && dv != 256) || B <= 0 || H <= 0 || N <= 0) return false;
    const long long items = (long long)B * H * ((N + kC - 1) / kC);
    // the per-chunk state rows address a 2-D tensor map (rows < 2^31) and
    // the grids one CTA (pair) per chunk
    return items * kDK < (1LL << 31) && items * 2 < (1LL << 31);
}

size_t bwd_tc_workspace_bytes(int B, int H, int N, int dv) { return bwd_tc_ws(B, H, N, dv).total; }

cudaError_t launch_bwd_tc(const BackwardArgs& in, cudaStream_t s) {
    BwdTcParams p;
    std::memset(&p, 0, sizeof(p));
    p.Q = in.Q; p.K = in.K; p.V = in.V; p.G = in.G; p.dO = in.dO;
    p.z = in.z; p.S0 = in.S0; p.dS_final = in.dS_final;
    p.dQ = in.dQ; p.dK = in.dK; p.dV = in.dV; p.dG = in.dG; p.dz = in.dz; p.dS0 = in.dS0;
    p.status = in.status;
    p.B = in.B; p.H = in.H; p.N = in.N; p.dv = in.dv; p.nc = (in.N + kC - 1) / kC;
    p.inv_tau = in.inv_tau; p.eps = in.eps; p.gn = in.gn;
    const BwdTcWs w = bwd_tc_ws(in.B, in.H, in.N, in.dv);
    uint8_t* ws = static_cast<uint8_t*>(in.workspace);
    p.incg = reinterpret_cast<float*>(ws + w.incg);
    p.sh = reinterpret_cast<__nv_bfloat16*>(ws + w.sh);
    p.sl = reinterpret_cast<__nv_bfloat16*>(ws + w.sl);
    p.dyh = reinterpret_cast<__nv_bfloat16*>(ws + w.dyh);
    p.dyl = reinterpret_cast<__nv_bfloat16*>(ws + w.dyl);
    p.rr = reinterpret_cast<float*>(ws + w.rr);
    p.xs = reinterpret_cast<float*>(ws + w.xs);
    p.decay = reinterpret_cast<float*>(ws + w.decay);
    p.bcg = reinterpret_cast<float*>(ws + w.bcg);
    p.fus = reinterpret_cast<float*>(ws + w.fus);
    const size_t srows = (size_t)in.B * in.H * p.nc * kDK;
    if (!map_tokens(&p.tmQ, in.Q, kDK, in.H, in.N, in.B) || !map_tokens(&p.tmK, in.K, kDK, in.H, in.N, in.B) ||
        !map_tokens(&p.tmV, in.V, in.dv, in.H, in.N, in.B) || !map_tokens(&p.tmDyH, p.dyh, in.dv, in.H, in.N, in.B) ||
        !map_tokens(&p.tmDyL, p.dyl, in.dv, in.H, in.N, in.B) || !map_states(&p.tmSH, p.sh, in.dv, srows) ||
        !map_states(&p.tmSL, p.sl, in.dv, srows) || !map_state_rows_f32(&p.tmInc, p.incg, in.dv, srows))
        return cudaErrorInvalidValue;
    return in.dv == 256 ? run_bwd_tc<256>(p, s) : run_bwd_tc<128>(p, s);
}

}  // namespace gret
