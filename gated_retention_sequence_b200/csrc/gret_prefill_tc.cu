// Tensor-core chunkwise prefill of the gated-retention mixer for sm_100a.
//
// Method ("YOCO 深度技术分析", sections 2.2 and 5.3.2; the chunk state R_i and
// the decay summary "beta" of the "分段递归表示" paragraph of the
// Medium-article translation).  Per (batch, head) unit and chunk of C tokens,
// with b_t the chunk-local cumulative log-decay (b_C the chunk total):
//   A      = Q_c K_c^T                                 (C x C, over d_k)
//   P[t,s] = A[t,s] e^{b_t - b_s} for s <= t, else 0
//   O_c    = P V_c + diag(e^{b_t}) Q_c S_prev           (C x d_v)
//   S      = e^{b_C} S_prev + (diag(e^{b_C - b_s}) K_c)^T V_c
//   out    = GroupNorm(O_c) (.) swish(G_c)
// All exponents are <= 0.
//
// B200 mapping.  Every product runs as a 128-row tcgen05.mma (bf16 operands,
// fp32 accumulation in tensor memory):
//   scores   D[t][s]          = Q K^T        A = Q (smem, K-major), B = K (K-major)
//   output   D[d][t] = O^T    = V^T P^T      A = V (smem, MN-major), B = P (K-major)
//                            + S^T Q~^T     A = bf16 copy of S^T (TMEM), B = Q~ (K-major)
//   state    D[d][k] = S^T   += V^T K~      A = V (MN-major), B = K~ (MN-major)
// so d_v (128 per half) is the MMA's M dimension and the chunk is its N
// dimension; a 64-token chunk needs no padding except in the small scores
// product.  S^T stays in fp32 tensor memory for the whole segment; once per
// chunk the compute warps read it, write a bf16 copy (the A operand of the
// inter-chunk product) and scale it by e^{b_C} in place before the state MMA
// accumulates.  Q, K and V tiles arrive by TMA (128-byte swizzle) into a
// 1-2 stage ring; G arrives into a 2-stage ring and the normalised output is
// written over it and stored by TMA.  Warp 8 issues the loads, thread 0 the
// MMAs; eight warps do the decay, the bf16 conversions and the epilogue.
//
// Parallelism.  A unit is split into P sequence segments (the chunkwise form
// applied to segments): a first pass computes each segment's state increment
// dS_p and total log-decay a_p from K, V and the gate alone; a combine pass
// folds them into each segment's initial state,
//   S_in(p+1) = e^{a_p} S_in(p) + dS_p,
// and the fused pass runs every segment from its S_in.  This is the state
// decomposition S(x || y) = e^{sum log gamma(y)} S(x) + S(y from 0).
#include <cuda.h>

#include <cstring>

#include "gret_common.cuh"
#include "gret_sm100.cuh"

namespace gret {
namespace {

using namespace sm100;

constexpr int DK = 128;
constexpr int kCW = 8;                  // compute warps
constexpr int kCT = kCW * 32;           // compute threads
constexpr int kThreadsTC = kCT + 32;    // + one producer warp

template <int DV, int C>
struct Cfg {
    static constexpr int NH = DV / 128;                     // d_v halves (MMA M = 128 each)
    static constexpr int NS = (DV == 128 && C == 128) ? 1 : 2;  // Q/K/V stages
    static constexpr int NG = 2;                            // G/O stages
    static constexpr int ROWB = 128;                        // bytes per swizzled row
    static constexpr int BOX = C * ROWB;                    // one [C x 64] bf16 box
    static constexpr int Q_BYTES = 2 * BOX;                 // d_k = 128 -> 2 boxes
    static constexpr int K_BYTES = 2 * BOX;
    static constexpr int V_BYTES = (DV / 64) * BOX;
    static constexpr int G_BYTES = (DV / 64) * BOX;
    static constexpr int P_BYTES = (C / 64) * BOX;          // rows t, C bf16 of s
    static constexpr int HT = C / 2;                        // tokens per thread, epilogue
    // tensor-memory columns
    static constexpr int TM_S = 0;                          // S^T: NH x 128 fp32 columns
    static constexpr int TM_O = NH * 128;                   // O^T: NH x C
    static constexpr int TM_X = NH * 128 + NH * C;          // scores (C) / bf16 S^T (NH x 64)
    static constexpr int X_COLS = (C > NH * 64) ? C : NH * 64;
    static constexpr int TM_USED = TM_X + X_COLS;
    static constexpr int TM_ALLOC = TM_USED <= 256 ? 256 : 512;
    // shared-memory layout (bytes from a 1024-aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + NS * Q_BYTES;
    static constexpr int OFF_V = OFF_K + NS * K_BYTES;
    static constexpr int OFF_G = OFF_V + NS * V_BYTES;
    static constexpr int OFF_P = OFF_G + NG * G_BYTES;
    static constexpr int OFF_B = OFF_P + P_BYTES;           // NS x C fp32 decay sums
    static constexpr int OFF_RED = OFF_B + NS * C * 4;      // kCW x HT x 2 fp32
    static constexpr int OFF_STAT = OFF_RED + kCW * HT * 2 * 4;   // C x (rstd, -mean * rstd)
    static constexpr int OFF_BAR = OFF_STAT + C * 8;
    static constexpr int NUM_BARS = 2 * NS + 2 * NG + 2;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;      // + alignment slack
    static_assert(TM_USED <= 512, "tensor memory budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(C % 32 == 0 && C <= 128, "chunk");
    // the padded rows (C..127) of the 128-row scores A operand must stay in
    // the allocation: they read the bytes after the last Q stage's boxes.
    static_assert(OFF_K + 2 * (128 - C) * ROWB <= SMEM, "scores padding rows");
};

struct TcParams {
    CUtensorMap tmQ, tmK, tmV, tmG, tmO;
    const float* bcum;       // [units][Npad] chunk-local cumulative log-decay
    float* seg_state;        // [units][P-1][DV][DK]  (S^T, fp32)
    float* seg_decay;        // [units][P-1]
    float* S_final;          // [units][DK][DV] or null
    unsigned int* status;
    int H, N, Npad, P, seg_len;
    float eps;
    int gn;                  // 1: GroupNorm + swish; 0: O = Y
    int has_g;
};

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }

// Scale the 8 bf16 values of one 16-byte shared-memory word by f.
__device__ __forceinline__ void scale_bf16x8(uint8_t* p, float f) {
    uint4 w = *reinterpret_cast<uint4*>(p);
    uint32_t* e = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&e[j]);
        float2 x = __bfloat1622float2(v);
        e[j] = pack_bf16x2(x.x * f, x.y * f);
    }
    *reinterpret_cast<uint4*>(p) = w;
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 16) tmem_ld_x16(taddr, r);
    else if constexpr (N == 32) tmem_ld_x32(taddr, r);
    else tmem_ld_x64(taddr, r);
}

// Sum each of the N values of a lane over the 32 lanes of the warp; on return
// v[j], j < N / 32, holds the total for value index lane * (N / 32) + j.
template <int N>
__device__ __forceinline__ void warp_transpose_sum(float (&v)[N], int lane) {
#pragma unroll
    for (int off = 16, n = N / 2; off >= 1; off >>= 1, n >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int j = 0; j < n; ++j) {
            float send = up ? v[j] : v[j + n];
            float keep = up ? v[j + n] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
}

template <int DV, int C, bool kFull>
__global__ void __launch_bounds__(kThreadsTC, 1) prefill_tc_kernel(const __grid_constant__ TcParams p) {
    using CF = Cfg<DV, C>;
    constexpr int NS = CF::NS, NG = CF::NG, NH = CF::NH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int nseg = kFull ? p.P : p.P - 1;
    const int u = blockIdx.x / nseg, seg = blockIdx.x % nseg;
    const int bb = u / p.H, hh = u % p.H;
    const int n_begin = seg * p.seg_len;
    const int n_end = min(p.N, n_begin + p.seg_len);
    const int nchunks = (n_end - n_begin + C - 1) / C;

    const int BF = 0, BE = NS, BGF = 2 * NS, BGE = 2 * NS + NG, BSC = 2 * NS + 2 * NG, BMMA = BSC + 1;
    auto bar = [&](int i) -> uint32_t { return sb + CF::OFF_BAR + 8 * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);

    if (tid == 0) {
        for (int i = 0; i < CF::NUM_BARS; ++i) mbar_init(bar(i), 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tmK);
        tma_prefetch_desc(&p.tmV);
        if (kFull) {
            tma_prefetch_desc(&p.tmQ);
            tma_prefetch_desc(&p.tmG);
            tma_prefetch_desc(&p.tmO);
        }
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), CF::TM_ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;

    if (warp == kCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int iq = 0, ig = (kFull && p.has_g) ? 0 : nchunks;
            while (iq < nchunks || ig < nchunks) {
                const bool do_q = iq < nchunks && (ig >= nchunks || iq <= ig + (NS - 1));
                if (do_q) {
                    const int s = iq % NS;
                    if (!mbar_wait(bar(BE + s), ((iq / NS) & 1) ^ 1, p.status, abort_flag)) break;
                    const int n0 = n_begin + iq * C;
                    const uint32_t bytes = CF::K_BYTES + CF::V_BYTES + C * 4 + (kFull ? CF::Q_BYTES : 0);
                    const uint32_t fb = bar(BF + s);
                    mbar_arrive_expect_tx(fb, bytes);
                    if (kFull) {
                        for (int j = 0; j < 2; ++j)
                            tma_load_4d(sb + CF::OFF_Q + s * CF::Q_BYTES + j * CF::BOX, &p.tmQ, j * 64, hh, n0, bb, fb);
                    }
                    for (int j = 0; j < 2; ++j)
                        tma_load_4d(sb + CF::OFF_K + s * CF::K_BYTES + j * CF::BOX, &p.tmK, j * 64, hh, n0, bb, fb);
                    for (int j = 0; j < DV / 64; ++j)
                        tma_load_4d(sb + CF::OFF_V + s * CF::V_BYTES + j * CF::BOX, &p.tmV, j * 64, hh, n0, bb, fb);
                    bulk_load(sb + CF::OFF_B + s * C * 4, p.bcum + (size_t)u * p.Npad + n0, C * 4, fb);
                    ++iq;
                } else {
                    const int g = ig % NG;
                    if (!mbar_wait(bar(BGE + g), ((ig / NG) & 1) ^ 1, p.status, abort_flag)) break;
                    const int n0 = n_begin + ig * C;
                    const uint32_t gb = bar(BGF + g);
                    mbar_arrive_expect_tx(gb, CF::G_BYTES);
                    for (int j = 0; j < DV / 64; ++j)
                        tma_load_4d(sb + CF::OFF_G + g * CF::G_BYTES + j * CF::BOX, &p.tmG, j * 64, hh, n0, bb, gb);
                    ++ig;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ compute warps
        const int q4 = warp & 3;       // tensor-memory lane quarter of this warp
        const int grp = warp >> 2;     // which of the two warps sharing the quarter
        const uint32_t lq = (uint32_t)(32 * q4) << 16;

        // Initial state S^T: zero, or the segment's S_in.
        {
            const float* src = nullptr;
            if (kFull && seg > 0) src = p.seg_state + ((size_t)u * (p.P - 1) + (seg - 1)) * DV * DK;
#pragma unroll
            for (int cb = 0; cb < (NH == 2 ? 2 : 1); ++cb) {
                const int half = NH == 2 ? grp : 0;
                const int k0 = NH == 2 ? cb * 64 : grp * 64;
                const int d = half * 128 + q4 * 32 + lane;
                uint32_t r[64];
                if (src) {
                    const float4* s4 = reinterpret_cast<const float4*>(src + (size_t)d * DK + k0);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float4 v = s4[j];
                        r[4 * j] = f2u(v.x); r[4 * j + 1] = f2u(v.y); r[4 * j + 2] = f2u(v.z); r[4 * j + 3] = f2u(v.w);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) r[j] = 0u;
                }
                tmem_st_x64(tm + lq + CF::TM_S + half * 128 + k0, r);
            }
            tmem_wait_st();
        }

        float seg_decay = 0.f;
        for (int i = 0; i < nchunks; ++i) {
            const int s = i % NS;
            const uint32_t sQ = sb + CF::OFF_Q + s * CF::Q_BYTES;
            const uint32_t sK = sb + CF::OFF_K + s * CF::K_BYTES;
            const uint32_t sV = sb + CF::OFF_V + s * CF::V_BYTES;
            const float* bc = reinterpret_cast<const float*>(sm + CF::OFF_B + s * C * 4);
            mbar_wait(bar(BF + s), (i / NS) & 1, p.status, abort_flag);
            const float bC = bc[C - 1];

            if (kFull) {
                // scores D[t][s] = Q K^T over d_k (M = 128 rows of t; rows >= C unused)
                if (tid == 0) {
                    tc_fence_after();
                    constexpr uint32_t id = idesc_bf16(128, C, false, false);
#pragma unroll
                    for (int k = 0; k < DK / 16; ++k) {
                        const uint32_t off = (k >> 2) * CF::BOX + (k & 3) * 32;
                        mma_ss(tm + CF::TM_X, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), id,
                               k > 0);
                    }
                    mma_commit(bar(BSC));
                }
                mbar_wait(bar(BSC), i & 1, p.status, abort_flag);
                tc_fence_after();
                // P[t][s] = A[t][s] e^{b_t - b_s} (s <= t) -> bf16, K-major rows t
                if (q4 * 32 < C) {
                    constexpr int HC = C / 2;
                    const int t = q4 * 32 + lane;
                    uint32_t r[HC];
                    tmem_ld<HC>(tm + lq + CF::TM_X + grp * HC, r);
                    tmem_wait_ld();
                    const float bt = bc[t];
#pragma unroll
                    for (int c8 = 0; c8 < HC / 8; ++c8) {
                        const int s0 = grp * HC + c8 * 8;
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int sa = s0 + 2 * e, sb2 = sa + 1;
                            const float v0 = sa <= t ? u2f(r[c8 * 8 + 2 * e]) * __expf(bt - bc[sa]) : 0.f;
                            const float v1 = sb2 <= t ? u2f(r[c8 * 8 + 2 * e + 1]) * __expf(bt - bc[sb2]) : 0.f;
                            w[e] = pack_bf16x2(v0, v1);
                        }
                        const int region = s0 >> 6, chunk = (s0 & 63) >> 3;
                        uint8_t* dst = sm + CF::OFF_P + region * CF::BOX + t * 128 + ((chunk ^ (t & 7)) << 4);
                        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            // K~ = diag(e^{b_C - b_s}) K and Q~ = diag(e^{b_t}) Q, in place.
            {
                uint8_t* Kp = sm + CF::OFF_K + s * CF::K_BYTES;
                for (int ci = tid; ci < C * 16; ci += kCT) {
                    const int row = (ci >> 3) % C;
                    scale_bf16x8(Kp + ci * 16, __expf(bC - bc[row]));
                }
                if (kFull) {
                    uint8_t* Qp = sm + CF::OFF_Q + s * CF::Q_BYTES;
                    for (int ci = tid; ci < C * 16; ci += kCT) {
                        const int row = (ci >> 3) % C;
                        scale_bf16x8(Qp + ci * 16, __expf(bc[row]));
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(1, kCT);   // every read of the scores is done
            tc_fence_after();
            // bf16 copy of S^T (A operand of the inter-chunk product), then S^T *= e^{b_C}
            {
                const float eC = __expf(bC);
#pragma unroll
                for (int cb = 0; cb < (NH == 2 ? 2 : 1); ++cb) {
                    const int half = NH == 2 ? grp : 0;
                    const int k0 = NH == 2 ? cb * 64 : grp * 64;
                    uint32_t r[64];
                    tmem_ld_x64(tm + lq + CF::TM_S + half * 128 + k0, r);
                    tmem_wait_ld();
                    if (kFull) {
                        uint32_t pk[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(u2f(r[2 * j]), u2f(r[2 * j + 1]));
                        tmem_st_x32(tm + lq + CF::TM_X + half * 64 + k0 / 2, pk);
                    }
#pragma unroll
                    for (int j = 0; j < 64; ++j) r[j] = f2u(u2f(r[j]) * eC);
                    tmem_st_x64(tm + lq + CF::TM_S + half * 128 + k0, r);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, kCT);
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const uint32_t vA = sV + 2 * h * CF::BOX;   // d_v rows h*128 .. +127 (two boxes)
                    if (kFull) {
                        constexpr uint32_t id_pv = idesc_bf16(128, C, true, false);
#pragma unroll
                        for (int k = 0; k < C / 16; ++k) {
                            const uint32_t poff = (k >> 2) * CF::BOX + (k & 3) * 32;
                            mma_ss(tm + CF::TM_O + h * C, sdesc_sw128(vA + k * 2048, CF::BOX, 1024),
                                   sdesc_sw128(sb + CF::OFF_P + poff, 16, 1024), id_pv, k > 0);
                        }
                        constexpr uint32_t id_qs = idesc_bf16(128, C, false, false);
#pragma unroll
                        for (int k = 0; k < DK / 16; ++k) {
                            const uint32_t qoff = (k >> 2) * CF::BOX + (k & 3) * 32;
                            mma_ts(tm + CF::TM_O + h * C, tm + CF::TM_X + h * 64 + k * 8,
                                   sdesc_sw128(sQ + qoff, 16, 1024), id_qs, 1);
                        }
                    }
                    constexpr uint32_t id_kv = idesc_bf16(128, DK, true, true);
#pragma unroll
                    for (int k = 0; k < C / 16; ++k) {
                        mma_ss(tm + CF::TM_S + h * 128, sdesc_sw128(vA + k * 2048, CF::BOX, 1024),
                               sdesc_sw128(sK + k * 2048, CF::BOX, 1024), id_kv, 1);
                    }
                }
                mma_commit(bar(BMMA));
                mma_commit(bar(BE + s));   // frees this Q/K/V stage for the producer
            }
            seg_decay += bC;
            mbar_wait(bar(BMMA), i & 1, p.status, abort_flag);
            tc_fence_after();

            if (kFull) {
                // ---------------------------------------------------- epilogue
                // Thread (q4, grp, lane) owns d_v channels h*128 + q4*32 + lane
                // (h < NH) for tokens grp*HT .. grp*HT + HT - 1.
                constexpr int HT = CF::HT;
                const int g = i % NG;
                if (p.has_g) mbar_wait(bar(BGF + g), (i / NG) & 1, p.status, abort_flag);
                uint8_t* Gp = sm + CF::OFF_G + g * CF::G_BYTES;
                const int t0 = grp * HT;
                const uint32_t oaddr = tm + lq + CF::TM_O + t0;
                float* red = reinterpret_cast<float*>(sm + CF::OFF_RED);
                float2* stat = reinterpret_cast<float2*>(sm + CF::OFF_STAT);
                if (p.gn) {
                    // per-token sums over this thread's channels, then over the
                    // warp's lanes, then over the four lane quarters
#pragma unroll
                    for (int pass = 0; pass < 2; ++pass) {
                        float v[HT];
#pragma unroll
                        for (int h = 0; h < NH; ++h) {
                            uint32_t r[HT];
                            tmem_ld<HT>(oaddr + h * C, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < HT; ++j) {
                                const float y = u2f(r[j]);
                                const float x = pass == 0 ? y : y * y;
                                v[j] = h == 0 ? x : v[j] + x;
                            }
                        }
                        warp_transpose_sum<HT>(v, lane);
#pragma unroll
                        for (int j = 0; j < HT / 32; ++j) red[(warp * HT + lane * (HT / 32) + j) * 2 + pass] = v[j];
                    }
                    named_bar_sync(1, kCT);
                    if (tid < C) {
                        const int gg = tid / HT, tl = tid % HT;
                        float s1 = 0.f, s2 = 0.f;
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            s1 += red[((gg * 4 + qq) * HT + tl) * 2];
                            s2 += red[((gg * 4 + qq) * HT + tl) * 2 + 1];
                        }
                        const float mean = s1 * (1.0f / DV);
                        const float var = fmaxf(s2 * (1.0f / DV) - mean * mean, 0.f);
                        const float rstd = rsqrtf(var + p.eps);
                        stat[tid] = make_float2(rstd, -mean * rstd);
                    }
                    named_bar_sync(1, kCT);
                }
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    uint32_t r[HT];
                    tmem_ld<HT>(oaddr + h * C, r);
                    tmem_wait_ld();
                    const int d = h * 128 + q4 * 32 + lane;
                    const int dj = d >> 6, dc = (d & 63) >> 3, de = (d & 7) * 2;
                    uint8_t* gcol = Gp + dj * CF::BOX + de;
#pragma unroll
                    for (int j = 0; j < HT; ++j) {
                        const int t = t0 + j;
                        __nv_bfloat16* gp = reinterpret_cast<__nv_bfloat16*>(gcol + t * 128 + ((dc ^ (t & 7)) << 4));
                        float o = u2f(r[j]);
                        if (p.gn) {
                            const float2 st = stat[t];
                            const float gv = __bfloat162float(*gp);
                            // GroupNorm as one FMA, then swish(g) = g * sigmoid(g)
                            o = fmaf(o, st.x, st.y) * __fdividef(gv, 1.0f + __expf(-gv));
                        }
                        *gp = __float2bfloat16_rn(o);
                    }
                }
                tc_fence_before();
                fence_proxy_async_smem();
                named_bar_sync(1, kCT);
                if (tid == 0) {
                    const int n0 = n_begin + i * C;
                    for (int j = 0; j < DV / 64; ++j)
                        tma_store_4d(&p.tmO, smem_u32(Gp + j * CF::BOX), j * 64, hh, n0, bb);
                    bulk_commit();
                    bulk_wait_read<1>();   // the store issued one chunk ago has read its buffer
                    if (i >= 1 && p.has_g) mbar_arrive(bar(BGE + (i - 1) % NG));
                }
            }
        }

        // ---------------------------------------------------------------- state out
        if (kFull) {
            if (tid == 0) bulk_wait<0>();
            if (p.S_final && seg == p.P - 1) {
                float* dst = p.S_final + (size_t)u * DK * DV;
#pragma unroll
                for (int cb = 0; cb < (NH == 2 ? 2 : 1); ++cb) {
                    const int half = NH == 2 ? grp : 0;
                    const int k0 = NH == 2 ? cb * 64 : grp * 64;
                    const int d = half * 128 + q4 * 32 + lane;
                    uint32_t r[64];
                    tmem_ld_x64(tm + lq + CF::TM_S + half * 128 + k0, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 64; ++j) dst[(size_t)(k0 + j) * DV + d] = u2f(r[j]);
                }
            }
        } else {
            float* dst = p.seg_state + ((size_t)u * (p.P - 1) + seg) * DV * DK;
#pragma unroll
            for (int cb = 0; cb < (NH == 2 ? 2 : 1); ++cb) {
                const int half = NH == 2 ? grp : 0;
                const int k0 = NH == 2 ? cb * 64 : grp * 64;
                const int d = half * 128 + q4 * 32 + lane;
                uint32_t r[64];
                tmem_ld_x64(tm + lq + CF::TM_S + half * 128 + k0, r);
                tmem_wait_ld();
                float4* d4 = reinterpret_cast<float4*>(dst + (size_t)d * DK + k0);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    d4[j] = make_float4(u2f(r[4 * j]), u2f(r[4 * j + 1]), u2f(r[4 * j + 2]), u2f(r[4 * j + 3]));
            }
            if (tid == 0) p.seg_decay[(size_t)u * (p.P - 1) + seg] = seg_decay;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, CF::TM_ALLOC);
    }
}

// Chunk-local inclusive sums of log gamma: bcum[u][n] = sum_{j in chunk, j <= n} lg_j.
// Padding tokens (n >= N) carry lg = 0, so they repeat the chunk total.
__global__ void gate_scan_kernel(const float* __restrict__ z, float* __restrict__ bcum, int H, int N,
                                 int Npad, float inv_tau) {
    __shared__ float wsum[4];
    const int C = blockDim.x;
    const int u = blockIdx.x, b = u / H, h = u % H;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int n = blockIdx.y * C + t;
    float x = n < N ? log_gamma(z[((size_t)b * N + n) * H + h], inv_tau) : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    for (int j = 0; j < w; ++j) x += wsum[j];
    bcum[(size_t)u * Npad + n] = x;
}

// Fold the segment increments into initial states, in place:
// slot p <- S_in(p + 1) = e^{a_p} S_in(p) + dS_p, with S_in(0) = 0.
__global__ void seg_combine_kernel(float* __restrict__ seg_state, const float* __restrict__ seg_decay, int P,
                                   int elems4) {
    const int u = blockIdx.y;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= elems4) return;
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < P - 1; ++p) {
        float4* slot = reinterpret_cast<float4*>(seg_state) + ((size_t)u * (P - 1) + p) * elems4 + e;
        const float f = __expf(seg_decay[(size_t)u * (P - 1) + p]);
        const float4 d = *slot;
        run = make_float4(fmaf(f, run.x, d.x), fmaf(f, run.y, d.y), fmaf(f, run.z, d.z), fmaf(f, run.w, d.w));
        *slot = run;
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// [B][N][H][d] bf16 viewed as a 4-D tensor (d, H, N, B); box (64, 1, C, 1).
bool make_map(CUtensorMap* m, const void* base, int d, int H, int N, int B, int C) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N * H * d * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    size_t bcum, state, decay, total;
};

WsLayout ws_layout(int B, int H, int N, int dk, int dv, int chunk, int segments) {
    const size_t units = (size_t)B * H;
    const size_t npad = (size_t)((N + chunk - 1) / chunk) * chunk;
    WsLayout w;
    w.bcum = 0;
    w.state = align256(units * npad * 4);
    w.decay = w.state + align256(segments > 1 ? units * (segments - 1) * (size_t)dk * dv * 4 : 0);
    w.total = w.decay + align256(segments > 1 ? units * (segments - 1) * 4 : 0);
    return w;
}

template <int DV, int C>
cudaError_t run_tc(const PrefillArgs& a, TcParams& tp, cudaStream_t s) {
    using CF = Cfg<DV, C>;
    auto kf = prefill_tc_kernel<DV, C, true>;
    auto ks = prefill_tc_kernel<DV, C, false>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM);
        cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM);
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    const int units = a.B * a.H;
    const int npad = tp.Npad;
    gate_scan_kernel<<<dim3(units, npad / C), C, 0, s>>>(a.z, const_cast<float*>(tp.bcum), a.H, a.N, npad,
                                                         a.inv_tau);
    if (tp.P > 1) {
        ks<<<units * (tp.P - 1), kThreadsTC, CF::SMEM, s>>>(tp);
        const int elems4 = DV * DK / 4;
        seg_combine_kernel<<<dim3((elems4 + 255) / 256, units), 256, 0, s>>>(tp.seg_state, tp.seg_decay, tp.P,
                                                                             elems4);
    }
    if (g_profile_start) cudaEventRecord(g_profile_start, s);
    kf<<<units * tp.P, kThreadsTC, CF::SMEM, s>>>(tp);
    if (g_profile_stop) cudaEventRecord(g_profile_stop, s);
    return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supported(int dk, int dv, int chunk, gret_dtype io) {
    if (io != GRET_BF16 || dk != DK) return false;
    return (dv == 128 && (chunk == 64 || chunk == 128)) || (dv == 256 && chunk == 64);
}

void prefill_tc_plan(int B, int H, int N, int chunk, int num_sms, int* segments, int* seg_len) {
    const int units = B * H;
    const int nchunks = (N + chunk - 1) / chunk;
    int P = num_sms / (units > 0 ? units : 1);
    if (P < 1) P = 1;
    if (P > nchunks) P = nchunks;
    const int per = (nchunks + P - 1) / P;
    *seg_len = per * chunk;
    *segments = (nchunks + per - 1) / per;
}

size_t prefill_tc_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk, int segments) {
    return ws_layout(B, H, N, dk, dv, chunk, segments).total;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
    TcParams tp;
    memset(&tp, 0, sizeof(tp));
    const int C = a.chunk;
    if (!make_map(&tp.tmQ, a.Q, DK, a.H, a.N, a.B, C) || !make_map(&tp.tmK, a.K, DK, a.H, a.N, a.B, C) ||
        !make_map(&tp.tmV, a.V, a.dv, a.H, a.N, a.B, C) || !make_map(&tp.tmO, a.O, a.dv, a.H, a.N, a.B, C) ||
        !make_map(&tp.tmG, a.G ? a.G : a.O, a.dv, a.H, a.N, a.B, C))
        return cudaErrorInvalidValue;
    const WsLayout w = ws_layout(a.B, a.H, a.N, a.dk, a.dv, C, a.segments);
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    tp.bcum = reinterpret_cast<const float*>(ws + w.bcum);
    tp.seg_state = reinterpret_cast<float*>(ws + w.state);
    tp.seg_decay = reinterpret_cast<float*>(ws + w.decay);
    tp.S_final = a.S_final;
    tp.status = a.status;
    tp.H = a.H;
    tp.N = a.N;
    tp.Npad = (a.N + C - 1) / C * C;
    tp.P = a.segments;
    tp.seg_len = a.seg_len;
    tp.eps = a.eps;
    tp.gn = a.epi == GRET_EPI_GN_SWISH ? 1 : 0;
    tp.has_g = (a.epi == GRET_EPI_GN_SWISH && a.G) ? 1 : 0;
    if (a.dv == 256 && C == 64) return run_tc<256, 64>(a, tp, s);
    if (a.dv == 128 && C == 128) return run_tc<128, 128>(a, tp, s);
    if (a.dv == 128 && C == 64) return run_tc<128, 64>(a, tp, s);
    return cudaErrorNotSupported;
}

}  // namespace gret
