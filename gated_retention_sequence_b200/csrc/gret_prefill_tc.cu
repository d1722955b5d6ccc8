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
// B200 mapping.  Every product runs as a 128-row tcgen05.mma with fp32
// accumulation in tensor memory:
//   scores   D[t][s]          = Q K^T        A = Q (smem, K-major), B = K (K-major)
//   output   D[d][t] = O^T    = T^T Q~^T     A = T^T in TMEM (tf32; 64-token chunks)
//                                            or its bf16 copy (128-token chunks), B = Q~
//                            + V^T P^T      A = V (smem, MN-major), B = P (K-major)
//   state    D[d][k] = T^T   += V^T K~      A = V (MN-major), B = K~ (MN-major)
// so d_v (128 per half) is the MMA's M dimension and the chunk is its N
// dimension.  The state lives in tensor memory for a whole segment as
// T = S / e^Lambda, rescaled only when the decay since the last rescale grows
// past e^kLazyMax ("lazy" scaling).  Q, K, V and G tiles arrive by TMA
// (128-byte swizzle); the normalised output is written over the G tile and
// stored by TMA.  One warp issues the MMAs, one the TMA traffic, and sixteen
// compute the decays, P, Q~, K~ and the GroupNorm * swish epilogue; with
// 64-token chunks they prepare chunk i + 1 before finishing chunk i (see
// prefill_tc_kernel).
//
// Parallelism.  A unit is split into P sequence segments (the chunkwise form
// applied to segments): a first pass computes each segment's state increment
// dS_p and total log-decay a_p from K, V and the gate alone; a combine pass
// folds them into each segment's initial state,
//   S_in(p+1) = e^{a_p} S_in(p) + dS_p,
// and the fused pass runs every segment from its S_in.  This is the state
// decomposition S(x || y) = e^{sum log gamma(y)} S(x) + S(y from 0).
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <type_traits>
#include <utility>

#include "gret_common.cuh"
#include "gret_sm100.cuh"

namespace gret {
namespace {

using namespace sm100;

constexpr int DK = 128;
constexpr int kCW = 16;                 // compute warps: four per tensor-memory lane quarter
constexpr int kCT = kCW * 32;           // compute threads per fused CTA
constexpr int kFusedThreads = kCT + 128; // + a warpgroup: an MMA-issuing warp, a TMA warp, two idle
// Register split of the fused kernel: it is launched with 96 registers a
// thread (65536 / 640, rounded down to 8); the issuing warpgroup gives up all
// but kIssueRegs and the four compute warpgroups take kComputeRegs.
constexpr int kLaunchRegs = 96;
constexpr int kIssueRegs = 64;
constexpr int kComputeRegs = 104;
static_assert(4 * 128 * kComputeRegs + 128 * kIssueRegs <= kFusedThreads * kLaunchRegs, "register split");
constexpr float kLazyMax = 64.0f;       // largest exponent the lazy state scale may reach
constexpr int kMaxSmem = 227 * 1024;    // dynamic shared memory per block

template <int DV, int C>
struct Cfg {
    static constexpr int NH = DV / 128;                     // d_v halves (MMA M = 128 each)
    static constexpr bool TF32 = (C == 64);                 // inter-chunk product in tf32
    static constexpr int NQK = 2;                           // Q/K stages
    static constexpr int NV = (DV == 128 && C == 64) ? 2 : 1;   // V stages
    static constexpr int NG = (C == 128) ? 1 : 2;           // G/O stages
    // software pipeline: chunk i + 1 is prepared (and its MMAs run) while the
    // epilogue of chunk i works from registers; needs two score buffers and
    // epilogue scratch of its own
    static constexpr bool PIPE = (C == 64);
    static constexpr int NSCB = PIPE ? 2 : 1;               // score buffers
    static constexpr int ROWB = 128;                        // bytes per swizzled row
    static constexpr int BOX = C * ROWB;                    // one [C x 64] bf16 box
    static constexpr int Q_BYTES = 2 * BOX;                 // d_k = 128 -> 2 boxes
    static constexpr int K_BYTES = 2 * BOX;
    static constexpr int V_BYTES = (DV / 64) * BOX;
    static constexpr int G_BYTES = (DV / 64) * BOX;
    static constexpr int P_BYTES = (C / 64) * BOX;          // rows t, C bf16 of s
    static constexpr int QT_BYTES = TF32 ? 4 * BOX : 0;     // rows t, 128 fp32 of k
    static constexpr int HT = C / 4;                        // tokens per thread, epilogue
    static constexpr int W = NH * 32;                       // state columns per thread
    // tensor-memory columns
    static constexpr int TM_S = 0;                          // T^T: NH x 128 fp32
    static constexpr int TM_O = NH * 128;                   // O^T: NH x C
    static constexpr int TM_SC = TM_O + NH * C;             // scores: NSCB x C
    static constexpr int TM_CP = TM_SC + NSCB * C;          // bf16 copy of T^T (bf16 mode): NH x 64
    static constexpr int TM_USED = TM_CP + (TF32 ? 0 : NH * 64);
    static constexpr int TM_ALLOC = TM_USED <= 256 ? 256 : 512;
    // shared memory (bytes from a 1024-aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + NQK * Q_BYTES;
    static constexpr int OFF_V = OFF_K + NQK * K_BYTES;
    static constexpr int OFF_G = OFF_V + NV * V_BYTES;
    static constexpr int OFF_P = OFF_G + NG * G_BYTES;
    static constexpr int OFF_QT = OFF_P + P_BYTES;
    // per Q/K stage: C fp32 decay sums b_t, then C fp32 block factors (gate scan)
    static constexpr int OFF_B = OFF_QT + QT_BYTES;
    static constexpr int OFF_BAR = OFF_B + NQK * 2 * C * 4;
    static constexpr int NUM_BARS = NQK + NV + NG + 12;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    // epilogue scratch: kCW x HT x 2 fp32 partial sums, then C x (rstd, -mean * rstd).
    // It gets its own space when that fits; otherwise it lives in the P buffer
    // (dead during the epilogue) and the warps meet once more before the next P.
    static constexpr int RED_BYTES = kCW * HT * 2 * 4 + C * 8;
    static constexpr int OFF_XRED = OFF_MISC + 16;
    static constexpr bool SEP_RED = OFF_XRED + RED_BYTES + 1024 <= kMaxSmem;
    static constexpr int OFF_RED = SEP_RED ? OFF_XRED : OFF_P;
    static constexpr int OFF_STAT = OFF_RED + kCW * HT * 2 * 4;
    static constexpr int USED = OFF_XRED + (SEP_RED ? RED_BYTES : 0);
    // room to round the dynamic shared memory base up to 1024 bytes; where less
    // than 1024 is left the kernel checks the base it got
    static constexpr int SLACK = USED + 1024 <= kMaxSmem ? 1024 : kMaxSmem - USED;
    static constexpr int SMEM = USED + SLACK;
    static_assert(SLACK >= 0, "shared memory budget");
    static_assert(SEP_RED || RED_BYTES <= P_BYTES, "epilogue scratch fits in P");
    static_assert(!PIPE || SEP_RED, "the pipelined epilogue needs scratch of its own");
    static_assert(TM_USED <= 512, "tensor memory budget");
    static_assert(C == 64 || C == 128, "chunk");
    static_assert(TF32 || NH == 1, "bf16 copy mode is laid out for one d_v half");
    // the padded rows (C..127) of the 128-row scores A operand read the bytes
    // after a Q stage's second box: the next Q stage or the first K stage.
    static_assert(OFF_K + (128 - C) * ROWB <= OFF_V, "scores padding rows stay in the allocation");
};

struct TcParams {
    CUtensorMap tmQ, tmK, tmV, tmG, tmO;
    CUtensorMap tmKs, tmVs;  // K and V in the state pass's sub-chunk tiles
    const float* bcum;       // [units][Npad] chunk-local cumulative log-decay
    const float* eblk;       // [units][Npad] block factors of the P columns (gate scan)
    float* seg_state;        // [units][slots][DV][DK]  (S^T, fp32)
    float* seg_decay;        // [units][slots]
    float* S_final;          // [units][DK][DV] or null
    const float* S0;         // [units][DK][DV] initial state, or null for zero
    const int* cu;           // packed batch: sequence b is token rows cu[b] .. cu[b+1]-1; or null
    int total;               // rows of the packed tensors
    void* O;                 // output base (tail rows of packed sequences are stored directly)
    const void* G;           // gate tensor (read directly by the output-rows kernel), or null
    unsigned int* status;
    int H, N, Npad, P, seg_len;
    int K, piece_len;        // state-pass pieces per segment and their length
    int piece_split;         // > 0: K = 2 pieces of piece_split and seg_len / C - piece_split chunks
    int slots;               // state-pass pieces (and seg_state slots) per unit
    // planned packed batch (varlen_plan_kernel): per unit {segments, segment
    // length, first seg_state slot, -}; the fused and state-pass work items
    // (unit, segment), longest segments first; the item counts
    const int4* unit_info;
    const int2* fused_items;
    const int2* state_items;
    const int* plan_count;
    float eps;
    int gn;                  // 1: GroupNorm + swish; 0: O = Y
    int has_g;
    int fault;               // test only: the fused kernel's first wait gives up (see gret_debug_inject_timeout)
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

// swish(g) = g sigmoid(g) = h (1 + tanh h) with h = g / 2, so that it costs one
// special-function operation (tanh.approx) instead of an exponential and a divide
__device__ __forceinline__ float swish_fast(float g) {
    const float h = 0.5f * g;
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(h));
    return fmaf(h, th, h);
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 16) tmem_ld_x16(taddr, r);
    else if constexpr (N == 32) tmem_ld_x32(taddr, r);
    else tmem_ld_x64(taddr, r);
}

template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[N]) {
    if constexpr (N == 16) tmem_st_x16(taddr, r);
    else if constexpr (N == 32) tmem_st_x32(taddr, r);
    else tmem_st_x64(taddr, r);
}

// One halving step of the cross-lane transpose-sum: lanes with bit OFF set
// keep the upper N/2 values, the others the lower N/2, and each adds its
// partner's copy of the half it keeps.
template <int N, int OFF>
__device__ __forceinline__ void transpose_sum_step(float (&v)[N], int lane) {
    if constexpr (OFF >= 1) {
        if constexpr (N >= 2) {
            constexpr int n = N / 2;
            const bool up = (lane & OFF) != 0;
#pragma unroll
            for (int j = 0; j < n; ++j) {
                const float send = up ? v[j] : v[j + n];
                const float keep = up ? v[j + n] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
            }
            transpose_sum_step<(n > 1 ? n : 1), OFF / 2>(reinterpret_cast<float(&)[(n > 1 ? n : 1)]>(v), lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
            transpose_sum_step<1, OFF / 2>(v, lane);
        }
    }
}

// Sum each of the N values of a lane over the 32 lanes of the warp.  On
// return, for N >= 32, v[j] (j < N / 32) holds the total of value index
// lane * (N / 32) + j; for N = 16, v[0] holds the total of index lane >> 1.
template <int N>
__device__ __forceinline__ void warp_transpose_sum(float (&v)[N], int lane) {
    static_assert(N == 16 || N % 32 == 0, "values per lane");
    transpose_sum_step<N, 16>(v, lane);
}

// Fused chunk loop for one (unit, segment).
//
// Roles.  Warps 0-15 compute, four per tensor-memory lane quarter.  In the
// fifth warpgroup, lane 0 of warp 16 issues every tcgen05 MMA and lane 0 of
// warp 17 every TMA load and store (warps 18-19 idle); the warpgroup hands
// most of its registers to the compute warps (kIssueRegs / kComputeRegs).
// Each compute warp tells the MMA warp when its share of a chunk's Q~ is
// ready (BQT: the inter-chunk MMAs start while P and K~ are still being
// computed), when its share of P and K~ is ready (BPREP), when its share of an
// eager state rescale is done (BTSC), and tells the TMA warp when its share of
// the output tile is staged in shared memory (BSTAGED).
//
// Schedule.  With 64-token chunks (PIPE) the compute warps take the output of
// chunk i from tensor memory into registers, prepare chunk i + 1 -- whose
// MMAs then run, its scores into the second score buffer -- and only then do
// the GroupNorm epilogue of chunk i.  With 128-token chunks there is no room
// for that, and each chunk is prepared, multiplied and finished in turn.
//
// State scaling.  Tensor memory holds T = S / E with E = e^Lambda, Lambda <= 0
// and the same in every thread.  A chunk is "lazy" when its largest K scale
// e^{-b_s - Lambda} stays within e^kLazyMax: then K~_s = e^{-b_s - Lambda} K_s,
// T += V^T K~ and Lambda += b_C, and T itself is not touched.  Otherwise the
// chunk is "eager": T is rescaled in place by e^{Lambda + b_C},
// K~_s = e^{b_C - b_s} K_s and Lambda = 0.  The inter-chunk read uses
// Q~_t = e^{b_t + Lambda} Q_t against T, and the state leaves as e^Lambda T.
// The MMA warp repeats the lazy/eager decision from the same decay sums with
// the same float operations, so both sides agree on it.
template <int DV, int C, bool PACKED>
__global__ void __launch_bounds__(kFusedThreads, 1) prefill_tc_kernel(const __grid_constant__ TcParams p) {
    using CF = Cfg<DV, C>;
    constexpr int NQK = CF::NQK, NV = CF::NV, NG = CF::NG, NH = CF::NH, W = CF::W, HT = CF::HT;
    constexpr bool TF32 = CF::TF32, PIPE = CF::PIPE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if constexpr (CF::SLACK < 1024) {
        if (sm + CF::USED > smem_raw + CF::SMEM) {   // the base is not aligned enough: report, do nothing
            if (tid == 0) atomicExch(p.status, kDevSmemLayout);
            return;
        }
    }

    // work item: a (unit, segment) of the uniform split, or of a packed
    // batch's plan (a block past the plan's item count has nothing to do)
    int u = 0, seg = 0, nseg_u = p.P, seg_len = p.seg_len;
    size_t in_slot = 0;                       // seg_state slot of S_in (seg > 0)
    if constexpr (!PACKED) {
        u = blockIdx.x / p.P;
        seg = blockIdx.x % p.P;
        in_slot = (size_t)u * p.slots + (size_t)seg * p.K - 1;
    } else {
        grid_dep_wait();
        if ((int)blockIdx.x >= p.plan_count[0]) return;
        const int2 it = p.fused_items[blockIdx.x];
        const int4 ui = p.unit_info[it.x];
        u = it.x;
        seg = it.y;
        nseg_u = ui.x;
        seg_len = ui.y;
        in_slot = (size_t)ui.z + seg - 1;
    }
    const int hh = u % p.H;
    const int n_begin = seg * seg_len;

    // Barriers.  The scores, the state MMA and the staged output have one
    // barrier per chunk parity, so that none of them can complete a phase
    // twice before its slowest waiter has seen the first: the next phase of
    // each pair needs a load that the waiter issues after its wait, or a step
    // of its own.  (Unpipelined, the scores use the first of their pair.)
    constexpr int BQK = 0, BV = NQK, BG = NQK + NV, BSC = NQK + NV + NG, BO = BSC + 2, BMMA = BSC + 3;
    constexpr int BQT = BSC + 5, BPREP = BSC + 6, BTSC = BSC + 7, BSTAGED = BSC + 8;
    // BDRAIN: the MMA warp's last commit, awaited before the tensor memory is
    // freed; BNEVER: nothing arrives at it (the injected timeout waits there)
    constexpr int BDRAIN = BSTAGED + 2, BNEVER = BSTAGED + 3;
    static_assert(BNEVER + 1 == CF::NUM_BARS, "barrier count");
    // barrier and parity of the scores of chunk j
    auto bsc = [&](int j) -> int { return PIPE ? BSC + (j & 1) : BSC; };
    auto bsc_par = [&](int j) -> uint32_t { return PIPE ? (j >> 1) & 1 : j & 1; };
    auto bar = [&](int i) -> uint32_t { return sb + CF::OFF_BAR + 8 * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);

    if (tid == 0) {
        for (int i = 0; i < CF::NUM_BARS; ++i) {
            // per-warp arrivals; BSTAGED takes one arrival after a block barrier
            // when the epilogue scratch shares the P buffer
            const bool per_warp =
                i == BQT || i == BPREP || i == BTSC || ((i == BSTAGED || i == BSTAGED + 1) && CF::SEP_RED);
            mbar_init(bar(i), per_warp ? kCW : 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tmQ);
        tma_prefetch_desc(&p.tmK);
        tma_prefetch_desc(&p.tmV);
        tma_prefetch_desc(&p.tmG);
        tma_prefetch_desc(&p.tmO);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), CF::TM_ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    // the setup above overlaps the previous kernel's tail; from here on this
    // kernel reads what the earlier ones wrote (decay sums, segment states)
    grid_dep_launch();
    grid_dep_wait();
    // this unit's sequence: batch bb of the uniform layout, or token rows
    // row0 .. row0 + Nu - 1 of a packed batch (PACKED)
    int bb = u / p.H, row0 = 0, Nu = p.N;
    if constexpr (PACKED) {
        bb = 0;
        packed_range(p.cu, u / p.H, p.total, row0, Nu);
        Nu = min(Nu, p.N);                    // tokens past max_seqlen are not processed
    }
    const int n_end = min(Nu, n_begin + seg_len);
    const int nchunks = n_end > n_begin ? (n_end - n_begin + C - 1) / C : 0;
    // a packed sequence's last chunk stops at its end: its output rows are
    // stored directly, since a full tile would overwrite the next sequence
    auto direct_tail = [&](int j) { return PACKED && n_end - (n_begin + j * C) < C; };
    if (warp >= kCW) {
      // ================================================================ issuing warpgroup
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" : : "n"(kIssueRegs));
      if (warp == kCW + 1) {
        if (lane == 0 && nchunks > 0) {
            // ============================================================ producer
            // the last chunk whose loads went into each stage (-1: none): on the
            // give-up path the loads still in flight are awaited before exit
            int last_qk[NQK], last_v[NV], last_g[NG];
            for (int x = 0; x < NQK; ++x) last_qk[x] = -1;
            for (int x = 0; x < NV; ++x) last_v[x] = -1;
            for (int x = 0; x < NG; ++x) last_g[x] = -1;
            auto issue_qk = [&](int j) {
                const int s = j % NQK, n0 = n_begin + j * C;
                last_qk[s] = j;
                const uint32_t fb = bar(BQK + s);
                mbar_arrive_expect_tx(fb, CF::Q_BYTES + CF::K_BYTES + 2 * C * 4);
                for (int x = 0; x < 2; ++x) {
                    tma_load_4d(sb + CF::OFF_Q + s * CF::Q_BYTES + x * CF::BOX, &p.tmQ, x * 64, hh, row0 + n0, bb, fb);
                    tma_load_4d(sb + CF::OFF_K + s * CF::K_BYTES + x * CF::BOX, &p.tmK, x * 64, hh, row0 + n0, bb, fb);
                }
                bulk_load(sb + CF::OFF_B + s * 2 * C * 4, p.bcum + (size_t)u * p.Npad + n0, C * 4, fb);
                bulk_load(sb + CF::OFF_B + (s * 2 + 1) * C * 4, p.eblk + (size_t)u * p.Npad + n0, C * 4, fb);
            };
            auto issue_v = [&](int j) {
                const int s = j % NV, n0 = n_begin + j * C;
                last_v[s] = j;
                const uint32_t fb = bar(BV + s);
                mbar_arrive_expect_tx(fb, CF::V_BYTES);
                for (int x = 0; x < DV / 64; ++x)
                    tma_load_4d(sb + CF::OFF_V + s * CF::V_BYTES + x * CF::BOX, &p.tmV, x * 64, hh, row0 + n0, bb, fb);
            };
            auto issue_g = [&](int j) {
                const int s = j % NG, n0 = n_begin + j * C;
                last_g[s] = j;
                const uint32_t fb = bar(BG + s);
                mbar_arrive_expect_tx(fb, CF::G_BYTES);
                for (int x = 0; x < DV / 64; ++x)
                    tma_load_4d(sb + CF::OFF_G + s * CF::G_BYTES + x * CF::BOX, &p.tmG, x * 64, hh, row0 + n0, bb, fb);
            };
            // the output tile of chunk j, written over G(j) in shared memory, goes
            // out; once the store has read the stage it takes the G of chunk j + NG
            auto store_out = [&](int j) -> bool {
                if (!mbar_wait(bar(BSTAGED + (j & 1)), (j >> 1) & 1, p.status, abort_flag)) return false;
                const uint32_t sG = sb + CF::OFF_G + (j % NG) * CF::G_BYTES;
                const int n0 = n_begin + j * C;
                if (!direct_tail(j)) {
                    for (int x = 0; x < DV / 64; ++x)
                        tma_store_4d(&p.tmO, sG + x * CF::BOX, x * 64, hh, row0 + n0, bb);
                    bulk_commit();
                    bulk_wait_read<0>();
                }
                if (p.has_g && j + NG < nchunks) issue_g(j + NG);
                return true;
            };
            if (p.fault) mbar_wait_injected_timeout(bar(BNEVER), p.status, abort_flag);
            if (!*abort_flag) {
                issue_qk(0);
                if (nchunks > 1) issue_qk(1);
                issue_v(0);
                if (NV == 2 && nchunks > 1) issue_v(1);
                if (p.has_g) {
                    issue_g(0);
                    if (NG == 2 && nchunks > 1) issue_g(1);
                }
                for (int i = 0; i < nchunks; ++i) {
                    // pipelined, the epilogue of chunk i - 1 ends after chunk i's preparation
                    if (PIPE && i >= 1 && !store_out(i - 1)) break;
                    // once the state MMA of chunk i is done, its Q/K and V stages are free
                    if (!mbar_wait(bar(BMMA + (i & 1)), (i >> 1) & 1, p.status, abort_flag)) break;
                    if (i + NQK < nchunks) issue_qk(i + NQK);
                    if (i + NV < nchunks) issue_v(i + NV);
                    if (!PIPE && !store_out(i)) break;
                }
                if (PIPE && !*abort_flag) store_out(nchunks - 1);
            }
            if (*abort_flag) {
                // gave up: no more loads are issued; let those in flight land
                // (at most one per stage) before the shared memory is released
                for (int x = 0; x < NQK; ++x)
                    if (last_qk[x] >= 0) mbar_wait_drain(bar(BQK + x), (last_qk[x] / NQK) & 1, kWaitCycles);
                for (int x = 0; x < NV; ++x)
                    if (last_v[x] >= 0) mbar_wait_drain(bar(BV + x), (last_v[x] / NV) & 1, kWaitCycles);
                for (int x = 0; x < NG; ++x)
                    if (last_g[x] >= 0) mbar_wait_drain(bar(BG + x), (last_g[x] / NG) & 1, kWaitCycles);
            }
            bulk_wait<0>();
        }
      } else if (warp == kCW) {
        if (lane == 0 && nchunks > 0) {
            // ============================================================ MMA issuer
            constexpr uint32_t id_sc = idesc_bf16(128, C, false, false);
            constexpr uint32_t id_qs = idesc_bf16(128, C, false, false);
            constexpr uint32_t id_qs32 = idesc_tf32(128, C, false, false);
            constexpr uint32_t id_pv = idesc_bf16(128, C, true, false);
            constexpr uint32_t id_kv = idesc_bf16(128, DK, true, true);
            // scores D[t][s] = Q K^T over d_k (M = 128 rows of t; rows >= C unused)
            auto issue_scores = [&](int j) {
                const int s = j % NQK;
                if (!mbar_wait(bar(BQK + s), (j / NQK) & 1, p.status, abort_flag)) return;
                tc_fence_after();
                const uint32_t sQ = sb + CF::OFF_Q + s * CF::Q_BYTES, sK = sb + CF::OFF_K + s * CF::K_BYTES;
                const uint32_t dst = tm + CF::TM_SC + (PIPE ? (j & 1) * C : 0);
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = (k >> 2) * CF::BOX + (k & 3) * 32;
                    mma_ss(dst, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), id_sc, k > 0);
                }
                mma_commit(bar(bsc(j)));
            };
            issue_scores(0);

            float lam = 0.f;
            int nsplit = 0;
            for (int i = 0; i < nchunks; ++i) {
                const int sq = i % NQK, sv = i % NV;
                const uint32_t sQ = sb + CF::OFF_Q + sq * CF::Q_BYTES;
                const uint32_t sK = sb + CF::OFF_K + sq * CF::K_BYTES;
                const uint32_t sV = sb + CF::OFF_V + sv * CF::V_BYTES;
                // the decay sums of chunk i landed before its scores were issued
                const float bC = reinterpret_cast<const float*>(sm + CF::OFF_B + sq * 2 * C * 4)[C - 1];
                const bool eager = (-bC - lam) > kLazyMax;

                // inter-chunk: O^T = T^T Q~^T, as soon as Q~ (and, with bf16 inter
                // products, the bf16 copy of T) is ready and the previous state
                // MMA has written T
                if (!mbar_wait(bar(BQT), i & 1, p.status, abort_flag)) break;
                if (i > 0 && !mbar_wait(bar(BMMA + ((i - 1) & 1)), ((i - 1) >> 1) & 1, p.status, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    if constexpr (TF32) {
#pragma unroll
                        for (int k = 0; k < DK / 8; ++k) {
                            const uint32_t qoff = (k >> 2) * CF::BOX + (k & 3) * 32;
                            mma_ts_tf32(tm + CF::TM_O + h * C, tm + CF::TM_S + h * 128 + k * 8,
                                        sdesc_sw128(sb + CF::OFF_QT + qoff, 16, 1024), id_qs32, k > 0);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < DK / 16; ++k) {
                            const uint32_t qoff = (k >> 2) * CF::BOX + (k & 3) * 32;
                            mma_ts(tm + CF::TM_O + h * C, tm + CF::TM_CP + h * 64 + k * 8,
                                   sdesc_sw128(sQ + qoff, 16, 1024), id_qs, k > 0);
                        }
                    }
                }
                // pipelined: the next chunk's scores go to the other score buffer
                // now, so that its P is ready to start when this chunk's output is
                if (PIPE && i + 1 < nchunks) issue_scores(i + 1);
                // intra-chunk: O^T += V^T P^T once P and K~ are ready
                if (!mbar_wait(bar(BPREP), i & 1, p.status, abort_flag)) break;
                tc_fence_after();
                if (!mbar_wait(bar(BV + sv), (i / NV) & 1, p.status, abort_flag)) break;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const uint32_t vA = sV + 2 * h * CF::BOX;   // d_v rows h*128 .. +127 (two boxes)
#pragma unroll
                    for (int k = 0; k < C / 16; ++k) {
                        const uint32_t poff = (k >> 2) * CF::BOX + (k & 3) * 32;
                        mma_ss(tm + CF::TM_O + h * C, sdesc_sw128(vA + k * 2048, CF::BOX, 1024),
                               sdesc_sw128(sb + CF::OFF_P + poff, 16, 1024), id_pv, 1);
                    }
                }
                mma_commit(bar(BO));
                if (TF32 && eager) {
                    // T is rescaled between the inter-chunk read and the state MMA
                    if (!mbar_wait(bar(BTSC), nsplit & 1, p.status, abort_flag)) break;
                    ++nsplit;
                    tc_fence_after();
                }
                // T^T += V^T K~ for both d_v halves
#pragma unroll
                for (int h = 0; h < NH; ++h) {
#pragma unroll
                    for (int k = 0; k < C / 16; ++k)
                        mma_ss(tm + CF::TM_S + h * 128, sdesc_sw128(sV + 2 * h * CF::BOX + k * 2048, CF::BOX, 1024),
                               sdesc_sw128(sK + k * 2048, CF::BOX, 1024), id_kv, 1);
                }
                mma_commit(bar(BMMA + (i & 1)));
                if (!PIPE && i + 1 < nchunks) issue_scores(i + 1);
                lam = eager ? 0.f : lam + bC;
            }
            // every MMA this thread issued has completed before the tensor
            // memory is freed, on the give-up path too
            mma_commit(bar(BDRAIN));
            mbar_wait_drain(bar(BDRAIN), 0, kWaitCycles);
        }
      }
    } else {
        // ================================================================ compute warps
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" : : "n"(kComputeRegs));
        const int q4 = warp & 3;       // tensor-memory lane quarter of this warp
        const int grp = warp >> 2;     // which of the four compute warps sharing the quarter
        const uint32_t lq = (uint32_t)(32 * q4) << 16;
        // every lane of this warp has finished its part of a step: one arrival
        auto warp_arrive = [&](int b) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(b));
        };

        // this thread's slice of T^T: lanes of quarter q4, columns col0 .. col0 + W - 1
        const int col0 = grp * W;
        const int s_half = col0 / 128, s_k0 = col0 % 128;
        const int s_d = s_half * 128 + q4 * 32 + lane;
        {
            uint32_t r[W];
            if (seg > 0) {
                const float* src = p.seg_state + in_slot * DV * DK + (size_t)s_d * DK + s_k0;
                const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
                for (int j = 0; j < W / 4; ++j) {
                    const float4 v = s4[j];
                    r[4 * j] = f2u(v.x); r[4 * j + 1] = f2u(v.y); r[4 * j + 2] = f2u(v.z); r[4 * j + 3] = f2u(v.w);
                }
            } else if (p.S0) {
                // the caller's initial state, [DK][DV]: lanes read consecutive d_v
                const float* src = p.S0 + (size_t)u * DK * DV + (size_t)s_k0 * DV + s_d;
#pragma unroll
                for (int j = 0; j < W; ++j) r[j] = f2u(src[(size_t)j * DV]);
            } else {
#pragma unroll
                for (int j = 0; j < W; ++j) r[j] = 0u;
            }
            tmem_st<W>(tm + lq + CF::TM_S + col0, r);
            tmem_wait_st();
        }

        float lam = 0.f;          // Lambda
        struct ChunkGate { float bC, escale; bool eager; };

        // ---- preparation of chunk i: Q~ (phase A), then P and K~ (phase B)
        auto prep = [&](int i) -> ChunkGate {
            const int sq = i % NQK;
            const float* bc = reinterpret_cast<const float*>(sm + CF::OFF_B + sq * 2 * C * 4);
            const float* eb = bc + C;     // block factors E_s
            uint8_t* Qp = sm + CF::OFF_Q + sq * CF::Q_BYTES;
            uint8_t* Kp = sm + CF::OFF_K + sq * CF::K_BYTES;
            mbar_wait(bar(BQK + sq), (i / NQK) & 1, p.status, abort_flag);
            const float bC = bc[C - 1];
            const bool eager = (-bC - lam) > kLazyMax;
            const float escale = __expf(lam + bC);
            const int valid = n_end - (n_begin + i * C);   // rows of this unit in the chunk (PACKED)

            // phase A: Q~ = e^{b_t + Lambda} Q for the inter-chunk read, which the
            // MMA warp starts as soon as every warp has done its share
            if constexpr (TF32) {
                // fp32 copy in its own buffer, so the scores MMA may still be reading Q
                for (int it = tid; it < C * 16; it += kCT) {
                    // row t, bf16 16-byte chunk c (d_k 8c .. 8c+7); consecutive items are
                    // consecutive rows, so the swizzle spreads each access phase over
                    // eight different bank groups
                    const int t = it % C, c = it / C;
                    const float f = __expf(bc[t] + lam);
                    const uint4 w = *reinterpret_cast<const uint4*>(Qp + (c >> 3) * CF::BOX + t * 128 +
                                                                    (((c & 7) ^ (t & 7)) << 4));
                    const uint32_t* e = reinterpret_cast<const uint32_t*>(&w);
                    float x[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e[j]));
                        x[2 * j] = f2.x * f;
                        x[2 * j + 1] = f2.y * f;
                    }
                    uint8_t* row = sm + CF::OFF_QT + (c >> 2) * CF::BOX + t * 128;
                    const int lc = 2 * (c & 3);
                    *reinterpret_cast<float4*>(row + ((lc ^ (t & 7)) << 4)) = make_float4(x[0], x[1], x[2], x[3]);
                    *reinterpret_cast<float4*>(row + (((lc + 1) ^ (t & 7)) << 4)) =
                        make_float4(x[4], x[5], x[6], x[7]);
                }
            } else {
                // in place, once the scores MMA has read Q
                mbar_wait(bar(bsc(i)), bsc_par(i), p.status, abort_flag);
                tc_fence_after();
                for (int it = tid; it < C * 16; it += kCT) {
                    const int row = (it >> 3) % C;
                    scale_bf16x8(Qp + it * 16, __expf(bc[row] + lam));
                }
                // bf16 copy of T (and the eager rescale); needs the previous state MMA
                if (i > 0) {
                    mbar_wait(bar(BMMA + ((i - 1) & 1)), ((i - 1) >> 1) & 1, p.status, abort_flag);
                    tc_fence_after();
                }
                uint32_t r[W];
                tmem_ld<W>(tm + lq + CF::TM_S + col0, r);
                tmem_wait_ld();
                uint32_t pk[W / 2];
#pragma unroll
                for (int j = 0; j < W / 2; ++j) pk[j] = pack_bf16x2(u2f(r[2 * j]), u2f(r[2 * j + 1]));
                tmem_st<W / 2>(tm + lq + CF::TM_CP + col0 / 2, pk);
                if (eager) {
#pragma unroll
                    for (int j = 0; j < W; ++j) r[j] = f2u(u2f(r[j]) * escale);
                    tmem_st<W>(tm + lq + CF::TM_S + col0, r);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(BQT);

            // phase B: P and K~, for the intra-chunk and state MMAs
            if constexpr (TF32) {
                mbar_wait(bar(bsc(i)), bsc_par(i), p.status, abort_flag);
                tc_fence_after();
            }
            // P[t][s] = A[t][s] e^{b_t - b_s} (s <= t) -> bf16, K-major rows t.  The
            // gate scan gives E_s = e^{b_{s0} - b_s} with s0 the first of the C/4
            // columns this warp owns, so e^{b_t - b_s} = e^{b_t - b_{s0}} E_s takes
            // one exponential per row.  A block whose decay drops by more than
            // kBlockMax is marked (E_{s0} < 0) and takes e^{b_t - b_s} directly.
            if (q4 * 32 < C) {
                constexpr int PC = C / 4;
                const int t = q4 * 32 + lane;
                const int sb0 = grp * PC;
                uint32_t r[PC];
                tmem_ld<PC>(tm + lq + CF::TM_SC + (PIPE ? (i & 1) * C : 0) + sb0, r);
                const float bt = bc[t];
                const bool fac = eb[sb0] >= 0.f;                 // the same for the whole warp
                const float f = __expf(fminf(bt - bc[sb0], 0.f));
                tmem_wait_ld();
                auto emit = [&](auto fac_tag) {
                    constexpr bool FAC = decltype(fac_tag)::value;
                    const float* src = FAC ? eb : bc;
#pragma unroll
                    for (int c8 = 0; c8 < PC / 8; ++c8) {
                        const int s0 = sb0 + c8 * 8;
                        const float4 a0 = *reinterpret_cast<const float4*>(src + s0);
                        const float4 a1 = *reinterpret_cast<const float4*>(src + s0 + 4);
                        const float xs[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int sa = s0 + 2 * e;
                            const float m0 = FAC ? f * xs[2 * e] : __expf(bt - xs[2 * e]);
                            const float m1 = FAC ? f * xs[2 * e + 1] : __expf(bt - xs[2 * e + 1]);
                            const float v0 = sa <= t ? u2f(r[c8 * 8 + 2 * e]) * m0 : 0.f;
                            const float v1 = sa + 1 <= t ? u2f(r[c8 * 8 + 2 * e + 1]) * m1 : 0.f;
                            w[e] = pack_bf16x2(v0, v1);
                        }
                        const int region = s0 >> 6, chunk = (s0 & 63) >> 3;
                        uint8_t* dst = sm + CF::OFF_P + region * CF::BOX + t * 128 + ((chunk ^ (t & 7)) << 4);
                        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                };
                if (fac) emit(std::true_type{});
                else emit(std::false_type{});
            }
            // K~ = e^{-b_s - Lambda} K (lazy) or e^{b_C - b_s} K (eager), in place, as
            // 16-byte items.  With 64-token chunks the warps that own tensor-memory
            // lanes 64..127 compute no P, so they take 3/4 of the items.
            {
                constexpr int NKI = C * 16;
                int it0, it1, step;
                if constexpr (C == 64) {
                    constexpr int cut = NKI * 3 / 4;
                    step = kCT / 2;
                    if (q4 >= 2) { it0 = (((grp << 1) | (q4 - 2)) << 5) + lane; it1 = cut; }
                    else { it0 = cut + (((grp << 1) | q4) << 5) + lane; it1 = NKI; }
                } else {
                    it0 = tid; it1 = NKI; step = kCT;
                }
                for (int it = it0; it < it1; it += step) {
                    const int row = (it >> 3) % C;
                    const float ex = eager ? (bC - bc[row]) : (-bc[row] - lam);
                    // rows past a packed unit's end (the next sequence's) add nothing;
                    // in the uniform layout they load as zeros
                    scale_bf16x8(Kp + it * 16, (!PACKED || row < valid) ? __expf(ex) : 0.f);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(BPREP);
            return ChunkGate{bC, escale, eager};
        };

        // ---- the output MMAs of chunk i are done: Y^T into registers, and the
        // eager state rescale where the inter-chunk read had to see T unscaled
        auto drain = [&](int i, const ChunkGate& cg, float (&y)[NH][HT]) {
            mbar_wait(bar(BO), i & 1, p.status, abort_flag);
            tc_fence_after();
            if (TF32 && cg.eager) {
                // in two halves, to keep the live registers down
#pragma unroll
                for (int hw = 0; hw < 2; ++hw) {
                    uint32_t r[W / 2];
                    tmem_ld<W / 2>(tm + lq + CF::TM_S + col0 + hw * (W / 2), r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < W / 2; ++j) r[j] = f2u(u2f(r[j]) * cg.escale);
                    tmem_st<W / 2>(tm + lq + CF::TM_S + col0 + hw * (W / 2), r);
                }
                tmem_wait_st();
                tc_fence_before();
                warp_arrive(BTSC);
            }
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                uint32_t r[HT];
                tmem_ld<HT>(tm + lq + CF::TM_O + h * C + grp * HT, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < HT; ++j) y[h][j] = u2f(r[j]);
            }
            tc_fence_before();
        };

        // ---- epilogue of chunk i from Y in registers: GroupNorm over d_v, times
        // swish(G), as bf16 over G in its stage, then handed to the TMA warp for
        // the store.  Thread (q4, grp, lane) owns d_v channels h*128 + q4*32 + lane
        // (h < NH) for tokens grp*HT .. grp*HT + HT - 1.
        auto epilogue = [&](int i, const float (&y)[NH][HT]) {
            const int g = i % NG;
            if (p.has_g) mbar_wait(bar(BG + g), (i / NG) & 1, p.status, abort_flag);
            uint8_t* Gp = sm + CF::OFF_G + g * CF::G_BYTES;
            const int t0 = grp * HT;
            float* red = reinterpret_cast<float*>(sm + CF::OFF_RED);
            float2* stat = reinterpret_cast<float2*>(sm + CF::OFF_STAT);
            if (p.gn) {
                // per-token sums over this thread's channels, then over the
                // warp's lanes, then over the four lane quarters
#pragma unroll
                for (int pass = 0; pass < 2; ++pass) {
                    float v[HT];
#pragma unroll
                    for (int j = 0; j < HT; ++j) {
                        float acc = pass == 0 ? y[0][j] : y[0][j] * y[0][j];
#pragma unroll
                        for (int h = 1; h < NH; ++h) acc += pass == 0 ? y[h][j] : y[h][j] * y[h][j];
                        v[j] = acc;
                    }
                    warp_transpose_sum<HT>(v, lane);
                    if constexpr (HT >= 32) {
#pragma unroll
                        for (int j = 0; j < HT / 32; ++j) red[(warp * HT + lane * (HT / 32) + j) * 2 + pass] = v[j];
                    } else {
                        if ((lane & 1) == 0) red[(warp * HT + (lane >> 1)) * 2 + pass] = v[0];
                    }
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
            auto d_of = [&](int h) { return h * 128 + q4 * 32 + lane; };
            int goff[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) goff[h] = (d_of(h) >> 6) * CF::BOX + (d_of(h) & 7) * 2;
            const int dc = ((q4 * 32 + lane) & 63) >> 3;   // the same for both halves
            // the last chunk of a packed sequence: its rows go straight to global memory
            const bool tail = direct_tail(i);
#pragma unroll
            for (int j = 0; j < HT; ++j) {
                const int t = t0 + j;
                const int rowoff = t * 128 + ((dc ^ (t & 7)) << 4);
                float2 st = make_float2(1.f, 0.f);
                if (p.gn) st = stat[t];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    __nv_bfloat16* gp = reinterpret_cast<__nv_bfloat16*>(Gp + goff[h] + rowoff);
                    float o = y[h][j];
                    // GroupNorm as one FMA, then times swish(g) = g * sigmoid(g)
                    if (p.gn) o = fmaf(o, st.x, st.y) * swish_fast(__bfloat162float(*gp));
                    if (!PACKED || !tail) {
                        *gp = __float2bfloat16_rn(o);
                    } else if (t < n_end - (n_begin + i * C)) {
                        __nv_bfloat16* Ot = static_cast<__nv_bfloat16*>(p.O) +
                                            ((size_t)(row0 + n_begin + i * C + t) * p.H + hh) * DV + d_of(h);
                        *Ot = __float2bfloat16_rn(o);
                    }
                }
            }
            fence_proxy_async_smem();
            if constexpr (CF::SEP_RED) {
                warp_arrive(BSTAGED + (i & 1));
            } else {
                // the next chunk's P overwrites the statistics: every warp has read them
                named_bar_sync(1, kCT);
                if (tid == 0) mbar_arrive(bar(BSTAGED + (i & 1)));
            }
        };

        if constexpr (PIPE) {
            // Y(i) -> registers; prepare chunk i + 1 (its MMAs start); epilogue of i
            ChunkGate cg = nchunks > 0 ? prep(0) : ChunkGate{0.f, 1.f, false};
            for (int i = 0; i < nchunks; ++i) {
                float y[NH][HT];
                drain(i, cg, y);
                lam = cg.eager ? 0.f : lam + cg.bC;
                if (i + 1 < nchunks) cg = prep(i + 1);
                epilogue(i, y);
            }
        } else {
            for (int i = 0; i < nchunks; ++i) {
                const ChunkGate cg = prep(i);
                float y[NH][HT];
                drain(i, cg, y);
                lam = cg.eager ? 0.f : lam + cg.bC;
                epilogue(i, y);
            }
        }

        // ------------------------------------------------------------ state out: e^Lambda T
        if (nchunks > 0) {
            mbar_wait(bar(BMMA + ((nchunks - 1) & 1)), ((nchunks - 1) >> 1) & 1, p.status, abort_flag);
            tc_fence_after();
        }
        if (p.S_final && seg == nseg_u - 1) {
            const float sc = __expf(lam);
            uint32_t r[W];
            tmem_ld<W>(tm + lq + CF::TM_S + col0, r);
            tmem_wait_ld();
            float* dst = p.S_final + (size_t)u * DK * DV;
#pragma unroll
            for (int j = 0; j < W; ++j) dst[(size_t)(s_k0 + j) * DV + s_d] = u2f(r[j]) * sc;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, CF::TM_ALLOC);
    }
}

// ---------------------------------------------------------------------------
// Segment state pass: dS_p = sum over the segment's tokens of
// e^{a_p - B_s} K_s^T V_s (B_s the log-decay from the segment start through s,
// a_p the segment total), from K, V and the decay sums alone.  The same
// lazy/eager state scaling as the fused kernels, decided per chunk of C tokens;
// the K/V tiles stream through a ring of sub-chunks of SUB tokens (64 where a
// whole 128-token chunk of d_v = 256 would leave room for two stages only), so
// that three or more stages of loads stay in flight per SM.
constexpr int kStateThreads = 256;

// tokens per staged K/V tile of the state pass
constexpr int state_sub(int dv, int C) { return (C == 128 && dv == 256) ? 64 : C; }

template <int DV, int C>
struct StateCfg {
    static constexpr int NH = DV / 128;
    static constexpr int SUB = state_sub(DV, C);
    static constexpr int NSUB = C / SUB;                    // sub-chunks per chunk
    static constexpr int BOX = SUB * 128;
    static constexpr int K_BYTES = 2 * BOX;
    static constexpr int V_BYTES = (DV / 64) * BOX;
    // as many K + V stages as about 210 KB hold (2-6), to keep loads in flight
    static constexpr int NS_FIT = (210 * 1024) / (K_BYTES + V_BYTES + C * 4);
    static constexpr int NS = NS_FIT > 6 ? 6 : NS_FIT;
    static_assert(NS >= 2, "state pass stages");
    static constexpr int W = NH * 64;                       // state columns per thread
    static constexpr int TM_ALLOC = NH * 128 <= 128 ? 128 : 256;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + NS * K_BYTES;
    // the decay sums of the whole chunk a sub-chunk belongs to
    static constexpr int OFF_B = OFF_V + NS * V_BYTES;
    static constexpr int OFF_BAR = OFF_B + NS * C * 4;
    // full and empty barrier per stage, then the drain barrier of the last commit
    static constexpr int OFF_MISC = OFF_BAR + (2 * NS + 1) * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

template <int DV, int C, bool PACKED>
__global__ void __launch_bounds__(kStateThreads, 1) prefill_state_kernel(const __grid_constant__ TcParams p) {
    using CF = StateCfg<DV, C>;
    constexpr int NS = CF::NS, NH = CF::NH, W = CF::W, SUB = CF::SUB, NSUB = CF::NSUB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, gi = warp >> 2;
    const uint32_t lq = (uint32_t)(32 * q4) << 16;

    // work item: a piece of the uniform split, or a segment of a packed
    // batch's plan (one piece per segment; a block past the plan's count has
    // nothing to do)
    int u = 0, seg = 0, piece_len = p.piece_len, n_begin = 0;
    size_t out_slot = 0;
    if constexpr (!PACKED) {
        if (p.piece_split > 0) {
            // each segment in a long and a short piece: the long ones first (the
            // lower block indices start first), the short ones after, two to an SM
            const int nseg = p.slots / 2, nlong = (int)gridDim.x / 2;
            const int b = (int)blockIdx.x, second = b >= nlong ? 1 : 0, bi = b - second * nlong;
            u = bi / nseg;
            const int sg = bi % nseg;
            seg = 2 * sg + second;
            n_begin = sg * p.seg_len + second * p.piece_split * C;
            piece_len = second ? p.seg_len - p.piece_split * C : p.piece_split * C;
        } else {
            u = blockIdx.x / p.slots;
            seg = blockIdx.x % p.slots;
            n_begin = seg * piece_len;
        }
        out_slot = (size_t)u * p.slots + seg;
    } else {
        grid_dep_wait();
        if ((int)blockIdx.x >= p.plan_count[1]) return;
        const int2 it = p.state_items[blockIdx.x];
        const int4 ui = p.unit_info[it.x];
        u = it.x;
        seg = it.y;
        piece_len = ui.y;
        n_begin = seg * piece_len;
        out_slot = (size_t)ui.z + seg;
    }
    const int hh = u % p.H;

    auto full = [&](int s) -> uint32_t { return sb + CF::OFF_BAR + 8 * s; };
    auto empty = [&](int s) -> uint32_t { return sb + CF::OFF_BAR + 8 * (NS + s); };
    const uint32_t drain_bar = sb + CF::OFF_BAR + 8 * (2 * NS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);

    if (tid == 0) {
        for (int i = 0; i < 2 * NS + 1; ++i) mbar_init(sb + CF::OFF_BAR + 8 * i, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tmKs);
        tma_prefetch_desc(&p.tmVs);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), CF::TM_ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;

    // everything above overlaps the previous kernel's tail; the loads need its
    // decay sums
    grid_dep_launch();
    grid_dep_wait();
    // this unit's sequence (see the fused kernel)
    int bb = u / p.H, row0 = 0, Nu = p.N;
    if constexpr (PACKED) {
        bb = 0;
        packed_range(p.cu, u / p.H, p.total, row0, Nu);
        Nu = min(Nu, p.N);                    // tokens past max_seqlen are not processed
    }
    const int n_end = min(Nu, n_begin + piece_len);
    // sub-chunks of SUB tokens; the pieces start on chunk boundaries
    const int nsub = n_end > n_begin ? (n_end - n_begin + SUB - 1) / SUB : 0;
    int last_issued = -1;     // thread 0: the last sub-chunk whose loads it issued
    auto issue = [&](int j) {
        const int s = j % NS, nc0 = n_begin + (j / NSUB) * C, n0 = nc0 + (j % NSUB) * SUB;
        last_issued = j;
        mbar_arrive_expect_tx(full(s), CF::K_BYTES + CF::V_BYTES + C * 4);
        for (int x = 0; x < 2; ++x)
            tma_load_4d(sb + CF::OFF_K + s * CF::K_BYTES + x * CF::BOX, &p.tmKs, x * 64, hh, row0 + n0, bb, full(s));
        for (int x = 0; x < DV / 64; ++x)
            tma_load_4d(sb + CF::OFF_V + s * CF::V_BYTES + x * CF::BOX, &p.tmVs, x * 64, hh, row0 + n0, bb, full(s));
        bulk_load(sb + CF::OFF_B + s * C * 4, p.bcum + (size_t)u * p.Npad + nc0, C * 4, full(s));
    };
    if (tid == 0)
        for (int j = 0; j < NS && j < nsub; ++j) issue(j);

    const int col0 = gi * W;
#pragma unroll 1
    for (int cb = 0; cb < W / 32; ++cb) {
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = 0u;
        tmem_st<32>(tm + lq + col0 + cb * 32, r);
    }
    tmem_wait_st();

    float lam = 0.f, seg_decay = 0.f;
    for (int i = 0; i < nsub; ++i) {
        const int s = i % NS, hs = i % NSUB;             // stage; sub-chunk within its chunk
        const float* bc = reinterpret_cast<const float*>(sm + CF::OFF_B + s * C * 4);
        mbar_wait(full(s), (i / NS) & 1, p.status, abort_flag);
        const float bC = bc[C - 1];
        // lam and the decision change only at chunk ends, so every sub-chunk
        // of a chunk takes the same one
        const bool eager = (-bC - lam) > kLazyMax;
        uint8_t* Kp = sm + CF::OFF_K + s * CF::K_BYTES;
        {
            constexpr int NIT = SUB * 16 / kStateThreads;   // 4 or 8 items per thread
            uint4 w[NIT];
            float e[NIT];
#pragma unroll
            for (int k = 0; k < NIT; ++k) {
                const int ci = tid + k * kStateThreads;
                w[k] = *reinterpret_cast<const uint4*>(Kp + ci * 16);
                e[k] = bc[hs * SUB + (ci >> 3) % SUB];
            }
            const int valid = n_end - (n_begin + i * SUB);   // rows of this unit in the sub-chunk
#pragma unroll
            for (int k = 0; k < NIT; ++k) {
                // rows past the unit's end (the next packed sequence's) add nothing
                const float sc = (!PACKED || ((tid + k * kStateThreads) >> 3) % SUB < valid)
                                     ? __expf(eager ? (bC - e[k]) : (-e[k] - lam)) : 0.f;
                uint32_t* x = reinterpret_cast<uint32_t*>(&w[k]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x[j]));
                    x[j] = pack_bf16x2(f2.x * sc, f2.y * sc);
                }
                *reinterpret_cast<uint4*>(Kp + (tid + k * kStateThreads) * 16) = w[k];
            }
        }
        if (eager && hs == 0) {
            // T *= e^{Lambda + b_C}, after the previous chunk's state MMA
            if (i > 0) {
                mbar_wait(empty((i - 1) % NS), ((i - 1) / NS) & 1, p.status, abort_flag);
                tc_fence_after();
            }
            const float escale = __expf(lam + bC);
#pragma unroll 1
            for (int cb = 0; cb < W / 32; ++cb) {
                uint32_t r[32];
                tmem_ld<32>(tm + lq + col0 + cb * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = f2u(u2f(r[j]) * escale);
                tmem_st<32>(tm + lq + col0 + cb * 32, r);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && !*abort_flag) {
            tc_fence_after();
            const uint32_t sK = sb + CF::OFF_K + s * CF::K_BYTES, sV = sb + CF::OFF_V + s * CF::V_BYTES;
            constexpr uint32_t id_kv = idesc_bf16(128, DK, true, true);
#pragma unroll
            for (int h = 0; h < NH; ++h) {
#pragma unroll
                for (int k = 0; k < SUB / 16; ++k)
                    mma_ss(tm + h * 128, sdesc_sw128(sV + 2 * h * CF::BOX + k * 2048, CF::BOX, 1024),
                           sdesc_sw128(sK + k * 2048, CF::BOX, 1024), id_kv, 1);
            }
            mma_commit(empty(s));
            // the stage the previous sub-chunk used is free once its MMAs are
            // done (they run before this one's, which queue behind them)
            if (i > 0 && i - 1 + NS < nsub &&
                mbar_wait(empty((i - 1) % NS), ((i - 1) / NS) & 1, p.status, abort_flag))
                issue(i - 1 + NS);
        }
        if (hs == NSUB - 1 || i == nsub - 1) {
            seg_decay += bC;
            lam = eager ? 0.f : lam + bC;
        }
    }
    if (tid == 0) {
        // every MMA issued has completed, and on the give-up path every load
        // issued has landed, before the tensor and shared memory are released
        // (loads into a stage are issued only after the previous chunk in
        // it was consumed, so the last NS chunks issued are the ones in flight)
        mma_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, kWaitCycles);
        if (*abort_flag)
            for (int j = last_issued; j >= 0 && j > last_issued - NS; --j)
                mbar_wait_drain(full(j % NS), (j / NS) & 1, kWaitCycles);
    }
    if (nsub > 0) {
        mbar_wait(empty((nsub - 1) % NS), ((nsub - 1) / NS) & 1, p.status, abort_flag);
        tc_fence_after();
    }
    {
        const float sc = __expf(lam);
        const int s_d = (col0 / 128) * 128 + q4 * 32 + lane, s_k0 = col0 % 128;
        float* dst = p.seg_state + out_slot * DV * DK + (size_t)s_d * DK + s_k0;
#pragma unroll 1
        for (int cb = 0; cb < W / 32; ++cb) {
            uint32_t r[32];
            tmem_ld<32>(tm + lq + col0 + cb * 32, r);
            tmem_wait_ld();
            float4* d4 = reinterpret_cast<float4*>(dst + cb * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                d4[j] = make_float4(u2f(r[4 * j]) * sc, u2f(r[4 * j + 1]) * sc, u2f(r[4 * j + 2]) * sc,
                                    u2f(r[4 * j + 3]) * sc);
        }
        if (tid == 0) p.seg_decay[out_slot] = seg_decay;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, CF::TM_ALLOC);
    }
}

// Chunk-local inclusive sums of log gamma: bcum[u][n] = sum_{j in chunk, j <= n} lg_j,
// and the P step's block factors eblk (below).
// Padding tokens (n >= N) carry lg = 0, so they repeat the chunk total.
constexpr int kScanThreads = 256;   // a block scans 256 / C chunks of one unit

__global__ void __launch_bounds__(kScanThreads) gate_scan_kernel(const float* __restrict__ z,
                                                                 const int* __restrict__ cu_seqlens, int total,
                                                                 float* __restrict__ bcum, float* __restrict__ eblk,
                                                                 int H, int N, int Npad, int C, float inv_tau,
                                                                 int nyb) {
    __shared__ float wsum[kScanThreads / 32];
    // the gate logits may come from the kernel before this one, and the kernels
    // before that may still read the workspace: wait for them first
    grid_dep_launch();
    grid_dep_wait();
    const int u = blockIdx.x, b = u / H, h = u % H;
    const int lane = threadIdx.x & 31, wg = threadIdx.x >> 5;
    const int t = threadIdx.x % C, w = t >> 5;                 // token and warp within the chunk
    // this unit's tokens are rows base .. base + Nu - 1; past its end the
    // decay stays flat (log gamma = 0), so a chunk's last sum is its decay
    int row0 = 0, Nu = N;
    if (cu_seqlens) packed_range(cu_seqlens, b, total, row0, Nu);
    const size_t base = cu_seqlens ? (size_t)row0 : (size_t)b * N;
    // a packed unit's chunks end with its own tokens (the kernels after this
    // one read no further), a uniform unit's at Npad
    const int nend = cu_seqlens ? min(Npad, (Nu + C - 1) / C * C) : Npad;
    // blocks of kScanThreads / C chunks, strided over the grid's y extent
    for (int by = blockIdx.y; by < nyb; by += gridDim.y) {
        if (by * kScanThreads >= nend) break;          // the same for every thread of the block
        const int ch = by * (kScanThreads / C) + threadIdx.x / C;
        const bool live = ch * C < nend;
        const int n = ch * C + t;
        float x = (live && n < Nu) ? log_gamma(z[(base + n) * H + h], inv_tau) : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[wg] = x;
        __syncthreads();
        for (int j = 0; j < w; ++j) x += wsum[wg - w + j];      // the chunk's earlier warps
        if (live) bcum[(size_t)u * Npad + n] = x;
        // block factors for the P step (p_block_factor)
        const float e = p_block_factor(x, lane, C / 4);
        if (live) eblk[(size_t)u * Npad + n] = e;
        __syncthreads();       // wsum is rewritten by the next block of chunks
    }
}

// Launch shape of the gate scan: units in x, blocks of chunks in y (at most
// the grid's y limit; the kernel strides over the rest).
static dim3 gate_scan_grid(int units, int npad, int C, int* nyb) {
    const int per = kScanThreads / C;
    *nyb = (npad / C + per - 1) / per;
    return dim3(units, *nyb < 65535 ? *nyb : 65535);
}

// Work plan of a packed batch (gret_prefill_varlen on the tensor-core path),
// made on the device from cu_seqlens.  A sequence of more than seg_max tokens
// is cut into ceil(chunks / (seg_max / C)) segments of equal chunk-multiple
// length, every head alike; the others stay whole.  The fused loop's work
// items (unit, segment) are listed longest segment first (a counting sort on
// the chunks per segment), so that the block scheduler starts the long ones
// first and no sequence finishes alone; the state pass's items are the
// segments before each split sequence's last, one slot each, numbered so that
// item i writes slot i.
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 1024;

struct PlanArgs {
    const int* cu;
    int total, S, H, C, seg_max, max_len;   // sequences are cut at max_len tokens
    int4* unit_info;        // [S * H]
    int2* fused_items;      // [max_fused]
    int2* state_items;      // [max_state]
    int* count;             // [2]: fused items, state items
    int2* seq_info;         // [S] scratch: segments, chunks per segment
    int* seq_order;         // [S] scratch: sequences, longest segments first
    int max_fused, max_state;
};

// Exclusive prefix sum of v over the block's threads; *total gets the sum.
__device__ __forceinline__ int block_exclusive_sum(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
        int t = lane < kPlanThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_sums[lane] = t;             // inclusive over warps
    }
    __syncthreads();
    const int excl = x - v + (w > 0 ? warp_sums[w - 1] : 0);
    const int tot = warp_sums[kPlanThreads / 32 - 1];
    __syncthreads();                     // warp_sums is reused by the next call
    *total = tot;
    return excl;
}

__global__ void __launch_bounds__(kPlanThreads) varlen_plan_kernel(const PlanArgs a) {
    __shared__ int offs[kPlanBuckets];
    __shared__ int warp_sums[kPlanThreads / 32];
    // the previous call's kernels may still read the plan in the workspace
    grid_dep_launch();
    grid_dep_wait();
    const int tid = threadIdx.x;
    const int maxch = a.seg_max / a.C;
    offs[tid] = 0;
    __syncthreads();
    auto bucket_of = [&](int per) { return kPlanBuckets - 1 - min(per, kPlanBuckets - 1); };
    // segments per sequence, and a histogram of chunks per segment
    for (int b = tid; b < a.S; b += kPlanThreads) {
        int row0, len;
        packed_range(a.cu, b, a.total, row0, len);
        len = min(len, a.max_len);
        const int nch = (len + a.C - 1) / a.C;
        const int P = nch > maxch ? (nch + maxch - 1) / maxch : 1;
        const int per = (nch + P - 1) / P;
        a.seq_info[b] = make_int2(P, per);
        atomicAdd(&offs[bucket_of(per)], 1);
    }
    __syncthreads();
    int tot = 0;
    const int start = block_exclusive_sum(offs[tid], warp_sums, &tot);
    offs[tid] = start;
    __syncthreads();
    for (int b = tid; b < a.S; b += kPlanThreads)
        a.seq_order[atomicAdd(&offs[bucket_of(a.seq_info[b].y)], 1)] = b;
    __syncthreads();
    // in that order: the fused items (sequence, segment, head) and, per split
    // sequence, its state slots; a block of up to kPlanThreads sequences at a
    // time, its (sequence, head) pairs spread over the threads
    __shared__ int4 blk[kPlanThreads];   // sequence, segments, first fused item, first state item
    int carry_f = 0, carry_s = 0;
    for (int r0 = 0; r0 < a.S; r0 += kPlanThreads) {
        const int r = r0 + tid;
        const int b = r < a.S ? a.seq_order[r] : -1;
        const int2 si = b >= 0 ? a.seq_info[b] : make_int2(0, 0);
        int tf = 0, ts = 0;
        const int ef = block_exclusive_sum(si.x, warp_sums, &tf) + carry_f;
        const int es = block_exclusive_sum(b >= 0 ? si.x - 1 : 0, warp_sums, &ts) + carry_s;
        blk[tid] = make_int4(b, si.x, ef, es);
        __syncthreads();
        const int nb = min(kPlanThreads, a.S - r0);
        for (int q = tid; q < nb * a.H; q += kPlanThreads) {
            const int4 e = blk[q / a.H];
            const int h = q % a.H, bq = e.x, P = e.y;
            const int u = bq * a.H + h;
            const int slot0 = e.w * a.H + h * (P - 1);
            a.unit_info[u] = make_int4(P, a.seq_info[bq].y * a.C, slot0, 0);
            for (int sg = 0; sg < P; ++sg) {
                const int it = (e.z + sg) * a.H + h;
                if (it < a.max_fused) a.fused_items[it] = make_int2(u, sg);
            }
            for (int sg = 0; sg + 1 < P; ++sg)
                if (slot0 + sg < a.max_state) a.state_items[slot0 + sg] = make_int2(u, sg);
        }
        __syncthreads();                 // blk is rewritten by the next block of sequences
        carry_f += tf;
        carry_s += ts;
    }
    if (tid == 0) {
        a.count[0] = min(carry_f * a.H, a.max_fused);
        a.count[1] = min(carry_s * a.H, a.max_state);
    }
}

// Fold the segment increments into initial states, in place:
// slot p <- S_in(p + 1) = e^{a_p} S_in(p) + dS_p, with S_in(0) = S0 (or 0).
__global__ void seg_combine_kernel(float* __restrict__ seg_state, const float* __restrict__ seg_decay,
                                   const float* __restrict__ S0, int nslots, int dk, int dv,
                                   const int4* __restrict__ unit_info, const int2* __restrict__ state_items,
                                   const int* __restrict__ plan_count) {
    grid_dep_launch();
    grid_dep_wait();       // the state pass's increments
    int u = blockIdx.x;
    const int elems4 = dk * dv / 4;
    const int e = blockIdx.y * blockDim.x + threadIdx.x;
    if (e >= elems4) return;
    // a packed batch's plan: block x is state item x, and the first segment's
    // item of each split unit folds that unit's slots (its own slot range)
    size_t base = (size_t)u * nslots;
    if (unit_info) {
        if ((int)blockIdx.x >= plan_count[1]) return;
        const int2 it = state_items[blockIdx.x];
        if (it.y != 0) return;
        u = it.x;
        const int4 ui = unit_info[u];
        nslots = ui.x - 1;
        base = (size_t)ui.z;
    }
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    if (S0) {   // slots hold S^T [dv][dk]; S0 is [dk][dv]
        const int d = (4 * e) / dk, k = (4 * e) % dk;
        const float* s0 = S0 + (size_t)u * dk * dv + (size_t)k * dv + d;
        run = make_float4(s0[0], s0[dv], s0[2 * dv], s0[3 * dv]);
    }
    for (int p = 0; p < nslots; ++p) {
        float4* slot = reinterpret_cast<float4*>(seg_state) + (base + p) * elems4 + e;
        const float f = __expf(seg_decay[base + p]);
        const float4 d = *slot;
        run = make_float4(fmaf(f, run.x, d.x), fmaf(f, run.y, d.y), fmaf(f, run.z, d.z), fmaf(f, run.w, d.w));
        *slot = run;
    }
}

// State-only pass: the pieces' increments are folded from the zero state --
// the fold through piece j is e^{a_j} (fold through piece j - 1) + slot j --
// and the last fold, S^T [DV][DK], becomes the slice's increment dS [DK][DV]
// through a shared-memory tile transpose; the pieces' log-decays sum to the
// slice's total.  The folds a resumed prefill reads, those that end a segment
// of `pieces` pieces before the last, are written back to their slots.
// One block per 32 x 32 tile of a unit's state, each thread four rows of it.
template <int DV>
__global__ void state_finish_kernel(float* __restrict__ seg_state, const float* __restrict__ seg_decay, int slots,
                                    int pieces, float* __restrict__ dS, float* __restrict__ decay) {
    __shared__ float tile[32][33];
    grid_dep_launch();
    grid_dep_wait();       // the state pass's pieces
    const int u = blockIdx.x;
    const int d0 = (blockIdx.y % (DV / 32)) * 32, k0 = (blockIdx.y / (DV / 32)) * 32;   // tile of S^T
    const int x = threadIdx.x, y = threadIdx.y;
    float run[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < slots; ++j) {
        float* src = seg_state + ((size_t)u * slots + j) * DV * DK + (size_t)d0 * DK + k0 + x;
        const float f = __expf(seg_decay[(size_t)u * slots + j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) run[i] = fmaf(f, run[i], src[(size_t)(y + 8 * i) * DK]);
        if ((j + 1) % pieces == 0 && j + 1 < slots) {
#pragma unroll
            for (int i = 0; i < 4; ++i) src[(size_t)(y + 8 * i) * DK] = run[i];
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) tile[y + 8 * i][x] = run[i];
    __syncthreads();
    float* dst = dS + (size_t)u * DK * DV;
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[(size_t)(k0 + y + 8 * i) * DV + d0 + x] = tile[x][y + 8 * i];
    if (blockIdx.y == 0 && x == 0 && y == 0) {
        float acc = 0.f;
        for (int k = 0; k < slots; ++k) acc += seg_decay[(size_t)u * slots + k];
        decay[u] = acc;
    }
}

// Prefill resumed after a state-only pass of the same tokens, whose folds from
// the zero state end each segment (`pieces` pieces) in slot seg * pieces - 1:
// each such slot j (the state after piece j, S^T layout) gains the initial
// state carried through the pieces' decays, slot_j += e^{a_0 + ... + a_j} S0
// -- the state decomposition with S0 as the state before the first piece.
__global__ void seg_shift_kernel(float* __restrict__ seg_state, const float* __restrict__ seg_decay,
                                 const float* __restrict__ S0, int slots, int pieces, int dk, int dv) {
    grid_dep_launch();
    grid_dep_wait();
    const int u = blockIdx.x;
    const int elems4 = dk * dv / 4;
    const int e = blockIdx.y * blockDim.x + threadIdx.x;
    if (e >= elems4) return;
    const int d = (4 * e) / dk, k = (4 * e) % dk;       // S^T element (d, k .. k + 3); S0 is [dk][dv]
    const float* s0 = S0 + (size_t)u * dk * dv + (size_t)k * dv + d;
    const float4 x = make_float4(s0[0], s0[dv], s0[2 * dv], s0[3 * dv]);
    float a = 0.f;
    for (int j = 0; j < slots; ++j) {
        a += seg_decay[(size_t)u * slots + j];
        if ((j + 1) % pieces != 0 || j + 1 == slots) continue;
        const float f = __expf(a);
        float4* slot = reinterpret_cast<float4*>(seg_state) + ((size_t)u * slots + j) * elems4 + e;
        float4 v = *slot;
        v = make_float4(fmaf(f, x.x, v.x), fmaf(f, x.y, v.y), fmaf(f, x.z, v.z), fmaf(f, x.w, v.w));
        *slot = v;
    }
}

// Sequence-parallel fold: S_in = e^{a_{p-1}} (... (e^{a_0} S0 + dS_0) ...) + dS_{p-1}
// over the slices before `slice`, elementwise, VW elements (float or float4)
// per thread.
__device__ __forceinline__ float fold_fma(float f, float r, float d) { return fmaf(f, r, d); }
__device__ __forceinline__ float4 fold_fma(float f, float4 r, float4 d) {
    return make_float4(fmaf(f, r.x, d.x), fmaf(f, r.y, d.y), fmaf(f, r.z, d.z), fmaf(f, r.w, d.w));
}

template <typename T>
__global__ void state_fold_kernel(const T* __restrict__ dS_all, const float* __restrict__ decay_all, int slice,
                                  const T* S0, T* S_in, int units, int nvec) {
    grid_dep_launch();
    grid_dep_wait();       // the increments may come from the kernel before this one
    const int u = blockIdx.x;
    const int e = blockIdx.y * blockDim.x + threadIdx.x;
    if (e >= nvec) return;
    const size_t at = (size_t)u * nvec + e;
    T run;
    if (S0) run = S0[at];                      // S0 may be S_in itself: read before the write
    else memset(&run, 0, sizeof(T));
    for (int q = 0; q < slice; ++q)
        run = fold_fma(__expf(decay_all[(size_t)q * units + u]), run, dS_all[(size_t)q * units * nvec + at]);
    S_in[at] = run;
}

// ---------------------------------------------------------------------------
// Fused chunk loop for 128-token chunks with d_v = 128, output held as rows.
//
// The same chunkwise form as prefill_tc_kernel, laid out the other way round
// for the output: O[t][d] sits in tensor memory with one token per lane, so the
// GroupNorm of a token is a sum along its own row and G / O move as 16-byte
// vectors, and P[t][s] feeds the intra-chunk product from tensor memory.
//   scores  D[t][s]  = Q K~^T        A = Q (smem, K-major), B = K~ (K-major)
//   inter   D[t][d]  = Q~ T           A = Q or Q~ (smem),    B = bf16 copy of T^T (smem, K-major)
//   intra   D[t][d] += P V            A = P (tensor memory, bf16), B = V (smem, MN-major)
//   state   D[d][k] += V^T K~         A = V (MN-major), B = K~ (MN-major): T^T, fp32, lanes = d
// The epilogue warps read G from a TMA-loaded tile and write the output over
// it in place; one TMA store per chunk then writes the tile to O, after which
// the tile takes the next chunk's G.
//
// Lazy chunks (the largest K scale e^{-b_s - Lambda} within e^kLazyMax) factor
// the decay: K~_s = e^{-b_s - Lambda} K_s is scaled once, before the scores, so
//   e^{-(b_t + Lambda)} Y_t = Q_t T + sum_{s <= t} (Q_t . K~_s) V_s,
// P is the masked scores alone, Q needs no scaling, and the row factor
// c_t = e^{b_t + Lambda} <= 1 enters the GroupNorm statistics in the
// epilogue; the state update T += V^T K~ uses the same K~ and Lambda += b_C.
// Eager chunks take the direct forms: P[t][s] = A[t][s] e^{b_t - b_s},
// Q~_t = e^{b_t + Lambda} Q_t against the unscaled T, then T *= e^{Lambda + b_C},
// K~_s = e^{b_C - b_s} K_s and Lambda = 0.  All exponents stay <= kLazyMax.
//
// Roles (896 threads, seven warpgroups).  Warps 0-15 (E): epilogue, four warps
// per tensor-memory lane quarter, each owning 32 of a token's 128 channels; the
// four quarters' partial sums of a token meet in spare tensor-memory columns of
// its lane (two sets, by chunk parity).  After the output of chunk i they scale
// K~ of a lazy chunk i + 2 (a quarter of a token row per thread).  Warps 16-19
// (P): masked scores -> bf16 P in tensor memory; causality leaves lane quarter
// q with q + 1 nonzero 32-column blocks, so warps 26 and 27 (lane quarters 2
// and 3) take the blocks past the second of the two heaviest quarters and no
// warp converts more than two.  The blocks above the diagonal stay zero and
// are written once.  Warps 20-23 (S): the bf16 copy of T after each state
// update, and for eager chunks the rescale of T and the scaling of Q~ and K~
// after the scores; the initial and final state.  Warp 24 lane 0 issues every
// MMA; warp 25 lane 0 every TMA load and the output store.  Per chunk the MMA
// warp issues the scores, the inter-chunk product, the state update (which
// needs neither P nor the output) and last the intra-chunk product, so that
// the tensor cores work while the P warps convert the scores; a chunk's V is
// released by its intra-chunk product, its Q and K by the state update.
constexpr int kRowsThreads = 896;
constexpr int kRowsRegs = 72;          // 65536 / 896, rounded down to 8
constexpr int kRowsSRegs = 56;         // the S warps hand registers to the P and issuing warps
constexpr int kRowsPRegs = 80;
constexpr int kRowsIssueRegs = 80;
static_assert(128 * kRowsSRegs + 128 * kRowsPRegs + 128 * kRowsIssueRegs <= 384 * kRowsRegs, "register split");

struct RowsCfg {
    static constexpr int C = 128, DV = 128;
    static constexpr int BOX = C * 128;             // one [128 rows x 64] bf16 box, 16 KB
    static constexpr int TILE = 2 * BOX;            // [128 rows x 128] bf16
    static constexpr int OFF_Q = 0;                 // 2 stages
    static constexpr int OFF_K = OFF_Q + 2 * TILE;  // 2 stages
    static constexpr int OFF_V = OFF_K + 2 * TILE;
    static constexpr int OFF_G = OFF_V + TILE;      // G
    static constexpr int OFF_T = OFF_G + TILE;      // bf16 T^T [d][k]
    static constexpr int OFF_B = OFF_T + TILE;      // per Q/K stage: C fp32 decay sums
    static constexpr int OFF_XIN = OFF_B + 2 * C * 4;   // CTA pair: the other CTA's per-token sums
    static constexpr int OFF_BAR = OFF_XIN + C * 8;
    static constexpr int NUM_BARS = 19;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int USED = OFF_MISC + 16;
    // the rest of the budget is slack for aligning the base to 1024 bytes (the
    // kernel checks that it sufficed)
    static constexpr int SMEM = kMaxSmem;
    static_assert(USED <= SMEM, "shared memory budget");
    // tensor-memory columns: O, scores, P, T^T, and the epilogue's exchange
    // (two sets of four (sum, sum of squares) pairs)
    static constexpr int TM_O = 0, TM_SC = 128, TM_P = 256, TM_T = 320, TM_X = 448, TM_ALLOC = 512;
    static_assert(TM_X + 16 <= TM_ALLOC, "tensor-memory columns");
};

// Scale the 16-byte chunks of one token row of a [128 x 128] bf16 tile (two
// 128-byte-swizzled boxes) by f; the logical chunk order spreads the 32 rows of
// a warp over all banks.
__device__ __forceinline__ void scale_tile_row(uint8_t* tile, int row, float f) {
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int c = 0; c < 8; ++c)
            scale_bf16x8(tile + x * RowsCfg::BOX + row * 128 + ((c ^ (row & 7)) << 4), f);
}

template <bool PAIR, bool PACKED>
__global__ void __launch_bounds__(kRowsThreads, 1) prefill_rows_kernel(const __grid_constant__ TcParams p) {
    using CF = RowsCfg;
    constexpr int C = CF::C, DV = CF::DV;      // DV: the output channels (and state rows) of this CTA
    constexpr int DVT = PAIR ? 2 * DV : DV;    // the unit's d_v
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (sm + CF::USED > smem_raw + CF::SMEM) {   // the base is not aligned enough: report, do nothing
        if (tid == 0) atomicExch(p.status, kDevSmemLayout);
        return;
    }
    // a CTA pair (cluster of two, consecutive blocks) shares one work item: rank r
    // owns output channels and state rows r * DV .. r * DV + DV - 1
    const int rank = PAIR ? (int)cluster_ctarank() : 0;
    const int ch0 = rank * DV;
    const int item = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    // work item: a (unit, segment) of the uniform split, or of a packed batch's
    // plan (a block past the plan's item count has nothing to do; both CTAs of a
    // pair read the same count)
    int u = 0, seg = 0, seg_len = p.seg_len;
    if constexpr (PACKED) {
        grid_dep_wait();
        if (item >= p.plan_count[0]) return;
        const int2 it = p.fused_items[item];
        u = it.x;
        seg = it.y;
        seg_len = p.unit_info[u].y;
    } else {
        u = item / p.P;
        seg = item % p.P;
    }
    // the seg_state slot of this segment's initial state (seg > 0), and whether
    // it is its unit's last segment (worked out where they are needed)
    auto in_slot = [&]() -> size_t {
        if constexpr (PACKED) return (size_t)p.unit_info[u].z + seg - 1;
        else return (size_t)u * p.slots + (size_t)seg * p.K - 1;
    };
    auto last_segment = [&]() -> bool {
        if constexpr (PACKED) return seg == p.unit_info[u].x - 1;
        else return seg == p.P - 1;
    };
    // this unit's tokens: rows row0 .. row0 + Nu - 1 of the (packed) tensors
    const int hh = u % p.H;
    int bb = u / p.H, row0 = 0, Nu = p.N;
    if constexpr (PACKED) {
        bb = 0;
        packed_range(p.cu, u / p.H, p.total, row0, Nu);
        Nu = min(Nu, p.N);                    // tokens past max_seqlen are not processed
    }
    const int n_begin = seg * seg_len;
    const int n_end = min(Nu, n_begin + seg_len);
    const int nchunks = n_end > n_begin ? (n_end - n_begin + C - 1) / C : 0;
    // rows of chunk j inside the sequence (a packed sequence's last chunk may
    // end before its 128 rows; the rest are the next sequence's)
    auto valid_rows = [&](int j) -> int { return min(C, n_end - (n_begin + j * C)); };

    // barriers; KT has one per Q/K stage so that no phase can complete twice
    // before the MMA warp has seen the first.  BG: the G tile of a chunk is in
    // (or, without G, the tile is free for the chunk's output); BGF: the
    // epilogue has written the chunk's output into the tile.
    // BXF / BXE (CTA pair): the other CTA's per-token sums are in this CTA's
    // exchange buffer / it has read the sums this CTA sent
    constexpr int BQK = 0, BV = 2, BG = 3, BSC = 4, BOD = 6, BST = 7, BKT = 8, BTC = 10, BQT = 11, BPR = 12,
                  BOF = 13, BGF = 14, BDRAIN = 15, BNEVER = 16, BXF = 17, BXE = 18;
    static_assert(BXE + 1 == CF::NUM_BARS, "barrier count");
    auto bar = [&](int i) -> uint32_t { return sb + CF::OFF_BAR + 8 * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);

    if (tid == 0) {
        for (int i = 0; i < CF::NUM_BARS; ++i) {
            // per-warp arrivals: sixteen epilogue warps, six P warps, or one
            // four-warp role
            const bool sixteen = i == BOF || i == BGF || i == BKT || i == BKT + 1;
            const bool four = i == BTC || i == BQT;
            mbar_init(bar(i), sixteen || i == BXE ? 16 : four ? 4 : i == BPR ? 6 : 1);
        }
        // the pair's exchange: armed for the first chunk's 128 pairs of sums
        if (PAIR && p.gn && nchunks > 0) mbar_arrive_expect_tx(bar(BXF), C * 8);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tmQ);
        tma_prefetch_desc(&p.tmK);
        tma_prefetch_desc(&p.tmV);
        tma_prefetch_desc(&p.tmG);
        tma_prefetch_desc(&p.tmO);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), CF::TM_ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the other CTA's barriers are initialised before either sends to them
    if constexpr (PAIR) cluster_sync_all();
    const uint32_t tm = *tmem_slot;
    grid_dep_launch();
    grid_dep_wait();

    const int role = warp >> 2;            // 0-3 E; 4 P; 5 S; 6 issuing warps
    const int q4 = warp & 3;               // tensor-memory lane quarter
    const uint32_t lq = (uint32_t)(32 * q4) << 16;
    const int row = 32 * q4 + lane;        // token t (E, P) or channel d / token row (S) of this thread
    auto warp_arrive = [&](int b) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(b));
    };
    auto stage_bc = [&](int i) -> const float* {
        return reinterpret_cast<const float*>(sm + CF::OFF_B + (i & 1) * C * 4);
    };
    // masked scores -> bf16 P for the 32-column blocks cb_lo..cb_hi of this
    // warp's lane quarter (a P warp, or a helper on the heavy quarters)
    auto p_rows = [&](int cb_lo, int cb_hi) {
        float lam = 0.f;
        for (int i = 0; i < nchunks; ++i) {
            const float* bc = stage_bc(i);
            // the scores landed (so did Q/K and bc)
            mbar_wait(bar(BSC + (i & 1)), (i >> 1) & 1, p.status, abort_flag);
            tc_fence_after();
            const float bC = bc[C - 1];
            const bool eager = (-bC - lam) > kLazyMax;
            const float bt = bc[row];
#pragma unroll 1
            for (int cb = cb_lo; cb <= cb_hi; ++cb) {
                uint32_t r[32], pk[16];
                tmem_ld_x32(tm + lq + CF::TM_SC + cb * 32, r);
                // a lazy chunk's column factors e^{-b_s - Lambda} (<= e^kLazyMax), one
                // per lane, shared by shuffles; the scores are Q K^T of the raw K
                const float cf = __expf(-bc[cb * 32 + lane] - lam);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int s0 = cb * 32 + 2 * j;
                    float v0 = u2f(r[2 * j]), v1 = u2f(r[2 * j + 1]);
                    if (eager) {
                        v0 *= __expf(fminf(bt - bc[s0], 0.f));
                        v1 *= __expf(fminf(bt - bc[s0 + 1], 0.f));
                    } else {
                        v0 *= __shfl_sync(0xffffffffu, cf, 2 * j);
                        v1 *= __shfl_sync(0xffffffffu, cf, 2 * j + 1);
                    }
                    pk[j] = pack_bf16x2(s0 <= row ? v0 : 0.f, s0 + 1 <= row ? v1 : 0.f);
                }
                tmem_st_x16(tm + lq + CF::TM_P + cb * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(BPR);
            lam = eager ? 0.f : lam + bC;
        }
    };

    if (role == 6) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" : : "n"(kRowsIssueRegs));
        if (warp == 25 && lane == 0 && nchunks > 0) {
            // ======================================================== TMA producer
            int last_qk[2] = {-1, -1}, last_v = -1, last_g = -1;
            auto issue_qk = [&](int j) {
                // n0: the chunk's first token within its unit (the decay sums are
                // per unit); row0 + n0: its row in the (packed) tensors
                const int s = j & 1, n0 = n_begin + j * C;
                last_qk[s] = j;
                const uint32_t fb = bar(BQK + s);
                mbar_arrive_expect_tx(fb, 2 * CF::TILE + C * 4);
                for (int x = 0; x < 2; ++x) {
                    tma_load_4d(sb + CF::OFF_Q + s * CF::TILE + x * CF::BOX, &p.tmQ, x * 64, hh, row0 + n0, bb, fb);
                    tma_load_4d(sb + CF::OFF_K + s * CF::TILE + x * CF::BOX, &p.tmK, x * 64, hh, row0 + n0, bb, fb);
                }
                bulk_load(sb + CF::OFF_B + s * C * 4, p.bcum + (size_t)u * p.Npad + n0, C * 4, fb);
            };
            auto issue_v = [&](int j) {
                last_v = j;
                mbar_arrive_expect_tx(bar(BV), CF::TILE);
                for (int x = 0; x < 2; ++x)
                    tma_load_4d(sb + CF::OFF_V + x * CF::BOX, &p.tmV, ch0 + x * 64, hh, row0 + n_begin + j * C, bb,
                                bar(BV));
            };
            // the tile of chunk j: its G, or (without G) a plain release for its output
            auto issue_g = [&](int j) {
                if (!p.has_g) {
                    mbar_arrive(bar(BG));
                    return;
                }
                last_g = j;
                mbar_arrive_expect_tx(bar(BG), CF::TILE);
                for (int x = 0; x < 2; ++x)
                    tma_load_4d(sb + CF::OFF_G + x * CF::BOX, &p.tmG, ch0 + x * 64, hh, row0 + n_begin + j * C, bb,
                                bar(BG));
            };
            if (p.fault) mbar_wait_injected_timeout(bar(BNEVER), p.status, abort_flag);
            if (!*abort_flag) {
                issue_qk(0);
                if (nchunks > 1) issue_qk(1);
                issue_v(0);
                issue_g(0);
                for (int i = 0; i < nchunks; ++i) {
                    // the state MMA of chunk i is the last reader of its Q/K stage and of V
                    if (!mbar_wait(bar(BST), i & 1, p.status, abort_flag)) break;
                    if (i + 2 < nchunks) issue_qk(i + 2);
                    if (i + 1 < nchunks) issue_v(i + 1);
                    // the output of chunk i leaves from the tile (rows past the end of
                    // the tensors fall outside the map and are not written; a packed
                    // sequence's short last chunk was stored row by row by the
                    // epilogue); once the store has read the tile it takes chunk i + 1
                    if (!mbar_wait(bar(BGF), i & 1, p.status, abort_flag)) break;
                    if (!PACKED || valid_rows(i) == C) {
                        for (int x = 0; x < 2; ++x)
                            tma_store_4d(&p.tmO, sb + CF::OFF_G + x * CF::BOX, ch0 + x * 64, hh, row0 + n_begin + i * C,
                                         bb);
                        bulk_commit();
                        bulk_wait_read<0>();
                    }
                    if (i + 1 < nchunks) issue_g(i + 1);
                }
            }
            bulk_wait<0>();
            if (*abort_flag) {
                for (int x = 0; x < 2; ++x)
                    if (last_qk[x] >= 0) mbar_wait_drain(bar(BQK + x), (last_qk[x] >> 1) & 1, kWaitCycles);
                if (last_v >= 0) mbar_wait_drain(bar(BV), last_v & 1, kWaitCycles);
                if (last_g >= 0) mbar_wait_drain(bar(BG), last_g & 1, kWaitCycles);
            }
        } else if (warp == 24 && lane == 0 && nchunks > 0) {
            // ======================================================== MMA issuer
            constexpr uint32_t id_kk = idesc_bf16(128, 128, false, false);   // scores, inter
            constexpr uint32_t id_pv = idesc_bf16(128, 128, false, true);    // intra: B = V MN-major
            constexpr uint32_t id_kv = idesc_bf16(128, 128, true, true);     // state
            float lam = 0.f;
            int neager = 0;         // eager chunks so far: BQT completes once per eager chunk
            for (int i = 0; i < nchunks; ++i) {
                const int s = i & 1;
                const uint32_t sQ = sb + CF::OFF_Q + s * CF::TILE, sK = sb + CF::OFF_K + s * CF::TILE;
                const uint32_t sV = sb + CF::OFF_V, sT = sb + CF::OFF_T;
                if (!mbar_wait(bar(BQK + s), (i >> 1) & 1, p.status, abort_flag)) break;
                const float bC = stage_bc(i)[C - 1];
                const bool eager = (-bC - lam) > kLazyMax;
                // scores of the raw Q and K, once P of the previous chunk has left the
                // score buffer (the intra-chunk product waited for it)
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = (k >> 2) * CF::BOX + (k & 3) * 32;
                    mma_ss(tm + CF::TM_SC, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), id_kk,
                           k > 0);
                }
                mma_commit(bar(BSC + s));
                // inter-chunk: O = Q T (lazy) or Q~ T (eager), once the bf16 copy of T
                // is ready and the epilogue has taken the previous output
                if (!mbar_wait(bar(BTC), i & 1, p.status, abort_flag)) break;
                if (eager && !mbar_wait(bar(BQT), neager & 1, p.status, abort_flag)) break;
                neager += eager ? 1 : 0;
                if (i > 0 && !mbar_wait(bar(BOF), (i - 1) & 1, p.status, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = (k >> 2) * CF::BOX + (k & 3) * 32;
                    mma_ss(tm + CF::TM_O, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sT + off, 16, 1024), id_kk,
                           k > 0);
                }
                // intra-chunk: O += P V
                if (!mbar_wait(bar(BPR), i & 1, p.status, abort_flag)) break;
                if (!mbar_wait(bar(BV), i & 1, p.status, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_ts(tm + CF::TM_O, tm + CF::TM_P + k * 8, sdesc_sw128(sV + k * 2048, CF::BOX, 1024), id_pv, 1);
                mma_commit(bar(BOD));
                // state: T^T += V^T K~, once the epilogue warps have scaled K~ in place
                // (after the scores read the raw K)
                if (!mbar_wait(bar(BKT + s), (i >> 1) & 1, p.status, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_ss(tm + CF::TM_T, sdesc_sw128(sV + k * 2048, CF::BOX, 1024),
                           sdesc_sw128(sK + k * 2048, CF::BOX, 1024), id_kv, 1);
                mma_commit(bar(BST));
                lam = eager ? 0.f : lam + bC;
            }
            // every MMA this thread issued has completed before tensor memory is freed
            mma_commit(bar(BDRAIN));
            mbar_wait_drain(bar(BDRAIN), 0, kWaitCycles);
        } else if (warp >= 26) {
            // helpers on lane quarters 2 and 3: blocks 2..q4
            p_rows(2, q4);
        }
    } else if (role == 5) {
        // ============================================================ S warps
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" : : "n"(kRowsSRegs));
        // initial state T^T[d][k] (lane d = row): zero, a caller's S0 [k][d], or a
        // segment's folded state [d][k]
        {
            uint32_t r[32];
            for (int cb = 0; cb < 4; ++cb) {
                if (seg > 0) {
                    const float4* s4 = reinterpret_cast<const float4*>(
                        p.seg_state + in_slot() * DVT * DK +
                        (size_t)(ch0 + row) * DK + cb * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 v = s4[j];
                        r[4 * j] = f2u(v.x); r[4 * j + 1] = f2u(v.y); r[4 * j + 2] = f2u(v.z); r[4 * j + 3] = f2u(v.w);
                    }
                } else if (p.S0) {
                    const float* src = p.S0 + (size_t)u * DK * DVT + (size_t)(cb * 32) * DVT + ch0 + row;
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = f2u(src[(size_t)j * DVT]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = 0u;
                }
                tmem_st_x32(tm + lq + CF::TM_T + cb * 32, r);
            }
            tmem_wait_st();
        }
        float lam = 0.f;
        for (int i = 0; i < nchunks; ++i) {
            const int s = i & 1;
            const float* bc = stage_bc(i);
            uint8_t* Qp = sm + CF::OFF_Q + s * CF::TILE;
            mbar_wait(bar(BQK + s), (i >> 1) & 1, p.status, abort_flag);
            const float bC = bc[C - 1];
            const bool eager = (-bC - lam) > kLazyMax;
            const float brow = bc[row];
            // bf16 copy of T^T for this chunk's inter-chunk product, once the
            // previous state update is done (it also finished the previous
            // inter-chunk product, the last reader of the copy); eager chunks
            // then rescale T for their state update
            if (i > 0) mbar_wait(bar(BST), (i - 1) & 1, p.status, abort_flag);
            tc_fence_after();
            const float escale = __expf(lam + bC);
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[32];
                tmem_ld_x32(tm + lq + CF::TM_T + cb * 32, r);
                tmem_wait_ld();
                uint8_t* trow = sm + CF::OFF_T + (cb >> 1) * CF::BOX + row * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int chunk = (cb & 1) * 4 + c;        // 16-byte chunk of the 128-byte row
                    uint4 w;
                    w.x = pack_bf16x2(u2f(r[8 * c]), u2f(r[8 * c + 1]));
                    w.y = pack_bf16x2(u2f(r[8 * c + 2]), u2f(r[8 * c + 3]));
                    w.z = pack_bf16x2(u2f(r[8 * c + 4]), u2f(r[8 * c + 5]));
                    w.w = pack_bf16x2(u2f(r[8 * c + 6]), u2f(r[8 * c + 7]));
                    *reinterpret_cast<uint4*>(trow + ((chunk ^ (row & 7)) << 4)) = w;
                }
                if (eager) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = f2u(u2f(r[j]) * escale);
                    tmem_st_x32(tm + lq + CF::TM_T + cb * 32, r);
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(BTC);
            if (eager) {
                // Q~ in place, once the scores have read Q (K~ is the E warps')
                mbar_wait(bar(BSC + s), (i >> 1) & 1, p.status, abort_flag);
                tc_fence_after();
                scale_tile_row(Qp, row, __expf(brow + lam));
                fence_proxy_async_smem();
                warp_arrive(BQT);
            }
            lam = eager ? 0.f : lam + bC;
        }
        // state out: e^Lambda T
        if (nchunks > 0) {
            mbar_wait(bar(BST), (nchunks - 1) & 1, p.status, abort_flag);
            tc_fence_after();
        }
        if (p.S_final && last_segment()) {
            const float sc = __expf(lam);
            float* dst = p.S_final + (size_t)u * DK * DVT + ch0;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[32];
                tmem_ld_x32(tm + lq + CF::TM_T + cb * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) dst[(size_t)(cb * 32 + j) * DVT + row] = u2f(r[j]) * sc;
            }
        }
    } else if (role == 4) {
        // ============================================================ P warps
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" : : "n"(kRowsPRegs));
        // the blocks above the diagonal, once
        {
            uint32_t z[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) z[j] = 0u;
            for (int cb = q4 + 1; cb < 4; ++cb) tmem_st_x16(tm + lq + CF::TM_P + cb * 16, z);
            tmem_wait_st();
        }
        p_rows(0, min(q4, 1));
    } else {
        // ============================================================ E warps
        const int hf = role;                       // which 32 channels of the token
        constexpr int QC = DV / 4;
        float lam = 0.f;
        const float* bsum = p.bcum + (size_t)u * p.Npad;
        // K~ of chunk j in place for its state update, once its scores have read
        // the raw K: e^{-b_s - Lambda} K_s (lazy) or e^{b_C - b_s} K_s (eager);
        // token row tid % 128, its 16-byte words 4 (tid / 128) .. + 3.  Chunks
        // are taken in order, so Lambda follows them.
        float lam_k = 0.f;
        auto scale_k = [&](int j) {
            const int s = j & 1, kr = tid & (C - 1), part = tid >> 7;
            const float* bc = stage_bc(j);
            mbar_wait(bar(BSC + s), (j >> 1) & 1, p.status, abort_flag);
            const float bCj = bc[C - 1];
            const bool eg = (-bCj - lam_k) > kLazyMax;
            // rows past the sequence's end (a packed batch's next sequence) add nothing
            const float f = kr < valid_rows(j) ? __expf(eg ? bCj - bc[kr] : -bc[kr] - lam_k) : 0.f;
            uint8_t* krow = sm + CF::OFF_K + s * CF::TILE + (part >> 1) * CF::BOX + kr * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) scale_bf16x8(krow + ((((part & 1) * 4 + c) ^ (kr & 7)) << 4), f);
            fence_proxy_async_smem();
            warp_arrive(BKT + s);
            lam_k = eg ? 0.f : lam_k + bCj;
        };
        for (int i = 0; i < nchunks; ++i) {
            scale_k(i);
            const int n0 = n_begin + i * C;
            const float bt = bsum[n0 + row], bC = bsum[n0 + C - 1];
            mbar_wait(bar(BOD), i & 1, p.status, abort_flag);
            tc_fence_after();
            uint32_t y[QC];
            tmem_ld_x32(tm + lq + CF::TM_O + hf * QC, y);
            tmem_wait_ld();
            tc_fence_before();
            warp_arrive(BOF);              // the next inter-chunk product may overwrite O
            const bool eager = (-bC - lam) > kLazyMax;
            // row factor c = e^{b_t + Lambda} of a lazy chunk; y = c u
            const float c = eager ? 1.f : __expf(bt + lam);
            float a = c, b0 = 0.f;
            if (p.gn) {
                // sums of u and of y^2 = (c u)^2 over this quarter (u itself may be
                // as large as e^64 y), then the token's four quarters through
                // spare tensor-memory columns of its lane (the set alternates with
                // the chunk, so a set is rewritten only after every quarter has
                // passed the next chunk's barrier, i.e. read this one)
                float s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int j = 0; j < QC; ++j) {
                    const float v = u2f(y[j]);
                    s1 += v;
                    const float yc = v * c;
                    s2 = fmaf(yc, yc, s2);
                }
                const uint32_t xs = tm + lq + CF::TM_X + 8 * (i & 1);
                const uint32_t mine[2] = {f2u(s1), f2u(s2)};
                tmem_st_x2(xs + 2 * hf, mine);
                tmem_wait_st();
                tc_fence_before();
                named_bar_sync(1 + q4, 128);
                tc_fence_after();
                uint32_t all[8];
                tmem_ld_x8(xs, all);
                tmem_wait_ld();
                float t1 = (u2f(all[0]) + u2f(all[2])) + (u2f(all[4]) + u2f(all[6]));
                float t2 = (u2f(all[1]) + u2f(all[3])) + (u2f(all[5]) + u2f(all[7]));
                if constexpr (PAIR) {
                    // the token's other 128 channels are the other CTA's: the first
                    // warp of each lane quarter sends this CTA's sums into the other's
                    // exchange buffer (once it has read the previous chunk's) with
                    // asynchronous stores that complete the transaction count of the
                    // other's BXF; every warp then reads the other's sums from its own
                    // buffer and says so.  Thread 0 arms BXF for the next chunk (1 KB)
                    // once it has seen this chunk's phase complete.
                    const uint32_t other = (uint32_t)(rank ^ 1);
                    if (hf == 0) {
                        if (i > 0) mbar_wait_cluster(bar(BXE), (i - 1) & 1, p.status, abort_flag);
                        st_async_f2(cluster_map(sb + CF::OFF_XIN + row * 8, other), cluster_map(bar(BXF), other),
                                    t1, t2);
                    }
                    mbar_wait_cluster(bar(BXF), i & 1, p.status, abort_flag);
                    if (tid == 0 && i + 1 < nchunks) mbar_arrive_expect_tx(bar(BXF), C * 8);
                    const float2 o = *reinterpret_cast<const float2*>(sm + CF::OFF_XIN + row * 8);
                    t1 += o.x;
                    t2 += o.y;
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote_relaxed(cluster_map(bar(BXE), other));
                }
                const float mean_u = t1 * (1.0f / DVT);
                const float mean_y = mean_u * c;
                const float var = fmaxf(t2 * (1.0f / DVT) - mean_y * mean_y, 0.f);
                a = c * rsqrtf(var + p.eps);
                b0 = -mean_u * a;
            }
            // this token's 32 output channels go over its G in the tile; a packed
            // sequence's short last chunk is stored row by row instead (the rows
            // after it are the next sequence's)
            mbar_wait(bar(BG), i & 1, p.status, abort_flag);
            uint8_t* grow = sm + CF::OFF_G + (hf >> 1) * CF::BOX + row * 128;
            const bool direct = PACKED && valid_rows(i) < C;
            uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.O) +
                                                   ((size_t)(row0 + n0 + row) * p.H + hh) * DVT + ch0 + hf * QC);
            const bool live = row < valid_rows(i);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint4* slot = reinterpret_cast<uint4*>(grow + ((((hf & 1) * 4 + ch) ^ (row & 7)) << 4));
                uint4 w = p.has_g ? *slot : make_uint4(0u, 0u, 0u, 0u);
                uint32_t* e = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float o0 = fmaf(u2f(y[ch * 8 + 2 * j]), a, b0), o1 = fmaf(u2f(y[ch * 8 + 2 * j + 1]), a, b0);
                    if (p.gn) {
                        const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e[j]));
                        o0 *= swish_fast(g.x);
                        o1 *= swish_fast(g.y);
                    }
                    e[j] = pack_bf16x2(o0, o1);
                }
                *slot = w;
                if (direct && live) orow[ch] = w;
            }
            fence_proxy_async_smem();
            warp_arrive(BGF);              // the tile holds this chunk's output
            lam = eager ? 0.f : lam + bC;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, CF::TM_ALLOC);
    }
    // neither CTA of a pair leaves while the other may still send to it
    if constexpr (PAIR) {
        __syncwarp();
        cluster_sync_all();
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
    size_t bcum, eblk, state, decay, total;
};

WsLayout ws_layout(int B, int H, int N, int dk, int dv, int chunk, int segments, int pieces) {
    const size_t units = (size_t)B * H;
    const size_t npad = (size_t)((N + chunk - 1) / chunk) * chunk;
    WsLayout w;
    w.bcum = 0;
    w.eblk = align256(units * npad * 4);
    w.state = w.eblk + align256(units * npad * 4);
    const size_t slots = segments > 1 ? (size_t)(segments - 1) * pieces : 0;
    w.decay = w.state + align256(units * slots * (size_t)dk * dv * 4);
    w.total = w.decay + align256(units * slots * 4);
    return w;
}

// Workspace of a packed batch on the tensor-core path: decay sums, the state
// pass's slots (at most max_state), and the plan.  seg_max is one and a half
// times one work slot's share of the batch's token-heads (at least four
// chunks): a sequence is cut only when it is much longer than that share, since
// the state pass over the segments before its last re-reads their K and V (about
// 0.37 of the bytes a prefill moves) and adds two launches, which costs more than
// the imbalance of a longest-first order whose longest item is up to 1.5 shares.
// The item bounds follow from
// sum over sequences of ceil(chunks / (seg_max / C)) <= S + (total / C + S) / (seg_max / C).
struct VarlenLayout {
    size_t bcum, eblk, state, decay, unit_info, fused, sitems, count, seq_info, seq_order, total;
    int seg_max, max_fused, max_state, npad;
};

VarlenLayout varlen_layout(int S, int H, int max_seqlen, int total, int dk, int dv, int chunk, int num_sms) {
    VarlenLayout w;
    const long long units = (long long)S * H;
    // concurrent work items: one per SM, or per pair of SMs for the d_v = 256 pair
    const long long slots = std::max<long long>(1, num_sms / prefill_tc_ctas_per_item(dv, chunk));
    const long long share = (3LL * total * H + 2LL * slots - 1) / (2LL * slots);
    long long seg_max = (share + chunk - 1) / chunk * chunk;
    if (seg_max < 4LL * chunk) seg_max = 4LL * chunk;
    if (seg_max > (1LL << 30)) seg_max = (1LL << 30) / chunk * chunk;
    const long long maxch = seg_max / chunk;
    const long long chunks_bound = ((long long)total + chunk - 1) / chunk + S;
    const long long long_bound = (chunks_bound + maxch - 1) / maxch;
    w.seg_max = (int)seg_max;
    w.max_fused = (int)std::min<long long>((long long)H * (S + long_bound), 1LL << 30);
    w.max_state = (int)std::min<long long>((long long)H * long_bound, 1LL << 30);
    w.npad = (max_seqlen + chunk - 1) / chunk * chunk;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
    w.bcum = take((size_t)units * w.npad * 4);
    w.eblk = take((size_t)units * w.npad * 4);
    w.state = take((size_t)w.max_state * dk * dv * 4);
    w.decay = take((size_t)w.max_state * 4);
    w.unit_info = take((size_t)units * 16);
    w.fused = take((size_t)w.max_fused * 8);
    w.sitems = take((size_t)w.max_state * 8);
    w.count = take(16);
    w.seq_info = take((size_t)S * 8);
    w.seq_order = take((size_t)S * 4);
    w.total = off;
    return w;
}

// Launch with programmatic stream serialisation: the kernel may start while the
// one before it in the stream finishes; each kernel waits (grid_dep_wait)
// before it touches what the earlier ones wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#ifndef GRET_ROWS_KERNEL
#define GRET_ROWS_KERNEL 1
#endif

// Launch with programmatic stream serialisation and clusters of two CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_pair(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Chunk loop over a uniform batch, or a packed batch's plan.  128-token chunks
// of d_v 128 or 256 (bf16) run the output-rows kernel (a CTA pair for 256),
// the others prefill_tc_kernel.
template <int DV, int C, bool PACKED>
cudaError_t run_tc(const PrefillArgs& a, TcParams& tp, cudaStream_t s, const PlanArgs* plan = nullptr) {
    constexpr bool ROWS = C == 128 && (DV == 128 || DV == 256) && GRET_ROWS_KERNEL;
    auto ks = prefill_state_kernel<DV, C, PACKED>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        if constexpr (!ROWS) {
            // the register split inside the fused kernel draws on the registers it
            // was launched with: never launch a build that has fewer
            auto kf = prefill_tc_kernel<DV, C, PACKED>;
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, kf) != cudaSuccess) return cudaErrorInvalidDeviceFunction;
            if (fa.numRegs * kFusedThreads < 4 * 128 * kComputeRegs + 128 * kIssueRegs)
                return cudaErrorInvalidConfiguration;
            cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<DV, C>::SMEM);
        } else {
            auto kr = prefill_rows_kernel<DV == 256, PACKED>;
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, kr) != cudaSuccess) return cudaErrorInvalidDeviceFunction;
            if (fa.numRegs > kRowsRegs) return cudaErrorInvalidConfiguration;
            cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, RowsCfg::SMEM);
        }
        cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, StateCfg<DV, C>::SMEM);
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    const int units = a.B * a.H;
    const int npad = tp.Npad;
    cudaError_t e = cudaSuccess;
    if constexpr (PACKED) {
        // gate scan, plan, state pass and combine over the plan's slots, fused loop
        int nyb = 0;
        const dim3 sgrid = gate_scan_grid(units, npad, C, &nyb);
        if (g_profile_gate_start) cudaEventRecord(g_profile_gate_start, s);
        e = launch_pdl(gate_scan_kernel, sgrid, dim3(kScanThreads), 0, s, a.z, a.cu_seqlens, a.total,
                       const_cast<float*>(tp.bcum), const_cast<float*>(tp.eblk), a.H, a.N, npad, C, a.inv_tau, nyb);
        if (g_profile_gate_stop) cudaEventRecord(g_profile_gate_stop, s);
        if (e != cudaSuccess) return e;
        e = launch_pdl(varlen_plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, *plan);
        if (e != cudaSuccess) return e;
        // a sequence is cut only when longer than seg_max (the plan clamps
        // lengths to max_len): otherwise there is no state pass to run
        if (plan->max_len > plan->seg_max) {
            e = launch_pdl(ks, dim3(plan->max_state), dim3(kStateThreads), StateCfg<DV, C>::SMEM, s, tp);
            if (e != cudaSuccess) return e;
            const int elems4 = DV * DK / 4;
            e = launch_pdl(seg_combine_kernel, dim3(plan->max_state, (elems4 + 255) / 256), dim3(256), 0, s,
                           tp.seg_state, static_cast<const float*>(tp.seg_decay), tp.S0, 0, DK, DV, tp.unit_info,
                           tp.state_items, tp.plan_count);
            if (e != cudaSuccess) return e;
        }
        if (g_profile_start) cudaEventRecord(g_profile_start, s);
        if constexpr (ROWS) {
            auto kr = prefill_rows_kernel<DV == 256, true>;
            if constexpr (DV == 256)
                e = launch_pdl_pair(kr, dim3(2 * plan->max_fused), dim3(kRowsThreads), RowsCfg::SMEM, s, tp);
            else
                e = launch_pdl(kr, dim3(plan->max_fused), dim3(kRowsThreads), RowsCfg::SMEM, s, tp);
        } else {
            e = launch_pdl(prefill_tc_kernel<DV, C, PACKED>, dim3(plan->max_fused), dim3(kFusedThreads),
                           Cfg<DV, C>::SMEM, s, tp);
        }
        if (g_profile_stop) cudaEventRecord(g_profile_stop, s);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    if (a.resume) {
        // the gate scan and the state pass ran in gret_prefill_state: shift its
        // folded slots by the initial state, then the fused loop
        if (tp.P > 1 && tp.S0) {
            const int elems4 = DV * DK / 4;
            e = launch_pdl(seg_shift_kernel, dim3(units, (elems4 + 255) / 256), dim3(256), 0, s, tp.seg_state,
                           static_cast<const float*>(tp.seg_decay), tp.S0, tp.slots, tp.K, DK, DV);
        }
    } else if (a.X) {
        // gate logits from the projection z = X W_gamma, fused with the scan
        const WsLayout w = ws_layout(a.B, a.H, a.N, a.dk, a.dv, C, a.segments, a.pieces);
        e = launch_gate_project_tc(a, const_cast<float*>(tp.bcum), const_cast<float*>(tp.eblk), npad,
                                   static_cast<uint8_t*>(a.workspace) + w.total, s);
    } else {
        int nyb = 0;
        const dim3 sgrid = gate_scan_grid(units, npad, C, &nyb);
        if (g_profile_gate_start) cudaEventRecord(g_profile_gate_start, s);
        e = launch_pdl(gate_scan_kernel, sgrid, dim3(kScanThreads), 0, s, a.z, a.cu_seqlens, a.total,
                       const_cast<float*>(tp.bcum), const_cast<float*>(tp.eblk), a.H, a.N, npad, C, a.inv_tau, nyb);
        if (g_profile_gate_stop) cudaEventRecord(g_profile_gate_stop, s);
    }
    if (e != cudaSuccess) return e;
    if (tp.P > 1 && !a.resume) {
        e = launch_pdl(ks, dim3(units * tp.slots), dim3(kStateThreads), StateCfg<DV, C>::SMEM, s, tp);
        if (e != cudaSuccess) return e;
        const int elems4 = DV * DK / 4;
        e = launch_pdl(seg_combine_kernel, dim3(units, (elems4 + 255) / 256), dim3(256), 0, s, tp.seg_state,
                       static_cast<const float*>(tp.seg_decay), tp.S0, tp.slots, DK, DV,
                       static_cast<const int4*>(nullptr), static_cast<const int2*>(nullptr),
                       static_cast<const int*>(nullptr));
        if (e != cudaSuccess) return e;
    }
    if constexpr (ROWS) {
        // 128-token chunks: the output-rows kernel (d_v 256: a pair of CTAs per
        // work item, each owning half of the channels)
        auto kr = prefill_rows_kernel<DV == 256, false>;
        if (g_profile_start) cudaEventRecord(g_profile_start, s);
        if constexpr (DV == 256)
            e = launch_pdl_pair(kr, dim3(2 * units * tp.P), dim3(kRowsThreads), RowsCfg::SMEM, s, tp);
        else
            e = launch_pdl(kr, dim3(units * tp.P), dim3(kRowsThreads), RowsCfg::SMEM, s, tp);
        if (g_profile_stop) cudaEventRecord(g_profile_stop, s);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    } else {
        auto kf = prefill_tc_kernel<DV, C, PACKED>;
        if (g_profile_start) cudaEventRecord(g_profile_start, s);
        e = launch_pdl(kf, dim3(units * tp.P), dim3(kFusedThreads), Cfg<DV, C>::SMEM, s, tp);
        if (g_profile_stop) cudaEventRecord(g_profile_stop, s);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
}

}  // namespace

bool prefill_tc_supported(int dk, int dv, int chunk, gret_dtype io) {
    if (io != GRET_BF16 || dk != DK) return false;
    return (dv == 128 && (chunk == 64 || chunk == 128)) || (dv == 256 && (chunk == 64 || chunk == 128));
}

// CTAs of one fused work item: the output-rows kernel for d_v = 256 is a pair.
int prefill_tc_ctas_per_item(int dv, int chunk) { return dv == 256 && chunk == 128 ? 2 : 1; }

// State-pass pieces of a split that leaves SMs idle with one piece per segment
// but would need a second wave with two equal ones (units * (P - 1) segments,
// between half the SMs and all of them): each segment is cut into a long piece
// of a chunks and a short one of b, a = k b, where k is the number of short
// pieces each remaining SM takes one after the other.  Returns a (0: no such cut).
static int uneven_piece_split(long long units, int segments, int per, int num_sms) {
    const long long n = units * (segments - 1);
    if (segments < 2 || per < 3 || n >= num_sms || 2 * n <= num_sms) return 0;
    const long long spare = num_sms - n;
    const long long k = (n + spare - 1) / spare;
    const int b = (int)(per / (k + 1));
    return b >= 1 ? per - b : 0;
}

int prefill_tc_piece_split(int B, int H, int chunk, int num_sms, int segments, int seg_len, int pieces) {
    const long long units = (long long)B * H;
    const int per = seg_len / chunk;
    if (pieces != 2 || segments < 2 || units < 1) return 0;
    const long long kmax = num_sms / (units * (segments - 1));
    if (kmax >= 2 && per % 2 == 0) return 0;                 // two equal pieces fit one wave
    return uneven_piece_split(units, segments, per, num_sms);
}

// Segments: about one fused CTA per SM.  State-pass pieces: each of the first
// P-1 segments is cut into K pieces (K divides the segment's chunk count) so
// that the state pass, too, has about one CTA per SM; where one piece per
// segment would leave SMs idle and two equal ones need a second wave, a long and
// a short piece (uneven_piece_split).
void prefill_tc_plan(int B, int H, int N, int chunk, int num_sms, int* segments, int* seg_len, int* pieces,
                     int ctas_per_item) {
    const int units = B * H > 0 ? B * H : 1;
    const int nchunks = (N + chunk - 1) / chunk;
    int P = num_sms / (units * (ctas_per_item > 1 ? ctas_per_item : 1));
    if (P < 1) P = 1;
    if (P > nchunks) P = nchunks;
    const int per = (nchunks + P - 1) / P;
    *seg_len = per * chunk;
    *segments = (nchunks + per - 1) / per;
    int K = 1;
    if (*segments > 1) {
        const int kmax = num_sms / (units * (*segments - 1));
        for (int k = kmax < per ? kmax : per; k >= 1; --k)
            if (per % k == 0) { K = k; break; }
        if (K == 1 && uneven_piece_split(units, *segments, per, num_sms) > 0) K = 2;
    }
    *pieces = K;
}

// Kernel launches of one call: gate scan and fused loop, plus the state pass
// and the combine for a split sequence.
int prefill_tc_launches(int segments, int pieces) {
    (void)pieces;
    return segments <= 1 ? 2 : 4;
}

// State-only pass (gret_prefill_state): it follows the prefill's own plan --
// P segments of seg_len tokens -- and cuts every segment into the same number
// of pieces (about one CTA per SM; the count divides the segment's chunks),
// so that a prefill resumed on the same tokens (gret_prefill_resume) finds the
// state before each of its segments among the folded pieces.
int prefill_tc_state_pieces(int B, int H, int chunk, int num_sms, int segments, int seg_len) {
    const int units = B * H > 0 ? B * H : 1;
    const int per = seg_len / chunk;
    int kmax = num_sms / (units * (segments > 0 ? segments : 1));
    if (kmax < 1) kmax = 1;
    for (int k = kmax < per ? kmax : per; k >= 1; --k)
        if (per % k == 0) return k;
    return 1;
}

size_t prefill_tc_state_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk, int num_sms) {
    int P = 1, seg_len = N, K = 1;
    prefill_tc_plan(B, H, N, chunk, num_sms, &P, &seg_len, &K, prefill_tc_ctas_per_item(dv, chunk));
    const int Ks = prefill_tc_state_pieces(B, H, chunk, num_sms, P, seg_len);
    return ws_layout(B, H, N, dk, dv, chunk, P + 1, Ks).total;
}

size_t prefill_tc_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk, int segments, int pieces) {
    return ws_layout(B, H, N, dk, dv, chunk, segments, pieces).total;
}

size_t prefill_tc_varlen_workspace_bytes(int S, int H, int max_seqlen, int total, int dk, int dv, int chunk,
                                         int num_sms) {
    return varlen_layout(S, H, max_seqlen, total, dk, dv, chunk, num_sms).total;
}

int prefill_tc_varlen_launches(int S, int H, int max_seqlen, int total, int dk, int dv, int chunk, int num_sms) {
    return max_seqlen > varlen_layout(S, H, max_seqlen, total, dk, dv, chunk, num_sms).seg_max ? 5 : 3;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
    TcParams tp;
    memset(&tp, 0, sizeof(tp));
    const int C = a.chunk;
    // a packed batch is one [total][H][d] tensor: (d, H, total, 1) maps, each
    // unit addressing its own rows
    const int mN = a.cu_seqlens ? a.total : a.N, mB = a.cu_seqlens ? 1 : a.B;
    if (!make_map(&tp.tmQ, a.Q, DK, a.H, mN, mB, C) || !make_map(&tp.tmK, a.K, DK, a.H, mN, mB, C) ||
        !make_map(&tp.tmV, a.V, a.dv, a.H, mN, mB, C) || !make_map(&tp.tmO, a.O, a.dv, a.H, mN, mB, C) ||
        !make_map(&tp.tmG, a.G ? a.G : a.O, a.dv, a.H, mN, mB, C) ||
        !make_map(&tp.tmKs, a.K, DK, a.H, mN, mB, state_sub(a.dv, C)) ||
        !make_map(&tp.tmVs, a.V, a.dv, a.H, mN, mB, state_sub(a.dv, C)))
        return cudaErrorInvalidValue;
    tp.cu = a.cu_seqlens;
    tp.total = a.total;
    tp.O = a.O;
    tp.G = a.G;
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    PlanArgs plan;
    memset(&plan, 0, sizeof(plan));
    if (a.cu_seqlens) {
        // a packed batch works from the plan its own kernel makes
        const VarlenLayout v = varlen_layout(a.B, a.H, a.N, a.total, a.dk, a.dv, C, a.num_sms);
        tp.bcum = reinterpret_cast<const float*>(ws + v.bcum);
        tp.eblk = reinterpret_cast<const float*>(ws + v.eblk);
        tp.seg_state = reinterpret_cast<float*>(ws + v.state);
        tp.seg_decay = reinterpret_cast<float*>(ws + v.decay);
        tp.unit_info = reinterpret_cast<const int4*>(ws + v.unit_info);
        tp.fused_items = reinterpret_cast<const int2*>(ws + v.fused);
        tp.state_items = reinterpret_cast<const int2*>(ws + v.sitems);
        tp.plan_count = reinterpret_cast<const int*>(ws + v.count);
        plan.cu = a.cu_seqlens;
        plan.total = a.total;
        plan.S = a.B;
        plan.H = a.H;
        plan.C = C;
        plan.seg_max = v.seg_max;
        plan.max_len = a.N;
        plan.unit_info = reinterpret_cast<int4*>(ws + v.unit_info);
        plan.fused_items = reinterpret_cast<int2*>(ws + v.fused);
        plan.state_items = reinterpret_cast<int2*>(ws + v.sitems);
        plan.count = reinterpret_cast<int*>(ws + v.count);
        plan.seq_info = reinterpret_cast<int2*>(ws + v.seq_info);
        plan.seq_order = reinterpret_cast<int*>(ws + v.seq_order);
        plan.max_fused = v.max_fused;
        plan.max_state = v.max_state;
    } else {
        // a resumed prefill reads the layout gret_prefill_state wrote: a slot for
        // every piece of every segment
        const WsLayout w = ws_layout(a.B, a.H, a.N, a.dk, a.dv, C, a.segments + (a.resume ? 1 : 0), a.pieces);
        tp.bcum = reinterpret_cast<const float*>(ws + w.bcum);
        tp.eblk = reinterpret_cast<const float*>(ws + w.eblk);
        tp.seg_state = reinterpret_cast<float*>(ws + w.state);
        tp.seg_decay = reinterpret_cast<float*>(ws + w.decay);
    }
    tp.S_final = a.S_final;
    tp.S0 = a.S0;
    tp.status = a.status;
    tp.H = a.H;
    tp.N = a.N;
    tp.Npad = (a.N + C - 1) / C * C;
    tp.P = a.segments;
    tp.seg_len = a.seg_len;
    tp.K = a.pieces;
    tp.piece_len = a.seg_len / a.pieces;
    tp.slots = (a.segments - (a.resume ? 0 : 1)) * a.pieces;
    tp.piece_split = (a.resume || a.cu_seqlens)
                         ? 0 : prefill_tc_piece_split(a.B, a.H, C, a.num_sms, a.segments, a.seg_len, a.pieces);
    tp.eps = a.eps;
    tp.gn = a.epi == GRET_EPI_GN_SWISH ? 1 : 0;
    tp.has_g = (a.epi == GRET_EPI_GN_SWISH && a.G) ? 1 : 0;
    tp.fault = a.fault;
    const bool packed = a.cu_seqlens != nullptr;
    if (a.dv == 256 && C == 64)
        return packed ? run_tc<256, 64, true>(a, tp, s, &plan) : run_tc<256, 64, false>(a, tp, s);
    if (a.dv == 256 && C == 128)
        return packed ? run_tc<256, 128, true>(a, tp, s, &plan) : run_tc<256, 128, false>(a, tp, s);
    if (a.dv == 128 && C == 128)
        return packed ? run_tc<128, 128, true>(a, tp, s, &plan) : run_tc<128, 128, false>(a, tp, s);
    if (a.dv == 128 && C == 64)
        return packed ? run_tc<128, 64, true>(a, tp, s, &plan) : run_tc<128, 64, false>(a, tp, s);
    return cudaErrorNotSupported;
}

template <int DV, int C>
static cudaError_t run_state_tc(const PrefillArgs& a, TcParams& tp, cudaStream_t s) {
    auto ks = prefill_state_kernel<DV, C, false>;
    cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, StateCfg<DV, C>::SMEM);
    const int units = a.B * a.H;
    int nyb = 0;
    const dim3 sgrid = gate_scan_grid(units, tp.Npad, C, &nyb);
    cudaError_t e = launch_pdl(gate_scan_kernel, sgrid, dim3(kScanThreads), 0, s,
                               a.z, static_cast<const int*>(nullptr), 0, const_cast<float*>(tp.bcum),
                               const_cast<float*>(tp.eblk), a.H, a.N, tp.Npad, C, a.inv_tau, nyb);
    if (e != cudaSuccess) return e;
    e = launch_pdl(ks, dim3(units * tp.slots), dim3(kStateThreads), StateCfg<DV, C>::SMEM, s, tp);
    if (e != cudaSuccess) return e;
    // fold every piece from the zero state, in place (slot j becomes the
    // increment from the slice's start through piece j), and write the last
    // fold as the slice's increment
    return launch_pdl(state_finish_kernel<DV>, dim3(units, (DV / 32) * (DK / 32)), dim3(32, 8), 0, s, tp.seg_state,
                      static_cast<const float*>(tp.seg_decay), tp.slots, tp.K, a.S_final, a.decay_out);
}

cudaError_t launch_prefill_state_tc(const PrefillArgs& a, int num_sms, cudaStream_t s) {
    TcParams tp;
    memset(&tp, 0, sizeof(tp));
    const int C = a.chunk;
    if (!make_map(&tp.tmKs, a.K, DK, a.H, a.N, a.B, state_sub(a.dv, C)) ||
        !make_map(&tp.tmVs, a.V, a.dv, a.H, a.N, a.B, state_sub(a.dv, C)))
        return cudaErrorInvalidValue;
    const int nchunks = (a.N + C - 1) / C;
    int P = 1, seg_len = a.N, Kp = 1;
    prefill_tc_plan(a.B, a.H, a.N, C, num_sms, &P, &seg_len, &Kp, prefill_tc_ctas_per_item(a.dv, C));
    const int K = prefill_tc_state_pieces(a.B, a.H, C, num_sms, P, seg_len);
    const WsLayout w = ws_layout(a.B, a.H, a.N, a.dk, a.dv, C, P + 1, K);
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    tp.bcum = reinterpret_cast<const float*>(ws + w.bcum);
    tp.eblk = reinterpret_cast<const float*>(ws + w.eblk);
    tp.seg_state = reinterpret_cast<float*>(ws + w.state);
    tp.seg_decay = reinterpret_cast<float*>(ws + w.decay);
    tp.status = a.status;
    tp.H = a.H;
    tp.N = a.N;
    tp.Npad = nchunks * C;
    tp.P = P;
    tp.seg_len = seg_len;
    tp.K = K;
    tp.piece_len = seg_len / K;
    tp.slots = P * K;              // every piece of every segment
    if (a.dv == 256 && C == 64) return run_state_tc<256, 64>(a, tp, s);
    if (a.dv == 256 && C == 128) return run_state_tc<256, 128>(a, tp, s);
    if (a.dv == 128 && C == 128) return run_state_tc<128, 128>(a, tp, s);
    if (a.dv == 128 && C == 64) return run_state_tc<128, 64>(a, tp, s);
    return cudaErrorNotSupported;
}

cudaError_t launch_state_fold(const float* dS_all, const float* decay_all, int num_slices, int slice,
                              const float* S0, float* S_in, int units, int elems, cudaStream_t s) {
    (void)num_slices;
    auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (elems % 4 == 0 && a16(dS_all) && a16(S0) && a16(S_in)) {
        const int nvec = elems / 4;
        return launch_pdl(state_fold_kernel<float4>, dim3(units, (nvec + 255) / 256), dim3(256), 0, s,
                          reinterpret_cast<const float4*>(dS_all), decay_all, slice,
                          reinterpret_cast<const float4*>(S0), reinterpret_cast<float4*>(S_in), units, nvec);
    }
    return launch_pdl(state_fold_kernel<float>, dim3(units, (elems + 255) / 256), dim3(256), 0, s, dS_all, decay_all,
                      slice, S0, S_in, units, elems);
}

}  // namespace gret
