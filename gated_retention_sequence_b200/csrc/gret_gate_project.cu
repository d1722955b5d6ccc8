// Gate projection z = X W_gamma, fused with the chunk decay scan on the
// tensor-core prefill path, and a CUDA-core projection for the other paths.
//
// "YOCO 深度技术分析", section 2.2: gamma = sigmoid(X W_gamma)^(1/tau) with
// one W_gamma column (R^{d x 1}) per head, so the gate logit of token n and
// head h is z[n][h] = sum_i X[n][i] W_gamma[i][h]; the Medium-article
// translation's "门控保留率" paragraph gives W_gamma the same shape.
//
// B200 mapping.  z for 128 tokens and all H heads is one tcgen05 product
//   D[t][h] = X[t][:] W_gamma[:][h]   (M = 128 tokens, N = H rounded up to
//                                      16, K = d_model in steps of 16)
// accumulated in fp32 in tensor memory, with X tiles (bf16, 128-byte swizzle)
// and W_gamma^T tiles arriving by TMA.  The gate precision is kept by feeding
// W_gamma as two bf16 halves, hi = bf16(W) and lo = bf16(W - hi): X is exact in
// bf16, so z = X hi + X lo carries W to about 2^-17 relative, against 2^-9 for
// a single bf16 copy (a z near 8 would otherwise move gamma's memory length by
// percents).  The halves are stacked as the rows of one B operand, so that one
// MMA of N = 2 x heads gives both products side by side.  The four epilogue
// warps then read z = D[t][h] + D[t][HP + h] straight from tensor memory
// (lane = token), form log gamma, and scan it along the tokens of each chunk
// (warp shuffles, then the earlier warps' totals of the chunk through shared
// memory), writing the same decay sums and P-block factors the plain gate scan
// writes: z itself never reaches HBM.
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <utility>

#include "gret_common.cuh"
#include "gret_sm100.cuh"

namespace gret {
namespace {

using namespace sm100;

constexpr int kProjRows = 128;      // tokens per CTA (the MMA's M)
constexpr int kProjThreads = 160;   // warps 0-3: scan epilogue, lane = token; warp 4: TMA and MMA
constexpr int kProjBox = 64;        // d_model columns per TMA box (128 bytes of bf16)

struct ProjParams {
    CUtensorMap tmX, tmW;
    float* bcum;            // [B*H][Npad] chunk-local cumulative log-decay
    float* eblk;            // [B*H][Npad] P-block factors
    unsigned int* status;
    int H, N, Npad, C, nk;  // nk: d_model steps of kProjBox
    float inv_tau;
};

template <int HP>
struct ProjCfg {
    static constexpr int XB = kProjRows * 128;      // X tile: 128 tokens x 64 bf16
    static constexpr int WB = 2 * HP * 128;         // W^T tile: hi then lo rows, HP each, x 64 bf16
    static constexpr int STAGE = XB + WB;           // X, stacked W
    // as many stages as about 192 KB hold (2-8): the kernel streams X once, so
    // the loads in flight per SM set its rate
    static constexpr int NS_FIT = (192 * 1024) / STAGE;
    static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
    static_assert(NS >= 2, "projection stages");
    static constexpr int OFF_BAR = NS * STAGE;
    static constexpr int NBAR = 2 * NS + 1;         // full, empty per stage; all MMAs done
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_WSUM = OFF_MISC + 16;  // [HP][4] each warp's scan total
    static constexpr int SMEM = OFF_WSUM + HP * 4 * 4 + 1024;
    static constexpr int TM_COLS = 2 * HP <= 32 ? 32 : 2 * HP <= 64 ? 64 : 2 * HP <= 128 ? 128 : 256;
    static_assert(2 * HP <= 256, "one MMA of N = 2 HP");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

template <int HP>
__global__ void __launch_bounds__(kProjThreads, 1) gate_project_scan_kernel(const __grid_constant__ ProjParams p) {
    using CF = ProjCfg<HP>;
    constexpr int NS = CF::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m = blockIdx.x, b = blockIdx.y;       // token tile, sequence

    auto full = [&](int s) -> uint32_t { return sb + CF::OFF_BAR + 8 * s; };
    auto empty = [&](int s) -> uint32_t { return sb + CF::OFF_BAR + 8 * (NS + s); };
    const uint32_t done = sb + CF::OFF_BAR + 8 * (2 * NS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CF::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CF::OFF_MISC + 4);
    float* wsum = reinterpret_cast<float*>(sm + CF::OFF_WSUM);

    if (tid == 0) {
        for (int i = 0; i < CF::NBAR; ++i) mbar_init(sb + CF::OFF_BAR + 8 * i, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tmX);
        tma_prefetch_desc(&p.tmW);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), CF::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    // the split weights come from the kernel before this one
    grid_dep_launch();
    grid_dep_wait();

    if (warp == 4) {
        if (lane == 0) {
            // ---------------------------------------------------- loads and MMAs
            int last = -1;      // the last step whose loads were issued
            auto issue = [&](int k) {
                const int s = k % NS;
                last = k;
                const uint32_t st = sb + s * CF::STAGE;
                mbar_arrive_expect_tx(full(s), CF::STAGE);
                tma_load_3d(st, &p.tmX, k * kProjBox, m * kProjRows, b, full(s));
                tma_load_2d(st + CF::XB, &p.tmW, k * kProjBox, 0, full(s));
            };
            for (int k = 0; k < NS && k < p.nk; ++k) issue(k);
            constexpr uint32_t idesc = idesc_bf16(kProjRows, 2 * HP, false, false);
            for (int k = 0; k < p.nk; ++k) {
                const int s = k % NS;
                if (!mbar_wait(full(s), (k / NS) & 1, p.status, abort_flag)) break;
                tc_fence_after();
                const uint32_t st = sb + s * CF::STAGE;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tm, sdesc_sw128(st + kk * 32, 16, 1024), sdesc_sw128(st + CF::XB + kk * 32, 16, 1024),
                           idesc, (k | kk) != 0);
                mma_commit(empty(s));
                // the previous step's stage is free once its MMAs have read it
                // (they run before this step's, which queue behind them), so the
                // issuer never waits on the MMAs it has just committed
                if (k > 0 && k - 1 + NS < p.nk) {
                    if (!mbar_wait(empty((k - 1) % NS), ((k - 1) / NS) & 1, p.status, abort_flag)) break;
                    issue(k - 1 + NS);
                }
            }
            mma_commit(done);
            // every MMA has completed, and on the give-up path every load issued
            // has landed, before the tensor and shared memory are released
            mbar_wait_drain(done, 0, kWaitCycles);
            if (*abort_flag)
                for (int k = last; k >= 0 && k > last - NS; --k) mbar_wait_drain(full(k % NS), (k / NS) & 1, kWaitCycles);
        }
    } else {
        // -------------------------------------------------------- scan epilogue
        mbar_wait(done, 0, p.status, abort_flag);
        tc_fence_after();
        const int n = m * kProjRows + warp * 32 + lane;        // this thread's token
        const int cw = p.C / 32;                               // warps per chunk (2 or 4)
        const int w0 = warp - warp % cw;                       // first warp of this thread's chunk
        const uint32_t lq = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
        for (int g = 0; g < HP / 16; ++g) {
            uint32_t r[16], rl[16];
            tmem_ld_x16(tm + lq + g * 16, r);             // X W_hi
            tmem_ld_x16(tm + lq + HP + g * 16, rl);       // X W_lo
            tmem_wait_ld();
            float x[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int h = g * 16 + j;
                const float z = __uint_as_float(r[j]) + __uint_as_float(rl[j]);
                // past the sequence's end the decay stays flat (log gamma = 0)
                x[j] = (h < p.H && n < p.N) ? log_gamma(z, p.inv_tau) : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x[j], o);
                    if (lane >= o) x[j] += y;
                }
                if (lane == 31) wsum[h * 4 + warp] = x[j];
            }
            named_bar_sync(1, 128);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int h = g * 16 + j;
                for (int w = w0; w < warp; ++w) x[j] += wsum[h * 4 + w];   // the chunk's earlier warps
                const float e = p_block_factor(x[j], lane, p.C / 4);
                if (h < p.H && n < p.Npad) {
                    const size_t at = ((size_t)b * p.H + h) * p.Npad + n;
                    p.bcum[at] = x[j];
                    p.eblk[at] = e;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, CF::TM_COLS);
    }
}

// W_gamma [d_model][H] fp32 -> hi, lo [HP][d_model] bf16 (rows h >= H zero);
// lo follows hi in memory, so the two form one [2 HP][d_model] operand.
__global__ void gate_weight_split_kernel(const float* __restrict__ W, int d_model, int H, int HP,
                                         __nv_bfloat16* __restrict__ whi, __nv_bfloat16* __restrict__ wlo) {
    // the previous call's kernels may still read this workspace
    grid_dep_launch();
    grid_dep_wait();
    const long long total = (long long)HP * d_model;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(e / d_model), i = (int)(e % d_model);
        const float w = h < H ? W[(size_t)i * H + h] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        whi[e] = hi;
        wlo[e] = __float2bfloat16_rn(w - __bfloat162float(hi));
    }
}

// z[r][h] = sum_i X[r][i] W[i][h] on CUDA cores, fp32 accumulation (the
// fp32 path and shapes the fused kernel does not take).  One thread per
// (token, head): the lanes of a warp share X[r][i] and read consecutive W.
template <typename T>
__global__ void gate_project_simt_kernel(const T* __restrict__ X, const float* __restrict__ W, long long rows,
                                         int d_model, int H, float* __restrict__ z) {
    const long long total = rows * H;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long r = e / H;
        const int h = (int)(e % H);
        const T* x = X + r * d_model;
        float acc = 0.f;
        for (int i = 0; i < d_model; ++i) acc = fmaf(to_f32(x[i]), W[(size_t)i * H + h], acc);
        z[e] = acc;
    }
}

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

// bf16 tensor of `rank` dims (innermost first), 128-byte swizzled boxes.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t strides[2];
    cuuint64_t st = 2;
    for (int i = 0; i + 1 < rank; ++i) {
        st *= dims[i];
        strides[i] = st;
    }
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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

template <int HP>
cudaError_t run_project(ProjParams& pp, int B, cudaStream_t s) {
    using CF = ProjCfg<HP>;
    auto k = gate_project_scan_kernel<HP>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM);
    if (e != cudaSuccess) return e;
    const dim3 grid((pp.Npad + kProjRows - 1) / kProjRows, B);
    return launch_pdl(k, grid, dim3(kProjThreads), CF::SMEM, s, pp);
}

}  // namespace

int gate_project_heads_padded(int H) {
    return H <= 16 ? 16 : H <= 32 ? 32 : H <= 64 ? 64 : H <= 128 ? 128 : 0;
}

bool gate_project_tc_supported(int H, int d_model) {
    // TMA rows of X are d_model bf16 apart (a multiple of 16 bytes)
    return gate_project_heads_padded(H) > 0 && d_model > 0 && d_model % 8 == 0;
}

size_t gate_project_tc_ws_bytes(int H, int d_model) {
    const size_t both = 2 * (size_t)gate_project_heads_padded(H) * d_model * 2;
    return (both + 255) & ~size_t(255);
}

cudaError_t launch_gate_project_tc(const PrefillArgs& a, float* bcum, float* eblk, int Npad, void* wsplit,
                                   cudaStream_t s) {
    const int HP = gate_project_heads_padded(a.H);
    __nv_bfloat16* whi = static_cast<__nv_bfloat16*>(wsplit);
    __nv_bfloat16* wlo = whi + (size_t)HP * a.d_model;
    const long long elems = (long long)HP * a.d_model;
    const int blocks = (int)std::min<long long>((elems + 255) / 256, 148 * 8);
    cudaError_t e = launch_pdl(gate_weight_split_kernel, dim3(blocks), dim3(256), 0, s, a.Wg, a.d_model, a.H, HP,
                               whi, wlo);
    if (e != cudaSuccess) return e;
    ProjParams pp;
    memset(&pp, 0, sizeof(pp));
    const cuuint64_t xd[3] = {(cuuint64_t)a.d_model, (cuuint64_t)a.N, (cuuint64_t)a.B};
    const cuuint32_t xb[3] = {kProjBox, kProjRows, 1};
    const cuuint64_t wd[2] = {(cuuint64_t)a.d_model, (cuuint64_t)(2 * HP)};
    const cuuint32_t wb[2] = {kProjBox, (cuuint32_t)(2 * HP)};
    if (!make_map(&pp.tmX, a.X, 3, xd, xb) || !make_map(&pp.tmW, whi, 2, wd, wb)) return cudaErrorInvalidValue;
    pp.bcum = bcum;
    pp.eblk = eblk;
    pp.status = a.status;
    pp.H = a.H;
    pp.N = a.N;
    pp.Npad = Npad;
    pp.C = a.chunk;
    pp.nk = (a.d_model + kProjBox - 1) / kProjBox;
    pp.inv_tau = a.inv_tau;
    if (g_profile_gate_start) cudaEventRecord(g_profile_gate_start, s);
    switch (HP) {
        case 16: e = run_project<16>(pp, a.B, s); break;
        case 32: e = run_project<32>(pp, a.B, s); break;
        case 64: e = run_project<64>(pp, a.B, s); break;
        default: e = run_project<128>(pp, a.B, s); break;
    }
    if (g_profile_gate_stop) cudaEventRecord(g_profile_gate_stop, s);
    return e;
}

cudaError_t launch_gate_project_simt(const PrefillArgs& a, float* z, cudaStream_t s) {
    const long long rows = (long long)a.B * a.N;
    const long long total = rows * a.H;
    const int blocks = (int)std::min<long long>((total + 255) / 256, 148 * 16);
    if (g_profile_gate_start) cudaEventRecord(g_profile_gate_start, s);
    if (a.io == GRET_BF16)
        gate_project_simt_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(a.X), a.Wg, rows, a.d_model, a.H, z);
    else
        gate_project_simt_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(a.X), a.Wg, rows,
                                                                a.d_model, a.H, z);
    if (g_profile_gate_stop) cudaEventRecord(g_profile_gate_stop, s);
    return cudaGetLastError();
}

}  // namespace gret
