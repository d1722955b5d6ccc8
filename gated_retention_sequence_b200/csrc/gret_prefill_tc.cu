// Tensor-core (tcgen05/TMEM) chunkwise prefill -- placeholder until the kernel lands.
#include "gret_common.cuh"

namespace gret {
bool prefill_tc_supported(int, int, int, gret_dtype) { return false; }
void prefill_tc_plan(int, int, int N, int, int, int* segments, int* seg_len) { *segments = 1; *seg_len = N; }
size_t prefill_tc_workspace_bytes(int, int, int, int, int) { return 0; }
cudaError_t launch_prefill_tc(const PrefillArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gret
