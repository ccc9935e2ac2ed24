// gemm.cu -- placeholder until the tcgen05 prefill GEMM lands.
#include "bl_common.cuh"

namespace bl {
size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }
int launch_gemm(const GemvArgs &, void *, size_t, cudaStream_t) { return BL_ERR_UNSUPPORTED; }
}  // namespace bl
