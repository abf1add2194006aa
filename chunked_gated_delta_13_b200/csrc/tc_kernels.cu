// Tensor-core kernel family of libsf_gdn (bf16 I/O, fp32 state).
#include "tc_kernels.cuh"

namespace sf {

bool tc_supports(bool, int, int, int, bool) { return false; }
size_t tc_workspace_bytes(const SeqView&, bool) { return 0; }
cudaError_t tc_fwd(const SeqView&, const FwdArgs&, void*, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_bwd(const SeqView&, const BwdArgs&, void*, cudaStream_t) { return cudaErrorNotSupported; }
int tc_launches(bool) { return 0; }

}  // namespace sf
