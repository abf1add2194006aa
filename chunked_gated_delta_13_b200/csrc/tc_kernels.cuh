// Tensor-core kernel family of libsf_gdn (bf16 I/O, fp32 state).
#pragma once

#include "sf_common.cuh"

namespace sf {

bool tc_supports(bool bf16, int dk, int dv, int C, bool use_beta);
size_t tc_workspace_bytes(const SeqView& s, bool backward);
cudaError_t tc_fwd(const SeqView& s, const FwdArgs& a, void* ws, cudaStream_t st);
cudaError_t tc_bwd(const SeqView& s, const BwdArgs& a, void* ws, cudaStream_t st);
int tc_launches(bool backward);
// Status word of the current device (bit 0: a kernel gave up waiting for one
// of its own bulk copies); synchronising; optionally cleared.
cudaError_t tc_device_status(int* status, bool clear);

}  // namespace sf
