// Tensor-core kernel family of libsf_gdn (bf16 I/O, fp32 state).
#pragma once

#include "sf_common.cuh"

namespace sf {

bool tc_supports(bool bf16, int dk, int dv, int C, bool use_beta);
size_t tc_workspace_bytes(const SeqView& s, bool backward);
cudaError_t tc_fwd(const SeqView& s, const FwdArgs& a, void* ws, cudaStream_t st);
cudaError_t tc_bwd(const SeqView& s, const BwdArgs& a, void* ws, cudaStream_t st);
int tc_launches(bool backward);

// Single stages of the path, for the pipelined segment chain.  A segment's
// "keep" region (tc_keep_bytes) holds what its forward stages produce and its
// backward stages read again: G, exp(G), -W, Khat, U^T, V_new^T and the
// chunk-entry states.  A "slot" region (tc_slot_bytes) holds the backward's
// per-chunk tiles dVi^T, dV_new^T, dS_C^T.  Both 256-byte aligned.
//   Prep    (f): k, v, g, beta -> keep            Scan    (f): keep, S_in -> keep, S_out
//   Out     (f): q, k, keep -> o                  Intra   (b): q, k, dO, keep -> slot
//   ScanBwd (b): q, dO, keep, slot, dS_out -> slot, dS_in (no forward recompute)
//   Grad    (b): q, k, v, beta, dO, keep, slot -> dq, dk, dv, dg, dbeta
enum class TcStage { Prep, Scan, Out, Intra, ScanBwd, Grad };
size_t tc_keep_bytes(const SeqView& s);
size_t tc_slot_bytes(const SeqView& s);
cudaError_t tc_stage(TcStage stage, const SeqView& s, const FwdArgs* f, const BwdArgs* b, void* keep, void* slot,
                     cudaStream_t st);
// Status word of the current device (bit 0: a kernel gave up waiting for one
// of its own bulk copies); synchronising; optionally cleared.
cudaError_t tc_device_status(int* status, bool clear);

}  // namespace sf
