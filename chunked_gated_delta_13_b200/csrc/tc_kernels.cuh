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
// "keep" region (tc_keep_bytes) holds what its forward stages and its intra
// stage produce for its later stages: G, exp(G), -W, L, Khat, U^T, V_new^T, the
// chunk-entry states, dVi^T and D^T.  A "slot" region (tc_slot_bytes) holds
// the reverse scan's per-chunk tiles dV_new^T, dS_C^T.  Both 256-byte aligned.
//   Prep    (f): k, v, g, beta -> keep            Scan    (f): keep, S_in -> keep, S_out
//   Out     (f): q, k, keep -> o                  Intra   (b): q, k, dO, keep (G) -> keep
//   OutOg (f, b): Out and Intra of one segment in one launch
//   ScanBwd (b): keep, dS_out -> slot, dS_in (no forward recompute)
//   Grad    (b): q, k, v, beta, dO, keep, slot -> dq, dk, dv, dg, dbeta
enum class TcStage { Prep, Scan, Out, OutOg, Intra, ScanBwd, Grad };
size_t tc_keep_bytes(const SeqView& s);
size_t tc_slot_bytes(const SeqView& s);
cudaError_t tc_stage(TcStage stage, const SeqView& s, const FwdArgs* f, const BwdArgs* b, void* keep, void* slot,
                     cudaStream_t st);
// Status word of the current device (bit 0: a kernel gave up waiting for one
// of its own bulk copies); synchronising; optionally cleared.
cudaError_t tc_device_status(int* status, bool clear);

}  // namespace sf
