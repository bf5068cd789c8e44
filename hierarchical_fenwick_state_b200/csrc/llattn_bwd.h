// Internal declarations of the backward pass (llattn_bwd in include/llattn.h).
#pragma once

#include <cuda_runtime.h>
#include <cstddef>

namespace llattn {

// One backward call after host-side validation.  Layouts as the forward's; every gradient is fp32.
struct BwdProblem {
  int in_dtype;          // LLATTN_F32 / LLATTN_BF16 (q, k, v, dout)
  const void* q;         // [tokens, H, dk]
  const void* k;
  const void* v;         // [tokens, H, dv]
  const void* dout;      // [tokens, H, dv]
  const float* log_a;    // [tokens, H]
  const float* lam;      // [tokens, H, L]
  float* dq;             // [tokens, H, dk]
  float* dk;
  float* dv;             // [tokens, H, dv]
  float* dlog_a;         // [tokens, H]
  float* dlam;           // [tokens, H, L]
  int nseq, H, T, d, L;  // d = dk = dv
  const int* cu_seqlens;  // device, may be null (dense)
  unsigned int* status;
};

// Scratch: the fp64 prefix sums of log_a by (sequence, local position, head), [nseq, T, H]
// (T bounds every sequence).
inline size_t bwd_workspace_bytes(int nseq, int H, int T) {
  return ((size_t)nseq * T * H * sizeof(double) + 255) / 256 * 256;
}

cudaError_t bwd(const BwdProblem& p, void* ws, cudaStream_t st);

// The tensor-core backward (bf16 inputs, d = 64): one launch for the pairs inside each aligned
// 128-token chunk (levels 0..7, the first write of every gradient), then one per level from
// kTcFirstLevel on; g = the fp64 prefix sums of log_a.  In place of the dense tiles and the
// CUDA-core level kernels.
constexpr int kTcFirstLevel = 8;
bool bwd_tc_supports(const BwdProblem& p);
cudaError_t bwd_levels_tc(const BwdProblem& p, const double* g, cudaStream_t st);

}  // namespace llattn
