// Internal interface of the Log-Linear Gated DeltaNet forward (llattn_gdn_fwd).
#pragma once

#include <cuda_runtime.h>

namespace llattn {

struct GdnProblem {
  int in_dtype;              // LLATTN_F32 / LLATTN_BF16: type of q, k, v
  const void* q;
  const void* k;
  const void* v;
  const float* log_alpha;    // [.., H] gate logs
  const float* beta;         // [.., H] write strengths
  const float* lam;          // [.., H, L]
  float* out;                // [.., H, dv]
  int nseq, H, T, dk, dv, L;
  const int* cu_seqlens;
  unsigned int* status;
};

bool gdn_supports(int dk, int dv, int T);
cudaError_t gdn_forward(const GdnProblem& p, cudaStream_t st);

}  // namespace llattn
