// Internal declarations of the decoding step (llattn_decode_step in include/llattn.h).
#pragma once

#include <cuda_runtime.h>
#include <cstddef>

namespace llattn {

// One decoding step after host-side validation.  Layouts as in include/llattn.h.
struct DecodeProblem {
  int in_dtype;          // LLATTN_F32 / LLATTN_BF16
  const void* q;         // [B, H, dk]
  const void* k;         // [B, H, dk]
  const void* v;         // [B, H, dv]
  const float* log_a;    // [B, H]
  const float* lam;      // [B, H, L]
  const int* pos;        // [B] device
  float* levels;         // [B, H, L-1, dk, dv]   slot j = level j+1, without its pending gates
  float* gate;           // [B, H, 2, L-1]        log of each slot's pending gate, by position parity
  float* out;            // [B, H, dv]
  int B, H, L, dk, dv;
  unsigned int* status;  // device status word
};

// Bytes of the caller's state buffer: the level slots, then the two gate rows.
inline size_t decode_state_bytes(int B, int H, int L, int dk, int dv) {
  const size_t bh = (size_t)B * H, ns = (size_t)(L - 1);
  return bh * ns * dk * dv * sizeof(float) + bh * 2 * ns * sizeof(float);
}

cudaError_t decode_step(const DecodeProblem& p, cudaStream_t st);

// The decoding state after a prompt (llattn_prefill_state): every sequence of a dense or packed
// batch, at the position equal to its length.
struct PrefillProblem {
  int in_dtype;          // LLATTN_F32 / LLATTN_BF16: type of k, v
  const void* k;         // [.., H, dk] token-major, as the forward's inputs
  const void* v;         // [.., H, dv]
  const float* log_a;    // [.., H]
  float* levels;         // the decoding state's level slots [B, H, L-1, dk, dv]
  float* gate;           // and its gate rows [B, H, 2, L-1]
  int B, H, T, L, dk, dv;
  const int* cu_seqlens; // device, or null (dense: every length is T)
  unsigned int* status;
};

cudaError_t prefill_state(const PrefillProblem& p, cudaStream_t st);

}  // namespace llattn
