// Device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace llattn {

__device__ __forceinline__ float ld_in(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Start (flattened token index) and length of sequence `s`.
struct SeqSpan {
  long long start;
  int len;
};

__device__ __forceinline__ SeqSpan seq_span(int s, int T, const int* cu, unsigned int* status) {
  if (cu == nullptr) return {(long long)s * T, T};
  int a = cu[s], b = cu[s + 1];
  int len = b - a;
  if (len < 0) {
    atomicOr(status, 4u);  // cu_seqlens decreasing
    len = 0;
  }
  if (len > T) {
    atomicOr(status, 1u);  // longer than the T bound: rows past T are not computed
    len = T;
  }
  return {(long long)a, len};
}

// Fenwick level of positions t, s (0-based, same sequence): 0 if equal, else 1 + msb(t ^ s).
__device__ __forceinline__ int fenwick_level(int t, int s) {
  unsigned x = (unsigned)(t ^ s);
  return x ? 32 - __clz(x) : 0;
}

}  // namespace llattn
