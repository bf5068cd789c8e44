// Internal declarations shared by the host API and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace llattn {

// Problem description after host-side validation.
struct Problem {
  int in_dtype;        // LLATTN_F32 / LLATTN_BF16
  const void* q;
  const void* k;
  const void* v;
  const float* log_a;
  const float* lam;
  float* out;
  int nseq;            // B (dense) or number of packed sequences
  int H, T, dk, dv, L;
  const int* cu_seqlens;  // device, may be null (dense)
  unsigned int* status;   // device status word of the current device
};

// Launch accounting (llattn_profile): every kernel launch calls count_launch();
// the launcher brackets its dominant kernel with main_kernel_begin/end.
void count_launch(int n = 1);
void main_kernel_begin(cudaStream_t st);
void main_kernel_end(cudaStream_t st);

// Bytes of scratch each path needs (256-byte granules).
size_t simt_workspace_bytes(int nseq, int H, int T, int dk, int dv, int chunk);
size_t tc_workspace_bytes(int nseq, int H, int T, int dk, int dv, int chunk, bool varlen);

// Kernel launchers; return a cudaError_t from the launches.
cudaError_t simt_forward(const Problem& p, int chunk, void* ws, cudaStream_t st);
// Short sequences on CUDA cores in one launch (the masked form; T <= 512).
bool simt_short_supports(int T, int L);
cudaError_t simt_short_forward(const Problem& p, cudaStream_t st);
cudaError_t tc_forward(const Problem& p, int chunk, void* ws, cudaStream_t st, bool serial);
bool tc_supports(int in_dtype, int dk, int dv, int chunk, int T);
// Segment length of the tensor-core path: the forced value (chunks, 0 = automatic), and the
// chunks per segment a call of this shape uses (0: each CTA walks a whole sequence).
void tc_set_segment_chunks(int chunks);
int tc_segment_chunks(int nseq, int H, int T, int dk, int dv, bool varlen);
bool tc_serial_supports(int in_dtype, int dk, int dv, int chunk, int T);

// TMA map of a [tokens, H, rowlen] bf16 tensor viewed as {rowlen, H, tokens}: box {64, 1, 128}
// (one 64-column slice of 128 rows), 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, int rowlen, int H, long long tokens);
// TMA map of a [tokens, H, rowlen] fp32 tensor viewed as {rowlen, H, tokens}: box {32, 1, 128}
// (one 32-column slice of 128 rows, 128-byte rows), 128-byte swizzle; for tile stores and
// reduce-adds.
cudaError_t make_out_map(CUtensorMap* m, void* base, int rowlen, int H, long long tokens);

// Device address of the fixed scratch array behind llattn_fwd_noalloc on the
// current device (looked up on the first call per device, then cached).
cudaError_t noalloc_scratch(void** ptr);

// Number of chunk-level Fenwick blocks kept per (sequence, head) for Nc chunks,
// and the offset of level b's blocks: level b holds blocks (b, j) for even j,
// i.e. ((Nc - 1) >> (b + 1)) + 1 of them (only levels with 2^b < Nc).
__host__ __device__ inline int chunk_levels(int Nc) {
  int nb = 0;
  while ((1 << nb) < Nc) ++nb;
  return nb;  // levels 0..nb-1 occur for Nc chunks
}
__host__ __device__ inline int blocks_at_level(int Nc, int b) {
  return ((Nc - 1) >> (b + 1)) + 1;
}
__host__ __device__ inline int level_offset(int Nc, int b) {
  int off = 0;
  for (int i = 0; i < b; ++i) off += blocks_at_level(Nc, i);
  return off;
}
__host__ __device__ inline int total_blocks(int Nc) {
  return level_offset(Nc, chunk_levels(Nc));
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace llattn
