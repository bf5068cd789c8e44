// One decoding step of log-linear attention (Mamba-2 form) for a batch of sequences.
//
// Log-Linear Attention (gist.science summaries, Italian "Sommario tecnico" section 2, "Forma
// Ricorrente e Parallelizzata", decoding bullet; Spanish "Resumen tecnico" section 2,
// "Particion Jerarquica"): at inference the layer keeps one d_k x d_v state per Fenwick level,
// O(log T) of them, and each new token's output is the level-weighted combination of those
// states.  For the token at 0-based position n of a sequence:
//
//   every occupied level is gated by a_n; level 0 is the token's own k_n v_n^T;
//   o_n = sum over level 0 and the occupied levels l of lam[n, l] * (q_n^T S_l);
//   with m the number of trailing one bits of n, levels 0..m add up into level m+1
//   (a binary-counter carry) and levels 1..m fall empty.
//
// Level l >= 1 is occupied exactly when bit l-1 of n is set, so the position is the whole
// occupancy record: no flags, and a state buffer never needs clearing.
//
// Memory design.  The step is bound by HBM: it must read every occupied state (popcount(n) of
// them, d_k*d_v*4 bytes each) and write the one carried state.  Gating the occupied states in
// place would rewrite each of them every step, doubling the traffic, so the gate is kept
// lazily: a slot stores its state as it was when written, plus (in a small side row) the log
// of the gate product it has missed since.  A step reads that scalar, folds exp(gate + log a_n)
// into the readout and the carry, and advances the scalars of the levels that survive.  The
// side row is double-buffered by the parity of n, so that the CTAs of one (sequence, head)
// that read the old values never race the one CTA that writes the new ones.
//
// Grid: one CTA of 256 threads per (32 value columns, head, sequence).  Thread (r, c4) owns
// rows r, r+32, ... of its 32-column slab and four adjacent columns, so every warp load is one
// 128-byte line per row, each state element is loaded once, and the readout is a reduction
// over the 32 row threads of each column (shuffles, then shared memory).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/llattn.h"
#include "llattn_common.cuh"
#include "llattn_decode.h"
#include "llattn_internal.h"

namespace llattn {
namespace {

constexpr int kThreads = 256;
constexpr int kCols = 32;                          // value columns per CTA
constexpr int kRowsPerPass = kThreads / (kCols / 4);  // 32 rows, four columns per thread

__device__ __forceinline__ float4 ld4_in(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ float4 ld4_in(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

__device__ __forceinline__ void fma4(float4& acc, float s, const float4& x) {
  acc.x = fmaf(s, x.x, acc.x);
  acc.y = fmaf(s, x.y, acc.y);
  acc.z = fmaf(s, x.z, acc.z);
  acc.w = fmaf(s, x.w, acc.w);
}

template <typename Tin, int DK>
__global__ void __launch_bounds__(kThreads) decode_step_kernel(DecodeProblem p) {
  constexpr int P = DK / kRowsPerPass;  // rows per thread
  __shared__ float s_q[DK], s_k[DK];
  __shared__ float s_lam[32];
  __shared__ float s_w[32];    // exp(pending gate + log a_n) of the i-th occupied slot
  __shared__ int s_slot[32];   // slot index of the i-th occupied level
  __shared__ float s_red[kThreads / 32][kCols];

  const int tid = threadIdx.x;
  const int cb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nslot = p.L - 1;
  const int n = p.pos[b];
  // Positions the slots and lam rows can hold: 0 <= n < 2^(L-1).
  if (n < 0 || (nslot < 31 && n >= (1 << nslot))) {
    if (tid == 0) atomicOr(p.status, LLATTN_DEV_DECODE_POS);
    return;
  }
  const unsigned un = static_cast<unsigned>(n);
  const int m = __ffs(~un) - 1;  // trailing one bits of n (n < 2^31, so ~n has a set bit)
  const int cnt = __popc(un);    // occupied levels
  const unsigned par = un & 1u, par1 = (un + 1u) & 1u;

  const size_t bh = (size_t)b * p.H + h;
  const Tin* q = static_cast<const Tin*>(p.q) + bh * DK;
  const Tin* k = static_cast<const Tin*>(p.k) + bh * DK;
  const Tin* v = static_cast<const Tin*>(p.v) + bh * p.dv;
  const float la = __ldg(p.log_a + bh);
  float* gate = p.gate + bh * 2 * nslot;

  if (tid < DK) {
    s_q[tid] = ld_in(q + tid);
    s_k[tid] = ld_in(k + tid);
  }
  if (tid < p.L) s_lam[tid] = __ldg(p.lam + bh * p.L + tid);
  if (tid < nslot && ((un >> tid) & 1u)) {
    const int rank = __popc(un & ((1u << tid) - 1u));
    s_slot[rank] = tid;
    s_w[rank] = expf(gate[par * nslot + tid] + la);
  }
  __syncthreads();

  const int c4 = tid & 7, r = tid >> 3;
  const int col = cb * kCols + 4 * c4;
  const float4 vv = ld4_in(v + col);

  // level 0: the token's own state k v^T, read out with lam[0] and carried
  float qr[P];
  float4 carry[P];
  float qk = 0.f;
#pragma unroll
  for (int t = 0; t < P; ++t) {
    qr[t] = s_q[r + kRowsPerPass * t];
    const float kr = s_k[r + kRowsPerPass * t];
    carry[t] = make_float4(kr * vv.x, kr * vv.y, kr * vv.z, kr * vv.w);
    qk = fmaf(qr[t], kr, qk);
  }
  float4 part = make_float4(0.f, 0.f, 0.f, 0.f);
  fma4(part, s_lam[0] * qk, vv);

  const size_t slot_stride = (size_t)DK * p.dv;
  const size_t row_stride = (size_t)kRowsPerPass * p.dv;
  float* base = p.levels + bh * nslot * slot_stride + (size_t)r * p.dv + col;

  // occupied levels: each element is read once, for the readout and (levels 1..m) the carry
#pragma unroll 2
  for (int i = 0; i < cnt; ++i) {
    const int j = s_slot[i];
    const float w = s_w[i];
    const float* src = base + j * slot_stride;
    float4 x[P];
#pragma unroll
    for (int t = 0; t < P; ++t) x[t] = __ldcs(reinterpret_cast<const float4*>(src + t * row_stride));
    float4 d = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int t = 0; t < P; ++t) fma4(d, qr[t], x[t]);
    fma4(part, s_lam[j + 1] * w, d);
    if (j < m) {
#pragma unroll
      for (int t = 0; t < P; ++t) fma4(carry[t], w, x[t]);
    }
  }

  // carry into level m+1 (slot m), which is empty at n; the last position a full counter can
  // hold (m == nslot) has no slot to carry into
  if (m < nslot) {
    float* dst = base + m * slot_stride;
#pragma unroll
    for (int t = 0; t < P; ++t) __stcs(reinterpret_cast<float4*>(dst + t * row_stride), carry[t]);
  }

  // readout: sum over the 32 row threads of each column
#pragma unroll
  for (int off = 8; off < 32; off <<= 1) {
    part.x += __shfl_xor_sync(0xffffffffu, part.x, off);
    part.y += __shfl_xor_sync(0xffffffffu, part.y, off);
    part.z += __shfl_xor_sync(0xffffffffu, part.z, off);
    part.w += __shfl_xor_sync(0xffffffffu, part.w, off);
  }
  const int lane = tid & 31, warp = tid >> 5;
  if (lane < 8) {
    s_red[warp][4 * lane + 0] = part.x;
    s_red[warp][4 * lane + 1] = part.y;
    s_red[warp][4 * lane + 2] = part.z;
    s_red[warp][4 * lane + 3] = part.w;
  }
  __syncthreads();
  if (tid < kCols) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) s += s_red[w][tid];
    p.out[bh * p.dv + cb * kCols + tid] = s;
  }

  // pending gates as of position n+1 (one CTA per (sequence, head) writes them): the carried
  // slot starts afresh, the levels that stay occupied add log a_n
  if (cb == 0 && tid < nslot && (((un + 1u) >> tid) & 1u))
    gate[par1 * nslot + tid] = (tid == m) ? 0.f : gate[par * nslot + tid] + la;
}

template <typename Tin>
cudaError_t launch(const DecodeProblem& p, cudaStream_t st) {
  const dim3 grid(p.dv / kCols, p.H, p.B);
  switch (p.dk) {
    case 32: decode_step_kernel<Tin, 32><<<grid, kThreads, 0, st>>>(p); break;
    case 64: decode_step_kernel<Tin, 64><<<grid, kThreads, 0, st>>>(p); break;
    case 128: decode_step_kernel<Tin, 128><<<grid, kThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t decode_step(const DecodeProblem& p, cudaStream_t st) {
  count_launch(1);
  main_kernel_begin(st);
  const cudaError_t e = p.in_dtype == LLATTN_BF16 ? launch<__nv_bfloat16>(p, st)
                                                  : launch<float>(p, st);
  main_kernel_end(st);
  return e;
}

}  // namespace llattn
