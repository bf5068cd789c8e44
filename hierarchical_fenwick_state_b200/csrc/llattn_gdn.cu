// Forward of Log-Linear Gated DeltaNet on CUDA cores (fp32 state, fp32 arithmetic).
//
// Log-Linear Attention (gist.science, Italian "Sommario tecnico" section 2,
// "Generalizzazione"; Spanish "Variantes Propuestas" item 2) lifts the gated delta rule
// to the hierarchical Fenwick structure.  The pages give no formula; the reading taken
// (the one the oracle pins) keeps one d_k x d_v state per Fenwick level, as the recurrent
// form of the Mamba-2 variant does ("Forma Ricorrente e Parallelizzata", decoding bullet):
//   1. every occupied level state takes the gated delta transition
//        S <- alpha_t (S - beta_t k_t (k_t^T S)),   alpha_t = exp(log_alpha[t]);
//   2. the token opens level 0 with S_0 = beta_t k_t v_t^T;
//   3. o_t = sum over occupied levels l of lam[t, l] S_l^T q_t;
//   4. levels 0..m merge into m + 1 (m = trailing one bits of t), as a binary counter.
//
// The transition acts on each column of S (one value index) on its own: column j of S_l
// is a d_k-vector s with s <- alpha (s - beta k (k . s)).  So one warp owns one value
// column of every level state, each lane holding d_k / 32 rows of it in registers, and
// the dot products k . s and q . s are warp reductions.  A CTA of eight warps takes eight
// columns of one (sequence, head) and walks the sequence token by token.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/llattn.h"
#include "llattn_common.cuh"
#include "llattn_gdn.h"
#include "llattn_internal.h"

namespace llattn {
namespace {

constexpr int kGdnWarps = 8;              // value columns per CTA
constexpr int kGdnMaxLev = 17;            // levels held (T <= 65536)

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename TIn, int R>   // R = d_k / 32 rows of each column per lane
__global__ void __launch_bounds__(kGdnWarps * 32)
gdn_recurrent_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                     const TIn* __restrict__ v, const float* __restrict__ log_alpha,
                     const float* __restrict__ beta, const float* __restrict__ lam,
                     float* __restrict__ out, int H, int T, int L, int dv,
                     const int* __restrict__ cu, unsigned int* status) {
  constexpr int DK = 32 * R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * kGdnWarps + warp;
  const int h = blockIdx.y, sq = blockIdx.z;
  const SeqSpan sp = seq_span(sq, T, cu, status);
  if (sp.len <= 0 || col >= dv) return;

  float s[kGdnMaxLev][R];
#pragma unroll
  for (int l = 0; l < kGdnMaxLev; ++l)
#pragma unroll
    for (int r = 0; r < R; ++r) s[l][r] = 0.f;
  uint32_t live = 0;   // bit l: level l holds a state (the binary counter of positions)

  for (int t = 0; t < sp.len; ++t) {
    const long long tok = sp.start + t;
    const long long base = tok * H + h;
    float kr[R], qr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      kr[r] = ld_in(k + base * DK + r * 32 + lane);
      qr[r] = ld_in(q + base * DK + r * 32 + lane);
    }
    const float a = __expf(__ldg(log_alpha + base));
    const float b = __ldg(beta + base);
    const float vj = ld_in(v + base * dv + col);
    const float* lr = lam + base * L;
    // 1. transition of the occupied levels (l >= 1; level 0 is rewritten below)
#pragma unroll
    for (int l = 1; l < kGdnMaxLev; ++l) {
      if (!((live >> l) & 1u)) continue;
      float p = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) p += kr[r] * s[l][r];
      p = warp_sum(p) * b;
#pragma unroll
      for (int r = 0; r < R; ++r) s[l][r] = a * (s[l][r] - p * kr[r]);
    }
    // 2. the new token's write
#pragma unroll
    for (int r = 0; r < R; ++r) s[0][r] = b * kr[r] * vj;
    live |= 1u;
    // 3. readout: sum over occupied levels of lam[t, l] (q . s_l)
    float acc = 0.f;
#pragma unroll
    for (int l = 0; l < kGdnMaxLev; ++l) {
      if (!((live >> l) & 1u)) continue;
      float p = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) p += qr[r] * s[l][r];
      acc += __ldg(lr + l) * p;
    }
    acc = warp_sum(acc);
    if (lane == 0) out[base * dv + col] = acc;
    // 4. promotion: levels 0..m into m + 1, m = trailing one bits of t
    if (t + 1 < sp.len) {
      const int m = __ffs(~t) - 1;
      float sum[R];
#pragma unroll
      for (int r = 0; r < R; ++r) sum[r] = 0.f;
#pragma unroll
      for (int l = 0; l < kGdnMaxLev; ++l) {
        if (l <= m) {
#pragma unroll
          for (int r = 0; r < R; ++r) {
            sum[r] += s[l][r];
            s[l][r] = 0.f;
          }
        }
      }
#pragma unroll
      for (int l = 1; l < kGdnMaxLev; ++l)
        if (l == m + 1)
#pragma unroll
          for (int r = 0; r < R; ++r) s[l][r] = sum[r];
      live = (live & ~((2u << m) - 1u)) | (1u << (m + 1));
    }
  }
}

template <typename TIn>
cudaError_t launch(const GdnProblem& p, cudaStream_t st) {
  const dim3 grid((p.dv + kGdnWarps - 1) / kGdnWarps, p.H, p.nseq);
  const TIn* q = static_cast<const TIn*>(p.q);
  const TIn* k = static_cast<const TIn*>(p.k);
  const TIn* v = static_cast<const TIn*>(p.v);
  switch (p.dk) {
    case 32:
      gdn_recurrent_kernel<TIn, 1><<<grid, kGdnWarps * 32, 0, st>>>(
          q, k, v, p.log_alpha, p.beta, p.lam, p.out, p.H, p.T, p.L, p.dv, p.cu_seqlens, p.status);
      break;
    case 64:
      gdn_recurrent_kernel<TIn, 2><<<grid, kGdnWarps * 32, 0, st>>>(
          q, k, v, p.log_alpha, p.beta, p.lam, p.out, p.H, p.T, p.L, p.dv, p.cu_seqlens, p.status);
      break;
    default:
      gdn_recurrent_kernel<TIn, 4><<<grid, kGdnWarps * 32, 0, st>>>(
          q, k, v, p.log_alpha, p.beta, p.lam, p.out, p.H, p.T, p.L, p.dv, p.cu_seqlens, p.status);
      break;
  }
  return cudaGetLastError();
}

}  // namespace

bool gdn_supports(int dk, int dv, int T) {
  return (dk == 32 || dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128) &&
         T <= (1 << (kGdnMaxLev - 1));
}

cudaError_t gdn_forward(const GdnProblem& p, cudaStream_t st) {
  if (!gdn_supports(p.dk, p.dv, p.T)) return cudaErrorNotSupported;
  main_kernel_begin(st);
  const cudaError_t e = p.in_dtype == LLATTN_BF16 ? launch<__nv_bfloat16>(p, st) : launch<float>(p, st);
  main_kernel_end(st);
  count_launch();
  return e;
}

}  // namespace llattn
