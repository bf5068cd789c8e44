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
//
// A level with no bucket holds an all-zero state, and the transition keeps it zero, so the
// transition runs over all levels without branches.  Their 16 dot products k . s_l are then
// reduced together: a butterfly that halves the set of values each lane carries at every
// step (16 shuffles in all, 5 dependent steps), after which lanes 2i and 2i + 1 hold the
// total of level i + 1, and one shuffle per level brings it back to every lane.
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
constexpr int kGdnMaxLev = 17;            // levels held at most (T <= 65536)

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Sums of 16 values over the warp: v[i] per lane in, the total of value i on every lane out.
// Step with offset o (16, 8, 4, 2) keeps half of the values each lane carries - the upper half
// where lane bit log2(o) is set - adding the partner's copy of that half and sending it the
// other half; the last step (offset 1) completes the sum.  Lanes 2i, 2i + 1 then hold total i.
__device__ __forceinline__ void warp_sum16(float (&v)[16], int lane) {
  const unsigned full = 0xffffffffu;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = lane & 16;
    const float keep = up ? v[i + 8] : v[i], send = up ? v[i] : v[i + 8];
    v[i] = keep + __shfl_xor_sync(full, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = lane & 8;
    const float keep = up ? v[i + 4] : v[i], send = up ? v[i] : v[i + 4];
    v[i] = keep + __shfl_xor_sync(full, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = lane & 4;
    const float keep = up ? v[i + 2] : v[i], send = up ? v[i] : v[i + 2];
    v[i] = keep + __shfl_xor_sync(full, send, 4);
  }
  {
    const bool up = lane & 2;
    const float keep = up ? v[1] : v[0], send = up ? v[0] : v[1];
    v[0] = keep + __shfl_xor_sync(full, send, 2);
  }
  v[0] += __shfl_xor_sync(full, v[0], 1);
  const float tot = v[0];   // total of value (lane >> 1) & 15
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __shfl_sync(full, tot, 2 * i);
}

// Promotion: levels 0..m merge into level m + 1 and empty (m = trailing one bits of t).  A
// switch on m (uniform over the warp) keeps every register index a constant.
template <int R, int NL, int M>
__device__ __forceinline__ void promote(float (&s)[NL][R]) {
  float sum[R];
#pragma unroll
  for (int r = 0; r < R; ++r) sum[r] = 0.f;
#pragma unroll
  for (int l = 0; l <= M; ++l)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      sum[r] += s[l][r];
      s[l][r] = 0.f;
    }
#pragma unroll
  for (int r = 0; r < R; ++r) s[M + 1][r] = sum[r];
}

// m <= NL - 2 for positions t + 1 < 2^(NL - 1); the cases past that are never taken
template <int R, int NL>
__device__ __forceinline__ void promote_m(float (&s)[NL][R], int m) {
#define LLATTN_GDN_PROMOTE(M) \
  case M:                     \
    if constexpr (M <= NL - 2) promote<R, NL, M>(s); \
    break;
  switch (m) {
    LLATTN_GDN_PROMOTE(0) LLATTN_GDN_PROMOTE(1) LLATTN_GDN_PROMOTE(2) LLATTN_GDN_PROMOTE(3)
    LLATTN_GDN_PROMOTE(4) LLATTN_GDN_PROMOTE(5) LLATTN_GDN_PROMOTE(6) LLATTN_GDN_PROMOTE(7)
    LLATTN_GDN_PROMOTE(8) LLATTN_GDN_PROMOTE(9) LLATTN_GDN_PROMOTE(10) LLATTN_GDN_PROMOTE(11)
    LLATTN_GDN_PROMOTE(12) LLATTN_GDN_PROMOTE(13) LLATTN_GDN_PROMOTE(14) LLATTN_GDN_PROMOTE(15)
    default: break;
  }
#undef LLATTN_GDN_PROMOTE
}

// R = d_k / 32 rows of each column per lane; NL = levels held (sequences up to 2^(NL-1) tokens)
template <typename TIn, int R, int NL>
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

  static_assert(NL >= 2 && NL <= kGdnMaxLev, "the batched reduction takes up to 16 levels");
  float s[NL][R];
#pragma unroll
  for (int l = 0; l < NL; ++l)
#pragma unroll
    for (int r = 0; r < R; ++r) s[l][r] = 0.f;
  uint32_t live = 0;   // bit l: level l holds a state (the binary counter of positions)

  // the inputs of token t are loaded during token t - 1 (their latency hides behind its work);
  // lane l holds lam[t, l] (one coalesced load), shuffled to every lane by level
  float kr[R], qr[R], a_t = 0.f, b_t = 0.f, v_t = 0.f, lam_t = 0.f;
  auto load = [&](int t, float (&kk)[R], float (&qq)[R], float& aa, float& bb, float& vv, float& ll) {
    const long long base = (sp.start + t) * H + h;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      kk[r] = ld_in(k + base * DK + r * 32 + lane);
      qq[r] = ld_in(q + base * DK + r * 32 + lane);
    }
    aa = __ldg(log_alpha + base);
    bb = __ldg(beta + base);
    vv = ld_in(v + base * dv + col);
    ll = lane < L ? __ldg(lam + base * L + lane) : 0.f;
  };
  load(0, kr, qr, a_t, b_t, v_t, lam_t);

  for (int t = 0; t < sp.len; ++t) {
    float nk[R], nq[R], na = 0.f, nb = 0.f, nv = 0.f, nl = 0.f;
    if (t + 1 < sp.len) load(t + 1, nk, nq, na, nb, nv, nl);
    const float a = __expf(a_t), b = b_t;
    // 1. transition of levels 1..NL-1 (level 0 is rewritten below); empty levels stay zero
    {
      float p[16];
#pragma unroll
      for (int l = 1; l <= 16; ++l) {
        p[l - 1] = 0.f;
        if (l < NL) {
#pragma unroll
          for (int r = 0; r < R; ++r) p[l - 1] += kr[r] * s[l][r];
        }
      }
      warp_sum16(p, lane);
#pragma unroll
      for (int l = 1; l < NL; ++l) {
        const float pb = p[l - 1] * b;
#pragma unroll
        for (int r = 0; r < R; ++r) s[l][r] = a * (s[l][r] - pb * kr[r]);
      }
    }
    // 2. the new token's write
#pragma unroll
    for (int r = 0; r < R; ++r) s[0][r] = b * kr[r] * v_t;
    live |= 1u;
    // 3. readout: sum over occupied levels of lam[t, l] (q . s_l)
    float acc = 0.f;
#pragma unroll
    for (int l = 0; l < NL; ++l) {
      if (!((live >> l) & 1u)) continue;   // uniform over the warp; lam past L is never read
      const float wl = __shfl_sync(0xffffffffu, lam_t, l);
      float p = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) p += qr[r] * s[l][r];
      acc += wl * p;
    }
    acc = warp_sum(acc);
    if (lane == 0) out[((sp.start + t) * H + h) * dv + col] = acc;
    // 4. promotion: levels 0..m into m + 1, m = trailing one bits of t
    if (t + 1 < sp.len) {
      const int m = __ffs(~t) - 1;
      promote_m<R, NL>(s, m);
      live = (live & ~((2u << m) - 1u)) | (1u << (m + 1));
#pragma unroll
      for (int r = 0; r < R; ++r) {
        kr[r] = nk[r];
        qr[r] = nq[r];
      }
      a_t = na;
      b_t = nb;
      v_t = nv;
      lam_t = nl;
    }
  }
}

template <typename TIn, int R, int NL>
void launch_r(const GdnProblem& p, const dim3& grid, cudaStream_t st) {
  gdn_recurrent_kernel<TIn, R, NL><<<grid, kGdnWarps * 32, 0, st>>>(
      static_cast<const TIn*>(p.q), static_cast<const TIn*>(p.k), static_cast<const TIn*>(p.v),
      p.log_alpha, p.beta, p.lam, p.out, p.H, p.T, p.L, p.dv, p.cu_seqlens, p.status);
}

// Levels held: 12 for sequences up to 2048 tokens, 14 up to 8192, 17 up to 65536 (level l >= 1
// is occupied only at positions t >= 2^(l-1)).
template <typename TIn, int R>
void launch_nl(const GdnProblem& p, const dim3& grid, cudaStream_t st) {
  if (p.T <= 2048) launch_r<TIn, R, 12>(p, grid, st);
  else if (p.T <= 8192) launch_r<TIn, R, 14>(p, grid, st);
  else launch_r<TIn, R, kGdnMaxLev>(p, grid, st);
}

template <typename TIn>
cudaError_t launch(const GdnProblem& p, cudaStream_t st) {
  const dim3 grid((p.dv + kGdnWarps - 1) / kGdnWarps, p.H, p.nseq);
  switch (p.dk) {
    case 32: launch_nl<TIn, 1>(p, grid, st); break;
    case 64: launch_nl<TIn, 2>(p, grid, st); break;
    default: launch_nl<TIn, 4>(p, grid, st); break;
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
