// Backward pass of log-linear attention (Mamba-2 form): the gradients of sum(dout * out) with
// respect to q, k, v, log_a and lam.
//
// Log-Linear Attention (gist.science summaries, Italian "Sommario tecnico" section 2, "Matrici
// Gerarchiche"): the output is ((Q K^T) .* M_H) V with M_H a hierarchical (HODLR) mask.  Read
// level by level, M_H has a simple block form: at level l >= 1 the positions fall into aligned
// blocks of 2^l tokens, and every key s in a block's left half meets every query t in its right
// half at level l, with weight lam[t, l] * exp(g_t - g_s) (g the inclusive prefix sum of log_a).
// With m the last position of the left half, exp(g_t - g_s) = exp(g_t - g_m) * exp(g_m - g_s),
// so each block's interaction has rank d and the backward needs, per block, only
//
//   S = sum over left-half s of exp(g_m - g_s) k_s v_s^T          (d x d)
//   U = sum over right-half t of lam[t,l] exp(g_t - g_m) q_t do_t^T (d x d)
//
// from which, for t in the right half and s in the left half,
//
//   w_t = exp(g_t - g_m) S do_t,    dlam[t, l] = q_t . w_t,    dq_t += lam[t, l] w_t,
//   dk_s += exp(g_m - g_s) U v_s,   dv_s += exp(g_m - g_s) U^T k_s,
//
// and dlam[s, l] = 0 on the left half (a left-half token has no partner at that level).
// Levels 0..5 (pairs inside an aligned 32-token tile) are done densely per tile: the score and
// gradient-score tiles, the mask, and the three small products.  The gate gradient follows from
// the row and column sums of the exponent's gradient, which equal q_t . dq_t and k_t . dk_t:
// dg_t = q_t . dq_t - k_t . dk_t, and dlog_a[r] = sum over t >= r of dg_t.
//
// Kernels, in stream order: the prefix sums g (fp64: the differences of long prefix sums must
// stay exact), the dense tiles (they initialise dq, dk, dv and dlam[:, 0..5]), one launch per
// level 6..L-1 (each token sits in one block per level, so the updates of one launch never
// collide), then dg per (token, head) and its reverse scan for dlog_a.  Arithmetic is fp32 on CUDA
// cores, d = dk = dv in {32, 64, 128}; with bf16 inputs at d = 64 the pair interactions (dense
// tiles and levels) run on the tensor cores instead (llattn_bwd_tc.cu).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include <atomic>

#include "../../include/llattn.h"
#include "llattn_bwd.h"
#include "llattn_common.cuh"
#include "llattn_internal.h"

namespace llattn {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kTile = 32;        // dense tile: levels 0..5
constexpr int kDenseLevels = 6;
constexpr int kThreads = 256;

// ---- g: inclusive prefix sums of log_a per (sequence, head), one CTA each ----
// Each thread sums a contiguous segment of the sequence, a block scan of the segment totals
// gives every segment its offset, and the thread writes its segment's prefix sums (fp64).
__global__ void __launch_bounds__(kThreads) bwd_prefix_g(BwdProblem p, double* g) {
  __shared__ double s_part[kThreads];
  const int h = blockIdx.x, sq = blockIdx.y, tid = threadIdx.x;
  const SeqSpan sp = seq_span(sq, p.T, p.cu_seqlens, p.status);
  const int seg = (sp.len + kThreads - 1) / kThreads;
  const int t0 = min(tid * seg, sp.len), t1 = min(t0 + seg, sp.len);
  const float* la = p.log_a + (size_t)sp.start * p.H + h;   // token t at la[t * H]
  double* gg = g + (size_t)sq * p.T * p.H + h;              // local position t at gg[t * H]
  // segments of up to 32 tokens (T <= 8192) stay in registers between the two walks
  constexpr int kReg = 32;
  const bool in_reg = seg <= kReg;
  float xr[kReg];
  double sum = 0.0;
  if (in_reg) {
#pragma unroll
    for (int i = 0; i < kReg; ++i) {
      xr[i] = t0 + i < t1 ? la[(size_t)(t0 + i) * p.H] : 0.f;
      sum += (double)xr[i];
    }
  } else {
    for (int t = t0; t < t1; ++t) sum += (double)la[(size_t)t * p.H];
  }
  s_part[tid] = sum;
  __syncthreads();
  // inclusive prefix sums of the per-thread totals (Hillis-Steele)
  for (int off = 1; off < kThreads; off <<= 1) {
    const double y = tid >= off ? s_part[tid - off] : 0.0;
    __syncthreads();
    s_part[tid] += y;
    __syncthreads();
  }
  double run = tid > 0 ? s_part[tid - 1] : 0.0;   // everything before this segment
  if (in_reg) {
#pragma unroll
    for (int i = 0; i < kReg; ++i) {
      run += (double)xr[i];
      if (t0 + i < t1) gg[(size_t)(t0 + i) * p.H] = run;
    }
  } else {
    for (int t = t0; t < t1; ++t) {
      run += (double)la[(size_t)t * p.H];
      gg[(size_t)t * p.H] = run;
    }
  }
}

// ---- levels 0..5: dense 32 x 32 tiles ----
// Dynamic shared memory of the dense tile kernel (over the 48 KB static limit at D = 128).
template <int D>
constexpr size_t dense_smem_bytes() {
  return kTile * sizeof(double) + (4 * kTile * (D + 1) + 3 * kTile * (kTile + 1) +
                                   kTile * kDenseLevels) * sizeof(float);
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kThreads) bwd_dense_tile(BwdProblem p, const double* g) {
  extern __shared__ __align__(16) unsigned char dsm[];
  double* s_g = reinterpret_cast<double*>(dsm);                          // [kTile]
  float (*s_q)[D + 1] = reinterpret_cast<float (*)[D + 1]>(dsm + kTile * sizeof(double));
  float (*s_k)[D + 1] = s_q + kTile;
  float (*s_v)[D + 1] = s_k + kTile;
  float (*s_do)[D + 1] = s_v + kTile;
  float (*s_pm)[kTile + 1] = reinterpret_cast<float (*)[kTile + 1]>(s_do + kTile);  // (do_i . v_j) M
  float (*s_pa)[kTile + 1] = s_pm + kTile;   // (q_i . k_j) M[i, j]
  float (*s_x)[kTile + 1] = s_pa + kTile;    // (do_i . v_j)(q_i . k_j) exp(g_i - g_j)
  float (*s_lam)[kDenseLevels] = reinterpret_cast<float (*)[kDenseLevels]>(s_x + kTile);

  const int tile = blockIdx.x, h = blockIdx.y, sq = blockIdx.z, tid = threadIdx.x;
  const SeqSpan sp = seq_span(sq, p.T, p.cu_seqlens, p.status);
  const int t0 = tile * kTile;
  if (t0 >= sp.len) return;
  const int n = min(kTile, sp.len - t0);
  const Tin* q = static_cast<const Tin*>(p.q);
  const Tin* k = static_cast<const Tin*>(p.k);
  const Tin* v = static_cast<const Tin*>(p.v);
  const Tin* dout = static_cast<const Tin*>(p.dout);
  const size_t row0 = (size_t)(sp.start + t0) * p.H + h;  // row of token t0; next token + H

  for (int e = tid; e < kTile * D; e += kThreads) {
    const int i = e / D, c = e % D;
    const bool ok = i < n;
    const size_t off = (row0 + (size_t)i * p.H) * D + c;
    s_q[i][c] = ok ? ld_in(q + off) : 0.f;
    s_k[i][c] = ok ? ld_in(k + off) : 0.f;
    s_v[i][c] = ok ? ld_in(v + off) : 0.f;
    s_do[i][c] = ok ? ld_in(dout + off) : 0.f;
  }
  const size_t grow0 = ((size_t)sq * p.T + t0) * p.H + h;  // g is indexed by local position
  if (tid < kTile) s_g[tid] = tid < n ? g[grow0 + (size_t)tid * p.H] : 0.0;
  for (int e = tid; e < kTile * kDenseLevels; e += kThreads) {
    const int i = e / kDenseLevels, l = e % kDenseLevels;
    s_lam[i][l] = (i < n && l < p.L) ? p.lam[(row0 + (size_t)i * p.H) * p.L + l] : 0.f;
  }
  __syncthreads();

  // pair tiles; positions t0+i, t0+j share the tile, so their level is that of (i, j)
  for (int e = tid; e < kTile * kTile; e += kThreads) {
    const int i = e / kTile, j = e % kTile;
    float pm = 0.f, pa = 0.f, x = 0.f;
    if (j <= i && i < n) {
      float a = 0.f, b = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        a = fmaf(s_q[i][c], s_k[j][c], a);
        b = fmaf(s_do[i][c], s_v[j][c], b);
      }
      const float E = expf((float)(s_g[i] - s_g[j]));
      const float m = s_lam[i][fenwick_level(i, j)] * E;
      pm = b * m;
      pa = a * m;
      x = a * b * E;
    }
    s_pm[i][j] = pm;
    s_pa[i][j] = pa;
    s_x[i][j] = x;
  }
  __syncthreads();

  // dlam[:, 0..5]: sums of s_x over each level's keys
  if (tid < kTile * kDenseLevels) {
    const int i = tid / kDenseLevels, l = tid % kDenseLevels;
    if (i < n && l < p.L) {
      float s = 0.f;
      for (int j = 0; j <= i; ++j)
        if (fenwick_level(i, j) == l) s += s_x[i][j];
      p.dlam[(row0 + (size_t)i * p.H) * p.L + l] = s;
    }
  }
  // dq = Pm K, dk = Pm^T Q, dv = Pa^T dO  (they start the accumulation of the later levels)
  for (int e = tid; e < kTile * D; e += kThreads) {
    const int i = e / D, c = e % D;
    if (i >= n) continue;
    float aq = 0.f, ak = 0.f, av = 0.f;
#pragma unroll 8
    for (int j = 0; j < kTile; ++j) {
      aq = fmaf(s_pm[i][j], s_k[j][c], aq);
      ak = fmaf(s_pm[j][i], s_q[j][c], ak);
      av = fmaf(s_pa[j][i], s_do[j][c], av);
    }
    const size_t off = (row0 + (size_t)i * p.H) * D + c;
    p.dq[off] = aq;
    p.dk[off] = ak;
    p.dv[off] = av;
  }
}

// ---- one level >= 6: the rank-d interaction of each aligned block's halves ----
// Dynamic shared memory of the level kernel.  Up to D = 64 the staged rows of phase 1 share
// space with S and U, and each thread holds both states' accumulators; at D = 128 (64
// accumulators per state per thread) S is stored after its pass so U can reuse the registers,
// which needs the staging space apart from S.
template <int D>
__host__ __device__ constexpr bool level_split() { return D > 64; }
template <int D>
constexpr size_t level_smem_bytes() {
  return (32 + 2 * D * (D + 1) + (level_split<D>() ? 2 * 32 * D : 0)) * sizeof(float);
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kThreads) bwd_level_block(BwdProblem p, const double* g, int lvl) {
  constexpr int R = D * D / kThreads;  // state elements per thread
  constexpr int E = D / 8;             // elements per lane of an 8-lane token group
  constexpr bool kSplit = level_split<D>();
  extern __shared__ __align__(16) float lsm[];
  float* s_w = lsm;                                                       // [32]
  float* s_mem = lsm + 32;              // phase 2: S and U; phase 1: staged rows (unless kSplit)
  float* s_stage = kSplit ? s_mem + 2 * D * (D + 1) : s_mem;
  float (*s_x)[D] = reinterpret_cast<float (*)[D]>(s_stage);              // [32][D]
  float (*s_y)[D] = reinterpret_cast<float (*)[D]>(s_stage + 32 * D);     // [32][D]
  float (*s_S)[D + 1] = reinterpret_cast<float (*)[D + 1]>(s_mem);       // [D][D+1]
  float (*s_U)[D + 1] = reinterpret_cast<float (*)[D + 1]>(s_mem + D * (D + 1));

  const int blk = blockIdx.x, h = blockIdx.y, sq = blockIdx.z, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const SeqSpan sp = seq_span(sq, p.T, p.cu_seqlens, p.status);
  const int half = 1 << (lvl - 1);
  const long long a0 = (long long)blk << lvl;
  if (a0 >= sp.len) return;
  const int lo = (int)a0;
  const int mid = lo + half;                           // first token of the right half
  const int lend = min(mid, sp.len);                   // left half [lo, lend)
  const int rend = (int)min((long long)lo + 2 * half, (long long)sp.len);  // right [mid, rend)
  const Tin* q = static_cast<const Tin*>(p.q);
  const Tin* k = static_cast<const Tin*>(p.k);
  const Tin* v = static_cast<const Tin*>(p.v);
  const Tin* dout = static_cast<const Tin*>(p.dout);
  auto row = [&](int t) { return (size_t)(sp.start + t) * p.H + h; };
  auto grow = [&](int t) { return ((size_t)sq * p.T + t) * p.H + h; };

  for (int t = lo + tid; t < lend; t += kThreads) p.dlam[row(t) * p.L + lvl] = 0.f;
  if (mid >= sp.len) return;  // no right half: nothing meets at this level
  const double gm = g[grow(mid - 1)];

  // phase 1: S over the left half, U over the right half
  float accS[R], accU[kSplit ? 1 : R];
#pragma unroll
  for (int r = 0; r < R; ++r) accS[r] = 0.f;
#pragma unroll
  for (int r = 0; r < (kSplit ? 1 : R); ++r) accU[r] = 0.f;
  for (int pass = 0; pass < 2; ++pass) {
    const int b0 = pass == 0 ? lo : mid, b1 = pass == 0 ? lend : rend;
    for (int base = b0; base < b1; base += 32) {
      if (tid < 32) {
        const int t = base + tid;
        float w = 0.f;
        if (t < b1)
          w = pass == 0 ? expf((float)(gm - g[grow(t)]))
                        : p.lam[row(t) * p.L + lvl] * expf((float)(g[grow(t)] - gm));
        s_w[tid] = w;
      }
      __syncthreads();
      for (int e = tid; e < 32 * D; e += kThreads) {
        const int i = e / D, c = e % D;
        const int t = base + i;
        float x = 0.f, y = 0.f;
        if (t < b1) {
          const size_t off = row(t) * D + c;
          x = s_w[i] * (pass == 0 ? ld_in(k + off) : ld_in(q + off));
          y = pass == 0 ? ld_in(v + off) : ld_in(dout + off);
        }
        s_x[i][c] = x;
        s_y[i][c] = y;
      }
      __syncthreads();
      const int nrow = min(32, b1 - base);
      for (int i = 0; i < nrow; ++i) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int e = tid + r * kThreads, a = e / D, b = e % D;
          if (kSplit || pass == 0) accS[r] = fmaf(s_x[i][a], s_y[i][b], accS[r]);
          else accU[r] = fmaf(s_x[i][a], s_y[i][b], accU[r]);
        }
      }
      __syncthreads();
    }
    if (kSplit) {
      // this pass's state goes to its own region; the registers start over for the next one
      float (*dst)[D + 1] = pass == 0 ? s_S : s_U;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int e = tid + r * kThreads, a = e / D, b = e % D;
        dst[a][b] = accS[r];
        accS[r] = 0.f;
      }
    }
  }
  if (!kSplit) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = tid + r * kThreads, a = e / D, b = e % D;
      s_S[a][b] = accS[r];
      s_U[a][b] = accU[kSplit ? 0 : r];
    }
  }
  __syncthreads();

  // phase 2: 32 tokens per pass, four per warp, one 8-lane group per token.  Lane j of a group
  // owns elements j, j+8, j+16, ... (E of them), so the 8 lanes read 8 consecutive words of a
  // state row (no bank conflicts), and the element b of the token's vector that a product needs
  // comes from lane b % 8 of the group, register b / 8.
  const int grp = lane >> 3, j = lane & 7, src0 = lane & ~7;
  // right half: w = e^{g_t - g_m} S do_t;  dlam[t, l] = q_t . w;  dq_t += lam[t, l] w
  for (int base = mid; base < rend; base += 32) {
    const int t = base + warp * 4 + grp;
    const bool ok = t < rend;
    const size_t rr = ok ? row(t) : 0;
    float xd[E], xq[E], w[E];
#pragma unroll
    for (int m = 0; m < E; ++m) {
      xd[m] = ok ? ld_in(dout + rr * D + j + 8 * m) : 0.f;
      xq[m] = ok ? ld_in(q + rr * D + j + 8 * m) : 0.f;
      w[m] = 0.f;
    }
#pragma unroll
    for (int b = 0; b < D; ++b) {
      const float db = __shfl_sync(kFull, xd[b >> 3], src0 | (b & 7));
#pragma unroll
      for (int m = 0; m < E; ++m) w[m] = fmaf(s_S[j + 8 * m][b], db, w[m]);
    }
    const float sc = ok ? expf((float)(g[grow(ok ? t : mid)] - gm)) : 0.f;
    const float lam = ok ? p.lam[rr * p.L + lvl] : 0.f;
    float dl = 0.f;
#pragma unroll
    for (int m = 0; m < E; ++m) {
      w[m] *= sc;
      dl = fmaf(xq[m], w[m], dl);
    }
    dl += __shfl_xor_sync(kFull, dl, 1);
    dl += __shfl_xor_sync(kFull, dl, 2);
    dl += __shfl_xor_sync(kFull, dl, 4);
    if (ok) {
#pragma unroll
      for (int m = 0; m < E; ++m) p.dq[rr * D + j + 8 * m] += lam * w[m];
      if (j == 0) p.dlam[rr * p.L + lvl] = dl;
    }
  }
  // left half: dk_s += e^{g_m - g_s} U v_s;  dv_s += e^{g_m - g_s} U^T k_s
  for (int base = lo; base < lend; base += 32) {
    const int s = base + warp * 4 + grp;
    const bool ok = s < lend;
    const size_t rr = ok ? row(s) : 0;
    float xv[E], xk[E], ak[E], av[E];
#pragma unroll
    for (int m = 0; m < E; ++m) {
      xv[m] = ok ? ld_in(v + rr * D + j + 8 * m) : 0.f;
      xk[m] = ok ? ld_in(k + rr * D + j + 8 * m) : 0.f;
      ak[m] = av[m] = 0.f;
    }
#pragma unroll
    for (int b = 0; b < D; ++b) {
      const float vb = __shfl_sync(kFull, xv[b >> 3], src0 | (b & 7));
      const float kb = __shfl_sync(kFull, xk[b >> 3], src0 | (b & 7));
#pragma unroll
      for (int m = 0; m < E; ++m) {
        ak[m] = fmaf(s_U[j + 8 * m][b], vb, ak[m]);   // (U v)[a],   a = j + 8m
        av[m] = fmaf(s_U[b][j + 8 * m], kb, av[m]);   // (U^T k)[c], c = j + 8m
      }
    }
    if (ok) {
      const float sc = expf((float)(gm - g[grow(s)]));
#pragma unroll
      for (int m = 0; m < E; ++m) {
        p.dk[rr * D + j + 8 * m] += sc * ak[m];
        p.dv[rr * D + j + 8 * m] += sc * av[m];
      }
    }
  }
}

// ---- dlog_a: dg_t = q_t . dq_t - k_t . dk_t per (token, head), one warp each, into dlog_a ----
template <typename Tin, int D>
__global__ void __launch_bounds__(kThreads) bwd_dg(BwdProblem p) {
  const int h = blockIdx.y, sq = blockIdx.z, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  const SeqSpan sp = seq_span(sq, p.T, p.cu_seqlens, p.status);
  if (t >= sp.len) return;
  const Tin* q = static_cast<const Tin*>(p.q);
  const Tin* k = static_cast<const Tin*>(p.k);
  const size_t rr = (size_t)(sp.start + t) * p.H + h;
  float a = 0.f;
#pragma unroll
  for (int c = lane; c < D; c += 32)
    a += ld_in(q + rr * D + c) * p.dq[rr * D + c] - ld_in(k + rr * D + c) * p.dk[rr * D + c];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(kFull, a, off);
  if (lane == 0) p.dlog_a[rr] = a;
}

// ---- dlog_a[r] = sum over t >= r of dg_t, in place, one CTA per (sequence, head) ----
__global__ void __launch_bounds__(kThreads) bwd_suffix_scan(BwdProblem p) {
  __shared__ double s_part[kThreads];
  const int h = blockIdx.x, sq = blockIdx.y, tid = threadIdx.x;
  const SeqSpan sp = seq_span(sq, p.T, p.cu_seqlens, p.status);
  const int seg = (sp.len + kThreads - 1) / kThreads;
  const int t0 = min(tid * seg, sp.len), t1 = min(t0 + seg, sp.len);
  float* x = p.dlog_a + (size_t)sp.start * p.H + h;   // token t at x[t * H]
  // segments of up to 32 tokens (T <= 8192) stay in registers between the two walks
  constexpr int kReg = 32;
  const bool in_reg = seg <= kReg;
  float xr[kReg];
  double sum = 0.0;
  if (in_reg) {
#pragma unroll
    for (int i = 0; i < kReg; ++i) {
      xr[i] = t0 + i < t1 ? x[(size_t)(t0 + i) * p.H] : 0.f;
      sum += xr[i];
    }
  } else {
    for (int t = t0; t < t1; ++t) sum += x[(size_t)t * p.H];
  }
  s_part[tid] = sum;
  __syncthreads();
  // suffix sums of the per-thread totals (Hillis-Steele, reading the later entries)
  for (int off = 1; off < kThreads; off <<= 1) {
    const double y = tid + off < kThreads ? s_part[tid + off] : 0.0;
    __syncthreads();
    s_part[tid] += y;
    __syncthreads();
  }
  double run = tid + 1 < kThreads ? s_part[tid + 1] : 0.0;  // everything after this segment
  if (in_reg) {
#pragma unroll
    for (int i = kReg - 1; i >= 0; --i) {
      run += xr[i];
      if (t0 + i < t1) x[(size_t)(t0 + i) * p.H] = (float)run;
    }
  } else {
    for (int t = t1 - 1; t >= t0; --t) {
      run += x[(size_t)t * p.H];
      x[(size_t)t * p.H] = (float)run;
    }
  }
}

template <typename Tin, int D>
cudaError_t launch(const BwdProblem& p, double* g, cudaStream_t st) {
  // the dynamic shared-memory opt-in is a per-device attribute of each kernel
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load()) {
    if ((e = cudaFuncSetAttribute(bwd_dense_tile<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)dense_smem_bytes<D>())) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_level_block<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)level_smem_bytes<D>())) != cudaSuccess)
      return e;
    attr_set[dev].store(true);
  }
  const dim3 seqs(p.H, p.nseq);
  bwd_prefix_g<<<seqs, kThreads, 0, st>>>(p, g);
  int n = 1;
  if (bwd_tc_supports(p)) {
    // bf16 at d = 64: every pair interaction on the tensor cores
    if ((e = bwd_levels_tc(p, g, st)) != cudaSuccess) return e;
  } else {
    bwd_dense_tile<Tin, D><<<dim3((p.T + kTile - 1) / kTile, p.H, p.nseq), kThreads,
                             dense_smem_bytes<D>(), st>>>(p, g);
    ++n;
    for (int lvl = kDenseLevels; lvl < p.L; ++lvl, ++n) {
      const int nblk = (int)(((long long)p.T + (1ll << lvl) - 1) >> lvl);
      bwd_level_block<Tin, D><<<dim3(nblk, p.H, p.nseq), kThreads, level_smem_bytes<D>(), st>>>(
          p, g, lvl);
    }
  }
  bwd_dg<Tin, D><<<dim3((p.T + kThreads / 32 - 1) / (kThreads / 32), p.H, p.nseq), kThreads, 0,
                   st>>>(p);
  bwd_suffix_scan<<<seqs, kThreads, 0, st>>>(p);
  count_launch(n + 2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t bwd(const BwdProblem& p, void* ws, cudaStream_t st) {
  double* g = static_cast<double*>(ws);
  main_kernel_begin(st);
  cudaError_t e;
  if (p.in_dtype == LLATTN_BF16)
    e = p.d == 32 ? launch<__nv_bfloat16, 32>(p, g, st)
                  : p.d == 64 ? launch<__nv_bfloat16, 64>(p, g, st) : launch<__nv_bfloat16, 128>(p, g, st);
  else
    e = p.d == 32 ? launch<float, 32>(p, g, st)
                  : p.d == 64 ? launch<float, 64>(p, g, st) : launch<float, 128>(p, g, st);
  main_kernel_end(st);
  return e;
}

}  // namespace llattn
