// CUDA-core (SIMT, fp32 arithmetic) chunkwise forward of log-linear attention.
//
// The chunkwise-parallel algorithm of "Log-Linear Attention" (gist.science,
// Italian "Sommario tecnico" section 2, "Forma Ricorrente e Parallelizzata",
// Training bullet; Spanish "Resumen tecnico" section 2, "Algoritmo de
// Entrenamiento (Chunk-scan)"): dense work inside each chunk of C tokens, and the
// hierarchical low-rank structure between chunks.  Between aligned chunks c' < c
// the Fenwick level depends on the chunk indices only,
//     l = 1 + log2(C) + msb(c XOR c'),
// so the keys a query chunk sees at chunk-level b (bit b of c set) form one
// dyadic block of 2^b chunks, (b, (c >> b) - 1), and the query reads that block's
// state K^T diag(decay) V once.  Three kernels:
//   1. simt_chunk_state    H_c = sum_{s in c} exp(g_end - g_s) k_s v_s^T, chunk log-decay G_c
//   2. simt_fenwick_blocks binary-counter merge of chunk states into the dyadic block
//                          states that queries read (one per even block index)
//   3. simt_intra_readout  intra-chunk masked part plus the lam-weighted readout
//                          of the block states, written to out (fp32)
// Sequences of at most 512 tokens can instead take simt_short_fwd (below), the masked form in
// one launch.
// This path is the fp32-input product path (it keeps fp32 accuracy end to end)
// and a cross-check for the tensor-core path on bf16 inputs.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "llattn_common.cuh"
#include "llattn_internal.h"
#include "../../include/llattn.h"

namespace llattn {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kMaxLevels = 32;

// ---------------------------------------------------------------------------------------------
// 1. chunk states
// ---------------------------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(kThreads)
simt_chunk_state(const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const float* __restrict__ log_a, float* __restrict__ Hws,
                 float* __restrict__ Gws, int H, int T, int dk, int dv, int C, int Nc,
                 const int* __restrict__ cu, unsigned int* status) {
  const int c = blockIdx.x, h = blockIdx.y, sq = blockIdx.z;
  const SeqSpan sp = seq_span(sq, T, cu, status);
  const int t0 = c * C;
  if (t0 >= sp.len) return;
  const int n = min(C, sp.len - t0);
  extern __shared__ float sm[];
  float* g = sm;           // C: inclusive cumsum of log_a within the chunk
  float* w = g + C;        // C: exp(g_end - g_s)
  float* Ks = w + C;       // C * dk
  float* Vs = Ks + C * dk; // C * dv
  const long long tok0 = sp.start + t0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) g[i] = log_a[(tok0 + i) * H + h];
  for (int e = threadIdx.x; e < n * dk; e += blockDim.x) {
    const int i = e / dk, d = e - i * dk;
    Ks[e] = ld_in(k + ((tok0 + i) * H + h) * dk + d);
  }
  for (int e = threadIdx.x; e < n * dv; e += blockDim.x) {
    const int i = e / dv, d = e - i * dv;
    Vs[e] = ld_in(v + ((tok0 + i) * H + h) * dv + d);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float acc = 0.f;
    for (int i = 0; i < n; ++i) { acc += g[i]; g[i] = acc; }
  }
  __syncthreads();
  const float G = g[n - 1];
  for (int i = threadIdx.x; i < n; i += blockDim.x) w[i] = expf(G - g[i]);
  __syncthreads();
  float* Hout = Hws + ((((long long)sq * H + h) * Nc + c) * dk) * dv;
  for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
    const int i = e / dv, j = e - i * dv;
    float acc = 0.f;
    for (int s = 0; s < n; ++s) acc = fmaf(Ks[s * dk + i] * w[s], Vs[s * dv + j], acc);
    Hout[e] = acc;
  }
  if (threadIdx.x == 0) Gws[((long long)sq * H + h) * Nc + c] = G;
}

// ---------------------------------------------------------------------------------------------
// 2. dyadic block states by a per-element binary counter over the chunks
// ---------------------------------------------------------------------------------------------
// Level states L_b hold, after chunk c, the blocks for the set bits of c+1, each
// relative to its own last token.  After chunk c with m trailing one bits, the
// new level-m block is H_c plus levels 0..m-1, each decayed by the log-decay of
// everything after it (the blocks below it and chunk c); that block is
// (m, ((c+1) >> m) - 1), an even index, read by chunks c+1 .. c+2^m.
__global__ void __launch_bounds__(kThreads)
simt_fenwick_blocks(const float* __restrict__ Hws, const float* __restrict__ Gws,
                    float* __restrict__ Rws, float* __restrict__ GRws, int H, int T,
                    int dkdv, int C, int Nc, int NB, const int* __restrict__ cu,
                    unsigned int* status) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int h = blockIdx.y, sq = blockIdx.z;
  const SeqSpan sp = seq_span(sq, T, cu, status);
  const int nch = (sp.len + C - 1) / C;
  if (e >= dkdv) return;
  float lv[kMaxLevels];
  float lg[kMaxLevels];
  const long long head = (long long)sq * H + h;
  const float* Hh = Hws + head * Nc * dkdv;
  const float* Gh = Gws + head * Nc;
  float* Rh = Rws + head * (long long)NB * dkdv;
  float* GRh = GRws + head * (long long)NB;
  for (int c = 0; c + 1 < nch; ++c) {
    const int m = __ffs(~c) - 1;  // trailing one bits of c
    float nw = Hh[(long long)c * dkdv + e];
    float acc = Gh[c];
    for (int b = 0; b < m; ++b) {
      nw = fmaf(expf(acc), lv[b], nw);
      acc += lg[b];
    }
    lv[m] = nw;
    lg[m] = acc;
    const int j = ((c + 1) >> m) - 1;
    const long long slot = level_offset(Nc, m) + (j >> 1);
    Rh[slot * dkdv + e] = nw;
    if (e == 0) GRh[slot] = acc;
  }
}

// ---------------------------------------------------------------------------------------------
// 3. intra-chunk part + lam-weighted readout of the block states
// ---------------------------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(kThreads)
simt_intra_readout(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, const float* __restrict__ log_a,
                   const float* __restrict__ lam, const float* __restrict__ Rws,
                   const float* __restrict__ GRws, float* __restrict__ out, int H, int T,
                   int dk, int dv, int L, int C, int logC, int Nc, int NB,
                   const int* __restrict__ cu, unsigned int* status) {
  const int c = blockIdx.x, h = blockIdx.y, sq = blockIdx.z;
  const SeqSpan sp = seq_span(sq, T, cu, status);
  const int t0 = c * C;
  if (t0 >= sp.len) return;
  const int n = min(C, sp.len - t0);
  extern __shared__ float sm[];
  float* g = sm;               // C
  float* lm = g + C;           // C * L
  float* Qs = lm + C * L;      // C * dk
  float* Ks = Qs + C * dk;     // C * dk
  float* Vs = Ks + C * dk;     // C * dv
  float* P = Vs + C * dv;      // C * C
  float* D = P + C * C;        // dk * 32 (a column tile of one block state)
  const long long tok0 = sp.start + t0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) g[i] = log_a[(tok0 + i) * H + h];
  for (int e = threadIdx.x; e < n * L; e += blockDim.x) {
    const int i = e / L, l = e - i * L;
    lm[e] = lam[((tok0 + i) * H + h) * L + l];
  }
  for (int e = threadIdx.x; e < n * dk; e += blockDim.x) {
    const int i = e / dk, d = e - i * dk;
    Qs[e] = ld_in(q + ((tok0 + i) * H + h) * dk + d);
    Ks[e] = ld_in(k + ((tok0 + i) * H + h) * dk + d);
  }
  for (int e = threadIdx.x; e < n * dv; e += blockDim.x) {
    const int i = e / dv, d = e - i * dv;
    Vs[e] = ld_in(v + ((tok0 + i) * H + h) * dv + d);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float acc = 0.f;
    for (int i = 0; i < n; ++i) { acc += g[i]; g[i] = acc; }
  }
  __syncthreads();
  // masked scores P[t][s] = lam[t, l(t,s)] * exp(g_t - g_s) * (q_t . k_s), s <= t
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int t = e / n, s = e - t * n;
    float val = 0.f;
    if (s <= t) {
      float dot = 0.f;
      for (int d = 0; d < dk; ++d) dot = fmaf(Qs[t * dk + d], Ks[s * dk + d], dot);
      val = dot * lm[t * L + fenwick_level(t, s)] * expf(g[t] - g[s]);
    }
    P[t * C + s] = val;
  }
  __syncthreads();
  // Per (t, j) outputs.  Each thread keeps up to kOutPerThread accumulators.
  const long long head = (long long)sq * H + h;
  constexpr int kOutPerThread = 32;  // C * dv <= 64 * 128 = 8192 = 32 * 256
  float acc[kOutPerThread];
  const int nout = n * dv;
#pragma unroll
  for (int r = 0; r < kOutPerThread; ++r) acc[r] = 0.f;
#pragma unroll
  for (int r = 0; r < kOutPerThread; ++r) {
    const int e = threadIdx.x + r * kThreads;
    if (e < nout) {
      const int t = e / dv, j = e - t * dv;
      float a = 0.f;
      for (int s = 0; s <= t; ++s) a = fmaf(P[t * C + s], Vs[s * dv + j], a);
      acc[r] = a;
    }
  }
  // Inter-chunk levels: bit b of c set -> block (b, (c >> b) - 1), decayed to the
  // start of chunk c by the blocks of the lower set bits (they fill the gap).
  float gap = 0.f;
  for (int b = 0; (1 << b) <= c; ++b) {
    if (!((c >> b) & 1)) continue;
    const int jb = (c >> b) - 1;
    const long long slot = level_offset(Nc, b) + (jb >> 1);
    const float* Dg = Rws + (head * NB + slot) * (long long)dk * dv;
    const int lev = 1 + logC + b;
    const float gap_b = gap;
    for (int j0 = 0; j0 < dv; j0 += 32) {
      __syncthreads();
      for (int e = threadIdx.x; e < dk * 32; e += blockDim.x) {
        const int i = e >> 5, jj = e & 31;
        D[e] = Dg[(long long)i * dv + j0 + jj];
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kOutPerThread; ++r) {
        const int e = threadIdx.x + r * kThreads;
        if (e < nout) {
          const int t = e / dv, j = e - t * dv;
          if (j >= j0 && j < j0 + 32) {
            float dot = 0.f;
            for (int i = 0; i < dk; ++i) dot = fmaf(Qs[t * dk + i], D[i * 32 + (j - j0)], dot);
            acc[r] = fmaf(lm[t * L + lev] * expf(g[t] + gap_b), dot, acc[r]);
          }
        }
      }
    }
    gap += GRws[head * NB + slot];
  }
#pragma unroll
  for (int r = 0; r < kOutPerThread; ++r) {
    const int e = threadIdx.x + r * kThreads;
    if (e < nout) {
      const int t = e / dv, j = e - t * dv;
      out[((tok0 + t) * H + h) * dv + j] = acc[r];
    }
  }
}

template <typename Tin>
cudaError_t launch_all(const Problem& p, int C, void* ws, cudaStream_t st) {
  const int Nc = (p.T + C - 1) / C;
  const int NB = total_blocks(Nc);
  const size_t dkdv = (size_t)p.dk * p.dv;
  const size_t nh = (size_t)p.nseq * p.H;
  char* base = static_cast<char*>(ws);
  float* Hws = reinterpret_cast<float*>(base);
  base += round_up(nh * Nc * dkdv * sizeof(float), 256);
  float* Gws = reinterpret_cast<float*>(base);
  base += round_up(nh * Nc * sizeof(float), 256);
  float* Rws = reinterpret_cast<float*>(base);
  base += round_up(nh * (size_t)NB * dkdv * sizeof(float), 256);
  float* GRws = reinterpret_cast<float*>(base);
  int logC = 0;
  while ((1 << logC) < C) ++logC;
  const Tin* q = static_cast<const Tin*>(p.q);
  const Tin* k = static_cast<const Tin*>(p.k);
  const Tin* v = static_cast<const Tin*>(p.v);

  const dim3 grid(Nc, p.H, p.nseq);
  const size_t sm1 = sizeof(float) * (2 * C + (size_t)C * (p.dk + p.dv));
  cudaError_t e = cudaFuncSetAttribute(simt_chunk_state<Tin>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
  if (e != cudaSuccess) return e;
  simt_chunk_state<Tin><<<grid, kThreads, sm1, st>>>(k, v, p.log_a, Hws, Gws, p.H, p.T, p.dk,
                                                      p.dv, C, Nc, p.cu_seqlens, p.status);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (Nc > 1) {
    const dim3 g2((unsigned)((dkdv + kThreads - 1) / kThreads), p.H, p.nseq);
    simt_fenwick_blocks<<<g2, kThreads, 0, st>>>(Hws, Gws, Rws, GRws, p.H, p.T, (int)dkdv, C, Nc,
                                                 NB, p.cu_seqlens, p.status);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t sm3 = sizeof(float) * ((size_t)C + (size_t)C * p.L + 2 * (size_t)C * p.dk +
                                      (size_t)C * p.dv + (size_t)C * C + (size_t)p.dk * 32);
  e = cudaFuncSetAttribute(simt_intra_readout<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sm3);
  if (e != cudaSuccess) return e;
  main_kernel_begin(st);
  simt_intra_readout<Tin><<<grid, kThreads, sm3, st>>>(q, k, v, p.log_a, p.lam, Rws, GRws, p.out,
                                                        p.H, p.T, p.dk, p.dv, p.L, C, logC, Nc,
                                                        NB, p.cu_seqlens, p.status);
  main_kernel_end(st);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// Short sequences (T <= 512): the masked quadratic form itself ("Matrici Gerarchiche": out =
// ((Q K^T) .* M_H) V), one launch.  At this size a whole sequence's keys fit a few shared-memory
// tiles, and the three chunkwise launches cost more than the arithmetic.
// A row block is 16 query rows of a (sequence, head), 16 threads per row.  Those 16 split the
// columns into CL interleaved slices (CL = max(dk, dv) / 32, so a slice holds at most 32
// columns) and the keys of each tile into KL = 16 / CL strided subsets: a thread forms the q.k
// dot product of its keys over its column slice (reduced over the CL slices by shuffles), and
// accumulates its keys' weighted v into its own slice of the output row.  The KL partial rows
// are summed by shuffles at the end.  Keys arrive in shared-memory tiles of 32 rows (16 for
// max(dk, dv) = 128), the next tile read into registers while the current one is used; a row is
// padded by CL floats, so the 16 lanes of a row read 16 different banks.
// Each thread reads a whole k and v row from shared memory per key, so a row block's cost is
// its shared-memory reads.  When the grid is small, a thread-block cluster of KS CTAs (2 or 4)
// shares one row block: rank r takes the key tiles r, r + KS, ..., and rank 0 adds the ranks'
// partial rows in rank order through distributed shared memory.
// The prefix sums g stay fp64 in shared memory, so the decay exp(g_t - g_s) is a difference of
// exact values.
// ---------------------------------------------------------------------------------------------
constexpr int kShortMaxT = 512;
constexpr int kShortRows = 16;
constexpr int kShortLanes = kThreads / kShortRows;   // 16 threads per query row

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads)
simt_short_fwd(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
               const float* __restrict__ log_a, const float* __restrict__ lam,
               float* __restrict__ out, int H, int T, int L, int KS, const int* __restrict__ cu,
               unsigned int* status) {
  constexpr int CL = (DK > DV ? DK : DV) / 32;      // column slices: 1, 2 or 4
  constexpr int KL = kShortLanes / CL;              // key subsets: 16, 8 or 4
  constexpr int TILE = CL == 4 ? 16 : 32;           // keys per tile
  constexpr int SK = DK / CL, SV = DV / CL;         // columns of this thread's slices
  constexpr int PK = DK + CL, PV = DV + CL;         // padded shared-memory rows
  constexpr int FK = TILE * DK / kThreads;          // tile elements each thread fetches
  constexpr int FV = TILE * DV / kThreads;
  static_assert(CL * KL == kShortLanes && FK >= 1 && FV >= 1 && TILE % KL == 0, "short split");
  __shared__ double s_g[kShortMaxT];
  __shared__ float s_k[TILE * PK], s_v[TILE * PV];
  __shared__ float s_lam[kShortRows][kMaxLevels / 2 + 1];
  __shared__ float s_o[kShortRows * DV];            // this CTA's partial rows
  const int rank = KS > 1 ? (int)(blockIdx.x % KS) : 0;
  const int rb = blockIdx.x / KS, h = blockIdx.y, sq = blockIdx.z, tid = threadIdx.x;
  const SeqSpan sp = seq_span(sq, T, cu, status);
  const int r0 = rb * kShortRows;
  if (r0 >= sp.len) return;                     // the whole cluster leaves together
  const int n = min(r0 + kShortRows, sp.len);   // keys 0 .. n-1 reach the rows r0 .. n-1
  auto row = [&](int t) { return (size_t)(sp.start + t) * H + h; };

  // a key tile into registers (element e of the tile is row e / D, column e % D)
  float fk[FK], fv[FV];
  auto fetch = [&](int k0) {
    const int m = min(TILE, n - k0);
#pragma unroll
    for (int u = 0; u < FK; ++u) {
      const int e = tid + u * kThreads, i = e / DK;
      fk[u] = i < m ? ld_in(k + row(k0 + i) * DK + (e % DK)) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < FV; ++u) {
      const int e = tid + u * kThreads, i = e / DV;
      fv[u] = i < m ? ld_in(v + row(k0 + i) * DV + (e % DV)) : 0.f;
    }
  };
  const int kfirst = rank * TILE, kstep = KS * TILE;
  if (kfirst < n) fetch(kfirst);

  // this thread's query row and column slice, and the row block's lam (loads in flight together
  // with the first key tile and log a)
  const int r = tid / kShortLanes, j = tid % kShortLanes, t = r0 + r;
  const int cl = j % CL, kl = j / CL;
  const bool row_ok = t < n;
  for (int e = tid; e < kShortRows * L; e += kThreads) {
    const int rr = e / L, l = e % L;
    s_lam[rr][l] = r0 + rr < n ? __ldg(lam + row(r0 + rr) * L + l) : 0.f;
  }
  float qs[SK];
#pragma unroll
  for (int e = 0; e < SK; ++e) qs[e] = row_ok ? ld_in(q + row(t) * DK + cl + CL * e) : 0.f;

  // prefix sums of log a over positions 0 .. n-1: per-thread pairs, a warp scan, a block carry
  {
    const int i0 = 2 * tid;
    const double a = i0 < n ? (double)__ldg(log_a + row(i0)) : 0.0;
    const double b = i0 + 1 < n ? (double)__ldg(log_a + row(i0 + 1)) : 0.0;
    double x = a + b;
    const int lane = tid & 31, w = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    __shared__ double s_w[kThreads / 32];
    if (lane == 31) s_w[w] = x;
    __syncthreads();
    double off = 0.0;
    for (int u = 0; u < w; ++u) off += s_w[u];
    x += off;                                   // inclusive sum through position i0 + 1
    if (i0 < n) s_g[i0] = x - b;
    if (i0 + 1 < n) s_g[i0 + 1] = x;
  }
  float acc[SV];
#pragma unroll
  for (int e = 0; e < SV; ++e) acc[e] = 0.f;
  __syncthreads();
  const double gt = row_ok ? s_g[t] : 0.0;

  for (int k0 = kfirst; k0 < n; k0 += kstep) {
    __syncthreads();   // the previous tile is consumed
#pragma unroll
    for (int u = 0; u < FK; ++u) {
      const int e = tid + u * kThreads;
      s_k[(e / DK) * PK + e % DK] = fk[u];
    }
#pragma unroll
    for (int u = 0; u < FV; ++u) {
      const int e = tid + u * kThreads;
      s_v[(e / DV) * PV + e % DV] = fv[u];
    }
    __syncthreads();
    if (k0 + kstep < n) fetch(k0 + kstep);
#pragma unroll
    for (int ii = 0; ii < TILE / KL; ++ii) {
      const int i = kl + KL * ii, s = k0 + i;
      const float* kr = s_k + i * PK + cl;
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int e = 0; e < SK; e += 2) {
        d0 = fmaf(qs[e], kr[CL * e], d0);
        if (e + 1 < SK) d1 = fmaf(qs[e + 1], kr[CL * (e + 1)], d1);
      }
      float d = d0 + d1;
#pragma unroll
      for (int o = 1; o < CL; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      if (row_ok && s <= t) {
        const int lev = s == t ? 0 : 32 - __clz(t ^ s);
        const float wgt = s_lam[r][lev] * expf((float)(gt - s_g[s])) * d;
        const float* vr = s_v + i * PV + cl;
#pragma unroll
        for (int e = 0; e < SV; ++e) acc[e] = fmaf(wgt, vr[CL * e], acc[e]);
      }
    }
  }
  // the KL partial rows of a query row (lanes kl * CL + cl), summed over kl
#pragma unroll
  for (int o = CL; o < kShortLanes; o <<= 1) {
#pragma unroll
    for (int e = 0; e < SV; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  }
  if (KS == 1) {
    if (row_ok && kl == 0) {
      float* o = out + row(t) * DV + cl;
#pragma unroll
      for (int e = 0; e < SV; ++e) o[CL * e] = acc[e];
    }
    return;
  }
  if (kl == 0) {
#pragma unroll
    for (int e = 0; e < SV; ++e) s_o[r * DV + cl + CL * e] = acc[e];
  }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();                                   // every rank's partial rows are written
  if (rank == 0) {
    for (int e = tid; e < (n - r0) * DV; e += kThreads) {
      float x = s_o[e];
      for (int src = 1; src < KS; ++src) x += cluster.map_shared_rank(s_o, src)[e];
      out[row(r0 + e / DV) * DV + e % DV] = x;
    }
  }
  cluster.sync();                                   // rank 0 has read them
}

template <typename Tin, int DK>
void launch_short_dk(const Problem& p, const cudaLaunchConfig_t& cfg, int KS) {
  const Tin* q = static_cast<const Tin*>(p.q);
  const Tin* k = static_cast<const Tin*>(p.k);
  const Tin* v = static_cast<const Tin*>(p.v);
  switch (p.dv) {
    case 32: cudaLaunchKernelEx(&cfg, simt_short_fwd<Tin, DK, 32>, q, k, v, p.log_a, p.lam, p.out, p.H, p.T, p.L, KS, p.cu_seqlens, p.status); break;
    case 64: cudaLaunchKernelEx(&cfg, simt_short_fwd<Tin, DK, 64>, q, k, v, p.log_a, p.lam, p.out, p.H, p.T, p.L, KS, p.cu_seqlens, p.status); break;
    default: cudaLaunchKernelEx(&cfg, simt_short_fwd<Tin, DK, 128>, q, k, v, p.log_a, p.lam, p.out, p.H, p.T, p.L, KS, p.cu_seqlens, p.status); break;
  }
}

// Cluster size of the short form: 4 CTAs per row block while the row blocks alone fill at most
// half the SMs, 2 while they fill at most all of them, else 1.
int short_split(long long row_blocks) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  return 2 * row_blocks <= sms ? 4 : row_blocks <= sms ? 2 : 1;
}

template <typename Tin>
void launch_short(const Problem& p, cudaStream_t st) {
  const int nrb = (p.T + kShortRows - 1) / kShortRows;
  const int KS = short_split((long long)nrb * p.H * p.nseq);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nrb * KS, p.H, p.nseq);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = KS > 1 ? 1 : 0;
  switch (p.dk) {
    case 32: launch_short_dk<Tin, 32>(p, cfg, KS); break;
    case 64: launch_short_dk<Tin, 64>(p, cfg, KS); break;
    default: launch_short_dk<Tin, 128>(p, cfg, KS); break;
  }
}

}  // namespace

size_t simt_workspace_bytes(int nseq, int H, int T, int dk, int dv, int C) {
  const size_t Nc = (size_t)((T + C - 1) / C);
  const size_t NB = (size_t)total_blocks((int)Nc);
  const size_t nh = (size_t)nseq * H;
  const size_t dkdv = (size_t)dk * dv;
  return round_up(nh * Nc * dkdv * sizeof(float), 256) + round_up(nh * Nc * sizeof(float), 256) +
         round_up(nh * NB * dkdv * sizeof(float), 256) + round_up(nh * NB * sizeof(float), 256);
}

cudaError_t simt_forward(const Problem& p, int C, void* ws, cudaStream_t st) {
  if (p.in_dtype == LLATTN_BF16) return launch_all<__nv_bfloat16>(p, C, ws, st);
  return launch_all<float>(p, C, ws, st);
}

bool simt_short_supports(int T, int L) { return T <= kShortMaxT && L <= kMaxLevels / 2 + 1; }

cudaError_t simt_short_forward(const Problem& p, cudaStream_t st) {
  if (!simt_short_supports(p.T, p.L)) return cudaErrorNotSupported;
  main_kernel_begin(st);
  if (p.in_dtype == LLATTN_BF16) launch_short<__nv_bfloat16>(p, st);
  else launch_short<float>(p, st);
  main_kernel_end(st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace llattn
