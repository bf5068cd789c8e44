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
// This path is the fp32-input product path (it keeps fp32 accuracy end to end)
// and a cross-check for the tensor-core path on bf16 inputs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "llattn_common.cuh"
#include "llattn_internal.h"
#include "../../include/llattn.h"

namespace llattn {
namespace {

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

}  // namespace llattn
