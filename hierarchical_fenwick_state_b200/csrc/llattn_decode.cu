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

#include <cooperative_groups.h>

#include <atomic>
#include <cstdint>

#include "../../include/llattn.h"
#include "llattn_common.cuh"
#include "llattn_decode.h"
#include "llattn_internal.h"

namespace llattn {
namespace cg = cooperative_groups;
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

// ---- the state after a prompt: level l's bucket of tokens, with its pending gate ----
//
// For a sequence of n tokens, the next token is at position n, and level l >= 1 holds the tokens
// s < n with l(n, s) = l: the bucket [lo, hi) = [P 2^l, P 2^l + 2^(l-1)), P = n >> l, present
// when bit l-1 of n is set ("Partizionamento Gerarchico").  Its state just before n is the sum
// over the bucket of (prod_{r=s+1..n-1} a_r) k_s v_s^T.  The slot stores that sum gated only to
// the bucket's last token hi-1, and the gate row holds the rest, sum_{r=hi..n-1} log a_r: the
// decoding step's lazy gate folds it in at read time, so the stored values stay of the size of
// one token's k v^T instead of underflowing under a long stretch of decay.
//
// Work split.  A cluster of eight CTAs takes one (level, head, sequence); CTA r takes the r-th
// stretch of the bucket counted from its end, walks it from the end in tiles of 32 tokens and
// sums f_s k_s v_s^T into a register tile (each thread a dk/16 x dv/16 block: per token it reads
// dk/16 + dv/16 staged values for dk*dv/256 FMAs).  The factor f_s = exp(D + suffix) <= 1, D the
// log decay from the tile's end to the bucket's end.  The eight partial states then meet in
// distributed shared memory: CTA r adds up its eighth of the elements over the ranks in rank
// order and stores it, so the result does not depend on scheduling.
namespace {

constexpr int kPfTile = 32;
constexpr int kPfCluster = 8;

template <int DK, int DV>
constexpr int prefill_smem_bytes() {
  return (DK * DV + kPfTile * (DK + DV)) * (int)sizeof(float);
}

// Sum over the CTA, returned to every thread (s_red: one float per warp; reusable on return).
__device__ __forceinline__ float block_sum(float x, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = x;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) t += s_red[w];
  __syncthreads();
  return t;
}

// N consecutive floats of shared memory (N in {2, 4, 8}, address aligned to min(N, 4) floats)
// in 64- or 128-bit loads.
template <int N>
__device__ __forceinline__ void ld_smem_vec(float (&x)[N], const float* src) {
  if constexpr (N == 2) {
    const float2 a = *reinterpret_cast<const float2*>(src);
    x[0] = a.x; x[1] = a.y;
  } else {
#pragma unroll
    for (int j = 0; j < N; j += 4) {
      const float4 a = *reinterpret_cast<const float4*>(src + j);
      x[j] = a.x; x[j + 1] = a.y; x[j + 2] = a.z; x[j + 3] = a.w;
    }
  }
}

template <typename Tin, int DK, int DV>
__global__ void __cluster_dims__(kPfCluster, 1, 1) __launch_bounds__(kThreads)
prefill_kernel(PrefillProblem p) {
  constexpr int TK = DK / 16, TV = DV / 16;   // the thread's block of the state
  static_assert(TK * TV * kThreads == DK * DV, "256 threads tile the state");
  extern __shared__ float4 pf_smem[];
  float* s_part = reinterpret_cast<float*>(pf_smem);   // [DK][DV] this CTA's partial state
  float* s_k = s_part + DK * DV;                       // [kPfTile][DK]
  float* s_v = s_k + kPfTile * DK;                     // [kPfTile][DV]
  __shared__ float s_f[kPfTile], s_red[kThreads / 32];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int lvl = blockIdx.x / kPfCluster + 1, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int nslot = p.L - 1;
  const SeqSpan sp = seq_span(b, p.T, p.cu_seqlens, p.status);
  const int n = sp.len;
  // both exits below are uniform over the cluster (they depend on the level, head, sequence)
  if (nslot < 31 && n >= (1 << nslot)) {   // the slots cannot hold position n
    if (lvl == 1 && rank == 0 && h == 0 && tid == 0) atomicOr(p.status, LLATTN_DEV_DECODE_POS);
    return;
  }
  float* g = p.gate + ((size_t)b * p.H + h) * 2 * nslot;
  if (!((n >> (lvl - 1)) & 1)) {           // no bucket at this level: nothing pending either
    if (rank == 0 && tid == 0) g[lvl - 1] = g[nslot + lvl - 1] = 0.f;
    return;
  }
  const int lo = (n >> lvl) << lvl, hi = lo + (1 << (lvl - 1));
  const int span = ((hi - lo + kPfCluster * kPfTile - 1) / (kPfCluster * kPfTile)) * kPfTile;
  const int r_hi = max(lo, hi - rank * span), r_lo = max(lo, hi - (rank + 1) * span);
  const Tin* k = static_cast<const Tin*>(p.k);
  const Tin* v = static_cast<const Tin*>(p.v);
  auto row = [&](int t) { return (size_t)(sp.start + t) * p.H + h; };

  if (rank == 0) {   // the pending gate: log decay of the tokens after the bucket, hi .. n-1
    float part = 0.f;
    for (int t = hi + tid; t < n; t += kThreads) part += __ldg(p.log_a + row(t));
    const float d0 = block_sum(part, s_red);
    if (tid == 0) g[lvl - 1] = g[nslot + lvl - 1] = d0;
  }
  // D: log decay from the end of this CTA's stretch to the bucket's last token
  float D = 0.f;
  {
    float part = 0.f;
    for (int t = r_hi + tid; t < hi; t += kThreads) part += __ldg(p.log_a + row(t));
    D = block_sum(part, s_red);
  }

  const int ty = tid >> 4, tx = tid & 15;
  float acc[TK][TV];
#pragma unroll
  for (int a = 0; a < TK; ++a)
#pragma unroll
    for (int c = 0; c < TV; ++c) acc[a][c] = 0.f;

  // The next tile's rows are loaded into registers while the current one is summed: thread
  // tid holds float4 number tid + j*256 of the tile's k rows (and of its v rows), warp 0 the
  // tile's log a (lane i: token t0 + i).  Rows past the stretch read as zeros.
  constexpr int NK = kPfTile * DK / 4 / kThreads, NV = kPfTile * DV / 4 / kThreads;
  static_assert(NK >= 1 && NV >= 1, "a tile is at least one float4 per thread");
  float4 rk[NK], rv[NV];
  float rla = 0.f;
  auto fetch = [&](int t0, int m) {
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int e = tid + j * kThreads, i = e / (DK / 4), c = 4 * (e % (DK / 4));
      rk[j] = i < m ? ld4_in(k + row(t0 + i) * DK + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e = tid + j * kThreads, i = e / (DV / 4), c = 4 * (e % (DV / 4));
      rv[j] = i < m ? ld4_in(v + row(t0 + i) * DV + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid < 32) rla = tid < m ? __ldg(p.log_a + row(t0 + tid)) : 0.f;
  };
  if (r_hi > r_lo) fetch(max(r_lo, r_hi - kPfTile), r_hi - max(r_lo, r_hi - kPfTile));

  for (int t1 = r_hi; t1 > r_lo; t1 -= kPfTile) {
    const int t0 = max(r_lo, t1 - kPfTile), m = t1 - t0;
    __syncthreads();   // the previous tile is summed: its staging can be overwritten
    if (tid < 32) {
      // factor of token t0 + lane: exp(D + sum of log a over t0+lane+1 .. t1-1), from the
      // suffix sums x = sum over t0+lane .. t1-1; D then moves past this tile (warp 0 keeps it)
      float x = rla;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, x, o);
        if (tid + o < 32) x += y;
      }
      s_f[tid] = __expf(D + (x - rla));
      D += __shfl_sync(0xffffffffu, x, 0);
    }
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int e = tid + j * kThreads;
      *reinterpret_cast<float4*>(s_k + (e / (DK / 4)) * DK + 4 * (e % (DK / 4))) = rk[j];
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e = tid + j * kThreads;
      *reinterpret_cast<float4*>(s_v + (e / (DV / 4)) * DV + 4 * (e % (DV / 4))) = rv[j];
    }
    __syncthreads();
    if (t0 > r_lo) fetch(max(r_lo, t0 - kPfTile), t0 - max(r_lo, t0 - kPfTile));
    for (int i = 0; i < m; ++i) {
      float kk[TK], vv[TV];
      ld_smem_vec<TK>(kk, s_k + i * DK + ty * TK);
      ld_smem_vec<TV>(vv, s_v + i * DV + tx * TV);
      const float f = s_f[i];
#pragma unroll
      for (int a = 0; a < TK; ++a) kk[a] *= f;
#pragma unroll
      for (int a = 0; a < TK; ++a)
#pragma unroll
        for (int c = 0; c < TV; ++c) acc[a][c] = fmaf(kk[a], vv[c], acc[a][c]);
    }
  }

  // partial state to shared memory, then each rank reduces its eighth over the cluster
#pragma unroll
  for (int a = 0; a < TK; ++a)
#pragma unroll
    for (int c = 0; c < TV; ++c) s_part[(ty * TK + a) * DV + tx * TV + c] = acc[a][c];
  cluster.sync();
  constexpr int kShare = DK * DV / 4 / kPfCluster;   // float4s each rank reduces
  float4* dst = reinterpret_cast<float4*>(p.levels + (((size_t)b * p.H + h) * nslot + (lvl - 1)) *
                                                         (size_t)DK * DV);
  for (int e = tid; e < kShare; e += kThreads) {
    const int idx = rank * kShare + e;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kPfCluster; ++q) {
      const float4 x = cluster.map_shared_rank(reinterpret_cast<float4*>(s_part), q)[idx];
      sum.x += x.x; sum.y += x.y; sum.z += x.z; sum.w += x.w;
    }
    dst[idx] = sum;
  }
  cluster.sync();   // no CTA leaves while another reads its partial
}

template <typename Tin, int DK, int DV>
cudaError_t launch_prefill_one(const PrefillProblem& p, cudaStream_t st) {
  // the dynamic shared-memory opt-in is a per-device attribute of each kernel
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load()) {
    if ((e = cudaFuncSetAttribute(prefill_kernel<Tin, DK, DV>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  prefill_smem_bytes<DK, DV>())) != cudaSuccess)
      return e;
    attr_set[dev].store(true);
  }
  const dim3 grid(kPfCluster * (p.L - 1), p.H, p.B);
  prefill_kernel<Tin, DK, DV><<<grid, kThreads, prefill_smem_bytes<DK, DV>(), st>>>(p);
  return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t launch_prefill_dk(const PrefillProblem& p, cudaStream_t st) {
  switch (p.dv) {
    case 32: return launch_prefill_one<Tin, DK, 32>(p, st);
    case 64: return launch_prefill_one<Tin, DK, 64>(p, st);
    default: return launch_prefill_one<Tin, DK, 128>(p, st);
  }
}

template <typename Tin>
cudaError_t launch_prefill(const PrefillProblem& p, cudaStream_t st) {
  switch (p.dk) {
    case 32: return launch_prefill_dk<Tin, 32>(p, st);
    case 64: return launch_prefill_dk<Tin, 64>(p, st);
    default: return launch_prefill_dk<Tin, 128>(p, st);
  }
}

}  // namespace

cudaError_t prefill_state(const PrefillProblem& p, cudaStream_t st) {
  if (p.L < 2) return cudaSuccess;   // no level slots
  count_launch(1);
  return p.in_dtype == LLATTN_BF16 ? launch_prefill<__nv_bfloat16>(p, st) : launch_prefill<float>(p, st);
}

cudaError_t decode_step(const DecodeProblem& p, cudaStream_t st) {
  count_launch(1);
  main_kernel_begin(st);
  const cudaError_t e = p.in_dtype == LLATTN_BF16 ? launch<__nv_bfloat16>(p, st)
                                                  : launch<float>(p, st);
  main_kernel_end(st);
  return e;
}

}  // namespace llattn
