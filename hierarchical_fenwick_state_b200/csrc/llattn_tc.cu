// Tensor-core forward of log-linear attention (Mamba-2 form) for sm_100a.
//
// One CTA owns one (sequence, head) and walks its chunks of 128 tokens in order,
// keeping the chunk-level Fenwick states on chip.  This is the chunkwise-parallel
// algorithm of "Log-Linear Attention" (gist.science, Italian "Sommario tecnico"
// section 2, "Forma Ricorrente e Parallelizzata", Training bullet; Spanish
// "Resumen tecnico" section 2, "Algoritmo de Entrenamiento (Chunk-scan)"): dense
// work inside a chunk, and between chunks the low-rank hierarchical structure of
// the mask M_H ("Matrici Gerarchiche"), whose level for keys in an earlier aligned
// chunk c' depends only on the chunk indices, l = 1 + log2(C) + msb(c XOR c').
// Query chunk c therefore reads one block state per set bit b of c: the 2^b
// chunks just before the aligned 2^(b+1)-chunk group of c.  Those block states
// form a binary counter over chunks (the recurrent form's "merge on promotion",
// "Forma Ricorrente"), kept here in shared memory as bf16 hi/lo pairs.
//
// Per chunk (all five steps fused in this one kernel; the weighted readout over
// levels is fused into the epilogue, as in "kernel ... que fusionan operaciones a
// traves de niveles jerarquicos", Spanish section 3, item 3):
//   a1 decay scan     g = inclusive cumsum of log a over the chunk (warp shuffles)
//   a4 intra-chunk    S = Q K^T (tcgen05, TMEM); P = S .* W, W[i,j] = lam[i,l(i,j)]
//                     exp(g_i - g_j) for j <= i; O = P V (P as bf16 hi+lo in TMEM)
//   a5 readout        R_b = Q S_b (tcgen05, S_b hi+lo from smem) for each set bit b;
//                     o_i = O_i + sum_b lam[i, 1+log2 C+b] exp(g_i + gap_b) R_b,i
//   a2 chunk state    H = (diag(exp(G - g)) K)^T V  (K scaled, split hi+lo)
//   a3 tree merge     new level m (trailing ones of c) = H + sum_{b<m} exp(.) S_b
// Every rounded bf16 operand is split into hi + lo parts (two MMAs), which keeps
// the result within fp32-accumulation error of the exact sum; out is fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/llattn.h"
#include "llattn_common.cuh"
#include "llattn_internal.h"
#include "llattn_tc_ptx.cuh"

namespace llattn {
namespace {

using namespace ptx;

constexpr int kC = 128;            // chunk length (rows of every MMA, M = 128)
constexpr int kLogC = 7;
constexpr int kD = 64;             // d_k = d_v
constexpr int kThreads = 256;      // 8 warps: warp w owns TMEM lanes 32*(w%4).., column half w/4
constexpr int kMaxChunks = 64;     // chunks one CTA walks (T <= 8192)
constexpr int kLevels = 6;         // chunk-level Fenwick levels kept on chip: log2(kMaxChunks)
constexpr int kMaxL = 25;          // lam levels supported (1 + ceil(log2 T), T <= 2^24)
constexpr int kRing = 4;           // TMEM accumulators for level readouts per batch

// ---- shared memory map (bytes from a 1024-byte aligned base) ----
constexpr uint32_t kTile = kC * 128;                // 128 rows x 128 B (64 bf16), swizzled
constexpr uint32_t kStage = 3 * kTile;              // Q, K, V of one chunk
constexpr uint32_t kOffKlo = 2 * kStage;            // low part of the decay-scaled K
constexpr uint32_t kOffSlots = kOffKlo + kTile;     // level states: hi (8 KB) + lo (8 KB)
constexpr uint32_t kSlot = 2 * 8192;
constexpr uint32_t kOffLam = kOffSlots + kLevels * kSlot;
constexpr uint32_t kOffG = kOffLam + kC * kMaxL * 4;
constexpr uint32_t kOffCj = kOffG + kC * 4;
constexpr uint32_t kOffScan = kOffCj + kC * 4;
constexpr uint32_t kOffBar = kOffScan + 64;
constexpr uint32_t kOffMisc = kOffBar + 64;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;  // + slack to align the base

// ---- TMEM columns ----
constexpr uint32_t kColS = 0;      // S = Q K^T (fp32, 128 cols), then P hi [0,64) / lo [64,128)
constexpr uint32_t kColO = 128;    // intra-chunk output P V (64 cols)
constexpr uint32_t kColH = 192;    // chunk state H (M = 64 layout, 64 cols)
constexpr uint32_t kColR = 256;    // kRing readout accumulators of 64 cols

constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
constexpr uint32_t kIdescR = idesc_bf16(128, 64, 0, 0);    // Q x S_b^T rows (K-major)
constexpr uint32_t kIdescPV = idesc_bf16(128, 64, 0, 1);   // P (TMEM) x V (N contiguous)
constexpr uint32_t kIdescH = idesc_bf16(64, 64, 1, 1);     // K^T (M contiguous) x V

__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t saddr) { return sdesc_sw128(saddr, 8192, 1024); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);  // a -> low 16 bits
  return *reinterpret_cast<uint32_t*>(&v);
}

// x ~= hi + lo with hi = bf16(x), lo = bf16(x - hi): packs (a, b) pairs of both parts.
__device__ __forceinline__ void split_pack(float a, float b, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float ah = __low2float(h), bh = __high2float(h);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = pack_bf16(a - ah, b - bh);
}

__device__ __forceinline__ float bf16_at(const uint8_t* p) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

__global__ void __launch_bounds__(kThreads, 1)
tc_fwd_d64(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
           const __grid_constant__ CUtensorMap tmv, const __nv_bfloat16* __restrict__ q,
           const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
           const float* __restrict__ log_a, const float* __restrict__ lam,
           float* __restrict__ out, int H, int T, int L, const int* __restrict__ cu,
           unsigned int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = warp & 3;          // TMEM sub-partition: lanes 32*sub .. 32*sub+31
  const int hf = warp >> 2;          // which 32/64-column half of a row this thread handles
  const int row = sub * 32 + lane;   // chunk row (TMEM lane) of this thread
  const uint32_t lane_off = uint32_t(sub * 32) << 16;
  const int h = blockIdx.x, sq = blockIdx.y;

  const SeqSpan sp = seq_span(sq, T, cu, status);
  if (sp.len <= 0) return;
  const int nch = (sp.len + kC - 1) / kC;
  const int LS = L | 1;              // odd row stride of the lam table: conflict-free

  uint8_t* stage[2] = {sm, sm + kStage};
  uint8_t* klo = sm + kOffKlo;
  uint8_t* slots = sm + kOffSlots;
  float* lamrow = reinterpret_cast<float*>(sm + kOffLam);
  float* gs = reinterpret_cast<float*>(sm + kOffG);
  float* cj = reinterpret_cast<float*>(sm + kOffCj);
  float* scan = reinterpret_cast<float*>(sm + kOffScan);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);  // 0,1 loads; 2 S; 3 R; 4 PV+H
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + kOffMisc);  // [0] TMEM base, [1] abort

  if (warp == 0) {
    tmem_alloc(&misc[0], 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    misc[1] = 0;
    prefetch_tensormap(&tmq);
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  auto is_full = [&](int c) { return (c + 1) * kC <= sp.len; };
  auto issue_load = [&](int c, int s) {
    const int tok0 = static_cast<int>(sp.start + (long long)c * kC);
    mbar_arrive_expect_tx(&bars[s], 3 * kTile);
    tma_load_3d(stage[s], &tmq, &bars[s], 0, h, tok0);
    tma_load_3d(stage[s] + kTile, &tmk, &bars[s], 0, h, tok0);
    tma_load_3d(stage[s] + 2 * kTile, &tmv, &bars[s], 0, h, tok0);
  };
  auto fail = [&]() {
    atomicOr(status, LLATTN_DEV_WAIT_TIMEOUT);
    misc[1] = 1;
  };

  // lam / log_a of the next chunk travel in registers while the current one computes.
  float pf_lam[(kMaxL + 1) / 2];
  float pf_la = 0.f;
  auto prefetch_scalars = [&](int c) {
    const int t = c * kC + row;
    const bool ok = t < sp.len;
    const long long tok = sp.start + t;
    const float* lr = lam + (tok * H + h) * L;
#pragma unroll
    for (int i = 0; i < (kMaxL + 1) / 2; ++i) {
      const int l = hf + 2 * i;
      pf_lam[i] = (ok && l < L) ? __ldg(lr + l) : 0.f;
    }
    if (hf == 0) pf_la = ok ? __ldg(log_a + tok * H + h) : 0.f;
  };

  float gtot[kLevels];  // total log-decay of each live level's block (uniform)
#pragma unroll
  for (int b = 0; b < kLevels; ++b) gtot[b] = 0.f;
  uint32_t ph_load[2] = {0u, 0u}, ph_S = 0u, ph_R = 0u, ph_PH = 0u;
  int pending = -1;  // stage with a TMA in flight that nobody has waited for

  prefetch_scalars(0);
  if (tid == 0 && is_full(0)) issue_load(0, 0);
  if (is_full(0)) pending = 0;

  for (int c = 0; c < nch; ++c) {
    const int s = c & 1;
    const int n = min(kC, sp.len - c * kC);
    const bool full = n == kC;
    const bool aborted = misc[1] != 0;

    // ---- per-chunk scalars: lam rows to smem, log_a cumsum (a1) ----
#pragma unroll
    for (int i = 0; i < (kMaxL + 1) / 2; ++i) {
      const int l = hf + 2 * i;
      if (l < L) lamrow[row * LS + l] = pf_lam[i];
    }
    const float la = pf_la;
    if (c + 1 < nch) prefetch_scalars(c + 1);
    if (tid == 0 && c + 1 < nch && is_full(c + 1) && !aborted) issue_load(c + 1, s ^ 1);
    if (!full) {
      // ragged last chunk: plain loads, rows past the sequence end zero-filled
      const long long tok0 = sp.start + (long long)c * kC;
#pragma unroll
      for (int tsr = 0; tsr < 3; ++tsr) {
        const __nv_bfloat16* src = tsr == 0 ? q : (tsr == 1 ? k : v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = hf * 32 + j * 8;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (row < n) val = *reinterpret_cast<const uint4*>(src + ((tok0 + row) * H + h) * kD + col);
          *reinterpret_cast<uint4*>(stage[s] + tsr * kTile + sw128_off(row, col)) = val;
        }
      }
      fence_proxy_async_smem();
    }
    if (hf == 0) {
      float x = la;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) scan[sub] = x;
      gs[row] = x;
    }
    __syncthreads();
    if (hf == 0) {
      float off = 0.f;
      for (int w = 0; w < sub; ++w) off += scan[w];
      gs[row] += off;
    }
    __syncthreads();
    const float g_row = gs[row];
    const float g0 = gs[0];
    const float gend = gs[n - 1];  // chunk total log-decay
    // exp(g_i - g_j) = exp(g_i - g_0) * exp(g_0 - g_j) while exp(g_0 - g_end) stays finite
    const bool factored = (g0 - gend) <= 80.f;
    if (hf == 0) cj[row] = factored ? __expf(g0 - g_row) : 0.f;
    __syncthreads();

    // ---- MMA issue: S = Q K^T, level readouts R_b = Q (S_b hi + S_b lo) ----
    const uint32_t qa = smem_u32(stage[s]);
    const uint32_t ka = qa + kTile;
    const uint32_t va = qa + 2 * kTile;
    int nlive = 0;
#pragma unroll
    for (int b = 0; b < kLevels; ++b) nlive += (c >> b) & 1;
    if (tid == 0) {
      if (full && !mbar_wait(&bars[s], ph_load[s])) fail();
      tc_fence_after();
      if (misc[1] == 0) {
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_ss(tmem + kColS, kdesc(qa + kk * 32), kdesc(ka + kk * 32), kIdescS, kk > 0);
      }
      mma_commit(&bars[2]);
      int slot_i = 0;
      for (int b = 0; b < kLevels && slot_i < kRing; ++b) {
        if (!((c >> b) & 1)) continue;
        const uint32_t d = tmem + kColR + 64 * slot_i;
        const uint32_t sb = smem_u32(slots + b * kSlot);
        if (misc[1] == 0) {
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(d, kdesc(qa + kk * 32), kdesc(sb + kk * 32), kIdescR, kk > 0);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(d, kdesc(qa + kk * 32), kdesc(sb + 8192 + kk * 32), kIdescR, 1);
        }
        ++slot_i;
      }
      mma_commit(&bars[3]);
    }
    if (full) {
      // every thread acquires the TMA'd tiles (the K scaling below reads them)
      if (tid != 0 && !mbar_wait(&bars[s], ph_load[s])) fail();
      ph_load[s] ^= 1u;
      if (pending == s) pending = -1;
    }
    if (c + 1 < nch && is_full(c + 1) && !aborted) pending = s ^ 1;

    // ---- intra-chunk mask (a4): P = S .* W, split into bf16 hi/lo, back into TMEM ----
    if (!mbar_wait(&bars[2], ph_S)) fail();
    ph_S ^= 1u;
    tc_fence_after();
    float sv[64];
    {
      float t0v[32], t1v[32];
      tmem_ld32(tmem + lane_off + kColS + 64 * hf, t0v);
      tmem_ld32(tmem + lane_off + kColS + 64 * hf + 32, t1v);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        sv[e] = t0v[e];
        sv[32 + e] = t1v[e];
      }
    }
    {
      const int i = row;
      const float ri = factored ? __expf(g_row - g0) : 0.f;
      const float* lr = lamrow + i * LS;
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const int j = 64 * hf + e;
        float p = 0.f;
        if (j <= i) {
          const int lev = (i == j) ? 0 : (32 - __clz(i ^ j));
          const float wl = lr[lev];
          const float w = factored ? wl * ri * cj[j] : wl * __expf(g_row - gs[j]);
          p = sv[e] * w;
        }
        sv[e] = p;
      }
    }
    __syncthreads();  // every S read of this row is done before P overwrites its columns
    {
      uint32_t phi[32], plo[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) split_pack(sv[2 * e], sv[2 * e + 1], phi[e], plo[e]);
      uint32_t a[16], b[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) { a[e] = phi[e]; b[e] = phi[16 + e]; }
      tmem_st16(tmem + lane_off + kColS + 32 * hf, a);
      tmem_st16(tmem + lane_off + kColS + 32 * hf + 16, b);
#pragma unroll
      for (int e = 0; e < 16; ++e) { a[e] = plo[e]; b[e] = plo[16 + e]; }
      tmem_st16(tmem + lane_off + kColS + 64 + 32 * hf, a);
      tmem_st16(tmem + lane_off + kColS + 64 + 32 * hf + 16, b);
      tmem_wait_st();
    }
    // ---- chunk state operand (a2): K rows scaled by exp(G - g_s), split hi (in place) / lo ----
    {
      const float ks = row < n ? __expf(gend - g_row) : 0.f;
      uint8_t* kt = stage[s] + kTile;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t off = sw128_off(row, hf * 32 + j * 8);
        uint4 raw = *reinterpret_cast<const uint4*>(kt + off);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
          split_pack(__low2float(pr) * ks, __high2float(pr) * ks, hi[e], lo[e]);
        }
        *reinterpret_cast<uint4*>(kt + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(klo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- MMA issue: O = P V (P from TMEM), H = K_s^T V ----
    if (tid == 0) {
      tc_fence_after();
      if (misc[1] == 0) {
        const uint32_t kl = smem_u32(klo);
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          mma_ts(tmem + kColO, tmem + kColS + 8 * kk, mndesc(va + kk * 2048), kIdescPV, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          mma_ts(tmem + kColO, tmem + kColS + 64 + 8 * kk, mndesc(va + kk * 2048), kIdescPV, 1);
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          mma_ss(tmem + kColH, mndesc(ka + kk * 2048), mndesc(va + kk * 2048), kIdescH, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          mma_ss(tmem + kColH, mndesc(kl + kk * 2048), mndesc(va + kk * 2048), kIdescH, 1);
      }
      mma_commit(&bars[4]);
    }

    // ---- epilogue (a5): o = O + sum_b w_b R_b, written as fp32 ----
    if (!mbar_wait(&bars[3], ph_R)) fail();
    ph_R ^= 1u;
    if (!mbar_wait(&bars[4], ph_PH)) fail();
    ph_PH ^= 1u;
    tc_fence_after();
    float o[32];
    tmem_ld32(tmem + lane_off + kColO + 32 * hf, o);
    tmem_wait_ld();
    {
      float gap = 0.f;   // log-decay between level b's block and this chunk
      int slot_i = 0;
      int done = 0;
      const float* lr = lamrow + row * LS;
#pragma unroll
      for (int b = 0; b < kLevels; ++b) {
        if (!((c >> b) & 1)) continue;
        if (slot_i == kRing) {
          // more live levels than accumulators: issue the next batch once these are read
          tc_fence_before();
          __syncthreads();
          if (tid == 0) {
            tc_fence_after();
            int si = 0;
            for (int bb = b; bb < kLevels && si < kRing; ++bb) {
              if (!((c >> bb) & 1)) continue;
              const uint32_t d = tmem + kColR + 64 * si;
              const uint32_t sb = smem_u32(slots + bb * kSlot);
              if (misc[1] == 0) {
                for (int kk = 0; kk < kD / 16; ++kk)
                  mma_ss(d, kdesc(qa + kk * 32), kdesc(sb + kk * 32), kIdescR, kk > 0);
                for (int kk = 0; kk < kD / 16; ++kk)
                  mma_ss(d, kdesc(qa + kk * 32), kdesc(sb + 8192 + kk * 32), kIdescR, 1);
              }
              ++si;
            }
            mma_commit(&bars[3]);
          }
          if (!mbar_wait(&bars[3], ph_R)) fail();
          ph_R ^= 1u;
          tc_fence_after();
          slot_i = 0;
        }
        float r[32];
        tmem_ld32(tmem + lane_off + kColR + 64 * slot_i + 32 * hf, r);
        tmem_wait_ld();
        const float w = lr[1 + kLogC + b] * __expf(g_row + gap);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = fmaf(w, r[e], o[e]);
        gap += gtot[b];
        ++slot_i;
        ++done;
      }
      (void)done;
    }
    if (row < n) {
      float* dst = out + ((sp.start + (long long)c * kC + row) * H + h) * kD + 32 * hf;
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
    }

    // ---- Fenwick merge (a3): level m = H + sum_{b<m} exp(decay after b) S_b ----
    if (c + 1 < nch) {
      const int m = __ffs(~c) - 1;
      float hv[32];
      tmem_ld32(tmem + lane_off + kColH + 32 * hf, hv);
      tmem_wait_ld();
      float acc = gend;
      if (lane < 16) {
        const int i = 16 * sub + lane;  // d_k row of H (M = 64 TMEM layout)
#pragma unroll
        for (int b = 0; b < kLevels; ++b) {
          if (b >= m) break;
          const float f = __expf(acc);
          const uint8_t* sl = slots + b * kSlot;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const uint32_t off = sw128_off(32 * hf + e, i);
            hv[e] = fmaf(f, bf16_at(sl + off) + bf16_at(sl + 8192 + off), hv[e]);
          }
          acc += gtot[b];
        }
        uint8_t* dsl = slots + m * kSlot;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const uint32_t off = sw128_off(32 * hf + e, i);
          const __nv_bfloat16 hb = __float2bfloat16_rn(hv[e]);
          const __nv_bfloat16 lb = __float2bfloat16_rn(hv[e] - __bfloat162float(hb));
          *reinterpret_cast<__nv_bfloat16*>(dsl + off) = hb;
          *reinterpret_cast<__nv_bfloat16*>(dsl + 8192 + off) = lb;
        }
      }
      // bookkeeping (uniform over the CTA): total log-decay of the new level-m block
      float tot = gend;
#pragma unroll
      for (int b = 0; b < kLevels; ++b)
        if (b < m) tot += gtot[b];
#pragma unroll
      for (int b = 0; b < kLevels; ++b)
        if (b == m) gtot[b] = tot;
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (misc[1] != 0) break;
  }

  // a TMA still in flight (only after an abort) must land before the CTA exits
  if (tid == 0 && pending >= 0) mbar_wait(&bars[pending], ph_load[pending], 100000000ull);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [tokens, H, 64] bf16 viewed as a 3-D tensor {64, H, tokens}; box {64, 1, 128}, 128 B swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, int H, long long tokens) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {kD, (cuuint64_t)H, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {kD * 2, (cuuint64_t)H * kD * 2};
  const cuuint32_t box[3] = {kD, 1, kC};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool tc_supports(int in_dtype, int dk, int dv, int chunk, int T) {
  return in_dtype == LLATTN_BF16 && dk == kD && dv == kD && chunk == kC && T <= kC * kMaxChunks;
}

size_t tc_workspace_bytes(int, int, int, int, int, int) { return 0; }

cudaError_t tc_forward(const Problem& p, int chunk, void*, cudaStream_t st) {
  if (!tc_supports(p.in_dtype, p.dk, p.dv, chunk, p.T)) return cudaErrorNotSupported;
  // TMA only ever fetches whole chunks inside a sequence, so the token extent can be
  // the dense size, or for packed batches any bound >= the real total (nseq * T).
  const long long tokens = (long long)p.nseq * p.T;
  if (tokens >= (1ll << 31)) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv;
  cudaError_t e;
  if ((e = make_map(&mq, p.q, p.H, tokens)) != cudaSuccess) return e;
  if ((e = make_map(&mk, p.k, p.H, tokens)) != cudaSuccess) return e;
  if ((e = make_map(&mv, p.v, p.H, tokens)) != cudaSuccess) return e;
  static bool attr_set = false;
  if (!attr_set) {
    if ((e = cudaFuncSetAttribute(tc_fwd_d64, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kSmemBytes)) != cudaSuccess)
      return e;
    attr_set = true;
  }
  const dim3 grid(p.H, p.nseq);
  main_kernel_begin(st);
  tc_fwd_d64<<<grid, kThreads, kSmemBytes, st>>>(
      mq, mk, mv, static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
      static_cast<const __nv_bfloat16*>(p.v), p.log_a, p.lam, p.out, p.H, p.T, p.L, p.cu_seqlens,
      p.status);
  main_kernel_end(st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace llattn
