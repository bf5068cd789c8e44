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
// "Forma Ricorrente"), kept here in shared memory (bf16 hi/lo pairs in the serial
// cross-check, fp16 in the pipelined kernel).
//
// Per chunk (all five steps fused in this one kernel; the weighted readout over
// levels is fused into the epilogue, as in "kernel ... que fusionan operaciones a
// traves de niveles jerarquicos", Spanish section 3, item 3):
//   a1 decay scan     g = inclusive cumsum of log a over the chunk (warp shuffles)
//   a4 intra-chunk    S = Q K^T (tcgen05, TMEM); P = S .* W, W[i,j] = lam[i,l(i,j)]
//                     exp(g_i - g_j) for j <= i; O = P V (P in TMEM)
//   a5 readout        R_b = Q S_b (tcgen05, S_b from smem) for each set bit b;
//                     o_i = O_i + sum_b lam[i, 1+log2 C+b] exp(g_i + gap_b) R_b,i
//   a2 chunk state    H = (diag(exp(G - g)) K)^T V  (K scaled)
//   a3 tree merge     new level m (trailing ones of c) = H + sum_{b<m} exp(.) S_b
// Operand precision.  S = Q K^T takes the bf16 inputs as they are.  The serial kernel
// splits every rounded operand (P, the scaled K, the level states) into bf16 hi + lo
// parts (two MMAs), which keeps it within fp32-accumulation error of the exact sum.
// The pipelined kernel rounds them once to fp16 instead (10-bit mantissa, V and a copy
// of Q converted exactly), which keeps the output within about 4e-3 of its RMS on the
// stress inputs (no decay, one level at a time) and needs intermediates below the fp16
// range (|P|, |V|, the scaled K and the level-state entries under 6.5e4).  out is fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
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

// x ~= hi + lo: hi = x with its low 16 bits cleared (a bf16 value, exact), lo = bf16(x - hi)
// (x - hi is exact in fp32 and below 2^-7 |x|, so hi + lo carries ~16 significant bits).
// Packs the (a, b) pairs of both parts; a goes to the low 16 bits.
__device__ __forceinline__ void split_pack(float a, float b, uint32_t& hi, uint32_t& lo) {
  const uint32_t ua = __float_as_uint(a) & 0xFFFF0000u, ub = __float_as_uint(b) & 0xFFFF0000u;
  hi = __byte_perm(ua, ub, 0x7632);  // high halves of a (low) and b (high)
  lo = pack_bf16(a - __uint_as_float(ua), b - __uint_as_float(ub));
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);  // a -> low 16 bits
  return *reinterpret_cast<uint32_t*>(&v);
}

// 8 bf16 values (a uint4) -> 8 fp16 values
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 x) {
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
    w[e] = pack_f16(f.x, f.y);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ float bf16_at(const uint8_t* p) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

__global__ void __launch_bounds__(kThreads, 1)
tc_fwd_serial(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
           const __grid_constant__ CUtensorMap tmv, const __nv_bfloat16* __restrict__ q,
           const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
           const float* __restrict__ log_a, const float* __restrict__ lam,
           float* __restrict__ out, int H, int T, int L, const int* __restrict__ cu,
           unsigned int* status) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, by pointer arithmetic on the shared array so that the compiler
  // keeps shared-memory (not generic) loads and stores for everything derived from it
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
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

  auto stage = [sm](int i) { return sm + i * kStage; };
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
    tma_load_3d(stage(s), &tmq, &bars[s], 0, h, tok0);
    tma_load_3d(stage(s) + kTile, &tmk, &bars[s], 0, h, tok0);
    tma_load_3d(stage(s) + 2 * kTile, &tmv, &bars[s], 0, h, tok0);
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
          *reinterpret_cast<uint4*>(stage(s) + tsr * kTile + sw128_off(row, col)) = val;
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
    const uint32_t qa = smem_u32(stage(s));
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
      uint8_t* kt = stage(s) + kTile;
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

// ==========================================================================================
// Pipelined variant: warp-specialised roles linked by mbarriers.
//   warp 0        TMA producer (Q, K, V tiles of chunk c into stage c % 3; output tiles out;
//                 L2 prefetch of lam / log a)
//   warp 1        MMA issuer for the intra-chunk part (S, P V)
//   warp 18       MMA issuer for the inter-chunk part (H^T, level readouts)
//   warps 2..9    group A      (decay scan, V to fp16, causal mask -> P, K scaling)
//   warps 10..17  group B      (P V + level readouts -> output tile, Fenwick merge of the
//                               chunk state, fp16 copy of the next Q)
// TMEM holds S/P (128 columns), the P V accumulator (64), H^T (64) and one readout
// accumulator spanning up to four adjacent levels (256), so one MMA chain reads them.
// P overwrites S in place, 16 keys at a time: the 16 fp32 columns of keys 16g..16g+15
// become 8 columns of fp16 pairs, so no thread ever writes columns that it or another
// thread has still to read.
// Every mbarrier that is waited on by phase parity is checked against overrun: a waiter
// that falls two phases behind would wait for the wrong phase, so each producer of a
// phase is held (by its own inputs) until the consumers of the previous phase are past it.
// ==========================================================================================
constexpr int kPW = 19;                       // warps
constexpr int kPThreads = kPW * 32;
constexpr int kPA0 = 2;                       // first warp of group A
constexpr int kPNA = 8 * 32;                  // group A threads
constexpr int kPB0 = 10;                      // first warp of group B
constexpr int kPNB = 8 * 32;                  // group B threads
constexpr int kPI2 = 18;                      // warp of the inter-chunk MMA issuer

constexpr int kPG = 3;                        // g buffers
constexpr uint32_t kPLamStride = 9;           // group A lam table: levels 0..7, odd stride
constexpr int kPNumBars = 31;

// Shared-memory map of the pipelined kernel for NLEV chunk-level Fenwick states kept on chip
// (T <= 128 * 2^NLEV) and an NST-stage Q/K/V ring (chunk c in stage c % NST).
template <int NLEV, int NST>
struct PipeLayout {
  static constexpr int kLev = NLEV, kSt = NST;
  static constexpr uint32_t kOffSlots = NST * kStage;         // level states, fp16 [d_v][d_k], 8 KB
  static constexpr uint32_t kOffQh = kOffSlots + NLEV * 8192;  // fp16 copy of Q for the readouts
  static constexpr uint32_t kOffLam = kOffQh + kTile;
  static constexpr uint32_t kOffG = kOffLam + kC * kPLamStride * 4;   // g[3][128]
  static constexpr uint32_t kOffCj = kOffG + kPG * kC * 4;
  // lam of the inter-chunk levels 1+log2 C+b (b < NLEV) times exp(g_i), per row: group A
  // writes it with the decay scan, group B reads it for the readout weights (g buffers' ring)
  static constexpr uint32_t kOffLamB = kOffCj + kC * 4;
  static constexpr uint32_t kOffScan = kOffLamB + kPG * kC * NLEV * 4;
  static constexpr uint32_t kOffBar = kOffScan + 64;
  static constexpr uint32_t kOffMisc = kOffBar + kPNumBars * 8;
  static constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory of the pipelined kernel exceeds 227 KB");
};
using PipeShort = PipeLayout<6, 3>;   // T <= 8192
using PipeLong = PipeLayout<7, 2>;    // T <= 16384
using PipeXL = PipeLayout<10, 2>;     // T <= 131072 (long sequences, walked in segments)

constexpr uint32_t kPColSP = 0;    // S = Q K^T, overwritten in place by P (fp16)
constexpr uint32_t kPColO = 128;   // P V accumulator
constexpr uint32_t kPColH = 192;   // V^T K~, rows duplicated in lanes 64..127
constexpr uint32_t kPColR = 256;   // readout accumulator: up to four adjacent levels
constexpr int kPSpan = 4;          // levels one readout chain covers (N = 64 per level)

// P V and the chunk state run in fp16: V is converted in place when its tile lands, P and
// the decay-scaled K are rounded once to fp16 (10-bit mantissa; no hi/lo split needed)
constexpr uint32_t kIdescHT = idesc_f16(128, 64, 1, 1);   // V^T (M contiguous) x K~ (N contiguous)
constexpr uint32_t kIdescPVh = idesc_f16(128, 64, 0, 1);  // P (TMEM) x V (N contiguous)

enum : int {
  B_FULL = 0, B_EMPTY = 3, B_SFULL = 6, B_PFULL = 7, B_SPEMPTY = 8, B_KS = 9, B_HFULL = 10,
  B_HEMPTY = 11, B_LV = 12, B_LV1 = 13, B_OFULL = 14, B_OEMPTY = 15, B_RFULL = 16,
  B_REMPTY = 17, B_GREADY = 18, B_GEMPTY = 21, B_DRAIN = 24, B_DRAIN2 = 25, B_OSTAGED = 26,
  B_FREE = 29, B_PREFILL = 30
};

// Wait on an mbarrier phase; returns false at once if the CTA has aborted, and aborts
// the CTA (flag + device status bit) if the wait exceeds its time limit.
__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity, uint32_t* abort_flag,
                                      unsigned int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  volatile uint32_t* ab = abort_flag;
  if (*ab) return false;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (*ab) return false;
    if (globaltimer_ns() - t0 > 2000000000ull) {
      atomicOr(status, LLATTN_DEV_WAIT_TIMEOUT);
      *ab = 1u;
      return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// The readouts of one chunk go out in chains: a chain starts at the lowest remaining set
// bit b0 of c and covers the set bits below b0 + kPSpan; its N = 64 * (b1 - b0 + 1)
// columns read the consecutive hi (then lo) level arrays in one MMA per K step.  A level
// inside the range whose bit is clear is computed and ignored.
template <int NLEV>
__device__ __forceinline__ bool next_chain(int c, int from, int& b0, int& b1) {
  int b = from;
  while (b < NLEV && !((c >> b) & 1)) ++b;
  if (b >= NLEV) return false;
  b0 = b;
  b1 = b;
  for (int x = b + 1; x < NLEV && x < b + kPSpan; ++x)
    if ((c >> x) & 1) b1 = x;
  return true;
}

// Launch arguments of the pipelined kernel beyond the tensors.
//   g          a CTA walks one segment of 2^g chunks (blockIdx.z); g >= 30: the whole sequence
//   ndv        64-column tiles of v and out per head (blockIdx.x = head * ndv + tile)
//   qcol       first q / k column this launch reads (d_k is taken 64 columns per launch)
//   dk_tot, dv_tot   row lengths of q / k and of v / out
//   accumulate add this launch's share into out (a later d_k slice) instead of storing it
//   blocks, block_decay, nblk, nseg   the pre-filled levels: per (sequence, head tile),
//              nblk dyadic block states over segments (fp16 slot images of 8 KB) and their
//              total log decays; nseg = segments per sequence (the grid's z extent)
struct SegArgs {
  int g, ndv, qcol, dk_tot, dv_tot, accumulate;
  const uint8_t* blocks;
  const float* block_decay;
  int nblk, nseg;
};

// Index of dyadic block (b, j) over segments (level b, even j: segments j*2^b .. (j+2)*2^b - 1
// minus the upper half, i.e. the 2^b segments just before an odd multiple of 2^b) among the
// blocks kept per (sequence, head tile): level b holds blocks_at_level(nseg, b) of them.
__host__ __device__ inline int seg_block_index(int nseg, int b, int j) {
  return level_offset(nseg, b) + (j >> 1);
}

// MN-major descriptor whose second 64-row group along M repeats the first (LBO = 0):
// an M = 128 MMA over a 64-wide operand yields the 64-row result twice.
__device__ __forceinline__ uint64_t mndesc_dup(uint32_t saddr) { return sdesc_sw128(saddr, 0, 1024); }

// GEN = false: a whole (sequence, head) per CTA with d_k = d_v = 64; true: segments, 64-column
// slices of wider heads and the accumulating pass (the SegArgs), at a few registers' cost.
template <int NLEV, int NST, bool GEN>
__global__ void __maxnreg__(96)
tc_fwd_pipe(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
            const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
            const __nv_bfloat16* __restrict__ q,
            const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
            const float* __restrict__ log_a, const float* __restrict__ lam,
            float* __restrict__ out, int H, int T, int L, const int* __restrict__ cu,
            unsigned int* status, const SegArgs sa) {
  using LY = PipeLayout<NLEV, NST>;
  constexpr int kLevels = NLEV;   // chunk-level states on chip in this instantiation
  constexpr int kPStages = NST;   // Q/K/V ring stages
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, by pointer arithmetic on the shared array so that the compiler
  // keeps shared-memory (not generic) loads and stores for everything derived from it
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = warp & 3;
  const int row = sub * 32 + lane;
  const uint32_t lane_off = uint32_t(sub * 32) << 16;
  // blockIdx.x = head * ndv + value tile (64 columns of v and out); blockIdx.z = segment
  const int ndv = GEN ? sa.ndv : 1;
  const int h = blockIdx.x / ndv, sq = blockIdx.y;
  const int vcol = GEN ? (blockIdx.x % ndv) * kD : 0;   // first v / out column of this CTA
  const int qcol = GEN ? sa.qcol : 0;                   // first q / k column of this launch
  const int dk_tot = GEN ? sa.dk_tot : kD, dv_tot = GEN ? sa.dv_tot : kD;
  const bool accum = GEN && sa.accumulate;
  const int segg = GEN ? sa.g : 30;

  const SeqSpan sp = seq_span(sq, T, cu, status);
  if (sp.len <= 0) return;
  // This CTA walks segment J: chunks c0 .. c0 + nch - 1 of the sequence, c0 = J * 2^g.
  // Loops below run over the local index c (ring stages and barrier phases); the global
  // chunk index c0 + c gives token positions and the Fenwick bits.  Levels g and above of
  // the segment's chunks are the bits of J: their block states come pre-filled.
  const int nch_seq = (sp.len + kC - 1) / kC;
  const int J = blockIdx.z;
  const int c0 = segg >= 30 ? 0 : (J << segg);
  if (segg >= 30 ? J > 0 : c0 >= nch_seq) return;
  const int nch = segg >= 30 ? nch_seq : min(nch_seq - c0, 1 << segg);

  auto stage = [sm](int i) { return sm + i * kStage; };
  uint8_t* slots = sm + LY::kOffSlots;
  uint8_t* qh = sm + LY::kOffQh;
  float* lamA = reinterpret_cast<float*>(sm + LY::kOffLam);
  float* gs = reinterpret_cast<float*>(sm + LY::kOffG);
  float* cj = reinterpret_cast<float*>(sm + LY::kOffCj);
  float* lamB = reinterpret_cast<float*>(sm + LY::kOffLamB);
  float* scan = reinterpret_cast<float*>(sm + LY::kOffScan);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + LY::kOffBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + LY::kOffMisc);  // [0] TMEM base, [1] abort
  uint32_t* abort_flag = &misc[1];

  if (warp == 0) {
    tmem_alloc(&misc[0], 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int i = 0; i < kPNumBars; ++i) {
      uint32_t cnt = 1;  // TMA / tcgen05.commit arrivals
      if (i >= B_EMPTY && i < B_EMPTY + kPStages) cnt = 2;  // both MMA issuers
      if (i == B_PFULL || i == B_KS || (i >= B_GREADY && i < B_GREADY + kPG)) cnt = kPNA;
      if (i == B_PREFILL) cnt = 1 + kPNB;   // the producer's copies and group B's Q copy
      if (i == B_HEMPTY || i == B_LV || i == B_LV1 || i == B_OEMPTY || i == B_REMPTY ||
          (i >= B_GEMPTY && i < B_GEMPTY + kPG) || (i >= B_OSTAGED && i < B_OSTAGED + kPStages))
        cnt = kPNB;
      mbar_init(&bars[i], cnt);
    }
    fence_mbar_init();
    misc[1] = 0;
    prefetch_tensormap(&tmq);
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // a later segment reads the pre-filled block states: the pre-pass must be complete (the first
  // segment of a sequence starts while it still runs)
  if (c0 > 0) griddep_wait();
  const uint32_t tmem = misc[0];
  auto W = [&](int b, uint32_t parity) { return pwait(&bars[b], parity, abort_flag, status); };
  auto is_full = [&](int c) { return (c0 + c + 1) * kC <= sp.len; };
  auto tok_of = [&](int c) { return sp.start + (long long)(c0 + c) * kC; };   // first token
  auto nrows = [&](int c) { return min(kC, sp.len - (c0 + c) * kC); };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Loads Q, K, V of chunk c into stage c % 3 once that stage is free: both MMA issuers are
    // done with chunk c - 3, whose output tile group B staged there, and this thread has
    // stored that tile (TMA store, waited until its shared-memory reads are done).  Doing the
    // store here keeps its wait out of group B's chunk loop.  A ragged last chunk is loaded
    // by group A with plain loads; B_FREE tells it the stage is free.
    if (lane == 0) {
      int last0 = -1, last1 = -1, last2 = -1;
      bool ok = true;
      auto store_out = [&](int cc) {
        if (!W(B_OSTAGED + cc % kPStages, (cc / kPStages) & 1)) return false;
        if (is_full(cc)) {
          const int tok0 = static_cast<int>(tok_of(cc));
          if (accum) {   // a later d_k slice adds its share to the output
            tma_reduce_add_3d(&tmo, stage(cc % kPStages), vcol, h, tok0);
            tma_reduce_add_3d(&tmo, stage(cc % kPStages) + kTile, vcol + 32, h, tok0);
          } else {
            tma_store_3d(&tmo, stage(cc % kPStages), vcol, h, tok0);
            tma_store_3d(&tmo, stage(cc % kPStages) + kTile, vcol + 32, h, tok0);
          }
          bulk_commit();
          bulk_wait_read();
        }
        return true;
      };
      if (c0 > 0) {
        // block states of the levels above the segment (set bits of J), ahead of the loads
        const uint8_t* blk = sa.blocks + (size_t)(sq * gridDim.x + blockIdx.x) * sa.nblk * 8192;
        uint32_t bytes = 0;
        for (int b = segg; b < NLEV; ++b)
          if ((J >> (b - segg)) & 1) bytes += 8192;
        mbar_arrive_expect_tx(&bars[B_PREFILL], bytes);
        for (int b = segg; b < NLEV; ++b) {
          const int bs = b - segg;
          if ((J >> bs) & 1)
            bulk_load(slots + b * 8192,
                      blk + (size_t)seg_block_index(sa.nseg, bs, (J >> bs) - 1) * 8192, 8192,
                      &bars[B_PREFILL]);
        }
      }
      for (int c = 0; c < nch; ++c) {
        const int s = c % kPStages, kk = c / kPStages;
        if (c >= kPStages && (!W(B_EMPTY + s, (kk & 1) ^ 1) || !store_out(c - kPStages))) {
          ok = false;
          break;
        }
        if (is_full(c)) {
          const int tok0 = static_cast<int>(tok_of(c));
          mbar_arrive_expect_tx(&bars[B_FULL + s], 3 * kTile);
          tma_load_3d(stage(s), &tmq, &bars[B_FULL + s], qcol, h, tok0);
          tma_load_3d(stage(s) + kTile, &tmk, &bars[B_FULL + s], qcol, h, tok0);
          tma_load_3d(stage(s) + 2 * kTile, &tmv, &bars[B_FULL + s], vcol, h, tok0);
          if (s == 0) last0 = c; else if (s == 1) last1 = c; else last2 = c;
        } else {
          mbar_arrive(&bars[B_FREE]);
        }
      }
      for (int cc = nch > kPStages ? nch - kPStages : 0; ok && cc < nch; ++cc) ok = store_out(cc);
      bulk_wait_all();  // output tiles written
      if (*reinterpret_cast<volatile uint32_t*>(abort_flag)) {
        // an aborted CTA still lets its own copies land before it exits
        if (c0 > 0) mbar_wait(&bars[B_PREFILL], 0, 200000000ull);
        if (last0 >= 0) mbar_wait(&bars[B_FULL + 0], (last0 / kPStages) & 1, 200000000ull);
        if (last1 >= 0) mbar_wait(&bars[B_FULL + 1], (last1 / kPStages) & 1, 200000000ull);
        if (last2 >= 0) mbar_wait(&bars[B_FULL + 2], (last2 / kPStages) & 1, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ intra-chunk MMA issuer
    // S(c) = Q K^T and P V(c); S(c + 1) overwrites P(c), so it follows P V(c).
    if (lane == 0) {
      bool ok = W(B_FULL, 0);
      if (ok) {
        tc_fence_after();
        const uint64_t qd = kdesc(smem_u32(stage(0))), kd = kdesc(smem_u32(stage(0)) + kTile);
#pragma unroll
        for (int x = 0; x < kD / 16; ++x) mma_ss(tmem + kPColSP, qd + 2 * x, kd + 2 * x, kIdescS, x > 0);
        mma_commit(&bars[B_SFULL]);
      }
      for (int c = 0; ok && c < nch; ++c) {
        const int s = c % kPStages;
        if (!W(B_PFULL, c & 1) || !W(B_OEMPTY, (c & 1) ^ 1)) break;
        tc_fence_after();
        // K-step x covers keys 16x..16x+15, their fp16 P in columns 16x..16x+7
        const uint64_t vd = mndesc(smem_u32(stage(s)) + 2 * kTile);
#pragma unroll
        for (int x = 0; x < kC / 16; ++x)
          mma_ts(tmem + kPColO, tmem + kPColSP + 16 * x, vd + 128 * x, kIdescPVh, x > 0);
        mma_commit(&bars[B_OFULL]);
        mma_commit(&bars[B_SPEMPTY]);
        mma_commit(&bars[B_EMPTY + s]);   // this issuer's reads of stage s are done
        if (c + 1 < nch) {
          const int s1 = (c + 1) % kPStages;
          if (!W(B_FULL + s1, ((c + 1) / kPStages) & 1) || !W(B_SPEMPTY, c & 1)) break;
          tc_fence_after();
          const uint64_t qd = kdesc(smem_u32(stage(s1))), kd = kdesc(smem_u32(stage(s1)) + kTile);
#pragma unroll
          for (int x = 0; x < kD / 16; ++x) mma_ss(tmem + kPColSP, qd + 2 * x, kd + 2 * x, kIdescS, x > 0);
          mma_commit(&bars[B_SFULL]);
        }
      }
      mma_commit(&bars[B_DRAIN]);
      mbar_wait(&bars[B_DRAIN], 0, 200000000ull);
    }
  } else if (warp < kPB0) {
    // ------------------------------------------------------------ group A
    const int wa = warp - kPA0;     // 0..7
    const int part = wa >> 2;       // column blocks part, part + 2; K columns 32*part..
    constexpr int kNP = (kLogC + 1 + kLevels + 1) / 2;   // lam levels per thread, over 2 parts
    float pf[kNP];
    float pf_la = 0.f;
    auto prefetch = [&](int c) {
      const int cg = c0 + c;
      const int t = cg * kC + row;
      const bool okt = t < sp.len;
      const long long tok = sp.start + t;
      const float* lr = lam + (tok * H + h) * L;
#pragma unroll
      for (int i = 0; i < kNP; ++i) {
        const int l = part + 2 * i;
        // inter-chunk levels only where chunk c reads them (bit l - 1 - log2 C of c): each
        // row load that touches another cache sector costs the mask/scan warps time
        const bool need = l <= kLogC || ((cg >> (l - 1 - kLogC)) & 1);
        pf[i] = (okt && l < L && need) ? __ldg(lr + l) : 0.f;
      }
      if (part == 0) pf_la = okt ? __ldg(log_a + tok * H + h) : 0.f;
    };
    // Decay scan of chunk c: g = inclusive cumsum of log a (warp shuffles + a cross-warp
    // carry), the column factors cj and the pre-scaled lam table.  It runs after the mask of
    // chunk c - 1 and before that chunk's K scaling, so it never waits behind the slowest
    // K scaling warp.
    float g_row = 0.f, g0 = 0.f, gend = 0.f;
    bool factored = true;
    // L2 prefetch of chunk cc's lam and log a.  For one head the rows of a chunk are short
    // pieces far apart; across the H heads they form one contiguous block per chunk, so each
    // head's CTA pulls its 1/H share of the block, and the per-row loads then hit L2.  Whole
    // chunks only (the block lies inside the tensors), and only where the 16-byte rule of
    // bulk copies holds; it is a hint and changes no result.
    auto l2_prefetch = [&](int cc) {
      if (cc >= nch || !is_full(cc)) return;
      const long long tok0 = tok_of(cc);
      const float* lb = lam + (tok0 * H + (long long)h * kC) * L;    // share h of the block
      const float* ab = log_a + tok0 * H + (long long)h * kC;
      if (((reinterpret_cast<uintptr_t>(lb) | (uint32_t)(kC * L * 4)) & 15u) == 0)
        bulk_prefetch_l2(lb, kC * L * 4);
      if ((reinterpret_cast<uintptr_t>(ab) & 15u) == 0) bulk_prefetch_l2(ab, kC * 4);
    };
    auto decay_scan = [&](int c) {
      const int gb = c % kPG, gk = c / kPG;  // g buffer and its use index
      if (wa == 0 && lane == 0) l2_prefetch(c + 2);
      const int n = nrows(c);
      float pfc[kNP];
#pragma unroll
      for (int i = 0; i < kNP; ++i) pfc[i] = pf[i];
      const float la = pf_la;
      if (c + 1 < nch) prefetch(c + 1);
      W(B_GEMPTY + gb, (gk & 1) ^ 1);   // group B is done with g[gb] of chunk c - 3
      float x = la;
      if (part == 0) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane == 31) scan[sub] = x;
      }
      named_sync(1, kPNA);  // also: every mask read of the previous chunk is done
      if (part == 0) {
        float off = 0.f;
        for (int w = 0; w < sub; ++w) off += scan[w];
        gs[gb * kC + row] = x + off;
      }
      named_sync(1, kPNA);
      g_row = gs[gb * kC + row];
      g0 = gs[gb * kC];
      gend = gs[gb * kC + n - 1];
      factored = (g0 - gend) <= 80.f;
      if (part == 0) cj[row] = factored ? __expf(g0 - g_row) : 0.f;
      // lam table of this row for levels 0..7, pre-multiplied by exp(g_i - g_0) when the
      // decay factorises (the column factor exp(g_0 - g_j) is cj)
      const float rsc = factored ? __expf(g_row - g0) : 1.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) lamA[row * kPLamStride + part + 2 * i] = pfc[i] * rsc;
      // inter-chunk levels for group B's readout weights, with the row's decay from the chunk
      // start (g_row <= 0, so the factor stays finite)
      const float eg = __expf(g_row);
#pragma unroll
      for (int i = 4; i < kNP; ++i) {
        const int b = part + 2 * i - (kLogC + 1);
        if (b < kLevels) lamB[(gb * kC + row) * kLevels + b] = pfc[i] * eg;
      }
      mbar_arrive(&bars[B_GREADY + gb]);
    };
    if (wa == 0 && lane == 0) l2_prefetch(1);
    prefetch(0);
    decay_scan(0);
    for (int c = 0; c < nch; ++c) {
      const int s = c % kPStages, kk = c / kPStages;
      const int n = nrows(c);
      if (!is_full(c)) {
        // ragged last chunk: plain loads into the stage, rows past the end zero-filled, once
        // the producer has stored the output tile of chunk c - 3 from it
        W(B_FREE, 0);
        const long long tok0 = tok_of(c);
#pragma unroll
        for (int tsr = 0; tsr < 3; ++tsr) {
          const __nv_bfloat16* src = tsr == 0 ? q : (tsr == 1 ? k : v);
          const int rowlen = tsr == 2 ? dv_tot : dk_tot;
          const int col0 = tsr == 2 ? vcol : qcol;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int col = part * 32 + j * 8;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (row < n) {
              val = *reinterpret_cast<const uint4*>(src + ((tok0 + row) * H + h) * rowlen + col0 + col);
              if (tsr == 2) val = bf16x8_to_f16x8(val);   // V in fp16
            }
            *reinterpret_cast<uint4*>(stage(s) + tsr * kTile + sw128_off(row, col)) = val;
          }
        }
        fence_proxy_async_smem();
        named_sync(1, kPNA);
        if (wa == 0 && lane == 0) mbar_arrive(&bars[B_FULL + s]);
      }
      W(B_FULL + s, kk & 1);
      if (is_full(c)) {
        // V to fp16 in place (the element layout is the same), while S(c) runs
        uint4* vt = reinterpret_cast<uint4*>(stage(s) + 2 * kTile);
        const int t = wa * 32 + lane;
#pragma unroll
        for (int i = 0; i < 4; ++i) vt[t + 256 * i] = bf16x8_to_f16x8(vt[t + 256 * i]);
        fence_proxy_async_smem();
      }
      W(B_SFULL, c & 1);
      tc_fence_after();
      named_sync(1, kPNA);  // cj and the lam table are visible to the whole group
      // ---- causal Fenwick mask on S -> P (fp16, in place), 16 keys at a time ----
      // The two warps of a sub-partition take alternate 16-key groups, so each gets half of
      // the diagonal block (per-element levels) and half of every off-diagonal block.
      const uint32_t spc = tmem + lane_off + kPColSP;
      const int rb = sub;
      const float* lr = lamA + row * kPLamStride;
#pragma unroll 1
      for (int g16 = part; g16 < 8; g16 += 2) {  // keys 16*g16 .. 16*g16+15
        const int kb = g16 >> 1;                // their 32-key block
        uint32_t hi[8];
        if (kb > rb) {
#pragma unroll
          for (int e = 0; e < 8; ++e) hi[e] = 0u;
        } else {
          float sv[16];
          tmem_ld16(spc + 16 * g16, sv);
          tmem_wait_ld();
          // weight of key j: (lam x exp(g_i - g_0)) x exp(g_0 - g_j) when that stays finite,
          // else lam x exp(g_i - g_j) element by element
          float cw[16];
          if (factored) {
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 c4 = *reinterpret_cast<const float4*>(cj + 16 * g16 + e);
              cw[e] = c4.x; cw[e + 1] = c4.y; cw[e + 2] = c4.z; cw[e + 3] = c4.w;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) cw[e] = __expf(g_row - gs[(c % kPG) * kC + 16 * g16 + e]);
          }
          if (kb < rb) {
            // off-diagonal: one Fenwick level, 1 + msb(i ^ j) = 6 + msb(rb ^ kb)
            const float wblk = lr[6 + (31 - __clz(rb ^ kb))];
#pragma unroll
            for (int e = 0; e < 16; e += 2)
              hi[e >> 1] = pack_f16(sv[e] * wblk * cw[e], sv[e + 1] * wblk * cw[e + 1]);
          } else {
            // diagonal block: level 1 + msb(lane ^ jj) (0 when equal: clz(0) = 32), j <= i
            const int j0 = 16 * (g16 & 1);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              float p[2];
#pragma unroll
              for (int t2 = 0; t2 < 2; ++t2) {
                const int jj = j0 + e + t2;
                const float val = sv[e + t2] * lr[32 - __clz(jj ^ lane)] * cw[e + t2];
                p[t2] = jj <= lane ? val : 0.f;
              }
              hi[e >> 1] = pack_f16(p[0], p[1]);
            }
          }
        }
        tmem_st8(spc + 16 * g16, hi);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL]);
      const float gend_c = gend;
      if (c + 1 < nch) decay_scan(c + 1);
      // ---- chunk-state operand: K rows scaled by exp(G - g_s), fp16, in place ----
      // (after the mask, overlapping P V(c) and S(c + 1) on the tensor cores).  The causal
      // mask loads sub-partitions 0..3 in the ratio 1:2:3:4, so the K rows are dealt out the
      // other way round: 48, 40, 24 and 16 rows to the two warps of sub-partitions 0..3.
      if (c + 1 < nch) {
        // H^T(c - 1) must be done before K scaling (c) is signalled: the MMA issuer waits for
        // the K-scaled barrier once per chunk, so this group may run at most one phase ahead
        if (c > 0) W(B_HFULL, (c - 1) & 1);
        uint8_t* kt = stage(s) + kTile;
        const int r0 = sub == 0 ? 0 : (sub == 1 ? 48 : (sub == 2 ? 88 : 112));
        const int nrows = sub == 0 ? 48 : (sub == 1 ? 40 : (sub == 2 ? 24 : 16));
        const int t64 = part * 32 + lane;
#pragma unroll 1
        for (int unit = t64; unit < nrows * 8; unit += 64) {
          const int kr = r0 + (unit >> 3);
          const float ks = kr < n ? __expf(gend_c - gs[(c % kPG) * kC + kr]) : 0.f;
          const uint32_t off = sw128_off(kr, (unit & 7) * 8);
          const uint4 raw = *reinterpret_cast<const uint4*>(kt + off);
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t hv4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
            hv4[e] = pack_f16(pr.x * ks, pr.y * ks);
          }
          *reinterpret_cast<uint4*>(kt + off) = make_uint4(hv4[0], hv4[1], hv4[2], hv4[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars[B_KS]);
      }

    }
  } else if (warp < kPI2) {
    // ------------------------------------------------------------ group B
    const int half = (warp - kPB0) >> 2;   // which 32 of the 64 output columns
    const int j_dv = row & 63;             // merge: row of H^T (a d_v index) ...
    const int dk0 = 32 * (row >> 6) + 16 * half;  // ... and the 16 d_k columns it merges
    float gtot[kLevels];
#pragma unroll
    for (int b = 0; b < kLevels; ++b) gtot[b] = 0.f;
    if (c0 > 0) {
      // The first chunk of a later segment reads the levels above the segment: its fp16 Q
      // copy (made for every other chunk during the previous merge) is made here, and the
      // pre-fill barrier, which the readouts wait for, also waits for it.
      W(B_FULL, 0);
      {
        const uint4* qsrc = reinterpret_cast<const uint4*>(stage(0));
        uint4* qdst = reinterpret_cast<uint4*>(qh);
        const int t = (warp - kPB0) * 32 + lane;
#pragma unroll
        for (int i = 0; i < 4; ++i) qdst[t + 256 * i] = bf16x8_to_f16x8(qsrc[t + 256 * i]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[B_PREFILL]);
      // total log decay of each pre-filled block (levels g.. : the set bits of J)
      const float* bd = sa.block_decay + (size_t)(sq * gridDim.x + blockIdx.x) * sa.nblk;
#pragma unroll
      for (int b = 0; b < kLevels; ++b) {
        const int bs = b - segg;
        if (bs >= 0 && ((J >> bs) & 1)) gtot[b] = bd[seg_block_index(sa.nseg, bs, (J >> bs) - 1)];
      }
    }
    uint32_t u = 0;
    // An fp16 operand out of range (|x| >= 65520 rounds to inf) reaches the output as inf
    // or NaN.  Any such value makes this thread's running sum of its outputs inf or NaN, so
    // one check of the sum at the end catches it; the host sees a status bit.
    float osum = 0.f;
    for (int c = 0; c < nch; ++c) {
      const int s = c % kPStages;
      const int n = nrows(c);
      const int cg = c0 + c;   // global chunk index: its bits are the levels read
      W(B_GREADY + c % kPG, (c / kPG) & 1);
      const float gend = gs[(c % kPG) * kC + n - 1];
      const float* lamv = lamB + ((c % kPG) * kC + row) * kLevels;
      // ---- epilogue: o = P V + sum_b lam[., 1+log2 C+b] exp(g + gap_b) R_b ----
      // P V first: it seeds the accumulator and frees the P V columns for chunk c + 1 at once.
      // Pairs of columns go through the packed f32x2 pipe.
      float2 o2[16];
      W(B_OFULL, c & 1);
      tc_fence_after();
      {
        float r0[32];
        tmem_ld32(tmem + lane_off + kPColO + 32 * half, r0);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) o2[e] = make_float2(r0[2 * e], r0[2 * e + 1]);
      }
      tc_fence_before();
      mbar_arrive(&bars[B_OEMPTY]);
      float gap = 0.f;
      int cur0 = -1, cur1 = -1;  // readout chain being drained
#pragma unroll
      for (int b = 0; b < kLevels; ++b) {
        if (!((cg >> b) & 1)) continue;
        if (b > cur1) {
          if (cur1 >= 0) {
            tc_fence_before();
            mbar_arrive(&bars[B_REMPTY]);
            ++u;
          }
          next_chain<NLEV>(cg, b, cur0, cur1);
          W(B_RFULL, u & 1);
          tc_fence_after();
        }
        const float w = lamv[b] * __expf(gap);
        const float2 w2 = make_float2(w, w);
        float r0[32];
        tmem_ld32(tmem + lane_off + kPColR + 64 * (b - cur0) + 32 * half, r0);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) o2[e] = __ffma2_rn(w2, make_float2(r0[2 * e], r0[2 * e + 1]), o2[e]);
        gap += gtot[b];
      }
      if (cur1 >= 0) {
        tc_fence_before();
        mbar_arrive(&bars[B_REMPTY]);
        ++u;
      }
      // ---- Fenwick merge: level m = H + sum_{b<m} exp(decay after block b) S_b ----
      if (c + 1 < nch) {
        const int m = __ffs(~cg) - 1;   // below g: a segment skips the merge after its last chunk
        // the lower levels do not depend on this chunk: sum them before H arrives
        float2 hv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) hv[e] = make_float2(0.f, 0.f);
        float acc = gend;
#pragma unroll
        for (int b = 0; b < kLevels; ++b) {
          if (b < m) {
            const float f = __expf(acc);
            const float2 f2 = make_float2(f, f);
            const uint8_t* sl = slots + b * 8192;
#pragma unroll
            for (int qd = 0; qd < 2; ++qd) {
              const uint32_t off = sw128_off(j_dv, dk0 + 8 * qd);
              const uint4 a4 = *reinterpret_cast<const uint4*>(sl + off);
              const uint32_t av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 ah = __half22float2(*reinterpret_cast<const __half2*>(&av[e]));
                hv[4 * qd + e] = __ffma2_rn(f2, ah, hv[4 * qd + e]);
              }
            }
            acc += gtot[b];
          }
        }
        W(B_HFULL, c & 1);
        tc_fence_after();
        {
          // H^T = V^T K~; this thread's 16 d_k columns
          float t16[16];
          tmem_ld16(tmem + lane_off + kPColH + dk0, t16);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            hv[e] = __fadd2_rn(hv[e], make_float2(t16[2 * e], t16[2 * e + 1]));
        }
        tc_fence_before();
        mbar_arrive(&bars[B_HEMPTY]);
        uint8_t* dsl = slots + m * 8192;
#pragma unroll
        for (int qd = 0; qd < 2; ++qd) {
          uint32_t hh[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) hh[e] = pack_f16(hv[4 * qd + e].x, hv[4 * qd + e].y);
          const uint32_t off = sw128_off(j_dv, dk0 + 8 * qd);
          *reinterpret_cast<uint4*>(dsl + off) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
        }
        // fp16 copy of Q(c + 1) for its readouts: every readout of chunk c has been drained,
        // and the level-ready signal below also releases this copy to the MMA issuer
        W(B_FULL + (c + 1) % kPStages, ((c + 1) / kPStages) & 1);
        {
          const uint4* qsrc = reinterpret_cast<const uint4*>(stage((c + 1) % kPStages));
          uint4* qdst = reinterpret_cast<uint4*>(qh);
          const int t = (warp - kPB0) * 32 + lane;
#pragma unroll
          for (int i = 0; i < 4; ++i) qdst[t + 256 * i] = bf16x8_to_f16x8(qsrc[t + 256 * i]);
        }
        fence_proxy_async_smem();
#pragma unroll
        for (int b = 0; b < kLevels; ++b)
          if (b == m) gtot[b] = acc;
        mbar_arrive(&bars[(c & 1) ? B_LV1 : B_LV]);
      }
      if (row < n) {
#pragma unroll
        for (int e = 0; e < 16; ++e) osum += o2[e].x + o2[e].y;
      }
      if (n == kC) {
        // Whole chunk: stage the 128 x 64 fp32 tile in the Q (columns 0..31) and K (32..63)
        // tiles of this stage -- every reader of them is done by now -- in the 128-byte
        // swizzle, and let TMA write it out; row-per-thread global stores would touch one
        // cache line per lane.
        uint8_t* stg = stage(s) + half * kTile;
#pragma unroll
        for (int qd = 0; qd < 8; ++qd)
          *reinterpret_cast<float4*>(stg + row * 128 + ((qd ^ (row & 7)) << 4)) =
              make_float4(o2[2 * qd].x, o2[2 * qd].y, o2[2 * qd + 1].x, o2[2 * qd + 1].y);
        fence_proxy_async_smem();
        mbar_arrive(&bars[B_OSTAGED + s]);  // the producer stores the tile
      } else {
        if (row < n) {
          float* dst = out + ((tok_of(c) + row) * H + h) * dv_tot + vcol + 32 * half;
          if (accum) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              atomicAdd(dst + 2 * e, o2[e].x);
              atomicAdd(dst + 2 * e + 1, o2[e].y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; e += 2)
              *reinterpret_cast<float4*>(dst + 2 * e) =
                  make_float4(o2[e].x, o2[e].y, o2[e + 1].x, o2[e + 1].y);
          }
        }
        mbar_arrive(&bars[B_OSTAGED + s]);  // nothing staged; keeps the phases in step
      }
      mbar_arrive(&bars[B_GEMPTY + c % kPG]);
    }
    const bool nonfinite = !(fabsf(osum) <= 3.402823466e38f);
    if (__any_sync(0xffffffffu, nonfinite) && lane == 0) atomicOr(status, LLATTN_DEV_NONFINITE);
  } else {
    // ------------------------------------------------------------ inter-chunk MMA issuer
    // Per chunk c: the readout chains of the set bits of c (they need the level states left
    // by the merge after chunk c - 1), then H^T(c) if a merge follows (it needs the scaled K
    // of chunk c).  Blocking waits, in chunk order: no barrier runs a phase ahead of this
    // waiter, and a waiting issuer takes no issue slots from the math warps.
    if (lane == 0) {
      uint32_t u = 0;  // readout chains issued so far
      bool prefilled = c0 == 0;
      for (int c = 0; c < nch; ++c) {
        const int s = c % kPStages;
        if (!W(B_FULL + s, (c / kPStages) & 1)) break;
        const uint32_t qa = smem_u32(stage(s)), ka = qa + kTile, va = qa + 2 * kTile;
        bool ok = true;
        int cb0 = 0, cb1 = 0;
        const int cg = c0 + c;
        for (bool more = next_chain<NLEV>(cg, 0, cb0, cb1); more; more = next_chain<NLEV>(cg, cb1 + 1, cb0, cb1)) {
          if (!prefilled) {   // the block states above the segment have landed
            if (!W(B_PREFILL, 0)) {
              ok = false;
              break;
            }
            prefilled = true;
          }
          if ((c > 0 && !W(((c - 1) & 1) ? B_LV1 : B_LV, ((c - 1) >> 1) & 1)) ||
              !W(B_REMPTY, (u & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qd = kdesc(smem_u32(qh));   // fp16 copy of Q(c)
          const uint64_t sd = kdesc(smem_u32(slots + cb0 * 8192));
          const uint32_t idr = idesc_f16(128, 64 * (cb1 - cb0 + 1), 0, 0);
#pragma unroll
          for (int x = 0; x < kD / 16; ++x) mma_ss(tmem + kPColR, qd + 2 * x, sd + 2 * x, idr, x > 0);
          mma_commit(&bars[B_RFULL]);
          ++u;
        }
        if (!ok) break;
        if (c + 1 < nch) {
          if (!W(B_KS, c & 1) || !W(B_HEMPTY, (c & 1) ^ 1)) break;
          tc_fence_after();
          // A = V^T (fp16, rows duplicated), B = K~ (fp16, in the K tile)
          const uint64_t vd = mndesc_dup(va);
          const uint64_t kd = mndesc(ka);
#pragma unroll
          for (int x = 0; x < kC / 16; ++x) mma_ss(tmem + kPColH, vd + 128 * x, kd + 128 * x, kIdescHT, x > 0);
          mma_commit(&bars[B_HFULL]);
        }
        mma_commit(&bars[B_EMPTY + s]);   // this issuer's reads of stage s are done
      }
      mma_commit(&bars[B_DRAIN2]);
      mbar_wait(&bars[B_DRAIN2], 0, 200000000ull);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ==========================================================================================
// Segment pre-pass.  A sequence walked in segments of 2^g chunks (one CTA each) needs, at the
// start of segment J, the levels above the segment: for every set bit b of J, the state of the
// 2^b segments just before J's aligned group of 2^(b+1) segments, decayed to that block's end.
// That is the Fenwick binary counter of the walk kernel one level up, over segments instead
// of chunks ([IT] "Partizionamento Gerarchico": the buckets are dyadic blocks, so a block of
// segments is a union of whole lower blocks).  tc_seg_total computes each segment's total
// state on the tensor cores; seg_blocks runs the counter and stores each block once, as the
// fp16 slot image the walk kernel copies into shared memory.
// ==========================================================================================
constexpr int kSegThreads = 288;   // warp 0: TMA producer and MMA issuer (lane 0); warps 1..8: math
constexpr int kSegMath = 256;
constexpr uint32_t kSegSmem = 2 * 2 * kTile + kC * 4 + 64 + 64 + 1024;

// One CTA per (head tile, sequence, segment J) for every segment but a sequence's last:
//   seg_state[item] = sum over the segment's tokens s of exp(G_end - g_s) v_s k_s^T, stored
//   [d_v][d_k] fp32 (the transposed state, as the walk kernel's merge forms it), and
//   seg_decay[item] = the segment's total log decay G_end - G_start.
// Chunks are taken last to first, so a running decay D (from the end of the chunk being
// scaled to the end of the segment) folds into each token's factor and one TMEM accumulator
// collects the whole sum: K~ = exp(D + sum_{r > s in chunk} log a_r) K, fp16, factors <= 1.
__global__ void __launch_bounds__(kSegThreads, 1)
tc_seg_total(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
             const float* __restrict__ log_a, int H, int T, const int* __restrict__ cu,
             unsigned int* status, const SegArgs sa, float* __restrict__ seg_state,
             float* __restrict__ seg_decay) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // seg_blocks may start now (it waits for this grid before it reads the totals), and with it
  // the walk, whose first segments need no pre-fill
  griddep_launch_dependents();
  const int h = blockIdx.x / sa.ndv, sq = blockIdx.y, J = blockIdx.z;
  const int vcol = (blockIdx.x % sa.ndv) * kD;
  const SeqSpan sp = seq_span(sq, T, cu, status);
  const int nch_seq = (sp.len + kC - 1) / kC;
  const int c0 = J << sa.g;
  // only segments followed by another one are read (and those are whole)
  if (c0 + (1 << sa.g) >= nch_seq) return;
  const int n = 1 << sa.g;
  auto stage = [sm](int i) { return sm + i * 2 * kTile; };   // K tile, then V tile
  float* fac = reinterpret_cast<float*>(sm + 4 * kTile);
  float* part = fac + kC;                                     // scan carries (4 floats)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 4 * kTile + kC * 4 + 64);
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 6);     // [0] TMEM base, [1] abort
  uint32_t* abort_flag = &misc[1];
  enum { S_FULL = 0, S_SCALED = 2, S_MDONE = 3, S_DRAIN = 4 };
  if (warp == 0) {
    tmem_alloc(&misc[0], 64);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(&bars[S_FULL], 1);
    mbar_init(&bars[S_FULL + 1], 1);
    mbar_init(&bars[S_SCALED], kSegMath);
    mbar_init(&bars[S_MDONE], 1);
    mbar_init(&bars[S_DRAIN], 1);
    fence_mbar_init();
    misc[1] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  auto W = [&](int b, uint32_t parity) { return pwait(&bars[b], parity, abort_flag, status); };
  // chunk processed at step i (last chunk first)
  auto chunk_tok = [&](int i) { return sp.start + (long long)(c0 + n - 1 - i) * kC; };

  if (warp == 0) {
    if (lane == 0) {
      auto load = [&](int i) {
        const int s = i & 1;
        const int tok0 = static_cast<int>(chunk_tok(i));
        mbar_arrive_expect_tx(&bars[S_FULL + s], 2 * kTile);
        tma_load_3d(stage(s), &tmk, &bars[S_FULL + s], sa.qcol, h, tok0);
        tma_load_3d(stage(s) + kTile, &tmv, &bars[S_FULL + s], vcol, h, tok0);
      };
      load(0);
      if (n > 1) load(1);
      int issued = 0, loads = n > 1 ? 2 : 1;
      for (int i = 0; i < n; ++i) {
        if (!W(S_SCALED, i & 1)) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(stage(i & 1)), va = ka + kTile;
        const uint64_t vd = mndesc_dup(va), kd = mndesc(ka);
#pragma unroll
        for (int x = 0; x < kC / 16; ++x)
          mma_ss(tmem, vd + 128 * x, kd + 128 * x, kIdescHT, (i > 0 || x > 0) ? 1u : 0u);
        mma_commit(&bars[S_MDONE]);
        ++issued;
        if (i + 2 < n) {   // the stage is free once this chunk's MMAs are done
          if (!W(S_MDONE, i & 1)) break;
          load(i + 2);
          ++loads;
        }
      }
      mma_commit(&bars[S_DRAIN]);
      mbar_wait(&bars[S_DRAIN], 0, 200000000ull);
      if (*reinterpret_cast<volatile uint32_t*>(abort_flag)) {
        // let this CTA's loads land before it exits
        for (int i = (loads > 2 ? loads - 2 : 0); i < loads; ++i)
          mbar_wait(&bars[S_FULL + (i & 1)], (i >> 1) & 1, 200000000ull);
      }
      (void)issued;
    }
  } else {
    // ------------------------------------------------ math warps: factors, K~ and V in fp16
    const int t = tid - 32;            // 0..255
    const int w = t >> 5;              // 0..7
    float D = 0.f;                     // log decay from the current chunk's end to the segment end
    // (a failed wait does not leave the loop: the named barriers below stay matched, and an
    // aborted CTA writes nothing)
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      W(S_FULL + s, (i >> 1) & 1);
      // inclusive prefix of log a inside the chunk by the first four warps
      float x = 0.f;
      if (t < kC) {
        x = __ldg(log_a + (chunk_tok(i) + t) * H + h);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane == 31) part[w] = x;
      }
      named_sync(1, kSegMath);
      const float Gc = part[0] + part[1] + part[2] + part[3];
      if (t < kC) {
        float off = 0.f;
        for (int q2 = 0; q2 < w; ++q2) off += part[q2];
        fac[t] = __expf(D + Gc - (x + off));   // exp(D + sum of log a after token t)
      }
      named_sync(1, kSegMath);
      // K rows scaled by their factor, V converted, both to fp16 in place
      uint8_t* kt = stage(s);
      uint4* vt = reinterpret_cast<uint4*>(stage(s) + kTile);
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const int unit = t + kSegMath * u4;            // 16-byte unit of the 128 x 128 B tile
        const float f = fac[unit >> 3];
        uint4 raw = *reinterpret_cast<const uint4*>(kt + unit * 16);
        uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
          wv[e] = pack_f16(pr.x * f, pr.y * f);
        }
        *reinterpret_cast<uint4*>(kt + unit * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        vt[unit] = bf16x8_to_f16x8(vt[unit]);
      }
      fence_proxy_async_smem();
      D += Gc;
      // one phase of S_SCALED at a time: the issuer has seen the previous one once its MMAs
      // of the previous chunk are done
      if (i > 0) W(S_MDONE, (i - 1) & 1);
      mbar_arrive(&bars[S_SCALED]);
    }
    if (W(S_MDONE, (n - 1) & 1) && !*reinterpret_cast<volatile uint32_t*>(abort_flag)) {
      tc_fence_after();
      // H^T rows (d_v) sit in TMEM lanes 0..63; warps with w % 4 in {0, 1} read them
      const int wq = (tid >> 5) & 3;
      if (wq < 2) {
        const int half = (tid >> 5) >= 5 ? 1 : 0;      // warps 1, 4 -> columns 0..31; 5, 8 -> 32..63
        float r[32];
        tmem_ld32(tmem + (uint32_t(wq * 32) << 16) + 32 * half, r);
        tmem_wait_ld();
        const size_t item = ((size_t)sq * gridDim.x + blockIdx.x) * (sa.nseg - 1) + J;
        float* dst = seg_state + item * (kD * kD) + (wq * 32 + lane) * kD + 32 * half;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(r[e], r[e + 1], r[e + 2], r[e + 3]);
        if (t == 0) seg_decay[item] = D;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// One CTA per (head tile, sequence): the binary counter over the sequence's segments.  After
// segment J's total is merged, the block it completes - the 2^m segments ending at J, m the
// trailing ones of J - is stored as an fp16 slot image ([d_v][d_k], 128-byte swizzle, the
// layout of the walk kernel's level states) with its total log decay.  Each thread owns 16
// consecutive elements of every state, so no thread reads another's.
constexpr int kBlkThreads = 256;
__global__ void __launch_bounds__(kBlkThreads)
seg_blocks(int T, const int* __restrict__ cu, unsigned int* status, const SegArgs sa,
           const float* __restrict__ seg_state, const float* __restrict__ seg_decay,
           uint8_t* __restrict__ blocks, float* __restrict__ block_decay) {
  extern __shared__ float cnt[];   // [levels][4096] fp32: the counter's slots
  griddep_launch_dependents();     // the walk may start: its first segments need no pre-fill
  griddep_wait();                  // the segment totals are complete
  const int t = threadIdx.x, sq = blockIdx.y;
  const SeqSpan sp = seq_span(sq, T, cu, status);
  const int nch_seq = (sp.len + kC - 1) / kC;
  const int nsq = (nch_seq + (1 << sa.g) - 1) >> sa.g;   // this sequence's segments
  const size_t pair = (size_t)sq * gridDim.x + blockIdx.x;
  const int r = t >> 2, col0 = (t & 3) * 16;             // this thread: row r, columns col0..+15
  float gdec[8];
#pragma unroll
  for (int b = 0; b < 8; ++b) gdec[b] = 0.f;
  for (int J = 0; J + 1 < nsq; ++J) {
    const size_t item = pair * (sa.nseg - 1) + J;
    const float4* src = reinterpret_cast<const float4*>(seg_state + item * (kD * kD) + r * kD + col0);
    float x[16];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const float4 f = src[q4];
      x[4 * q4] = f.x; x[4 * q4 + 1] = f.y; x[4 * q4 + 2] = f.z; x[4 * q4 + 3] = f.w;
    }
    const int m = __ffs(~J) - 1;
    float acc = seg_decay[item];
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (b < m) {
        const float f = __expf(acc);
        const float* sl = cnt + b * (kD * kD) + r * kD + col0;
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] += f * sl[e];
        acc += gdec[b];
      }
    }
    float* dsl = cnt + m * (kD * kD) + r * kD + col0;
#pragma unroll
    for (int e = 0; e < 16; ++e) dsl[e] = x[e];
#pragma unroll
    for (int b = 0; b < 8; ++b)
      if (b == m) gdec[b] = acc;
    // block (m, j) with j = (J + 1) / 2^m - 1, read by segments J + 1 .. J + 2^m
    const int blk = seg_block_index(sa.nseg, m, ((J + 1) >> m) - 1);
    uint8_t* img = blocks + (pair * sa.nblk + blk) * 8192;
#pragma unroll
    for (int q8 = 0; q8 < 2; ++q8) {
      uint32_t hv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) hv[e] = pack_f16(x[8 * q8 + 2 * e], x[8 * q8 + 2 * e + 1]);
      *reinterpret_cast<uint4*>(img + sw128_off(r, col0 + 8 * q8)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
    if (t == 0) block_decay[pair * sa.nblk + blk] = acc;
  }
}

}  // namespace

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

// [tokens, H, rowlen] bf16 viewed as a 3-D tensor {rowlen, H, tokens}; box {64, 1, 128}
// (one 64-column slice of a row), 128 B swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, int rowlen, int H, long long tokens) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)rowlen, (cuuint64_t)H, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)rowlen * 2, (cuuint64_t)H * rowlen * 2};
  const cuuint32_t box[3] = {kD, 1, kC};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// out [tokens, H, rowlen] fp32 as {rowlen, H, tokens}; box {32, 1, 128} (128 B rows), 128 B swizzle.
cudaError_t make_out_map(CUtensorMap* m, void* base, int rowlen, int H, long long tokens) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)rowlen, (cuuint64_t)H, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)rowlen * 4, (cuuint64_t)H * rowlen * 4};
  const cuuint32_t box[3] = {32, 1, kC};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// How a call is cut into CTAs.  One CTA (one per SM: shared memory and TMEM) walks 2^g chunks
// of one (sequence, head, 64-column value tile); a whole sequence when g = kNoSplit.  The time
// estimate, in chunk steps, is waves x (2^g + 2 steps of pipeline fill), plus the pre-pass for
// split sequences (about 2 steps of launches and a step per 8 chunk-tiles per SM of segment
// totals).  Packed batches count items at half the length bound (T only bounds them).
constexpr int kNoSplit = 30;
struct SegPlan {
  int g = kNoSplit, nseg = 1, nblk = 0;
};

std::atomic<int> g_seg_chunks_override{0};   // llattn_set_segment_chunks

SegPlan seg_plan(int nseq, int H, int T, int dk, int dv, bool varlen) {
  (void)dk;
  SegPlan pl;
  const int nch = (T + kC - 1) / kC;
  const int forced = g_seg_chunks_override.load();
  if (forced > 0) {
    int g = 0;
    while ((1 << g) < forced) ++g;
    if ((1 << g) >= nch) return pl;   // one segment covers every sequence
    const int nseg = (nch + (1 << g) - 1) >> g;
    if (chunk_levels(nseg) <= 8) {
      pl.g = g;
      pl.nseg = nseg;
      pl.nblk = total_blocks(nseg);
      return pl;
    }
  }
  const int vh = H * (dv / kD);
  const int nsm = sm_count();
  auto waves = [&](long long items) { return (double)((items + nsm - 1) / nsm); };
  // dense: equal items, so whole waves; packed: lengths spread over [0, T], so the work of the
  // items (at half the bound each, with ~3 steps of fixed cost per item) spread over the SMs,
  // plus the longest item
  auto estimate = [&](int len, long long per_seq, double pre) {
    if (!varlen) return waves((long long)nseq * vh * per_seq) * (len + 2) + pre;
    const double avg = 0.5 * nch;
    const double items = std::ceil(avg / len);
    return (double)nseq * vh * (avg + 3.0 * items) / nsm + len + pre;
  };
  double best = estimate(nch, 1, 0.0);
  for (int g = 1; (1 << g) < nch; ++g) {
    const int nseg = (nch + (1 << g) - 1) >> g;
    if (chunk_levels(nseg) > 8) continue;   // the counter over segments keeps <= 8 levels
    const double per = varlen ? 0.5 : 1.0;
    const double pre = 2.0 + (double)nseq * vh * (per * nch) / (8.0 * nsm);
    const double est = estimate(1 << g, nseg, pre);
    if (est < best) {
      best = est;
      pl.g = g;
      pl.nseg = nseg;
    }
  }
  pl.nblk = pl.nseg > 1 ? total_blocks(pl.nseg) : 0;
  return pl;
}

struct SegWorkspace {
  float* seg_state = nullptr;
  float* seg_decay = nullptr;
  uint8_t* blocks = nullptr;
  float* block_decay = nullptr;
  size_t bytes = 0;
};

SegWorkspace seg_workspace(const SegPlan& pl, int nseq, int H, int dv, void* base) {
  SegWorkspace w;
  if (pl.nseg <= 1) return w;
  const size_t pairs = (size_t)nseq * H * (dv / kD);
  const size_t items = pairs * (pl.nseg - 1);
  const size_t a = round_up(items * kD * kD * sizeof(float), 256);
  const size_t b = round_up(items * sizeof(float), 256);
  const size_t c = round_up(pairs * pl.nblk * 8192, 256);
  const size_t d = round_up(pairs * pl.nblk * sizeof(float), 256);
  w.bytes = a + b + c + d;
  if (base != nullptr) {
    uint8_t* p = static_cast<uint8_t*>(base);
    w.seg_state = reinterpret_cast<float*>(p);
    w.seg_decay = reinterpret_cast<float*>(p + a);
    w.blocks = p + a + b;
    w.block_decay = reinterpret_cast<float*>(p + a + b + c);
  }
  return w;
}

// A launch that may overlap the tail of the previous kernel in the stream (programmatic
// dependent launch): used only after this library's own pre-pass kernels, which trigger it.
struct PdlLaunch {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  PdlLaunch(const dim3& grid, int threads, size_t smem, cudaStream_t st, bool pdl) {
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 1 : 0;
  }
};

template <typename LY, bool GEN>
cudaError_t launch_walk(const dim3& grid, cudaStream_t st, const CUtensorMap& mq,
                        const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                        const Problem& p, const SegArgs& sa, bool pdl) {
  PdlLaunch l(grid, kPThreads, LY::kSmemBytes, st, pdl);
  return cudaLaunchKernelEx(&l.cfg, tc_fwd_pipe<LY::kLev, LY::kSt, GEN>, mq, mk, mv, mo,
                            static_cast<const __nv_bfloat16*>(p.q),
                            static_cast<const __nv_bfloat16*>(p.k),
                            static_cast<const __nv_bfloat16*>(p.v), p.log_a, p.lam, p.out, p.H,
                            p.T, p.L, p.cu_seqlens, p.status, sa);
}

}  // namespace

// The pipelined kernel keeps one fp16 state per chunk level on chip: 6 levels for T <= 8192,
// 7 for T <= 16384 and 10 for T <= 131072 (walked in segments with the levels above a
// segment pre-filled).  d_k and d_v are 64 or 128: 64-column slices of q . k add up, and
// value columns are independent.  The serial cross-check takes d = 64, T <= 8192.
bool tc_supports(int in_dtype, int dk, int dv, int chunk, int T) {
  return in_dtype == LLATTN_BF16 && (dk == 64 || dk == 128) && (dv == 64 || dv == 128) &&
         chunk == kC && T <= kC * (1 << PipeXL::kLev);
}

bool tc_serial_supports(int in_dtype, int dk, int dv, int chunk, int T) {
  return in_dtype == LLATTN_BF16 && dk == kD && dv == kD && chunk == kC && T <= kC * kMaxChunks;
}

void tc_set_segment_chunks(int chunks) { g_seg_chunks_override.store(chunks); }

int tc_segment_chunks(int nseq, int H, int T, int dk, int dv, bool varlen) {
  const SegPlan pl = seg_plan(nseq, H, T, dk, dv, varlen);
  return pl.nseg > 1 ? (1 << pl.g) : 0;
}

size_t tc_workspace_bytes(int nseq, int H, int T, int dk, int dv, int chunk, bool varlen) {
  (void)chunk;
  return seg_workspace(seg_plan(nseq, H, T, dk, dv, varlen), nseq, H, dv, nullptr).bytes;
}

cudaError_t tc_forward(const Problem& p, int chunk, void* ws, cudaStream_t st, bool serial) {
  if (!(serial ? tc_serial_supports : tc_supports)(p.in_dtype, p.dk, p.dv, chunk, p.T))
    return cudaErrorNotSupported;
  // TMA only ever fetches whole chunks inside a sequence, so the token extent can be
  // the dense size, or for packed batches any bound >= the real total (nseq * T).
  const long long tokens = (long long)p.nseq * p.T;
  if (tokens >= (1ll << 31)) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv;
  cudaError_t e;
  if ((e = make_map(&mq, p.q, p.dk, p.H, tokens)) != cudaSuccess) return e;
  if ((e = make_map(&mk, p.k, p.dk, p.H, tokens)) != cudaSuccess) return e;
  if ((e = make_map(&mv, p.v, p.dv, p.H, tokens)) != cudaSuccess) return e;
  CUtensorMap mo;
  if ((e = make_out_map(&mo, p.out, p.dv, p.H, tokens)) != cudaSuccess) return e;
  // the shared-memory opt-in is a per-device attribute of each kernel
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load()) {
    if ((e = cudaFuncSetAttribute(tc_fwd_serial, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kSmemBytes)) != cudaSuccess)
      return e;
    const struct { const void* fn; int bytes; } walks[5] = {
        {(const void*)tc_fwd_pipe<PipeShort::kLev, PipeShort::kSt, false>, (int)PipeShort::kSmemBytes},
        {(const void*)tc_fwd_pipe<PipeLong::kLev, PipeLong::kSt, false>, (int)PipeLong::kSmemBytes},
        {(const void*)tc_fwd_pipe<PipeShort::kLev, PipeShort::kSt, true>, (int)PipeShort::kSmemBytes},
        {(const void*)tc_fwd_pipe<PipeLong::kLev, PipeLong::kSt, true>, (int)PipeLong::kSmemBytes},
        {(const void*)tc_fwd_pipe<PipeXL::kLev, PipeXL::kSt, true>, (int)PipeXL::kSmemBytes}};
    for (const auto& f : walks)
      if ((e = cudaFuncSetAttribute(f.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, f.bytes)) !=
          cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(tc_seg_total, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kSegSmem)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(seg_blocks, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  8 * kD * kD * (int)sizeof(float))) != cudaSuccess)
      return e;
    attr_set[dev].store(true);
  }
  main_kernel_begin(st);
  if (serial) {
    const dim3 grid(p.H, p.nseq);
    tc_fwd_serial<<<grid, kThreads, kSmemBytes, st>>>(
        mq, mk, mv, static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
        static_cast<const __nv_bfloat16*>(p.v), p.log_a, p.lam, p.out, p.H, p.T, p.L,
        p.cu_seqlens, p.status);
    main_kernel_end(st);
    count_launch();
    return cudaGetLastError();
  }
  const bool varlen = p.cu_seqlens != nullptr;
  const SegPlan pl = seg_plan(p.nseq, p.H, p.T, p.dk, p.dv, varlen);
  const SegWorkspace w = seg_workspace(pl, p.nseq, p.H, p.dv, ws);
  if (pl.nseg > 1 && ws == nullptr) return cudaErrorInvalidValue;
  const int ndv = p.dv / kD, vh = p.H * ndv;
  const int nch = (p.T + kC - 1) / kC;
  // every d_k slice of 64 columns is one pass; the later ones add into out
  for (int i = 0; i < p.dk / kD; ++i) {
    const SegArgs sa{pl.g, ndv, i * kD, p.dk, p.dv, i > 0 ? 1 : 0, w.blocks, w.block_decay,
                     pl.nblk, pl.nseg};
    // Segments: the pre-pass (totals, then the counter over segments), then the walk.  The
    // totals kernel waits for everything before it, as any launch.  Where its grid leaves SMs
    // free, the counter and the walk are dependent launches that may start while their
    // predecessor runs: the counter waits for the totals before it reads them, and only the
    // walk's later segments wait for the counter (griddepcontrol), so the first segment of
    // every sequence overlaps the pre-pass.  A pre-pass that fills the GPU gains nothing from
    // it (measured 1-2% slower), so those launch in plain stream order.
    const bool pdl = pl.nseg > 1 && (long long)vh * p.nseq * (pl.nseg - 1) < sm_count();
    if (pl.nseg > 1) {
      tc_seg_total<<<dim3(vh, p.nseq, pl.nseg - 1), kSegThreads, kSegSmem, st>>>(
          mk, mv, p.log_a, p.H, p.T, p.cu_seqlens, p.status, sa, w.seg_state, w.seg_decay);
      PdlLaunch l(dim3(vh, p.nseq), kBlkThreads, chunk_levels(pl.nseg) * kD * kD * sizeof(float),
                  st, pdl);
      if ((e = cudaLaunchKernelEx(&l.cfg, seg_blocks, p.T, p.cu_seqlens, p.status, sa,
                                  static_cast<const float*>(w.seg_state),
                                  static_cast<const float*>(w.seg_decay), w.blocks,
                                  w.block_decay)) != cudaSuccess)
        break;
      count_launch(2);
    }
    const dim3 grid(vh, p.nseq, pl.nseg);
    const bool gen = pl.nseg > 1 || p.dk != kD || p.dv != kD;
    if (nch <= (1 << PipeShort::kLev)) {      // 6 levels on chip, three-stage ring
      e = gen ? launch_walk<PipeShort, true>(grid, st, mq, mk, mv, mo, p, sa, pdl)
              : launch_walk<PipeShort, false>(grid, st, mq, mk, mv, mo, p, sa, pdl);
    } else if (nch <= (1 << PipeLong::kLev)) {   // 7 levels, two stages (shared memory)
      e = gen ? launch_walk<PipeLong, true>(grid, st, mq, mk, mv, mo, p, sa, pdl)
              : launch_walk<PipeLong, false>(grid, st, mq, mk, mv, mo, p, sa, pdl);
    } else {                                  // 10 levels, two stages, always in segments
      e = launch_walk<PipeXL, true>(grid, st, mq, mk, mv, mo, p, sa, pdl);
    }
    count_launch();
    if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) break;
  }
  main_kernel_end(st);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace llattn
