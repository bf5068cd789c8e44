// Backward pass on the tensor cores (bf16 inputs, d = 64): the pairs inside each aligned chunk
// of 128 tokens (levels 0..7), then one launch per level >= 8.
//
// Log-Linear Attention (gist.science summaries, Italian "Sommario tecnico" section 2, "Matrici
// Gerarchiche"): at level l the positions fall into aligned blocks of 2^l tokens, and every key
// s in a block's left half meets every query t in its right half with weight
// lam[t, l] exp(g_t - g_s).  With m the last position of the left half the interaction has
// rank d, and the block needs only
//
//   S = sum over left-half s of exp(g_m - g_s) k_s v_s^T             (d x d)
//   U = sum over right-half t of lam[t, l] exp(g_t - g_m) q_t do_t^T  (d x d)
//
// for   w_t = exp(g_t - g_m) S do_t,  dlam[t, l] = q_t . w_t,  dq_t += lam[t, l] w_t,
//       dk_s += exp(g_m - g_s) U v_s,  dv_s += exp(g_m - g_s) U^T k_s   (dlam = 0 on the left).
//
// Levels >= 8: one CTA takes one block and walks it twice in tiles of 128 tokens.  Pass 1 reduces S and U
// over the tiles on the tensor cores (K^T V and Q^T dO shapes, M = 64, the token index as the
// reduction dimension) into TMEM.  Pass 2 multiplies every tile by them: W = dO S^T,
// DK = V U^T, DV = K U (M = 128 rows per tile), and the epilogue applies the exponential
// factors, forms dlam and adds into dq, dk, dv: a whole tile's contributions are staged in
// shared memory and added by TMA reduce-adds (the add happens in L2, no gradient row is read
// into the SM); a tile that runs past the sequence end adds its rows by plain
// read-modify-writes.  A level whose blocks fill at most half the CTA slots (two per SM) runs
// two CTAs per block: the key side reduces U and adds into the left half's dk, dv, the query
// side reduces S and adds into the right half's dq, dlam.
//
// Precision: q, k, v and dO enter as the bf16 values they are.  The operands the method derives
// (the decay-scaled rows of K and Q, and S, U) are split into a bf16 high part and a bf16
// remainder, x = hi + lo with |lo| <= 2^-8 |x|, and each product takes both parts (two MMAs into
// the same fp32 accumulator): about 16 significant bits per operand, so the gradients stay at
// fp32-accumulation accuracy.  Factors: exp(g_m - g_s) <= 1 on the left half; on the right,
// exp(g_t - g_m) <= 1 times lam.
//
// Loads: whole tiles inside the sequence by TMA (128-byte swizzle, the layout the MMA
// descriptors read); a tile that runs past the sequence end by plain loads with zero fill, so
// no load ever leaves the tensors.  Waits are bounded (mbarrier with a time limit; a timeout
// sets LLATTN_DEV_WAIT_TIMEOUT and the CTA stops issuing work).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <type_traits>

#include "../../include/llattn.h"
#include "llattn_bwd.h"
#include "llattn_common.cuh"
#include "llattn_internal.h"
#include "llattn_tc_ptx.cuh"

namespace llattn {
namespace {

using namespace ptx;

constexpr int kC = 128;          // tile rows (tokens)
constexpr int kD = 64;           // d_k = d_v
constexpr int kThreads = 256;    // warp w: TMEM lanes 32*(w%4).., column half w/4

// ---- shared memory (bytes from a 1024-byte aligned base) ----
constexpr uint32_t kTileB = kC * 128;            // 128 rows x 128 B, 128-byte swizzle
constexpr uint32_t kOffQ = 0, kOffK = kTileB, kOffV = 2 * kTileB, kOffDO = 3 * kTileB;

// Level kernel: a tile lies in one half of its block (half >= 128 tokens), so it needs two
// inputs: X = K, Y = V on the left, X = Q, Y = dO on the right.  In pass 2 a whole tile's
// gradient contributions are staged in the tiles the MMAs are done with (plus E) and added to
// dq, dk, dv by TMA reduce-adds.  About 98 KB and 128 TMEM columns, so two CTAs share an SM
// and overlap their tile chains.
constexpr uint32_t kState = kD * 128;            // 64 rows x 128 B
constexpr uint32_t kLOffX = 0, kLOffY = kTileB, kLOffXlo = 2 * kTileB, kLOffE = 3 * kTileB;
constexpr uint32_t kLOffShi = 4 * kTileB, kLOffSlo = kLOffShi + kState;
constexpr uint32_t kLOffUhi = kLOffSlo + kState, kLOffUlo = kLOffUhi + kState;
constexpr uint32_t kLOffDl = kLOffUlo + kState;  // dlam partials of column half 1: [128] fp32
constexpr uint32_t kLOffBar = kLOffDl + kC * 4;  // [0] loads, [1] MMAs
constexpr uint32_t kLOffMisc = kLOffBar + 16;    // [0] TMEM base, [1] abort
constexpr uint32_t kSmemBytes = kLOffMisc + 16 + 1024;
static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two level CTAs per SM");

// ---- TMEM columns of the level kernel (128 allocated) ----
constexpr uint32_t kColS = 0, kColU = 64;        // pass 1: M = 64 accumulators
constexpr uint32_t kColW = 0;                    // pass 2, right tiles: M = 128
constexpr uint32_t kColDK = 0, kColDV = 64;      // pass 2, left tiles: M = 128

constexpr uint32_t kIdescRed = idesc_bf16(64, 64, 1, 1);     // X^T (M contiguous) x Y (N contiguous)
constexpr uint32_t kIdescKK = idesc_bf16(128, 64, 0, 0);     // rows (K-major) x state rows (K-major)
constexpr uint32_t kIdescKN = idesc_bf16(128, 64, 0, 1);     // rows (K-major) x state (N contiguous)

__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t saddr) { return sdesc_sw128(saddr, 8192, 1024); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);  // a -> low 16 bits
  return *reinterpret_cast<uint32_t*>(&v);
}

// x = hi + lo: hi = bf16(x) (round to nearest), lo = bf16(x - hi); pairs (a, b), a in the low
// 16 bits of each word.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16(a - hf.x, b - hf.y);
}

__device__ __forceinline__ float2 bf2_at(const uint8_t* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}


__global__ void __launch_bounds__(kThreads, 2)
bwd_level_tc(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
             const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
             const __grid_constant__ CUtensorMap tdq, const __grid_constant__ CUtensorMap tdk,
             const __grid_constant__ CUtensorMap tdv, const BwdProblem p,
             const double* __restrict__ g, int lvl, int split) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = warp & 3, hf = warp >> 2, row = sub * 32 + lane;
  const uint32_t lane_off = uint32_t(sub * 32) << 16;
  // split != 0: two CTAs per block, blockIdx.x = 2 * block + side.  The key side (0) reduces U
  // over the right half and adds into dk, dv of the left; the query side (1) reduces S over the
  // left half and adds into dq, dlam of the right.  Otherwise one CTA does both.
  const int blk = split ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int side = split ? (int)(blockIdx.x & 1) : -1;
  const int h = blockIdx.y, sq = blockIdx.z;
  const SeqSpan sp = seq_span(sq, p.T, p.cu_seqlens, p.status);
  const int half = 1 << (lvl - 1);               // a multiple of 128 (lvl >= 8)
  const long long a0 = (long long)blk << lvl;
  if (a0 >= sp.len) return;
  const int lo = (int)a0, mid = lo + half;
  const int lend = min(mid, sp.len);                                          // left [lo, lend)
  const int rend = (int)min((long long)lo + 2 * half, (long long)sp.len);    // right [mid, rend)
  auto row_of = [&](int t) { return (size_t)(sp.start + t) * p.H + h; };
  auto grow = [&](int t) { return ((size_t)sq * p.T + t) * p.H + h; };
  if (side <= 0)
    for (int t = lo + tid; t < lend; t += kThreads) p.dlam[row_of(t) * p.L + lvl] = 0.f;
  if (mid >= sp.len) return;   // no right half: nothing meets at this level

  uint8_t* tx = sm + kLOffX;
  uint8_t* ty = sm + kLOffY;
  uint8_t* txlo = sm + kLOffXlo;
  uint8_t* te = sm + kLOffE;
  uint8_t* shi = sm + kLOffShi;
  uint8_t* slo = sm + kLOffSlo;
  uint8_t* uhi = sm + kLOffUhi;
  uint8_t* ulo = sm + kLOffUlo;
  float* s_dl = reinterpret_cast<float*>(sm + kLOffDl);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kLOffBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + kLOffMisc);

  if (warp == 0) {
    tmem_alloc(&misc[0], 128);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    misc[1] = 0;
    prefetch_tensormap(&tmq);
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    prefetch_tensormap(&tmo);
    prefetch_tensormap(&tdq);
    prefetch_tensormap(&tdk);
    prefetch_tensormap(&tdv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const double gm = g[grow(mid - 1)];
  uint32_t ph_ld = 0u, ph_mma = 0u;
  int stuck = -1;               // barrier whose wait timed out (its parity in stuck_par)
  uint32_t stuck_par = 0u;
  auto bwait = [&](int b, uint32_t& ph) {
    if (!mbar_wait(&bars[b], ph)) {
      atomicOr(p.status, LLATTN_DEV_WAIT_TIMEOUT);
      misc[1] = 1;
      if (stuck < 0) {
        stuck = b;
        stuck_par = ph;
      }
    }
    ph ^= 1u;
  };

  // The tile of 128 tokens from t0: X, Y = K, V (left) or Q, dO (right).  A whole tile inside
  // the sequence comes by TMA (returns true: wait on bars[0]); a tile running past the sequence
  // end by plain loads of its rows, the rest zero.
  auto load = [&](int t0, bool left) {
    if (t0 + kC <= sp.len) {
      if (tid == 0) {
        mbar_arrive_expect_tx(&bars[0], 2 * kTileB);
        const int z = (int)(sp.start + t0);
        tma_load_3d(tx, left ? &tmk : &tmq, &bars[0], 0, h, z);
        tma_load_3d(ty, left ? &tmv : &tmo, &bars[0], 0, h, z);
      }
      return true;
    }
    const int n = sp.len - t0;
    const __nv_bfloat16* sx = static_cast<const __nv_bfloat16*>(left ? p.k : p.q);
    const __nv_bfloat16* sy = static_cast<const __nv_bfloat16*>(left ? p.v : p.dout);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int col = 32 * hf + 8 * jj;
      uint4 vx = make_uint4(0u, 0u, 0u, 0u), vy = vx;
      if (row < n) {
        vx = *reinterpret_cast<const uint4*>(sx + row_of(t0 + row) * kD + col);
        vy = *reinterpret_cast<const uint4*>(sy + row_of(t0 + row) * kD + col);
      }
      *reinterpret_cast<uint4*>(tx + sw128_off(row, col)) = vx;
      *reinterpret_cast<uint4*>(ty + sw128_off(row, col)) = vy;
    }
    fence_proxy_async_smem();
    return false;
  };

  const uint32_t xa = smem_u32(tx), ya = smem_u32(ty), xla = smem_u32(txlo);
  const uint32_t sha = smem_u32(shi), sla = smem_u32(slo), uha = smem_u32(uhi), ula = smem_u32(ulo);
  const int nt = (rend - lo + kC - 1) / kC;
  const int nl = (lend - lo + kC - 1) / kC;   // tiles [0, nl) are left, [nl, nt) right
  // the tiles each pass walks: both halves, or for a split block the other side's half in
  // pass 1 and this side's half in pass 2
  const int p1b = side == 0 ? nl : 0, p1e = side == 1 ? nl : nt;
  const int p2b = side == 1 ? nl : 0, p2e = side == 0 ? nl : nt;

  // ---- pass 1: S = sum exp(g_m - g_s) k_s v_s^T (left), U = sum lam exp(g_t - g_m) q_t do_t^T ----
  bool s_started = false, u_started = false;
  // this row's prefix sum (and lam on the right) of tile j, read one tile ahead
  auto row_in = [&](int j, double& gt, float& lt) {
    const int t = lo + j * kC + row;
    const bool left = lo + j * kC < mid;
    gt = 0.0;
    lt = 0.f;
    if (j < nt && t < (left ? lend : rend)) {
      gt = g[grow(t)];
      if (!left) lt = p.lam[row_of(t) * p.L + lvl];
    }
  };
  double g_next;
  float l_next;
  row_in(p1b, g_next, l_next);
  for (int j = p1b; j < p1e; ++j) {
    if (misc[1] != 0) break;
    const int t0 = lo + j * kC;
    const bool left = t0 < mid;
    const bool tma = load(t0, left);
    const int t = t0 + row;
    const double gt = g_next;
    const float lt = l_next;
    row_in(j + 1, g_next, l_next);
    float f = 0.f;
    if (left) {
      if (t < lend) f = expf((float)(gm - gt));
    } else if (t < rend) {
      f = lt * expf((float)(gt - gm));
    }
    if (tma) bwait(0, ph_ld);
    // X rows times f, split: hi in place, remainder in Xlo
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const uint32_t off = sw128_off(row, 32 * hf + 8 * jj);
      const uint4 raw = *reinterpret_cast<const uint4*>(tx + off);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      uint32_t hi[4], lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        split2(x.x * f, x.y * f, hi[e], lw[e]);
      }
      *reinterpret_cast<uint4*>(tx + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(txlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      if (misc[1] == 0) {
        const uint32_t d = tmem + (left ? kColS : kColU);
        const bool started = left ? s_started : u_started;
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          mma_ss(d, mndesc(xa + kk * 2048), mndesc(ya + kk * 2048), kIdescRed,
                 (started || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          mma_ss(d, mndesc(xla + kk * 2048), mndesc(ya + kk * 2048), kIdescRed, 1u);
      }
      mma_commit(&bars[1]);
    }
    s_started = s_started || left;
    u_started = u_started || !left;
    bwait(1, ph_mma);   // the tiles may be overwritten once the MMAs have read them
    tc_fence_after();
  }

  // ---- S and U to shared memory, hi / lo (M = 64 accumulators: row i = 16 sub + lane) ----
  if (misc[1] == 0) {
    auto store_state = [&](uint8_t* dhi, uint8_t* dlo, const float (&x)[32]) {
      const int i = 16 * sub + lane;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t hi[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split2(x[8 * jj + 2 * e], x[8 * jj + 2 * e + 1], hi[e], lw[e]);
        const uint32_t off = sw128_off(i, 32 * hf + 8 * jj);
        *reinterpret_cast<uint4*>(dhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(dlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    };
    float x[32];
    tmem_ld32(tmem + lane_off + kColS + 32 * hf, x);
    tmem_wait_ld();
    if (lane < 16) store_state(shi, slo, x);
    tmem_ld32(tmem + lane_off + kColU + 32 * hf, x);
    tmem_wait_ld();
    if (lane < 16) store_state(uhi, ulo, x);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();

  // ---- pass 2: W = dO S^T (right tiles), DK = V U^T and DV = K U (left tiles) ----
  // A whole tile's contributions go through shared memory to TMA reduce-adds (dq from Y and
  // Xlo; dk from Y and Xlo, dv from X and E, one buffer per 32-column half): no gradient row is
  // read into the SM, and the add happens in L2.  A tile running past the sequence end adds
  // its rows by plain read-modify-writes instead.
  // this row's prefix sum (and lam on the right) of pass-2 tile j, read one tile ahead
  auto row2_in = [&](int j, double& gt, float& lt) {
    const int t = lo + j * kC + row;
    const bool left = lo + j * kC < mid;
    gt = gm;
    lt = 0.f;
    if (j < p2e && t < (left ? lend : rend)) {
      gt = g[grow(t)];
      if (!left) lt = p.lam[row_of(t) * p.L + lvl];
    }
  };
  double g2_next;
  float l2_next;
  row2_in(p2b, g2_next, l2_next);
  for (int j = p2b; j < p2e; ++j) {
    if (misc[1] != 0) break;
    const int t0 = lo + j * kC;
    const bool left = t0 < mid;
    const bool whole = t0 + kC <= sp.len;
    // the previous tile's reduce-adds must have read their staging before X, Y are reloaded
    if (tid == 0) bulk_wait_read();
    if (!whole) __syncthreads();   // plain loads by every thread: after that wait
    const bool tma = load(t0, left);
    if (tma) bwait(0, ph_ld);
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      if (misc[1] == 0) {
        if (!left) {
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(tmem + kColW, kdesc(ya + kk * 32), kdesc(sha + kk * 32), kIdescKK, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(tmem + kColW, kdesc(ya + kk * 32), kdesc(sla + kk * 32), kIdescKK, 1u);
        } else {
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(tmem + kColDK, kdesc(ya + kk * 32), kdesc(uha + kk * 32), kIdescKK, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(tmem + kColDK, kdesc(ya + kk * 32), kdesc(ula + kk * 32), kIdescKK, 1u);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(tmem + kColDV, kdesc(xa + kk * 32), mndesc(uha + kk * 2048), kIdescKN, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss(tmem + kColDV, kdesc(xa + kk * 32), mndesc(ula + kk * 2048), kIdescKN, 1u);
        }
      }
      mma_commit(&bars[1]);
    }
    const int t = t0 + row;
    const bool right_row = !left && t < rend;
    const bool left_row = left && t < lend;
    const size_t r = (right_row || left_row) ? row_of(t) : 0;
    const double gt = g2_next;
    const float lam = l2_next;
    row2_in(j + 1, g2_next, l2_next);
    bwait(1, ph_mma);
    tc_fence_after();
    const bool ok = misc[1] == 0;
    float dlp = 0.f;
    if (whole) {
      // staging of this thread's 32 columns of its row (128-byte swizzle, the reduce map's box)
      auto stage = [&](uint8_t* dst, const float (&c)[32]) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + sw128_off(row, 2 * e)) =
              make_float4(c[e], c[e + 1], c[e + 2], c[e + 3]);
      };
      float w[32];
      if (!left) {
        tmem_ld32(tmem + lane_off + kColW + 32 * hf, w);
        tmem_wait_ld();
        const float sc = expf((float)(gt - gm));
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float2 q01 = bf2_at(tx + sw128_off(row, 32 * hf + e));
          const float2 q23 = bf2_at(tx + sw128_off(row, 32 * hf + e + 2));
          const float w0 = sc * w[e], w1 = sc * w[e + 1], w2 = sc * w[e + 2], w3 = sc * w[e + 3];
          dlp = fmaf(q01.x, w0, fmaf(q01.y, w1, fmaf(q23.x, w2, fmaf(q23.y, w3, dlp))));
          w[e] = lam * w0;
          w[e + 1] = lam * w1;
          w[e + 2] = lam * w2;
          w[e + 3] = lam * w3;
        }
        stage(hf ? txlo : ty, w);
      } else {
        const float f = expf((float)(gm - gt));
        tmem_ld32(tmem + lane_off + kColDK + 32 * hf, w);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] *= f;
        stage(hf ? txlo : ty, w);
        tmem_ld32(tmem + lane_off + kColDV + 32 * hf, w);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] *= f;
        stage(hf ? te : tx, w);
      }
      fence_proxy_async_smem();
    } else if (!left) {
      float w[32];
      tmem_ld32(tmem + lane_off + kColW + 32 * hf, w);
      tmem_wait_ld();
      if (right_row && ok) {
        float* dst = p.dq + r * kD + 32 * hf;
        const float sc = expf((float)(gt - gm));
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float2 q01 = bf2_at(tx + sw128_off(row, 32 * hf + e));
          const float2 q23 = bf2_at(tx + sw128_off(row, 32 * hf + e + 2));
          const float w0 = sc * w[e], w1 = sc * w[e + 1], w2 = sc * w[e + 2], w3 = sc * w[e + 3];
          dlp = fmaf(q01.x, w0, fmaf(q01.y, w1, fmaf(q23.x, w2, fmaf(q23.y, w3, dlp))));
          float4 a = *reinterpret_cast<const float4*>(dst + e);
          a.x = fmaf(lam, w0, a.x);
          a.y = fmaf(lam, w1, a.y);
          a.z = fmaf(lam, w2, a.z);
          a.w = fmaf(lam, w3, a.w);
          *reinterpret_cast<float4*>(dst + e) = a;
        }
      }
    } else {
      const bool own = left_row && ok;
      const float f = own ? expf((float)(gm - gt)) : 0.f;
      float v[32];
      tmem_ld32(tmem + lane_off + kColDK + 32 * hf, v);
      tmem_wait_ld();
      if (own) {
        float* dk = p.dk + r * kD + 32 * hf;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 a = *reinterpret_cast<float4*>(dk + e);
          a.x = fmaf(f, v[e], a.x);
          a.y = fmaf(f, v[e + 1], a.y);
          a.z = fmaf(f, v[e + 2], a.z);
          a.w = fmaf(f, v[e + 3], a.w);
          *reinterpret_cast<float4*>(dk + e) = a;
        }
      }
      tmem_ld32(tmem + lane_off + kColDV + 32 * hf, v);
      tmem_wait_ld();
      if (own) {
        float* dv = p.dv + r * kD + 32 * hf;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 a = *reinterpret_cast<float4*>(dv + e);
          a.x = fmaf(f, v[e], a.x);
          a.y = fmaf(f, v[e + 1], a.y);
          a.z = fmaf(f, v[e + 2], a.z);
          a.w = fmaf(f, v[e + 3], a.w);
          *reinterpret_cast<float4*>(dv + e) = a;
        }
      }
    }
    if (!left && hf == 1) s_dl[row] = dlp;
    tc_fence_before();
    __syncthreads();   // TMEM drained, the staging written, s_dl filled
    if (!left && hf == 0 && right_row && ok) p.dlam[r * p.L + lvl] = dlp + s_dl[row];
    if (whole && tid == 0 && misc[1] == 0) {
      const int z = (int)(sp.start + t0);
      if (!left) {
        tma_reduce_add_3d(&tdq, ty, 0, h, z);
        tma_reduce_add_3d(&tdq, txlo, 32, h, z);
      } else {
        tma_reduce_add_3d(&tdk, ty, 0, h, z);
        tma_reduce_add_3d(&tdk, txlo, 32, h, z);
        tma_reduce_add_3d(&tdv, tx, 0, h, z);
        tma_reduce_add_3d(&tdv, te, 32, h, z);
      }
      bulk_commit();
    }
  }

  // a copy or MMA batch whose wait timed out must land before the CTA exits
  if (stuck >= 0 && tid == 0) mbar_wait(&bars[stuck], stuck_par, 100000000ull);
  if (tid == 0) bulk_wait_all();   // the reduce-adds have read their staging and landed
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---- levels 0..7: the pairs inside one aligned chunk of 128 tokens ----
//
// With A = Q K^T, B = dO V^T and the chunk's mask M[t, s] = lam[t, l(t, s)] exp(g_t - g_s) for
// s <= t (l <= 7 inside an aligned chunk):
//   dQ = (M .* B) K,  dK = (M .* B)^T Q,  dV = (M .* A)^T dO,
//   dlam[t, l] = sum over s with l(t, s) = l of exp(g_t - g_s) A[t, s] B[t, s].
// One CTA per chunk: A and B on the tensor cores into TMEM, the masked products P1 = M .* B and
// P2 = M .* A to shared memory (bf16 hi / lo, each as two 64-column halves in the 128-byte
// swizzle), then the three products, which give this chunk's share of dq, dk and dv: the first
// write of every gradient row (the levels >= 8 add to it).
constexpr uint32_t kHalfB = kC * 128;                 // [128 rows][64 cols] bf16
constexpr uint32_t kMatB = 2 * kHalfB;                // two halves: columns 0..63, 64..127
constexpr uint32_t kIOffP1h = 4 * kTileB, kIOffP1l = kIOffP1h + kMatB;
constexpr uint32_t kIOffP2h = kIOffP1l + kMatB, kIOffP2l = kIOffP2h + kMatB;
constexpr uint32_t kIOffG = kIOffP2l + kMatB;         // g of the chunk's rows: [128] fp64
constexpr uint32_t kIOffLam = kIOffG + kC * 8;        // lam[t, 0..7]: [128][9] fp32 (odd stride)
constexpr uint32_t kIOffDl = kIOffLam + kC * 9 * 4;   // dlam partials of column half 1: [128][8]
constexpr uint32_t kIOffCj = kIOffDl + kC * 8 * 4;   // exp(g_0 - g_s) of the chunk's keys: [128]
constexpr uint32_t kIOffBar = kIOffCj + kC * 4;
constexpr uint32_t kIOffMisc = kIOffBar + 16;
constexpr uint32_t kISmemBytes = kIOffMisc + 16 + 1024;
static_assert(kISmemBytes <= 227 * 1024, "shared memory");

constexpr uint32_t kIColA = 0, kIColB = 128, kIColDQ = 256, kIColDK = 320, kIColDV = 384;
constexpr uint32_t kIdescAB = idesc_bf16(128, 128, 0, 0);   // rows x rows^T (both K-major)
constexpr uint32_t kIdescTN = idesc_bf16(128, 64, 1, 1);    // P^T (M contiguous) x rows (N contiguous)

// MN-major operand of M = 128 stored as two 64-element groups 16 KB apart (the halves).
__device__ __forceinline__ uint64_t mndesc2(uint32_t saddr) { return sdesc_sw128(saddr, kHalfB, 1024); }

__global__ void __launch_bounds__(kThreads, 1)
bwd_intra_tc(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
             const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
             const __grid_constant__ CUtensorMap tdq, const __grid_constant__ CUtensorMap tdk,
             const __grid_constant__ CUtensorMap tdv, const BwdProblem p,
             const double* __restrict__ g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = warp & 3, hf = warp >> 2, row = sub * 32 + lane;
  const uint32_t lane_off = uint32_t(sub * 32) << 16;
  const int ch = blockIdx.x, h = blockIdx.y, sq = blockIdx.z;
  const SeqSpan sp = seq_span(sq, p.T, p.cu_seqlens, p.status);
  const int t0 = ch * kC;
  if (t0 >= sp.len) return;
  const int n = min(kC, sp.len - t0);
  auto row_of = [&](int t) { return (size_t)(sp.start + t) * p.H + h; };

  uint8_t* tq = sm + kOffQ;
  uint8_t* tk = sm + kOffK;
  uint8_t* tv = sm + kOffV;
  uint8_t* tdo = sm + kOffDO;
  uint8_t* p1h = sm + kIOffP1h;
  uint8_t* p1l = sm + kIOffP1l;
  uint8_t* p2h = sm + kIOffP2h;
  uint8_t* p2l = sm + kIOffP2l;
  double* s_g = reinterpret_cast<double*>(sm + kIOffG);
  float* s_lam = reinterpret_cast<float*>(sm + kIOffLam);
  float* s_dl = reinterpret_cast<float*>(sm + kIOffDl);
  float* s_cj = reinterpret_cast<float*>(sm + kIOffCj);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kIOffBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + kIOffMisc);

  if (warp == 0) {
    tmem_alloc(&misc[0], 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    misc[1] = 0;
  }
  // the chunk's tiles: TMA when the whole chunk lies inside the sequence, else plain loads
  const bool tma = n == kC;
  if (tma) {
    if (tid == 32) {
      mbar_arrive_expect_tx(&bars[0], 4 * kTileB);
      const int z = (int)(sp.start + t0);
      tma_load_3d(tq, &tmq, &bars[0], 0, h, z);
      tma_load_3d(tk, &tmk, &bars[0], 0, h, z);
      tma_load_3d(tv, &tmv, &bars[0], 0, h, z);
      tma_load_3d(tdo, &tmo, &bars[0], 0, h, z);
    }
  } else {
    const struct { const void* src; uint8_t* dst; } ts[4] = {
        {p.q, tq}, {p.k, tk}, {p.v, tv}, {p.dout, tdo}};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(ts[x].src);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int col = 32 * hf + 8 * jj;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (row < n) val = *reinterpret_cast<const uint4*>(src + row_of(t0 + row) * kD + col);
        *reinterpret_cast<uint4*>(ts[x].dst + sw128_off(row, col)) = val;
      }
    }
    fence_proxy_async_smem();
  }
  // row scalars while the tiles fly
  if (hf == 0) s_g[row] = row < n ? g[((size_t)sq * p.T + t0 + row) * p.H + h] : 0.0;
  else {
#pragma unroll
    for (int l = 0; l < 8; ++l)
      s_lam[row * 9 + l] = (row < n && l < p.L) ? p.lam[row_of(t0 + row) * p.L + l] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Decay of a pair: exp(g_t - g_s) = exp(g_t - g_0) exp(g_0 - g_s) when the chunk's decay
  // range is at most 80, where both factors are normal fp32 numbers (one product per pair, the
  // key factors tabled once); a chunk of stronger decay takes exp(g_t - g_s) pair by pair.
  const double g0 = s_g[0];
  const bool factored = g0 - s_g[n - 1] <= 80.0;
  if (hf == 1) s_cj[row] = (factored && row < n) ? expf((float)(g0 - s_g[row])) : 0.f;
  const uint32_t tmem = misc[0];
  uint32_t ph_mma = 0u;
  int stuck = -1;
  uint32_t stuck_par = 0u;
  auto bwait = [&](int b, uint32_t ph) {
    if (!mbar_wait(&bars[b], ph)) {
      atomicOr(p.status, LLATTN_DEV_WAIT_TIMEOUT);
      misc[1] = 1;
      if (stuck < 0) {
        stuck = b;
        stuck_par = ph;
      }
    }
  };
  if (tma) bwait(0, 0u);
  const uint32_t qa = smem_u32(tq), ka = smem_u32(tk), va = smem_u32(tv), da = smem_u32(tdo);

  // ---- A = Q K^T, B = dO V^T ----
  if (tid == 0) {
    tc_fence_after();
    if (misc[1] == 0) {
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk)
        mma_ss(tmem + kIColA, kdesc(qa + kk * 32), kdesc(ka + kk * 32), kIdescAB, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk)
        mma_ss(tmem + kIColB, kdesc(da + kk * 32), kdesc(va + kk * 32), kIdescAB, kk > 0 ? 1u : 0u);
    }
    mma_commit(&bars[1]);
  }
  bwait(1, ph_mma);
  ph_mma ^= 1u;
  tc_fence_after();

  // ---- masks: P1 = M .* B, P2 = M .* A (hi / lo), and dlam's level sums ----
  __syncthreads();   // the key factors are in place
  {
    const int t = row;
    const double gt = s_g[t];
    const float* lr = s_lam + t * 9;
    float dl[8];
#pragma unroll
    for (int l = 0; l < 8; ++l) dl[l] = 0.f;
    const uint32_t hoff = hf * kHalfB;   // this thread's columns are half hf of each matrix
    const float rsc = (factored && t < n) ? expf((float)(gt - g0)) : 0.f;
    auto masks = [&](auto fac) {
    constexpr bool kFac = decltype(fac)::value;
    // decay of the pair (t, s)
    auto decay = [&](int s) { return kFac ? rsc * s_cj[s] : expf((float)(gt - s_g[s])); };
#pragma unroll 1
    for (int c16 = 0; c16 < 4; ++c16) {
      const int s0 = 64 * hf + 16 * c16;
      float p1[16], p2[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) p1[e] = p2[e] = 0.f;
      if (s0 <= 32 * sub + 31) {   // warp-uniform: some row of this warp reaches these keys
        float av[16], bv[16];
        tmem_ld16(tmem + lane_off + kIColA + s0, av);
        tmem_ld16(tmem + lane_off + kIColB + s0, bv);
        tmem_wait_ld();
        if (t < n && s0 <= t) {
          if ((t >> 4) != (s0 >> 4)) {
            // every key of the group is earlier, at one level: 1 + msb(t ^ s), fixed by bits >= 4
            const int lev = 32 - __clz(t ^ s0);
            const float lam = lr[lev];
            float xs = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float E = decay(s0 + e);
              const float m = lam * E;
              p1[e] = m * bv[e];
              p2[e] = m * av[e];
              xs = fmaf(E * av[e], bv[e], xs);
            }
#pragma unroll
            for (int l = 0; l < 8; ++l) dl[l] += l == lev ? xs : 0.f;
          } else {
            // the row's own 16-key block: levels 0..4 element by element, keys s <= t only
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int s = s0 + e;
              if (s <= t) {
                const float E = decay(s);
                const int lev = 32 - __clz(t ^ s);   // 0 when s == t
                const float m = lr[lev] * E;
                p1[e] = m * bv[e];
                p2[e] = m * av[e];
                const float xe = E * av[e] * bv[e];
#pragma unroll
                for (int l = 0; l < 5; ++l) dl[l] += l == lev ? xe : 0.f;
              }
            }
          }
        }
      }
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        uint32_t h1[4], l1[4], h2[4], l2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          split2(p1[8 * hq + 2 * e], p1[8 * hq + 2 * e + 1], h1[e], l1[e]);
          split2(p2[8 * hq + 2 * e], p2[8 * hq + 2 * e + 1], h2[e], l2[e]);
        }
        const uint32_t off = hoff + sw128_off(t, 16 * c16 + 8 * hq);
        *reinterpret_cast<uint4*>(p1h + off) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
        *reinterpret_cast<uint4*>(p1l + off) = make_uint4(l1[0], l1[1], l1[2], l1[3]);
        *reinterpret_cast<uint4*>(p2h + off) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
        *reinterpret_cast<uint4*>(p2l + off) = make_uint4(l2[0], l2[1], l2[2], l2[3]);
      }
    }
    };
    if (factored) masks(std::true_type{});
    else masks(std::false_type{});
    if (hf == 1) {
#pragma unroll
      for (int l = 0; l < 8; ++l) s_dl[t * 8 + l] = dl[l];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (hf == 0 && t < n) {
      float* dst = p.dlam + row_of(t0 + t) * p.L;
#pragma unroll
      for (int l = 0; l < 8; ++l)
        if (l < p.L) dst[l] = dl[l] + s_dl[t * 8 + l];
    }
  }

  // ---- dQ = P1 K, dK = P1^T Q, dV = P2^T dO (hi and lo parts) ----
  if (tid == 0) {
    tc_fence_after();
    if (misc[1] == 0) {
      const uint32_t a1h = smem_u32(p1h), a1l = smem_u32(p1l), a2h = smem_u32(p2h), a2l = smem_u32(p2l);
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk) {
        const uint32_t ko = (kk >> 2) * kHalfB + (kk & 3) * 32;   // K-major: half, then 16 keys
        mma_ss(tmem + kIColDQ, kdesc(a1h + ko), mndesc(ka + kk * 2048), kIdescKN, kk > 0 ? 1u : 0u);
        mma_ss(tmem + kIColDQ, kdesc(a1l + ko), mndesc(ka + kk * 2048), kIdescKN, 1u);
      }
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk) {
        mma_ss(tmem + kIColDK, mndesc2(a1h + kk * 2048), mndesc(qa + kk * 2048), kIdescTN, kk > 0 ? 1u : 0u);
        mma_ss(tmem + kIColDK, mndesc2(a1l + kk * 2048), mndesc(qa + kk * 2048), kIdescTN, 1u);
        mma_ss(tmem + kIColDV, mndesc2(a2h + kk * 2048), mndesc(da + kk * 2048), kIdescTN, kk > 0 ? 1u : 0u);
        mma_ss(tmem + kIColDV, mndesc2(a2l + kk * 2048), mndesc(da + kk * 2048), kIdescTN, 1u);
      }
    }
    mma_commit(&bars[1]);
  }
  bwait(1, ph_mma);
  ph_mma ^= 1u;
  tc_fence_after();
  // A whole chunk's dq, dk, dv go through the spent P tiles (one 16 KB half per 32 columns, in
  // the 128-byte swizzle of the store map's box) to TMA tile stores: whole 128-byte rows, where
  // per-thread row stores would touch 32 lines per warp instruction.  A ragged last chunk
  // stores its rows with plain stores (a whole box would reach the next sequence's rows).
  {
    const bool ok = row < n && misc[1] == 0;
    const size_t r = ok ? row_of(t0 + row) * kD + 32 * hf : 0;
    const struct { uint32_t col; float* dst; uint8_t* stage; const CUtensorMap* map; } outs[3] = {
        {kIColDQ, p.dq, p1h, &tdq}, {kIColDK, p.dk, p1l, &tdk}, {kIColDV, p.dv, p2h, &tdv}};
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      float v[32];
      tmem_ld32(tmem + lane_off + outs[x].col + 32 * hf, v);
      tmem_wait_ld();
      if (tma) {
        uint8_t* dst = outs[x].stage + hf * kHalfB;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + sw128_off(row, 2 * e)) =
              make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      } else if (ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(outs[x].dst + r + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
    }
    if (tma) {
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0 && misc[1] == 0) {
        const int z = (int)(sp.start + t0);
#pragma unroll
        for (int x = 0; x < 3; ++x) {
          tma_store_3d(outs[x].map, outs[x].stage, 0, h, z);
          tma_store_3d(outs[x].map, outs[x].stage + kHalfB, 32, h, z);
        }
        bulk_commit();
        bulk_wait_all();   // the stores have read the staging and landed before the CTA exits
      }
    }
  }
  if (stuck >= 0 && tid == 0) mbar_wait(&bars[stuck], stuck_par, 100000000ull);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr int kSplitDen = 2;   // split a level whose blocks fill at most 1 / kSplitDen of the slots

int sm_count_bwd() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

}  // namespace

bool bwd_tc_supports(const BwdProblem& p) {
  return p.in_dtype == LLATTN_BF16 && p.d == kD && (long long)p.nseq * p.T < (1ll << 31);
}

cudaError_t bwd_levels_tc(const BwdProblem& p, const double* g, cudaStream_t st) {
  if (!bwd_tc_supports(p)) return cudaErrorNotSupported;
  // TMA only fetches whole tiles inside a sequence, so for a packed batch any token extent
  // >= the real total serves (nseq * T bounds it)
  const long long tokens = (long long)p.nseq * p.T;
  CUtensorMap mq, mk, mv, mo, mdq, mdk, mdv;
  cudaError_t e;
  if ((e = make_map(&mq, p.q, kD, p.H, tokens)) != cudaSuccess ||
      (e = make_map(&mk, p.k, kD, p.H, tokens)) != cudaSuccess ||
      (e = make_map(&mv, p.v, kD, p.H, tokens)) != cudaSuccess ||
      (e = make_map(&mo, p.dout, kD, p.H, tokens)) != cudaSuccess ||
      (e = make_out_map(&mdq, p.dq, kD, p.H, tokens)) != cudaSuccess ||
      (e = make_out_map(&mdk, p.dk, kD, p.H, tokens)) != cudaSuccess ||
      (e = make_out_map(&mdv, p.dv, kD, p.H, tokens)) != cudaSuccess)
    return e;
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load()) {
    if ((e = cudaFuncSetAttribute(bwd_level_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_intra_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kISmemBytes)) != cudaSuccess)
      return e;
    attr_set[dev].store(true);
  }
  // levels 0..7: one CTA per chunk, the first write of dq, dk, dv and dlam[:, 0..7]
  bwd_intra_tc<<<dim3((p.T + kC - 1) / kC, p.H, p.nseq), kThreads, kISmemBytes, st>>>(
      mq, mk, mv, mo, mdq, mdk, mdv, p, g);
  count_launch();
  const long long slots = 2ll * sm_count_bwd();   // two level CTAs per SM
  for (int lvl = kTcFirstLevel; lvl < p.L; ++lvl) {
    const int nblk = (int)(((long long)p.T + (1ll << lvl) - 1) >> lvl);
    // blocks that leave CTA slots free are taken by two CTAs each (half the tile steps each)
    const int split = (long long)nblk * p.H * p.nseq * kSplitDen <= slots ? 1 : 0;
    bwd_level_tc<<<dim3(nblk << split, p.H, p.nseq), kThreads, kSmemBytes, st>>>(
        mq, mk, mv, mo, mdq, mdk, mdv, p, g, lvl, split);
    count_launch();
  }
  return cudaGetLastError();
}

}  // namespace llattn
