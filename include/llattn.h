/*
 * llattn.h - C ABI of the B200-native log-linear attention forward (Mamba-2 form).
 *
 * Operation.  For every sequence, head and 0-based sequence-local position t:
 *
 *   o_t = sum_{s <= t} lam[t, l(t,s)] * (prod_{r=s+1..t} a_r) * (q_t . k_s) * v_s
 *   l(t,s) = 0 if s == t, else 1 + floor(log2(t XOR s)),   a_r = exp(log_a[r]),
 *
 * i.e. linear attention whose causal mask is replaced by the hierarchical
 * (HODLR) mask of a Fenwick-tree partition of the prefix, with Mamba-2's
 * scalar selective gate and one weight per (query token, level).  Sources:
 * "Log-Linear Attention" (gist.science summaries, Italian "Sommario tecnico"
 * section 2 and Spanish "Resumen tecnico" section 2): the Fenwick partition into
 * buckets of exponentially growing size (Partizionamento Gerarchico / Particion
 * Jerarquica), the hierarchical mask M_H (Matrici Gerarchiche), the O(log T)
 * level states combined with per-level weights (Forma Ricorrente), the
 * chunkwise-parallel forward in O(T log T) (Training bullet / Algoritmo de
 * Entrenamiento), and the Log-Linear Mamba-2 variant (Variantes Propuestas 1).
 * lam is applied as given (the caller applies any positivity transform); there
 * is no softmax, no 1/sqrt(d) scale and no normalisation.
 *
 * Layouts (all row-major, contiguous, token-major, level innermost):
 *   q, k   [B, T, H, dk]        v [B, T, H, dv]       out [B, T, H, dv] (fp32)
 *   log_a  [B, T, H] (fp32)     lam [B, T, H, L] (fp32), L = llattn_num_levels(T)
 * Packed variable-length batches (cu_seqlens != NULL): B = number of sequences,
 * tensors are [total, H, .] with total = cu_seqlens[B], cu_seqlens is a DEVICE
 * int32 array of B+1 non-decreasing offsets starting at 0, and T is an upper
 * bound on every sequence length (it fixes L and the launch grid).  Fenwick
 * positions and the gate product restart at every sequence start.
 *
 * Ownership.  Every tensor pointer is caller-owned DEVICE memory; the library
 * never frees or retains it.  q, k, v and out must be 16-byte aligned, log_a and
 * lam 4-byte aligned; out must not alias any input.  Calls are asynchronous on
 * `stream` (a cudaStream_t; NULL = legacy default stream) and return once the
 * kernels are enqueued; `out` is fully overwritten for every token of every
 * sequence (rows outside [0, total) are not touched).
 *
 * Output precision.  out is fp32 for every input type: rounding the output to
 * bf16 alone moves it by up to ~4% of its RMS on these heavy-tailed outputs.
 *
 * Errors.  Every entry point returns an llattn_status and never aborts.  Bad
 * arguments are rejected before any launch.  Launch failures map to
 * LLATTN_ERR_CUDA.  Conditions only the device can see (a varlen sequence longer
 * than T, a bounded wait that ran out) set bits in a per-device status word that
 * llattn_device_status() reads; the affected output rows are then unspecified.
 */
#ifndef LLATTN_H_
#define LLATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LLATTN_API __attribute__((visibility("default")))
#else
#define LLATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LLATTN_OK = 0,
  LLATTN_ERR_ARG = 1,         /* null pointer, negative size, aliasing */
  LLATTN_ERR_SHAPE = 2,       /* unsupported dk/dv, T or sizes out of range */
  LLATTN_ERR_ALIGN = 3,       /* pointer misaligned (16 B for q/k/v/out, 4 B for log_a/lam) */
  LLATTN_ERR_DTYPE = 4,       /* unknown input dtype code */
  LLATTN_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  LLATTN_ERR_TIMEOUT = 6,     /* a bounded device-side wait ran out (see llattn_device_status) */
  LLATTN_ERR_WORKSPACE = 7,   /* caller workspace too small or misaligned */
  LLATTN_ERR_UNSUPPORTED = 8, /* valid request this build has no kernel for */
  LLATTN_ERR_NOALLOC_LIMIT = 9 /* llattn_fwd_noalloc: problem too big for its fixed scratch */
} llattn_status;

/* Input element types for llattn_fwd_ex. */
enum { LLATTN_F32 = 0, LLATTN_BF16 = 1 };

/* Kernel paths for llattn_fwd_ex.
 *   AUTO            tcgen05 path where one exists for the shape, else SIMT.  With chunk 0, a
 *                   call that resolves to SIMT with T <= 512 runs the masked (quadratic) form
 *                   in one launch instead of the chunkwise kernels: at that length the whole
 *                   key range of a query fits a few shared-memory tiles.  It needs no
 *                   workspace and computes in fp32 like SIMT.
 *   SIMT            CUDA-core kernels (any dk, dv in {32,64,128}; fp32 or bf16 inputs).
 *   TCGEN05         tensor-core kernel, warp-specialised pipeline (bf16 inputs, d_k and
 *                   d_v in {64, 128}, chunk 128, T <= 131072; the serial cross-check d = 64,
 *                   T <= 8192; it rounds P, V, the decay-scaled K and the level states once
 *                   to fp16, so those intermediates must stay below 6.5e4 in magnitude -
 *                   true for L2-normalised q, k and moderate v, lam; a value out of range
 *                   sets LLATTN_DEV_NONFINITE; use SIMT then).
 *   TCGEN05_SERIAL  the same arithmetic with one warp group walking each chunk's steps in
 *                   order (a slower cross-check of the pipelined kernel). */
enum {
  LLATTN_PATH_AUTO = 0,
  LLATTN_PATH_SIMT = 1,
  LLATTN_PATH_TCGEN05 = 2,
  LLATTN_PATH_TCGEN05_SERIAL = 3
};

/* Device status bits (llattn_device_status). */
enum {
  LLATTN_DEV_SEQ_TOO_LONG = 1u,  /* a varlen sequence was longer than T */
  LLATTN_DEV_WAIT_TIMEOUT = 2u,  /* an mbarrier / pipeline wait hit its iteration limit */
  LLATTN_DEV_BAD_CU_SEQLENS = 4u, /* cu_seqlens decreasing */
  LLATTN_DEV_DECODE_POS = 8u,    /* decode step or prefill state: a position outside [0, 2^(L-1)) */
  LLATTN_DEV_NONFINITE = 16u     /* tensor-core forward: an output value came out inf or NaN.
                                  * With finite inputs this means an intermediate rounded to
                                  * fp16 (P, V, the decay-scaled K, a level state, Q) left
                                  * the fp16 range (|x| >= 65520): any such overflow reaches
                                  * the output as inf or NaN.  Rerun on LLATTN_PATH_SIMT. */
};

/* Version of this ABI (increments on any signature change). */
LLATTN_API int llattn_abi_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
LLATTN_API const char* llattn_status_str(llattn_status s);

/* Number of Fenwick levels for sequences of at most T tokens: 1 + ceil(log2 T)
 * (1 for T <= 1).  This is the innermost extent of lam. */
LLATTN_API int llattn_num_levels(int T);

/*
 * llattn_fwd - forward with bf16 q, k, v (each a uint16 bf16 bit pattern),
 * fp32 log_a and lam, fp32 out, on the default (tensor-core) path.  Scratch
 * for inter-chunk states comes from a per-device buffer the library grows on
 * demand and keeps until exit; calls that overlap on the GPU (two streams)
 * must use llattn_fwd_ex with their own workspaces instead.
 * B, H >= 0, T >= 0, dk and dv in {32, 64, 128}.  Returns LLATTN_OK on success.
 */
LLATTN_API llattn_status llattn_fwd(const void* q, const void* k, const void* v, const float* log_a,
                         const float* lam, float* out, int B, int H, int T, int dk, int dv,
                         const int* cu_seqlens, void* stream);

/* llattn_fwd_bf16 - the same call as llattn_fwd, named for its input type. */
LLATTN_API llattn_status llattn_fwd_bf16(const void* q, const void* k, const void* v,
                                         const float* log_a, const float* lam, float* out, int B,
                                         int H, int T, int dk, int dv, const int* cu_seqlens,
                                         void* stream);

/* llattn_fwd_f32 - the same operation on fp32 q, k, v (CUDA-core fp32 path, no
 * tensor cores, so results meet a 1e-4 relative bound; the automatic path, so T <= 512 runs
 * the one-launch masked form).  Arguments as llattn_fwd. */
LLATTN_API llattn_status llattn_fwd_f32(const float* q, const float* k, const float* v, const float* log_a,
                             const float* lam, float* out, int B, int H, int T, int dk, int dv,
                             const int* cu_seqlens, void* stream);

/*
 * llattn_workspace_bytes - device scratch that llattn_fwd_ex needs for this
 * shape, dtype and path (0 is possible).  chunk = 0 selects the default chunk
 * length of the path.  varlen != 0 sizes for packed sequences bounded by T.
 */
LLATTN_API llattn_status llattn_workspace_bytes(int in_dtype, int path, int chunk, int B, int H, int T,
                                     int dk, int dv, int varlen, size_t* bytes);

/*
 * llattn_fwd_ex - the general entry point.
 *   in_dtype   LLATTN_F32 or LLATTN_BF16 (type of q, k, v).
 *   path       LLATTN_PATH_* (SIMT accepts both dtypes, TCGEN05 bf16 only).
 *   chunk      chunk length (power of two; 0 = default of the path: SIMT 16 for
 *              T <= 256 else 64, TCGEN05 128).  The result does not depend on it
 *              beyond rounding.
 *   workspace  caller-owned device scratch of at least llattn_workspace_bytes()
 *              bytes (256-byte aligned), or NULL to use the library's per-device
 *              buffer as llattn_fwd does.
 */
LLATTN_API llattn_status llattn_fwd_ex(int in_dtype, int path, int chunk, const void* q, const void* k,
                            const void* v, const float* log_a, const float* lam, float* out,
                            int B, int H, int T, int dk, int dv, const int* cu_seqlens,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * llattn_device_status - read (and, if clear != 0, reset) the status word of the
 * current device.  Synchronises the device.  *flags receives LLATTN_DEV_* bits.
 */
LLATTN_API llattn_status llattn_device_status(unsigned int* flags, int clear);

/*
 * Segments of the tensor-core path.  Each CTA walks a run of 128-token chunks of one
 * (sequence, head, 64-column value tile), keeping one fp16 state per Fenwick level of the run
 * on chip.  Long sequences, or batches with fewer such runs than the GPU has SMs, are cut into
 * aligned segments of 2^g chunks walked in parallel.  The levels above a segment (its
 * position's set bits, one level up) come from two pre-pass kernels: the segments' total
 * states on the tensor cores, then the Fenwick binary counter over segments, whose dyadic
 * block states the walk copies in ([IT] section 2, "Partizionamento Gerarchico"; Spanish
 * section 2, "Algoritmo de Entrenamiento (Chunk-scan)": the chunk-level scan, applied over
 * groups of chunks).  The scratch for those states is part of llattn_workspace_bytes().
 *
 * llattn_segment_plan - the chunks per segment a tensor-core call of this shape uses
 *   (*chunks_per_segment = 0: every CTA walks a whole sequence, or the shape has no
 *   tensor-core path).  varlen != 0 for packed batches (T then bounds the lengths).
 * llattn_set_segment_chunks - force the segment length for later calls of this process:
 *   chunks = 0 restores the automatic choice, else a power of two >= 2 (a length that would
 *   need more than 8 counter levels over segments falls back to the automatic choice).  A
 *   tuning and testing knob; the result does not depend on it beyond rounding.  Not
 *   thread-safe with respect to calls already being planned on other threads.
 */
LLATTN_API llattn_status llattn_segment_plan(int B, int H, int T, int dk, int dv, int varlen,
                                             int* chunks_per_segment);
LLATTN_API llattn_status llattn_set_segment_chunks(int chunks);

/*
 * llattn_stream_status - the same read, ordered on one stream instead of the whole
 * device: waits for the work already enqueued on `stream` (a cudaStream_t; NULL =
 * legacy default stream), then copies the status word back (and clears it, if
 * clear != 0) on that stream.  The word is per device, so it also holds bits set by
 * kernels of other streams that have finished by then.  Returns LLATTN_ERR_TIMEOUT
 * when LLATTN_DEV_WAIT_TIMEOUT is set, else LLATTN_OK (or a CUDA error).
 */
LLATTN_API llattn_status llattn_stream_status(unsigned int* flags, int clear, void* stream);

/*
 * llattn_fwd_host - the forward on HOST buffers, for callers whose data is not
 * on the GPU.  Copies q, k, v, log_a, lam (and cu_seqlens) into device staging
 * memory the library owns (grown on demand, kept per device until exit), runs
 * the default path (tensor cores for bf16, CUDA cores for fp32), copies out back
 * and synchronises `stream` before returning.  Host buffers should be pinned
 * (page-locked) for the copies to run at full speed.  in_dtype: LLATTN_BF16
 * (q, k, v as uint16 bf16 bit patterns) or LLATTN_F32.  cu_seqlens, if not NULL,
 * is a HOST int32 array [B+1]; the other arguments are as in llattn_fwd.
 * Dense batches of two or more sequences are pipelined row by row: the upload of one
 * row, the forward of another and the download of a third overlap (two copy streams
 * the library keeps per device, ordered against `stream` with events).
 * Concurrent calls from several threads are serialised on an internal lock.
 */
LLATTN_API llattn_status llattn_fwd_host(int in_dtype, const void* q, const void* k, const void* v,
                              const float* log_a, const float* lam, float* out, int B, int H,
                              int T, int dk, int dv, const int* cu_seqlens, void* stream);

/*
 * llattn_fwd_noalloc - the forward for callers that must not have a library
 * allocate device memory on their behalf.  Typical cases: an application whose
 * own allocator reserves nearly all of the GPU's memory up front, where a
 * cudaMalloc issued here would fail or eat into memory that allocator has
 * promised elsewhere; a service that must know its whole device footprint before
 * it takes traffic; and latency-bound code, because the buffer behind llattn_fwd
 * grows by cudaFree + cudaMalloc, and cudaFree waits for the whole device,
 * stalling every stream of the process.  This entry point has no counterpart in
 * the log-linear attention papers; it is packaging around the same operation.
 *
 * It computes what llattn_fwd_ex computes with path LLATTN_PATH_SIMT and the
 * default chunk (CUDA cores, fp32 arithmetic; in_dtype LLATTN_F32 or
 * LLATTN_BF16), and takes its inter-chunk scratch from one array of
 * LLATTN_NOALLOC_SCRATCH_BYTES (32 MiB) per device that is part of the library's
 * device code itself.  Arguments, layouts, ownership, the device status word and
 * the other error codes are those of llattn_fwd_ex.
 *
 * Size limit.  The problem's scratch, as reported by llattn_workspace_bytes(
 * in_dtype, LLATTN_PATH_SIMT, 0, B, H, T, dk, dv, cu_seqlens != NULL, &n), must
 * not exceed LLATTN_NOALLOC_SCRATCH_BYTES.  Larger problems return
 * LLATTN_ERR_NOALLOC_LIMIT (after the shape and dtype checks, before the pointer
 * checks) without making any CUDA call.  For scale: B=2, H=16, T=2048, dk=dv=64 needs 31.5 MiB and fits;
 * B=4, H=32, T=8192 does not.
 *
 * Setup.  The first call on a device that has work to do looks up the array's
 * address there (cudaGetSymbolAddress, with that device current), keeps it, and
 * returns LLATTN_ERR_CUDA if the lookup fails.  That first call should come
 * before any stream capture.  Later calls only launch kernels.
 *
 * Zeroing.  Each call writes every scratch entry it reads before reading it, so
 * no part of the array has to start at zero and nothing is cleared between calls.
 * The device status word keeps its meaning (sticky until llattn_device_status
 * clears it).
 *
 * Concurrency.  There is one array per device, shared by every caller in the
 * process.  Calls whose kernels can overlap on the GPU (on different streams, or
 * from host threads that do not order their streams) race on it and can corrupt
 * one another's output.  Calls on one stream run one after another and are safe.
 * With launch recording on (llattn_profile(1)) the library may create CUDA events
 * for its timing pairs; it is off by default.
 */
#define LLATTN_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
LLATTN_API llattn_status llattn_fwd_noalloc(int in_dtype, const void* q, const void* k,
                                            const void* v, const float* log_a, const float* lam,
                                            float* out, int B, int H, int T, int dk, int dv,
                                            const int* cu_seqlens, void* stream);

/*
 * Decoding: one new token per sequence per call, over the O(log T) level states.
 *
 * Log-Linear Attention (gist.science summaries, Italian "Sommario tecnico" section 2, "Forma
 * Ricorrente e Parallelizzata", decoding bullet; Spanish "Resumen tecnico" section 2,
 * "Particion Jerarquica"): at inference the layer keeps one d_k x d_v state per Fenwick
 * level and combines them with the per-level weights.  For the token at 0-based position n
 * of a sequence, with Mamba-2's scalar gate a_n = exp(log_a):
 *   1. every occupied level l >= 1 is gated by a_n; level 0 is k_n v_n^T;
 *   2. o_n = sum over level 0 and the occupied levels l of lam[l] * (q_n^T S_l);
 *   3. with m the number of trailing one bits of n, levels 0..m are summed into level m+1
 *      and levels 1..m fall empty (a binary-counter carry).
 * Level l >= 1 is occupied exactly when bit l-1 of n is set, so a sequence's position is its
 * whole occupancy record.  Decoding tokens 0..T-1 of a sequence this way gives the outputs
 * llattn_fwd gives for that sequence (same operation, one token at a time).
 *
 * llattn_decode_state_bytes - size of the state buffer of B sequences x H heads whose
 * positions stay below 2^(L-1) (L = llattn_num_levels(T) for sequences of at most T tokens):
 * B*H*(L-1)*dk*dv*4 + B*H*2*(L-1)*4 bytes.  1 <= L <= 32.
 *
 * llattn_decode_step - one step for every sequence of the batch.
 *   in_dtype  LLATTN_BF16 (q, k, v as uint16 bf16 bit patterns) or LLATTN_F32.
 *   q, k      [B, H, dk]; v [B, H, dv]: each sequence's new token.  log_a [B, H] fp32;
 *             lam [B, H, L] fp32 (level innermost; entries above the position's highest
 *             level are read but unused).  out [B, H, dv] fp32, fully overwritten.
 *   pos       DEVICE int32 [B]: tokens sequence b has absorbed, i.e. the new token's position.
 *             Read only: the caller advances it for the next step.  Setting pos[b] = 0 starts
 *             sequence b afresh; nothing else in the state has to be reset or cleared.
 *   state     DEVICE fp32 buffer of llattn_decode_state_bytes(), caller-owned and kept
 *             between steps (non-NULL even when that size is 0, i.e. L = 1).  Layout: levels [B, H, L-1, dk, dv] (slot j = level j+1, row-major
 *             dk x dv), then gate [B, H, 2, L-1].  A slot holds its level's state as it was
 *             when written; gate[b, h, p, j] is the log of the gate product slot j has missed
 *             since then, valid at positions of parity p.  The level's state just before
 *             position n is exp(gate[b, h, n & 1, j]) * levels[b, h, j].  To start from states
 *             computed elsewhere, write them to levels with gate[b, h, pos[b] & 1, :] = 0.
 *   dk, dv    in {32, 64, 128}.  B, H <= 65535.
 * Pointers: q, k, v, state and out 16-byte aligned, log_a, lam and pos 4-byte aligned; out
 * must not overlap the inputs or the state.  Asynchronous on `stream`.  A position outside
 * [0, 2^(L-1)) leaves that sequence's output and state untouched and sets
 * LLATTN_DEV_DECODE_POS in the device status word.  Steps that share a state buffer must run
 * in order (one stream); arithmetic is fp32 on CUDA cores (an HBM-bound step: it reads each
 * occupied level state once and writes the carried one).
 */
LLATTN_API llattn_status llattn_decode_state_bytes(int B, int H, int L, int dk, int dv,
                                                   size_t* bytes);
LLATTN_API llattn_status llattn_decode_step(int in_dtype, const void* q, const void* k,
                                            const void* v, const float* log_a, const float* lam,
                                            const int* pos, float* state, float* out, int B,
                                            int H, int L, int dk, int dv, void* stream);

/*
 * llattn_prefill_state - the decoding state after a prompt: for every sequence of a dense or
 * packed batch, the state llattn_decode_step expects at position n = the sequence's length,
 * so that decoding continues the prompt (its outputs come from llattn_fwd).
 *
 * Log-Linear Attention (gist.science summaries, Italian "Sommario tecnico" section 2,
 * "Partizionamento Gerarchico"; Spanish "Resumen tecnico" section 2, "Particion Jerarquica"):
 * seen from position n, the earlier tokens fall into the Fenwick buckets of n: level l >= 1
 * holds the tokens s < n with l(n, s) = l, i.e. [P 2^l, P 2^l + 2^(l-1)) with P = n >> l,
 * non-empty exactly when bit l-1 of n is set.  Its state just before n is
 *   sum over s in that bucket of (prod_{r=s+1..n-1} a_r) k_s v_s^T,   a_r = exp(log_a[r]).
 * It is written in the decoding state's lazy-gate form: slot l-1 receives the sum gated only
 * up to the bucket's last token (prod over r = s+1 .. P 2^l + 2^(l-1) - 1), and both gate rows
 * gate[b, h, 0..1, l-1] receive the log of the rest, sum of log_a[r] over the tokens after the
 * bucket, so that exp(gate) * slot is the state (the stored values never underflow however
 * long the decay after the bucket).  Levels without a bucket get gate 0 and keep their slot's
 * contents (decoding never reads them).
 *   in_dtype  LLATTN_BF16 (k, v as uint16 bf16 bit patterns) or LLATTN_F32.
 *   k, v      DEVICE: dense [B, T, H, dk] / [B, T, H, dv], or packed [total, H, dk] /
 *             [total, H, dv] with cu_seqlens, as llattn_fwd takes them.  log_a [.., H] fp32.
 *             q and lam are not needed: the state holds no readout.
 *   state     DEVICE fp32 buffer of llattn_decode_state_bytes(B, H, L, dk, dv), caller-owned,
 *             laid out as llattn_decode_step describes; the occupied level slots and all
 *             gate entries of every (sequence, head) are written.  Decoding then starts with
 *             pos[b] = n.
 *   cu_seqlens DEVICE int32 [B + 1] or NULL (every length is T).  A length above T is cut
 *             to T and sets LLATTN_DEV_SEQ_TOO_LONG; a decreasing one sets LLATTN_DEV_BAD_CU_SEQLENS.
 *   L         the decode state's level count: lengths n must be below 2^(L-1) (a sequence at
 *             n >= 2^(L-1) is left unwritten and sets LLATTN_DEV_DECODE_POS).
 *   dk, dv    in {32, 64, 128}.  B, H <= 65535, 0 <= T <= 2^24, 1 <= L <= 32.
 * Pointers: k, v and state 16-byte aligned, log_a and cu_seqlens 4-byte aligned; state must not
 * overlap the inputs.  Asynchronous on `stream`; fp32 arithmetic on CUDA cores, one CTA per
 * (level, head, sequence) walking its bucket from the end (the suffix decay factors are at
 * most 1).  It reads each prompt token's k and v once per level whose bucket holds it, i.e.
 * once in all.
 */
LLATTN_API llattn_status llattn_prefill_state(int in_dtype, const void* k, const void* v,
                                              const float* log_a, float* state, int B, int H,
                                              int T, int L, int dk, int dv,
                                              const int* cu_seqlens, void* stream);

/*
 * Backward pass: the gradients of sum(dout * out) with respect to q, k, v, log_a and lam, for
 * the operation llattn_fwd computes (same inputs, same layouts, dense or packed).
 *
 * Log-Linear Attention (gist.science summaries, Italian "Sommario tecnico" section 2, "Matrici
 * Gerarchiche"): out = ((Q K^T) .* M_H) V with M_H the hierarchical (HODLR) mask
 * M_H[t, s] = lam[t, l(t, s)] * prod_{r=s+1..t} a_r.  Level by level, the mask couples the
 * left and right halves of aligned blocks of 2^l positions with a rank-d factor, and the
 * gradients are computed that way:
 *   dq_t   = sum_{s<=t} M_H[t,s] (dout_t . v_s) k_s      dk_s = sum_{t>=s} M_H[t,s] (dout_t . v_s) q_t
 *   dv_s   = sum_{t>=s} M_H[t,s] (q_t . k_s) dout_t
 *   dlam[t, l]  = sum over s with l(t,s) == l of prod a * (q_t . k_s)(dout_t . v_s)
 *   dlog_a[r]   = sum over t >= r of (q_t . dq_t - k_t . dk_t)   (positions within a sequence)
 * dlam is zero at levels a token has no partner at; dlog_a at a sequence's first position is
 * zero up to rounding (no gate product contains it).
 *
 * llattn_bwd_workspace_bytes - scratch llattn_bwd needs: B*T*H*8 bytes (fp64 prefix sums of
 * log_a), rounded up to 256.  dk == dv in {32, 64, 128}; other head sizes return
 * LLATTN_ERR_SHAPE.
 *
 * llattn_bwd
 *   in_dtype   LLATTN_BF16 or LLATTN_F32: the type of q, k, v and dout (bf16 as uint16 bit
 *              patterns).  With bf16 inputs at d = 64 the pair interactions run on the
 *              tensor cores (within each aligned 128-token chunk, then level by level over
 *              larger aligned blocks), every derived operand split into bf16 high and low
 *              parts (fp32-accumulation accuracy); otherwise arithmetic is fp32 on CUDA
 *              cores.
 *   q, k, v, log_a, lam, B, H, T, cu_seqlens   as in llattn_fwd.
 *   dout       [B, T, H, dv] (packed: [total, H, dv]), the gradient of the loss at out.
 *   dq, dk, dv [.., H, d] fp32; dlog_a [.., H] fp32; dlam [.., H, L] fp32: fully overwritten
 *              for every token of every sequence, with one exception: a packed sequence
 *              longer than T is cut at T (as in the forward), its rows past T are left
 *              unwritten, and LLATTN_DEV_SEQ_TOO_LONG is set in the device status word.
 *   workspace  caller-owned device scratch of llattn_bwd_workspace_bytes() bytes (256-byte
 *              aligned), or NULL for the library's per-device buffer (as llattn_fwd).
 * Pointers: q, k, v, dout, dq, dk, dv 16-byte aligned, the rest 4-byte aligned; no gradient
 * may overlap an input or another gradient.  Asynchronous on `stream`.
 */
LLATTN_API llattn_status llattn_bwd_workspace_bytes(int B, int H, int T, int dk, int dv,
                                                    size_t* bytes);
LLATTN_API llattn_status llattn_bwd(int in_dtype, const void* q, const void* k, const void* v,
                                    const float* log_a, const float* lam, const void* dout,
                                    float* dq, float* dk, float* dv, float* dlog_a, float* dlam,
                                    int B, int H, int T, int dk_dim, int dv_dim,
                                    const int* cu_seqlens, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * llattn_gdn_fwd - forward of Log-Linear Gated DeltaNet, the second variant of the pages
 * (gist.science "Log-Linear Attention", Italian "Sommario tecnico" section 2,
 * "Generalizzazione"; Spanish "Variantes Propuestas" item 2: the log-linear structure applied
 * to the gated delta rule).  The pages print no formula for it; the operation computed is
 *
 *   o_t = sum_{s <= t} lam[t, l(t,s)] * beta_s * (q_t^T A_t A_{t-1} ... A_{s+1} k_s) * v_s,
 *   A_r = alpha_r (I - beta_r k_r k_r^T),   alpha_r = exp(log_alpha[r]),
 *
 * with l(t, s) the Fenwick level of llattn_fwd: one gated-delta state per Fenwick level,
 * every occupied level taking the transition A_t, the token's write beta_t k_t v_t^T opening
 * level 0, levels weighted by lam and merged on promotion.  With lam == 1 it is plain Gated
 * DeltaNet; with A_t = alpha_t I it is llattn_fwd's operation with v_s scaled by beta_s.
 *   in_dtype   LLATTN_BF16 or LLATTN_F32 (type of q, k, v).  Arithmetic and the state are fp32
 *              on CUDA cores (the recurrent form, token by token; one warp per value column).
 *   q, k       [B, T, H, dk] (packed: [total, H, dk]); the delta rule expects unit-norm k.
 *   v          [B, T, H, dv];  log_alpha, beta [B, T, H] fp32;  lam [B, T, H, L] fp32.
 *   out        [B, T, H, dv] fp32, fully overwritten (rows outside [0, total) untouched).
 *   dk, dv in {32, 64, 128}, T <= 65536; cu_seqlens as in llattn_fwd.
 * Pointers 4-byte aligned; out must not overlap an input.  Asynchronous on `stream`; no
 * scratch memory.  Errors as llattn_fwd.
 */
LLATTN_API llattn_status llattn_gdn_fwd(int in_dtype, const void* q, const void* k,
                                        const void* v, const float* log_alpha, const float* beta,
                                        const float* lam, float* out, int B, int H, int T, int dk,
                                        int dv, const int* cu_seqlens, void* stream);

/*
 * Launch accounting, for benchmarks.  llattn_profile(1) starts recording a pair
 * of CUDA events on the call's stream around the dominant kernel of every
 * forward (the one that streams q, k, v, lam and writes out); llattn_profile(0)
 * stops.  llattn_profile_read returns the summed device time of those kernels
 * (synchronising on the recorded events), how many were timed, and how many
 * kernels of this library were launched in total since the last reset (counted
 * whether or not recording is on); reset != 0 clears all three.
 */
LLATTN_API llattn_status llattn_profile(int enable);
LLATTN_API llattn_status llattn_profile_read(double* main_kernel_ms, long long* main_launches,
                                             long long* total_launches, int reset);

/* llattn_last_cuda_error - the cudaError_t behind the last LLATTN_ERR_CUDA of
 * this thread (0 if none). */
LLATTN_API int llattn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LLATTN_H_ */
