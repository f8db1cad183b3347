/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention prefill library.
 *
 * The library computes the chunked forward (prefill) of Kimi Delta Attention
 * (KDA) for head dimension dk = dv = 128 on one GPU. Per sequence and head:
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = scale * S_t^T q_t
 *
 * with S a 128 x 128 fp32 state (rows: key channels, columns: value
 * channels), g_t a natural-log decay per key channel and beta_t a scalar.
 * KDA is Gated DeltaNet with one decay per channel instead of one scalar
 * decay for the whole state, keeping the history in a fixed-size state
 * (page "Kimi K3 开源满月…", section "KDA 内核到底难在哪"; page
 * "FlashKDA: CUTLASS Kernel من Moonshot لـ Kimi", section "سياق Kimi Linear").
 * Head dimension 128 only and forward only, as for FlashKDA (same FlashKDA
 * page, section "المتطلبات الأساسية"; page "Moonshot AI … FlashKDA …
 * (kucoin)"). Sequences of different lengths are packed along the token axis
 * and described by cu_seqlens in the FlashAttention convention (FlashKDA page,
 * section "تكامل مباشر مع flash-linear-attention").
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers on the current CUDA device.
 *   - The caller owns all inputs and outputs. kda_fwd takes a scratch ring
 *     (num_seqs * H * 16 slots of 15104 bytes) from a library-private
 *     stream-ordered memory pool and returns it in stream order after the
 *     kernel; the pool keeps its memory for later calls.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.
 *   - Argument errors are reported synchronously through the return code and
 *     nothing is enqueued; the functions never abort the process.
 *   - Results are deterministic: no atomics, no split reductions, and each
 *     (sequence, head) is computed independently of the rest of the batch, so
 *     a sequence gives bit-identical results alone or inside any batch.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_HEAD_DIM 128
#define KDA_ABI_VERSION 2

typedef enum kda_status {
  KDA_OK = 0,
  KDA_ERR_NULL = 1,        /* a required pointer is NULL */
  KDA_ERR_SHAPE = 2,       /* invalid sizes (negative T, H < 1, num_seqs < 1,
                              cu_seqlens NULL with num_seqs != 1, int overflow) */
  KDA_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  KDA_ERR_UNSUPPORTED = 4, /* the current device is not sm_100 (B200) */
  KDA_ERR_CUDA = 5,        /* a CUDA runtime call or the launch failed */
  KDA_ERR_CAPACITY = 6     /* kda_fwd_noalloc: num_seqs * num_heads exceeds
                              KDA_NOALLOC_MAX_PAIRS */
} kda_status_t;

/*
 * kda_fwd -- chunked KDA forward (prefill) for a packed batch.
 *
 * Layouts (row-major, contiguous, T = total_tokens, H = num_heads, N = num_seqs):
 *   q, k, v, out   bf16  [T, H, 128]
 *   g              fp32  [T, H, 128]   natural-log decay per key channel.
 *                  Precondition: -5 <= g <= 0 (the gate lower bound of
 *                  FlashKDA, page "Kimi K3 开源满月…", section
 *                  "KDA 内核到底难在哪"); outside it results are undefined
 *                  (may be inf/NaN), never an out-of-bounds access.
 *   beta           fp32  [T, H]
 *   initial_state  fp32  [N, H, 128 (key), 128 (value)] or NULL (zero state)
 *   final_state    fp32  [N, H, 128, 128] or NULL (not written); may alias
 *                  initial_state (each (sequence, head) reads its slice before
 *                  writing it).
 *   cu_seqlens     int32 [N + 1] on the device, cu[0] = 0, non-decreasing,
 *                  cu[N] = T; or NULL, meaning one sequence of T tokens
 *                  (then num_seqs must be 1). Its contents are not checked on
 *                  the host (that would need a synchronisation); the kernel
 *                  clamps every boundary into [0, T], so bad contents give
 *                  wrong results, never an out-of-bounds access.
 *   scale          the output scale (usually 1/sqrt(128)).
 * Alignment: every tensor pointer must be 16-byte aligned.
 * Zero-length sequences are allowed: their final state equals their initial
 * state (or zeros). T = 0 is allowed; then q, k, v, g, beta and out may be
 * NULL (they are never read or written).
 * Returns KDA_OK once the work is enqueued.
 */
kda_status_t kda_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     float scale, const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                     int32_t num_heads, const float* initial_state, void* out, float* final_state,
                     void* stream);

/*
 * kda_fwd_noalloc -- kda_fwd without any device-memory allocation.
 *
 * The method's sources have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory while they run. kda_fwd draws its
 * scratch ring from a stream-ordered memory pool, which such callers cannot
 * allow: serving engines that reserve the whole device for their own arena up
 * front, or deployments where CUDA memory pools are unavailable
 * (cudaDevAttrMemoryPoolsSupported = 0).
 *
 * Arguments, layouts, results and errors are those of kda_fwd, except:
 *   - The scratch ring lives in a fixed-size array in device memory that the
 *     library declares at file scope: every GPU that loads the library holds
 *     it (KDA_NOALLOC_MAX_PAIRS * 16 slots * 15232 bytes = 7.8 MB) until the
 *     process exits.
 *   - num_seqs * num_heads must not exceed KDA_NOALLOC_MAX_PAIRS; larger
 *     problems return KDA_ERR_CAPACITY and nothing is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (the kernel overwrites every slot before reading it, so nothing
 *     needs clearing). Calls whose kernels overlap on the GPU -- on different
 *     streams, or from different threads -- race on it and give wrong results;
 *     order them on one stream.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define KDA_NOALLOC_MAX_PAIRS 32
kda_status_t kda_fwd_noalloc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             float scale, const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                             int32_t num_heads, const float* initial_state, void* out, float* final_state,
                             void* stream);

/*
 * kda_set_slice_columns -- value columns per CTA for later calls (tuning).
 *
 * Each (sequence, head) runs as one thread-block cluster whose CTAs split the
 * 128 value columns. columns = 32 uses 4 CTAs per (sequence, head); 16 uses
 * 8, which doubles the SMs working on the same serial chains when there are
 * few sequences and heads. columns = 0 (the default) chooses per call: 16
 * when num_seqs * num_heads * 4 is at most half the device's SM count, else
 * 32. Each column's arithmetic is the same either way, so the results are
 * bitwise identical. Process-wide; affects kda_fwd and
 * kda_fwd_noalloc. Returns KDA_ERR_SHAPE for any other value (the setting is
 * then unchanged).
 */
kda_status_t kda_set_slice_columns(int32_t columns);

/* Human-readable text of a status code (static storage, never NULL). */
const char* kda_status_string(kda_status_t status);

/* Text of the last CUDA error seen by this thread inside the library
 * (static thread-local storage; "" if none). */
const char* kda_last_cuda_error(void);

/*
 * kda_wait_timeouts -- health counter of the current device.
 *
 * Every wait inside the kernel (on a pipeline stage, on a peer CTA of the
 * cluster) is bounded; a wait that runs out of budget increments a device
 * counter and lets the kernel finish instead of hanging (its results are then
 * undefined). This reads the counter into *count (synchronising with the
 * device) and resets it to zero when `reset` is non-zero. A healthy run leaves
 * it at 0.
 */
kda_status_t kda_wait_timeouts(uint32_t* count, int32_t reset);

/* KDA_ABI_VERSION of the loaded library. */
int32_t kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
