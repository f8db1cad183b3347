/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention prefill library.
 *
 * The library computes the chunked forward (prefill) of Kimi Delta Attention
 * (KDA) for head dimension dk = dv = 128 on one GPU, and the one-token decode
 * step against resident states. Per sequence and head:
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
 *   - Tensors are described by kda_tensor_t: a DEVICE pointer on the current
 *     CUDA device, a dtype, a shape and element strides (any order of the
 *     outer dimensions; see kda_fwd for what each tensor must satisfy).
 *   - The caller owns all inputs and outputs. kda_fwd takes a scratch ring
 *     (num_seqs * H slots of KDA_RING_BYTES_PER_PAIR bytes) from a
 *     library-private stream-ordered memory pool and returns it in stream
 *     order after the kernel; the pool keeps its memory for later calls.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.
 *   - Argument errors are reported synchronously through the return code and
 *     nothing is enqueued; the functions never abort the process.
 *   - Results are deterministic: no atomics, no split reductions, and each
 *     (sequence, head) is computed independently of the rest of the batch, so
 *     a sequence gives bit-identical results alone or inside any batch.
 *   - First-call setup per device (capability check, kernel attributes, the
 *     memory pool) is guarded by a lock: concurrent first calls from several
 *     host threads are safe.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_HEAD_DIM 128
#define KDA_ABI_VERSION 5

typedef enum kda_status {
  KDA_OK = 0,
  KDA_ERR_NULL = 1,        /* a required tensor or pointer is NULL */
  KDA_ERR_SHAPE = 2,       /* wrong ndim or shape, or inconsistent sizes
                              (T, H, num_seqs), or an int overflow */
  KDA_ERR_ALIGN = 3,       /* a data pointer is not 16-byte aligned */
  KDA_ERR_UNSUPPORTED = 4, /* the current device is not sm_100 (B200) */
  KDA_ERR_CUDA = 5,        /* a CUDA runtime call or the launch failed */
  KDA_ERR_CAPACITY = 6,    /* kda_fwd_noalloc: num_seqs * num_heads exceeds
                              KDA_NOALLOC_MAX_PAIRS */
  KDA_ERR_DTYPE = 7,       /* a tensor has the wrong dtype */
  KDA_ERR_STRIDE = 8,      /* a tensor's strides are not supported (see kda_fwd) */
  KDA_ERR_DEVICE = 9,      /* kda_device_status: the device recorded a fault */
  KDA_ERR_VALUE = 10       /* a scalar argument is outside its range */
} kda_status_t;

typedef enum kda_dtype { KDA_BF16 = 1, KDA_F32 = 2, KDA_I32 = 3 } kda_dtype_t;

/*
 * A strided tensor in device memory. shape[0..ndim) and stride[0..ndim) are
 * in elements; entries at or beyond ndim are ignored. The caller keeps
 * ownership of `data`.
 */
typedef struct kda_tensor {
  void* data;
  int32_t ndim;
  kda_dtype_t dtype;
  int64_t shape[4];
  int64_t stride[4];
} kda_tensor_t;

/* Scratch bytes per (sequence, head) that kda_fwd takes from its pool. */
#define KDA_RING_BYTES_PER_PAIR (6 * 66560)

/*
 * kda_fwd -- chunked KDA forward (prefill) for a packed batch.
 *
 * Tensors (T = total tokens, H = heads, N = num_seqs):
 *   q, k, v, out   bf16  [T, H, 128]
 *   g              fp32  [T, H, 128]   natural-log decay per key channel.
 *                  Precondition: -5 <= g <= 0 (the gate lower bound of
 *                  FlashKDA, page "Kimi K3 开源满月…", section
 *                  "KDA 内核到底难在哪"); outside it results are undefined
 *                  (may be inf/NaN), never an out-of-bounds access.
 *   beta           fp32  [T, H]
 *   initial_state  fp32  [N, H, 128 (key), 128 (value)], contiguous, or NULL
 *                  (zero state)
 *   final_state    fp32  [N, H, 128, 128], contiguous, or NULL (not
 *                  written); may alias initial_state (each (sequence, head)
 *                  reads its slice before writing it).
 *   cu_seqlens     int32 [N + 1] on the device, cu[0] = 0, non-decreasing,
 *                  cu[N] = T; or NULL, meaning one sequence of T tokens (then
 *                  num_seqs must be 1). Its contents are not read on the host
 *                  (that would need a synchronisation): the kernel clamps every
 *                  boundary into [0, T], so bad contents give wrong results but
 *                  never an out-of-bounds access, and it records them in the
 *                  device status word (kda_device_status).
 *   scale          the output scale (usually 1/sqrt(128)).
 * Strides: the last dimension of q, k, v, g and out must have stride 1; their
 *   token and head strides must be positive multiples of 16 bytes (8 bf16 or
 *   4 fp32 elements), so that views of a fused projection output (for
 *   example q, k, v as slices of one [T, H, 3 * 128] tensor) work without a
 *   copy. out must not overlap itself (token and head strides nest). beta may
 *   have any positive strides. States must be contiguous.
 * Alignment: every data pointer must be 16-byte aligned, except beta's (4 bytes).
 * Zero-length sequences are allowed: their final state equals their initial
 * state (or zeros). T = 0 is allowed; then the token tensors' data pointers
 * may be NULL and their strides are not checked (they are never read or
 * written).
 * Errors: KDA_ERR_NULL (a required descriptor or pointer missing),
 * KDA_ERR_DTYPE, KDA_ERR_SHAPE, KDA_ERR_STRIDE, KDA_ERR_ALIGN,
 * KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA; nothing is enqueued on any error.
 * Returns KDA_OK once the work is enqueued.
 */
kda_status_t kda_fwd(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v,
                     const kda_tensor_t* g, const kda_tensor_t* beta, float scale,
                     const int32_t* cu_seqlens, int32_t num_seqs,
                     const kda_tensor_t* initial_state, const kda_tensor_t* out,
                     const kda_tensor_t* final_state, void* stream);

/*
 * kda_fwd_fused -- kda_fwd with the gate preprocessing of a KDA layer fused
 * into the kernel: it takes the raw tensors that precede the recurrence.
 *
 *   q, k   bf16 [T, H, 128]  raw projections; the kernel L2-normalises each
 *                            (token, head) row: q / max(||q||_2, 1e-6)
 *   g      fp32 [T, H, 128]  gate logits x; the decay is
 *                            g = max(log sigmoid(x), lower_bound)
 *   beta   fp32 [T, H]       logits b; the write strength is sigmoid(b)
 *   lower_bound              in [-5, 0): the gate lower bound that keeps every
 *                            decay factor of a chunk in range (page "Kimi K3
 *                            开源满月…", section "KDA 内核到底难在哪", uses -5);
 *                            else KDA_ERR_VALUE
 * Everything else (v, states, cu_seqlens, out, layouts, strides, scratch,
 * errors) is as for kda_fwd. The preprocessed q, k, g and beta exist only
 * inside the kernel (fp32, then the bf16 operands of the tensor-core
 * products); they are never written to memory. Always runs the 16-token path
 * (kda_set_path does not apply), with the time split where kda_fwd would
 * take it.
 */
kda_status_t kda_fwd_fused(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v,
                           const kda_tensor_t* g, const kda_tensor_t* beta, float scale, float lower_bound,
                           const int32_t* cu_seqlens, int32_t num_seqs,
                           const kda_tensor_t* initial_state, const kda_tensor_t* out,
                           const kda_tensor_t* final_state, void* stream);

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
 *     it (KDA_NOALLOC_MAX_PAIRS * KDA_RING_BYTES_PER_PAIR = 12.8 MB) until the
 *     process exits.
 *   - num_seqs * num_heads must not exceed KDA_NOALLOC_MAX_PAIRS; larger
 *     problems return KDA_ERR_CAPACITY and nothing is launched.
 *   - The first call on a device loads the library's device code there (CUDA
 *     loads modules lazily), which allocates the array, and then looks up its
 *     device address (cudaGetSymbolAddress) with that device current. Make that
 *     first call before reserving the device's memory for an arena, and before
 *     any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (the kernel overwrites every slot before reading it, so nothing
 *     needs clearing). Calls whose kernels overlap on the GPU -- on different
 *     streams, or from different threads -- race on it and give wrong results;
 *     order them on one stream.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define KDA_NOALLOC_MAX_PAIRS 32
kda_status_t kda_fwd_noalloc(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v,
                             const kda_tensor_t* g, const kda_tensor_t* beta, float scale,
                             const int32_t* cu_seqlens, int32_t num_seqs,
                             const kda_tensor_t* initial_state, const kda_tensor_t* out,
                             const kda_tensor_t* final_state, void* stream);

/*
 * kda_set_path -- which kernel later calls use (tuning and testing).
 *
 *   64: 64-token chunks on tcgen05 tensor cores, one 4-CTA cluster per
 *       (sequence, head): the whole state in tensor memory on one SM, three
 *       SMs preparing the chunks' operands.
 *   16: 16-token chunks on mma.sync, the value columns split over a cluster
 *       of 4 (or 8) CTAs with the state in registers.
 *    0: the default: the path that measured faster on B200 for the workloads
 *       tried so far, currently 16.
 * The two paths round differently (their results agree within the library's
 * accuracy bounds, not bitwise). Process-wide. Returns KDA_ERR_SHAPE for any
 * other value (the setting is then unchanged).
 */
kda_status_t kda_set_path(int32_t path);

/*
 * kda_set_slice_columns -- value columns per CTA of the 16-token path.
 *
 * columns = 32 uses 4 CTAs per (sequence, head); 16 uses 8, which doubles the
 * SMs working on the same serial chains when there are few sequences and
 * heads. columns = 0 (the default) chooses per call: 16 when
 * num_seqs * num_heads * 4 is at most half the device's SM count, else 32.
 * Each column's arithmetic is the same either way, so the results are bitwise
 * identical. Process-wide. Returns KDA_ERR_SHAPE for any other value (the
 * setting is then unchanged).
 */
kda_status_t kda_set_slice_columns(int32_t columns);

/*
 * kda_set_schedule -- how the 16-token path maps (sequence, head) pairs onto
 * clusters.
 *   mode 1: one cluster per pair; the hardware starts each cluster when an
 *           earlier one has finished.
 *   mode 2: G persistent clusters, G = the number the device holds at once,
 *           capped at `clusters` when that is > 0, and at the number of pairs;
 *           cluster c runs the pairs c, c + G, c + 2G, ... (pair = sequence *
 *           num_heads + head) back to back, the next pair's operands being
 *           prepared while the previous one's last chunks run. A small cap
 *           makes every cluster take many pairs (testing).
 *   mode 0 (default): 2 with no cap when the pairs outnumber the resident
 *           clusters, else 1 (`clusters` is ignored).
 * Each pair's arithmetic is the same either way, so the results are bitwise
 * identical. Process-wide. Returns KDA_ERR_SHAPE for any other mode or a
 * negative `clusters` (the setting is then unchanged).
 */
kda_status_t kda_set_schedule(int32_t mode, int32_t clusters);

/*
 * kda_set_time_split -- the time-split prefill of kda_fwd (16-token path).
 *
 * A batch of ONE sequence (num_seqs = 1) with few heads leaves most SMs idle:
 * each head is one serial chain. The time split runs two parts of the
 * sequence at once: the first from the initial state, the second twice in
 * parallel -- from the zero state, and with v = 0 from the identity, which
 * gives the map from its (not yet known) start state to its outputs and end
 * state -- and then combines them (o_t += S_a^T o_M(t), S_T = M S_a + B; the
 * recurrence is linear in its initial state). The first part takes ~57 % of
 * the tokens on 16-column slices when the device has 16 * H SMs for the three
 * runs, else ~49 % on 32-column slices, so that the runs end together. It takes extra scratch from the
 * pool (about T/2 x H x 768 bytes plus three rings and three states) and two
 * helper streams (created once per device; the call stays ordered on
 * `stream`). Results agree with the unsplit path within the library's
 * accuracy bounds, not bitwise.
 *   mode 0 (default): split when num_seqs = 1, T >= 4096 and the device holds
 *                     all 3 * H clusters of the three launches at once;
 *   mode 1: never;   mode 2: whenever num_seqs = 1 and T >= 32 (testing).
 * kda_fwd_noalloc never splits. Process-wide. Returns KDA_ERR_SHAPE for any
 * other mode (the setting is then unchanged).
 */
kda_status_t kda_set_time_split(int32_t mode);

/*
 * kda_decode -- one decode step for a batch of B requests: each request's
 * per-head state advances by one token (the recurrence above with T = 1) in
 * place, and the token's output is written.
 *
 * The sources describe a fixed-size state per head as what makes long-context
 * decoding cheap (FlashKDA page, section "سياق Kimi Linear"); this is that
 * step for states kept resident in device memory between calls (for example a
 * serving engine's pool of request states).
 *
 * Tensors (B = requests, H = heads, P = state slots):
 *   q, k, v, out   bf16  [B, H, 128]     one token per request
 *   g              fp32  [B, H, 128]     precondition -5 <= g <= 0, as for kda_fwd
 *   beta           fp32  [B, H]
 *   state          fp32  [P, H, 128 (key), 128 (value)], contiguous; read and
 *                  written in place
 *   state_indices  int32 [B] on the device: the state slot of each request;
 *                  or NULL, meaning slot b for request b (then P >= B).
 *                  Slots of one call must be distinct (requests sharing a
 *                  slot race). A slot outside [0, P) skips its request (its
 *                  out row is not written) and sets KDA_DEVICE_BAD_STATE_INDEX
 *                  in the device status word.
 * Strides and alignment of the token tensors: as for kda_fwd (B in place of
 * T). state_indices must be 4-byte aligned. B = 0 is allowed (nothing runs).
 * Errors: KDA_ERR_NULL, KDA_ERR_DTYPE, KDA_ERR_SHAPE, KDA_ERR_STRIDE,
 * KDA_ERR_ALIGN, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA; nothing is enqueued on any
 * error. Allocates nothing. Returns KDA_OK once the work is enqueued.
 */
kda_status_t kda_decode(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v,
                        const kda_tensor_t* g, const kda_tensor_t* beta, float scale,
                        const kda_tensor_t* state, const int32_t* state_indices,
                        const kda_tensor_t* out, void* stream);

/*
 * kda_bwd -- gradients of the prefill (training): for a loss with gradient
 * dout = dLoss/do (and dfinal_state = dLoss/dS_final), the gradients of q, k,
 * v, g, beta and the initial state.
 *
 * The sources name only a Triton implementation that trains (page "Moonshot
 * AI … FlashKDA … (kucoin)"); this is the plain reverse-mode derivative of the
 * recurrence above, token by token:
 *   L = dLoss/dS_t;  L += scale q_t dO_t^T;  dq_t = scale S_t dO_t;
 *   with S' = Diag(exp g_t) S_{t-1}, u = v_t - S'^T k_t, lk = L^T k_t:
 *   dv_t = beta_t lk, dbeta_t = lk . u, dk_t = beta_t (L u - S' lk),
 *   dS' = L - beta_t k_t lk^T, dg_t = rowsum(dS' * S'), L <- Diag(exp g_t) dS'.
 *
 * Inputs: q, k, v, g, beta, scale, cu_seqlens, num_seqs, initial_state as for
 * kda_fwd (same layouts, strides and preconditions); dout bf16 [T, H, 128]
 * (strides as for kda_fwd's inputs); dfinal_state fp32 [N, H, 128, 128]
 * contiguous or NULL (zero).
 * Outputs (fp32, contiguous, written in full): dq, dk, dv, dg [T, H, 128];
 * dbeta [T, H]; dinitial_state [N, H, 128, 128] or NULL (not written). The
 * gradient of g is for the natural-log decay itself.
 * Scratch from the pool: a state checkpoint every 4 tokens (16 KiB per token
 * and head) and four partial sums of dq, dk, dg (6 KiB per token and head),
 * about 23 KB per token and head in all (T = 8192, H = 32: 6 GB). Results
 * are deterministic. Runs on the CUDA cores (rank-1 updates token by token): much
 * slower than kda_fwd. Errors as for kda_fwd; nothing is enqueued on any
 * error. Returns KDA_OK once the work is enqueued.
 */
kda_status_t kda_bwd(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v,
                     const kda_tensor_t* g, const kda_tensor_t* beta, float scale,
                     const int32_t* cu_seqlens, int32_t num_seqs, const kda_tensor_t* initial_state,
                     const kda_tensor_t* dout, const kda_tensor_t* dfinal_state,
                     const kda_tensor_t* dq, const kda_tensor_t* dk, const kda_tensor_t* dv,
                     const kda_tensor_t* dg, const kda_tensor_t* dbeta,
                     const kda_tensor_t* dinitial_state, void* stream);

/* Human-readable text of a status code (static storage, never NULL). */
const char* kda_status_string(kda_status_t status);

/* Text of the last CUDA error seen by this thread inside the library
 * (static thread-local storage; "" if none). */
const char* kda_last_cuda_error(void);

/*
 * kda_device_status -- the current device's status word.
 *
 * Bits (OR-ed over every kernel since the last reset):
 *   KDA_DEVICE_BAD_CU_SEQLENS  some cu_seqlens was not a non-decreasing
 *                              partition of [0, T) (those results are wrong)
 *   KDA_DEVICE_WAIT_TIMEOUT    a bounded in-kernel wait ran out of budget (the
 *                              kernel stopped early; its results are undefined)
 *   KDA_DEVICE_BAD_STATE_INDEX kda_decode met a state index outside [0, P)
 *                              (that request was skipped)
 * Writes the bits to *flags (synchronising with the device), clears them when
 * `reset` is non-zero, and returns KDA_ERR_DEVICE if any bit is set, else
 * KDA_OK (or KDA_ERR_NULL / KDA_ERR_CUDA).
 */
#define KDA_DEVICE_BAD_CU_SEQLENS 1u
#define KDA_DEVICE_WAIT_TIMEOUT 2u
#define KDA_DEVICE_BAD_STATE_INDEX 4u
kda_status_t kda_device_status(uint32_t* flags, int32_t reset);

/*
 * kda_wait_timeouts -- how many bounded in-kernel waits ran out of budget on
 * the current device since the last reset (0 for a healthy run). Every wait
 * inside the kernels (on a pipeline stage, on a peer CTA of the cluster) is
 * bounded; a wait that runs out increments this counter and makes its CTA
 * stop issuing work, so the GPU is never left hanging. Synchronises with the
 * device; resets the counter when `reset` is non-zero.
 */
kda_status_t kda_wait_timeouts(uint32_t* count, int32_t reset);

/* KDA_ABI_VERSION of the loaded library. */
int32_t kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
