// kda_fwd64.cuh -- chunk-64 Kimi Delta Attention forward (prefill) on tcgen05.
//
// Work decomposition
//   One thread-block cluster of four CTAs per (sequence, head). CTA 0 runs the
//   serial state recurrence over 64-token chunks with the whole 128 x 128
//   state (all value columns) in tensor memory; CTAs 1-3 prepare the chunks'
//   operands (chunk c is prepared by CTA 1 + c mod 3) and hand them over
//   through a ring of slots in global memory that stays resident in L2, with
//   remote mbarrier arrivals as the signals.
//
// Per chunk of C = 64 tokens (Gamma_i = inclusive cumulative log-decay inside
// the chunk, e_i = exp(g_i) per key channel, gamma = exp(Gamma_last)):
//   E_i = exp(Gamma_i),  F_i = exp(Gamma_last - Gamma_i)     (both in (0, 1])
//   A_ij   = sum_c k_ic k_jc exp(Gamma_ic - Gamma_jc)   (j < i),   L = diag(beta) A
//   Aqk_ij = sum_c q_ic k_jc exp(Gamma_ic - Gamma_jc)   (j <= i)
//   Tb = (I + L)^{-1} diag(beta),  W = Tb (k * E),  U = Tb V
//   Vnew = U - W S,   O = scale (Qd S + Aqk Vnew) with Qd = q * E,
//   S <- Diag(gamma) S + Kend^T Vnew with Kend = k * F.
// This is the chunk form of S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1}
// + beta_t k_t v_t^T, o_t = scale S_t^T q_t: the strictly lower triangular L
// collects the delta-rule corrections inside the chunk, and Vnew are the
// chunk's effective writes (page "Kimi K3 开源满月…", section "KDA 内核到底难在哪":
// chunks rewritten as small matrix products with one state chain between
// them; section "反转二": one fused kernel on tcgen05 and tensor memory with
// chunk intermediates kept on chip, larger chunks made safe by anchoring the
// exponents).
//
// Exponent anchoring. exp(Gamma_i - Gamma_j) cannot be factored as
// exp(Gamma_i) exp(-Gamma_j) over 64 tokens (g >= -5 gives exp(320)). The
// chunk is split into four 16-token blocks; for row block I the products use
// the anchor a_I = Gamma at the start of block I:
//   diagonal block:   (k_i exp(Gamma_i - a_I)) . (k_j exp(a_I - Gamma_j)),  exp(a_I - Gamma_j) <= e^80
//   block J < I:      (k_i exp(Gamma_i - a_I)) . (k_j exp(Gamma_endJ - Gamma_j) delta_JI)
// where delta_JI is the decay over the blocks strictly between J and I; every
// factor of the off-diagonal form is at most 1. One tcgen05 product with
// M = 128 (64 key rows and 64 query rows) and N = 160 (the four diagonal
// right-hand tiles and the six off-diagonal ones) yields A and Aqk at once.
//
// Chain step n (CTA 0), all products M = 128, N = 128 (value columns):
//   D[n%2] = [Tb ; 0] V                        (issued one step ahead)
//   D[n%2] += [-W ; Qd] S_n                    -> rows 0-63: Vnew, rows 64-127: O part
//   S_tmem += Kend^T Vnew                      (S_tmem holds Diag(gamma) S_n before)
//   D[n%2] += [* ; Aqk] Vnew                   -> rows 64-127: O
// with S_n and Vnew as bf16 copies in shared memory and the fp32 state kept
// in tensor memory. Tensor memory columns: D[0] 0-127, D[1] 128-255, S 256-383.

#pragma once

#include "kda_prims.cuh"

namespace kda {
namespace c64 {

constexpr int CH = 64;                 // tokens per chunk
constexpr int NPROD = 3;               // operand CTAs per cluster
constexpr int CLUSTER = NPROD + 1;
constexpr int RING = 6;                // ring slots per (sequence, head); multiple of NPROD
constexpr int NTHREADS = 352;          // warps 0-7 workers / readout, 8 tcgen05 issuer, 9 loads, 10 stores
constexpr int WARP_MMA = 8;
constexpr int WARP_LOAD = 9;
constexpr int WARP_STORE = 10;     // operand CTAs: bulk stores of a finished chunk to its ring slot
constexpr uint32_t TMEM_COLS = 512;
static_assert(RING % NPROD == 0, "a ring slot must always belong to the same operand CTA");

// ---- ring slot in global memory: the byte images the chain CTA copies in
constexpr uint32_t SL_AS = 0;          // 32 KB: [-W ; Qd] as an A tile (2 K-atoms x 128 rows x 128 B)
constexpr uint32_t SL_TB = 32768;      // 8 KB: Tb rows (64 x 128 B)
constexpr uint32_t SL_AQK = 40960;     // 8 KB: Aqk rows (64 x 128 B)
constexpr uint32_t SL_KT = 49152;      // 16 KB: Kend^T (128 key rows x 128 B of tokens)
constexpr uint32_t SL_G = 65536;       // 512 B: gamma fp32 [128]
constexpr uint32_t SLOT_BYTES = 66560;

// ---- chain CTA shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t E_AS = 0;           // early stage: [-W ; Qd] A tile
constexpr uint32_t E_AU = 32768;       //   [Tb ; 0] A tile (rows 64-127 stay zero)
constexpr uint32_t E_V = 49152;        //   V chunk, two 64-column TMA boxes (MN-major B)
constexpr uint32_t E_G = 65536;        //   gamma
constexpr uint32_t E_BYTES = 66560;
constexpr uint32_t C_TUV = 2 * E_BYTES;     // late stage: [* ; Aqk] A tile (16 KB)
constexpr uint32_t C_KT = C_TUV + 16384;    //   Kend^T A tile (16 KB)
constexpr uint32_t C_BS = C_KT + 16384;     // bf16 S_n, MN-major B (2 atoms x 128 key rows)
constexpr uint32_t C_BV = C_BS + 32768;     // bf16 Vnew, MN-major B (2 atoms x 64 token rows)
constexpr uint32_t C_BAR = C_BV + 16384;
// ---- operand CTA shared memory
constexpr uint32_t P_Q = 0, P_K = 16384, P_G = 32768, P_BETA = 65536;  // raw chunk (TMA)
constexpr uint32_t P_AI = 66560;       // 32 KB: [X ; Q] A tile; after the product: L (fp32) + Xt
constexpr uint32_t P_BI = P_AI + 32768;     // 40 KB: 160-row B tile; after the product: T, Tt (fp32)
constexpr uint32_t P_KE = P_BI + 40960;     // 16 KB: k * E, MN-major B (tokens x keys)
constexpr uint32_t P_AW = P_KE + 16384;     // 16 KB: [Tb ; 0] A tile
constexpr uint32_t P_GT = P_AW + 16384;     // per-block decay totals fp32 [4][128] + beta [64]
constexpr uint32_t P_ST = P_GT + 3072;      // staging: Qd rows (2 x 8 KB), Kend^T (16 KB), gamma (512 B)
constexpr uint32_t P_AQK = P_AI + 20480;    // staging of Aqk rows (8 KB) beside L and Xt
// -W rows are staged at P_BI (2 x 8 KB) once T is no longer needed; Tb rows are P_AW's first 8 KB
constexpr uint32_t LP = 68;            // fp32 row pitch of L, T, Tt (conflict-free float4 rows)
constexpr uint32_t BAR_BYTES = 512;
constexpr uint32_t SMEM_BYTES = C_BAR + BAR_BYTES + 1024;  // + alignment slack
static_assert(P_ST + 33280 <= C_BAR, "operand CTA layout fits below the barrier block");
static_assert(64 * LP * 4 + 48 * 16 * 4 <= P_AQK - P_AI, "Aqk staging beside L and Xt");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(64 * LP * 4 + 48 * 16 * 4 <= 32768 && 2 * 64 * LP * 4 <= 40960, "inverse scratch fits");

struct Bars {
  unsigned long long e_full[2], e_empty[2], l_full, l_empty;
  unsigned long long ms_done, ds_done, ov_done, vnew_ready, s_ready, o_read;
  unsigned long long slot_ready[RING];   // chain CTA: arrived by the slot's operand CTA
  unsigned long long slot_free[RING];    // operand CTA: arrived by the chain CTA's loader
  unsigned long long raw_full, raw_empty, gate_done, intra_done, tb_done, w_done;
  unsigned long long drained;            // the issuer's last commit (tensor memory idle)
  unsigned long long staged, staging_free;  // operand CTA: chunk outputs staged / stored
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= BAR_BYTES, "barrier block");

struct Params {
  const float* beta;
  const int32_t* cu;       // may be null: one sequence [0, T)
  const float* init;       // may be null
  __nv_bfloat16* out;
  float* fin;              // may be null
  unsigned char* ring;     // [num_seqs * H][RING] slots of SLOT_BYTES
  int64_t T;
  int64_t beta_st, beta_sh;   // element strides of beta over tokens and heads
  int64_t out_st, out_sh;     // element strides of out over tokens and heads
  int32_t H;
  float scale;
};

struct Maps {
  CUtensorMap q, k, g, v;  // q, k, g: box {128, 1, 64}; v: box {64, 1, 64}, 128-byte swizzle
};

// ------------------------------------------------------------- primitives
// Bounded waits. A wait gives up when its budget runs out or when another
// thread of the CTA has already given up (the CTA's abort flag); it then
// records the timeout, raises the flag and returns false, and the caller skips
// its remaining work. No thread ever blocks without a bound.
__device__ __forceinline__ bool wait_cta(unsigned long long* m, uint32_t parity, volatile int* abort_flag) {
  if (mbar_test_wait(m, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(m, parity)) return true;
    if ((i & 15u) == 0 && *abort_flag) return false;
    if ((i & 63u) == 0 && clock64() - t0 > kWaitCycles) {
      atomicAdd(&g_wait_timeouts, 1u);
      *abort_flag = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_cl(unsigned long long* m, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait_cl(m, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cl(m, parity)) return true;
    if ((i & 15u) == 0 && *abort_flag) return false;
    if ((i & 63u) == 0 && clock64() - t0 > kWaitCycles) {
      atomicAdd(&g_wait_timeouts, 1u);
      *abort_flag = 1;
      return false;
    }
  }
}

// K-major operand, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// MN-major operand, 128-byte swizzle: 64-element column atoms `lbo` bytes
// apart, 8-row K groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr, uint32_t lbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor: bf16 x bf16 -> fp32, A K-major, B K- or MN-major.
__host__ __device__ constexpr uint32_t idesc(int M, int N, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(unsigned long long* m) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(m))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive fp32 columns (one row per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// Byte offset of bf16 element (row, col) in a 128-byte-swizzled tile whose
// 64-column atoms are `atom` bytes apart (K-major: row = M/N index, col = K;
// MN-major: row = K index, col = M/N).
__host__ __device__ __forceinline__ uint32_t sw_off(uint32_t row, uint32_t col, uint32_t atom) {
  return (col >> 6) * atom + (row >> 3) * 1024u + (row & 7u) * 128u + ((((col & 63u) >> 3) ^ (row & 7u)) << 4) +
         ((col & 7u) << 1);
}
// Byte offset of the 16-byte chunk holding columns [8j, 8j + 8) of `row`.
__host__ __device__ __forceinline__ uint32_t sw_chunk(uint32_t row, uint32_t j, uint32_t atom) {
  return (j >> 3) * atom + (row >> 3) * 1024u + (row & 7u) * 128u + (((j & 7u) ^ (row & 7u)) << 4);
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}
__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Pair index of off-diagonal block (J, I), J < I, in the 160-row right-hand tile.
__host__ __device__ constexpr int pair_index(int J, int I) { return I * (I - 1) / 2 + J; }

// Row i (block Ii) of A (scaled by beta_i, strictly lower) or of Aqk (lower,
// diagonal included) takes the 16 columns of block J from the product tile
// that pairs row block IB with column block J.
template <int J, int IB>
__device__ __forceinline__ void take_block(float (&row)[64], const float (&v)[16], int Ii, int i, bool isq, float bi) {
  if (Ii != IB) return;
#pragma unroll
  for (int cc = 0; cc < 16; ++cc) {
    const int jx = 16 * J + cc;
    row[jx] = isq ? ((jx <= i) ? v[cc] : 0.f) : ((jx < i) ? bi * v[cc] : 0.f);
  }
}

// ================================================================== kernel
__global__ void __cluster_dims__(CLUSTER, 1, 1) __launch_bounds__(NTHREADS, 1)
    kda_fwd64_kernel(const Params p, const __grid_constant__ Maps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t rank = cluster_rank();
  Bars& bar = *reinterpret_cast<Bars*>(sm + C_BAR);  // same offset in every CTA (remote arrivals)
  volatile int* abort_flag = &bar.abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int h = blockIdx.y;
  const int seq = blockIdx.z;
  const int H = p.H;
  const int64_t T = p.T;
  int64_t t0 = 0, t1 = T;
  if (p.cu) {
    if (tid == 0 && rank == 0 && h == 0) check_bounds(p.cu, seq, static_cast<int>(gridDim.z), T);
    t0 = p.cu[seq];
    t1 = p.cu[seq + 1];
    t0 = t0 < 0 ? 0 : (t0 > T ? T : t0);
    t1 = t1 < t0 ? t0 : (t1 > T ? T : t1);
  }
  const int nch = static_cast<int>((t1 - t0 + CH - 1) / CH);
  unsigned char* ring = p.ring + (static_cast<size_t>(seq) * H + h) * RING * SLOT_BYTES;

  if (tid == 0) {
    if (rank == 0) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bar.e_full[s], 1);
        mbar_init(&bar.e_empty[s], 1);
      }
      mbar_init(&bar.l_full, 1);
      mbar_init(&bar.l_empty, 1);
      mbar_init(&bar.ms_done, 1);
      mbar_init(&bar.ds_done, 1);
      mbar_init(&bar.ov_done, 1);
      mbar_init(&bar.vnew_ready, 4);
      mbar_init(&bar.s_ready, 8);
      mbar_init(&bar.o_read, 4);
      for (int s = 0; s < RING; ++s) mbar_init(&bar.slot_ready[s], 1);
    } else {
      for (int s = 0; s < RING; ++s) mbar_init(&bar.slot_free[s], 1);
      mbar_init(&bar.raw_full, 1 + 32);
      mbar_init(&bar.raw_empty, 8);
      mbar_init(&bar.gate_done, 8);
      mbar_init(&bar.intra_done, 1);
      mbar_init(&bar.tb_done, 8);
      mbar_init(&bar.w_done, 1);
      mbar_init(&bar.staged, 8);
      mbar_init(&bar.staging_free, 1);
    }
    mbar_init(&bar.drained, 1);
    bar.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == WARP_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bar.tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // zero the tile halves that are never loaded: rows 64-127 of both [Tb ; 0]
  // tiles (chain) or of [Tb ; 0] (operand CTA), rows 0-63 of [* ; Aqk]
  if (rank == 0) {
    for (int i = tid; i < 3 * 512; i += NTHREADS) {
      const int part = i >> 9, w = i & 511;  // 512 x 16 B = 8 KB per part
      const uint32_t off = part == 0 ? E_AU + 8192 : part == 1 ? E_BYTES + E_AU + 8192 : C_TUV;
      st_shared_v4(sbase + off + 16u * w, make_uint4(0, 0, 0, 0));
    }
  } else {
    for (int i = tid; i < 512; i += NTHREADS) st_shared_v4(sbase + P_AW + 8192 + 16u * i, make_uint4(0, 0, 0, 0));
  }
  fence_proxy_async_shared();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  cluster_sync();  // every CTA's barriers exist before any remote arrive

  if (rank == 0) {
    // ================================================================ chain CTA
    if (warp == WARP_MMA) {
      if (lane == 0 && nch > 0) {
        constexpr uint32_t ID = idesc(128, 128, 1);
        const uint32_t tS = tmem + 256;
        bool ok = wait_cta(&bar.e_full[0], 0, abort_flag);
        tc_fence_after();
        auto issue_u = [&](int b) {  // D[b] = [Tb ; 0] V
          const uint32_t e = sbase + (b ? E_BYTES : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma(tmem + 128u * b, desc_k(e + E_AU + 32u * kk), desc_mn(e + E_V + 2048u * kk, 8192), ID, kk > 0);
        };
        if (ok) issue_u(0);
        for (int n = 0; n < nch && ok && !*abort_flag; ++n) {
          const int b = n & 1;
          const uint32_t e = sbase + (b ? E_BYTES : 0u);
          const uint32_t d = tmem + 128u * b;
          ok = wait_cta(&bar.s_ready, n & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          // Vnew / O part: D[b] += [-W ; Qd] S_n
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma(d, desc_k(e + E_AS + (kk >> 2) * 16384u + 32u * (kk & 3)), desc_mn(sbase + C_BS + 2048u * kk, 16384),
                 ID, 1);
          umma_commit(&bar.ms_done);
          umma_commit(&bar.e_empty[b]);
          ok = wait_cta(&bar.vnew_ready, n & 1, abort_flag) && wait_cta(&bar.l_full, n & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          // S_tmem += Kend^T Vnew
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma(tS, desc_k(sbase + C_KT + 32u * kk), desc_mn(sbase + C_BV + 2048u * kk, 8192), ID, 1);
          umma_commit(&bar.ds_done);
          // O rows: D[b] += [* ; Aqk] Vnew
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma(d, desc_k(sbase + C_TUV + 32u * kk), desc_mn(sbase + C_BV + 2048u * kk, 8192), ID, 1);
          umma_commit(&bar.ov_done);
          umma_commit(&bar.l_empty);
          // next chunk's U into the other accumulator, once its previous O rows were read
          if (n + 1 < nch) {
            ok = wait_cta(&bar.e_full[b ^ 1], ((n + 1) >> 1) & 1, abort_flag);
            if (ok && n >= 1) ok = wait_cta(&bar.o_read, (n - 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_u(b ^ 1);
          }
        }
        if (!ok) *abort_flag = 1;
        // every product issued here completes before tensor memory is freed
        umma_commit(&bar.drained);
        mbar_wait(&bar.drained, 0);
      }
    } else if (warp == WARP_LOAD) {
      if (lane == 0 && nch > 0) {
        auto load_early = [&](int n) -> bool {
          const int b = n & 1, s = n % RING;
          if (!wait_cta(&bar.e_empty[b], ((n >> 1) & 1) ^ 1, abort_flag)) return false;
          if (!wait_cl(&bar.slot_ready[s], (n / RING) & 1, abort_flag)) return false;
          fence_proxy_async_global();
          unsigned char* slot = ring + static_cast<size_t>(s) * SLOT_BYTES;
          unsigned char* e = sm + (b ? E_BYTES : 0u);
          mbar_arrive_expect_tx(&bar.e_full[b], 32768u + 8192u + 512u + 16384u);
          bulk_g2s(e + E_AS, slot + SL_AS, 32768u, &bar.e_full[b]);
          bulk_g2s(e + E_AU, slot + SL_TB, 8192u, &bar.e_full[b]);
          bulk_g2s(e + E_G, slot + SL_G, 512u, &bar.e_full[b]);
          const int tok = static_cast<int>(t0 + static_cast<int64_t>(n) * CH);
          tma_load_3d(e + E_V, &tm.v, 0, h, tok, &bar.e_full[b]);
          tma_load_3d(e + E_V + 8192, &tm.v, 64, h, tok, &bar.e_full[b]);
          return true;
        };
        auto load_late = [&](int n) -> bool {
          const int s = n % RING;
          if (!wait_cta(&bar.l_empty, (n & 1) ^ 1, abort_flag)) return false;
          unsigned char* slot = ring + static_cast<size_t>(s) * SLOT_BYTES;
          mbar_arrive_expect_tx(&bar.l_full, 8192u + 16384u);
          bulk_g2s(sm + C_TUV + 8192, slot + SL_AQK, 8192u, &bar.l_full);
          bulk_g2s(sm + C_KT, slot + SL_KT, 16384u, &bar.l_full);
          return true;
        };
        // last early / late load issued, and last whose landing this warp saw
        int ei = -1, li = -1, seen = -1;
        bool ok = load_early(0);
        if (ok) ei = 0;
        for (int n = 0; n < nch && ok && !*abort_flag; ++n) {
          ok = load_late(n);
          if (ok) li = n;
          if (ok && n + 1 < nch) {
            ok = load_early(n + 1);
            if (ok) ei = n + 1;
          }
          // the slot's bytes have landed: give it back to its operand CTA
          if (ok) ok = wait_cta(&bar.e_full[n & 1], (n >> 1) & 1, abort_flag) && wait_cta(&bar.l_full, n & 1, abort_flag);
          if (ok) seen = n;
          if (ok) mbar_arrive_remote_relaxed(&bar.slot_free[n % RING], 1u + static_cast<uint32_t>(n % NPROD));
        }
        if (!ok) *abort_flag = 1;
        // After an abort, copies this warp issued may still be landing in
        // shared memory. They read global memory only, so they complete: wait
        // for each (bounded, not abortable) before the CTA may exit.
        for (int i = seen + 1; i <= ei; ++i) mbar_wait(&bar.e_full[i & 1], (i >> 1) & 1);
        for (int i = seen + 1; i <= li; ++i) mbar_wait(&bar.l_full, i & 1);
      }
    } else if (warp < 8) {
      // ======================================================= readout warps
      const int qd = warp & 3, hf = warp >> 2;
      const int r = 32 * qd + lane;        // tensor-memory lane = row
      const uint32_t lane_off = static_cast<uint32_t>(32 * qd) << 16;
      const uint32_t c0 = 64u * hf;
      const size_t sidx = (static_cast<size_t>(seq) * H + h) * D * D;
      float s[64];
      {
        const float* src = p.init ? p.init + sidx + static_cast<size_t>(r) * D + c0 : nullptr;
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          const float4 v4 = src ? __ldg(reinterpret_cast<const float4*>(src + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
          s[j] = v4.x; s[j + 1] = v4.y; s[j + 2] = v4.z; s[j + 3] = v4.w;
        }
      }
      // bf16 S (B operand) and Diag(gamma) S (tensor memory) for step n
      auto publish_state = [&](int n) -> bool {
        if (!__all_sync(0xffffffffu, wait_cta(&bar.e_full[n & 1], (n >> 1) & 1, abort_flag))) return false;
        const float gm = reinterpret_cast<const float*>(sm + (n & 1 ? E_BYTES : 0u) + E_G)[r];
#pragma unroll
        for (int j = 0; j < 8; ++j) st_shared_v4(sbase + C_BS + sw_chunk(r, 8u * hf + j, 16384), pack8(&s[8 * j]));
        float v[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = s[32 * half + j] * gm;
          tmem_st32(tmem + lane_off + 256u + c0 + 32u * half, v);
        }
        tc_wait_st();
        fence_proxy_async_shared();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.s_ready);
        return true;
      };
      bool ok = true;
      if (nch == 0) {
        if (p.fin) {
          float* dst = p.fin + sidx + static_cast<size_t>(r) * D + c0;
#pragma unroll
          for (int j = 0; j < 64; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
        }
      } else {
        ok = publish_state(0);
      }
      for (int n = 0; n < nch && ok && !*abort_flag; ++n) {
        const int b = n & 1;
        const uint32_t dcol = tmem + lane_off + 128u * b + c0;
        const int64_t cs = t0 + static_cast<int64_t>(n) * CH;
        const int m = static_cast<int>((t1 - cs) < CH ? (t1 - cs) : CH);
        if (qd < 2) {
          // ---- Vnew rows: bf16 B operand of the step's second products
          if (!(ok = __all_sync(0xffffffffu, wait_cta(&bar.ms_done, n & 1, abort_flag)))) break;
          tc_fence_after();
          float v[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld32(dcol + 32u * half, v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(sbase + C_BV + sw_chunk(r, 8u * hf + 4u * half + j, 8192), pack8(&v[8 * j]));
          }
          fence_proxy_async_shared();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.vnew_ready);
        }
        // ---- state rows: S_{n+1}
        if (!(ok = __all_sync(0xffffffffu, wait_cta(&bar.ds_done, n & 1, abort_flag)))) break;
        tc_fence_after();
        {
          float v[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld32(tmem + lane_off + 256u + c0 + 32u * half, v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) s[32 * half + j] = v[j];
          }
        }
        if (n + 1 < nch) {
          if (!(ok = publish_state(n + 1))) break;
        } else if (p.fin) {
          float* dst = p.fin + sidx + static_cast<size_t>(r) * D + c0;
#pragma unroll
          for (int j = 0; j < 64; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
        }
        if (qd >= 2) {
          // ---- O rows
          if (!(ok = __all_sync(0xffffffffu, wait_cta(&bar.ov_done, n & 1, abort_flag)))) break;
          tc_fence_after();
          const int i = r - 64;
          __nv_bfloat16* dst = p.out + (cs + i) * p.out_st + static_cast<int64_t>(h) * p.out_sh + c0;
          float v[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld32(dcol + 32u * half, v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= p.scale;
            if (i < m) {
#pragma unroll
              for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(dst + 32 * half + 8 * j) = pack8(&v[8 * j]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.o_read);
        }
      }
      if (!ok) *abort_flag = 1;
    }
  } else {
    // ============================================================= operand CTAs
    const int pr = static_cast<int>(rank) - 1;
    const int nmine = nch > pr ? (nch - pr + NPROD - 1) / NPROD : 0;
    float* gt = reinterpret_cast<float*>(sm + P_GT);          // [4][128] block totals
    float* bet = reinterpret_cast<float*>(sm + P_GT + 2048);  // [64] beta
    if (warp == WARP_LOAD) {
      int issued = -1;  // last raw chunk whose loads this warp issued
      for (int j = 0; j < nmine && !*abort_flag; ++j) {
        const int c = pr + NPROD * j;
        const int64_t cs = t0 + static_cast<int64_t>(c) * CH;
        if (!wait_cta(&bar.raw_empty, (j & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        issued = j;
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar.raw_full, 16384u + 16384u + 32768u);
          const int tok = static_cast<int>(cs);
          tma_load_3d(sm + P_Q, &tm.q, 0, h, tok, &bar.raw_full);
          tma_load_3d(sm + P_K, &tm.k, 0, h, tok, &bar.raw_full);
          tma_load_3d(sm + P_G, &tm.g, 0, h, tok, &bar.raw_full);
        }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int i = lane + 32 * rr;
          const bool ok = cs + i < t1;
          cp_async4(sm + P_BETA + 4 * i, p.beta + (ok ? (cs + i) * p.beta_st + h * p.beta_sh : 0), ok ? 4u : 0u);
        }
        cp_async_arrive(&bar.raw_full);
      }
      // the last issued chunk's copies (global reads, so they complete) have
      // landed before the CTA may exit, also after an abort; earlier chunks'
      // phases completed before raw_empty let the next one be issued
      if (issued >= 0) mbar_wait(&bar.raw_full, issued & 1);
    } else if (warp == WARP_MMA) {
      if (lane == 0) {
        bool ok = true;
        for (int j = 0; j < nmine && ok && !*abort_flag; ++j) {
          ok = wait_cta(&bar.gate_done, j & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          constexpr uint32_t IDI = idesc(128, 160, 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma(tmem, desc_k(sbase + P_AI + (kk >> 2) * 16384u + 32u * (kk & 3)),
                 desc_k(sbase + P_BI + (kk >> 2) * 20480u + 32u * (kk & 3)), IDI, kk > 0);
          umma_commit(&bar.intra_done);
          ok = wait_cta(&bar.tb_done, j & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          constexpr uint32_t IDW = idesc(128, 128, 1);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma(tmem + 256, desc_k(sbase + P_AW + 32u * kk), desc_mn(sbase + P_KE + 2048u * kk, 8192), IDW, kk > 0);
          umma_commit(&bar.w_done);
        }
        if (!ok) *abort_flag = 1;
        umma_commit(&bar.drained);
        mbar_wait(&bar.drained, 0);
      }
    } else if (warp == WARP_STORE) {
      // ============================================================ store warp
      // A staged chunk goes to its ring slot as eight bulk copies; the staging
      // is free again once they have read it, and the chain CTA is told once
      // they have completed.
      if (lane == 0) {
        bool ok = true;
        for (int j = 0; j < nmine && ok && !*abort_flag; ++j) {
          const int c = pr + NPROD * j;
          const int slot_i = c % RING;
          unsigned char* slot = ring + static_cast<size_t>(slot_i) * SLOT_BYTES;
          ok = wait_cta(&bar.staged, j & 1, abort_flag) &&
               wait_cl(&bar.slot_free[slot_i], ((c / RING) & 1) ^ 1, abort_flag);
          if (!ok) break;
          bulk_s2g_nc(slot + SL_AS, sm + P_BI, 8192u);                  // -W rows, key atom 0
          bulk_s2g_nc(slot + SL_AS + 8192, sm + P_ST, 8192u);           // Qd rows, key atom 0
          bulk_s2g_nc(slot + SL_AS + 16384, sm + P_BI + 8192, 8192u);   // -W rows, key atom 1
          bulk_s2g_nc(slot + SL_AS + 24576, sm + P_ST + 8192, 8192u);   // Qd rows, key atom 1
          bulk_s2g_nc(slot + SL_TB, sm + P_AW, 8192u);
          bulk_s2g_nc(slot + SL_AQK, sm + P_AQK, 8192u);
          bulk_s2g_nc(slot + SL_KT, sm + P_ST + 16384, 16384u);
          bulk_s2g_nc(slot + SL_G, sm + P_ST + 32768, 512u);
          bulk_commit();
          bulk_wait_read<0>();
          mbar_arrive(&bar.staging_free);
          bulk_wait<0>();
          // the slot's bytes are written: make them visible to the cluster, then signal
          fence_proxy_async_global();
          fence_acq_rel_cluster();
          mbar_arrive_remote_relaxed(&bar.slot_ready[slot_i], 0u);
        }
        if (!ok) *abort_flag = 1;
      }
    } else {
      // ================================================= worker warps (256 threads)
      const int pp = tid & 63;        // channel pair: channels 2pp, 2pp + 1
      const int I = tid >> 6;         // 16-token block
      const uint32_t cA = 2u * pp;
      float* L = reinterpret_cast<float*>(sm + P_AI);                 // [64][LP]
      float* Xt = reinterpret_cast<float*>(sm + P_AI + 64 * LP * 4);  // [48][16]
      float* Tm = reinterpret_cast<float*>(sm + P_BI);                // [64][LP]
      float* Tt = reinterpret_cast<float*>(sm + P_BI + 64 * LP * 4);  // [64][LP], transposed
      bool ok = true;
      // Every iteration passes the same named barriers in every warp; after a
      // failed wait a warp skips its work (ok is warp-uniform) but not the barriers.
      for (int j = 0; j < nmine; ++j) {
        const int c = pr + NPROD * j;
        const int64_t cs = t0 + static_cast<int64_t>(c) * CH;
        const int m = static_cast<int>((t1 - cs) < CH ? (t1 - cs) : CH);
        ok = ok && wait_cta(&bar.raw_full, j & 1, abort_flag) && wait_cta(&bar.staging_free, (j & 1) ^ 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        // ---------------------------------------------------------- gates
        // Per thread: channels cA, cA + 1 over the 16 tokens of block I.
        // Px: decay from the block start through token jj (inclusive);
        // Sx: decay after token jj to the block end (exclusive). Rows past
        // the sequence end get e = 1 and k = q = 0.
        float Px[16], Py[16], Sx[16], Sy[16];
        auto ldk = [&](int jj) -> float2 {
          const int i = 16 * I + jj;
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sm + P_K + (i * D + cA) * 2));
          return i < m ? f : make_float2(0.f, 0.f);
        };
        auto ldq = [&](int jj) -> float2 {
          const int i = 16 * I + jj;
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sm + P_Q + (i * D + cA) * 2));
          return i < m ? f : make_float2(0.f, 0.f);
        };
        if (ok) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int i = 16 * I + jj;
            const float2 gg = *reinterpret_cast<const float2*>(sm + P_G + (i * D + cA) * 4);
            Px[jj] = i < m ? __expf(gg.x) : 1.f;  // e_i for now
            Py[jj] = i < m ? __expf(gg.y) : 1.f;
          }
          float ax = 1.f, ay = 1.f;
#pragma unroll
          for (int jj = 15; jj >= 0; --jj) {
            Sx[jj] = ax;
            Sy[jj] = ay;
            ax *= Px[jj];
            ay *= Py[jj];
          }
          ax = 1.f;
          ay = 1.f;
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            ax *= Px[jj];
            ay *= Py[jj];
            Px[jj] = ax;
            Py[jj] = ay;
          }
          if (pp == 0) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) bet[16 * I + jj] = reinterpret_cast<const float*>(sm + P_BETA)[16 * I + jj];
          }
          gt[I * 128 + cA] = Px[15];
          gt[I * 128 + cA + 1] = Py[15];
          const float rgx = __frcp_rn(Px[15]), rgy = __frcp_rn(Py[15]);
          // block-local tiles: X = k Px and Q = q Px (rows 0-63 / 64-127 of the
          // A tile), diagonal right-hand rows k exp(a_I - Gamma) = k Sx / gamma_I
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const uint32_t i = 16 * I + jj;
            const float2 kf = ldk(jj), qf = ldq(jj);
            *reinterpret_cast<uint32_t*>(sm + P_AI + sw_off(i, cA, 16384)) = pack_bf16(kf.x * Px[jj], kf.y * Py[jj]);
            *reinterpret_cast<uint32_t*>(sm + P_AI + sw_off(64 + i, cA, 16384)) = pack_bf16(qf.x * Px[jj], qf.y * Py[jj]);
            *reinterpret_cast<uint32_t*>(sm + P_BI + sw_off(i, cA, 20480)) =
                pack_bf16(kf.x * Sx[jj] * rgx, kf.y * Sy[jj] * rgy);
          }
        }
        named_bar(1, 256);  // block totals of every block are in gt
        if (ok) {
          float gx[4], gy[4];
#pragma unroll
          for (int K = 0; K < 4; ++K) {
            gx[K] = gt[K * 128 + cA];
            gy[K] = gt[K * 128 + cA + 1];
          }
          float prex = 1.f, prey = 1.f, postx = 1.f, posty = 1.f;
#pragma unroll
          for (int K = 0; K < 4; ++K) {
            if (K < I) { prex *= gx[K]; prey *= gy[K]; }
            if (K > I) { postx *= gx[K]; posty *= gy[K]; }
          }
          // off-diagonal right-hand rows: block J = I against every later block I2
#pragma unroll
          for (int I2 = 1; I2 < 4; ++I2) {
            if (I2 <= I) continue;
            float dx = 1.f, dy = 1.f;
#pragma unroll
            for (int K = 0; K < 4; ++K)
              if (K > I && K < I2) { dx *= gx[K]; dy *= gy[K]; }
            const uint32_t row0 = 64u + 16u * pair_index(I, I2);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const float2 kf = ldk(jj);
              *reinterpret_cast<uint32_t*>(sm + P_BI + sw_off(row0 + jj, cA, 20480)) =
                  pack_bf16(kf.x * Sx[jj] * dx, kf.y * Sy[jj] * dy);
            }
          }
          // k E (E from the chunk start, B operand of W); staged Qd rows
          // (rows 64-127 of the [-W ; Qd] tile: half-atom images of 8 KB)
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const uint32_t i = 16 * I + jj;
            const float2 kf = ldk(jj), qf = ldq(jj);
            *reinterpret_cast<uint32_t*>(sm + P_KE + sw_off(i, cA, 8192)) =
                pack_bf16(kf.x * Px[jj] * prex, kf.y * Py[jj] * prey);
            *reinterpret_cast<uint32_t*>(sm + P_ST + sw_off(i, cA, 8192)) =
                pack_bf16(qf.x * Px[jj] * prex, qf.y * Py[jj] * prey);
          }
          // staged Kend^T rows (keys cA, cA + 1; tokens of block I) and gamma
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float kex[8], key[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const float2 kf = ldk(8 * hh + x);
              kex[x] = kf.x * Sx[8 * hh + x] * postx;
              key[x] = kf.y * Sy[8 * hh + x] * posty;
            }
            st_shared_v4(sbase + P_ST + 16384 + sw_chunk(cA, 2u * I + hh, 0), pack8(kex));
            st_shared_v4(sbase + P_ST + 16384 + sw_chunk(cA + 1, 2u * I + hh, 0), pack8(key));
          }
          if (I == 0) {
            *reinterpret_cast<float2*>(sm + P_ST + 32768 + 4 * cA) =
                make_float2(gx[0] * gx[1] * gx[2] * gx[3], gy[0] * gy[1] * gy[2] * gy[3]);
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar.raw_empty);  // raw inputs are no longer read
            mbar_arrive(&bar.gate_done);
          }
        }
        // --------------------------------------------- A and Aqk from tensor memory
        ok = ok && wait_cta(&bar.intra_done, j & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (ok && warp < 4) {
          const int rr = 32 * warp + lane;  // tensor-memory lane
          const int i = rr & 63;
          const int Ii = i >> 4;
          const bool isq = rr >= 64;
          const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16);
          const float bi = bet[i];
          float row[64];
#pragma unroll
          for (int jx = 0; jx < 64; ++jx) row[jx] = 0.f;
          // blocks (J, I) with J <= I; warp parity selects I in {0, 1} or {2, 3}
          float v[16];
          if ((warp & 1) == 0) {
            tmem_ld16(ta + 0, v); tc_wait_ld(); take_block<0, 0>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 16, v); tc_wait_ld(); take_block<1, 1>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 64 + 16 * pair_index(0, 1), v); tc_wait_ld(); take_block<0, 1>(row, v, Ii, i, isq, bi);
          } else {
            tmem_ld16(ta + 32, v); tc_wait_ld(); take_block<2, 2>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 48, v); tc_wait_ld(); take_block<3, 3>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 64 + 16 * pair_index(0, 2), v); tc_wait_ld(); take_block<0, 2>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 64 + 16 * pair_index(1, 2), v); tc_wait_ld(); take_block<1, 2>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 64 + 16 * pair_index(0, 3), v); tc_wait_ld(); take_block<0, 3>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 64 + 16 * pair_index(1, 3), v); tc_wait_ld(); take_block<1, 3>(row, v, Ii, i, isq, bi);
            tmem_ld16(ta + 64 + 16 * pair_index(2, 3), v); tc_wait_ld(); take_block<2, 3>(row, v, Ii, i, isq, bi);
          }
          if (isq) {
#pragma unroll
            for (int jc = 0; jc < 8; ++jc) st_shared_v4(sbase + P_AQK + sw_chunk(i, jc, 0), pack8(&row[8 * jc]));
          } else {
#pragma unroll
            for (int jx = 0; jx < 64; jx += 4)
              *reinterpret_cast<float4*>(L + i * LP + jx) = make_float4(row[jx], row[jx + 1], row[jx + 2], row[jx + 3]);
          }
        }
        tc_fence_before();
        // zero T and Tt (the parts above the diagonal must read as 0)
        for (int x = tid; x < 2 * 64 * static_cast<int>(LP) / 4; x += 256)
          reinterpret_cast<float4*>(Tm)[x] = make_float4(0.f, 0.f, 0.f, 0.f);
        named_bar(1, 256);
        // ------------------------------------ T = (I + L)^{-1}: diagonal blocks
        // One thread per (block, column): forward substitution over the block's
        // 16 rows, two partial sums per row.
        if (ok && tid < 64) {
          const int Ib = tid >> 4, cc = tid & 15, base = 16 * Ib;
          float x[16];
#pragma unroll
          for (int rr = 0; rr < 16; ++rr) {
            const float* lr = L + (base + rr) * LP + base;
            float a0 = (rr == cc) ? 1.f : 0.f, a1 = 0.f;
#pragma unroll
            for (int mm = 0; mm < rr; ++mm) {
              if (mm & 1) a1 = fmaf(-lr[mm], x[mm], a1);
              else a0 = fmaf(-lr[mm], x[mm], a0);
            }
            x[rr] = a0 + a1;
          }
#pragma unroll
          for (int rr = 0; rr < 16; ++rr) {
            Tm[(base + rr) * LP + base + cc] = x[rr];
            Tt[(base + cc) * LP + base + rr] = x[rr];
          }
        }
        named_bar(1, 256);
        // ---------------- off-diagonal blocks: T_IJ = -T_II sum_{J<=K<I} L_IK T_KJ
        // Block row Ib at a time. Thread (row ir, column slot csl) owns the
        // columns csl + 16 q (q < Ib): independent sums share each L / T row load.
        {
          const int ir = tid & 15, csl = tid >> 4;
          for (int Ib = 1; Ib < 4; ++Ib) {
            const int i = 16 * Ib + ir;
            if (ok) {
              float acc[3] = {0.f, 0.f, 0.f};
              for (int mm = 0; mm < 16 * Ib; mm += 4) {
                const float4 l4 = *reinterpret_cast<const float4*>(L + i * LP + mm);
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                  if (q < Ib) {
                    const float4 t4 = *reinterpret_cast<const float4*>(Tt + (csl + 16 * q) * LP + mm);
                    acc[q] = fmaf(l4.x, t4.x, fmaf(l4.y, t4.y, fmaf(l4.z, t4.z, fmaf(l4.w, t4.w, acc[q]))));
                  }
                }
              }
#pragma unroll
              for (int q = 0; q < 3; ++q)
                if (q < Ib) Xt[(csl + 16 * q) * 16 + ir] = acc[q];
            }
            named_bar(1, 256);
            if (ok) {
              float acc[3] = {0.f, 0.f, 0.f};
#pragma unroll
              for (int mm = 0; mm < 16; mm += 4) {
                const float4 t4 = *reinterpret_cast<const float4*>(Tm + i * LP + 16 * Ib + mm);
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                  if (q < Ib) {
                    const float4 x4 = *reinterpret_cast<const float4*>(Xt + (csl + 16 * q) * 16 + mm);
                    acc[q] = fmaf(t4.x, x4.x, fmaf(t4.y, x4.y, fmaf(t4.z, x4.z, fmaf(t4.w, x4.w, acc[q]))));
                  }
                }
              }
#pragma unroll
              for (int q = 0; q < 3; ++q) {
                if (q < Ib) {
                  const int jcol = csl + 16 * q;
                  Tm[i * LP + jcol] = -acc[q];
                  Tt[jcol * LP + i] = -acc[q];
                }
              }
            }
            named_bar(1, 256);
          }
        }
        // ------------------------------------------- Tb = T diag(beta), bf16
        if (ok) {
          const int i = tid >> 2, q4 = tid & 3;
          float tb[16];
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) tb[cc] = Tm[i * LP + 16 * q4 + cc] * bet[16 * q4 + cc];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) st_shared_v4(sbase + P_AW + sw_chunk(i, 2u * q4 + hh, 0), pack8(&tb[8 * hh]));
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(&bar.tb_done);
        // ------------------------------------------------------- -W rows
        ok = ok && wait_cta(&bar.w_done, j & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        named_bar(1, 256);  // T and Tt are dead: -W is staged over them
        if (ok && (warp & 3) < 2) {
          const int qd = warp & 3, hf = warp >> 2;
          const int i = 32 * qd + lane;
          const uint32_t ta = tmem + (static_cast<uint32_t>(32 * qd) << 16) + 256u + 64u * hf;
          float v[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld32(ta + 32u * half, v);
            tc_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = -v[x];
#pragma unroll
            for (int jc = 0; jc < 4; ++jc)
              st_shared_v4(sbase + P_BI + 8192u * hf + sw_chunk(i, 4u * half + jc, 0), pack8(&v[8 * jc]));
          }
        }
        tc_fence_before();
        fence_proxy_async_shared();
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(&bar.staged);
        named_bar(1, 256);
      }
      if (!ok) *abort_flag = 1;
    }
  }
  // every role is done with tensor memory and with its peers' barriers
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == WARP_MMA) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  __syncwarp();
  cluster_sync();
}

}  // namespace c64
}  // namespace kda
