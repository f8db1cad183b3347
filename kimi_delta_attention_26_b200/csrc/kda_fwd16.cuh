// kda_fwd16.cuh -- chunk-16 Kimi Delta Attention forward (prefill) on mma.sync.
//
// Work decomposition
//   One thread-block cluster per (sequence, head): one CTA per value slice of
//   NS columns (NS = 32: four CTAs; NS = 16, for few sequences and heads:
//   eight). Columns of the state evolve independently (the recurrence
//   multiplies S only from the left), so the slices' state chains never
//   exchange data. What they share is the chunk-local work on keys, queries
//   and gates, which is identical for every slice: CTA n mod (cluster size)
//   produces the shared operands of chunk n once, stores them to an
//   L2-resident ring in global memory and signals every CTA of the cluster
//   with remote mbarrier arrivals; every CTA then pulls the chunk with one
//   bulk copy.
//
//   Warp roles inside a CTA (warp w issues on sub-partition w mod 4):
//     0-1   chain:  the serial state recurrence of this CTA's value slice (warp 0
//                   only when NS = 16). Warp w
//                   owns S^T[16 value columns x 128 keys] in mma.sync accumulator
//                   registers for the whole sequence and computes X, Vnew, O and
//                   the state update of those columns; it shares nothing with
//                   the other chain warp.
//     2,3,6,7 gate: (producer) two key channels x eight tokens per thread: decay
//                   factors and the bf16 operand tiles of the chunks this CTA owns.
//     4     pload:  (producer) TMA loads of q, k, g (and beta) for owned chunks.
//     5     cload:  (consumer) bulk-loads every chunk's shared operands from the
//                   ring and the value slice with TMA, in order, for the chain.
//     10    mma:    (producer) A = Kd KR^T and Aqk = Qd KR^T, 16 x 16 each, then
//                   T = (I + L)^{-1} by forward substitution and T diag(beta).
//     11    store:  (producer) bulk-stores a finished chunk to its ring slot and
//                   signals the cluster.
//     8     notify: (consumer) relays each landed stage to the chain warps
//                   through hardware named barriers and returns the ring slot
//                   to its producer. When NS = 16 this role runs on warp 1 (the
//                   unused second chain warp), off the chain's sub-partition.
//     9     bounds: records a cu_seqlens that is not a partition of [0, T)
//                   in the device status word (rank 0 of head 0's clusters).
//
// Per chunk of C = 16 tokens, with Gamma_i the inclusive cumulative log-decay
// inside the chunk (e_i = exp(g_i) per channel):
//   E_i = prod_{s<=i} e_s = exp(Gamma_i),  F_i = prod_{s>i} e_s = exp(Gamma_last - Gamma_i)
//   Kd = -k*E,  Qd = q*E,  KR = k*F/gamma = k*exp(-Gamma),  Kend = k*F,  gamma = E_last
//   A   = tril(k E (k/E)^T, -1) = -tril(Kd KR^T, -1),  L = diag(beta) A,  Aqk = tril(Qd KR^T)
//   Tb  = (I + L)^{-1} diag(beta)
//   X   = V + Kd S  (= V - k*E S),   Vnew = Tb X       (the chunk's delta-rule writes)
//   O   = scale (Qd S + Aqk Vnew)
//   S  <- Diag(gamma) S + Kend^T Vnew
// All factors stay within [e^-80, e^80] because -5 <= g <= 0 and a chunk has 16
// tokens: the bound that lets FlashKDA keep 16-token causal blocks on dense
// tensor-core products (page "Kimi K3 开源满月…", section "KDA 内核到底难在哪":
// 16-token chunks, lower_bound = -5). The chain works on transposes,
//   X^T = V^T + S^T Kd^T,  Vnew^T = X^T Tb^T,  S^T <- S^T Diag(gamma) + Vnew^T Kend,
//   O^T = scale (S^T Qd^T + Vnew^T Aqk^T),
// so that every product takes the register-resident state (or X, Vnew) as its
// A operand and a shared-memory tile as its B operand.
//
// Tensor cores: mma.sync m16n8k16 (bf16 in, fp32 accumulate). On this part a
// dependent m16n8k16 completes in ~21 cycles while a tcgen05.mma of the shapes
// this recurrence has (M <= 128, N <= 128, K = 16) costs ~90 cycles of issue
// plus a ~250-cycle commit/mbarrier round trip; the chain is a serial sequence
// of such small products, so it stays on the synchronous path.

#pragma once

#include "kda_prims.cuh"

namespace kda {

constexpr int C = 16;             // chunk length (tokens)
// Value columns per CTA (NS) is a template parameter of the kernel: 32 (four
// CTAs per (sequence, head), two chain warps each) or, when that grid would
// leave most SMs idle, 16 (eight CTAs, one chain warp each).
constexpr int RING = 16;          // ring slots per (sequence, head); multiple of the cluster size
constexpr int PRSTAGE = 2;        // producer raw-input stages
constexpr int PSTAGE = 3;         // producer operand stages
constexpr int CSTAGE = 6;         // consumer stages (cload -> chain)
// Warp w issues on sub-partition w mod 4. The two chain warps get partitions 0
// and 1 with only the light load and notify warps beside them; the gate, mma
// and store warps, which burst through ALU and shared-memory work, share
// partitions 2 and 3. Warp 9 only checks the sequence bounds once. (Measured:
// a per-chunk helper beside a chain warp costs it time, so with one chain warp
// the notify role moves to partition 1.)
constexpr int MAX_CHAIN = 2;      // chain warps 0 (and 1), 16 value columns each
constexpr int NGATE = 4;          // gate warps 2, 3, 6, 7
constexpr int WARP_PLOAD = 4;
constexpr int WARP_CLOAD = 5;
// relays stage completion to the chain warps
template <int NS>
__host__ __device__ constexpr int notify_warp() { return NS == 16 ? 1 : 8; }
constexpr int WARP_MMA = 10;      // also solves (I + L)^{-1}
constexpr int WARP_STORE = 11;
constexpr int NTHREADS = 12 * 32;
__host__ __device__ constexpr bool is_gate_warp(int w) { return (w & 3) >= 2 && w < 8; }
__host__ __device__ constexpr int gate_warp_index(int w) { return (w & 1) + ((w >> 2) << 1); }

// Hardware named barriers: 0 is the CTA-wide one, 1 the gate group's, and
// 2 + s tells the chain warps that consumer stage s has landed (the chain
// warps and the notify warp meet there; one barrier for both chain warps
// measured faster than one per warp).
constexpr int BAR_GATE = 1;
constexpr int BAR_FULL0 = 2;
static_assert(BAR_FULL0 + CSTAGE <= 16, "named barrier ids");
static_assert(RING % (D / 16) == 0, "a ring slot must always belong to the same producer CTA");

// Padded row pitches: 272 B and 48 B rows keep 8-row ldmatrix reads on distinct banks.
constexpr int LDK = D + 8;
constexpr int LDC = C + 8;

// Position of key channel c's decay in Ops::gam: a chain lane with quad index
// tq needs channels 8t + 2tq and 8t + 2tq + 1 (t = 0..15), so those 32 sit in
// one 160-byte row (rows on distinct banks), read with eight 16-byte loads.
__host__ __device__ constexpr int gamma_index(int c) { return ((c >> 1) & 3) * 40 + 2 * (c >> 3) + (c & 1); }

// Raw inputs of one owned chunk, as the TMA boxes land (beta by 4-byte copies).
struct __align__(128) RawStage {
  __nv_bfloat16 q[C][D];
  __nv_bfloat16 k[C][D];
  float g[C][D];
  float beta[C];
  float pad_[32 - C];
};
constexpr uint32_t kRawBytes = C * D * 2 * 2 + C * D * 4;  // bytes the TMA boxes bring

// Shared operands of one chunk; byte-for-byte the layout of a ring slot.
struct __align__(128) Ops {
  __nv_bfloat16 kd[C][LDK];   // -k * exp(Gamma)
  __nv_bfloat16 qd[C][LDK];   //  q * exp(Gamma)
  __nv_bfloat16 ke[C][LDK];   //  k * exp(Gamma_last - Gamma)
  __nv_bfloat16 tb[C][LDC];   //  (I + L)^{-1} diag(beta)
  __nv_bfloat16 aqk[C][LDC];  //  causal Qd KR^T
  float gam[4][40];           //  exp(Gamma_last), permuted for the chain (gamma_index)
};
constexpr uint32_t kSlotBytes = sizeof(Ops);

struct __align__(128) ProdStage {
  Ops ops;
  __nv_bfloat16 kr[C][LDK];   // k * exp(-Gamma)
  float L[C][C + 4];          // 80-byte rows: 16-byte aligned for row-broadcast loads
  float beta[C];
};

template <int NS>
struct __align__(128) ChainStage {
  Ops ops;
  __nv_bfloat16 v[C][NS];     // value slice, as its TMA box lands
};
template <int NS>
__host__ __device__ constexpr uint32_t chain_bytes() { return kSlotBytes + C * NS * 2; }

template <int NS>
struct __align__(128) Shared {
  RawStage raw[PRSTAGE];
  ProdStage prod[PSTAGE];
  ChainStage<NS> cst[CSTAGE];
  float2 gprod[2][2][64];    // per-half decay products exchanged inside the gate group
  float gnorm[2][4][16];     // fused preprocessing: per-gate-warp partial squared norms (8 q, 8 k)
  unsigned long long raw_full[PRSTAGE], raw_empty[PRSTAGE];
  unsigned long long prod_free[PSTAGE], gate_done[PSTAGE], solved[PSTAGE];
  unsigned long long c_full[CSTAGE], c_empty[CSTAGE];
  unsigned long long ready[RING];      // arrived (remotely) by the slot's producer
  unsigned long long slot_free[RING];  // arrived (remotely) by every CTA of the cluster
};
static_assert(sizeof(Ops) % 128 == 0 && sizeof(RawStage) % 128 == 0, "stage alignment");
static_assert(sizeof(ProdStage) % 128 == 0 && sizeof(ChainStage<16>) % 128 == 0 && sizeof(ChainStage<32>) % 128 == 0,
              "stage alignment");
static_assert(sizeof(Shared<32>) <= 227 * 1024 && sizeof(Shared<16>) <= 227 * 1024, "shared memory budget");

// ---------------------------------------------------------------- the kernel
struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* g;
  const float* beta;
  const int32_t* cu;       // may be null: one sequence [0, T)
  const float* init;       // may be null
  __nv_bfloat16* out;
  float* fin;              // may be null
  unsigned char* ring;     // [num_seqs * H][RING] slots of kSlotBytes
  int64_t T;
  int64_t beta_st, beta_sh;  // element strides of beta over tokens and heads
  int64_t out_st, out_sh;    // element strides of out over tokens and heads
  int32_t H;
  int32_t N;               // sequences (items are the N * H (sequence, head) pairs)
  float scale;
  float* outf;             // fp32 outputs [T, H, 128] (kModeOutF32 only)
  int64_t outf_st;         // token stride of outf
  float exp_lb;            // exp(lower_bound) (fused gate preprocessing only)
};
// Launch modes of the time-split prefill (a template argument of the kernel;
// 0 for a plain call):
//   kModeZeroV        the value tensor reads as zero (v is not loaded);
//   kModeIdentityInit every (sequence, head) starts from the 128 x 128
//                     identity (value column c = key c), which turns the
//                     final state into the segment's transition map;
//   kModeOutF32       o is written in fp32 to outf (token stride outf_st)
//                     instead of bf16 to out.
constexpr uint32_t kModeZeroV = 1u, kModeIdentityInit = 2u, kModeOutF32 = 4u;
constexpr float kNormEps2 = 1e-12f;  // (1e-6)^2: the norm floor of the fused normalisation, squared

struct TensorMaps {
  CUtensorMap q, k, g, v;
};

// FG: the fused gate preprocessing is compiled in: q and k are raw
// projections, L2-normalised here per (token, head) (q / max(||q||, 1e-6));
// g holds gate logits x, whose decay factor is exp(max(log sigmoid(x),
// lower_bound)) = max(sigmoid(x), exp_lb); beta holds logits b, used as
// sigmoid(b). MODE: the launch mode above. The plain kernel (FG = false,
// MODE = 0) carries the code of neither.
template <int NS, bool FG, uint32_t MODE>
__global__ void __cluster_dims__(D / NS, 1, 1) __launch_bounds__(NTHREADS, 1)
    kda_fwd_kernel(const Params p, const __grid_constant__ TensorMaps tm) {
  constexpr int NSLICE = D / NS;   // CTAs per (sequence, head) = cluster size
  constexpr int NCHAIN = NS / 16;  // chain warps
  static_assert(NS == 16 || NS == 32, "value slice of 16 or 32 columns");
  static_assert(NCHAIN <= MAX_CHAIN, "warp layout");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared<NS>& sh = *reinterpret_cast<Shared<NS>*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int gq = lane >> 2;  // fragment row group
  const int tq = lane & 3;   // fragment column pair

  const int rank = blockIdx.x;  // value slice = rank inside the cluster
  const int dv0 = rank * NS;
  const int H = p.H;
  const int64_t T = p.T;

  // Work items are the (sequence, head) pairs, item = seq * H + h. A cluster
  // takes items first, first + stride, ...: one item with the grid
  // (NSLICE, H, N); several, back to back, with the persistent grid
  // (NSLICE, G, 1), so that an item's pipeline fill overlaps the previous
  // item's tail. Every pipeline counter (stages, ring slots, chunk ownership)
  // runs over all the chunks of the cluster's items, in order.
  const int nitems = p.N * H;
  const int first = static_cast<int>(blockIdx.z * gridDim.y + blockIdx.y);
  const int stride = static_cast<int>(gridDim.y * gridDim.z);
  // (seq, h) of an item and its token range; returns its number of chunks
  auto item_at = [&](int it, int& seq, int& h, int64_t& t0, int64_t& t1) -> int {
    seq = it / H;
    h = it - seq * H;
    t0 = 0;
    t1 = T;
    if (p.cu) {
      t0 = p.cu[seq];
      t1 = p.cu[seq + 1];
      t0 = t0 < 0 ? 0 : (t0 > T ? T : t0);
      t1 = t1 < t0 ? t0 : (t1 > T ? T : t1);
    }
    return static_cast<int>((t1 - t0 + C - 1) / C);
  };
  // chunk g of the cluster (counted over its items) is produced by CTA g mod NSLICE:
  // the first chunk of an item this CTA produces, the item starting at chunk gbase
  auto owned_first = [&](int64_t gbase) { return static_cast<int>(((rank - gbase) % NSLICE + NSLICE) % NSLICE); };
  unsigned char* ring = p.ring + static_cast<size_t>(first) * RING * kSlotBytes;

  if (tid == 0) {
    for (int s = 0; s < PRSTAGE; ++s) {
      mbar_init(&sh.raw_full[s], 1 + C);  // expect_tx arrive + one per beta lane
      mbar_init(&sh.raw_empty[s], NGATE);
    }
    for (int s = 0; s < PSTAGE; ++s) {
      mbar_init(&sh.prod_free[s], 1);
      mbar_init(&sh.gate_done[s], NGATE);
      mbar_init(&sh.solved[s], 1);
    }
    for (int s = 0; s < CSTAGE; ++s) {
      mbar_init(&sh.c_full[s], 1);
      mbar_init(&sh.c_empty[s], NCHAIN);
    }
    for (int s = 0; s < RING; ++s) {
      mbar_init(&sh.ready[s], 1);
      mbar_init(&sh.slot_free[s], NSLICE);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // every CTA's barriers exist before any remote arrive
  cluster_sync();

  if (warp < NCHAIN) {
    // =========================================================== chain warps
    // Warp w owns S^T[16 value columns x 128 keys] (columns 16w .. 16w+15 of
    // the slice) for the whole sequence: tile sacc[u] holds keys 8u .. 8u+7 as
    // an m16n8 accumulator, so lane (gq, tq) holds columns gq (+8) x keys
    // 8u+2tq (+1). Packed to bf16 these registers are, unchanged, the A
    // fragments of products over the keys (X^T = S^T Kd^T, O^T = S^T Qd^T).
    // Nothing of the state leaves the registers and the warp needs no partner.
    const int cv = 16 * warp;          // first value column (slice-local)
    float sacc[16][4];
    const int64_t out_st = p.out_st;
    int64_t gc = 0;                    // the cluster's chunks so far
    for (int it = first; it < nitems; it += stride) {
      int seq, h;
      int64_t t0, t1;
      const int nch = item_at(it, seq, h, t0, t1);
      const size_t sbase = (static_cast<size_t>(seq) * H + h) * D * D;
      // this lane's output columns of head h; rows step by the token stride
      __nv_bfloat16* const out_base = p.out + static_cast<int64_t>(h) * p.out_sh + dv0 + cv + 2 * tq;
#pragma unroll
      for (int u = 0; u < 16; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = 8 * u + 2 * tq + (e & 1);
          const int col = dv0 + cv + gq + 8 * (e >> 1);
          sacc[u][e] = (MODE & kModeIdentityInit) ? (key == col ? 1.f : 0.f)
                       : p.init ? __ldg(p.init + sbase + static_cast<size_t>(key) * D + col) : 0.f;
        }

      for (int n = 0; n < nch; ++n, ++gc) {
        const int s = static_cast<int>(gc % CSTAGE);
        const int64_t cs = t0 + static_cast<int64_t>(n) * C;
        const int m = static_cast<int>((t1 - cs) < C ? (t1 - cs) : C);
        ChainStage<NS>& st = sh.cst[s];

        // stage s has landed (the notify warp observed its mbarrier)
        named_bar(BAR_FULL0 + s, 32 * (NCHAIN + 1));

        // Every product on the chain takes the register-resident operand as its
        // A fragment, so nothing on the chain needs a transpose:
        //   X^T = V^T + S^T Kd^T,  Vnew^T = X^T Tb^T,  S^T <- S^T Diag(gamma) + Vnew^T Kend,
        //   O^T = S^T Qd^T + Vnew^T Aqk^T  (times scale at the store).
        // The products are ordered for one in-order warp on one tensor pipe: the
        // state's own chain (X -> Vnew -> S) goes first at every step and the O
        // products, which nothing waits for, fill the pipe while a chain result
        // drains through conversion.
        uint32_t bk[8][4];
#pragma unroll
        for (int t = 0; t < 8; ++t) ldsm_x4(bk[t], &st.ops.kd[(lane & 7) + ((lane >> 4) << 3)][16 * t + ((lane >> 3) & 1) * 8]);
        // ---- X^T (two accumulator chains per 8-token tile); each key tile of S
        // is packed to bf16 (sa: the chunk-start state, also used by O) and then
        // scaled by gamma for the update. Lane (gq, tq) of tile nt holds columns
        // gq (+8) x tokens 8nt + 2tq (+1).
        float xa[2][4], xb[2][4] = {};
        {
          uint32_t vt[4];
          if constexpr ((MODE & kModeZeroV) != 0u) {
            vt[0] = vt[1] = vt[2] = vt[3] = 0u;
          } else {
            ldsm_x4_t(vt, &st.v[(lane & 7) + ((lane >> 3) & 1) * 8][cv + (lane >> 4) * 8]);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int nt = j & 1, e0 = 2 * (j >> 1);
            xa[nt][e0] = __uint_as_float(vt[j] << 16);
            xa[nt][e0 + 1] = __uint_as_float(vt[j] & 0xffff0000u);
          }
        }
        uint32_t sa[8][4];
        const float4* gp = reinterpret_cast<const float4*>(&st.ops.gam[tq][0]);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          sa[t][0] = pack_bf16(sacc[2 * t][0], sacc[2 * t][1]);
          sa[t][1] = pack_bf16(sacc[2 * t][2], sacc[2 * t][3]);
          sa[t][2] = pack_bf16(sacc[2 * t + 1][0], sacc[2 * t + 1][1]);
          sa[t][3] = pack_bf16(sacc[2 * t + 1][2], sacc[2 * t + 1][3]);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            if (t & 1)
              mma(xb[nt], sa[t], bk[t][2 * nt], bk[t][2 * nt + 1]);
            else
              mma(xa[nt], sa[t], bk[t][2 * nt], bk[t][2 * nt + 1]);
          }
          const float4 g4 = gp[t];
          mul2(sacc[2 * t][0], sacc[2 * t][1], g4.x, g4.y);
          mul2(sacc[2 * t][2], sacc[2 * t][3], g4.x, g4.y);
          mul2(sacc[2 * t + 1][0], sacc[2 * t + 1][1], g4.z, g4.w);
          mul2(sacc[2 * t + 1][2], sacc[2 * t + 1][3], g4.z, g4.w);
        }
        // ---- O^T = S^T Qd^T (chunk-start state) + Vnew^T Aqk^T, in three installments
        float oa[2][4] = {}, ob[2][4] = {};
        auto o_steps = [&](int t_begin, int t_end) {
#pragma unroll
          for (int t = t_begin; t < t_end; ++t) {
            uint32_t bq[4];
            ldsm_x4(bq, &st.ops.qd[(lane & 7) + ((lane >> 4) << 3)][16 * t + ((lane >> 3) & 1) * 8]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              if (t & 1)
                mma(ob[nt], sa[t], bq[2 * nt], bq[2 * nt + 1]);
              else
                mma(oa[nt], sa[t], bq[2 * nt], bq[2 * nt + 1]);
            }
          }
        };
        o_steps(0, 3);
        // ---- Vnew^T = X^T Tb^T
        uint32_t bt[4];
        ldsm_x4(bt, &st.ops.tb[(lane & 7) + ((lane >> 4) << 3)][((lane >> 3) & 1) * 8]);
        float vn[2][4] = {};
        {
          uint32_t ax[4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            ax[2 * nt] = pack_bf16(xa[nt][0] + xb[nt][0], xa[nt][1] + xb[nt][1]);
            ax[2 * nt + 1] = pack_bf16(xa[nt][2] + xb[nt][2], xa[nt][3] + xb[nt][3]);
          }
          mma(vn[0], ax, bt[0], bt[1]);
          mma(vn[1], ax, bt[2], bt[3]);
        }
        // kd fragments are dead: the same registers take Kend
#pragma unroll
        for (int t = 0; t < 8; ++t) ldsm_x4_t(bk[t], &st.ops.ke[(lane & 7) + ((lane >> 3) & 1) * 8][16 * t + (lane >> 4) * 8]);
        o_steps(3, 6);
        // Vnew^T as an A fragment (rows = columns, k = tokens)
        uint32_t av[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          av[2 * nt] = pack_bf16(vn[nt][0], vn[nt][1]);
          av[2 * nt + 1] = pack_bf16(vn[nt][2], vn[nt][3]);
        }
        // ---- S^T <- S^T Diag(gamma) + Vnew^T Kend  (gamma applied above)
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          mma(sacc[2 * t], av, bk[t][0], bk[t][1]);
          mma(sacc[2 * t + 1], av, bk[t][2], bk[t][3]);
        }
        o_steps(6, 8);
        {
          uint32_t ba[4];
          ldsm_x4(ba, &st.ops.aqk[(lane & 7) + ((lane >> 4) << 3)][((lane >> 3) & 1) * 8]);
          mma(oa[0], av, ba[0], ba[1]);
          mma(oa[1], av, ba[2], ba[3]);
        }
        // the stage is no longer read by this warp
        mbar_arrive_warp(&sh.c_empty[s]);
        if constexpr ((MODE & kModeOutF32) != 0u) {
          // fp32 O: lane (gq, tq) of tile nt holds columns gq (+8) x tokens
          // 8nt + 2tq (+1)
          float* fbase = p.outf + static_cast<int64_t>(h) * D + dv0 + cv + gq;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int tok = 8 * nt + 2 * tq + (e & 1);
              if (tok < m) fbase[(cs + tok) * p.outf_st + 8 * (e >> 1)] = (oa[nt][e] + ob[nt][e]) * p.scale;
            }
        } else {
          // ---- store O: an 8x8 transpose per tile turns (column, token pair)
          // into (token, column pair)
          uint32_t r[2][2];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            r[nt][0] = movmatrix_t(pack_bf16((oa[nt][0] + ob[nt][0]) * p.scale, (oa[nt][1] + ob[nt][1]) * p.scale));
            r[nt][1] = movmatrix_t(pack_bf16((oa[nt][2] + ob[nt][2]) * p.scale, (oa[nt][3] + ob[nt][3]) * p.scale));
          }
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int tok = 8 * nt + gq;
            if (tok < m) {
              __nv_bfloat16* dst = out_base + (cs + tok) * out_st;
              *reinterpret_cast<uint32_t*>(dst) = r[nt][0];
              *reinterpret_cast<uint32_t*>(dst + 8) = r[nt][1];
            }
          }
        }
      }
      if (p.fin) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = 8 * u + 2 * tq + (e & 1);
            const int col = dv0 + cv + gq + 8 * (e >> 1);
            p.fin[sbase + static_cast<size_t>(key) * D + col] = sacc[u][e];
          }
      }
    }  // items
  } else if (is_gate_warp(warp)) {
    // ============================================================ gate warps
    // Thread layout: channel pair cp (channels 2cp, 2cp+1), token half th
    // (tokens 8th .. 8th+7). The decay products of the two halves meet through
    // shared memory.
    const int gt = gate_warp_index(warp) * 32 + lane;
    const int cp = gt & 63;
    const int th = gt >> 6;
    const int c0 = 2 * cp;
    int64_t gbase = 0, jg = 0;  // the item's first chunk; this CTA's produced chunks so far
    for (int it = first; it < nitems; it += stride) {
      int seq, h;
      int64_t t0, t1;
      const int nch = item_at(it, seq, h, t0, t1);
      for (int n = owned_first(gbase); n < nch; n += NSLICE, ++jg) {
        const int j = static_cast<int>(jg & 1);  // parity of the exchange buffers
        const int rs = static_cast<int>(jg % PRSTAGE), ps = static_cast<int>(jg % PSTAGE);
        const uint32_t rph = static_cast<uint32_t>(jg / PRSTAGE) & 1u;
        const uint32_t pph = static_cast<uint32_t>(jg / PSTAGE) & 1u;
        const int64_t cs = t0 + static_cast<int64_t>(n) * C;
        const int m = static_cast<int>((t1 - cs) < C ? (t1 - cs) : C);
        RawStage& rw = sh.raw[rs];
        ProdStage& st = sh.prod[ps];
        mbar_wait(&sh.raw_full[rs], rph);

        // ---- raw inputs of this thread (rows past the sequence end masked)
        constexpr bool fused = FG;
        float2 e[8], kv[8], qv[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int i = 8 * th + jj;
          const bool ok = i < m;
          const float2 gg = *reinterpret_cast<const float2*>(&rw.g[i][c0]);
          const __nv_bfloat162 kk = *reinterpret_cast<const __nv_bfloat162*>(&rw.k[i][c0]);
          const __nv_bfloat162 qq = *reinterpret_cast<const __nv_bfloat162*>(&rw.q[i][c0]);
          float2 ee;
          if constexpr (fused) {  // exp(max(log sigmoid(x), lb)) = max(sigmoid(x), exp(lb))
            ee = make_float2(fmaxf(__fdividef(1.f, 1.f + __expf(-gg.x)), p.exp_lb),
                             fmaxf(__fdividef(1.f, 1.f + __expf(-gg.y)), p.exp_lb));
          } else {
            ee = make_float2(__expf(gg.x), __expf(gg.y));
          }
          e[jj] = ok ? ee : make_float2(1.f, 1.f);
          kv[jj] = ok ? __bfloat1622float2(kk) : make_float2(0.f, 0.f);
          qv[jj] = ok ? __bfloat1622float2(qq) : make_float2(0.f, 0.f);
        }
        float bv = 0.f;
        if (gt < C) {
          const float b = rw.beta[gt];
          bv = gt < m ? (fused ? __fdividef(1.f, 1.f + __expf(-b)) : b) : 0.f;
        }
        mbar_arrive_warp(&sh.raw_empty[rs]);
        // fused preprocessing: this warp's partial squared norms of its 8
        // tokens' q and k (its 64 channels), reduced over the warp by a
        // butterfly that halves the values each step: afterwards lane pair
        // (l, l ^ 1) holds value 8 (l >> 4 & 1) + 4 (l >> 3 & 1) + 2 (l >> 2 & 1)
        // + (l >> 1 & 1) of [q0..q7, k0..k7]
        if constexpr (fused) {
          float sv[16];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            sv[jj] = fmaf(qv[jj].x, qv[jj].x, qv[jj].y * qv[jj].y);
            sv[8 + jj] = fmaf(kv[jj].x, kv[jj].x, kv[jj].y * kv[jj].y);
          }
#pragma unroll
          for (int w = 8, off = 16; w >= 1; w >>= 1, off >>= 1) {
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int x = 0; x < w; ++x) {
              const float send = upper ? sv[x] : sv[w + x];
              const float got = __shfl_xor_sync(0xffffffffu, send, off);
              sv[x] = (upper ? sv[w + x] : sv[x]) + got;
            }
          }
          sv[0] += __shfl_xor_sync(0xffffffffu, sv[0], 1);
          if ((lane & 1) == 0) {
            const int idx = 8 * ((lane >> 4) & 1) + 4 * ((lane >> 3) & 1) + 2 * ((lane >> 2) & 1) + ((lane >> 1) & 1);
            sh.gnorm[j & 1][gate_warp_index(warp)][idx] = sv[0];
          }
        }

        // ---- decay products: this half's total, exchanged with the other half
        float2 P = make_float2(1.f, 1.f);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          P.x *= e[jj].x;
          P.y *= e[jj].y;
        }
        mbar_wait(&sh.prod_free[ps], pph ^ 1u);
        sh.gprod[j & 1][th][cp] = P;
        if (gt < C) st.beta[gt] = bv;
        named_bar(BAR_GATE, NGATE * 32);
        const float2 Po = sh.gprod[j & 1][th ^ 1][cp];
        if constexpr (fused) {  // full norms of this half's tokens: this warp's 64 channels + the partner warp's
          const int wi = gate_warp_index(warp);
          const float* a = sh.gnorm[j & 1][wi];
          const float* b = sh.gnorm[j & 1][wi ^ 1];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float rq = rsqrtf(fmaxf(a[jj] + b[jj], kNormEps2));
            const float rk = rsqrtf(fmaxf(a[8 + jj] + b[8 + jj], kNormEps2));
            qv[jj].x *= rq;
            qv[jj].y *= rq;
            kv[jj].x *= rk;
            kv[jj].y *= rk;
          }
        }
        // E before this half (1 for the first half), F after it (1 for the second)
        float2 E = th ? Po : make_float2(1.f, 1.f);
        float2 F = th ? make_float2(1.f, 1.f) : Po;
        const float2 gamma = make_float2(P.x * Po.x, P.y * Po.y);
        const float2 rg = make_float2(__frcp_rn(gamma.x), __frcp_rn(gamma.y));
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int i = 8 * th + jj;
          E.x *= e[jj].x;
          E.y *= e[jj].y;
          *reinterpret_cast<uint32_t*>(&st.ops.kd[i][c0]) = pack_bf16(-kv[jj].x * E.x, -kv[jj].y * E.y);
          *reinterpret_cast<uint32_t*>(&st.ops.qd[i][c0]) = pack_bf16(qv[jj].x * E.x, qv[jj].y * E.y);
        }
#pragma unroll
        for (int jj = 7; jj >= 0; --jj) {
          const int i = 8 * th + jj;
          const float kfx = kv[jj].x * F.x, kfy = kv[jj].y * F.y;
          *reinterpret_cast<uint32_t*>(&st.ops.ke[i][c0]) = pack_bf16(kfx, kfy);
          *reinterpret_cast<uint32_t*>(&st.kr[i][c0]) = pack_bf16(kfx * rg.x, kfy * rg.y);
          F.x *= e[jj].x;
          F.y *= e[jj].y;
        }
        if (th == 0) *reinterpret_cast<float2*>(&st.ops.gam[0][0] + gamma_index(c0)) = gamma;
        fence_proxy_async_shared();
        mbar_arrive_warp(&sh.gate_done[ps]);
      }
      gbase += nch;
    }  // items
  } else if (warp == WARP_MMA) {
    // ============================================================= mma warp
    int64_t gbase = 0, jg = 0;
    for (int it = first; it < nitems; it += stride) {
      int seq, h;
      int64_t t0, t1;
      const int nch = item_at(it, seq, h, t0, t1);
      for (int n = owned_first(gbase); n < nch; n += NSLICE, ++jg) {
        const int ps = static_cast<int>(jg % PSTAGE);
        const uint32_t pph = static_cast<uint32_t>(jg / PSTAGE) & 1u;
        ProdStage& st = sh.prod[ps];
        mbar_wait(&sh.gate_done[ps], pph);
        float accA[2][4] = {}, accQ[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t ak[4], aq[4], b[4];
          ldsm_x4(ak, &st.ops.kd[lane & 15][16 * kk + (lane >> 4) * 8]);
          ldsm_x4(aq, &st.ops.qd[lane & 15][16 * kk + (lane >> 4) * 8]);
          ldsm_x4(b, &st.kr[(lane & 7) + ((lane >> 4) << 3)][16 * kk + ((lane >> 3) & 1) * 8]);
          mma(accA[0], ak, b[0], b[1]);
          mma(accA[1], ak, b[2], b[3]);
          mma(accQ[0], aq, b[0], b[1]);
          mma(accQ[1], aq, b[2], b[3]);
        }
        // accA = -A (Kd carries the sign): L = diag(beta) A = -beta_i accA
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int i = gq + 8 * (e2 >> 1);
            const int jc = 8 * nt + 2 * tq + (e2 & 1);
            st.L[i][jc] = (jc < i) ? -st.beta[i] * accA[nt][e2] : 0.f;
            st.ops.aqk[i][jc] = __float2bfloat16_rn((jc <= i) ? accQ[nt][e2] : 0.f);
          }
        __syncwarp();
        // (I + L)^{-1} on the same warp: lanes 0-15, one column each
        if (lane < C) {
          // column `col` of T = (I + L)^{-1}: x_i = [i == col] - sum_{m<i} L[i][m] x_m,
          // reading each row of L with 16-byte loads that all lanes share
          const int col = lane;
          float xs[C];
#pragma unroll
          for (int i = 0; i < C; ++i) {
            float acc0 = (i == col) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
            for (int m4 = 0; m4 < (i + 3) / 4; ++m4) {
              const float4 l4 = *reinterpret_cast<const float4*>(&st.L[i][4 * m4]);
              if (4 * m4 + 0 < i) acc0 = fmaf(-l4.x, xs[4 * m4 + 0], acc0);
              if (4 * m4 + 1 < i) acc1 = fmaf(-l4.y, xs[4 * m4 + 1], acc1);
              if (4 * m4 + 2 < i) acc0 = fmaf(-l4.z, xs[4 * m4 + 2], acc0);
              if (4 * m4 + 3 < i) acc1 = fmaf(-l4.w, xs[4 * m4 + 3], acc1);
            }
            xs[i] = acc0 + acc1;
          }
          const float bc = st.beta[col];
#pragma unroll
          for (int i = 0; i < C; ++i) st.ops.tb[i][col] = __float2bfloat16_rn(xs[i] * bc);
        }
        fence_proxy_async_shared();
        mbar_arrive_warp(&sh.solved[ps]);
      }
      gbase += nch;
    }  // items
  } else if (warp == WARP_STORE) {
    // ============================================================ store warp
    // Up to two stores in flight: a chunk's slot is announced to the cluster
    // once its store has completed, which is checked after the next store is
    // issued (the last one after the loop).
    if (lane == 0) {
      auto announce = [&](int64_t g, int ps) {
        // The slot's bytes were written by the bulk-copy engine and that
        // write has completed (bulk_wait above). The proxy fence makes them
        // visible to this thread's generic proxy and one cluster-scope
        // release fence orders them before every signal that follows, so the
        // relaxed arrivals below carry them to the consumers' acquire waits
        // (one fence per chunk rather than a release per arrival).
        fence_proxy_async_global();
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        for (int c = 0; c < NSLICE; ++c)
          mbar_arrive_remote_relaxed(&sh.ready[g % RING], static_cast<uint32_t>(c));
        mbar_arrive(&sh.prod_free[ps]);
      };
      int64_t gbase = 0, jg = 0, prev_g = -1;
      int prev_ps = 0;
      for (int it = first; it < nitems; it += stride) {
        int seq, h;
        int64_t t0, t1;
        const int nch = item_at(it, seq, h, t0, t1);
        for (int n = owned_first(gbase); n < nch; n += NSLICE, ++jg) {
          const int64_t g = gbase + n;
          const int ps = static_cast<int>(jg % PSTAGE);
          const uint32_t pph = static_cast<uint32_t>(jg / PSTAGE) & 1u;
          const int slot = static_cast<int>(g % RING);
          mbar_wait(&sh.solved[ps], pph);
          // the slot's previous chunk (g - RING) has been copied by every CTA of the cluster
          mbar_wait_cl(&sh.slot_free[slot], (static_cast<uint32_t>(g / RING) & 1u) ^ 1u);
          fence_proxy_async_shared();
          bulk_s2g(ring + static_cast<size_t>(slot) * kSlotBytes, &sh.prod[ps].ops, kSlotBytes);
          if (prev_g >= 0) {
            bulk_wait<1>();
            announce(prev_g, prev_ps);
          }
          prev_g = g;
          prev_ps = ps;
        }
        gbase += nch;
      }
      if (prev_g >= 0) {
        bulk_wait<0>();
        announce(prev_g, prev_ps);
      }
    }
  } else if (warp == WARP_PLOAD) {
    // ====================================================== producer loads
    // lane 0: TMA boxes of q, k, g; lanes 1-16: beta (zero past the sequence end)
    int64_t gbase = 0, jg = 0;
    for (int it = first; it < nitems; it += stride) {
      int seq, h;
      int64_t t0, t1;
      const int nch = item_at(it, seq, h, t0, t1);
      for (int n = owned_first(gbase); n < nch; n += NSLICE, ++jg) {
        const int rs = static_cast<int>(jg % PRSTAGE);
        const uint32_t rph = static_cast<uint32_t>(jg / PRSTAGE) & 1u;
        const int64_t cs = t0 + static_cast<int64_t>(n) * C;
        const int tok = static_cast<int>(cs);
        RawStage& rw = sh.raw[rs];
        mbar_wait(&sh.raw_empty[rs], rph ^ 1u);
        if (lane == 0) {
          mbar_arrive_expect_tx(&sh.raw_full[rs], kRawBytes);
          tma_load_3d(&rw.q[0][0], &tm.q, 0, h, tok, &sh.raw_full[rs]);
          tma_load_3d(&rw.k[0][0], &tm.k, 0, h, tok, &sh.raw_full[rs]);
          tma_load_3d(&rw.g[0][0], &tm.g, 0, h, tok, &sh.raw_full[rs]);
        } else if (lane <= C) {
          const int r = lane - 1;
          const bool ok = cs + r < t1;
          cp_async4(&rw.beta[r], p.beta + (ok ? (cs + r) * p.beta_st + h * p.beta_sh : 0), ok ? 4u : 0u);
          cp_async_arrive(&sh.raw_full[rs]);
        }
      }
      gbase += nch;
    }  // items
  } else if (warp == notify_warp<NS>()) {
    // ==================================================== stage notifications
    // Waiting on a transaction mbarrier costs the waiter ~100 cycles even when
    // the phase completed long ago; this warp takes that cost off the chain's
    // critical path and releases each chain warp through a hardware barrier.
    // The mbarrier acquire makes the landed bytes visible to this warp and the
    // barrier orders them before the chain warps' reads.
    int64_t gc = 0;
    for (int it = first; it < nitems; it += stride) {
      int seq, h;
      int64_t t0, t1;
      const int nch = item_at(it, seq, h, t0, t1);
      for (int n = 0; n < nch; ++n, ++gc) {
        const int s = static_cast<int>(gc % CSTAGE);
        mbar_wait(&sh.c_full[s], static_cast<uint32_t>(gc / CSTAGE) & 1u);
        __syncwarp();
        named_bar_arrive(BAR_FULL0 + s, 32 * (NCHAIN + 1));
        // the ring slot has been copied here: give it back to its producer
        if (lane == 0)
          mbar_arrive_remote_relaxed(&sh.slot_free[gc % RING], static_cast<uint32_t>(gc % NSLICE));
      }
    }  // items
  } else if (warp == 9) {
    if (lane == 0 && p.cu && rank == 0) {
      for (int it = first; it < nitems; it += stride) {
        const int seq = it / H;
        if (it - seq * H == 0) check_bounds(p.cu, seq, p.N, T);
      }
    }
  } else if (warp == WARP_CLOAD) {
    // ====================================================== consumer loads
    if (lane == 0) {
      int64_t gc = 0;
      for (int it = first; it < nitems; it += stride) {
        int seq, h;
        int64_t t0, t1;
        const int nch = item_at(it, seq, h, t0, t1);
        for (int n = 0; n < nch; ++n, ++gc) {
          const int s = static_cast<int>(gc % CSTAGE);
          const uint32_t ph = static_cast<uint32_t>(gc / CSTAGE) & 1u;
          const int slot = static_cast<int>(gc % RING);
          const int tok = static_cast<int>(t0 + static_cast<int64_t>(n) * C);
          ChainStage<NS>& st = sh.cst[s];
          mbar_wait(&sh.c_empty[s], ph ^ 1u);
          mbar_wait_cl(&sh.ready[slot], static_cast<uint32_t>(gc / RING) & 1u);
          fence_proxy_async_global();
          mbar_arrive_expect_tx(&sh.c_full[s], (MODE & kModeZeroV) ? kSlotBytes : chain_bytes<NS>());
          bulk_g2s(&st.ops, ring + static_cast<size_t>(slot) * kSlotBytes, kSlotBytes, &sh.c_full[s]);
          if constexpr ((MODE & kModeZeroV) == 0u) tma_load_3d(&st.v[0][0], &tm.v, dv0, h, tok, &sh.c_full[s]);
        }
      }  // items
    }
  }
  // no CTA leaves while a peer may still arrive on its barriers
  __syncwarp();
  cluster_sync();
}

}  // namespace kda
