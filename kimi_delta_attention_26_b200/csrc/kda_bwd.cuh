// kda_bwd.cuh -- backward pass of the Kimi Delta Attention recurrence
// (gradients of q, k, v, g, beta and the initial state), token by token.
//
// Per (sequence, head), with S' = Diag(exp g_t) S_{t-1} and u = v_t - S'^T k_t:
//   S_t = S' + beta k u^T,   o_t = scale S_t^T q_t.
// Walking the tokens backwards with L = dLoss/dS_t (the final-state gradient
// at the end of the sequence):
//   L   += scale q dO^T            dq = scale S_t dO
//   lk   = L^T k                   dv = beta lk,   dbeta = lk . u
//   dk   = beta (L u - S' lk)
//   dS'  = L - beta k lk^T         dg_r = sum_c dS'_rc S'_rc
//   L    = Diag(exp g) dS'         (and at the start, d initial state = L).
// (The recurrence of page "Kimi K3 开源满月…", section "KDA 内核到底难在哪";
// the pages name only a Triton implementation that trains, page "Moonshot AI …
// FlashKDA … (kucoin)".)
//
// Work decomposition. Value columns evolve independently, so one warp owns
// 16 value columns of one (sequence, head): lane l holds key rows 4l..4l+3 of
// S and of L for those columns (64 + 64 fp32 registers). dv and the initial-
// state gradient are column-local and written directly; dq, dk, dg and dbeta
// sum over all 128 columns, so every warp writes its partial sums and a second
// kernel adds the eight slices in a fixed order (deterministic results).
// States are needed backwards in time: a first forward pass stores the state
// every 4 tokens to global scratch; each 4-token block is then recomputed
// from its checkpoint into lane-private shared memory and walked backwards.
// Reductions over the keys (S'^T k, L^T k) are warp reduce-scatters followed
// by gathers. This is the plain token-level form: every step is a rank-1
// update, so it runs on the CUDA cores, not the tensor cores. The chain of
// steps is serial, so every global load is taken off it: each block's token
// inputs and checkpoint are copied into shared memory (cp.async) while the
// previous block is being processed.

#pragma once

#include "kda_prims.cuh"

namespace kda {
namespace bwd {

constexpr int NCOL = 4;               // value columns per warp
constexpr int LOGC = 2;               // log2(NCOL)
constexpr int NSLICE = D / NCOL;      // warps per (sequence, head)
constexpr int BLK = 4;                // tokens per checkpoint block
constexpr int WARPS = 8;              // warps per CTA: 32 value columns of one head
constexpr int NPART = NSLICE / WARPS; // CTAs per (sequence, head) = partial sums per gradient
constexpr int CCOL = NCOL * WARPS;    // value columns per CTA
constexpr int NTHREADS = 32 * WARPS;
constexpr int SLOT = 4 * NCOL;        // floats of one lane's share of a state
constexpr int NF4 = NCOL;             // float4 of one lane's share of a state (4 keys x NCOL columns)
static_assert(NCOL == (1 << LOGC) && NCOL == 4, "the token layout below assumes 4 columns per warp");

// One token's inputs for the CTA: k, q (bf16) and g for all 128 keys, v and dO
// for the CTA's 32 value columns, beta.
struct __align__(16) TokSmem {
  __nv_bfloat16 k[D], q[D];
  float g[D];
  __nv_bfloat16 v[CCOL], o[CCOL];
  float b;
  float pad[3];
};
constexpr int TOK_CHUNKS = (2 * D * 2 + D * 4 + 2 * CCOL * 2) / 16;  // 16-byte copies per token (beta apart)

// Shared memory: per warp the block's states and two checkpoint buffers; per
// CTA two token-block buffers and the per-token partial sums of the 8 warps.
constexpr uint32_t STATE_BYTES = 32 * SLOT * 4;
constexpr uint32_t WARP_SMEM = BLK * STATE_BYTES + 2 * STATE_BYTES;
constexpr uint32_t TOK_OFF = WARPS * WARP_SMEM;
constexpr uint32_t RED_OFF = TOK_OFF + 2 * BLK * sizeof(TokSmem);
constexpr uint32_t RED_BYTES = BLK * 3 * WARPS * 32 * 16;   // [token][dq, dk, dg][warp][lane] float4
constexpr uint32_t REDB_OFF = RED_OFF + RED_BYTES;
constexpr uint32_t SMEM_BYTES = REDB_OFF + BLK * WARPS * 4;

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* dout;
  const float* g;
  const float* beta;
  const int32_t* cu;       // may be null: one sequence [0, T)
  const float* init;       // [N, H, 128, 128] or null
  const float* dfin;       // [N, H, 128, 128] or null
  float* dv;               // [T, H, 128]
  float* dinit;            // [N, H, 128, 128] or null
  float* pq;               // partials [NPART][T][H][128] of dq, dk, dg; [NPART][T][H] of dbeta
  float* pk;
  float* pg;
  float* pb;
  float* ck;               // checkpoints [(T / 4 + N + 1)][H][NSLICE][NF4 float4 of a lane][32 lanes]
  int64_t T;
  int64_t q_st, q_sh, k_st, k_sh, v_st, v_sh, o_st, o_sh, g_st, g_sh, b_st, b_sh;  // element strides
  int H;
  float scale;
};

// Sum over the 32 lanes of each of NCOL per-lane values; every lane gets all
// NCOL sums. Reduce-scatter over lane bits 4, 3, ... (each step halves the
// values a lane keeps), then plain butterflies over the remaining lane bits,
// then a gather from a lane that holds each sum.
__device__ __forceinline__ void allreduce(float (&x)[NCOL]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = NCOL / 2, off = 16; w >= 1; w >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? x[i] : x[w + i];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      x[i] = (upper ? x[w + i] : x[i]) + got;
    }
  }
  float mine = x[0];
#pragma unroll
  for (int off = 16 >> LOGC; off >= 1; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  // lane l holds the sum of value (l >> (5 - LOGC))
#pragma unroll
  for (int c = 0; c < NCOL; ++c) x[c] = __shfl_sync(0xffffffffu, mine, c << (5 - LOGC));
}

struct Token {
  float k[4], q[4], e[4];   // this lane's 4 keys
  float v[NCOL], o[NCOL];   // the warp's value columns (v, dO)
  float b;
};

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Issue the copies of tokens [tb, tb + n) into buf, spread over the CTA's
// threads: per token TOK_CHUNKS 16-byte pieces (k, q, g rows of head h; v and
// dO of the CTA's columns cc0 ..) and beta.
__device__ __forceinline__ void fetch_tokens(const Params& p, int64_t tb, int n, int h, int cc0, TokSmem* buf) {
  constexpr int PER = TOK_CHUNKS + 1;
  for (int i = threadIdx.x; i < n * PER; i += NTHREADS) {
    const int s = i / PER, c = i % PER;
    const int64_t t = tb + s;
    TokSmem& x = buf[s];
    if (c < 16) {
      cp16(&x.k[8 * c], p.k + t * p.k_st + h * p.k_sh + 8 * c);
    } else if (c < 32) {
      cp16(&x.q[8 * (c - 16)], p.q + t * p.q_st + h * p.q_sh + 8 * (c - 16));
    } else if (c < 64) {
      cp16(&x.g[4 * (c - 32)], p.g + t * p.g_st + h * p.g_sh + 4 * (c - 32));
    } else if (c < 68) {
      cp16(&x.v[8 * (c - 64)], p.v + t * p.v_st + h * p.v_sh + cc0 + 8 * (c - 64));
    } else if (c < 72) {
      cp16(&x.o[8 * (c - 68)], p.dout + t * p.o_st + h * p.o_sh + cc0 + 8 * (c - 68));
    } else {
      cp_async4(&x.b, p.beta + t * p.b_st + h * p.b_sh, 4u);
    }
  }
}
static_assert(TOK_CHUNKS == 72, "fetch_tokens' chunk map");

__device__ __forceinline__ void read_token(const TokSmem& s, int lane, int warp, Token& x) {
  const uint2 kk = *reinterpret_cast<const uint2*>(&s.k[4 * lane]);
  const uint2 qq = *reinterpret_cast<const uint2*>(&s.q[4 * lane]);
  const float4 gg = *reinterpret_cast<const float4*>(&s.g[4 * lane]);
  const uint2 vv = *reinterpret_cast<const uint2*>(&s.v[NCOL * warp]);
  const uint2 oo = *reinterpret_cast<const uint2*>(&s.o[NCOL * warp]);
  x.k[0] = __uint_as_float(kk.x << 16); x.k[1] = __uint_as_float(kk.x & 0xffff0000u);
  x.k[2] = __uint_as_float(kk.y << 16); x.k[3] = __uint_as_float(kk.y & 0xffff0000u);
  x.q[0] = __uint_as_float(qq.x << 16); x.q[1] = __uint_as_float(qq.x & 0xffff0000u);
  x.q[2] = __uint_as_float(qq.y << 16); x.q[3] = __uint_as_float(qq.y & 0xffff0000u);
  x.e[0] = __expf(gg.x); x.e[1] = __expf(gg.y); x.e[2] = __expf(gg.z); x.e[3] = __expf(gg.w);
  x.v[0] = __uint_as_float(vv.x << 16); x.v[1] = __uint_as_float(vv.x & 0xffff0000u);
  x.v[2] = __uint_as_float(vv.y << 16); x.v[3] = __uint_as_float(vv.y & 0xffff0000u);
  x.o[0] = __uint_as_float(oo.x << 16); x.o[1] = __uint_as_float(oo.x & 0xffff0000u);
  x.o[2] = __uint_as_float(oo.y << 16); x.o[3] = __uint_as_float(oo.y & 0xffff0000u);
  x.b = s.b;
}

// Packed fp32 pairs (the two value columns 2j, 2j + 1 of a lane's key row):
// one f32x2 instruction does both, halving the issue count of the rank-1
// updates.
__device__ __forceinline__ unsigned long long pk2(float2 v) {
  return (static_cast<unsigned long long>(__float_as_uint(v.y)) << 32) | __float_as_uint(v.x);
}
__device__ __forceinline__ float2 up2(unsigned long long r) {
  return make_float2(__uint_as_float(static_cast<uint32_t>(r)), __uint_as_float(static_cast<uint32_t>(r >> 32)));
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {  // a * b + c
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(pk2(a)), "l"(pk2(b)), "l"(pk2(c)));
  return up2(r);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk2(a)), "l"(pk2(b)));
  return up2(r);
}
__device__ __forceinline__ float2 dup(float a) { return make_float2(a, a); }

// A lane's share of a state: key rows 4l + i (i < 4) x the warp's 4 columns,
// as two column pairs.
using Share = float2[4][2];

// sum_i k_i X[i][.] over this lane's 4 keys, for both column pairs
__device__ __forceinline__ void key_dot(const Token& x, const Share& X, float (&out)[NCOL]) {
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float2 a = fmul2(dup(x.k[0]), X[0][j]);
    a = ffma2(dup(x.k[1]), X[1][j], a);
    a = ffma2(dup(x.k[2]), X[2][j], a);
    a = ffma2(dup(x.k[3]), X[3][j], a);
    out[2 * j] = a.x;
    out[2 * j + 1] = a.y;
  }
}

// One forward step S <- S' + beta k (v - S'^T k)^T on this lane's share.
__device__ __forceinline__ void step_forward(Share& S, const Token& x) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    S[i][0] = fmul2(dup(x.e[i]), S[i][0]);
    S[i][1] = fmul2(dup(x.e[i]), S[i][1]);
  }
  float w[NCOL];
  key_dot(x, S, w);
  allreduce(w);
  const float2 bu[2] = {make_float2(x.b * (x.v[0] - w[0]), x.b * (x.v[1] - w[1])),
                        make_float2(x.b * (x.v[2] - w[2]), x.b * (x.v[3] - w[3]))};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    S[i][0] = ffma2(dup(x.k[i]), bu[0], S[i][0]);
    S[i][1] = ffma2(dup(x.k[i]), bu[1], S[i][1]);
  }
}

// Grid (NPART, H, N): warp w of CTA x owns value columns
// NCOL (WARPS x + w) .. + NCOL - 1 of head y, sequence z.
__global__ void __launch_bounds__(NTHREADS) kda_bwd_kernel(const Params p) {
  extern __shared__ __align__(16) unsigned char smem_b[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x, slice = WARPS * part + warp;
  const int h = blockIdx.y, seq = blockIdx.z, H = p.H;
  const int r0 = 4 * lane, c0 = NCOL * slice, cc0 = CCOL * part;
  int64_t t0 = 0, t1 = p.T;
  if (p.cu) {
    check_bounds(p.cu, seq, gridDim.z, p.T);
    t0 = p.cu[seq];
    t1 = p.cu[seq + 1];
    t0 = t0 < 0 ? 0 : (t0 > p.T ? p.T : t0);
    t1 = t1 < t0 ? t0 : (t1 > p.T ? p.T : t1);
  }
  const int64_t len = t1 - t0;
  const int64_t nblk = (len + BLK - 1) / BLK;
  const size_t state_off = (static_cast<size_t>(seq) * H + h) * D * D;
  // A lane's share of a state is NF4 float4 (key row i, columns c0 .. c0 + 3 at
  // element i); the 32 lanes' element e are adjacent, so every access of a
  // warp touches 512 contiguous bytes (conflict-free in shared memory).
  // Checkpoint j of this warp: block index t0 / 4 + seq + j (the ranges of
  // different sequences are disjoint and end below T / 4 + N + 1).
  auto ck_ptr = [&](int64_t j) {
    const int64_t blk = t0 / BLK + seq + j;
    return reinterpret_cast<float4*>(p.ck + ((static_cast<size_t>(blk) * H + h) * NSLICE + slice) * (32 * SLOT)) +
           lane;
  };
  unsigned char* wsm = smem_b + warp * WARP_SMEM;
  float4* const st_base = reinterpret_cast<float4*>(wsm) + lane;                       // BLK states
  float4* const ckb_base = reinterpret_cast<float4*>(wsm + BLK * STATE_BYTES) + lane;  // 2 checkpoint buffers
  TokSmem* const tok_base = reinterpret_cast<TokSmem*>(smem_b + TOK_OFF);               // 2 x BLK tokens (CTA)
  float4* const red = reinterpret_cast<float4*>(smem_b + RED_OFF);                      // [tok][3][warp][lane]
  float* const redb = reinterpret_cast<float*>(smem_b + REDB_OFF);                      // [tok][warp]
  auto st_ptr = [&](int j) { return st_base + j * NF4 * 32; };
  auto ckb_ptr = [&](int64_t j) { return ckb_base + (j & 1) * NF4 * 32; };
  auto tok_ptr = [&](int64_t j) { return tok_base + (j & 1) * BLK; };
  auto block_len = [&](int64_t j) {
    const int64_t tb = t0 + j * BLK;
    return static_cast<int>((tb + BLK < t1) ? BLK : t1 - tb);
  };
  auto store_state = [&](float4* dst, const Share& S) {
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i * 32] = make_float4(S[i][0].x, S[i][0].y, S[i][1].x, S[i][1].y);
  };
  auto load_state = [&](const float4* src, Share& S) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v4 = src[i * 32];
      S[i][0] = make_float2(v4.x, v4.y);
      S[i][1] = make_float2(v4.z, v4.w);
    }
  };
  // an fp32 [N, H, 128, 128] state's share of this lane (or zeros)
  auto load_global = [&](const float* base, Share& S) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v4 = base ? *reinterpret_cast<const float4*>(base + state_off + static_cast<size_t>(r0 + i) * D + c0)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      S[i][0] = make_float2(v4.x, v4.y);
      S[i][1] = make_float2(v4.z, v4.w);
    }
  };

  // ---- forward pass: the state before every 4-token block
  Share S;
  load_global(p.init, S);
  if (nblk > 0) fetch_tokens(p, t0, block_len(0), h, cc0, tok_ptr(0));
  cp_commit();
  for (int64_t j = 0; j < nblk; ++j) {
    // the next block's inputs are in flight while this one runs
    if (j + 1 < nblk) fetch_tokens(p, t0 + (j + 1) * BLK, block_len(j + 1), h, cc0, tok_ptr(j + 1));
    cp_commit();
    store_state(ck_ptr(j), S);
    cp_wait<1>();
    __syncthreads();
    const TokSmem* tk = tok_ptr(j);
    const int n = block_len(j);
    for (int s = 0; s < n; ++s) {
      Token x;
      read_token(tk[s], lane, warp, x);
      step_forward(S, x);
    }
    __syncthreads();  // every warp is done with this buffer before it is refilled
  }
  cp_wait<0>();
  // this warp's own checkpoints (each lane reads back what it wrote) are
  // ordered before the copies below
  __threadfence_block();
  __syncthreads();

  // ---- backward pass
  Share L;
  load_global(p.dfin, L);
  const size_t ppart = static_cast<size_t>(part) * static_cast<size_t>(p.T) * H;
  auto fetch_block = [&](int64_t j) {
    const float4* src = ck_ptr(j);
    float4* dst = ckb_ptr(j);
#pragma unroll
    for (int e = 0; e < NF4; ++e) cp16(dst + e * 32, src + e * 32);
    fetch_tokens(p, t0 + j * BLK, block_len(j), h, cc0, tok_ptr(j));
  };
  if (nblk > 0) fetch_block(nblk - 1);
  cp_commit();
  for (int64_t j = nblk - 1; j >= 0; --j) {
    const int64_t tb = t0 + j * BLK;
    const int n = block_len(j);
    if (j > 0) fetch_block(j - 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const TokSmem* tk = tok_ptr(j);
    // states before each token of the block: st[0] = checkpoint, st[s] after s steps
    load_state(ckb_ptr(j), S);
    for (int s = 0; s < n; ++s) {
      store_state(st_ptr(s), S);
      if (s + 1 < n) {
        Token x;
        read_token(tk[s], lane, warp, x);
        step_forward(S, x);
      }
    }
    for (int s = n - 1; s >= 0; --s) {
      const int64_t t = tb + s;
      Token x;
      read_token(tk[s], lane, warp, x);
      // S' = Diag(exp g) S_{t-1} (from the block's stored state); L += scale q dO^T
      load_state(st_ptr(s), S);
      const float2 so[2] = {make_float2(p.scale * x.o[0], p.scale * x.o[1]),
                            make_float2(p.scale * x.o[2], p.scale * x.o[3])};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          S[i][j] = fmul2(dup(x.e[i]), S[i][j]);
          L[i][j] = ffma2(dup(x.q[i]), so[j], L[i][j]);
        }
      float w[NCOL], lk[NCOL];
      key_dot(x, S, w);
      key_dot(x, L, lk);
      allreduce(w);
      allreduce(lk);
      float u[NCOL], db = 0.f;
#pragma unroll
      for (int c = 0; c < NCOL; ++c) {
        u[c] = x.v[c] - w[c];
        db = fmaf(lk[c], u[c], db);
      }
      // column-local: dv = beta lk (lane c writes column c)
      float dvc = 0.f;
#pragma unroll
      for (int c = 0; c < NCOL; ++c) dvc = (lane == c) ? x.b * lk[c] : dvc;
      if (lane < NCOL) p.dv[(static_cast<size_t>(t) * H + h) * D + c0 + lane] = dvc;
      if (lane == 0) redb[s * WARPS + warp] = db;
      // per key (this lane's 4): dq, dk, dg; then L <- Diag(exp g) dS'
      const float2 u2[2] = {make_float2(u[0], u[1]), make_float2(u[2], u[3])};
      const float2 lk2[2] = {make_float2(lk[0], lk[1]), make_float2(lk[2], lk[3])};
      const float2 o2[2] = {make_float2(x.o[0], x.o[1]), make_float2(x.o[2], x.o[3])};
      float dq[4], dk[4], dg[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float bk = x.b * x.k[i];
        float2 aq = make_float2(0.f, 0.f), lu = aq, sl = aq, ag = aq;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 st = ffma2(dup(bk), u2[j], S[i][j]);   // S_t = S' + beta k u^T
          aq = ffma2(st, o2[j], aq);
          lu = ffma2(L[i][j], u2[j], lu);
          sl = ffma2(S[i][j], lk2[j], sl);
          const float2 dsp = ffma2(dup(-bk), lk2[j], L[i][j]);
          ag = ffma2(dsp, S[i][j], ag);
          L[i][j] = fmul2(dup(x.e[i]), dsp);
        }
        dq[i] = p.scale * (aq.x + aq.y);
        dk[i] = x.b * ((lu.x + lu.y) - (sl.x + sl.y));
        dg[i] = ag.x + ag.y;
      }
      red[((s * 3 + 0) * WARPS + warp) * 32 + lane] = make_float4(dq[0], dq[1], dq[2], dq[3]);
      red[((s * 3 + 1) * WARPS + warp) * 32 + lane] = make_float4(dk[0], dk[1], dk[2], dk[3]);
      red[((s * 3 + 2) * WARPS + warp) * 32 + lane] = make_float4(dg[0], dg[1], dg[2], dg[3]);
    }
    __syncthreads();
    // the CTA's partial sums of the block's tokens: 8 warps added in order
    for (int i = threadIdx.x; i < n * 3 * 32; i += NTHREADS) {
      const int s = i / 96, v = (i / 32) % 3, l = i % 32;
      float4 a = red[((s * 3 + v) * WARPS) * 32 + l];
#pragma unroll
      for (int w2 = 1; w2 < WARPS; ++w2) {
        const float4 b = red[((s * 3 + v) * WARPS + w2) * 32 + l];
        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
      }
      float* const o = v == 0 ? p.pq : (v == 1 ? p.pk : p.pg);
      *reinterpret_cast<float4*>(o + (ppart + static_cast<size_t>(tb + s) * H + h) * D + 4 * l) = a;
    }
    if (threadIdx.x < n) {
      float a = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < WARPS; ++w2) a += redb[threadIdx.x * WARPS + w2];
      p.pb[ppart + static_cast<size_t>(tb + threadIdx.x) * H + h] = a;
    }
    __syncthreads();  // the block's buffers are free for refilling
  }
  cp_wait<0>();
  if (p.dinit) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(p.dinit + state_off + static_cast<size_t>(r0 + i) * D + c0) =
          make_float4(L[i][0].x, L[i][0].y, L[i][1].x, L[i][1].y);
  }
}

// dq, dk, dg = the sum of the NPART partials, in order; dbeta likewise.
// n4 = T * H * 128 / 4 float4 groups, nb = T * H.
__global__ void __launch_bounds__(256) kda_bwd_reduce_kernel(const float* __restrict__ pq, const float* __restrict__ pk,
                                                             const float* __restrict__ pg, const float* __restrict__ pb,
                                                             float* dq, float* dk, float* dg, float* dbeta, int64_t n4,
                                                             int64_t nb) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a, c = a;
#pragma unroll
    for (int s = 0; s < NPART; ++s) {
      const float4 x = reinterpret_cast<const float4*>(pq)[s * n4 + i];
      const float4 y = reinterpret_cast<const float4*>(pk)[s * n4 + i];
      const float4 z = reinterpret_cast<const float4*>(pg)[s * n4 + i];
      a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
      b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
      c.x += z.x; c.y += z.y; c.z += z.z; c.w += z.w;
    }
    reinterpret_cast<float4*>(dq)[i] = a;
    reinterpret_cast<float4*>(dk)[i] = b;
    reinterpret_cast<float4*>(dg)[i] = c;
  }
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nb; i += stride) {
    float a = 0.f;
#pragma unroll
    for (int s = 0; s < NPART; ++s) a += pb[s * nb + i];
    dbeta[i] = a;
  }
}

}  // namespace bwd
}  // namespace kda
