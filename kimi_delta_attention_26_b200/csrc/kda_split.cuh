// kda_split.cuh -- combine step of the time-split prefill.
//
// A long sequence with few heads leaves most SMs idle: each (sequence, head)
// is one serial chain. The time split runs the sequence's two halves at the
// same time. The first half [0, Ta) runs as usual from the initial state. The
// second half [Ta, T) does not know its start state S_a yet, so it runs twice
// from known states, in parallel with the first:
//   from the zero state            -> outputs o_loc(t) and end state B,
//   with v = 0 from the identity   -> "outputs" o_M(t) = scale M(t)^T q_t and
//                                     end state M (M(t) maps the half's
//                                     start state to its state at t).
// The recurrence is linear in the initial state, S(t) = S_loc(t) + M(t) S_a,
// so once the first half's end state S_a is known:
//   o_t = o_loc(t) + S_a^T o_M(t)             (this file: split_correct_kernel)
//   S_T = M S_a + B                           (this file: split_state_kernel)
// (the affine state map of a segment, page "Kimi K3 开源满月…", section
// "反转一": the per-(sequence, head) grid leaves the GPU idle for small H).

#pragma once

#include "kda_prims.cuh"

namespace kda {
namespace split {

constexpr int TOK = 32;         // tokens per tile (one pipeline stage)
constexpr int NSTAGE = 4;       // tiles in flight per CTA
constexpr int BP = D + 8;       // padded bf16 row pitch of the S_a tile (conflict-free ldmatrix)
constexpr int NCOMPUTE = 8;     // warps 0-7: 2 token halves x 4 column quarters; warp 8 issues the loads
constexpr int NTHREADS = 32 * (NCOMPUTE + 1);
// One stage: o_M as two 128-byte-swizzled boxes [32 tokens][64 bf16] and
// o_loc as four boxes [32 tokens][32 fp32]; every box is 4 KB.
constexpr uint32_t BOX_BYTES = TOK * 128u;
constexpr uint32_t STAGE_BYTES = 6u * BOX_BYTES;
constexpr uint32_t SA_OFF = NSTAGE * STAGE_BYTES;                      // S_a tile, bf16 [128 key][BP]
constexpr uint32_t BAR_OFF = SA_OFF + D * BP * 2u;
constexpr uint32_t SMEM_BYTES = BAR_OFF + 2u * NSTAGE * 8u + 1024u;   // + alignment slack
static_assert((D * BP * 2u) % 8u == 0u, "barrier alignment");

struct CorrectMaps {
  CUtensorMap om, oloc;
};

// Byte offset of 16-byte chunk `c` of row `r` in a box written by TMA with
// 128-byte swizzling (rows of 128 bytes, chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw128(int r, int c) { return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4)); }

// o[t] = bf16(o_loc[t] + S_a^T o_M[t]) for the tokens of the second half.
// Grid (n, H), persistent over 32-token tiles: each CTA stages its head's S_a
// once, as one bf16 tile (the precision in which the chain itself feeds the
// state to its products), and walks tiles blockIdx.x, blockIdx.x + n, ...
// o_M is bf16 [T1, H, 128], o_loc fp32 [T1, H, 128], both read through TMA
// into a 4-stage ring of shared memory so that enough bytes are in flight to
// stream them at HBM speed.
__global__ void __launch_bounds__(NTHREADS) split_correct_kernel(const __grid_constant__ CorrectMaps tm,
                                                                 const float* __restrict__ sa, __nv_bfloat16* out,
                                                                 int64_t out_st, int64_t out_sh, int64_t T1) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(sm + SA_OFF);
  unsigned long long* full = reinterpret_cast<unsigned long long*>(sm + BAR_OFF);
  unsigned long long* empty = full + NSTAGE;
  const int h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = static_cast<int>((T1 + TOK - 1) / TOK);
  const int first = blockIdx.x, step = gridDim.x;
  const int mine = first < ntiles ? (ntiles - first + step - 1) / step : 0;
  if (tid == 0) {
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NCOMPUTE);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const float* S = sa + static_cast<size_t>(h) * D * D;
  for (int i = tid; i < D * D / 4; i += NTHREADS) {
    const int key = (4 * i) / D, col = (4 * i) % D;
    const float4 v = *reinterpret_cast<const float4*>(S + 4 * i);
    uint2 pk;
    pk.x = pack_bf16(v.x, v.y);
    pk.y = pack_bf16(v.z, v.w);
    *reinterpret_cast<uint2*>(bs + key * BP + col) = pk;
  }
  __syncthreads();
  if (warp == NCOMPUTE) {
    // ---- loads: tile j of this CTA into stage j % NSTAGE
    if (lane == 0) {
      for (int j = 0; j < mine; ++j) {
        const int st = j % NSTAGE;
        if (j >= NSTAGE) mbar_wait(&empty[st], ((j / NSTAGE) - 1) & 1);
        const int tok = (first + j * step) * TOK;
        unsigned char* dst = sm + st * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
        tma_load_3d(dst, &tm.om, 0, h, tok, &full[st]);
        tma_load_3d(dst + BOX_BYTES, &tm.om, 64, h, tok, &full[st]);
        for (int b = 0; b < 4; ++b) tma_load_3d(dst + (2 + b) * BOX_BYTES, &tm.oloc, 32 * b, h, tok, &full[st]);
      }
    }
    return;
  }
  const int th = warp & 1, cq = warp >> 1;  // token half, column quarter (32 value columns)
  const int gq = lane >> 2, tq = lane & 3;
  for (int j = 0; j < mine; ++j) {
    const int st = j % NSTAGE;
    mbar_wait(&full[st], (j / NSTAGE) & 1);
    const unsigned char* stage = sm + st * STAGE_BYTES;
    float acc[4][4] = {};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      // A: 16 tokens x 16 keys of o_M (box ks / 4, chunks 2 (ks % 4) and +1)
      uint32_t a[4];
      const int r = 16 * th + (lane & 15);
      ldsm_x4(a, stage + (ks >> 2) * BOX_BYTES + sw128(r, 2 * (ks & 3) + (lane >> 4)));
#pragma unroll
      for (int np = 0; np < 2; ++np) {  // pairs of 8-column tiles of this warp's 32 columns
        const int c = 32 * cq + 16 * np;
        uint32_t b[4];
        ldsm_x4_t(b, bs + (16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8) * BP + c + (lane >> 4) * 8);
        mma(acc[2 * np], a, b[0], b[1]);
        mma(acc[2 * np + 1], a, b[2], b[3]);
      }
    }
    // epilogue: + o_loc (box cq of the stage), one rounding to bf16
    const unsigned char* lbox = stage + (2 + cq) * BOX_BYTES;
    const int64_t tok0 = static_cast<int64_t>(first + j * step) * TOK + 16 * th;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = 16 * th + gq + 8 * hr;
      const int64_t row = tok0 + gq + 8 * hr;
      float2 l[4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
        l[nt] = *reinterpret_cast<const float2*>(lbox + sw128(r, 2 * nt + (tq >> 1)) + 8 * (tq & 1));
      if (row < T1) {
        __nv_bfloat16* o = out + row * out_st + static_cast<int64_t>(h) * out_sh + 32 * cq + 2 * tq;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
          *reinterpret_cast<uint32_t*>(o + 8 * nt) =
              pack_bf16(l[nt].x + acc[nt][2 * hr], l[nt].y + acc[nt][2 * hr + 1]);
      }
    }
    mbar_arrive_warp(&empty[st]);
  }
}

// final[h] = M[h] S_a[h] + B[h] (fp32, 128 x 128 per head). Grid (8, H): 16
// key rows per CTA, one value column per thread (its column of S_a in
// registers, the 16 rows of M in shared memory).
__global__ void __launch_bounds__(128) split_state_kernel(const float* __restrict__ Mm, const float* __restrict__ sa,
                                                          const float* __restrict__ Bm, float* fin) {
  __shared__ float sM[16][D];
  const int h = blockIdx.y, r0 = 16 * blockIdx.x, col = threadIdx.x;
  const size_t base = static_cast<size_t>(h) * D * D;
  float sc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) sc[c] = sa[base + static_cast<size_t>(c) * D + col];
  for (int i = 0; i < 16; ++i) sM[i][col] = Mm[base + static_cast<size_t>(r0 + i) * D + col];
  __syncthreads();
  for (int i = 0; i < 16; ++i) {
    float acc = Bm[base + static_cast<size_t>(r0 + i) * D + col];
#pragma unroll
    for (int c = 0; c < D; ++c) acc = fmaf(sM[i][c], sc[c], acc);
    fin[base + static_cast<size_t>(r0 + i) * D + col] = acc;
  }
}

}  // namespace split
}  // namespace kda
