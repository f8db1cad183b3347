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

constexpr int TOK = 64;         // tokens per tile of the correction
constexpr int BP = D + 8;       // padded bf16 row pitch of the S_a tile (conflict-free ldmatrix)
constexpr int NTHREADS = 256;   // 8 warps: 4 token tiles x 2 column halves
constexpr uint32_t SMEM_BYTES = D * BP * 2u;

// o[t] = bf16(o_loc[t] + S_a^T o_M[t]) for the tokens of the second half.
// Grid (n, H), persistent over 64-token tiles: each CTA stages its head's S_a
// once, as one bf16 tile (the precision in which the chain itself feeds the
// state to its products), and walks tiles blockIdx.x, blockIdx.x + n, ...
// o_M is bf16 [T1, H, 128], o_loc fp32 [T1, H, 128]. Each warp issues all
// loads of a tile (its o_M fragments and o_loc values) before its products.
__global__ void __launch_bounds__(NTHREADS) split_correct_kernel(const float* __restrict__ oloc,
                                                                 const __nv_bfloat16* __restrict__ om,
                                                                 const float* __restrict__ sa, __nv_bfloat16* out,
                                                                 int64_t out_st, int64_t out_sh, int64_t T1, int H) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(smem_raw);   // [128 key][BP]
  const int h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
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
  const int mt = warp & 3, nh = warp >> 2;
  const size_t rstride = static_cast<size_t>(H) * D;  // o_loc and o_M rows
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * TOK; t0 < T1; t0 += static_cast<int64_t>(gridDim.x) * TOK) {
    const int64_t row0 = t0 + 16 * mt + gq, row1 = row0 + 8;
    const bool v0 = row0 < T1, v1 = row1 < T1;
    const uint32_t* a0p = reinterpret_cast<const uint32_t*>(om + static_cast<size_t>(row0) * rstride + h * D);
    const uint32_t* a1p = reinterpret_cast<const uint32_t*>(om + static_cast<size_t>(row1) * rstride + h * D);
    const float* l0p = oloc + static_cast<size_t>(row0) * rstride + static_cast<size_t>(h) * D + 64 * nh + 2 * tq;
    const float* l1p = oloc + static_cast<size_t>(row1) * rstride + static_cast<size_t>(h) * D + 64 * nh + 2 * tq;
    uint32_t a[D / 16][4];
    float2 l[8][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int kw = 8 * ks + tq;  // 32-bit word of keys 16 ks + 2 tq (+1)
      a[ks][0] = v0 ? a0p[kw] : 0u;
      a[ks][1] = v1 ? a1p[kw] : 0u;
      a[ks][2] = v0 ? a0p[kw + 4] : 0u;
      a[ks][3] = v1 ? a1p[kw + 4] : 0u;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      l[nt][0] = v0 ? *reinterpret_cast<const float2*>(l0p + 8 * nt) : make_float2(0.f, 0.f);
      l[nt][1] = v1 ? *reinterpret_cast<const float2*>(l1p + 8 * nt) : make_float2(0.f, 0.f);
    }
    float acc[8][4] = {};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // pairs of 8-column tiles
        const int c = 64 * nh + 16 * np;
        uint32_t b[4];
        ldsm_x4_t(b, bs + (16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8) * BP + c + (lane >> 4) * 8);
        mma(acc[2 * np], a[ks], b[0], b[1]);
        mma(acc[2 * np + 1], a[ks], b[2], b[3]);
      }
    }
    // epilogue: + o_loc, one rounding to bf16
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int col = 64 * nh + 8 * nt + 2 * tq;
      if (v0)
        *reinterpret_cast<uint32_t*>(out + row0 * out_st + static_cast<int64_t>(h) * out_sh + col) =
            pack_bf16(l[nt][0].x + acc[nt][0], l[nt][0].y + acc[nt][1]);
      if (v1)
        *reinterpret_cast<uint32_t*>(out + row1 * out_st + static_cast<int64_t>(h) * out_sh + col) =
            pack_bf16(l[nt][1].x + acc[nt][2], l[nt][1].y + acc[nt][3]);
    }
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
