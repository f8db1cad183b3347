// kda_decode.cuh -- one decode step of Kimi Delta Attention for a batch of
// requests, each against its own resident fp32 state.
//
// Per request b and head h, with the state S (128 key rows x 128 value
// columns, fp32) and the request's token (q, k, v bf16; g fp32 log-decay per
// key channel; beta fp32):
//   S' = Diag(exp g) S                      (decay)
//   u  = S'^T k,   w = S'^T q               (two reductions over the key rows)
//   d  = beta (v - u)                       (the effective write)
//   S  <- S' + k d^T                        = (I - beta k k^T) S' + beta k v^T
//   o  = scale (w + (q . k) d)              = scale S_new^T q
// This is the token recurrence S_t = (I - beta_t k_t k_t^T) Diag(exp g_t)
// S_{t-1} + beta_t k_t v_t^T, o_t = scale S_t^T q_t for one token (page
// "FlashKDA: CUTLASS Kernel من Moonshot لـ Kimi", section "سياق Kimi Linear":
// a fixed-size state per head is what makes long-context decoding cheap).
//
// The step reads and writes the whole state once: 128 KiB per (request, head)
// against ~1.5 KB of token data, so it is bound by HBM bandwidth. One CTA per
// (request, head) keeps its state slice in registers between the read and the
// write: warp w holds key rows 16w..16w+15, lane l holds value columns
// 4l..4l+3 of each (a float4 per row, so a warp reads and writes one 512-byte
// row per instruction, fully coalesced). All sixteen row loads of a thread are
// issued before any arithmetic.

#pragma once

#include "kda_prims.cuh"

namespace kda {
namespace dec {

constexpr int NTHREADS = 256;             // 8 warps x 16 key rows
constexpr int ROWS = D / (NTHREADS / 32); // key rows per warp
constexpr unsigned int kFlagBadIndex = 4u;  // a state index outside [0, pool) (KDA_DEVICE_BAD_STATE_INDEX)

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* g;
  const float* beta;
  float* state;              // [pool, H, 128, 128], read and written in place
  const int32_t* idx;        // [B] state slot of each request, or null: slot b
  __nv_bfloat16* out;
  int64_t q_st, q_sh, k_st, k_sh, v_st, v_sh, g_st, g_sh, b_st, b_sh, o_st, o_sh;  // element strides
  int64_t pool;
  int H;
  float scale;
};

__global__ void __launch_bounds__(NTHREADS) kda_decode_kernel(Params p) {
  __shared__ float s_k[D], s_q[D], s_e[D];
  __shared__ float s_red[2][NTHREADS / 32][D];  // per-warp partial u and w
  __shared__ float s_d[D];
  __shared__ float s_qk[NTHREADS / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t b = blockIdx.x / p.H;
  const int h = static_cast<int>(blockIdx.x % p.H);
  int64_t slot = b;
  if (p.idx) {
    slot = p.idx[b];
    if (slot < 0 || slot >= p.pool) {  // uniform over the CTA: skip the request, record it
      if (tid == 0) atomicOr(&g_device_flags, kFlagBadIndex);
      return;
    }
  }
  float* S = p.state + (static_cast<size_t>(slot) * p.H + h) * D * D;
  // the thread's 16 rows x 4 columns, loads issued first
  float4 s[ROWS];
#pragma unroll
  for (int i = 0; i < ROWS; ++i)
    s[i] = __ldcs(reinterpret_cast<const float4*>(S + (ROWS * warp + i) * D) + lane);
  if (tid < D) {
    const float kk = __bfloat162float(p.k[b * p.k_st + h * p.k_sh + tid]);
    const float qq = __bfloat162float(p.q[b * p.q_st + h * p.q_sh + tid]);
    s_k[tid] = kk;
    s_q[tid] = qq;
    s_e[tid] = __expf(p.g[b * p.g_st + h * p.g_sh + tid]);
    float qk = qq * kk;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);
    if (lane == 0) s_qk[warp] = qk;
  }
  __syncthreads();
  // decay, then the partial reductions of this warp's rows
  float4 u = make_float4(0.f, 0.f, 0.f, 0.f), w = u;
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const int r = ROWS * warp + i;
    const float e = s_e[r], kr = s_k[r], qr = s_q[r];
    s[i].x *= e;
    s[i].y *= e;
    s[i].z *= e;
    s[i].w *= e;
    u.x = fmaf(kr, s[i].x, u.x);
    u.y = fmaf(kr, s[i].y, u.y);
    u.z = fmaf(kr, s[i].z, u.z);
    u.w = fmaf(kr, s[i].w, u.w);
    w.x = fmaf(qr, s[i].x, w.x);
    w.y = fmaf(qr, s[i].y, w.y);
    w.z = fmaf(qr, s[i].z, w.z);
    w.w = fmaf(qr, s[i].w, w.w);
  }
  reinterpret_cast<float4*>(s_red[0][warp])[lane] = u;
  reinterpret_cast<float4*>(s_red[1][warp])[lane] = w;
  __syncthreads();
  if (tid < D) {  // column tid: finish the reductions, the write and the output
    float uc = 0.f, wc = 0.f, qk = 0.f;
#pragma unroll
    for (int j = 0; j < NTHREADS / 32; ++j) {
      uc += s_red[0][j][tid];
      wc += s_red[1][j][tid];
    }
#pragma unroll
    for (int j = 0; j < D / 32; ++j) qk += s_qk[j];
    const float vc = __bfloat162float(p.v[b * p.v_st + h * p.v_sh + tid]);
    const float dc = p.beta[b * p.b_st + h * p.b_sh] * (vc - uc);
    s_d[tid] = dc;
    p.out[b * p.o_st + h * p.o_sh + tid] = __float2bfloat16_rn(p.scale * fmaf(qk, dc, wc));
  }
  __syncthreads();
  const float4 d4 = reinterpret_cast<const float4*>(s_d)[lane];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const float kr = s_k[ROWS * warp + i];
    float4 x = s[i];
    x.x = fmaf(kr, d4.x, x.x);
    x.y = fmaf(kr, d4.y, x.y);
    x.z = fmaf(kr, d4.z, x.z);
    x.w = fmaf(kr, d4.w, x.w);
    __stcs(reinterpret_cast<float4*>(S + (ROWS * warp + i) * D) + lane, x);
  }
}

}  // namespace dec
}  // namespace kda
