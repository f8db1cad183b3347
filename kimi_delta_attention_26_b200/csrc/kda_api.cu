// kda_api.cu -- the C ABI of libkda.so (declared in include/kda.h): argument
// checks on kda_tensor_t descriptors, per-device setup, scratch rings, tensor
// maps, and the launch of one of the two prefill kernels:
//   kda_fwd16.cuh  16-token chunks on mma.sync (the default path)
//   kda_fwd64.cuh  64-token chunks on tcgen05
// and, for one long sequence with few heads, the time-split prefill (the
// 16-token kernel on both halves at once, combined by kda_split.cuh).
// This file is the library's only translation unit.

#include "kda_prims.cuh"
#include "kda_fwd16.cuh"
#include "kda_fwd64.cuh"
#include "kda_split.cuh"
#include "kda_decode.cuh"
#include "kda_bwd.cuh"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <mutex>

namespace {

thread_local char g_last_cuda_error[256] = "";

kda_status_t cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return KDA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------ argument checks
// A token tensor [T, H, inner] (inner = 128) or [T, H] (inner = 0) after
// validation: base pointer and element strides over tokens and heads.
struct TokView {
  void* data;
  int64_t st, sh;
};

int elem_bytes(kda_dtype_t dt) { return dt == KDA_BF16 ? 2 : 4; }

// T and H are taken from q; every other tensor must match them.
kda_status_t view_tokens(const kda_tensor_t* t, kda_dtype_t dt, int64_t T, int64_t H, bool inner, bool is_out,
                         TokView* res) {
  if (!t) return KDA_ERR_NULL;
  if (t->dtype != dt) return KDA_ERR_DTYPE;
  if (t->ndim != (inner ? 3 : 2)) return KDA_ERR_SHAPE;
  if (t->shape[0] != T || t->shape[1] != H || (inner && t->shape[2] != KDA_HEAD_DIM)) return KDA_ERR_SHAPE;
  const int64_t st = t->stride[0], sh = t->stride[1];
  res->data = t->data;
  res->st = st;
  res->sh = sh;
  if (T == 0) return KDA_OK;  // no element is ever read or written: layout is irrelevant
  if (st <= 0 || sh <= 0) return KDA_ERR_STRIDE;
  if (inner) {
    const int64_t unit = 16 / elem_bytes(dt);  // 16-byte multiples (tensor-map strides, vector stores)
    if (t->stride[2] != 1 || st % unit != 0 || sh % unit != 0) return KDA_ERR_STRIDE;
    if (st * elem_bytes(dt) >= (int64_t(1) << 40) || sh * elem_bytes(dt) >= (int64_t(1) << 40)) return KDA_ERR_STRIDE;
    if (is_out) {
      // rows of 128 elements must not overlap: one of the two outer strides nests the other
      const bool nest_h = sh >= KDA_HEAD_DIM && (T <= 1 || st >= H * sh);
      const bool nest_t = st >= KDA_HEAD_DIM && (H <= 1 || sh >= T * st);
      if (!nest_h && !nest_t) return KDA_ERR_STRIDE;
    }
  }
  if (!t->data) return KDA_ERR_NULL;
  // tensor-map bases and vector accesses need 16 bytes; beta is read 4 bytes at a time
  if (inner ? !aligned16(t->data) : (reinterpret_cast<uintptr_t>(t->data) & 3u) != 0) return KDA_ERR_ALIGN;
  return KDA_OK;
}

kda_status_t check_state(const kda_tensor_t* t, int64_t N, int64_t H) {
  if (!t) return KDA_OK;
  if (t->dtype != KDA_F32) return KDA_ERR_DTYPE;
  if (t->ndim != 4 || t->shape[0] != N || t->shape[1] != H || t->shape[2] != KDA_HEAD_DIM ||
      t->shape[3] != KDA_HEAD_DIM)
    return KDA_ERR_SHAPE;
  const int64_t d = KDA_HEAD_DIM;
  if (t->stride[3] != 1 || t->stride[2] != d || (H > 1 && t->stride[1] != d * d) || (N > 1 && t->stride[0] != H * d * d))
    return KDA_ERR_STRIDE;
  if (!t->data) return KDA_ERR_NULL;
  if (!aligned16(t->data)) return KDA_ERR_ALIGN;
  return KDA_OK;
}

struct Problem {
  TokView q, k, v, g, beta, out;
  const float* init;
  float* fin;
  const int32_t* cu;
  int32_t num_seqs, num_heads;
  int64_t T;
  float scale;
  bool fused = false;    // kda_fwd_fused: raw q/k, gate and beta logits
  float exp_lb = 0.f;    // exp(lower_bound) of the fused gate
};

kda_status_t check_args(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v, const kda_tensor_t* g,
                        const kda_tensor_t* beta, float scale, const int32_t* cu_seqlens, int32_t num_seqs,
                        const kda_tensor_t* initial_state, const kda_tensor_t* out, const kda_tensor_t* final_state,
                        Problem* P) {
  if (!q || !k || !v || !g || !beta || !out) return KDA_ERR_NULL;
  if (q->ndim != 3) return KDA_ERR_SHAPE;
  const int64_t T = q->shape[0], H = q->shape[1];
  if (T < 0 || H < 1 || num_seqs < 1) return KDA_ERR_SHAPE;
  if (!cu_seqlens && num_seqs != 1) return KDA_ERR_SHAPE;
  if (H > 65535 || num_seqs > 65535) return KDA_ERR_SHAPE;            // grid.y / grid.z limits
  if (T > int64_t(INT32_MAX) - 256) return KDA_ERR_SHAPE;             // tensor-map coordinates are 32-bit
  if (T > (int64_t(1) << 40) / (H * KDA_HEAD_DIM)) return KDA_ERR_SHAPE;
  kda_status_t st;
  if ((st = view_tokens(q, KDA_BF16, T, H, true, false, &P->q)) != KDA_OK) return st;
  if ((st = view_tokens(k, KDA_BF16, T, H, true, false, &P->k)) != KDA_OK) return st;
  if ((st = view_tokens(v, KDA_BF16, T, H, true, false, &P->v)) != KDA_OK) return st;
  if ((st = view_tokens(g, KDA_F32, T, H, true, false, &P->g)) != KDA_OK) return st;
  if ((st = view_tokens(beta, KDA_F32, T, H, false, false, &P->beta)) != KDA_OK) return st;
  if ((st = view_tokens(out, KDA_BF16, T, H, true, true, &P->out)) != KDA_OK) return st;
  if ((st = check_state(initial_state, num_seqs, H)) != KDA_OK) return st;
  if ((st = check_state(final_state, num_seqs, H)) != KDA_OK) return st;
  if (cu_seqlens && !aligned16(cu_seqlens)) return KDA_ERR_ALIGN;
  P->init = initial_state ? static_cast<const float*>(initial_state->data) : nullptr;
  P->fin = final_state ? static_cast<float*>(final_state->data) : nullptr;
  P->cu = cu_seqlens;
  P->num_seqs = num_seqs;
  P->num_heads = static_cast<int32_t>(H);
  P->T = T;
  P->scale = scale;
  return KDA_OK;
}

// ------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

kda_status_t load_encoder() {
  if (g_encode) return KDA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult qr = cudaDriverEntryPointSymbolNotFound;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr);
  if (e != cudaSuccess) return cuda_fail(e);
  if (qr != cudaDriverEntryPointSuccess || !fn) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled not available");
    return KDA_ERR_CUDA;
  }
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return KDA_OK;
}

// [T, H, 128] view with element strides (st, sh); box {box_inner, 1, box_tok}
// starting at column 0 / box_inner.
kda_status_t encode_3d(CUtensorMap* map, const TokView& t, CUtensorMapDataType dt, int eb, int64_t T, int H,
                       int box_inner, int box_tok, CUtensorMapSwizzle swz) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kda::D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(t.sh) * eb, static_cast<cuuint64_t>(t.st) * eb};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1u, static_cast<cuuint32_t>(box_tok)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = g_encode(map, dt, 3, t.data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed (%d)",
                  static_cast<int>(r));
    return KDA_ERR_CUDA;
  }
  return KDA_OK;
}

// ------------------------------------------------------------ device setup
constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;                      // guards first-call setup of every device
std::atomic<int> g_device_ready[kMaxDevices];  // 0 unknown, 1 ready, -1 unsupported
int g_num_sms[kMaxDevices];
int g_max_clusters32[kMaxDevices];  // co-resident 4-CTA clusters of the 32-column kernel
int g_max_clusters16[kMaxDevices];  // co-resident 8-CTA clusters of the 16-column kernel
// Library-private stream-ordered pool for the scratch rings. It keeps freed
// memory (release threshold = max), so steady-state calls never map memory
// and the process's default pool is left untouched.
std::atomic<cudaMemPool_t> g_pool[kMaxDevices];
std::atomic<void*> g_noalloc_ring_addr[kMaxDevices];
std::atomic<int> g_slice_columns{0};  // 16-token path: 0 chooses per call, 16 or 32 forces
std::atomic<int> g_path{0};           // 0 (the default path), 16 or 64
std::atomic<int> g_schedule{0};       // 16-token path: 0 automatic, 1 one cluster per pair, 2 persistent
std::atomic<int> g_sched_clusters{0};  // persistent clusters: 0 as many as are resident, else at most this

// The 16-token kernel's instantiations: value slice NS, fused gate FG and
// launch mode MODE (the time split's modes run only with 32-column slices).
constexpr uint32_t kSplitL = kda::kModeOutF32;                          // second half from zero
constexpr uint32_t kSplitM = kda::kModeZeroV | kda::kModeIdentityInit;  // second half's map

template <int NS, bool FG, uint32_t MODE>
cudaError_t set_smem_one() {
  return cudaFuncSetAttribute(kda::kda_fwd_kernel<NS, FG, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(sizeof(kda::Shared<NS>)));
}

cudaError_t set_smem16() {
  cudaError_t e;
  if ((e = set_smem_one<16, false, 0>()) != cudaSuccess || (e = set_smem_one<16, true, 0>()) != cudaSuccess ||
      (e = set_smem_one<32, false, 0>()) != cudaSuccess || (e = set_smem_one<32, true, 0>()) != cudaSuccess ||
      (e = set_smem_one<32, false, kSplitL>()) != cudaSuccess ||
      (e = set_smem_one<32, true, kSplitL>()) != cudaSuccess ||
      (e = set_smem_one<32, false, kSplitM>()) != cudaSuccess || (e = set_smem_one<32, true, kSplitM>()) != cudaSuccess)
    return e;
  return cudaSuccess;
}

// Grid (D / NS, gy, gz): gy * gz clusters, cluster c taking the (sequence,
// head) items c, c + gy * gz, ...
template <int NS, bool FG, uint32_t MODE>
void launch_one(const kda::Params& p, const kda::TensorMaps& tm, int gy, int gz, cudaStream_t stream) {
  kda::kda_fwd_kernel<NS, FG, MODE><<<dim3(kda::D / NS, gy, gz), kda::NTHREADS, sizeof(kda::Shared<NS>), stream>>>(p,
                                                                                                              tm);
}

// Capability check and kernel attributes for `dev` (current), once.
kda_status_t check_device(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
  const int state = g_device_ready[dev].load(std::memory_order_acquire);
  if (state == 1) return KDA_OK;
  if (state == -1) return KDA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_device_ready[dev].load() == 1) return KDA_OK;
  int major = 0, minor = 0, sms = 0;
  cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (major != 10 || minor != 0) {
    g_device_ready[dev].store(-1);
    return KDA_ERR_UNSUPPORTED;
  }
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if ((e = set_smem16()) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaFuncSetAttribute(kda::split::split_correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kda::split::SMEM_BYTES))) != cudaSuccess)
    return cuda_fail(e);
  if ((e = cudaFuncSetAttribute(kda::bwd::kda_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kda::bwd::SMEM_BYTES))) != cudaSuccess)
    return cuda_fail(e);
  if ((e = cudaFuncSetAttribute(kda::c64::kda_fwd64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kda::c64::SMEM_BYTES))) != cudaSuccess)
    return cuda_fail(e);
  // How many clusters of the 16-token kernel the GPU holds at once: clusters
  // are placed whole inside one GPC, so this can be below SMs / cluster size.
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(kda::D / 32, 1, 1);
  cfg.blockDim = dim3(kda::NTHREADS, 1, 1);
  cfg.dynamicSmemBytes = sizeof(kda::Shared<32>);
  int clusters = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&clusters, kda::kda_fwd_kernel<32, false, 0>, &cfg)) != cudaSuccess)
    return cuda_fail(e);
  g_max_clusters32[dev] = clusters;
  cfg.gridDim = dim3(kda::D / 16, 1, 1);
  cfg.dynamicSmemBytes = sizeof(kda::Shared<16>);
  if ((e = cudaOccupancyMaxActiveClusters(&clusters, kda::kda_fwd_kernel<16, false, 0>, &cfg)) != cudaSuccess)
    return cuda_fail(e);
  g_max_clusters16[dev] = clusters;
  g_num_sms[dev] = sms;
  g_device_ready[dev].store(1, std::memory_order_release);
  return KDA_OK;
}

// The pool of kda_fwd's scratch rings, created once per device.
kda_status_t prepare_pool(int dev) {
  if (g_pool[dev].load(std::memory_order_acquire)) return KDA_OK;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_pool[dev].load()) return KDA_OK;
  cudaMemPoolProps props;
  std::memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.handleTypes = cudaMemHandleTypeNone;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t pool = nullptr;
  cudaError_t e = cudaMemPoolCreate(&pool, &props);
  if (e != cudaSuccess) return cuda_fail(e);
  uint64_t keep = ~0ull;
  e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
  if (e != cudaSuccess) {
    cudaMemPoolDestroy(pool);
    return cuda_fail(e);
  }
  g_pool[dev].store(pool, std::memory_order_release);
  return KDA_OK;
}

// 0 picks the path that measured faster on B200 for every workload so far:
// the 16-token one.
int use_path() {
  const int p = g_path.load();
  return p == 64 ? 64 : 16;
}

// 16-token path: 32-column slices unless that grid would fill at most half of
// the SMs (few heads and sequences); then 16-column slices.
int slice_columns(int dev, int32_t num_seqs, int32_t num_heads) {
  const int forced = g_slice_columns.load();
  if (forced == 16 || forced == 32) return forced;
  const int64_t ctas32 = int64_t(num_seqs) * num_heads * (KDA_HEAD_DIM / 32);
  return 2 * ctas32 <= g_num_sms[dev] ? 16 : 32;
}

size_t ring_bytes(int path, const Problem& P) {
  const size_t pairs = static_cast<size_t>(P.num_seqs) * P.num_heads;
  return path == 16 ? pairs * kda::RING * kda::kSlotBytes : pairs * kda::c64::RING * kda::c64::SLOT_BYTES;
}

// ---------------------------------------------------- allocation-free variant
// Scratch ring of kda_fwd_noalloc: a fixed-size array at file scope in device
// memory, sized for either path at KDA_NOALLOC_MAX_PAIRS pairs. Host code
// cannot use the symbol as an address; its device address is looked up once
// per device (with that device current) and passed to the kernel.
constexpr size_t kNoAllocBytes16 = static_cast<size_t>(KDA_NOALLOC_MAX_PAIRS) * kda::RING * kda::kSlotBytes;
constexpr size_t kNoAllocBytes64 = static_cast<size_t>(KDA_NOALLOC_MAX_PAIRS) * kda::c64::RING * kda::c64::SLOT_BYTES;
constexpr size_t kNoAllocRingBytes = kNoAllocBytes16 > kNoAllocBytes64 ? kNoAllocBytes16 : kNoAllocBytes64;
static_assert(kda::c64::RING * kda::c64::SLOT_BYTES == KDA_RING_BYTES_PER_PAIR, "header constant");
static_assert(kda::dec::kFlagBadIndex == KDA_DEVICE_BAD_STATE_INDEX, "header constant");
static_assert(kda::kFlagBadCuSeqlens == KDA_DEVICE_BAD_CU_SEQLENS, "header constant");
static __device__ __align__(256) unsigned char g_noalloc_ring[kNoAllocRingBytes];

kda_status_t noalloc_setup(int dev) {
  if (g_noalloc_ring_addr[dev].load(std::memory_order_acquire)) return KDA_OK;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_noalloc_ring_addr[dev].load()) return KDA_OK;
  void* addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_ring);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!addr) return KDA_ERR_CUDA;
  g_noalloc_ring_addr[dev].store(addr, std::memory_order_release);
  return KDA_OK;
}

// --------------------------------------------------------------- launches
kda_status_t launch16(const Problem& P, unsigned char* ring, int dev, cudaStream_t stream, uint32_t mode = 0,
                      float* outf = nullptr, int ns_forced = 0) {
  kda::Params p;
  p.q = static_cast<const __nv_bfloat16*>(P.q.data);
  p.k = static_cast<const __nv_bfloat16*>(P.k.data);
  p.v = static_cast<const __nv_bfloat16*>(P.v.data);
  p.g = static_cast<const float*>(P.g.data);
  p.beta = static_cast<const float*>(P.beta.data);
  p.cu = P.cu;
  p.init = P.init;
  p.out = static_cast<__nv_bfloat16*>(P.out.data);
  p.fin = P.fin;
  p.ring = ring;
  p.T = P.T;
  p.beta_st = P.beta.st;
  p.beta_sh = P.beta.sh;
  p.out_st = P.out.st;
  p.out_sh = P.out.sh;
  p.H = P.num_heads;
  p.N = P.num_seqs;
  p.scale = P.scale;
  p.exp_lb = P.exp_lb;
  p.outf = outf;
  p.outf_st = static_cast<int64_t>(P.num_heads) * kda::D;
  const int ns = ns_forced ? ns_forced : slice_columns(dev, P.num_seqs, P.num_heads);
  kda::TensorMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (P.T > 0) {
    kda_status_t st = load_encoder();
    if (st != KDA_OK) return st;
    const int H = P.num_heads;
    constexpr auto NONE = CU_TENSOR_MAP_SWIZZLE_NONE;
    if ((st = encode_3d(&tm.q, P.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.T, H, kda::D, kda::C, NONE)) != KDA_OK ||
        (st = encode_3d(&tm.k, P.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.T, H, kda::D, kda::C, NONE)) != KDA_OK ||
        (st = encode_3d(&tm.g, P.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P.T, H, kda::D, kda::C, NONE)) != KDA_OK ||
        (st = encode_3d(&tm.v, P.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.T, H, ns, kda::C, NONE)) != KDA_OK)
      return st;
  }
  const int H = P.num_heads, N = P.num_seqs;
  if (mode != 0 && ns != 32) return KDA_ERR_UNSUPPORTED;  // not reached: the split forces 32 columns
  // One cluster per (sequence, head) item, or, when the items outnumber the
  // clusters the device holds at once, that many persistent clusters that
  // take the items round robin (each cluster's next item then starts filling
  // its pipeline while the previous one drains).
  int gy = H, gz = N;
  {
    const int64_t items = static_cast<int64_t>(N) * H;
    int resident = ns == 32 ? g_max_clusters32[dev] : g_max_clusters16[dev];
    const int sched = g_schedule.load(), cap = g_sched_clusters.load();
    if (sched == 2 && cap > 0 && cap < resident) resident = cap;
    if (resident > 0 && items > 1 && (sched == 2 || (sched == 0 && items > resident))) {
      gy = static_cast<int>(items < resident ? items : resident);
      gz = 1;
    }
  }
  if (mode == 0 && ns == 16) {
    if (P.fused) launch_one<16, true, 0>(p, tm, gy, gz, stream);
    else launch_one<16, false, 0>(p, tm, gy, gz, stream);
  } else if (mode == 0) {
    if (P.fused) launch_one<32, true, 0>(p, tm, gy, gz, stream);
    else launch_one<32, false, 0>(p, tm, gy, gz, stream);
  } else if (mode == kSplitL) {
    if (P.fused) launch_one<32, true, kSplitL>(p, tm, gy, gz, stream);
    else launch_one<32, false, kSplitL>(p, tm, gy, gz, stream);
  } else if (mode == kSplitM) {
    if (P.fused) launch_one<32, true, kSplitM>(p, tm, gy, gz, stream);
    else launch_one<32, false, kSplitM>(p, tm, gy, gz, stream);
  } else {
    return KDA_ERR_UNSUPPORTED;
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return KDA_OK;
}

kda_status_t launch64(const Problem& P, unsigned char* ring, cudaStream_t stream) {
  namespace c = kda::c64;
  c::Params p;
  p.beta = static_cast<const float*>(P.beta.data);
  p.cu = P.cu;
  p.init = P.init;
  p.out = static_cast<__nv_bfloat16*>(P.out.data);
  p.fin = P.fin;
  p.ring = ring;
  p.T = P.T;
  p.beta_st = P.beta.st;
  p.beta_sh = P.beta.sh;
  p.out_st = P.out.st;
  p.out_sh = P.out.sh;
  p.H = P.num_heads;
  p.scale = P.scale;
  c::Maps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (P.T > 0) {
    kda_status_t st = load_encoder();
    if (st != KDA_OK) return st;
    const int H = P.num_heads;
    constexpr auto NONE = CU_TENSOR_MAP_SWIZZLE_NONE;
    if ((st = encode_3d(&tm.q, P.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.T, H, kda::D, c::CH, NONE)) != KDA_OK ||
        (st = encode_3d(&tm.k, P.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.T, H, kda::D, c::CH, NONE)) != KDA_OK ||
        (st = encode_3d(&tm.g, P.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P.T, H, kda::D, c::CH, NONE)) != KDA_OK ||
        (st = encode_3d(&tm.v, P.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.T, H, 64, c::CH,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != KDA_OK)
      return st;
  }
  c::kda_fwd64_kernel<<<dim3(c::CLUSTER, P.num_heads, P.num_seqs), c::NTHREADS, c::SMEM_BYTES, stream>>>(p, tm);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return KDA_OK;
}

// ---------------------------------------------------------- time-split prefill
std::atomic<int> g_split{0};                 // 0 automatic, 1 never, 2 whenever possible
std::atomic<cudaStream_t> g_side[kMaxDevices][2];  // helper streams of the time split, per device

// One long sequence whose (head) chains would leave most SMs idle: its two
// halves run at once (three 16-token launches of one 4-CTA cluster per head
// each). Automatic only where all 3 H clusters are resident together (else
// the third launch waits for a whole wave and the split loses) and the
// sequence is long enough to repay the combine step (measured on B200: from
// T = 8192 the split wins for every H with 3 H resident clusters).
bool split_applies(const Problem& P, int dev) {
  const int mode = g_split.load();
  if (mode == 1 || P.num_seqs != 1 || P.T < 32) return false;
  if (mode == 2) return true;
  // measured on B200 (H = 2 and 8): 0.96x at T = 2048, 1.17-1.20x at 4096
  return P.T >= 4096 && 3 * static_cast<int64_t>(P.num_heads) <= g_max_clusters32[dev];
}

// Tokens [t0, t0 + len) of P's single sequence.
Problem token_range(const Problem& P, int64_t t0, int64_t len) {
  Problem S = P;
  auto shift = [&](TokView& t, int eb) {
    if (t.data) t.data = static_cast<unsigned char*>(t.data) + t0 * t.st * eb;
  };
  shift(S.q, 2);
  shift(S.k, 2);
  shift(S.v, 2);
  shift(S.g, 4);
  shift(S.beta, 4);
  shift(S.out, 2);
  S.T = len;
  S.cu = nullptr;
  S.num_seqs = 1;
  return S;
}

kda_status_t side_streams(int dev, cudaStream_t (&s)[2]) {
  if (!g_side[dev][1].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    for (int i = 0; i < 2; ++i) {
      if (g_side[dev][i].load()) continue;
      cudaStream_t st = nullptr;
      const cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
      if (e != cudaSuccess) return cuda_fail(e);
      g_side[dev][i].store(st, std::memory_order_release);
    }
  }
  s[0] = g_side[dev][0].load();
  s[1] = g_side[dev][1].load();
  return KDA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// First half from the initial state on `stream`; second half from zero (o_loc,
// end state B) and, with v = 0, from the identity (o_M, end state M) on two
// helper streams; then o = o_loc + S_a^T o_M and S_T = M S_a + B.
kda_status_t launch16_split(const Problem& P, int dev, cudaStream_t stream) {
  namespace sp = kda::split;
  // The first half runs on 16-column slices (8-CTA clusters) when the device
  // has room for its H clusters beside the second half's 2H 4-CTA clusters
  // (16 H SMs in all). Measured on B200 (T = 131072, H = 8), a 16-column
  // chain then runs ~25 % faster per chunk than the second half's fp32-output
  // run, so the first half takes ~57 % of the tokens. On 32-column slices it
  // runs ~4 % slower per token than that run (the identity run, with v = 0, is
  // faster still) and takes ~49 % of them.
  const int H = P.num_heads;
  const bool a16 = 16 * static_cast<int64_t>(H) <= g_num_sms[dev] && H <= g_max_clusters16[dev];
  const int64_t T = P.T, Ta = (T * (a16 ? 73 : 63) / 128) & ~static_cast<int64_t>(kda::C - 1), T1 = T - Ta;
  const size_t st_bytes = round256(static_cast<size_t>(H) * kda::D * kda::D * 4);
  const size_t o_bytes = round256(static_cast<size_t>(T1) * H * kda::D * 4);     // o_loc, fp32
  const size_t om_bytes = round256(static_cast<size_t>(T1) * H * kda::D * 2);    // o_M, bf16
  const size_t ring_b = round256(static_cast<size_t>(H) * kda::RING * kda::kSlotBytes);
  cudaStream_t side[2];
  kda_status_t st = side_streams(dev, side);
  if (st != KDA_OK) return st;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&scratch, 3 * st_bytes + o_bytes + om_bytes + 3 * ring_b,
                                          g_pool[dev].load(), stream);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned char* b = static_cast<unsigned char*>(scratch);
  float* sa = reinterpret_cast<float*>(b);
  float* bm = reinterpret_cast<float*>(b + st_bytes);
  float* mm = reinterpret_cast<float*>(b + 2 * st_bytes);
  float* oloc = reinterpret_cast<float*>(b + 3 * st_bytes);
  __nv_bfloat16* om = reinterpret_cast<__nv_bfloat16*>(b + 3 * st_bytes + o_bytes);
  unsigned char* rings = b + 3 * st_bytes + o_bytes + om_bytes;
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
  for (int i = 0; i < 3 && st == KDA_OK; ++i)
    if ((e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming)) != cudaSuccess) st = cuda_fail(e);
  if (st == KDA_OK) {
    Problem A = token_range(P, 0, Ta);
    A.fin = sa;
    Problem L = token_range(P, Ta, T1);
    L.init = nullptr;
    L.fin = bm;
    L.out.data = nullptr;
    Problem M = L;
    M.fin = mm;
    M.out.data = om;  // bf16 [T1, H, 128], packed
    M.out.st = static_cast<int64_t>(H) * kda::D;
    M.out.sh = kda::D;
    // the helper streams start once the scratch exists, not after the first half
    if ((e = cudaEventRecord(ev[0], stream)) != cudaSuccess) st = cuda_fail(e);
    for (int i = 0; i < 2 && st == KDA_OK; ++i)
      if ((e = cudaStreamWaitEvent(side[i], ev[0], 0)) != cudaSuccess) st = cuda_fail(e);
    if (st == KDA_OK) st = launch16(A, rings, dev, stream, 0, nullptr, a16 ? 16 : 32);
    if (st == KDA_OK) st = launch16(L, rings + ring_b, dev, side[0], kSplitL, oloc, 32);
    if (st == KDA_OK) st = launch16(M, rings + 2 * ring_b, dev, side[1], kSplitM, nullptr, 32);
    for (int i = 0; i < 2 && st == KDA_OK; ++i) {
      if ((e = cudaEventRecord(ev[1 + i], side[i])) != cudaSuccess) st = cuda_fail(e);
      else if ((e = cudaStreamWaitEvent(stream, ev[1 + i], 0)) != cudaSuccess) st = cuda_fail(e);
    }
    if (st == KDA_OK) {
      // persistent: one CTA per SM in all, each staging its head's S_a once
      const int64_t tiles = (T1 + sp::TOK - 1) / sp::TOK;
      const int64_t per_head = std::max<int64_t>(1, std::min<int64_t>(tiles, g_num_sms[dev] / H));
      sp::CorrectMaps cm;
      std::memset(&cm, 0, sizeof(cm));
      const TokView vom{om, static_cast<int64_t>(H) * kda::D, kda::D};
      const TokView vol{oloc, static_cast<int64_t>(H) * kda::D, kda::D};
      constexpr auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
      if ((st = load_encoder()) == KDA_OK &&
          (st = encode_3d(&cm.om, vom, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T1, H, 64, sp::TOK, SW)) == KDA_OK &&
          (st = encode_3d(&cm.oloc, vol, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, T1, H, 32, sp::TOK, SW)) == KDA_OK)
        sp::split_correct_kernel<<<dim3(static_cast<unsigned>(per_head), H), sp::NTHREADS, sp::SMEM_BYTES, stream>>>(
            cm, sa, static_cast<__nv_bfloat16*>(P.out.data) + Ta * P.out.st, P.out.st, P.out.sh, T1);
    }
    if (st == KDA_OK) {
      if (P.fin) sp::split_state_kernel<<<dim3(kda::D / 16, H), 128, 0, stream>>>(mm, sa, bm, P.fin);
      if ((e = cudaGetLastError()) != cudaSuccess) st = cuda_fail(e);
    }
  }
  for (int i = 0; i < 3; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);  // released once the work that records or waits on it is done
  const cudaError_t ef = cudaFreeAsync(scratch, stream);
  if (st == KDA_OK && ef != cudaSuccess) return cuda_fail(ef);
  return st;
}

kda_status_t launch(const Problem& P, unsigned char* ring, int path, int dev, cudaStream_t stream) {
  return path == 16 ? launch16(P, ring, dev, stream) : launch64(P, ring, stream);
}

kda_status_t prologue(int* dev) {
  g_last_cuda_error[0] = '\0';
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_device(*dev);
}

// kda_fwd and kda_fwd_fused after validation: the time split where it
// applies, else one launch on a ring from the pool.
kda_status_t fwd_pooled(const Problem& P, void* stream) {
  kda_status_t st;
  int dev = 0;
  if ((st = prologue(&dev)) != KDA_OK) return st;
  if ((st = prepare_pool(dev)) != KDA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int path = P.fused ? 16 : use_path();
  if (path == 16 && split_applies(P, dev)) return launch16_split(P, dev, cs);
  // Ring of chunk operands, one per (sequence, head): stream-ordered scratch
  // from the library's pool, released in stream order after the kernel.
  void* ring = nullptr;
  if (P.T > 0) {
    const cudaError_t e = cudaMallocFromPoolAsync(&ring, ring_bytes(path, P), g_pool[dev].load(), cs);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  st = launch(P, static_cast<unsigned char*>(ring), path, dev, cs);
  if (ring) {
    const cudaError_t ef = cudaFreeAsync(ring, cs);
    if (st == KDA_OK && ef != cudaSuccess) return cuda_fail(ef);
  }
  return st;
}

}  // namespace

extern "C" {

kda_status_t kda_fwd(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v, const kda_tensor_t* g,
                     const kda_tensor_t* beta, float scale, const int32_t* cu_seqlens, int32_t num_seqs,
                     const kda_tensor_t* initial_state, const kda_tensor_t* out, const kda_tensor_t* final_state,
                     void* stream) {
  g_last_cuda_error[0] = '\0';
  Problem P;
  kda_status_t st = check_args(q, k, v, g, beta, scale, cu_seqlens, num_seqs, initial_state, out, final_state, &P);
  if (st != KDA_OK) return st;
  return fwd_pooled(P, stream);
}

kda_status_t kda_fwd_fused(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v,
                           const kda_tensor_t* g, const kda_tensor_t* beta, float scale, float lower_bound,
                           const int32_t* cu_seqlens, int32_t num_seqs, const kda_tensor_t* initial_state,
                           const kda_tensor_t* out, const kda_tensor_t* final_state, void* stream) {
  g_last_cuda_error[0] = '\0';
  // the 16-token chunks keep every decay factor within e^(16 lower_bound) >= e^-80
  if (!(lower_bound >= -5.f && lower_bound < 0.f)) return KDA_ERR_VALUE;
  Problem P;
  kda_status_t st = check_args(q, k, v, g, beta, scale, cu_seqlens, num_seqs, initial_state, out, final_state, &P);
  if (st != KDA_OK) return st;
  P.fused = true;
  P.exp_lb = std::exp(lower_bound);
  return fwd_pooled(P, stream);
}

kda_status_t kda_fwd_noalloc(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v,
                             const kda_tensor_t* g, const kda_tensor_t* beta, float scale,
                             const int32_t* cu_seqlens, int32_t num_seqs, const kda_tensor_t* initial_state,
                             const kda_tensor_t* out, const kda_tensor_t* final_state, void* stream) {
  g_last_cuda_error[0] = '\0';
  Problem P;
  kda_status_t st = check_args(q, k, v, g, beta, scale, cu_seqlens, num_seqs, initial_state, out, final_state, &P);
  if (st != KDA_OK) return st;
  if (int64_t(P.num_seqs) * P.num_heads > KDA_NOALLOC_MAX_PAIRS) return KDA_ERR_CAPACITY;
  int dev = 0;
  if ((st = prologue(&dev)) != KDA_OK) return st;
  if ((st = noalloc_setup(dev)) != KDA_OK) return st;
  return launch(P, static_cast<unsigned char*>(g_noalloc_ring_addr[dev].load()), use_path(), dev,
                static_cast<cudaStream_t>(stream));
}

kda_status_t kda_decode(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v, const kda_tensor_t* g,
                        const kda_tensor_t* beta, float scale, const kda_tensor_t* state,
                        const int32_t* state_indices, const kda_tensor_t* out, void* stream) {
  g_last_cuda_error[0] = '\0';
  if (!q || !k || !v || !g || !beta || !state || !out) return KDA_ERR_NULL;
  if (q->ndim != 3 || state->ndim != 4) return KDA_ERR_SHAPE;
  const int64_t B = q->shape[0], H = q->shape[1], pool = state->shape[0];
  if (B < 0 || H < 1 || pool < 1 || H > 65535) return KDA_ERR_SHAPE;
  if (!state_indices && pool < B) return KDA_ERR_SHAPE;
  if (B * H > int64_t(INT32_MAX)) return KDA_ERR_SHAPE;  // one CTA per (request, head) in grid.x
  if (pool > (int64_t(1) << 40) / (H * KDA_HEAD_DIM * KDA_HEAD_DIM)) return KDA_ERR_SHAPE;
  TokView tq, tk, tv, tg, tb, to;
  kda_status_t st;
  if ((st = view_tokens(q, KDA_BF16, B, H, true, false, &tq)) != KDA_OK) return st;
  if ((st = view_tokens(k, KDA_BF16, B, H, true, false, &tk)) != KDA_OK) return st;
  if ((st = view_tokens(v, KDA_BF16, B, H, true, false, &tv)) != KDA_OK) return st;
  if ((st = view_tokens(g, KDA_F32, B, H, true, false, &tg)) != KDA_OK) return st;
  if ((st = view_tokens(beta, KDA_F32, B, H, false, false, &tb)) != KDA_OK) return st;
  if ((st = view_tokens(out, KDA_BF16, B, H, true, true, &to)) != KDA_OK) return st;
  if ((st = check_state(state, pool, H)) != KDA_OK) return st;
  if (state_indices && (reinterpret_cast<uintptr_t>(state_indices) & 3u) != 0) return KDA_ERR_ALIGN;
  int dev = 0;
  if ((st = prologue(&dev)) != KDA_OK) return st;
  if (B == 0) return KDA_OK;
  kda::dec::Params p;
  p.q = static_cast<const __nv_bfloat16*>(tq.data);
  p.k = static_cast<const __nv_bfloat16*>(tk.data);
  p.v = static_cast<const __nv_bfloat16*>(tv.data);
  p.g = static_cast<const float*>(tg.data);
  p.beta = static_cast<const float*>(tb.data);
  p.state = static_cast<float*>(state->data);
  p.idx = state_indices;
  p.out = static_cast<__nv_bfloat16*>(to.data);
  p.q_st = tq.st; p.q_sh = tq.sh;
  p.k_st = tk.st; p.k_sh = tk.sh;
  p.v_st = tv.st; p.v_sh = tv.sh;
  p.g_st = tg.st; p.g_sh = tg.sh;
  p.b_st = tb.st; p.b_sh = tb.sh;
  p.o_st = to.st; p.o_sh = to.sh;
  p.pool = pool;
  p.H = static_cast<int>(H);
  p.scale = scale;
  kda::dec::kda_decode_kernel<<<static_cast<unsigned>(B * H), kda::dec::NTHREADS, 0,
                                static_cast<cudaStream_t>(stream)>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return KDA_OK;
}

kda_status_t kda_bwd(const kda_tensor_t* q, const kda_tensor_t* k, const kda_tensor_t* v, const kda_tensor_t* g,
                     const kda_tensor_t* beta, float scale, const int32_t* cu_seqlens, int32_t num_seqs,
                     const kda_tensor_t* initial_state, const kda_tensor_t* dout, const kda_tensor_t* dfinal_state,
                     const kda_tensor_t* dq, const kda_tensor_t* dk, const kda_tensor_t* dv, const kda_tensor_t* dg,
                     const kda_tensor_t* dbeta, const kda_tensor_t* dinitial_state, void* stream) {
  g_last_cuda_error[0] = '\0';
  if (!dout || !dq || !dk || !dv || !dg || !dbeta) return KDA_ERR_NULL;
  // inputs as for kda_fwd (dout in the place of out: bf16 [T, H, 128])
  Problem P;
  kda_status_t st =
      check_args(q, k, v, g, beta, scale, cu_seqlens, num_seqs, initial_state, dout, dfinal_state, &P);
  if (st != KDA_OK) return st;
  const int64_t T = P.T, H = P.num_heads, N = P.num_seqs;
  // gradients: fp32, contiguous
  auto contiguous = [&](const kda_tensor_t* t, bool inner) -> kda_status_t {
    if (t->dtype != KDA_F32) return KDA_ERR_DTYPE;
    if (t->ndim != (inner ? 3 : 2) || t->shape[0] != T || t->shape[1] != H || (inner && t->shape[2] != KDA_HEAD_DIM))
      return KDA_ERR_SHAPE;
    if (T == 0) return KDA_OK;
    if (inner ? (t->stride[2] != 1 || t->stride[1] != KDA_HEAD_DIM || (T > 1 && t->stride[0] != H * KDA_HEAD_DIM))
              : (t->stride[1] != 1 || (T > 1 && t->stride[0] != H)))
      return KDA_ERR_STRIDE;
    if (!t->data) return KDA_ERR_NULL;
    if (!aligned16(t->data)) return KDA_ERR_ALIGN;
    return KDA_OK;
  };
  if ((st = contiguous(dq, true)) != KDA_OK || (st = contiguous(dk, true)) != KDA_OK ||
      (st = contiguous(dv, true)) != KDA_OK || (st = contiguous(dg, true)) != KDA_OK ||
      (st = contiguous(dbeta, false)) != KDA_OK)
    return st;
  if ((st = check_state(dinitial_state, N, H)) != KDA_OK) return st;
  int dev = 0;
  if ((st = prologue(&dev)) != KDA_OK) return st;
  if ((st = prepare_pool(dev)) != KDA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  namespace b = kda::bwd;
  const size_t ck_bytes = round256(static_cast<size_t>(T / b::BLK + N + 1) * H * b::NSLICE * 32 * b::SLOT * 4);
  const size_t part_bytes = round256(static_cast<size_t>(b::NPART) * T * H * kda::D * 4);
  const size_t pb_bytes = round256(static_cast<size_t>(b::NPART) * T * H * 4);
  void* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&scratch, ck_bytes + 3 * part_bytes + pb_bytes, g_pool[dev].load(), cs);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned char* sb = static_cast<unsigned char*>(scratch);
  b::Params p;
  p.q = static_cast<const __nv_bfloat16*>(P.q.data);
  p.k = static_cast<const __nv_bfloat16*>(P.k.data);
  p.v = static_cast<const __nv_bfloat16*>(P.v.data);
  p.dout = static_cast<const __nv_bfloat16*>(P.out.data);
  p.g = static_cast<const float*>(P.g.data);
  p.beta = static_cast<const float*>(P.beta.data);
  p.cu = P.cu;
  p.init = P.init;
  p.dfin = P.fin;
  p.dv = static_cast<float*>(dv->data);
  p.dinit = dinitial_state ? static_cast<float*>(dinitial_state->data) : nullptr;
  p.ck = reinterpret_cast<float*>(sb);
  p.pq = reinterpret_cast<float*>(sb + ck_bytes);
  p.pk = reinterpret_cast<float*>(sb + ck_bytes + part_bytes);
  p.pg = reinterpret_cast<float*>(sb + ck_bytes + 2 * part_bytes);
  p.pb = reinterpret_cast<float*>(sb + ck_bytes + 3 * part_bytes);
  p.T = T;
  p.q_st = P.q.st; p.q_sh = P.q.sh;
  p.k_st = P.k.st; p.k_sh = P.k.sh;
  p.v_st = P.v.st; p.v_sh = P.v.sh;
  p.o_st = P.out.st; p.o_sh = P.out.sh;
  p.g_st = P.g.st; p.g_sh = P.g.sh;
  p.b_st = P.beta.st; p.b_sh = P.beta.sh;
  p.H = static_cast<int>(H);
  p.scale = scale;
  b::kda_bwd_kernel<<<dim3(b::NPART, static_cast<unsigned>(H), static_cast<unsigned>(N)), b::NTHREADS, b::SMEM_BYTES,
                      cs>>>(p);
  if (T > 0) {
    const int64_t n4 = T * H * kda::D / 4, nb = T * H;
    const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, 8 * static_cast<int64_t>(g_num_sms[dev]));
    b::kda_bwd_reduce_kernel<<<static_cast<unsigned>(blocks), 256, 0, cs>>>(
        p.pq, p.pk, p.pg, p.pb, static_cast<float*>(dq->data), static_cast<float*>(dk->data),
        static_cast<float*>(dg->data), static_cast<float*>(dbeta->data), n4, nb);
  }
  e = cudaGetLastError();
  const cudaError_t ef = cudaFreeAsync(scratch, cs);
  if (e != cudaSuccess) return cuda_fail(e);
  if (ef != cudaSuccess) return cuda_fail(ef);
  return KDA_OK;
}

kda_status_t kda_set_path(int32_t path) {
  if (path != 0 && path != 16 && path != 64) return KDA_ERR_SHAPE;
  g_path.store(path);
  return KDA_OK;
}

kda_status_t kda_set_time_split(int32_t mode) {
  if (mode < 0 || mode > 2) return KDA_ERR_SHAPE;
  g_split.store(mode);
  return KDA_OK;
}

kda_status_t kda_set_schedule(int32_t mode, int32_t clusters) {
  if (mode < 0 || mode > 2 || clusters < 0) return KDA_ERR_SHAPE;
  g_schedule.store(mode);
  g_sched_clusters.store(clusters);
  return KDA_OK;
}

kda_status_t kda_set_slice_columns(int32_t columns) {
  if (columns != 0 && columns != 16 && columns != 32) return KDA_ERR_SHAPE;
  g_slice_columns.store(columns);
  return KDA_OK;
}

const char* kda_status_string(kda_status_t s) {
  switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_NULL: return "a required tensor or pointer is NULL";
    case KDA_ERR_SHAPE: return "invalid shape or sizes";
    case KDA_ERR_ALIGN: return "a data pointer is not 16-byte aligned";
    case KDA_ERR_UNSUPPORTED: return "the current device is not sm_100 (B200)";
    case KDA_ERR_CUDA: return "a CUDA call failed (see kda_last_cuda_error)";
    case KDA_ERR_CAPACITY: return "num_seqs * num_heads exceeds the fixed scratch of kda_fwd_noalloc";
    case KDA_ERR_DTYPE: return "a tensor has the wrong dtype";
    case KDA_ERR_STRIDE: return "a tensor's strides are not supported";
    case KDA_ERR_DEVICE: return "the device recorded a fault (see kda_device_status)";
    case KDA_ERR_VALUE: return "a scalar argument is out of its range";
  }
  return "unknown status";
}

const char* kda_last_cuda_error(void) { return g_last_cuda_error; }

kda_status_t kda_device_status(uint32_t* flags, int32_t reset) {
  if (!flags) return KDA_ERR_NULL;
  g_last_cuda_error[0] = '\0';
  uint32_t bits = 0, waits = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&bits, kda::g_device_flags, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpyFromSymbol(&waits, kda::g_wait_timeouts, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_fail(e);
  if (waits) bits |= KDA_DEVICE_WAIT_TIMEOUT;
  *flags = bits;
  if (reset) {
    const uint32_t zero = 0;
    if ((e = cudaMemcpyToSymbol(kda::g_device_flags, &zero, sizeof(uint32_t))) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemcpyToSymbol(kda::g_wait_timeouts, &zero, sizeof(uint32_t))) != cudaSuccess) return cuda_fail(e);
  }
  return bits ? KDA_ERR_DEVICE : KDA_OK;
}

kda_status_t kda_wait_timeouts(uint32_t* count, int32_t reset) {
  if (!count) return KDA_ERR_NULL;
  g_last_cuda_error[0] = '\0';
  cudaError_t e = cudaMemcpyFromSymbol(count, kda::g_wait_timeouts, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_fail(e);
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(kda::g_wait_timeouts, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return KDA_OK;
}

int32_t kda_abi_version(void) { return KDA_ABI_VERSION; }

}  // extern "C"
