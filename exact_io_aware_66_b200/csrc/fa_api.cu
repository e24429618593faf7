// fa_api.cu — host side of the C ABI declared in include/fa.h: argument validation, TMA
// tensor-map encoding, kernel launches and error reporting. No device memory is allocated
// here except one cached 4-byte status word per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/fa.h"
#include "fa_bwd.cuh"
#include "fa_bwd_d256.cuh"
#include "fa_bwd_q128.cuh"
#include "fa_fwd_d256.cuh"
#include "fa_fwd_fp8.cuh"
#include "fa_fwd.cuh"

namespace {

thread_local char g_err[512] = "";

fa_status set_err(fa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

fa_status cuda_err(cudaError_t e, const char* what) {
  return set_err(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---- optional per-kernel device timing (fa_profile_enable / fa_profile_read) ----
// fwd, bwd preprocess, bwd main, bwd dQ convert, fp8 fwd, fp8 V transpose, d = 256 fwd,
// d = 256 bwd dV pass, d = 256 bwd dK/dQ pass
constexpr int kKernelKinds = 9;
const char* const kKernelNames[kKernelKinds] = {
    "fa_fwd_kernel",     "fa_bwd_preprocess",  "fa_bwd_main",       "fa_bwd_dq_convert",
    "fa_fwd_fp8_kernel", "fa_fp8_transpose_v", "fa_fwd_d256_kernel", "fa_bwd_d256_dv",
    "fa_bwd_d256_dkdq"};
struct ProfileRec {
  int kind;
  cudaEvent_t start, stop;
};
struct ProfileState {
  bool on = false;
  std::vector<ProfileRec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};
thread_local ProfileState g_prof;

// RAII bracket around one kernel launch: records an event pair on `stream` when profiling is on.
struct ProfileScope {
  int kind;
  cudaStream_t stream;
  cudaEvent_t start = nullptr;
  ProfileScope(int k, cudaStream_t s) : kind(k), stream(s) {
    if (g_prof.on && (start = g_prof.get())) cudaEventRecord(start, stream);
  }
  ~ProfileScope() {
    if (!start) return;
    cudaEvent_t stop = g_prof.get();
    if (!stop) {
      g_prof.pool.push_back(start);
      return;
    }
    cudaEventRecord(stop, stream);
    g_prof.recs.push_back({kind, start, stop});
  }
};

// ---- failure-detection test hook (fa_debug_stall_next) ----
// When armed on the calling thread, the next launch of the chosen kernel kind carries a load
// for its producer to leave out and a short limit for its MMA warp's waits; it is disarmed by
// that launch.
struct StallHook {
  int kind = -1;  // kernel kind (0 forward, 2 backward main) or -1: not armed
  int skip = 0;
  unsigned long long limit_ns = 0;
};
thread_local StallHook g_stall;

template <class P>
void apply_stall(int kind, P& p) {
  if (g_stall.kind != kind) return;
  p.dbg_skip = g_stall.skip;
  p.limit_ns = g_stall.limit_ns;
  g_stall.kind = -1;
}

constexpr int kMaxDevices = 64;
struct DeviceState {
  int* status = nullptr;  // device status word
  bool checked = false;   // compute capability verified
  bool is_sm100 = false;
  // cudaFuncSetAttribute done for [d == 128][causal][dropout] (atomic: calls from several host
  // threads may launch concurrently; setting an attribute twice is harmless)
  std::atomic<bool> fwd_attr[2][2][2] = {};
  std::atomic<bool> fwd96_attr[2] = {};  // [causal]: d = 96 without dropout
  std::atomic<bool> fp8_attr[2] = {};  // [causal]
  std::atomic<bool> d256_attr[2] = {};  // [causal]
  std::atomic<bool> bwd_attr[2][2][2] = {};
  std::atomic<bool> bwd128_attr[6] = {};  // [2 (d = 128) or 4 (d = 96) + causal]
  std::atomic<bool> bwd256_attr[2] = {};  // [causal]
  int n_sm = 0;  // multiprocessors (grid of the persistent kernels)
};
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Per-device state for the current device; verifies the device is sm_100 and owns the status
// word. Returns nullptr (with the error set) on failure.
DeviceState* device_state(fa_status* st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *st = cuda_err(e, "cudaGetDevice");
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *st = set_err(FA_ERR_CUDA, "device index %d out of range", dev);
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& ds = g_dev[dev];
  if (!ds.checked) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    ds.is_sm100 = (major == 10 && minor == 0);
    cudaDeviceGetAttribute(&ds.n_sm, cudaDevAttrMultiProcessorCount, dev);
    ds.checked = true;
  }
  if (!ds.is_sm100) {
    *st = set_err(FA_ERR_CUDA, "device %d is not an sm_100 (B200) GPU", dev);
    return nullptr;
  }
  if (!ds.status) {
    e = cudaMalloc(&ds.status, sizeof(int));
    if (e != cudaSuccess) {
      *st = cuda_err(e, "cudaMalloc(status word)");
      return nullptr;
    }
    e = cudaMemset(ds.status, 0, sizeof(int));
    if (e != cudaSuccess) {
      *st = cuda_err(e, "cudaMemset(status word)");
      return nullptr;
    }
  }
  *st = FA_OK;
  return &ds;
}

// 3-D tiled map over a contiguous [BH, N, cols] tensor: dims {cols, N, BH}, box
// {box_cols, box_rows, 1}. Rows n >= N read as zero and are not written.
fa_status make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType type, int elem_bytes,
                   int cols, int N, int BH, int box_cols, int box_rows, CUtensorMapSwizzle swz,
                   long long row_stride = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return set_err(FA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (row_stride == 0) row_stride = cols;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_stride) * elem_bytes,
                           static_cast<cuuint64_t>(N) * row_stride * elem_bytes};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, type, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_err(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FA_OK;
}

fa_status make_bf16_map(CUtensorMap* m, const void* ptr, int d, int N, int BH, int box_rows) {
  return make_map(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, BH, 64, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Problem shape shared by every entry point: q, o, dO, dq are [B, H, N_q, d]; k, v, dk, dv are
// [B, H_kv, N_kv, d]; lse is [B, H, N_q]. mask: 0 none, 1 causal aligned at the top left
// (key j visible to query i iff j <= i), 2 causal aligned at the bottom right (iff
// j <= i + N_kv - N_q).
struct Shape {
  int B, H, H_kv, N_q, N_kv, d;
  float scale;
  int mask;
  bool dropout = false;     // set by apply_dropout for a drop probability that rounds above 0
  fa::DropoutParams drop{};
  size_t q_bytes() const { return static_cast<size_t>(B) * H * N_q * d * 2; }
  size_t kv_bytes() const { return static_cast<size_t>(B) * H_kv * N_kv * d * 2; }
  size_t lse_bytes() const { return static_cast<size_t>(B) * H * N_q * 4; }
  int off() const { return mask == 2 ? N_kv - N_q : 0; }
};

// Query heads per forward scheduling group: consecutive heads whose K and V (kv_row_bytes per
// key row of a key/value head, shared by `qgroup` query heads) fill about a quarter of the
// 126 MB L2, so that K/V tiles are still resident when the group's other query blocks read them.
int fwd_head_group(const Shape& s, double kv_row_bytes) {
  const double per_qhead = static_cast<double>(s.N_kv) * kv_row_bytes / (s.H / s.H_kv);
  const int g = static_cast<int>(32.0 * 1024 * 1024 / per_qhead);
  const int BH = s.B * s.H;
  return g < 1 ? 1 : (g > BH ? BH : g);
}

fa_status check_shape(const Shape& s) {
  if (s.B < 1 || s.H < 1 || s.H_kv < 1 || s.N_q < 1 || s.N_kv < 1)
    return set_err(FA_ERR_INVALID_ARG, "B, H, H_kv, N_q, N_kv must be >= 1 (got %d, %d, %d, %d, %d)",
                   s.B, s.H, s.H_kv, s.N_q, s.N_kv);
  if (s.H % s.H_kv != 0)
    return set_err(FA_ERR_INVALID_ARG, "H=%d is not a multiple of H_kv=%d", s.H, s.H_kv);
  if (s.d != 64 && s.d != 96 && s.d != 128 && s.d != 256)
    return set_err(FA_ERR_UNSUPPORTED, "head dim d=%d not in {64, 96, 128, 256}", s.d);
  if (s.mask < 0 || s.mask > 2) return set_err(FA_ERR_INVALID_ARG, "mask mode %d unknown", s.mask);
  const long long rows_q = 1LL * s.B * s.H * s.N_q, rows_kv = 1LL * s.B * s.H_kv * s.N_kv;
  if (rows_q >= (1LL << 31) || rows_kv >= (1LL << 31))
    return set_err(FA_ERR_UNSUPPORTED, "B*H*N_q=%lld or B*H_kv*N_kv=%lld >= 2^31", rows_q, rows_kv);
  if (!std::isfinite(s.scale) || !(s.scale > 0.f))
    return set_err(FA_ERR_INVALID_ARG, "scale must be finite and > 0 (got %g)", (double)s.scale);
  return FA_OK;
}

// Dropout settings of the extended entry points (NULL: none). The drop probability is rounded
// to p8 / 256, p8 = min(255, floor(256 p + 1/2)); p8 = 0 runs the kernels without dropout.
fa_status apply_dropout(Shape& s, const fa_dropout* d) {
  if (!d) return FA_OK;
  if (!std::isfinite(d->p) || d->p < 0.f || d->p >= 1.f)
    return set_err(FA_ERR_INVALID_ARG, "dropout probability %g not in [0, 1)", (double)d->p);
  const int p8 = std::min(255, static_cast<int>(std::floor(256.0 * d->p + 0.5)));
  if (p8 == 0) return FA_OK;
  s.dropout = true;
  s.drop.seed_lo = static_cast<uint32_t>(d->seed & 0xffffffffull);
  s.drop.seed_hi = static_cast<uint32_t>(d->seed >> 32);
  s.drop.offset = d->offset;
  s.drop.add4 = static_cast<uint32_t>(256 - p8) * 0x01010101u;
  s.drop.keep_scale = static_cast<float>(256.0 / (256 - p8));
  return FA_OK;
}

template <int D, bool CAUSAL, bool DROPOUT, int DM = D>
fa_status launch_fwd(DeviceState* ds, const void* q, const void* k, const void* v, void* o,
                     float* lse, const Shape& s, cudaStream_t stream) {
  using L = fa::FwdLayout<D>;
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, DROPOUT, DM>;
  std::atomic<bool>& attr = DM == 96 ? ds->fwd96_attr[CAUSAL] : ds->fwd_attr[D == 128][CAUSAL][DROPOUT];
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute(fwd smem)");
    // The kernel redistributes registers with setmaxnreg, whose split assumes 128 per thread
    // at launch; any other allocation could make setmaxnreg.inc wait forever.
    cudaFuncAttributes fattr;
    e = cudaFuncGetAttributes(&fattr, kern);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncGetAttributes(fwd)");
    if (fattr.numRegs != 128)
      return set_err(FA_ERR_CUDA, "forward kernel built with %d registers per thread, 128 expected",
                     fattr.numRegs);
    attr = true;
  }
  const int BH = s.B * s.H, BHkv = s.B * s.H_kv;
  CUtensorMap tq, tk, tv, to;
  fa_status st;
  // global width s.d (96 runs the D = 128 kernel: the loads zero-fill columns 96..127, the
  // stores clip them)
  if ((st = make_bf16_map(&tq, q, s.d, s.N_q, BH, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tk, k, s.d, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tv, v, s.d, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&to, o, s.d, s.N_q, BH, 32)) != FA_OK) return st;
  fa::FwdParams p;
  p.lse = lse;
  p.status = ds->status;
  p.N = s.N_q;
  p.N_kv = s.N_kv;
  p.BH = BH;
  p.group = s.H / s.H_kv;
  p.off = s.off();
  p.n_qblocks = (s.N_q + 255) / 256;
  p.hgroup = fwd_head_group(s, 4.0 * s.d);
  p.scale = s.scale;
  p.scale_log2 = s.scale * 1.4426950408889634f;
  p.drop = s.drop;
  apply_stall(0, p);
  const long long grid = 1LL * p.n_qblocks * BH;
  if (grid >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  ProfileScope prof(0, stream);
  kern<<<static_cast<unsigned>(grid), fa::kFwdThreads, L::kAlloc, stream>>>(tq, tk, tv, to, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_fwd launch");
  return FA_OK;
}

template <int D, bool CAUSAL, bool DROPOUT>
fa_status launch_bwd(DeviceState* ds, const void* q, const void* k, const void* v, const void* o,
                     const void* dO, const float* lse, void* dq, void* dk, void* dv,
                     void* workspace, const Shape& s, cudaStream_t stream) {
  using L = fa::BwdLayout<D>;
  auto kern = fa::fa_bwd_main<D, CAUSAL, DROPOUT>;
  std::atomic<bool>& attr = ds->bwd_attr[D == 128][CAUSAL][DROPOUT];
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute(bwd smem)");
    attr = true;
  }
  const int BH = s.B * s.H, BHkv = s.B * s.H_kv, N = s.N_q;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws);
  float* Dvec = reinterpret_cast<float*>(ws + fa::bwd_ws_offset_D(BH, N, s.d));
  float* lse2 = reinterpret_cast<float*>(ws + fa::bwd_ws_offset_lse2(BH, N, s.d));
  int* sched = reinterpret_cast<int*>(ws + fa::bwd_ws_offset_sched(BH, N, s.d));
  const int n64 = static_cast<int>(fa::bwd_n64(N));
  const long long rows = 1LL * BH * N;

  CUtensorMap tq, tk, tv, tdo, tl, tD, tacc, tdk, tdv;
  fa_status st;
  if ((st = make_bf16_map(&tq, q, s.d, N, BH, 64)) != FA_OK) return st;
  if ((st = make_bf16_map(&tk, k, s.d, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tv, v, s.d, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdo, dO, s.d, N, BH, 64)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdk, dk, s.d, s.N_kv, BHkv, 32)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdv, dv, s.d, s.N_kv, BHkv, 32)) != FA_OK) return st;
  // per-row fp32 vectors: [BH][N_q] with a row stride of N64 elements, 64-element boxes
  if ((st = make_map(&tl, lse2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, BH, 1, 64, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE, n64)) != FA_OK)
    return st;
  if ((st = make_map(&tD, Dvec, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, BH, 1, 64, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE, n64)) != FA_OK)
    return st;
  // dQ accumulator: fp32 [BH][N_q][d], reduction boxes of 32 columns x 64 rows
  if ((st = make_map(&tacc, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, s.d, N, BH, 32, 64,
                     CU_TENSOR_MAP_SWIZZLE_NONE)) != FA_OK)
    return st;

  const long long prep_threads = rows * (s.d <= 64 ? 8 : 16);
  const long long prep_blocks = (prep_threads + fa::kPrepThreads - 1) / fa::kPrepThreads;
  if (prep_blocks >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  {
    ProfileScope prof(1, stream);
    const auto* o16 = static_cast<const __nv_bfloat16*>(o);
    const auto* do16 = static_cast<const __nv_bfloat16*>(dO);
    const unsigned nb = static_cast<unsigned>(prep_blocks);
    if (s.d == 96)
      fa::fa_bwd_preprocess<96><<<nb, fa::kPrepThreads, 0, stream>>>(o16, do16, lse, dq_acc, Dvec,
                                                                     lse2, rows, N, n64,
        sched);
    else
      fa::fa_bwd_preprocess<D><<<nb, fa::kPrepThreads, 0, stream>>>(o16, do16, lse, dq_acc, Dvec,
                                                                    lse2, rows, N, n64,
        sched);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd preprocess launch");

  fa::BwdParams p;
  p.status = ds->status;
  p.N = N;
  p.N_kv = s.N_kv;
  p.BH_kv = BHkv;
  p.qgroup = s.H / s.H_kv;
  p.off = s.off();
  p.n_kv = (s.N_kv + 127) / 128;
  p.n_q = (N + 63) / 64;
  p.d = s.d;
  {
    // key/value heads per scheduling group: a group's K, V, and its query heads' Q, dO (bf16)
    // and fp32 dQ accumulator should stay within about half of the 126 MB L2
    const double per_head = static_cast<double>(s.N_kv) * D * 4 +
                            static_cast<double>(p.qgroup) * N * D * (2 + 2 + 4);
    const int g = static_cast<int>(64.0 * 1024 * 1024 / per_head);
    p.group = g < 1 ? 1 : (g > BHkv ? BHkv : g);
  }
  p.scale = s.scale;
  p.scale_log2 = s.scale * 1.4426950408889634f;
  p.drop = s.drop;
  apply_stall(2, p);
  // persistent: one CTA per SM (at most one per unit), units handed out by the counter
  const long long units = 1LL * p.n_kv * BHkv;
  if (units >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  p.n_units = static_cast<int>(units);
  p.sched_counter = sched;
  const int n_sm = ds->n_sm > 0 ? ds->n_sm : 148;
  const unsigned grid = static_cast<unsigned>(units < n_sm ? units : n_sm);
  {
    ProfileScope prof(2, stream);
    kern<<<grid, fa::kBwdThreads, L::kAlloc, stream>>>(tq, tk, tv, tdo, tl, tD, tacc, tdk, tdv,
                                                        p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd main launch");

  const long long n8 = rows * s.d / 8;
  {
    ProfileScope prof(3, stream);
    fa::fa_bwd_dq_convert<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(
        dq_acc, static_cast<__nv_bfloat16*>(dq), n8);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd convert launch");
  return FA_OK;
}

// Backward at d = 64 and d = 128 (and 96) without dropout: the 128-row query tile kernel
// (fa_bwd_q128.cuh), between the same preprocess and dQ conversion as launch_bwd.
template <int D, bool CAUSAL, int DM = D>
fa_status launch_bwd_q128(DeviceState* ds, const void* q, const void* k, const void* v,
                          const void* o, const void* dO, const float* lse, void* dq, void* dk,
                          void* dv, void* workspace, const Shape& s, cudaStream_t stream) {
  using L = fa::Bwd128Layout<D>;
  auto kern = fa::fa_bwd_main_q128<D, CAUSAL, DM>;
  std::atomic<bool>& attr = ds->bwd128_attr[(D == 128 ? (DM == 96 ? 4 : 2) : 0) + CAUSAL];
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute(q128 bwd smem)");
    cudaFuncAttributes fattr;  // the setmaxnreg split assumes 128 registers per thread
    e = cudaFuncGetAttributes(&fattr, kern);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncGetAttributes(q128 bwd)");
    if (fattr.numRegs != static_cast<int>(fa::Bwd128Regs::kLaunch))
      return set_err(FA_ERR_CUDA, "q128 backward kernel built with %d registers per thread",
                     fattr.numRegs);
    if (fattr.sharedSizeBytes != 0)
      return set_err(FA_ERR_CUDA, "q128 backward kernel has %zu bytes of static shared memory",
                     fattr.sharedSizeBytes);
    attr = true;
  }
  const int BH = s.B * s.H, BHkv = s.B * s.H_kv, N = s.N_q;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws);
  float* Dvec = reinterpret_cast<float*>(ws + fa::bwd_ws_offset_D(BH, N, s.d));
  float* lse2 = reinterpret_cast<float*>(ws + fa::bwd_ws_offset_lse2(BH, N, s.d));
  int* sched = reinterpret_cast<int*>(ws + fa::bwd_ws_offset_sched(BH, N, s.d));
  const int n64 = static_cast<int>(fa::bwd_n64(N));
  const long long rows = 1LL * BH * N;

  CUtensorMap tq, tk, tv, tdo, tl, tD, tacc, tdk, tdv;
  fa_status st;
  if ((st = make_bf16_map(&tq, q, s.d, N, BH, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tk, k, s.d, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tv, v, s.d, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdo, dO, s.d, N, BH, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdk, dk, s.d, s.N_kv, BHkv, 32)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdv, dv, s.d, s.N_kv, BHkv, 32)) != FA_OK) return st;
  // per-row fp32 vectors: [BH][N_q] with a row stride of N64 elements, 128-element boxes
  if ((st = make_map(&tl, lse2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, BH, 1, 128, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE, n64)) != FA_OK)
    return st;
  if ((st = make_map(&tD, Dvec, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, BH, 1, 128, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE, n64)) != FA_OK)
    return st;
  // dQ accumulator: fp32 [BH][N_q][d], reduction boxes of 32 columns x 64 rows; at d = 64,
  // 32 x 32 boxes in the 128-byte swizzled layout (the drain writes query rows)
  if ((st = make_map(&tacc, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, s.d, N, BH, 32,
                     D == 64 ? 32 : 64,
                     D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE)) != FA_OK)
    return st;

  const long long prep_threads = rows * (D == 64 ? 8 : 16);
  const long long prep_blocks = (prep_threads + fa::kPrepThreads - 1) / fa::kPrepThreads;
  if (prep_blocks >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  {
    ProfileScope prof(1, stream);
    const auto* o16 = static_cast<const __nv_bfloat16*>(o);
    const auto* do16 = static_cast<const __nv_bfloat16*>(dO);
    const unsigned nb = static_cast<unsigned>(prep_blocks);
    if (s.d == 96)
      fa::fa_bwd_preprocess<96><<<nb, fa::kPrepThreads, 0, stream>>>(o16, do16, lse, dq_acc, Dvec,
                                                                     lse2, rows, N, n64,
        sched);
    else
      fa::fa_bwd_preprocess<D><<<nb, fa::kPrepThreads, 0, stream>>>(o16, do16, lse, dq_acc,
                                                                    Dvec, lse2, rows, N, n64,
        sched);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd preprocess launch");

  fa::BwdParams p{};
  p.status = ds->status;
  p.N = N;
  p.N_kv = s.N_kv;
  p.BH_kv = BHkv;
  p.qgroup = s.H / s.H_kv;
  p.off = s.off();
  p.n_kv = (s.N_kv + 127) / 128;
  p.n_q = (N + 127) / 128;
  p.d = s.d;
  {
    // key/value heads per scheduling group, sized as in launch_bwd
    const double per_head = static_cast<double>(s.N_kv) * 128 * 4 +
                            static_cast<double>(p.qgroup) * N * 128 * (2 + 2 + 4);
    const int g = static_cast<int>(64.0 * 1024 * 1024 / per_head);
    p.group = g < 1 ? 1 : (g > BHkv ? BHkv : g);
  }
  p.scale = s.scale;
  p.scale_log2 = s.scale * 1.4426950408889634f;
  apply_stall(2, p);
  // persistent: one CTA per SM (at most one per unit), units handed out by the counter
  const long long units = 1LL * p.n_kv * BHkv;
  if (units >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  p.n_units = static_cast<int>(units);
  p.sched_counter = sched;
  const int n_sm = ds->n_sm > 0 ? ds->n_sm : 148;
  const unsigned grid = static_cast<unsigned>(units < n_sm ? units : n_sm);
  {
    ProfileScope prof(2, stream);
    kern<<<grid, fa::kBwdThreads, L::kBytes, stream>>>(tq, tk, tv, tdo, tl, tD, tacc, tdk, tdv,
                                                        p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd main (q128) launch");

  const long long n8 = rows * s.d / 8;
  {
    ProfileScope prof(3, stream);
    fa::fa_bwd_dq_convert<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(
        dq_acc, static_cast<__nv_bfloat16*>(dq), n8);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd convert launch");
  return FA_OK;
}

// Backward at d = 256 (fa_bwd_d256.cuh): preprocess, the dV pass, the dK/dQ pass, dQ conversion.
template <bool CAUSAL>
fa_status launch_bwd_d256(DeviceState* ds, const void* q, const void* k, const void* v,
                          const void* o, const void* dO, const float* lse, void* dq, void* dk,
                          void* dv, void* workspace, const Shape& s, cudaStream_t stream) {
  using LA = fa::Bwd256DvLayout;
  using LB = fa::Bwd256DkdqLayout;
  auto kern_a = fa::fa_bwd_d256_dv<CAUSAL>;
  auto kern_b = fa::fa_bwd_d256_dkdq<CAUSAL>;
  std::atomic<bool>& attr = ds->bwd256_attr[CAUSAL];
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(kern_a, cudaFuncAttributeMaxDynamicSharedMemorySize, LA::kAlloc);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute(d256 bwd dV smem)");
    e = cudaFuncSetAttribute(kern_b, cudaFuncAttributeMaxDynamicSharedMemorySize, LB::kAlloc);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute(d256 bwd dK/dQ smem)");
    attr = true;
  }
  const int BH = s.B * s.H, BHkv = s.B * s.H_kv, N = s.N_q;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws);
  float* Dvec = reinterpret_cast<float*>(ws + fa::bwd_ws_offset_D(BH, N, 256));
  float* lse2 = reinterpret_cast<float*>(ws + fa::bwd_ws_offset_lse2(BH, N, 256));
  const int n64 = static_cast<int>(fa::bwd_n64(N));
  const long long rows = 1LL * BH * N;

  CUtensorMap tq, tk, tv, tdo, tl, tD, tacc, tdk, tdv;
  fa_status st;
  if ((st = make_bf16_map(&tq, q, 256, N, BH, 64)) != FA_OK) return st;
  if ((st = make_bf16_map(&tk, k, 256, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tv, v, 256, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdo, dO, 256, N, BH, 64)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdk, dk, 256, s.N_kv, BHkv, 32)) != FA_OK) return st;
  if ((st = make_bf16_map(&tdv, dv, 256, s.N_kv, BHkv, 32)) != FA_OK) return st;
  // per-row fp32 vectors: [BH][N_q] with a row stride of N64 elements, 64-element boxes
  if ((st = make_map(&tl, lse2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, BH, 1, 64, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE, n64)) != FA_OK)
    return st;
  if ((st = make_map(&tD, Dvec, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, BH, 1, 64, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE, n64)) != FA_OK)
    return st;
  // dQ accumulator: fp32 [BH][N_q][256], reduction boxes of 32 columns x 32 rows
  if ((st = make_map(&tacc, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 256, N, BH, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_NONE)) != FA_OK)
    return st;

  const long long prep_threads = rows * 32;
  const long long prep_blocks = (prep_threads + fa::kPrepThreads - 1) / fa::kPrepThreads;
  if (prep_blocks >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  {
    ProfileScope prof(1, stream);
    fa::fa_bwd_preprocess<256><<<static_cast<unsigned>(prep_blocks), fa::kPrepThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, dq_acc,
        Dvec, lse2, rows, N, n64,
        nullptr);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd preprocess launch");

  fa::BwdParams p{};
  p.status = ds->status;
  p.N = N;
  p.N_kv = s.N_kv;
  p.BH_kv = BHkv;
  p.qgroup = s.H / s.H_kv;
  p.off = s.off();
  p.n_kv = (s.N_kv + 127) / 128;
  p.n_q = (N + 63) / 64;
  p.d = 256;
  {
    // key/value heads per scheduling group, sized as in launch_bwd
    const double per_head = static_cast<double>(s.N_kv) * 256 * 4 +
                            static_cast<double>(p.qgroup) * N * 256 * (2 + 2 + 4);
    const int g = static_cast<int>(64.0 * 1024 * 1024 / per_head);
    p.group = g < 1 ? 1 : (g > BHkv ? BHkv : g);
  }
  p.scale = s.scale;
  p.scale_log2 = s.scale * 1.4426950408889634f;
  apply_stall(2, p);
  const long long grid = 1LL * p.n_kv * BHkv;
  if (grid >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  {
    ProfileScope prof(7, stream);
    kern_a<<<static_cast<unsigned>(grid), fa::kBwdThreads, LA::kAlloc, stream>>>(tq, tk, tdo, tl,
                                                                                 tdv, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd (d = 256) dV pass launch");
  p.dbg_skip = -1;  // the test hook applies to the first pass only
  p.limit_ns = FA_SPIN_LIMIT_NS;
  {
    ProfileScope prof(8, stream);
    kern_b<<<static_cast<unsigned>(grid), fa::kBwdThreads, LB::kAlloc, stream>>>(
        tq, tk, tv, tdo, tl, tD, tacc, tdk, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd (d = 256) dK/dQ pass launch");

  const long long n8 = rows * 256 / 8;
  {
    ProfileScope prof(3, stream);
    fa::fa_bwd_dq_convert<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(
        dq_acc, static_cast<__nv_bfloat16*>(dq), n8);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_bwd convert launch");
  return FA_OK;
}

template <int D, bool CAUSAL>
fa_status fwd_dispatch_d(DeviceState* ds, const void* q, const void* k, const void* v, void* o,
                         float* lse, const Shape& s, cudaStream_t stream) {
  if constexpr (D == 128) {
    // d = 96 without dropout on the d = 128 layout, its products over 96 columns
    if (s.d == 96 && !s.dropout) return launch_fwd<128, CAUSAL, false, 96>(ds, q, k, v, o, lse, s, stream);
  }
  return s.dropout ? launch_fwd<D, CAUSAL, true>(ds, q, k, v, o, lse, s, stream)
                   : launch_fwd<D, CAUSAL, false>(ds, q, k, v, o, lse, s, stream);
}

// Forward for d = 256 (fa_fwd_d256.cuh): one 128-row query tile per CTA.
template <bool CAUSAL>
fa_status launch_fwd_d256(DeviceState* ds, const void* q, const void* k, const void* v, void* o,
                          float* lse, const Shape& s, cudaStream_t stream) {
  using L = fa::Fwd256Layout;
  auto kern = fa::fa_fwd_d256_kernel<CAUSAL>;
  std::atomic<bool>& attr = ds->d256_attr[CAUSAL];
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute(d256 fwd smem)");
    cudaFuncAttributes fattr;  // the setmaxnreg split assumes 128 registers per thread
    e = cudaFuncGetAttributes(&fattr, kern);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncGetAttributes(d256 fwd)");
    if (fattr.numRegs != 128)
      return set_err(FA_ERR_CUDA, "d256 forward kernel built with %d registers per thread",
                     fattr.numRegs);
    attr = true;
  }
  const int BH = s.B * s.H, BHkv = s.B * s.H_kv;
  CUtensorMap tq, tk, tv, to;
  fa_status st;
  if ((st = make_bf16_map(&tq, q, 256, s.N_q, BH, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tk, k, 256, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&tv, v, 256, s.N_kv, BHkv, 128)) != FA_OK) return st;
  if ((st = make_bf16_map(&to, o, 256, s.N_q, BH, 32)) != FA_OK) return st;
  fa::FwdParams p;
  p.lse = lse;
  p.status = ds->status;
  p.N = s.N_q;
  p.N_kv = s.N_kv;
  p.BH = BH;
  p.group = s.H / s.H_kv;
  p.off = s.off();
  p.n_qblocks = (s.N_q + 127) / 128;
  p.hgroup = fwd_head_group(s, 4.0 * 256);
  p.scale = s.scale;
  p.scale_log2 = s.scale * 1.4426950408889634f;
  const long long grid = 1LL * p.n_qblocks * BH;
  if (grid >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  ProfileScope prof(6, stream);
  kern<<<static_cast<unsigned>(grid), fa::kFwdThreads, L::kAlloc, stream>>>(tq, tk, tv, to, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_fwd (d = 256) launch");
  return FA_OK;
}

fa_status fwd_dispatch(DeviceState* ds, const void* q, const void* k, const void* v, void* o,
                       float* lse, const Shape& s, cudaStream_t stream) {
  const bool causal = s.mask != 0;
  if (s.d == 256) {
    if (s.dropout) return set_err(FA_ERR_UNSUPPORTED, "dropout is not supported at d = 256");
    return causal ? launch_fwd_d256<true>(ds, q, k, v, o, lse, s, stream)
                  : launch_fwd_d256<false>(ds, q, k, v, o, lse, s, stream);
  }
  if (s.d == 64)
    return causal ? fwd_dispatch_d<64, true>(ds, q, k, v, o, lse, s, stream)
                  : fwd_dispatch_d<64, false>(ds, q, k, v, o, lse, s, stream);
  return causal ? fwd_dispatch_d<128, true>(ds, q, k, v, o, lse, s, stream)
                : fwd_dispatch_d<128, false>(ds, q, k, v, o, lse, s, stream);
}

template <int D, bool CAUSAL>
fa_status bwd_dispatch_d(DeviceState* ds, const void* q, const void* k, const void* v,
                         const void* o, const void* dO, const float* lse, void* dq, void* dk,
                         void* dv, void* workspace, const Shape& s, cudaStream_t stream) {
  if (s.dropout)
    return launch_bwd<D, CAUSAL, true>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream);
  if constexpr (D == 128) {
    // d = 96 on the d = 128 layout, its products over 96 columns
    if (s.d == 96)
      return launch_bwd_q128<128, CAUSAL, 96>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s,
                                              stream);
  }
  return launch_bwd_q128<D, CAUSAL>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream);
}

fa_status bwd_dispatch(DeviceState* ds, const void* q, const void* k, const void* v, const void* o,
                       const void* dO, const float* lse, void* dq, void* dk, void* dv,
                       void* workspace, const Shape& s, cudaStream_t stream) {
  const bool causal = s.mask != 0;
  if (s.d == 256) {
    if (s.dropout) return set_err(FA_ERR_UNSUPPORTED, "dropout is not supported at d = 256");
    return causal ? launch_bwd_d256<true>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream)
                  : launch_bwd_d256<false>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream);
  }
  if (s.d == 64)
    return causal ? bwd_dispatch_d<64, true>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream)
                  : bwd_dispatch_d<64, false>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream);
  return causal ? bwd_dispatch_d<128, true>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream)
                : bwd_dispatch_d<128, false>(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s, stream);
}

// Argument checks of the forward (nothing is launched when one fails), then the launch.
fa_status fwd_checked(const void* q, const void* k, const void* v, void* o, float* lse,
                      const Shape& s, void* stream) {
  fa_status st = check_shape(s);
  if (st != FA_OK) return st;
  if (!q || !k || !v || !o || !lse) return set_err(FA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return set_err(FA_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  const void* ins[3] = {q, k, v};
  const size_t insz[3] = {s.q_bytes(), s.kv_bytes(), s.kv_bytes()};
  for (int b = 0; b < 3; ++b)
    if (overlaps(o, s.q_bytes(), ins[b], insz[b]) || overlaps(lse, s.lse_bytes(), ins[b], insz[b]))
      return set_err(FA_ERR_INVALID_ARG, "outputs must not alias inputs");
  if (overlaps(o, s.q_bytes(), lse, s.lse_bytes()))
    return set_err(FA_ERR_INVALID_ARG, "o and lse overlap");
  DeviceState* ds = device_state(&st);
  if (!ds) return st;
  return fwd_dispatch(ds, q, k, v, o, lse, s, static_cast<cudaStream_t>(stream));
}

size_t bwd_workspace(const Shape& s) {
  return fa::bwd_workspace_bytes(static_cast<size_t>(s.B) * s.H, s.N_q, s.d);
}

// Argument checks of the backward (nothing is launched when one fails), then the launch.
fa_status bwd_checked(const void* q, const void* k, const void* v, const void* o, const void* dO,
                      const float* lse, void* dq, void* dk, void* dv, void* workspace,
                      size_t workspace_bytes, const Shape& s, void* stream) {
  fa_status st = check_shape(s);
  if (st != FA_OK) return st;
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv)
    return set_err(FA_ERR_INVALID_ARG, "null pointer argument");
  const void* ptrs[10] = {q, k, v, o, dO, lse, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return set_err(FA_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  const size_t need = bwd_workspace(s);
  if (!workspace || workspace_bytes < need)
    return set_err(FA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes,
                   need);
  const size_t qb = s.q_bytes(), kvb = s.kv_bytes();
  const void* ins[6] = {q, k, v, o, dO, lse};
  const size_t insz[6] = {qb, kvb, kvb, qb, qb, s.lse_bytes()};
  void* outs[4] = {dq, dk, dv, workspace};
  const size_t outsz[4] = {qb, kvb, kvb, need};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], outsz[a], ins[b], insz[b]))
        return set_err(FA_ERR_INVALID_ARG, "outputs/workspace must not alias inputs");
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a], outsz[a], outs[b], outsz[b]))
        return set_err(FA_ERR_INVALID_ARG, "outputs/workspace must not overlap each other");
  }
  DeviceState* ds = device_state(&st);
  if (!ds) return st;
  return bwd_dispatch(ds, q, k, v, o, dO, lse, dq, dk, dv, workspace, s,
                      static_cast<cudaStream_t>(stream));
}

// ---- FP8 forward ----
size_t fp8_vt_ld(int N_kv) { return (static_cast<size_t>(N_kv) + 15) / 16 * 16; }
size_t fp8_workspace(const Shape& s) {
  return static_cast<size_t>(s.B) * s.H_kv * s.d * fp8_vt_ld(s.N_kv);
}

template <bool CAUSAL>
fa_status launch_fwd_fp8(DeviceState* ds, const void* q8, const void* k8, const void* v8,
                         float q_descale, float k_descale, float v_descale, void* o, float* lse,
                         void* workspace, const Shape& s, cudaStream_t stream) {
  using L = fa::Fp8Layout;
  auto kern = fa::fa_fwd_fp8_kernel<CAUSAL>;
  std::atomic<bool>& attr = ds->fp8_attr[CAUSAL];
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute(fp8 fwd smem)");
    cudaFuncAttributes fattr;  // setmaxnreg split assumes 128 registers per thread at launch
    e = cudaFuncGetAttributes(&fattr, kern);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncGetAttributes(fp8 fwd)");
    if (fattr.numRegs != 128)
      return set_err(FA_ERR_CUDA, "fp8 forward kernel built with %d registers per thread",
                     fattr.numRegs);
    attr = true;
  }
  const int BH = s.B * s.H, BHkv = s.B * s.H_kv;
  const int ld = static_cast<int>(fp8_vt_ld(s.N_kv));
  uint8_t* vt = static_cast<uint8_t*>(workspace);
  CUtensorMap tq, tk, tvt, to;
  fa_status st;
  // E4M3 operands: 128-byte rows (d = 64 is zero-extended by the out-of-bounds fill)
  if ((st = make_map(&tq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, s.N_q, BH, 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
    return st;
  if ((st = make_map(&tk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, s.N_kv, BHkv, 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
    return st;
  if ((st = make_map(&tvt, vt, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.N_kv, s.d, BHkv, 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B, ld)) != FA_OK)
    return st;
  if ((st = make_bf16_map(&to, o, s.d, s.N_q, BH, 32)) != FA_OK) return st;

  {
    const dim3 grid((s.N_kv + fa::kTrKeys - 1) / fa::kTrKeys, (s.d + 63) / 64, BHkv);
    if (grid.z > 65535) return set_err(FA_ERR_UNSUPPORTED, "B*H_kv > 65535 for the fp8 path");
    ProfileScope prof(5, stream);
    fa::fa_fp8_transpose_v<<<grid, 256, 0, stream>>>(static_cast<const uint8_t*>(v8), vt, s.N_kv,
                                                      s.d, ld);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fp8 V transpose launch");

  fa::Fp8Params p;
  p.lse = lse;
  p.status = ds->status;
  p.N = s.N_q;
  p.N_kv = s.N_kv;
  p.BH = BH;
  p.group = s.H / s.H_kv;
  p.off = s.off();
  p.n_qblocks = (s.N_q + 255) / 256;
  p.hgroup = fwd_head_group(s, 2.0 * s.d);
  p.o_boxes = (s.d + 63) / 64;
  p.scale_log2 = s.scale * 1.4426950408889634f * q_descale * k_descale;
  p.o_scale = v_descale;
  const long long grid = 1LL * p.n_qblocks * BH;
  if (grid >= (1LL << 31)) return set_err(FA_ERR_UNSUPPORTED, "grid too large");
  {
    ProfileScope prof(4, stream);
    kern<<<static_cast<unsigned>(grid), fa::kFwdThreads, L::kAlloc, stream>>>(tq, tk, tvt, to, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fp8 forward launch");
  return FA_OK;
}

fa_status fp8_checked(const void* q8, const void* k8, const void* v8, float qd, float kd,
                      float vd, void* o, float* lse, const Shape& s, void* workspace,
                      size_t workspace_bytes, void* stream) {
  fa_status st = check_shape(s);
  if (st != FA_OK) return st;
  if (s.d > 128) return set_err(FA_ERR_UNSUPPORTED, "the FP8 forward supports d <= 128");
  if (!q8 || !k8 || !v8 || !o || !lse) return set_err(FA_ERR_INVALID_ARG, "null pointer argument");
  for (float x : {qd, kd, vd})
    if (!std::isfinite(x) || !(x > 0.f))
      return set_err(FA_ERR_INVALID_ARG, "descale factors must be finite and > 0");
  const void* ptrs[6] = {q8, k8, v8, o, lse, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return set_err(FA_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  const size_t need = fp8_workspace(s);
  if (!workspace || workspace_bytes < need)
    return set_err(FA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes,
                   need);
  const size_t qb = static_cast<size_t>(s.B) * s.H * s.N_q * s.d;
  const size_t kvb = static_cast<size_t>(s.B) * s.H_kv * s.N_kv * s.d;
  const void* ins[3] = {q8, k8, v8};
  const size_t insz[3] = {qb, kvb, kvb};
  void* outs[3] = {o, lse, workspace};
  const size_t outsz[3] = {s.q_bytes(), s.lse_bytes(), need};
  for (int a = 0; a < 3; ++a) {
    for (int b = 0; b < 3; ++b)
      if (overlaps(outs[a], outsz[a], ins[b], insz[b]))
        return set_err(FA_ERR_INVALID_ARG, "outputs/workspace must not alias inputs");
    for (int b = a + 1; b < 3; ++b)
      if (overlaps(outs[a], outsz[a], outs[b], outsz[b]))
        return set_err(FA_ERR_INVALID_ARG, "outputs/workspace must not overlap each other");
  }
  DeviceState* ds = device_state(&st);
  if (!ds) return st;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return s.mask != 0
             ? launch_fwd_fp8<true>(ds, q8, k8, v8, qd, kd, vd, o, lse, workspace, s, cs)
             : launch_fwd_fp8<false>(ds, q8, k8, v8, qd, kd, vd, o, lse, workspace, s, cs);
}

Shape from_public(const fa_attn_shape* p) {
  return Shape{p->B, p->H, p->H_kv, p->N_q, p->N_kv, p->d, p->scale, p->mask};
}

// ---- failure-detection self-test ----
// One thread waits, through the same bounded mbar_wait the attention kernels use, on an mbarrier
// that nothing ever arrives at. The wait gives up after `limit_ns`, the kernel records
// FA_ERR_TIMEOUT in the status word exactly as a timed-out attention kernel does, and returns.
__global__ void fa_selftest_timeout_kernel(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar_storage;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  const uint32_t bar = fa::smem_u32(&bar_storage);
  fa::mbar_init(bar, 1);
  fa::fence_barrier_init();
  if (!fa::mbar_wait(bar, 0, &abort_flag, limit_ns)) atomicExch(status, FA_ERR_TIMEOUT);
}

// ---- fa_bwd_noalloc: backward whose scratch is built into the library ----
// The backward needs scratch (fp32 dQ accumulator, row terms D and -lse*log2e). For callers that
// cannot allocate device memory, fa_bwd_noalloc uses this file-scope array instead of a
// caller-provided workspace. Every GPU that loads this library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
// In-kernel timeout code of fa_bwd_noalloc calls (the hang guard of the bounded waits).
static __device__ int g_noalloc_status;

struct NoAllocDevice {
  bool ready = false;
  void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int* status = nullptr;    // device address of g_noalloc_status on this device
  bool bwd_attr[2][2][2] = {};
  bool bwd128_attr[6] = {};
  int n_sm = 0;
  bool bwd256_attr[2] = {};
};

void copy_flags(std::atomic<bool> (&dst)[2][2][2], const bool (&src)[2][2][2]) {
  for (int a = 0; a < 2; ++a)
    for (int b = 0; b < 2; ++b)
      for (int c = 0; c < 2; ++c) dst[a][b][c].store(src[a][b][c]);
}
void copy_flags(bool (&dst)[2][2][2], const std::atomic<bool> (&src)[2][2][2]) {
  for (int a = 0; a < 2; ++a)
    for (int b = 0; b < 2; ++b)
      for (int c = 0; c < 2; ++c) dst[a][b][c] = src[a][b][c].load();
}
NoAllocDevice g_noalloc[kMaxDevices];

}  // namespace

extern "C" {

const char* fa_last_error_string(void) { return g_err; }

const char* fa_version(void) { return "exact_io_aware_66_b200 0.1 (sm_100a)"; }

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, void* stream) {
  g_err[0] = '\0';
  return fwd_checked(q, k, v, o, lse, Shape{B, H, H, N, N, d, scale, causal ? 1 : 0}, stream);
}

fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                    const fa_attn_shape* shape, const fa_dropout* dropout, void* stream) {
  g_err[0] = '\0';
  if (!shape) return set_err(FA_ERR_INVALID_ARG, "null shape");
  Shape s = from_public(shape);
  const fa_status st = apply_dropout(s, dropout);
  if (st != FA_OK) return st;
  return fwd_checked(q, k, v, o, lse, s, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 96 && d != 128 && d != 256)) return 0;
  return fa::bwd_workspace_bytes(static_cast<size_t>(B) * H, N, d);
}

size_t fa_bwd_ex_workspace_size(const fa_attn_shape* shape) {
  if (!shape) return 0;
  const Shape s = from_public(shape);
  const char saved = g_err[0];
  const bool ok = check_shape(s) == FA_OK;
  if (saved == '\0') g_err[0] = '\0';
  return ok ? bwd_workspace(s) : 0;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                 void* stream) {
  g_err[0] = '\0';
  return bwd_checked(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes,
                     Shape{B, H, H, N, N, d, scale, causal ? 1 : 0}, stream);
}

fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dO,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, const fa_attn_shape* shape,
                    const fa_dropout* dropout, void* stream) {
  g_err[0] = '\0';
  if (!shape) return set_err(FA_ERR_INVALID_ARG, "null shape");
  Shape s = from_public(shape);
  const fa_status st = apply_dropout(s, dropout);
  if (st != FA_OK) return st;
  return bwd_checked(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, s, stream);
}

size_t fa_fwd_fp8_workspace_size(const fa_attn_shape* shape) {
  if (!shape) return 0;
  const Shape s = from_public(shape);
  const char saved = g_err[0];
  const bool ok = check_shape(s) == FA_OK && s.d <= 128;
  if (saved == '\0') g_err[0] = '\0';
  return ok ? fp8_workspace(s) : 0;
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_descale,
                     float k_descale, float v_descale, void* o, float* lse,
                     const fa_attn_shape* shape, void* workspace, size_t workspace_bytes,
                     void* stream) {
  g_err[0] = '\0';
  if (!shape) return set_err(FA_ERR_INVALID_ARG, "null shape");
  return fp8_checked(q8, k8, v8, q_descale, k_descale, v_descale, o, lse, from_public(shape),
                     workspace, workspace_bytes, stream);
}

fa_status fa_profile_enable(int on) {
  g_prof.on = on != 0;
  return FA_OK;
}

fa_status fa_profile_read(double* ms, long long* launches, int n) {
  g_err[0] = '\0';
  if (!ms || !launches || n < kKernelKinds)
    return set_err(FA_ERR_INVALID_ARG, "fa_profile_read needs arrays of %d entries", kKernelKinds);
  for (int i = 0; i < n; ++i) {
    ms[i] = 0.0;
    launches[i] = 0;
  }
  fa_status st = FA_OK;
  for (const ProfileRec& r : g_prof.recs) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.stop);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.start, r.stop);
    if (e != cudaSuccess && st == FA_OK) st = cuda_err(e, "profile event");
    ms[r.kind] += t;
    launches[r.kind] += 1;
    g_prof.pool.push_back(r.start);
    g_prof.pool.push_back(r.stop);
  }
  g_prof.recs.clear();
  return st;
}

const char* fa_kernel_name(int kind) {
  return (kind >= 0 && kind < kKernelKinds) ? kKernelNames[kind] : "";
}

// Backward with built-in scratch (see include/fa.h). Allocates nothing: no cudaMalloc, no
// cudaFree, no allocating library routine. Set-up (once per device, on the first call with
// that device current): the device addresses of the scratch array and of the status word are
// taken with cudaGetSymbolAddress.
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const void* dO, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, float scale, int causal, void* stream) {
  g_err[0] = '\0';
  const Shape shape{B, H, H, N, N, d, scale, causal ? 1 : 0};
  fa_status st = check_shape(shape);
  if (st != FA_OK) return st;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need > kNoAllocScratchBytes)
    return set_err(FA_ERR_UNSUPPORTED,
                   "fa_bwd_noalloc: these sizes need %zu bytes of scratch, more than the %zu "
                   "bytes built into the library (use fa_bwd with a workspace)",
                   need, kNoAllocScratchBytes);
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv)
    return set_err(FA_ERR_INVALID_ARG, "null pointer argument");
  const void* ptrs[9] = {q, k, v, o, dO, lse, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return set_err(FA_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  const size_t tbytes = static_cast<size_t>(B) * H * N * d * 2;
  const size_t lbytes = static_cast<size_t>(B) * H * N * 4;
  const void* ins[6] = {q, k, v, o, dO, lse};
  const size_t insz[6] = {tbytes, tbytes, tbytes, tbytes, tbytes, lbytes};
  void* outs[3] = {dq, dk, dv};
  for (int a = 0; a < 3; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], tbytes, ins[b], insz[b]))
        return set_err(FA_ERR_INVALID_ARG, "outputs must not alias inputs");
    for (int b = a + 1; b < 3; ++b)
      if (overlaps(outs[a], tbytes, outs[b], tbytes))
        return set_err(FA_ERR_INVALID_ARG, "outputs must not overlap each other");
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return set_err(FA_ERR_CUDA, "device index %d out of range", dev);
  DeviceState local;  // per-call view: status word and attribute flags of the no-alloc path
  {
    std::lock_guard<std::mutex> lock(g_mu);
    NoAllocDevice& nd = g_noalloc[dev];
    if (!nd.ready) {
      int major = 0, minor = 0;
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
      if (!(major == 10 && minor == 0))
        return set_err(FA_ERR_CUDA, "device %d is not an sm_100 (B200) GPU", dev);
      void* scratch = nullptr;
      e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_err(e, "cudaGetSymbolAddress(scratch)");
      void* status = nullptr;
      e = cudaGetSymbolAddress(&status, g_noalloc_status);
      if (e != cudaSuccess) return cuda_err(e, "cudaGetSymbolAddress(status)");
      nd.scratch = scratch;
      nd.status = static_cast<int*>(status);
      cudaDeviceGetAttribute(&nd.n_sm, cudaDevAttrMultiProcessorCount, dev);
      nd.ready = true;
    }
    local.status = nd.status;
    local.checked = local.is_sm100 = true;
    local.n_sm = nd.n_sm;
    copy_flags(local.bwd_attr, nd.bwd_attr);
    for (int c = 0; c < 6; ++c) local.bwd128_attr[c].store(nd.bwd128_attr[c]);
    for (int c = 0; c < 2; ++c) local.bwd256_attr[c].store(nd.bwd256_attr[c]);
  }
  // The first kernel of the backward rewrites every scratch byte the later ones read (dQ
  // accumulator zeroed, D and -lse*log2e recomputed), so the previous call's contents do not
  // matter.
  st = bwd_dispatch(&local, q, k, v, o, dO, lse, dq, dk, dv, g_noalloc[dev].scratch, shape,
                    static_cast<cudaStream_t>(stream));
  {
    std::lock_guard<std::mutex> lock(g_mu);
    copy_flags(g_noalloc[dev].bwd_attr, local.bwd_attr);
    for (int c = 0; c < 6; ++c) g_noalloc[dev].bwd128_attr[c] = local.bwd128_attr[c].load();
    for (int c = 0; c < 2; ++c) g_noalloc[dev].bwd256_attr[c] = local.bwd256_attr[c].load();
  }
  return st;
}

fa_status fa_selftest_timeout(int limit_us, void* stream) {
  g_err[0] = '\0';
  if (limit_us < 1 || limit_us > 10000000)
    return set_err(FA_ERR_INVALID_ARG, "limit_us must be in [1, 10^7] (got %d)", limit_us);
  fa_status st;
  DeviceState* ds = device_state(&st);
  if (!ds) return st;
  fa_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      ds->status, 1000ull * static_cast<unsigned long long>(limit_us));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "fa_selftest_timeout launch");
  return FA_OK;
}

fa_status fa_debug_stall_next(int kind, int skip, int limit_us) {
  g_err[0] = '\0';
  if (kind == -1) {
    g_stall.kind = -1;
    return FA_OK;
  }
  if (kind != 0 && kind != 2)
    return set_err(FA_ERR_INVALID_ARG, "kind must be 0 (forward), 2 (backward main) or -1");
  if (skip < 0) return set_err(FA_ERR_INVALID_ARG, "skip must be >= 0 (got %d)", skip);
  if (limit_us < 1 || limit_us > 10000000)
    return set_err(FA_ERR_INVALID_ARG, "limit_us must be in [1, 10^7] (got %d)", limit_us);
  g_stall.kind = kind;
  g_stall.skip = skip;
  g_stall.limit_ns = 1000ull * static_cast<unsigned long long>(limit_us);
  return FA_OK;
}

fa_status fa_check_status(void* stream) {
  g_err[0] = '\0';
  // Allocates nothing: it reads the words that exist (the allocating entry points' word once
  // it has been created, and the built-in word of fa_bwd_noalloc once that path is set up),
  // so callers of fa_bwd_noalloc can use it too.
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return set_err(FA_ERR_CUDA, "device index %d out of range", dev);
  int* words[2] = {nullptr, nullptr};
  {
    std::lock_guard<std::mutex> lock(g_mu);
    words[0] = g_dev[dev].status;
    if (g_noalloc[dev].ready) words[1] = g_noalloc[dev].status;
  }
  e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_err(e, "cudaStreamSynchronize");
  int code = 0;
  for (int* w : words) {
    if (!w) continue;
    int h = 0;
    e = cudaMemcpy(&h, w, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_err(e, "read status word");
    if (h != 0) {
      e = cudaMemset(w, 0, sizeof(int));
      if (e != cudaSuccess) return cuda_err(e, "clear status word");
      if (code == 0) code = h;
    }
  }
  if (code != 0)
    return set_err(FA_ERR_TIMEOUT, code == 7 ? "a kernel found its shared memory misaligned (code 7)"
                                             : "a bounded in-kernel wait timed out (code %d)", code);
  return FA_OK;
}

}  // extern "C"
