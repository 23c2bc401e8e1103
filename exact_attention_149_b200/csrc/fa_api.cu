// Host side of the C ABI declared in include/fa.h: argument validation, TMA
// descriptor encoding, launch configuration. The whole library is this one
// translation unit (kernels are included as headers), so the device status
// word in ptx.cuh is shared by every kernel and read back here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/fa.h"
#include "ptx.cuh"
#include "fwd_kernel.cuh"
#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"

namespace {

thread_local std::string g_last_error;

fa_status fail(fa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

fa_status ok() {
  g_last_error.clear();
  return FA_OK;
}

#define FA_CUDA_CHECK(expr)                                                            \
  do {                                                                                 \
    cudaError_t e_ = (expr);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return fail(FA_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));       \
  } while (0)

// ---------------------------------------------------------------------------
// device checks
// ---------------------------------------------------------------------------
fa_status check_device() {
  static std::mutex mu;
  static int arch_state[128] = {0};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 128) return fail(FA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (arch_state[dev] == 0) {
    int major = 0, minor = 0;
    FA_CUDA_CHECK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    FA_CUDA_CHECK(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    arch_state[dev] = (major == 10 && minor == 0) ? 1 : 2;
    if (arch_state[dev] == 2)
      return fail(FA_ERR_UNSUPPORTED, "device %d has compute capability %d.%d; this library is built for sm_100a (10.0)",
                  dev, major, minor);
  }
  if (arch_state[dev] != 1) return fail(FA_ERR_UNSUPPORTED, "device %d is not compute capability 10.0", dev);
  return FA_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D map over a (tokens, heads, D) row-major 16-bit tensor; box = 64 columns
// (128 B, one swizzle row) x 1 head x `rows` tokens, 128-byte swizzle.
// tok_stride: elements from one token's row to the next (default H * D; the
// qkv-packed layout interleaves three tensors per token)
fa_status make_map_thd(CUtensorMap* map, const void* base, fa_dtype dt, int D, int H, long long T,
                       int rows, long long tok_stride = -1) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  const long long ts = tok_stride >= 0 ? tok_stride : static_cast<long long>(H) * D;
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(ts) * 2};
  cuuint32_t box[3] = {64u, 1u, static_cast<cuuint32_t>(rows)};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = enc(map, dt == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FA_OK;
}

// 3-D map over a (tokens, heads, D) tensor of one-byte FP8 elements; box =
// 128 columns (128 B, one swizzle row) x 1 head x `rows` tokens, 128-byte
// swizzle; D a multiple of 128.
fa_status make_map_thd8(CUtensorMap* map, const void* base, int D, int H, long long T, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H) * D};
  cuuint32_t box[3] = {128u, 1u, static_cast<cuuint32_t>(rows)};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FA_OK;
}

// int8 / int4 cache (T, H, row_bytes) bytes, row_bytes = D (int8) or D / 2
// (int4): one box is `rows` tokens x the whole row of one head; 128-byte rows
// arrive with the 128-byte swizzle (16-byte group g of row r at g ^ (r & 7)),
// 64-byte rows with the 64-byte swizzle when swz64 is set (group g of row r
// at g ^ ((r >> 1) & 3)), unswizzled otherwise
fa_status make_map_i8(CUtensorMap* map, const void* base, int D, int H, long long T, int rows,
                      bool swz64 = false) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H) * D};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(D), 1u, static_cast<cuuint32_t>(rows)};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                            : (swz64 && D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE),
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FA_OK;
}

// ---------------------------------------------------------------------------
// optional per-kernel timing (events around each launch on the caller's stream)
// ---------------------------------------------------------------------------
struct TimingRecord {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_timing_mu;
bool g_timing_on = false;
std::vector<TimingRecord> g_timing_records;

cudaEvent_t timing_event() {
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// RAII helper: records an event before the launch in its scope and one after.
class KernelTimer {
 public:
  KernelTimer(const char* name, cudaStream_t st) : name_(name), st_(st) {
    std::lock_guard<std::mutex> lock(g_timing_mu);
    if (!g_timing_on) return;
    start_ = timing_event();
    if (start_ != nullptr) cudaEventRecord(start_, st_);
  }
  ~KernelTimer() {
    if (start_ == nullptr) return;
    cudaEvent_t stop = timing_event();
    if (stop == nullptr) {
      cudaEventDestroy(start_);
      return;
    }
    cudaEventRecord(stop, st_);
    std::lock_guard<std::mutex> lock(g_timing_mu);
    g_timing_records.push_back({name_, start_, stop});
  }
  KernelTimer(const KernelTimer&) = delete;
  KernelTimer& operator=(const KernelTimer&) = delete;

 private:
  const char* name_;
  cudaStream_t st_;
  cudaEvent_t start_ = nullptr;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// common option validation for fwd/bwd
// ALiBi slopes: NULL, or a 4-byte aligned device float array read at
// b * batch_stride + h (batch_stride 0: one (Hq) vector for every sequence).
fa_status check_alibi(const float* slopes, int batch_stride, int Hq) {
  if (slopes == nullptr) return FA_OK;
  if (reinterpret_cast<uintptr_t>(slopes) & 3u)
    return fail(FA_ERR_INVALID_ARG, "alibi_slopes must be 4-byte aligned");
  if (batch_stride != 0 && batch_stride < Hq)
    return fail(FA_ERR_INVALID_ARG, "alibi_batch_stride must be 0 or >= Hq (got %d)", batch_stride);
  return FA_OK;
}

// allow256: the call also takes D = 256 (forward and backward)
fa_status check_common(int B, int Hq, int Hkv, int S, int D, float scale, int wl, int wr,
                       float softcap, fa_dtype dt, const int32_t* cu, int total, bool allow256 = false) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1)
    return fail(FA_ERR_INVALID_ARG, "B, Hq, Hkv and S must be >= 1 (got %d, %d, %d, %d)", B, Hq, Hkv, S);
  if (Hq % Hkv != 0) return fail(FA_ERR_INVALID_ARG, "Hq (%d) must be an integer multiple of Hkv (%d)", Hq, Hkv);
  if (D != 64 && D != 128 && !(allow256 && D == 256))
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128%s)", D, allow256 ? " or 256" : "");
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
  if (wl < -1 || wr < -1) return fail(FA_ERR_INVALID_ARG, "window bounds must be >= -1 (got %d, %d)", wl, wr);
  if (!(softcap >= 0.f) || !std::isfinite(softcap))
    return fail(FA_ERR_INVALID_ARG, "softcap must be finite and >= 0");
  if (dt != FA_BF16 && dt != FA_FP16) return fail(FA_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dt));
  if (cu != nullptr && total < 1) return fail(FA_ERR_INVALID_ARG, "total_tokens must be >= 1 with cu_seqlens");
  if (static_cast<long long>(Hq) * D * 2 % 16 != 0 || static_cast<long long>(Hkv) * D * 2 % 16 != 0)
    return fail(FA_ERR_INVALID_ARG, "row strides must be multiples of 16 bytes");
  const long long T = cu ? static_cast<long long>(total) : static_cast<long long>(B) * S;
  if (T > (1ll << 31) - 1) return fail(FA_ERR_INVALID_ARG, "too many tokens");
  return FA_OK;
}

template <typename K>
fa_status set_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess)
    return fail(FA_ERR_CUDA, "cudaFuncSetAttribute(smem=%d) failed: %s", bytes, cudaGetErrorString(e));
  return FA_OK;
}

// blocks of a forward launch: n_qblocks per (sequence, head), or, with
// seq_blocks (varlen), the bound Hq * (ceil(total / rows) + B) on the blocks
// that sequences of those lengths need
inline long long fwd_grid(const fa::FwdParams& p, int rows) {
  if (p.seq_blocks) return static_cast<long long>(p.Hq) * ((p.total + rows - 1) / rows + p.B);
  return static_cast<long long>(p.n_qblocks) * p.B * p.Hq;
}
// varlen launches with at most this many sequences number their blocks
// sequence by sequence (one warp's two lanes a sequence find each block's)
constexpr int kSeqBlocksMaxB = 64;

template <int kD, bool kBF16, bool kCap>
fa_status launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const fa::FwdParams& p, cudaStream_t st) {
  using Sh = fa::FwdShape<kD>;
  auto kern = p.alibi ? fa::fwd_kernel<kD, kBF16, kCap, true> : fa::fwd_kernel<kD, kBF16, kCap, false>;
  fa_status s = set_smem(kern, Sh::kSmemBytes);
  if (s != FA_OK) return s;
  const long long grid = fwd_grid(p, Sh::kRows);
  if (grid > 0x7fffffffll) return fail(FA_ERR_INVALID_ARG, "grid too large");
  {
    KernelTimer timer("fwd", st);
    kern<<<static_cast<unsigned>(grid), Sh::kThreads, Sh::kSmemBytes, st>>>(tq, tk, tv, p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "fwd launch failed: %s", cudaGetErrorString(e));
  return FA_OK;
}

template <int kD, bool kBF16, bool kCap>
fa_status launch_fwd8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      const fa::FwdParams& p, cudaStream_t st) {
  using Sh = fa::FwdShape<kD, true>;
  auto kern = p.alibi ? fa::fwd_kernel<kD, kBF16, kCap, true, true>
                      : fa::fwd_kernel<kD, kBF16, kCap, false, true>;
  fa_status s = set_smem(kern, Sh::kSmemBytes);
  if (s != FA_OK) return s;
  const long long grid = fwd_grid(p, Sh::kRows);
  if (grid > 0x7fffffffll) return fail(FA_ERR_INVALID_ARG, "grid too large");
  {
    KernelTimer timer("fwd_fp8", st);
    kern<<<static_cast<unsigned>(grid), Sh::kThreads, Sh::kSmemBytes, st>>>(tq, tk, tv, p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "fwd_fp8 launch failed: %s", cudaGetErrorString(e));
  return FA_OK;
}

}  // namespace

namespace fa {

// Evaluates one of the FMA-pipe approximations the kernels use, and the CUDA
// math function it stands in for, on the same inputs (two values per thread,
// as the kernels evaluate them): 0 ex2_poly2 / exp2f, 1 tanh_poly2 / tanhf,
// 2 the degree-2 folded tanh (tanh_fold2 with a = c = 1) / tanhf.
__global__ void poly_selftest_kernel(int which, const float* x, float* out_poly, float* out_ref,
                                     int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  float2 r, ref;
  if (which == 0) {
    r = ex2_poly2(v);
    ref = make_float2(exp2f(v.x), exp2f(v.y));
  } else if (which == 1) {
    r = tanh_poly2(v);
    ref = make_float2(tanhf(v.x), tanhf(v.y));
  } else {
    float pk[3];
    fold_tanh(kTanhLo, 1.f, 1.f, pk);
    r = tanh_fold2(v, pk);
    ref = make_float2(tanhf(v.x), tanhf(v.y));
  }
  out_poly[i] = r.x;
  out_ref[i] = ref.x;
  if (i + 1 < n) {
    out_poly[i + 1] = r.y;
    out_ref[i + 1] = ref.y;
  }
}

}  // namespace fa

namespace {

// q, k, v rows of token t start at t * q_tok (t * kv_tok) elements
fa_status fwd_impl(const void* q, const void* k, const void* v, long long q_tok, long long kv_tok,
                   void* out, float* lse, int B, int Hq, int Hkv, int S, int D, float scale,
                   int causal, int window_left, int window_right, float softcap,
                   const float* alibi_slopes, int alibi_batch_stride, const int32_t* cu_seqlens,
                   int total_tokens, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !out || !lse) return fail(FA_ERR_INVALID_ARG, "fa_fwd: null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: tensors must be 16-byte aligned");
  fa_status s = check_common(B, Hq, Hkv, S, D, scale, window_left, window_right, softcap, dtype,
                             cu_seqlens, total_tokens, true);
  if (s != FA_OK) return s;
  if ((s = check_alibi(alibi_slopes, alibi_batch_stride, Hq)) != FA_OK) return s;
  if ((s = check_device()) != FA_OK) return s;

  const long long T = cu_seqlens ? total_tokens : static_cast<long long>(B) * S;
  CUtensorMap tq, tk, tv;
  if ((s = make_map_thd(&tq, q, dtype, D, Hq, T, 128, q_tok)) != FA_OK) return s;
  if ((s = make_map_thd(&tk, k, dtype, D, Hkv, T, 128, kv_tok)) != FA_OK) return s;
  if ((s = make_map_thd(&tv, v, dtype, D, Hkv, T, 128, kv_tok)) != FA_OK) return s;

  fa::FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.total = static_cast<int>(T);
  p.group = Hq / Hkv;
  const int rows_per_cta = D == 256 ? fa::FwdShape<256>::kRows : fa::FwdShape<128>::kRows;
  p.n_qblocks = (S + rows_per_cta - 1) / rows_per_cta;
  const float log2e = 1.4426950408889634f;
  p.scale_log2 = scale * log2e;
  p.softcap = softcap;
  p.cap_in = softcap > 0.f ? scale / softcap : 0.f;
  p.cap_out_log2 = softcap * log2e;
  p.wl = window_left;
  p.wr = causal ? 0 : window_right;
  p.o = out;
  p.lse = lse;
  p.cu_seqlens = cu_seqlens;
  p.seq_blocks = cu_seqlens != nullptr && B <= kSeqBlocksMaxB;
  p.alibi = alibi_slopes;
  p.alibi_bstride = alibi_batch_stride;
  p.wait_ns = fa::kWaitTimeoutNs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool cap = softcap > 0.f;
  if (D == 256) {
    if (dtype == FA_BF16)
      s = cap ? launch_fwd<256, true, true>(tq, tk, tv, p, st) : launch_fwd<256, true, false>(tq, tk, tv, p, st);
    else
      s = cap ? launch_fwd<256, false, true>(tq, tk, tv, p, st) : launch_fwd<256, false, false>(tq, tk, tv, p, st);
  } else if (D == 128) {
    if (dtype == FA_BF16)
      s = cap ? launch_fwd<128, true, true>(tq, tk, tv, p, st) : launch_fwd<128, true, false>(tq, tk, tv, p, st);
    else
      s = cap ? launch_fwd<128, false, true>(tq, tk, tv, p, st) : launch_fwd<128, false, false>(tq, tk, tv, p, st);
  } else {
    if (dtype == FA_BF16)
      s = cap ? launch_fwd<64, true, true>(tq, tk, tv, p, st) : launch_fwd<64, true, false>(tq, tk, tv, p, st);
    else
      s = cap ? launch_fwd<64, false, true>(tq, tk, tv, p, st) : launch_fwd<64, false, false>(tq, tk, tv, p, st);
  }
  if (s != FA_OK) return s;
  return ok();
}

}  // namespace

extern "C" {

const char* fa_last_error(void) { return g_last_error.c_str(); }

const char* fa_version(void) { return "exact-attention-b200 0.1.0 (sm_100a)"; }

fa_status fa_kernel_timing_enable(int enable) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  g_timing_on = enable != 0;
  return ok();
}

fa_status fa_kernel_timing_reset(void) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  for (auto& r : g_timing_records) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_timing_records.clear();
  return ok();
}

fa_status fa_kernel_timing_read(const char* name, float* total_ms, int* launches) {
  if (name == nullptr || total_ms == nullptr || launches == nullptr)
    return fail(FA_ERR_INVALID_ARG, "fa_kernel_timing_read: null argument");
  std::lock_guard<std::mutex> lock(g_timing_mu);
  float sum = 0.f;
  int n = 0;
  for (auto& r : g_timing_records) {
    if (std::strcmp(r.name, name) != 0) continue;
    cudaError_t e = cudaEventSynchronize(r.stop);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.start, r.stop);
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "timing event: %s", cudaGetErrorString(e));
    sum += ms;
    ++n;
  }
  *total_ms = sum;
  *launches = n;
  return ok();
}

fa_status fa_get_device_status(int* status_out) {
  if (status_out == nullptr) return fail(FA_ERR_INVALID_ARG, "status_out is NULL");
  int v = 0, site = 0;
  const int zero = 0;
  FA_CUDA_CHECK(cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof(int)));
  FA_CUDA_CHECK(cudaMemcpyFromSymbol(&site, fa::g_wait_site, sizeof(int)));
  FA_CUDA_CHECK(cudaMemcpyToSymbol(fa::g_device_status, &zero, sizeof(int)));
  FA_CUDA_CHECK(cudaMemcpyToSymbol(fa::g_wait_site, &zero, sizeof(int)));
  if (v == fa::kDevTimeout) {
    *status_out = static_cast<int>(FA_ERR_TIMEOUT);
    // the message names the wait that gave up first (when the kernel
    // recorded one: 100 * kernel + wait, see bwd_wait)
    g_last_error = "a kernel gave up on a bounded wait";
    if (site != 0) g_last_error += " (wait site " + std::to_string(site) + ")";
    return FA_OK;
  }
  if (v == fa::kDevBadIndex)
    *status_out = static_cast<int>(FA_ERR_INVALID_ARG);
  else
    *status_out = 0;
  return ok();
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                 int Hkv, int S, int D, float scale, int causal, int window_left, int window_right,
                 float softcap, const float* alibi_slopes, int alibi_batch_stride,
                 const int32_t* cu_seqlens, int total_tokens, fa_dtype dtype, void* stream) {
  return fwd_impl(q, k, v, -1, -1, out, lse, B, Hq, Hkv, S, D, scale, causal, window_left,
                  window_right, softcap, alibi_slopes, alibi_batch_stride, cu_seqlens, total_tokens,
                  dtype, stream);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int Hq, int Hkv, int S, int D, float scale, float q_descale, float k_descale,
                     float v_descale, int causal, int window_left, int window_right, float softcap,
                     const float* alibi_slopes, int alibi_batch_stride, const int32_t* cu_seqlens,
                     int total_tokens, fa_dtype out_dtype, void* stream) {
  if (!q || !k || !v || !out || !lse) return fail(FA_ERR_INVALID_ARG, "fa_fwd_fp8: null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd_fp8: tensors must be 16-byte aligned");
  if (D != 128 && D != 256)
    return fail(FA_ERR_UNSUPPORTED, "fa_fwd_fp8: head dim %d not supported (128 or 256)", D);
  fa_status s = check_common(B, Hq, Hkv, S, D, scale, window_left, window_right, softcap, out_dtype,
                             cu_seqlens, total_tokens, true);
  if (s != FA_OK) return s;
  for (float d : {q_descale, k_descale, v_descale})
    if (!(d > 0.f) || !std::isfinite(d))
      return fail(FA_ERR_INVALID_ARG, "fa_fwd_fp8: descales must be finite and > 0");
  if ((s = check_alibi(alibi_slopes, alibi_batch_stride, Hq)) != FA_OK) return s;
  if ((s = check_device()) != FA_OK) return s;

  const long long T = cu_seqlens ? total_tokens : static_cast<long long>(B) * S;
  CUtensorMap tq, tk, tv;
  if ((s = make_map_thd8(&tq, q, D, Hq, T, 128)) != FA_OK) return s;
  if ((s = make_map_thd8(&tk, k, D, Hkv, T, 128)) != FA_OK) return s;
  if ((s = make_map_thd8(&tv, v, D, Hkv, T, 128)) != FA_OK) return s;

  // the logits' scale carries both input descales; the output carries v's
  const double eff = static_cast<double>(scale) * q_descale * k_descale;
  if (!std::isfinite(eff)) return fail(FA_ERR_INVALID_ARG, "fa_fwd_fp8: scale * descales overflows");
  fa::FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.total = static_cast<int>(T);
  p.group = Hq / Hkv;
  const int rows_per_cta = D == 256 ? fa::FwdShape<256, true>::kRows : fa::FwdShape<128, true>::kRows;
  p.n_qblocks = (S + rows_per_cta - 1) / rows_per_cta;
  p.scale_log2 = static_cast<float>(eff * 1.4426950408889634);
  p.softcap = softcap;
  p.cap_in = softcap > 0.f ? static_cast<float>(eff / softcap) : 0.f;
  p.cap_out_log2 = static_cast<float>(static_cast<double>(softcap) * 1.4426950408889634);
  p.wl = window_left;
  p.wr = causal ? 0 : window_right;
  p.o = out;
  p.lse = lse;
  p.cu_seqlens = cu_seqlens;
  p.seq_blocks = cu_seqlens != nullptr && B <= kSeqBlocksMaxB;
  p.alibi = alibi_slopes;
  p.alibi_bstride = alibi_batch_stride;
  p.o_scale = v_descale;
  p.wait_ns = fa::kWaitTimeoutNs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool cap = softcap > 0.f;
  const bool bf = out_dtype == FA_BF16;
  if (D == 256)
    s = bf ? (cap ? launch_fwd8<256, true, true>(tq, tk, tv, p, st) : launch_fwd8<256, true, false>(tq, tk, tv, p, st))
           : (cap ? launch_fwd8<256, false, true>(tq, tk, tv, p, st) : launch_fwd8<256, false, false>(tq, tk, tv, p, st));
  else
    s = bf ? (cap ? launch_fwd8<128, true, true>(tq, tk, tv, p, st) : launch_fwd8<128, true, false>(tq, tk, tv, p, st))
           : (cap ? launch_fwd8<128, false, true>(tq, tk, tv, p, st) : launch_fwd8<128, false, false>(tq, tk, tv, p, st));
  if (s != FA_OK) return s;
  return ok();
}

fa_status fa_selftest_fwd_timeout(const void* q, const void* k, const void* v, void* out, float* lse,
                                  int B, int H, int S, float scale, unsigned long long wait_limit_ns,
                                  fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !out || !lse) return fail(FA_ERR_INVALID_ARG, "fa_selftest_fwd_timeout: null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(FA_ERR_INVALID_ARG, "fa_selftest_fwd_timeout: tensors must be 16-byte aligned");
  if (wait_limit_ns < 1000000ull || wait_limit_ns > fa::kWaitTimeoutNs)
    return fail(FA_ERR_INVALID_ARG, "fa_selftest_fwd_timeout: the wait limit must lie in [1 ms, 4 s]");
  fa_status s = check_common(B, H, H, S, 128, scale, -1, -1, 0.f, dtype, nullptr, 0);
  if (s != FA_OK) return s;
  if ((s = check_device()) != FA_OK) return s;
  const long long T = static_cast<long long>(B) * S;
  CUtensorMap tq, tk, tv;
  if ((s = make_map_thd(&tq, q, dtype, 128, H, T, 128)) != FA_OK) return s;
  if ((s = make_map_thd(&tk, k, dtype, 128, H, T, 128)) != FA_OK) return s;
  if ((s = make_map_thd(&tv, v, dtype, 128, H, T, 128)) != FA_OK) return s;
  fa::FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.Hq = p.Hkv = H;
  p.S = S;
  p.total = static_cast<int>(T);
  p.group = 1;
  p.n_qblocks = (S + fa::FwdShape<128>::kRows - 1) / fa::FwdShape<128>::kRows;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wl = p.wr = -1;
  p.o = out;
  p.lse = lse;
  p.wait_ns = wait_limit_ns;
  using Sh = fa::FwdShape<128>;
  auto kern = dtype == FA_BF16 ? fa::fwd_kernel<128, true, false, false, false, true>
                               : fa::fwd_kernel<128, false, false, false, false, true>;
  if ((s = set_smem(kern, Sh::kSmemBytes)) != FA_OK) return s;
  const long long grid = static_cast<long long>(p.n_qblocks) * B * H;
  if (grid > 0x7fffffffll) return fail(FA_ERR_INVALID_ARG, "grid too large");
  kern<<<static_cast<unsigned>(grid), Sh::kThreads, Sh::kSmemBytes, static_cast<cudaStream_t>(stream)>>>(
      tq, tk, tv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "selftest launch failed: %s", cudaGetErrorString(e));
  return ok();
}

fa_status fa_selftest_poly(int which, const float* x, float* out_poly, float* out_ref, int n,
                           void* stream) {
  if (which < 0 || which > 2) return fail(FA_ERR_INVALID_ARG, "fa_selftest_poly: which must be 0, 1 or 2");
  if (n < 0 || (n > 0 && (!x || !out_poly || !out_ref)))
    return fail(FA_ERR_INVALID_ARG, "fa_selftest_poly: bad arguments");
  fa_status s = check_device();
  if (s != FA_OK) return s;
  if (n == 0) return ok();
  const int pairs = (n + 1) / 2;
  fa::poly_selftest_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      which, x, out_poly, out_ref, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "selftest launch failed: %s", cudaGetErrorString(e));
  return ok();
}

fa_status fa_fwd_qkvpacked(const void* qkv, void* out, float* lse, int B, int H, int S, int D,
                           float scale, int causal, int window_left, int window_right,
                           float softcap, const float* alibi_slopes, int alibi_batch_stride,
                           const int32_t* cu_seqlens, int total_tokens, fa_dtype dtype,
                           void* stream) {
  if (!qkv) return fail(FA_ERR_INVALID_ARG, "fa_fwd_qkvpacked: null qkv");
  if (H < 1 || (D != 64 && D != 128 && D != 256))
    return fail(D != 64 && D != 128 && D != 256 ? FA_ERR_UNSUPPORTED : FA_ERR_INVALID_ARG,
                "fa_fwd_qkvpacked: H must be >= 1 and D 64, 128 or 256");
  const long long hd = static_cast<long long>(H) * D;
  const uint16_t* base = static_cast<const uint16_t*>(qkv);
  return fwd_impl(base, base + hd, base + 2 * hd, 3 * hd, 3 * hd, out, lse, B, H, H, S, D, scale,
                  causal, window_left, window_right, softcap, alibi_slopes, alibi_batch_stride,
                  cu_seqlens, total_tokens, dtype, stream);
}

}  // extern "C"

#include "bwd_api.inc"
#include "decode_api.inc"
#include "noalloc_api.inc"
