// C-ABI entry points (include/svdq.h): argument validation on the host, the
// device-capability gate, tensor-map encoding and kernel launches.
#include <atomic>
#include <cstring>
#include <mutex>

#include "../../include/svdq.h"
#include "device.cuh"
#include "kernels.h"

namespace svdq {

// One error word per device (each device gets its own copy of this module).
__device__ unsigned g_error_word;

namespace {

std::atomic<unsigned long long> g_wait_ns{2000000000ull};
std::atomic<int> g_force_major{0}, g_force_minor{0};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_err_ptr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};
int g_major[kMaxDevices] = {-1};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device's capability, SM count and error-word address (cached).
svdq_status device_info(unsigned** err, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess) return SVDQ_ERR_CUDA;
    g_major[dev] = major;
    g_num_sms[dev] = sms;
    g_err_ptr[dev] = static_cast<unsigned*>(ptr);
  }
  int major = g_major[dev];
  if (g_force_major.load() != 0) major = g_force_major.load();
  if (major != 10) return SVDQ_ERR_UNSUPPORTED_ARCH;
  if (err) *err = g_err_ptr[dev];
  if (num_sms) *num_sms = g_num_sms[dev];
  return SVDQ_OK;
}

svdq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA; }

svdq_status check_common(svdq_precision p, int K, int r) {
  if (p != SVDQ_NVFP4 && p != SVDQ_INT4) return SVDQ_ERR_INVALID_ARG;
  if (K <= 0 || r < 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 64) return SVDQ_ERR_SHAPE;
  if (r % 16) return SVDQ_ERR_SHAPE;
  if (r > (p == SVDQ_NVFP4 ? 32 : 64)) return SVDQ_ERR_SHAPE;
  return SVDQ_OK;
}

}  // namespace

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

namespace {
EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && f)
      fn = reinterpret_cast<EncodeFn>(f);
  }
  return fn;
}
}  // namespace

namespace {

// Everything an encoding depends on (a map is a pure function of these).
struct TmapKey {
  uint64_t base, dims[3], strides[2];
  uint32_t box[3], rank, dtype, swz;
  bool operator==(const TmapKey& o) const { return std::memcmp(this, &o, sizeof(*this)) == 0; }
};
struct TmapSlot {
  bool used = false;
  TmapKey key;
  CUtensorMap map;
};
constexpr int kTmapSlots = 512;
std::mutex g_tmap_mu;
TmapSlot g_tmap[kTmapSlots];

bool encode_cached(CUtensorMap* map, const TmapKey& k) {
  uint64_t h = 1469598103934665603ull;
  const unsigned char* b = reinterpret_cast<const unsigned char*>(&k);
  for (size_t i = 0; i < sizeof(k); ++i) h = (h ^ b[i]) * 1099511628211ull;
  TmapSlot& slot = g_tmap[h % kTmapSlots];
  {
    std::lock_guard<std::mutex> lk(g_tmap_mu);
    if (slot.used && slot.key == k) {
      *map = slot.map;
      return true;
    }
  }
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  for (uint32_t i = 0; i < k.rank; ++i) {
    dims[i] = k.dims[i];
    box[i] = k.box[i];
    if (i + 1 < k.rank) strides[i] = k.strides[i];
  }
  std::memset(map, 0, sizeof(*map));
  if (fn(map, (CUtensorMapDataType)k.dtype, k.rank, reinterpret_cast<void*>(k.base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, (CUtensorMapSwizzle)k.swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lk(g_tmap_mu);
  slot.used = true;
  slot.key = k;
  slot.map = *map;
  return true;
}

struct SmemSet {
  const void* func;
  int dev, bytes;
};
std::mutex g_smem_mu;
SmemSet g_smem_set[256];
int g_smem_n = 0;

}  // namespace

cudaError_t ensure_smem(const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_smem_mu);
  for (int i = 0; i < g_smem_n; ++i)
    if (g_smem_set[i].func == func && g_smem_set[i].dev == dev && g_smem_set[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < g_smem_n; ++i)
    if (g_smem_set[i].func == func && g_smem_set[i].dev == dev) {
      g_smem_set[i].bytes = bytes;
      return cudaSuccess;
    }
  if (g_smem_n < 256) g_smem_set[g_smem_n++] = SmemSet{func, dev, bytes};
  return cudaSuccess;
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.base = reinterpret_cast<uint64_t>(base);
  k.dims[0] = inner;
  k.dims[1] = outer;
  k.strides[0] = row_bytes;
  k.box[0] = box_inner;
  k.box[1] = box_outer;
  k.rank = 2;
  k.dtype = (uint32_t)dtype;
  k.swz = (uint32_t)swz;
  return encode_cached(map, k);
}

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.base = reinterpret_cast<uint64_t>(base);
  k.dims[0] = d0;
  k.dims[1] = d1;
  k.dims[2] = d2;
  k.strides[0] = stride1;
  k.strides[1] = stride2;
  k.box[0] = b0;
  k.box[1] = b1;
  k.box[2] = b2;
  k.rank = 3;
  k.dtype = (uint32_t)dtype;
  k.swz = (uint32_t)CU_TENSOR_MAP_SWIZZLE_NONE;
  return encode_cached(map, k);
}

}  // namespace svdq

using namespace svdq;

extern "C" {

const char* svdq_status_str(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_SHAPE: return "shape violates the layer's size rules";
    case SVDQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SVDQ_ERR_UNSUPPORTED_ARCH: return "device is not compute capability 10.x (B200 / sm_100a)";
    case SVDQ_ERR_CUDA: return "CUDA runtime error";
    case SVDQ_ERR_TIMEOUT: return "a device-side bounded wait ran out";
  }
  return "unknown status";
}

size_t svdq_scale_bytes(svdq_precision p, int rows, int K) {
  if (rows < 0 || K <= 0 || K % 64) return 0;
  if (p == SVDQ_NVFP4) return (size_t)((rows + 127) / 128) * 128 * (size_t)(K / 16);
  if (p == SVDQ_INT4) return (size_t)rows * (size_t)int4_act_scale_pitch(K) * 2;
  return 0;
}

size_t svdq_lr_up_elems(svdq_precision p, int N, int r) {
  if (N < 0 || r < 0) return 0;
  if (p == SVDQ_NVFP4) return (size_t)N * 2 * r;
  if (p == SVDQ_INT4) return (size_t)N * r;
  return 0;
}

svdq_status svdq_pack_weight(svdq_precision p, int K, int N, int r, const float* W, const float* lambda,
                             const uint16_t* L1, const uint16_t* L2, float act_tensor_scale, uint8_t* w_codes,
                             void* w_scales, float* w_tensor_scale, float* inv_lambda, uint16_t* lr_up,
                             void* stream) {
  svdq_status st = check_common(p, K, r);
  if (st != SVDQ_OK) return st;
  if (N <= 0) return SVDQ_ERR_INVALID_ARG;
  if (N % 8) return SVDQ_ERR_SHAPE;
  if (!W || !lambda || !w_codes || !w_scales || !w_tensor_scale || !inv_lambda) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!L1 || !L2 || !lr_up)) return SVDQ_ERR_INVALID_ARG;
  if (p == SVDQ_NVFP4 && !(act_tensor_scale > 0.0f && act_tensor_scale < 3.0e38f)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(lambda) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(w_tensor_scale) || !aligned16(inv_lambda) || (r > 0 && (!aligned16(L1) || !aligned16(L2) ||
                                                                       !aligned16(lr_up))))
    return SVDQ_ERR_ALIGN;
  if ((st = device_info(nullptr, nullptr)) != SVDQ_OK) return st;
  PackArgs a{W, lambda, L1, L2, w_codes, w_scales, w_tensor_scale, inv_lambda, lr_up, K, N, r, act_tensor_scale};
  return from_cuda(launch_pack((int)p, a, svdq_scale_bytes(p, N, K), static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_quantize_act(svdq_precision p, int M, int K, int r, const uint16_t* x, const float* inv_lambda,
                              const float* w_tensor_scale, const uint16_t* L1, uint8_t* x_codes, void* x_scales,
                              uint16_t* P, void* stream) {
  svdq_status st = check_common(p, K, r);
  if (st != SVDQ_OK) return st;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!x || !inv_lambda || !x_codes || !x_scales) return SVDQ_ERR_INVALID_ARG;
  if (p == SVDQ_NVFP4 && !w_tensor_scale) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!L1 || !P)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(inv_lambda) || !aligned16(x_codes) || !aligned16(x_scales) ||
      (p == SVDQ_NVFP4 && (reinterpret_cast<uintptr_t>(w_tensor_scale) & 7)) ||
      (r > 0 && (!aligned16(L1) || !aligned16(P))))
    return SVDQ_ERR_ALIGN;
  unsigned* err = nullptr;
  if ((st = device_info(&err, nullptr)) != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p == SVDQ_NVFP4 && M % 128) {
    // zero the scales of the padding rows of the last 128-row block
    const size_t rb = (size_t)(M / 128), per_rb = (size_t)(K / 64) * 512;
    if (cudaMemsetAsync(static_cast<uint8_t*>(x_scales) + rb * per_rb, 0, per_rb, s) != cudaSuccess)
      return SVDQ_ERR_CUDA;
  }
  QuantActArgs a{x, inv_lambda, L1, x_codes, x_scales, P, M, K, r, p == SVDQ_NVFP4 ? w_tensor_scale : nullptr};
  return from_cuda(launch_quant_act((int)p, a, err, g_wait_ns.load(), s));
}

svdq_status svdq_w4a4_linear(svdq_precision p, int M, int K, int N, int r, const uint8_t* x_codes,
                             const void* x_scales, const uint16_t* P, const uint8_t* w_codes, const void* w_scales,
                             const float* w_tensor_scale, const uint16_t* lr_up, const uint16_t* bias, void* y,
                             svdq_out_dtype out, void* stream) {
  svdq_status st = check_common(p, K, r);
  if (st != SVDQ_OK) return st;
  if (M < 0 || N <= 0) return SVDQ_ERR_INVALID_ARG;
  if (N % 8) return SVDQ_ERR_SHAPE;
  if (out != SVDQ_OUT_BF16 && out != SVDQ_OUT_F32 && out != SVDQ_OUT_I32_GROUPS && out != SVDQ_OUT_BF16_GELU)
    return SVDQ_ERR_INVALID_ARG;
  if (out == SVDQ_OUT_I32_GROUPS && p != SVDQ_INT4) return SVDQ_ERR_INVALID_ARG;
  if (out == SVDQ_OUT_BF16_GELU && p != SVDQ_NVFP4) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!x_codes || !x_scales || !w_codes || !w_scales || !w_tensor_scale || !y) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!P || !lr_up)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(w_tensor_scale) || !aligned16(y) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3)) ||
      (r > 0 && (!aligned16(P) || !aligned16(lr_up))))
    return SVDQ_ERR_ALIGN;
  unsigned* err = nullptr;
  int sms = 0;
  if ((st = device_info(&err, &sms)) != SVDQ_OK) return st;
  GemmArgs a{x_codes, x_scales, P,  w_codes, w_scales, w_tensor_scale, lr_up, bias, y, M, K, N, r, (int)out, err,
             g_wait_ns.load(), sms};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return from_cuda(p == SVDQ_NVFP4 ? launch_gemm_nvfp4(a, s) : launch_gemm_int4(a, s));
}

size_t svdq_rope_packed_bytes(int M) {
  if (M < 0) return 0;
  return (size_t)((M + 31) / 32) * 16384;
}

svdq_status svdq_rope_pack(int M, const float* cos_t, const float* sin_t, float* rope, void* stream) {
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!cos_t || !sin_t || !rope) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(cos_t) || !aligned16(sin_t) || !aligned16(rope)) return SVDQ_ERR_ALIGN;
  const uintptr_t r0 = reinterpret_cast<uintptr_t>(rope), r1 = r0 + svdq_rope_packed_bytes(M);
  for (const float* t : {cos_t, sin_t}) {
    const uintptr_t t0 = reinterpret_cast<uintptr_t>(t), t1 = t0 + (size_t)M * 64 * sizeof(float);
    if (r0 < t1 && t0 < r1) return SVDQ_ERR_INVALID_ARG;
  }
  svdq_status st = device_info(nullptr, nullptr);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_rope_pack(M, cos_t, sin_t, rope, static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_w4a4_linear_qkv(int M, int K, int heads, int r, const uint8_t* x_codes, const void* x_scales,
                                 const uint16_t* P, const uint8_t* w_codes, const void* w_scales,
                                 const float* w_tensor_scale, const uint16_t* lr_up, const uint16_t* bias,
                                 const uint16_t* norm_q, const uint16_t* norm_k, float eps, const float* rope,
                                 uint16_t* y, void* stream) {
  svdq_status st = check_common(SVDQ_NVFP4, K, r);
  if (st != SVDQ_OK) return st;
  if (M < 0 || heads <= 0 || heads > (1 << 20) / 384) return SVDQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f && eps < 3.0e38f)) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!x_codes || !x_scales || !w_codes || !w_scales || !w_tensor_scale || !y || !norm_q || !norm_k || !rope)
    return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!P || !lr_up)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(w_tensor_scale) || !aligned16(y) || !aligned16(norm_q) || !aligned16(norm_k) ||
      !aligned16(rope) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3)) ||
      (r > 0 && (!aligned16(P) || !aligned16(lr_up))))
    return SVDQ_ERR_ALIGN;
  unsigned* err = nullptr;
  int sms = 0;
  if ((st = device_info(&err, &sms)) != SVDQ_OK) return st;
  const int N = 3 * heads * 128;
  GemmArgs a{x_codes, x_scales, P,  w_codes, w_scales, w_tensor_scale, lr_up, bias, y, M, K, N, r, (int)SVDQ_OUT_BF16,
             err, g_wait_ns.load(), sms};
  a.qkv_heads = heads;
  a.norm_q = norm_q;
  a.norm_k = norm_k;
  a.eps = eps;
  a.rope = rope;
  return from_cuda(launch_gemm_nvfp4(a, static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_qkv_norm_rope(int M, int heads, const uint16_t* norm_q, const uint16_t* norm_k, float eps,
                               const float* cos_t, const float* sin_t, uint16_t* y, void* stream) {
  if (M < 0 || heads <= 0 || heads > (1 << 20) / 384) return SVDQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f && eps < 3.0e38f)) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!norm_q || !norm_k || !cos_t || !sin_t || !y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(norm_q) || !aligned16(norm_k) || !aligned16(cos_t) || !aligned16(sin_t) || !aligned16(y))
    return SVDQ_ERR_ALIGN;
  svdq_status st = device_info(nullptr, nullptr);
  if (st != SVDQ_OK) return st;
  NormRopeArgs a{y, norm_q, norm_k, cos_t, sin_t, M, heads, eps};
  return from_cuda(launch_norm_rope(a, static_cast<cudaStream_t>(stream)));
}

svdq_status awq_pack_weight(int K, int N, const float* W, uint8_t* q, uint16_t* scales, uint16_t* zeros,
                            void* stream) {
  if (K <= 0 || N <= 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 || N % 8) return SVDQ_ERR_SHAPE;
  if (!W || !q || !scales || !zeros) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(q) || !aligned16(scales) || !aligned16(zeros)) return SVDQ_ERR_ALIGN;
  svdq_status st = device_info(nullptr, nullptr);
  if (st != SVDQ_OK) return st;
  AwqPackArgs a{W, q, scales, zeros, K, N};
  return from_cuda(launch_awq_pack(a, static_cast<cudaStream_t>(stream)));
}

svdq_status awq_w4a16_linear(int M, int K, int N, const uint16_t* x, const uint8_t* q, const uint16_t* scales,
                             const uint16_t* zeros, const uint16_t* bias, uint16_t* y, void* stream) {
  if (M < 0 || K <= 0 || N <= 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 || N % 8 || K > 16384) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!x || !q || !scales || !zeros || !y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(scales) || !aligned16(zeros) || !aligned16(y) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 1)))
    return SVDQ_ERR_ALIGN;
  unsigned* err = nullptr;
  svdq_status st = device_info(&err, nullptr);
  if (st != SVDQ_OK) return st;
  AwqArgs a{x, q, scales, zeros, bias, y, M, K, N};
  return from_cuda(launch_awq(a, err, g_wait_ns.load(), static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_device_error(unsigned* bits) {
  unsigned* err = nullptr;
  svdq_status st = device_info(&err, nullptr);
  if (st != SVDQ_OK) return st;
  unsigned v = 0;
  if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (bits) *bits = v;
  if (v & kErrTimeout) return SVDQ_ERR_TIMEOUT;
  if (v) return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

void svdq_set_wait_limit_ns(unsigned long long ns) { g_wait_ns.store(ns ? ns : 1); }

svdq_status svdq_probe_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3, uint16_t* bf16,
                               void* stream) {
  if (n < 0 || (n > 0 && !in)) return SVDQ_ERR_INVALID_ARG;
  svdq_status st = device_info(nullptr, nullptr);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_probe_convert(in, n, e2m1, e4m3, bf16, static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_probe_wait_timeout(unsigned long long limit_ns, void* stream) {
  unsigned* err = nullptr;
  svdq_status st = device_info(&err, nullptr);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_probe_wait(err, limit_ns, static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_probe_mma_peak(int iters, int mode, void* stream) {
  if (iters < 1 || iters > (1 << 20) || mode < 0 || mode > 4) return SVDQ_ERR_INVALID_ARG;
  unsigned* err = nullptr;
  int sms = 0;
  svdq_status st = device_info(&err, &sms);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_probe_mma(iters, mode, sms, err, g_wait_ns.load(), static_cast<cudaStream_t>(stream)));
}

void svdq_debug_force_arch(int major, int minor) {
  g_force_major.store(major);
  g_force_minor.store(minor);
}

}  // extern "C"
