// Library-wide host code: device error word, status, error strings, tensor-map
// creation through the driver entry point, and the fault-injection switch.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "api_internal.h"
#include "ptx.cuh"

namespace idx {

namespace {
constexpr int kMaxDevicesForWord = 64;
int current_device_for_word() {
  int d = 0;
  cudaGetDevice(&d);
  return (d >= 0 && d < kMaxDevicesForWord) ? d : 0;
}
}  // namespace

__device__ unsigned int g_error_word = 0;

unsigned int* device_error_word() {
  static std::atomic<unsigned int*> addr[kMaxDevicesForWord];
  const int d = current_device_for_word();
  unsigned int* a = addr[d].load();
  if (!a) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess) return nullptr;
    a = static_cast<unsigned int*>(ptr);
    addr[d].store(a);
  }
  return a;
}

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_smem_optin[kMaxDevices];
std::atomic<int> g_last_cuda_error{0};
std::atomic<unsigned int> g_last_device_bits{0};
std::atomic<unsigned int> g_debug_flags{0};
std::atomic<unsigned long long> g_debug_budget{0};
constexpr unsigned long long kDefaultBudgetNs = 2000000000ull;  // 2 s

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return (d >= 0 && d < kMaxDevices) ? d : 0;
}
}  // namespace

int num_sms() {
  const int d = current_device();
  int v = g_sms[d].load();
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0) v = 148;
    g_sms[d].store(v);
  }
  return v;
}

int max_dynamic_smem() {
  const int d = current_device();
  int v = g_smem_optin[d].load();
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess || v <= 0)
      v = 227 * 1024;
    g_smem_optin[d].store(v);
  }
  return v;
}

int smem_per_sm() {
  static std::atomic<int> cache[kMaxDevices];
  const int d = current_device();
  int v = cache[d].load();
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerMultiprocessor, d) != cudaSuccess || v <= 0)
      v = 228 * 1024;
    cache[d].store(v);
  }
  return v;
}

int ensure_smem_limit(const void* func, int smem) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> limits;   // (device, kernel) → bytes set
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return check_launch();
  std::lock_guard<std::mutex> lock(mu);
  int& have = limits[{dev, func}];
  if (have >= smem) return IDX_OK;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return check_launch();
  have = smem;
  return IDX_OK;
}

int check_launch() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return IDX_OK;
  g_last_cuda_error.store(static_cast<int>(e));
  return e == cudaErrorNoKernelImageForDevice || e == cudaErrorInvalidDeviceFunction ? IDX_ERR_UNSUPPORTED
                                                                                       : IDX_ERR_LAUNCH;
}

static void resolve_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
}

bool make_tmap_u8_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                     uint32_t box_rows) {
  resolve_encode();
  if (!g_encode) return false;
  if (reinterpret_cast<uintptr_t>(base) & 15) return false;
  const cuuint64_t dims[3] = {inner, mid, outer};
  const cuuint64_t strides[2] = {inner, inner * mid};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner) {
  resolve_encode();
  if (!g_encode) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((inner * 4) & 15)) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 4};
  const cuuint32_t box[2] = {box_inner, 1};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner) {
  resolve_encode();
  if (!g_encode) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (inner & 15)) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, 1};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d_bf16_sw128(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  resolve_encode();
  if (!g_encode) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((cols * 2) & 15)) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};   // 64 bf16 = one 128-byte swizzle row
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_scales(CUtensorMap* map, const void* base, int scale_fmt, uint64_t T_cap, uint64_t B,
                      uint32_t box_inner) {
  return scale_fmt == kScaleE8M0 ? make_tmap_u8_2d(map, base, T_cap, B, box_inner)
                                 : make_tmap_f32_2d(map, base, T_cap, B, box_inner);
}

DebugState debug_state() {
  DebugState s;
  s.flags = g_debug_flags.load();
  const unsigned long long b = g_debug_budget.load();
  s.budget_ns = b ? b : kDefaultBudgetNs;
  return s;
}

}  // namespace idx

using namespace idx;

extern "C" int idx_status(idx_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    g_last_cuda_error.store(static_cast<int>(cudaGetLastError()));
    return IDX_ERR_CUDA;
  }
  unsigned int bits = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&bits, g_error_word, sizeof(bits)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) {
    g_last_cuda_error.store(static_cast<int>(cudaGetLastError()));
    return IDX_ERR_CUDA;
  }
  g_last_device_bits.store(bits);
  return bits ? IDX_ERR_DEVICE : IDX_OK;
}

extern "C" unsigned int idx_device_error_bits(void) { return g_last_device_bits.load(); }

extern "C" int idx_last_cuda_error(void) { return g_last_cuda_error.load(); }

extern "C" const char* idx_error_string(int code) {
  switch (code) {
    case IDX_OK: return "ok";
    case IDX_ERR_NULL: return "a required pointer is NULL";
    case IDX_ERR_SHAPE: return "a size argument is out of range";
    case IDX_ERR_FMT: return "fmt must be IDX_FMT_FP32 or IDX_FMT_UE8M0";
    case IDX_ERR_K: return "k must be positive";
    case IDX_ERR_ALIGN: return "a pointer is not aligned as required";
    case IDX_ERR_LAUNCH: return "the CUDA launch failed";
    case IDX_ERR_DEVICE: return "a kernel reported an error (see idx_device_error_bits)";
    case IDX_ERR_CUDA: return "the stream reported a CUDA error";
    case IDX_ERR_UNSUPPORTED: return "no device code for this GPU (sm_100a required)";
    case IDX_ERR_SCRATCH: return "the scratch is too small (the library's fixed 64 MiB buffer, or the caller's workspace)";
    default: return "unknown status";
  }
}

extern "C" size_t idx_workspace_size(int B, int n, int max_len, int k) {
  (void)k;
  if (B <= 0 || n <= 0 || max_len <= 0) return 0;
  // Decode-shaped calls select in shared memory (fused score + top-k): their
  // cache stream is HBM-bound either way, and the fused kernel skips the
  // score round trip and the second launch.
  const int64_t rows = static_cast<int64_t>(B) * n;
  if (n <= 2) return 0;
  // one fp32 score row of max_len columns per query row
  return static_cast<size_t>(rows) * static_cast<size_t>(max_len) * sizeof(float);
}

extern "C" void idx_debug_set(unsigned int flags, unsigned long long budget_ns) {
  g_debug_flags.store(flags);
  g_debug_budget.store(budget_ns);
}
