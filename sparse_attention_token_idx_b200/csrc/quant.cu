// Rotation + block-FP8 quantisation of 128-feature rows, and the key-cache
// append ("Hadamard rotation" and "Index key cache" pages).
//
// One warp per row: lane l holds features 4l … 4l+3.  The Sylvester Hadamard
// transform H_128 is seven butterfly stages in float64 (strides 1 and 2 inside
// a lane, strides 4 … 64 across lanes with xor-shuffles), then one float64
// multiply by the correctly rounded 128^-1/2 and one round-to-nearest-even to
// bf16.  The quantiser takes amax over the 128 bf16 values (floored at 1e-4),
// scale = fl32(amax / 448) (IEEE division; ue8m0 rounds it up to a power of
// two), and codes = e4m3(fl32(x / scale)) with the hardware's round-to-nearest-
// even, saturating conversion.  Every warp stores one contiguous 128-byte row.
#include <cuda_runtime.h>
#include <cstdint>

#include "api_internal.h"
#include "ptx.cuh"

namespace idx {

namespace {

constexpr unsigned long long kInvSqrtDBits = 0x3FB6A09E667F3BCDull;  // correctly rounded 2^-3.5 (binary64)
constexpr uint32_t kInvSqrtDfBits = 0x3DB504F3u;                     // fl32(128^-1/2)
constexpr uint32_t kAmaxFloorBits = 0x38D1B717u;                     // fl32(1e-4)
constexpr int kRowsPerBlock = 8;                      // 8 warps

__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// float64 → bf16 bits, round to nearest even, from the binary64 / bfloat16
// encodings: 8 significant bits, exponent range of binary32, subnormal quantum 2^-133.
__device__ __forceinline__ uint32_t f64_to_bf16_rne(double v) {
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(v));
  const uint32_t sign = static_cast<uint32_t>(u >> 63) << 15;
  const double a = fabs(v);
  if (a < 0x1p-126) {
    // subnormal (or zero) bf16: integer multiple of 2^-133, 128 · 2^-133 = smallest normal
    const double m = rint(a * 0x1p133);  // exact scaling; rint rounds half to even
    return sign | static_cast<uint32_t>(m);
  }
  unsigned long long mag = u & 0x7FFFFFFFFFFFFFFFull;
  // keep 7 of the 52 fraction bits: add half-ulp minus one plus the kept LSB, truncate
  mag += (1ull << 44) - 1 + ((mag >> 45) & 1ull);
  mag &= ~((1ull << 45) - 1);
  const int e64 = static_cast<int>(mag >> 52);           // biased binary64 exponent
  const int e32 = e64 - 1023 + 127;                       // biased binary32/bf16 exponent
  if (e32 >= 255) return sign | 0x7F80u;                  // overflow → inf
  const uint32_t frac7 = static_cast<uint32_t>((mag >> 45) & 0x7Full);
  return sign | (static_cast<uint32_t>(e32) << 7) | frac7;
}

__device__ __forceinline__ float scale_from_amax(float amax, int fmt) {
  const float s = __fdiv_rn(fmaxf(amax, __uint_as_float(kAmaxFloorBits)), 448.0f);
  if (fmt == IDX_FMT_UE8M0) {
    const uint32_t b = __float_as_uint(s);
    if (b & 0x007FFFFFu) return __uint_as_float((b & 0xFF800000u) + 0x00800000u);
  }
  return s;
}

__device__ __forceinline__ uint32_t e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Rotate and quantise the row whose 4 features this lane holds (as bf16 bits).
// Returns the lane's 4 codes packed little-endian and the row scale.
__device__ __forceinline__ uint32_t rotate_quant_lane(uint2 in, int fmt, float* scale_out) {
  const int lane = threadIdx.x & 31;
  double v[4];
  v[0] = bf16_to_f32(in.x & 0xFFFFu);
  v[1] = bf16_to_f32(in.x >> 16);
  v[2] = bf16_to_f32(in.y & 0xFFFFu);
  v[3] = bf16_to_f32(in.y >> 16);
  // stride 1: (0,1), (2,3)
  double a0 = __dadd_rn(v[0], v[1]), a1 = __dsub_rn(v[0], v[1]);
  double a2 = __dadd_rn(v[2], v[3]), a3 = __dsub_rn(v[2], v[3]);
  // stride 2: (0,2), (1,3)
  v[0] = __dadd_rn(a0, a2);
  v[2] = __dsub_rn(a0, a2);
  v[1] = __dadd_rn(a1, a3);
  v[3] = __dsub_rn(a1, a3);
  // strides 4 … 64: partner lane differs in bit m; the lower index keeps a+b, the upper a−b
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const double o = __shfl_xor_sync(0xFFFFFFFFu, v[e], m);
      v[e] = upper ? __dsub_rn(o, v[e]) : __dadd_rn(v[e], o);
    }
  }
  float x[4];
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[e] = bf16_to_f32(f64_to_bf16_rne(__dmul_rn(v[e], __longlong_as_double(static_cast<long long>(kInvSqrtDBits)))));
    amax = fmaxf(amax, fabsf(x[e]));
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, m));
  const float s = scale_from_amax(amax, fmt);
  *scale_out = s;
  const uint32_t c01 = e4m3x2(__fdiv_rn(x[1], s), __fdiv_rn(x[0], s));
  const uint32_t c23 = e4m3x2(__fdiv_rn(x[3], s), __fdiv_rn(x[2], s));
  return c01 | (c23 << 16);
}

// MODE 0: plain rows.  MODE 1: query rows with weight folding.  MODE 2: cache append.
template <int MODE>
__global__ void __launch_bounds__(kRowsPerBlock * 32) quant_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                                  uint8_t* __restrict__ codes,
                                                                  float* __restrict__ scales, int fmt,
                                                                  const float* __restrict__ w_raw,
                                                                  float* __restrict__ w_out,
                                                                  const int32_t* __restrict__ positions, int n,
                                                                  int T_cap, unsigned int* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * kRowsPerBlock;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + (threadIdx.x >> 5); r < rows;
       r += warps_total) {
    int64_t dst_row = r;
    if (MODE == 2) {
      const int64_t b = r / n;
      const int64_t i = r - b * n;
      const int p = positions[b];
      if (p < 0 || static_cast<int64_t>(p) + n > T_cap) {
        if (lane == 0 && i == 0) raise_error(err, IDX_DEV_ERR_POSITION);
        continue;
      }
      dst_row = b * static_cast<int64_t>(T_cap) + p + i;
    }
    const uint2 in = reinterpret_cast<const uint2*>(x + r * IDX_DIM)[lane];
    float s;
    const uint32_t packed = rotate_quant_lane(in, fmt, &s);
    reinterpret_cast<uint32_t*>(codes + dst_row * IDX_DIM)[lane] = packed;
    if (lane == 0) {
      if (MODE == 1) {
        const float w = __fmul_rn(__fmul_rn(__fmul_rn(w_raw[r], 0.125f), s), __uint_as_float(kInvSqrtDfBits));
        w_out[r] = w;
      } else {
        scales[dst_row] = s;
      }
    }
  }
}

__global__ void e4m3_encode_kernel(const float* __restrict__ x, int64_t count, uint8_t* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    out[i] = static_cast<uint8_t>(e4m3x2(0.0f, x[i]) & 0xFFu);
  }
}

int quant_grid(int64_t rows) {
  const int64_t blocks = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  return static_cast<int>(blocks < cap ? blocks : cap);
}

}  // namespace

}  // namespace idx

using namespace idx;

extern "C" int idx_quant(const uint16_t* x_bf16, int64_t rows, uint8_t* x_fp8, float* x_scale, int fmt,
                         idx_stream_t stream) {
  if (rows < 0) return IDX_ERR_SHAPE;
  if (fmt != IDX_FMT_FP32 && fmt != IDX_FMT_UE8M0) return IDX_ERR_FMT;
  if (rows == 0) return IDX_OK;
  if (!x_bf16 || !x_fp8 || !x_scale) return IDX_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(x_bf16) | reinterpret_cast<uintptr_t>(x_fp8)) & 7) return IDX_ERR_ALIGN;
  quant_kernel<0><<<quant_grid(rows), kRowsPerBlock * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x_bf16, rows, x_fp8, x_scale, fmt, nullptr, nullptr, nullptr, 1, 0, nullptr);
  return check_launch();
}

extern "C" int idx_quant_queries(const uint16_t* q_bf16, const float* w_raw, int64_t tokens, uint8_t* q_fp8,
                                 float* w, int fmt, idx_stream_t stream) {
  if (tokens < 0) return IDX_ERR_SHAPE;
  if (fmt != IDX_FMT_FP32 && fmt != IDX_FMT_UE8M0) return IDX_ERR_FMT;
  if (tokens == 0) return IDX_OK;
  if (!q_bf16 || !w_raw || !q_fp8 || !w) return IDX_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(q_bf16) | reinterpret_cast<uintptr_t>(q_fp8)) & 7) return IDX_ERR_ALIGN;
  const int64_t rows = tokens * IDX_HEADS;
  quant_kernel<1><<<quant_grid(rows), kRowsPerBlock * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      q_bf16, rows, q_fp8, nullptr, fmt, w_raw, w, nullptr, 1, 0, nullptr);
  return check_launch();
}

extern "C" int idx_quant_append(const uint16_t* k_bf16, const int32_t* positions, int B, int n, uint8_t* k_cache,
                                float* k_scale_cache, int T_cap, int fmt, idx_stream_t stream) {
  if (B < 0 || n < 0 || T_cap <= 0) return IDX_ERR_SHAPE;
  if (fmt != IDX_FMT_FP32 && fmt != IDX_FMT_UE8M0) return IDX_ERR_FMT;
  if (B == 0 || n == 0) return IDX_OK;
  if (n > T_cap) return IDX_ERR_SHAPE;
  if (!k_bf16 || !positions || !k_cache || !k_scale_cache) return IDX_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(k_bf16) | reinterpret_cast<uintptr_t>(k_cache)) & 7) return IDX_ERR_ALIGN;
  const int64_t rows = static_cast<int64_t>(B) * n;
  quant_kernel<2><<<quant_grid(rows), kRowsPerBlock * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      k_bf16, rows, k_cache, k_scale_cache, fmt, nullptr, nullptr, positions, n, T_cap, device_error_word());
  return check_launch();
}

extern "C" int idx_e4m3_encode(const float* x, int64_t count, uint8_t* out, idx_stream_t stream) {
  if (count < 0) return IDX_ERR_SHAPE;
  if (count == 0) return IDX_OK;
  if (!x || !out) return IDX_ERR_NULL;
  const int64_t blocks = (count + 255) / 256;
  const int grid = static_cast<int>(blocks < 148 * 64 ? blocks : 148 * 64);
  e4m3_encode_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, count, out);
  return check_launch();
}
