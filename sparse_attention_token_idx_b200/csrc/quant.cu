// Rotation + block-FP8 quantisation of 128-feature rows, and the key-cache
// append ("Hadamard rotation" and "Index key cache" pages).
//
// Four lanes per row: lane q holds features 32q … 32q+31.  The Sylvester
// Hadamard transform H_128 is seven butterfly stages in float64 (strides 1 … 16
// inside a lane, strides 32 and 64 across the four lanes with xor-shuffles),
// then one float64 multiply by the correctly rounded 128^-1/2 and one
// round-to-nearest-even to bf16 (cvt.rn.bf16.f64).  The quantiser takes amax over the 128 bf16 values (floored at 1e-4),
// scale = fl32(amax / 448) (IEEE division; ue8m0 rounds it up to a power of
// two), and codes = e4m3(fl32(x / scale)) with the hardware's round-to-nearest-
// even, saturating conversion.  Each lane stores 32 contiguous code bytes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "api_internal.h"
#include "ptx.cuh"

namespace idx {

namespace {

constexpr unsigned long long kInvSqrtDBits = 0x3FB6A09E667F3BCDull;  // correctly rounded 2^-3.5 (binary64)
constexpr uint32_t kInvSqrtDfBits = 0x3DB504F3u;                     // fl32(128^-1/2)
constexpr uint32_t kAmaxFloorBits = 0x38D1B717u;                     // fl32(1e-4)
constexpr int kWarpsPerBlock = 8;                     // 8 warps × 8 rows

__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// float64 → bf16 value (as float), round to nearest even (the PTX conversion
// cvt.rn.bf16.f64 rounds the binary64 value once, subnormals included).
__device__ __forceinline__ float f64_to_bf16_as_f32(double v) {
  uint16_t h;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
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

// x / s, correctly rounded (IEEE binary32 division), for the quantiser.
// ue8m0 scales are powers of two, so x times the exact reciprocal is the same
// value (one rounding of the same exact quotient); other scales divide.
struct Divider {
  float s, y;
  bool pow2;
  __device__ __forceinline__ Divider(float scale, int fmt) : s(scale) {
    pow2 = fmt == IDX_FMT_UE8M0;
    y = pow2 ? __frcp_rn(scale) : 0.f;
  }
  __device__ __forceinline__ float div(float x) const { return pow2 ? __fmul_rn(x, y) : __fdiv_rn(x, s); }
};

// Rows are handled by quads: 4 lanes per 128-feature row, lane q holding
// features 32q … 32q+31, 8 rows per warp.  Strides 1 … 16 of the butterfly run
// inside a lane; strides 32 and 64 pair lane q with q^1 and q^2.
struct QuadRow {
  uint4 codes[2];   // this lane's 32 e4m3 codes
  float scale;
};

__device__ __forceinline__ void load_quad(const uint4* src, double (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 a = src[i];
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      v[8 * i + 2 * m] = bf16_to_f32(w[m] & 0xFFFFu);
      v[8 * i + 2 * m + 1] = bf16_to_f32(w[m] >> 16);
    }
  }
}

// Sum of the row's 128 values (SQUARE: of their squares, each rounded) in
// feature order (0, 1, …, 127), float64: lane q continues the running sum of
// lane q − 1.  All 32 lanes of the warp call it.
template <bool SQUARE>
__device__ __forceinline__ double quad_sequential_sum(const double (&v)[32]) {
  const int lane = threadIdx.x & 31, q = lane & 3;
  double acc = 0.0;
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    if (q == st) {
#pragma unroll
      for (int e = 0; e < 32; ++e) acc = __dadd_rn(acc, SQUARE ? __dmul_rn(v[e], v[e]) : v[e]);
    }
    acc = __shfl_sync(0xFFFFFFFFu, acc, (lane & ~3) | st);
  }
  return acc;
}

__device__ __forceinline__ double bf16_round_f64(double x) { return static_cast<double>(f64_to_bf16_as_f32(x)); }

// Key LayerNorm over the row (Indexer.forward excerpt: k_norm after the key
// projection): mean and biased variance by feature-order sums, then
// ((x − mean) / sqrt(var + eps)) · gain + bias, float64 with one rounding per
// operation, then bf16.  All lanes call it; `apply` selects whose row changes.
__device__ __forceinline__ void quad_layer_norm(double (&v)[32], bool apply, const float* __restrict__ gain,
                                                const float* __restrict__ bias, double eps) {
  const int q = threadIdx.x & 3;
  const double mean = __dmul_rn(quad_sequential_sum<false>(v), 0.0078125);
  // rows that are not normalised keep their values (their statistics go unused)
  if (apply) {
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = __dsub_rn(v[e], mean);
  }
  const double var = __dmul_rn(quad_sequential_sum<true>(v), 0.0078125);
  const double sd = __dsqrt_rn(__dadd_rn(var, eps));
  if (apply) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const double g = __ldg(gain + 32 * q + e), b = __ldg(bias + 32 * q + e);
      v[e] = bf16_round_f64(__dadd_rn(__dmul_rn(__ddiv_rn(v[e], sd), g), b));
    }
  }
}

// Rotary embedding of features 0 … 63, not interleaved (Indexer.forward
// excerpt): feature i (lane 0) and i + 32 (lane 1) turn by angle θ_i,
// (a, b) → (a cos − b sin, b cos + a sin); the products are exact in float64,
// so each result is rounded once, then to bf16.  All lanes call it.
__device__ __forceinline__ void quad_rope(double (&v)[32], const float* __restrict__ cos_row,
                                          const float* __restrict__ sin_row) {
  const int q = threadIdx.x & 3;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const double o = __shfl_xor_sync(0xFFFFFFFFu, v[e], 1);
    if (q < 2) {
      const double c = __ldg(cos_row + e), s = __ldg(sin_row + e);
      const double vc = __dmul_rn(v[e], c), os = __dmul_rn(o, s);
      v[e] = bf16_round_f64(q == 0 ? __dsub_rn(vc, os) : __dadd_rn(vc, os));
    }
  }
}

__device__ __forceinline__ QuadRow rotate_quant_v(double (&v)[32], int fmt);

__device__ __forceinline__ QuadRow rotate_quant_quad(const uint4* src, int fmt) {
  double v[32];
  load_quad(src, v);
  return rotate_quant_v(v, fmt);
}

__device__ __forceinline__ QuadRow rotate_quant_v(double (&v)[32], int fmt) {
  const int q = threadIdx.x & 3;
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if ((j & h) == 0) {
        const double a = v[j], b = v[j + h];
        v[j] = __dadd_rn(a, b);
        v[j + h] = __dsub_rn(a, b);
      }
    }
  }
  // cross-lane stages: the lower index keeps a + b, the upper gets a − b, i.e.
  // partner ± own — one FMA with ±1 (exact product, one rounding: the same
  // value as the add or subtract)
#pragma unroll
  for (int m = 1; m <= 2; m <<= 1) {
    const double sgn = (q & m) ? -1.0 : 1.0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const double o = __shfl_xor_sync(0xFFFFFFFFu, v[e], m);
      v[e] = __fma_rn(sgn, v[e], o);
    }
  }
  const double c = __longlong_as_double(static_cast<long long>(kInvSqrtDBits));
  float x[32];
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    x[e] = f64_to_bf16_as_f32(__dmul_rn(v[e], c));
    amax = fmaxf(amax, fabsf(x[e]));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  QuadRow r;
  r.scale = scale_from_amax(amax, fmt);
  const Divider dv(r.scale, fmt);
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = e4m3x2(dv.div(x[4 * i + 1]), dv.div(x[4 * i]));
    const uint32_t hi = e4m3x2(dv.div(x[4 * i + 3]), dv.div(x[4 * i + 2]));
    pk[i] = lo | (hi << 16);
  }
  r.codes[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  r.codes[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  return r;
}

// One launch for any mix of:
//   rows [0, plain_rows)              plain rows → codes / scales           (idx_quant)
//   rows [0, q_rows)                  query rows → codes, folded weights    (idx_quant_queries)
//   rows [q_rows, q_rows + k_rows)    key rows   → cache slots             (idx_quant_append)
struct QuantArgs {
  // plain / query rows
  const uint16_t* x;
  uint8_t* codes;
  float* scales;          // plain rows only
  const float* w_raw;     // query rows: fold weights when non-null
  float* w_out;
  int64_t rows;           // rows of the first kind
  // key rows (append)
  const uint16_t* k;
  const int32_t* positions;
  uint8_t* k_cache;
  float* k_scale_cache;
  uint8_t* k_scale_e8;    // instead of k_scale_cache: the scale's e8m0 byte (ue8m0 only)
  int64_t k_rows;
  int n, T_cap;
  int fmt;
  unsigned int* err;
  // front end (FRONT kernels): per-token RoPE tables [tokens, 32] (tokens = the
  // key rows, each with 64 query rows) and the key LayerNorm's gain / bias / eps
  const float* rope_cos;
  const float* rope_sin;
  const float* ln_gain;
  const float* ln_bias;
  double ln_eps;
};

template <bool FRONT>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) quant_kernel(const QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const int q = lane & 3;
  const int64_t total = a.rows + a.k_rows;
  const int64_t quads_total = static_cast<int64_t>(gridDim.x) * kWarpsPerBlock * 8;
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5)) * 8; base < total;
       base += quads_total) {
    const int64_t r = base + (lane >> 2);
    const bool live = r < total;
    const bool is_key = live && r >= a.rows;
    bool store = live;
    const uint16_t* src;
    uint8_t* dst;
    int64_t slot = 0;
    if (is_key) {
      const int64_t kr = r - a.rows;
      const int64_t b = kr / a.n;
      const int64_t i = kr - b * a.n;
      const int p = a.positions[b];
      if (p < 0 || static_cast<int64_t>(p) + a.n > a.T_cap) {
        if (q == 0 && i == 0) raise_error(a.err, IDX_DEV_ERR_POSITION);
        store = false;
      }
      slot = b * static_cast<int64_t>(a.T_cap) + p + i;
      src = a.k + kr * IDX_DIM;
      dst = a.k_cache + slot * IDX_DIM;
    } else if (live) {
      src = a.x + r * IDX_DIM;
      dst = a.codes + r * IDX_DIM;
    } else {
      // past the end: compute on a valid row (all lanes take part in the shuffles), store nothing
      src = a.rows > 0 ? a.x : a.k;
      dst = nullptr;
    }
    QuadRow out;
    if constexpr (FRONT) {
      double v[32];
      load_quad(reinterpret_cast<const uint4*>(src + 32 * q), v);
      // the row's token: key row kr, or query row r of token r / 64 (0 past the end)
      const int64_t tok = is_key ? r - a.rows : (live ? r / IDX_HEADS : 0);
      // warps of query rows only skip the LayerNorm (warp-uniform: the shuffles stay converged)
      if (__any_sync(0xFFFFFFFFu, is_key)) quad_layer_norm(v, is_key, a.ln_gain, a.ln_bias, a.ln_eps);
      quad_rope(v, a.rope_cos + tok * (IDX_ROPE_DIM / 2), a.rope_sin + tok * (IDX_ROPE_DIM / 2));
      out = rotate_quant_v(v, a.fmt);
    } else {
      out = rotate_quant_quad(reinterpret_cast<const uint4*>(src + 32 * q), a.fmt);
    }
    if (store) {
      uint4* d = reinterpret_cast<uint4*>(dst + 32 * q);
      d[0] = out.codes[0];
      d[1] = out.codes[1];
      if (q == 0) {
        if (is_key) {
          // a ue8m0 scale is a normal power of two: its byte is the fp32 exponent field
          if (a.k_scale_e8) a.k_scale_e8[slot] = static_cast<uint8_t>(__float_as_uint(out.scale) >> 23);
          else a.k_scale_cache[slot] = out.scale;
        } else if (a.w_raw) {
          a.w_out[r] = __fmul_rn(__fmul_rn(__fmul_rn(a.w_raw[r], 0.125f), out.scale),
                                 __uint_as_float(kInvSqrtDfBits));
        } else {
          a.scales[r] = out.scale;
        }
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
  const int64_t rows_per_block = kWarpsPerBlock * 8;
  const int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  return static_cast<int>(blocks < cap ? blocks : cap);
}

int launch_quant(const QuantArgs& a, cudaStream_t stream, bool front = false) {
  const int64_t total = a.rows + a.k_rows;
  if (total == 0) return IDX_OK;
  if (front)
    quant_kernel<true><<<quant_grid(total), kWarpsPerBlock * 32, 0, stream>>>(a);
  else
    quant_kernel<false><<<quant_grid(total), kWarpsPerBlock * 32, 0, stream>>>(a);
  return check_launch();
}

QuantArgs empty_args(int fmt) {
  QuantArgs a = {};
  a.fmt = fmt;
  a.n = 1;
  return a;
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
  if ((reinterpret_cast<uintptr_t>(x_bf16) | reinterpret_cast<uintptr_t>(x_fp8)) & 15) return IDX_ERR_ALIGN;
  QuantArgs a = empty_args(fmt);
  a.x = x_bf16;
  a.codes = x_fp8;
  a.scales = x_scale;
  a.rows = rows;
  return launch_quant(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int idx_quant_queries(const uint16_t* q_bf16, const float* w_raw, int64_t tokens, uint8_t* q_fp8,
                                 float* w, int fmt, idx_stream_t stream) {
  return idx_quant_queries_append(q_bf16, w_raw, tokens, q_fp8, w, nullptr, nullptr, 0, 0, nullptr, nullptr, 1, fmt,
                                  stream);
}

extern "C" int idx_quant_append(const uint16_t* k_bf16, const int32_t* positions, int B, int n, uint8_t* k_cache,
                                float* k_scale_cache, int T_cap, int fmt, idx_stream_t stream) {
  return idx_quant_queries_append(nullptr, nullptr, 0, nullptr, nullptr, k_bf16, positions, B, n, k_cache,
                                  k_scale_cache, T_cap, fmt, stream);
}

extern "C" int idx_quant_queries_append(const uint16_t* q_bf16, const float* w_raw, int64_t tokens, uint8_t* q_fp8,
                                        float* w, const uint16_t* k_bf16, const int32_t* positions, int B, int n,
                                        uint8_t* k_cache, float* k_scale_cache, int T_cap, int fmt,
                                        idx_stream_t stream) {
  if (tokens < 0 || B < 0 || n < 0 || T_cap <= 0) return IDX_ERR_SHAPE;
  if (fmt != IDX_FMT_FP32 && fmt != IDX_FMT_UE8M0) return IDX_ERR_FMT;
  const bool has_q = tokens > 0;
  const bool has_k = B > 0 && n > 0;
  if (has_k && n > T_cap) return IDX_ERR_SHAPE;
  if (has_q && (!q_bf16 || !w_raw || !q_fp8 || !w)) return IDX_ERR_NULL;
  if (has_k && (!k_bf16 || !positions || !k_cache || !k_scale_cache)) return IDX_ERR_NULL;
  if (has_q && ((reinterpret_cast<uintptr_t>(q_bf16) | reinterpret_cast<uintptr_t>(q_fp8)) & 15)) return IDX_ERR_ALIGN;
  if (has_k && ((reinterpret_cast<uintptr_t>(k_bf16) | reinterpret_cast<uintptr_t>(k_cache)) & 15)) return IDX_ERR_ALIGN;
  QuantArgs a = empty_args(fmt);
  if (has_q) {
    a.x = q_bf16;
    a.codes = q_fp8;
    a.w_raw = w_raw;
    a.w_out = w;
    a.rows = tokens * IDX_HEADS;
  }
  if (has_k) {
    a.k = k_bf16;
    a.positions = positions;
    a.k_cache = k_cache;
    a.k_scale_cache = k_scale_cache;
    a.k_rows = static_cast<int64_t>(B) * n;
    a.n = n;
    a.T_cap = T_cap;
    a.err = device_error_word();
    if (!a.err) return check_launch();
  }
  return launch_quant(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int idx_quant_append_e8(const uint16_t* k_bf16, const int32_t* positions, int B, int n,
                                   uint8_t* k_cache, uint8_t* k_scale_e8, int T_cap, idx_stream_t stream) {
  if (B < 0 || n < 0 || T_cap <= 0) return IDX_ERR_SHAPE;
  if (B == 0 || n == 0) return IDX_OK;
  if (n > T_cap) return IDX_ERR_SHAPE;
  if (!k_bf16 || !positions || !k_cache || !k_scale_e8) return IDX_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(k_bf16) | reinterpret_cast<uintptr_t>(k_cache)) & 15) return IDX_ERR_ALIGN;
  QuantArgs a = empty_args(IDX_FMT_UE8M0);
  a.k = k_bf16;
  a.positions = positions;
  a.k_cache = k_cache;
  a.k_scale_e8 = k_scale_e8;
  a.k_rows = static_cast<int64_t>(B) * n;
  a.n = n;
  a.T_cap = T_cap;
  a.err = device_error_word();
  if (!a.err) return check_launch();
  return launch_quant(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int idx_front_quant_append(const uint16_t* q_proj, const float* w_raw, const uint16_t* k_proj,
                                      const float* rope_cos, const float* rope_sin, const float* ln_gain,
                                      const float* ln_bias, float ln_eps, const int32_t* positions, int B, int n,
                                      uint8_t* q_fp8, float* w, uint8_t* k_cache, float* k_scale_cache, int T_cap,
                                      int fmt, idx_stream_t stream) {
  if (B < 0 || n < 0 || T_cap <= 0) return IDX_ERR_SHAPE;
  if (fmt != IDX_FMT_FP32 && fmt != IDX_FMT_UE8M0) return IDX_ERR_FMT;
  if (!(ln_eps >= 0.0f) || ln_eps > 3.0e38f) return IDX_ERR_SHAPE;   // NaN, negative or infinite
  if (B == 0 || n == 0) return IDX_OK;
  if (n > T_cap) return IDX_ERR_SHAPE;
  if (!q_proj || !w_raw || !k_proj || !rope_cos || !rope_sin || !ln_gain || !ln_bias || !positions || !q_fp8 || !w ||
      !k_cache || !k_scale_cache)
    return IDX_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(q_proj) | reinterpret_cast<uintptr_t>(q_fp8) | reinterpret_cast<uintptr_t>(k_proj) |
       reinterpret_cast<uintptr_t>(k_cache)) & 15)
    return IDX_ERR_ALIGN;
  const int64_t tokens = static_cast<int64_t>(B) * n;
  QuantArgs a = empty_args(fmt);
  a.x = q_proj;
  a.codes = q_fp8;
  a.w_raw = w_raw;
  a.w_out = w;
  a.rows = tokens * IDX_HEADS;
  a.k = k_proj;
  a.positions = positions;
  a.k_cache = k_cache;
  a.k_scale_cache = k_scale_cache;
  a.k_rows = tokens;
  a.n = n;
  a.T_cap = T_cap;
  a.rope_cos = rope_cos;
  a.rope_sin = rope_sin;
  a.ln_gain = ln_gain;
  a.ln_bias = ln_bias;
  a.ln_eps = static_cast<double>(ln_eps);
  a.err = device_error_word();
  if (!a.err) return check_launch();
  return launch_quant(a, reinterpret_cast<cudaStream_t>(stream), true);
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
