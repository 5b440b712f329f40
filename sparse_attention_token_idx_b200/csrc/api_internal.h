// Host-side helpers shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/idx.h"

namespace idx {

int num_sms();                       // SM count of the current device (cached per device)
int check_launch();                  // IDX_OK, or IDX_ERR_LAUNCH after recording cudaGetLastError()
int max_dynamic_smem();              // opt-in shared memory per block of the current device
int smem_per_sm();                   // shared memory per SM of the current device
// Raise `func`'s dynamic shared-memory limit to at least `smem` bytes on the
// current device (remembered per device and kernel, so that a process driving
// several GPUs sets it once on each).  IDX_OK, or check_launch()'s code.
int ensure_smem_limit(const void* func, int smem);

// Tensor map for a [outer, mid, inner] uint8 array (row pitch `inner` bytes,
// plane pitch mid·inner bytes), box {128 bytes, box_rows, 1}, 128-byte swizzle.
bool make_tmap_u8_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                     uint32_t box_rows);

unsigned int* device_error_word();  // device address of the error word on the current device

// Tensor map for a [outer, inner] float32 array (row pitch inner·4 bytes, a
// multiple of 16), box {box_inner, 1}, no swizzle.
bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner);

// Tensor map for a [outer, inner] uint8 array (row pitch inner bytes, a
// multiple of 16), box {box_inner, 1}, no swizzle.
bool make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner);

// Tensor map for a [rows, cols] bf16 array (row pitch cols·2 bytes, a multiple
// of 16), box {64 elements, box_rows}, 128-byte swizzle (K-major MMA operands).
bool make_tmap_2d_bf16_sw128(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows);

// Key-scale storage of a score call: fp32 values, or e8m0 bytes (2^(byte − 127)).
enum { kScaleF32 = 0, kScaleE8M0 = 1 };

// Options of a score call beyond the method's definition.
struct ScoreVariant {
  int scale_fmt;      // kScaleF32 or kScaleE8M0
  int out_bf16;       // unfused scores in bf16 (round to nearest even) instead of fp32
  float mask_value;   // unfused scores: value of masked columns (−inf, or a finite bound)
};
bool make_tmap_scales(CUtensorMap* map, const void* base, int scale_fmt, uint64_t T_cap, uint64_t B,
                      uint32_t box_inner);

unsigned long long* trace_buffer();  // device address of the phase-trace buffer

// Flat-partition scorer (flat_score.cu): scores of every visible (row, key) of
// the call into scores [B, n, ld], one persistent CTA per SM; columns past a
// row's last key tile are left unwritten.  IDX_ERR_UNSUPPORTED when the call
// has more row blocks than the kernel's shared-memory index holds.
int launch_flat_score(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale_cache,
                      int scale_fmt, const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal,
                      float* scores, int64_t ld, cudaStream_t stream);

// Sparse latent attention on the tensor cores (mla_tc.cu): IDX_ERR_UNSUPPORTED
// when the shape is not one it serves (H not a multiple of 128, q unaligned).
int launch_sparse_mla_tc(const uint16_t* q, const uint16_t* kv, const int32_t* indices, int B, int H, int64_t T_cap,
                         int k, float softmax_scale, float* out, cudaStream_t stream);

struct DebugState {
  unsigned int flags;
  unsigned long long budget_ns;
};
DebugState debug_state();

}  // namespace idx
