// Sparse latent attention for one decode token per sequence over the positions
// the indexer selected ("Join query parts" page, MQA decode excerpt): per head,
// scores against the selected 576-feature cache rows (512 latent + 64 rotary),
// a softmax over them, and the latent output (the rows' first 512 features
// weighted by the softmax).
//
// One CTA per (sequence, group of 16 heads), 16 warps: warp h owns head h of the
// group.  The selection is walked in chunks of 32 positions: the CTA gathers the
// chunk's rows into shared memory (bf16, rows padded to an odd number of words
// so that 32 rows read at one column hit 32 banks), lane t of each warp scores
// row t for its head, the warp updates its running max / sum (online softmax),
// and each lane accumulates 16 of the head's 512 output columns.  Arithmetic is
// fp32 on the CUDA cores.  This kernel serves head counts that are not a
// multiple of 128; blocks of 128 heads run on the tensor cores (mla_tc.cu).
#include <cuda_runtime.h>
#include <cstdint>

#include "api_internal.h"

namespace idx {
namespace {

constexpr int kMlaLat = 512;                 // latent width
constexpr int kMlaDim = 576;                 // latent + rotary
constexpr int kMlaHeads = 16;                // heads per CTA (one warp each)
constexpr int kMlaChunk = 32;                // selected positions per step (one per lane)
constexpr int kMlaThreads = kMlaHeads * 32;
constexpr int kMlaRowWords = kMlaDim / 2 + 1;   // 289 words per shared row: odd, conflict-free
constexpr int kMlaCols = kMlaLat / 32;       // output columns per lane

struct MlaSmem {
  float q[kMlaHeads][kMlaDim];
  uint32_t rows[kMlaChunk][kMlaRowWords];    // bf16 pairs
  float p[kMlaHeads][kMlaChunk];
  int tok[kMlaChunk];
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(kMlaThreads, 2)
    sparse_mla_decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kv,
                             const int32_t* __restrict__ indices, int H, int64_t T_cap, int k, float scale,
                             float* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  MlaSmem& sm = *reinterpret_cast<MlaSmem*>(smem_raw);
  const int groups = H / kMlaHeads;
  const int64_t b = blockIdx.x / groups;
  const int h0 = static_cast<int>(blockIdx.x % groups) * kMlaHeads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const uint16_t* qb = q + (b * H + h0) * kMlaDim;
  for (int i = tid; i < kMlaHeads * kMlaDim; i += kMlaThreads)
    (&sm.q[0][0])[i] = __uint_as_float(static_cast<uint32_t>(qb[i]) << 16);

  const int32_t* sel = indices + b * k;
  const uint4* kvb = reinterpret_cast<const uint4*>(kv + b * T_cap * kMlaDim);
  float m = -INFINITY, l = 0.f;
  float o[kMlaCols];
#pragma unroll
  for (int j = 0; j < kMlaCols; ++j) o[j] = 0.f;

  for (int c0 = 0; c0 < k; c0 += kMlaChunk) {
    __syncthreads();   // the previous chunk's rows and weights are no longer read
    if (tid < kMlaChunk) {
      const int j = c0 + tid;
      const int t = j < k ? sel[j] : -1;
      sm.tok[tid] = (t >= 0 && t < T_cap) ? t : -1;
    }
    __syncthreads();
    // gather: 32 rows × 72 16-byte pieces
    for (int i = tid; i < kMlaChunk * (kMlaDim / 8); i += kMlaThreads) {
      const int r = i / (kMlaDim / 8), u = i - r * (kMlaDim / 8);
      const int t = sm.tok[r];
      const uint4 v = t >= 0 ? __ldg(kvb + static_cast<int64_t>(t) * (kMlaDim / 8) + u) : make_uint4(0u, 0u, 0u, 0u);
      uint32_t* d = &sm.rows[r][4 * u];
      d[0] = v.x;
      d[1] = v.y;
      d[2] = v.z;
      d[3] = v.w;
    }
    __syncthreads();

    // score of row `lane` for head `warp`
    float s = -INFINITY;
    if (sm.tok[lane] >= 0) {
      const float* qh = sm.q[warp];
      const uint32_t* row = sm.rows[lane];
      float acc = 0.f;
#pragma unroll 8
      for (int d2 = 0; d2 < kMlaDim / 2; ++d2) {
        const uint32_t w = row[d2];
        acc = fmaf(qh[2 * d2], bf16_lo(w), acc);
        acc = fmaf(qh[2 * d2 + 1], bf16_hi(w), acc);
      }
      s = acc * scale;
    }
    // online softmax over the chunk (one warp = one head)
    float cmax = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xFFFFFFFFu, cmax, off));
    const float m_new = fmaxf(m, cmax);
    float p = 0.f, alpha = 1.f;
    if (m_new != -INFINITY) {
      p = s == -INFINITY ? 0.f : expf(s - m_new);
      alpha = m == -INFINITY ? 0.f : expf(m - m_new);
    }
    float psum = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xFFFFFFFFu, psum, off);
    l = l * alpha + psum;
    m = m_new;
    sm.p[warp][lane] = p;
    __syncwarp();

    // o[col] = alpha · o[col] + Σ_t p_t · row_t[col], columns lane + 32·j
#pragma unroll
    for (int j = 0; j < kMlaCols; ++j) o[j] *= alpha;
    const uint16_t* rows16 = reinterpret_cast<const uint16_t*>(&sm.rows[0][0]);
    for (int t = 0; t < kMlaChunk; ++t) {
      const float pt = sm.p[warp][t];
      const uint16_t* row = rows16 + t * (2 * kMlaRowWords);
#pragma unroll
      for (int j = 0; j < kMlaCols; ++j)
        o[j] = fmaf(pt, __uint_as_float(static_cast<uint32_t>(row[lane + 32 * j]) << 16), o[j]);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float* ob = out + (b * H + h0 + warp) * kMlaLat;
#pragma unroll
  for (int j = 0; j < kMlaCols; ++j) ob[lane + 32 * j] = o[j] * inv;
}

}  // namespace
}  // namespace idx

using namespace idx;

extern "C" int idx_sparse_mla_decode(const uint16_t* q, const uint16_t* kv, const int32_t* indices, int B, int H,
                                     int64_t T_cap, int k, float softmax_scale, float* out, idx_stream_t stream) {
  if (B < 0 || H <= 0 || H % kMlaHeads || T_cap <= 0) return IDX_ERR_SHAPE;
  if (k <= 0) return IDX_ERR_K;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f) return IDX_ERR_SHAPE;
  if (B == 0) return IDX_OK;
  if (!q || !kv || !indices || !out) return IDX_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(kv) & 15) return IDX_ERR_ALIGN;
  // 128-head blocks run on the tensor cores; other head counts on the CUDA cores
  const int rt = launch_sparse_mla_tc(q, kv, indices, B, H, T_cap, k, softmax_scale, out,
                                      reinterpret_cast<cudaStream_t>(stream));
  if (rt != IDX_ERR_UNSUPPORTED) return rt;
  const int64_t blocks = static_cast<int64_t>(B) * (H / kMlaHeads);
  if (blocks > 0x7FFFFFFF) return IDX_ERR_SHAPE;
  const int smem = static_cast<int>(sizeof(MlaSmem));
  if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(sparse_mla_decode_kernel), smem)) return r;
  sparse_mla_decode_kernel<<<static_cast<unsigned>(blocks), kMlaThreads, static_cast<size_t>(smem),
                             reinterpret_cast<cudaStream_t>(stream)>>>(q, kv, indices, H, T_cap, k, softmax_scale,
                                                                       out);
  return check_launch();
}
