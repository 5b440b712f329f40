// Top-k over scores already in memory (Indexer.forward excerpt: top
// min(index_topk, ·) positions per row; NKI indexer page: int32, unordered).
//
// One thread-block cluster of G CTAs per query row; each CTA loads a
// contiguous slice of the row's visible scores into shared memory as
// order-preserving keys, then the cluster runs the same radix select as the
// fused score kernel.
#include <cuda_runtime.h>
#include <cstdint>

#include "api_internal.h"
#include "ptx.cuh"
#include "select.cuh"

namespace idx {
namespace {

constexpr int kTopkThreads = 256;
constexpr int kTopkCandMax = 4096;   // candidate list entries (at most)

constexpr int kTraceSlotsT = 16;

// Candidates are the keys of the threshold bin of the level-1 histogram, a
// small part of a row; a quarter of the slice (1024 … 4096 entries) holds
// them, and a list that overflows falls back to scanning the slice.
int topk_cand_cap(int chunk_cap) {
  int c = chunk_cap / 4;
  c = c < 1024 ? 1024 : c;
  return c > kTopkCandMax ? kTopkCandMax : c;
}

struct TopkParams {
  const float* scores;
  const int32_t* lengths;
  int32_t* indices;
  int64_t ld;
  int B, n, max_len, causal, k, G, chunk_cap, cand_cap;
  unsigned int* err;
  unsigned long long* trace;   // per-CTA phase stamps, or null
};

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);   // shared-space pointer
  SelectSmem& sel = *reinterpret_cast<SelectSmem*>(smem);
  uint32_t* hist1 = reinterpret_cast<uint32_t*>(smem + sizeof(SelectSmem));
  int* cand = reinterpret_cast<int*>(smem + sizeof(SelectSmem) + kHistBins * 4);
  uint32_t* sc_s = reinterpret_cast<uint32_t*>(smem + sizeof(SelectSmem) + kHistBins * 4 + p.cand_cap * 4);
  unsigned long long* tr = (p.trace && blockIdx.x < 8192) ? p.trace + blockIdx.x * kTraceSlotsT : nullptr;
  if (tr && threadIdx.x == 0) tr[0] = globaltimer_ns();
  const uint32_t rank = cluster_rank();
  const int G = p.G;
  const int64_t row = blockIdx.x / G;          // b * n + i
  const int b = static_cast<int>(row / p.n);
  const int i = static_cast<int>(row - static_cast<int64_t>(b) * p.n);
  const int len = p.lengths[b];
  const bool bad = len < p.n || len > p.max_len;
  if (bad && rank == 0 && threadIdx.x == 0 && i == 0) raise_error(p.err, IDX_DEV_ERR_LENGTH);
  const int vis = bad ? 0 : (p.causal ? len - p.n + i + 1 : len);
  const int chunk = vis > 0 ? (vis + G - 1) / G : 0;
  const int start = static_cast<int>(rank) * chunk;
  const int nloc = max(0, min(start + chunk, vis) - start);
  const float* src = p.scores + row * p.ld + start;
  int32_t* out = p.indices + row * p.k;
  const int kt = min(p.k, vis);
  if (kt == vis) {
    // every visible position is selected: no scores needed, slot s holds position s
    for (int t = threadIdx.x; t < nloc; t += blockDim.x) out[start + t] = start + t;
    if (rank == 0)
      for (int t = kt + threadIdx.x; t < p.k; t += blockDim.x) out[t] = -1;
    if (tr && threadIdx.x == 0) tr[4] = globaltimer_ns();
    return;   // uniform over the cluster (same vis): no CTA waits at a cluster barrier
  }
  for (int t = threadIdx.x; t < kHistBins; t += blockDim.x) hist1[t] = 0;
  __syncthreads();
  // four independent loads in flight per thread
  const int nthr = blockDim.x;
  for (int t0 = threadIdx.x; t0 < nloc; t0 += 4 * nthr) {
    float f[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = t0 + e * nthr;
      f[e] = t < nloc ? __ldg(src + t) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = t0 + e * nthr;
      if (t < nloc) {
        const uint32_t u = order_key(f[e]);
        sc_s[t] = u;
        atomicAdd(&hist1[u >> 21], 1u);
      }
    }
  }
  // pad the slice with key 0 up to a multiple of 4 (the selection reads whole vectors)
  if (threadIdx.x < 4 && nloc + static_cast<int>(threadIdx.x) < ((nloc + 3) & ~3)) sc_s[nloc + threadIdx.x] = 0u;
  __syncthreads();
  if (tr && threadIdx.x == 0) tr[3] = globaltimer_ns();
  cluster_select_row(sel, sc_s, nloc, start, kt, hist1, cand, p.cand_cap, 0, false, out, G, rank, tr);
  if (rank == 0)
    for (int t = kt + threadIdx.x; t < p.k; t += blockDim.x) out[t] = -1;
  if (G > 1) cluster_sync();
  if (tr && threadIdx.x == 0) tr[4] = globaltimer_ns();
}

int pow2_floor_i(int x) {
  int r = 1;
  while (r * 2 <= x) r *= 2;
  return r;
}

}  // namespace
}  // namespace idx

using namespace idx;

extern "C" int idx_topk(const float* scores, const int32_t* lengths, int B, int n, int64_t ld, int max_len,
                        int causal, int k, int32_t* indices, void* ws, size_t ws_bytes, idx_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (B < 0 || n < 0) return IDX_ERR_SHAPE;
  if (k <= 0) return IDX_ERR_K;
  if (B == 0 || n == 0) return IDX_OK;
  if (!scores || !lengths || !indices) return IDX_ERR_NULL;
  if (causal != 0 && causal != 1) return IDX_ERR_SHAPE;
  if (max_len < n || max_len > IDX_MAX_LEN || static_cast<int64_t>(max_len) > ld) return IDX_ERR_SHAPE;
  const int64_t rows = static_cast<int64_t>(B) * n;
  const int sms = num_sms();
  int G = rows < sms ? pow2_floor_i(static_cast<int>(sms / rows)) : 1;
  if (G > 8) G = 8;
  while (G > 1 && (max_len + G - 1) / G < 512) G /= 2;
  const int budget = 64 * 1024;
  while (G < 8 && static_cast<int64_t>((max_len + G - 1) / G) * 4 > budget) G *= 2;
  const int chunk_cap = ((max_len + G - 1) / G + 3) / 4 * 4;   // whole 16-byte vectors
  const int cand_cap = topk_cand_cap(chunk_cap);
  const int smem = 128 + static_cast<int>(sizeof(SelectSmem)) + (kHistBins + cand_cap) * 4 + chunk_cap * 4;
  if (smem > max_dynamic_smem()) return IDX_ERR_SHAPE;
  if (rows * G > 0x7FFFFFFF) return IDX_ERR_SHAPE;
  static int configured = -1;
  if (configured < smem) {
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return check_launch();
    configured = smem;
  }
  TopkParams p{scores, lengths, indices, ld, B, n, max_len, causal, k, G, chunk_cap, cand_cap, device_error_word(),
               (debug_state().flags & 2u) ? trace_buffer() : nullptr};
  if (!p.err) return check_launch();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * G), 1, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(G);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, topk_kernel, p);
  return check_launch();
}
