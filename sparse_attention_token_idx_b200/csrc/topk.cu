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

// ---------------------------------------------------------------------------
// Rows held by one CTA.  The visible scores arrive by 1-D bulk copies of 16 KB,
// all issued at once; as each lands, a pass over shared memory turns it into
// order keys, counts the level-1 histogram and its coarse sums, and keeps the
// short list of keys that may reach the top k (row_filter_*); then
// cta_select_row writes the positions straight to global memory.  Several
// CTAs share an SM, so one row's selection overlaps another's copies.

constexpr int kRowThreads = 512;    // one-CTA rows longer than 8192 keys: 16 warps
constexpr int kRowChunk = 4096;     // floats per bulk copy
constexpr int kRowMaxChunks = 4;    // rows of up to 16384 keys

struct RowLayout {
  int hist1, scratch, keys, bars, total;
};

__host__ __device__ inline RowLayout row_layout(int chunk_cap, int list_cap, int cand_cap) {
  RowLayout l;
  l.hist1 = (static_cast<int>(sizeof(CtaSelSmem)) + 127) / 128 * 128;
  l.scratch = l.hist1 + kHistBins * 4;
  l.keys = l.scratch + ((list_cap + cand_cap) * 2 + 15) / 16 * 16;
  l.bars = l.keys + chunk_cap * 4;
  l.total = l.bars + kRowMaxChunks * 8;
  return l;
}

struct RowParams {
  const float* scores;
  const int32_t* lengths;
  int32_t* indices;
  int64_t ld;
  int B, n, max_len, causal, k;
  int chunk_cap, list_cap, cand_cap;
  unsigned long long budget_ns;
  unsigned int* err;
  unsigned long long* trace;
};

__global__ void __launch_bounds__(kRowThreads, 2) topk_row_kernel(const RowParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);   // shared-space pointer
  const RowLayout L = row_layout(p.chunk_cap, p.list_cap, p.cand_cap);
  CtaSelSmem& sel = *reinterpret_cast<CtaSelSmem*>(smem);
  uint32_t* hist1 = reinterpret_cast<uint32_t*>(smem + L.hist1);
  uint16_t* list16 = reinterpret_cast<uint16_t*>(smem + L.scratch);
  uint16_t* cand16 = list16 + p.list_cap;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);   // fp32 scores until converted
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  __shared__ int timed_out;
  const int tid = threadIdx.x, nthr = blockDim.x;
  unsigned long long* tr = (p.trace && blockIdx.x < 8192) ? p.trace + blockIdx.x * kTraceSlotsT : nullptr;
  if (tr && tid == 0) tr[0] = globaltimer_ns();
  const int64_t row = blockIdx.x;              // b * n + i
  const int b = static_cast<int>(row / p.n);
  const int i = static_cast<int>(row - static_cast<int64_t>(b) * p.n);
  const int len = p.lengths[b];
  const bool bad = len < p.n || len > p.max_len;
  if (bad && tid == 0 && i == 0) raise_error(p.err, IDX_DEV_ERR_LENGTH);
  const int vis = bad ? 0 : (p.causal ? len - p.n + i + 1 : len);
  int32_t* out = p.indices + row * p.k;
  const int kt = min(p.k, vis);
  if (kt == vis) {   // every visible position is selected (or none is visible)
    for (int t = tid; t < p.k; t += nthr) out[t] = t < kt ? t : -1;
    return;
  }
  const float* src = p.scores + row * p.ld;
  const int n4 = (vis + 3) & ~3;               // floats copied: within the row, since ld % 4 == 0
  const int nchunks = (n4 + kRowChunk - 1) / kRowChunk;
  if (tid == 0) {
    for (int c = 0; c < nchunks; ++c) mbar_init(&bars[c], 1);
    fence_barrier_init();
    for (int c = 0; c < nchunks; ++c) {
      const int cnt = min(kRowChunk, n4 - c * kRowChunk);
      mbar_arrive_expect_tx(&bars[c], static_cast<uint32_t>(cnt) * 4u);
      bulk_load(keys + c * kRowChunk, src + c * kRowChunk, static_cast<uint32_t>(cnt) * 4u, &bars[c]);
    }
    row_filter_reset(sel);
    timed_out = 0;
  }
  select_prepare(sel);
  for (int t = tid; t < kHistBins; t += nthr) hist1[t] = 0u;
  __syncthreads();
  // the list pays off when the k best are a small share of the row
  const bool use_list = p.list_cap > 0 && vis >= 4 * kt;
  const int warp = tid >> 5;
  // floats [lo, hi) → order keys in place (key 0 past vis), counted in the
  // level-1 histogram; with `list`, keys at or above the bound go to the list
  // (one shared atomic per warp and 128 keys).  Trip count uniform per warp.
  const uint32_t lt = lanemask_lt();
  auto convert = [&](int lo, int hi, bool list, bool keys_ready) {
    const uint32_t bound = *reinterpret_cast<const volatile uint32_t*>(&sel.filt_lo);
    for (int base = lo; base < hi; base += 4 * nthr) {
      const int i0 = base + 4 * tid;
      uint32_t u[4] = {0u, 0u, 0u, 0u};
      if (i0 < hi) {
        const uint4 v = *reinterpret_cast<const uint4*>(keys + i0);
        const uint32_t f[4] = {v.x, v.y, v.z, v.w};
        if (keys_ready) {
#pragma unroll
          for (int e = 0; e < 4; ++e) u[e] = f[e];
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) u[e] = i0 + e < vis ? order_key(__uint_as_float(f[e])) : 0u;
          *reinterpret_cast<uint4*>(keys + i0) = make_uint4(u[0], u[1], u[2], u[3]);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (u[e] != 0u) atomicAdd(&hist1[u[e] >> 21], 1u);
        }
      }
      if (!list) continue;
      uint32_t m[4];
      int tot = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        m[e] = __ballot_sync(0xFFFFFFFFu, u[e] != 0u && u[e] >= bound);
        tot += __popc(m[e]);
      }
      if (tot == 0) continue;
      int pos = 0;
      if ((tid & 31) == 0) pos = atomicAdd(&sel.list_cnt, tot);
      pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = pos + __popc(m[e] & lt);
        if ((m[e] >> (tid & 31) & 1u) && q < p.list_cap) list16[q] = static_cast<uint16_t>(i0 + e);
        pos += __popc(m[e]);
      }
    }
  };
  auto wait_chunk = [&](int c) -> bool {   // block-uniform: false when the copies gave up
    if (tid == 0 && !timed_out) {
      volatile int* flag = &timed_out;
      mbar_wait(&bars[c], 0, p.budget_ns, flag, p.err);
    }
    return !__syncthreads_or(timed_out);
  };
  bool ok = true;
  for (int c = 0; c < nchunks && ok; ++c) {
    ok = wait_chunk(c);
    if (!ok) break;
    if (tr && tid == 0 && c == 0) tr[1] = globaltimer_ns();
    const int lo = c * kRowChunk, hi = min(lo + kRowChunk, n4);
    if (c == 0 && use_list) {
      // the first chunk alone sets the bound (1.5 × its expected share of the k
      // best), then its keys are listed against it
      convert(lo, hi, false, false);
      if (tr && tid == 0) tr[2] = globaltimer_ns();
      __syncthreads();
      if (warp == 0) {
        const int target = row_filter_target(hi, vis, kt);
        if (target > 0) row_filter_raise_fine(sel, hist1, target);
      }
      __syncthreads();
      if (tr && tid == 0) tr[5] = globaltimer_ns();
      convert(lo, hi, true, true);
    } else {
      if (c == 2 && use_list && warp == 0) {
        // raised once more on the first two chunks' counts (complete: every warp
        // passed the barrier of this chunk's wait)
        const int target = row_filter_target(lo, vis, kt);
        if (target > 0) row_filter_raise_fine(sel, hist1, target);
      }
      convert(lo, hi, use_list, false);
    }
    if (tr && tid == 0 && c == 0) tr[6] = globaltimer_ns();
  }
  if (!ok) {
    // give up on this row: let every copy land (bounded) before the CTA exits
    if (tid == 0) {
      int dummy = 0;
      for (int d = 0; d < nchunks; ++d) mbar_wait(&bars[d], 0, p.budget_ns, &dummy, p.err);
    }
    __syncthreads();
    for (int t = tid; t < p.k; t += nthr) out[t] = -1;
    return;
  }
  __syncthreads();
  if (tid < 64) {   // level-1 coarse sums
    const uint4* h = reinterpret_cast<const uint4*>(hist1 + 32 * tid);
    uint32_t sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 v = h[q];
      sum += v.x + v.y + v.z + v.w;
    }
    sel.coarse[0][tid] = sum;
  }
  __syncthreads();
  if (tr && tid == 0) tr[3] = globaltimer_ns();
  cta_select_row(sel, keys, vis, 0, kt, hist1, true, use_list ? list16 : nullptr, p.list_cap, cand16, p.cand_cap,
                 out, nullptr, tr, nullptr);
  for (int t = kt + tid; t < p.k; t += nthr) out[t] = -1;
  if (tr && tid == 0) tr[4] = globaltimer_ns();
}

// ---------------------------------------------------------------------------
// A sequence's keys split over G GPUs: each GPU selects the k best of its
// slice and contributes them as (score, position) pairs; one exchange gives
// every GPU all G·k candidates of a row, and the merge selects the row's k best
// among them.  Exact: a key in the row's top k is in its own slice's top k.

__global__ void __launch_bounds__(256) gather_scores_kernel(const float* __restrict__ scores, int64_t ld,
                                                            const int32_t* __restrict__ idx, int64_t rows, int k,
                                                            const int32_t* __restrict__ counts, int32_t offset,
                                                            idx_cand_t* __restrict__ cand) {
  const int64_t total = rows * k;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = t / k;
    const int32_t i0 = idx[t];
    const int32_t i = (counts && i0 >= counts[r]) ? -1 : i0;
    idx_cand_t c;
    c.score = i >= 0 ? scores[r * ld + i] : -INFINITY;
    c.pos = i >= 0 ? i + offset : -1;
    cand[t] = c;
  }
}

constexpr int kMergeMax = 16384;   // candidates per row (16-bit slots, one CTA)
constexpr int kMergeThreads = 512;

struct MergeLayout {
  int hist1, cand, keys, pos, sel, total;
};

// shared memory: selection state | level-1 histogram | bin-b1 slot list |
// order keys [m4] | positions [m4] | selected slots [m4]
__host__ __device__ inline MergeLayout merge_layout(int m4, int cand_cap) {
  MergeLayout l;
  l.hist1 = (static_cast<int>(sizeof(CtaSelSmem)) + 127) / 128 * 128;
  l.cand = l.hist1 + kHistBins * 4;
  l.keys = l.cand + (cand_cap * 2 + 15) / 16 * 16;
  l.pos = l.keys + m4 * 4;
  l.sel = l.pos + m4 * 4;
  l.total = l.sel + m4 * 4;
  return l;
}

// One CTA per row.  Candidates [G, rows, kin] (rank-major, as an all-gather of
// the per-GPU [rows, kin] arrays lays them out); slot s = g·kin + j of row r.
// PAIRS2: kin even and cand 16-byte aligned, so two pairs come in one load.
template <bool PAIRS2>
__global__ void __launch_bounds__(kMergeThreads) merge_topk_kernel(const idx_cand_t* __restrict__ cand, int G,
                                                                   int64_t rows, int kin, int k, int cand_cap,
                                                                   int32_t* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  const int m = G * kin, m4 = (m + 3) & ~3;
  const MergeLayout L = merge_layout(m4, cand_cap);
  CtaSelSmem& sel = *reinterpret_cast<CtaSelSmem*>(smem);
  uint32_t* hist1 = reinterpret_cast<uint32_t*>(smem + L.hist1);
  uint16_t* cand16 = reinterpret_cast<uint16_t*>(smem + L.cand);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
  int32_t* pos_s = reinterpret_cast<int32_t*>(smem + L.pos);
  int32_t* sel_s = reinterpret_cast<int32_t*>(smem + L.sel);
  __shared__ int nvalid, next;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int64_t row = blockIdx.x;
  int32_t* o = out + row * k;
  select_prepare(sel);
  for (int t = tid; t < kHistBins; t += nthr) hist1[t] = 0u;
  for (int t = m + tid; t < m4; t += nthr) keys[t] = 0u;
  if (tid == 0) {
    nvalid = 0;
    next = 0;
  }
  __syncthreads();
  int mine = 0;
  // empty slots (position −1) get key 0: below every bin a score maps to
  auto put = [&](int s, float score, int32_t p) {
    const bool ok = p >= 0;
    const uint32_t key = ok ? order_key(score) : 0u;
    keys[s] = key;
    pos_s[s] = p;
    if (ok) {
      select_count_key(sel, hist1, key);
      ++mine;
    }
  };
  constexpr int U = 4;   // loads in flight per thread
  if (PAIRS2) {
    const int half = kin >> 1, items = G * half;
    for (int j0 = tid; j0 < items; j0 += U * nthr) {
      int4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * nthr;
        if (j < items) {
          const int g = j / half, jj = j - g * half;
          v[u] = __ldg(reinterpret_cast<const int4*>(cand + (static_cast<int64_t>(g) * rows + row) * kin) + jj);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * nthr;
        if (j < items) {
          const int g = j / half, s = g * kin + 2 * (j - g * half);
          put(s, __int_as_float(v[u].x), v[u].y);
          put(s + 1, __int_as_float(v[u].z), v[u].w);
        }
      }
    }
  } else {
    for (int s0 = tid; s0 < m; s0 += U * nthr) {
      int2 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int s = s0 + u * nthr;
        if (s < m) {
          const int g = s / kin;
          v[u] = __ldg(reinterpret_cast<const int2*>(cand + (static_cast<int64_t>(g) * rows + row) * kin) +
                       (s - g * kin));
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int s = s0 + u * nthr;
        if (s < m) put(s, __int_as_float(v[u].x), v[u].y);
      }
    }
  }
  for (int o2 = 16; o2 > 0; o2 >>= 1) mine += __shfl_xor_sync(0xFFFFFFFFu, mine, o2);
  if ((tid & 31) == 0 && mine) atomicAdd(&nvalid, mine);
  __syncthreads();
  const int v = nvalid;
  const int kt = min(k, v);
  if (kt == v) {
    // every candidate is kept: compact them in slot order (one shared counter per warp step)
    for (int base = 0; base < m4; base += nthr) {
      const int s = base + tid;
      const bool take = s < m && keys[s] != 0u;
      const uint32_t mk = __ballot_sync(0xFFFFFFFFu, take);
      int at = 0;
      if ((tid & 31) == 0 && mk) at = atomicAdd(&next, __popc(mk));
      at = __shfl_sync(0xFFFFFFFFu, at, 0) + __popc(mk & lanemask_lt());
      if (take) o[at] = pos_s[s];
    }
    for (int t = kt + tid; t < k; t += nthr) o[t] = -1;
    return;
  }
  // slots of the kt best (into shared memory), then their positions
  cta_select_row(sel, keys, m, 0, kt, hist1, true, nullptr, 0, cand16, cand_cap, sel_s, nullptr, nullptr, nullptr);
  __syncthreads();
  for (int t = tid; t < k; t += nthr) o[t] = t < kt ? pos_s[sel_s[t]] : -1;
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
  // one CTA per row when the row fits a CTA and enough rows cover the GPU:
  // bulk copies need 16-byte aligned rows
  const bool aligned = (reinterpret_cast<uintptr_t>(scores) & 15u) == 0 && (ld & 3) == 0;
  if (aligned && max_len <= kRowChunk * kRowMaxChunks && (rows >= 64 || rows * 2 >= sms) && rows <= 0x7FFFFFFF) {
    const int chunk_cap = (max_len + 3) & ~3;
    const int list_cap = chunk_cap >= 4 * k ? (min(6144, chunk_cap / 2) & ~3) : 0;
    const int cand_cap = min(2048, chunk_cap);
    const RowLayout L = row_layout(chunk_cap, list_cap, cand_cap);
    const int smem = L.total + 128;
    if (smem > max_dynamic_smem()) return IDX_ERR_SHAPE;
    if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(topk_row_kernel), smem)) return r;
    const DebugState dbg = debug_state();
    RowParams rp{scores, lengths, indices, ld, B, n, max_len, causal, k, chunk_cap, list_cap, cand_cap,
                 dbg.budget_ns, device_error_word(), (dbg.flags & 2u) ? trace_buffer() : nullptr};
    if (!rp.err) return check_launch();
    // long rows: 16 warps per CTA hide shared-memory latency; short rows: more CTAs per SM
    const int threads = chunk_cap > 2 * kRowChunk ? kRowThreads : kTopkThreads;
    topk_row_kernel<<<static_cast<unsigned>(rows), threads, static_cast<size_t>(smem),
                      reinterpret_cast<cudaStream_t>(stream)>>>(rp);
    return check_launch();
  }
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
  if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(topk_kernel), smem)) return r;
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

extern "C" int idx_gather_scores(const float* scores, int64_t ld, const int32_t* idx, int64_t rows, int k,
                                 const int32_t* counts, int32_t offset, idx_cand_t* cand, idx_stream_t stream) {
  if (rows < 0 || k < 0 || ld <= 0) return IDX_ERR_SHAPE;
  if (rows == 0 || k == 0) return IDX_OK;
  if (!scores || !idx || !cand) return IDX_ERR_NULL;
  const int64_t total = rows * k;
  const int64_t blocks = (total + 255) / 256;
  const int grid = static_cast<int>(blocks < 148 * 16 ? blocks : 148 * 16);
  gather_scores_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(scores, ld, idx, rows, k, counts,
                                                                                 offset, cand);
  return check_launch();
}

extern "C" int idx_merge_topk(const idx_cand_t* cand, int G, int64_t rows, int kin, int k, int32_t* out,
                              idx_stream_t stream) {
  if (G <= 0 || rows < 0 || kin <= 0) return IDX_ERR_SHAPE;
  if (k <= 0) return IDX_ERR_K;
  if (rows == 0) return IDX_OK;
  if (!cand || !out) return IDX_ERR_NULL;
  if (static_cast<int64_t>(G) * kin > kMergeMax || rows > 0x7FFFFFFF) return IDX_ERR_SHAPE;
  const int m4 = (G * kin + 3) & ~3;
  const int cand_cap = 2048;
  const int smem = merge_layout(m4, cand_cap).total + 128;
  const bool pairs2 = (kin % 2) == 0 && (reinterpret_cast<uintptr_t>(cand) & 15u) == 0;
  auto kern = pairs2 ? merge_topk_kernel<true> : merge_topk_kernel<false>;
  if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem)) return r;
  kern<<<static_cast<unsigned>(rows), kMergeThreads, static_cast<size_t>(smem),
         reinterpret_cast<cudaStream_t>(stream)>>>(cand, G, rows, kin, k, cand_cap, out);
  return check_launch();
}
