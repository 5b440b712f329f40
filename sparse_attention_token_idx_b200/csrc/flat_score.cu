// Index scores ("Index scores" page: score equation S^I and the fp8_index
// docstring; causal mask from the Indexer.forward excerpt) with a flat work
// partition, for score + top-k calls that go through a workspace.
//
// Every (row block, key tile) pair of the call is one unit: a row block is NT
// query rows of one sequence (its 64·NT query heads on the MMA's N side), a
// key tile is 128 cached keys.  Units are numbered row block by row block and
// each CTA — one per SM, persistent — takes an equal contiguous range, so the
// SMs stream equal shares of the cache whatever the mix of lengths (decode
// batches, causal triangles).  Roles as in the per-item kernel:
//   warp 0      TMA producer: per row block the query heads (3-D tensor map)
//               and the folded weights (1-D bulk copy) into one of two slots,
//               and per unit a 128-key tile into a STAGES ring (freed once the
//               MMA has read it) and its scales into a deeper ring that the
//               epilogue frees, so key stages are never held by the epilogue;
//   warp 1      owns TMEM and issues tcgen05.mma kind::f8f6f4 (keys on M, the
//               row block's heads on N, K = 128 as four K = 32 steps) into
//               NUM_ACC accumulators;
//   warps 2 …   epilogue: thread ↔ key, S = k_scale · Σ_h w_h · max(L_h, 0),
//               −inf past each row's visible count, fp32 row-major stores.
// The producer and the MMA issuer sleep in their waits (mbar_wait_sleep), so
// that their polling leaves the issue slots to the epilogue warps, which bound
// the kernel (measured on the chunked-prefill workload: 693 → 685 µs); the
// epilogue warps poll (sleeping there measured slower).
// A query slot is refilled only after the MMA warp and every epilogue warp
// are done with its row block.  Columns past a row block's last tile are not
// written: the top-k that reads the workspace stops at each row's visible
// count.  Every wait is bounded; a CTA that gives up raises
// IDX_DEV_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "api_internal.h"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace idx {
namespace {

constexpr int kFKeys = 128;
constexpr int kFTileBytes = kFKeys * IDX_DIM;   // 16 KB
constexpr int kFlatMaxItems = 4096;              // row blocks per call (prefix sums in shared memory)
constexpr int kFScaleSlots = 16;                 // key-scale ring: outlives the key stages (epilogue reads)

struct FlatParams {
  const float* w;            // [B, n, 64] folded weights
  const int32_t* lengths;    // [B]
  float* scores;             // [B, n, ld]
  int64_t ld;
  int B, n, max_len, causal;
  int ntb;                   // row blocks per sequence
  int items;                 // B · ntb
  unsigned int debug_flags;
  unsigned long long budget_ns;
  unsigned int* err;
  unsigned long long* trace;   // per-CTA phase stamps (16 slots), or null
  int scale_u8;                // key scales stored as e8m0 bytes (else fp32)
};

template <int NT, int STAGES, int NUM_ACC, int EPI_WARPS, int TSPLIT, bool W_REGS>
struct FCfg {
  static constexpr int N = NT * IDX_HEADS;
  static constexpr int kThreads = (2 + EPI_WARPS) * 32;
  static constexpr int kAccCols = NUM_ACC * N;
  static constexpr int kTmemCols = kAccCols <= 32 ? 32 : kAccCols <= 64 ? 64 : kAccCols <= 128 ? 128
                                 : kAccCols <= 256 ? 256 : 512;
  static_assert(kAccCols <= 512, "TMEM holds 512 columns");
  static_assert(kThreads <= 32 * 32, "per-warp scan totals");
  static constexpr int kTokGroups = EPI_WARPS / 4 / TSPLIT;
  static_assert(EPI_WARPS % (4 * TSPLIT) == 0 && NT % kTokGroups == 0, "epilogue split");
  static constexpr int kTokPerWarp = NT / kTokGroups;
  static constexpr int kWarpsPerTile = EPI_WARPS / TSPLIT;
  static constexpr int kQBytes = N * IDX_DIM;     // a multiple of 1024 (128-byte swizzle atoms)
  static constexpr int kWBytes = N * 4;
  static constexpr int kOffQ = 0;                 // two slots
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffScale = kOffK + STAGES * kFTileBytes;
  static constexpr int kOffW = kOffScale + kFScaleSlots * kFKeys * 4;   // two slots
  static constexpr int kOffBar = kOffW + 2 * kWBytes;
  static constexpr int kNumBars = 2 * STAGES + kFScaleSlots + 2 * NUM_ACC + 2 + 2 + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffScan = kOffMisc + 16;                    // per-warp totals, 32 warps at most
  static constexpr int kOffPrefix = (kOffScan + 32 * 4 + 15) / 16 * 16;
  static int smem_bytes(int items) { return 1024 + kOffPrefix + (items + 1) * 4; }
};

// Row block `item` of the call: sequence, first row, and the keys its rows see.
template <int NT>
struct Block {
  int b, row0, len;
  bool bad;
  __device__ __forceinline__ void set(const FlatParams& p, int item) {
    b = item / p.ntb;
    row0 = (item - b * p.ntb) * NT;
    len = p.lengths[b];
    bad = len < p.n || len > p.max_len;
  }
  __device__ __forceinline__ int vis(const FlatParams& p, int row) const {   // keys row `row` sees
    return (row < p.n && !bad) ? (p.causal ? len - p.n + row + 1 : len) : 0;
  }
  __device__ __forceinline__ int tiles(const FlatParams& p) const {
    const int last = min(row0 + NT, p.n) - 1;
    return (vis(p, last) + kFKeys - 1) / kFKeys;
  }
};

// Walks this CTA's units in order: (row block, key tile), skipping empty blocks.
struct Walker {
  int item, tile, ntile;
  __device__ __forceinline__ void start(const int* prefix, int items, int64_t u0) {
    int lo = 0, hi = items - 1;   // last item whose first unit is ≤ u0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= u0) lo = mid; else hi = mid - 1;
    }
    item = lo;
    tile = static_cast<int>(u0 - prefix[lo]);
    ntile = prefix[lo + 1] - prefix[lo];
  }
  __device__ __forceinline__ void next(const int* prefix, int items) {
    ++tile;
    while (tile >= ntile && item < items - 1) {
      ++item;
      tile = 0;
      ntile = prefix[item + 1] - prefix[item];
    }
  }
};

template <int NT, int STAGES, int NUM_ACC, int EPI_WARPS, int TSPLIT, bool W_REGS>
__global__ void __launch_bounds__(FCfg<NT, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>::kThreads, 1)
    flat_score_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_s, const FlatParams p) {
  using C = FCfg<NT, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>;
  constexpr int N = C::N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* q_s = smem + C::kOffQ;
  uint8_t* k_s = smem + C::kOffK;
  float* scale_s = reinterpret_cast<float*>(smem + C::kOffScale);
  float* w_s = reinterpret_cast<float*>(smem + C::kOffW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* sc_empty = bars + 2 * STAGES;   // [kFScaleSlots]
  uint64_t* acc_full = sc_empty + kFScaleSlots;
  uint64_t* acc_empty = acc_full + NUM_ACC;
  uint64_t* q_full = acc_empty + NUM_ACC;   // [2]
  uint64_t* q_empty = q_full + 2;           // [2]
  uint64_t* drain_bar = q_empty + 2;
  uint64_t* never_bar = drain_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* scan_w = reinterpret_cast<int*>(smem + C::kOffScan);       // per-warp totals
  int* prefix = reinterpret_cast<int*>(smem + C::kOffPrefix);     // [items + 1]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x, nthr = blockDim.x;
  unsigned long long* tr = p.trace ? p.trace + static_cast<size_t>(blockIdx.x) * 16 : nullptr;
  if (tr && tid == 0) tr[0] = globaltimer_ns();

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);   // the MMA is done with the keys
    }
    for (int c = 0; c < kFScaleSlots; ++c) mbar_init(&sc_empty[c], C::kWarpsPerTile);   // epilogue done with the scales
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], C::kWarpsPerTile);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&q_full[q], 1);
      mbar_init(&q_empty[q], 1 + EPI_WARPS);   // MMA done with the heads, every epilogue warp with the weights
    }
    mbar_init(drain_bar, 1);
    mbar_init(never_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_s);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);

  // ---- units per row block → prefix sums (block scan over contiguous runs)
  {
    const int per = (p.items + nthr - 1) / nthr;
    const int i0 = min(p.items, tid * per), i1 = min(p.items, i0 + per);
    int local = 0;
    Block<NT> blk;
    for (int i = i0; i < i1; ++i) {
      blk.set(p, i);
      if (blk.bad && blk.row0 == 0) raise_error(p.err, IDX_DEV_ERR_LENGTH);
      local += blk.tiles(p);
    }
    int inc = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane == 31) scan_w[warp] = inc;
    __syncthreads();
    int base = 0;
    for (int w2 = 0; w2 < warp; ++w2) base += scan_w[w2];
    int run = base + inc - local;
    for (int i = i0; i < i1; ++i) {
      prefix[i] = run;
      blk.set(p, i);
      run += blk.tiles(p);
    }
    if (tid == nthr - 1) prefix[p.items] = base + inc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t budget = p.budget_ns;
  const int64_t total = prefix[p.items];
  const int64_t u0 = total * blockIdx.x / gridDim.x;
  const int64_t u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int nunits = static_cast<int>(u1 - u0);
  if (tr && tid == 0) {
    tr[1] = globaltimer_ns();
    tr[6] = static_cast<unsigned long long>(nunits);
  }

  int tma_issued = 0;      // producer: units whose key tile was requested
  int q_issued = 0;        // producer: row blocks whose heads were requested
  bool mma_issued = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nunits > 0) {
      Walker wk;
      wk.start(prefix, p.items, u0);
      Block<NT> blk;
      int cur = -1;
      for (int k = 0; k < nunits; ++k, wk.next(prefix, p.items)) {
        if (wk.item != cur) {
          cur = wk.item;
          blk.set(p, cur);
          const int slot = q_issued & 1;
          if (q_issued >= 2 && !mbar_wait_sleep(&q_empty[slot], ((q_issued >> 1) - 1) & 1, budget, abort_flag, p.err))
            break;
          const int rows = min(NT, p.n - blk.row0);
          mbar_arrive_expect_tx(&q_full[slot], static_cast<uint32_t>(C::kQBytes + rows * IDX_HEADS * 4));
          tma_load_3d(q_s + slot * C::kQBytes, &tmap_q, &q_full[slot], 0, blk.row0 * IDX_HEADS, blk.b);
          bulk_load(w_s + slot * N, p.w + (static_cast<int64_t>(blk.b) * p.n + blk.row0) * IDX_HEADS,
                    static_cast<uint32_t>(rows * IDX_HEADS * 4), &q_full[slot]);
          ++q_issued;
        }
        const int s = k % STAGES;
        const int c = k % kFScaleSlots;
        if (!mbar_wait_sleep(&empty[s], ((k / STAGES) & 1) ^ 1, budget, abort_flag, p.err)) break;
        if (!mbar_wait_sleep(&sc_empty[c], ((k / kFScaleSlots) & 1) ^ 1, budget, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&full[s], kFTileBytes + kFKeys * (p.scale_u8 ? 1 : 4));
        tma_load_3d(k_s + s * kFTileBytes, &tmap_k, &full[s], 0, wk.tile * kFKeys, blk.b);
        tma_load_2d(scale_s + c * kFKeys, &tmap_s, &full[s], wk.tile * kFKeys, blk.b);
        tma_issued = k + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nunits > 0) {
      if (p.debug_flags & 1u) mbar_wait(never_bar, 0, budget, abort_flag, p.err);  // fault injection
      Walker wk;
      wk.start(prefix, p.items, u0);
      int cur = -1, qseq = -1;
      constexpr uint32_t idesc = idesc_e4m3_f32(128, N);
      for (int k = 0; k < nunits && !*abort_flag; ++k, wk.next(prefix, p.items)) {
        if (wk.item != cur) {
          cur = wk.item;
          ++qseq;
          if (!mbar_wait_sleep(&q_full[qseq & 1], (qseq >> 1) & 1, budget, abort_flag, p.err)) break;
        }
        const int s = k % STAGES;
        const int a = k % NUM_ACC;
        if (!mbar_wait_sleep(&full[s], (k / STAGES) & 1, budget, abort_flag, p.err)) break;
        if (!mbar_wait_sleep(&acc_empty[a], ((k / NUM_ACC) & 1) ^ 1, budget, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(q_s + (qseq & 1) * C::kQBytes);
        const uint32_t k_addr = smem_u32(k_s + s * kFTileBytes);
        const uint32_t d = tmem_base + static_cast<uint32_t>(a * N);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_e4m3(d, smem_desc_k128_sw128(k_addr + kk * 32), smem_desc_k128_sw128(q_addr + kk * 32), idesc,
                   kk > 0 ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&acc_full[a]);
        if (wk.tile == wk.ntile - 1 || k == nunits - 1) mma_commit(&q_empty[qseq & 1]);
        mma_issued = true;
      }
      if (mma_issued) mma_commit(drain_bar);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;                  // TMEM lanes this warp may read
    const int tphase = (ew >> 2) % TSPLIT;      // this warp takes units k ≡ tphase (mod TSPLIT)
    const int tok_lo = ((ew >> 2) / TSPLIT) * C::kTokPerWarp;
    const int kl = quad * 32 + lane;            // key within the tile
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    // W_REGS: this warp's 64 head weights (one row) in registers, packed in
    // pairs for the f32x2 FMA, reloaded per row block; otherwise they are read
    // from shared memory (broadcast 16-byte loads) to stay within the registers
    static_assert(C::kTokPerWarp == 1, "one query row per epilogue warp");
    unsigned long long wp[W_REGS ? 32 : 1];
    if (nunits > 0) {
      Walker wk;
      wk.start(prefix, p.items, u0);
      Block<NT> blk;
      int cur = -1, qseq = -1;
      for (int k = 0; k < nunits; ++k, wk.next(prefix, p.items)) {
        if (wk.item != cur) {
          cur = wk.item;
          ++qseq;
          blk.set(p, cur);
          // the weights landed with the heads: wait for them here too
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&q_full[qseq & 1], (qseq >> 1) & 1, budget, abort_flag, p.err) ? 1 : 0;
          if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
          if constexpr (W_REGS) {
            const float* wr = w_s + (qseq & 1) * N + tok_lo * 64;
#pragma unroll
            for (int i = 0; i < 32; ++i) wp[i] = pack2(wr[2 * i], wr[2 * i + 1]);
          }
        }
        const bool last_of_block = wk.tile == wk.ntile - 1 || k == nunits - 1;
        if (k % TSPLIT == tphase) {
          const int a = k % NUM_ACC;
          const int c = k % kFScaleSlots;
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&acc_full[a], (k / NUM_ACC) & 1, budget, abort_flag, p.err) ? 1 : 0;
          if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
          if (tr && k == 0 && ew == 0 && lane == 0) tr[2] = globaltimer_ns();
          tc_fence_after();
          // landed with the keys (same barrier); an e8m0 byte is the exponent field of its value
          const float ks = p.scale_u8 ? __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint8_t*>(
                                            scale_s + c * kFKeys)[kl]) << 23)
                                      : scale_s[c * kFKeys + kl];
          const int key = wk.tile * kFKeys + kl;
          const float* wrow = w_s + (qseq & 1) * N;
          uint32_t r[64];
          load_logits(lane_base + static_cast<uint32_t>(a * N + tok_lo * 64), r);
          float sc;
          if constexpr (W_REGS) sc = relu_head_sum(r, wp, ks);
          else sc = relu_head_sum(r, wrow + tok_lo * 64, ks);
          const int row = blk.row0 + tok_lo;
          if (row < p.n && key < p.ld)
            p.scores[(static_cast<int64_t>(blk.b) * p.n + row) * p.ld + key] = key < blk.vis(p, row) ? sc : -INFINITY;
          // the accumulator and the scale slot go back after the arithmetic
          // (handing them back right after the TMEM load measured slower)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&acc_empty[a]);
            mbar_arrive(&sc_empty[c]);
          }
        }
        if (last_of_block) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&q_empty[qseq & 1]);
        }
      }
    }
  }

  if (tr && warp == 2 && lane == 0) tr[3] = globaltimer_ns();
  // ------------------------------------------------------------ teardown
  if (warp == 0 && lane == 0) {
    // wait for copies still in flight (bounded) before the CTA's shared memory is released
    int dummy = 0;
    for (int q = max(0, q_issued - 2); q < q_issued; ++q) mbar_wait(&q_full[q & 1], (q >> 1) & 1, budget, &dummy, p.err);
    for (int t = max(0, tma_issued - STAGES); t < tma_issued; ++t)
      mbar_wait(&full[t % STAGES], (t / STAGES) & 1, budget, &dummy, p.err);
  }
  if (warp == 1 && lane == 0 && mma_issued) {
    int dummy = 0;
    mbar_wait(drain_bar, 0, budget, &dummy, p.err);   // all issued MMAs finished
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
  if (tr && tid == 0) {
    unsigned int smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    tr[5] = globaltimer_ns();
    tr[7] = smid;
  }
}

template <int NT, int STAGES, int NUM_ACC, int EPI_WARPS, int TSPLIT, bool W_REGS>
int launch_flat_t(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale_cache,
                  int scale_fmt, const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal,
                  float* scores, int64_t ld, cudaStream_t stream) {
  using C = FCfg<NT, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>;
  const int ntb = (n + NT - 1) / NT;
  const int64_t items = static_cast<int64_t>(B) * ntb;
  if (items > kFlatMaxItems) return IDX_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(w) & 15) return IDX_ERR_ALIGN;
  const int smem = C::smem_bytes(static_cast<int>(items));
  if (smem > max_dynamic_smem()) return IDX_ERR_SHAPE;
  CUtensorMap tk, tq, ts;
  if (!make_tmap_u8_3d(&tk, k_cache, IDX_DIM, static_cast<uint64_t>(T_cap), static_cast<uint64_t>(B), kFKeys))
    return IDX_ERR_ALIGN;
  if (!make_tmap_u8_3d(&tq, q_fp8, IDX_DIM, static_cast<uint64_t>(n) * IDX_HEADS, static_cast<uint64_t>(B), C::N))
    return IDX_ERR_ALIGN;
  if (!make_tmap_scales(&ts, k_scale_cache, scale_fmt, static_cast<uint64_t>(T_cap), static_cast<uint64_t>(B), kFKeys))
    return IDX_ERR_ALIGN;
  auto kern = flat_score_kernel<NT, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>;
  if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem)) return r;
  FlatParams p;
  p.w = w;
  p.lengths = lengths;
  p.scores = scores;
  p.ld = ld;
  p.B = B;
  p.n = n;
  p.max_len = max_len;
  p.causal = causal;
  p.ntb = ntb;
  p.items = static_cast<int>(items);
  const DebugState dbg = debug_state();
  p.debug_flags = dbg.flags;
  p.budget_ns = dbg.budget_ns;
  p.err = device_error_word();
  p.trace = (dbg.flags & 2u) ? trace_buffer() : nullptr;
  p.scale_u8 = scale_fmt == kScaleE8M0 ? 1 : 0;
  if (!p.err) return check_launch();
  kern<<<static_cast<unsigned>(num_sms()), C::kThreads, static_cast<size_t>(smem), stream>>>(tk, tq, ts, p);
  return check_launch();
}

}  // namespace

// Scores of every visible (row, key) of the call into `scores` [B, n, ld]
// (columns past each row block's last key tile left as they were).
int launch_flat_score(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale_cache,
                      int scale_fmt, const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal,
                      float* scores, int64_t ld, cudaStream_t stream) {
  if (n <= 2)
    return launch_flat_t<1, 6, 4, 8, 2, true>(q_fp8, w, k_cache, k_scale_cache, scale_fmt, lengths, B, n, T_cap,
                                              max_len, causal, scores, ld, stream);
  return launch_flat_t<4, 4, 2, 16, 1, false>(q_fp8, w, k_cache, k_scale_cache, scale_fmt, lengths, B, n, T_cap,
                                              max_len, causal, scores, ld, stream);
}

}  // namespace idx
