// Index scores and fused top-k ("Index scores" page: score equation S^I and
// the fp8_index docstring; causal mask and top-k from the Indexer.forward
// excerpt).
//
// Work item = (sequence b, block of NT query rows), served by a cluster of G
// CTAs that split the visible keys into contiguous slices.  Per CTA:
//   warp 0      TMA producer: the NT·64 query heads once, then 128-key tiles of
//               the FP8 cache (16 KB each, 128-byte swizzle) into a STAGES ring;
//   warp 1      owns TMEM and issues tcgen05.mma kind::f8f6f4 with the keys on
//               M (128 lanes) and the query heads on N (NT·64 columns), K = 128
//               as four K = 32 steps, fp32 accumulators in NUM_ACC TMEM buffers;
//   warps 2 …   epilogue: thread ↔ key (TMEM lane), reads its NT·64 logits,
//               S = k_scale · Σ_h w_h · max(L_h, 0) in fp32 registers, masks
//               keys past each row's visible count, and writes the score either
//               to global memory (idx_score) or, as an order-preserving key,
//               to shared memory for the cluster-wide select (idx_score_topk).
// Every wait is bounded (2 s by default); a CTA that gives up raises
// IDX_DEV_ERR_TIMEOUT, drains its outstanding copies and MMAs, frees TMEM and
// returns, and the cluster agrees on skipping the select so that no CTA is
// left at a cluster barrier.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>
#include <map>
#include <mutex>

#include "api_internal.h"
#include "epilogue.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace idx {

// Phase timestamps per CTA (globaltimer, ns), written only when the trace flag
// (bit 1 of the debug flags) is set; read back with idx_debug_trace().
constexpr int kTraceCtas = 8192;
constexpr int kTraceSlots = 16;
__device__ unsigned long long g_trace[kTraceCtas * kTraceSlots];

namespace {

constexpr int kTileKeys = 128;
constexpr int kTileBytes = kTileKeys * IDX_DIM;  // 16 KB

struct ScoreParams {
  const float* w;            // [B, n, 64]
  const void* k_scale;       // [B, T_cap] fp32 or e8m0 bytes (read through the tensor map)
  const int32_t* lengths;    // [B]
  void* scores;              // [B, n, ld] fp32 or bf16 (unfused)
  int32_t* indices;          // [B, n, k] (fused)
  int64_t ld;
  int B, n, T_cap, max_len, causal, k;
  int G;                     // cluster size
  int ntb;                   // query-row blocks per sequence
  int chunk_cap;             // keys per CTA the shared score buffer holds
  unsigned int debug_flags;
  unsigned long long budget_ns;
  unsigned int* err;         // device error word
  int scale_u8;              // key scales stored as e8m0 bytes (else fp32)
  int out_bf16;              // unfused: bf16 scores (else fp32)
  float mask_value;          // unfused: value of masked columns
  int w_bulk;                // w 16-byte aligned: the row block's weights arrive with its queries
};

template <int NT, bool FUSED, int STAGES, int NUM_ACC, int EPI_WARPS, int TSPLIT, bool W_REGS>
struct Cfg {
  static constexpr int N = NT * IDX_HEADS;
  static constexpr int kThreads = (2 + EPI_WARPS) * 32;
  static constexpr int kAccCols = NUM_ACC * N;
  static constexpr int kTmemCols = kAccCols <= 32 ? 32 : kAccCols <= 64 ? 64 : kAccCols <= 128 ? 128
                                 : kAccCols <= 256 ? 256 : 512;
  static_assert(kAccCols <= 512, "TMEM holds 512 columns");
  // epilogue warps: 4 TMEM lane quadrants × token groups × tile phases (TSPLIT)
  static constexpr int kTokGroups = EPI_WARPS / 4 / TSPLIT;
  static_assert(EPI_WARPS % (4 * TSPLIT) == 0 && NT % kTokGroups == 0, "epilogue split");
  static constexpr int kTokPerWarp = NT / kTokGroups;
  static constexpr int kWarpsPerTile = EPI_WARPS / TSPLIT;   // warps that consume one tile
  static constexpr int kQBytes = N * IDX_DIM;
  static constexpr int kCand = NT == 1 ? 4096 : 1024;     // scratch ints of the select
  // one row per CTA: 16-bit entries of the scratch that hold the production-time list
  static constexpr int kList = (FUSED && NT == 1) ? 6144 : 0;
  // key scales sit in their own ring, freed by the epilogue, so that a key stage
  // is freed as soon as the MMA has read it: producer ≤ STAGES tiles ahead of the
  // MMA, the MMA ≤ NUM_ACC ahead of the epilogue
  static constexpr int kScaleSlots = 2 * STAGES;
  // one commit per tile: when the stages are a multiple of the accumulators, the
  // epilogue waits on the commit that frees the tile's key stage (it tracks the
  // same MMAs).  Its phase cannot run ahead of the epilogue: tile t + STAGES,
  // the next to complete it, writes tile t's accumulator, which the epilogue
  // releases only after reading it.  Measured on the B = 128 decode: 68.7 → 66.1 µs.
  static constexpr bool kOneCommit = STAGES % NUM_ACC == 0;
  static_assert(kScaleSlots >= STAGES + NUM_ACC, "scale ring");
  // unfused one-row CTAs are small work items: two share an SM (register budget
  // 65536 / (2 × threads)), so one CTA's set-up and drain overlap the other's stream
  static constexpr int kMinCtas = (!FUSED && NT == 1) ? 2 : 1;
  // shared memory carve (offsets from a 1024-aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffScale = kOffK + STAGES * kTileBytes;
  static constexpr int kOffW = kOffScale + kScaleSlots * kTileKeys * 4;
  static constexpr int kOffBar = kOffW + N * 4;
  static constexpr int kNumBars = 2 * STAGES + kScaleSlots + 2 * NUM_ACC + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffSel = (kOffMisc + 64 + 127) / 128 * 128;
  static constexpr int kOffHist1 = kOffSel + (FUSED ? static_cast<int>(sizeof(SelectSmem)) : 0);
  static constexpr int kOffCand = kOffHist1 + (FUSED ? NT * kHistBins * 4 : 0);
  static constexpr int kOffScores = kOffCand + (FUSED ? kCand * 4 : 0);
  static int smem_bytes(int chunk_cap) {
    return 1024 + kOffScores + (FUSED ? NT * chunk_cap * 4 : 0);
  }
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// CL: a fused call whose rows are split over a cluster (G > 1).  Fused calls
// with one CTA per row use the CL = false instance, which carries only the
// one-CTA selection: a smaller kernel, whose selection code stays in the
// instruction cache from one launch to the next.
template <int NT, bool FUSED, int STAGES, int NUM_ACC, int EPI_WARPS, int TSPLIT, bool W_REGS, bool CL>
__global__ void __launch_bounds__(Cfg<NT, FUSED, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>::kThreads,
                                  Cfg<NT, FUSED, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>::kMinCtas)
    score_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                 const __grid_constant__ CUtensorMap tmap_s, const ScoreParams p) {
  using C = Cfg<NT, FUSED, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>;
  constexpr int N = C::N;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (128-byte swizzle atoms), kept as a shared-space pointer
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* q_s = smem + C::kOffQ;
  uint8_t* k_s = smem + C::kOffK;
  float* scale_s = reinterpret_cast<float*>(smem + C::kOffScale);
  float* w_s = reinterpret_cast<float*>(smem + C::kOffW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* sc_empty = bars + 2 * STAGES;   // [C::kScaleSlots]
  uint64_t* acc_full = sc_empty + C::kScaleSlots;
  uint64_t* acc_empty = acc_full + NUM_ACC;
  uint64_t* q_full = acc_empty + NUM_ACC;
  uint64_t* drain_bar = q_full + 1;
  uint64_t* never_bar = q_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  SelectSmem& sel = *reinterpret_cast<SelectSmem*>(smem + C::kOffSel);
  uint32_t* hist1 = reinterpret_cast<uint32_t*>(smem + C::kOffHist1);
  int* cand = reinterpret_cast<int*>(smem + C::kOffCand);
  uint16_t* list16 = reinterpret_cast<uint16_t*>(cand);   // first C::kList entries of the scratch
  uint32_t* sc_s = reinterpret_cast<uint32_t*>(smem + C::kOffScores);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool trace = (p.debug_flags & 2u) && blockIdx.x < kTraceCtas;
  unsigned long long* tr = g_trace + static_cast<size_t>(blockIdx.x) * kTraceSlots;
  if (trace && threadIdx.x == 0) {
    unsigned int smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    tr[0] = globaltimer_ns();
    tr[7] = smid;
  }
  // fused calls split a row over a cluster (the selection exchanges through
  // distributed shared memory); unfused calls split it over plain CTAs
  const uint32_t rank = FUSED ? (CL ? cluster_rank() : 0u) : static_cast<uint32_t>(blockIdx.x % p.G);
  const int G = (FUSED && !CL) ? 1 : p.G;
  const int item = blockIdx.x / G;
  const int b = item % p.B;
  const int tb = p.ntb - 1 - item / p.B;   // longest (latest) row blocks first
  const int row0 = tb * NT;
  int tma_issued = 0;     // producer lane (thread 0): K tiles whose loads were issued
  bool q_issued = false;  // producer lane: the query load was issued
  // Thread 0 is also the TMA producer: it starts the query and the first
  // STAGES key tiles during the set-up, so that their DRAM latency overlaps it
  // (the ring is empty, no slot needs to be waited for).
  auto issue_first = [&](int tiles, int start0) {
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_s);
    const int wrows = min(NT, p.n - row0);
    mbar_arrive_expect_tx(q_full, C::kQBytes + (p.w_bulk ? wrows * IDX_HEADS * 4 : 0));
    tma_load_3d(q_s, &tmap_q, q_full, 0, row0 * IDX_HEADS, b);
    if (p.w_bulk)
      bulk_load(w_s, p.w + (static_cast<int64_t>(b) * p.n + row0) * IDX_HEADS,
                static_cast<uint32_t>(wrows * IDX_HEADS * 4), q_full);
    q_issued = true;
    const int pre = tiles < STAGES ? tiles : STAGES;
    for (int t = 0; t < pre; ++t) {
      mbar_arrive_expect_tx(&full[t], kTileBytes + kTileKeys * (p.scale_u8 ? 1 : 4));
      tma_load_3d(k_s + t * kTileBytes, &tmap_k, &full[t], 0, start0 + t * kTileKeys, b);
      tma_load_2d(scale_s + t * kTileKeys, &tmap_s, &full[t], start0 + t * kTileKeys, b);
    }
    tma_issued = pre;
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);   // the MMA is done with the keys
    }
    for (int c = 0; c < C::kScaleSlots; ++c) mbar_init(&sc_empty[c], C::kWarpsPerTile);   // epilogue done with the scales
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], C::kWarpsPerTile);
    }
    mbar_init(q_full, 1);
    mbar_init(drain_bar, 1);
    mbar_init(never_bar, 1);
    *abort_flag = 0;
    if constexpr (FUSED) row_filter_reset(sel.cta);
    fence_barrier_init();
    // one CTA per row block: the slice starts at key 0 and the host bound
    // max_len sizes the first requests, so they leave before lengths[b] has
    // arrived; tiles past the row's keys are drained at the end like any other
    if (G == 1) issue_first(ceil_div(p.max_len, kTileKeys), 0);
  }
  const int len = p.lengths[b];
  const bool bad = len < p.n || len > p.max_len;
  if (bad && rank == 0 && threadIdx.x == 0) raise_error(p.err, IDX_DEV_ERR_LENGTH);

  // visible keys of row j of this block (0 for rows past n or a bad length)
  auto row_exists = [&](int j) { return row0 + j < p.n; };
  auto row_vis = [&](int j) {
    const int tok = row0 + j;
    return (tok < p.n && !bad) ? (p.causal ? len - p.n + tok + 1 : len) : 0;
  };
  int vis_max = 0;
#pragma unroll
  for (int j = 0; j < NT; ++j) vis_max = max(vis_max, row_vis(j));
  const int chunk = vis_max > 0 ? ceil_div(ceil_div(vis_max, G), kTileKeys) * kTileKeys : 0;
  const int start = static_cast<int>(rank) * chunk;
  const int end = min(start + chunk, vis_max);
  const int ntiles = end > start ? ceil_div(end - start, kTileKeys) : 0;
  auto tile_of = [](int t) { return t; };   // tiles are visited in order
  // a slice of a split row starts where this CTA's share does
  if (G > 1 && threadIdx.x == 0 && ntiles > 0) issue_first(ntiles, start);
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  // the weights arrive with the queries (bulk copy on q_full) when aligned;
  // otherwise, and for rows past n, they are written here
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const int j = i / IDX_HEADS;
    const int tok = row0 + j;
    if (tok >= p.n) w_s[i] = 0.f;
    else if (!p.w_bulk) w_s[i] = p.w[(static_cast<int64_t>(b) * p.n + tok) * IDX_HEADS + (i % IDX_HEADS)];
  }
  if constexpr (FUSED) {
    for (int i = threadIdx.x; i < NT * kHistBins; i += blockDim.x) hist1[i] = 0;
    if constexpr (NT == 1) select_prepare(sel.cta);   // one row: the selection state is set up here
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t budget = p.budget_ns;
  if (trace && threadIdx.x == 0) tr[1] = globaltimer_ns();
  bool mma_issued = false;  // MMA lane: at least one tcgen05.mma issued

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      int t = tma_issued;   // the first tiles went out during set-up
      for (; t < ntiles; ++t) {
        const int s = t % STAGES;
        const int c = t % C::kScaleSlots;
        if (!mbar_wait_sleep(&empty[s], ((t / STAGES) & 1) ^ 1, budget, abort_flag, p.err)) break;
        if (!mbar_wait_sleep(&sc_empty[c], ((t / C::kScaleSlots) & 1) ^ 1, budget, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&full[s], kTileBytes + kTileKeys * (p.scale_u8 ? 1 : 4));
        const int tt = tile_of(t);
        tma_load_3d(k_s + s * kTileBytes, &tmap_k, &full[s], 0, start + tt * kTileKeys, b);
        tma_load_2d(scale_s + c * kTileKeys, &tmap_s, &full[s], start + tt * kTileKeys, b);
      }
      tma_issued = t;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      if (p.debug_flags & 1u) mbar_wait(never_bar, 0, budget, abort_flag, p.err);  // fault injection: nothing arrives
      if (ntiles > 0 && mbar_wait_sleep(q_full, 0, budget, abort_flag, p.err)) {
        constexpr uint32_t idesc = idesc_e4m3_f32(128, N);
        const uint32_t q_addr = smem_u32(q_s);
        for (int t = 0; t < ntiles; ++t) {
          const int s = t % STAGES;
          const int a = t % NUM_ACC;
          if (!mbar_wait_sleep(&full[s], (t / STAGES) & 1, budget, abort_flag, p.err)) break;
          if (!mbar_wait_sleep(&acc_empty[a], ((t / NUM_ACC) & 1) ^ 1, budget, abort_flag, p.err)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(k_s + s * kTileBytes);
          const uint32_t d = tmem_base + static_cast<uint32_t>(a * N);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_e4m3(d, smem_desc_k128_sw128(k_addr + kk * 32), smem_desc_k128_sw128(q_addr + kk * 32), idesc,
                     kk > 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          if constexpr (!C::kOneCommit) mma_commit(&acc_full[a]);
          mma_issued = true;
        }
      }
      if (mma_issued) mma_commit(drain_bar);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;                  // TMEM lanes this warp may read
    const int tphase = (ew >> 2) % TSPLIT;      // this warp takes tiles t ≡ tphase (mod TSPLIT)
    const int tok_lo = ((ew >> 2) / TSPLIT) * C::kTokPerWarp;
    const int kl = quad * 32 + lane;            // key within the tile
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    // W_REGS: this warp's 64 head weights (one row) in registers, packed in
    // pairs for the f32x2 FMA; otherwise they are read from shared memory
    // (broadcast 16-byte loads) to stay within the register budget.
    static_assert(C::kTokPerWarp == 1, "one query row per epilogue warp");
    unsigned long long wp[W_REGS ? 32 : 1];
    // the weights landed with the queries: wait for them before reading w_s
    bool w_ok = true;
    if (ntiles > 0) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait_sleep(q_full, 0, budget, abort_flag, p.err) ? 1 : 0;
      w_ok = __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
    }
    if constexpr (W_REGS) {
#pragma unroll
      for (int i = 0; i < 32; ++i) wp[i] = pack2(w_s[tok_lo * 64 + 2 * i], w_s[tok_lo * 64 + 2 * i + 1]);
    }
    for (int t = tphase; w_ok && t < ntiles; t += TSPLIT) {
      const int a = t % NUM_ACC;
      const int s = t % STAGES;
      const int tt = tile_of(t);
      const int key = start + tt * kTileKeys + kl;
      const int sc_slot = t % C::kScaleSlots;
      int ok = 1;
      if (lane == 0) {
        if constexpr (C::kOneCommit)   // the stage's release commit also marks the tile's MMAs done
          ok = mbar_wait_sleep(&empty[t % STAGES], (t / STAGES) & 1, budget, abort_flag, p.err) ? 1 : 0;
        else
          ok = mbar_wait_sleep(&acc_full[a], (t / NUM_ACC) & 1, budget, abort_flag, p.err) ? 1 : 0;
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      if (trace && t == 0 && ew == 0 && lane == 0) tr[2] = globaltimer_ns();
      tc_fence_after();
      // landed with the keys (same barrier); an e8m0 byte is the exponent field of its value
      const float ks = p.scale_u8 ? __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint8_t*>(
                                        scale_s + sc_slot * kTileKeys)[kl]) << 23)
                                  : scale_s[sc_slot * kTileKeys + kl];
      const int j = tok_lo;
      uint32_t r[64];
      load_logits(lane_base + static_cast<uint32_t>(a * N + j * 64), r);
      float sc;
      if constexpr (W_REGS) sc = relu_head_sum(r, wp, ks);
      else sc = relu_head_sum(r, w_s + j * 64, ks);
      const bool visible = key < row_vis(j);
      if constexpr (FUSED) {
        const uint32_t u = order_key(sc);
        sc_s[j * p.chunk_cap + tt * kTileKeys + kl] = visible ? u : 0u;
        if (visible) {
          if constexpr (NT == 1) select_count_key(sel.cta, hist1, u);   // with the coarse sums
          else atomicAdd(&hist1[j * kHistBins + (u >> 21)], 1u);
        }
        // one row per CTA: keys that may reach the top k go to the short list
        if constexpr (C::kList > 0)
          if (G == 1) row_filter_append(sel.cta, list16, C::kList, u, visible, tt * kTileKeys + kl);
      } else {
        if (row_exists(j) && key < p.ld) {
          const int64_t at = (static_cast<int64_t>(b) * p.n + row0 + j) * p.ld + key;
          const float v = visible ? sc : p.mask_value;
          if (p.out_bf16) static_cast<__nv_bfloat16*>(p.scores)[at] = __float2bfloat16_rn(v);
          else static_cast<float*>(p.scores)[at] = v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acc_empty[a]);
        mbar_arrive(&sc_empty[sc_slot]);
      }
      // the first epilogue warp raises the list's bound after tile 4 and every 8 tiles
      if constexpr (C::kList > 0) {
        if (G == 1 && ew == 0 && (t == 4 || (t >= 8 && (t & 7) == 0))) {
          const int v0 = row_vis(0);
          const int target = row_filter_target((t + 1) * kTileKeys, v0, min(p.k, v0));
          if (target > 0) row_filter_raise(sel.cta, hist1, target);
        }
      }
    }
  }
  __syncthreads();
  if (trace && threadIdx.x == 0) tr[3] = globaltimer_ns();

  if constexpr (!FUSED) {
    // columns of this CTA's share that no tile covered: the mask value
    const int64_t col_lo = static_cast<int64_t>(start) + static_cast<int64_t>(ntiles) * kTileKeys;
    const int64_t share_hi = (static_cast<int>(rank) == G - 1) ? p.ld : (p.ld < static_cast<int64_t>(start) + chunk ? p.ld : static_cast<int64_t>(start) + chunk);
    const int64_t lo = (vis_max == 0 && static_cast<int>(rank) == G - 1) ? 0 : col_lo;
    if (share_hi > lo) {
      for (int j = 0; j < NT; ++j) {
        if (!row_exists(j)) continue;
        const int64_t row_at = (static_cast<int64_t>(b) * p.n + row0 + j) * p.ld;
        if (p.out_bf16) {
          __nv_bfloat16* row = static_cast<__nv_bfloat16*>(p.scores) + row_at;
          const __nv_bfloat16 m = __float2bfloat16_rn(p.mask_value);
          for (int64_t c = lo + threadIdx.x; c < share_hi; c += blockDim.x) row[c] = m;
          continue;
        }
        float* row = static_cast<float*>(p.scores) + row_at;
        const float m = p.mask_value;
        // scalar head up to a 16-byte boundary, 16-byte stores, scalar tail
        const int64_t head = (4 - ((reinterpret_cast<uintptr_t>(row + lo) >> 2) & 3)) & 3;
        const int64_t body_lo = lo + (head < share_hi - lo ? head : share_hi - lo);
        const int64_t nvec = (share_hi - body_lo) >> 2;
        for (int64_t c = lo + threadIdx.x; c < body_lo; c += blockDim.x) row[c] = m;
        float4* rv = reinterpret_cast<float4*>(row + body_lo);
        const float4 m4 = make_float4(m, m, m, m);
        for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) rv[v] = m4;
        for (int64_t c = body_lo + 4 * nvec + threadIdx.x; c < share_hi; c += blockDim.x) row[c] = m;
      }
    }
  } else {
    // Whether some CTA of the cluster gave up is learnt inside the selection
    // (its first exchange); rows where every visible position is selected need
    // no scores and are written regardless.
#pragma unroll 1
    for (int j = 0; j < NT; ++j) {
      if (!row_exists(j)) continue;
      if (j > 0) __syncthreads();   // the previous row's staged output has been written out
      int32_t* out = p.indices + (static_cast<int64_t>(b) * p.n + row0 + j) * p.k;
      const int v = row_vis(j);
      const int kt = min(p.k, v);
      const int nloc = max(0, min(end, v) - start);
      if (kt == v) {
        // every visible position is selected: slot s holds position s
        for (int i = threadIdx.x; i < nloc; i += blockDim.x) out[start + i] = start + i;
        if (rank == 0)
          for (int i = kt + threadIdx.x; i < p.k; i += blockDim.x) out[i] = -1;
      } else {
        if (trace && j == 0 && threadIdx.x == 0) tr[6] = globaltimer_ns();
        cluster_select_row(sel, sc_s + j * p.chunk_cap, nloc, start, kt, hist1 + j * kHistBins, cand, C::kCand,
                           C::kList, NT == 1, out, G, rank, (trace && j == 0) ? tr : nullptr,
                           const_cast<const int*>(abort_flag));
        if (rank == 0)
          for (int i = kt + threadIdx.x; i < p.k; i += blockDim.x) out[i] = -1;
      }
    }
    if (CL && G > 1) cluster_sync(); else __syncthreads();
  }

  if (trace && threadIdx.x == 0) tr[4] = globaltimer_ns();
  // ------------------------------------------------------------ teardown
  if (warp == 0 && lane == 0) {
    // wait for copies still in flight (bounded) before the CTA's shared memory is released
    int dummy = 0;
    if (q_issued) mbar_wait(q_full, 0, budget, &dummy, p.err);
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
  if (trace && threadIdx.x == 0) tr[5] = globaltimer_ns();
}

// ---------------------------------------------------------------- host side
struct Plan {
  int G;
  int chunk_cap;
  int ntb;
  int smem;
};

int pow2_floor(int x) {
  int p = 1;
  while (p * 2 <= x) p *= 2;
  return p;
}

template <int NT, bool FUSED, int STAGES, int NUM_ACC, int EPI_WARPS, int TSPLIT, bool W_REGS>
int launch_score(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale_cache,
                 const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal, void* scores,
                 int64_t ld, int k, int32_t* indices, cudaStream_t stream, int score_budget_bytes,
                 const ScoreVariant& var) {
  using C = Cfg<NT, FUSED, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS>;
  const int ntb = (n + NT - 1) / NT;
  const int64_t items = static_cast<int64_t>(B) * ntb;
  const int sms = num_sms();
  auto chunk_of = [&](int g) { return ((max_len + g - 1) / g + kTileKeys - 1) / kTileKeys * kTileKeys; };
  // TMEM has 512 columns per SM and tcgen05.alloc waits for free columns: the
  // shared-memory request keeps co-resident CTAs within 512 columns in total
  const int tmem_ctas = 512 / C::kTmemCols;
  const int per_sm = smem_per_sm();
  const int min_keys_per_cta = 512;
  int G = 1;
  if (FUSED) {
    // cluster size: enough CTAs to cover the GPU once, and a score slice that fits
    if (items < sms) G = pow2_floor(static_cast<int>(sms / items));
    G = G > 8 ? 8 : G;
    while (G > 1 && (max_len + G - 1) / G < min_keys_per_cta) G /= 2;
    while (G < 8 && NT * chunk_of(G) * 4 > score_budget_bytes) G *= 2;
  } else if (items < 4 * static_cast<int64_t>(sms)) {
    // rows split over plain CTAs: the split whose busiest SM streams the fewest
    // keys (CTAs spread evenly over the SMs), with a fixed cost per CTA
    int64_t best = -1;
    for (int g = 1; g <= 16; g *= 2) {
      if (g > 1 && (max_len + g - 1) / g < min_keys_per_cta) break;
      const int64_t ctas = items * g;
      const int64_t per_sm_ctas = (ctas + sms - 1) / sms;
      const int64_t cost = per_sm_ctas * (chunk_of(g) + 128);
      if (best < 0 || cost < best) {
        best = cost;
        G = g;
      }
    }
  }
  const int chunk_cap = chunk_of(G);
  int smem = C::smem_bytes(FUSED ? chunk_cap : 0);
  while (per_sm / (smem + 1024) > tmem_ctas) smem += 1024;
  if (smem > max_dynamic_smem()) return IDX_ERR_SHAPE;
  if (items * G > 0x7FFFFFFF) return IDX_ERR_SHAPE;

  CUtensorMap tk, tq, ts;
  if (!make_tmap_u8_3d(&tk, k_cache, IDX_DIM, static_cast<uint64_t>(T_cap), static_cast<uint64_t>(B), kTileKeys))
    return IDX_ERR_ALIGN;
  if (!make_tmap_u8_3d(&tq, q_fp8, IDX_DIM, static_cast<uint64_t>(n) * IDX_HEADS, static_cast<uint64_t>(B), C::N))
    return IDX_ERR_ALIGN;
  if (!make_tmap_scales(&ts, k_scale_cache, var.scale_fmt, static_cast<uint64_t>(T_cap), static_cast<uint64_t>(B),
                        kTileKeys))
    return IDX_ERR_ALIGN;

  auto kern = score_kernel<NT, FUSED, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS, false>;
  if constexpr (FUSED)
    if (G > 1) kern = score_kernel<NT, FUSED, STAGES, NUM_ACC, EPI_WARPS, TSPLIT, W_REGS, true>;
  if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem)) return r;
  ScoreParams p;
  p.w = w;
  p.k_scale = k_scale_cache;
  p.lengths = lengths;
  p.scores = scores;
  p.indices = indices;
  p.ld = ld;
  p.B = B;
  p.n = n;
  p.T_cap = T_cap;
  p.max_len = max_len;
  p.causal = causal;
  p.k = k;
  p.G = G;
  p.ntb = ntb;
  p.chunk_cap = chunk_cap;
  p.scale_u8 = var.scale_fmt == kScaleE8M0 ? 1 : 0;
  p.out_bf16 = var.out_bf16;
  p.mask_value = var.mask_value;
  p.w_bulk = (reinterpret_cast<uintptr_t>(w) & 15) == 0 ? 1 : 0;
  const DebugState dbg = debug_state();
  p.debug_flags = dbg.flags;
  p.budget_ns = dbg.budget_ns;
  p.err = device_error_word();
  if (!p.err) return check_launch();

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(items * G), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(FUSED ? G : 1);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tk, tq, ts, p) != cudaSuccess) return check_launch();
  return check_launch();
}

int check_score_args(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale_cache,
                     const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal,
                     int scale_fmt = kScaleF32) {
  if (scale_fmt != kScaleF32 && scale_fmt != kScaleE8M0) return IDX_ERR_FMT;
  if (B < 0 || n < 0 || T_cap <= 0) return IDX_ERR_SHAPE;
  if (B == 0 || n == 0) return IDX_OK;
  if (!q_fp8 || !w || !k_cache || !k_scale_cache || !lengths) return IDX_ERR_NULL;
  if (max_len < n || max_len > T_cap || max_len > IDX_MAX_LEN) return IDX_ERR_SHAPE;
  if (causal != 0 && causal != 1) return IDX_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(q_fp8) | reinterpret_cast<uintptr_t>(k_cache) |
       reinterpret_cast<uintptr_t>(k_scale_cache)) & 15)
    return IDX_ERR_ALIGN;
  // the scale rows are read by TMA: 16-byte pitch
  if (T_cap % (scale_fmt == kScaleE8M0 ? 16 : 4) != 0) return IDX_ERR_SHAPE;
  if (static_cast<int64_t>(n) * IDX_HEADS > 0x7FFFFFFF) return IDX_ERR_SHAPE;
  return 1;  // proceed
}

// decode-shaped calls (one or a few rows per sequence) use one row per CTA;
// prefill-shaped calls four rows (N = 256).
constexpr int kDecodeRowsMax = 2;

}  // namespace

}  // namespace idx

using namespace idx;

extern "C" int idx_score_ex(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale,
                            int scale_fmt, const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal,
                            void* scores, int64_t ld, int score_dtype, float mask_value, idx_stream_t stream) {
  const int c = check_score_args(q_fp8, w, k_cache, k_scale, lengths, B, n, T_cap, max_len, causal, scale_fmt);
  if (c <= 0) return c;
  if (!scores) return IDX_ERR_NULL;
  if (ld <= 0) return IDX_ERR_SHAPE;
  if (score_dtype != IDX_SCORE_F32 && score_dtype != IDX_SCORE_BF16) return IDX_ERR_FMT;
  if (mask_value != mask_value) return IDX_ERR_SHAPE;   // NaN
  const ScoreVariant var{scale_fmt, score_dtype == IDX_SCORE_BF16 ? 1 : 0, mask_value};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (n <= kDecodeRowsMax)
    return launch_score<1, false, 4, 4, 8, 2, false>(q_fp8, w, k_cache, k_scale, lengths, B, n, T_cap, max_len,
                                                     causal, scores, ld, 0, nullptr, s, 0, var);
  return launch_score<4, false, 4, 2, 16, 1, false>(q_fp8, w, k_cache, k_scale, lengths, B, n, T_cap, max_len, causal,
                                                    scores, ld, 0, nullptr, s, 0, var);
}

extern "C" int idx_score(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const float* k_scale_cache,
                         const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal, float* scores,
                         int64_t ld, idx_stream_t stream) {
  return idx_score_ex(q_fp8, w, k_cache, k_scale_cache, IDX_SCALE_F32, lengths, B, n, T_cap, max_len, causal, scores,
                      ld, IDX_SCORE_F32, -INFINITY, stream);
}

namespace {
// idx_score_visible with either key-scale storage
int score_visible(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale, int scale_fmt,
                  const int32_t* lengths, int B, int n, int T_cap, int max_len, int causal, float* scores, int64_t ld,
                  idx_stream_t stream) {
  const int c = check_score_args(q_fp8, w, k_cache, k_scale, lengths, B, n, T_cap, max_len, causal, scale_fmt);
  if (c <= 0) return c;
  if (!scores) return IDX_ERR_NULL;
  if (ld < max_len) return IDX_ERR_SHAPE;
  // flat partition over every SM when the call fits its index, else per row block
  const int r = launch_flat_score(q_fp8, w, k_cache, k_scale, scale_fmt, lengths, B, n, T_cap, max_len, causal,
                                  scores, ld, reinterpret_cast<cudaStream_t>(stream));
  if (r != IDX_ERR_UNSUPPORTED) return r;
  return idx_score_ex(q_fp8, w, k_cache, k_scale, scale_fmt, lengths, B, n, T_cap, max_len, causal, scores, ld,
                      IDX_SCORE_F32, -INFINITY, stream);
}
}  // namespace

extern "C" int idx_score_visible(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache,
                                 const float* k_scale_cache, const int32_t* lengths, int B, int n, int T_cap,
                                 int max_len, int causal, float* scores, int64_t ld, idx_stream_t stream) {
  return score_visible(q_fp8, w, k_cache, k_scale_cache, IDX_SCALE_F32, lengths, B, n, T_cap, max_len, causal, scores,
                       ld, stream);
}

extern "C" int idx_score_topk_ex(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache, const void* k_scale,
                                 int scale_fmt, const int32_t* lengths, int B, int n, int T_cap, int max_len,
                                 int causal, int k, int32_t* indices, void* ws, size_t ws_bytes,
                                 idx_stream_t stream) {
  const int c = check_score_args(q_fp8, w, k_cache, k_scale, lengths, B, n, T_cap, max_len, causal, scale_fmt);
  if (c <= 0) return c;
  if (k <= 0) return IDX_ERR_K;
  if (!indices) return IDX_ERR_NULL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const ScoreVariant var{scale_fmt, 0, -INFINITY};
  // Prefill-shaped calls with a workspace: scores of all rows to the workspace
  // (the flat-partition scorer at full tensor throughput), then the top-k
  // kernel with several rows per SM in flight.  A row's selection then overlaps
  // other rows' work instead of stalling its CTA's MMA pipeline.
  const size_t need = idx_workspace_size(B, n, max_len, k);
  if (ws && ws_bytes >= need && need > 0) {
    if (reinterpret_cast<uintptr_t>(ws) & 15) return IDX_ERR_ALIGN;
    float* scores = static_cast<float*>(ws);
    const int r = score_visible(q_fp8, w, k_cache, k_scale, scale_fmt, lengths, B, n, T_cap, max_len, causal,
                                scores, max_len, stream);
    if (r != IDX_OK) return r;
    return idx_topk(scores, lengths, B, n, max_len, max_len, causal, k, indices, nullptr, 0, stream);
  }
  // decode: four key stages (six, with a smaller selection scratch to fit,
  // measured 72.4 against 68.4 µs on the B = 128 decode)
  if (n <= kDecodeRowsMax)
    return launch_score<1, true, 4, 4, 8, 2, true>(q_fp8, w, k_cache, k_scale, lengths, B, n, T_cap, max_len, causal,
                                                   nullptr, 0, k, indices, s, 64 * 1024, var);
  return launch_score<4, true, 3, 2, 16, 1, false>(q_fp8, w, k_cache, k_scale, lengths, B, n, T_cap, max_len, causal,
                                                   nullptr, 0, k, indices, s, 64 * 1024, var);
}

extern "C" int idx_score_topk(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache,
                              const float* k_scale_cache, const int32_t* lengths, int B, int n, int T_cap,
                              int max_len, int causal, int k, int32_t* indices, void* ws, size_t ws_bytes,
                              idx_stream_t stream) {
  return idx_score_topk_ex(q_fp8, w, k_cache, k_scale_cache, IDX_SCALE_F32, lengths, B, n, T_cap, max_len, causal, k,
                           indices, ws, ws_bytes, stream);
}

extern "C" int idx_debug_trace(unsigned long long* host_out, int max_ctas) {
  if (!host_out || max_ctas <= 0) return IDX_ERR_NULL;
  const int n = max_ctas < kTraceCtas ? max_ctas : kTraceCtas;
  if (cudaMemcpyFromSymbol(host_out, g_trace, sizeof(unsigned long long) * kTraceSlots * n) != cudaSuccess)
    return check_launch();
  return IDX_OK;
}

namespace idx {
unsigned long long* trace_buffer() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_trace) != cudaSuccess) return nullptr;
  return static_cast<unsigned long long*>(ptr);
}
}  // namespace idx

// ---------------------------------------------------------------------------
// Allocation-free variant of the prefill-shaped score + top-k.
//
// Some callers cannot allocate device memory at the moment they call in — for
// example code that enqueues work while its stream is being captured into a
// CUDA graph, or an inference-engine plugin whose enqueue step is not allowed
// to allocate.  They cannot provide the score workspace idx_score_topk uses
// for prefill-shaped calls, so this entry point keeps that workspace in a
// fixed buffer owned by the library.
namespace idx {
namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;   // 64 MiB: B·n·max_len ≤ 16 Mi scores
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];

// Device address of g_static_scratch on the current device (host code cannot
// use the symbol itself: on the host it only names a stand-in), looked up once
// per device.  nullptr when the lookup fails (its CUDA error is recorded).
float* static_scratch() {
  static std::mutex mu;
  static std::map<int, float*> addr;   // device ordinal → address
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    check_launch();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  float*& a = addr[dev];
  if (!a) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) {
      check_launch();
      return nullptr;
    }
    a = static_cast<float*>(ptr);
  }
  return a;
}

}  // namespace
}  // namespace idx

extern "C" int idx_score_topk_noalloc(const uint8_t* q_fp8, const float* w, const uint8_t* k_cache,
                                      const float* k_scale_cache, const int32_t* lengths, int B, int n, int T_cap,
                                      int max_len, int causal, int k, int32_t* indices, idx_stream_t stream) {
  const int c = check_score_args(q_fp8, w, k_cache, k_scale_cache, lengths, B, n, T_cap, max_len, causal);
  if (c <= 0) return c;
  if (k <= 0) return IDX_ERR_K;
  if (!indices) return IDX_ERR_NULL;
  const size_t need = idx_workspace_size(B, n, max_len, k);
  if (need > kStaticScratchBytes) return IDX_ERR_SCRATCH;
  // the buffer's address is looked up on the first call on a device, whatever
  // the call's shape, so that a decode-shaped first call also does the lookup
  float* scratch = static_scratch();
  if (!scratch) return IDX_ERR_LAUNCH;
  if (need == 0)   // decode-shaped: the single kernel needs no scratch
    return idx_score_topk(q_fp8, w, k_cache, k_scale_cache, lengths, B, n, T_cap, max_len, causal, k, indices,
                          nullptr, 0, stream);
  return idx_score_topk(q_fp8, w, k_cache, k_scale_cache, lengths, B, n, T_cap, max_len, causal, k, indices,
                        scratch, kStaticScratchBytes, stream);
}
