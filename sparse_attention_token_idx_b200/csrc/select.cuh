// Cluster-wide top-k selection over scores held in shared memory.
//
// A row's visible scores are split over the G CTAs of a thread-block cluster,
// each holding its contiguous slice as order-preserving uint32 keys.  The
// k_t-th largest key is found by radix refinement on 11 + 11 + 10 bits:
//   level 1  the histogram of the top 11 bits was built while the scores were
//            produced; the G histograms are summed through distributed shared
//            memory and every CTA finds the same threshold bin b1;
//   pass A   keys above b1 are selected; keys in b1 are counted by their next
//            11 bits and their slice positions kept in a candidate list;
//   level 2  summed histogram → b2;  pass B over the candidates → level 3 → b3;
//   pass C   candidates above the 32-bit threshold are selected, equal ones
//            fill the remaining slots.
// Whenever the threshold bin holds exactly the slots still open, all of it is
// taken and the refinement stops.  Every pass first counts per thread, then a
// block scan and a cluster-wide prefix of the per-CTA totals give each thread
// its output offsets, then it writes — no atomics with a return value in the
// sweeps.  Selected positions are staged in CTA 0's shared memory (through
// distributed shared memory) and written to global memory once per row with
// coalesced stores, so that no cluster barrier waits on scattered global
// writes; a one-CTA "cluster" uses block barriers only.  Control flow (and so
// every cluster barrier) depends only on the
// summed histograms, identical in all CTAs.  The output order is unspecified
// (a set), as the NKI indexer page states for its top-k output.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace idx {

constexpr int kHistBins = 2048;
constexpr int kStage = 2048;     // staged output slots per row (larger k writes straight to global)

// Barrier and shared-memory access for a real cluster (CL) or a single CTA.
template <bool CL>
struct Grp {
  static __device__ __forceinline__ void sync() {
    if constexpr (CL) cluster_sync(); else __syncthreads();
  }
  static __device__ __forceinline__ uint32_t ld(const uint32_t* p, uint32_t r) {
    if constexpr (CL) return dsmem_ld_u32(dsmem_addr(p, r)); else return *p;
  }
};

// State of the one-CTA selection (cta_select_row) and of the row filter.
struct alignas(16) CtaSelSmem {
  uint32_t hist[kHistBins];      // level-2 histogram
  uint32_t hist3[kHistBins / 2]; // level-3 histogram (own buffer: one barrier per exchange)
  uint32_t coarse[3][64];        // coarse sums (32 fine bins per entry) of levels 1-3
  uint32_t ctr_gc;               // output slots taken (low 16 bits) | bin-b1 keys listed (high)
  uint32_t ctr_tie;              // above the 32-bit threshold (low) | ties seen (high)
  uint32_t filt_lo;              // row filter: keys below this bound are not listed
  int list_cnt;                  // row filter: list entries taken
};

struct alignas(16) SelectSmem {
  CtaSelSmem cta;                // one-CTA path; its hist / hist3 are also the cluster path's
  uint32_t hsum[kHistBins];      // cluster-summed histogram
  int warp_a[32];
  int warp_b[32];
  int bin;
  int above;
  int cta_cnt[2][2];             // this CTA's pass totals, double-buffered by exchange parity
  int cta_base[2];               // cluster prefix of those totals for this CTA
  int any_abort;
  int pad[3];
  int32_t out_s[kStage];         // staged positions of the current row (CTA 0's copy is the one used)
};

// Block-wide exclusive scan of two counters.  Returns the thread's offsets; the
// block totals land in *tot_a / *tot_b (same value in every thread).
static __device__ __noinline__ void block_scan2(SelectSmem& sm, int a, int b, int& ea, int& eb, int& tot_a,
                                         int& tot_b) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xFFFFFFFFu, ia, o);
    const int vb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
    if (lane >= o) {
      ia += va;
      ib += vb;
    }
  }
  if (lane == 31) {
    sm.warp_a[warp] = ia;
    sm.warp_b[warp] = ib;
  }
  __syncthreads();
  int wa = 0, wb = 0, ta = 0, tb = 0;
  for (int w = 0; w < nw; ++w) {
    const int xa = sm.warp_a[w], xb = sm.warp_b[w];
    if (w < warp) {
      wa += xa;
      wb += xb;
    }
    ta += xa;
    tb += xb;
  }
  ea = wa + ia - a;
  eb = wb + ib - b;
  tot_a = ta;
  tot_b = tb;
  __syncthreads();   // warp_a / warp_b may be reused right away
}

// Block-wide: bins in descending order of value; find the bin that holds the
// rem-th largest element.  Result in sm.bin, and sm.above = count in higher bins.
static __device__ __noinline__ void find_bin(SelectSmem& sm, const uint32_t* hist, int nb, int rem) {
  const int nthr = blockDim.x;
  const int tid = threadIdx.x;
  const int per = (nb + nthr - 1) / nthr;
  const int hi = nb - tid * per;            // thread tid covers bins [lo, hi), highest bins first
  const int lo = hi - per;
  int csum = 0;
  for (int bn = (lo > 0 ? lo : 0); bn < hi; ++bn) csum += static_cast<int>(hist[bn]);
  if (tid == 0) {   // safe defaults should no bin hold the rem-th element (cannot happen on valid data)
    sm.bin = 0;
    sm.above = 0;
  }
  int excl, dummy, tot, tot2;
  block_scan2(sm, csum, 0, excl, dummy, tot, tot2);
  if (csum > 0 && excl < rem && rem <= excl + csum) {
    int acc = excl;
    for (int bn = hi - 1; bn >= lo && bn >= 0; --bn) {
      const int c = hist[bn];
      if (acc + c >= rem) {
        sm.bin = bn;
        sm.above = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

// Exchange over the cluster: after one barrier, sum `local` (nb bins) of all
// CTAs into sm.hsum, or (nb = 0) read the lower ranks' pass totals
// cta_cnt[parity] into sm.cta_base.  Entry: every CTA's `local` / cta_cnt are
// final.  Each exchanged buffer is written again only after a later barrier,
// which no CTA passes before finishing its reads here.
template <bool CL>
__device__ __forceinline__ void cluster_exchange(SelectSmem& sm, const uint32_t* local, int nb, int G,
                                                 uint32_t rank, int parity, const int* abort_flag = nullptr) {
  __syncthreads();
  if constexpr (CL) {
    // One shared-memory barrier: every buffer read here is written again only
    // after a later barrier, which no CTA passes before finishing these reads.
    cluster_sync_shared();
    // 16-byte loads from every rank's histogram through generic pointers, all
    // independent, so that the remote reads overlap
    const uint4* src[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) src[r] = reinterpret_cast<const uint4*>(dsmem_ptr(local, r < G ? r : 0));
    for (int i4 = threadIdx.x; i4 < nb / 4; i4 += blockDim.x) {
      uint4 acc = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r < G) {
          const uint4 v = src[r][i4];
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
      }
      reinterpret_cast<uint4*>(sm.hsum)[i4] = acc;
    }
    if (nb == 0 && threadIdx.x < 2) {
      int base = 0;
      for (int r = 0; r < static_cast<int>(rank); ++r)
        base += static_cast<int>(dsmem_ld_u32(dsmem_addr(&sm.cta_cnt[parity][threadIdx.x], r)));
      sm.cta_base[threadIdx.x] = base;
    }
    if (abort_flag && threadIdx.x == 32) {
      int any = 0;
      for (int r = 0; r < G; ++r) any |= *dsmem_ptr(abort_flag, r);
      sm.any_abort = any;
    }
    __syncthreads();
  } else {
    for (int i = threadIdx.x; i < nb; i += blockDim.x) sm.hsum[i] = local[i];
    if (threadIdx.x < 2) sm.cta_base[threadIdx.x] = 0;
    if (abort_flag && threadIdx.x == 32) sm.any_abort = *abort_flag;
    __syncthreads();
  }
}

// Output writer of one row: positions go to CTA 0's staging buffer when the row
// fits, else straight to global memory.
template <bool CL>
struct RowOut {
  int32_t* out;
  uint32_t stage_base;   // shared::cluster address of CTA 0's out_s (CL)
  int32_t* stage_local;  // local out_s (single CTA)
  bool staged;
  __device__ __forceinline__ void put(int slot, int32_t v) const {
    if constexpr (CL) {
      if (staged) dsmem_st_u32(stage_base + 4u * static_cast<uint32_t>(slot), static_cast<uint32_t>(v));
      else out[slot] = v;
    } else {
      int32_t* dst = staged ? stage_local : out;   // one pointer, one predicated store
      dst[slot] = v;
    }
  }
};

// End of a row: all staged positions are in CTA 0's buffer after the barrier
// (a full release/acquire barrier: the staging stores went to another CTA's
// shared memory); CTA 0 writes them out with coalesced stores.
template <bool CL>
__device__ __forceinline__ void flush_row(SelectSmem& sm, const RowOut<CL>& ro, int kt, uint32_t rank) {
  Grp<CL>::sync();
  if (rank == 0) {
    if (sm.any_abort)   // a CTA of the cluster gave up: its scores are not valid
      for (int i = threadIdx.x; i < kt; i += blockDim.x) ro.out[i] = -1;
    else if (ro.staged)
      for (int i = threadIdx.x; i < kt; i += blockDim.x) ro.out[i] = sm.out_s[i];
  }
}

// Exchange only the per-CTA pass totals (no histogram).
template <bool CL>
__device__ __forceinline__ void exchange_counts(SelectSmem& sm, int G, uint32_t rank, int parity) {
  if constexpr (CL) {
    cluster_exchange<true>(sm, nullptr, 0, G, rank, parity);
  } else {
    if (threadIdx.x < 2) sm.cta_base[threadIdx.x] = 0;
    __syncthreads();
  }
}

// Level-1 histogram → hist the selection reads: a cluster sums into hsum, a
// single CTA reads its own histogram in place.
template <bool CL>
__device__ __forceinline__ const uint32_t* summed_hist(SelectSmem& sm, const uint32_t* local, int nb, int G,
                                                       uint32_t rank, const int* abort_flag = nullptr) {
  if constexpr (CL) {
    cluster_exchange<true>(sm, local, nb, G, rank, 0, abort_flag);
    return sm.hsum;
  } else {
    if (abort_flag && threadIdx.x == 0) sm.any_abort = *abort_flag;
    __syncthreads();
    return local;
  }
}

// Select the kt best of a row whose keys are split over the cluster.
//   keys[0 … nloc)  this CTA's slice (positions start … start+nloc−1), 16-byte
//                   aligned, and holding key 0 from nloc up to the next multiple of 4
//   hist1           this CTA's histogram of keys >> 21 over the slice
//   cand[0 … cap)   scratch for candidate slice indices
//   out             the row's k output slots (global memory)
// Requires kt < visible (the caller handles "take everything").  All threads
// of all CTAs in the cluster call this with the same kt.
template <bool CL>
__device__ __forceinline__ void cluster_select_row_t(SelectSmem& sm, const uint32_t* keys, int nloc, int start,
                                                     int kt, const uint32_t* hist1, int* cand, int cap,
                                                     int32_t* out, int G, uint32_t rank,
                                                     unsigned long long* tr, const int* abort_flag) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  auto stamp = [&](int slot) {
    if (tr && tid == 0) tr[slot] = globaltimer_ns();
  };
  if (tid == 0) sm.any_abort = 0;
  RowOut<CL> ro;
  ro.out = out;
  ro.staged = kt <= kStage;
  ro.stage_local = sm.out_s;
  ro.stage_base = CL ? dsmem_addr(sm.out_s, 0) : 0u;
  for (int i = tid; i < kHistBins; i += nthr) sm.cta.hist[i] = 0;
  for (int i = tid; i < kHistBins / 2; i += nthr) sm.cta.hist3[i] = 0;

  // ---- level 1
  const uint32_t* H = summed_hist<CL>(sm, hist1, kHistBins, G, rank, abort_flag);
  if (sm.any_abort) {   // same value in every CTA of the cluster: skip the selection, flush writes -1
    flush_row<CL>(sm, ro, kt, rank);
    return;
  }
  find_bin(sm, H, kHistBins, kt);
  const uint32_t b1 = static_cast<uint32_t>(sm.bin);
  int rem = kt - sm.above;
  const bool done1 = static_cast<int>(H[b1]) == rem;
  stamp(8);

  // ---- pass A: count.  4 keys per 16-byte load, keys compared against bin
  // edges (no shifts), no bounds test per key: the slice is padded with key 0
  // up to a multiple of 4, and 0 lies below every bin a visible score can fall
  // in (a finite score maps to a key ≥ 0x007FFFFF, i.e. bin ≥ 3).
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  const int nvec = (nloc + 3) >> 2;
  const uint32_t lo1 = b1 << 21;              // first key of bin b1
  const uint32_t hi1 = lo1 | 0x1FFFFFu;       // last key of bin b1
  // done1: everything from bin b1 up is selected; otherwise keys above bin b1
  // are selected and keys inside it become candidates
  const uint32_t sel_above = done1 ? lo1 - 1u : hi1;
  int cg = 0, ce = 0;
  for (int v = tid; v < nvec; v += nthr) {
    const uint4 q = kv[v];
    cg += (q.x > sel_above) + (q.y > sel_above) + (q.z > sel_above) + (q.w > sel_above);
    ce += (q.x >= lo1) + (q.y >= lo1) + (q.z >= lo1) + (q.w >= lo1);
  }
  ce = done1 ? 0 : ce - cg;                   // keys inside bin b1
  int og, oe, tg, te;
  block_scan2(sm, cg, ce, og, oe, tg, te);
  if (tid == 0) sm.cta_cnt[0][0] = tg;
  exchange_counts<CL>(sm, G, rank, 0);
  const bool overflow = te > cap;
  stamp(10);
  if (tr && tid == 0) tr[15] = static_cast<unsigned long long>(te);
  // ---- pass A: write
  {
    int wg = sm.cta_base[0] + og, we = oe;
    const bool keep = !overflow && !done1;
    for (int v = tid; v < nvec; v += nthr) {
      const uint4 q = kv[v];
      const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * v + e;
        const bool g = kk[e] > sel_above;
        const bool c = keep && !g && kk[e] >= lo1;
        if (g) ro.put(wg, start + i);
        if (c) cand[we] = i;
        wg += g ? 1 : 0;
        we += c ? 1 : 0;
      }
    }
  }
  if (done1) {
    flush_row<CL>(sm, ro, kt, rank);
    return;
  }
  int out_base = kt - rem;                   // slots holding everything above b1, cluster-wide
  const int nscan = overflow ? nloc : te;
  __syncthreads();
  // ---- level-2 histogram over the candidates (or the whole slice on overflow)
  if (!overflow) {
    for (int c = tid; c < te; c += nthr) atomicAdd(&sm.cta.hist[(keys[cand[c]] >> 10) & 0x7FF], 1u);
  } else {
    for (int i = tid; i < nloc; i += nthr) {
      const uint32_t key = keys[i];
      if ((key >> 21) == b1) atomicAdd(&sm.cta.hist[(key >> 10) & 0x7FF], 1u);
    }
  }
  stamp(11);
  // ---- level 2
  const uint32_t* H2 = summed_hist<CL>(sm, sm.cta.hist, kHistBins, G, rank);
  find_bin(sm, H2, kHistBins, rem);
  const uint32_t b2 = static_cast<uint32_t>(sm.bin);
  rem -= sm.above;
  const bool done2 = static_cast<int>(H2[b2]) == rem;
  __syncthreads();                           // everyone has read H2 (it may be sm.cta.hist)
  // ---- pass B: over the candidates
  const int trips_b = (nscan + nthr - 1) / nthr;
  cg = 0;
  for (int it = 0; it < trips_b; ++it) {
    const int j = it * nthr + tid;
    if (j < nscan) {
      const uint32_t key = keys[overflow ? j : cand[j]];
      if ((key >> 21) == b1) {
        const uint32_t mid = (key >> 10) & 0x7FF;
        const bool eq = mid == b2;
        cg += (mid > b2 || (done2 && eq)) ? 1 : 0;
        if (!done2 && eq) atomicAdd(&sm.cta.hist3[key & 0x3FF], 1u);
      }
    }
  }
  stamp(12);
  block_scan2(sm, cg, 0, og, oe, tg, te);
  if (tid == 0) sm.cta_cnt[1][0] = tg;
  exchange_counts<CL>(sm, G, rank, 1);
  {
    int wg = out_base + sm.cta_base[0] + og;
    for (int it = 0; it < trips_b; ++it) {
      const int j = it * nthr + tid;
      if (j < nscan) {
        const int li = overflow ? j : cand[j];
        const uint32_t key = keys[li];
        if ((key >> 21) == b1) {
          const uint32_t mid = (key >> 10) & 0x7FF;
          if (mid > b2 || (done2 && mid == b2)) ro.put(wg++, start + li);
        }
      }
    }
  }
  if (done2) {
    flush_row<CL>(sm, ro, kt, rank);
    return;
  }
  stamp(13);
  // ---- level 3
  const uint32_t* H3 = summed_hist<CL>(sm, sm.cta.hist3, 1024, G, rank);
  find_bin(sm, H3, 1024, rem);
  const uint32_t b3 = static_cast<uint32_t>(sm.bin);
  const int above3 = sm.above;
  const int n_gt = kt - rem + above3;        // slots before the ties
  rem -= above3;
  const uint32_t pre22 = (b1 << 11) | b2;
  // ---- pass C: above the 32-bit threshold, then ties
  cg = 0;
  ce = 0;
  for (int it = 0; it < trips_b; ++it) {
    const int j = it * nthr + tid;
    if (j < nscan) {
      const uint32_t key = keys[overflow ? j : cand[j]];
      if ((key >> 10) == pre22) {
        const uint32_t low = key & 0x3FF;
        cg += low > b3 ? 1 : 0;
        ce += low == b3 ? 1 : 0;
      }
    }
  }
  block_scan2(sm, cg, ce, og, oe, tg, te);
  if (tid == 0) {
    sm.cta_cnt[0][0] = tg;
    sm.cta_cnt[0][1] = te;
  }
  exchange_counts<CL>(sm, G, rank, 0);
  {
    int wg = n_gt - above3 + sm.cta_base[0] + og;
    int we = sm.cta_base[1] + oe;
    for (int it = 0; it < trips_b; ++it) {
      const int j = it * nthr + tid;
      if (j < nscan) {
        const int li = overflow ? j : cand[j];
        const uint32_t key = keys[li];
        if ((key >> 10) == pre22) {
          const uint32_t low = key & 0x3FF;
          if (low > b3) {
            ro.put(wg++, start + li);
          } else if (low == b3) {
            if (we < rem) ro.put(n_gt + we, start + li);
            ++we;
          }
        }
      }
    }
  }
  stamp(14);
  flush_row<CL>(sm, ro, kt, rank);
}

// ---------------------------------------------------------------------------
// One-CTA selection.
//
// A row held by a single CTA is selected with the same 11 + 11 + 10-bit
// refinement, arranged for few barriers and little work per key:
//   - while the scores are produced, the level-1 histogram and its coarse sums
//     (32 bins per entry) are counted, and keys at or above a running lower
//     bound of the level-1 threshold bin go to a short index list
//     (row_filter_append / row_filter_raise).  After the last score the exact
//     bin b1 says whether the list is complete (b1 at or above the last bound);
//     pass A then visits the list, otherwise the whole slice;
//   - every warp finds a threshold bin on its own (no barrier): a prefix over
//     the coarse histogram picks an entry, a prefix over its 32 fine bins
//     picks the bin; all warps read the same histograms;
//   - a pass gives each warp a contiguous segment of the items; a lane counts
//     its items, the warp scans the lane counts and reserves its output range
//     with one shared atomic, and each lane writes its items as one run — no
//     barrier inside a pass.  The level-2 and level-3 histograms are counted
//     in the pass before the level that reads them.
// Barriers per row after the scores: 1 (threshold in the top 11 bits), 2 (22
// bits), 3 (32 bits), plus one before the first level when the caller did not
// prepare the state (select_prepare).  Output order is unspecified (a set).

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Zero the level-2/3 histograms, their coarse sums, the level-1 coarse sums
// and the pass counters (block-wide; a barrier must follow before use).
__device__ __forceinline__ void select_prepare(CtaSelSmem& sm) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  for (int i = tid; i < kHistBins / 4; i += nthr) reinterpret_cast<uint4*>(sm.hist)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = tid; i < kHistBins / 8; i += nthr) reinterpret_cast<uint4*>(sm.hist3)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = tid; i < 3 * 64; i += nthr) sm.coarse[i / 64][i % 64] = 0u;
  if (tid == 0) {
    sm.ctr_gc = 0u;
    sm.ctr_tie = 0u;
  }
}

// Bins in descending order of key; the bin holding the rem-th largest key
// (rem ≥ 1) and the number of keys in higher bins.  NB fine bins, NB/32
// coarse entries (64 or 32).  Warp-collective.
template <int NB>
__device__ __forceinline__ void warp_find_bin(const uint32_t* hist, const uint32_t* coarse, int rem, int& bin,
                                              int& above) {
  constexpr int NC = NB / 32;
  static_assert(NC == 64 || NC == 32, "coarse histogram of 32 or 64 entries");
  const int lane = threadIdx.x & 31;
  int c0, c1 = 0;   // lane's coarse entries, higher one first
  if constexpr (NC == 64) {
    const uint2 v = *reinterpret_cast<const uint2*>(coarse + NC - 2 - 2 * lane);
    c0 = static_cast<int>(v.y);
    c1 = static_cast<int>(v.x);
  } else {
    c0 = static_cast<int>(coarse[NC - 1 - lane]);
  }
  const int s = c0 + c1;
  int inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += t;
  }
  const uint32_t hit = __ballot_sync(0xFFFFFFFFu, inc >= rem);
  if (hit == 0u) {   // fewer than rem keys in the histogram: not reachable with valid counts
    bin = 0;
    above = 0;
    return;
  }
  const int L = __ffs(hit) - 1;
  const int exc = inc - s;
  const bool first = exc + c0 >= rem;
  int sup = NC == 64 ? (first ? NC - 1 - 2 * lane : NC - 2 - 2 * lane) : NC - 1 - lane;
  int sup_above = first ? exc : exc + c0;
  sup = __shfl_sync(0xFFFFFFFFu, sup, L);
  sup_above = __shfl_sync(0xFFFFFFFFu, sup_above, L);
  const int h = static_cast<int>(hist[sup * 32 + 31 - lane]);
  int inc2 = h;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, inc2, o);
    if (lane >= o) inc2 += t;
  }
  const uint32_t hit2 = __ballot_sync(0xFFFFFFFFu, sup_above + inc2 >= rem);
  const int J = hit2 ? __ffs(hit2) - 1 : 31;   // the coarse entry guarantees a hit
  bin = sup * 32 + 31 - J;
  above = sup_above + __shfl_sync(0xFFFFFFFFu, inc2 - h, J);
}

// Production side, per key: level-1 histogram and its coarse sums.
__device__ __forceinline__ void select_count_key(CtaSelSmem& sm, uint32_t* hist1, uint32_t key) {
  atomicAdd(&hist1[key >> 21], 1u);
  atomicAdd(&sm.coarse[0][key >> 26], 1u);
}

// Production side of the row filter, warp-collective (all 32 lanes, each with
// its own key): visible keys at or above the current bound are appended to the
// list at slice index idx.  Entries past the capacity are dropped (the count
// still grows, which marks the list incomplete).
__device__ __forceinline__ void row_filter_append(CtaSelSmem& sm, uint16_t* list, int cap, uint32_t key,
                                                  bool visible, int idx) {
  const uint32_t lo = *reinterpret_cast<const volatile uint32_t*>(&sm.filt_lo);
  const bool p = visible && key >= lo;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, p);
  if (m == 0u) return;
  int base = 0;
  if ((threadIdx.x & 31) == 0) base = atomicAdd(&sm.list_cnt, __popc(m));
  base = __shfl_sync(0xFFFFFFFFu, base, 0);
  const int pos = base + __popc(m & lanemask_lt());
  if (p && pos < cap) list[pos] = static_cast<uint16_t>(idx);
}

// As row_filter_append, with the caller's own test (`take`, visible and at or
// above a bound it read once).
__device__ __forceinline__ void row_filter_append_at(CtaSelSmem& sm, uint16_t* list, int cap, uint32_t key,
                                                     bool take, int idx) {
  (void)key;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
  if (m == 0u) return;
  int base = 0;
  if ((threadIdx.x & 31) == 0) base = atomicAdd(&sm.list_cnt, __popc(m));
  base = __shfl_sync(0xFFFFFFFFu, base, 0);
  const int pos = base + __popc(m & lanemask_lt());
  if (take && pos < cap) list[pos] = static_cast<uint16_t>(idx);
}

// As row_filter_raise, for producers that count only the fine histogram: each
// lane sums 64 bins, then the lane's 64 bins are resolved in pairs.
__device__ __forceinline__ void row_filter_raise_fine(CtaSelSmem& sm, const uint32_t* hist1, int target) {
  const int lane = threadIdx.x & 31;
  // lane l sums bins 1984 − 64l … 2047 − 64l (descending over the lanes)
  const uint4* h4 = reinterpret_cast<const uint4*>(hist1 + 1984 - 64 * lane);
  int s = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint4 v = h4[i];
    s += static_cast<int>(v.x + v.y + v.z + v.w);
  }
  int inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += t;
  }
  const uint32_t hit = __ballot_sync(0xFFFFFFFFu, inc >= target);
  if (hit == 0u) return;
  const int L = __ffs(hit) - 1;
  const int exc_l = __shfl_sync(0xFFFFFFFFu, inc - s, L);
  const int hi = 2047 - 64 * L;             // lane j takes bins hi − 2j (higher) and hi − 2j − 1
  const uint2 pr = *reinterpret_cast<const uint2*>(hist1 + hi - 2 * lane - 1);
  const int a = static_cast<int>(pr.y), b = static_cast<int>(pr.x);
  int inc2 = a + b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, inc2, o);
    if (lane >= o) inc2 += t;
  }
  const uint32_t hit2 = __ballot_sync(0xFFFFFFFFu, exc_l + inc2 >= target);
  const int J = hit2 ? __ffs(hit2) - 1 : 31;
  const int exc2 = __shfl_sync(0xFFFFFFFFu, inc2 - a - b, J);
  const int aJ = __shfl_sync(0xFFFFFFFFu, a, J);
  const int bin = exc_l + exc2 + aJ >= target ? hi - 2 * J : hi - 2 * J - 1;
  if (lane == 0) {
    const uint32_t lo = static_cast<uint32_t>(bin) << 21;
    if (lo > sm.filt_lo) sm.filt_lo = lo;
  }
}

// Raise the bound, one warp (warp-collective): the highest bin L such that at
// least `target` of the keys counted so far lie in bins ≥ L.  Other warps may
// still be adding to the histograms; every count read is at most its final
// value, so L never exceeds what the keys seen so far support.
__device__ __forceinline__ void row_filter_raise(CtaSelSmem& sm, const uint32_t* hist1, int target) {
  int bin, above;
  warp_find_bin<kHistBins>(hist1, sm.coarse[0], target, bin, above);
  // a miss (fewer than target keys counted) or a racy read leaves bin 0: no raise
  if ((threadIdx.x & 31) == 0) {
    const uint32_t lo = static_cast<uint32_t>(bin) << 21;
    if (lo > sm.filt_lo) sm.filt_lo = lo;
  }
}

// Target count for row_filter_raise after m of a row's vis keys: 1.5 × the
// expected share of the kt best among them, plus a margin; 0 = do not raise.
__device__ __forceinline__ int row_filter_target(int m, int vis, int kt) {
  if (vis <= 0 || m <= 0) return 0;
  const int t = static_cast<int>(1.5f * static_cast<float>(kt) * static_cast<float>(m) / static_cast<float>(vis)) + 32;
  return t < m ? t : 0;
}

// Reset the row filter (one thread; a barrier must follow before production).
__device__ __forceinline__ void row_filter_reset(CtaSelSmem& sm) {
  sm.filt_lo = 0u;
  sm.list_cnt = 0;
}

// Items of a pass: entries of a 16-bit index list, or the slice itself (key 0
// past nloc).  A lane takes 4 consecutive items per step.
struct PassItems {
  const uint32_t* keys;
  const uint16_t* list;   // null: the slice
  int n;                  // list entries, or slice length rounded up to 4
  __device__ __forceinline__ void fetch(int i0, uint32_t (&kk)[4], int (&ix)[4]) const {
    if (list) {
      const uint2 e = *reinterpret_cast<const uint2*>(list + i0);
      ix[0] = static_cast<int>(e.x & 0xFFFFu);
      ix[1] = static_cast<int>(e.x >> 16);
      ix[2] = static_cast<int>(e.y & 0xFFFFu);
      ix[3] = static_cast<int>(e.y >> 16);
#pragma unroll
      for (int u = 0; u < 4; ++u) kk[u] = i0 + u < n ? keys[ix[u]] : 0u;
    } else {
      const uint4 q = *reinterpret_cast<const uint4*>(keys + i0);
      kk[0] = q.x;
      kk[1] = q.y;
      kk[2] = q.z;
      kk[3] = q.w;
#pragma unroll
      for (int u = 0; u < 4; ++u) ix[u] = i0 + u;
    }
  }
};

// This warp's segment of a pass over n items (4-aligned bounds).
__device__ __forceinline__ void warp_segment(int n, int& beg, int& end) {
  const int nw = static_cast<int>(blockDim.x >> 5), warp = static_cast<int>(threadIdx.x >> 5);
  const int seg = ((n + nw - 1) / nw + 3) & ~3;
  beg = warp * seg;
  end = min(n, beg + seg);
}

// Warp-collective: reserve this warp's range of a pass from a shared counter
// (packed counts allowed: fields never carry into each other) and return the
// lane's first offset.
__device__ __forceinline__ uint32_t warp_reserve(uint32_t* ctr, uint32_t mine) {
  const int lane = threadIdx.x & 31;
  uint32_t inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += t;
  }
  uint32_t base = 0u;
  if (lane == 31 && inc != 0u) base = atomicAdd(ctr, inc);
  return __shfl_sync(0xFFFFFFFFu, base, 31) + inc - mine;
}

// Select the kt best keys of a row held by one CTA.
//   keys[0 … nloc)    order keys of the slice (positions start …), 16-byte
//                     aligned, key 0 from nloc up to the next multiple of 4
//   hist1             histogram of keys >> 21 over the visible keys
//   prepared          the caller ran select_prepare (then a barrier) before the
//                     scores and counted sm.coarse[0] with select_count_key;
//                     otherwise this call clears and sums with one barrier
//   list, list_cap    the production-time list (null: pass A scans the slice);
//                     list_cap a multiple of 4
//   cand, cand_cap    scratch for the keys of the level-1 threshold bin
//                     (cand_cap a multiple of 4)
//   out               the row's output slots (global memory)
//   stage             shared memory for kStage positions, or null: when given
//                     and kt ≤ kStage, positions are staged there and written
//                     to `out` with coalesced stores at the end
// Requires 0 < kt < number of visible keys; all threads of the CTA call it.
__device__ __forceinline__ void cta_select_row(CtaSelSmem& sm, const uint32_t* keys, int nloc, int start, int kt,
                                               const uint32_t* hist1, bool prepared, const uint16_t* list,
                                               int list_cap, uint16_t* cand, int cand_cap, int32_t* out,
                                               int32_t* stage, unsigned long long* tr,
                                               const volatile int* abort_flag) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  auto stamp = [&](int slot) {
    if (tr && tid == 0) tr[slot] = globaltimer_ns();
  };
  const bool staged = stage && kt <= kStage;
  int32_t* const dst = staged ? stage : out;
  uint32_t* const hist2 = sm.hist;
  uint32_t* const hist3 = sm.hist3;
  uint32_t* const coarse1 = sm.coarse[0];
  uint32_t* const coarse2 = sm.coarse[1];
  uint32_t* const coarse3 = sm.coarse[2];
  if (!prepared) {
    select_prepare(sm);
    if (tid < 64) {
      const uint4* h = reinterpret_cast<const uint4*>(hist1 + 32 * tid);
      uint32_t s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = h[i];
        s += v.x + v.y + v.z + v.w;
      }
      coarse1[tid] = s;
    }
    __syncthreads();
  }
  if (abort_flag && *abort_flag) {   // the scores are not valid: the row reads −1
    for (int i = tid; i < kt; i += nthr) out[i] = -1;
    return;
  }

  // ---- level 1 (every warp)
  int b1, above1;
  warp_find_bin<kHistBins>(hist1, coarse1, kt, b1, above1);
  int rem = kt - above1;                      // keys still to take from bin b1 (≥ 1)
  const int n1 = static_cast<int>(hist1[b1]);
  const bool done1 = n1 == rem;
  const bool clist = !done1 && n1 <= cand_cap;   // bin-b1 keys listed; else later passes rescan the slice
  const uint32_t lo1 = static_cast<uint32_t>(b1) << 21;
  const int nlist = list ? sm.list_cnt : 0;
  const bool use_list = list && nlist <= list_cap && lo1 >= sm.filt_lo;
  stamp(8);
  if (tr && tid == 0) {
    tr[9] = use_list ? static_cast<unsigned long long>(nlist) : ~0ull;
    tr[15] = static_cast<unsigned long long>(n1);
  }

  // ---- pass A: keys above bin b1 are selected (all of bin b1 too when it
  // holds exactly the open slots); keys in b1 are listed and histogrammed
  // done1: keys ≥ lo1 are selected, so no key is both ≤ sel_above and ≥ lo1
  const uint32_t sel_above = done1 ? lo1 - 1u : lo1 | 0x1FFFFFu;
  {
    const PassItems it{keys, use_list ? list : nullptr, use_list ? nlist : (nloc + 3) & ~3};
    int beg, end;
    warp_segment(it.n, beg, end);
    const int lane4 = 4 * (tid & 31);
    uint32_t cnt = 0;   // selected | candidates << 16
    for (int i0 = beg + lane4; i0 < end; i0 += 128) {
      uint32_t kk[4];
      int ix[4];
      it.fetch(i0, kk, ix);
#pragma unroll
      for (int u = 0; u < 4; ++u) cnt += (kk[u] > sel_above ? 1u : 0u) + (kk[u] >= lo1 ? 0x10000u : 0u);
    }
    // the high half counted keys ≥ lo1: keep those inside b1 (none when done1)
    cnt -= (cnt & 0xFFFFu) << 16;
    const uint32_t off = warp_reserve(&sm.ctr_gc, cnt);
    int og = static_cast<int>(off & 0xFFFFu), oc = static_cast<int>(off >> 16);
    for (int i0 = beg + lane4; i0 < end; i0 += 128) {
      uint32_t kk[4];
      int ix[4];
      it.fetch(i0, kk, ix);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (kk[u] > sel_above) {
          if (og < kt) dst[og] = start + ix[u];
          ++og;
        } else if (kk[u] >= lo1) {
          if (clist && oc < cand_cap) cand[oc] = static_cast<uint16_t>(ix[u]);
          ++oc;
          const uint32_t mid = (kk[u] >> 10) & 0x7FFu;
          atomicAdd(&hist2[mid], 1u);
          atomicAdd(&coarse2[mid >> 5], 1u);
        }
      }
    }
  }
  __syncthreads();                                                   // barrier 1
  stamp(10);
  if (done1) {
    if (staged)
      for (int i = tid; i < kt; i += nthr) out[i] = stage[i];
    return;
  }
  // items of the later passes: the listed keys of bin b1, or the slice filtered by b1
  const PassItems it{keys, clist ? cand : nullptr, clist ? n1 : (nloc + 3) & ~3};
  int beg, end;
  warp_segment(it.n, beg, end);
  const int lane4 = 4 * (tid & 31);

  // ---- level 2 (every warp) and pass B
  int b2, above2;
  warp_find_bin<kHistBins>(hist2, coarse2, rem, b2, above2);
  rem -= above2;
  const bool done2 = static_cast<int>(hist2[b2]) == rem;
  const uint32_t pre22 = static_cast<uint32_t>(b1) << 11 | static_cast<uint32_t>(b2);
  // selected: the 22-bit prefix above pre22 (or equal when done2) within bin b1
  const uint32_t sel22 = done2 ? pre22 - 1u : pre22;
  stamp(11);
  {
    uint32_t cnt = 0;
    for (int i0 = beg + lane4; i0 < end; i0 += 128) {
      uint32_t kk[4];
      int ix[4];
      it.fetch(i0, kk, ix);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t h22 = kk[u] >> 10;
        cnt += ((h22 >> 11) == static_cast<uint32_t>(b1) && h22 > sel22) ? 1u : 0u;
      }
    }
    int og = static_cast<int>(warp_reserve(&sm.ctr_gc, cnt) & 0xFFFFu);
    for (int i0 = beg + lane4; i0 < end; i0 += 128) {
      uint32_t kk[4];
      int ix[4];
      it.fetch(i0, kk, ix);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t h22 = kk[u] >> 10;
        if ((h22 >> 11) != static_cast<uint32_t>(b1)) continue;
        if (h22 > sel22) {
          if (og < kt) dst[og] = start + ix[u];
          ++og;
        } else if (!done2 && h22 == pre22) {
          const uint32_t low = kk[u] & 0x3FFu;
          atomicAdd(&hist3[low], 1u);
          atomicAdd(&coarse3[low >> 5], 1u);
        }
      }
    }
  }
  __syncthreads();                                                   // barrier 2
  stamp(12);
  if (!done2) {
    // ---- level 3 (every warp) and pass C: above the 32-bit threshold, then ties
    int b3, above3;
    warp_find_bin<kHistBins / 2>(hist3, coarse3, rem, b3, above3);
    const int n_gt = kt - rem + above3;       // ties start at this slot
    rem -= above3;                            // ties to take (≥ 1)
    const uint32_t thr = pre22 << 10 | static_cast<uint32_t>(b3);
    stamp(13);
    uint32_t cnt = 0;
    for (int i0 = beg + lane4; i0 < end; i0 += 128) {
      uint32_t kk[4];
      int ix[4];
      it.fetch(i0, kk, ix);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if ((kk[u] >> 10) == pre22) cnt += (kk[u] > thr ? 1u : 0u) + (kk[u] == thr ? 0x10000u : 0u);
    }
    const uint32_t off = warp_reserve(&sm.ctr_tie, cnt);   // ctr_tie: above | ties << 16, from 0
    int og = n_gt - above3 + static_cast<int>(off & 0xFFFFu), oe = static_cast<int>(off >> 16);
    for (int i0 = beg + lane4; i0 < end; i0 += 128) {
      uint32_t kk[4];
      int ix[4];
      it.fetch(i0, kk, ix);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if ((kk[u] >> 10) != pre22) continue;
        if (kk[u] > thr) {
          if (og < n_gt) dst[og] = start + ix[u];
          ++og;
        } else if (kk[u] == thr) {
          if (oe < rem) dst[n_gt + oe] = start + ix[u];
          ++oe;
        }
      }
    }
    __syncthreads();                                                 // barrier 3
  }
  stamp(14);
  if (staged)
    for (int i = tid; i < kt; i += nthr) out[i] = stage[i];
}

// Select the kt best of a row, one CTA or a cluster.  `cand` is cap ints of
// scratch: a cluster uses it as its candidate list; one CTA splits it into the
// production-time list (its first list_cap 16-bit entries; list_cap a multiple
// of 4, 0 = none) and 16-bit candidate slots.  `prepared`: see cta_select_row.
__device__ __forceinline__ void cluster_select_row(SelectSmem& sm, const uint32_t* keys, int nloc, int start,
                                                   int kt, const uint32_t* hist1, int* cand, int cap, int list_cap,
                                                   bool prepared, int32_t* out, int G, uint32_t rank,
                                                   unsigned long long* tr = nullptr,
                                                   const int* abort_flag = nullptr) {
  if (G == 1) {
    uint16_t* s16 = reinterpret_cast<uint16_t*>(cand);
    cta_select_row(sm.cta, keys, nloc, start, kt, hist1, prepared, list_cap > 0 ? s16 : nullptr, list_cap,
                   s16 + list_cap, (2 * cap - list_cap) & ~3, out, sm.out_s, tr, abort_flag);
  } else {
    cluster_select_row_t<true>(sm, keys, nloc, start, kt, hist1, cand, cap, out, G, rank, tr, abort_flag);
  }
}

}  // namespace idx
