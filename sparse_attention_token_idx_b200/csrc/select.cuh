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

struct SelectSmem {
  uint32_t hist[kHistBins];      // this CTA's level-2 histogram
  uint32_t hist3[kHistBins / 2]; // this CTA's level-3 histogram (own buffer: one barrier per exchange)
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
  for (int i = tid; i < kHistBins; i += nthr) sm.hist[i] = 0;
  for (int i = tid; i < kHistBins / 2; i += nthr) sm.hist3[i] = 0;

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
    for (int c = tid; c < te; c += nthr) atomicAdd(&sm.hist[(keys[cand[c]] >> 10) & 0x7FF], 1u);
  } else {
    for (int i = tid; i < nloc; i += nthr) {
      const uint32_t key = keys[i];
      if ((key >> 21) == b1) atomicAdd(&sm.hist[(key >> 10) & 0x7FF], 1u);
    }
  }
  stamp(11);
  // ---- level 2
  const uint32_t* H2 = summed_hist<CL>(sm, sm.hist, kHistBins, G, rank);
  find_bin(sm, H2, kHistBins, rem);
  const uint32_t b2 = static_cast<uint32_t>(sm.bin);
  rem -= sm.above;
  const bool done2 = static_cast<int>(H2[b2]) == rem;
  __syncthreads();                           // everyone has read H2 (it may be sm.hist)
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
        if (!done2 && eq) atomicAdd(&sm.hist3[key & 0x3FF], 1u);
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
  const uint32_t* H3 = summed_hist<CL>(sm, sm.hist3, 1024, G, rank);
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

__device__ __forceinline__ void cluster_select_row(SelectSmem& sm, const uint32_t* keys, int nloc, int start,
                                                   int kt, const uint32_t* hist1, int* cand, int cap,
                                                   int32_t* out, int G, uint32_t rank,
                                                   unsigned long long* tr = nullptr,
                                                   const int* abort_flag = nullptr) {
  if (G == 1)
    cluster_select_row_t<false>(sm, keys, nloc, start, kt, hist1, cand, cap, out, G, rank, tr, abort_flag);
  else
    cluster_select_row_t<true>(sm, keys, nloc, start, kt, hist1, cand, cap, out, G, rank, tr, abort_flag);
}

}  // namespace idx
