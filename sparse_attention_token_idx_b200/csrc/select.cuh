// Cluster-wide top-k selection over scores held in shared memory.
//
// A row's visible scores are split over the G CTAs of a thread-block cluster,
// each holding its contiguous slice as order-preserving uint32 keys.  The
// k_t-th largest key is found by radix refinement (11, 11, 10 bits): each CTA
// histograms its matching keys, every CTA sums all G histograms through
// distributed shared memory and takes the same decision, so the control flow
// (and every cluster barrier) is identical in all CTAs.  The final pass writes
// the positions: keys above the threshold prefix all go out, keys equal to it
// fill the remaining slots; slots come from two counters in CTA 0's shared
// memory, bumped once per warp.  Output order is unspecified (a set), as the
// NKI indexer page states for its top-k output.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace idx {

constexpr int kHistBins = 2048;

struct SelectSmem {
  uint32_t hist_local[kHistBins];
  uint32_t hist_sum[kHistBins];
  int warp_tot[32];
  int bin;
  int above;
  uint32_t cnt_gt;  // used in CTA 0 only
  uint32_t cnt_eq;  // used in CTA 0 only
  int any_abort;
  int pad[3];
};

// Block-wide: given descending-order bin counts, find the bin that holds the
// rem-th largest element; result in sm.bin / sm.above (count in higher bins).
__device__ __forceinline__ void find_bin(SelectSmem& sm, const uint32_t* hist, int nb, int rem) {
  const int nthr = blockDim.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int per = (nb + nthr - 1) / nthr;
  const int hi = nb - tid * per;            // thread tid covers bins [lo, hi), highest bins first
  const int lo = hi - per;
  int csum = 0;
  for (int bn = hi - 1; bn >= lo && bn >= 0; --bn) csum += hist[bn];
  // inclusive warp scan
  int incl = csum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) sm.warp_tot[warp] = incl;
  __syncthreads();
  int wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += sm.warp_tot[w];
  const int excl = wbase + incl - csum;
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

// Select the kt best of the row whose keys are split over the cluster.
//   keys[0 … nloc)   this CTA's slice, positions start … start+nloc−1 (keys of
//                    masked positions must not be in the slice).
//   vis              visible keys of the row (sum of all slices' nloc).
//   kt               min(k, vis) (the caller handles kt == vis separately).
//   out              the row's k output slots (global memory).
// All threads of all CTAs in the cluster must call this with the same vis/kt.
__device__ __forceinline__ void cluster_select_row(SelectSmem& sm, const uint32_t* keys, int nloc, int start,
                                                   int kt, int32_t* out, int G, uint32_t rank) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  uint32_t prefix = 0;
  int pbits = 0;
  int rem = kt;
  if (rank == 0 && tid == 0) {
    sm.cnt_gt = 0;
    sm.cnt_eq = 0;
  }
  for (int pass = 0; pass < 3; ++pass) {
    const int width = pass < 2 ? 11 : 10;
    const int shift = 32 - pbits - width;
    const int nb = 1 << width;
    for (int i = tid; i < nb; i += nthr) sm.hist_local[i] = 0;
    __syncthreads();
    for (int i = tid; i < nloc; i += nthr) {
      const uint32_t u = keys[i];
      if (pbits == 0 || (u >> (32 - pbits)) == prefix) atomicAdd(&sm.hist_local[(u >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    cluster_sync();
    for (int i = tid; i < nb; i += nthr) {
      uint32_t s = 0;
      for (int r = 0; r < G; ++r) s += dsmem_ld_u32(dsmem_addr(&sm.hist_local[i], r));
      sm.hist_sum[i] = s;
    }
    __syncthreads();
    find_bin(sm, sm.hist_sum, nb, rem);
    const int bin = sm.bin;
    rem -= sm.above;
    prefix = (prefix << width) | static_cast<uint32_t>(bin);
    pbits += width;
    const bool done = static_cast<int>(sm.hist_sum[bin]) == rem;
    cluster_sync();  // nobody clears hist_local while another CTA still reads it
    if (done) break;
  }
  // output pass
  const int n_gt = kt - rem;
  const uint32_t gt_addr = dsmem_addr(&sm.cnt_gt, 0);
  const uint32_t eq_addr = dsmem_addr(&sm.cnt_eq, 0);
  const int lane = tid & 31;
  const int sh = 32 - pbits;
  for (int base = 0; base < nloc; base += nthr) {
    const int i = base + tid;
    bool gt = false, eq = false;
    if (i < nloc) {
      const uint32_t top = sh >= 32 ? 0u : (keys[i] >> sh);
      gt = top > prefix;
      eq = top == prefix;
    }
    const uint32_t mgt = __ballot_sync(0xFFFFFFFFu, gt);
    const uint32_t meq = __ballot_sync(0xFFFFFFFFu, eq);
    const uint32_t below = (1u << lane) - 1u;
    if (mgt) {
      uint32_t b0 = 0;
      if (lane == 0) b0 = dsmem_atom_add_u32(gt_addr, __popc(mgt));
      b0 = __shfl_sync(0xFFFFFFFFu, b0, 0);
      if (gt) out[b0 + __popc(mgt & below)] = start + i;
    }
    if (meq) {
      uint32_t b0 = 0;
      if (lane == 0) b0 = dsmem_atom_add_u32(eq_addr, __popc(meq));
      b0 = __shfl_sync(0xFFFFFFFFu, b0, 0);
      const uint32_t slot = b0 + __popc(meq & below);
      if (eq && slot < static_cast<uint32_t>(rem)) out[n_gt + slot] = start + i;
    }
  }
  cluster_sync();  // counters of CTA 0 are reused by the next row
}

}  // namespace idx
