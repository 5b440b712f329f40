// Sparse latent attention on the tensor cores ("Join query parts" page, MQA
// decode excerpt): for one decode token per sequence and each of 128 heads,
// scores against the selected 576-feature cache rows (512 latent + 64 rotary),
// a softmax over them, and the latent output Σ_t p_t · row_t[0:512].
//
// One CTA per (sequence, block of 128 heads, half of the 512 output columns):
// the two halves recompute the same scores (a softmax needs all of them) and
// each accumulates 256 output columns.  The queries stay resident for the
// whole walk: features 0-383 in TMEM as the A operand of the score MMAs (six
// 64-feature tiles, two bf16 per 32-bit column), features 384-575 in shared
// memory (three 128-byte-swizzled tiles, by TMA).  TMEM: query tiles at
// columns 0-191, one 64-column score tile at 192, the output half at 256.
// The selection is walked in chunks of 64 positions:
//   warps 6…    gather the chunk's rows (16-byte cp.async, 1152 B per row) into
//               shared memory as nine 64-feature K tiles in the 128-byte swizzle
//               layout (row = position); unselected slots are zeros; two chunk
//               buffers;
//   warp 0      loads the three shared-memory query tiles once;
//   warp 1      owns TMEM and issues tcgen05.mma kind::f16 (bf16 → fp32):
//               S = Q · Kᵀ into the score tile (N = 64, K = 576: 24 MMAs with
//               A in TMEM, 12 with A in shared memory), and O += P · V (N = 256,
//               K = 64 positions) where V is this CTA's four 64-feature tiles of
//               the same gathered bytes read as an MN-major operand; the
//               product of chunk c − 1 goes before the scores of chunk c, so
//               that its buffer is refilled while those scores run;
//   warps 2-5   load their head's query features 0-383 into TMEM at the start;
//               then softmax, thread ↔ head: read the score row from TMEM, mask
//               unselected slots, keep a running reference maximum m (raised
//               only when a chunk's maximum exceeds it by more than 8, then the
//               O row and the running sum are rescaled), p = exp(s − m) rounded
//               to bf16 into the P tile (A operand, 128 × 64, 128-byte swizzle)
//               and summed (fp32) as rounded; at the end O / Σp.
// Every wait is bounded; a CTA that gives up raises IDX_DEV_ERR_TIMEOUT, waits
// for its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "api_internal.h"
#include "ptx.cuh"

namespace idx {
namespace {

constexpr int kTcHeads = 128;              // heads per CTA (TMEM lanes)
constexpr int kTcDim = 576;                // latent + rotary
constexpr int kTcHalf = 256;               // output columns per CTA
constexpr int kTcChunk = 64;               // positions per chunk
constexpr int kTcKTiles = kTcDim / 64;     // 9 feature tiles of 64
constexpr int kTcGatherWarps = 4;          // warps 6 … 6 + kTcGatherWarps − 1
constexpr int kTcThreads = (6 + kTcGatherWarps) * 32;
constexpr int kTcGatherThreads = kTcGatherWarps * 32;
constexpr int kTcRowsPerWarp = 64 / kTcGatherWarps;   // chunk rows each gather warp copies
constexpr float kTcRescale = 8.f;          // raise the reference maximum past this margin
constexpr int kTcQTmemTiles = 6;           // query feature tiles held in TMEM (features 0-383)
constexpr int kTcQSmemTiles = kTcKTiles - kTcQTmemTiles;   // the rest in shared memory

constexpr int kQTile = kTcHeads * 128;               // 16 KB
constexpr int kKvTile = kTcChunk * 128;              // 8 KB per 64-feature tile of a chunk
constexpr int kKvChunk = kTcKTiles * kKvTile;        // 72 KB
constexpr int kPTile = kTcHeads * 128;               // 16 KB: 128 heads × 64 positions bf16

constexpr int kOffQ = 0;
constexpr int kOffKv = kOffQ + kTcQSmemTiles * kQTile;
constexpr int kOffP = kOffKv + 2 * kKvChunk;
constexpr int kOffBar = kOffP + kPTile;
// barriers: q_full kv_full[2] kv_empty[2] s_full s_empty p_full p_empty o_done drain
constexpr int kNumBars = 1 + 2 + 2 + 6;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kTcSmem = 1024 + kOffMisc + 16;

// TMEM columns: query tiles (32 columns each), the score tile, the output half
constexpr uint32_t kColQ = 0;
constexpr uint32_t kColS = kTcQTmemTiles * 32;
constexpr uint32_t kColO = 256;
static_assert(kColS + kTcChunk <= kColO, "TMEM columns");

// kind::f16, A = B = bf16, D = f32; b_mn: B operand MN-major
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn ? (1u << 16) : 0u) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with A read from TMEM (row m in lane m, two bf16 per 32-bit column).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// MN-major operand in the 128-byte swizzle layout: 64 elements (128 B) along MN
// per row, rows along K in 8-row (1024 B) atoms; `mn_stride` bytes to the next
// 64-element group along MN.
__device__ __forceinline__ uint64_t smem_desc_mn128_sw128(uint32_t saddr, uint32_t mn_stride) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((mn_stride >> 4) & 0x3FFF) << 16;   // leading byte offset: next MN group
  d |= static_cast<uint64_t>(1024 >> 4) << 32;                    // stride byte offset: next 8 K rows
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// byte offset of 16-byte piece c (0..7) of row r in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

struct TcParams {
  const uint16_t* q;         // [B, H, 576]
  const uint16_t* kv;        // [B, T_cap, 576]
  const int32_t* indices;    // [B, k]
  float* out;                // [B, H, 512]
  int64_t T_cap;
  int H, k, nchunks;
  float scale;
  unsigned long long budget_ns;
  unsigned int* err;
};

__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* q_s = smem + kOffQ;
  uint8_t* kv_s = smem + kOffKv;
  uint8_t* p_s = smem + kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars;          // the shared-memory query tiles have landed
  uint64_t* kv_full = bars + 1;     // [2]
  uint64_t* kv_empty = bars + 3;    // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* s_empty = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* p_empty = bars + 8;
  uint64_t* o_done = bars + 9;
  uint64_t* drain_bar = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = p.H / kTcHeads;
  const int half = blockIdx.x & 1;
  const int64_t bg = blockIdx.x >> 1;                 // (sequence, head block)
  const int64_t b = bg / groups;
  const int h0 = static_cast<int>(bg % groups) * kTcHeads;
  const int nch = p.nchunks;
  const uint64_t budget = p.budget_ns;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], kTcGatherThreads);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    mbar_init(p_full, 4);
    mbar_init(p_empty, 1);
    mbar_init(o_done, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_q);
    // query features 384-575: three 64-feature tiles, once
    mbar_arrive_expect_tx(q_full, kTcQSmemTiles * kQTile);
    for (int t = 0; t < kTcQSmemTiles; ++t)
      tma_load_2d(q_s + t * kQTile, &tmap_q, q_full, (kTcQTmemTiles + t) * 64, static_cast<int>(b * p.H + h0));
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 2 && warp < 6) {
    // query features 0-383 of head h into TMEM lane h: 32 columns per 64 features
    const int h = (warp & 3) * 32 + lane;
    const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (b * p.H + h0 + h) * kTcDim);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll 1
    for (int t = 0; t < kTcQTmemTiles; ++t) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = __ldg(qrow + t * 8 + i);
        r[4 * i] = v.x;
        r[4 * i + 1] = v.y;
        r[4 * i + 2] = v.z;
        r[4 * i + 3] = v.w;
      }
      tmem_st32(lane_base + kColQ + static_cast<uint32_t>(t * 32), r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  bool mma_issued = false;

  if (warp == 0) {
    // the query tiles were requested during set-up
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16(kTcHeads, kTcChunk, false);
      constexpr uint32_t id_o = idesc_bf16(kTcHeads, kTcHalf, true);
      bool ok = mbar_wait(q_full, 0, budget, abort_flag, p.err);
      const uint32_t d_s = tmem + kColS;
      // O += P(c − 1) · V(c − 1), then S(c): the product frees chunk c − 1's
      // buffer before the scores of chunk c start, so that the gather of chunk
      // c + 1 runs under the MMAs of chunk c (the scores are issued as soon as
      // the softmax has read the previous ones out of TMEM)
      for (int c = 0; c <= nch && ok; ++c) {
        if (c >= 1) {
          const int pc = c - 1, buf = pc & 1;
          if (!mbar_wait(p_full, pc & 1, budget, abort_flag, p.err)) break;
          tc_fence_after();
          const uint32_t p_addr = smem_u32(p_s);
          // this CTA's value columns: feature tiles 4·half … 4·half + 3 of the chunk
          const uint32_t v_addr = smem_u32(kv_s + buf * kKvChunk + (4 * half) * kKvTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)     // 16 positions per instruction: two 8-row atoms
            mma_f16(tmem + kColO, smem_desc_k128_sw128(p_addr + kk * 32),
                    smem_desc_mn128_sw128(v_addr + kk * 2048, kKvTile), id_o, (pc > 0 || kk > 0) ? 1u : 0u);
          mma_commit(p_empty);
          mma_commit(&kv_empty[buf]);
          if (pc == nch - 1) mma_commit(o_done);
          mma_issued = true;
        }
        if (c < nch) {
          const int buf = c & 1;
          ok = mbar_wait(&kv_full[buf], (c >> 1) & 1, budget, abort_flag, p.err);
          if (ok && c >= 1) ok = mbar_wait(s_empty, (c - 1) & 1, budget, abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kv_addr = smem_u32(kv_s + buf * kKvChunk);
          for (int kt = 0; kt < kTcKTiles; ++kt) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {   // 16 bf16 (32 bytes) per instruction
              const uint64_t bd = smem_desc_k128_sw128(kv_addr + kt * kKvTile + kk * 32);
              const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
              if (kt < kTcQTmemTiles)
                mma_f16_ta(d_s, tmem + kColQ + static_cast<uint32_t>(kt * 32 + kk * 8), bd, id_s, acc);
              else
                mma_f16(d_s, smem_desc_k128_sw128(smem_u32(q_s + (kt - kTcQTmemTiles) * kQTile) + kk * 32), bd, id_s,
                        acc);
            }
          }
          mma_commit(s_full);
          mma_issued = true;
        }
      }
      if (mma_issued) mma_commit(drain_bar);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int h = quad * 32 + lane;                   // head within the block (TMEM lane)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int32_t* sel = p.indices + b * p.k;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      // which of the chunk's 64 slots select a cache row (two indices per lane),
      // read before the wait for the scores so that the loads overlap it
      uint32_t vmask[2];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int j = c * kTcChunk + g * 32 + lane;
        const int t = j < p.k ? __ldg(sel + j) : -1;
        vmask[g] = __ballot_sync(0xFFFFFFFFu, t >= 0 && t < p.T_cap);
      }
      int w = 1;
      if (lane == 0) w = mbar_wait(s_full, c & 1, budget, abort_flag, p.err) ? 1 : 0;
      if (!__shfl_sync(0xFFFFFFFFu, w, 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32_nowait(lane_base + kColS, r);
      tmem_ld32_nowait(lane_base + kColS + 32u, r + 32);
      tmem_wait();
      tmem_regs_ready(r);
      tmem_regs_ready(r + 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      float cmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float s = (vmask[j >> 5] >> (j & 31)) & 1u ? __uint_as_float(r[j]) * p.scale : -INFINITY;
        r[j] = __float_as_uint(s);
        cmax = fmaxf(cmax, s);
      }
      // P and O are free once the previous chunk's P · V has completed
      if (c >= 1) {
        if (lane == 0) w = mbar_wait(p_empty, (c - 1) & 1, budget, abort_flag, p.err) ? 1 : 0;
        if (!__shfl_sync(0xFFFFFFFFu, w, 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // raise the reference maximum where a head's chunk maximum passed it:
      // the running sum and the O row are rescaled.  The TMEM loads and stores
      // are warp-collective, so the whole warp walks the O rows when any lane
      // raises (α = 1 for the others; a head with no earlier position has O = 0)
      const bool raise = cmax > m_ref + kTcRescale || (m_ref == -INFINITY && cmax > -INFINITY);
      const float alpha = !raise ? 1.f : (m_ref == -INFINITY ? 0.f : __expf(m_ref - cmax));
      if (c >= 1 && __any_sync(0xFFFFFFFFu, raise)) {
#pragma unroll 1
        for (int q = 0; q < kTcHalf / 32; ++q) {
          uint32_t o[32];
          tmem_ld32_nowait(lane_base + kColO + static_cast<uint32_t>(q * 32), o);
          tmem_wait();
          tmem_regs_ready(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(lane_base + kColO + static_cast<uint32_t>(q * 32), o);
        }
        tmem_wait_st();
      }
      if (raise) {
        l *= alpha;
        m_ref = cmax;
      }
      // p = exp(s − m), rounded to bf16 into the P row (64 positions = 128 B),
      // summed as rounded
      uint8_t* prow = p_s;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        uint32_t wv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float s0 = __uint_as_float(r[c16 * 8 + 2 * e]);
          const float s1 = __uint_as_float(r[c16 * 8 + 2 * e + 1]);
          const __nv_bfloat16 p0 = __float2bfloat16_rn(s0 == -INFINITY ? 0.f : __expf(s0 - m_ref));
          const __nv_bfloat16 p1 = __float2bfloat16_rn(s1 == -INFINITY ? 0.f : __expf(s1 - m_ref));
          l += __bfloat162float(p0);
          l += __bfloat162float(p1);
          wv[e] = static_cast<uint32_t>(__bfloat16_as_ushort(p0)) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(p1)) << 16);
        }
        *reinterpret_cast<uint4*>(prow + sw128(h, c16)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---- the output half: O / Σp
    int w = ok ? 1 : 0;
    if (ok && lane == 0) w = mbar_wait(o_done, 0, budget, abort_flag, p.err) ? 1 : 0;
    w = __shfl_sync(0xFFFFFFFFu, w, 0);
    if (w) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* ob = p.out + ((b * p.H) + h0 + h) * 512 + half * kTcHalf;
#pragma unroll 1
      for (int q = 0; q < kTcHalf / 32; ++q) {
        float v[32];
        tmem_ld32(lane_base + kColO + static_cast<uint32_t>(q * 32), v);
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(ob + q * 32 + i) = make_float4(v[i] * inv, v[i + 1] * inv, v[i + 2] * inv, v[i + 3] * inv);
      }
    }
  } else {
    // ------------------------------------------------------------ gather
    // gather warp gw copies rows gw, gw + W, gw + 2W, … of a chunk (W gather
    // warps): its first lanes fetch those rows' positions once, then each row
    // goes out as 72 consecutive 16-byte pieces across the warp (lane l:
    // pieces l, l + 32, l + 64)
    const int gw = warp - 6;
    const uint16_t* kvb = p.kv + b * p.T_cap * kTcDim;
    const int32_t* sel = p.indices + b * p.k;
    bool ok = true;
    for (int c = 0; c <= nch && ok; ++c) {
      // the previous chunk's copies have landed: make them visible to the MMAs
      // and announce them first — the buffer this chunk needs is freed by the
      // product of chunk c − 2, which the MMA warp issues before the scores of
      // chunk c − 1
      if (c >= 1) {
        cp_async_wait<0>();
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[(c - 1) & 1]);
      }
      if (c == nch) break;
      const int buf = c & 1;
      int pos = -1;
      if (lane < kTcRowsPerWarp) {
        const int j = c * kTcChunk + gw + kTcGatherWarps * lane;
        pos = j < p.k ? __ldg(sel + j) : -1;
      }
      if (c >= 2) {
        int w = 1;
        if (lane == 0) w = mbar_wait(&kv_empty[buf], ((c >> 1) - 1) & 1, budget, abort_flag, p.err) ? 1 : 0;
        if (!__shfl_sync(0xFFFFFFFFu, w, 0)) {
          ok = false;
          break;
        }
      }
      const uint32_t base = smem_u32(kv_s + buf * kKvChunk);
#pragma unroll 1
      for (int i = 0; i < kTcRowsPerWarp; ++i) {
        const int r = gw + kTcGatherWarps * i;
        const int t = __shfl_sync(0xFFFFFFFFu, pos, i);
        const bool valid = t >= 0 && t < p.T_cap;
        const uint16_t* src = kvb + static_cast<int64_t>(valid ? t : 0) * kTcDim;
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          const int piece = lane + 32 * q;
          if (piece < kTcDim / 8) {
            const uint32_t dst = base + static_cast<uint32_t>((piece >> 3) * kKvTile) + sw128(r, piece & 7);
            if (valid) cp_async16(dst, src + piece * 8);
            else asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
          }
        }
      }
      cp_async_commit();
    }
    cp_async_wait<0>();
  }
  __syncthreads();
  // ------------------------------------------------------------ teardown
  if (warp == 0 && lane == 0) {
    int dummy = 0;
    mbar_wait(q_full, 0, budget, &dummy, p.err);   // the query tiles have landed before the memory goes
  }
  if (warp == 1 && lane == 0 && mma_issued) {
    int dummy = 0;
    mbar_wait(drain_bar, 0, budget, &dummy, p.err);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

// Launch of the tensor-core kernel; IDX_ERR_UNSUPPORTED when the shape is not
// one it serves (H not a multiple of 128, q not 16-byte aligned).
int launch_sparse_mla_tc(const uint16_t* q, const uint16_t* kv, const int32_t* indices, int B, int H, int64_t T_cap,
                         int k, float softmax_scale, float* out, cudaStream_t stream) {
  if (H % kTcHeads || (reinterpret_cast<uintptr_t>(q) & 15)) return IDX_ERR_UNSUPPORTED;
  CUtensorMap tq;
  if (!make_tmap_2d_bf16_sw128(&tq, q, kTcDim, static_cast<uint64_t>(B) * H, kTcHeads)) return IDX_ERR_UNSUPPORTED;
  const int64_t blocks = static_cast<int64_t>(B) * (H / kTcHeads) * 2;
  if (blocks > 0x7FFFFFFF) return IDX_ERR_SHAPE;
  if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(sparse_mla_tc_kernel), kTcSmem)) return r;
  TcParams p;
  p.q = q;
  p.kv = kv;
  p.indices = indices;
  p.out = out;
  p.T_cap = T_cap;
  p.H = H;
  p.k = k;
  p.nchunks = (k + kTcChunk - 1) / kTcChunk;
  p.scale = softmax_scale;
  const DebugState dbg = debug_state();
  p.budget_ns = dbg.budget_ns;
  p.err = device_error_word();
  if (!p.err) return check_launch();
  sparse_mla_tc_kernel<<<static_cast<unsigned>(blocks), kTcThreads, kTcSmem, stream>>>(tq, p);
  return check_launch();
}

}  // namespace idx
