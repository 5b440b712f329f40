// The indexer's projections, the first steps of the Indexer.forward excerpt
// ("Index scores" page): q = wq_b(qr), k = wk(x), and the head weights
// weights_proj(x.float()).
//
// q and k are bf16 GEMMs on the tensor cores, C[m, n] = Σ_k A[m, k]·B[n, k]
// with A the activations [M, K] and B the Linear weight [N, K] (both K
// contiguous), fp32 accumulation in TMEM, then one round-to-nearest-even to
// bf16.  A CTA computes a 128-row × BN-column tile:
//   warp 0      TMA producer: 64-wide K tiles of A (128 × 128 B) and B
//               (BN × 128 B), 128-byte swizzle, into a STAGES ring;
//   warp 1      owns TMEM (BN fp32 columns) and issues tcgen05.mma kind::f16
//               (bf16 × bf16 → f32), M = 128, N = BN, K = 16 per instruction;
//   warps 2-5   epilogue: thread ↔ row (TMEM lane), 32 columns per TMEM load,
//               bf16 (or, for a split-K slice, fp32 partials) to global memory.
// When M is small (decode: one token per sequence) the tile grid cannot fill
// the GPU, so K is split over S CTAs that write fp32 partial sums; a second
// kernel adds the S slices in a fixed order and rounds once to bf16.
// The head weights x·w_projᵀ (x bf16, w_proj fp32) run on the same tensor-core
// GEMM: every fp32 weight is split into three bf16 parts, hi = bf16(w),
// mid = bf16(w − hi), lo = bf16(w − hi − mid), which carry its 24 significand
// bits, so x·w = x·hi + x·mid + x·lo with every product exact in fp32.  The
// three parts are stacked as the 192 rows of one B operand; the epilogue adds
// the three column groups per head, (lo + mid) + hi, in fp32.
// Every wait is bounded; a CTA that gives up raises IDX_DEV_ERR_TIMEOUT,
// waits for its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "api_internal.h"
#include "ptx.cuh"

namespace idx {
namespace {

constexpr int kGemmM = 128;      // rows per CTA (TMEM lanes)
constexpr int kGemmK = 64;       // bf16 elements per K tile: one 128-byte swizzle row
constexpr int kGemmThreads = 192;

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                  // D format f32
         | (1u << 7) | (1u << 10)                   // A, B: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Two fp32 values rounded to nearest-even bf16, packed low | high << 16.
__device__ __forceinline__ uint32_t bf16_pair(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

struct GemmParams {
  int M, N, K;
  int k_tiles;             // K tiles per CTA (its split-K slice)
  void* out;               // bf16 [M, N] or fp32 partials [S, M, N]; GROUPS = 3: fp32 [M, N / 3] or [S, M, N / 3]
  int partial;             // write fp32 partials of this CTA's slice
  unsigned long long budget_ns;
  unsigned int* err;
};

template <int BN, int STAGES>
struct GemmCfg {
  static constexpr int kATile = kGemmM * kGemmK * 2;     // 16 KB
  static constexpr int kBTile = BN * kGemmK * 2;
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kOffBar = STAGES * kStage;
  static constexpr int kOffMisc = kOffBar + (2 * STAGES + 2) * 8;
  static constexpr int kSmem = 1024 + kOffMisc + 16;
  static constexpr int kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;   // a power of two
};

// grid: x = N / BN column tiles, y = row tiles, z = split-K slices.
// GROUPS = 1: C tile to bf16 (or fp32 partials).  GROUPS = 3: the BN columns are
// three stacked groups (weight parts hi, mid, lo); the output is their fp32 sum,
// BN / 3 columns wide, as the result (one slice) or as slice partials.
template <int BN, int STAGES, int GROUPS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const GemmParams p) {
  using C = GemmCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* drain_bar = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kGemmM;
  const int kt0 = blockIdx.z * p.k_tiles;
  const int nk = min(p.k_tiles, p.K / kGemmK - kt0);

  int issued = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    const int pre = nk < STAGES ? nk : STAGES;
    for (int t = 0; t < pre; ++t) {
      mbar_arrive_expect_tx(&full[t], C::kStage);
      tma_load_2d(smem + t * C::kStage, &tmap_a, &full[t], (kt0 + t) * kGemmK, m0);
      tma_load_2d(smem + t * C::kStage + C::kATile, &tmap_b, &full[t], (kt0 + t) * kGemmK, n0);
    }
    issued = pre;
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t budget = p.budget_ns;
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      int t = issued;
      for (; t < nk; ++t) {
        const int s = t % STAGES;
        if (!mbar_wait(&empty[s], ((t / STAGES) & 1) ^ 1, budget, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&full[s], C::kStage);
        tma_load_2d(smem + s * C::kStage, &tmap_a, &full[s], (kt0 + t) * kGemmK, m0);
        tma_load_2d(smem + s * C::kStage + C::kATile, &tmap_b, &full[s], (kt0 + t) * kGemmK, n0);
      }
      issued = t;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGemmM, BN);
      for (int t = 0; t < nk; ++t) {
        const int s = t % STAGES;
        if (!mbar_wait(&full[s], (t / STAGES) & 1, budget, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::kStage);
        const uint32_t b_addr = a_addr + C::kATile;
#pragma unroll
        for (int kk = 0; kk < kGemmK / 16; ++kk)   // 16 bf16 = 32 bytes per instruction
          mma_bf16(tmem_base, smem_desc_k128_sw128(a_addr + kk * 32), smem_desc_k128_sw128(b_addr + kk * 32), idesc,
                   (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_issued = true;
      }
      if (mma_issued) {
        mma_commit(acc_full);
        mma_commit(drain_bar);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = m0 + quad * 32 + lane;
    int ok = 1;
    if (lane == 0) ok = (nk > 0 && mbar_wait(acc_full, 0, budget, abort_flag, p.err)) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (ok) {
      tc_fence_after();
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      if constexpr (GROUPS == 3) {
        constexpr int kOut = BN / 3;
        static_assert(kOut % 32 == 0, "column groups of whole TMEM loads");
#pragma unroll 1
        for (int c = 0; c < kOut / 32; ++c) {
          float hi[32], mid[32], lo[32];
          tmem_ld32(lane_base + static_cast<uint32_t>(c * 32), hi);
          tmem_ld32(lane_base + static_cast<uint32_t>(kOut + c * 32), mid);
          tmem_ld32(lane_base + static_cast<uint32_t>(2 * kOut + c * 32), lo);
          if (row < p.M) {
            float* dst = static_cast<float*>(p.out) + (static_cast<int64_t>(blockIdx.z) * p.M + row) * kOut + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) =
                  make_float4((lo[i] + mid[i]) + hi[i], (lo[i + 1] + mid[i + 1]) + hi[i + 1],
                              (lo[i + 2] + mid[i + 2]) + hi[i + 2], (lo[i + 3] + mid[i + 3]) + hi[i + 3]);
          }
        }
      } else {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(lane_base + static_cast<uint32_t>(c * 32), v);
        if (row < p.M) {
          if (p.partial) {
            float* dst = static_cast<float*>(p.out) +
                         (static_cast<int64_t>(blockIdx.z) * p.M + row) * p.N + n0 + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          } else {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N + n0 + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 u;
              u.x = bf16_pair(v[i], v[i + 1]);
              u.y = bf16_pair(v[i + 2], v[i + 3]);
              u.z = bf16_pair(v[i + 4], v[i + 5]);
              u.w = bf16_pair(v[i + 6], v[i + 7]);
              *reinterpret_cast<uint4*>(dst + i) = u;
            }
          }
        }
      }
      }
    }
  }
  __syncthreads();
  // ------------------------------------------------------------ teardown
  if (warp == 0 && lane == 0) {
    int dummy = 0;
    for (int t = max(0, issued - STAGES); t < issued; ++t)
      mbar_wait(&full[t % STAGES], (t / STAGES) & 1, budget, &dummy, p.err);
  }
  if (warp == 1 && lane == 0 && mma_issued) {
    int dummy = 0;
    mbar_wait(drain_bar, 0, budget, &dummy, p.err);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// out[i] = Σ_s part[s, i], slices added in order s = 0, 1, …, then rounded
// once to the output type (bf16 to nearest-even, or kept fp32).
template <typename OutT>
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int S, int64_t MN, OutT* __restrict__ out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < MN;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float acc = part[i];
    for (int s = 1; s < S; ++s) acc += part[s * MN + i];
    if constexpr (sizeof(OutT) == 2)
      out[i] = __float2bfloat16_rn(acc);
    else
      out[i] = acc;
  }
}

// w_proj [64, hidden] fp32 → three bf16 parts [3][64][hidden]: hi = bf16(w),
// mid = bf16(w − hi), lo = bf16(w − hi − mid).  Both differences are exact in
// fp32 (each subtracts a rounding of the value itself, Sterbenz), and the last
// rounding is of a remainder below 2⁻¹⁶·|w|, so hi + mid + lo = w within 2⁻²⁴·|w|.
__global__ void split_weights_kernel(const float* __restrict__ w, int64_t count, __nv_bfloat16* __restrict__ parts) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    parts[i] = hi;
    parts[count + i] = mid;
    parts[2 * count + i] = __float2bfloat16_rn(r2);
  }
}

int grid_for(int64_t count) {
  const int64_t b = (count + 255) / 256;
  return static_cast<int>(b < 148 * 8 ? b : 148 * 8);
}

// Split of K for an M × N product: enough CTAs to cover the SMs, slices of at
// least 4 K tiles; every slice gets ceil(k_tiles / S) tiles and S is then
// trimmed so that no slice is empty.
void split_k(int64_t tiles_mn, int k_tiles, int sms, int& S, int& per) {
  S = 1;
  while (tiles_mn * S * 2 <= sms && k_tiles / (S * 2) >= 4) S *= 2;
  per = (k_tiles + S - 1) / S;
  S = (k_tiles + per - 1) / per;
}

// Column tile of a bf16 projection: 256 when the tiles alone fill the GPU.
int column_tile(int64_t M, int N, int sms) {
  const int64_t row_tiles = (M + kGemmM - 1) / kGemmM;
  if (N % 256 == 0 && row_tiles * (N / 256) >= sms) return 256;
  return N % 128 == 0 ? 128 : 64;
}

// fp32 partial sums one bf16 projection needs (0 without split-K).
size_t partial_floats(int64_t M, int N, int K, int sms) {
  const int BN = column_tile(M, N, sms);
  int S, per;
  split_k(((M + kGemmM - 1) / kGemmM) * (N / BN), K / kGemmK, sms, S, per);
  return S > 1 ? static_cast<size_t>(S) * static_cast<size_t>(M) * static_cast<size_t>(N) : 0;
}

template <int BN, int GROUPS>
int launch_gemm(const uint16_t* A, const uint16_t* Bw, int64_t M, int N, int K, void* out, float* part, int S,
                int per, cudaStream_t stream) {
  constexpr int STAGES = 4;
  using C = GemmCfg<BN, STAGES>;
  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16_sw128(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kGemmM))
    return IDX_ERR_ALIGN;
  if (!make_tmap_2d_bf16_sw128(&tb, Bw, static_cast<uint64_t>(K), static_cast<uint64_t>(N), BN)) return IDX_ERR_ALIGN;
  auto kern = gemm_bf16_kernel<BN, STAGES, GROUPS>;
  if (const int r = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::kSmem)) return r;
  GemmParams p;
  p.M = static_cast<int>(M);
  p.N = N;
  p.K = K;
  p.k_tiles = per;
  p.partial = S > 1 ? 1 : 0;
  p.out = S > 1 ? static_cast<void*>(part) : out;
  const DebugState dbg = debug_state();
  p.budget_ns = dbg.budget_ns;
  p.err = device_error_word();
  if (!p.err) return check_launch();
  const dim3 grid(static_cast<unsigned>(N / BN), static_cast<unsigned>((M + kGemmM - 1) / kGemmM),
                  static_cast<unsigned>(S));
  kern<<<grid, kGemmThreads, C::kSmem, stream>>>(ta, tb, p);
  if (const int r = check_launch()) return r;
  if (S > 1) {
    const int64_t MN = M * (N / GROUPS);
    if constexpr (GROUPS == 1)
      splitk_reduce_kernel<<<grid_for(MN), 256, 0, stream>>>(part, S, MN, static_cast<__nv_bfloat16*>(out));
    else
      splitk_reduce_kernel<<<grid_for(MN), 256, 0, stream>>>(part, S, MN, static_cast<float*>(out));
    return check_launch();
  }
  return IDX_OK;
}

// The split-K slices of one product: as split_k proposes, then fewer while the
// partial sums (M × out_cols fp32 per slice) would not fit in part_floats.
void slices_for(int64_t M, int N, int BN, int out_cols, int K, size_t part_floats, int& S, int& per) {
  const int k_tiles = K / kGemmK;
  split_k(((M + kGemmM - 1) / kGemmM) * (N / BN), k_tiles, num_sms(), S, per);
  while (S > 1 && static_cast<size_t>(S) * static_cast<size_t>(M) * out_cols > part_floats) {
    per *= 2;
    S = (k_tiles + per - 1) / per;
  }
  if (S <= 1) {
    S = 1;
    per = k_tiles;
  }
}

// One bf16 projection: the column tile and the split-K slices for this shape.
int project_bf16(const uint16_t* A, const uint16_t* Bw, int64_t M, int N, int K, uint16_t* out, float* part,
                 size_t part_floats, cudaStream_t stream) {
  const int BN = column_tile(M, N, num_sms());
  int S, per;
  slices_for(M, N, BN, N, K, part_floats, S, per);
  switch (BN) {
    case 256: return launch_gemm<256, 1>(A, Bw, M, N, K, out, part, S, per, stream);
    case 128: return launch_gemm<128, 1>(A, Bw, M, N, K, out, part, S, per, stream);
    default: return launch_gemm<64, 1>(A, Bw, M, N, K, out, part, S, per, stream);
  }
}

constexpr int kHeadCols = 3 * IDX_HEADS;   // the stacked weight parts: one 192-column tile

// Bytes of the three bf16 weight parts, rounded up to keep what follows aligned.
size_t weight_parts_bytes(int hidden) {
  return (static_cast<size_t>(kHeadCols) * static_cast<size_t>(hidden) * 2 + 255) & ~static_cast<size_t>(255);
}

}  // namespace
}  // namespace idx

using namespace idx;

extern "C" size_t idx_project_workspace_size(int64_t tokens, int hidden, int q_lora) {
  if (tokens <= 0 || hidden <= 0 || q_lora <= 0 || hidden % kGemmK || q_lora % kGemmK) return 0;
  const int sms = num_sms();
  const size_t q = partial_floats(tokens, IDX_HEADS * IDX_DIM, q_lora, sms);
  const size_t k = partial_floats(tokens, IDX_DIM, hidden, sms);
  int S, per;
  split_k((tokens + kGemmM - 1) / kGemmM, hidden / kGemmK, sms, S, per);
  const size_t w = S > 1 ? static_cast<size_t>(S) * static_cast<size_t>(tokens) * IDX_HEADS : 0;
  size_t m = q > k ? q : k;
  m = m > w ? m : w;
  return weight_parts_bytes(hidden) + m * sizeof(float);
}

extern "C" int idx_project(const uint16_t* x, const uint16_t* qr, int64_t tokens, int hidden, int q_lora,
                           const uint16_t* wq_b, const uint16_t* wk, const float* w_proj, uint16_t* q_proj,
                           uint16_t* k_proj, float* w_raw, void* ws, size_t ws_bytes, idx_stream_t stream) {
  if (tokens < 0 || hidden <= 0 || q_lora <= 0) return IDX_ERR_SHAPE;
  if (hidden % kGemmK || q_lora % kGemmK) return IDX_ERR_SHAPE;
  if (tokens == 0) return IDX_OK;
  if (!x || !qr || !wq_b || !wk || !w_proj || !q_proj || !k_proj || !w_raw || !ws) return IDX_ERR_NULL;
  if (tokens > 0x7FFFFFFF / IDX_HEADS / IDX_DIM) return IDX_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(qr) | reinterpret_cast<uintptr_t>(wq_b) |
       reinterpret_cast<uintptr_t>(wk) | reinterpret_cast<uintptr_t>(q_proj) | reinterpret_cast<uintptr_t>(k_proj) |
       reinterpret_cast<uintptr_t>(w_raw) | reinterpret_cast<uintptr_t>(ws)) & 15)
    return IDX_ERR_ALIGN;
  const size_t parts_bytes = weight_parts_bytes(hidden);
  if (ws_bytes < idx_project_workspace_size(tokens, hidden, q_lora)) return IDX_ERR_SCRATCH;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint16_t* parts = static_cast<uint16_t*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + parts_bytes);
  const size_t part_floats = (ws_bytes - parts_bytes) / sizeof(float);
  const int64_t wcount = static_cast<int64_t>(IDX_HEADS) * hidden;
  split_weights_kernel<<<grid_for(wcount), 256, 0, s>>>(w_proj, wcount, reinterpret_cast<__nv_bfloat16*>(parts));
  int r = check_launch();
  if (r != IDX_OK) return r;
  r = project_bf16(qr, wq_b, tokens, IDX_HEADS * IDX_DIM, q_lora, q_proj, part, part_floats, s);
  if (r != IDX_OK) return r;
  r = project_bf16(x, wk, tokens, IDX_DIM, hidden, k_proj, part, part_floats, s);
  if (r != IDX_OK) return r;
  int S, per;
  slices_for(tokens, kHeadCols, kHeadCols, IDX_HEADS, hidden, part_floats, S, per);
  return launch_gemm<kHeadCols, 3>(x, parts, tokens, kHeadCols, hidden, w_raw, part, S, per, s);
}
