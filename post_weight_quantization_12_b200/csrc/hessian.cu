// S1 -- proxy Hessian accumulation S += X^T X (lower triangle), X token-major [n_tokens x ldx].
//
// "Part 2: Adaptive Rounding: Optimal Brain Quantizer (OBQ)", section "Goal": the input covariance
// is the proxy Hessian; "Part 3: Adaptive Rounding: GPTQ", "Algorithm GPTQ": H = X X^T + lambda I.
//
// bf16 path: a persistent tcgen05 SYRK. Output is cut into 256 x 256 lower-triangle super-tiles;
// each CTA owns one super-tile per round and walks the whole token range for it, so all CTAs read
// the same token slab at about the same time (the slab is fetched from HBM once and served to the
// others from L2). Per 32-token stage, TMA brings the 256-channel slabs of X for the tile's rows (A)
// and columns (B) into shared memory with 128-byte swizzle; both operands are MN-major (channels
// contiguous), which tcgen05 reads directly. One thread issues 2 x 2 MMAs of 128 x 256 x 16 into two
// TMEM accumulators (the super-tile's upper and lower 128-row halves, 512 TMEM columns). Four
// epilogue warps drain TMEM and add the tile into S; each super-tile belongs to one CTA, so the
// result is deterministic and needs no atomics.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace syrk {
constexpr int kBK = 32;                    // tokens per stage
constexpr int kStages = 6;
constexpr int kBoxCh = 64;                 // channels per TMA box (128 bytes of bf16)
constexpr int kBoxBytes = kBoxCh * kBK * 2;          // 4 KB
constexpr int kSlabBytes = 4 * kBoxBytes;            // 256 channels x 32 tokens = 16 KB
constexpr int kStageBytes = 2 * kSlabBytes;          // A slab + B slab
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kThreads = 192;              // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t kTmemCols = 512;
// The tensor core adds each 16-deep product into the fp32 accumulator with a rounding that is
// biased toward zero, so the relative error of a TMEM sum grows with the number of MMAs folded
// into it (about 6e-8 per MMA measured on B200). Every kKbPerFlush stages (2048 tokens) the
// chunk sum is added into S with IEEE fp32 adds and the accumulator restarts.
constexpr int kKbPerFlush = 64;
constexpr uint32_t kIdesc = make_idesc(/*bf16*/ 1, /*A MN-major*/ 1, /*B MN-major*/ 1, 128, 256);
}  // namespace syrk

__device__ __forceinline__ void decode_lower(int st, int& I, int& J) {
  int i = static_cast<int>((sqrtf(8.0f * static_cast<float>(st) + 1.0f) - 1.0f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= st) ++i;
  while (i * (i + 1) / 2 > st) --i;
  I = i;
  J = st - i * (i + 1) / 2;
}

__global__ void __launch_bounds__(syrk::kThreads, 1)
hessian_syrk_bf16_tc(const __grid_constant__ CUtensorMap tmap, float* __restrict__ S, int cols,
                     int n_kblocks, int kb_per_flush, int n_super, int32_t* info) {
  using namespace syrk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full, acc_empty, mma_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 128);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmap);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      for (int st = blockIdx.x; st < n_super && !abort_flag; st += gridDim.x) {
        int I, J;
        decode_lower(st, I, J);
        const bool diag = (I == J);
        for (int kb = 0; kb < n_kblocks; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag, info)) goto producer_done;
          uint8_t* a = smem + s * kStageBytes;
          uint8_t* b = a + kSlabBytes;
          mbar_arrive_expect_tx(&full_bar[s], diag ? kSlabBytes : kStageBytes);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tma_load_2d(a + q * kBoxBytes, &tmap, &full_bar[s], I * 256 + q * kBoxCh, kb * kBK);
          if (!diag) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tma_load_2d(b + q * kBoxBytes, &tmap, &full_bar[s], J * 256 + q * kBoxCh, kb * kBK);
          }
          ++issued;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
    producer_done:
      // Let every copy already issued land before the CTA can exit.
      for (long long i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_drain_bounded(&full_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int s = 0;
      uint32_t ph = 0, aph = 0;
      for (int st = blockIdx.x; st < n_super && !abort_flag; st += gridDim.x) {
        int I, J;
        decode_lower(st, I, J);
        const bool diag = (I == J);
        for (int kc = 0; kc < n_kblocks; kc += kb_per_flush) {
          // a fresh chunk sum in TMEM; the epilogue folds it into S with IEEE fp32 adds
          if (!mbar_wait_bounded(&acc_empty, aph ^ 1u, &abort_flag, info)) goto mma_done_label;
          tc_fence_after();
          const int kc_end = min(n_kblocks, kc + kb_per_flush);
          for (int kb = kc; kb < kc_end; ++kb) {
            if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, info)) goto mma_done_label;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
            const uint32_t b_addr = diag ? a_addr : a_addr + kSlabBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t bdesc = smem_desc(b_addr + kk * 2048, kBoxBytes, 1024, kSwizzle128B);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint64_t adesc = smem_desc(a_addr + 2 * h * kBoxBytes + kk * 2048, kBoxBytes,
                                                 1024, kSwizzle128B);
                tc_mma_f16(tmem + h * 256, adesc, bdesc, kIdesc, (kb > kc || kk > 0) ? 1u : 0u);
              }
            }
            tc_commit(&empty_bar[s]);
            if (++s == kStages) { s = 0; ph ^= 1u; }
          }
          tc_commit(&acc_full);
          aph ^= 1u;
        }
      }
    mma_done_label:
      tc_commit(&mma_done);
      mbar_drain_bounded(&mma_done, 0);
    }
  } else {
    // ---------------- epilogue: TMEM -> S (read-add-write, lower super-tile) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r_in_half = q * 32 + lane;
    uint32_t aph = 0;
    for (int st = blockIdx.x; st < n_super && !abort_flag; st += gridDim.x) {
      int I, J;
      decode_lower(st, I, J);
      for (int kc = 0; kc < n_kblocks; kc += kb_per_flush) {
        if (!mbar_wait_bounded(&acc_full, aph, &abort_flag, info)) goto epilogue_done;
        tc_fence_after();
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int i = I * 256 + h * 128 + r_in_half;
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 256 + c * 32, v);
            tmem_wait_ld();
            const int j0 = J * 256 + c * 32;
            if (i < cols) {
              float4* row = reinterpret_cast<float4*>(S + static_cast<size_t>(i) * cols + j0);
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                if (j0 + 4 * t < cols) {
                  float4 o = row[t];
                  o.x += __uint_as_float(v[4 * t + 0]);
                  o.y += __uint_as_float(v[4 * t + 1]);
                  o.z += __uint_as_float(v[4 * t + 2]);
                  o.w += __uint_as_float(v[4 * t + 3]);
                  row[t] = o;
                }
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty);
        aph ^= 1u;
      }
    }
  epilogue_done:;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// fp32 inputs: CUDA-core SYRK on 64 x 64 lower tiles with the token range split over blockIdx.y;
// partial tiles are added into S with atomics (exact fp32 products, fp32 sums).
__global__ void __launch_bounds__(256)
hessian_syrk_f32_simt(const float* __restrict__ X, int64_t ldx, float* __restrict__ S, int cols,
                      int64_t n_tokens, int64_t tok_per_split) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  int I, J;
  decode_lower(blockIdx.x, I, J);
  const int i0 = I * 64, j0 = J * 64;
  const int64_t t_begin = static_cast<int64_t>(blockIdx.y) * tok_per_split;
  const int64_t t_end = min(n_tokens, t_begin + tok_per_split);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int64_t t0 = t_begin; t0 < t_end; t0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int kk = e >> 6, c = e & 63;
      const int64_t t = t0 + kk;
      const bool tok_ok = t < t_end;
      As[kk][c] = (tok_ok && i0 + c < cols) ? X[t * ldx + i0 + c] : 0.f;
      Bs[kk][c] = (tok_ok && j0 + c < cols) ? X[t * ldx + j0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kk][ty * 4 + u];
        b[u] = Bs[kk][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= cols) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int j = j0 + tx * 4 + v;
      if (j < cols) atomicAdd(S + static_cast<size_t>(i) * cols + j, acc[u][v]);
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------------

gptq_status launch_hessian_bf16(float* S, int64_t cols, const void* X, int64_t n_tokens,
                                int64_t ldx, int32_t* info, cudaStream_t stream) {
  using namespace syrk;
  CUtensorMap tmap;
  gptq_status st = encode_tmap_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, 2,
                                  static_cast<uint64_t>(cols), static_cast<uint64_t>(n_tokens),
                                  static_cast<uint64_t>(ldx), kBoxCh, kBK,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GPTQ_OK) return st;
  static bool attr_done = false;  // benign race: setting the same attribute twice is harmless
  if (!attr_done) {
    if (cudaFuncSetAttribute(hessian_syrk_bf16_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
      return GPTQ_ECUDA;
    attr_done = true;
  }
  const int n_s = static_cast<int>((cols + 255) / 256);
  const int n_super = n_s * (n_s + 1) / 2;
  const int64_t n_kb = (n_tokens + kBK - 1) / kBK;
  if (n_kb > INT32_MAX / kBK) return GPTQ_EUNSUPPORTED;
  const int grid = n_super < num_sms() ? n_super : num_sms();
  hessian_syrk_bf16_tc<<<grid, kThreads, kSmemBytes, stream>>>(
      tmap, S, static_cast<int>(cols), static_cast<int>(n_kb), kKbPerFlush, n_super, info);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

gptq_status launch_hessian_f32(float* S, int64_t cols, const float* X, int64_t n_tokens,
                               int64_t ldx, cudaStream_t stream) {
  const int n_t = static_cast<int>((cols + 63) / 64);
  const int n_tiles = n_t * (n_t + 1) / 2;
  // enough splits to give every SM a few CTAs, each with at least 256 tokens
  int64_t splits = (4 * num_sms() + n_tiles - 1) / n_tiles;
  const int64_t max_splits = (n_tokens + 255) / 256;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  if (splits > 65535) splits = 65535;
  int64_t per = (n_tokens + splits - 1) / splits;
  per = (per + 15) / 16 * 16;
  splits = (n_tokens + per - 1) / per;
  dim3 grid(n_tiles, static_cast<unsigned>(splits));
  hessian_syrk_f32_simt<<<grid, 256, 0, stream>>>(X, ldx, S, static_cast<int>(cols), n_tokens, per);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

}  // namespace gptq
