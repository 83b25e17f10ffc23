// W4A16 product for batches of activation rows (n > 16) on the tcgen05 tensor cores.
//
// "GPTQ second-order quantization" blog, "What the original results established" (W4A16: BF16
// activations, the weights moved as packed 4-bit codes and dequantized inside the kernel) and
// "Group-wise quantization" (one scale and zero point per row or per group of input channels).
// Where the decode-size product (w4a16.cu) is a matrix-vector product, a batch of activation rows
// makes it a matrix product, which belongs on the tensor cores:
//   Y[n][r] = sum_c X[n][c] s[r, g(c)] (q[r][c] - z[r, g(c)]).
//
// A CTA owns 128 weight rows (the MMA's M) and a tile of up to N activation rows (the MMA's N) and
// walks the columns in chunks of 128 (one group at group size 128):
//   warp 0     TMA: the chunk's activations (N rows x 128 bf16, 128-byte swizzle, K-major) and its
//              packed codes (128 rows x 64 bytes, 64-byte swizzle) into a ring of 4-6 stages,
//              deep enough to cover the load latency;
//   warps 2-..  dequantize (4 warps, or 8 when the activation tile is small): each thread turns
//              its share of a weight row's 128 codes into q - z, exact in bf16, and writes them
//              K-major with the 128-byte swizzle into one of two A tiles, the MMA's A operand;
//   warp 1     MMA: D[r][n] = sum over the chunk of (q - z)[r][k] X[n][k], eight 128 x N x 16
//              bf16 MMAs into one of two TMEM buffers, fp32;
//   warps 6-9  fold: each thread (one weight row, a TMEM lane) adds s[r, g] D[r][:] into fp32
//              registers, so every chunk is scaled by its own group's scale in fp32 and the chunks
//              are added in order (deterministic); at the end it writes its column of Y, 32
//              consecutive outputs per warp store.
// Products of bf16 X and the small integers q - z are exact in fp32; a chunk's sum takes eight
// tensor-core accumulations, which is all the accumulator rounding a result sees per chunk.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace gptq {
namespace {

namespace wg {
constexpr int kM = 128;                      // weight rows per CTA
constexpr int kK = 128;                      // columns per chunk
constexpr int kABytes = kM * kK * 2;         // q - z, bf16: two halves of 128 rows x 128 B
constexpr int kCodeBytes = kM * kK / 2;      // packed codes of the chunk: 128 rows x 64 B
template <int N>
struct Cfg {
  // the activation / code ring (small stages, deep) and two dequantized A tiles
  static constexpr int kStages = N <= 64 ? 6 : 4;
  static constexpr int kDqWarps = N <= 64 ? 8 : 4;               // dequantizing warps
  static constexpr int kDqThreads = 32 * kDqWarps;
  static constexpr int kThreads = 32 * (2 + kDqWarps + 4);       // TMA, MMA, dequantize, fold
  static constexpr int kFoldWarp0 = 2 + kDqWarps;
  static constexpr int kXBytes = N * kK * 2;                     // two halves of N rows x 128 B
  static constexpr int kStageBytes = kXBytes + kCodeBytes;
  static constexpr int kSmem = 2 * kABytes + kStages * kStageBytes + 1024;
  static constexpr uint32_t kTmemCols = 2 * N;                   // two accumulator buffers
};
}  // namespace wg

template <int N>
__global__ void __launch_bounds__(wg::Cfg<N>::kThreads, 1)
w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tcodes, const __grid_constant__ CUtensorMap tx,
                  int64_t rows, int64_t cols, const float* __restrict__ scales,
                  const uint8_t* __restrict__ zeros, int G, int chunks_per_group, int64_t n,
                  float* __restrict__ Y, int64_t ldy, int32_t* info) {
  // gridDim.z == 2 splits the chunks in two halves whose results are added into a zeroed Y: a sum
  // of exactly two terms onto zero is the same whichever lands first.
  using namespace wg;
  using C = Cfg<N>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  // A tiles b = 0, 1 (32 KB each), then ring stage s: X (N x 256 B) | codes (8 KB); every part
  // 1024-byte aligned
  auto a_tile = [&](int b) { return smem + b * kABytes; };
  auto x_tile = [&](int s) { return smem + 2 * kABytes + s * C::kStageBytes; };
  auto c_tile = [&](int s) { return smem + 2 * kABytes + s * C::kStageBytes + C::kXBytes; };
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t a_full[2], a_empty[2];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * N;
  const int all_chunks = static_cast<int>((cols + kK - 1) / kK);
  const int c_begin = static_cast<int>(static_cast<int64_t>(all_chunks) * blockIdx.z / gridDim.z);
  const int c_end = static_cast<int>(static_cast<int64_t>(all_chunks) * (blockIdx.z + 1) / gridDim.z);
  const int nchunks = c_end - c_begin;    // this CTA's chunks c_begin .. c_end - 1
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_full[b], C::kDqThreads);
      mbar_init(&a_empty[b], 1);
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int c = 0; c < nchunks && !abort_flag; ++c) {
        const int s = c % kStages;
        const uint32_t ph = static_cast<uint32_t>((c / kStages) & 1);
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag, info)) break;
        mbar_arrive_expect_tx(&full_bar[s], C::kXBytes + kCodeBytes);
        const int cc = c_begin + c;
        tma_load_2d(x_tile(s), &tx, &full_bar[s], cc * kK, static_cast<int>(n0));
        tma_load_2d(x_tile(s) + N * 128, &tx, &full_bar[s], cc * kK + 64, static_cast<int>(n0));
        tma_load_2d(c_tile(s), &tcodes, &full_bar[s], cc * (kK / 8), static_cast<int>(r0));
        ++issued;
      }
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_drain_bounded(&full_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(/*bf16*/ 1, 0, 0, kM, N);
      for (int c = 0; c < nchunks && !abort_flag; ++c) {
        const int s = c % kStages, buf = c & 1;   // buf: the A tile and the TMEM buffer
        const uint32_t ph = static_cast<uint32_t>((c / kStages) & 1);
        if (!mbar_wait_bounded(&a_full[buf], (c >> 1) & 1, &abort_flag, info)) break;
        if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, info)) break;
        if (!mbar_wait_bounded(&acc_empty[buf], ((c >> 1) & 1) ^ 1u, &abort_flag, info)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(a_tile(buf)), x_addr = smem_u32(x_tile(s));
        const uint32_t d = tmem + static_cast<uint32_t>(buf * N);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = smem_desc(a_addr + h * (kM * 128) + kk * 32, 16, 1024,
                                             kSwizzle128B);
            const uint64_t bdesc = smem_desc(x_addr + h * (N * 128) + kk * 32, 16, 1024,
                                             kSwizzle128B);
            tc_mma_f16(d, adesc, bdesc, idesc, (h | kk) ? 1u : 0u);
          }
        tc_commit(&empty_bar[s]);       // the stage's activations and codes are done with
        tc_commit(&a_empty[buf]);       // the A tile may be rewritten
        tc_commit(&acc_full[buf]);
      }
      tc_commit(&mma_done);
      mbar_drain_bounded(&mma_done, 0);
    }
  } else if (warp < C::kFoldWarp0) {
    // ---- dequantize: thread t owns weight row i = t % 128 of the chunk; with eight warps, two
    // threads share a row, one per 64-column half ----
    constexpr int kHalves = C::kDqThreads / 128;          // 1 or 2 threads per row
    const int t = threadIdx.x - 64;
    const int i = t % 128, hpart = t / 128;
    const int64_t r = r0 + i;
    const bool live = r < rows;
    // the zero point of each chunk's group, fetched one chunk ahead
    auto zero_of = [&](int c) -> uint32_t {
      return live ? static_cast<uint32_t>(zeros[r * G + (c_begin + c) / chunks_per_group]) : 0u;
    };
    uint32_t z_next = nchunks > 0 ? zero_of(0) : 0u;
    for (int c = 0; c < nchunks && !abort_flag; ++c) {
      const int s = c % kStages, b = c & 1;
      const uint32_t ph = static_cast<uint32_t>((c / kStages) & 1);
      const uint32_t z = z_next;
      if (c + 1 < nchunks) z_next = zero_of(c + 1);
      const uint32_t zz = (0x4300u | z) | ((0x4300u | z) << 16);   // bf16x2 of 128 + z
      if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, info)) break;
      // the A tile of chunk c - 2 must have been read by its MMAs
      if (!mbar_wait_bounded(&a_empty[b], ((c >> 1) & 1) ^ 1u, &abort_flag, info)) break;
      // the codes tile arrives with the 64-byte swizzle: 16-byte chunk q of row i sits at
      // chunk q ^ ((i / 2) % 4), so a warp's reads of one chunk index spread over all banks
      const uint8_t* crow = c_tile(s) + i * 64;
      const int sw = (i >> 1) & 3;
      uint8_t* dst = a_tile(b) + i * 128;
      const __nv_bfloat162 zb = *reinterpret_cast<const __nv_bfloat162*>(&zz);
#pragma unroll
      for (int qq = 0; qq < 4 / kHalves; ++qq) {
        const int q4 = hpart * (4 / kHalves) + qq;
        const uint4 cw = *reinterpret_cast<const uint4*>(crow + ((q4 ^ sw) << 4));
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int w = 4 * q4 + e;           // columns 8w .. 8w + 7 of the chunk
          const uint32_t lo = words[e] & 0x0F0F0F0Fu;          // codes 0, 2, 4, 6
          const uint32_t hi = (words[e] >> 4) & 0x0F0F0F0Fu;   // codes 1, 3, 5, 7
          const uint32_t t01 = __byte_perm(lo, hi, 0x5140);    // codes 0, 1, 2, 3
          const uint32_t t23 = __byte_perm(lo, hi, 0x7362);    // codes 4, 5, 6, 7
          // bf16 pairs (128 + q, 128 + q'): the byte 0x43 above each code
          uint32_t p[4] = {__byte_perm(t01, 0x43434343u, 0x4140),
                           __byte_perm(t01, 0x43434343u, 0x4342),
                           __byte_perm(t23, 0x43434343u, 0x4140),
                           __byte_perm(t23, 0x43434343u, 0x4342)};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const __nv_bfloat162 d2 = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&p[k]), zb);
            p[k] = *reinterpret_cast<const uint32_t*>(&d2);
          }
          // K-major, 128-byte swizzle: half w / 8, 16-byte chunk (w % 8) ^ (row % 8)
          *reinterpret_cast<uint4*>(dst + (w >> 3) * (kM * 128) +
                                    (((w & 7) ^ (i & 7)) << 4)) = make_uint4(p[0], p[1], p[2], p[3]);
        }
      }
      fence_proxy_async_smem();              // the tensor core reads these writes
      mbar_arrive(&a_full[b]);
    }
  } else {
    // ---- fold (the last four warps): thread = weight row r0 + 32 (warp % 4) + lane = its TMEM
    // lane ----
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    const int64_t r = r0 + rl;
    const bool live = r < rows;
    float acc[N];
#pragma unroll
    for (int j = 0; j < N; ++j) acc[j] = 0.f;
    bool ok = true;
    auto scale_of = [&](int c) -> float {
      return live ? scales[r * G + (c_begin + c) / chunks_per_group] : 0.f;
    };
    float s_next = nchunks > 0 ? scale_of(0) : 0.f;
    for (int c = 0; c < nchunks; ++c) {
      const int buf = c & 1;
      const float sc = s_next;
      if (c + 1 < nchunks) s_next = scale_of(c + 1);
      if (!mbar_wait_bounded(&acc_full[buf], (c >> 1) & 1, &abort_flag, info)) { ok = false; break; }
      tc_fence_after();
      const uint32_t t = tmem + static_cast<uint32_t>(buf * N) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < N / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t + cc * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[cc * 32 + j] = fmaf(sc, __uint_as_float(v[j]), acc[cc * 32 + j]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    if (ok && live) {
      // column r of Y: for each activation row, the warp's 32 lanes write 32 consecutive floats
      if (gridDim.z == 1) {
#pragma unroll
        for (int j = 0; j < N; ++j)
          if (n0 + j < n) Y[(n0 + j) * ldy + r] = acc[j];
      } else {
#pragma unroll
        for (int j = 0; j < N; ++j)
          if (n0 + j < n) atomicAdd(Y + (n0 + j) * ldy + r, acc[j]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int N>
gptq_status launch_gemm(const CUtensorMap& tcodes, const CUtensorMap& tx, int64_t rows,
                        int64_t cols, const float* scales, const uint8_t* zeros, int G,
                        int chunks_per_group, int64_t n, float* y, int64_t ldy, int32_t* info,
                        cudaStream_t stream) {
  using C = wg::Cfg<N>;
  const gptq_status st =
      set_max_dynamic_smem(reinterpret_cast<const void*>(w4a16_gemm_kernel<N>), C::kSmem);
  if (st != GPTQ_OK) return st;
  const int64_t gx = (rows + wg::kM - 1) / wg::kM, gy = (n + N - 1) / N;
  if (gx > INT_MAX || gy > 65535) return GPTQ_EUNSUPPORTED;
  // twice the tiles still fit one CTA per SM: two CTAs per tile, each on half of the columns,
  // adding into a zeroed Y
  const int64_t nchunks = (cols + wg::kK - 1) / wg::kK;
  const int gz = (2 * gx * gy <= num_sms() && nchunks >= 4) ? 2 : 1;
  if (gz == 2 && cudaMemset2DAsync(y, static_cast<size_t>(ldy) * 4, 0,
                                   static_cast<size_t>(rows) * 4, static_cast<size_t>(n),
                                   stream) != cudaSuccess)
    return GPTQ_ECUDA;
  return launch_pdl(w4a16_gemm_kernel<N>,
                    dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), gz),
                    dim3(C::kThreads), C::kSmem, stream, tcodes, tx, rows, cols, scales, zeros,
                    G, chunks_per_group, n, y, ldy, info);
}

}  // namespace

gptq_status run_w4a16_gemm(const uint32_t* packed, const float* scales, const uint8_t* zeros,
                           int64_t rows, int64_t cols, int group, const void* x, int64_t n,
                           int64_t ldx, float* y, int64_t ldy, int32_t* info,
                           cudaStream_t stream) {
  // activation tile: 32, 64 or 128 rows (rows past n arrive as zeros and are not stored)
  const int N = n <= 32 ? 32 : n <= 64 ? 64 : 128;
  CUtensorMap tcodes, tx;
  gptq_status st = encode_tmap_2d(&tcodes, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, 4, cols / 8,
                                  rows, cols / 8, wg::kK / 8, wg::kM, CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != GPTQ_OK) return st;
  st = encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, 2, cols, n, ldx, 64, N,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GPTQ_OK) return st;
  const int G = group > 0 ? static_cast<int>(cols / group) : 1;
  const int cpg = group > 0 ? group / wg::kK : INT_MAX;
  switch (N) {
    case 32:
      return launch_gemm<32>(tcodes, tx, rows, cols, scales, zeros, G, cpg, n, y, ldy, info,
                             stream);
    case 64:
      return launch_gemm<64>(tcodes, tx, rows, cols, scales, zeros, G, cpg, n, y, ldy, info,
                             stream);
    default:
      return launch_gemm<128>(tcodes, tx, rows, cols, scales, zeros, G, cpg, n, y, ldy, info,
                              stream);
  }
}

}  // namespace gptq
