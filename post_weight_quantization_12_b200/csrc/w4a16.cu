// Packed 4-bit weights and the W4A16 product that consumes them.
//
// "GPTQ second-order quantization" blog, "What the original results established": GPTQ is
// weight-only; in the W4A16 path the activations stay BF16 and the speed comes from moving fewer
// weight bytes through a kernel that unpacks and dequantizes them ("Group-wise quantization": one
// scale and zero point per row or per group of input channels, with the group size traded against
// scale traffic). The product is HBM-bound: every weight code is read once, so the kernel is built
// around keeping enough code bytes in flight (a TMA ring per warp) and spending as few
// instructions per weight as possible (two-code-at-a-time dequantization, tensor-core dot
// products).
//
// Layout of the packed codes: eight codes per little-endian 32-bit word, row after row; code
// (r, c) sits in bits 4 (c mod 8) .. 4 (c mod 8) + 3 of word (r, c div 8). Packed 3-bit codes (for
// 3-bit grids): 32 codes per three words, the group's codes forming one 96-bit little-endian
// number, code (r, c) in its bits 3 (c mod 32) .. 3 (c mod 32) + 2; the group of columns 32k ..
// 32k + 31 of row r is words 3k .. 3k + 2 of the row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace gptq {
namespace {

// ------------------------------------------------------------------------------------------------
// Packing
// ------------------------------------------------------------------------------------------------

// Eight codes (bytes of x: codes 0 .. 3, of y: codes 4 .. 7) -> one word whose byte i holds codes
// 2i (low nibble) and 2i + 1 (high nibble).
__device__ __forceinline__ uint32_t pack8_4bit(uint32_t x, uint32_t y) {
  const uint32_t a = x & 0x0F0F0F0Fu, b = y & 0x0F0F0F0Fu;
  const uint32_t even = __byte_perm(a, b, 0x6420);  // codes 0, 2, 4, 6
  const uint32_t odd = __byte_perm(a, b, 0x7531);   // codes 1, 3, 5, 7
  return even | (odd << 4);
}

// One thread per output word: eight consecutive codes of a row (8 bytes) -> one 32-bit word.
__global__ void __launch_bounds__(256)
pack_codes_4bit_kernel(const uint8_t* __restrict__ codes, int64_t rows, int64_t words_per_row,
                       int64_t ldc, uint32_t* __restrict__ packed, int32_t* info) {
  griddep_wait();
  const int64_t total = rows * words_per_row;
  bool bad = false;
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < total;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = k / words_per_row, w = k - r * words_per_row;
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(codes + r * ldc + 8 * w));
    bad |= ((v.x | v.y) & 0xF0F0F0F0u) != 0u;
    packed[k] = pack8_4bit(v.x, v.y);
  }
  if (bad) record_info(info, GPTQ_INFO_BAD_CODE);
  griddep_launch_dependents();
}

// One thread per 32 consecutive codes of a row (two 16-byte loads) -> four words (one 16-byte
// store): cols % 32 == 0, ldc % 16 == 0 and both buffers 16-byte aligned.
__global__ void __launch_bounds__(256)
pack_codes_4bit_vec_kernel(const uint8_t* __restrict__ codes, int64_t rows,
                           int64_t groups_per_row, int64_t ldc, uint32_t* __restrict__ packed,
                           int32_t* info) {
  griddep_wait();
  const int64_t total = rows * groups_per_row;
  bool bad = false;
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < total;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = k / groups_per_row, gk = k - r * groups_per_row;
    const uint4* src = reinterpret_cast<const uint4*>(codes + r * ldc + 32 * gk);
    const uint4 p = __ldg(src), q = __ldg(src + 1);
    bad |= ((p.x | p.y | p.z | p.w | q.x | q.y | q.z | q.w) & 0xF0F0F0F0u) != 0u;
    // rows of the packed codes are dense: group gk of row r is 16-byte word k
    reinterpret_cast<uint4*>(packed)[k] =
        make_uint4(pack8_4bit(p.x, p.y), pack8_4bit(p.z, p.w), pack8_4bit(q.x, q.y),
                   pack8_4bit(q.z, q.w));
  }
  if (bad) record_info(info, GPTQ_INFO_BAD_CODE);
  griddep_launch_dependents();
}

// Eight 3-bit codes (bytes of x, each < 8) -> 24 bits, code j at bits 3j: pairs, then quads, then
// the eight, each step moving the upper half down next to the lower one.
__device__ __forceinline__ uint32_t pack8_3bit(uint2 v) {
  uint64_t x = static_cast<uint64_t>(v.x) | (static_cast<uint64_t>(v.y) << 32);
  x = (x | (x >> 5)) & 0x003F003F003F003Full;
  x = (x | (x >> 10)) & 0x00000FFF00000FFFull;
  x = (x | (x >> 20)) & 0xFFFFFFull;
  return static_cast<uint32_t>(x);
}

// One thread per group of 32 codes of a row (32 bytes) -> three 32-bit words: the group's codes
// as one 96-bit little-endian number, code i in bits 3i .. 3i + 2.
__global__ void __launch_bounds__(256)
pack_codes_3bit_kernel(const uint8_t* __restrict__ codes, int64_t rows, int64_t groups_per_row,
                       int64_t ldc, uint32_t* __restrict__ packed, int32_t* info) {
  griddep_wait();
  const int64_t total = rows * groups_per_row;
  bool bad = false;
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < total;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = k / groups_per_row, gk = k - r * groups_per_row;
    const uint2* src = reinterpret_cast<const uint2*>(codes + r * ldc + 32 * gk);
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint2 v = __ldg(src + i);
      bad |= ((v.x | v.y) & 0xF8F8F8F8u) != 0u;
      q[i] = pack8_3bit(make_uint2(v.x & 0x07070707u, v.y & 0x07070707u));
    }
    uint32_t* dst = packed + 3 * k;         // rows are dense: 3 words per group
    dst[0] = q[0] | (q[1] << 24);
    dst[1] = (q[1] >> 8) | (q[2] << 16);
    dst[2] = (q[2] >> 16) | (q[3] << 8);
  }
  if (bad) record_info(info, GPTQ_INFO_BAD_CODE);
  griddep_launch_dependents();
}

// ------------------------------------------------------------------------------------------------
// W4A16 product
// ------------------------------------------------------------------------------------------------
constexpr int kMt = 16;                          // rows of one mma tile (the mma's M)
constexpr int kRows = 32;                        // rows of one CTA: two mma tiles per warp
constexpr int kChunk = 128;                      // columns a warp takes per step: 4 lanes x 32
constexpr int kStages = 3;                       // TMA ring depth per warp
constexpr int kCodeBytes = kRows * kChunk / 2;   // codes of one stage: 32 rows x 64 bytes
constexpr int kXRowBytes = kChunk * 2;           // one activation row of one stage (bf16)
constexpr int kMaxWarps = 16;

// Bytes of one ring stage: the code tile, then `xh` activation rows of the same 128 columns.
__host__ __device__ constexpr int stage_bytes(int xh) { return kCodeBytes + xh * kXRowBytes; }

// D = A * B + C for one m16n8k16 tile, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = a * b + c on bf16 pairs (one packed half-precision FMA instruction).
__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// The eight codes of one word as four bf16 pairs (q_p - z, q_{p+4} - z), p = 0..3. The nibbles
// are first split into bytes (even nibbles of w in `lo`, odd ones in `hi`); a byte permute then
// pairs two of those bytes with the byte 0x43 above each, making two bf16 numbers whose exponent
// is 2^7 and whose unit in the last place is 1, i.e. exactly 128 + q. Adding -(128 + z) (`negz`,
// both halves) is exact too (integers of magnitude below 256), so the tensor core sees the exact
// q - z. (A byte permute plus masks measured faster here than shift-and-mask extraction.)
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t negz, uint32_t (&p)[4]) {
  constexpr uint32_t kOne = 0x3F803F80u;    // (1.0, 1.0) in bf16
  constexpr uint32_t kMagic = 0x43434343u;  // high byte of bf16 128.0, in every byte
  const uint32_t lo = w & 0x0F0F0F0Fu;         // bytes: q0 q2 q4 q6
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // bytes: q1 q3 q5 q7
  p[0] = bf16x2_fma(__byte_perm(lo, kMagic, 0x4240), kOne, negz);  // (q0, q4)
  p[1] = bf16x2_fma(__byte_perm(hi, kMagic, 0x4240), kOne, negz);  // (q1, q5)
  p[2] = bf16x2_fma(__byte_perm(lo, kMagic, 0x4341), kOne, negz);  // (q2, q6)
  p[3] = bf16x2_fma(__byte_perm(hi, kMagic, 0x4341), kOne, negz);  // (q3, q7)
}

// y[n][r] = sum_c x[n][c] * s[r, g(c)] * (q[r][c] - z[r, g(c)]) for 32 rows per CTA. Each of
// the CTA's W warps takes the 128-column chunks w, w + W, w + 2W, ... and streams them through
// its own ring of kStages TMA buffers; a stage holds the 32 x 128 code tile and the matching
// 128 columns of the first `xh` activation rows (xh >= n, rows past n and columns past `cols`
// arrive as zeros). The warps' partial sums are added in warp order at the end, so the result
// does not depend on timing.
//
// Per chunk and warp, lane (g = lane / 4, t = lane % 4) holds 32 codes (columns 32t .. 32t + 31
// of the chunk) of each of the rows g, g + 8 (mma tile 0) and g + 16, g + 24 (mma tile 1), and
// the activations of vector n = g (NT = 2: also n = g + 8); both tiles use the same activation
// fragments. The mma's k index is a permutation of the columns, the same for both operands: in
// step 2i (2i + 1) lane t's k slots {2t, 2t+1, 2t+8, 2t+9} are its columns 8i + {0, 4, 1, 5}
// ({2, 6, 3, 7}), which is the order the nibble pairs come out of dequant_word.
// Eight steps cover the chunk; its sum is then scaled by the row's group scale in fp32.
// The group of chunk ch is (ch * gmul) >> 32 with gmul = ceil(2^32 / (group / 128)) -- exact for
// the sizes the host admits -- and gmul = 0 for one scale per row. Zero points are fetched one
// chunk ahead. Lanes whose vector n is past xh read row xh - 1 (their products land
// in output columns that are never stored).
template <int NT>
__global__ void __launch_bounds__(kMaxWarps * 32) __maxnreg__(NT == 1 ? 80 : 128)
w4a16_gemv_kernel(const __grid_constant__ CUtensorMap tcodes, const __grid_constant__ CUtensorMap tx,
                  int xh, const float* __restrict__ scales, const uint8_t* __restrict__ zeros,
                  int rows, int cols, uint64_t gmul, int n_groups, int n_act,
                  float* __restrict__ y, int64_t ldy, int32_t* info) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ volatile int abort_flag;
  const int nwarps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int sbytes = stage_bytes(xh);
  uint8_t* ring = smem + warp * (kStages * sbytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + nwarps * (kStages * sbytes)) +
                   warp * kStages;
  const int row0 = blockIdx.x * kRows;
  const int nchunks = (cols + kChunk - 1) / kChunk;

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbarrier_init();
  }
  if (threadIdx.x == 0) abort_flag = 0;
  __syncthreads();
  griddep_wait();

  int issued = 0;  // loads this warp has started (lane 0's count)
  if (lane == 0) {
    prefetch_tmap(&tcodes);
    prefetch_tmap(&tx);
    for (int s = 0; s < kStages; ++s) {
      const int ch = warp + s * nwarps;
      if (ch >= nchunks) break;
      mbar_arrive_expect_tx(&bars[s], sbytes);
      tma_load_2d(ring + s * sbytes, &tcodes, &bars[s], ch * (kChunk / 8), row0);
      tma_load_2d(ring + s * sbytes + kCodeBytes, &tx, &bars[s], ch * kChunk, 0);
      ++issued;
    }
  }

  // Offsets of this lane's four rows in the [rows x n_groups] metadata (below 2^31: the host
  // checks); rows past the end read the last row's (their results are not stored).
  int moff[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) moff[m] = min(row0 + g + 8 * m, rows - 1) * n_groups;
  int xoff[NT];  // byte offset of this lane's activations inside a stage
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    xoff[nt] = kCodeBytes + min(nt * 8 + g, xh - 1) * kXRowBytes + 64 * t;

  float acc[2][NT][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][nt][e] = 0.f;

  // zero points of the chunk about to be consumed
  uint32_t zq[4];
  {
    const uint32_t gi = static_cast<uint32_t>((static_cast<uint64_t>(warp) * gmul) >> 32);
#pragma unroll
    for (int m = 0; m < 4; ++m) zq[m] = __ldg(zeros + moff[m] + gi);
  }

  bool ok = true;
  int j = 0;  // chunks this warp has consumed
  uint32_t phase = 0;
  for (int base = warp; ok && base < nchunks; base += kStages * nwarps, phase ^= 1u) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      const int ch = base + s * nwarps;
      if (ch >= nchunks) break;
      // scales of this chunk (first needed after its products), zero points of the next chunk
      // of this warp (clamped: the last chunk reloads its own)
      const uint32_t gi = static_cast<uint32_t>((static_cast<uint64_t>(ch) * gmul) >> 32);
      const int chn = min(ch + nwarps, nchunks - 1);
      const uint32_t gin = static_cast<uint32_t>((static_cast<uint64_t>(chn) * gmul) >> 32);
      float sc[4];
      uint32_t zq_n[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        sc[m] = __ldg(scales + moff[m] + gi);
        zq_n[m] = __ldg(zeros + moff[m] + gin);
      }
      uint32_t nz[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) nz[m] = (0xC300u + zq[m]) * 0x00010001u;  // -(128 + z), twice

      const bool got = __all_sync(0xffffffffu,
                                  mbar_wait_bounded(&bars[s], phase, &abort_flag, info));
      if (!got) {
        ok = false;
        break;
      }
      const uint8_t* st = ring + s * sbytes;
      uint4 wv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
        wv[m] = *reinterpret_cast<const uint4*>(st + (g + 8 * m) * 64 + t * 16);

      float d[2][NT][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[h][nt][e] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t b[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          // x[8i .. 8i+7] of this lane's columns, natural order
          const uint4 v = *reinterpret_cast<const uint4*>(st + xoff[nt] + 16 * i);
          b[nt][0] = __byte_perm(v.x, v.z, 0x5410);  // (x0, x4)
          b[nt][1] = __byte_perm(v.x, v.z, 0x7632);  // (x1, x5)
          b[nt][2] = __byte_perm(v.y, v.w, 0x5410);  // (x2, x6)
          b[nt][3] = __byte_perm(v.y, v.w, 0x7632);  // (x3, x7)
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t w_lo = i == 0 ? wv[2 * h].x : i == 1 ? wv[2 * h].y
                              : i == 2 ? wv[2 * h].z : wv[2 * h].w;
          const uint32_t w_hi = i == 0 ? wv[2 * h + 1].x : i == 1 ? wv[2 * h + 1].y
                              : i == 2 ? wv[2 * h + 1].z : wv[2 * h + 1].w;
          uint32_t p0[4], p1[4];
          dequant_word(w_lo, nz[2 * h], p0);
          dequant_word(w_hi, nz[2 * h + 1], p1);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_bf16(d[h][nt], p0[0], p1[0], p0[1], p1[1], b[nt][0], b[nt][1]);
            mma_bf16(d[h][nt], p0[2], p1[2], p0[3], p1[3], b[nt][2], b[nt][3]);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[h][nt][0] = fmaf(sc[2 * h], d[h][nt][0], acc[h][nt][0]);
          acc[h][nt][1] = fmaf(sc[2 * h], d[h][nt][1], acc[h][nt][1]);
          acc[h][nt][2] = fmaf(sc[2 * h + 1], d[h][nt][2], acc[h][nt][2]);
          acc[h][nt][3] = fmaf(sc[2 * h + 1], d[h][nt][3], acc[h][nt][3]);
        }
#pragma unroll
      for (int m = 0; m < 4; ++m) zq[m] = zq_n[m];
      ++j;

      // Every lane has consumed stage s (its codes and activations fed the products above):
      // refill it.
      __syncwarp();
      if (lane == 0) {
        const int nxt = ch + kStages * nwarps;
        if (nxt < nchunks) {
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&bars[s], sbytes);
          tma_load_2d(ring + s * sbytes, &tcodes, &bars[s], nxt * (kChunk / 8), row0);
          tma_load_2d(ring + s * sbytes + kCodeBytes, &tx, &bars[s], nxt * kChunk, 0);
          ++issued;
        }
      }
    }
  }
  griddep_launch_dependents();

  if (!ok && lane == 0) {
    // Let the loads still in flight land before the ring is reused or the CTA exits.
    for (int k = j; k < issued; ++k) mbar_drain_bounded(&bars[k % kStages], (k / kStages) & 1);
  }
  __syncwarp();

  // Partial sums of this warp -> its (now idle) ring: part[row][n], 32 x 8NT floats.
  float* part = reinterpret_cast<float*>(ring);
  constexpr int kLd = 8 * NT;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int ra = h * kMt + g, rb = h * kMt + g + 8;
      part[ra * kLd + nt * 8 + 2 * t] = acc[h][nt][0];
      part[ra * kLd + nt * 8 + 2 * t + 1] = acc[h][nt][1];
      part[rb * kLd + nt * 8 + 2 * t] = acc[h][nt][2];
      part[rb * kLd + nt * 8 + 2 * t + 1] = acc[h][nt][3];
    }
  __syncthreads();
  if (abort_flag) return;
  for (int k = threadIdx.x; k < kRows * kLd; k += blockDim.x) {
    const int row = k % kRows, n = k / kRows;
    const int r = row0 + row;
    if (n >= n_act || r >= rows) continue;
    float sum = 0.f;
    for (int w = 0; w < nwarps; ++w)
      sum += reinterpret_cast<const float*>(smem + w * (kStages * sbytes))[row * kLd + n];
    y[static_cast<int64_t>(n) * ldy + r] = sum;
  }
}

size_t gemv_smem_bytes(int nwarps, int xh) {
  return static_cast<size_t>(nwarps) * kStages * (stage_bytes(xh) + 8);
}

// Warps per CTA for a layer of `ctas` CTAs: the most warps per CTA whose CTAs all fit on the
// device at once (no second, partial wave of CTAs at the end); if no choice fits them all, the one
// with the most warps resident. Occupancy per warp count comes from the runtime (registers and
// shared memory of the kernel as built) and is cached per device and activation tile height.
template <int NT>
int pick_warps(int64_t ctas, int64_t nchunks, int xh) {
  static std::mutex mu;
  static int occ[64][5][kMaxWarps + 1] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  const int xi = xh <= 1 ? 0 : xh <= 2 ? 1 : xh <= 4 ? 2 : xh <= 8 ? 3 : 4;
  std::lock_guard<std::mutex> lock(mu);
  if (occ[dev][xi][0] == 0) {
    // dynamic shared memory allowed per CTA: the opt-in limit less the kernel's static part
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaFuncGetAttributes(&fa, w4a16_gemv_kernel<NT>) != cudaSuccess)
      return -1;
    const size_t limit = static_cast<size_t>(optin) - fa.sharedSizeBytes;
    if (set_max_dynamic_smem(reinterpret_cast<const void*>(w4a16_gemv_kernel<NT>),
                             static_cast<int>(limit)) != GPTQ_OK)
      return -1;
    for (int w = 1; w <= kMaxWarps; ++w) {
      int b = 0;
      const size_t sm = gemv_smem_bytes(w, xh);
      if (sm > limit) break;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, w4a16_gemv_kernel<NT>, 32 * w, sm) !=
          cudaSuccess)
        return -1;
      occ[dev][xi][w] = b;
    }
    occ[dev][xi][0] = 1;
  }
  const int64_t sms = num_sms();
  int best = 0;
  int64_t best_resident = -1;
  bool best_fits = false;
  for (int w = 1; w <= kMaxWarps && w <= nchunks; ++w) {
    const int64_t slots = static_cast<int64_t>(occ[dev][xi][w]) * sms;
    if (slots <= 0) continue;
    const bool fits = ctas <= slots;
    const int64_t resident = (fits ? ctas : slots) * w;
    if ((fits && !best_fits) || (fits == best_fits && resident > best_resident)) {
      best = w;
      best_resident = resident;
      best_fits = fits;
    }
  }
  return best;
}

template <int NT>
gptq_status launch_gemv(const CUtensorMap& tcodes, const CUtensorMap& tx, int xh, int64_t rows,
                        int64_t cols, const float* scales, const uint8_t* zeros, uint64_t gmul,
                        int n_groups, int n, float* y, int64_t ldy, int32_t* info,
                        cudaStream_t stream) {
  const int64_t ctas = (rows + kRows - 1) / kRows;
  const int nwarps = pick_warps<NT>(ctas, (cols + kChunk - 1) / kChunk, xh);
  if (nwarps <= 0) return GPTQ_ECUDA;
  return launch_pdl(w4a16_gemv_kernel<NT>, dim3(static_cast<unsigned>(ctas)), dim3(nwarps * 32),
                    gemv_smem_bytes(nwarps, xh), stream, tcodes, tx, xh, scales, zeros,
                    static_cast<int>(rows), static_cast<int>(cols), gmul, n_groups, n, y, ldy,
                    info);
}

}  // namespace

gptq_status run_pack_codes_4bit(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ldc,
                                uint32_t* packed, int32_t* info, cudaStream_t stream) {
  if (cols % 32 == 0 && ldc % 16 == 0 && (reinterpret_cast<uintptr_t>(codes) & 15u) == 0 &&
      (reinterpret_cast<uintptr_t>(packed) & 15u) == 0) {
    const int64_t total = rows * (cols / 32);
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, 16 * num_sms());
    return launch_pdl(pack_codes_4bit_vec_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256),
                      0, stream, codes, rows, cols / 32, ldc, packed, info);
  }
  const int64_t words = rows * (cols / 8);
  int64_t blocks = (words + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  return launch_pdl(pack_codes_4bit_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                    stream, codes, rows, cols / 8, ldc, packed, info);
}

gptq_status run_pack_codes_3bit(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ldc,
                                uint32_t* packed, int32_t* info, cudaStream_t stream) {
  const int64_t total = rows * (cols / 32);
  const int64_t blocks = std::min<int64_t>((total + 255) / 256, 16 * num_sms());
  return launch_pdl(pack_codes_3bit_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                    stream, codes, rows, cols / 32, ldc, packed, info);
}

gptq_status run_w4a16_gemv(const uint32_t* packed, const float* scales, const uint8_t* zeros,
                           int64_t rows, int64_t cols, int group, const void* x, int64_t n,
                           int64_t ldx, float* y, int64_t ldy, int32_t* info,
                           cudaStream_t stream) {
  // Activation tile height: n rounded up to a power of two (rows past n arrive as zeros).
  const int xh = n <= 1 ? 1 : n <= 2 ? 2 : n <= 4 ? 4 : n <= 8 ? 8 : 16;
  CUtensorMap tcodes, tx;
  gptq_status st = encode_tmap_2d(&tcodes, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, 4, cols / 8,
                                  rows, cols / 8, kChunk / 8, kRows, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != GPTQ_OK) return st;
  st = encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, 2, cols, n, ldx, kChunk, xh,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != GPTQ_OK) return st;
  const int n_groups = group > 0 ? static_cast<int>(cols / group) : 1;
  // chunk -> group index as (chunk * gmul) >> 32 with gmul = ceil(2^32 / d), d = group / 128
  // chunks per group: exact while chunk * d <= 2^32, which cols <= 2^22 guarantees. gmul = 0
  // maps every chunk to group 0 (one scale per row).
  const uint64_t d = group > 0 ? static_cast<uint64_t>(group / kChunk) : 0;
  const uint64_t gmul = d == 0 ? 0 : ((1ull << 32) + d - 1) / d;
  if (n <= 8)
    return launch_gemv<1>(tcodes, tx, xh, rows, cols, scales, zeros, gmul, n_groups,
                          static_cast<int>(n), y, ldy, info, stream);
  return launch_gemv<2>(tcodes, tx, xh, rows, cols, scales, zeros, gmul, n_groups,
                        static_cast<int>(n), y, ldy, info, stream);
}

}  // namespace gptq
