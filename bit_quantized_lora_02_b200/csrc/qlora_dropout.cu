// qlora_dropout.cu -- adapter dropout for the QLoRA linear layer.
//
// "LoRA and QLoRA: Efficient Fine-Tuning of Large Language Models"
// (fromzero2ai.dev), "Python Implementation: Fine-Tuning with PEFT and
// BitsAndBytes", step 4, configures lora_dropout = 0.05 for the adapted
// layers.  Dropout acts on the adapter's input only:
//     Y = X W^T + s (drop(X) A^T) B^T,   drop(X) = X * keep * 1 / (1 - p),
// so the frozen base path sees X unchanged.  The pages name no random-number
// generator; the keep decisions come from the counter-based Philox4x32-10
// generator (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC 2011).  Element i = m k + j (flat row-major index of X) uses
// output word i mod 4 of Philox4x32-10 at counter (i div 4 as two 32-bit
// words, offset as two 32-bit words) under key (seed as two 32-bit words); it
// is kept when (word >> 8) * 2^-24 >= RN32(p).  With t = ceil(RN32(p) 2^24)
// (exact: p is scaled by a power of two) the test is the integer comparison
// (word >> 8) >= t.
//
// The decisions are packed into a keep bitmask (bit b of word w <-> element
// 32 w + b, 1 = kept), written once per call by k_dropout_bits into the
// workspace and read by the kernels that need it:
//   T_s = BF16(s / (1 - p) * (X . keep) A^T)  the low-rank GEMM masks each X
//                                           stage in shared memory
//                                           (qlora_gemm.cu) or the few-token
//                                           down projection masks its loads;
//   dA  = 1 / (1 - p) * U_s^T (X . keep)    the same masking in the dA GEMM;
//   dX  = dY W^ + (U_s A) . keep / (1 - p)  the dX GEMM runs without its LoRA
//                                           K steps and k_lora_up_dropout adds
//                                           the masked term in place;
//   dB  = dY^T T_s                          unchanged (T_s is already masked).
// Because the mask is regenerated from (seed, offset) in the backward, no mask
// has to be kept between the two calls.
#include <cstdio>

#include "qlora_device.cuh"
#include "qlora_internal.h"

namespace qlora {

namespace {

// Philox4x32 with 10 rounds (SC 2011): per round the two multiplies give
// (hi, lo) pairs, the words are permuted and mixed with the key, and the key
// advances by the Weyl constants.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    // one widening multiply gives both halves of each product
    const uint64_t p0 = static_cast<uint64_t>(c.x) * 0xD2511F53u;
    const uint64_t p1 = static_cast<uint64_t>(c.z) * 0xCD9E8D57u;
    const uint32_t lo0 = static_cast<uint32_t>(p0), hi0 = static_cast<uint32_t>(p0 >> 32);
    const uint32_t lo1 = static_cast<uint32_t>(p1), hi1 = static_cast<uint32_t>(p1 >> 32);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// One thread per 32-element word of the bitmask: 8 Philox calls (counters
// 8w .. 8w + 7).  Elements at or past n get a 0 bit.  The words are computed
// before waiting on the previous kernel, so the generator overlaps its tail.
__global__ void __launch_bounds__(256) k_dropout_bits(int64_t n, uint32_t thr, uint32_t seed_lo, uint32_t seed_hi,
                                                     uint32_t off_lo, uint32_t off_hi, uint32_t* __restrict__ bits) {
  griddep_launch_dependents();
  const int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nw = (n + 31) >> 5;
  // (word >> 8) >= thr  <=>  word >= thr * 2^8 (thr <= 2^24; thr == 2^24 would
  // drop everything and needs p = 1, which is refused)
  const uint32_t thr8 = thr << 8;
  uint32_t word = 0;
  if (w < nw) {
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint64_t q = static_cast<uint64_t>(w) * 8u + static_cast<uint64_t>(t);
      const uint4 r = philox4x32_10(
          make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32), off_lo, off_hi), seed_lo, seed_hi);
      word |= (r.x >= thr8 ? 1u : 0u) << (4 * t);
      word |= (r.y >= thr8 ? 1u : 0u) << (4 * t + 1);
      word |= (r.z >= thr8 ? 1u : 0u) << (4 * t + 2);
      word |= (r.w >= thr8 ? 1u : 0u) << (4 * t + 3);
    }
    // elements past n (a ragged last word) are not kept
    const int64_t valid = n - 32 * w;
    if (valid < 32) word &= (1u << valid) - 1u;
  }
  griddep_wait();   // the previous kernel may still read an earlier mask in the same workspace
  if (w < nw) bits[w] = word;
}

// ---------------------------------------------------------------------------
// dX += (U_s A) . keep / (1 - p), in place on the bf16 dX.
//
// One CTA per 64 tokens x 128 input columns, 256 threads.  The rank-r
// contraction U_s A is tiny (r multiply-adds per element) and runs on
// mma.sync.m16n8k16 from shared-memory tiles of U_s (64 x 64 per rank chunk)
// and A (64 x 128), as in the merge kernel.  Each thread then takes 32
// consecutive columns of one token row: 64 bytes of dX, one mask word, one
// rounding to bf16.  Bound: HBM (2 B read + 2 B written per element of dX).
// ---------------------------------------------------------------------------
constexpr int kUpRows = 64;
constexpr int kUpCols = 128;
constexpr int kRChunk = 64;
constexpr int kUStride = kRChunk + 8;    // bf16 per row of the U_s tile (16 B pad: conflict-free ldmatrix)
constexpr int kAStride = kUpCols + 8;    // bf16 per row of the A tile
// result tile: 64 rows x 128 fp32, 16-byte chunks XOR-swizzled per row and
// 32-column quarter q (chunk c of quarter q at (c ^ h) within the quarter,
// h = 2 ((row mod 4) ^ q) + (q mod 2)).  A half-warp's 8-byte fragment stores
// (four rows x two chunks) and a quarter-warp's 16-byte epilogue reads (two
// rows x four quarters) each hit all 32 banks once.
__device__ __forceinline__ int res_index(int row, int col) {
  const int chunk = col >> 2, q = chunk >> 3;
  const int h = (((row & 3) ^ q) << 1) | (q & 1);
  return row * 128 + (((q << 3) | ((chunk & 7) ^ h)) << 2) + (col & 3);
}
constexpr uint32_t kTileBytes = (kUpRows * kUStride + kRChunk * kAStride) * 2;
constexpr uint32_t kResBytes = kUpRows * kUpCols * 4;
constexpr uint32_t kUpSmem = kTileBytes > kResBytes ? kTileBytes : kResBytes;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256, 3)
    k_lora_up_dropout(const uint16_t* __restrict__ U, int rp, const uint16_t* __restrict__ A, int r,
                      const uint32_t* __restrict__ keep, float dscale, int64_t M, int64_t k,
                      uint16_t* __restrict__ dX) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* sU = reinterpret_cast<uint16_t*>(smem);
  uint16_t* sA = sU + kUpRows * kUStride;
  float* sR = reinterpret_cast<float*>(smem);   // after the contraction
  griddep_launch_dependents();
  griddep_wait();

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kUpRows;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kUpCols;
  const int wr = warp >> 1;   // token rows 16 wr .. 16 wr + 15
  const int wc = warp & 1;    // columns 64 wc .. 64 wc + 63

  // this thread's part of the epilogue: row tid / 4, columns 32 (tid % 4) ..;
  // its dX bytes and mask word are loaded first so their latency overlaps the
  // contraction
  const int row = tid >> 2, quarter = tid & 3;
  const int64_t m = m0 + row;
  const int64_t c = c0 + 32 * quarter;
  const bool live = (m < M) && (c < k);
  uint4 x4[4] = {};
  uint32_t kw = 0;
  uint16_t* xrow = dX + m * k + c;
  if (live) {
#pragma unroll
    for (int i = 0; i < 4; ++i) x4[i] = *reinterpret_cast<const uint4*>(xrow + 8 * i);
    kw = __ldg(keep + ((m * k + c) >> 5));
  }

  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;

  for (int j0 = 0; j0 < r; j0 += kRChunk) {
    // U_s (M x rp, row-major; rp % 64 == 0): 64 rows x 64 columns, 16-byte loads
    for (int i = tid; i < kUpRows * (kRChunk / 8); i += 256) {
      const int rr = i >> 3, j8 = i & 7;
      const int64_t mm = m0 + rr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (mm < M) v = __ldg(reinterpret_cast<const uint4*>(U + mm * rp + j0 + 8 * j8));
      *reinterpret_cast<uint4*>(sU + rr * kUStride + 8 * j8) = v;
    }
    // A (r x k, row-major; k % 64 == 0): 64 rows x 128 columns, zero past r and k
    for (int i = tid; i < kRChunk * (kUpCols / 8); i += 256) {
      const int j = i / (kUpCols / 8), c8 = i % (kUpCols / 8);
      const int64_t cc = c0 + 8 * c8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j0 + j < r && cc < k) v = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j0 + j) * k + cc));
      *reinterpret_cast<uint4*>(sA + j * kAStride + 8 * c8) = v;
    }
    __syncthreads();
    const uint32_t sU_addr = smem_u32(sU), sA_addr = smem_u32(sA);
#pragma unroll
    for (int kk = 0; kk < kRChunk / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sU_addr + 2u * ((16 * wr + (lane & 15)) * kUStride + 16 * kk + 8 * (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int krow = 16 * kk + (lane & 15);
        const int ncol = 64 * wc + 16 * np + 8 * (lane >> 4);
        ldsm_x4_t(sA_addr + 2u * (krow * kAStride + ncol), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
  }

  // fp32 tile to shared memory: fragment (nt, e) holds row 16 wr + lane/4 (+8
  // for e >= 2), column 64 wc + 8 nt + 2 (lane % 4) + (e & 1)
  {
    const int g = lane >> 2, q2 = 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int col = 64 * wc + 8 * nt + q2;
      *reinterpret_cast<float2*>(sR + res_index(16 * wr + g, col)) = make_float2(acc[nt][0], acc[nt][1]);
      *reinterpret_cast<float2*>(sR + res_index(16 * wr + g + 8, col)) = make_float2(acc[nt][2], acc[nt][3]);
    }
  }
  __syncthreads();
  if (!live) return;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    const float4 lo = *reinterpret_cast<const float4*>(sR + res_index(row, 32 * quarter + 8 * ch));
    const float4 hi = *reinterpret_cast<const float4*>(sR + res_index(row, 32 * quarter + 8 * ch + 4));
    const float a8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    const uint32_t w4[4] = {x4[ch].x, x4[ch].y, x4[ch].z, x4[ch].w};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int e0 = 8 * ch + 2 * h;
      const float g0 = ((kw >> e0) & 1u) ? dscale : 0.0f;
      const float g1 = ((kw >> (e0 + 1)) & 1u) ? dscale : 0.0f;
      const float v0 = __fmaf_rn(g0, a8[2 * h], bf16_lo(w4[h]));
      const float v1 = __fmaf_rn(g1, a8[2 * h + 1], bf16_hi(w4[h]));
      o[h] = pack_bf16x2(v0, v1);
    }
    *reinterpret_cast<uint4*>(xrow + 8 * ch) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

uint32_t dropout_threshold(float p) {
  // RN32(p) * 2^24 is exact; its ceiling is the smallest 24-bit draw kept
  const double t = static_cast<double>(p) * 16777216.0;
  const double c = static_cast<double>(static_cast<uint64_t>(t));
  return static_cast<uint32_t>(c < t ? c + 1.0 : c);
}

cudaError_t launch_dropout_bits(int64_t n, const DropoutArgs& d, uint32_t* bits, cudaStream_t st) {
  const int64_t nw = (n + 31) >> 5;
  if (nw == 0) return cudaSuccess;
  const int64_t blocks = (nw + 255) / 256;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  {
    ProfScope ps_(QLORA_KC_AUX, st);
    const cudaError_t e = launch_pdl(k_dropout_bits, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, nullptr, n,
                                     d.thr, static_cast<uint32_t>(d.seed), static_cast<uint32_t>(d.seed >> 32),
                                     static_cast<uint32_t>(d.offset), static_cast<uint32_t>(d.offset >> 32), bits);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_lora_up_dropout(const uint16_t* U, int rp, const uint16_t* A, int r, const uint32_t* keep,
                                   float dscale, int64_t M, int64_t k, uint16_t* dX, cudaStream_t st) {
  if ((M + kUpRows - 1) / kUpRows > 65535) return cudaErrorInvalidConfiguration;   // grid y limit
  cudaError_t e = set_smem(k_lora_up_dropout, kUpSmem);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((k + kUpCols - 1) / kUpCols), static_cast<unsigned>((M + kUpRows - 1) / kUpRows));
  {
    ProfScope ps_(QLORA_KC_LORA_GEMM, st);
    e = launch_pdl(k_lora_up_dropout, grid, dim3(256), kUpSmem, st, nullptr, U, rp, A, r, keep, dscale, M, k, dX);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace qlora
