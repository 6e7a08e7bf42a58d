// qlora_merge.cu -- folding the adapter into the weight after training.
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora), "Merging LoRA weights
// for inference": once A and B are trained, W_merged = W0 + (alpha/r) B A has
// W0's shape and replaces the two paths (h = W_merged x).  For a quantized base
// the page defers the precision question to QLoRA; here the base is the
// reconstructed NF4 weight W^ (doubleDequant, bf16, the weight the forward
// uses), and
//     W_out[n][c] = BF16(fma(s, acc[n][c], W^[n][c])),  acc = sum_j B[n][j] A[j][c]
// with s = RN32(alpha / r), acc accumulated in fp32 on the tensor cores (order
// unspecified) and one rounding to bf16 (nearest even).  Re-quantising the
// merged weight is nf4_quantize on W_out.
//
// k_lora_merge: one CTA per 64 weight rows x 128 columns, 256 threads (three
// CTAs per SM).
//   0. Every thread first loads its 32 codes (16 bytes) and its block's
//      constants, so their DRAM latency overlaps steps 1 and 2.
//   1. For each 64-wide chunk of r, B's 64 x 64 and A's 64 x 128 tiles are
//      copied to shared memory (zero padded past r, d and k) and every warp
//      runs mma.sync.m16n8k16 (bf16 in, fp32 accumulate) over its 16 x 64
//      piece.  The contraction is tiny (r multiply-adds per weight); the tensor
//      cores only keep it off the critical path.
//   2. The fp32 tile goes to shared memory.
//   3. Each thread expands its half block (32 weights), adds s * acc with one
//      fma and writes 64 bytes of bf16 (four threads per row, so a row's 256
//      bytes are written contiguously).
// Bound: HBM (0.5 B of codes + 2 B of output per weight).
#include <cstdio>

#include "nf4_scale.cuh"
#include "nf4_table.h"
#include "qlora_device.cuh"
#include "qlora_internal.h"

namespace qlora {

namespace {

constexpr int kMergeRows = 64;
constexpr int kMergeCols = 128;
constexpr int kRChunk = 64;
constexpr int kBStride = kRChunk + 8;         // bf16 per row of the B tile (16 B pad: no ldmatrix conflicts)
constexpr int kAStride = kMergeCols + 8;      // bf16 per row of the A tile
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
constexpr uint32_t kTileBytes = (kMergeRows * kBStride + kRChunk * kAStride) * 2;
constexpr uint32_t kResBytes = kMergeRows * kMergeCols * 4;
constexpr uint32_t kMergeSmem = kTileBytes > kResBytes ? kTileBytes : kResBytes;

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

__global__ void __launch_bounds__(256, 3) k_lora_merge(const uint8_t* __restrict__ codes, const ScaleSrc sc,
                                                    const uint16_t* __restrict__ A, const uint16_t* __restrict__ B,
                                                    int64_t d, int64_t k, int r, float s, uint16_t* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* sB = reinterpret_cast<uint16_t*>(smem);
  uint16_t* sA = sB + kMergeRows * kBStride;
  float* sR = reinterpret_cast<float*>(smem);   // after the contraction
  griddep_launch_dependents();
  griddep_wait();

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kMergeRows;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kMergeCols;
  const int wr = warp >> 1;   // rows 16 wr .. 16 wr + 15
  const int wc = warp & 1;    // columns 64 wc .. 64 wc + 63

  // this thread's half block of the epilogue: row tid / 4, columns 32 (tid % 4) ..
  const int row = tid >> 2, quarter = tid & 3;
  const int64_t n = n0 + row;
  const int64_t c = c0 + 32 * quarter;
  const bool live = (n < d) && (c < k);
  uint4 cw4 = make_uint4(0, 0, 0, 0);
  ScaleRaw raw{};
  if (live) {
    cw4 = ldg_nc_v4(codes + ((n * k + c) >> 1));
    raw = scale_fetch(sc, (n * k + c) >> 6);
  }
  const float mean = sc.dq ? __ldg(sc.mean) : 0.0f;

  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;

  for (int j0 = 0; j0 < r; j0 += kRChunk) {
    // B (d x r, row-major): 64 rows x 64 columns of the chunk.  Rows are 2r
    // bytes: 16-byte loads when r % 8 == 0, element loads otherwise.
    if ((r & 7) == 0) {
      for (int i = tid; i < kMergeRows * (kRChunk / 8); i += 256) {
        const int row = i >> 3, j8 = i & 7;
        const int64_t n = n0 + row;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < d && j0 + 8 * j8 < r) v = __ldg(reinterpret_cast<const uint4*>(B + n * r + j0 + 8 * j8));
        *reinterpret_cast<uint4*>(sB + row * kBStride + 8 * j8) = v;
      }
    } else {
      for (int i = tid; i < kMergeRows * kRChunk; i += 256) {
        const int row = i / kRChunk, j = i % kRChunk;
        const int64_t n = n0 + row;
        uint16_t v = 0;
        if (n < d && j0 + j < r) v = B[n * r + j0 + j];
        sB[row * kBStride + j] = v;
      }
    }
    // A (r x k, row-major; k % 64 == 0 so rows are 16-byte aligned): 64 rows
    // x 128 columns, 16-byte loads
    for (int i = tid; i < kRChunk * (kMergeCols / 8); i += 256) {
      const int j = i / (kMergeCols / 8), c8 = i % (kMergeCols / 8);
      const int64_t c = c0 + 8 * c8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j0 + j < r && c < k) v = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j0 + j) * k + c));
      *reinterpret_cast<uint4*>(sA + j * kAStride + 8 * c8) = v;
    }
    __syncthreads();
    const uint32_t sB_addr = smem_u32(sB), sA_addr = smem_u32(sA);
#pragma unroll
    for (int kk = 0; kk < kRChunk / 16; ++kk) {
      // A operand (B rows, row-major 16 x 16): lanes 0-15 rows 0-15 at k 0,
      // lanes 16-31 the same rows at k 8
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sB_addr + 2u * ((16 * wr + (lane & 15)) * kBStride + 16 * kk + 8 * (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        // B operand (A rows j, columns c): two 8-column tiles, transposed
        // loads; lanes 0-7 k 0-7, 8-15 k 8-15 of tile 2np, 16-31 the same of
        // tile 2np + 1
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
  constexpr uint32_t kCB[16] = {QLORA_NF4_TABLE_BITS};
  float C[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) C[j] = __uint_as_float(kCB[j]);
  ScaleRecip recip;
  // the block's reconstructed weights, as doubleDequant stores them:
  // BF16(RN32(C[q] * s^))
  const Nf4Tab tab = make_tab(scale_value(sc.dq, mean, raw, recip), C);
  uint16_t* orow = out + n * k + c;
  const uint32_t cw[4] = {cw4.x, cw4.y, cw4.z, cw4.w};
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    const uint4 wq = dq8(cw[ch], tab);   // 8 bf16 weights, element i in halfword i
    const float4 lo = *reinterpret_cast<const float4*>(sR + res_index(row, 32 * quarter + 8 * ch));
    const float4 hi = *reinterpret_cast<const float4*>(sR + res_index(row, 32 * quarter + 8 * ch + 4));
    const float a8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    const uint32_t w4[4] = {wq.x, wq.y, wq.z, wq.w};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float v0 = __fmaf_rn(s, a8[2 * h], __uint_as_float(w4[h] << 16));
      const float v1 = __fmaf_rn(s, a8[2 * h + 1], __uint_as_float(w4[h] & 0xFFFF0000u));
      o[h] = pack_bf16x2(v0, v1);
    }
    *reinterpret_cast<uint4*>(orow + 8 * ch) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_lora_merge(const qlora_nf4_t& q, const uint16_t* A, const uint16_t* B, int r, float s,
                              uint16_t* out, cudaStream_t st) {
  if ((q.d + kMergeRows - 1) / kMergeRows > 65535) return cudaErrorInvalidConfiguration;   // grid y limit
  const cudaError_t e = set_smem(k_lora_merge, kMergeSmem);
  if (e != cudaSuccess) return e;
  ScaleSrc sc{};
  sc.dq = q.double_quant;
  sc.absmax = q.absmax;
  sc.c2 = q.c2;
  sc.c1 = q.c1;
  sc.mean = q.mean;
  const dim3 grid(static_cast<unsigned>((q.k + kMergeCols - 1) / kMergeCols),
                  static_cast<unsigned>((q.d + kMergeRows - 1) / kMergeRows));
  {
    ProfScope ps_(QLORA_KC_AUX, st);
    const cudaError_t el = launch_pdl(k_lora_merge, grid, dim3(256), kMergeSmem, st, nullptr, q.codes, sc, A,
                                      B, q.d, q.k, r, s, out);
    if (el != cudaSuccess) return el;
  }
  return cudaGetLastError();
}

}  // namespace qlora
