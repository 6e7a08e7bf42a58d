// nf4_quant.cu -- blockwise NF4 quantisation with double quantisation of the
// block constants, and the standalone double dequantisation.
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora):
//   "Quantizing and dequantizing with the codebook"  (blocks of 64, absmax
//      scale, nearest code with the smaller index on ties, exact-zero code for
//      an all-zero block, reconstruction scale * C[code]);
//   "First, how does k-bit quantization work?"       (Int8 absmax: c = 127 /
//      absmax, q = round(c x), all-zero input -> zeros and a nonzero scale);
//   "Double quantization and double dequantization"  (8-bit constants in groups
//      of 256, one FP32 second-level scale per group, a stored mean;
//      doubleDequant in BF16).
//
// Kernels (all memory-bound streaming kernels, no waits):
//   k_nf4_quant    one pass over W0: block absmax (4-lane shuffle max), code
//                  search, nibble packing; per-CTA exponent histogram of the
//                  absmax values (for the exact mean) when DQ is on.
//   k_dq_groups    warp 0 of each CTA: exact sum of the histogram in 32-bit
//                  limbs, rounded once to fp64, divided, rounded to fp32 (the
//                  mean); then one warp per group of 256 scales: subtract the
//                  mean, absmax, c1 = 127 / absmax, c2 = round-half-even(c1 v);
//                  with E4M3 constants (the page's "c2_FP8" label) c1 =
//                  448 / absmax and c2 = E4M3(c1 v), nearest even.
//   k_nf4_dequant  one pass over the codes: scale reconstruction and
//                  BF16(C[q] * s^), 16-byte vector stores.
#include <cmath>
#include <cstdint>
#include <cstring>

#include <cuda_fp8.h>

#include "nf4_scale.cuh"
#include "nf4_table.h"
#include "qlora_device.cuh"
#include "qlora_internal.h"

namespace qlora {

static const uint32_t h_nf4_bits[16] = {QLORA_NF4_TABLE_BITS};

void host_codebook(float out[16]) { std::memcpy(out, h_nf4_bits, sizeof(h_nf4_bits)); }

// ----------------------------------------------------------------------------
// Code search table.
//
// The nearest-code rule compares fp32 distances |RN32(xn - C[j])| with the
// smaller index winning ties.  Both distances are monotone in xn, so between
// neighbours C[j] and C[j+1] the choice flips exactly once: t_j is the largest
// fp32 xn for which C[j] still wins, and code(xn) = #{ j : xn > t_j }.
//
// To find which t_j to compare against with one lookup, xn is bucketed into 33
// cells by cell(xn) = RN_even(16 xn + 16) (one FFMA against a 1.5 * 2^23 bias,
// read off the low mantissa bits).  cell() is monotone, each cell holds at
// most one threshold (neighbouring t_j are > 1/16 apart), so
//     code(xn) = base[cell] + (xn > thr[cell])
// with base[c] = #{ j : cell(t_j) < c } and thr[c] the threshold in cell c
// (3.0, never exceeded, when the cell has none).  This is exact for every fp32
// xn in [-1, 1]; the host builds the table once from C with IEEE fp32
// arithmetic.
// ----------------------------------------------------------------------------
constexpr float kCellBias = 12582928.0f;   // 1.5 * 2^23 + 16
constexpr uint32_t kCellBiasBits = 0x4B400000u;

struct QuantLut {
  float thr[33];
  float base[33];  // integer counts stored as fp32 bit patterns
};

static float f_of(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

static bool left_wins(float x, float a, float b) {
  volatile float da = x - a;   // each difference rounded to fp32 once
  volatile float db = x - b;
  return std::fabs(da) <= std::fabs(db);
}

static int host_cell(float x) {
  float y = std::fmaf(x, 16.0f, kCellBias);
  uint32_t u;
  std::memcpy(&u, &y, 4);
  return static_cast<int>(u - kCellBiasBits);
}

static bool g_lut_ok = false;

static QuantLut build_lut() {
  QuantLut L;
  float C[16];
  for (int j = 0; j < 16; ++j) C[j] = f_of(h_nf4_bits[j]);
  float t[15];
  for (int j = 0; j < 15; ++j) {
    float x = static_cast<float>((static_cast<double>(C[j]) + static_cast<double>(C[j + 1])) * 0.5);
    while (!left_wins(x, C[j], C[j + 1])) x = std::nextafterf(x, -2.0f);
    for (;;) {
      float up = std::nextafterf(x, 2.0f);
      if (!left_wins(up, C[j], C[j + 1])) break;
      x = up;
    }
    t[j] = x;
  }
  int cell_of[15];
  bool ok = true;
  for (int j = 0; j < 15; ++j) {
    cell_of[j] = host_cell(t[j]);
    if (cell_of[j] < 0 || cell_of[j] > 32) ok = false;
    if (j && cell_of[j] <= cell_of[j - 1]) ok = false;     // at most one threshold per cell
    if (j && !(t[j] > t[j - 1])) ok = false;
  }
  for (int c = 0; c <= 32; ++c) {
    uint32_t base = 0;
    float thr = 3.0f;
    for (int j = 0; j < 15; ++j) {
      if (cell_of[j] < c) ++base;
      if (cell_of[j] == c) thr = t[j];
    }
    L.thr[c] = thr;
    std::memcpy(&L.base[c], &base, 4);
  }
  g_lut_ok = ok;
  return L;
}

static const QuantLut& quant_lut() {
  static QuantLut lut;
  static std::once_flag once;
  std::call_once(once, [] { lut = build_lut(); });
  return lut;
}

bool quant_lut_valid() {
  quant_lut();
  return g_lut_ok;
}

void quant_thresholds(float out[15]) {
  // the decision thresholds t_j, recovered from the cell table (host only)
  const QuantLut& L = quant_lut();
  int j = 0;
  for (int c = 0; c <= 32 && j < 15; ++c)
    if (L.thr[c] < 2.0f) out[j++] = L.thr[c];
}

// ----------------------------------------------------------------------------
// Quantisation kernel
// ----------------------------------------------------------------------------
// xn = RN32(w / s).  For a block scale in [2^-60, 2^60] this uses the
// correctly rounded reciprocal r = RN32(1/s) and one residual correction
// (Markstein's final division step: y = RN(w r); e = fma(-s, y, w);
// q = fma(e, r, y)).  For bf16 operands this equals IEEE division whenever
// |w/s| >= 2^-102 (checked exhaustively over all bf16 significand pairs);
// smaller quotients all map to the exact-zero code either way.  Outside that
// scale range the kernel falls back to IEEE division.
//
// Two-lane fp32 arithmetic (sm_100 packed f32x2): each lane is one IEEE
// round-to-nearest fp32 operation, so a pair gives the same bits as two
// scalar operations for half the instructions.
__device__ __forceinline__ void mul2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2,%3};\n\tmov.b64 b, {%4,%5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0,%1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fma2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                        float c1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2,%3};\n\tmov.b64 b, {%4,%5};\n\tmov.b64 c, {%6,%7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0,%1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// One thread handles 16 consecutive weights (two 16-byte loads); 4 lanes share
// a 64-weight block.  The cell table is replicated 16 times with a stride that
// puts copy i on bank pair i, and lane l reads copy l % 16, so every lookup of
// a half-warp hits 16 distinct bank pairs (no bank conflicts).
template <bool kDQ>
__global__ void __launch_bounds__(256) k_nf4_quant(const uint16_t* __restrict__ W, int64_t N,
                                                   uint8_t* __restrict__ codes, float* __restrict__ absmax_f32,
                                                   uint16_t* __restrict__ absmax_bf16,
                                                   unsigned long long* __restrict__ hist, const QuantLut lut) {
  __shared__ float2 s_lut[33 * 16];
  __shared__ uint32_t s_hist[256];
  const int tid = threadIdx.x;
  for (int i = tid; i < 33 * 16; i += 256) s_lut[i] = make_float2(lut.thr[i >> 4], lut.base[i >> 4]);
  if (kDQ) s_hist[tid] = 0;
  __syncthreads();
  griddep_launch_dependents();
  griddep_wait();

  const int lane = tid & 31;
  // byte address of cell c in this lane's copy is lut_lane + 128 c; with
  // c = bits(y) - kCellBiasBits the subtraction folds into the base (mod 2^32)
  const uint32_t lut_lane = smem_u32(s_lut) + 8u * static_cast<uint32_t>(lane & 15) - 128u * kCellBiasBits;
  const int64_t ngroups = (N + 15) >> 4;                     // groups of 16 elements
  const int64_t stride = static_cast<int64_t>(gridDim.x) * 256;
  for (int64_t g0 = static_cast<int64_t>(blockIdx.x) * 256 + (tid & ~31); g0 < ngroups; g0 += stride) {
    const int64_t g = g0 + lane;
    const int64_t e0 = g << 4;
    float w[16];
    const bool full = (e0 + 16 <= N);
    if (full) {
      const uint4 v0 = ldg_nc_v4(W + e0);
      const uint4 v1 = ldg_nc_v4(W + e0 + 8);
      const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        w[2 * i] = bf16_lo(u[i]);
        w[2 * i + 1] = bf16_hi(u[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        w[i] = (e0 + i < N) ? __uint_as_float(static_cast<uint32_t>(W[e0 + i]) << 16) : 0.0f;
    }
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(w[i]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    const float s = am;   // block absmax (bf16-exact)

    uint32_t lo = 0x77777777u, hi = 0x77777777u;   // exact-zero code for an all-zero block
    if (s != 0.0f) {
      const bool fast = (s >= 0x1p-60f) && (s <= 0x1p60f);
      const float r = __frcp_rn(s);
      float xn[16];
      if (fast) {
        // y = RN(w r), e = fma(-s, y, w), xn = fma(e, r, y), two weights at a time
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          float y0, y1, e0, e1;
          mul2_rn(y0, y1, w[i], w[i + 1], r, r);
          fma2_rn(e0, e1, -s, -s, y0, y1, w[i], w[i + 1]);
          fma2_rn(xn[i], xn[i + 1], e0, e1, r, r, y0, y1);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) xn[i] = __fdiv_rn(w[i], s);
      }
      lo = 0;
      hi = 0;
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        float y0, y1;
        fma2_rn(y0, y1, xn[i], xn[i + 1], 16.0f, 16.0f, kCellBias, kCellBias);
        float2 e0, e1;
        asm("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(e0.x), "=f"(e0.y) : "r"(lut_lane + __float_as_uint(y0) * 128u));
        asm("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(e1.x), "=f"(e1.y) : "r"(lut_lane + __float_as_uint(y1) * 128u));
        const uint32_t q0 = __float_as_uint(e0.y) + (xn[i] > e0.x ? 1u : 0u);
        const uint32_t q1 = __float_as_uint(e1.y) + (xn[i + 1] > e1.x ? 1u : 0u);
        if (i < 8) lo += (q0 << (4 * i)) + (q1 << (4 * i + 4));
        else hi += (q0 << (4 * (i - 8))) + (q1 << (4 * (i - 8) + 4));
      }
    }
    if (e0 < N) {
      if (full) {
        uint32_t* c32 = reinterpret_cast<uint32_t*>(codes + (e0 >> 1));
        c32[0] = lo;
        c32[1] = hi;
      } else {
        const int valid = static_cast<int>(N - e0);             // 1..15
        const uint64_t all = (static_cast<uint64_t>(hi) << 32) | lo;
        const uint64_t packed = all & ((1ull << (4 * valid)) - 1ull);   // pad nibbles are 0
        const int nbytes = (valid + 1) >> 1;
        for (int b = 0; b < nbytes; ++b) codes[(e0 >> 1) + b] = static_cast<uint8_t>(packed >> (8 * b));
      }
      if ((g & 3) == 0) {
        const int64_t blk = e0 >> 6;
        if (kDQ) {
          const uint32_t bits = __float_as_uint(s);
          absmax_bf16[blk] = static_cast<uint16_t>(bits >> 16);
          const uint32_t E = (bits >> 23) & 0xFFu;
          const uint32_t m = (bits >> 16) & 0x7Fu;
          atomicAdd(&s_hist[E], E ? (128u + m) : m);
        } else {
          absmax_f32[blk] = s;
        }
      }
    }
  }
  if (kDQ) {
    __syncthreads();
    const uint32_t h = s_hist[tid];
    if (h) atomicAdd(&hist[tid], static_cast<unsigned long long>(h));
  }
}

__global__ void k_zero_u64(unsigned long long* p, int n) {
  griddep_launch_dependents();
  griddep_wait();   // the previous call's constants kernel may still read the histogram
  for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = 0ull;
}

// ----------------------------------------------------------------------------
// Exact mean of the block scales.  Each scale is a bf16 value
// sig * 2^(max(E,1) - 134) with an 8-bit significand; the histogram holds, per
// exponent field E, the exact integer sum of significands.  The total is an
// integer multiple of 2^-133 below 2^384: one warp accumulates it in twelve
// 32-bit limbs (each lane takes the exponents lane + 32m, whose limb index is
// m or m - 1, so the limb array stays in registers), reduces the limbs across
// the warp, and lane 0 propagates carries and rounds once to fp64 (nearest,
// ties to even); then mean = RN32(RN64(sum) / M_b).
// ----------------------------------------------------------------------------
__device__ float exact_mean_warp(const unsigned long long* __restrict__ hist, int64_t nblocks) {
  const int lane = threadIdx.x & 31;
  unsigned long long acc[12];
#pragma unroll
  for (int j = 0; j < 12; ++j) acc[j] = 0ull;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int E = lane + 32 * m;
    const unsigned long long v = __ldcg(hist + E);
    const int sh = (E ? E : 1) - 1;
    const int bo = sh & 31;
    const unsigned long long p0 = (v << bo) & 0xFFFFFFFFull;
    const unsigned long long p1 = (v >> (32 - bo)) & 0xFFFFFFFFull;
    const unsigned long long p2 = bo ? (v >> (64 - bo)) : 0ull;
    if ((sh >> 5) == m) {
      acc[m] += p0;
      acc[m + 1] += p1;
      acc[m + 2] += p2;
    } else if (m > 0) {   // lane 0, m >= 1: limb index m - 1
      acc[m - 1] += p0;
      acc[m] += p1;
      acc[m + 1] += p2;
    }
  }
#pragma unroll
  for (int j = 0; j < 12; ++j)
#pragma unroll
    for (int o = 16; o; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
  float mean = 0.0f;
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < 11; ++j) {
      acc[j + 1] += acc[j] >> 32;
      acc[j] &= 0xFFFFFFFFull;
    }
    unsigned long long Wd[6];
#pragma unroll
    for (int i = 0; i < 6; ++i) Wd[i] = acc[2 * i] | (acc[2 * i + 1] << 32);
    int top = -1;
#pragma unroll
    for (int i = 5; i >= 0; --i)
      if (top < 0 && Wd[i]) top = 64 * i + 63 - __clzll(static_cast<long long>(Wd[i]));
    double S = 0.0;
    if (top >= 0 && top < 53) {
      S = ldexp(static_cast<double>(Wd[0]), -133);   // exact
    } else if (top >= 53) {
      auto bits = [&](int lo) -> unsigned long long {   // 64 bits starting at bit `lo`
        const int w = lo >> 6, b = lo & 63;
        unsigned long long x = Wd[w] >> b;
        if (b && w + 1 < 6) x |= Wd[w + 1] << (64 - b);
        return x;
      };
      unsigned long long m = bits(top - 52) & ((1ull << 53) - 1ull);
      const int rpos = top - 53;
      const bool rbit = (bits(rpos) & 1ull) != 0;
      bool sticky = false;
      const int rw = rpos >> 6;
      for (int i = 0; i < rw; ++i) sticky |= (Wd[i] != 0);
      sticky |= (Wd[rw] & ((1ull << (rpos & 63)) - 1ull)) != 0;
      if (rbit && (sticky || (m & 1ull))) ++m;   // ties to even; 2^53 stays exact
      S = ldexp(static_cast<double>(m), top - 52 - 133);
    }
    mean = __double2float_rn(__ddiv_rn(S, static_cast<double>(nblocks)));
  }
  return __shfl_sync(0xffffffffu, mean, 0);
}

// ----------------------------------------------------------------------------
// Double quantisation of the scales: one warp per group of 256.
// ----------------------------------------------------------------------------
// kFP8: the constants are E4M3 bytes, c1 = RN32(448 / max|v|) and
// c2 = E4M3(RN32(c1 v)) rounded to nearest even, saturating at 448 (c1 v can
// pass 448 only by an fp32 rounding).  Otherwise symmetric Int8 as above.
template <bool kFP8>
__global__ void __launch_bounds__(256) k_dq_groups(const uint16_t* __restrict__ absmax_bf16, int64_t nblocks,
                                                   const unsigned long long* __restrict__ hist,
                                                   float* __restrict__ mean_out, int8_t* __restrict__ c2,
                                                   float* __restrict__ c1) {
  __shared__ float s_mean;
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    const float m = exact_mean_warp(hist, nblocks);   // every CTA derives the same value
    if (lane == 0) {
      s_mean = m;
      if (blockIdx.x == 0) *mean_out = m;
    }
  }
  __syncthreads();
  const int64_t ngroups = (nblocks + 255) >> 8;
  const float mu = s_mean;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); g < ngroups;
       g += static_cast<int64_t>(gridDim.x) * 8) {
    const int64_t j0 = g * 256 + lane * 8;
    float v[8];
    float am = 0.0f;
    if (j0 + 8 <= nblocks) {
      uint4 raw = ldg_nc_v4(absmax_bf16 + j0);
      const uint32_t r4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __fsub_rn(bf16_lo(r4[i]), mu);
        v[2 * i + 1] = __fsub_rn(bf16_hi(r4[i]), mu);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        v[i] = (j0 + i < nblocks)
                   ? __fsub_rn(__uint_as_float(static_cast<uint32_t>(absmax_bf16[j0 + i]) << 16), mu)
                   : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
#pragma unroll
    for (int o = 16; o; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    const float c = (am == 0.0f) ? 1.0f : __fdiv_rn(kFP8 ? 448.0f : 127.0f, am);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t b;
      if (kFP8) {
        b = static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fmul_rn(c, v[i]), __NV_SATFINITE, __NV_E4M3));
      } else {
        int q = 0;
        if (am != 0.0f) {
          q = __float2int_rn(__fmul_rn(c, v[i]));
          q = max(-127, min(127, q));
        }
        b = static_cast<uint32_t>(q) & 0xFFu;
      }
      if (i < 4) lo |= b << (8 * i);
      else hi |= b << (8 * (i - 4));
    }
    if (j0 + 8 <= nblocks) {
      *reinterpret_cast<uint2*>(c2 + j0) = make_uint2(lo, hi);
    } else {
      for (int i = 0; i < 8; ++i)
        if (j0 + i < nblocks)
          c2[j0 + i] = static_cast<int8_t>(((i < 4) ? (lo >> (8 * i)) : (hi >> (8 * (i - 4)))) & 0xFFu);
    }
    if (lane == 0) c1[g] = c;
  }
}

// ----------------------------------------------------------------------------
// Standalone double dequantisation: W_out[i] = BF16(RN32(C[q_i] * s^_j)).
//
// One thread per 64-weight block: its 32 code bytes are loaded first (two
// 16-byte loads when the codes are 16-byte aligned, else eight 4-byte loads),
// so every thread keeps 32 bytes in flight; s^ is computed once per block;
// the block's 16 values T[j] = BF16(RN32(C[j] * s^)) are built in registers
// and each 4-bit code is resolved with byte permutes (the GEMMs' expansion,
// bit-identical to the per-weight formula); the block's 128 bytes go out as
// eight 16-byte stores.  A ragged last block (N % 64 != 0) is expanded element
// by element.
// ----------------------------------------------------------------------------
// kDQ: 0 = fp32 absmax per block, 1 = Int8 c2, 2 = E4M3 c2.
template <int kDQ>
__device__ __forceinline__ float dequant_scale(int64_t blk, const float* __restrict__ absmax,
                                               const int8_t* __restrict__ c2, const float* __restrict__ c1, float mu) {
  if (kDQ == 1) return __fadd_rn(__fdiv_rn(static_cast<float>(__ldg(c2 + blk)), __ldg(c1 + (blk >> 8))), mu);
  if (kDQ == 2) {
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(__ldg(c2 + blk)), __NV_E4M3);
    return __fadd_rn(__fdiv_rn(__half2float(__half(hr)), __ldg(c1 + (blk >> 8))), mu);   // E4M3 -> fp32 is exact
  }
  return __ldg(absmax + blk);
}

template <int kDQ, bool kVec16>
__global__ void __launch_bounds__(256, 4) k_nf4_dequant(const uint8_t* __restrict__ codes, int64_t N,
                                                     const float* __restrict__ absmax, const int8_t* __restrict__ c2,
                                                     const float* __restrict__ c1, const float* __restrict__ mean,
                                                     uint16_t* __restrict__ out) {
  constexpr uint32_t kCB[16] = {QLORA_NF4_TABLE_BITS};
  float C[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) C[j] = __uint_as_float(kCB[j]);
  griddep_launch_dependents();
  griddep_wait();
  const float mu = kDQ ? __ldg(mean) : 0.0f;
  const int64_t nfull = N >> 6;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t blk = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; blk < nfull; blk += stride) {
    const uint8_t* src = codes + (blk << 5);
    uint32_t cw[8];
    if (kVec16) {
      const uint4 a = ldg_nc_v4(src), b = ldg_nc_v4(src + 16);
      cw[0] = a.x; cw[1] = a.y; cw[2] = a.z; cw[3] = a.w;
      cw[4] = b.x; cw[5] = b.y; cw[6] = b.z; cw[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) cw[i] = __ldg(reinterpret_cast<const unsigned int*>(src) + i);
    }
    const Nf4Tab tab = make_tab(dequant_scale<kDQ>(blk, absmax, c2, c1, mu), C);
    uint4* dst = reinterpret_cast<uint4*>(out + (blk << 6));
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = dq8(cw[i], tab);
  }
  // ragged last block: the elements past 64 * nfull, eight per thread of CTA 0
  const int64_t e0 = (nfull << 6) + 8 * static_cast<int64_t>(threadIdx.x);
  if (blockIdx.x == 0 && threadIdx.x < 8 && e0 < N) {
    const Nf4Tab tab = make_tab(dequant_scale<kDQ>(nfull, absmax, c2, c1, mu), C);
    uint32_t cw = 0;
    for (int64_t b = e0 >> 1; b < ((N + 1) >> 1) && b < (e0 >> 1) + 4; ++b)
      cw |= static_cast<uint32_t>(codes[b]) << (8 * (b - (e0 >> 1)));
    const uint4 v = dq8(cw, tab);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    for (int i = 0; i < 8 && e0 + i < N; ++i) out[e0 + i] = static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1)));
  }
}

// ----------------------------------------------------------------------------
// Host launchers
// ----------------------------------------------------------------------------
static int grid_for(int64_t nthreads) {
  int64_t ctas = (nthreads + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (ctas > cap) ctas = cap;
  if (ctas < 1) ctas = 1;
  return static_cast<int>(ctas);
}

size_t quant_workspace_bytes(int64_t N, bool dq) {
  if (!dq) return 0;
  const int64_t nblk = (N + 63) / 64;
  return 256 * sizeof(unsigned long long) + align_up(static_cast<size_t>(nblk) * 2 + 16, 256);
}

cudaError_t launch_quantize(const uint16_t* W, int64_t N, const qlora_nf4_t& q, void* ws, cudaStream_t st) {
  const int grid = grid_for((N + 15) / 16);
  const int64_t nblk = (N + 63) / 64;
  if (!q.double_quant) {
    {
      ProfScope ps_(QLORA_KC_QUANT, st);
      const cudaError_t e = launch_pdl(k_nf4_quant<false>, dim3(grid), dim3(256), 0, st, nullptr, W, N, q.codes,
                                       q.absmax, static_cast<uint16_t*>(nullptr),
                                       static_cast<unsigned long long*>(nullptr), quant_lut());
      if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
  }
  auto* hist = static_cast<unsigned long long*>(ws);
  auto* amax16 = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + 256 * sizeof(unsigned long long));
  {
    ProfScope ps_(QLORA_KC_DQ_CONST, st);
    const cudaError_t e = launch_pdl(k_zero_u64, dim3(1), dim3(256), 0, st, nullptr, hist, 256);
    if (e != cudaSuccess) return e;
  }
  {
    ProfScope ps_(QLORA_KC_QUANT, st);
    const cudaError_t e = launch_pdl(k_nf4_quant<true>, dim3(grid), dim3(256), 0, st, nullptr, W, N, q.codes,
                                     static_cast<float*>(nullptr), amax16, hist, quant_lut());
    if (e != cudaSuccess) return e;
  }
  const int64_t ngroups = (nblk + 255) / 256;
  {
    ProfScope ps_(QLORA_KC_DQ_CONST, st);
    // every CTA derives the mean itself, so keep the grid near one wave and loop over groups
    const int64_t want = (ngroups + 7) / 8;
    const int grid_g = static_cast<int>(want < 2 * num_sms() ? want : 2 * num_sms());
    const cudaError_t e =
        q.double_quant == 2
            ? launch_pdl(k_dq_groups<true>, dim3(grid_g), dim3(256), 0, st, nullptr, amax16, nblk, hist, q.mean, q.c2,
                         q.c1)
            : launch_pdl(k_dq_groups<false>, dim3(grid_g), dim3(256), 0, st, nullptr, amax16, nblk, hist, q.mean,
                         q.c2, q.c1);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <int kDQ>
static cudaError_t launch_dequant_mode(const qlora_nf4_t& q, int64_t N, uint16_t* out, int grid, cudaStream_t st) {
  const float* absmax = kDQ ? nullptr : q.absmax;
  const int8_t* c2 = kDQ ? q.c2 : nullptr;
  const float* c1 = kDQ ? q.c1 : nullptr;
  const float* mean = kDQ ? q.mean : nullptr;
  const bool vec16 = (reinterpret_cast<uintptr_t>(q.codes) & 15u) == 0;
  return vec16 ? launch_pdl(k_nf4_dequant<kDQ, true>, dim3(grid), dim3(256), 0, st, nullptr, q.codes, N, absmax, c2,
                            c1, mean, out)
               : launch_pdl(k_nf4_dequant<kDQ, false>, dim3(grid), dim3(256), 0, st, nullptr, q.codes, N, absmax, c2,
                            c1, mean, out);
}

cudaError_t launch_dequantize(const qlora_nf4_t& q, int64_t N, uint16_t* out, cudaStream_t st) {
  const int grid = grid_for(N >> 6 > 0 ? N >> 6 : 1);   // one thread per complete 64-weight block
  ProfScope ps_(QLORA_KC_DEQUANT, st);
  const cudaError_t e = q.double_quant == 2 ? launch_dequant_mode<2>(q, N, out, grid, st)
                        : q.double_quant    ? launch_dequant_mode<1>(q, N, out, grid, st)
                                            : launch_dequant_mode<0>(q, N, out, grid, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Quantisation with library-owned scratch (nf4_quantize_noalloc).
//
// Double quantisation needs device scratch between its kernels: the 256-entry
// exponent histogram of the block scales and a bf16 copy of every block scale.
// nf4_quantize takes that scratch from the caller.  Some callers have no way to
// provide it: a plugin running inside a host application whose memory manager
// owns all device memory, or a service that reserves its memory up front and
// must not call cudaMalloc later (it can synchronize the device and can fail
// once memory is fragmented).  For them the scratch lives in the file-scope
// array below, sized for QLORA_NOALLOC_MAX_WEIGHTS weights (about 8 MiB, held by
// every GPU that loads the library until the process exits).
//
// Host code must not pass the array's name to a kernel: on the host that name
// is only a stand-in, not a device address.  Every call asks the runtime for
// the real address with cudaGetSymbolAddress, with the call's device current.
// That is a host-side lookup (it allocates nothing); the first one on a device
// may load the library's device code there.  The address is not cached: after
// the caller destroys and recreates the device's context (cudaDeviceReset, for
// instance) the module is loaded again and the array may sit elsewhere, and a
// cached address would then point at freed memory.
// ----------------------------------------------------------------------------
constexpr size_t noalloc_scratch_bytes() {
  return 256 * sizeof(unsigned long long) +
         ((static_cast<size_t>(QLORA_NOALLOC_MAX_WEIGHTS / 64) * 2 + 16 + 255) / 256) * 256;
}

static __device__ __align__(256) unsigned char g_noalloc_scratch[noalloc_scratch_bytes()];

cudaError_t noalloc_scratch(void** out, size_t* bytes) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  *bytes = noalloc_scratch_bytes();
  return cudaSuccess;
}

}  // namespace qlora
