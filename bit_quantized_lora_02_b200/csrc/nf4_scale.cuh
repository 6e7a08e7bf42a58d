// nf4_scale.cuh -- the per-block scale s^ of the NF4 weight and the expansion
// of a block's codes to bf16, shared by the GEMM and merge kernels.
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora), "Double quantization
// and double dequantization": with double quantization each 64-weight block
// stores an 8-bit c2 and each group of 256 blocks an fp32 c1; the block scale
// is rebuilt as c2 / c1 plus the mean that was subtracted before the second
// quantisation.  Without it the fp32 absmax is stored directly.
#pragma once

#include <cstdint>

#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "qlora_device.cuh"

namespace qlora {

// Block scale s^ for NF4 block `blk`.
//
// A grouped weight stacks the NF4 buffers of up to four projections that share
// their input (q, k, v or gate, up), each quantised on its own: codes, c2 (or
// absmax) and c1 are laid out back to back, and each projection keeps its own
// mean.  Rows from gstart[i] on belong to projection i + 1; a plain weight has
// ngrp <= 1 and reads mean[0].
struct ScaleSrc {
  const float* absmax;   // DQ off
  const int8_t* c2;      // DQ on
  const float* c1;
  const float* mean;     // device, one per projection, DQ on
  int dq;
  int ngrp;              // projections stacked in the weight (0 or 1: a plain weight)
  int64_t gstart[3];     // first row of projections 1, 2, 3
};

// Projection that weight row `row` belongs to.
__host__ __device__ __forceinline__ int group_of(const ScaleSrc& s, int64_t row) {
  int g = 0;
#pragma unroll
  for (int j = 0; j < 3; ++j) g += (j + 1 < s.ngrp && row >= s.gstart[j]) ? 1 : 0;
  return g;
}

__device__ __forceinline__ float group_mean(const ScaleSrc& s, int64_t row) {
  return s.dq ? __ldg(s.mean + group_of(s, row)) : 0.0f;
}

struct ScaleRaw {
  float a;   // absmax (DQ off) or c1 (DQ on)
  int b;     // c2
};

__device__ __forceinline__ ScaleRaw scale_fetch(const ScaleSrc& s, int64_t blk) {
  ScaleRaw r;
  if (s.dq) {
    r.b = __ldg(s.c2 + blk);
    r.a = __ldg(s.c1 + (blk >> 8));
  } else {
    r.a = __ldg(s.absmax + blk);
    r.b = 0;
  }
  return r;
}

// s^ = RN32(RN32(c2 / c1) + mean) with DQ, else the stored absmax.
//
// The quotient uses the correctly rounded reciprocal rc = RN32(1/c1), kept
// while consecutive blocks share their group constant (a group spans 256
// blocks, so it changes rarely), and one residual correction:
//     y = RN(c2 rc);  e = fma(-c1, y, c2);  q = fma(e, rc, y).
// For integer |c2| <= 127 and c1 in [2^-60, 2^60] this equals IEEE division
// for every fp32 significand of c1, and so it does for every finite E4M3 value
// as numerator (a zero numerator of either sign gives +0, which leaves
// RN(q + mean) unchanged); tests/host_checks/division_check.c checks both
// exhaustively.  Outside that range the IEEE division is used.
struct ScaleRecip {
  float c1 = 0.0f;   // constant the reciprocal belongs to (0 never occurs: c1 > 0)
  float rc = 0.0f;
  bool fast = false;
};

// c2 as the numerator: the int8 value, or the E4M3 byte decoded (exact).
__device__ __forceinline__ float c2_numerator(int dq, int c2) {
  if (dq == 2) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c2 & 0xFF), __NV_E4M3);
    return __half2float(__half(h));
  }
  return static_cast<float>(c2);
}

__device__ __forceinline__ float scale_value(int dq, float mean, ScaleRaw r, ScaleRecip& rec) {
  if (!dq) return r.a;
  if (r.a != rec.c1) {
    rec.c1 = r.a;
    rec.rc = __frcp_rn(r.a);
    rec.fast = (r.a >= 0x1p-60f) && (r.a <= 0x1p60f);
  }
  const float w = c2_numerator(dq, r.b);
  float q;
  if (rec.fast) {
    const float y = __fmul_rn(w, rec.rc);
    const float e = __fmaf_rn(-r.a, y, w);
    q = __fmaf_rn(e, rec.rc, y);
  } else {
    q = __fdiv_rn(w, r.a);
  }
  return __fadd_rn(q, mean);
}

// ============================================================================
// Expansion of one 64-weight NF4 block (into the GEMMs' swizzled W rows and
// the merged weight).
//
// The block's 16 reconstruction values T[j] = BF16(RN32(C[j] * s^)) are built
// once per block (bit-identical to BF16(C[q] * s^) per weight), split into four
// registers of low bytes and four of high bytes, and every 4-bit code is then
// resolved with byte permutes: PRMT selects by the code's low 3 bits from each
// half of the table and a sign-replicated mask of the code's top bit picks the
// half.  About 2.75 integer instructions per weight, no shared-memory lookups.
// ============================================================================
struct Nf4Tab {
  uint32_t L[4], H[4];
};

__device__ __forceinline__ Nf4Tab make_tab(float sh, const float (&C)[16]) {
  uint32_t P[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) P[i] = pack_bf16x2(__fmul_rn(C[2 * i], sh), __fmul_rn(C[2 * i + 1], sh));
  Nf4Tab t;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    t.L[i] = prmt(P[2 * i], P[2 * i + 1], 0x6420u);
    t.H[i] = prmt(P[2 * i], P[2 * i + 1], 0x7531u);
  }
  return t;
}

// 8 codes (code i in bits 4i..4i+3) -> 8 bf16 (element i in halfword i).
__device__ __forceinline__ uint4 dq8(uint32_t c, const Nf4Tab& t) {
  const uint32_t xl = c & 0x7777u;
  const uint32_t xh = (c >> 16) & 0x7777u;
  const uint32_t d4 = c << 4;
  const uint32_t ml = prmt(d4, c, 0xD9C8u);   // 0xFF in byte i iff code i >= 8 (i = 0..3)
  const uint32_t mh = prmt(d4, c, 0xFBEAu);   // same for codes 4..7
  uint4 o;
  {
    const uint32_t la = prmt(t.L[0], t.L[1], xl), lb = prmt(t.L[2], t.L[3], xl);
    const uint32_t ha = prmt(t.H[0], t.H[1], xl), hb = prmt(t.H[2], t.H[3], xl);
    const uint32_t lo = (la & ~ml) | (lb & ml);
    const uint32_t hi = (ha & ~ml) | (hb & ml);
    o.x = prmt(lo, hi, 0x5140u);
    o.y = prmt(lo, hi, 0x7362u);
  }
  {
    const uint32_t la = prmt(t.L[0], t.L[1], xh), lb = prmt(t.L[2], t.L[3], xh);
    const uint32_t ha = prmt(t.H[0], t.H[1], xh), hb = prmt(t.H[2], t.H[3], xh);
    const uint32_t lo = (la & ~mh) | (lb & mh);
    const uint32_t hi = (ha & ~mh) | (hb & mh);
    o.z = prmt(lo, hi, 0x5140u);
    o.w = prmt(lo, hi, 0x7362u);
  }
  return o;
}

}  // namespace qlora
