// nf4_scale.cuh -- the per-block scale s^ of the NF4 weight inside the GEMM
// kernels.
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora), "Double quantization
// and double dequantization": with double quantization each 64-weight block
// stores an 8-bit c2 and each group of 256 blocks an fp32 c1; the block scale
// is rebuilt as c2 / c1 plus the mean that was subtracted before the second
// quantisation.  Without it the fp32 absmax is stored directly.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace qlora {

// Block scale s^ for NF4 block `blk`.
struct ScaleSrc {
  const float* absmax;   // DQ off
  const int8_t* c2;      // DQ on
  const float* c1;
  const float* mean;     // device scalar, DQ on
  int dq;
};

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
// for every fp32 significand of c1 (checked exhaustively on the host); outside
// that range the IEEE division is used.
struct ScaleRecip {
  float c1 = 0.0f;   // constant the reciprocal belongs to (0 never occurs: c1 > 0)
  float rc = 0.0f;
  bool fast = false;
};

__device__ __forceinline__ float scale_value(int dq, float mean, ScaleRaw r, ScaleRecip& rec) {
  if (!dq) return r.a;
  if (r.a != rec.c1) {
    rec.c1 = r.a;
    rec.rc = __frcp_rn(r.a);
    rec.fast = (r.a >= 0x1p-60f) && (r.a <= 0x1p60f);
  }
  const float w = static_cast<float>(r.b);
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

}  // namespace qlora
