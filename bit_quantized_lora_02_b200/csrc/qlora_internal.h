// qlora_internal.h -- host-side declarations shared by the library's sources.
#pragma once

#include <cstddef>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/qlora.h"

namespace qlora {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int num_sms();                    // SM count of the current device (cached per device)

// NF4 table and the code-search table (nf4_quant.cu)
void host_codebook(float out[16]);
bool quant_lut_valid();
void quant_thresholds(float out[15]);

// quantize / dequantize (nf4_quant.cu)
size_t quant_workspace_bytes(int64_t N, bool dq);
cudaError_t launch_quantize(const uint16_t* W, int64_t N, const qlora_nf4_t& q, void* ws, cudaStream_t st);
cudaError_t launch_dequantize(const qlora_nf4_t& q, int64_t N, uint16_t* out, cudaStream_t st);
cudaError_t launch_lora_merge(const qlora_nf4_t& q, const uint16_t* A, const uint16_t* B, int r, float s,
                              uint16_t* out, cudaStream_t st);
// device address and size of the library-owned quantisation scratch (current device)
cudaError_t noalloc_scratch(void** out, size_t* bytes);

// adapter dropout (qlora_dropout.cu)
struct DropoutArgs {
  float p;           // drop probability, 0 <= p < 1
  uint32_t thr;      // ceil(p * 2^24): a 24-bit draw at or above it keeps the element
  float dscale;      // RN32(1 / RN32(1 - p)), the scale of kept elements
  uint64_t seed, offset;
};
uint32_t dropout_threshold(float p);
// keep bitmask of n elements (bit b of word w <-> element 32 w + b) into bits[ceil(n / 32)]
cudaError_t launch_dropout_bits(int64_t n, const DropoutArgs& d, uint32_t* bits, cudaStream_t st);
// dX (M x k, bf16, in place) += dscale * keep . (U A), U = U_s (M x rp), A (r x k)
cudaError_t launch_lora_up_dropout(const uint16_t* U, int rp, const uint16_t* A, int r, const uint32_t* keep,
                                   float dscale, int64_t M, int64_t k, uint16_t* dX, cudaStream_t st);

// linear layer (qlora_gemm.cu)
struct LinearArgs {
  const uint16_t* X;    // M x k
  const uint16_t* dY;   // M x d (backward)
  int64_t M, d, k;
  const qlora_nf4_t* q;
  const uint16_t* A;    // r x k
  const uint16_t* B;    // d x r
  int32_t r, rp;        // rank and padded rank (multiple of 64)
  float s;              // alpha / r in fp32
  uint16_t* Y;          // M x d
  uint16_t* T;          // M x rp, bf16(s X A^T)
  const uint16_t* Tin;  // backward: saved T (or nullptr)
  uint16_t* dX;         // M x k
  float* dA;            // r x k
  float* dB;            // d x r
  void* ws;
  size_t ws_bytes;
  // adapter dropout (drop == nullptr: none).  The keep bitmask lives in the
  // workspace past the plain layer's part, at dropout_mask_offset().
  const DropoutArgs* drop;
  // Grouped projections sharing X: q stacks ngrp projections (rows from
  // gstart[i] on belong to projection i + 1, each with its own mean); r is the
  // rank of all of them together (A, T_s, U_s, dA stack the projections'
  // ranks), r_group the rank of one; B and dB are (d x r_group) with the
  // projections' rows stacked.  A plain layer has ngrp = 0 and r_group = r.
  int32_t r_group;
  int32_t ngrp;
  int64_t gstart[3];
};

size_t fwd_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r);
size_t bwd_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r);
// with adapter dropout: the plain layer's workspace, then the keep bitmask of X
size_t dropout_mask_offset(int64_t M, int64_t d, int64_t k, int32_t r, bool bwd);
size_t dropout_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r, bool bwd);
// Returns 0 on success, a negative qlora_status otherwise; `why` names the failure.
int launch_linear_fwd(const LinearArgs& a, cudaStream_t st, const char** why);
int launch_linear_bwd(const LinearArgs& a, cudaStream_t st, const char** why);

// few-token forward (qlora_fewtok.cu): M <= kFewTokMax tokens, weights streamed
// once with register-resident dequantisation.  `tm_codes` maps the packed codes
// as (k/2 bytes) x d rows, box 128 x 256, 128-byte swizzle.
constexpr int kFewTokMax = 16;
bool fewtok_eligible(int64_t M, int64_t d, int64_t k);
size_t fewtok_workspace_bytes(int64_t M, int64_t d, int64_t k, int rp);
int launch_fewtok_fwd(const LinearArgs& a, uint16_t* T, void* ws, const CUtensorMap* tm_codes, cudaStream_t st,
                      const char** why, const uint32_t* keep);

// Raise a kernel's dynamic shared-memory limit once per (kernel, device); the
// attribute call costs host time on every launch otherwise.  Instantiations of
// one kernel template share a function type, so the key is the address.
// Launch with programmatic dependent launch allowed (the kernel calls
// griddep_wait() before touching memory) and, when `cluster` is given, as
// thread-block clusters of that shape.
template <typename... ExpTypes, typename... ActTypes>
cudaError_t launch_pdl(void (*kernel)(ExpTypes...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       const dim3* cluster, ActTypes&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster->x;
    attr[n].val.clusterDim.y = cluster->y;
    attr[n].val.clusterDim.z = cluster->z;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<ActTypes&&>(args)...);
}

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, uint32_t> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const std::pair<const void*, int> key(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

// tracing (qlora_prof.cu): construct around each kernel launch
struct ProfScope {
  int kc;
  cudaStream_t st;
  void* a;
  ProfScope(int kc, cudaStream_t st);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;
};

// status word (qlora_abi.cu)
cudaError_t read_and_clear_status(int* out);

}  // namespace qlora
