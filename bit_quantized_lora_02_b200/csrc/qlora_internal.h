// qlora_internal.h -- host-side declarations shared by the library's sources.
#pragma once

#include <cstddef>
#include <cstdint>

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
// device address and size of the library-owned quantisation scratch (current device)
cudaError_t noalloc_scratch(void** out, size_t* bytes);

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
};

size_t fwd_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r);
size_t bwd_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r);
// Returns 0 on success, a negative qlora_status otherwise; `why` names the failure.
int launch_linear_fwd(const LinearArgs& a, cudaStream_t st, const char** why);
int launch_linear_bwd(const LinearArgs& a, cudaStream_t st, const char** why);

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
