// qlora_abi.cu -- the extern "C" entry points declared in include/qlora.h:
// argument validation, buffer-size arithmetic, error reporting.  Every compute
// step runs in the kernels of nf4_quant.cu and qlora_gemm.cu.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "qlora_device.cuh"
#include "qlora_internal.h"

namespace qlora {

__device__ int g_status = 0;

// Self-test of the failure path every kernel's waits share: one CTA takes 32
// TMEM columns, then waits on an mbarrier that nothing ever arrives at with
// the same bounded loop as mbar_wait but a caller-chosen limit.  When the
// limit runs out it records DEV_WAIT_TIMEOUT_SELFTEST in the status word,
// releases its TMEM like any kernel winding down after a failed wait, and
// writes 2 to *result after the release (1 would mean the barrier completed,
// which cannot happen).  No fault, trap or endless loop is involved.
__global__ void k_selftest_wait_timeout(uint64_t limit_ns, int* result) {
  __shared__ uint64_t bar;
  __shared__ uint32_t slot;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&slot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = slot;
  int outcome = 0;
  if (threadIdx.x == 0) {
    const uint32_t a = smem_u32(&bar);
    const uint64_t t0 = globaltimer_ns();
    outcome = 2;
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_wait(a, 0)) {
        outcome = 1;
        break;
      }
      if ((it & 63u) == 0 && globaltimer_ns() - t0 > limit_ns) {
        report(DEV_WAIT_TIMEOUT_SELFTEST);
        abort_flag = 1;
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
  __syncthreads();
  if (threadIdx.x == 0) *result = outcome;
}

cudaError_t read_and_clear_status(int* out) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_status, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace qlora

using namespace qlora;

static thread_local std::string t_err;

static int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

static int ok() {
  t_err.clear();
  return QLORA_OK;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The library links its own CUDA runtime, whose current device is independent
// of the caller's runtime.  Make the device that owns `p` current before
// launching anything (kernels must run where the data lives).
static int bind_device(const void* p) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(QLORA_ERR_CUDA, "pointer attributes: %s", cudaGetErrorString(e));
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(QLORA_ERR_INVALID_ARG, "expected a device pointer");
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != attr.device) {
    e = cudaSetDevice(attr.device);
    if (e != cudaSuccess) return fail(QLORA_ERR_CUDA, "set device: %s", cudaGetErrorString(e));
  }
  return QLORA_OK;
}

static int check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(QLORA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// N = d * k without overflow, both non-negative.
static bool elem_count(int64_t d, int64_t k, int64_t* n) {
  if (d < 0 || k < 0) return false;
  if (d && k > INT64_MAX / 4 / d) return false;
  *n = d * k;
  return true;
}

static int check_nf4(const qlora_nf4_t* q, int64_t* N) {
  if (!q) return fail(QLORA_ERR_INVALID_ARG, "quantized weight descriptor is NULL");
  if (!elem_count(q->d, q->k, N)) return fail(QLORA_ERR_INVALID_ARG, "bad weight shape d=%lld k=%lld",
                                                (long long)q->d, (long long)q->k);
  if (q->blocksize != 64) return fail(QLORA_ERR_UNSUPPORTED, "blocksize %d not supported (64 only)", q->blocksize);
  if (q->double_quant < 0 || q->double_quant > 2)
    return fail(QLORA_ERR_INVALID_ARG, "double_quant must be 0, 1 or 2");
  if (*N == 0) return ok();
  if (!q->codes) return fail(QLORA_ERR_INVALID_ARG, "codes is NULL");
  if (!aligned(q->codes, 4)) return fail(QLORA_ERR_ALIGNMENT, "codes must be 4-byte aligned");
  if (q->double_quant) {
    if (!q->c2 || !q->c1 || !q->mean) return fail(QLORA_ERR_INVALID_ARG, "c2, c1 and mean are required with DQ");
    if (!aligned(q->c2, 8)) return fail(QLORA_ERR_ALIGNMENT, "c2 must be 8-byte aligned");
    if (!aligned(q->c1, 4) || !aligned(q->mean, 4)) return fail(QLORA_ERR_ALIGNMENT, "c1/mean must be 4-byte aligned");
  } else {
    if (!q->absmax) return fail(QLORA_ERR_INVALID_ARG, "absmax is required without DQ");
    if (!aligned(q->absmax, 4)) return fail(QLORA_ERR_ALIGNMENT, "absmax must be 4-byte aligned");
  }
  return ok();
}

extern "C" {

int qlora_nf4_sizes(int64_t d, int64_t k, int32_t blocksize, int32_t double_quant, size_t sizes[5],
                    size_t* quant_workspace_bytes_out) {
  int64_t N = 0;
  if (!sizes) return fail(QLORA_ERR_INVALID_ARG, "sizes is NULL");
  if (!elem_count(d, k, &N)) return fail(QLORA_ERR_INVALID_ARG, "bad weight shape");
  if (blocksize != 64) return fail(QLORA_ERR_UNSUPPORTED, "blocksize %d not supported (64 only)", blocksize);
  if (double_quant < 0 || double_quant > 2) return fail(QLORA_ERR_INVALID_ARG, "double_quant must be 0, 1 or 2");
  const int64_t nblk = ceil_div(N, 64);
  const int64_t ngrp = ceil_div(nblk, 256);
  sizes[QLORA_BUF_CODES] = static_cast<size_t>((N + 1) / 2);
  sizes[QLORA_BUF_ABSMAX] = double_quant ? 0 : static_cast<size_t>(nblk) * 4;
  sizes[QLORA_BUF_C2] = double_quant ? static_cast<size_t>(nblk) : 0;
  sizes[QLORA_BUF_C1] = double_quant ? static_cast<size_t>(ngrp) * 4 : 0;
  sizes[QLORA_BUF_MEAN] = double_quant ? (N ? 4 : 0) : 0;
  if (quant_workspace_bytes_out) *quant_workspace_bytes_out = quant_workspace_bytes(N, double_quant != 0);
  return ok();
}

int nf4_quantize(const uint16_t* W0, const qlora_nf4_t* q, void* workspace, size_t workspace_bytes,
                 qlora_stream_t stream) {
  int64_t N = 0;
  int rc = check_nf4(q, &N);
  if (rc) return rc;
  if (N == 0) return ok();
  if (!W0) return fail(QLORA_ERR_INVALID_ARG, "W0 is NULL");
  if (!aligned(W0, 16)) return fail(QLORA_ERR_ALIGNMENT, "W0 must be 16-byte aligned");
  if (q->double_quant) {
    const size_t need = quant_workspace_bytes(N, true);
    if (!workspace || workspace_bytes < need)
      return fail(QLORA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? workspace_bytes : 0);
    if (!aligned(workspace, 16)) return fail(QLORA_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  }
  if (!quant_lut_valid()) return fail(QLORA_ERR_UNSUPPORTED, "code-search table failed its self-check");
  if ((rc = bind_device(W0))) return rc;
  return check_cuda(launch_quantize(W0, N, *q, workspace, static_cast<cudaStream_t>(stream)), "nf4_quantize launch");
}

int nf4_quantize_noalloc(const uint16_t* W0, const qlora_nf4_t* q, qlora_stream_t stream) {
  int64_t N = 0;
  int rc = check_nf4(q, &N);
  if (rc) return rc;
  if (N == 0) return ok();
  if (!W0) return fail(QLORA_ERR_INVALID_ARG, "W0 is NULL");
  if (!aligned(W0, 16)) return fail(QLORA_ERR_ALIGNMENT, "W0 must be 16-byte aligned");
  if (N > QLORA_NOALLOC_MAX_WEIGHTS)
    return fail(QLORA_ERR_UNSUPPORTED,
                "nf4_quantize_noalloc: %lld weights exceed the built-in scratch limit of %lld; "
                "use nf4_quantize with a workspace",
                (long long)N, (long long)QLORA_NOALLOC_MAX_WEIGHTS);
  if (!quant_lut_valid()) return fail(QLORA_ERR_UNSUPPORTED, "code-search table failed its self-check");
  if ((rc = bind_device(W0))) return rc;
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (q->double_quant) {
    cudaError_t e = noalloc_scratch(&scratch, &scratch_bytes);
    if (e != cudaSuccess) return fail(QLORA_ERR_CUDA, "scratch address lookup: %s", cudaGetErrorString(e));
    if (scratch_bytes < quant_workspace_bytes(N, true))
      return fail(QLORA_ERR_UNSUPPORTED, "built-in scratch too small");
  }
  return check_cuda(launch_quantize(W0, N, *q, scratch, static_cast<cudaStream_t>(stream)),
                    "nf4_quantize_noalloc launch");
}

int nf4_dequantize(const qlora_nf4_t* q, uint16_t* W_out, qlora_stream_t stream) {
  int64_t N = 0;
  int rc = check_nf4(q, &N);
  if (rc) return rc;
  if (N == 0) return ok();
  if (!W_out) return fail(QLORA_ERR_INVALID_ARG, "W_out is NULL");
  if (!aligned(W_out, 16)) return fail(QLORA_ERR_ALIGNMENT, "W_out must be 16-byte aligned");
  if ((rc = bind_device(W_out))) return rc;
  return check_cuda(launch_dequantize(*q, N, W_out, static_cast<cudaStream_t>(stream)), "nf4_dequantize launch");
}

int32_t qlora_rank_pad(int32_t r) { return r <= 0 ? 0 : ((r + 63) / 64) * 64; }

static int check_linear_shape(int64_t M, int64_t d, int64_t k, int32_t r) {
  if (M < 0) return fail(QLORA_ERR_INVALID_ARG, "M must be >= 0");
  if (r < 1 || r > 256) return fail(QLORA_ERR_UNSUPPORTED, "rank r=%d outside 1..256", r);
  if (d <= 0 || k <= 0) return fail(QLORA_ERR_INVALID_ARG, "weight shape must be positive");
  if (k % 64) return fail(QLORA_ERR_UNSUPPORTED, "k=%lld must be a multiple of 64", (long long)k);
  if (d % 8) return fail(QLORA_ERR_UNSUPPORTED, "d=%lld must be a multiple of 8", (long long)d);
  if (M > (int64_t(1) << 31) || d > (int64_t(1) << 31) || k > (int64_t(1) << 31))
    return fail(QLORA_ERR_UNSUPPORTED, "dimension above 2^31");
  return ok();
}

int qlora_linear_workspace_size(int64_t M, int64_t d, int64_t k, int32_t r, int32_t backward, size_t* bytes) {
  if (!bytes) return fail(QLORA_ERR_INVALID_ARG, "bytes is NULL");
  int rc = check_linear_shape(M, d, k, r);
  if (rc) return rc;
  *bytes = backward ? bwd_workspace_bytes(M, d, k, r) : fwd_workspace_bytes(M, d, k, r);
  return ok();
}

// The tensor-core kernels read the packed codes with TMA: 16-byte alignment.
static int check_codes_tma(const qlora_nf4_t* q) {
  if (!aligned(q->codes, 16)) return fail(QLORA_ERR_ALIGNMENT, "codes must be 16-byte aligned for the linear layer");
  return QLORA_OK;
}

static int check_ptr16(const void* p, const char* name, bool required) {
  if (!p) return required ? fail(QLORA_ERR_INVALID_ARG, "%s is NULL", name) : ok();
  if (!aligned(p, 16)) return fail(QLORA_ERR_ALIGNMENT, "%s must be 16-byte aligned", name);
  return ok();
}

}  // extern "C"

// Adapter dropout arguments: p finite in [0, 1).  p == 0 (or no struct) is the
// plain layer, bit for bit.
static int check_dropout(const qlora_dropout_t* drop, DropoutArgs* out, bool* on) {
  *on = false;
  if (!drop) return QLORA_OK;
  const float p = drop->p;
  if (!(p >= 0.0f && p < 1.0f)) return fail(QLORA_ERR_INVALID_ARG, "dropout probability must lie in [0, 1)");
  if (p == 0.0f) return QLORA_OK;
  const float keep = 1.0f - p;   // RN32(1 - p)
  out->p = p;
  out->thr = dropout_threshold(p);
  out->dscale = 1.0f / keep;     // RN32(1 / RN32(1 - p))
  out->seed = drop->seed;
  out->offset = drop->offset;
  *on = true;
  return QLORA_OK;
}

static int linear_fwd(const uint16_t* X, int64_t M, const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B,
                      int32_t r, float alpha, const qlora_dropout_t* drop, uint16_t* Y, uint16_t* T_save,
                      void* workspace, size_t workspace_bytes, qlora_stream_t stream, const char* name) {
  DropoutArgs dargs{};
  bool dropping = false;
  int64_t N = 0;
  int rc = check_nf4(q, &N);
  if (rc) return rc;
  if ((rc = check_linear_shape(M, q->d, q->k, r))) return rc;
  if (M == 0) return ok();
  if ((rc = check_codes_tma(q))) return rc;
  if ((rc = check_ptr16(X, "X", true)) || (rc = check_ptr16(A, "A", true)) || (rc = check_ptr16(B, "B", true)) ||
      (rc = check_ptr16(Y, "Y", true)) || (rc = check_ptr16(T_save, "T_save", false)))
    return rc;
  if ((rc = check_dropout(drop, &dargs, &dropping))) return rc;
  const size_t need = dropping ? dropout_workspace_bytes(M, q->d, q->k, r, false) : fwd_workspace_bytes(M, q->d, q->k, r);
  if (need && (!workspace || workspace_bytes < need))
    return fail(QLORA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? workspace_bytes : 0);
  if (workspace && (rc = check_ptr16(workspace, "workspace", false))) return rc;
  if ((rc = bind_device(X))) return rc;
  LinearArgs a{};
  a.X = X; a.M = M; a.d = q->d; a.k = q->k; a.q = q; a.A = A; a.B = B; a.r = r; a.rp = qlora_rank_pad(r);
  a.s = alpha / static_cast<float>(r);
  a.Y = Y; a.T = T_save; a.ws = workspace; a.ws_bytes = workspace_bytes;
  a.drop = dropping ? &dargs : nullptr;
  const char* why = "";
  rc = launch_linear_fwd(a, static_cast<cudaStream_t>(stream), &why);
  if (rc) return fail(rc, "%s: %s", name, why);
  return ok();
}

static int linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_nf4_t* q, const uint16_t* A,
                      const uint16_t* B, int32_t r, float alpha, const qlora_dropout_t* drop, const uint16_t* T_save,
                      uint16_t* dX, float* dA, float* dB, void* workspace, size_t workspace_bytes,
                      qlora_stream_t stream, const char* name) {
  DropoutArgs dargs{};
  bool dropping = false;
  int64_t N = 0;
  int rc = check_nf4(q, &N);
  if (rc) return rc;
  if ((rc = check_linear_shape(M, q->d, q->k, r))) return rc;
  if ((rc = check_ptr16(dA, "dA", true)) || (rc = check_ptr16(dB, "dB", true))) return rc;
  if (M > 0 && (rc = check_codes_tma(q))) return rc;
  if ((rc = check_ptr16(dY, "dY", M > 0)) || (rc = check_ptr16(X, "X", M > 0)) || (rc = check_ptr16(A, "A", true)) ||
      (rc = check_ptr16(B, "B", true)) || (rc = check_ptr16(dX, "dX", false)) ||
      (rc = check_ptr16(T_save, "T_save", false)))
    return rc;
  if ((rc = check_dropout(drop, &dargs, &dropping))) return rc;
  const size_t need = dropping ? dropout_workspace_bytes(M, q->d, q->k, r, true) : bwd_workspace_bytes(M, q->d, q->k, r);
  if (need && (!workspace || workspace_bytes < need))
    return fail(QLORA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? workspace_bytes : 0);
  if (workspace && (rc = check_ptr16(workspace, "workspace", false))) return rc;
  if ((rc = bind_device(dA))) return rc;
  LinearArgs a{};
  a.dY = dY; a.X = X; a.M = M; a.d = q->d; a.k = q->k; a.q = q; a.A = A; a.B = B; a.r = r;
  a.rp = qlora_rank_pad(r);
  a.s = alpha / static_cast<float>(r);
  a.Tin = T_save; a.dX = dX; a.dA = dA; a.dB = dB; a.ws = workspace; a.ws_bytes = workspace_bytes;
  a.drop = dropping ? &dargs : nullptr;
  const char* why = "";
  rc = launch_linear_bwd(a, static_cast<cudaStream_t>(stream), &why);
  if (rc) return fail(rc, "%s: %s", name, why);
  return ok();
}

// Grouped projections: n projections that share X, their NF4 buffers stacked.
// Checks the group and fills the grouping fields of `a`; *d_total and *r_all
// are the stacked weight's rows and the projections' ranks together.
static int check_group(const qlora_nf4_group_t* g, int32_t r, LinearArgs* a) {
  if (!g) return fail(QLORA_ERR_INVALID_ARG, "group descriptor is NULL");
  if (g->n < 1 || g->n > QLORA_MAX_GROUP) return fail(QLORA_ERR_INVALID_ARG, "group of %d projections (1..4)", g->n);
  int64_t total = 0;
  for (int i = 0; i < g->n; ++i) {
    if (g->d[i] <= 0) return fail(QLORA_ERR_INVALID_ARG, "projection %d has %lld rows", i, (long long)g->d[i]);
    if (i + 1 < g->n && g->d[i] % 256)
      return fail(QLORA_ERR_UNSUPPORTED, "projection %d: rows %lld not a multiple of 256 (all but the last must be)",
                  i, (long long)g->d[i]);
    total += g->d[i];
  }
  if (total != g->w.d)
    return fail(QLORA_ERR_INVALID_ARG, "stacked weight has %lld rows, the projections %lld", (long long)g->w.d,
                (long long)total);
  if (g->n > 1 && r % 8) return fail(QLORA_ERR_UNSUPPORTED, "grouped projections need r %% 8 == 0 (r=%d)", r);
  if (static_cast<int64_t>(g->n) * r > 256)
    return fail(QLORA_ERR_UNSUPPORTED, "n * r = %lld above 256", static_cast<long long>(g->n) * r);
  a->ngrp = g->n;
  a->r_group = r;
  int64_t row = 0;
  for (int i = 0; i < 3; ++i) {
    row += (i < g->n) ? g->d[i] : 0;
    a->gstart[i] = row;
  }
  return QLORA_OK;
}

extern "C" {

int qlora_grouped_workspace_size(int64_t M, const qlora_nf4_group_t* g, int32_t r, int32_t backward,
                                 size_t* bytes) {
  if (!bytes) return fail(QLORA_ERR_INVALID_ARG, "bytes is NULL");
  LinearArgs a{};
  int rc = check_group(g, r, &a);
  if (rc) return rc;
  const int32_t rall = g->n * r;
  if ((rc = check_linear_shape(M, g->w.d, g->w.k, rall))) return rc;
  *bytes = backward ? bwd_workspace_bytes(M, g->w.d, g->w.k, rall) : fwd_workspace_bytes(M, g->w.d, g->w.k, rall);
  return ok();
}

int qlora_linear_fwd_grouped(const uint16_t* X, int64_t M, const qlora_nf4_group_t* g, const uint16_t* A,
                             const uint16_t* B, int32_t r, float alpha, uint16_t* Y, uint16_t* T_save,
                             void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  LinearArgs a{};
  int rc = check_group(g, r, &a);
  if (rc) return rc;
  const qlora_nf4_t* q = &g->w;
  const int32_t rall = g->n * r;
  int64_t N = 0;
  if ((rc = check_nf4(q, &N))) return rc;
  if ((rc = check_linear_shape(M, q->d, q->k, rall))) return rc;
  if (M == 0) return ok();
  if ((rc = check_codes_tma(q))) return rc;
  if ((rc = check_ptr16(X, "X", true)) || (rc = check_ptr16(A, "A", true)) || (rc = check_ptr16(B, "B", true)) ||
      (rc = check_ptr16(Y, "Y", true)) || (rc = check_ptr16(T_save, "T_save", false)))
    return rc;
  const size_t need = fwd_workspace_bytes(M, q->d, q->k, rall);
  if (need && (!workspace || workspace_bytes < need))
    return fail(QLORA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? workspace_bytes : 0);
  if (workspace && (rc = check_ptr16(workspace, "workspace", false))) return rc;
  if ((rc = bind_device(X))) return rc;
  a.X = X; a.M = M; a.d = q->d; a.k = q->k; a.q = q; a.A = A; a.B = B; a.r = rall; a.rp = qlora_rank_pad(rall);
  a.s = alpha / static_cast<float>(r);
  a.Y = Y; a.T = T_save; a.ws = workspace; a.ws_bytes = workspace_bytes;
  const char* why = "";
  rc = launch_linear_fwd(a, static_cast<cudaStream_t>(stream), &why);
  if (rc) return fail(rc, "qlora_linear_fwd_grouped: %s", why);
  return ok();
}

int qlora_linear_bwd_grouped(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_nf4_group_t* g,
                             const uint16_t* A, const uint16_t* B, int32_t r, float alpha, const uint16_t* T_save,
                             uint16_t* dX, float* dA, float* dB, void* workspace, size_t workspace_bytes,
                             qlora_stream_t stream) {
  LinearArgs a{};
  int rc = check_group(g, r, &a);
  if (rc) return rc;
  const qlora_nf4_t* q = &g->w;
  const int32_t rall = g->n * r;
  int64_t N = 0;
  if ((rc = check_nf4(q, &N))) return rc;
  if ((rc = check_linear_shape(M, q->d, q->k, rall))) return rc;
  if ((rc = check_ptr16(dA, "dA", true)) || (rc = check_ptr16(dB, "dB", true))) return rc;
  if (M > 0 && (rc = check_codes_tma(q))) return rc;
  if ((rc = check_ptr16(dY, "dY", M > 0)) || (rc = check_ptr16(X, "X", M > 0)) || (rc = check_ptr16(A, "A", true)) ||
      (rc = check_ptr16(B, "B", true)) || (rc = check_ptr16(dX, "dX", false)) ||
      (rc = check_ptr16(T_save, "T_save", false)))
    return rc;
  const size_t need = bwd_workspace_bytes(M, q->d, q->k, rall);
  if (need && (!workspace || workspace_bytes < need))
    return fail(QLORA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? workspace_bytes : 0);
  if (workspace && (rc = check_ptr16(workspace, "workspace", false))) return rc;
  if ((rc = bind_device(dA))) return rc;
  a.dY = dY; a.X = X; a.M = M; a.d = q->d; a.k = q->k; a.q = q; a.A = A; a.B = B; a.r = rall;
  a.rp = qlora_rank_pad(rall);
  a.s = alpha / static_cast<float>(r);
  a.Tin = T_save; a.dX = dX; a.dA = dA; a.dB = dB; a.ws = workspace; a.ws_bytes = workspace_bytes;
  const char* why = "";
  rc = launch_linear_bwd(a, static_cast<cudaStream_t>(stream), &why);
  if (rc) return fail(rc, "qlora_linear_bwd_grouped: %s", why);
  return ok();
}

int qlora_linear_fwd(const uint16_t* X, int64_t M, const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B,
                     int32_t r, float alpha, uint16_t* Y, uint16_t* T_save, void* workspace, size_t workspace_bytes,
                     qlora_stream_t stream) {
  return linear_fwd(X, M, q, A, B, r, alpha, nullptr, Y, T_save, workspace, workspace_bytes, stream,
                    "qlora_linear_fwd");
}

int qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_nf4_t* q, const uint16_t* A,
                     const uint16_t* B, int32_t r, float alpha, const uint16_t* T_save, uint16_t* dX, float* dA,
                     float* dB, void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  return linear_bwd(dY, X, M, q, A, B, r, alpha, nullptr, T_save, dX, dA, dB, workspace, workspace_bytes, stream,
                    "qlora_linear_bwd");
}

int qlora_linear_fwd_dropout(const uint16_t* X, int64_t M, const qlora_nf4_t* q, const uint16_t* A,
                             const uint16_t* B, int32_t r, float alpha, const qlora_dropout_t* drop, uint16_t* Y,
                             uint16_t* T_save, void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  return linear_fwd(X, M, q, A, B, r, alpha, drop, Y, T_save, workspace, workspace_bytes, stream,
                    "qlora_linear_fwd_dropout");
}

int qlora_linear_bwd_dropout(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_nf4_t* q,
                             const uint16_t* A, const uint16_t* B, int32_t r, float alpha,
                             const qlora_dropout_t* drop, const uint16_t* T_save, uint16_t* dX, float* dA, float* dB,
                             void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  return linear_bwd(dY, X, M, q, A, B, r, alpha, drop, T_save, dX, dA, dB, workspace, workspace_bytes, stream,
                    "qlora_linear_bwd_dropout");
}

int qlora_linear_dropout_workspace_size(int64_t M, int64_t d, int64_t k, int32_t r, int32_t backward,
                                        size_t* bytes) {
  if (!bytes) return fail(QLORA_ERR_INVALID_ARG, "bytes is NULL");
  int rc = check_linear_shape(M, d, k, r);
  if (rc) return rc;
  *bytes = dropout_workspace_bytes(M, d, k, r, backward != 0);
  return ok();
}

int qlora_dropout_mask(int64_t M, int64_t k, const qlora_dropout_t* drop, uint32_t* keep_bits,
                       qlora_stream_t stream) {
  if (!drop) return fail(QLORA_ERR_INVALID_ARG, "dropout descriptor is NULL");
  int64_t n = 0;
  if (!elem_count(M, k, &n)) return fail(QLORA_ERR_INVALID_ARG, "bad shape M=%lld k=%lld", (long long)M, (long long)k);
  const float p = drop->p;
  if (!(p >= 0.0f && p < 1.0f)) return fail(QLORA_ERR_INVALID_ARG, "dropout probability must lie in [0, 1)");
  if (n == 0) return ok();
  if (!keep_bits) return fail(QLORA_ERR_INVALID_ARG, "keep_bits is NULL");
  if (!aligned(keep_bits, 4)) return fail(QLORA_ERR_ALIGNMENT, "keep_bits must be 4-byte aligned");
  int rc = bind_device(keep_bits);
  if (rc) return rc;
  DropoutArgs dargs{};
  dargs.p = p;
  dargs.thr = dropout_threshold(p);
  dargs.dscale = 1.0f / (1.0f - p);
  dargs.seed = drop->seed;
  dargs.offset = drop->offset;
  return check_cuda(launch_dropout_bits(n, dargs, keep_bits, static_cast<cudaStream_t>(stream)),
                    "qlora_dropout_mask launch");
}

int qlora_lora_merge(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int32_t r, float alpha,
                     uint16_t* W_out, qlora_stream_t stream) {
  int64_t N = 0;
  int rc = check_nf4(q, &N);
  if (rc) return rc;
  if ((rc = check_linear_shape(0, q->d, q->k, r))) return rc;
  if (!aligned(q->codes, 16)) return fail(QLORA_ERR_ALIGNMENT, "codes must be 16-byte aligned for the merge");
  if ((rc = check_ptr16(A, "A", true)) || (rc = check_ptr16(B, "B", true)) || (rc = check_ptr16(W_out, "W_out", true)))
    return rc;
  if ((rc = bind_device(W_out))) return rc;
  return check_cuda(launch_lora_merge(*q, A, B, r, alpha / static_cast<float>(r), W_out,
                                      static_cast<cudaStream_t>(stream)),
                    "qlora_lora_merge launch");
}

int qlora_nf4_codebook(float out[16]) {
  if (!out) return fail(QLORA_ERR_INVALID_ARG, "out is NULL");
  host_codebook(out);
  return ok();
}

int qlora_device_status(qlora_stream_t stream, int32_t* status) {
  if (!status) return fail(QLORA_ERR_INVALID_ARG, "status is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QLORA_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  int s = 0;
  e = read_and_clear_status(&s);
  if (e != cudaSuccess) return fail(QLORA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  *status = s;
  if (s) return fail(QLORA_ERR_DEVICE, "a kernel reported failed check %d", s);
  return ok();
}

int qlora_selftest_wait_timeout(uint32_t limit_us, int32_t* result, qlora_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return fail(QLORA_ERR_INVALID_ARG, "limit_us must lie in 1..1000000");
  if (!result) return fail(QLORA_ERR_INVALID_ARG, "result is NULL");
  if (!aligned(result, 4)) return fail(QLORA_ERR_ALIGNMENT, "result must be 4-byte aligned");
  int rc = bind_device(result);
  if (rc) return rc;
  k_selftest_wait_timeout<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us, result);
  return check_cuda(cudaGetLastError(), "qlora_selftest_wait_timeout launch");
}

const char* qlora_last_error(void) { return t_err.c_str(); }

}  // extern "C"
