// qlora_gemm.cu -- the QLoRA linear layer's forward and backward on tcgen05
// tensor cores.
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora):
//   "How does it work?" / "How does alpha/r control adapter strength?"
//       h = W0 x + (alpha/r) B (A x), A r x k, B d x r;
//   "Double quantization and double dequantization"
//       Y = X doubleDequant(c1, c2, W_NF4) + X L1 L2 in BF16, and the backward
//       that flows "through the reconstructed base transformations" into the
//       adapters only (no gradient for the 4-bit weights).
//
// With s = alpha / r (fp32) the library computes
//     T_s = BF16(s X A^T)                 (M x rp, rp = r padded to 64)
//     Y   = X W^T + T_s B^T               (one GEMM: [X | T_s] [W | B]^T)
//     U_s = BF16(s dY B)                  (M x rp)
//     dX  = dY W + U_s A                  (one GEMM: [dY | U_s] [W ; A])
//     dA  = U_s^T X,   dB = dY^T T_s      (fp32)
// where W = doubleDequant(...) is rebuilt tile by tile in shared memory and
// never written to device memory.
//
// Kernels
//   k_qlora_pair<false> forward, more than 128 tokens.  A cluster of two CTAs
//                         (tcgen05.mma.cta_group::2) computes 512 tokens x 256
//                         weight rows: each CTA stages its 256 token rows of X
//                         and the packed codes of its 128 weight rows by TMA,
//                         16 dequant warps expand the codes to bf16 in the
//                         128-byte-swizzled K-major layout the tensor core
//                         reads, and one thread of the first CTA issues the
//                         MMAs into two 128 x 256 fp32 TMEM accumulators per
//                         CTA; the LoRA term is one (or more) extra 64-wide K
//                         steps.
//   k_qlora_pair<true>    dX, 512 tokens x 256 input columns per pair; the
//                         dequant warps write W in the MN-major swizzled layout
//                         (the reduction runs over W's rows).
//   k_qlora_swap<NT>      33..128 tokens: W rows are the MMA's M side (128 per
//                         tile), the tokens its N side, so the tensor core is
//                         not padded to 128 tokens; split over K.
//   k_thin<false,*>       T_s and U_s (K-major activations; A read K-major, B
//                         read MN-major straight from its storage).
//   k_thin<true,true>     dA and dB (MN-major operands, the reduction runs over
//                         tokens).  The K splits of a tile form a cluster and are
//                         added in shared memory.
//   k_reduce_bf16         deterministic sum of the main GEMM's split-K partials.
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "nf4_scale.cuh"
#include "nf4_table.h"
#include "qlora_device.cuh"
#include "qlora_internal.h"

namespace qlora {



// ============================================================================
// Cluster helpers
// ============================================================================
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16 bytes at the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  float4 v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(remote)
               : "memory");
  return v;
}

// ============================================================================
// Tensor maps
// ============================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor: `inner` elements per row (contiguous), `outer` rows,
// `row_bytes` between rows.  Box = box_inner x box_outer.
static bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool map_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                     uint32_t box_rows) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cols, rows, cols * 2, box_cols, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}


__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// ============================================================================
// Parameters shared by the fused kernels
// ============================================================================
struct MainParams {
  int64_t M, d, k;
  int32_t r, rp;            // adapter rank (all projections of a group together) and r padded to 64
  int32_t r_group;          // rank of one projection (== r for a plain weight)
  int32_t kpb;              // NF4 blocks per weight row (k / 64)
  ScaleSrc sc;
  const uint16_t* lora;     // forward: B (d x r_group, projections stacked); backward: A (r x k)
  uint16_t* out;            // bf16 output (splits == 1)
  float* partial;           // fp32 [splits][M][n_out] (splits > 1)
  int64_t n_out;            // output columns: d (forward) or k (backward)
  int32_t steps_main;       // main K steps in total
  int32_t steps_per_split;
  int32_t ext_steps;        // rp / 64
  int32_t splits;
  int32_t ncp;              // paired kernel: 256-column pairs across the output
};



// Forward LoRA extension steps of the output rows starting at `row0` (all in
// one projection): T_s columns [g r_group, (g + 1) r_group) of projection g
// meet that projection's rows of B, so only the 64-wide steps overlapping that
// window are run.  A plain weight has g = 0 and runs steps [0, rp / 64).
struct ExtWindow {
  int e_lo, n;    // first extension step and their count
  int g;          // projection
};
__device__ __forceinline__ ExtWindow ext_window(const MainParams& p, int64_t row0) {
  ExtWindow w;
  w.g = group_of(p.sc, row0);
  const int lo = w.g * p.r_group, hi = lo + p.r_group;
  w.e_lo = lo / 64;
  w.n = (hi + 63) / 64 - w.e_lo;
  return w;
}
// bf16 bits of B[n][j] for T_s column j (0 outside the row's projection window)
__device__ __forceinline__ uint32_t ext_b(const MainParams& p, const ExtWindow& w, int64_t n, int64_t j) {
  const int64_t jl = j - static_cast<int64_t>(w.g) * p.r_group;
  return (n < p.d && jl >= 0 && jl < p.r_group) ? static_cast<uint32_t>(__ldg(p.lora + n * p.r_group + jl)) : 0u;
}

// ============================================================================
// Swapped forward (33..128 tokens): the weight rows are the MMA's M side (128
// per CTA), the NT tokens its N side.  K step 128 (two NF4 blocks per weight
// row); the LoRA extension steps are 64 wide.
// ============================================================================
template <int NT>
struct SwapCfg {
  static constexpr int kStepK = 128;
  static constexpr int kWRows = 128;                                   // W rows per K step
  static constexpr uint32_t kActAtomBytes = NT * 128;                  // one 64-wide K atom of the activations
  static constexpr uint32_t kActBytes = kActAtomBytes * (kStepK / 64);
  static constexpr uint32_t kCodeBytes = kWRows * kStepK / 2;
  // Two rings: TMA stages in shared memory (activations + packed codes) and
  // dequantized W tiles in tensor memory, written by the dequant warps with
  // tcgen05.st and read by the MMA as its A operand, so the expanded weights
  // never pass through shared memory (with few tokens the shared-memory
  // round trip of every weight was the limit).
  static constexpr uint32_t kStageBytes = kActBytes + kCodeBytes;     // one TMA stage
  static constexpr int kWBufs = 4;   // W tiles being written or waiting + one the MMAs read
  static constexpr int kStagesRaw = static_cast<int>((200u * 1024u) / kStageBytes);
  static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
  // TMEM: the fp32 accumulator in columns [0, 128), W tile sw (128 rows x 128
  // K, two bf16 per 32-bit column) in columns [128 + 64 sw, 192 + 64 sw)
  static constexpr uint32_t kAccCols = 128;
  static constexpr uint32_t kWCols = kStepK / 2;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kAccCols + kWBufs * kWCols <= kTmemCols, "TMEM holds the accumulator and the W ring");
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 512 /*barriers*/;
  // two groups of 8 dequant warps take alternate steps; every thread expands
  // one whole block into its TMEM lane (the dequant rate is what matters with
  // few tokens)
  static constexpr int kGroups = 2;
  static constexpr int kGroupThreads = 256;
  static constexpr int kThreads = 64 + kGroups * kGroupThreads;
  static constexpr uint32_t kIdesc = make_idesc_bf16(128, NT, false, false);
};

template <int NT>
__global__ void __launch_bounds__(576, 1)
    k_qlora_swap(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
                 const __grid_constant__ CUtensorMap tm_ext, const MainParams p) {
  using Cfg = SwapCfg<NT>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  constexpr int SW = Cfg::kWBufs;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * Cfg::kStageBytes);
  uint64_t* full_bar = bars;                // TMA data landed (act + codes)
  uint64_t* empty_bar = bars + S;           // MMAs reading the TMA stage completed
  uint64_t* wready_bar = bars + 2 * S;      // a dequant group filled the W buffer
  uint64_t* wfree_bar = bars + 2 * S + SW;  // MMAs reading the W buffer completed
  uint64_t* tmem_full = bars + 2 * S + 2 * SW;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_full + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 128;   // first W row of the tile
  const int split = blockIdx.z;
  const int s_begin = split * p.steps_per_split;
  const int s_end = min(p.steps_main, s_begin + p.steps_per_split);
  const int n_main = max(0, s_end - s_begin);
  const ExtWindow xw = ext_window(p, n0);
  const int n_local = n_main + (split == 0 ? xw.n : 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < SW; ++i) {
      mbar_init(&wready_bar[i], Cfg::kGroupThreads / 32);
      mbar_init(&wfree_bar[i], 1);
    }
    mbar_init(tmem_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_ext);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();   // after the TMEM allocation
  griddep_wait();                // inputs written by the previous kernel

  auto act_tile = [&](int st) { return base + st * Cfg::kStageBytes; };
  auto code_tile = [&](int st) { return base + st * Cfg::kStageBytes + Cfg::kActBytes; };
  auto w_col = [&](int sw) { return Cfg::kAccCols + static_cast<uint32_t>(sw) * Cfg::kWCols; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int l = 0; l < n_local; ++l) {
        const int st = l % S;
        const uint32_t ph = (l / S) & 1;
        if (!mbar_wait(&empty_bar[st], ph ^ 1, abort_flag, DEV_WAIT_TIMEOUT_MMA)) break;
        if (l < n_main) {
          const int i = s_begin + l;
          mbar_arrive_expect_tx(&full_bar[st], Cfg::kActBytes + Cfg::kCodeBytes);
          tma_load_2d(act_tile(st), &tm_act, &full_bar[st], 128 * i, 0);
          tma_load_2d(act_tile(st) + Cfg::kActAtomBytes, &tm_act, &full_bar[st], 128 * i + 64, 0);
          tma_load_2d(code_tile(st), &tm_codes, &full_bar[st], 64 * i, static_cast<int>(n0));
        } else {
          const int e = xw.e_lo + l - n_main;
          mbar_arrive_expect_tx(&full_bar[st], Cfg::kActAtomBytes);
          tma_load_2d(act_tile(st), &tm_ext, &full_bar[st], 64 * e, 0);
        }
        ++issued;
      }
      if (*abort_flag) {
        // let every copy still in flight land before the CTA exits
        const int first = issued > S ? issued - S : 0;
        for (int l = first; l < issued; ++l) {
          const uint32_t a = smem_u32(&full_bar[l % S]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, (l / S) & 1) && globaltimer_ns() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int l = 0; l < n_local; ++l) {
        const int st = l % S;
        const uint32_t ph = (l / S) & 1;
        const int sw = l % SW;
        const uint32_t phw = (l / SW) & 1;
        if (!mbar_wait(&full_bar[st], ph, abort_flag, DEV_WAIT_TIMEOUT_TMA)) break;
        if (!mbar_wait(&wready_bar[sw], phw, abort_flag, DEV_WAIT_TIMEOUT_DEQUANT)) break;
        tc_fence_after();
        const uint64_t db0 = make_sdesc_sw128(smem_u32(act_tile(st)), 16u, 1024u);
        const uint32_t a_w = tmem_base + w_col(sw);
        if (l < n_main) {
#pragma unroll
          for (int kk = 0; kk < Cfg::kStepK / 16; ++kk) {
            // K slice kk: 8 TMEM columns of W; 32 bytes into the 128-byte-swizzled activation atom
            const uint64_t ob = (Cfg::kActAtomBytes * static_cast<uint32_t>(kk >> 2) + 32u * (kk & 3)) >> 4;
            umma_bf16_ta(tmem_base, a_w + 8u * kk, db0 + ob, Cfg::kIdesc, (l > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // LoRA steps are 64 wide
            umma_bf16_ta(tmem_base, a_w + 8u * kk, db0 + ((32u * kk) >> 4), Cfg::kIdesc, 1u);
        }
        umma_commit(&empty_bar[st]);
        umma_commit(&wfree_bar[sw]);
      }
      umma_commit(tmem_full);   // also drains MMAs on the abort path
    }
  } else {
    // ------------------------------------------------------------ dequant warps
    // Two groups take alternate K steps; a step's 256 NF4 blocks (two per W
    // row) go one to a thread, each expanding the block's eight 16-byte chunks.
    constexpr int G = Cfg::kGroups;
    const int t = threadIdx.x - 64;            // 0..511
    const int grp = t / Cfg::kGroupThreads;
    // A warp may only address its own 32-lane quarter of TMEM (warp % 4), and
    // TMEM lane = W row: warp wl of a group (0..7) takes rows 32 (warp % 4) ..
    // + 31 and block `sub` = wl / 4 of the step's two blocks per row.
    const int wl = (warp - 2) & 7;
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);
    // the codebook as register immediates (no memory traffic)
    constexpr uint32_t kCB[16] = {QLORA_NF4_TABLE_BITS};
    float C[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) C[j] = __uint_as_float(kCB[j]);
    const ScaleSrc sc = p.sc;
    const float mean = group_mean(sc, n0);   // the tile's 128 rows lie in one projection
    // row = W row (0..127), sub = which of the step's two blocks
    const int row = 32 * static_cast<int>(quarter) + lane;
    const int sub = wl >> 2;
    const uint32_t lane_addr = quarter << 21;   // TMEM lane 32 * quarter in bits 16..31
    // Code tile rows are 64 B with the TMA 64-byte swizzle: 16-byte chunk j of
    // row r sits at j ^ ((r >> 1) & 3), which spreads a quarter-warp's reads
    // over all banks.
    const uint32_t c_row = row * 64u;
    const uint32_t lc0 = 2u * sub;
    const uint32_t c_xor = (row >> 1) & 3u;
    auto block_of = [&](int i, bool& valid) -> int64_t {
      const int64_t wr = n0 + row;
      const int64_t bc = 2ll * i + sub;
      valid = (wr < p.d) && (bc < p.kpb);
      return wr * p.kpb + bc;
    };
    // this group's steps are l = grp, grp + G, ...; block constants are
    // fetched two of its own steps ahead
    ScaleRaw pre0{}, pre1{};
    ScaleRecip recip;
    bool pre0_valid = false, pre1_valid = false;
    if (grp < n_main) {
      const int64_t b0 = block_of(s_begin + grp, pre0_valid);
      if (pre0_valid) pre0 = scale_fetch(sc, b0);
    }
    if (grp + G < n_main) {
      const int64_t b1 = block_of(s_begin + grp + G, pre1_valid);
      if (pre1_valid) pre1 = scale_fetch(sc, b1);
    }
    for (int l = grp; l < n_local; l += G) {
      const int st = l % S;
      const uint32_t ph = (l / S) & 1;
      const int sw = l % SW;
      const uint32_t phw = (l / SW) & 1;
      bool okw = mbar_wait(&wfree_bar[sw], phw ^ 1, abort_flag, DEV_WAIT_TIMEOUT_MMA);
      okw = okw && mbar_wait(&full_bar[st], ph, abort_flag, DEV_WAIT_TIMEOUT_TMA);
      if (!__all_sync(0xffffffffu, okw)) break;
      tc_fence_after();   // the MMAs that read this W buffer have completed
      const uint32_t wt = tmem_base + lane_addr + w_col(sw) + 32u * static_cast<uint32_t>(sub);
      if (l < n_main) {
        const ScaleRaw cur = pre0;
        const bool cur_valid = pre0_valid;
        pre0 = pre1;
        pre0_valid = pre1_valid;
        if (l + 2 * G < n_main) {
          const int64_t bn = block_of(s_begin + l + 2 * G, pre1_valid);
          if (pre1_valid) pre1 = scale_fetch(sc, bn);
        }
        const uint32_t ctile = smem_u32(code_tile(st)) + c_row;
        uint32_t w8[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 cw = lds128(ctile + 16u * ((lc0 + h) ^ c_xor));
          w8[4 * h] = cw.x;
          w8[4 * h + 1] = cw.y;
          w8[4 * h + 2] = cw.z;
          w8[4 * h + 3] = cw.w;
        }
        // the block's 64 weights as 32 bf16 pairs, weight 2i in the low half
        // of column i (K order), into this thread's TMEM lane
        uint32_t v[32];
        if (cur_valid) {
          const Nf4Tab tab = make_tab(scale_value(sc.dq, mean, cur, recip), C);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 o = dq8(w8[c], tab);
            v[4 * c] = o.x;
            v[4 * c + 1] = o.y;
            v[4 * c + 2] = o.z;
            v[4 * c + 3] = o.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = 0u;
        }
        tmem_st32(wt, v);
      } else if (sub == 0) {
        // LoRA extension step (64 wide): B row n against T_s columns 64e + [0, 64)
        // into the first 32 columns of the W buffer
        const int e = xw.e_lo + l - n_main;
        const int64_t n = n0 + row;
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c)
          v[c] = ext_b(p, xw, n, 64ll * e + 2 * c) | (ext_b(p, xw, n, 64ll * e + 2 * c + 1) << 16);
        tmem_st32(wt, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&wready_bar[sw]);
    }

    // ------------------------------------------------------------ epilogue
    // warp w may read TMEM lanes 32 (w % 4) ..; the four warps sharing a lane
    // quarter split the token columns (idx = 0..3).  Lanes = W rows n.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(tmem_full, 0, abort_flag, DEV_WAIT_TIMEOUT_EPILOGUE));
    tc_fence_after();
    if (ok) {
      const int q = warp & 3;
      const int idx = (warp - 2) >> 2;
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      const int64_t n = n0 + 32 * q + lane;
      for (int cb = idx; cb < NT / 16; cb += 4) {
        uint32_t v[16];
        tmem_ld16(lane_base + 16 * cb, v);
        tmem_ld_wait();
        if (n < p.d) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int64_t tok = 16 * cb + j;
            if (tok < p.M) {
              if (p.splits == 1) {
                const uint32_t b = pack_bf16x2(__uint_as_float(v[j]), 0.0f);
                p.out[tok * p.n_out + n] = static_cast<uint16_t>(b & 0xFFFFu);
              } else {
                p.partial[(static_cast<int64_t>(split) * p.M + tok) * p.n_out + n] = __uint_as_float(v[j]);
              }
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  if (warp == 1 && lane == 0) {
    // the accumulator must be idle before its columns are released
    const uint32_t a = smem_u32(tmem_full);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// ============================================================================
// Paired fused kernel: tcgen05.mma.cta_group::2.
//
// Two CTAs of a cluster (ranks 0 and 1, adjacent 256-token tiles) share one
// MMA of M = 256 (128 token rows from each CTA) and N = 256 weight rows
// (forward) or input columns (backward), of which each CTA holds and
// dequantises one half.  With two accumulators per CTA a pair covers 512 tokens
// x 256 columns, so every dequantised weight feeds 512 tokens and each CTA
// expands half the weights per K step of the single-CTA kernel for the same
// tensor work.
//
//   * Each CTA loads its own activation tile and its half of the codes (TMA,
//     local barriers) and dequantises its half of W into its own shared memory.
//   * Two dequant groups of 8 warps take alternate K steps; when a group's W
//     half is written (after its own TMA stage landed) each of its warps
//     fences its stores to the async proxy and arrives on rank 0's wready
//     barrier (remotely from rank 1, with the default arrive semantics, as
//     transform warps feeding a 2-SM MMA do), so the barrier completing means
//     both halves of W and both activation tiles are there.  (A cluster-scope
//     release on that arrive costs about a microsecond per step.)
//   * One thread of rank 0 issues the MMAs for both CTAs; its commits arrive on
//     the stage / W-buffer / accumulator barriers of both CTAs (multicast).
//   * TMEM is allocated and freed by warp 1 of both CTAs together.
// ============================================================================
template <bool BWD>
struct PairCfg {
  static constexpr int kWRows = BWD ? 64 : 128;          // this CTA's half of the W tile per K step
  static constexpr int kWCols = BWD ? 128 : 64;
  static constexpr uint32_t kActBytes = 256u * 128u;     // 256 tokens x 64 K, bf16
  static constexpr uint32_t kWBytes = kWRows * kWCols * 2;
  static constexpr uint32_t kCodeBytes = kWRows * kWCols / 2;
  static constexpr uint32_t kStageBytes = kActBytes + kCodeBytes;
  static constexpr int kWBufs = 4;                       // two groups writing, one waiting, one read
  static constexpr uint32_t kFixedBytes = kWBufs * kWBytes + 1024 /*align*/ + 512 /*barriers*/;
  static constexpr int kStagesRaw = static_cast<int>((227u * 1024u - kFixedBytes) / kStageBytes);
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static_assert(kStages >= 3, "shared memory for at least three TMA stages");
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + kFixedBytes;
  static constexpr int kGroups = 2, kGroupThreads = 256, kTPB = 2, kCPT = 4;
  static constexpr int kThreads = 576;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdesc = make_idesc_bf16(256, 256, false, BWD);
};

__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma2_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (once) on the mbarrier at this offset in both CTAs of the pair when
// every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma2_commit_both(uint64_t* bar) {
  const uint16_t mask = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}
// Arrive on the mbarrier at this offset in cluster CTA `rank` (default
// semantics, as the peer CTA of a 2-SM MMA signals its leader that operands it
// wrote are ready; the writer fences its stores to the async proxy first).
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* bar, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(rank));
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// mbar_wait for barriers that another CTA of the cluster arrives on.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, int code) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait_cluster(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(a, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        report(code);
        *abort = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

template <bool BWD>
__global__ void __launch_bounds__(576, 1)
    k_qlora_pair(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
                 const __grid_constant__ CUtensorMap tm_ext, const MainParams p) {
  using Cfg = PairCfg<BWD>;
  constexpr int S = Cfg::kStages;
  constexpr int SW = Cfg::kWBufs;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  uint8_t* wbase = base + S * Cfg::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(wbase + SW * Cfg::kWBytes);
  uint64_t* full_bar = bars;                // this CTA's TMA stage landed (act + codes)
  uint64_t* empty_bar = bars + S;           // the MMAs reading the stage completed (both CTAs)
  uint64_t* wready_bar = bars + 2 * S;      // rank 0 only: both halves of W written
  uint64_t* wfree_bar = bars + 2 * S + SW;  // the MMAs reading the W buffer completed (both CTAs)
  uint64_t* tmem_full = bars + 2 * S + 2 * SW;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_full + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  // The two CTAs of a pair are neighbours along x (peer CTAs of cta_group::2).
  // Clusters are numbered column pair first, so the clusters resident at one
  // time share one or two token tiles and each activation tile is read from
  // DRAM about once.  (Bands of several token pairs, which read gate/up's codes
  // once per band instead of once per token pair, halved their DRAM reads but
  // made the forward 6-8% slower on every shape measured.)
  const int64_t cl = static_cast<int64_t>(blockIdx.x) >> 1;
  const int64_t n0 = (cl % p.ncp) * 256;                                 // output columns of the pair
  const int64_t m0 = ((cl / p.ncp) * 2 + (blockIdx.x & 1)) * 256;       // this CTA's tokens
  const int64_t h0 = n0 + 128 * static_cast<int64_t>(rank);     // this CTA's half of the columns
  const int split = blockIdx.z;
  const int s_begin = split * p.steps_per_split;
  const int s_end = min(p.steps_main, s_begin + p.steps_per_split);
  const int n_main = max(0, s_end - s_begin);
  // forward: the pair's 256 output rows lie in one projection (same window in
  // both CTAs); backward: every projection's adapter term reaches every dX
  // column, so all extension steps run
  ExtWindow xw;
  if (BWD) {
    xw.g = 0;
    xw.e_lo = 0;
    xw.n = p.ext_steps;
  } else {
    xw = ext_window(p, n0);
  }
  const int n_local = n_main + (split == 0 ? xw.n : 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < SW; ++i) {
      mbar_init(&wready_bar[i], 2 * (Cfg::kGroupThreads / 32));   // one group's warps of both CTAs (rank 0 only)
      mbar_init(&wfree_bar[i], 1);
    }
    mbar_init(tmem_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_ext);
  }
  // both CTAs' barriers exist before either CTA arrives on the other's
  __syncthreads();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (warp == 1) {
    tmem_alloc2(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();   // after the TMEM allocation
  griddep_wait();                // inputs written by the previous kernel

  auto act_tile = [&](int st) { return base + st * Cfg::kStageBytes; };
  auto code_tile = [&](int st) { return base + st * Cfg::kStageBytes + Cfg::kActBytes; };
  auto w_tile = [&](int sw) { return wbase + sw * Cfg::kWBytes; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int issued = 0;
      for (int l = 0; l < n_local; ++l) {
        const int st = l % S;
        const uint32_t ph = (l / S) & 1;
        if (!mbar_wait(&empty_bar[st], ph ^ 1, abort_flag, DEV_WAIT_TIMEOUT_MMA)) break;
        if (l < n_main) {
          const int i = s_begin + l;
          mbar_arrive_expect_tx(&full_bar[st], Cfg::kActBytes + Cfg::kCodeBytes);
          tma_load_2d(act_tile(st), &tm_act, &full_bar[st], 64 * i, static_cast<int>(m0));
          if (BWD)
            tma_load_2d(code_tile(st), &tm_codes, &full_bar[st], static_cast<int>(h0 / 2), 64 * i);
          else
            tma_load_2d(code_tile(st), &tm_codes, &full_bar[st], 32 * i, static_cast<int>(h0));
        } else {
          const int e = xw.e_lo + l - n_main;
          mbar_arrive_expect_tx(&full_bar[st], Cfg::kActBytes);
          tma_load_2d(act_tile(st), &tm_ext, &full_bar[st], 64 * e, static_cast<int>(m0));
        }
        ++issued;
      }
      if (*abort_flag) {
        const int first = issued > S ? issued - S : 0;
        for (int l = first; l < issued; ++l) {
          const uint32_t a = smem_u32(&full_bar[l % S]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, (l / S) & 1) && globaltimer_ns() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0 only)
    if (lane == 0 && rank == 0) {
      for (int l = 0; l < n_local; ++l) {
        const int st = l % S;
        const uint32_t ph = (l / S) & 1;
        const int sw = l % SW;
        const uint32_t phw = (l / SW) & 1;
        if (!mbar_wait(&full_bar[st], ph, abort_flag, DEV_WAIT_TIMEOUT_TMA)) break;
        if (!mbar_wait(&wready_bar[sw], phw, abort_flag, DEV_WAIT_TIMEOUT_DEQUANT)) break;
        tc_fence_after();
        const uint32_t a_act = smem_u32(act_tile(st));
        const uint32_t a_w = smem_u32(w_tile(sw));
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = make_sdesc_sw128(a_act + 32u * kk, 16u, 1024u);
          const uint64_t db = BWD ? make_sdesc_sw128(a_w + 2048u * kk, 8192u, 1024u)
                                  : make_sdesc_sw128(a_w + 32u * kk, 16u, 1024u);
          const uint32_t acc = (l > 0 || kk > 0) ? 1u : 0u;
          umma2_bf16(tmem_base, da, db, Cfg::kIdesc, acc);
          // token rows 128..255 of each CTA: second accumulator, same W
          const uint64_t da1 = make_sdesc_sw128(a_act + 16384u + 32u * kk, 16u, 1024u);
          umma2_bf16(tmem_base + 256u, da1, db, Cfg::kIdesc, acc);
        }
        umma2_commit_both(&empty_bar[st]);
        umma2_commit_both(&wfree_bar[sw]);
      }
      umma2_commit_both(tmem_full);   // also drains MMAs on the abort path
    }
  } else {
    // ------------------------------------------------------------ dequant warps (both CTAs)
    constexpr int G = Cfg::kGroups, TPB = Cfg::kTPB, CPT = Cfg::kCPT;
    const int t = threadIdx.x - 64;            // 0..511
    const int grp = t / Cfg::kGroupThreads;
    const int tgt = t % Cfg::kGroupThreads;
    const int tg = tgt / TPB;                  // block of the step (0..127)
    const int c_first = (tgt % TPB) * CPT;     // first 16-byte chunk of this thread
    constexpr uint32_t kCB[16] = {QLORA_NF4_TABLE_BITS};
    float C[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) C[j] = __uint_as_float(kCB[j]);
    const ScaleSrc sc = p.sc;
    // forward: the CTA's 128 weight rows lie in one projection; backward: a K
    // step's 64 weight rows do (the mean is re-read per step for a grouped weight)
    const float mean = group_mean(sc, BWD ? 64ll * s_begin : h0);
    const bool step_mean = BWD && sc.ngrp > 1;
    //   Fwd: row = W row of this CTA's half (0..127)
    //   Bwd: row = W row within the 64-row K step, sub = 64-column chunk of this CTA's half
    const int row = BWD ? (tg & 63) : tg;
    const int sub = BWD ? (tg >> 6) : 0;
    const uint32_t w_off = BWD ? 8192u * sub : 0u;
    // code rows: 32 B (Fwd, plain), 64 B (Bwd, TMA 64-byte swizzle: 16-byte
    // chunk j of row r sits at j ^ ((r >> 1) & 3))
    constexpr uint32_t kCodeRow = BWD ? 64u : 32u;
    const uint32_t c_row = row * kCodeRow;
    const uint32_t lc0 = (BWD ? 2u * sub : 0u) + static_cast<uint32_t>(c_first / 4);
    const uint32_t c_xor = BWD ? ((row >> 1) & 3u) : 0u;
    auto block_of = [&](int i, bool& valid) -> int64_t {
      int64_t wr, bc;
      if (BWD) {
        wr = 64ll * i + row;
        bc = h0 / 64 + sub;
      } else {
        wr = h0 + row;
        bc = i;
      }
      valid = (wr < p.d) && (bc < p.kpb);
      return wr * p.kpb + bc;
    };
    ScaleRaw pre0{}, pre1{};
    ScaleRecip recip;
    bool pre0_valid = false, pre1_valid = false;
    if (grp < n_main) {
      const int64_t b0 = block_of(s_begin + grp, pre0_valid);
      if (pre0_valid) pre0 = scale_fetch(sc, b0);
    }
    if (grp + G < n_main) {
      const int64_t b1 = block_of(s_begin + grp + G, pre1_valid);
      if (pre1_valid) pre1 = scale_fetch(sc, b1);
    }
    for (int l = grp; l < n_local; l += G) {
      const int st = l % S;
      const uint32_t ph = (l / S) & 1;
      const int sw = l % SW;
      const uint32_t phw = (l / SW) & 1;
      bool okw = mbar_wait(&wfree_bar[sw], phw ^ 1, abort_flag, DEV_WAIT_TIMEOUT_MMA);
      okw = okw && mbar_wait(&full_bar[st], ph, abort_flag, DEV_WAIT_TIMEOUT_TMA);
      if (!__all_sync(0xffffffffu, okw)) break;
      const uint32_t wt = smem_u32(w_tile(sw)) + w_off;
      if (l < n_main) {
        const ScaleRaw cur = pre0;
        const bool cur_valid = pre0_valid;
        pre0 = pre1;
        pre0_valid = pre1_valid;
        if (l + 2 * G < n_main) {
          const int64_t bn = block_of(s_begin + l + 2 * G, pre1_valid);
          if (pre1_valid) pre1 = scale_fetch(sc, bn);
        }
        const uint32_t ctile = smem_u32(code_tile(st)) + c_row;
        uint32_t w8[CPT];
#pragma unroll
        for (int h = 0; h < CPT / 4; ++h) {
          const uint4 cw = lds128(ctile + 16u * ((lc0 + h) ^ c_xor));
          w8[4 * h] = cw.x;
          w8[4 * h + 1] = cw.y;
          w8[4 * h + 2] = cw.z;
          w8[4 * h + 3] = cw.w;
        }
        if (cur_valid) {
          const float mean_l = step_mean ? group_mean(sc, 64ll * (s_begin + l)) : mean;
          const Nf4Tab tab = make_tab(scale_value(sc.dq, mean_l, cur, recip), C);
#pragma unroll
          for (int c = 0; c < CPT; ++c) sts128(wt + sw128_offset(row, c_first + c), dq8(w8[c], tab));
        } else {
#pragma unroll
          for (int c = 0; c < CPT; ++c) sts128(wt + sw128_offset(row, c_first + c), make_uint4(0, 0, 0, 0));
        }
      } else {
        // LoRA extension step (64 wide): this CTA's half of the adapter into the W tile
        const int e = xw.e_lo + l - n_main;
        if (BWD) {
          // A (r x k): K row j = 64e + row, N columns h0 + 64 sub + [0, 64)
          const int64_t j = 64ll * e + row;
          const int64_t col = h0 + 64 * sub;
          const bool v = (j < p.r) && (col < p.k);
          const uint16_t* srcp = p.lora + j * p.k + col;
#pragma unroll
          for (int c = c_first; c < c_first + CPT; ++c) {
            uint4 val = make_uint4(0, 0, 0, 0);
            if (v) val = __ldg(reinterpret_cast<const uint4*>(srcp + 8 * c));
            sts128(wt + sw128_offset(row, c), val);
          }
        } else {
          // B row n against T_s columns 64e + [0, 64)
          const int64_t n = h0 + row;
#pragma unroll
          for (int c = c_first; c < c_first + CPT; ++c) {
            uint32_t h[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) h[q] = ext_b(p, xw, n, 64ll * e + 8 * c + q);
            sts128(wt + sw128_offset(row, c),
                   make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16)));
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(&wready_bar[sw]);
        else
          mbar_arrive_remote(&wready_bar[sw], 0);
      }
    }

    // ------------------------------------------------------------ epilogue (both CTAs)
    const bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(tmem_full, 0, abort_flag, DEV_WAIT_TIMEOUT_EPILOGUE));
    tc_fence_after();
    if (ok) {
      const int q = warp & 3;
      const int idx = (warp - 2) >> 2;
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      const int acc = idx >> 1;                       // which 128-token half of this CTA's tile
      const int64_t m = m0 + 128 * acc + 32 * q + lane;
      for (int cb = 0; cb < 4; ++cb) {
        const int col0 = 128 * (idx & 1) + 32 * cb;
        uint32_t v[32];
        tmem_ld32(lane_base + 256u * acc + col0, v);
        tmem_ld_wait();
        if (m < p.M) {
          const int64_t n = n0 + col0;
          if (p.splits == 1) {
            uint16_t* dst = p.out + m * p.n_out + n;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              if (n + 8 * g + 8 <= p.n_out) {
                uint4 o;
                o.x = pack_bf16x2(__uint_as_float(v[8 * g + 0]), __uint_as_float(v[8 * g + 1]));
                o.y = pack_bf16x2(__uint_as_float(v[8 * g + 2]), __uint_as_float(v[8 * g + 3]));
                o.z = pack_bf16x2(__uint_as_float(v[8 * g + 4]), __uint_as_float(v[8 * g + 5]));
                o.w = pack_bf16x2(__uint_as_float(v[8 * g + 6]), __uint_as_float(v[8 * g + 7]));
                *reinterpret_cast<uint4*>(dst + 8 * g) = o;
              }
            }
          } else {
            float* dst = p.partial + (static_cast<int64_t>(split) * p.M + m) * p.n_out + n;
#pragma unroll
            for (int g = 0; g < 8; ++g)
              if (n + 4 * g + 4 <= p.n_out)
                *reinterpret_cast<uint4*>(dst + 4 * g) = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  if (warp == 1 && lane == 0) {
    // this CTA's accumulator must be idle before the pair's columns are released
    const uint32_t a = smem_u32(tmem_full);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_cluster(a, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
  }
  tc_fence_before();
  __syncthreads();
  // neither CTA leaves while the other's MMAs or remote arrivals may still
  // touch its shared memory
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem_base, Cfg::kTmemCols);
  }
}

// ============================================================================
// Thin GEMM: D[128 x rp] = A_tile * B_tile^T over K.
//   kMN = false: A, B K-major (T_s: X and A; U_s: dY and B^T).
//   kMN = true : A, B MN-major, reduction over tokens (dA^T: X^T and U_s;
//                dB: dY^T and T_s).
// K is split over the CTAs of one thread-block cluster (blockIdx.y = rank,
// at most 8).  Each CTA parks its fp32 tile in its own shared memory; after a
// cluster barrier CTA q adds rows [q 128 / S, (q + 1) 128 / S) of the S tiles
// in rank order through distributed shared memory and writes the result, so
// no partial sums go through HBM and the sum order is fixed.
// ============================================================================
enum ThinOut : int {
  THIN_BF16 = 0,   // out16[row][j] = BF16(scale * D)       (T_s, U_s; rp columns)
  THIN_DA = 1,     // outf[j][row]  = D for j < r           (dA from dA^T; row stride `ld`)
  THIN_DB = 2,     // outf[row][j]  = D for j < r           (dB; row stride r)
};

struct ThinParams {
  int64_t rows;          // output rows in total (M, k or d)
  int32_t rp;            // output columns (multiple of 64)
  int32_t steps;         // K steps in total
  int32_t steps_per_split;
  int32_t mode;          // ThinOut
  int32_t r;
  int64_t ld;            // THIN_DA: row stride of dA (= k)
  float scale;           // applied to every output (1 for a plain dA / dB)
  uint16_t* out16;
  float* outf;
  // Adapter dropout on the A operand X (nullptr: none): keep bitmask of the
  // M x k activations (bit b of word w <-> flat element 32 w + b).  Dropped
  // elements are zeroed in shared memory before the tensor core reads them.
  const uint32_t* keep;
  int64_t keep_rows;     // M
  int64_t keep_ld;       // k
  // THIN_DB of a grouped weight: output rows from gstart[i] on belong to
  // projection i + 1, whose dB takes columns [g r_group, (g + 1) r_group) of
  // the tile (a plain weight: ngrp <= 1, r_group = r)
  int32_t ngrp;
  int32_t r_group;
  int64_t gstart[3];
};

// Zero the dropped elements of one 128-byte row (64 bf16) of a tile stored
// with the 128-byte swizzle; bit e of `bits` keeps element e of the row.  A
// mask byte becomes four 32-bit lane masks without a table: multiplying its
// low (high) nibble by 2^7 + 2^14 + 2^21 + 2^28 moves bit i to bit 8 i + 7,
// the sign bit of byte i (the partial products never overlap), and a byte
// permute with sign replication widens each sign bit to 16 bits.
__device__ __forceinline__ void mask_row_sw128(uint32_t tile, uint32_t r, uint64_t bits) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t b = static_cast<uint32_t>(bits >> (8 * c)) & 0xFFu;
    if (b == 0xFFu) continue;
    const uint32_t lo = (b & 0xFu) * 0x10204080u, hi = (b >> 4) * 0x10204080u;
    const uint32_t addr = tile + sw128_offset(r, static_cast<uint32_t>(c));
    uint4 v = lds128(addr);
    v.x &= prmt(lo, 0u, 0x9988u);
    v.y &= prmt(lo, 0u, 0xBBAAu);
    v.z &= prmt(hi, 0u, 0x9988u);
    v.w &= prmt(hi, 0u, 0xBBAAu);
    sts128(addr, v);
  }
}

struct ThinCfg {
  static constexpr int kStages = 4;
  static constexpr uint32_t kABytes = 128 * 128;      // 128 rows x 64 K (K-major) or 2 x (64 K x 64 MN)
  // B holds rp x 64 bf16; shared memory is sized by rp so that two CTAs fit on
  // an SM when rp <= 64 (one streams while the other sets up or drains)
  __host__ __device__ static uint32_t stage_bytes(int rp) { return kABytes + 128u * static_cast<uint32_t>(rp); }
  __host__ __device__ static uint32_t smem_bytes(int rp) { return kStages * stage_bytes(rp) + 1024 + 256; }
};

template <bool kAMN, bool kBMN>
__global__ void __launch_bounds__(128, 2)
    k_thin(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, const ThinParams p) {
  using Cfg = ThinCfg;
  constexpr int S = Cfg::kStages;
  const uint32_t stage_bytes = Cfg::stage_bytes(p.rp);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * stage_bytes);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + S;
  uint64_t* tmem_full = bars + 2 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S + 2);
  uint64_t* masked_bar = bars + 2 * S + 3;   // dropout: the stage's X tile has been masked

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 128;
  const int split = blockIdx.y;
  const int s_begin = split * p.steps_per_split;
  const int s_end = min(p.steps, s_begin + p.steps_per_split);
  const int n_local = max(0, s_end - s_begin);
  const int rp = p.rp;
  const uint32_t tmem_cols = rp <= 64 ? 64u : (rp <= 128 ? 128u : 256u);
  const uint32_t b_bytes = static_cast<uint32_t>(rp) * 128u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
      mbar_init(&masked_bar[i], 2);   // one arrival per masking warp
    }
    mbar_init(tmem_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();   // after the TMEM allocation
  griddep_wait();                // inputs written by the previous kernel
  auto a_tile = [&](int st) { return base + st * stage_bytes; };
  auto b_tile = [&](int st) { return base + st * stage_bytes + Cfg::kABytes; };

  if (warp == 0 && lane == 0) {
    int issued = 0;
    for (int l = 0; l < n_local; ++l) {
      const int st = l % S;
      const uint32_t ph = (l / S) & 1;
      if (!mbar_wait(&empty_bar[st], ph ^ 1, abort_flag, DEV_WAIT_TIMEOUT_MMA)) break;
      const int i = s_begin + l;
      mbar_arrive_expect_tx(&full_bar[st], Cfg::kABytes + b_bytes);
      if (!kAMN) {
        tma_load_2d(a_tile(st), &tm_a, &full_bar[st], 64 * i, static_cast<int>(row0));
      } else {
        tma_load_2d(a_tile(st), &tm_a, &full_bar[st], static_cast<int>(row0), 64 * i);
        tma_load_2d(a_tile(st) + 8192, &tm_a, &full_bar[st], static_cast<int>(row0) + 64, 64 * i);
      }
      if (!kBMN) {
        tma_load_2d(b_tile(st), &tm_b, &full_bar[st], 64 * i, 0);
      } else {
        for (int c = 0; c < rp / 64; ++c) tma_load_2d(b_tile(st) + 8192 * c, &tm_b, &full_bar[st], 64 * c, 64 * i);
      }
      ++issued;
    }
    if (*abort_flag) {
      const int first = issued > S ? issued - S : 0;
      for (int l = first; l < issued; ++l) {
        const uint32_t a = smem_u32(&full_bar[l % S]);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, (l / S) & 1) && globaltimer_ns() - t0 < 100000000ull) {
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = make_idesc_bf16(128, static_cast<uint32_t>(rp), kAMN, kBMN);
    uint64_t* ready = p.keep ? masked_bar : full_bar;
    for (int l = 0; l < n_local; ++l) {
      const int st = l % S;
      const uint32_t ph = (l / S) & 1;
      if (!mbar_wait(&ready[st], ph, abort_flag, p.keep ? DEV_WAIT_TIMEOUT_DEQUANT : DEV_WAIT_TIMEOUT_TMA)) break;
      tc_fence_after();
      const uint32_t aa = smem_u32(a_tile(st));
      const uint32_t bb = smem_u32(b_tile(st));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = kAMN ? make_sdesc_sw128(aa + 2048u * kk, 8192u, 1024u)
                                 : make_sdesc_sw128(aa + 32u * kk, 16u, 1024u);
        const uint64_t db = kBMN ? make_sdesc_sw128(bb + 2048u * kk, 8192u, 1024u)
                                 : make_sdesc_sw128(bb + 32u * kk, 16u, 1024u);
        umma_bf16(tmem_base, da, db, idesc, (l > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&empty_bar[st]);
    }
    umma_commit(tmem_full);
  } else if (warp >= 2 && p.keep) {
    // adapter dropout: warps 2 and 3 zero the dropped activations of each
    // stage's X tile before the MMA thread may read it.  The mask bits of a
    // stage are fetched before its TMA wait, so their latency overlaps it.
    const int t = static_cast<int>(threadIdx.x) - 64;   // 0..63
    for (int l = 0; l < n_local; ++l) {
      const int st = l % S;
      const uint32_t ph = (l / S) & 1;
      const int i = s_begin + l;
      uint64_t bits[2] = {~0ull, ~0ull};
      bool live[2] = {false, false};
      const unsigned long long* kb = reinterpret_cast<const unsigned long long*>(p.keep);
      if (!kAMN) {
        // 128 token rows x 64 features (columns 64 i ..): rows t and t + 64
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t m = row0 + t + 64 * h;
          live[h] = m < p.keep_rows;
          if (live[h]) bits[h] = __ldg(kb + ((m * p.keep_ld + 64ll * i) >> 6));
        }
      } else {
        // two halves of 64 token rows (64 i + t) x 64 features (row0 + 64 h ..)
        const int64_t m = 64ll * i + t;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t f = row0 + 64 * h;
          live[h] = m < p.keep_rows && f < p.keep_ld;
          if (live[h]) bits[h] = __ldg(kb + ((m * p.keep_ld + f) >> 6));
        }
      }
      const bool okw = mbar_wait(&full_bar[st], ph, abort_flag, DEV_WAIT_TIMEOUT_TMA);
      if (!__all_sync(0xffffffffu, okw)) break;
      const uint32_t at = smem_u32(a_tile(st));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!live[h]) continue;   // rows past M or columns past k were filled with zeros by the copy
        if (!kAMN)
          mask_row_sw128(at, static_cast<uint32_t>(t + 64 * h), bits[h]);
        else
          mask_row_sw128(at + 8192u * h, static_cast<uint32_t>(t), bits[h]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&masked_bar[st]);
    }
  }
  __syncwarp();

  // epilogue, 1: every warp moves its 32 TMEM lanes (rows) into this CTA's
  // fp32 tile in shared memory, over the now idle stages (rows padded by 4
  // floats so that a quarter-warp's 16-byte stores hit distinct banks)
  const bool ok = __all_sync(0xffffffffu, mbar_wait(tmem_full, 0, abort_flag, DEV_WAIT_TIMEOUT_EPILOGUE));
  __syncthreads();   // the producer has drained any copy still in flight into the stages
  tc_fence_after();
  const uint32_t ldr = static_cast<uint32_t>(rp + 4);   // floats per tile row
  float* red = reinterpret_cast<float*>(base);
  {
    const int trow = 32 * warp + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * warp) << 16);
    const bool zero = !ok || n_local == 0;
    // rp is a multiple of 64: two 32-column loads in flight per wait
    for (int cb = 0; cb < rp / 32; cb += 2) {
      uint32_t v0[32], v1[32];
      tmem_ld32(lane_base + 32 * cb, v0);
      tmem_ld32(lane_base + 32 * (cb + 1), v1);
      tmem_ld_wait();
      float* dst = red + trow * ldr + 32 * cb;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        *reinterpret_cast<uint4*>(dst + 4 * g) =
            zero ? make_uint4(0, 0, 0, 0) : make_uint4(v0[4 * g], v0[4 * g + 1], v0[4 * g + 2], v0[4 * g + 3]);
        *reinterpret_cast<uint4*>(dst + 32 + 4 * g) =
            zero ? make_uint4(0, 0, 0, 0) : make_uint4(v1[4 * g], v1[4 * g + 1], v1[4 * g + 2], v1[4 * g + 3]);
      }
    }
  }
  // 2: every CTA of the cluster has parked its tile (all CTAs always take both
  // cluster barriers, also on the abort path)
  cluster_sync_all();
  // 3: this CTA adds its row slice of the cluster's tiles in rank order
  {
    const int S2 = static_cast<int>(gridDim.y);
    const int q = static_cast<int>(blockIdx.y);
    const int r0 = q * 128 / S2, r1 = (q + 1) * 128 / S2, nr = r1 - r0;
    const int c4n = rp / 4;
    const uint32_t red_addr = smem_u32(red);
    for (int idx = threadIdx.x; idx < nr * c4n; idx += blockDim.x) {
      // dA writes transposed rows: consecutive threads take consecutive rows
      const int rr = (p.mode == THIN_DA) ? r0 + idx % nr : r0 + idx / c4n;
      const int c4 = (p.mode == THIN_DA) ? idx / nr : idx % c4n;
      const uint32_t off = (static_cast<uint32_t>(rr) * ldr + 4u * static_cast<uint32_t>(c4)) * 4u;
      // all peers' loads in flight first, then the sum in rank order
      float4 v[8];
#pragma unroll
      for (int pr = 0; pr < 8; ++pr)
        if (pr < S2) v[pr] = ld_cluster_f4(red_addr + off, static_cast<uint32_t>(pr));
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int pr = 0; pr < 8; ++pr) {
        if (pr < S2) {
          acc.x += v[pr].x;
          acc.y += v[pr].y;
          acc.z += v[pr].z;
          acc.w += v[pr].w;
        }
      }
      const int64_t row = row0 + rr;
      if (row >= p.rows) continue;
      const int j0 = 4 * c4;
      if (p.mode == THIN_BF16) {
        uint2 o;
        o.x = pack_bf16x2(acc.x * p.scale, acc.y * p.scale);
        o.y = pack_bf16x2(acc.z * p.scale, acc.w * p.scale);
        *reinterpret_cast<uint2*>(p.out16 + row * rp + j0) = o;
      } else {
        const float e[4] = {acc.x * p.scale, acc.y * p.scale, acc.z * p.scale, acc.w * p.scale};
        if (p.mode == THIN_DA) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (j0 + u < p.r) p.outf[static_cast<int64_t>(j0 + u) * p.ld + row] = e[u];
        } else {
          int g = 0;   // projection of this output row (128-row tiles never straddle two)
#pragma unroll
          for (int jg = 0; jg < 3; ++jg) g += (jg + 1 < p.ngrp && row0 >= p.gstart[jg]) ? 1 : 0;
          const int lo = g * p.r_group;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (j0 + u >= lo && j0 + u < lo + p.r_group) p.outf[row * p.r_group + (j0 + u - lo)] = e[u];
        }
      }
    }
  }
  // 4: peers keep their tiles until every CTA of the cluster has read them
  cluster_sync_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ============================================================================
// Reductions over split-K partials (fixed order: deterministic)
// ============================================================================
// out_bf16[i] = BF16(scale * sum_s partial[s][i]), n4 = count / 4
__global__ void k_reduce_bf16(const float* __restrict__ partial, int splits, int64_t count, float scale,
                              uint16_t* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t n4 = count >> 2;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(partial)[i];
    for (int s = 1; s < splits; ++s) {
      const float4 v = reinterpret_cast<const float4*>(partial + s * count)[i];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x * scale, acc.y * scale);
    o.y = pack_bf16x2(acc.z * scale, acc.w * scale);
    reinterpret_cast<uint2*>(out)[i] = o;
  }
}

// Bt[j][n] = B[n][j] for j < r, 0 for r <= j < rp
// B' (d x r, bf16) block diagonal from the stacked B (d x r_group): row n of
// projection g holds its B row in columns [g r_group, (g + 1) r_group), zeros
// elsewhere.  Eight columns per thread (r % 8 == 0 for grouped weights).
struct BlockDiag {
  int64_t d;
  int32_t r_group, r, ngrp;
  int64_t gstart[3];
};
__global__ void k_blockdiag_B(const uint16_t* __restrict__ B, const BlockDiag bd, uint16_t* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();   // a previous call's kernels may still read the workspace
  const int64_t n8 = bd.d * bd.r / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = (8 * i) / bd.r;
    const int j0 = static_cast<int>(8 * i - n * bd.r);
    int g = 0;
#pragma unroll
    for (int jg = 0; jg < 3; ++jg) g += (jg + 1 < bd.ngrp && n >= bd.gstart[jg]) ? 1 : 0;
    const int lo = g * bd.r_group;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j0 >= lo && j0 < lo + bd.r_group)   // r_group % 8 == 0: the 8 columns lie in the window together
      v = __ldg(reinterpret_cast<const uint4*>(B + n * bd.r_group + (j0 - lo)));
    *reinterpret_cast<uint4*>(out + 8 * i) = v;
  }
}

__global__ void k_transpose_B(const uint16_t* __restrict__ B, int64_t d, int r, int rp, uint16_t* __restrict__ Bt) {
  __shared__ uint16_t tile[32][34];
  griddep_launch_dependents();
  griddep_wait();
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int j0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int yy = ty; yy < 32; yy += 8) {
    const int64_t n = n0 + yy;
    const int j = j0 + tx;
    tile[yy][tx] = (n < d && j < r) ? B[n * r + j] : static_cast<uint16_t>(0);
  }
  __syncthreads();
  for (int yy = ty; yy < 32; yy += 8) {
    const int j = j0 + yy;
    const int64_t n = n0 + tx;
    if (j < rp && n < d) Bt[static_cast<int64_t>(j) * d + n] = tile[tx][yy];
  }
}

// ============================================================================
// Host side: split heuristics, workspace layout, launches
// ============================================================================
constexpr int kSms = 148;   // B200: split counts are planned for 148 SMs


// Number of K splits so that `tiles * splits` fills the machine, each split
// keeping at least `min_steps` K steps.
static int plan_splits(int64_t tiles, int steps, int min_steps, int slots_per_sm) {
  const int64_t slots = static_cast<int64_t>(kSms) * slots_per_sm;
  if (tiles >= slots || steps <= min_steps) return 1;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 32; ++s) {
    const int per = static_cast<int>(ceil_div(steps, s));
    if (per < min_steps && s > 1) break;
    const int real = static_cast<int>(ceil_div(steps, per));
    const int64_t ctas = tiles * real;
    const int64_t waves = ceil_div(ctas, slots);
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * slots);
    // prefer filling the machine; among similar fills prefer fewer splits
    const double score = eff * (ctas >= slots ? 1.0 : static_cast<double>(ctas) / slots);
    if (score > best_eff + 0.02) {
      best_eff = score;
      best = real;
    }
  }
  return best;
}

// Low-rank GEMMs are bound by reading their activation operand once: about one
// CTA per SM, each streaming at least 8 K steps, keeps per-CTA fixed costs
// (barrier set-up, TMEM allocation, the fp32 partial write) small.
static int plan_thin_splits(int64_t tiles, int steps, int rp) {
  const int64_t slots = static_cast<int64_t>(kSms) * (rp <= 64 ? 2 : 1);
  int64_t s = tiles > 0 ? slots / tiles : 1;
  if (s < 1) s = 1;
  const int64_t cap = steps / 8 > 1 ? steps / 8 : 1;
  if (s > cap) s = cap;
  if (s > 8) s = 8;   // the splits form one thread-block cluster (portable size)
  return static_cast<int>(s);
}

struct Plan {
  // thin GEMMs
  int splits_T, splits_U, splits_dA, splits_dB;
  // main
  int main_splits;
  int nt;   // swap token tile (0 = non-swap)
  bool fewtok;   // forward through the few-token kernels
  // workspace offsets (bytes)
  size_t off_T, off_Bt, off_U, off_main, total;
};

// Swapped forward (33..128 tokens): split K only as far as one wave of CTAs
// (one per SM) is filled.  Each CTA pays a fixed set-up and drain per launch
// and a split adds an fp32 partial pass, so a second, partly empty wave of
// whole-K CTAs beats many short split CTAs: on 28672 x 8192 at M = 32, one
// split (224 CTAs in two waves) took 128 us against 148 us for seven.
static int plan_swap_splits(int64_t tiles, int steps) {
  int s = static_cast<int>(tiles >= kSms ? 1 : kSms / tiles);
  if (s > 8) s = 8;
  while (s > 1 && steps / s < 4) --s;
  return s < 1 ? 1 : s;
}

static int swap_nt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  return 0;
}

static Plan make_plan(int64_t M, int64_t d, int64_t k, int32_t r, bool bwd, bool need_T) {
  Plan pl{};
  const int rp = qlora_rank_pad(r);
  const int64_t mt = ceil_div(M, 128);
  pl.splits_T = plan_thin_splits(mt, static_cast<int>(k / 64), rp);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  pl.off_T = need_T ? take(static_cast<size_t>(M) * rp * 2) : 0;
  if (!bwd && fewtok_eligible(M, d, k)) {
    pl.fewtok = true;
    pl.off_main = take(fewtok_workspace_bytes(M, d, k, rp));
  } else if (!bwd) {
    pl.nt = swap_nt(M);
    const int steps = static_cast<int>(k / 64);
    if (pl.nt) {
      pl.main_splits = plan_swap_splits(ceil_div(d, 128), static_cast<int>(ceil_div(k, 128)));
    } else {
      pl.main_splits = plan_splits(ceil_div(d, 256) * 2 * ceil_div(M, 512), steps, 8, 1);
    }
    pl.off_main = pl.main_splits > 1 ? take(static_cast<size_t>(pl.main_splits) * M * d * 4) : 0;
  } else {
    pl.nt = 0;
    const int dsteps = static_cast<int>(ceil_div(d, 64));
    pl.splits_U = plan_thin_splits(mt, dsteps, rp);
    pl.off_Bt = take(static_cast<size_t>(rp) * d * 2);
    pl.off_U = take(static_cast<size_t>(M) * rp * 2);
    const int msteps = static_cast<int>(ceil_div(M, 64));
    pl.splits_dA = plan_thin_splits(ceil_div(k, 128), msteps, rp);
    pl.splits_dB = plan_thin_splits(ceil_div(d, 128), msteps, rp);
    pl.main_splits = plan_splits(ceil_div(k, 256) * 2 * ceil_div(M, 512), dsteps, 8, 1);
    pl.off_main = pl.main_splits > 1 ? take(static_cast<size_t>(pl.main_splits) * M * k * 4) : 0;
  }
  pl.total = off;
  return pl;
}

size_t fwd_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r) {
  // T_s always has a workspace home so the caller may pass T_save == NULL
  return make_plan(M, d, k, r, false, true).total;
}
size_t bwd_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r) {
  return make_plan(M, d, k, r, true, true).total;
}
size_t dropout_mask_offset(int64_t M, int64_t d, int64_t k, int32_t r, bool bwd) {
  return align_up(bwd ? bwd_workspace_bytes(M, d, k, r) : fwd_workspace_bytes(M, d, k, r), 256);
}
size_t dropout_workspace_bytes(int64_t M, int64_t d, int64_t k, int32_t r, bool bwd) {
  return dropout_mask_offset(M, d, k, r, bwd) + align_up(static_cast<size_t>((M * k + 31) / 32) * 4, 256);
}

static int grid1d(int64_t work, int per_block) {
  int64_t g = ceil_div(work, per_block);
  const int64_t cap = static_cast<int64_t>(kSms) * 16;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

#define QL_CHECK_LAUNCH(what)                    \
  do {                                           \
    cudaError_t e_ = cudaGetLastError();         \
    if (e_ != cudaSuccess) {                     \
      *why = what;                               \
      return QLORA_ERR_CUDA;                     \
    }                                            \
  } while (0)

// T_s = BF16(s X A^T) (or U_s = BF16(s dY B) with `act` = dY and `bmat` = B^T)
// b_mn = false: bmat is (brows x K) row-major, read K-major (A of the layer).
// b_mn = true : bmat is (K x brows) row-major, read MN-major (B of the layer,
//               K = d, N = r), which needs brows * 2 bytes to be a multiple of 16.
// One low-rank GEMM: grid (row tiles, K splits), the splits of a row tile
// forming one cluster that reduces in shared memory.
template <bool kAMN, bool kBMN>
static int launch_thin(const CUtensorMap& ta, const CUtensorMap& tb, ThinParams tp, int64_t tiles, int splits,
                       cudaStream_t st, const char** why) {
  tp.steps_per_split = static_cast<int>(ceil_div(tp.steps, splits));
  const int real = static_cast<int>(ceil_div(tp.steps, tp.steps_per_split));
  const uint32_t smem = ThinCfg::smem_bytes(tp.rp);
  if (set_smem(k_thin<kAMN, kBMN>, smem) != cudaSuccess) {
    *why = "smem attribute (thin GEMM)";
    return QLORA_ERR_CUDA;
  }
  cudaError_t e;
  {
    ProfScope ps_(QLORA_KC_LORA_GEMM, st);
    const dim3 cl(1, static_cast<unsigned>(real), 1);
    e = launch_pdl(k_thin<kAMN, kBMN>, dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(real)), dim3(128), smem,
                   st, &cl, ta, tb, tp);
  }
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    *why = "thin GEMM launch";
    return QLORA_ERR_CUDA;
  }
  return 0;
}

// T_s = BF16(s X A^T) (or U_s = BF16(s dY B) with `act` = dY and `bmat` = B^T)
// b_mn = false: bmat is (brows x K) row-major, read K-major (A of the layer).
// b_mn = true : bmat is (K x brows) row-major, read MN-major (B of the layer,
//               K = d, N = r), which needs brows * 2 bytes to be a multiple of 16.
static int run_lowrank_down(const uint16_t* act, int64_t M, int64_t K, const uint16_t* bmat, int64_t brows,
                            bool b_mn, int rp, float s, int splits, uint16_t* out, cudaStream_t st, const char** why,
                            const uint32_t* keep = nullptr) {
  CUtensorMap ta, tb;
  const bool okb = b_mn ? map_bf16(&tb, bmat, brows, K, 64, 64) : map_bf16(&tb, bmat, K, brows, 64, rp);
  if (!map_bf16(&ta, act, K, M, 64, 128) || !okb) {
    *why = "tensor map encoding failed (thin GEMM)";
    return QLORA_ERR_CUDA;
  }
  ThinParams tp{};
  tp.rows = M;
  tp.rp = rp;
  tp.steps = static_cast<int>(ceil_div(K, 64));
  tp.mode = THIN_BF16;
  tp.scale = s;
  tp.out16 = out;
  tp.keep = keep;
  tp.keep_rows = M;
  tp.keep_ld = K;
  return b_mn ? launch_thin<false, true>(ta, tb, tp, ceil_div(M, 128), splits, st, why)
              : launch_thin<false, false>(ta, tb, tp, ceil_div(M, 128), splits, st, why);
}

template <int NT>
static int launch_swap(const CUtensorMap& ta, const CUtensorMap& tc, const CUtensorMap& te, const MainParams& mp,
                       dim3 grid, cudaStream_t st, const char** why) {
  using Cfg = SwapCfg<NT>;
  if (set_smem(k_qlora_swap<NT>, Cfg::kSmemBytes) != cudaSuccess) {
    *why = "smem attribute (swapped GEMM)";
    return QLORA_ERR_CUDA;
  }
  cudaError_t e;
  {
    ProfScope ps_(QLORA_KC_FWD_GEMM, st);
    e = launch_pdl(k_qlora_swap<NT>, grid, dim3(Cfg::kThreads), Cfg::kSmemBytes, st, nullptr, ta, tc, te, mp);
  }
  if (e != cudaSuccess) {
    *why = "swapped GEMM launch";
    return QLORA_ERR_CUDA;
  }
  QL_CHECK_LAUNCH("swapped GEMM launch");
  return 0;
}

// The paired kernel: clusters of two CTAs (grid x = 2 x token pairs x column pairs).
template <bool BWD>
static int launch_pair(const CUtensorMap& ta, const CUtensorMap& tc, const CUtensorMap& te, const MainParams& mp,
                       dim3 grid, cudaStream_t st, const char** why) {
  using Cfg = PairCfg<BWD>;
  if (set_smem(k_qlora_pair<BWD>, Cfg::kSmemBytes) != cudaSuccess) {
    *why = "smem attribute (paired GEMM)";
    return QLORA_ERR_CUDA;
  }
  cudaError_t e;
  {
    ProfScope ps_(BWD ? QLORA_KC_BWD_GEMM : QLORA_KC_FWD_GEMM, st);
    const dim3 cl(2, 1, 1);
    e = launch_pdl(k_qlora_pair<BWD>, grid, dim3(Cfg::kThreads), Cfg::kSmemBytes, st, &cl, ta, tc, te, mp);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    static thread_local char msg[160];
    snprintf(msg, sizeof msg, "paired GEMM launch: %s (%s)", cudaGetErrorName(e), cudaGetErrorString(e));
    *why = msg;
    return QLORA_ERR_CUDA;
  }
  return 0;
}

static ScaleSrc scale_src(const qlora_nf4_t& q, const LinearArgs& a) {
  ScaleSrc s{};
  s.dq = q.double_quant;
  s.absmax = q.absmax;
  s.c2 = q.c2;
  s.c1 = q.c1;
  s.mean = q.mean;
  s.ngrp = a.ngrp;
  for (int i = 0; i < 3; ++i) s.gstart[i] = a.gstart[i];
  return s;
}

static int32_t rank_group(const LinearArgs& a) { return a.r_group > 0 ? a.r_group : a.r; }

// Adapter dropout: the keep bitmask of X in the workspace (nullptr without
// dropout), generated for this call from (seed, offset).
static int dropout_mask(const LinearArgs& a, bool bwd, cudaStream_t st, const char** why, const uint32_t** keep) {
  *keep = nullptr;
  if (!a.drop) return 0;
  uint32_t* bits = reinterpret_cast<uint32_t*>(static_cast<char*>(a.ws) +
                                               dropout_mask_offset(a.M, a.d, a.k, a.r, bwd));
  if (launch_dropout_bits(a.M * a.k, *a.drop, bits, st) != cudaSuccess) {
    *why = "dropout mask launch";
    return QLORA_ERR_CUDA;
  }
  *keep = bits;
  return 0;
}

int launch_linear_fwd(const LinearArgs& a, cudaStream_t st, const char** why) {
  const int64_t M = a.M, d = a.d, k = a.k;
  const int rp = a.rp;
  const bool own_T = (a.T == nullptr);
  Plan pl = make_plan(M, d, k, a.r, false, true);
  char* ws = static_cast<char*>(a.ws);
  uint16_t* T = own_T ? reinterpret_cast<uint16_t*>(ws + pl.off_T) : a.T;
  const uint32_t* keep = nullptr;
  int rc = dropout_mask(a, false, st, why, &keep);
  if (rc) return rc;
  // with dropout, T_s = BF16(s / (1 - p) * (X . keep) A^T)
  const float s_down = a.drop ? a.s * a.drop->dscale : a.s;
  if (pl.fewtok) {
    CUtensorMap tm;
    if (!make_map(&tm, a.q->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, k / 2, d, k / 2, 128, 256,
                  CU_TENSOR_MAP_SWIZZLE_128B)) {
      *why = "tensor map encoding failed (few-token forward)";
      return QLORA_ERR_CUDA;
    }
    return launch_fewtok_fwd(a, T, ws + pl.off_main, &tm, st, why, keep);
  }
  rc = run_lowrank_down(a.X, M, k, a.A, a.r, false, rp, s_down, pl.splits_T, T, st, why, keep);
  if (rc) return rc;

  const qlora_nf4_t& q = *a.q;
  MainParams mp{};
  mp.M = M; mp.d = d; mp.k = k; mp.r = a.r; mp.rp = rp;
  mp.kpb = static_cast<int32_t>(k / 64);
  mp.sc = scale_src(q, a);
  mp.r_group = rank_group(a);
  mp.lora = a.B;
  mp.n_out = d;
  mp.steps_main = static_cast<int32_t>(pl.nt ? ceil_div(k, 128) : k / 64);   // the swapped kernel steps 128 wide
  mp.ext_steps = rp / 64;
  mp.steps_per_split = static_cast<int32_t>(ceil_div(mp.steps_main, pl.main_splits));
  mp.splits = static_cast<int32_t>(ceil_div(mp.steps_main, mp.steps_per_split));
  mp.out = a.Y;
  mp.partial = reinterpret_cast<float*>(ws + pl.off_main);
  CUtensorMap t_act, t_codes, t_ext;
  const int nt = pl.nt;
  bool ok;
  if (nt) {
    ok = map_bf16(&t_act, a.X, k, M, 64, nt) &&
         make_map(&t_codes, q.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, k / 2, d, k / 2, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_64B) &&
         map_bf16(&t_ext, T, rp, M, 64, nt);
  } else {
    // paired kernel: each CTA loads the codes of its 128-row half
    ok = map_bf16(&t_act, a.X, k, M, 64, 256) &&
         make_map(&t_codes, q.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, k / 2, d, k / 2, 32, 128,
                  CU_TENSOR_MAP_SWIZZLE_NONE) &&
         map_bf16(&t_ext, T, rp, M, 64, 256);
  }
  if (!ok) {
    *why = "tensor map encoding failed (forward)";
    return QLORA_ERR_CUDA;
  }
  dim3 grid;
  if (nt) {
    grid = dim3(static_cast<unsigned>(ceil_div(d, 128)), 1, static_cast<unsigned>(mp.splits));
  } else {
    // token tiles rounded up to whole pairs (a CTA past M still dequantises its half)
    mp.ncp = static_cast<int32_t>(ceil_div(d, 256));
    grid = dim3(static_cast<unsigned>(2 * ceil_div(M, 512) * mp.ncp), 1, static_cast<unsigned>(mp.splits));
  }
  switch (nt) {
    case 16: rc = launch_swap<16>(t_act, t_codes, t_ext, mp, grid, st, why); break;
    case 32: rc = launch_swap<32>(t_act, t_codes, t_ext, mp, grid, st, why); break;
    case 64: rc = launch_swap<64>(t_act, t_codes, t_ext, mp, grid, st, why); break;
    case 128: rc = launch_swap<128>(t_act, t_codes, t_ext, mp, grid, st, why); break;
    default: rc = launch_pair<false>(t_act, t_codes, t_ext, mp, grid, st, why); break;
  }
  if (rc) return rc;
  if (mp.splits > 1) {
    const int64_t count = M * d;
    {
      ProfScope ps_(QLORA_KC_AUX, st);
      (void)launch_pdl(k_reduce_bf16, dim3(static_cast<unsigned>(grid1d(count / 4, 256))), dim3(256), 0, st,
                       nullptr, mp.partial, mp.splits, count, 1.0f, a.Y);
    }
    QL_CHECK_LAUNCH("reduce launch (forward)");
  }
  return 0;
}

int launch_linear_bwd(const LinearArgs& a, cudaStream_t st, const char** why) {
  const int64_t M = a.M, d = a.d, k = a.k;
  const int rp = a.rp, r = a.r;
  Plan pl = make_plan(M, d, k, r, true, true);
  char* ws = static_cast<char*>(a.ws);
  const qlora_nf4_t& q = *a.q;
  int rc;
  if (M == 0) {
    cudaMemsetAsync(a.dA, 0, static_cast<size_t>(r) * k * 4, st);
    cudaMemsetAsync(a.dB, 0, static_cast<size_t>(d) * rank_group(a) * 4, st);
    return 0;
  }
  // adapter dropout: the same keep decisions as the forward, regenerated
  const uint32_t* keep = nullptr;
  rc = dropout_mask(a, true, st, why, &keep);
  if (rc) return rc;
  const float dscale = a.drop ? a.drop->dscale : 1.0f;
  // T_s (recompute when not saved)
  const uint16_t* T = a.Tin;
  if (!T) {
    uint16_t* Tw = reinterpret_cast<uint16_t*>(ws + pl.off_T);
    rc = run_lowrank_down(a.X, M, k, a.A, r, false, rp, a.s * dscale, pl.splits_T, Tw, st, why, keep);
    if (rc) return rc;
    T = Tw;
  }
  // U_s = BF16(s dY B).  B (d x r) is read as an MN-major operand straight from
  // its row-major storage when its rows are 16-byte multiples; otherwise a
  // K-major copy B^T (rp x d) is made first.
  uint16_t* U = reinterpret_cast<uint16_t*>(ws + pl.off_U);
  if (a.ngrp > 1) {
    // grouped: U_s = s dY B' with B' (d x r) block diagonal, projection i's B
    // in columns [i r_group, (i + 1) r_group); one pass over dY for all
    uint16_t* Bd = reinterpret_cast<uint16_t*>(ws + pl.off_Bt);
    BlockDiag bd{};
    bd.d = d;
    bd.r_group = rank_group(a);
    bd.r = r;
    bd.ngrp = a.ngrp;
    for (int i = 0; i < 3; ++i) bd.gstart[i] = a.gstart[i];
    {
      ProfScope ps_(QLORA_KC_AUX, st);
      (void)launch_pdl(k_blockdiag_B, dim3(static_cast<unsigned>(grid1d(d * r / 8, 256))), dim3(256), 0, st, nullptr,
                       a.B, bd, Bd);
    }
    QL_CHECK_LAUNCH("block-diagonal B launch");
    rc = run_lowrank_down(a.dY, M, d, Bd, r, true, rp, a.s, pl.splits_U, U, st, why);
  } else if (r % 8 == 0) {
    rc = run_lowrank_down(a.dY, M, d, a.B, r, true, rp, a.s, pl.splits_U, U, st, why);
  } else {
    uint16_t* Bt = reinterpret_cast<uint16_t*>(ws + pl.off_Bt);
    {
      ProfScope ps_(QLORA_KC_AUX, st);
      (void)launch_pdl(k_transpose_B, dim3(static_cast<unsigned>(ceil_div(d, 32)), static_cast<unsigned>(rp / 32)),
                       dim3(256), 0, st, nullptr, a.B, d, r, rp, Bt);
    }
    QL_CHECK_LAUNCH("transpose launch");
    rc = run_lowrank_down(a.dY, M, d, Bt, rp, false, rp, a.s, pl.splits_U, U, st, why);
  }
  if (rc) return rc;

  // dX = dY W + U_s A
  if (a.dX) {
    MainParams mp{};
    mp.M = M; mp.d = d; mp.k = k; mp.r = r; mp.rp = rp;
    mp.kpb = static_cast<int32_t>(k / 64);
    mp.sc = scale_src(q, a);
    mp.r_group = rank_group(a);
    mp.lora = a.A;
    mp.n_out = k;
    mp.steps_main = static_cast<int32_t>(ceil_div(d, 64));
    // with dropout the adapter term is masked elementwise, so it cannot share
    // the base accumulator: it is added afterwards by the dropout kernel
    mp.ext_steps = keep ? 0 : rp / 64;
    mp.steps_per_split = static_cast<int32_t>(ceil_div(mp.steps_main, pl.main_splits));
    mp.splits = static_cast<int32_t>(ceil_div(mp.steps_main, mp.steps_per_split));
    mp.out = a.dX;
    mp.partial = reinterpret_cast<float*>(ws + pl.off_main);
    CUtensorMap t_act, t_codes, t_ext;
    if (!map_bf16(&t_act, a.dY, d, M, 64, 256) ||
        !make_map(&t_codes, q.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, k / 2, d, k / 2, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_64B) ||
        !map_bf16(&t_ext, U, rp, M, 64, 256)) {
      *why = "tensor map encoding failed (backward)";
      return QLORA_ERR_CUDA;
    }
    mp.ncp = static_cast<int32_t>(ceil_div(k, 256));
    dim3 grid(static_cast<unsigned>(2 * ceil_div(M, 512) * mp.ncp), 1, static_cast<unsigned>(mp.splits));
    rc = launch_pair<true>(t_act, t_codes, t_ext, mp, grid, st, why);
    if (rc) return rc;
    if (mp.splits > 1) {
      const int64_t count = M * k;
      {
        ProfScope ps_(QLORA_KC_AUX, st);
        (void)launch_pdl(k_reduce_bf16, dim3(static_cast<unsigned>(grid1d(count / 4, 256))), dim3(256), 0, st,
                         nullptr, mp.partial, mp.splits, count, 1.0f, a.dX);
      }
      QL_CHECK_LAUNCH("reduce launch (dX)");
    }
    if (keep && launch_lora_up_dropout(U, rp, a.A, r, keep, dscale, M, k, a.dX, st) != cudaSuccess) {
      *why = "dropout adapter-term launch (dX)";
      return QLORA_ERR_CUDA;
    }
  }

  // dA^T = X^T U_s  and  dB = dY^T T_s  (reduction over tokens, MN-major operands)
  {
    CUtensorMap ta, tb;
    if (!map_bf16(&ta, a.X, k, M, 64, 64) || !map_bf16(&tb, U, rp, M, 64, 64)) {
      *why = "tensor map encoding failed (dA)";
      return QLORA_ERR_CUDA;
    }
    ThinParams tp{};
    tp.rows = k;
    tp.rp = rp;
    tp.steps = static_cast<int>(ceil_div(M, 64));
    tp.mode = THIN_DA;
    tp.r = r;
    tp.ld = k;
    tp.outf = a.dA;
    tp.scale = dscale;          // dA = U_s^T (X . keep) / (1 - p)
    tp.keep = keep;
    tp.keep_rows = M;
    tp.keep_ld = k;
    rc = launch_thin<true, true>(ta, tb, tp, ceil_div(k, 128), pl.splits_dA, st, why);
    if (rc) return rc;
  }
  {
    CUtensorMap ta, tb;
    if (!map_bf16(&ta, a.dY, d, M, 64, 64) || !map_bf16(&tb, T, rp, M, 64, 64)) {
      *why = "tensor map encoding failed (dB)";
      return QLORA_ERR_CUDA;
    }
    ThinParams tp{};
    tp.rows = d;
    tp.rp = rp;
    tp.steps = static_cast<int>(ceil_div(M, 64));
    tp.mode = THIN_DB;
    tp.r = r;
    tp.outf = a.dB;
    tp.scale = 1.0f;
    tp.ngrp = a.ngrp;
    tp.r_group = rank_group(a);
    for (int i = 0; i < 3; ++i) tp.gstart[i] = a.gstart[i];
    rc = launch_thin<true, true>(ta, tb, tp, ceil_div(d, 128), pl.splits_dB, st, why);
    if (rc) return rc;
  }
  return 0;
}


}  // namespace qlora
