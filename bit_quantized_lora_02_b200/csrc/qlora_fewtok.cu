// qlora_fewtok.cu -- the QLoRA forward for a few tokens (M <= 32).
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora), "Double quantization
// and double dequantization": Y = X doubleDequant(c1, c2, W_NF4)^T + X L1 L2,
// with the LoRA term written as (alpha/r) (X A^T) B^T ("How does alpha/r
// control adapter strength?").
//
// With a handful of tokens each 4-bit weight takes part in at most 32
// products, so the layer is bound by streaming the packed codes from HBM
// (half a byte per weight).  This path keeps the expanded weights in registers
// and is organised around keeping enough bytes in flight:
//
//   * Work items are 256 weight rows x 256 columns (32 KB of codes; 128 rows
//     for 17..32 tokens, so that a warp's partial sums stay in registers),
//     split evenly over one CTA per SM.  TMA brings each item's code tile and the
//     matching 256 columns of X (one 3-D box) through a ring of up to five
//     stages; the refill of the stage of item i with item i + S is issued by
//     warp i mod 16, so issuing costs no single warp more than its share.  The
//     8-bit block constants c2 come with the first item of each group of four
//     (16 blocks x the item's rows, two slots).  A row's group constant c1 changes
//     at most every 256 blocks and is reloaded only when it does.  (Without
//     TMA-able c2 rows, or without double quantisation, the per-block
//     constants are loaded one item ahead.)
//   * A code byte (two weights) is expanded with one shared-memory lookup: a
//     256-entry table holds the bf16 pair (C[low nibble], C[high nibble]),
//     replicated per lane (a lane always reads its own bank).  Entries are
//     256 bytes apart from a 64 KB-aligned base, so a single byte permute
//     turns a code byte into its lookup address.
//   * Products run on mma.sync m16n8k16 (bf16 operands, fp32 accumulation):
//     the weights are the register-resident A operand and 8 tokens the N side
//     (one, two or four token groups).
//     Inside a 64-weight block the K order is permuted so that each lane's own
//     code bytes fill its fragment slots; X is read with the same permutation.
//     Tensor-core instructions that take their operands from shared memory
//     would need every expanded weight written to and read back from shared
//     memory, which at this arithmetic intensity costs more than the HBM
//     stream itself.
//   * The codebook enters the products unscaled; each block's partial sum is
//     multiplied by its scale s^ in fp32.  C[q] in bf16 times s^ carries the
//     same bound, 2^-9 relative, as the bf16 weight BF16(C[q] s^) that the
//     dequantisation produces.
//   * When a CTA leaves a row block it writes its partial sums.  A second
//     kernel, k_fewtok_finish, adds each row block's partial sums in CTA
//     order, adds the LoRA term T_s B^T (mma.sync) and writes Y.
//   * The down projection T_s = BF16(s X A^T) costs no launch of its own: the
//     first 32 CTAs of the main kernel prefetch 32 shares of K of X and A
//     into L2 when they start and compute their partial sums of X A^T after
//     their last item; the finish kernel adds the 32 in order (every CTA for
//     its row block's columns, and all CTAs together for the saved T_s).
//
// Both kernels are programmatic dependents: the streaming kernel builds its
// lookup table and barriers while the kernel before it drains and waits for
// it before reading any input; the finish kernel is scheduled as the
// streaming kernel's CTAs exit.
#include <cstdio>

#include "nf4_scale.cuh"
#include "nf4_table.h"
#include "qlora_device.cuh"
#include "qlora_internal.h"

namespace qlora {

namespace {

constexpr int kFtWarps = 16;                                // 4 per SM sub-partition: up to 128 registers
constexpr int kFtThreads = kFtWarps * 32;
constexpr int kFtK = 256;                                   // weights per row per item
constexpr int kFtMaxTok = 32;                               // tokens this path takes
constexpr int kFtMaxStages = 5;
constexpr uint32_t kFtTableBytes = 65536;
constexpr uint32_t kFtSmemBytes = 227u * 1024u;             // the whole window; placed in the kernel
constexpr int kFtC2Slots = 2;

// NTOK = 8 or 16 tokens: items of 256 weight rows, each warp 64 rows (four
// 16-row MMA groups).  NTOK = 32: items of 128 rows, each warp 32 rows (two
// groups), so that a warp's partial sums (rows x 32 tokens) still fit in
// registers.  Row blocks (the rows whose partial sums a CTA writes and the
// finish kernel combines) are one item high.
template <int NTOK>
struct FtCfg {
  static constexpr int kTG = NTOK / 8;                             // token groups of 8 (MMA N)
  static constexpr int kRows = NTOK == 32 ? 128 : 256;             // weight rows per item
  static constexpr int kSetRows = kRows / 4;                       // rows of a warp (its row set)
  static constexpr int kRG = kSetRows / 16;                        // 16-row MMA groups of a warp
  static constexpr int kLaneRows = kSetRows / 32;                  // rows whose s^ one lane computes
  static constexpr uint32_t kCodeBytes = kRows * kFtK / 2;         // codes of an item
  static constexpr uint32_t kXBox = NTOK * 128u;                   // 64 columns of X for NTOK tokens
  static constexpr uint32_t kStageBytes = kCodeBytes + 4u * kXBox;
  static constexpr uint32_t kC2Box = 16u * kRows;                  // c2 of 16 blocks (four items)
  static constexpr uint32_t kScratch = 4u * kRG * kTG * 32u * 16u;  // [row set][row group, token group][lane] float4
  static constexpr uint32_t kMisc = 128;                           // barriers and flags
};
constexpr int ft_rows(int ntok) { return ntok == 32 ? 128 : 256; }

constexpr int kFtTProd = 32;   // CTAs of the main kernel that compute partial sums of X A^T

struct FtParams {
  int64_t M, d, k;
  int32_t kpb;          // NF4 blocks per weight row
  int32_t r, rp;         // r: the rank of one projection (B's row length); rp: T_s's row length
  int32_t rA;            // rows of A (every projection's r rows, stacked)
  ScaleSrc sc;            // grouped weights: rows from sc.gstart[i] on belong to projection i + 1
  const uint16_t* X;    // M x k
  const uint16_t* A;    // rA x k
  const uint32_t* keep;  // adapter dropout: keep bits of X (bit b of word w <-> element 32 w + b), or null
  float s_down;         // s, times 1 / (1 - p) of the kept elements with adapter dropout
  const uint16_t* B;    // d x r (projections' rows stacked)
  uint16_t* T;          // M x rp, T_s (written by the finish kernel)
  uint16_t* Y;          // M x d
  float* partial;       // [G][segmax][NTOK][rows of a row block]
  float* tpart;         // [tprod][32][rp]: each producer CTA's sums of X A^T over its share of K
  int32_t items, KC, G, segmax, tprod;
  int32_t c2_tma;       // c2 arrives through the TMA ring (double quantisation, kpb % 16 == 0)
};

// Shared-memory placement.  The lookup table needs a 64 KB-aligned base.  For
// each possible table position the ring stages (1 KB-aligned for the 128-byte
// swizzle) fill the space below and above it, then the small pieces (c2 ring,
// scratch, barriers) take the first gap that holds them; the position that
// leaves room for the most stages wins.  Stages below the table are numbered
// first: stage i < nlo sits at lo0 + i * stage bytes, the rest at hi0 + ...
struct FtLayout {
  uint32_t table, misc, scratch, c2, lo0, hi0;
  int nlo, nst;
  bool ok;
};

template <int NTOK>
__device__ __forceinline__ FtLayout ft_layout(uint32_t raw) {
  using Cfg = FtCfg<NTOK>;
  constexpr uint32_t SB = Cfg::kStageBytes;
  FtLayout best{};
  best.ok = false;
  const uint32_t end = raw + kFtSmemBytes;
  for (uint32_t T = (raw + kFtTableBytes - 1u) & ~(kFtTableBytes - 1u); T + kFtTableBytes <= end; T += kFtTableBytes) {
    const uint32_t lo0 = (raw + 1023u) & ~1023u, hi0 = T + kFtTableBytes;
    const int maxlo = lo0 <= T ? static_cast<int>((T - lo0) / SB) : 0;
    const int maxhi = static_cast<int>((end - hi0) / SB);
    for (int nlo = maxlo; nlo >= 0; --nlo) {
      int nhi = maxhi;
      if (nlo + nhi > kFtMaxStages) nhi = kFtMaxStages - nlo;
      if (nhi < 0) continue;
      for (; nhi >= 0; --nhi) {
        if (best.ok && nlo + nhi <= best.nst) break;
        uint32_t a = lo0 + nlo * SB, b = hi0 + nhi * SB;
        auto take = [&](uint32_t bytes, uint32_t align, uint32_t& out) -> bool {
          uint32_t x = (a + align - 1u) & ~(align - 1u);
          if (x + bytes <= T) {
            out = x;
            a = x + bytes;
            return true;
          }
          x = (b + align - 1u) & ~(align - 1u);
          if (x + bytes <= end) {
            out = x;
            b = x + bytes;
            return true;
          }
          return false;
        };
        FtLayout L{};
        if (take(kFtC2Slots * Cfg::kC2Box, 128u, L.c2) && take(Cfg::kScratch, 16u, L.scratch) &&
            take(Cfg::kMisc, 16u, L.misc)) {
          L.table = T;
          L.lo0 = lo0;
          L.hi0 = hi0;
          L.nlo = nlo;
          L.nst = nlo + nhi;
          L.ok = L.nst >= 3;
          if (L.ok) best = L;
          break;
        }
      }
    }
  }
  return best;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Lookup in the constant code-byte table (written once before a CTA-wide
// barrier): no ordering constraints, so the compiler may batch them.
__device__ __forceinline__ uint32_t lds32_const(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// D += A B: 16 x 8 x 16, bf16 inputs, fp32 accumulators (register fragments).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A B (no accumulator input).
__device__ __forceinline__ void mma16816_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// The CTA whose item range holds item i (ranges: [c I / G, (c+1) I / G)).
__device__ __forceinline__ int cta_of_item(int64_t i, int items, int G) {
  return static_cast<int>(((i + 1) * G + items - 1) / items) - 1;
}
__device__ __forceinline__ int first_item(int c, int items, int G) {
  return static_cast<int>(static_cast<int64_t>(c) * items / G);
}

// Two bf16 at an even element offset as one 32-bit word (4-byte aligned).
__device__ __forceinline__ uint32_t ld_pair(const uint16_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

}  // namespace

// ============================================================================
// Partial sums of X A^T on mma.sync, computed by the first tprod CTAs of the
// main kernel after their last item (their shares of X and A were prefetched
// into L2 at the start): 16 tokens are the M side (one or two halves of 16),
// 8 ranks the N side.  Producer q takes the 16-column steps
// [n16 q / tprod, n16 (q + 1) / tprod) of K; its
// warps split the rank groups of 8 and, within one, the steps; the warps of a
// rank group add their sums in warp order through shared memory and write
// tpart[q][token][rank].  The finish kernel adds the producers' sums in order,
// so T_s = BF16(s X A^T) is the same on every run.
// With adapter dropout `keep` is the keep bitmask of X and dropped elements
// enter the products as zeros; s_down then includes the 1 / (1 - p).
// ============================================================================
// 32-bit lane mask of a bf16 pair from its two keep bits (bit 0: low element)
__device__ __forceinline__ uint32_t pair_keep_mask(uint32_t two) {
  return ((two & 1u) ? 0x0000FFFFu : 0u) | ((two & 2u) ? 0xFFFF0000u : 0u);
}

// L2 prefetch of producer q's columns of X and A (one bulk prefetch per row:
// 32 bytes per 16-column step, 16-byte aligned since k % 64 == 0)
__device__ __forceinline__ void ft_down_prefetch(const FtParams& p, int q) {
  const int64_t n16 = p.k >> 4;
  const int64_t q0 = n16 * q / p.tprod, q1 = n16 * (q + 1) / p.tprod;
  const uint32_t bytes = static_cast<uint32_t>(32 * (q1 - q0));
  if (bytes == 0) return;
  for (int row = threadIdx.x; row < p.M + p.rA; row += blockDim.x) {
    const uint16_t* src = (row < p.M ? p.X + static_cast<int64_t>(row) * p.k
                                     : p.A + static_cast<int64_t>(row - p.M) * p.k) + 16 * q0;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
  }
}

// NH token halves of 16 (NH = 2 for the 32-token kernel, whose scratch holds
// the 16 KB of red that two halves need)
template <int NH>
__device__ __forceinline__ void ft_down_part(const FtParams& p, int q, float4* red, int warp, int lane) {
  const int g = lane >> 2, c = lane & 3;
  const int64_t k = p.k;
  const int nrg = (p.rA + 7) >> 3;                        // rank groups of 8
  const int wpg = nrg >= kFtWarps ? 1 : kFtWarps / nrg;   // warps per rank group
  const int per_pass = kFtWarps / wpg;                    // rank groups per pass
  const int sub = warp % wpg, slot = warp / wpg;
  const int64_t n16 = k >> 4;
  const int64_t q0 = n16 * q / p.tprod, q1 = n16 * (q + 1) / p.tprod;
  const int64_t s0 = q0 + (q1 - q0) * sub / wpg, s1 = q0 + (q1 - q0) * (sub + 1) / wpg;
  for (int rg0 = 0; rg0 < nrg; rg0 += per_pass) {
    const int rgi = rg0 + slot;
    const bool active = slot < per_pass && rgi < nrg;
    float acc[NH][4];
#pragma unroll
    for (int h = 0; h < NH; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.0f;
    if (active) {
      const int j0 = 8 * rgi;
      const bool jv = j0 + g < p.rA;
      const uint16_t* ar = p.A + static_cast<int64_t>(j0 + g) * k + 2 * c;
#pragma unroll 8
      for (int64_t st = s0; st < s1; ++st) {
        const int64_t k0 = 16 * st;
        const uint32_t b0 = jv ? ld_pair(ar + k0) : 0u, b1 = jv ? ld_pair(ar + k0 + 8) : 0u;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          // tokens 16 h + g (fragment rows 0..7) and 16 h + g + 8 (rows 8..15)
          const int ta_tok = 16 * h + g, tb_tok = ta_tok + 8;
          const bool ta = ta_tok < p.M, tb = tb_tok < p.M;
          const uint16_t* xa = p.X + static_cast<int64_t>(ta_tok) * k + 2 * c + k0;
          const uint16_t* xb = p.X + static_cast<int64_t>(tb_tok) * k + 2 * c + k0;
          uint32_t a0 = ta ? ld_pair(xa) : 0u, a2 = ta ? ld_pair(xa + 8) : 0u;
          uint32_t a1 = tb ? ld_pair(xb) : 0u, a3 = tb ? ld_pair(xb + 8) : 0u;
          if (p.keep) {
            // keep bits of columns k0 .. k0 + 15 of the two tokens (k0 % 16 == 0,
            // k % 64 == 0: the 16 bits sit in one word at bit 0 or 16)
            if (ta) {
              const int64_t e = static_cast<int64_t>(ta_tok) * k + k0;
              const uint32_t w = __ldg(p.keep + (e >> 5)) >> (e & 31);
              a0 &= pair_keep_mask(w >> (2 * c));
              a2 &= pair_keep_mask(w >> (8 + 2 * c));
            }
            if (tb) {
              const int64_t e = static_cast<int64_t>(tb_tok) * k + k0;
              const uint32_t w = __ldg(p.keep + (e >> 5)) >> (e & 31);
              a1 &= pair_keep_mask(w >> (2 * c));
              a3 &= pair_keep_mask(w >> (8 + 2 * c));
            }
          }
          mma16816(acc[h], a0, a1, a2, a3, b0, b1);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < NH; ++h)
      red[(h * kFtWarps + warp) * 32 + lane] = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
    __syncthreads();
    if (active && sub == 0) {
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float4 t = red[(h * kFtWarps + warp) * 32 + lane];
        for (int u = 1; u < wpg; ++u) {
          const float4 v = red[(h * kFtWarps + warp + u) * 32 + lane];
          t.x += v.x;
          t.y += v.y;
          t.z += v.z;
          t.w += v.w;
        }
        // fragment element e: token 16 h + g + 8 (e >> 1), rank 8 rgi + 2 c + (e & 1) (< rp)
        float* dst = p.tpart + (static_cast<int64_t>(q) * kFtMaxTok + 16 * h) * p.rp + 8 * rgi + 2 * c;
        dst[g * p.rp] = t.x;
        dst[g * p.rp + 1] = t.y;
        dst[(g + 8) * p.rp] = t.z;
        dst[(g + 8) * p.rp + 1] = t.w;
      }
    }
    __syncthreads();   // red is reused by the next pass (and, after the last, by the flushes)
  }
}

// T_s[tok][j] = BF16(s_down * sum over producers of tpart[.][tok][j]), the
// producers added in order.  ft_t_load issues the loads (zeros when !live),
// ft_t_bits adds and rounds.
__device__ __forceinline__ void ft_t_load(const FtParams& p, int tok, int j, bool live, float (&v)[kFtTProd]) {
  const float* src = p.tpart + static_cast<int64_t>(tok) * p.rp + j;
#pragma unroll
  for (int q = 0; q < kFtTProd; ++q)
    v[q] = (live && q < p.tprod) ? __ldcg(src + static_cast<int64_t>(q) * kFtMaxTok * p.rp) : 0.0f;
}
__device__ __forceinline__ uint16_t ft_t_bits(const FtParams& p, const float (&v)[kFtTProd]) {
  float t = v[0];
#pragma unroll
  for (int q = 1; q < kFtTProd; ++q) t += v[q];
  return static_cast<uint16_t>(pack_bf16x2(p.s_down * t, 0.0f) & 0xFFFFu);
}
__device__ __forceinline__ uint16_t ft_t_value(const FtParams& p, int tok, int j, bool live) {
  float v[kFtTProd];
  ft_t_load(p, tok, j, live, v);
  return ft_t_bits(p, v);
}

// ============================================================================
// Main kernel
// ============================================================================
// Combine the four warps that share a 64-row set (one per 64-column block of
// the item) and write the CTA's partial sums of the row block it leaves: in
// three rounds the warps of block b = 1, 2, 3 park their sums in shared memory
// (slot [row set][row group, token group][lane] of 16 bytes, so that a warp's
// stores and loads cover consecutive banks) and the block-0 warp adds them in
// order.  MMA row g of row group rg is weight row 16 rg + pg (and + 8).
template <int NTOK>
__device__ __forceinline__ void ft_flush(float (&acc)[FtCfg<NTOK>::kRG][FtCfg<NTOK>::kTG][4], float* scratch,
                                         float* part, int rs, int bk, int lane, int pg) {
  using Cfg = FtCfg<NTOK>;
  constexpr int TG = Cfg::kTG, RG = Cfg::kRG, R = Cfg::kRows;
  float4* scr = reinterpret_cast<float4*>(scratch) + rs * RG * TG * 32 + lane;
  for (int b = 1; b < 4; ++b) {
    __syncthreads();   // the slot is free (block-0 warps have read the previous round)
    if (bk == b) {
#pragma unroll
      for (int rg = 0; rg < RG; ++rg)
#pragma unroll
        for (int t = 0; t < TG; ++t)
          scr[(rg * TG + t) * 32] = make_float4(acc[rg][t][0], acc[rg][t][1], acc[rg][t][2], acc[rg][t][3]);
    }
    __syncthreads();
    if (bk == 0) {
#pragma unroll
      for (int rg = 0; rg < RG; ++rg)
#pragma unroll
        for (int t = 0; t < TG; ++t) {
          const float4 v = scr[(rg * TG + t) * 32];
          acc[rg][t][0] += v.x;
          acc[rg][t][1] += v.y;
          acc[rg][t][2] += v.z;
          acc[rg][t][3] += v.w;
        }
    }
  }
  if (bk == 0) {
    const int c = lane & 3;
#pragma unroll
    for (int rg = 0; rg < RG; ++rg)
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        const int row = Cfg::kSetRows * rs + 16 * rg + pg;
        const int tok = 8 * t + 2 * c;
        part[tok * R + row] = acc[rg][t][0];
        part[(tok + 1) * R + row] = acc[rg][t][1];
        part[tok * R + row + 8] = acc[rg][t][2];
        part[(tok + 1) * R + row + 8] = acc[rg][t][3];
      }
  }
#pragma unroll
  for (int rg = 0; rg < RG; ++rg)
#pragma unroll
    for (int t = 0; t < TG; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[rg][t][e] = 0.0f;
}

// Row block rb: Y = BF16(sum of the CTAs' partial sums + T_s B^T); warp w
// takes rows 16 w .. 16 w + 15 of the block.  All global loads of a batch are
// issued before any is used (a row block has a few contributors and r / 16
// LoRA steps).
// T_s of the row block's projection in shared memory: token tok's columns at
// ts + tok * kTsWords (32-bit pairs), zero past M tokens and past r columns
constexpr int kTsWords = 132;   // 128 pairs (r <= 256) + 4: a warp's pair loads hit 32 distinct banks

// between() runs after the partial sums are added and before the LoRA term
// reads ts; it fills ts and ends with a CTA barrier.
template <int NTOK, class Between>
__device__ __forceinline__ void ft_finish(const FtParams& p, int rb, int warp, int lane, const uint32_t* ts,
                                          Between between) {
  constexpr int TG = NTOK / 8;
  constexpr int R = FtCfg<NTOK>::kRows;
  constexpr int kC = TG <= 2 ? 4 : 2;   // contributors per batch
  constexpr int kS = 4;                 // LoRA K steps (16 ranks each) per batch
  const int g = lane >> 2, c = lane & 3;
  const int64_t na = static_cast<int64_t>(rb) * R + 16 * warp + g, nb = na + 8;
  const int ra = 16 * warp + g;
  float v[TG][4];
#pragma unroll
  for (int t = 0; t < TG; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) v[t][e] = 0.0f;
  const int64_t i0 = static_cast<int64_t>(rb) * p.KC;
  const int cf = cta_of_item(i0, p.items, p.G), cl = cta_of_item(i0 + p.KC - 1, p.items, p.G);
  for (int c0 = cf; c0 <= cl; c0 += kC) {
    float pv[kC][TG][4];
#pragma unroll
    for (int u = 0; u < kC; ++u) {
      const int cc = c0 + u;
      const bool ok = cc <= cl;
      const int seg = ok ? rb - first_item(cc, p.items, p.G) / p.KC : 0;
      const float* part = p.partial + (static_cast<int64_t>(ok ? cc : cf) * p.segmax + seg) * NTOK * R;
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        const int tok = 8 * t + 2 * c;
        pv[u][t][0] = ok ? part[tok * R + ra] : 0.0f;
        pv[u][t][1] = ok ? part[(tok + 1) * R + ra] : 0.0f;
        pv[u][t][2] = ok ? part[tok * R + ra + 8] : 0.0f;
        pv[u][t][3] = ok ? part[(tok + 1) * R + ra + 8] : 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kC; ++u)
#pragma unroll
      for (int t = 0; t < TG; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) v[t][e] += pv[u][t][e];
  }
  between();
  // LoRA term: rows of B are the A operand, T_s^T (the row block's
  // projection's columns, in shared memory) the B operand.
  const bool even = (p.r & 1) == 0;
  auto bpair = [&](int64_t n, int j) -> uint32_t {
    if (n >= p.d || j >= p.r) return 0u;
    const uint16_t* src = p.B + n * p.r + j;
    if (even) return ld_pair(src);
    const uint32_t lo = src[0], hi = (j + 1 < p.r) ? src[1] : 0u;
    return lo | (hi << 16);
  };
  for (int k0 = 0; 16 * k0 < p.r; k0 += kS) {
    uint32_t af[kS][4], bf[kS][TG][2];
#pragma unroll
    for (int u = 0; u < kS; ++u) {
      const int j0 = 16 * (k0 + u) + 2 * c;
      const bool ok = 16 * (k0 + u) < p.r;
      af[u][0] = ok ? bpair(na, j0) : 0u;
      af[u][1] = ok ? bpair(nb, j0) : 0u;
      af[u][2] = ok ? bpair(na, j0 + 8) : 0u;
      af[u][3] = ok ? bpair(nb, j0 + 8) : 0u;
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        const int tok = 8 * t + g;
        const uint32_t* trow = ts + tok * kTsWords;
        bf[u][t][0] = ok ? trow[j0 >> 1] : 0u;
        bf[u][t][1] = ok ? trow[(j0 >> 1) + 4] : 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < kS; ++u)
#pragma unroll
      for (int t = 0; t < TG; ++t) mma16816(v[t], af[u][0], af[u][1], af[u][2], af[u][3], bf[u][t][0], bf[u][t][1]);
  }
#pragma unroll
  for (int t = 0; t < TG; ++t) {
    const int tok = 8 * t + 2 * c;
    auto put = [&](int tk, int64_t n, float x) {
      if (tk < p.M && n < p.d) p.Y[static_cast<int64_t>(tk) * p.d + n] = static_cast<uint16_t>(pack_bf16x2(x, 0.0f));
    };
    put(tok, na, v[t][0]);
    put(tok + 1, na, v[t][1]);
    put(tok, nb, v[t][2]);
    put(tok + 1, nb, v[t][3]);
  }
}

// One CTA per row block, one warp per 16 rows; launched as the programmatic
// dependent of the main kernel.  The T_s values a thread produces (one of the row block's
// projection, one of the saved M x rp output) have their loads issued before
// the partial sums' loads, so both arrive in one round trip.
template <int NTOK>
__global__ void __launch_bounds__(kFtThreads) k_fewtok_finish(const FtParams p) {
  __shared__ uint32_t ts[NTOK * kTsWords];
  griddep_wait();   // the main kernel's partial sums of W^ X and of X A^T
  const int tid = threadIdx.x;
  const int toff = group_of(p.sc, static_cast<int64_t>(blockIdx.x) * FtCfg<NTOK>::kRows) * p.r;
  const int ncol = (p.r + 15) / 16 * 16;   // columns the LoRA steps read (zero past r)
  const int nts = NTOK * ncol;
  const int tt = tid / ncol, tj = tid - tt * ncol;
  float tv[kFtTProd];
  ft_t_load(p, tt, toff + tj, tid < nts && tt < p.M && tj < p.r, tv);
  const int64_t nT = p.M * p.rp, e0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + tid;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int st0 = static_cast<int>(e0 / p.rp), sj0 = static_cast<int>(e0 - static_cast<int64_t>(st0) * p.rp);
  float sv[kFtTProd];
  ft_t_load(p, st0, sj0, e0 < nT && sj0 < p.rA, sv);
  uint16_t* ts16 = reinterpret_cast<uint16_t*>(ts);
  ft_finish<NTOK>(p, blockIdx.x, tid >> 5, tid & 31, ts, [&]() {
    // the row block's projection's T_s columns (zero past M tokens and past r)
    if (tid < nts) ts16[tt * 2 * kTsWords + tj] = ft_t_bits(p, tv);
    for (int i = tid + blockDim.x; i < nts; i += blockDim.x) {
      const int tok = i / ncol, j = i - tok * ncol;
      ts16[tok * 2 * kTsWords + j] = ft_t_value(p, tok, toff + j, tok < p.M && j < p.r);
    }
    // this CTA's share of the saved T_s (zero past rA columns)
    if (e0 < nT) p.T[e0] = ft_t_bits(p, sv);
    for (int64_t e = e0 + stride; e < nT; e += stride) {
      const int tok = static_cast<int>(e / p.rp), j = static_cast<int>(e - static_cast<int64_t>(tok) * p.rp);
      p.T[e] = ft_t_value(p, tok, j, j < p.rA);
    }
    __syncthreads();
  });
}

// CM selects how the block constants arrive: 0 = any mode (c2 loaded one item
// ahead, or absmax without double quantisation, or c2 through TMA), 1 = Int8
// c2 through TMA, 2 = E4M3 c2 through TMA.  Modes 1 and 2 carry no per-item
// branches on the mode and check a row's c1 group only when its block index
// reaches the next group boundary.
template <int NTOK, int CM>
__global__ void __launch_bounds__(kFtThreads, 1)
    k_qlora_fewtok(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_c2, const __grid_constant__ FtParams p) {
  using Cfg = FtCfg<NTOK>;
  constexpr int TG = Cfg::kTG;
  extern __shared__ __align__(1024) uint8_t ft_smem[];
  const uint32_t raw = smem_u32(ft_smem);
  const FtLayout L = ft_layout<NTOK>(raw);
  if (!L.ok) {
    if (threadIdx.x == 0) report(DEV_SMEM_LAYOUT);
    return;
  }
  auto gptr = [&](uint32_t a) { return ft_smem + (a - raw); };
  uint64_t* full = reinterpret_cast<uint64_t*>(gptr(L.misc));
  uint64_t* empty = full + kFtMaxStages;
  volatile int* last_item = reinterpret_cast<volatile int*>(full + 2 * kFtMaxStages);   // per stage, for draining
  volatile int* abort_flag = last_item + kFtMaxStages;
  const int S = L.nst;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it0 = first_item(blockIdx.x, p.items, p.G);
  const int it1 = first_item(blockIdx.x + 1, p.items, p.G);
  const int n_items = it1 - it0;
  auto stage = [&](int st) {
    return st < L.nlo ? L.lo0 + static_cast<uint32_t>(st) * Cfg::kStageBytes
                      : L.hi0 + static_cast<uint32_t>(st - L.nlo) * Cfg::kStageBytes;
  };

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kFtWarps);
    }
    for (int i = 0; i < kFtMaxStages; ++i) last_item[i] = -1;
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
    if (p.c2_tma) tma_prefetch_desc(&tm_c2);
  }
  {
    // code-byte table: entry e = (C[e & 15], C[e >> 4]) in bf16; lane l's copy
    // of entry e at e * 256 + 4 l
    constexpr uint32_t kCB[16] = {QLORA_NF4_TABLE_BITS};
    for (int i = threadIdx.x; i < 256 * 32; i += kFtThreads) {
      const int e = i >> 5;
      const uint32_t v = pack_bf16x2(__uint_as_float(kCB[e & 15]), __uint_as_float(kCB[e >> 4]));
      sts32(L.table + static_cast<uint32_t>(e) * 256u + static_cast<uint32_t>(i & 31) * 4u, v);
    }
  }
  __syncthreads();
  // Launched as a programmatic dependent: the set-up above overlaps the kernel
  // before; from here on inputs are read (X, the codes and constants, keep bits)
  griddep_wait();

  // warp = (row set rs: a quarter of the item's rows) x (block bk: 64 columns of the item)
  const int rs = warp & 3, bk = warp >> 2;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t lanebase = L.table + static_cast<uint32_t>(lane) * 4u;
  // MMA row g (and g + 8) of a 16-row group is weight row pg (and pg + 8) of
  // it, pg = 0, 2, 4, 6, 1, 3, 5, 7 for g = 0..7: the rows' 128-byte swizzle
  // then spreads the 8-byte code loads of each half-warp over all 32 banks
  const int pg = ((g & 3) << 1) | (g >> 2);
  // this lane's 8 code bytes of row kSetRows rs + pg in the 128-byte-swizzled tile
  const uint32_t code_off = static_cast<uint32_t>(Cfg::kSetRows * rs + pg) * 128u +
                            16u * static_cast<uint32_t>((2 * bk + (c >> 1)) ^ pg) + 8u * static_cast<uint32_t>(c & 1);
  // this lane's 16 columns of X (token 8 t + g) in the 128-byte-swizzled X chunk of block bk
  const uint32_t x_off = Cfg::kCodeBytes + static_cast<uint32_t>(bk) * Cfg::kXBox + static_cast<uint32_t>(g) * 128u;
  const uint32_t x_c0 = 16u * static_cast<uint32_t>((2 * c) ^ g), x_c1 = 16u * static_cast<uint32_t>((2 * c + 1) ^ g);
  float mean = p.sc.dq ? __ldg(p.sc.mean) : 0.0f;   // of the current row block's projection

  // ---- TMA issue of item j into stage sj: the code tile, the item's 256
  // columns of X and, at the first item of a group of four, the group's c2
  // (slot = group index mod 2; a slot is refilled only after the item that
  // read it has been released, at least five items later).
  auto issue_item = [&](int j, int sj) {
    const int gi = it0 + j, irb = gi / p.KC, ikc = gi - irb * p.KC;
    const bool c2n = p.c2_tma && (j == 0 || (ikc & 3) == 0);
    mbar_arrive_expect_tx(&full[sj], Cfg::kStageBytes + (c2n ? Cfg::kC2Box : 0u));
    uint8_t* dst = gptr(stage(sj));
    tma_load_2d(dst, &tm_codes, &full[sj], ikc * (kFtK / 2), irb * Cfg::kRows);
    tma_load_3d(dst + Cfg::kCodeBytes, &tm_x, &full[sj], 0, 0, 4 * ikc);
    if (c2n)
      tma_load_2d(gptr(L.c2 + ((gi >> 2) & 1) * Cfg::kC2Box), &tm_c2, &full[sj], 4 * (ikc & ~3), irb * Cfg::kRows);
    last_item[sj] = j;
  };
  if (threadIdx.x == 0)
    for (int j = 0; j < n_items && j < S; ++j) issue_item(j, j);
  float* scratch = reinterpret_cast<float*>(gptr(L.scratch));
  // the first tprod CTAs compute partial sums of X A^T after their last item;
  // their shares of X and A are brought into L2 now, behind the first items' copies
  if (static_cast<int>(blockIdx.x) < p.tprod) ft_down_prefetch(p, blockIdx.x);

  // ---- block constants.  This lane computes s^ for row lane (and, with
  // 64-row sets, lane + 32) of its row set and block bk of each item.
  const bool dq = p.sc.dq != 0, c2_tma = p.c2_tma != 0;
  // Per row: flat index of block 0 of the row, the current group of 256
  // blocks and its constant c1 with the correctly rounded reciprocal (s^ =
  // RN(RN(c2 / c1) + mean) through one residual correction; see nf4_scale.cuh).
  struct RowConst {
    int32_t base, grp;   // 32-bit: the launcher requires every row's block indices below 2^31
    float c1, rc;
    bool fast, valid;
  };
  RowConst rw[2];
  int32_t nxt = 0;       // (CM != 0) the block index at which a row of this lane enters another group
  auto set_rows = [&](int rbx) {
    const int64_t r0 = static_cast<int64_t>(rbx) * Cfg::kRows + Cfg::kSetRows * rs + lane;
    // a row block (256 or 128 rows) lies in one projection of a grouped weight
    if (dq && p.sc.ngrp > 1) mean = group_mean(p.sc, static_cast<int64_t>(rbx) * Cfg::kRows);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      rw[h].valid = h < Cfg::kLaneRows && r0 + 32 * h < p.d;
      rw[h].base = static_cast<int32_t>((r0 + 32 * h) * p.kpb);
      rw[h].grp = -1;
      // rows past d: finite placeholders (their sums are never written)
      rw[h].c1 = 1.0f;
      rw[h].rc = 1.0f;
      rw[h].fast = true;
    }
    nxt = 0;
  };
  // (CM != 0) reload c1 where a row's group changed at block blk (clamped to
  // the row's last block in a ragged tail) and find the next boundary
  auto refresh = [&](int32_t blk) {
    const int32_t bq = blk < p.kpb ? blk : p.kpb - 1;
    nxt = INT32_MAX;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (!rw[h].valid) continue;
      const int32_t gq = (rw[h].base + bq) >> 8;
      if (gq != rw[h].grp) {
        rw[h].grp = gq;
        rw[h].c1 = __ldg(p.sc.c1 + gq);
        rw[h].rc = __frcp_rn(rw[h].c1);
        rw[h].fast = (rw[h].c1 >= 0x1p-60f) && (rw[h].c1 <= 0x1p60f);
      }
      nxt = min(nxt, ((gq + 1) << 8) - rw[h].base);
    }
  };
  auto row_scale = [&](RowConst& R, int32_t blk, int c2v) -> float {
    const int32_t gq = (R.base + blk) >> 8;
    if (gq != R.grp) {
      R.grp = gq;
      R.c1 = __ldg(p.sc.c1 + gq);
      R.rc = __frcp_rn(R.c1);
      R.fast = (R.c1 >= 0x1p-60f) && (R.c1 <= 0x1p60f);
    }
    const float w = c2_numerator(p.sc.dq, c2v);
    float q;
    if (R.fast) {
      const float y = __fmul_rn(w, R.rc);
      const float e = __fmaf_rn(-R.c1, y, w);
      q = __fmaf_rn(e, R.rc, y);
    } else {
      q = __fdiv_rn(w, R.c1);
    }
    return __fadd_rn(q, mean);
  };
  // c2 (loaded path) or absmax of the next item
  uint32_t nc2 = 0;
  float nab0 = 0.0f, nab1 = 0.0f;
  auto prefetch = [&](int rbx, int kcx) {
    if (dq && c2_tma) return;
    const int64_t blk = 4ll * kcx + bk;
    const int64_t r0 = static_cast<int64_t>(rbx) * Cfg::kRows + Cfg::kSetRows * rs + lane;
    const bool bv = blk < p.kpb;
    if (dq) {
      const uint32_t a = (bv && r0 < p.d) ? static_cast<uint8_t>(__ldg(p.sc.c2 + r0 * p.kpb + blk)) : 0u;
      const uint32_t b = (Cfg::kLaneRows == 2 && bv && r0 + 32 < p.d)
                             ? static_cast<uint8_t>(__ldg(p.sc.c2 + (r0 + 32) * p.kpb + blk))
                             : 0u;
      nc2 = a | (b << 8);
    } else {
      nab0 = (bv && r0 < p.d) ? __ldg(p.sc.absmax + r0 * p.kpb + blk) : 0.0f;
      nab1 = (Cfg::kLaneRows == 2 && bv && r0 + 32 < p.d) ? __ldg(p.sc.absmax + (r0 + 32) * p.kpb + blk) : 0.0f;
    }
  };
  set_rows(it0 / p.KC);
  if (n_items > 0) prefetch(it0 / p.KC, it0 - (it0 / p.KC) * p.KC);

  constexpr int RG = Cfg::kRG;
  float acc[RG][TG][4];
#pragma unroll
  for (int rg = 0; rg < RG; ++rg)
#pragma unroll
    for (int t = 0; t < TG; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[rg][t][e] = 0.0f;

  // ---- leaving a row block: the CTA's partial sums out
  int seg = 0;
  auto leave_block = [&](int) {
    ft_flush<NTOK>(acc, scratch,
                   p.partial + (static_cast<int64_t>(blockIdx.x) * p.segmax + seg) * NTOK * Cfg::kRows, rs, bk,
                   lane, pg);
    ++seg;
  };

  int st = 0, rb = it0 / p.KC, kc = it0 - rb * p.KC;
  uint32_t ph = 0;
  int pst = 0;        // stage and parity of the previous item
  uint32_t pph = 0;
  uint32_t c2w0 = 0, c2w1 = 0;   // c2 of this lane's two rows for the four items of the group
  const bool loaded_consts = CM == 0 && !(dq && c2_tma);
  for (int i = 0; i < n_items; ++i) {
    const uint32_t cur_c2 = nc2;
    const float cur_ab0 = nab0, cur_ab1 = nab1;
    if (loaded_consts && i + 1 < n_items) prefetch(kc + 1 == p.KC ? rb + 1 : rb, kc + 1 == p.KC ? 0 : kc + 1);

    mbar_wait(&full[st], ph, abort_flag, DEV_WAIT_TIMEOUT_TMA);
    const uint32_t sb = stage(st);
    if ((CM != 0 || p.c2_tma) && (i == 0 || (kc & 3) == 0)) {
      // first item of a group of four: the group's c2, rows lane (and lane + 32)
      // of the row set; byte 4 t + bk is block bk of item t of the group
      const uint32_t cb =
          L.c2 + (((it0 + i) >> 2) & 1) * Cfg::kC2Box + static_cast<uint32_t>(Cfg::kSetRows * rs + lane) * 16u;
      const uint32_t sel = 0x40u + 0x11u * static_cast<uint32_t>(bk);   // byte bk of each word
      const uint4 ra = lds128(cb);
      c2w0 = prmt(prmt(ra.x, ra.y, sel), prmt(ra.z, ra.w, sel), 0x5410u);
      if constexpr (Cfg::kLaneRows == 2) {
        const uint4 rb8 = lds128(cb + 32u * 16u);
        c2w1 = prmt(prmt(rb8.x, rb8.y, sel), prmt(rb8.z, rb8.w, sel), 0x5410u);
      }
    }

    uint2 cw[RG][2];
#pragma unroll
    for (int rg = 0; rg < RG; ++rg)
#pragma unroll
      for (int h = 0; h < 2; ++h) cw[rg][h] = lds64(sb + code_off + static_cast<uint32_t>(16 * rg + 8 * h) * 128u);
    uint4 xv[TG][2];
#pragma unroll
    for (int t = 0; t < TG; ++t) {
      xv[t][0] = lds128(sb + x_off + static_cast<uint32_t>(8 * t) * 128u + x_c0);
      xv[t][1] = lds128(sb + x_off + static_cast<uint32_t>(8 * t) * 128u + x_c1);
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&empty[st]);
      // this warp's turn: refill the stage of item i - 1 (released by every
      // warp one item ago) with item i - 1 + S
      if (i > 0 && (i & (kFtWarps - 1)) == warp && i - 1 + S < n_items &&
          mbar_wait(&empty[pst], pph, abort_flag, DEV_WAIT_TIMEOUT_DEQUANT))
        issue_item(i - 1 + S, pst);
    }
    pst = st;
    pph = ph;
    if (++st == S) {
      st = 0;
      ph ^= 1u;
    }

    float sm0 = 0.0f, sm1 = 0.0f;
    if constexpr (CM != 0) {
      // s^ = RN(RN(c2 / c1) + mean) for this lane's two rows; the quotient
      // through the reciprocal and one residual step (exact for c1 in
      // [2^-60, 2^60], else the IEEE division)
      const int32_t blk = 4 * kc + bk;
      if (blk >= nxt) refresh(blk);
      const int sh = 8 * (kc & 3);
      auto numer = [&](uint32_t word) -> float {
        return c2_numerator(CM, static_cast<int>(static_cast<int8_t>(static_cast<uint8_t>(word >> sh))));
      };
      const float w0 = numer(c2w0), w1 = numer(c2w1);
      const float y0 = __fmul_rn(w0, rw[0].rc), y1 = __fmul_rn(w1, rw[1].rc);
      float q0 = __fmaf_rn(__fmaf_rn(-rw[0].c1, y0, w0), rw[0].rc, y0);
      float q1 = __fmaf_rn(__fmaf_rn(-rw[1].c1, y1, w1), rw[1].rc, y1);
      if (!(rw[0].fast && rw[1].fast)) {
        if (!rw[0].fast) q0 = __fdiv_rn(w0, rw[0].c1);
        if (!rw[1].fast) q1 = __fdiv_rn(w1, rw[1].c1);
      }
      // blocks past the row's end (ragged K) contribute nothing; keep their scale finite
      const bool bv = blk < p.kpb;
      sm0 = bv ? __fadd_rn(q0, mean) : 0.0f;
      sm1 = bv ? __fadd_rn(q1, mean) : 0.0f;
    } else {
      const int32_t blk = 4 * kc + bk;
      const bool bv = blk < p.kpb;
      if (dq) {
        const uint32_t c2p = c2_tma ? (((c2w0 >> (8 * (kc & 3))) & 0xFFu) | (((c2w1 >> (8 * (kc & 3))) & 0xFFu) << 8))
                                    : cur_c2;
        if (bv && rw[0].valid) sm0 = row_scale(rw[0], blk, static_cast<int>(static_cast<int8_t>(c2p & 0xFFu)));
        if (bv && rw[1].valid) sm1 = row_scale(rw[1], blk, static_cast<int>(static_cast<int8_t>(c2p >> 8)));
      } else {
        sm0 = bv && rw[0].valid ? cur_ab0 : 0.0f;
        sm1 = bv && rw[1].valid ? cur_ab1 : 0.0f;
      }
    }
    // The row groups go one after another, so only one row group's block sums
    // are live.  MMA step j takes this lane's weights 4j .. 4j+3: code bytes 2j
    // and 2j + 1, i.e. bytes 2 (j & 1) and 2 (j & 1) + 1 of word j >> 1; the
    // byte permute puts the code byte into bits 8-15 of the lane's table
    // address.  Row group rg's scales: weight rows 16 rg + pg and + 8 of the
    // row set, computed by lanes (16 rg + pg) mod 32 and + 8 (s^ of rows 0..31
    // in sm0, of rows 32..63 in sm1).
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) {
      float tmq[TG][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sa = 0x7604u | ((2u * (j & 1)) << 4);
        const uint32_t sb = 0x7604u | ((2u * (j & 1) + 1u) << 4);
        const uint32_t w0 = (j < 2) ? cw[rg][0].x : cw[rg][0].y;
        const uint32_t w1 = (j < 2) ? cw[rg][1].x : cw[rg][1].y;
        const uint32_t a0 = lds32_const(prmt(w0, lanebase, sa));
        const uint32_t a2 = lds32_const(prmt(w0, lanebase, sb));
        const uint32_t a1 = lds32_const(prmt(w1, lanebase, sa));
        const uint32_t a3 = lds32_const(prmt(w1, lanebase, sb));
#pragma unroll
        for (int t = 0; t < TG; ++t) {
          const uint4 xq = xv[t][j >> 1];
          const uint32_t b0 = (j & 1) ? xq.z : xq.x;
          const uint32_t b1 = (j & 1) ? xq.w : xq.y;
          if (j == 0)
            mma16816_first(tmq[t], a0, a1, a2, a3, b0, b1);
          else
            mma16816(tmq[t], a0, a1, a2, a3, b0, b1);
        }
      }
      const float smr = rg < 2 ? sm0 : sm1;
      const float s0 = __shfl_sync(0xffffffffu, smr, 16 * (rg & 1) + pg);
      const float s1 = __shfl_sync(0xffffffffu, smr, 16 * (rg & 1) + 8 + pg);
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        acc[rg][t][0] = fmaf(tmq[t][0], s0, acc[rg][t][0]);
        acc[rg][t][1] = fmaf(tmq[t][1], s0, acc[rg][t][1]);
        acc[rg][t][2] = fmaf(tmq[t][2], s1, acc[rg][t][2]);
        acc[rg][t][3] = fmaf(tmq[t][3], s1, acc[rg][t][3]);
      }
    }
    // leaving the row block (the next item starts another one, or the range ends)
    if (++kc == p.KC || i + 1 == n_items) {
      leave_block(rb);
      kc = 0;
      ++rb;
      set_rows(rb);
    }
  }
  __syncthreads();   // the flushes' reads of the scratch slots are done
  if (static_cast<int>(blockIdx.x) < p.tprod)
    ft_down_part<NTOK == 32 ? 2 : 1>(p, blockIdx.x, reinterpret_cast<float4*>(scratch), warp, lane);
  if (threadIdx.x == 0 && *abort_flag) {
    // let the copies still in flight land before the CTA exits
    for (int sj = 0; sj < S; ++sj) {
      const int j = last_item[sj];
      if (j < 0) continue;
      const uint32_t a = smem_u32(&full[sj]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, (j / S) & 1) && globaltimer_ns() - t0 < 100000000ull) {
      }
    }
  }
}

// ============================================================================
// Host side
// ============================================================================
namespace {

struct FtPlan {
  int ntok, KC, RB, items, G, segmax, tprod;
  size_t part_bytes, tpart_bytes;
};

FtPlan ft_plan(int64_t M, int64_t d, int64_t k, int rp) {
  FtPlan f{};
  f.ntok = M <= 8 ? 8 : M <= 16 ? 16 : 32;
  const int rows = ft_rows(f.ntok);
  f.KC = static_cast<int>(ceil_div(k, kFtK));
  f.RB = static_cast<int>(ceil_div(d, rows));
  f.items = f.KC * f.RB;
  f.G = f.items < 148 ? f.items : 148;
  const int per = static_cast<int>(ceil_div(f.items, f.G));
  f.segmax = static_cast<int>(ceil_div(per, f.KC)) + 1;
  f.part_bytes = static_cast<size_t>(f.G) * f.segmax * f.ntok * rows * 4;
  f.tprod = f.G < kFtTProd ? f.G : kFtTProd;
  f.tpart_bytes = static_cast<size_t>(f.tprod) * kFtMaxTok * rp * 4;
  return f;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// X (M x k bf16) as a 3-D tensor (64 columns, M rows, k / 64 chunks) in boxes
// of 64 columns x ntok rows x 4 chunks: one item's 256 columns in one copy,
// stored chunk by chunk (rows >= M read as zero)
bool map_x(CUtensorMap* m, const uint16_t* X, int64_t M, int64_t k, int ntok) {
  void* fp = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fp == nullptr)
    return false;
  cuuint64_t dims[3] = {64u, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(k / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(k) * 2, 128u};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(ntok), 4u};
  cuuint32_t estr[3] = {1, 1, 1};
  return reinterpret_cast<EncodeTiledFn>(fp)(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(X), dims,
                                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// c2 (d x kpb int8) in boxes of 16 blocks x `rows` rows
bool map_c2(CUtensorMap* m, const int8_t* c2, int64_t kpb, int64_t d, int rows) {
  void* fp = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fp == nullptr)
    return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kpb), static_cast<cuuint64_t>(d)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kpb)};
  cuuint32_t box[2] = {16u, static_cast<cuuint32_t>(rows)};
  cuuint32_t estr[2] = {1, 1};
  return reinterpret_cast<EncodeTiledFn>(fp)(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(c2), dims,
                                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// packed codes (d rows of k / 2 bytes) in boxes of 128 bytes (256 weights) x
// `rows` rows, 128-byte swizzle
bool map_codes(CUtensorMap* m, const uint8_t* codes, int64_t d, int64_t k, int rows) {
  void* fp = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fp == nullptr)
    return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k / 2), static_cast<cuuint64_t>(d)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k / 2)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(rows)};
  cuuint32_t estr[2] = {1, 1};
  return reinterpret_cast<EncodeTiledFn>(fp)(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims,
                                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fewtok_eligible(int64_t M, int64_t d, int64_t k) {
  // block indices of every row of every row block (rows past d included) fit in 31 bits
  return M >= 1 && M <= kFtMaxTok && d >= 1 && k >= 64 && k % 64 == 0 &&
         ceil_div(d, 256) * 256 * (k / 64) < (int64_t{1} << 31);
}

size_t fewtok_workspace_bytes(int64_t M, int64_t d, int64_t k, int rp) {
  const FtPlan f = ft_plan(M, d, k, rp);
  return align_up(f.part_bytes, 256) + align_up(f.tpart_bytes, 256);
}

template <int NTOK>
static int ft_launch(const LinearArgs& a, const FtPlan& f, const CUtensorMap& tm256, uint16_t* T, float* part,
                     float* tpart, cudaStream_t st, const char** why, const uint32_t* keep) {
  constexpr int R = FtCfg<NTOK>::kRows;
  CUtensorMap tx, tc2, tm128;
  if (!map_x(&tx, a.X, a.M, a.k, NTOK)) {
    *why = "tensor map encoding failed (few-token X)";
    return QLORA_ERR_CUDA;
  }
  // the caller's code map has 256-row boxes; 128-row items need their own
  if (R != 256 && !map_codes(&tm128, a.q->codes, a.d, a.k, R)) {
    *why = "tensor map encoding failed (few-token codes)";
    return QLORA_ERR_CUDA;
  }
  const CUtensorMap& tm = R == 256 ? tm256 : tm128;
  // c2 through TMA when its rows are 16-byte multiples and its base is 16-byte aligned
  const int64_t kpb = a.k / 64;
  const bool c2_tma = a.q->double_quant && kpb % 16 == 0 && (reinterpret_cast<uintptr_t>(a.q->c2) & 15u) == 0 &&
                      map_c2(&tc2, a.q->c2, kpb, a.d, R);
  if (!c2_tma) tc2 = tx;   // unused
  // Int8 or E4M3 c2 through TMA take the kernels without per-item mode branches
  auto kern = !c2_tma ? k_qlora_fewtok<NTOK, 0> : a.q->double_quant == 2 ? k_qlora_fewtok<NTOK, 2>
                                                                         : k_qlora_fewtok<NTOK, 1>;
  if (set_smem(kern, kFtSmemBytes) != cudaSuccess) {
    *why = "smem attribute (few-token)";
    return QLORA_ERR_CUDA;
  }
  FtParams p{};
  p.M = a.M;
  p.d = a.d;
  p.k = a.k;
  p.kpb = static_cast<int32_t>(a.k / 64);
  p.r = a.r_group > 0 ? a.r_group : a.r;
  p.rp = a.rp;
  p.rA = a.r;
  p.X = a.X;
  p.A = a.A;
  p.keep = keep;
  p.s_down = (keep && a.drop) ? a.s * a.drop->dscale : a.s;
  p.tpart = tpart;
  p.tprod = f.tprod;
  p.sc.dq = a.q->double_quant;
  p.sc.ngrp = a.ngrp;
  for (int i = 0; i < 3; ++i) p.sc.gstart[i] = a.gstart[i];
  p.sc.absmax = a.q->absmax;
  p.sc.c2 = a.q->c2;
  p.sc.c1 = a.q->c1;
  p.sc.mean = a.q->mean;
  p.B = a.B;
  p.T = T;
  p.Y = a.Y;
  p.partial = part;
  p.items = f.items;
  p.KC = f.KC;
  p.G = f.G;
  p.segmax = f.segmax;
  p.c2_tma = c2_tma ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(f.G));
  cfg.blockDim = dim3(kFtThreads);
  cfg.dynamicSmemBytes = kFtSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  {
    ProfScope ps_(QLORA_KC_FWD_GEMM, st);
    e = cudaLaunchKernelEx(&cfg, kern, tm, tx, tc2, p);
  }
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    *why = "few-token forward launch";
    return QLORA_ERR_CUDA;
  }
  cfg.gridDim = dim3(static_cast<unsigned>(f.RB));
  cfg.blockDim = dim3(static_cast<unsigned>(R / 16 * 32));   // one warp per 16 rows of the row block
  cfg.dynamicSmemBytes = 0;
  {
    ProfScope ps_(QLORA_KC_AUX, st);
    e = cudaLaunchKernelEx(&cfg, k_fewtok_finish<NTOK>, p);
  }
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    *why = "few-token finish launch";
    return QLORA_ERR_CUDA;
  }
  return 0;
}

int launch_fewtok_fwd(const LinearArgs& a, uint16_t* T, void* ws, const CUtensorMap* tm_codes, cudaStream_t st,
                      const char** why, const uint32_t* keep) {
  const FtPlan f = ft_plan(a.M, a.d, a.k, a.rp);
  char* w = static_cast<char*>(ws);
  float* part = reinterpret_cast<float*>(w);
  float* tpart = reinterpret_cast<float*>(w + align_up(f.part_bytes, 256));
  return f.ntok == 8    ? ft_launch<8>(a, f, *tm_codes, T, part, tpart, st, why, keep)
         : f.ntok == 16 ? ft_launch<16>(a, f, *tm_codes, T, part, tpart, st, why, keep)
                        : ft_launch<32>(a, f, *tm_codes, T, part, tpart, st, why, keep);
}

}  // namespace qlora
