// qlora_fewtok.cu -- the QLoRA forward for a few tokens (M <= 16).
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora), "Double quantization
// and double dequantization": Y = X doubleDequant(c1, c2, W_NF4)^T + X L1 L2,
// with the LoRA term written as (alpha/r) (X A^T) B^T ("How does alpha/r
// control adapter strength?").
//
// With a handful of tokens each 4-bit weight takes part in at most 16
// products, so the layer is bound by streaming the packed codes from HBM
// (half a byte per weight) and by the work of expanding them.  This path keeps
// the expanded weights in registers:
//
//   * TMA streams code tiles of 256 weight rows x 256 columns (32 KB) through a
//     ring in shared memory, issued by one lane of warp 0 a few items ahead of
//     the 16 warps that consume them; one CTA per SM and an even static split
//     of the (row block, K chunk) items over the CTAs, so every SM streams the
//     same number of bytes.
//   * A code byte (two weights) is expanded with one shared-memory lookup: a
//     256-entry table holds the bf16 pair (C[low nibble], C[high nibble]).  It
//     is replicated per lane (no bank conflicts) with 256 bytes per entry at a
//     64 KB-aligned base, so one byte permute forms each lookup address.
//   * Products run on mma.sync m16n8k16 (bf16 operands, fp32 accumulation):
//     the weights are the register-resident A operand and 8 tokens the N side.
//     Inside a 64-weight block the K order is permuted so that each lane's own
//     code bytes fill its fragment slots; X is read with the same permutation.
//   * The codebook enters the products unscaled; each block's partial sum is
//     multiplied by its scale s^ in fp32.  C[q] in bf16 times s^ carries the
//     same bound, 2^-9 relative, as the bf16 weight BF16(C[q] s^) that the
//     dequantisation produces.
//   * Partial sums of a row block that several CTAs share are added, in CTA
//     order, by the CTA that finishes the block last (one ticket per row
//     block).  It also adds the LoRA term T_s B^T (mma.sync) and writes Y.
//
// T_s = BF16(s X A^T) comes from k_lora_down_fewtok, a cluster kernel launched
// just before; the main kernel is its programmatic dependent, streams weights
// while it runs, and waits for it (griddepcontrol.wait) only before the
// tickets.  The down kernel also clears the tickets.
#include <cstdio>

#include "nf4_scale.cuh"
#include "nf4_table.h"
#include "qlora_device.cuh"
#include "qlora_internal.h"

namespace qlora {

namespace {

constexpr int kFtWarps = 16;                                // 4 per SM sub-partition: up to 128 registers
constexpr int kFtThreads = kFtWarps * 32;
constexpr int kFtRows = 256;                                // weight rows per item
constexpr int kFtK = 256;                                   // weights per row per item
constexpr uint32_t kFtStageBytes = kFtRows * kFtK / 2;      // 32 KB of codes
constexpr int kFtMaxStages = 4;
constexpr uint32_t kFtTableBytes = 65536;
constexpr uint32_t kFtSmemBytes = 227u * 1024u;             // the whole window; placed in the kernel
constexpr int kFtCluster = 8;                               // CTAs of one down-projection cluster

struct FtParams {
  int64_t M, d, k;
  int32_t kpb;          // NF4 blocks per weight row
  int32_t r, rp;
  ScaleSrc sc;
  const uint16_t* X;    // M x k
  const uint16_t* B;    // d x r
  const uint16_t* T;    // M x rp, T_s (written by the down kernel)
  uint16_t* Y;          // M x d
  float* partial;       // [G][segmax][NTOK][256]
  unsigned* tickets;    // [RB]
  int32_t items, KC, G, segmax;
};

// Shared-memory placement.  The lookup table needs a 64 KB-aligned base; the
// ring stages (1 KB-aligned for the 128-byte swizzle), the barriers and the
// reduction scratch fill the space before and after it.
struct FtLayout {
  uint32_t table, misc, scratch;
  uint32_t stage0, stage1, stage2, stage3;
  int nst;
  bool ok;
};

template <int TG>
__device__ __forceinline__ FtLayout ft_layout(uint32_t raw) {
  constexpr uint32_t kMisc = 128;
  constexpr uint32_t kScratch = 4u * 32u * 16u * TG * 4u;     // [row set][lane][16 TG floats]
  FtLayout L{};
  const uint32_t end = raw + kFtSmemBytes;
  L.table = (raw + 65535u) & ~65535u;
  L.ok = L.table + kFtTableBytes <= end;
  uint32_t a0 = raw, a1 = L.table, b0 = L.table + kFtTableBytes, b1 = end;
  auto take = [&](uint32_t bytes, uint32_t align, uint32_t& out) -> bool {
    uint32_t x = (a0 + align - 1u) & ~(align - 1u);
    if (x + bytes <= a1) {
      out = x;
      a0 = x + bytes;
      return true;
    }
    x = (b0 + align - 1u) & ~(align - 1u);
    if (x + bytes <= b1) {
      out = x;
      b0 = x + bytes;
      return true;
    }
    return false;
  };
  L.ok = L.ok && take(kMisc + kScratch, 16u, L.misc);
  L.scratch = L.misc + kMisc;
  uint32_t s[kFtMaxStages] = {0, 0, 0, 0};
  L.nst = 0;
#pragma unroll
  for (int i = 0; i < kFtMaxStages; ++i)
    if (take(kFtStageBytes, 1024u, s[i])) ++L.nst;
  L.stage0 = s[0];
  L.stage1 = s[1];
  L.stage2 = s[2];
  L.stage3 = s[3];
  L.ok = L.ok && L.nst >= 2;
  return L;
}

__device__ __forceinline__ uint32_t ft_stage(const FtLayout& L, int st) {
  return st == 0 ? L.stage0 : (st == 1 ? L.stage1 : (st == 2 ? L.stage2 : L.stage3));
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
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

// D += A B: 16 x 8 x 16, bf16 inputs, fp32 accumulators (register fragments).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}


__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(const void* local, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The CTA whose item range holds item i (ranges: [c I / G, (c+1) I / G)).
__device__ __forceinline__ int cta_of_item(int64_t i, int items, int G) {
  return static_cast<int>(((i + 1) * G + items - 1) / items) - 1;
}
__device__ __forceinline__ int first_item(int c, int items, int G) {
  return static_cast<int>(static_cast<int64_t>(c) * items / G);
}

}  // namespace

// ============================================================================
// T_s = BF16(s X A^T) for M <= NTOK tokens.  One cluster of 8 CTAs per group
// of 8 ranks: CTA q of the cluster sums over the q-th eighth of K (warp w =
// rank 8 g + w, lanes strided over 8-column chunks), and CTA 0 adds the eight
// partial sums in order through distributed shared memory.
// ============================================================================
template <int NTOK>
__global__ void __cluster_dims__(kFtCluster, 1, 1) __launch_bounds__(256)
    k_lora_down_fewtok(const uint16_t* __restrict__ X, const uint16_t* __restrict__ A, int M, int64_t k, int r,
                       int rp, float s, uint16_t* __restrict__ T, unsigned* __restrict__ tickets, int n_tickets) {
  griddep_launch_dependents();
  __shared__ float part[8][NTOK];
  const uint32_t q = cluster_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = static_cast<int>(blockIdx.x / kFtCluster) * 8 + warp;
  const int64_t nch = k >> 3;
  const int64_t c0 = nch * q / kFtCluster, c1 = nch * (q + 1) / kFtCluster;
  float acc[NTOK];
#pragma unroll
  for (int m = 0; m < NTOK; ++m) acc[m] = 0.0f;
  if (j < r) {
    for (int64_t ch = c0 + lane; ch < c1; ch += 32) {
      const uint4 av = ldg_nc_v4(A + static_cast<int64_t>(j) * k + ch * 8);
      const float a[8] = {bf16_lo(av.x), bf16_hi(av.x), bf16_lo(av.y), bf16_hi(av.y),
                          bf16_lo(av.z), bf16_hi(av.z), bf16_lo(av.w), bf16_hi(av.w)};
#pragma unroll
      for (int m = 0; m < NTOK; ++m) {
        if (m < M) {
          const uint4 xv = ldg_nc_v4(X + static_cast<int64_t>(m) * k + ch * 8);
          float v = acc[m];
          v = fmaf(bf16_lo(xv.x), a[0], v);
          v = fmaf(bf16_hi(xv.x), a[1], v);
          v = fmaf(bf16_lo(xv.y), a[2], v);
          v = fmaf(bf16_hi(xv.y), a[3], v);
          v = fmaf(bf16_lo(xv.z), a[4], v);
          v = fmaf(bf16_hi(xv.z), a[5], v);
          v = fmaf(bf16_lo(xv.w), a[6], v);
          v = fmaf(bf16_hi(xv.w), a[7], v);
          acc[m] = v;
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < NTOK; ++m) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
  }
  if (lane == 0) {
#pragma unroll
    for (int m = 0; m < NTOK; ++m) part[warp][m] = acc[m];
  }
  cluster_sync_all();
  if (q == 0 && threadIdx.x < 8 * NTOK) {
    const int w = threadIdx.x / NTOK, m = threadIdx.x % NTOK;
    float sum = 0.0f;
    for (uint32_t p = 0; p < kFtCluster; ++p) sum += ld_cluster_f32(&part[w][m], p);
    const int jj = static_cast<int>(blockIdx.x / kFtCluster) * 8 + w;
    if (m < M && jj < rp) {
      const uint32_t b = pack_bf16x2(jj < r ? s * sum : 0.0f, 0.0f);
      T[static_cast<int64_t>(m) * rp + jj] = static_cast<uint16_t>(b & 0xFFFFu);
    }
  }
  cluster_sync_all();   // peers keep their shared memory until CTA 0 has read it
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_tickets; i += blockDim.x) tickets[i] = 0u;
}

// ============================================================================
// Main kernel
// ============================================================================
// Combine the four warps that share a 64-row set (one per 64-column block of
// the item) and write the CTA's partial sums of the finished row block.
template <int TG>
__device__ __forceinline__ void ft_flush(float (&acc)[4][TG][4], float* scratch, float* part, int rs, int bk,
                                         int lane) {
  float* scr = scratch + (rs * 32 + lane) * 16 * TG;
  __syncthreads();
  for (int b = 1; b < 4; ++b) {
    if (bk == b) {
#pragma unroll
      for (int rg = 0; rg < 4; ++rg)
#pragma unroll
        for (int t = 0; t < TG; ++t)
          *reinterpret_cast<float4*>(scr + (rg * TG + t) * 4) =
              make_float4(acc[rg][t][0], acc[rg][t][1], acc[rg][t][2], acc[rg][t][3]);
    }
    __syncthreads();
    if (bk == 0) {
#pragma unroll
      for (int rg = 0; rg < 4; ++rg)
#pragma unroll
        for (int t = 0; t < TG; ++t) {
          const float4 v = *reinterpret_cast<const float4*>(scr + (rg * TG + t) * 4);
          acc[rg][t][0] += v.x;
          acc[rg][t][1] += v.y;
          acc[rg][t][2] += v.z;
          acc[rg][t][3] += v.w;
        }
    }
    __syncthreads();
  }
  if (bk == 0) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int rg = 0; rg < 4; ++rg)
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        const int row = 64 * rs + 16 * rg + g;
        const int tok = 8 * t + 2 * c;
        part[tok * kFtRows + row] = acc[rg][t][0];
        part[(tok + 1) * kFtRows + row] = acc[rg][t][1];
        part[tok * kFtRows + row + 8] = acc[rg][t][2];
        part[(tok + 1) * kFtRows + row + 8] = acc[rg][t][3];
      }
  }
#pragma unroll
  for (int rg = 0; rg < 4; ++rg)
#pragma unroll
    for (int t = 0; t < TG; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[rg][t][e] = 0.0f;
}

// Last CTA of row block rb: Y = BF16(sum of the CTAs' partial sums + T_s B^T).
// Warp w takes rows 16 w .. 16 w + 15 of the block.
template <int NTOK>
__device__ __forceinline__ void ft_finish(const FtParams& p, int rb, int warp, int lane) {
  constexpr int TG = NTOK / 8;
  const int g = lane >> 2, c = lane & 3;
  const int64_t na = static_cast<int64_t>(rb) * kFtRows + 16 * warp + g, nb = na + 8;
  const int ra = 16 * warp + g;
  float v[TG][4];
#pragma unroll
  for (int t = 0; t < TG; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) v[t][e] = 0.0f;
  const int64_t i0 = static_cast<int64_t>(rb) * p.KC;
  const int cf = cta_of_item(i0, p.items, p.G), cl = cta_of_item(i0 + p.KC - 1, p.items, p.G);
  for (int cc = cf; cc <= cl; ++cc) {
    const int seg = rb - first_item(cc, p.items, p.G) / p.KC;
    const float* part = p.partial + (static_cast<int64_t>(cc) * p.segmax + seg) * NTOK * kFtRows;
#pragma unroll
    for (int t = 0; t < TG; ++t) {
      const int tok = 8 * t + 2 * c;
      v[t][0] += part[tok * kFtRows + ra];
      v[t][1] += part[(tok + 1) * kFtRows + ra];
      v[t][2] += part[tok * kFtRows + ra + 8];
      v[t][3] += part[(tok + 1) * kFtRows + ra + 8];
    }
  }
  // LoRA term: rows of B are the A operand, T_s^T the B operand.
  auto bpair = [&](int64_t n, int j) -> uint32_t {
    uint32_t lo = 0, hi = 0;
    if (n < p.d) {
      if (j < p.r) lo = p.B[n * p.r + j];
      if (j + 1 < p.r) hi = p.B[n * p.r + j + 1];
    }
    return lo | (hi << 16);
  };
  for (int ks = 0; ks < p.rp / 16; ++ks) {
    const int j0 = 16 * ks + 2 * c;
    if (16 * ks >= p.r) break;
    const uint32_t a0 = bpair(na, j0), a1 = bpair(nb, j0), a2 = bpair(na, j0 + 8), a3 = bpair(nb, j0 + 8);
#pragma unroll
    for (int t = 0; t < TG; ++t) {
      const int tok = 8 * t + g;
      uint32_t b0 = 0, b1 = 0;
      if (tok < p.M) {
        const uint32_t* trow = reinterpret_cast<const uint32_t*>(p.T + static_cast<int64_t>(tok) * p.rp);
        b0 = trow[j0 >> 1];
        b1 = trow[(j0 + 8) >> 1];
      }
      mma16816(v[t], a0, a1, a2, a3, b0, b1);
    }
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

template <int NTOK>
__global__ void __launch_bounds__(kFtThreads, 1)
    k_qlora_fewtok(const __grid_constant__ CUtensorMap tm_codes, const FtParams p) {
  constexpr int TG = NTOK / 8;
  extern __shared__ __align__(1024) uint8_t ft_smem[];
  const uint32_t raw = smem_u32(ft_smem);
  const FtLayout L = ft_layout<TG>(raw);
  if (!L.ok) {
    if (threadIdx.x == 0) report(DEV_SMEM_LAYOUT);
    return;
  }
  auto gptr = [&](uint32_t a) { return ft_smem + (a - raw); };
  uint64_t* full = reinterpret_cast<uint64_t*>(gptr(L.misc));
  uint64_t* empty = full + kFtMaxStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 2 * kFtMaxStages);
  volatile int* last_flag = abort_flag + 1;
  const int S = L.nst;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it0 = first_item(blockIdx.x, p.items, p.G);
  const int it1 = first_item(blockIdx.x + 1, p.items, p.G);
  const int n_items = it1 - it0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kFtWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_codes);
  }
  {
    // code-byte table: entry e = (C[e & 15], C[e >> 4]) in bf16, one copy per lane
    constexpr uint32_t kCB[16] = {QLORA_NF4_TABLE_BITS};
    for (int i = threadIdx.x; i < 256 * 32; i += kFtWarps * 32) {
      const int e = i >> 5;
      const uint32_t v = pack_bf16x2(__uint_as_float(kCB[e & 15]), __uint_as_float(kCB[e >> 4]));
      sts32(L.table + static_cast<uint32_t>(e) * 256u + static_cast<uint32_t>(i & 31) * 4u, v);
    }
  }
  __syncthreads();

  {
    // ------------------------------------------------------------ consumers
    // warp = (row set rs: 64 rows) x (block bk: 64 columns of the item)
    const int rs = warp & 3, bk = warp >> 2;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t lanebase = L.table + static_cast<uint32_t>(lane) * 4u;
    // this lane's 8 code bytes of row 64 rs + g in the 128-byte-swizzled tile
    const uint32_t lane_off = static_cast<uint32_t>(64 * rs + g) * 128u +
                              16u * static_cast<uint32_t>((2 * bk + (c >> 1)) ^ g) + 8u * static_cast<uint32_t>(c & 1);
    float* scratch = reinterpret_cast<float*>(gptr(L.scratch));
    float acc[4][TG][4];
#pragma unroll
    for (int rg = 0; rg < 4; ++rg)
#pragma unroll
      for (int t = 0; t < TG; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[rg][t][e] = 0.0f;
    const float mean = p.sc.dq ? __ldg(p.sc.mean) : 0.0f;
    ScaleRecip rec0, rec1;

    // inputs of item gi that do not come through the ring: the block scales of
    // this lane's two rows (16 c + g and +8 of the row set) and the lane's 16
    // columns of X for each token group
    auto fetch = [&](int rb, int kc, ScaleRaw& r0, ScaleRaw& r1, bool& v0, bool& v1, uint4 (&xv)[TG][2]) {
      const int64_t blk = 4ll * kc + bk;
      const int64_t n0 = static_cast<int64_t>(rb) * kFtRows + 64 * rs + 16 * c + g;
      const bool bv = blk < p.kpb;
      v0 = bv && (n0 < p.d);
      v1 = bv && (n0 + 8 < p.d);
      if (v0) r0 = scale_fetch(p.sc, n0 * p.kpb + blk);
      if (v1) r1 = scale_fetch(p.sc, (n0 + 8) * p.kpb + blk);
      const int64_t kb = 64ll * blk + 16 * c;
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        const int tok = 8 * t + g;
        if (bv && tok < p.M) {
          const uint16_t* src = p.X + static_cast<int64_t>(tok) * p.k + kb;
          xv[t][0] = ldg_nc_v4(src);
          xv[t][1] = ldg_nc_v4(src + 8);
        } else {
          xv[t][0] = make_uint4(0, 0, 0, 0);
          xv[t][1] = make_uint4(0, 0, 0, 0);
        }
      }
    };

    // lane 0 of warp 0 keeps S - 1 items in flight ahead of its own position
    const bool producer = (threadIdx.x == 0);
    int pst = 0, issued = 0;
    uint32_t pph = 0;
    auto issue = [&]() {
      if (!mbar_wait(&empty[pst], pph ^ 1u, abort_flag, DEV_WAIT_TIMEOUT_DEQUANT)) return;
      const int gi = it0 + issued, rb = gi / p.KC, kc = gi - rb * p.KC;
      mbar_arrive_expect_tx(&full[pst], kFtStageBytes);
      tma_load_2d(gptr(ft_stage(L, pst)), &tm_codes, &full[pst], kc * (kFtK / 2), rb * kFtRows);
      ++issued;
      if (++pst == S) {
        pst = 0;
        pph ^= 1u;
      }
    };
    if (producer)
      while (issued < n_items && issued < S - 1 && !*abort_flag) issue();

    int st = 0, cur_rb = -1, seg = -1;
    uint32_t ph = 0;
    ScaleRaw nr0{}, nr1{};
    bool nv0 = false, nv1 = false;
    uint4 nx[TG][2];
    // (row block, K chunk) of the current item
    int crb = it0 / p.KC, ckc = it0 - crb * p.KC;
    if (n_items > 0) fetch(crb, ckc, nr0, nr1, nv0, nv1, nx);
    for (int i = 0; i < n_items; ++i) {
      const int rb = crb;
      const bool wrap = (ckc + 1 == p.KC);
      const int nrb = wrap ? crb + 1 : crb, nkc = wrap ? 0 : ckc + 1;   // the next item
      crb = nrb;
      ckc = nkc;
      if (rb != cur_rb) {
        if (cur_rb >= 0)
          ft_flush<TG>(acc, scratch, p.partial + (static_cast<int64_t>(blockIdx.x) * p.segmax + seg) * NTOK * kFtRows,
                       rs, bk, lane);
        cur_rb = rb;
        ++seg;
      }
      const ScaleRaw r0 = nr0, r1 = nr1;
      const bool v0 = nv0, v1 = nv1;
      uint4 xv[TG][2];
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        xv[t][0] = nx[t][0];
        xv[t][1] = nx[t][1];
      }
      if (i + 1 < n_items) fetch(nrb, nkc, nr0, nr1, nv0, nv1, nx);

      mbar_wait(&full[st], ph, abort_flag, DEV_WAIT_TIMEOUT_TMA);
      const uint32_t sbase = ft_stage(L, st) + lane_off;
      uint2 cw[4][2];
#pragma unroll
      for (int rg = 0; rg < 4; ++rg)
#pragma unroll
        for (int h = 0; h < 2; ++h) cw[rg][h] = lds64(sbase + static_cast<uint32_t>(16 * rg + 8 * h) * 128u);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == S) {
        st = 0;
        ph ^= 1u;
      }
      // refill the stage every warp released one item ago
      if (producer && issued < n_items && !*abort_flag) issue();

      const float sm0 = v0 ? scale_value(p.sc.dq, mean, r0, rec0) : 0.0f;
      const float sm1 = v1 ? scale_value(p.sc.dq, mean, r1, rec1) : 0.0f;
      // four independent accumulation chains (one per 16-row group), stepped
      // together so consecutive tensor-core ops never wait on each other
      float tmp[4][TG][4];
#pragma unroll
      for (int rg = 0; rg < 4; ++rg)
#pragma unroll
        for (int t = 0; t < TG; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) tmp[rg][t][e] = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // MMA step j takes this lane's weights 4j .. 4j+3 (bytes 2j, 2j+1)
        const uint32_t sa = 0x7604u | ((2u * (j & 1)) << 4);
        const uint32_t sb = 0x7604u | ((2u * (j & 1) + 1u) << 4);
#pragma unroll
        for (int rg = 0; rg < 4; ++rg) {
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
            mma16816(tmp[rg][t], a0, a1, a2, a3, b0, b1);
          }
        }
      }
#pragma unroll
      for (int rg = 0; rg < 4; ++rg) {
        const float s0 = __shfl_sync(0xffffffffu, sm0, 4 * g + rg);
        const float s1 = __shfl_sync(0xffffffffu, sm1, 4 * g + rg);
#pragma unroll
        for (int t = 0; t < TG; ++t) {
          acc[rg][t][0] = fmaf(tmp[rg][t][0], s0, acc[rg][t][0]);
          acc[rg][t][1] = fmaf(tmp[rg][t][1], s0, acc[rg][t][1]);
          acc[rg][t][2] = fmaf(tmp[rg][t][2], s1, acc[rg][t][2]);
          acc[rg][t][3] = fmaf(tmp[rg][t][3], s1, acc[rg][t][3]);
        }
      }
    }
    if (cur_rb >= 0)
      ft_flush<TG>(acc, scratch, p.partial + (static_cast<int64_t>(blockIdx.x) * p.segmax + seg) * NTOK * kFtRows,
                   rs, bk, lane);
    if (producer && *abort_flag) {
      // let the copies still in flight land before the CTA exits
      const int first = issued > S ? issued - S : 0;
      for (int l = first; l < issued; ++l) {
        const uint32_t a = smem_u32(&full[l % S]);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, (l / S) & 1) && globaltimer_ns() - t0 < 100000000ull) {
        }
      }
    }
  }

  // ------------------------------------------------------------ row-block tickets
  __syncthreads();
  griddep_wait();   // T_s and the cleared tickets of the down kernel
  if (*abort_flag || n_items == 0) return;
  const int rb_first = it0 / p.KC, rb_last = (it1 - 1) / p.KC;
  for (int rb = rb_first; rb <= rb_last; ++rb) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const int64_t i0 = static_cast<int64_t>(rb) * p.KC;
      const int ncontrib = cta_of_item(i0 + p.KC - 1, p.items, p.G) - cta_of_item(i0, p.items, p.G) + 1;
      const unsigned t = atomicAdd(&p.tickets[rb], 1u);
      *last_flag = (t == static_cast<unsigned>(ncontrib - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (*last_flag) {
      __threadfence();
      ft_finish<NTOK>(p, rb, warp, lane);
    }
  }
}

// ============================================================================
// Host side
// ============================================================================
namespace {

struct FtPlan {
  int ntok, KC, RB, items, G, segmax;
  size_t part_bytes, ticket_bytes;
};

FtPlan ft_plan(int64_t M, int64_t d, int64_t k) {
  FtPlan f{};
  f.ntok = M <= 8 ? 8 : 16;
  f.KC = static_cast<int>(ceil_div(k, kFtK));
  f.RB = static_cast<int>(ceil_div(d, kFtRows));
  f.items = f.KC * f.RB;
  f.G = f.items < 148 ? f.items : 148;
  const int per = static_cast<int>(ceil_div(f.items, f.G));
  f.segmax = static_cast<int>(ceil_div(per, f.KC)) + 1;
  f.part_bytes = static_cast<size_t>(f.G) * f.segmax * f.ntok * kFtRows * 4;
  f.ticket_bytes = static_cast<size_t>(f.RB) * 4;
  return f;
}

cudaError_t ft_set_smem(const void* fn) {
  static bool done[2] = {false, false};
  // one attribute per instantiation; the call is cheap but not free
  const int idx = fn == reinterpret_cast<const void*>(k_qlora_fewtok<8>) ? 0 : 1;
  if (done[idx]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kFtSmemBytes));
  if (e == cudaSuccess) done[idx] = true;
  return e;
}

}  // namespace

bool fewtok_eligible(int64_t M, int64_t d, int64_t k) {
  return M >= 1 && M <= kFewTokMax && d >= 1 && k >= 64 && k % 64 == 0;
}

size_t fewtok_workspace_bytes(int64_t M, int64_t d, int64_t k) {
  const FtPlan f = ft_plan(M, d, k);
  return align_up(f.part_bytes, 256) + align_up(f.ticket_bytes, 256);
}

template <int NTOK>
static int ft_launch(const LinearArgs& a, const FtPlan& f, const CUtensorMap& tm, uint16_t* T, float* part,
                     unsigned* tickets, cudaStream_t st, const char** why) {
  {
    ProfScope ps_(QLORA_KC_LORA_GEMM, st);
    k_lora_down_fewtok<NTOK><<<static_cast<unsigned>(kFtCluster * (a.rp / 8)), 256, 0, st>>>(
        a.X, a.A, static_cast<int>(a.M), a.k, a.r, a.rp, a.s, T, tickets, f.RB);
  }
  if (cudaGetLastError() != cudaSuccess) {
    *why = "few-token down-projection launch";
    return QLORA_ERR_CUDA;
  }
  if (ft_set_smem(reinterpret_cast<const void*>(k_qlora_fewtok<NTOK>)) != cudaSuccess) {
    *why = "smem attribute (few-token)";
    return QLORA_ERR_CUDA;
  }
  FtParams p{};
  p.M = a.M;
  p.d = a.d;
  p.k = a.k;
  p.kpb = static_cast<int32_t>(a.k / 64);
  p.r = a.r;
  p.rp = a.rp;
  p.sc.dq = a.q->double_quant;
  p.sc.absmax = a.q->absmax;
  p.sc.c2 = a.q->c2;
  p.sc.c1 = a.q->c1;
  p.sc.mean = a.q->mean;
  p.X = a.X;
  p.B = a.B;
  p.T = T;
  p.Y = a.Y;
  p.partial = part;
  p.tickets = tickets;
  p.items = f.items;
  p.KC = f.KC;
  p.G = f.G;
  p.segmax = f.segmax;
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
    e = cudaLaunchKernelEx(&cfg, k_qlora_fewtok<NTOK>, tm, p);
  }
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    *why = "few-token forward launch";
    return QLORA_ERR_CUDA;
  }
  return 0;
}

int launch_fewtok_fwd(const LinearArgs& a, uint16_t* T, void* ws, const CUtensorMap* tm_codes, cudaStream_t st,
                      const char** why) {
  const FtPlan f = ft_plan(a.M, a.d, a.k);
  char* w = static_cast<char*>(ws);
  float* part = reinterpret_cast<float*>(w);
  unsigned* tickets = reinterpret_cast<unsigned*>(w + align_up(f.part_bytes, 256));
  return f.ntok == 8 ? ft_launch<8>(a, f, *tm_codes, T, part, tickets, st, why)
                     : ft_launch<16>(a, f, *tm_codes, T, part, tickets, st, why);
}

}  // namespace qlora
