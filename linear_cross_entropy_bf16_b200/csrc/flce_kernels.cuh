// Device code of the fused linear cross-entropy forward (sm_100a).
//
// Operation: D. Ineshin, "Een gefuseerde forward-kernel voor lineaire
// cross-entropy op Apple-GPU's" (2026), section 1.  Z = H W^T; each vocab tile
// is folded into a running online log-sum-exp state (m, s) with
//   m' = max(m, m_t),  s' = s exp(m - m') + sum_j exp(z_j - m'),
// the target logit is captured from the tile that holds it, and after the last
// tile logsumexp = m + log s and loss = logsumexp - z_target.
//
// B200 design (not the page's one-dispatch-per-tile chain):
//   * flce_tc_kernel: a persistent, warp-specialised tcgen05 GEMM.  One CTA
//     per SM walks work units (128 tokens x one vocab slab of 256-column
//     tiles).  Warp 0 streams H and W K-blocks with TMA into a shared-memory
//     ring (192 KiB), warp 1 issues 128x256x16 bf16 MMAs into a
//     double-buffered fp32 TMEM accumulator, and warps 2-5 (one TMEM lane,
//     i.e. one token, per thread) fold each finished tile into (m, s) and
//     capture the target logit.  Logits never leave TMEM/registers.
//   * flce_tc2_kernel: the same on CTA pairs (cta_group::2, 256x256 tiles):
//     each CTA stages its own 128 token rows and half of the
//     W tile, the even CTA issues the pair MMAs.  Used for N > 128.
//   * In the forward both also merge (tc::fused_merge): the CTA that writes
//     the last slab state of a 128-token row block merges that block in its
//     epilogue, and the one that merges the last row block forms the mean,
//     so the whole forward is one launch.
//   * Both are templates on the stage layout (tc::StageLayout): H and W
//     blocks of two consecutive K blocks per stage for bf16 inputs; H with
//     W's hi and lo blocks for a quantised head (two products); H's and W's
//     hi and lo blocks for fp32 inputs (three products, Hhi Whi + Hhi Wlo +
//     Hlo Whi).
//   * flce_split3_kernel: for fp32 inputs, splits H and W into bf16 [hi | lo]
//     rows for the split layout (three segments for the backward's GEMMs).
//   * flce_dequant_split_kernel: expands one chunk of an affine
//     group-quantised head into bf16 [hi | lo] rows for the same kernels.
//   * flce_merge_kernel: the same merge as a kernel of its own, after the
//     contraction alone (flce_partials): combines the P slab states of each
//     token in a fixed order (the recurrence of section 1 applied to whole
//     slabs), writes lse/loss, and reduces the mean deterministically in
//     fp64; the shard kernels do the same across vocabulary shards or chunks.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"

namespace flce {

// ----------------------------------------------------------------- constants

constexpr int kTileCols = 256;   // vocab columns per tile (UMMA N, TMEM columns)
constexpr int kMaxSlabs = 512;   // partial states per token, at most

// workspace layout: [header 256 B][row-block arrival counters][partials float2[P][N]]
// [block sums double]; the host's state_layout() gives the offsets
constexpr size_t kHeaderBytes = 256;
constexpr uint32_t kWsMagic = 0x464C4345u;  // "FLCE"

// device status bits (workspace header word 0)
constexpr uint32_t kStatTarget = 1u;    // some y_i outside [0, V)
constexpr uint32_t kStatTimeout = 2u;   // a bounded wait ran out
constexpr uint32_t kStatBadWs = 4u;     // merge found a workspace not prepared by partials

struct WsHeader {
  uint32_t status;    // OR of kStat* bits for the current call
  uint32_t counter;   // merge blocks finished (last one computes the mean)
  uint32_t magic;     // kWsMagic once the partials stage has run
  int32_t slabs;      // P used by the partials stage
  int64_t N;
  int64_t V;
};
static_assert(sizeof(WsHeader) <= kHeaderBytes, "header");

constexpr float kLog2e = 1.4426950408889634f;  // log2(e): exp(x) = 2^(x log2 e)

// ----------------------------------------------------------------- targets

// Target ids, stored as int64 (the default) or int32.
struct Targets {
  const void* p;
  int32_t is32;
  __device__ __forceinline__ int64_t operator[](int64_t i) const {
    return is32 ? int64_t(static_cast<const int32_t*>(p)[i]) : static_cast<const int64_t*>(p)[i];
  }
};

// ----------------------------------------------------------------- schedule

struct Schedule {
  int32_t token_blocks;  // TB
  int32_t slabs;         // P
  int32_t slab_base;     // tiles per slab (NT / P)
  int32_t slab_rem;      // the first slab_rem slabs hold one more tile
  int32_t units;         // TB * P
  int32_t group_blocks;  // GT: token blocks per raster group
};

// Work-unit order.  Token blocks are taken in groups of GT; inside a group the
// order is slab-major (all GT token blocks of slab 0, then of slab 1, ...).
// Units handed out round-robin therefore run, at any moment, over a few
// consecutive slabs of one group: each W tile is read by GT token blocks close
// together in time, and only GT blocks of H are live in L2.
__device__ __forceinline__ void unit_coords(const Schedule& s, int u, int& slab, int& tblock,
                                            int& tile0, int& ntiles) {
  const int per_group = s.group_blocks * s.slabs;
  const int g = u / per_group;
  const int l = u - g * per_group;
  const int gt = min(s.group_blocks, s.token_blocks - g * s.group_blocks);  // last group may be short
  slab = l / gt;
  tblock = g * s.group_blocks + (l - slab * gt);
  tile0 = slab * s.slab_base + min(slab, s.slab_rem);
  ntiles = s.slab_base + (slab < s.slab_rem ? 1 : 0);
}

// Partition-aware order of the pair kernel.  The B200's L2 is two partitions,
// each caching what its own SMs read, so data that every SM reads gets about
// half of the L2.  In this order the CTA pairs on partition 0 take the first
// U0 units of the token-block-major order (token blocks [0, q) and slabs
// [0, r) of block q, U0 = q P + r) and the pairs on partition 1 the rest,
// each side slab-major over its own blocks: each partition's L2 holds only
// its own rows of H, and the two sides stream the same W tiles at the same
// time.  The split (q, r) makes U0 / U the share of the pairs on partition 0.
__host__ __device__ inline int32_t part_units(const Schedule& s, int32_t q, int32_t r, int side) {
  const int32_t u0 = q * s.slabs + r;
  return side == 0 ? u0 : s.units - u0;
}

// Slab and token block of unit k (< part_units) of partition `side`.
__host__ __device__ inline void part_unit(const Schedule& s, int32_t q, int32_t r, int side, int k,
                                          int& slab, int& tblock) {
  if (side == 0) {
    // slabs [0, r) hold blocks [0, q]; slabs [r, P) blocks [0, q)
    const int head = r * (q + 1);
    if (k < head) {
      slab = k / (q + 1);
      tblock = k - slab * (q + 1);
    } else {
      const int k2 = k - head;  // q > 0 whenever a unit lies here
      slab = r + k2 / q;
      tblock = k2 - (slab - r) * q;
    }
  } else {
    // slabs [0, r) hold blocks [q + 1, TB); slabs [r, P) blocks [q, TB)
    const int c = s.token_blocks - q - 1;
    const int head = r * c;
    if (k < head) {  // c > 0 whenever a unit lies here
      slab = k / c;
      tblock = q + 1 + (k - slab * c);
    } else {
      const int k2 = k - head;
      slab = r + k2 / (c + 1);
      tblock = q + (k2 - (slab - r) * (c + 1));
    }
  }
}

// A pair that arrived as number `arrival` on partition `side` (counted from
// 0 by the header counter) takes rank `arrival` there, unless the side
// already has its planned `pairs[side]`: then it takes the highest rank of
// the other side that no pair can reach.  With pairs[0] + pairs[1] pairs in
// all, every planned (side, rank) is taken exactly once, however the pairs
// land.
__host__ __device__ inline void part_take(const int32_t (&pairs)[2], int& side, int& rank) {
  if (rank >= pairs[side]) {
    rank = pairs[side ^ 1] - 1 - (rank - pairs[side]);
    side ^= 1;
  }
}

__host__ __device__ inline void slab_tiles(const Schedule& s, int slab, int& tile0, int& ntiles) {
  tile0 = slab * s.slab_base + (slab < s.slab_rem ? slab : s.slab_rem);
  ntiles = s.slab_base + (slab < s.slab_rem ? 1 : 0);
}

// ----------------------------------------------------------------- bounded waits

// Bounded mbarrier waits.  `flag` is the CTA's shared abort flag: once any
// role of the CTA gives up, the others stop waiting too.  `status` is the
// workspace status word in global memory.

// Wait for phase `parity` of the mbarrier at `bar`, for at most limit_ns.
// Returns false (after recording kStatTimeout and raising the CTA abort flag)
// when the limit runs out, or when another role of this CTA has aborted
// (flag == nullptr: ignore other roles, only the time limit applies).
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int* flag,
                                       uint32_t* status, uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((n & 31u) == 0) {
      if (flag != nullptr && *flag) return false;
      if (ptx::globaltimer_ns() - t0 > limit_ns) {
        if (flag != nullptr) *flag = 1;
        ptx::griddep_wait();  // after the kernel that cleared the status word
        atomicOr(status, kStatTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* flag,
                                             uint32_t* status, uint64_t limit_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, flag, status, limit_ns);
}

// z[idx] for a register array and a runtime idx in [0, 32), as a five-level
// select tree with compile-time indices (an indexed read would move the whole
// array to local memory).
__device__ __forceinline__ float pick32(const float (&z)[32], int idx) {
  float a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = (idx & 16) ? z[j + 16] : z[j];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = (idx & 8) ? a[j + 8] : a[j];
#pragma unroll
  for (int j = 0; j < 4; ++j) a[j] = (idx & 4) ? a[j + 4] : a[j];
#pragma unroll
  for (int j = 0; j < 2; ++j) a[j] = (idx & 2) ? a[j + 2] : a[j];
  return (idx & 1) ? a[1] : a[0];
}

// ----------------------------------------------------------------- epilogue

// Fold one finished accumulator tile into this thread's running state.  The
// thread owns one TMEM lane (one token); `taddr` addresses that lane at
// column 0 of the tile, `ncols` columns exist (the rest of the tile lies past
// V), and `rel` is the target's column inside the tile (any value outside
// [0, ncols) means the target is elsewhere).  Per 32-column chunk:
//   m_t = max_j z_j,  m' = max(m, m_t),
//   s'  = s * exp(m - m') + sum_j exp(z_j - m')     (the page, section 1)
// with exp(x) evaluated as 2^(x log2 e).  Must be called by all 32 lanes.
__device__ __forceinline__ void fold_tile(uint32_t taddr, int ncols, int64_t rel, float& m, float& s,
                                          float& zt, bool& got) {
#pragma unroll 1
  for (int c = 0; c < kTileCols / 32; ++c) {
    if (c * 32 >= ncols) break;  // warp-uniform: the rest of the tile is past V
    uint32_t u32[32];
    ptx::tmem_ld32_wait(taddr + uint32_t(c * 32), u32);
    float z[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) z[j] = __uint_as_float(u32[j]);
    if (ncols - c * 32 < 32) {  // ragged last tile: columns >= V do not exist
      const int lim = ncols - c * 32;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j >= lim) z[j] = -INFINITY;
    }
    // target capture: the tile holding y_i records z_{i, y_i}
    const int64_t rc = rel - c * 32;
    if (rc >= 0 && rc < 32) {
      zt = pick32(z, int(rc));
      got = true;
    }
    // m_t = max_j z_j over this chunk, tree-reduced
    float mx[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) mx[j] = fmaxf(z[j], z[j + 16]);
#pragma unroll
    for (int w2 = 8; w2 >= 1; w2 >>= 1)
#pragma unroll
      for (int j = 0; j < w2; ++j) mx[j] = fmaxf(mx[j], mx[j + w2]);
    const float m_new = fmaxf(m, mx[0]);
    const float ms = __fmul_rn(m_new, kLog2e);
    // sum_j exp(z_j - m') as 2^(z_j log2 e - m' log2 e).  The product and the
    // difference are rounded separately (no fused multiply-add), so the
    // column holding the maximum contributes exactly 2^0 = 1: s >= 1, hence
    // lse >= max_j z_j >= z_target and every loss is >= 0 (exactly 0 for V = 1).
    float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 32; ++j) e[j & 3] += ptx::ex2(__fsub_rn(__fmul_rn(z[j], kLog2e), ms));
    // s' = s exp(m - m') + sum; m = -inf on the first chunk gives exp(-inf) = 0
    s = fmaf(s, ptx::ex2((m - m_new) * kLog2e), (e[0] + e[1]) + (e[2] + e[3]));
    m = m_new;
  }
}

// ----------------------------------------------------------------- merge helpers

// The merge of one token's P slab states part[p * N] (p = 0 .. P-1), the
// recurrence of section 1 applied to whole slabs in slab order:
// m = max_p m_p, s = sum_p s_p exp(m_p - m), accumulated in fp64, with a
// running maximum over batches of 16 slabs (one pass); returns lse = m + log s (log in fp64).  Each factor
// exp(m_p - m) is evaluated as 2^((m_p - m) log2 e) on the SFU, as the
// contraction's own exponentials are: relative error about 2^-22 per term,
// and the slab holding the maximum contributes exactly s_p.  Every slab holds
// at least one real column, so m is finite.
// Loads slab states p0 .. p0 + 15 of a token (past P: empty states).
__device__ __forceinline__ void load_slab_batch(float2 (&b)[16], const float2* part, int p0, int P,
                                                int N) {
#pragma unroll
  for (int j = 0; j < 16; ++j)
    b[j] = p0 + j < P ? __ldcg(part + size_t(p0 + j) * size_t(N)) : make_float2(-INFINITY, 0.f);
}

// Folds one batch of 16 states into the running (M, S).
__device__ __forceinline__ void fold_slab_batch(const float2 (&b)[16], float& M, double& S) {
  float mb = b[0].x;
#pragma unroll
  for (int j = 1; j < 16; ++j) mb = fmaxf(mb, b[j].x);
  if (mb > M) {  // rescale the running sum (on the first batch S = 0 and 2^-inf = 0)
    S *= double(ptx::ex2(__fmul_rn(M - mb, kLog2e)));
    M = mb;
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) S += double(b[j].y * ptx::ex2(__fmul_rn(b[j].x - M, kLog2e)));
}

__device__ __forceinline__ double merge_slab_states(const float2* part, int P, int N) {
  // Batches of 16 states in three register buffers that take turns: a batch
  // is loaded two batches ahead of its fold, so that the L2 round trips
  // overlap the folds (no buffer is copied into another, which would wait
  // for the loads).  The arithmetic is batch by batch in slab order.
  float2 b0[16], b1[16], b2[16];
  load_slab_batch(b0, part, 0, P, N);
  if (P > 16) load_slab_batch(b1, part, 16, P, N);
  float M = -INFINITY;
  double S = 0.0;
  for (int p0 = 0; p0 < P; p0 += 48) {
    if (p0 + 32 < P) load_slab_batch(b2, part, p0 + 32, P, N);
    fold_slab_batch(b0, M, S);
    if (p0 + 16 >= P) break;
    if (p0 + 48 < P) load_slab_batch(b0, part, p0 + 48, P, N);
    fold_slab_batch(b1, M, S);
    if (p0 + 32 >= P) break;
    if (p0 + 64 < P) load_slab_batch(b1, part, p0 + 64, P, N);
    fold_slab_batch(b2, M, S);
  }
  return double(M) + log(S);
}

// Fixed-order sum of one value per thread over 128 threads (four warps): a
// warp shuffle tree, then the four warps in order.  `sync` is a barrier over
// the 128 threads; the result is valid in thread 0.
template <class Sync>
__device__ __forceinline__ double sum128(double v, int t, volatile double* red, Sync sync) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
  if ((t & 31) == 0) red[t >> 5] = v;
  sync();
  return ((red[0] + red[1]) + red[2]) + red[3];
}

// Row block `rb` (128 tokens, thread t holding token loss `l`) records its
// loss sum; the row block that finishes last of `nblocks` adds the block sums
// (thread t: blocks t, t + 128, ... in order, then sum128) into the mean and
// the sum, and resets the counter (a single block's sum is the total: no
// count).  The same order for any set of finishing times, so results are
// bitwise deterministic.
template <class Sync>
__device__ __forceinline__ void rowblock_finish(double l, int t, int rb, int nblocks,
                                                double* block_sums, uint32_t* counter, float* mean,
                                                float* sum, int N, volatile double* red,
                                                volatile int* flag, Sync sync) {
  const double b = sum128(l, t, red, sync);
  if (nblocks == 1) {  // the only block: its sum is the total (no count, no reload)
    if (t == 0) {
      if (mean != nullptr) *mean = float(b / double(N));
      if (sum != nullptr) *sum = float(b);
    }
    return;
  }
  if (t == 0) {
    block_sums[rb] = b;
    ptx::fence_acq_rel_gpu();  // release: this block sum before the count
    const bool last = atomicAdd(counter, 1u) == uint32_t(nblocks - 1);
    if (last) ptx::fence_acq_rel_gpu();  // acquire: every block sum, seen through the count
    *flag = last;
  }
  sync();  // the other threads read block sums after thread 0's acquire, through L2 only
  if (!*flag || (mean == nullptr && sum == nullptr)) return;
  double v = 0.0;
  for (int r = t; r < nblocks; r += 128) v += __ldcg(block_sums + r);
  const double total = sum128(v, t, red, sync);
  if (t == 0) {
    if (mean != nullptr) *mean = float(total / double(N));
    if (sum != nullptr) *sum = float(total);
    *counter = 0;
  }
}

// ----------------------------------------------------------------- tcgen05 kernel

namespace tc {

// What one pipeline stage holds (64-column K blocks of H and W, 128 B swizzle
// rows) and the products the MMA issuer forms from it into the tile's
// accumulator, each product being four 16-deep MMAs:
//   kPlain    H and W blocks of two consecutive K blocks: H W^T over 128 K
//             columns per stage (bf16 inputs).  Two products per barrier
//             round trip: with one K block per stage the tensor pipe idled
//             about 9% of its active cycles between stages, and the headline
//             forward ran 6.5% slower.
//   kSplitW   H, W_hi, W_lo of one K block: H W_hi^T + H W_lo^T (a quantised
//             head expanded to bf16 hi + lo; H is staged once for both).
//   kSplitHW  H_hi, H_lo, W_hi, W_lo of one K block: hi hi + hi lo + lo hi
//             (fp32 inputs split into bf16 hi + lo, the bf16x3 scheme; four
//             blocks feed three products while they are in shared memory).
//   kPlain1   H and W blocks of one K block (bf16 inputs, batches small
//             enough that streaming W from HBM bounds the contraction: the
//             deeper ring of smaller stages keeps more bytes in flight).
// The second block of a pair comes from the same tensor map, `seg_h` /
// `seg_w` elements further along the row: the next K block (kPlain, 64) or
// the lo part of the same K block (the split layouts, one segment).
enum StageLayout : int { kPlain = 0, kSplitW = 1, kSplitHW = 2, kPlain1 = 3 };

template <int L>
struct Layout {
  static constexpr int NA = (L == kSplitW || L == kPlain1) ? 1 : 2;    // H blocks per stage
  static constexpr int NB = L == kPlain1 ? 1 : 2;                      // W blocks per stage
  static constexpr int NP = L == kSplitHW ? 3 : (L == kPlain1 ? 1 : 2); // products per stage
  static constexpr int KSTEP = L == kPlain ? 128 : 64;                 // K columns per stage
  // product p reads H block pa(p) and W block pb(p)
  static __device__ __forceinline__ int pa(int p) {
    return L == kPlain ? p : ((L == kSplitHW && p == 2) ? 1 : 0);
  }
  static __device__ __forceinline__ int pb(int p) { return L == kPlain ? p : (p == 1 ? 1 : 0); }
};

// Pipeline depth for a stage of `stage_bytes`: as many as fit in 192 KiB.
constexpr int stages_for(int stage_bytes) { return (192 * 1024) / stage_bytes; }

constexpr int BM = 128;                      // tokens per tile (UMMA M, TMEM lanes)
constexpr int BN = kTileCols;                // vocab columns per tile (UMMA N)
constexpr int BK = 64;                       // bf16 per K block = 128 B = one swizzle row
constexpr int UMMA_K = 16;                   // K per tcgen05.mma (32 bytes)
constexpr int A_BYTES = BM * BK * 2;         // 16 KiB per H block
constexpr int B_BYTES = BN * BK * 2;         // 32 KiB per W block
constexpr int NUM_THREADS = 192;             // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int EPI_WARPS = 4;
constexpr uint32_t TMEM_COLS = 512;          // two BN-column fp32 accumulators

// Stage geometry per layout: 2 stages of 96 KiB (kPlain, kSplitHW), 2 of
// 80 KiB (kSplitW), 4 of 48 KiB (kPlain1).
template <int L>
struct Cfg {
  static constexpr int STAGE_BYTES = Layout<L>::NA * A_BYTES + Layout<L>::NB * B_BYTES;
  static constexpr int STAGES = stages_for(STAGE_BYTES);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(STAGES >= 2 && 2 * STAGES + 12 <= 32,
                "stage ring, barriers, merge scratch and the pair's work");
};

// Instruction descriptor of tcgen05.mma kind::f16: D fp32 (bits 4-5 = 1),
// A and B bf16 (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                            (uint32_t(BM >> 4) << 24);

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 B, 8-row swizzle atoms of 1024 B
// (stride byte offset 1024), version 1 (bit 46), swizzle mode 2 (bits 61-63).
// `addr` is the shared address of the first element used by this MMA; moving
// along K inside the 128-byte row is a plain +32 B per 16 bf16.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// The merge fused into the contraction (the whole forward in one kernel):
// where to count slab arrivals per 128-token row block and where the merged
// results go.  arrivals == nullptr: the kernel only writes the slab states.
struct FusedMerge {
  uint32_t* arrivals;   // [row blocks] slab states written so far (zeroed before the launch)
  float* loss;          // [N]
  float* lse;           // [N]
  float* mean;          // may be null
  float* sum;           // may be null
  double* block_sums;   // [row blocks] fixed-order loss sum of each row block
  int32_t row_blocks;   // token blocks x CTAs per unit: 128 tokens each
};

// The partition-aware order (part_unit) of the pair kernel's units.  Each
// pair learns its partition from its SM id and its rank in that partition
// from a counter in the workspace header (cleared before every call), and
// takes every pairs[side]-th unit of its side's list from its rank on.  The
// host launches exactly pairs[0] + pairs[1] pairs; a pair whose rank is at or
// beyond its side's planned count (the map was wrong, or the hardware placed
// the pairs otherwise) takes the highest rank of the other side instead,
// which is then missing there, so every unit of both lists is computed once
// however the pairs land.
struct PartArgs {
  uint32_t* reg;         // [2] pairs seen per partition; null: plain round-robin order
  int32_t pairs[2];      // pairs the order plans on each partition
  int32_t q, r;          // partition 0 takes U0 = q P + r units
  uint8_t side[256];     // partition of each SM id
};

struct Args {
  Targets y;
  int64_t y_offset;        // first vocabulary id of W's rows (a vocabulary shard); 0 otherwise
  float2* part;            // [P][N] (m, s) per slab and token
  float* target_logit;     // [N]
  WsHeader* hdr;
  int32_t N, V, D;
  int32_t kblocks;         // stages per tile: K steps of Layout<L>::KSTEP columns
  int32_t seg_h;           // split layouts: column of H's lo block 0 (elements); else 0
  int32_t seg_w;           // split layouts: column of W's lo block 0 (elements); else 0
  Schedule sch;
  uint64_t wait_limit_ns;
  FusedMerge fm;
  int32_t wait_operands;   // 1: H or W is written by the kernel launched just before this
                           // one, which this one may overlap: the producer waits for it
  PartArgs porder;         // pair kernel: the partition-aware order, or plain round-robin
};

// Barrier over the 128 epilogue threads (warps 2-5) of a contraction CTA:
// named barrier 1 (warps 0 and 1 keep streaming and issuing meanwhile).
struct EpiSync {
  __device__ __forceinline__ void operator()() const { ptx::named_bar_sync(1, 128); }
};

// Unit k of a pair's work: of the plain order (side < 0) or of partition
// side's list.
__device__ __forceinline__ void work_coords(const Args& a, int side, int k, int& slab, int& tblock,
                                            int& tile0, int& ntiles) {
  if (side < 0) {
    unit_coords(a.sch, k, slab, tblock, tile0, ntiles);
    return;
  }
  part_unit(a.sch, a.porder.q, a.porder.r, side, k, slab, tblock);
  slab_tiles(a.sch, slab, tile0, ntiles);
}

// Called by all 128 epilogue threads after the CTA wrote its (m, s) states
// of one vocab slab for the 128 tokens of row block `rb` (thread t owns token
// `row`; `yi` is its target).  Counts the slab in; the CTA that brings in a
// row block's last slab merges that block (merge_slab_states per token, lse,
// loss = lse - z_target, NaN and the status bit for a target outside [0, V)),
// and the CTA that merges the last row block forms the mean and the sum
// (rowblock_finish).  `flag` and `red` are this CTA's shared memory.  The
// arithmetic is flce_merge_kernel's, so the one-launch forward and the
// two-stage one agree bit for bit; which CTA merges a block changes nothing.
__device__ __forceinline__ void fused_merge(const Args& a, int rb, int row, bool valid, int64_t yi,
                                            int t, volatile int* flag, volatile double* red) {
  const EpiSync epi_sync;
  // Every epilogue thread has written its state and target logit; the barrier
  // orders those writes before thread 0's release fence and count, and the
  // CTA that counts last acquires them (and all other CTAs' states of this
  // block) before its barrier.  The merge reads them through L2 (ld.cg).
  epi_sync();
  if (t == 0) {
    ptx::fence_acq_rel_gpu();
    const bool last = atomicAdd(&a.fm.arrivals[rb], 1u) == uint32_t(a.sch.slabs - 1);
    if (last) ptx::fence_acq_rel_gpu();
    *flag = last;
  }
  epi_sync();
  if (!*flag) return;
  double l = 0.0;
  if (valid) {
    const bool target_ok = yi >= 0 && yi < a.V;
    const float zt = target_ok ? __ldcg(a.target_logit + row) : 0.f;  // in flight with the states
    const double lse = merge_slab_states(a.part + row, a.sch.slabs, a.N);
    float loss_f;
    if (!target_ok) {  // no slab holds the target: invalid input
      loss_f = __int_as_float(0x7fc00000);
      a.target_logit[row] = loss_f;
      atomicOr(&a.hdr->status, kStatTarget);
    } else {
      loss_f = float(lse - double(zt));
    }
    a.fm.loss[row] = loss_f;
    a.fm.lse[row] = float(lse);
    l = double(loss_f);
  }
  rowblock_finish(l, t, rb, a.fm.row_blocks, a.fm.block_sums, &a.hdr->counter, a.fm.mean,
                  a.fm.sum, a.N, red, flag, epi_sync);
}

template <int L>
__global__ void __launch_bounds__(NUM_THREADS, 1)
flce_tc_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
               const Args a) {
  using LY = Layout<L>;
  constexpr int STAGES = Cfg<L>::STAGES;
  constexpr int STAGE_BYTES = Cfg<L>::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full_bar = bars;                  // [STAGES] TMA landed
  uint64_t* empty_bar = bars + STAGES;        // [STAGES] MMAs done reading the slot
  uint64_t* tfull_bar = bars + 2 * STAGES;    // [2] accumulator ready
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;  // [2] accumulator drained
  uint64_t* done_bar = bars + 2 * STAGES + 4;    // all MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* merge_flag = abort_flag + 1;                                   // fused merge: decision
  double* merge_red = reinterpret_cast<double*>(bars + 2 * STAGES + 7);  // fused merge: [4] warp sums

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(ptx::smem_addr(&full_bar[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_addr(&tfull_bar[b]), 1);
      ptx::mbar_init(ptx::smem_addr(&tempty_bar[b]), EPI_WARPS);
    }
    ptx::mbar_init(ptx::smem_addr(done_bar), 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tensormap(&tmH);
    ptx::prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    ptx::griddep_wait();  // the header is cleared by the kernel before this one
    a.hdr->slabs = a.sch.slabs;
    a.hdr->N = a.N;
    a.hdr->V = a.V;
    a.hdr->magic = kWsMagic;
  }

  uint32_t* status = &a.hdr->status;
  const uint64_t lim = a.wait_limit_ns;
  const Schedule& sch = a.sch;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      if (a.wait_operands) ptx::griddep_wait();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_parity = 0;  // per stage: ever issued / parity of last issue
      bool ok = true;
      for (int u = blockIdx.x; ok && u < sch.units; u += gridDim.x) {
        int slab, tb, t0, nt;
        unit_coords(sch, u, slab, tb, t0, nt);
        for (int t = t0; ok && t < t0 + nt; ++t) {
          for (int kb = 0; kb < a.kblocks; ++kb) {
            if (!wait_bounded(ptx::smem_addr(&empty_bar[stage]), phase ^ 1u, abort_flag, status, lim)) {
              ok = false;
              break;
            }
            const uint32_t fb = ptx::smem_addr(&full_bar[stage]);
            const uint32_t sa = ptx::smem_addr(smem + stage * STAGE_BYTES);
            ptx::mbar_arrive_expect_tx(fb, STAGE_BYTES);
#pragma unroll
            for (int i = 0; i < LY::NA; ++i)
              ptx::tma_load_2d(sa + i * A_BYTES, &tmH, fb, kb * LY::KSTEP + i * a.seg_h, tb * BM);
#pragma unroll
            for (int i = 0; i < LY::NB; ++i)
              ptx::tma_load_2d(sa + LY::NA * A_BYTES + i * B_BYTES, &tmW, fb,
                               kb * LY::KSTEP + i * a.seg_w, t * BN);
            used |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      // Every issued copy must land before the CTA may exit.  On the normal
      // path each of these waits returns at once.
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s))
          wait_bounded(ptx::smem_addr(&full_bar[s]), (last_parity >> s) & 1u, nullptr, status, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < sch.units; u += gridDim.x) {
        int slab, tb, t0, nt;
        unit_coords(sch, u, slab, tb, t0, nt);
        for (int t = 0; ok && t < nt; ++t) {
          if (!wait_bounded(ptx::smem_addr(&tempty_bar[acc]), acc_phase ^ 1u, abort_flag, status, lim)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
          for (int kb = 0; kb < a.kblocks; ++kb) {
            if (!wait_bounded(ptx::smem_addr(&full_bar[stage]), phase, abort_flag, status, lim)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after_sync();
            const uint32_t sa = ptx::smem_addr(smem + stage * STAGE_BYTES);
#pragma unroll
            for (int p = 0; p < LY::NP; ++p) {
              const uint32_t sa_a = sa + LY::pa(p) * A_BYTES;
              const uint32_t sa_b = sa + LY::NA * A_BYTES + LY::pb(p) * B_BYTES;
#pragma unroll
              for (int k = 0; k < BK / UMMA_K; ++k) {
                const uint64_t ad = sw128_desc(sa_a + k * UMMA_K * 2);
                const uint64_t bd = sw128_desc(sa_b + k * UMMA_K * 2);
                ptx::mma_bf16(d_tmem, ad, bd, kIdesc, (kb | p | k) != 0 ? 1u : 0u);
              }
            }
            ptx::mma_commit(ptx::smem_addr(&empty_bar[stage]));  // slot free once read
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          ptx::mma_commit(ptx::smem_addr(&tfull_bar[acc]));  // accumulator complete
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
      // Retire every MMA this thread issued before TMEM is released.
      ptx::mma_commit(ptx::smem_addr(done_bar));
      wait_bounded(ptx::smem_addr(done_bar), 0, nullptr, status, lim);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // The header and the row-block counters may be cleared by the kernel just
    // before this one, which lets this one start early (programmatic launch):
    // wait for it before touching them (or the outputs).
    ptx::griddep_wait();
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row_in_tile = quad * 32 + lane;  // token row of this thread inside the tile
    const uint32_t lane_addr = uint32_t(quad * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < sch.units; u += gridDim.x) {
      int slab, tb, t0, nt;
      unit_coords(sch, u, slab, tb, t0, nt);
      const int row = tb * BM + row_in_tile;
      const bool valid = row < a.N;
      const int64_t yi = valid ? a.y[row] - a.y_offset : -1;  // target column within W
      float m = -INFINITY, s = 0.f, zt = 0.f;
      bool got = false;
      for (int t = t0; t < t0 + nt; ++t) {
        bool w = wait_bounded(ptx::smem_addr(&tfull_bar[acc]), acc_phase, abort_flag, status, lim);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after_sync();
        const int v0 = t * BN;
        fold_tile(tmem_base + lane_addr + uint32_t(acc * BN), min(BN, a.V - v0), yi - v0, m, s,
                  zt, got);
        ptx::tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&tempty_bar[acc]));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) break;
      if (valid) {
        a.part[size_t(slab) * size_t(a.N) + size_t(row)] = make_float2(m, s);
        if (got) a.target_logit[row] = zt;
      }
      if (a.fm.arrivals != nullptr)
        fused_merge(a, tb, row, valid, yi, threadIdx.x - 64, merge_flag, merge_red);
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();  // lanes 1..31 of warps 0 and 1 wait here for their lane 0
  ptx::tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace tc

// ----------------------------------------------------------------- tcgen05 pair kernel

// The same contraction with 256 x 256 tiles computed by a CTA pair
// (cta_group::2).  Each CTA stages its own 128 token rows of H and its own
// 128 vocab rows of W per K block (no multicast); the even CTA issues
// 256x256x16 MMAs that read both CTAs' shared memory and write 128 rows x 256
// columns into each CTA's TMEM.  Per unit of work a pair reads 2 MB of H and
// 2 MB of W (D = 4096) where two single-CTA 128x256 tiles read 6 MB, and the
// smaller per-CTA stage (32 KB) affords a 6-deep ring.
namespace tc2 {

constexpr int BM = 128;                      // token rows per CTA
constexpr int PAIR_M = 2 * BM;               // token rows per pair tile (UMMA M)
constexpr int BN = kTileCols;                // vocab columns per tile (UMMA N)
constexpr int HALF_N = BN / 2;               // W rows staged by each CTA
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int A_BYTES = BM * BK * 2;         // 16 KiB per H block
constexpr int B_BYTES = HALF_N * BK * 2;     // 16 KiB per W block (this CTA's half of the tile)
constexpr int NUM_THREADS = 192;             // warp 0 TMA, warp 1 MMA (even CTA), warps 2..5 epilogue
constexpr int EPI_WARPS = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint16_t kPairMask = 0x3;

// Stage geometry per layout: 3 stages of 64 KiB (kPlain, kSplitHW), 4 of
// 48 KiB (kSplitW), 6 of 32 KiB (kPlain1); both CTAs' copies of a stage
// complete on the even CTA's barrier.
template <int L>
struct Cfg {
  static constexpr int STAGE_BYTES = tc::Layout<L>::NA * A_BYTES + tc::Layout<L>::NB * B_BYTES;
  static constexpr int STAGES = tc::stages_for(STAGE_BYTES);
  static constexpr uint32_t PAIR_TX_BYTES = 2 * STAGE_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
  static_assert(STAGES >= 2 && 2 * STAGES + 12 <= 32,
                "stage ring, barriers, merge scratch and the pair's work");
};

// kind::f16 descriptor as in the single-CTA kernel, with M = 256 (bits 24-28).
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                            (uint32_t(PAIR_M >> 4) << 24);

template <int L>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
flce_tc2_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
                const tc::Args a) {
  using LY = tc::Layout<L>;
  constexpr int STAGES = Cfg<L>::STAGES;
  constexpr int STAGE_BYTES = Cfg<L>::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full_bar = bars;                     // [STAGES] (even CTA) both CTAs' copies landed
  uint64_t* empty_bar = bars + STAGES;           // [STAGES] MMAs done reading the slot
  uint64_t* tfull_bar = bars + 2 * STAGES;       // [2] accumulator ready
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;  // [2] (even CTA) drained by both CTAs
  uint64_t* done_bar = bars + 2 * STAGES + 4;    // (even CTA) all MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* merge_flag = abort_flag + 1;                                   // fused merge: decision
  double* merge_red = reinterpret_cast<double*>(bars + 2 * STAGES + 7);  // fused merge: [4] warp sums

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();    // 0 = even CTA (issues the MMAs)
  const int pair = int(ptx::cluster_id_x());
  const int npairs = int(ptx::cluster_count_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(ptx::smem_addr(&full_bar[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_addr(&tfull_bar[b]), 1);
      ptx::mbar_init(ptx::smem_addr(&tempty_bar[b]), 2 * EPI_WARPS);
    }
    ptx::mbar_init(ptx::smem_addr(done_bar), 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tensormap(&tmH);
    ptx::prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_addr(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  // This pair's work: plain round-robin over all units (side -1), or every
  // pairs[side]-th unit of its partition's list from its rank on (PartArgs).
  int* work = reinterpret_cast<int*>(bars + 2 * STAGES + 11);  // [2] side, first unit
  if (threadIdx.x == 0 && rank == 0) {
    int side = -1, first = pair;
    if (a.porder.reg != nullptr) {
      ptx::griddep_wait();  // the counters are cleared by the kernel before this one
      side = a.porder.side[ptx::smid() & 255u];
      first = int(atomicAdd(&a.porder.reg[side], 1u));
      part_take(a.porder.pairs, side, first);
    }
    work[0] = side;
    work[1] = first;
    ptx::st_shared_cluster_u32(ptx::map_to_cta(ptx::smem_addr(&work[0]), 1), uint32_t(side));
    ptx::st_shared_cluster_u32(ptx::map_to_cta(ptx::smem_addr(&work[1]), 1), uint32_t(first));
  }
  ptx::tc_fence_before_sync();
  ptx::cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  ptx::tc_fence_after_sync();
  const int work_side = work[0], work_first = work[1];
  const int work_stride = work_side < 0 ? npairs : a.porder.pairs[work_side];
  const int work_count =
      work_side < 0 ? a.sch.units : part_units(a.sch, a.porder.q, a.porder.r, work_side);
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    ptx::griddep_wait();  // the header is cleared by the kernel before this one
    a.hdr->slabs = a.sch.slabs;
    a.hdr->N = a.N;
    a.hdr->V = a.V;
    a.hdr->magic = kWsMagic;
  }

  uint32_t* status = &a.hdr->status;
  const uint64_t lim = a.wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      if (a.wait_operands) ptx::griddep_wait();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_parity = 0;
      bool ok = true;
      for (int u = work_first; ok && u < work_count; u += work_stride) {
        int slab, tb, t0, nt;
        work_coords(a, work_side, u, slab, tb, t0, nt);
        const int hrow = tb * PAIR_M + int(rank) * BM;
        for (int t = t0; ok && t < t0 + nt; ++t) {
          const int wrow = t * BN + int(rank) * HALF_N;
          for (int kb = 0; kb < a.kblocks; ++kb) {
            if (!wait_bounded(ptx::smem_addr(&empty_bar[stage]), phase ^ 1u, abort_flag, status,
                              lim)) {
              ok = false;
              break;
            }
            const uint32_t fb_local = ptx::smem_addr(&full_bar[stage]);
            const uint32_t fb_even = ptx::map_to_cta(fb_local, 0);
            const uint32_t sa = ptx::smem_addr(smem + stage * STAGE_BYTES);
            if (rank == 0) ptx::mbar_arrive_expect_tx(fb_local, Cfg<L>::PAIR_TX_BYTES);
#pragma unroll
            for (int i = 0; i < LY::NA; ++i)
              ptx::tma_load_2d_pair(sa + i * A_BYTES, &tmH, fb_even, kb * LY::KSTEP + i * a.seg_h,
                                    hrow);
#pragma unroll
            for (int i = 0; i < LY::NB; ++i)
              ptx::tma_load_2d_pair(sa + LY::NA * A_BYTES + i * B_BYTES, &tmW, fb_even,
                                    kb * LY::KSTEP + i * a.seg_w, wrow);
            used |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      // The even CTA's full barriers count both CTAs' bytes: once its last
      // phase on each slot has completed, no copy of this pair is in flight.
      if (rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (used & (1u << s))
            wait_bounded(ptx::smem_addr(&full_bar[s]), (last_parity >> s) & 1u, nullptr, status,
                         lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = work_first; ok && u < work_count; u += work_stride) {
        int slab, tb, t0, nt;
        work_coords(a, work_side, u, slab, tb, t0, nt);
        for (int t = 0; ok && t < nt; ++t) {
          if (!wait_bounded(ptx::smem_addr(&tempty_bar[acc]), acc_phase ^ 1u, abort_flag, status,
                            lim)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
          for (int kb = 0; kb < a.kblocks; ++kb) {
            if (!wait_bounded(ptx::smem_addr(&full_bar[stage]), phase, abort_flag, status, lim)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after_sync();
            const uint32_t sa = ptx::smem_addr(smem + stage * STAGE_BYTES);
#pragma unroll
            for (int p = 0; p < LY::NP; ++p) {
              const uint32_t sa_a = sa + LY::pa(p) * A_BYTES;
              const uint32_t sa_b = sa + LY::NA * A_BYTES + LY::pb(p) * B_BYTES;
#pragma unroll
              for (int k = 0; k < BK / UMMA_K; ++k) {
                const uint64_t ad = tc::sw128_desc(sa_a + k * UMMA_K * 2);
                const uint64_t bd = tc::sw128_desc(sa_b + k * UMMA_K * 2);
                ptx::mma_bf16_pair(d_tmem, ad, bd, kIdesc, (kb | p | k) != 0 ? 1u : 0u);
              }
            }
            ptx::mma_commit_pair_mc(ptx::smem_addr(&empty_bar[stage]), kPairMask);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          ptx::mma_commit_pair_mc(ptx::smem_addr(&tfull_bar[acc]), kPairMask);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
      ptx::mma_commit_pair(ptx::smem_addr(done_bar));
      wait_bounded(ptx::smem_addr(done_bar), 0, nullptr, status, lim);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    ptx::griddep_wait();  // as in flce_tc_kernel
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_addr = uint32_t(quad * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int u = work_first; ok && u < work_count; u += work_stride) {
      int slab, tb, t0, nt;
      work_coords(a, work_side, u, slab, tb, t0, nt);
      const int row = tb * PAIR_M + int(rank) * BM + row_in_tile;
      const bool valid = row < a.N;
      const int64_t yi = valid ? a.y[row] - a.y_offset : -1;  // target column within W
      float m = -INFINITY, s = 0.f, zt = 0.f;
      bool got = false;
      for (int t = t0; t < t0 + nt; ++t) {
        bool w = wait_bounded(ptx::smem_addr(&tfull_bar[acc]), acc_phase, abort_flag, status, lim);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after_sync();
        const int v0 = t * BN;
        fold_tile(tmem_base + lane_addr + uint32_t(acc * BN), min(BN, a.V - v0), yi - v0, m, s,
                  zt, got);
        ptx::tc_fence_before_sync();
        __syncwarp();
        if (lane == 0)
          ptx::mbar_arrive_cluster(ptx::map_to_cta(ptx::smem_addr(&tempty_bar[acc]), 0));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) break;
      if (valid) {
        a.part[size_t(slab) * size_t(a.N) + size_t(row)] = make_float2(m, s);
        if (got) a.target_logit[row] = zt;
      }
      if (a.fm.arrivals != nullptr)
        tc::fused_merge(a, 2 * tb + int(rank), row, valid, yi, threadIdx.x - 64, merge_flag,
                        merge_red);
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  ptx::tc_fence_before_sync();
  __syncthreads();
  // Neither CTA leaves while the other may still read its shared memory or
  // signal its barriers; the even CTA's MMAs have retired (done_bar).
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// Calibration of the partition-aware order, once per device (host side:
// calibrate_partitions in flce.cu).  Both kernels take the pair kernel's dynamic
// shared memory, so that each CTA has an SM to itself.
//
// Latency of dependent atomic adds, which complete at the L2 slice that
// homes the line, from each CTA's SM to each of `nlines` zeroed lines (the
// lines stay zero: each add adds 0, and each address depends on the value
// before it).  CTAs start on different lines so that they do not queue on
// one slice.
__global__ void __launch_bounds__(32, 1)
flce_part_latency_kernel(uint32_t* lines, int32_t nlines, int32_t stride_words, uint32_t* lat,
                         int32_t* smid_of_block) {
  if (threadIdx.x != 0) return;
  smid_of_block[blockIdx.x] = int32_t(ptx::smid());
  uint32_t v = 0;
  for (int k = 0; k < nlines; ++k) {
    const int l = (k + int(blockIdx.x)) % nlines;
    uint32_t* p = lines + size_t(l) * size_t(stride_words);
    v = atomicAdd(p + (v >> 31), 0u);
    const long long t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 16; ++i) v = atomicAdd(p + (v >> 31), 0u);
    const long long t1 = clock64() + (long long)(v >> 31);
    lat[size_t(blockIdx.x) * size_t(nlines) + size_t(l)] = uint32_t((t1 - t0) / 16);
  }
}

// Where the pairs land when as many as can be resident are launched at once:
// each records the SM of its even CTA, then waits (at most 1 s) until all have
// arrived, so that none leaves its SMs to a later one.  `arrived` starts at
// zero; *timed_out is set if the wait ran out.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(32, 1)
flce_part_cluster_kernel(int32_t* smid_of_pair, uint32_t* arrived, uint32_t* timed_out) {
  if (threadIdx.x != 0) return;
  if (ptx::cluster_ctarank() == 0) smid_of_pair[ptx::cluster_id_x()] = int32_t(ptx::smid());
  atomicAdd(arrived, 1u);
  const uint32_t all = 2u * ptx::cluster_count_x();
  const uint64_t t0 = ptx::globaltimer_ns();
  while (*reinterpret_cast<volatile uint32_t*>(arrived) < all) {
    if (ptx::globaltimer_ns() - t0 > 1000000000ull) {
      atomicOr(timed_out, 1u);
      break;
    }
  }
}

}  // namespace tc2

// ----------------------------------------------------------------- fp32 inputs

// fp32 inputs run on the same bf16 tensor-core kernels after a split of
// every value into two bf16 values (Henry, Tang and Heinecke, "Leveraging
// the bfloat16 artificial intelligence datatype for higher-precision
// computations", ARITH 2019):  hi = bf16(x),  lo = bf16(x - hi),  so that
// |x - hi - lo| <= 2^-16 |x|.  The forward lays H and W out as [hi | lo]
// rows (segments of Dp = D rounded up to 64, zero padded); the contraction
// kernels stage the four parts of each K block together (tc::kSplitHW) and
// accumulate
//   Z = Hhi Whi^T + Hhi Wlo^T + Hlo Whi^T
// in fp32 in TMEM: each product h w is off by at most about 3 * 2^-16 |h w|
// (the dropped lo*lo term and the two rounding residues).  (The backward lays
// H out as [hi | hi | lo] and W as [hi | lo | hi] and walks K = 3 segments.)
namespace split {

constexpr int NUM_THREADS = 256;   // 8 warps, one row per warp at a time

struct Args {
  const float* src;       // (src_rows, D) fp32, row stride ld elements
  int64_t ld;
  int64_t rows;           // rows written; rows >= src_rows are written as zeros
  int64_t src_rows;
  int32_t D;
  int32_t Dp;             // one segment: D rounded up (to 64 for the forward, 8 for the backward)
  int32_t nseg;           // segments per row: 3, or 2 for [hi | lo]
  int32_t lo_segment;     // the segment that holds lo; every other one holds hi
  __nv_bfloat16* dst;     // (rows, nseg Dp) bf16, contiguous
  uint32_t* zero;         // first matrix only: words cleared by block 0 (a forward's
  int32_t zero_words;     // workspace header and counters), or null
};

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 a, __nv_bfloat16 b) {
  return uint32_t(__bfloat16_as_ushort(a)) | (uint32_t(__bfloat16_as_ushort(b)) << 16);
}

// Each lane converts groups of 8 consecutive elements of its warp's row: it
// loads 32 bytes of fp32 (two float4 when `kVec`, i.e. D % 8 == 0, ld % 4 ==
// 0 and a 16-byte-aligned base) and stores 16 bytes to each of the
// segments.  Purely bandwidth-bound: 4 bytes in, 4 or 6 bytes out per
// element.  One launch splits two matrices (the forward's H and W): the rows
// of `first`, then those of `second` (second.rows may be 0); both share D, Dp
// and the segment layout.
template <bool kVec>
__global__ void __launch_bounds__(NUM_THREADS) flce_split3_kernel(const Args first,
                                                                  const Args second) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (NUM_THREADS / 32);
  const int groups = first.Dp / 8;
  const int64_t total = first.rows + second.rows;
  ptx::griddep_launch_dependents();  // a contraction after this launch may start (and wait)
  if (blockIdx.x == 0 && first.zero != nullptr)
    for (int i = threadIdx.x; i < first.zero_words; i += NUM_THREADS) first.zero[i] = 0u;
  for (int64_t rr = int64_t(blockIdx.x) * (NUM_THREADS / 32) + (threadIdx.x >> 5); rr < total;
       rr += warps) {
    const bool in_first = rr < first.rows;
    const Args& a = in_first ? first : second;
    const int64_t r = in_first ? rr : rr - first.rows;
    const bool pad_row = r >= a.src_rows;   // zero padding below the source rows
    const float* row = a.src + (pad_row ? 0 : r) * a.ld;
    uint4* out = reinterpret_cast<uint4*>(a.dst + r * a.nseg * int64_t(a.Dp));
    for (int g = lane; g < groups; g += 32) {
      const int k0 = g * 8;
      float x[8];
      if (k0 >= a.D || pad_row) {
        // zero padding from D to the segment length (or a padding row): nothing is read
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = 0.f;
      } else if (kVec) {        // D % 8 == 0: all 8 elements lie inside the row
        const float4 u = __ldg(reinterpret_cast<const float4*>(row + k0));
        const float4 v = __ldg(reinterpret_cast<const float4*>(row + k0 + 4));
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
        x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = (k0 + j < a.D) ? __ldg(row + k0 + j) : 0.f;
      }
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * j]);
        const __nv_bfloat16 h1 = __float2bfloat16_rn(x[2 * j + 1]);
        // hi lies within a factor 2 of x, so x - hi is exact in fp32
        // (Sterbenz's lemma); its bf16 rounding is the lo part.
        const __nv_bfloat16 l0 = __float2bfloat16_rn(x[2 * j] - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(x[2 * j + 1] - __bfloat162float(h1));
        hi[j] = pack_bf16x2(h0, h1);
        lo[j] = pack_bf16x2(l0, l1);
      }
      const uint4 vh = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      const uint4 vl = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      for (int seg = 0; seg < a.nseg; ++seg) out[seg * groups + g] = seg == a.lo_segment ? vl : vh;
    }
  }
}

// bf16 H padded with zero rows: dst (rows_out, D) = src (N rows, row stride
// ld) followed by rows_out - N zero rows.  16-byte vectors (D and ld are
// multiples of 8 and src is 16-byte aligned for bf16 inputs).
// Clears `n` words at `p` (a forward's workspace header and row-block
// counters) in one block, and lets the contraction launched after it with
// programmatic serialization start at once; the contraction waits for it
// (griddep_wait) before it touches those words.
__global__ void __launch_bounds__(128) flce_clear_header_kernel(uint32_t* p, int32_t n) {
  ptx::griddep_launch_dependents();
  for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = 0u;
}

// Block 0 also clears `zero_words` words at `zero` (a forward's workspace
// header and counters) when `zero` is not null.
__global__ void __launch_bounds__(256) flce_pad_rows_kernel(const uint4* src, int64_t ld_vec,
                                                            int32_t N, int32_t d_vec,
                                                            int32_t rows_out, uint4* dst,
                                                            uint32_t* zero, int32_t zero_words) {
  ptx::griddep_launch_dependents();  // a contraction after this launch may start (and wait)
  if (blockIdx.x == 0 && zero != nullptr)
    for (int i = threadIdx.x; i < zero_words; i += blockDim.x) zero[i] = 0u;
  const int64_t total = int64_t(rows_out) * d_vec;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / d_vec, c = i - r * d_vec;
    dst[i] = r < N ? __ldg(src + r * ld_vec + c) : make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace split

// ----------------------------------------------------------------- quantised head

// Affine group-quantised W (the MLX format): row j, element k holds an
// unsigned BITS-bit code q_jk, packed 32 / BITS to a uint32 word with the
// lowest bits first, and group g = k / G of the row has a bf16 scale s_jg and
// bias b_jg:  W_jk = s_jg q_jk + b_jg.
// One chunk of vocabulary rows at a time is expanded into the layout the
// tensor-core kernels read: per row two K segments of Ds = D rounded up to 64,
// [hi | lo] with hi = bf16(W_jk) and lo = bf16(W_jk - hi) (zero padded from D
// to Ds).  H is bf16 already: the contraction kernels stage each K block of H
// once beside both parts of W (tc::kSplitW) and accumulate H hi^T + H lo^T,
// which is H W^T up to |W - hi - lo| <= 2^-16 |W| per weight.
namespace quant {

constexpr int NUM_THREADS = 256;   // 8 warps, one vocabulary row per warp at a time

struct Args {
  const uint32_t* wq;             // (V, D * BITS / 32) codes
  const __nv_bfloat16* scales;    // (V, D / G)
  const __nv_bfloat16* biases;    // (V, D / G)
  int64_t row0;                   // first vocabulary row of the chunk
  int64_t rows;                   // rows in the chunk
  int32_t D;                      // a multiple of G
  int32_t Ds;                     // D rounded up to 64
  int32_t G;                      // 32, 64 or 128
  __nv_bfloat16* dst;             // (rows, 2 Ds) bf16, contiguous
};

// The 8 codes of elements k0 .. k0 + 7 (k0 a multiple of 8) of one row.
template <int BITS>
__device__ __forceinline__ void load_codes(const uint32_t* row_words, int k0, uint32_t (&q)[8]) {
  if constexpr (BITS == 4) {
    const uint32_t w = __ldg(row_words + k0 / 8);
#pragma unroll
    for (int t = 0; t < 8; ++t) q[t] = (w >> (4 * t)) & 0xFu;
  } else if constexpr (BITS == 8) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(row_words + k0 / 4));
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      q[t] = (w.x >> (8 * t)) & 0xFFu;
      q[t + 4] = (w.y >> (8 * t)) & 0xFFu;
    }
  } else {
    static_assert(BITS == 2, "2, 4 or 8 bits");
    const uint32_t w = __ldg(row_words + k0 / 16) >> (k0 % 16 == 0 ? 0 : 16);
#pragma unroll
    for (int t = 0; t < 8; ++t) q[t] = (w >> (2 * t)) & 0x3u;
  }
}

template <int BITS>
__global__ void __launch_bounds__(NUM_THREADS) flce_dequant_split_kernel(const Args a) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (NUM_THREADS / 32);
  const int groups = a.Ds / 8;
  const int64_t words_per_row = int64_t(a.D) * BITS / 32;
  const int64_t groups_per_row = a.D / a.G;
  for (int64_t r = int64_t(blockIdx.x) * (NUM_THREADS / 32) + (threadIdx.x >> 5); r < a.rows;
       r += warps) {
    const int64_t j = a.row0 + r;
    const uint32_t* row_words = a.wq + j * words_per_row;
    uint4* out = reinterpret_cast<uint4*>(a.dst + r * 2 * int64_t(a.Ds));
    for (int g = lane; g < groups; g += 32) {
      const int k0 = g * 8;
      uint4 vh = make_uint4(0u, 0u, 0u, 0u), vl = vh;
      if (k0 < a.D) {
        uint32_t q[8];
        load_codes<BITS>(row_words, k0, q);
        const int64_t gi = j * groups_per_row + k0 / a.G;
        const float sc = __bfloat162float(a.scales[gi]);
        const float bi = __bfloat162float(a.biases[gi]);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          // s q + b rounded once to fp32 (s q alone is exact: at most 16 bits)
          const float w0 = fmaf(sc, float(q[2 * t]), bi);
          const float w1 = fmaf(sc, float(q[2 * t + 1]), bi);
          const __nv_bfloat16 h0 = __float2bfloat16_rn(w0);
          const __nv_bfloat16 h1 = __float2bfloat16_rn(w1);
          hi[t] = split::pack_bf16x2(h0, h1);
          lo[t] = split::pack_bf16x2(__float2bfloat16_rn(w0 - __bfloat162float(h0)),
                                     __float2bfloat16_rn(w1 - __bfloat162float(h1)));
        }
        vh = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        vl = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      out[g] = vh;
      out[groups + g] = vl;
    }
  }
}

}  // namespace quant

// ----------------------------------------------------------------- merge + mean

constexpr int kMergeThreads = 256;

struct MergeArgs {
  const float2* part;
  Targets y;
  float* target_logit;
  float* loss;
  float* lse;
  float* mean;          // may be null
  float* sum;           // may be null: sum_i loss_i from the same fp64 total as the mean
  double* block_sums;   // [gridDim.x]: one per kMergeTokensPerBlock tokens
  WsHeader* hdr;
  int32_t N, V;
  int32_t max_slabs;    // capacity of the partial array in this workspace
};

// The two-stage forward's merge (after flce_partials): one thread per token,
// one 128-token row block per CTA, with exactly the fused merge's arithmetic
// (merge_slab_states, then rowblock_finish for the mean and the sum), so the
// two-stage forward and the one-launch forward agree bit for bit.
constexpr int kMergeTokensPerBlock = 128;
constexpr int kMergeBlockThreads = kMergeTokensPerBlock;

struct BlockSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

__global__ void __launch_bounds__(kMergeBlockThreads) flce_merge_kernel(const MergeArgs a) {
  __shared__ double red[4];
  __shared__ int flag;
  const int t = threadIdx.x;
  const int i = blockIdx.x * kMergeTokensPerBlock + t;
  const WsHeader h = *a.hdr;
  const bool ws_ok = h.magic == kWsMagic && h.N == a.N && h.V == a.V && h.slabs >= 1 &&
                     h.slabs <= a.max_slabs;
  double l = 0.0;
  if (i < a.N) {
    float loss_f, lse_f;
    if (!ws_ok) {
      loss_f = lse_f = __int_as_float(0x7fc00000);
      if (i == 0) atomicOr(&a.hdr->status, kStatBadWs);
    } else {
      const double lse = merge_slab_states(a.part + i, h.slabs, a.N);
      const int64_t yi = a.y[i];
      lse_f = float(lse);
      if (yi < 0 || yi >= a.V) {
        loss_f = __int_as_float(0x7fc00000);
        a.target_logit[i] = loss_f;
        atomicOr(&a.hdr->status, kStatTarget);
      } else {
        loss_f = float(lse - double(a.target_logit[i]));
      }
    }
    a.loss[i] = loss_f;
    a.lse[i] = lse_f;
    l = double(loss_f);
  }
  rowblock_finish(l, t, int(blockIdx.x), int(gridDim.x), a.block_sums, &a.hdr->counter, a.mean,
                  a.sum, a.N, red, &flag, BlockSync{});
}

// ----------------------------------------------------------------- vocabulary shards

// One vocabulary shard's contribution per token, after flce_partials on the
// shard: its slab states folded into one (m, s) (the section-1 recurrence
// over slabs), the target logit if the shard holds the target, and 1/0 for
// "holds it".  Layout: float4 {m, s, target, owned}.
__global__ void __launch_bounds__(kMergeThreads) flce_shard_state_kernel(
    const float2* part, const WsHeader* hdr, const int64_t* y, int32_t N, int64_t v_offset,
    int64_t v_count, int32_t max_slabs, const float* target_logit, float4* out,
    uint32_t* status) {
  const int i = blockIdx.x * kMergeThreads + threadIdx.x;
  if (i >= N) return;
  const WsHeader h = *hdr;
  float4 r;
  if (h.magic != kWsMagic || h.N != N || h.V != v_count || h.slabs < 1 || h.slabs > max_slabs) {
    r = make_float4(__int_as_float(0x7fc00000), 0.f, 0.f, 0.f);
    if (i == 0) atomicOr(status, kStatBadWs);
  } else {
    float M = -INFINITY;
    for (int p = 0; p < h.slabs; ++p) M = fmaxf(M, part[size_t(p) * N + i].x);
    double S = 0.0;
    for (int p = 0; p < h.slabs; ++p) {
      const float2 st = part[size_t(p) * N + i];
      S += double(st.y) * exp(double(st.x) - double(M));
    }
    const int64_t rel = y[i] - v_offset;
    const bool owned = rel >= 0 && rel < v_count;
    r = make_float4(M, float(S), owned ? target_logit[i] : 0.f, owned ? 1.f : 0.f);
  }
  out[i] = r;
}

// Combines the per-token states of G shards (in shard order): m = max_r m_r,
// s = sum_r s_r exp(m_r - m), lse = m + log s; the target logit comes from
// the shard that holds it (exactly one for a valid target); loss = lse -
// target; mean and sum as in flce_merge_kernel.
__global__ void __launch_bounds__(kMergeThreads) flce_merge_shards_kernel(
    const float4* states, int32_t G, const int64_t* y, int32_t N, int64_t V_total, float* loss,
    float* lse, float* target_logit, float* mean, float* sum, double* block_sums, WsHeader* hdr) {
  __shared__ double warp_sums[kMergeThreads / 32];
  __shared__ bool is_last;
  const int i = blockIdx.x * kMergeThreads + threadIdx.x;
  double l = 0.0;
  if (i < N) {
    float M = -INFINITY;
    for (int r = 0; r < G; ++r) M = fmaxf(M, states[size_t(r) * N + i].x);
    double S = 0.0;
    float t = 0.f;
    int owners = 0;
    for (int r = 0; r < G; ++r) {
      const float4 st = states[size_t(r) * N + i];
      S += double(st.y) * exp(double(st.x) - double(M));
      if (st.w != 0.f) {
        t = st.z;
        ++owners;
      }
    }
    const double lse_d = double(M) + log(S);
    const int64_t yi = y[i];
    float loss_f;
    if (yi < 0 || yi >= V_total || owners != 1) {
      loss_f = t = __int_as_float(0x7fc00000);
      atomicOr(&hdr->status, kStatTarget);
    } else {
      loss_f = float(lse_d - double(t));
    }
    loss[i] = loss_f;
    lse[i] = float(lse_d);
    target_logit[i] = t;
    l = double(loss_f);
  }
  if (mean == nullptr && sum == nullptr) return;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) l += __shfl_down_sync(0xffffffffu, l, off);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = l;
  __syncthreads();
  if (threadIdx.x == 0) {
    double b = 0.0;
    for (int w = 0; w < kMergeThreads / 32; ++w) b += warp_sums[w];
    block_sums[blockIdx.x] = b;
    ptx::fence_acq_rel_gpu();  // release: this block sum before the count
    const uint32_t ticket = atomicAdd(&hdr->counter, 1u);
    is_last = ticket == gridDim.x - 1;
  }
  __syncthreads();
  if (is_last && threadIdx.x == 0) {
    ptx::fence_acq_rel_gpu();  // acquire: every block sum, seen through the count
    const volatile double* bs = block_sums;
    double total = 0.0;
    for (int b = 0; b < int(gridDim.x); ++b) total += bs[b];
    if (mean != nullptr) *mean = float(total / double(N));
    if (sum != nullptr) *sum = float(total);
    hdr->counter = 0;
  }
}

// ----------------------------------------------------------------- self-test

// One thread waits on a barrier that nothing will complete; the bounded wait
// gives up after limit_ns, records kStatTimeout and the kernel returns.
__global__ void flce_wait_probe_kernel(WsHeader* hdr, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int flag;
  if (threadIdx.x != 0) return;
  flag = 0;
  ptx::mbar_init(ptx::smem_addr(&bar), 1);
  ptx::fence_barrier_init();
  wait_bounded(ptx::smem_addr(&bar), 0, &flag, &hdr->status, limit_ns);
}

}  // namespace flce
