// Device code of the backward of the fused linear cross-entropy (sm_100a).
//
// For the weighted loss sum_i g_i loss_i, with loss_i = logsumexp(Z_i) -
// Z_{i, y_i} and Z = H W^T (D. Ineshin, "Een gefuseerde forward-kernel voor
// lineaire cross-entropy op Apple-GPU's", 2026, section 1):
//   dZ_ij = g_i (exp(z_ij - lse_i) - [j == y_i]),   dH = dZ W,   dW = dZ^T H.
// As on the page (section 1), the backward keeps the forward's log-sum-exp
// and regenerates the logits tile by tile, one vocabulary chunk at a time, so
// only an (N x chunk) slice of dZ ever exists.  Per chunk C of W's rows:
//   K1  Z_C = H W_C^T on the tensor cores; the epilogue turns each tile into
//       dZ_C (bf16, token-major);
//   K2  dH (+)= dZ_C W_C     A = dZ_C (K = vocab, contiguous: K-major),
//                            B = W_C read as (d, vocab) with d contiguous
//                            (MN-major);
//   K3  dW_C  = dZ_C^T H     A = dZ_C read as (vocab, token) with vocab
//                            contiguous (MN-major), B = H read as (d, token)
//                            with d contiguous (MN-major).
// All three are one CTA-pair GEMM kernel (C = A B^T, 256 x 256 pair tiles,
// 6-stage TMA ring, double-buffered TMEM accumulators) with different
// epilogues and operand orders; the tensor cores read MN-major operands
// directly, so nothing is transposed in memory.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "flce_kernels.cuh"
#include "ptx_sm100.cuh"

namespace flce {
namespace bwd {

// ----------------------------------------------------------------- tile schedule

struct GemmShape {
  int32_t M, N, K;        // C (M x N) = A (M x K) B^T (B is N x K)
  int32_t tiles_m, tiles_n;
  int32_t group_m;        // m-blocks per raster group
  int32_t tiles;          // tiles_m * tiles_n
  int32_t kblocks;        // ceil(K / 64)
  int32_t kblocks_a;      // K-blocks of A; A's K coordinate wraps modulo this (== kblocks,
                          // except for the quantised head's [H | H])
};

// Tile t -> (m-block, n-block): groups of group_m m-blocks, n-major inside a
// group, so the pairs running together share B tiles and keep few A rows live.
__device__ __forceinline__ void tile_coords(const GemmShape& s, int t, int& mb, int& nb) {
  const int per_group = s.group_m * s.tiles_n;
  const int g = t / per_group;
  const int l = t - g * per_group;
  const int gm = min(s.group_m, s.tiles_m - g * s.group_m);
  nb = l / gm;
  mb = g * s.group_m + (l - nb * gm);
}

// ----------------------------------------------------------------- epilogues
//
// Each epilogue processes, for one thread, one accumulator row (a TMEM lane)
// of a 256-column tile: `row` is the global row of C, `n0` the first column,
// `taddr` the thread's lane at column 0 of the accumulator.  All 32 lanes of
// a warp call it together (TMEM loads are warp-wide).

// K1: dZ from the regenerated logits.
struct EpiGradLogits {
  // 32 values rounded to bf16 at dst (columns col0 .. col0 + 31 of a row,
  // those below clen), 16-byte stores when all 32 are in the chunk.
  __device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const float (&d)[32],
                                              int col0) const {
    if (col0 + 32 <= clen) {
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(d[q * 8 + 2 * e], d[q * 8 + 2 * e + 1]);
        d4[q] = *reinterpret_cast<uint4*>(h);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < clen) dst[j] = __float2bfloat16_rn(d[j]);
    }
  }

  const float* lse;          // (N) from the forward
  const int64_t* y;          // (N)
  const float* grad;         // (N) upstream gradient, or null (then every g_i = 1)
  float grad_scale;          // multiplies grad
  int32_t N;                 // tokens
  int32_t V;                 // vocabulary size (for the target check)
  int64_t y_offset;          // vocabulary id of W's first row (a vocabulary shard); else 0
  int32_t c0;                // first row of this chunk within W
  int32_t clen;              // vocabulary rows in this chunk
  __nv_bfloat16* dz;         // (N x ldz) token-major slice, columns = chunk vocab
  __nv_bfloat16* dz_lo;      // null, or (N x ldz): bf16(dZ - dz) for fp32 inputs, so that
                             // dz + dz_lo carries dZ to 2^-16 relative
  int32_t ldz;
  uint32_t* status;

  __device__ __forceinline__ void operator()(int row, int n0, uint32_t taddr) const {
    const bool valid = row < N;
    float l2 = 0.f, gi = 0.f;
    int64_t yrel = -1;
    if (valid) {
      l2 = lse[row] * kLog2e;
      gi = grad_scale * (grad ? grad[row] : 1.f);
      const int64_t yi = y[row];
      if (yi < 0 || yi >= V) atomicOr(status, kStatTarget);
      yrel = yi - y_offset - c0;
    }
#pragma unroll 1
    for (int c = 0; c < kTileCols / 32; ++c) {
      const int col0 = n0 + c * 32;
      if (col0 >= clen) break;  // warp-uniform
      uint32_t u[32];
      ptx::tmem_ld32_wait(taddr + uint32_t(c * 32), u);
      float d[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = col0 + j;
        const float p = ptx::ex2(fmaf(__uint_as_float(u[j]), kLog2e, -l2));
        d[j] = (col < clen) ? gi * (p - (int64_t(col) == yrel ? 1.f : 0.f)) : 0.f;
      }
      if (!valid) continue;
      // token-major: 32 consecutive vocab entries of this row
      const size_t at = size_t(row) * size_t(ldz) + col0;
      store_row32(dz + at, d, col0);
      if (dz_lo != nullptr) {
#pragma unroll
        for (int j = 0; j < 32; ++j) d[j] -= __bfloat162float(__float2bfloat16_rn(d[j]));
        store_row32(dz_lo + at, d, col0);
      }
    }
  }
};

// K2 / K3: an fp32 tile stored into (or added onto) a row-major fp32 matrix.
struct EpiStoreF32 {
  float* out;       // row r of C goes to out + (row_base + r) * ld
  int32_t ld;
  int32_t rows;     // valid rows of C
  int32_t cols;     // valid columns of C
  int32_t row_base;
  int32_t accumulate;  // 0: store, 1: out += C

  __device__ __forceinline__ void operator()(int row, int n0, uint32_t taddr) const {
#pragma unroll 1
    for (int c = 0; c < kTileCols / 32; ++c) {
      const int col0 = n0 + c * 32;
      if (col0 >= cols) break;  // warp-uniform
      uint32_t u[32];
      ptx::tmem_ld32_wait(taddr + uint32_t(c * 32), u);
      if (row >= rows) continue;
      float* dst = out + size_t(row_base + row) * size_t(ld) + col0;
      if (col0 + 32 <= cols && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 v = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                                 __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
          if (accumulate) {
            const float4 o = d4[q];
            v.x += o.x;
            v.y += o.y;
            v.z += o.z;
            v.w += o.w;
          }
          d4[q] = v;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < cols)
            dst[j] = accumulate ? dst[j] + __uint_as_float(u[j]) : __uint_as_float(u[j]);
      }
    }
  }
};

// ----------------------------------------------------------------- pair GEMM

constexpr int BM = 128;               // rows of C per CTA
constexpr int PAIR_M = 2 * BM;        // rows of C per pair tile (UMMA M)
constexpr int BN = kTileCols;         // columns of C per tile (UMMA N)
constexpr int HALF_N = BN / 2;        // rows of B staged by each CTA
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = HALF_N * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t PAIR_TX_BYTES = 2 * STAGE_BYTES;
constexpr int NUM_THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint16_t kPairMask = 0x3;
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                (uint32_t(PAIR_M >> 4) << 24);
constexpr int MN_CHUNK = 64;                 // MN elements per 128-byte swizzle row
constexpr int MN_BOX_BYTES = MN_CHUNK * BK * 2;  // one 64 (MN) x 64 (K) box: 8 KiB

// Shared-memory descriptor of an MN-major operand staged as 64 (MN) x 64 (K)
// TMA boxes with 128-byte swizzling: each K row holds 64 MN elements (128 B),
// 8-row K groups are 1024 B apart (stride byte offset) and consecutive
// 64-element MN chunks are one box, 8 KiB, apart (leading byte offset).  One
// K = 16 step of the MMA covers 16 rows, i.e. +2048 B.
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(MN_BOX_BYTES >> 4) << 16) |
         (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// C = A B^T on CTA pairs, C tiles handed to `epi`.  Same pipeline and
// barrier protocol as the forward's pair kernel (see tc2::flce_tc2_kernel):
// warp 0 of each CTA streams its A rows and its half of the B rows by TMA,
// warp 1 of the even CTA issues the pair MMAs, warps 2-5 of both CTAs run the
// epilogue on their own TMEM rows.  Bounded waits throughout.
// kAmn / kBmn: the operand is MN-major (its tensor map's inner dimension is
// M resp. N, the outer one K); otherwise K-major (inner dimension K).
template <class Epi, bool kAmn, bool kBmn>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmShape shape, const Epi epi, uint32_t* status, uint64_t wait_limit_ns) {
  constexpr uint32_t kIdesc = kIdescBase | (kAmn ? (1u << 15) : 0u) | (kBmn ? (1u << 16) : 0u);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* done_bar = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
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
    ptx::prefetch_tensormap(&tmA);
    ptx::prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_addr(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before_sync();
  ptx::cluster_sync();
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t lim = wait_limit_ns;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_parity = 0;
      bool ok = true;
      for (int t = pair; ok && t < shape.tiles; t += npairs) {
        int mb, nb;
        tile_coords(shape, t, mb, nb);
        const int arow = mb * PAIR_M + int(rank) * BM;
        const int brow = nb * BN + int(rank) * HALF_N;
        for (int kb = 0, ka = 0; kb < shape.kblocks; ++kb) {
          if (!wait_bounded(ptx::smem_addr(&empty_bar[stage]), phase ^ 1u, abort_flag, status,
                            lim)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = ptx::smem_addr(&full_bar[stage]);
          const uint32_t fb_even = ptx::map_to_cta(fb_local, 0);
          const uint32_t sa = ptx::smem_addr(smem + stage * STAGE_BYTES);
          if (rank == 0) ptx::mbar_arrive_expect_tx(fb_local, PAIR_TX_BYTES);
          if (kAmn) {  // two 64 (M) x 64 (K) boxes
            ptx::tma_load_2d_pair(sa, &tmA, fb_even, arow, ka * BK);
            ptx::tma_load_2d_pair(sa + MN_BOX_BYTES, &tmA, fb_even, arow + MN_CHUNK, ka * BK);
          } else {     // one 64 (K) x 128 (M) box
            ptx::tma_load_2d_pair(sa, &tmA, fb_even, ka * BK, arow);
          }
          if (++ka == shape.kblocks_a) ka = 0;
          if (kBmn) {
            ptx::tma_load_2d_pair(sa + A_BYTES, &tmB, fb_even, brow, kb * BK);
            ptx::tma_load_2d_pair(sa + A_BYTES + MN_BOX_BYTES, &tmB, fb_even, brow + MN_CHUNK,
                                  kb * BK);
          } else {
            ptx::tma_load_2d_pair(sa + A_BYTES, &tmB, fb_even, kb * BK, brow);
          }
          used |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (used & (1u << s))
            wait_bounded(ptx::smem_addr(&full_bar[s]), (last_parity >> s) & 1u, nullptr, status,
                         lim);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; ok && t < shape.tiles; t += npairs) {
        if (!wait_bounded(ptx::smem_addr(&tempty_bar[acc]), acc_phase ^ 1u, abort_flag, status,
                          lim)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        for (int kb = 0; kb < shape.kblocks; ++kb) {
          if (!wait_bounded(ptx::smem_addr(&full_bar[stage]), phase, abort_flag, status, lim)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint32_t sa = ptx::smem_addr(smem + stage * STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            // K-major: +32 B along the 128-byte row; MN-major: +16 rows of 128 B
            const uint64_t ad = kAmn ? sw128_desc_mn(sa + k * UMMA_K * 128)
                                     : tc::sw128_desc(sa + k * UMMA_K * 2);
            const uint64_t bd = kBmn ? sw128_desc_mn(sa + A_BYTES + k * UMMA_K * 128)
                                     : tc::sw128_desc(sa + A_BYTES + k * UMMA_K * 2);
            ptx::mma_bf16_pair(d_tmem, ad, bd, kIdesc, (kb | k) != 0 ? 1u : 0u);
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
      ptx::mma_commit_pair(ptx::smem_addr(done_bar));
      wait_bounded(ptx::smem_addr(done_bar), 0, nullptr, status, lim);
    }
  } else {
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_addr = uint32_t(quad * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < shape.tiles; t += npairs) {
      int mb, nb;
      tile_coords(shape, t, mb, nb);
      bool w = wait_bounded(ptx::smem_addr(&tfull_bar[acc]), acc_phase, abort_flag, status, lim);
      if (!__all_sync(0xffffffffu, w)) break;
      ptx::tc_fence_after_sync();
      epi(mb * PAIR_M + int(rank) * BM + row_in_tile, nb * BN,
          tmem_base + lane_addr + uint32_t(acc * BN));
      ptx::tc_fence_before_sync();
      __syncwarp();
      if (lane == 0)
        ptx::mbar_arrive_cluster(ptx::map_to_cta(ptx::smem_addr(&tempty_bar[acc]), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncwarp();
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace bwd
}  // namespace flce
