// Host-side schedule of the forward contraction: workspace sizes, the
// split-V slab count, the raster groups and the work-unit order that
// flce_tc_kernel / flce_tc2_kernel walk.  Included by flce.cu only (inside
// its anonymous namespace, after flce_kernels.cuh); no device code.
//
// Operation scheduled: the vocabulary tiles of section 1 of D. Ineshin, "Een
// gefuseerde forward-kernel voor lineaire cross-entropy op Apple-GPU's"
// (2026), cut into slabs that run in parallel and merge afterwards.
#pragma once

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool sizes_ok(int64_t N, int64_t V, int64_t D, flce_dtype dtype) {
  if (N < 0 || V < 1 || D < 1) return false;
  if (dtype != FLCE_BF16 && dtype != FLCE_FP32) return false;
  return true;
}

int64_t slab_capacity(int64_t V) { return std::min<int64_t>(cdiv(V, kTileCols), kMaxSlabs); }

// 128-token row blocks the fused merge counts: two per 256-token block, which
// covers one per 128-token block of the single-CTA kernel.
int64_t row_block_capacity(int64_t N) { return 2 * cdiv(std::max<int64_t>(N, 1), 256); }

// Byte offsets in the workspace of the forward's state: the header, one
// arrival counter per row block (zeroed with the header before every call),
// the (m, s) partial states [slab][token], and the block sums of the mean.
struct StateLayout {
  size_t counters = 0, part = 0, sums = 0, total = 0;
};

StateLayout state_layout(int64_t N, int64_t V) {
  StateLayout L;
  L.counters = kHeaderBytes;
  L.part = L.counters + align256(size_t(4) * size_t(row_block_capacity(N)));
  L.sums = L.part + align256(size_t(8) * size_t(N) * size_t(slab_capacity(V)));
  // block results of the mean: one per kMergeTokensPerBlock tokens (the merge
  // kernel), which also covers one per kMergeThreads tokens (the shard merge)
  // and one per row block (the fused merge)
  const int64_t nsums =
      std::max<int64_t>({1, cdiv(N, kMergeTokensPerBlock), row_block_capacity(N)});
  L.total = L.sums + align256(size_t(8) * size_t(nsums));
  return L;
}

// Header, counters, (m, s) partial states and the mean's block sums.
size_t state_bytes_for(int64_t N, int64_t V) { return state_layout(N, V).total; }

// fp32 inputs run on bf16 hi / lo parts.  The forward lays H and W out as
// [hi | lo] rows (the kernel stages a K block of each part side by side), so a
// segment must end on a 64-element K block: D rounded up to 64.  The backward
// lays both out in three segments of D rounded up to 8.
int64_t fwd_split_segment(int64_t D) { return (D + 63) / 64 * 64; }
int64_t bwd_split_segment(int64_t D) { return (D + 7) / 8 * 8; }

// bf16 elements per row of the operands the forward's tensor-core kernels
// stage: D for bf16 inputs, the hi and lo segments for fp32 inputs.
int64_t k_extent(int64_t D, flce_dtype dtype) {
  return dtype == FLCE_FP32 ? 2 * fwd_split_segment(D) : D;
}

// Batches of fewer than this many tokens read H from a copy padded with zero
// rows up to it.  All CTAs read the same H rows every K block; with 1 to 8
// rows those few lines are a hot spot that slowed the whole W stream by 20%
// on B200 (N = 1 and 8: 254-270 us against 208-212 us at N = 32 and 128, V =
// 151936, D = 4096), and 32 rows spread the reads enough.
constexpr int64_t kMinHRows = 32;
int64_t padded_h_rows(int64_t N) { return std::max<int64_t>(N, kMinHRows); }

// bf16 inputs with N < kMinHRows: the padded copy of H (kMinHRows, D) bf16.
size_t fwd_pad_h_bytes(int64_t N, int64_t D) {
  return N < kMinHRows ? align256(size_t(kMinHRows) * size_t(D) * 2) : 0;
}

// Workspace for the forward's split copies of fp32 inputs: H (padded_h_rows,
// 2 Dp) and W (V, 2 Dp) bf16, each 256-byte aligned.
size_t fwd_split_h_bytes(int64_t N, int64_t D) {
  return align256(size_t(padded_h_rows(N)) * size_t(2 * fwd_split_segment(D)) * 2);
}
size_t fwd_split_w_bytes(int64_t V, int64_t D) {
  return align256(size_t(V) * size_t(2 * fwd_split_segment(D)) * 2);
}

// The backward's split copies: (rows, 3 Dp) bf16.
size_t bwd_split_bytes_for(int64_t rows, int64_t D) {
  return align256(size_t(rows) * size_t(3 * bwd_split_segment(D)) * 2);
}

size_t workspace_bytes_for(int64_t N, int64_t V, int64_t D, flce_dtype dtype) {
  size_t b = state_bytes_for(N, V);
  if (dtype == FLCE_FP32) b += fwd_split_h_bytes(N, D) + fwd_split_w_bytes(V, D);
  else b += fwd_pad_h_bytes(N, D);
  return b;
}

// Makespan, in tiles, of the busiest worker when the units of a schedule are
// handed out round-robin (worker c takes units c, c + g, c + 2g, ...) in the
// grouped order of unit_coords.  Unit sizes are base + 1 tiles for slabs
// < rem and base otherwise.  In group k the long units form one contiguous
// run of rem * gt_k units starting at k * gt * P; a run of L units gives every
// worker floor(L / g) of them plus one more to L mod g consecutive workers
// (mod g), which a circular difference array accumulates.
int64_t grouped_makespan(int64_t tb, int64_t gt, int64_t P, int64_t base, int64_t rem, int64_t g,
                         std::vector<int64_t>& diff) {
  const int64_t U = tb * P;
  diff.assign(size_t(g) + 1, 0);
  int64_t every = 0;
  for (int64_t k = 0; k * gt < tb; ++k) {
    const int64_t gk = std::min(gt, tb - k * gt);
    const int64_t L = rem * gk;
    every += L / g;
    const int64_t r = L % g, a = (k * gt * P) % g;
    if (r == 0) continue;
    diff[size_t(a)] += 1;
    if (a + r <= g) {
      diff[size_t(a + r)] -= 1;
    } else {
      diff[size_t(g)] -= 1;
      diff[0] += 1;
      diff[size_t(a + r - g)] -= 1;
    }
  }
  int64_t best = 0, run = 0;
  for (int64_t c = 0; c < g; ++c) {
    run += diff[size_t(c)];
    const int64_t units_c = U / g + (c < U % g ? 1 : 0);
    best = std::max(best, units_c * base + every + run);
  }
  return best;
}

// Choose P (slabs per token block) for `tb` token blocks in groups of `gt`,
// `nt` vocab tiles and `g` concurrent workers: the smallest makespan, plus a
// small per-unit cost (a partial state write and a pipeline restart).
void choose_slabs(int64_t tb, int64_t gt, int64_t nt, int64_t g, int64_t pcap, int32_t& P_out,
                  int64_t& makespan_out) {
  double best = 1e300;
  int32_t bestP = 1;
  int64_t best_ms = 0;
  std::vector<int64_t> diff;
  for (int64_t P = 1; P <= std::min(nt, pcap); ++P) {
    const int64_t ms = grouped_makespan(tb, gt, P, nt / P, nt % P, g, diff);
    // Slabs of unequal length let the workers drift apart over the run, and
    // the workers that share a W tile then fetch it from HBM at different
    // times; equal slabs keep them in step.  So a schedule with a remainder
    // pays 1% of its makespan (at N=8192 V=151936 D=4096 on a B200: 99 equal
    // slabs of 6 tiles ran 7.70 ms per launch against 7.79 ms for 30 slabs
    // of 19-20 tiles, sustained under the power cap).
    const double cost = double(ms) * (nt % P != 0 ? 1.01 : 1.0) + 0.05 * double(cdiv(tb * P, g));
    if (cost < best - 1e-9) {
      best = cost;
      bestP = int32_t(P);
      best_ms = ms;
    }
  }
  P_out = bestP;
  makespan_out = best_ms;
}

// Token blocks per raster group: as many as keep the live part of H within
// kGroupHBytes, so that it and the W tiles in flight stay in one die's L2
// partition.
constexpr int64_t kGroupHBytes = 32ll << 20;

int64_t group_blocks_for(int64_t tb, int64_t block_rows, int64_t D, int64_t elem_bytes) {
  const int64_t per_block = std::max<int64_t>(1, block_rows * D * elem_bytes);
  return std::max<int64_t>(1, std::min(tb, kGroupHBytes / per_block));
}

// The contraction runs on CTA pairs (256-token tiles) unless the batch fits
// one 128-token tile, where half of every pair tile would be padding.
bool use_pair_kernel(int64_t N) { return N > tc::BM; }

// `workers`: CTAs (single-CTA kernels) or CTA pairs (pair kernel) that run at once.
flce_status make_plan(int64_t N, int64_t V, int64_t D, flce_dtype dtype, int64_t workers,
                      flce_plan_t* p) {
  std::memset(p, 0, sizeof(*p));
  p->N = N;
  p->V = V;
  p->D = D;
  p->dtype = int32_t(dtype);
  p->tile_cols = kTileCols;
  const bool pair = use_pair_kernel(N);
  p->ctas_per_unit = pair ? 2 : 1;
  p->block_rows = pair ? tc2::PAIR_M : tc::BM;
  p->k_block = tc::BK;
  p->token_blocks = cdiv(std::max<int64_t>(N, 1), p->block_rows);
  p->vocab_tiles = cdiv(V, kTileCols);
  const int64_t g = std::max<int64_t>(1, workers);
  // Sized by the bf16 rows of H (for fp32 inputs: their hi parts).  fp32's
  // [hi | lo] rows hold twice the bytes per block, yet at N=8192 V=151936
  // D=4096 a group of 16 blocks (64 MB of H) measured faster than one sized by
  // the full rows (7 blocks: 23.1-23.5 against 24.6-25.2 ms; DRAM reads 30.1
  // against 35.4 GB per launch): fewer slabs in flight share each W tile.
  p->group_blocks = int32_t(group_blocks_for(p->token_blocks, p->block_rows, D, 2));
  int64_t ms = 0;
  choose_slabs(p->token_blocks, p->group_blocks, p->vocab_tiles, g, slab_capacity(V), p->slabs,
               ms);
  p->slab_base = int32_t(p->vocab_tiles / p->slabs);
  p->slab_rem = int32_t(p->vocab_tiles % p->slabs);
  p->units = p->token_blocks * p->slabs;
  p->grid = int32_t(std::min<int64_t>(g, p->units) * p->ctas_per_unit);
  p->makespan_tiles = ms;
  p->workspace_bytes = workspace_bytes_for(N, V, D, dtype);
  return FLCE_OK;
}

int64_t nominal_workers(int32_t sms, int64_t N) {
  return use_pair_kernel(N) ? std::max<int64_t>(1, sms / 2) : int64_t(sms);
}

