// libflce.so: host side of the C ABI declared in include/flce.h.
//
// Argument validation, the split-V schedule, TMA tensor maps and the kernel
// launches for the fused linear cross-entropy forward (D. Ineshin, "Een
// gefuseerde forward-kernel voor lineaire cross-entropy op Apple-GPU's",
// 2026, section 1).  Every launch is asynchronous on the caller's stream; the
// library allocates nothing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "flce.h"
#include "flce_backward.cuh"
#include "flce_kernels.cuh"

namespace {

using namespace flce;

// A named NVTX range around each public entry point that enqueues GPU work,
// so profiler timelines show which library call issued which kernels.  NVTX
// is header-only and does nothing unless a profiling tool is attached.
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
#define FLCE_TRACE() TraceRange flce_trace_range_(__func__)

constexpr uint64_t kDefaultWaitLimitNs = 4000000000ull;  // 4 s in one wait: far beyond any real stage

#include "flce_schedule.h"

// ---------------------------------------------------------------- tensor maps, device facts, launches

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool load_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// Row-major (rows, D) bf16 matrix with row stride ld elements, boxes of
// 64 x box_rows, 128-byte swizzle, zero fill outside the matrix (ragged N, V
// and D).
bool encode_bf16_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t D, int64_t ld,
                      int box_rows) {
  cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
  cuuint32_t box[2] = {cuuint32_t(tc::BK), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct DeviceInfo {
  int sms = 0;
  int major = 0, minor = 0;
};

flce_status device_info(DeviceInfo& di) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&di.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&di.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FLCE_ERR_CUDA;
  // The kernels are built for sm_100a only (B200).
  if (di.major != 10 || di.minor != 0) return FLCE_ERR_UNSUPPORTED;
  return FLCE_OK;
}

// A kernel's dynamic shared-memory limit is a per-device setting: raise it
// once for each (kernel, device) pair, on the current device.
flce_status ensure_smem_limit(const void* fn, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& d : done)
    if (d.first == fn && d.second == dev) return FLCE_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return FLCE_ERR_CUDA;
  done.emplace_back(fn, dev);
  return FLCE_OK;
}

template <int L>
flce_status set_smem_limits_for() {
  flce_status s = ensure_smem_limit(reinterpret_cast<const void*>(tc::flce_tc_kernel<L>),
                                    tc::Cfg<L>::SMEM_BYTES);
  if (s != FLCE_OK) return s;
  return ensure_smem_limit(reinterpret_cast<const void*>(tc2::flce_tc2_kernel<L>),
                           tc2::Cfg<L>::SMEM_BYTES);
}

flce_status set_smem_limits() {
  flce_status s = set_smem_limits_for<tc::kPlain>();
  if (s == FLCE_OK) s = set_smem_limits_for<tc::kSplitW>();
  if (s == FLCE_OK) s = set_smem_limits_for<tc::kSplitHW>();
  if (s == FLCE_OK) s = set_smem_limits_for<tc::kPlain1>();
  return s;
}

// CTA pairs of the pair kernel that can be resident at once on the current
// device (queried once per device; SM count / 2 if the query is unavailable).
int64_t resident_pairs(int dev, int sms) {
  static std::mutex mu;
  static int cached[64] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(sms & ~1), 1, 1);
  cfg.blockDim = dim3(tc2::NUM_THREADS, 1, 1);
  // every layout of the pair kernel takes the same 192 KiB ring (one CTA per SM)
  cfg.dynamicSmemBytes = tc2::Cfg<tc::kPlain>::SMEM_BYTES;
  if (cudaOccupancyMaxActiveClusters(&n, tc2::flce_tc2_kernel<tc::kPlain>, &cfg) != cudaSuccess ||
      n < 1) {
    (void)cudaGetLastError();
    n = sms / 2;
  }
  n = std::min(n, sms / 2);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

flce_status check_forward_args(const void* H, const void* W, const int64_t* y, int64_t N,
                               int64_t V, int64_t D, flce_dtype dtype, const void* ws,
                               size_t ws_bytes) {
  if (!sizes_ok(N, V, D, dtype)) return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!H || !W || !y || !ws) return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FLCE_ERR_INVALID_ARG;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || D >= (int64_t(1) << 31))
    return FLCE_ERR_UNSUPPORTED;
  if (dtype == FLCE_BF16 && (D % 8 != 0 || !aligned16(H) || !aligned16(W)))
    return FLCE_ERR_UNSUPPORTED;
  if (dtype == FLCE_FP32 && ((reinterpret_cast<uintptr_t>(H) | reinterpret_cast<uintptr_t>(W)) & 3u))
    return FLCE_ERR_INVALID_ARG;
  if (dtype == FLCE_FP32 && k_extent(D, dtype) >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  if (ws_bytes < workspace_bytes_for(N, V, D, dtype)) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  return FLCE_OK;
}

// Device facts and the number of concurrent workers (CTAs or CTA pairs) the
// contraction kernel gets for N tokens; sets the kernels' shared-memory limit.
flce_status contraction_workers(int64_t N, DeviceInfo& di, int64_t& workers) {
  flce_status s = device_info(di);
  if (s != FLCE_OK) return s;
  if ((s = set_smem_limits()) != FLCE_OK) return s;
  workers = nominal_workers(di.sms, N);
  if (use_pair_kernel(N)) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
    workers = resident_pairs(dev, di.sms);
  }
  return FLCE_OK;
}

// The bf16 operands of one contraction: rows of H (N rows) and of W (V rows),
// `cols_*` columns stored with row stride `ld_*` elements.  The kernel runs
// `kblocks` pipeline stages per tile (tc::StageLayout): kPlain stages K
// blocks 2j and 2j + 1 (seg_* = 64, the next block), kPlain1 one K block
// (seg_* unused); in the split layouts the
// lo part of K block kb sits seg_* columns after its hi part in the same row:
// fp32 inputs split into [hi | lo] H and W rows (kSplitHW), a quantised head
// expanded into [hi | lo] W rows against H itself (kSplitW).
struct Operands {
  const void* H;
  int64_t ldh, cols_h, seg_h;
  const void* W;
  int64_t ldw, cols_w, seg_w;
  int64_t kblocks;
  int layout;        // tc::StageLayout
  int64_t h_rows;    // rows of the H buffer the tensor map covers; 0: N
};

// Batches of at most this many tokens stream W from HBM faster than the
// tensor cores consume it, so they run the one-K-block ring (tc::kPlain1);
// larger ones stage two K blocks per stage (tc::kPlain).  At V=151936
// D=4096 on B200 the one-block ring streamed W 2-6% faster at N = 1..256, and
// the two-block ring ran the N=8192 forward 6.5% faster.
constexpr int64_t kStreamBoundTokens = 256;

Operands bf16_operands(const void* H, int64_t ldh, const void* W, int64_t ldw, int64_t N,
                       int64_t D) {
  if (N <= kStreamBoundTokens)
    return Operands{H, ldh, D, 0, W, ldw, D, 0, cdiv(D, tc::BK), tc::kPlain1};
  return Operands{H, ldh, D, tc::BK, W, ldw, D, tc::BK, cdiv(D, 2 * tc::BK), tc::kPlain};
}

template <int L>
cudaError_t launch_contraction_kernel(bool pair, unsigned grid, const CUtensorMap& tmH,
                                      const CUtensorMap& tmW, const tc::Args& a, bool early,
                                      cudaStream_t st) {
  // early: programmatic serialization, so that the kernel's prologue and first
  // loads overlap the header-clearing kernel launched just before it
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(pair ? tc2::NUM_THREADS : tc::NUM_THREADS);
  cfg.dynamicSmemBytes = pair ? tc2::Cfg<L>::SMEM_BYTES : tc::Cfg<L>::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = early ? attr : nullptr;
  cfg.numAttrs = early ? 1 : 0;
  if (pair) return cudaLaunchKernelEx(&cfg, tc2::flce_tc2_kernel<L>, tmH, tmW, a);
  return cudaLaunchKernelEx(&cfg, tc::flce_tc_kernel<L>, tmH, tmW, a);
}

// ---- The partition-aware order of the pair kernel (tc::PartArgs) ----
//
// Which L2 partition each SM reads through is found once per device by two
// small kernels on the caller's stream, whose results the host waits for:
// dependent atomic adds from every SM to lines spread over memory (an add
// completes at the slice that homes its line, so each line shows a short
// latency from the SMs of its partition and a long one from the others), and
// a launch of as many CTA pairs as can be resident that records where they
// land.  Measured on B200: 266-272 against 708-773 cycles, SMs in two groups
// of 70 and 78 (74 and 74 on another GPU); N=8192 V=151936 D=4096 read 1.70
// GB from DRAM per launch in this order against 3.38 GB (same box, same
// call), and the results are bitwise those of the plain order.
constexpr int kPartLines = 64;
constexpr int kPartLineWords = 4096;  // lines 16 KiB apart
constexpr size_t kPartLinesBytes = size_t(kPartLines) * kPartLineWords * 4;
constexpr int kPartMaxSms = 256;
constexpr size_t kPartCalBytes =
    kPartLinesBytes + size_t(kPartMaxSms) * kPartLines * 4 + size_t(2 * kPartMaxSms + 2) * 4;
// Units per pair below which the order is not used: each side's share of the
// units is rounded, so a side may run one unit more per pair than the plain
// order (N=2048 V=32000 D=1024, one unit per pair, ran 66% slower).
constexpr int64_t kPartMinUnitsPerPair = 16;
// Each partition's rows of H (bf16 bytes) must stay well inside its half of
// the L2 beside the W tiles in flight.
constexpr int64_t kPartHBytes = 40ll << 20;
// The order's two pair counters sit in the workspace header, after WsHeader.
constexpr size_t kPartRegOffset = 128;
static_assert(sizeof(WsHeader) <= kPartRegOffset && kPartRegOffset + 8 <= kHeaderBytes, "header");

struct PartMap {
  bool tried = false, ok = false;
  int32_t npairs = 0;       // pairs resident when the map was taken
  int32_t pairs[2] = {0, 0};
  uint8_t side[kPartMaxSms] = {};
};
std::mutex g_part_mu;
PartMap g_part_map[64];

// Takes the map of the current device (first kPartCalBytes of `ws` as
// scratch, on `st`, waiting for the result).  Leaves m.ok false when the
// latencies do not fall into two clear groups.
void calibrate_partitions(int sms, int npairs, uint8_t* ws, cudaStream_t st, PartMap& m) {
  m.tried = true;
  if (sms > kPartMaxSms || npairs < 2) return;
  const int smem = tc2::Cfg<tc::kPlain>::SMEM_BYTES;
  if (ensure_smem_limit(reinterpret_cast<const void*>(tc2::flce_part_latency_kernel), smem) !=
          FLCE_OK ||
      ensure_smem_limit(reinterpret_cast<const void*>(tc2::flce_part_cluster_kernel), smem) != FLCE_OK)
    return;
  uint32_t* lines = reinterpret_cast<uint32_t*>(ws);
  uint32_t* lat = reinterpret_cast<uint32_t*>(ws + kPartLinesBytes);
  int32_t* smid_blk = reinterpret_cast<int32_t*>(lat + size_t(kPartMaxSms) * kPartLines);
  int32_t* smid_pair = smid_blk + kPartMaxSms;
  uint32_t* ctr = reinterpret_cast<uint32_t*>(smid_pair + kPartMaxSms);  // arrived, timed out
  if (cudaMemsetAsync(ws, 0, kPartCalBytes, st) != cudaSuccess) return;
  tc2::flce_part_latency_kernel<<<unsigned(sms), 32, smem, st>>>(lines, kPartLines, kPartLineWords,
                                                                  lat, smid_blk);
  tc2::flce_part_cluster_kernel<<<unsigned(2 * npairs), 32, smem, st>>>(smid_pair, ctr, ctr + 1);
  std::vector<uint32_t> hl;
  std::vector<int32_t> hb, hp;
  hl.resize(size_t(sms) * kPartLines);
  hb.resize(size_t(sms));
  hp.resize(size_t(npairs));
  uint32_t hc[2] = {0, 0};
  if (cudaGetLastError() != cudaSuccess ||
      cudaMemcpyAsync(hl.data(), lat, hl.size() * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(hb.data(), smid_blk, hb.size() * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(hp.data(), smid_pair, hp.size() * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(hc, ctr, 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return;
  }
  if (hc[1] != 0) return;  // not every pair could be resident at once
  // near (0) or far (1) per block and line, for the lines whose latencies split
  // clearly (the longest at least 1.5 x the shortest)
  std::vector<int> usable;
  std::vector<uint8_t> far(hl.size());
  for (int l = 0; l < kPartLines; ++l) {
    uint32_t lo = ~0u, hi = 0;
    for (int b = 0; b < sms; ++b) {
      lo = std::min(lo, hl[size_t(b) * kPartLines + l]);
      hi = std::max(hi, hl[size_t(b) * kPartLines + l]);
    }
    if (lo == 0 || uint64_t(hi) * 2 < uint64_t(lo) * 3) continue;
    usable.push_back(l);
    for (int b = 0; b < sms; ++b)
      far[size_t(b) * kPartLines + l] = uint64_t(hl[size_t(b) * kPartLines + l]) * 2 > uint64_t(lo) + hi;
  }
  if (usable.size() < 16) return;
  uint8_t side[kPartMaxSms] = {};
  bool seen[kPartMaxSms] = {};
  for (int b = 0; b < sms; ++b) {
    int agree = 0;
    for (int l : usable) agree += far[size_t(b) * kPartLines + l] == far[l];
    const int n = int(usable.size());
    if (agree * 10 > n && agree * 10 < 9 * n) return;  // neither side clearly
    const int sm = hb[size_t(b)];
    if (sm < 0 || sm >= kPartMaxSms) return;
    const uint8_t sd = agree * 2 > n ? 0 : 1;
    if (seen[sm] && side[sm] != sd) return;
    side[sm] = sd;
    seen[sm] = true;
  }
  int32_t pairs[2] = {0, 0};
  for (int p = 0; p < npairs; ++p) {
    const int sm = hp[size_t(p)];
    if (sm < 0 || sm >= kPartMaxSms) return;
    ++pairs[side[sm]];
  }
  if (pairs[0] == 0 || pairs[1] == 0) return;
  std::memcpy(m.side, side, sizeof(side));
  m.pairs[0] = pairs[0];
  m.pairs[1] = pairs[1];
  m.npairs = npairs;
  m.ok = true;
}

// Whether a forward with this plan gains from the partition order: the pair
// kernel with kPartMinUnitsPerPair units per pair, and more token blocks than
// one raster group holds, so that the plain order streams W more than once
// (N=8192 V=40000 D=128, a single group, ran 4% slower in the partition
// order).
bool part_order_sized(const flce_plan_t& plan) {
  const int64_t npairs = plan.grid / 2;
  return plan.ctas_per_unit == 2 && npairs >= 2 && plan.units >= kPartMinUnitsPerPair * npairs &&
         plan.token_blocks > plan.group_blocks;
}

// Takes the current device's map at the first forward sized for the order,
// unless `st` is being captured into a graph (then that forward and the ones
// after it use the plain order until one runs outside a capture).
void maybe_calibrate(const flce_plan_t& plan, int sms, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!part_order_sized(plan) || ws_bytes < kPartCalBytes) return;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return;
  std::lock_guard<std::mutex> lock(g_part_mu);
  if (g_part_map[dev].tried) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    (void)cudaGetLastError();
    return;
  }
  calibrate_partitions(sms, int(plan.grid / 2), static_cast<uint8_t*>(ws), st, g_part_map[dev]);
}

// The partition order for this launch, if the device's map allows it: the
// split (q, r) gives partition 0 its pairs' share of the units.
bool part_order(const flce_plan_t& plan, int64_t D, uint32_t* reg, tc::PartArgs& pa) {
  if (!part_order_sized(plan)) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  PartMap m;
  {
    std::lock_guard<std::mutex> lock(g_part_mu);
    m = g_part_map[dev];
  }
  const int64_t npairs = plan.grid / 2;
  if (!m.ok || m.npairs != npairs) return false;
  const int64_t U = plan.units, P = plan.slabs, TB = plan.token_blocks;
  const int64_t u0 = (U * m.pairs[0] + npairs / 2) / npairs;
  if (u0 <= 0 || u0 >= U) return false;
  const int64_t q = u0 / P, r = u0 % P;
  const int64_t blocks = std::max<int64_t>(q + (r > 0 ? 1 : 0), TB - q);
  if (blocks * plan.block_rows * D * 2 > kPartHBytes) return false;
  pa.reg = reg;
  pa.pairs[0] = m.pairs[0];
  pa.pairs[1] = m.pairs[1];
  pa.q = int32_t(q);
  pa.r = int32_t(r);
  std::memcpy(pa.side, m.side, sizeof(pa.side));
  return true;
}

// Outputs of the merge when it runs inside the contraction kernel (the whole
// forward in one launch); see tc::fused_merge.
struct MergeOutputs {
  float* loss;
  float* lse;
  float* mean;  // may be null
  float* sum;   // may be null
};

// Who clears the workspace header (status word) and the row-block counters
// (the first state_layout().part bytes) before the contraction: a one-block
// kernel launched here, which the contraction overlaps (programmatic launch);
// the kernel launched just before that writes the operands (the fp32 split
// or the tiny-batch H copy, which clear them in their first block; the
// contraction overlaps it too and its producer waits for it); or nobody (a
// chunk of a chunked call, whose caller cleared the header once).
enum class HeaderReset { kHere, kDoneBefore, kNone };

// The contraction with the online (m, s) epilogue.  Writes (m, s) per (slab,
// token) into the workspace's state and the target logits W owns; with
// `merged` also the merged loss, lse, mean and sum (then y_offset must be 0,
// V the whole vocabulary, and the header and counters cleared for this call).
flce_status launch_contraction(const Operands& op, Targets y, int64_t y_offset, int64_t N,
                               int64_t V, const flce_plan_t& plan, float* out_target, void* ws,
                               HeaderReset reset, cudaStream_t st,
                               const MergeOutputs* merged = nullptr) {
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
  const StateLayout L = state_layout(N, V);
  float2* part = reinterpret_cast<float2*>(wsb + L.part);
  if (merged != nullptr && (reset == HeaderReset::kNone || y_offset != 0)) return FLCE_ERR_INVALID_ARG;
  if (reset == HeaderReset::kHere) {
    split::flce_clear_header_kernel<<<1, 128, 0, st>>>(reinterpret_cast<uint32_t*>(hdr),
                                                       int32_t(L.part / 4));
    if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  }

  Schedule sch;
  sch.token_blocks = int32_t(plan.token_blocks);
  sch.slabs = plan.slabs;
  sch.slab_base = plan.slab_base;
  sch.slab_rem = plan.slab_rem;
  sch.units = int32_t(plan.units);
  sch.group_blocks = plan.group_blocks;

  if (!load_encoder()) return FLCE_ERR_CUDA;
  const bool pair = plan.ctas_per_unit == 2;
  CUtensorMap tmH, tmW;
  if (!encode_bf16_rows(&tmH, op.H, op.h_rows > 0 ? op.h_rows : N, op.cols_h, op.ldh, tc::BM) ||
      !encode_bf16_rows(&tmW, op.W, V, op.cols_w, op.ldw, pair ? tc2::HALF_N : tc::BN))
    return FLCE_ERR_UNSUPPORTED;
  tc::Args a;
  a.y = y;
  a.y_offset = y_offset;
  a.part = part;
  a.target_logit = out_target;
  a.hdr = hdr;
  a.N = int32_t(N);
  a.V = int32_t(V);
  a.D = int32_t(op.kblocks * tc::BK);
  a.kblocks = int32_t(op.kblocks);
  a.seg_h = int32_t(op.seg_h);
  a.seg_w = int32_t(op.seg_w);
  a.sch = sch;
  a.wait_limit_ns = kDefaultWaitLimitNs;
  a.fm = tc::FusedMerge{};
  a.porder.reg = nullptr;
  // the partition order needs its pair counters cleared by this call
  if (reset != HeaderReset::kNone &&
      !part_order(plan, op.cols_h, reinterpret_cast<uint32_t*>(wsb + kPartRegOffset), a.porder))
    a.porder.reg = nullptr;
  if (merged != nullptr) {
    a.fm.arrivals = reinterpret_cast<uint32_t*>(wsb + L.counters);
    a.fm.loss = merged->loss;
    a.fm.lse = merged->lse;
    a.fm.mean = merged->mean;
    a.fm.sum = merged->sum;
    a.fm.block_sums = reinterpret_cast<double*>(wsb + L.sums);
    a.fm.row_blocks = int32_t(plan.token_blocks * plan.ctas_per_unit);
  }
  const unsigned grid = unsigned(plan.grid);
  // Launched to overlap the kernel before it: the header clear (which it
  // waits for before touching the header), or the split / padded copy of the
  // operands (which the producer waits for before its first load).
  const bool early = reset == HeaderReset::kHere || reset == HeaderReset::kDoneBefore;
  a.wait_operands = reset == HeaderReset::kDoneBefore ? 1 : 0;
  cudaError_t e;
  switch (op.layout) {
    case tc::kPlain:
      e = launch_contraction_kernel<tc::kPlain>(pair, grid, tmH, tmW, a, early, st);
      break;
    case tc::kSplitW:
      e = launch_contraction_kernel<tc::kSplitW>(pair, grid, tmH, tmW, a, early, st);
      break;
    case tc::kSplitHW:
      e = launch_contraction_kernel<tc::kSplitHW>(pair, grid, tmH, tmW, a, early, st);
      break;
    case tc::kPlain1:
      e = launch_contraction_kernel<tc::kPlain1>(pair, grid, tmH, tmW, a, early, st);
      break;
    default: return FLCE_ERR_INVALID_ARG;
  }
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

// fp32 inputs: split `src` (rows, D; row stride ld) into its bf16 (rows,
// nseg Dp) copy at `dst`: lo in segment lo_segment, hi in the others.  With
// src2 (rows2 rows, row stride ld2, copy at dst2) a second matrix of the same
// D is split in the same launch.  rows_out > rows: the first copy gets zero
// rows after the source rows, up to rows_out.
flce_status launch_split(const void* src, int64_t ld, int64_t rows, int64_t D, int64_t Dp,
                         int nseg, int lo_segment, void* dst, int sms, cudaStream_t st,
                         const void* src2 = nullptr, int64_t ld2 = 0, int64_t rows2 = 0,
                         void* dst2 = nullptr, int64_t rows_out = 0, void* zero = nullptr,
                         size_t zero_bytes = 0) {
  split::Args a;
  a.src = static_cast<const float*>(src);
  a.ld = ld;
  a.rows = rows;
  a.D = int32_t(D);
  a.Dp = int32_t(Dp);
  a.nseg = nseg;
  a.lo_segment = lo_segment;
  a.dst = static_cast<__nv_bfloat16*>(dst);
  a.src_rows = rows;
  if (rows_out > rows) a.rows = rows_out;  // zero rows after the source rows
  a.zero = static_cast<uint32_t*>(zero);
  a.zero_words = int32_t(zero_bytes / 4);
  split::Args b = a;
  b.src = static_cast<const float*>(src2);
  b.ld = ld2;
  b.rows = src2 != nullptr ? rows2 : 0;
  b.src_rows = b.rows;
  b.dst = static_cast<__nv_bfloat16*>(dst2);
  b.zero = nullptr;
  b.zero_words = 0;
  const int64_t warps_per_block = split::NUM_THREADS / 32;
  const int64_t blocks = std::max<int64_t>(
      1, std::min<int64_t>(cdiv(a.rows + b.rows, warps_per_block), int64_t(sms) * 8));
  const bool vec = D % 8 == 0 && ld % 4 == 0 && aligned16(src) &&
                   (b.rows == 0 || (ld2 % 4 == 0 && aligned16(src2)));
  if (vec)
    split::flce_split3_kernel<true><<<unsigned(blocks), split::NUM_THREADS, 0, st>>>(a, b);
  else
    split::flce_split3_kernel<false><<<unsigned(blocks), split::NUM_THREADS, 0, st>>>(a, b);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

// bf16 H of a batch of fewer than kMinHRows tokens, copied with zero rows up to
// kMinHRows into `dst` (kMinHRows x D, contiguous); see kMinHRows.
// `zero` (zero_bytes, a multiple of 4, may be null) is cleared by the same launch.
flce_status launch_pad_h(const void* H, int64_t ldh, int64_t N, int64_t D, void* dst, int sms,
                         cudaStream_t st, void* zero = nullptr, size_t zero_bytes = 0) {
  const int64_t nvec = kMinHRows * (D / 8);
  split::flce_pad_rows_kernel<<<unsigned(std::min<int64_t>(cdiv(nvec, 256), 4 * int64_t(sms))), 256,
                                0, st>>>(static_cast<const uint4*>(H), ldh / 8, int32_t(N),
                                         int32_t(D / 8), int32_t(kMinHRows),
                                         static_cast<uint4*>(dst), static_cast<uint32_t*>(zero),
                                         int32_t(zero_bytes / 4));
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

// Stage 1 of the forward for bf16 or fp32 H and W (fp32: split first); with
// `merged`, the whole forward (the merge runs inside the contraction kernel).
flce_status launch_partials(const void* H, int64_t ldh, const void* W, int64_t ldw, Targets y,
                            int64_t y_offset, int64_t N, int64_t V, int64_t D, flce_dtype dtype,
                            float* out_target, void* ws, cudaStream_t st,
                            const MergeOutputs* merged = nullptr) {
  DeviceInfo di;
  int64_t workers = 0;
  flce_status s = contraction_workers(N, di, workers);
  if (s != FLCE_OK) return s;
  flce_plan_t plan;
  make_plan(N, V, D, dtype, workers, &plan);
  // the first forward of this size on the device maps its L2 partitions
  maybe_calibrate(plan, di.sms, ws, state_layout(N, V).total, st);

  // The operands the tensor-core kernels read: H and W themselves (bf16), or
  // their [hi | lo] split copies in the workspace (fp32), each K block's four
  // parts staged together for the three products hi hi + hi lo + lo hi.
  Operands op = bf16_operands(H, ldh, W, ldw, N, D);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  // the header and counters: cleared by the kernel that runs first in this call
  HeaderReset reset = HeaderReset::kHere;
  const size_t reset_bytes = state_layout(N, V).part;
  if (dtype == FLCE_FP32) {
    const int64_t Dp = fwd_split_segment(D);
    uint8_t* hs = wsb + state_bytes_for(N, V);
    uint8_t* wsplit = hs + fwd_split_h_bytes(N, D);
    // H (padded with zero rows up to kMinHRows) and W in one launch
    if ((s = launch_split(H, ldh, N, D, Dp, 2, 1, hs, di.sms, st, W, ldw, V, wsplit,
                          padded_h_rows(N), wsb, reset_bytes)) != FLCE_OK)
      return s;
    reset = HeaderReset::kDoneBefore;
    op = Operands{hs, 2 * Dp, 2 * Dp, Dp, wsplit, 2 * Dp, 2 * Dp, Dp, Dp / tc::BK, tc::kSplitHW,
                  padded_h_rows(N)};
  } else if (N < kMinHRows) {
    // a tiny batch: H read from a copy padded with zero rows (kMinHRows)
    uint8_t* hp = wsb + state_bytes_for(N, V);
    if ((s = launch_pad_h(H, ldh, N, D, hp, di.sms, st, wsb, reset_bytes)) != FLCE_OK) return s;
    reset = HeaderReset::kDoneBefore;
    op.H = hp;
    op.ldh = D;
    op.h_rows = kMinHRows;
  }
  return launch_contraction(op, y, y_offset, N, V, plan, out_target, ws, reset, st, merged);
}

flce_status launch_merge(Targets y, int64_t N, int64_t V, float* out_loss, float* out_lse,
                         float* out_target, float* out_mean, float* out_sum, const void* ws,
                         size_t ws_bytes,
                         cudaStream_t st) {
  uint8_t* wsb = static_cast<uint8_t*>(const_cast<void*>(ws));
  const StateLayout L = state_layout(N, V);
  MergeArgs m;
  m.hdr = reinterpret_cast<WsHeader*>(wsb);
  m.part = reinterpret_cast<const float2*>(wsb + L.part);
  m.block_sums = reinterpret_cast<double*>(wsb + L.sums);
  m.y = y;
  m.target_logit = out_target;
  m.loss = out_loss;
  m.lse = out_lse;
  m.mean = out_mean;
  m.sum = out_sum;
  m.N = int32_t(N);
  m.V = int32_t(V);
  m.max_slabs = int32_t(slab_capacity(V));
  (void)ws_bytes;
  const int blocks = int(cdiv(N, kMergeTokensPerBlock));
  flce_merge_kernel<<<blocks, kMergeBlockThreads, 0, st>>>(m);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t flce_workspace_size(int64_t N, int64_t V, int64_t D, flce_dtype dtype) {
  if (!sizes_ok(N, V, D, dtype)) return 0;
  return workspace_bytes_for(N, V, D, dtype);
}

flce_status flce_plan(int64_t N, int64_t V, int64_t D, flce_dtype dtype, int32_t sm_count,
                      flce_plan_t* plan) {
  if (!plan || sm_count < 1 || !sizes_ok(N, V, D, dtype)) return FLCE_ERR_INVALID_ARG;
  return make_plan(N, V, D, dtype, nominal_workers(sm_count, N), plan);
}

flce_status flce_partials(const void* H, const void* W, const int64_t* y, int64_t N, int64_t V,
                          int64_t D, flce_dtype dtype, float* out_target_logit, void* workspace,
                          size_t workspace_bytes, void* stream) {
  FLCE_TRACE();
  flce_status s = check_forward_args(H, W, y, N, V, D, dtype, workspace, workspace_bytes);
  if (s != FLCE_OK || N == 0) return s;
  if (!out_target_logit) return FLCE_ERR_INVALID_ARG;
  return launch_partials(H, D, W, D, Targets{y, 0}, 0, N, V, D, dtype, out_target_logit, workspace,
                         static_cast<cudaStream_t>(stream));
}

flce_status flce_merge(const int64_t* y, int64_t N, int64_t V, float* out_loss, float* out_lse,
                       float* out_target_logit, float* out_mean, const void* workspace,
                       size_t workspace_bytes, void* stream) {
  FLCE_TRACE();
  if (N < 0 || V < 1) return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!y || !out_loss || !out_lse || !out_target_logit || !workspace) return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FLCE_ERR_INVALID_ARG;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < state_bytes_for(N, V)) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  return launch_merge(Targets{y, 0}, N, V, out_loss, out_lse, out_target_logit, out_mean, nullptr,
                      workspace,
                      workspace_bytes, static_cast<cudaStream_t>(stream));
}

flce_status flce_forward(const void* H, const void* W, const int64_t* y, int64_t N, int64_t V,
                         int64_t D, flce_dtype dtype, float* out_loss, float* out_lse,
                         float* out_target_logit, float* out_mean, void* workspace,
                         size_t workspace_bytes, void* stream) {
  FLCE_TRACE();
  flce_status s = check_forward_args(H, W, y, N, V, D, dtype, workspace, workspace_bytes);
  if (s != FLCE_OK || N == 0) return s;
  if (!out_loss || !out_lse || !out_target_logit) return FLCE_ERR_INVALID_ARG;
  // one launch: the merge runs in the contraction kernel's epilogue
  const MergeOutputs merged{out_loss, out_lse, out_mean, nullptr};
  return launch_partials(H, D, W, D, Targets{y, 0}, 0, N, V, D, dtype, out_target_logit, workspace,
                         static_cast<cudaStream_t>(stream), &merged);
}

flce_status flce_forward_ex(const flce_forward_args* a, void* workspace, size_t workspace_bytes,
                            void* stream) {
  FLCE_TRACE();
  if (!a) return FLCE_ERR_INVALID_ARG;
  const flce_dtype dtype = flce_dtype(a->dtype);
  if (!sizes_ok(a->N, a->V, a->D, dtype)) return FLCE_ERR_INVALID_ARG;
  if (a->y_dtype != FLCE_INDEX_INT64 && a->y_dtype != FLCE_INDEX_INT32) return FLCE_ERR_INVALID_ARG;
  const int64_t ldh = a->ldh == 0 ? a->D : a->ldh;
  const int64_t ldw = a->ldw == 0 ? a->D : a->ldw;
  if (ldh < a->D || ldw < a->D) return FLCE_ERR_INVALID_ARG;
  if (dtype == FLCE_BF16 && (ldh % 8 != 0 || ldw % 8 != 0)) return FLCE_ERR_UNSUPPORTED;
  flce_status s = check_forward_args(a->H, a->W, static_cast<const int64_t*>(a->y), a->N, a->V,
                                     a->D, dtype, workspace, workspace_bytes);
  if (s != FLCE_OK || a->N == 0) return s;
  if (!a->out_loss || !a->out_lse || !a->out_target_logit) return FLCE_ERR_INVALID_ARG;
  if (ldh >= (int64_t(1) << 31) || ldw >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Targets y{a->y, a->y_dtype == FLCE_INDEX_INT32 ? 1 : 0};
  const MergeOutputs merged{a->out_loss, a->out_lse, a->out_mean, a->out_sum};
  return launch_partials(a->H, ldh, a->W, ldw, y, 0, a->N, a->V, a->D, dtype, a->out_target_logit,
                         workspace, st, &merged);
}

flce_status flce_partials_shard(const void* H, const void* W_shard, const int64_t* y, int64_t N,
                                int64_t V_shard, int64_t v_offset, int64_t D, flce_dtype dtype,
                                float* out_target_logit, void* workspace, size_t workspace_bytes,
                                void* stream) {
  FLCE_TRACE();
  if (v_offset < 0) return FLCE_ERR_INVALID_ARG;
  flce_status s =
      check_forward_args(H, W_shard, y, N, V_shard, D, dtype, workspace, workspace_bytes);
  if (s != FLCE_OK || N == 0) return s;
  if (!out_target_logit) return FLCE_ERR_INVALID_ARG;
  return launch_partials(H, D, W_shard, D, Targets{y, 0}, v_offset, N, V_shard, D, dtype,
                         out_target_logit,
                         workspace, static_cast<cudaStream_t>(stream));
}

flce_status flce_shard_state(const int64_t* y, int64_t N, int64_t V_shard, int64_t v_offset,
                             const float* target_logit, const void* workspace,
                             size_t workspace_bytes, float* out_state, void* stream) {
  FLCE_TRACE();
  if (N < 0 || V_shard < 1 || v_offset < 0) return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!y || !target_logit || !workspace || !out_state) return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(out_state) & 15u) != 0)
    return FLCE_ERR_INVALID_ARG;
  if (N >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < state_bytes_for(N, V_shard)) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  const uint8_t* wsb = static_cast<const uint8_t*>(workspace);
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(wsb);
  flce_shard_state_kernel<<<unsigned(cdiv(N, kMergeThreads)), kMergeThreads, 0,
                            static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float2*>(wsb + state_layout(N, V_shard).part), hdr, y, int32_t(N),
      v_offset, V_shard,
      int32_t(slab_capacity(V_shard)), target_logit, reinterpret_cast<float4*>(out_state),
      const_cast<uint32_t*>(&hdr->status));
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

size_t flce_merge_shards_scratch_size(int64_t N) {
  if (N < 0) return 0;
  return kHeaderBytes + align256(size_t(8) * size_t(std::max<int64_t>(1, cdiv(N, kMergeThreads))));
}

flce_status flce_merge_shards(const float* states, int32_t G, const int64_t* y, int64_t N,
                              int64_t V_total, float* out_loss, float* out_lse,
                              float* out_target_logit, float* out_mean, float* out_sum,
                              void* scratch,
                              size_t scratch_bytes, void* stream) {
  FLCE_TRACE();
  if (G < 1 || N < 0 || V_total < 1) return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!states || !y || !out_loss || !out_lse || !out_target_logit || !scratch)
    return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(states) & 15u) != 0)
    return FLCE_ERR_INVALID_ARG;
  if (N >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  if (scratch_bytes < flce_merge_shards_scratch_size(N)) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* sb = static_cast<uint8_t*>(scratch);
  if (cudaMemsetAsync(sb, 0, kHeaderBytes, st) != cudaSuccess) return FLCE_ERR_CUDA;
  flce_merge_shards_kernel<<<unsigned(cdiv(N, kMergeThreads)), kMergeThreads, 0, st>>>(
      reinterpret_cast<const float4*>(states), G, y, int32_t(N), V_total, out_loss, out_lse,
      out_target_logit, out_mean, out_sum, reinterpret_cast<double*>(sb + kHeaderBytes),
      reinterpret_cast<WsHeader*>(sb));
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

flce_status flce_check(const void* workspace, void* stream) {
  if (!workspace) return FLCE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLCE_ERR_CUDA;
  uint32_t status = 0;
  if (cudaMemcpy(&status, workspace, sizeof(status), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FLCE_ERR_CUDA;
  if (status & kStatTimeout) return FLCE_ERR_TIMEOUT;
  if (status & kStatTarget) return FLCE_ERR_TARGET_OUT_OF_RANGE;
  if (status & kStatBadWs) return FLCE_ERR_INVALID_ARG;
  return FLCE_OK;
}

const char* flce_status_string(flce_status status) {
  switch (status) {
    case FLCE_OK: return "ok";
    case FLCE_ERR_INVALID_ARG: return "invalid argument";
    case FLCE_ERR_UNSUPPORTED: return "unsupported device, shape or alignment";
    case FLCE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case FLCE_ERR_CUDA: return "CUDA error";
    case FLCE_ERR_TARGET_OUT_OF_RANGE: return "target outside [0, V)";
    case FLCE_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

flce_status flce_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint64_t limit_ns,
                                       void* stream) {
  if (!workspace || workspace_bytes < kHeaderBytes) return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FLCE_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 1000000000ull) return FLCE_ERR_INVALID_ARG;
  DeviceInfo di;
  flce_status s = device_info(di);
  if (s != FLCE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, st) != cudaSuccess) return FLCE_ERR_CUDA;
  flce_wait_probe_kernel<<<1, 32, 0, st>>>(static_cast<WsHeader*>(workspace), limit_ns);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------- backward

namespace {

// Vocabulary rows per backward chunk.  bf16: 32768 halves the launches and
// the read-modify-write passes over dH against 16384, 1-2% faster at N=8192
// V=151936 D=4096 (dZ slice 0.54 GB there).  fp32 inputs and the quantised
// head also hold a split or expanded copy of each W chunk; for them 16384
// measured as fast or faster (fp32: 0.6-1.7%) with half the workspace.
constexpr int64_t kBwdChunkCols = 32768;
constexpr int64_t kBwdChunkColsSplit = 16384;

inline int64_t round_up(int64_t x, int64_t m) { return cdiv(x, m) * m; }

struct BwdLayout {
  int64_t chunk;
  size_t off_dz, off_dzl, off_h3, off_w3, total;
};

// bf16: [256 B header][dZ slice: N x chunk bf16].
// fp32 inputs add the lo parts of the dZ slice (N x chunk bf16) and the bf16
// hi/lo split copies of H (N x 3 Dp, [hi | hi | lo]) and of one chunk of W
// (chunk x 3 Dp, [hi | lo | hi]).
BwdLayout bwd_layout(int64_t N, int64_t V, int64_t D, flce_dtype dtype) {
  BwdLayout L;
  L.chunk = std::min(round_up(V, kTileCols),
                     dtype == FLCE_FP32 ? kBwdChunkColsSplit : kBwdChunkCols);
  L.off_dz = kHeaderBytes;
  size_t end = L.off_dz + align256(size_t(N) * size_t(L.chunk) * 2);
  L.off_dzl = L.off_h3 = L.off_w3 = 0;
  if (dtype == FLCE_FP32) {
    L.off_dzl = end;
    end += align256(size_t(N) * size_t(L.chunk) * 2);
    L.off_h3 = end;
    end += bwd_split_bytes_for(N, D);
    L.off_w3 = end;
    end += bwd_split_bytes_for(L.chunk, D);
  }
  L.total = end;
  return L;
}

// Row-major bf16 matrix (rows x cols, row stride ld elements) as a TMA map
// with 64 (cols) x box_rows boxes, 128-byte swizzle and zero fill outside.
// K-major operands use box_rows = 128 (operand rows per CTA); MN-major
// operands use box_rows = 64 (K rows per stage).
bool encode_bf16_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                    int box_rows) {
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
  cuuint32_t box[2] = {cuuint32_t(bwd::BK), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bwd::GemmShape gemm_shape(int64_t M, int64_t Nc, int64_t K) {
  bwd::GemmShape g;
  g.M = int32_t(M);
  g.N = int32_t(Nc);
  g.K = int32_t(K);
  g.tiles_m = int32_t(cdiv(M, bwd::PAIR_M));
  g.tiles_n = int32_t(cdiv(Nc, bwd::BN));
  // keep about 32 MB of A live per raster group
  g.group_m = int32_t(std::max<int64_t>(
      1, std::min<int64_t>(g.tiles_m, kGroupHBytes / std::max<int64_t>(1, bwd::PAIR_M * K * 2))));
  g.tiles = g.tiles_m * g.tiles_n;
  g.kblocks = int32_t(cdiv(K, bwd::BK));
  g.kblocks_a = g.kblocks;
  return g;
}

template <class Epi, bool kAmn, bool kBmn>
flce_status launch_gemm(const CUtensorMap& A, const CUtensorMap& B, const bwd::GemmShape& g,
                        const Epi& epi, uint32_t* status, int64_t pairs, cudaStream_t st) {
  flce_status s = ensure_smem_limit(
      reinterpret_cast<const void*>(bwd::gemm_pair_kernel<Epi, kAmn, kBmn>), bwd::SMEM_BYTES);
  if (s != FLCE_OK) return s;
  const int grid = int(2 * std::min<int64_t>(pairs, g.tiles));
  bwd::gemm_pair_kernel<Epi, kAmn, kBmn><<<grid, bwd::NUM_THREADS, bwd::SMEM_BYTES, st>>>(
      A, B, g, epi, status, kDefaultWaitLimitNs);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

}  // namespace

extern "C" flce_status flce_partition_order(int32_t token_blocks, int32_t slabs,
                                            int32_t side0_units, int32_t* out) {
  if (token_blocks < 1 || slabs < 1 || out == nullptr ||
      int64_t(token_blocks) * slabs >= (int64_t(1) << 30) || side0_units < 0 ||
      side0_units > token_blocks * slabs)
    return FLCE_ERR_INVALID_ARG;
  Schedule s{};
  s.token_blocks = token_blocks;
  s.slabs = slabs;
  s.units = token_blocks * slabs;
  const int32_t q = side0_units / slabs, r = side0_units % slabs;
  int64_t o = 0;
  for (int side = 0; side < 2; ++side)
    for (int k = 0; k < part_units(s, q, r, side); ++k) {
      int slab = 0, tb = 0;
      part_unit(s, q, r, side, k, slab, tb);
      out[o++] = slab;
      out[o++] = tb;
    }
  return FLCE_OK;
}

extern "C" flce_status flce_partition_map(int32_t* out_pairs) {
  if (out_pairs == nullptr) return FLCE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FLCE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_part_mu);
  const PartMap& m = g_part_map[dev];
  if (!m.ok) return FLCE_ERR_UNSUPPORTED;
  out_pairs[0] = m.pairs[0];
  out_pairs[1] = m.pairs[1];
  return FLCE_OK;
}

extern "C" flce_status flce_partition_take(int32_t pairs0, int32_t pairs1, int32_t side,
                                           int32_t arrival, int32_t* out_side,
                                           int32_t* out_rank) {
  if (pairs0 < 1 || pairs1 < 1 || (side != 0 && side != 1) || arrival < 0 ||
      arrival >= pairs0 + pairs1 || out_side == nullptr || out_rank == nullptr)
    return FLCE_ERR_INVALID_ARG;
  const int32_t pairs[2] = {pairs0, pairs1};
  int sd = side, rank = arrival;
  part_take(pairs, sd, rank);
  *out_side = sd;
  *out_rank = rank;
  return FLCE_OK;
}

extern "C" size_t flce_backward_workspace_size(int64_t N, int64_t V, int64_t D, flce_dtype dtype) {
  if (!sizes_ok(N, V, D, dtype) || N < 1) return 0;
  return bwd_layout(N, V, D, dtype).total;
}

namespace {

// The backward over W's rows [0, V) (a whole head, or one vocabulary shard
// whose first row is vocabulary id y_offset of a V_total-word vocabulary).
flce_status backward_impl(const void* H, const void* W, const int64_t* y, const float* lse,
                          const float* grad_loss, float grad_scale, int64_t N, int64_t V,
                          int64_t y_offset, int64_t V_total, int64_t D, flce_dtype dtype,
                          float* dH, float* dW, void* workspace, size_t workspace_bytes,
                          void* stream, cudaEvent_t dh_ready) {
  if (!sizes_ok(N, V, D, dtype)) return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!H || !W || !y || !lse || !dH || !dW || !workspace) return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FLCE_ERR_INVALID_ARG;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || D >= (int64_t(1) << 31))
    return FLCE_ERR_UNSUPPORTED;
  const bool fp32 = dtype == FLCE_FP32;
  if (!fp32 && (D % 8 != 0 || !aligned16(H) || !aligned16(W))) return FLCE_ERR_UNSUPPORTED;
  if (fp32 && ((reinterpret_cast<uintptr_t>(H) | reinterpret_cast<uintptr_t>(W)) & 3u))
    return FLCE_ERR_INVALID_ARG;
  if (fp32 && k_extent(D, dtype) >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  const BwdLayout L = bwd_layout(N, V, D, dtype);
  if (workspace_bytes < L.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;

  DeviceInfo di;
  flce_status s = device_info(di);
  if (s != FLCE_OK) return s;
  if (!load_encoder()) return FLCE_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if ((s = set_smem_limits()) != FLCE_OK) return s;
  const int64_t pairs = resident_pairs(dev, di.sms);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(ws + L.off_dz);  // (N x chunk)
  __nv_bfloat16* dzl = fp32 ? reinterpret_cast<__nv_bfloat16*>(ws + L.off_dzl) : nullptr;
  if (cudaMemsetAsync(hdr, 0, kHeaderBytes, st) != cudaSuccess) return FLCE_ERR_CUDA;

  // The bf16 operands.  bf16 inputs: H and W themselves.  fp32 inputs: the
  // split copies, K1 contracting [hi | hi | lo] against [hi | lo | hi] over
  // K = 3 Dp; K2 and K3 read the hi and lo segments as strided views.
  const int64_t Dp = bwd_split_segment(D);
  const int64_t K1 = fp32 ? 3 * Dp : D;   // K of the logits contraction
  const int64_t ldk = fp32 ? 3 * Dp : D;  // row stride of the H and W operands
  const __nv_bfloat16* Hb = static_cast<const __nv_bfloat16*>(H);
  const __nv_bfloat16* W3 = nullptr;
  if (fp32) {
    Hb = reinterpret_cast<const __nv_bfloat16*>(ws + L.off_h3);
    W3 = reinterpret_cast<const __nv_bfloat16*>(ws + L.off_w3);
    if ((s = launch_split(H, D, N, D, Dp, 3, 2, ws + L.off_h3, di.sms, st)) != FLCE_OK) return s;
  }
  CUtensorMap mH_k, mH_mn, mH_mn_lo;
  if (!encode_bf16_2d(&mH_k, Hb, N, K1, ldk, bwd::BM) ||     // K1 A: (N, K1)
      !encode_bf16_2d(&mH_mn, Hb, N, D, ldk, bwd::BK))       // K3 B (hi): d contiguous, K = N
    return FLCE_ERR_UNSUPPORTED;
  if (fp32 && !encode_bf16_2d(&mH_mn_lo, Hb + 2 * Dp, N, D, ldk, bwd::BK))  // K3 B (lo)
    return FLCE_ERR_UNSUPPORTED;
  for (int64_t c0 = 0; c0 < V; c0 += L.chunk) {
    const int64_t clen = std::min(L.chunk, V - c0);
    const __nv_bfloat16* Wc = static_cast<const __nv_bfloat16*>(W) + c0 * D;
    if (fp32) {
      if ((s = launch_split(static_cast<const float*>(W) + c0 * D, D, clen, D, Dp, 3, 1,
                            ws + L.off_w3, di.sms, st)) != FLCE_OK)
        return s;
      Wc = W3;
    }
    CUtensorMap mW_k, mW_mn, mW_mn_lo, mDz_k, mDz_mn, mDzl_k, mDzl_mn;
    if (!encode_bf16_2d(&mW_k, Wc, clen, K1, ldk, bwd::HALF_N) ||  // K1 B: (clen, K1)
        !encode_bf16_2d(&mW_mn, Wc, clen, D, ldk, bwd::BK) ||      // K2 B (hi): d contiguous
        !encode_bf16_2d(&mDz_k, dz, N, clen, L.chunk, bwd::BM) ||  // K2 A: K = vocab
        !encode_bf16_2d(&mDz_mn, dz, N, clen, L.chunk, bwd::BK))   // K3 A: vocab contiguous
      return FLCE_ERR_UNSUPPORTED;
    if (fp32 && (!encode_bf16_2d(&mW_mn_lo, Wc + Dp, clen, D, ldk, bwd::BK) ||
                 !encode_bf16_2d(&mDzl_k, dzl, N, clen, L.chunk, bwd::BM) ||
                 !encode_bf16_2d(&mDzl_mn, dzl, N, clen, L.chunk, bwd::BK)))
      return FLCE_ERR_UNSUPPORTED;
    // K1: dZ for this chunk from the regenerated logits
    bwd::EpiGradLogits e1;
    e1.lse = lse;
    e1.y = y;
    e1.grad = grad_loss;
    e1.grad_scale = grad_scale;
    e1.N = int32_t(N);
    e1.V = int32_t(V_total);
    e1.y_offset = y_offset;
    e1.c0 = int32_t(c0);
    e1.clen = int32_t(clen);
    e1.dz = dz;
    e1.dz_lo = dzl;
    e1.ldz = int32_t(L.chunk);
    e1.status = &hdr->status;
    s = launch_gemm<bwd::EpiGradLogits, false, false>(mH_k, mW_k, gemm_shape(N, clen, K1), e1,
                                                      &hdr->status, pairs, st);
    if (s != FLCE_OK) return s;
    // K2: dH (+)= dZ_C W_C; fp32: dz W_hi + dz W_lo + dz_lo W_hi, in that order
    const CUtensorMap* k2[3][2] = {{&mDz_k, &mW_mn}, {&mDz_k, &mW_mn_lo}, {&mDzl_k, &mW_mn}};
    for (int p = 0; p < (fp32 ? 3 : 1); ++p) {
      bwd::EpiStoreF32 e2;
      e2.out = dH;
      e2.ld = int32_t(D);
      e2.rows = int32_t(N);
      e2.cols = int32_t(D);
      e2.row_base = 0;
      e2.accumulate = (c0 > 0 || p > 0) ? 1 : 0;
      s = launch_gemm<bwd::EpiStoreF32, false, true>(*k2[p][0], *k2[p][1], gemm_shape(N, D, clen),
                                                     e2, &hdr->status, pairs, st);
      if (s != FLCE_OK) return s;
    }
    // dH is final once the last chunk's dH GEMMs are queued: a collective on
    // it can start while the dW GEMMs below finish.
    if (dh_ready && c0 + L.chunk >= V && cudaEventRecord(dh_ready, st) != cudaSuccess)
      return FLCE_ERR_CUDA;
    // K3: dW_C = dZ_C^T H; fp32: dz^T H_hi + dz^T H_lo + dz_lo^T H_hi, in that order
    const CUtensorMap* k3[3][2] = {{&mDz_mn, &mH_mn}, {&mDz_mn, &mH_mn_lo}, {&mDzl_mn, &mH_mn}};
    for (int p = 0; p < (fp32 ? 3 : 1); ++p) {
      bwd::EpiStoreF32 e3;
      e3.out = dW;
      e3.ld = int32_t(D);
      e3.rows = int32_t(clen);
      e3.cols = int32_t(D);
      e3.row_base = int32_t(c0);
      e3.accumulate = p > 0 ? 1 : 0;
      s = launch_gemm<bwd::EpiStoreF32, true, true>(*k3[p][0], *k3[p][1], gemm_shape(clen, D, N),
                                                    e3, &hdr->status, pairs, st);
      if (s != FLCE_OK) return s;
    }
  }
  return FLCE_OK;
}

}  // namespace

extern "C" flce_status flce_backward(const void* H, const void* W, const int64_t* y,
                                     const float* lse, const float* grad_loss, float grad_scale,
                                     int64_t N, int64_t V, int64_t D, flce_dtype dtype, float* dH,
                                     float* dW, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  FLCE_TRACE();
  return backward_impl(H, W, y, lse, grad_loss, grad_scale, N, V, 0, V, D, dtype, dH, dW,
                       workspace, workspace_bytes, stream, nullptr);
}

extern "C" flce_status flce_backward_shard(const void* H, const void* W_shard, const int64_t* y,
                                           const float* lse, const float* grad_loss,
                                           float grad_scale, int64_t N, int64_t V_shard,
                                           int64_t v_offset, int64_t V_total, int64_t D,
                                           flce_dtype dtype, float* dH_partial, float* dW_shard,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream, void* dh_ready_event) {
  FLCE_TRACE();
  if (v_offset < 0 || V_shard < 1 || V_total < v_offset + V_shard || V_total >= (int64_t(1) << 31))
    return FLCE_ERR_INVALID_ARG;
  return backward_impl(H, W_shard, y, lse, grad_loss, grad_scale, N, V_shard, v_offset, V_total,
                       D, dtype, dH_partial, dW_shard, workspace, workspace_bytes, stream,
                       static_cast<cudaEvent_t>(dh_ready_event));
}

// ---------------------------------------------------------------- no-allocation entry point
//
// Some callers cannot allocate device memory at the point where they need the
// loss: code running inside an allocator or memory-pool callback, a runtime
// that forbids cudaMalloc while it owns the device memory budget, or a host
// that has no workspace to hand over.  flce_forward_noalloc serves them: its
// scratch (the workspace of flce_forward) is one file-scope device array
// that the CUDA module carries, so the call itself allocates nothing.

namespace {

// Every GPU on which this library's module is loaded holds this array until
// the process exits.  In host code the name is only a stand-in: the device
// address comes from cudaGetSymbolAddress, with the device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FLCE_NOALLOC_SCRATCH_BYTES];

// The looked-up address is cached per device together with the id of the
// CUDA context it was found in (cuCtxGetId: unique for the life of the
// process, never reused).  A call made in another context (a non-primary
// context, or a primary context re-created after cudaDeviceReset, which
// reloads the module elsewhere) looks the address up again.
constexpr int kMaxDevices = 64;
struct NoallocSlot {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
std::mutex g_noalloc_mu;
NoallocSlot g_noalloc_slot[kMaxDevices];

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);
PfnCtxGetCurrent g_ctx_get_current = nullptr;
PfnCtxGetId g_ctx_get_id = nullptr;
std::once_flag g_ctx_fns_once;

bool load_ctx_fns() {
  std::call_once(g_ctx_fns_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<PfnCtxGetCurrent>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<PfnCtxGetId>(fn);
  });
  return g_ctx_get_current != nullptr && g_ctx_get_id != nullptr;
}

// Id of the context current on this thread; binds the current device's primary
// context first if none is current (the runtime does so on its first call).
flce_status current_ctx_id(unsigned long long* id) {
  if (!load_ctx_fns()) return FLCE_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return FLCE_ERR_CUDA;
  if (ctx == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return FLCE_ERR_CUDA;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return FLCE_ERR_CUDA;
  }
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? FLCE_OK : FLCE_ERR_CUDA;
}

// Device address of the scratch array in the current context (looked up on
// the first call in that context, with its device current).
flce_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FLCE_ERR_UNSUPPORTED;
  unsigned long long id = 0;
  flce_status s = current_ctx_id(&id);
  if (s != FLCE_OK) return s;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  if (slot.ptr == nullptr || slot.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FLCE_ERR_CUDA;
    slot.ptr = p;
    slot.ctx_id = id;
  }
  *out = slot.ptr;
  return FLCE_OK;
}

}  // namespace

extern "C" flce_status flce_forward_noalloc(const void* H, const void* W, const int64_t* y,
                                            int64_t N, int64_t V, int64_t D, flce_dtype dtype,
                                            float* out_loss, float* out_lse,
                                            float* out_target_logit, float* out_mean,
                                            void* stream) {
  FLCE_TRACE();
  if (!sizes_ok(N, V, D, dtype)) return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  // The problem must fit the built-in scratch; nothing larger is ever allocated.
  if (workspace_bytes_for(N, V, D, dtype) > size_t(FLCE_NOALLOC_SCRATCH_BYTES))
    return FLCE_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  flce_status s = noalloc_scratch(&scratch);
  if (s != FLCE_OK) return s;
  // flce_forward checks the remaining arguments; it clears the scratch header
  // (status word and merge counter) on the stream before its kernels run, and
  // every other scratch byte it reads is written earlier in the same call.
  return flce_forward(H, W, y, N, V, D, dtype, out_loss, out_lse, out_target_logit, out_mean,
                      scratch, size_t(FLCE_NOALLOC_SCRATCH_BYTES), stream);
}

// ---------------------------------------------------------------- quantised head

namespace {

// Vocabulary rows expanded at a time (a multiple of the 256-column tile).
constexpr int64_t kQuantChunkRows = 16384;

bool quant_format_ok(int32_t bits, int64_t G, int64_t D) {
  if (bits != 2 && bits != 4 && bits != 8) return false;
  if (G != 32 && G != 64 && G != 128) return false;
  return D >= G && D % G == 0;
}

// One K segment of the expanded W: D rounded up to the 64-element K block.
int64_t quant_segment(int64_t D) { return cdiv(D, tc::BK) * tc::BK; }

// Workspace of the quantised forward: the slab state of one chunk (header,
// partials, the mean's block sums), one float4 per (chunk, token), and the
// expanded [hi | lo] bf16 rows of one chunk.
struct QuantLayout {
  int64_t C = 0, chunks = 0;
  size_t state = 0, states = 0, expanded = 0, pad = 0, total = 0;
};

QuantLayout quant_layout(int64_t N, int64_t V, int64_t D) {
  QuantLayout L;
  L.C = std::min(V, kQuantChunkRows);
  L.chunks = cdiv(V, L.C);
  L.state = state_bytes_for(N, L.C);
  L.states = align256(size_t(16) * size_t(N) * size_t(L.chunks));
  L.expanded = align256(size_t(L.C) * size_t(2 * quant_segment(D)) * 2);
  L.pad = fwd_pad_h_bytes(N, D);   // fewer than kMinHRows tokens: H padded with zero rows
  L.total = L.state + L.states + L.expanded + L.pad;
  return L;
}

flce_status launch_dequant(const uint32_t* wq, const void* scales, const void* biases,
                           int32_t bits, int32_t G, int64_t row0, int64_t rows, int64_t D,
                           void* dst, int sms, cudaStream_t st) {
  quant::Args a;
  a.wq = wq;
  a.scales = static_cast<const __nv_bfloat16*>(scales);
  a.biases = static_cast<const __nv_bfloat16*>(biases);
  a.row0 = row0;
  a.rows = rows;
  a.D = int32_t(D);
  a.Ds = int32_t(quant_segment(D));
  a.G = G;
  a.dst = static_cast<__nv_bfloat16*>(dst);
  const int64_t warps_per_block = quant::NUM_THREADS / 32;
  const unsigned blocks = unsigned(std::max<int64_t>(
      1, std::min<int64_t>(cdiv(rows, warps_per_block), int64_t(sms) * 8)));
  if (bits == 4)
    quant::flce_dequant_split_kernel<4><<<blocks, quant::NUM_THREADS, 0, st>>>(a);
  else if (bits == 8)
    quant::flce_dequant_split_kernel<8><<<blocks, quant::NUM_THREADS, 0, st>>>(a);
  else
    quant::flce_dequant_split_kernel<2><<<blocks, quant::NUM_THREADS, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

}  // namespace

extern "C" size_t flce_quantized_workspace_size(int64_t N, int64_t V, int64_t D, int32_t bits,
                                                int32_t group_size) {
  if (N < 0 || V < 1 || D < 1 || !quant_format_ok(bits, group_size, D)) return 0;
  return quant_layout(N, V, D).total;
}

extern "C" flce_status flce_forward_quantized(const void* H, const uint32_t* wq,
                                              const void* scales, const void* biases,
                                              int32_t bits, int32_t group_size, const int64_t* y,
                                              int64_t N, int64_t V, int64_t D, float* out_loss,
                                              float* out_lse, float* out_target_logit,
                                              float* out_mean, float* out_sum, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  FLCE_TRACE();
  if (N < 0 || V < 1 || D < 1 || !quant_format_ok(bits, group_size, D))
    return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!H || !wq || !scales || !biases || !y || !out_loss || !out_lse || !out_target_logit ||
      !workspace)
    return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      ((reinterpret_cast<uintptr_t>(scales) | reinterpret_cast<uintptr_t>(biases)) & 1u) != 0)
    return FLCE_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(wq)) return FLCE_ERR_UNSUPPORTED;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || 2 * quant_segment(D) >= (int64_t(1) << 31))
    return FLCE_ERR_UNSUPPORTED;
  const QuantLayout L = quant_layout(N, V, D);
  if (workspace_bytes < L.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DeviceInfo di;
  int64_t workers = 0;
  flce_status s = contraction_workers(N, di, workers);
  if (s != FLCE_OK) return s;

  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
  float4* states = reinterpret_cast<float4*>(wsb + L.state);
  void* expanded = wsb + L.state + L.states;
  const int64_t Ds = quant_segment(D);
  // One header for the whole call: its status word collects every stage's
  // findings, and the final merge's block counter starts at zero.
  if (cudaMemsetAsync(hdr, 0, kHeaderBytes, st) != cudaSuccess) return FLCE_ERR_CUDA;
  // A batch of fewer than kMinHRows tokens reads H from a copy padded with zero rows.
  const void* h_op = H;
  int64_t h_rows = 0;
  if (N < kMinHRows) {
    void* hp = wsb + L.state + L.states + L.expanded;
    if ((s = launch_pad_h(H, D, N, D, hp, di.sms, st)) != FLCE_OK) return s;
    h_op = hp;
    h_rows = kMinHRows;
  }
  for (int64_t c = 0; c < L.chunks; ++c) {
    const int64_t c0 = c * L.C;
    const int64_t rows = std::min(L.C, V - c0);
    if ((s = launch_dequant(wq, scales, biases, bits, group_size, c0, rows, D, expanded, di.sms,
                            st)) != FLCE_OK)
      return s;
    flce_plan_t plan;
    make_plan(N, rows, D, FLCE_BF16, workers, &plan);
    // H against the chunk's [hi | lo] rows: H W_hi^T + H W_lo^T per K block
    const Operands op{h_op, D, D, 0, expanded, 2 * Ds, 2 * Ds, Ds, Ds / tc::BK, tc::kSplitW,
                      h_rows};
    if ((s = launch_contraction(op, Targets{y, 0}, c0, N, rows, plan, out_target_logit, workspace,
                                HeaderReset::kNone, st)) != FLCE_OK)
      return s;
    flce_shard_state_kernel<<<unsigned(cdiv(N, kMergeThreads)), kMergeThreads, 0, st>>>(
        reinterpret_cast<const float2*>(wsb + state_layout(N, rows).part), hdr, y, int32_t(N), c0,
        rows,
        int32_t(slab_capacity(rows)), out_target_logit, states + c * N, &hdr->status);
    if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  }
  double* block_sums = reinterpret_cast<double*>(wsb + state_layout(N, L.C).sums);
  flce_merge_shards_kernel<<<unsigned(cdiv(N, kMergeThreads)), kMergeThreads, 0, st>>>(
      states, int32_t(L.chunks), y, int32_t(N), V, out_loss, out_lse, out_target_logit, out_mean,
      out_sum,
      block_sums, hdr);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

// ---------------------------------------------------------------- quantised head: backward

namespace {

// [256 B header][dZ slice: N x chunk bf16][one chunk of W expanded: chunk x 2 Ds bf16]
struct QuantBwdLayout {
  int64_t chunk = 0;
  size_t off_dz = 0, off_exp = 0, total = 0;
};

QuantBwdLayout quant_bwd_layout(int64_t N, int64_t V, int64_t D) {
  QuantBwdLayout L;
  L.chunk = std::min(round_up(V, kTileCols), kBwdChunkColsSplit);
  L.off_dz = kHeaderBytes;
  L.off_exp = L.off_dz + align256(size_t(N) * size_t(L.chunk) * 2);
  L.total = L.off_exp + align256(size_t(L.chunk) * size_t(2 * quant_segment(D)) * 2);
  return L;
}

}  // namespace

extern "C" size_t flce_backward_quantized_workspace_size(int64_t N, int64_t V, int64_t D,
                                                         int32_t bits, int32_t group_size) {
  if (N < 1 || V < 1 || D < 1 || !quant_format_ok(bits, group_size, D)) return 0;
  return quant_bwd_layout(N, V, D).total;
}

extern "C" flce_status flce_backward_quantized(const void* H, const uint32_t* wq,
                                               const void* scales, const void* biases,
                                               int32_t bits, int32_t group_size, const int64_t* y,
                                               const float* lse, const float* grad_loss,
                                               float grad_scale, int64_t N, int64_t V, int64_t D,
                                               float* dH, void* workspace, size_t workspace_bytes,
                                               void* stream) {
  FLCE_TRACE();
  if (N < 0 || V < 1 || D < 1 || !quant_format_ok(bits, group_size, D))
    return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!H || !wq || !scales || !biases || !y || !lse || !dH || !workspace)
    return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      ((reinterpret_cast<uintptr_t>(scales) | reinterpret_cast<uintptr_t>(biases)) & 1u) != 0)
    return FLCE_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(wq)) return FLCE_ERR_UNSUPPORTED;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) ||
      2 * quant_segment(D) >= (int64_t(1) << 31))
    return FLCE_ERR_UNSUPPORTED;
  const QuantBwdLayout L = quant_bwd_layout(N, V, D);
  if (workspace_bytes < L.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;

  DeviceInfo di;
  flce_status s = device_info(di);
  if (s != FLCE_OK) return s;
  if (!load_encoder()) return FLCE_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if ((s = set_smem_limits()) != FLCE_OK) return s;
  const int64_t pairs = resident_pairs(dev, di.sms);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(ws + L.off_dz);
  const __nv_bfloat16* ex = reinterpret_cast<const __nv_bfloat16*>(ws + L.off_exp);
  const int64_t Ds = quant_segment(D);
  if (cudaMemsetAsync(hdr, 0, kHeaderBytes, st) != cudaSuccess) return FLCE_ERR_CUDA;

  CUtensorMap mH_k;
  if (!encode_bf16_2d(&mH_k, H, N, D, D, bwd::BM)) return FLCE_ERR_UNSUPPORTED;  // K1 A
  for (int64_t c0 = 0; c0 < V; c0 += L.chunk) {
    const int64_t clen = std::min(L.chunk, V - c0);
    // W rows [c0, c0 + clen) as bf16 [hi | lo] (row stride 2 Ds)
    if ((s = launch_dequant(wq, scales, biases, bits, group_size, c0, clen, D, ws + L.off_exp,
                            di.sms, st)) != FLCE_OK)
      return s;
    CUtensorMap mW_k, mW_hi, mW_lo, mDz_k;
    if (!encode_bf16_2d(&mW_k, ex, clen, 2 * Ds, 2 * Ds, bwd::HALF_N) ||  // K1 B: [hi | lo]
        !encode_bf16_2d(&mW_hi, ex, clen, D, 2 * Ds, bwd::BK) ||          // K2 B: hi, MN-major
        !encode_bf16_2d(&mW_lo, ex + Ds, clen, D, 2 * Ds, bwd::BK) ||     // K2 B: lo, MN-major
        !encode_bf16_2d(&mDz_k, dz, N, clen, L.chunk, bwd::BM))           // K2 A
      return FLCE_ERR_UNSUPPORTED;
    // K1: logits [H | H] [hi | lo]^T over K = 2 Ds (H's K coordinate wraps
    // after Ds), then dZ for the chunk
    bwd::EpiGradLogits e1;
    e1.lse = lse;
    e1.y = y;
    e1.grad = grad_loss;
    e1.grad_scale = grad_scale;
    e1.N = int32_t(N);
    e1.V = int32_t(V);
    e1.y_offset = 0;
    e1.c0 = int32_t(c0);
    e1.clen = int32_t(clen);
    e1.dz = dz;
    e1.dz_lo = nullptr;
    e1.ldz = int32_t(L.chunk);
    e1.status = &hdr->status;
    bwd::GemmShape g1 = gemm_shape(N, clen, 2 * Ds);
    g1.kblocks_a = int32_t(Ds / bwd::BK);
    s = launch_gemm<bwd::EpiGradLogits, false, false>(mH_k, mW_k, g1, e1, &hdr->status, pairs,
                                                      st);
    if (s != FLCE_OK) return s;
    // K2: dH (+)= dZ_C W_hi + dZ_C W_lo, in that order
    const CUtensorMap* bs[2] = {&mW_hi, &mW_lo};
    for (int p = 0; p < 2; ++p) {
      bwd::EpiStoreF32 e2;
      e2.out = dH;
      e2.ld = int32_t(D);
      e2.rows = int32_t(N);
      e2.cols = int32_t(D);
      e2.row_base = 0;
      e2.accumulate = (c0 > 0 || p > 0) ? 1 : 0;
      s = launch_gemm<bwd::EpiStoreF32, false, true>(mDz_k, *bs[p], gemm_shape(N, D, clen), e2,
                                                     &hdr->status, pairs, st);
      if (s != FLCE_OK) return s;
    }
  }
  return FLCE_OK;
}

// ---------------------------------------------------------------- forward from host memory

namespace {

// Vocabulary rows copied per chunk (a multiple of the 256-column tile).
constexpr int64_t kHostChunkRows = 8192;

// Workspace of the host-input forward: one chunk's slab state, a float4 per
// (chunk, token), device copies of H and y, the outputs, and two staging
// buffers for W chunks.
struct HostLayout {
  int64_t C = 0, chunks = 0;
  size_t state = 0, states = 0, h = 0, y = 0, outs = 0, staging = 0, total = 0;
};

HostLayout host_layout(int64_t N, int64_t V, int64_t D) {
  HostLayout L;
  L.C = std::min(V, kHostChunkRows);
  L.chunks = cdiv(V, L.C);
  L.state = state_bytes_for(N, L.C);
  L.states = align256(size_t(16) * size_t(N) * size_t(L.chunks));
  L.h = align256(size_t(padded_h_rows(N)) * size_t(D) * 2);   // H, zero rows up to kMinHRows
  L.y = align256(size_t(N) * 8);
  L.outs = align256(size_t(N) * 12 + 4);
  L.staging = align256(size_t(L.C) * size_t(D) * 2);
  L.total = L.state + L.states + L.h + L.y + L.outs + 2 * L.staging;
  return L;
}

// Events created for one call; destroyed when the call returns (CUDA keeps a
// destroyed event's pending work valid).
struct CallEvents {
  cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  bool create() {
    for (auto& e : ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
  ~CallEvents() {
    for (auto& e : ev)
      if (e) cudaEventDestroy(e);
  }
};

}  // namespace

extern "C" size_t flce_forward_host_workspace_size(int64_t N, int64_t V, int64_t D,
                                                   flce_dtype dtype) {
  if (!sizes_ok(N, V, D, dtype) || dtype != FLCE_BF16 || D % 8 != 0) return 0;
  return host_layout(N, V, D).total;
}

extern "C" flce_status flce_forward_host(const void* H_host, const void* W_host,
                                         const int64_t* y_host, int64_t N, int64_t V, int64_t D,
                                         flce_dtype dtype, float* loss_host, float* lse_host,
                                         float* target_logit_host, float* mean_host,
                                         void* workspace, size_t workspace_bytes, void* stream,
                                         void* copy_stream) {
  FLCE_TRACE();
  if (!sizes_ok(N, V, D, dtype)) return FLCE_ERR_INVALID_ARG;
  if (N == 0) return FLCE_OK;
  if (!H_host || !W_host || !y_host || !loss_host || !workspace) return FLCE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FLCE_ERR_INVALID_ARG;
  if (dtype != FLCE_BF16 || D % 8 != 0) return FLCE_ERR_UNSUPPORTED;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || D >= (int64_t(1) << 31))
    return FLCE_ERR_UNSUPPORTED;
  const HostLayout L = host_layout(N, V, D);
  if (workspace_bytes < L.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t cs = copy_stream ? static_cast<cudaStream_t>(copy_stream) : st;
  DeviceInfo di;
  int64_t workers = 0;
  flce_status s = contraction_workers(N, di, workers);
  if (s != FLCE_OK) return s;
  CallEvents events;
  if (!events.create()) return FLCE_ERR_CUDA;
  cudaEvent_t* ready = events.ev;       // [2] staging buffer b holds its chunk
  cudaEvent_t* freed = events.ev + 2;   // [2] staging buffer b has been read
  cudaEvent_t start = events.ev[4];     // all work queued on `stream` before this call

  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
  size_t off = L.state;
  float4* states = reinterpret_cast<float4*>(wsb + off);
  off += L.states;
  void* Hd = wsb + off;
  off += L.h;
  int64_t* yd = reinterpret_cast<int64_t*>(wsb + off);
  off += L.y;
  float* loss_d = reinterpret_cast<float*>(wsb + off);
  float* lse_d = loss_d + N;
  float* tgt_d = lse_d + N;
  float* mean_d = tgt_d + N;
  off += L.outs;
  uint8_t* staging[2] = {wsb + off, wsb + off + L.staging};
  const size_t row_bytes = size_t(D) * 2;
  const uint8_t* Wh = static_cast<const uint8_t*>(W_host);

  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // The copies below overwrite H, y and the staging buffers in the workspace:
  // they wait for earlier work on `stream` (a previous call may still read them).
  if (cs != st && (!ok(cudaEventRecord(start, st)) || !ok(cudaStreamWaitEvent(cs, start, 0))))
    return FLCE_ERR_CUDA;
  if (!ok(cudaMemsetAsync(hdr, 0, kHeaderBytes, st))) return FLCE_ERR_CUDA;
  // H and y first, on the copy stream, ahead of the W chunks (a batch of fewer
  // than kMinHRows tokens gets zero rows after its own, see kMinHRows).
  if (!ok(cudaMemcpyAsync(Hd, H_host, size_t(N) * row_bytes, cudaMemcpyHostToDevice, cs)) ||
      !ok(cudaMemcpyAsync(yd, y_host, size_t(N) * 8, cudaMemcpyHostToDevice, cs)))
    return FLCE_ERR_CUDA;
  if (N < kMinHRows && !ok(cudaMemsetAsync(static_cast<uint8_t*>(Hd) + size_t(N) * row_bytes, 0,
                                           size_t(kMinHRows - N) * row_bytes, cs)))
    return FLCE_ERR_CUDA;
  for (int64_t c = 0; c < L.chunks; ++c) {
    const int b = int(c & 1);
    const int64_t c0 = c * L.C;
    const int64_t rows = std::min(L.C, V - c0);
    // Buffer b last held chunk c - 2: wait until its contraction has read it.
    if (c >= 2 && !ok(cudaStreamWaitEvent(cs, freed[b], 0))) return FLCE_ERR_CUDA;
    if (!ok(cudaMemcpyAsync(staging[b], Wh + size_t(c0) * row_bytes, size_t(rows) * row_bytes,
                            cudaMemcpyHostToDevice, cs)) ||
        !ok(cudaEventRecord(ready[b], cs)) || !ok(cudaStreamWaitEvent(st, ready[b], 0)))
      return FLCE_ERR_CUDA;
    flce_plan_t plan;
    make_plan(N, rows, D, FLCE_BF16, workers, &plan);
    Operands op = bf16_operands(Hd, D, staging[b], D, N, D);
    op.h_rows = padded_h_rows(N);
    if ((s = launch_contraction(op, Targets{yd, 0}, c0, N, rows, plan, tgt_d, workspace,
                                HeaderReset::kNone, st)) != FLCE_OK)
      return s;
    flce_shard_state_kernel<<<unsigned(cdiv(N, kMergeThreads)), kMergeThreads, 0, st>>>(
        reinterpret_cast<const float2*>(wsb + state_layout(N, rows).part), hdr, yd, int32_t(N), c0,
        rows,
        int32_t(slab_capacity(rows)), tgt_d, states + c * N, &hdr->status);
    if (!ok(cudaGetLastError()) || !ok(cudaEventRecord(freed[b], st))) return FLCE_ERR_CUDA;
  }
  double* block_sums = reinterpret_cast<double*>(wsb + state_layout(N, L.C).sums);
  flce_merge_shards_kernel<<<unsigned(cdiv(N, kMergeThreads)), kMergeThreads, 0, st>>>(
      states, int32_t(L.chunks), yd, int32_t(N), V, loss_d, lse_d, tgt_d, mean_d, nullptr,
      block_sums, hdr);
  if (!ok(cudaGetLastError())) return FLCE_ERR_CUDA;
  const size_t nb = size_t(N) * 4;
  if (!ok(cudaMemcpyAsync(loss_host, loss_d, nb, cudaMemcpyDeviceToHost, st)) ||
      (lse_host && !ok(cudaMemcpyAsync(lse_host, lse_d, nb, cudaMemcpyDeviceToHost, st))) ||
      (target_logit_host &&
       !ok(cudaMemcpyAsync(target_logit_host, tgt_d, nb, cudaMemcpyDeviceToHost, st))) ||
      (mean_host && !ok(cudaMemcpyAsync(mean_host, mean_d, 4, cudaMemcpyDeviceToHost, st))))
    return FLCE_ERR_CUDA;
  // The copy stream's last work (the final chunk's copy) is already ordered
  // before `stream` through ready[]; nothing else is left on it.
  return FLCE_OK;
}
