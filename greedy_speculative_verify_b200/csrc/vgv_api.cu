// C ABI of the verifier hot path (declared in include/vgv.h): argument
// validation, workspace layout, TMA descriptors and kernel launches. One
// translation unit so the device status word is a single symbol.
#include <cudaTypedefs.h>
#include <string.h>

#include <mutex>
#include <utility>
#include <vector>

#include "vgv.h"
#include "common.cuh"
#include "combine.cuh"
#include "decode_loop.cuh"
#include "mtp.cuh"
#include "attention.cuh"
#include "proj_tc.cuh"
#include "gemm_moe.cuh"
#include "gemm_tm.cuh"
#include "layer_entry.cuh"
#include "entry_small.cuh"
#include "lmhead.cuh"
#include "router.cuh"
#include "step_small.cuh"
#include "sort.cuh"

namespace {

constexpr int kH = 1280, kI = 896, kE = 64, kS = 2, kTopK = 6;
constexpr int kMaxDevices = 64;
constexpr int kEntryMaxGrid = 256;  // CTAs of the layer-entry kernel at most

// Bytes of expert weights the layer entry prefetches into L2: the gate|up rows
// of the first routed experts, which the expert kernel's first wave of units
// streams (about one unit per SM).
#ifndef VG_ENTRY_PREFETCH_MB
#define VG_ENTRY_PREFETCH_MB 96
#endif
#ifndef VG_SMALL_ENTRY_PREFETCH_MB
#define VG_SMALL_ENTRY_PREFETCH_MB 0
#endif
#ifndef VG_PRE_L2_CHUNKS
#define VG_PRE_L2_CHUNKS 0
#endif
#ifndef VG_ENTRY_PF_UNITS
#define VG_ENTRY_PF_UNITS 0
#endif
#ifndef VG_ENTRY_PF_CHUNKS
#define VG_ENTRY_PF_CHUNKS 20
#endif
constexpr size_t kEntryPrefetchBytes = (size_t)VG_ENTRY_PREFETCH_MB << 20;
// the two-token entry shares its SMs with the expert kernel, whose CTAs request
// their first weights themselves; any prefetch of its own is on top of that
constexpr size_t kSmallEntryPrefetchBytes = (size_t)VG_SMALL_ENTRY_PREFETCH_MB << 20;
constexpr int kEntryPrefetchMinT = 64;  // 384 assignments: each expert untouched with probability < 0.3%
// Static first units of the expert kernel (its first weights requested before
// the routing is known) from this many tokens on, when the two-token entry runs:
// then every expert is touched with probability > 99.7%, so the requested
// weights are nearly always needed
constexpr int kStaticFirstMinT = 64;
constexpr int kPreL2Chunks = VG_PRE_L2_CHUNKS;  // further k-chunks of the first unit prefetched to L2

struct DevState {
  bool init = false;
  int sms = 0;
};
DevState g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// ------------------------------------------------------------- timing hook
struct ProfHook {
  std::vector<cudaEvent_t> starts, stops;
  int64_t count = 0;
};
ProfHook g_prof[VG_KERNEL_KINDS];
std::mutex g_prof_mu;
bool g_prof_any = false;

// Records an event on `s`; while `s` is being captured into a graph the record
// must be marked external to become a timing node of the graph.
void record_event(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, s);
}

// Brackets one launch of `kind` with the hook's events, if any are set.
struct ProfScope {
  int kind;
  cudaStream_t s;
  int64_t slot = -1;
  ProfScope(int k, cudaStream_t st) : kind(k), s(st) {
    if (!g_prof_any) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    ProfHook& h = g_prof[kind];
    if (h.starts.empty()) return;
    slot = h.count++ % (int64_t)h.starts.size();
    record_event(h.starts[slot], s);
  }
  ~ProfScope() {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    ProfHook& h = g_prof[kind];
    if ((int64_t)h.stops.size() > slot) record_event(h.stops[slot], s);
  }
};

vg_status cuda_fail() {
  (void)cudaGetLastError();
  return VG_ERR_CUDA;
}

// Per-device one-time set-up: SM count, shared-memory opt-in for the big kernels.
vg_status device_state(DevState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail();
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& d = g_dev[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return cuda_fail();
    if (cudaFuncSetAttribute(vg::moe_expert_gemms_tm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vg::kTmSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vg::moe_expert_gemms<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vg::FgCfg<128>::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vg::moe_expert_gemms<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vg::FgCfg<64>::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vg::moe_expert_gemms<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vg::FgCfg<16>::kSmemBytes) != cudaSuccess)
      return cuda_fail();
    if (cudaFuncSetAttribute(vg::moe_layer_entry<kTopK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vg::layer_entry_smem()) != cudaSuccess)
      return cuda_fail();
    if (cudaFuncSetAttribute(vg::router_topk_tiled<kTopK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vg::kRtPartBytes) != cudaSuccess)
      return cuda_fail();
    if (cudaFuncSetAttribute(vg::verify_step_small<kTopK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vg::kSsSmemBytes) != cudaSuccess)
      return cuda_fail();
    if (cudaFuncSetAttribute(vg::attn_proj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, vg::kPtSmemBytes) !=
            cudaSuccess)
      return cuda_fail();
    if (cudaFuncSetAttribute(vg::lmhead_argmax_accept, cudaFuncAttributeMaxDynamicSharedMemorySize, vg::kLmSmemBytes) !=
        cudaSuccess)
      return cuda_fail();
    // Kernels that follow each other with dependent launches share SMs only if
    // their shared-memory configurations agree: every kernel of the decode
    // chain asks for the largest shared-memory carveout.
    {
      const int kMax = cudaSharedmemCarveoutMaxShared;
      const cudaFuncAttribute kC = cudaFuncAttributePreferredSharedMemoryCarveout;
      if (cudaFuncSetAttribute(vg::moe_entry_small<kTopK>, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::moe_layer_entry<kTopK>, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::moe_expert_gemms<16>, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::moe_expert_gemms<64>, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::moe_expert_gemms<128>, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::moe_expert_gemms_tm, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::moe_combine<true>, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::moe_combine<false>, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::lmhead_argmax_accept, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::embed_rows, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::spec_rows, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::spec_rows_given, kC, kMax) != cudaSuccess ||
          cudaFuncSetAttribute(vg::spec_commit, kC, kMax) != cudaSuccess)
        return cuda_fail();
    }
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return cuda_fail();
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.init = true;
  }
  *out = &d;
  return VG_OK;
}

// bf16 tensor map with 128-byte swizzle; dims/strides innermost first, strides in bytes.
vg_status make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                   const uint32_t* box) {
  uint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VG_OK : VG_ERR_CUDA;
}

// Rows of a TMA box: `full`, or the tensor's row count rounded up to 8 when the
// tensor is shorter than one full box.
int box_rows(int64_t rows, int full) { return rows >= full ? full : (int)((rows + 7) / 8 * 8); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool dims_supported(const vg_moe_dims* d) {
  return d->hidden == kH && d->intermediate == kI && d->n_routed == kE && d->n_shared == kS && d->top_k == kTopK;
}

struct MoeWs {
  size_t idx, w, offsets, perm, inv, xperm, act, o, ccnt, cbase, ecnt, sched, gbar, total;
  int sched_len;
};

// Tile width of the expert GEMMs: 16-token tiles (six pipeline stages) for a
// handful of tokens, 64-token tiles (five stages) at decode sizes, 128-token
// tiles for prefill-sized segments.
constexpr int kCombineAllLoadsMaxT = 1024;  // tokens up to which the combine issues all loads first
static_assert(kTopK <= vg::kCombineMaxK && kS <= vg::kCombineMaxS, "the combine's unrolled loads cover k and S");

int expert_tile(int T) { return T <= 16 ? 16 : T <= 1024 ? 64 : 128; }

// Rows of x_perm beyond the T k assignments: with fixed first units (64-token
// tiles) every routed expert's first tile has its own 64 rows ahead of them.
size_t xperm_extra_rows(int T) { return expert_tile(T) == 64 ? (size_t)kE * 64 : 0; }

// Upper bound of the expert GEMMs' token tiles: routed segments cut at the tile
// width plus one partial tile per routed expert, plus the shared experts' tiles.
int max_tiles(int T) {
  const int nt = expert_tile(T);
  return vg::cdiv(T * kTopK, nt) + kE + kS * vg::cdiv(T, nt);
}

// CTAs of the expert kernel: one per SM, at most one per unit.
int expert_grid(const DevState* dev, int T) {
  return std::min(dev->sms, (kI / vg::kBM + kH / (2 * vg::kBM)) * max_tiles(T));
}


MoeWs moe_layout(int T) {
  const size_t N = (size_t)T * kTopK;
  const size_t nch = (N + vg::kSortChunk - 1) / vg::kSortChunk;
  MoeWs L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.idx = take(N * 4);
  L.w = take(N * 4);
  L.offsets = take((kE + 1) * 4);
  L.perm = take(N * 4);
  L.inv = take(N * 4);
  L.xperm = take((N + xperm_extra_rows(T)) * kH * 2);
  L.act = take((size_t)(kTopK + kS) * T * kI * 2);
  L.o = take((size_t)(kTopK + kS) * T * kH * 2);
  L.ccnt = take(nch * kE * 4);
  L.cbase = take(nch * kE * 4);
  L.ecnt = take((size_t)kEntryMaxGrid * kE * 4);
  L.sched_len = 1 + max_tiles(T);
  L.sched = take((size_t)L.sched_len * 4);
  L.gbar = take(8);
  L.total = off;
  return L;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Device buffers of one layer inside the workspace (or the caller's taps).
struct LayerBufs {
  int32_t *idx, *offsets, *perm, *inv, *sched, *ccnt, *cbase, *ecnt;
  float* gw;
  uint32_t* gbar;
  __nv_bfloat16 *xperm, *act, *o;
  int sched_len;
};

LayerBufs carve(void* workspace, int T, const vg_moe_taps* taps) {
  const MoeWs L = moe_layout(T);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  LayerBufs b{};
  b.idx = (taps && taps->topk_idx) ? taps->topk_idx : reinterpret_cast<int32_t*>(ws + L.idx);
  b.gw = (taps && taps->topk_weight) ? taps->topk_weight : reinterpret_cast<float*>(ws + L.w);
  b.offsets = (taps && taps->expert_offsets) ? taps->expert_offsets : reinterpret_cast<int32_t*>(ws + L.offsets);
  b.perm = (taps && taps->perm) ? taps->perm : reinterpret_cast<int32_t*>(ws + L.perm);
  b.inv = (taps && taps->inv_perm) ? taps->inv_perm : reinterpret_cast<int32_t*>(ws + L.inv);
  b.act = (taps && taps->act) ? static_cast<__nv_bfloat16*>(taps->act) : reinterpret_cast<__nv_bfloat16*>(ws + L.act);
  b.o = (taps && taps->expert_out) ? static_cast<__nv_bfloat16*>(taps->expert_out)
                                   : reinterpret_cast<__nv_bfloat16*>(ws + L.o);
  b.xperm = reinterpret_cast<__nv_bfloat16*>(ws + L.xperm);
  b.sched = reinterpret_cast<int32_t*>(ws + L.sched);
  b.sched_len = L.sched_len;
  b.ccnt = reinterpret_cast<int32_t*>(ws + L.ccnt);
  b.cbase = reinterpret_cast<int32_t*>(ws + L.cbase);
  b.ecnt = reinterpret_cast<int32_t*>(ws + L.ecnt);
  b.gbar = reinterpret_cast<uint32_t*>(ws + L.gbar);
  return b;
}

// Up to two tokens per CTA, next to the expert kernel (entry_small.cuh).
bool entry_small_path(const DevState* dev, int T) {
#ifndef VG_SMALL_ENTRY
  (void)dev;
  (void)T;
  return false;  // measured slower than the one-token entry at 128 tokens: ~28 against ~18 us per layer
#else
  return vg::cdiv(T, vg::kEsTok) <= std::min(dev->sms, vg::kEsMaxGrid);
#endif
}
bool small_path(const DevState* dev, int T);
int expert_grid(const DevState* dev, int T);
bool static_first_units(const DevState* dev, int T) {
#ifdef VG_NO_STATIC_FIRST
  return false;
#endif
  // the layer-entry kernel lays out the token rows of the fixed first tiles, and
  // every CTA of the expert kernel has a primary gate/up unit of its own
  return T >= kStaticFirstMinT && vg::cdiv(T, vg::kEsTok) <= std::min(dev->sms, vg::kEsMaxGrid) &&
         expert_tile(T) == 64 && !entry_small_path(dev, T) && small_path(dev, T) &&
         expert_grid(dev, T) <= (kE + kS) * (kI / vg::kBM);
}

// The layer-entry kernel takes decode sizes: at most kEntryMaxOwn tokens per CTA
// of its cooperative grid.
#ifndef VG_ENTRY_TOK_PER_CTA
#define VG_ENTRY_TOK_PER_CTA 1
#endif
int entry_grid(const DevState* dev, int T) {
  const int g = std::min(std::min(std::min(dev->sms, kEntryMaxGrid), vg::kEntryMaxGridDev), T);
  // with fixed first units the expert kernel's CTAs stream weights on every SM
  // the entry leaves free, so the entry may take several tokens per CTA
  const int per = T >= kStaticFirstMinT ? VG_ENTRY_TOK_PER_CTA : 1;
  return std::max(1, std::min(g, vg::cdiv(T, per)));
}
bool small_path(const DevState* dev, int T) {
  return (int64_t)T * kTopK <= vg::kSortSmallMax && vg::cdiv(T, entry_grid(dev, T)) <= vg::kEntryMaxOwn;
}

// The previous layer's combine, when it is folded into this layer's entry.
struct PrevCombine {
  const __nv_bfloat16* x;  // previous layer's input (residual)
  const LayerBufs* b;      // previous layer's buffers (o, inv, gw)
};

// Router, top-k and grouping of a layer whose input is xcur (computed first from
// `prev` when given: decode path only). Large token counts: separate kernels.
// `nbar` counts the grid barriers passed on b.gbar since it was zeroed (host side:
// every launch passes the same number, so it is known without reading the device).
// Bytes of expert weights the layer entry prefetches into L2: the gate|up rows
// of the first routed experts, which the expert kernel's first wave of units
// streams (about one unit per SM).

// Launch of a decode-path kernel with programmatic stream serialization (the
// kernel waits for its predecessor itself, see griddep_wait), plain or
// cooperative.
enum class Launch { kPlain, kCooperative };  // a distinct type: no argument converts to it by accident
template <typename... KArgs, typename... Args>
cudaError_t launch_dep(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t s, Launch kind,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kind == Launch::kCooperative ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

vg_status launch_entry(DevState* dev, int T, const PrevCombine* prev, const __nv_bfloat16* x_in,
                       __nv_bfloat16* x_out, const void* router_w, const float* router_bias, const void* expert_w,
                       const LayerBufs& b, uint32_t* nbar, cudaStream_t s) {
  using namespace vg;
  const int N = T * kTopK;
  if (small_path(dev, T)) {
    EntryArgs a{};
    if (prev) {
      a.prev_o = prev->b->o;
      a.prev_inv = prev->b->inv;
      a.prev_gate = prev->b->gw;
      a.prev_x = prev->x;
      a.prev_add_residual = 1;
      a.x_out = x_out;
    }
    a.x_in = x_in;
    a.bias = router_bias;
    a.T = T;
    a.k = kTopK;
    a.S = kS;
    a.idx = b.idx;
    a.gate = b.gw;
    a.offsets = b.offsets;
    a.perm = b.perm;
    a.inv = b.inv;
    a.x_perm = b.xperm;
    a.primary_rows = static_first_units(dev, T) ? 64 : 0;
    a.counts = b.ecnt;
    a.sched = b.sched;
    a.sched_len = b.sched_len;
    a.gbar = b.gbar;
    a.gbar_base = *nbar;
    const size_t gu_bytes = (size_t)2 * kI * kH * 2;
    a.prefetch_base = static_cast<const uint8_t*>(expert_w);
    // only when nearly every expert is touched: otherwise most of the prefetched
    // bytes would belong to experts no token chose
    a.n_prefetch = T >= kEntryPrefetchMinT ? (int)min((size_t)kE, kEntryPrefetchBytes / gu_bytes) : 0;
    a.prefetch_bytes = (uint32_t)gu_bytes;
    a.prefetch_stride = (uint64_t)3 * kI * kH * 2;
    if (entry_small_path(dev, T)) {
      const int grid = cdiv(T, kEsTok);
      if (grid > 1) *nbar += 1;
      a.n_prefetch = T >= kEntryPrefetchMinT ? (int)min((size_t)kE, kSmallEntryPrefetchBytes / gu_bytes) : 0;
      ProfScope ps(VG_KERNEL_ROUTER, s);
      if (launch_dep(moe_entry_small<kTopK>, grid, kEsThreads, 0, s, Launch::kCooperative,
                     static_cast<const __nv_bfloat16*>(router_w), a) != cudaSuccess)
        return cuda_fail();
      return VG_OK;
    }
    const int grid = entry_grid(dev, T);
    if (grid > 1) *nbar += 1;
    CUtensorMap mR, mGu;
    const uint64_t dR[2] = {kH, kE}, sR[1] = {kH * 2};
    const uint32_t bR[2] = {64, kE};
    if (make_map(&mR, router_w, 2, dR, sR, bR)) return VG_ERR_CUDA;
    // tile prefetch of the expert kernel's first wave (its fixed first units)
    // when those units are fixed; the map is the expert kernel's gate/up view
    const uint64_t dGu[4] = {kH, kI, 2, kE};
    const uint64_t sGu[3] = {kH * 2, (uint64_t)kI * kH * 2, (uint64_t)3 * kI * kH * 2};
    const uint32_t bGu[4] = {kBK, kBM, 2, 1};
    if (make_map(&mGu, expert_w, 4, dGu, sGu, bGu)) return VG_ERR_CUDA;
    if (static_first_units(dev, T)) {
      a.pf_mblk = kI / kBM;
      a.pf_units = std::min(std::min(dev->sms, VG_ENTRY_PF_UNITS), kE * a.pf_mblk);
      a.pf_chunks = VG_ENTRY_PF_CHUNKS;
    }
    ProfScope ps(VG_KERNEL_ROUTER, s);
    if (launch_dep(moe_layer_entry<kTopK>, grid, kEntryThreads, layer_entry_smem(), s, Launch::kCooperative, mR, mGu,
                   a) != cudaSuccess)
      return cuda_fail();
    return VG_OK;
  }
  const __nv_bfloat16* xcur = x_in;
  if (prev) {
    moe_combine<false><<<cdiv(T * (kH / 8), 256), 256, 0, s>>>(prev->x, prev->b->o, prev->b->inv, prev->b->gw, T,
                                                              kH, kTopK, kS, 1, x_out);
    xcur = x_out;
  }
  {
    ProfScope ps(VG_KERNEL_ROUTER, s);
    router_topk_tiled<kTopK><<<cdiv(T, 128), 256, kRtPartBytes, s>>>(xcur, static_cast<const __nv_bfloat16*>(router_w),
                                                                     router_bias, T, kH, b.idx, b.gw);
  }
  if (cudaGetLastError() != cudaSuccess) return VG_ERR_CUDA;
  {
    ProfScope ps(VG_KERNEL_GROUPING, s);
    const int nch = cdiv(N, kSortChunk);
    expert_hist_chunks<<<nch, 1024, 0, s>>>(b.idx, N, b.ccnt);
    expert_scan_chunks<<<1, 1024, 0, s>>>(b.ccnt, nch, N, b.offsets, b.cbase, b.sched, b.sched_len);
    expert_scatter_chunks<<<nch, 1024, 0, s>>>(b.idx, N, kTopK, b.cbase, b.perm, b.inv, xcur, kH, b.xperm);
  }
  if (cudaGetLastError() != cudaSuccess) return VG_ERR_CUDA;
  return VG_OK;
}

// Expert GEMMs (gate/up + SwiGLU, down) of a layer with input x.
vg_status launch_experts(DevState* dev, int T, const void* x, const void* expert_w, const void* shared_w,
                         const LayerBufs& b, cudaStream_t s) {
  using namespace vg;
  const int N = T * kTopK;
  const uint64_t estride = (uint64_t)3 * kI * kH * 2;
  const __nv_bfloat16* dr = static_cast<const __nv_bfloat16*>(expert_w) + (size_t)2 * kI * kH;
  const __nv_bfloat16* dsh = static_cast<const __nv_bfloat16*>(shared_w) + (size_t)2 * kI * kH;
  CUtensorMap mGuR, mGuS, mDnR, mDnS, mXr, mXs, mAct;
  // gate/up as (k, row, gate|up, expert): one box = the gate and up tiles of a row block
  const uint64_t dGu[4] = {kH, kI, 2, kE}, dGuS[4] = {kH, kI, 2, kS};
  const uint64_t sGu[3] = {kH * 2, (uint64_t)kI * kH * 2, estride};
  const uint32_t bGu[4] = {kBK, kBM, 2, 1};
  // down as (k, row, expert): one box = 256 rows, two M tiles
  const uint64_t dDn[3] = {kI, kH, kE}, dDnS[3] = {kI, kH, kS}, sDn[2] = {kI * 2, estride};
  const uint32_t bDn[3] = {kBK, 2 * kBM, 1};
  const uint64_t dXr[2] = {kH, (uint64_t)(N + (static_first_units(dev, T) ? kE * 64 : 0))}, dXs[2] = {kH, (uint64_t)T}, sX[1] = {kH * 2};
  const uint64_t dAct[2] = {kI, (uint64_t)(kTopK + kS) * T}, sAct[1] = {kI * 2};
  const int nt = expert_tile(T);
  // token-major kernel (128-token tiles): its token operand is one 128-row box;
  // otherwise a box never exceeds the token slot
#ifndef VG_PREFILL_WEIGHT_MAJOR
  const bool tm = nt == 128;
#else
  const bool tm = false;
#endif
  const int bx = tm ? kTmM : std::min(kBoxRows, nt);
  const uint32_t bXr[2] = {kBK, (uint32_t)box_rows(N, bx)};
  const uint32_t bXs[2] = {kBK, (uint32_t)box_rows(T, bx)};
  const uint32_t bAct[2] = {kBK, (uint32_t)box_rows((int64_t)(kTopK + kS) * T, bx)};
  if (make_map(&mGuR, expert_w, 4, dGu, sGu, bGu) || make_map(&mGuS, shared_w, 4, dGuS, sGu, bGu) ||
      make_map(&mDnR, dr, 3, dDn, sDn, bDn) || make_map(&mDnS, dsh, 3, dDnS, sDn, bDn) ||
      make_map(&mXr, b.xperm, 2, dXr, sX, bXr) || make_map(&mXs, x, 2, dXs, sX, bXs) ||
      make_map(&mAct, b.act, 2, dAct, sAct, bAct))
    return VG_ERR_CUDA;
  FusedArgs a{};
  a.offsets = b.offsets;
  a.T = T;
  a.E = kE;
  a.S = kS;
  a.mblk_gu = kI / kBM;
  a.mblk_dn = kH / (2 * kBM);
  a.kc_gu = kH / kBK;
  a.kc_dn = kI / kBK;
  a.box_xr = (int)bXr[1];
  a.box_xs = (int)bXs[1];
  a.box_act = (int)bAct[1];
  a.sched = b.sched;
  a.act = b.act;
  a.out = b.o;
  const int grid = expert_grid(dev, T);
  a.static_first = static_first_units(dev, T) ? 1 : 0;
  a.pre_l2_chunks = kPreL2Chunks;
  ProfScope ps(VG_KERNEL_EXPERTS, s);
  const cudaError_t e =
      tm ? launch_dep(moe_expert_gemms_tm, grid, 192, kTmSmemBytes, s, Launch::kPlain, mGuR, mGuS, mDnR, mDnS, mXr,
                      mXs, mAct, a)
      : nt == 16
          ? launch_dep(moe_expert_gemms<16>, grid, 192, FgCfg<16>::kSmemBytes, s, Launch::kPlain, mGuR, mGuS, mDnR, mDnS, mXr,
                       mXs, mAct, a)
      : nt == 64
          ? launch_dep(moe_expert_gemms<64>, grid, 192, FgCfg<64>::kSmemBytes, s, Launch::kPlain, mGuR, mGuS, mDnR, mDnS, mXr,
                       mXs, mAct, a)
          : launch_dep(moe_expert_gemms<128>, grid, 192, FgCfg<128>::kSmemBytes, s, Launch::kPlain, mGuR, mGuS, mDnR, mDnS,
                       mXr, mXs, mAct, a);
  return e == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

vg_status launch_combine(int T, const void* x, const LayerBufs& b, int add_residual, void* out, cudaStream_t s) {
  using namespace vg;
  ProfScope ps(VG_KERNEL_COMBINE, s);
  // few tokens: every load of a thread at once (latency); many: one row at a time (throughput)
  const cudaError_t e = launch_dep(T <= kCombineAllLoadsMaxT ? moe_combine<true> : moe_combine<false>,
                                   cdiv(T * (kH / 8), 256), 256, 0, s, Launch::kPlain,
                                   static_cast<const __nv_bfloat16*>(x), (const __nv_bfloat16*)b.o,
                                   (const int32_t*)b.inv, (const float*)b.gw, T, kH, kTopK, kS, add_residual,
                                   static_cast<__nv_bfloat16*>(out));
  return e == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

// One layer: entry, expert GEMMs, combine into out.
vg_status launch_moe(DevState* dev, int T, const void* x, const void* router_w, const float* router_bias,
                     const void* expert_w, const void* shared_w, int add_residual, void* out,
                     const vg_moe_taps* taps, void* workspace, cudaStream_t s) {
  const LayerBufs b = carve(workspace, T, taps);
  if (cudaMemsetAsync(b.gbar, 0, 8, s) != cudaSuccess) return cuda_fail();
  uint32_t nbar = 0;
  vg_status st = launch_entry(dev, T, nullptr, static_cast<const __nv_bfloat16*>(x), nullptr, router_w, router_bias,
                              expert_w, b, &nbar, s);
  if (st == VG_OK) st = launch_experts(dev, T, x, expert_w, shared_w, b, s);
  if (st == VG_OK) st = launch_combine(T, x, b, add_residual, out, s);
  return st;
}

// Verify workspace: the running argmax key of every row, then the CTA counter.
size_t verify_ws_bytes(int B, int K, int V) {
  (void)V;
  const size_t R = (size_t)B * (K + 1);
  return align256(R * 8) + 256;
}

// The fused LM head + argmax + accept launch. `best` [R] and `done` must be
// zero; the kernel leaves them zero.
vg_status launch_verify(DevState* dev, int B, int K, int V, const void* h, const void* lm_head, const int32_t* drafts,
                        int32_t* argmax, int32_t* accepted, int32_t* out_tokens, unsigned long long* best,
                        uint32_t* done, cudaStream_t s) {
  using namespace vg;
  const int R = B * (K + 1);
  LmArgs a{};
  a.R = R;
  a.V = V;
  a.k_chunks = kH / kBK;
  a.n_mblk = cdiv(R, kLmM);
  a.n_vblk = cdiv(V, kLmN);
  a.group_tiles = kLmGroupTiles;
  a.n_groups = cdiv(a.n_vblk, kLmGroupTiles);
  a.a_box_rows = box_rows(R, kLmM);
  a.b_box_rows = box_rows(V, kLmN);
  a.B = B;
  a.K = K;
  a.drafts = drafts;
  a.argmax = argmax;
  a.accepted = accepted;
  a.out_tokens = out_tokens;
  a.best = best;
  a.done = done;
  CUtensorMap mH, mLM;
  {
    const uint64_t dH[2] = {(uint64_t)kH, (uint64_t)R}, sH[1] = {(uint64_t)kH * 2};
    const uint32_t bH[2] = {kBK, (uint32_t)a.a_box_rows};
    const uint64_t dL[2] = {(uint64_t)kH, (uint64_t)V};
    const uint32_t bL[2] = {kBK, (uint32_t)a.b_box_rows};
    if (make_map(&mH, h, 2, dH, sH, bH) || make_map(&mLM, lm_head, 2, dL, sH, bL)) return VG_ERR_CUDA;
  }
  const int grid = min(dev->sms, a.n_mblk * a.n_groups);
  ProfScope ps(VG_KERNEL_LM_HEAD, s);
  if (launch_dep(lmhead_argmax_accept, grid, 192, kLmSmemBytes, s, Launch::kPlain, mH, mLM, a) != cudaSuccess)
    return cuda_fail();
  return VG_OK;
}

}  // namespace

extern "C" {

const char* vg_status_string(vg_status s) {
  switch (s) {
    case VG_OK: return "VG_OK";
    case VG_ERR_INVALID_ARG: return "VG_ERR_INVALID_ARG";
    case VG_ERR_UNSUPPORTED: return "VG_ERR_UNSUPPORTED";
    case VG_ERR_WORKSPACE: return "VG_ERR_WORKSPACE";
    case VG_ERR_CUDA: return "VG_ERR_CUDA";
    case VG_ERR_TIMEOUT: return "VG_ERR_TIMEOUT";
    case VG_ERR_DEVICE_BOUNDS: return "VG_ERR_DEVICE_BOUNDS";
  }
  return "VG_UNKNOWN";
}

int32_t vg_abi_version(void) { return 2; }

size_t vg_moe_workspace_bytes(const vg_moe_dims* dims, int32_t T_max) {
  if (dims == nullptr || !dims_supported(dims) || T_max < 0) return 0;
  return moe_layout(T_max > 0 ? T_max : 1).total;
}

static vg_status validate_moe(const vg_moe_dims* dims, int32_t T, const void* x, const void* router_w,
                              const void* expert_w, const void* shared_w, void* out, void* workspace,
                              size_t workspace_bytes) {
  if (dims == nullptr || T < 0) return VG_ERR_INVALID_ARG;
  if (!dims_supported(dims)) return VG_ERR_UNSUPPORTED;
  if (T > (1 << 22)) return VG_ERR_UNSUPPORTED;
  if (T == 0) return VG_OK;
  if (!x || !router_w || !expert_w || !shared_w || !out) return VG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(router_w) || !aligned16(expert_w) || !aligned16(shared_w) || !aligned16(out))
    return VG_ERR_INVALID_ARG;
  const size_t need = moe_layout(T).total;
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return VG_ERR_WORKSPACE;
  const size_t row_bytes = (size_t)T * kH * 2;
  if (overlaps(out, row_bytes, x, row_bytes) || overlaps(out, row_bytes, workspace, workspace_bytes))
    return VG_ERR_INVALID_ARG;
  return VG_OK;
}

vg_status vg_moe_ffn(const vg_moe_dims* dims, int32_t T, const void* x, const void* router_w,
                     const float* router_bias, const void* expert_w, const void* shared_w, int32_t add_residual,
                     void* out, const vg_moe_taps* taps, void* workspace, size_t workspace_bytes,
                     vg_stream_t stream) {
  vg_status st = validate_moe(dims, T, x, router_w, expert_w, shared_w, out, workspace, workspace_bytes);
  if (st != VG_OK || T == 0) return st;
  DevState* dev = nullptr;
  if ((st = device_state(&dev)) != VG_OK) return st;
  return launch_moe(dev, T, x, router_w, router_bias, expert_w, shared_w, add_residual ? 1 : 0, out, taps,
                    workspace, reinterpret_cast<cudaStream_t>(stream));
}

size_t vg_moe_stack_workspace_bytes(const vg_moe_dims* dims, int32_t T_max) {
  const size_t m = vg_moe_workspace_bytes(dims, T_max);
  if (m == 0) return 0;
  return m + 2 * align256((size_t)(T_max > 0 ? T_max : 1) * kH * 2);
}

vg_status vg_moe_ffn_stack(const vg_moe_dims* dims, int32_t n_layers, int32_t T, const void* x,
                           const void* const* router_w, const float* const* router_bias,
                           const void* const* expert_w, const void* const* shared_w, void* out, void* workspace,
                           size_t workspace_bytes, vg_stream_t stream) {
  if (dims == nullptr || n_layers < 1 || T < 0 || !router_w || !expert_w || !shared_w) return VG_ERR_INVALID_ARG;
  if (!dims_supported(dims)) return VG_ERR_UNSUPPORTED;
  if (T == 0) return VG_OK;
  const size_t mw = moe_layout(T).total;
  const size_t hb = align256((size_t)T * kH * 2);
  if (workspace == nullptr || workspace_bytes < mw + 2 * hb) return VG_ERR_WORKSPACE;
  for (int l = 0; l < n_layers; ++l)
    if (!router_w[l] || !expert_w[l] || !shared_w[l] || !aligned16(router_w[l]) || !aligned16(expert_w[l]) ||
        !aligned16(shared_w[l]))
      return VG_ERR_INVALID_ARG;
  vg_status st = validate_moe(dims, T, x, router_w[0], expert_w[0], shared_w[0], out, workspace, workspace_bytes);
  if (st != VG_OK) return st;
  DevState* dev = nullptr;
  if ((st = device_state(&dev)) != VG_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* buf[2] = {reinterpret_cast<__nv_bfloat16*>(ws + mw), reinterpret_cast<__nv_bfloat16*>(ws + mw + hb)};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // x_0 = x; x_l (l >= 1) = buf[(l-1) & 1] is computed by layer l's entry from
  // layer l-1's expert outputs; the last layer's combine writes out.
  const LayerBufs b = carve(workspace, T, nullptr);
  if (cudaMemsetAsync(b.gbar, 0, 8, s) != cudaSuccess) return cuda_fail();
  uint32_t nbar = 0;
  const __nv_bfloat16* xin = static_cast<const __nv_bfloat16*>(x);
  for (int l = 0; l < n_layers; ++l) {
    const __nv_bfloat16* xl = xin;
    PrevCombine prev{xin, &b};
    __nv_bfloat16* xout = nullptr;
    if (l > 0) {
      xout = buf[(l - 1) & 1];
      xl = xout;
    }
    st = launch_entry(dev, T, l > 0 ? &prev : nullptr, xin, xout, router_w[l], router_bias ? router_bias[l] : nullptr,
                      expert_w[l], b, &nbar, s);
    if (st == VG_OK) st = launch_experts(dev, T, xl, expert_w[l], shared_w[l], b, s);
    if (st != VG_OK) return st;
    xin = xl;
  }
  st = launch_combine(T, xin, b, 1, out, s);
  if (st != VG_OK) return st;
  return VG_OK;
}

size_t vg_verify_workspace_bytes(int32_t B, int32_t K, int32_t H, int32_t V) {
  if (B < 0 || K < 0 || K > 255 || H != kH || V < 1) return 0;
  if ((int64_t)B * (K + 1) >= (1 << 24)) return 0;
  return verify_ws_bytes(B > 0 ? B : 1, K, V);
}

vg_status vg_verify_greedy(int32_t B, int32_t K, int32_t H, int32_t V, const void* h, const void* lm_head,
                           const int32_t* drafts, int32_t* argmax, int32_t* accepted, int32_t* out_tokens,
                           void* workspace, size_t workspace_bytes, vg_stream_t stream) {
  using namespace vg;
  if (B < 0 || K < 0 || V < 1) return VG_ERR_INVALID_ARG;
  if (H != kH || K > 255 || (int64_t)B * (K + 1) >= (1 << 24)) return VG_ERR_UNSUPPORTED;
  if (B == 0) return VG_OK;
  if (!h || !lm_head || !argmax || !accepted || !out_tokens || (K > 0 && !drafts)) return VG_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(lm_head)) return VG_ERR_INVALID_ARG;
  const int R = B * (K + 1);
  if (workspace == nullptr || workspace_bytes < verify_ws_bytes(B, K, V) || !aligned16(workspace))
    return VG_ERR_WORKSPACE;
  DevState* dev = nullptr;
  vg_status st = device_state(&dev);
  if (st != VG_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return launch_verify(dev, B, K, V, h, lm_head, drafts, argmax, accepted, out_tokens,
                       reinterpret_cast<unsigned long long*>(ws),
                       reinterpret_cast<uint32_t*>(ws + align256((size_t)R * 8)), reinterpret_cast<cudaStream_t>(stream));
}

vg_status vg_get_device_status(vg_stream_t stream, int32_t* info) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return cuda_fail();
  int32_t st = 0, inf = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&st, vg::g_status, sizeof(st)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&inf, vg::g_status_info, sizeof(inf)) != cudaSuccess ||
      cudaMemcpyToSymbol(vg::g_status, &zero, sizeof(zero)) != cudaSuccess ||
      cudaMemcpyToSymbol(vg::g_status_info, &zero, sizeof(zero)) != cudaSuccess)
    return cuda_fail();
  if (info) *info = inf;
  return static_cast<vg_status>(st);
}

vg_status vg_profile_set_events(int32_t kind, const vg_event_t* starts, const vg_event_t* stops, int32_t n) {
  if (kind < 0 || kind >= VG_KERNEL_KINDS || n < 0 || (n > 0 && (!starts || !stops))) return VG_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (!starts[i] || !stops[i]) return VG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ProfHook& h = g_prof[kind];
  h.starts.assign(reinterpret_cast<const cudaEvent_t*>(starts), reinterpret_cast<const cudaEvent_t*>(starts) + n);
  h.stops.assign(reinterpret_cast<const cudaEvent_t*>(stops), reinterpret_cast<const cudaEvent_t*>(stops) + n);
  h.count = 0;
  bool any = false;
  for (auto& k : g_prof) any = any || !k.starts.empty();
  g_prof_any = any;
  return VG_OK;
}

int64_t vg_profile_count(int32_t kind) {
  if (kind < 0 || kind >= VG_KERNEL_KINDS) return -1;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return g_prof[kind].count;
}

vg_status vg_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) return VG_ERR_INVALID_ARG;
  if (cudaMemcpyToSymbol(vg::g_wait_timeout_ns, &ns, sizeof(ns)) != cudaSuccess) return cuda_fail();
  return VG_OK;
}

}  // extern "C"

namespace vg {
__global__ void debug_wait_flag_kernel(const int32_t* flag, int32_t expect, uint64_t max_ns) {
  const uint64_t t0 = globaltimer();
  while (true) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v == expect) return;
    if (globaltimer() - t0 > max_ns) {
      record_error(kErrTimeout, 901);
      return;
    }
    __nanosleep(1000);
  }
}
}  // namespace vg

extern "C" vg_status vg_debug_wait_flag(const int32_t* flag, int32_t expect, uint64_t max_ns, vg_stream_t stream) {
  if (flag == nullptr || max_ns == 0 || max_ns > 60000000000ull) return VG_ERR_INVALID_ARG;
  vg::debug_wait_flag_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(flag, expect, max_ns);
  return cudaGetLastError() == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

namespace vg {
// The pipeline-stage wait (mbar_wait) and the grid barrier, each made to run
// out: no copy, MMA or other CTA's work is in flight when they give up.
__global__ void debug_wait_site_kernel(int32_t which, uint32_t* ctr, uint64_t max_ns) {
  if (which == VG_WAIT_MBARRIER) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
      mbar_init(&bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, max_ns)) record_error(kErrTimeout, 903);
  } else {
    grid_barrier(ctr, gridDim.x + 1, max_ns, 902);  // one arrival more than the grid has CTAs
  }
}
}  // namespace vg

extern "C" vg_status vg_debug_wait_site(int32_t which, uint32_t* ctr, uint64_t max_ns, vg_stream_t stream) {
  if ((which != VG_WAIT_MBARRIER && which != VG_WAIT_GRID_BARRIER) || max_ns == 0 || max_ns > 60000000000ull)
    return VG_ERR_INVALID_ARG;
  if (which == VG_WAIT_GRID_BARRIER && (ctr == nullptr || (reinterpret_cast<uintptr_t>(ctr) & 3u) != 0))
    return VG_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (which == VG_WAIT_MBARRIER) {
    vg::debug_wait_site_kernel<<<1, 32, 0, s>>>(which, ctr, max_ns);
    return cudaGetLastError() == cudaSuccess ? VG_OK : cuda_fail();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, vg::debug_wait_site_kernel, which, ctr, max_ns) == cudaSuccess ? VG_OK
                                                                                                : cuda_fail();
}

// ------------------------------------------------------------------ no-alloc
// Scratch of vg_verify_greedy_noalloc: a file-scope device array (its host-side
// name is only a stand-in; the device address comes from cudaGetSymbolAddress).
namespace {
constexpr size_t kNoAllocKeys = VG_NOALLOC_SCRATCH_BYTES / sizeof(uint64_t);
constexpr size_t kNoAllocCounterSlots = 1;  // the last slot holds the CTA counter
static __device__ __align__(256) uint64_t g_noalloc_scratch[kNoAllocKeys];
uint64_t* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Once per device, with that device current: the array's device address.
vg_status noalloc_scratch(uint64_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail();
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return cuda_fail();
    g_noalloc_ptr[dev] = static_cast<uint64_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return VG_OK;
}
}  // namespace

extern "C" vg_status vg_verify_greedy_noalloc(int32_t B, int32_t K, int32_t H, int32_t V, const void* h,
                                              const void* lm_head, const int32_t* drafts, int32_t* argmax,
                                              int32_t* accepted, int32_t* out_tokens, vg_stream_t stream) {
  using namespace vg;
  if (B < 0 || K < 0 || V < 1) return VG_ERR_INVALID_ARG;
  if (H != kH || K > 255 || (int64_t)B * (K + 1) >= (1 << 24)) return VG_ERR_UNSUPPORTED;
  if (B == 0) return VG_OK;
  if (!h || !lm_head || !argmax || !accepted || !out_tokens || (K > 0 && !drafts)) return VG_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(lm_head)) return VG_ERR_INVALID_ARG;
  const int R = B * (K + 1);
  if ((uint64_t)R > kNoAllocKeys - kNoAllocCounterSlots) return VG_ERR_WORKSPACE;
  DevState* dev = nullptr;
  vg_status st = device_state(&dev);
  if (st != VG_OK) return st;
  uint64_t* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != VG_OK) return st;
  // keys in the first R slots, the CTA counter in the last slot: both zero at
  // load time, and every call leaves them zero
  return launch_verify(dev, B, K, V, h, lm_head, drafts, argmax, accepted, out_tokens,
                       reinterpret_cast<unsigned long long*>(scratch),
                       reinterpret_cast<uint32_t*>(scratch + kNoAllocKeys - 1), reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------ decode loop
namespace {
bool spec_state_ok(const vg_spec_state* st) {
  if (st == nullptr || st->B < 0 || st->K < 0 || st->K > 64 || st->V <= 0 || st->cap < 0 || st->ref_len < 0)
    return false;
  if (!(st->p >= 0.0f && st->p <= 1.0f)) return false;
  if (st->B == 0) return true;
  if (!st->last || !st->pos || !st->step || !st->tokens || (st->cap > 0 && !st->committed)) return false;
  if (st->K > 0 && !st->drafts) return false;
  if (st->ref_len > 0 && !st->ref) return false;
  return true;
}
vg::SpecState spec_dev(const vg_spec_state* st) {
  vg::SpecState s{};
  s.B = st->B;
  s.K = st->K;
  s.V = st->V;
  s.last = st->last;
  s.pos = st->pos;
  s.committed = st->committed;
  s.cap = st->cap;
  s.ref = st->ref;
  s.ref_len = st->ref_len;
  s.p = st->p;
  s.seed = st->seed;
  s.step = st->step;
  s.tokens = st->tokens;
  s.drafts = st->drafts;
  return s;
}
}  // namespace

extern "C" vg_status vg_embed_rows(const int32_t* tokens, int32_t n, const void* emb, int32_t V, int32_t H, void* out,
                                   vg_stream_t stream) {
  if (n < 0 || V <= 0 || H <= 0 || H % 8 != 0) return VG_ERR_INVALID_ARG;
  if (n == 0) return VG_OK;
  if (!tokens || !emb || !out || !aligned16(emb) || !aligned16(out)) return VG_ERR_INVALID_ARG;
  if (overlaps(emb, (size_t)V * H * 2, out, (size_t)n * H * 2)) return VG_ERR_INVALID_ARG;
  const cudaError_t e = launch_dep(vg::embed_rows, vg::cdiv(n, 8), 256, 0, reinterpret_cast<cudaStream_t>(stream), Launch::kPlain,
                                   tokens, (int)n, static_cast<const __nv_bfloat16*>(emb), (int)V, (int)H,
                                   static_cast<__nv_bfloat16*>(out));
  return e == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

extern "C" vg_status vg_spec_rows(const vg_spec_state* st, vg_stream_t stream) {
  if (!spec_state_ok(st)) return VG_ERR_INVALID_ARG;
  if (st->B == 0) return VG_OK;
  const cudaError_t e = launch_dep(vg::spec_rows, vg::cdiv(st->B, 128), 128, 0, reinterpret_cast<cudaStream_t>(stream),
                                   Launch::kPlain, spec_dev(st));
  return e == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

extern "C" vg_status vg_spec_commit(const vg_spec_state* st, const int32_t* accepted, const int32_t* out_tokens,
                                    vg_stream_t stream) {
  if (!spec_state_ok(st) || (st->B > 0 && (!accepted || !out_tokens))) return VG_ERR_INVALID_ARG;
  if (st->B == 0) return VG_OK;
  const cudaError_t e = launch_dep(vg::spec_commit, vg::cdiv(st->B, 128), 128, 0,
                                   reinterpret_cast<cudaStream_t>(stream), Launch::kPlain, spec_dev(st), accepted, out_tokens);
  return e == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

extern "C" vg_status vg_spec_rows_given(const vg_spec_state* st, vg_stream_t stream) {
  if (!spec_state_ok(st)) return VG_ERR_INVALID_ARG;
  if (st->B == 0) return VG_OK;
  const cudaError_t e = launch_dep(vg::spec_rows_given, vg::cdiv(st->B, 128), 128, 0,
                                   reinterpret_cast<cudaStream_t>(stream), Launch::kPlain, spec_dev(st));
  return e == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

// ------------------------------------------------------------ draft block
namespace {
// One dense product y = W x on the expert GEMM kernel, as a single shared
// expert over T token rows (no routed experts, offsets[0] = 0):
//  * with_gu: w is an expert block (gate | up | down), x the [T, H] input rows,
//    act a [T, I] scratch for the SwiGLU activations: out = FFN(x);
//  * otherwise w is [n_out, k_dn] (n_out a multiple of 256) and acts as the
//    down projection of a unit list with no gate/up units (no readiness to wait
//    for): out [T, n_out] = act w^T, act the [T, k_dn] input rows.
vg_status launch_dense(DevState* dev, int T, const void* w, bool with_gu, int k_dn, int n_out, const void* x,
                       void* act, void* out, int32_t* sched, int32_t* zero_offsets, cudaStream_t s) {
  using namespace vg;
  const int nt = expert_tile(T), bx = std::min(kBoxRows, nt);
  const int tiles = cdiv(T, nt);
  const uint64_t block = with_gu ? (uint64_t)3 * kI * kH * 2 : (uint64_t)n_out * k_dn * 2;
  const uint8_t* w8 = static_cast<const uint8_t*>(w);
  const void* wdn = with_gu ? static_cast<const void*>(w8 + (size_t)2 * kI * kH * 2) : w;
  CUtensorMap mGu, mDn, mX, mAct;
  const uint64_t dGu[4] = {kH, kI, 2, 1}, sGu[3] = {kH * 2, (uint64_t)kI * kH * 2, (uint64_t)3 * kI * kH * 2};
  const uint32_t bGu[4] = {kBK, kBM, 2, 1};
  const uint64_t dDn[3] = {(uint64_t)k_dn, (uint64_t)n_out, 1}, sDn[2] = {(uint64_t)k_dn * 2, block};
  const uint32_t bDn[3] = {kBK, 2 * kBM, 1};
  const void* xs = with_gu ? x : act;  // without gate/up the x map is never read
  const uint64_t dX[2] = {kH, (uint64_t)T}, sX[1] = {(uint64_t)(with_gu ? kH : k_dn) * 2};
  const uint32_t bX[2] = {kBK, (uint32_t)box_rows(T, bx)};
  const uint64_t dAct[2] = {(uint64_t)k_dn, (uint64_t)T}, sAct[1] = {(uint64_t)k_dn * 2};
  const uint32_t bAct[2] = {kBK, (uint32_t)box_rows(T, bx)};
  // without gate/up the gate/up map is never read either: any valid map will do
  if (make_map(&mGu, with_gu ? w : wdn, 4, dGu, sGu, bGu) || make_map(&mDn, wdn, 3, dDn, sDn, bDn) ||
      make_map(&mX, xs, 2, dX, sX, bX) || make_map(&mAct, act, 2, dAct, sAct, bAct))
    return VG_ERR_CUDA;
  FusedArgs a{};
  a.offsets = zero_offsets;
  a.T = T;
  a.E = 0;
  a.S = 1;
  a.mblk_gu = with_gu ? kI / kBM : 0;
  a.mblk_dn = n_out / (2 * kBM);
  a.kc_gu = kH / kBK;
  a.kc_dn = k_dn / kBK;
  a.box_xr = (int)bX[1];
  a.box_xs = (int)bX[1];
  a.box_act = (int)bAct[1];
  a.sched = sched;
  a.act = static_cast<__nv_bfloat16*>(act);
  a.out = static_cast<__nv_bfloat16*>(out);
  if (cudaMemsetAsync(sched, 0, (size_t)(1 + tiles) * 4, s) != cudaSuccess) return cuda_fail();
  const int grid = min(dev->sms, (a.mblk_gu + a.mblk_dn) * tiles);
  auto go = [&](auto kern, int smem) {
    return launch_dep(kern, grid, 192, smem, s, Launch::kPlain, mGu, mGu, mDn, mDn, mX, mX, mAct, a);
  };
  const cudaError_t e = nt == 16   ? go(moe_expert_gemms<16>, FgCfg<16>::kSmemBytes)
                        : nt == 64 ? go(moe_expert_gemms<64>, FgCfg<64>::kSmemBytes)
                                   : go(moe_expert_gemms<128>, FgCfg<128>::kSmemBytes);
  return e == cudaSuccess ? VG_OK : VG_ERR_CUDA;
}

struct MtpWs {
  size_t u, z, zn, act, o, g, sched, zero, arg, acc, tok, vws, total;
};
MtpWs mtp_layout(int B, int V) {
  MtpWs L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.u = take((size_t)B * 2 * kH * 2);
  L.z = take((size_t)B * kH * 2);
  L.zn = take((size_t)B * kH * 2);
  L.act = take((size_t)B * kI * 2);
  L.o = take((size_t)B * kH * 2);
  L.g = take((size_t)B * kH * 2);
  L.sched = take((size_t)(2 + vg::cdiv(B, 16)) * 4);
  L.zero = take(16);
  L.arg = take((size_t)B * 4);
  L.acc = take((size_t)B * 4);
  L.tok = take((size_t)B * 4);
  L.vws = take(verify_ws_bytes(B, 0, V));
  L.total = off;
  return L;
}
}  // namespace

extern "C" size_t vg_mtp_workspace_bytes(int32_t B, int32_t V) {
  if (B < 0 || V < 1) return 0;
  return mtp_layout(B, V).total;
}

extern "C" vg_status vg_mtp_draft(int32_t B, int32_t K, const vg_mtp_weights* w, const void* h, int32_t rows_per_seq,
                                  const int32_t* accepted, const int32_t* y0, int32_t* drafts, void* hidden_out,
                                  void* workspace, size_t workspace_bytes, vg_stream_t stream) {
  using namespace vg;
  if (B < 0 || K < 0 || w == nullptr || w->V < 1 || rows_per_seq < 1) return VG_ERR_INVALID_ARG;
  if (B == 0 || K == 0) return VG_OK;
  if (!w->proj || !w->ffn || !w->gamma_h || !w->gamma_e || !w->gamma_f || !w->emb || !w->lm_head || !h || !y0 ||
      !drafts)
    return VG_ERR_INVALID_ARG;
  if (!aligned16(w->proj) || !aligned16(w->ffn) || !aligned16(w->emb) || !aligned16(w->lm_head) || !aligned16(h) ||
      !aligned16(hidden_out))
    return VG_ERR_INVALID_ARG;
  const MtpWs L = mtp_layout(B, w->V);
  if (workspace == nullptr || workspace_bytes < L.total || !aligned16(workspace)) return VG_ERR_WORKSPACE;
  DevState* dev = nullptr;
  vg_status st = device_state(&dev);
  if (st != VG_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto bf = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(ws + o); };
  auto i32 = [&](size_t o) { return reinterpret_cast<int32_t*>(ws + o); };
  // zero offsets of the dense products, and the verify workspace (the LM-head
  // kernel needs it zero-filled and leaves it so)
  if (cudaMemsetAsync(ws + L.zero, 0, 16, s) != cudaSuccess ||
      cudaMemsetAsync(ws + L.vws, 0, verify_ws_bytes(B, 0, w->V), s) != cudaSuccess)
    return cuda_fail();
  // g_i: in the caller's hidden_out when given, else in the workspace
  auto g_of = [&](int i) {
    return hidden_out ? static_cast<__nv_bfloat16*>(hidden_out) + (size_t)(i - 1) * B * kH : bf(L.g);
  };
  for (int i = 1; i <= K; ++i) {
    MtpPrep p{};
    p.g = i == 1 ? static_cast<const __nv_bfloat16*>(h) : g_of(i - 1);
    p.rows_per_seq = i == 1 ? rows_per_seq : 1;
    p.acc = i == 1 ? accepted : nullptr;
    p.y = i == 1 ? y0 : i32(L.arg);
    p.emb = static_cast<const __nv_bfloat16*>(w->emb);
    p.V = w->V;
    p.H = kH;
    p.gamma_h = w->gamma_h;
    p.gamma_e = w->gamma_e;
    p.u = bf(L.u);
    p.drafts = i == 1 ? nullptr : drafts;
    p.K = K;
    p.slot = i - 2;
    if (launch_dep(mtp_prep, B, kMtpThreads, 0, s, Launch::kPlain, p) != cudaSuccess) return cuda_fail();
    if ((st = launch_dense(dev, B, w->proj, false, 2 * kH, kH, nullptr, bf(L.u), bf(L.z), i32(L.sched),
                           i32(L.zero), s)) != VG_OK)
      return st;
    if (launch_dep(mtp_rmsnorm, B, kMtpThreads, 0, s, Launch::kPlain, (const __nv_bfloat16*)bf(L.z), w->gamma_f,
                   (int)kH, bf(L.zn)) != cudaSuccess)
      return cuda_fail();
    if ((st = launch_dense(dev, B, w->ffn, true, kI, kH, bf(L.zn), bf(L.act), bf(L.o), i32(L.sched), i32(L.zero),
                           s)) != VG_OK)
      return st;
    if (launch_dep(mtp_residual, cdiv(B * kH / 8, 256), 256, 0, s, Launch::kPlain, (const __nv_bfloat16*)bf(L.z),
                   (const __nv_bfloat16*)bf(L.o), B * kH, g_of(i)) != cudaSuccess)
      return cuda_fail();
    if ((st = vg_verify_greedy(B, 0, kH, w->V, g_of(i), w->lm_head, nullptr, i32(L.arg), i32(L.acc), i32(L.tok),
                               ws + L.vws, verify_ws_bytes(B, 0, w->V), stream)) != VG_OK)
      return st;
  }
  if (launch_dep(mtp_collect, cdiv(B, 128), 128, 0, s, Launch::kPlain, (const int32_t*)i32(L.arg), (int)B, (int)K,
                 (int)K - 1, drafts) != cudaSuccess)
    return cuda_fail();
  return VG_OK;
}

// ------------------------------------------------------------ verifier attention
namespace {
struct AttnWs {
  size_t pk, q, o, part, total;
};
constexpr int kProjSplits = kH / vg::kPtK;  // partial sums of a projection (5)
AttnWs attn_layout(int B, int K, int L_max) {
  const size_t R = (size_t)B * (K + 1);
  AttnWs L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.pk = take((size_t)kProjSplits * R * 3 * kH * 4);  // projection partials (q/k/v, then the output's)
  L.q = take(R * kH * 2);
  L.o = take(R * kH * 2);
  L.part = take((size_t)B * vg::kAttnHeads * vg::cdiv(L_max, vg::kAttnChunk) * (K + 1) * (2 + vg::kAttnDim) * 4);
  L.total = off;
  return L;
}
}  // namespace

extern "C" size_t vg_attn_workspace_bytes(int32_t B, int32_t K, int32_t L_max) {
  if (B < 0 || K < 0 || K + 1 > vg::kAttnMaxRows || L_max < 1 || L_max > 32768) return 0;
  return attn_layout(B, K, L_max).total;
}

extern "C" vg_status vg_attn_verify(int32_t B, int32_t K, int32_t L_max, const void* x, const void* w_qkv,
                                    const void* w_o, void* kv_cache, const int32_t* lens, void* out, void* o_out,
                                    void* workspace, size_t workspace_bytes, vg_stream_t stream) {
  using namespace vg;
  if (B < 0 || K < 0 || K + 1 > kAttnMaxRows || L_max < 1 || L_max > 32768) return VG_ERR_INVALID_ARG;
  if (B == 0) return VG_OK;
  // launch sizes count (row, head-pair) items and the cache's rows in int
  if ((int64_t)B * (K + 1) * kH >= ((int64_t)1 << 31) || (int64_t)B * 2 * L_max >= ((int64_t)1 << 31))
    return VG_ERR_UNSUPPORTED;
  if (!x || !w_qkv || !w_o || !kv_cache || !lens || !out) return VG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(w_o) || !aligned16(kv_cache) || !aligned16(out) ||
      !aligned16(o_out))
    return VG_ERR_INVALID_ARG;
  const int R = B * (K + 1);
  const size_t rows_bytes = (size_t)R * kH * 2, cache_bytes = (size_t)B * 2 * L_max * kH * 2;
  if (overlaps(x, rows_bytes, out, rows_bytes) || overlaps(kv_cache, cache_bytes, out, rows_bytes)) return VG_ERR_INVALID_ARG;
  if (o_out && (overlaps(x, rows_bytes, o_out, rows_bytes) || overlaps(out, rows_bytes, o_out, rows_bytes) ||
                overlaps(kv_cache, cache_bytes, o_out, rows_bytes)))
    return VG_ERR_INVALID_ARG;
  const AttnWs L = attn_layout(B, K, L_max);
  if (workspace == nullptr || workspace_bytes < L.total || !aligned16(workspace)) return VG_ERR_WORKSPACE;
  DevState* dev = nullptr;
  vg_status st = device_state(&dev);
  if (st != VG_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto bf = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(ws + o); };
  float* pk = reinterpret_cast<float*>(ws + L.pk);
  // x W^T as fp32 partial sums over the 5 slices of the reduction, on the tensor cores
  auto launch_proj = [&](const void* act, const void* wgt, int n_out) {
    CUtensorMap mW, mX;
    const uint64_t dW[2] = {kH, (uint64_t)n_out}, dX[2] = {kH, (uint64_t)R}, sK[1] = {kH * 2};
    const uint32_t bW[2] = {kBK, kBM}, bX[2] = {kBK, (uint32_t)box_rows(R, kPtRows)};
    if (make_map(&mW, wgt, 2, dW, sK, bW) || make_map(&mX, act, 2, dX, sK, bX)) return cudaErrorInvalidValue;
    cudaLaunchConfig_t pc = {};  // 3-d grid: (128 outputs, 256-wide reduction slice, 128 rows)
    pc.gridDim = dim3(n_out / kBM, kProjSplits, cdiv(R, kPtRows));
    pc.blockDim = dim3(192);
    pc.dynamicSmemBytes = kPtSmemBytes;
    pc.stream = s;
    cudaLaunchAttribute pa[1];
    pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pa[0].val.programmaticStreamSerializationAllowed = 1;
    pc.attrs = pa;
    pc.numAttrs = 1;
    return cudaLaunchKernelEx(&pc, attn_proj_tc, mW, mX, R, n_out, (int)bX[1], pk);
  };
  // q/k/v = x W_qkv^T as split partial sums
  if (launch_proj(x, w_qkv, 3 * kH) != cudaSuccess) return cuda_fail();
  AttnArgs a{};
  a.B = B;
  a.K1 = K + 1;
  a.L_max = L_max;
  a.lens = lens;
  a.qkv_part = pk;
  a.splits = kProjSplits;
  a.q = bf(L.q);
  a.cache = static_cast<__nv_bfloat16*>(kv_cache);
  a.part = reinterpret_cast<float*>(ws + L.part);
  a.n_chunks = cdiv(L_max, kAttnChunk);
  a.o = o_out ? static_cast<__nv_bfloat16*>(o_out) : bf(L.o);
  if (launch_dep(attn_rope_append, cdiv(R * kH / 2, 256), 256, 0, s, Launch::kPlain, a) != cudaSuccess)
    return cuda_fail();
  cudaLaunchConfig_t cfg = {};  // 2-d grid: (sequence x head, chunk)
  cfg.gridDim = dim3(B * kAttnHeads, a.n_chunks);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  {
    ProfScope ps(VG_KERNEL_ATTENTION, s);
    if (cudaLaunchKernelEx(&cfg, attn_chunk, a) != cudaSuccess) return cuda_fail();
  }
  if (launch_dep(attn_merge, B * kAttnHeads * (K + 1), kAttnDim, 0, s, Launch::kPlain, a) != cudaSuccess)
    return cuda_fail();
  // out = x + W_o o: split partials (over the q/k/v partials, consumed by now), then the residual
  if (launch_proj(a.o, w_o, kH) != cudaSuccess) return cuda_fail();
  if (launch_dep(attn_residual, cdiv(R * kH / 4, 256), 256, 0, s, Launch::kPlain, static_cast<const __nv_bfloat16*>(x),
                 (const float*)pk, kProjSplits, R * kH, static_cast<__nv_bfloat16*>(out)) != cudaSuccess)
    return cuda_fail();
  return VG_OK;
}

// ------------------------------------------------------------ small-batch step
namespace {
struct SsWs {
  size_t ctrl, part_gu, part_dn, act, o, total;
};
SsWs ss_layout() {
  using namespace vg;
  SsWs L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.ctrl = take(sizeof(SsCtrl));
  L.part_gu = take((size_t)kSsSlots * kSsMbGu * kSsKsGu * kSsPartFloats * 4);
  L.part_dn = take((size_t)kSsSlots * kSsMbDn * kSsKsDn * kSsPartFloats * 4);
  L.act = take((size_t)kSsSlots * kSsN * kI * 2);
  L.o = take((size_t)kSsSlots * kSsN * kH * 2);
  L.total = off;
  return L;
}
}  // namespace

extern "C" size_t vg_verify_step_small_workspace_bytes(void) { return ss_layout().total; }

extern "C" vg_status vg_verify_step_small(const vg_moe_dims* dims, int32_t n_layers, int32_t B, int32_t K,
                                          const void* x, const void* const* router_w,
                                          const float* const* router_bias, const void* const* expert_w,
                                          const void* const* shared_w, const void* lm_head, int32_t V,
                                          const int32_t* drafts, int32_t* argmax, int32_t* accepted,
                                          int32_t* out_tokens, void* states_out, int32_t* topk_idx_out,
                                          void* workspace, size_t workspace_bytes, vg_stream_t stream) {
  using namespace vg;
  if (dims == nullptr || B < 0 || K < 0 || V < 1 || n_layers < 1 || !router_w || !expert_w || !shared_w)
    return VG_ERR_INVALID_ARG;
  if (!dims_supported(dims) || n_layers > kSsMaxLayers || (int64_t)B * (K + 1) > kSsN) return VG_ERR_UNSUPPORTED;
  if (B == 0) return VG_OK;
  if (!x || !lm_head || !argmax || !accepted || !out_tokens || (K > 0 && !drafts)) return VG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(lm_head) || !aligned16(states_out)) return VG_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!router_w[l] || !expert_w[l] || !shared_w[l] || !aligned16(router_w[l]) || !aligned16(expert_w[l]) ||
        !aligned16(shared_w[l]))
      return VG_ERR_INVALID_ARG;
  const SsWs W = ss_layout();
  if (workspace == nullptr || workspace_bytes < W.total || !aligned16(workspace)) return VG_ERR_WORKSPACE;
  DevState* dev = nullptr;
  vg_status st = device_state(&dev);
  if (st != VG_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  SsMaps maps;
  memset(&maps, 0, sizeof(maps));
  const uint64_t estride = (uint64_t)3 * kI * kH * 2;
  const uint64_t dGu[4] = {kH, kI, 2, kE}, dGuS[4] = {kH, kI, 2, kS};
  const uint64_t sGu[3] = {kH * 2, (uint64_t)kI * kH * 2, estride};
  const uint32_t bGu[4] = {kBK, kBM, 2, 1};
  const uint64_t dDn[3] = {kI, kH, kE}, dDnS[3] = {kI, kH, kS}, sDn[2] = {kI * 2, estride};
  const uint32_t bDn[3] = {kBK, 2 * kBM, 1};
  for (int l = 0; l < n_layers; ++l) {
    const __nv_bfloat16* dr = static_cast<const __nv_bfloat16*>(expert_w[l]) + (size_t)2 * kI * kH;
    const __nv_bfloat16* dsh = static_cast<const __nv_bfloat16*>(shared_w[l]) + (size_t)2 * kI * kH;
    if (make_map(&maps.gu[l][0], expert_w[l], 4, dGu, sGu, bGu) ||
        make_map(&maps.gu[l][1], shared_w[l], 4, dGuS, sGu, bGu) || make_map(&maps.dn[l][0], dr, 3, dDn, sDn, bDn) ||
        make_map(&maps.dn[l][1], dsh, 3, dDnS, sDn, bDn))
      return VG_ERR_CUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  {
    const uint64_t dA[2] = {kI, (uint64_t)kSsSlots * kSsN}, sA[1] = {kI * 2};
    const uint32_t bA[2] = {kBK, kSsN};
    const uint64_t dL[2] = {kH, (uint64_t)V}, sL[1] = {kH * 2};
    const uint32_t bL[2] = {kBK, (uint32_t)box_rows(V, kBM)};
    if (make_map(&maps.act, ws + W.act, 2, dA, sA, bA) || make_map(&maps.lm, lm_head, 2, dL, sL, bL))
      return VG_ERR_CUDA;
  }
  if (V < kBM) return VG_ERR_UNSUPPORTED;  // the LM-head units read 128-row boxes
  SsArgs a{};
  a.T = B * (K + 1);
  a.B = B;
  a.K = K;
  a.L = n_layers;
  a.V = V;
  a.x = static_cast<const __nv_bfloat16*>(x);
  for (int l = 0; l < n_layers; ++l) {
    a.router_w[l] = static_cast<const __nv_bfloat16*>(router_w[l]);
    a.router_b[l] = router_bias ? router_bias[l] : nullptr;
  }
  a.drafts = drafts;
  a.argmax = argmax;
  a.accepted = accepted;
  a.out_tokens = out_tokens;
  a.states = static_cast<__nv_bfloat16*>(states_out);
  a.topk_idx = topk_idx_out;
  a.part_gu = reinterpret_cast<float*>(ws + W.part_gu);
  a.part_dn = reinterpret_cast<float*>(ws + W.part_dn);
  a.act = reinterpret_cast<__nv_bfloat16*>(ws + W.act);
  a.o = reinterpret_cast<__nv_bfloat16*>(ws + W.o);
  a.ctrl = reinterpret_cast<SsCtrl*>(ws + W.ctrl);
  if (cudaMemsetAsync(ws + W.ctrl, 0, sizeof(SsCtrl), s) != cudaSuccess) return cuda_fail();
  ProfScope ps(VG_KERNEL_EXPERTS, s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(dev->sms);
  cfg.blockDim = dim3(kSsThreads);
  cfg.dynamicSmemBytes = kSsSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, verify_step_small<kTopK>, maps, a) != cudaSuccess) return cuda_fail();
  return VG_OK;
}
