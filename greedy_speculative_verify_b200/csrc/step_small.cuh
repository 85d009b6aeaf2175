// The whole verify step for a handful of rows (T = B (K+1) <= 16, the batch-1
// case: K = 3 gives 4 rows, K = 1 gives 2) in one persistent launch: the
// layers' MoE feed-forward blocks, the LM-head argmax and the prefix accept.
//
// At these sizes a step is a stream of weights (about 150 MB per layer for the
// ~22 experts 4 tokens touch, plus the 331 MB LM head), and launch gaps and
// dependent waits between kernels cost as much as the stream itself. Here one
// CTA per SM (cooperative launch) runs every phase:
//
//  R. routing, computed by every CTA for all T rows (identical results
//     everywhere, so no barrier): the previous layer's weighted combine (the
//     order of combine.cuh) into the token tile in shared memory, the router
//     logits (four quarter fma chains, the order of router.cuh), top-6 and
//     softmax (topk_softmax_warp), and the layer's expert slots: the touched
//     routed experts in increasing order, then the two shared experts. The
//     token tile is the B operand of every gate/up product and of the LM head:
//     16 rows (rows >= T are zero) x 1280, stored as 20 K-major 64-column
//     chunks with the 128-byte swizzle, as a TMA load would lay them out.
//  E. expert units from a per-layer ticket counter: a gate/up unit is (slot,
//     128-row block, one of kSsKsGu pieces of the 20 k-chunks), a down unit
//     (slot, 256-row block, one of kSsKsDn pieces of the 14 k-chunks); the
//     split spreads the ~150 MB of a layer over all SMs (measured best: gate/up
//     in halves, down whole; finer pieces lose more to per-unit work than they
//     gain in balance). The tensor cores compute 128 weight rows x 16 token
//     columns per unit. A whole unit applies SwiGLU (gate/up: activations,
//     bf16) or rounds (down: expert outputs, bf16) straight from its
//     accumulator; a split unit stores its fp32 partial sums, and the last of
//     the block's k-pieces to arrive (a counter per 32-row quarter) adds the
//     pieces in k order (so the result does not depend on timing) first. Down units stream their weights first and wait (bounded)
//     until all gate/up blocks of their slot are reduced; a counter of reduced
//     down blocks ends the layer for every CTA.
//  V. after the last layer's combine, LM-head units of 128 vocabulary rows;
//     each folds its best (value, index) key per row into a 64-bit atomic max
//     (the key of lmhead.cuh), and the last CTA to finish writes the argmax,
//     accepts each sequence's longest agreeing prefix plus the bonus token, and
//     clears the keys.
//
// Warp roles in phases E and V: warp 0 issues TMA loads of the weights (and of
// the activations for down units) into a 4-stage ring, warp 1 issues
// tcgen05.mma, warps 2-5 drain the double-buffered accumulators. All eight
// warps compute phase R. Every wait is bounded; a timeout records
// VG_ERR_TIMEOUT and makes the CTA finish its current phase without new work.
#pragma once
#include "common.cuh"
#include "gemm_moe.cuh"
#include "lmhead.cuh"
#include "router.cuh"

namespace vg {

#ifndef VG_SS_ROUTER_UNROLL
#define VG_SS_ROUTER_UNROLL 10
#endif
constexpr int kSsRouterUnroll = VG_SS_ROUTER_UNROLL;  // router weight loads in flight per thread
constexpr int kSsMaxLayers = 12;
constexpr int kSsN = 16;              // token columns of every product (MMA N)
constexpr int kSsThreads = 256;
constexpr int kSsStages = 4;
constexpr int kSsWBytes = 2 * kBM * kBK * 2;                  // 32 KB of weights per stage
constexpr int kSsActBytes = kSsN * kBK * 2;                   // 2 KB activation tile (down units)
constexpr int kSsStageBytes = kSsWBytes + kSsActBytes;
constexpr int kSsTokBytes = (1280 / kBK) * kSsN * kBK * 2;    // 40 KB token tile
constexpr int kSsSlots = 66;                                  // 64 routed + 2 shared experts at most
#ifndef VG_SS_KS_GU
#define VG_SS_KS_GU 2
#endif
#ifndef VG_SS_KS_DN
#define VG_SS_KS_DN 1
#endif
constexpr int kSsKsGu = VG_SS_KS_GU;                          // k-pieces of a gate/up block (20 chunks split evenly)
constexpr int kSsKsDn = VG_SS_KS_DN;                          // k-pieces of a down block (14 chunks split evenly)
static_assert(20 % kSsKsGu == 0 && 14 % kSsKsDn == 0, "k-pieces must split the chunks evenly");
constexpr int kSsMbGu = 7, kSsMbDn = 5;                       // 128-row gate/up, 256-row down blocks
constexpr int kSsTmemCols = 64;                               // 2 buffers x (D0 16 | D1 16)
constexpr int kSsSmemBytes = kSsStages * kSsStageBytes + kSsTokBytes + 1024;  // + alignment slack

// Partial sums of one unit: [2 accumulators][16 columns][128 rows] fp32.
constexpr int kSsPartFloats = 2 * kSsN * kBM;

// Control words (zeroed before the launch).
struct SsCtrl {
  uint32_t ticket[kSsMaxLayers + 1];
  uint32_t ready_gu[kSsMaxLayers][kSsSlots];               // reduced (block, quarter) pairs: 28 when done
  uint32_t cnt_gu[kSsMaxLayers][kSsSlots][kSsMbGu][4];     // k-pieces arrived per (block, quarter)
  uint32_t cnt_dn[kSsMaxLayers][kSsSlots][kSsMbDn][4];
  uint32_t done_dn[kSsMaxLayers];                          // reduced down (block, quarter) pairs
  uint32_t lm_done;                                        // CTAs past the LM head
  uint32_t pad;
  unsigned long long best[kSsN];                           // running argmax key per row
};

struct SsMaps {
  CUtensorMap gu[kSsMaxLayers][2];  // gate/up views (k, row, gate|up, expert): routed, shared
  CUtensorMap dn[kSsMaxLayers][2];  // down views (k, row, expert): routed, shared
  CUtensorMap act;                  // activation slots [kSsSlots * 16, I], 16-row boxes
  CUtensorMap lm;                   // LM head [V, H], 128-row boxes
};

struct SsArgs {
  int T, B, K, L, V;
  const __nv_bfloat16* x;                        // [T, H] input of layer 0
  const __nv_bfloat16* router_w[kSsMaxLayers];   // [64, H]
  const float* router_b[kSsMaxLayers];           // [64] or null
  const int32_t* drafts;                         // [B, K] (null when K == 0)
  int32_t* argmax;                               // [T]
  int32_t* accepted;                             // [B]
  int32_t* out_tokens;                           // [B, K+1]
  __nv_bfloat16* states;                         // [L+1, T, H] or null: each layer's input, then the final states
  int32_t* topk_idx;                             // [L, T, 6] or null
  float* part_gu;                                // [slots][7][4][kSsPartFloats]
  float* part_dn;                                // [slots][5][2][kSsPartFloats]
  __nv_bfloat16* act;                            // [slots][16][I]
  __nv_bfloat16* o;                              // [slots][16][H]
  SsCtrl* ctrl;
};

// Byte offset of 16-byte column chunk c8 (columns 8 c8 .. 8 c8 + 7) of row t in
// the token tile: K-major 64-column chunks of 16 rows x 128 bytes, 128-byte swizzle.
__device__ __forceinline__ uint32_t ss_tok_off(int t, int c8) {
  const int kc = c8 >> 3, cc = c8 & 7;
  return (uint32_t)(kc * (kSsN * 128) + t * 128 + ((cc ^ (t & 7)) << 4));
}

__device__ __forceinline__ float ss_f(uint32_t v, int hi) { return hi ? bf16_hi(v) : bf16_lo(v); }

__device__ __forceinline__ bool ss_wait_geq(const uint32_t* p, uint32_t target, uint64_t limit) {
  const uint64_t t0 = globaltimer();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if (v >= target) return true;
    if (globaltimer() - t0 > limit) return false;
    __nanosleep(100);
  }
}

template <int K6>
__global__ void __launch_bounds__(kSsThreads, 1)
    verify_step_small(const __grid_constant__ SsMaps maps, const SsArgs a) {
  constexpr int H = 1280, I = 896, E = 64, HQ = H / 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;                                    // [stages][32 KB weights | 2 KB activations]
  uint8_t* tok = smem + kSsStages * kSsStageBytes;          // token tile, 1024-aligned
  __shared__ __align__(8) uint64_t full[kSsStages], empty[kSsStages], tfull[2], tempty[2];
  __shared__ __align__(8) uint64_t ufull[kFgRing], uempty[kFgRing], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_s;
  __shared__ volatile int ring[kFgRing];
  __shared__ float part_s[4][kSsN][E];     // router quarter sums [quarter][row][expert]
  __shared__ float logit_s[kSsN][E];
  __shared__ int32_t idx_s[kSsN][K6];      // this layer's experts per row
  __shared__ float g_s[kSsN][K6];          // this layer's gates
  __shared__ int32_t sl_s[kSsN][K6];       // slot of each (row, j)
  __shared__ int32_t slot_exp[kSsSlots];   // expert of each slot
  __shared__ int32_t exp_slot[E];          // slot of each routed expert (-1: untouched)
  __shared__ int n_slots_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t limit = g_wait_timeout_ns;
  const int T = a.T;
  griddep_launch_dependents();

  if (tid == 0) {
    for (int i = 0; i < kSsStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kFgEpiWarps);
    }
    for (int i = 0; i < kFgRing; ++i) {
      mbar_init(&ufull[i], 1);
      mbar_init(&uempty[i], 1 + kFgEpiWarps);
    }
    mbar_init(&mma_done, 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int l = 0; l < a.L; ++l) {
      prefetch_tmap(&maps.gu[l][0]);
      prefetch_tmap(&maps.gu[l][1]);
      prefetch_tmap(&maps.dn[l][0]);
      prefetch_tmap(&maps.dn[l][1]);
    }
    prefetch_tmap(&maps.act);
    prefetch_tmap(&maps.lm);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kSsTmemCols);
    tmem_relinquish();
  }
  // every layer's router matrix to L2 (immutable), kept there past the weight
  // stream (which is marked evict-first); 16 KB slices spread over the CTAs
  const uint64_t pol_keep = policy_evict_last();
  if (tid == 0) {
    constexpr int kSlices = E * H * 2 / 16384;
    for (int i = blockIdx.x; i < a.L * kSlices; i += gridDim.x) {
      const int l = i / kSlices, sl = i - l * kSlices;
      bulk_prefetch_l2_hint(a.router_w[l] + (size_t)sl * 8192, 16384, pol_keep);
    }
  }
  for (int i = tid; i < kSsTokBytes / 16; i += kSsThreads) reinterpret_cast<uint4*>(tok)[i] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  griddep_wait();  // x and the drafts may come from the previous kernel

  // role state, carried across phases (the mbarrier phases continue)
  int p_stage = 0, p_slot = 0;
  uint32_t p_phase = 0, p_rphase = 0, p_issued = 0, p_last_par = 0;
  int m_stage = 0, m_slot = 0, m_lu = 0;
  uint32_t m_phase = 0, m_rphase = 0;
  int e_slot = 0, e_lu = 0;
  uint32_t e_rphase = 0;

  // Combine of layer l-1 into the token tile (l >= 1), in the order of
  // combine.cuh: shared outputs, then the routed outputs weighted in slot
  // order j, then the residual; one bf16 rounding. Also writes the states.
  auto combine_into_tile = [&](int l) {
    for (int i = tid; i < T * (H / 8); i += kSsThreads) {
      const int t = i / (H / 8), c8 = i - t * (H / 8);
      uint4* tp = reinterpret_cast<uint4*>(tok + ss_tok_off(t, c8));
      float y[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) y[k] = 0.0f;
      if (l > 0) {
        for (int s = 0; s < 2; ++s) {
          const int slot = n_slots_s - 2 + s;
          const uint4 v = __ldcg(reinterpret_cast<const uint4*>(a.o + ((size_t)slot * kSsN + t) * H) + c8);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) y[k] += ss_f(w[k >> 1], k & 1);
        }
        for (int j = 0; j < K6; ++j) {
          const float gj = g_s[t][j];
          if (!VG_IN_BOUNDS((unsigned)sl_s[t][j] < (unsigned)kSsSlots, 411)) continue;
          const uint4 v = __ldcg(reinterpret_cast<const uint4*>(a.o + ((size_t)sl_s[t][j] * kSsN + t) * H) + c8);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) y[k] = __fmaf_rn(gj, ss_f(w[k >> 1], k & 1), y[k]);
        }
        const uint4 xv = *tp;
        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] += ss_f(w[k >> 1], k & 1);
        uint4 r;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]), h3 = __floats2bfloat162_rn(y[6], y[7]);
        r.x = *reinterpret_cast<uint32_t*>(&h0);
        r.y = *reinterpret_cast<uint32_t*>(&h1);
        r.z = *reinterpret_cast<uint32_t*>(&h2);
        r.w = *reinterpret_cast<uint32_t*>(&h3);
        *tp = r;
      } else {
        *tp = reinterpret_cast<const uint4*>(a.x + (size_t)t * H)[c8];
      }
      if (a.states != nullptr && blockIdx.x == 0)
        reinterpret_cast<uint4*>(a.states + ((size_t)l * T + t) * H)[c8] = *tp;
    }
  };

  // Phases 0 .. L-1: layer l (routing, then its expert units); phase L: the
  // last layer's combine, then the LM-head units.
  for (int l = 0; l <= a.L && !abort_s; ++l) {
    const int kind = l == a.L ? 1 : 0;
    // ---------------------------------------------------------------- R
    combine_into_tile(l);
    fence_proxy_async_shared();  // the tensor cores read the tile
    __syncthreads();
    if (kind == 0) {
      {
        // router logits: thread (quarter q, expert e), rows in groups of four chains;
        // CTAs start at different router rows, so that they do not all request
        // the same L2 lines at the same moment
        const int q = ((tid >> 6) + (blockIdx.x >> 6)) & 3, e = ((tid & 63) + blockIdx.x) & 63;
        const uint4* wsrc = reinterpret_cast<const uint4*>(a.router_w[l] + (size_t)e * H + q * HQ);
        for (int t0 = 0; t0 < T; t0 += 4) {
          float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll(kSsRouterUnroll)
          for (int i = 0; i < HQ / 8; ++i) {
            const uint4 wq = ldg_hint(wsrc + i, pol_keep);  // an L2 hit: the router matrices were prefetched
            const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
            const int c8 = q * (HQ / 8) + i;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const uint4 xv = *reinterpret_cast<const uint4*>(tok + ss_tok_off(t0 + r, c8));
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int k = 0; k < 8; ++k)
                acc[r] = __fmaf_rn(ss_f(xw[k >> 1], k & 1), ss_f(wv[k >> 1], k & 1), acc[r]);
            }
          }
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (t0 + r < T) part_s[q][t0 + r][e] = acc[r];
        }
      }
      __syncthreads();
      for (int i = tid; i < T * E; i += kSsThreads) {
        const int t = i >> 6, e = i & 63;
        float v = (part_s[0][t][e] + part_s[1][t][e]) + (part_s[2][t][e] + part_s[3][t][e]);
        if (a.router_b[l] != nullptr) v = __fadd_rn(v, a.router_b[l][e]);
        logit_s[t][e] = v;
      }
      if (tid < E) exp_slot[tid] = -1;
      __syncthreads();
      for (int t = warp; t < T; t += kSsThreads / 32) topk_softmax_warp<K6>(logit_s[t], lane, idx_s[t], g_s[t]);
      __syncthreads();
      if (tid < T * K6) {
        const int t = tid / K6, j = tid - t * K6;
        int e = idx_s[t][j];
        if ((unsigned)e >= (unsigned)E) {  // only non-finite logits get here
          record_error(kErrBounds, 178);
          idx_s[t][j] = e = 0;
        }
        exp_slot[e] = 1;
        if (a.topk_idx != nullptr && blockIdx.x == 0) a.topk_idx[((size_t)l * T + t) * K6 + j] = e;
      }
      __syncthreads();
      if (warp == 0) {  // slots: touched routed experts in increasing order, then the two shared experts
        int base = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
          const int e = e0 + lane;
          const bool used = exp_slot[e] >= 0;
          const uint32_t m = __ballot_sync(0xffffffffu, used);
          const int pos = base + __popc(m & ((1u << lane) - 1u));
          __syncwarp();
          if (used) {
            exp_slot[e] = pos;
            slot_exp[pos] = e;
          }
          base += __popc(m);
        }
        if (lane < 2) slot_exp[base + lane] = E + lane;
        if (lane == 0) n_slots_s = base + 2;
      }
      __syncthreads();
      if (tid < T * K6) {
        const int t = tid / K6, j = tid - t * K6;
        sl_s[t][j] = exp_slot[idx_s[t][j]];
      }
      __syncthreads();
    }

    // ---------------------------------------------------------------- E / V
    uint32_t* tk = &a.ctrl->ticket[l];
    const int n_units = kind == 1 ? cdiv(a.V, kBM) : n_slots_s * (kSsMbGu * kSsKsGu + kSsMbDn * kSsKsDn);
    const int n_gu = n_slots_s * kSsMbGu * kSsKsGu;
    if (warp == 0) {
      if (lane == 0) {
        const uint64_t pol_w = policy_evict_first();
        // the next ticket is requested one unit ahead so its round trip overlaps the loads
        int next_u = (int)atomicAdd(tk, 1u);
        while (true) {
          int u = abort_s ? -1 : next_u;
          if (u >= n_units) u = -1;
          if (u >= 0) next_u = (int)atomicAdd(tk, 1u);
          if (!mbar_wait(&uempty[p_slot], p_rphase ^ 1, limit)) {
            record_error(kErrTimeout, 170);
            abort_s = 1;
            u = -1;
          }
          ring[p_slot] = u;
          mbar_arrive(&ufull[p_slot]);
          if (++p_slot == kFgRing) {
            p_slot = 0;
            p_rphase ^= 1;
          }
          if (u < 0) break;
          // what to load: kc0 .. kc0 + nk - 1 of a weight view, (down) activation rows
          const CUtensorMap* mw;
          int nk, kc0, wrow = 0, ecoord = 0, act_row = -1, slot = 0;
          bool four_d = false;
          uint32_t wbytes = kSsWBytes;
          if (kind == 1) {
            mw = &maps.lm;
            nk = H / kBK;
            kc0 = 0;
            wrow = u * kBM;
            wbytes = kBM * kBK * 2;
          } else if (u < n_gu) {
            slot = u / (kSsMbGu * kSsKsGu);
            const int rem = u - slot * (kSsMbGu * kSsKsGu);
            const int mb = rem / kSsKsGu, ks = rem - mb * kSsKsGu;
            const int e = slot_exp[slot];
            mw = e < E ? &maps.gu[l][0] : &maps.gu[l][1];
            ecoord = e < E ? e : e - E;
            nk = (H / kBK) / kSsKsGu;
            kc0 = ks * nk;
            wrow = mb * kBM;
            four_d = true;
          } else {
            const int v = u - n_gu;
            slot = v / (kSsMbDn * kSsKsDn);
            const int rem = v - slot * (kSsMbDn * kSsKsDn);
            const int mb = rem / kSsKsDn, ks = rem - mb * kSsKsDn;
            const int e = slot_exp[slot];
            mw = e < E ? &maps.dn[l][0] : &maps.dn[l][1];
            ecoord = e < E ? e : e - E;
            nk = (I / kBK) / kSsKsDn;
            kc0 = ks * nk;
            wrow = mb * 2 * kBM;
            act_row = slot * kSsN;
          }
          const int npre = act_row >= 0 ? min(kSsStages, nk) : 0;  // weights before the activations
          const int st0 = p_stage;
          bool ok = true;
          for (int j = 0; j < nk && ok; ++j) {
            if (!mbar_wait(&empty[p_stage], p_phase ^ 1, limit)) {
              record_error(kErrTimeout, 171);
              abort_s = 1;
              ok = false;
              break;
            }
            uint8_t* st = tiles + p_stage * kSsStageBytes;
            mbar_arrive_expect_tx(&full[p_stage], wbytes + (act_row >= 0 ? kSsActBytes : 0));
            const int kc = kc0 + j;
            if (four_d)
              tma_load_4d_hint(st, mw, &full[p_stage], kc * kBK, wrow, 0, ecoord, pol_w);
            else if (kind == 1)
              tma_load_2d_hint(st, mw, &full[p_stage], kc * kBK, wrow, pol_w);
            else
              tma_load_3d_hint(st, mw, &full[p_stage], kc * kBK, wrow, ecoord, pol_w);
            if (act_row >= 0 && j >= npre) tma_load_2d(st + kSsWBytes, &maps.act, &full[p_stage], kc * kBK, act_row);
            if (act_row >= 0 && j + 1 == npre) {
              // the slot's activations are complete when all its gate/up blocks are reduced
              if (!ss_wait_geq(&a.ctrl->ready_gu[l][slot], kSsMbGu * 4, limit)) {
                record_error(kErrTimeout, 172);
                abort_s = 1;  // load anyway so every armed stage completes
              }
              fence_proxy_async_global();
              for (int jj = 0; jj < npre; ++jj) {
                const int sj = (st0 + jj) % kSsStages;
                tma_load_2d(tiles + sj * kSsStageBytes + kSsWBytes, &maps.act, &full[sj], (kc0 + jj) * kBK, act_row);
              }
            }
            p_issued |= 1u << p_stage;
            p_last_par = (p_last_par & ~(1u << p_stage)) | (p_phase << p_stage);
            if (++p_stage == kSsStages) {
              p_stage = 0;
              p_phase ^= 1;
            }
          }
          if (!ok) {
            // push the end marker so the other roles leave this phase
            if (mbar_wait(&uempty[p_slot], p_rphase ^ 1, limit)) {
              ring[p_slot] = -1;
              mbar_arrive(&ufull[p_slot]);
              if (++p_slot == kFgRing) {
                p_slot = 0;
                p_rphase ^= 1;
              }
            }
            break;
          }
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        const uint32_t idesc = idesc_bf16_f32(kBM, kSsN);
        while (true) {
          if (!mbar_wait(&ufull[m_slot], m_rphase, limit)) {
            record_error(kErrTimeout, 173);
            abort_s = 1;
            break;
          }
          const int u = ring[m_slot];
          mbar_arrive(&uempty[m_slot]);
          if (++m_slot == kFgRing) {
            m_slot = 0;
            m_rphase ^= 1;
          }
          if (u < 0) break;
          const bool down = kind == 0 && u >= n_gu;
          int nk, kc0;
          if (kind == 1) {
            nk = H / kBK;
            kc0 = 0;
          } else if (!down) {
            nk = (H / kBK) / kSsKsGu;
            kc0 = (u % kSsKsGu) * nk;
          } else {
            nk = (I / kBK) / kSsKsDn;
            kc0 = ((u - n_gu) % kSsKsDn) * nk;
          }
          const int ab = m_lu & 1;
          const uint32_t ap = (m_lu >> 1) & 1;
          ++m_lu;
          if (!mbar_wait(&tempty[ab], ap ^ 1, limit)) {
            record_error(kErrTimeout, 174);
            abort_s = 1;
            break;
          }
          tc_fence_after();
          const uint32_t d0 = tmem_base + ab * 32, d1 = d0 + 16;
          bool ok = true;
          for (int j = 0; j < nk; ++j) {
            if (!mbar_wait(&full[m_stage], m_phase, limit)) {
              record_error(kErrTimeout, 175);
              abort_s = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(tiles + m_stage * kSsStageBytes);
            const uint64_t da0 = sw128_kmajor_desc(st), da1 = sw128_kmajor_desc(st + kBM * kBK * 2);
            const uint64_t db = down ? sw128_kmajor_desc(st + kSsWBytes)
                                     : sw128_kmajor_desc(smem_u32(tok + (kc0 + j) * (kSsN * 128)));
#pragma unroll
            for (int k16 = 0; k16 < kBK / 16; ++k16) {
              const uint32_t acc = (j | k16) != 0;
              umma_bf16(d0, da0 + 2 * k16, db + 2 * k16, idesc, acc);
              if (kind == 0) umma_bf16(d1, da1 + 2 * k16, db + 2 * k16, idesc, acc);
            }
            umma_commit(&empty[m_stage]);
            if (++m_stage == kSsStages) {
              m_stage = 0;
              m_phase ^= 1;
            }
          }
          if (!ok) break;
          umma_commit(&tfull[ab]);
        }
      }
    } else if (warp >= 2 && warp < 6) {
      const int q = warp & 3;
      const int row = q * 32 + lane;
      while (true) {
        if (!mbar_wait(&ufull[e_slot], e_rphase, limit)) {
          record_error(kErrTimeout, 176);
          abort_s = 1;
          break;
        }
        const int u = ring[e_slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&uempty[e_slot]);
        if (++e_slot == kFgRing) {
          e_slot = 0;
          e_rphase ^= 1;
        }
        if (u < 0) break;
        const int ab = e_lu & 1;
        const uint32_t ap = (e_lu >> 1) & 1;
        ++e_lu;
        if (!mbar_wait(&tfull[ab], ap, limit)) {
          record_error(kErrTimeout, 177);
          abort_s = 1;
          break;
        }
        tc_fence_after();
        const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + ab * 32;
        uint32_t r0[16], r1[16];
        tmem_ld16(t0, r0);
        if (kind == 0) tmem_ld16(t0 + 16, r1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[ab]);  // the accumulator is in registers now
        if (kind == 1) {
          // LM head: vocabulary row v = 128 u + row against the 16 token columns
          const int v = u * kBM + row;
#pragma unroll
          for (int j = 0; j < kSsN; ++j) {
            uint64_t key = v < a.V ? argmax_key(__uint_as_float(r0[j]), (uint32_t)v) : 0ull;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const uint64_t other = __shfl_xor_sync(0xffffffffu, key, o);
              key = other > key ? other : key;
            }
            if (lane == j && j < T) atomicMax(&a.ctrl->best[j], (unsigned long long)key);
          }
          continue;
        }
        const bool down = u >= n_gu;
        int slot, mb, ks;
        float* part;
        uint32_t* cnt;
        int nks;
        if (!down) {
          slot = u / (kSsMbGu * kSsKsGu);
          const int rem = u - slot * (kSsMbGu * kSsKsGu);
          mb = rem / kSsKsGu;
          ks = rem - mb * kSsKsGu;
          nks = kSsKsGu;
          part = a.part_gu + (size_t)((slot * kSsMbGu + mb) * kSsKsGu) * kSsPartFloats;
          cnt = &a.ctrl->cnt_gu[l][slot][mb][q];
        } else {
          const int v = u - n_gu;
          slot = v / (kSsMbDn * kSsKsDn);
          const int rem = v - slot * (kSsMbDn * kSsKsDn);
          mb = rem / kSsKsDn;
          ks = rem - mb * kSsKsDn;
          nks = kSsKsDn;
          part = a.part_dn + (size_t)((slot * kSsMbDn + mb) * kSsKsDn) * kSsPartFloats;
          cnt = &a.ctrl->cnt_dn[l][slot][mb][q];
        }
        float s0[kSsN], s1[kSsN];
        if (nks == 1) {  // the unit covers the whole reduction
#pragma unroll
          for (int j = 0; j < kSsN; ++j) {
            s0[j] = __uint_as_float(r0[j]);
            s1[j] = __uint_as_float(r1[j]);
          }
        } else {
          // this k-piece's partial sums: [accumulator][column][row], coalesced over rows
          float* mine = part + (size_t)ks * kSsPartFloats;
#pragma unroll
          for (int j = 0; j < kSsN; ++j) {
            __stcg(mine + j * kBM + row, __uint_as_float(r0[j]));
            __stcg(mine + kSsN * kBM + j * kBM + row, __uint_as_float(r1[j]));
          }
          __syncwarp();
          uint32_t old = 0;
          if (lane == 0) old = atomic_add_acq_rel(cnt, 1u);  // releases the warp's partials
          old = __shfl_sync(0xffffffffu, old, 0);
          if (old != (uint32_t)(nks - 1)) continue;  // not the last k-piece of this (block, quarter)
#pragma unroll
          for (int j = 0; j < kSsN; ++j) s0[j] = s1[j] = 0.0f;
          for (int p = 0; p < nks; ++p) {  // in k order
            const float* pp = part + (size_t)p * kSsPartFloats;
#pragma unroll
            for (int j = 0; j < kSsN; ++j) {
              s0[j] += __ldcg(pp + j * kBM + row);
              s1[j] += __ldcg(pp + kSsN * kBM + j * kBM + row);
            }
          }
        }
        if (!down) {
          __nv_bfloat16* dst = a.act + (size_t)slot * kSsN * I + mb * kBM + row;
#pragma unroll
          for (int j = 0; j < kSsN; ++j) dst[(size_t)j * I] = __float2bfloat16_rn(silu(s0[j]) * s1[j]);
          fence_proxy_async_global();  // read back through TMA by the down units
          __syncwarp();
          if (lane == 0) atomic_add_acq_rel(&a.ctrl->ready_gu[l][slot], 1u);
        } else {
          __nv_bfloat16* dst = a.o + (size_t)slot * kSsN * H + mb * 2 * kBM + row;
#pragma unroll
          for (int j = 0; j < kSsN; ++j) {
            dst[(size_t)j * H] = __float2bfloat16_rn(s0[j]);
            dst[(size_t)j * H + kBM] = __float2bfloat16_rn(s1[j]);
          }
          __syncwarp();
          if (lane == 0) atomic_add_acq_rel(&a.ctrl->done_dn[l], 1u);
        }
      }
    }
    __syncthreads();
    if (kind == 0) {
      if (tid == 0 && !abort_s &&
          !ss_wait_geq(&a.ctrl->done_dn[l], (uint32_t)(n_slots_s * kSsMbDn * 4), limit)) {
        record_error(kErrTimeout, 179);
        abort_s = 1;
      }
      __syncthreads();
    }
  }

  // every issued copy has landed before the CTA goes on
  if (warp == 0 && lane == 0)
    for (int s = 0; s < kSsStages; ++s)
      if (p_issued & (1u << s)) mbar_wait(&full[s], (p_last_par >> s) & 1, limit);
  if (warp == 1 && lane == 0) {
    umma_commit(&mma_done);
    mbar_wait(&mma_done, 0, limit);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kSsTmemCols);
  }
  __shared__ int last_s;
  if (tid == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(&a.ctrl->lm_done, 1u);
    last_s = old == gridDim.x - 1;
  }
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  for (int t = tid; t < T; t += kSsThreads) {
    const unsigned long long k = atomicExch(&a.ctrl->best[t], 0ull);
    const int32_t v = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
    a.argmax[t] = VG_IN_BOUNDS(v >= 0 && v < a.V, 410) ? v : 0;
  }
  __syncthreads();
  for (int b = tid; b < a.B; b += kSsThreads) {
    const int32_t* arg = a.argmax + (size_t)b * (a.K + 1);
    const int32_t* d = a.drafts + (size_t)b * a.K;
    int acc = 0;
    while (acc < a.K && d[acc] == arg[acc]) ++acc;
    a.accepted[b] = acc;
    int32_t* o = a.out_tokens + (size_t)b * (a.K + 1);
    for (int i = 0; i <= a.K; ++i) o[i] = i < acc ? d[i] : (i == acc ? arg[acc] : -1);
  }
}

}  // namespace vg
