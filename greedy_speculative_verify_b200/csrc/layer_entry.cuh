// Entry of an MoE layer at decode sizes (T * k <= 8192): everything between
// two expert-GEMM launches in one cooperative kernel —
//   [combine of the previous layer ->] router logits + top-k + softmax ->
//   stable grouping by expert + row gather
// — with a grid barrier after the combine and after the routing. A CTA routes
// groups of 2 tokens (c, c + G, ...) with the whole router matrix in shared
// memory, requested by bulk copies at entry so that its latency hides behind
// the combine phase (TMA tiles with the 128-byte swizzle); each logit is four
// quarter fma chains (one thread each) combined as (q0 + q1) + (q2 + q3). The arithmetic of every phase is the one
// of the separate kernels (router.cuh, sort.cuh, combine.cuh).
#pragma once
#include "combine.cuh"
#include "common.cuh"
#include "router.cuh"
#include "sort.cuh"

namespace vg {

struct EntryArgs {
  // combine of the previous layer; prev_o == nullptr when the layer input is x_in
  const __nv_bfloat16* prev_o;
  const int32_t* prev_inv;
  const float* prev_gate;
  const __nv_bfloat16* prev_x;
  int32_t prev_add_residual;
  const __nv_bfloat16* x_in;  // layer input (no combine phase)
  __nv_bfloat16* x_out;       // layer input written by the combine phase
  const __nv_bfloat16* w;     // router [64, H]
  const float* bias;          // [64] or nullptr
  int32_t T, H, k, S;
  float* logits;              // [T, 64]
  int32_t* idx;               // [T, k]
  float* gate;                // [T, k]
  int32_t* offsets;           // [65]
  int32_t* perm;              // [T k]
  int32_t* inv;               // [T k]
  __nv_bfloat16* x_perm;      // [T k, H]
  int32_t* sched;             // expert kernel's counters, cleared here
  int32_t sched_len;
  uint32_t* gbar;             // grid barrier counter, zeroed before the first launch on it
  uint32_t gbar_base;         // barriers already passed on gbar before this launch
};

constexpr int kEntryTok = 2;                            // tokens routed per group
constexpr int kEntryThreads = kEntryTok * kRouterE * 4;  // one thread per quarter chain: 512

// Shared memory: the whole router matrix as H/64 TMA tiles of [64 rows x 64 k]
// with the 128-byte swizzle (8 KB each), the group's token rows as bf16 (bulk
// copy target) and as fp32; the grouping phase reuses the same bytes for its
// two [N] arrays once the logits are done.
__host__ __device__ constexpr int layer_entry_route_bytes(int H) {
  return kRouterE * H * 2 + kEntryTok * H * 2 + kEntryTok * H * 4;
}
__host__ __device__ constexpr int layer_entry_smem(int H, int N) {
  return 1024 + (layer_entry_route_bytes(H) > 2 * N * 4 ? layer_entry_route_bytes(H) : 2 * N * 4);
}

template <int K>
__global__ void __launch_bounds__(kEntryThreads, 1) moe_layer_entry(const __grid_constant__ CUtensorMap mR,
                                                                    const EntryArgs a) {
  extern __shared__ uint8_t esm_raw[];
  uint8_t* esm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(esm_raw) + 1023) & ~uintptr_t(1023));
  const int H = a.H, HQ = H / 4;
  uint8_t* ws = esm;                                                       // [H/64][64 rows][128 B]
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(esm + kRouterE * H * 2);  // [tok][H]
  float* xf = reinterpret_cast<float*>(xs + kEntryTok * H);                      // [tok][H]
  const int N = a.T * a.k;
  int32_t* perm_s = reinterpret_cast<int32_t*>(esm);           // [N], after the logits
  int32_t* keys_s = perm_s + N;                                // [N]
  __shared__ __align__(8) uint64_t bars[2];                    // weights, token rows
  __shared__ float part[4][kEntryTok][kRouterE];               // [quarter][token][expert]
  __shared__ float logit[kEntryTok][kRouterE];
  __shared__ int cnt[kSortE], run[kSortE];
  __shared__ int wcnt[32][kSortE];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const uint64_t limit = g_wait_timeout_ns;
  const __nv_bfloat16* xcur = a.prev_o != nullptr ? a.x_out : a.x_in;
  const int n_groups = cdiv(a.T, kEntryTok);

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    if (c < n_groups) {  // the router matrix is streamed in while the combine phase runs
      mbar_arrive_expect_tx(&bars[0], kRouterE * H * 2);
      const int nkc = H / 64;
      for (int i = 0; i < nkc; ++i) {  // CTAs start at different tiles: spread over L2 slices
        const int kc = (i + c) % nkc;
        tma_load_2d(ws + kc * 8192, &mR, &bars[0], kc * 64, 0);
      }
    }
  }
  bool ok = true;

  // ---- phase 1: the previous layer's weighted combine -> this layer's input
  uint32_t nbar = a.gbar_base;
  if (a.prev_o != nullptr) {
    const int per_row = H / 8;
    const int total = a.T * per_row, per_cta = cdiv(total, G);  // an even, contiguous share per CTA
    for (int i = c * per_cta + tid; i < min(total, (c + 1) * per_cta); i += blockDim.x) {
      const int t = i / per_row, cc = i - t * per_row;
      reinterpret_cast<uint4*>(a.x_out + (size_t)t * H)[cc] =
          combine8(a.prev_x, a.prev_o, a.prev_inv, a.prev_gate, a.T, H, a.k, a.S, a.prev_add_residual, t, cc);
    }
    if (G > 1) ok = grid_barrier(a.gbar, (++nbar) * G, limit, 151);
    else __syncthreads();
  }

  // ---- phase 2: router logits and top-k of kEntryTok tokens per group. A warp
  // runs one quarter chain of one token for 32 experts: lane-consecutive experts
  // read distinct 16-byte swizzle slots of the same k, so reads are
  // conflict-free, and the fp32 token row is a broadcast.
  const int qq = warp / (2 * kEntryTok), tl = (warp >> 1) % kEntryTok, e = ((warp & 1) << 5) | lane;
  int it = 0;
  for (int g = c; ok && g < n_groups; g += G, ++it) {
    const int t0 = g * kEntryTok;
    __syncthreads();  // the previous group's rows and logits are no longer read
    if (tid == 0) {
      fence_proxy_async_global();  // rows written by generic stores, read by bulk copies
      mbar_arrive_expect_tx(&bars[1], kEntryTok * H * 2);
      for (int r = 0; r < kEntryTok; ++r)
        bulk_load(xs + r * H, xcur + (size_t)min(t0 + r, a.T - 1) * H, H * 2, &bars[1]);
    }
    if (!mbar_wait(&bars[1], it & 1, limit)) {
      record_error(kErrTimeout, 152);
      ok = false;
      break;
    }
    for (int i = tid; i < kEntryTok * H / 2; i += blockDim.x) {  // token rows to fp32, once
      const uint32_t v = reinterpret_cast<const uint32_t*>(xs)[i];
      reinterpret_cast<float2*>(xf)[i] = make_float2(bf16_lo(v), bf16_hi(v));
    }
    __syncthreads();
    if (!mbar_wait(&bars[0], 0, limit)) {
      record_error(kErrTimeout, 155);
      ok = false;
      break;
    }
    const float4* xr = reinterpret_cast<const float4*>(xf + tl * H + qq * HQ);
    const uint8_t* wrow = ws + e * 128;
    float acc = 0.0f;
#pragma unroll 8
    for (int p = 0; p < HQ / 8; ++p) {
      const int k = qq * HQ + p * 8;  // 8 consecutive k in one 16-byte slot
      const int kc = k >> 6, j = (k >> 3) & 7;
      const uint4 wv = *reinterpret_cast<const uint4*>(wrow + kc * 8192 + ((j ^ (e & 7)) << 4));
      const float4 x0 = xr[2 * p], x1 = xr[2 * p + 1];
      acc = __fmaf_rn(x0.x, bf16_lo(wv.x), acc);
      acc = __fmaf_rn(x0.y, bf16_hi(wv.x), acc);
      acc = __fmaf_rn(x0.z, bf16_lo(wv.y), acc);
      acc = __fmaf_rn(x0.w, bf16_hi(wv.y), acc);
      acc = __fmaf_rn(x1.x, bf16_lo(wv.z), acc);
      acc = __fmaf_rn(x1.y, bf16_hi(wv.z), acc);
      acc = __fmaf_rn(x1.z, bf16_lo(wv.w), acc);
      acc = __fmaf_rn(x1.w, bf16_hi(wv.w), acc);
    }
    part[qq][tl][e] = acc;
    __syncthreads();
    if (tid < kEntryTok * kRouterE) {
      const int t2 = tid >> 6, e2 = tid & 63;
      float l = (part[0][t2][e2] + part[1][t2][e2]) + (part[2][t2][e2] + part[3][t2][e2]);
      if (a.bias != nullptr) l = __fadd_rn(l, a.bias[e2]);
      logit[t2][e2] = l;
    }
    __syncthreads();
    if (warp < kEntryTok && t0 + warp < a.T) {
      const int t = t0 + warp;
      topk_softmax_warp<K>(logit[warp], lane, a.idx + (size_t)t * K, a.gate + (size_t)t * K);
    }
  }
  if (G > 1) ok = grid_barrier(a.gbar, (++nbar) * G, limit, 153) && ok;
  else __syncthreads();
  if (!ok) return;

  // ---- phase 3: stable grouping (every CTA sorts; CTA 0 publishes) + gather
  if (tid < kSortE) cnt[tid] = 0;
  if (c == 0)
    for (int i = tid; i < a.sched_len; i += blockDim.x) a.sched[i] = 0;
  for (int i = tid; i < N; i += blockDim.x) keys_s[i] = __ldcg(a.idx + i);
  __syncthreads();
  for (int i = tid; i < N; i += blockDim.x) atomicAdd(&cnt[keys_s[i]], 1);
  __syncthreads();
  if (warp == 0) {
    scan64_warp(cnt, run, lane);
    if (c == 0) {
      a.offsets[2 * lane] = run[2 * lane];
      a.offsets[2 * lane + 1] = run[2 * lane + 1];
      if (lane == 0) a.offsets[kSortE] = N;
    }
  }
  __syncthreads();
  for (int base = 0; base < N; base += blockDim.x) {
    const int pos = chunk_positions(keys_s, base, N, run, wcnt);
    if (pos >= 0) {
      perm_s[pos] = base + tid;
      if (c == 0) {
        a.perm[pos] = base + tid;
        a.inv[base + tid] = pos;
      }
    }
  }
  __syncthreads();
  for (int row = c * (blockDim.x / 32) + warp; row < N; row += G * (blockDim.x / 32)) {
    const uint4* src = reinterpret_cast<const uint4*>(xcur + (size_t)(perm_s[row] / a.k) * H);
    uint4* dst = reinterpret_cast<uint4*>(a.x_perm + (size_t)row * H);
    for (int cc = lane; cc < H / 8; cc += 32) dst[cc] = __ldcg(src + cc);
  }
}

}  // namespace vg
