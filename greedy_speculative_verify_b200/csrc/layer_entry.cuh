// Entry of an MoE layer at decode sizes (T * k <= 8192): everything between
// two expert-GEMM launches in one cooperative kernel, with a single grid
// barrier.
//
// CTA c owns the contiguous tokens [c*P, (c+1)*P), P = ceil(T / grid):
//   A. for its tokens: [the previous layer's weighted combine ->] this layer's
//      input rows (kept in shared memory, also written out), router logits,
//      top-k + softmax; then its per-expert assignment counts go to global
//      memory;
//   -- grid barrier --
//   B. every CTA derives the expert offsets from all counts, and the position
//      of each of its own assignments: offset of the expert + assignments to
//      that expert in lower CTAs + rank among its own (assignment ids increase
//      with the token, so this is the stable order); it writes perm / inv and
//      copies its rows to their gathered positions straight from shared memory.
//
// The router matrix sits in shared memory as H/64 TMA tiles with the 128-byte
// swizzle, requested at entry so its latency hides behind the combine. Each
// logit is four quarter fma chains combined as (q0 + q1) + (q2 + q3), the
// order of the router's definition (router.cuh). Thread (group, quarter,
// expert) runs the chains of up to two tokens at once, so each weight pair is
// unpacked once for both; lane-consecutive experts read distinct swizzle slots.
// Top-k is a rank count: the logit of expert e of a token is at rank
// #{e' : l[e'] > l[e] or (l[e'] == l[e] and e' < e)}, which selects by
// (logit descending, expert ascending) as the separate router kernel does.
// The kernel also prefetches into L2 the first weights the expert kernel will
// stream, while HBM is otherwise idle. Both the router tiles and the prefetch
// are requested before waiting for the previous kernel (dependent launch).
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
  const float* bias;          // [64] or nullptr
  int32_t T, k, S;
  int32_t* idx;               // [T, k]
  float* gate;                // [T, k]
  int32_t* offsets;           // [65]
  int32_t* perm;              // [T k]
  int32_t* inv;               // [T k]
  // x_perm rows: primary_rows == 0: permutation order, [T k, H]; otherwise the
  // first primary_rows rows of expert e's segment at e * primary_rows and the
  // rest at 64 primary_rows + (position in the permutation), so the first tile
  // of every expert lies where the expert kernel can find it before the offsets
  __nv_bfloat16* x_perm;
  int32_t primary_rows;
  int32_t* counts;            // [grid, 64] per-CTA assignment counts (scratch)
  int32_t* sched;             // expert kernel's counters, cleared here
  int32_t sched_len;
  uint32_t* gbar;             // grid barrier counter, zeroed before the first launch on it
  uint32_t gbar_base;         // barriers already passed on gbar before this launch
  // L2 prefetch: n_prefetch blocks of prefetch_bytes, block i at base + i * stride
  const uint8_t* prefetch_base;
  int32_t n_prefetch;
  uint32_t prefetch_bytes;
  uint64_t prefetch_stride;
  // L2 prefetch by weight tile: the first pf_units gate/up units of the expert
  // kernel's fixed first wave (unit u = row block u % mblk of routed expert
  // u / mblk), pf_chunks 64-wide k-chunks each, through the gate/up tensor map
  int32_t pf_units, pf_mblk, pf_chunks;
};

constexpr int kEntryH = 1280;                          // hidden size of the kernel
constexpr int kEntryThreads = 512;                     // 2 groups x 4 quarters x 64 experts
constexpr int kEntryGroupTok = 2;                      // tokens per group and pass
constexpr int kEntryPassTok = 2 * kEntryGroupTok;      // tokens per pass
constexpr int kEntryMaxOwn = 12;                       // tokens a CTA may own (T <= 12 * grid)
constexpr int kEntrySlices = kEntryThreads / kRouterE; // CTA slices in the offsets phase
constexpr int kEntryMaxGridDev = 160;                  // CTAs of the kernel at most (the host keeps grid <= SMs <= this)

// Shared memory: router tiles, owned token rows (bf16), the pass's rows in
// fp32, plus 1 KB alignment slack.
__host__ __device__ constexpr int layer_entry_smem() {
  return 1024 + kRouterE * kEntryH * 2 + kEntryMaxOwn * kEntryH * 2 + kEntryPassTok * kEntryH * 4;
}

// L2 prefetch of n_prefetch weight blocks in 1 MB pieces, spread over the CTAs.
__device__ __forceinline__ void entry_l2_prefetch(const EntryArgs& a, int c, int G) {
  if (a.n_prefetch <= 0) return;
  constexpr uint32_t kPiece = 1u << 20;
  const uint32_t pieces_per = cdiv((int)a.prefetch_bytes, (int)kPiece);
  for (uint32_t i = c; i < (uint32_t)a.n_prefetch * pieces_per; i += G) {
    const uint32_t blk = i / pieces_per, pc = i - blk * pieces_per;
    const uint32_t off = pc * kPiece;
    bulk_prefetch_l2(a.prefetch_base + blk * a.prefetch_stride + off, min(kPiece, a.prefetch_bytes - off));
  }
}

// NT quarter chains (one per token) over the thread's quarter of h; each
// weight pair is unpacked once for all NT tokens. `wq` is the thread's row in
// the swizzled tile of its quarter's first 64 columns, `xq` the quarter's
// first fp32 input of token 0 (token j at + j * kEntryH). The chains run in
// 40 steps of 8 columns; the next step's weights and inputs are loaded while
// the current step's 8 FMAs run.
template <int NT>
__device__ __forceinline__ void quarter_chains(const uint8_t* wq, int sw, const float* xq, float* acc) {
  constexpr int kSteps = kEntryH / 4 / 8;  // 40 steps of 8 columns
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j] = 0.0f;
  auto wptr = [&](int i) {
    return reinterpret_cast<const uint4*>(wq + (i >> 3) * 8192 + (((i & 7) ^ sw) << 4));
  };
  uint4 wv = *wptr(0);
  float4 xa[NT], xb[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    xa[j] = reinterpret_cast<const float4*>(xq + j * kEntryH)[0];
    xb[j] = reinterpret_cast<const float4*>(xq + j * kEntryH)[1];
  }
#pragma unroll 4
  for (int i = 0; i < kSteps; ++i) {
    const int in = i + 1 < kSteps ? i + 1 : i;  // the last step reloads its own data
    const uint4 wn = *wptr(in);
    float4 xan[NT], xbn[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      xan[j] = reinterpret_cast<const float4*>(xq + j * kEntryH + in * 8)[0];
      xbn[j] = reinterpret_cast<const float4*>(xq + j * kEntryH + in * 8)[1];
    }
    const float w[8] = {bf16_lo(wv.x), bf16_hi(wv.x), bf16_lo(wv.y), bf16_hi(wv.y),
                        bf16_lo(wv.z), bf16_hi(wv.z), bf16_lo(wv.w), bf16_hi(wv.w)};
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      acc[j] = __fmaf_rn(xa[j].x, w[0], acc[j]);
      acc[j] = __fmaf_rn(xa[j].y, w[1], acc[j]);
      acc[j] = __fmaf_rn(xa[j].z, w[2], acc[j]);
      acc[j] = __fmaf_rn(xa[j].w, w[3], acc[j]);
      acc[j] = __fmaf_rn(xb[j].x, w[4], acc[j]);
      acc[j] = __fmaf_rn(xb[j].y, w[5], acc[j]);
      acc[j] = __fmaf_rn(xb[j].z, w[6], acc[j]);
      acc[j] = __fmaf_rn(xb[j].w, w[7], acc[j]);
      xa[j] = xan[j];
      xb[j] = xbn[j];
    }
    wv = wn;
  }
}

template <int K>
__global__ void __launch_bounds__(kEntryThreads, 1) moe_layer_entry(const __grid_constant__ CUtensorMap mR,
                                                                    const __grid_constant__ CUtensorMap mGu,
                                                                    const EntryArgs a) {
  constexpr int H = kEntryH, HQ = H / 4;
  extern __shared__ uint8_t esm_raw[];
  uint8_t* esm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(esm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ws = esm;                                                              // [H/64][64 rows][128 B]
  __nv_bfloat16* xo = reinterpret_cast<__nv_bfloat16*>(esm + kRouterE * H * 2);   // [own][H]
  float* xf = reinterpret_cast<float*>(xo + kEntryMaxOwn * H);                    // [kEntryPassTok][H]
  __shared__ __align__(8) uint64_t bars[2];                                       // weights, token rows
  __shared__ __align__(16) float part[4][kEntryPassTok][kRouterE];                // [quarter][token][expert]
  __shared__ float logit[kEntryPassTok][kRouterE];
  __shared__ float sum_s[kEntryPassTok][2];
  __shared__ int32_t idx_s[kEntryMaxOwn * K];
  __shared__ int cnt_s[kRouterE], tot_s[kRouterE], pre_s[kRouterE], off_s[kRouterE];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const uint64_t limit = g_wait_timeout_ns;
  const int P = cdiv(a.T, G);
  const int t_begin = min(a.T, c * P), t_end = min(a.T, t_begin + P), n_own = t_end - t_begin;

  griddep_launch_dependents();
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    if (n_own > 0) {  // the router matrix is streamed in while the combine runs
      mbar_arrive_expect_tx(&bars[0], kRouterE * H * 2);
      constexpr int nkc = H / 64;
      for (int i = 0; i < nkc; ++i) {  // CTAs start at different tiles: spread over L2 slices
        const int kc = (i + c) % nkc;
        tma_load_2d(ws + kc * 8192, &mR, &bars[0], kc * 64, 0);
      }
    }
    // the first weights the expert kernel streams go to L2 now, while HBM is idle
    for (int u = c; u < a.pf_units; u += G) {
      const int e = u / a.pf_mblk, mb = u - e * a.pf_mblk;
      for (int kc = 0; kc < a.pf_chunks; ++kc) tma_prefetch_4d(&mGu, kc * 64, mb * 128, 0, e);
    }
    entry_l2_prefetch(a, c, G);  // the expert kernel's first weights, to L2 while this kernel routes
  }
  if (tid < kRouterE) cnt_s[tid] = 0;
  __syncthreads();
  griddep_wait();  // the router tiles and the L2 prefetch are under way; now the previous kernel's data
  bool ok = true;

  // ---- A1: this CTA's input rows
  if (a.prev_o != nullptr) {
    constexpr int per_row = H / 8;
    for (int i = tid; i < n_own * per_row; i += blockDim.x) {
      const int tl = i / per_row, cc = i - tl * per_row, t = t_begin + tl;
      const uint4 v = combine8(a.prev_x, a.prev_o, a.prev_inv, a.prev_gate, a.T, H, a.k, a.S, a.prev_add_residual, t, cc);
      reinterpret_cast<uint4*>(a.x_out + (size_t)t * H)[cc] = v;
      reinterpret_cast<uint4*>(xo + (size_t)tl * H)[cc] = v;
      if (tl < kEntryPassTok) {  // the first pass's rows in fp32 too
        float4* xf4 = reinterpret_cast<float4*>(xf + (size_t)tl * H + cc * 8);
        xf4[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
        xf4[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
      }
    }
  } else if (n_own > 0) {
    if (tid == 0) {
      mbar_arrive_expect_tx(&bars[1], n_own * H * 2);
      for (int r = 0; r < n_own; ++r) bulk_load(xo + r * H, a.x_in + (size_t)(t_begin + r) * H, H * 2, &bars[1]);
    }
    if (!mbar_wait(&bars[1], 0, limit)) {
      record_error(kErrTimeout, 152);
      ok = false;
    }
  }
  if (n_own > 0 && !mbar_wait(&bars[0], 0, limit)) {
    record_error(kErrTimeout, 155);
    ok = false;
  }
  ok = __syncthreads_and(ok);  // one decision for the whole CTA

  // ---- A2: logits, top-k and gates, kEntryPassTok tokens at a time
  const int grp = tid >> 8, qq = (tid >> 6) & 3, e = tid & 63;
  for (int g0 = 0; ok && g0 < n_own; g0 += kEntryPassTok) {
    const int n_pass = min(kEntryPassTok, n_own - g0);
    if (g0 > 0 || a.prev_o == nullptr) {  // the combine wrote the first pass's fp32 rows
      for (int i = tid; i < n_pass * H / 2; i += blockDim.x) {  // the pass's rows to fp32
        const uint32_t v = reinterpret_cast<const uint32_t*>(xo + (size_t)g0 * H)[i];
        reinterpret_cast<float2*>(xf)[i] = make_float2(bf16_lo(v), bf16_hi(v));
      }
      __syncthreads();
    }
    const int tok0 = grp * kEntryGroupTok, n_grp = min(kEntryGroupTok, n_pass - tok0);  // warp-uniform
    if (n_grp > 0) {
      const uint8_t* wq = ws + qq * (HQ / 64) * 8192 + e * 128;
      const float* xq = xf + tok0 * H + qq * HQ;
      float acc[kEntryGroupTok];
      if (n_grp == 2) {
        quarter_chains<2>(wq, e & 7, xq, acc);
        part[qq][tok0 + 1][e] = acc[1];
      } else {
        quarter_chains<1>(wq, e & 7, xq, acc);
      }
      part[qq][tok0][e] = acc[0];
    }
    __syncthreads();
    const int tk = tid >> 6;  // (token, expert) threads for the rest of the pass
    float l = 0.0f;
    int rank = kRouterE;
    if (tk < n_pass) {
      l = (part[0][tk][e] + part[1][tk][e]) + (part[2][tk][e] + part[3][tk][e]);
      if (a.bias != nullptr) l = __fadd_rn(l, a.bias[e]);
      logit[tk][e] = l;
    }
    __syncthreads();
    float mx = l;  // the token's largest logit, taken in the same scan
    if (tk < n_pass) {
      rank = 0;
#pragma unroll 8
      for (int j = 0; j < kRouterE; ++j) {
        const float o = logit[tk][j];
        rank += (o > l || (o == l && j < e)) ? 1 : 0;
        mx = fmaxf(mx, o);
      }
    }
    float ex = 0.0f;
    if (tk < n_pass) {
      ex = expf(l - mx);
      float s = ex;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) sum_s[tk][(tid >> 5) & 1] = s;
    }
    __syncthreads();
    if (tk < n_pass && rank < K) {
      const int own = g0 + tk, t = t_begin + own;
      idx_s[own * K + rank] = e;
      a.idx[(size_t)t * K + rank] = e;
      a.gate[(size_t)t * K + rank] = ex / (sum_s[tk][0] + sum_s[tk][1]);
    }
    __syncthreads();
  }
  for (int i = tid; ok && i < n_own * K; i += blockDim.x) {
    int key = idx_s[i];
    if ((unsigned)key >= (unsigned)kRouterE) {  // only non-finite logits get here
      record_error(kErrBounds, 154);
      idx_s[i] = key = 0;
    }
    atomicAdd(&cnt_s[key], 1);
  }
  __syncthreads();
  if (tid < kRouterE) a.counts[(size_t)c * kRouterE + tid] = cnt_s[tid];
  if (G > 1) ok = grid_barrier(a.gbar, (a.gbar_base + 1) * G, limit, 153) && ok;
  else __syncthreads();
  if (!ok) return;

  // ---- B: offsets, positions of this CTA's assignments, rows to their positions
  {
    int* red = reinterpret_cast<int*>(&part[0][0][0]);  // [2][kEntrySlices][64]
    const int s = tid >> 6;
    int tot = 0, pre = 0;
    // every count this thread needs is requested at once: one L2 round trip
    int v[kEntryMaxGridDev / kEntrySlices];
#pragma unroll
    for (int i = 0; i < kEntryMaxGridDev / kEntrySlices; ++i) {
      const int cc = s + i * kEntrySlices;
      v[i] = cc < G ? __ldcg(a.counts + (size_t)cc * kRouterE + e) : 0;
    }
#pragma unroll
    for (int i = 0; i < kEntryMaxGridDev / kEntrySlices; ++i) {
      tot += v[i];
      pre += s + i * kEntrySlices < c ? v[i] : 0;
    }
    red[s * kRouterE + e] = tot;
    red[(kEntrySlices + s) * kRouterE + e] = pre;
    __syncthreads();
    if (tid < kRouterE) {
      int t2 = 0, p2 = 0;
#pragma unroll
      for (int j = 0; j < kEntrySlices; ++j) {
        t2 += red[j * kRouterE + tid];
        p2 += red[(kEntrySlices + j) * kRouterE + tid];
      }
      tot_s[tid] = t2;
      pre_s[tid] = p2;
    }
  }
  __syncthreads();
  if (warp == 0) scan64_warp(tot_s, off_s, lane);
  __syncthreads();
  const int N = a.T * a.k;
  if (c == 0) {
    if (tid <= kRouterE) a.offsets[tid] = tid < kRouterE ? off_s[tid] : N;
    for (int i = tid; i < a.sched_len; i += blockDim.x) a.sched[i] = 0;
  }
  const int a_begin = t_begin * K;
  int my_pos = -1;
  if (tid < n_own * K) {
    const int key = idx_s[tid];
    int rank = 0;
    for (int j2 = 0; j2 < tid; ++j2) rank += idx_s[j2] == key;
    my_pos = off_s[key] + pre_s[key] + rank;
    if (VG_IN_BOUNDS((unsigned)my_pos < (unsigned)N && a_begin + tid < N, 402)) {
      a.perm[my_pos] = a_begin + tid;
      a.inv[a_begin + tid] = my_pos;
      const int r = pre_s[key] + rank;  // rank within the expert's segment
      const int P = a.primary_rows;
      my_pos = P == 0 ? my_pos : r < P ? key * P + r : kRouterE * P + my_pos;  // the row of x_perm
    } else {
      my_pos = -1;
    }
  }
  __syncthreads();  // every rank was taken from idx_s before it is overwritten
  if (tid < n_own * K) idx_s[tid] = my_pos;
  __syncthreads();
  [[maybe_unused]] const int xperm_rows = N + kRouterE * a.primary_rows;  // bound of the gather checks
  for (int i = warp; i < n_own * K; i += blockDim.x / 32) {
    if (!VG_IN_BOUNDS((unsigned)idx_s[i] < (unsigned)xperm_rows, 403)) continue;
    const uint4* src = reinterpret_cast<const uint4*>(xo + (size_t)(i / K) * H);
    uint4* dst = reinterpret_cast<uint4*>(a.x_perm + (size_t)idx_s[i] * H);
    for (int cc = lane; cc < H / 8; cc += 32) dst[cc] = src[cc];
  }
}

}  // namespace vg
