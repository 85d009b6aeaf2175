// Entry of an MoE layer at decode sizes up to two tokens per CTA (T <= 2 x the
// grid), built to share an SM with a CTA of the expert-GEMM kernel.
//
// Same work and outputs as moe_layer_entry (the previous layer's weighted
// combine, router logits, top-k and softmax, per-CTA expert counts, one grid
// barrier, offsets, stable positions, perm / inv and the row gather), with a
// footprint small enough (about 19 KB of shared memory, 256 threads of at most
// 192 registers) that it is resident next to the expert kernel of the previous
// layer while that one runs. Consequences, with dependent launches:
//  * the kernel is already on the SMs when the previous expert kernel ends, and
//    its router weights are already in registers: each thread (quarter q,
//    expert e) loads its 320 weights of row e before waiting for the previous
//    kernel (the weights are immutable);
//  * its own dependent, the next expert kernel, is launched as soon as every
//    CTA here has started, so the SMs the previous expert kernel frees take the
//    next expert kernel's CTAs at once, and those stream their first weights
//    while the routing is computed here.
//
// CTA c owns tokens 2c and 2c+1. Logits follow the router's definition
// (router.cuh): four quarter fma chains in increasing h from +0, combined as
// (q0 + q1) + (q2 + q3), then + b_e; thread (q, e) runs the chains of both
// tokens, unpacking each weight pair once. Top-k and softmax: one warp per
// token (topk_softmax_warp). Positions: offset of the expert + assignments to
// that expert in lower CTAs + rank among this CTA's own, so the permutation is
// the stable order of assignment ids.
#pragma once
#include "combine.cuh"
#include "common.cuh"
#include "layer_entry.cuh"
#include "router.cuh"
#include "sort.cuh"

namespace vg {

constexpr int kEsTok = 2;        // tokens per CTA
constexpr int kEsThreads = 256;  // 4 quarters x 64 experts
constexpr int kEsMaxGrid = 160;  // CTAs at most (the counts phase reads up to 40 per thread)

template <int K>
__global__ void __maxnreg__(192) moe_entry_small(const __nv_bfloat16* __restrict__ router_w, const EntryArgs a) {
  constexpr int H = kEntryH, HQ = H / 4, NW = HQ / 8;  // 40 vectors of 8 weights per thread
  constexpr int per_row = H / 8;
  __shared__ __align__(16) float xf[kEsTok][H];
  __shared__ __align__(16) __nv_bfloat16 xb[kEsTok][H];
  __shared__ float part[4][kEsTok][kRouterE];
  __shared__ float logit[kEsTok][kRouterE];
  __shared__ int32_t idx_s[kEsTok * K];
  __shared__ float gate_s[kEsTok * K];
  __shared__ int cnt_s[kRouterE], tot_s[kRouterE], pre_s[kRouterE], off_s[kRouterE];
  __shared__ int red_s[2][4][kRouterE];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int q = tid >> 6, e = tid & 63;
  const int t_begin = c * kEsTok;
  const int n_own = max(0, min(kEsTok, a.T - t_begin));
  const uint64_t limit = g_wait_timeout_ns;

  griddep_launch_dependents();
  uint4 w[NW];  // row e, h = 320 q .. 320 q + 319
  {
    const uint4* src = reinterpret_cast<const uint4*>(router_w + (size_t)e * H + q * HQ);
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = __ldg(src + i);
  }
  if (tid == 0 && a.n_prefetch > 0) {  // the first weights the expert kernel streams go to L2 now
    constexpr uint32_t kPiece = 1u << 20;
    const uint32_t pieces_per = cdiv((int)a.prefetch_bytes, (int)kPiece);
    for (uint32_t i = c; i < (uint32_t)a.n_prefetch * pieces_per; i += G) {
      const uint32_t blk = i / pieces_per, pc = i - blk * pieces_per;
      const uint32_t off = pc * kPiece;
      bulk_prefetch_l2(a.prefetch_base + blk * a.prefetch_stride + off, min(kPiece, a.prefetch_bytes - off));
    }
  }
  if (tid < kRouterE) cnt_s[tid] = 0;
  if (n_own < kEsTok) {  // the absent token's row reads as zeros (its logits are never used)
    for (int i = tid; i < H; i += kEsThreads) xf[1][i] = 0.0f;
  }
  griddep_wait();  // from here on, data the previous kernels wrote

  // ---- A1: this CTA's input rows: bf16 (for the gather) and fp32 (for the logits)
  for (int i = tid; i < n_own * per_row; i += kEsThreads) {
    const int tl = i / per_row, cc = i - tl * per_row, t = t_begin + tl;
    uint4 v;
    if (a.prev_o != nullptr) {
      v = combine8(a.prev_x, a.prev_o, a.prev_inv, a.prev_gate, a.T, H, a.k, a.S, a.prev_add_residual, t, cc);
      reinterpret_cast<uint4*>(a.x_out + (size_t)t * H)[cc] = v;
    } else {
      v = reinterpret_cast<const uint4*>(a.x_in + (size_t)t * H)[cc];
    }
    reinterpret_cast<uint4*>(&xb[tl][0])[cc] = v;
    float4* f = reinterpret_cast<float4*>(&xf[tl][cc * 8]);
    f[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    f[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
  __syncthreads();

  // ---- A2: quarter chains of both tokens
  {
    const float* x0 = &xf[0][q * HQ];
    const float* x1 = &xf[1][q * HQ];
    float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const float wv[8] = {bf16_lo(w[i].x), bf16_hi(w[i].x), bf16_lo(w[i].y), bf16_hi(w[i].y),
                           bf16_lo(w[i].z), bf16_hi(w[i].z), bf16_lo(w[i].w), bf16_hi(w[i].w)};
      const float4 a0 = *reinterpret_cast<const float4*>(x0 + 8 * i);
      const float4 a1 = *reinterpret_cast<const float4*>(x0 + 8 * i + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(x1 + 8 * i);
      const float4 b1 = *reinterpret_cast<const float4*>(x1 + 8 * i + 4);
      acc0 = __fmaf_rn(a0.x, wv[0], acc0);
      acc1 = __fmaf_rn(b0.x, wv[0], acc1);
      acc0 = __fmaf_rn(a0.y, wv[1], acc0);
      acc1 = __fmaf_rn(b0.y, wv[1], acc1);
      acc0 = __fmaf_rn(a0.z, wv[2], acc0);
      acc1 = __fmaf_rn(b0.z, wv[2], acc1);
      acc0 = __fmaf_rn(a0.w, wv[3], acc0);
      acc1 = __fmaf_rn(b0.w, wv[3], acc1);
      acc0 = __fmaf_rn(a1.x, wv[4], acc0);
      acc1 = __fmaf_rn(b1.x, wv[4], acc1);
      acc0 = __fmaf_rn(a1.y, wv[5], acc0);
      acc1 = __fmaf_rn(b1.y, wv[5], acc1);
      acc0 = __fmaf_rn(a1.z, wv[6], acc0);
      acc1 = __fmaf_rn(b1.z, wv[6], acc1);
      acc0 = __fmaf_rn(a1.w, wv[7], acc0);
      acc1 = __fmaf_rn(b1.w, wv[7], acc1);
    }
    part[q][0][e] = acc0;
    part[q][1][e] = acc1;
  }
  __syncthreads();

  // ---- A3: logits, then top-k and softmax, one warp per token
  if (tid < kEsTok * kRouterE) {
    const int tk = tid >> 6;
    float l = (part[0][tk][e] + part[1][tk][e]) + (part[2][tk][e] + part[3][tk][e]);
    if (a.bias != nullptr) l = __fadd_rn(l, a.bias[e]);
    logit[tk][e] = l;
  }
  __syncthreads();
  if (warp < n_own) topk_softmax_warp<K>(logit[warp], lane, &idx_s[warp * K], &gate_s[warp * K]);
  __syncthreads();
  if (tid < n_own * K) {
    int key = idx_s[tid];
    if ((unsigned)key >= (unsigned)kRouterE) {  // only non-finite logits get here
      record_error(kErrBounds, 157);
      idx_s[tid] = key = 0;
    }
    a.idx[(size_t)t_begin * K + tid] = key;
    a.gate[(size_t)t_begin * K + tid] = gate_s[tid];
    atomicAdd(&cnt_s[key], 1);
  }
  __syncthreads();
  if (tid < kRouterE) a.counts[(size_t)c * kRouterE + tid] = cnt_s[tid];
  if (G > 1) {
    if (!grid_barrier(a.gbar, (a.gbar_base + 1) * G, limit, 158)) return;
  } else {
    __syncthreads();
  }

  // ---- B: offsets and the positions of this CTA's assignments
  {
    const int s = tid >> 6;  // CTAs s, s + 4, s + 8, ...: all loads issued together
    int tot = 0, pre = 0;
#pragma unroll
    for (int i = 0; i < kEsMaxGrid / 4; ++i) {
      const int cc = s + 4 * i;
      if (cc < G) {
        const int v = __ldcg(a.counts + (size_t)cc * kRouterE + e);
        tot += v;
        pre += cc < c ? v : 0;
      }
    }
    red_s[0][s][e] = tot;
    red_s[1][s][e] = pre;
  }
  __syncthreads();
  if (tid < kRouterE) {
    tot_s[tid] = (red_s[0][0][tid] + red_s[0][1][tid]) + (red_s[0][2][tid] + red_s[0][3][tid]);
    pre_s[tid] = (red_s[1][0][tid] + red_s[1][1][tid]) + (red_s[1][2][tid] + red_s[1][3][tid]);
  }
  __syncthreads();
  if (warp == 0) scan64_warp(tot_s, off_s, lane);
  __syncthreads();
  const int N = a.T * a.k;
  if (c == 0) {
    if (tid <= kRouterE) a.offsets[tid] = tid < kRouterE ? off_s[tid] : N;
    for (int i = tid; i < a.sched_len; i += kEsThreads) a.sched[i] = 0;
  }
  const int a_begin = t_begin * K;
  int my_pos = -1;
  if (tid < n_own * K) {
    const int key = idx_s[tid];
    int rank = 0;
    for (int j2 = 0; j2 < tid; ++j2) rank += idx_s[j2] == key;
    my_pos = off_s[key] + pre_s[key] + rank;
    a.perm[my_pos] = a_begin + tid;
    a.inv[a_begin + tid] = my_pos;
  }
  __syncthreads();  // every rank was taken from idx_s before it is overwritten
  if (tid < n_own * K) idx_s[tid] = my_pos;
  __syncthreads();
  for (int i = tid; i < n_own * K * per_row; i += kEsThreads) {
    const int asg = i / per_row, cc = i - asg * per_row;
    reinterpret_cast<uint4*>(a.x_perm + (size_t)idx_s[asg] * H)[cc] =
        reinterpret_cast<const uint4*>(&xb[asg / K][0])[cc];
  }
}

}  // namespace vg
