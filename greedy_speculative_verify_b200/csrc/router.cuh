// Router of the MoE layer: fp32 logits, top-k selection and softmax gates.
//
// Top-6 of 64 routed experts per token ("Jina AI's 3.4B OCR model targets faster
// page parsing", "A compressed visual front end"; jina-ocr-v1 model card,
// architecture paragraph). The pages give no formula. Reading used here:
//  * l[t,e] = sum_h x[t,h] w[e,h] in fp32 as four partial sums over the
//    contiguous quarters of h, each an fma chain in increasing h from +0,
//    combined as (q0 + q1) + (q2 + q3), then + bias[e] in one fp32 addition.
//    The order is part of the definition so that the selected experts are
//    reproducible bit for bit; the quarter chains keep the critical path at
//    H/4 dependent fmas.
//  * selection by (l descending, e ascending); softmax over all E logits,
//    weights not renormalised over the selected experts.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kRouterE = 64;

// One warp selects the top-K of 64 logits of one token and writes the expert
// ids (descending logit, lower id first among equal logits) and the softmax
// probabilities over all 64 at those ids.
template <int K>
__device__ __forceinline__ void topk_softmax_warp(const float* l, int lane, int32_t* idx_out, float* w_out) {
  const float v0 = l[lane], v1 = l[lane + 32];
  bool u0 = false, u1 = false;
  float sel_v[K];
  int sel_i[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    float bv;
    int bi;
    if (!u0 && (u1 || v0 >= v1)) {
      bv = v0;
      bi = lane;
    } else if (!u1) {
      bv = v1;
      bi = lane + 32;
    } else {
      bv = -INFINITY;
      bi = 1 << 30;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    sel_v[j] = bv;
    sel_i[j] = bi;
    if (bi == lane) u0 = true;
    if (bi == lane + 32) u1 = true;
  }
  const float m = sel_v[0];
  float s = expf(v0 - m) + expf(v1 - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
#pragma unroll
  for (int j = 0; j < K; ++j) {
    if (lane == j) {
      idx_out[j] = sel_i[j];
      w_out[j] = expf(sel_v[j] - m) / s;
    }
  }
}

// Decode sizes compute the logits inside the layer-entry kernel (layer_entry.cuh).

// Large token counts: a 128-token x 64-expert block tile, staged through shared
// memory 32 k at a time; each thread owns 8 tokens x 4 experts and runs every
// output's chain in increasing k. The finished quarter sums wait in (dynamic)
// shared memory rather than registers, so that two blocks fit an SM.
constexpr int kRtPartBytes = 2 * 128 * (kRouterE + 1) * 4;  // (q0 + q1) and q2 of a block tile

template <int K>
__global__ void __launch_bounds__(256, 2) router_topk_tiled(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ w,
                                                         const float* __restrict__ bias, int T, int H,
                                                         int32_t* __restrict__ idx_out,
                                                         float* __restrict__ w_out) {
  constexpr int BT = 128, BK = 32, XS = BT + 4, WS = kRouterE + 4, LS = kRouterE + 1;
  __shared__ __align__(16) float buf[BT * LS];  // k-loop: xs[BK][XS] | ws[BK][WS]; after: logits[BT][LS]
  float* xs = buf;
  float* ws = buf + BK * XS;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const int t0 = blockIdx.x * BT;
  // quarter sums: acc runs the current quarter's chains; p01 and p2 keep the
  // finished ones until (q0 + q1) + (q2 + q3) (H/4 is a multiple of BK); each
  // thread reads back only the entries it wrote
  extern __shared__ float rt_part[];
  float* p01 = rt_part;               // [BT][LS]
  float* p2 = rt_part + BT * LS;      // [BT][LS]
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  const int HQ = H / 4;

  // the next chunk's x and w are loaded into registers while the current one
  // is multiplied, so the loads never stall the fma loop
  uint4 xv[2], wv;
  auto load_chunk = [&](int k0) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int q = tid + r * 256;
      const int tok = q >> 2, kq = (q & 3) * 8;
      xv[r] = make_uint4(0, 0, 0, 0);
      if (t0 + tok < T) xv[r] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + tok) * H + k0 + kq));
    }
    wv = __ldg(reinterpret_cast<const uint4*>(w + (size_t)(tid >> 2) * H + k0 + (tid & 3) * 8));
  };
  load_chunk(0);
  for (int k0 = 0; k0 < H; k0 += BK) {
    // x tile: 128 tokens x 32 k = 512 uint4
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int q = tid + r * 256;
      const int tok = q >> 2, kq = (q & 3) * 8;
      const uint4 v = xv[r];
      xs[(kq + 0) * XS + tok] = bf16_lo(v.x);
      xs[(kq + 1) * XS + tok] = bf16_hi(v.x);
      xs[(kq + 2) * XS + tok] = bf16_lo(v.y);
      xs[(kq + 3) * XS + tok] = bf16_hi(v.y);
      xs[(kq + 4) * XS + tok] = bf16_lo(v.z);
      xs[(kq + 5) * XS + tok] = bf16_hi(v.z);
      xs[(kq + 6) * XS + tok] = bf16_lo(v.w);
      xs[(kq + 7) * XS + tok] = bf16_hi(v.w);
    }
    {
      const int ex = tid >> 2, kq = (tid & 3) * 8;
      const uint4 v = wv;
      ws[(kq + 0) * WS + ex] = bf16_lo(v.x);
      ws[(kq + 1) * WS + ex] = bf16_hi(v.x);
      ws[(kq + 2) * WS + ex] = bf16_lo(v.y);
      ws[(kq + 3) * WS + ex] = bf16_hi(v.y);
      ws[(kq + 4) * WS + ex] = bf16_lo(v.z);
      ws[(kq + 5) * WS + ex] = bf16_hi(v.z);
      ws[(kq + 6) * WS + ex] = bf16_lo(v.w);
      ws[(kq + 7) * WS + ex] = bf16_hi(v.w);
    }
    if (k0 + BK < H) load_chunk(k0 + BK);
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(xs + kk * XS + ty * 8);
      const float4 a1 = *reinterpret_cast<const float4*>(xs + kk * XS + ty * 8 + 4);
      const float4 b = *reinterpret_cast<const float4*>(ws + kk * WS + tx * 4);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
    const int qend = (k0 + BK) / HQ;  // a quarter ends with this chunk when (k0 + BK) % HQ == 0
    if ((k0 + BK) % HQ == 0 && qend < 4) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float* a01 = p01 + (ty * 8 + i) * LS + tx * 4 + j;
          if (qend == 1) *a01 = acc[i][j];
          else if (qend == 2) *a01 = *a01 + acc[i][j];
          else p2[(ty * 8 + i) * LS + tx * 4 + j] = acc[i][j];
          acc[i][j] = 0.0f;
        }
    }
  }
  // the last quarter ends with the last chunk: the logit is (q0 + q1) + (q2 + q3)
  float q01[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = (ty * 8 + i) * LS + tx * 4 + j;
      q01[i][j] = p01[o] + (p2[o] + acc[i][j]);
    }
  float* logits = buf;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = tx * 4 + j;
    const float b = bias != nullptr ? bias[e] : 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float v = q01[i][j];
      if (bias != nullptr) v = __fadd_rn(v, b);
      logits[(ty * 8 + i) * LS + e] = v;
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < BT; r += 8) {
    const int t = t0 + r;
    if (t < T) topk_softmax_warp<K>(logits + r * LS, lane, idx_out + (size_t)t * K, w_out + (size_t)t * K);
  }
}

}  // namespace vg
