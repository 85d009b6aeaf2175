// Weighted combine of an MoE layer: y[t] = [x[t] +] sum_s o_shared[s][t] +
// sum_j g[t,j] * o[inv[t,j]], rounded once to bf16. Expert outputs o are the
// rows of the expert kernel: routed ones in permutation order, shared expert s
// on token t at row k*T + s*T + t. The summation order is fixed (shared
// experts, then routed slots j = 0..k-1, then the residual).
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kCombineMaxK = 8, kCombineMaxS = 4;  // bounds of k and S the unrolled loads cover

__device__ __forceinline__ void acc8(float* y, const uint4 v) {
  y[0] += bf16_lo(v.x); y[1] += bf16_hi(v.x); y[2] += bf16_lo(v.y); y[3] += bf16_hi(v.y);
  y[4] += bf16_lo(v.z); y[5] += bf16_hi(v.z); y[6] += bf16_lo(v.w); y[7] += bf16_hi(v.w);
}

// Eight consecutive outputs y[t, 8c .. 8c+7] as one 16-byte vector. Every load
// is issued before the first sum (the routed rows' indices, then all rows), so
// the thread waits for two memory round trips, not one per expert; the sums
// then run in the fixed order above. Requires k <= kCombineMaxK and
// S <= kCombineMaxS (the launch validates both).
__device__ __forceinline__ uint4 combine8(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ o,
                                          const int32_t* __restrict__ inv, const float* __restrict__ g, int T, int H,
                                          int k, int S, int add_residual, int t, int c) {
  int p[kCombineMaxK];
  float gj[kCombineMaxK];
#pragma unroll
  for (int j = 0; j < kCombineMaxK; ++j) {
    p[j] = j < k ? __ldg(inv + t * k + j) : -1;
    gj[j] = j < k ? __ldg(g + t * k + j) : 0.0f;
  }
  uint4 vs[kCombineMaxS], vr[kCombineMaxK], vx = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int s = 0; s < kCombineMaxS; ++s)
    if (s < S) vs[s] = __ldg(reinterpret_cast<const uint4*>(o + ((size_t)k * T + (size_t)s * T + t) * H) + c);
  if (add_residual) vx = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H) + c);
#pragma unroll
  for (int j = 0; j < kCombineMaxK; ++j) {
    if (j < k && !VG_IN_BOUNDS((unsigned)p[j] < (unsigned)(k * T), 401)) p[j] = -1;
    if (j < k && p[j] >= 0) vr[j] = __ldg(reinterpret_cast<const uint4*>(o + (size_t)p[j] * H) + c);
  }
  float y[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) y[j] = 0.0f;
#pragma unroll
  for (int s = 0; s < kCombineMaxS; ++s)
    if (s < S) acc8(y, vs[s]);
#pragma unroll
  for (int j = 0; j < kCombineMaxK; ++j) {
    if (j < k && p[j] >= 0) {
      const uint4 v = vr[j];
      const float gg = gj[j];
      y[0] = __fmaf_rn(gg, bf16_lo(v.x), y[0]); y[1] = __fmaf_rn(gg, bf16_hi(v.x), y[1]);
      y[2] = __fmaf_rn(gg, bf16_lo(v.y), y[2]); y[3] = __fmaf_rn(gg, bf16_hi(v.y), y[3]);
      y[4] = __fmaf_rn(gg, bf16_lo(v.z), y[4]); y[5] = __fmaf_rn(gg, bf16_hi(v.z), y[5]);
      y[6] = __fmaf_rn(gg, bf16_lo(v.w), y[6]); y[7] = __fmaf_rn(gg, bf16_hi(v.w), y[7]);
    }
  }
  if (add_residual) acc8(y, vx);
  uint4 r;
  __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
  __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]), h3 = __floats2bfloat162_rn(y[6], y[7]);
  r.x = *reinterpret_cast<uint32_t*>(&h0);
  r.y = *reinterpret_cast<uint32_t*>(&h1);
  r.z = *reinterpret_cast<uint32_t*>(&h2);
  r.w = *reinterpret_cast<uint32_t*>(&h3);
  return r;
}

// The same sums with the loads of one expert row at a time: fewer registers,
// so more threads in flight when the kernel streams many tokens.
__device__ __forceinline__ uint4 combine8_seq(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ o,
                                          const int32_t* __restrict__ inv, const float* __restrict__ g, int T, int H,
                                          int k, int S, int add_residual, int t, int c) {
  float y[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) y[j] = 0.0f;
  for (int s = 0; s < S; ++s) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(o + ((size_t)k * T + (size_t)s * T + t) * H) + c);
    y[0] += bf16_lo(v.x); y[1] += bf16_hi(v.x); y[2] += bf16_lo(v.y); y[3] += bf16_hi(v.y);
    y[4] += bf16_lo(v.z); y[5] += bf16_hi(v.z); y[6] += bf16_lo(v.w); y[7] += bf16_hi(v.w);
  }
  for (int j = 0; j < k; ++j) {
    const int p = inv[t * k + j];
    if (!VG_IN_BOUNDS((unsigned)p < (unsigned)(k * T), 401)) continue;
    const float gj = g[t * k + j];
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(o + (size_t)p * H) + c);
    y[0] = __fmaf_rn(gj, bf16_lo(v.x), y[0]); y[1] = __fmaf_rn(gj, bf16_hi(v.x), y[1]);
    y[2] = __fmaf_rn(gj, bf16_lo(v.y), y[2]); y[3] = __fmaf_rn(gj, bf16_hi(v.y), y[3]);
    y[4] = __fmaf_rn(gj, bf16_lo(v.z), y[4]); y[5] = __fmaf_rn(gj, bf16_hi(v.z), y[5]);
    y[6] = __fmaf_rn(gj, bf16_lo(v.w), y[6]); y[7] = __fmaf_rn(gj, bf16_hi(v.w), y[7]);
  }
  if (add_residual) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H) + c);
    y[0] += bf16_lo(v.x); y[1] += bf16_hi(v.x); y[2] += bf16_lo(v.y); y[3] += bf16_hi(v.y);
    y[4] += bf16_lo(v.z); y[5] += bf16_hi(v.z); y[6] += bf16_lo(v.w); y[7] += bf16_hi(v.w);
  }
  uint4 r;
  __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
  __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]), h3 = __floats2bfloat162_rn(y[6], y[7]);
  r.x = *reinterpret_cast<uint32_t*>(&h0);
  r.y = *reinterpret_cast<uint32_t*>(&h1);
  r.z = *reinterpret_cast<uint32_t*>(&h2);
  r.w = *reinterpret_cast<uint32_t*>(&h3);
  return r;
}

// One thread per 8 consecutive hidden elements; kAllLoadsFirst picks
// combine8 (few tokens: latency) or combine8_seq (many tokens: throughput).
template <bool kAllLoadsFirst>
__global__ void __launch_bounds__(256) moe_combine(const __nv_bfloat16* __restrict__ x,
                                                   const __nv_bfloat16* __restrict__ o,
                                                   const int32_t* __restrict__ inv, const float* __restrict__ g,
                                                   int T, int H, int k, int S, int add_residual,
                                                   __nv_bfloat16* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int per_row = H / 8;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * per_row) return;
  const int t = i / per_row, c = i - t * per_row;
  reinterpret_cast<uint4*>(out + (size_t)t * H)[c] =
      kAllLoadsFirst ? combine8(x, o, inv, g, T, H, k, S, add_residual, t, c)
                     : combine8_seq(x, o, inv, g, T, H, k, S, add_residual, t, c);
}

}  // namespace vg
