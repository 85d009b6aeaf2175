// Recursive draft block (FastMTP): one dense block reused for each of the K
// draft steps, fed its own hidden state and its own last token ("Jina AI's
// 3.4B OCR model targets faster page parsing", "FastMTP cuts decoding work";
// "jina-ocr-v1: Schnellere Dokumentenanalyse auf kostengünstigen GPUs",
// "Modell und Training" and "Erste Schritte"). The block's inside is not on the
// pages; the reading computed here, step i = 1..K from (g, y) = (g_{i-1}, y_{i-1}):
//   u   = [rmsnorm(g) * gamma_h ; rmsnorm(E[y]) * gamma_e]     (bf16, 2H)
//   z   = W_p u                                                (bf16, H)
//   g_i = z + FFN(rmsnorm(z) * gamma_f)                        (bf16, H)
//   y_i = argmax(LM g_i)
// with rmsnorm(x) = x / sqrt(mean(x^2) + 1e-6), FFN a SwiGLU of one expert's
// shape. The two matrix products run on the expert GEMM kernel (W_p as a
// down-only unit list over K = 2H, the FFN as a single shared expert), the
// argmax on the LM-head kernel; this header has the row-wise kernels around them.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kMtpThreads = 256;
constexpr float kRmsEps = 1e-6f;

// Sum over the block (kMtpThreads threads) of one value per thread; every thread
// gets the total. `red` holds kMtpThreads / 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int w = 0; w < kMtpThreads / 32; ++w) s += red[w];
  return s;
}

// dst[0..H) = bf16(src * (1 / sqrt(mean(src^2) + eps)) * gamma), one row, in
// fp32 (H a multiple of 8: 8 elements per step).
__device__ __forceinline__ void rmsnorm_row(const __nv_bfloat16* __restrict__ src, const float* __restrict__ gamma,
                                            int H, __nv_bfloat16* __restrict__ dst, float* red) {
  float ss = 0.0f;
  for (int c = threadIdx.x; c < H / 8; c += kMtpThreads) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a = bf16_lo(w[q]), b = bf16_hi(w[q]);
      ss = __fmaf_rn(a, a, ss);
      ss = __fmaf_rn(b, b, ss);
    }
  }
  const float tot = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(tot / (float)H + kRmsEps);
  for (int c = threadIdx.x; c < H / 8; c += kMtpThreads) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int h = 8 * c + 2 * q;
      const __nv_bfloat162 r =
          __floats2bfloat162_rn(bf16_lo(w[q]) * inv * gamma[h], bf16_hi(w[q]) * inv * gamma[h + 1]);
      o[q] = *reinterpret_cast<const uint32_t*>(&r);
    }
    reinterpret_cast<uint4*>(dst)[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

struct MtpPrep {
  const __nv_bfloat16* g;     // hidden rows: row of sequence b = b * rows_per_seq + (acc ? acc[b] : 0)
  int32_t rows_per_seq;
  const int32_t* acc;         // [B] or nullptr
  const int32_t* y;           // [B] tokens
  const __nv_bfloat16* emb;   // [V, H]
  int32_t V, H;
  const float* gamma_h;
  const float* gamma_e;
  __nv_bfloat16* u;           // [B, 2H]
  int32_t* drafts;            // [B, K] or nullptr: drafts[b, slot] = y[b]
  int32_t K, slot;
};

// One block per sequence: the block's input row u.
__global__ void __launch_bounds__(kMtpThreads) mtp_prep(const MtpPrep p) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float red[kMtpThreads / 32];
  const int b = blockIdx.x, H = p.H;
  int yb = p.y[b];
  if (p.drafts != nullptr && threadIdx.x == 0) p.drafts[(size_t)b * p.K + p.slot] = yb;
  if ((unsigned)yb >= (unsigned)p.V) {
    if (threadIdx.x == 0) record_error(kErrBounds, 311);
    yb = 0;
  }
  int row = b * p.rows_per_seq;
  if (p.acc != nullptr) {
    const int a = p.acc[b];
    if ((unsigned)a < (unsigned)p.rows_per_seq) row += a;
    else if (threadIdx.x == 0) record_error(kErrBounds, 312);
  }
  __nv_bfloat16* ub = p.u + (size_t)b * 2 * H;
  rmsnorm_row(p.g + (size_t)row * H, p.gamma_h, H, ub, red);
  rmsnorm_row(p.emb + (size_t)yb * H, p.gamma_e, H, ub + H, red);
}

// One block per row: dst = bf16(rmsnorm(src) * gamma).
__global__ void __launch_bounds__(kMtpThreads) mtp_rmsnorm(const __nv_bfloat16* __restrict__ src,
                                                           const float* __restrict__ gamma, int H,
                                                           __nv_bfloat16* __restrict__ dst) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float red[kMtpThreads / 32];
  rmsnorm_row(src + (size_t)blockIdx.x * H, gamma, H, dst + (size_t)blockIdx.x * H, red);
}

// g = bf16(z + o), n elements (a multiple of 8).
__global__ void __launch_bounds__(256) mtp_residual(const __nv_bfloat16* __restrict__ z,
                                                    const __nv_bfloat16* __restrict__ o, int n,
                                                    __nv_bfloat16* __restrict__ g) {
  griddep_launch_dependents();
  griddep_wait();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n / 8) return;
  const uint4 a = reinterpret_cast<const uint4*>(z)[c], b = reinterpret_cast<const uint4*>(o)[c];
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
  uint32_t r[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 s = __floats2bfloat162_rn(bf16_lo(wa[q]) + bf16_lo(wb[q]), bf16_hi(wa[q]) + bf16_hi(wb[q]));
    r[q] = *reinterpret_cast<const uint32_t*>(&s);
  }
  reinterpret_cast<uint4*>(g)[c] = make_uint4(r[0], r[1], r[2], r[3]);
}

// drafts[b, slot] = y[b].
__global__ void __launch_bounds__(128) mtp_collect(const int32_t* __restrict__ y, int B, int K, int slot,
                                                   int32_t* __restrict__ drafts) {
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) drafts[(size_t)b * K + slot] = y[b];
}

}  // namespace vg
