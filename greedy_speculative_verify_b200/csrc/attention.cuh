// Verifier attention over a KV cache: one layer of a verify step scores the
// K+1 new rows of every sequence (its last committed token and K drafts)
// against that sequence's cached positions. The pages give the decoder's
// position limit (32,768; jina-ocr-v1 model card, architecture paragraph) but
// not its attention; the reading computed here: 10 heads of 128, q/k/v from
// one projection [3H, H], RoFormer rotary positions (pair (2j, 2j+1) of a head
// turned by p * 10000^(-2j/128)), the new k/v written to the cache at
// positions L .. L+K, row i attending causally to positions 0 .. L+i with
// scores q.k / sqrt(128), out = x + W_o o.
//
// attn_rope_append: rotates q and k of the new rows, stores q, appends k and v.
// attn_chunk: flash-decoding partials — one CTA per (sequence, head, chunk of
//   kAttnChunk cache positions): the chunk's score max, exp-sum and
//   exp-weighted value sum for each new row.
// attn_merge: merges a (sequence, head, row)'s chunk partials into o.
// The projections run on the expert GEMM kernel (dense unit lists).
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kAttnHeads = 10, kAttnDim = 128;
constexpr int kAttnChunk = 256;   // cache positions per CTA
constexpr int kAttnMaxRows = 8;   // K + 1 <= 8 new rows per sequence
constexpr int kAttnThreads = 256;

struct AttnArgs {
  int32_t B, K1, L_max;          // K1 = K + 1 rows per sequence
  const int32_t* lens;           // [B] cached positions before this step
  const __nv_bfloat16* qkv;      // [B*K1, 3H]
  __nv_bfloat16* q;              // [B*K1, H] rotated queries
  __nv_bfloat16* cache;          // [B, 2, L_max, H]
  float* part;                   // [B, heads, n_chunks, K1, 2 + dim]: m, l, acc
  int32_t n_chunks;
  __nv_bfloat16* o;              // [B*K1, H]
};

__device__ __forceinline__ bool attn_len_ok(const AttnArgs& a, int b, int* L) {
  *L = a.lens[b];
  return *L >= 0 && *L + a.K1 <= a.L_max;
}

// One thread per (row, pair) of q and of k.
__global__ void __launch_bounds__(256) attn_rope_append(const AttnArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int H = kAttnHeads * kAttnDim, pairs = H / 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int R = a.B * a.K1;
  if (idx >= R * pairs) return;
  const int r = idx / pairs, pr = idx - r * pairs;
  const int b = r / a.K1, i = r - b * a.K1;
  int L;
  if (!attn_len_ok(a, b, &L)) {
    if (pr == 0 && i == 0) record_error(kErrBounds, 321);
    return;
  }
  const int j = pr % (kAttnDim / 2);  // pair index inside its head
  const double ang = (double)(L + i) * pow(10000.0, -2.0 * j / kAttnDim);
  double sn, cs;
  sincos(ang, &sn, &cs);
  const __nv_bfloat16* row = a.qkv + (size_t)r * 3 * H;
  auto turn = [&](const __nv_bfloat16* src, __nv_bfloat16* dst) {
    const float x0 = __bfloat162float(src[2 * pr]), x1 = __bfloat162float(src[2 * pr + 1]);
    const double y0 = (double)x0 * cs - (double)x1 * sn, y1 = (double)x0 * sn + (double)x1 * cs;
    dst[2 * pr] = __float2bfloat16_rn((float)y0);
    dst[2 * pr + 1] = __float2bfloat16_rn((float)y1);
  };
  turn(row, a.q + (size_t)r * H);
  __nv_bfloat16* kc = a.cache + ((size_t)b * 2 * a.L_max + (L + i)) * H;
  __nv_bfloat16* vc = a.cache + ((size_t)(b * 2 + 1) * a.L_max + (L + i)) * H;
  turn(row + H, kc);
  vc[2 * pr] = row[2 * H + 2 * pr];
  vc[2 * pr + 1] = row[2 * H + 2 * pr + 1];
}

// grid (B * heads, n_chunks); each thread scores one cache position against
// every new row, then each thread accumulates (row, dim) outputs.
__global__ void __launch_bounds__(kAttnThreads) attn_chunk(const AttnArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int H = kAttnHeads * kAttnDim;
  __shared__ float qs[kAttnMaxRows][kAttnDim];
  __shared__ float ps[kAttnMaxRows][kAttnChunk];
  __shared__ float red[kAttnThreads / 32];
  __shared__ float mx[kAttnMaxRows], sm[kAttnMaxRows];
  const int b = blockIdx.x / kAttnHeads, h = blockIdx.x - b * kAttnHeads, c = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int L;
  const bool ok = attn_len_ok(a, b, &L);
  const int visible = ok ? L + a.K1 : 0;  // positions any row of this step may see
  const int p0 = c * kAttnChunk, n = max(0, min(kAttnChunk, visible - p0));
  float* part = a.part + (((size_t)b * kAttnHeads + h) * a.n_chunks + c) * a.K1 * (2 + kAttnDim);
  if (n == 0) {  // nothing here: an empty partial
    for (int t = tid; t < a.K1; t += blockDim.x) {
      part[(size_t)t * (2 + kAttnDim)] = -INFINITY;
      part[(size_t)t * (2 + kAttnDim) + 1] = 0.0f;
    }
    for (int t = tid; t < a.K1 * kAttnDim; t += blockDim.x)
      part[(size_t)(t / kAttnDim) * (2 + kAttnDim) + 2 + t % kAttnDim] = 0.0f;
    return;
  }
  for (int t = tid; t < a.K1 * kAttnDim; t += blockDim.x) {
    const int r = t / kAttnDim, d = t - r * kAttnDim;
    qs[r][d] = __bfloat162float(a.q[((size_t)b * a.K1 + r) * H + h * kAttnDim + d]);
  }
  __syncthreads();
  const float scale = 1.0f / sqrtf((float)kAttnDim);
  // scores: thread = cache position p0 + tid
  if (tid < n) {
    const uint4* kp = reinterpret_cast<const uint4*>(a.cache + ((size_t)b * 2 * a.L_max + p0 + tid) * H + h * kAttnDim);
    float acc[kAttnMaxRows];
#pragma unroll
    for (int r = 0; r < kAttnMaxRows; ++r) acc[r] = 0.0f;
#pragma unroll 4
    for (int q8 = 0; q8 < kAttnDim / 8; ++q8) {
      const uint4 v = __ldg(kp + q8);
      const float kv[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                           bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
      for (int r = 0; r < kAttnMaxRows; ++r) {
        if (r < a.K1) {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[r] = __fmaf_rn(qs[r][8 * q8 + e], kv[e], acc[r]);
        }
      }
    }
    const int pos = p0 + tid;
    for (int r = 0; r < a.K1; ++r) ps[r][tid] = pos <= L + r ? acc[r] * scale : -INFINITY;  // causal
  }
  for (int r = 0; r < a.K1; ++r)
    if (tid >= n) ps[r][tid] = -INFINITY;
  __syncthreads();
  // per row: max and exp-sum over the chunk
  for (int r = 0; r < a.K1; ++r) {
    float m = ps[r][tid];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (tid == 0) {
      float mm = red[0];
      for (int w = 1; w < kAttnThreads / 32; ++w) mm = fmaxf(mm, red[w]);
      mx[r] = mm;
    }
    __syncthreads();
    const float e = ps[r][tid] == -INFINITY ? 0.0f : expf(ps[r][tid] - mx[r]);
    ps[r][tid] = e;
    float s = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    __syncthreads();
    if (lane == 0) red[warp] = s;
    __syncthreads();
    if (tid == 0) {
      float ss = 0.0f;
      for (int w = 0; w < kAttnThreads / 32; ++w) ss += red[w];
      sm[r] = ss;
    }
    __syncthreads();
  }
  // weighted values: thread = (dim, half of the rows)
  const int d = tid & (kAttnDim - 1), half = tid >> 7;
  float acc[kAttnMaxRows / 2];
#pragma unroll
  for (int j = 0; j < kAttnMaxRows / 2; ++j) acc[j] = 0.0f;
  const __nv_bfloat16* vp = a.cache + ((size_t)(b * 2 + 1) * a.L_max + p0) * H + h * kAttnDim + d;
  for (int t = 0; t < n; ++t) {
    const float v = __bfloat162float(vp[(size_t)t * H]);
#pragma unroll
    for (int j = 0; j < kAttnMaxRows / 2; ++j) {
      const int r = half + 2 * j;
      if (r < a.K1) acc[j] = __fmaf_rn(ps[r][t], v, acc[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < kAttnMaxRows / 2; ++j) {
    const int r = half + 2 * j;
    if (r < a.K1) part[(size_t)r * (2 + kAttnDim) + 2 + d] = acc[j];
  }
  if (tid < a.K1) {
    part[(size_t)tid * (2 + kAttnDim)] = mx[tid];
    part[(size_t)tid * (2 + kAttnDim) + 1] = sm[tid];
  }
}

// grid B * heads * K1, kAttnDim threads: o = sum_c acc_c e^(m_c - m) / sum_c l_c e^(m_c - m).
__global__ void __launch_bounds__(kAttnDim) attn_merge(const AttnArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int H = kAttnHeads * kAttnDim;
  const int r = blockIdx.x % a.K1, bh = blockIdx.x / a.K1, b = bh / kAttnHeads, h = bh - b * kAttnHeads;
  const int d = threadIdx.x;
  const float* part = a.part + ((size_t)b * kAttnHeads + h) * a.n_chunks * a.K1 * (2 + kAttnDim);
  int L;
  const int n_used = attn_len_ok(a, b, &L) ? cdiv(L + a.K1, kAttnChunk) : 0;
  float m = -INFINITY;
  for (int c = 0; c < n_used; ++c) m = fmaxf(m, part[((size_t)c * a.K1 + r) * (2 + kAttnDim)]);
  float l = 0.0f, acc = 0.0f;
  for (int c = 0; c < n_used; ++c) {
    const float* pc = part + ((size_t)c * a.K1 + r) * (2 + kAttnDim);
    if (pc[0] == -INFINITY) continue;
    const float w = expf(pc[0] - m);
    l = __fmaf_rn(pc[1], w, l);
    acc = __fmaf_rn(pc[2 + d], w, acc);
  }
  a.o[((size_t)b * a.K1 + r) * H + h * kAttnDim + d] = __float2bfloat16_rn(l > 0.0f ? acc / l : 0.0f);
}

}  // namespace vg
