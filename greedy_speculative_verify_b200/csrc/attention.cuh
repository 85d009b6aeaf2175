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
//   exp-weighted value sum for each new row; every key and value of the chunk
//   is read once for all K+1 rows.
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

__device__ __forceinline__ void attn_unpack8(const uint4 u, float (&f)[8]) {
  f[0] = bf16_lo(u.x), f[1] = bf16_hi(u.x), f[2] = bf16_lo(u.y), f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z), f[5] = bf16_hi(u.z), f[6] = bf16_lo(u.w), f[7] = bf16_hi(u.w);
}

// Sum of v[0 .. N) over the 2^NS lanes lane ^ m, m built from the bits O, O/2,
// ..., O >> (NS - 1). While more than one value is live, a step keeps half of
// them (the upper half on lanes whose bit O is set) and adds the partner lane's
// copy of that half, so N values cost N - 1 shuffles instead of N * NS; once
// one value is left the remaining steps are plain xor sums. On return
// v[0 .. max(1, N >> NS)) hold the sums of the flat indices base, base + 1, ...,
// and lanes that differ only in the bits of dup hold the same values.
template <int C, int O, int NS, int N>
__device__ __forceinline__ void xor_reduce(float (&v)[C], int lane, int& base, int& dup) {
  if constexpr (NS > 0) {
    if constexpr (N >= 2) {
      constexpr int half = N / 2;
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = up ? v[i] : v[i + half];
        const float keep = up ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      if (up) base += half;
      xor_reduce<C, O / 2, NS - 1, half>(v, lane, base, dup);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      dup |= O;
      xor_reduce<C, O / 2, NS - 1, 1>(v, lane, base, dup);
    }
  }
}

// grid (B * heads, n_chunks), K1 = K + 1 new rows per sequence. Three phases
// over the chunk's positions:
//   scores:  a half-warp reads one key (16 lanes x 8 dimensions, 256 contiguous
//            bytes), every lane holding its 8 dimensions of all K1 queries in
//            registers; the K1 dot products are summed over the half-warp by
//            xor_reduce and written as pt[position][row];
//   softmax: warp r takes row r: chunk max, exp, exp-sum (-> m, l);
//   values:  warp w owns dimensions 16w .. 16w+15, its lanes split the
//            positions 16 ways (16-byte value loads, the K1 weights of a
//            position read as one or two 16-byte shared loads); the 16 partial
//            sums are combined by xor_reduce at the end.
template <int K1>
__global__ void __launch_bounds__(kAttnThreads, 2) attn_chunk(const AttnArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int H = kAttnHeads * kAttnDim;
  constexpr int KP = K1 <= 1 ? 1 : K1 <= 2 ? 2 : K1 <= 4 ? 4 : 8;  // rows padded to a power of two
  constexpr int PW = 2 + kAttnDim;                                   // floats per row of a partial
  static_assert(K1 >= 1 && K1 <= kAttnMaxRows && kAttnMaxRows <= 8 && kAttnThreads == 256 && kAttnDim == 128 &&
                    kAttnChunk == 256,
                "the lane maps below assume 8 warps, 128 dimensions, 256 positions, at most 8 rows");
  __shared__ __align__(16) float pt[kAttnChunk][8];  // scores, then exp-weights: [position][row]
  const int b = blockIdx.x / kAttnHeads, h = blockIdx.x - b * kAttnHeads, c = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int L;
  const bool ok = attn_len_ok(a, b, &L);
  const int visible = ok ? L + K1 : 0;  // positions any row of this step may see
  const int p0 = c * kAttnChunk, n = max(0, min(kAttnChunk, visible - p0));
  float* part = a.part + (((size_t)b * kAttnHeads + h) * a.n_chunks + c) * K1 * PW;
  if (n == 0) {  // nothing here: an empty partial
    for (int t = tid; t < K1; t += blockDim.x) {
      part[(size_t)t * PW] = -INFINITY;
      part[(size_t)t * PW + 1] = 0.0f;
    }
    for (int t = tid; t < K1 * kAttnDim; t += blockDim.x) part[(size_t)(t / kAttnDim) * PW + 2 + t % kAttnDim] = 0.0f;
    return;
  }
  const float scale = 1.0f / sqrtf((float)kAttnDim);
  {  // scores
    const int dg = lane & 15, sub = lane >> 4;
    float q[KP][8];
#pragma unroll
    for (int r = 0; r < KP; ++r) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (r < K1) u = *reinterpret_cast<const uint4*>(a.q + ((size_t)b * K1 + r) * H + h * kAttnDim + 8 * dg);
      attn_unpack8(u, q[r]);
    }
    const __nv_bfloat16* kb = a.cache + ((size_t)b * 2 * a.L_max + p0) * H + h * kAttnDim + 8 * dg;
#pragma unroll 8
    for (int j = 0; j < kAttnChunk / 16; ++j) {
      const int t = warp * (kAttnChunk / 8) + 2 * j + sub;
      uint4 u = make_uint4(0, 0, 0, 0);
      if (t < n) u = __ldg(reinterpret_cast<const uint4*>(kb + (size_t)t * H));
      float k8[8];
      attn_unpack8(u, k8);
      float sc[KP];
#pragma unroll
      for (int r = 0; r < KP; ++r) {
        float d = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) d = __fmaf_rn(q[r][e], k8[e], d);
        sc[r] = d;
      }
      int r = 0, dup = 0;
      xor_reduce<KP, 8, 4, KP>(sc, lane, r, dup);
      if ((lane & dup) == 0 && r < K1 && t < n) pt[t][r] = p0 + t <= L + r ? sc[0] * scale : -INFINITY;  // causal
    }
  }
  __syncthreads();
  if (warp < K1) {  // softmax statistics of row `warp` over the chunk
    const int r = warp;
    float v[kAttnChunk / 32];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kAttnChunk / 32; ++i) {
      const int t = lane + 32 * i;
      v[i] = t < n ? pt[t][r] : -INFINITY;
      m = fmaxf(m, v[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.0f;
#pragma unroll
    for (int i = 0; i < kAttnChunk / 32; ++i) {
      const int t = lane + 32 * i;
      const float e = v[i] == -INFINITY ? 0.0f : expf(v[i] - m);
      if (t < n) pt[t][r] = e;
      l += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      part[(size_t)r * PW] = m;
      part[(size_t)r * PW + 1] = l;
    }
  }
  __syncthreads();
  {  // exp-weighted values
    const int dq = lane & 1, pg = lane >> 1;
    const int d0 = 16 * warp + 8 * dq;
    float acc[8 * KP];
#pragma unroll
    for (int i = 0; i < 8 * KP; ++i) acc[i] = 0.0f;
    const __nv_bfloat16* vb = a.cache + ((size_t)(b * 2 + 1) * a.L_max + p0) * H + h * kAttnDim + d0;
#pragma unroll 8
    for (int i = 0; i < kAttnChunk / 16; ++i) {
      const int t = pg + 16 * i;
      uint4 u = make_uint4(0, 0, 0, 0);
      float4 pa = make_float4(0.0f, 0.0f, 0.0f, 0.0f), pb = pa;
      if (t < n) {
        u = __ldg(reinterpret_cast<const uint4*>(vb + (size_t)t * H));
        pa = *reinterpret_cast<const float4*>(&pt[t][0]);
        if constexpr (KP > 4) pb = *reinterpret_cast<const float4*>(&pt[t][4]);
      }
      float v8[8];
      attn_unpack8(u, v8);
      const float p[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int r = 0; r < KP; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r * 8 + e] = __fmaf_rn(p[r], v8[e], acc[r * 8 + e]);
    }
    int base = 0, dup = 0;
    xor_reduce<8 * KP, 16, 4, 8 * KP>(acc, lane, base, dup);
    constexpr int live = (8 * KP) >> 4 > 0 ? (8 * KP) >> 4 : 1;
    if ((lane & dup) == 0) {
#pragma unroll
      for (int i = 0; i < live; ++i) {
        const int f = base + i, r = f >> 3, e = f & 7;
        if (r < K1) part[(size_t)r * PW + 2 + d0 + e] = acc[i];
      }
    }
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
