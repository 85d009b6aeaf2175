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
//   is read once for all K+1 rows, both products on the tensor cores.
// attn_merge: merges a (sequence, head, row)'s chunk partials into o.
// The q/k/v and output projections are fp32 partial sums over 256-wide slices
// of the reduction (attn_proj_tc, proj_tc.cuh), summed in a fixed order by
// their readers (attn_rope_append, attn_residual), which round the sum to bf16.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kAttnHeads = 10, kAttnDim = 128;
constexpr int kAttnChunk = 256;   // cache positions per CTA
constexpr int kAttnMaxRows = 8;   // K + 1 <= 8 new rows per sequence
constexpr int kAttnThreads = 256; // 8 warps of 32 positions


struct AttnArgs {
  int32_t B, K1, L_max;          // K1 = K + 1 rows per sequence
  const int32_t* lens;           // [B] cached positions before this step
  const float* qkv_part;         // [splits, B*K1, 3H] fp32 partial sums of x W_qkv^T
  int32_t splits;
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

// D += A B on the tensor cores, one m16n8k16 tile (bf16 operands, fp32
// accumulators), g = lane / 4, t = lane % 4: a0 = A[g][2t, 2t+1],
// a1 = A[g+8][2t, 2t+1], a2 = A[g][2t+8, 2t+9], a3 = A[g+8][2t+8, 2t+9],
// b0 = B[2t, 2t+1][g], b1 = B[2t+8, 2t+9][g], d = D[g][2t, 2t+1], D[g+8][2t, 2t+1].
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 of the fixed-order sum of `splits` partials p[0], p[stride], ...
__device__ __forceinline__ float proj_sum_bf16(const float* p, int splits, size_t stride) {
  float v = 0.0f;
  for (int s = 0; s < splits; ++s) v += p[(size_t)s * stride];
  return __bfloat162float(__float2bfloat16_rn(v));
}

// out = bf16(x + bf16(sum_s part[s])), four elements per thread (n a multiple of 4).
__global__ void __launch_bounds__(256) attn_residual(const __nv_bfloat16* __restrict__ x,
                                                     const float* __restrict__ part, int splits, int n,
                                                     __nv_bfloat16* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n / 4) return;
  float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int s = 0; s < splits; ++s) {
    const float4 p = reinterpret_cast<const float4*>(part + (size_t)s * n)[c];
    v.x += p.x, v.y += p.y, v.z += p.z, v.w += p.w;
  }
  const uint2 xv = reinterpret_cast<const uint2*>(x)[c];
  const float y0 = __bfloat162float(__float2bfloat16_rn(v.x)), y1 = __bfloat162float(__float2bfloat16_rn(v.y));
  const float y2 = __bfloat162float(__float2bfloat16_rn(v.z)), y3 = __bfloat162float(__float2bfloat16_rn(v.w));
  const __nv_bfloat162 lo = __floats2bfloat162_rn(bf16_lo(xv.x) + y0, bf16_hi(xv.x) + y1);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(bf16_lo(xv.y) + y2, bf16_hi(xv.y) + y3);
  reinterpret_cast<uint2*>(out)[c] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
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
  const size_t stride = (size_t)R * 3 * H;  // one partial of the projection
  const float* row = a.qkv_part + (size_t)r * 3 * H;
  // q, k, v = bf16 of the projection (the sum of its partials)
  auto val = [&](int col) { return proj_sum_bf16(row + col, a.splits, stride); };
  auto turn = [&](int col, __nv_bfloat16* dst) {
    const float x0 = val(col + 2 * pr), x1 = val(col + 2 * pr + 1);
    const double y0 = (double)x0 * cs - (double)x1 * sn, y1 = (double)x0 * sn + (double)x1 * cs;
    dst[2 * pr] = __float2bfloat16_rn((float)y0);
    dst[2 * pr + 1] = __float2bfloat16_rn((float)y1);
  };
  turn(0, a.q + (size_t)r * H);
  __nv_bfloat16* kc = a.cache + ((size_t)b * 2 * a.L_max + (L + i)) * H;
  __nv_bfloat16* vc = a.cache + ((size_t)(b * 2 + 1) * a.L_max + (L + i)) * H;
  turn(H, kc);
  vc[2 * pr] = __float2bfloat16_rn(val(2 * H + 2 * pr));
  vc[2 * pr + 1] = __float2bfloat16_rn(val(2 * H + 2 * pr + 1));
}

// mma_16816 with A's rows 8..15 zero (the K+1 <= 8 new rows in a 16-row tile).
__device__ __forceinline__ void mma_16816_top(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  mma_16816(d, a0, 0u, a2, 0u, b0, b1);
}

// Transpose of an 8 x 8 bf16 tile held one 32-bit pair per lane (lane (g, t)
// holds row g, columns 2t, 2t+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

// grid (B * heads, n_chunks), 256 threads, two CTAs per SM; warp w takes
// positions 32w .. 32w+31 of the chunk, lane = (g, t) = (lane / 4, lane % 4),
// the K+1 <= 8 new rows as rows 0..7 of 16-row tensor-core tiles (rows 8..15
// zero).
//   scores: S = Q K^T over 8 positions per tile; a lane loads 16 contiguous
//     bytes of one key from global memory (dimensions 32s + 8t .. +7, s =
//     0..3), giving the B operands of two k-steps; the queries are loaded with
//     the same dimension order, so the contraction is unchanged;
//   softmax over the warp's 32 positions, per row: max and the exp-weights,
//     rounded to bf16 pairs that are already the A operand of the next product
//     (the exp-sum is taken over the rounded weights);
//   values: O += P V, 16 positions per k-step; a lane loads 16 contiguous bytes
//     of a value row and movmatrix turns them into B operands, so lane (g, t)
//     ends with dimensions 32s + 8t .. +7 of row g;
//   the 8 warps' (max, exp-sum, values) are merged in shared memory into the
//     chunk's partial.
// Positions past the visible ones read as zero keys and values. (Staging the
// keys and values through shared memory with TMA measured slower for this
// access pattern, a 256-byte piece of every 2,560-byte cache row, than these
// 16-byte loads from all 256 threads; so did merging the partials in the last
// CTA of each (sequence, head), whose fence and counter lengthen every CTA.)
__global__ void __launch_bounds__(kAttnThreads, 2) attn_chunk(const AttnArgs a) {
  constexpr int H = kAttnHeads * kAttnDim;
  constexpr int PW = 2 + kAttnDim;  // floats per row of a partial
  constexpr int OW = kAttnDim + 4;  // padded row of the per-warp values
  constexpr int NW = kAttnThreads / 32;
  static_assert(kAttnMaxRows <= 8 && NW * 32 == kAttnChunk && kAttnDim == 128,
                "the lane maps below assume warps of 32 positions, 128 dimensions, at most 8 rows");
  __shared__ float wm[NW][8], wl[NW][8];            // per warp and row: max, exp-sum
  __shared__ __align__(16) float wo[NW][8][OW];     // per warp and row: exp-weighted values
  const int b = blockIdx.x / kAttnHeads, h = blockIdx.x - b * kAttnHeads, c = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int K1 = a.K1;
  griddep_launch_dependents();
  griddep_wait();  // the rotated queries and the new keys and values come from the previous kernel
  int L;
  const bool ok = attn_len_ok(a, b, &L);
  const int visible = ok ? L + K1 : 0;  // positions any row of this step may see
  const int p0 = c * kAttnChunk, n = max(0, min(kAttnChunk, visible - p0));
  float* part = a.part + (((size_t)b * kAttnHeads + h) * a.n_chunks + c) * K1 * PW;
  if (n > 0) {
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    const int wp = 32 * warp;  // the warp's first position in the chunk
    // ---- scores
    uint4 qf[4];
#pragma unroll
    for (int s = 0; s < 4; ++s)
      qf[s] = g < K1 ? *reinterpret_cast<const uint4*>(a.q + ((size_t)b * K1 + g) * H + h * kAttnDim + 32 * s + 8 * t)
                     : zero4;
    const __nv_bfloat16* kb = a.cache + ((size_t)b * 2 * a.L_max + p0 + wp) * H + h * kAttnDim + 8 * t;
    float sc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int pos = 8 * j + g;  // the key this lane loads
      uint4 kf[4];
#pragma unroll
      for (int s = 0; s < 4; ++s)
        kf[s] = wp + pos < n ? __ldg(reinterpret_cast<const uint4*>(kb + (size_t)pos * H + 32 * s)) : zero4;
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[j][e] = 0.0f;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        mma_16816_top(sc[j], qf[s].x, qf[s].y, kf[s].x, kf[s].y);
        mma_16816_top(sc[j], qf[s].z, qf[s].w, kf[s].z, kf[s].w);
      }
    }
    // ---- softmax of row g over the warp's positions (lanes 4g .. 4g+3 share the row)
    const float scale = 1.0f / sqrtf((float)kAttnDim);
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = wp + 8 * j + 2 * t + e;
        const bool seen = g < K1 && pos < n && p0 + pos <= L + g;  // causal
        sc[j][e] = seen ? sc[j][e] * scale : -INFINITY;
        m = fmaxf(m, sc[j][e]);
      }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    uint32_t pf[4];  // exp-weights of positions 8j + 2t, 8j + 2t + 1 as bf16 pairs
    float l = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float e0 = sc[j][0] == -INFINITY ? 0.0f : expf(sc[j][0] - m);
      const float e1 = sc[j][1] == -INFINITY ? 0.0f : expf(sc[j][1] - m);
      const __nv_bfloat162 pp = __floats2bfloat162_rn(e0, e1);
      pf[j] = *reinterpret_cast<const uint32_t*>(&pp);
      l += __low2float(pp) + __high2float(pp);
    }
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    // ---- values: O = P V over the warp's positions, two k-steps of 16
    float o[4][4][4];  // [dimension block s][tile j][accumulator]: row g, dimensions 32s + 8t + 2j + {0, 1}
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[s][j][e] = 0.0f;
    const __nv_bfloat16* vb = a.cache + ((size_t)(b * 2 + 1) * a.L_max + p0 + wp) * H + h * kAttnDim + 8 * t;
#pragma unroll
    for (int kp = 0; kp < 2; ++kp) {
      const int lo = 16 * kp + g, hi = lo + 8;  // the value rows this lane reads
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint4 vl = wp + lo < n ? __ldg(reinterpret_cast<const uint4*>(vb + (size_t)lo * H + 32 * s)) : zero4;
        const uint4 vh = wp + hi < n ? __ldg(reinterpret_cast<const uint4*>(vb + (size_t)hi * H + 32 * s)) : zero4;
        const uint32_t rl[4] = {vl.x, vl.y, vl.z, vl.w}, rh[4] = {vh.x, vh.y, vh.z, vh.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_16816_top(o[s][j], pf[2 * kp], pf[2 * kp + 1], movmatrix_trans(rl[j]), movmatrix_trans(rh[j]));
      }
    }
    // ---- merge the warps into the chunk's partial
    if (t == 0) {
      wm[warp][g] = m;
      wl[warp][g] = l;
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      float* dst = &wo[warp][g][32 * s + 8 * t];
      *reinterpret_cast<float4*>(dst) = make_float4(o[s][0][0], o[s][0][1], o[s][1][0], o[s][1][1]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(o[s][2][0], o[s][2][1], o[s][3][0], o[s][3][1]);
    }
    __syncthreads();
    for (int i = tid; i < K1 * (kAttnDim / 4); i += kAttnThreads) {
      const int r = i / (kAttnDim / 4), d4 = 4 * (i % (kAttnDim / 4));
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) mm = fmaxf(mm, wm[w][r]);
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      float ls = 0.0f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        if (wm[w][r] == -INFINITY) continue;  // no visible position in that warp's share
        const float f = expf(wm[w][r] - mm);
        ls = __fmaf_rn(wl[w][r], f, ls);
        const float4 v = *reinterpret_cast<const float4*>(&wo[w][r][d4]);
        acc.x = __fmaf_rn(v.x, f, acc.x);
        acc.y = __fmaf_rn(v.y, f, acc.y);
        acc.z = __fmaf_rn(v.z, f, acc.z);
        acc.w = __fmaf_rn(v.w, f, acc.w);
      }
      float* pr = part + (size_t)r * PW;
      pr[2 + d4] = acc.x;
      pr[3 + d4] = acc.y;
      pr[4 + d4] = acc.z;
      pr[5 + d4] = acc.w;
      if (d4 == 0) {
        pr[0] = mm;
        pr[1] = ls;
      }
    }
  } else {  // nothing visible here: an empty partial
    for (int i = tid; i < K1; i += blockDim.x) {
      part[(size_t)i * PW] = -INFINITY;
      part[(size_t)i * PW + 1] = 0.0f;
    }
    for (int i = tid; i < K1 * kAttnDim; i += blockDim.x) part[(size_t)(i / kAttnDim) * PW + 2 + i % kAttnDim] = 0.0f;
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
