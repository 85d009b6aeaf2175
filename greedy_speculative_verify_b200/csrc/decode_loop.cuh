// Multi-step speculative decoding on a synthetic Markov decoder, kept on the
// device: the token-side bookkeeping between verify steps.
//
// The decoder maps its last token to the next one: embedding row -> MoE layer
// stack -> LM head -> argmax. A speculative step verifies K drafted tokens per
// sequence in one pass over K+1 rows and commits the longest agreeing prefix
// plus the verifier's own token ("jina-ocr-v1: Schnellere Dokumentenanalyse auf
// kostengünstigen GPUs", "Modell und Training"); committing that way yields
// exactly the tokens plain greedy decoding yields, which is what a loop built on
// these kernels lets one check on the GPU. K = 0 is plain greedy decoding.
//
// embed_rows: out[i] = emb[tokens[i]] (bf16 rows); one warp per row.
// spec_rows:  the next verify rows of every sequence: its last committed token,
//   then K drafts. Draft i stands for the decoder's own token at committed
//   position pos + i: with probability p it is that token, taken from a
//   reference continuation (a plain greedy run), else a uniform token. The
//   draws come from SplitMix64 (Steele, Lea and Flood, "Fast splittable
//   pseudorandom number generators", OOPSLA 2014) on a counter made of the
//   seed, the step, the sequence and the draft index, so a step is repeatable.
// spec_commit: appends the step's committed tokens (accepted drafts + bonus)
//   and advances the sequence; then the step counter.
#pragma once
#include "common.cuh"

namespace vg {

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void __launch_bounds__(256) embed_rows(const int32_t* __restrict__ tokens, int n,
                                                  const __nv_bfloat16* __restrict__ emb, int V, int H,
                                                  __nv_bfloat16* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= n) return;
  const int t = tokens[row];
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * H);
  if ((unsigned)t >= (unsigned)V) {
    if (lane == 0) record_error(kErrBounds, 301);
    for (int c = lane; c < H / 8; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(emb + (size_t)t * H);
  for (int c = lane; c < H / 8; c += 32) dst[c] = __ldg(src + c);
}

struct SpecState {
  int32_t B, K, V;
  int32_t* last;        // [B] last committed token (the start token before any step)
  int32_t* pos;         // [B] tokens committed so far
  int32_t* committed;   // [B, cap]
  int32_t cap;
  const int32_t* ref;   // [B, ref_len] reference continuation: token at committed position j
  int32_t ref_len;
  float p;
  uint64_t seed;
  int32_t* step;        // [1] steps taken (device counter)
  int32_t* tokens;      // [B, K+1] next verify rows
  int32_t* drafts;      // [B, K]
};

// One thread per sequence.
__global__ void __launch_bounds__(128) spec_rows(const SpecState s) {
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= s.B) return;
  const int step = *s.step, p0 = s.pos[b];
  const int K1 = s.K + 1;
  s.tokens[(size_t)b * K1] = s.last[b];
  for (int i = 1; i <= s.K; ++i) {
    const uint64_t ctr = s.seed ^ ((uint64_t)step << 40) ^ ((uint64_t)b << 16) ^ (uint64_t)i;
    const uint64_t r1 = splitmix64(ctr), r2 = splitmix64(ctr ^ 0x5555555555555555ull);
    const float u = (float)(r1 >> 40) * (1.0f / 16777216.0f);  // 24 random bits in [0, 1)
    const int j = p0 + i - 1;
    int d = (int)(r2 % (uint64_t)s.V);
    if (u < s.p && j < s.ref_len) d = s.ref[(size_t)b * s.ref_len + j];
    s.tokens[(size_t)b * K1 + i] = d;
    s.drafts[(size_t)b * s.K + i - 1] = d;
  }
}

// Rows from drafts already in s.drafts (written by another drafter).
__global__ void __launch_bounds__(128) spec_rows_given(const SpecState s) {
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= s.B) return;
  const int K1 = s.K + 1;
  s.tokens[(size_t)b * K1] = s.last[b];
  for (int i = 1; i <= s.K; ++i) s.tokens[(size_t)b * K1 + i] = s.drafts[(size_t)b * s.K + i - 1];
}

__global__ void __launch_bounds__(128) spec_commit(const SpecState s, const int32_t* __restrict__ accepted,
                                                   const int32_t* __restrict__ out_tokens) {
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < s.B) {
    int a = accepted[b];
    if (a < 0 || a > s.K) {
      record_error(kErrBounds, 302);
      a = 0;
    }
    const int p0 = s.pos[b];
    for (int j = 0; j <= a; ++j)
      if (p0 + j < s.cap) s.committed[(size_t)b * s.cap + p0 + j] = out_tokens[(size_t)b * (s.K + 1) + j];
    s.pos[b] = p0 + a + 1;
    s.last[b] = out_tokens[(size_t)b * (s.K + 1) + a];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *s.step += 1;
}

}  // namespace vg
