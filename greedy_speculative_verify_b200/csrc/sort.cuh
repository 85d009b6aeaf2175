// Token-to-expert grouping: histogram, offsets and the stable permutation of
// the T*k assignments (assignment a = t*k + j has key idx[t, j]), plus the
// gather of each assignment's token row into permutation order so the expert
// GEMMs read contiguous rows.
//
// Stability comes from processing assignments in increasing id, 1024 at a time:
// inside a warp, __match_any_sync groups equal keys and the rank is the number
// of lower lanes with the same key; across warps, per-warp key counts in shared
// memory give the base. Nothing depends on the order of atomic operations.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kSortE = 64;
constexpr int kSortChunk = 1024;       // assignments per pass (one per thread)
constexpr int kSortSmallMax = 8192;    // decode path (layer-entry kernel) up to this many assignments

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Positions of the blockDim.x assignments a = base + threadIdx.x given the
// running start of every expert's segment `run` (shared). Returns -1 for a >= N.
// Advances `run` by this chunk's counts. Must be called by every thread of the
// block (at most 1024).
__device__ __forceinline__ int chunk_positions(const int32_t* __restrict__ keys, int base, int N, int* run,
                                               int (*wcnt)[kSortE]) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a = base + tid;
  int key = -1;
  if (a < N) {
    key = keys[a];
    if ((unsigned)key >= (unsigned)kSortE) {
      record_error(kErrBounds, 201);
      key = -1;
    }
  }
  for (int i = tid; i < 32 * kSortE; i += blockDim.x) wcnt[i / kSortE][i % kSortE] = 0;
  __syncthreads();
  const uint32_t m = __match_any_sync(0xffffffffu, key);
  const int rank = __popc(m & lanemask_lt());
  if (key >= 0 && lane == __ffs(m) - 1) wcnt[warp][key] = __popc(m);
  __syncthreads();
  int pos = -1;
  if (key >= 0) {
    pos = run[key] + rank;
    for (int w = 0; w < warp; ++w) pos += wcnt[w][key];
  }
  __syncthreads();
  if (tid < kSortE) {
    int s = 0;
    for (int w = 0; w < 32; ++w) s += wcnt[w][tid];
    run[tid] += s;
  }
  __syncthreads();
  return pos;
}

// Exclusive scan of 64 counts by one warp (2 per lane).
__device__ __forceinline__ void scan64_warp(const int* cnt, int* out_excl, int lane) {
  const int c0 = cnt[2 * lane], c1 = cnt[2 * lane + 1];
  int s = c0 + c1, inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  const int excl = inc - s;
  out_excl[2 * lane] = excl;
  out_excl[2 * lane + 1] = excl + c0;
}

// Copies token rows x[perm_pos -> token] into x_perm, rows [r0, r1) handled by
// this block with a grid-independent stride. Rows are H bf16 (H % 8 == 0).
__device__ __forceinline__ void gather_rows(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ xp,
                                            int H, int row, int token) {
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)token * H);
  uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)row * H);
  for (int c = threadIdx.x & 31; c < H / 8; c += 32) dst[c] = __ldg(src + c);
}

// Multi-kernel path, pass 1: per-chunk histograms [nchunks][64].
__global__ void __launch_bounds__(1024) expert_hist_chunks(const int32_t* __restrict__ keys, int N,
                                                           int32_t* __restrict__ chunk_cnt) {
  __shared__ int cnt[kSortE];
  if (threadIdx.x < kSortE) cnt[threadIdx.x] = 0;
  __syncthreads();
  const int a = blockIdx.x * kSortChunk + threadIdx.x;
  if (a < N) {
    const int key = keys[a];
    if ((unsigned)key < (unsigned)kSortE) atomicAdd(&cnt[key], 1);
  }
  __syncthreads();
  if (threadIdx.x < kSortE) chunk_cnt[blockIdx.x * kSortE + threadIdx.x] = cnt[threadIdx.x];
}

// Pass 2 (one block of 64 threads): offsets and each chunk's per-expert base.
__global__ void __launch_bounds__(1024) expert_scan_chunks(const int32_t* __restrict__ chunk_cnt, int nchunks, int N,
                                                           int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ chunk_base,
                                                           int32_t* __restrict__ sched, int sched_len) {
  // thread (slice sl, expert e) sums the counts of a contiguous range of
  // chunks, requested together; the slices' sums give each expert's total and
  // each range's starting point (integer sums: the order does not matter)
  constexpr int kSl = 1024 / kSortE;
  __shared__ int part[kSl][kSortE];
  __shared__ int tot[kSortE], off[kSortE];
  const int e = threadIdx.x % kSortE, sl = threadIdx.x / kSortE;
  for (int i = threadIdx.x; i < sched_len; i += blockDim.x) sched[i] = 0;  // expert GEMM tickets + readiness
  const int R = (nchunks + kSl - 1) / kSl, c0 = min(nchunks, sl * R), c1 = min(nchunks, c0 + R);
  int s = 0;
#pragma unroll 8
  for (int c = c0; c < c1; ++c) s += chunk_cnt[c * kSortE + e];
  part[sl][e] = s;
  __syncthreads();
  if (threadIdx.x < kSortE) {
    int t = 0;
    for (int j = 0; j < kSl; ++j) t += part[j][e];
    tot[e] = t;
  }
  __syncthreads();
  if (threadIdx.x < 32) scan64_warp(tot, off, threadIdx.x);
  __syncthreads();
  if (threadIdx.x < kSortE) offsets[e] = off[e];
  if (threadIdx.x == 0) offsets[kSortE] = N;
  int run = off[e];
  for (int j = 0; j < sl; ++j) run += part[j][e];
#pragma unroll 8
  for (int c = c0; c < c1; ++c) {
    chunk_base[c * kSortE + e] = run;
    run += chunk_cnt[c * kSortE + e];
  }
}

// Pass 3: stable positions inside each chunk, perm/inv, and the row gather.
__global__ void __launch_bounds__(1024) expert_scatter_chunks(const int32_t* __restrict__ keys, int N, int k,
                                                              const int32_t* __restrict__ chunk_base,
                                                              int32_t* __restrict__ perm,
                                                              int32_t* __restrict__ inv,
                                                              const __nv_bfloat16* __restrict__ x, int H,
                                                              __nv_bfloat16* __restrict__ x_perm) {
  __shared__ int run[kSortE];
  __shared__ int wcnt[32][kSortE];
  __shared__ int pos_s[kSortChunk];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid < kSortE) run[tid] = chunk_base[blockIdx.x * kSortE + tid];
  __syncthreads();
  const int base = blockIdx.x * kSortChunk;
  int pos = chunk_positions(keys, base, N, run, wcnt);
  const int a = base + tid;
  if (pos >= 0 && !VG_IN_BOUNDS(pos < N, 408)) pos = -1;
  pos_s[tid] = pos;
  if (pos >= 0) {
    perm[pos] = a;
    inv[a] = pos;
  }
  __syncthreads();
  if (H == 1280) {
    // two rows per warp at a time, every 16-byte load of both issued before the stores
    constexpr int kPer = 1280 / 8 / 32;  // 16-byte pieces per lane and row
    const int lane = tid & 31;
    for (int i = warp; i < kSortChunk; i += 64) {
      const int i1 = i + 32;
      const int p0 = pos_s[i], p1 = i1 < kSortChunk ? pos_s[i1] : -1;
      uint4 v0[kPer], v1[kPer];
      const uint4* s0 = reinterpret_cast<const uint4*>(x + (size_t)((base + i) / k) * H);
      const uint4* s1 = reinterpret_cast<const uint4*>(x + (size_t)((base + i1) / k) * H);
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        if (p0 >= 0) v0[j] = __ldg(s0 + lane + 32 * j);
        if (p1 >= 0) v1[j] = __ldg(s1 + lane + 32 * j);
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        if (p0 >= 0) reinterpret_cast<uint4*>(x_perm + (size_t)p0 * H)[lane + 32 * j] = v0[j];
        if (p1 >= 0) reinterpret_cast<uint4*>(x_perm + (size_t)p1 * H)[lane + 32 * j] = v1[j];
      }
    }
  } else {
    for (int i = warp; i < kSortChunk; i += 32) {
      const int p = pos_s[i];
      if (p >= 0) gather_rows(x, x_perm, H, p, (base + i) / k);
    }
  }
}

}  // namespace vg
