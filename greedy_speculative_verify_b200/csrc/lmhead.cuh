// Greedy-verify epilogue: LM-head logits fused with the argmax, then the
// longest-prefix accept with the bonus token.
//
// The verifier checks each drafted token greedily and commits the longest
// prefix on which draft and verifier agree plus one token of its own
// ("jina-ocr-v1: Schnellere Dokumentenanalyse auf kostengünstigen GPUs",
// "Modell und Training"; the bonus token counted in tau: same page,
// "Spekulatives Decoding auf einer L4"). Vocabulary 129,280 (jina-ocr-v1 model
// card, architecture paragraph).
//
// lmhead_argmax: tcgen05 GEMM with the verify rows as M (128 per tile) and a
// 176-row vocabulary slab as N; the fp32 logits never leave tensor memory. The
// epilogue thread that owns row r scans its 176 columns in increasing vocabulary
// order and keeps the best (value, index) as one 64-bit key: the order-
// preserving image of the fp32 value in the high word and (2^32-1-v) in the low
// word, so that the larger key is the larger logit and, among equal logits,
// the lower index. A work unit is a group of consecutive vocabulary tiles for
// one 128-row block; the key is carried across the group's tiles and one key
// per (group, row) goes to the workspace.
//
// argmax_accept: reduces the keys of a row (max), writes argmax, and for each
// sequence counts the leading drafts equal to the argmax of the preceding
// position, then writes the committed tokens.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kLmM = 128;    // verify rows per tile
constexpr int kLmN = 176;    // vocabulary rows per tile (129,280 = 734.5 tiles: about 5 waves on 148 SMs)
constexpr int kLmStages = 5;
constexpr int kLmABytes = kLmM * kBK * 2;    // 16 KB
constexpr int kLmBBytes = kLmN * kBK * 2;    // 22 KB
constexpr int kLmStageBytes = kLmABytes + kLmBBytes;
constexpr int kLmAccCols = 256;              // column stride of the two accumulator buffers
constexpr int kLmTmemCols = 512;
constexpr int kLmSmemBytes = kLmStages * kLmStageBytes + 2048 + 1024;
constexpr int kLmGroupTiles = 5;             // 735 tiles -> 147 groups: one per SM at 128 rows

__device__ __forceinline__ uint64_t argmax_key(float z, uint32_t v) {
  uint32_t u = __float_as_uint(z);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;  // -0 and +0 are the same logit
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - v);
}

__global__ void __launch_bounds__(192, 1)
    lmhead_argmax(const __grid_constant__ CUtensorMap mapH, const __grid_constant__ CUtensorMap mapLM, int R,
                  int V, int k_chunks, int n_mblk, int n_vblk, int group_tiles, int n_groups, int a_box_rows,
                  int b_box_rows, uint64_t* __restrict__ part) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* aux = smem + kLmStages * kLmStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux);
  uint64_t* empty = full + kLmStages;
  uint64_t* tfull = empty + kLmStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kLmStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&mapH);
    prefetch_tmap(&mapLM);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kLmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the hidden states come from the previous kernel
  const uint32_t tmem_base = *tmem_slot;
  const int total = n_groups * n_mblk;  // unit = (vocabulary group, row block), row block fastest
  const uint64_t limit = g_wait_timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_h = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      const uint32_t bytes = (a_box_rows + b_box_rows) * kBK * 2;
      for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
        const int g = u / n_mblk, mb = u - g * n_mblk;
        const int vb1 = min(n_vblk, (g + 1) * group_tiles);
        for (int vb = g * group_tiles; vb < vb1 && !*abort_flag; ++vb) {
          for (int kc = 0; kc < k_chunks; ++kc) {
            if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
              record_error(kErrTimeout, 121);
              *abort_flag = 1;
              break;
            }
            uint8_t* st = tiles + stage * kLmStageBytes;
            mbar_arrive_expect_tx(&full[stage], bytes);
            tma_load_2d_hint(st, &mapH, &full[stage], kc * kBK, mb * kLmM, pol_h);
            tma_load_2d_hint(st + kLmABytes, &mapLM, &full[stage], kc * kBK, vb * kLmN, pol_w);
            issued |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
            if (++stage == kLmStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      }
      for (int s = 0; s < kLmStages; ++s)
        if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kLmM, kLmN);
      int stage = 0;
      uint32_t phase = 0;
      int lt = 0;  // local tile counter: selects the accumulator buffer
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        const int g = u / n_mblk;
        const int vb1 = min(n_vblk, (g + 1) * group_tiles);
        for (int vb = g * group_tiles; vb < vb1 && ok; ++vb, ++lt) {
          if (*abort_flag) {
            ok = false;
            break;
          }
          const int ab = lt & 1;
          const uint32_t ap = (lt >> 1) & 1;
          if (!mbar_wait(&tempty[ab], ap ^ 1, limit)) {
            record_error(kErrTimeout, 122);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + ab * kLmAccCols;
          for (int kc = 0; kc < k_chunks; ++kc) {
            if (!mbar_wait(&full[stage], phase, limit)) {
              record_error(kErrTimeout, 123);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(tiles + stage * kLmStageBytes);
            const uint64_t a = sw128_kmajor_desc(st);
            const uint64_t b = sw128_kmajor_desc(st + kLmABytes);
#pragma unroll
            for (int k16 = 0; k16 < kBK / 16; ++k16)
              umma_bf16(d, a + 2 * k16, b + 2 * k16, idesc, (kc | k16) != 0);
            umma_commit(&empty[stage]);
            if (++stage == kLmStages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (ok) umma_commit(&tfull[ab]);
        }
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, limit);
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int lt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const int g = u / n_mblk, mb = u - g * n_mblk;
      const int vb1 = min(n_vblk, (g + 1) * group_tiles);
      uint64_t best = 0;  // running (value, index) key of this row over the group's tiles
      for (int vb = g * group_tiles; vb < vb1; ++vb, ++lt) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        const int ab = lt & 1;
        const uint32_t ap = (lt >> 1) & 1;
        if (!mbar_wait(&tfull[ab], ap, limit)) {
          record_error(kErrTimeout, 124);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + ab * kLmAccCols;
        const int v0 = vb * kLmN;
#pragma unroll 1
        for (int c0 = 0; c0 < kLmN; c0 += 16) {
          uint32_t z[16];
          tmem_ld16(t0 + c0, z);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int v = v0 + c0 + j;
            if (v < V) {
              const uint64_t key = argmax_key(__uint_as_float(z[j]), (uint32_t)v);
              best = key > best ? key : best;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[ab]);
      }
      const int r = mb * kLmM + row;
      if (ok && r < R) part[(size_t)g * R + r] = best;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kLmTmemCols);
  }
}

// One block handles whole sequences: spb = max(1, 32 / (K+1)) of them; its 32
// warps reduce the rows' keys, then one thread per sequence accepts.
__global__ void __launch_bounds__(1024) argmax_accept(const uint64_t* __restrict__ part, int n_groups, int R, int B,
                                                      int K, const int32_t* __restrict__ drafts,
                                                      int32_t* __restrict__ argmax, int32_t* __restrict__ accepted,
                                                      int32_t* __restrict__ out_tokens) {
  __shared__ int32_t arg_s[256];
  griddep_launch_dependents();
  griddep_wait();
  const int spb = max(1, 32 / (K + 1));
  const int seq0 = blockIdx.x * spb;
  const int nseq = min(spb, B - seq0);
  const int row0 = seq0 * (K + 1), nrows = nseq * (K + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rr = warp; rr < nrows; rr += 32) {
    const int r = row0 + rr;
    uint64_t best = 0;
    for (int g = lane; g < n_groups; g += 32) {
      const uint64_t k2 = part[(size_t)g * R + r];
      best = k2 > best ? k2 : best;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    if (lane == 0) {
      const int32_t a = (int32_t)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
      arg_s[rr] = a;
      argmax[r] = a;
    }
  }
  __syncthreads();
  if ((int)threadIdx.x < nseq) {
    const int b = seq0 + threadIdx.x;
    const int32_t* arg = arg_s + threadIdx.x * (K + 1);
    const int32_t* d = drafts + (size_t)b * K;
    int a = 0;
    while (a < K && d[a] == arg[a]) ++a;
    accepted[b] = a;
    int32_t* o = out_tokens + (size_t)b * (K + 1);
    for (int i = 0; i <= K; ++i) o[i] = i < a ? d[i] : (i == a ? arg[a] : -1);
  }
}

}  // namespace vg
