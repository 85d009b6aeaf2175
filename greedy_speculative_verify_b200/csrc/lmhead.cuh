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
// lmhead_argmax_accept: tcgen05 GEMM with the verify rows as M (128 per tile)
// and a 176-row vocabulary slab as N; the fp32 logits never leave tensor
// memory. The epilogue thread that owns row r scans its 176 columns in
// increasing vocabulary order and keeps the best (value, index) as one 64-bit
// key: the order-preserving image of the fp32 value in the high word and
// (2^32-1-v) in the low word, so that the larger key is the larger logit and,
// among equal logits, the lower index. A work unit is a group of consecutive
// vocabulary tiles for one 128-row block; the key is carried across the
// group's tiles and folded into the row's global key with an atomic max. The
// last CTA to finish decodes the argmax, counts for each sequence the leading
// drafts equal to the argmax of the preceding position, and writes the
// committed tokens.
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

struct LmArgs {
  int R, V, k_chunks, n_mblk, n_vblk, group_tiles, n_groups, a_box_rows, b_box_rows;
  int B, K;
  const int32_t* drafts;         // [B, K]; may be null when K == 0
  int32_t* argmax;               // [R]
  int32_t* accepted;             // [B]
  int32_t* out_tokens;           // [B, K+1]
  unsigned long long* best;      // [R] running max key per row: zero at entry, left zero
  uint32_t* done;                // CTAs finished: zero at entry, left zero
};

// Grid: one CTA per SM over units (vocabulary group, 128-row block). Before it
// waits for the previous kernel, the producer already streams the vocabulary
// tiles of its first stages (the LM head is immutable; only the hidden states
// come from the previous kernel). Each unit folds its rows' best keys into
// `best` with a 64-bit atomic max (order-independent, so the result does not
// depend on the CTAs' timing); the last CTA to finish turns the keys into the
// argmax, accepts each sequence's longest agreeing prefix plus the bonus token,
// and clears `best` and `done` for the next call.
__global__ void __launch_bounds__(192, 1)
    lmhead_argmax_accept(const __grid_constant__ CUtensorMap mapH, const __grid_constant__ CUtensorMap mapLM,
                         const LmArgs a) {
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
  __shared__ int last_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = a.n_groups * a.n_mblk;  // unit = (vocabulary group, row block), row block fastest
  const uint32_t a_bytes = a.a_box_rows * kBK * 2, b_bytes = a.b_box_rows * kBK * 2;
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
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t limit = g_wait_timeout_ns;

  // vocabulary tiles of the first stages of this CTA's first unit, in the
  // order the main loop consumes them: before the dependency wait
  int npre = 0;
  const uint64_t pol_w = policy_evict_first();
  if (warp == 0 && lane == 0 && (int)blockIdx.x < total) {
    const int g = blockIdx.x / a.n_mblk;
    const int vb1 = min(a.n_vblk, (g + 1) * a.group_tiles);
    for (int vb = g * a.group_tiles; vb < vb1 && npre < kLmStages; ++vb)
      for (int kc = 0; kc < a.k_chunks && npre < kLmStages; ++kc, ++npre) {
        mbar_expect_tx(&full[npre], b_bytes);
        tma_load_2d_hint(tiles + npre * kLmStageBytes + kLmABytes, &mapLM, &full[npre], kc * kBK, vb * kLmN, pol_w);
      }
  }
  griddep_wait();  // the hidden states (and the workspace) come from earlier kernels

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_h = policy_evict_last();
      int stage = 0, it = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
        const int g = u / a.n_mblk, mb = u - g * a.n_mblk;
        const int vb1 = min(a.n_vblk, (g + 1) * a.group_tiles);
        for (int vb = g * a.group_tiles; vb < vb1 && !*abort_flag; ++vb) {
          for (int kc = 0; kc < a.k_chunks; ++kc, ++it) {
            if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
              record_error(kErrTimeout, 121);
              *abort_flag = 1;
              break;
            }
            uint8_t* st = tiles + stage * kLmStageBytes;
            const bool pre = it < npre;  // its vocabulary tile is already in flight
            mbar_arrive_expect_tx(&full[stage], pre ? a_bytes : a_bytes + b_bytes);
            tma_load_2d_hint(st, &mapH, &full[stage], kc * kBK, mb * kLmM, pol_h);
            if (!pre) tma_load_2d_hint(st + kLmABytes, &mapLM, &full[stage], kc * kBK, vb * kLmN, pol_w);
            issued |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
            if (++stage == kLmStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      }
      // stages armed before the wait but never reached (an abort): arrive, so
      // their copies complete the phase and can be drained below
      for (; it < npre; ++it) {
        mbar_arrive(&full[it]);
        issued |= 1u << it;
        last_par &= ~(1u << it);
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
        const int g = u / a.n_mblk;
        const int vb1 = min(a.n_vblk, (g + 1) * a.group_tiles);
        for (int vb = g * a.group_tiles; vb < vb1 && ok; ++vb, ++lt) {
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
          for (int kc = 0; kc < a.k_chunks; ++kc) {
            if (!mbar_wait(&full[stage], phase, limit)) {
              record_error(kErrTimeout, 123);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(tiles + stage * kLmStageBytes);
            const uint64_t da = sw128_kmajor_desc(st);
            const uint64_t db = sw128_kmajor_desc(st + kLmABytes);
#pragma unroll
            for (int k16 = 0; k16 < kBK / 16; ++k16)
              umma_bf16(d, da + 2 * k16, db + 2 * k16, idesc, (kc | k16) != 0);
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
      const int g = u / a.n_mblk, mb = u - g * a.n_mblk;
      const int vb1 = min(a.n_vblk, (g + 1) * a.group_tiles);
      uint64_t best = 0;  // running (value, index) key of this row over the group's tiles
      for (int vb = g * a.group_tiles; vb < vb1; ++vb, ++lt) {
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
            if (v < a.V) {
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
      if (ok && r < a.R) atomicMax(a.best + r, (unsigned long long)best);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kLmTmemCols);
  }

  // ---- the last CTA to finish: argmax, prefix accept, and the workspace back to zero
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's key updates precede its arrival
    const uint32_t old = atomicAdd(a.done, 1u);
    if (old >= gridDim.x) record_error(kErrBounds, 125);  // the counter was not zero at entry
    last_s = old == gridDim.x - 1;
  }
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  for (int r = threadIdx.x; r < a.R; r += blockDim.x) {
    const unsigned long long k = atomicExch(a.best + r, 0ull);
    const int32_t v = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
    a.argmax[r] = VG_IN_BOUNDS(v >= 0 && v < a.V, 409) ? v : 0;
  }
  __syncthreads();  // every argmax of this CTA is visible to all its threads
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    const int32_t* arg = a.argmax + (size_t)b * (a.K + 1);
    const int32_t* d = a.drafts + (size_t)b * a.K;
    int acc = 0;
    while (acc < a.K && d[acc] == arg[acc]) ++acc;
    a.accepted[b] = acc;
    int32_t* o = a.out_tokens + (size_t)b * (a.K + 1);
    for (int i = 0; i <= a.K; ++i) o[i] = i < acc ? d[i] : (i == acc ? arg[acc] : -1);
  }
  if (threadIdx.x == 0) atomicExch(a.done, 0u);
}

}  // namespace vg
