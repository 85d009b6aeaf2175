// Expert GEMMs of the MoE layer at prefill sizes, token-major: the tokens of a
// 128-token tile are the M = 128 operand (A) and a 256-row weight slab is the
// N = 256 operand (B), so each k-step is one tcgen05.mma of 128 x 256 x 16.
//
// Per pipeline stage (48 KB): the tile's 128 token rows of one 64-wide k-chunk
// (16 KB) and one 32 KB weight box (the same boxes as the decode kernel):
//   gate/up unit (tile, 128-row block r): gate rows 128 r .. 128 r + 127 then
//       the up rows of the same block, stacked as the 256 rows of B, so column
//       j of the accumulator is gate row j and column 128 + j is up row j of
//       the block: act[token, 128 r + j] = bf16(silu(D[., j]) * D[., 128 + j]);
//   down unit (tile, 256-row block r): rows 256 r .. 256 r + 255 of W_down;
//       out[token, 256 r + j] = bf16(D[., j]).
// Against the weight-major decode kernel (two 128 x N MMAs sharing the token
// operand) a k-step reads 12 KB of operands from shared memory instead of 16 KB
// for the same 2 x 128 x 256 x 16 FLOP, and the epilogue thread owns one
// token's row, so it writes 256 (gate/up) or 512 (down) contiguous bytes.
//
// Scheduling, readiness words, warp roles and bounded waits are those of the
// decode kernel (gemm_moe.cuh): persistent CTAs take units from a ticket
// counter, gate/up units first, then down units, which stream their weights
// first and wait for their tile's activations. A tile shorter than 128 tokens
// computes all 128 rows (the rows past the expert's segment belong to the next
// expert or read as zero past the tensor's end) and stores only its own.
#pragma once
#include "common.cuh"
#include "gemm_moe.cuh"

namespace vg {

constexpr int kTmM = 128;                       // tokens per tile (MMA M)
constexpr int kTmN = 256;                       // weight rows per unit (MMA N)
constexpr int kTmStages = 4;
constexpr int kTmABytes = kTmM * kBK * 2;       // 16 KB of token rows
constexpr int kTmBBytes = kTmN * kBK * 2;       // 32 KB weight box
constexpr int kTmStageBytes = kTmABytes + kTmBBytes;
constexpr int kTmAccCols = kTmN;                // one accumulator buffer
constexpr int kTmTmemCols = 2 * kTmAccCols;     // double buffered: all 512 columns
constexpr int kTmSmemBytes = kTmStages * kTmStageBytes + 2048 + 1024;

// Packs 16 fp32 values as bf16 into two 16-byte vectors.
__device__ __forceinline__ void pack16_bf16(const float (&v)[16], uint4& lo, uint4& hi) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    p[j] = *reinterpret_cast<uint32_t*>(&b);
  }
  lo = make_uint4(p[0], p[1], p[2], p[3]);
  hi = make_uint4(p[4], p[5], p[6], p[7]);
}

__global__ void __launch_bounds__(192, 1)
    moe_expert_gemms_tm(const __grid_constant__ CUtensorMap mGuR, const __grid_constant__ CUtensorMap mGuS,
                        const __grid_constant__ CUtensorMap mDnR, const __grid_constant__ CUtensorMap mDnS,
                        const __grid_constant__ CUtensorMap mXr, const __grid_constant__ CUtensorMap mXs,
                        const __grid_constant__ CUtensorMap mAct, const FusedArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* aux = smem + kTmStages * kTmStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux);
  uint64_t* empty = full + kTmStages;
  uint64_t* tfull = empty + kTmStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* ufull = tempty + 2;
  uint64_t* uempty = ufull + kFgRing;
  uint64_t* mma_done = uempty + kFgRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);  // kFgRing tickets
  FgSched* sch = reinterpret_cast<FgSched*>(aux + 512);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_exp = args.E + args.S;
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTmStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kFgEpiWarps);
    }
    for (int i = 0; i < kFgRing; ++i) {
      mbar_init(&ufull[i], 1);
      mbar_init(&uempty[i], 1 + kFgEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&mGuR);
    prefetch_tmap(&mGuS);
    prefetch_tmap(&mDnR);
    prefetch_tmap(&mDnS);
    prefetch_tmap(&mXr);
    prefetch_tmap(&mXs);
    prefetch_tmap(&mAct);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmTmemCols);
    tmem_relinquish();
  }
  griddep_wait();  // the grouping is read from here on
  if (warp == 2) {
    const int kT = args.offsets[args.E];
    for (int e = lane; e < n_exp; e += 32) {
      if (e < args.E) {
        const int o0 = args.offsets[e], o1 = args.offsets[e + 1];
        sch->xrow[e] = o0;
        sch->arow[e] = o0;
        sch->n[e] = o1 - o0;
      } else {
        const int s = e - args.E;
        sch->xrow[e] = 0;
        sch->arow[e] = kT + s * args.T;
        sch->n[e] = args.T;
      }
    }
    __syncwarp();
    if (lane == 0) {
      int acc = 0;
      for (int e = 0; e < n_exp; ++e) {
        sch->pref[e] = acc;
        acc += cdiv(sch->n[e], kTmM);
      }
      sch->pref[n_exp] = acc;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = *tmem_slot;
  const int n_tiles = sch->pref[n_exp];
  const int total = n_tiles * (args.mblk_gu + args.mblk_dn);
  const uint64_t limit = g_wait_timeout_ns;
  int32_t* ticket = args.sched;
  int32_t* ready = args.sched + 1;
  const int ready_target = args.mblk_gu * kFgEpiWarps;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // prefill tiles re-read each weight slab once per token tile: normal L2 priority
      const uint64_t pol_w = policy_evict_normal();
      int stage = 0, slot = 0;
      uint32_t phase = 0, rphase = 0, issued = 0, last_par = 0;
      auto next_stage = [&]() {
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kTmStages) {
          stage = 0;
          phase ^= 1;
        }
      };
      int next_u = atomicAdd(ticket, 1);
      while (true) {
        int u = next_u;
        if (u >= total || *abort_flag) u = -1;
        if (u >= 0) next_u = atomicAdd(ticket, 1);
        if (!mbar_wait(&uempty[slot], rphase ^ 1, limit)) {
          record_error(kErrTimeout, 140);
          *abort_flag = 1;
          u = -1;
        }
        ring[slot] = u;
        mbar_arrive(&ufull[slot]);
        if (++slot == kFgRing) {
          slot = 0;
          rphase ^= 1;
        }
        if (u < 0) break;
        const FgUnit un = fg_decode(u, *sch, n_exp, args, kTmM);
        const bool shared = un.e >= args.E;
        const int ecoord = shared ? un.e - args.E : un.e;
        const CUtensorMap* mW = un.down ? (shared ? &mDnS : &mDnR) : (shared ? &mGuS : &mGuR);
        const CUtensorMap* mT = un.down ? &mAct : (shared ? &mXs : &mXr);
        const int trow = un.down ? un.arow : un.xrow;
        const int nst = un.down ? args.kc_dn : args.kc_gu;
        const int wrow = un.down ? un.mb * kTmN : un.mb * kBM;
        bool ok = true;
        // weights of the first stages go out before the activations are known to be ready
        const int npre = un.down ? min(kTmStages, nst) : 0;
        const int st0 = stage;
        for (int kc = 0; kc < nst && ok; ++kc) {
          if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
            record_error(kErrTimeout, 141);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = tiles + stage * kTmStageBytes;
          mbar_arrive_expect_tx(&full[stage], kTmStageBytes);
          if (un.down)
            tma_load_3d_hint(st + kTmABytes, mW, &full[stage], kc * kBK, wrow, ecoord, pol_w);
          else
            tma_load_4d_hint(st + kTmABytes, mW, &full[stage], kc * kBK, wrow, 0, ecoord, pol_w);
          if (kc >= npre) tma_load_2d(st, mT, &full[stage], kc * kBK, trow);
          if (kc + 1 == npre) {
            // every stage of the prefetch holds its weights in flight: now wait for the tile
            const uint64_t t0 = globaltimer();
            while (ld_acquire(ready + un.tile) < ready_target) {
              if (globaltimer() - t0 > limit) {
                record_error(kErrTimeout, 142);
                *abort_flag = 1;
                break;  // load anyway so every armed stage completes
              }
              __nanosleep(64);
            }
            fence_proxy_async_global();
            for (int j = 0; j < npre; ++j)
              tma_load_2d(tiles + ((st0 + j) % kTmStages) * kTmStageBytes, mT, &full[(st0 + j) % kTmStages],
                          j * kBK, trow);
          }
          next_stage();
        }
        if (!ok) break;
      }
      // every issued copy has landed before the CTA may exit
      for (int s = 0; s < kTmStages; ++s)
        if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kTmM, kTmN);
      int stage = 0, slot = 0, lu = 0;
      uint32_t phase = 0, rphase = 0;
      while (true) {
        if (!mbar_wait(&ufull[slot], rphase, limit)) {
          record_error(kErrTimeout, 143);
          *abort_flag = 1;
          break;
        }
        const int u = ring[slot];
        mbar_arrive(&uempty[slot]);
        if (++slot == kFgRing) {
          slot = 0;
          rphase ^= 1;
        }
        if (u < 0 || *abort_flag) break;
        const FgUnit un = fg_decode(u, *sch, n_exp, args, kTmM);
        const int ab = lu & 1;
        const uint32_t ap = (lu >> 1) & 1;
        ++lu;
        if (!mbar_wait(&tempty[ab], ap ^ 1, limit)) {
          record_error(kErrTimeout, 144);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + ab * kTmAccCols;
        const int nst = un.down ? args.kc_dn : args.kc_gu;
        bool ok = true;
        for (int kc = 0; kc < nst; ++kc) {
          if (!mbar_wait(&full[stage], phase, limit)) {
            record_error(kErrTimeout, 145);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(tiles + stage * kTmStageBytes);
          const uint64_t da = sw128_kmajor_desc(st);
          const uint64_t db = sw128_kmajor_desc(st + kTmABytes);
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16) umma_bf16(d, da + 2 * k16, db + 2 * k16, idesc, (kc | k16) != 0);
          umma_commit(&empty[stage]);
          if (++stage == kTmStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[ab]);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, limit);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;  // the token row of the tile this thread owns
    int slot = 0, lu = 0;
    uint32_t rphase = 0;
    while (true) {
      if (!mbar_wait(&ufull[slot], rphase, limit)) {
        record_error(kErrTimeout, 146);
        *abort_flag = 1;
        break;
      }
      const int u = ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[slot]);
      if (++slot == kFgRing) {
        slot = 0;
        rphase ^= 1;
      }
      if (u < 0 || *abort_flag) break;
      const FgUnit un = fg_decode(u, *sch, n_exp, args, kTmM);
      const int ab = lu & 1;
      const uint32_t ap = (lu >> 1) & 1;
      ++lu;
      if (!mbar_wait(&tfull[ab], ap, limit)) {
        record_error(kErrTimeout, 147);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      // the unit's rows lie inside the activation / output buffers: routed rows, then S x T shared rows
      const bool rows_ok = VG_IN_BOUNDS(un.arow >= 0 && un.arow + un.nrows <= sch->arow[args.E] + args.S * args.T,
                                        406);
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + ab * kTmAccCols;
      const bool mine = rows_ok && row < un.nrows;
      if (un.down) {
        const int ld = args.mblk_dn * kTmN;
        uint4* dst = reinterpret_cast<uint4*>(args.out + (size_t)(un.arow + row) * ld + un.mb * kTmN);
#pragma unroll 1
        for (int c0 = 0; c0 < kTmN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(t0 + c0, r);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
          uint4 lo, hi;
          pack16_bf16(v, lo, hi);
          if (mine) {
            dst[c0 / 8] = lo;
            dst[c0 / 8 + 1] = hi;
          }
        }
      } else {
        const int ld = args.mblk_gu * kBM;
        uint4* dst = reinterpret_cast<uint4*>(args.act + (size_t)(un.arow + row) * ld + un.mb * kBM);
#pragma unroll 1
        for (int c0 = 0; c0 < kBM; c0 += 16) {
          uint32_t g[16], up[16];
          tmem_ld16(t0 + c0, g);
          tmem_ld16(t0 + kBM + c0, up);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = silu(__uint_as_float(g[j])) * __uint_as_float(up[j]);
          uint4 lo, hi;
          pack16_bf16(v, lo, hi);
          if (mine) {
            dst[c0 / 8] = lo;
            dst[c0 / 8 + 1] = hi;
          }
        }
      }
      tc_fence_before();
      if (!un.down) fence_proxy_async_global();  // the activations are read back through TMA
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[ab]);
        if (!un.down) {
          __threadfence();
          atomicAdd(ready + un.tile, 1);
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmTmemCols);
  }
}

}  // namespace vg
