// Expert GEMMs of the MoE layer on tcgen05 tensor cores: gate/up with the
// SwiGLU epilogue and down, in one persistent launch.
//
// Orientation ("swap AB"): the weight rows are the M = 128 operand (A) and the
// tokens routed to an expert are the N operand (B), so one tile streams a
// 128-row slab of one expert's weights once for all of that expert's tokens
// (up to 128 per tile). At decode sizes (about 12 tokens per expert) this is a
// weight stream bound by HBM; at prefill sizes (thousands of tokens per expert)
// the same kernel runs full 128 x 128 tiles and is bound by the tensor pipe.
//
//   gate/up unit: D_gate = W_gate[rows] X^T, D_up = W_up[rows] X^T,
//                 act[token, row] = bf16(silu(D_gate) * D_up)
//   down unit:    D = W_down[rows] act^T, out[token, row] = bf16(D)
//
// Token tiles: each expert's tokens (its segment of the permutation; all T
// tokens for the two shared experts, which ride along as experts E and E+1)
// are cut into tiles of up to 128. Units are (tile, 128-row block): first all
// gate/up units, then all down units. CTAs are persistent and take units from
// a global ticket counter, so no SM idles while units remain. A down unit needs
// the activations of its tile, i.e. all gate/up units of that tile: their
// epilogues count up a per-tile readiness word (release), and the producer of a
// down unit first streams the unit's weights into the free pipeline stages and
// only then waits (acquire, bounded) for the readiness word before loading the
// activations. Tickets are handed out in order and only to running CTAs, so a
// waited-for unit is always already running somewhere: no deadlock, no
// assumption about co-residency.
//
// Warp roles (192 threads): warp 0 takes tickets and issues TMA loads into a
// 4-stage ring; warp 1 owns the tensor memory and one of its threads issues
// tcgen05.mma; warps 2-5 drain the double-buffered TMEM accumulator (each warp
// its own 32-lane quarter) and store the epilogue. Every wait is bounded; a
// timeout records VG_ERR_TIMEOUT, the CTA drains its in-flight copies and MMAs
// (bounded again), frees its tensor memory and exits.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kBM = 128;       // weight rows per tile
constexpr int kBK = 64;        // K elements per stage: one 128-byte swizzle row
constexpr int kNMax = 128;     // tokens per tile
constexpr int kBoxRows = 16;   // token rows per TMA box of the B operand
constexpr int kMaxExperts = 72;

constexpr int kFgStages = 4;
constexpr int kFgABytes = kBM * kBK * 2;                  // 16 KB
constexpr int kFgBBytes = kNMax * kBK * 2;                // 16 KB
constexpr int kFgStageBytes = 2 * kFgABytes + kFgBBytes;  // A_gate | A_up (or A_down) | B
constexpr int kFgAccCols = 2 * kNMax;                     // one accumulator buffer (gate | up)
constexpr int kFgTmemCols = 2 * kFgAccCols;               // double buffered: 512
constexpr int kFgAuxBytes = 2048;
constexpr int kFgSmemBytes = kFgStages * kFgStageBytes + kFgAuxBytes + 1024;  // + alignment slack
constexpr int kFgRing = 4;                                // unit-ticket ring between the roles
constexpr int kFgEpiWarps = 4;

struct FusedArgs {
  const int32_t* offsets;  // [E+1] routed segment offsets in permutation order
  int32_t T, E, S;
  int32_t mblk_gu;         // I / 128
  int32_t mblk_dn;         // H / 128
  int32_t kc_gu;           // H / 64
  int32_t kc_dn;           // I / 64
  int32_t a_up_row;        // first up row inside an expert's gate|up rows (= I)
  int32_t box_xr, box_xs, box_act;  // rows per B box of each B map
  int32_t* sched;          // [0]: ticket counter, [1 + t]: readiness of tile t; zero at launch
  __nv_bfloat16* act;      // [(k+S)T, I]: routed rows in permutation order, then shared
  __nv_bfloat16* out;      // [(k+S)T, H]: expert outputs, same rows
};

struct FgSched {
  int xrow[kMaxExperts];   // first row of the expert's tokens in its gate/up B map
  int arow[kMaxExperts];   // first row of the expert's activations / outputs
  int n[kMaxExperts];      // tokens of the expert
  int pref[kMaxExperts + 1];
};

struct FgUnit {
  int down;  // 0: gate/up, 1: down
  int tile, e, mb, nrows, xrow, arow;
};

__device__ __forceinline__ FgUnit fg_decode(int u, const FgSched& s, int n_exp, const FusedArgs& a) {
  FgUnit un;
  const int u1 = s.pref[n_exp] * a.mblk_gu;
  int v = u, nm = a.mblk_gu;
  un.down = u >= u1;
  if (un.down) {
    v = u - u1;
    nm = a.mblk_dn;
  }
  un.tile = v / nm;
  un.mb = v - un.tile * nm;
  int e = 0;
  while (e + 1 < n_exp && s.pref[e + 1] <= un.tile) ++e;
  const int nb = un.tile - s.pref[e];
  un.e = e;
  un.nrows = min(kNMax, s.n[e] - nb * kNMax);
  un.xrow = s.xrow[e] + nb * kNMax;
  un.arow = s.arow[e] + nb * kNMax;
  return un;
}

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__global__ void __launch_bounds__(192, 1)
    moe_expert_gemms(const __grid_constant__ CUtensorMap mGuR, const __grid_constant__ CUtensorMap mGuS,
                     const __grid_constant__ CUtensorMap mDnR, const __grid_constant__ CUtensorMap mDnS,
                     const __grid_constant__ CUtensorMap mXr, const __grid_constant__ CUtensorMap mXs,
                     const __grid_constant__ CUtensorMap mAct, const FusedArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* aux = smem + kFgStages * kFgStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux);
  uint64_t* empty = full + kFgStages;
  uint64_t* tfull = empty + kFgStages;
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

  if (threadIdx.x == 0) {
    for (int i = 0; i < kFgStages; ++i) {
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
    tmem_alloc(tmem_slot, kFgTmemCols);
    tmem_relinquish();
  }
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
        acc += cdiv(sch->n[e], kNMax);
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
      const uint64_t pol_w = policy_evict_first();
      int stage = 0, slot = 0;
      uint32_t phase = 0, rphase = 0, issued = 0, last_par = 0;
      auto next_stage = [&]() {
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kFgStages) {
          stage = 0;
          phase ^= 1;
        }
      };
      while (true) {
        int u = atomicAdd(ticket, 1);
        if (u >= total || *abort_flag) u = -1;
        if (!mbar_wait(&uempty[slot], rphase ^ 1, limit)) {
          record_error(kErrTimeout, 130);
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
        const FgUnit un = fg_decode(u, *sch, n_exp, args);
        const bool shared = un.e >= args.E;
        const int ecoord = shared ? un.e - args.E : un.e;
        const CUtensorMap* mA = un.down ? (shared ? &mDnS : &mDnR) : (shared ? &mGuS : &mGuR);
        const CUtensorMap* mB = un.down ? &mAct : (shared ? &mXs : &mXr);
        const int box = un.down ? args.box_act : (shared ? args.box_xs : args.box_xr);
        const int brow0 = un.down ? un.arow : un.xrow;
        const int nbox = cdiv(un.nrows, box);
        const int kcs = un.down ? args.kc_dn : args.kc_gu;
        const uint32_t bytes = (un.down ? 1 : 2) * kFgABytes + nbox * box * kBK * 2;
        bool ok = true;
        auto load_b = [&](int st, int kc) {
          uint8_t* bt = tiles + st * kFgStageBytes + 2 * kFgABytes;
          for (int j = 0; j < nbox; ++j)
            tma_load_2d(bt + j * box * kBK * 2, mB, &full[st], kc * kBK, brow0 + j * box);
        };
        // weights of the first stages go out before the activations are known to be ready
        const int npre = un.down ? min(kFgStages, kcs) : 0;
        const int st0 = stage;
        for (int kc = 0; kc < kcs && ok; ++kc) {
          if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
            record_error(kErrTimeout, 131);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = tiles + stage * kFgStageBytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          const int kx = kc * kBK;
          tma_load_3d_hint(st, mA, &full[stage], kx, un.mb * kBM, ecoord, pol_w);
          if (!un.down) tma_load_3d_hint(st + kFgABytes, mA, &full[stage], kx, args.a_up_row + un.mb * kBM, ecoord, pol_w);
          if (kc >= npre) load_b(stage, kc);
          if (kc + 1 == npre) {
            // every stage of the prefetch holds its weights in flight: now wait for the tile
            const uint64_t t0 = globaltimer();
            while (ld_acquire(ready + un.tile) < ready_target) {
              if (globaltimer() - t0 > limit) {
                record_error(kErrTimeout, 132);
                *abort_flag = 1;
                break;  // load anyway so every armed stage completes
              }
              __nanosleep(64);
            }
            fence_proxy_async_global();
            for (int j = 0; j < npre; ++j) load_b((st0 + j) % kFgStages, j);
          }
          next_stage();
        }
        if (!ok) break;
      }
      // every issued copy has landed before the CTA may exit
      for (int s = 0; s < kFgStages; ++s)
        if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0, slot = 0, lu = 0;
      uint32_t phase = 0, rphase = 0;
      while (true) {
        if (!mbar_wait(&ufull[slot], rphase, limit)) {
          record_error(kErrTimeout, 133);
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
        const FgUnit un = fg_decode(u, *sch, n_exp, args);
        const int ab = lu & 1;
        const uint32_t ap = (lu >> 1) & 1;
        ++lu;
        if (!mbar_wait(&tempty[ab], ap ^ 1, limit)) {
          record_error(kErrTimeout, 134);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(kBM, cdiv(un.nrows, 16) * 16);
        const uint32_t d0 = tmem_base + ab * kFgAccCols;
        const uint32_t d1 = d0 + kNMax;
        const int kcs = un.down ? args.kc_dn : args.kc_gu;
        bool ok = true;
        for (int kc = 0; kc < kcs; ++kc) {
          if (!mbar_wait(&full[stage], phase, limit)) {
            record_error(kErrTimeout, 135);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(tiles + stage * kFgStageBytes);
          const uint64_t a0 = sw128_kmajor_desc(st);
          const uint64_t a1 = sw128_kmajor_desc(st + kFgABytes);
          const uint64_t b = sw128_kmajor_desc(st + 2 * kFgABytes);
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16) {
            const uint32_t acc = (kc | k16) != 0;
            umma_bf16(d0, a0 + 2 * k16, b + 2 * k16, idesc, acc);
            if (!un.down) umma_bf16(d1, a1 + 2 * k16, b + 2 * k16, idesc, acc);
          }
          umma_commit(&empty[stage]);
          if (++stage == kFgStages) {
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
    const int row = q * 32 + lane;
    int slot = 0, lu = 0;
    uint32_t rphase = 0;
    while (true) {
      if (!mbar_wait(&ufull[slot], rphase, limit)) {
        record_error(kErrTimeout, 136);
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
      const FgUnit un = fg_decode(u, *sch, n_exp, args);
      const int ab = lu & 1;
      const uint32_t ap = (lu >> 1) & 1;
      ++lu;
      if (!mbar_wait(&tfull[ab], ap, limit)) {
        record_error(kErrTimeout, 137);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + ab * kFgAccCols;
      const int ld = un.down ? args.mblk_dn * kBM : args.mblk_gu * kBM;
      __nv_bfloat16* dst = (un.down ? args.out : args.act) + (size_t)un.arow * ld + un.mb * kBM + row;
      for (int c0 = 0; c0 < un.nrows; c0 += 16) {
        uint32_t g[16], v[16];
        tmem_ld16(t0 + c0, g);
        if (!un.down) tmem_ld16(t0 + kNMax + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (c0 + j < un.nrows) {
            const float r = un.down ? __uint_as_float(g[j]) : silu(__uint_as_float(g[j])) * __uint_as_float(v[j]);
            dst[(size_t)(c0 + j) * ld] = __float2bfloat16_rn(r);
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
    tmem_dealloc(tmem_base, kFgTmemCols);
  }
}

// Weighted combine of the layer: out[t] = bf16(res + sum_s o_shared[s][t] +
// sum_j g[t,j] * o[inv[t,j]]) with res = x[t] if add_residual else 0. One
// thread per 8 consecutive hidden elements; fixed summation order.
__global__ void __launch_bounds__(256) moe_combine(const __nv_bfloat16* __restrict__ x,
                                                   const __nv_bfloat16* __restrict__ o,
                                                   const int32_t* __restrict__ inv, const float* __restrict__ g,
                                                   int T, int H, int k, int S, int add_residual,
                                                   __nv_bfloat16* __restrict__ out) {
  const int per_row = H / 8;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * per_row) return;
  const int t = i / per_row, c = i - t * per_row;
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
  reinterpret_cast<uint4*>(out + (size_t)t * H)[c] = r;
}

}  // namespace vg
