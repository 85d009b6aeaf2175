// Expert GEMMs of the MoE layer on tcgen05 tensor cores: gate/up with the
// SwiGLU epilogue and down, in one persistent launch.
//
// Orientation ("swap AB"): the weight rows are the M = 128 operand (A) and the
// tokens routed to an expert are the N operand (B), so one tile streams a slab
// of one expert's weights once for all of that expert's tokens (up to NMAX per
// tile). At decode sizes (about 12 tokens per expert) this is a weight stream
// bound by HBM; at prefill sizes (thousands of tokens per expert) the same
// kernel runs full 128 x 128 tiles and is bound by the tensor pipe.
//
// Every pipeline stage carries two 128 x 64 weight tiles (32 KB, one TMA
// instruction) and one 64-wide k-chunk of the tile's token rows, and feeds two
// accumulators that share the token operand:
//   gate/up unit (tile, 128-row block r): the gate and up rows of block r
//       (one box of a 4-d view: k, row, gate|up, expert) into D0 = gate,
//       D1 = up; act[token, r rows] = bf16(silu(D0) * D1);
//   down unit (tile, 256-row block r): rows 256 r .. 256 r + 255 of W_down (one
//       256-row box) into D0 = lower, D1 = upper 128 rows; out[token, rows] = bf16(D).
//
// Token tiles: each expert's tokens (its segment of the permutation; all T
// tokens for the two shared experts, which ride along as experts E and E+1)
// are cut into tiles of up to NMAX. Units are first all gate/up units, then all
// down units. CTAs are persistent and take units from a global ticket counter,
// so no SM idles while units remain. A down unit needs the activations of its
// tile, i.e. all gate/up units of that tile: their epilogues count up a
// per-tile readiness word (release), and the producer of a down unit first
// streams the unit's weights into the free pipeline stages and only then waits
// (acquire, bounded) for the readiness word before loading the activations.
// Tickets are handed out in order and only to running CTAs, so a waited-for
// unit is always already running somewhere: no deadlock, no assumption about
// co-residency.
//
// Warp roles (192 threads): warp 0 takes tickets and issues TMA loads into the
// stage ring; warp 1 owns the tensor memory and one of its threads issues
// tcgen05.mma; warps 2-5 drain the double-buffered TMEM accumulator (each warp
// its own 32-lane quarter) and store the epilogue. Every wait is bounded; a
// timeout records VG_ERR_TIMEOUT, the CTA drains its in-flight copies and MMAs
// (bounded again), frees its tensor memory and exits.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kBM = 128;       // weight rows per MMA tile
constexpr int kBK = 64;        // K elements per stage: one 128-byte swizzle row
constexpr int kBoxRows = 32;   // token rows per TMA box of the B operand
constexpr int kMaxExperts = 72;

// Three configurations of the same kernel, by tile width NMAX:
//  * NMAX = 128, 4 stages: prefill-sized expert segments, 128 x 128 tiles;
//  * NMAX = 64, 5 stages: decode sizes, where the token slot of a stage is
//    small and the freed shared memory buys a fifth stage of weights in flight;
//  * NMAX = 16, 6 stages: a handful of tokens (batch-1 verify), where every
//    expert's tokens fit one 16-row tile and a sixth stage fits.
#ifndef VG_FG_STAGES_64
#define VG_FG_STAGES_64 5
#endif

template <int NMAX>
struct FgCfg {
  static constexpr int kStages = NMAX == 128 ? 4 : NMAX == 64 ? VG_FG_STAGES_64 : 6;
  static constexpr int kABytes = 2 * kBM * kBK * 2;      // two 16 KB weight tiles
  static constexpr int kBBytes = NMAX * kBK * 2;         // token slot
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kAccCols = 2 * NMAX;              // one accumulator buffer (D0 | D1)
  static constexpr int kTmemCols = 2 * kAccCols;         // double buffered
  static constexpr int kAuxBytes = 2048;
  static constexpr int kSmemBytes = kStages * kStageBytes + kAuxBytes + 1024;  // + alignment slack
};
constexpr int kFgTileBytes = kBM * kBK * 2;               // one 128 x 64 weight tile
constexpr int kFgRing = 4;                                // unit-ticket ring between the roles
constexpr int kFgEpiWarps = 4;

struct FusedArgs {
  const int32_t* offsets;  // [E+1] routed segment offsets in permutation order
  int32_t T, E, S;
  int32_t mblk_gu;         // I / 128 gate/up row blocks
  int32_t mblk_dn;         // H / 256 down row blocks
  int32_t kc_gu;           // H / 64
  int32_t kc_dn;           // I / 64
  int32_t box_xr, box_xs, box_act;  // rows per B box of each B map
  int32_t* sched;          // [0]: ticket counter, [1 + t]: readiness of tile t; zero at launch
  __nv_bfloat16* act;      // [(k+S)T, I]: routed rows in permutation order, then shared
  __nv_bfloat16* out;      // [(k+S)T, H]: expert outputs, same rows
  // 1: every expert has a primary tile (its first NMAX tokens, possibly none),
  // tiles 0 .. E+S-1 in expert order, then the further tiles; CTA b's first unit
  // is unit b (a gate/up unit of a primary tile, known before the routing), and
  // its weights are requested before the kernel waits for the previous one.
  // The gate/up token rows of routed expert e's primary tile are rows
  // e NMAX .. e NMAX + NMAX - 1 of the B map, its further tiles' rows follow
  // E NMAX + (segment offset), so the first unit's token rows are requested
  // right after the wait, before the offsets are read
  int32_t static_first;
  int32_t pre_l2_chunks;   // static_first: k-chunks of the first unit past the stages, prefetched to L2
};

struct FgSched {
  int xrow[kMaxExperts];   // first row of the expert's tokens in its gate/up B map
  int arow[kMaxExperts];   // first row of the expert's activations / outputs
  int n[kMaxExperts];      // tokens of the expert
  // first tile of each expert (static_first: first tile beyond its primary one,
  // counted from tile E+S); pref[E+S] = the total
  int pref[kMaxExperts + 1];
};

struct FgUnit {
  int down;  // 0: gate/up, 1: down
  int tile, e, mb, nrows, xrow, arow;
};

__device__ __forceinline__ FgUnit fg_decode(int u, const FgSched& s, int n_exp, const FusedArgs& a, int nmax) {
  FgUnit un;
  const int n_tiles = s.pref[n_exp] + (a.static_first ? n_exp : 0);
  const int u1 = n_tiles * a.mblk_gu;  // gate/up units come first
  int v = u, nm = a.mblk_gu;
  un.down = u >= u1;
  if (un.down) {
    v = u - u1;
    nm = a.mblk_dn;
  }
  un.tile = v / nm;
  un.mb = v - un.tile * nm;
  int e, nb;
  if (a.static_first && un.tile < n_exp) {  // primary tile of expert `tile`
    e = un.tile;
    nb = 0;
  } else {
    // the expert of the tile: the last e with pref[e] <= t (experts without
    // (further) tiles have pref[e] == pref[e + 1] and are skipped by taking the last)
    const int t = a.static_first ? un.tile - n_exp : un.tile;
    int lo = 0, hi = n_exp - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s.pref[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    e = lo;
    nb = t - s.pref[e] + (a.static_first ? 1 : 0);
  }
  un.e = e;
  un.nrows = max(0, min(nmax, s.n[e] - nb * nmax));  // 0 only for the primary tile of an expert without tokens
  un.xrow = a.static_first && nb == 0 && e < a.E ? e * nmax : s.xrow[e] + nb * nmax;
  un.arow = s.arow[e] + nb * nmax;
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

template <int NMAX>
__global__ void __launch_bounds__(192, 1)
    moe_expert_gemms(const __grid_constant__ CUtensorMap mGuR, const __grid_constant__ CUtensorMap mGuS,
                     const __grid_constant__ CUtensorMap mDnR, const __grid_constant__ CUtensorMap mDnS,
                     const __grid_constant__ CUtensorMap mXr, const __grid_constant__ CUtensorMap mXs,
                     const __grid_constant__ CUtensorMap mAct, const FusedArgs args) {
  using C = FgCfg<NMAX>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* aux = smem + C::kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* ufull = tempty + 2;
  uint64_t* uempty = ufull + kFgRing;
  uint64_t* mma_done = uempty + kFgRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);  // kFgRing tickets
  uint64_t* sched_ready = reinterpret_cast<uint64_t*>(aux + 256);        // the schedule below is built
  FgSched* sch = reinterpret_cast<FgSched*>(aux + 512);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_exp = args.E + args.S;
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
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
    mbar_init(sched_ready, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // static_first: the weights of this CTA's first unit (gate/up of row block
  // blockIdx.x % mblk_gu of expert blockIdx.x / mblk_gu) go out before the wait;
  // its token rows follow once the routing is known
  const int npre0 = args.static_first ? min(C::kStages, args.kc_gu) : 0;
  if (npre0 > 0 && threadIdx.x == 0) {
    const int e0 = blockIdx.x / args.mblk_gu, mb0 = blockIdx.x - e0 * args.mblk_gu;
    const bool sh = e0 >= args.E;
    const CUtensorMap* mA = sh ? &mGuS : &mGuR;
    const int ec = sh ? e0 - args.E : e0;
    const uint64_t pol_w = NMAX <= 64 ? policy_evict_first() : policy_evict_normal();
    for (int kc = 0; kc < npre0; ++kc) {
      mbar_expect_tx(&full[kc], C::kABytes);
      tma_load_4d_hint(tiles + kc * C::kStageBytes, mA, &full[kc], kc * kBK, mb0 * kBM, 0, ec, pol_w);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  const uint64_t limit = g_wait_timeout_ns;
  // barriers and TMEM are published before the wait: no CTA-wide barrier follows it
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (warp == 3 && lane == 0) {
    // an epilogue warp, idle until the first unit's MMAs: descriptors, and
    // further k-chunks of the first unit to L2, off the producer's path
    prefetch_tmap(&mGuR);
    prefetch_tmap(&mGuS);
    prefetch_tmap(&mDnR);
    prefetch_tmap(&mDnS);
    prefetch_tmap(&mXr);
    prefetch_tmap(&mXs);
    prefetch_tmap(&mAct);
    if (npre0 > 0) {
      const int e0 = blockIdx.x / args.mblk_gu, mb0 = blockIdx.x - e0 * args.mblk_gu;
      const bool sh = e0 >= args.E;
      const int kc1 = min(args.kc_gu, npre0 + args.pre_l2_chunks);
      for (int kc = npre0; kc < kc1; ++kc) tma_prefetch_4d(sh ? &mGuS : &mGuR, kc * kBK, mb0 * kBM, 0, sh ? e0 - args.E : e0);
    }
  }
  griddep_wait();  // the grouping is read from here on

  // static_first: every role decodes the fixed first unit itself. The producer
  // and the MMA issuer take it as a full tile whose token rows are known
  // without the offsets (rows past the expert's tokens are computed and
  // dropped), so its token rows are requested right after the wait; the
  // epilogue reads the expert's row count and output rows from the offsets.
  const bool epi = warp >= 2;
  const int kT = epi ? args.offsets[args.E] : 0;  // routed rows; shared expert s owns rows kT + s T ..
  [[maybe_unused]] const int rows_total = kT + args.S * args.T;  // bound of the epilogue's row checks
  const int first_u = args.static_first ? (int)blockIdx.x : -1;
  FgUnit first{};
  if (args.static_first) {
    const int e0 = blockIdx.x / args.mblk_gu;
    first.tile = first.e = e0;
    first.mb = blockIdx.x - e0 * args.mblk_gu;
    const bool routed = e0 < args.E;
    first.xrow = routed ? e0 * NMAX : 0;
    first.nrows = NMAX;
    first.arow = -1;
    if (epi) {
      int n;
      if (routed) {
        const int o0 = args.offsets[e0], o1 = args.offsets[e0 + 1];
        first.arow = o0;
        n = o1 - o0;
      } else {
        first.arow = kT + (e0 - args.E) * args.T;
        n = args.T;
      }
      first.nrows = max(0, min(NMAX, n));
    }
  }
  if (warp == 2) {
    // the schedule: rows and tile prefix of every expert, kPer experts per lane
    constexpr int kPer = (kMaxExperts + 31) / 32;
    int o[kPer + 1];
#pragma unroll
    for (int i = 0; i <= kPer; ++i) {  // every offset this lane needs, requested at once
      const int e = lane * kPer + i;
      o[i] = e <= args.E ? args.offsets[e] : 0;
    }
    const int xbase = args.static_first ? args.E * NMAX : 0;  // further tiles' token rows
    int cnt[kPer], local = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane * kPer + i;
      int n = 0;
      if (e < n_exp) {
        const bool routed = e < args.E;
        n = routed ? o[i + 1] - o[i] : args.T;
        sch->xrow[e] = routed ? xbase + o[i] : 0;
        sch->arow[e] = routed ? o[i] : kT + (e - args.E) * args.T;
        sch->n[e] = n;
      }
      const int nt = cdiv(n, NMAX);
      cnt[i] = e < n_exp ? (args.static_first ? max(0, nt - 1) : nt) : 0;
      local += cnt[i];
    }
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    int run = incl - local;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane * kPer + i;
      if (e < n_exp) sch->pref[e] = run;
      run += cnt[i];
    }
    if (lane == 31) sch->pref[n_exp] = incl;
    __syncwarp();
    if (lane == 0) mbar_arrive(sched_ready);  // releases the schedule to the other roles
  }
  // every unit but the fixed first one is decoded from the schedule; each role
  // waits for it once
  bool sched_seen = false;
  auto wait_sched = [&](int site) -> bool {
    if (!sched_seen) {
      if (!mbar_wait(sched_ready, 0, limit)) {
        record_error(kErrTimeout, site);
        *abort_flag = 1;
        return false;
      }
      sched_seen = true;
    }
    return true;
  };
  auto decode = [&](int u, FgUnit& un, int site) -> bool {
    if (u == first_u) {
      un = first;
      return true;
    }
    if (!wait_sched(site)) return false;
    un = fg_decode(u, *sch, n_exp, args, NMAX);
    return true;
  };

  int32_t* ticket = args.sched;
  int32_t* ready = args.sched + 1;
  const int ready_target = args.mblk_gu * kFgEpiWarps;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // decode tiles read an expert's weights once: stream them past L2; prefill
      // tiles re-read them once per token tile, so they stay at normal priority
      const uint64_t pol_w = NMAX <= 64 ? policy_evict_first() : policy_evict_normal();
      int stage = 0, slot = 0;
      uint32_t phase = 0, rphase = 0, issued = 0, last_par = 0;
      auto next_stage = [&]() {
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
        }
      };
      // the next ticket is requested one unit ahead so its round trip overlaps the loads
      const int tbase = args.static_first ? (int)gridDim.x : 0;  // tickets after the fixed first units
      int next_u = args.static_first ? (int)blockIdx.x : atomicAdd(ticket, 1);
      bool pre_pending = npre0 > 0;  // stages 0 .. npre0-1 armed before the wait, not yet handed on
      int total = -1;  // units of this launch, once the schedule is known
      while (true) {
        int u = next_u;
        if (u >= 0 && u != first_u) {
          if (total < 0)
            total = wait_sched(139) ? (sch->pref[n_exp] + (args.static_first ? n_exp : 0)) *
                                          (args.mblk_gu + args.mblk_dn)
                                    : 0;
          if (u >= total) u = -1;
        }
        if (*abort_flag) u = -1;
        const bool pre_unit = pre_pending && u >= 0;  // the first unit: its weight stages are armed
        // the fixed first unit asks for its successor only once its armed stages
        // have their token rows requested: every CTA starts it at once, and the
        // ticket's round trip is not on the way to the first MMA
        bool want_ticket = u >= 0;
        if (want_ticket && !pre_unit) {
          next_u = tbase + atomicAdd(ticket, 1);
          want_ticket = false;
        }
        FgUnit un{};
        if (u >= 0) {
          if (!decode(u, un, 139)) u = -1;
          else if (un.nrows == 0 && !pre_unit) continue;  // a tile without tokens: nothing to compute
        }
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
        pre_pending = false;
        if (un.nrows == 0) {
          // the pre-armed unit of an expert no token chose: its weight copies
          // complete the armed stages, which the MMA issuer then releases
          for (int kc = 0; kc < npre0; ++kc) {
            mbar_arrive(&full[stage]);
            next_stage();
          }
          if (want_ticket) next_u = tbase + atomicAdd(ticket, 1);
          continue;
        }
        const bool shared = un.e >= args.E;
        const int ecoord = shared ? un.e - args.E : un.e;
        const CUtensorMap* mA = un.down ? (shared ? &mDnS : &mDnR) : (shared ? &mGuS : &mGuR);
        const CUtensorMap* mB = un.down ? &mAct : (shared ? &mXs : &mXr);
        const int box = un.down ? args.box_act : (shared ? args.box_xs : args.box_xr);
        const int brow0 = un.down ? un.arow : un.xrow;
        const int nbox = cdiv(un.nrows, box);
        const int nst = un.down ? args.kc_dn : args.kc_gu;
        const int arow = un.down ? un.mb * 2 * kBM : un.mb * kBM;
        const uint32_t bytes = C::kABytes + nbox * box * kBK * 2;
        bool ok = true;
        auto load_b = [&](int st, int kc) {
          uint8_t* bt = tiles + st * C::kStageBytes + C::kABytes;
          for (int b = 0; b < nbox; ++b) tma_load_2d(bt + b * box * kBK * 2, mB, &full[st], kc * kBK, brow0 + b * box);
        };
        // weights of the first stages go out before the activations are known to be ready
        const int npre = un.down ? min(C::kStages, nst) : 0;
        const int st0 = stage;
        for (int kc = 0; kc < nst && ok; ++kc) {
          if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
            record_error(kErrTimeout, 131);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = tiles + stage * C::kStageBytes;
          if (pre_unit && kc < npre0) {  // weights in flight since before the wait
            mbar_arrive_expect_tx(&full[stage], bytes - C::kABytes);
          } else {
            mbar_arrive_expect_tx(&full[stage], bytes);
            if (un.down)
              tma_load_3d_hint(st, mA, &full[stage], kc * kBK, arow, ecoord, pol_w);
            else
              tma_load_4d_hint(st, mA, &full[stage], kc * kBK, arow, 0, ecoord, pol_w);
          }
          if (kc >= npre) load_b(stage, kc);
          if (want_ticket && kc + 1 >= npre0) {
            next_u = tbase + atomicAdd(ticket, 1);
            want_ticket = false;
          }
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
            for (int j = 0; j < npre; ++j) load_b((st0 + j) % C::kStages, j);
          }
          next_stage();
        }
        if (!ok) break;
      }
      if (pre_pending) {  // aborted before the first unit: complete its armed stages
        for (int kc = 0; kc < npre0; ++kc) {
          mbar_arrive(&full[kc]);
          issued |= 1u << kc;
          last_par &= ~(1u << kc);
        }
      }
      // every issued copy has landed before the CTA may exit
      for (int s = 0; s < C::kStages; ++s)
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
        FgUnit un;
        if (!decode(u, un, 148)) break;
        if (un.nrows == 0) {  // the pre-armed unit of an unused expert: release its stages
          bool ok = true;
          for (int kc = 0; kc < npre0; ++kc) {
            if (!mbar_wait(&full[stage], phase, limit)) {
              record_error(kErrTimeout, 138);
              *abort_flag = 1;
              ok = false;
              break;
            }
            mbar_arrive(&empty[stage]);
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          continue;
        }
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
        const uint32_t d0 = tmem_base + ab * C::kAccCols;
        const uint32_t d1 = d0 + NMAX;
        const int nst = un.down ? args.kc_dn : args.kc_gu;
        bool ok = true;
        for (int kc = 0; kc < nst; ++kc) {
          if (!mbar_wait(&full[stage], phase, limit)) {
            record_error(kErrTimeout, 135);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(tiles + stage * C::kStageBytes);
          const uint64_t a0 = sw128_kmajor_desc(st);
          const uint64_t a1 = sw128_kmajor_desc(st + kFgTileBytes);
          const uint64_t b = sw128_kmajor_desc(st + C::kABytes);
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16) {
            const uint32_t acc = (kc | k16) != 0;
            umma_bf16(d0, a0 + 2 * k16, b + 2 * k16, idesc, acc);
            umma_bf16(d1, a1 + 2 * k16, b + 2 * k16, idesc, acc);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::kStages) {
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
      FgUnit un;
      if (!decode(u, un, 149)) break;
      if (un.nrows == 0 && u != first_u) continue;  // nothing was computed for it
      const int ab = lu & 1;
      const uint32_t ap = (lu >> 1) & 1;
      ++lu;
      if (!mbar_wait(&tfull[ab], ap, limit)) {
        record_error(kErrTimeout, 137);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      // the unit's rows lie inside the activation / output buffers: routed rows, then S x T shared rows
      const bool rows_ok = VG_IN_BOUNDS(un.arow >= 0 && un.arow + un.nrows <= rows_total, 404);
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + ab * C::kAccCols;
      if (un.down) {
        const int ld = args.mblk_dn * 2 * kBM;
        __nv_bfloat16* dst = args.out + (size_t)un.arow * ld + un.mb * 2 * kBM + row;
        for (int c0 = 0; c0 < un.nrows; c0 += 16) {
          uint32_t g[16], v[16];
          tmem_ld16(t0 + c0, g);
          tmem_ld16(t0 + NMAX + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (rows_ok && c0 + j < un.nrows) {
              dst[(size_t)(c0 + j) * ld] = __float2bfloat16_rn(__uint_as_float(g[j]));
              dst[(size_t)(c0 + j) * ld + kBM] = __float2bfloat16_rn(__uint_as_float(v[j]));
            }
          }
        }
      } else {
        const int ld = args.mblk_gu * kBM;
        __nv_bfloat16* dst = args.act + (size_t)un.arow * ld + un.mb * kBM + row;
        for (int c0 = 0; c0 < un.nrows; c0 += 16) {
          uint32_t g[16], v[16];
          tmem_ld16(t0 + c0, g);
          tmem_ld16(t0 + NMAX + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (rows_ok && c0 + j < un.nrows)
              dst[(size_t)(c0 + j) * ld] = __float2bfloat16_rn(silu(__uint_as_float(g[j])) * __uint_as_float(v[j]));
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
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace vg
