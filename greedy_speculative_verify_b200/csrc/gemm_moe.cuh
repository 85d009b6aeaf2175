// Grouped expert GEMMs of the MoE layer on tcgen05 tensor cores.
//
// Orientation ("swap AB"): the weight rows are the M = 128 operand (A) and the
// tokens routed to an expert are the N operand (B), so one tile streams a
// 128-row slab of one expert's weights exactly once for all of that expert's
// tokens (up to 128 per tile). At decode sizes (about 12 tokens per expert)
// this is a weight-streaming GEMM bound by HBM; at prefill sizes (thousands of
// tokens per expert) the same kernel runs full 128 x 128 tiles and is bound by
// the tensor pipe.
//
//   gate/up mode: D_gate = W_gate[rows] * X^T, D_up = W_up[rows] * X^T,
//                 act[token, row] = bf16(silu(D_gate) * D_up)
//   down mode:    D = W_down[rows] * act^T, out[token, row] = bf16(D)
//
// The two shared experts ride in the same launch as experts E and E+1 with all
// T tokens. Work unit = (expert, 128-token block, 128-row block); units are
// enumerated on the device from the routing offsets, so nothing returns to the
// host. Each CTA is persistent and walks units u = blockIdx.x + i * gridDim.x.
//
// Warp roles (192 threads): warp 0 issues TMA loads into a multi-stage shared
// memory ring; warp 1 owns the tensor-memory allocation and one of its threads
// issues tcgen05.mma; warps 2-5 drain the double-buffered TMEM accumulator
// (each warp reads its own 32-lane quarter) and store the epilogue. Every wait
// is bounded; a timeout records VG_ERR_TIMEOUT, the CTA drains its in-flight
// copies and MMAs (bounded again), frees its tensor memory and exits.
#pragma once
#include "common.cuh"

namespace vg {

constexpr int kBM = 128;       // weight rows per tile
constexpr int kBK = 64;        // K elements per stage: one 128-byte swizzle row
constexpr int kNMax = 128;     // tokens per tile
constexpr int kBoxRows = 16;   // token rows per TMA box of the B operand
constexpr int kMaxExperts = 72;

template <bool GATEUP>
struct GemmCfg {
  static constexpr int kStages = GATEUP ? 4 : 6;
  static constexpr int kABytes = kBM * kBK * 2;  // 16 KB
  static constexpr int kNumA = GATEUP ? 2 : 1;
  static constexpr int kBBytes = kNMax * kBK * 2;  // 16 KB
  static constexpr int kStageBytes = kNumA * kABytes + kBBytes;
  static constexpr int kAccCols = GATEUP ? 2 * kNMax : kNMax;  // one accumulator buffer
  static constexpr int kTmemCols = 2 * kAccCols;                // double buffered: 512 / 256
  static constexpr int kAuxBytes = 2048;
  static constexpr int kSmemBytes = kStages * kStageBytes + kAuxBytes + 1024;  // + alignment slack
};

struct GemmArgs {
  const int32_t* offsets;   // [E+1] routed segment offsets in permutation order (device)
  int32_t T, E, S;
  int32_t n_mblk;           // 128-row blocks of the output width
  int32_t k_chunks;         // reduction length / 64
  int32_t a_up_row;         // gate/up: first up row inside an expert's A rows (= I)
  int32_t b_shared_base;    // B row of shared expert 0, token 0
  int32_t b_shared_stride;  // B rows between shared experts
  int32_t out_shared_base;  // output row of shared expert 0, token 0 (= k*T)
  int32_t out_ld;           // output row length (elements)
  int32_t b_box_r;          // rows per B box of the routed / shared map (16, or the
  int32_t b_box_s;          //   tensor's row count rounded up to 8 when it is smaller)
  __nv_bfloat16* out;
};

struct Unit {
  int e, mb, b_row, out_row, nrows;
};

struct Sched {
  int b_start[kMaxExperts];
  int out_start[kMaxExperts];
  int n[kMaxExperts];
  int pref[kMaxExperts + 1];
};

__device__ __forceinline__ Unit decode_unit(int u, const Sched& s, int n_exp, int n_mblk) {
  const int tile = u / n_mblk;
  Unit un;
  un.mb = u - tile * n_mblk;
  int e = 0;
  while (e + 1 < n_exp && s.pref[e + 1] <= tile) ++e;
  const int nb = tile - s.pref[e];
  un.e = e;
  un.b_row = s.b_start[e] + nb * kNMax;
  un.out_row = s.out_start[e] + nb * kNMax;
  un.nrows = min(kNMax, s.n[e] - nb * kNMax);
  return un;
}

template <bool GATEUP>
__global__ void __launch_bounds__(192, 1)
    moe_grouped_gemm(const __grid_constant__ CUtensorMap mapA_r, const __grid_constant__ CUtensorMap mapA_s,
                     const __grid_constant__ CUtensorMap mapB_r, const __grid_constant__ CUtensorMap mapB_s,
                     const GemmArgs args) {
  using C = GemmCfg<GATEUP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* aux = smem + C::kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  Sched* sch = reinterpret_cast<Sched*>(aux + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_exp = args.E + args.S;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
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
    prefetch_tmap(&mapA_r);
    prefetch_tmap(&mapA_s);
    prefetch_tmap(&mapB_r);
    prefetch_tmap(&mapB_s);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) {
    for (int e = lane; e < n_exp; e += 32) {
      if (e < args.E) {
        const int o0 = args.offsets[e], o1 = args.offsets[e + 1];
        sch->b_start[e] = o0;
        sch->out_start[e] = o0;
        sch->n[e] = o1 - o0;
      } else {
        const int s = e - args.E;
        sch->b_start[e] = args.b_shared_base + s * args.b_shared_stride;
        sch->out_start[e] = args.out_shared_base + s * args.T;
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
  const int total = sch->pref[n_exp] * args.n_mblk;
  const uint64_t limit = g_wait_timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint64_t pol_w = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
        const Unit un = decode_unit(u, *sch, n_exp, args.n_mblk);
        const bool shared = un.e >= args.E;
        const CUtensorMap* mA = shared ? &mapA_s : &mapA_r;
        const CUtensorMap* mB = shared ? &mapB_s : &mapB_r;
        const int ecoord = shared ? un.e - args.E : un.e;
        const int box = shared ? args.b_box_s : args.b_box_r;
        const int nbox = cdiv(un.nrows, box);
        const uint32_t bytes = C::kNumA * C::kABytes + nbox * box * kBK * 2;
        for (int kc = 0; kc < args.k_chunks; ++kc) {
          if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
            record_error(kErrTimeout, GATEUP ? 101 : 111);
            *abort_flag = 1;
            break;
          }
          uint8_t* st = tiles + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          const int kx = kc * kBK;
          tma_load_3d_hint(st, mA, &full[stage], kx, un.mb * kBM, ecoord, pol_w);
          if (GATEUP) tma_load_3d_hint(st + C::kABytes, mA, &full[stage], kx, args.a_up_row + un.mb * kBM, ecoord, pol_w);
          uint8_t* bt = st + C::kNumA * C::kABytes;
          for (int j = 0; j < nbox; ++j) tma_load_2d(bt + j * box * kBK * 2, mB, &full[stage], kx, un.b_row + j * box);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every issued copy has landed before the CTA may exit
      for (int s = 0; s < C::kStages; ++s)
        if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int lu = 0;
      for (int u = blockIdx.x; u < total; u += gridDim.x, ++lu) {
        if (*abort_flag) break;
        const Unit un = decode_unit(u, *sch, n_exp, args.n_mblk);
        const int ab = lu & 1;
        const uint32_t ap = (lu >> 1) & 1;
        if (!mbar_wait(&tempty[ab], ap ^ 1, limit)) {
          record_error(kErrTimeout, GATEUP ? 102 : 112);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const int N = cdiv(un.nrows, 16) * 16;
        const uint32_t idesc = idesc_bf16_f32(kBM, N);
        const uint32_t d0 = tmem_base + ab * C::kAccCols;
        const uint32_t d1 = d0 + kNMax;
        bool ok = true;
        for (int kc = 0; kc < args.k_chunks; ++kc) {
          if (!mbar_wait(&full[stage], phase, limit)) {
            record_error(kErrTimeout, GATEUP ? 103 : 113);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(tiles + stage * C::kStageBytes);
          const uint64_t a0 = sw128_kmajor_desc(st);
          const uint64_t a1 = sw128_kmajor_desc(st + C::kABytes);
          const uint64_t b = sw128_kmajor_desc(st + C::kNumA * C::kABytes);
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16) {
            const uint32_t acc = (kc | k16) != 0;
            umma_bf16(d0, a0 + 2 * k16, b + 2 * k16, idesc, acc);
            if (GATEUP) umma_bf16(d1, a1 + 2 * k16, b + 2 * k16, idesc, acc);
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
    int lu = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++lu) {
      if (*abort_flag) break;
      const Unit un = decode_unit(u, *sch, n_exp, args.n_mblk);
      const int ab = lu & 1;
      const uint32_t ap = (lu >> 1) & 1;
      if (!mbar_wait(&tfull[ab], ap, limit)) {
        record_error(kErrTimeout, GATEUP ? 104 : 114);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + ab * C::kAccCols;
      __nv_bfloat16* out = args.out + (size_t)un.out_row * args.out_ld + un.mb * kBM + row;
      for (int c0 = 0; c0 < un.nrows; c0 += 16) {
        uint32_t g[16], v[16];
        tmem_ld16(t0 + c0, g);
        if (GATEUP) tmem_ld16(t0 + kNMax + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (c0 + j < un.nrows) {
            float r;
            if (GATEUP)
              r = silu(__uint_as_float(g[j])) * __uint_as_float(v[j]);
            else
              r = __uint_as_float(g[j]);
            out[(size_t)(c0 + j) * args.out_ld] = __float2bfloat16_rn(r);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
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
