// Projection of the verifier attention (q/k/v and output) on tcgen05 tensor
// cores, as fp32 partial sums over 256-wide slices of the reduction:
//   part[s][r][n] = sum over k in [256 s, 256 s + 256) of x[r][k] W[n][k],
// x bf16 [R, K], W bf16 [N, K] (N a multiple of 128, K of 256). Readers sum the
// slices in s order and round once to bf16 (attention.cuh).
//
// One CTA per unit (128 weight rows, slice s, 128-row tile of x): grid
// (N / 128, K / 256, cdiv(R, 128)). The weights are the M = 128 operand and
// the rows of x the N operand (up to 128 per MMA, rounded to 16), so each
// weight byte is read once per row tile; the slice's four 64-wide k-chunks of
// both operands are requested at once by one thread (TMA, 128-byte swizzle)
// into four stages, and the accumulator (128 weight rows x N columns, fp32)
// lives in tensor memory. Four epilogue warps each store 32 weight rows for
// every row of x (consecutive lanes write consecutive n, 128-byte segments).
// Every wait is bounded: a timeout records VG_ERR_TIMEOUT and the CTA drains
// its copies before it exits.
#pragma once
#include "common.cuh"
#include "gemm_moe.cuh"

namespace vg {

constexpr int kPtK = 256;                      // reduction slice of one partial
constexpr int kPtChunks = kPtK / kBK;          // 4 k-chunks of 64
constexpr int kPtRows = 128;                   // rows of x per tile (MMA N at most)
constexpr int kPtWBytes = kBM * kBK * 2;       // 16 KB weight chunk
constexpr int kPtXBytes = kPtRows * kBK * 2;   // 16 KB x chunk (a box of up to 128 rows)
constexpr int kPtStageBytes = kPtWBytes + kPtXBytes;
constexpr int kPtSmemBytes = kPtChunks * kPtStageBytes + 1024;

__global__ void __launch_bounds__(192, 1) attn_proj_tc(const __grid_constant__ CUtensorMap mW,
                                                       const __grid_constant__ CUtensorMap mX, int R, int N,
                                                       int x_box_rows, float* __restrict__ part) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kPtChunks], mma_done;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = blockIdx.x, sl = blockIdx.y, rt = blockIdx.z;
  const int rows = min(kPtRows, R - rt * kPtRows);  // rows of x in this tile
  const int ncols = (rows + 15) / 16 * 16;          // MMA N
  const uint64_t limit = g_wait_timeout_ns;
  const uint32_t x_bytes = (uint32_t)x_box_rows * kBK * 2;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPtChunks; ++i) mbar_init(&full[i], 1);
    mbar_init(&mma_done, 1);
    fence_mbar_init();
    prefetch_tmap(&mW);
    prefetch_tmap(&mX);
    // the weights are immutable: requested before the wait for the previous kernel
    for (int c = 0; c < kPtChunks; ++c) {
      mbar_expect_tx(&full[c], kPtWBytes);
      tma_load_2d(smem + c * kPtStageBytes, &mW, &full[c], sl * kPtK + c * kBK, nb * kBM);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kPtRows);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  griddep_wait();  // x comes from the previous kernel
  if (threadIdx.x == 0) {
    for (int c = 0; c < kPtChunks; ++c) {
      mbar_arrive_expect_tx(&full[c], x_bytes);
      tma_load_2d(smem + c * kPtStageBytes + kPtWBytes, &mX, &full[c], sl * kPtK + c * kBK, rt * kPtRows);
    }
  }
  if (threadIdx.x == 32) {  // MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kBM, ncols);
    bool ok = true;
    for (int c = 0; c < kPtChunks && ok; ++c) {
      if (!mbar_wait(&full[c], 0, limit)) {
        record_error(kErrTimeout, 330);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t st = smem_u32(smem + c * kPtStageBytes);
      const uint64_t da = sw128_kmajor_desc(st), db = sw128_kmajor_desc(st + kPtWBytes);
#pragma unroll
      for (int k16 = 0; k16 < kBK / 16; ++k16) umma_bf16(tmem, da + 2 * k16, db + 2 * k16, idesc, (c | k16) != 0);
    }
    umma_commit(&mma_done);  // arrives once every MMA issued above has completed
  }
  if (warp >= 2) {
    const int q = warp & 3;
    const int n = nb * kBM + q * 32 + lane;  // the weight row this thread owns
    const bool ok = mbar_wait(&mma_done, 0, limit);
    if (!ok && lane == 0) record_error(kErrTimeout, 331);
    tc_fence_after();
    float* dst = part + ((size_t)sl * R + (size_t)rt * kPtRows) * N + n;
    for (int c0 = 0; ok && c0 < ncols; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c0 + j < rows) dst[(size_t)(c0 + j) * N] = __uint_as_float(v[j]);
    }
  }
  // every copy has landed before the CTA exits (also after a timeout)
  if (threadIdx.x == 0)
    for (int c = 0; c < kPtChunks; ++c) mbar_wait(&full[c], 0, limit);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPtRows);
  }
}

}  // namespace vg
