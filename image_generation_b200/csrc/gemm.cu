// tcgen05 GEMM for the DiT block linears: acc[m, n] = A[m, :] . W[n, :]
// (A bf16 [M, K] row-major, W bf16 [N, K] in nn.Linear layout, fp32 accumulate
// in tensor memory), with the block's epilogues fused:
//   QKV projection + RoPE on Q and K      (step a4)
//   out-projection / FFN2 + gated residual (steps a6, a9): x += gate * acc
//   FFN1 + GELU                            (step a8)
//
// Structure (one CTA per SM, persistent over output tiles of 128 x 256):
//   warp 0      TMA producer: A tile [128 x 64] and W tile [256 x 64] per
//               k-block, 128-byte swizzle, into a 4-stage shared-memory ring;
//   warp 1      MMA issuer: 4 x tcgen05.mma (M128 N256 K16) per k-block into
//               one of two TMEM accumulators (2 x 256 columns), commit frees
//               the ring slot, a final commit hands the tile to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes (one output row
//               per thread), fused math, direct global stores; then the
//               accumulator is released so the next tile's MMAs overlap.
#include "gemm_epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

using namespace gemm_detail;

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, false, false);

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_bf16_tcgen05(const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_b, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);

  __shared__ int aborted;
  if (grid_aborted(p.status, &aborted)) return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto FULL = [&](int s) { return bar0 + 8u * s; };
  auto EMPTY = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto TFULL = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto TEMPTY = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t DRAIN = bar0 + 8u * (2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL(a), 1);
      mbar_init(TEMPTY(a), 128);
    }
    mbar_init(DRAIN, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tma_a);
    tma_prefetch_desc(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int kblocks = p.k / BK;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(EMPTY(stage), phase ^ 1, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(FULL(stage), STAGE_BYTES);
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          tma_load_2d(sa, &tma_a, kb * BK, tm * BM, FULL(stage));
          tma_load_2d(sa + A_BYTES, &tma_b, kb * BK, tn * BN, FULL(stage));
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Before the CTA can exit, every load it issued must have landed.
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (--stage < 0) {
          stage = STAGES - 1;
          phase ^= 1;
        }
        mbar_wait(FULL(stage), phase, p.status, false);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(TEMPTY(acc), acc_phase ^ 1, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(FULL(stage), phase, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t da = desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t db = desc_sw128(sb + kk * 32, 16, 1024);
            umma_bf16(d, da, db, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(EMPTY(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(TFULL(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // Every MMA this thread issued completes before TMEM is released.
      umma_commit(DRAIN);
      mbar_wait(DRAIN, 0, p.status, false);
    }
  } else {
    const int sub = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = sub * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int tm, tn;
      tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
      const bool ok = mbar_wait(TFULL(acc), acc_phase, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(acc * BN);
      epilogue_tile<EPI, BN>(p, tbase, tm * BM + row_in_tile, tn * BN);
      tc_fence_before();
      mbar_arrive(TEMPTY(acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int EPI>
cudaError_t launch_one(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p, int grid,
                       cudaStream_t s) {
  static PerDevice smem_attr;
  cudaError_t e = set_smem_once(smem_attr, gemm_bf16_tcgen05<EPI>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  gemm_bf16_tcgen05<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(a, b, p);
  return cudaGetLastError();
}

}  // namespace

int gemm_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_gemm(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p,
                        int epilogue, int grid, cudaStream_t s) {
  switch (epilogue) {
    case kEpiStore:
      return launch_one<kEpiStore>(a, b, p, grid, s);
    case kEpiQkvRope:
      return launch_one<kEpiQkvRope>(a, b, p, grid, s);
    case kEpiGelu:
      return launch_one<kEpiGelu>(a, b, p, grid, s);
    case kEpiGatedResidual:
      return launch_one<kEpiGatedResidual>(a, b, p, grid, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace h3
