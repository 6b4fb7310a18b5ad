// MXFP8 block-scaled tcgen05 GEMM for the DiT block linears (step a11: the
// MXFP8 variant of a4, a6, a8, a9): acc[m, n] = sum_k A[m, k] W[n, k] with A
// and W in E4M3 and one E8M0 scale per 32 consecutive k for every row of
// each, fp32 accumulate in tensor memory; the same fused epilogues as the
// bf16 GEMM (RoPE on Q/K with a bf16 store, gated residual on the fp32
// stream, and GELU written back as MXFP8 for the next linear).
//
// Structure (one CTA per SM, persistent over 128 x 128 output tiles):
//   warp 0      TMA producer: A [128 x 128 B] and W [128 x 128 B] per k-block
//               (128-byte swizzle) plus the two 512-byte scale blocks of that
//               k-block (bulk copies), into a 6-stage shared-memory ring;
//   warp 1      MMA issuer: per k-block, tcgen05.cp moves the A and W scale
//               blocks into tensor memory (32x128b, copied to all four lane
//               quarters), then 4 x tcgen05.mma.kind::mxf8f6f4.block_scale
//               (M128 N128 K32) select scale byte kk of each 32-bit column;
//   warps 2..5  epilogue, as in the bf16 GEMM.
// Tiles of 128 columns keep each W tile on one 128-row scale block and leave
// tensor memory for two accumulators (2 x 128 columns) and the scale blocks of
// every stage (6 x 8 columns).
#include "gemm_epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

using namespace gemm_detail;

constexpr int BM = kGemmBM, BN = kGemmMxBN, BK = kGemmMxBK;
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int SF_BYTES = 512;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + 2 * SF_BYTES;  // 33 KiB, keeps 1 KiB alignment
constexpr int THREADS = 192;
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 2 * BN;  // scale blocks after the two accumulators

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_mxf8_tcgen05(const __grid_constant__ CUtensorMap tma_a,
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
          bulk_load(sa + A_BYTES + B_BYTES,
                    p.a_sf + (static_cast<size_t>(tm) * kblocks + kb) * SF_BYTES, SF_BYTES,
                    FULL(stage));
          bulk_load(sa + A_BYTES + B_BYTES + SF_BYTES,
                    p.b_sf + (static_cast<size_t>(tn) * kblocks + kb) * SF_BYTES, SF_BYTES,
                    FULL(stage));
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
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
          const uint32_t sfa_t = tmem + SF_COL0 + 8 * stage;
          const uint32_t sfb_t = sfa_t + 4;
          tmem_cp_sf(sfa_t, desc_sf_copy(sb + B_BYTES));
          tmem_cp_sf(sfb_t, desc_sf_copy(sb + B_BYTES + SF_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t da = desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t db = desc_sw128(sb + kk * 32, 16, 1024);
            umma_mxf8(d, da, db, idesc_mxf8(BM, BN, kk), sfa_t, sfb_t, (kb | kk) != 0 ? 1u : 0u);
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
      umma_commit(DRAIN);
      mbar_wait(DRAIN, 0, p.status, false);
    }
  } else {
    const int sub = warp & 3;
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
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_mxf8_tcgen05<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  gemm_mxf8_tcgen05<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(a, b, p);
  return cudaGetLastError();
}

// One thread per block of 32 consecutive elements of a row: bf16 in,
// E4M3 + E8M0 scale out.
__global__ void mx_quantize_kernel(const uint16_t *__restrict__ src, long long ld, int rows, int k,
                                   uint8_t *__restrict__ dst, uint8_t *__restrict__ sf) {
  const int blocks_per_row = k / 32;
  const long long total = static_cast<long long>(rows) * blocks_per_row;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(i / blocks_per_row);
    const int blk = static_cast<int>(i - static_cast<long long>(row) * blocks_per_row);
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src + row * ld + 32 * blk);
    float v[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 w = __ldg(s4 + q);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * q + 2 * j] = __uint_as_float(ww[j] << 16);
        v[8 * q + 2 * j + 1] = __uint_as_float(ww[j] & 0xffff0000u);
      }
    }
    uint32_t qv[8];
    const uint32_t sb = mx_quant32(v, qv);
    uint8_t *d = dst + static_cast<size_t>(row) * k + 32 * blk;
    st_global_v4(d, qv[0], qv[1], qv[2], qv[3]);
    st_global_v4(d + 16, qv[4], qv[5], qv[6], qv[7]);
    sf[mx_sf_offset(row, blk, k / 128)] = static_cast<uint8_t>(sb);
  }
}

}  // namespace

cudaError_t launch_gemm_mx(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p,
                           int epilogue, int grid, cudaStream_t s) {
  switch (epilogue) {
    case kEpiQkvRope:
      return launch_one<kEpiQkvRope>(a, b, p, grid, s);
    case kEpiGatedResidual:
      return launch_one<kEpiGatedResidual>(a, b, p, grid, s);
    case kEpiGeluMx:
      return launch_one<kEpiGeluMx>(a, b, p, grid, s);
    case kEpiStore:
      return launch_one<kEpiStore>(a, b, p, grid, s);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_mx_quantize(const void *src, long long ld, int rows, int k, uint8_t *dst,
                               uint8_t *sf, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const long long total = static_cast<long long>(rows) * (k / 32);
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 148LL * 16 ? want : 148LL * 16);
  mx_quantize_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(src), ld, rows, k, dst, sf);
  return cudaGetLastError();
}

}  // namespace h3
