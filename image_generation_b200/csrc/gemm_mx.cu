// MXFP8 block-scaled tcgen05 GEMM for the DiT block linears (step a11: the
// MXFP8 variant of a4, a6, a8, a9): acc[m, n] = sum_k A[m, k] W[n, k] with A
// and W in E4M3 and one E8M0 scale per 32 consecutive k for every row of
// each, fp32 accumulate in tensor memory; the same fused epilogues as the
// bf16 GEMM (RoPE on Q/K with a bf16 store, gated residual on the fp32
// stream, and GELU written back as MXFP8 for the next linear).
//
// Structure (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: A [128 x 128 B] and W [BN x 128 B] per k-block
//               (128-byte swizzle) plus that k-block's scale blocks (bulk
//               copies), into a ring of shared-memory stages;
//   warp 1      MMA issuer: per k-block, tcgen05.cp moves the A and W scale
//               blocks into tensor memory (32x128b, copied to all four lane
//               quarters), then 4 x tcgen05.mma.kind::mxf8f6f4.block_scale
//               (M128 N=BN K32) select scale byte kk of each 32-bit column;
//   warps 2..5  epilogue, as in the bf16 GEMM.
// Two tile widths:
//   BN 128  W scales in the standard layout (one 512-byte block per 128 rows
//           and k-block); two accumulators (2 x 128 columns) and the scales
//           of six stages (6 x 8 columns) in tensor memory;
//   BN 224  W scales repacked per tile (two 512-byte blocks covering rows
//           224 t .. 224 t + 255 per k-block, made once when the weights are
//           quantized); two accumulators (2 x 224 columns) and the scales of
//           four stages (4 x 12 columns). An M128 N224 K32 MMA does 1.75x the
//           work of an N128 one for about 1.3x its issue cost.
#include "gemm_epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

using namespace gemm_detail;

constexpr int BM = kGemmBM, BK = kGemmMxBK;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SF_BYTES = 512;

template <int BN>
struct MxTile {
  static constexpr bool WIDE = BN != kGemmMxBN;
  static constexpr int STAGES = WIDE ? 4 : 6;
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int SFB_BYTES = WIDE ? 2 * SF_BYTES : SF_BYTES;
  // stages keep 1 KiB alignment (128-byte swizzle atoms)
  static constexpr int LOAD_BYTES = A_BYTES + B_BYTES + SF_BYTES + SFB_BYTES;  // per k-block
  static constexpr int STAGE_BYTES = (LOAD_BYTES + 1023) / 1024 * 1024;
  static constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + NUM_BARS * 8 + 16;
  static constexpr uint32_t SF_COL0 = 2 * BN;        // scales after the two accumulators
  static constexpr uint32_t SF_COLS = WIDE ? 12 : 8;  // per stage: A (4) then W (4 or 8)
};
static_assert(MxTile<kGemmMxWideBN>::SF_COL0 + 4 * 12 <= TMEM_COLS, "TMEM budget");
static_assert(MxTile<kGemmMxWideBN>::SMEM_BYTES <= 227 * 1024, "shared memory budget");

template <int EPI, int BN>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_mxf8_tcgen05(const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_b, const GemmParams p) {
  using T = MxTile<BN>;
  constexpr int STAGES = T::STAGES, A_BYTES = T::A_BYTES, B_BYTES = T::B_BYTES;
  constexpr int STAGE_BYTES = T::STAGE_BYTES, NUM_BARS = T::NUM_BARS;
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
          mbar_arrive_expect_tx(FULL(stage), T::LOAD_BYTES);
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          tma_load_2d(sa, &tma_a, kb * BK, tm * BM, FULL(stage));
          tma_load_2d(sa + A_BYTES, &tma_b, kb * BK, tn * BN, FULL(stage));
          bulk_load(sa + A_BYTES + B_BYTES,
                    p.a_sf + (static_cast<size_t>(tm) * kblocks + kb) * SF_BYTES, SF_BYTES,
                    FULL(stage));
          bulk_load(sa + A_BYTES + B_BYTES + SF_BYTES,
                    p.b_sf + (static_cast<size_t>(tn) * kblocks + kb) * T::SFB_BYTES, T::SFB_BYTES,
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
          const uint32_t sfa_t = tmem + T::SF_COL0 + T::SF_COLS * stage;
          const uint32_t sfb_t = sfa_t + 4;
          tmem_cp_sf(sfa_t, desc_sf_copy(sb + B_BYTES));
          tmem_cp_sf(sfb_t, desc_sf_copy(sb + B_BYTES + SF_BYTES));
          if (T::WIDE) tmem_cp_sf(sfb_t + 4, desc_sf_copy(sb + B_BYTES + 2 * SF_BYTES));
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

template <int EPI, int BN>
cudaError_t launch_one(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p, int grid,
                       cudaStream_t s) {
  static PerDevice smem_attr;
  cudaError_t e = set_smem_once(smem_attr, gemm_mxf8_tcgen05<EPI, BN>, MxTile<BN>::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  gemm_mxf8_tcgen05<EPI, BN><<<grid, THREADS, MxTile<BN>::SMEM_BYTES, s>>>(a, b, p);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_bn(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p, int grid,
                      bool wide, cudaStream_t s) {
  return wide ? launch_one<EPI, kGemmMxWideBN>(a, b, p, grid, s)
              : launch_one<EPI, kGemmMxBN>(a, b, p, grid, s);
}

// Repack W scales (standard layout) for 224-row tiles: byte i of the output
// belongs to tile i / (kb * 1024), k-block (i / 1024) % kb, half (i / 512) % 2
// and, inside that 512-byte block, row r and scale j of the standard in-block
// order; rows past n read as zero.
__global__ void mx_tile_sf_kernel(const uint8_t *__restrict__ sf, int n, int k,
                                  uint8_t *__restrict__ tiled, long long total) {
  const int kblocks = k / 128;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long blk = i / 512;
    const int within = static_cast<int>(i % 512);
    const int half = static_cast<int>(blk % 2);
    const int kb = static_cast<int>((blk / 2) % kblocks);
    const long long tile = blk / 2 / kblocks;
    const int r = within / 16 + 32 * ((within % 16) / 4);
    const int j = within % 4;
    const long long row = tile * kGemmMxWideBN + 128 * half + r;
    tiled[i] = row < n ? sf[mx_sf_offset(static_cast<int>(row), 4 * kb + j, kblocks)] : 0;
  }
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
                           int epilogue, int grid, bool wide, cudaStream_t s) {
  switch (epilogue) {
    case kEpiQkvRope:
      return launch_bn<kEpiQkvRope>(a, b, p, grid, wide, s);
    case kEpiGatedResidual:
      return launch_bn<kEpiGatedResidual>(a, b, p, grid, wide, s);
    case kEpiGeluMx:
      return launch_bn<kEpiGeluMx>(a, b, p, grid, wide, s);
    case kEpiStore:
      return launch_bn<kEpiStore>(a, b, p, grid, wide, s);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_mx_tile_sf(const uint8_t *sf, int n, int k, uint8_t *tiled, cudaStream_t s) {
  const long long total = static_cast<long long>(mx_sf_tiled_bytes(n, k));
  if (total <= 0) return cudaSuccess;
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 148LL * 16 ? want : 148LL * 16);
  mx_tile_sf_kernel<<<grid, 256, 0, s>>>(sf, n, k, tiled, total);
  return cudaGetLastError();
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
