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
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int GROUP_M = 16;
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, false, false);

// Grouped raster: GROUP_M row-tiles sweep all column tiles together so that
// the CTAs running at once share A and W tiles in L2.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int &tm, int &tn) {
  const int group = GROUP_M * tiles_n;
  const int g = t / group;
  const int first = g * GROUP_M;
  const int gm = min(GROUP_M, tiles_m - first);
  const int local = t - g * group;
  tm = first + local % gm;
  tn = local / gm;
}

__device__ __forceinline__ float gelu_f(float x, int tanh_form) {
  if (tanh_form) {
    const float u = 0.7978845608028654f * (x + 0.044715f * x * x * x);
    return 0.5f * x * (1.0f + tanhf(u));
  }
  return 0.5f * x * (1.0f + erff(x * 0.7071067811865476f));
}

// Store `W` consecutive fp32 values as bf16 (W multiple of 8, 16-byte aligned).
template <int W>
__device__ __forceinline__ void store_bf16_row(void *dst, const float *v) {
#pragma unroll
  for (int q = 0; q < W / 8; ++q) {
    st_global_v4(static_cast<uint16_t *>(dst) + 8 * q, pack_bf16x2(v[8 * q + 0], v[8 * q + 1]),
                 pack_bf16x2(v[8 * q + 2], v[8 * q + 3]), pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                 pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
  }
}

// One rotary unit: 2*S accumulator columns holding S rotation pairs (j, S + j).
template <int S>
__device__ __forceinline__ void rope_unit(const GemmParams &p, uint32_t taddr, int row, int col,
                                          int pair_base, bool row_ok) {
  float v[2 * S];
  {
    uint32_t r[32];
    tmem_ld32(taddr, r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  }
  if constexpr (S == 24) {
    uint32_t r[16];
    tmem_ld16(taddr + 32, r);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[32 + i] = __uint_as_float(r[i]);
  }
  if (!row_ok) return;
  const float4 *cs = reinterpret_cast<const float4 *>(
      p.rope + (static_cast<size_t>(row) * (p.head_dim / 2) + pair_base) * 2);
#pragma unroll
  for (int j = 0; j < S; j += 2) {
    const float4 t = __ldg(cs + j / 2);  // cos_j, sin_j, cos_j+1, sin_j+1
    const float a0 = v[j], b0 = v[S + j], a1 = v[j + 1], b1 = v[S + j + 1];
    v[j] = a0 * t.x - b0 * t.y;
    v[S + j] = b0 * t.x + a0 * t.y;
    v[j + 1] = a1 * t.z - b1 * t.w;
    v[S + j + 1] = b1 * t.z + a1 * t.w;
  }
  store_bf16_row<2 * S>(static_cast<uint16_t *>(p.out) + static_cast<size_t>(row) * p.ldo + col, v);
}

template <int EPI>
__device__ __forceinline__ void plain_chunk(const GemmParams &p, uint32_t taddr, int row, int col,
                                            bool row_ok) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  if (!row_ok) return;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if constexpr (EPI == kEpiGatedResidual) {
    float4 *x = reinterpret_cast<float4 *>(static_cast<float *>(p.out) +
                                           static_cast<size_t>(row) * p.ldo + col);
    const float4 *g = reinterpret_cast<const float4 *>(p.gate + col);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 a = x[q];
      const float4 gg = __ldg(g + q);
      a.x = fmaf(gg.x, v[4 * q + 0], a.x);
      a.y = fmaf(gg.y, v[4 * q + 1], a.y);
      a.z = fmaf(gg.z, v[4 * q + 2], a.z);
      a.w = fmaf(gg.w, v[4 * q + 3], a.w);
      x[q] = a;
    }
  } else {
    if constexpr (EPI == kEpiGelu) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = gelu_f(v[i], p.gelu_tanh);
    }
    store_bf16_row<32>(static_cast<uint16_t *>(p.out) + static_cast<size_t>(row) * p.ldo + col, v);
  }
}

template <int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmParams &p, uint32_t tbase, int row,
                                              int col_tile) {
  const bool row_ok = row < p.m;
  if constexpr (EPI == kEpiQkvRope) {
    int c = 0;
    while (c < BN) {
      const int col = col_tile + c;
      if (col >= p.n) break;
      if (col < p.rope_cols) {
        const int h_off = col % p.head_dim;
        int s, pb;
        if (h_off == 0) {
          s = p.sec[0];
          pb = 0;
        } else if (h_off == 2 * p.sec[0]) {
          s = p.sec[1];
          pb = p.sec[0];
        } else {
          s = p.sec[2];
          pb = p.sec[0] + p.sec[1];
        }
        if (s == 16) {
          rope_unit<16>(p, tbase + c, row, col, pb, row_ok);
          c += 32;
        } else {
          rope_unit<24>(p, tbase + c, row, col, pb, row_ok);
          c += 48;
        }
      } else {
        plain_chunk<kEpiStore>(p, tbase + c, row, col, row_ok);
        c += 32;
      }
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      const int col = col_tile + c;
      if (col >= p.n) break;
      plain_chunk<EPI>(p, tbase + c, row, col, row_ok);
    }
  }
}

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
      epilogue_tile<EPI>(p, tbase, tm * BM + row_in_tile, tn * BN);
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
    cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
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
