// tcgen05 GEMM over CTA pairs for the DiT block linears: the same product and
// fused epilogues as the one-CTA kernel (acc[m, n] = A[m, :] . W[n, :], bf16
// operands, fp32 accumulate), on output tiles of 256 x 256 computed by a
// cluster of two CTAs with tcgen05.mma.cta_group::2 (M256 N256 K16).
//
// Each CTA of the pair loads its own 128 rows of A and its own 128 rows of W
// (half of the tile's 256 output columns); the pair MMA reads both halves of
// W from the two CTAs' shared memory and writes rows 0..127 of the tile into
// the first CTA's TMEM and rows 128..255 into the second's. Per SM this moves
// 32 KB from L2 per 64-deep k-block instead of 48 KB for the same MACs, which
// is what bounds the one-CTA kernel.
//
// Roles (both CTAs, 192 threads):
//   warp 0      TMA producer for this CTA's A and W halves, 6-stage ring;
//               the loads complete on the first CTA's FULL barrier, which
//               takes one arrival (with its byte count) from each producer;
//   warp 1      TMEM allocation for the pair; in the first CTA only, the MMA
//               issuer: 4 pair MMAs per k-block into one of two 256-column
//               accumulators; each commit arrives on both CTAs' EMPTY / TFULL;
//   warps 2..5  epilogue of this CTA's 128 rows, unchanged from the one-CTA
//   (..9)       kernel; every thread then arrives on the first CTA's TEMPTY.
//               With PARTS = 2 (launches whose K is at most 2048, where a
//               tile's mainloop is short next to a GELU or residual epilogue),
//               eight warps share it, two per TMEM lane quarter, each taking
//               every other 32-column unit of the tile.
//
// The decision to skip work after an earlier failure is taken for the pair
// as a whole, and a CTA leaves only after both producers' loads have landed,
// so no copy or remote arrival can reach a CTA that has exited.
#include "gemm_epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

using namespace gemm_detail;

constexpr int BM = 128;  // rows per CTA (256 per pair)
constexpr int BN = 256;  // columns per tile (128 rows of W per CTA)
constexpr int BK = kGemmBK;
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = (BN / 2) * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
template <int PARTS>
constexpr int threads_for() {
  return 64 + 128 * PARTS;
}
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, BN, false, false);
constexpr uint16_t kBothCtas = 0x3, kFirstCta = 0x1;

template <int EPI, int PARTS>
__global__ void __launch_bounds__(threads_for<PARTS>(), 1)
    gemm_bf16_pair(const __grid_constant__ CUtensorMap tma_a,
                   const __grid_constant__ CUtensorMap tma_b, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
  __shared__ int entry_status;
  __shared__ int loads_issued;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto FULL = [&](int s) { return bar0 + 8u * s; };
  auto EMPTY = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto TFULL = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto TEMPTY = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t DRAIN = bar0 + 8u * (2 * STAGES + 4);

  if (threadIdx.x == 0) {
    entry_status = *reinterpret_cast<const volatile int *>(p.status);
    loads_issued = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(FULL(s), 2);  // one arrival per producer of the pair
      mbar_init(EMPTY(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL(a), 1);
      mbar_init(TEMPTY(a), 2 * 128 * PARTS);  // both CTAs' epilogue threads
    }
    mbar_init(DRAIN, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tma_a);
    tma_prefetch_desc(&tma_b);
  }
  cluster_sync();  // barriers initialised and entry status visible pair-wide
  const int peer_status =
      static_cast<int>(ld_shared_cluster_u32(map_to_cta(smem_u32(&entry_status), peer)));
  const bool skip = (entry_status | peer_status) != 0;
  if (!skip && warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // the peer has read our status word; TMEM allocated in both
  if (skip) return;
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int kblocks = p.k / BK;
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full_leader = map_to_cta(FULL(0), 0);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += pairs) {
        int tm, tn;
        tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
        const int row_a = tm * 2 * BM + static_cast<int>(rank) * BM;
        const int row_b = tn * BN + static_cast<int>(rank) * (BN / 2);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(EMPTY(stage), phase ^ 1, p.status)) {
            ok = false;
            break;
          }
          const uint32_t full = full_leader + 8u * stage;
          if (leader)
            mbar_arrive_expect_tx(FULL(stage), STAGE_BYTES);
          else
            mbar_arrive_expect_tx_cluster(full, STAGE_BYTES);
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          tma_load_2d_pair(sa, &tma_a, kb * BK, row_a, full);
          tma_load_2d_pair(sa + A_BYTES, &tma_b, kb * BK, row_b, full);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      loads_issued = issued;
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += pairs) {
        if (!mbar_wait_cluster(TEMPTY(acc), acc_phase ^ 1, p.status)) {
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
            umma_bf16_pair(d, da, db, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(EMPTY(stage), kBothCtas);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(TFULL(acc), kBothCtas);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // Every pair MMA (and the arrivals its commits make) completes before
      // either CTA may release TMEM or exit.
      umma_commit_pair(DRAIN, kFirstCta);
      mbar_wait(DRAIN, 0, p.status, false);
    }
  } else {
    const int sub = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = sub * 32 + lane;
    const uint32_t tempty_leader = map_to_cta(TEMPTY(0), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < num_tiles; t += pairs) {
      int tm, tn;
      tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
      const bool ok = mbar_wait(TFULL(acc), acc_phase, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(acc * BN);
      epilogue_tile<EPI, BN>(p, tbase, tm * 2 * BM + static_cast<int>(rank) * BM + row_in_tile,
                             tn * BN, (warp - 2) >> 2, PARTS);
      tc_fence_before();
      if (leader)
        mbar_arrive(TEMPTY(acc));
      else
        mbar_arrive_cluster(tempty_leader + 8u * acc);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  // Drain: every load either producer issued must land before its CTA exits.
  // A stage's FULL phase completes once both producers arrived and all bytes
  // landed; where one producer stopped early (after a failure elsewhere) the
  // first CTA arrives in its place, then waits out the last STAGES loads.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (leader && threadIdx.x == 0) {
    const int mine = loads_issued;
    const int theirs =
        static_cast<int>(ld_shared_cluster_u32(map_to_cta(smem_u32(&loads_issued), peer)));
    const int lo = mine < theirs ? mine : theirs;
    const int hi = mine < theirs ? theirs : mine;
    for (int i = lo; i < hi; ++i) mbar_arrive(FULL(i % STAGES));
    for (int i = hi - STAGES > 0 ? hi - STAGES : 0; i < hi; ++i)
      mbar_wait(FULL(i % STAGES), (i / STAGES) & 1, p.status, false);
  }
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

template <int EPI, int PARTS>
cudaError_t launch_one(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p, int grid,
                       cudaStream_t s) {
  static PerDevice smem_attr;
  cudaError_t e = set_smem_once(smem_attr, gemm_bf16_pair<EPI, PARTS>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(threads_for<PARTS>(), 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_bf16_pair<EPI, PARTS>, a, b, p);
}

// The epilogue on eight warps where the mainloop is short (K <= 2048).
template <int EPI>
cudaError_t launch_parts(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p, int grid,
                         cudaStream_t s) {
  return p.k <= 2048 ? launch_one<EPI, 2>(a, b, p, grid, s) : launch_one<EPI, 1>(a, b, p, grid, s);
}

template <int EPI>
int occupancy_clusters();

// Clusters that fit at once on the current device, found once per device (0
// when the kernel cannot be configured there).
template <int EPI>
int max_pairs_for() {
  static PerDevice pairs;
  int n = 0;
  if (per_device(pairs, [](int *v) {
        *v = 0;
        // both forms hold one CTA per SM (the same shared memory)
        if (cudaFuncSetAttribute(gemm_bf16_pair<EPI, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM_BYTES) != cudaSuccess) {
          cudaGetLastError();
          return cudaSuccess;
        }
        *v = occupancy_clusters<EPI>();
        return cudaSuccess;
      }, &n) != cudaSuccess)
    return 0;
  return n;
}

template <int EPI>
int occupancy_clusters() {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(threads_for<1>(), 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_bf16_pair<EPI, 1>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

}  // namespace

int gemm_pair_max_clusters(int epilogue) {
  switch (epilogue) {
    case kEpiStore:
      return max_pairs_for<kEpiStore>();
    case kEpiQkvRope:
      return max_pairs_for<kEpiQkvRope>();
    case kEpiGelu:
      return max_pairs_for<kEpiGelu>();
    case kEpiGatedResidual:
      return max_pairs_for<kEpiGatedResidual>();
    default:
      return 0;
  }
}

cudaError_t launch_gemm_pair(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p,
                             int epilogue, int grid, cudaStream_t s) {
  if (grid <= 0 || (grid & 1)) return cudaErrorInvalidValue;
  switch (epilogue) {
    case kEpiStore:
      return launch_parts<kEpiStore>(a, b, p, grid, s);
    case kEpiQkvRope:
      return launch_parts<kEpiQkvRope>(a, b, p, grid, s);
    case kEpiGelu:
      return launch_parts<kEpiGelu>(a, b, p, grid, s);
    case kEpiGatedResidual:
      return launch_parts<kEpiGatedResidual>(a, b, p, grid, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace h3
