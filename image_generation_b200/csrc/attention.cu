// Joint bidirectional attention on tcgen05 (step a5):
//   O_h = softmax(Q_h K_h^T / sqrt(d_h)) V_h over all tokens, no mask,
// for the single packed text+image stream.
//
// One CTA per (128-query tile, head); the KV sequence is walked in tiles of
// 128 with an online softmax:
//   warp 0      TMA: Q once; K and V tiles into a 2-stage ring. Every 128-row
//               tile is loaded as 64-column boxes (128-byte swizzle) of a 3-D
//               view [tokens, heads, d_h]; columns past d_h read as zero.
//   warp 1      MMA: S_j = Q K_j^T (M128 N128, K = d_h) into one of two TMEM
//               S buffers, then O += P_{j-1} V_{j-1} (M128 N = d_h, K128) with
//               P from shared memory (K-major) and V as an MN-major operand.
//   warps 2..5  softmax, one query row per thread: read S_j from TMEM, running
//               max in log2 units, p = 2^(s*scale*log2e - m), P as bf16 into
//               shared memory. O is rescaled in TMEM only when the running max
//               grows by more than 8 (a factor 256); otherwise the stale max is
//               kept, which leaves the final O / l unchanged.
// Tensor memory: S0 [0,128), S1 [128,256), O [256, 256 + d_h).
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int NS = 2;                       // K/V ring stages
constexpr uint32_t BOX = 128 * 128;         // one [128 rows x 64 bf16] swizzled box
constexpr uint32_t Q_BYTES = 2 * BOX;
constexpr uint32_t KV_BYTES = 2 * BOX;      // one K or V tile (d_h <= 128)
constexpr uint32_t STAGE_BYTES = 2 * KV_BYTES;
constexpr uint32_t P_BYTES = 2 * BOX;       // P [128 q x 128 kv] as two 64-kv boxes
constexpr int THREADS = 192;
constexpr int NUM_BARS = 1 + 2 * NS + 4 + 2 + 1;
constexpr int SMEM_BYTES = Q_BYTES + NS * STAGE_BYTES + P_BYTES + 1024 + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units

template <int DH>
__global__ void __launch_bounds__(THREADS, 1)
    attn_fwd_tcgen05(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const AttnParams p) {
  static_assert(DH == 96 || DH == 128, "head_dim");
  constexpr int DCH = (DH + 63) / 64;  // 64-column boxes per row
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV, false, false);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(BQ, DH, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + Q_BYTES;
  const uint32_t sP = sKV + NS * STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Q_BYTES + NS * STAGE_BYTES + P_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
  uint8_t *pP = smem + Q_BYTES + NS * STAGE_BYTES;

  const uint32_t b0 = smem_u32(bars);
  const uint32_t Q_FULL = b0;
  auto KV_FULL = [&](int s) { return b0 + 8u * (1 + s); };
  auto KV_EMPTY = [&](int s) { return b0 + 8u * (1 + NS + s); };
  auto S_FULL = [&](int b) { return b0 + 8u * (1 + 2 * NS + b); };
  auto S_EMPTY = [&](int b) { return b0 + 8u * (3 + 2 * NS + b); };
  const uint32_t P_FULL = b0 + 8u * (5 + 2 * NS);
  const uint32_t PV_DONE = b0 + 8u * (6 + 2 * NS);
  const uint32_t DRAIN = b0 + 8u * (7 + 2 * NS);

  __shared__ int aborted;
  if (grid_aborted(p.status, &aborted)) return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * BQ;
  const int nkv = p.tiles_kv;

  if (threadIdx.x == 0) {
    mbar_init(Q_FULL, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(KV_FULL(s), 1);
      mbar_init(KV_EMPTY(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(S_FULL(b), 1);
      mbar_init(S_EMPTY(b), 128);
    }
    mbar_init(P_FULL, 128);
    mbar_init(PV_DONE, 1);
    mbar_init(DRAIN, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(Q_FULL, DCH * BOX);
      for (int c = 0; c < DCH; ++c) tma_load_3d(sQ + c * BOX, &tq, 64 * c, head, q0, Q_FULL);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (!mbar_wait(KV_EMPTY(st), ph ^ 1, p.status)) break;
        mbar_arrive_expect_tx(KV_FULL(st), 2 * DCH * BOX);
        const uint32_t k_dst = sKV + st * STAGE_BYTES;
        const uint32_t v_dst = k_dst + KV_BYTES;
        for (int c = 0; c < DCH; ++c) {
          tma_load_3d(k_dst + c * BOX, &tk, 64 * c, head, j * BKV, KV_FULL(st));
          tma_load_3d(v_dst + c * BOX, &tv, 64 * c, head, j * BKV, KV_FULL(st));
        }
        issued = j + 1;
      }
      // Every load issued must land before the CTA exits.
      mbar_wait(Q_FULL, 0, p.status, false);
      for (int j = issued - 1; j >= 0 && j >= issued - NS; --j)
        mbar_wait(KV_FULL(j % NS), (j / NS) & 1, p.status, false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t tO = tmem + 256;
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(P_FULL, i & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t v_src = sKV + (i % NS) * STAGE_BYTES + KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t da = desc_sw128(sP + (kk / 4) * BOX + (kk % 4) * 32, 16, 1024);
          const uint64_t db = desc_sw128(v_src + kk * 16 * 128, BOX, 1024);
          umma_bf16(tO, da, db, IDESC_O, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(KV_EMPTY(i % NS));
        umma_commit(PV_DONE);
        return true;
      };
      bool ok = mbar_wait(Q_FULL, 0, p.status);
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % NS;
        if (!mbar_wait(KV_FULL(st), (j / NS) & 1, p.status)) {
          ok = false;
          break;
        }
        const int sb = j & 1;
        if (!mbar_wait(S_EMPTY(sb), ((j >> 1) & 1) ^ 1, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_src = sKV + st * STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk / 4) * BOX + (kk % 4) * 32;
          umma_bf16(tmem + 128 * sb, desc_sw128(sQ + off, 16, 1024),
                    desc_sw128(k_src + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(S_FULL(sb));
        if (j > 0 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) issue_pv(nkv - 1);
      umma_commit(DRAIN);
      mbar_wait(DRAIN, 0, p.status, false);
    }
  } else {
    // softmax warps: warp w reads TMEM lanes [32 (w % 4), +32), one query row each
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(sub * 32) << 16);
    const float sl2 = p.scale_log2;
    float m = 0.f, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      ok = mbar_wait(S_FULL(sb), (j >> 1) & 1, p.status);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tl + 128 * sb + 32 * c, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      mbar_arrive(S_EMPTY(sb));

      const int valid = p.n - j * BKV;
      if (valid < BKV) {
#pragma unroll
        for (int i = 0; i < BKV; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int i = 1; i < BKV; ++i) mx = fmaxf(mx, s[i]);
      mx *= sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m = mx;
      } else if (mx > m + RESCALE_THRESHOLD) {
        alpha = ex2_approx(m - mx);
        m = mx;
        rescale = true;
      }
      float sum = 0.f;
      uint32_t pk[BKV / 2];
#pragma unroll
      for (int i = 0; i < BKV; i += 2) {
        const float e0 = ex2_approx(fmaf(s[i], sl2, -m));
        const float e1 = ex2_approx(fmaf(s[i + 1], sl2, -m));
        sum += e0 + e1;
        pk[i / 2] = pack_bf16x2(e0, e1);
      }
      l = l * alpha + sum;

      if (j > 0) {
        // PV(j-1) must be done: it reads the P buffer and accumulates into O.
        ok = mbar_wait(PV_DONE, (j - 1) & 1, p.status);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tl + 256 + 32 * c, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tl + 256 + 32 * c, r);
          }
        }
      }
      // P row into the K-major 128-byte-swizzled layout the MMA reads:
      // kv chunk q (8 values, 16 bytes) of box q/8 sits at chunk (q%8) ^ (row%8).
#pragma unroll
      for (int q = 0; q < BKV / 8; ++q) {
        uint8_t *dst = pP + (q / 8) * BOX + row * 128 + (((q % 8) ^ (row & 7)) * 16);
        *reinterpret_cast<uint4 *>(dst) =
            make_uint4(pk[4 * q + 0], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(P_FULL);
    }
    if (ok) ok = mbar_wait(PV_DONE, (nkv - 1) & 1, p.status);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int qrow = q0 + row;
      uint16_t *dst = static_cast<uint16_t *>(p.o) + static_cast<size_t>(qrow) * p.ldo + head * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tl + 256 + 32 * c, r);
        if (qrow < p.n) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            st_global_v4(dst + 32 * c + 8 * q,
                         pack_bf16x2(__uint_as_float(r[8 * q + 0]) * inv_l,
                                     __uint_as_float(r[8 * q + 1]) * inv_l),
                         pack_bf16x2(__uint_as_float(r[8 * q + 2]) * inv_l,
                                     __uint_as_float(r[8 * q + 3]) * inv_l),
                         pack_bf16x2(__uint_as_float(r[8 * q + 4]) * inv_l,
                                     __uint_as_float(r[8 * q + 5]) * inv_l),
                         pack_bf16x2(__uint_as_float(r[8 * q + 6]) * inv_l,
                                     __uint_as_float(r[8 * q + 7]) * inv_l));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int DH>
cudaError_t launch_dh(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                      const AttnParams &p, int heads, cudaStream_t s) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tcgen05<DH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid((p.n + BQ - 1) / BQ, heads);
  attn_fwd_tcgen05<DH><<<grid, THREADS, SMEM_BYTES, s>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                             const AttnParams &p, int head_dim, int heads, cudaStream_t s) {
  if (head_dim == 96) return launch_dh<96>(q, k, v, p, heads, s);
  if (head_dim == 128) return launch_dh<128>(q, k, v, p, heads, s);
  return cudaErrorInvalidValue;
}

}  // namespace h3
