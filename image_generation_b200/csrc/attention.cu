// Joint bidirectional attention on tcgen05 (step a5):
//   O_h = softmax(Q_h K_h^T / sqrt(d_h)) V_h over all tokens, no mask,
// for the single packed text+image stream.
//
// One CTA per (256 queries = two 128-row tiles, head). The KV sequence is
// walked in tiles of 64 keys with an online softmax. Each query tile owns two
// S buffers in tensor memory, so the tensor core computes S_t(j+2) while the
// softmax of tile t works on S_t(j), and the two query tiles interleave:
//   warp 0      TMA: Q0 and Q1 once; K and V tiles into a 4-stage ring (64-
//               column boxes of a 3-D [tokens, heads, d_h] view, 128-byte
//               swizzle; columns past d_h read as zero).
//   warps 1, 10 MMA issuers, one per query tile t: S_t(j) = Q_t K_j^T (M128
//               N64 K d_h) into S buffer j % 2 of tile t; O_t += P_t(j) V_j
//               (M128 N d_h K64) with P_t(j) read from TMEM (the first 32
//               columns of its S buffer, bf16 pairs) and V as an MN-major
//               operand from shared memory. Order per j: PV_t(j), S_t(j+2).
//               One issuer per tile keeps a tile that runs ahead from waiting
//               behind the other tile's softmax.
//   warps 2..5  softmax of query tile 0, one row per thread; warps 6..9 the
//               same for tile 1: read S_t(j), running max in log2 units,
//               P = 2^(s*scale*log2e - m) back over S_t(j) as bf16. O_t is
//               rescaled in TMEM only when the running max grows by more than
//               8 (a factor 256), after waiting for PV_t(j-1); otherwise the
//               stale max is kept, which leaves O / l unchanged. After the
//               last tile it normalises O_t by the row sum and stores it.
// Tensor memory (512 columns): S buffers of tile t at 64 * (2t + b), b = 0, 1;
// at d_h 128, O0 at [256, 384) and O1 at [384, 512); at d_h 96, O0 at
// [256, 352), O1 at [352, 448), and the first 64 dimensions of Q_t at
// [448 + 32 t, 480 + 32 t), written once by the softmax warps in the layout P
// uses, so that four of the six K16 steps of each S MMA take A from tensor
// memory instead of re-reading Q from shared memory.
// Ordering: one thread's MMAs run in issue order; S_t(j+2) is issued after
// PV_t(j), which read P_t(j) from the same columns, by the same thread. A K/V
// stage is released once both issuers have committed past its last use.
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {

// Per-phase clock stamps of one CTA (the build with -DH3_ATTN_STAMPS only;
// the product build compiles the stamp points away). Slot layout, one row of
// kStampSlots per 64-key step j: softmax of query tile t (its first warp,
// lane 0) at 6t + {S seen, scores loaded, row max, exponentials, P stored,
// P handed back}; issuer of tile t at 12 + 3t + {P seen, PV issued, S(j+2)
// issued}; TMA producer at 18 (stage free); hand-back of each softmax warp
// of tile t at 20 + 4t + (warp % 4); issuer of tile t at 28 + t once K_j has
// landed.
constexpr int kStampSlots = 32, kStampSteps = 300;
#ifdef H3_ATTN_STAMPS
__device__ unsigned long long g_attn_stamps[kStampSlots * kStampSteps];
#define H3_STAMP(on, j, slot)                                                      \
  do {                                                                             \
    if ((on) && (j) < kStampSteps) g_attn_stamps[(j) * kStampSlots + (slot)] = clock64(); \
  } while (0)
// the stamp may not move above the computation of `v`
#define H3_STAMP_AFTER(on, j, slot, v)      \
  do {                                      \
    asm volatile("" ::"r"(__float_as_uint(v))); \
    H3_STAMP(on, j, slot);                  \
  } while (0)
#else
#define H3_STAMP(on, j, slot) \
  do {                        \
  } while (0)
#define H3_STAMP_AFTER(on, j, slot, v) \
  do {                                 \
  } while (0)
#endif

namespace {

constexpr int BQ = kAttnBQ;                  // rows of one query tile
constexpr int BKV = kAttnBKV;                // keys per KV tile (64)
constexpr int SBUF = 2;                      // S buffers per query tile (128 columns each tile)
constexpr int NS = 4;                        // K/V ring stages (128 KiB)
constexpr uint32_t QBOX = 128 * 128;         // one [128 rows x 64 bf16] swizzled box
constexpr uint32_t KBOX = BKV * 128;         // one [64 rows x 64 bf16] swizzled box
constexpr uint32_t Q_BYTES = 2 * QBOX;       // one query tile (d_h <= 128)
constexpr uint32_t KV_BYTES = 2 * KBOX;      // one K or V tile
constexpr uint32_t STAGE_BYTES = 2 * KV_BYTES;
constexpr int THREADS = 352;                 // 11 warps
// q_full, kv_full/empty[NS], s_full[2][2], p_full[2][2], pv_done[2], o_full[2], drain[2].
// P_FULL is per S buffer: with two S buffers a softmax group can finish steps
// j and j+1 before the MMA warp looks for step j, and a single barrier would
// then have moved two phases, which a parity wait cannot tell apart.
constexpr int NUM_BARS = 1 + 2 * NS + 4 + 4 + 2 + 2 + 2 + 2;
constexpr int SMEM_BYTES = 2 * Q_BYTES + NS * STAGE_BYTES + 1024 + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;    // log2 units
// d_h 96: Q's first 64 dimensions of tile t live in TMEM at QT_COL + 32 t (A
// operand of four of the six S MMAs), which moves O_1 to 352.
constexpr uint32_t QT_COL = 448;

// One row's scores for 64 keys from TMEM; keys at or past `valid` are -inf
// (only the last KV tile has any).
H3_DEV void load_scores64(uint32_t taddr, float (&s)[64], int valid) {
  uint32_t r[64];
  tmem_ld64(taddr, r);
#pragma unroll
  for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(r[i]);
  if (valid < 64) {
#pragma unroll
    for (int i = 0; i < 64; ++i)
      if (i >= valid) s[i] = -INFINITY;
  }
}

// Max of 64 scores: eight independent chains (a two-input max, then three
// three-input maxes each), then a three-level combine.
H3_DEV float row_max64(const float (&s)[64]) {
  float a[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) a[c] = fmaxf(s[c], s[8 + c]);
#pragma unroll
  for (int i = 16; i < 64; i += 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c) a[c] = fmax3(a[c], s[i + c], s[i + 8 + c]);
  }
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

// p_i = 2^(s_i * scale_log2 - m) for 64 scores, two at a time: added into the
// four partial row sums and packed as bf16 pairs (the A operand of PV).
H3_DEV void exp_pack64(const float (&s)[64], float sl2, float m, uint64_t (&part)[4],
                       uint32_t (&pk)[32]) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m, -m);
#pragma unroll
  for (int i = 0; i < 64; i += 2) {
    const uint64_t y2 = f2_fma(f2_pack(s[i], s[i + 1]), sl2x2, negm2);
    float y0, y1;
    f2_unpack(y2, y0, y1);
    const uint64_t e2 = f2_pack(ex2_approx(y0), ex2_approx(y1));
    part[(i / 2) & 3] = f2_add(part[(i / 2) & 3], e2);
    float e0, e1;
    f2_unpack(e2, e0, e1);
    pk[i / 2] = pack_bf16x2(e0, e1);
  }
}

// O_t (+)= P_t V with P_t in TMEM (kind::f16, A from tensor memory).
H3_DEV void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// OUT_MX: write O as MXFP8 (E4M3 + a scale per 32 of head_dim) for the
// MXFP8 out-projection instead of bf16. 352 threads = 11 warps, spread
// 3/3/3/2 over the four SM sub-partitions, each with a 16K-register file:
// at most 168 registers per thread.
template <int DH, bool OUT_MX>
__global__ void __launch_bounds__(THREADS, 1)
    attn_fwd_tcgen05(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const AttnParams p) {
  static_assert(DH == 96 || DH == 128, "head_dim");
  constexpr int DCH = (DH + 63) / 64;  // 64-column boxes per row
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV, false, false);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(BQ, DH, false, true);
  constexpr bool QT = DH == 96;                  // Q (first 64 dims) in TMEM
  constexpr uint32_t O_STRIDE = QT ? 96 : 128;   // O_t at 256 + O_STRIDE t

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(smem);  // Q0 then Q1
  const uint32_t sKV = sQ + 2 * Q_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 2 * Q_BYTES + NS * STAGE_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);

  const uint32_t b0 = smem_u32(bars);
  const uint32_t Q_FULL = b0;
  auto KV_FULL = [&](int s) { return b0 + 8u * (1 + s); };
  auto KV_EMPTY = [&](int s) { return b0 + 8u * (1 + NS + s); };
  auto S_FULL = [&](int t, int b) { return b0 + 8u * (1 + 2 * NS + 2 * t + b); };
  auto P_FULL = [&](int t, int b) { return b0 + 8u * (5 + 2 * NS + 2 * t + b); };
  auto PV_DONE = [&](int t) { return b0 + 8u * (9 + 2 * NS + t); };
  auto O_FULL = [&](int t) { return b0 + 8u * (11 + 2 * NS + t); };
  auto DRAIN = [&](int t) { return b0 + 8u * (13 + 2 * NS + t); };
  auto Q_TMEM = [&](int t) { return b0 + 8u * (15 + 2 * NS + t); };

  __shared__ int aborted;
  if (grid_aborted(p.status, &aborted)) return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * 2 * BQ;
  // sequence blockIdx.z of a batch of equal-length sequences stored one after
  // another (rows z n .. z n + n - 1); query rows past n are computed but not
  // stored, keys past n are masked below
  const int seq0 = blockIdx.z * p.n;
  const int nkv = p.tiles_kv;
#ifdef H3_ATTN_STAMPS
  const bool stamp_cta = blockIdx.x == 20 && blockIdx.y == 10 && blockIdx.z == 0;
#endif

  if (threadIdx.x == 0) {
    mbar_init(Q_FULL, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(KV_FULL(s), 1);
      mbar_init(KV_EMPTY(s), 2);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(S_FULL(t, 0), 1);
      mbar_init(S_FULL(t, 1), 1);
      mbar_init(P_FULL(t, 0), 128);
      mbar_init(P_FULL(t, 1), 128);
      mbar_init(PV_DONE(t), 1);
      mbar_init(O_FULL(t), 1);
    }
    mbar_init(DRAIN(0), 1);
    mbar_init(DRAIN(1), 1);
    mbar_init(Q_TMEM(0), 128);
    mbar_init(Q_TMEM(1), 128);
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
      mbar_arrive_expect_tx(Q_FULL, 2 * DCH * QBOX);
      for (int t = 0; t < 2; ++t)
        for (int c = 0; c < DCH; ++c)
          tma_load_3d(sQ + t * Q_BYTES + c * QBOX, &tq, 64 * c, head, seq0 + q0 + t * BQ, Q_FULL);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % NS;
        if (!mbar_wait(KV_EMPTY(st), ((j / NS) & 1) ^ 1, p.status)) break;
        H3_STAMP(stamp_cta, j, 18);
        mbar_arrive_expect_tx(KV_FULL(st), 2 * DCH * KBOX);
        const uint32_t k_dst = sKV + st * STAGE_BYTES;
        const uint32_t v_dst = k_dst + KV_BYTES;
        for (int c = 0; c < DCH; ++c) {
          tma_load_3d(k_dst + c * KBOX, &tk, 64 * c, head, seq0 + j * BKV, KV_FULL(st));
          tma_load_3d(v_dst + c * KBOX, &tv, 64 * c, head, seq0 + j * BKV, KV_FULL(st));
        }
        issued = j + 1;
      }
      // Every load issued must land before the CTA exits.
      mbar_wait(Q_FULL, 0, p.status, false);
      for (int j = issued - 1; j >= 0 && j >= issued - NS; --j)
        mbar_wait(KV_FULL(j % NS), (j / NS) & 1, p.status, false);
    }
  } else if (warp == 1 || warp == 10) {
    if (lane == 0) {
      const int t = warp == 1 ? 0 : 1;
      const uint32_t s_base = tmem + 128u * t;
      const uint32_t q_src = sQ + t * Q_BYTES;
      const uint32_t o_tmem = tmem + 256 + O_STRIDE * t;
      const uint32_t q_tmem = tmem + QT_COL + 32 * t;
      auto issue_s = [&](int j) -> bool {
        if (!mbar_wait(KV_FULL(j % NS), (j / NS) & 1, p.status)) return false;
        H3_STAMP(stamp_cta, j, 28 + t);
        tc_fence_after();
        const uint32_t k_src = sKV + (j % NS) * STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t d = s_base + static_cast<uint32_t>(BKV * (j % SBUF));
          const uint64_t db = desc_sw128(k_src + (kk / 4) * KBOX + (kk % 4) * 32, 16, 1024);
          if (QT && kk < 4)
            umma_bf16_ts(d, q_tmem + 8 * kk, db, IDESC_S, kk > 0 ? 1u : 0u);
          else
            umma_bf16(d, desc_sw128(q_src + (kk / 4) * QBOX + (kk % 4) * 32, 16, 1024), db,
                      IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(S_FULL(t, j % SBUF));
        return true;
      };
      bool ok = mbar_wait(Q_FULL, 0, p.status);
      if (QT && ok) {
        ok = mbar_wait(Q_TMEM(t), 0, p.status);  // the softmax group wrote Q_t into TMEM
        tc_fence_after();
      }
      for (int j = 0; j < SBUF && j < nkv && ok; ++j) ok = issue_s(j);
      for (int j = 0; j < nkv && ok; ++j) {
        if (!mbar_wait(P_FULL(t, j % SBUF), (j / SBUF) & 1, p.status)) {
          ok = false;
          break;
        }
        H3_STAMP(stamp_cta, j, 12 + 3 * t);
        tc_fence_after();
        const uint32_t v_src = sKV + (j % NS) * STAGE_BYTES + KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          // A: P_t(j) in TMEM, 16 keys = 8 packed columns per step
          umma_bf16_ts(o_tmem, s_base + static_cast<uint32_t>(BKV * (j % SBUF)) + 8 * kk,
                       desc_sw128(v_src + kk * 16 * 128, KBOX, 1024), IDESC_O,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(PV_DONE(t));
        umma_commit(KV_EMPTY(j % NS));  // this tile no longer reads K_j, V_j
        if (j + 1 == nkv) umma_commit(O_FULL(t));
        H3_STAMP(stamp_cta, j, 13 + 3 * t);
        if (j + SBUF < nkv && !issue_s(j + SBUF)) {
          ok = false;
          break;
        }
        H3_STAMP(stamp_cta, j, 14 + 3 * t);
      }
      umma_commit(DRAIN(t));
      mbar_wait(DRAIN(t), 0, p.status, false);
    }
  } else {
    // softmax group t = 0 (warps 2..5) or 1 (warps 6..9); warp w reads TMEM
    // lanes [32 (w % 4), +32): one query row per thread
    const int t = (warp - 2) >> 2;  // warps 2..9 only: warp 10 is an issuer
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t tO = tmem + lane_off + 256 + O_STRIDE * t;
    const float sl2 = p.scale_log2;
    float m = 0.f, l = 0.f;
    bool ok = true;
    if (QT) {
      // this row's first 64 dims of Q (box 0 of the 128-byte-swizzled tile:
      // 16-byte chunk c of row r at chunk c ^ (r % 8)) into TMEM, packed as
      // the S MMA's A operand, the layout P is written in
      ok = mbar_wait(Q_FULL, 0, p.status);
      if (__all_sync(0xffffffffu, ok)) {
        const uint8_t *qrow = smem + t * Q_BYTES + row * 128;
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4 *>(qrow + ((c ^ (row & 7)) << 4));
          r[4 * c + 0] = v.x;
          r[4 * c + 1] = v.y;
          r[4 * c + 2] = v.z;
          r[4 * c + 3] = v.w;
        }
        tmem_st32(tmem + lane_off + QT_COL + 32 * t, r);
      }
      tc_fence_before();
      mbar_arrive(Q_TMEM(t));  // always, so the issuer's wait ends either way
    }
    for (int j = 0; j < nkv; ++j) {
      const uint32_t tS = tmem + lane_off + 128u * t + static_cast<uint32_t>(BKV * (j % SBUF));
      ok = mbar_wait(S_FULL(t, j % SBUF), (j / SBUF) & 1, p.status);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
#ifdef H3_ATTN_STAMPS
      const bool me = stamp_cta && sub == 0 && lane == 0;
#endif
      H3_STAMP(me, j, 6 * t + 0);
      tc_fence_after();
      const int valid = p.n - j * BKV;  // keys of this tile that exist
      float alpha = 1.f;
      bool rescale = false;
      auto update_max = [&](float mx) {  // mx: row max of the raw scores
        mx *= sl2;
        if (j == 0) {
          m = mx;
        } else if (mx > m + RESCALE_THRESHOLD) {
          alpha = ex2_approx(m - mx);
          m = mx;
          rescale = true;
        }
      };
      uint64_t part[4] = {0, 0, 0, 0};
      {
        float sc[64];
        load_scores64(tS, sc, valid);
        H3_STAMP_AFTER(me, j, 6 * t + 1, sc[63]);
        update_max(row_max64(sc));
        H3_STAMP_AFTER(me, j, 6 * t + 2, m);
        uint32_t pk[32];
        exp_pack64(sc, sl2, m, part, pk);
        H3_STAMP_AFTER(me, j, 6 * t + 3, __uint_as_float(pk[31]));
        tmem_st32(tS, pk);
        H3_STAMP(me, j, 6 * t + 4);
      }
      float sum;
      {
        const uint64_t t2 = f2_add(f2_add(part[0], part[1]), f2_add(part[2], part[3]));
        float a0, a1;
        f2_unpack(t2, a0, a1);
        sum = a0 + a1;
      }
      l = l * alpha + sum;
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        // O_t must hold PV_t(j-1) in full before it is rescaled
        ok = mbar_wait(PV_DONE(t), (j - 1) & 1, p.status);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + 32 * c, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + 32 * c, r);
        }
      }
      tc_fence_before();
      mbar_arrive(P_FULL(t, j % SBUF));
      H3_STAMP(me, j, 6 * t + 5);
      H3_STAMP(stamp_cta && lane == 0, j, 20 + 4 * t + sub);
    }
    if (ok) ok = mbar_wait(O_FULL(t), 0, p.status);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int qrow = q0 + t * BQ + row;  // within the sequence
      const size_t grow = static_cast<size_t>(seq0) + qrow;
      // where this row's output goes: row grow of o, or, with the second
      // Ulysses all-to-all fused in, row grow % rows of the output of the
      // rank that holds the token, at this rank's head-group columns
      void *obase = p.o;
      uint8_t *sfbase = p.o_sf;
      size_t orow = grow;
      int col0 = head * DH;
      if (p.o_scatter_ranks != 0) {
        int owner = static_cast<int>(grow / static_cast<size_t>(p.o_rows_per_rank));
        owner = owner < kMaxScatterRanks ? owner : 0;  // only rows past n reach beyond
        orow = grow - static_cast<size_t>(owner) * p.o_rows_per_rank;
        col0 += p.o_col0;
        obase = p.o_scatter[owner];
        sfbase = p.o_sf_scatter[owner];
      }
      uint16_t *dst = static_cast<uint16_t *>(obase) + orow * p.ldo + col0;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + 32 * c, r);
        if constexpr (OUT_MX) {
          if (qrow < p.n) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * inv_l;
            uint32_t q[8];
            const uint32_t sb = mx_quant32(v, q);
            uint8_t *d8 = static_cast<uint8_t *>(obase) + orow * p.ldo + col0 + 32 * c;
            st_global_v4(d8, q[0], q[1], q[2], q[3]);
            st_global_v4(d8 + 16, q[4], q[5], q[6], q[7]);
            sfbase[mx_sf_offset(static_cast<int>(orow), col0 / 32 + c,
                                static_cast<int>(p.ldo / 128))] = static_cast<uint8_t>(sb);
          }
          continue;
        }
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

template <int DH, bool OUT_MX>
cudaError_t launch_dh(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                      const AttnParams &p, int heads, cudaStream_t s) {
  static PerDevice smem_attr;
  cudaError_t e = set_smem_once(smem_attr, attn_fwd_tcgen05<DH, OUT_MX>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((p.n + 2 * BQ - 1) / (2 * BQ), heads, p.batch);
  attn_fwd_tcgen05<DH, OUT_MX><<<grid, THREADS, SMEM_BYTES, s>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

int attention_stamps(unsigned long long *host, int slots, int steps) {
#ifdef H3_ATTN_STAMPS
  if (slots != kStampSlots || steps != kStampSteps) return -1;
  return cudaMemcpyFromSymbol(host, g_attn_stamps, sizeof(g_attn_stamps)) == cudaSuccess ? 0 : -2;
#else
  (void)host;
  (void)slots;
  (void)steps;
  return 1;  // a build without the stamp points
#endif
}

cudaError_t launch_attention(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                             const AttnParams &p, int head_dim, int heads, bool out_mx,
                             cudaStream_t s) {
  if (head_dim == 96)
    return out_mx ? launch_dh<96, true>(q, k, v, p, heads, s) : launch_dh<96, false>(q, k, v, p, heads, s);
  if (head_dim == 128)
    return out_mx ? launch_dh<128, true>(q, k, v, p, heads, s)
                  : launch_dh<128, false>(q, k, v, p, heads, s);
  return cudaErrorInvalidValue;
}

}  // namespace h3
