// Epilogues shared by the bf16 and MXFP8 tcgen05 GEMMs: each epilogue thread
// owns one output row of the tile (its TMEM lane) and walks the tile's columns
// in 32-column chunks (48 for a 24-pair rotary section), applying the fused
// step: plain bf16 store, RoPE on Q and K, GELU (bf16 or MXFP8 out), or the
// AdaLN-gated residual update of the fp32 stream; with a bias vector (the VAE
// decoder's linears) the bias is added to the product first.
#pragma once

#include <cuda_fp8.h>

#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace gemm_detail {

#ifndef H3_GEMM_GROUP_M
#define H3_GEMM_GROUP_M 16
#endif
constexpr int GROUP_M = H3_GEMM_GROUP_M;

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

// erf(z) for z >= 0 by Abramowitz & Stegun, Handbook of Mathematical
// Functions, 7.1.26: 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) e^(-z^2)
// with t = 1 / (1 + p z), |error| <= 1.5e-7 (far below the bf16 or E4M3
// rounding of the GELU output). Two MUFU operations (reciprocal, 2^x) and a
// handful of FMAs per element, which keeps the FFN1 epilogue cheap.
__device__ __forceinline__ float erf_nonneg(float z) {
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, z, 1.0f)));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  poly *= t;
  const float e = ex2_approx(-(z * z) * 1.4426950408889634f);  // e^(-z^2)
  return fmaf(-poly, e, 1.0f);
}

__device__ __forceinline__ float gelu_f(float x, int tanh_form) {
  if (tanh_form) {
    const float u = 0.7978845608028654f * (x + 0.044715f * x * x * x);
    return 0.5f * x * (1.0f + tanhf(u));
  }
  // x Phi(x) = x (1 + erf(x / sqrt 2)) / 2, erf odd
  const float er = copysignf(erf_nonneg(fabsf(x) * 0.7071067811865476f), x);
  return x * fmaf(0.5f, er, 0.5f);
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

// Where the bf16 output element (row, col) goes: the row-major output, or,
// with the first Ulysses all-to-all fused into QKV + RoPE, the receive buffer
// of the rank that attends over col's head group, at this rank's block of
// sequence rows. A store unit (32 columns, or one rotary section) lies inside
// one head, so it goes to one rank and stays contiguous there.
__device__ __forceinline__ uint16_t *out_bf16(const GemmParams &p, int row, int col) {
  if (p.scatter_ranks == 0)
    return static_cast<uint16_t *>(p.out) + static_cast<size_t>(row) * p.ldo + col;
  const int q = col / p.scatter_inner;  // 0 Q, 1 K, 2 V
  const int c = col - q * p.scatter_inner;
  const int g = c / p.scatter_cols;     // head group = destination rank
  const size_t r = static_cast<size_t>(p.scatter_rank) * p.m + row;
  return static_cast<uint16_t *>(p.scatter[g]) + r * (3 * p.scatter_cols) + q * p.scatter_cols +
         (c - g * p.scatter_cols);
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
  store_bf16_row<2 * S>(out_bf16(p, row, col), v);
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
  if (p.bias) {
    const float4 *b = reinterpret_cast<const float4 *>(p.bias + col);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 bb = __ldg(b + q);
      v[4 * q + 0] += bb.x;
      v[4 * q + 1] += bb.y;
      v[4 * q + 2] += bb.z;
      v[4 * q + 3] += bb.w;
    }
  }
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
  } else if constexpr (EPI == kEpiGeluMx) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gelu_f(v[i], p.gelu_tanh);
    uint32_t q[8];
    const uint32_t sb = mx_quant32(v, q);
    uint8_t *dst = static_cast<uint8_t *>(p.out) + static_cast<size_t>(row) * p.ldo + col;
    st_global_v4(dst, q[0], q[1], q[2], q[3]);
    st_global_v4(dst + 16, q[4], q[5], q[6], q[7]);
    p.out_sf[mx_sf_offset(row, col / 32, p.n / 128)] = static_cast<uint8_t>(sb);
  } else {
    if constexpr (EPI == kEpiGelu) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = gelu_f(v[i], p.gelu_tanh);
    }
    store_bf16_row<32>(out_bf16(p, row, col), v);
  }
}

// part / parts: the thread handles every parts-th unit (32 columns, or a
// rotary section) of the tile starting at unit `part`, so several epilogue
// warps on one TMEM lane quarter can share a tile.
template <int EPI, int BN>
__device__ __forceinline__ void epilogue_tile(const GemmParams &p, uint32_t tbase, int row,
                                              int col_tile, int part = 0, int parts = 1) {
  const bool row_ok = row < p.m;
  int unit = 0;
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
        const bool mine = unit++ % parts == part;
        if (s == 16) {
          if (mine) rope_unit<16>(p, tbase + c, row, col, pb, row_ok);
          c += 32;
        } else {
          if (mine) rope_unit<24>(p, tbase + c, row, col, pb, row_ok);
          c += 48;
        }
      } else {
        if (unit++ % parts == part) plain_chunk<kEpiStore>(p, tbase + c, row, col, row_ok);
        c += 32;
      }
    }
  } else {
#pragma unroll 1
    for (int c = 32 * part; c < BN; c += 32 * parts) {
      const int col = col_tile + c;
      if (col >= p.n) break;
      plain_chunk<EPI>(p, tbase + c, row, col, row_ok);
    }
  }
}


}  // namespace gemm_detail
}  // namespace h3
