// The image VAE's 2-D ViT decoder (MiniMax-H3-Image model card, "Model
// Architecture": 24 layers, 16x spatial downsampling, 24 latent channels;
// "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin", "Faster Decoding":
// independent image tiles). The layers run on the block's kernels (paired
// tcgen05 GEMM with a bias in the epilogue, the attention kernel batched over
// tiles); this file holds the decoder's own memory-bound steps:
//   layernorm        (x - mean) / sqrt(var + eps) * gain + bias, fp32 rows in,
//                    bf16 out; the row stays in registers for both passes (one
//                    warp per row up to 2048 wide, one CTA per row beyond)
//   vae_pos_table    the tile-local 2-D sin-cos position table [T*T, W]
//   vae_embed        latent [C, Hl, Wl] -> tokens in tile order (tile-major,
//                    row-major inside a tile): W_in z + b_in + table, fp32
//   vae_pixels       tokens [n, 3*16*16] (bf16, the output linear's result)
//                    -> image [3, 16 Hl, 16 Wl] fp32, feature ch*256 + 16 i + j
//                    of token (r, c) at pixel (16 r + i, 16 c + j) of ch
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int kLnThreads = 256;
constexpr int kLnMaxVec = 8;  // float4s per thread: W <= 8192

__device__ __forceinline__ float warp_sum_ln(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over the CTA through `red` (kLnThreads / 32 floats); every thread gets it.
__device__ __forceinline__ float block_sum(float v, float *red) {
  v = warp_sum_ln(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kLnThreads / 32; ++w) t += red[w];
  __syncthreads();  // red is reused by the next sum
  return t;
}

__global__ void __launch_bounds__(kLnThreads)
    layernorm_kernel(const float *__restrict__ x, const float *__restrict__ gain,
                     const float *__restrict__ bias, uint16_t *__restrict__ out, int n, int d,
                     float eps) {
  __shared__ float red[kLnThreads / 32];
  const int nv = d / 4;
  const float inv_d = 1.f / static_cast<float>(d);
  for (int row = blockIdx.x; row < n; row += gridDim.x) {
    const float4 *xr = reinterpret_cast<const float4 *>(x + static_cast<size_t>(row) * d);
    float4 v[kLnMaxVec];
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < kLnMaxVec; ++u) {
      const int i = threadIdx.x + u * kLnThreads;
      v[u] = i < nv ? __ldcs(xr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      s += (v[u].x + v[u].y) + (v[u].z + v[u].w);
    }
    const float mean = block_sum(s, red) * inv_d;
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kLnMaxVec; ++u) {
      const int i = threadIdx.x + u * kLnThreads;
      if (i < nv) {
        const float a = v[u].x - mean, b = v[u].y - mean, c = v[u].z - mean, e = v[u].w - mean;
        ss += (a * a + b * b) + (c * c + e * e);
      }
    }
    const float rstd = rsqrtf(block_sum(ss, red) * inv_d + eps);
#pragma unroll
    for (int u = 0; u < kLnMaxVec; ++u) {
      const int i = threadIdx.x + u * kLnThreads;
      if (i < nv) {
        const float4 g = __ldg(reinterpret_cast<const float4 *>(gain) + i);
        const float4 b = __ldg(reinterpret_cast<const float4 *>(bias) + i);
        reinterpret_cast<uint2 *>(out + static_cast<size_t>(row) * d)[i] =
            make_uint2(pack_bf16x2(fmaf((v[u].x - mean) * rstd, g.x, b.x),
                                   fmaf((v[u].y - mean) * rstd, g.y, b.y)),
                       pack_bf16x2(fmaf((v[u].z - mean) * rstd, g.z, b.z),
                                   fmaf((v[u].w - mean) * rstd, g.w, b.w)));
      }
    }
  }
}

// Rows of at most 2048 floats: one warp per row, the row in registers (up to
// 16 float4 per lane), both reductions by shuffles - no block-wide barrier.
constexpr int kLnWarpMaxVec = 16;

__global__ void __launch_bounds__(256)
    layernorm_warp_kernel(const float *__restrict__ x, const float *__restrict__ gain,
                          const float *__restrict__ bias, uint16_t *__restrict__ out, int n, int d,
                          float eps) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nv = d / 4;
  const float inv_d = 1.f / static_cast<float>(d);
  for (int row = blockIdx.x * warps + (threadIdx.x >> 5); row < n; row += gridDim.x * warps) {
    const float4 *xr = reinterpret_cast<const float4 *>(x + static_cast<size_t>(row) * d);
    float4 v[kLnWarpMaxVec];
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < kLnWarpMaxVec; ++u) {
      const int i = lane + 32 * u;
      v[u] = i < nv ? __ldcs(xr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      s += (v[u].x + v[u].y) + (v[u].z + v[u].w);
    }
    const float mean = warp_sum_ln(s) * inv_d;
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kLnWarpMaxVec; ++u) {
      if (lane + 32 * u < nv) {
        const float a = v[u].x - mean, b = v[u].y - mean, c = v[u].z - mean, e = v[u].w - mean;
        ss += (a * a + b * b) + (c * c + e * e);
      }
    }
    const float rstd = rsqrtf(warp_sum_ln(ss) * inv_d + eps);
#pragma unroll
    for (int u = 0; u < kLnWarpMaxVec; ++u) {
      const int i = lane + 32 * u;
      if (i < nv) {
        const float4 g = __ldg(reinterpret_cast<const float4 *>(gain) + i);
        const float4 b = __ldg(reinterpret_cast<const float4 *>(bias) + i);
        reinterpret_cast<uint2 *>(out + static_cast<size_t>(row) * d)[i] =
            make_uint2(pack_bf16x2(fmaf((v[u].x - mean) * rstd, g.x, b.x),
                                   fmaf((v[u].y - mean) * rstd, g.y, b.y)),
                       pack_bf16x2(fmaf((v[u].z - mean) * rstd, g.z, b.z),
                                   fmaf((v[u].w - mean) * rstd, g.w, b.w)));
      }
    }
  }
}

// table[p][k]: the first W/2 channels encode the row p / T, the last W/2 the
// column p % T, each as [sin(q w_k) for k < W/4] then [cos(q w_k)], with
// w_k = 10000^(-k / (W/4)); in double, rounded once to fp32.
__global__ void vae_pos_table_kernel(int T, int W, float *__restrict__ table) {
  const long long total = static_cast<long long>(T) * T * W;
  const int q = W / 4;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(e / W), ch = static_cast<int>(e % W);
    const int part = ch / q, k = ch % q;
    const double pos = part < 2 ? static_cast<double>(p / T) : static_cast<double>(p % T);
    const double a = pos * exp(-static_cast<double>(k) / q * log(10000.0));
    table[e] = static_cast<float>((part & 1) ? cos(a) : sin(a));
  }
}

// CTA tile: 64 tokens x 128 output columns, all K = C (<= 32) latent channels.
constexpr int kEmbTok = 64, kEmbCol = 128, kEmbMaxC = 32, kEmbThreads = 256;

__global__ void __launch_bounds__(kEmbThreads)
    vae_embed_kernel(const float *__restrict__ z, int C, int Hl, int Wl, int T,
                     const float *__restrict__ w_in, const float *__restrict__ b_in,
                     const float *__restrict__ table, int W, float *__restrict__ out) {
  __shared__ float A[kEmbTok][kEmbMaxC + 1];
  __shared__ float B[kEmbMaxC][kEmbCol];
  const int n_tok = Hl * Wl;
  const int tiles_w = Wl / T;
  const int t0 = blockIdx.x * kEmbTok, c0 = blockIdx.y * kEmbCol;
  for (int e = threadIdx.x; e < kEmbTok * C; e += kEmbThreads) {
    const int t = e / C, ch = e - t * C;
    const int g = t0 + t;
    float v = 0.f;
    if (g < n_tok) {
      const int tile = g / (T * T), local = g - tile * T * T;
      const int y = (tile / tiles_w) * T + local / T;
      const int x = (tile % tiles_w) * T + local % T;
      v = z[(static_cast<size_t>(ch) * Hl + y) * Wl + x];
    }
    A[t][ch] = v;
  }
  for (int e = threadIdx.x; e < kEmbCol * C; e += kEmbThreads) {
    const int c = e / C, ch = e - c * C;
    B[ch][c] = c0 + c < W ? w_in[static_cast<size_t>(c0 + c) * C + ch] : 0.f;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  for (int k = 0; k < C; ++k) {
    float av[4], bv[8];
#pragma unroll
    for (int a = 0; a < 4; ++a) av[a] = A[4 * ty + a][k];
#pragma unroll
    for (int b = 0; b < 8; ++b) bv[b] = B[k][tx + 16 * b];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int g = t0 + 4 * ty + a;
    if (g >= n_tok) continue;
    const int local = g % (T * T);
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int col = c0 + tx + 16 * b;
      if (col >= W) continue;
      out[static_cast<size_t>(g) * W + col] =
          acc[a][b] + b_in[col] + table[static_cast<size_t>(local) * W + col];
    }
  }
}

// One thread per (channel, pixel row i of a token, token): 16 pixels, read as
// 32 bytes of the token's row and written as 64 contiguous bytes; tokens vary
// fastest, so a warp writes whole runs of an image row.
__global__ void vae_pixels_kernel(const uint16_t *__restrict__ tok, int Hl, int Wl, int T,
                                  float *__restrict__ img) {
  const long long n_tok = static_cast<long long>(Hl) * Wl;
  const long long total = 48 * n_tok;
  const int tiles_w = Wl / T;
  const long long img_w = 16LL * Wl, plane = 256LL * Hl * Wl;
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long g = u % n_tok;
    const int ci = static_cast<int>(u / n_tok);  // ch * 16 + i
    const int ch = ci >> 4, i = ci & 15;
    const long long tile = g / (T * T);
    const int local = static_cast<int>(g - tile * T * T);
    const long long y = (tile / tiles_w) * T + local / T;
    const long long x = (tile % tiles_w) * T + local % T;
    const uint4 *src = reinterpret_cast<const uint4 *>(tok + g * 768 + ch * 256 + 16 * i);
    const uint4 a = __ldcs(src), b = __ldcs(src + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float4 *dst = reinterpret_cast<float4 *>(img + ch * plane + (16 * y + i) * img_w + 16 * x);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_float4(__uint_as_float(w[2 * q] << 16), __uint_as_float(w[2 * q] & 0xffff0000u),
                           __uint_as_float(w[2 * q + 1] << 16),
                           __uint_as_float(w[2 * q + 1] & 0xffff0000u));
  }
}

int grid_of(long long units, int threads, int num_sms) {
  const long long want = (units + threads - 1) / threads;
  const long long cap = 16LL * num_sms;
  return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_layernorm(const float *x, const float *gain, const float *bias, void *out,
                             int n, int d, float eps, int num_sms, cudaStream_t s) {
  if (d % 4 || d > 4 * kLnMaxVec * kLnThreads) return cudaErrorInvalidValue;
  if (d <= 4 * 32 * kLnWarpMaxVec) {
    const int rows_per_cta = 8;
    const long long want = (n + rows_per_cta - 1) / rows_per_cta;
    const int grid = static_cast<int>(want < 16LL * num_sms ? want : 16LL * num_sms);
    layernorm_warp_kernel<<<grid, 32 * rows_per_cta, 0, s>>>(x, gain, bias,
                                                              static_cast<uint16_t *>(out), n, d, eps);
    return cudaGetLastError();
  }
  const int grid = n < 8 * num_sms ? n : 8 * num_sms;
  layernorm_kernel<<<grid, kLnThreads, 0, s>>>(x, gain, bias, static_cast<uint16_t *>(out), n, d,
                                               eps);
  return cudaGetLastError();
}

cudaError_t launch_vae_pos_table(int T, int W, float *table, int num_sms, cudaStream_t s) {
  if (T < 1 || W % 4) return cudaErrorInvalidValue;
  vae_pos_table_kernel<<<grid_of(static_cast<long long>(T) * T * W, 256, num_sms), 256, 0, s>>>(
      T, W, table);
  return cudaGetLastError();
}

cudaError_t launch_vae_embed(const float *z, int C, int Hl, int Wl, int T, const float *w_in,
                             const float *b_in, const float *table, int W, float *out,
                             cudaStream_t s) {
  if (C < 1 || C > kEmbMaxC || T < 1 || Hl % T || Wl % T) return cudaErrorInvalidValue;
  const int n_tok = Hl * Wl;
  const dim3 grid((n_tok + kEmbTok - 1) / kEmbTok, (W + kEmbCol - 1) / kEmbCol);
  vae_embed_kernel<<<grid, kEmbThreads, 0, s>>>(z, C, Hl, Wl, T, w_in, b_in, table, W, out);
  return cudaGetLastError();
}

cudaError_t launch_vae_pixels(const void *tokens, int Hl, int Wl, int T, float *img, int num_sms,
                              cudaStream_t s) {
  if (T < 1 || Hl % T || Wl % T) return cudaErrorInvalidValue;
  const long long units = 48LL * Hl * Wl;
  vae_pixels_kernel<<<grid_of(units, 256, num_sms), 256, 0, s>>>(
      static_cast<const uint16_t *>(tokens), Hl, Wl, T, img);
  return cudaGetLastError();
}

}  // namespace h3
