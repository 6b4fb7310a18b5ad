// The steps on either side of the block loop (MiniMax-H3-Image model card,
// "Model Architecture": the image VAE's latent has 24 channels at 16x
// downsampling, the DiT patchifies it with a 2x2 patch, and the embedding,
// timestep and output layers are FP32):
//   embed_latent      2x2 patchify of a latent [C, Hl, Wl] gathered straight
//                     into an FP32 GEMM (K = 4 C) with bias: x_img tokens;
//   output_modulation [shift | scale] = W_mod SiLU(c) + b_mod (GEMV);
//   output_euler      per-row RMS of the image tokens, then an FP32 GEMM whose
//                     A operand is normalised and modulated as it is loaded,
//                     with an epilogue that adds the bias, undoes the patchify
//                     and applies the Euler step z += dt * v to the latent.
// Token (r, c) of a latent is row-major over its (Hl/2, Wl/2) patch grid;
// feature ch * 4 + 2 i + j of a token is latent pixel (2 r + i, 2 c + j) of
// channel ch.
#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

__device__ __forceinline__ float silu_io(float x) { return x / (1.f + expf(-x)); }

__device__ __forceinline__ float warp_sum_io(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- embedding
// CTA tile: 64 tokens x 128 output columns, all K = 4 C (<= 128) at once.
// Thread (tx, ty) = (tid % 16, tid / 16) owns tokens 4 ty .. 4 ty + 3 and
// columns tx + 16 j, j < 8 (shared-memory reads conflict-free: a warp reads
// two A rows by broadcast and 16 consecutive B columns).
constexpr int kEmbTok = 64, kEmbCol = 128, kEmbMaxK = 128, kEmbThreads = 256;
constexpr int kEmbSmem = (kEmbTok + kEmbCol) * kEmbMaxK * 4;

template <typename OutT>
__global__ void __launch_bounds__(kEmbThreads)
    embed_latent_kernel(const float *__restrict__ z, int C, int Hl, int Wl,
                        const float *__restrict__ w_in, const float *__restrict__ b_in, int D,
                        OutT *__restrict__ out) {
  extern __shared__ float sm[];
  float *A = sm;                    // [kEmbTok][K]
  float *B = sm + kEmbTok * kEmbMaxK;  // [K][kEmbCol]
  const int K = 4 * C;
  const int w = Wl / 2;
  const int n_tok = (Hl / 2) * w;
  const int t0 = blockIdx.x * kEmbTok, c0 = blockIdx.y * kEmbCol;
  for (int e = threadIdx.x; e < kEmbTok * K; e += kEmbThreads) {
    const int t = e / K, f = e - t * K;
    const int tok = t0 + t;
    float v = 0.f;
    if (tok < n_tok) {
      const int r = tok / w, c = tok - r * w;
      const int ch = f >> 2, i = (f >> 1) & 1, j = f & 1;
      v = z[(static_cast<size_t>(ch) * Hl + 2 * r + i) * Wl + 2 * c + j];
    }
    A[t * K + f] = v;
  }
  for (int e = threadIdx.x; e < kEmbCol * K; e += kEmbThreads) {
    const int c = e / K, f = e - c * K;
    B[f * kEmbCol + c] = c0 + c < D ? w_in[static_cast<size_t>(c0 + c) * K + f] : 0.f;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  for (int f = 0; f < K; ++f) {
    float av[4], bv[8];
#pragma unroll
    for (int a = 0; a < 4; ++a) av[a] = A[(4 * ty + a) * K + f];
#pragma unroll
    for (int b = 0; b < 8; ++b) bv[b] = B[f * kEmbCol + tx + 16 * b];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int tok = t0 + 4 * ty + a;
    if (tok >= n_tok) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int col = c0 + tx + 16 * b;
      if (col >= D) continue;
      const float v = acc[a][b] + b_in[col];
      if constexpr (sizeof(OutT) == 2)
        out[static_cast<size_t>(tok) * D + col] = static_cast<OutT>(pack_bf16x2(v, 0.f) & 0xffffu);
      else
        out[static_cast<size_t>(tok) * D + col] = v;
    }
  }
}

// ---------------------------------------------------------------- modulation
// mod[r] = W_mod[r] . SiLU(c) + b_mod[r], r < 2 D; one warp per row.
__global__ void output_modulation_kernel(const float *__restrict__ c, const float *__restrict__ w,
                                         const float *__restrict__ b, float *__restrict__ mod,
                                         int D) {
  extern __shared__ float sc[];
  for (int i = threadIdx.x; i < D; i += blockDim.x) sc[i] = silu_io(c[i]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + warp;
  if (r >= 2 * D) return;
  const float *row = w + static_cast<size_t>(r) * D;
  float acc = 0.f;
  for (int i = lane; i < D; i += 32) acc = fmaf(row[i], sc[i], acc);
  acc = warp_sum_io(acc);
  if (lane == 0) mod[r] = acc + b[r];
}

// ---------------------------------------------------------------- output + Euler
template <typename InT>
__device__ __forceinline__ float load_tok(const InT *p, size_t i) {
  if constexpr (sizeof(InT) == 2)
    return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
  else
    return p[i];
}

// rinv[t] = 1 / sqrt(mean_d x[t][d]^2 + eps); one warp per token.
template <typename InT>
__global__ void row_rinv_kernel(const InT *__restrict__ x, int n, int D, float eps,
                                float *__restrict__ rinv) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= n) return;
  float ss = 0.f;
  for (int d = lane; d < D; d += 32) {
    const float v = load_tok(x, static_cast<size_t>(t) * D + d);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum_io(ss);
  if (lane == 0) rinv[t] = rsqrtf(ss / static_cast<float>(D) + eps);
}

// CTA tile: 32 tokens x all N = 4 C (<= 128) outputs, K = D in chunks of 64.
// Thread (tx, ty) = (tid % 32, tid / 32) owns tokens 4 ty .. 4 ty + 3 and
// outputs tx + 32 m, m < 4. B is stored [k][N] with a row stride of
// kOutN + 1 floats so the transposing stores are conflict-free.
constexpr int kOutTok = 32, kOutK = 64, kOutN = 128, kOutThreads = 256;

template <typename InT>
__global__ void __launch_bounds__(kOutThreads)
    output_euler_kernel(const InT *__restrict__ x, const float *__restrict__ rinv,
                        const float *__restrict__ shift, const float *__restrict__ scale,
                        const float *__restrict__ w_out, const float *__restrict__ b_out, int D,
                        float *__restrict__ z, int C, int Hl, int Wl, float dt) {
  __shared__ float A[kOutTok][kOutK];
  __shared__ float B[kOutK][kOutN + 1];
  const int N = 4 * C;
  const int w = Wl / 2;
  const int n_tok = (Hl / 2) * w;
  const int t0 = blockIdx.x * kOutTok;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int m = 0; m < 4; ++m) acc[a][m] = 0.f;
  for (int k0 = 0; k0 < D; k0 += kOutK) {
    for (int e = threadIdx.x; e < kOutTok * kOutK; e += kOutThreads) {
      const int t = e / kOutK, k = e - t * kOutK;
      const int tok = t0 + t, d = k0 + k;
      float v = 0.f;
      if (tok < n_tok && d < D)
        v = fmaf(load_tok(x, static_cast<size_t>(tok) * D + d) * rinv[tok], 1.f + scale[d],
                 shift[d]);
      A[t][k] = v;
    }
    for (int e = threadIdx.x; e < kOutN * kOutK; e += kOutThreads) {
      const int f = e / kOutK, k = e - f * kOutK;
      const int d = k0 + k;
      B[k][f] = f < N && d < D ? w_out[static_cast<size_t>(f) * D + d] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kOutK; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) av[a] = A[4 * ty + a][k];
#pragma unroll
      for (int m = 0; m < 4; ++m) bv[m] = B[k][tx + 32 * m];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[a][m] = fmaf(av[a], bv[m], acc[a][m]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int tok = t0 + 4 * ty + a;
    if (tok >= n_tok) continue;
    const int r = tok / w, c = tok - r * w;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int f = tx + 32 * m;
      if (f >= N) continue;
      const int ch = f >> 2, i = (f >> 1) & 1, j = f & 1;
      float *zp = z + (static_cast<size_t>(ch) * Hl + 2 * r + i) * Wl + 2 * c + j;
      *zp = fmaf(dt, acc[a][m] + b_out[f], *zp);
    }
  }
}

}  // namespace

cudaError_t launch_embed_latent(const float *z, int C, int Hl, int Wl, const float *w_in,
                                const float *b_in, int D, void *out, bool out_fp32,
                                cudaStream_t s) {
  if (C <= 0 || 4 * C > kEmbMaxK || Hl < 2 || Wl < 2 || (Hl | Wl) & 1) return cudaErrorInvalidValue;
  const int n_tok = (Hl / 2) * (Wl / 2);
  const dim3 grid((n_tok + kEmbTok - 1) / kEmbTok, (D + kEmbCol - 1) / kEmbCol);
  static PerDevice attr_f32, attr_bf16;
  cudaError_t e = set_smem_once(attr_f32, embed_latent_kernel<float>, kEmbSmem);
  if (e == cudaSuccess) e = set_smem_once(attr_bf16, embed_latent_kernel<uint16_t>, kEmbSmem);
  if (e != cudaSuccess) return e;
  if (out_fp32)
    embed_latent_kernel<float><<<grid, kEmbThreads, kEmbSmem, s>>>(z, C, Hl, Wl, w_in, b_in, D,
                                                                  static_cast<float *>(out));
  else
    embed_latent_kernel<uint16_t><<<grid, kEmbThreads, kEmbSmem, s>>>(
        z, C, Hl, Wl, w_in, b_in, D, static_cast<uint16_t *>(out));
  return cudaGetLastError();
}

cudaError_t launch_output_modulation(const float *c, const float *w_mod, const float *b_mod,
                                     float *mod, int D, cudaStream_t s) {
  const int rows_per_cta = 8;  // 256 threads
  const int grid = (2 * D + rows_per_cta - 1) / rows_per_cta;
  output_modulation_kernel<<<grid, 32 * rows_per_cta, D * sizeof(float), s>>>(c, w_mod, b_mod,
                                                                             mod, D);
  return cudaGetLastError();
}

cudaError_t launch_output_euler(const void *x, bool in_fp32, const float *mod, const float *w_out,
                                const float *b_out, int D, float eps, float *z, int C, int Hl,
                                int Wl, float dt, float *rinv_scratch, cudaStream_t s) {
  if (C <= 0 || 4 * C > kOutN || Hl < 2 || Wl < 2 || (Hl | Wl) & 1) return cudaErrorInvalidValue;
  const int n_tok = (Hl / 2) * (Wl / 2);
  const int warps = 8;
  const int g1 = (n_tok + warps - 1) / warps;
  const int g2 = (n_tok + kOutTok - 1) / kOutTok;
  const float *shift = mod, *scale = mod + D;
  if (in_fp32) {
    const float *xf = static_cast<const float *>(x);
    row_rinv_kernel<float><<<g1, 32 * warps, 0, s>>>(xf, n_tok, D, eps, rinv_scratch);
    output_euler_kernel<float><<<g2, kOutThreads, 0, s>>>(xf, rinv_scratch, shift, scale, w_out,
                                                         b_out, D, z, C, Hl, Wl, dt);
  } else {
    const uint16_t *xb = static_cast<const uint16_t *>(x);
    row_rinv_kernel<uint16_t><<<g1, 32 * warps, 0, s>>>(xb, n_tok, D, eps, rinv_scratch);
    output_euler_kernel<uint16_t><<<g2, kOutThreads, 0, s>>>(xb, rinv_scratch, shift, scale,
                                                            w_out, b_out, D, z, C, Hl, Wl, dt);
  }
  return cudaGetLastError();
}

}  // namespace h3
