// Memory-bound steps of the block and step:
//   a1  timestep sinusoid + fp32 MLP (two GEMVs)            time_embed_*
//   a2  per-step AdaLN projection for every block (GEMV over bf16 weights,
//       HBM-bound: 6 D^2 bf16 per block)                     adaln_project
//   a3/a7 RMSNorm + (1 + scale), + shift, bf16 out           rmsnorm_modulate
//   RoPE cos/sin table of the packed sequence                rope_table
//   packing [text; images] into the fp32 residual and back   pack / unpack
#include <math.h>

#include <mutex>

#include "kernels.h"
#include "ptx.cuh"

namespace h3 {
namespace {

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- a1
// hidden[j] = SiLU(W1[j] . e(t) + b1[j]); one warp per output row.
__global__ void time_hidden_kernel(float t, float t_scale, const float *__restrict__ w1,
                                   const float *__restrict__ b1, float *__restrict__ hidden,
                                   int d) {
  __shared__ float e[256];
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    // frequency 10000^(-i/128); argument t_scale * t * freq, in double
    const double w = exp(-static_cast<double>(i) / 128.0 * log(10000.0));
    const double a = static_cast<double>(t_scale) * static_cast<double>(t) * w;
    e[i] = static_cast<float>(cos(a));
    e[128 + i] = static_cast<float>(sin(a));
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * (blockDim.x >> 5) + warp;
  if (j >= d) return;
  const float *row = w1 + static_cast<size_t>(j) * 256;
  float acc = 0.f;
#pragma unroll
  for (int i = lane; i < 256; i += 32) acc = fmaf(row[i], e[i], acc);
  acc = warp_sum(acc);
  if (lane == 0) hidden[j] = silu_f(acc + b1[j]);
}

// c[j] = W2[j] . hidden + b2[j]; one warp per output row, float4 loads.
__global__ void time_out_kernel(const float *__restrict__ w2, const float *__restrict__ b2,
                                const float *__restrict__ hidden, float *__restrict__ c, int d) {
  extern __shared__ float hs[];
  for (int i = threadIdx.x; i < d; i += blockDim.x) hs[i] = hidden[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * (blockDim.x >> 5) + warp;
  if (j >= d) return;
  const float4 *row = reinterpret_cast<const float4 *>(w2 + static_cast<size_t>(j) * d);
  float acc = 0.f;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 w = __ldg(row + i);
    acc = fmaf(w.x, hs[4 * i + 0], acc);
    acc = fmaf(w.y, hs[4 * i + 1], acc);
    acc = fmaf(w.z, hs[4 * i + 2], acc);
    acc = fmaf(w.w, hs[4 * i + 3], acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) c[j] = acc + b2[j];
}

// ---------------------------------------------------------------- a2
// mod[l][r] = W_ada[l][r] . SiLU(c) + b_ada[l][r], r < 6D, for l in [first, first+count).
// Persistent CTAs; each warp owns one weight row at a time and keeps up to
// kAdaUnroll 16-byte loads in flight per lane.
constexpr int kAdaThreads = 256;
constexpr int kAdaUnroll = 6;

__global__ void __launch_bounds__(kAdaThreads)
    adaln_kernel(const float *__restrict__ c, const void *const *__restrict__ w_ada,
                 const float *const *__restrict__ b_ada, int first, int count,
                 float *__restrict__ mod, int d) {
  extern __shared__ float sc[];  // SiLU(c), d floats
  for (int i = threadIdx.x; i < d; i += blockDim.x) sc[i] = silu_f(c[i]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const long long rows_per_block = 6LL * d;
  const long long total = rows_per_block * count;
  const int chunks = d / 8;  // 16-byte chunks of a bf16 row
  for (long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp; r < total;
       r += warps_total) {
    const int lb = static_cast<int>(r / rows_per_block);
    const long long rr = r - lb * rows_per_block;
    const uint4 *row =
        reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(w_ada[first + lb]) + rr * d);
    float acc = 0.f;
    for (int base = 0; base < chunks; base += 32 * kAdaUnroll) {
      uint4 v[kAdaUnroll];
#pragma unroll
      for (int u = 0; u < kAdaUnroll; ++u) {
        const int ch = base + u * 32 + lane;
        v[u] = ch < chunks ? __ldcs(row + ch) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kAdaUnroll; ++u) {
        const int ch = base + u * 32 + lane;
        if (ch < chunks) {
          const float *s = sc + 8 * ch;
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc = fmaf(__uint_as_float(w[q] << 16), s[2 * q], acc);
            acc = fmaf(__uint_as_float(w[q] & 0xffff0000u), s[2 * q + 1], acc);
          }
        }
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) mod[r] = acc + b_ada[first + lb][rr];
  }
}

// ---------------------------------------------------------------- a3 / a7
// One CTA per row (grid-stride); the row stays in registers between the
// sum-of-squares pass and the output pass.
constexpr int kNormThreads = 256;
constexpr int kNormMaxVec = 8;  // float4s per thread: D <= 8192

// MX: the output is MXFP8 (E4M3 + E8M0 scale per 32), each group of 8
// consecutive threads holding one 32-element block.
template <bool MX>
__global__ void __launch_bounds__(kNormThreads)
    rmsnorm_modulate_kernel(const float *__restrict__ x, const float *__restrict__ shift,
                            const float *__restrict__ scale, void *__restrict__ out_v,
                            uint8_t *__restrict__ out_sf, int n, int d, float eps) {
  __shared__ float red[kNormThreads / 32];
  const int nv = d / 4;
  const float inv_d = 1.f / static_cast<float>(d);
  for (int row = blockIdx.x; row < n; row += gridDim.x) {
    const float4 *xr = reinterpret_cast<const float4 *>(x + static_cast<size_t>(row) * d);
    float4 v[kNormMaxVec];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kNormMaxVec; ++u) {
      const int i = threadIdx.x + u * kNormThreads;
      if (i < nv) {
        v[u] = __ldcs(xr + i);
        ss += v[u].x * v[u].x + v[u].y * v[u].y + v[u].z * v[u].z + v[u].w * v[u].w;
      }
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kNormThreads / 32; ++w) tot += red[w];
    const float rinv = rsqrtf(tot * inv_d + eps);
#pragma unroll
    for (int u = 0; u < kNormMaxVec; ++u) {
      const int i = threadIdx.x + u * kNormThreads;
      if (u * kNormThreads >= nv) break;  // uniform across the block
      float a = 0.f, b = 0.f, cc = 0.f, dd = 0.f;
      if (i < nv) {
        const float4 sh = __ldg(reinterpret_cast<const float4 *>(shift) + i);
        const float4 sc = __ldg(reinterpret_cast<const float4 *>(scale) + i);
        a = fmaf(v[u].x * rinv, 1.f + sc.x, sh.x);
        b = fmaf(v[u].y * rinv, 1.f + sc.y, sh.y);
        cc = fmaf(v[u].z * rinv, 1.f + sc.z, sh.z);
        dd = fmaf(v[u].w * rinv, 1.f + sc.w, sh.w);
      }
      if constexpr (MX) {
        float am = fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(cc), fabsf(dd)));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
        const uint32_t sb = mx_scale_byte(am);
        const float m = mx_inv_scale(sb);
        if (i < nv) {
          reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(out_v) +
                                       static_cast<size_t>(row) * d)[i] =
              mx_pack4(a * m, b * m, cc * m, dd * m);
          if ((i & 7) == 0) out_sf[mx_sf_offset(row, i >> 3, d / 128)] = static_cast<uint8_t>(sb);
        }
      } else if (i < nv) {
        reinterpret_cast<uint2 *>(static_cast<uint16_t *>(out_v) + static_cast<size_t>(row) * d)[i] =
            make_uint2(pack_bf16x2(a, b), pack_bf16x2(cc, dd));
      }
    }
    __syncthreads();  // red[] is reused by the next row
  }
}

// ---------------------------------------------------------------- self-test
__global__ void selftest_wait_kernel(int *status, long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    // nothing ever arrives: the wait must give up and record the timeout
    mbar_wait_limit(smem_u32(&bar), 0, status, limit_cycles);
  }
}

// ---------------------------------------------------------------- RoPE table
struct GridArray {
  GridDesc g[kMaxGrids];
};

__global__ void rope_table_kernel(GridArray grids, int n_grids, int n_txt, int n, int s0, int s1,
                                  int s2, float theta, float *__restrict__ table) {
  const int pairs = s0 + s1 + s2;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(n) * pairs) return;
  const int row = static_cast<int>(idx / pairs);
  const int pr = static_cast<int>(idx - static_cast<long long>(row) * pairs);
  int pos[3] = {0, 0, 0};
  if (row >= n_txt) {
    int r = row - n_txt;
    for (int g = 0; g < n_grids; ++g) {
      const int cnt = grids.g[g].height * grids.g[g].width;
      if (r < cnt) {
        pos[0] = grids.g[g].frame;
        pos[1] = r / grids.g[g].width;
        pos[2] = r % grids.g[g].width;
        break;
      }
      r -= cnt;
    }
  }
  int axis, j, s;
  if (pr < s0) {
    axis = 0; j = pr; s = s0;
  } else if (pr < s0 + s1) {
    axis = 1; j = pr - s0; s = s1;
  } else {
    axis = 2; j = pr - s0 - s1; s = s2;
  }
  const double w = exp(-static_cast<double>(j) / static_cast<double>(s) * log(static_cast<double>(theta)));
  const double a = static_cast<double>(pos[axis]) * w;
  table[2 * idx] = static_cast<float>(cos(a));
  table[2 * idx + 1] = static_cast<float>(sin(a));
}

// ---------------------------------------------------------------- pack / unpack
// Four elements per thread-iteration; token buffers are bf16 or fp32.
__device__ __forceinline__ float4 load4(const uint16_t *p, long long e) {
  const uint2 v = *reinterpret_cast<const uint2 *>(p + e);
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                     __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
}
__device__ __forceinline__ float4 load4(const float *p, long long e) {
  return *reinterpret_cast<const float4 *>(p + e);
}
__device__ __forceinline__ void store4(uint16_t *p, long long e, float4 v) {
  *reinterpret_cast<uint2 *>(p + e) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}
__device__ __forceinline__ void store4(float *p, long long e, float4 v) {
  *reinterpret_cast<float4 *>(p + e) = v;
}

template <typename T>
__global__ void pack_kernel(const T *__restrict__ x_txt, int n_txt, const T *__restrict__ x_img,
                            int n_img, int d, float *__restrict__ resid) {
  const long long nq = static_cast<long long>(n_txt + n_img) * d / 4;
  const long long txt_elems = static_cast<long long>(n_txt) * d;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < nq;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = 4 * i;
    reinterpret_cast<float4 *>(resid)[i] =
        e < txt_elems ? load4(x_txt, e) : load4(x_img, e - txt_elems);
  }
}

template <typename T>
__global__ void unpack_kernel(const float *__restrict__ resid, int n_txt, int n_img, int d,
                              T *__restrict__ x_txt, T *__restrict__ x_img) {
  const long long nq = static_cast<long long>(n_txt + n_img) * d / 4;
  const long long txt_elems = static_cast<long long>(n_txt) * d;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < nq;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = 4 * i;
    const float4 v = reinterpret_cast<const float4 *>(resid)[i];
    if (e < txt_elems)
      store4(x_txt, e, v);
    else
      store4(x_img, e - txt_elems, v);
  }
}

}  // namespace

cudaError_t launch_time_embed(float t, float t_scale, const float *w1, const float *b1,
                              const float *w2, const float *b2, float *hidden, float *c_out,
                              int d, int * /*status*/, cudaStream_t s) {
  const int warps = 8;
  const int grid = (d + warps - 1) / warps;
  time_hidden_kernel<<<grid, 32 * warps, 0, s>>>(t, t_scale, w1, b1, hidden, d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = static_cast<size_t>(d) * sizeof(float);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(time_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  time_out_kernel<<<grid, 32 * warps, smem, s>>>(w2, b2, hidden, c_out, d);
  return cudaGetLastError();
}

// Scratch of the allocation-free timestep MLP: the hidden layer between its
// two GEMVs. Every GPU that loads the library holds these 32 KiB until exit.
static __device__ __align__(256) float g_time_hidden_scratch[kStaticTimeMaxHidden];

// Device address of the scratch array on the current device, looked up once
// per device (host code cannot use the symbol itself as a device pointer).
static cudaError_t time_scratch_address(float **out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static float *addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_time_hidden_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<float *>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_time_embed_static(float t, float t_scale, const float *w1, const float *b1,
                                     const float *w2, const float *b2, float *c_out, int d,
                                     cudaStream_t s) {
  if (d < 1 || d > kStaticTimeMaxHidden) return cudaErrorInvalidValue;
  float *hidden = nullptr;
  cudaError_t e = time_scratch_address(&hidden);
  if (e != cudaSuccess) return e;
  // the hidden layer is fully rewritten before it is read: nothing to clear
  return launch_time_embed(t, t_scale, w1, b1, w2, b2, hidden, c_out, d, nullptr, s);
}

cudaError_t launch_adaln(const float *c, const void *const *w_ada, const float *const *b_ada,
                         int first, int count, float *mod_out, int d, int num_sms,
                         cudaStream_t s) {
  const size_t smem = static_cast<size_t>(d) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(adaln_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const long long rows = 6LL * d * count;
  const long long want = (rows + 7) / 8;
  const int grid = static_cast<int>(want < 4LL * num_sms ? want : 4LL * num_sms);
  adaln_kernel<<<grid, kAdaThreads, smem, s>>>(c, w_ada, b_ada, first, count, mod_out, d);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_modulate(const float *x, const float *shift, const float *scale,
                                    void *out, int n, int d, float eps, int num_sms,
                                    cudaStream_t s, uint8_t *out_sf) {
  if (d > 4 * kNormMaxVec * kNormThreads) return cudaErrorInvalidValue;
  const int grid = n < 8 * num_sms ? n : 8 * num_sms;
  if (out_sf)
    rmsnorm_modulate_kernel<true><<<grid, kNormThreads, 0, s>>>(x, shift, scale, out, out_sf, n, d,
                                                                 eps);
  else
    rmsnorm_modulate_kernel<false><<<grid, kNormThreads, 0, s>>>(x, shift, scale, out, nullptr, n,
                                                                  d, eps);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(int *status, long long limit_cycles, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, limit_cycles);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(const GridDesc *grids, int n_grids, int n_txt, int n,
                              const int sec[3], float theta, float *table, cudaStream_t s) {
  if (n_grids > kMaxGrids) return cudaErrorInvalidValue;
  GridArray ga{};
  for (int i = 0; i < n_grids; ++i) ga.g[i] = grids[i];
  const long long total = static_cast<long long>(n) * (sec[0] + sec[1] + sec[2]);
  const int threads = 256;
  const int grid = static_cast<int>((total + threads - 1) / threads);
  rope_table_kernel<<<grid, threads, 0, s>>>(ga, n_grids, n_txt, n, sec[0], sec[1], sec[2], theta,
                                             table);
  return cudaGetLastError();
}

cudaError_t launch_pack(const void *x_txt, int n_txt, const void *x_img, int n_img, int d,
                        bool fp32_tokens, float *resid, cudaStream_t s) {
  if (fp32_tokens)
    pack_kernel<float><<<1184, 256, 0, s>>>(static_cast<const float *>(x_txt), n_txt,
                                            static_cast<const float *>(x_img), n_img, d, resid);
  else
    pack_kernel<uint16_t><<<1184, 256, 0, s>>>(static_cast<const uint16_t *>(x_txt), n_txt,
                                               static_cast<const uint16_t *>(x_img), n_img, d,
                                               resid);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const float *resid, int n_txt, int n_img, int d, bool fp32_tokens,
                          void *x_txt, void *x_img, cudaStream_t s) {
  if (fp32_tokens)
    unpack_kernel<float><<<1184, 256, 0, s>>>(resid, n_txt, n_img, d, static_cast<float *>(x_txt),
                                              static_cast<float *>(x_img));
  else
    unpack_kernel<uint16_t><<<1184, 256, 0, s>>>(resid, n_txt, n_img, d,
                                                 static_cast<uint16_t *>(x_txt),
                                                 static_cast<uint16_t *>(x_img));
  return cudaGetLastError();
}

}  // namespace h3
