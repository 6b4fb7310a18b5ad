// Host-side launchers of the sm_100a kernels (internal to libh3dit).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace h3 {

enum Epilogue : int { kEpiStore = 0, kEpiQkvRope = 1, kEpiGelu = 2, kEpiGatedResidual = 3 };

struct GemmParams {
  int m, n, k;
  int tiles_m, tiles_n;
  void *out;
  long long ldo;          // elements
  const float *gate;      // gated residual: [n]
  const float *rope;      // QKV: [m][head_dim/2][2]
  int head_dim;           // QKV
  int rope_cols;          // QKV: RoPE on columns < rope_cols (Q and K)
  int sec[3];             // QKV: rotation pairs per axis
  int gelu_tanh;
  int *status;
};

struct AttnParams {
  int n;                  // tokens
  int tiles_kv;
  void *o;
  long long ldo;          // elements
  float scale_log2;       // log2(e) / sqrt(head_dim)
  int *status;
};

// Tile of the tcgen05 GEMM (rows x columns of the output).
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;

cudaError_t launch_gemm(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p,
                        int epilogue, int grid, cudaStream_t s);
int gemm_smem_bytes();

cudaError_t launch_attention(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                             const AttnParams &p, int head_dim, int heads, cudaStream_t s);

cudaError_t launch_time_embed(float t, float t_scale, const float *w1, const float *b1,
                              const float *w2, const float *b2, float *hidden, float *c_out,
                              int d, int *status, cudaStream_t s);
// The timestep MLP with its hidden vector in the library's static scratch
// array (at most kStaticTimeMaxHidden floats); no allocation.
constexpr int kStaticTimeMaxHidden = 8192;
cudaError_t launch_time_embed_static(float t, float t_scale, const float *w1, const float *b1,
                                     const float *w2, const float *b2, float *c_out, int d,
                                     cudaStream_t s);
cudaError_t launch_adaln(const float *c, const void *const *w_ada, const float *const *b_ada,
                         int first, int count, float *mod_out, int d, int num_sms,
                         cudaStream_t s);
cudaError_t launch_rmsnorm_modulate(const float *x, const float *shift, const float *scale,
                                    void *out, int n, int d, float eps, int num_sms,
                                    cudaStream_t s);

struct GridDesc {
  int frame, height, width;
};
constexpr int kMaxGrids = 32;
cudaError_t launch_rope_table(const GridDesc *grids, int n_grids, int n_txt, int n,
                              const int sec[3], float theta, float *table, cudaStream_t s);
cudaError_t launch_pack(const void *x_txt, int n_txt, const void *x_img, int n_img, int d,
                        bool fp32_tokens, float *resid, cudaStream_t s);
cudaError_t launch_unpack(const float *resid, int n_txt, int n_img, int d, bool fp32_tokens,
                          void *x_txt, void *x_img, cudaStream_t s);

}  // namespace h3
