// Host-side launchers of the sm_100a kernels (internal to libh3dit).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

namespace h3 {

// A value computed once per device for the whole process (a kernel attribute
// such as the dynamic shared-memory limit takes effect only on the device
// that is current when it is set, and occupancy differs between devices).
// Each launcher keeps one of these per kernel instance; the first launch on a
// device computes it under a lock, later ones read it without one, so host
// threads that drive different devices may race on first use.
constexpr int kMaxDevices = 64;
struct PerDevice {
  std::mutex mu;
  std::atomic<int> value[kMaxDevices];
  PerDevice() {
    for (auto &v : value) v.store(-1, std::memory_order_relaxed);
  }
};
// Runs `compute(int *v)` on the current device unless it has succeeded there
// before; *out (optional) receives the stored value (>= 0).
template <typename F>
inline cudaError_t per_device(PerDevice &pd, F &&compute, int *out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int v = pd.value[dev].load(std::memory_order_acquire);
  if (v < 0) {
    std::lock_guard<std::mutex> lock(pd.mu);
    v = pd.value[dev].load(std::memory_order_relaxed);
    if (v < 0) {
      int got = 0;
      e = compute(&got);
      if (e != cudaSuccess) return e;
      v = got < 0 ? 0 : got;
      pd.value[dev].store(v, std::memory_order_release);
    }
  }
  if (out) *out = v;
  return cudaSuccess;
}
// The common case: raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
inline cudaError_t set_smem_once(PerDevice &pd, K *kernel, int bytes) {
  return per_device(pd, [&](int *v) {
    *v = 1;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
}

enum Epilogue : int {
  kEpiStore = 0,
  kEpiQkvRope = 1,
  kEpiGelu = 2,
  kEpiGatedResidual = 3,
  kEpiGeluMx = 4,  // GELU, written as MXFP8 (E4M3 + per-32 E8M0 scales)
};

// MXFP8 scale-factor layout (one E8M0 byte per 32 elements along K) for a
// matrix [rows, K], K a multiple of 128: 512-byte blocks of 128 rows x 4
// scales, block (row/128, k/128) at ((row/128) * (K/128) + k/128) * 512, and
// inside a block row r's scale s at (r % 32) * 16 + ((r / 32) % 4) * 4 + s % 4.
// This is the order tcgen05.cp (32x128b, warpx4) moves into tensor memory
// for the block-scaled MMA: lane r % 32, column (r / 32) % 4, byte s % 4.
__host__ __device__ inline size_t mx_sf_offset(int row, int s, int k_chunks) {
  return (static_cast<size_t>(row >> 7) * k_chunks + (s >> 2)) * 512 + (row & 31) * 16 +
         ((row >> 5) & 3) * 4 + (s & 3);
}
inline size_t mx_sf_bytes(long long rows, long long k) {
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>(k / 128) * 512;
}

// Ranks a fused Ulysses exchange can address (destination pointers carried
// in the kernel parameters).
constexpr int kMaxScatterRanks = 8;

struct GemmParams {
  int m, n, k;
  int tiles_m, tiles_n;
  void *out;
  long long ldo;          // elements
  const float *gate;      // gated residual: [n]
  const float *bias;      // optional [n], added to the product before the epilogue step
  const float *rope;      // QKV: [m][head_dim/2][2]
  int head_dim;           // QKV
  int rope_cols;          // QKV: RoPE on columns < rope_cols (Q and K)
  int sec[3];             // QKV: rotation pairs per axis
  int gelu_tanh;
  int *status;
  // MXFP8 only
  const uint8_t *a_sf, *b_sf;  // scale factors of A [m, k] and W [n, k]
  uint8_t *out_sf;             // GELU-MXFP8 epilogue: scales of out [m, n]
  // QKV + RoPE with the first Ulysses all-to-all fused in (scatter_ranks > 0):
  // column c of matrix q (0 Q, 1 K, 2 V) in head group g = c / scatter_cols
  // of output row r goes to scatter[g] at row scatter_rank * m + r, column
  // q * scatter_cols + c % scatter_cols, of a [ranks * m, 3 * scatter_cols]
  // bf16 buffer; `out` is unused.
  void *scatter[kMaxScatterRanks];
  int scatter_ranks, scatter_rank;
  int scatter_inner;           // heads * head_dim (width of one of Q, K, V)
  int scatter_cols;            // columns of one head group
};

struct AttnParams {
  int n;                  // tokens of one sequence (blockIdx.z picks the sequence)
  int batch;              // sequences, stored one after another (rows z n .. z n + n - 1)
  int tiles_kv;
  void *o;
  long long ldo;          // elements
  float scale_log2;       // log2(e) / sqrt(head_dim)
  int *status;
  uint8_t *o_sf;          // MXFP8 output: scales of o [n, heads*head_dim]
  // The second Ulysses all-to-all fused in (o_scatter_ranks > 0): output row
  // t goes to o_scatter[t / o_rows_per_rank] at row t % o_rows_per_rank,
  // column o_col0 + head * head_dim, with row stride ldo (and its MXFP8
  // scales to o_sf_scatter of the same rank); `o` and `o_sf` are unused.
  void *o_scatter[kMaxScatterRanks];
  uint8_t *o_sf_scatter[kMaxScatterRanks];  // MXFP8 output: the owners' scale arrays
  int o_scatter_ranks;
  int o_rows_per_rank;
  int o_col0;
};

// Tile of the tcgen05 GEMM (rows x columns of the output).
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;

// Copies the attention kernel's clock stamps (built with -DH3_ATTN_STAMPS)
// to host: 0 on success, 1 in a build without them, negative on errors.
int attention_stamps(unsigned long long *host, int slots, int steps);

cudaError_t launch_gemm(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p,
                        int epilogue, int grid, cudaStream_t s);
int gemm_smem_bytes();

// The same GEMM on 256 x 256 tiles computed by clusters of two CTAs
// (tcgen05.mma.cta_group::2); grid = 2 x the number of clusters.
#ifndef H3_GEMM_PAIR
#define H3_GEMM_PAIR 1
#endif
cudaError_t launch_gemm_pair(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p,
                             int epilogue, int grid, cudaStream_t s);
// Clusters of the paired kernel that fit on the device at once (0: unusable).
int gemm_pair_max_clusters(int epilogue);

// Attention tiles: 128 queries per query tile (two per CTA), 64 keys per KV
// tile (two S buffers per query tile in TMEM).
constexpr int kAttnBQ = 128;
constexpr int kAttnBKV = 64;
cudaError_t launch_attention(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                             const AttnParams &p, int head_dim, int heads, bool out_mx,
                             cudaStream_t s);

// MXFP8 block-scaled GEMM (tiles 128 x 128, K-blocks of 128): A [m, k] and
// W [n, k] as E4M3 with scales in the mx_sf layout.
constexpr int kGemmMxBN = 128;
constexpr int kGemmMxBK = 128;
// Wide tiles (128 x 224) take W scales repacked per tile: for tile t and
// k-block kb, the two 512-byte blocks of rows 224 t .. 224 t + 127 and
// 224 t + 128 .. 224 t + 255 (standard in-block order) at (t * (k/128) + kb) * 1024.
constexpr int kGemmMxWideBN = 224;
inline size_t mx_sf_tiled_bytes(long long n, long long k) {
  return static_cast<size_t>(n / kGemmMxWideBN) * static_cast<size_t>(k / 128) * 1024;
}
cudaError_t launch_gemm_mx(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p,
                           int epilogue, int grid, bool wide, cudaStream_t s);
// Around the block loop (io_layers.cu): 2x2 patchify + FP32 embedding into
// tokens; the output layer's modulation; output layer + unpatchify + Euler.
cudaError_t launch_embed_latent(const float *z, int C, int Hl, int Wl, const float *w_in,
                                const float *b_in, int D, void *out, bool out_fp32,
                                cudaStream_t s);
cudaError_t launch_output_modulation(const float *c, const float *w_mod, const float *b_mod,
                                     float *mod, int D, cudaStream_t s);
cudaError_t launch_output_euler(const void *x, bool in_fp32, const float *mod, const float *w_out,
                                const float *b_out, int D, float eps, float *z, int C, int Hl,
                                int Wl, float dt, float *rinv_scratch, cudaStream_t s);
// Ulysses sequence parallelism (sp.cu): the re-layouts around the two
// all-to-alls; cw = columns of one head group per matrix (I / ranks).
cudaError_t launch_sp_pack_qkv(const void *qkv, int n, int ranks, int cw, void *send, int num_sms,
                               cudaStream_t s);
cudaError_t launch_sp_unpack_o(const void *recv, int n, int ranks, int cw, void *o, int num_sms,
                               cudaStream_t s);
// The VAE decoder's own steps (vae.cu).
cudaError_t launch_layernorm(const float *x, const float *gain, const float *bias, void *out,
                             int n, int d, float eps, int num_sms, cudaStream_t s);
cudaError_t launch_vae_pos_table(int T, int W, float *table, int num_sms, cudaStream_t s);
cudaError_t launch_vae_embed(const float *z, int C, int Hl, int Wl, int T, const float *w_in,
                             const float *b_in, const float *table, int W, float *out,
                             cudaStream_t s);
cudaError_t launch_vae_pixels(const void *tokens, int Hl, int Wl, int T, float *img, int num_sms,
                              cudaStream_t s);
cudaError_t launch_mx_tile_sf(const uint8_t *sf, int n, int k, uint8_t *tiled, cudaStream_t s);
// bf16 [rows, k] (row stride ld elements) -> E4M3 [rows, k] + scales.
cudaError_t launch_mx_quantize(const void *src, long long ld, int rows, int k, uint8_t *dst,
                               uint8_t *sf, cudaStream_t s);

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
                                    cudaStream_t s, uint8_t *out_sf = nullptr);

// Bounded-wait self-test: one thread waits on an mbarrier that nothing
// arrives on, gives up after limit_cycles and records the timeout in *status.
cudaError_t launch_selftest_wait(int *status, long long limit_cycles, cudaStream_t s);

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
