/*
 * h3dit.h - C ABI of the B200 (sm_100a) DiT-block library for MiniMax-H3-Image.
 *
 * What it computes: the denoising forward of the dense single-stream DiT
 * block, repeated over the blocks of one sampling step.
 *   - MiniMax-H3-Image model card, "Model Architecture": text and image tokens
 *     form one packed sequence through a single-stream transformer with
 *     50 layers, hidden 5376, 56 heads, FFN 14336 and 3D multimodal RoPE;
 *     BF16 weights, FP32 timestep layers.
 *   - apxml "MiniMax H3 Image", "Architecture Diagram": per block, RMSNorm with
 *     timestep scale/shift -> joint attention -> "+" -> RMSNorm with timestep
 *     scale/shift -> GELU MLP -> "+".
 *   - "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin", "Faster DiT":
 *     the AdaLN conditioning projection is computed once and reused.
 *
 * Conventions shared by every entry point
 *   - Every pointer named "device" is CUDA device memory owned by the caller;
 *     the library never frees it. bf16 tensors are passed as raw 16-bit
 *     patterns (`void*`). Device pointers must be 16-byte aligned.
 *   - Matrices are row-major. Weights use the nn.Linear layout [out, in].
 *   - All work is enqueued on `cuda_stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and is asynchronous. No call synchronises except
 *     h3dit_sync_status (and h3dit_create, once, before it returns). Calls
 *     never abort or exit the process.
 *   - A context is used from one host thread at a time; two calls on one
 *     context must not overlap on the GPU (they share its workspace).
 *   - On an error, nothing is enqueued (validation happens first) unless the
 *     status is H3DIT_ERR_CUDA; h3dit_last_error(ctx) gives the message.
 */
#ifndef H3DIT_H
#define H3DIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t h3dit_status;
#define H3DIT_OK 0
#define H3DIT_ERR_INVALID_ARG (-1) /* a NULL, misaligned or out-of-range argument */
#define H3DIT_ERR_UNSUPPORTED (-2) /* a shape or head_dim this build does not run */
#define H3DIT_ERR_WORKSPACE (-3)   /* workspace too small or misaligned */
#define H3DIT_ERR_CUDA (-4)        /* a CUDA runtime or launch error */
#define H3DIT_ERR_TIMEOUT (-5)     /* a kernel's bounded wait gave up (see h3dit_sync_status) */

/* Empty inputs: a stage call whose row or token count is 0 (m of the
 * linears, n of the norms and the attention, n_local / n_total of the
 * sequence-parallel calls, rows of h3dit_mx_quantize, an empty RoPE table)
 * checks its counts and shape arguments, then returns H3DIT_OK without
 * launching anything or examining its data pointers, which may be NULL. */

/* Epilogues of h3dit_linear (steps a4, a6/a9, a8 of the block). */
#define H3DIT_EPI_STORE 0          /* out bf16 [m, n] = a w^T                          */
#define H3DIT_EPI_QKV_ROPE 1       /* as STORE, RoPE on columns < 2*heads*head_dim    */
#define H3DIT_EPI_GELU 2           /* out bf16 [m, n] = GELU(a w^T)                    */
#define H3DIT_EPI_GATED_RESIDUAL 3 /* out fp32 [m, n] += gate[col] * (a w^T)          */

#define H3DIT_PRECISION_BF16 0
#define H3DIT_PRECISION_MXFP8 1

typedef struct h3dit_config {
  int32_t hidden;           /* D, multiple of 64 (5376 for the model)                  */
  int32_t heads;            /* H (56)                                                  */
  int32_t head_dim;         /* d_h, 96 or 128 (the pages give both readings)           */
  int32_t ffn;              /* F, multiple of 64 (14336)                               */
  int32_t n_blocks;         /* L, blocks run by h3dit_step (50)                        */
  int32_t max_tokens;       /* largest packed sequence any call will pass              */
  int32_t rope_sections[3]; /* rotation pairs per (frame,row,col) axis; sum = d_h/2    */
  float rope_theta;         /* RoPE base (10000)                                       */
  float norm_eps;           /* RMSNorm epsilon (1e-6)                                  */
  float t_scale;            /* sinusoid argument is t_scale * t (1000)                 */
  int32_t gelu_tanh;        /* 0: exact erf GELU, 1: tanh approximation                */
  int32_t precision;        /* H3DIT_PRECISION_BF16, or _MXFP8: the four block linears
                               on MXFP8 operands (hidden, heads*head_dim and ffn must
                               then be multiples of 128)                            */
  int32_t io_fp32;          /* token buffers x_txt / x_img: 0 = bf16, 1 = fp32         */
} h3dit_config;

/* Timestep MLP, fp32, nn.Linear layout: Linear(256 -> D), SiLU, Linear(D -> D). */
typedef struct h3dit_time_weights {
  const float *w_t1; /* device [D, 256] */
  const float *b_t1; /* device [D]      */
  const float *w_t2; /* device [D, D]   */
  const float *b_t2; /* device [D]      */
} h3dit_time_weights;

/* One block's weights (bf16 unless noted), borrowed for the context's life. */
typedef struct h3dit_block_weights {
  const void *w_qkv;  /* device [3I, D]; rows [Q heads | K heads | V heads], I = H*d_h    */
  const void *w_o;    /* device [D, I]                                                   */
  const void *w_ff1;  /* device [F, D]                                                   */
  const void *w_ff2;  /* device [D, F]                                                   */
  const void *w_ada;  /* device [6D, D]; chunks shift1,scale1,gate1,shift2,scale2,gate2  */
  const float *b_ada; /* device fp32 [6D]                                                */
} h3dit_block_weights;

/* One latent image in the packed sequence: its RoPE frame index and grid.
 * Image tokens are row-major over (height, width). The target is frame 0;
 * reference image k is frame k. Text tokens sit at position (0, 0, 0). */
typedef struct h3dit_grid {
  int32_t frame, height, width;
} h3dit_grid;

typedef struct h3dit_ctx h3dit_ctx;

/* Name of a status code (static string). */
const char *h3dit_status_string(h3dit_status s);

/* Last error message of a context ("" if none; static text if ctx is NULL). */
const char *h3dit_last_error(const h3dit_ctx *ctx);

/* Bytes of device workspace h3dit_create needs for `cfg`, or 0 if `cfg` is
 * invalid. It covers the fp32 residual stream, the bf16 activations (xm,
 * Q|K|V, attention output, FFN hidden), the per-step modulation table
 * [n_blocks][6][D], the timestep vectors, the RoPE table and a status word;
 * with H3DIT_PRECISION_MXFP8 also the MXFP8 activations and their scales and
 * every block's quantized linears (E4M3 weights, their scales, and the
 * scales repacked for 224-column tiles where N is a multiple of 224). */
size_t h3dit_workspace_bytes(const h3dit_config *cfg);

/* Create a context. `blocks` points to cfg->n_blocks host structs whose
 * pointers must stay valid until h3dit_destroy. Each block's six weight
 * pointers are either all device memory or all pinned host memory
 * (cudaHostAlloc / cudaHostRegister, e.g. torch's pin_memory); host blocks are
 * streamed to the GPU layer by layer (see h3dit_attach_staging); pageable host
 * memory or a mix within one block is H3DIT_ERR_INVALID_ARG, and host blocks
 * with H3DIT_PRECISION_MXFP8 are H3DIT_ERR_UNSUPPORTED. The timestep weights
 * are device memory. `workspace` is device memory of at least
 * h3dit_workspace_bytes(cfg) bytes, 256-byte aligned, lent to the context for
 * its life. Copies the weight pointer table to the device and, with
 * H3DIT_PRECISION_MXFP8, quantizes every block's linears, on `cuda_stream`,
 * then synchronises that stream once before returning (the host-side table
 * must have been consumed). On error *out is set to NULL. */
h3dit_status h3dit_create(const h3dit_config *cfg, const h3dit_time_weights *time_w,
                          const h3dit_block_weights *blocks, void *workspace, size_t ws_bytes,
                          void *cuda_stream, h3dit_ctx **out);

/* Frees the host state of a context (NULL-safe). Device memory is the caller's. */
void h3dit_destroy(h3dit_ctx *ctx);

/* ---- Layerwise weight streaming ------------------------------------------
 * "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin", "Fitting Smaller
 * GPUs", and the vLLM-Omni recipe's "Deployment profiles" (DLO): the DiT's
 * blocks stay in pinned host memory and move to the GPU one block at a time.
 * Here a context whose blocks are partly or wholly in pinned host memory
 * copies each such block's six weight tensors (one cudaMemcpyAsync each) into
 * one of two device staging slots on a copy stream. The slots alternate: the
 * copy of the next-but-one host block starts as soon as a block has finished
 * with its slot, so it overlaps the block in between. Device-resident blocks
 * run as usual (their AdaLN projections still in one launch per step); a
 * host block's AdaLN projection is computed from its slot just before it
 * runs. Results are bit-identical to the same weights held on the device.
 * Every call is still ordered on its `cuda_stream`: the copy stream forks
 * from it at entry and joins it at exit (so a step can be graph-captured).
 * Placement: a block's copy can overlap only the compute that runs between
 * its slot's release and its own turn. With host blocks spaced evenly
 * through the step (resident blocks between them), each copy overlaps two or
 * more blocks of compute; with the host blocks in one run, only one. */

/* Bytes of staging memory h3dit_attach_staging needs for `cfg` (two slots of
 * one block's weights and a small pointer table), or 0 if `cfg` is invalid. */
size_t h3dit_staging_bytes(const h3dit_config *cfg);

/* Lend the context `staging`, device memory of at least
 * h3dit_staging_bytes(&cfg) bytes, 256-byte aligned, for its life (or until
 * the next attach), and the stream the weight copies run on: `copy_stream`,
 * or a stream the context creates (and destroys) when it is NULL. Writes the
 * slots' pointer table with one synchronous copy. Without staging, a call
 * that runs a host block returns H3DIT_ERR_WORKSPACE before enqueuing it. */
h3dit_status h3dit_attach_staging(h3dit_ctx *ctx, void *staging, size_t bytes, void *copy_stream);

/* Number of blocks whose weights are in host memory (-1 for a NULL ctx). */
int32_t h3dit_streamed_blocks(const h3dit_ctx *ctx);

/* Run block `block` in place on the packed sequence [x_txt; images]:
 *   x_txt  device [n_txt, D] (may be NULL when n_txt == 0), in/out;
 *   x_img  device [sum h*w, D], in/out, images in `grids` order;
 *          both bf16, or fp32 when cfg->io_fp32 is set;
 *   mod    device fp32 [6, D] modulation for this block, or NULL to compute it
 *          from `t` (timestep MLP then this block's AdaLN projection).
 * The residual stream is kept in fp32 inside the call; with bf16 token
 * buffers the result is rounded to bf16 once. Needs
 * 1 <= n_txt + sum h*w <= max_tokens. */
h3dit_status h3dit_block_forward(h3dit_ctx *ctx, int32_t block, float t, const float *mod,
                                 void *x_img, const h3dit_grid *grids, int32_t n_grids,
                                 void *x_txt, int32_t n_txt, void *cuda_stream);

/* One sampling step in place: the timestep MLP and all n_blocks AdaLN
 * projections once, then the n_blocks blocks in order with an fp32 residual
 * stream, written back to the token buffers at the end. Arguments as in
 * h3dit_block_forward. */
h3dit_status h3dit_step(h3dit_ctx *ctx, float t, void *x_img, const h3dit_grid *grids,
                        int32_t n_grids, void *x_txt, int32_t n_txt, void *cuda_stream);

/* Synchronise `cuda_stream`, then read and clear the context's device status
 * word. Returns H3DIT_ERR_TIMEOUT if a kernel's bounded wait gave up since the
 * last call, H3DIT_ERR_CUDA on a CUDA error, else H3DIT_OK. */
h3dit_status h3dit_sync_status(h3dit_ctx *ctx, void *cuda_stream);

/* ---- The steps of the path, one entry point each (same kernels the block
 * and step run; used to check and time each step on its own). ---------- */

/* a1: c = W_t2 SiLU(W_t1 e(t) + b_t1) + b_t2 with e(t) the 256-channel
 * sinusoid [cos | sin] of t_scale*t at frequencies 10000^(-i/128).
 * c_out: device fp32 [D]. Uses the context workspace as scratch. */
h3dit_status h3dit_time_embed(h3dit_ctx *ctx, float t, float *c_out, void *cuda_stream);

/* a2: mod[l] = W_ada[l] SiLU(c) + b_ada[l] for blocks l in [first, first+count).
 * c: device fp32 [D]; mod_out: device fp32 [count, 6, D]. */
h3dit_status h3dit_adaln_project(h3dit_ctx *ctx, const float *c, int32_t first, int32_t count,
                                 float *mod_out, void *cuda_stream);

/* a3/a7: xm = x / sqrt(mean(x^2) + eps) * (1 + scale) + shift, per row.
 * x: device fp32 [n, D]; shift, scale: device fp32 [D]; xm_out: device bf16 [n, D]. */
h3dit_status h3dit_rmsnorm_modulate(h3dit_ctx *ctx, const float *x, const float *shift,
                                    const float *scale, void *xm_out, int32_t n,
                                    void *cuda_stream);

/* RoPE table of the packed sequence: table_out device fp32 [n, d_h/2, 2]
 * holding (cos, sin) of each rotation pair's angle, pairs ordered frame axis,
 * row axis, col axis; n = n_txt + sum h*w. */
h3dit_status h3dit_rope_table(h3dit_ctx *ctx, const h3dit_grid *grids, int32_t n_grids,
                              int32_t n_txt, float *table_out, void *cuda_stream);

/* a4/a6/a8/a9: acc = a w^T with a device bf16 [m, k], w device bf16 [n, k];
 * k and n multiples of 64 and 32; then the epilogue (H3DIT_EPI_*):
 *   STORE / GELU  out: device bf16 [m, n];
 *   QKV_ROPE      out: device bf16 [m, n] with n = 3*heads*head_dim and
 *                 rope_table the table of h3dit_rope_table for these m tokens;
 *   GATED_RESIDUAL out: device fp32 [m, n], updated in place; gate: fp32 [n]. */
h3dit_status h3dit_linear(h3dit_ctx *ctx, int32_t epilogue, const void *a, const void *w,
                          int32_t m, int32_t n, int32_t k, void *out, const float *gate,
                          const float *rope_table, void *cuda_stream);

/* a5: O_h = softmax(Q_h K_h^T / sqrt(d_h)) V_h over all n tokens, no mask, for
 * every head. q, k, v: device bf16 [n, heads, d_h] rows with row stride ld_qkv
 * elements (the Q|K|V output of the QKV step has ld_qkv = 3*heads*d_h);
 * o: device bf16 [n, heads*d_h] with row stride ld_o. */
h3dit_status h3dit_attention(h3dit_ctx *ctx, const void *q, const void *k, const void *v,
                             int32_t ld_qkv, void *o, int32_t ld_o, int32_t n,
                             void *cuda_stream);

/* ---- Ulysses sequence parallelism over P ranks -------------------------
 * "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin", "Faster DiT"
 * (Ulysses SP4) and the vLLM-Omni recipe's "Deployment profiles" (SP 2,
 * SP 4). Each of P ranks holds n_local = N / P consecutive tokens of the
 * packed sequence and runs every step of the block but the attention on
 * them, with all heads. Around the attention two all-to-alls (NCCL, by the
 * caller) trade that for all N tokens and heads / P: the re-layouts on either
 * side are below, and h3dit_attention_heads runs the attention on the head
 * group. ranks must divide cfg->heads, and heads*head_dim/ranks must be a
 * multiple of 8. */

/* a5 for `heads` (1 .. cfg->heads) heads: as h3dit_attention with the heads
 * count given instead of cfg->heads (o gets heads*head_dim columns). */
h3dit_status h3dit_attention_heads(h3dit_ctx *ctx, int32_t heads, const void *q, const void *k,
                                   const void *v, int32_t ld_qkv, void *o, int32_t ld_o, int32_t n,
                                   void *cuda_stream);

/* Before the first all-to-all: qkv device bf16 [n_local, 3I] (this rank's
 * tokens, the QKV step's output) -> send device bf16 [ranks][n_local][3I/ranks]
 * (dense), where block d holds, for each row, the Q | K | V columns of heads
 * d*H/ranks .. (d+1)*H/ranks - 1. Sent block d to rank d, the receive buffer
 * [ranks][n_local][3I/ranks] of rank d is the Q|K|V matrix of its heads for
 * all tokens in sequence order, for h3dit_attention_heads with heads = H/ranks
 * and ld_qkv = 3I/ranks. */
h3dit_status h3dit_sp_pack_qkv(h3dit_ctx *ctx, const void *qkv, int32_t n_local, int32_t ranks,
                               void *send, void *cuda_stream);

/* After the second all-to-all (the attention output [N, I/ranks] of this
 * rank's heads sent in row blocks of n_local): recv device bf16
 * [ranks][n_local][I/ranks], block s from head group s -> o device bf16
 * [n_local, I] with head group s at columns s*I/ranks .. (s+1)*I/ranks - 1. */
h3dit_status h3dit_sp_unpack_o(h3dit_ctx *ctx, const void *recv, int32_t n_local, int32_t ranks,
                               void *o, void *cuda_stream);

/* The same two exchanges fused into the kernels that produce the data, for
 * ranks whose buffers are mapped into one another's address space (peer
 * memory over NVLink, opened with h3dit_ipc_open; or, on one GPU, plain
 * device buffers of emulated ranks). No NCCL call and no re-layout kernel:
 * the producing kernel stores each 16-byte piece straight into the rank that
 * needs it. ranks: 1 .. H3DIT_MAX_SCATTER_RANKS, dividing cfg->heads, with
 * heads*head_dim/ranks a multiple of 8; every pointer 16-byte aligned.
 * The calls do not synchronise between ranks: before a rank reads what the
 * others wrote (the attention after the QKV call, the out-projection after the
 * attention call), every rank's call must have completed, and before a rank
 * writes into a buffer, its owner must be done reading the previous
 * contents. The caller provides this with a barrier after each call (a
 * stream synchronise and a host barrier across the ranks); on one GPU, stream
 * order provides it. Errors: H3DIT_ERR_INVALID_ARG for NULL or misaligned
 * pointers, rank outside [0, ranks) or a bad count; H3DIT_ERR_UNSUPPORTED for
 * ranks that do not divide the heads, more than H3DIT_MAX_SCATTER_RANKS ranks,
 * or n_total not a multiple of ranks. */
#define H3DIT_MAX_SCATTER_RANKS 8

/* a4 with the first all-to-all: RMS-normalised, modulated tokens xm (device
 * bf16 [n_local, D], this rank's rows `rank` * n_local ..) times w_qkv, RoPE
 * on Q and K with rope_rows (this rank's rows of the sequence's table), each
 * head group's Q | K | V columns stored into recv[g] (device bf16
 * [ranks * n_local, 3I/ranks], rank g's receive buffer; recv is a host array
 * of `ranks` pointers) at rows rank*n_local .. - the layout that
 * h3dit_sp_pack_qkv plus the all-to-all produce. */
h3dit_status h3dit_sp_qkv_scatter(h3dit_ctx *ctx, const void *xm, int32_t n_local,
                                  const void *w_qkv, const float *rope_rows, void *const *recv,
                                  int32_t ranks, int32_t rank, void *cuda_stream);

/* a5 with the second all-to-all: attention of this rank's head group (heads
 * rank*H/ranks ..) over all n_total tokens, reading qkv (device bf16
 * [n_total, 3I/ranks], this rank's receive buffer), each output row t stored
 * into o[t / n_local] (device bf16 [n_local, I], the out-projection input of
 * the rank that holds token t; o is a host array of `ranks` pointers) at row
 * t % n_local, columns rank*I/ranks .. (rank+1)*I/ranks - 1. */
h3dit_status h3dit_sp_attention_scatter(h3dit_ctx *ctx, const void *qkv, int32_t n_total,
                                        void *const *o, int32_t ranks, int32_t rank,
                                        void *cuda_stream);

/* The same two fused exchanges for a context with H3DIT_PRECISION_MXFP8 (the
 * MXFP8 block of h3dit_block_linear_mx, run over ranks).
 * h3dit_sp_qkv_scatter_mx: as h3dit_sp_qkv_scatter, from this rank's
 * quantized rows xq (device E4M3 [n_local, D]) and their scales xq_sf (the
 * layout h3dit_rmsnorm_modulate_mx writes), with the context's quantized QKV
 * weights of `block`; the receive buffers stay bf16.
 * h3dit_sp_attention_scatter_mx: as h3dit_sp_attention_scatter, but each
 * output row is written as MXFP8, the input h3dit_block_linear_mx's
 * out-projection takes: E4M3 into o[t / n_local] (device [n_local, I]) and the
 * scales into o_sf[t / n_local] (device, h3dit_mx_scale_bytes(n_local, I)
 * bytes, the layout h3dit_mx_quantize writes), both host arrays of `ranks`
 * pointers. */
h3dit_status h3dit_sp_qkv_scatter_mx(h3dit_ctx *ctx, const void *xq, const void *xq_sf,
                                     int32_t n_local, int32_t block, const float *rope_rows,
                                     void *const *recv, int32_t ranks, int32_t rank,
                                     void *cuda_stream);
h3dit_status h3dit_sp_attention_scatter_mx(h3dit_ctx *ctx, const void *qkv, int32_t n_total,
                                           void *const *o, void *const *o_sf, int32_t ranks,
                                           int32_t rank, void *cuda_stream);

/* Peer-memory mapping for the calls above (CUDA IPC; host calls, no kernel).
 * h3dit_ipc_get_handle writes H3DIT_IPC_HANDLE_BYTES bytes that name the
 * allocation holding the device pointer dev_ptr, and *offset_out, dev_ptr's
 * byte offset in it; another process on the same node opens them with
 * h3dit_ipc_open, which maps the allocation (peer access enabled on demand)
 * and returns the address of the same byte in *dev_ptr_out. h3dit_ipc_close
 * unmaps what h3dit_ipc_open returned (pass that pointer, offset included).
 * Errors: H3DIT_ERR_INVALID_ARG for NULL arguments, H3DIT_ERR_CUDA when the
 * runtime refuses (the handle is from this process, the peer is not
 * reachable). */
#define H3DIT_IPC_HANDLE_BYTES 64
h3dit_status h3dit_ipc_get_handle(const void *dev_ptr, void *handle_out, uint64_t *offset_out);
h3dit_status h3dit_ipc_open(const void *handle, uint64_t offset, void **dev_ptr_out);
h3dit_status h3dit_ipc_close(void *dev_ptr, uint64_t offset);

/* ---- a11: the MXFP8 variant of the four block linears ------------------
 * "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin", "Faster DiT" and
 * "Rubin Bringup": MXFP8 GEMMs for the eligible DiT linears. Format (a
 * reading; the page names it only): OCP MX - E4M3 elements, one E8M0 scale
 * 2^X per 32 consecutive elements along the reduction axis (K), with
 * X = floor(log2(amax of the 32)) - 8, elements rounded to nearest even and
 * saturated at +-448. Scales are stored one byte each (X + 127) in 512-byte
 * blocks of 128 rows x 4 scales: block (row/128, k/128) at offset
 * ((row/128) * (K/128) + k/128) * 512, and within it row r's scale for
 * k-block s at (r % 32) * 16 + ((r / 32) % 4) * 4 + (k/32) % 4.
 * With cfg->precision = H3DIT_PRECISION_MXFP8, h3dit_create quantizes the
 * four linears of every block into the workspace, and block_forward / step
 * run them on MXFP8 activations made by their producers (RMSNorm, the
 * attention epilogue, the GELU epilogue); attention itself stays bf16. */

/* Bytes of the scale array of a [rows, k] MXFP8 matrix (0 unless k % 128 == 0). */
size_t h3dit_mx_scale_bytes(int32_t rows, int32_t k);

/* bf16 [rows, k] (device, dense) -> E4M3 [rows, k] (device, one byte each)
 * plus scales (device, h3dit_mx_scale_bytes(rows, k) bytes). */
h3dit_status h3dit_mx_quantize(h3dit_ctx *ctx, const void *src, int32_t rows, int32_t k, void *dst,
                               void *sf, void *cuda_stream);

/* MXFP8 linear: acc = a w^T with a E4M3 [m, k] + a_sf and w E4M3 [n, k] + w_sf;
 * k and n multiples of 128; epilogues as h3dit_linear, except GELU, which
 * writes MXFP8: out E4M3 [m, n] + out_sf (h3dit_mx_scale_bytes(m, n)). */
h3dit_status h3dit_linear_mx(h3dit_ctx *ctx, int32_t epilogue, const void *a, const void *a_sf,
                             const void *w, const void *w_sf, int32_t m, int32_t n, int32_t k,
                             void *out, void *out_sf, const float *gate, const float *rope_table,
                             void *cuda_stream);

/* The block's four linears, for h3dit_block_linear_mx. */
#define H3DIT_LINEAR_QKV 0  /* QKV + RoPE:            out bf16 [m, 3*heads*head_dim] */
#define H3DIT_LINEAR_OUT 1  /* out-proj, gated:       out fp32 [m, hidden] += gate * acc */
#define H3DIT_LINEAR_FFN1 2 /* FFN1 + GELU to MXFP8:  out E4M3 [m, ffn] + out_sf */
#define H3DIT_LINEAR_FFN2 3 /* FFN2, gated:           out fp32 [m, hidden] += gate * acc */

/* One of block `block`'s MXFP8 linears on the context's own quantized
 * weights (precision H3DIT_PRECISION_MXFP8 only), with that linear's
 * epilogue and through exactly the kernel h3dit_block_forward runs for it:
 * 128 x 224 tiles with the weight scales repacked per tile where N is a
 * multiple of 224 and every tile starts on a rotary-section boundary, else
 * 128 x 128 tiles. `a` E4M3 [m, k] + a_sf (h3dit_mx_scale_bytes(m, k)), k the
 * linear's input width; rope_table for H3DIT_LINEAR_QKV, gate for OUT and
 * FFN2, out_sf for FFN1. Returns H3DIT_ERR_UNSUPPORTED on a bf16 context. */
h3dit_status h3dit_block_linear_mx(h3dit_ctx *ctx, int32_t block, int32_t which, const void *a,
                                   const void *a_sf, int32_t m, void *out, void *out_sf,
                                   const float *gate, const float *rope_table, void *cuda_stream);

/* a3/a7 with an MXFP8 output: out E4M3 [n, D] + out_sf. */
h3dit_status h3dit_rmsnorm_modulate_mx(h3dit_ctx *ctx, const float *x, const float *shift,
                                       const float *scale, void *out, void *out_sf, int32_t n,
                                       void *cuda_stream);

/* a5 with an MXFP8 output for the MXFP8 out-projection: o E4M3
 * [n, heads*head_dim] (dense) + o_sf; heads*head_dim a multiple of 128. */
h3dit_status h3dit_attention_mx(h3dit_ctx *ctx, const void *q, const void *k, const void *v,
                                int32_t ld_qkv, void *o, void *o_sf, int32_t n, void *cuda_stream);

/* ---- Around the block loop: latent in, velocity out, sampler step --------
 * MiniMax-H3-Image model card, "Model Architecture": the image VAE's latent
 * has 24 channels at 16x spatial downsampling; the DiT patchifies it with a
 * 2x2 patch (one token per 32x32 pixels); the embedding, timestep and output
 * layers are FP32. The real per-step output heads and sampling schedule are
 * not on the pages; a DiT output layer predicting the flow velocity dz/dt and
 * an Euler step stand in for them.
 * Latents are device fp32 [C, Hl, Wl] (channel-major), Hl and Wl even, C <= 32.
 * Token (r, c) of a latent is row-major over its (Hl/2, Wl/2) patch grid, the
 * order h3dit_grid gives an image; feature ch*4 + 2i + j of a token is latent
 * pixel (2r + i, 2c + j) of channel ch. */

/* Patchify + FP32 patch embedding: x_img_out[t] = W_in patch(t) + b_in.
 *   w_in device fp32 [D, 4C]; b_in device fp32 [D];
 *   x_img_out device [(Hl/2)(Wl/2), D] in the context's token dtype (bf16,
 *   or fp32 with io_fp32), ready for h3dit_step as the target image. */
h3dit_status h3dit_embed_latent(h3dit_ctx *ctx, const float *latent, int32_t channels,
                                int32_t lat_h, int32_t lat_w, const float *w_in, const float *b_in,
                                void *x_img_out, void *cuda_stream);

/* The output layer's modulation: mod_out[0:D] = shift, mod_out[D:2D] = scale,
 * = W_mod SiLU(c) + b_mod. c device fp32 [D] (h3dit_time_embed's output);
 * w_mod device fp32 [2D, D]; b_mod [2D]; mod_out device fp32 [2D]. */
h3dit_status h3dit_output_modulation(h3dit_ctx *ctx, const float *c, const float *w_mod,
                                     const float *b_mod, float *mod_out, void *cuda_stream);

/* Output layer, unpatchify and one Euler step of the flow, in place on the
 * latent: v = unpatchify((RMSNorm(x) (1 + scale) + shift) W_out^T + b_out);
 * latent += dt * v (dt = t_next - t, negative when denoising from t = 1 to 0).
 *   x_img device [(Hl/2)(Wl/2), D], the target image's tokens after h3dit_step,
 *   in the context's token dtype; mod device fp32 [2D] from
 *   h3dit_output_modulation; w_out device fp32 [4C, D]; b_out [4C].
 * Uses the context's residual workspace as scratch (one float per token). */
h3dit_status h3dit_output_euler(h3dit_ctx *ctx, const void *x_img, const float *mod,
                                const float *w_out, const float *b_out, float *latent,
                                int32_t channels, int32_t lat_h, int32_t lat_w, float dt,
                                void *cuda_stream);

/* The FP32 layers around the block loop, for h3dit_denoise (C = latent
 * channels; all device fp32, nn.Linear layout). */
typedef struct h3dit_io_weights {
  const float *w_in;  /* [D, 4C] patch embedding      */
  const float *b_in;  /* [D]                          */
  const float *w_mod; /* [2D, D] output modulation    */
  const float *b_mod; /* [2D]  (shift rows, then scale rows) */
  const float *w_out; /* [4C, D] output layer         */
  const float *b_out; /* [4C]                         */
} h3dit_io_weights;

/* The whole sampling loop on one target latent, in place: n_steps Euler steps
 * of the flow from t = 1 (noise) to t = 0 at t_k = 1 - k / n_steps (the model
 * card's "6 sampling steps" with the plain uniform schedule; the real schedule
 * file is not on the pages). Each step runs, all on `cuda_stream`:
 *   the timestep MLP and every block's AdaLN projection at t_k, and the output
 *   layer's modulation; the text states x_txt and the patch embedding of the
 *   latent packed into the fp32 residual stream [text; image]; the n_blocks
 *   blocks; the output layer on the image rows; latent += (t_{k+1} - t_k) v.
 *   latent  device fp32 [C, Hl, Wl], noise in, denoised latent out; Hl, Wl
 *           even, C <= 32; the target image is frame 0 of grid (Hl/2, Wl/2);
 *   x_txt   device [n_txt, D] in the context's token dtype, read only (the
 *           same text states enter every step); NULL when n_txt == 0;
 *   n_steps 1 .. 1000.
 * Needs n_txt + (Hl/2)(Wl/2) <= max_tokens. The token buffers of h3dit_step
 * are not used: the residual stream stays in the workspace between the
 * embedding and the output layer. */
h3dit_status h3dit_denoise(h3dit_ctx *ctx, const h3dit_io_weights *io, float *latent,
                           int32_t channels, int32_t lat_h, int32_t lat_w, const void *x_txt,
                           int32_t n_txt, int32_t n_steps, void *cuda_stream);

/* ---- The image VAE's ViT decoder (shape level) -------------------------
 * MiniMax-H3-Image model card, "Model Architecture": the image VAE has a CNN
 * encoder and a 2D ViT decoder with 24 layers, 16x spatial downsampling and
 * 24 latent channels. "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin",
 * "Faster Decoding": the VAE decodes independent image tiles. The pages give
 * no more, so the decoder is a plain reading of those words, run on random
 * weights for its shape and cost:
 *   - one token per latent pixel: Linear(C -> W) + bias, plus a fixed 2-D
 *     sin-cos position table over the position inside the tile (first W/2
 *     channels the row r, last W/2 the column c, each [sin(p w_k) | cos(p w_k)]
 *     for k < W/4 with w_k = 10000^(-k/(W/4)));
 *   - `layers` pre-norm ViT layers: x += (attention over the tile's tokens of
 *     LN1(x) W_qkv^T + b_qkv) W_o^T + b_o; x += GELU(LN2(x) W_1^T + b_1) W_2^T
 *     + b_2; LayerNorm with gain and bias; attention unmasked, scale
 *     1/sqrt(head_dim), no rotary embedding;
 *   - a final LayerNorm, Linear(W -> 3*16*16) + bias, and each token's 768
 *     outputs as its 16 x 16 RGB pixel block (feature ch*256 + 16i + j at
 *     pixel (16r + i, 16c + j) of channel ch);
 *   - the latent cut into non-overlapping tile x tile pieces decoded
 *     independently (all tiles of a call at once: the row-wise steps over all
 *     tokens, the attention batched over tiles).
 * Linears run on bf16 operands with fp32 accumulation (the pages report a
 * BF16 decode control; the checkpoint is FP32); the residual stream is fp32. */

typedef struct h3dit_vae_config {
  int32_t width;      /* W, multiple of 64 (1280)                                 */
  int32_t heads;      /* attention heads (10)                                     */
  int32_t head_dim;   /* 96 or 128 (128)                                          */
  int32_t mlp;        /* MLP width, multiple of 64 (5120)                         */
  int32_t layers;     /* ViT layers (24)                                          */
  int32_t tile;       /* latent pixels per tile side (32 = 512 image pixels)      */
  int32_t channels;   /* latent channels, 1 .. 32 (24)                            */
  int32_t max_tokens; /* largest latent Hl*Wl a decode will pass                  */
  float eps;          /* LayerNorm epsilon (1e-6)                                 */
} h3dit_vae_config;

/* One decoder layer: bf16 matrices in the nn.Linear layout, fp32 vectors,
 * all device memory borrowed for the context's life. */
typedef struct h3dit_vae_layer_weights {
  const float *ln1_g, *ln1_b; /* [W]                                                  */
  const void *w_qkv;          /* [3 H d, W]; rows [Q heads | K heads | V heads]       */
  const float *b_qkv;         /* [3 H d]                                              */
  const void *w_o;            /* [W, H d]                                             */
  const float *b_o;           /* [W]                                                  */
  const float *ln2_g, *ln2_b; /* [W]                                                  */
  const void *w_1;            /* [mlp, W]                                             */
  const float *b_1;           /* [mlp]                                                */
  const void *w_2;            /* [W, mlp]                                             */
  const float *b_2;           /* [W]                                                  */
} h3dit_vae_layer_weights;

typedef struct h3dit_vae_weights {
  const float *w_in, *b_in;              /* fp32 [W, C], [W]                          */
  const h3dit_vae_layer_weights *layers; /* host array of cfg->layers                 */
  const float *lnf_g, *lnf_b;            /* [W]                                       */
  const void *w_out;                     /* bf16 [768, W]                             */
  const float *b_out;                    /* [768]                                     */
} h3dit_vae_weights;

/* Device workspace a decoder context needs, or 0 if `cfg` is invalid. */
size_t h3dit_vae_workspace_bytes(const h3dit_vae_config *cfg);

/* A decoder context (used with h3dit_vae_decode, the stage entry points
 * below, h3dit_sync_status, the profile hooks and h3dit_destroy; the DiT
 * calls refuse it). Workspace as in h3dit_create. Writes the position table
 * into the workspace on `cuda_stream` and synchronises it once. */
h3dit_status h3dit_vae_create(const h3dit_vae_config *cfg, const h3dit_vae_weights *w,
                              void *workspace, size_t ws_bytes, void *cuda_stream,
                              h3dit_ctx **out);

/* latent device fp32 [C, Hl, Wl] -> image device fp32 [3, 16 Hl, 16 Wl].
 * Hl and Wl must be multiples of cfg->tile (H3DIT_ERR_UNSUPPORTED otherwise)
 * and Hl*Wl <= max_tokens. */
h3dit_status h3dit_vae_decode(h3dit_ctx *ctx, const float *latent, int32_t lat_h, int32_t lat_w,
                              float *image, void *cuda_stream);

/* LayerNorm with gain and bias: x device fp32 [n, width] -> out device bf16
 * [n, width] (width = the context's hidden, or W of a decoder context). */
h3dit_status h3dit_layernorm(h3dit_ctx *ctx, const float *x, const float *gain, const float *bias,
                             void *out, int32_t n, void *cuda_stream);

/* h3dit_linear with a bias b (device fp32 [n]) added to the product before the
 * epilogue step: STORE and GELU write bf16 (a w^T + b), GATED_RESIDUAL adds
 * gate * (a w^T + b) to the fp32 out; QKV_ROPE is not offered with a bias. */
h3dit_status h3dit_linear_bias(h3dit_ctx *ctx, int32_t epilogue, const void *a, const void *w,
                               const float *bias, int32_t m, int32_t n, int32_t k, void *out,
                               const float *gate, void *cuda_stream);

/* a5 over `batch` independent sequences of n tokens stored one after another
 * (rows z*n .. z*n + n - 1 of q, k, v and o): as h3dit_attention_heads with
 * heads = cfg heads, each sequence attending only to itself. */
h3dit_status h3dit_attention_batched(h3dit_ctx *ctx, const void *q, const void *k, const void *v,
                                     int32_t ld_qkv, void *o, int32_t ld_o, int32_t n,
                                     int32_t batch, void *cuda_stream);

/* ---- Timestep condition without any device allocation ----------------- */

/* Largest `hidden` h3dit_time_embed_static accepts. */
#define H3DIT_STATIC_TIME_MAX_HIDDEN 8192

/* a1 without a context or a workspace: c_out = W_t2 SiLU(W_t1 e(t) + b_t1) + b_t2,
 * the same computation and kernels as h3dit_time_embed. The paper has no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory at all - for example code running inside a host application
 * that owns every device allocation and hands a plugin only the buffers it
 * reads and writes, or a serving process that forbids allocation after
 * start-up to keep its footprint fixed. Such a caller cannot provide the
 * workspace a context needs, so this entry point takes the weights and the
 * output directly and keeps its one scratch vector (the hidden layer, `hidden`
 * floats) in a fixed array inside the library.
 *   w_t1 device fp32 [hidden, 256]; b_t1 [hidden]; w_t2 [hidden, hidden];
 *   b_t2 [hidden]; c_out device fp32 [hidden]; t_scale as in h3dit_config.
 * Neither this call nor the library allocates or frees device memory for it.
 * The scratch array holds H3DIT_STATIC_TIME_MAX_HIDDEN floats (32 KiB) on every
 * GPU that loads the library, until the process exits; hidden larger than
 * that returns H3DIT_ERR_UNSUPPORTED, bad pointers or hidden < 1 or not a
 * multiple of 4 return H3DIT_ERR_INVALID_ARG, both before anything is
 * enqueued. The first call on a device looks up the array's device address
 * for that device (once per device, with it current) and keeps it for the
 * life of the process; make that first call before any stream capture. A
 * cudaDeviceReset on a device destroys the array with the context and the
 * kept address then no longer refers to it, so do not call this entry point
 * on a device after resetting it. Every call on a device shares the one array and
 * overwrites all of it that it reads, so nothing carries over between calls;
 * two calls that overlap on the GPU (different streams, not ordered) race on
 * it and must be avoided. */
h3dit_status h3dit_time_embed_static(const float *w_t1, const float *b_t1, const float *w_t2,
                                     const float *b_t2, int32_t hidden, float t, float t_scale,
                                     float *c_out, void *cuda_stream);

/* ---- Failure detection ---------------------------------------------------
 * Every wait inside the library's kernels (on an mbarrier fed by TMA or by
 * another warp) gives up after about one second, records H3DIT_ERR_TIMEOUT in
 * the context's status word and lets the kernel unwind; kernels that start
 * while the word is set do no work. h3dit_sync_status reports and clears it.
 * This entry point exercises that path on purpose without faulting anything:
 * one thread waits on an mbarrier that nothing arrives on, for limit_us
 * microseconds (1 .. 1e6), then records the timeout and returns. */
h3dit_status h3dit_selftest_bounded_wait(h3dit_ctx *ctx, int32_t limit_us, void *cuda_stream);

/* ---- Measurement hooks (for benchmarks and profilers) ----------------- */

/* Kernel kinds the library launches, for h3dit_profile_end. */
#define H3DIT_KERNEL_TIME_EMBED 0 /* a1 (two small launches)      */
#define H3DIT_KERNEL_ADALN 1      /* a2                            */
#define H3DIT_KERNEL_RMSNORM 2    /* a3, a7                        */
#define H3DIT_KERNEL_QKV 3        /* a4                            */
#define H3DIT_KERNEL_ATTENTION 4  /* a5                            */
#define H3DIT_KERNEL_OUT_PROJ 5   /* a6                            */
#define H3DIT_KERNEL_FFN1 6       /* a8                            */
#define H3DIT_KERNEL_FFN2 7       /* a9                            */
#define H3DIT_KERNEL_ROPE_TABLE 8 /* RoPE table of the sequence    */
#define H3DIT_KERNEL_PACK 9       /* packing / unpacking tokens    */
#define H3DIT_KERNEL_MX_QUANTIZE 10 /* h3dit_mx_quantize           */
#define H3DIT_KERNEL_IO 11        /* patch embedding, output layer + Euler */
#define H3DIT_KERNEL_COUNT 12

/* Start recording a CUDA event pair around every kernel the context launches
 * (on the stream it is launched on), dropping earlier records. */
h3dit_status h3dit_profile_begin(h3dit_ctx *ctx);

/* Stop recording; wait for the recorded events and write, per kernel kind,
 * the summed device time in ms and the number of launches (arrays of
 * H3DIT_KERNEL_COUNT entries; either may be NULL). */
h3dit_status h3dit_profile_end(h3dit_ctx *ctx, float *ms_out, int64_t *launches_out);

/* Kernels this context has enqueued since it was created. */
int64_t h3dit_launch_count(const h3dit_ctx *ctx);

/* Per-phase clock stamps of the attention kernel, for the diagnostic build
 * (`python -m image_generation_b200.build --stamps` writes
 * libh3dit_stamps.so with the stamp points compiled in; the product library
 * has none and returns H3DIT_ERR_UNSUPPORTED). One CTA of every launch (query
 * tiles 40-41 of head 10) records clock64() at fixed points of each 64-key
 * step into a device table of H3DIT_ATTN_STAMP_SLOTS x H3DIT_ATTN_STAMP_STEPS
 * entries (step-major; the slot layout is documented in csrc/attention.cu);
 * this copies the table of the last such launch to `host` (synchronous).
 * slots and steps must equal the two constants. */
#define H3DIT_ATTN_STAMP_SLOTS 32
#define H3DIT_ATTN_STAMP_STEPS 300
h3dit_status h3dit_attention_stamps(uint64_t *host, int32_t slots, int32_t steps);

#ifdef __cplusplus
}
#endif
#endif /* H3DIT_H */
