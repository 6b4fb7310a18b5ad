// C ABI of libh3dit (declared in include/h3dit.h): argument checks, the
// workspace plan, TMA tensor-map encoding and the order of kernel launches
// for one DiT block and one sampling step. All compute runs in the kernels of
// gemm.cu, gemm_pair.cu, gemm_mx.cu, attention.cu and elementwise.cu; this
// file only marshals.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/h3dit.h"
#include "kernels.h"

using namespace h3;

namespace {

constexpr size_t kAlign = 256;
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-block MXFP8 weights (E4M3 + scales), made at create.
struct MxWeights {
  size_t qkv, qkv_sf, o, o_sf, ff1, ff1_sf, ff2, ff2_sf;
  // W scales repacked for 224-column tiles (kNoTiled where N is not a multiple of 224)
  size_t qkv_sft, o_sft, ff1_sft, ff2_sft;
};
constexpr size_t kNoTiled = ~static_cast<size_t>(0);

struct Layout {
  size_t status, resid, xm, qkv, attn, u, mod, cvec, hidden, omod, rope, wptr, bptr;
  // MXFP8 precision only
  size_t xq, xq_sf, oq, oq_sf, uq, uq_sf, wq, wq_block;
  MxWeights wq_off;  // offsets inside one block's slice of the wq arena
  size_t total;
};

bool config_ok(const h3dit_config *c) {
  if (!c) return false;
  if (c->hidden <= 0 || c->hidden % 64 || c->hidden > 8192) return false;
  if (c->heads <= 0 || (c->head_dim != 96 && c->head_dim != 128)) return false;
  if (c->ffn <= 0 || c->ffn % 64) return false;
  if (c->n_blocks <= 0 || c->max_tokens <= 0) return false;
  const int pairs = c->rope_sections[0] + c->rope_sections[1] + c->rope_sections[2];
  if (2 * pairs != c->head_dim) return false;
  for (int a = 0; a < 3; ++a)
    if (c->rope_sections[a] != 16 && c->rope_sections[a] != 24) return false;
  if (!(c->norm_eps >= 0.f) || !(c->rope_theta > 0.f)) return false;
  if (c->precision != H3DIT_PRECISION_BF16 && c->precision != H3DIT_PRECISION_MXFP8) return false;
  if (c->io_fp32 != 0 && c->io_fp32 != 1) return false;
  if (c->precision == H3DIT_PRECISION_MXFP8 &&
      (c->hidden % 128 || (c->heads * c->head_dim) % 128 || c->ffn % 128))
    return false;
  return true;
}

Layout plan(const h3dit_config *c) {
  Layout L{};
  const size_t N = static_cast<size_t>(c->max_tokens);
  const size_t D = c->hidden, I = static_cast<size_t>(c->heads) * c->head_dim, F = c->ffn;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes, kAlign);
    return at;
  };
  L.status = take(kAlign);
  L.resid = take(N * D * 4);
  L.xm = take(N * D * 2);
  L.qkv = take(N * 3 * I * 2);
  L.attn = take(N * I * 2);
  L.u = take(N * F * 2);
  L.mod = take(static_cast<size_t>(c->n_blocks) * 6 * D * 4);
  L.cvec = take(D * 4);
  L.hidden = take(D * 4);
  L.omod = take(2 * D * 4);
  L.rope = take(N * (c->head_dim / 2) * 2 * 4);
  L.wptr = take(static_cast<size_t>(c->n_blocks) * sizeof(void *));
  L.bptr = take(static_cast<size_t>(c->n_blocks) * sizeof(void *));
  if (c->precision == H3DIT_PRECISION_MXFP8) {
    L.xq = take(N * D);
    L.xq_sf = take(mx_sf_bytes(N, D));
    L.oq = take(N * I);
    L.oq_sf = take(mx_sf_bytes(N, I));
    L.uq = take(N * F);
    L.uq_sf = take(mx_sf_bytes(N, F));
    size_t b = 0;
    auto sub = [&](size_t bytes) {
      const size_t at = b;
      b = round_up(b + bytes, kAlign);
      return at;
    };
    L.wq_off.qkv = sub(3 * I * D);
    L.wq_off.qkv_sf = sub(mx_sf_bytes(3 * I, D));
    L.wq_off.o = sub(D * I);
    L.wq_off.o_sf = sub(mx_sf_bytes(D, I));
    L.wq_off.ff1 = sub(F * D);
    L.wq_off.ff1_sf = sub(mx_sf_bytes(F, D));
    L.wq_off.ff2 = sub(D * F);
    L.wq_off.ff2_sf = sub(mx_sf_bytes(D, F));
    auto tiled = [&](size_t n, size_t k) {
      return n % kGemmMxWideBN ? kNoTiled : sub(mx_sf_tiled_bytes(n, k));
    };
    L.wq_off.qkv_sft = tiled(3 * I, D);
    L.wq_off.o_sft = tiled(D, I);
    L.wq_off.ff1_sft = tiled(F, D);
    L.wq_off.ff2_sft = tiled(D, F);
    L.wq_block = b;
    L.wq = take(b * static_cast<size_t>(c->n_blocks));
  }
  L.total = off;
  return L;
}

// Layerwise weight streaming: two slots, each holding one block's weights
// (same layout as h3dit_block_weights), then a table of the two slots' w_ada
// and b_ada pointers for the AdaLN kernel.
struct Staging {
  size_t part[6];  // offsets in a slot: w_qkv, w_o, w_ff1, w_ff2, w_ada, b_ada
  size_t bytes[6]; // bytes of each part
  size_t slot;     // bytes of one slot
  size_t table;    // offset of the pointer table (2 x w_ada, then 2 x b_ada)
  size_t total;
};

Staging staging_plan(const h3dit_config *c) {
  Staging S{};
  const size_t D = c->hidden, I = static_cast<size_t>(c->heads) * c->head_dim, F = c->ffn;
  const size_t b[6] = {3 * I * D * 2, D * I * 2, F * D * 2, D * F * 2, 6 * D * D * 2, 6 * D * 4};
  size_t off = 0;
  for (int i = 0; i < 6; ++i) {
    S.part[i] = off;
    S.bytes[i] = b[i];
    off = round_up(off + b[i], kAlign);
  }
  S.slot = off;
  S.table = 2 * S.slot;
  S.total = S.table + kAlign;
  return S;
}

// A VAE decoder context runs its layers through the block's machinery: the
// same workspace plan with hidden = W, ffn = mlp, n_blocks = layers.
bool vae_config_ok(const h3dit_vae_config *v) {
  if (!v) return false;
  if (v->width <= 0 || v->width % 64 || v->width > 8192) return false;
  if (v->heads <= 0 || (v->head_dim != 96 && v->head_dim != 128)) return false;
  if (v->mlp <= 0 || v->mlp % 64 || v->layers <= 0) return false;
  if (v->tile <= 0 || v->channels < 1 || v->channels > 32 || v->max_tokens <= 0) return false;
  return v->eps >= 0.f;
}

h3dit_config vae_internal(const h3dit_vae_config *v) {
  h3dit_config c{};
  c.hidden = v->width;
  c.heads = v->heads;
  c.head_dim = v->head_dim;
  c.ffn = v->mlp < 768 ? 768 : v->mlp;  // the FFN buffer also holds the [n, 768] pixel rows
  c.n_blocks = v->layers;
  c.max_tokens = v->max_tokens;
  c.rope_sections[0] = 16;
  c.rope_sections[1] = c.rope_sections[2] = v->head_dim == 96 ? 16 : 24;
  c.rope_theta = 10000.f;
  c.norm_eps = v->eps;
  c.t_scale = 1000.f;
  c.precision = H3DIT_PRECISION_BF16;
  return c;
}

// Workspace beyond the block plan: the position table [tile^2, W] and a
// vector of W ones (the unit gate of the residual updates).
size_t vae_extra_bytes(const h3dit_vae_config *v) {
  const size_t W = v->width, T = v->tile;
  return round_up(T * T * W * 4, kAlign) + round_up(W * 4, kAlign);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

struct ProfRecord {
  int kind;
  cudaEvent_t begin, end;
};

struct h3dit_ctx {
  h3dit_config cfg;
  bool profiling = false;
  std::vector<ProfRecord> records;
  std::vector<cudaEvent_t> event_pool;
  long long launches = 0;
  h3dit_time_weights tw;
  std::vector<h3dit_block_weights> blocks;
  uint8_t *ws = nullptr;
  size_t ws_bytes = 0;
  Layout L{};
  int num_sms = 148;
  std::string err;
  // layerwise weight streaming: blocks whose weights are pinned host memory
  std::vector<uint8_t> streamed;  // per block: 1 = weights in host memory
  int n_streamed = 0;
  uint8_t *staging = nullptr;     // two slots + pointer table (h3dit_attach_staging)
  Staging SP{};
  cudaStream_t copy = nullptr;
  bool own_copy = false;
  cudaEvent_t fork = nullptr, join = nullptr, ready[2] = {nullptr, nullptr},
              slot_free[2] = {nullptr, nullptr};
  // a VAE decoder context (h3dit_vae_create): its layers and extra workspace
  bool vae = false;
  h3dit_vae_config vcfg{};
  h3dit_vae_weights vw{};
  std::vector<h3dit_vae_layer_weights> vlayers;
  size_t vpos = 0, vones = 0;  // workspace offsets: position table, a vector of ones

  int *status() { return reinterpret_cast<int *>(ws + L.status); }
  float *resid() { return reinterpret_cast<float *>(ws + L.resid); }
  void *xm() { return ws + L.xm; }
  void *qkv() { return ws + L.qkv; }
  void *attn() { return ws + L.attn; }
  void *u() { return ws + L.u; }
  float *mod(int l) { return reinterpret_cast<float *>(ws + L.mod) + static_cast<size_t>(l) * 6 * cfg.hidden; }
  float *cvec() { return reinterpret_cast<float *>(ws + L.cvec); }
  float *hidden() { return reinterpret_cast<float *>(ws + L.hidden); }
  float *omod() { return reinterpret_cast<float *>(ws + L.omod); }
  float *rope() { return reinterpret_cast<float *>(ws + L.rope); }
  const void *const *wptr() { return reinterpret_cast<const void *const *>(ws + L.wptr); }
  const float *const *bptr() { return reinterpret_cast<const float *const *>(ws + L.bptr); }
  int inner() const { return cfg.heads * cfg.head_dim; }
  bool mx() const { return cfg.precision == H3DIT_PRECISION_MXFP8; }
  uint8_t *wq(int l, size_t part) { return ws + L.wq + static_cast<size_t>(l) * L.wq_block + part; }

  h3dit_status fail(h3dit_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    err = buf;
    return s;
  }
  h3dit_status cuda(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return H3DIT_OK;
    return fail(H3DIT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  cudaEvent_t take_event() {
    if (!event_pool.empty()) {
      cudaEvent_t e = event_pool.back();
      event_pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void recycle_records() {
    for (auto &r : records) {
      event_pool.push_back(r.begin);
      event_pool.push_back(r.end);
    }
    records.clear();
  }
  h3dit_block_weights slot_weights(int s) const {
    uint8_t *b = staging + static_cast<size_t>(s) * SP.slot;
    return {b + SP.part[0], b + SP.part[1], b + SP.part[2], b + SP.part[3], b + SP.part[4],
            reinterpret_cast<const float *>(b + SP.part[5])};
  }
  void release_streaming() {
    for (cudaEvent_t *e : {&fork, &join, &ready[0], &ready[1], &slot_free[0], &slot_free[1]})
      if (*e) {
        cudaEventDestroy(*e);
        *e = nullptr;
      }
    if (own_copy && copy) cudaStreamDestroy(copy);
    copy = nullptr;
    own_copy = false;
    staging = nullptr;
  }
  ~h3dit_ctx() {
    recycle_records();
    for (cudaEvent_t e : event_pool) cudaEventDestroy(e);
    release_streaming();
  }
};

namespace {
// Counts the kernels of one library step and, while profiling, brackets them
// with a CUDA event pair on the launch stream.
struct Launch {
  h3dit_ctx *ctx;
  cudaStream_t s;
  ProfRecord rec{};
  bool on = false;
  Launch(h3dit_ctx *c, int kind, cudaStream_t st, int kernels = 1) : ctx(c), s(st) {
    ctx->launches += kernels;
    if (ctx->profiling) {
      rec.kind = kind;
      rec.begin = ctx->take_event();
      rec.end = ctx->take_event();
      on = rec.begin && rec.end && cudaEventRecord(rec.begin, s) == cudaSuccess;
    }
  }
  ~Launch() {
    if (on && cudaEventRecord(rec.end, s) == cudaSuccess) {
      ctx->records.push_back(rec);
      return;
    }
    // not recorded: the events go back to the pool
    if (rec.begin) ctx->event_pool.push_back(rec.begin);
    if (rec.end) ctx->event_pool.push_back(rec.end);
  }
};
}  // namespace

namespace {

h3dit_status encode_2d(h3dit_ctx *ctx, CUtensorMap *m, const void *base, uint64_t inner,
                       uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return ctx->fail(H3DIT_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return ctx->fail(H3DIT_ERR_CUDA, "tensor map encode failed (%d)", (int)r);
  return H3DIT_OK;
}

// [tokens, heads, head_dim] view with a token stride of `ld` elements, read
// in boxes of 64 columns x `box_rows` tokens.
h3dit_status encode_heads(h3dit_ctx *ctx, CUtensorMap *m, const void *base, int n, int heads,
                          int head_dim, int ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return ctx->fail(H3DIT_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                 static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return ctx->fail(H3DIT_ERR_CUDA, "tensor map encode failed (%d)", (int)r);
  return H3DIT_OK;
}

// Destination buffers of a fused Ulysses exchange, one per rank (and, for
// an MXFP8 attention output, each rank's scale array).
struct ScatterTargets {
  void *const *ptr;
  int ranks, rank;
  void *const *sf = nullptr;
};

h3dit_status run_linear(h3dit_ctx *ctx, int epi, const void *a, const void *w, int m, int n,
                        int k, void *out, long long ldo, const float *gate, const float *rope,
                        cudaStream_t s, const float *bias = nullptr, int kind_override = -1,
                        const ScatterTargets *scatter = nullptr) {
  if (epi < H3DIT_EPI_STORE || epi > H3DIT_EPI_GATED_RESIDUAL)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "unknown epilogue %d", epi);
  if (m < 0 || n <= 0 || k <= 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "bad shape %d x %d x %d", m, n, k);
  if (k % kGemmBK || n % 32)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "linear needs k %% 64 == 0 and n %% 32 == 0 (k=%d n=%d)", k, n);
  if (m == 0) return H3DIT_OK;  // no rows: no work, and the data pointers are not examined
  if (!a || !w || (!scatter && (!out || !aligned16(out))) || !aligned16(a) || !aligned16(w))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "linear: NULL or misaligned pointer");
  if (epi == H3DIT_EPI_GATED_RESIDUAL && (!gate || !aligned16(gate)))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "gated residual needs a 16-byte aligned gate");
  if (bias && (!aligned16(bias) || epi == H3DIT_EPI_QKV_ROPE))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "bias must be 16-byte aligned, and not with QKV + RoPE");
  GemmParams p{};
  p.bias = bias;
  if (epi == H3DIT_EPI_QKV_ROPE) {
    const int I = ctx->inner(), dh = ctx->cfg.head_dim;
    const int *sec = ctx->cfg.rope_sections;
    if (n != 3 * I) return ctx->fail(H3DIT_ERR_INVALID_ARG, "QKV epilogue needs n == 3*heads*head_dim");
    if (!rope || !aligned16(rope)) return ctx->fail(H3DIT_ERR_INVALID_ARG, "QKV epilogue needs a RoPE table");
    // each output tile must start on a rotary-section boundary of a head
    for (int c = 0; c < 2 * I; c += kGemmBN) {
      const int h = c % dh;
      if (h != 0 && h != 2 * sec[0] && h != 2 * (sec[0] + sec[1]))
        return ctx->fail(H3DIT_ERR_UNSUPPORTED, "rope sections do not align with 256-column tiles");
    }
    p.head_dim = dh;
    p.rope_cols = 2 * I;
    p.sec[0] = sec[0];
    p.sec[1] = sec[1];
    p.sec[2] = sec[2];
    if (scatter) {
      // each rank's receive buffer is [ranks * m, 3 * I / ranks]; every
      // 32- or 48-column store unit sits in one head and starts on a
      // multiple of 8 columns, so the 16-byte stores stay aligned
      p.scatter_ranks = scatter->ranks;
      p.scatter_rank = scatter->rank;
      p.scatter_inner = I;
      p.scatter_cols = I / scatter->ranks;
      for (int g = 0; g < scatter->ranks; ++g) p.scatter[g] = scatter->ptr[g];
    }
  }
  // More than one 128-row block: 256 x 256 tiles on CTA pairs, which halves
  // the W traffic per SM; a single row block stays on the one-CTA kernel.
  const int max_pairs = H3_GEMM_PAIR && m > kGemmBM ? gemm_pair_max_clusters(epi) : 0;
  const bool paired = max_pairs > 0;
  CUtensorMap ta, tb;
  h3dit_status st = encode_2d(ctx, &ta, a, k, m, static_cast<uint64_t>(k) * 2, kGemmBK, kGemmBM);
  if (st) return st;
  st = encode_2d(ctx, &tb, w, k, n, static_cast<uint64_t>(k) * 2, kGemmBK,
                 paired ? kGemmBN / 2 : kGemmBN);
  if (st) return st;
  p.m = m;
  p.n = n;
  p.k = k;
  p.tiles_m = (m + (paired ? 2 * kGemmBM : kGemmBM) - 1) / (paired ? 2 * kGemmBM : kGemmBM);
  p.tiles_n = (n + kGemmBN - 1) / kGemmBN;
  p.out = out;
  p.ldo = ldo;
  p.gate = gate;
  p.rope = rope;
  p.gelu_tanh = ctx->cfg.gelu_tanh;
  p.status = ctx->status();
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < ctx->num_sms ? tiles : ctx->num_sms;
  const int kind = kind_override >= 0         ? kind_override
                   : epi == H3DIT_EPI_QKV_ROPE ? H3DIT_KERNEL_QKV
                   : epi == H3DIT_EPI_GELU     ? H3DIT_KERNEL_FFN1
                   : k == ctx->inner()         ? H3DIT_KERNEL_OUT_PROJ
                   : epi == H3DIT_EPI_STORE    ? H3DIT_KERNEL_FFN1
                                               : H3DIT_KERNEL_FFN2;
  Launch L(ctx, kind, s);
  if (paired) {
    int pairs = tiles < max_pairs ? tiles : max_pairs;
    if (pairs > ctx->num_sms / 2) pairs = ctx->num_sms / 2;
    return ctx->cuda(launch_gemm_pair(ta, tb, p, epi, 2 * pairs, s), "paired gemm launch");
  }
  return ctx->cuda(launch_gemm(ta, tb, p, epi, grid, s), "gemm launch");
}

h3dit_status encode_fp8(h3dit_ctx *ctx, CUtensorMap *m, const void *base, uint64_t k, uint64_t rows,
                        uint32_t box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return ctx->fail(H3DIT_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {k, rows};
  const cuuint64_t strides[1] = {k};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kGemmMxBK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return ctx->fail(H3DIT_ERR_CUDA, "tensor map encode failed (%d)", (int)r);
  return H3DIT_OK;
}

// MXFP8 linear: a, w E4M3 with scales in the mx layout; epilogues as
// run_linear, except that GELU writes MXFP8 (out E4M3 [m, n] + out_sf).
h3dit_status run_linear_mx(h3dit_ctx *ctx, int epi, const void *a, const void *a_sf, const void *w,
                           const void *w_sf, int m, int n, int k, void *out, long long ldo,
                           void *out_sf, const float *gate, const float *rope, cudaStream_t s,
                           const void *w_sf_tiled = nullptr,
                           const ScatterTargets *scatter = nullptr) {
  if (epi < H3DIT_EPI_STORE || epi > H3DIT_EPI_GATED_RESIDUAL)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "unknown epilogue %d", epi);
  if (m < 0 || n <= 0 || k <= 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "bad shape %d x %d x %d", m, n, k);
  if (k % kGemmMxBK || n % kGemmMxBN)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "MXFP8 linear needs k and n multiples of 128 (k=%d n=%d)", k, n);
  if (m == 0) return H3DIT_OK;  // no rows: no work, and the data pointers are not examined
  if (!a || !a_sf || !w || !w_sf || (!scatter && (!out || !aligned16(out))) || !aligned16(a) ||
      !aligned16(a_sf) || !aligned16(w) || !aligned16(w_sf))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "MXFP8 linear: NULL or misaligned pointer");
  if (epi == H3DIT_EPI_GATED_RESIDUAL && (!gate || !aligned16(gate)))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "gated residual needs a 16-byte aligned gate");
  if (epi == H3DIT_EPI_GELU && (!out_sf || ldo != n))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "MXFP8 GELU output needs out_sf and a dense [m, n] out");
  GemmParams p{};
  if (epi == H3DIT_EPI_QKV_ROPE) {
    const int I = ctx->inner(), dh = ctx->cfg.head_dim;
    const int *sec = ctx->cfg.rope_sections;
    if (n != 3 * I) return ctx->fail(H3DIT_ERR_INVALID_ARG, "QKV epilogue needs n == 3*heads*head_dim");
    if (!rope || !aligned16(rope)) return ctx->fail(H3DIT_ERR_INVALID_ARG, "QKV epilogue needs a RoPE table");
    for (int c = 0; c < 2 * I; c += kGemmMxBN) {
      const int h = c % dh;
      if (h != 0 && h != 2 * sec[0] && h != 2 * (sec[0] + sec[1]))
        return ctx->fail(H3DIT_ERR_UNSUPPORTED, "rope sections do not align with 128-column tiles");
    }
    // wide tiles only where each 224-column tile starts on a section boundary
    for (int c = 0; c < 2 * I && w_sf_tiled; c += kGemmMxWideBN) {
      const int h = c % dh;
      if (h != 0 && h != 2 * sec[0] && h != 2 * (sec[0] + sec[1])) w_sf_tiled = nullptr;
    }
    p.head_dim = dh;
    p.rope_cols = 2 * I;
    p.sec[0] = sec[0];
    p.sec[1] = sec[1];
    p.sec[2] = sec[2];
    if (scatter) {  // as in run_linear: the first Ulysses all-to-all in the epilogue
      p.scatter_ranks = scatter->ranks;
      p.scatter_rank = scatter->rank;
      p.scatter_inner = I;
      p.scatter_cols = I / scatter->ranks;
      for (int g = 0; g < scatter->ranks; ++g) p.scatter[g] = scatter->ptr[g];
    }
  }
  const bool wide = w_sf_tiled && n % kGemmMxWideBN == 0;
  const int bn = wide ? kGemmMxWideBN : kGemmMxBN;
  CUtensorMap ta, tb;
  h3dit_status st = encode_fp8(ctx, &ta, a, k, m);
  if (st) return st;
  if ((st = encode_fp8(ctx, &tb, w, k, n, bn))) return st;
  p.m = m;
  p.n = n;
  p.k = k;
  p.tiles_m = (m + kGemmBM - 1) / kGemmBM;
  p.tiles_n = n / bn;
  p.out = out;
  p.ldo = ldo;
  p.gate = gate;
  p.rope = rope;
  p.gelu_tanh = ctx->cfg.gelu_tanh;
  p.status = ctx->status();
  p.a_sf = static_cast<const uint8_t *>(a_sf);
  p.b_sf = static_cast<const uint8_t *>(wide ? w_sf_tiled : w_sf);
  p.out_sf = static_cast<uint8_t *>(out_sf);
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < ctx->num_sms ? tiles : ctx->num_sms;
  const int kernel_epi = epi == H3DIT_EPI_GELU ? kEpiGeluMx : epi;
  const int kind = epi == H3DIT_EPI_QKV_ROPE   ? H3DIT_KERNEL_QKV
                   : epi == H3DIT_EPI_GELU     ? H3DIT_KERNEL_FFN1
                   : k == ctx->inner()         ? H3DIT_KERNEL_OUT_PROJ
                   : epi == H3DIT_EPI_STORE    ? H3DIT_KERNEL_FFN1
                                               : H3DIT_KERNEL_FFN2;
  Launch L(ctx, kind, s);
  return ctx->cuda(launch_gemm_mx(ta, tb, p, kernel_epi, grid, wide, s), "MXFP8 gemm launch");
}

h3dit_status run_attention(h3dit_ctx *ctx, const void *q, const void *k, const void *v, int ld,
                           void *o, int ldo, int n, cudaStream_t s, void *o_sf = nullptr,
                           int heads = 0, int batch = 1,
                           const ScatterTargets *scatter = nullptr) {
  if (heads == 0) heads = ctx->cfg.heads;
  if (n < 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "n < 0");
  if (batch < 1 || static_cast<long long>(n) * batch > (1LL << 30))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "bad sequence batch");
  if (heads < 1 || heads > ctx->cfg.heads)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "heads %d outside [1, %d]", heads, ctx->cfg.heads);
  if (n == 0) return H3DIT_OK;  // no tokens: no work, and the data pointers are not examined
  if (!q || !k || !v || (!scatter && (!o || !aligned16(o))) || !aligned16(q) || !aligned16(k) ||
      !aligned16(v))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "attention: NULL or misaligned pointer");
  const int I = heads * ctx->cfg.head_dim;
  if (ld < I || ld % 8 || ldo < I || ldo % 8)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "attention: row strides must be >= heads*head_dim and multiples of 8");
  CUtensorMap tq, tk, tv;
  h3dit_status st;
  const int rows = n * batch;
  if ((st = encode_heads(ctx, &tq, q, rows, heads, ctx->cfg.head_dim, ld, kAttnBQ))) return st;
  if ((st = encode_heads(ctx, &tk, k, rows, heads, ctx->cfg.head_dim, ld, kAttnBKV))) return st;
  if ((st = encode_heads(ctx, &tv, v, rows, heads, ctx->cfg.head_dim, ld, kAttnBKV))) return st;
  AttnParams p{};
  p.n = n;
  p.batch = batch;
  p.tiles_kv = (n + kAttnBKV - 1) / kAttnBKV;
  p.o = o;
  p.ldo = ldo;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(ctx->cfg.head_dim));
  p.status = ctx->status();
  p.o_sf = static_cast<uint8_t *>(o_sf);
  if (o_sf && (ldo != I || I % 128 || !aligned16(o_sf)))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "MXFP8 attention output needs ld_o == heads*head_dim, a multiple of 128");
  const bool out_mx = o_sf != nullptr || (scatter && scatter->sf);
  if (scatter && scatter->sf) {
    // an MXFP8 output scattered to [n / ranks, ld_o] E4M3 rows of every head
    if (ldo != ctx->inner() || ldo % 128)
      return ctx->fail(H3DIT_ERR_INVALID_ARG,
                       "MXFP8 scattered output needs ld_o == heads*head_dim, a multiple of 128");
    for (int g = 0; g < scatter->ranks; ++g) {
      if (!scatter->sf[g] || !aligned16(scatter->sf[g]))
        return ctx->fail(H3DIT_ERR_INVALID_ARG, "scale array of rank %d is NULL or misaligned", g);
      p.o_sf_scatter[g] = static_cast<uint8_t *>(scatter->sf[g]);
    }
  }
  if (scatter) {
    // rank r's rows of the sequence go to its [n / ranks, ld_o] output, at
    // this rank's head group's columns
    p.o_scatter_ranks = scatter->ranks;
    p.o_rows_per_rank = n / scatter->ranks;
    p.o_col0 = scatter->rank * I;
    for (int g = 0; g < scatter->ranks; ++g) p.o_scatter[g] = scatter->ptr[g];
  }
  Launch L(ctx, H3DIT_KERNEL_ATTENTION, s);
  return ctx->cuda(launch_attention(tq, tk, tv, p, ctx->cfg.head_dim, heads, out_mx, s),
                   "attention launch");
}

h3dit_status check_tokens(h3dit_ctx *ctx, void *x_img, const h3dit_grid *grids, int n_grids,
                          void *x_txt, int n_txt, int *n_img_out) {
  if (n_txt < 0 || n_grids < 0 || n_grids > kMaxGrids)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "bad n_txt or n_grids (max %d grids)", kMaxGrids);
  if (n_grids > 0 && !grids) return ctx->fail(H3DIT_ERR_INVALID_ARG, "grids is NULL");
  long long n_img = 0;
  for (int g = 0; g < n_grids; ++g) {
    if (grids[g].height <= 0 || grids[g].width <= 0 || grids[g].frame < 0)
      return ctx->fail(H3DIT_ERR_INVALID_ARG, "grid %d has a bad shape", g);
    n_img += static_cast<long long>(grids[g].height) * grids[g].width;
  }
  const long long n = n_img + n_txt;
  if (n < 1 || n > ctx->cfg.max_tokens)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "token count %lld outside [1, max_tokens=%d]", n, ctx->cfg.max_tokens);
  if (n_img > 0 && (!x_img || !aligned16(x_img)))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "x_img is NULL or misaligned");
  if (n_txt > 0 && (!x_txt || !aligned16(x_txt)))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "x_txt is NULL or misaligned");
  *n_img_out = static_cast<int>(n_img);
  return H3DIT_OK;
}

h3dit_status rope_table_into(h3dit_ctx *ctx, const h3dit_grid *grids, int n_grids, int n_txt,
                             int n, float *table, cudaStream_t s) {
  GridDesc g[kMaxGrids];
  for (int i = 0; i < n_grids; ++i) g[i] = GridDesc{grids[i].frame, grids[i].height, grids[i].width};
  Launch L(ctx, H3DIT_KERNEL_ROPE_TABLE, s);
  return ctx->cuda(launch_rope_table(g, n_grids, n_txt, n, ctx->cfg.rope_sections,
                                     ctx->cfg.rope_theta, table, s),
                   "rope table launch");
}

h3dit_status run_rmsnorm(h3dit_ctx *ctx, const float *x, const float *shift, const float *scale,
                         void *out, int n, cudaStream_t s, uint8_t *out_sf = nullptr) {
  Launch L(ctx, H3DIT_KERNEL_RMSNORM, s);
  return ctx->cuda(launch_rmsnorm_modulate(x, shift, scale, out, n, ctx->cfg.hidden,
                                           ctx->cfg.norm_eps, ctx->num_sms, s, out_sf),
                   "rmsnorm launch");
}

h3dit_status run_pack(h3dit_ctx *ctx, const void *x_txt, int n_txt, const void *x_img, int n_img,
                      cudaStream_t s) {
  Launch L(ctx, H3DIT_KERNEL_PACK, s);
  return ctx->cuda(launch_pack(x_txt, n_txt, x_img, n_img, ctx->cfg.hidden, ctx->cfg.io_fp32 != 0,
                               ctx->resid(), s),
                   "pack launch");
}

h3dit_status run_unpack(h3dit_ctx *ctx, int n_txt, int n_img, void *x_txt, void *x_img,
                        cudaStream_t s) {
  Launch L(ctx, H3DIT_KERNEL_PACK, s);
  return ctx->cuda(launch_unpack(ctx->resid(), n_txt, n_img, ctx->cfg.hidden,
                                 ctx->cfg.io_fp32 != 0, x_txt, x_img, s),
                   "unpack launch");
}

// Steps a3..a9 with the four linears on MXFP8 operands (a11).
h3dit_status block_body_mx(h3dit_ctx *ctx, int l, const float *mod, int n, cudaStream_t s) {
  const int D = ctx->cfg.hidden, I = ctx->inner(), F = ctx->cfg.ffn;
  const MxWeights &o = ctx->L.wq_off;
  auto tiled = [&](size_t off) -> const void * { return off == kNoTiled ? nullptr : ctx->wq(l, off); };
  uint8_t *xq = ctx->ws + ctx->L.xq, *xq_sf = ctx->ws + ctx->L.xq_sf;
  uint8_t *oq = ctx->ws + ctx->L.oq, *oq_sf = ctx->ws + ctx->L.oq_sf;
  uint8_t *uq = ctx->ws + ctx->L.uq, *uq_sf = ctx->ws + ctx->L.uq_sf;
  h3dit_status st = run_rmsnorm(ctx, ctx->resid(), mod, mod + D, xq, n, s, xq_sf);
  if (st) return st;
  if ((st = run_linear_mx(ctx, H3DIT_EPI_QKV_ROPE, xq, xq_sf, ctx->wq(l, o.qkv), ctx->wq(l, o.qkv_sf),
                          n, 3 * I, D, ctx->qkv(), 3 * I, nullptr, nullptr, ctx->rope(), s,
                          tiled(o.qkv_sft))))
    return st;
  const uint16_t *qkv = static_cast<const uint16_t *>(ctx->qkv());
  if ((st = run_attention(ctx, qkv, qkv + I, qkv + 2 * I, 3 * I, oq, I, n, s, oq_sf))) return st;
  if ((st = run_linear_mx(ctx, H3DIT_EPI_GATED_RESIDUAL, oq, oq_sf, ctx->wq(l, o.o), ctx->wq(l, o.o_sf),
                          n, D, I, ctx->resid(), D, nullptr, mod + 2 * D, nullptr, s,
                          tiled(o.o_sft))))
    return st;
  if ((st = run_rmsnorm(ctx, ctx->resid(), mod + 3 * D, mod + 4 * D, xq, n, s, xq_sf))) return st;
  if ((st = run_linear_mx(ctx, H3DIT_EPI_GELU, xq, xq_sf, ctx->wq(l, o.ff1), ctx->wq(l, o.ff1_sf), n,
                          F, D, uq, F, uq_sf, nullptr, nullptr, s, tiled(o.ff1_sft))))
    return st;
  return run_linear_mx(ctx, H3DIT_EPI_GATED_RESIDUAL, uq, uq_sf, ctx->wq(l, o.ff2),
                       ctx->wq(l, o.ff2_sf), n, D, F, ctx->resid(), D, nullptr, mod + 5 * D,
                       nullptr, s, tiled(o.ff2_sft));
}

// Steps a3..a9 on the packed fp32 residual of n tokens (workspace).
h3dit_status block_body(h3dit_ctx *ctx, int l, const h3dit_block_weights &w, const float *mod,
                        int n, cudaStream_t s) {
  if (ctx->mx()) return block_body_mx(ctx, l, mod, n, s);
  const int D = ctx->cfg.hidden, I = ctx->inner(), F = ctx->cfg.ffn;
  const float *sh1 = mod, *sc1 = mod + D, *g1 = mod + 2 * D;
  const float *sh2 = mod + 3 * D, *sc2 = mod + 4 * D, *g2 = mod + 5 * D;
  h3dit_status st = run_rmsnorm(ctx, ctx->resid(), sh1, sc1, ctx->xm(), n, s);
  if (st) return st;
  if ((st = run_linear(ctx, H3DIT_EPI_QKV_ROPE, ctx->xm(), w.w_qkv, n, 3 * I, D, ctx->qkv(), 3 * I,
                       nullptr, ctx->rope(), s)))
    return st;
  const uint16_t *qkv = static_cast<const uint16_t *>(ctx->qkv());
  if ((st = run_attention(ctx, qkv, qkv + I, qkv + 2 * I, 3 * I, ctx->attn(), I, n, s))) return st;
  if ((st = run_linear(ctx, H3DIT_EPI_GATED_RESIDUAL, ctx->attn(), w.w_o, n, D, I, ctx->resid(), D,
                       g1, nullptr, s)))
    return st;
  if ((st = run_rmsnorm(ctx, ctx->resid(), sh2, sc2, ctx->xm(), n, s))) return st;
  if ((st = run_linear(ctx, H3DIT_EPI_GELU, ctx->xm(), w.w_ff1, n, F, D, ctx->u(), F, nullptr,
                       nullptr, s)))
    return st;
  return run_linear(ctx, H3DIT_EPI_GATED_RESIDUAL, ctx->u(), w.w_ff2, n, D, F, ctx->resid(), D, g2,
                    nullptr, s);
}

// AdaLN projections of the blocks in [l0, l1) whose weights are on the
// device, one launch per run of consecutive such blocks (one launch per step
// when every block is resident); streamed blocks get theirs from their slot.
h3dit_status adaln_resident(h3dit_ctx *ctx, int l0, int l1, cudaStream_t s) {
  int l = l0;
  while (l < l1) {
    if (ctx->streamed[l]) {
      ++l;
      continue;
    }
    int e = l;
    while (e < l1 && !ctx->streamed[e]) ++e;
    Launch L(ctx, H3DIT_KERNEL_ADALN, s);
    h3dit_status st = ctx->cuda(launch_adaln(ctx->cvec(), ctx->wptr(), ctx->bptr(), l, e - l,
                                             ctx->mod(l), ctx->cfg.hidden, ctx->num_sms, s),
                                "adaln launch");
    if (st) return st;
    l = e;
  }
  return H3DIT_OK;
}

// Host weights of block l into staging slot `slot` on the copy stream, then
// mark the slot ready (one cudaMemcpyAsync per weight tensor).
h3dit_status copy_block(h3dit_ctx *ctx, int l, int slot) {
  const h3dit_block_weights &w = ctx->blocks[l];
  const void *src[6] = {w.w_qkv, w.w_o, w.w_ff1, w.w_ff2, w.w_ada, w.b_ada};
  uint8_t *dst = ctx->staging + static_cast<size_t>(slot) * ctx->SP.slot;
  for (int i = 0; i < 6; ++i) {
    cudaError_t e = cudaMemcpyAsync(dst + ctx->SP.part[i], src[i], ctx->SP.bytes[i],
                                    cudaMemcpyHostToDevice, ctx->copy);
    if (e != cudaSuccess) return ctx->cuda(e, "weight streaming copy");
  }
  return ctx->cuda(cudaEventRecord(ctx->ready[slot], ctx->copy), "weight streaming event");
}

// Blocks [l0, l1) on the packed residual of n tokens. Resident blocks run on
// their own weights with the modulation already in mod(l) (or `mod_one` for
// a single block); a streamed block waits for its slot, gets its AdaLN
// projection from the slot (unless `mod_one` is given) and runs on the slot.
// Two slots alternate: the copy of streamed block i+2 starts on the copy
// stream as soon as block i has finished with the slot, so it overlaps the
// compute of block i+1. The copy stream forks from `s` at entry and joins it
// at exit, so the whole call is ordered on `s` (and can be graph-captured).
h3dit_status run_blocks(h3dit_ctx *ctx, int l0, int l1, int n, cudaStream_t s,
                        const float *mod_one = nullptr) {
  auto mod_of = [&](int l) { return mod_one ? mod_one : ctx->mod(l); };
  std::vector<int> order;
  for (int l = l0; l < l1; ++l)
    if (ctx->streamed[l]) order.push_back(l);
  h3dit_status st;
  if (order.empty()) {
    for (int l = l0; l < l1; ++l)
      if ((st = block_body(ctx, l, ctx->blocks[l], mod_of(l), n, s))) return st;
    return H3DIT_OK;
  }
  if (!ctx->staging)
    return ctx->fail(H3DIT_ERR_WORKSPACE,
                     "blocks with host weights need staging memory (h3dit_attach_staging)");
  if ((st = ctx->cuda(cudaEventRecord(ctx->fork, s), "fork event"))) return st;
  if ((st = ctx->cuda(cudaStreamWaitEvent(ctx->copy, ctx->fork, 0), "fork wait"))) return st;
  const int first = static_cast<int>(order.size()) < 2 ? static_cast<int>(order.size()) : 2;
  for (int i = 0; i < first; ++i)
    if ((st = copy_block(ctx, order[i], i))) return st;
  size_t i = 0;
  for (int l = l0; l < l1; ++l) {
    if (!ctx->streamed[l]) {
      if ((st = block_body(ctx, l, ctx->blocks[l], mod_of(l), n, s))) return st;
      continue;
    }
    const int slot = static_cast<int>(i % 2);
    if ((st = ctx->cuda(cudaStreamWaitEvent(s, ctx->ready[slot], 0), "slot wait"))) return st;
    if (!mod_one) {
      const void *const *wt = reinterpret_cast<const void *const *>(ctx->staging + ctx->SP.table);
      const float *const *bt =
          reinterpret_cast<const float *const *>(ctx->staging + ctx->SP.table + 2 * sizeof(void *));
      Launch L(ctx, H3DIT_KERNEL_ADALN, s);
      if ((st = ctx->cuda(launch_adaln(ctx->cvec(), wt, bt, slot, 1, ctx->mod(l), ctx->cfg.hidden,
                                       ctx->num_sms, s),
                          "adaln launch")))
        return st;
    }
    if ((st = block_body(ctx, l, ctx->slot_weights(slot), mod_of(l), n, s))) return st;
    if (i + 2 < order.size()) {
      if ((st = ctx->cuda(cudaEventRecord(ctx->slot_free[slot], s), "slot event"))) return st;
      if ((st = ctx->cuda(cudaStreamWaitEvent(ctx->copy, ctx->slot_free[slot], 0), "slot wait")))
        return st;
      if ((st = copy_block(ctx, order[i + 2], slot))) return st;
    }
    ++i;
  }
  if ((st = ctx->cuda(cudaEventRecord(ctx->join, ctx->copy), "join event"))) return st;
  return ctx->cuda(cudaStreamWaitEvent(s, ctx->join, 0), "join wait");
}

h3dit_status run_layernorm(h3dit_ctx *ctx, const float *x, const float *g, const float *b,
                           void *out, int n, cudaStream_t s) {
  Launch L(ctx, H3DIT_KERNEL_RMSNORM, s);
  return ctx->cuda(launch_layernorm(x, g, b, out, n, ctx->cfg.hidden, ctx->cfg.norm_eps,
                                    ctx->num_sms, s),
                   "layernorm launch");
}

// One decoder layer on the n tokens of `tiles` tiles in the fp32 residual.
h3dit_status vae_layer(h3dit_ctx *ctx, const h3dit_vae_layer_weights &w, int n, int tiles,
                       cudaStream_t s) {
  const int W = ctx->cfg.hidden, I = ctx->inner(), M = ctx->vcfg.mlp;
  const int per_tile = ctx->vcfg.tile * ctx->vcfg.tile;
  const float *ones = reinterpret_cast<const float *>(ctx->ws + ctx->vones);
  uint16_t *qkv = static_cast<uint16_t *>(ctx->qkv());
  h3dit_status st = run_layernorm(ctx, ctx->resid(), w.ln1_g, w.ln1_b, ctx->xm(), n, s);
  if (st) return st;
  if ((st = run_linear(ctx, H3DIT_EPI_STORE, ctx->xm(), w.w_qkv, n, 3 * I, W, qkv, 3 * I, nullptr,
                       nullptr, s, w.b_qkv, H3DIT_KERNEL_QKV)))
    return st;
  if ((st = run_attention(ctx, qkv, qkv + I, qkv + 2 * I, 3 * I, ctx->attn(), I, per_tile, s,
                          nullptr, 0, tiles)))
    return st;
  if ((st = run_linear(ctx, H3DIT_EPI_GATED_RESIDUAL, ctx->attn(), w.w_o, n, W, I, ctx->resid(), W,
                       ones, nullptr, s, w.b_o, H3DIT_KERNEL_OUT_PROJ)))
    return st;
  if ((st = run_layernorm(ctx, ctx->resid(), w.ln2_g, w.ln2_b, ctx->xm(), n, s))) return st;
  if ((st = run_linear(ctx, H3DIT_EPI_GELU, ctx->xm(), w.w_1, n, M, W, ctx->u(), M, nullptr,
                       nullptr, s, w.b_1, H3DIT_KERNEL_FFN1)))
    return st;
  return run_linear(ctx, H3DIT_EPI_GATED_RESIDUAL, ctx->u(), w.w_2, n, W, M, ctx->resid(), W, ones,
                    nullptr, s, w.b_2, H3DIT_KERNEL_FFN2);
}

}  // namespace

extern "C" {

const char *h3dit_status_string(h3dit_status s) {
  switch (s) {
    case H3DIT_OK: return "ok";
    case H3DIT_ERR_INVALID_ARG: return "invalid argument";
    case H3DIT_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case H3DIT_ERR_WORKSPACE: return "workspace too small or misaligned";
    case H3DIT_ERR_CUDA: return "CUDA error";
    case H3DIT_ERR_TIMEOUT: return "a kernel's bounded wait timed out";
    default: return "unknown status";
  }
}

const char *h3dit_last_error(const h3dit_ctx *ctx) {
  if (!ctx) return "no context";
  return ctx->err.c_str();
}

size_t h3dit_workspace_bytes(const h3dit_config *cfg) {
  if (!config_ok(cfg)) return 0;
  return plan(cfg).total;
}

h3dit_status h3dit_create(const h3dit_config *cfg, const h3dit_time_weights *time_w,
                          const h3dit_block_weights *blocks, void *workspace, size_t ws_bytes,
                          void *cuda_stream, h3dit_ctx **out) {
  if (!out) return H3DIT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!time_w || !blocks) return H3DIT_ERR_INVALID_ARG;
  if (!config_ok(cfg)) {
    // a config that is valid but for the MXFP8 shape rules is unsupported, not invalid
    if (cfg && cfg->precision == H3DIT_PRECISION_MXFP8) {
      h3dit_config c2 = *cfg;
      c2.precision = H3DIT_PRECISION_BF16;
      if (config_ok(&c2)) return H3DIT_ERR_UNSUPPORTED;
    }
    return H3DIT_ERR_INVALID_ARG;
  }
  if (!time_w->w_t1 || !time_w->b_t1 || !time_w->w_t2 || !time_w->b_t2 ||
      !aligned16(time_w->w_t2))
    return H3DIT_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_blocks; ++l) {
    const h3dit_block_weights &b = blocks[l];
    if (!b.w_qkv || !b.w_o || !b.w_ff1 || !b.w_ff2 || !b.w_ada || !b.b_ada) return H3DIT_ERR_INVALID_ARG;
    if (!aligned16(b.w_qkv) || !aligned16(b.w_o) || !aligned16(b.w_ff1) || !aligned16(b.w_ff2) ||
        !aligned16(b.w_ada))
      return H3DIT_ERR_INVALID_ARG;
  }
  const Layout L = plan(cfg);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) || ws_bytes < L.total)
    return H3DIT_ERR_WORKSPACE;

  h3dit_ctx *ctx = new (std::nothrow) h3dit_ctx();
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  ctx->cfg = *cfg;
  ctx->tw = *time_w;
  ctx->blocks.assign(blocks, blocks + cfg->n_blocks);
  ctx->ws = static_cast<uint8_t *>(workspace);
  ctx->ws_bytes = ws_bytes;
  ctx->L = L;
  int dev = 0;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    delete ctx;
    return H3DIT_ERR_CUDA;
  }
  // where each block's weights live: all on the device, or all in pinned
  // host memory (streamed layer by layer through staging slots)
  ctx->streamed.assign(cfg->n_blocks, 0);
  for (int l = 0; l < cfg->n_blocks; ++l) {
    const h3dit_block_weights &b = blocks[l];
    const void *ptrs[6] = {b.w_qkv, b.w_o, b.w_ff1, b.w_ff2, b.w_ada, b.b_ada};
    int host = 0, device = 0;
    for (const void *p : ptrs) {
      cudaPointerAttributes a{};
      if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        a.type = cudaMemoryTypeUnregistered;
      }
      if (a.type == cudaMemoryTypeHost)
        ++host;
      else if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged)
        ++device;
    }
    if (host == 6) {
      ctx->streamed[l] = 1;
      ++ctx->n_streamed;
    } else if (device != 6) {
      delete ctx;
      return H3DIT_ERR_INVALID_ARG;  // mixed, or pageable host memory
    }
  }
  if (ctx->n_streamed && ctx->mx()) {
    delete ctx;
    return H3DIT_ERR_UNSUPPORTED;  // MXFP8 quantizes every block at create
  }
  std::vector<const void *> wp(cfg->n_blocks), bp(cfg->n_blocks);
  for (int l = 0; l < cfg->n_blocks; ++l) {
    wp[l] = blocks[l].w_ada;
    bp[l] = blocks[l].b_ada;
  }
  cudaError_t e = cudaMemsetAsync(ctx->status(), 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(ctx->ws + L.wptr, wp.data(), wp.size() * sizeof(void *),
                        cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(ctx->ws + L.bptr, bp.data(), bp.size() * sizeof(void *),
                        cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && ctx->mx()) {
    // MXFP8 copies of the four block linears (a11), quantized once here
    const int D = cfg->hidden, I = ctx->inner(), F = cfg->ffn;
    const MxWeights &o = L.wq_off;
    for (int l = 0; l < cfg->n_blocks && e == cudaSuccess; ++l) {
      const h3dit_block_weights &b = blocks[l];
      e = launch_mx_quantize(b.w_qkv, D, 3 * I, D, ctx->wq(l, o.qkv), ctx->wq(l, o.qkv_sf), s);
      if (e == cudaSuccess) e = launch_mx_quantize(b.w_o, I, D, I, ctx->wq(l, o.o), ctx->wq(l, o.o_sf), s);
      if (e == cudaSuccess)
        e = launch_mx_quantize(b.w_ff1, D, F, D, ctx->wq(l, o.ff1), ctx->wq(l, o.ff1_sf), s);
      if (e == cudaSuccess)
        e = launch_mx_quantize(b.w_ff2, F, D, F, ctx->wq(l, o.ff2), ctx->wq(l, o.ff2_sf), s);
      // and their scales repacked for the 224-column tiles
      const struct {
        size_t sf, sft;
        int n, k;
      } rep[4] = {{o.qkv_sf, o.qkv_sft, 3 * I, D},
                  {o.o_sf, o.o_sft, D, I},
                  {o.ff1_sf, o.ff1_sft, F, D},
                  {o.ff2_sf, o.ff2_sft, D, F}};
      for (int r = 0; r < 4 && e == cudaSuccess; ++r)
        if (rep[r].sft != kNoTiled)
          e = launch_mx_tile_sf(ctx->wq(l, rep[r].sf), rep[r].n, rep[r].k, ctx->wq(l, rep[r].sft), s);
    }
  }
  // the host vectors die with this call: the copies must have been consumed
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    delete ctx;
    return H3DIT_ERR_CUDA;
  }
  *out = ctx;
  return H3DIT_OK;
}

void h3dit_destroy(h3dit_ctx *ctx) { delete ctx; }

size_t h3dit_staging_bytes(const h3dit_config *cfg) {
  if (!config_ok(cfg)) return 0;
  return staging_plan(cfg).total;
}

int32_t h3dit_streamed_blocks(const h3dit_ctx *ctx) { return ctx ? ctx->n_streamed : -1; }

h3dit_status h3dit_attach_staging(h3dit_ctx *ctx, void *staging, size_t bytes, void *copy_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  const Staging S = staging_plan(&ctx->cfg);
  if (!staging || (reinterpret_cast<uintptr_t>(staging) % kAlign) || bytes < S.total)
    return ctx->fail(H3DIT_ERR_WORKSPACE, "staging needs %zu bytes, 256-byte aligned", S.total);
  ctx->release_streaming();
  ctx->SP = S;
  ctx->staging = static_cast<uint8_t *>(staging);
  cudaError_t e = cudaSuccess;
  if (copy_stream) {
    ctx->copy = static_cast<cudaStream_t>(copy_stream);
  } else {
    e = cudaStreamCreateWithFlags(&ctx->copy, cudaStreamNonBlocking);
    ctx->own_copy = e == cudaSuccess;
  }
  for (cudaEvent_t *ev : {&ctx->fork, &ctx->join, &ctx->ready[0], &ctx->ready[1],
                          &ctx->slot_free[0], &ctx->slot_free[1]})
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e == cudaSuccess) {
    // the AdaLN kernel's pointer table for the two slots: w_ada[2], b_ada[2]
    const void *table[4];
    for (int s = 0; s < 2; ++s) {
      const h3dit_block_weights w = ctx->slot_weights(s);
      table[s] = w.w_ada;
      table[2 + s] = w.b_ada;
    }
    e = cudaMemcpy(ctx->staging + S.table, table, sizeof(table), cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    ctx->release_streaming();
    return ctx->cuda(e, "attach staging");
  }
  return H3DIT_OK;
}

h3dit_status h3dit_sync_status(h3dit_ctx *ctx, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return ctx->cuda(e, "stream synchronize");
  int dev_status = 0;
  e = cudaMemcpy(&dev_status, ctx->status(), sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return ctx->cuda(e, "status read");
  if (dev_status != 0) {
    cudaMemset(ctx->status(), 0, sizeof(int));
    return ctx->fail(H3DIT_ERR_TIMEOUT, "a kernel's bounded wait gave up (device status %d)", dev_status);
  }
  return H3DIT_OK;
}

h3dit_status h3dit_time_embed(h3dit_ctx *ctx, float t, float *c_out, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  if (!c_out) return ctx->fail(H3DIT_ERR_INVALID_ARG, "c_out is NULL");
  const h3dit_time_weights &w = ctx->tw;
  Launch L(ctx, H3DIT_KERNEL_TIME_EMBED, static_cast<cudaStream_t>(cuda_stream), 2);
  return ctx->cuda(launch_time_embed(t, ctx->cfg.t_scale, w.w_t1, w.b_t1, w.w_t2, w.b_t2,
                                     ctx->hidden(), c_out, ctx->cfg.hidden, ctx->status(),
                                     static_cast<cudaStream_t>(cuda_stream)),
                   "time embed launch");
}

h3dit_status h3dit_adaln_project(h3dit_ctx *ctx, const float *c, int32_t first, int32_t count,
                                 float *mod_out, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  if (!c || !mod_out) return ctx->fail(H3DIT_ERR_INVALID_ARG, "NULL pointer");
  if (first < 0 || count < 0 || first + count > ctx->cfg.n_blocks)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "block range [%d, %d) outside [0, %d)", first,
                     first + count, ctx->cfg.n_blocks);
  if (count == 0) return H3DIT_OK;
  Launch L(ctx, H3DIT_KERNEL_ADALN, static_cast<cudaStream_t>(cuda_stream));
  return ctx->cuda(launch_adaln(c, ctx->wptr(), ctx->bptr(), first, count, mod_out,
                                ctx->cfg.hidden, ctx->num_sms,
                                static_cast<cudaStream_t>(cuda_stream)),
                   "adaln launch");
}

h3dit_status h3dit_rmsnorm_modulate(h3dit_ctx *ctx, const float *x, const float *shift,
                                    const float *scale, void *xm_out, int32_t n,
                                    void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (n < 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return H3DIT_OK;
  if (!x || !shift || !scale || !xm_out || !aligned16(x) || !aligned16(shift) ||
      !aligned16(scale) || !aligned16(xm_out))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  return run_rmsnorm(ctx, x, shift, scale, xm_out, n, static_cast<cudaStream_t>(cuda_stream));
}

h3dit_status h3dit_rope_table(h3dit_ctx *ctx, const h3dit_grid *grids, int32_t n_grids,
                              int32_t n_txt, float *table_out, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (n_txt < 0 || n_grids < 0 || n_grids > kMaxGrids || (n_grids > 0 && !grids))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "bad grids");
  long long n = n_txt;
  for (int g = 0; g < n_grids; ++g) {
    if (grids[g].height <= 0 || grids[g].width <= 0 || grids[g].frame < 0)
      return ctx->fail(H3DIT_ERR_INVALID_ARG, "grid %d has a bad shape", g);
    n += static_cast<long long>(grids[g].height) * grids[g].width;
  }
  if (n == 0) return H3DIT_OK;
  if (!table_out) return ctx->fail(H3DIT_ERR_INVALID_ARG, "table_out is NULL");
  if (n > (1LL << 30)) return ctx->fail(H3DIT_ERR_INVALID_ARG, "too many tokens");
  return rope_table_into(ctx, grids, n_grids, n_txt, static_cast<int>(n), table_out,
                         static_cast<cudaStream_t>(cuda_stream));
}

namespace {
// Shape rules shared by the latent entry points: C in [1, 32], even sides,
// and at most max_tokens tokens.
h3dit_status check_latent(h3dit_ctx *ctx, const float *latent, int channels, int lat_h,
                          int lat_w) {
  if (!latent || !aligned16(latent)) return ctx->fail(H3DIT_ERR_INVALID_ARG, "latent is NULL or misaligned");
  if (channels < 1 || channels > 32)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "latent channels %d outside [1, 32]", channels);
  if (lat_h < 2 || lat_w < 2 || (lat_h & 1) || (lat_w & 1))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "latent sides %d x %d must be even and >= 2", lat_h, lat_w);
  const long long n = static_cast<long long>(lat_h / 2) * (lat_w / 2);
  if (n > ctx->cfg.max_tokens)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "%lld tokens exceed max_tokens=%d", n, ctx->cfg.max_tokens);
  return H3DIT_OK;
}
}  // namespace

h3dit_status h3dit_embed_latent(h3dit_ctx *ctx, const float *latent, int32_t channels,
                                int32_t lat_h, int32_t lat_w, const float *w_in, const float *b_in,
                                void *x_img_out, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  h3dit_status st = check_latent(ctx, latent, channels, lat_h, lat_w);
  if (st) return st;
  if (!w_in || !b_in || !x_img_out || !aligned16(w_in) || !aligned16(b_in) || !aligned16(x_img_out))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "embedding: NULL or misaligned pointer");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  Launch L(ctx, H3DIT_KERNEL_IO, s);
  return ctx->cuda(launch_embed_latent(latent, channels, lat_h, lat_w, w_in, b_in, ctx->cfg.hidden,
                                       x_img_out, ctx->cfg.io_fp32 != 0, s),
                   "embed latent launch");
}

h3dit_status h3dit_output_modulation(h3dit_ctx *ctx, const float *c, const float *w_mod,
                                     const float *b_mod, float *mod_out, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (!c || !w_mod || !b_mod || !mod_out)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "output modulation: NULL pointer");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  Launch L(ctx, H3DIT_KERNEL_IO, s);
  return ctx->cuda(launch_output_modulation(c, w_mod, b_mod, mod_out, ctx->cfg.hidden, s),
                   "output modulation launch");
}

h3dit_status h3dit_output_euler(h3dit_ctx *ctx, const void *x_img, const float *mod,
                                const float *w_out, const float *b_out, float *latent,
                                int32_t channels, int32_t lat_h, int32_t lat_w, float dt,
                                void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  h3dit_status st = check_latent(ctx, latent, channels, lat_h, lat_w);
  if (st) return st;
  if (!x_img || !mod || !w_out || !b_out)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "output layer: NULL pointer");
  if (!(dt == dt)) return ctx->fail(H3DIT_ERR_INVALID_ARG, "dt is NaN");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  Launch L(ctx, H3DIT_KERNEL_IO, s, 2);
  return ctx->cuda(launch_output_euler(x_img, ctx->cfg.io_fp32 != 0, mod, w_out, b_out,
                                       ctx->cfg.hidden, ctx->cfg.norm_eps, latent, channels, lat_h,
                                       lat_w, dt, ctx->resid(), s),
                   "output layer launch");
}

h3dit_status h3dit_linear(h3dit_ctx *ctx, int32_t epilogue, const void *a, const void *w,
                          int32_t m, int32_t n, int32_t k, void *out, const float *gate,
                          const float *rope_table, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  return run_linear(ctx, epilogue, a, w, m, n, k, out, n, gate, rope_table,
                    static_cast<cudaStream_t>(cuda_stream));
}

h3dit_status h3dit_attention(h3dit_ctx *ctx, const void *q, const void *k, const void *v,
                             int32_t ld_qkv, void *o, int32_t ld_o, int32_t n,
                             void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  return run_attention(ctx, q, k, v, ld_qkv, o, ld_o, n, static_cast<cudaStream_t>(cuda_stream));
}

h3dit_status h3dit_attention_heads(h3dit_ctx *ctx, int32_t heads, const void *q, const void *k,
                                   const void *v, int32_t ld_qkv, void *o, int32_t ld_o, int32_t n,
                                   void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (heads < 1) return ctx->fail(H3DIT_ERR_INVALID_ARG, "heads < 1");
  return run_attention(ctx, q, k, v, ld_qkv, o, ld_o, n, static_cast<cudaStream_t>(cuda_stream),
                       nullptr, heads);
}

namespace {
// Counts first; with no tokens the data pointers are not examined.
h3dit_status check_sp(h3dit_ctx *ctx, const void *a, const void *b, int n_local, int ranks) {
  if (n_local < 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "n_local < 0");
  if (ranks < 1 || ctx->cfg.heads % ranks)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "%d ranks do not divide %d heads", ranks, ctx->cfg.heads);
  if ((ctx->inner() / ranks) % 8)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a head group's width is not a multiple of 8");
  if (n_local > 0 && (!a || !b || !aligned16(a) || !aligned16(b)))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "sequence parallel re-layout: NULL or misaligned pointer");
  return H3DIT_OK;
}
}  // namespace

h3dit_status h3dit_sp_pack_qkv(h3dit_ctx *ctx, const void *qkv, int32_t n_local, int32_t ranks,
                               void *send, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  h3dit_status st = check_sp(ctx, qkv, send, n_local, ranks);
  if (st || n_local == 0) return st;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  Launch L(ctx, H3DIT_KERNEL_PACK, s);
  return ctx->cuda(launch_sp_pack_qkv(qkv, n_local, ranks, ctx->inner() / ranks, send,
                                      ctx->num_sms, s),
                   "sequence parallel pack launch");
}

h3dit_status h3dit_sp_unpack_o(h3dit_ctx *ctx, const void *recv, int32_t n_local, int32_t ranks,
                               void *o, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  h3dit_status st = check_sp(ctx, recv, o, n_local, ranks);
  if (st || n_local == 0) return st;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  Launch L(ctx, H3DIT_KERNEL_PACK, s);
  return ctx->cuda(launch_sp_unpack_o(recv, n_local, ranks, ctx->inner() / ranks, o, ctx->num_sms,
                                      s),
                   "sequence parallel unpack launch");
}

namespace {
h3dit_status check_scatter(h3dit_ctx *ctx, void *const *dst, int ranks, int rank, int count) {
  if (ranks < 1 || ranks > kMaxScatterRanks)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "%d ranks: the fused exchange addresses 1 .. %d",
                     ranks, kMaxScatterRanks);
  if (rank < 0 || rank >= ranks)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "rank %d outside [0, %d)", rank, ranks);
  if (count < 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "negative token count");
  if (count == 0) return H3DIT_OK;  // no tokens: the destinations are not examined
  if (!dst) return ctx->fail(H3DIT_ERR_INVALID_ARG, "NULL destination array");
  for (int g = 0; g < ranks; ++g)
    if (!dst[g] || !aligned16(dst[g]))
      return ctx->fail(H3DIT_ERR_INVALID_ARG, "destination of rank %d is NULL or misaligned", g);
  return H3DIT_OK;
}
}  // namespace

h3dit_status h3dit_sp_qkv_scatter(h3dit_ctx *ctx, const void *xm, int32_t n_local,
                                  const void *w_qkv, const float *rope_rows, void *const *recv,
                                  int32_t ranks, int32_t rank, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  h3dit_status st = check_scatter(ctx, recv, ranks, rank, n_local);
  if (st) return st;
  if ((st = check_sp(ctx, xm, w_qkv, n_local, ranks)) || n_local == 0) return st;
  const ScatterTargets sc{recv, ranks, rank};
  const int I = ctx->inner();
  return run_linear(ctx, H3DIT_EPI_QKV_ROPE, xm, w_qkv, n_local, 3 * I, ctx->cfg.hidden, nullptr,
                    0, nullptr, rope_rows, static_cast<cudaStream_t>(cuda_stream), nullptr, -1,
                    &sc);
}

h3dit_status h3dit_sp_attention_scatter(h3dit_ctx *ctx, const void *qkv, int32_t n_total,
                                        void *const *o, int32_t ranks, int32_t rank,
                                        void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  h3dit_status st = check_scatter(ctx, o, ranks, rank, n_total);
  if (st) return st;
  if ((st = check_sp(ctx, qkv, n_total ? o[0] : nullptr, n_total, ranks)) || n_total == 0) return st;
  if (n_total % ranks)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "%d tokens do not split over %d ranks", n_total, ranks);
  const ScatterTargets sc{o, ranks, rank};
  const int I = ctx->inner(), cw = I / ranks;
  const uint16_t *q = static_cast<const uint16_t *>(qkv);
  return run_attention(ctx, q, q + cw, q + 2 * cw, 3 * cw, nullptr, I, n_total,
                       static_cast<cudaStream_t>(cuda_stream), nullptr, ctx->cfg.heads / ranks, 1,
                       &sc);
}

h3dit_status h3dit_sp_qkv_scatter_mx(h3dit_ctx *ctx, const void *xq, const void *xq_sf,
                                     int32_t n_local, int32_t block, const float *rope_rows,
                                     void *const *recv, int32_t ranks, int32_t rank,
                                     void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (!ctx->mx()) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "the context is not MXFP8");
  if (block < 0 || block >= ctx->cfg.n_blocks)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "block %d outside [0, %d)", block, ctx->cfg.n_blocks);
  h3dit_status st = check_scatter(ctx, recv, ranks, rank, n_local);
  if (st) return st;
  if ((st = check_sp(ctx, xq, xq_sf, n_local, ranks)) || n_local == 0) return st;
  const MxWeights &o = ctx->L.wq_off;
  const int I = ctx->inner();
  const ScatterTargets sc{recv, ranks, rank};
  return run_linear_mx(ctx, H3DIT_EPI_QKV_ROPE, xq, xq_sf, ctx->wq(block, o.qkv),
                       ctx->wq(block, o.qkv_sf), n_local, 3 * I, ctx->cfg.hidden, nullptr, 3 * I,
                       nullptr, nullptr, rope_rows, static_cast<cudaStream_t>(cuda_stream),
                       o.qkv_sft == kNoTiled ? nullptr : ctx->wq(block, o.qkv_sft), &sc);
}

h3dit_status h3dit_sp_attention_scatter_mx(h3dit_ctx *ctx, const void *qkv, int32_t n_total,
                                           void *const *o, void *const *o_sf, int32_t ranks,
                                           int32_t rank, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  h3dit_status st = check_scatter(ctx, o, ranks, rank, n_total);
  if (st) return st;
  if (n_total > 0 && !o_sf) return ctx->fail(H3DIT_ERR_INVALID_ARG, "NULL scale array list");
  if ((st = check_sp(ctx, qkv, n_total ? o[0] : nullptr, n_total, ranks)) || n_total == 0)
    return st;
  if (n_total % ranks)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "%d tokens do not split over %d ranks", n_total, ranks);
  const ScatterTargets sc{o, ranks, rank, o_sf};
  const int I = ctx->inner(), cw = I / ranks;
  const uint16_t *q = static_cast<const uint16_t *>(qkv);
  return run_attention(ctx, q, q + cw, q + 2 * cw, 3 * cw, nullptr, I, n_total,
                       static_cast<cudaStream_t>(cuda_stream), nullptr, ctx->cfg.heads / ranks, 1,
                       &sc);
}

namespace {
typedef CUresult (*AddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);
AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
  }
  return fn;
}
}  // namespace

h3dit_status h3dit_ipc_get_handle(const void *dev_ptr, void *handle_out, uint64_t *offset_out) {
  static_assert(sizeof(cudaIpcMemHandle_t) == H3DIT_IPC_HANDLE_BYTES, "IPC handle size");
  if (!dev_ptr || !handle_out || !offset_out) return H3DIT_ERR_INVALID_ARG;
  AddressRangeFn range = address_range_fn();
  if (!range) return H3DIT_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return H3DIT_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) {
    cudaGetLastError();
    return H3DIT_ERR_CUDA;
  }
  std::memcpy(handle_out, &h, sizeof h);
  *offset_out = reinterpret_cast<uintptr_t>(dev_ptr) - static_cast<uintptr_t>(base);
  return H3DIT_OK;
}

h3dit_status h3dit_ipc_open(const void *handle, uint64_t offset, void **dev_ptr_out) {
  if (!handle || !dev_ptr_out) return H3DIT_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof h);
  void *base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return H3DIT_ERR_CUDA;
  }
  *dev_ptr_out = static_cast<uint8_t *>(base) + offset;
  return H3DIT_OK;
}

h3dit_status h3dit_ipc_close(void *dev_ptr, uint64_t offset) {
  if (!dev_ptr) return H3DIT_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle(static_cast<uint8_t *>(dev_ptr) - offset) != cudaSuccess) {
    cudaGetLastError();
    return H3DIT_ERR_CUDA;
  }
  return H3DIT_OK;
}

h3dit_status h3dit_block_forward(h3dit_ctx *ctx, int32_t block, float t, const float *mod,
                                 void *x_img, const h3dit_grid *grids, int32_t n_grids,
                                 void *x_txt, int32_t n_txt, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  if (block < 0 || block >= ctx->cfg.n_blocks)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "block %d outside [0, %d)", block, ctx->cfg.n_blocks);
  if (mod && !aligned16(mod)) return ctx->fail(H3DIT_ERR_INVALID_ARG, "mod is misaligned");
  int n_img = 0;
  h3dit_status st = check_tokens(ctx, x_img, grids, n_grids, x_txt, n_txt, &n_img);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int n = n_txt + n_img;
  if ((st = rope_table_into(ctx, grids, n_grids, n_txt, n, ctx->rope(), s))) return st;
  if (!mod) {
    if ((st = h3dit_time_embed(ctx, t, ctx->cvec(), s))) return st;
    if ((st = adaln_resident(ctx, block, block + 1, s))) return st;
  }
  if ((st = run_pack(ctx, x_txt, n_txt, x_img, n_img, s))) return st;
  if ((st = run_blocks(ctx, block, block + 1, n, s, mod))) return st;
  return run_unpack(ctx, n_txt, n_img, x_txt, x_img, s);
}

h3dit_status h3dit_step(h3dit_ctx *ctx, float t, void *x_img, const h3dit_grid *grids,
                        int32_t n_grids, void *x_txt, int32_t n_txt, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  int n_img = 0;
  h3dit_status st = check_tokens(ctx, x_img, grids, n_grids, x_txt, n_txt, &n_img);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int n = n_txt + n_img;
  if ((st = rope_table_into(ctx, grids, n_grids, n_txt, n, ctx->rope(), s))) return st;
  if ((st = h3dit_time_embed(ctx, t, ctx->cvec(), s))) return st;
  if ((st = adaln_resident(ctx, 0, ctx->cfg.n_blocks, s))) return st;
  if ((st = run_pack(ctx, x_txt, n_txt, x_img, n_img, s))) return st;
  if ((st = run_blocks(ctx, 0, ctx->cfg.n_blocks, n, s))) return st;
  return run_unpack(ctx, n_txt, n_img, x_txt, x_img, s);
}

h3dit_status h3dit_denoise(h3dit_ctx *ctx, const h3dit_io_weights *io, float *latent,
                           int32_t channels, int32_t lat_h, int32_t lat_w, const void *x_txt,
                           int32_t n_txt, int32_t n_steps, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "a decoder context runs h3dit_vae_decode");
  if (!io || !io->w_in || !io->b_in || !io->w_mod || !io->b_mod || !io->w_out || !io->b_out ||
      !aligned16(io->w_in) || !aligned16(io->b_in))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "denoise: NULL or misaligned FP32 layer weights");
  h3dit_status st = check_latent(ctx, latent, channels, lat_h, lat_w);
  if (st) return st;
  if (n_steps < 1 || n_steps > 1000)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "n_steps %d outside [1, 1000]", n_steps);
  if (n_txt < 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "n_txt < 0");
  if (n_txt > 0 && (!x_txt || !aligned16(x_txt)))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "x_txt is NULL or misaligned");
  const int D = ctx->cfg.hidden;
  const int h = lat_h / 2, w = lat_w / 2;
  const long long n = static_cast<long long>(n_txt) + static_cast<long long>(h) * w;
  if (n > ctx->cfg.max_tokens)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "%lld tokens exceed max_tokens=%d", n, ctx->cfg.max_tokens);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const h3dit_grid grid{0, h, w};
  if ((st = rope_table_into(ctx, &grid, 1, n_txt, static_cast<int>(n), ctx->rope(), s))) return st;
  // the image rows of the packed fp32 residual stream [text; image]
  float *x_img = ctx->resid() + static_cast<size_t>(n_txt) * D;
  // the FFN hidden buffer is free once the blocks have run: one float per
  // image token of it holds the output layer's row scales
  float *rinv = static_cast<float *>(ctx->u());
  for (int k = 0; k < n_steps; ++k) {
    const double tk = 1.0 - static_cast<double>(k) / n_steps;
    const double tn = 1.0 - static_cast<double>(k + 1) / n_steps;
    const float t = static_cast<float>(tk);
    if ((st = h3dit_time_embed(ctx, t, ctx->cvec(), s))) return st;
    if ((st = adaln_resident(ctx, 0, ctx->cfg.n_blocks, s))) return st;
    {
      Launch L(ctx, H3DIT_KERNEL_IO, s);
      if ((st = ctx->cuda(launch_output_modulation(ctx->cvec(), io->w_mod, io->b_mod, ctx->omod(),
                                                   D, s),
                          "output modulation launch")))
        return st;
    }
    if (n_txt > 0 && (st = run_pack(ctx, x_txt, n_txt, nullptr, 0, s))) return st;
    {
      Launch L(ctx, H3DIT_KERNEL_IO, s);
      if ((st = ctx->cuda(launch_embed_latent(latent, channels, lat_h, lat_w, io->w_in, io->b_in,
                                              D, x_img, true, s),
                          "embed latent launch")))
        return st;
    }
    if ((st = run_blocks(ctx, 0, ctx->cfg.n_blocks, static_cast<int>(n), s))) return st;
    Launch L(ctx, H3DIT_KERNEL_IO, s, 2);
    if ((st = ctx->cuda(launch_output_euler(x_img, true, ctx->omod(), io->w_out, io->b_out, D,
                                            ctx->cfg.norm_eps, latent, channels, lat_h, lat_w,
                                            static_cast<float>(tn - tk), rinv, s),
                        "output layer launch")))
      return st;
  }
  return H3DIT_OK;
}

size_t h3dit_vae_workspace_bytes(const h3dit_vae_config *cfg) {
  if (!vae_config_ok(cfg)) return 0;
  const h3dit_config ic = vae_internal(cfg);
  return plan(&ic).total + vae_extra_bytes(cfg);
}

h3dit_status h3dit_vae_create(const h3dit_vae_config *cfg, const h3dit_vae_weights *w,
                              void *workspace, size_t ws_bytes, void *cuda_stream,
                              h3dit_ctx **out) {
  if (!out) return H3DIT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!vae_config_ok(cfg) || !w || !w->layers) return H3DIT_ERR_INVALID_ARG;
  const void *need[] = {w->w_in, w->b_in, w->lnf_g, w->lnf_b, w->w_out, w->b_out};
  for (const void *p : need)
    if (!p || !aligned16(p)) return H3DIT_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->layers; ++l) {
    const h3dit_vae_layer_weights &v = w->layers[l];
    const void *lp[] = {v.ln1_g, v.ln1_b, v.w_qkv, v.b_qkv, v.w_o, v.b_o,
                        v.ln2_g, v.ln2_b, v.w_1, v.b_1, v.w_2, v.b_2};
    for (const void *p : lp)
      if (!p || !aligned16(p)) return H3DIT_ERR_INVALID_ARG;
  }
  const h3dit_config ic = vae_internal(cfg);
  const Layout L = plan(&ic);
  const size_t total = L.total + vae_extra_bytes(cfg);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) || ws_bytes < total)
    return H3DIT_ERR_WORKSPACE;
  h3dit_ctx *ctx = new (std::nothrow) h3dit_ctx();
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  ctx->cfg = ic;
  ctx->vae = true;
  ctx->vcfg = *cfg;
  ctx->vlayers.assign(w->layers, w->layers + cfg->layers);
  ctx->vw = *w;
  ctx->vw.layers = ctx->vlayers.data();
  ctx->ws = static_cast<uint8_t *>(workspace);
  ctx->ws_bytes = ws_bytes;
  ctx->L = L;
  ctx->vpos = L.total;
  ctx->vones = L.total + round_up(static_cast<size_t>(cfg->tile) * cfg->tile * cfg->width * 4, kAlign);
  ctx->streamed.assign(cfg->layers, 0);
  int dev = 0;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    delete ctx;
    return H3DIT_ERR_CUDA;
  }
  std::vector<float> ones(cfg->width, 1.0f);
  cudaError_t e = cudaMemsetAsync(ctx->status(), 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = launch_vae_pos_table(cfg->tile, cfg->width, reinterpret_cast<float *>(ctx->ws + ctx->vpos),
                             ctx->num_sms, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(ctx->ws + ctx->vones, ones.data(), ones.size() * sizeof(float),
                        cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // the host vector dies with this call
  if (e != cudaSuccess) {
    delete ctx;
    return H3DIT_ERR_CUDA;
  }
  *out = ctx;
  return H3DIT_OK;
}

h3dit_status h3dit_vae_decode(h3dit_ctx *ctx, const float *latent, int32_t lat_h, int32_t lat_w,
                              float *image, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (!ctx->vae) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "not a decoder context (h3dit_vae_create)");
  if (!latent || !image || !aligned16(latent) || !aligned16(image))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "decode: NULL or misaligned latent or image");
  const int T = ctx->vcfg.tile;
  if (lat_h < 1 || lat_w < 1) return ctx->fail(H3DIT_ERR_INVALID_ARG, "empty latent");
  if (lat_h % T || lat_w % T)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "latent sides %d x %d are not multiples of the tile %d",
                     lat_h, lat_w, T);
  const long long n = static_cast<long long>(lat_h) * lat_w;
  if (n > ctx->cfg.max_tokens)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "%lld tokens exceed max_tokens=%d", n, ctx->cfg.max_tokens);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int W = ctx->cfg.hidden, tiles = static_cast<int>(n / (static_cast<long long>(T) * T));
  h3dit_status st;
  {
    Launch L(ctx, H3DIT_KERNEL_IO, s);
    if ((st = ctx->cuda(launch_vae_embed(latent, ctx->vcfg.channels, lat_h, lat_w, T, ctx->vw.w_in,
                                         ctx->vw.b_in,
                                         reinterpret_cast<const float *>(ctx->ws + ctx->vpos), W,
                                         ctx->resid(), s),
                        "decoder embedding launch")))
      return st;
  }
  for (int l = 0; l < ctx->vcfg.layers; ++l)
    if ((st = vae_layer(ctx, ctx->vlayers[l], static_cast<int>(n), tiles, s))) return st;
  if ((st = run_layernorm(ctx, ctx->resid(), ctx->vw.lnf_g, ctx->vw.lnf_b, ctx->xm(),
                          static_cast<int>(n), s)))
    return st;
  if ((st = run_linear(ctx, H3DIT_EPI_STORE, ctx->xm(), ctx->vw.w_out, static_cast<int>(n), 768, W,
                       ctx->u(), 768, nullptr, nullptr, s, ctx->vw.b_out, H3DIT_KERNEL_IO)))
    return st;
  Launch L(ctx, H3DIT_KERNEL_IO, s);
  return ctx->cuda(launch_vae_pixels(ctx->u(), lat_h, lat_w, T, image, ctx->num_sms, s),
                   "decoder pixels launch");
}

h3dit_status h3dit_layernorm(h3dit_ctx *ctx, const float *x, const float *gain, const float *bias,
                             void *out, int32_t n, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (n < 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return H3DIT_OK;
  if (!x || !gain || !bias || !out || !aligned16(x) || !aligned16(gain) || !aligned16(bias) ||
      !aligned16(out))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  return run_layernorm(ctx, x, gain, bias, out, n, static_cast<cudaStream_t>(cuda_stream));
}

h3dit_status h3dit_linear_bias(h3dit_ctx *ctx, int32_t epilogue, const void *a, const void *w,
                               const float *bias, int32_t m, int32_t n, int32_t k, void *out,
                               const float *gate, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (!bias) return ctx->fail(H3DIT_ERR_INVALID_ARG, "bias is NULL");
  return run_linear(ctx, epilogue, a, w, m, n, k, out, n, gate, nullptr,
                    static_cast<cudaStream_t>(cuda_stream), bias);
}

h3dit_status h3dit_attention_batched(h3dit_ctx *ctx, const void *q, const void *k, const void *v,
                                     int32_t ld_qkv, void *o, int32_t ld_o, int32_t n,
                                     int32_t batch, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  return run_attention(ctx, q, k, v, ld_qkv, o, ld_o, n, static_cast<cudaStream_t>(cuda_stream),
                       nullptr, 0, batch);
}

size_t h3dit_mx_scale_bytes(int32_t rows, int32_t k) {
  if (rows <= 0 || k <= 0 || k % 128) return 0;
  return mx_sf_bytes(rows, k);
}

h3dit_status h3dit_mx_quantize(h3dit_ctx *ctx, const void *src, int32_t rows, int32_t k, void *dst,
                               void *sf, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (rows < 0 || k <= 0 || k % 128)
    return ctx->fail(H3DIT_ERR_UNSUPPORTED, "MXFP8 quantization needs k a multiple of 128");
  if (rows == 0) return H3DIT_OK;
  if (!src || !dst || !sf || !aligned16(src) || !aligned16(dst))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  Launch L(ctx, H3DIT_KERNEL_MX_QUANTIZE, static_cast<cudaStream_t>(cuda_stream));
  return ctx->cuda(launch_mx_quantize(src, k, rows, k, static_cast<uint8_t *>(dst),
                                      static_cast<uint8_t *>(sf),
                                      static_cast<cudaStream_t>(cuda_stream)),
                   "quantize launch");
}

h3dit_status h3dit_linear_mx(h3dit_ctx *ctx, int32_t epilogue, const void *a, const void *a_sf,
                             const void *w, const void *w_sf, int32_t m, int32_t n, int32_t k,
                             void *out, void *out_sf, const float *gate, const float *rope_table,
                             void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  return run_linear_mx(ctx, epilogue, a, a_sf, w, w_sf, m, n, k, out, n, out_sf, gate, rope_table,
                       static_cast<cudaStream_t>(cuda_stream));
}

h3dit_status h3dit_block_linear_mx(h3dit_ctx *ctx, int32_t block, int32_t which, const void *a,
                                   const void *a_sf, int32_t m, void *out, void *out_sf,
                                   const float *gate, const float *rope_table, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (!ctx->mx()) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "the context is not MXFP8");
  if (block < 0 || block >= ctx->cfg.n_blocks)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "block %d outside [0, %d)", block, ctx->cfg.n_blocks);
  const int D = ctx->cfg.hidden, I = ctx->inner(), F = ctx->cfg.ffn;
  const MxWeights &o = ctx->L.wq_off;
  auto tiled = [&](size_t off) -> const void * {
    return off == kNoTiled ? nullptr : ctx->wq(block, off);
  };
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  switch (which) {
    case H3DIT_LINEAR_QKV:
      return run_linear_mx(ctx, H3DIT_EPI_QKV_ROPE, a, a_sf, ctx->wq(block, o.qkv),
                           ctx->wq(block, o.qkv_sf), m, 3 * I, D, out, 3 * I, nullptr, nullptr,
                           rope_table, s, tiled(o.qkv_sft));
    case H3DIT_LINEAR_OUT:
      return run_linear_mx(ctx, H3DIT_EPI_GATED_RESIDUAL, a, a_sf, ctx->wq(block, o.o),
                           ctx->wq(block, o.o_sf), m, D, I, out, D, nullptr, gate, nullptr, s,
                           tiled(o.o_sft));
    case H3DIT_LINEAR_FFN1:
      return run_linear_mx(ctx, H3DIT_EPI_GELU, a, a_sf, ctx->wq(block, o.ff1),
                           ctx->wq(block, o.ff1_sf), m, F, D, out, F, out_sf, nullptr, nullptr, s,
                           tiled(o.ff1_sft));
    case H3DIT_LINEAR_FFN2:
      return run_linear_mx(ctx, H3DIT_EPI_GATED_RESIDUAL, a, a_sf, ctx->wq(block, o.ff2),
                           ctx->wq(block, o.ff2_sf), m, D, F, out, D, nullptr, gate, nullptr, s,
                           tiled(o.ff2_sft));
    default:
      return ctx->fail(H3DIT_ERR_INVALID_ARG, "unknown linear %d", which);
  }
}

h3dit_status h3dit_rmsnorm_modulate_mx(h3dit_ctx *ctx, const float *x, const float *shift,
                                       const float *scale, void *out, void *out_sf, int32_t n,
                                       void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (n < 0) return ctx->fail(H3DIT_ERR_INVALID_ARG, "n < 0");
  if (ctx->cfg.hidden % 128) return ctx->fail(H3DIT_ERR_UNSUPPORTED, "MXFP8 needs hidden % 128 == 0");
  if (n == 0) return H3DIT_OK;
  if (!x || !shift || !scale || !out || !out_sf || !aligned16(x) || !aligned16(shift) ||
      !aligned16(scale) || !aligned16(out))
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  return run_rmsnorm(ctx, x, shift, scale, out, n, static_cast<cudaStream_t>(cuda_stream),
                     static_cast<uint8_t *>(out_sf));
}

h3dit_status h3dit_attention_mx(h3dit_ctx *ctx, const void *q, const void *k, const void *v,
                                int32_t ld_qkv, void *o, void *o_sf, int32_t n, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (!o_sf) return ctx->fail(H3DIT_ERR_INVALID_ARG, "o_sf is NULL");
  return run_attention(ctx, q, k, v, ld_qkv, o, ctx->inner(), n,
                       static_cast<cudaStream_t>(cuda_stream), o_sf);
}

h3dit_status h3dit_time_embed_static(const float *w_t1, const float *b_t1, const float *w_t2,
                                     const float *b_t2, int32_t hidden, float t, float t_scale,
                                     float *c_out, void *cuda_stream) {
  if (!w_t1 || !b_t1 || !w_t2 || !b_t2 || !c_out || !aligned16(w_t2)) return H3DIT_ERR_INVALID_ARG;
  if (hidden < 1 || hidden % 4) return H3DIT_ERR_INVALID_ARG;
  if (hidden > H3DIT_STATIC_TIME_MAX_HIDDEN) return H3DIT_ERR_UNSUPPORTED;
  static_assert(H3DIT_STATIC_TIME_MAX_HIDDEN == kStaticTimeMaxHidden, "scratch size");
  cudaError_t e = launch_time_embed_static(t, t_scale, w_t1, b_t1, w_t2, b_t2, c_out, hidden,
                                           static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? H3DIT_OK : H3DIT_ERR_CUDA;
}

h3dit_status h3dit_selftest_bounded_wait(h3dit_ctx *ctx, int32_t limit_us, void *cuda_stream) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  if (limit_us < 1 || limit_us > 1000000)
    return ctx->fail(H3DIT_ERR_INVALID_ARG, "limit_us must be in [1, 1e6]");
  int dev = 0, khz = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0)
    khz = 2000000;
  const long long cycles = static_cast<long long>(limit_us) * (khz / 1000);
  return ctx->cuda(launch_selftest_wait(ctx->status(), cycles, static_cast<cudaStream_t>(cuda_stream)),
                   "self-test launch");
}

h3dit_status h3dit_attention_stamps(uint64_t *host, int32_t slots, int32_t steps) {
  if (!host) return H3DIT_ERR_INVALID_ARG;
  const int r = attention_stamps(reinterpret_cast<unsigned long long *>(host), slots, steps);
  return r == 0 ? H3DIT_OK : r == 1 || r == -1 ? H3DIT_ERR_UNSUPPORTED : H3DIT_ERR_CUDA;
}

h3dit_status h3dit_profile_begin(h3dit_ctx *ctx) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  ctx->recycle_records();
  ctx->profiling = true;
  return H3DIT_OK;
}

h3dit_status h3dit_profile_end(h3dit_ctx *ctx, float *ms_out, int64_t *launches_out) {
  if (!ctx) return H3DIT_ERR_INVALID_ARG;
  ctx->profiling = false;
  float ms[H3DIT_KERNEL_COUNT] = {};
  int64_t cnt[H3DIT_KERNEL_COUNT] = {};
  for (const ProfRecord &r : ctx->records) {
    cudaError_t e = cudaEventSynchronize(r.end);
    float t = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.begin, r.end);
    if (e != cudaSuccess) {
      ctx->recycle_records();
      return ctx->cuda(e, "profile event");
    }
    ms[r.kind] += t;
    cnt[r.kind] += 1;
  }
  ctx->recycle_records();
  for (int k = 0; k < H3DIT_KERNEL_COUNT; ++k) {
    if (ms_out) ms_out[k] = ms[k];
    if (launches_out) launches_out[k] = cnt[k];
  }
  return H3DIT_OK;
}

int64_t h3dit_launch_count(const h3dit_ctx *ctx) { return ctx ? ctx->launches : 0; }

}  // extern "C"
