// Ulysses sequence parallelism ("H3-Image Day-0 Support: 4K in 0.87s with
// Vera Rubin", "Faster DiT": Ulysses SP4; the vLLM-Omni recipe's "Deployment
// profiles", SP 2 / SP 4): every rank holds n consecutive tokens of the packed
// sequence and all heads; around the attention two all-to-alls trade that for
// all tokens and heads / P. These kernels are the re-layouts on either side
// of the exchanges (the exchanges themselves are NCCL's), 16-byte chunks:
//   pack_qkv   qkv [n, 3I] of this rank's tokens, columns [Q | K | V] with
//              heads in order -> send [P][n][3 I/P]: block d holds, for every
//              row, Q | K | V of heads d H/P .. (d + 1) H/P - 1. After the
//              all-to-all, rank d's receive buffer [P][n][3 I/P] is the Q|K|V
//              matrix of its heads for all P n tokens in sequence order, the
//              layout the attention kernel reads (row stride 3 I/P).
//   unpack_o   recv [P][n][I/P], the attention output of this rank's tokens
//              from every head group -> o [n, I], head group s at columns
//              s I/P .. (s + 1) I/P - 1 (the out-projection's A operand).
#include "kernels.h"

namespace h3 {
namespace {

// cw: columns per head group and matrix (I / P); chunks are 8 bf16.
__global__ void sp_pack_qkv_kernel(const uint4 *__restrict__ qkv, int n, int ranks, int cw,
                                   uint4 *__restrict__ send) {
  const long long row_chunks = 3LL * cw / 8;  // chunks of one row of one block
  const long long total = static_cast<long long>(ranks) * n * row_chunks;
  const long long src_row = 3LL * cw * ranks / 8;  // chunks of one qkv row
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e % row_chunks;
    const long long rt = e / row_chunks;  // d * n + t
    const int t = static_cast<int>(rt % n);
    const int d = static_cast<int>(rt / n);
    const int col = static_cast<int>(8 * c);
    const int which = col / cw;  // 0 = Q, 1 = K, 2 = V
    const int off = col - which * cw;
    const long long src_col = static_cast<long long>(which) * cw * ranks +
                              static_cast<long long>(d) * cw + off;
    send[e] = __ldcs(qkv + t * src_row + src_col / 8);
  }
}

__global__ void sp_unpack_o_kernel(const uint4 *__restrict__ recv, int n, int ranks, int cw,
                                   uint4 *__restrict__ o) {
  const long long row_chunks = static_cast<long long>(cw) * ranks / 8;
  const long long total = static_cast<long long>(n) * row_chunks;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e % row_chunks;
    const int t = static_cast<int>(e / row_chunks);
    const int col = static_cast<int>(8 * c);
    const int s = col / cw;
    const int off = col - s * cw;
    o[e] = __ldcs(recv + ((static_cast<long long>(s) * n + t) * cw + off) / 8);
  }
}

int grid_for(long long chunks, int num_sms) {
  const long long want = (chunks + 255) / 256;
  const long long cap = 8LL * num_sms;
  return static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace

cudaError_t launch_sp_pack_qkv(const void *qkv, int n, int ranks, int cw, void *send, int num_sms,
                               cudaStream_t s) {
  if (n <= 0 || ranks <= 0 || cw <= 0 || cw % 8) return cudaErrorInvalidValue;
  const long long chunks = 3LL * ranks * n * cw / 8;
  sp_pack_qkv_kernel<<<grid_for(chunks, num_sms), 256, 0, s>>>(
      static_cast<const uint4 *>(qkv), n, ranks, cw, static_cast<uint4 *>(send));
  return cudaGetLastError();
}

cudaError_t launch_sp_unpack_o(const void *recv, int n, int ranks, int cw, void *o, int num_sms,
                               cudaStream_t s) {
  if (n <= 0 || ranks <= 0 || cw <= 0 || cw % 8) return cudaErrorInvalidValue;
  const long long chunks = static_cast<long long>(ranks) * n * cw / 8;
  sp_unpack_o_kernel<<<grid_for(chunks, num_sms), 256, 0, s>>>(
      static_cast<const uint4 *>(recv), n, ranks, cw, static_cast<uint4 *>(o));
  return cudaGetLastError();
}

}  // namespace h3
