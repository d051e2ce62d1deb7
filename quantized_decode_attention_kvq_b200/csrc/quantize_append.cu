// quantize_append.cu -- quantize-on-append into the paged Tier-1 cache.
//
// "Runtime-Certified Bounded-Error Quantized Attention", Methodology 1
// (Tier 1): keys as INT8 codes (here per token and k_group channels,
// symmetric; or INT4 after the randomized Walsh-Hadamard rotation of the KQV
// scheme in "Statistical Inference and Quality Measures of KV Cache
// Quantisations Inspired by TurboQuant"), values as per-group INT4 codes with
// scale/offset, and the per-block error annotation eta_b (Methodology 2,
// E_val) raised as each token lands in its block.
//
// One warp quantizes one (token, kv head) with quantize_token_warp
// (quantize_token.cuh), after finding the token's page through the page table;
// with outlier extraction, the median-multiplier chunk of K and of V goes to
// the block's outlier section first ("Hurwitz Quaternion Multiplicative
// Quantization for KV Cache Compression", Method 3).
#include "kvq_internal.cuh"
#include "quantize_token.cuh"

namespace kvq {

template <int D, int KB, int KG, bool OUT>
__global__ void __launch_bounds__(256) quantize_append_kernel(const AppendArgs a) {
  constexpr int E = D / 32;             // channels per lane
  const BlockLayout L{D, KB, KG, OUT ? 1 : 0};
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int64_t total = (int64_t)a.num_seqs * a.num_tokens * a.hkv;
  if (item >= total) return;
  const int h = (int)(item % a.hkv);
  const int t = (int)((item / a.hkv) % a.num_tokens);
  const int s = (int)(item / ((int64_t)a.hkv * a.num_tokens));
  // The token's k and v (always inside the caller's [num_seqs][num_tokens]
  // input) are loaded first: they do not depend on where the token goes, so
  // their latency overlaps the position -> page-table lookups below.
  const int64_t base = s * a.seq_stride + h * a.head_stride + (int64_t)t * a.tok_stride;
  float xk[E], xv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    xk[e] = load_elem(a.k, a.in_bf16, base + lane * E + e);
    xv[e] = load_elem(a.v, a.in_bf16, base + lane * E + e);
  }
  if (a.valid && t >= a.valid[s]) return;
  const int pos = a.start_pos[s] + t;
  const int lp = pos / kPage;
  if (pos < 0 || lp >= a.max_pages) {
    if (lane == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
    return;
  }
  const int page = a.page_table[(int64_t)s * a.max_pages + lp];
  if (page < 0 || page >= a.num_pages) {
    if (lane == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
    return;
  }
  const int slot = pos % kPage;
  uint8_t* blk = a.pool + ((int64_t)page * a.hkv + h) * L.bytes();
  quantize_token_warp<D, KB, KG, OUT>(xk, xv, blk, slot, a.eta + (int64_t)page * a.hkv + h, a.signs,
                                 a.rot_c, a.err, lane);
}

using AppendKernel = void (*)(const AppendArgs);

AppendKernel select_append_kernel(int d, int kbits, int kgroup, int out) {
#define KVQ_APPEND_CASE(D_, KB_, KG_)                                                \
  if (d == D_ && kbits == KB_ && kgroup == KG_)                                      \
    return out ? quantize_append_kernel<D_, KB_, KG_, true>                          \
               : quantize_append_kernel<D_, KB_, KG_, false>;
  KVQ_APPEND_CASE(128, 8, 128)
  KVQ_APPEND_CASE(128, 8, 64)
  KVQ_APPEND_CASE(128, 8, 32)
  KVQ_APPEND_CASE(128, 4, 128)
  KVQ_APPEND_CASE(128, 4, 64)
  KVQ_APPEND_CASE(128, 4, 32)
  KVQ_APPEND_CASE(64, 8, 64)
  KVQ_APPEND_CASE(64, 8, 32)
  KVQ_APPEND_CASE(64, 4, 64)
  KVQ_APPEND_CASE(64, 4, 32)
#undef KVQ_APPEND_CASE
  return nullptr;
}

cudaError_t launch_append(const AppendArgs& a, int d, int kbits, int kgroup, int out,
                          cudaStream_t stream) {
  AppendKernel k = select_append_kernel(d, kbits, kgroup, out);
  if (!k) return cudaErrorInvalidValue;
  const int64_t items = (int64_t)a.num_seqs * a.num_tokens * a.hkv;
  if (items == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (items + warps - 1) / warps;
  k<<<(unsigned)blocks, warps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
