// fallback_exact.cu -- exact dense attention for queries whose certified
// bound exceeded tau ("Runtime-Certified Bounded-Error Quantized Attention",
// Methodology 1, Fallback: page in the Tier-2 originals and run exact
// scaled-dot-product attention for the affected head; Methodology 3,
// per-head rung, applied per query).
//
// The originals of one (sequence, kv head) sit in the staging buffer as
// K [n][D] then V [n][D] (bf16 or fp32).  One CTA recomputes one flagged
// query row: 8 warps split the tokens, each keeps an online softmax in fp32
// (lane l owns channels [l*E, l*E+E), scores reduced across the warp with
// shuffles), and the warps merge in shared memory.
#include "kvq_internal.cuh"

namespace kvq {

constexpr int kFbWarps = 8;
template <int D>
__global__ void __launch_bounds__(kFbWarps * 32) fallback_exact_kernel(const __grid_constant__ FbArgs a) {
  constexpr int E = D / 32;
  const FbItem it = a.items[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float s_m[kFbWarps], s_l[kFbWarps];
  __shared__ float s_o[kFbWarps][D];
  float q[E];
#pragma unroll
  for (int e = 0; e < E; ++e) q[e] = load_elem(a.q, a.q_bf16, it.q_row * D + lane * E + e) * a.s_att;
  const void* K = a.staging + it.k_off;
  const void* V = a.staging + it.v_off;
  float m = -INFINITY, l = 0.f, o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o[e] = 0.f;
  for (int t = warp; t < it.n; t += kFbWarps) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) s = fmaf(q[e], load_elem(K, a.kv_bf16, (int64_t)t * D + lane * E + e), s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(m, s);
    const float al = expf(m - mn);
    const float p = expf(s - mn);
    l = fmaf(l, al, p);
#pragma unroll
    for (int e = 0; e < E; ++e)
      o[e] = fmaf(o[e], al, p * load_elem(V, a.kv_bf16, (int64_t)t * D + lane * E + e));
    m = mn;
  }
  if (lane == 0) {
    s_m[warp] = m;
    s_l[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) s_o[warp][lane * E + e] = o[e];
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < kFbWarps; ++w) M = fmaxf(M, s_m[w]);
  float L = 0.f;
  for (int w = 0; w < kFbWarps; ++w)
    if (s_m[w] != -INFINITY) L = fmaf(s_l[w], expf(s_m[w] - M), L);
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int w = 0; w < kFbWarps; ++w)
      if (s_m[w] != -INFINITY) acc = fmaf(s_o[w][c], expf(s_m[w] - M), acc);
    a.out[it.q_row * D + c] = L > 0.f ? acc / L : 0.f;
  }
}

cudaError_t launch_fallback(const FbArgs& a, int d, cudaStream_t stream) {
  if (a.num_items <= 0) return cudaSuccess;
  if (d == 128)
    fallback_exact_kernel<128><<<a.num_items, kFbWarps * 32, 0, stream>>>(a);
  else if (d == 64)
    fallback_exact_kernel<64><<<a.num_items, kFbWarps * 32, 0, stream>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}


}  // namespace kvq
