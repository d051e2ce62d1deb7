// fallback_exact.cu -- exact dense attention for queries whose certified
// bound exceeded tau ("Runtime-Certified Bounded-Error Quantized Attention",
// Methodology 1, Fallback: page in the Tier-2 originals and run exact
// scaled-dot-product attention for the affected head; Methodology 3,
// per-head rung, applied per query).
//
// The originals of one (sequence, kv head) sit in the staging buffer as
// K [n][D] then V [n][D] (bf16 or fp32).  One CTA takes one item: up to
// kFbRows flagged query rows of that (sequence, kv head) over a token range,
// so each K/V row is read once for all of them.  8 warps split the range;
// a warp holds kFbUnroll tokens in flight (lane l owns channels
// [l*E, l*E+E), scores summed across the warp with shuffles) and keeps one
// fp32 online softmax per row; the warps merge in shared memory.  An item
// that covers the whole range writes the output row; the chunks of a split
// range leave (o, m, l) in the scratch and fallback_merge_kernel combines
// them.  The work is bound by the host-to-device copy of the originals,
// which the host side overlaps with these kernels.
#include "kvq_internal.cuh"

namespace kvq {

static_assert(sizeof(FbArgs) <= 4000, "the fallback argument block must fit the 4 KB limit");

constexpr int kFbWarps = 8;
constexpr int kFbUnroll = 8;

__device__ __forceinline__ void load_chans(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load_chans(const __nv_bfloat16* p, float (&x)[2]) {
  const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
  x[0] = __uint_as_float(u << 16);
  x[1] = __uint_as_float(u & 0xffff0000u);
}
__device__ __forceinline__ void load_chans(const float* p, float (&x)[4]) {
  const float4 f = __ldg(reinterpret_cast<const float4*>(p));
  x[0] = f.x;
  x[1] = f.y;
  x[2] = f.z;
  x[3] = f.w;
}
__device__ __forceinline__ void load_chans(const float* p, float (&x)[2]) {
  const float2 f = __ldg(reinterpret_cast<const float2*>(p));
  x[0] = f.x;
  x[1] = f.y;
}

template <int D, typename T>
__global__ void __launch_bounds__(kFbWarps * 32) fallback_exact_kernel(const __grid_constant__ FbArgs a) {
  constexpr int E = D / 32, U = kFbUnroll, R = kFbRows;
  const FbItem& it = a.items[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nr = it.nrows;
  __shared__ float s_m[kFbWarps][R], s_l[kFbWarps][R];
  __shared__ float s_o[kFbWarps][R][D];

  float q[R][E], m[R], l[R], o[R][E];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      o[r][e] = 0.f;
      q[r][e] = r < nr ? load_elem(a.q, a.q_bf16, (it.row0 + it.roff[r]) * D + lane * E + e) * a.s_att
                       : 0.f;
    }
  }
  const T* K = reinterpret_cast<const T*>(a.staging + it.k_off);
  const T* V = reinterpret_cast<const T*>(a.staging + it.v_off);
  for (int tb = it.t0 + warp * U; tb < it.t1; tb += kFbWarps * U) {
    const int valid = it.t1 - tb;  // >= 1; tokens u >= valid are masked
    float kx[U][E], vx[U][E];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t t = min(tb + u, it.t1 - 1);  // an in-range address for masked tokens
      load_chans(K + t * D + lane * E, kx[u]);
      load_chans(V + t * D + lane * E, vx[u]);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r >= nr) break;
      float s[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        s[u] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) s[u] = fmaf(q[r][e], kx[u][e], s[u]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], off);
      float mx = m[r];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (u < valid) mx = fmaxf(mx, s[u]);
      const float sc = expf(m[r] - mx);  // 0 while m is -inf
      l[r] *= sc;
#pragma unroll
      for (int e = 0; e < E; ++e) o[r][e] *= sc;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float p = u < valid ? expf(s[u] - mx) : 0.f;
        l[r] += p;
#pragma unroll
        for (int e = 0; e < E; ++e) o[r][e] = fmaf(p, vx[u][e], o[r][e]);
      }
      m[r] = mx;
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r >= nr) break;
    if (lane == 0) {
      s_m[warp][r] = m[r];
      s_l[warp][r] = l[r];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) s_o[warp][r][lane * E + e] = o[r][e];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nr * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kFbWarps; ++w) M = fmaxf(M, s_m[w][r]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < kFbWarps; ++w)
      if (s_m[w][r] != -INFINITY) {
        const float f = expf(s_m[w][r] - M);
        L = fmaf(s_l[w][r], f, L);
        acc = fmaf(s_o[w][r][c], f, acc);
      }
    if (it.nchunk == 1) {
      a.out[(it.row0 + it.roff[r]) * D + c] = L > 0.f ? acc / L : 0.f;
    } else {
      float* p = a.scratch + ((size_t)blockIdx.x * R + r) * (D + 2);
      p[c] = acc;
      if (c == 0) {
        p[D] = M;
        p[D + 1] = L;
      }
    }
  }
}

// Items [i, i + nchunk) with chunk 0 at i are the chunks of one row group.
template <int D>
__global__ void __launch_bounds__(256) fallback_merge_kernel(const __grid_constant__ FbArgs a) {
  const FbItem& it = a.items[blockIdx.x];
  if (it.nchunk <= 1 || it.chunk != 0) return;
  const int nc = it.nchunk;
  for (int idx = threadIdx.x; idx < it.nrows * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D;
    float M = -INFINITY;
    for (int j = 0; j < nc; ++j)
      M = fmaxf(M, a.scratch[((size_t)(blockIdx.x + j) * kFbRows + r) * (D + 2) + D]);
    float L = 0.f, acc = 0.f;
    for (int j = 0; j < nc; ++j) {
      const float* p = a.scratch + ((size_t)(blockIdx.x + j) * kFbRows + r) * (D + 2);
      if (p[D] != -INFINITY) {
        const float f = expf(p[D] - M);
        L = fmaf(p[D + 1], f, L);
        acc = fmaf(p[c], f, acc);
      }
    }
    a.out[(it.row0 + it.roff[r]) * D + c] = L > 0.f ? acc / L : 0.f;
  }
}

template <int D>
cudaError_t launch_fallback_d(const FbArgs& a, cudaStream_t stream) {
  if (a.kv_bf16)
    fallback_exact_kernel<D, __nv_bfloat16><<<a.num_items, kFbWarps * 32, 0, stream>>>(a);
  else
    fallback_exact_kernel<D, float><<<a.num_items, kFbWarps * 32, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.any_split) return e;
  fallback_merge_kernel<D><<<a.num_items, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fallback(const FbArgs& a, int d, cudaStream_t stream) {
  if (a.num_items <= 0) return cudaSuccess;
  if (d == 128) return launch_fallback_d<128>(a, stream);
  if (d == 64) return launch_fallback_d<64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
