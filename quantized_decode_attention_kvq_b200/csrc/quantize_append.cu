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
// One warp quantizes one (token, kv head): lane l holds channels
// [l*E, l*E + E), E = d/32.  All codec arithmetic is IEEE fp32 in a fixed
// order (division and subtraction round-to-nearest, rint ties-to-even,
// directed fp16 rounding of scale and zero), so codes, scales and eta are
// bit-identical to a sequential implementation of the same definition.
#include "kvq_internal.cuh"

namespace kvq {

template <int D, int KB, int KG>
__global__ void __launch_bounds__(256) quantize_append_kernel(const AppendArgs a) {
  constexpr int E = D / 32;             // channels per lane
  constexpr int NB = D / 32;            // 32-channel blocks
  constexpr int Q = KB == 8 ? 127 : 7;
  constexpr int LPG_K = KG / E;         // lanes per key group
  constexpr int LPG_V = 32 / E;         // lanes per value group
  const BlockLayout L{D, KB, KG};
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
  if (a.signs) warp_rotate<E>(xk, a.signs, lane, a.rot_c);

  // ---------------- keys: symmetric, per token and KG channels --------------
  {
    bool bad = false;
    float am = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      bad |= !isfinite(xk[e]);
      am = fmaxf(am, fabsf(xk[e]));
    }
#pragma unroll
    for (int o = 1; o < LPG_K; o *= 2) {
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      bad |= __shfl_xor_sync(0xffffffffu, (int)bad, o) != 0;
    }
    const __half s16 = __float2half_ru(__fdiv_rn(am, (float)Q));
    float sc = __half2float(s16);
    if (!isfinite(sc)) bad = true;
    if (bad) sc = 0.0f;
    int code[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float r = sc == 0.0f ? 0.0f : rintf(__fdiv_rn(xk[e], sc));
      r = fminf(fmaxf(r, (float)-Q), (float)Q);
      code[e] = (int)r;
    }
    const int g = lane / LPG_K;
    if (lane % LPG_K == 0) {
      const __half st = bad ? __float2half_rn(0.0f) : s16;
      reinterpret_cast<__half*>(blk + L.ks_off())[slot * L.ngk() + g] = st;
      if (bad) set_error(a.err, KVQ_ERR_RANGE);
    }
    uint8_t* row = blk + slot * L.k_row();
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const int c = lane * E + e;            // even channel of the pair
      const int b = c / 32, w = c % 32;
      if (KB == 8) {
        int byte = (w / 8) * (8 * NB) + 8 * b + (w % 8);
        // 128-byte rows: 16-byte chunk index XOR slot % 8 (bank-conflict-free
        // reads of the page's 16 rows without any swizzle on the copy)
        if (D == 128) byte = (((byte >> 4) ^ (slot & 7)) << 4) | (byte & 15);
        row[byte] = (uint8_t)(int8_t)code[e];
        row[byte + 1] = (uint8_t)(int8_t)code[e + 1];
      } else {
        const int byte = (w / 8) * (4 * NB) + 4 * b + (w % 8) / 2;
        row[byte] = (uint8_t)((code[e] & 0xF) | ((code[e + 1] & 0xF) << 4));
      }
    }
  }

  // ---------------- values: asymmetric 4-bit, per token and 32 channels ----
  {
    bool bad = false;
    float lo = xv[0], hi = xv[0];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      bad |= !isfinite(xv[e]);
      lo = fminf(lo, xv[e]);
      hi = fmaxf(hi, xv[e]);
    }
#pragma unroll
    for (int o = 1; o < LPG_V; o *= 2) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      bad |= __shfl_xor_sync(0xffffffffu, (int)bad, o) != 0;
    }
    const __half z16 = __float2half_rd(lo);
    const float z = __half2float(z16);
    const __half s16 = __float2half_ru(__fdiv_rn(__fsub_rn(hi, z), 15.0f));
    const float sc = __half2float(s16);
    if (!isfinite(z) || !isfinite(sc)) bad = true;
    int code[E];
    float err = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float r = (sc == 0.0f || bad) ? 0.0f : rintf(__fdiv_rn(__fsub_rn(xv[e], z), sc));
      r = fminf(fmaxf(r, 0.0f), 15.0f);
      code[e] = (int)r;
      const float vh = __fmaf_rn(r, sc, z);
      err = fmaxf(err, fabsf(__fsub_rn(xv[e], vh)));
    }
    if (bad) err = 0.0f;
    const int g = lane / LPG_V;
    if (lane % LPG_V == 0) {
      __half2 sz = bad ? __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f))
                       : __halves2half2(s16, z16);
      reinterpret_cast<__half2*>(blk + L.vm_off())[slot * NB + g] = sz;
      if (bad) set_error(a.err, KVQ_ERR_RANGE);
    }
    uint8_t* row = blk + L.v_off() + slot * L.v_row();
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const int c = lane * E + e;
      const int gg = c / 32, w = c % 32;
      const int byte = (w / 4) * (2 * NB) + 2 * gg + (w % 4) / 2;
      row[byte] = (uint8_t)((code[e] & 0xF) | ((code[e + 1] & 0xF) << 4));
    }
#pragma unroll
    for (int o = 1; o < 32; o *= 2) err = fmaxf(err, __shfl_xor_sync(0xffffffffu, err, o));
    if (lane == 0) {
      const float eu = nextafterf(err, INFINITY);
      // non-negative floats order like their bit patterns
      atomicMax(reinterpret_cast<int*>(a.eta + (int64_t)page * a.hkv + h), __float_as_int(eu));
    }
  }
}

using AppendKernel = void (*)(const AppendArgs);

AppendKernel select_append_kernel(int d, int kbits, int kgroup) {
#define KVQ_APPEND_CASE(D_, KB_, KG_) \
  if (d == D_ && kbits == KB_ && kgroup == KG_) return quantize_append_kernel<D_, KB_, KG_>;
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

cudaError_t launch_append(const AppendArgs& a, int d, int kbits, int kgroup,
                          cudaStream_t stream) {
  AppendKernel k = select_append_kernel(d, kbits, kgroup);
  if (!k) return cudaErrorInvalidValue;
  const int64_t items = (int64_t)a.num_seqs * a.num_tokens * a.hkv;
  if (items == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (items + warps - 1) / warps;
  k<<<(unsigned)blocks, warps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
