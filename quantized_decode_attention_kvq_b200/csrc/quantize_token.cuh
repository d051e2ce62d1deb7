// quantize_token.cuh -- the Tier-1 codec of one (token, kv head), executed by
// one warp: lane l holds channels [l*E, l*E + E), E = d/32.
//
// "Runtime-Certified Bounded-Error Quantized Attention", Methodology 1
// (Tier 1): keys as INT8 codes (here per token and k_group channels,
// symmetric; or INT4 after the randomized Walsh-Hadamard rotation of the KQV
// scheme in "Statistical Inference and Quality Measures of KV Cache
// Quantisations Inspired by TurboQuant"), values as per-group INT4 codes with
// scale/offset, and the per-block error annotation eta_b (Methodology 2,
// E_val) raised with an atomic max as the token lands in its block.  All codec
// arithmetic is IEEE fp32 in a fixed order (division and subtraction
// round-to-nearest, rint ties-to-even, directed fp16 rounding of scale and
// zero), so codes, scales and eta are bit-identical to a sequential
// implementation of the same definition.  Used by the append kernel and by
// the decode kernel's fused append.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

// Writes the token's codes and metadata into slot `slot` of block `blk` and
// raises *eta_slot.  xk, xv: the token's k and v (fp32, this lane's channels);
// xk is rotated in place when `signs` is not NULL.  Returns, in every lane,
// the value the token contributes to eta (its max value error, one ulp up).
template <int D, int KB, int KG>
__device__ __forceinline__ float quantize_token_warp(float (&xk)[D / 32], float (&xv)[D / 32],
                                                    uint8_t* blk, int slot, float* eta_slot,
                                                    const int8_t* signs, float rot_c,
                                                    int32_t* err_word, int lane) {
  constexpr int E = D / 32;             // channels per lane
  constexpr int NB = D / 32;            // 32-channel blocks
  constexpr int Q = KB == 8 ? 127 : 7;
  constexpr int LPG_K = KG / E;         // lanes per key group
  constexpr int LPG_V = 32 / E;         // lanes per value group
  const BlockLayout L{D, KB, KG};
  if (signs) warp_rotate<E>(xk, signs, lane, rot_c);

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
      if (bad) set_error(err_word, KVQ_ERR_RANGE);
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
      if (bad) set_error(err_word, KVQ_ERR_RANGE);
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
    const float eu = nextafterf(err, INFINITY);
    if (lane == 0) {
      // non-negative floats order like their bit patterns
      atomicMax(reinterpret_cast<int*>(eta_slot), __float_as_int(eu));
    }
    return eu;
  }
}

}  // namespace kvq
