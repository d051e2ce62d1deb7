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
//
// With outlier extraction (OUT) the median-multiplier rule of "Hurwitz
// Quaternion Multiplicative Quantization for KV Cache Compression" (Method 3)
// runs first on each vector (K after the rotation, V): the chunk it picks is
// stored in fp16 in the block's outlier section, and the group codec above
// runs on the remaining channels.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

// Median-multiplier chunk choice over one vector held by a warp (lane l holds
// channels [l*E, l*E + E), E = D/32; a chunk is 4 channels, so E = 4 gives a
// chunk per lane and E = 2 a chunk per lane pair).  Chunk norm
// sqrt((x0*x0 + x1*x1) + (x2*x2 + x3*x3)), each operation rounded once; the
// median of the D/4 norms is 0.5 * (a + b) of the two middle ones; the chunk
// with the largest norm above 3 * median is returned (ties: the lower index),
// or -1 if there is none or a norm is NaN.  Same value in every lane.
template <int D>
__device__ __forceinline__ int med3_chunk_warp(const float (&x)[D / 32], int lane) {
  constexpr int E = D / 32;
  constexpr int LPC = 4 / E;           // lanes per chunk
  constexpr int NC = D / 4;            // chunks
  static_assert(E == 2 || E == 4, "4-channel chunks need 2 or 4 channels per lane");
  float r;
  if constexpr (E == 4) {
    r = __fsqrt_rn(__fadd_rn(__fadd_rn(__fmul_rn(x[0], x[0]), __fmul_rn(x[1], x[1])),
                             __fadd_rn(__fmul_rn(x[2], x[2]), __fmul_rn(x[3], x[3]))));
  } else {
    const float p = __fadd_rn(__fmul_rn(x[0], x[0]), __fmul_rn(x[1], x[1]));
    const float o = __shfl_xor_sync(0xffffffffu, p, 1);
    r = __fsqrt_rn(__fadd_rn(p, o));   // (x0^2 + x1^2) + (x2^2 + x3^2): addition commutes
  }
  if (__any_sync(0xffffffffu, isnan(r))) return -1;
  // rank of this lane's chunk in ascending order (equal norms by chunk index)
  const int c = lane / LPC;
  int rank = 0;
#pragma unroll 8
  for (int j = 0; j < NC; ++j) {
    const float rj = __shfl_sync(0xffffffffu, r, j * LPC);
    rank += (rj < r) || (rj == r && j < c);
  }
  const bool leader = lane % LPC == 0;
  const unsigned lo_l = __ballot_sync(0xffffffffu, leader && rank == NC / 2 - 1);
  const unsigned hi_l = __ballot_sync(0xffffffffu, leader && rank == NC / 2);
  const float a = __shfl_sync(0xffffffffu, r, __ffs(lo_l) - 1);
  const float b = __shfl_sync(0xffffffffu, r, __ffs(hi_l) - 1);
  const float thr = __fmul_rn(3.0f, __fmul_rn(0.5f, __fadd_rn(a, b)));
  float best = r > thr ? r : -1.0f;   // norms are >= 0
#pragma unroll
  for (int o = 1; o < 32; o *= 2) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
  if (best < 0.0f) return -1;
  const unsigned who = __ballot_sync(0xffffffffu, r > thr && r == best);
  return (__ffs(who) - 1) / LPC;
}

// Writes the token's codes and metadata into slot `slot` of block `blk` and
// raises *eta_slot.  xk, xv: the token's k and v (fp32, this lane's channels);
// xk is rotated in place when `signs` is not NULL.  Returns, in every lane,
// the value the token contributes to eta (its max value error, one ulp up).
template <int D, int KB, int KG, bool OUT = false>
__device__ __forceinline__ float quantize_token_warp(float (&xk)[D / 32], float (&xv)[D / 32],
                                                    uint8_t* blk, int slot, float* eta_slot,
                                                    const int8_t* signs, float rot_c,
                                                    int32_t* err_word, int lane) {
  constexpr int E = D / 32;             // channels per lane
  constexpr int NB = D / 32;            // 32-channel blocks
  constexpr int Q = KB == 8 ? 127 : 7;
  constexpr int LPG_K = KG / E;         // lanes per key group
  constexpr int LPG_V = 32 / E;         // lanes per value group
  const BlockLayout L{D, KB, KG, OUT ? 1 : 0};
  if (signs) warp_rotate<E>(xk, signs, lane, rot_c);

  // ---------------- outlier chunks (OUT): fp16 copies, taken out of the codec --
  int ck = -1, cv = -1;
  float out_err = 0.0f;   // fp16 rounding error of this lane's extracted values
  bool in_ck = false, in_cv = false;
  if constexpr (OUT) {
    ck = med3_chunk_warp<D>(xk, lane);
    cv = med3_chunk_warp<D>(xv, lane);
    constexpr int LPC = 4 / E;
    in_ck = ck >= 0 && lane / LPC == ck;
    in_cv = cv >= 0 && lane / LPC == cv;
    uint8_t* os = blk + L.out_off();
    __half hk[E], hv[E];
    bool bad = false;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      hk[e] = __float2half_rn(0.0f);
      hv[e] = __float2half_rn(0.0f);
      if (in_ck) {
        if (!isfinite(xk[e]) || fabsf(xk[e]) > 65504.0f) bad = true;
        else hk[e] = __float2half_rn(xk[e]);
        xk[e] = 0.0f;   // zero leaves the group's max |x| as the kept channels make it
      }
      if (in_cv) {
        if (!isfinite(xv[e]) || fabsf(xv[e]) > 65504.0f) {
          bad = true;
        } else {
          hv[e] = __float2half_rn(xv[e]);
          out_err = fmaxf(out_err, fabsf(__fsub_rn(xv[e], __half2float(hv[e]))));
        }
      }
    }
    if (bad) set_error(err_word, KVQ_ERR_RANGE);
    // chunk indices; the chunk values (zeros when nothing was extracted)
    if (lane == 0) {
      os[slot] = ck < 0 ? kNoOutlier : (uint8_t)ck;
      os[kPage + slot] = cv < 0 ? kNoOutlier : (uint8_t)cv;
    }
    uint8_t* k16 = os + 2 * kPage + slot * 8;
    uint8_t* v16 = os + 2 * kPage + kPage * 8 + slot * 8;
    const int part = (lane % LPC) * E * 2;   // byte offset of this lane's channels
    if (in_ck || (ck < 0 && lane < LPC)) {
      if constexpr (E == 4)
        *reinterpret_cast<uint2*>(k16) = make_uint2(h2_as_u32(__halves2half2(hk[0], hk[1])),
                                                    h2_as_u32(__halves2half2(hk[2], hk[3])));
      else
        *reinterpret_cast<uint32_t*>(k16 + part) = h2_as_u32(__halves2half2(hk[0], hk[1]));
    }
    if (in_cv || (cv < 0 && lane < LPC)) {
      if constexpr (E == 4)
        *reinterpret_cast<uint2*>(v16) = make_uint2(h2_as_u32(__halves2half2(hv[0], hv[1])),
                                                    h2_as_u32(__halves2half2(hv[2], hv[3])));
      else
        *reinterpret_cast<uint32_t*>(v16 + part) = h2_as_u32(__halves2half2(hv[0], hv[1]));
    }
    // V: the extracted channels take the value of the group's first kept
    // channel (channel 0 of the group, or channel 4 when the chunk opens the
    // group), which changes neither its min, its max nor its largest error;
    // their codes are set to 0 below
    if (cv >= 0) {
      const bool opens = (4 * cv) % 32 == 0;
      const int src = (lane / LPG_V) * LPG_V + (opens ? 4 / E : 0);
      const float fill = __shfl_sync(0xffffffffu, xv[0], src);
      if (in_cv) {
#pragma unroll
        for (int e = 0; e < E; ++e) xv[e] = fill;
      }
    }
  }

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
      code[e] = in_cv ? 0 : (int)r;
      const float vh = __fmaf_rn(r, sc, z);
      err = fmaxf(err, fabsf(__fsub_rn(xv[e], vh)));
    }
    if (bad) err = 0.0f;
    err = fmaxf(err, out_err);
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
