// adaptive.cu -- adaptive precision and the first rungs of the fallback ladder
// ("Runtime-Certified Bounded-Error Quantized Attention", Methodology 3):
// a light scoring pass with the quantized keys estimates each block's
// attention mass; per query row the top-K* blocks covering tau_cov of that
// mass take full-precision keys from Tier 2; blocks whose estimated share of
// the value error (mass x eta) exceeds v_tol take full-precision values; the
// row's output and certified bound are recomputed; the ranking-consistency
// check compares the order of the key-promoted blocks by estimated mass with
// their order by exact mass and flags the row when they disagree.
//
// A block is one 16-token page of one kv head.  Only rows the decode flagged
// run through here, so these kernels favour plainness over speed:
//   adaptive_select_kernel   one CTA per flagged (sequence, kv head): the
//                            quantized scores of every token (lanes = tokens),
//                            block log-masses, value selection, a bitonic sort
//                            by mass (ties by lower page) and K* by a prefix
//                            sum; the union of promoted pages goes to the host,
//                            which pages in only those.
//   adaptive_correct_kernel  one CTA per (unit, page range): per token and
//                            row the exact or the quantized score and value,
//                            the online softmax, the bound's sums, the exact
//                            log-mass of every key-promoted page.
//   adaptive_finish_kernel   per unit: merge the page ranges, the bound,
//                            the ranking check, out / bound / flags.
#include "kvq_internal.cuh"

namespace kvq {

constexpr int kAdThreads = 256;
constexpr int kAdWarps = kAdThreads / 32;

// ---- one channel of one token row of a packed block (the documented layout) ----
template <int D, int KB>
__device__ __forceinline__ int ad_key_code(const uint8_t* blk, int slot, int c) {
  constexpr int NB = D / 32;
  const int b = c / 32, w = c % 32, s = w / 8, i = w % 8;
  if constexpr (KB == 8) {
    int p = s * 8 * NB + 8 * b + i;
    if constexpr (D == 128) p = (((p >> 4) ^ (slot & 7)) << 4) | (p & 15);
    return (int)(int8_t)__ldg(blk + slot * D + p);
  } else {
    const int p = s * 4 * NB + 4 * b + i / 2;
    const unsigned byte = __ldg(blk + slot * (D / 2) + p);
    const unsigned nib = (c & 1) ? (byte >> 4) : (byte & 15u);
    return nib >= 8 ? (int)nib - 16 : (int)nib;
  }
}
template <int D>
__device__ __forceinline__ int ad_val_code(const uint8_t* vrow, int c) {
  constexpr int NB = D / 32;
  const int g = c / 32, w = c % 32;
  const unsigned byte = __ldg(vrow + (w / 4) * 2 * NB + 2 * g + (w % 4) / 2);
  return (c & 1) ? (int)(byte >> 4) : (int)(byte & 15u);
}
__device__ __forceinline__ float ad_half(const uint8_t* p) {
  return __half2float(*reinterpret_cast<const __half*>(p));
}

int adaptive_select_smem(int max_pages, int d) {
  int npow = 1;
  while (npow < max_pages) npow <<= 1;
  return 4 * d * 4 + 4 * max_pages * 4 + npow * 8 + ((max_pages + 15) / 16) * 16 + 64;
}

// ------------------------------------------------------------------------------------
template <int D, int KB, int KG>
__global__ void __launch_bounds__(kAdThreads) adaptive_select_kernel(const __grid_constant__ AdArgs a) {
  constexpr int E = D / 32, NGK = D / KG;
  const BlockLayout L{D, KB, KG, a.outliers};
  extern __shared__ __align__(16) uint8_t smem[];
  const AdUnit u = a.units[blockIdx.x];
  const int R = u.nrows, mp = a.max_pages;
  int npow = 1;
  while (npow < mp) npow <<= 1;
  float* qs = reinterpret_cast<float*>(smem);                            // [4][D]
  float* lse = qs + 4 * D;                                                // [4][mp]
  unsigned long long* key = reinterpret_cast<unsigned long long*>(
      smem + ((4 * D + 4 * mp) * 4 + 7) / 8 * 8);                         // [npow]
  uint8_t* uni = reinterpret_cast<uint8_t*>(key + npow);                  // [mp]
  __shared__ float red[kAdWarps];
  __shared__ int s_kstar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int n = a.seq_lens[u.seq];
  n = max(0, min(n, mp * kPage));
  const int npg = (n + kPage - 1) / kPage;
  // the flagged rows' queries (rotated like the keys when the cache is)
  if (warp < 4) {
    float x[E];
    const int64_t row = warp < R ? u.rows[warp] : 0;
#pragma unroll
    for (int e = 0; e < E; ++e)
      x[e] = warp < R ? load_elem(a.q, a.q_bf16, row * D + lane * E + e) : 0.f;
    if (a.signs) warp_rotate<E>(x, a.signs, lane, a.rot_c);
#pragma unroll
    for (int e = 0; e < E; ++e) qs[warp * D + lane * E + e] = x[e];
  }
  for (int i = tid; i < mp; i += kAdThreads) uni[i] = 0;
  __syncthreads();

  // ---- scoring pass: lane = (page of the pair, token slot) -----------------------
  const int32_t* ptab = a.page_table + (int64_t)u.seq * mp;
  for (int pp = 2 * warp; pp < npg; pp += 2 * kAdWarps) {
    const int lp = pp + (lane >> 4), slot = lane & 15;
    const int tok = lp * kPage + slot;
    const bool in = lp < npg && tok < n;
    const int page = lp < npg ? __ldg(ptab + lp) : -1;
    const bool ok = in && page >= 0 && page < a.num_pages;
    if (in && !ok) set_error(a.err, KVQ_ERR_INVALID_ARG);
    float z[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    if (ok) {
      const uint8_t* blk = a.pool + ((int64_t)page * a.hkv + u.kvh) * L.bytes();
      float dot[4] = {0.f, 0.f, 0.f, 0.f};
      for (int g = 0; g < NGK; ++g) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int c = g * KG; c < (g + 1) * KG; ++c) {
          const float code = (float)ad_key_code<D, KB>(blk, slot, c);
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[r] = fmaf(qs[r * D + c], code, acc[r]);
        }
        const float sk = ad_half(blk + L.ks_off() + (slot * NGK + g) * 2);
#pragma unroll
        for (int r = 0; r < 4; ++r) dot[r] = fmaf(acc[r], sk, dot[r]);
      }
      if (a.outliers) {   // an extracted key chunk: its fp16 values (its codes are 0)
        const uint8_t* os = blk + L.out_off();
        const int ck = os[slot];
        if (ck < D / 4) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float kv = ad_half(os + 2 * kPage + slot * 8 + 2 * i);
#pragma unroll
            for (int r = 0; r < 4; ++r) dot[r] = fmaf(qs[r * D + 4 * ck + i], kv, dot[r]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) z[r] = a.s_att * dot[r];
    }
    // log-mass of each page: the half-warp of its 16 tokens
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float m = z[r];
#pragma unroll
      for (int o = 1; o < 16; o *= 2) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float s = m == -INFINITY ? 0.f : expf(z[r] - m);
#pragma unroll
      for (int o = 1; o < 16; o *= 2) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (slot == 0 && lp < npg && r < R) lse[r * mp + lp] = m == -INFINITY ? -INFINITY : m + logf(s);
    }
  }
  __syncthreads();

  // ---- per row: masses, value selection, order, K* ----------------------------------
  for (int r = 0; r < R; ++r) {
    const int rs = u.rslot + r;
    float* lr = lse + r * mp;
    // the row's log-normalizer over its pages
    float m = -INFINITY;
    for (int b = tid; b < npg; b += kAdThreads) m = fmaxf(m, lr[b]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < kAdWarps; ++w) m = fmaxf(m, red[w]);
    __syncthreads();
    float s = 0.f;
    for (int b = tid; b < npg; b += kAdThreads) s += lr[b] == -INFINITY ? 0.f : expf(lr[b] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[warp] = s;
    __syncthreads();
    s = 0.f;
#pragma unroll
    for (int w = 0; w < kAdWarps; ++w) s += red[w];
    const float lnorm = m == -INFINITY ? 0.f : m + logf(s);
    // masses; value promotion on them; sort keys (mass descending, page ascending)
    int nv = 0;
    for (int b = tid; b < npow; b += kAdThreads) {
      if (b < npg) {
        const float mass = lr[b] == -INFINITY ? 0.f : expf(lr[b] - lnorm);
        const int page = __ldg(ptab + b);
        const float eta = page >= 0 && page < a.num_pages
                              ? __ldg(a.eta + (int64_t)page * a.hkv + u.kvh) : 0.f;
        const bool vprom = mass * eta > a.v_tol;
        a.vp[(int64_t)rs * mp + b] = vprom ? 1 : 0;
        a.kp[(int64_t)rs * mp + b] = 0;
        if (vprom) uni[b] = 1;
        nv += vprom;
        key[b] = ((unsigned long long)(~__float_as_uint(mass)) << 32) | (unsigned)b;
      } else {
        key[b] = ~0ull;
        if (b < mp) {
          a.vp[(int64_t)rs * mp + b] = 0;
          a.kp[(int64_t)rs * mp + b] = 0;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, o);
    __syncthreads();
    if (lane == 0) red[warp] = __int_as_float(nv);
    // bitonic sort of the keys, ascending
    for (int k = 2; k <= npow; k <<= 1)
      for (int j = k >> 1; j > 0; j >>= 1) {
        __syncthreads();
        for (int i = tid; i < npow; i += kAdThreads) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const unsigned long long x = key[i], y = key[ixj];
            if ((x > y) == ((i & k) == 0)) {
              key[i] = y;
              key[ixj] = x;
            }
          }
        }
      }
    __syncthreads();
    // K*: the fewest leading blocks whose mass reaches tau_cov (fp32 running sum)
    if (warp == 0) {
      int kstar = a.tau_cov <= 0.f ? 0 : npg;
      float total = 0.f;
      for (int base = 0; a.tau_cov > 0.f && base < npg; base += 32) {
        const int k = base + lane;
        float x = k < npg ? __uint_as_float(~(unsigned)(key[k] >> 32)) : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o *= 2) {
          const float y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, k < npg && total + x >= a.tau_cov);
        if (hit) {
          kstar = base + __ffs(hit);
          break;
        }
        total += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) {
        s_kstar = kstar;
        int nvt = 0;
        for (int w = 0; w < kAdWarps; ++w) nvt += __float_as_int(red[w]);
        a.nkey[rs] = kstar;
        a.nval[rs] = nvt;
      }
    }
    __syncthreads();
    const int kstar = s_kstar;
    for (int k = tid; k < kstar; k += kAdThreads) {
      const int b = (int)(key[k] & 0xffffffffu);
      a.kp[(int64_t)rs * mp + b] = 1;
      a.korder[(int64_t)rs * mp + k] = b;
      uni[b] = 1;
    }
    __syncthreads();
  }
  for (int b = tid; b < mp; b += kAdThreads) a.um[(int64_t)blockIdx.x * mp + b] = uni[b];
}

// ------------------------------------------------------------------------------------
// Per item record in a.part: per row r < 4 [m, l, A, B, E, max Delta, 0, 0, o[D]],
// then the item's value range per 32-channel group [top max][zero min] and max eta.
template <int D, int KB, int KG>
__global__ void __launch_bounds__(kAdThreads) adaptive_correct_kernel(const __grid_constant__ AdArgs a) {
  constexpr int E = D / 32, NGK = D / KG, NB = D / 32;
  constexpr int Q = KB == 8 ? 127 : 7;
  constexpr int LPC = 4 / E;   // lanes per 4-channel chunk
  const BlockLayout L{D, KB, KG, a.outliers};
  const AdItem it = a.items[blockIdx.x];
  const AdUnit u = a.units[it.unit];
  const int R = u.nrows, mp = a.max_pages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int n = a.seq_lens[u.seq];
  n = max(0, min(n, mp * kPage));
  const int es = a.kv_bf16 ? 2 : 4;

  // queries: original (exact scores) and rotated (scores on the codes); row constants
  float q0[4][E], qr[4][E], cg[4][NGK], cb[4], ce[4], cr[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t row = r < R ? u.rows[r] : 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      q0[r][e] = r < R ? load_elem(a.q, a.q_bf16, row * D + lane * E + e) : 0.f;
      qr[r][e] = q0[r][e];
    }
    if (a.signs) warp_rotate<E>(qr[r], a.signs, lane, a.rot_c);
    float n0 = 0.f, n2 = 0.f, l1[NGK];
#pragma unroll
    for (int g = 0; g < NGK; ++g) l1[g] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      n0 = fmaf(q0[r][e], q0[r][e], n0);
      n2 = fmaf(qr[r][e], qr[r][e], n2);
      l1[(lane * E + e) / KG] += fabsf(qr[r][e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n0 += __shfl_xor_sync(0xffffffffu, n0, o);
      n2 += __shfl_xor_sync(0xffffffffu, n2, o);
#pragma unroll
      for (int g = 0; g < NGK; ++g) l1[g] += __shfl_xor_sync(0xffffffffu, l1[g], o);
    }
#pragma unroll
    for (int g = 0; g < NGK; ++g) cg[r][g] = kKappa * a.s_att * 0.5f * l1[g];
    cb[r] = a.signs ? kKappa * a.s_att * kRotSlack * sqrtf((float)D) * (float)Q * sqrtf(n2) : 0.f;
    ce[r] = kKappa * a.s_att * kRotSlack * sqrtf(n0);
    cr[r] = a.signs ? kKappa * a.s_att * kRotSlack * sqrtf(n2) : 0.f;
  }

  float m[4], l[4], A[4], Bs[4], Ev[4], dmax[4], o[4][E];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m[r] = -INFINITY;
    l[r] = A[r] = Bs[r] = Ev[r] = dmax[r] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[r][e] = 0.f;
  }
  const int g_lane = (lane * E) / 32;          // this lane's value group
  float vtop = -INFINITY, vzmin = INFINITY, etamax = 0.f;
  const int32_t* ptab = a.page_table + (int64_t)u.seq * mp;
  const int32_t* smap = a.smap + (int64_t)it.unit * mp;
  const uint8_t* stK = a.staging + u.stage_off;
  const uint8_t* stV = stK + (int64_t)u.nstaged * kPage * D * es;

  for (int lp = it.p0 + warp; lp < it.p1; lp += kAdWarps) {
    const int page = __ldg(ptab + lp);
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
      etamax = INFINITY;   // no certified bound for this unit
      continue;
    }
    const uint8_t* blk = a.pool + ((int64_t)page * a.hkv + u.kvh) * L.bytes();
    const float eta = __ldg(a.eta + (int64_t)page * a.hkv + u.kvh);
    etamax = fmaxf(etamax, eta);
    bool kpr[4], vpr[4];
    bool anyk = false, anyv = false;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      kpr[r] = r < R && a.kp[(int64_t)(u.rslot + r) * mp + lp] != 0;
      vpr[r] = r < R && a.vp[(int64_t)(u.rslot + r) * mp + lp] != 0;
      anyk |= kpr[r];
      anyv |= vpr[r];
    }
    const int si = smap[lp];
    if ((anyk || anyv) && si < 0) {   // a promoted page that was not staged
      if (lane == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
      etamax = INFINITY;
      continue;
    }
    float pm[4], pl[4];   // this page's exact log-mass trackers
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      pm[r] = -INFINITY;
      pl[r] = 0.f;
    }
    const int ntok = min(kPage, n - lp * kPage);
    for (int slot = 0; slot < ntok; ++slot) {
      // quantized key and value of this lane's channels; the token's key scales
      float kh[E], vh[E], ks[NGK];
      float smax = 0.f;
#pragma unroll
      for (int g = 0; g < NGK; ++g) {
        ks[g] = ad_half(blk + L.ks_off() + (slot * NGK + g) * 2);
        smax = fmaxf(smax, ks[g]);
      }
      const float sv = ad_half(blk + L.vm_off() + (slot * NB + g_lane) * 4);
      const float zv = ad_half(blk + L.vm_off() + (slot * NB + g_lane) * 4 + 2);
      vtop = fmaxf(vtop, __fmaf_rn(15.0f, sv, zv));
      vzmin = fminf(vzmin, zv);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int c = lane * E + e;
        kh[e] = ks[c / KG] * (float)ad_key_code<D, KB>(blk, slot, c);
        vh[e] = __fmaf_rn((float)ad_val_code<D>(blk + L.v_off() + slot * (D / 2), c), sv, zv);
      }
      // extracted chunks (their codes are 0): the fp16 values; the key chunk's
      // share of Delta per row, summed by the chunk's lanes and broadcast
      int ck = kNoOutlier;
      float dlo[4] = {0.f, 0.f, 0.f, 0.f};
      if (a.outliers) {
        const uint8_t* os = blk + L.out_off();
        ck = os[slot];
        const int cv = os[kPage + slot];
        const int part = (lane % LPC) * E;   // this lane's first channel in its chunk
        if (cv < D / 4 && lane / LPC == cv) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            vh[e] = ad_half(os + 2 * kPage + kPage * 8 + slot * 8 + 2 * (part + e));
            vtop = fmaxf(vtop, vh[e]);
            vzmin = fminf(vzmin, vh[e]);
          }
        }
        if (ck < D / 4) {
          float u[4] = {0.f, 0.f, 0.f, 0.f}, kn = 0.f;
          if (lane / LPC == ck) {
#pragma unroll
            for (int e = 0; e < E; ++e) {
              kh[e] = ad_half(os + 2 * kPage + slot * 8 + 2 * (part + e));
              kn = fmaf(kh[e], kh[e], kn);
#pragma unroll
              for (int r = 0; r < 4; ++r)
                u[r] = fmaf(fabsf(qr[r][e]), fmaf(fabsf(kh[e]), 0x1p-11f, 0x1p-25f), u[r]);
            }
          }
#pragma unroll
          for (int o2 = 1; o2 < LPC; o2 *= 2) {
            kn += __shfl_xor_sync(0xffffffffu, kn, o2);
#pragma unroll
            for (int r = 0; r < 4; ++r) u[r] += __shfl_xor_sync(0xffffffffu, u[r], o2);
          }
          kn = __shfl_sync(0xffffffffu, kn, ck * LPC);
#pragma unroll
          for (int r = 0; r < 4; ++r)
            dlo[r] = fmaf(kKappa * a.s_att, __shfl_sync(0xffffffffu, u[r], ck * LPC),
                          cr[r] * sqrtf(kn));
        }
      }
      // originals of a promoted page
      float kx[E], vx[E], kn2 = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) kx[e] = vx[e] = 0.f;
      if (anyk || anyv) {
        const int64_t off = ((int64_t)si * kPage + slot) * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if (anyk) kx[e] = load_elem(stK, a.kv_bf16, off + e);
          if (anyv) vx[e] = load_elem(stV, a.kv_bf16, off + e);
          kn2 = fmaf(kx[e], kx[e], kn2);
        }
#pragma unroll
        for (int off2 = 16; off2 > 0; off2 >>= 1) kn2 += __shfl_xor_sync(0xffffffffu, kn2, off2);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (r >= R) break;
        float sdot = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) sdot = kpr[r] ? fmaf(q0[r][e], kx[e], sdot) : fmaf(qr[r][e], kh[e], sdot);
#pragma unroll
        for (int off2 = 16; off2 > 0; off2 >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, off2);
        const float z = a.s_att * sdot;
        float dl;
        if (kpr[r]) {
          dl = ce[r] * sqrtf(kn2);
        } else {
          dl = cb[r] * smax + dlo[r];
#pragma unroll
          for (int g = 0; g < NGK; ++g) dl = fmaf(cg[r][g], ks[g], dl);
        }
        const float mn = fmaxf(m[r], z);
        const float sc = m[r] == -INFINITY ? 0.f : expf(m[r] - mn);
        const float p = expf(z - mn);
        m[r] = mn;
        l[r] = fmaf(l[r], sc, p);
        A[r] = fmaf(A[r], sc, p * expm1f(dl));
        Bs[r] = fmaf(Bs[r], sc, p * expf(-dl));
        Ev[r] = fmaf(Ev[r], sc, vpr[r] ? 0.f : p * eta);
        dmax[r] = fmaxf(dmax[r], dl);
#pragma unroll
        for (int e = 0; e < E; ++e) o[r][e] = fmaf(o[r][e], sc, p * (vpr[r] ? vx[e] : vh[e]));
        if (kpr[r]) {
          const float pn = fmaxf(pm[r], z);
          pl[r] = (pm[r] == -INFINITY ? 0.f : pl[r] * expf(pm[r] - pn)) + expf(z - pn);
          pm[r] = pn;
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (kpr[r]) a.blse[(int64_t)(u.rslot + r) * mp + lp] = pm[r] + logf(pl[r]);
    }
  }

  // ---- merge the warps into the item's record ----------------------------------------
  // value range: lanes of one value group, then warps
#pragma unroll
  for (int off2 = 1; off2 < 32 / E; off2 *= 2) {
    vtop = fmaxf(vtop, __shfl_xor_sync(0xffffffffu, vtop, off2));
    vzmin = fminf(vzmin, __shfl_xor_sync(0xffffffffu, vzmin, off2));
  }
  etamax = fmaxf(etamax, __shfl_xor_sync(0xffffffffu, etamax, 16));
  __shared__ float s_st[kAdWarps][4][6];
  __shared__ float s_o[kAdWarps][4][D];
  __shared__ float s_rg[kAdWarps][2 * NB + 1];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if (lane == 0) {
      s_st[warp][r][0] = m[r];
      s_st[warp][r][1] = l[r];
      s_st[warp][r][2] = A[r];
      s_st[warp][r][3] = Bs[r];
      s_st[warp][r][4] = Ev[r];
      s_st[warp][r][5] = dmax[r];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) s_o[warp][r][lane * E + e] = o[r][e];
  }
  if (lane % (32 / E) == 0) {
    s_rg[warp][g_lane] = vtop;
    s_rg[warp][NB + g_lane] = vzmin;
  }
  if (lane == 0) s_rg[warp][2 * NB] = etamax;
  __syncthreads();
  const size_t PF = adaptive_part_floats(D);
  float* rec = a.part + (size_t)blockIdx.x * PF;
  for (int idx = tid; idx < 4 * (D + 8); idx += kAdThreads) {
    const int r = idx / (D + 8), c = idx % (D + 8);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAdWarps; ++w) M = fmaxf(M, s_st[w][r][0]);
    float acc = 0.f;
    if (c == 0) {
      acc = M;
    } else if (c == 5) {
#pragma unroll
      for (int w = 0; w < kAdWarps; ++w) acc = fmaxf(acc, s_st[w][r][5]);
    } else if (c < 8) {
      if (c < 5) {
#pragma unroll
        for (int w = 0; w < kAdWarps; ++w)
          if (s_st[w][r][0] != -INFINITY) acc = fmaf(s_st[w][r][c], expf(s_st[w][r][0] - M), acc);
      }
    } else {
#pragma unroll
      for (int w = 0; w < kAdWarps; ++w)
        if (s_st[w][r][0] != -INFINITY) acc = fmaf(s_o[w][r][c - 8], expf(s_st[w][r][0] - M), acc);
    }
    rec[idx] = acc;
  }
  if (tid < 2 * NB + 1) {
    float v = tid < NB ? -INFINITY : (tid < 2 * NB ? INFINITY : 0.f);
#pragma unroll
    for (int w = 0; w < kAdWarps; ++w)
      v = tid < NB ? fmaxf(v, s_rg[w][tid]) : (tid < 2 * NB ? fminf(v, s_rg[w][tid]) : fmaxf(v, s_rg[w][tid]));
    rec[4 * (D + 8) + tid] = v;
  }
}

// ------------------------------------------------------------------------------------
// One CTA (4 warps) per unit; warp r finishes row r.
template <int D>
__global__ void __launch_bounds__(128) adaptive_finish_kernel(const __grid_constant__ AdArgs a) {
  constexpr int E = D / 32, NB = D / 32;
  const AdUnit u = a.units[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= u.nrows) return;
  const int r = warp, rs = u.rslot + r, mp = a.max_pages;
  const int64_t row = u.rows[r];
  // the unit's items are consecutive, starting at the one whose `first` is itself
  int i0 = -1, ni = 0;
  for (int i = 0; i < a.num_items; ++i)
    if (a.items[i].unit == (int)blockIdx.x) {
      if (i0 < 0) i0 = i;
      ++ni;
    }
  const size_t PF = adaptive_part_floats(D);
  float M = -INFINITY;
  for (int i = 0; i < ni; ++i) M = fmaxf(M, a.part[(size_t)(i0 + i) * PF + r * (D + 8)]);
  float t[4] = {0.f, 0.f, 0.f, 0.f}, dm = 0.f, ov[E];
#pragma unroll
  for (int e = 0; e < E; ++e) ov[e] = 0.f;
  float top[NB], zmin[NB], etamax = 0.f;
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    top[g] = -INFINITY;
    zmin[g] = INFINITY;
  }
  for (int i = 0; i < ni; ++i) {
    const float* rec = a.part + (size_t)(i0 + i) * PF;
    const float* st = rec + r * (D + 8);
    dm = fmaxf(dm, st[5]);
    if (st[0] != -INFINITY) {
      const float f = expf(st[0] - M);
#pragma unroll
      for (int k = 0; k < 4; ++k) t[k] = fmaf(st[1 + k], f, t[k]);
#pragma unroll
      for (int e = 0; e < E; ++e) ov[e] = fmaf(st[8 + lane * E + e], f, ov[e]);
    }
    const float* rg = rec + 4 * (D + 8);
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      top[g] = fmaxf(top[g], rg[g]);
      zmin[g] = fminf(zmin[g], rg[NB + g]);
    }
    etamax = fmaxf(etamax, rg[2 * NB]);
  }
  const float lsum = t[0];
#pragma unroll
  for (int e = 0; e < E; ++e) a.out[row * D + lane * E + e] = lsum > 0.f ? ov[e] / lsum : 0.f;
  if (lane == 0) {
    const bool skipped = etamax == INFINITY;
    float bd = skipped ? INFINITY : 0.f;
    if (!skipped && lsum > 0.f) {
      float range = 0.f;
#pragma unroll
      for (int g = 0; g < NB; ++g) range = fmaxf(range, top[g] - zmin[g]);
      const float tv = fminf(tanhf(0.5f * dm), t[1] / t[2]);
      bd = kKappa * (tv * (range + 2.0f * etamax) + t[3] / lsum);
    }
    // ranking check: exact log-masses along the estimated order
    bool fail = false;
    float lmin = INFINITY;
    const int K = a.nkey[rs];
    for (int k = 0; k < K; ++k) {
      const float Lb = a.blse[(int64_t)rs * mp + a.korder[(int64_t)rs * mp + k]];
      if (Lb - lmin > a.rank_tol) fail = true;
      lmin = fminf(lmin, Lb);
    }
    a.bound[row] = bd;
    a.flags[row] = (skipped || fail || bd > a.tau) ? 1 : 0;
    a.rank_fail[rs] = fail ? 1 : 0;
  }
}

// ------------------------------------------------------------------------------------
template <int D, int KB, int KG>
cudaError_t select_launch(const AdArgs& a, int smem, cudaStream_t s) {
  auto k = adaptive_select_kernel<D, KB, KG>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k<<<a.num_units, kAdThreads, smem, s>>>(a);
  return cudaGetLastError();
}
template <int D, int KB, int KG>
cudaError_t correct_launch(const AdArgs& a, cudaStream_t s) {
  adaptive_correct_kernel<D, KB, KG><<<a.num_items, kAdThreads, 0, s>>>(a);
  return cudaGetLastError();
}

#define KVQ_AD_CASES(X)  \
  X(128, 8, 128)         \
  X(128, 8, 64)          \
  X(128, 8, 32)          \
  X(128, 4, 128)         \
  X(128, 4, 64)          \
  X(128, 4, 32)          \
  X(64, 8, 64)           \
  X(64, 8, 32)           \
  X(64, 4, 64)           \
  X(64, 4, 32)

cudaError_t launch_adaptive_select(const AdArgs& a, int d, int kbits, int kgroup, int smem,
                                   cudaStream_t s) {
  if (a.num_units <= 0) return cudaSuccess;
#define X(D_, KB_, KG_) \
  if (d == D_ && kbits == KB_ && kgroup == KG_) return select_launch<D_, KB_, KG_>(a, smem, s);
  KVQ_AD_CASES(X)
#undef X
  return cudaErrorInvalidValue;
}

cudaError_t launch_adaptive_correct(const AdArgs& a, int d, int kbits, int kgroup, cudaStream_t s) {
  if (a.num_items <= 0) return cudaSuccess;
#define X(D_, KB_, KG_) \
  if (d == D_ && kbits == KB_ && kgroup == KG_) return correct_launch<D_, KB_, KG_>(a, s);
  KVQ_AD_CASES(X)
#undef X
  return cudaErrorInvalidValue;
}

cudaError_t launch_adaptive_finish(const AdArgs& a, int d, cudaStream_t s) {
  if (a.num_units <= 0) return cudaSuccess;
  if (d == 128) adaptive_finish_kernel<128><<<a.num_units, 128, 0, s>>>(a);
  else if (d == 64) adaptive_finish_kernel<64><<<a.num_units, 128, 0, s>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace kvq
