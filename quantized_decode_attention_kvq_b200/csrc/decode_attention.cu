// decode_attention.cu -- fused split-K decode attention over the packed
// Tier-1 cache with the certified per-query error bound computed in the same
// pass ("Runtime-Certified Bounded-Error Quantized Attention", Methodology 2:
// E_key from the total-variation distance between exact and quantized
// softmax, bounded through the per-token score perturbation Delta; E_val from
// the block errors eta_b weighted by attention mass; both from scales, query
// norms and the value range only).
//
// Grid (split, kv head, sequence); 4 warps per CTA.  Each warp streams its
// own pages of the split through an S-stage ring in shared memory: one TMA
// tiled load brings the page's K codes (128B-swizzled when rows are 128 B),
// one bulk copy brings V codes + K scales + V scale/zero; completion on an
// mbarrier per stage, every wait bounded.
//
// Per page (16 tokens x up to 4 query rows of one GQA group):
//   QK^T  int8 tensor cores, exact: q' (rotated if the cache is) is held in
//         fixed point, q' * 2^F rounded to int32 and split into four signed
//         base-256 digits; codes x digits accumulate exactly in int32, the
//         digit sums are recombined in fp32 and scaled by the per-token
//         group scale.  (4-bit keys enter as code+8 with the bias folded
//         into the accumulator's initial value.)
//   softmax online, base 2, per query row.
//   bound  Delta_j = kappa*scale*(sum_g |q'_g|_1 sK_{j,g}/2 [+ rotation
//         allowance]); per row the running sums A = sum w (e^Delta - 1),
//         B = sum w e^-Delta, E = sum w eta_b, max Delta; per kv head the
//         value range [min z, max fmaf(15, s, z)] per group.
//   PV    fp16 tensor cores: V codes are exact in fp16; the per-token group
//         scale is folded into P' = w * sV (split hi + lo, both fp16, so the
//         product keeps ~22 bits) and the zero point is added as
//         sum_j w_j zV_{j,g} on CUDA cores.
// Warps merge in shared memory; splits merge in the last CTA of each
// (sequence, kv head) to finish: o = O/l, TV = min(tanh(maxDelta/2), A/B),
// E_key = TV*(range + 2 max eta), E_val = E/l, bound = kappa*(E_key+E_val),
// flag = bound > tau.
#include "kvq_internal.cuh"

namespace kvq {

constexpr int kWarps = 4;
constexpr int kRows = 4;  // query rows per kv head handled by one CTA
constexpr int kHdr = 16;  // floats of the per-split record header

__host__ __device__ constexpr int record_floats(int d) { return kHdr + kRows * (8 + d); }

template <int D, int KB, int KG, int S>
struct DecodeCfg {
  static constexpr int NB = D / 32;
  static constexpr int NGK = D / KG;
  static constexpr int KRB = D * KB / 8;          // K row bytes
  static constexpr int KT = kPage * KRB;          // K tile bytes
  static constexpr int VRB = D / 2;               // V row bytes
  static constexpr int VB = kPage * VRB;
  static constexpr int KSB = kPage * NGK * 2;
  static constexpr int VMB = kPage * NB * 4;
  static constexpr int REST = VB + KSB + VMB;     // bytes after the K codes
  static constexpr int BLOCK = KT + REST;
  static constexpr bool SWZ = KRB == 128;
  static constexpr int KSTR = KRB / 4;            // K stripe bytes per lane
  static constexpr int VSTR = VRB / 8;            // V stripe bytes per lane
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_KT = 0;
  static constexpr int SZ_KT = kWarps * S * KT;
  static constexpr int OFF_RS = OFF_KT + SZ_KT;
  static constexpr int SZ_RS = kWarps * S * REST;
  static constexpr int OFF_BAR = (OFF_RS + SZ_RS + 15) / 16 * 16;
  static constexpr int OFF_PG = OFF_BAR + kWarps * S * 8;
  static constexpr int OFF_Q = (OFF_PG + kWarps * S * 4 + 15) / 16 * 16;   // int qfix[4][D]
  static constexpr int OFF_QF = OFF_Q + kRows * D * 4;                      // float q'[4][D]
  static constexpr int OFF_RC = OFF_QF + kRows * D * 4;                     // row constants
  static constexpr int RC_FLOATS = kRows * (2 + NGK);                       // zs, cb, cg[NGK]
  static constexpr int OFF_FLAG = OFF_RC + RC_FLOATS * 4;
  static constexpr int END = OFF_FLAG + 16;
  // merge area (aliases the stage buffers once the page loop is over)
  static constexpr int MW_FLOATS = kRows * D + kRows * 8 + kRows * NB + 2 * NB + 1;
  static constexpr int MERGE_BYTES = (kWarps + 1) * MW_FLOATS * 4;
  static constexpr int SMEM = 1024 + (END > MERGE_BYTES ? END : MERGE_BYTES);
  static_assert(MERGE_BYTES <= OFF_BAR, "merge area must fit in the stage buffers");
};

__device__ __forceinline__ int q_digit(int v, int i) {
  int d0 = (int)(int8_t)(v & 0xFF);
  if (i == 0) return d0;
  v = (v - d0) >> 8;
  int d1 = (int)(int8_t)(v & 0xFF);
  if (i == 1) return d1;
  v = (v - d1) >> 8;
  int d2 = (int)(int8_t)(v & 0xFF);
  if (i == 2) return d2;
  return (v - d2) >> 8;
}

template <int D>
__device__ __forceinline__ void finalize_row(const DecodeArgs& a, int b, int kvh, int r,
                                             float l, float A, float B, float E, float dmax,
                                             float range, float etamax, const float* o_row,
                                             int c0, int cstep, bool write_stats) {
  if (r >= a.R) return;
  const int qi = r / a.G, h = kvh * a.G + r % a.G;
  const int64_t row = ((int64_t)b * a.nq + qi) * a.hq + h;
  if (a.out) {
    const float inv_l = l > 0.f ? 1.0f / l : 0.f;
    for (int c = c0; c < D; c += cstep) a.out[row * D + c] = o_row[c] * inv_l;
  }
  if (write_stats) {
    float bd = 0.f;
    if (l > 0.f) {
      const float tv = fminf(tanhf(0.5f * dmax), A / B);
      const float ekey = tv * (range + 2.0f * etamax);
      const float evl = E / l;
      bd = kKappa * (ekey + evl);
    }
    a.bound[row] = bd;
    a.flags[row] = bd > a.tau ? 1 : 0;
  }
}

template <int D, int KB, int KG, int S>
__global__ void __launch_bounds__(kWarps * 32, 3)
    decode_mma_kernel(const __grid_constant__ DecodeArgs a,
                      const __grid_constant__ CUtensorMap kmap) {
  using C = DecodeCfg<D, KB, KG, S>;
  constexpr int NB = C::NB, NGK = C::NGK;
  constexpr int Q = KB == 8 ? 127 : 7;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~(uintptr_t)1023);
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c4 = lane & 3, g8 = lane >> 2;

  int n = a.seq_lens[b];
  if (n < 0) n = 0;
  if (n > a.max_pages * kPage) {
    if (tid == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
    n = a.max_pages * kPage;
  }
  const int npages = (n + kPage - 1) / kPage;
  const int active = npages == 0 ? 1 : (npages + a.pps - 1) / a.pps;
  if (split >= active) return;
  if (npages == 0) {  // empty context: zero output, zero bound
    for (int r = 0; r < a.R; ++r) {
      const int qi = r / a.G, h = kvh * a.G + r % a.G;
      const int64_t row = ((int64_t)b * a.nq + qi) * a.hq + h;
      if (a.out)
        for (int c = tid; c < D; c += blockDim.x) a.out[row * D + c] = 0.f;
      if (tid == 0) {
        a.bound[row] = 0.f;
        a.flags[row] = 0;
      }
    }
    return;
  }
  const int p0 = split * a.pps;
  const int p1 = min(p0 + a.pps, npages);

  uint8_t* ktile = sm + C::OFF_KT + warp * S * C::KT;
  uint8_t* rest = sm + C::OFF_RS + warp * S * C::REST;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR) + warp * S;
  int* spage = reinterpret_cast<int*>(sm + C::OFF_PG) + warp * S;
  int* qfix = reinterpret_cast<int*>(sm + C::OFF_Q);
  float* qf = reinterpret_cast<float*>(sm + C::OFF_QF);
  float* rc = reinterpret_cast<float*>(sm + C::OFF_RC);

  // ---- pipeline start: page indices, barriers, first S copies --------------
  const int first = p0 + warp;
  const int nloc = first < p1 ? (p1 - first + kWarps - 1) / kWarps : 0;
  const int32_t* ptab = a.page_table + (int64_t)b * a.max_pages;
  auto fetch_chunk = [&](int c) -> int {
    const int j = c * 32 + lane;
    return j < nloc ? __ldg(ptab + first + j * kWarps) : -1;
  };
  int pt_chunk = -1, pt_val = -1, pt_next = fetch_chunk(0);
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }
  if (tid == 0) prefetch_tensormap(&kmap);
  __syncwarp();

  auto issue = [&](int j) {  // whole warp calls; lane 0 issues the copies of local page j
    const int c = j >> 5;
    if (c != pt_chunk) {
      pt_val = (c == pt_chunk + 1) ? pt_next : fetch_chunk(c);
      pt_next = fetch_chunk(c + 1);
      pt_chunk = c;
    }
    const int page = __shfl_sync(0xffffffffu, pt_val, j & 31);
    const int st = j % S;
    if (lane == 0) {
      const bool ok = page >= 0 && page < a.num_pages;
      spage[st] = ok ? page : -1;
      if (ok) {
        const int64_t blk = (int64_t)page * a.hkv + kvh;
        mbar_arrive_expect_tx(&bar[st], C::BLOCK);
        tma_load_3d(ktile + st * C::KT, &kmap, 0, 0, (int)blk, &bar[st]);
        bulk_g2s(rest + st * C::REST, a.pool + blk * C::BLOCK + C::KT, C::REST, &bar[st]);
      } else {
        set_error(a.err, KVQ_ERR_INVALID_ARG);
        mbar_arrive(&bar[st]);
      }
    }
    __syncwarp();  // publish spage[st] to the warp
  };
  for (int j = 0; j < S && j < nloc; ++j) issue(j);

  // ---- query rows: load, rotate, fixed point, norms -------------------------
  for (int i = tid; i < kRows * D; i += blockDim.x) {
    const int r = i / D, c = i % D;
    float x = 0.f;
    if (r < a.R) {
      const int qi = r / a.G, h = kvh * a.G + r % a.G;
      const int64_t row = ((int64_t)b * a.nq + qi) * a.hq + h;
      x = load_elem(a.q, a.q_bf16, row * D + c);
    }
    qf[i] = x;
  }
  __syncthreads();
  if (warp < kRows) {
    const int r = warp;
    constexpr int E = D / 32;
    float x[E];
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = qf[r * D + lane * E + e];
    if (a.signs) warp_rotate<E>(x, a.signs, lane, a.rot_c);
    float am = 0.f, l2 = 0.f, l1[NGK];
#pragma unroll
    for (int g = 0; g < NGK; ++g) l1[g] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      am = fmaxf(am, fabsf(x[e]));
      l2 = fmaf(x[e], x[e], l2);
      l1[(lane * E + e) / KG] += fabsf(x[e]);
    }
#pragma unroll
    for (int o = 1; o < 32; o *= 2) {
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      l2 += __shfl_xor_sync(0xffffffffu, l2, o);
#pragma unroll
      for (int g = 0; g < NGK; ++g) l1[g] += __shfl_xor_sync(0xffffffffu, l1[g], o);
    }
    int ex = 0;
    if (am > 0.f) frexpf(am, &ex);
    int F = am > 0.f ? 30 - ex : 0;
    F = min(F, 100);
#pragma unroll
    for (int e = 0; e < E; ++e) qfix[r * D + lane * E + e] = __float2int_rn(ldexpf(x[e], F));
    if (lane == 0) {
      rc[r] = ldexpf(a.s_att * kLog2e, -F);                      // zs: score scale, log2 units
      rc[kRows + r] = a.signs ? kKappa * a.s_att * kRotSlack * sqrtf((float)D) * (float)Q *
                                    sqrtf(l2)
                              : 0.f;                               // cb
#pragma unroll
      for (int g = 0; g < NGK; ++g)
        rc[2 * kRows + r * NGK + g] = kKappa * a.s_att * 0.5f * l1[g];   // cg
    }
  }
  __syncthreads();

  // ---- per-lane constant fragments -------------------------------------------
  // B fragment of the QK^T MMA: column n = g8 <-> (row n/2, digit 2*nt + n%2);
  // k index (4*c4 + e | 16 + 4*c4 + e) <-> the lane's stripe channels.
  uint32_t qb[NB][2][2];
  {
    const int r = g8 >> 1, dl = g8 & 1;
#pragma unroll
    for (int ks = 0; ks < NB; ++ks)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int ch = KB == 8 ? 32 * ks + 8 * c4 + 4 * jj + e : 32 * ks + 8 * c4 + 2 * e + jj;
            const int dg = q_digit(qfix[r * D + ch], 2 * nt + dl);
            w |= (uint32_t)(dg & 0xFF) << (8 * e);
          }
          qb[ks][nt][jj] = w;
        }
  }
  // initial accumulators: 4-bit key codes enter as code + 8
  int cinit[NGK][2][2];
#pragma unroll
  for (int g = 0; g < NGK; ++g)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int dd = 0; dd < 2; ++dd) {
        int s = 0;
        if (KB == 4)
          for (int c = g * KG; c < (g + 1) * KG; ++c) s += q_digit(qfix[c4 * D + c], 2 * nt + dd);
        cinit[g][nt][dd] = -8 * s;
      }
  const float zs = rc[c4];
  const float cb = rc[kRows + c4];
  float cg[NGK];
#pragma unroll
  for (int g = 0; g < NGK; ++g) cg[g] = rc[2 * kRows + c4 * NGK + g];

  // ---- accumulators ------------------------------------------------------------
  float m2 = -INFINITY, lsum = 0.f, Asum = 0.f, Bsum = 0.f, Esum = 0.f, dmax = 0.f;
  float zacc[NB];
  float opv[2 * NB][4];
#pragma unroll
  for (int g = 0; g < NB; ++g) zacc[g] = 0.f;
#pragma unroll
  for (int t = 0; t < 2 * NB; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) opv[t][e] = 0.f;
  float vhi = -INFINITY, vlo = INFINITY, etamax = 0.f;
  const int hP = g8 & 3;
  const bool lo_part = g8 >= 4;

  const float* eta_kv = a.eta + kvh;
  float eta_next = 0.f;
  if (nloc > 0) {
    __syncwarp();
    const int pg = spage[0];
    eta_next = pg >= 0 ? __ldg(eta_kv + (int64_t)pg * a.hkv) : 0.f;
  }

  // ---- page loop ---------------------------------------------------------------
  for (int j = 0; j < nloc; ++j) {
    const int st = j % S;
    const uint32_t par = (uint32_t)((j / S) & 1);
    bool ok = mbar_wait(&bar[st], par);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) set_error(a.err, KVQ_ERR_TIMEOUT);
      break;
    }
    const int page = spage[st];
    const float eta_cur = eta_next;
    if (j + 1 < nloc) {
      const int pn = spage[(j + 1) % S];
      eta_next = pn >= 0 ? __ldg(eta_kv + (int64_t)pn * a.hkv) : 0.f;
    }
    if (page >= 0) {
      const uint8_t* kt = ktile + st * C::KT;
      const uint8_t* rs = rest + st * C::REST;
      const int tok0 = (first + j * kWarps) * kPage;
      const int nval = min(kPage, n - tok0);
      etamax = fmaxf(etamax, eta_cur);

      // --- K codes of rows g8, g8+8 (this lane's stripe) -> QK^T on int8 MMA ---
      constexpr int KW = C::KSTR / 4;    // 32-bit words per stripe
      uint32_t wk[2][KW];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int row = g8 + 8 * rr;
        if constexpr (C::KSTR >= 16) {
#pragma unroll
          for (int hh = 0; hh < C::KSTR / 16; ++hh) {
            int chunk = (c4 * C::KSTR) / 16 + hh;
            if (C::SWZ) chunk ^= (row & 7);
            const uint4 v4 = *reinterpret_cast<const uint4*>(kt + row * C::KRB + chunk * 16);
            wk[rr][4 * hh + 0] = v4.x;
            wk[rr][4 * hh + 1] = v4.y;
            wk[rr][4 * hh + 2] = v4.z;
            wk[rr][4 * hh + 3] = v4.w;
          }
        } else {
          const uint2 v2 = *reinterpret_cast<const uint2*>(kt + row * C::KRB + c4 * C::KSTR);
          wk[rr][0] = v2.x;
          wk[rr][1] = v2.y;
        }
      }
      int acc[NGK][2][4];
#pragma unroll
      for (int g = 0; g < NGK; ++g)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          acc[g][nt][0] = cinit[g][nt][0];
          acc[g][nt][1] = cinit[g][nt][1];
          acc[g][nt][2] = cinit[g][nt][0];
          acc[g][nt][3] = cinit[g][nt][1];
        }
#pragma unroll
      for (int ks = 0; ks < NB; ++ks) {
        const int g = (32 * ks) / KG;
        uint32_t a0, a1, a2, a3;
        if (KB == 8) {
          a0 = wk[0][2 * ks];
          a1 = wk[1][2 * ks];
          a2 = wk[0][2 * ks + 1];
          a3 = wk[1][2 * ks + 1];
        } else {
          const uint32_t x0 = wk[0][ks], x1 = wk[1][ks];
          a0 = (x0 & 0x0F0F0F0Fu) ^ 0x08080808u;
          a2 = ((x0 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
          a1 = (x1 & 0x0F0F0F0Fu) ^ 0x08080808u;
          a3 = ((x1 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma_s8(acc[g][nt], a0, a1, a2, a3, qb[ks][nt][0], qb[ks][nt][1]);
      }

      // --- scores (log2 units) and Delta for tokens g8, g8+8 of row c4 -------------
      const __half* ksc = reinterpret_cast<const __half*>(rs + C::VB);
      float zt[2], dl[2];
      bool vt[2];
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        const int tok = g8 + 8 * sl;
        vt[sl] = tok < nval;
        float dot = 0.f, dsum = 0.f, smax = 0.f;
#pragma unroll
        for (int g = 0; g < NGK; ++g) {
          const float s = __half2float(ksc[tok * NGK + g]);
          const float d0 = (float)acc[g][0][2 * sl], d1 = (float)acc[g][0][2 * sl + 1];
          const float d2 = (float)acc[g][1][2 * sl], d3 = (float)acc[g][1][2 * sl + 1];
          const float raw = fmaf(d3, 16777216.f, fmaf(d2, 65536.f, fmaf(d1, 256.f, d0)));
          dot = fmaf(raw, s, dot);
          dsum = fmaf(cg[g], s, dsum);
          smax = fmaxf(smax, s);
        }
        zt[sl] = vt[sl] ? dot * zs : -INFINITY;
        dl[sl] = fmaf(cb, smax, dsum);
      }

      // --- online softmax and bound sums (row c4) -------------------------------
      float mx = fmaxf(zt[0], zt[1]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mnew = fmaxf(m2, mx);
      const float alpha = exp2f(m2 - mnew);
      m2 = mnew;
      const float w0 = exp2f(zt[0] - mnew), w1 = exp2f(zt[1] - mnew);
      float ta = 0.f, tb = 0.f, tw = 0.f;
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        if (vt[sl]) {
          const float w = sl ? w1 : w0;
          ta = fmaf(w, expm1f(dl[sl]), ta);
          tb = fmaf(w, expf(-dl[sl]), tb);
          tw += w;
          dmax = fmaxf(dmax, dl[sl]);
        }
      }
      lsum = fmaf(lsum, alpha, tw);
      Asum = fmaf(Asum, alpha, ta);
      Bsum = fmaf(Bsum, alpha, tb);
      Esum = fmaf(Esum, alpha, tw * eta_cur);

      // --- value range of group c4 over tokens g8, g8+8 --------------------------
      const uint32_t* vm = reinterpret_cast<const uint32_t*>(rs + C::VB + C::KSB);
      if (c4 < NB) {
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          if (vt[sl]) {
            const __half2 sz = u32_as_h2(vm[(g8 + 8 * sl) * NB + c4]);
            const float s = __low2float(sz), z = __high2float(sz);
            vhi = fmaxf(vhi, __fmaf_rn(15.0f, s, z));
            vlo = fminf(vlo, z);
          }
        }
      }

      // --- rescale the PV state when a row max moved --------------------------------
      if (__any_sync(0xffffffffu, alpha != 1.0f)) {
        const int base = lane & ~3;
        const float a0 = __shfl_sync(0xffffffffu, alpha, base | (2 * (c4 & 1)));
        const float a1 = __shfl_sync(0xffffffffu, alpha, base | (2 * (c4 & 1) + 1));
        const float az = __shfl_sync(0xffffffffu, alpha, base | hP);
#pragma unroll
        for (int t = 0; t < 2 * NB; ++t) {
          opv[t][0] *= a0;
          opv[t][1] *= a1;
          opv[t][2] *= a0;
          opv[t][3] *= a1;
        }
#pragma unroll
        for (int g = 0; g < NB; ++g) zacc[g] *= az;
      }

      // --- P' = w * sV for tokens c4 + 4k, row hP (hi or lo half) -----------------
      float x[4];
      x[0] = __shfl_sync(0xffffffffu, w0, 4 * c4 + hP);
      x[1] = __shfl_sync(0xffffffffu, w0, 4 * c4 + 16 + hP);
      x[2] = __shfl_sync(0xffffffffu, w1, 4 * c4 + hP);
      x[3] = __shfl_sync(0xffffffffu, w1, 4 * c4 + 16 + hP);
      bool vx[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) vx[k] = c4 + 4 * k < nval;

      // V code stripes (row g8) of tokens c4 + 4k
      uint32_t vw[4][C::VSTR / 4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint8_t* p = rs + (c4 + 4 * k) * C::VRB + g8 * C::VSTR;
        if constexpr (C::VSTR == 8) {
          const uint2 v2 = *reinterpret_cast<const uint2*>(p);
          vw[k][0] = v2.x;
          vw[k][1] = v2.y;
        } else {
          vw[k][0] = *reinterpret_cast<const uint32_t*>(p);
        }
      }
#pragma unroll
      for (int g = 0; g < NB; ++g) {
        float P[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __half2 sz = u32_as_h2(vm[(c4 + 4 * k) * NB + g]);
          const float s = __low2float(sz), z = __high2float(sz);
          P[k] = vx[k] ? x[k] * s : 0.f;
          zacc[g] = vx[k] ? fmaf(x[k], z, zacc[g]) : zacc[g];
        }
        uint32_t bf[2];
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          const __half2 hi = __floats2half2_rn(P[2 * pr], P[2 * pr + 1]);
          const float2 hf = __half22float2(hi);
          const __half2 lo = __floats2half2_rn(P[2 * pr] - hf.x, P[2 * pr + 1] - hf.y);
          bf[pr] = lo_part ? h2_as_u32(lo) : h2_as_u32(hi);
        }
        // A fragments for m-tiles 2g (low nibbles) and 2g+1 (high nibbles)
        const int wsel = (2 * g) / 4;            // word of the stripe holding group g
        const int p = (2 * g) % 4;               // byte offset of group g in that word
        const uint32_t sel = (uint32_t)(p | ((p + 1) << 4) | ((4 + p) << 8) | ((5 + p) << 12));
        const uint32_t r01 = prmt(vw[0][wsel], vw[1][wsel], sel);   // tokens c4, c4+4
        const uint32_t r23 = prmt(vw[2][wsel], vw[3][wsel], sel);   // tokens c4+8, c4+12
        const uint32_t r01s = r01 >> 8, r23s = r23 >> 8;
        const __half2 k1024 = __float2half2_rn(1024.f);
        const __half2 k16inv = __float2half2_rn(0.0625f);
        const __half2 km64 = __float2half2_rn(-64.f);
        auto lo_n = [&](uint32_t r) {
          return h2_as_u32(__hsub2(u32_as_h2((r & 0x000F000Fu) | 0x64006400u), k1024));
        };
        auto hi_n = [&](uint32_t r) {
          return h2_as_u32(__hfma2(u32_as_h2((r & 0x00F000F0u) | 0x64006400u), k16inv, km64));
        };
        mma_f16(opv[2 * g], lo_n(r01), lo_n(r01s), lo_n(r23), lo_n(r23s), bf[0], bf[1]);
        mma_f16(opv[2 * g + 1], hi_n(r01), hi_n(r01s), hi_n(r23), hi_n(r23s), bf[0], bf[1]);
      }
    }
    __syncwarp();
    if (j + S < nloc) issue(j + S);
  }

  // ---- warp reductions ----------------------------------------------------------
#pragma unroll
  for (int o = 4; o < 32; o *= 2) {
    lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    Asum += __shfl_xor_sync(0xffffffffu, Asum, o);
    Bsum += __shfl_xor_sync(0xffffffffu, Bsum, o);
    Esum += __shfl_xor_sync(0xffffffffu, Esum, o);
    dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
    vhi = fmaxf(vhi, __shfl_xor_sync(0xffffffffu, vhi, o));
    vlo = fminf(vlo, __shfl_xor_sync(0xffffffffu, vlo, o));
  }
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    zacc[g] += __shfl_xor_sync(0xffffffffu, zacc[g], 1);
    zacc[g] += __shfl_xor_sync(0xffffffffu, zacc[g], 2);
  }
#pragma unroll
  for (int t = 0; t < 2 * NB; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) opv[t][e] += __shfl_xor_sync(0xffffffffu, opv[t][e], 2);

  __syncthreads();  // every warp is done with its stage buffers
  // merge area: per warp w: o[4][D], st[4][8], z[4][NB], vhi[NB], vlo[NB], eta
  float* mw = reinterpret_cast<float*>(sm) + warp * C::MW_FLOATS;
  float* mo = mw;
  float* mst = mw + kRows * D;
  float* mz = mst + kRows * 8;
  float* mr = mz + kRows * NB;
  if (c4 < 2) {  // hi-part lanes own the combined hi+lo sums
#pragma unroll
    for (int g = 0; g < NB; ++g)
#pragma unroll
      for (int hn = 0; hn < 2; ++hn) {
        const int chR = 32 * g + 4 * g8 + hn, chR8 = chR + 2;
        const int h0 = 2 * c4, h1 = 2 * c4 + 1;
        mo[h0 * D + chR] = opv[2 * g + hn][0];
        mo[h1 * D + chR] = opv[2 * g + hn][1];
        mo[h0 * D + chR8] = opv[2 * g + hn][2];
        mo[h1 * D + chR8] = opv[2 * g + hn][3];
      }
  }
  if (g8 == 0) {  // lanes 0..3 hold row c4's statistics
    mst[c4 * 8 + 0] = m2;
    mst[c4 * 8 + 1] = lsum;
    mst[c4 * 8 + 2] = Asum;
    mst[c4 * 8 + 3] = Bsum;
    mst[c4 * 8 + 4] = Esum;
    mst[c4 * 8 + 5] = dmax;
    if (c4 < NB) {
      mr[c4] = vhi;
      mr[NB + c4] = vlo;
    }
  }
  if (c4 == 0 && g8 < 4) {
#pragma unroll
    for (int g = 0; g < NB; ++g) mz[g8 * NB + g] = zacc[g];
  }
  if (lane == 0) mr[2 * NB] = etamax;
  __syncthreads();

  // ---- CTA merge: all warps -> one record in shared memory ----------------------
  float* cm = reinterpret_cast<float*>(sm) + kWarps * C::MW_FLOATS;   // merged record
  float* cst = cm + kRows * D;
  float* cr = cst + kRows * 8;
  if (tid < kRows) {
    const int r = tid;
    float M = -INFINITY;
    for (int w = 0; w < kWarps; ++w)
      M = fmaxf(M, reinterpret_cast<float*>(sm)[w * C::MW_FLOATS + kRows * D + r * 8]);
    float L = 0.f, A = 0.f, Bv = 0.f, Ev = 0.f, Dm = 0.f;
    for (int w = 0; w < kWarps; ++w) {
      const float* s = reinterpret_cast<float*>(sm) + w * C::MW_FLOATS + kRows * D + r * 8;
      const float f = s[0] == -INFINITY ? 0.f : exp2f(s[0] - M);
      L = fmaf(f, s[1], L);
      A = fmaf(f, s[2], A);
      Bv = fmaf(f, s[3], Bv);
      Ev = fmaf(f, s[4], Ev);
      Dm = fmaxf(Dm, s[5]);
    }
    cst[r * 8 + 0] = M;
    cst[r * 8 + 1] = L;
    cst[r * 8 + 2] = A;
    cst[r * 8 + 3] = Bv;
    cst[r * 8 + 4] = Ev;
    cst[r * 8 + 5] = Dm;
  } else if (tid == kRows) {
    float hi[NB], lo[NB], et = 0.f;
    for (int g = 0; g < NB; ++g) {
      hi[g] = -INFINITY;
      lo[g] = INFINITY;
    }
    for (int w = 0; w < kWarps; ++w) {
      const float* r = reinterpret_cast<float*>(sm) + w * C::MW_FLOATS + kRows * D + kRows * 8 +
                       kRows * NB;
      for (int g = 0; g < NB; ++g) {
        hi[g] = fmaxf(hi[g], r[g]);
        lo[g] = fminf(lo[g], r[NB + g]);
      }
      et = fmaxf(et, r[2 * NB]);
    }
    for (int g = 0; g < NB; ++g) {
      cr[g] = hi[g];
      cr[NB + g] = lo[g];
    }
    cr[2 * NB] = et;
  }
  __syncthreads();
  for (int i = tid; i < kRows * D; i += blockDim.x) {
    const int r = i / D, c = i % D;
    const float M = cst[r * 8];
    float o = 0.f;
    for (int w = 0; w < kWarps; ++w) {
      const float* mwp = reinterpret_cast<float*>(sm) + w * C::MW_FLOATS;
      const float mwr = mwp[kRows * D + r * 8];
      if (mwr == -INFINITY) continue;
      const float f = exp2f(mwr - M);
      o = fmaf(f, mwp[i] + mwp[kRows * D + kRows * 8 + r * NB + c / 32], o);
    }
    cm[i] = o;
  }
  __syncthreads();

  auto range_of = [&](const float* r) {
    float rg = 0.f;
    for (int g = 0; g < NB; ++g) rg = fmaxf(rg, r[g] - r[NB + g]);
    return rg;
  };

  if (active == 1) {  // the only split: finish here
    for (int r = 0; r < kRows; ++r) {
      const float* s = cst + r * 8;
      finalize_row<D>(a, b, kvh, r, s[1], s[2], s[3], s[4], s[5], range_of(cr), cr[2 * NB],
                      cm + r * D, tid, blockDim.x, tid == 0);
    }
    return;
  }

  // ---- write this split's record; the last CTA of (b, kvh) merges all --------------
  const int64_t unit = (int64_t)b * a.hkv + kvh;
  const int splits = gridDim.x;
  float* rec = a.part + (unit * splits + split) * record_floats(D);
  for (int i = tid; i < 2 * NB + 1; i += blockDim.x) rec[1 + i] = cr[i];
  for (int i = tid; i < kRows * 8; i += blockDim.x) rec[kHdr + (i / 8) * (8 + D) + i % 8] = cst[i];
  for (int i = tid; i < kRows * D; i += blockDim.x)
    rec[kHdr + (i / D) * (8 + D) + 8 + i % D] = cm[i];
  __threadfence();
  __syncthreads();
  int* flag = reinterpret_cast<int*>(sm + C::OFF_FLAG);
  if (tid == 0) {
    const int prev = atomicAdd(a.counters + unit, 1);
    *flag = prev == active - 1;
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  const float* recs = a.part + unit * splits * record_floats(D);
  // statistics per row (every thread recomputes what it needs; reads hit L2)
  float* fst = cst;   // reuse: merged stats of all splits
  if (tid < kRows) {
    const int r = tid;
    float M = -INFINITY;
    for (int s = 0; s < active; ++s)
      M = fmaxf(M, __ldcg(recs + s * record_floats(D) + kHdr + r * (8 + D)));
    float L = 0.f, A = 0.f, Bv = 0.f, Ev = 0.f, Dm = 0.f;
    for (int s = 0; s < active; ++s) {
      const float* st = recs + s * record_floats(D) + kHdr + r * (8 + D);
      const float ms = __ldcg(st);
      const float f = ms == -INFINITY ? 0.f : exp2f(ms - M);
      L = fmaf(f, __ldcg(st + 1), L);
      A = fmaf(f, __ldcg(st + 2), A);
      Bv = fmaf(f, __ldcg(st + 3), Bv);
      Ev = fmaf(f, __ldcg(st + 4), Ev);
      Dm = fmaxf(Dm, __ldcg(st + 5));
    }
    fst[r * 8 + 0] = M;
    fst[r * 8 + 1] = L;
    fst[r * 8 + 2] = A;
    fst[r * 8 + 3] = Bv;
    fst[r * 8 + 4] = Ev;
    fst[r * 8 + 5] = Dm;
  } else if (tid == kRows) {
    for (int g = 0; g < NB; ++g) {
      float hi = -INFINITY, lo = INFINITY;
      for (int s = 0; s < active; ++s) {
        hi = fmaxf(hi, __ldcg(recs + s * record_floats(D) + 1 + g));
        lo = fminf(lo, __ldcg(recs + s * record_floats(D) + 1 + NB + g));
      }
      cr[g] = hi;
      cr[NB + g] = lo;
    }
    float et = 0.f;
    for (int s = 0; s < active; ++s) et = fmaxf(et, __ldcg(recs + s * record_floats(D) + 1 + 2 * NB));
    cr[2 * NB] = et;
  }
  __syncthreads();
  for (int i = tid; i < kRows * D; i += blockDim.x) {
    const int r = i / D, c = i % D;
    const float M = fst[r * 8];
    float o = 0.f;
    for (int s = 0; s < active; ++s) {
      const float* st = recs + s * record_floats(D) + kHdr + r * (8 + D);
      const float ms = __ldcg(st);
      if (ms == -INFINITY) continue;
      o = fmaf(exp2f(ms - M), __ldcg(st + 8 + c), o);
    }
    cm[i] = o;
  }
  __syncthreads();
  for (int r = 0; r < kRows; ++r) {
    const float* s = fst + r * 8;
    finalize_row<D>(a, b, kvh, r, s[1], s[2], s[3], s[4], s[5], range_of(cr), cr[2 * NB],
                    cm + r * D, tid, blockDim.x, tid == 0);
  }
  if (tid == 0) a.counters[unit] = 0;  // leave the workspace ready for the next call
}

// ------------------------------------------------------------------------------------
template <int D, int KB, int KG>
DecodeVariant make_variant() {
  constexpr int S = 3;
  return DecodeVariant{decode_mma_kernel<D, KB, KG, S>, DecodeCfg<D, KB, KG, S>::SMEM,
                       record_floats(D)};
}

DecodeVariant select_decode_kernel(int d, int kbits, int kgroup) {
#define KVQ_DECODE_CASE(D_, KB_, KG_) \
  if (d == D_ && kbits == KB_ && kgroup == KG_) return make_variant<D_, KB_, KG_>();
  KVQ_DECODE_CASE(128, 8, 128)
  KVQ_DECODE_CASE(128, 8, 64)
  KVQ_DECODE_CASE(128, 8, 32)
  KVQ_DECODE_CASE(128, 4, 128)
  KVQ_DECODE_CASE(128, 4, 64)
  KVQ_DECODE_CASE(128, 4, 32)
  KVQ_DECODE_CASE(64, 8, 64)
  KVQ_DECODE_CASE(64, 8, 32)
  KVQ_DECODE_CASE(64, 4, 64)
  KVQ_DECODE_CASE(64, 4, 32)
#undef KVQ_DECODE_CASE
  return DecodeVariant{nullptr, 0, 0};
}

int decode_threads() { return kWarps * 32; }

}  // namespace kvq
