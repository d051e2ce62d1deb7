// decode_kernel.cuh -- fused split-K decode attention over the packed
// Tier-1 cache with the certified per-query error bound computed in the same
// pass ("Runtime-Certified Bounded-Error Quantized Attention", Methodology 2:
// E_key from the total-variation distance between exact and quantized
// softmax, bounded through the per-token score perturbation Delta; E_val from
// the block errors eta_b weighted by attention mass; both from scales, query
// norms and the value range only).
//
// Grid (split, kv head, sequence); 4 warps per CTA.  Each warp streams its
// own pages of the split through an S-stage ring in shared memory: one bulk
// copy (cp.async.bulk) brings the page's whole block -- K codes (stored with
// their 16-byte chunks pre-permuted for conflict-free reads), V codes, K
// scales, V scale/zero; completion on an mbarrier per stage, every wait bounded.
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
//         product keeps ~22 bits); the zero point adds sum_j w_j zV_{j,g}
//         through one more MMA per page (rows = groups).
// With outlier extraction (OUT; "Hurwitz Quaternion Multiplicative
// Quantization for KV Cache Compression", Method 3) the block's outlier
// section comes with the same copy: an extracted K chunk adds q'_chunk . k16
// to the token's score and half an fp16 ulp per channel (and, for rotated
// keys, its norm in the rotation allowance) to Delta; an extracted V chunk
// (code 0, so the tensor-core path gave it the group zero z) adds
// w * (v16 - z) to the PV accumulators of its channels and widens the value
// range of its group to the stored values.
// Warps merge in shared memory; splits merge in the last CTA of each
// (sequence, kv head) to finish: o = O/l, TV = min(tanh(maxDelta/2), A/B),
// E_key = TV*(range + 2 max eta), E_val = E/l, bound = kappa*(E_key+E_val),
// flag = bound > tau.
#pragma once

#include <type_traits>

#include "kvq_internal.cuh"
#include "quantize_token.cuh"

namespace kvq {

constexpr int kWarps = 4;
constexpr int kRows = 4;  // query rows per kv head handled by one CTA
constexpr int kHdr = 16;  // floats of the per-split record header

__host__ __device__ constexpr int record_floats(int d) { return kHdr + kRows * (8 + d); }

template <int D, int KB, int KG, int S, bool OUT = false>
struct DecodeCfg {
  static constexpr int NB = D / 32;
  static constexpr int NGK = D / KG;
  static constexpr int KRB = D * KB / 8;          // K row bytes
  static constexpr int KT = kPage * KRB;          // K tile bytes
  static constexpr int VRB = D / 2;               // V row bytes
  static constexpr int VB = kPage * VRB;
  static constexpr int KSB = kPage * NGK * 2;
  static constexpr int VMB = kPage * NB * 4;
  static constexpr int OS = KT + VB + KSB + VMB;  // the outlier section (OUT)
  static constexpr int REST = VB + KSB + VMB + (OUT ? kOutBytes : 0);   // after the K codes
  static constexpr int BLOCK = KT + REST;
  static constexpr bool SWZ = KRB == 128;
  static constexpr int KSTR = KRB / 4;            // K stripe bytes per lane
  static constexpr int VSTR = VRB / 8;            // V stripe bytes per lane
  // shared memory carve-up (offsets from a 128-aligned base): per warp S stages
  // of one whole block each (K codes, then V codes and metadata)
  static constexpr int OFF_ST = 0;
  static constexpr int SZ_ST = kWarps * S * BLOCK;
  static constexpr int OFF_BAR = (OFF_ST + SZ_ST + 15) / 16 * 16;
  static constexpr int OFF_PG = OFF_BAR + kWarps * S * 8;
  static constexpr int OFF_Q = (OFF_PG + kWarps * S * 4 + 15) / 16 * 16;   // int8 qdig[4][4][D]
  static constexpr int OFF_QB = OFF_Q + kRows * 4 * D;                      // int qsum[4][NGK][4]
  static constexpr int OFF_QF = OFF_QB + kRows * NGK * 4 * 4;               // float q'[4][D]
  static constexpr int OFF_RC = OFF_QF + kRows * D * 4;                     // row constants
  static constexpr int RC_FLOATS = kRows * (2 + NGK + (OUT ? 1 : 0));       // zs, cb, cg[NGK], cr
  static constexpr int META_FLOATS = kPage * NB + kPage * NGK;              // per warp
  static constexpr int OFF_META = (OFF_RC + RC_FLOATS * 4 + 15) / 16 * 16;
  static constexpr int OFF_FLAG = OFF_META + kWarps * META_FLOATS * 4;
  // OUT: q' chunk-major, [chunk][row][4] fp32 (the 4 rows of one chunk are
  // neighbouring 16-byte vectors: conflict-free reads by the lanes of a token)
  static constexpr int OFF_QC = OFF_FLAG + 16;
  static constexpr int END = OFF_QC + (OUT ? kRows * D * 4 : 0);
  // merge area (aliases the stage buffers once the page loop is over)
  static constexpr int MW_FLOATS = kRows * D + kRows * 8 + kRows * NB + 2 * NB + 1;
  static constexpr int MERGE_BYTES = (kWarps + 1) * MW_FLOATS * 4;
  static constexpr int SMEM = 128 + (END > MERGE_BYTES ? END : MERGE_BYTES);
  static_assert(MERGE_BYTES <= OFF_BAR, "merge area must fit in the stage buffers");
};

// weight of the last split when the append is fused (its appending warp spends
// about two pages' time on the new token before starting on its pages)
constexpr float kAppendLastSplit = 0.85f;

// resident CTAs per SM the register budget is sized for (4 = 128 registers)
template <int D, int KB, int KG>
constexpr int min_ctas() { return 4; }

// First page of split s when npages pages are shared by n splits in decreasing
// sizes (split i weighs 10(n-1) - i, so the first is 10/9 of the last): the
// grid puts the split index in its slow dimension, later splits are launched
// later, and with fewer pages the splits of a (sequence, kv head) end together.
// (fp32 arithmetic: no 64-bit division on the kernel's start path; every CTA
// evaluates the same expression, so neighbouring splits agree on their border,
// and the result is monotone in s with split_start(0) = 0, split_start(n) = npages).
// last_w scales the last split's weight (the fused append gives its warp extra
// work before its pages).
__device__ __forceinline__ int split_start(int s, int n, int npages, float last_w) {
  if (s <= 0) return 0;
  if (s >= n) return npages;
  const float k = 10.0f * (float)(n - 1);
  const float w = (float)s * k - 0.5f * (float)s * (float)(s - 1);
  const float wn = (float)(n - 1) * k - 0.5f * (float)(n - 1) * (float)(n - 2) +
                   last_w * (k - (float)(n - 1));
  return min(npages, (int)__fmul_rn((float)npages, __fdiv_rn(w, wn)));
}

// The step's new token of (b, kvh) into slot (n - 1) % 16 of physical page pg
// (kvq_decode_attention_append); returns the token's eta contribution.  Not
// inlined: its registers stay out of the decode's allocation.
template <int D, int KB, int KG, bool OUT>
__device__ __noinline__ float fused_append(const DecodeArgs& a, int b, int kvh, int n, int pg,
                                           int lane) {
  constexpr int E = D / 32;
  float xk[E], xv[E];
  const int64_t base = b * a.app_seq_stride + kvh * a.app_head_stride + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    xk[e] = load_elem(a.app_k, a.app_bf16, base + e);
    xv[e] = load_elem(a.app_v, a.app_bf16, base + e);
  }
  float eu = 0.f;
  if ((unsigned)pg < (unsigned)a.num_pages) {
    const BlockLayout L{D, KB, KG, OUT ? 1 : 0};
    uint8_t* blk = const_cast<uint8_t*>(a.pool) + ((int64_t)pg * a.hkv + kvh) * L.bytes();
    eu = quantize_token_warp<D, KB, KG, OUT>(xk, xv, blk, (n - 1) % kPage,
                                        const_cast<float*>(a.eta) + (int64_t)pg * a.hkv + kvh,
                                        a.signs, a.rot_c, a.err, lane);
    asm volatile("fence.proxy.async.global;" ::: "memory");
  } else if (lane == 0) {
    set_error(a.err, KVQ_ERR_INVALID_ARG);
  }
  __syncwarp();
  return eu;
}

// The ring stage of a page step: a compile-time constant, or a runtime index.
template <int I>
__device__ __forceinline__ constexpr int stage_index(std::integral_constant<int, I>) { return I; }
__device__ __forceinline__ int stage_index(int st) { return st; }

// APPEND: the fused step (kvq_decode_attention_append); a separate
// instantiation, so the plain decode carries none of its code or registers.
template <int D, int KB, int KG, int S, bool APPEND, bool OUT>
__global__ void __launch_bounds__(kWarps * 32, min_ctas<D, KB, KG>())
    decode_mma_kernel(const __grid_constant__ DecodeArgs a) {
  using C = DecodeCfg<D, KB, KG, S, OUT>;
  static_assert(S < 32, "the issue side must stay within one 32-page chunk of the loop");
  constexpr int NB = C::NB, NGK = C::NGK;
  constexpr int Q = KB == 8 ? 127 : 7;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte aligned base; pointer arithmetic on the __shared__ array keeps
  // every access below in the shared address space
  uint8_t* sm = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  // grid (unit, split): the unit = (sequence, kv head) index runs fastest, so
  // every unit's first split is launched before any unit's second one
  const int split = blockIdx.y, kvh = blockIdx.x % a.hkv, b = blockIdx.x / a.hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c4 = lane & 3, g8 = lane >> 2;
  // This warp's ring barriers need nothing from memory: set them up first.
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR) + warp * S;
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }
  // Launched with programmatic serialization, the CTA may start while the
  // previous grid in the stream is still running.  Until pdl_wait it only
  // prefetches into L2 the pages its warps will copy first, at the indices the
  // page table holds now for a full-length context: these are hints (clamped
  // to the pool, and a prefetch changes no memory), so nothing computed below
  // depends on what the previous grid writes.  Every load that does comes
  // after the wait.
  {
    const int sp0 = split_start(split, gridDim.y, a.max_pages, APPEND ? kAppendLastSplit : 1.0f);
    const int sp1 = split_start(split + 1, gridDim.y, a.max_pages, APPEND ? kAppendLastSplit : 1.0f);
    const int lp = sp0 + warp + lane * kWarps;
    if (lane < S && lp < sp1) {
      const int pg = __ldcg(a.page_table + (int64_t)b * a.max_pages + lp);
      if (pg >= 0 && pg < a.num_pages)
        bulk_prefetch_l2(a.pool + ((int64_t)pg * a.hkv + kvh) * C::BLOCK, C::BLOCK);
    }
  }
  pdl_wait();
  pdl_release();

  // The context length, the query rows and this warp's first 32 page indices
  // are loaded together: none of these addresses depends on the others (the
  // page indices assume a full-length context and are reloaded otherwise).
  const int nsp = gridDim.y;
  constexpr float kLastW = APPEND ? kAppendLastSplit : 1.0f;
  const int p0_spec = split_start(split, nsp, a.max_pages, kLastW);
  const int p1_spec = split_start(split + 1, nsp, a.max_pages, kLastW);
  const int32_t* ptab = a.page_table + (int64_t)b * a.max_pages;
  int n = a.seq_lens[b];
  int pt_first = p0_spec + warp + lane * kWarps < p1_spec
                     ? __ldg(ptab + p0_spec + warp + lane * kWarps) : -1;
  constexpr int E = D / 32;
  if constexpr (APPEND) {
    // the warp that appends when the context is full-length (the usual case):
    // start pulling the step's new token toward L2 now
    const int lp = a.max_pages - 1;
    if (lp >= p0_spec && lp < p1_spec && (lp - p0_spec) % kWarps == warp && lane < 2) {
      const int esz = a.app_bf16 ? 2 : 4;
      const char* src = static_cast<const char*>(lane == 0 ? a.app_k : a.app_v) +
                        (b * a.app_seq_stride + kvh * a.app_head_stride) * esz;
      for (int off = 0; off < D * esz; off += 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(src + off));
    }
  }
  constexpr int QPT = kRows * D / (kWarps * 32);   // query elements per thread
  // raw element bits, all loads issued before any is used (the bf16 -> fp32
  // conversion waits until the rows are written to shared memory)
  uint32_t qraw[QPT];
  const bool qb16 = a.q_bf16;
#pragma unroll
  for (int k = 0; k < QPT; ++k) {
    const int i = tid + k * kWarps * 32, r = i / D, c = i % D;
    const int qi = r / a.G, h = kvh * a.G + r % a.G;
    const int64_t e = (((int64_t)b * a.nq + qi) * a.hq + h) * D + c;
    const int64_t eo = r < a.R ? e : 0;   // an in-range address for padding rows
    qraw[k] = qb16 ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(a.q) + eo)
                   : __float_as_uint(__ldg(reinterpret_cast<const float*>(a.q) + eo));
    if (r >= a.R) qraw[k] = 0u;
  }

  if (n < 0) n = 0;
  // A context longer than the page table is cut to it; the pages past the cut
  // are never read, so the unit's results are marked uncertified (below).
  const bool clamped = n > a.max_pages * kPage;
  if (clamped) {
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
  const int p0 = split_start(split, active, npages, kLastW);
  const int p1 = split_start(split + 1, active, npages, kLastW);
  const int first = p0 + warp;
  if (p0 != p0_spec || p1 != p1_spec)
    pt_first = first + lane * kWarps < p1 ? __ldg(ptab + first + lane * kWarps) : -1;
  // The fused append is done by the warp whose local pages include the
  // sequence's last page, before that page's copy: codes and metadata go to
  // global memory through the generic proxy, and the proxy fence orders them
  // before the bulk copy (async proxy) that reads the page back.  When the last
  // page is among the warp's first S it runs here; otherwise just before the
  // page loop, so the rest of the CTA does not wait for it at the prologue's
  // barriers.  Returns the token's eta contribution (0 if the page is invalid).
  const bool app_here =
      APPEND && npages - 1 >= p0 && npages - 1 < p1 && (npages - 1 - p0) % kWarps == warp;
  const int j_last = (npages - 1 - first) / kWarps;   // local index of the last page
  auto do_append = [&]() -> float {
    return fused_append<D, KB, KG, OUT>(a, b, kvh, n, ptab[npages - 1], lane);
  };
  if (app_here && j_last < S) (void)do_append();

  uint8_t* stage0 = sm + C::OFF_ST + warp * S * C::BLOCK;
  int* spage = reinterpret_cast<int*>(sm + C::OFF_PG) + warp * S;
  int8_t* qdig = reinterpret_cast<int8_t*>(sm + C::OFF_Q);
  int* qsum = reinterpret_cast<int*>(sm + C::OFF_QB);
  float* qf = reinterpret_cast<float*>(sm + C::OFF_QF);
  float* rc = reinterpret_cast<float*>(sm + C::OFF_RC);

  // ---- pipeline start: page indices, barriers, first S copies --------------
  const int nloc = first < p1 ? (p1 - first + kWarps - 1) / kWarps : 0;
  auto fetch_chunk = [&](int c) -> int {
    const int j = c * 32 + lane;
    return j < nloc ? __ldg(ptab + first + j * kWarps) : -1;
  };
  int pt_chunk = -1, pt_val = -1, pt_next = lane < nloc ? pt_first : -1;
  // eta of the pages: lane l holds eta of local page 32c + l of the chunk c being
  // issued (eta_iss) and of the chunk being processed (eta_proc).  Each is loaded
  // when the issue side enters its chunk, S pages before the first of them is
  // processed, and read by a shuffle -- no per-page load on the loop's path.
  const float* eta_kv = a.eta + kvh;
  float eta_iss = 0.f, eta_proc = 0.f;
  __syncwarp();

  auto issue = [&](int j, int st) {  // whole warp; lane 0 issues local page j into stage st
    const int c = j >> 5;
    if (c != pt_chunk) {
      pt_val = (c == pt_chunk + 1) ? pt_next : fetch_chunk(c);
      pt_next = fetch_chunk(c + 1);
      pt_chunk = c;
      // (the fused append raises eta in this kernel: read it from L2, not L1)
      eta_iss = (unsigned)pt_val < (unsigned)a.num_pages
                    ? (APPEND ? __ldcg(eta_kv + (int64_t)pt_val * a.hkv)
                              : __ldg(eta_kv + (int64_t)pt_val * a.hkv))
                    : 0.f;
    }
    const int page = __shfl_sync(0xffffffffu, pt_val, j & 31);
    if (lane == 0) {
      const bool ok = page >= 0 && page < a.num_pages;
      spage[st] = ok ? page : -1;
      if (ok) {
        const int64_t blk = (int64_t)page * a.hkv + kvh;
        mbar_arrive_expect_tx(&bar[st], C::BLOCK);
        // a launch reads each cache page once: its lines are evicted first
        bulk_g2s_hint(stage0 + st * C::BLOCK, a.pool + blk * C::BLOCK, C::BLOCK, &bar[st],
                      l2_evict_first_policy());
      } else {
        set_error(a.err, KVQ_ERR_INVALID_ARG);
        mbar_arrive(&bar[st]);
      }
    }
    __syncwarp();  // publish spage[st] to the warp
  };
  for (int j = 0; j < S && j < nloc; ++j) issue(j, j);

  // ---- query rows: rotate, fixed point, norms (loaded before the copies) -----
#pragma unroll
  for (int k = 0; k < QPT; ++k)
    qf[tid + k * kWarps * 32] = qb16 ? __uint_as_float(qraw[k] << 16) : __uint_as_float(qraw[k]);
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
    // q' * 2^F in int32, split into four signed base-256 digits, stored in the
    // order the MMA B fragments read them: for 4-bit keys, position
    // 32b + 8s + 4(i%2) + i/2 holds channel 32b + 8s + i (even/odd nibbles)
    int ds[4] = {0, 0, 0, 0};  // digit sums over this lane's channels (one key group)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = lane * E + e;
      int v = __float2int_rn(ldexpf(x[e], F));
      const int i8 = c % 8;
      const int pos = KB == 8 ? c : (c - i8) + 4 * (i8 % 2) + i8 / 2;
#pragma unroll
      for (int d = 0; d < 4; ++d) {
        const int dg = d < 3 ? (int)(int8_t)(v & 0xFF) : v;
        v = (v - dg) >> 8;
        qdig[(r * 4 + d) * D + pos] = (int8_t)dg;
        ds[d] += dg;
      }
    }
    if (KB == 4) {  // sum of every digit over each key group (bias of code + 8)
#pragma unroll
      for (int d = 0; d < 4; ++d)
#pragma unroll
        for (int o = 1; o < KG / E; o *= 2) ds[d] += __shfl_xor_sync(0xffffffffu, ds[d], o);
      if ((lane * E) % KG == 0) {
        const int g = (lane * E) / KG;
#pragma unroll
        for (int d = 0; d < 4; ++d) qsum[(r * NGK + g) * 4 + d] = ds[d];
      }
    }
    if (lane == 0) {
      rc[r] = ldexpf(a.s_att * kLog2e, -F);                      // zs: score scale, log2 units
      rc[kRows + r] = a.signs ? kKappa * a.s_att * kRotSlack * sqrtf((float)D) * (float)Q *
                                    sqrtf(l2)
                              : 0.f;                               // cb
#pragma unroll
      for (int g = 0; g < NGK; ++g)
        rc[2 * kRows + r * NGK + g] = kKappa * a.s_att * 0.5f * l1[g];   // cg
      // cr: an extracted key chunk's share of the rotation allowance, per unit
      // of the chunk's norm
      if constexpr (OUT)
        rc[(2 + NGK) * kRows + r] = a.signs ? kKappa * a.s_att * kRotSlack * sqrtf(l2) : 0.f;
    }
    // the extracted key chunks are scored against q' in fp32
    if constexpr (OUT) {
      float* qc = reinterpret_cast<float*>(sm + C::OFF_QC);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int c = lane * E + e;
        qc[((c / 4) * kRows + r) * 4 + c % 4] = x[e];
      }
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
      for (int nt = 0; nt < 2; ++nt) {
        const uint2 w2 = *reinterpret_cast<const uint2*>(qdig + (r * 4 + 2 * nt + dl) * D + 32 * ks +
                                                         8 * c4);
        qb[ks][nt][0] = w2.x;
        qb[ks][nt][1] = w2.y;
      }
  }
  // 4-bit key codes enter as code + 8: per key group, the bias -8 * (sum of each
  // digit of row c4 over the group), recombined like the accumulators
  // (digits 0 + 256 * 1 -> blo, digits 2 + 256 * 3 -> bhi)
  int blo[NGK], bhi[NGK];
#pragma unroll
  for (int g = 0; g < NGK; ++g) {
    const int* qs = qsum + (c4 * NGK + g) * 4;
    blo[g] = KB == 4 ? -8 * (qs[0] + 256 * qs[1]) : 0;
    bhi[g] = KB == 4 ? -8 * (qs[2] + 256 * qs[3]) : 0;
  }
  const float zs = rc[c4];
  const float cb = rc[kRows + c4];
  float cg[NGK];
#pragma unroll
  for (int g = 0; g < NGK; ++g) cg[g] = rc[2 * kRows + c4 * NGK + g];

  // ---- accumulators ------------------------------------------------------------
  float m2 = -INFINITY, lsum = 0.f, Asum = 0.f, Bsum = 0.f, Esum = 0.f, dmax = 0.f;
  // PV accumulators: m-tile 2g holds the low-nibble channels of group g (codes
  // entered as fp16 subnormals c*2^-24), m-tile 2g+1 the high-nibble channels
  // (16c*2^-24); the power-of-two factors are removed after the loop.
  float opv[2 * NB][4];
  float zmv[4];  // zero-point MMA: rows = groups, columns = (row, hi/lo part)
#pragma unroll
  for (int t = 0; t < 2 * NB; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) opv[t][e] = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) zmv[e] = 0.f;
  constexpr int EPL = NB / 2;  // V metadata entries converted per lane and page
  // etamax = +inf marks a unit with a page that was not read (an index outside
  // the pool, a wait that ran out, a context cut to the page table): every
  // merge below takes maxima, so the mark reaches the finish, which then
  // reports bound = +inf and flag = 1 instead of a bound over the pages read.
  float vhi[EPL], vlo[EPL], etamax = clamped ? INFINITY : 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    vhi[i] = -INFINITY;
    vlo[i] = INFINITY;
  }
  const int hP = g8 & 3;
  const bool lo_part = g8 >= 4;
  float* vs32 = reinterpret_cast<float*>(sm + C::OFF_META) + warp * C::META_FLOATS;
  float* ks32 = vs32 + kPage * NB;
  // hi part of a value: its top 11 significant bits (exact in fp16); lo lanes
  // take the remainder, so hi + lo reproduces the fp32 value to ~2^-22
  // (two at a time: v = K1*t + K2*x with (K1, K2) = (1, 0) or (-1, 1))
  const float2 K1 = lo_part ? make_float2(-1.f, -1.f) : make_float2(1.f, 1.f);
  const float2 K2 = lo_part ? make_float2(1.f, 1.f) : make_float2(0.f, 0.f);
  auto hilo2 = [&](float2 v) -> uint32_t {
    const float2 t = make_float2(__int_as_float(__float_as_int(v.x) & 0xFFFFE000),
                                 __int_as_float(__float_as_int(v.y) & 0xFFFFE000));
    const float2 r = fma2(t, K1, mul2(v, K2));
    return h2_as_u32(__floats2half2_rn(r.x, r.y));
  };

  // this lane's fixed offsets inside a stage
  constexpr int KW = C::KSTR / 4;                        // 32-bit words per key stripe
  constexpr int KCH = C::KSTR >= 16 ? C::KSTR / 16 : 1;  // 16-byte chunks per key stripe
  int koff[KCH];                                         // row g8; row g8+8 is +8 rows
#pragma unroll
  for (int hh = 0; hh < KCH; ++hh) {
    if constexpr (C::KSTR >= 16) {
      int chunk = (c4 * C::KSTR) / 16 + hh;
      if (C::SWZ) chunk ^= (g8 & 7);
      koff[hh] = g8 * C::KRB + chunk * 16;
    } else {
      koff[hh] = g8 * C::KRB + c4 * C::KSTR;
    }
  }
  const int voff = c4 * C::VRB + g8 * C::VSTR;           // V stripe of token c4 (+4 rows per k)
  const int zgrp = g8 < NB ? g8 : 0;

  // the fused append when the last page comes later: after the q prologue, so
  // only this warp (whose split is the shortest) starts its pages later
  if (app_here && j_last >= S) {
    const float eu = do_append();
    // the last page's eta, if its chunk was already loaded, gets the token too
    if ((j_last >> 5) == pt_chunk && lane == (j_last & 31)) eta_iss = fmaxf(eta_iss, eu);
  }

  // ---- page loop ---------------------------------------------------------------
  // One step per local page j, in ring stage j % S.  The stage is a template
  // constant (the loop is unrolled by S), so every shared-memory address below is
  // a fixed offset; FULL pages (all 16 tokens inside the context, every page but
  // possibly a sequence's last) skip the per-token context masks.
  auto page_step = [&](auto st_c, auto full_c, int j, uint32_t par) -> bool {
    const int st = stage_index(st_c);
    constexpr bool FULL = decltype(full_c)::value;
    const bool ok = mbar_wait(&bar[st], par);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) set_error(a.err, KVQ_ERR_TIMEOUT);
      etamax = INFINITY;
      return false;
    }
    const int page = spage[st];
    if ((j & 31) == 0) eta_proc = eta_iss;   // the issue side is S < 32 pages ahead
    const float eta_cur = __shfl_sync(0xffffffffu, eta_proc, j & 31);
    if (page >= 0) {
      const uint8_t* kt = stage0 + st * C::BLOCK;
      const uint8_t* rs = kt + C::KT;
      const int nval = FULL ? kPage : min(kPage, n - (first + j * kWarps) * kPage);
      etamax = fmaxf(etamax, eta_cur);
      const uint32_t* vm = reinterpret_cast<const uint32_t*>(rs + C::VB + C::KSB);
      const __half* ksc = reinterpret_cast<const __half*>(rs + C::VB);

      // --- page metadata to fp32 once for the warp; value range per group -------
      {
        uint32_t mw[EPL];
        if constexpr (EPL == 2) {
          const uint2 v2 = reinterpret_cast<const uint2*>(vm)[lane];
          mw[0] = v2.x;
          mw[1] = v2.y;
        } else {
          mw[0] = vm[lane];
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane * EPL + i;  // token e / NB, group e % NB
          const float2 sz = __half22float2(u32_as_h2(mw[i]));
          const bool in = e / NB < nval;
          const int tok = e / NB, gg = e % NB;   // table [group][token % 4][token / 4]
          vs32[gg * kPage + (tok % 4) * 4 + tok / 4] = in ? sz.x : 0.f;
          vhi[i] = in ? fmaxf(vhi[i], __fmaf_rn(15.0f, sz.x, sz.y)) : vhi[i];
          vlo[i] = in ? fminf(vlo[i], sz.y) : vlo[i];
        }
        for (int e = lane; e < kPage * NGK; e += 32) ks32[e] = __half2float(ksc[e]);
      }

      // --- K codes of rows g8, g8+8 (this lane's stripe) -> QK^T on int8 MMA ---
      uint32_t wk[2][KW];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const uint8_t* kr = kt + rr * 8 * C::KRB;
        if constexpr (C::KSTR >= 16) {
#pragma unroll
          for (int hh = 0; hh < KCH; ++hh) {
            const uint4 v4 = *reinterpret_cast<const uint4*>(kr + koff[hh]);
            wk[rr][4 * hh + 0] = v4.x;
            wk[rr][4 * hh + 1] = v4.y;
            wk[rr][4 * hh + 2] = v4.z;
            wk[rr][4 * hh + 3] = v4.w;
          }
        } else {
          const uint2 v2 = *reinterpret_cast<const uint2*>(kr + koff[0]);
          wk[rr][0] = v2.x;
          wk[rr][1] = v2.y;
        }
      }
      __syncwarp();  // the fp32 metadata table is complete

      // --- scores (log2 units) and Delta for tokens g8, g8+8 of row c4 -------------
      // Each key group's int32 accumulators are folded into the fp32 score as
      // soon as its k-steps are done, so one group's accumulators are live at a time.
      float sg[2][NGK];
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        const int tok = g8 + 8 * sl;
        if constexpr (NGK == 4) {
          const float4 f4 = *reinterpret_cast<const float4*>(ks32 + tok * 4);
          sg[sl][0] = f4.x;
          sg[sl][1] = f4.y;
          sg[sl][2] = f4.z;
          sg[sl][3] = f4.w;
        } else {
#pragma unroll
          for (int g = 0; g < NGK; ++g) sg[sl][g] = ks32[tok * NGK + g];
        }
      }
      float dot[2] = {0.f, 0.f}, dsum[2] = {0.f, 0.f};
#pragma unroll
      for (int g = 0; g < NGK; ++g) {
        int acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
        for (int ks = g * (KG / 32); ks < (g + 1) * (KG / 32); ++ks) {
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
          for (int nt = 0; nt < 2; ++nt) mma_s8(acc[nt], a0, a1, a2, a3, qb[ks][nt][0], qb[ks][nt][1]);
        }
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          // digits 0,1 and 2,3 recombined exactly in int32, then once in fp32
          const int lo = acc[0][2 * sl] + acc[0][2 * sl + 1] * 256 + blo[g];
          const int hi = acc[1][2 * sl] + acc[1][2 * sl + 1] * 256 + bhi[g];
          const float raw = fmaf((float)hi, 65536.f, (float)lo);
          dot[sl] = fmaf(raw, sg[sl][g], dot[sl]);
          dsum[sl] = fmaf(cg[g], sg[sl][g], dsum[sl]);
        }
      }
      float zt[2], dl[2];
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        const bool vt = g8 + 8 * sl < nval;
        float smax = sg[sl][0];   // scales are >= 0
#pragma unroll
        for (int g = 1; g < NGK; ++g) smax = fmaxf(smax, sg[sl][g]);
        zt[sl] = vt ? dot[sl] * zs : -INFINITY;
        dl[sl] = vt ? fmaf(cb, smax, dsum[sl]) : 0.f;
      }
      if constexpr (OUT) {
        // extracted key chunks of tokens g8, g8+8 (their codes are 0): the fp16
        // values' score against q' of row c4, and Delta's share for them, half
        // an fp16 ulp per channel, |k - k16| <= 2^-11 |k16| + 2^-25 (and, for
        // rotated keys, the chunk's norm in the rotation allowance)
        const uint8_t* os = kt + C::OS;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int tok = g8 + 8 * sl;
          const int ck = os[tok];
          if (ck < D / 4 && (FULL || tok < nval)) {
            const uint2 kw = *reinterpret_cast<const uint2*>(os + 2 * kPage + tok * 8);
            const float2 k01 = __half22float2(u32_as_h2(kw.x));
            const float2 k23 = __half22float2(u32_as_h2(kw.y));
            const float4 q4 = reinterpret_cast<const float4*>(sm + C::OFF_QC)[ck * kRows + c4];
            const float d4 = fmaf(q4.w, k23.y, fmaf(q4.z, k23.x, fmaf(q4.y, k01.y, q4.x * k01.x)));
            zt[sl] = fmaf(d4, a.s_att * kLog2e, zt[sl]);
            // sum |q_i| (2^-11 |k_i| + 2^-25) = 2^-11 sum |q_i k_i| + 2^-25 sum |q_i|
            const float qk = fmaf(fabsf(q4.w), fabsf(k23.y),
                                  fmaf(fabsf(q4.z), fabsf(k23.x),
                                       fmaf(fabsf(q4.y), fabsf(k01.y), fabsf(q4.x) * fabsf(k01.x))));
            const float q1 = (fabsf(q4.x) + fabsf(q4.y)) + (fabsf(q4.z) + fabsf(q4.w));
            dl[sl] = fmaf(kKappa * a.s_att, fmaf(qk, 0x1p-11f, q1 * 0x1p-25f), dl[sl]);
            if (a.signs) {   // rotated keys: the chunk's norm (a few ulps of it are in kappa)
              const float kn =
                  fmaf(k23.y, k23.y, fmaf(k23.x, k23.x, fmaf(k01.y, k01.y, k01.x * k01.x)));
              const float cr = rc[(2 + NGK) * kRows + c4];
              dl[sl] = fmaf(cr, kn > 0.f ? kn * rsqrtf(kn) : 0.f, dl[sl]);
            }
          }
        }
      }

      // --- online softmax and bound sums (row c4) -------------------------------
      float mx = fmaxf(zt[0], zt[1]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      // The reference max moves only when the page max exceeds it by more than
      // 2 (log2 units): weights stay <= 4, so w * sV fits fp16 for any finite
      // value scale, and the accumulators are rescaled on few pages.
      const float mref = mx > m2 + 2.0f ? mx : m2;
      const float alpha = ex2(m2 - mref);
      m2 = mref;
      const float w0 = ex2(zt[0] - mref), w1 = ex2(zt[1] - mref);
      // tokens outside the context have w = 0 and Delta = 0
      const float2 d2 = make_float2(dl[0], dl[1]);
      const float2 e2 = mul2(d2, make_float2(kLog2e, kLog2e));
      const float2 ep = make_float2(ex2(e2.x), ex2(e2.y));
      const float2 en = make_float2(ex2(-e2.x), ex2(-e2.y));
      // e^d - 1: below 2^-6 the Taylor series to d^3 (truncation < 2e-7 relative);
      // above it e^d - 1 directly (relative error < 2^-22 * e^d / (e^d - 1) < 2e-5)
      float2 pl = fma2(d2, make_float2(1.0f / 6, 1.0f / 6), make_float2(0.5f, 0.5f));
      pl = fma2(d2, pl, make_float2(1.0f, 1.0f));
      pl = mul2(d2, pl);
      const float em0 = d2.x < 0.015625f ? pl.x : ep.x - 1.0f;
      const float em1 = d2.y < 0.015625f ? pl.y : ep.y - 1.0f;
      const float ta = fmaf(w1, em1, w0 * em0);
      const float tb = fmaf(w1, en.y, w0 * en.x);
      dmax = fmaxf(dmax, fmaxf(d2.x, d2.y));
      const float tw = w0 + w1;
      lsum = fmaf(lsum, alpha, tw);
      Asum = fmaf(Asum, alpha, ta);
      Bsum = fmaf(Bsum, alpha, tb);
      Esum = fmaf(Esum, alpha, tw * eta_cur);

      // --- rescale the PV state when a row max moved --------------------------------
      if (__any_sync(0xffffffffu, alpha != 1.0f)) {
        const int base = lane & ~3;
        const float a0 = __shfl_sync(0xffffffffu, alpha, base | (2 * (c4 & 1)));
        const float a1 = __shfl_sync(0xffffffffu, alpha, base | (2 * (c4 & 1) + 1));
#pragma unroll
        for (int t = 0; t < 2 * NB; ++t) {
          opv[t][0] *= a0;
          opv[t][1] *= a1;
          opv[t][2] *= a0;
          opv[t][3] *= a1;
        }
        zmv[0] *= a0;
        zmv[1] *= a1;
      }

      // --- weights w of tokens c4 + 4k for row hP (the MMA B layout) --------------
      float x[4];
      x[0] = __shfl_sync(0xffffffffu, w0, 4 * c4 + hP);
      x[1] = __shfl_sync(0xffffffffu, w0, 4 * c4 + 16 + hP);
      x[2] = __shfl_sync(0xffffffffu, w1, 4 * c4 + hP);
      x[3] = __shfl_sync(0xffffffffu, w1, 4 * c4 + 16 + hP);

      // --- zero points: sum_j w_j zV_{j,g} on one MMA (rows = groups) -------------
      {
        uint32_t zw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int tok = c4 + 4 * k;
          const uint32_t wv = vm[tok * NB + zgrp];
          // rows g8 >= NB of this MMA are padding (never read): no mask on FULL pages
          zw[k] = FULL || (g8 < NB && tok < nval) ? wv : 0u;
        }
        const uint32_t bz0 = hilo2(make_float2(x[0], x[1]));
        const uint32_t bz1 = hilo2(make_float2(x[2], x[3]));
        mma_f16(zmv, prmt(zw[0], zw[1], 0x7632u), 0u, prmt(zw[2], zw[3], 0x7632u), 0u, bz0, bz1);
      }

      // --- PV: V code stripes (row g8) of tokens c4 + 4k ---------------------------
      uint32_t vw[4][C::VSTR / 4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint8_t* p = rs + voff + 4 * k * C::VRB;
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
        // P' = w * sV of tokens c4 + 4k (zero outside the context), fp16 hi or lo part
        const float4 sv = *reinterpret_cast<const float4*>(vs32 + g * kPage + c4 * 4);
        const uint32_t b01 = hilo2(mul2(make_float2(x[0], x[1]), make_float2(sv.x, sv.y)));
        const uint32_t b23 = hilo2(mul2(make_float2(x[2], x[3]), make_float2(sv.z, sv.w)));
        const int wsel = (2 * g) / 4;            // stripe word holding group g
        const int p = (2 * g) % 4;               // byte offset of group g in that word
        const uint32_t sel = (uint32_t)(p | ((p + 1) << 4) | ((4 + p) << 8) | ((5 + p) << 12));
        const uint32_t r01 = prmt(vw[0][wsel], vw[1][wsel], sel);   // tokens c4, c4+4
        const uint32_t r23 = prmt(vw[2][wsel], vw[3][wsel], sel);   // tokens c4+8, c4+12
        const uint32_t r01s = r01 >> 8, r23s = r23 >> 8;
        mma_f16(opv[2 * g], r01 & 0x000F000Fu, r01s & 0x000F000Fu, r23 & 0x000F000Fu,
                r23s & 0x000F000Fu, b01, b23);
        mma_f16(opv[2 * g + 1], r01 & 0x00F000F0u, r01s & 0x00F000F0u, r23 & 0x00F000F0u,
                r23s & 0x00F000F0u, b01, b23);
      }
      if constexpr (OUT) {
        // extracted value chunks (code 0: the MMAs gave their channels the group
        // zero z), one token at a time: w * (v16 - z) into the accumulators of
        // the chunk's channels, the stored values into the group's range
        const uint8_t* os = kt + C::OS;
        const int cvl = lane < kPage ? os[kPage + lane] : kNoOutlier;
        unsigned pend = __ballot_sync(0xffffffffu, cvl < D / 4 && (FULL || lane < nval));
        while (pend) {
          const int t = __ffs(pend) - 1;
          pend &= pend - 1;
          const int cv = __shfl_sync(0xffffffffu, cvl, t);
          const int gv = cv / 8;   // the chunk's 32-channel group
          const uint2 vw2 = *reinterpret_cast<const uint2*>(os + 2 * kPage + 8 * kPage + t * 8);
          const float2 v01 = __half22float2(u32_as_h2(vw2.x));
          const float2 v23 = __half22float2(u32_as_h2(vw2.y));
          // weights of token t for rows 2 c4 and 2 c4 + 1 (lanes c4 < 2 own them)
          const float wt = t < 8 ? w0 : w1;
          const float wa = __shfl_sync(0xffffffffu, wt, 4 * (t & 7) + 2 * (c4 & 1));
          const float wb = __shfl_sync(0xffffffffu, wt, 4 * (t & 7) + 2 * (c4 & 1) + 1);
          if (g8 == (cv & 7) && c4 < 2) {
            // channel 4 cv + i: m-tile 2 gv + (i & 1), entries 2 (i >> 1) + row
            // parity, in units of 2^-24 (low nibbles) or 2^-20 (high nibbles)
            const float zv = __high2float(u32_as_h2(vm[t * NB + gv]));
            const float d0 = (v01.x - zv) * 0x1p-24f, d1 = (v01.y - zv) * 0x1p-20f;
            const float d2 = (v23.x - zv) * 0x1p-24f, d3 = (v23.y - zv) * 0x1p-20f;
#pragma unroll
            for (int g = 0; g < NB; ++g) {
              if (g == gv) {
                opv[2 * g][0] = fmaf(wa, d0, opv[2 * g][0]);
                opv[2 * g][1] = fmaf(wb, d0, opv[2 * g][1]);
                opv[2 * g][2] = fmaf(wa, d2, opv[2 * g][2]);
                opv[2 * g][3] = fmaf(wb, d2, opv[2 * g][3]);
                opv[2 * g + 1][0] = fmaf(wa, d1, opv[2 * g + 1][0]);
                opv[2 * g + 1][1] = fmaf(wb, d1, opv[2 * g + 1][1]);
                opv[2 * g + 1][2] = fmaf(wa, d3, opv[2 * g + 1][2]);
                opv[2 * g + 1][3] = fmaf(wb, d3, opv[2 * g + 1][3]);
              }
            }
          }
          // the lane whose range entry i covers group gv: (lane * EPL + i) % NB = gv
          if (lane == gv / EPL) {
            const float hi = fmaxf(fmaxf(v01.x, v01.y), fmaxf(v23.x, v23.y));
            const float lo = fminf(fminf(v01.x, v01.y), fminf(v23.x, v23.y));
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
              if (i == gv % EPL) {
                vhi[i] = fmaxf(vhi[i], hi);
                vlo[i] = fminf(vlo[i], lo);
              }
            }
          }
        }
      }
    } else {
      etamax = INFINITY;   // the page was not read
    }
    __syncwarp();
    if (j + S < nloc) issue(j + S, st);
    return true;
  };
  const int last_page = npages - 1;
  uint32_t par = 0;
  bool going = true;
  int jstop = nloc;   // the page whose wait ran out, if one did
  // Full pages (every page but possibly the sequence's last) run through the
  // mask-free step, one copy per ring stage; a partial last page, always this
  // warp's last local page, through one masked copy with a runtime stage.
  const bool last_partial =
      nloc > 0 && n % kPage != 0 && first + (nloc - 1) * kWarps == last_page;
  const int nfull = last_partial ? nloc - 1 : nloc;
  for (int j0 = 0; j0 < nfull && going; j0 += S) {
    static_for<0, S>([&](auto u_c) {
      const int j = j0 + decltype(u_c)::value;
      if (!going || j >= nfull) return;
      going = page_step(u_c, std::true_type{}, j, par);
      if (!going) jstop = j;
    });
    par ^= 1u;
  }
  if (going && last_partial) {
    const int j = nloc - 1;
    going = page_step(j % S, std::false_type{}, j, (uint32_t)((j / S) & 1));
    if (!going) jstop = j;
  }
  // After a wait that ran out, the copies still in flight (pages jstop ..
  // min(jstop + S, nloc) - 1, issued but not consumed) are waited for, each
  // with the same bounded wait, before their stages become the merge area.
  if (!going) {
    for (int j = jstop; j < nloc && j < jstop + S; ++j) {
      static_for<0, S>([&](auto u_c) {
        constexpr int u = decltype(u_c)::value;
        if (j % S == u) (void)mbar_wait(&bar[u], (uint32_t)((j / S) & 1));
      });
    }
  }

  // ---- warp reductions ----------------------------------------------------------
#pragma unroll
  for (int o = 4; o < 32; o *= 2) {
    lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    Asum += __shfl_xor_sync(0xffffffffu, Asum, o);
    Bsum += __shfl_xor_sync(0xffffffffu, Bsum, o);
    Esum += __shfl_xor_sync(0xffffffffu, Esum, o);
    dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
  }
#pragma unroll
  for (int o = 2; o < 32; o *= 2)
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      vhi[i] = fmaxf(vhi[i], __shfl_xor_sync(0xffffffffu, vhi[i], o));
      vlo[i] = fminf(vlo[i], __shfl_xor_sync(0xffffffffu, vlo[i], o));
    }
#pragma unroll
  for (int t = 0; t < 2 * NB; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) opv[t][e] += __shfl_xor_sync(0xffffffffu, opv[t][e], 2);
#pragma unroll
  for (int e = 0; e < 2; ++e) zmv[e] += __shfl_xor_sync(0xffffffffu, zmv[e], 2);

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
        const float f = hn ? 1048576.0f : 16777216.0f;   // 2^20, 2^24
        const int chR = 32 * g + 4 * g8 + hn, chR8 = chR + 2;
        const int h0 = 2 * c4, h1 = 2 * c4 + 1;
        mo[h0 * D + chR] = opv[2 * g + hn][0] * f;
        mo[h1 * D + chR] = opv[2 * g + hn][1] * f;
        mo[h0 * D + chR8] = opv[2 * g + hn][2] * f;
        mo[h1 * D + chR8] = opv[2 * g + hn][3] * f;
      }
    if (g8 < NB) {
      mz[(2 * c4) * NB + g8] = zmv[0];
      mz[(2 * c4 + 1) * NB + g8] = zmv[1];
    }
  }
  if (g8 == 0) {  // lanes 0..3 hold row c4's statistics
    mst[c4 * 8 + 0] = m2;
    mst[c4 * 8 + 1] = lsum;
    mst[c4 * 8 + 2] = Asum;
    mst[c4 * 8 + 3] = Bsum;
    mst[c4 * 8 + 4] = Esum;
    mst[c4 * 8 + 5] = dmax;
  }
  if (lane < 2) {  // lane parity selects the groups of the range entries
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int g = (lane * EPL + i) % NB;
      mr[g] = vhi[i];
      mr[NB + g] = vlo[i];
    }
  }
  if (lane == 0) mr[2 * NB] = etamax;
  __syncthreads();

  // ---- merges: warp r owns query row r ----------------------------------------
  // (1) the CTA's warps -> one record; (2) the last CTA of (b, kvh) merges the
  // records of all splits.  Lane l owns channels [l*CPL, l*CPL + CPL).
  constexpr int CPL = D / 32;
  constexpr int RF = record_floats(D);
  const int r = warp;
  const float* wa = reinterpret_cast<const float*>(sm);   // per-warp areas, MW_FLOATS each
  float mW = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) mW = fmaxf(mW, wa[w * C::MW_FLOATS + kRows * D + r * 8]);
  float st5[5] = {0.f, 0.f, 0.f, 0.f, 0.f};   // l, A, B, E (rescaled), max Delta
  float o[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) o[e] = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float* mwp = wa + w * C::MW_FLOATS;
    const float* stw = mwp + kRows * D + r * 8;
    const float f = stw[0] == -INFINITY ? 0.f : ex2(stw[0] - mW);
#pragma unroll
    for (int t = 0; t < 4; ++t) st5[t] = fmaf(f, stw[1 + t], st5[t]);
    st5[4] = fmaxf(st5[4], stw[5]);
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      const int c = lane * CPL + e;
      o[e] = fmaf(f, mwp[r * D + c] + mwp[kRows * D + kRows * 8 + r * NB + c / 32], o[e]);
    }
  }
  float rg[2 * NB + 1];   // group maxima, group minima, eta
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    rg[g] = -INFINITY;
    rg[NB + g] = INFINITY;
  }
  rg[2 * NB] = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float* rw = wa + w * C::MW_FLOATS + kRows * D + kRows * 8 + kRows * NB;
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      rg[g] = fmaxf(rg[g], rw[g]);
      rg[NB + g] = fminf(rg[NB + g], rw[NB + g]);
    }
    rg[2 * NB] = fmaxf(rg[2 * NB], rw[2 * NB]);
  }

  auto finalize = [&](float l, float A, float Bv, float E, float dm,
                      const float (&rgv)[2 * NB + 1], const float (&ov)[CPL]) {
    if (r >= a.R) return;
    const int qi = r / a.G, h = kvh * a.G + r % a.G;
    const int64_t row = ((int64_t)b * a.nq + qi) * a.hq + h;
    if (a.out) {
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
      for (int e = 0; e < CPL; ++e) a.out[row * D + lane * CPL + e] = ov[e] * inv_l;
    }
    if (lane == 0) {
      // a page of the unit was not read: no certified bound
      const bool skipped = rgv[2 * NB] == INFINITY;
      float bd = skipped ? INFINITY : 0.f;
      if (!skipped && l > 0.f) {
        float range = 0.f;
#pragma unroll
        for (int g = 0; g < NB; ++g) range = fmaxf(range, rgv[g] - rgv[NB + g]);
        const float tv = fminf(tanhf(0.5f * dm), A / Bv);
        bd = kKappa * (tv * (range + 2.0f * rgv[2 * NB]) + E / l);
      }
      a.bound[row] = bd;
      a.flags[row] = skipped || bd > a.tau ? 1 : 0;
    }
  };

  if (active == 1) {  // the only split: finish here
    finalize(st5[0], st5[1], st5[2], st5[3], st5[4], rg, o);
    return;
  }

  // ---- write this split's record; the last CTA of (b, kvh) merges all --------------
  const int64_t unit = (int64_t)b * a.hkv + kvh;
  const int splits = gridDim.y;
  // A unit's records (splits x RF floats) are grouped by kind so the merging CTA
  // reads each kind with neighbouring lanes on neighbouring addresses: headers
  // [split][kHdr], row statistics [row][split][8], outputs [split][row][D].
  float* ubase = a.part + unit * splits * RF;
  float* rec = ubase + (int64_t)split * kHdr;
  float* rst = ubase + (int64_t)splits * kHdr + ((int64_t)r * splits + split) * 8;
  float* rout = ubase + (int64_t)splits * (kHdr + kRows * 8) + ((int64_t)split * kRows + r) * D;
  // header: the value range per group and eta at floats 4..(4 + 2 NB), 16-byte
  // aligned so the merging CTA reads them as whole vectors (the rest is zero)
  constexpr int HV = (2 * NB + 1 + 3) / 4;   // float4 vectors of the header
  static_assert(4 + 4 * HV <= kHdr, "the record header holds the range and eta");
  if (r == 0 && lane < HV) {
    float hv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = 4 * lane + i;
      hv[i] = 0.f;
#pragma unroll
      for (int t = 0; t < 2 * NB + 1; ++t)
        if (t == idx) hv[i] = rg[t];
    }
    reinterpret_cast<float4*>(rec + 4)[lane] = make_float4(hv[0], hv[1], hv[2], hv[3]);
  }
  if (lane == 0) {
    rst[0] = mW;
#pragma unroll
    for (int t = 0; t < 5; ++t) rst[1 + t] = st5[t];
  }
#pragma unroll
  for (int e = 0; e < CPL; ++e) rout[lane * CPL + e] = o[e];
  // The barrier orders every thread's record stores before thread 0's ticket;
  // the ticket's release publishes them at GPU scope and, for the last CTA,
  // its acquire makes every other CTA's records visible to the whole CTA
  // (through the second barrier).
  __syncthreads();
  int* flag = reinterpret_cast<int*>(sm + C::OFF_FLAG);
  if (tid == 0) {
    const int prev = atomic_add_acq_rel(a.counters + unit, 1);
    *flag = prev == active - 1;
  }
  __syncthreads();
  if (!*flag) return;

  // ---- last CTA: merge the records of all active splits, row r per warp -------------
  // Splits are taken in chunks of 32 * KS: lane l reads the statistics of splits
  // c0 + l + 32k together, the chunk's running maximum rescales what came before,
  // and the outputs are read 16 splits at a time (lane l owns CPL channels), each
  // split's weight broadcast from the lane that read its statistics.
  using VT = typename std::conditional<CPL == 4, float4, float2>::type;
  constexpr int KS = 4;
  constexpr int SUB = 16;
  const float* recs = a.part + unit * splits * RF;
  float Mr = -INFINITY;
  float t5[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    rg[g] = -INFINITY;
    rg[NB + g] = INFINITY;
  }
  rg[2 * NB] = 0.f;
#pragma unroll
  for (int e = 0; e < CPL; ++e) o[e] = 0.f;
  auto out_of = [&](int sp) -> const VT* {
    return reinterpret_cast<const VT*>(recs + (int64_t)splits * (kHdr + kRows * 8) +
                                       ((int64_t)sp * kRows + r) * D + lane * CPL);
  };
  for (int c0 = 0; c0 < active; c0 += 32 * KS) {
    float4 sa[KS];  // (m, l, A, B) of split c0 + 32k + lane
    float2 sb[KS];  // (E, max Delta)
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const int sp = c0 + 32 * k + lane;
      sa[k] = make_float4(-INFINITY, 0.f, 0.f, 0.f);
      sb[k] = make_float2(0.f, 0.f);
      if (sp < active) {
        const float* st = recs + (int64_t)splits * kHdr + ((int64_t)r * splits + sp) * 8;
        sa[k] = __ldcg(reinterpret_cast<const float4*>(st));
        sb[k] = __ldcg(reinterpret_cast<const float2*>(st + 4));
        if (r == 0) {   // the header is the same for every row: warp 0 reads it
          const float4* rp = reinterpret_cast<const float4*>(recs + (int64_t)sp * kHdr + 4);
          float hv[4 * HV];
#pragma unroll
          for (int c = 0; c < HV; ++c) {
            const float4 x = __ldcg(rp + c);
            hv[4 * c] = x.x;
            hv[4 * c + 1] = x.y;
            hv[4 * c + 2] = x.z;
            hv[4 * c + 3] = x.w;
          }
#pragma unroll
          for (int g = 0; g < NB; ++g) {
            rg[g] = fmaxf(rg[g], hv[g]);
            rg[NB + g] = fminf(rg[NB + g], hv[NB + g]);
          }
          rg[2 * NB] = fmaxf(rg[2 * NB], hv[2 * NB]);
        }
      }
    }
    // the first outputs of the chunk are read together with its statistics
    VT v0[SUB];
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      const int sp = c0 + i;
      v0[i] = sp < active ? __ldcg(out_of(sp)) : VT{};
    }
    float Mc = -INFINITY;
#pragma unroll
    for (int k = 0; k < KS; ++k) Mc = fmaxf(Mc, sa[k].x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Mc = fmaxf(Mc, __shfl_xor_sync(0xffffffffu, Mc, off));
    const float Mn = fmaxf(Mr, Mc);
    const float sc = Mr == -INFINITY ? 0.f : ex2(Mr - Mn);
    Mr = Mn;
#pragma unroll
    for (int t = 0; t < 4; ++t) t5[t] *= sc;
#pragma unroll
    for (int e = 0; e < CPL; ++e) o[e] *= sc;
    float f[KS], p5[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      f[k] = sa[k].x == -INFINITY ? 0.f : ex2(sa[k].x - Mn);
      p5[0] = fmaf(f[k], sa[k].y, p5[0]);
      p5[1] = fmaf(f[k], sa[k].z, p5[1]);
      p5[2] = fmaf(f[k], sa[k].w, p5[2]);
      p5[3] = fmaf(f[k], sb[k].x, p5[3]);
      p5[4] = fmaxf(p5[4], sb[k].y);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int t = 0; t < 4; ++t) p5[t] += __shfl_xor_sync(0xffffffffu, p5[t], off);
      p5[4] = fmaxf(p5[4], __shfl_xor_sync(0xffffffffu, p5[4], off));
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) t5[t] += p5[t];
    t5[4] = fmaxf(t5[4], p5[4]);
    auto accumulate = [&](int ib, const VT (&v)[SUB]) {
#pragma unroll
      for (int i = 0; i < SUB; ++i) {
        const float fs = __shfl_sync(0xffffffffu, f[(ib + i) / 32], (ib + i) % 32);
        if constexpr (CPL == 4) {
          o[0] = fmaf(fs, v[i].x, o[0]);
          o[1] = fmaf(fs, v[i].y, o[1]);
          o[2] = fmaf(fs, v[i].z, o[2]);
          o[3] = fmaf(fs, v[i].w, o[3]);
        } else {
          o[0] = fmaf(fs, v[i].x, o[0]);
          o[1] = fmaf(fs, v[i].y, o[1]);
        }
      }
    };
    accumulate(0, v0);
#pragma unroll
    for (int ib = SUB; ib < 32 * KS; ib += SUB) {
      if (c0 + ib < active) {  // warp-uniform
        VT v[SUB];
#pragma unroll
        for (int i = 0; i < SUB; ++i) {
          const int sp = c0 + ib + i;
          v[i] = sp < active ? __ldcg(out_of(sp)) : VT{};
        }
        accumulate(ib, v);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      rg[g] = fmaxf(rg[g], __shfl_xor_sync(0xffffffffu, rg[g], off));
      rg[NB + g] = fminf(rg[NB + g], __shfl_xor_sync(0xffffffffu, rg[NB + g], off));
    }
    rg[2 * NB] = fmaxf(rg[2 * NB], __shfl_xor_sync(0xffffffffu, rg[2 * NB], off));
  }
  {  // warp 0's header merge to every warp (the stage buffers are free by now)
    float* rgs = reinterpret_cast<float*>(sm + C::OFF_ST);
    if (r == 0 && lane == 0) {
#pragma unroll
      for (int i = 0; i < 2 * NB + 1; ++i) rgs[i] = rg[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2 * NB + 1; ++i) rg[i] = rgs[i];
  }
  finalize(t5[0], t5[1], t5[2], t5[3], t5[4], rg, o);
  __syncthreads();
  if (tid == 0) a.counters[unit] = 0;  // leave the workspace ready for the next call
}

// One codec's decode variant: the plain and the fused-append kernels.
template <int D, int KB, int KG, bool OUT>
DecodeVariant make_variant() {
  constexpr int S = 3;
  return DecodeVariant{decode_mma_kernel<D, KB, KG, S, false, OUT>,
                       decode_mma_kernel<D, KB, KG, S, true, OUT>,
                       DecodeCfg<D, KB, KG, S, OUT>::SMEM, record_floats(D)};
}

}  // namespace kvq
