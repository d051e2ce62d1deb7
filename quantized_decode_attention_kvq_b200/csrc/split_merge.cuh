// split_merge.cuh -- merging the split records of a split-K decode whose
// splits all write a record (the KQV and HQMQ decodes): the row statistics
// by the log-sum-exp rule across the lanes of a warp, the value-range and eta
// header, and the empty record of a split that holds none of its unit's pages.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

// ---- merge of split records' row statistics ----------------------------------
// One row's (m, l, A, B, E, dmax) of `active` split records, the record of
// split sp at st0 + sp * stride (m = -inf: the split saw none of the row's
// context).  The lanes take splits lane, lane + 32, ... (their loads all in
// flight at once) and then combine by the log-sum-exp rule across the warp;
// every lane returns the merged values.
struct SplitStats {
  float M, l, A, B, E, dm;
};
// m_own (optional) receives m of split `lane`.
__device__ __forceinline__ SplitStats merge_split_stats(const float* st0, int64_t stride,
                                                        int active, int lane,
                                                        float* m_own = nullptr) {
  SplitStats t{-INFINITY, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (m_own) *m_own = -INFINITY;
  for (int sp = lane; sp < active; sp += 32) {
    const float* st = st0 + sp * stride;
    const float ms = __ldcg(st);
    if (m_own && sp == lane) *m_own = ms;
    if (ms == -INFINITY) continue;
    const float Mn = fmaxf(t.M, ms);
    const float fo = t.M == -INFINITY ? 0.f : ex2(t.M - Mn), fs = ex2(ms - Mn);
    t.l = fmaf(t.l, fo, fs * __ldcg(st + 1));
    t.A = fmaf(t.A, fo, fs * __ldcg(st + 2));
    t.B = fmaf(t.B, fo, fs * __ldcg(st + 3));
    t.E = fmaf(t.E, fo, fs * __ldcg(st + 4));
    t.dm = fmaxf(t.dm, __ldcg(st + 5));
    t.M = Mn;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float Mo = __shfl_xor_sync(0xffffffffu, t.M, o);
    const float lo = __shfl_xor_sync(0xffffffffu, t.l, o);
    const float Ao = __shfl_xor_sync(0xffffffffu, t.A, o);
    const float Bo = __shfl_xor_sync(0xffffffffu, t.B, o);
    const float Eo = __shfl_xor_sync(0xffffffffu, t.E, o);
    const float dmo = __shfl_xor_sync(0xffffffffu, t.dm, o);
    const float Mn = fmaxf(t.M, Mo);
    const float f1 = t.M == -INFINITY ? 0.f : ex2(t.M - Mn);
    const float f2 = Mo == -INFINITY ? 0.f : ex2(Mo - Mn);
    t.l = fmaf(t.l, f1, lo * f2);
    t.A = fmaf(t.A, f1, Ao * f2);
    t.B = fmaf(t.B, f1, Bo * f2);
    t.E = fmaf(t.E, f1, Eo * f2);
    t.dm = fmaxf(t.dm, dmo);
    t.M = Mn;
  }
  return t;
}
// The unit's value-range and eta header over `active` split records (record
// sp at ubase + sp * stride: range max [NB], range min [NB], eta max), the
// lanes taking splits lane, lane + 32, ...; lane 0 writes the merged header
// to out[0 .. 2 NB].
template <int NB>
__device__ __forceinline__ void merge_split_header(const float* ubase, int64_t stride, int active,
                                                   int lane, float* out) {
  float hi[NB], lo[NB], eta = 0.f;
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    hi[g] = -INFINITY;
    lo[g] = INFINITY;
  }
  for (int sp = lane; sp < active; sp += 32) {
    const float* h = ubase + sp * stride;
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      hi[g] = fmaxf(hi[g], __ldcg(h + g));
      lo[g] = fminf(lo[g], __ldcg(h + NB + g));
    }
    eta = fmaxf(eta, __ldcg(h + 2 * NB));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      hi[g] = fmaxf(hi[g], __shfl_xor_sync(0xffffffffu, hi[g], o));
      lo[g] = fminf(lo[g], __shfl_xor_sync(0xffffffffu, lo[g], o));
    }
    eta = fmaxf(eta, __shfl_xor_sync(0xffffffffu, eta, o));
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      out[g] = hi[g];
      out[NB + g] = lo[g];
    }
    out[2 * NB] = eta;
  }
}
// The record of a split that holds none of its unit's pages: a neutral header
// (range max -inf, min +inf, eta 0), m = -inf for every row and zero outputs,
// so that a merge may read every split's record.  Called by the whole CTA.
__device__ __forceinline__ void write_empty_record(float* rec, int nb, int hdr, int rows,
                                                   int nout) {
  for (int i = threadIdx.x; i < hdr + rows * 8 + nout; i += blockDim.x) {
    float v = 0.f;
    if (i < hdr)
      v = i < nb ? -INFINITY : (i < 2 * nb ? INFINITY : 0.f);
    else if (i < hdr + rows * 8)
      v = (i - hdr) % 8 == 0 ? -INFINITY : 0.f;
    rec[i] = v;
  }
}
// The weight ex2(m_sp - M) of split base + lane (0 past `active` or for m = -inf).
__device__ __forceinline__ float split_weight(const float* st0, int64_t stride, int active,
                                              int base, int lane, float M) {
  const int sp = base + lane;
  const float ms = sp < active ? __ldcg(st0 + sp * stride) : -INFINITY;
  return ms == -INFINITY ? 0.f : ex2(ms - M);
}


}  // namespace kvq
