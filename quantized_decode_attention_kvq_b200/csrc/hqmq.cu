// hqmq.cu -- the HQMQ codec of "Hurwitz Quaternion Multiplicative Quantization
// for KV Cache Compression" (Method 1-2): every 4-channel chunk of K and V is
// a quaternion split into its radius and its direction on S^3; the direction
// is coded by the product codebook {q_p q_s} of the 24 Hurwitz units (the
// binary tetrahedral group 2T) and a random secondary set per (kv head, role),
// the radius in fp8 E4M3; optionally with Method 3's Med3x chunks kept in
// fp16.  The certified bound of "Runtime-Certified Bounded-Error Quantized
// Attention" (Methodology 2) carries over with a per-token Euclidean key
// error.
//
//   hqmq_append_kernel    one warp per (token, kv head, role) at d = 128 (per
//                         (token, kv head) at d = 64): each lane codes one
//                         (chunk, role) pair (the direction through
//                         y = x conj(q_s) and 2T's closed-form best unit, the
//                         radius by the fp8 conversion; or the chunk in fp16
//                         when Med3x extracts it), then |k|, eps and |v| as
//                         sequential chains over the channels, eta and the
//                         value range
//   hqmq_partial_kernel   grid (sequence x kv head, split), 4 warps, each
//                         streaming its pages through a 2-stage bulk-copy
//                         ring; the CTA builds its kv head's 2 x 24 S
//                         codewords (fp16) in shared memory first.  Scores
//                         with one lane per (token, half of the chunks), PV
//                         with one lane per chunk (packed fp32x2 arithmetic),
//                         online softmax and the bound's sums as for the
//                         other codecs; the extracted chunks' terms in the
//                         Med3x instantiation
//   hqmq_merge_kernel     per (sequence, kv head): the split records' merge,
//                         the output, the bound and the flag
// The arithmetic that decides a code or a stored value (the chunk norm, the
// direction's inner products, the codeword products, the error chains) is the
// fixed-order fp32 sequence the codec's definition gives, so codes, radii,
// norms, eps and eta are bit-identical to a sequential implementation.
#include <cuda_fp8.h>

#include <algorithm>
#include <map>
#include <mutex>

#include "kvq_internal.cuh"
#include "split_merge.cuh"

namespace kvq {
namespace {

// ---------------------------------------------------------------- codebook ---
// unit p of 2T: p = 0..7 the axis units (+-1, +-i, +-j, +-k as 2 n + [negative]),
// p = 8..23 the half units (component n negative when bit n of p - 8 is set)
__device__ __forceinline__ void hq_unit(int p, float a[4]) {
#pragma unroll
  for (int n = 0; n < 4; ++n)
    a[n] = p < 8 ? (n == p / 2 ? ((p & 1) ? -1.f : 1.f) : 0.f)
                 : ((((p - 8) >> n) & 1) ? -0.5f : 0.5f);
}

// codeword i = 24 s + p: the Hamilton product q_p q_s, each component's four
// (exact) term products added left to right
__device__ __forceinline__ float4 hq_codeword(int i, const float4 b) {
  float a[4];
  hq_unit(i % 24, a);
  const float c0 = __fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(a[0], b.x), -__fmul_rn(a[1], b.y)),
                                       -__fmul_rn(a[2], b.z)), -__fmul_rn(a[3], b.w));
  const float c1 = __fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(a[0], b.y), __fmul_rn(a[1], b.x)),
                                       __fmul_rn(a[2], b.w)), -__fmul_rn(a[3], b.z));
  const float c2 = __fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(a[0], b.z), -__fmul_rn(a[1], b.w)),
                                       __fmul_rn(a[2], b.x)), __fmul_rn(a[3], b.y));
  const float c3 = __fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(a[0], b.w), __fmul_rn(a[1], b.z)),
                                       -__fmul_rn(a[2], b.y)), __fmul_rn(a[3], b.x));
  return make_float4(c0, c1, c2, c3);
}

// The direction code of chunk x: for each secondary unit q_s, y = x conj(q_s)
// (each component a sequential fmaf chain over x0..x3); the best axis unit
// gives max_n |y_n| (the first n on ties), the best half unit
// 0.5 (((|y0| + |y1|) + |y2|) + |y3|) with y's signs, taken only when strictly
// larger; a later s wins only when strictly larger.
__device__ __forceinline__ int hq_direction(const float x[4], const float4* sec, int S) {
  int best = 0;
  float bv = -INFINITY;
#pragma unroll 4
  for (int s = 0; s < S; ++s) {
    const float4 b = sec[s];
    const float y0 = __fmaf_rn(x[3], b.w, __fmaf_rn(x[2], b.z, __fmaf_rn(x[1], b.y, __fmul_rn(x[0], b.x))));
    const float y1 = __fmaf_rn(x[3], b.z, __fmaf_rn(-x[2], b.w, __fmaf_rn(x[1], b.x, __fmul_rn(-x[0], b.y))));
    const float y2 = __fmaf_rn(-x[3], b.y, __fmaf_rn(x[2], b.x, __fmaf_rn(x[1], b.w, __fmul_rn(-x[0], b.z))));
    const float y3 = __fmaf_rn(x[3], b.x, __fmaf_rn(x[2], b.y, __fmaf_rn(-x[1], b.z, __fmul_rn(-x[0], b.w))));
    const float a0 = fabsf(y0), a1 = fabsf(y1), a2 = fabsf(y2), a3 = fabsf(y3);
    int n0 = 0;
    float v = a0, yn = y0;
    if (a1 > v) { n0 = 1; v = a1; yn = y1; }
    if (a2 > v) { n0 = 2; v = a2; yn = y2; }
    if (a3 > v) { n0 = 3; v = a3; yn = y3; }
    int p = 2 * n0 + (yn < 0.f ? 1 : 0);
    const float h = __fmul_rn(0.5f, __fadd_rn(__fadd_rn(__fadd_rn(a0, a1), a2), a3));
    if (h > v) {
      v = h;
      p = 8 + (y0 < 0.f ? 1 : 0) + (y1 < 0.f ? 2 : 0) + (y2 < 0.f ? 4 : 0) + (y3 < 0.f ? 8 : 0);
    }
    if (v > bv) {
      bv = v;
      best = 24 * s + p;
    }
  }
  return best;
}

// the reconstruction's codeword: each component rounded to fp16 (nearest even)
__device__ __forceinline__ float4 hq_round16(const float4 c) {
  return make_float4(__half2float(__float2half_rn(c.x)), __half2float(__float2half_rn(c.y)),
                     __half2float(__float2half_rn(c.z)), __half2float(__float2half_rn(c.w)));
}
// the same as the decode's table entry: four fp16 in two words
__device__ __forceinline__ uint2 hq_pack16(const float4 c) {
  return make_uint2(h2_as_u32(__floats2half2_rn(c.x, c.y)), h2_as_u32(__floats2half2_rn(c.z, c.w)));
}
__device__ __forceinline__ float4 hq_unpack16(const uint2 w) {
  const float2 a = __half22float2(u32_as_h2(w.x)), b = __half22float2(u32_as_h2(w.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// fp8 E4M3: round to nearest even, saturating at 448; and back (exact)
__device__ __forceinline__ uint32_t e4m3_rn(float r) {
  return (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}

// Med3x (Method 3) over one vector whose NCH chunk norms are held one per
// lane by an aligned group of NCH lanes (the warp, or a half-warp): the chunk
// with the largest norm above 3 x the median (0.5 (a + b) of the two middle
// norms; equal norms ranked by chunk index), -1 for none or when a norm is NaN.
// Every lane of the warp runs every shuffle and ballot (the two half-warps'
// groups may have different answers), and the answer is chosen at the end.
template <int NCH>
__device__ __forceinline__ int med3_group(float r, int lane) {
  const int c = lane % NCH, g0 = lane - c;
  const unsigned gmask = NCH == 32 ? 0xffffffffu : (0xffffu << g0);
  const bool any_nan = (__ballot_sync(0xffffffffu, isnan(r)) & gmask) != 0u;
  int rank = 0;
#pragma unroll 8
  for (int j = 0; j < NCH; ++j) {
    const float rj = __shfl_sync(0xffffffffu, r, j, NCH);
    rank += (rj < r) || (rj == r && j < c);
  }
  const unsigned lo_l = __ballot_sync(0xffffffffu, rank == NCH / 2 - 1) & gmask;
  const unsigned hi_l = __ballot_sync(0xffffffffu, rank == NCH / 2) & gmask;
  // (a group with a NaN norm may have no such lanes: any lane will do, the
  // answer is -1 then)
  const float a = __shfl_sync(0xffffffffu, r, lo_l ? __ffs(lo_l) - 1 : g0);
  const float b = __shfl_sync(0xffffffffu, r, hi_l ? __ffs(hi_l) - 1 : g0);
  const float thr = __fmul_rn(3.0f, __fmul_rn(0.5f, __fadd_rn(a, b)));
  float best = r > thr ? r : -1.0f;   // norms are >= 0
#pragma unroll
  for (int o = 1; o < NCH; o *= 2) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
  const unsigned who = __ballot_sync(0xffffffffu, r > thr && r == best) & gmask;
  return any_nan || best < 0.0f || who == 0u ? -1 : __ffs(who) - 1 - g0;
}

}  // namespace

// ================================================================ append =====
// One warp per item, 4 warps per CTA looping over the items.  At d = 128 an
// item is one role of one (token, kv head), lane l coding chunk l, so K and V
// search in parallel warps; at d = 64 an item is the (token, kv head), lane l
// coding (chunk l % 16, role l / 16).
constexpr int kHqAppendWarps = 4;

template <int D>
__global__ void __launch_bounds__(kHqAppendWarps * 32) hqmq_append_kernel(const HqAppendArgs ha) {
  constexpr int NC = D / 4;
  constexpr bool SPLIT = NC == 32;   // one role per item
  constexpr int GL = 8;              // lanes per 32-channel group of V chunks
  const AppendArgs& a = ha.a;
  const HqLayout L{D, ha.outliers};
  const int S = ha.S;
  __shared__ __align__(16) float stg[kHqAppendWarps][3][D];   // per warp: k, k - k^, v
  __shared__ float4 ssec[kHqAppendWarps][2 * KVQ_HQMQ_MAX_S];  // per warp: the item's units
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float* xk = stg[w][0];
  float* ek = stg[w][1];
  float* xv = stg[w][2];
  const int64_t total = (int64_t)a.num_seqs * a.num_tokens * a.hkv * (SPLIT ? 2 : 1);
  for (int64_t item = (int64_t)blockIdx.x * kHqAppendWarps + w; item < total;
       item += (int64_t)gridDim.x * kHqAppendWarps) {
    const int rsel = SPLIT ? (int)(item & 1) : 0;   // the item's role when split
    const int64_t it = SPLIT ? item >> 1 : item;
    const int h = (int)(it % a.hkv);
    const int t = (int)((it / a.hkv) % a.num_tokens);
    const int s = (int)(it / ((int64_t)a.hkv * a.num_tokens));
    if (a.valid && t >= a.valid[s]) continue;
    const int pos = a.start_pos[s] + t;
    const int lp = pos / kPage;
    if (pos < 0 || lp >= a.max_pages) {
      if (lane == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
      continue;
    }
    const int page = a.page_table[(int64_t)s * a.max_pages + lp];
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
      continue;
    }
    const int slot = pos % kPage;
    const int64_t base = s * a.seq_stride + h * a.head_stride + (int64_t)t * a.tok_stride;
    uint8_t* blk = a.pool + ((int64_t)page * a.hkv + h) * L.bytes();
    const bool has_k = !SPLIT || rsel == 0, has_v = !SPLIT || rsel == 1;
    __syncwarp();   // the previous item's chains and searches have read the staging rows
    {   // the item's secondary units (its role's, or K's then V's) in one coalesced load
      const float4* src = reinterpret_cast<const float4*>(ha.sec) + (int64_t)h * 2 * S +
                          (SPLIT ? rsel * S : 0);
      for (int i = lane; i < (SPLIT ? S : 2 * S); i += 32) ssec[w][i] = __ldg(src + i);
    }
    __syncwarp();
    const int role = SPLIT ? rsel : lane / 16;
    const int ch = SPLIT ? lane : lane % 16;
    const float4* secs = ssec[w] + (SPLIT ? 0 : role * S);
    float x[4];
#pragma unroll
    for (int n = 0; n < 4; ++n) x[n] = load_elem(role ? a.v : a.k, a.in_bf16, base + 4 * ch + n);
    bool fin = true;
#pragma unroll
    for (int n = 0; n < 4; ++n) fin = fin && isfinite(x[n]);
    const float r = __fsqrt_rn(__fadd_rn(__fadd_rn(__fmul_rn(x[0], x[0]), __fmul_rn(x[1], x[1])),
                                         __fadd_rn(__fmul_rn(x[2], x[2]), __fmul_rn(x[3], x[3]))));
    // Med3x: the vector's extracted chunk (its lanes are this item's, or this
    // half-warp's at d = 64)
    const int cx = ha.outliers ? med3_group<SPLIT ? 32 : 16>(r, lane) : -1;
    const bool ext = cx == ch;
    int code = 0;
    uint32_t rq = 0;
    const bool rok = ext || isfinite(r);
    if (!ext && rok) {
      code = hq_direction(x, secs, S);
      rq = e4m3_rn(r);
    }
    reinterpret_cast<uint16_t*>(blk + (role ? L.vi() : 0))[kPage * ch + slot] = (uint16_t)code;
    blk[(role ? L.vr() : L.kr()) + kPage * ch + slot] = (uint8_t)rq;
    const float4 cw = hq_round16(hq_codeword(code, secs[code / 24]));
    const float rv = e4m3_value(rq);
    float xh[4] = {__fmul_rn(rv, cw.x), __fmul_rn(rv, cw.y), __fmul_rn(rv, cw.z),
                   __fmul_rn(rv, cw.w)};
    bool bad16 = false;
    if (ha.outliers) {
      // the extracted chunk in fp16 (a value that is not finite or beyond
      // 65504 is stored as 0 and is a range error); the section's chunk index
      // and values are written for every token (zeros when none)
      uint8_t* os = blk + L.out_off();
      if (ch == 0) os[role * kPage + slot] = cx < 0 ? (uint8_t)kNoOutlier : (uint8_t)cx;
      if (ch == (cx < 0 ? 0 : cx)) {
        __half hv[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          hv[n] = __float2half_rn(0.f);
          if (ext) {
            if (!isfinite(x[n]) || fabsf(x[n]) > 65504.0f)
              bad16 = true;
            else
              hv[n] = __float2half_rn(x[n]);
            xh[n] = __half2float(hv[n]);
          }
        }
        *reinterpret_cast<uint2*>(os + 2 * kPage + role * kPage * 8 + slot * 8) =
            make_uint2(h2_as_u32(__halves2half2(hv[0], hv[1])), h2_as_u32(__halves2half2(hv[2], hv[3])));
      }
    }
    float err = 0.f, hi = 0.f, lo = 0.f;
    if (role == 0) {
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        xk[4 * ch + n] = x[n];
        ek[4 * ch + n] = __fsub_rn(x[n], xh[n]);
      }
    } else {
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        xv[4 * ch + n] = x[n];
        err = fmaxf(err, fabsf(__fsub_rn(x[n], xh[n])));
        hi = fmaxf(hi, xh[n]);
        lo = fminf(lo, xh[n]);
      }
    }
    const bool bad_k = __any_sync(0xffffffffu, role == 0 && !fin);
    const bool bad_v = __any_sync(0xffffffffu, role == 1 && !fin);
    const bool bad_r = __any_sync(0xffffffffu, !rok || bad16);
#pragma unroll
    for (int o = 1; o < 32; o *= 2) err = fmaxf(err, __shfl_xor_sync(0xffffffffu, err, o));
#pragma unroll
    for (int o = 1; o < GL; o *= 2) {
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    }
    __syncwarp();
    // |k|, |k - k^| and |v|: sequential chains over the channels
    float nk2 = 0.f, e2 = 0.f, nv2 = 0.f;
    if (has_k) {
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(xk + c);
        const float4 e4 = *reinterpret_cast<const float4*>(ek + c);
        nk2 = __fmaf_rn(k4.w, k4.w, __fmaf_rn(k4.z, k4.z, __fmaf_rn(k4.y, k4.y, __fmaf_rn(k4.x, k4.x, nk2))));
        e2 = __fmaf_rn(e4.w, e4.w, __fmaf_rn(e4.z, e4.z, __fmaf_rn(e4.y, e4.y, __fmaf_rn(e4.x, e4.x, e2))));
      }
    }
    if (has_v) {
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 v4 = *reinterpret_cast<const float4*>(xv + c);
        nv2 = __fmaf_rn(v4.w, v4.w, __fmaf_rn(v4.z, v4.z, __fmaf_rn(v4.y, v4.y, __fmaf_rn(v4.x, v4.x, nv2))));
      }
    }
    if (lane == 0) {
      if (bad_k || bad_v || bad_r) set_error(a.err, KVQ_ERR_RANGE);
      int* eta = reinterpret_cast<int*>(a.eta + (int64_t)page * a.hkv + h);
      if (has_k) {
        const float en = __fsqrt_rn(e2);
        reinterpret_cast<float*>(blk + L.kn())[slot] = __fsqrt_rn(nk2);
        reinterpret_cast<float*>(blk + L.ke())[slot] =
            bad_k ? INFINITY : nextafterf(__fmaf_rn(en, 0x1p-16f, en), INFINITY);
        // a non-finite key makes the token's eta +inf (its value warp cannot see it)
        if (SPLIT && bad_k) atomicMax(eta, __float_as_int(INFINITY));
      }
      if (has_v) {
        const float eu = bad_v || (!SPLIT && bad_k)
                             ? INFINITY
                             : nextafterf(__fmaf_rn(0x1p-16f, __fsqrt_rn(nv2), err), INFINITY);
        atomicMax(eta, __float_as_int(eu));
      }
    }
    // the V chunks' 32-channel groups: lanes 8 g .. 8 g + 7 of a value item
    // (d 128), or 16 + 8 g .. (d 64); the block's range starts at [0, 0]
    const int vlane = SPLIT ? (rsel == 1 ? lane : -1) : lane - 16;
    if (vlane >= 0 && vlane % GL == 0) {
      float* rg = reinterpret_cast<float*>(blk + L.rg()) + 2 * (vlane / GL);
      if (hi > 0.f) atomicMax(reinterpret_cast<int*>(rg), __float_as_int(hi));
      if (lo < 0.f) atomicMax(reinterpret_cast<unsigned int*>(rg + 1), __float_as_uint(lo));
    }
  }
}

template <int D>
cudaError_t launch_hqmq_append_d(const HqAppendArgs& a, cudaStream_t stream) {
  static std::mutex mu;
  static std::map<int, int> sms_of;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = sms_of.find(dev);
    if (it == sms_of.end()) {
      if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
      it = sms_of.emplace(dev, sms).first;
    }
    sms = it->second;
  }
  const int64_t items = (int64_t)a.a.num_seqs * a.a.num_tokens * a.a.hkv * (D == 128 ? 2 : 1);
  const int64_t blocks = std::min<int64_t>((items + kHqAppendWarps - 1) / kHqAppendWarps, 8 * sms);
  hqmq_append_kernel<D><<<(unsigned)blocks, kHqAppendWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_hqmq_append(const HqAppendArgs& a, int d, cudaStream_t stream) {
  const int64_t items = (int64_t)a.a.num_seqs * a.a.num_tokens * a.a.hkv;
  if (items == 0) return cudaSuccess;
  if (d == 128) return launch_hqmq_append_d<128>(a, stream);
  if (d == 64) return launch_hqmq_append_d<64>(a, stream);
  return cudaErrorInvalidValue;
}

// ================================================================ decode =====
constexpr int kHqWarps = 4;
constexpr int kHqRows = 4;
constexpr int kHqStages = 2;
constexpr int kHqHdr = 16;   // floats: range max [NB], range min [NB], eta max
__host__ __device__ constexpr int hq_rec_floats(int d) { return kHqHdr + kHqRows * 8 + kHqRows * d; }

template <int D, bool OUT>
struct HqCfg {
  static constexpr int NC = D / 4;
  static constexpr int BLOCK = 24 * D + 8 * kPage + D / 4 + (OUT ? kOutBytes : 0);   // HqLayout bytes()
  static constexpr int OFF_ST = 0;                                          // [warp][stage][BLOCK]
  static constexpr int OFF_W = OFF_ST + kHqWarps * kHqStages * BLOCK;       // [warp][16][4] f32
  static constexpr int OFF_Q = OFF_W + kHqWarps * kPage * kHqRows * 4;      // q [chunk][row] float4
  static constexpr int OFF_QN = OFF_Q + NC * kHqRows * 16;                  // |q|_2 [4]
  static constexpr int OFF_BAR = (OFF_QN + 16 + 15) / 16 * 16;              // [warp][stage] u64
  static constexpr int OFF_PG = OFF_BAR + kHqWarps * kHqStages * 8;         // [warp][stage] i32
  static constexpr int OFF_TAB = (OFF_PG + kHqWarps * kHqStages * 4 + 15) / 16 * 16;  // [2][24 S] 4 x fp16
  // merge of the CTA's warps (aliases the stages): per warp [4][D], [4][8], header
  static constexpr int MW = kHqRows * D + kHqRows * 8 + kHqHdr;
  static constexpr int MERGE = kHqWarps * MW * 4;
  static_assert(MERGE <= OFF_W, "the merge area must stay inside the stages");
  static_assert(BLOCK % 16 == 0, "bulk copies move multiples of 16 bytes");
  static __host__ __device__ constexpr int smem(int S) { return 128 + OFF_TAB + 2 * 24 * S * 8; }
};

template <int D, bool OUT>
__global__ void __launch_bounds__(kHqWarps * 32, 4) hqmq_partial_kernel(const HqDecodeArgs ha) {
  using C = HqCfg<D, OUT>;
  constexpr int NC = C::NC, NB = D / 32, E = D / 32;
  constexpr int HC = NC / 2;          // chunks per half-warp in the scores
  constexpr int TPL = 16 * NC / 32;   // tokens per lane in PV
  const DecodeArgs& a = ha.a;
  const HqLayout L{D, OUT ? 1 : 0};
  const int S = ha.S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  const int split = blockIdx.y, kvh = blockIdx.x % a.hkv, b = blockIdx.x / a.hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR) + warp * kHqStages;
  int* spage = reinterpret_cast<int*>(sm + C::OFF_PG) + warp * kHqStages;
  if (lane == 0) {
    for (int s = 0; s < kHqStages; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }
  int n = a.seq_lens[b];
  if (n < 0) n = 0;
  const bool clamped = n > a.max_pages * kPage;
  if (clamped) {
    if (tid == 0) set_error(a.err, KVQ_ERR_INVALID_ARG);
    n = a.max_pages * kPage;
  }
  const int npages = (n + kPage - 1) / kPage;
  const int p0 = split * a.pps;
  if (p0 >= npages) {   // a split past the context: an empty record for the merge
    write_empty_record(a.part + ((int64_t)blockIdx.x * gridDim.y + split) * hq_rec_floats(D), NB,
                       kHqHdr, kHqRows, kHqRows * D);
    return;
  }
  const int p1 = min(npages, p0 + a.pps);

  // ---- pages of this warp: p0 + warp, p0 + warp + 4, ...; the first copies
  // go out before the tables are built ----
  const int first = p0 + warp;
  const int nloc = first < p1 ? (p1 - first + kHqWarps - 1) / kHqWarps : 0;
  uint8_t* stage0 = sm + C::OFF_ST + warp * kHqStages * C::BLOCK;
  const int32_t* ptab = a.page_table + (int64_t)b * a.max_pages;
  int pt_chunk = -1, pt_val = -1;
  auto issue = [&](int j, int st) {
    if ((j >> 5) != pt_chunk) {
      pt_chunk = j >> 5;
      const int jl = 32 * pt_chunk + lane;
      pt_val = jl < nloc ? __ldg(ptab + first + jl * kHqWarps) : -1;
    }
    const int pgv = __shfl_sync(0xffffffffu, pt_val, j & 31);
    if (lane == 0) {
      const bool ok = pgv >= 0 && pgv < a.num_pages;
      spage[st] = ok ? pgv : -1;
      if (ok) {
        mbar_arrive_expect_tx(&bar[st], C::BLOCK);
        bulk_g2s_hint(stage0 + st * C::BLOCK, a.pool + ((int64_t)pgv * a.hkv + kvh) * C::BLOCK,
                      C::BLOCK, &bar[st], l2_evict_first_policy());
      } else {
        set_error(a.err, KVQ_ERR_INVALID_ARG);
        mbar_arrive(&bar[st]);
      }
    }
    __syncwarp();
  };
  __syncwarp();   // the barriers are initialized
  for (int j = 0; j < kHqStages && j < nloc; ++j) issue(j, j);

  // ---- the kv head's codewords in fp16, K then V: [2][24 S] ----
  uint2* tab = reinterpret_cast<uint2*>(sm + C::OFF_TAB);
  {
    const float4* secs = reinterpret_cast<const float4*>(ha.sec) + (int64_t)kvh * 2 * S;
    for (int i = tid; i < 48 * S; i += blockDim.x) {
      const int role = i / (24 * S), ci = i - role * 24 * S;
      tab[i] = hq_pack16(hq_codeword(ci, __ldg(secs + role * S + ci / 24)));
    }
  }
  // ---- query rows (warp r = row r): q [chunk][row] as float4, |q|_2 ----
  float4* qs = reinterpret_cast<float4*>(sm + C::OFF_Q);
  float* qn = reinterpret_cast<float*>(sm + C::OFF_QN);
  {
    const int r = warp;
    float x[E];
    if (r < a.R) {
      const int qi = r / a.G, hq = kvh * a.G + r % a.G;
      const int64_t e0 = (((int64_t)b * a.nq + qi) * a.hq + hq) * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = load_elem(a.q, a.q_bf16, e0 + e);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = 0.f;
    }
    float l2 = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = lane * E + e;
      reinterpret_cast<float*>(qs + (c / 4) * kHqRows + r)[c % 4] = x[e];
      l2 = fmaf(x[e], x[e], l2);
    }
#pragma unroll
    for (int o = 1; o < 32; o *= 2) l2 += __shfl_xor_sync(0xffffffffu, l2, o);
    if (lane == 0) qn[r] = sqrtf(l2);
  }
  __syncthreads();
  const uint2* tabK = tab;
  const uint2* tabV = tab + 24 * S;
  // a code beyond the table (only a pool not written by this codec holds one)
  // reads the last codeword instead of memory past the table
  const int ncw = 24 * S;
  // scores: lane (token t, chunk half hc) takes rows r0 = 2 hc, r0 + 1 after
  // the halves are combined
  const int t = lane & 15, hc = lane >> 4, r0 = 2 * hc;
  float cq1[2], cq2[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    cq1[k] = kKappa * a.s_att * qn[r0 + k];
    cq2[k] = kKappa * a.s_att * kRotSlack * qn[r0 + k];
  }
  const float zsc = a.s_att * kLog2e;
  // PV: lane owns chunk pc for tokens t0 .. t0 + TPL - 1
  const int pc = lane % NC, t0 = (lane / NC) * TPL;

  // PV accumulators: row r, channels (0, 1) and (2, 3) of the lane's chunk,
  // each pair one packed fp32x2 register
  float2 acc[kHqRows][2];
#pragma unroll
  for (int r = 0; r < kHqRows; ++r) acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
  float m2[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f}, Asum[2] = {0.f, 0.f},
        Bsum[2] = {0.f, 0.f}, Esum[2] = {0.f, 0.f}, dmax[2] = {0.f, 0.f};
  float rhi[NB], rlo[NB], etamax = clamped ? INFINITY : 0.f;
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    rhi[g] = -INFINITY;
    rlo[g] = INFINITY;
  }
  // the page's weights [token][row]
  float* wts = reinterpret_cast<float*>(sm + C::OFF_W) + warp * kPage * kHqRows;
  int jstop = nloc;
  for (int j = 0; j < nloc; ++j) {
    const int st = j % kHqStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&bar[st], (uint32_t)((j / kHqStages) & 1)))) {
      if (lane == 0) set_error(a.err, KVQ_ERR_TIMEOUT);
      etamax = INFINITY;
      jstop = j;
      break;
    }
    const int pg = spage[st];
    if (pg < 0) {
      etamax = INFINITY;   // the page was not read
    } else {
      const uint8_t* blk = stage0 + st * C::BLOCK;
      const float* fk = reinterpret_cast<const float*>(blk + L.kn());
      const float* fe = reinterpret_cast<const float*>(blk + L.ke());
      const float* frg = reinterpret_cast<const float*>(blk + L.rg());
      const int nval = min(kPage, n - (first + j * kHqWarps) * kPage);
      const float eta_pg = __ldg(a.eta + (int64_t)pg * a.hkv + kvh);
      etamax = fmaxf(etamax, eta_pg);
#pragma unroll
      for (int g = 0; g < NB; ++g) {
        rhi[g] = fmaxf(rhi[g], frg[2 * g]);
        rlo[g] = fminf(rlo[g], frg[2 * g + 1]);
      }
      // ---- scores: q . k^ of token t over half hc of the chunks (the upper
      // half starts one chunk later, so the two halves' loads fall in
      // different banks) ----
      // per row: the channel pairs (0, 1) and (2, 3) summed as packed fp32x2
      float2 s2[kHqRows];
#pragma unroll
      for (int r = 0; r < kHqRows; ++r) s2[r] = make_float2(0.f, 0.f);
      {
        const uint16_t* kidx = reinterpret_cast<const uint16_t*>(blk);
        const uint8_t* krad = blk + L.kr();
#pragma unroll 4
        for (int cc = 0; cc < HC; ++cc) {
          const int c = hc ? HC + (cc + 1) % HC : cc;
          const int idx = min((int)kidx[kPage * c + t], ncw - 1);
          const float rv = e4m3_value(krad[kPage * c + t]);
          const float4 cw = hq_unpack16(tabK[idx]);
          const float2 rr = make_float2(rv, rv);
          const float2 k01 = mul2(make_float2(cw.x, cw.y), rr);   // exact products
          const float2 k23 = mul2(make_float2(cw.z, cw.w), rr);
#pragma unroll
          for (int r = 0; r < kHqRows; ++r) {
            const float4 qv = qs[c * kHqRows + r];
            s2[r] = fma2(make_float2(qv.x, qv.y), k01, s2[r]);
            s2[r] = fma2(make_float2(qv.z, qv.w), k23, s2[r]);
          }
        }
      }
      if constexpr (OUT) {
        // token t's extracted key chunk, kept in fp16 (its code and radius are
        // 0): its score term, added by the half-warp whose chunks hold it
        const uint8_t* os = blk + L.out_off();
        const int cx = os[t];
        if (cx < NC && (hc ? cx >= HC : cx < HC)) {
          const float4 k16 = hq_unpack16(*reinterpret_cast<const uint2*>(os + 2 * kPage + t * 8));
#pragma unroll
          for (int r = 0; r < kHqRows; ++r) {
            const float4 qv = qs[cx * kHqRows + r];
            s2[r] = fma2(make_float2(qv.x, qv.y), make_float2(k16.x, k16.y), s2[r]);
            s2[r] = fma2(make_float2(qv.z, qv.w), make_float2(k16.z, k16.w), s2[r]);
          }
        }
      }
      float s4[kHqRows];
#pragma unroll
      for (int r = 0; r < kHqRows; ++r) {
        s4[r] = s2[r].x + s2[r].y;
        s4[r] += __shfl_xor_sync(0xffffffffu, s4[r], 16);
      }
      const bool vt = t < nval;
      float zt[2], dl[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float sk = hc ? s4[2 + k] : s4[k];
        zt[k] = vt ? sk * zsc : -INFINITY;
        dl[k] = vt ? fmaf(cq1[k], fe[t], cq2[k] * fk[t]) : 0.f;
      }
      // ---- online softmax and the bound's sums, rows r0 + k ----
      float alpha[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float mx = zt[k];
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        const float mref = mx > m2[k] + 2.0f ? mx : m2[k];
        alpha[k] = ex2(m2[k] - mref);
        m2[k] = mref;
        const float wv = ex2(zt[k] - mref);
        const float d = dl[k];
        const float ed = ex2(d * kLog2e), en = ex2(-d * kLog2e);
        const float em = d < 0.015625f ? d * fmaf(d, fmaf(d, 1.0f / 6, 0.5f), 1.0f) : ed - 1.0f;
        lsum[k] = fmaf(lsum[k], alpha[k], wv);
        Asum[k] = fmaf(Asum[k], alpha[k], wv * em);
        Bsum[k] = fmaf(Bsum[k], alpha[k], wv * en);
        Esum[k] = fmaf(Esum[k], alpha[k], wv * eta_pg);
        dmax[k] = fmaxf(dmax[k], d);
        wts[t * 4 + r0 + k] = wv;   // 0 outside the context
      }
      if (__any_sync(0xffffffffu, alpha[0] != 1.0f || alpha[1] != 1.0f)) {
#pragma unroll
        for (int r = 0; r < kHqRows; ++r) {
          // row r's factor sits in the lanes of half r / 2, slot r % 2
          const float ar = __shfl_sync(0xffffffffu, alpha[r & 1], 16 * (r >> 1));
#pragma unroll
          for (int h = 0; h < 2; ++h) acc[r][h] = mul2(acc[r][h], make_float2(ar, ar));
        }
      }
      __syncwarp();
      // ---- PV: chunk pc of tokens t0 .. t0 + TPL - 1 ----
      {
        const uint16_t* vidx = reinterpret_cast<const uint16_t*>(blk + L.vi()) + kPage * pc + t0;
        const uint8_t* vrad = blk + L.vr() + kPage * pc + t0;
        uint32_t iw[TPL / 2], rw[TPL / 4];
#pragma unroll
        for (int i = 0; i < TPL / 8; ++i) {
          const uint4 v4 = reinterpret_cast<const uint4*>(vidx)[i];
          iw[4 * i] = v4.x;
          iw[4 * i + 1] = v4.y;
          iw[4 * i + 2] = v4.z;
          iw[4 * i + 3] = v4.w;
        }
        if constexpr (TPL == 16) {
          const uint4 r4 = *reinterpret_cast<const uint4*>(vrad);
          rw[0] = r4.x;
          rw[1] = r4.y;
          rw[2] = r4.z;
          rw[3] = r4.w;
        } else {
          const uint2 r2 = *reinterpret_cast<const uint2*>(vrad);
          rw[0] = r2.x;
          rw[1] = r2.y;
        }
        const float4* w4p = reinterpret_cast<const float4*>(wts) + t0;
#pragma unroll
        for (int tt = 0; tt < TPL; ++tt) {
          const int idx = min((int)((iw[tt / 2] >> (16 * (tt & 1))) & 0xFFFFu), ncw - 1);
          const float rv = e4m3_value((rw[tt / 4] >> (8 * (tt & 3))) & 0xFFu);
          const float4 cw = hq_unpack16(tabV[idx]);
          const float2 rr = make_float2(rv, rv);
          const float2 v01 = mul2(make_float2(cw.x, cw.y), rr);   // exact products
          const float2 v23 = mul2(make_float2(cw.z, cw.w), rr);
          const float4 w4 = w4p[tt];   // one load; the pairs (w, w) are built in registers
          const float2 w2[kHqRows] = {make_float2(w4.x, w4.x), make_float2(w4.y, w4.y),
                                      make_float2(w4.z, w4.z), make_float2(w4.w, w4.w)};
#pragma unroll
          for (int r = 0; r < kHqRows; ++r) {
            acc[r][0] = fma2(w2[r], v01, acc[r][0]);
            acc[r][1] = fma2(w2[r], v23, acc[r][1]);
          }
        }
        if constexpr (OUT) {
          // extracted value chunks (code and radius 0) of this lane's chunk:
          // w * v16 for those tokens
          const uint8_t* os = blk + L.out_off();
#pragma unroll
          for (int tt = 0; tt < TPL; ++tt) {
            const int tk = t0 + tt;
            if (os[kPage + tk] == pc) {
              const float4 v16 =
                  hq_unpack16(*reinterpret_cast<const uint2*>(os + 2 * kPage + kPage * 8 + tk * 8));
              const float4 w4 = w4p[tt];
              const float wr[kHqRows] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
              for (int r = 0; r < kHqRows; ++r) {
                const float2 w2 = make_float2(wr[r], wr[r]);
                acc[r][0] = fma2(w2, make_float2(v16.x, v16.y), acc[r][0]);
                acc[r][1] = fma2(w2, make_float2(v16.z, v16.w), acc[r][1]);
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (j + kHqStages < nloc) issue(j + kHqStages, st);
  }
  // after a wait that ran out, the copies still in flight are waited for
  // (bounded) before the stages become the merge area
  if (jstop < nloc)
    for (int j = jstop; j < nloc && j < jstop + kHqStages; ++j)
      (void)mbar_wait(&bar[j % kHqStages], (uint32_t)((j / kHqStages) & 1));

  // ---- per-warp sums: the rows' lanes (one half-warp each); at d = 64 the
  // two token halves of each chunk ----
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int o = 1; o < 16; o *= 2) {
      lsum[k] += __shfl_xor_sync(0xffffffffu, lsum[k], o);
      Asum[k] += __shfl_xor_sync(0xffffffffu, Asum[k], o);
      Bsum[k] += __shfl_xor_sync(0xffffffffu, Bsum[k], o);
      Esum[k] += __shfl_xor_sync(0xffffffffu, Esum[k], o);
      dmax[k] = fmaxf(dmax[k], __shfl_xor_sync(0xffffffffu, dmax[k], o));
    }
  if constexpr (TPL < 16) {
#pragma unroll
    for (int r = 0; r < kHqRows; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        acc[r][h].x += __shfl_xor_sync(0xffffffffu, acc[r][h].x, 16);
        acc[r][h].y += __shfl_xor_sync(0xffffffffu, acc[r][h].y, 16);
      }
  }
  __syncthreads();   // every warp is done with its stages
  float* mw = reinterpret_cast<float*>(sm) + warp * C::MW;
  if (lane < NC) {
#pragma unroll
    for (int r = 0; r < kHqRows; ++r)
      *reinterpret_cast<float4*>(mw + r * D + 4 * lane) =
          make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
  }
  if (lane == 0 || lane == 16) {   // the lanes of half hc hold rows 2 hc, 2 hc + 1
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      float* stt = mw + kHqRows * D + (r0 + k) * 8;
      stt[0] = m2[k];
      stt[1] = lsum[k];
      stt[2] = Asum[k];
      stt[3] = Bsum[k];
      stt[4] = Esum[k];
      stt[5] = dmax[k];
    }
  }
  if (lane == 0) {
    float* hd = mw + kHqRows * D + kHqRows * 8;
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      hd[g] = rhi[g];
      hd[NB + g] = rlo[g];
    }
    hd[2 * NB] = etamax;
  }
  __syncthreads();
  // ---- warp r merges row r of the 4 warps into this split's record ----
  const int r = warp;
  const float* smf = reinterpret_cast<const float*>(sm);
  float* rec = a.part + ((int64_t)blockIdx.x * gridDim.y + split) * hq_rec_floats(D);
  float mW = -INFINITY;
#pragma unroll
  for (int w = 0; w < kHqWarps; ++w) mW = fmaxf(mW, smf[w * C::MW + kHqRows * D + r * 8]);
  float st5[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
  float o1[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o1[e] = 0.f;
#pragma unroll
  for (int w = 0; w < kHqWarps; ++w) {
    const float* mwp = smf + w * C::MW;
    const float* stw = mwp + kHqRows * D + r * 8;
    const float f = stw[0] == -INFINITY ? 0.f : ex2(stw[0] - mW);
#pragma unroll
    for (int k = 0; k < 4; ++k) st5[k] = fmaf(f, stw[1 + k], st5[k]);
    st5[4] = fmaxf(st5[4], stw[5]);
#pragma unroll
    for (int e = 0; e < E; ++e) o1[e] = fmaf(f, mwp[r * D + lane * E + e], o1[e]);
  }
  if (r == 0 && lane < kHqHdr) {
    float hv = 0.f;
    if (lane < 2 * NB + 1) {
      hv = lane < NB ? -INFINITY : (lane < 2 * NB ? INFINITY : 0.f);
#pragma unroll
      for (int w = 0; w < kHqWarps; ++w) {
        const float x = smf[w * C::MW + kHqRows * D + kHqRows * 8 + lane];
        hv = lane < NB ? fmaxf(hv, x) : (lane < 2 * NB ? fminf(hv, x) : fmaxf(hv, x));
      }
    }
    rec[lane] = hv;
  }
  if (lane == 0) {
    float* rs = rec + kHqHdr + r * 8;
    rs[0] = mW;
#pragma unroll
    for (int k = 0; k < 5; ++k) rs[1 + k] = st5[k];
  }
#pragma unroll
  for (int e = 0; e < E; ++e) rec[kHqHdr + kHqRows * 8 + r * D + lane * E + e] = o1[e];
}

template <int D>
__global__ void __launch_bounds__(kHqWarps * 32) hqmq_merge_kernel(const HqDecodeArgs ha) {
  constexpr int E = D / 32, NB = D / 32;
  constexpr int RF = hq_rec_floats(D);
  const DecodeArgs& a = ha.a;
  __shared__ float shd[kHqHdr];
  const int unit = blockIdx.x, kvh = unit % a.hkv, b = unit / a.hkv;
  const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // every split wrote a record (an empty one when it held none of the pages),
  // so neither the context length nor one load after another is needed: warp
  // 0 merges the header while every warp merges its row's statistics and
  // outputs
  const int nsp = ha.nsp;
  const float* ubase = a.part + (int64_t)unit * nsp * RF;
  if (r == 0) merge_split_header<NB>(ubase, RF, nsp, lane, shd);
  const float* st0 = ubase + kHqHdr + r * 8;
  float m_own;
  const SplitStats t = merge_split_stats(st0, RF, nsp, lane, &m_own);
  float o1[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o1[e] = 0.f;
  for (int base = 0; base < nsp; base += 32) {
    const float wl = base == 0 ? (m_own == -INFINITY ? 0.f : ex2(m_own - t.M))
                               : split_weight(st0, RF, nsp, base, lane, t.M);
    const int cnt = min(32, nsp - base);
#pragma unroll 4
    for (int k = 0; k < cnt; ++k) {
      const float w = __shfl_sync(0xffffffffu, wl, k);
      const float* orow = ubase + (int64_t)(base + k) * RF + kHqHdr + kHqRows * 8 + r * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) o1[e] = fmaf(w, __ldcg(orow + e), o1[e]);
    }
  }
  __syncthreads();   // the header
  if (r >= a.R) return;
  const int qi = r / a.G, hq = kvh * a.G + r % a.G;
  const int64_t row = ((int64_t)b * a.nq + qi) * a.hq + hq;
  const float l = t.l;
  const float inv_l = l > 0.f ? 1.0f / l : 0.f;   // l = 0: an empty context, output 0
  if (a.out) {
#pragma unroll
    for (int e = 0; e < E; ++e) a.out[row * D + lane * E + e] = o1[e] * inv_l;
  }
  if (lane == 0) {
    const bool skipped = shd[2 * NB] == INFINITY;   // a page of the unit was not read
    float bd = skipped ? INFINITY : 0.f;
    if (!skipped && l > 0.f) {
      float range = 0.f;
#pragma unroll
      for (int g = 0; g < NB; ++g) range = fmaxf(range, shd[g] - shd[NB + g]);
      const float tv = fminf(tanhf(0.5f * t.dm), t.A / t.B);
      bd = kKappa * (tv * (range + 2.0f * shd[2 * NB]) + t.E / l);
    }
    a.bound[row] = bd;
    a.flags[row] = skipped || (l > 0.f && bd > a.tau) ? 1 : 0;
  }
}

const void* hqmq_partial_kernel(int d, int out) {
  if (d == 128) return out ? reinterpret_cast<const void*>(hqmq_partial_kernel<128, true>)
                           : reinterpret_cast<const void*>(hqmq_partial_kernel<128, false>);
  if (d == 64) return out ? reinterpret_cast<const void*>(hqmq_partial_kernel<64, true>)
                          : reinterpret_cast<const void*>(hqmq_partial_kernel<64, false>);
  return nullptr;
}
int hqmq_partial_smem(int d, int S, int out) {
  if (d == 128) return out ? HqCfg<128, true>::smem(S) : HqCfg<128, false>::smem(S);
  return out ? HqCfg<64, true>::smem(S) : HqCfg<64, false>::smem(S);
}
int hqmq_record_floats(int d) { return hq_rec_floats(d); }
int hqmq_threads() { return kHqWarps * 32; }

template <int D, bool OUT>
static void launch_hqmq_partial(const HqDecodeArgs& a, dim3 grid, cudaStream_t stream) {
  hqmq_partial_kernel<D, OUT><<<grid, kHqWarps * 32, HqCfg<D, OUT>::smem(a.S), stream>>>(a);
}

cudaError_t launch_hqmq_decode(const HqDecodeArgs& a, int d, int units, int splits,
                               cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  const dim3 grid((unsigned)units, (unsigned)splits, 1);
  if (d == 128) {
    if (a.outliers) launch_hqmq_partial<128, true>(a, grid, stream);
    else launch_hqmq_partial<128, false>(a, grid, stream);
    hqmq_merge_kernel<128><<<units, kHqWarps * 32, 0, stream>>>(a);
  } else if (d == 64) {
    if (a.outliers) launch_hqmq_partial<64, true>(a, grid, stream);
    else launch_hqmq_partial<64, false>(a, grid, stream);
    hqmq_merge_kernel<64><<<units, kHqWarps * 32, 0, stream>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kvq
