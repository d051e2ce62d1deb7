// kqv.cu -- the KQV codec of "Statistical Inference and Quality Measures of KV
// Cache Quantisations Inspired by TurboQuant" (Quantisation schemes: KQV):
// K and V rotated by the randomized Walsh-Hadamard transform, K coded by the
// 4-bit scalar MSE (Lloyd-Max) quantizer of the rotated unit vector's
// coordinates, V by the 3-bit one plus the 1-bit QJL sketch of its residual,
// with the certified bound of "Runtime-Certified Bounded-Error Quantized
// Attention" (Methodology 2) carried over to this codec.
//
//   kvq_kqv_codebook      host: the Lloyd-Max quantizer of N(0, 1) by
//                         Lloyd's iteration on the decision thresholds, the
//                         Gaussian limit of the page's Beta coordinate
//                         marginal, scaled by 1/sqrt(d)
//   kqv_append_kernel     one warp per (token, kv head): rotation, norms,
//                         codes, the sketch (S r, one projection per lane
//                         and pass), the reconstruction for eta and the value
//                         range
//   kqv_partial_kernel    grid (sequence x kv head, split), 4 warps, each warp
//                         streaming its pages through a 2-stage bulk-copy
//                         ring: scores on fp16 tensor cores (one byte of
//                         codes = one A register, looked up as the centroids'
//                         fp16 hi and lo parts from a bank-replicated shared
//                         table; q' as hi and lo B columns), online softmax,
//                         the bound's sums, PV on the CUDA cores as two
//                         accumulations per lane (the codebook part per
//                         channel, the sketch part per projection)
//   kqv_merge_kernel      per (sequence, kv head): the split records' merge,
//                         the sketch part through S^T, the inverse rotation,
//                         the bound and the flag
// Every dot product or squared norm whose rounding decides a code or a
// sketch bit is the sequential fmaf chain over the channels that the codec's
// definition fixes, so codes, bits, norms and eta are bit-identical to a
// sequential implementation.
#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>

#include "kvq_internal.cuh"
#include "split_merge.cuh"

namespace kvq {

// ================================================================ codebook ====
namespace {

constexpr double kPi = 3.14159265358979323846;

double normal_pdf(double x) { return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) / std::sqrt(2.0 * kPi); }
// P(X > x) for X ~ N(0, 1)
double normal_sf(double x) { return std::isinf(x) ? 0.0 : 0.5 * std::erfc(x / std::sqrt(2.0)); }

// Lloyd's iteration on the positive decision thresholds of the symmetric
// quantizer with L = 2^bits levels: the centroids of the cells they bound
// (conditional means, closed form for the normal density), then the
// midpoints of neighbouring centroids as the new thresholds, until no
// threshold moves by more than 2^-52 of the largest centroid.  Writes the L
// centroids, ascending and exactly antisymmetric.
void lloyd_max_normal(int bits, double* cent) {
  const int L = 1 << bits, half = L / 2;
  double thr[33];                        // thr[0] = 0 < thr[1] < ... ; thr[half] = +inf
  double c[32];
  for (int i = 0; i <= half; ++i) thr[i] = i == half ? INFINITY : 3.0 * i / half;
  for (int it = 0; it < 1000000; ++it) {
    for (int i = 0; i < half; ++i)
      c[i] = (normal_pdf(thr[i]) - normal_pdf(thr[i + 1])) /
             (normal_sf(thr[i]) - normal_sf(thr[i + 1]));
    double moved = 0.0;
    for (int i = 1; i < half; ++i) {
      const double t = 0.5 * (c[i - 1] + c[i]);
      moved = std::fmax(moved, std::fabs(t - thr[i]));
      thr[i] = t;
    }
    if (moved <= std::ldexp(c[half - 1], -52)) {
      for (int i = 0; i < half; ++i)   // the centroids of the final thresholds
        c[i] = (normal_pdf(thr[i]) - normal_pdf(thr[i + 1])) /
               (normal_sf(thr[i]) - normal_sf(thr[i + 1]));
      break;
    }
  }
  for (int i = 0; i < half; ++i) {
    cent[half + i] = c[i];
    cent[half - 1 - i] = -c[i];
  }
}

int codebook_f32(int bits, int d, float* cent, float* thr) {
  double c[64];
  lloyd_max_normal(bits, c);
  const int L = 1 << bits;
  const double sd = std::sqrt((double)d);
  for (int i = 0; i < L; ++i) cent[i] = (float)(c[i] / sd);
  for (int i = 0; i + 1 < L; ++i) thr[i] = (float)((c[i] + c[i + 1]) / (2.0 * sd));
  return KVQ_OK;
}

}  // namespace

int kqv_tables(int d, KqvTables* t) {
  static std::mutex mu;
  static std::map<int, KqvTables> cache;
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(d);
  if (it == cache.end()) {
    KqvTables x;
    codebook_f32(4, d, x.kcent, x.kthr);
    codebook_f32(3, d, x.vcent, x.vthr);
    it = cache.emplace(d, x).first;
  }
  *t = it->second;
  return KVQ_OK;
}

// ================================================================ append =====
template <int L>
__device__ __forceinline__ int kqv_code(float u, const float* thr) {
  int k = 0;
#pragma unroll
  for (int i = 0; i + 1 < L; ++i) k += thr[i] < u;
  return k;
}

// One warp per (token, kv head), 8 warps per CTA looping over the items; the
// CTA first stages S in shared memory with rows padded to D + 1 floats, so the
// lanes' reads of a column (the sketch) and of a row (the reconstruction)
// fall in distinct banks.
constexpr int kKqAppendWarps = 8;
template <int D>
constexpr int kqv_append_smem() { return (D * (D + 1) + kKqAppendWarps * 3 * D) * 4; }

template <int D>
__global__ void __launch_bounds__(kKqAppendWarps * 32) kqv_append_kernel(const KqvAppendArgs ka) {
  constexpr int E = D / 32;
  constexpr int LPG = 32 / E;           // lanes per 32-channel group
  constexpr int SP = D + 1;             // padded row of S
  const AppendArgs& a = ka.a;
  const KqvLayout L{D};
  extern __shared__ float smf[];
  float* Ss = smf;                                        // S [D][D + 1]
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float* xs = smf + D * SP + w * 3 * D;                   // per warp: rotated vector,
  float* rs = xs + D;                                     // residual,
  float* ts = rs + D;                                     // reconstruction
  for (int idx = threadIdx.x; idx < D * D; idx += blockDim.x)
    Ss[(idx / D) * SP + idx % D] = __ldg(ka.qjl + idx);
  __syncthreads();
  const int64_t total = (int64_t)a.num_seqs * a.num_tokens * a.hkv;
  for (int64_t item = (int64_t)blockIdx.x * kKqAppendWarps + w; item < total;
       item += (int64_t)gridDim.x * kKqAppendWarps) {
    const int h = (int)(item % a.hkv);
    const int t = (int)((item / a.hkv) % a.num_tokens);
    const int s = (int)(item / ((int64_t)a.hkv * a.num_tokens));
    const int64_t base = s * a.seq_stride + h * a.head_stride + (int64_t)t * a.tok_stride;
    float xk[E], xv[E], vin[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      xk[e] = load_elem(a.k, a.in_bf16, base + lane * E + e);
      xv[e] = vin[e] = load_elem(a.v, a.in_bf16, base + lane * E + e);
    }
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
    uint8_t* blk = a.pool + ((int64_t)page * a.hkv + h) * L.bytes();

    // ---- keys: rotate, norm, codes, eps ----
    warp_rotate<E>(xk, a.signs, lane, a.rot_c);
    __syncwarp();   // the previous item's reads of xs are done
#pragma unroll
    for (int e = 0; e < E; ++e) xs[lane * E + e] = xk[e];
    __syncwarp();
    float nk = 0.f;
    for (int c = 0; c < D; ++c) nk = __fmaf_rn(xs[c], xs[c], nk);
    nk = __fsqrt_rn(nk);
    const bool okk = isfinite(nk);
    if (!okk) nk = 0.f;
    int code[E];
    float eps = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float u = nk > 0.f ? __fdiv_rn(xk[e], nk) : 0.f;
      code[e] = kqv_code<16>(u, ka.t.kthr);
      const float kh = __fmul_rn(nk, ka.t.kcent[code[e]]);
      if (nk > 0.f) eps = fmaxf(eps, fabsf(__fsub_rn(xk[e], kh)));
    }
#pragma unroll
    for (int o = 1; o < 32; o *= 2) eps = fmaxf(eps, __shfl_xor_sync(0xffffffffu, eps, o));
    {
      uint8_t* kc = blk + slot * (D / 2) + lane * (E / 2);
#pragma unroll
      for (int e = 0; e < E; e += 2) kc[e / 2] = (uint8_t)(code[e] | (code[e + 1] << 4));
    }
    __syncwarp();   // every lane has read xs

    // ---- values: rotate, norm, codes, residual, its norm ----
    warp_rotate<E>(xv, a.signs, lane, a.rot_c);
#pragma unroll
    for (int e = 0; e < E; ++e) xs[lane * E + e] = xv[e];
    __syncwarp();
    float nv = 0.f;
    for (int c = 0; c < D; ++c) nv = __fmaf_rn(xs[c], xs[c], nv);
    nv = __fsqrt_rn(nv);
    const bool okv = isfinite(nv);
    if (!okv) nv = 0.f;
    int vcode[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float u = nv > 0.f ? __fdiv_rn(xv[e], nv) : 0.f;
      vcode[e] = kqv_code<8>(u, ka.t.vthr);
      rs[lane * E + e] = __fsub_rn(u, ka.t.vcent[vcode[e]]);
    }
    __syncwarp();
    float rn = 0.f;
    for (int c = 0; c < D; ++c) rn = __fmaf_rn(rs[c], rs[c], rn);
    rn = __fsqrt_rn(rn);

    // ---- the QJL sketch: projection i = lane + 32 m, a sequential chain over c
    // (E independent chains per lane) ----
    float acc[E];
#pragma unroll
    for (int m = 0; m < E; ++m) acc[m] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float rc = rs[c];
#pragma unroll
      for (int m = 0; m < E; ++m) acc[m] = __fmaf_rn(Ss[(lane + 32 * m) * SP + c], rc, acc[m]);
    }
    uint32_t word[E];
#pragma unroll
    for (int m = 0; m < E; ++m) word[m] = __ballot_sync(0xffffffffu, acc[m] >= 0.f);
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < E; ++m)
        reinterpret_cast<uint32_t*>(blk + L.vs() + slot * (D / 8))[m] = word[m];
      reinterpret_cast<float*>(blk + L.kn())[slot] = nk;
      reinterpret_cast<float*>(blk + L.ke())[slot] = nextafterf(eps, INFINITY);
      reinterpret_cast<float*>(blk + L.vn())[slot] = nv;
      reinterpret_cast<float*>(blk + L.vr())[slot] = rn;
    }
    {
      uint8_t* vc = blk + L.vc() + slot * (D / 2) + lane * (E / 2);
#pragma unroll
      for (int e = 0; e < E; e += 2) vc[e / 2] = (uint8_t)(vcode[e] | (vcode[e + 1] << 4));
    }

    // ---- reconstruction: sum_i S_ic b_i for channels c = lane + 32 m (a
    // sequential chain over i each), then v^' = nv (c3 + rho sum) ----
#pragma unroll
    for (int m = 0; m < E; ++m) acc[m] = 0.f;
#pragma unroll
    for (int mw = 0; mw < E; ++mw)
      for (int bi = 0; bi < 32; ++bi) {
        const float sgn = (word[mw] >> bi) & 1u ? 1.f : -1.f;
        const float* row = Ss + (32 * mw + bi) * SP + lane;
#pragma unroll
        for (int m = 0; m < E; ++m) acc[m] = __fmaf_rn(row[32 * m], sgn, acc[m]);
      }
#pragma unroll
    for (int m = 0; m < E; ++m) ts[lane + 32 * m] = acc[m];
    __syncwarp();
    const float rho = __fmul_rn(ka.qjl_c, rn);
    float vh[E];
#pragma unroll
    for (int e = 0; e < E; ++e)
      vh[e] = __fmul_rn(nv, __fadd_rn(ka.t.vcent[vcode[e]], __fmul_rn(rho, ts[lane * E + e])));
    warp_hadamard<E>(vh, lane, a.rot_c);
    float err = 0.f, hi = 0.f, lo = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (a.signs[lane * E + e] < 0) vh[e] = -vh[e];
      err = fmaxf(err, fabsf(__fsub_rn(vin[e], vh[e])));
      hi = fmaxf(hi, vh[e]);
      lo = fminf(lo, vh[e]);
    }
#pragma unroll
    for (int o = 1; o < 32; o *= 2) err = fmaxf(err, __shfl_xor_sync(0xffffffffu, err, o));
#pragma unroll
    for (int o = 1; o < LPG; o *= 2) {
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    }
    if (!okk || !okv) err = 0.f;
    if (lane == 0) {
      if (!okk || !okv) set_error(a.err, KVQ_ERR_RANGE);
      const float eu = nextafterf(__fmaf_rn(0x1p-16f, nv, err), INFINITY);
      atomicMax(reinterpret_cast<int*>(a.eta + (int64_t)page * a.hkv + h), __float_as_int(eu));
    }
    if (lane % LPG == 0) {
      // the block's range starts at [0, 0]: a maximum >= 0 orders like its int
      // bits, a minimum <= 0 (sign bit set) like its unsigned bits, reversed
      float* rg = reinterpret_cast<float*>(blk + L.rg()) + 2 * (lane / LPG);
      if (hi > 0.f) atomicMax(reinterpret_cast<int*>(rg), __float_as_int(hi));
      if (lo < 0.f) atomicMax(reinterpret_cast<unsigned int*>(rg + 1), __float_as_uint(lo));
    }
  }
}

template <int D>
cudaError_t launch_kqv_append_d(const KqvAppendArgs& a, cudaStream_t stream) {
  // opt in to the staged S's shared memory once per device
  static std::mutex mu;
  static std::map<int, int> sms_of;
  constexpr int smem = kqv_append_smem<D>();
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = sms_of.find(dev);
    if (it == sms_of.end()) {
      if ((e = cudaFuncSetAttribute(kqv_append_kernel<D>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
              cudaSuccess ||
          (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
      it = sms_of.emplace(dev, sms).first;
    }
    sms = it->second;
  }
  const int64_t items = (int64_t)a.a.num_seqs * a.a.num_tokens * a.a.hkv;
  const int64_t blocks = std::min<int64_t>((items + kKqAppendWarps - 1) / kKqAppendWarps, 2 * sms);
  kqv_append_kernel<D><<<(unsigned)blocks, kKqAppendWarps * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_kqv_append(const KqvAppendArgs& a, int d, cudaStream_t stream) {
  const int64_t items = (int64_t)a.a.num_seqs * a.a.num_tokens * a.a.hkv;
  if (items == 0) return cudaSuccess;
  if (d == 128) return launch_kqv_append_d<128>(a, stream);
  if (d == 64) return launch_kqv_append_d<64>(a, stream);
  return cudaErrorInvalidValue;
}

// ================================================================ decode =====
constexpr int kKqWarps = 4;
constexpr int kKqRows = 4;
constexpr int kKqStages = 2;
constexpr int kKqHdr = 16;   // floats: range max [NB], range min [NB], eta max
__host__ __device__ constexpr int kqv_rec_floats(int d) { return kKqHdr + kKqRows * 8 + 2 * kKqRows * d; }

template <int D>
struct KqCfg {
  // KqvLayout{D}.bytes(): codes, sketch, four fp32 per token, the range
  static constexpr int BLOCK = kPage * D + kPage * D / 8 + 16 * kPage + (D / 32) * 8;
  static constexpr int OFF_ST = 0;                                           // [warp][stage][BLOCK]
  static constexpr int OFF_W = OFF_ST + kKqWarps * kKqStages * BLOCK;        // [warp][2][16][4] f32
  static constexpr int OFF_LUT = OFF_W + kKqWarps * 2 * kPage * kKqRows * 4; // [16 + 8][32] f32
  static constexpr int OFF_Q = OFF_LUT + 24 * 32 * 4;                       // q' [4][D] f32
  static constexpr int OFF_QN = OFF_Q + kKqRows * D * 4;                    // |q'|_1, |q'|_2 [4][2]
  static constexpr int OFF_BAR = (OFF_QN + 32 + 15) / 16 * 16;              // [warp][stage] u64
  static constexpr int OFF_PG = OFF_BAR + kKqWarps * kKqStages * 8;          // [warp][stage] i32
  static constexpr int END = OFF_PG + kKqWarps * kKqStages * 4;
  // merge of the CTA's warps (aliases the stages): per warp [4][D] x 2, [4][8], header
  static constexpr int MW = 2 * kKqRows * D + kKqRows * 8 + kKqHdr;
  static constexpr int MERGE = kKqWarps * MW * 4;
  static constexpr int SMEM = 128 + (END > MERGE ? END : MERGE);
  static_assert(MERGE <= OFF_BAR, "the merge area must not reach the barriers");
};

template <int D>
__global__ void __launch_bounds__(kKqWarps * 32) kqv_partial_kernel(const KqvDecodeArgs ka) {
  using C = KqCfg<D>;
  constexpr int E = D / 32, NB = D / 32;
  const DecodeArgs& a = ka.a;
  const KqvLayout L{D};
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  const int split = blockIdx.y, kvh = blockIdx.x % a.hkv, b = blockIdx.x / a.hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR) + warp * kKqStages;
  int* spage = reinterpret_cast<int*>(sm + C::OFF_PG) + warp * kKqStages;
  if (lane == 0) {
    for (int s = 0; s < kKqStages; ++s) mbar_init(&bar[s], 1);
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
    write_empty_record(a.part + ((int64_t)blockIdx.x * gridDim.y + split) * kqv_rec_floats(D), NB,
                       kKqHdr, kKqRows, 2 * kKqRows * D);
    return;
  }
  const int p1 = min(npages, p0 + a.pps);

  // ---- tables and query rows ----
  // [24][32]: rows 0..15 the key centroids as packed fp16 (hi, lo) with
  // hi + lo = the fp32 centroid to ~2^-22; rows 16..23 the value centroids
  // (fp32); every entry replicated per lane, so lookups never conflict
  float* lut = reinterpret_cast<float*>(sm + C::OFF_LUT);
  uint32_t* lutk = reinterpret_cast<uint32_t*>(lut);
  for (int i = tid; i < 24 * 32; i += blockDim.x) {
    const int k = i / 32;
    if (k < 16) {
      const float c = ka.t.kcent[k];
      const __half hi = __float2half_rn(c);
      const __half lo = __float2half_rn(c - __half2float(hi));
      lutk[i] = h2_as_u32(__halves2half2(hi, lo));
    } else {
      lut[i] = ka.t.vcent[k - 16];
    }
  }
  float* qs = reinterpret_cast<float*>(sm + C::OFF_Q);
  float* qn = reinterpret_cast<float*>(sm + C::OFF_QN);
  {
    const int r = warp;   // 4 warps, 4 rows
    float x[E];
    if (r < a.R) {
      const int qi = r / a.G, hq = kvh * a.G + r % a.G;
      const int64_t e0 = (((int64_t)b * a.nq + qi) * a.hq + hq) * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = load_elem(a.q, a.q_bf16, e0 + e);
      warp_rotate<E>(x, a.signs, lane, a.rot_c);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = 0.f;
    }
    float l1 = 0.f, l2 = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qs[r * D + lane * E + e] = x[e];
      l1 += fabsf(x[e]);
      l2 = fmaf(x[e], x[e], l2);
    }
#pragma unroll
    for (int o = 1; o < 32; o *= 2) {
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      l2 += __shfl_xor_sync(0xffffffffu, l2, o);
    }
    if (lane == 0) {
      qn[2 * r] = l1;
      qn[2 * r + 1] = sqrtf(l2);
    }
  }
  __syncthreads();
  // B fragments of the QK^T MMA (m16n8k16, k = 16 channels per step): column
  // n = g8 holds row n % 4 of q', its fp16 hi part (n < 4) or the remainder
  // (n >= 4); k pairs (2 c4, 2 c4 + 1) and (2 c4 + 8, 2 c4 + 9)
  constexpr int KS = D / 16;
  const int g8 = lane >> 2, c4 = lane & 3;
  uint32_t qb[KS][2];
  {
    const int qr = g8 & 3;
    const bool lo_part = g8 >= 4;
    auto part = [&](float v) -> __half {
      const __half hi = __float2half_rn(v);
      return lo_part ? __float2half_rn(v - __half2float(hi)) : hi;
    };
#pragma unroll
    for (int kk = 0; kk < KS; ++kk)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = 16 * kk + 8 * h + 2 * c4;
        qb[kk][h] = h2_as_u32(__halves2half2(part(qs[qr * D + c]), part(qs[qr * D + c + 1])));
      }
  }
  // this lane's scores: token g8 (c4 < 2) or g8 + 8 (c4 >= 2), rows r0, r0 + 1
  const int r0 = 2 * (c4 & 1);
  float cq1[2], cq2[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    cq1[k] = kKappa * a.s_att * qn[2 * (r0 + k)];
    cq2[k] = kKappa * a.s_att * kRotSlack * qn[2 * (r0 + k) + 1];
  }
  const float zsc = a.s_att * kLog2e;

  // ---- pages of this warp: p0 + warp, p0 + warp + 4, ... ----
  const int first = p0 + warp;
  const int nloc = first < p1 ? (p1 - first + kKqWarps - 1) / kKqWarps : 0;
  uint8_t* stage0 = sm + C::OFF_ST + warp * kKqStages * C::BLOCK;
  const int32_t* ptab = a.page_table + (int64_t)b * a.max_pages;
  // lane l holds the page index of local page 32 c + l of chunk c (loaded a
  // chunk at a time, so no issue waits on a page-table load of its own)
  int pt_chunk = -1, pt_val = -1;
  auto issue = [&](int j, int st) {
    if ((j >> 5) != pt_chunk) {
      pt_chunk = j >> 5;
      const int jl = 32 * pt_chunk + lane;
      pt_val = jl < nloc ? __ldg(ptab + first + jl * kKqWarps) : -1;
    }
    const int pgv = __shfl_sync(0xffffffffu, pt_val, j & 31);
    if (lane == 0) {
      const int pg = pgv;
      const bool ok = pg >= 0 && pg < a.num_pages;
      spage[st] = ok ? pg : -1;
      if (ok) {
        mbar_arrive_expect_tx(&bar[st], C::BLOCK);
        bulk_g2s_hint(stage0 + st * C::BLOCK, a.pool + ((int64_t)pg * a.hkv + kvh) * C::BLOCK,
                      C::BLOCK, &bar[st], l2_evict_first_policy());
      } else {
        set_error(a.err, KVQ_ERR_INVALID_ARG);
        mbar_arrive(&bar[st]);
      }
    }
    __syncwarp();
  };
  for (int j = 0; j < kKqStages && j < nloc; ++j) issue(j, j);

  // PV accumulators of channel (and projection) e: rows (0, 1) and (2, 3) as
  // packed fp32x2 pairs
  float2 acc1[E][2], acc2[E][2];
#pragma unroll
  for (int e = 0; e < E; ++e)
#pragma unroll
    for (int h = 0; h < 2; ++h) acc1[e][h] = acc2[e][h] = make_float2(0.f, 0.f);
  float m2[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f}, Asum[2] = {0.f, 0.f},
        Bsum[2] = {0.f, 0.f}, Esum[2] = {0.f, 0.f}, dmax[2] = {0.f, 0.f};
  float rhi[NB], rlo[NB], etamax = clamped ? INFINITY : 0.f;
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    rhi[g] = -INFINITY;
    rlo[g] = INFINITY;
  }
  float* wts = reinterpret_cast<float*>(sm + C::OFF_W) + warp * 2 * kPage * kKqRows;
  int jstop = nloc;
  for (int j = 0; j < nloc; ++j) {
    const int st = j % kKqStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&bar[st], (uint32_t)((j / kKqStages) & 1)))) {
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
      const float* fv = reinterpret_cast<const float*>(blk + L.vn());
      const float* fr = reinterpret_cast<const float*>(blk + L.vr());
      const float* frg = reinterpret_cast<const float*>(blk + L.rg());
      const int nval = min(kPage, n - (first + j * kKqWarps) * kPage);
      const float eta_pg = __ldg(a.eta + (int64_t)pg * a.hkv + kvh);
      etamax = fmaxf(etamax, eta_pg);
#pragma unroll
      for (int g = 0; g < NB; ++g) {
        rhi[g] = fmaxf(rhi[g], frg[2 * g]);
        rlo[g] = fminf(rlo[g], frg[2 * g + 1]);
      }
      // ---- QK^T on fp16 tensor cores: tokens = M, channels = K ----
      // One byte of a token's codes is one A register (two channels); the
      // lane needs byte c4 of every 4-byte word of rows g8 and g8 + 8.
      float sc4[4] = {0.f, 0.f, 0.f, 0.f};
      {
        uint32_t wr[2][D / 8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4* rowp = reinterpret_cast<const uint4*>(blk + (g8 + 8 * h) * (D / 2));
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            const uint4 v4 = rowp[q];
            wr[h][4 * q] = v4.x;
            wr[h][4 * q + 1] = v4.y;
            wr[h][4 * q + 2] = v4.z;
            wr[h][4 * q + 3] = v4.w;
          }
        }
        const uint32_t bsel = 0x4440u | (uint32_t)c4;   // byte c4, zero-extended
        auto afrag = [&](uint32_t word, uint32_t& ahi, uint32_t& alo) {
          const uint32_t byte = prmt(word, 0u, bsel);
          const uint32_t v0 = lutk[(byte & 15u) * 32 + lane];
          const uint32_t v1 = lutk[(byte >> 4) * 32 + lane];
          ahi = prmt(v0, v1, 0x5410u);
          alo = prmt(v0, v1, 0x7632u);
        };
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          uint32_t h0, l0, h1, l1, h2, l2, h3, l3;
          afrag(wr[0][2 * kk], h0, l0);       // token g8, channels 16 kk + 2 c4, +1
          afrag(wr[1][2 * kk], h1, l1);       // token g8 + 8
          afrag(wr[0][2 * kk + 1], h2, l2);   // token g8, channels 16 kk + 8 + 2 c4, +1
          afrag(wr[1][2 * kk + 1], h3, l3);
          mma_f16(sc4, h0, h1, h2, h3, qb[kk][0], qb[kk][1]);
          mma_f16(sc4, l0, l1, l2, l3, qb[kk][0], qb[kk][1]);
        }
      }
      // columns 2 c4, 2 c4 + 1: the hi (c4 < 2) or lo part of rows r0, r0 + 1
#pragma unroll
      for (int k = 0; k < 4; ++k) sc4[k] += __shfl_xor_sync(0xffffffffu, sc4[k], 2);
      const int t = g8 + 8 * (c4 >> 1);
      const bool vt = t < nval;
      const float nk = fk[t];
      float zt[2], dl[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float sraw = c4 < 2 ? sc4[k] : sc4[2 + k];
        zt[k] = vt ? sraw * nk * zsc : -INFINITY;
        dl[k] = vt ? fmaf(cq1[k], fe[t], cq2[k] * nk) : 0.f;
      }
      // ---- online softmax and the bound's sums, rows r0 + k, once per page ----
      float alpha[2];
      const float wvn = vt ? fv[t] : 0.f, wrn = vt ? fr[t] : 0.f;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float mx = zt[k];
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
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
        // weights of the PV accumulations (0 outside the context: the slots
        // past it may hold another sequence's norms)
        const float wa = wv * wvn;
        wts[t * 4 + r0 + k] = wa;
        wts[kPage * 4 + t * 4 + r0 + k] = wa * wrn;
      }
      if (__any_sync(0xffffffffu, alpha[0] != 1.0f || alpha[1] != 1.0f)) {
        // row r's factor sits in lanes with c4 & 1 == r / 2, slot r % 2
        float ar[kKqRows];
#pragma unroll
        for (int r = 0; r < kKqRows; ++r) ar[r] = __shfl_sync(0xffffffffu, alpha[r & 1], r >> 1);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 a2 = make_float2(ar[2 * h], ar[2 * h + 1]);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            acc1[e][h] = mul2(acc1[e][h], a2);
            acc2[e][h] = mul2(acc2[e][h], a2);
          }
        }
      }
      __syncwarp();
      // ---- PV: lane l owns channels (and projections) [l E, l E + E) ----
#pragma unroll 4
      for (int t = 0; t < kPage; ++t) {
        const float4 wa4 = reinterpret_cast<const float4*>(wts)[t];
        const float4 wb4 = reinterpret_cast<const float4*>(wts + kPage * 4)[t];
        const uint8_t* vc = blk + L.vc() + t * (D / 2) + lane * (E / 2);
        const unsigned sb = blk[L.vs() + t * (D / 8) + (lane * E) / 8] >> ((lane * E) % 8);
        float cv[E], sg[E];
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          const unsigned byte = vc[e / 2];
          cv[e] = lut[(16 + (byte & 15u)) * 32 + lane];
          cv[e + 1] = lut[(16 + (byte >> 4)) * 32 + lane];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) sg[e] = (sb >> e) & 1u ? 1.f : -1.f;
        const float2 wa2[2] = {make_float2(wa4.x, wa4.y), make_float2(wa4.z, wa4.w)};
        const float2 wb2[2] = {make_float2(wb4.x, wb4.y), make_float2(wb4.z, wb4.w)};
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float2 c2 = make_float2(cv[e], cv[e]), s2 = make_float2(sg[e], sg[e]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            acc1[e][h] = fma2(wa2[h], c2, acc1[e][h]);
            acc2[e][h] = fma2(wb2[h], s2, acc2[e][h]);
          }
        }
      }
    }
    __syncwarp();
    if (j + kKqStages < nloc) issue(j + kKqStages, st);
  }
  // after a wait that ran out, the copies still in flight are waited for
  // (bounded) before the stages become the merge area
  if (jstop < nloc)
    for (int j = jstop; j < nloc && j < jstop + kKqStages; ++j)
      (void)mbar_wait(&bar[j % kKqStages], (uint32_t)((j / kKqStages) & 1));

  // ---- per-warp sums over the lanes of each row (lanes with the same c4 & 1) ----
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int o = 2; o < 32; o *= 2) {
      lsum[k] += __shfl_xor_sync(0xffffffffu, lsum[k], o);
      Asum[k] += __shfl_xor_sync(0xffffffffu, Asum[k], o);
      Bsum[k] += __shfl_xor_sync(0xffffffffu, Bsum[k], o);
      Esum[k] += __shfl_xor_sync(0xffffffffu, Esum[k], o);
      dmax[k] = fmaxf(dmax[k], __shfl_xor_sync(0xffffffffu, dmax[k], o));
    }
  __syncthreads();   // every warp is done with its stages
  float* mw = reinterpret_cast<float*>(sm) + warp * C::MW;
#pragma unroll
  for (int r = 0; r < kKqRows; ++r)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      mw[r * D + lane * E + e] = (r & 1) ? acc1[e][r >> 1].y : acc1[e][r >> 1].x;
      mw[kKqRows * D + r * D + lane * E + e] = (r & 1) ? acc2[e][r >> 1].y : acc2[e][r >> 1].x;
    }
  if (lane < 2) {   // lane c4 = lane holds rows 2 lane, 2 lane + 1
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      float* stt = mw + 2 * kKqRows * D + (2 * lane + k) * 8;
      stt[0] = m2[k];
      stt[1] = lsum[k];
      stt[2] = Asum[k];
      stt[3] = Bsum[k];
      stt[4] = Esum[k];
      stt[5] = dmax[k];
    }
  }
  if (lane == 0) {
    float* hd = mw + 2 * kKqRows * D + kKqRows * 8;
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
  float* rec = a.part + ((int64_t)blockIdx.x * gridDim.y + split) * kqv_rec_floats(D);
  float mW = -INFINITY;
#pragma unroll
  for (int w = 0; w < kKqWarps; ++w) mW = fmaxf(mW, reinterpret_cast<float*>(sm)[w * C::MW + 2 * kKqRows * D + r * 8]);
  float st5[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
  float o1[E], o2[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o1[e] = o2[e] = 0.f;
#pragma unroll
  for (int w = 0; w < kKqWarps; ++w) {
    const float* mwp = reinterpret_cast<float*>(sm) + w * C::MW;
    const float* stw = mwp + 2 * kKqRows * D + r * 8;
    const float f = stw[0] == -INFINITY ? 0.f : ex2(stw[0] - mW);
#pragma unroll
    for (int k = 0; k < 4; ++k) st5[k] = fmaf(f, stw[1 + k], st5[k]);
    st5[4] = fmaxf(st5[4], stw[5]);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      o1[e] = fmaf(f, mwp[r * D + lane * E + e], o1[e]);
      o2[e] = fmaf(f, mwp[kKqRows * D + r * D + lane * E + e], o2[e]);
    }
  }
  if (r == 0 && lane < kKqHdr) {
    float hv = 0.f;
    if (lane < 2 * NB + 1) {
      hv = lane < NB ? -INFINITY : (lane < 2 * NB ? INFINITY : 0.f);
#pragma unroll
      for (int w = 0; w < kKqWarps; ++w) {
        const float x = reinterpret_cast<float*>(sm)[w * C::MW + 2 * kKqRows * D + kKqRows * 8 + lane];
        hv = lane < NB ? fmaxf(hv, x) : (lane < 2 * NB ? fminf(hv, x) : fmaxf(hv, x));
      }
    }
    rec[lane] = hv;
  }
  if (lane == 0) {
    float* rs = rec + kKqHdr + r * 8;
    rs[0] = mW;
#pragma unroll
    for (int k = 0; k < 5; ++k) rs[1 + k] = st5[k];
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    rec[kKqHdr + kKqRows * 8 + r * D + lane * E + e] = o1[e];
    rec[kKqHdr + kKqRows * 8 + kKqRows * D + r * D + lane * E + e] = o2[e];
  }
}

template <int D>
__global__ void __launch_bounds__(kKqWarps * 32) kqv_merge_kernel(const KqvDecodeArgs ka) {
  constexpr int E = D / 32, NB = D / 32;
  constexpr int RF = kqv_rec_floats(D);
  const DecodeArgs& a = ka.a;
  __shared__ float sB[kKqWarps][D];
  __shared__ float sO[kKqWarps][D];
  __shared__ float shd[kKqHdr];
  const int unit = blockIdx.x, kvh = unit % a.hkv, b = unit / a.hkv;
  const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = r / a.G, hq = kvh * a.G + r % a.G;
  const int64_t row = ((int64_t)b * a.nq + qi) * a.hq + hq;
  // every split wrote a record (an empty one when it held none of the pages):
  // warp 0 merges the header while every warp merges its row's statistics and
  // its two accumulations, the records' loads independent of one another
  const int nsp = ka.nsp;
  const float* ubase = a.part + (int64_t)unit * nsp * RF;
  if (r == 0) merge_split_header<NB>(ubase, RF, nsp, lane, shd);
  const float* st0 = ubase + kKqHdr + r * 8;
  float m_own;
  const SplitStats t = merge_split_stats(st0, RF, nsp, lane, &m_own);
  const float l = t.l, A = t.A, Bv = t.B, Ev = t.E, dm = t.dm;
  float o1[E], o2[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o1[e] = o2[e] = 0.f;
  for (int base = 0; base < nsp; base += 32) {
    const float wl = base == 0 ? (m_own == -INFINITY ? 0.f : ex2(m_own - t.M))
                               : split_weight(st0, RF, nsp, base, lane, t.M);
    const int cnt = min(32, nsp - base);
#pragma unroll 4
    for (int k = 0; k < cnt; ++k) {
      const float w = __shfl_sync(0xffffffffu, wl, k);
      const float* rec = ubase + (int64_t)(base + k) * RF + kKqHdr + kKqRows * 8 + r * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        o1[e] = fmaf(w, __ldcg(rec + e), o1[e]);
        o2[e] = fmaf(w, __ldcg(rec + kKqRows * D + e), o2[e]);
      }
    }
  }
  const float inv_l = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    sB[r][lane * E + e] = o2[e] * inv_l;
    sO[r][lane * E + e] = o1[e] * inv_l;
  }
  __syncthreads();   // sB, sO of every warp and the merged header
  // o' = o1 / l + sqrt(pi/2)/d * S^T (o2 / l): thread c < D takes channel c of
  // the 4 rows (coalesced reads of S, one pass for the CTA)
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float acc[kKqRows] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      const float sv = __ldg(ka.qjl + (int64_t)i * D + c);
#pragma unroll
      for (int rr = 0; rr < kKqRows; ++rr) acc[rr] = fmaf(sv, sB[rr][i], acc[rr]);
    }
#pragma unroll
    for (int rr = 0; rr < kKqRows; ++rr) sO[rr][c] = fmaf(ka.qjl_c, acc[rr], sO[rr][c]);
  }
  __syncthreads();
  // then o = sigma o (c H o')
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = sO[r][lane * E + e];
  warp_hadamard<E>(x, lane, a.rot_c);
  if (r >= a.R) return;
  if (a.out) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = lane * E + e;
      a.out[row * D + c] = a.signs[c] < 0 ? -x[e] : x[e];
    }
  }
  if (lane == 0) {
    const bool skipped = shd[2 * NB] == INFINITY;   // a page of the unit was not read
    float bd = skipped ? INFINITY : 0.f;
    if (!skipped && l > 0.f) {
      float range = 0.f;
#pragma unroll
      for (int g = 0; g < NB; ++g) range = fmaxf(range, shd[g] - shd[NB + g]);
      const float tv = fminf(tanhf(0.5f * dm), A / Bv);
      bd = kKappa * (tv * (range + 2.0f * shd[2 * NB]) + Ev / l);
    }
    a.bound[row] = bd;
    a.flags[row] = skipped || (l > 0.f && bd > a.tau) ? 1 : 0;   // l = 0: an empty context
  }
}

const void* kqv_partial_kernel(int d) {
  if (d == 128) return reinterpret_cast<const void*>(kqv_partial_kernel<128>);
  if (d == 64) return reinterpret_cast<const void*>(kqv_partial_kernel<64>);
  return nullptr;
}
int kqv_partial_smem(int d) { return d == 128 ? KqCfg<128>::SMEM : KqCfg<64>::SMEM; }
int kqv_record_floats(int d) { return kqv_rec_floats(d); }
int kqv_threads() { return kKqWarps * 32; }

cudaError_t launch_kqv_decode(const KqvDecodeArgs& a, int d, int units, int splits,
                              cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  const dim3 grid((unsigned)units, (unsigned)splits, 1);
  if (d == 128) {
    kqv_partial_kernel<128><<<grid, kKqWarps * 32, KqCfg<128>::SMEM, stream>>>(a);
    kqv_merge_kernel<128><<<units, kKqWarps * 32, 0, stream>>>(a);
  } else if (d == 64) {
    kqv_partial_kernel<64><<<grid, kKqWarps * 32, KqCfg<64>::SMEM, stream>>>(a);
    kqv_merge_kernel<64><<<units, kKqWarps * 32, 0, stream>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kvq

extern "C" int kvq_kqv_codebook(int32_t bits, int32_t head_dim, float* centroids,
                                float* thresholds) {
  if (bits < 1 || bits > 6 || head_dim < 1 || !centroids || !thresholds) return KVQ_ERR_INVALID_ARG;
  double c[64];
  kvq::lloyd_max_normal(bits, c);
  const int L = 1 << bits;
  const double sd = std::sqrt((double)head_dim);
  for (int i = 0; i < L; ++i) centroids[i] = (float)(c[i] / sd);
  for (int i = 0; i + 1 < L; ++i) thresholds[i] = (float)((c[i] + c[i + 1]) / (2.0 * sd));
  return KVQ_OK;
}
