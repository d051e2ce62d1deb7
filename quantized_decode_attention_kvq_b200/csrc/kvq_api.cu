// kvq_api.cu -- the C ABI (include/kvq.h): argument validation, status codes,
// launch planning (split-K sizing against the SM count and occupancy), and the
// host orchestration of the exact fallback
// (flag read-back with a bounded wait, Tier-2 page-in with cudaMemcpyAsync on
// a side stream, recomputation kernel, stream hand-back).

#include <chrono>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <thread>
#include <tuple>
#include <tuple>
#include <vector>

#include "kvq_internal.cuh"

using namespace kvq;

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_kqv(const kvq_cache* c) {
  if (c->k_bits != 4 || c->v_bits != 3 || c->k_group != c->head_dim || c->v_group != c->head_dim)
    return fail(KVQ_ERR_UNSUPPORTED, "the KQV codec takes k_bits 4, v_bits 3 and groups of head_dim");
  if (c->k_rotate != 1 || !c->rot_signs)
    return fail(KVQ_ERR_INVALID_ARG, "the KQV codec needs k_rotate 1 and rot_signs");
  if (!c->qjl) return fail(KVQ_ERR_INVALID_ARG, "the KQV codec needs the QJL matrix");
  if (c->outliers != 0) return fail(KVQ_ERR_UNSUPPORTED, "the KQV codec has no outlier extraction");
  return KVQ_OK;
}

int check_hqmq(const kvq_cache* c) {
  if (c->k_bits != 6 || c->v_bits != 6 || c->k_group != 4 || c->v_group != 4)
    return fail(KVQ_ERR_UNSUPPORTED, "the HQMQ codec takes k_bits = v_bits = 6 and groups of 4");
  if (c->k_rotate != 0) return fail(KVQ_ERR_UNSUPPORTED, "the HQMQ codec does not rotate keys");
  if (c->outliers != 0 && c->outliers != 1) return fail(KVQ_ERR_INVALID_ARG, "outliers not 0/1");
  if (!c->hq_sec) return fail(KVQ_ERR_INVALID_ARG, "the HQMQ codec needs the secondary units");
  if (c->hq_s < 1 || c->hq_s > KVQ_HQMQ_MAX_S)
    return fail(KVQ_ERR_UNSUPPORTED, "hq_s %d unsupported (1..%d)", c->hq_s, KVQ_HQMQ_MAX_S);
  return KVQ_OK;
}

int check_cache(const kvq_cache* c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
  if (c->page_size != KVQ_PAGE_SIZE) return fail(KVQ_ERR_UNSUPPORTED, "page_size must be 16");
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d unsupported (64 or 128)", c->head_dim);
  if (c->codec != KVQ_CODEC_INT && c->codec != KVQ_CODEC_KQV && c->codec != KVQ_CODEC_HQMQ)
    return fail(KVQ_ERR_INVALID_ARG, "codec %d unknown", c->codec);
  if (c->codec != KVQ_CODEC_INT) {
    if (int rc = c->codec == KVQ_CODEC_KQV ? check_kqv(c) : check_hqmq(c)) return rc;
    if (c->num_kv_heads < 1) return fail(KVQ_ERR_INVALID_ARG, "num_kv_heads < 1");
    if (c->num_pages < 0) return fail(KVQ_ERR_INVALID_ARG, "num_pages < 0");
    if (!c->pool || !c->v_eta) return fail(KVQ_ERR_INVALID_ARG, "pool or v_eta is NULL");
    if (!aligned16(c->pool)) return fail(KVQ_ERR_INVALID_ARG, "pool not 16-byte aligned");
    return KVQ_OK;
  }
  if (c->k_bits != 8 && c->k_bits != 4)
    return fail(KVQ_ERR_UNSUPPORTED, "k_bits %d unsupported (8 or 4)", c->k_bits);
  if (c->k_group != 32 && c->k_group != 64 && c->k_group != 128)
    return fail(KVQ_ERR_UNSUPPORTED, "k_group %d unsupported (32, 64, 128)", c->k_group);
  if (c->head_dim % c->k_group)
    return fail(KVQ_ERR_UNSUPPORTED, "k_group %d does not divide head_dim %d", c->k_group,
                c->head_dim);
  if (c->v_bits != 4 || c->v_group != 32)
    return fail(KVQ_ERR_UNSUPPORTED, "values must be 4-bit with group 32");
  if (c->num_kv_heads < 1) return fail(KVQ_ERR_INVALID_ARG, "num_kv_heads < 1");
  if (c->num_pages < 0) return fail(KVQ_ERR_INVALID_ARG, "num_pages < 0");
  if (c->k_rotate != 0 && c->k_rotate != 1) return fail(KVQ_ERR_INVALID_ARG, "k_rotate not 0/1");
  if (c->k_rotate && !c->rot_signs) return fail(KVQ_ERR_INVALID_ARG, "k_rotate needs rot_signs");
  if (c->outliers != 0 && c->outliers != 1) return fail(KVQ_ERR_INVALID_ARG, "outliers not 0/1");
  if (!c->pool || !c->v_eta) return fail(KVQ_ERR_INVALID_ARG, "pool or v_eta is NULL");
  if (!aligned16(c->pool)) return fail(KVQ_ERR_INVALID_ARG, "pool not 16-byte aligned");
  return KVQ_OK;
}

BlockLayout layout_of(const kvq_cache* c) {
  return BlockLayout{c->head_dim, c->k_bits, c->k_group, c->outliers};
}

float rot_constant(int d) { return (float)(1.0 / std::sqrt((double)d)); }
// fp32(sqrt(pi/2) / d): the QJL estimate's scale per unit of |r|
float kqv_qjl_constant(int d) { return (float)(std::sqrt(3.14159265358979323846 / 2.0) / d); }

struct DeviceInfo {
  int sms = 0, major = 0, max_smem = 0;
};

int device_info(DeviceInfo* out, int* dev_out) {
  static std::mutex mu;
  static std::map<int, DeviceInfo> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    DeviceInfo di;
    if ((e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&di.major, cudaDevAttrComputeCapabilityMajor, dev)) !=
        cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&di.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                    dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    it = cache.emplace(dev, di).first;
  }
  *out = it->second;
  if (dev_out) *dev_out = dev;
  if (out->major != 10)
    return fail(KVQ_ERR_UNSUPPORTED, "device %d has compute capability %d.x; sm_100a required",
                dev, out->major);
  return KVQ_OK;
}

// blocks of the decode kernel resident per SM (after opting into its shared memory)
int decode_occupancy(const DecodeVariant& v, int* occ) {
  static std::mutex mu;
  static std::map<std::pair<int, void*>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto key = std::make_pair(dev, reinterpret_cast<void*>(v.kernel));
  auto it = cache.find(key);
  if (it == cache.end()) {
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(v.kernel),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(reinterpret_cast<const void*>(v.kernel_append),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, reinterpret_cast<const void*>(v.kernel),
                                                      decode_threads(), v.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (n < 1) n = 1;
    it = cache.emplace(key, n).first;
  }
  *occ = it->second;
  return KVQ_OK;
}

struct Plan {
  int splits = 1, pps = 1;
  size_t part_bytes = 0, counter_bytes = 0;
  size_t total() const { return counter_bytes + part_bytes; }
};

constexpr int kMaxPagesPerSplit = 256;

// Split-K sizing: fill every SM's resident slots once with (sequence, kv head,
// split) CTAs; long contexts cap the pages of one split so a ragged batch
// spreads over several waves.
// blocks of the KQV codec's partial decode kernel resident per SM
int kqv_occupancy(int d, int* occ) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto key = std::make_pair(dev, d);
  auto it = cache.find(key);
  if (it == cache.end()) {
    const void* k = kqv_partial_kernel(d);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kqv_partial_smem(d));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kqv_threads(), kqv_partial_smem(d));
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    it = cache.emplace(key, n < 1 ? 1 : n).first;
  }
  *occ = it->second;
  return KVQ_OK;
}

// blocks of the HQMQ codec's partial decode kernel resident per SM (its shared
// memory grows with the secondary set)
int hqmq_occupancy(int d, int S, int out, int* occ) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto key = std::make_tuple(dev, d, S, out);
  auto it = cache.find(key);
  if (it == cache.end()) {
    const void* k = hqmq_partial_kernel(d, out);
    const int smem = hqmq_partial_smem(d, KVQ_HQMQ_MAX_S, out);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, hqmq_threads(),
                                                      hqmq_partial_smem(d, S, out));
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    it = cache.emplace(key, n < 1 ? 1 : n).first;
  }
  *occ = it->second;
  return KVQ_OK;
}

int make_plan(const kvq_cache* c, int num_seqs, int max_pages, Plan* p) {
  const bool kqv = c->codec == KVQ_CODEC_KQV, hqmq = c->codec == KVQ_CODEC_HQMQ;
  DecodeVariant v{nullptr, nullptr, 0, 0};
  if (!kqv && !hqmq) {
    v = select_decode_kernel(c->head_dim, c->k_bits, c->k_group, c->outliers);
    if (!v.kernel) return fail(KVQ_ERR_UNSUPPORTED, "no decode kernel for this codec");
  }
  DeviceInfo di;
  int rc = device_info(&di, nullptr);
  if (rc) return rc;
  int occ = 1;
  if ((rc = kqv    ? kqv_occupancy(c->head_dim, &occ)
            : hqmq ? hqmq_occupancy(c->head_dim, c->hq_s, c->outliers, &occ)
                   : decode_occupancy(v, &occ)))
    return rc;
  const int64_t units = (int64_t)num_seqs * c->num_kv_heads;
  const int64_t slots = (int64_t)di.sms * occ;
  int64_t splits = units > 0 ? std::max<int64_t>(1, slots / units) : 1;
  int64_t pps = (max_pages + splits - 1) / splits;
  if (pps > kMaxPagesPerSplit) pps = kMaxPagesPerSplit;
  // KVQ_PAGES_PER_SPLIT overrides the split size (tuning and tests)
  if (const char* env = std::getenv("KVQ_PAGES_PER_SPLIT")) {
    const long o = std::strtol(env, nullptr, 10);
    if (o > 0) pps = o;
  }
  if (pps < 1) pps = 1;
  splits = (max_pages + pps - 1) / pps;
  if (splits < 1) splits = 1;
  p->splits = (int)splits;
  p->pps = (int)pps;
  p->counter_bytes = ((size_t)units * sizeof(int) + 255) / 256 * 256;
  p->part_bytes = (size_t)units * splits *
                  (kqv ? kqv_record_floats(c->head_dim)
                       : hqmq ? hqmq_record_floats(c->head_dim) : v.record) *
                  sizeof(float);
  return KVQ_OK;
}

// The step's new token for kvq_decode_attention_append (NULL: plain decode).
struct NewToken {
  const void* k;
  const void* v;
  int bf16;
  int64_t seq_stride, head_stride;
};

int decode_impl(const kvq_cache* cache, const void* q, int q_dtype, int32_t num_seqs,
                int32_t num_queries, int32_t num_q_heads, const int32_t* page_table,
                int32_t max_pages, const int32_t* seq_lens, float softmax_scale, float tau,
                float* out, float* bound, uint8_t* flags, void* ws, size_t ws_bytes,
                cudaStream_t stream, const NewToken* nt = nullptr) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (num_seqs < 0 || num_queries < 1 || num_q_heads < 1 || max_pages < 1)
    return fail(KVQ_ERR_INVALID_ARG, "bad sizes (num_seqs %d, num_queries %d, num_q_heads %d, "
                "max_pages_per_seq %d)", num_seqs, num_queries, num_q_heads, max_pages);
  if (num_q_heads % cache->num_kv_heads)
    return fail(KVQ_ERR_INVALID_ARG, "num_q_heads %d not a multiple of num_kv_heads %d",
                num_q_heads, cache->num_kv_heads);
  const int G = num_q_heads / cache->num_kv_heads;
  if ((int64_t)num_queries * G > 4)
    return fail(KVQ_ERR_UNSUPPORTED, "num_queries * (num_q_heads/num_kv_heads) = %d > 4",
                num_queries * G);
  if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad q_dtype");
  if (num_seqs == 0) return KVQ_OK;
  if (!q || !page_table || !seq_lens || !bound || !flags)
    return fail(KVQ_ERR_INVALID_ARG, "NULL q, page_table, seq_lens, bound or flags");
  if (std::isnan(tau)) return fail(KVQ_ERR_INVALID_ARG, "tau is NaN");
  Plan plan;
  if ((rc = make_plan(cache, num_seqs, max_pages, &plan))) return rc;
  if (!ws || ws_bytes < plan.total())
    return fail(KVQ_ERR_INVALID_ARG, "workspace %zu bytes < %zu required", ws_bytes,
                plan.total());
  if (!aligned16(ws)) return fail(KVQ_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  const bool kqv = cache->codec == KVQ_CODEC_KQV, hqmq = cache->codec == KVQ_CODEC_HQMQ;
  if ((kqv || hqmq) && nt)
    return fail(KVQ_ERR_UNSUPPORTED, "the %s codec has no fused append", kqv ? "KQV" : "HQMQ");
  DecodeVariant v{nullptr, nullptr, 0, 0};
  if (!kqv && !hqmq)
    v = select_decode_kernel(cache->head_dim, cache->k_bits, cache->k_group, cache->outliers);
  DecodeArgs a;
  a.pool = static_cast<const uint8_t*>(cache->pool);
  a.eta = cache->v_eta;
  a.signs = cache->k_rotate ? cache->rot_signs : nullptr;
  a.err = cache->error_word;
  a.q = q;
  a.q_bf16 = q_dtype == KVQ_BF16;
  a.page_table = page_table;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.num_seqs = num_seqs;
  a.nq = num_queries;
  a.hq = num_q_heads;
  a.hkv = cache->num_kv_heads;
  a.G = G;
  a.R = num_queries * G;
  a.num_pages = cache->num_pages;
  a.pps = plan.pps;
  a.s_att = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / std::sqrt((double)cache->head_dim));
  a.tau = tau;
  a.rot_c = rot_constant(cache->head_dim);
  a.out = out;
  a.bound = bound;
  a.flags = flags;
  a.counters = static_cast<int*>(ws);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + plan.counter_bytes);
  a.app_k = nt ? nt->k : nullptr;
  a.app_v = nt ? nt->v : nullptr;
  a.app_bf16 = nt ? nt->bf16 : 0;
  a.app_seq_stride = nt ? nt->seq_stride : 0;
  a.app_head_stride = nt ? nt->head_stride : 0;
  // (sequence x kv head, split): the split index in the slow dimension
  const int64_t units = (int64_t)num_seqs * cache->num_kv_heads;
  if (units > 0x7fffffffLL || plan.splits > 65535)
    return fail(KVQ_ERR_UNSUPPORTED, "grid too large (%lld units, %d splits)", (long long)units,
                plan.splits);
  if (kqv) {
    KqvDecodeArgs ka;
    ka.a = a;
    ka.qjl = cache->qjl;
    ka.qjl_c = kqv_qjl_constant(cache->head_dim);
    ka.nsp = plan.splits;
    kqv_tables(cache->head_dim, &ka.t);
    cudaError_t e = launch_kqv_decode(ka, cache->head_dim, (int)units, plan.splits, stream);
    if (e != cudaSuccess) return cuda_fail(e, "KQV decode launch");
    return KVQ_OK;
  }
  if (hqmq) {
    HqDecodeArgs ha;
    ha.a = a;
    ha.sec = cache->hq_sec;
    ha.S = cache->hq_s;
    ha.nsp = plan.splits;
    ha.outliers = cache->outliers;
    cudaError_t e = launch_hqmq_decode(ha, cache->head_dim, (int)units, plan.splits, stream);
    if (e != cudaSuccess) return cuda_fail(e, "HQMQ decode launch");
    return KVQ_OK;
  }
  dim3 grid((unsigned)units, (unsigned)plan.splits, 1);
  cudaError_t e = launch_pdl(nt ? v.kernel_append : v.kernel, grid, dim3(decode_threads()),
                             (size_t)v.smem, stream, a);
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  return KVQ_OK;
}

bool fault_injected(const char* what) {
  const char* f = std::getenv("KVQ_FAULT");
  return f && std::strcmp(f, what) == 0;
}

}  // namespace

extern "C" {

const char* kvq_status_string(int s) {
  switch (s) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_RANGE: return "KVQ_ERR_RANGE";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
    case KVQ_ERR_TIMEOUT: return "KVQ_ERR_TIMEOUT";
    case KVQ_ERR_DEVICE: return "KVQ_ERR_DEVICE";
    default: return "KVQ_UNKNOWN_STATUS";
  }
}

const char* kvq_last_error(void) { return g_last_error.c_str(); }

size_t kvq_block_bytes(const kvq_cache* cache) {
  if (!cache || cache->page_size != KVQ_PAGE_SIZE) return 0;
  if (cache->head_dim != 64 && cache->head_dim != 128) return 0;
  if (cache->codec == KVQ_CODEC_KQV) {
    if (cache->k_bits != 4 || cache->v_bits != 3 || cache->k_group != cache->head_dim ||
        cache->v_group != cache->head_dim || cache->outliers != 0)
      return 0;
    return (size_t)KqvLayout{cache->head_dim}.bytes();
  }
  if (cache->codec == KVQ_CODEC_HQMQ) {
    if (cache->k_bits != 6 || cache->v_bits != 6 || cache->k_group != 4 || cache->v_group != 4 ||
        cache->k_rotate != 0 || (cache->outliers != 0 && cache->outliers != 1))
      return 0;
    return (size_t)HqLayout{cache->head_dim, cache->outliers}.bytes();
  }
  if (cache->codec != KVQ_CODEC_INT || (cache->k_bits != 8 && cache->k_bits != 4)) return 0;
  if (cache->k_group != 32 && cache->k_group != 64 && cache->k_group != 128) return 0;
  if (cache->head_dim % cache->k_group || cache->v_bits != 4 || cache->v_group != 32) return 0;
  if (cache->outliers != 0 && cache->outliers != 1) return 0;
  return (size_t)layout_of(cache).bytes();
}

size_t kvq_pool_bytes(const kvq_cache* cache) {
  const size_t bb = kvq_block_bytes(cache);
  if (!bb || cache->num_pages < 0 || cache->num_kv_heads < 1) return 0;
  return bb * (size_t)cache->num_pages * (size_t)cache->num_kv_heads;
}

int kvq_quantize_append(const kvq_cache* cache, const void* k, const void* v, int in_dtype,
                        int64_t seq_stride, int64_t head_stride, int64_t token_stride,
                        int32_t num_seqs, int32_t num_tokens, const int32_t* valid_tokens,
                        const int32_t* start_pos, const int32_t* page_table,
                        int32_t max_pages_per_seq, kvq_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad in_dtype");
  if (num_seqs < 0 || num_tokens < 0 || max_pages_per_seq < 1)
    return fail(KVQ_ERR_INVALID_ARG, "bad sizes");
  if (num_seqs == 0 || num_tokens == 0) return KVQ_OK;
  if (!k || !v || !start_pos || !page_table)
    return fail(KVQ_ERR_INVALID_ARG, "NULL k, v, start_pos or page_table");
  if (seq_stride < 0 || head_stride < 0 || token_stride < 0)
    return fail(KVQ_ERR_INVALID_ARG, "negative stride");
  DeviceInfo di;
  if ((rc = device_info(&di, nullptr))) return rc;
  AppendArgs a;
  a.pool = static_cast<uint8_t*>(cache->pool);
  a.eta = cache->v_eta;
  a.signs = cache->k_rotate ? cache->rot_signs : nullptr;
  a.err = cache->error_word;
  a.k = k;
  a.v = v;
  a.in_bf16 = in_dtype == KVQ_BF16;
  a.seq_stride = seq_stride;
  a.head_stride = head_stride;
  a.tok_stride = token_stride;
  a.num_seqs = num_seqs;
  a.num_tokens = num_tokens;
  a.hkv = cache->num_kv_heads;
  a.num_pages = cache->num_pages;
  a.max_pages = max_pages_per_seq;
  a.valid = valid_tokens;
  a.start_pos = start_pos;
  a.page_table = page_table;
  a.rot_c = rot_constant(cache->head_dim);
  if (cache->codec == KVQ_CODEC_KQV) {
    KqvAppendArgs ka;
    ka.a = a;
    ka.qjl = cache->qjl;
    ka.qjl_c = kqv_qjl_constant(cache->head_dim);
    kqv_tables(cache->head_dim, &ka.t);
    cudaError_t e = launch_kqv_append(ka, cache->head_dim, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "KQV append kernel launch");
    return KVQ_OK;
  }
  if (cache->codec == KVQ_CODEC_HQMQ) {
    HqAppendArgs ha;
    ha.a = a;
    ha.sec = cache->hq_sec;
    ha.S = cache->hq_s;
    ha.outliers = cache->outliers;
    cudaError_t e = launch_hqmq_append(ha, cache->head_dim, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "HQMQ append kernel launch");
    return KVQ_OK;
  }
  cudaError_t e = launch_append(a, cache->head_dim, cache->k_bits, cache->k_group, cache->outliers,
                                reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
  return KVQ_OK;
}

size_t kvq_workspace_size(const kvq_cache* cache, int32_t num_seqs, int32_t num_queries,
                          int32_t num_q_heads, int32_t max_pages_per_seq) {
  if (check_cache(cache) || num_seqs < 0 || num_queries < 1 || num_q_heads < 1 ||
      max_pages_per_seq < 1)
    return 0;
  Plan p;
  if (make_plan(cache, num_seqs, max_pages_per_seq, &p)) return 0;
  return p.total();
}

int kvq_decode_attention(const kvq_cache* cache, const void* q, int q_dtype, int32_t num_seqs,
                         int32_t num_queries, int32_t num_q_heads, const int32_t* page_table,
                         int32_t max_pages_per_seq, const int32_t* seq_lens,
                         float softmax_scale, float tau, float* out, float* bound,
                         uint8_t* flags, void* workspace, size_t workspace_bytes,
                         kvq_stream_t stream) {
  if (!out && num_seqs > 0) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
  return decode_impl(cache, q, q_dtype, num_seqs, num_queries, num_q_heads, page_table,
                     max_pages_per_seq, seq_lens, softmax_scale, tau, out, bound, flags,
                     workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int kvq_error_bound(const kvq_cache* cache, const void* q, int q_dtype, int32_t num_seqs,
                    int32_t num_queries, int32_t num_q_heads, const int32_t* page_table,
                    int32_t max_pages_per_seq, const int32_t* seq_lens, float softmax_scale,
                    float tau, float* bound, uint8_t* flags, void* workspace,
                    size_t workspace_bytes, kvq_stream_t stream) {
  return decode_impl(cache, q, q_dtype, num_seqs, num_queries, num_q_heads, page_table,
                     max_pages_per_seq, seq_lens, softmax_scale, tau, nullptr, bound, flags,
                     workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int kvq_decode_attention_append(const kvq_cache* cache, const void* k_new, const void* v_new,
                                int in_dtype, int64_t new_seq_stride, int64_t new_head_stride,
                                const void* q, int q_dtype, int32_t num_seqs, int32_t num_queries,
                                int32_t num_q_heads, const int32_t* page_table,
                                int32_t max_pages_per_seq, const int32_t* seq_lens,
                                float softmax_scale, float tau, float* out, float* bound,
                                uint8_t* flags, void* workspace, size_t workspace_bytes,
                                kvq_stream_t stream) {
  if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad in_dtype");
  if (new_seq_stride < 0 || new_head_stride < 0)
    return fail(KVQ_ERR_INVALID_ARG, "negative stride");
  if (num_seqs > 0 && (!k_new || !v_new)) return fail(KVQ_ERR_INVALID_ARG, "NULL k_new or v_new");
  if (!out && num_seqs > 0) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
  const NewToken nt{k_new, v_new, in_dtype == KVQ_BF16, new_seq_stride, new_head_stride};
  return decode_impl(cache, q, q_dtype, num_seqs, num_queries, num_q_heads, page_table,
                     max_pages_per_seq, seq_lens, softmax_scale, tau, out, bound, flags, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream), &nt);
}

size_t kvq_fallback_staging_size(const kvq_cache* cache, int orig_dtype, int32_t max_ctx) {
  if (!cache || (cache->head_dim != 64 && cache->head_dim != 128) || max_ctx < 0) return 0;
  if (orig_dtype != KVQ_F32 && orig_dtype != KVQ_BF16) return 0;
  const size_t es = orig_dtype == KVQ_BF16 ? 2 : 4;
  const size_t one = ((size_t)max_ctx * cache->head_dim * es + 255) / 256 * 256;
  return fallback_scratch_bytes(cache->head_dim) + 2 * one;
}

int kvq_fallback_exact(const kvq_cache* cache, const void* k_orig_host, const void* v_orig_host,
                       int orig_dtype, int64_t orig_seq_stride, int64_t orig_head_stride,
                       const void* q, int q_dtype, int32_t num_seqs, int32_t num_queries,
                       int32_t num_q_heads, const int32_t* seq_lens_host, float softmax_scale,
                       const uint8_t* flags, uint8_t* flags_host, float* out, void* staging,
                       size_t staging_bytes, kvq_stream_t main_stream, kvq_stream_t side_stream,
                       int32_t timeout_ms, int32_t* num_fallback) {
  if (num_fallback) *num_fallback = 0;
  if (!cache) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
  if (cache->head_dim != 64 && cache->head_dim != 128)
    return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d unsupported", cache->head_dim);
  if (cache->num_kv_heads < 1) return fail(KVQ_ERR_INVALID_ARG, "num_kv_heads < 1");
  if (orig_dtype != KVQ_F32 && orig_dtype != KVQ_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad orig_dtype");
  if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad q_dtype");
  if (num_seqs < 0 || num_queries < 1 || num_q_heads < 1 || num_q_heads % cache->num_kv_heads)
    return fail(KVQ_ERR_INVALID_ARG, "bad sizes");
  if (num_seqs == 0) return KVQ_OK;
  if (!k_orig_host || !v_orig_host || !q || !seq_lens_host || !flags || !flags_host || !out ||
      !staging || !num_fallback)
    return fail(KVQ_ERR_INVALID_ARG, "NULL argument");
  if (orig_seq_stride < 0 || orig_head_stride < 0) return fail(KVQ_ERR_INVALID_ARG, "negative stride");
  if (reinterpret_cast<uintptr_t>(staging) % 16)
    return fail(KVQ_ERR_INVALID_ARG, "staging is not 16-byte aligned");
  const int D = cache->head_dim, hkv = cache->num_kv_heads, G = num_q_heads / hkv;
  const size_t es = orig_dtype == KVQ_BF16 ? 2 : 4;
  int32_t max_n = 0;
  for (int s = 0; s < num_seqs; ++s) {
    if (seq_lens_host[s] < 0) return fail(KVQ_ERR_INVALID_ARG, "negative seq_len");
    max_n = std::max(max_n, seq_lens_host[s]);
  }
  if (staging_bytes < kvq_fallback_staging_size(cache, orig_dtype, max_n))
    return fail(KVQ_ERR_INVALID_ARG, "staging %zu bytes < %zu required", staging_bytes,
                kvq_fallback_staging_size(cache, orig_dtype, max_n));
  DeviceInfo di;
  int rc = device_info(&di, nullptr);
  if (rc) return rc;
  cudaStream_t ms = reinterpret_cast<cudaStream_t>(main_stream);
  cudaStream_t ss = reinterpret_cast<cudaStream_t>(side_stream);
  const size_t rows = (size_t)num_seqs * num_queries * num_q_heads;

  // the decode, the flags on the host, the copies of the open batch, and the
  // last recompute that read each staging half
  cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  cudaEvent_t& ev_dec = ev[0];
  cudaEvent_t& ev_flags = ev[1];
  cudaEvent_t& ev_copied = ev[2];
  cudaEvent_t* ev_half = ev + 3;
  auto cleanup = [&]() {
    for (cudaEvent_t& x : ev)
      if (x) cudaEventDestroy(x);
  };
  cudaError_t e;
  for (cudaEvent_t& x : ev)
    if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess) {
      cleanup();
      return cuda_fail(e, "cudaEventCreate");
    }
  // flags -> host on the side stream, after the decode on the main stream
  if ((e = cudaEventRecord(ev_dec, ms)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(ss, ev_dec, 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(flags_host, flags, rows, cudaMemcpyDeviceToHost, ss)) != cudaSuccess ||
      (e = cudaEventRecord(ev_flags, ss)) != cudaSuccess) {
    cleanup();
    return cuda_fail(e, "flag read-back");
  }
  // bounded wait for the flags
  {
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
      const double ms_el =
          std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
      if (ms_el >= (double)timeout_ms) {
        cleanup();
        return fail(KVQ_ERR_TIMEOUT, "flags not ready after %d ms", timeout_ms);
      }
      e = cudaEventQuery(ev_flags);
      if (e == cudaSuccess) break;
      if (e != cudaErrorNotReady) {
        cleanup();
        return cuda_fail(e, "cudaEventQuery");
      }
      std::this_thread::sleep_for(std::chrono::microseconds(20));
    }
  }
  // Page in and recompute.  The staging buffer holds the merge scratch, then
  // two halves when there is room for the longest (sequence, kv head) in each,
  // else one region.  The originals go in on `side`; a batch's recompute runs
  // on `main` after its copies, and the next copies into the same half wait
  // for that recompute, so one half is being filled while the other is read.
  const size_t scratch = fallback_scratch_bytes(D);
  const size_t pair_max = 2 * (((size_t)max_n * D * es + 255) / 256 * 256);
  const size_t region = staging_bytes - scratch;
  const int halves = pair_max > 0 && region >= 2 * pair_max ? 2 : 1;
  const size_t half_bytes = halves == 2 ? region / 2 / 256 * 256 : region;
  FbArgs fa;
  std::memset(&fa, 0, sizeof(fa));
  fa.staging = static_cast<const uint8_t*>(staging);
  fa.q = q;
  fa.out = out;
  fa.scratch = static_cast<float*>(staging);
  fa.q_bf16 = q_dtype == KVQ_BF16;
  fa.kv_bf16 = orig_dtype == KVQ_BF16;
  fa.s_att = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / std::sqrt((double)D));
  int half = 0;
  bool half_read[2] = {false, false};
  size_t used = 0;
  int32_t count = 0;
  // the recompute of the items gathered so far, after every copy issued so far
  auto launch = [&]() -> int {
    if (fa.num_items == 0) return KVQ_OK;
    if ((e = cudaEventRecord(ev_copied, ss)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(ms, ev_copied, 0)) != cudaSuccess)
      return cuda_fail(e, "copy hand-off");
    if ((e = launch_fallback(fa, D, ms)) != cudaSuccess) return cuda_fail(e, "fallback kernel launch");
    fa.num_items = 0;
    fa.any_split = 0;
    return KVQ_OK;
  };
  // close the batch in the current half and open the other one
  auto next_half = [&]() -> int {
    int r = launch();
    if (r) return r;
    if ((e = cudaEventRecord(ev_half[half], ms)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    half_read[half] = true;
    half = (half + 1) % halves;
    used = 0;
    if (half_read[half] && (e = cudaStreamWaitEvent(ss, ev_half[half], 0)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamWaitEvent");
    return KVQ_OK;
  };
  std::vector<int64_t> rws;
  for (int s = 0; s < num_seqs; ++s) {
    for (int h = 0; h < hkv; ++h) {
      rws.clear();
      for (int i = 0; i < num_queries; ++i)
        for (int gq = 0; gq < G; ++gq) {
          const int64_t row = ((int64_t)s * num_queries + i) * num_q_heads + h * G + gq;
          if (flags_host[row]) rws.push_back(row);
        }
      if (rws.empty()) continue;
      const int n = seq_lens_host[s];
      const size_t one = ((size_t)n * D * es + 255) / 256 * 256;
      if (used + 2 * one > half_bytes)
        if ((rc = next_half())) { cleanup(); return rc; }
      const int64_t koff = (int64_t)(scratch + half * half_bytes + used);
      const int64_t voff = koff + (int64_t)one;
      if (n > 0) {
        if (fault_injected("memcpy")) {
          cleanup();
          return fail(KVQ_ERR_CUDA, "cudaMemcpyAsync failed (injected fault)");
        }
        const uint8_t* kh = static_cast<const uint8_t*>(k_orig_host) +
                            ((int64_t)s * orig_seq_stride + (int64_t)h * orig_head_stride) * es;
        const uint8_t* vh = static_cast<const uint8_t*>(v_orig_host) +
                            ((int64_t)s * orig_seq_stride + (int64_t)h * orig_head_stride) * es;
        if ((e = cudaMemcpyAsync(static_cast<uint8_t*>(staging) + koff, kh, (size_t)n * D * es,
                                 cudaMemcpyHostToDevice, ss)) != cudaSuccess ||
            (e = cudaMemcpyAsync(static_cast<uint8_t*>(staging) + voff, vh, (size_t)n * D * es,
                                 cudaMemcpyHostToDevice, ss)) != cudaSuccess) {
          cleanup();
          return cuda_fail(e, "cudaMemcpyAsync (Tier-2 page-in)");
        }
      }
      used += 2 * one;
      // items: row groups of up to kFbRows, each cut into nchunk token ranges
      const int nchunk = n <= kFbMinChunk ? 1 : std::min(kFbMaxChunks, (n + kFbMinChunk - 1) / kFbMinChunk);
      const int clen = (n + nchunk - 1) / nchunk;
      for (size_t g0 = 0; g0 < rws.size(); g0 += kFbRows) {
        const int nrw = (int)std::min<size_t>(kFbRows, rws.size() - g0);
        if (fa.num_items + nchunk > kFbMaxItems)
          if ((rc = launch())) { cleanup(); return rc; }
        for (int c = 0; c < nchunk; ++c) {
          FbItem& it = fa.items[fa.num_items++];
          it.k_off = koff;
          it.v_off = voff;
          it.row0 = rws[g0];
          it.t0 = c * clen;
          it.t1 = std::min(n, (c + 1) * clen);
          for (int r = 0; r < kFbRows; ++r) it.roff[r] = r < nrw ? (int32_t)(rws[g0 + r] - rws[g0]) : 0;
          it.nrows = (int16_t)nrw;
          it.chunk = (int16_t)c;
          it.nchunk = (int16_t)nchunk;
        }
        if (nchunk > 1) fa.any_split = 1;
        count += nrw;
      }
    }
  }
  if ((rc = launch())) { cleanup(); return rc; }
  cleanup();
  *num_fallback = count;
  return KVQ_OK;
}

}  // extern "C"

namespace {

// Work-buffer layout of kvq_adaptive_precision for at most `units` flagged
// (sequence, kv head) units, `slots` flagged rows and `mp` pages per sequence.
struct AdLayout {
  size_t units, items, kp, vp, korder, blse, nkey, nval, rank_fail, um, smap, part, total;
};
constexpr int kAdMaxChunks = 8;      // page ranges per unit in the correction
constexpr int kAdMinChunkPages = 16;
constexpr int kAdMaxPages = 8192;    // the selection sorts one row's pages in shared memory

AdLayout ad_layout(int64_t units, int64_t slots, int64_t mp, int d) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  AdLayout L;
  size_t o = 0;
  L.units = o; o += up(units * sizeof(AdUnit));
  L.items = o; o += up(units * kAdMaxChunks * sizeof(AdItem));
  L.kp = o; o += up(slots * mp);
  L.vp = o; o += up(slots * mp);
  L.korder = o; o += up(slots * mp * 4);
  L.blse = o; o += up(slots * mp * 4);
  L.nkey = o; o += up(slots * 4);
  L.nval = o; o += up(slots * 4);
  L.rank_fail = o; o += up(slots);
  L.um = o; o += up(units * mp);
  L.smap = o; o += up(units * mp * 4);
  L.part = o; o += up(units * kAdMaxChunks * adaptive_part_floats(d) * sizeof(float));
  L.total = o;
  return L;
}

// Pinned host scratch: the units, the union of promoted pages per unit and
// the staged-page maps, each written once per call.
size_t ad_host_bytes(int64_t units, int64_t mp) {
  return ((size_t)units * sizeof(AdUnit) + 255) / 256 * 256 + (size_t)units * mp +
         (size_t)units * mp * 4 + 256;
}

// Polls `ev` until it completes or the deadline passes (a deadline already
// passed times out at once, as a timeout of 0 ms does).
int wait_event_until(cudaEvent_t ev, std::chrono::steady_clock::time_point deadline,
                     const char* what) {
  for (;;) {
    if (std::chrono::steady_clock::now() >= deadline)
      return fail(KVQ_ERR_TIMEOUT, "%s: not complete before the deadline", what);
    cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return KVQ_OK;
    if (e != cudaErrorNotReady) return cuda_fail(e, what);
    std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

}  // namespace

extern "C" {

size_t kvq_adaptive_work_size(const kvq_cache* cache, int32_t num_seqs, int32_t num_queries,
                              int32_t num_q_heads, int32_t max_pages_per_seq) {
  if (check_cache(cache) || cache->codec != KVQ_CODEC_INT || num_seqs < 0 ||
      num_queries < 1 ||
      num_q_heads < 1 || max_pages_per_seq < 1 || max_pages_per_seq > kAdMaxPages)
    return 0;
  const int64_t units = (int64_t)num_seqs * cache->num_kv_heads;
  const int64_t slots = (int64_t)num_seqs * num_queries * num_q_heads;
  return ad_layout(units, slots, max_pages_per_seq, cache->head_dim).total;
}

size_t kvq_adaptive_host_size(const kvq_cache* cache, int32_t num_seqs,
                              int32_t max_pages_per_seq) {
  if (!cache || cache->num_kv_heads < 1 || num_seqs < 0 || max_pages_per_seq < 1) return 0;
  return ad_host_bytes((int64_t)num_seqs * cache->num_kv_heads, max_pages_per_seq);
}

size_t kvq_adaptive_staging_size(const kvq_cache* cache, int orig_dtype,
                                 int32_t max_pages_per_seq) {
  if (!cache || (cache->head_dim != 64 && cache->head_dim != 128) || max_pages_per_seq < 1)
    return 0;
  if (orig_dtype != KVQ_F32 && orig_dtype != KVQ_BF16) return 0;
  const size_t es = orig_dtype == KVQ_BF16 ? 2 : 4;
  return 2 * (size_t)max_pages_per_seq * KVQ_PAGE_SIZE * cache->head_dim * es;
}

int kvq_adaptive_precision(const kvq_cache* cache, const void* k_orig_host,
                           const void* v_orig_host, int orig_dtype, int64_t orig_seq_stride,
                           int64_t orig_head_stride, const void* q, int q_dtype,
                           int32_t num_seqs, int32_t num_queries, int32_t num_q_heads,
                           const int32_t* page_table, int32_t max_pages_per_seq,
                           const int32_t* seq_lens, const int32_t* seq_lens_host,
                           float softmax_scale, float tau, float tau_cov, float v_tol,
                           float rank_tol, uint8_t* flags, uint8_t* flags_host, float* out,
                           float* bound, uint8_t* promoted_keys, uint8_t* promoted_values,
                           void* work, size_t work_bytes, void* host_work,
                           size_t host_work_bytes, void* staging, size_t staging_bytes,
                           kvq_stream_t main_stream, kvq_stream_t side_stream,
                           int32_t timeout_ms, int32_t* num_rows, int32_t* num_flagged) {
  if (num_rows) *num_rows = 0;
  if (num_flagged) *num_flagged = 0;
  int rc = check_cache(cache);
  if (rc) return rc;
  if (cache->codec != KVQ_CODEC_INT)
    return fail(KVQ_ERR_UNSUPPORTED, "the adaptive-precision ladder reads Tier-1 caches only");
  if (orig_dtype != KVQ_F32 && orig_dtype != KVQ_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad orig_dtype");
  if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad q_dtype");
  if (num_seqs < 0 || num_queries < 1 || num_q_heads < 1 || max_pages_per_seq < 1 ||
      num_q_heads % cache->num_kv_heads)
    return fail(KVQ_ERR_INVALID_ARG, "bad sizes");
  const int D = cache->head_dim, hkv = cache->num_kv_heads, G = num_q_heads / hkv;
  if ((int64_t)num_queries * G > 4)
    return fail(KVQ_ERR_UNSUPPORTED, "num_queries * (num_q_heads/num_kv_heads) = %d > 4",
                num_queries * G);
  if (max_pages_per_seq > kAdMaxPages)
    return fail(KVQ_ERR_UNSUPPORTED, "max_pages_per_seq %d > %d", max_pages_per_seq, kAdMaxPages);
  if (std::isnan(tau) || std::isnan(tau_cov) || std::isnan(v_tol) || std::isnan(rank_tol))
    return fail(KVQ_ERR_INVALID_ARG, "NaN threshold");
  if (num_seqs == 0) return KVQ_OK;
  if (!k_orig_host || !v_orig_host || !q || !page_table || !seq_lens || !seq_lens_host ||
      !flags || !flags_host || !out || !bound || !work || !host_work || !staging ||
      !num_rows || !num_flagged)
    return fail(KVQ_ERR_INVALID_ARG, "NULL argument");
  if (orig_seq_stride < 0 || orig_head_stride < 0) return fail(KVQ_ERR_INVALID_ARG, "negative stride");
  if (!aligned16(work) || !aligned16(staging) || !aligned16(host_work))
    return fail(KVQ_ERR_INVALID_ARG, "work, host_work or staging not 16-byte aligned");
  const int mp = max_pages_per_seq;
  const int64_t units_max = (int64_t)num_seqs * hkv;
  const int64_t rows = (int64_t)num_seqs * num_queries * num_q_heads;
  const AdLayout WL = ad_layout(units_max, rows, mp, D);
  if (work_bytes < WL.total)
    return fail(KVQ_ERR_INVALID_ARG, "work %zu bytes < %zu required", work_bytes, WL.total);
  if (host_work_bytes < ad_host_bytes(units_max, mp))
    return fail(KVQ_ERR_INVALID_ARG, "host_work %zu bytes < %zu required", host_work_bytes,
                ad_host_bytes(units_max, mp));
  const size_t es = orig_dtype == KVQ_BF16 ? 2 : 4;
  const size_t page_bytes = (size_t)KVQ_PAGE_SIZE * D * es;
  for (int s = 0; s < num_seqs; ++s)
    if (seq_lens_host[s] < 0 || seq_lens_host[s] > mp * KVQ_PAGE_SIZE)
      return fail(KVQ_ERR_INVALID_ARG, "seq_lens_host[%d] = %d outside [0, %d]", s,
                  seq_lens_host[s], mp * KVQ_PAGE_SIZE);
  DeviceInfo di;
  if ((rc = device_info(&di, nullptr))) return rc;
  const int smem = adaptive_select_smem(mp, D);
  if (smem > di.max_smem)
    return fail(KVQ_ERR_UNSUPPORTED, "selection needs %d bytes of shared memory", smem);
  cudaStream_t ms = reinterpret_cast<cudaStream_t>(main_stream);
  cudaStream_t ss = reinterpret_cast<cudaStream_t>(side_stream);
  const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);

  cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
  auto cleanup = [&]() {
    for (cudaEvent_t& x : ev)
      if (x) cudaEventDestroy(x);
  };
  cudaError_t e;
  for (cudaEvent_t& x : ev)
    if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess) {
      cleanup();
      return cuda_fail(e, "cudaEventCreate");
    }
  auto bail = [&](int code) { cleanup(); return code; };
  // 1. the decode's flags on the host (side stream, after the decode on main)
  if ((e = cudaEventRecord(ev[0], ms)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(ss, ev[0], 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(flags_host, flags, rows, cudaMemcpyDeviceToHost, ss)) != cudaSuccess ||
      (e = cudaEventRecord(ev[1], ss)) != cudaSuccess)
    return bail(cuda_fail(e, "flag read-back"));
  if ((rc = wait_event_until(ev[1], deadline, "flag read-back"))) return bail(rc);

  // 2. flagged units and their rows (row slots are the flagged rows, in order)
  uint8_t* hw = static_cast<uint8_t*>(host_work);
  AdUnit* hunits = reinterpret_cast<AdUnit*>(hw);
  uint8_t* hum = hw + ((size_t)units_max * sizeof(AdUnit) + 255) / 256 * 256;
  int32_t* hsmap = reinterpret_cast<int32_t*>(hum + (size_t)units_max * mp);
  hsmap = reinterpret_cast<int32_t*>((reinterpret_cast<uintptr_t>(hsmap) + 15) / 16 * 16);
  int nu = 0, nslots = 0;
  for (int s = 0; s < num_seqs; ++s)
    for (int h = 0; h < hkv; ++h) {
      AdUnit un;
      std::memset(&un, 0, sizeof(un));
      un.seq = s;
      un.kvh = h;
      un.rslot = nslots;
      for (int i = 0; i < num_queries; ++i)
        for (int gq = 0; gq < G; ++gq) {
          const int64_t row = ((int64_t)s * num_queries + i) * num_q_heads + h * G + gq;
          if (flags_host[row]) un.rows[un.nrows++] = (int32_t)row;
        }
      if (un.nrows == 0) continue;
      nslots += un.nrows;
      hunits[nu++] = un;
    }
  *num_rows = nslots;
  if (nu == 0) return bail(KVQ_OK);

  uint8_t* wb = static_cast<uint8_t*>(work);
  AdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.pool = static_cast<const uint8_t*>(cache->pool);
  a.eta = cache->v_eta;
  a.signs = cache->k_rotate ? cache->rot_signs : nullptr;
  a.err = cache->error_word;
  a.q = q;
  a.q_bf16 = q_dtype == KVQ_BF16;
  a.kv_bf16 = orig_dtype == KVQ_BF16;
  a.page_table = page_table;
  a.max_pages = mp;
  a.seq_lens = seq_lens;
  a.nq = num_queries;
  a.hq = num_q_heads;
  a.hkv = hkv;
  a.G = G;
  a.num_pages = cache->num_pages;
  a.outliers = cache->outliers;
  a.s_att = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / std::sqrt((double)D));
  a.rot_c = rot_constant(D);
  a.tau = tau;
  a.tau_cov = tau_cov;
  a.v_tol = v_tol;
  a.rank_tol = rank_tol;
  a.kp = wb + WL.kp;
  a.vp = wb + WL.vp;
  a.korder = reinterpret_cast<int32_t*>(wb + WL.korder);
  a.blse = reinterpret_cast<float*>(wb + WL.blse);
  a.nkey = reinterpret_cast<int32_t*>(wb + WL.nkey);
  a.nval = reinterpret_cast<int32_t*>(wb + WL.nval);
  a.rank_fail = wb + WL.rank_fail;
  a.out = out;
  a.bound = bound;
  a.flags = flags;
  a.staging = static_cast<const uint8_t*>(staging);
  AdUnit* d_units = reinterpret_cast<AdUnit*>(wb + WL.units);
  AdItem* d_items = reinterpret_cast<AdItem*>(wb + WL.items);
  uint8_t* d_um = wb + WL.um;
  int32_t* d_smap = reinterpret_cast<int32_t*>(wb + WL.smap);

  // 3. scoring pass and selection for every flagged unit; the union of promoted
  //    pages per unit back to the host
  if ((e = cudaMemcpyAsync(d_units, hunits, (size_t)nu * sizeof(AdUnit), cudaMemcpyHostToDevice,
                           ms)) != cudaSuccess)
    return bail(cuda_fail(e, "unit list H2D"));
  a.units = d_units;
  a.num_units = nu;
  a.um = d_um;
  if ((e = launch_adaptive_select(a, D, cache->k_bits, cache->k_group, smem, ms)) != cudaSuccess)
    return bail(cuda_fail(e, "selection kernel launch"));
  if ((e = cudaMemcpyAsync(hum, d_um, (size_t)nu * mp, cudaMemcpyDeviceToHost, ms)) != cudaSuccess ||
      (e = cudaEventRecord(ev[2], ms)) != cudaSuccess)
    return bail(cuda_fail(e, "promoted-page read-back"));
  if ((rc = wait_event_until(ev[2], deadline, "promoted-page read-back"))) return bail(rc);

  // 4. staged-page maps; batches of units whose promoted pages fit the staging
  std::vector<int64_t> stage_bytes(nu);
  for (int iu = 0; iu < nu; ++iu) {
    const uint8_t* um = hum + (size_t)iu * mp;
    int32_t* sm = hsmap + (size_t)iu * mp;
    int k = 0;
    for (int b = 0; b < mp; ++b) sm[b] = um[b] ? k++ : -1;
    hunits[iu].nstaged = k;
    stage_bytes[iu] = 2 * (int64_t)k * (int64_t)page_bytes;
    if (stage_bytes[iu] > (int64_t)staging_bytes)
      return bail(fail(KVQ_ERR_INVALID_ARG, "staging %zu bytes < %lld needed by one (sequence, "
                       "kv head)", staging_bytes, (long long)stage_bytes[iu]));
  }
  if ((e = cudaMemcpyAsync(d_smap, hsmap, (size_t)nu * mp * 4, cudaMemcpyHostToDevice, ms)) !=
      cudaSuccess)
    return bail(cuda_fail(e, "page map H2D"));
  bool staging_read = false;   // ev[3]: the last correction that read the staging
  std::vector<AdItem> items;
  for (int b0 = 0; b0 < nu;) {
    // the batch [b0, b1)
    int64_t used = 0;
    int b1 = b0;
    while (b1 < nu && used + stage_bytes[b1] <= (int64_t)staging_bytes) used += stage_bytes[b1++];
    items.clear();
    int64_t off = 0;
    for (int iu = b0; iu < b1; ++iu) {
      hunits[iu].stage_off = off;
      off += stage_bytes[iu];
      const int n = seq_lens_host[hunits[iu].seq];
      const int npg = (n + KVQ_PAGE_SIZE - 1) / KVQ_PAGE_SIZE;
      const int nch = std::max(1, std::min(kAdMaxChunks, (npg + kAdMinChunkPages - 1) / kAdMinChunkPages));
      const int per = (npg + nch - 1) / nch;
      const int first = (int)items.size();
      for (int c = 0; c < nch; ++c) {
        AdItem it;
        it.unit = iu - b0;
        it.p0 = std::min(npg, c * per);
        it.p1 = std::min(npg, (c + 1) * per);
        it.chunk = c;
        it.nchunk = nch;
        it.first = first;
        items.push_back(it);
      }
    }
    // the batch's unit records (stage offsets) and items
    if ((e = cudaMemcpyAsync(d_units + b0, hunits + b0, (size_t)(b1 - b0) * sizeof(AdUnit),
                             cudaMemcpyHostToDevice, ms)) != cudaSuccess ||
        (e = cudaMemcpyAsync(d_items, items.data(), items.size() * sizeof(AdItem),
                             cudaMemcpyHostToDevice, ms)) != cudaSuccess)
      return bail(cuda_fail(e, "batch H2D"));
    // page-in on the side stream, after the correction that last read the staging
    if (staging_read && (e = cudaStreamWaitEvent(ss, ev[3], 0)) != cudaSuccess)
      return bail(cuda_fail(e, "cudaStreamWaitEvent"));
    for (int iu = b0; iu < b1; ++iu) {
      const AdUnit& un = hunits[iu];
      const int n = seq_lens_host[un.seq];
      const uint8_t* um = hum + (size_t)iu * mp;
      const int32_t* sm = hsmap + (size_t)iu * mp;
      const int64_t src0 = ((int64_t)un.seq * orig_seq_stride + (int64_t)un.kvh * orig_head_stride) * es;
      uint8_t* dk = static_cast<uint8_t*>(staging) + un.stage_off;
      uint8_t* dv = dk + (size_t)un.nstaged * page_bytes;
      for (int b = 0; b < mp;) {
        if (!um[b]) { ++b; continue; }
        int e2 = b;
        while (e2 < mp && um[e2]) ++e2;
        const int64_t t0 = (int64_t)b * KVQ_PAGE_SIZE;
        const int64_t t1 = std::min<int64_t>((int64_t)e2 * KVQ_PAGE_SIZE, n);
        if (t1 > t0) {
          if (fault_injected("memcpy")) return bail(fail(KVQ_ERR_CUDA, "cudaMemcpyAsync failed (injected fault)"));
          const size_t bytes = (size_t)(t1 - t0) * D * es;
          const size_t soff = (size_t)sm[b] * page_bytes;
          const uint8_t* kh = static_cast<const uint8_t*>(k_orig_host) + src0 + t0 * D * es;
          const uint8_t* vh = static_cast<const uint8_t*>(v_orig_host) + src0 + t0 * D * es;
          if ((e = cudaMemcpyAsync(dk + soff, kh, bytes, cudaMemcpyHostToDevice, ss)) != cudaSuccess ||
              (e = cudaMemcpyAsync(dv + soff, vh, bytes, cudaMemcpyHostToDevice, ss)) != cudaSuccess)
            return bail(cuda_fail(e, "cudaMemcpyAsync (Tier-2 page-in)"));
        }
        b = e2;
      }
    }
    // correction and finish on main, after the copies
    AdArgs ab = a;
    ab.units = d_units + b0;
    ab.num_units = b1 - b0;
    ab.items = d_items;
    ab.num_items = (int)items.size();
    ab.smap = d_smap + (size_t)b0 * mp;
    ab.part = reinterpret_cast<float*>(wb + WL.part);
    if ((e = cudaEventRecord(ev[0], ss)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(ms, ev[0], 0)) != cudaSuccess)
      return bail(cuda_fail(e, "copy hand-off"));
    if ((e = launch_adaptive_correct(ab, D, cache->k_bits, cache->k_group, ms)) != cudaSuccess ||
        (e = launch_adaptive_finish(ab, D, ms)) != cudaSuccess)
      return bail(cuda_fail(e, "correction kernel launch"));
    if ((e = cudaEventRecord(ev[3], ms)) != cudaSuccess) return bail(cuda_fail(e, "cudaEventRecord"));
    staging_read = true;
    // the items and unit records of the next batch overwrite these: wait (bounded)
    if (b1 < nu && (rc = wait_event_until(ev[3], deadline, "correction batch"))) return bail(rc);
    b0 = b1;
  }
  // 5. per-row promotion maps for the caller; the new flags on the host
  for (int iu = 0; iu < nu && (promoted_keys || promoted_values); ++iu)
    for (int r = 0; r < hunits[iu].nrows; ++r) {
      const int64_t row = hunits[iu].rows[r];
      const size_t so = (size_t)(hunits[iu].rslot + r) * mp;
      if (promoted_keys &&
          (e = cudaMemcpyAsync(promoted_keys + row * mp, a.kp + so, mp, cudaMemcpyDeviceToDevice, ms)) != cudaSuccess)
        return bail(cuda_fail(e, "promotion map copy"));
      if (promoted_values &&
          (e = cudaMemcpyAsync(promoted_values + row * mp, a.vp + so, mp, cudaMemcpyDeviceToDevice, ms)) != cudaSuccess)
        return bail(cuda_fail(e, "promotion map copy"));
    }
  if ((e = cudaMemcpyAsync(flags_host, flags, rows, cudaMemcpyDeviceToHost, ms)) != cudaSuccess ||
      (e = cudaEventRecord(ev[2], ms)) != cudaSuccess)
    return bail(cuda_fail(e, "flag read-back"));
  if ((rc = wait_event_until(ev[2], deadline, "final flag read-back"))) return bail(rc);
  int cnt = 0;
  for (int64_t r = 0; r < rows; ++r) cnt += flags_host[r] != 0;
  *num_flagged = cnt;
  return bail(KVQ_OK);
}

int kvq_device_error(const kvq_cache* cache, kvq_stream_t stream, int32_t* code) {
  if (!cache || !code) return fail(KVQ_ERR_INVALID_ARG, "NULL argument");
  *code = KVQ_OK;
  if (!cache->error_word) return KVQ_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int32_t v = 0;
  if ((e = cudaMemcpyAsync(&v, cache->error_word, sizeof(v), cudaMemcpyDeviceToHost, s)) !=
          cudaSuccess ||
      (e = cudaMemsetAsync(cache->error_word, 0, sizeof(v), s)) != cudaSuccess ||
      (e = cudaStreamSynchronize(s)) != cudaSuccess)
    return cuda_fail(e, "error word read-back");
  *code = v;
  return KVQ_OK;
}

}  // extern "C"

// ---- decode without caller-provided workspace ---------------------------------------
// For callers that cannot allocate device memory at the point of the call (an
// allocator-free runtime, a host that hands the library fixed buffers, code
// running where cudaMalloc is forbidden or would synchronize): the split-K
// scratch lives in this static device array instead of a caller workspace.
// Each GPU that loads the library holds KVQ_NOALLOC_SCRATCH_BYTES of it until
// the process exits.
namespace {
__device__ __align__(256) uint8_t g_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a stand-in, so the address is looked up with that device
// current.  It is looked up again on every call made outside a stream capture
// (a device reset reloads the module, and the array may move); while `stream`
// is capturing, the runtime cannot be asked, so the address cached by the last
// call outside a capture on this device is used.
int noalloc_scratch(cudaStream_t stream, void** out) {
  static std::mutex mu;
  static void* addr[256] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 256) return fail(KVQ_ERR_UNSUPPORTED, "device index %d", dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if ((e = cudaStreamIsCapturing(stream, &cap)) != cudaSuccess)
    return cuda_fail(e, "cudaStreamIsCapturing");
  std::lock_guard<std::mutex> lk(mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    addr[dev] = p;
  } else if (!addr[dev]) {
    return fail(KVQ_ERR_INVALID_ARG, "the first kvq_decode_attention_noalloc call on device %d "
                "must come before any stream capture", dev);
  }
  *out = addr[dev];
  return KVQ_OK;
}
}  // namespace

extern "C" {

int kvq_decode_attention_noalloc(const kvq_cache* cache, const void* q, int q_dtype,
                                 int32_t num_seqs, int32_t num_queries, int32_t num_q_heads,
                                 const int32_t* page_table, int32_t max_pages_per_seq,
                                 const int32_t* seq_lens, float softmax_scale, float tau,
                                 float* out, float* bound, uint8_t* flags, kvq_stream_t stream) {
  if (!out && num_seqs > 0) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
  int rc = check_cache(cache);
  if (rc) return rc;
  if (num_seqs == 0) return KVQ_OK;
  const size_t need =
      kvq_workspace_size(cache, num_seqs, num_queries, num_q_heads, max_pages_per_seq);
  if (need == 0)
    return fail(KVQ_ERR_INVALID_ARG, "invalid decode shape (num_queries %d, num_q_heads %d, "
                "max_pages_per_seq %d)", num_queries, num_q_heads, max_pages_per_seq);
  if (need > (size_t)KVQ_NOALLOC_SCRATCH_BYTES)
    return fail(KVQ_ERR_UNSUPPORTED, "this shape needs %zu bytes of split-K scratch; the "
                "static scratch of kvq_decode_attention_noalloc holds %d bytes",
                need, KVQ_NOALLOC_SCRATCH_BYTES);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(s, &scratch))) return rc;
  // the per-(sequence, kv head) counters at the front of the scratch must start
  // at zero whatever an earlier call left there
  const size_t counters = ((size_t)num_seqs * cache->num_kv_heads * sizeof(int) + 255) / 256 * 256;
  cudaError_t e = cudaMemsetAsync(scratch, 0, counters, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(scratch counters)");
  return decode_impl(cache, q, q_dtype, num_seqs, num_queries, num_q_heads, page_table,
                     max_pages_per_seq, seq_lens, softmax_scale, tau, out, bound, flags, scratch,
                     (size_t)KVQ_NOALLOC_SCRATCH_BYTES, s);
}

}  // extern "C"
