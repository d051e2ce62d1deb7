// kvq_internal.cuh -- argument blocks and launch entry points shared between
// the host API (kvq_api.cu) and the kernel translation units.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

struct AppendArgs {
  uint8_t* pool;
  float* eta;
  const int8_t* signs;  // NULL unless keys are rotated
  int32_t* err;
  const void* k;
  const void* v;
  int in_bf16;
  int64_t seq_stride, head_stride, tok_stride;
  int num_seqs, num_tokens, hkv, num_pages, max_pages;
  const int32_t* valid;
  const int32_t* start_pos;
  const int32_t* page_table;
  float rot_c;
};

struct DecodeArgs {
  const uint8_t* pool;
  const float* eta;
  const int8_t* signs;
  int32_t* err;
  const void* q;
  int q_bf16;
  const int32_t* page_table;
  int max_pages;
  const int32_t* seq_lens;
  int num_seqs, nq, hq, hkv, G, R, num_pages;
  int pps;  // pages per split
  float s_att, tau, rot_c;
  float* out;  // NULL: bound only
  float* bound;
  uint8_t* flags;
  float* part;
  int* counters;
  // fused append (NULL app_k: none): the new token of sequence s, kv head h at
  // element s * app_seq_stride + h * app_head_stride, written at position
  // seq_lens[s] - 1 before the decode reads the page
  const void* app_k;
  const void* app_v;
  int app_bf16;
  int64_t app_seq_stride, app_head_stride;
};

using DecodeKernel = void (*)(const DecodeArgs);
struct DecodeVariant {
  DecodeKernel kernel;
  DecodeKernel kernel_append;  // the same with the step's append fused in
  int smem;    // dynamic shared memory bytes
  int record;  // floats per split record
};

// Exact fallback work items.  One item = one CTA: up to kFbRows flagged query
// rows of one (sequence, kv head) over the token range [t0, t1) of its staged
// originals.  A (sequence, kv head) longer than kFbMinChunk tokens is cut into
// up to kFbMaxChunks ranges (consecutive items, chunk 0..nchunk-1) whose
// partial softmax states go to the scratch and are merged by a second kernel.
constexpr int kFbRows = 8;
constexpr int kFbMaxItems = 48;     // items per launch (the argument block stays < 4 KB)
constexpr int kFbMaxChunks = 8;
constexpr int kFbMinChunk = 128;    // tokens
struct FbItem {
  int64_t k_off;             // bytes into staging: K [n][D], then V at v_off
  int64_t v_off;
  int64_t row0;              // flattened (sequence, query, q head) index of row offset 0
  int32_t t0, t1;            // token range of this item
  int32_t roff[kFbRows];     // row = row0 + roff[r], r < nrows
  int16_t nrows, chunk, nchunk, pad;
};
struct FbArgs {
  const uint8_t* staging;
  const void* q;
  float* out;
  float* scratch;            // [kFbMaxItems][kFbRows][D + 2]: o (unnormalised), m, l
  int q_bf16, kv_bf16;
  float s_att;
  int num_items;
  int any_split;             // some item has nchunk > 1: the merge kernel runs
  int pad;
  FbItem items[kFbMaxItems];
};
// bytes of the merge scratch at the start of the staging buffer
inline size_t fallback_scratch_bytes(int d) {
  return ((size_t)kFbMaxItems * kFbRows * (d + 2) * sizeof(float) + 255) / 256 * 256;
}

// Launch with programmatic stream serialization (the kernel calls pdl_wait
// before any access that depends on earlier work in the stream): its launch
// and its first prefetches overlap the end of the grid before it.
template <typename Arg>
cudaError_t launch_pdl(void (*kernel)(Arg), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       const Arg& arg) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, arg);
}

// ---- adaptive precision (adaptive.cu) ------------------------------------------
// One flagged (sequence, kv head) with its flagged query rows (at most 4).
struct AdUnit {
  int32_t seq, kvh, nrows, rslot;   // rslot: this unit's first row slot
  int32_t rows[4];                  // flattened (sequence, query, q head) row indices
  int64_t stage_off;                // bytes into staging: its promoted pages' K, then V
  int32_t nstaged, pad;             // pages staged
};
// One correction item: pages [p0, p1) of unit `unit`.
struct AdItem {
  int32_t unit, p0, p1, chunk, nchunk, first;   // first: the unit's first item
};
struct AdArgs {
  const uint8_t* pool;
  const float* eta;
  const int8_t* signs;
  int32_t* err;
  const void* q;
  int q_bf16, kv_bf16;
  const int32_t* page_table;
  int max_pages;
  const int32_t* seq_lens;
  int nq, hq, hkv, G, num_pages;
  int outliers;                // the cache's blocks end in the outlier section
  float s_att, rot_c, tau, tau_cov, v_tol, rank_tol;
  const AdUnit* units;
  int num_units;
  const AdItem* items;
  int num_items;
  // per row slot, [slots][max_pages]: key / value promotion, the key-promoted
  // pages in selection order, exact block log-masses; per slot counts
  uint8_t* kp;
  uint8_t* vp;
  int32_t* korder;
  float* blse;
  int32_t* nkey;
  int32_t* nval;
  uint8_t* um;                 // [units][max_pages]: kp | vp over the unit's rows
  const int32_t* smap;         // [units][max_pages]: staged index of a page, or -1
  const uint8_t* staging;
  float* part;                 // [items][4 rows][D + 8] and [items][2 NB + 1]
  float* out;
  float* bound;
  uint8_t* flags;
  uint8_t* rank_fail;          // per row slot
};
// bytes of the per-item partial records
__host__ __device__ inline size_t adaptive_part_floats(int d) { return 4 * (size_t)(d + 8) + 2 * (d / 32) + 4; }
cudaError_t launch_adaptive_select(const AdArgs& a, int d, int kbits, int kgroup, int smem,
                                   cudaStream_t s);
cudaError_t launch_adaptive_correct(const AdArgs& a, int d, int kbits, int kgroup, cudaStream_t s);
cudaError_t launch_adaptive_finish(const AdArgs& a, int d, cudaStream_t s);
int adaptive_select_smem(int max_pages, int d);

// ---- the KQV codec (kqv.cu) -------------------------------------------------
// Byte layout of one (page, kv head) block: K codes (nibbles), V codes
// (3-bit in nibbles), V sketch bits, then per token |k'|, eps, |v'|, |r|
// (fp32), then the block's v^ max / min per 32-channel group.
struct KqvLayout {
  int d;
  __host__ __device__ int vc() const { return kPage * d / 2; }
  __host__ __device__ int vs() const { return kPage * d; }
  __host__ __device__ int kn() const { return kPage * d + kPage * d / 8; }
  __host__ __device__ int ke() const { return kn() + 4 * kPage; }
  __host__ __device__ int vn() const { return kn() + 8 * kPage; }
  __host__ __device__ int vr() const { return kn() + 12 * kPage; }
  __host__ __device__ int rg() const { return kn() + 16 * kPage; }
  __host__ __device__ int bytes() const { return rg() + (d / 32) * 8; }
};
// fp32 codebooks: 4-bit keys, 3-bit values
struct KqvTables {
  float kcent[16], kthr[15], vcent[8], vthr[7];
};
struct KqvAppendArgs {
  AppendArgs a;
  const float* qjl;   // S [d][d]
  float qjl_c;        // fp32(sqrt(pi/2) / d)
  KqvTables t;
};
struct KqvDecodeArgs {
  DecodeArgs a;       // out, bound, flags, part as for the Tier-1 decode; no fused append
  const float* qjl;
  float qjl_c;
  int nsp;            // splits of the partial grid (records per unit)
  KqvTables t;
};
int kqv_tables(int d, KqvTables* t);   // host; cached per head_dim
cudaError_t launch_kqv_append(const KqvAppendArgs& a, int d, cudaStream_t s);
// the partial kernel over (unit, split), then the merge per unit
cudaError_t launch_kqv_decode(const KqvDecodeArgs& a, int d, int units, int splits,
                              cudaStream_t s);
const void* kqv_partial_kernel(int d);
int kqv_partial_smem(int d);
int kqv_record_floats(int d);
int kqv_threads();

// ---- the HQMQ codec (hqmq.cu) ------------------------------------------------
// Byte layout of one (page, kv head) block, chunk-major (token t of chunk c at
// [c][t]): K codes u16, V codes u16, K radii e4m3, V radii e4m3, then per
// token |k| and eps (fp32), then the block's v^ max / min per 32-channel group,
// then (out) the Med3x section of the Tier-1 layout.
struct HqLayout {
  int d;
  int out = 0;
  __host__ __device__ int nc() const { return d / 4; }
  __host__ __device__ int vi() const { return kPage * nc() * 2; }
  __host__ __device__ int kr() const { return kPage * nc() * 4; }
  __host__ __device__ int vr() const { return kr() + kPage * nc(); }
  __host__ __device__ int kn() const { return vr() + kPage * nc(); }
  __host__ __device__ int ke() const { return kn() + 4 * kPage; }
  __host__ __device__ int rg() const { return kn() + 8 * kPage; }
  __host__ __device__ int out_off() const { return rg() + (d / 32) * 8; }
  __host__ __device__ int bytes() const { return out_off() + (out ? kOutBytes : 0); }
};
struct HqAppendArgs {
  AppendArgs a;
  const float* sec;   // [hkv][2][S][4] unit quaternions
  int S;
  int outliers;       // Med3x extraction (0 or 1)
};
struct HqDecodeArgs {
  DecodeArgs a;       // out, bound, flags, part as for the Tier-1 decode; no fused append
  const float* sec;
  int S;
  int nsp;            // splits of the partial grid (records per unit)
  int outliers;
};
cudaError_t launch_hqmq_append(const HqAppendArgs& a, int d, cudaStream_t s);
// the partial kernel over (unit, split), then the merge per unit
cudaError_t launch_hqmq_decode(const HqDecodeArgs& a, int d, int units, int splits,
                               cudaStream_t s);
const void* hqmq_partial_kernel(int d, int out);
int hqmq_partial_smem(int d, int S, int out);
int hqmq_record_floats(int d);
int hqmq_threads();

cudaError_t launch_append(const AppendArgs& a, int d, int kbits, int kgroup, int out,
                          cudaStream_t s);
// out: the cache's outlier extraction (0 or 1)
DecodeVariant select_decode_kernel(int d, int kbits, int kgroup, int out);
DecodeVariant select_decode_kernel_med3(int d, int kbits, int kgroup);
int decode_threads();
// the recompute (and, when an item was split, the merge) on `stream`
cudaError_t launch_fallback(const FbArgs& a, int d, cudaStream_t stream);

}  // namespace kvq
