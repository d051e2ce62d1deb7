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

constexpr int kFbMaxItems = 64;
struct FbItem {
  int64_t k_off;  // bytes into staging
  int64_t v_off;
  int64_t q_row;  // flattened (sequence, query, q head)
  int n;
  int pad;
};
struct FbArgs {
  const uint8_t* staging;
  const void* q;
  int q_bf16, kv_bf16;
  float s_att;
  float* out;
  int num_items;
  FbItem items[kFbMaxItems];
};

cudaError_t launch_append(const AppendArgs& a, int d, int kbits, int kgroup, cudaStream_t s);
DecodeVariant select_decode_kernel(int d, int kbits, int kgroup);
int decode_threads();
cudaError_t launch_fallback(const FbArgs& a, int d, cudaStream_t stream);

}  // namespace kvq
