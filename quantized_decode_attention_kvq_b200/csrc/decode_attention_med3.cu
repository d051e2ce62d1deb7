// decode_attention_med3.cu -- the decode kernels (decode_kernel.cuh) of every
// supported codec of a cache with outlier extraction (the median-multiplier
// rule of "Hurwitz Quaternion Multiplicative Quantization for KV Cache
// Compression", Method 3).  A translation unit of their own, so they compile
// in parallel with the variants without extraction.
#include "decode_kernel.cuh"

namespace kvq {

DecodeVariant select_decode_kernel_med3(int d, int kbits, int kgroup) {
#define KVQ_DECODE_CASE(D_, KB_, KG_) \
  if (d == D_ && kbits == KB_ && kgroup == KG_) return make_variant<D_, KB_, KG_, true>();
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
  return DecodeVariant{nullptr, nullptr, 0, 0};
}

}  // namespace kvq
