// decode_attention.cu -- the decode kernels (decode_kernel.cuh) of every
// supported codec of a cache without outlier extraction, and the selection of
// a codec's variant.  The variants of caches with outlier extraction are
// compiled in decode_attention_med3.cu.
#include "decode_kernel.cuh"

namespace kvq {

DecodeVariant select_decode_kernel(int d, int kbits, int kgroup, int out) {
  if (out) return select_decode_kernel_med3(d, kbits, kgroup);
#define KVQ_DECODE_CASE(D_, KB_, KG_) \
  if (d == D_ && kbits == KB_ && kgroup == KG_) return make_variant<D_, KB_, KG_, false>();
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

int decode_threads() { return kWarps * 32; }

}  // namespace kvq
