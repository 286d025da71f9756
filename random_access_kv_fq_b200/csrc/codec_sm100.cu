// sm_100a fast paths of fq_encode / fq_decode.
#include "codec_sm100.h"

namespace fq {
namespace sm100 {

bool encode_supported(fq_dtype, const Shape&, const void*, const void*, const void*) {
  return false;
}
cudaError_t launch_encode(const void*, fq_dtype, int64_t, const Shape&, const float*,
                          const float*, uint8_t*, uint16_t*, const void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
bool decode_supported(fq_dtype, const Shape&, const void*, const void*, const void*) {
  return false;
}
cudaError_t launch_decode(const uint8_t*, const uint16_t*, int64_t, const Shape&, const float*,
                          const float*, void*, fq_dtype, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace sm100
}  // namespace fq
