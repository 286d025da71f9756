// sm_100a fast paths of fq_encode / fq_decode (declarations; see codec_sm100.cu).
#pragma once

#include "fq_internal.h"

namespace fq {
namespace sm100 {

// True when the fast kernel handles this call (shape, dtype and pointer alignment).
bool encode_supported(fq_dtype xt, const Shape& s, const void* x, const void* codes,
                      const void* norms);
cudaError_t launch_encode(const void* x, fq_dtype xt, int64_t n, const Shape& s,
                          const float* rot, const float* cb, uint8_t* codes, uint16_t* norms,
                          const void* index, cudaStream_t st);

bool decode_supported(fq_dtype yt, const Shape& s, const void* codes, const void* norms,
                      const void* y);
cudaError_t launch_decode(const uint8_t* codes, const uint16_t* norms, int64_t n,
                          const Shape& s, const float* rot, const float* cb, void* y,
                          fq_dtype yt, cudaStream_t st);

}  // namespace sm100
}  // namespace fq
