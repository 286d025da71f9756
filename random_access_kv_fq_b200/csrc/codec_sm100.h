// sm_100a fast paths of fq_encode / fq_decode (encode_sm100.cu, encode_large_sm100.cu,
// decode_sm100.cu, decode_large_sm100.cu).
#pragma once

#include "fq_internal.h"

namespace fq {
namespace sm100 {

// True when the fast kernel handles this call (shape, dtype and pointer alignment).
bool encode_supported(fq_dtype xt, const Shape& s, const void* x, const void* codes,
                      const void* norms);
// rho != nullptr: also <z, zhat> per vector in fp16 (the rescale variant's stored rho).
cudaError_t launch_encode(const void* x, fq_dtype xt, int64_t n, const Shape& s,
                          const float* rot, const float* cb, uint8_t* codes, uint16_t* norms,
                          const void* index, cudaStream_t st, uint16_t* rho = nullptr);

// Large codebooks (d = 128, k = 4, N = 512 .. 4096, no index): tensor-core brute force.
bool encode_large_supported(fq_dtype xt, const Shape& s, const void* x, const void* codes,
                            const float* cb, const void* index);
cudaError_t launch_encode_large(const void* x, int64_t n, const Shape& s, const float* rot,
                                const float* cb, uint8_t* codes, uint16_t* norms,
                                cudaStream_t st);
// d = 128, k = 4, N = 4096 with a grid index (top-c or exact without overflow lists): tensor-core
// rotation and a candidate search; an index that does not describe the codebook falls back to
// exact brute force inside the kernel.
bool encode_grid_supported(fq_dtype xt, const Shape& s, const void* x, const void* codes,
                           const float* cb, const void* index);
cudaError_t launch_encode_grid(const void* x, int64_t n, const float* rot, const float* cb,
                               const void* index, uint8_t* codes, uint16_t* norms,
                               cudaStream_t st);

// Half- and full-vector codes (d = 64 with k = 32 or 64, d = 128 with k = 64) with an
// FQ_INDEX_TENSOR index: tensor-core GEMM search with exact re-scoring (encode_highk_sm100.cu).
bool highk_supported(fq_dtype xt, const Shape& s, const void* x, const void* index,
                     const float* rot, const float* cb);
cudaError_t launch_encode_highk(const void* x, int64_t n, const Shape& s, const float* rot,
                                const float* cb, const void* index, uint8_t* codes,
                                uint16_t* norms, cudaStream_t st);

// d = 128, k = 4, N <= 4096: tensor-core inverse rotation (decode_large_sm100.cu).
bool decode_large_supported(fq_dtype yt, const Shape& s, const void* codes, const void* norms,
                            const void* y, const float* cb);
cudaError_t launch_decode_large(const uint8_t* codes, const uint16_t* norms, int64_t n,
                                const Shape& s, const float* rot, const float* cb, void* y,
                                fq_dtype yt, cudaStream_t st,
                                Gather gather = Gather{nullptr, 0});

bool decode_supported(fq_dtype yt, const Shape& s, const void* codes, const void* norms,
                      const void* y);
// rho != nullptr: the rescale variant, y = S nu (Pi^T zbar) with S of `rule` (FQ_RESCALE_*).
cudaError_t launch_decode(const uint8_t* codes, const uint16_t* norms, int64_t n,
                          const Shape& s, const float* rot, const float* cb, void* y,
                          fq_dtype yt, cudaStream_t st, const uint16_t* rho = nullptr,
                          int rule = 0);

}  // namespace sm100
}  // namespace fq
