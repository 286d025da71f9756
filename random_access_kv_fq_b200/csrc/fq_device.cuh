// Small device helpers shared by the kernels of libfq.
#pragma once

#include <cstdint>

#include <cuda_fp16.h>

namespace fq {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Warp-wide argmin of (dist, idx): smallest distance, lowest index among equal distances.
__device__ __forceinline__ void warp_argmin(float& dist, int& idx) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float od = __shfl_xor_sync(0xffffffffu, dist, o);
    int oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (od < dist || (od == dist && oi < idx)) {
      dist = od;
      idx = oi;
    }
  }
}

__device__ __forceinline__ float load_as_float(const __half* p, int64_t i) {
  return __half2float(p[i]);
}
__device__ __forceinline__ float load_as_float(const float* p, int64_t i) { return p[i]; }

__device__ __forceinline__ uint16_t f32_to_f16_bits(float v) {
  return __half_as_ushort(__float2half_rn(v));
}
__device__ __forceinline__ float f16_bits_to_f32(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// Reads index j (B bits, LSB-first at record bit j*B) of a record that starts at `rec`.
// Reads only bytes that belong to the record (at most 3 for B <= 16).
__device__ __forceinline__ int record_index(const uint8_t* rec, int j, int B) {
  int bit = j * B;
  int byte = bit >> 3;
  int sh = bit & 7;
  int need = (sh + B + 7) >> 3;  // bytes spanned
  uint32_t w = rec[byte];
  if (need > 1) w |= uint32_t(rec[byte + 1]) << 8;
  if (need > 2) w |= uint32_t(rec[byte + 2]) << 16;
  return int((w >> sh) & ((1u << B) - 1u));
}

}  // namespace fq
