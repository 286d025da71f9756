// TurboQuant_prod, the inner-product variant of scalar TurboQuant (TurboQuant notes sec. 3.2),
// on the GPU: one warp per vector, fp32, any d <= 256.
//
//   encode:  nu = |x|, u = x / nu, y = Pi u, idx_r = nearest level of the scalar Lloyd-Max
//            codebook c1 to y_r (b - 1 bits per coordinate), residual r = u - Pi^T c1[idx],
//            gamma = |r|, q = sign(S r) (QJL, sec. 2.2; sign(0) = +1) with S a d x d matrix of
//            iid N(0, 1) entries (input data);
//   decode:  x_hat = nu (Pi^T c1[idx] + gamma sqrt(pi / 2) / d S^T q).
// Records: the indices as a FibQuant record with k = 1 (index r at bits [r B1, (r + 1) B1)),
// the signs as d bits (bit r of byte r / 8 set when q_r = +1), the norm and gamma as fp16.
#include <cuda_fp16.h>

#include "fq_device.cuh"
#include "fq_internal.h"

namespace fq {
namespace {

constexpr int kWarpsV = 8;
constexpr float kSqrtHalfPi = 1.2533141373155003f;  // sqrt(pi / 2)

struct ProdArgs {
  int64_t n;
  int d, N1, B1, P1, PS;
  const float* rot;   // [d, d]
  const float* c1;    // [N1]
  const float* qjl;   // [d, d]
};

template <typename TX>
__global__ void __launch_bounds__(kWarpsV * 32)
    encode_prod_kernel(const TX* __restrict__ x, ProdArgs a, uint8_t* __restrict__ codes,
                       uint8_t* __restrict__ signs, uint16_t* __restrict__ norms,
                       uint16_t* __restrict__ gamma) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d;
  float* yv = smem + warp * 3 * d;   // Pi u, then c1[idx] (in place)
  float* res = yv + d;               // residual u - Pi^T c1[idx]
  int* ids = reinterpret_cast<int*>(res + d);
  for (int64_t v = (int64_t)blockIdx.x * kWarpsV + warp; v < a.n;
       v += (int64_t)gridDim.x * kWarpsV) {
    float xv[kMaxD / 32];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxD / 32; ++i) {
      const int c = lane + 32 * i;
      xv[i] = c < d ? load_as_float(x + v * d, c) : 0.f;
      ss = fmaf(xv[i], xv[i], ss);
    }
    const float nu = sqrtf(warp_sum(ss));
    const float inv = nu > 0.f ? 1.f / nu : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxD / 32; ++i) xv[i] *= inv;
    // y = Pi u
    for (int r = 0; r < d; ++r) {
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxD / 32; ++i) {
        const int c = lane + 32 * i;
        if (c < d) p = fmaf(__ldg(a.rot + (size_t)r * d + c), xv[i], p);
      }
      p = warp_sum(p);
      if (lane == 0) yv[r] = p;
    }
    __syncwarp();
    // nearest level per coordinate (lowest index on ties), then the level's value
    for (int r = lane; r < d; r += 32) {
      float best = INFINITY;
      int bi = 0;
      for (int i = 0; i < a.N1; ++i) {
        const float dist = fabsf(yv[r] - __ldg(a.c1 + i));
        if (dist < best) {
          best = dist;
          bi = i;
        }
      }
      ids[r] = bi;
      yv[r] = __ldg(a.c1 + bi);
    }
    __syncwarp();
    // residual r = u - Pi^T c1[idx] (this lane's columns) and gamma = |r|
    float g2 = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxD / 32; ++i) {
      const int c = lane + 32 * i;
      if (c < d) {
        float back = 0.f;
        for (int r = 0; r < d; ++r) back = fmaf(__ldg(a.rot + (size_t)r * d + c), yv[r], back);
        const float rr = xv[i] - back;
        res[c] = rr;
        g2 = fmaf(rr, rr, g2);
      }
    }
    const float gam = sqrtf(warp_sum(g2));
    __syncwarp();
    // QJL signs of S r, packed 8 per byte
    for (int b = lane; b < a.PS; b += 32) {
      uint32_t byte = 0;
      for (int t = 0; t < 8; ++t) {
        const int i = 8 * b + t;
        if (i < d) {
          float sr = 0.f;
          for (int c = 0; c < d; ++c) sr = fmaf(__ldg(a.qjl + (size_t)i * d + c), res[c], sr);
          byte |= uint32_t(sr >= 0.f) << t;
        }
      }
      signs[v * a.PS + b] = (uint8_t)byte;
    }
    // indices as a k = 1 record
    for (int b = lane; b < a.P1; b += 32) {
      uint32_t byte = 0;
      for (int t = 0; t < 8; ++t) {
        const int i = 8 * b + t;
        const int r = i / a.B1;
        if (r < d) byte |= uint32_t((ids[r] >> (i - r * a.B1)) & 1) << t;
      }
      codes[v * a.P1 + b] = (uint8_t)byte;
    }
    if (lane == 0) {
      norms[v] = f32_to_f16_bits(nu);
      gamma[v] = f32_to_f16_bits(gam);
    }
    __syncwarp();
  }
}

template <typename TY>
__global__ void __launch_bounds__(kWarpsV * 32)
    decode_prod_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ signs,
                       const uint16_t* __restrict__ norms, const uint16_t* __restrict__ gamma,
                       ProdArgs a, TY* __restrict__ y) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d;
  float* lv = smem + warp * 2 * d;   // c1[idx]
  float* qv = lv + d;                // +-1
  for (int64_t v = (int64_t)blockIdx.x * kWarpsV + warp; v < a.n;
       v += (int64_t)gridDim.x * kWarpsV) {
    for (int r = lane; r < d; r += 32) {
      lv[r] = __ldg(a.c1 + record_index(codes + v * a.P1, r, a.B1));
      qv[r] = ((signs[v * a.PS + (r >> 3)] >> (r & 7)) & 1) ? 1.f : -1.f;
    }
    __syncwarp();
    const float nu = f16_bits_to_f32(norms[v]);
    const float coef = f16_bits_to_f32(gamma[v]) * kSqrtHalfPi / (float)d;
#pragma unroll
    for (int i = 0; i < kMaxD / 32; ++i) {
      const int c = lane + 32 * i;
      if (c < d) {
        float mse = 0.f, qj = 0.f;
        for (int r = 0; r < d; ++r) {
          mse = fmaf(__ldg(a.rot + (size_t)r * d + c), lv[r], mse);
          qj = fmaf(__ldg(a.qjl + (size_t)r * d + c), qv[r], qj);
        }
        const float val = nu * fmaf(coef, qj, mse);
        if constexpr (sizeof(TY) == 2)
          y[v * d + c] = __float2half_rn(val);
        else
          y[v * d + c] = val;
      }
    }
    __syncwarp();
  }
}

int grid_v(int64_t n) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + kWarpsV - 1) / kWarpsV;
  const int64_t cap = (int64_t)sms * 16;
  return (int)(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_encode_prod(const void* x, fq_dtype xt, int64_t n, int d, int N1, int B1,
                               int P1, const float* rot, const float* c1, const float* qjl,
                               uint8_t* codes, uint8_t* signs, uint16_t* norms, uint16_t* gamma,
                               cudaStream_t st) {
  ProdArgs a{n, d, N1, B1, P1, (d + 7) / 8, rot, c1, qjl};
  const size_t smem = (size_t)kWarpsV * 3 * d * sizeof(float);
  if (xt == FQ_F16)
    encode_prod_kernel<__half><<<grid_v(n), kWarpsV * 32, smem, st>>>(
        static_cast<const __half*>(x), a, codes, signs, norms, gamma);
  else
    encode_prod_kernel<float><<<grid_v(n), kWarpsV * 32, smem, st>>>(
        static_cast<const float*>(x), a, codes, signs, norms, gamma);
  return cudaGetLastError();
}

cudaError_t launch_decode_prod(const uint8_t* codes, const uint8_t* signs, const uint16_t* norms,
                               const uint16_t* gamma, int64_t n, int d, int N1, int B1, int P1,
                               const float* rot, const float* c1, const float* qjl, void* y,
                               fq_dtype yt, cudaStream_t st) {
  ProdArgs a{n, d, N1, B1, P1, (d + 7) / 8, rot, c1, qjl};
  const size_t smem = (size_t)kWarpsV * 2 * d * sizeof(float);
  if (yt == FQ_F16)
    decode_prod_kernel<__half><<<grid_v(n), kWarpsV * 32, smem, st>>>(
        codes, signs, norms, gamma, a, static_cast<__half*>(y));
  else
    decode_prod_kernel<float><<<grid_v(n), kWarpsV * 32, smem, st>>>(
        codes, signs, norms, gamma, a, static_cast<float*>(y));
  return cudaGetLastError();
}

}  // namespace fq
