// TurboQuant_prod, the inner-product variant of scalar TurboQuant (TurboQuant notes sec. 3.2),
// on the GPU, fp32, any d <= 256:
//
//   encode:  nu = |x|, u = x / nu, y = Pi u, idx_r = nearest level of the scalar Lloyd-Max
//            codebook c1 to y_r (b - 1 bits per coordinate), residual r = u - Pi^T c1[idx],
//            gamma = |r|, q = sign(S r) (QJL, sec. 2.2; sign(0) = +1) with S a d x d matrix of
//            iid N(0, 1) entries (input data);
//   decode:  x_hat = nu (Pi^T c1[idx] + gamma sqrt(pi / 2) / d S^T q).
// Records: the indices as a FibQuant record with k = 1 (index r at bits [r B1, (r + 1) B1)),
// the signs as d bits (bit r of byte r / 8 set when q_r = +1), the norm and gamma as fp16.
//
// Tiles of 64 vectors, 256 threads.  The three products of the encoder (Pi u, Pi^T c1[idx],
// S r) and the decoder's single product ([c1[idx] | coef q] . [Pi ; S], K = 2d) are fp32 FFMA
// tile products with the right-hand matrix streamed through shared memory in chunks of 32 rows;
// every thread owns 4 rows x d/16 columns.
#include <cuda_fp16.h>

#include "fq_device.cuh"
#include "fq_internal.h"

namespace fq {
namespace {

constexpr int kTV = 64;          // vectors per tile
constexpr int kThreadsV = 256;
constexpr int kKC = 32;          // rows of the right-hand matrix per chunk
constexpr float kSqrtHalfPi = 1.2533141373155003f;  // sqrt(pi / 2)

struct ProdArgs {
  int64_t n;
  int d, N1, B1, P1, PS;
  const float* rot;   // [d, d]
  const float* c1;    // [N1]
  const float* qjl;   // [d, d]
};

// acc[i][j] (row 4 rg + i, column cg + 16 j) = sum_k A[row][k] Bm(k, column), k < K; A in shared
// memory with row stride `as`; Bm(k, c) (c < ncols) is read from global memory into `ps`.
template <int RN, class BM>
__device__ __forceinline__ void tile_product(const float* A, int as, int K, int ncols, float* ps,
                                             BM bm, float (&acc)[4][RN]) {
  const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < RN; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kKC) {
    const int kc = (K - k0) < kKC ? (K - k0) : kKC;
    __syncthreads();  // the previous chunk is consumed (and A is complete)
    for (int e = tid; e < kc * 16 * RN; e += kThreadsV) {
      const int kk = e / (16 * RN), c = e - kk * 16 * RN;
      ps[kk * 16 * RN + c] = c < ncols ? bm(k0 + kk, c) : 0.f;
    }
    __syncthreads();
    for (int kk = 0; kk < kc; ++kk) {
      float a[4], b[RN];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = A[(4 * rg + i) * as + k0 + kk];
#pragma unroll
      for (int j = 0; j < RN; ++j) b[j] = ps[kk * 16 * RN + cg + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
}

template <typename TX, int RN>
__global__ void __launch_bounds__(kThreadsV)
    encode_prod_kernel(const TX* __restrict__ x, ProdArgs a, uint8_t* __restrict__ codes,
                       uint8_t* __restrict__ signs, uint16_t* __restrict__ norms,
                       uint16_t* __restrict__ gamma) {
  extern __shared__ float smem[];
  const int d = a.d, st = d + 1;
  float* us = smem;                      // [64][d + 1]: u, then the residual
  float* ys = us + kTV * st;             // [64][d + 1]: Pi u, then c1[idx], then S r
  float* ps = ys + kTV * st;             // [32][16 RN]
  float* nus = ps + kKC * 16 * RN;       // [64]
  float* gms = nus + kTV;                // [64]
  uint16_t* ids = reinterpret_cast<uint16_t*>(gms + kTV);  // [64][d]
  const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
  const int64_t n_tiles = (a.n + kTV - 1) / kTV;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * kTV;
    __syncthreads();
    for (int e = tid; e < kTV * d; e += kThreadsV) {
      const int r = e / d, c = e - r * d;
      us[r * st + c] = row0 + r < a.n ? load_as_float(x + (row0 + r) * d, c) : 0.f;
    }
    __syncthreads();
    if (tid < kTV) {
      float ss = 0.f;
      for (int c = 0; c < d; ++c) ss = fmaf(us[tid * st + c], us[tid * st + c], ss);
      const float nu = sqrtf(ss);
      nus[tid] = nu;
      const float inv = nu > 0.f ? 1.f / nu : 0.f;
      for (int c = 0; c < d; ++c) us[tid * st + c] *= inv;
    }
    float acc[4][RN];
    // y = Pi u: Bm(c, j) = Pi[j][c]
    tile_product<RN>(us, st, d, d, ps,
                     [&](int k, int c) { return __ldg(a.rot + (size_t)c * d + k); }, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < RN; ++j) {
        const int c = cg + 16 * j;
        if (c < d) ys[(4 * rg + i) * st + c] = acc[i][j];
      }
    __syncthreads();
    // nearest level per coordinate (lowest index on ties), then the level's value
    for (int e = tid; e < kTV * d; e += kThreadsV) {
      const int r = e / d, c = e - r * d;
      const float yv = ys[r * st + c];
      float best = INFINITY;
      int bi = 0;
      for (int i = 0; i < a.N1; ++i) {
        const float dist = fabsf(yv - __ldg(a.c1 + i));
        if (dist < best) {
          best = dist;
          bi = i;
        }
      }
      ids[r * d + c] = (uint16_t)bi;
      ys[r * st + c] = __ldg(a.c1 + bi);
    }
    // residual r = u - Pi^T c1[idx]: Bm(j, c) = Pi[j][c]
    tile_product<RN>(ys, st, d, d, ps,
                     [&](int k, int c) { return __ldg(a.rot + (size_t)k * d + c); }, acc);
    __syncthreads();  // every thread is done reading c1[idx] and u before they are overwritten
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < RN; ++j) {
        const int c = cg + 16 * j;
        if (c < d) us[(4 * rg + i) * st + c] -= acc[i][j];
      }
    __syncthreads();
    if (tid < kTV) {
      float g2 = 0.f;
      for (int c = 0; c < d; ++c) g2 = fmaf(us[tid * st + c], us[tid * st + c], g2);
      gms[tid] = sqrtf(g2);
    }
    // QJL: S r, Bm(c, i) = S[i][c]
    tile_product<RN>(us, st, d, d, ps,
                     [&](int k, int c) { return __ldg(a.qjl + (size_t)c * d + k); }, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < RN; ++j) {
        const int c = cg + 16 * j;
        if (c < d) ys[(4 * rg + i) * st + c] = acc[i][j];
      }
    __syncthreads();
    // records: signs (8 per byte), indices (k = 1 record), norm and gamma
    for (int e = tid; e < kTV * a.PS; e += kThreadsV) {
      const int r = e / a.PS, b = e - r * a.PS;
      if (row0 + r >= a.n) continue;
      uint32_t byte = 0;
      for (int t = 0; t < 8; ++t) {
        const int i = 8 * b + t;
        if (i < d) byte |= uint32_t(ys[r * st + i] >= 0.f) << t;
      }
      signs[(row0 + r) * a.PS + b] = (uint8_t)byte;
    }
    for (int e = tid; e < kTV * a.P1; e += kThreadsV) {
      const int r = e / a.P1, b = e - r * a.P1;
      if (row0 + r >= a.n) continue;
      uint32_t byte = 0;
      for (int t = 0; t < 8; ++t) {
        const int i = 8 * b + t;
        const int c = i / a.B1;
        if (c < d) byte |= uint32_t((ids[r * d + c] >> (i - c * a.B1)) & 1) << t;
      }
      codes[(row0 + r) * a.P1 + b] = (uint8_t)byte;
    }
    if (tid < kTV && row0 + tid < a.n) {
      norms[row0 + tid] = f32_to_f16_bits(nus[tid]);
      gamma[row0 + tid] = f32_to_f16_bits(gms[tid]);
    }
  }
}

template <typename TY, int RN>
__global__ void __launch_bounds__(kThreadsV)
    decode_prod_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ signs,
                       const uint16_t* __restrict__ norms, const uint16_t* __restrict__ gamma,
                       ProdArgs a, TY* __restrict__ y) {
  extern __shared__ float smem[];
  const int d = a.d, st = 2 * d + 1;
  float* zs = smem;                      // [64][2d + 1]: [c1[idx] | coef q]
  float* ps = zs + kTV * st;             // [32][16 RN]
  float* nus = ps + kKC * 16 * RN;       // [64]
  const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
  const int64_t n_tiles = (a.n + kTV - 1) / kTV;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * kTV;
    __syncthreads();
    for (int e = tid; e < kTV * 2 * d; e += kThreadsV) {
      const int r = e / (2 * d), c = e - r * 2 * d;
      const int64_t v = row0 + r;
      float val = 0.f;
      if (v < a.n) {
        if (c < d) {
          val = __ldg(a.c1 + record_index(codes + v * a.P1, c, a.B1));
        } else {
          const int i = c - d;
          const float coef = f16_bits_to_f32(gamma[v]) * kSqrtHalfPi / (float)d;
          val = ((signs[v * a.PS + (i >> 3)] >> (i & 7)) & 1) ? coef : -coef;
        }
      }
      zs[r * st + c] = val;
    }
    if (tid < kTV) nus[tid] = row0 + tid < a.n ? f16_bits_to_f32(norms[row0 + tid]) : 0.f;
    float acc[4][RN];
    tile_product<RN>(zs, st, 2 * d, d, ps,
                     [&](int k, int c) {
                       return k < d ? __ldg(a.rot + (size_t)k * d + c)
                                    : __ldg(a.qjl + (size_t)(k - d) * d + c);
                     },
                     acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * rg + i;
      const int64_t v = row0 + r;
      if (v < a.n) {
#pragma unroll
        for (int j = 0; j < RN; ++j) {
          const int c = cg + 16 * j;
          if (c < d) {
            const float val = nus[r] * acc[i][j];
            if constexpr (sizeof(TY) == 2)
              y[v * d + c] = __float2half_rn(val);
            else
              y[v * d + c] = val;
          }
        }
      }
    }
  }
}

int grid_v(int64_t n) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + kTV - 1) / kTV;
  const int64_t cap = (int64_t)sms * 4;
  return (int)(want < cap ? want : cap);
}

int rn_of(int d) { return (d + 15) / 16 <= 4 ? 4 : ((d + 15) / 16 <= 8 ? 8 : 16); }

}  // namespace

cudaError_t launch_encode_prod(const void* x, fq_dtype xt, int64_t n, int d, int N1, int B1,
                               int P1, const float* rot, const float* c1, const float* qjl,
                               uint8_t* codes, uint8_t* signs, uint16_t* norms, uint16_t* gamma,
                               cudaStream_t st) {
  ProdArgs a{n, d, N1, B1, P1, (d + 7) / 8, rot, c1, qjl};
  const int rn = rn_of(d);
  const size_t smem = ((size_t)2 * kTV * (d + 1) + (size_t)kKC * 16 * rn + 2 * kTV) *
                          sizeof(float) + (size_t)kTV * d * sizeof(uint16_t);
  cudaError_t e = cudaSuccess;
#define FQ_PROD_ENC(TX, RN)                                                                    \
  {                                                                                            \
    auto kern = encode_prod_kernel<TX, RN>;                                                    \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);    \
    if (e != cudaSuccess) return e;                                                            \
    kern<<<grid_v(n), kThreadsV, smem, st>>>(static_cast<const TX*>(x), a, codes, signs,       \
                                             norms, gamma);                                    \
    return cudaGetLastError();                                                                 \
  }
  if (xt == FQ_F16) {
    if (rn == 4) FQ_PROD_ENC(__half, 4)
    if (rn == 8) FQ_PROD_ENC(__half, 8)
    FQ_PROD_ENC(__half, 16)
  }
  if (rn == 4) FQ_PROD_ENC(float, 4)
  if (rn == 8) FQ_PROD_ENC(float, 8)
  FQ_PROD_ENC(float, 16)
#undef FQ_PROD_ENC
  return e;
}

cudaError_t launch_decode_prod(const uint8_t* codes, const uint8_t* signs, const uint16_t* norms,
                               const uint16_t* gamma, int64_t n, int d, int N1, int B1, int P1,
                               const float* rot, const float* c1, const float* qjl, void* y,
                               fq_dtype yt, cudaStream_t st) {
  ProdArgs a{n, d, N1, B1, P1, (d + 7) / 8, rot, c1, qjl};
  const int rn = rn_of(d);
  const size_t smem = ((size_t)kTV * (2 * d + 1) + (size_t)kKC * 16 * rn + kTV) * sizeof(float);
  cudaError_t e = cudaSuccess;
#define FQ_PROD_DEC(TY, RN)                                                                    \
  {                                                                                            \
    auto kern = decode_prod_kernel<TY, RN>;                                                    \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);    \
    if (e != cudaSuccess) return e;                                                            \
    kern<<<grid_v(n), kThreadsV, smem, st>>>(codes, signs, norms, gamma, a,                    \
                                             static_cast<TY*>(y));                             \
    return cudaGetLastError();                                                                 \
  }
  if (yt == FQ_F16) {
    if (rn == 4) FQ_PROD_DEC(__half, 4)
    if (rn == 8) FQ_PROD_DEC(__half, 8)
    FQ_PROD_DEC(__half, 16)
  }
  if (rn == 4) FQ_PROD_DEC(float, 4)
  if (rn == 8) FQ_PROD_DEC(float, 8)
  FQ_PROD_DEC(float, 16)
#undef FQ_PROD_DEC
  return e;
}

}  // namespace fq
