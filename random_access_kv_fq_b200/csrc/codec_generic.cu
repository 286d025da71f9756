// Generic FibQuant encode / decode: one warp per vector, any supported (d, k, N), fp16 or
// fp32 input.  This is the reference-grade CUDA path: every step of the encoder and decoder
// of the FibQuant summary (sec. 2.3) runs here in fp32 with straightforward data movement.
// The sm_100a fast paths (tensor-core rotation, pruned search, staged records) live in
// encode_sm100.cu, encode_large_sm100.cu, decode_sm100.cu and decode_large_sm100.cu and handle
// the common shapes; this file covers every other shape.
#include <cuda_fp16.h>

#include "fq_device.cuh"
#include "fq_internal.h"

namespace fq {
namespace {

constexpr int kWarps = 8;

// Nearest codeword of block zb (k coordinates) among all N codewords, lanes striding over
// codewords; direct-form squared distance; lowest index on ties.
__device__ __forceinline__ int brute_nearest(const float* zb, int k, const float* __restrict__ cb,
                                             int N, int lane) {
  float best = INFINITY;
  int bi = 0x7fffffff;
  for (int c = lane; c < N; c += 32) {
    float dist = 0.f;
    for (int r = 0; r < k; ++r) {
      float t = zb[r] - __ldg(cb + (size_t)c * k + r);
      dist = fmaf(t, t, dist);
    }
    if (dist < best) {  // c increases, so strict < keeps the lowest index per lane
      best = dist;
      bi = c;
    }
  }
  warp_argmin(best, bi);
  return bi;
}

// Candidate-list search through a grid index (see IndexHeader).  Returns -1 when the index
// does not describe this (k, N, d') so that the caller uses brute force.
__device__ __forceinline__ int index_nearest(const float* zb, int k, const float* __restrict__ cb,
                                             const uint8_t* __restrict__ index, int lane) {
  const IndexHeader* h = reinterpret_cast<const IndexHeader*>(index);
  int flat = 0, stride = 1;
  for (int a = 0; a < k; ++a) {
    float t = (zb[a] - h->lo) * h->inv_h;
    int c = (int)floorf(t);
    c = c < 0 ? 0 : (c >= h->L ? h->L - 1 : c);
    flat += c * stride;
    stride *= h->L;
  }
  const uint8_t* entry = index + h->cells_offset + (size_t)flat * h->entry_bytes;
  uint32_t ov = kNoOverflow;
  if (index_has_overflow(*h))
    ov = *reinterpret_cast<const uint32_t*>(entry + h->entry_bytes - 4);
  const uint16_t* ovl = reinterpret_cast<const uint16_t*>(index + h->overflow_offset);
  int n_extra = (ov == kNoOverflow) ? 0 : ovl[ov];
  int total = h->slots + n_extra;
  float best = INFINITY;
  int bi = 0x7fffffff;
  for (int i = lane; i < total; i += 32) {
    int c = (i < h->slots) ? index_entry_id(entry, i, h->id_bytes) : ovl[ov + 1 + (i - h->slots)];
    float dist = 0.f;
    for (int r = 0; r < k; ++r) {
      float t = zb[r] - __ldg(cb + (size_t)c * k + r);
      dist = fmaf(t, t, dist);
    }
    if (dist < best || (dist == best && c < bi)) {
      best = dist;
      bi = c;
    }
  }
  warp_argmin(best, bi);
  return bi;
}

__device__ __forceinline__ bool index_matches(const uint8_t* index, int k, int N, int dp) {
  if (index == nullptr) return false;
  const IndexHeader* h = reinterpret_cast<const IndexHeader*>(index);
  return h->magic == kIndexMagic && h->version == kIndexVersion && h->k == k && h->N == N &&
         h->dp == dp;
}

// Record slot of input row v: v itself, or (append mode) slot lengths[b] of sequence b's
// [T]-record plane for row v = b * hkv + g; -1 when that slot is outside the plane (the row is
// then not written).
__device__ __forceinline__ int64_t dest_row(const AppendMap& map, int64_t v) {
  if (map.lengths == nullptr) return v;
  const int64_t b = v / map.hkv;
  const int64_t len = map.lengths[b];
  if (len < 0 || len >= map.T) return -1;
  return v * map.T + len;
}

template <typename TX>
__global__ void __launch_bounds__(kWarps * 32)
    encode_generic_kernel(const TX* __restrict__ x, int64_t n, Shape s,
                          const float* __restrict__ rot, const float* __restrict__ cb,
                          uint8_t* __restrict__ codes, uint16_t* __restrict__ norms,
                          const uint8_t* __restrict__ index, AppendMap map,
                          uint16_t* __restrict__ rho_out) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* zs = smem + warp * (s.dp + s.m);
  int* ids = reinterpret_cast<int*>(zs + s.dp);
  const bool use_index = index_matches(index, s.k, s.N, s.dp);
  for (int64_t v = (int64_t)blockIdx.x * kWarps + warp; v < n; v += (int64_t)gridDim.x * kWarps) {
    const TX* xr = x + v * s.d;
    // a1: norm, fp32, eight partial sums per lane then a butterfly (bounded rounding error)
    float xv[kMaxD / 32];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxD / 32; ++i) {
      int c = lane + 32 * i;
      xv[i] = (c < s.d) ? load_as_float(xr, c) : 0.f;
      ss = fmaf(xv[i], xv[i], ss);
    }
    ss = warp_sum(ss);
    const float nu = sqrtf(ss);
    const float inv = nu > 0.f ? 1.f / nu : 0.f;
    // a2: z = Pi pad(x) / nu (only the first d columns of Pi meet nonzero inputs)
    for (int r = 0; r < s.dp; ++r) {
      const float* pr = rot + (size_t)r * s.dp;
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxD / 32; ++i) {
        int c = lane + 32 * i;
        if (c < s.d) p = fmaf(__ldg(pr + c), xv[i], p);
      }
      p = warp_sum(p);
      if (lane == 0) zs[r] = p * inv;
    }
    __syncwarp();
    // a3 + a4: blocks of k coordinates, nearest codeword
    for (int j = 0; j < s.m; ++j) {
      const float* zb = zs + j * s.k;
      int bi = -1;
      if (use_index) bi = index_nearest(zb, s.k, cb, index, lane);
      if (bi < 0) bi = brute_nearest(zb, s.k, cb, s.N, lane);
      if (lane == 0) ids[j] = (nu > 0.f) ? bi : 0;
    }
    __syncwarp();
    // a5: pack, one byte per lane step; bit i of the record is bit (i % B) of index i / B
    // Block Sphere VQ key design 3: rho = <z, zbar>, the alignment of the unit rotated vector
    // with its reconstruction (stored as fp16 like the norm; 1 for a zero vector)
    if (rho_out != nullptr) {
      float part = 0.f;
      for (int e = lane; e < s.dp; e += 32) {
        const int j = e / s.k;
        part = fmaf(zs[e], __ldg(cb + (size_t)ids[j] * s.k + (e - j * s.k)), part);
      }
      part = warp_sum(part);
      if (lane == 0) rho_out[v] = f32_to_f16_bits(nu > 0.f ? part : 1.f);
    }
    const int64_t dst = dest_row(map, v);
    if (dst < 0) {
      __syncwarp();
      continue;
    }
    uint8_t* rec = codes + dst * s.P;
    for (int b = lane; b < s.P; b += 32) {
      uint32_t byte = 0;
      for (int t = 0; t < 8; ++t) {
        int i = 8 * b + t;
        int j = i / s.B;
        if (j < s.m) byte |= uint32_t((ids[j] >> (i - j * s.B)) & 1) << t;
      }
      rec[b] = (uint8_t)byte;
    }
    if (lane == 0) norms[dst] = f32_to_f16_bits(nu);
    __syncwarp();
  }
}

template <typename TY>
__device__ __forceinline__ void store_out(TY* p, int64_t i, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, int64_t i, float v) {
  p[i] = v;
}
template <>
__device__ __forceinline__ void store_out<__half>(__half* p, int64_t i, float v) {
  p[i] = __float2half_rn(v);
}

template <typename TY>
__global__ void __launch_bounds__(kWarps * 32)
    decode_generic_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ norms,
                          int64_t n, Shape s, const float* __restrict__ rot,
                          const float* __restrict__ cb, TY* __restrict__ y, Gather gather,
                          Rescale rs) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* zs = smem + warp * s.dp;
  for (int64_t v = (int64_t)blockIdx.x * kWarps + warp; v < n; v += (int64_t)gridDim.x * kWarps) {
    // gather mode: output row v decodes record ids[v]; an id outside the plane gives NaN
    const int64_t src = gather.ids ? gather.ids[v] : v;
    if (src < 0 || (gather.ids && src >= gather.n_records)) {
#pragma unroll
      for (int i = 0; i < kMaxD / 32; ++i) {
        int c = lane + 32 * i;
        if (c < s.d) store_out(y, v * s.d + c, __int_as_float(0x7fc00000));
      }
      continue;
    }
    const uint8_t* rec = codes + src * s.P;
    // a6 + a7: unpack each index and gather its codeword into the concatenated zhat
    for (int j = lane; j < s.m; j += 32) {
      int c = record_index(rec, j, s.B);
      for (int r = 0; r < s.k; ++r) zs[j * s.k + r] = __ldg(cb + (size_t)c * s.k + r);
    }
    __syncwarp();
    // a8: y = nu (Pi^T zhat)[0:d], times S of Block Sphere VQ key design 3 when rescaling
    float nu = f16_bits_to_f32(norms[src]);
    if (rs.rho != nullptr) {
      const float rho = f16_bits_to_f32(rs.rho[src]);
      float zz = 0.f;
      for (int e = lane; e < s.dp; e += 32) zz = fmaf(zs[e], zs[e], zz);
      zz = warp_sum(zz);
      const float S = rs.rule == FQ_RESCALE_MSE ? rho / zz
                      : rs.rule == FQ_RESCALE_UNBIASED ? 1.f / rho : 1.f;
      nu *= S;
    }
    float acc[kMaxD / 32];
#pragma unroll
    for (int i = 0; i < kMaxD / 32; ++i) acc[i] = 0.f;
    for (int r = 0; r < s.dp; ++r) {
      const float zr = zs[r];
      const float* pr = rot + (size_t)r * s.dp;
#pragma unroll
      for (int i = 0; i < kMaxD / 32; ++i) {
        int c = lane + 32 * i;
        if (c < s.d) acc[i] = fmaf(__ldg(pr + c), zr, acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < kMaxD / 32; ++i) {
      int c = lane + 32 * i;
      if (c < s.d) store_out(y, v * s.d + c, nu * acc[i]);
    }
    __syncwarp();
  }
}

int generic_grid(int64_t n) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (n + kWarps - 1) / kWarps;
  int64_t cap = (int64_t)sms * 16;
  return (int)(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_encode_generic(const void* x, fq_dtype xt, int64_t n, const Shape& s,
                                  const float* rot, const float* cb, uint8_t* codes,
                                  uint16_t* norms, const void* index, cudaStream_t st,
                                  AppendMap map, uint16_t* rho) {
  size_t smem = (size_t)kWarps * (s.dp + s.m) * sizeof(float);
  int grid = generic_grid(n);
  const uint8_t* ix = static_cast<const uint8_t*>(index);
  if (xt == FQ_F16)
    encode_generic_kernel<__half><<<grid, kWarps * 32, smem, st>>>(
        static_cast<const __half*>(x), n, s, rot, cb, codes, norms, ix, map, rho);
  else
    encode_generic_kernel<float><<<grid, kWarps * 32, smem, st>>>(
        static_cast<const float*>(x), n, s, rot, cb, codes, norms, ix, map, rho);
  return cudaGetLastError();
}

cudaError_t launch_decode_generic(const uint8_t* codes, const uint16_t* norms, int64_t n,
                                  const Shape& s, const float* rot, const float* cb, void* y,
                                  fq_dtype yt, cudaStream_t st, Gather gather, Rescale rs) {
  size_t smem = (size_t)kWarps * s.dp * sizeof(float);
  int grid = generic_grid(n);
  if (yt == FQ_F16)
    decode_generic_kernel<__half><<<grid, kWarps * 32, smem, st>>>(codes, norms, n, s, rot, cb,
                                                                   static_cast<__half*>(y), gather, rs);
  else
    decode_generic_kernel<float><<<grid, kWarps * 32, smem, st>>>(codes, norms, n, s, rot, cb,
                                                                  static_cast<float*>(y), gather,
                                                                  rs);
  return cudaGetLastError();
}

}  // namespace fq
