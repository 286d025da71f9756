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

// Tiled decode for any shape: 64 vectors per tile, 256 threads.  The gathered codewords of the
// tile (zhat, fp32) sit in shared memory; the inverse rotation is an fp32 FFMA product of the
// [64 x d'] zhat tile with [d' x d] of Pi, streamed through shared memory in chunks of 32 rows;
// every thread owns 4 rows x d/16 columns of the output.
constexpr int kTileR = 64;
constexpr int kDecThreads = 256;
constexpr int kKChunk = 32;

template <typename TY, int RN>
__global__ void __launch_bounds__(kDecThreads)
    decode_tiled_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ norms,
                        int64_t n, Shape s, const float* __restrict__ rot,
                        const float* __restrict__ cb, TY* __restrict__ y, Gather gather,
                        Rescale rs) {
  extern __shared__ float smem[];
  const int zstride = s.dp + 1;                     // padded rows: conflict-free column reads
  float* zs = smem;                                 // [64][d' + 1] zhat
  float* ps = zs + kTileR * zstride;                // [32][16 RN] chunk of Pi rows
  float* scale = ps + kKChunk * 16 * RN;            // [64] nu (times S), NaN for a bad id
  int64_t* src = reinterpret_cast<int64_t*>(scale + kTileR);  // [64] record of each row
  const int tid = threadIdx.x;
  const int rg = tid >> 4, cg = tid & 15;           // rows 4 rg .. 4 rg + 3, columns cg + 16 j
  const int64_t n_tiles = (n + kTileR - 1) / kTileR;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * kTileR;
    __syncthreads();  // the previous tile's zhat and scales are consumed
    if (tid < kTileR) {
      const int64_t v = row0 + tid;
      int64_t r = -1;
      if (v < n) {
        r = gather.ids ? gather.ids[v] : v;
        if (r < 0 || (gather.ids && r >= gather.n_records)) r = -2;  // outside the plane
      }
      src[tid] = r;
      scale[tid] = r >= 0 ? f16_bits_to_f32(norms[r]) : (r == -2 ? __int_as_float(0x7fc00000) : 0.f);
    }
    __syncthreads();
    // a6: unpack each index once (into the rows' first columns of ps, which is free here)
    int* pid = reinterpret_cast<int*>(ps);
    const bool fit = kTileR * s.m <= kKChunk * 16 * RN;
    if (fit)
      for (int e = tid; e < kTileR * s.m; e += kDecThreads) {
        const int r = e / s.m, j = e - r * s.m;
        const int64_t rec = src[r];
        pid[e] = rec >= 0 ? record_index(codes + rec * s.P, j, s.B) : -1;
      }
    __syncthreads();
    // a7: gather the codewords into the concatenated zhat (consecutive threads read consecutive
    // coordinates of a codeword)
    for (int e = tid; e < kTileR * s.dp; e += kDecThreads) {
      const int r = e / s.dp, c = e - r * s.dp;
      const int j = c / s.k;
      int idx;
      if (fit) {
        idx = pid[r * s.m + j];
      } else {
        const int64_t rec = src[r];
        idx = rec >= 0 ? record_index(codes + rec * s.P, j, s.B) : -1;
      }
      zs[r * zstride + c] = idx >= 0 ? __ldg(cb + (size_t)idx * s.k + (c - j * s.k)) : 0.f;
    }
    __syncthreads();
    if (rs.rho != nullptr && tid < kTileR && src[tid] >= 0) {
      // S of Block Sphere VQ key design 3 from the stored rho and |zbar|^2
      float zz = 0.f;
      for (int c = 0; c < s.dp; ++c) zz = fmaf(zs[tid * zstride + c], zs[tid * zstride + c], zz);
      const float rho = f16_bits_to_f32(rs.rho[src[tid]]);
      const float S = rs.rule == FQ_RESCALE_MSE ? rho / zz
                      : rs.rule == FQ_RESCALE_UNBIASED ? 1.f / rho : 1.f;
      scale[tid] *= S;
    }
    // a8: y = nu (zhat Pi)[0:d] (rows of Pi are output coordinates of the rotation: y_c =
    // sum_k zhat_k Pi[k][c])
    float acc[4][RN];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < RN; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < s.dp; k0 += kKChunk) {
      const int kc = (s.dp - k0) < kKChunk ? (s.dp - k0) : kKChunk;
      __syncthreads();  // the previous chunk is consumed (and the scales are written)
      for (int e = tid; e < kc * 16 * RN; e += kDecThreads) {
        const int kk = e / (16 * RN), c = e - kk * 16 * RN;
        ps[kk * 16 * RN + c] = c < s.d ? __ldg(rot + (size_t)(k0 + kk) * s.dp + c) : 0.f;
      }
      __syncthreads();
      for (int kk = 0; kk < kc; ++kk) {
        float a[4], b[RN];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = zs[(4 * rg + i) * zstride + k0 + kk];
#pragma unroll
        for (int j = 0; j < RN; ++j) b[j] = ps[kk * 16 * RN + cg + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * rg + i;
      const int64_t v = row0 + r;
      if (v < n) {
        const float sc = scale[r];
#pragma unroll
        for (int j = 0; j < RN; ++j) {
          const int c = cg + 16 * j;
          if (c < s.d) store_out(y, v * s.d + c, sc * acc[i][j]);
        }
      }
    }
  }
}

// Tiled encode for any shape without a search index: 64 vectors per tile, 256 threads.  The x
// tile (fp32) sits in shared memory; the rotation is an fp32 FFMA product with Pi^T streamed
// through shared memory in chunks of 32 input coordinates; then one thread per (vector, block)
// searches all N codewords (from shared memory when they fit), lowest index on ties, and the
// records are packed byte by byte.
constexpr int kEncCbSmem = 8192;  // codebook floats kept in shared memory

// Nearest of N codewords of K coordinates to the block zb (direct-form squared distances, the
// block in registers; strict < over increasing c keeps the lowest index on ties).
template <int K>
__device__ __forceinline__ int nearest_small(const float* zb, const float* cbp, int N) {
  float z[K];
#pragma unroll
  for (int q = 0; q < K; ++q) z[q] = zb[q];
  float best = INFINITY;
  int bi = 0;
#pragma unroll 4
  for (int c = 0; c < N; ++c) {
    float dist = 0.f;
#pragma unroll
    for (int q = 0; q < K; ++q) {
      const float t = z[q] - cbp[c * K + q];
      dist = fmaf(t, t, dist);
    }
    if (dist < best) {
      best = dist;
      bi = c;
    }
  }
  return bi;
}

template <typename TX, int RN>
__global__ void __launch_bounds__(kDecThreads)
    encode_tiled_kernel(const TX* __restrict__ x, int64_t n, Shape s,
                        const float* __restrict__ rot, const float* __restrict__ cb,
                        uint8_t* __restrict__ codes, uint16_t* __restrict__ norms,
                        AppendMap map, uint16_t* __restrict__ rho_out) {
  extern __shared__ float smem[];
  const int xstride = s.d + 1, zstride = s.dp + 1;
  float* xs = smem;                                  // [64][d + 1] input tile
  float* zs = xs + kTileR * xstride;                 // [64][d' + 1] z = Pi x / nu
  float* ps = zs + kTileR * zstride;                 // [32][16 RN] chunk of Pi^T
  float* nus = ps + kKChunk * 16 * RN;               // [64] norms
  float* cbs = nus + kTileR;                         // [N k] codebook (when it fits)
  const bool cb_smem = s.N * s.k <= kEncCbSmem;
  int* ids = reinterpret_cast<int*>(cbs + (cb_smem ? s.N * s.k : 0));  // [64][m]
  const int tid = threadIdx.x;
  const int rg = tid >> 4, cg = tid & 15;
  if (cb_smem)
    for (int e = tid; e < s.N * s.k; e += kDecThreads) cbs[e] = __ldg(cb + e);
  const float* cbp = cb_smem ? cbs : cb;
  const int64_t n_tiles = (n + kTileR - 1) / kTileR;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * kTileR;
    __syncthreads();  // the previous tile is fully consumed
    for (int e = tid; e < kTileR * s.d; e += kDecThreads) {
      const int r = e / s.d, c = e - r * s.d;
      xs[r * xstride + c] = row0 + r < n ? load_as_float(x + (row0 + r) * s.d, c) : 0.f;
    }
    __syncthreads();
    if (tid < kTileR) {  // a1: nu, fp32 sum of exact squares
      float ss = 0.f;
      for (int c = 0; c < s.d; ++c) ss = fmaf(xs[tid * xstride + c], xs[tid * xstride + c], ss);
      nus[tid] = sqrtf(ss);
    }
    // a2: z[r][j] = sum_c Pi[j][c] x[r][c] (only the first d columns of Pi meet inputs)
    float acc[4][RN];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < RN; ++j) acc[i][j] = 0.f;
    for (int c0 = 0; c0 < s.d; c0 += kKChunk) {
      const int kc = (s.d - c0) < kKChunk ? (s.d - c0) : kKChunk;
      __syncthreads();
      for (int e = tid; e < kc * 16 * RN; e += kDecThreads) {
        const int j = e / kc, cc = e - j * kc;     // consecutive threads: consecutive c of row j
        ps[cc * 16 * RN + j] = j < s.dp ? __ldg(rot + (size_t)j * s.dp + c0 + cc) : 0.f;
      }
      __syncthreads();
      for (int cc = 0; cc < kc; ++cc) {
        float a[4], b[RN];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = xs[(4 * rg + i) * xstride + c0 + cc];
#pragma unroll
        for (int j = 0; j < RN; ++j) b[j] = ps[cc * 16 * RN + cg + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
    }
    __syncthreads();  // nus written
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * rg + i;
      const float nu = nus[r];
      const float inv = nu > 0.f ? 1.f / nu : 0.f;
#pragma unroll
      for (int j = 0; j < RN; ++j) {
        const int col = cg + 16 * j;
        if (col < s.dp) zs[r * zstride + col] = acc[i][j] * inv;
      }
    }
    __syncthreads();
    // a3 + a4: one thread per (vector, block), all N codewords, lowest index on ties
    for (int e = tid; e < kTileR * s.m; e += kDecThreads) {
      const int r = e / s.m, j = e - r * s.m;
      const float* zb = zs + r * zstride + j * s.k;
      int bi;
      switch (s.k) {
        case 1: bi = nearest_small<1>(zb, cbp, s.N); break;
        case 2: bi = nearest_small<2>(zb, cbp, s.N); break;
        case 3: bi = nearest_small<3>(zb, cbp, s.N); break;
        case 4: bi = nearest_small<4>(zb, cbp, s.N); break;
        default: {
          float best = INFINITY;
          bi = 0;
          for (int c = 0; c < s.N; ++c) {
            const float* cw = cbp + (size_t)c * s.k;
            float dist = 0.f;
            for (int q = 0; q < s.k; ++q) {
              const float t = zb[q] - cw[q];
              dist = fmaf(t, t, dist);
            }
            if (dist < best) {
              best = dist;
              bi = c;
            }
          }
        }
      }
      ids[r * s.m + j] = nus[r] > 0.f ? bi : 0;
    }
    __syncthreads();
    // a5: records (byte by byte), norms, and rho when asked for
    for (int e = tid; e < kTileR * s.P; e += kDecThreads) {
      const int r = e / s.P, b = e - r * s.P;
      if (row0 + r >= n) continue;
      const int64_t dst = dest_row(map, row0 + r);
      if (dst < 0) continue;
      uint32_t byte = 0;
      for (int t = 0; t < 8; ++t) {
        const int i = 8 * b + t;
        const int j = i / s.B;
        if (j < s.m) byte |= uint32_t((ids[r * s.m + j] >> (i - j * s.B)) & 1) << t;
      }
      codes[dst * s.P + b] = (uint8_t)byte;
    }
    if (tid < kTileR && row0 + tid < n) {
      const int64_t v = row0 + tid;
      const int64_t dst = dest_row(map, v);
      if (dst >= 0) norms[dst] = f32_to_f16_bits(nus[tid]);
      if (rho_out != nullptr) {
        // Block Sphere VQ key design 3: rho = <z, zbar> (fp16 like the norm; 1 for a zero vector)
        float part = 0.f;
        for (int c = 0; c < s.dp; ++c) {
          const int j = c / s.k;
          part = fmaf(zs[tid * zstride + c], cbp[(size_t)ids[tid * s.m + j] * s.k + (c - j * s.k)],
                      part);
        }
        rho_out[v] = f32_to_f16_bits(nus[tid] > 0.f ? part : 1.f);
      }
    }
  }
}

size_t encode_tiled_smem(const Shape& s, int rn) {
  const bool cb_smem = s.N * s.k <= kEncCbSmem;
  return ((size_t)kTileR * (s.d + 1) + (size_t)kTileR * (s.dp + 1) + (size_t)kKChunk * 16 * rn +
          kTileR + (cb_smem ? (size_t)s.N * s.k : 0)) * sizeof(float) +
         (size_t)kTileR * s.m * sizeof(int);
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
  // without an index and with a codebook small enough for a per-thread brute force: the tiled
  // kernel; otherwise one warp per vector (candidate lists, or lanes striding over codewords)
  if (index == nullptr && s.N <= 1024 && n >= 2048) {
    const int rn = (s.dp + 15) / 16 <= 4 ? 4 : ((s.dp + 15) / 16 <= 8 ? 8 : 16);
    const size_t smem = encode_tiled_smem(s, rn);
    if (smem <= 200 * 1024) {
      int dev = 0, sms = 148;
      if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      const int64_t tiles = (n + kTileR - 1) / kTileR;
      const int grid = (int)(tiles < (int64_t)sms * 8 ? tiles : (int64_t)sms * 8);
      cudaError_t e = cudaSuccess;
#define FQ_ENC_TILED(TX, RN)                                                                   \
  {                                                                                            \
    auto kern = encode_tiled_kernel<TX, RN>;                                                   \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);    \
    if (e != cudaSuccess) return e;                                                            \
    kern<<<grid, kDecThreads, smem, st>>>(static_cast<const TX*>(x), n, s, rot, cb, codes,     \
                                          norms, map, rho);                                    \
    return cudaGetLastError();                                                                 \
  }
      if (xt == FQ_F16) {
        if (rn == 4) FQ_ENC_TILED(__half, 4)
        if (rn == 8) FQ_ENC_TILED(__half, 8)
        FQ_ENC_TILED(__half, 16)
      }
      if (rn == 4) FQ_ENC_TILED(float, 4)
      if (rn == 8) FQ_ENC_TILED(float, 8)
      FQ_ENC_TILED(float, 16)
#undef FQ_ENC_TILED
    }
  }
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
  const int rn = (s.d + 15) / 16 <= 4 ? 4 : ((s.d + 15) / 16 <= 8 ? 8 : 16);
  const size_t smem = ((size_t)kTileR * (s.dp + 1) + (size_t)kKChunk * 16 * rn + kTileR) *
                          sizeof(float) + kTileR * sizeof(int64_t);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (n + kTileR - 1) / kTileR;
  const int grid = (int)(tiles < (int64_t)sms * 8 ? tiles : (int64_t)sms * 8);
  cudaError_t e = cudaSuccess;
#define FQ_DEC_TILED(TY, RN)                                                                   \
  {                                                                                            \
    auto kern = decode_tiled_kernel<TY, RN>;                                                   \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);    \
    if (e != cudaSuccess) return e;                                                            \
    kern<<<grid, kDecThreads, smem, st>>>(codes, norms, n, s, rot, cb, static_cast<TY*>(y),    \
                                          gather, rs);                                         \
    return cudaGetLastError();                                                                 \
  }
  if (yt == FQ_F16) {
    if (rn == 4) FQ_DEC_TILED(__half, 4)
    if (rn == 8) FQ_DEC_TILED(__half, 8)
    FQ_DEC_TILED(__half, 16)
  }
  if (rn == 4) FQ_DEC_TILED(float, 4)
  if (rn == 8) FQ_DEC_TILED(float, 8)
  FQ_DEC_TILED(float, 16)
#undef FQ_DEC_TILED
  return e;
}

}  // namespace fq
