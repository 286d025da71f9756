// sm_100a fq_encode for d = 128, k = 4, N = 4096 with a grid candidate index (top-c or exact
// without overflow lists): Block Sphere VQ notes, key design 2 (Cartesian grid LUT).
//
// Per block z (4 coordinates of the rotated unit vector), the cell of z on the index's L^4 grid
// names up to 8 candidate codewords; the nearest of them by the direct fp32 squared distance
// wins, the lower index on equality (as the oracle).  An index that does not describe this
// codebook is ignored and every block is searched exactly over all N codewords.
//
// One persistent CTA per SM, 128-vector tiles, software-pipelined across tiles:
//   warp 0       TMA loads of x tiles (two 64-column boxes, 128-byte swizzle) into a
//                two-stage ring
//   warp 1       the rotation of each tile on the tensor cores, A = the x tile in shared memory,
//                B = [Pi_hi ; 2^12 Pi_lo] (fp16 head and scaled residual of Pi), into one of two
//                256-column accumulators in tensor memory
//   warps 2-17   four warpgroups, thread (warpgroup w, row r): the norm of row r from the x
//                tile (32 columns each, partial sums combined in a fixed order), then blocks
//                8w .. 8w + 7 of row r: z from the accumulator, the 8 cells, the 8 index
//                entries loaded at once from L2, the candidates from a shared fp32 codebook
//                table; the 96 record bits are staged in shared memory and the tile's records
//                leave with coalesced 16-byte stores.
// The loads of tile i + 1 and its rotation overlap the search of tile i.
#include <cstdint>

#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "codec_sm100.h"
#include "fq_device.cuh"
#include "sm100_ptx.cuh"

namespace fq {
namespace sm100 {
namespace {

constexpr int kRowsG = 128;
constexpr int kDG = 128;
constexpr int kBG = 12;                    // index bits (N = 4096)
constexpr int kNG = 1 << kBG;
constexpr int kPG = 32 * kBG / 8;          // 48-byte records
constexpr int kSearchThreads = 512;
constexpr int kThreadsG = 64 + kSearchThreads;
constexpr float kLoScaleG = 1.0f / 4096.0f;
constexpr int kXStage = kRowsG * kDG * 2;  // 32 KB: two [128 x 64] fp16 boxes

__device__ unsigned int g_encg_wait_timeouts = 0;  // CTAs whose bounded waits gave up

struct GCfg {
  static constexpr int OFF_PI = 0;                      // [2 K halves][256 rows x 128 B]
  static constexpr int OFF_X = OFF_PI + 2 * 256 * 128;  // [2 stages][2 boxes][128 x 128 B]
  static constexpr int OFF_TBL = OFF_X + 2 * kXStage;   // N x float4 codebook
  static constexpr int OFF_REC = OFF_TBL + kNG * 16;    // [128 rows][48 B] records
  static constexpr int OFF_PART = OFF_REC + kRowsG * kPG;  // [4 quarters][128 rows] norm partials
  static constexpr int OFF_BAR = OFF_PART + kRowsG * 4 * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

struct GParams {
  int64_t n;
  const float* rot;
  const float* cb;
  const uint8_t* index;
  uint8_t* codes;
  uint16_t* norms;
};

// Bounded wait that gives up early when another role raised the abort flag.  try_wait suspends
// the waiting warp in hardware between polls, so waiting warps take no issue slots from the
// working ones.
__device__ __forceinline__ bool wait_g(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t it = 0; it < ptx::kSpinLimit; ++it) {
    if (ptx::mbar_try(bar, parity)) return true;
    if ((it & 15u) == 15u && *abort) return false;
  }
  *abort = 1;
  return false;
}

// Barrier among the 512 search threads that also ORs a predicate across them.
__device__ __forceinline__ bool search_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(kSearchThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool better_g(float v, int i, float bv, int bi) {
  return v < bv || (v == bv && i < bi);
}

// Exact brute force over all N codewords (an index that does not describe this codebook).
// Out of line: it only runs for such an index, and the hot loop stays small.
__device__ __noinline__ int brute_exact(float z0, float z1, float z2, float z3,
                                        const float4* tbl) {
  float best = INFINITY;
  int bi = 0;
  for (int c = 0; c < kNG; ++c) {
    const float4 cv = tbl[c];
    const float d0 = z0 - cv.x, d1 = z1 - cv.y, d2 = z2 - cv.z, d3 = z3 - cv.w;
    const float dd = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, d3 * d3)));
    if (dd < best) {
      best = dd;
      bi = c;
    }
  }
  return bi;
}

__global__ void __launch_bounds__(kThreadsG, 1)
    encode_grid_kernel(const __grid_constant__ CUtensorMap xmap, GParams p) {
  using C = GCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sPi = smem + C::OFF_PI;
  uint8_t* sX = smem + C::OFF_X;
  float4* sTbl = reinterpret_cast<float4*>(smem + C::OFF_TBL);
  uint8_t* sRec = smem + C::OFF_REC;
  float* sPart = reinterpret_cast<float*>(smem + C::OFF_PART);
  uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // [2] x tile landed
  uint64_t* x_empty = x_full + 2;    // [2] rotation done and norms read (2 arrivals)
  uint64_t* z_full = x_empty + 2;    // [2] rotation accumulator ready
  uint64_t* z_empty = z_full + 2;    // [2] accumulator read (16 search warps)
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(z_empty + 2);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (p.n + kRowsG - 1) / kRowsG;
  const int n_local =
      (blockIdx.x < n_tiles) ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

  // ---- set-up ----
  if (warp == 1) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&x_full[s], 1);
      ptx::mbar_init(&x_empty[s], 2);
      ptx::mbar_init(&z_full[s], 1);
      ptx::mbar_init(&z_empty[s], kSearchThreads / 32);
    }
    *sAbort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&xmap);
  }
  const IndexHeader h = *reinterpret_cast<const IndexHeader*>(p.index);
  const bool use_index = h.magic == kIndexMagic && h.version == kIndexVersion && h.k == 4 &&
                         h.N == kNG && h.dp == kDG && h.id_bytes == 2 && h.slots >= 1 &&
                         h.slots <= 8 && h.entry_bytes <= 16 && (h.entry_bytes & 3) == 0 &&
                         !index_has_overflow(h);
  // rotation operand: row c of B holds Pi[c][k] over k (fp16 head rows 0..127, 2^12-scaled
  // residual rows 128..255), two 64-wide K halves in the 128-byte swizzle
#pragma unroll 1
  for (int e0 = 0; e0 < kDG * kDG; e0 += 8 * kThreadsG) {
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = e0 + q * kThreadsG + tid;
      v[q] = e < kDG * kDG ? __ldg(p.rot + e) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = e0 + q * kThreadsG + tid;
      if (e < kDG * kDG) {
        const int n = e >> 7, c = e & 127;
        const __half hi = __float2half_rn(v[q]);
        const __half lo = __float2half_rn((v[q] - __half2float(hi)) * 4096.0f);
        uint8_t* half_tile = sPi + (c >> 6) * (256 * 128);
        *reinterpret_cast<__half*>(half_tile + ptx::sw128_offset(n, c & 63)) = hi;
        *reinterpret_cast<__half*>(half_tile + ptx::sw128_offset(128 + n, c & 63)) = lo;
      }
    }
  }
#pragma unroll 1
  for (int c0 = 0; c0 < kNG; c0 += 4 * kThreadsG) {
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q * kThreadsG + tid;
      v[q] = c < kNG ? __ldg(reinterpret_cast<const float4*>(p.cb) + c) : make_float4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q * kThreadsG + tid;
      if (c < kNG) sTbl[c] = v[q];
    }
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;

  if (warp == 0) {
    // ---- producer: x tiles into the two-stage ring ----
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_local; ++i) {
        const int s = i & 1;
        if (i >= 2 && !wait_g(&x_empty[s], (uint32_t)((i >> 1) - 1) & 1u, sAbort)) break;
        const int64_t tile = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
        ptx::mbar_arrive_expect_tx(&x_full[s], kXStage);
        ptx::tma_load_2d(sX + s * kXStage, &xmap, &x_full[s], 0, (int)(tile * kRowsG));
        ptx::tma_load_2d(sX + s * kXStage + kXStage / 2, &xmap, &x_full[s], 64,
                         (int)(tile * kRowsG));
        issued = i + 1;
      }
      for (int t = issued - 2 < 0 ? 0 : issued - 2; t < issued; ++t)  // in flight: land first
        ptx::mbar_wait(&x_full[t & 1], (uint32_t)(t >> 1) & 1u);
    }
  } else if (warp == 1) {
    // ---- MMA issuer: D_b = X [Pi_hi ; 2^12 Pi_lo]^T ----
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16_f32(128, 256);
      const uint32_t pi = ptx::smem_u32(sPi), xs = ptx::smem_u32(sX);
      int issued = 0;
      for (int i = 0; i < n_local; ++i) {
        const int s = i & 1;
        if (!wait_g(&x_full[s], (uint32_t)(i >> 1) & 1u, sAbort)) break;
        if (i >= 2 && !wait_g(&z_empty[s], (uint32_t)((i >> 1) - 1) & 1u, sAbort)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          ptx::umma_f16(tmem + (uint32_t)(s * 256),
                        ptx::sdesc_kmajor_sw128(xs + s * kXStage + (ks >> 2) * (kXStage / 2) +
                                                (ks & 3) * 32),
                        ptx::sdesc_kmajor_sw128(pi + (ks >> 2) * (256 * 128) + (ks & 3) * 32),
                        idesc, ks > 0 ? 1u : 0u);
        ptx::umma_commit(&x_empty[s]);
        ptx::umma_commit(&z_full[s]);
        issued = i + 1;
      }
      if (issued > 0) ptx::mbar_wait(&z_full[(issued - 1) & 1], (uint32_t)((issued - 1) >> 1) & 1u);
    }
  } else {
    // ---- search threads: warpgroup wg, row r (this warp's tensor-memory lane quarter) ----
    const int sw = warp - 2;                       // 0..15
    const int wg = sw >> 2;
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int st = tid - 64;                       // 0..511
    for (int i = 0; i < n_local; ++i) {
      const int s = i & 1;
      const int64_t tile = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
      const int64_t vrow = tile * kRowsG + r;
      // norm: squares of x[r][32 wg .. 32 wg + 31] from the swizzled tile
      bool fail = !wait_g(&x_full[s], (uint32_t)(i >> 1) & 1u, sAbort);
      if (!fail) {
        const uint8_t* box = sX + s * kXStage + (wg >> 1) * (kXStage / 2);
        float part = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t chunk = (uint32_t)((wg & 1) * 4 + q);
          const uint4 v = *reinterpret_cast<const uint4*>(
              box + (r >> 3) * 1024 + (r & 7) * 128 + (((chunk ^ (uint32_t)(r & 7)) & 7u) << 4));
          const __half2* h2 = reinterpret_cast<const __half2*>(&v);
          float a = 0.f;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f = __half22float2(h2[u]);
            a = fmaf(f.x, f.x, a);
            a = fmaf(f.y, f.y, a);
          }
          part += a;
        }
        sPart[wg * kRowsG + r] = part;
      }
      if (search_sync_or(fail)) break;  // partials in place; the x stage is no longer read
      if (st == 0) ptx::mbar_arrive(&x_empty[s]);
      const float nu = sqrtf((sPart[r] + sPart[kRowsG + r]) + (sPart[2 * kRowsG + r] + sPart[3 * kRowsG + r]));
      const float rinv = nu > 0.f ? __frcp_rn(nu) : 0.f;
      if (wg == 0 && vrow < p.n) p.norms[vrow] = f32_to_f16_bits(nu);
      // z of this thread's 8 blocks: (D_hi + 2^-12 D_lo) / nu
      fail = !wait_g(&z_full[s], (uint32_t)(i >> 1) & 1u, sAbort);
      float z[32];
      if (!fail) {
        ptx::tc_fence_after();
        const uint32_t dz = tmem + lane_base + (uint32_t)(s * 256 + 32 * wg);
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          uint32_t hv[16], lv[16];
          ptx::tmem_ld16(dz + 16 * h16, hv);
          ptx::tmem_ld16(dz + 128 + 16 * h16, lv);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            z[16 * h16 + e] = fmaf(__uint_as_float(lv[e]), kLoScaleG * rinv,
                                   __uint_as_float(hv[e]) * rinv);
        }
        ptx::tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&z_empty[s]);
      uint32_t rec[3] = {0u, 0u, 0u};
      if (!fail && nu > 0.f) {  // a zero vector keeps index 0 in every block
        if (use_index) {
          uint4 ent[8];
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            int flat = 0, mul = 1;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const float t = (z[4 * b + a] - h.lo) * h.inv_h;
              int c = (int)floorf(t);
              c = c < 0 ? 0 : (c >= h.L ? h.L - 1 : c);
              flat += c * mul;
              mul *= h.L;
            }
            const uint8_t* e = p.index + h.cells_offset + (size_t)flat * h.entry_bytes;
            ent[b] = h.entry_bytes == 16
                         ? __ldg(reinterpret_cast<const uint4*>(e))
                         : make_uint4(__ldg(reinterpret_cast<const uint32_t*>(e)),
                                      h.entry_bytes > 4 ? __ldg(reinterpret_cast<const uint32_t*>(e) + 1) : 0u,
                                      h.entry_bytes > 8 ? __ldg(reinterpret_cast<const uint32_t*>(e) + 2) : 0u, 0u);
          }
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            const uint32_t words[4] = {ent[b].x, ent[b].y, ent[b].z, ent[b].w};
            float best = INFINITY;
            int bi = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              if (q < h.slots) {
                const int c = (int)((words[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
                const float4 cv = sTbl[c];
                const float d0 = z[4 * b] - cv.x, d1 = z[4 * b + 1] - cv.y;
                const float d2 = z[4 * b + 2] - cv.z, d3 = z[4 * b + 3] - cv.w;
                const float dd = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, d3 * d3)));
                if (q == 0 || better_g(dd, c, best, bi)) {
                  best = dd;
                  bi = c;
                }
              }
            }
            const uint32_t ix = (uint32_t)bi & (kNG - 1);
            const uint32_t bit = (uint32_t)(b * kBG);
            rec[bit >> 5] |= ix << (bit & 31);
            if ((bit & 31) + kBG > 32) rec[(bit >> 5) + 1] |= ix >> (32 - (bit & 31));
          }
        } else {
#pragma unroll
          for (int b = 0; b < 8; ++b) {  // no usable index: exact brute force over the table
            const int bi = brute_exact(z[4 * b], z[4 * b + 1], z[4 * b + 2], z[4 * b + 3], sTbl);
            const uint32_t ix = (uint32_t)bi & (kNG - 1);
            const uint32_t bit = (uint32_t)(b * kBG);
            rec[bit >> 5] |= ix << (bit & 31);
            if ((bit & 31) + kBG > 32) rec[(bit >> 5) + 1] |= ix >> (32 - (bit & 31));
          }
        }
      }
      uint32_t* rr = reinterpret_cast<uint32_t*>(sRec + r * kPG) + 3 * wg;
      rr[0] = rec[0];
      rr[1] = rec[1];
      rr[2] = rec[2];
      if (search_sync_or(fail)) break;  // the tile's records are staged
      // coalesced 16-byte stores of the tile's records (contiguous in global memory)
      const int64_t rows_here = (p.n - tile * kRowsG) < kRowsG ? (p.n - tile * kRowsG) : kRowsG;
      const int n16 = (int)(rows_here * kPG / 16);
      if (st < n16)
        reinterpret_cast<uint4*>(p.codes + tile * kRowsG * kPG)[st] =
            reinterpret_cast<const uint4*>(sRec)[st];
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *sAbort) atomicAdd(&g_encg_wait_timeouts, 1u);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 grid_tensor_map_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

}  // namespace

bool encode_grid_supported(fq_dtype xt, const Shape& s, const void* x, const void* codes,
                           const float* cb, const void* index) {
  if (xt != FQ_F16 || s.d != kDG || s.k != 4 || s.B != kBG || index == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(codes) & 15) ||
      (reinterpret_cast<uintptr_t>(cb) & 15) || (reinterpret_cast<uintptr_t>(index) & 15))
    return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10 && grid_tensor_map_fn() != nullptr;
}

cudaError_t launch_encode_grid(const void* x, int64_t n, const float* rot, const float* cb,
                               const void* index, uint8_t* codes, uint16_t* norms,
                               cudaStream_t st) {
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)kDG, (cuuint64_t)n};
  const cuuint64_t strides[1] = {(cuuint64_t)kDG * 2};
  const cuuint32_t box[2] = {64, kRowsG};
  const cuuint32_t estr[2] = {1, 1};
  auto fn = grid_tensor_map_fn();
  if (!fn) return cudaErrorNotSupported;
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  GParams p{n, rot, cb, static_cast<const uint8_t*>(index), codes, norms};
  cudaError_t e = cudaFuncSetAttribute(encode_grid_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, GCfg::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (n + kRowsG - 1) / kRowsG;
  const int ctas = (int)(tiles < sms ? tiles : sms);
  encode_grid_kernel<<<ctas, kThreadsG, GCfg::SMEM, st>>>(map, p);
  return cudaGetLastError();
}

}  // namespace sm100
cudaError_t wait_timeouts_encode_grid(bool clear, unsigned* count) {
  return read_wait_counter(sm100::g_encg_wait_timeouts, clear, count);
}

}  // namespace fq
