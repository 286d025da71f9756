// sm_100a fq_encode for large codebooks: d = 128, k = 4, N = 512 .. 4096, brute-force search on
// the tensor cores with exact fp32 re-ranking of near ties.
//
// Block Sphere VQ notes, key design 2: brute force over N codewords is the throughput
// bottleneck for large codebooks.  The nearest codeword of a block z minimises
//   s(n) = |c_n|^2 + 1 - 2 z.c_n          (= |z - c_n|^2 - |z|^2 + 1),
// a contraction over the 4 coordinates plus a per-codeword constant.  It runs as one K = 16
// fp16 MMA per chunk of 128 codewords, with both sides split into fp16 head and residual parts
// so that the product keeps ~20 bits:
//   A row  (block z)      [ z_hi(4) | z_hi(4)  | z_res(4) | 1       | 1        | 0 0 ]
//   B row  (codeword n)   [ a_hi(4) | a_res(4) | a_hi(4)  | cc_hi   | cc_res   | 0 0 ]
// with a = -2 c_n, cc = |c_n|^2 + 1, x_res = fp16(x - x_hi); the dropped z_res . a_res term is
// ~2^-22 of the score.  The scan keeps, per quarter of the codebook, the two 8-codeword groups
// with the lowest approximate minima; every such group whose minimum lies within kTie of the
// overall best is then re-scored with exact fp32 squared distances to the block (from the fp32
// codebook): the lower distance wins, the lower index on equality, as in the oracle.
//
// One persistent CTA per SM, 128-vector tiles, 17 warps:
//   warps 0-15  four warpgroups; warpgroup 0 (one thread per vector) loads x into tensor memory,
//               computes nu and, per block, the A operand, and resolves the block's codeword;
//               every warpgroup scans one quarter (32 scores) of each 128-codeword chunk:
//               a minimum tree down to four 8-codeword groups and a branch-free update of
//               the best and runner-up group; after each block it re-scores those groups
//   warp 16     issues the rotation MMA and the chunk MMAs (three score buffers in tensor
//               memory, so that two chunks are computed ahead of the one being scanned)
// Tensor memory: columns 0..255 rotation accumulators (hi | lo), combined once per tile into
// fp32 z in columns 0..127; 128..511 three 128-column score buffers (the second also stages x
// during the rotation).
#include <cstdint>

#include <cuda.h>
#include <cuda_fp16.h>

#include "codec_sm100.h"
#include "fq_device.cuh"
#include "sm100_ptx.cuh"

namespace fq {
namespace sm100 {
namespace {

constexpr int kRowsL = 128;               // vectors per tile
constexpr int kScanThreads = 512;
constexpr int kThreadsL = kScanThreads + 32;
constexpr int kDL = 128;                  // d = d'
constexpr int kML = 32;                   // blocks per vector (k = 4)
constexpr int kChunk = 128;               // codewords per MMA
constexpr int kBufs = 3;                  // score buffers in tensor memory (128 columns each)
constexpr uint32_t kTmScore = 128;        // first score buffer column
constexpr int kPer = kChunk / 4;          // scores of a chunk per scanning warpgroup
constexpr float kLoScaleL = 1.0f / 4096.0f;
constexpr float kTie = 1.0f / 8192.0f;    // approximate-score band re-ranked exactly

__device__ unsigned int g_encl_wait_timeouts = 0;

template <int B>
struct LCfg {
  static constexpr int N = 1 << B;
  static constexpr int CHUNKS = N / kChunk;
  static constexpr int P = kML * B / 8;   // 36 .. 48 bytes
  // shared memory (1024-aligned base)
  static constexpr int OFF_PI = 0;                         // [256 x 128] fp16, two sw128 halves
  static constexpr int OFF_CB = OFF_PI + 2 * 256 * 128;    // [N x 16] fp16, no swizzle
  static constexpr int OFF_A = OFF_CB + N * 32;            // two [128 x 16] fp16 A tiles
  static constexpr int OFF_RES = OFF_A + 2 * kRowsL * 32;  // [2][4 warpgroups][128] partials
  static constexpr int OFF_REC = OFF_RES + 2 * 4 * kRowsL * 16;  // records of the tile
  static constexpr int OFF_BAR = OFF_REC + kRowsL * P;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

struct LParams {
  int64_t n;
  const uint16_t* x;
  const float* rot;
  const float* cb;
  uint8_t* codes;
  uint16_t* norms;
};

__device__ __forceinline__ uint32_t h2u_l(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// Bounded wait (at most 2^22 polls, well under a second) that gives up early when another role
// raised the abort flag.  One lane per warp polls with the non-blocking test, so a completed
// phase is seen at once.
__device__ __forceinline__ bool wait_l(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t it = 0; it < (ptx::kSpinLimit << 2); ++it) {
    if (ptx::mbar_test(bar, parity)) return true;
    if ((it & 63u) == 63u && *abort) return false;
  }
  *abort = 1;
  return false;
}

// (value, index) lexicographic "better than"
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v < bv || (v == bv && i < bi);
}

// Barrier among the 512 scanning threads that also ORs a predicate across them.
__device__ __forceinline__ bool scan_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(kScanThreads)
      : "memory");
  return r != 0;
}

// fp16 head and residual of v (the residual is v - head, rounded to fp16)
__device__ __forceinline__ void split_hr(float v, __half& h, __half& r) {
  h = __float2half_rn(v);
  r = __float2half_rn(v - __half2float(h));
}

template <int B>
__global__ void __launch_bounds__(kThreadsL, 1) encode_large_kernel(LParams p) {
  using C = LCfg<B>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sPi = smem + C::OFF_PI;
  uint8_t* sCbOp = smem + C::OFF_CB;
  uint8_t* sA = smem + C::OFF_A;                        // buffer b at b * 4096
  float4* sRes = reinterpret_cast<float4*>(smem + C::OFF_RES);  // [2 blocks][4 wg][128]
  uint64_t* x_ready = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // x staged (4 warps)
  uint64_t* rot_done = x_ready + 1;                                   // rotation MMA done
  uint64_t* a_ready = rot_done + 1;                                   // [2] A tile built (4 warps)
  uint64_t* full = a_ready + 2;                                       // [3] scores ready
  uint64_t* empty = full + kBufs;                                     // [3] scores read (16 warps)
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(empty + kBufs);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);
  uint32_t* sRec = reinterpret_cast<uint32_t*>(smem + C::OFF_REC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = warp >> 2;                     // 0..3 scanners, 4 = MMA warp
  const int row = 32 * (warp & 3) + lane;       // tile row (vector) of this lane
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  const int64_t n_tiles = (p.n + kRowsL - 1) / kRowsL;
  const int n_local =
      (blockIdx.x < n_tiles) ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

  // ---- set-up ----
  if (warp == 16) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(x_ready, kRowsL / 32);
    ptx::mbar_init(rot_done, 1);
    for (int b = 0; b < 2; ++b) ptx::mbar_init(&a_ready[b], kRowsL / 32);
    for (int b = 0; b < kBufs; ++b) {
      ptx::mbar_init(&full[b], 1);
      ptx::mbar_init(&empty[b], kScanThreads / 32);
    }
    *sAbort = 0;
    ptx::fence_mbar_init();
  }
  // rotation operand: row n < 128 holds Pi_hi[n][:], row 128 + n holds Pi_lo[n][:] (2^12-scaled);
  // K split into two 128-byte-swizzled halves
#pragma unroll 1
  for (int e0 = 0; e0 < kDL * kDL; e0 += 8 * kThreadsL) {
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = e0 + q * kThreadsL + tid;
      v[q] = e < kDL * kDL ? __ldg(p.rot + e) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = e0 + q * kThreadsL + tid;
      if (e < kDL * kDL) {
        const int n = e >> 7, c = e & 127;
        const __half hi = __float2half_rn(v[q]);
        const __half lo = __float2half_rn((v[q] - __half2float(hi)) * 4096.0f);
        uint8_t* half_tile = sPi + (c >> 6) * (256 * 128);
        *reinterpret_cast<__half*>(half_tile + ptx::sw128_offset(n, c & 63)) = hi;
        *reinterpret_cast<__half*>(half_tile + ptx::sw128_offset(128 + n, c & 63)) = lo;
      }
    }
  }
  // codeword operand rows: [a_hi(4) a_res(4) | a_hi(4) cc_hi cc_res 0 0], a = -2c, cc = |c|^2 + 1
  for (int n = tid; n < C::N; n += kThreadsL) {
    const float4 c = __ldg(reinterpret_cast<const float4*>(p.cb) + n);
    const float cc = fmaf(c.x, c.x, fmaf(c.y, c.y, fmaf(c.z, c.z, fmaf(c.w, c.w, 1.f))));
    __half ah[4], ar[4], ch, cr;
    split_hr(-2.f * c.x, ah[0], ar[0]);
    split_hr(-2.f * c.y, ah[1], ar[1]);
    split_hr(-2.f * c.z, ah[2], ar[2]);
    split_hr(-2.f * c.w, ah[3], ar[3]);
    split_hr(cc, ch, cr);
    const __half z0 = __float2half_rn(0.f);
    uint8_t* r0 = sCbOp + ptx::noswz16_offset((uint32_t)n, 0);
    *reinterpret_cast<uint4*>(r0) =
        make_uint4(h2u_l(__halves2half2(ah[0], ah[1])), h2u_l(__halves2half2(ah[2], ah[3])),
                   h2u_l(__halves2half2(ar[0], ar[1])), h2u_l(__halves2half2(ar[2], ar[3])));
    *reinterpret_cast<uint4*>(r0 + 128) =
        make_uint4(h2u_l(__halves2half2(ah[0], ah[1])), h2u_l(__halves2half2(ah[2], ah[3])),
                   h2u_l(__halves2half2(ch, cr)), h2u_l(__halves2half2(z0, z0)));
  }
  for (int e = tid; e < kRowsL * C::P / 4; e += kThreadsL) sRec[e] = 0u;
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;
  constexpr uint32_t TM_X = 256;  // x staging (second score buffer)

  if (warp == 16) {
    // ---- MMA issuer: rotation of each tile, then CHUNKS score MMAs per block ----
    uint32_t g = 0;               // score MMAs issued (alternating buffers)
    int rot_issued = 0;
    if (lane == 0) {
      constexpr uint32_t idesc_rot = ptx::idesc_f16_f32(128, 256);
      constexpr uint32_t idesc_s = ptx::idesc_f16_f32(128, kChunk);
      const uint32_t pi = ptx::smem_u32(sPi), cbA = ptx::smem_u32(sCbOp), aA = ptx::smem_u32(sA);
      uint32_t na[2] = {0u, 0u};  // A-ready phases consumed per buffer
      bool ok = true;
      for (int i = 0; i < n_local && ok; ++i) {
        ok = wait_l(x_ready, (uint32_t)i & 1u, sAbort);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          ptx::umma_f16_ts(tmem, tmem + TM_X + 8 * ks,
                           ptx::sdesc_kmajor_sw128(pi + (ks >> 2) * (256 * 128) + (ks & 3) * 32),
                           idesc_rot, ks > 0 ? 1u : 0u);
        ptx::umma_commit(rot_done);
        rot_issued = i + 1;
        // the score buffers overlap the x staging: let the rotation finish first
        ok = wait_l(rot_done, (uint32_t)i & 1u, sAbort);
        for (int j = 0; j < kML && ok; ++j) {
          const int b = j & 1;
          ok = wait_l(&a_ready[b], na[b] & 1u, sAbort);
          if (!ok) break;
          ++na[b];
          const uint64_t ad = ptx::sdesc_kmajor_noswz(aA + b * 4096, 128, 256);
          for (int c = 0; c < C::CHUNKS; ++c, ++g) {
            const int buf = g % kBufs;
            if (g >= kBufs && !(ok = wait_l(&empty[buf], ((g / kBufs) - 1) & 1u, sAbort))) break;
            ptx::tc_fence_after();
            ptx::umma_f16(tmem + kTmScore + kChunk * buf, ad,
                          ptx::sdesc_kmajor_noswz(cbA + kChunk * 32 * c, 128, 256), idesc_s, 0u);
            ptx::umma_commit(&full[buf]);
          }
        }
      }
      if (*sAbort) {  // let this CTA's MMAs in flight land (bounded)
        if (rot_issued > 0) ptx::mbar_wait(rot_done, (uint32_t)(rot_issued - 1) & 1u);
        for (uint32_t t = g >= kBufs ? g - kBufs : 0; t < g; ++t)
          ptx::mbar_wait(&full[t % kBufs], (t / kBufs) & 1u);
      }
    }
    __syncwarp();
  } else {
    // ---- scanners (warpgroup wg: columns 32 wg .. 32 wg + 31 of every chunk) ----
    uint32_t g = 0;
    float nu = 0.f, rinv = 0.f;
    bool aborted = false;
    // A tile of block j for this row (warpgroup 0): z from the rotation in tensor memory
    auto build_a = [&](int j) {
      uint32_t zw[4];
      ptx::tmem_ld4(tmem + lane_base + 4 * j, zw);
      ptx::tmem_wait_ld();
      __half zh[4], zr[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) split_hr(__uint_as_float(zw[a]), zh[a], zr[a]);
      const __half one = __float2half_rn(1.f), z0 = __float2half_rn(0.f);
      uint8_t* r0 = sA + (j & 1) * 4096 + ptx::noswz16_offset((uint32_t)row, 0);
      const uint32_t w0 = h2u_l(__halves2half2(zh[0], zh[1])), w1 = h2u_l(__halves2half2(zh[2], zh[3]));
      *reinterpret_cast<uint4*>(r0) = make_uint4(w0, w1, w0, w1);
      *reinterpret_cast<uint4*>(r0 + 128) =
          make_uint4(h2u_l(__halves2half2(zr[0], zr[1])), h2u_l(__halves2half2(zr[2], zr[3])),
                     h2u_l(__halves2half2(one, one)), h2u_l(__halves2half2(z0, z0)));
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&a_ready[j & 1]);
    };
    for (int i = 0; i < n_local && !aborted; ++i) {
      const int64_t tile = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
      const int64_t vrow = tile * kRowsL + row;
      bool fail = false;
      if (wg == 0) {
        // x row -> tensor memory (A operand of the rotation), nu from the exact fp16 squares
        // in four 16-word pieces
        const uint4* src = reinterpret_cast<const uint4*>(p.x + vrow * kDL);
        float part[8];
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t r16[16];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint4 v = vrow < p.n ? __ldg(src + 4 * q + e) : make_uint4(0u, 0u, 0u, 0u);
            r16[4 * e] = v.x; r16[4 * e + 1] = v.y; r16[4 * e + 2] = v.z; r16[4 * e + 3] = v.w;
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float a2 = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&r16[8 * h + e]));
              a2 = fmaf(f.x, f.x, a2);
              a2 = fmaf(f.y, f.y, a2);
            }
            part[2 * q + h] = a2;
          }
          ptx::tmem_st16(tmem + lane_base + TM_X + 16 * q, r16);
        }
        nu = sqrtf(((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7])));
        rinv = nu > 0.f ? __frcp_rn(nu) : 0.f;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(x_ready);
        fail = !wait_l(rot_done, (uint32_t)i & 1u, sAbort);
        fail = __any_sync(0xffffffffu, fail);
        ptx::tc_fence_after();
        if (!fail) {
          // z = (D_hi + 2^-12 D_lo) / nu into columns 0..127 (frees 128..255 for scores)
#pragma unroll 1
          for (int q = 0; q < 16; ++q) {
            uint32_t h[8], l[8];
            ptx::tmem_ld8(tmem + lane_base + 8 * q, h);
            ptx::tmem_ld8(tmem + lane_base + 128 + 8 * q, l);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e)
              h[e] = __float_as_uint(
                  fmaf(__uint_as_float(l[e]), kLoScaleL * rinv, __uint_as_float(h[e]) * rinv));
            ptx::tmem_st8(tmem + lane_base + 8 * q, h);
          }
          ptx::tmem_wait_st();
          build_a(0);
        }
      }
      for (int j = 0; j < kML; ++j) {
        if (wg == 0 && j + 1 < kML && !fail) build_a(j + 1);
        // Per chunk, this warpgroup's 32 scores reduce to four minima of 8-codeword groups.
        // The best group (bg) and the runner-up group (sg: the best group of another chunk, or
        // the second group of the best chunk) are kept with selects only, as group ids
        // 4 * chunk + group; the codewords inside them are re-scored exactly after the block.
        float best = INFINITY, second = INFINITY;
        int bg = 0, sg = -1;
#pragma unroll 1
        for (int c = 0; c < C::CHUNKS; ++c, ++g) {
          const uint32_t buf = g % kBufs;
          bool ok = true;  // one lane polls the barrier for the warp
          if (lane == 0 && !fail) ok = wait_l(&full[buf], (g / kBufs) & 1u, sAbort);
          fail = fail || __shfl_sync(0xffffffffu, (int)ok, 0) == 0;
          __syncwarp();
          if (fail) continue;
          ptx::tc_fence_after();
          uint32_t v[kPer];
          ptx::tmem_ld_cols<0, kPer>(tmem + lane_base + kTmScore + kChunk * buf + kPer * wg, v);
          ptx::tmem_wait_ld();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&empty[buf]);
          static_assert(kPer == 32, "four 8-column groups per chunk quarter");
          float m2[16], m4[8];
#pragma unroll
          for (int q = 0; q < 16; ++q)
            m2[q] = fminf(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1]));
#pragma unroll
          for (int q = 0; q < 8; ++q) m4[q] = fminf(m2[2 * q], m2[2 * q + 1]);
          // minima of the groups of columns 8k .. 8k + 7
          const float o0 = fminf(m4[0], m4[1]), o1 = fminf(m4[2], m4[3]);
          const float o2 = fminf(m4[4], m4[5]), o3 = fminf(m4[6], m4[7]);
          const bool a01 = o1 < o0, a23 = o3 < o2;
          const float w01 = a01 ? o1 : o0, l01 = a01 ? o0 : o1;
          const float w23 = a23 ? o3 : o2, l23 = a23 ? o2 : o3;
          const bool top = w23 < w01;
          const float mv = top ? w23 : w01;
          const int gid = top ? 2 + (int)a23 : (int)a01;
          const float lt = top ? w01 : w23;  // loser of the final comparison
          const int lid = top ? (int)a01 : 2 + (int)a23;
          const float lw = top ? l23 : l01;  // loser inside the winning pair
          const int wid = top ? 2 + (int)!a23 : (int)!a01;
          const bool rl = lt <= lw;
          const float rv = rl ? lt : lw;     // runner-up group of this chunk
          const int rid = rl ? lid : wid;
          const bool nb = mv < best;         // the earlier group is kept on equal minima
          const bool ns = !nb && mv < second;
          const bool keep_old = best <= rv;  // on a new best: old best or this chunk's runner-up
          second = nb ? (keep_old ? best : rv) : (ns ? mv : second);
          sg = nb ? (keep_old ? bg : 4 * c + rid) : (ns ? 4 * c + gid : sg);
          best = nb ? mv : best;
          bg = nb ? 4 * c + gid : bg;
        }
        float4* mine = sRes + ((j & 1) * 4 + wg) * kRowsL + row;
        *mine = make_float4(best, __int_as_float(bg), second, __int_as_float(sg));
        if (scan_sync_or(fail)) {
          aborted = true;
          break;
        }
        // Every codeword that can be the nearest lies in a group whose approximate minimum is
        // within kTie of the overall approximate best (the approximation errs by ~2^-20).  Each
        // warpgroup re-scores such groups of its own quarter with exact fp32 squared distances
        // (lower distance, then lower index, as the oracle); warpgroup 0 merges the quarters.
        {
          float bv = INFINITY;
#pragma unroll
          for (int w = 0; w < 4; ++w) bv = fminf(bv, sRes[((j & 1) * 4 + w) * kRowsL + row].x);
          const float lim = bv + kTie;
          float z[4];  // the block, from the combined rotation in tensor memory
          {
            uint32_t zw[4];
            ptx::tc_fence_after();
            ptx::tmem_ld4(tmem + lane_base + 4 * j, zw);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int a = 0; a < 4; ++a) z[a] = __uint_as_float(zw[a]);
          }
          float ev = INFINITY;
          int idx = 0;
          const float4* cb4 = reinterpret_cast<const float4*>(p.cb) + kPer * wg;
          auto resolve = [&](int grp, bool take) {  // direct squared distances, as the oracle
            const int n0 = (grp >> 2) * kChunk + 8 * (grp & 3);  // within this quarter
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 c = __ldg(cb4 + n0 + q);
              const float d0 = z[0] - c.x, d1 = z[1] - c.y, d2 = z[2] - c.z, d3 = z[3] - c.w;
              const float dd = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, d3 * d3)));
              const int n = n0 + kPer * wg + q;
              if (take && better(dd, n, ev, idx)) {
                ev = dd;
                idx = n;
              }
            }
          };
          const bool n1 = best <= lim, n2 = sg >= 0 && second <= lim;
          if (__any_sync(0xffffffffu, n1 || n2)) resolve(n1 ? bg : (n2 ? sg : bg), n1 || n2);
          if (__any_sync(0xffffffffu, n1 && n2)) resolve(sg >= 0 ? sg : 0, n1 && n2);
          mine->z = ev;
          mine->w = __int_as_float(idx);
          ptx::tc_fence_before();
        }
        scan_sync_or(false);
        if (wg == 0) {
          float ev = INFINITY;
          int idx = 0;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float4 e = sRes[((j & 1) * 4 + w) * kRowsL + row];
            if (better(e.z, __float_as_int(e.w), ev, idx)) {
              ev = e.z;
              idx = __float_as_int(e.w);
            }
          }
          if (!(nu > 0.f)) idx = 0;
          const uint32_t bit = (uint32_t)(j * B);
          uint32_t* rw = sRec + row * B;  // this row's record words (B words = 32 B bits)
          rw[bit >> 5] |= (uint32_t)idx << (bit & 31);
          if ((bit & 31) + B > 32) rw[(bit >> 5) + 1] |= (uint32_t)idx >> (32 - (bit & 31));
        }
      }
      if (aborted) break;
      if (wg == 0) {  // the tile's record and norm of this row
        uint32_t* rw = sRec + row * B;
        if (vrow < p.n) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(p.codes + vrow * C::P);
#pragma unroll
          for (int q = 0; q < B; ++q) dst[q] = rw[q];
          p.norms[vrow] = f32_to_f16_bits(nu);
        }
#pragma unroll
        for (int q = 0; q < B; ++q) rw[q] = 0u;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *sAbort) atomicAdd(&g_encl_wait_timeouts, 1u);
  if (warp == 16) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int B>
cudaError_t launch_large(const LParams& p, cudaStream_t st) {
  using C = LCfg<B>;
  auto kern = encode_large_kernel<B>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (p.n + kRowsL - 1) / kRowsL;
  const int ctas = (int)(tiles < sms ? tiles : sms);
  kern<<<ctas, kThreadsL, C::SMEM, st>>>(p);
  return cudaGetLastError();
}


}  // namespace

bool encode_large_supported(fq_dtype xt, const Shape& s, const void* x, const void* codes,
                            const float* cb, const void* index) {
  if (xt != FQ_F16 || s.d != kDL || s.k != 4 || index != nullptr) return false;
  if (s.B < 9 || s.B > 12) return false;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(codes) & 3) ||
      (reinterpret_cast<uintptr_t>(cb) & 15))
    return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10;
}

cudaError_t launch_encode_large(const void* x, int64_t n, const Shape& s, const float* rot,
                                const float* cb, uint8_t* codes, uint16_t* norms,
                                cudaStream_t st) {
  LParams p{n, static_cast<const uint16_t*>(x), rot, cb, codes, norms};
  switch (s.B) {
    case 9: return launch_large<9>(p, st);
    case 10: return launch_large<10>(p, st);
    case 11: return launch_large<11>(p, st);
    case 12: return launch_large<12>(p, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace sm100
cudaError_t wait_timeouts_encode_large(bool clear, unsigned* count) {
  return read_wait_counter(sm100::g_encl_wait_timeouts, clear, count);
}

}  // namespace fq
