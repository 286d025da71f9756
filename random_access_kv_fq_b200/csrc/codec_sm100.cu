// sm_100a fast path of fq_encode for fp16 keys/values with d = 64 (k = 2, 3, 4; N <= 256).
//
// Per 128-vector tile (the FibQuant encoder, summary sec. 2.3):
//   TMA      x tile [128 x 64] fp16 -> shared memory (128-byte swizzle, double buffered)
//   tcgen05  D = x * [Pi_hi ; Pi_lo]^T into tensor memory: Pi is split into two fp16 parts,
//            Pi = Pi_hi + 2^-12 Pi_lo, so that with exact fp16 inputs the rotation keeps ~22
//            bits (fp32-class) instead of fp16's 11; both parts share one MMA (N = 2 d').
//   epilogue one thread per vector: z' = D_hi + 2^-12 D_lo, nu from the fp16 inputs in shared
//            memory (pairwise fp32 sum of exact squares), z = z' / nu, nearest codeword per
//            k-block (brute force over the shared-memory codebook, or the grid candidate
//            lists of the search index), indices packed LSB-first into the record, records
//            staged in shared memory and written with 16-byte stores.
// A CTA runs two such pipelines (warps 0-3 and 4-7) that share the rotation, codebook and
// index tables; while one tile is searched, the tensor core already rotates the next.
#include <algorithm>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "codec_sm100.h"
#include "fq_device.cuh"
#include "sm100_ptx.cuh"

namespace fq {

__device__ unsigned int g_fq_wait_timeouts = 0;

namespace sm100 {
namespace {

constexpr int kRows = 128;           // vectors per tile (UMMA M)
constexpr int kGroups = 2;           // pipelines per CTA
constexpr int kThreads = 128 * kGroups;
constexpr int kStages = 2;           // x tiles in flight per pipeline
constexpr int kXBytes = kRows * 128; // 64 fp16 per row
constexpr int kTmemCols = 512;       // 256 columns per pipeline
constexpr int kIndexSmemBudget = 96 * 1024;
constexpr float kLoScale = 1.0f / 4096.0f;  // Pi = Pi_hi + 2^-12 Pi_lo

struct EncParams {
  int64_t n;
  int N;
  const float* rot;
  const float* cb;
  const uint8_t* index;
  uint8_t* codes;
  uint16_t* norms;
};

template <int K, int DP, int B>
struct EncCfg {
  static constexpr int M = DP / K;
  static constexpr int NB = ((2 * DP + 15) / 16) * 16;  // rows of the stacked [Pi_hi; Pi_lo]
  static constexpr int P = (M * B + 7) / 8;
  static constexpr int W = (P + 3) / 4;
  static constexpr int CB_STRIDE = (K <= 3) ? 1 : 2;    // float4 per codeword
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int OFF_X = 0;
  static constexpr int OFF_B = OFF_X + kGroups * kStages * kXBytes;
  static constexpr int OFF_STAGE = OFF_B + NB * 128;
  static constexpr int STAGE_BYTES = ((kRows * P + 15) / 16) * 16;
  static constexpr int OFF_CB = OFF_STAGE + kGroups * STAGE_BYTES;
  static constexpr int CB_BYTES = 256 * CB_STRIDE * 16;
  static constexpr int OFF_BAR = OFF_CB + CB_BYTES;
  static constexpr int OFF_IX = OFF_BAR + 128;
  static constexpr int SMEM = OFF_IX + kIndexSmemBudget + 1024;  // + alignment slack
};

// acc + lo^2 + hi^2 for the two fp16 values packed in hw (the products are exact)
__device__ __forceinline__ float sq2_acc(uint32_t hw, float acc) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "fma.rn.f32.f16 %0, lo, lo, %0;\n\tfma.rn.f32.f16 %0, hi, hi, %0;\n\t}"
      : "+f"(acc)
      : "r"(hw));
  return acc;
}

__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;" ::"r"(g + 1), "r"(128) : "memory");
}

// ---- nearest-codeword search policies ------------------------------------------------------
// Scores are 1 + |c|^2 - 2 z.c: the squared distance minus |z|^2 (common to all candidates)
// plus a constant.  Candidates are scanned in increasing index order with a strict less-than,
// so equal distances keep the lowest index, as in the oracle.
__device__ __forceinline__ void take_if_less(float s, int c, float& best, int& bi) {
  const bool lt = s < best;
  best = lt ? s : best;
  bi = lt ? c : bi;
}

// score of codeword c from the shared-memory table (-2c, 1 + |c|^2)
template <int K>
__device__ __forceinline__ float score_tbl(const float4* __restrict__ tbl, int c, const float (&zb)[K]) {
  if constexpr (K <= 3) {
    const float4 t = tbl[c];
    float s = fmaf(zb[0], t.x, t.w);
    if constexpr (K >= 2) s = fmaf(zb[1], t.y, s);
    if constexpr (K >= 3) s = fmaf(zb[2], t.z, s);
    return s;
  } else {
    const float4 t = tbl[2 * c];
    const float cc = tbl[2 * c + 1].x;
    float s = fmaf(zb[0], t.x, cc);
    s = fmaf(zb[1], t.y, s);
    s = fmaf(zb[2], t.z, s);
    return fmaf(zb[3], t.w, s);
  }
}

// flat grid cell: c_a = clamp(floor((z_a - lo) / h), 0, L - 1); the floor is a round-down add
// of 2^23 (no conversion instruction)
template <int K>
__device__ __forceinline__ int grid_cell(const float (&zb)[K], float scale, float off, float top,
                                         int L) {
  int flat = 0, mul = 1;
#pragma unroll
  for (int a = 0; a < K; ++a) {
    const float t = fminf(fmaxf(fmaf(zb[a], scale, off), 0.f), top);
    flat += (__float_as_int(__fadd_rd(t, 8388608.0f)) - 0x4B000000) * mul;
    mul *= L;
  }
  return flat;
}

struct GridParams {
  const uint8_t* cells;
  float scale, off, top;
  int L, slots, entry, idb;
};

// Exact grid lists of at most 4W one-byte ids per cell in W 32-bit words (branch-free; the
// padding repeats the last id, which cannot change the result).
template <int K, int B, int W>
struct SearchWords {
  GridParams g;
  const float4* tbl;
  __device__ __forceinline__ int find(const float (&zb)[K]) const {
    const uint32_t* e = reinterpret_cast<const uint32_t*>(g.cells) +
                        (size_t)grid_cell<K>(zb, g.scale, g.off, g.top, g.L) * W;
    uint32_t ids[W];
    if constexpr (W == 2) {
      const uint2 v = *reinterpret_cast<const uint2*>(e);
      ids[0] = v.x;
      ids[1] = v.y;
    } else {
#pragma unroll
      for (int w = 0; w < W; ++w) ids[w] = e[w];
    }
    int bi = ids[0] & 0xFFu;
    float best = score_tbl<K>(tbl, bi, zb);
#pragma unroll
    for (int q = 1; q < 4 * W; ++q) {
      const int c = (ids[q / 4] >> (8 * (q % 4))) & 0xFFu;
      take_if_less(score_tbl<K>(tbl, c, zb), c, best, bi);
    }
    return bi;
  }
};

// Exact grid lists of any length (runtime slot count).
template <int K, int B>
struct SearchList {
  GridParams g;
  const float4* tbl;
  __device__ __forceinline__ int find(const float (&zb)[K]) const {
    const uint8_t* e =
        g.cells + (size_t)grid_cell<K>(zb, g.scale, g.off, g.top, g.L) * g.entry;
    float best = INFINITY;
    int bi = 0;
    for (int q = 0; q < g.slots; ++q) {
      const int c = g.idb == 1 ? e[q] : reinterpret_cast<const uint16_t*>(e)[q];
      take_if_less(score_tbl<K>(tbl, c, zb), c, best, bi);
    }
    return bi;
  }
};

// All N codewords from the shared-memory table.
template <int K, int B>
struct SearchAll {
  const float4* tbl;
  int N;
  __device__ __forceinline__ int find(const float (&zb)[K]) const {
    float best = INFINITY;
    int bi = 0;
#pragma unroll 4
    for (int c = 0; c < N; ++c) take_if_less(score_tbl<K>(tbl, c, zb), c, best, bi);
    return bi;
  }
};

// All N = 2^B <= 16 codewords held in registers; two candidates scored per packed FMA.
template <int K, int B>
struct SearchRegs {
  static constexpr int N = 1 << B;
  static constexpr int NP = (N + 1) / 2;
  float2 m[NP][K];
  float2 cc[NP];
  __device__ __forceinline__ void load(const float4* __restrict__ tbl) {
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      float a[2][4], c2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = (2 * q + h < N) ? 2 * q + h : 2 * q;
        if constexpr (K <= 3) {
          const float4 t = tbl[c];
          a[h][0] = t.x; a[h][1] = t.y; a[h][2] = t.z; a[h][3] = 0.f;
          c2[h] = t.w;
        } else {
          const float4 t = tbl[2 * c];
          a[h][0] = t.x; a[h][1] = t.y; a[h][2] = t.z; a[h][3] = t.w;
          c2[h] = tbl[2 * c + 1].x;
        }
      }
#pragma unroll
      for (int k = 0; k < K; ++k) m[q][k] = make_float2(a[0][k], a[1][k]);
      cc[q] = make_float2(c2[0], c2[1]);
    }
  }
  __device__ __forceinline__ int find(const float (&zb)[K]) const {
    float best = INFINITY;
    int bi = 0;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      float2 s = cc[q];
#pragma unroll
      for (int k = 0; k < K; ++k) s = __ffma2_rn(make_float2(zb[k], zb[k]), m[q][k], s);
      take_if_less(s.x, 2 * q, best, bi);
      if (2 * q + 1 < N) take_if_less(s.y, 2 * q + 1, best, bi);
    }
    return bi;
  }
};

template <int K, int DP, int B, bool GRID>
__global__ void __launch_bounds__(kThreads, 1)
    encode_f16_d64_kernel(const __grid_constant__ CUtensorMap xmap, EncParams p) {
  using C = EncCfg<K, DP, B>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem + C::OFF_X;
  uint8_t* sB = smem + C::OFF_B;
  float4* sCb = reinterpret_cast<float4*>(smem + C::OFF_CB);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // per group: full[2], mma
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 96);
  int* sFlag = reinterpret_cast<int*>(smem + C::OFF_BAR + 104);
  uint8_t* sIxSmem = smem + C::OFF_IX;

  const int tid = threadIdx.x;
  const int g = tid >> 7;
  const int lt = tid & 127;
  const int warp = tid >> 5;

  // ---- set-up: tensor memory, barriers, rotation / codebook / index tables ----
  const int64_t n_tiles = (p.n + kRows - 1) / kRows;
  const int64_t stride = (int64_t)gridDim.x * kGroups;
  const int64_t first = (int64_t)blockIdx.x * kGroups + g;
  uint64_t* full = bars + 3 * g;
  uint64_t* mma_bar = bars + 3 * g + 2;
  uint8_t* Xg = sX + g * kStages * kXBytes;
  const bool leader = (lt == 0);
  auto issue_load = [&](int64_t tile, int s) {
    ptx::mbar_arrive_expect_tx(&full[s], kXBytes);
    ptx::tma_load_2d(Xg + s * kXBytes, &xmap, &full[s], 0, (int)(tile * kRows));
  };
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (leader) {  // each pipeline starts its first x loads before the tables are built
    for (int i = 0; i < 3; ++i) ptx::mbar_init(&bars[3 * g + i], 1);
    sFlag[g] = 0;
    ptx::fence_mbar_init();
    if (first < n_tiles) {
      ptx::prefetch_tensormap(&xmap);
      for (int s = 0; s < kStages; ++s)
        if (first + s * stride < n_tiles) issue_load(first + s * stride, s);
    }
  }
  // B operand: row r < DP holds Pi_hi[r][0:64], row DP + r holds Pi_lo[r][0:64], rest zero.
  // Coalesced loads (consecutive threads read consecutive columns), all issued before use.
  {
    constexpr int kElems = DP * 64;  // Pi[:, 0:64]
    constexpr int kIter = (kElems + kThreads - 1) / kThreads;
    float v[kIter];
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int e = tid + it * kThreads;
      if (e < kElems) v[it] = __ldg(p.rot + (size_t)(e >> 6) * DP + (e & 63));
    }
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int e = tid + it * kThreads;
      if (e < kElems) {
        const int r = e >> 6, c = e & 63;
        const __half hi = __float2half_rn(v[it]);
        *reinterpret_cast<__half*>(sB + ptx::sw128_offset(r, c)) = hi;
        *reinterpret_cast<__half*>(sB + ptx::sw128_offset(DP + r, c)) =
            __float2half_rn((v[it] - __half2float(hi)) * 4096.0f);
      }
    }
    for (int e = tid; e < (C::NB - 2 * DP) * 64; e += kThreads)
      *reinterpret_cast<__half*>(sB + ptx::sw128_offset(2 * DP + (e >> 6), e & 63)) =
          __float2half_rn(0.f);
  }
  // codebook table: (-2c, 1 + |c|^2) per codeword (see the search policies)
  for (int c = tid; c < p.N; c += kThreads) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    float cc = 1.f;
#pragma unroll
    for (int a = 0; a < K; ++a) {
      v[a] = __ldg(p.cb + (size_t)c * K + a);
      cc = fmaf(v[a], v[a], cc);
    }
    if constexpr (K <= 3) {
      sCb[c] = make_float4(-2.f * v[0], -2.f * v[1], -2.f * v[2], cc);
    } else {
      sCb[2 * c] = make_float4(-2.f * v[0], -2.f * v[1], -2.f * v[2], -2.f * v[3]);
      sCb[2 * c + 1] = make_float4(cc, 0.f, 0.f, 0.f);
    }
  }
  // search index: used when it describes this (k, N, d') and has no overflow lists
  int mode = 2;  // 0 / 3: four / eight one-byte ids per cell, 1: any list, 2: all codewords
  GridParams gp{};
  if (GRID && p.index != nullptr) {
    const IndexHeader h = *reinterpret_cast<const IndexHeader*>(p.index);
    if (h.magic == kIndexMagic && h.version == kIndexVersion && h.k == K && h.N == p.N &&
        h.dp == DP && !index_has_overflow(h)) {
      mode = (h.id_bytes == 1 && h.entry_bytes == 4) ? 0
             : (h.id_bytes == 1 && h.entry_bytes == 8) ? 3 : 1;
      gp.L = h.L;
      gp.slots = h.slots;
      gp.entry = h.entry_bytes;
      gp.idb = h.id_bytes;
      gp.scale = h.inv_h;
      gp.off = -h.lo * h.inv_h;
      gp.top = (float)(h.L - 1);
      const size_t bytes = (size_t)h.n_cells * h.entry_bytes;
      if (bytes <= (size_t)kIndexSmemBudget) {
        const uint4* src = reinterpret_cast<const uint4*>(p.index + h.cells_offset);
        uint4* dst = reinterpret_cast<uint4*>(sIxSmem);
        const int nv = (int)(bytes / 16);
        for (int i0 = 0; i0 < nv; i0 += 8 * kThreads) {
          uint4 t[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int i = i0 + q * kThreads + tid;
            if (i < nv) t[q] = __ldg(src + i);
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int i = i0 + q * kThreads + tid;
            if (i < nv) dst[i] = t[q];
          }
        }
        for (size_t i = (bytes / 16) * 16 + tid; i < bytes; i += kThreads)
          sIxSmem[i] = p.index[h.cells_offset + i];
        gp.cells = sIxSmem;
      } else {
        gp.cells = p.index + h.cells_offset;
      }
    }
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;

  // ---- pipeline g ----
  uint8_t* stage = smem + C::OFF_STAGE + g * C::STAGE_BYTES;
  const uint32_t acc = tmem + g * 256;
  constexpr uint32_t idesc = ptx::idesc_f16_f32(128, C::NB);
  const uint32_t sB_addr = ptx::smem_u32(sB);

  auto issue_mma = [&](int s, uint32_t parity) -> bool {
    if (!ptx::mbar_wait(&full[s], parity)) return false;
    ptx::tc_fence_after();
    const uint32_t a_addr = ptx::smem_u32(Xg + s * kXBytes);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      ptx::umma_f16(acc, ptx::sdesc_kmajor_sw128(a_addr + kk * 32),
                    ptx::sdesc_kmajor_sw128(sB_addr + kk * 32), idesc, kk > 0 ? 1u : 0u);
    ptx::umma_commit(mma_bar);
    return true;
  };

  if (leader && first < n_tiles) {
    if (!issue_mma(0, 0)) atomicExch(&sFlag[g], 1);
  }

  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  // The tile loop, instantiated once per search policy; the policy is chosen once per CTA so
  // that only one version is hot in the instruction cache.
  auto run = [&](const auto& search) {
  int i = 0;
  for (int64_t tile = first; tile < n_tiles; tile += stride, ++i) {
    const int s = i & 1;
    bool ok = ptx::mbar_wait(mma_bar, i & 1);
    ptx::tc_fence_after();
    // nu from the exact fp16 inputs (fp16 x fp16 products are exact in fp32): eight 8-term
    // partial sums, then a balanced tree
    const uint8_t* xrow = Xg + s * kXBytes + lt * 128;
    float part[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(xrow + (((c ^ (lt & 7)) & 7) << 4));
      float a2 = 0.f;
      a2 = sq2_acc(v.x, a2);
      a2 = sq2_acc(v.y, a2);
      a2 = sq2_acc(v.z, a2);
      a2 = sq2_acc(v.w, a2);
      part[c] = a2;
    }
    const float ss = ((part[0] + part[1]) + (part[2] + part[3])) +
                     ((part[4] + part[5]) + (part[6] + part[7]));
    const float nu = sqrtf(ss);
    const float rinv = nu > 0.f ? __frcp_rn(nu) : 0.f;
    // unit rotated vector z = (D_hi + 2^-12 D_lo) / nu, two coordinates per packed op
    float z[DP];
    const float2 r2 = make_float2(rinv, rinv);
    const float2 l2 = make_float2(kLoScale * rinv, kLoScale * rinv);
#pragma unroll
    for (int c = 0; c + 16 <= DP; c += 16) {
      uint32_t h[16], l[16];
      ptx::tmem_ld16(acc + lane_base + c, h);
      ptx::tmem_ld16(acc + lane_base + DP + c, l);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const float2 hv = make_float2(__uint_as_float(h[e]), __uint_as_float(h[e + 1]));
        const float2 lv = make_float2(__uint_as_float(l[e]), __uint_as_float(l[e + 1]));
        const float2 zz = __ffma2_rn(lv, l2, __fmul2_rn(hv, r2));
        z[c + e] = zz.x;
        z[c + e + 1] = zz.y;
      }
    }
    if constexpr (DP % 16 == 2) {
      uint32_t h[2], l[2];
      ptx::tmem_ld2(acc + lane_base + (DP - 2), h);
      ptx::tmem_ld2(acc + lane_base + DP + (DP - 2), l);
      ptx::tmem_wait_ld();
      const float2 hv = make_float2(__uint_as_float(h[0]), __uint_as_float(h[1]));
      const float2 lv = make_float2(__uint_as_float(l[0]), __uint_as_float(l[1]));
      const float2 zz = __ffma2_rn(lv, l2, __fmul2_rn(hv, r2));
      z[DP - 2] = zz.x;
      z[DP - 1] = zz.y;
    }

    ptx::tc_fence_before();
    if (!ok) atomicExch(&sFlag[g], 1);
    group_sync(g);  // TMEM and the x stage of this tile are no longer read
    if (*(volatile int*)&sFlag[g]) break;  // only this pipeline's threads write its flag
    if (leader) {
      ptx::tc_fence_after();
      if (tile + kStages * stride < n_tiles) issue_load(tile + kStages * stride, s);
      if (tile + stride < n_tiles && !issue_mma(s ^ 1, ((i + 1) >> 1) & 1))
        atomicExch(&sFlag[g], 1);
    }

    // nearest codeword per block, packed LSB-first
    uint32_t w[C::W];
#pragma unroll
    for (int q = 0; q < C::W; ++q) w[q] = 0u;
#pragma unroll
    for (int j = 0; j < C::M; ++j) {
      float zb[K];
#pragma unroll
      for (int a = 0; a < K; ++a) zb[a] = z[j * K + a];
      const int bi = search.find(zb);
      const int off = j * B;  // compile-time after unrolling
      w[off / 32] |= (uint32_t)bi << (off % 32);
      if ((off % 32) + B > 32) w[off / 32 + 1] |= (uint32_t)bi >> (32 - off % 32);
    }
    if (!(nu > 0.f)) {
#pragma unroll
      for (int q = 0; q < C::W; ++q) w[q] = 0u;
    }
    // stage the record at byte lt * P with the widest aligned stores
    uint8_t* rec = stage + lt * C::P;
    if constexpr (C::P % 16 == 0) {
#pragma unroll
      for (int q = 0; q < C::P / 16; ++q)
        reinterpret_cast<uint4*>(rec)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    } else if constexpr (C::P % 4 == 0) {
#pragma unroll
      for (int q = 0; q < C::P / 4; ++q) reinterpret_cast<uint32_t*>(rec)[q] = w[q];
    } else if constexpr (C::P % 2 == 0) {
#pragma unroll
      for (int q = 0; q < C::P / 2; ++q)
        reinterpret_cast<uint16_t*>(rec)[q] = (uint16_t)(w[q / 2] >> (16 * (q & 1)));
    } else {
#pragma unroll
      for (int q = 0; q < C::P; ++q) rec[q] = (uint8_t)(w[q / 4] >> (8 * (q & 3)));
    }
    const int64_t row = tile * kRows + lt;
    if (row < p.n) p.norms[row] = f32_to_f16_bits(nu);
    group_sync(g);
    // coalesced copy of the tile's records
    const int64_t rem = p.n - tile * kRows;
    const int64_t rows = rem < kRows ? rem : (int64_t)kRows;
    uint8_t* dst = p.codes + tile * kRows * C::P;
    const int bytes = (int)(rows * C::P);
    for (int q = lt; q < bytes / 16; q += 128)
      reinterpret_cast<uint4*>(dst)[q] = reinterpret_cast<const uint4*>(stage)[q];
    for (int q = (bytes / 16) * 16 + lt; q < bytes; q += 128) dst[q] = stage[q];
  }
  };

  if constexpr (!GRID && B <= 4) {
    SearchRegs<K, B> sr;
    sr.load(sCb);
    run(sr);
  } else {
    if (mode == 0)
      run(SearchWords<K, B, 1>{gp, sCb});
    else if (mode == 3)
      run(SearchWords<K, B, 2>{gp, sCb});
    else if (mode == 1)
      run(SearchList<K, B>{gp, sCb});
    else
      run(SearchAll<K, B>{sCb, p.N});
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && (sFlag[0] | sFlag[1])) atomicAdd(&g_fq_wait_timeouts, 1u);
  if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ---- host side --------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

bool is_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10;
}

template <int K, int DP, int B, bool GRID>
cudaError_t launch_enc_kernel(const void* x, int64_t n, const EncParams& p, cudaStream_t st) {
  using C = EncCfg<K, DP, B>;
  CUtensorMap map;
  const cuuint64_t dims[2] = {64, (cuuint64_t)n};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {64, kRows};
  const cuuint32_t estr[2] = {1, 1};
  auto fn = encode_tiled_fn();
  if (!fn) return cudaErrorNotSupported;
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = encode_f16_d64_kernel<K, DP, B, GRID>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (n + kRows - 1) / kRows;
  const int64_t ctas = std::min<int64_t>((tiles + kGroups - 1) / kGroups, sm_count());
  kern<<<(int)ctas, kThreads, C::SMEM, st>>>(map, p);
  return cudaGetLastError();
}

template <int K, int DP, int B>
cudaError_t launch_enc(const void* x, int64_t n, const EncParams& p, cudaStream_t st) {
  if (p.index != nullptr) return launch_enc_kernel<K, DP, B, true>(x, n, p, st);
  return launch_enc_kernel<K, DP, B, false>(x, n, p, st);
}

template <int K, int DP>
cudaError_t dispatch_B(int B, const void* x, int64_t n, const EncParams& p, cudaStream_t st) {
  switch (B) {
    case 1: return launch_enc<K, DP, 1>(x, n, p, st);
    case 2: return launch_enc<K, DP, 2>(x, n, p, st);
    case 3: return launch_enc<K, DP, 3>(x, n, p, st);
    case 4: return launch_enc<K, DP, 4>(x, n, p, st);
    case 5: return launch_enc<K, DP, 5>(x, n, p, st);
    case 6: return launch_enc<K, DP, 6>(x, n, p, st);
    case 7: return launch_enc<K, DP, 7>(x, n, p, st);
    case 8: return launch_enc<K, DP, 8>(x, n, p, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace

bool encode_supported(fq_dtype xt, const Shape& s, const void* x, const void* codes,
                      const void* norms) {
  (void)norms;
  if (xt != FQ_F16 || s.d != 64 || s.N > 256 || s.k < 2 || s.k > 4) return false;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(codes) & 15))
    return false;
  return is_sm100() && encode_tiled_fn() != nullptr;
}

cudaError_t launch_encode(const void* x, fq_dtype, int64_t n, const Shape& s, const float* rot,
                          const float* cb, uint8_t* codes, uint16_t* norms, const void* index,
                          cudaStream_t st) {
  if (n > (int64_t)1 << 31) return cudaErrorNotSupported;
  EncParams p;
  p.n = n;
  p.N = s.N;
  p.rot = rot;
  p.cb = cb;
  p.index = static_cast<const uint8_t*>(index);
  p.codes = codes;
  p.norms = norms;
  switch (s.k) {
    case 2: return dispatch_B<2, 64>(s.B, x, n, p, st);
    case 3: return dispatch_B<3, 66>(s.B, x, n, p, st);
    case 4: return dispatch_B<4, 64>(s.B, x, n, p, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace sm100
}  // namespace fq
