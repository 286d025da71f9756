// sm_100a fast path of fq_encode for fp16 keys/values with d = 64 (k = 2, 3, 4; N <= 256).
//
// The FibQuant encoder (summary sec. 2.3) per vector x: nu = |x|, z = Pi pad(x) / nu, split z
// into d'/k blocks, nearest codeword per block, indices packed LSB-first into a fixed-size
// record next to the fp16 norm.
//
// A CTA runs four independent pipelines (128 threads each, one thread per vector of a
// 128-vector tile; 16 warps per SM so that one pipeline's waits are covered by the others):
//   TMA      x tile [128 x 64] fp16 -> shared memory (128-byte swizzle)
//   tcgen05  D = x * [Pi_hi ; Pi_lo]^T, coordinates 0..63 of the rotation, into 128 columns of
//            tensor memory: Pi is split into fp16 parts Pi = Pi_hi + 2^-12 Pi_lo, so with exact
//            fp16 inputs the rotation keeps ~22 bits (fp32 class); for d' = 66 (k = 3) the two
//            remaining coordinates are fp32 dot products on the CUDA cores
//   nu       from the fp16 inputs in shared memory (exact squares, fp32 sums)
//   search   blocks in groups of up to 16 coordinates: a runtime loop loads each group's
//            (D_hi, D_lo) columns from tensor memory and searches its blocks (brute force over
//            a codebook held in registers, the grid candidate lists of the search index, or
//            the shared-memory codebook), so the hot code stays small
//   pack     each group's indices are OR-ed into the vector's record in shared memory; the
//            tile's records leave with coalesced 16-byte stores.
// The rescale variant (Block Sphere VQ key design 3, a template flag) also sums, block by block,
// z_b . c of the chosen codeword from the same table and writes rho = <z, zhat> beside the norm.
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

constexpr int kRows = 128;              // vectors per tile (UMMA M)
constexpr int kPipes = 4;               // pipelines per CTA
constexpr int kThreads = 128 * kPipes;
constexpr int kXBytes = kRows * 128;    // one fp16 x tile, 64 values per row
constexpr int kIndexSmemBudget = 80 * 1024;
constexpr float kLoScale = 1.0f / 4096.0f;

__device__ unsigned int g_enc_wait_timeouts = 0;

constexpr int round16(int v) { return (v + 15) / 16 * 16; }

template <int K, int DP, int B>
struct EncCfg {
  static constexpr int M = DP / K;
  static constexpr int P = (M * B + 7) / 8;
  // search groups: G blocks (at most 16 coordinates) per tensor-memory load; the blocks past the
  // last full group (k = 3: blocks 20, 21, coordinates 60..65) form a tail group
  static constexpr int G = (K == 2) ? 8 : (K == 3 ? 5 : 4);
  static constexpr int NG = (M * K <= 64) ? M / G : 64 / (G * K);
  static constexpr int TAIL = M - NG * G;
  // codeword table: k = 2 (c0, c1) as 8 bytes in 16 bank-private copies; k = 3 (-2c, 1 + |c|^2)
  // as 16 bytes in 8 copies; k = 4 as two float4 (one copy).  Lane l reads copy l % REP, so a
  // shared-memory phase of random reads never meets a bank twice.
  static constexpr int ENTRY = (K == 2) ? 8 : (K == 3 ? 16 : 32);
  static constexpr int REP = (K == 2) ? 16 : (K == 3 ? 8 : 1);
  static constexpr int REC = round16(kRows * P) + 16;   // record staging of one pipeline
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int OFF_X = 0;                                // kPipes x tiles
  static constexpr int OFF_B = kPipes * kXBytes;                 // [128 rows x 64] fp16
  static constexpr int OFF_PX = OFF_B + 128 * 128;               // Pi rows 64, 65 (k = 3), fp32
  static constexpr int OFF_REC = OFF_PX + 512;
  static constexpr int OFF_CB = OFF_REC + kPipes * REC;
  static constexpr int OFF_BAR = OFF_CB + 256 * ENTRY * REP;
  static constexpr int OFF_IX = OFF_BAR + 128;
  static constexpr int SMEM = OFF_IX + kIndexSmemBudget + 1024;  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(G * B <= 64, "a group's indices fit one 64-bit word");
};

struct EncParams {
  int64_t n;
  int N;
  const float* rot;
  const float* cb;
  const uint8_t* index;
  uint8_t* codes;
  uint16_t* norms;
  uint16_t* rho;  // the rescale variant: rho = <z, zhat> per vector (fp16), else nullptr
};

// z_b . c of the codeword c whose table entry this lane reads (the table holds c for k = 2 and
// -2c for k = 3, 4)
template <int K>
__device__ __forceinline__ float zdot_tbl(const void* __restrict__ tbl, int c,
                                          const float (&zb)[K]) {
  if constexpr (K == 2) {
    const float2 t = reinterpret_cast<const float2*>(tbl)[c * 16];
    return fmaf(zb[1], t.y, zb[0] * t.x);
  } else if constexpr (K == 3) {
    const float4 t = reinterpret_cast<const float4*>(tbl)[c * 8];
    return -0.5f * fmaf(zb[2], t.z, fmaf(zb[1], t.y, zb[0] * t.x));
  } else {
    const float4 t = reinterpret_cast<const float4*>(tbl)[2 * c];
    return -0.5f * fmaf(zb[3], t.w, fmaf(zb[2], t.z, fmaf(zb[1], t.y, zb[0] * t.x)));
  }
}

// acc + lo^2 + hi^2 for the two fp16 values packed in hw (the products are exact)
__device__ __forceinline__ float sq2_acc(uint32_t hw, float acc) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "fma.rn.f32.f16 %0, lo, lo, %0;\n\tfma.rn.f32.f16 %0, hi, hi, %0;\n\t}"
      : "+f"(acc)
      : "r"(hw));
  return acc;
}

// ---- nearest-codeword search policies ------------------------------------------------------
// Scores are 1 + |c|^2 - 2 z.c: the squared distance minus |z|^2 (common to all candidates)
// plus a constant.  Candidates are scanned in increasing index order with a strict less-than,
// so equal distances keep the lowest index, as in the oracle.  `tbl` is this lane's copy of the
// codeword table (see EncCfg).
__device__ __forceinline__ void take_if_less(float s, int c, float& best, int& bi) {
  const bool lt = s < best;
  best = lt ? s : best;
  bi = lt ? c : bi;
}

template <int K>
__device__ __forceinline__ float score_tbl(const void* __restrict__ tbl, int c,
                                           const float (&zb)[K]) {
  if constexpr (K == 2) {  // (c0 - 2 z0) c0 + (c1 - 2 z1) c1 + 1
    const float2 t = reinterpret_cast<const float2*>(tbl)[c * 16];
    const float s = fmaf(t.y, fmaf(-2.f, zb[1], t.y), 1.f);
    return fmaf(t.x, fmaf(-2.f, zb[0], t.x), s);
  } else if constexpr (K == 3) {
    const float4 t = reinterpret_cast<const float4*>(tbl)[c * 8];
    float s = fmaf(zb[0], t.x, t.w);
    s = fmaf(zb[1], t.y, s);
    return fmaf(zb[2], t.z, s);
  } else {
    const float4 t = reinterpret_cast<const float4*>(tbl)[2 * c];
    const float cc = reinterpret_cast<const float4*>(tbl)[2 * c + 1].x;
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
template <int K, int W>
struct SearchWords {
  GridParams g;
  const void* tbl;
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
template <int K>
struct SearchList {
  GridParams g;
  const void* tbl;
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
template <int K>
struct SearchAll {
  const void* tbl;
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
  __device__ __forceinline__ void load(const void* __restrict__ tbl) {
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      float a[2][4], c2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = (2 * q + h < N) ? 2 * q + h : 2 * q;
        if constexpr (K == 2) {
          const float2 t = reinterpret_cast<const float2*>(tbl)[c * 16];
          a[h][0] = -2.f * t.x; a[h][1] = -2.f * t.y; a[h][2] = a[h][3] = 0.f;
          c2[h] = fmaf(t.x, t.x, fmaf(t.y, t.y, 1.f));
        } else if constexpr (K == 3) {
          const float4 t = reinterpret_cast<const float4*>(tbl)[c * 8];
          a[h][0] = t.x; a[h][1] = t.y; a[h][2] = t.z; a[h][3] = 0.f;
          c2[h] = t.w;
        } else {
          const float4 t = reinterpret_cast<const float4*>(tbl)[2 * c];
          a[h][0] = t.x; a[h][1] = t.y; a[h][2] = t.z; a[h][3] = t.w;
          c2[h] = reinterpret_cast<const float4*>(tbl)[2 * c + 1].x;
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

// ORs the 64-bit field v into the record bits starting at `bit` of the staging area (the field
// spans at most three words; neighbouring records may share a word, hence the atomics).
__device__ __forceinline__ void or_bits(uint32_t* st, uint32_t bit, uint64_t v) {
  const uint32_t w = bit >> 5, sh = bit & 31;
  const uint64_t lo = v << sh;
  const uint32_t hi = sh ? (uint32_t)(v >> (64 - sh)) : 0u;
  if ((uint32_t)lo) atomicOr(st + w, (uint32_t)lo);
  if ((uint32_t)(lo >> 32)) atomicOr(st + w + 1, (uint32_t)(lo >> 32));
  if (hi) atomicOr(st + w + 2, hi);
}

// Barrier among the 128 threads of one pipeline that also ORs a predicate across them.
__device__ __forceinline__ bool pipe_sync_or(int pipe, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(pipe + 1), "r"(128)
      : "memory");
  return r != 0;
}

template <int K, int DP, int B, bool GRID, bool RHO>
__global__ void __launch_bounds__(kThreads, 1)
    encode_kernel(const __grid_constant__ CUtensorMap xmap, EncParams p) {
  using C = EncCfg<K, DP, B>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem + C::OFF_X;
  uint8_t* sB = smem + C::OFF_B;
  float2* sPx = reinterpret_cast<float2*>(smem + C::OFF_PX);  // (Pi[64][c], Pi[65][c])
  float4* sCb = reinterpret_cast<float4*>(smem + C::OFF_CB);
  uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // one per pipeline
  uint64_t* mma_done = x_full + kPipes;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(mma_done + kPipes);
  uint8_t* sIx = smem + C::OFF_IX;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int pipe = tid >> 7, lt = tid & 127;
  const int64_t n_tiles = (p.n + kRows - 1) / kRows;
  const int64_t stride = (int64_t)gridDim.x * kPipes;
  const int64_t first = (int64_t)blockIdx.x * kPipes + pipe;
  uint8_t* xs = sX + pipe * kXBytes;
  auto issue_load = [&](int pp, int64_t tile) {
    ptx::mbar_arrive_expect_tx(&x_full[pp], kXBytes);
    ptx::tma_load_2d(sX + pp * kXBytes, &xmap, &x_full[pp], 0, (int)(tile * kRows));
  };

  // ---- set-up: tensor memory, barriers and the first x tiles, then the tables ----
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    for (int q = 0; q < kPipes; ++q) {
      ptx::mbar_init(&x_full[q], 1);
      ptx::mbar_init(&mma_done[q], 1);
    }
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&xmap);
    for (int q = 0; q < kPipes; ++q)
      if ((int64_t)blockIdx.x * kPipes + q < n_tiles) issue_load(q, (int64_t)blockIdx.x * kPipes + q);
  }
  // B operand: row n < 64 holds Pi_hi[n][0:64], row 64 + n holds Pi_lo[n][0:64]
  {
    constexpr int kIter = 64 * 64 / kThreads;  // all loads issued before the first use
    float v[kIter];
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int e = tid + it * kThreads;
      v[it] = __ldg(p.rot + (size_t)(e >> 6) * DP + (e & 63));
    }
#pragma unroll
    for (int it = 0; it < kIter; ++it) {
      const int e = tid + it * kThreads;
      const int n = e >> 6, c = e & 63;
      const __half hi = __float2half_rn(v[it]);
      *reinterpret_cast<__half*>(sB + ptx::sw128_offset(n, c)) = hi;
      *reinterpret_cast<__half*>(sB + ptx::sw128_offset(64 + n, c)) =
          __float2half_rn((v[it] - __half2float(hi)) * 4096.0f);
    }
  }
  if constexpr (DP > 64) {  // rotation rows 64 and 65 (k = 3), fp32, for the CUDA cores
    for (int c = tid; c < 64; c += kThreads)
      sPx[c] = make_float2(__ldg(p.rot + (size_t)64 * DP + c), __ldg(p.rot + (size_t)65 * DP + c));
  }
  // codebook table: (-2c, 1 + |c|^2) per codeword, REP copies
  for (int c = tid; c < p.N; c += kThreads) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    float cc = 1.f;
#pragma unroll
    for (int a = 0; a < K; ++a) {
      v[a] = __ldg(p.cb + (size_t)c * K + a);
      cc = fmaf(v[a], v[a], cc);
    }
    if constexpr (K == 2) {
      float2* t2 = reinterpret_cast<float2*>(sCb);
#pragma unroll
      for (int r = 0; r < C::REP; ++r) t2[c * C::REP + r] = make_float2(v[0], v[1]);
    } else if constexpr (K == 3) {
      const float4 t = make_float4(-2.f * v[0], -2.f * v[1], -2.f * v[2], cc);
#pragma unroll
      for (int r = 0; r < C::REP; ++r) sCb[c * C::REP + r] = t;
    } else {
      sCb[2 * c] = make_float4(-2.f * v[0], -2.f * v[1], -2.f * v[2], -2.f * v[3]);
      sCb[2 * c + 1] = make_float4(cc, 0.f, 0.f, 0.f);
    }
  }
  // record staging starts zeroed (records are assembled with atomicOr)
  for (int q = tid; q < kPipes * C::REC / 16; q += kThreads)
    reinterpret_cast<uint4*>(smem + C::OFF_REC)[q] = make_uint4(0u, 0u, 0u, 0u);
  // search index: used when it describes this (k, N, d') and has no overflow lists
  int mode = 2;  // 0: one word of ids, 3: two words, 1: list of any length, 2: brute force
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
        uint4* dst = reinterpret_cast<uint4*>(sIx);
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
          sIx[i] = p.index[h.cells_offset + i];
        gp.cells = sIx;
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

  // ---- pipeline `pipe`: tiles first, first + stride, ... ----
  const uint32_t acc = tmem + pipe * 128;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  uint32_t* st = reinterpret_cast<uint32_t*>(smem + C::OFF_REC + pipe * C::REC);
  const void* tbl = reinterpret_cast<const uint8_t*>(sCb) + C::ENTRY * (lt & (C::REP - 1));
  constexpr uint32_t idesc = ptx::idesc_f16_f32(128, 128);
  const uint32_t sB_addr = ptx::smem_u32(sB), x_addr = ptx::smem_u32(xs);
  bool failed = false;
  int64_t issued_tile = first;  // leader: the tile whose x load is in flight (or consumed)
  int mmas = 0;                 // leader: MMAs committed

  auto run = [&](const auto& search) {
    int i = 0;
    for (int64_t tile = first; tile < n_tiles; tile += stride, ++i) {
      bool fail = !ptx::mbar_wait(&x_full[pipe], (uint32_t)i & 1u);
      if (lt == 0 && !fail) {  // rotation of this tile into the pipeline's 128 columns
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_f16(acc, ptx::sdesc_kmajor_sw128(x_addr + kk * 32),
                        ptx::sdesc_kmajor_sw128(sB_addr + kk * 32), idesc, kk > 0 ? 1u : 0u);
        ptx::umma_commit(&mma_done[pipe]);
        ++mmas;
      }
      // nu from the exact fp16 inputs (fp16 x fp16 products are exact in fp32): eight 8-term
      // partial sums, then a balanced tree; for d' = 66 also z[64], z[65] (times nu) in fp32
      const uint8_t* xrow = xs + lt * 128;
      float part[8];
      float2 x6 = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(xrow + (((c ^ (lt & 7)) & 7) << 4));
        float a2 = 0.f;
        a2 = sq2_acc(v.x, a2);
        a2 = sq2_acc(v.y, a2);
        a2 = sq2_acc(v.z, a2);
        a2 = sq2_acc(v.w, a2);
        part[c] = a2;
        if constexpr (DP > 64) {
          const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&hw[q]));
            x6 = __ffma2_rn(make_float2(xf.x, xf.x), sPx[8 * c + 2 * q], x6);
            x6 = __ffma2_rn(make_float2(xf.y, xf.y), sPx[8 * c + 2 * q + 1], x6);
          }
        }
      }
      const float ss = ((part[0] + part[1]) + (part[2] + part[3])) +
                       ((part[4] + part[5]) + (part[6] + part[7]));
      const float nu = sqrtf(ss);
      const float rinv = nu > 0.f ? __frcp_rn(nu) : 0.f;
      // the x stage is free once every thread has read its row
      if (pipe_sync_or(pipe, fail)) {
        failed = true;
        break;
      }
      if (lt == 0 && tile + stride < n_tiles) {
        issue_load(pipe, tile + stride);
        issued_tile = tile + stride;
      }
      fail = !ptx::mbar_wait(&mma_done[pipe], (uint32_t)i & 1u);
      ptx::tc_fence_after();
      const uint32_t bit0 = (uint32_t)lt * (C::P * 8);
      float rho = 0.f;  // RHO: <z, zhat>, block by block
      const float2 r2 = make_float2(rinv, rinv);
      const float2 l2 = make_float2(kLoScale * rinv, kLoScale * rinv);
      // groups of G blocks: z = (D_hi + 2^-12 D_lo) / nu from tensor memory, nearest codewords
#pragma unroll 1
      for (int gi = 0; gi < C::NG; ++gi) {
        uint32_t h[16], l[16];
        ptx::tmem_ld16(acc + lane_base + gi * C::G * K, h);
        ptx::tmem_ld16(acc + lane_base + 64 + gi * C::G * K, l);
        ptx::tmem_wait_ld();
        float z[16];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float2 hv = make_float2(__uint_as_float(h[e]), __uint_as_float(h[e + 1]));
          const float2 lv = make_float2(__uint_as_float(l[e]), __uint_as_float(l[e + 1]));
          const float2 zz = __ffma2_rn(lv, l2, __fmul2_rn(hv, r2));
          z[e] = zz.x;
          z[e + 1] = zz.y;
        }
        uint64_t v = 0;
#pragma unroll
        for (int b = 0; b < C::G; ++b) {
          float zb[K];
#pragma unroll
          for (int a = 0; a < K; ++a) zb[a] = z[b * K + a];
          const int c = search.find(zb);
          v |= (uint64_t)c << (b * B);
          if constexpr (RHO) rho += zdot_tbl<K>(tbl, c, zb);
        }
        if (nu > 0.f) or_bits(st, bit0 + (uint32_t)(gi * C::G * B), v);
      }
      if constexpr (C::TAIL > 0) {  // k = 3: blocks 20, 21 (coordinates 60..63 and 64, 65)
        uint32_t h[4], l[4];
        ptx::tmem_ld4(acc + lane_base + 60, h);
        ptx::tmem_ld4(acc + lane_base + 124, l);
        ptx::tmem_wait_ld();
        float z[6];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          z[e] = fmaf(__uint_as_float(l[e]), kLoScale * rinv, __uint_as_float(h[e]) * rinv);
        z[4] = x6.x * rinv;
        z[5] = x6.y * rinv;
        uint64_t v = 0;
#pragma unroll
        for (int b = 0; b < C::TAIL; ++b) {
          float zb[K];
#pragma unroll
          for (int a = 0; a < K; ++a) zb[a] = z[b * K + a];
          const int c = search.find(zb);
          v |= (uint64_t)c << (b * B);
          if constexpr (RHO) rho += zdot_tbl<K>(tbl, c, zb);
        }
        if (nu > 0.f) or_bits(st, bit0 + (uint32_t)(C::NG * C::G * B), v);
      }
      const int64_t row = tile * kRows + lt;
      if (row < p.n) {
        p.norms[row] = f32_to_f16_bits(nu);
        if constexpr (RHO) p.rho[row] = f32_to_f16_bits(nu > 0.f ? rho : 1.f);  // zero: rho = 1
      }
      ptx::tc_fence_before();
      // tensor memory is free for the next tile's MMA; the tile's records are complete
      if (pipe_sync_or(pipe, fail)) {
        failed = true;
        break;
      }
      // coalesced copy of the tile's records; the staging is left zeroed
      const int64_t rem = p.n - tile * kRows;
      const int bytes = (int)((rem < kRows ? rem : (int64_t)kRows) * C::P);
      uint8_t* dst = p.codes + tile * kRows * C::P;
      uint4* s4 = reinterpret_cast<uint4*>(st);
      for (int q = lt; q < bytes / 16; q += 128) {
        reinterpret_cast<uint4*>(dst)[q] = s4[q];
        s4[q] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (lt == 0) {
        const uint8_t* sb = reinterpret_cast<const uint8_t*>(st);
        for (int b = (bytes / 16) * 16; b < bytes; ++b) dst[b] = sb[b];
        for (int q = bytes / 16; q < C::REC / 16; ++q) s4[q] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };

  if constexpr (B <= 4 && !GRID) {  // N <= 16 without an index: brute force from registers
    SearchRegs<K, B> sr;
    sr.load(tbl);
    run(sr);
  } else {
    if (mode == 0)
      run(SearchWords<K, 1>{gp, tbl});
    else if (mode == 3)
      run(SearchWords<K, 2>{gp, tbl});
    else if (mode == 1)
      run(SearchList<K>{gp, tbl});
    else
      run(SearchAll<K>{tbl, p.N});
  }

  // after a timed-out wait: let this pipeline's own copy and MMA in flight land (bounded)
  if (failed && lt == 0) {
    if (issued_tile < n_tiles) {
      const int li = (int)((issued_tile - first) / stride);
      ptx::mbar_wait(&x_full[pipe], (uint32_t)li & 1u);
    }
    if (mmas > 0) ptx::mbar_wait(&mma_done[pipe], (uint32_t)(mmas - 1) & 1u);
    atomicAdd(&g_enc_wait_timeouts, 1u);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// The driver's tensor-map encoder, looked up once.  A function-local static is initialised
// exactly once even when several host threads make their first call together.
PFN_cuTensorMapEncodeTiled_v12000 enc_tensor_map_fn() {
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

template <int K, int DP, int B, bool GRID, bool RHO>
cudaError_t launch_kernel(const void* x, const EncParams& p, cudaStream_t st) {
  using C = EncCfg<K, DP, B>;
  CUtensorMap map;
  const cuuint64_t dims[2] = {64, (cuuint64_t)p.n};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {64, kRows};
  const cuuint32_t estr[2] = {1, 1};
  auto fn = enc_tensor_map_fn();
  if (!fn) return cudaErrorNotSupported;
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = encode_kernel<K, DP, B, GRID, RHO>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (p.n + kRows - 1) / kRows;
  const int64_t want = (tiles + kPipes - 1) / kPipes;
  const int ctas = (int)(want < sms ? want : sms);
  kern<<<ctas, kThreads, C::SMEM, st>>>(map, p);
  return cudaGetLastError();
}

template <int K, int DP, int B>
cudaError_t launch_rate(const void* x, const EncParams& p, cudaStream_t st) {
  // with an index, codebooks of 16 codewords and more search their grid candidate lists (3
  // candidates at N = 16 against 16 from registers); smaller ones keep the register brute force
  const bool grid = p.index != nullptr && B >= 4;
  if (p.rho != nullptr)
    return grid ? launch_kernel<K, DP, B, true, true>(x, p, st)
                : launch_kernel<K, DP, B, false, true>(x, p, st);
  return grid ? launch_kernel<K, DP, B, true, false>(x, p, st)
              : launch_kernel<K, DP, B, false, false>(x, p, st);
}

template <int K, int DP>
cudaError_t by_b(int B, const void* x, const EncParams& p, cudaStream_t st) {
  switch (B) {
    case 1: return launch_rate<K, DP, 1>(x, p, st);
    case 2: return launch_rate<K, DP, 2>(x, p, st);
    case 3: return launch_rate<K, DP, 3>(x, p, st);
    case 4: return launch_rate<K, DP, 4>(x, p, st);
    case 5: return launch_rate<K, DP, 5>(x, p, st);
    case 6: return launch_rate<K, DP, 6>(x, p, st);
    case 7: return launch_rate<K, DP, 7>(x, p, st);
    case 8: return launch_rate<K, DP, 8>(x, p, st);
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
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10 && enc_tensor_map_fn() != nullptr;
}

cudaError_t launch_encode(const void* x, fq_dtype, int64_t n, const Shape& s, const float* rot,
                          const float* cb, uint8_t* codes, uint16_t* norms, const void* index,
                          cudaStream_t st, uint16_t* rho) {
  if (n > (int64_t)INT32_MAX)  // tensor-map row coordinates are 32-bit
    return launch_encode_generic(x, FQ_F16, n, s, rot, cb, codes, norms, index, st,
                                 AppendMap{nullptr, 1, 0}, rho);
  EncParams p{n, s.N, rot, cb, static_cast<const uint8_t*>(index), codes, norms, rho};
  switch (s.k) {
    case 2: return by_b<2, 64>(s.B, x, p, st);
    case 3: return by_b<3, 66>(s.B, x, p, st);
    case 4: return by_b<4, 64>(s.B, x, p, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace sm100
cudaError_t wait_timeouts_encode(bool clear, unsigned* count) {
  return read_wait_counter(sm100::g_enc_wait_timeouts, clear, count);
}

}  // namespace fq
