// sm_100a fast path of fq_decode for d = 64 (k = 2, 3, 4; N <= 256), fp16 or fp32 output.
//
// The FibQuant decoder (summary sec. 2.3): unpack the record, gather the codewords,
// concatenate them into zhat, apply the inverse rotation and scale by the norm:
//   y = nu (Pi^T zhat)[0:64].
// As one 128-row tile: Y = nu * (Zhat Pi)[:, 0:64], a [128 x d'] x [d' x 64] product on the
// tensor cores.  zhat and Pi are split into fp16 hi and 2^12-scaled lo parts so that the
// product keeps ~22 bits:
//   D[:, 0:128]  = Zhi * [PiT_hi ; PiT_lo]^T     (N = 128)
//   D[:, 64:128] += Zlo * PiT_hi^T               (N = 64)
//   y = nu (D[:, 0:64] + 2^-12 D[:, 64:128]).
//
// Warp roles of a persistent CTA (one per SM, tiles blockIdx.x, blockIdx.x + grid, ...):
//   warp 0      bulk async copies of each tile's records and norms into a ring of kStages
//   warp 1      tensor-memory allocation and the MMAs of each tile
//   warps 2-9   gather: two threads per row unpack the row's record and write its zhat row
//               (hi, lo; half of the coordinates each) into one of two A-operand buffers in
//               tensor memory (the thread's own lane), so the A operand never touches shared
//               memory; they first build the codeword table
//   warps 10-13 epilogue: one thread per row reads its accumulator row from one of two
//               tensor-memory buffers, scales by nu and writes it into a 128-byte swizzled
//               staging tile that one TMA tensor store per warp copies out; they first build
//               the rotation operand, which the MMA warp waits for
// so the copies, the gather of tile i + 1, the MMAs and the epilogue of tile i overlap.
// The rescale variant (Block Sphere VQ key design 3, a template flag) scales each row by S nu
// instead: its epilogue thread unpacks the row's record, sums |c|^2 of its codewords for the MSE
// rule and reads the stored rho.
// Every wait is bounded; a timed-out wait raises an abort flag that ends all roles.
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

constexpr int kRows = 128;
constexpr int kStages = 8;
constexpr int kGatherThreads = 256;  // two threads per row
constexpr int kEpiThreads = 128;     // one thread per row
constexpr int kThreads = 64 + kGatherThreads + kEpiThreads;
constexpr float kLoScale = 1.0f / 4096.0f;

constexpr int round16(int v) { return (v + 15) / 16 * 16; }

template <int K, int DP, int B, bool F16>
struct DecCfg {
  static constexpr int M = DP / K;
  static constexpr int N = 1 << B;
  static constexpr int P = (M * B + 7) / 8;
  static constexpr int KSTEPS = (DP + 15) / 16;          // 4 (d' = 64) or 5 (d' = 66)
  static constexpr bool EXTRA = KSTEPS > 4;             // fifth K step, no-swizzle layout
  // tensor memory: two accumulator buffers (128 columns each), then two A-operand buffers of
  // zhat rows (fp16 pairs per column: hi in A_COLS columns, lo in the next A_COLS)
  static constexpr int A_COLS = KSTEPS * 8;
  static constexpr int TM_A = 256;
  static constexpr int B_BYTES = 128 * 128 + (EXTRA ? 128 * 32 : 0);
  static constexpr int REC = round16(kRows * P);
  static constexpr int STAGE = REC + 256;               // records, then the tile's norms
  // codeword table: fp16 (hi | lo) per codeword, one bank-private copy per lane of a
  // shared-memory phase (16 lanes for 8-byte entries, 8 lanes for 16-byte entries)
  static constexpr int CBE = (K == 2) ? 8 : 16;
  static constexpr int REP = (K == 2) ? 16 : 8;
  // shared memory layout (1024-aligned operand tiles first)
  static constexpr int OFF_B = 0;
  // output staging: per epilogue warp two [32 rows x 128 B] tiles (fp16) or two pairs of them
  // (fp32, columns 0..31 and 32..63), 128-byte swizzled for the TMA tensor store
  static constexpr int OUT_TILE = (F16 ? 1 : 2) * 32 * 128;
  static constexpr int OFF_OUT = ((B_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_RING = OFF_OUT + 4 * 2 * OUT_TILE;
  static constexpr int OFF_CB = OFF_RING + kStages * STAGE;
  static constexpr int OFF_CC = OFF_CB + N * REP * CBE;  // |c|^2 per codeword (the rescale)
  static constexpr int OFF_BAR = OFF_CC + N * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// fp16 hi part and 2^12-scaled fp16 lo part of v
__device__ __forceinline__ void split_f16(float v, __half& hi, __half& lo) {
  hi = __float2half_rn(v);
  lo = __float2half_rn((v - __half2float(hi)) * 4096.0f);
}

__device__ __forceinline__ uint32_t h2u(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// Bounded wait that also gives up when another role has raised the abort flag.
__device__ __forceinline__ bool wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t it = 0; it < ptx::kSpinLimit; ++it) {
    if (ptx::mbar_try(bar, parity)) return true;
    if (*abort) return false;
  }
  *abort = 1;
  return false;
}

// The P-byte record at byte offset o of shared memory `base` as little-endian words (zero
// bytes after the record); reads whole words from o & ~3 on.
template <int P, int NW>
__device__ __forceinline__ void read_rec(const uint8_t* base, uint32_t o, uint32_t (&w)[NW]) {
  if constexpr (P % 4 == 0) {
#pragma unroll
    for (int q = 0; q < P / 4; ++q) w[q] = reinterpret_cast<const uint32_t*>(base + o)[q];
#pragma unroll
    for (int q = P / 4; q < NW; ++q) w[q] = 0u;
  } else {
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(base + (o & ~3u));
    const uint32_t sh = (o & 3u) * 8u;
    constexpr int NR = (P + 3) / 4 + 1;
    uint32_t raw[NR];
#pragma unroll
    for (int q = 0; q < NR; ++q) raw[q] = wp[q];
#pragma unroll
    for (int q = 0; q < NR - 1; ++q) w[q] = __funnelshift_r(raw[q], raw[q + 1], sh);
#pragma unroll
    for (int q = NR - 1; q < NW; ++q) w[q] = 0u;
    w[(P - 1) / 4] &= (1u << (8 * (P % 4))) - 1u;
  }
}

template <int P, int NW>
__device__ __forceinline__ void read_rec_global(const uint8_t* rec, uint32_t (&w)[NW]) {
#pragma unroll
  for (int q = 0; q < NW; ++q) w[q] = 0u;
#pragma unroll
  for (int q = 0; q < P; ++q) w[q / 4] |= uint32_t(rec[q]) << (8 * (q & 3));
}

template <int B, int NW>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[NW], int j) {
  const int off = j * B;
  uint32_t v = w[off / 32] >> (off % 32);
  if ((off % 32) + B > 32) v |= w[off / 32 + 1] << (32 - off % 32);
  return v & ((1u << B) - 1u);
}

// Output word PW of a zhat row (coordinates 2 PW, 2 PW + 1) from the codeword entries of its
// blocks: `hi` picks the (hi0 hi1, hi2 hi3) words of an entry, else the (lo0 lo1, lo2 lo3) ones.
template <int K, int M, int PW>
__device__ __forceinline__ uint32_t zword(const uint4 (&e)[M], bool hi) {
  constexpr int c0 = 2 * PW, c1 = 2 * PW + 1;
  if constexpr (c0 >= K * M) {
    return 0u;
  } else {
    constexpr int j0 = c0 / K, q0 = c0 % K;
    const uint32_t a = hi ? (q0 < 2 ? e[j0].x : e[j0].y) : (q0 < 2 ? e[j0].z : e[j0].w);
    if constexpr (c1 >= K * M) {
      return (q0 & 1) ? (a >> 16) : (a & 0xFFFFu);
    } else {
      constexpr int j1 = c1 / K, q1 = c1 % K;
      const uint32_t b = hi ? (q1 < 2 ? e[j1].x : e[j1].y) : (q1 < 2 ? e[j1].z : e[j1].w);
      if constexpr (j0 == j1 && (q0 < 2) == (q1 < 2) && (q0 & 1) == 0) return a;
      constexpr uint32_t sel = ((q0 & 1) ? 0x32u : 0x10u) | ((q1 & 1) ? 0x7600u : 0x5400u);
      return __byte_perm(a, b, sel);
    }
  }
}

template <int K, int M, int C8>
__device__ __forceinline__ uint4 zchunk(const uint4 (&e)[M], bool hi) {
  return make_uint4(zword<K, M, 4 * C8 + 0>(e, hi), zword<K, M, 4 * C8 + 1>(e, hi),
                    zword<K, M, 4 * C8 + 2>(e, hi), zword<K, M, 4 * C8 + 3>(e, hi));
}

__device__ unsigned int g_dec_wait_timeouts = 0;

struct DecArgs {
  int64_t n;
  const float* rot;
  const float* cb;
  const uint8_t* codes;
  const uint16_t* norms;
  void* y;
  const uint16_t* rho;  // the rescale variant: stored rho per record (fp16) and the S rule
  int rule;
};

// Gather of one half of a zhat row into the tensor-memory A operand (this thread's lane): half 0
// writes coordinates 0..31 (columns 0..15 of the hi and lo parts), half 1 coordinates 32..63
// and, for d' = 66, the fifth K step (coordinates 64, 65 and zeros up to 79).
template <int K, int B, int M, int REP, int NW, int H, bool EXTRA>
__device__ __forceinline__ void gather_half(const uint32_t (&w)[NW], const uint8_t* sCb,
                                            uint32_t vrep, uint32_t ta_hi, uint32_t ta_lo) {
  constexpr int J0 = (32 * H) / K;                                   // first block used
  constexpr int J1 = (H == 0) ? 31 / K : M - 1;                      // last block used
  uint4 e[M];
#pragma unroll
  for (int j = 0; j < M; ++j) {
    if (j >= J0 && j <= J1) {
      const uint32_t ix = field<B>(w, j) * REP + vrep;
      if constexpr (K == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(sCb + ix * 8);
        e[j] = make_uint4(v.x, 0u, v.y, 0u);
      } else {
        e[j] = *reinterpret_cast<const uint4*>(sCb + ix * 16);
      }
    } else {
      e[j] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  uint32_t hw[16], lw[16];
#define FQ_DCHUNK(C8, Q)                          \
  {                                               \
    const uint4 h4 = zchunk<K, M, (C8)>(e, true);  \
    const uint4 l4 = zchunk<K, M, (C8)>(e, false); \
    hw[4 * (Q) + 0] = h4.x;                       \
    hw[4 * (Q) + 1] = h4.y;                       \
    hw[4 * (Q) + 2] = h4.z;                       \
    hw[4 * (Q) + 3] = h4.w;                       \
    lw[4 * (Q) + 0] = l4.x;                       \
    lw[4 * (Q) + 1] = l4.y;                       \
    lw[4 * (Q) + 2] = l4.z;                       \
    lw[4 * (Q) + 3] = l4.w;                       \
  }
  if constexpr (H == 0) {
    FQ_DCHUNK(0, 0) FQ_DCHUNK(1, 1) FQ_DCHUNK(2, 2) FQ_DCHUNK(3, 3)
    ptx::tmem_st16(ta_hi, hw);
    ptx::tmem_st16(ta_lo, lw);
  } else {
    FQ_DCHUNK(4, 0) FQ_DCHUNK(5, 1) FQ_DCHUNK(6, 2) FQ_DCHUNK(7, 3)
    ptx::tmem_st16(ta_hi + 16, hw);
    ptx::tmem_st16(ta_lo + 16, lw);
    if constexpr (EXTRA) {  // coordinates 64..79: 64, 65 and zeros
      const uint4 h4 = zchunk<K, M, 8>(e, true);
      const uint4 l4 = zchunk<K, M, 8>(e, false);
      const uint32_t h8[8] = {h4.x, h4.y, h4.z, h4.w, 0u, 0u, 0u, 0u};
      const uint32_t l8[8] = {l4.x, l4.y, l4.z, l4.w, 0u, 0u, 0u, 0u};
      ptx::tmem_st8(ta_hi + 32, h8);
      ptx::tmem_st8(ta_lo + 32, l8);
    }
  }
#undef FQ_DCHUNK
}

__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int K, int DP, int B, bool F16, bool RS>
__global__ void __launch_bounds__(kThreads, 1)
    decode_ws_kernel(const __grid_constant__ CUtensorMap ymap, DecArgs p) {
  using C = DecCfg<K, DP, B, F16>;
  constexpr int P = C::P;
  constexpr int NW = (P + 3) / 4 + 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sRing = smem + C::OFF_RING;
  uint8_t* sCb = smem + C::OFF_CB;
  uint8_t* sOut = smem + C::OFF_OUT;
  uint64_t* r_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // records landed
  uint64_t* r_empty = r_full + kStages;        // stage read by all gather and epilogue threads
  uint64_t* a_full = r_empty + kStages;        // A buffer written (gather threads)
  uint64_t* a_empty = a_full + 2;              // A buffer read by the MMAs
  uint64_t* d_full = a_empty + 2;              // accumulator ready
  uint64_t* d_empty = d_full + 2;              // accumulator read (epilogue threads)
  uint64_t* b_ready = d_empty + 2;             // B operand in place
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(b_ready + 1);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (p.n + kRows - 1) / kRows;
  const int64_t grid = gridDim.x;
  const int n_local = (blockIdx.x < n_tiles) ? (int)((n_tiles - 1 - blockIdx.x) / grid + 1) : 0;
  auto tile_of = [&](int i) { return (int64_t)blockIdx.x + (int64_t)i * grid; };
  auto rows_of = [&](int64_t tile) {
    const int64_t r = p.n - tile * kRows;
    return r < kRows ? (int)r : kRows;
  };
  // a (last, ragged) tile whose records or norms do not fill whole 16-byte units is read from
  // global memory by the threads themselves
  auto direct = [&](int rows) { return ((rows * P) & 15) != 0 || ((rows * 2) & 15) != 0; };
  auto issue = [&](int i) {  // thread 0
    const int s = i % kStages;
    const int64_t tile = tile_of(i);
    const int rows = rows_of(tile);
    if (direct(rows)) {
      ptx::mbar_arrive_expect_tx(&r_full[s], 0);
      return;
    }
    ptx::mbar_arrive_expect_tx(&r_full[s], (uint32_t)(rows * P + rows * 2));
    ptx::bulk_load(sRing + s * C::STAGE, p.codes + tile * kRows * P, (uint32_t)(rows * P),
                   &r_full[s]);
    ptx::bulk_load(sRing + s * C::STAGE + C::REC, p.norms + tile * kRows, (uint32_t)(rows * 2),
                   &r_full[s]);
  };

  // ---- set-up: barriers, tensor memory and the first copies; the tables are built by the
  //      roles themselves so that they overlap the first tiles
  if (warp == 1) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  int issued = 0;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&r_full[s], 1);
      ptx::mbar_init(&r_empty[s], kGatherThreads + kEpiThreads);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&a_full[b], kGatherThreads);
      ptx::mbar_init(&a_empty[b], 1);
      ptx::mbar_init(&d_full[b], 1);
      ptx::mbar_init(&d_empty[b], kEpiThreads);
    }
    ptx::mbar_init(b_ready, kEpiThreads);
    *sAbort = 0;
    ptx::fence_mbar_init();
    for (; issued < kStages && issued < n_local; ++issued) issue(issued);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;
  int mma_done = 0;

  if (warp == 0) {
    // ---- producer: refill each ring stage once all readers of its previous tile are done
    if (lane == 0) {
      for (int i = issued; i < n_local; ++i) {
        const int s = i % kStages;
        if (!wait_ab(&r_empty[s], (uint32_t)((i / kStages) - 1) & 1u, sAbort)) break;
        issue(i);
        issued = i + 1;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: tile i into accumulator buffer i % 2
    if (lane == 0 && n_local > 0 && wait_ab(b_ready, 0u, sAbort)) {
      constexpr uint32_t idesc128 = ptx::idesc_f16_f32(128, 128);
      constexpr uint32_t idesc64 = ptx::idesc_f16_f32(128, 64);
      // descriptors of the B operand's K steps, built once
      const uint32_t bB = ptx::smem_u32(sB);
      uint64_t bd[C::KSTEPS];
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks)
        bd[ks] = ks < 4 ? ptx::sdesc_kmajor_sw128(bB + ks * 32)
                        : ptx::sdesc_kmajor_noswz(bB + 128 * 128, 128, 256);
      for (int i = 0; i < n_local; ++i) {
        const int b = i & 1;
        if (!wait_ab(&a_full[b], (uint32_t)(i >> 1) & 1u, sAbort)) break;
        if (i >= 2 && !wait_ab(&d_empty[b], (uint32_t)((i >> 1) - 1) & 1u, sAbort)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + b * 128;
        const uint32_t ah = tmem + C::TM_A + b * 2 * C::A_COLS, al = ah + C::A_COLS;
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks)
          ptx::umma_f16_ts(d, ah + 8 * ks, bd[ks], idesc128, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks)
          ptx::umma_f16_ts(d + 64, al + 8 * ks, bd[ks], idesc64, 1u);
        ptx::umma_commit(&a_empty[b]);
        ptx::umma_commit(&d_full[b]);
        mma_done = i + 1;
      }
    }
  } else if (warp < 2 + kGatherThreads / 32) {
    // ---- gather: codeword table first (REP bank-private copies), then row r, half h of tile
    //      i into A buffer i % 2
    const int t = tid - 64;
    for (int e = t; e < C::N * C::REP; e += kGatherThreads) {
      const int c = e / C::REP;
      __half hi[4], lo[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        hi[a] = lo[a] = __float2half_rn(0.f);
        if (a < K) split_f16(__ldg(p.cb + (size_t)c * K + a), hi[a], lo[a]);
      }
      if constexpr (K == 2) {
        *reinterpret_cast<uint2*>(sCb + e * 8) =
            make_uint2(h2u(__halves2half2(hi[0], hi[1])), h2u(__halves2half2(lo[0], lo[1])));
      } else {
        *reinterpret_cast<uint4*>(sCb + e * 16) =
            make_uint4(h2u(__halves2half2(hi[0], hi[1])), h2u(__halves2half2(hi[2], hi[3])),
                       h2u(__halves2half2(lo[0], lo[1])), h2u(__halves2half2(lo[2], lo[3])));
      }
    }
    named_sync(1, kGatherThreads);
    const int r = 32 * (warp & 3) + lane, half = t >> 7;  // rows of this warp's TMEM lanes
    const uint32_t vrep = (uint32_t)(lane & (C::REP - 1));
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    for (int i = 0; i < n_local; ++i) {
      const int s = i % kStages, b = i & 1;
      const int64_t tile = tile_of(i);
      const int rows = rows_of(tile);
      bool ok = wait_ab(&r_full[s], (uint32_t)(i / kStages) & 1u, sAbort);
      if (__any_sync(0xffffffffu, !ok)) break;
      uint32_t w[NW];
      if (r >= rows) {
#pragma unroll
        for (int q = 0; q < NW; ++q) w[q] = 0u;
      } else if (direct(rows)) {
        read_rec_global<P>(p.codes + (tile * kRows + r) * P, w);
      } else {
        read_rec<P>(sRing + s * C::STAGE, (uint32_t)(r * P), w);
      }
      ptx::mbar_arrive(&r_empty[s]);
      if (i >= 2) ok = wait_ab(&a_empty[b], (uint32_t)((i >> 1) - 1) & 1u, sAbort);
      if (__any_sync(0xffffffffu, !ok)) break;
      ptx::tc_fence_after();
      const uint32_t ah = tmem + lane_base + C::TM_A + b * 2 * C::A_COLS, al = ah + C::A_COLS;
      if (half == 0)
        gather_half<K, B, C::M, C::REP, NW, 0, C::EXTRA>(w, sCb, vrep, ah, al);
      else
        gather_half<K, B, C::M, C::REP, NW, 1, C::EXTRA>(w, sCb, vrep, ah, al);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&a_full[b]);
    }
  } else {
    // ---- epilogue: first the B operand rows n < 64: Pi^T_hi[n][r] = hi(Pi[r][n]), rows
    //      64 + n: lo(Pi[r][n]) (8 consecutive r per 16-byte store, zero past d'); then row
    //      32 (warp % 4) + lane of tile i from accumulator i % 2
    const int t = tid - 64 - kGatherThreads;
    {
      constexpr int kGroups8 = C::KSTEPS * 2;  // groups of 8 K columns (r)
      for (int item = t; item < 64 * kGroups8; item += kEpiThreads) {
        const int n = item & 63, r8 = item >> 6;
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int r = 8 * r8 + q;
          v[q] = r < DP ? __ldg(p.rot + (size_t)r * DP + n) : 0.f;
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          __half h0, l0, h1, l1;
          split_f16(v[2 * q], h0, l0);
          split_f16(v[2 * q + 1], h1, l1);
          hw[q] = h2u(__halves2half2(h0, h1));
          lw[q] = h2u(__halves2half2(l0, l1));
        }
        uint8_t* dh;
        uint8_t* dl;
        if (r8 < 8) {
          dh = sB + ptx::sw128_offset(n, 8 * r8);
          dl = sB + ptx::sw128_offset(64 + n, 8 * r8);
        } else {
          dh = sB + 128 * 128 + ptx::noswz16_offset(n, 8 * (r8 - 8));
          dl = sB + 128 * 128 + ptx::noswz16_offset(64 + n, 8 * (r8 - 8));
        }
        *reinterpret_cast<uint4*>(dh) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(dl) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(b_ready);
      if constexpr (RS) {  // |c|^2 per codeword for the MSE rule's |zbar|^2
        float* sCc = reinterpret_cast<float*>(smem + C::OFF_CC);
        for (int c = t; c < C::N; c += kEpiThreads) {
          float cc = 0.f;
#pragma unroll
          for (int a = 0; a < K; ++a) {
            const float v = __ldg(p.cb + (size_t)c * K + a);
            cc = fmaf(v, v, cc);
          }
          sCc[c] = cc;
        }
        named_sync(2, kEpiThreads);
      }
    }
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    for (int i = 0; i < n_local; ++i) {
      const int s = i % kStages, b = i & 1;
      const int64_t tile = tile_of(i);
      const int rows = rows_of(tile);
      bool ok = wait_ab(&r_full[s], (uint32_t)(i / kStages) & 1u, sAbort);
      if (__any_sync(0xffffffffu, !ok)) break;
      float nu = 0.f;
      if (r < rows)
        nu = f16_bits_to_f32(direct(rows) ? p.norms[tile * kRows + r]
                                          : *reinterpret_cast<const uint16_t*>(
                                                sRing + s * C::STAGE + C::REC + 2 * r));
      if constexpr (RS) {
        // Block Sphere VQ key design 3: y = S nu (Pi^T zbar), S from the stored rho and, for
        // the MSE rule, |zbar|^2 = sum_j |c_j|^2 over the record's codewords
        if (r < rows) {
          uint32_t w[NW];
          if (direct(rows)) read_rec_global<P>(p.codes + (tile * kRows + r) * P, w);
          else read_rec<P>(sRing + s * C::STAGE, (uint32_t)(r * P), w);
          const float* sCc = reinterpret_cast<const float*>(smem + C::OFF_CC);
          float zz = 0.f;
#pragma unroll
          for (int j = 0; j < C::M; ++j) zz += sCc[field<B>(w, j)];
          const float rho = f16_bits_to_f32(p.rho[tile * kRows + r]);
          const float S = p.rule == FQ_RESCALE_MSE ? rho / zz
                          : p.rule == FQ_RESCALE_UNBIASED ? 1.f / rho : 1.f;
          nu *= S;
        }
      }
      ptx::mbar_arrive(&r_empty[s]);
      ok = wait_ab(&d_full[b], (uint32_t)(i >> 1) & 1u, sAbort);
      if (__any_sync(0xffffffffu, !ok)) break;
      ptx::tc_fence_after();
      // the staging tile used two tiles ago must have been read out by its TMA store
      uint8_t* ob = sOut + (q4 * 2 + (i & 1)) * C::OUT_TILE;
      if (lane == 0) ptx::bulk_wait_group_read<1>();
      __syncwarp();
      const uint32_t d = tmem + b * 128 + lane_base;
      const float2 nu2 = make_float2(nu, nu);
      const float2 lo2 = make_float2(kLoScale, kLoScale);
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {  // output columns 32 hc .. 32 hc + 31
        uint32_t h[32], l[32];
        ptx::tmem_ld_cols<0, 32>(d + 32 * hc, h);
        ptx::tmem_ld_cols<0, 32>(d + 64 + 32 * hc, l);
        ptx::tmem_wait_ld();
        if (hc == 1) {
          ptx::tc_fence_before();
          ptx::mbar_arrive(&d_empty[b]);
        }
        float2 v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 hv = make_float2(__uint_as_float(h[2 * e]), __uint_as_float(h[2 * e + 1]));
          const float2 lv = make_float2(__uint_as_float(l[2 * e]), __uint_as_float(l[2 * e + 1]));
          v[e] = __fmul2_rn(nu2, __ffma2_rn(lv, lo2, hv));
        }
        if constexpr (F16) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(ob + ptx::sw128_offset(lane, 8 * (4 * hc + c))) =
                make_uint4(h2u(__float22half2_rn(v[4 * c])), h2u(__float22half2_rn(v[4 * c + 1])),
                           h2u(__float22half2_rn(v[4 * c + 2])),
                           h2u(__float22half2_rn(v[4 * c + 3])));
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c)  // 4 fp32 per 16-byte chunk, one 32-column tile per hc
            *reinterpret_cast<float4*>(ob + hc * 4096 + ptx::sw128_offset(lane, 8 * c)) =
                make_float4(v[2 * c].x, v[2 * c].y, v[2 * c + 1].x, v[2 * c + 1].y);
        }
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      const int64_t row0 = tile * kRows + 32 * q4;
      if (lane == 0 && row0 < p.n) {
        ptx::tma_store_2d(&ymap, ob, 0, (int)row0);
        if constexpr (!F16) ptx::tma_store_2d(&ymap, ob + 4096, 32, (int)row0);
        ptx::bulk_commit_group();
      }
    }
    if (lane == 0) ptx::bulk_wait_group_all();
  }

  // ---- after an abort: let this CTA's own copies and MMAs in flight land (bounded)
  if (*sAbort) {
    if (tid == 0)
      for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
        ptx::mbar_wait(&r_full[t % kStages], (uint32_t)(t / kStages) & 1u);
    if (tid == 32 && mma_done > 0)
      ptx::mbar_wait(&d_full[(mma_done - 1) & 1], (uint32_t)((mma_done - 1) >> 1) & 1u);
  }
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *sAbort) atomicAdd(&g_dec_wait_timeouts, 1u);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// The driver's tensor-map encoder, looked up once.  A function-local static is initialised
// exactly once even when several host threads make their first call together.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_fn() {
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

template <int K, int DP, int B, bool F16, bool RS>
cudaError_t launch_ws(const DecArgs& p, cudaStream_t st) {
  using C = DecCfg<K, DP, B, F16>;
  // output y [n x 64] (fp16 rows of 128 B, fp32 rows of 256 B), stored in boxes of 32 rows and
  // 128 bytes with the 128-byte swizzle
  CUtensorMap map;
  const cuuint64_t dims[2] = {64, (cuuint64_t)p.n};
  const cuuint64_t strides[1] = {F16 ? 128u : 256u};
  const cuuint32_t box[2] = {F16 ? 64u : 32u, 32u};
  const cuuint32_t estr[2] = {1, 1};
  auto fn = tensor_map_fn();
  if (!fn) return cudaErrorNotSupported;
  if (fn(&map, F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p.y,
         dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = decode_ws_kernel<K, DP, B, F16, RS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (p.n + kRows - 1) / kRows;
  const int ctas = (int)(tiles < sms ? tiles : sms);
  kern<<<ctas, kThreads, C::SMEM, st>>>(map, p);
  return cudaGetLastError();
}

template <int K, int DP, bool F16, bool RS>
cudaError_t by_b_rs(int B, const DecArgs& p, cudaStream_t st) {
  switch (B) {
    case 1: return launch_ws<K, DP, 1, F16, RS>(p, st);
    case 2: return launch_ws<K, DP, 2, F16, RS>(p, st);
    case 3: return launch_ws<K, DP, 3, F16, RS>(p, st);
    case 4: return launch_ws<K, DP, 4, F16, RS>(p, st);
    case 5: return launch_ws<K, DP, 5, F16, RS>(p, st);
    case 6: return launch_ws<K, DP, 6, F16, RS>(p, st);
    case 7: return launch_ws<K, DP, 7, F16, RS>(p, st);
    case 8: return launch_ws<K, DP, 8, F16, RS>(p, st);
  }
  return cudaErrorNotSupported;
}

template <int K, int DP, bool F16>
cudaError_t by_b(int B, const DecArgs& p, cudaStream_t st) {
  return p.rho != nullptr ? by_b_rs<K, DP, F16, true>(B, p, st)
                          : by_b_rs<K, DP, F16, false>(B, p, st);
}

}  // namespace

bool decode_supported(fq_dtype yt, const Shape& s, const void* codes, const void* norms,
                      const void* y) {
  (void)yt;
  if (s.d != 64 || s.N > 256 || s.k < 2 || s.k > 4) return false;
  if ((reinterpret_cast<uintptr_t>(y) & 15) || (reinterpret_cast<uintptr_t>(codes) & 15) ||
      (reinterpret_cast<uintptr_t>(norms) & 15))
    return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10;
}

cudaError_t launch_decode(const uint8_t* codes, const uint16_t* norms, int64_t n,
                          const Shape& s, const float* rot, const float* cb, void* y,
                          fq_dtype yt, cudaStream_t st, const uint16_t* rho, int rule) {
  if (n > (int64_t)INT32_MAX)  // tensor-map row coordinates are 32-bit
    return launch_decode_generic(codes, norms, n, s, rot, cb, y, yt, st, Gather{nullptr, 0},
                                 Rescale{rho, rule});
  DecArgs p{n, rot, cb, codes, norms, y, rho, rule};
  const bool f16 = yt == FQ_F16;
  switch (s.k) {
    case 2: return f16 ? by_b<2, 64, true>(s.B, p, st) : by_b<2, 64, false>(s.B, p, st);
    case 3: return f16 ? by_b<3, 66, true>(s.B, p, st) : by_b<3, 66, false>(s.B, p, st);
    case 4: return f16 ? by_b<4, 64, true>(s.B, p, st) : by_b<4, 64, false>(s.B, p, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace sm100
cudaError_t wait_timeouts_decode(bool clear, unsigned* count) {
  return read_wait_counter(sm100::g_dec_wait_timeouts, clear, count);
}

}  // namespace fq
