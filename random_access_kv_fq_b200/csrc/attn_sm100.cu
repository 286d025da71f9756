// sm_100a fused decode attention over FibQuant-compressed keys and values (d = 64, keys with
// k = 2, values with k = 2, 3 or 4, codebooks of at most 256 codewords, 8 or 16 query heads
// per kv head).
//
// One CTA owns one (batch, kv head, context split) and walks it in tiles of 128 tokens, one
// thread per token:
//   records a ring of kStages shared-memory stages is filled ahead of use by bulk async copies
//           (16-byte aligned windows around each tile's key/value records and norms); tiles
//           whose window would leave its buffer are read straight from global memory instead.
//   keys    the thread unpacks its token's key indices and writes the rotated key zhat^K (64
//           coordinates, as fp16 hi and 2^12-scaled lo parts) into tensor memory, where it is
//           the A operand of two tcgen05 chains: Zhi * [q~_hi ; q~_lo]^T and Zlo * q~_hi^T
//           (the group's rotated queries, split the same way), so the scores keep ~22 bits;
//   softmax lazy running maximum in log2 units: the reference maximum of a head moves only
//           when a score passes it by more than tau, so p = 2^(s - m) <= 2^tau, and the value
//           accumulators are rescaled only on those rare tiles;
//   values  weights w = p nu^V / sigma (sigma = a running bound on the value norms, raised on
//           the same rare tiles, so w fits fp16) are split into hi and lo fp16 rows of a
//           K-major B tile (heads x tokens); zhat^V coordinates 0..63 are split into hi (rows
//           0..63) and lo (rows 64..127) of one MN-major A tile (coordinates x tokens); one
//           tcgen05 chain accumulates A * B^T in tensor memory over the whole split, which
//           yields sum_t w zhat^V to ~22 bits once the hi/lo products are combined;
//           coordinates 64 and 65 (k = 3, d' = 66) are accumulated in fp32 on the CUDA cores.
//   output  (max, sum, acc[d'_V]) per head in the partials layout of the generic kernel; the
//           shared combine kernel merges splits and applies Pi_V^T.
// Both the weights and the value codewords need the hi/lo split: fp16 alone for either misses
// the 2e-3 output tolerance when the softmax is diffuse (the output then cancels heavily).
#include <cuda_fp16.h>

#include "fq_device.cuh"
#include "fq_internal.h"
#include "sm100_ptx.cuh"

namespace fq {

__device__ unsigned int g_fq_wait_timeouts = 0;  // CTAs whose bounded waits gave up

namespace attn100 {
namespace {

constexpr int kT = 128;      // tokens per tile
constexpr int kThr = 128;    // one thread per token (and per TMEM lane)
constexpr int kStages = 4;   // record tiles in flight
constexpr float kLoScale = 1.0f / 4096.0f;
constexpr float kTau2 = 11.0f;           // lazy-max slack, log2 units (p <= 2048)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr int round16(int v) { return (v + 15) / 16 * 16; }

template <int G, int KB, int KV, int VB>
struct Cfg {
  static constexpr int NK = 1 << KB, NV = 1 << VB;
  static constexpr int MK = 32;                        // key blocks (k = 2, d' = 64)
  static constexpr int PK = (MK * KB + 7) / 8;
  static constexpr int DPV = KV * ((64 + KV - 1) / KV);
  static constexpr int MV = DPV / KV;
  static constexpr int PV = (MV * VB + 7) / 8;
  static constexpr int N1 = 2 * G;                     // [q~_hi ; q~_lo] rows
  static constexpr int N2 = 16;                        // q~_hi rows (plus q~_lo rows if G = 8)
  static constexpr int NVM = 2 * G;                    // value MMA N: [w_hi ; w_lo]
  // tensor memory columns: key A operand (hi | lo), scores, value accumulators
  static constexpr int C_AH = 0, C_AL = 32, C_D1 = 64, C_D2 = C_D1 + N1, C_DV = C_D2 + N2;
  static constexpr int TMEM_COLS = (C_DV + NVM <= 128) ? 128 : 256;
  static constexpr int MIN_CTAS = (TMEM_COLS == 128) ? 3 : 2;  // CTAs sharing an SM
  // value codeword table: 8 bank-private copies when small (conflict-free 16-byte lookups)
  static constexpr int VREP = (NV <= 64) ? 8 : 1;
  // one ring stage: key records, value records, key norms, value norms (each a 16-byte aligned
  // window of up to 30 bytes more than the tile, plus read-ahead slack for the word reader)
  static constexpr int CAPK = round16(kT * PK) + 48;
  static constexpr int CAPV = round16(kT * PV) + 48;
  static constexpr int CAPN = round16(kT * 2) + 48;
  static constexpr int S_K = 0, S_V = CAPK, S_NK = CAPK + CAPV, S_NV = S_NK + CAPN;
  static constexpr int STAGE = S_NV + CAPN;
  // shared memory (1024-aligned tiles first)
  static constexpr int OFF_AV = 0;                     // [16 token groups][hi, lo atom][8][128 B]
  static constexpr int OFF_P = 32768;                  // [2 token atoms][32 rows][128 B]
  static constexpr int OFF_Q = 40960;                  // [N1 rows x 64] fp16
  static constexpr int OFF_RING = OFF_Q + 4096;
  static constexpr int OFF_KT = OFF_RING + kStages * STAGE;
  static constexpr int OFF_VT = OFF_KT + round16(NK * 8);
  static constexpr int OFF_MISC = OFF_VT + NV * VREP * 16;
  static constexpr int SMEM_USED = OFF_MISC + 1024 + 1024;  // + alignment slack
  // with 256 tensor-memory columns only two CTAs may share an SM
  static constexpr int SMEM = (TMEM_COLS == 256 && SMEM_USED < 80 * 1024) ? 80 * 1024 : SMEM_USED;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(32 * 1024 >= 64 * 65 * 4 + 16 * 64 * 4, "prologue scratch fits the value tile");
};

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

template <int P>
struct Rec {
  static constexpr int NW = (P + 3) / 4 + 1;  // words of a record plus one zero word
};

// The P-byte record starting at shared byte offset o of `base`, as little-endian words with
// zero bytes after the record.  Reads whole words from o & ~3 on (the stage has slack).
template <int P>
__device__ __forceinline__ void smem_record(const uint8_t* base, uint32_t o,
                                            uint32_t (&w)[Rec<P>::NW]) {
  constexpr int NW = Rec<P>::NW;
  if constexpr (P % 16 == 0) {
    if ((o & 15u) == 0) {
#pragma unroll
      for (int q = 0; q < P / 16; ++q) {
        const uint4 v = *reinterpret_cast<const uint4*>(base + o + 16 * q);
        w[4 * q] = v.x;
        w[4 * q + 1] = v.y;
        w[4 * q + 2] = v.z;
        w[4 * q + 3] = v.w;
      }
      w[NW - 1] = 0u;
      return;
    }
  }
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(base + (o & ~3u));
  const uint32_t sh = (o & 3u) * 8u;
  uint32_t raw[NW];
#pragma unroll
  for (int q = 0; q < NW; ++q) raw[q] = wp[q];
#pragma unroll
  for (int q = 0; q < NW - 1; ++q) w[q] = __funnelshift_r(raw[q], raw[q + 1], sh);
  w[NW - 1] = 0u;
  if constexpr (P % 4 != 0) w[(P - 1) / 4] &= (1u << (8 * (P % 4))) - 1u;
}

// The same record read byte by byte from global memory (tiles outside the bulk-copy windows).
template <int P>
__device__ __forceinline__ void gmem_record(const uint8_t* rec, uint32_t (&w)[Rec<P>::NW]) {
#pragma unroll
  for (int q = 0; q < Rec<P>::NW; ++q) w[q] = 0u;
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

// 16-byte aligned window [a0, a1) around the n bytes at g; true when it lies inside [lo, hi).
__device__ __forceinline__ bool window(const uint8_t* g, uint32_t n, const uint8_t* lo,
                                       const uint8_t* hi, uint32_t& off, uint32_t& bytes) {
  const uintptr_t p = reinterpret_cast<uintptr_t>(g);
  const uintptr_t a0 = p & ~uintptr_t(15);
  const uintptr_t a1 = (p + n + 15) & ~uintptr_t(15);
  off = (uint32_t)(p - a0);
  bytes = (uint32_t)(a1 - a0);
  return a0 >= reinterpret_cast<uintptr_t>(lo) && a1 <= reinterpret_cast<uintptr_t>(hi);
}

// Global sources of one tile: key records, value records, key norms, value norms.
struct TileSrc {
  const uint8_t* g[4];
  uint32_t n[4];
};


__device__ __forceinline__ float ex2_approx(float x) {  // 2^x (PTX ex2.approx; 2^-inf = 0)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Output word p of the value tile (zhat^V coordinates 2p and 2p + 1) from the codeword entries
// of the token's blocks: `hi` selects the (hi0 hi1, hi2 hi3) words, else the (lo.., lo..) ones.
template <int KV, int MV, int PW>
__device__ __forceinline__ uint32_t value_word(const uint4 (&e)[MV], bool hi) {
  constexpr int c0 = 2 * PW, c1 = 2 * PW + 1;
  constexpr int j0 = c0 / KV, q0 = c0 % KV, j1 = c1 / KV, q1 = c1 % KV;
  const uint32_t a = hi ? (q0 < 2 ? e[j0].x : e[j0].y) : (q0 < 2 ? e[j0].z : e[j0].w);
  const uint32_t b = hi ? (q1 < 2 ? e[j1].x : e[j1].y) : (q1 < 2 ? e[j1].z : e[j1].w);
  if constexpr (j0 == j1 && (q0 < 2) == (q1 < 2) && (q0 & 1) == 0) return a;  // already a pair
  constexpr uint32_t sel = ((q0 & 1) ? 0x32u : 0x10u) | ((q1 & 1) ? 0x7600u : 0x5400u);
  return __byte_perm(a, b, sel);
}

template <int KV, int MV, int C8>
__device__ __forceinline__ void value_chunk(const uint4 (&e)[MV], bool hi, uint32_t (&o)[4]) {
  o[0] = value_word<KV, MV, 4 * C8 + 0>(e, hi);
  o[1] = value_word<KV, MV, 4 * C8 + 1>(e, hi);
  o[2] = value_word<KV, MV, 4 * C8 + 2>(e, hi);
  o[3] = value_word<KV, MV, 4 * C8 + 3>(e, hi);
}

template <int G, int KB, int KV, int VB, bool RAGGED>
__global__ void __launch_bounds__(kThr, Cfg<G, KB, KV, VB>::MIN_CTAS)
    attn_partial_sm100(AttnArgs a) {
  using C = Cfg<G, KB, KV, VB>;
  constexpr int PK = C::PK, PV = C::PV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sAV = smem + C::OFF_AV;
  uint8_t* sP = smem + C::OFF_P;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sRing = smem + C::OFF_RING;
  uint2* sKT = reinterpret_cast<uint2*>(smem + C::OFF_KT);
  uint4* sVT = reinterpret_cast<uint4*>(smem + C::OFF_VT);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_MISC);  // one per ring stage
  uint64_t* bar_k = full + kStages;                                  // score MMAs done
  uint64_t* bar_v = bar_k + 1;                                       // value MMAs done
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 64);
  int4* sHdr = reinterpret_cast<int4*>(smem + C::OFF_MISC + 128);    // per stage: part offsets
  float* sM = reinterpret_cast<float*>(smem + C::OFF_MISC + 256);  // running max [16], log2
  float* sAlpha = sM + 16;                                          // [16]
  float* sSig = sAlpha + 16;                                        // sigma, old/new ratio
  float* sRed = sSig + 4;                                           // [4 warps][17]
  float* sL = sRed + 4 * 17;                                        // [4 warps][16]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int64_t t_begin = (int64_t)split * a.tokens_per_split;
  const int64_t len_b = attn_seq_len(a, b);  // a split past the sequence's end stays empty
  const int64_t t_end = (t_begin + a.tokens_per_split < len_b) ? t_begin + a.tokens_per_split : len_b;
  const int n_tiles = t_end > t_begin ? (int)((t_end - t_begin + kT - 1) / kT) : 0;
  const size_t kv_base = ((size_t)b * a.Hkv + g) * (size_t)a.T;
  if constexpr (RAGGED) if (n_tiles == 0) {
    // a split past its sequence's end: its empty partials (m = -inf, l = 0, acc = 0) and
    // nothing else (no tensor memory, tables or queries); only with per-sequence lengths, so
    // that the full step's kernel is not touched by the extra path
    constexpr int dpv2 = C::DPV + 2;
    for (int e = threadIdx.x; e < G * dpv2; e += kThr) {
      const int h = e / dpv2, c = e % dpv2;
      a.partials[(((size_t)b * a.Hq + (size_t)g * G + h) * a.splits + split) * dpv2 + c] =
          c == 0 ? -INFINITY : 0.f;
    }
    return;
  }

  // sources of tile i: key records, value records, key norms, value norms
  auto src_of = [&](int i) {
    TileSrc s;
    const int64_t t0 = t_begin + (int64_t)i * kT;
    const uint32_t nt = (uint32_t)((t_end - t0) < kT ? (t_end - t0) : kT);
    const size_t row = kv_base + (size_t)t0;
    s.g[0] = a.k_codes + row * PK;
    s.n[0] = nt * PK;
    s.g[1] = a.v_codes + row * PV;
    s.n[1] = nt * PV;
    s.g[2] = reinterpret_cast<const uint8_t*>(a.k_norms + row);
    s.n[2] = nt * 2;
    s.g[3] = reinterpret_cast<const uint8_t*>(a.v_norms + row);
    s.n[3] = nt * 2;
    return s;
  };
  // thread 0: start the bulk copies of tile i into its ring stage; the stage header records
  // where each part starts in the stage, or -1 where the part is read from global memory
  auto issue_tile = [&](int i) {
    const size_t total = (size_t)a.B * a.Hkv * (size_t)a.T;
    const uint8_t* lo[4] = {a.k_codes, a.v_codes, reinterpret_cast<const uint8_t*>(a.k_norms),
                            reinterpret_cast<const uint8_t*>(a.v_norms)};
    const uint8_t* hi[4] = {a.k_codes + total * PK, a.v_codes + total * PV,
                            reinterpret_cast<const uint8_t*>(a.k_norms + total),
                            reinterpret_cast<const uint8_t*>(a.v_norms + total)};
    constexpr int part_off[4] = {C::S_K, C::S_V, C::S_NK, C::S_NV};
    const int s = i % kStages;
    const TileSrc src = src_of(i);
    uint32_t off[4], bytes[4], tx = 0;
    int hdr[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const bool bulk = window(src.g[p], src.n[p], lo[p], hi[p], off[p], bytes[p]);
      hdr[p] = bulk ? part_off[p] + (int)off[p] : -1;
      if (bulk) tx += bytes[p];
    }
    sHdr[s] = make_int4(hdr[0], hdr[1], hdr[2], hdr[3]);
    ptx::mbar_arrive_expect_tx(&full[s], tx);  // releases the header to the waiting threads
#pragma unroll
    for (int p = 0; p < 4; ++p)
      if (hdr[p] >= 0)
        ptx::bulk_load(sRing + s * C::STAGE + part_off[p], src.g[p] - off[p], bytes[p], &full[s]);
  };

  // ---- set-up ----
  // Single-thread work is spread over three warps so that no warp serialises all of it:
  // thread 0 issues the score MMAs, thread 32 the bulk copies, thread 64 the value MMAs.
  int issued = 0;  // thread 0 during set-up, then thread 32: tiles handed to the ring
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) ptx::mbar_init(&full[s], 1);
    ptx::mbar_init(bar_k, 1);
    ptx::mbar_init(bar_v, 1);
    ptx::fence_mbar_init();
    for (; issued < kStages && issued < n_tiles; ++issued) issue_tile(issued);
    sSig[0] = 0.f;
    sSig[1] = 0.f;
  }
  if (tid < 16) sM[tid] = -INFINITY;
  // Pi_K (rows padded to 65 floats) and the group's queries, staged in the value tile's space
  float* sRot = reinterpret_cast<float*>(sAV);
  float* sQf = sRot + 64 * 65;
  {  // loads issued eight at a time before their stores
#pragma unroll 1
    for (int i0 = 0; i0 < 64 * 64 / kThr; i0 += 8) {
      float v[8];
#pragma unroll
      for (int it = 0; it < 8; ++it) v[it] = __ldg(a.rotK + tid + (i0 + it) * kThr);
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int e = tid + (i0 + it) * kThr;
        sRot[(e >> 6) * 65 + (e & 63)] = v[it];
      }
    }
    const uint16_t* qg = a.q + ((size_t)b * a.Hq + (size_t)g * G) * 64;
    uint16_t qv[G * 64 / kThr];
#pragma unroll
    for (int it = 0; it < G * 64 / kThr; ++it) qv[it] = qg[tid + it * kThr];
#pragma unroll
    for (int it = 0; it < G * 64 / kThr; ++it) sQf[tid + it * kThr] = f16_bits_to_f32(qv[it]);
  }
  // key table: (hi0, hi1 | lo0, lo1) per codeword
  for (int c = tid; c < C::NK; c += kThr) {
    const float c0 = __ldg(a.cbK + 2 * c), c1 = __ldg(a.cbK + 2 * c + 1);
    const __half h0 = __float2half_rn(c0), h1 = __float2half_rn(c1);
    const __half l0 = __float2half_rn((c0 - __half2float(h0)) * 4096.0f);
    const __half l1 = __float2half_rn((c1 - __half2float(h1)) * 4096.0f);
    sKT[c] = make_uint2(h2_bits(__halves2half2(h0, h1)), h2_bits(__halves2half2(l0, l1)));
  }
  // value table: (hi0..3 | lo0..3) per codeword, VREP bank-private copies
  for (int e = tid; e < C::NV * C::VREP; e += kThr) {
    const int c = e / C::VREP;
    __half hv[4], lv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float v = q < KV ? __ldg(a.cbV + (size_t)c * KV + q) : 0.f;
      hv[q] = __float2half_rn(v);
      lv[q] = __float2half_rn((v - __half2float(hv[q])) * 4096.0f);
    }
    sVT[e] = make_uint4(h2_bits(__halves2half2(hv[0], hv[1])), h2_bits(__halves2half2(hv[2], hv[3])),
                        h2_bits(__halves2half2(lv[0], lv[1])), h2_bits(__halves2half2(lv[2], lv[3])));
  }
  // the weight tile starts at zero (rows of absent heads stay zero)
  for (int e = tid; e < 8192 / 16; e += kThr)
    reinterpret_cast<uint4*>(sP)[e] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  // rotated queries q~_h = Pi_K q_h, fp16 hi rows [0, G) and 2^12-scaled lo rows [G, 2G) of
  // the scores' B operand
  for (int e = tid; e < G * 64; e += kThr) {
    const int h = e >> 6, r = e & 63;
    const float* pr = sRot + r * 65;
    const float* qh = sQf + h * 64;
    float acc = 0.f;
#pragma unroll 16
    for (int c = 0; c < 64; ++c) acc = fmaf(pr[c], qh[c], acc);
    const __half hq = __float2half_rn(acc);
    const __half lq = __float2half_rn((acc - __half2float(hq)) * 4096.0f);
    *reinterpret_cast<__half*>(sQ + ptx::sw128_offset(h, r)) = hq;
    *reinterpret_cast<__half*>(sQ + ptx::sw128_offset(G + h, r)) = lq;
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;

  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t idesc1 = ptx::idesc_f16_f32(128, C::N1);
  constexpr uint32_t idesc2 = ptx::idesc_f16_f32(128, C::N2);
  constexpr uint32_t idescv = ptx::idesc_f16_f32_amn(128, C::NVM);
  const uint32_t aQ = ptx::smem_u32(sQ), aV = ptx::smem_u32(sAV), aP = ptx::smem_u32(sP);
  if (tid == 32) issued = kStages < n_tiles ? kStages : n_tiles;  // thread 0 issued these
  const float sc0 = a.scale * kLog2e;
  // this thread's (token tid) addresses in the swizzled tiles, per row / chunk class r = 0..7
  uint32_t p_off[8], av_off[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    p_off[r] = (tid >> 6) * 4096 + r * 128 + (((((tid & 63) >> 3) ^ r) & 7) << 4) + (tid & 7) * 2;
    av_off[r] = (tid >> 3) * 2048 + (tid & 7) * 128 + (((r ^ tid) & 7) << 4);
  }
  const uint32_t vrep = C::VREP > 1 ? (uint32_t)(lane & (C::VREP - 1)) : 0u;

  float lpart[G], x64[G], x65[G], m2[G];  // l, fp32 accumulators of coordinates 64, 65, max
#pragma unroll
  for (int h = 0; h < G; ++h) {
    lpart[h] = x64[h] = x65[h] = 0.f;
    m2[h] = -INFINITY;
  }
  float sig = 0.f, inv_sig = 0.f;
  bool failed = false;
  int last_k = -1, last_v = -1;  // threads 0 / 64: last committed score / value MMA (tile)

  // weights w = p nu / sigma into the B tile: hi in row h, 2^12-scaled lo in row G + h
  auto write_weights = [&](const float (&pv)[G], float wn) {
#pragma unroll
    for (int h = 0; h < G; h += 2) {
      const float w0 = pv[h] * wn, w1 = pv[h + 1] * wn;
      const __half2 whi = __floats2half2_rn(w0, w1);
      const float2 back = __half22float2(whi);
      const __half2 wlo = __floats2half2_rn((w0 - back.x) * 4096.0f, (w1 - back.y) * 4096.0f);
      *reinterpret_cast<__half*>(sP + p_off[h & 7] + (h >> 3) * 1024) = __low2half(whi);
      *reinterpret_cast<__half*>(sP + p_off[(h + 1) & 7] + ((h + 1) >> 3) * 1024) = __high2half(whi);
      *reinterpret_cast<__half*>(sP + p_off[(G + h) & 7] + ((G + h) >> 3) * 1024) = __low2half(wlo);
      *reinterpret_cast<__half*>(sP + p_off[(G + h + 1) & 7] + ((G + h + 1) >> 3) * 1024) =
          __high2half(wlo);
    }
  };

  for (int i = 0; i < n_tiles; ++i) {
    const int s = i % kStages;
    const int64_t t0 = t_begin + (int64_t)i * kT;
    const int nt = (int)((t_end - t0) < kT ? (t_end - t0) : kT);
    const bool valid = tid < nt;
    bool fail = !ptx::mbar_wait(&full[s], (uint32_t)(i / kStages) & 1u);

    // ---- this thread's records and norms (from the ring, or global memory at buffer edges)
    uint32_t wk[Rec<PK>::NW], wv[Rec<PV>::NW];
    float nk = 0.f, nv = 0.f;
    if (valid) {
      const int4 hd = sHdr[s];
      const uint8_t* stage = sRing + s * C::STAGE;
      const size_t row = kv_base + (size_t)t0 + tid;
      if (hd.x >= 0) smem_record<PK>(stage, (uint32_t)hd.x + tid * PK, wk);
      else gmem_record<PK>(a.k_codes + row * PK, wk);
      if (hd.y >= 0) smem_record<PV>(stage, (uint32_t)hd.y + tid * PV, wv);
      else gmem_record<PV>(a.v_codes + row * PV, wv);
      nk = f16_bits_to_f32(hd.z >= 0 ? *reinterpret_cast<const uint16_t*>(stage + hd.z + 2 * tid)
                                     : a.k_norms[row]);
      nv = f16_bits_to_f32(hd.w >= 0 ? *reinterpret_cast<const uint16_t*>(stage + hd.w + 2 * tid)
                                     : a.v_norms[row]);
    } else {
#pragma unroll
      for (int q = 0; q < Rec<PK>::NW; ++q) wk[q] = 0u;
#pragma unroll
      for (int q = 0; q < Rec<PV>::NW; ++q) wv[q] = 0u;
    }

    // ---- keys: zhat^K (hi | lo) into this lane of the tensor-memory A operand
    {
      uint32_t h0[16], h1[16], l0[16], l1[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint2 e0 = sKT[field<KB>(wk, j)];
        const uint2 e1 = sKT[field<KB>(wk, j + 16)];
        h0[j] = e0.x;
        l0[j] = e0.y;
        h1[j] = e1.x;
        l1[j] = e1.y;
      }
      ptx::tmem_st16(tmem + lane_base + C::C_AH, h0);
      ptx::tmem_st16(tmem + lane_base + C::C_AH + 16, h1);
      ptx::tmem_st16(tmem + lane_base + C::C_AL, l0);
      ptx::tmem_st16(tmem + lane_base + C::C_AL + 16, l1);
      ptx::tmem_wait_st();
    }
    ptx::tc_fence_before();
    if (__syncthreads_or(fail)) {  // the stage is consumed and the key operand is in place
      failed = true;
      break;
    }
    if (tid == 0) {
      ptx::tc_fence_after();
      // descriptor of the first K step; later steps add their byte offset / 16 to the start
      // address field (the sums stay inside the 14-bit field for shared-memory addresses)
      const uint64_t dq0 = ptx::sdesc_kmajor_sw128(aQ);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)  // + 32 B per K step
        ptx::umma_f16_ts(tmem + C::C_D1, tmem + C::C_AH + 8 * ks, dq0 + 2 * ks, idesc1,
                         ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ptx::umma_f16_ts(tmem + C::C_D2, tmem + C::C_AL + 8 * ks, dq0 + 2 * ks, idesc2,
                         ks > 0 ? 1u : 0u);
      ptx::umma_commit(bar_k);
      last_k = i;
    } else if (tid == 32 && issued < n_tiles) {
      issue_tile(issued++);
    }

    // ---- values: zhat^V_t (hi rows 0..63, lo rows 64..127) as column t of the MN-major A
    //      tile (the previous value MMA must be done before this tile and the weights are
    //      overwritten)
    if (i > 0) fail |= !ptx::mbar_wait(bar_v, (uint32_t)(i - 1) & 1u);
    float z64 = 0.f, z65 = 0.f;
    {
      uint4 e[C::MV];
#pragma unroll
      for (int j = 0; j < C::MV; ++j) e[j] = sVT[field<VB>(wv, j) * C::VREP + vrep];
      uint32_t o[4];
#define FQ_VCHUNK(C8)                                                                       \
  value_chunk<KV, C::MV, C8>(e, true, o);                                                   \
  *reinterpret_cast<uint4*>(sAV + av_off[C8]) = make_uint4(o[0], o[1], o[2], o[3]);         \
  value_chunk<KV, C::MV, C8>(e, false, o);                                                  \
  *reinterpret_cast<uint4*>(sAV + av_off[C8] + 1024) = make_uint4(o[0], o[1], o[2], o[3]);
      FQ_VCHUNK(0) FQ_VCHUNK(1) FQ_VCHUNK(2) FQ_VCHUNK(3)
      FQ_VCHUNK(4) FQ_VCHUNK(5) FQ_VCHUNK(6) FQ_VCHUNK(7)
#undef FQ_VCHUNK
      if constexpr (C::DPV > 64) {  // coordinates 64 and 65: components 1, 2 of the last block
        const uint4 el = e[C::MV - 1];
        z64 = fmaf(__high2float(*reinterpret_cast<const __half2*>(&el.z)), kLoScale,
                   __high2float(*reinterpret_cast<const __half2*>(&el.x)));
        z65 = fmaf(__low2float(*reinterpret_cast<const __half2*>(&el.w)), kLoScale,
                   __low2float(*reinterpret_cast<const __half2*>(&el.y)));
      }
    }

    // ---- scores of this thread's token (log2 units) and optimistic weights
    fail |= !ptx::mbar_wait(bar_k, (uint32_t)i & 1u);
    ptx::tc_fence_after();
    float s2[G];
    {
      uint32_t d1[C::N1], d2[16];
      ptx::tmem_ld_cols<0, C::N1>(tmem + lane_base + C::C_D1, d1);
      ptx::tmem_ld_cols<0, 16>(tmem + lane_base + C::C_D2, d2);
      ptx::tmem_wait_ld();
      const float sc = nk * sc0;
#pragma unroll
      for (int h = 0; h < G; ++h)
        s2[h] = valid ? fmaf(__uint_as_float(d1[G + h]) + __uint_as_float(d2[h]), kLoScale,
                             __uint_as_float(d1[h])) * sc
                      : -INFINITY;
    }
    bool over = nv > sig;
    float pv[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      over |= s2[h] > m2[h] + kTau2;
      pv[h] = ex2_approx(s2[h] - m2[h]);
    }
    write_weights(pv, nv * inv_sig);
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    if (__syncthreads_or(over || fail)) {
      // rare tile: a score passed its head's maximum by more than tau, or a value norm passed
      // sigma (or a wait timed out)
      if (__syncthreads_or(fail)) {
        failed = true;
        break;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float v = warp_max(s2[h]);
        if (lane == 0) sRed[warp * 17 + h] = v;
      }
      {
        const float v = warp_max(nv);
        if (lane == 0) sRed[warp * 17 + 16] = v;
      }
      __syncthreads();
      if (tid < G) {
        const float mo = sM[tid];
        const float tm = fmaxf(fmaxf(sRed[tid], sRed[17 + tid]), fmaxf(sRed[34 + tid], sRed[51 + tid]));
        const float mn = fmaxf(mo, tm);
        sAlpha[tid] = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
        sM[tid] = mn;
      }
      if (tid == 32) {
        const float so = sSig[0];
        const float nm = fmaxf(fmaxf(sRed[16], sRed[33]), fmaxf(sRed[50], sRed[67]));
        const float sn = nm > so ? 2.f * nm : so;
        sSig[0] = sn;
        sSig[1] = sn > 0.f ? so / sn : 0.f;
      }
      __syncthreads();
      sig = sSig[0];
      inv_sig = sig > 0.f ? 1.f / sig : 0.f;
      const float ratio = sSig[1];
      float beta[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m2[h] = sM[h];
        const float al = sAlpha[h];
        lpart[h] *= al;
        beta[h] = al * ratio;
        x64[h] *= beta[h];
        x65[h] *= beta[h];
        pv[h] = ex2_approx(s2[h] - m2[h]);
      }
      if (i > 0) {  // this lane's value accumulators (the previous value MMA is done)
        uint32_t v[C::NVM];
        ptx::tmem_ld_cols<0, C::NVM>(tmem + lane_base + C::C_DV, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < G; ++h) {
          v[h] = __float_as_uint(__uint_as_float(v[h]) * beta[h]);
          v[G + h] = __float_as_uint(__uint_as_float(v[G + h]) * beta[h]);
        }
#pragma unroll
        for (int c = 0; c < C::NVM; c += 16) {
          uint32_t r16[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) r16[q] = v[c + q];
          ptx::tmem_st16(tmem + lane_base + C::C_DV + c, r16);
        }
        ptx::tmem_wait_st();
      }
      write_weights(pv, nv * inv_sig);
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
    }
    {
      const float wn = nv * inv_sig;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        lpart[h] += pv[h];
        if constexpr (C::DPV > 64) {
          x64[h] = fmaf(pv[h] * wn, z64, x64[h]);
          x65[h] = fmaf(pv[h] * wn, z65, x65[h]);
        }
      }
    }
    if (tid == 64) {
      ptx::tc_fence_after();
      const uint64_t dv0 = ptx::sdesc_mnmajor_sw128(aV, 1024, 2048);
      const uint64_t dp0 = ptx::sdesc_kmajor_sw128(aP);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)  // A: + 4096 B per step; B: + 4096 B per 4 steps, + 32 B
        ptx::umma_f16(tmem + C::C_DV, dv0 + 256 * ks, dp0 + 256 * (ks >> 2) + 2 * (ks & 3),
                      idescv, (i > 0 || ks > 0) ? 1u : 0u);
      ptx::umma_commit(bar_v);
      last_v = i;
    }
  }

  // ---- after a timed-out wait: let this CTA's own copies and MMAs in flight land (bounded)
  if (failed) {
    if (tid == 32)
      for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
        ptx::mbar_wait(&full[t % kStages], (uint32_t)(t / kStages) & 1u);
    if (tid == 0 && last_k >= 0) ptx::mbar_wait(bar_k, (uint32_t)last_k & 1u);
    if (tid == 64 && last_v >= 0) ptx::mbar_wait(bar_v, (uint32_t)last_v & 1u);
  }
  __syncwarp();

  // ---- partials of this split: (m, l, acc[d'_V]) per head, acc scaled back by sigma
  if (!failed && n_tiles > 0 && !ptx::mbar_wait(bar_v, (uint32_t)(n_tiles - 1) & 1u))
    failed = true;
  ptx::tc_fence_after();
  __syncthreads();
  float* sComb = reinterpret_cast<float*>(sAV);  // [64 coords][16 heads]: lo-row products
  float* sX = sComb + 64 * 16;                   // [4 warps][2][16]: coordinates 64, 65
  uint32_t dv[C::NVM];
  ptx::tmem_ld_cols<0, C::NVM>(tmem + lane_base + C::C_DV, dv);  // [w_hi heads | w_lo heads]
  ptx::tmem_wait_ld();
  if (n_tiles == 0) {  // an empty split (past its sequence's end): m = -inf, l = 0, acc = 0
#pragma unroll
    for (int q = 0; q < C::NVM; ++q) dv[q] = 0u;
  }
  if (tid >= 64) {  // zhat_lo rows: only the w_hi product matters at this precision
#pragma unroll
    for (int h = 0; h < G; ++h) sComb[(tid - 64) * 16 + h] = __uint_as_float(dv[h]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float l = warp_sum(lpart[h]);
    float a64 = 0.f, a65 = 0.f;
    if constexpr (C::DPV > 64) {
      a64 = warp_sum(x64[h]);
      a65 = warp_sum(x65[h]);
    }
    if (lane == 0) {
      sL[warp * 16 + h] = l;
      sX[(warp * 2 + 0) * 16 + h] = a64;
      sX[(warp * 2 + 1) * 16 + h] = a65;
    }
  }
  __syncthreads();
  const int dpv2 = C::DPV + 2;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const size_t base = (((size_t)b * a.Hq + (size_t)g * G + h) * a.splits + split) * dpv2;
    if (tid < 64) {
      const float v = __uint_as_float(dv[h]) +
                      kLoScale * (__uint_as_float(dv[G + h]) + sComb[tid * 16 + h]);
      a.partials[base + 2 + tid] = v * sig;
    }
    if constexpr (C::DPV > 64) {
      if (tid == 64 || tid == 65) {
        const int q = tid - 64;
        float v = 0.f;
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) v += sX[(ww * 2 + q) * 16 + h];
        a.partials[base + 2 + tid] = v * sig;
      }
    }
    if (tid == 0) {
      a.partials[base] = m2[h] * kLn2;  // natural-log units for the combine kernel
      a.partials[base + 1] = (sL[h] + sL[16 + h]) + (sL[32 + h] + sL[48 + h]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && failed) atomicAdd(&g_fq_wait_timeouts, 1u);
  if (warp == 0) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int G, int KB, int KV, int VB>
cudaError_t launch(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<G, KB, KV, VB>;
  // the empty-split shortcut for per-sequence lengths is built for 8 query heads per kv head
  // (the attention workloads' ratio); other ratios run the full kernel, which handles empty
  // splits too
  auto kern = attn_partial_sm100<G, KB, KV, VB, false>;
  if constexpr (G == 8)
    if (a.lengths != nullptr) kern = attn_partial_sm100<G, KB, KV, VB, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.splits, a.Hkv, a.B), kThr, C::SMEM, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_combine(a, st);
}

template <int G, int KB, int KV>
cudaError_t by_vb(const AttnArgs& a, cudaStream_t st) {
  switch (a.vs.B) {
    case 2: return launch<G, KB, KV, 2>(a, st);
    case 3: return launch<G, KB, KV, 3>(a, st);
    case 4: return launch<G, KB, KV, 4>(a, st);
    case 6: return launch<G, KB, KV, 6>(a, st);
    case 8: return launch<G, KB, KV, 8>(a, st);
  }
  return cudaErrorNotSupported;
}

template <int G, int KB>
cudaError_t by_kv(const AttnArgs& a, cudaStream_t st) {
  switch (a.vs.k) {
    case 2: return by_vb<G, KB, 2>(a, st);
    case 3: return by_vb<G, KB, 3>(a, st);
    case 4: return by_vb<G, KB, 4>(a, st);
  }
  return cudaErrorNotSupported;
}

template <int G>
cudaError_t by_kb(const AttnArgs& a, cudaStream_t st) {
  switch (a.ks.B) {
    case 2: return by_kv<G, 2>(a, st);
    case 3: return by_kv<G, 3>(a, st);
    case 4: return by_kv<G, 4>(a, st);
    case 6: return by_kv<G, 6>(a, st);
    case 8: return by_kv<G, 8>(a, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace

bool supported(const AttnArgs& a) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return false;
  const int G = a.Hq / a.Hkv;
  if (a.d != 64 || a.ks.k != 2 || a.vs.k < 2 || a.vs.k > 4) return false;
  if (a.ks.N > 256 || a.vs.N > 256) return false;
  if (G != 8 && G != 16) return false;
  if (a.tokens_per_split % kT != 0) return false;
  const int kb = a.ks.B, vb = a.vs.B;
  auto ok_b = [](int bb) { return bb == 2 || bb == 3 || bb == 4 || bb == 6 || bb == 8; };
  return ok_b(kb) && ok_b(vb);
}

cudaError_t launch(const AttnArgs& a, cudaStream_t st) {
  const int G = a.Hq / a.Hkv;
  if (G == 8) return by_kb<8>(a, st);
  return by_kb<16>(a, st);
}

}  // namespace attn100
cudaError_t wait_timeouts_attn(bool clear, unsigned* count) {
  return read_wait_counter(g_fq_wait_timeouts, clear, count);
}

}  // namespace fq
