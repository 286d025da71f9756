// sm_100a fused decode attention over FibQuant-compressed keys and values (d = 64, keys with
// k = 2, values with k = 2, 3 or 4, codebooks of at most 256 codewords, 8 or 16 query heads
// per kv head).
//
// One CTA owns one (batch, kv head, context split) and walks it in tiles of 128 tokens:
//   keys    each thread unpacks its token's key indices and writes the rotated key zhat^K
//           (64 coordinates) into two UMMA A tiles as fp16 hi and 2^12-scaled lo parts; one
//           tcgen05 chain multiplies Zhi by [q~_hi ; q~_lo] (the group's rotated queries, also
//           split) and a second Zlo by q~_hi, so the scores keep ~22 bits;
//   softmax lazy running maximum: the reference maximum of a head moves only when a score
//           passes it by more than tau = 8, so p = exp(s - m) <= e^8 and the accumulators are
//           rescaled only on those rare tiles;
//   values  weights w = p nu^V / sigma (sigma = the largest value norm of the split, so w fits
//           fp16) are split into hi and lo fp16 rows of a K-major B tile (heads x tokens); the
//           token's zhat^V coordinates 0..63 are split into hi (rows 0..63) and lo (rows
//           64..127) of one MN-major A tile (coordinates x tokens); one tcgen05 chain
//           accumulates A * B^T in tensor memory over the whole split, which yields
//           sum_t w zhat^V to ~22 bits once the hi/lo products are combined; coordinates 64
//           and 65 (k = 3, d' = 66) are accumulated in fp32 on the CUDA cores.
//   output  (max, sum, acc[d'_V]) per head in the partials layout of the generic kernel; the
//           shared combine kernel merges splits and applies Pi_V^T.
// Both the weights and the value codewords need the hi/lo split: fp16 alone for either misses
// the 2e-3 output tolerance when the softmax is diffuse (the output then cancels heavily).
#include <cuda_fp16.h>

#include "fq_device.cuh"
#include "fq_internal.h"
#include "sm100_ptx.cuh"

namespace fq {

extern __device__ unsigned int g_fq_wait_timeouts;

namespace attn100 {
namespace {

constexpr int kT = 128;      // tokens per tile
constexpr int kThr = 128;    // one thread per token (and per TMEM lane)
constexpr float kLoScale = 1.0f / 4096.0f;
constexpr float kTau = 8.0f;

template <int G, int KB, int KV, int VB>
struct Cfg {
  static constexpr int MK = 32;                        // key blocks (k = 2, d' = 64)
  static constexpr int PK = (MK * KB + 7) / 8;
  static constexpr int DPV = KV * ((64 + KV - 1) / KV);
  static constexpr int MV = DPV / KV;
  static constexpr int PV = (MV * VB + 7) / 8;
  static constexpr int N1 = ((2 * G + 15) / 16) * 16;  // [q~_hi ; q~_lo] rows
  static constexpr int N2 = ((G + 15) / 16) * 16;
  // tensor memory columns: scores (hi | lo), scores (lo chain), values [w_hi heads | w_lo heads]
  static constexpr int C_D1 = 0, C_D2 = 32, C_DV = 64, TMEM_COLS = 128;
  // shared memory (1024-aligned tiles first)
  static constexpr int OFF_AH = 0;                     // [128 tokens x 64] fp16, 128B swizzle
  static constexpr int OFF_AL = 16384;
  static constexpr int OFF_AV = 32768;                 // [16 token groups][hi, lo atom][8][128 B]
  static constexpr int OFF_P = 65536;                  // [2 token atoms][32 rows][128 B]
  static constexpr int OFF_Q = 73728;                  // [N1 rows x 64] fp16
  static constexpr int OFF_RK = OFF_Q + N1 * 128;      // key records of the tile
  static constexpr int OFF_RV = OFF_RK + ((kT * PK + 15) / 16) * 16;
  static constexpr int OFF_KT = OFF_RV + ((kT * PV + 15) / 16) * 16;  // key codeword table
  static constexpr int OFF_VT = OFF_KT + 256 * 8;      // value codeword table (hi | lo)
  static constexpr int OFF_RED = OFF_VT + 256 * 16;    // scores of one tile [G][128] fp32
  static constexpr int OFF_MISC = OFF_RED + G * kT * 4;
  static constexpr int SMEM = OFF_MISC + 512 + 1024;
};

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }
__device__ __forceinline__ __half2 bits_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }

// Copy n bytes of records from global to shared memory (16-byte vectors when both ends allow).
__device__ __forceinline__ void stage_bytes(uint8_t* dst, const uint8_t* src, int n, int tid) {
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    for (int q = tid; q < n / 16; q += kThr)
      reinterpret_cast<uint4*>(dst)[q] = __ldg(reinterpret_cast<const uint4*>(src) + q);
    for (int q = (n / 16) * 16 + tid; q < n; q += kThr) dst[q] = src[q];
  } else {
    for (int q = tid; q < n; q += kThr) dst[q] = src[q];
  }
}

// Reads the P-byte record at rec into little-endian words.
template <int P>
__device__ __forceinline__ void read_record(const uint8_t* rec, uint32_t (&w)[(P + 3) / 4 + 1]) {
#pragma unroll
  for (int q = 0; q < (P + 3) / 4 + 1; ++q) w[q] = 0u;
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

template <int G, int KB, int KV, int VB>
__global__ void __launch_bounds__(kThr) attn_partial_sm100(AttnArgs a) {
  using C = Cfg<G, KB, KV, VB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sAH = smem + C::OFF_AH;
  uint8_t* sAL = smem + C::OFF_AL;
  uint8_t* sAV = smem + C::OFF_AV;
  uint8_t* sP = smem + C::OFF_P;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sRK = smem + C::OFF_RK;
  uint8_t* sRV = smem + C::OFF_RV;
  uint2* sKT = reinterpret_cast<uint2*>(smem + C::OFF_KT);
  uint4* sVT = reinterpret_cast<uint4*>(smem + C::OFF_VT);
  float* sRed = reinterpret_cast<float*>(smem + C::OFF_RED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_MISC);  // bar_k, bar_v
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 16);
  int* sFlag = reinterpret_cast<int*>(smem + C::OFF_MISC + 20);
  float* sSigma = reinterpret_cast<float*>(smem + C::OFF_MISC + 24);
  float* sM = reinterpret_cast<float*>(smem + C::OFF_MISC + 32);         // running max [G]
  float* sAlpha = sM + 16;                                               // rescale [G]
  float* sTmax = sAlpha + 16;                                            // tile max [G]
  float* sL = sTmax + 16;                                                // [4 warps][16]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int64_t t_begin = (int64_t)split * a.tokens_per_split;
  const int64_t t_end = (t_begin + a.tokens_per_split < a.T) ? t_begin + a.tokens_per_split : a.T;
  const size_t kv_base = ((size_t)b * a.Hkv + g) * (size_t)a.T;

  if (warp == 0) {
    ptx::tmem_alloc(sTmem, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(&bars[0], 1);
    ptx::mbar_init(&bars[1], 1);
    sFlag[0] = 0;
    ptx::fence_mbar_init();
  }
  if (tid < 16) sM[tid] = -INFINITY;
  // sigma = largest value norm of the split (keeps the weights w = p nu / sigma within fp16)
  {
    float mx = 0.f;
    for (int64_t t = t_begin + tid; t < t_end; t += kThr)
      mx = fmaxf(mx, fabsf(f16_bits_to_f32(a.v_norms[kv_base + t])));
    mx = warp_max(mx);
    if (lane == 0) sL[warp] = mx;
  }
  // rotated queries q~_h = Pi_K q_h, split into fp16 hi rows [0, G) and 2^12-scaled lo rows
  // [G, 2G) of the scores' B operand
  for (int e = tid; e < G * 64; e += kThr) {
    const int h = e >> 6, r = e & 63;
    const uint16_t* qh = a.q + ((size_t)b * a.Hq + (size_t)g * G + h) * 64;
    const float* pr = a.rotK + (size_t)r * 64;
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < 64; ++c) acc = fmaf(__ldg(pr + c), f16_bits_to_f32(qh[c]), acc);
    const __half hi = __float2half_rn(acc);
    const __half lo = __float2half_rn((acc - __half2float(hi)) * 4096.0f);
    *reinterpret_cast<__half*>(sQ + ptx::sw128_offset(h, r)) = hi;
    *reinterpret_cast<__half*>(sQ + ptx::sw128_offset(G + h, r)) = lo;
  }
  for (int e = tid; e < (C::N1 - 2 * G) * 64; e += kThr)
    *reinterpret_cast<__half*>(sQ + ptx::sw128_offset(2 * G + (e >> 6), e & 63)) =
        __float2half_rn(0.f);
  // key table: (hi0, hi1 | lo0, lo1) per codeword; value table: (hi0..3 | lo0..3)
  for (int c = tid; c < a.ks.N; c += kThr) {
    const float c0 = __ldg(a.cbK + 2 * c), c1 = __ldg(a.cbK + 2 * c + 1);
    const __half h0 = __float2half_rn(c0), h1 = __float2half_rn(c1);
    const __half l0 = __float2half_rn((c0 - __half2float(h0)) * 4096.0f);
    const __half l1 = __float2half_rn((c1 - __half2float(h1)) * 4096.0f);
    sKT[c] = make_uint2(h2_bits(__halves2half2(h0, h1)), h2_bits(__halves2half2(l0, l1)));
  }
  for (int c = tid; c < a.vs.N; c += kThr) {
    __half hv[4], lv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float v = q < KV ? __ldg(a.cbV + (size_t)c * KV + q) : 0.f;
      hv[q] = __float2half_rn(v);
      lv[q] = __float2half_rn((v - __half2float(hv[q])) * 4096.0f);
    }
    sVT[c] = make_uint4(h2_bits(__halves2half2(hv[0], hv[1])), h2_bits(__halves2half2(hv[2], hv[3])),
                        h2_bits(__halves2half2(lv[0], lv[1])), h2_bits(__halves2half2(lv[2], lv[3])));
  }
  // the weight tile starts at zero (rows of absent heads stay zero)
  for (int e = tid; e < 8192 / 16; e += kThr)
    reinterpret_cast<uint4*>(sP)[e] = make_uint4(0u, 0u, 0u, 0u);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (tid == 0) {
    const float sg = fmaxf(fmaxf(sL[0], sL[1]), fmaxf(sL[2], sL[3]));
    sSigma[0] = sg > 0.f ? sg : 1.f;
  }
  const uint32_t tmem = *sTmem;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t idesc1 = ptx::idesc_f16_f32(128, C::N1);
  constexpr uint32_t idesc2 = ptx::idesc_f16_f32(128, C::N2);
  constexpr uint32_t idescv = ptx::idesc_f16_f32_amn(128, 32);
  const uint32_t aH = ptx::smem_u32(sAH), aL = ptx::smem_u32(sAL), aQ = ptx::smem_u32(sQ);
  const uint32_t aV = ptx::smem_u32(sAV), aP = ptx::smem_u32(sP);
  __syncthreads();
  const float inv_sigma = 1.f / sSigma[0];

  float lpart[G], x64[G], x65[G];  // l and the fp32 accumulators of coordinates 64, 65
#pragma unroll
  for (int h = 0; h < G; ++h) lpart[h] = x64[h] = x65[h] = 0.f;

  int i = 0;
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kT, ++i) {
    const int nt = (t_end - t0 < kT) ? (int)(t_end - t0) : kT;
    const bool valid = tid < nt;
    // records of the tile
    stage_bytes(sRK, a.k_codes + (kv_base + t0) * C::PK, nt * C::PK, tid);
    stage_bytes(sRV, a.v_codes + (kv_base + t0) * C::PV, nt * C::PV, tid);
    const float nk = valid ? f16_bits_to_f32(a.k_norms[kv_base + t0 + tid]) : 0.f;
    const float nv = valid ? f16_bits_to_f32(a.v_norms[kv_base + t0 + tid]) : 0.f;
    __syncthreads();

    // ---- keys: zhat^K rows (hi / lo) into the two A tiles
    {
      uint32_t w[(C::PK + 3) / 4 + 1];
      read_record<C::PK>(sRK + tid * C::PK, w);
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = blocks 4c..4c+3
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint2 e = valid ? sKT[field<KB>(w, 4 * c + q)] : make_uint2(0u, 0u);
          hw[q] = e.x;
          lw[q] = e.y;
        }
        *reinterpret_cast<uint4*>(sAH + ptx::sw128_offset(tid, 8 * c)) =
            make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(sAL + ptx::sw128_offset(tid, 8 * c)) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ptx::umma_f16(tmem + C::C_D1, ptx::sdesc_kmajor_sw128(aH + ks * 32),
                      ptx::sdesc_kmajor_sw128(aQ + ks * 32), idesc1, ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ptx::umma_f16(tmem + C::C_D2, ptx::sdesc_kmajor_sw128(aL + ks * 32),
                      ptx::sdesc_kmajor_sw128(aQ + ks * 32), idesc2, ks > 0 ? 1u : 0u);
      ptx::umma_commit(&bars[0]);
    }

    // ---- values: zhat^V_t (hi rows 0..63, lo rows 64..127) as column t of the MN-major A
    //      tile; the previous value MMA must be done before the tile is overwritten
    if (i > 0 && !ptx::mbar_wait(&bars[1], (i - 1) & 1)) sFlag[0] = 1;
    float z64 = 0.f, z65 = 0.f;
    {
      uint32_t w[(C::PV + 3) / 4 + 1];
      read_record<C::PV>(sRV + tid * C::PV, w);
      const int grp = tid >> 3, row = tid & 7;
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // coordinates 8c..8c+7
        uint32_t hw[4] = {0u, 0u, 0u, 0u}, lw[4] = {0u, 0u, 0u, 0u};
        const int j0 = (8 * c) / KV;
        const int j1 = (8 * c + 7) / KV;
#pragma unroll
        for (int j = j0; j <= j1; ++j) {
          const uint4 e = valid ? sVT[field<VB>(w, j)] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int q = 0; q < KV; ++q) {
            const int hp = KV * j + q;
            if (hp >= 8 * c && hp < 8 * c + 8) {
              const int pos = hp - 8 * c;
              const uint32_t hh = ((q < 2 ? e.x : e.y) >> (16 * (q & 1))) & 0xFFFFu;
              const uint32_t ll = ((q < 2 ? e.z : e.w) >> (16 * (q & 1))) & 0xFFFFu;
              hw[pos >> 1] |= hh << (16 * (pos & 1));
              lw[pos >> 1] |= ll << (16 * (pos & 1));
            }
          }
        }
        const int sw = ((c ^ row) & 7) << 4;
        *reinterpret_cast<uint4*>(sAV + (grp * 2 + 0) * 1024 + row * 128 + sw) =
            make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(sAV + (grp * 2 + 1) * 1024 + row * 128 + sw) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      if constexpr (C::DPV > 64) {  // coordinates 64, 65 of the last block, in fp32
        const uint4 e = valid ? sVT[field<VB>(w, C::MV - 1)] : make_uint4(0u, 0u, 0u, 0u);
        const int q0 = 64 - KV * (C::MV - 1);  // position of coordinate 64 inside the block
        auto coord = [&](int q) {
          const uint32_t hh = ((q < 2 ? e.x : e.y) >> (16 * (q & 1))) & 0xFFFFu;
          const uint32_t ll = ((q < 2 ? e.z : e.w) >> (16 * (q & 1))) & 0xFFFFu;
          return fmaf(__half2float(__ushort_as_half((unsigned short)ll)), kLoScale,
                      __half2float(__ushort_as_half((unsigned short)hh)));
        };
        z64 = coord(q0);
        z65 = coord(q0 + 1);
      }
    }

    // ---- scores for this thread's token
    if (!ptx::mbar_wait(&bars[0], i & 1)) sFlag[0] = 1;
    ptx::tc_fence_after();
    float s[G];
    {
      uint32_t d1[16], d2[16], d1b[16];
      ptx::tmem_ld16(tmem + lane_base + C::C_D1, d1);
      ptx::tmem_ld16(tmem + lane_base + C::C_D2, d2);
      if constexpr (G > 8) ptx::tmem_ld16(tmem + lane_base + C::C_D1 + 16, d1b);
      ptx::tmem_wait_ld();
      const float sc = nk * a.scale;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float hi = __uint_as_float(d1[h]);
        const int lo_col = G + h;
        const float lo = __uint_as_float(lo_col < 16 ? d1[lo_col] : d1b[lo_col - 16]);
        const float lo2 = __uint_as_float(d2[h]);
        s[h] = valid ? fmaf(lo + lo2, kLoScale, hi) * sc : -INFINITY;
      }
    }
    // lazy running maximum: recompute it only when some score passes it by more than tau
    bool over = false;
#pragma unroll
    for (int h = 0; h < G; ++h) over |= s[h] > sM[h] + kTau;
    if (__syncthreads_or(over)) {
#pragma unroll
      for (int h = 0; h < G; ++h) sRed[h * kT + tid] = s[h];
      __syncthreads();
      for (int h = warp; h < G; h += 4) {
        float m = fmaxf(fmaxf(sRed[h * kT + lane], sRed[h * kT + lane + 32]),
                        fmaxf(sRed[h * kT + lane + 64], sRed[h * kT + lane + 96]));
        m = warp_max(m);
        if (lane == 0) sTmax[h] = m;
      }
      __syncthreads();
      if (tid < G) {
        const float mo = sM[tid], mn = fmaxf(mo, sTmax[tid]);
        sAlpha[tid] = (mo == -INFINITY) ? 0.f : __expf(mo - mn);
        sM[tid] = mn;
      }
      __syncthreads();
#pragma unroll
      for (int h = 0; h < G; ++h) {
        lpart[h] *= sAlpha[h];
        x64[h] *= sAlpha[h];
        x65[h] *= sAlpha[h];
      }
      if (i > 0) {  // rescale this lane's value accumulators (the previous MMA is done)
        uint32_t v[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          ptx::tmem_ld16(tmem + lane_base + C::C_DV + 16 * half, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 16; ++h)
            if (h < G) v[h] = __float_as_uint(__uint_as_float(v[h]) * sAlpha[h]);
          ptx::tmem_st16(tmem + lane_base + C::C_DV + 16 * half, v);
        }
        ptx::tmem_wait_st();
      }
    }
    // weights w = p nu / sigma, hi in row h and 2^12-scaled lo in row 16 + h of the B tile
    const float wn = valid ? nv * inv_sigma : 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float pv = valid ? __expf(s[h] - sM[h]) : 0.f;
      lpart[h] += pv;
      const float wv = pv * wn;
      x64[h] = fmaf(wv, z64, x64[h]);
      x65[h] = fmaf(wv, z65, x65[h]);
      const __half whi = __float2half_rn(wv);
      const __half wlo = __float2half_rn((wv - __half2float(whi)) * 4096.0f);
      const int t = tid;
      const int base = (t >> 6) * 4096 + ((((t & 63) >> 3) ^ (h & 7)) << 4) + (t & 7) * 2 + (h & 7) * 128;
      *reinterpret_cast<__half*>(sP + base + (h >> 3) * 1024) = whi;
      *reinterpret_cast<__half*>(sP + base + (2 + (h >> 3)) * 1024) = wlo;
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        ptx::umma_f16(tmem + C::C_DV,
                      ptx::sdesc_mnmajor_sw128(aV + ks * 2 * 2048, 1024, 2048),
                      ptx::sdesc_kmajor_sw128(aP + (ks >> 2) * 4096 + (ks & 3) * 32), idescv,
                      (i > 0 || ks > 0) ? 1u : 0u);
      ptx::umma_commit(&bars[1]);
    }
    if (*(volatile int*)sFlag) break;
  }

  // ---- partials of this split: (m, l, acc[d'_V]) per head, acc scaled back by sigma
  if (i > 0 && !ptx::mbar_wait(&bars[1], (i - 1) & 1)) sFlag[0] = 1;
  ptx::tc_fence_after();
  const float sigma = sSigma[0];
  float* sComb = reinterpret_cast<float*>(sAV);  // [64 coords][16 heads]: lo-row products
  float* sX = sComb + 64 * 16;                   // [4 warps][2][16]: coordinates 64, 65
  uint32_t vh[16], vl[16];
  ptx::tmem_ld16(tmem + lane_base + C::C_DV, vh);       // heads, w_hi
  ptx::tmem_ld16(tmem + lane_base + C::C_DV + 16, vl);  // heads, w_lo
  ptx::tmem_wait_ld();
  if (tid >= 64) {  // zhat_lo rows: only the w_hi product matters at this precision
#pragma unroll
    for (int h = 0; h < 16; ++h) sComb[(tid - 64) * 16 + h] = __uint_as_float(vh[h]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float l = warp_sum(lpart[h]);
    const float a64 = warp_sum(x64[h]);
    const float a65 = warp_sum(x65[h]);
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
      const float v = __uint_as_float(vh[h]) +
                      kLoScale * (__uint_as_float(vl[h]) + sComb[tid * 16 + h]);
      a.partials[base + 2 + tid] = v * sigma;
    }
    if constexpr (C::DPV > 64) {
      if (tid == 64 || tid == 65) {
        const int q = tid - 64;
        float v = 0.f;
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) v += sX[(ww * 2 + q) * 16 + h];
        a.partials[base + 2 + tid] = v * sigma;
      }
    }
    if (tid == 0) {
      a.partials[base] = sM[h];
      a.partials[base + 1] = sL[h] + sL[16 + h] + sL[32 + h] + sL[48 + h];
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && sFlag[0]) atomicAdd(&g_fq_wait_timeouts, 1u);
  if (warp == 0) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int G, int KB, int KV, int VB>
cudaError_t launch(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<G, KB, KV, VB>;
  auto kern = attn_partial_sm100<G, KB, KV, VB>;
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
}  // namespace fq
