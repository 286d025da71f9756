// sm_100a fq_encode for high-dimensional blocks: half-vector (k = d/2) and full-vector (k = d)
// codes with d = 64 or 128, k = 32 or 64, N = 256 .. 65536 codewords.
//
// FibQuant summary sec. 4.2: the extreme-compression end of the memory-fidelity frontier uses
// blocks of half or all of the vector (34.1x at k = d/2, N = 2^15 on d = 64).  There the nearest-
// codeword search is a true GEMM: every block z (k coordinates) against all N codewords,
//   s(n) = |c_n|^2 - 2 z.c_n             (= |z - c_n|^2 - |z|^2),
// which runs on the tensor cores with both sides split into an fp16 head and an fp16 residual
// so that the approximate score keeps ~22 bits:
//   A row (block z)      [ z_hi(k) | z_hi(k) | z_lo(k) | 1     | 1     | 0 ... ]
//   B row (codeword n)   [ a_hi(k) | a_lo(k) | a_hi(k) | cc_hi | cc_lo | 0 ... ]
// with a = -2 c_n and cc = |c_n|^2 (the dropped z_lo . a_lo term is ~2^-22 of a score).  The B
// rows are prepared once on the host (fq_build_search_index, kind FQ_INDEX_TENSOR) in the
// tensor cores' shared-memory layout, so chunks of codewords stream into shared memory with one
// bulk copy each and no conversion on the device.
//
// Per block the scan keeps the two 8-codeword groups with the lowest approximate minima; both
// are then re-scored with exact fp32 squared distances (lower distance, then lower index, as
// the oracle).  If the true nearest codeword were in neither group, three codewords would lie
// within twice the score error (~2^-20) of each other: a near tie, where the parity rules
// accept either answer.
//
// One persistent CTA per SM, tiles of 128 blocks (64 or 128 vectors), 6 warps:
//   warp 0     bulk-copies codebook chunks into a ring of shared-memory stages
//   warp 1     issues the score MMAs (M = 128 blocks, N = one chunk of codewords, K = 3k + 16)
//              into two tensor-memory score buffers
//   warps 2-5  one thread per block (its tensor-memory lane): norm and rotation (fp32 FFMA),
//              the A operand, the scan of every chunk's scores, the exact re-score and the
//              record.
#include <cstdint>

#include <cuda_fp16.h>

#include "codec_sm100.h"
#include "fq_device.cuh"
#include "sm100_ptx.cuh"

namespace fq {
namespace sm100 {
namespace {

constexpr int kRowsH = 128;
constexpr int kThreadsH = 192;

__device__ unsigned int g_enchk_wait_timeouts = 0;  // CTAs whose bounded waits gave up

template <int KB, int MB, int D>
struct HCfg {
  static_assert(KB * MB == D, "k = d / MB");
  static constexpr int KOP = 3 * KB + 16;            // operand K (fp16 elements)
  static constexpr int SBO = KOP * 16;               // bytes between 8-row groups
  static constexpr int CH = KB <= 32 ? 256 : 128;    // codewords per chunk (MMA N)
  static constexpr int CHB = CH * KOP * 2;           // bytes of one chunk
  static constexpr int STAGES = KB <= 32 ? 3 : 2;
  static constexpr int TMEM_COLS = 2 * CH;           // two score buffers
  static constexpr int VPT = kRowsH / MB;            // vectors per tile
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_A = OFF_RING + STAGES * CHB;
  static constexpr int OFF_BAR = OFF_A + kRowsH * KOP * 2;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;   // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(CHB % 16 == 0 && (OFF_A % 1024) == 0, "bulk-copy and operand alignment");
};

struct HParams {
  const IndexHeader* hdr; // the index buffer's header (device memory)
  int64_t n;
  const uint16_t* x;      // [n, D] fp16 bits
  const float* rot;       // [D, D]
  const float* cb;        // [N, KB] fp32
  const uint8_t* op;      // prepared codebook operand: N / CH chunks of CHB bytes
  int N;                  // codewords
  int B;                  // bits per index
  int P;                  // record bytes
  uint8_t* codes;
  uint16_t* norms;
};

// Byte offset of element e of row r in the no-swizzle K-major layout (8 x 16-byte core matrices,
// 128 bytes apart along K, sbo bytes apart along the rows).
__device__ __forceinline__ uint32_t op_off(uint32_t r, uint32_t e, uint32_t sbo) {
  return (r >> 3) * sbo + (e >> 3) * 128u + (r & 7u) * 16u + (e & 7u) * 2u;
}

// Bounded wait that gives up early when another role raised the abort flag.
__device__ __forceinline__ bool wait_h(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t it = 0; it < (ptx::kSpinLimit << 2); ++it) {
    if (ptx::mbar_test(bar, parity)) return true;
    if ((it & 63u) == 63u && *abort) return false;
  }
  *abort = 1;
  return false;
}

__device__ __forceinline__ uint32_t h2u_h(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

template <int KB, int MB, int D>
__global__ void __launch_bounds__(kThreadsH, 1) encode_highk_kernel(HParams p) {
  using C = HCfg<KB, MB, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sRing = smem + C::OFF_RING;
  uint8_t* sA = smem + C::OFF_A;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);   // [STAGES] chunk landed
  uint64_t* empty = full + C::STAGES;                                  // [STAGES] chunk consumed
  uint64_t* d_full = empty + C::STAGES;                                // [2] scores ready
  uint64_t* d_empty = d_full + 2;                                      // [2] scores read
  uint64_t* a_full = d_empty + 2;                                      // A tile written
  uint64_t* a_empty = a_full + 1;                                      // A tile's MMAs done
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(a_empty + 1);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nc = p.N / C::CH;                       // chunks per tile
  // an index that does not describe this codebook in this layout is ignored: the blocks are
  // then searched exactly on the CUDA cores (slow, but the same result)
  const IndexHeader hd = *p.hdr;
  const bool use_op = hd.magic == kIndexMagic && hd.version == kIndexVersion &&
                      hd.kind == FQ_INDEX_TENSOR && hd.k == KB && hd.N == p.N && hd.dp == D &&
                      hd.slots == C::CH && hd.entry_bytes == C::CHB && hd.id_bytes == C::KOP &&
                      hd.cells_offset == kTensorIndexDataOffset;
  const int64_t rows = p.n * MB;
  const int64_t n_tiles = (rows + kRowsH - 1) / kRowsH;
  const int n_local = blockIdx.x < n_tiles
                          ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

  if (warp == 0) {
    ptx::tmem_alloc(sTmem, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&d_full[b], 1);
      ptx::mbar_init(&d_empty[b], 128);
    }
    ptx::mbar_init(a_full, 128);
    ptx::mbar_init(a_empty, 1);
    *sAbort = 0;
    ptx::fence_mbar_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const int64_t total_chunks = use_op ? (int64_t)n_local * nc : 0;

  if (warp == 0) {
    // ---- producer: the codebook operand, chunk after chunk, for every local tile
    int64_t g = 0;
    if (lane == 0) {
      for (; g < total_chunks; ++g) {
        const int s = (int)(g % C::STAGES);
        if (g >= C::STAGES &&
            !wait_h(&empty[s], (uint32_t)((g / C::STAGES) - 1) & 1u, sAbort))
          break;
        ptx::mbar_arrive_expect_tx(&full[s], C::CHB);
        ptx::bulk_load(sRing + s * C::CHB, p.op + (size_t)(g % nc) * C::CHB, C::CHB, &full[s]);
      }
      // let the copies in flight land before the CTA can exit (bounded)
      for (int64_t t = g - C::STAGES < 0 ? 0 : g - C::STAGES; t < g; ++t)
        ptx::mbar_wait(&full[t % C::STAGES], (uint32_t)(t / C::STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16_f32(128, C::CH);
      const uint32_t aA = ptx::smem_u32(sA), aR = ptx::smem_u32(sRing);
      int64_t g = 0;
      int64_t committed = -1;  // last chunk whose MMAs were committed
      bool ok = true;
      for (int t = 0; t < (use_op ? n_local : 0) && ok; ++t) {
        if (!wait_h(a_full, (uint32_t)t & 1u, sAbort)) break;
        ptx::tc_fence_after();
        for (int c = 0; c < nc; ++c, ++g) {
          const int s = (int)(g % C::STAGES), b = (int)(g & 1);
          if (!wait_h(&full[s], (uint32_t)(g / C::STAGES) & 1u, sAbort) ||
              (g >= 2 && !wait_h(&d_empty[b], (uint32_t)((g >> 1) - 1) & 1u, sAbort))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d_t = tmem + (uint32_t)(b * C::CH);
#pragma unroll
          for (int ks = 0; ks < C::KOP / 16; ++ks)
            ptx::umma_f16(d_t, ptx::sdesc_kmajor_noswz(aA + 256u * ks, 128, C::SBO),
                          ptx::sdesc_kmajor_noswz(aR + s * C::CHB + 256u * ks, 128, C::SBO),
                          idesc, ks > 0 ? 1u : 0u);
          ptx::umma_commit(&empty[s]);
          ptx::umma_commit(&d_full[b]);
          if (c == nc - 1) ptx::umma_commit(a_empty);
          committed = g;
        }
      }
      if (committed >= 0)  // the last MMAs land before the tensor memory is released
        ptx::mbar_wait(&d_full[committed & 1], (uint32_t)(committed >> 1) & 1u);
    }
  } else {
    // ---- one thread per block: rotation, A operand, scan, exact re-score, record
    const int q = warp & 3;                              // tensor-memory lane quarter
    const int r = q * 32 + lane;                         // row of the tile (= lane)
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int64_t g = 0;
    for (int t = 0; t < n_local; ++t) {
      const int64_t tile = blockIdx.x + (int64_t)t * gridDim.x;
      const int64_t v = tile * C::VPT + r / MB;          // vector of this row
      const int j = r % MB;                              // block of that vector
      const bool live = v < p.n;
      // norm and z block j = (Pi x / nu)[j k, (j + 1) k), fp32
      float z[KB];
#pragma unroll
      for (int i = 0; i < KB; ++i) z[i] = 0.f;
      float ss = 0.f;
      if (live) {
        const uint4* xr = reinterpret_cast<const uint4*>(p.x + v * D);
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 8) {
          const uint4 xv = __ldg(xr + c0 / 8);
          float xf[8];
          const __half2* h2 = reinterpret_cast<const __half2*>(&xv);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f = __half22float2(h2[u]);
            xf[2 * u] = f.x;
            xf[2 * u + 1] = f.y;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) ss = fmaf(xf[u], xf[u], ss);
#pragma unroll
          for (int i = 0; i < KB; ++i) {
            const float4* pr = reinterpret_cast<const float4*>(p.rot + (size_t)(j * KB + i) * D + c0);
            const float4 a0 = __ldg(pr), a1 = __ldg(pr + 1);
            float acc = z[i];
            acc = fmaf(a0.x, xf[0], acc);
            acc = fmaf(a0.y, xf[1], acc);
            acc = fmaf(a0.z, xf[2], acc);
            acc = fmaf(a0.w, xf[3], acc);
            acc = fmaf(a1.x, xf[4], acc);
            acc = fmaf(a1.y, xf[5], acc);
            acc = fmaf(a1.z, xf[6], acc);
            acc = fmaf(a1.w, xf[7], acc);
            z[i] = acc;
          }
        }
      }
      const float nu = sqrtf(ss);
      const float inv = nu > 0.f ? 1.f / nu : 0.f;
      if (!use_op) {  // exact search over all codewords from the fp32 codebook
        float bd = INFINITY;
        int best = 0;
#pragma unroll 1
        for (int n = 0; n < p.N; ++n) {
          const float4* cr = reinterpret_cast<const float4*>(p.cb + (size_t)n * KB);
          float dist = 0.f;
#pragma unroll
          for (int i = 0; i < KB; i += 4) {
            const float4 cv = __ldg(cr + i / 4);
            const float u0 = z[i] * inv - cv.x, u1 = z[i + 1] * inv - cv.y;
            const float u2 = z[i + 2] * inv - cv.z, u3 = z[i + 3] * inv - cv.w;
            dist = fmaf(u0, u0, dist);
            dist = fmaf(u1, u1, dist);
            dist = fmaf(u2, u2, dist);
            dist = fmaf(u3, u3, dist);
          }
          if (dist < bd) {
            bd = dist;
            best = n;
          }
        }
        if (!(nu > 0.f)) best = 0;
        uint32_t word = (uint32_t)best;
        if constexpr (MB == 2) word |= __shfl_down_sync(0xffffffffu, word, 1) << p.B;
        if (live && j == 0) {
          uint8_t* rec = p.codes + v * p.P;
          for (int bb = 0; bb < p.P; ++bb) rec[bb] = (uint8_t)(word >> (8 * bb));
          p.norms[v] = f32_to_f16_bits(nu);
        }
        continue;
      }
      // the previous tile's MMAs must be done with the A tile before it is rewritten
      bool fail = false;
      if (t > 0) fail = !wait_h(a_empty, (uint32_t)(t - 1) & 1u, sAbort);
      if (fail || *sAbort) break;
      {
        __half zh[KB], zl[KB];
#pragma unroll
        for (int i = 0; i < KB; ++i) {
          const float zi = z[i] * inv;
          zh[i] = __float2half_rn(zi);
          zl[i] = __float2half_rn(zi - __half2float(zh[i]));
        }
#pragma unroll
        for (int e8 = 0; e8 < C::KOP / 8; ++e8) {
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 8 * e8 + 2 * u;
            __half h0, h1;
            auto pick = [&](int ee) -> __half {
              if (ee < KB) return zh[ee];
              if (ee < 2 * KB) return zh[ee - KB];
              if (ee < 3 * KB) return zl[ee - 2 * KB];
              return (ee < 3 * KB + 2) ? __float2half_rn(1.f) : __float2half_rn(0.f);
            };
            h0 = pick(e);
            h1 = pick(e + 1);
            w[u] = h2u_h(__halves2half2(h0, h1));
          }
          *reinterpret_cast<uint4*>(sA + op_off((uint32_t)r, (uint32_t)(8 * e8), C::SBO)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(a_full);
      // scan every chunk's scores: the best and runner-up 8-codeword group by approximate min
      float b1 = INFINITY, b2 = INFINITY;
      int g1 = 0, g2 = 0;
      for (int c = 0; c < nc; ++c, ++g) {
        const int b = (int)(g & 1);
        if (!wait_h(&d_full[b], (uint32_t)(g >> 1) & 1u, sAbort)) {
          fail = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_t = tmem + lane_base + (uint32_t)(b * C::CH);
#pragma unroll 1
        for (int c0 = 0; c0 < C::CH; c0 += 32) {
          uint32_t s0[16], s1[16];
          ptx::tmem_ld16(d_t + c0, s0);
          ptx::tmem_ld16(d_t + c0 + 16, s1);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            const uint32_t* sv = gg < 2 ? s0 + 8 * gg : s1 + 8 * (gg - 2);
            float m = __uint_as_float(sv[0]);
#pragma unroll
            for (int u = 1; u < 8; ++u) m = fminf(m, __uint_as_float(sv[u]));
            const int gid = (c * C::CH + c0) / 8 + gg;
            const bool lt1 = m < b1, lt2 = m < b2;
            b2 = lt1 ? b1 : (lt2 ? m : b2);
            g2 = lt1 ? g1 : (lt2 ? gid : g2);
            b1 = lt1 ? m : b1;
            g1 = lt1 ? gid : g1;
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&d_empty[b]);
      }
      if (fail) break;
      // exact fp32 re-score of both groups (z = head + residual from the A tile)
      int best = 0;
      {
        float zz[KB];
#pragma unroll
        for (int i = 0; i < KB; i += 8) {
          const uint4 hv = *reinterpret_cast<const uint4*>(sA + op_off((uint32_t)r, (uint32_t)i, C::SBO));
          const uint4 lv = *reinterpret_cast<const uint4*>(sA + op_off((uint32_t)r, (uint32_t)(2 * KB + i), C::SBO));
          const __half2* hh = reinterpret_cast<const __half2*>(&hv);
          const __half2* ll = reinterpret_cast<const __half2*>(&lv);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 fh = __half22float2(hh[u]), fl = __half22float2(ll[u]);
            zz[i + 2 * u] = fh.x + fl.x;
            zz[i + 2 * u + 1] = fh.y + fl.y;
          }
        }
        float bd = INFINITY;
        best = 0x7fffffff;
#pragma unroll 1
        for (int cand = 0; cand < 16; ++cand) {
          const int n = (cand < 8 ? g1 : g2) * 8 + (cand & 7);
          const float4* cr = reinterpret_cast<const float4*>(p.cb + (size_t)n * KB);
          float dist = 0.f;
#pragma unroll
          for (int i = 0; i < KB; i += 4) {
            const float4 cv = __ldg(cr + i / 4);
            float u0 = zz[i] - cv.x, u1 = zz[i + 1] - cv.y, u2 = zz[i + 2] - cv.z, u3 = zz[i + 3] - cv.w;
            dist = fmaf(u0, u0, dist);
            dist = fmaf(u1, u1, dist);
            dist = fmaf(u2, u2, dist);
            dist = fmaf(u3, u3, dist);
          }
          if (dist < bd || (dist == bd && n < best)) {
            bd = dist;
            best = n;
          }
        }
        if (!(nu > 0.f)) best = 0;
      }
      // record: index j at bits [j B, (j + 1) B), LSB first; the block-0 thread writes it
      uint32_t word = (uint32_t)best;
      if constexpr (MB == 2) {
        const uint32_t other = __shfl_down_sync(0xffffffffu, word, 1);
        word |= other << p.B;
      }
      if (live && j == 0) {
        uint8_t* rec = p.codes + v * p.P;
        for (int bb = 0; bb < p.P; ++bb) rec[bb] = (uint8_t)(word >> (8 * bb));
        p.norms[v] = f32_to_f16_bits(nu);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *sAbort) atomicAdd(&g_enchk_wait_timeouts, 1u);
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int KB, int MB, int D>
cudaError_t launch_hk(const HParams& p, cudaStream_t st) {
  using C = HCfg<KB, MB, D>;
  auto kern = encode_highk_kernel<KB, MB, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (p.n * MB + kRowsH - 1) / kRowsH;
  const int ctas = (int)(tiles < sms ? tiles : sms);
  kern<<<ctas, kThreadsH, C::SMEM, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool highk_supported(fq_dtype xt, const Shape& s, const void* x, const void* index,
                     const float* rot, const float* cb) {
  if (xt != FQ_F16 || index == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(rot) & 15) || (reinterpret_cast<uintptr_t>(cb) & 15))
    return false;
  if (!((s.d == 64 && (s.k == 32 || s.k == 64)) || (s.d == 128 && s.k == 64))) return false;
  if (s.dp != s.d || s.N < (s.k <= 32 ? 256 : 128) || s.N > 65536) return false;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(index) & 15))
    return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10;
}

cudaError_t launch_encode_highk(const void* x, int64_t n, const Shape& s, const float* rot,
                                const float* cb, const void* index, uint8_t* codes,
                                uint16_t* norms, cudaStream_t st) {
  HParams p;
  p.n = n;
  p.x = static_cast<const uint16_t*>(x);
  p.rot = rot;
  p.cb = cb;
  p.hdr = static_cast<const IndexHeader*>(index);
  p.op = static_cast<const uint8_t*>(index) + kTensorIndexDataOffset;
  p.N = s.N;
  p.B = s.B;
  p.P = s.P;
  p.codes = codes;
  p.norms = norms;
  if (s.d == 64 && s.k == 32) return launch_hk<32, 2, 64>(p, st);
  if (s.d == 64 && s.k == 64) return launch_hk<64, 1, 64>(p, st);
  if (s.d == 128 && s.k == 64) return launch_hk<64, 2, 128>(p, st);
  return cudaErrorNotSupported;
}

}  // namespace sm100
cudaError_t wait_timeouts_encode_highk(bool clear, unsigned* count) {
  return read_wait_counter(sm100::g_enchk_wait_timeouts, clear, count);
}

}  // namespace fq
