// sm_100a fq_decode for d = 128, k = 4 (32 blocks per vector), N = 2^B <= 4096.
//
// FibQuant summary, decoder (sec. 2.3): unpack the m indices of a record, concatenate the
// codewords into zhat, rotate back and rescale: y = nu (Pi^T zhat)[0:d].  With d = d' = 128 the
// inverse rotation of a 128-vector tile is one 128 x 128 x 128 product on the tensor cores,
//   D[row][c] = sum_r zhat[row][r] Pi[r][c],
// with both operands split into an fp16 head and an fp16 residual (x_lo = fp16(x - x_hi), kept
// unscaled: a subnormal residual still carries the value to ~2^-25 absolute) and three products
// accumulated into one fp32 accumulator:
//   D = Z_hi Pi_hi + Z_hi Pi_lo + Z_lo Pi_hi      (the dropped Z_lo Pi_lo term is ~2^-22 of D).
// The zhat rows are gathered from a shared-memory table of the codebook (per codeword: four fp16
// heads, then four fp16 residuals) and written straight into tensor memory, where they are the A
// operand; Pi^T (head rows, residual rows) is the B operand in shared memory (128-byte swizzle).
//
// One persistent CTA per SM with two independent pipelines of 128 threads (one thread per row).
// Each pipeline owns 256 tensor-memory columns (A_hi 64 | A_lo 64 | D 128) and runs
// gather -> MMA -> scale-and-store for its tiles; the two pipelines' phases overlap.  A full,
// aligned tile's records and norms arrive by bulk copies into a double buffer two tiles ahead;
// fp16 output is staged in shared memory in the 128-byte swizzle and leaves with TMA tensor
// stores (full lines instead of 32 row fragments per store instruction).  Gathered token lists,
// the ragged last tile and unaligned planes read their records per thread; fp32 output is
// stored per thread.
#include <cstdint>
#include <cstring>

#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "codec_sm100.h"
#include "fq_device.cuh"
#include "sm100_ptx.cuh"

namespace fq {
namespace sm100 {
namespace {

constexpr int kRowsDL = 128;                 // vectors per tile (UMMA M)
constexpr int kPipesDL = 2;
constexpr int kThreadsDL = 128 * kPipesDL;
constexpr int kDimDL = 128;                  // d = d'
constexpr int kBlocksDL = 32;                // m = d / k with k = 4

__device__ unsigned int g_decl_wait_timeouts = 0;  // CTAs whose bounded waits gave up

template <int B>
struct DLCfg {
  static constexpr int N = 1 << B;
  static constexpr int P = kBlocksDL * B / 8;  // 4 B bytes: whole 32-bit words
  static constexpr int NW = B + 1;             // record words plus a zero word
  static constexpr int REC = kRowsDL * P;      // one tile's records (a multiple of 16 bytes)
  static constexpr int NRM = kRowsDL * 2;      // one tile's norms
  static constexpr int OFF_PI = 0;             // [head | residual][2 K halves][128 x 128 B]
  static constexpr int OFF_TBL = 4 * 16384;    // N x 16 B: heads (4 fp16), residuals (4 fp16)
  static constexpr int OFF_OUT = (OFF_TBL + N * 16 + 1023) / 1024 * 1024;  // [pipe][2 boxes][128 x 128 B] fp16
  static constexpr int OFF_REC = OFF_OUT + kPipesDL * 32768;  // [pipe][2][REC]
  static constexpr int OFF_NRM = OFF_REC + kPipesDL * 2 * REC;  // [pipe][2][NRM]
  static constexpr int OFF_BAR = OFF_NRM + kPipesDL * 2 * NRM;
  static constexpr int SMEM = OFF_BAR + 64 + 1024;  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(OFF_OUT % 1024 == 0 && REC % 16 == 0, "TMA and bulk-copy alignment");
};

struct DLArgs {
  int64_t n;
  const uint8_t* codes;
  const uint16_t* norms;
  const float* rot;
  const float* cb;
  void* y;
  Gather gather;  // output row r decodes record gather.ids[r] (ids == nullptr: record r)
  int bulk;       // full tiles' records and norms by bulk copies (16-byte aligned planes)
  int tma;        // fp16 output by TMA tensor stores
};

__device__ __forceinline__ uint32_t h2u_dl(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// fp16 head and unscaled fp16 residual of v
__device__ __forceinline__ void split_hl(float v, __half& hi, __half& lo) {
  hi = __float2half_rn(v);
  lo = __float2half_rn(v - __half2float(hi));
}

// Barrier of one pipeline's 128 threads that also ORs a predicate across them.
__device__ __forceinline__ bool pipe_sync_or_dl(int pipe, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(pipe + 1)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void pipe_sync_dl(int pipe) {
  asm volatile("bar.sync %0, 128;" ::"r"(pipe + 3) : "memory");
}

template <int B, bool F16>
__global__ void __launch_bounds__(kThreadsDL, 1)
    decode_large_kernel(const __grid_constant__ CUtensorMap ymap, DLArgs p) {
  using C = DLCfg<B>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sPi = smem + C::OFF_PI;
  uint4* sTbl = reinterpret_cast<uint4*>(smem + C::OFF_TBL);
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // one per pipeline
  uint64_t* rec_full = mma_done + kPipesDL;                               // [pipe][2]
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(rec_full + 2 * kPipesDL);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int pipe = tid >> 7, lt = tid & 127;
  const int64_t n_tiles = (p.n + kRowsDL - 1) / kRowsDL;
  const int64_t stride = (int64_t)gridDim.x * kPipesDL;
  const int64_t first = (int64_t)blockIdx.x * kPipesDL + pipe;

  // ---- set-up: tensor memory, barriers, Pi^T operand, codebook table ----
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    for (int q = 0; q < kPipesDL; ++q) ptx::mbar_init(&mma_done[q], 1);
    for (int q = 0; q < 2 * kPipesDL; ++q) ptx::mbar_init(&rec_full[q], 1);
    *sAbort = 0;
    ptx::fence_mbar_init();
    if (F16 && p.tma) ptx::prefetch_tensormap(&ymap);
  }
  // B operand: row c holds Pi[r][c] over r (K-major), heads at +0, residuals at +32 KB; each a
  // pair of 64-wide K halves in the 128-byte swizzle.  Coalesced reads along c.
#pragma unroll 1
  for (int e0 = 0; e0 < kDimDL * kDimDL; e0 += 16 * kThreadsDL) {
    float v[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = __ldg(p.rot + e0 + q * kThreadsDL + tid);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = e0 + q * kThreadsDL + tid;
      const int r = e >> 7, c = e & 127;
      __half hi, lo;
      split_hl(v[q], hi, lo);
      const uint32_t o = (uint32_t)(r >> 6) * 16384u + ptx::sw128_offset((uint32_t)c, (uint32_t)(r & 63));
      *reinterpret_cast<__half*>(sPi + o) = hi;
      *reinterpret_cast<__half*>(sPi + 32768 + o) = lo;
    }
  }
  // codebook table: per codeword (h0 h1, h2 h3, l0 l1, l2 l3)
#pragma unroll 1
  for (int c0 = 0; c0 < C::N; c0 += 4 * kThreadsDL) {
    float4 cv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q * kThreadsDL + tid;
      cv[q] = c < C::N ? __ldg(reinterpret_cast<const float4*>(p.cb) + c)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q * kThreadsDL + tid;
      if (c < C::N) {
        __half h[4], l[4];
        split_hl(cv[q].x, h[0], l[0]);
        split_hl(cv[q].y, h[1], l[1]);
        split_hl(cv[q].z, h[2], l[2]);
        split_hl(cv[q].w, h[3], l[3]);
        sTbl[c] = make_uint4(h2u_dl(__halves2half2(h[0], h[1])), h2u_dl(__halves2half2(h[2], h[3])),
                             h2u_dl(__halves2half2(l[0], l[1])), h2u_dl(__halves2half2(l[2], l[3])));
      }
    }
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;

  // ---- pipeline `pipe`: tiles first, first + stride, ... ----
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  const uint32_t t_pipe = tmem + (uint32_t)pipe * 256;      // A_hi | A_lo | D, lane 0
  const uint32_t ta_hi = t_pipe + lane_base, ta_lo = ta_hi + 64, td = ta_hi + 128;
  constexpr uint32_t idesc = ptx::idesc_f16_f32(128, 128);
  const uint32_t pi_addr = ptx::smem_u32(sPi);
  const int n_local = first < n_tiles ? (int)((n_tiles - 1 - first) / stride + 1) : 0;

  // tile i of this pipeline arrives by bulk copies when it is full and the planes are aligned
  uint8_t* sRec = smem + C::OFF_REC + pipe * 2 * C::REC;
  uint8_t* sNrm = smem + C::OFF_NRM + pipe * 2 * C::NRM;
  auto bulk_tile = [&](int i) {
    const int64_t tile = first + (int64_t)i * stride;
    return p.bulk && (tile + 1) * kRowsDL <= p.n;
  };
  auto issue_rec = [&](int i) {  // thread lt == 0
    const int64_t tile = first + (int64_t)i * stride;
    uint64_t* bar = &rec_full[pipe * 2 + (i & 1)];
    ptx::mbar_arrive_expect_tx(bar, C::REC + C::NRM);
    ptx::bulk_load(sRec + (i & 1) * C::REC, p.codes + tile * C::REC, C::REC, bar);
    ptx::bulk_load(sNrm + (i & 1) * C::NRM,
                   reinterpret_cast<const uint8_t*>(p.norms + tile * kRowsDL), C::NRM, bar);
  };
  int rec_issued = 0;    // thread lt == 0: bulk copies issued (tiles 0 .. rec_issued - 1)
  int rec_consumed = 0;  // tiles whose records this thread has read
  auto load_rec = [&](int i, uint32_t (&w)[C::NW], float& nu) {
    rec_consumed = i + 1;
    if (bulk_tile(i)) {  // from the double buffer (bounded wait for the copy)
      const bool ok = ptx::mbar_wait(&rec_full[pipe * 2 + (i & 1)], (uint32_t)(i >> 1) & 1u);
      if (!ok) *sAbort = 1;
      // a record is P = 4 B bytes: 16-byte reads when P is a multiple of 16 (B % 4 == 0),
      // else 4-byte reads (every record starts on a 4-byte boundary)
      const uint8_t* rp = sRec + (i & 1) * C::REC + lt * C::P;
      if constexpr (B % 4 == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(rp);
#pragma unroll
        for (int q = 0; q < B / 4; ++q) {
          const uint4 v = src[q];
          w[4 * q] = v.x;
          w[4 * q + 1] = v.y;
          w[4 * q + 2] = v.z;
          w[4 * q + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < B; ++q) w[q] = reinterpret_cast<const uint32_t*>(rp)[q];
      }
      w[B] = 0u;
      nu = f16_bits_to_f32(reinterpret_cast<const uint16_t*>(sNrm + (i & 1) * C::NRM)[lt]);
      return;
    }
    const int64_t row = (first + (int64_t)i * stride) * kRowsDL + lt;
    int64_t rec = row;
    if (p.gather.ids != nullptr && row < p.n) {
      rec = __ldg(p.gather.ids + row);
      if (rec < 0 || rec >= p.gather.n_records) {  // outside the plane: a NaN row, no read
#pragma unroll
        for (int q = 0; q < C::NW; ++q) w[q] = 0u;
        nu = __int_as_float(0x7fc00000);
        return;
      }
    }
    if (row < p.n) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(p.codes + rec * C::P);
#pragma unroll
      for (int q = 0; q < B; ++q) w[q] = __ldg(src + q);
      nu = f16_bits_to_f32(__ldg(p.norms + rec));
    } else {
#pragma unroll
      for (int q = 0; q < B; ++q) w[q] = 0u;
      nu = 0.f;
    }
    w[B] = 0u;
  };
  // index j of a record: B bits from bit j B on (little-endian, LSB first)
  auto field = [&](const uint32_t (&w)[C::NW], int j) {
    const int off = j * B;
    return __funnelshift_r(w[off >> 5], w[(off >> 5) + 1], off & 31) & ((1u << B) - 1u);
  };

  uint32_t w[C::NW];
  float nu = 0.f;
  bool failed = false;
  int committed = 0;  // MMA batches committed by this pipeline's thread 0
  int stored = 0;     // TMA output stores committed by this pipeline's thread 0
  if (lt == 0)
    for (; rec_issued < 2 && rec_issued < n_local; ++rec_issued)
      if (bulk_tile(rec_issued)) issue_rec(rec_issued);
  if (n_local > 0) load_rec(0, w, nu);
  for (int i = 0; i < n_local; ++i) {
    const int64_t tile = first + (int64_t)i * stride;
    // zhat row -> tensor memory (heads and residuals), 8 blocks (16 columns) at a time
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 e[8];
#pragma unroll
      for (int b = 0; b < 8; ++b) e[b] = sTbl[field(w, 8 * q + b)];
      uint32_t h16[16], l16[16];
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        h16[2 * b] = e[b].x;
        h16[2 * b + 1] = e[b].y;
        l16[2 * b] = e[b].z;
        l16[2 * b + 1] = e[b].w;
      }
      ptx::tmem_st16(ta_hi + 16 * q, h16);
      ptx::tmem_st16(ta_lo + 16 * q, l16);
    }
    // the next tile's record loads are in flight during this tile's MMAs and stores
    uint32_t wn[C::NW];
    float nun = 0.f;
    if (i + 1 < n_local) load_rec(i + 1, wn, nun);
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    if (pipe_sync_or_dl(pipe, failed)) {
      failed = true;
      break;
    }
    if (lt == 0) {
      // every thread of the pipeline has read tile i's records: their buffer takes tile i + 2
      if (rec_issued < n_local && rec_issued <= i + 2) {
        if (bulk_tile(rec_issued)) issue_rec(rec_issued);
        ++rec_issued;
      }
      ptx::tc_fence_after();
      // D = Z_hi Pi_hi + Z_hi Pi_lo + Z_lo Pi_hi; K step ks: A columns 8 ks.., B + 32 B per step
      // inside a 64-wide K half
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        ptx::umma_f16_ts(t_pipe + 128, t_pipe + 8 * ks,
                         ptx::sdesc_kmajor_sw128(pi_addr + (ks >> 2) * 16384 + (ks & 3) * 32),
                         idesc, ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        ptx::umma_f16_ts(t_pipe + 128, t_pipe + 8 * ks,
                         ptx::sdesc_kmajor_sw128(pi_addr + 32768 + (ks >> 2) * 16384 + (ks & 3) * 32),
                         idesc, 1u);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        ptx::umma_f16_ts(t_pipe + 128, t_pipe + 64 + 8 * ks,
                         ptx::sdesc_kmajor_sw128(pi_addr + (ks >> 2) * 16384 + (ks & 3) * 32),
                         idesc, 1u);
      ptx::umma_commit(&mma_done[pipe]);
      ++committed;
    }
    // pipeline-uniform outcome of the wait (the fp16 epilogue has pipeline barriers)
    const bool ok = !pipe_sync_or_dl(pipe, !ptx::mbar_wait(&mma_done[pipe], (uint32_t)i & 1u));
    if (!ok) {
      failed = true;
      *sAbort = 1;
    } else {
      // y = nu D (fp16 or fp32), this thread's row
      ptx::tc_fence_after();
      const int64_t row = tile * kRowsDL + lt;
      const bool live = row < p.n;
      if (F16 && p.tma) {
        // the previous tile's output stores have read the staging buffer
        if (lt == 0) ptx::bulk_wait_group_read<0>();
        pipe_sync_dl(pipe);
        uint8_t* out = smem + C::OFF_OUT + pipe * 32768;
#pragma unroll
        for (int c0 = 0; c0 < kDimDL; c0 += 32) {
          uint32_t va[16], vb[16];
          ptx::tmem_ld16(td + c0, va);
          ptx::tmem_ld16(td + c0 + 16, vb);
          ptx::tmem_wait_ld();
          uint32_t o[16];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            o[q] = h2u_dl(__floats2half2_rn(nu * __uint_as_float(va[2 * q]),
                                            nu * __uint_as_float(va[2 * q + 1])));
            o[8 + q] = h2u_dl(__floats2half2_rn(nu * __uint_as_float(vb[2 * q]),
                                                nu * __uint_as_float(vb[2 * q + 1])));
          }
          // columns c0 .. c0 + 31 = 4 chunks of 16 bytes in box c0 / 64, 128-byte swizzle
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t chunk = (uint32_t)((c0 & 63) / 8 + q);
            *reinterpret_cast<uint4*>(out + (c0 >> 6) * 16384 + lt * 128 +
                                      (((chunk ^ (uint32_t)(lt & 7)) & 7u) << 4)) =
                make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
        }
        ptx::fence_proxy_async_smem();
        pipe_sync_dl(pipe);
        if (lt == 0) {
          ptx::tma_store_2d(&ymap, out, 0, (int)(tile * kRowsDL));
          ptx::tma_store_2d(&ymap, out + 16384, 64, (int)(tile * kRowsDL));
          ptx::bulk_commit_group();
          ++stored;
        }
      } else
      {
#pragma unroll
      for (int c0 = 0; c0 < kDimDL; c0 += 32) {
        uint32_t va[16], vb[16];
        ptx::tmem_ld16(td + c0, va);
        ptx::tmem_ld16(td + c0 + 16, vb);
        ptx::tmem_wait_ld();
        if (live) {
          if constexpr (F16) {
            uint32_t o[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              o[q] = h2u_dl(__floats2half2_rn(nu * __uint_as_float(va[2 * q]),
                                              nu * __uint_as_float(va[2 * q + 1])));
              o[8 + q] = h2u_dl(__floats2half2_rn(nu * __uint_as_float(vb[2 * q]),
                                                  nu * __uint_as_float(vb[2 * q + 1])));
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.y) + row * kDimDL + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.y) + row * kDimDL + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_float4(nu * __uint_as_float(va[4 * q]), nu * __uint_as_float(va[4 * q + 1]),
                                   nu * __uint_as_float(va[4 * q + 2]), nu * __uint_as_float(va[4 * q + 3]));
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[4 + q] = make_float4(nu * __uint_as_float(vb[4 * q]), nu * __uint_as_float(vb[4 * q + 1]),
                                       nu * __uint_as_float(vb[4 * q + 2]), nu * __uint_as_float(vb[4 * q + 3]));
          }
        }
      }
      }
    }
    ptx::tc_fence_before();
#pragma unroll
    for (int q = 0; q < C::NW; ++q) w[q] = wn[q];
    nu = nun;
  }

  // let this pipeline's MMAs, record copies and output stores in flight land before the
  // tensor memory is released and the CTA exits (bounded waits)
  if (lt == 0 && committed > 0) ptx::mbar_wait(&mma_done[pipe], (uint32_t)(committed - 1) & 1u);
  if (lt == 0)  // copies issued but never read (after a failure): land them first
    for (int t = rec_consumed; t < rec_issued; ++t)
      if (bulk_tile(t)) ptx::mbar_wait(&rec_full[pipe * 2 + (t & 1)], (uint32_t)(t >> 1) & 1u);
  if (lt == 0 && stored > 0) ptx::bulk_wait_group_all();
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *sAbort) atomicAdd(&g_decl_wait_timeouts, 1u);
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 dl_tensor_map_fn() {
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

template <int B, bool F16>
cudaError_t launch_dl(const DLArgs& p0, cudaStream_t st) {
  using C = DLCfg<B>;
  DLArgs p = p0;
  CUtensorMap map;
  std::memset(&map, 0, sizeof(map));
  p.tma = 0;
  auto fn = dl_tensor_map_fn();
  if (F16 && fn != nullptr && (reinterpret_cast<uintptr_t>(p.y) & 15) == 0 &&
      p.n < ((int64_t)1 << 31)) {
    // output y [n x 128] fp16 (256-byte rows), stored in boxes of 128 rows x 64 columns with the
    // 128-byte swizzle
    const cuuint64_t dims[2] = {(cuuint64_t)kDimDL, (cuuint64_t)p.n};
    const cuuint64_t strides[1] = {(cuuint64_t)kDimDL * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)kRowsDL};
    const cuuint32_t estr[2] = {1, 1};
    if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.y, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      p.tma = 1;
  }
  p.bulk = p.gather.ids == nullptr && (reinterpret_cast<uintptr_t>(p.codes) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(p.norms) & 15) == 0;
  auto kern = decode_large_kernel<B, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (p.n + kRowsDL - 1) / kRowsDL;
  const int64_t want = (tiles + kPipesDL - 1) / kPipesDL;
  const int ctas = (int)(want < sms ? want : sms);
  kern<<<ctas, kThreadsDL, C::SMEM, st>>>(map, p);
  return cudaGetLastError();
}

}  // namespace

bool decode_large_supported(fq_dtype yt, const Shape& s, const void* codes, const void* norms,
                            const void* y, const float* cb) {
  (void)yt;
  if (s.d != kDimDL || s.dp != kDimDL || s.k != 4 || s.B < 2 || s.B > 12) return false;
  if ((reinterpret_cast<uintptr_t>(codes) & 3) || (reinterpret_cast<uintptr_t>(norms) & 1) ||
      (reinterpret_cast<uintptr_t>(y) & 15) || (reinterpret_cast<uintptr_t>(cb) & 15))
    return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10;
}

cudaError_t launch_decode_large(const uint8_t* codes, const uint16_t* norms, int64_t n,
                                const Shape& s, const float* rot, const float* cb, void* y,
                                fq_dtype yt, cudaStream_t st, Gather gather) {
  DLArgs p{n, codes, norms, rot, cb, y, gather, 0, 0};
  const bool f16 = yt == FQ_F16;
  switch (s.B) {
#define FQ_DL_CASE(BB) \
  case BB:             \
    return f16 ? launch_dl<BB, true>(p, st) : launch_dl<BB, false>(p, st);
    FQ_DL_CASE(2) FQ_DL_CASE(3) FQ_DL_CASE(4) FQ_DL_CASE(5) FQ_DL_CASE(6) FQ_DL_CASE(7)
    FQ_DL_CASE(8) FQ_DL_CASE(9) FQ_DL_CASE(10) FQ_DL_CASE(11) FQ_DL_CASE(12)
#undef FQ_DL_CASE
  }
  return cudaErrorNotSupported;
}

}  // namespace sm100
cudaError_t wait_timeouts_decode_large(bool clear, unsigned* count) {
  return read_wait_counter(sm100::g_decl_wait_timeouts, clear, count);
}

}  // namespace fq
