// Internal declarations shared by the translation units of libfq (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/fq.h"

namespace fq {

constexpr int kMaxD = 256;
constexpr int kMaxK = 256;
constexpr int kMaxN = 65536;

struct Shape {
  int d, k, N;   // as passed
  int dp;        // padded dimension k * ceil(d / k)
  int m;         // blocks per vector
  int B;         // bits per index
  int P;         // payload bytes per record
};

// Validates (d, k, N) against the ABI limits and fills the derived sizes.
fq_status make_shape(int d, int k, int N, Shape* s);

// ---- search index (host builder and device view) ------------------------------------------
// Layout of the buffer made by fq_build_search_index (little-endian, 8-byte aligned):
//   IndexHeader (64 bytes)
//   cells:    n_cells entries of `entry_bytes` bytes.  An entry holds `slots` candidate ids of
//             `id_bytes` bytes each (1 when N <= 256, else 2), sorted by increasing index; the
//             rest of the id area (up to a 4-byte boundary) repeats the last inline id; when max_candidates > slots (exact kind only)
//             the entry ends with a uint32 overflow word.
//   overflow: uint16 array; an overflow word w != 0xFFFFFFFF points at element w, which holds
//             the number of further candidates followed by their ids (all larger than the
//             inline ones).
// Cell of a block z (k coordinates): c_a = clamp(floor((z_a - lo) * inv_h), 0, L - 1),
// flat = sum_a c_a L^a.  Every list is built for the cell enlarged by a margin, so the fp32
// rounding of this mapping cannot move a block to a cell whose list misses its nearest
// codeword (exact kind).
struct IndexHeader {
  uint32_t magic;        // kIndexMagic
  uint32_t version;      // kIndexVersion
  int32_t kind;          // fq_index_kind
  int32_t k, N, L;
  int32_t dp;            // padded dimension the grid range was computed for
  int32_t slots;         // inline candidate slots per cell
  float lo;              // grid origin on every axis (-R)
  float inv_h;           // 1 / cell width
  int32_t n_cells;       // L^k
  int32_t entry_bytes;   // bytes per cell entry (multiple of 4)
  uint32_t cells_offset; // byte offset of the cell table
  uint32_t overflow_offset;
  uint32_t overflow_elems;
  uint16_t max_candidates;  // longest candidate list
  uint16_t id_bytes;        // 1 or 2
};
static_assert(sizeof(IndexHeader) == 64, "index header is 64 bytes");
constexpr uint32_t kIndexMagic = 0x58495146u;  // "FQIX"
constexpr uint32_t kIndexVersion = 2;
constexpr uint32_t kNoOverflow = 0xFFFFFFFFu;
// FQ_INDEX_TENSOR buffers: the header, then (from this byte offset) N / slots chunks of
// entry_bytes bytes, each holding `slots` codeword rows of id_bytes (= 3k + 16) fp16 elements
// in the tensor cores' no-swizzle K-major layout (8-row x 16-byte core matrices, 128 bytes
// apart along K, 16 * (3k + 16) bytes apart along the rows); row n of the codebook holds
// [a_hi(k) | a_lo(k) | a_hi(k) | cc_hi | cc_lo | 0 x 14] with a = -2 c_n, cc = |c_n|^2 and
// x_lo = fp16(x - x_hi).
constexpr uint32_t kTensorIndexDataOffset = 128;

__host__ __device__ inline bool index_has_overflow(const IndexHeader& h) {
  return h.kind == FQ_INDEX_EXACT && h.max_candidates > h.slots;
}
__host__ __device__ inline int index_entry_id(const uint8_t* entry, int i, int id_bytes) {
  return id_bytes == 1 ? entry[i] : reinterpret_cast<const uint16_t*>(entry)[i];
}

// ---- random access ---------------------------------------------------------------------------
// Gather mode of a decode: output row v decodes record ids[v] of a plane of n_records records
// (ids == nullptr: record v).  Ids outside [0, n_records) decode as NaN rows.
struct Gather {
  const int64_t* ids;
  int64_t n_records;
};
// Append mode of an encode: input row v = b * hkv + g is written to record slot
// (b * hkv + g) * T + lengths[b] of a [B, hkv, T] plane (lengths == nullptr: record v).  A slot
// outside [0, T) is not written.
struct AppendMap {
  const int32_t* lengths;
  int hkv;
  int64_t T;
};

// Target-aware rescale of a decode (Block Sphere VQ key design 3): y = nu S (Pi^T zbar)[0:d] with
// S from the stored rho (fp16 plane) and the rule (rho == nullptr: S = 1).
struct Rescale {
  const uint16_t* rho;
  int rule;  // fq_rescale_rule
};

// ---- launchers (return cudaGetLastError() of the launch) ----------------------------------
cudaError_t launch_encode_generic(const void* x, fq_dtype xt, int64_t n, const Shape& s,
                                  const float* rot, const float* cb, uint8_t* codes,
                                  uint16_t* norms, const void* index, cudaStream_t st,
                                  AppendMap map = AppendMap{nullptr, 1, 0},
                                  uint16_t* rho = nullptr);
cudaError_t launch_decode_generic(const uint8_t* codes, const uint16_t* norms, int64_t n,
                                  const Shape& s, const float* rot, const float* cb, void* y,
                                  fq_dtype yt, cudaStream_t st,
                                  Gather gather = Gather{nullptr, 0},
                                  Rescale rs = Rescale{nullptr, 0});

// TurboQuant_prod (variants.cu)
cudaError_t launch_encode_prod(const void* x, fq_dtype xt, int64_t n, int d, int N1, int B1,
                               int P1, const float* rot, const float* c1, const float* qjl,
                               uint8_t* codes, uint8_t* signs, uint16_t* norms, uint16_t* gamma,
                               cudaStream_t st);
cudaError_t launch_decode_prod(const uint8_t* codes, const uint8_t* signs, const uint16_t* norms,
                               const uint16_t* gamma, int64_t n, int d, int N1, int B1, int P1,
                               const float* rot, const float* c1, const float* qjl, void* y,
                               fq_dtype yt, cudaStream_t st);

struct AttnArgs {
  const uint16_t* q;
  int B, Hq, Hkv;
  int64_t T;
  int d;
  const uint8_t* k_codes;
  const uint16_t* k_norms;
  Shape ks;
  const float* rotK;
  const float* cbK;
  const uint8_t* v_codes;
  const uint16_t* v_norms;
  Shape vs;
  const float* rotV;
  const float* cbV;
  float scale;
  float* out;
  float* partials;  // [B, Hq, splits, dpV + 2]
  int splits;
  int64_t tokens_per_split;
  // per-sequence context lengths (device, [B]; nullptr: every sequence has T tokens).  Sequence
  // b attends over its first clamp(lengths[b] + length_bias, 0, T) tokens.
  const int32_t* lengths;
  int length_bias;
  // when non-null, the combine kernel adds one to lengths[b] (capped at T) after reading the
  // partials: the decode step that appended its own token advances its sequence
  int32_t* lengths_out;
};

// Tokens of sequence b that an attention step reads.
__host__ __device__ inline int64_t attn_seq_len(const AttnArgs& a, int b) {
  if (a.lengths == nullptr) return a.T;
  int64_t L = (int64_t)a.lengths[b] + a.length_bias;
  return L < 0 ? 0 : (L > a.T ? a.T : L);
}
// Validates the arguments of fq_attn_decode (everything but the workspace) and fills `a` and
// the workspace bytes the call needs; nothing is enqueued.  T = 0 returns FQ_OK with *need = 0.
fq_status attn_prepare(const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d,
                       const uint8_t* k_codes, const uint16_t* k_norms, int kK, int NK,
                       const float* rotK, const float* cbK, const uint8_t* v_codes,
                       const uint16_t* v_norms, int kV, int NV, const float* rotV,
                       const float* cbV, float scale, float* out, AttnArgs* a, size_t* need);
// Context splits per (batch, kv head): about three 128-token-tile CTAs per SM, twice as many
// when per-sequence lengths leave the splits past each sequence's end empty (ragged).  The
// workspace is sized for the ragged count, which is never the smaller.
int attn_splits(int B, int Hkv, int64_t T, bool ragged = false);
int64_t attn_tokens_per_split(int64_t T, int splits);
size_t attn_partials_bytes(int B, int Hq, int splits, int dpV);
size_t attn_smem_bytes(const AttnArgs& a);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st);
cudaError_t launch_attn_combine(const AttnArgs& a, cudaStream_t st);

// ---- bounded-wait failure counters ---------------------------------------------------------
// Every kernel file whose kernels wait on mbarriers keeps a __device__ count of the CTAs whose
// bounded waits gave up.  Its reader adds that count on the current device to *count and zeroes
// it when `clear` is set (synchronous copies; the caller synchronises the device first).
template <class Sym>
inline cudaError_t read_wait_counter(const Sym& sym, bool clear, unsigned* count) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, sym, sizeof(v));
  if (e != cudaSuccess) return e;
  *count += v;
  if (clear && v != 0) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(sym, &zero, sizeof(zero));
  }
  return e;
}
cudaError_t wait_timeouts_encode(bool clear, unsigned* count);        // encode_sm100.cu
cudaError_t wait_timeouts_encode_large(bool clear, unsigned* count);  // encode_large_sm100.cu
cudaError_t wait_timeouts_decode(bool clear, unsigned* count);        // decode_sm100.cu
cudaError_t wait_timeouts_decode_large(bool clear, unsigned* count);  // decode_large_sm100.cu
cudaError_t wait_timeouts_attn(bool clear, unsigned* count);          // attn_sm100.cu
cudaError_t wait_timeouts_selftest(bool clear, unsigned* count);      // selftest.cu
cudaError_t wait_timeouts_encode_highk(bool clear, unsigned* count);  // encode_highk_sm100.cu
cudaError_t wait_timeouts_encode_grid(bool clear, unsigned* count);   // encode_grid_sm100.cu
cudaError_t launch_selftest_wait(uint32_t polls, cudaStream_t st);     // selftest.cu

// sm_100a tensor-core attention (attn_sm100.cu) for the shapes it supports.
namespace attn100 {
bool supported(const AttnArgs& a);
cudaError_t launch(const AttnArgs& a, cudaStream_t st);
}  // namespace attn100

}  // namespace fq
