// Internal declarations shared by the translation units of libfq (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/fq.h"

namespace fq {

constexpr int kMaxD = 256;
constexpr int kMaxK = 8;
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
// Layout of the buffer made by fq_build_search_index (all little-endian, 8-byte aligned):
//   IndexHeader (64 bytes)
//   cells:    n_cells entries of `entry_bytes` bytes each; an entry is `slots` uint16 candidate
//             ids followed (when entry_bytes > 2*slots) by padding and a uint32 overflow word;
//             ids of a cell with fewer candidates than slots are padded by repeating the first.
//   overflow: uint16 array; an overflow word w != 0xFFFFFFFF points at element w, which holds
//             the number of extra candidates followed by their ids.
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
  uint32_t max_candidates;  // longest candidate list (inline + overflow)
};
static_assert(sizeof(IndexHeader) == 64, "index header is 64 bytes");
constexpr uint32_t kIndexMagic = 0x58495146u;  // "FQIX"
constexpr uint32_t kIndexVersion = 1;
constexpr uint32_t kNoOverflow = 0xFFFFFFFFu;

// ---- launchers (return cudaGetLastError() of the launch) ----------------------------------
cudaError_t launch_encode_generic(const void* x, fq_dtype xt, int64_t n, const Shape& s,
                                  const float* rot, const float* cb, uint8_t* codes,
                                  uint16_t* norms, const void* index, cudaStream_t st);
cudaError_t launch_decode_generic(const uint8_t* codes, const uint16_t* norms, int64_t n,
                                  const Shape& s, const float* rot, const float* cb, void* y,
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
};
int attn_splits(int B, int Hkv, int64_t T);
int64_t attn_tokens_per_split(int64_t T, int splits);
size_t attn_partials_bytes(int B, int Hq, int splits, int dpV);
size_t attn_smem_bytes(const AttnArgs& a);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st);

}  // namespace fq
