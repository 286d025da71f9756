// extern "C" entry points of libfq: argument validation and dispatch.  No entry point
// allocates device memory, synchronises the stream, or keeps state between calls.
#include <cmath>
#include <cstdint>

#include "fq_internal.h"
#include "codec_sm100.h"

namespace fq {

fq_status make_shape(int d, int k, int N, Shape* s) {
  if (d < 1 || d > kMaxD || k < 1 || k > kMaxK || k > d) return FQ_ERR_UNSUPPORTED;
  if (N < 2 || N > kMaxN || (N & (N - 1)) != 0) return FQ_ERR_UNSUPPORTED;
  int B = 0;
  while ((1 << B) < N) ++B;
  s->d = d;
  s->k = k;
  s->N = N;
  s->dp = k * ((d + k - 1) / k);
  s->m = s->dp / k;
  s->B = B;
  s->P = (s->m * B + 7) / 8;
  return FQ_OK;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static fq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FQ_OK : FQ_ERR_CUDA; }

}  // namespace fq

using namespace fq;

extern "C" {

int fq_abi_version(void) { return 1; }

const char* fq_status_string(fq_status st) {
  switch (st) {
    case FQ_OK: return "ok";
    case FQ_ERR_INVALID_ARG: return "invalid argument";
    case FQ_ERR_UNSUPPORTED: return "unsupported size";
    case FQ_ERR_ALIGNMENT: return "misaligned pointer";
    case FQ_ERR_WORKSPACE: return "workspace or index buffer missing or too small";
    case FQ_ERR_CUDA: return "CUDA error";
    case FQ_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int fq_padded_dim(int d, int k) {
  Shape s;
  if (make_shape(d, k, 2, &s) != FQ_OK) return 0;
  return s.dp;
}

size_t fq_payload_bytes(int d, int k, int N) {
  Shape s;
  if (make_shape(d, k, N, &s) != FQ_OK) return 0;
  return (size_t)s.P;
}

fq_status fq_encode(const void* x, fq_dtype x_type, int64_t n, int d, int k, int N,
                    const float* rot, const float* codebook, uint8_t* codes, uint16_t* norms,
                    const void* search_index, void* stream) {
  Shape s;
  fq_status st = make_shape(d, k, N, &s);
  if (st != FQ_OK) return st;
  if (n < 0 || (x_type != FQ_F16 && x_type != FQ_F32)) return FQ_ERR_INVALID_ARG;
  if (n == 0) return FQ_OK;
  if (!x || !rot || !codebook || !codes || !norms) return FQ_ERR_INVALID_ARG;
  if (!aligned(x, x_type == FQ_F16 ? 2 : 4) || !aligned(norms, 2) || !aligned(rot, 4) ||
      !aligned(codebook, 4) || (search_index && !aligned(search_index, 8)))
    return FQ_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (sm100::highk_supported(x_type, s, x, search_index, rot, codebook))
    return from_cuda(sm100::launch_encode_highk(x, n, s, rot, codebook, search_index, codes,
                                                norms, cs));
  if (sm100::encode_large_supported(x_type, s, x, codes, codebook, search_index))
    return from_cuda(sm100::launch_encode_large(x, n, s, rot, codebook, codes, norms, cs));
  if (sm100::encode_grid_supported(x_type, s, x, codes, codebook, search_index))
    return from_cuda(sm100::launch_encode_grid(x, n, rot, codebook, search_index, codes, norms, cs));
  if (sm100::encode_supported(x_type, s, x, codes, norms))
    return from_cuda(sm100::launch_encode(x, x_type, n, s, rot, codebook, codes, norms,
                                          search_index, cs));
  return from_cuda(launch_encode_generic(x, x_type, n, s, rot, codebook, codes, norms,
                                         search_index, cs));
}

fq_status fq_decode(const uint8_t* codes, const uint16_t* norms, int64_t n, int d, int k, int N,
                    const float* rot, const float* codebook, void* y, fq_dtype y_type,
                    void* stream) {
  Shape s;
  fq_status st = make_shape(d, k, N, &s);
  if (st != FQ_OK) return st;
  if (n < 0 || (y_type != FQ_F16 && y_type != FQ_F32)) return FQ_ERR_INVALID_ARG;
  if (n == 0) return FQ_OK;
  if (!codes || !norms || !rot || !codebook || !y) return FQ_ERR_INVALID_ARG;
  if (!aligned(norms, 2) || !aligned(rot, 4) || !aligned(codebook, 4) ||
      !aligned(y, y_type == FQ_F16 ? 2 : 4))
    return FQ_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (sm100::decode_large_supported(y_type, s, codes, norms, y, codebook))
    return from_cuda(sm100::launch_decode_large(codes, norms, n, s, rot, codebook, y, y_type, cs));
  if (sm100::decode_supported(y_type, s, codes, norms, y))
    return from_cuda(sm100::launch_decode(codes, norms, n, s, rot, codebook, y, y_type, cs));
  return from_cuda(launch_decode_generic(codes, norms, n, s, rot, codebook, y, y_type, cs));
}

}  // extern "C"

namespace fq {

static fq_status attn_shapes(int B, int Hq, int Hkv, int64_t T, int d, int kK, int NK, int kV,
                             int NV, Shape* ks, Shape* vs) {
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 0 || Hq % Hkv != 0) return FQ_ERR_INVALID_ARG;
  if (Hq / Hkv > 16 || d > 128) return FQ_ERR_UNSUPPORTED;
  fq_status st = make_shape(d, kK, NK, ks);
  if (st != FQ_OK) return st;
  st = make_shape(d, kV, NV, vs);
  if (st != FQ_OK) return st;
  if (NK > 1024 || NV > 1024) return FQ_ERR_UNSUPPORTED;
  return FQ_OK;
}

fq_status attn_prepare(const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d,
                       const uint8_t* k_codes, const uint16_t* k_norms, int kK, int NK,
                       const float* rotK, const float* cbK, const uint8_t* v_codes,
                       const uint16_t* v_norms, int kV, int NV, const float* rotV,
                       const float* cbV, float scale, float* out, AttnArgs* a, size_t* need) {
  *need = 0;
  fq_status st = attn_shapes(B, Hq, Hkv, T, d, kK, NK, kV, NV, &a->ks, &a->vs);
  if (st != FQ_OK) return st;
  if (!std::isfinite(scale)) return FQ_ERR_INVALID_ARG;
  if (!q || !out) return FQ_ERR_INVALID_ARG;
  if (T == 0) return FQ_OK;
  if (!k_codes || !k_norms || !rotK || !cbK || !v_codes || !v_norms || !rotV || !cbV)
    return FQ_ERR_INVALID_ARG;
  if (!aligned(q, 2) || !aligned(k_norms, 2) || !aligned(v_norms, 2) || !aligned(rotK, 4) ||
      !aligned(cbK, 4) || !aligned(rotV, 4) || !aligned(cbV, 4) || !aligned(out, 4))
    return FQ_ERR_ALIGNMENT;
  a->q = q;
  a->B = B;
  a->Hq = Hq;
  a->Hkv = Hkv;
  a->T = T;
  a->d = d;
  a->k_codes = k_codes;
  a->k_norms = k_norms;
  a->rotK = rotK;
  a->cbK = cbK;
  a->v_codes = v_codes;
  a->v_norms = v_norms;
  a->rotV = rotV;
  a->cbV = cbV;
  a->scale = scale;
  a->out = out;
  a->partials = nullptr;
  a->lengths = nullptr;
  a->length_bias = 0;
  a->lengths_out = nullptr;
  a->splits = attn_splits(B, Hkv, T);
  a->tokens_per_split = attn_tokens_per_split(T, a->splits);
  *need = attn_partials_bytes(B, Hq, attn_splits(B, Hkv, T, true), a->vs.dp);
  if (attn_smem_bytes(*a) > 200 * 1024) return FQ_ERR_UNSUPPORTED;
  return FQ_OK;
}

}  // namespace fq

extern "C" {

size_t fq_attn_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int d, int kV) {
  Shape ks, vs;
  if (attn_shapes(B, Hq, Hkv, T, d, 1, 2, kV, 2, &ks, &vs) != FQ_OK) return 0;
  if (T == 0) return 0;
  return attn_partials_bytes(B, Hq, attn_splits(B, Hkv, T, true), vs.dp);
}

fq_status fq_attn_decode(const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d,
                         const uint8_t* k_codes, const uint16_t* k_norms, int kK, int NK,
                         const float* rotK, const float* cbK, const uint8_t* v_codes,
                         const uint16_t* v_norms, int kV, int NV, const float* rotV,
                         const float* cbV, float scale, float* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  AttnArgs a;
  size_t need = 0;
  fq_status st = attn_prepare(q, B, Hq, Hkv, T, d, k_codes, k_norms, kK, NK, rotK, cbK, v_codes,
                              v_norms, kV, NV, rotV, cbV, scale, out, &a, &need);
  if (st != FQ_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (T == 0)
    return from_cuda(cudaMemsetAsync(out, 0, (size_t)B * Hq * d * sizeof(float), cs));
  if (!workspace || workspace_bytes < need) return FQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return FQ_ERR_ALIGNMENT;
  a.partials = static_cast<float*>(workspace);
  return from_cuda(launch_attn(a, cs));
}

fq_status fq_decode_gather(const uint8_t* codes, const uint16_t* norms, int64_t n_records,
                           const int64_t* token_ids, int64_t n_ids, int d, int k, int N,
                           const float* rot, const float* codebook, void* y, fq_dtype y_type,
                           void* stream) {
  Shape s;
  fq_status st = make_shape(d, k, N, &s);
  if (st != FQ_OK) return st;
  if (n_ids < 0 || n_records < 0 || (y_type != FQ_F16 && y_type != FQ_F32))
    return FQ_ERR_INVALID_ARG;
  if (n_ids == 0) return FQ_OK;
  if (!token_ids || !rot || !codebook || !y || (n_records > 0 && (!codes || !norms)))
    return FQ_ERR_INVALID_ARG;
  if (!aligned(token_ids, 8) || !aligned(norms, 2) || !aligned(rot, 4) || !aligned(codebook, 4) ||
      !aligned(y, y_type == FQ_F16 ? 2 : 4))
    return FQ_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const Gather g{token_ids, n_records};
  if (sm100::decode_large_supported(y_type, s, codes, norms, y, codebook))
    return from_cuda(sm100::launch_decode_large(codes, norms, n_ids, s, rot, codebook, y, y_type,
                                                cs, g));
  return from_cuda(launch_decode_generic(codes, norms, n_ids, s, rot, codebook, y, y_type, cs, g));
}

fq_status fq_attn_decode_lengths(const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d,
                                 const int32_t* lengths, const uint8_t* k_codes,
                                 const uint16_t* k_norms, int kK, int NK, const float* rotK,
                                 const float* cbK, const uint8_t* v_codes,
                                 const uint16_t* v_norms, int kV, int NV, const float* rotV,
                                 const float* cbV, float scale, float* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  AttnArgs a;
  size_t need = 0;
  fq_status st = attn_prepare(q, B, Hq, Hkv, T, d, k_codes, k_norms, kK, NK, rotK, cbK, v_codes,
                              v_norms, kV, NV, rotV, cbV, scale, out, &a, &need);
  if (st != FQ_OK) return st;
  if (!lengths) return FQ_ERR_INVALID_ARG;
  if (!aligned(lengths, 4)) return FQ_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (T == 0)
    return from_cuda(cudaMemsetAsync(out, 0, (size_t)B * Hq * d * sizeof(float), cs));
  if (!workspace || workspace_bytes < need) return FQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return FQ_ERR_ALIGNMENT;
  a.partials = static_cast<float*>(workspace);
  a.lengths = lengths;
  a.splits = attn_splits(B, Hkv, T, true);
  a.tokens_per_split = attn_tokens_per_split(T, a.splits);
  return from_cuda(launch_attn(a, cs));
}

fq_status fq_attn_decode_append(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                int B, int Hq, int Hkv, int64_t T, int d, int32_t* lengths,
                                uint8_t* k_codes, uint16_t* k_norms, int kK, int NK,
                                const float* rotK, const float* cbK, uint8_t* v_codes,
                                uint16_t* v_norms, int kV, int NV, const float* rotV,
                                const float* cbV, float scale, float* out, void* workspace,
                                size_t workspace_bytes, void* stream) {
  AttnArgs a;
  size_t need = 0;
  fq_status st = attn_prepare(q, B, Hq, Hkv, T, d, k_codes, k_norms, kK, NK, rotK, cbK, v_codes,
                              v_norms, kV, NV, rotV, cbV, scale, out, &a, &need);
  if (st != FQ_OK) return st;
  if (T == 0) return FQ_ERR_UNSUPPORTED;  // no slot to append to
  if (!lengths || !k_new || !v_new) return FQ_ERR_INVALID_ARG;
  if (!aligned(lengths, 4) || !aligned(k_new, 2) || !aligned(v_new, 2)) return FQ_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < need) return FQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return FQ_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // the step's own key and value: one record each per (batch, kv head), into slot lengths[b]
  const AppendMap map{lengths, Hkv, T};
  cudaError_t e = launch_encode_generic(k_new, FQ_F16, (int64_t)B * Hkv, a.ks, rotK, cbK, k_codes,
                                        k_norms, nullptr, cs, map);
  if (e != cudaSuccess) return FQ_ERR_CUDA;
  e = launch_encode_generic(v_new, FQ_F16, (int64_t)B * Hkv, a.vs, rotV, cbV, v_codes, v_norms,
                            nullptr, cs, map);
  if (e != cudaSuccess) return FQ_ERR_CUDA;
  a.partials = static_cast<float*>(workspace);
  a.lengths = lengths;
  a.splits = attn_splits(B, Hkv, T, true);
  a.tokens_per_split = attn_tokens_per_split(T, a.splits);
  a.length_bias = 1;
  a.lengths_out = lengths;
  return from_cuda(launch_attn(a, cs));
}

fq_status fq_encode_rho(const void* x, fq_dtype x_type, int64_t n, int d, int k, int N,
                        const float* rot, const float* codebook, uint8_t* codes,
                        uint16_t* norms, uint16_t* rho, const void* search_index, void* stream) {
  Shape s;
  fq_status st = make_shape(d, k, N, &s);
  if (st != FQ_OK) return st;
  if (n < 0 || (x_type != FQ_F16 && x_type != FQ_F32)) return FQ_ERR_INVALID_ARG;
  if (n == 0) return FQ_OK;
  if (!x || !rot || !codebook || !codes || !norms || !rho) return FQ_ERR_INVALID_ARG;
  if (!aligned(x, x_type == FQ_F16 ? 2 : 4) || !aligned(norms, 2) || !aligned(rho, 2) ||
      !aligned(rot, 4) || !aligned(codebook, 4) || (search_index && !aligned(search_index, 8)))
    return FQ_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (sm100::encode_supported(x_type, s, x, codes, norms))
    return from_cuda(sm100::launch_encode(x, x_type, n, s, rot, codebook, codes, norms,
                                          search_index, cs, rho));
  return from_cuda(launch_encode_generic(x, x_type, n, s, rot, codebook, codes, norms,
                                         search_index, cs, AppendMap{nullptr, 1, 0}, rho));
}

fq_status fq_decode_rescaled(const uint8_t* codes, const uint16_t* norms, const uint16_t* rho,
                             int64_t n, int d, int k, int N, const float* rot,
                             const float* codebook, int rule, void* y, fq_dtype y_type,
                             void* stream) {
  Shape s;
  fq_status st = make_shape(d, k, N, &s);
  if (st != FQ_OK) return st;
  if (n < 0 || (y_type != FQ_F16 && y_type != FQ_F32)) return FQ_ERR_INVALID_ARG;
  if (rule != FQ_RESCALE_PLAIN && rule != FQ_RESCALE_MSE && rule != FQ_RESCALE_UNBIASED)
    return FQ_ERR_INVALID_ARG;
  if (n == 0) return FQ_OK;
  if (!codes || !norms || !rho || !rot || !codebook || !y) return FQ_ERR_INVALID_ARG;
  if (!aligned(norms, 2) || !aligned(rho, 2) || !aligned(rot, 4) || !aligned(codebook, 4) ||
      !aligned(y, y_type == FQ_F16 ? 2 : 4))
    return FQ_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (sm100::decode_supported(y_type, s, codes, norms, y))
    return from_cuda(sm100::launch_decode(codes, norms, n, s, rot, codebook, y, y_type, cs, rho,
                                          rule));
  return from_cuda(launch_decode_generic(codes, norms, n, s, rot, codebook, y, y_type, cs,
                                         Gather{nullptr, 0}, Rescale{rho, rule}));
}

static fq_status prod_shape(int d, int N1, int* B1, int* P1) {
  Shape s;
  fq_status st = make_shape(d, 1, N1, &s);
  if (st != FQ_OK) return st;
  if (N1 > 256) return FQ_ERR_UNSUPPORTED;
  *B1 = s.B;
  *P1 = s.P;
  return FQ_OK;
}

fq_status fq_encode_prod(const void* x, fq_dtype x_type, int64_t n, int d, int N1,
                         const float* rot, const float* c1, const float* qjl, uint8_t* codes,
                         uint8_t* signs, uint16_t* norms, uint16_t* gamma, void* stream) {
  int B1 = 0, P1 = 0;
  fq_status st = prod_shape(d, N1, &B1, &P1);
  if (st != FQ_OK) return st;
  if (n < 0 || (x_type != FQ_F16 && x_type != FQ_F32)) return FQ_ERR_INVALID_ARG;
  if (n == 0) return FQ_OK;
  if (!x || !rot || !c1 || !qjl || !codes || !signs || !norms || !gamma)
    return FQ_ERR_INVALID_ARG;
  if (!aligned(x, x_type == FQ_F16 ? 2 : 4) || !aligned(norms, 2) || !aligned(gamma, 2) ||
      !aligned(rot, 4) || !aligned(c1, 4) || !aligned(qjl, 4))
    return FQ_ERR_ALIGNMENT;
  return from_cuda(launch_encode_prod(x, x_type, n, d, N1, B1, P1, rot, c1, qjl, codes, signs,
                                      norms, gamma, static_cast<cudaStream_t>(stream)));
}

fq_status fq_decode_prod(const uint8_t* codes, const uint8_t* signs, const uint16_t* norms,
                         const uint16_t* gamma, int64_t n, int d, int N1, const float* rot,
                         const float* c1, const float* qjl, void* y, fq_dtype y_type,
                         void* stream) {
  int B1 = 0, P1 = 0;
  fq_status st = prod_shape(d, N1, &B1, &P1);
  if (st != FQ_OK) return st;
  if (n < 0 || (y_type != FQ_F16 && y_type != FQ_F32)) return FQ_ERR_INVALID_ARG;
  if (n == 0) return FQ_OK;
  if (!codes || !signs || !norms || !gamma || !rot || !c1 || !qjl || !y)
    return FQ_ERR_INVALID_ARG;
  if (!aligned(norms, 2) || !aligned(gamma, 2) || !aligned(rot, 4) || !aligned(c1, 4) ||
      !aligned(qjl, 4) || !aligned(y, y_type == FQ_F16 ? 2 : 4))
    return FQ_ERR_ALIGNMENT;
  return from_cuda(launch_decode_prod(codes, signs, norms, gamma, n, d, N1, B1, P1, rot, c1, qjl,
                                      y, y_type, static_cast<cudaStream_t>(stream)));
}

fq_status fq_wait_status(unsigned* timed_out, int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FQ_ERR_CUDA;
  unsigned n = 0;
  cudaError_t (*readers[])(bool, unsigned*) = {wait_timeouts_encode, wait_timeouts_encode_large,
                                               wait_timeouts_encode_highk,
                                               wait_timeouts_encode_grid,
                                               wait_timeouts_decode, wait_timeouts_decode_large,
                                               wait_timeouts_attn, wait_timeouts_selftest};
  for (auto rd : readers)
    if (rd(clear != 0, &n) != cudaSuccess) return FQ_ERR_CUDA;
  if (timed_out) *timed_out = n;
  return n ? FQ_ERR_TIMEOUT : FQ_OK;
}

fq_status fq_selftest_wait_timeout(uint32_t polls, void* stream) {
  if (polls < 1 || polls > (1u << 20)) return FQ_ERR_INVALID_ARG;
  return from_cuda(launch_selftest_wait(polls, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
