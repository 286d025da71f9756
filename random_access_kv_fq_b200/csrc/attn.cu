// Fused decode attention over a FibQuant-compressed KV cache.
//
// The FibQuant summary (sec. 5, "system compatibility") notes that the fixed-address records
// keep decompression fusable into the attention kernel.  The form computed here:
//   q~_h = Pi_K pad(q_h)                           (query rotated once per head)
//   LUT_h[j][c] = q~_h[jk:(j+1)k] . C_K[c]           (per-block dot-product tables)
//   s_ht = scale * nu^K_t * sum_j LUT_h[j][idx^K_tj] (scores straight from the key codes)
//   acc_h = sum_t softmax(s)_ht nu^V_t zhat^V_t      (values accumulated in the rotated domain)
//   out_h = (Pi_V^T acc_h)[0:d]                      (inverse rotation once per head)
// which equals softmax(q khat^T scale) vhat with khat, vhat the decoded caches.
//
// Work split: one CTA per (batch, kv head, context split) runs the online softmax over its
// token range for all Hq/Hkv query heads of the group and writes (max, sum, acc[d'_V]) per
// head; a second kernel merges the splits (flash-decoding style) and applies Pi_V^T.
#include <cuda_fp16.h>

#include "fq_device.cuh"
#include "fq_internal.h"

namespace fq {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;       // tokens per tile
constexpr int kAccPer = 9;      // accumulator entries per thread: 16 heads * 135 / 256
constexpr int kMaxGroup = 16;
// Context splits: one wave of the tensor-core kernel (three 128-token-tile CTAs per SM on the
// 148 SMs of a B200), split lengths a multiple of 128 tokens.
constexpr int kTargetCtas = 148 * 3;
constexpr int kSplitGrain = 128;

struct SmemLayout {
  int qt, lut, cv, S, kid, vid, kn, vn, alpha, mrun, lrun, total;  // float offsets
};

__host__ __device__ inline SmemLayout smem_layout(int G, const Shape& ks, const Shape& vs) {
  SmemLayout L;
  int o = 0;
  L.qt = o;    o += G * ks.dp;
  L.lut = o;   o += G * ks.m * ks.N;
  L.cv = o;    o += vs.N * vs.k;
  L.S = o;     o += G * kTile;
  L.kid = o;   o += kTile * (ks.m + 1);
  L.vid = o;   o += kTile * (vs.m + 1);
  L.kn = o;    o += kTile;
  L.vn = o;    o += kTile;
  L.alpha = o; o += kMaxGroup;
  L.mrun = o;  o += kMaxGroup;
  L.lrun = o;  o += kMaxGroup;
  L.total = o;
  return L;
}

__global__ void __launch_bounds__(kThreads) attn_partial_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  const int G = a.Hq / a.Hkv;
  const Shape ks = a.ks, vs = a.vs;
  const SmemLayout L = smem_layout(G, ks, vs);
  float* qt = sm + L.qt;
  float* lut = sm + L.lut;
  float* cv = sm + L.cv;
  float* S = sm + L.S;
  int* kid = reinterpret_cast<int*>(sm + L.kid);
  int* vid = reinterpret_cast<int*>(sm + L.vid);
  float* kn = sm + L.kn;
  float* vn = sm + L.vn;
  float* alpha = sm + L.alpha;
  float* mrun = sm + L.mrun;
  float* lrun = sm + L.lrun;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int64_t t_begin = (int64_t)split * a.tokens_per_split;
  int64_t t_end = t_begin + a.tokens_per_split;
  const int64_t len_b = attn_seq_len(a, b);  // a split past the sequence's end stays empty
  if (t_end > len_b) t_end = len_b;

  // rotate the group's queries once: q~_h = Pi_K pad(q_h)
  for (int e = tid; e < G * ks.dp; e += kThreads) {
    int h = e / ks.dp, r = e % ks.dp;
    const uint16_t* qh = a.q + ((size_t)b * a.Hq + (size_t)g * G + h) * a.d;
    const float* pr = a.rotK + (size_t)r * ks.dp;
    float acc = 0.f;
    for (int c = 0; c < a.d; ++c) acc = fmaf(__ldg(pr + c), f16_bits_to_f32(qh[c]), acc);
    qt[e] = acc;
  }
  for (int e = tid; e < vs.N * vs.k; e += kThreads) cv[e] = __ldg(a.cbV + e);
  if (tid < kMaxGroup) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.f;
  }
  __syncthreads();
  // per-block dot-product tables LUT_h[j][c]
  for (int e = tid; e < G * ks.m * ks.N; e += kThreads) {
    int c = e % ks.N;
    int hj = e / ks.N;
    int j = hj % ks.m, h = hj / ks.m;
    const float* qb = qt + h * ks.dp + j * ks.k;
    float acc = 0.f;
    for (int r = 0; r < ks.k; ++r) acc = fmaf(qb[r], __ldg(a.cbK + (size_t)c * ks.k + r), acc);
    lut[e] = acc;
  }

  float acc[kAccPer];
#pragma unroll
  for (int i = 0; i < kAccPer; ++i) acc[i] = 0.f;
  const int n_acc = G * vs.dp;

  const size_t kv_base = ((size_t)b * a.Hkv + g) * (size_t)a.T;
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int nt = (int)((t_end - t0) < kTile ? (t_end - t0) : kTile);
    __syncthreads();  // previous tile fully consumed (and LUT ready on the first pass)
    // norms and unpacked indices of the tile
    for (int t = tid; t < kTile; t += kThreads) {
      kn[t] = (t < nt) ? f16_bits_to_f32(a.k_norms[kv_base + t0 + t]) : 0.f;
      vn[t] = (t < nt) ? f16_bits_to_f32(a.v_norms[kv_base + t0 + t]) : 0.f;
    }
    for (int e = tid; e < nt * ks.m; e += kThreads) {
      int t = e / ks.m, j = e % ks.m;
      kid[t * (ks.m + 1) + j] = record_index(a.k_codes + (kv_base + t0 + t) * ks.P, j, ks.B);
    }
    for (int e = tid; e < nt * vs.m; e += kThreads) {
      int t = e / vs.m, j = e % vs.m;
      vid[t * (vs.m + 1) + j] = record_index(a.v_codes + (kv_base + t0 + t) * vs.P, j, vs.B);
    }
    __syncthreads();
    // scores from the key codes through the tables
    for (int e = tid; e < G * kTile; e += kThreads) {
      int h = e / kTile, t = e % kTile;
      float s = -INFINITY;
      if (t < nt) {
        const float* lh = lut + (size_t)h * ks.m * ks.N;
        const int* kr = kid + t * (ks.m + 1);
        float sum = 0.f;
        for (int j = 0; j < ks.m; ++j) sum += lh[j * ks.N + kr[j]];
        s = sum * kn[t] * a.scale;
      }
      S[h * kTile + t] = s;
    }
    __syncthreads();
    // online softmax update, one warp per head
    {
      const int warp = tid >> 5, lane = tid & 31;
      for (int h = warp; h < G; h += kThreads / 32) {
        float mx = -INFINITY;
        for (int t = lane; t < kTile; t += 32) mx = fmaxf(mx, S[h * kTile + t]);
        mx = warp_max(mx);
        const float mnew = fmaxf(mrun[h], mx);
        float psum = 0.f;
        for (int t = lane; t < kTile; t += 32) {
          float p = (t < nt) ? __expf(S[h * kTile + t] - mnew) : 0.f;
          psum += p;
          S[h * kTile + t] = p * vn[t];  // weight of zhat^V_t
        }
        psum = warp_sum(psum);
        if (lane == 0) {
          float al = __expf(mrun[h] - mnew);
          alpha[h] = al;
          lrun[h] = lrun[h] * al + psum;
          mrun[h] = mnew;
        }
      }
    }
    __syncthreads();
    // values: acc_h[r] = alpha_h acc_h[r] + sum_t w_ht C_V[idx^V_t,block(r)][r % k]
#pragma unroll
    for (int i = 0; i < kAccPer; ++i) {
      int e = tid + i * kThreads;
      if (e < n_acc) {
        int h = e / vs.dp, r = e % vs.dp;
        int j = r / vs.k, comp = r % vs.k;
        float v = acc[i] * alpha[h];
        const float* wh = S + h * kTile;
        for (int t = 0; t < nt; ++t) v = fmaf(wh[t], cv[vid[t * (vs.m + 1) + j] * vs.k + comp], v);
        acc[i] = v;
      }
    }
  }
  __syncthreads();
  // write this split's partials
  const int dpv2 = vs.dp + 2;
#pragma unroll
  for (int i = 0; i < kAccPer; ++i) {
    int e = tid + i * kThreads;
    if (e < n_acc) {
      int h = e / vs.dp, r = e % vs.dp;
      size_t base = (((size_t)b * a.Hq + (size_t)g * G + h) * a.splits + split) * dpv2;
      a.partials[base + 2 + r] = acc[i];
    }
  }
  if (tid < G) {
    size_t base = (((size_t)b * a.Hq + (size_t)g * G + tid) * a.splits + split) * dpv2;
    a.partials[base] = mrun[tid];
    a.partials[base + 1] = lrun[tid];
  }
}

__global__ void __launch_bounds__(128) attn_combine_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, b = blockIdx.y;
  const int dpv = a.vs.dp, dpv2 = dpv + 2;
  float* accr = sm;  // [dpv]
  __shared__ float red[2];
  const float* base = a.partials + ((size_t)b * a.Hq + h) * a.splits * (size_t)dpv2;
  if (threadIdx.x < 32) {
    float mx = -INFINITY;
    for (int s = threadIdx.x; s < a.splits; s += 32) mx = fmaxf(mx, base[(size_t)s * dpv2]);
    mx = warp_max(mx);
    float l = 0.f;
    for (int s = threadIdx.x; s < a.splits; s += 32) {
      float ms = base[(size_t)s * dpv2];
      if (ms > -INFINITY) l += base[(size_t)s * dpv2 + 1] * __expf(ms - mx);
    }
    l = warp_sum(l);
    if (threadIdx.x == 0) {
      red[0] = mx;
      red[1] = l;
    }
  }
  __syncthreads();
  // an empty sequence (every split empty: l = 0) attends to nothing and outputs zero
  const float mx = red[0], inv_l = red[1] > 0.f ? 1.f / red[1] : 0.f;
  for (int r = threadIdx.x; r < dpv; r += blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < a.splits; ++s) {
      float ms = base[(size_t)s * dpv2];
      if (ms > -INFINITY) v = fmaf(base[(size_t)s * dpv2 + 2 + r], __expf(ms - mx), v);
    }
    accr[r] = v * inv_l;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < a.d; c += blockDim.x) {
    float v = 0.f;
    for (int r = 0; r < dpv; ++r) v = fmaf(__ldg(a.rotV + (size_t)r * dpv + c), accr[r], v);
    a.out[((size_t)b * a.Hq + h) * a.d + c] = v;
  }
  // the step that appended its own token advances its sequence (after every read of lengths)
  if (a.lengths_out != nullptr && h == 0 && threadIdx.x == 0) {
    const int32_t L = a.lengths_out[b];
    if (L >= 0 && L < a.T) a.lengths_out[b] = L + 1;
  }
}

}  // namespace

int attn_splits(int B, int Hkv, int64_t T, bool ragged) {
  int64_t pairs = (int64_t)B * Hkv;
  // With per-sequence lengths the splits past a sequence's end exit at once and the step lasts
  // as long as the busiest split: twice as many, half as long.
  int64_t want = (ragged ? 2 * kTargetCtas : kTargetCtas) / pairs;
  int64_t tiles = (T + kSplitGrain - 1) / kSplitGrain;
  if (want > tiles) want = tiles;
  if (want < 1) want = 1;
  if (want > 4096) want = 4096;
  int64_t tps = attn_tokens_per_split(T, (int)want);
  return (int)((T + tps - 1) / tps);
}

int64_t attn_tokens_per_split(int64_t T, int splits) {
  int64_t tps = (T + splits - 1) / splits;
  return ((tps + kSplitGrain - 1) / kSplitGrain) * kSplitGrain;
}

size_t attn_partials_bytes(int B, int Hq, int splits, int dpV) {
  return (size_t)B * Hq * splits * (size_t)(dpV + 2) * sizeof(float);
}

size_t attn_smem_bytes(const AttnArgs& a) {
  return (size_t)smem_layout(a.Hq / a.Hkv, a.ks, a.vs).total * sizeof(float);
}

cudaError_t launch_attn_combine(const AttnArgs& a, cudaStream_t st) {
  attn_combine_kernel<<<dim3(a.Hq, a.B), 128, a.vs.dp * sizeof(float), st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  if (attn100::supported(a)) return attn100::launch(a, st);
  size_t smem = attn_smem_bytes(a);
  cudaError_t e = cudaFuncSetAttribute(attn_partial_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.splits, a.Hkv, a.B);
  attn_partial_kernel<<<grid, kThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_combine(a, st);
}

}  // namespace fq
