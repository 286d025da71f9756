// Host-side builder of the grid candidate index used by fq_encode's pruned search.
//
// Block Sphere VQ notes, key design 2 ("Cartesian LUT"): split the k-dimensional block space
// into a grid with L cells per axis, keep a short candidate list per cell, and search only
// that list instead of all N codewords.  Two list rules:
//   FQ_INDEX_TOPC  - the c codewords nearest to the cell centre, as the notes describe
//                    (approximate: a block near a cell edge can have its nearest codeword
//                    outside the list);
//   FQ_INDEX_EXACT - every codeword that is the nearest one for some point of the (slightly
//                    enlarged) cell, so the search returns the brute-force answer.  A codeword
//                    n is listed when (i) its distance to the cell is at most the smallest
//                    farthest-corner distance of any codeword (otherwise another codeword is
//                    closer everywhere in the cell) and (ii) no other codeword is closer than
//                    n at every point of the cell (checked exactly: the difference of squared
//                    distances is linear, so its minimum over the box sits at a corner).
// Grid range: [-R, R]^k with R = max |codeword coordinate| + 3 / sqrt(d'); coordinates
// outside clamp to the edge cells, so the edge cells' boxes extend to the unit-ball bound.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include <cuda_fp16.h>

#include "fq_internal.h"

namespace fq {
namespace {

uint16_t half_bits(float v) {
  const __half h = __float2half_rn(v);
  uint16_t b;
  std::memcpy(&b, &h, 2);
  return b;
}
float half_value(float v) { return __half2float(__float2half_rn(v)); }

// FQ_INDEX_TENSOR: the codebook as tensor-core B-operand tiles (layout: kTensorIndexDataOffset).
fq_status build_tensor_index(const float* cb, const Shape& s, void* index_host,
                             size_t capacity, size_t* bytes) {
  const int k = s.k, N = s.N;
  if (k % 16 != 0 || k > 64) return FQ_ERR_UNSUPPORTED;
  const int ch = k <= 32 ? 256 : 128;
  if (N < ch) return FQ_ERR_UNSUPPORTED;
  const int kop = 3 * k + 16, sbo = kop * 16;
  const size_t chunk_bytes = (size_t)ch * kop * 2;
  const size_t total = kTensorIndexDataOffset + (size_t)(N / ch) * chunk_bytes;
  *bytes = total;
  if (!index_host || capacity < total) return FQ_ERR_WORKSPACE;
  for (size_t i = 0; i < (size_t)N * k; ++i)
    if (!std::isfinite(cb[i])) return FQ_ERR_INVALID_ARG;
  uint8_t* out = static_cast<uint8_t*>(index_host);
  std::memset(out, 0, total);
  IndexHeader hdr;
  std::memset(&hdr, 0, sizeof(hdr));
  hdr.magic = kIndexMagic;
  hdr.version = kIndexVersion;
  hdr.kind = FQ_INDEX_TENSOR;
  hdr.k = k;
  hdr.N = N;
  hdr.dp = s.dp;
  hdr.slots = ch;
  hdr.n_cells = N / ch;
  hdr.entry_bytes = (int32_t)chunk_bytes;
  hdr.cells_offset = kTensorIndexDataOffset;
  hdr.id_bytes = (uint16_t)kop;
  std::memcpy(out, &hdr, sizeof(hdr));
  std::vector<float> row(kop);
  for (int n = 0; n < N; ++n) {
    double cc = 0;
    for (int a = 0; a < k; ++a) cc += (double)cb[(size_t)n * k + a] * cb[(size_t)n * k + a];
    for (int a = 0; a < k; ++a) {
      const float av = -2.0f * cb[(size_t)n * k + a];
      const float hi = half_value(av);
      row[a] = hi;
      row[k + a] = av - hi;   // rounded to fp16 below
      row[2 * k + a] = hi;
    }
    const float ccf = (float)cc;
    row[3 * k] = half_value(ccf);
    row[3 * k + 1] = ccf - half_value(ccf);
    for (int e = 3 * k + 2; e < kop; ++e) row[e] = 0.f;
    uint8_t* base = out + kTensorIndexDataOffset + (size_t)(n / ch) * chunk_bytes;
    const int r = n % ch;
    for (int e = 0; e < kop; ++e) {
      const uint16_t b = half_bits(row[e]);
      std::memcpy(base + (size_t)(r / 8) * sbo + (e / 8) * 128 + (r % 8) * 16 + (e % 8) * 2, &b, 2);
    }
  }
  return FQ_OK;
}

struct Grid {
  int k, N, L, dp, n_cells;
  double R, h;      // as defined by the rule (float64)
  float lo_f, inv_h_f;  // what the device uses
  double h_dev;     // cell width the device's fp32 mapping implies
};

void cell_box(const Grid& g, int flat, double* lo, double* hi) {
  const double margin = 1e-3 * g.h_dev + 1e-6;
  for (int a = 0; a < g.k; ++a) {
    int i = flat % g.L;
    flat /= g.L;
    double l = (double)g.lo_f + i * g.h_dev - margin;
    double u = (double)g.lo_f + (i + 1) * g.h_dev + margin;
    if (i == 0) l = std::min(l, -1.001);
    if (i == g.L - 1) u = std::max(u, 1.001);
    lo[a] = l;
    hi[a] = u;
  }
}

// Candidates of one cell under the exact rule, sorted by (distance to the box, index).
void exact_candidates(const Grid& g, const double* C, const double* cc, int flat,
                      std::vector<int>& out) {
  double lo[kMaxK], hi[kMaxK];
  cell_box(g, flat, lo, hi);
  const int N = g.N, k = g.k;
  std::vector<double> dmin(N);
  double thr = INFINITY;
  for (int n = 0; n < N; ++n) {
    double mn = 0, mx = 0;
    for (int a = 0; a < k; ++a) {
      double c = C[(size_t)n * k + a];
      double t = c < lo[a] ? lo[a] - c : (c > hi[a] ? c - hi[a] : 0.0);
      mn += t * t;
      double f = std::max(std::fabs(c - lo[a]), std::fabs(c - hi[a]));
      mx += f * f;
    }
    dmin[n] = mn;
    thr = std::min(thr, mx);
  }
  std::vector<int> cand;
  for (int n = 0; n < N; ++n)
    if (dmin[n] <= thr * (1.0 + 1e-12) + 1e-15) cand.push_back(n);
  // pairwise dominance: m dominates n on the box if |p-c_n|^2 - |p-c_m|^2 > 0 for all p
  out.clear();
  for (int n : cand) {
    bool dominated = false;
    for (int mm : cand) {
      if (mm == n) continue;
      double f = cc[n] - cc[mm];
      for (int a = 0; a < k; ++a) {
        double dl = C[(size_t)mm * k + a] - C[(size_t)n * k + a];
        f += 2.0 * std::min(lo[a] * dl, hi[a] * dl);
      }
      if (f > 1e-12) {
        dominated = true;
        break;
      }
    }
    if (!dominated) out.push_back(n);
  }
  std::sort(out.begin(), out.end());  // by index: a strict-less scan keeps the lowest on ties
}

void topc_candidates(const Grid& g, const double* C, int flat, int c, std::vector<int>& out) {
  double centre[kMaxK];
  for (int a = 0; a < g.k; ++a) {
    int i = flat % g.L;
    flat /= g.L;
    centre[a] = -g.R + (i + 0.5) * g.h;
  }
  std::vector<std::pair<double, int>> dist(g.N);
  for (int n = 0; n < g.N; ++n) {
    double s = 0;
    for (int a = 0; a < g.k; ++a) {
      double t = centre[a] - C[(size_t)n * g.k + a];
      s += t * t;
    }
    dist[n] = {s, n};
  }
  std::partial_sort(dist.begin(), dist.begin() + c, dist.end());
  out.resize(c);
  for (int i = 0; i < c; ++i) out[i] = dist[i].second;
  std::sort(out.begin(), out.end());
}

}  // namespace
}  // namespace fq

using namespace fq;

extern "C" fq_status fq_build_search_index(const float* codebook_host, int d, int k, int N,
                                           int kind, int L, int c, void* index_host,
                                           size_t index_capacity, size_t* index_bytes) {
  Shape s;
  fq_status st = make_shape(d, k, N, &s);
  if (st != FQ_OK) return st;
  if (!codebook_host || !index_bytes) return FQ_ERR_INVALID_ARG;
  if (kind == FQ_INDEX_TENSOR)
    return build_tensor_index(codebook_host, s, index_host, index_capacity, index_bytes);
  if (kind != FQ_INDEX_EXACT && kind != FQ_INDEX_TOPC) return FQ_ERR_INVALID_ARG;
  if (L < 2 || L > 256) return FQ_ERR_UNSUPPORTED;
  double cells_d = std::pow((double)L, k);
  if (cells_d > (double)(1 << 22)) return FQ_ERR_UNSUPPORTED;
  if (c < 1 || c > 64 || (kind == FQ_INDEX_TOPC && c > N)) return FQ_ERR_UNSUPPORTED;

  Grid g;
  g.k = k;
  g.N = N;
  g.L = L;
  g.dp = s.dp;
  g.n_cells = (int)cells_d;
  std::vector<double> C((size_t)N * k), cc(N);
  double maxabs = 0;
  for (int n = 0; n < N; ++n) {
    double sq = 0;
    for (int a = 0; a < k; ++a) {
      double v = codebook_host[(size_t)n * k + a];
      if (!std::isfinite(v)) return FQ_ERR_INVALID_ARG;
      C[(size_t)n * k + a] = v;
      sq += v * v;
      maxabs = std::max(maxabs, std::fabs(v));
    }
    cc[n] = sq;
  }
  g.R = maxabs + 3.0 / std::sqrt((double)s.dp);
  g.h = 2.0 * g.R / L;
  g.lo_f = (float)(-g.R);
  g.inv_h_f = (float)(1.0 / g.h);
  g.h_dev = 1.0 / (double)g.inv_h_f;

  const int slots = c;
  std::vector<std::vector<int>> lists(g.n_cells);
  unsigned nth = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
  std::vector<std::thread> pool;
  for (unsigned t = 0; t < nth; ++t) {
    pool.emplace_back([&, t]() {
      std::vector<int> tmp;
      for (int f = (int)t; f < g.n_cells; f += (int)nth) {
        if (kind == FQ_INDEX_EXACT)
          exact_candidates(g, C.data(), cc.data(), f, tmp);
        else
          topc_candidates(g, C.data(), f, c, tmp);
        lists[f] = tmp;
      }
    });
  }
  for (auto& th : pool) th.join();

  const int id_bytes = N <= 256 ? 1 : 2;
  size_t ov_elems = 0;
  uint32_t max_cand = 0;
  for (auto& l : lists) {
    if (l.empty()) return FQ_ERR_INVALID_ARG;  // cannot happen: the nearest codeword survives
    if ((int)l.size() > slots) ov_elems += 1 + (l.size() - slots);
    max_cand = std::max<uint32_t>(max_cand, (uint32_t)l.size());
  }
  if (max_cand > 65535) return FQ_ERR_UNSUPPORTED;
  const bool overflow = kind == FQ_INDEX_EXACT && (int)max_cand > slots;
  const int ids_bytes = ((slots * id_bytes + 3) / 4) * 4;
  const int entry_bytes = ids_bytes + (overflow ? 4 : 0);
  const size_t cells_off = sizeof(IndexHeader);
  size_t ov_off = cells_off + (size_t)g.n_cells * entry_bytes;
  ov_off = (ov_off + 7) & ~size_t(7);
  size_t total = ov_off + ov_elems * 2;
  total = (total + 7) & ~size_t(7);
  if (total > 0xFFFFFFFFull) return FQ_ERR_UNSUPPORTED;
  *index_bytes = total;
  if (!index_host || index_capacity < total) return FQ_ERR_WORKSPACE;

  uint8_t* out = static_cast<uint8_t*>(index_host);
  std::memset(out, 0, total);
  IndexHeader hdr;
  hdr.magic = kIndexMagic;
  hdr.version = kIndexVersion;
  hdr.kind = kind;
  hdr.k = k;
  hdr.N = N;
  hdr.L = L;
  hdr.dp = s.dp;
  hdr.slots = slots;
  hdr.lo = g.lo_f;
  hdr.inv_h = g.inv_h_f;
  hdr.n_cells = g.n_cells;
  hdr.entry_bytes = entry_bytes;
  hdr.cells_offset = (uint32_t)cells_off;
  hdr.overflow_offset = (uint32_t)ov_off;
  hdr.overflow_elems = (uint32_t)ov_elems;
  hdr.max_candidates = (uint16_t)max_cand;
  hdr.id_bytes = (uint16_t)id_bytes;
  std::memcpy(out, &hdr, sizeof(hdr));
  uint16_t* ovl = reinterpret_cast<uint16_t*>(out + ov_off);
  size_t ov_pos = 0;
  for (int f = 0; f < g.n_cells; ++f) {
    const auto& l = lists[f];
    uint8_t* e = out + cells_off + (size_t)f * entry_bytes;
    const int pad_slots = ids_bytes / id_bytes;  // pad the whole id area with the last id
    for (int i = 0; i < pad_slots; ++i) {
      int id = l[std::min<int>(std::min(i, slots - 1), (int)l.size() - 1)];
      if (id_bytes == 1)
        e[i] = (uint8_t)id;
      else
        reinterpret_cast<uint16_t*>(e)[i] = (uint16_t)id;
    }
    if (overflow) {
      uint32_t w = kNoOverflow;
      if ((int)l.size() > slots) {
        w = (uint32_t)ov_pos;
        ovl[ov_pos++] = (uint16_t)(l.size() - slots);
        for (size_t i = slots; i < l.size(); ++i) ovl[ov_pos++] = (uint16_t)l[i];
      }
      std::memcpy(e + ids_bytes, &w, 4);
    }
  }
  return FQ_OK;
}
