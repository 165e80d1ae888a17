// mask.cu -- block scoring and Top-p / Top-k routing (FVAttn: Adaptive Sparse
// Attention with Runtime Load Balancing for Video Generation, abstract:
// "Top-p routing, a Top-k safety floor"), plus the longest-first work order
// that absorbs the uneven per-head workloads the abstract describes.
//
// Launches on the caller's stream:
//   pool_kernel        mean of the real tokens of every block of qt and kt
//                      (summed in fp64). HBM-bound: reads qt and kt once.
//   score_kernel       pooled scores Qbar_i . Kbar_j / sqrt(d) in fp64 for a
//                      chunk of heads (64 x 64 tiles, fp64 FMA on CUDA cores)
//                      into a scratch that stays in L2 until:
//   cut_kernel         one warp per row: fp64 row softmax over the key
//                      blocks, the Top-p cut by bisection on the probability
//                      bits (no sort) with the Top-k floor; writes the bitmask
//                      row and row_cnt. (score, cut) repeat per chunk of heads.
//   head_scan_kernel   one warp per head: row_ptr within the head, the head's
//                      longest-first order (stable counting sort, so the
//                      result is deterministic) and total; the last CTA orders
//                      the heads and offsets them.
//   finalize_kernel    one warp per row: global row_ptr, the work_order entry
//                      and the ascending col_idx from the bitmask.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace sba {

namespace {

// ------------------------------------------------------------------ pooling

template <typename T>
__device__ __forceinline__ void accum_vec(double* acc, const uint4& v);

template <>
__device__ __forceinline__ void accum_vec<__nv_bfloat16>(double* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // bf16 -> fp32 is a shift (exact), fp32 -> fp64 exact
    acc[2 * i] += static_cast<double>(__uint_as_float(w[i] << 16));
    acc[2 * i + 1] += static_cast<double>(__uint_as_float(w[i] & 0xFFFF0000u));
  }
}

template <>
__device__ __forceinline__ void accum_vec<float>(double* acc, const uint4& v) {
  acc[0] += static_cast<double>(__uint_as_float(v.x));
  acc[1] += static_cast<double>(__uint_as_float(v.y));
  acc[2] += static_cast<double>(__uint_as_float(v.z));
  acc[3] += static_cast<double>(__uint_as_float(v.w));
}

// One warp per (tensor, b*h, block): z = 0 pools qt, z = 1 pools kt. Lane l
// owns the 16-byte column vector l % vpr of the rows l / vpr, l / vpr + 32/vpr,
// ... (a warp instruction reads 512 contiguous bytes), four loads in flight;
// the row groups are combined with shuffles. Sums in fp64 (a sum of bf16 or
// fp32 values is exact there for any realistic spread of exponents), one
// division by the number of real tokens. No shared memory, no block barrier.
constexpr int kPoolWarps = 8;
constexpr int kPoolUnroll = 4;

template <typename T>
__global__ void __launch_bounds__(kPoolWarps * 32)
    pool_kernel(KGeom g, const char* __restrict__ qt, const char* __restrict__ kt,
                double* __restrict__ qbar, double* __restrict__ kbar) {
  constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
  const int lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * kPoolWarps + (threadIdx.x >> 5);
  const int64_t per_tensor = static_cast<int64_t>(g.B) * g.H * g.nb;
  if (item >= 2 * per_tensor) return;
  const int z = item >= per_tensor ? 1 : 0;
  const int64_t bj = item - z * per_tensor;  // (b*H + h) * nb + j
  const int j = static_cast<int>(bj % g.nb);
  const int64_t bh = bj / g.nb;
  const char* src = z == 0 ? qt : kt;
  double* dst = z == 0 ? qbar : kbar;
  const int vpr = g.d / EPV;  // vectors per row: 8, 16 or 32
  const int rpi = 32 / vpr;   // rows per warp instruction
  const int c = lane % vpr, rsub = lane / vpr;
  // the block's real tokens occupy its first len slots (both orders)
  const int len = block_len(g, j);
  const int64_t row_bytes = static_cast<int64_t>(g.d) * sizeof(T);
  const char* base = src + (bh * g.Npad + static_cast<int64_t>(j) * g.bs) * row_bytes + c * 16;
  double acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.0;
  for (int o0 = rsub; o0 < len; o0 += rpi * kPoolUnroll) {
    uint4 v[kPoolUnroll];
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u) {
      const int o = o0 + u * rpi;
      if (o < len) v[u] = __ldg(reinterpret_cast<const uint4*>(base + o * row_bytes));
    }
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u)
      if (o0 + u * rpi < len) accum_vec<T>(acc, v[u]);
  }
  for (int off = vpr; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (rsub == 0) {
    const double dlen = static_cast<double>(len);
    double* out = dst + bj * g.d + c * EPV;
#pragma unroll
    for (int e = 0; e < EPV; ++e) out[e] = acc[e] / dlen;
  }
}

// ---------------------------------------------------------- score + select
// All of it in fp64, so that the routing decision is the exact one except
// where the cumulative mass at the cut lies within rounding of p.
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

struct SelectArgs {
  float top_p[256];
};

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// (one warp-wide reduction instruction)
__device__ __forceinline__ int warp_sum_int(int v) { return __reduce_add_sync(0xffffffffu, v); }

// Pooled scores of a chunk of heads: S[bh - h0][i][j] = (Qbar_i . Kbar_j) / sqrt(d)
// in fp64, each product summed over c = 0 .. d-1 in order. A CTA computes a
// 64 x 64 tile of one head (thread: 4 x 4 outputs), with 16-column slices of
// the two operands staged transposed in shared memory (prefetching the next
// slice into registers measured slower: it cost a resident CTA per SM).
// grid (ceil(nb/64), ceil(nb/64), heads in the chunk).
constexpr int kScoreTile = 64;
constexpr int kScoreK = 16;

__global__ void __launch_bounds__(256)
    score_kernel(KGeom g, int h0, const double* __restrict__ qbar, const double* __restrict__ kbar,
                 double* __restrict__ S) {
  // one padding double per row spreads the transposed stores of a warp (8 rows
  // x 4 columns) over more banks
  __shared__ double qs[kScoreK][kScoreTile + 1];
  __shared__ double ks[kScoreK][kScoreTile + 1];
  const int d = g.d, nb = g.nb;
  const int bh = h0 + static_cast<int>(blockIdx.z);
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const double* qsrc = qbar + static_cast<int64_t>(bh) * nb * d;
  const double* ksrc = kbar + static_cast<int64_t>(bh) * nb * d;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
  // loader: thread -> (row lr, 4 columns lc..lc+3) of a 64 x 16 slice
  const int lr = tid >> 2, lc = (tid & 3) * 4;
  const int iq = i0 + lr, jk = j0 + lr;
  for (int c0 = 0; c0 < d; c0 += kScoreK) {
    __syncthreads();
    {
      double2 q01 = make_double2(0.0, 0.0), q23 = q01, k01 = q01, k23 = q01;
      if (iq < nb) {
        const double2* src = reinterpret_cast<const double2*>(qsrc + static_cast<int64_t>(iq) * d + c0 + lc);
        q01 = __ldg(src);
        q23 = __ldg(src + 1);
      }
      if (jk < nb) {
        const double2* src = reinterpret_cast<const double2*>(ksrc + static_cast<int64_t>(jk) * d + c0 + lc);
        k01 = __ldg(src);
        k23 = __ldg(src + 1);
      }
      qs[lc + 0][lr] = q01.x;
      qs[lc + 1][lr] = q01.y;
      qs[lc + 2][lr] = q23.x;
      qs[lc + 3][lr] = q23.y;
      ks[lc + 0][lr] = k01.x;
      ks[lc + 1][lr] = k01.y;
      ks[lc + 2][lr] = k23.x;
      ks[lc + 3][lr] = k23.y;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kScoreK; ++c) {
      // rows ty + 16a, columns tx + 16b: a half-warp reads 16 consecutive
      // doubles of ks (one wavefront) and a broadcast of qs
      double qv[4], kv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qv[a] = qs[c][ty + 16 * a];
#pragma unroll
      for (int b = 0; b < 4; ++b) kv[b] = ks[c][tx + 16 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fma(qv[a], kv[b], acc[a][b]);
    }
  }
  const double sqrt_d = sqrt(static_cast<double>(d));
  double* dst = S + static_cast<int64_t>(blockIdx.z) * nb * nb;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i >= nb) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + tx + 16 * b;
      if (j < nb) dst[static_cast<int64_t>(i) * nb + j] = acc[a][b] / sqrt_d;
    }
  }
}

// One warp per (head, query block) row of the chunk: the row's pooled scores
// (from score_kernel) -> fp64 softmax over the key blocks, then the cut: the
// largest probability v with mass(P >= v) >= p found by bisection on the bit
// pattern of v (warp mass sums), the ties of v taken in index order until the
// mass reaches p; the Top-k floor by the same bisection on counts. No sort.
// Writes the row's bitmask words and row_cnt. grid ceil(rows of chunk / 8).
// KE: probabilities per lane (the smallest of 8, 16, 32 with 32*KE >= nb).
template <int KE>
__global__ void __launch_bounds__(kSelThreads)
    cut_kernel(KGeom g, int h0, int nheads, const double* __restrict__ S, SelectArgs sa, int top_k,
               uint32_t* __restrict__ bitmask, int32_t* __restrict__ row_cnt) {
  const int nb = g.nb;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rloc = blockIdx.x * kSelWarps + warp;  // row within the chunk
  if (rloc >= nheads * nb) return;
  const int bh = h0 + rloc / nb;
  const int i = rloc % nb;
  const double* srow = S + static_cast<int64_t>(rloc) * nb;
  __shared__ double cbuf_all[kSelWarps][32];
  double* cbuf = cbuf_all[warp];
  uint32_t h;
  {
    uint32_t bq;
    g.dv_H.divmod(static_cast<uint32_t>(bh), bq, h);
  }
  const double p = static_cast<double>(sa.top_p[h]);
  const int E = (nb + 31) >> 5;
  {
    // softmax in fp64: shift by the row max, exp, divide by the sum
    double pv[KE];
    double mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < KE; ++e) {
      const int j = lane + 32 * e;
      pv[e] = (e < E && j < nb) ? __ldcg(srow + j) : -INFINITY;
      mx = fmax(mx, pv[e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    double esum = 0.0;
#pragma unroll
    for (int e = 0; e < KE; ++e) {
      const int j = lane + 32 * e;
      pv[e] = (e < E && j < nb) ? exp(pv[e] - mx) : 0.0;
      esum += pv[e];
    }
    esum = warp_sum(esum);
    const double inv = 1.0 / esum;  // one division per row
#pragma unroll
    for (int e = 0; e < KE; ++e) {
      const int j = lane + 32 * e;
      pv[e] = (e < E && j < nb) ? pv[e] * inv : -1.0;  // -1: not a key block
    }
    // mass and count of the row's probabilities >= v (the -1 entries never
    // pass: every v tried is a non-negative double, bit 62 of its pattern
    // being clear)
    auto ge_sums = [&](double v, double& m, int& c) {
      double mm = 0.0;
      int cc = 0;
#pragma unroll
      for (int e = 0; e < KE; ++e)
        if (e < E && pv[e] >= v) {
          mm += pv[e];
          ++cc;
        }
      m = warp_sum(mm);
      c = warp_sum_int(cc);
    };
    // the same for a threshold whose low 32 bits are zero: the comparison of
    // two non-negative doubles is that of their bit patterns, so the high
    // words decide it (an integer compare; the -1 entries are negative)
    auto ge_sums_hi = [&](int vhi, double& m, int& c) {
      double mm = 0.0;
      int cc = 0;
#pragma unroll
      for (int e = 0; e < KE; ++e)
        if (e < E && __double2hiint(pv[e]) >= vhi) {
          mm += pv[e];
          ++cc;
        }
      m = warp_sum(mm);
      c = warp_sum_int(cc);
    };
    auto as_double = [](unsigned long long b) { return __longlong_as_double(static_cast<long long>(b)); };
    // The single probability in [lo, hi) (bit patterns), found once the
    // bisection interval holds exactly one element.
    auto only_in = [&](unsigned long long lo, unsigned long long hi) -> unsigned long long {
      double f = -1.0;
      const double a = as_double(lo), b = as_double(hi);
#pragma unroll
      for (int e = 0; e < KE; ++e)
        if (e < E && pv[e] >= a && pv[e] < b) f = pv[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) f = fmax(f, __shfl_xor_sync(0xffffffffu, f, o));
      return static_cast<unsigned long long>(__double_as_longlong(f));
    };
    // Bisection over bit patterns for the largest element v with
    // pred(mass(P >= v), count(P >= v)). Invariant: pred holds at lo and fails
    // at hi, so the answer lies in [lo, hi); stop once one element is left
    // there (or the interval is one pattern wide).
    // Once at most 32 elements are left in [lo, hi) they are gathered one per
    // lane (through this warp's slice of shared memory) and the remaining
    // steps sum only them on top of the mass and count at hi.
    // the row's smallest and largest probability, as bit patterns
    unsigned long long pat_min, pat_max;
    {
      double pmin = 2.0, pmax = 0.0;
#pragma unroll
      for (int e = 0; e < KE; ++e)
        if (e < E && pv[e] >= 0.0) {
          pmin = fmin(pmin, pv[e]);
          pmax = fmax(pmax, pv[e]);
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        pmin = fmin(pmin, __shfl_xor_sync(0xffffffffu, pmin, o));
        pmax = fmax(pmax, __shfl_xor_sync(0xffffffffu, pmax, o));
      }
      pat_min = static_cast<unsigned long long>(__double_as_longlong(pmin));
      pat_max = static_cast<unsigned long long>(__double_as_longlong(pmax));
    }
    double total;
    int cnt_all;
    ge_sums(0.0, total, cnt_all);
    auto bisect = [&](bool by_mass, double p_or_n) -> unsigned long long {
      // start from the row's own range: lo = the common bit prefix of its
      // smallest and largest probability (every element is >= lo), hi = lo
      // plus one unit of the highest bit where they differ (> the largest)
      const unsigned long long diff = pat_min ^ pat_max;
      int b = diff ? 63 - __clzll(static_cast<long long>(diff)) : -1;
      const unsigned long long span = b >= 0 ? (1ull << (b + 1)) : 1ull;
      unsigned long long lo = pat_min & ~(span - 1ull), hi = lo + span;
      double m, m_hi = 0.0;
      int c_lo = cnt_all, c_hi = 0;
      for (; b >= 0 && c_lo - c_hi > 32; --b) {
        const unsigned long long mid = lo | (1ull << b);
        int c;
        if ((mid & 0xffffffffull) == 0ull)  // the high words decide
          ge_sums_hi(static_cast<int>(mid >> 32), m, c);
        else
          ge_sums(as_double(mid), m, c);
        const bool ok = by_mass ? (m >= p_or_n) : (static_cast<double>(c) >= p_or_n);
        if (ok) {
          lo = mid;
          c_lo = c;
        } else {
          hi = mid;
          c_hi = c;
          m_hi = m;
        }
      }
      if (c_lo - c_hi <= 1) return c_lo - c_hi == 1 ? only_in(lo, hi) : lo;
      // gather the candidates in [lo, hi)
      const double a = as_double(lo), bv = as_double(hi);
      int mine = 0;
#pragma unroll
      for (int e = 0; e < KE; ++e)
        if (e < E && pv[e] >= a && pv[e] < bv) ++mine;
      int incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int slot = incl - mine;
      __syncwarp();
#pragma unroll
      for (int e = 0; e < KE; ++e)
        if (e < E && pv[e] >= a && pv[e] < bv) cbuf[slot++] = pv[e];
      __syncwarp();
      const double cand = lane < c_lo - c_hi ? cbuf[lane] : -1.0;
      __syncwarp();
      // every candidate against every other: the mass and count of the
      // probabilities >= each candidate (those at or above hi are in m_hi,
      // c_hi); the answer is the largest candidate whose predicate holds
      double am = 0.0;
      int ac = 0;
#pragma unroll 4
      for (int jl = 0; jl < 32; ++jl) {
        const double v = __shfl_sync(0xffffffffu, cand, jl);
        if (v >= cand) {
          am += v;
          ++ac;
        }
      }
      const bool ok = by_mass ? (m_hi + am >= p_or_n) : (static_cast<double>(c_hi + ac) >= p_or_n);
      double f = (ok && cand >= 0.0) ? cand : -1.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) f = fmax(f, __shfl_xor_sync(0xffffffffu, f, o));
      return static_cast<unsigned long long>(__double_as_longlong(f));
    };
    // Top-p: n_p = the length of the shortest prefix, in descending order
    // (ties: lower index first), whose cumulative mass reaches p; all blocks
    // when p >= 1 or when the sum never reaches p.
    int n_p = nb;
    unsigned long long vsel = 0ull;  // the value at the cut
    int take = 0;                    // ties of vsel taken, lowest index first
    bool have_cut = false;
    if (p < 1.0 && total >= p) {
      const unsigned long long T = bisect(true, p);
      // elements above the cut, then ties of the cut value one at a time
      double m_gt = 0.0;
      int c_gt = 0, c_eq = 0;
      const double vT = as_double(T);
#pragma unroll
      for (int e = 0; e < KE; ++e) {
        if (e < E) {
          if (pv[e] > vT) {
            m_gt += pv[e];
            ++c_gt;
          } else if (pv[e] == vT) {
            ++c_eq;
          }
        }
      }
      m_gt = warp_sum(m_gt);
      c_gt = warp_sum_int(c_gt);
      c_eq = warp_sum_int(c_eq);
      int m = 0;
      double acc = m_gt;
      while (m < c_eq) {
        acc += vT;
        ++m;
        if (acc >= p) break;
      }
      n_p = c_gt + m;
      vsel = T;
      take = m;
      have_cut = true;
    }
    const int n = min(nb, max(top_k, n_p));
    if (n == nb) {
      vsel = 0ull;
      take = nb;
      have_cut = false;  // keep everything
    } else if (n > n_p || !have_cut) {
      // Top-k floor: the n-th largest by value (ties: lower index first)
      const unsigned long long T = bisect(false, static_cast<double>(n));
      const double vT = as_double(T);
      int c_gt = 0;
#pragma unroll
      for (int e = 0; e < KE; ++e)
        if (e < E && pv[e] > vT) ++c_gt;
      c_gt = warp_sum_int(c_gt);
      vsel = T;
      take = n - c_gt;
      have_cut = true;
    }
    // mark the selection: everything above vsel, and the first `take` ties
    // of vsel in index order (j = lane + 32 e: e-major, then lane)
    const int64_t row = static_cast<int64_t>(bh) * nb + i;
    const int nwords = E;
    const double vs = as_double(vsel);
    int before = 0;  // ties of vsel at lower indices
    uint32_t myword = 0u;
#pragma unroll
    for (int e = 0; e < KE; ++e) {
      if (e < E) {
        const bool real = pv[e] >= 0.0;
        bool keep;
        if (!have_cut) {
          keep = real;
        } else {
          const bool tie = pv[e] == vs;
          const uint32_t tb = __ballot_sync(0xffffffffu, tie);
          const int rank = before + __popc(tb & ((1u << lane) - 1u));
          keep = pv[e] > vs || (tie && rank < take);
          before += __popc(tb);
        }
        const uint32_t w = __ballot_sync(0xffffffffu, keep);
        if (lane == e) myword = w;
      }
    }
    if (lane < nwords) bitmask[row * nwords + lane] = myword;
    if (lane == 0) row_cnt[row] = n;
    __syncwarp();
  }
}

// --------------------------------------------------- row_ptr + work order
// Two launches, parallel over heads:
//   head_scan_kernel   one warp per head: the head's total, the exclusive
//                      scan of its rows' counts (row_ptr relative to the
//                      head's first row, written into row_ptr) and each
//                      row's place in the head's longest-first order (a
//                      stable counting sort by count, descending, through a
//                      per-warp bin table). The last CTA to finish turns the
//                      head totals into head offsets and head ranks (heads by
//                      total descending, ties: lower head first) and writes
//                      row_ptr[R].
//   finalize_kernel    one warp per row: row_ptr += the head's offset, the
//                      row's work_order entry, and its col_idx from the
//                      bitmask (one coalesced store per bitmask word).
// Scratch (int32): pos [R], then head totals, offsets and ranks [3][BH].
constexpr int kScanWarps = 8;

__global__ void __launch_bounds__(kScanWarps * 32)
    head_scan_kernel(int BH, int nb, const int32_t* __restrict__ row_cnt, int32_t* __restrict__ row_ptr,
                     int32_t* __restrict__ scratch, Ctrl* __restrict__ ctrl) {
  extern __shared__ int bins[];  // [kScanWarps][nb + 1]
  __shared__ int last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int R = BH * nb, nc = nb + 1;
  int32_t* pos = scratch;
  int32_t* htot = scratch + R;
  int32_t* hoff = htot + BH;
  int32_t* hrank = hoff + BH;
  const int h = blockIdx.x * kScanWarps + warp;
  if (h < BH) {
    int* myh = bins + warp * nc;
    for (int c = lane; c < nc; c += 32) myh[c] = 0;
    __syncwarp();
    const int base_row = h * nb;
    // counts, the within-head exclusive scan, and the histogram of counts
    int run = 0;
    for (int b = 0; b < nb; b += 32) {
      const int i = b + lane;
      const bool act = i < nb;
      int c = act ? row_cnt[base_row + i] : 0;
      if (act && (c < 0 || c > nb)) {
        atomicOr(&ctrl->status, kStatusCheck);
        c = 0;
      }
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (act) row_ptr[base_row + i] = run + incl - c;
      run += __shfl_sync(0xffffffffu, incl, 31);
      const unsigned m = __match_any_sync(0xffffffffu, act ? c : -1);
      if (act && lane == __ffs(m) - 1) myh[c] += __popc(m);
      __syncwarp();
    }
    if (lane == 0) htot[h] = run;
    // start of each count's run = rows with a larger count: scan bins from nb down
    const int seg = (nc + 31) / 32;
    const int q0 = min(nc, lane * seg), q1 = min(nc, q0 + seg);
    int ls = 0;
    for (int q = q0; q < q1; ++q) ls += myh[nb - q];
    int incl = ls;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int rs = incl - ls;
    __syncwarp();
    for (int q = q0; q < q1; ++q) {
      const int t = myh[nb - q];
      myh[nb - q] = rs;
      rs += t;
    }
    __syncwarp();
    for (int b = 0; b < nb; b += 32) {
      const int i = b + lane;
      const bool act = i < nb;
      int c = act ? row_cnt[base_row + i] : -1;
      if (act && (c < 0 || c > nb)) c = 0;
      const unsigned m = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(m & ((1u << lane) - 1u));
      if (act) pos[base_row + i] = myh[c] + rank;
      __syncwarp();
      if (act && lane == __ffs(m) - 1) myh[c] += __popc(m);
      __syncwarp();
    }
  }
  // the last CTA out: head offsets (exclusive scan of the totals) and ranks
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&ctrl->scan_done, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (warp == 0) {
    int run = 0;
    for (int b = 0; b < BH; b += 32) {
      const int x = b + lane;
      const int t = x < BH ? __ldcg(&htot[x]) : 0;
      int incl = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (x < BH) hoff[x] = run + incl - t;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) row_ptr[R] = run;
  }
  for (int x = threadIdx.x; x < BH; x += blockDim.x) {
    const int tx = __ldcg(&htot[x]);
    int rk = 0;
    for (int y = 0; y < BH; ++y) {
      const int ty = __ldcg(&htot[y]);
      rk += (ty > tx) || (ty == tx && y < x);
    }
    hrank[x] = rk;
  }
  if (threadIdx.x == 0) ctrl->scan_done = 0u;
}

__global__ void __launch_bounds__(256)
    finalize_kernel(int BH, int nb, const uint32_t* __restrict__ bitmask, const int32_t* __restrict__ scratch,
                    int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                    int32_t* __restrict__ work_order) {
  const int lane = threadIdx.x & 31;
  const int R = BH * nb;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= R) return;
  const int h = r / nb;
  const int32_t* pos = scratch;
  const int32_t* hoff = scratch + R + BH;
  const int32_t* hrank = hoff + BH;
  const int start = row_ptr[r] + hoff[h];
  if (lane == 0) {
    row_ptr[r] = start;
    work_order[hrank[h] * nb + pos[r]] = r;
  }
  // col_idx: bit `lane` of word e lands after the set bits below it
  const int nwords = (nb + 31) >> 5;
  const uint32_t w = lane < nwords ? bitmask[static_cast<int64_t>(r) * nwords + lane] : 0u;
  const int cnt = __popc(w);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const int excl = incl - cnt;
  for (int e = 0; e < nwords; ++e) {
    const uint32_t we = __shfl_sync(0xffffffffu, w, e);
    const int pe = __shfl_sync(0xffffffffu, excl, e);
    if ((we >> lane) & 1u) col_idx[start + pe + __popc(we & ((1u << lane) - 1u))] = e * 32 + lane;
  }
}

// row_ptr (exclusive scan of row_cnt), work_order and col_idx from bitmask
// and row_cnt: shared by the Top-p and the stripe masks. iscratch: int32
// [R + 3*B*H] of workspace the caller no longer needs.
cudaError_t launch_scan_expand(const sba_plan* p, const uint32_t* bitmask, const int32_t* row_cnt,
                               int32_t* row_ptr, int32_t* col_idx, int32_t* work_order,
                               int32_t* iscratch, Ctrl* ctrl, cudaStream_t st) {
  const int R = p->info.rows;
  const int nb = p->info.nb;
  const int BH = p->g.B * p->g.H;
  const size_t smem = static_cast<size_t>(kScanWarps) * (nb + 1) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(head_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  head_scan_kernel<<<(BH + kScanWarps - 1) / kScanWarps, kScanWarps * 32, smem, st>>>(
      BH, nb, row_cnt, row_ptr, iscratch, ctrl);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  finalize_kernel<<<(R + 7) / 8, 256, 0, st>>>(BH, nb, bitmask, iscratch, row_ptr, col_idx, work_order);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_build_mask(const sba_plan* p, const void* qt, const void* kt,
                              const float* top_p, int top_k, uint32_t* bitmask, int32_t* row_cnt,
                              int32_t* row_ptr, int32_t* col_idx, int32_t* work_order,
                              double* qbar, double* kbar, double* scores, size_t scores_bytes,
                              Ctrl* ctrl, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  const int BH = g.B * g.H;

  const int64_t pool_items = 2ll * BH * g.nb;
  const unsigned pg = static_cast<unsigned>((pool_items + kPoolWarps - 1) / kPoolWarps);
  if (p->g.dtype == SBA_BF16)
    pool_kernel<__nv_bfloat16><<<pg, kPoolWarps * 32, 0, st>>>(g, static_cast<const char*>(qt),
                                                               static_cast<const char*>(kt), qbar, kbar);
  else
    pool_kernel<float><<<pg, kPoolWarps * 32, 0, st>>>(g, static_cast<const char*>(qt),
                                                       static_cast<const char*>(kt), qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  SelectArgs sa;
  for (int h = 0; h < 256; ++h) sa.top_p[h] = h < g.H ? top_p[h] : 1.0f;
  // scores then cut, a chunk of heads at a time (the chunk's scores fit the
  // scratch and stay in L2 between the two launches)
  const size_t per_head = static_cast<size_t>(g.nb) * g.nb * sizeof(double);
  const int hc = static_cast<int>(std::min<size_t>(BH, scores_bytes / per_head));
  if (hc < 1) return cudaErrorInvalidValue;
  const int nt = (g.nb + kScoreTile - 1) / kScoreTile;
  for (int h0 = 0; h0 < BH; h0 += hc) {
    const int nh = std::min(hc, BH - h0);
    score_kernel<<<dim3(nt, nt, nh), 256, 0, st>>>(g, h0, qbar, kbar, scores);
    const unsigned cg = static_cast<unsigned>((nh * g.nb + kSelWarps - 1) / kSelWarps);
    if (g.nb <= 256)
      cut_kernel<8><<<cg, kSelThreads, 0, st>>>(g, h0, nh, scores, sa, top_k, bitmask, row_cnt);
    else if (g.nb <= 512)
      cut_kernel<16><<<cg, kSelThreads, 0, st>>>(g, h0, nh, scores, sa, top_k, bitmask, row_cnt);
    else
      cut_kernel<32><<<cg, kSelThreads, 0, st>>>(g, h0, nh, scores, sa, top_k, bitmask, row_cnt);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  // the pooled query means are no longer needed: their space is the scan's scratch
  return launch_scan_expand(p, bitmask, row_cnt, row_ptr, col_idx, work_order,
                            reinterpret_cast<int32_t*>(qbar), ctrl, st);
}

// ------------------------------------------------------------ stripe masks
// Parameterized Stripe Attention for Efficient Video Generation (Approach):
// M(Tw, To, Ts, Sw, So, Ss). One warp per (head, query block) row writes the
// row's bitmask words with ballots and its count; the CSR and the work order
// come from the same scan and expand launches as the Top-p mask.
namespace {

struct StripeArgs {
  int16_t p[256][6];  // Tw, To, Ts, Sw, So, Ss per head
};

__device__ __forceinline__ bool in_stripe(int x, int w, int o, int s) {
  const int y = x - o;
  if (s == 0) return y >= 0 && y < w;
  int m = y % s;
  if (m < 0) m += s;
  return m < w;
}

// grid (ceil(nb / 8), B*H), 256 threads: warp w handles query block
// blockIdx.x*8 + w of head blockIdx.y.
__global__ void __launch_bounds__(256)
    stripe_kernel(KGeom g, StripeArgs sa, uint32_t* __restrict__ bitmask,
                  int32_t* __restrict__ row_cnt) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp;
  if (i >= g.nb) return;  // whole warp
  const int bh = blockIdx.y;
  uint32_t b, h;
  g.dv_H.divmod(static_cast<uint32_t>(bh), b, h);
  const int Tw = sa.p[h][0], To = sa.p[h][1], Ts = sa.p[h][2];
  const int Sw = sa.p[h][3], So = sa.p[h][4], Ss = sa.p[h][5];
  const int nS = g.nH * g.nW;
  const int qt = i / nS, qs = i - qt * nS;
  const int words = (g.nb + 31) >> 5;
  const int64_t r = static_cast<int64_t>(bh) * g.nb + i;
  int cnt = 0;
  for (int c = 0; c < words; ++c) {
    const int j = c * 32 + lane;
    bool keep = false;
    if (j < g.nb) {
      const int kt = j / nS, ks = j - kt * nS;
      keep = in_stripe(kt - qt, Tw, To, Ts) && in_stripe(ks - qs, Sw, So, Ss);
    }
    const uint32_t word = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) bitmask[r * words + c] = word;
    cnt += __popc(word);
  }
  if (lane == 0) row_cnt[r] = cnt;
}

}  // namespace

cudaError_t launch_build_stripe_mask(const sba_plan* p, const sba_stripe* params,
                                     uint32_t* bitmask, int32_t* row_cnt, int32_t* row_ptr,
                                     int32_t* col_idx, int32_t* work_order, void* workspace,
                                     cudaStream_t st) {
  KGeom g = make_kgeom(p);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(static_cast<char*>(workspace) + p->ws_ctrl);
  StripeArgs sa;
  for (int h = 0; h < 256; ++h) {
    const sba_stripe q = h < g.H ? params[h] : sba_stripe{0, 0, 0, 0, 0, 0};
    const int32_t v[6] = {q.Tw, q.To, q.Ts, q.Sw, q.So, q.Ss};
    for (int k = 0; k < 6; ++k) sa.p[h][k] = static_cast<int16_t>(v[k]);
  }
  dim3 grid((g.nb + 7) / 8, g.B * g.H);
  stripe_kernel<<<grid, 256, 0, st>>>(g, sa, bitmask, row_cnt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_scan_expand(p, bitmask, row_cnt, row_ptr, col_idx, work_order,
                            reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + p->ws_qbar), ctrl, st);
}

// ------------------------------------------------------------------------
// Allocation-free variant of sba_build_mask.
//
// Some callers cannot hand the library a workspace: plugin hosts whose
// interface passes only inputs and outputs, and services that reserve all
// device memory at start-up and forbid any later cudaMalloc (an allocation
// there can synchronise the device or fail under memory pressure in the middle
// of serving). For them the pooled means and the control block live in one
// file-scope device array that every GPU loading this library holds until the
// process exits.
// ------------------------------------------------------------------------

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_mask_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];

// Device address of g_mask_scratch on the current device (host code must
// never pass the symbol itself to a kernel: on the host it only names a
// stand-in). Outside stream capture the address is looked up on every call
// (cheap, and right again after a device reset reloads the module); a failed
// lookup is returned and not remembered. Inside a capture, where the lookup
// may not be allowed, the last successful lookup on this device is used.
cudaError_t scratch_address(cudaStream_t st, void** out) {
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_mask_scratch);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    g_scratch_addr[dev] = ptr;
    *out = ptr;
    return cudaSuccess;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  *out = g_scratch_addr[dev];
  return *out ? cudaSuccess : cudaErrorStreamCaptureUnsupported;
}

size_t noalloc_pooled_bytes(const sba_plan* p) {
  return (static_cast<size_t>(p->info.rows) * p->g.d * sizeof(double) + 255) & ~size_t(255);
}

// control block, pooled means, then at least one head's pooled scores
size_t noalloc_scratch_need(const sba_plan* p) {
  return sizeof(Ctrl) + 2 * noalloc_pooled_bytes(p) +
         static_cast<size_t>(p->info.nb) * p->info.nb * sizeof(double);
}

}  // namespace

}  // namespace sba

extern "C" sba_status sba_build_mask_noalloc(const sba_plan* plan, const void* qt, const void* kt,
                                             const float* top_p, int32_t top_k, uint32_t* bitmask,
                                             int32_t* row_cnt, int32_t* row_ptr, int32_t* col_idx,
                                             int32_t* work_order, void* stream) {
  using namespace sba;
  set_error("");
  if (!plan || !qt || !kt || !top_p || !bitmask || !row_cnt || !row_ptr || !col_idx || !work_order) {
    set_error("sba_build_mask_noalloc: NULL argument");
    return SBA_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(qt) | reinterpret_cast<uintptr_t>(kt)) & 15u) {
    set_error("qt and kt must be 16-byte aligned");
    return SBA_ERR_INVALID_ARG;
  }
  if (top_k < 0) {
    set_error("top_k must be >= 0");
    return SBA_ERR_INVALID_ARG;
  }
  for (int h = 0; h < plan->g.H; ++h) {
    const float p = top_p[h];
    if (!(p > 0.0f) || !(p <= 1.0f)) {
      set_error("top_p[%d] = %g; must lie in (0, 1]", h, (double)p);
      return SBA_ERR_INVALID_ARG;
    }
  }
  const size_t need = noalloc_scratch_need(plan);
  if (need > kNoAllocScratchBytes) {
    set_error("sba_build_mask_noalloc needs %zu bytes of scratch (2*B*H*nb*d + nb*nb doubles + 256) but "
              "its static scratch holds %zu; use sba_build_mask with a workspace",
              need, kNoAllocScratchBytes);
    return SBA_ERR_CAPACITY;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  cudaError_t e = scratch_address(st, &scratch);
  if (e != cudaSuccess || !scratch) {
    set_error("cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    return SBA_ERR_CUDA;
  }
  char* sc = static_cast<char*>(scratch);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(sc);
  double* qbar = reinterpret_cast<double*>(sc + sizeof(Ctrl));
  double* kbar = reinterpret_cast<double*>(sc + sizeof(Ctrl) + noalloc_pooled_bytes(plan));
  // the rest of the scratch holds pooled scores, as many heads at a time as fit
  const size_t scores_off = sizeof(Ctrl) + 2 * noalloc_pooled_bytes(plan);
  double* scores = reinterpret_cast<double*>(sc + scores_off);
  // the control block keeps the previous call's contents: start from zero
  e = cudaMemsetAsync(ctrl, 0, sizeof(Ctrl), st);
  if (e == cudaSuccess)
    e = launch_build_mask(plan, qt, kt, top_p, top_k, bitmask, row_cnt, row_ptr, col_idx, work_order,
                          qbar, kbar, scores, kNoAllocScratchBytes - scores_off, ctrl, st);
  if (e != cudaSuccess) {
    set_error("sba_build_mask_noalloc launch: %s", cudaGetErrorString(e));
    return SBA_ERR_CUDA;
  }
  return SBA_OK;
}

extern "C" sba_status sba_noalloc_status(void* stream) {
  using namespace sba;
  set_error("");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  cudaError_t e = scratch_address(st, &scratch);
  if (e != cudaSuccess || !scratch) {
    set_error("cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    return SBA_ERR_CUDA;
  }
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    set_error("cudaStreamSynchronize: %s", cudaGetErrorString(e));
    return SBA_ERR_CUDA;
  }
  uint32_t word = 0;
  e = cudaMemcpy(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(scratch, 0, sizeof(word));
  if (e != cudaSuccess) {
    set_error("reading the scratch status word: %s", cudaGetErrorString(e));
    return SBA_ERR_CUDA;
  }
  if (word & kStatusTimeout) {
    set_error("a bounded device wait gave up");
    return SBA_ERR_DEVICE_TIMEOUT;
  }
  if (word & kStatusCheck) {
    set_error("a device-side input check failed");
    return SBA_ERR_DEVICE_CHECK;
  }
  return SBA_OK;
}
