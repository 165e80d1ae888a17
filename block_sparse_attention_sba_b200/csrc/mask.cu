// mask.cu -- block scoring and Top-p / Top-k routing (FVAttn: Adaptive Sparse
// Attention with Runtime Load Balancing for Video Generation, abstract:
// "Top-p routing, a Top-k safety floor"), plus the longest-first work order
// that absorbs the uneven per-head workloads the abstract describes.
//
// Four launches on the caller's stream:
//   pool_kernel        mean of the real tokens of every block of qt and kt
//                      (fp32). HBM-bound: reads qt and kt once.
//   select_kernel      per (b, h) and 16 query blocks: pooled scores on CUDA
//                      cores in fp32, row softmax, a warp bitonic sort of
//                      (probability, index) keys in shared memory, a warp scan
//                      of the sorted masses, the Top-p cut with the Top-k
//                      floor; writes the bitmask row and row_cnt.
//   scan_order_kernel  one CTA: row_ptr (exclusive scan of row_cnt) and the
//                      work order (stable counting sort by row_cnt, longest
//                      first) with per-warp segment counters, so the result is
//                      deterministic.
//   expand_kernel      one warp per row: bitmask -> ascending col_idx.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace sba {

namespace {

// ------------------------------------------------------------------ pooling
constexpr int kPoolThreads = 256;

template <typename T>
__device__ __forceinline__ void accum_vec(double* acc, const uint4& v);

template <>
__device__ __forceinline__ void accum_vec<__nv_bfloat16>(double* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
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

// grid (nb, B*H, 2): z = 0 pools qt, z = 1 pools kt. Sums in fp64 (a sum of
// bf16 or fp32 values is exact there for any realistic spread of exponents),
// one division by the number of real tokens.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(KGeom g, const char* __restrict__ qt, const char* __restrict__ kt,
                double* __restrict__ qbar, double* __restrict__ kbar) {
  constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
  const int j = blockIdx.x, bh = blockIdx.y;
  const char* src = blockIdx.z == 0 ? qt : kt;
  double* dst = blockIdx.z == 0 ? qbar : kbar;
  const int vpr = g.d / EPV;            // vectors per row (8..32)
  const int groups = kPoolThreads / vpr;  // row groups
  const int c = threadIdx.x % vpr;
  const int rg = threadIdx.x / vpr;

  // the block's real tokens occupy its first len slots (both orders)
  const int len = block_len(g, j);

  const int64_t row_bytes = static_cast<int64_t>(g.d) * sizeof(T);
  const char* base = src + (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * row_bytes;
  double acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.0;
  for (int o = rg; o < len; o += groups) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + o * row_bytes + c * 16));
    accum_vec<T>(acc, v);
  }
  __shared__ double red[kPoolThreads * 8];
  // red[rg][d]: reduce over row groups
#pragma unroll
  for (int e = 0; e < EPV; ++e) red[rg * g.d + c * EPV + e] = acc[e];
  __syncthreads();
  const double dlen = static_cast<double>(len);
  for (int col = threadIdx.x; col < g.d; col += kPoolThreads) {
    double s = 0.0;
    for (int r = 0; r < groups; ++r) s += red[r * g.d + col];
    dst[(static_cast<int64_t>(bh) * g.nb + j) * g.d + col] = s / dlen;
  }
}

// ---------------------------------------------------------- score + select
// All of it in fp64, so that the routing decision is the exact one except
// where the cumulative mass at the cut lies within rounding of p.
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kRQ = 16;      // query blocks per CTA
constexpr int kMaxE = 32;    // probabilities per lane (nb <= 1024)

struct SelectArgs {
  float top_p[256];
};

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// grid (ceil(nb/kRQ), B*H), kSelThreads threads. Dynamic shared memory:
//   qs [kRQ][d] f64 | S [kRQ][nb] f64
// Phase 1: thread t computes the scores of key blocks t, t+256, ... against
// the CTA's kRQ query blocks (fp64 FMA, K rows streamed from L1).
// Phase 2: one warp per query block: fp64 softmax over the key blocks, then
// the cut: the largest probability v with mass(P >= v) >= p found by
// bisection on the bit pattern of v (warp mass sums), the ties of v taken in
// index order until the mass reaches p; the Top-k floor by the same
// bisection on counts. No sort.
__global__ void __launch_bounds__(kSelThreads, 2)
    select_kernel(KGeom g, const double* __restrict__ qbar, const double* __restrict__ kbar,
                  SelectArgs sa, int top_k, uint32_t* __restrict__ bitmask,
                  int32_t* __restrict__ row_cnt) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int d = g.d, nb = g.nb;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * kRQ;
  double* qs = reinterpret_cast<double*>(smem);
  double* S = qs + kRQ * d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double* qsrc = qbar + static_cast<int64_t>(bh) * nb * d;
  const double* ksrc = kbar + static_cast<int64_t>(bh) * nb * d;

  // stage the query rows (zero rows past nb)
  for (int e = tid; e < kRQ * d; e += kSelThreads) {
    const int r = e / d, c = e % d;
    qs[e] = (q0 + r < nb) ? qsrc[static_cast<int64_t>(q0 + r) * d + c] : 0.0;
  }
  __syncthreads();
  const double sqrt_d = sqrt(static_cast<double>(d));
  for (int j = tid; j < nb; j += kSelThreads) {
    double acc[kRQ];
#pragma unroll
    for (int r = 0; r < kRQ; ++r) acc[r] = 0.0;
    const double2* krow = reinterpret_cast<const double2*>(ksrc + static_cast<int64_t>(j) * d);
    for (int c2 = 0; c2 < d / 2; ++c2) {
      const double2 kv = __ldg(krow + c2);
#pragma unroll
      for (int r = 0; r < kRQ; ++r) {
        const double2 qv = reinterpret_cast<const double2*>(qs + r * d)[c2];
        acc[r] = fma(qv.x, kv.x, acc[r]);
        acc[r] = fma(qv.y, kv.y, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRQ; ++r) S[r * nb + j] = acc[r] / sqrt_d;
  }
  __syncthreads();

  uint32_t h;
  {
    uint32_t bq;
    g.dv_H.divmod(static_cast<uint32_t>(bh), bq, h);
  }
  const double p = static_cast<double>(sa.top_p[h]);
  const int E = (nb + 31) >> 5;
  for (int r = warp; r < kRQ; r += kSelWarps) {
    const int i = q0 + r;
    if (i >= nb) break;
    const double* srow = S + r * nb;
    // softmax in fp64: shift by the row max, exp, divide by the sum
    double mx = -INFINITY;
    for (int j = lane; j < nb; j += 32) mx = fmax(mx, srow[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    double pv[kMaxE];
    double esum = 0.0;
#pragma unroll
    for (int e = 0; e < kMaxE; ++e) {
      const int j = lane + 32 * e;
      pv[e] = (e < E && j < nb) ? exp(srow[j] - mx) : 0.0;
      esum += pv[e];
    }
    esum = warp_sum(esum);
#pragma unroll
    for (int e = 0; e < kMaxE; ++e) {
      const int j = lane + 32 * e;
      pv[e] = (e < E && j < nb) ? pv[e] / esum : -1.0;  // -1: not a key block
    }
    // mass and count of the row's probabilities >= v (the -1 entries never
    // pass: every v tried is a non-negative double, bit 62 of its pattern
    // being clear)
    auto ge_sums = [&](double v, double& m, int& c) {
      double mm = 0.0;
      int cc = 0;
#pragma unroll
      for (int e = 0; e < kMaxE; ++e)
        if (e < E && pv[e] >= v) {
          mm += pv[e];
          ++cc;
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mm += __shfl_xor_sync(0xffffffffu, mm, o);
        cc += __shfl_xor_sync(0xffffffffu, cc, o);
      }
      m = mm;
      c = cc;
    };
    auto as_double = [](unsigned long long b) { return __longlong_as_double(static_cast<long long>(b)); };
    // The single probability in [lo, hi) (bit patterns), found once the
    // bisection interval holds exactly one element.
    auto only_in = [&](unsigned long long lo, unsigned long long hi) -> unsigned long long {
      double f = -1.0;
      const double a = as_double(lo), b = as_double(hi);
#pragma unroll
      for (int e = 0; e < kMaxE; ++e)
        if (e < E && pv[e] >= a && pv[e] < b) f = pv[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) f = fmax(f, __shfl_xor_sync(0xffffffffu, f, o));
      return static_cast<unsigned long long>(__double_as_longlong(f));
    };
    // Bisection over bit patterns for the largest element v with
    // pred(mass(P >= v), count(P >= v)). Invariant: pred holds at lo and fails
    // at hi, so the answer lies in [lo, hi); stop once one element is left
    // there (or the interval is one pattern wide).
    auto bisect = [&](bool by_mass, double p_or_n) -> unsigned long long {
      unsigned long long lo = 0ull, hi = 1ull << 62;
      double m;
      int c_lo, c_hi = 0;
      ge_sums(0.0, m, c_lo);
      for (int b = 61; b >= 0 && c_lo - c_hi > 1; --b) {
        const unsigned long long mid = lo | (1ull << b);
        int c;
        ge_sums(as_double(mid), m, c);
        const bool ok = by_mass ? (m >= p_or_n) : (static_cast<double>(c) >= p_or_n);
        if (ok) {
          lo = mid;
          c_lo = c;
        } else {
          hi = mid;
          c_hi = c;
        }
      }
      return c_lo - c_hi == 1 ? only_in(lo, hi) : lo;
    };
    // Top-p: n_p = the length of the shortest prefix, in descending order
    // (ties: lower index first), whose cumulative mass reaches p; all blocks
    // when p >= 1 or when the sum never reaches p.
    int n_p = nb;
    unsigned long long vsel = 0ull;  // the value at the cut
    int take = 0;                    // ties of vsel taken, lowest index first
    bool have_cut = false;
    double total;
    int cnt_all;
    ge_sums(0.0, total, cnt_all);
    if (p < 1.0 && total >= p) {
      const unsigned long long T = bisect(true, p);
      // elements above the cut, then ties of the cut value one at a time
      double m_gt = 0.0;
      int c_gt = 0, c_eq = 0;
      const double vT = as_double(T);
#pragma unroll
      for (int e = 0; e < kMaxE; ++e) {
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
      for (int e = 0; e < kMaxE; ++e)
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
    for (int e = 0; e < kMaxE; ++e) {
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
constexpr int kScanThreads = 1024;
constexpr int kScanWarps = kScanThreads / 32;

// Exclusive scan of one value per thread across the CTA; returns the prefix
// and writes the total to *total (shared).
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += t;
    }
    warp_sums[lane] = si - s;
    if (lane == 31) *total = si;
  }
  __syncthreads();
  const int res = warp_sums[warp] + incl - v;
  __syncthreads();
  return res;
}

// One CTA of 1024 threads. Dynamic shared memory: hist [kScanWarps][nb+1]
// ints (one bin table per warp), head totals [BH] and head ranks [BH].
// Work order: heads by total selected blocks descending (ties: lower head
// first), then, inside a head, rows by count descending (ties: lower row
// first). Each warp sorts whole heads with a stable counting sort over its own
// bin table, so the result is deterministic.
__global__ void __launch_bounds__(kScanThreads)
    scan_order_kernel(int R, int nb, int BH, const int32_t* __restrict__ row_cnt,
                      int32_t* __restrict__ row_ptr, int32_t* __restrict__ work_order,
                      uint32_t* __restrict__ status) {
  extern __shared__ int ssm[];
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nc = nb + 1;
  int* hist = ssm;                         // [kScanWarps][nc]
  int* htot = hist + kScanWarps * nc;      // [BH]
  int* hrank = htot + BH;                  // [BH]

  // ---- row_ptr: each thread owns a contiguous chunk of rows
  const int per = (R + kScanThreads - 1) / kScanThreads;
  const int r0 = min(R, tid * per), r1 = min(R, r0 + per);
  int local = 0;
  for (int r = r0; r < r1; ++r) local += row_cnt[r];
  int run = block_exclusive_scan(local, warp_sums, &total);
  for (int r = r0; r < r1; ++r) {
    row_ptr[r] = run;
    run += row_cnt[r];
  }
  if (tid == 0) row_ptr[R] = total;

  // ---- head totals (one warp per head)
  for (int h = warp; h < BH; h += kScanWarps) {
    int sum = 0;
    for (int i = lane; i < nb; i += 32) sum += row_cnt[h * nb + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) htot[h] = sum;
  }
  __syncthreads();
  // ---- head ranks: number of heads that come first
  for (int h = tid; h < BH; h += kScanThreads) {
    const int th = htot[h];
    int rk = 0;
    for (int x = 0; x < BH; ++x) {
      const int tx = htot[x];
      rk += (tx > th) || (tx == th && x < h);
    }
    hrank[h] = rk;
  }
  __syncthreads();

  // ---- inside each head: stable counting sort by count, descending
  int* myh = hist + warp * nc;
  for (int h = warp; h < BH; h += kScanWarps) {
    for (int c = lane; c < nc; c += 32) myh[c] = 0;
    __syncwarp();
    const int base_row = h * nb;
    for (int b = 0; b < nb; b += 32) {
      const int i = b + lane;
      const bool act = i < nb;
      int c = act ? row_cnt[base_row + i] : -1;
      if (act && (c < 0 || c > nb)) {
        atomicOr(status, kStatusCheck);
        c = 0;
      }
      const unsigned m = __match_any_sync(0xffffffffu, c);
      if (act && lane == __ffs(m) - 1) myh[c] += __popc(m);
      __syncwarp();
    }
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
    const int out_base = hrank[h] * nb;
    for (int b = 0; b < nb; b += 32) {
      const int i = b + lane;
      const bool act = i < nb;
      int c = act ? row_cnt[base_row + i] : -1;
      if (act && (c < 0 || c > nb)) c = 0;
      const unsigned m = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(m & ((1u << lane) - 1u));
      const int pos = act ? myh[c] + rank : 0;
      __syncwarp();
      if (act) work_order[out_base + pos] = base_row + i;
      if (act && lane == __ffs(m) - 1) myh[c] += __popc(m);
      __syncwarp();
    }
  }
}

// ------------------------------------------------------------- CSR expand
__global__ void __launch_bounds__(256)
    expand_kernel(int R, int nb, const uint32_t* __restrict__ bitmask,
                  const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= R) return;
  const int nwords = (nb + 31) >> 5;
  uint32_t w = lane < nwords ? bitmask[static_cast<int64_t>(r) * nwords + lane] : 0u;
  const int cnt = __popc(w);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  int pos = row_ptr[r] + incl - cnt;
  while (w) {
    const int b = __ffs(w) - 1;
    col_idx[pos++] = lane * 32 + b;
    w &= w - 1;
  }
}

// row_ptr (exclusive scan of row_cnt), work_order and col_idx from bitmask
// and row_cnt: shared by the Top-p and the stripe masks.
cudaError_t launch_scan_expand(const sba_plan* p, const uint32_t* bitmask, const int32_t* row_cnt,
                               int32_t* row_ptr, int32_t* col_idx, int32_t* work_order,
                               uint32_t* status, cudaStream_t st) {
  const int R = p->info.rows;
  const int nb = p->info.nb;
  const int BH = p->g.B * p->g.H;
  const size_t scan_smem = (static_cast<size_t>(kScanWarps) * (nb + 1) + 2 * static_cast<size_t>(BH)) * sizeof(int);
  if (scan_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(scan_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(scan_smem));
    if (e != cudaSuccess) return e;
  }
  scan_order_kernel<<<1, kScanThreads, scan_smem, st>>>(R, nb, BH, row_cnt, row_ptr, work_order,
                                                        status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  expand_kernel<<<(R + 7) / 8, 256, 0, st>>>(R, nb, bitmask, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace

static size_t select_smem_bytes(int d, int nb) {
  return static_cast<size_t>(kRQ) * d * sizeof(double) + static_cast<size_t>(kRQ) * nb * sizeof(double);
}

cudaError_t launch_build_mask(const sba_plan* p, const void* qt, const void* kt,
                              const float* top_p, int top_k, uint32_t* bitmask, int32_t* row_cnt,
                              int32_t* row_ptr, int32_t* col_idx, int32_t* work_order,
                              double* qbar, double* kbar, uint32_t* status, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  const int BH = g.B * g.H;

  dim3 pg(g.nb, BH, 2);
  if (p->g.dtype == SBA_BF16)
    pool_kernel<__nv_bfloat16><<<pg, kPoolThreads, 0, st>>>(g, static_cast<const char*>(qt),
                                                            static_cast<const char*>(kt), qbar, kbar);
  else
    pool_kernel<float><<<pg, kPoolThreads, 0, st>>>(g, static_cast<const char*>(qt),
                                                    static_cast<const char*>(kt), qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const size_t sel_smem = select_smem_bytes(g.d, g.nb);
  if (sel_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sel_smem));
    if (e != cudaSuccess) return e;
  }
  SelectArgs sa;
  for (int h = 0; h < 256; ++h) sa.top_p[h] = h < g.H ? top_p[h] : 1.0f;
  dim3 sg((g.nb + kRQ - 1) / kRQ, BH);
  select_kernel<<<sg, kSelThreads, sel_smem, st>>>(g, qbar, kbar, sa, top_k, bitmask, row_cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  return launch_scan_expand(p, bitmask, row_cnt, row_ptr, col_idx, work_order, status, st);
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
  return launch_scan_expand(p, bitmask, row_cnt, row_ptr, col_idx, work_order, &ctrl->status, st);
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

size_t noalloc_scratch_need(const sba_plan* p) { return sizeof(Ctrl) + 2 * noalloc_pooled_bytes(p); }

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
    set_error("sba_build_mask_noalloc needs %zu bytes of scratch (2*B*H*nb*d doubles + 256) but "
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
  // the control block keeps the previous call's contents: start from zero
  e = cudaMemsetAsync(ctrl, 0, sizeof(Ctrl), st);
  if (e == cudaSuccess)
    e = launch_build_mask(plan, qt, kt, top_p, top_k, bitmask, row_cnt, row_ptr, col_idx, work_order,
                          qbar, kbar, &ctrl->status, st);
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
