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
__device__ __forceinline__ void accum_vec(float* acc, const uint4& v);

template <>
__device__ __forceinline__ void accum_vec<__nv_bfloat16>(float* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void accum_vec<float>(float* acc, const uint4& v) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}

// grid (nb, B*H, 2): z = 0 pools qt, z = 1 pools kt.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(KGeom g, const char* __restrict__ qt, const char* __restrict__ kt,
                float* __restrict__ qbar, float* __restrict__ kbar) {
  constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
  const int j = blockIdx.x, bh = blockIdx.y;
  const char* src = blockIdx.z == 0 ? qt : kt;
  float* dst = blockIdx.z == 0 ? qbar : kbar;
  const int vpr = g.d / EPV;            // vectors per row (8..32)
  const int groups = kPoolThreads / vpr;  // row groups
  const int c = threadIdx.x % vpr;
  const int rg = threadIdx.x / vpr;

  // the block's real tokens occupy its first len slots (both orders)
  const int len = block_len(g, j);

  const int64_t row_bytes = static_cast<int64_t>(g.d) * sizeof(T);
  const char* base = src + (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * row_bytes;
  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
  for (int o = rg; o < len; o += groups) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + o * row_bytes + c * 16));
    accum_vec<T>(acc, v);
  }
  __shared__ float red[kPoolThreads * 8];
  // red[rg][d]: reduce over row groups
#pragma unroll
  for (int e = 0; e < EPV; ++e) red[rg * g.d + c * EPV + e] = acc[e];
  __syncthreads();
  const float inv_len = 1.0f / static_cast<float>(len);
  for (int col = threadIdx.x; col < g.d; col += kPoolThreads) {
    float s = 0.f;
    for (int r = 0; r < groups; ++r) s += red[r * g.d + col];
    dst[(static_cast<int64_t>(bh) * g.nb + j) * g.d + col] = s * inv_len;
  }
}

// ---------------------------------------------------------- score + select
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kRQ = 16;      // query blocks per CTA
constexpr int kKC = 64;      // key blocks per shared-memory chunk

struct SelectArgs {
  float top_p[256];
};

__device__ __forceinline__ unsigned long long key_of(float p, int j) {
  return (static_cast<unsigned long long>(~__float_as_uint(p)) << 32) | static_cast<uint32_t>(j);
}

// Ascending bitonic sort of n (power of two, >= 32) 64-bit keys by one warp.
__device__ void warp_bitonic_sort(unsigned long long* a, int n) {
  const int lane = threadIdx.x & 31;
  for (int k = 2; k <= n; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = lane; i < (n >> 1); i += 32) {
        const int lo = 2 * jj * (i / jj) + (i % jj);
        const int hi = lo + jj;
        const unsigned long long x = a[lo], y = a[hi];
        const bool up = (lo & k) == 0;
        if ((x > y) == up) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncwarp();
    }
  }
}

// grid (ceil(nb/kRQ), B*H). Dynamic shared memory:
//   qs [kRQ][d+4] f32 | S [kRQ][nkp] f32 | union{ ks [kKC][d+4] f32,
//   sort keys [kSelWarps][nkp] u64 } | words [kSelWarps][32] u32
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(KGeom g, const float* __restrict__ qbar, const float* __restrict__ kbar,
                  SelectArgs sa, int top_k, int nkp, uint32_t* __restrict__ bitmask,
                  int32_t* __restrict__ row_cnt) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int d = g.d, nb = g.nb, ld = d + 4;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * kRQ;
  float* qs = reinterpret_cast<float*>(smem);
  float* S = qs + kRQ * ld;
  unsigned char* uni = reinterpret_cast<unsigned char*>(S + kRQ * nkp);
  float* ks = reinterpret_cast<float*>(uni);
  const size_t uni_bytes = max(static_cast<size_t>(kKC) * ld * 4, static_cast<size_t>(kSelWarps) * nkp * 8);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(uni);
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(uni + uni_bytes);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* qsrc = qbar + static_cast<int64_t>(bh) * nb * d;
  const float* ksrc = kbar + static_cast<int64_t>(bh) * nb * d;

  // stage the query rows (zero rows past nb)
  for (int e = tid; e < kRQ * d; e += kSelThreads) {
    const int r = e / d, c = e % d;
    qs[r * ld + c] = (q0 + r < nb) ? qsrc[static_cast<int64_t>(q0 + r) * d + c] : 0.f;
  }
  const float scale = rsqrtf(static_cast<float>(d));
  const int kk = tid % kKC;       // key within chunk
  const int rg = tid / kKC;       // rows rg*4 .. rg*4+3
  for (int j0 = 0; j0 < nb; j0 += kKC) {
    __syncthreads();
    for (int e = tid; e < kKC * (d / 4); e += kSelThreads) {
      const int r = e / (d / 4), c4 = e % (d / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + r < nb) v = *reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(j0 + r) * d + c4 * 4);
      *reinterpret_cast<float4*>(ks + r * ld + c4 * 4) = v;
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float* krow = ks + kk * ld;
    for (int c = 0; c < d; c += 4) {
      const float4 kv = *reinterpret_cast<const float4*>(krow + c);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (rg * 4 + r) * ld + c);
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
    if (j0 + kk < nb) {
#pragma unroll
      for (int r = 0; r < 4; ++r) S[(rg * 4 + r) * nkp + j0 + kk] = acc[r] * scale;
    }
  }
  __syncthreads();  // all scores written; ks area becomes sort keys

  uint32_t h;
  {
    uint32_t bq;
    g.dv_H.divmod(static_cast<uint32_t>(bh), bq, h);
  }
  const float p = sa.top_p[h];
  unsigned long long* kw = keys + static_cast<size_t>(warp) * nkp;
  uint32_t* words = wbuf + warp * 32;
  const int seg = nkp / 32;
  for (int r = warp; r < kRQ; r += kSelWarps) {
    const int i = q0 + r;
    if (i >= nb) break;
    const float* srow = S + r * nkp;
    float mx = -INFINITY;
    for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, srow[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int j = lane; j < nb; j += 32) sum += expf(srow[j] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
    for (int j = lane; j < nkp; j += 32)
      kw[j] = (j < nb) ? key_of(expf(srow[j] - mx) * inv, j) : ~0ull;
    words[lane] = 0u;
    __syncwarp();
    warp_bitonic_sort(kw, nkp);

    // cumulative mass along the sorted order: lane owns positions [lane*seg, +seg)
    float local = 0.f;
    for (int e = 0; e < seg; ++e) local += __uint_as_float(~static_cast<uint32_t>(kw[lane * seg + e] >> 32));
    float incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    float run = incl - local;
    int hit = 0x7fffffff;
    for (int e = 0; e < seg; ++e) {
      run += __uint_as_float(~static_cast<uint32_t>(kw[lane * seg + e] >> 32));
      if (run >= p) {
        hit = lane * seg + e;
        break;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) hit = min(hit, __shfl_xor_sync(0xffffffffu, hit, o));
    int n_p = (p >= 1.0f || hit >= nb) ? nb : hit + 1;
    const int n = min(nb, max(top_k, n_p));
    for (int e = lane; e < n; e += 32) {
      const uint32_t j = static_cast<uint32_t>(kw[e] & 0xffffffffu);
      atomicOr(&words[j >> 5], 1u << (j & 31));
    }
    __syncwarp();
    const int64_t row = static_cast<int64_t>(bh) * nb + i;
    const int nwords = (nb + 31) >> 5;
    if (lane < nwords) bitmask[row * nwords + lane] = words[lane];
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
  static thread_local int configured_scan = 0;
  if (scan_smem > 48 * 1024 && configured_scan < static_cast<int>(scan_smem)) {
    cudaError_t e = cudaFuncSetAttribute(scan_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(scan_smem));
    if (e != cudaSuccess) return e;
    configured_scan = static_cast<int>(scan_smem);
  }
  scan_order_kernel<<<1, kScanThreads, scan_smem, st>>>(R, nb, BH, row_cnt, row_ptr, work_order,
                                                        status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  expand_kernel<<<(R + 7) / 8, 256, 0, st>>>(R, nb, bitmask, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace

static size_t select_smem_bytes(int d, int nkp) {
  const int ld = d + 4;
  size_t b = static_cast<size_t>(kRQ) * ld * 4 + static_cast<size_t>(kRQ) * nkp * 4;
  b += std::max(static_cast<size_t>(kKC) * ld * 4, static_cast<size_t>(kSelWarps) * nkp * 8);
  b += kSelWarps * 32 * 4;
  return b;
}

cudaError_t launch_build_mask(const sba_plan* p, const void* qt, const void* kt,
                              const float* top_p, int top_k, uint32_t* bitmask, int32_t* row_cnt,
                              int32_t* row_ptr, int32_t* col_idx, int32_t* work_order,
                              void* workspace, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  char* ws = static_cast<char*>(workspace);
  float* qbar = reinterpret_cast<float*>(ws + p->ws_qbar);
  float* kbar = reinterpret_cast<float*>(ws + p->ws_kbar);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(ws + p->ws_ctrl);
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

  int nkp = 32;
  while (nkp < g.nb) nkp <<= 1;
  const size_t sel_smem = select_smem_bytes(g.d, nkp);
  static thread_local int configured_sel = 0;
  if (sel_smem > 48 * 1024 && configured_sel < static_cast<int>(sel_smem)) {
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sel_smem));
    if (e != cudaSuccess) return e;
    configured_sel = static_cast<int>(sel_smem);
  }
  SelectArgs sa;
  for (int h = 0; h < 256; ++h) sa.top_p[h] = h < g.H ? top_p[h] : 1.0f;
  dim3 sg((g.nb + kRQ - 1) / kRQ, BH);
  select_kernel<<<sg, kSelThreads, sel_smem, st>>>(g, qbar, kbar, sa, top_k, nkp, bitmask, row_cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  return launch_scan_expand(p, bitmask, row_cnt, row_ptr, col_idx, work_order, &ctrl->status, st);
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

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_mask_scratch[kNoAllocScratchBytes];

std::once_flag g_scratch_once[kMaxDevices];
void* g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// Device address of g_mask_scratch on the current device. The lookup runs once
// per device, on that device's first call (host code must never pass the
// symbol itself to a kernel: on the host it only names a stand-in).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_scratch_once[dev], [dev] {
    void* ptr = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&ptr, g_mask_scratch);
    g_scratch_addr[dev] = g_scratch_err[dev] == cudaSuccess ? ptr : nullptr;
  });
  *out = g_scratch_addr[dev];
  return g_scratch_err[dev];
}

size_t noalloc_scratch_need(const sba_plan* p) {
  const size_t pooled = (static_cast<size_t>(p->info.rows) * p->g.d * sizeof(float) + 255) & ~size_t(255);
  return sizeof(Ctrl) + 2 * pooled;
}

// The same four launches as launch_build_mask, with the scratch pointers given.
cudaError_t launch_build_mask_scratch(const sba_plan* p, const void* qt, const void* kt,
                                      const float* top_p, int top_k, uint32_t* bitmask,
                                      int32_t* row_cnt, int32_t* row_ptr, int32_t* col_idx,
                                      int32_t* work_order, char* scratch, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  const size_t pooled = (static_cast<size_t>(p->info.rows) * p->g.d * sizeof(float) + 255) & ~size_t(255);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(scratch);
  float* qbar = reinterpret_cast<float*>(scratch + sizeof(Ctrl));
  float* kbar = reinterpret_cast<float*>(scratch + sizeof(Ctrl) + pooled);
  const int BH = g.B * g.H;
  // the control block keeps the previous call's contents: start from zero
  cudaError_t e = cudaMemsetAsync(ctrl, 0, sizeof(Ctrl), st);
  if (e != cudaSuccess) return e;
  dim3 pg(g.nb, BH, 2);
  if (p->g.dtype == SBA_BF16)
    pool_kernel<__nv_bfloat16><<<pg, kPoolThreads, 0, st>>>(g, static_cast<const char*>(qt),
                                                            static_cast<const char*>(kt), qbar, kbar);
  else
    pool_kernel<float><<<pg, kPoolThreads, 0, st>>>(g, static_cast<const char*>(qt),
                                                    static_cast<const char*>(kt), qbar, kbar);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int nkp = 32;
  while (nkp < g.nb) nkp <<= 1;
  const size_t sel_smem = select_smem_bytes(g.d, nkp);
  if (sel_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sel_smem));
    if (e != cudaSuccess) return e;
  }
  SelectArgs sa;
  for (int h = 0; h < 256; ++h) sa.top_p[h] = h < g.H ? top_p[h] : 1.0f;
  dim3 sg((g.nb + kRQ - 1) / kRQ, BH);
  select_kernel<<<sg, kSelThreads, sel_smem, st>>>(g, qbar, kbar, sa, top_k, nkp, bitmask, row_cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int R = p->info.rows;
  const size_t scan_smem = (static_cast<size_t>(kScanWarps) * (g.nb + 1) + 2 * static_cast<size_t>(BH)) * sizeof(int);
  if (scan_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(scan_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(scan_smem));
    if (e != cudaSuccess) return e;
  }
  scan_order_kernel<<<1, kScanThreads, scan_smem, st>>>(R, g.nb, BH, row_cnt, row_ptr, work_order,
                                                        &ctrl->status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  expand_kernel<<<(R + 7) / 8, 256, 0, st>>>(R, g.nb, bitmask, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace

}  // namespace sba

extern "C" sba_status sba_build_mask_noalloc(const sba_plan* plan, const void* qt, const void* kt,
                                             const float* top_p, int32_t top_k, uint32_t* bitmask,
                                             int32_t* row_cnt, int32_t* row_ptr, int32_t* col_idx,
                                             int32_t* work_order, void* stream) {
  using namespace sba;
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
    set_error("sba_build_mask_noalloc needs %zu bytes of scratch (2*B*H*nb*d floats + 256) but "
              "its static scratch holds %zu; use sba_build_mask with a workspace",
              need, kNoAllocScratchBytes);
    return SBA_ERR_CAPACITY;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess || !scratch) {
    set_error("cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    return SBA_ERR_CUDA;
  }
  e = launch_build_mask_scratch(plan, qt, kt, top_p, top_k, bitmask, row_cnt, row_ptr, col_idx,
                                work_order, static_cast<char*>(scratch),
                                static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_error("sba_build_mask_noalloc launch: %s", cudaGetErrorString(e));
    return SBA_ERR_CUDA;
  }
  return SBA_OK;
}
