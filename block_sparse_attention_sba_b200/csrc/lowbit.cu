// lowbit.cu -- V-Smooth value quantisation for the low-bit P.V path
// (VC-Attention: Value Smoothing and Softmax Casting for Low-bit Attention,
// abstract: quantise only the residual after subtracting the block mean and
// restore the mean from the row sums).
//
// For every key block j of a head: mu_j = mean of V over the block's real
// tokens (summed in fp64, rounded once to fp32); R = V - mu_j in fp32 (zero on
// padding slots); one power-of-two scale per head, 2^e with e the smallest
// integer such that max|R| <= 448 * 2^e (e = 0 when R is all zero); codes =
// E4M3(R * 2^-e) with round-to-nearest-even and saturation. The codes of a
// block are stored transposed, [d][bs] bytes, so that a block is a K-major
// operand of the fp8 tensor-core product (rows = channels, keys contiguous).
//
// One persistent launch. Work items are per block: a statistics item (mu_j,
// the block's max |R|, folded into the head's maximum with an integer atomic
// max on the float's bits, which orders non-negative floats) and a
// quantisation item (needs the head's e, i.e. every statistics item of the
// head). Items are taken from a counter in the order S0 .. S(L-1), S(L),
// Q0, S(L+1), Q1, ..., S(BH-1), Q(BH-1-L), then Q(BH-L) .. Q(BH-1) (S:
// statistics of a head's blocks, Q: its quantisation; the lag L, in heads,
// grows with the items in flight, see the launcher), so a quantisation item
// only waits on items that resident CTAs have already taken (bounded wait on
// the head's completed-statistics count), and it re-reads its block a few
// heads after the statistics pass read it, from L2. Each CTA takes its next
// item while it works on the current one and stages that item's block with
// one bulk asynchronous copy into the second of two shared-memory buffers, so
// the load of one block overlaps the arithmetic on the other. A quantisation item recomputes its
// block's means from the staged copy (the same code in the same order, so
// the same bits as the statistics item wrote). The last CTA resets the
// counters.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sba {

namespace {

constexpr int kSmoothThreads = 256;

// Smallest e with amax <= 448 * 2^e (0 for amax == 0), exact in fp32.
__device__ __forceinline__ int scale_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int e;
  frexpf(amax / 448.0f, &e);  // first guess, then settle it exactly
  while (amax > ldexpf(448.0f, e)) ++e;
  while (e > -149 && amax <= ldexpf(448.0f, e - 1)) --e;
  return e;
}

// Two fp32 values -> two E4M3 codes, lo in bits 0..7 (RNE, saturating).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

struct SmoothArgs {
  const __nv_bfloat16* vt;
  uint8_t* vq;
  float* vmean;
  int32_t* vexp;
  uint32_t* heads;      // [B*H] statistics items completed, then [B*H] the
                        // head's max |R| as float bits (all zero between calls)
  Ctrl* ctrl;
  uint64_t budget_ns;
  int lag;              // heads between a head's statistics and its quantisation
};

// Item number -> (quantisation?, head bh, block j). Segments of nb items:
// S0 .. S(L-1), then S(h), Q(h-L) for h = L .. BH-1, then Q(BH-L) .. Q(BH-1)
// (S: a head's statistics, Q: its quantisation, L: the lag in heads,
// 1 <= L <= BH). Every S(h) comes before every Q(h).
__device__ __forceinline__ void smooth_item(uint32_t item, int nb, int BH, int L, bool& quant,
                                            int& bh, int& j) {
  const int seg = static_cast<int>(item / static_cast<uint32_t>(nb));
  j = static_cast<int>(item - static_cast<uint32_t>(seg) * static_cast<uint32_t>(nb));
  if (seg < L) {
    quant = false;
    bh = seg;
  } else if (seg < L + 2 * (BH - L)) {
    const int t = seg - L, h = L + t / 2;
    quant = (t & 1) != 0;
    bh = quant ? h - L : h;
  } else {
    quant = true;
    bh = seg - BH;
  }
}

__device__ __forceinline__ float block_max_f(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kSmoothThreads / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// Per-channel means of the staged block's len real rows into smu[0..d):
// thread = (channel pair, row group), fp64 sums, one division, one rounding
// to fp32. Deterministic: both item kinds get the same bits.
__device__ __forceinline__ void block_means(const __nv_bfloat162* b2, int len, int d, double* dsum,
                                            float* smu) {
  const int tid = threadIdx.x, npair = d / 2, groups = kSmoothThreads / npair;
  const int cp = tid % npair, rg = tid / npair;
  double s0 = 0.0, s1 = 0.0;
  for (int o = rg; o < len; o += groups) {
    const float2 f = __bfloat1622float2(b2[o * npair + cp]);
    s0 += static_cast<double>(f.x);
    s1 += static_cast<double>(f.y);
  }
  dsum[2 * tid] = s0;
  dsum[2 * tid + 1] = s1;
  __syncthreads();
  if (tid < d) {
    double t = 0.0;
    for (int r = 0; r < groups; ++r) t += dsum[2 * (r * npair + tid / 2) + (tid & 1)];
    smu[tid] = static_cast<float>(t / static_cast<double>(len));
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSmoothThreads)
    smooth_v_kernel(KGeom g, SmoothArgs a) {
  extern __shared__ __align__(128) unsigned char sm_raw[];  // two [bs][d] bf16 buffers
  __shared__ double dsum[2 * kSmoothThreads];
  __shared__ float red[kSmoothThreads / 32];
  __shared__ float smu[128];
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t s_item[2];
  __shared__ int s_abort, s_e;
  const int tid = threadIdx.x, d = g.d, nb = g.nb;
  const int BH = g.B * g.H;
  const int npair = d / 2;
  const uint32_t n_items = 2u * static_cast<uint32_t>(BH) * static_cast<uint32_t>(nb);
  const uint32_t buf_bytes = static_cast<uint32_t>(g.bs * d * 2);
  uint32_t* status = &a.ctrl->status;
  uint32_t* head_max = a.heads + BH;
  // thread 0: uses of each buffer issued and waited for (a copy still in
  // flight when the loop ends early is waited for before the CTA exits)
  uint32_t issued0 = 0u, issued1 = 0u, waited0 = 0u, waited1 = 0u;
  auto issue = [&](uint32_t it, int b) {
    bool qq;
    int bh, j;
    smooth_item(it, nb, BH, a.lag, qq, bh, j);
    const uint32_t bytes = static_cast<uint32_t>(block_len(g, j) * d * 2);
    const __nv_bfloat16* src = a.vt + (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * d;
    const uint32_t bar = smem_u32(&bars[b]);
    fence_proxy_async_smem();  // the buffer's previous reads come first
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load_1d(smem_u32(sm_raw + b * buf_bytes), src, bytes, bar);
    if (b) ++issued1; else ++issued0;
  };
  if (tid == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    fence_barrier_init();
    s_abort = 0;
    const uint32_t first = atomicAdd(&a.ctrl->aux_next, 1u);
    s_item[0] = first;
    if (first < n_items) issue(first, 0);
  }
  __syncthreads();
  for (uint32_t k = 0;; ++k) {
    const int buf = static_cast<int>(k & 1u);
    const uint32_t item = s_item[buf];
    if (item >= n_items) break;
    if (tid == 0) {
      // take the next item and start its copy into the other buffer (free:
      // the previous item's reads ended at its closing barrier)
      const uint32_t next = atomicAdd(&a.ctrl->aux_next, 1u);
      s_item[buf ^ 1] = next;
      if (next < n_items) issue(next, buf ^ 1);
    }
    bool quant;
    int bh, j;
    smooth_item(item, nb, BH, a.lag, quant, bh, j);
    const int len = block_len(g, j);
    const bool got = mbar_wait(smem_u32(&bars[buf]), (k >> 1) & 1u, a.budget_ns, &s_abort, status);
    if (tid == 0 && got) {
      if (buf) ++waited1; else ++waited0;
    }
    __syncthreads();
    if (s_abort) break;
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(sm_raw + buf * buf_bytes);
    block_means(b2, len, d, dsum, smu);
    const int cp = tid % npair, rg = tid / npair, groups = kSmoothThreads / npair;
    if (!quant) {
      if (tid < d) a.vmean[(static_cast<int64_t>(bh) * nb + j) * d + tid] = smu[tid];
      const float mu0 = smu[2 * cp], mu1 = smu[2 * cp + 1];
      float amax = 0.f;
      for (int o = rg; o < len; o += groups) {
        const float2 f = __bfloat1622float2(b2[o * npair + cp]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x - mu0), fabsf(f.y - mu1)));
      }
      amax = block_max_f(amax, red);
      if (tid == 0) {
        // non-negative floats order like their bit patterns
        atomicMax(head_max + bh, __float_as_uint(amax));
        __threadfence();  // means and maximum before the count (after the barrier above)
        atomicAdd(a.heads + bh, 1u);
      }
    } else {
      if (tid == 0) {
        // wait until every statistics item of the head is done
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(a.heads + bh) < static_cast<uint32_t>(nb)) {
          if (globaltimer_ns() - t0 > a.budget_ns) {
            atomicOr(status, kStatusTimeout);
            break;
          }
          __nanosleep(128);
        }
        const int e = scale_exponent(__uint_as_float(ld_acquire_gpu(head_max + bh)));
        s_e = e;
        if (j == 0) a.vexp[bh] = e;
      }
      __syncthreads();
      const float inv = ldexpf(1.0f, -s_e);  // exact power of two
      // 32 codes of two channels per thread: one 32-byte sector per channel
      uint8_t* dst = a.vq + (static_cast<int64_t>(bh) * nb + j) * d * g.bs;
      const int nhg = g.bs / 32;
      for (int idx = tid; idx < npair * nhg; idx += kSmoothThreads) {
        const int c2 = idx % npair, hg = idx / npair;
        const float mu0 = smu[2 * c2], mu1 = smu[2 * c2 + 1];
        uint32_t w0[8], w1[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float x0[4], x1[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int o = hg * 32 + 4 * q + u;
            if (o < len) {
              const float2 f = __bfloat1622float2(b2[o * npair + c2]);
              x0[u] = (f.x - mu0) * inv;
              x1[u] = (f.y - mu1) * inv;
            } else {
              x0[u] = 0.f;
              x1[u] = 0.f;
            }
          }
          w0[q] = e4m3x2(x0[0], x0[1]) | (e4m3x2(x0[2], x0[3]) << 16);
          w1[q] = e4m3x2(x1[0], x1[1]) | (e4m3x2(x1[2], x1[3]) << 16);
        }
        uint4* p0 = reinterpret_cast<uint4*>(dst + static_cast<int64_t>(2 * c2) * g.bs + hg * 32);
        uint4* p1 = reinterpret_cast<uint4*>(dst + static_cast<int64_t>(2 * c2 + 1) * g.bs + hg * 32);
        p0[0] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
        p0[1] = make_uint4(w0[4], w0[5], w0[6], w0[7]);
        p1[0] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
        p1[1] = make_uint4(w1[4], w1[5], w1[6], w1[7]);
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
    // copies still in flight (only after a timed-out wait): bounded wait
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const uint32_t iss = b ? issued1 : issued0, wt = b ? waited1 : waited0;
      if (iss > wt) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(smem_u32(&bars[b]), (iss - 1u) & 1u) &&
               globaltimer_ns() - t0 < a.budget_ns) {
        }
      }
    }
    // the last CTA out resets the work counter and the head words
    __threadfence();
    const uint32_t prev = atomicAdd(&a.ctrl->aux_done, 1u);
    if (prev == gridDim.x - 1) {
      for (int h = 0; h < 2 * BH; ++h) a.heads[h] = 0u;
      atomicExch(&a.ctrl->aux_next, 0u);
      atomicExch(&a.ctrl->aux_done, 0u);
      __threadfence();
    }
  }
}

}  // namespace

cudaError_t launch_smooth_v(const sba_plan* p, const void* vt, void* vq, float* vmean,
                            int32_t* vexp, void* workspace, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  char* ws = static_cast<char*>(workspace);
  SmoothArgs a;
  a.vt = static_cast<const __nv_bfloat16*>(vt);
  a.vq = static_cast<uint8_t*>(vq);
  a.vmean = vmean;
  a.vexp = vexp;
  a.heads = reinterpret_cast<uint32_t*>(ws + p->ws_heads);
  a.ctrl = reinterpret_cast<Ctrl*>(ws + p->ws_ctrl);
  a.budget_ns = p->wait_budget_ns;
  const int smem = 2 * g.bs * g.d * 2;
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(smooth_v_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, smooth_v_kernel, kSmoothThreads, smem);
  if (e != cudaSuccess) return e;
  // persistent: every CTA resident at once (a quantisation item waits on
  // statistics items that resident CTAs took earlier)
  const int64_t items = 2ll * g.B * g.H * g.nb;
  const int grid = static_cast<int>(std::min<int64_t>(items, static_cast<int64_t>(std::max(1, per_sm)) * sms));
  // Lag: the items taken between a head's last statistics item and its first
  // quantisation item ((2L-1) nb) cover twice the items the CTAs hold (two
  // each), so a quantisation item rarely waits; capped so that the lagged
  // heads' values (L heads of nb blocks) stay within 48 MiB of L2.
  const int64_t BH = static_cast<int64_t>(g.B) * g.H;
  const int64_t head_bytes = static_cast<int64_t>(g.nb) * g.bs * g.d * 2;
  int64_t lag = ((4ll * grid + g.nb - 1) / g.nb + 2) / 2;
  lag = std::min(lag, std::max<int64_t>(1, (int64_t(48) << 20) / head_bytes));
  a.lag = static_cast<int>(std::max<int64_t>(1, std::min(lag, BH)));
  smooth_v_kernel<<<grid, kSmoothThreads, smem, st>>>(g, a);
  return cudaGetLastError();
}

}  // namespace sba
