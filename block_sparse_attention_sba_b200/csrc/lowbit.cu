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

constexpr int kSmoothBufs = 2;  // blocks staged per CTA

// Per staged block: the item, and for a quantisation item the head's e.
struct SmoothSlot {
  uint32_t item;
  int32_t e;
};

// Warp roles: warps 0..7 process blocks (kSmoothThreads threads), warp 8
// produces: it takes items from the counter, resolves a quantisation item's
// dependency (the head's statistics complete), reads the head's exponent and
// the block's means, and stages the block with one bulk copy into a ring of
// kSmoothBufs buffers (full / empty mbarriers).
//
// Statistics item, one pass over the staged block: per channel the fp64 sum
// and the fp32 minimum and maximum over the real rows (thread = channel pair x
// row group, rows strided by the group count), combined in group order.
// mu = fp32(sum / len); max |R| over the block = max(vmax - mu, mu - vmin) in
// fp32 (rounding is monotone, so the largest |fl(v - mu)| is at the largest
// or the smallest v).
// Quantisation item, one pass: thread = 4 channels x 16 rows; codes of one
// channel's 16 rows are one 16-byte store. The consumer warps meet only inside
// a statistics item (an mbarrier, bounded waits) and otherwise run through
// the ring independently.
__global__ void __launch_bounds__(kSmoothThreads + 32)
    smooth_v_kernel(KGeom g, SmoothArgs a) {
  extern __shared__ __align__(128) unsigned char sm_raw[];  // [bufs][bs][d] bf16, then [bufs][d] f32
  // groups * d = 512 for d = 64 and 128 (groups = 2 * kSmoothThreads / d)
  __shared__ double dsum[512];                // [groups][d] partial sums
  __shared__ float dmin[512], dmax[512];      // [groups][d] partial minima / maxima
  __shared__ float red[kSmoothThreads / 32];
  __shared__ __align__(8) uint64_t full[kSmoothBufs], empty[kSmoothBufs], sbar;
  __shared__ SmoothSlot slot[kSmoothBufs];
  __shared__ int s_abort;
  const int tid = threadIdx.x, d = g.d, nb = g.nb;
  const int BH = g.B * g.H;
  const uint32_t n_items = 2u * static_cast<uint32_t>(BH) * static_cast<uint32_t>(nb);
  const uint32_t buf_bytes = static_cast<uint32_t>(g.bs * d * 2);
  float* means = reinterpret_cast<float*>(sm_raw + kSmoothBufs * buf_bytes);
  uint32_t* status = &a.ctrl->status;
  uint32_t* head_max = a.heads + BH;
  volatile int* abort_flag = &s_abort;
  if (tid == 0) {
    for (int b = 0; b < kSmoothBufs; ++b) {
      mbar_init(smem_u32(&full[b]), 1);
      mbar_init(smem_u32(&empty[b]), kSmoothThreads / 32);
    }
    mbar_init(smem_u32(&sbar), kSmoothThreads);  // the consumers' own barrier
    fence_barrier_init();
    s_abort = 0;
  }
  __syncthreads();
  if (tid >= kSmoothThreads) {
    // ---------------------------------------------------------- producer
    const int lane = tid & 31;
    uint32_t issued = 0;  // ring uses issued (lane 0)
    for (uint32_t k = 0;; ++k) {
      const int b = static_cast<int>(k % kSmoothBufs);
      const uint32_t use = k / kSmoothBufs;
      uint32_t item = 0;
      if (lane == 0) item = atomicAdd(&a.ctrl->aux_next, 1u);
      item = __shfl_sync(0xffffffffu, item, 0);
      bool quant = false;
      int bh = 0, j = 0, e = 0;
      if (item < n_items) {
        smooth_item(item, nb, BH, a.lag, quant, bh, j);
        if (quant && lane == 0) {
          // every statistics item of the head done (bounded wait)
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_gpu(a.heads + bh) < static_cast<uint32_t>(nb)) {
            if (*abort_flag) break;
            if (globaltimer_ns() - t0 > a.budget_ns) {
              atomicOr(status, kStatusTimeout);
              *abort_flag = 1;
              break;
            }
            __nanosleep(64);
          }
          e = scale_exponent(__uint_as_float(ld_acquire_gpu(head_max + bh)));
        }
        __syncwarp();
      }
      // the buffer's previous block processed (bounded wait)
      bool ok = true;
      if (use > 0) ok = mbar_wait(smem_u32(&empty[b]), (use - 1) & 1u, a.budget_ns, abort_flag, status);
      // leave together (the lanes below exchange values)
      if (__any_sync(0xffffffffu, !ok || *abort_flag)) break;
      if (item < n_items && quant) {
        // the block's means (written before the head's count moved)
        const float* src = a.vmean + (static_cast<int64_t>(bh) * nb + j) * d;
        for (int c = lane; c < d / 4; c += 32)
          reinterpret_cast<float4*>(means + b * d)[c] = __ldcg(reinterpret_cast<const float4*>(src) + c);
      }
      __syncwarp();
      if (lane == 0) {
        slot[b].item = item < n_items ? item : n_items;
        slot[b].e = e;
        const uint32_t bar = smem_u32(&full[b]);
        if (item < n_items) {
          const uint32_t bytes = static_cast<uint32_t>(block_len(g, j) * d * 2);
          const __nv_bfloat16* src =
              a.vt + (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * d;
          fence_proxy_async_smem();  // the buffer's previous reads come first
          mbar_arrive_expect_tx(bar, bytes);
          bulk_load_1d(smem_u32(sm_raw + b * buf_bytes), src, bytes, bar);
          ++issued;
        } else {
          mbar_arrive(bar);  // end of work: the consumers see the sentinel
        }
      }
      if (item >= n_items) break;
    }
    if (lane == 0 && *abort_flag) {
      // copies possibly in flight after an abort: bounded wait for the last
      // issued use of each buffer
      for (uint32_t u = (issued > kSmoothBufs ? issued - kSmoothBufs : 0u); u < issued; ++u) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(smem_u32(&full[u % kSmoothBufs]), (u / kSmoothBufs) & 1u) &&
               globaltimer_ns() - t0 < a.budget_ns) {
        }
      }
    }
  } else {
    // --------------------------------------------------------- consumers
    const int warp = tid >> 5, lane = tid & 31;
    const int npair = d / 2, groups = kSmoothThreads / npair;
    const int nq = d / 4, nrg = g.bs / 16;
    uint32_t sph = 0;  // phases of sbar passed (the same count in every consumer)
    // all consumers meet (bounded wait); false once the CTA aborts
    auto consumers_meet = [&]() {
      mbar_arrive(smem_u32(&sbar));
      const bool ok = mbar_wait(smem_u32(&sbar), sph & 1u, a.budget_ns, abort_flag, status);
      ++sph;
      return ok;
    };
    for (uint32_t k = 0;; ++k) {
      const int b = static_cast<int>(k % kSmoothBufs);
      const uint32_t use = k / kSmoothBufs;
      // warps leave as a whole (lanes exchange values below); a warp that
      // leaves after an abort ends the other consumers' waits through the
      // abort flag, since every wait here is an mbarrier wait
      const bool got = mbar_wait(smem_u32(&full[b]), use & 1u, a.budget_ns, abort_flag, status);
      if (__any_sync(0xffffffffu, !got)) break;
      const uint32_t item = slot[b].item;
      if (item >= n_items) break;
      bool quant;
      int bh, j;
      smooth_item(item, nb, BH, a.lag, quant, bh, j);
      const int len = block_len(g, j);
      const unsigned char* blk = sm_raw + b * buf_bytes;
      if (!quant) {
        const int cp = tid % npair, rg = tid / npair;
        const uint32_t* w = reinterpret_cast<const uint32_t*>(blk);
        double s0 = 0.0, s1 = 0.0;
        float mn0 = INFINITY, mn1 = INFINITY, mx0 = -INFINITY, mx1 = -INFINITY;
        for (int o = rg; o < len; o += groups) {
          const uint32_t v = w[o * npair + cp];
          const float f0 = __uint_as_float(v << 16), f1 = __uint_as_float(v & 0xffff0000u);
          s0 += static_cast<double>(f0);
          s1 += static_cast<double>(f1);
          mn0 = fminf(mn0, f0);
          mn1 = fminf(mn1, f1);
          mx0 = fmaxf(mx0, f0);
          mx1 = fmaxf(mx1, f1);
        }
        dsum[rg * d + 2 * cp] = s0;
        dsum[rg * d + 2 * cp + 1] = s1;
        dmin[rg * d + 2 * cp] = mn0;
        dmin[rg * d + 2 * cp + 1] = mn1;
        dmax[rg * d + 2 * cp] = mx0;
        dmax[rg * d + 2 * cp + 1] = mx1;
        if (__any_sync(0xffffffffu, !consumers_meet())) break;
        if (tid < d) {
          double t = 0.0;
          float vmin = INFINITY, vmax = -INFINITY;
          for (int r = 0; r < groups; ++r) {
            t += dsum[r * d + tid];
            vmin = fminf(vmin, dmin[r * d + tid]);
            vmax = fmaxf(vmax, dmax[r * d + tid]);
          }
          const float mu = static_cast<float>(t / static_cast<double>(len));
          a.vmean[(static_cast<int64_t>(bh) * nb + j) * d + tid] = mu;
          float am = fmaxf(0.f, fmaxf(vmax - mu, mu - vmin));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
          if (lane == 0) red[warp] = am;
        }
        if (__any_sync(0xffffffffu, !consumers_meet())) break;
        if (tid == 0) {
          float am = red[0];
          for (int w2 = 1; w2 < d / 32; ++w2) am = fmaxf(am, red[w2]);
          // non-negative floats order like their bit patterns
          atomicMax(head_max + bh, __float_as_uint(am));
          __threadfence();  // means and maximum before the count (after the barrier above)
          atomicAdd(a.heads + bh, 1u);
        }
      } else {
        const int e = slot[b].e;
        if (tid == 0 && j == 0) a.vexp[bh] = e;
        const float inv = ldexpf(1.0f, -e);  // exact power of two
        const float2 inv2 = make_float2(inv, inv), nz2 = make_float2(-0.0f, -0.0f);
        const float* mu = means + b * d;
        uint8_t* dst = a.vq + (static_cast<int64_t>(bh) * nb + j) * d * g.bs;
        for (int idx = tid; idx < nq * nrg; idx += kSmoothThreads) {
          const int cq = idx % nq, rg = idx / nq;
          const float4 m4 = *reinterpret_cast<const float4*>(mu + 4 * cq);
          const float2 nm01 = make_float2(-m4.x, -m4.y), nm23 = make_float2(-m4.z, -m4.w);
          uint32_t wc[4][4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            // rows rg*16 + 4q .. +3: x[u][c] for channel c of the quad
            float x[4][4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int o = rg * 16 + 4 * q + u;
              if (o < len) {
                const uint2 v = *reinterpret_cast<const uint2*>(blk + (static_cast<size_t>(o) * d + 4 * cq) * 2);
                // R = v - mu (fp32), then R * 2^-e (exact: -0 addend keeps signs)
                const float2 r01 = ffma2(fadd2(make_float2(__uint_as_float(v.x << 16),
                                                           __uint_as_float(v.x & 0xffff0000u)),
                                               nm01),
                                         inv2, nz2);
                const float2 r23 = ffma2(fadd2(make_float2(__uint_as_float(v.y << 16),
                                                           __uint_as_float(v.y & 0xffff0000u)),
                                               nm23),
                                         inv2, nz2);
                x[u][0] = r01.x;
                x[u][1] = r01.y;
                x[u][2] = r23.x;
                x[u][3] = r23.y;
              } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) x[u][c] = 0.f;
              }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
              wc[c][q] = e4m3x2(x[0][c], x[1][c]) | (e4m3x2(x[2][c], x[3][c]) << 16);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(4 * cq + c) * g.bs + rg * 16) =
                make_uint4(wc[c][0], wc[c][1], wc[c][2], wc[c][3]);
        }
      }
      // this warp is done with the buffer
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[b]));
    }
  }
  __syncthreads();
  if (tid == 0) {
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
  const int smem = kSmoothBufs * (g.bs * g.d * 2 + g.d * 4);
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(smooth_v_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, smooth_v_kernel, kSmoothThreads + 32, smem);
  if (e != cudaSuccess) return e;
  // persistent: every CTA resident at once (a quantisation item waits on
  // statistics items that resident CTAs took earlier)
  const int64_t items = 2ll * g.B * g.H * g.nb;
  const int grid = static_cast<int>(std::min<int64_t>(items, static_cast<int64_t>(std::max(1, per_sm)) * sms));
  // Lag: the items taken between a head's last statistics item and its first
  // quantisation item ((2L-1) nb) cover twice the items the CTAs hold (a
  // ring's worth and one more each), so a quantisation item rarely waits;
  // capped so that the lagged heads' values (L heads of nb blocks) stay
  // within 48 MiB of L2.
  const int64_t BH = static_cast<int64_t>(g.B) * g.H;
  const int64_t head_bytes = static_cast<int64_t>(g.nb) * g.bs * g.d * 2;
  const int64_t held = static_cast<int64_t>(grid) * (kSmoothBufs + 1);
  int64_t lag = ((2 * held + g.nb - 1) / g.nb + 2) / 2;
  lag = std::min(lag, std::max<int64_t>(1, (int64_t(48) << 20) / head_bytes));
  a.lag = static_cast<int>(std::max<int64_t>(1, std::min(lag, BH)));
  smooth_v_kernel<<<grid, kSmoothThreads + 32, smem, st>>>(g, a);
  return cudaGetLastError();
}

}  // namespace sba
