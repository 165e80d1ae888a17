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
// One persistent launch. Work items are per block: a statistics item (mu_j
// and the block's max |R|) and a quantisation item (needs the head's e, i.e.
// every statistics item of the head). Items are taken from a counter in the
// order S0, S1, Q0, S2, Q1, ..., S(BH-1), Q(BH-2), Q(BH-1) (S: statistics of
// a head's blocks, Q: its quantisation), so a quantisation item only waits on
// items that resident CTAs have already taken (bounded wait on the head's
// completed-statistics count), and it re-reads its block about two heads
// after the statistics pass read it, from L2. Both item kinds stage the block
// in shared memory with 16-byte loads. The last CTA resets the counters.
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
  float* block_amax;    // [B*H][nb]
  uint32_t* heads;      // [B*H] statistics items completed (zero between calls)
  Ctrl* ctrl;
  uint64_t budget_ns;
};

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

__global__ void __launch_bounds__(kSmoothThreads)
    smooth_v_kernel(KGeom g, SmoothArgs a) {
  extern __shared__ __align__(16) unsigned char sm_raw[];
  __nv_bfloat16* blk = reinterpret_cast<__nv_bfloat16*>(sm_raw);  // [bs][d]
  __shared__ double dsum[kSmoothThreads];
  __shared__ float red[kSmoothThreads / 32];
  __shared__ float smu[128];
  __shared__ int s_item;
  const int tid = threadIdx.x, d = g.d, nb = g.nb;
  const int BH = g.B * g.H;
  const int vpr = d / 8;  // 16-byte vectors per row
  const uint32_t n_items = 2u * static_cast<uint32_t>(BH) * static_cast<uint32_t>(nb);
  uint32_t* status = &a.ctrl->status;
  for (;;) {
    if (tid == 0) s_item = static_cast<int>(atomicAdd(&a.ctrl->aux_next, 1u));
    __syncthreads();
    const uint32_t item = static_cast<uint32_t>(s_item);
    __syncthreads();
    if (item >= n_items) break;
    const uint32_t seg = item / static_cast<uint32_t>(nb);
    const int j = static_cast<int>(item - seg * static_cast<uint32_t>(nb));
    bool quant;
    int bh;
    if (seg == 0) {
      quant = false;
      bh = 0;
    } else if (seg & 1u) {
      bh = static_cast<int>((seg + 1) / 2);
      quant = bh >= BH;
      if (quant) bh = BH - 1;
    } else {
      quant = true;
      bh = static_cast<int>(seg / 2) - 1;
    }
    const int len = block_len(g, j);
    const __nv_bfloat16* src = a.vt + (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * d;
    if (quant) {
      // wait until every statistics item of the head is done
      if (tid == 0) {
        const uint64_t t0 = globaltimer_ns();
        volatile uint32_t* cnt = a.heads + bh;
        while (*cnt < static_cast<uint32_t>(nb)) {
          if (globaltimer_ns() - t0 > a.budget_ns) {
            atomicOr(status, kStatusTimeout);
            break;
          }
          __nanosleep(256);
        }
        __threadfence();
      }
      __syncthreads();
    }
    // stage the block's real rows (16-byte loads, four in flight per thread)
    const int nvec = len * vpr;
    for (int v0 = tid; v0 < nvec; v0 += 4 * kSmoothThreads) {
      uint4 r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * kSmoothThreads;
        if (v < nvec) r[u] = __ldg(reinterpret_cast<const uint4*>(src) + v);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * kSmoothThreads;
        if (v < nvec) reinterpret_cast<uint4*>(blk)[v] = r[u];
      }
    }
    __syncthreads();
    if (!quant) {
      // per-channel sums in fp64 over the real rows: thread = (row group, channel)
      const int groups = kSmoothThreads / d;
      const int c = tid % d, rg = tid / d;
      double sum = 0.0;
      for (int o = rg; o < len; o += groups) sum += static_cast<double>(__bfloat162float(blk[o * d + c]));
      dsum[tid] = sum;
      __syncthreads();
      if (tid < d) {
        double t = 0.0;
        for (int r = 0; r < groups; ++r) t += dsum[r * d + tid];
        const float mu = static_cast<float>(t / static_cast<double>(len));
        smu[tid] = mu;
        a.vmean[(static_cast<int64_t>(bh) * nb + j) * d + tid] = mu;
        __threadfence();  // visible device-wide before the head count moves
      }
      __syncthreads();
      float amax = 0.f;
      const float mu = smu[c];
      for (int o = rg; o < len; o += groups)
        amax = fmaxf(amax, fabsf(__bfloat162float(blk[o * d + c]) - mu));
      amax = block_max_f(amax, red);
      if (tid == 0) {
        a.block_amax[static_cast<int64_t>(bh) * nb + j] = amax;
        __threadfence();
        atomicAdd(a.heads + bh, 1u);
      }
    } else {
      // the head's exponent from its blocks' maxima
      float amax = 0.f;
      for (int k = tid; k < nb; k += kSmoothThreads)
        amax = fmaxf(amax, __ldcg(&a.block_amax[static_cast<int64_t>(bh) * nb + k]));
      amax = block_max_f(amax, red);
      const int e = scale_exponent(amax);
      if (j == 0 && tid == 0) a.vexp[bh] = e;
      const float inv = ldexpf(1.0f, -e);  // exact power of two
      if (tid < d) smu[tid] = __ldcg(&a.vmean[(static_cast<int64_t>(bh) * nb + j) * d + tid]);
      __syncthreads();
      // 16 codes of one channel per store: (channel, group of 16 slots)
      uint8_t* dst = a.vq + (static_cast<int64_t>(bh) * nb + j) * d * g.bs;
      const int ng = g.bs / 16;
      for (int idx = tid; idx < d * ng; idx += kSmoothThreads) {
        const int c = idx % d, og = idx / d;
        const float mu = smu[c];
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float x[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int o = og * 16 + 4 * q + u;
            x[u] = o < len ? (__bfloat162float(blk[o * d + c]) - mu) * inv : 0.f;
          }
          w[q] = e4m3x2(x[0], x[1]) | (e4m3x2(x[2], x[3]) << 16);
        }
        *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(c) * g.bs + og * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncthreads();
  }
  // the last CTA out resets the work counter and the head counters
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&a.ctrl->aux_done, 1u);
    if (prev == gridDim.x - 1) {
      for (int h = 0; h < BH; ++h) a.heads[h] = 0u;
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
  // per-block residual maxima live in the pooled-means area of the workspace
  a.block_amax = reinterpret_cast<float*>(ws + p->ws_qbar);
  a.heads = reinterpret_cast<uint32_t*>(ws + p->ws_heads);
  a.ctrl = reinterpret_cast<Ctrl*>(ws + p->ws_ctrl);
  a.budget_ns = p->wait_budget_ns;
  const int smem = g.bs * g.d * 2;
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
  smooth_v_kernel<<<grid, kSmoothThreads, smem, st>>>(g, a);
  return cudaGetLastError();
}

}  // namespace sba
