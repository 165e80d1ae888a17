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
// Two launches: per-block means and residual maxima, then per-block
// quantisation (each CTA reduces its head's maxima to e).
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace sba {

namespace {

constexpr int kSmoothThreads = 128;  // one thread per channel (d <= 128)

// Real-token test of slot o of block j (cube or Hilbert order): the real
// tokens are the block's first block_len slots.
__device__ __forceinline__ bool slot_real(const KGeom& g, int j, int o) { return o < block_len(g, j); }

// grid (nb, B*H): mu_j (fp32) and max |V - mu_j| over the block's real slots.
__global__ void __launch_bounds__(kSmoothThreads)
    smooth_stats_kernel(KGeom g, const __nv_bfloat16* __restrict__ vt, float* __restrict__ vmean,
                        float* __restrict__ block_amax) {
  const int j = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  const int64_t base = (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * g.d;
  __shared__ float red[kSmoothThreads / 32];
  float mu = 0.f;
  if (c < g.d) {
    double sum = 0.0;
    int cnt = 0;
    for (int o = 0; o < g.bs; ++o) {
      if (!slot_real(g, j, o)) continue;
      sum += static_cast<double>(__bfloat162float(vt[base + static_cast<int64_t>(o) * g.d + c]));
      ++cnt;
    }
    mu = static_cast<float>(sum / static_cast<double>(cnt));
    vmean[(static_cast<int64_t>(bh) * g.nb + j) * g.d + c] = mu;
  }
  float amax = 0.f;
  if (c < g.d) {
    for (int o = 0; o < g.bs; ++o) {
      if (!slot_real(g, j, o)) continue;
      const float r = __bfloat162float(vt[base + static_cast<int64_t>(o) * g.d + c]) - mu;
      amax = fmaxf(amax, fabsf(r));
    }
  }
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((c & 31) == 0) red[c >> 5] = amax;
  __syncthreads();
  if (c == 0) {
    float m = red[0];
    for (int w = 1; w < kSmoothThreads / 32; ++w) m = fmaxf(m, red[w]);
    block_amax[static_cast<int64_t>(bh) * g.nb + j] = m;
  }
}

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

// grid (nb, B*H): codes of block j, transposed to [d][bs].
__global__ void __launch_bounds__(kSmoothThreads)
    smooth_quant_kernel(KGeom g, const __nv_bfloat16* __restrict__ vt,
                        const float* __restrict__ vmean, const float* __restrict__ block_amax,
                        uint8_t* __restrict__ vq, int32_t* __restrict__ vexp) {
  const int j = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  __shared__ float red[kSmoothThreads / 32];
  float amax = 0.f;
  for (int k = c; k < g.nb; k += kSmoothThreads)
    amax = fmaxf(amax, block_amax[static_cast<int64_t>(bh) * g.nb + k]);
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((c & 31) == 0) red[c >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int w = 1; w < kSmoothThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const int e = scale_exponent(amax);
  if (j == 0 && c == 0) vexp[bh] = e;
  if (c >= g.d) return;
  const float inv = ldexpf(1.0f, -e);  // exact power of two
  const float mu = vmean[(static_cast<int64_t>(bh) * g.nb + j) * g.d + c];
  const int64_t src = (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * g.d + c;
  uint8_t* dst = vq + ((static_cast<int64_t>(bh) * g.nb + j) * g.d + c) * g.bs;
  for (int k0 = 0; k0 < g.bs; k0 += 16) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int o = k0 + 4 * q + u;
        x[u] = slot_real(g, j, o)
                   ? (__bfloat162float(vt[src + static_cast<int64_t>(o) * g.d]) - mu) * inv
                   : 0.f;
      }
      w[q] = e4m3x2(x[0], x[1]) | (e4m3x2(x[2], x[3]) << 16);
    }
    *reinterpret_cast<uint4*>(dst + k0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_smooth_v(const sba_plan* p, const void* vt, void* vq, float* vmean,
                            int32_t* vexp, void* workspace, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  // per-block residual maxima live in the pooled-means area of the workspace
  float* block_amax = reinterpret_cast<float*>(static_cast<char*>(workspace) + p->ws_qbar);
  dim3 grid(g.nb, g.B * g.H);
  smooth_stats_kernel<<<grid, kSmoothThreads, 0, st>>>(g, static_cast<const __nv_bfloat16*>(vt),
                                                       vmean, block_amax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  smooth_quant_kernel<<<grid, kSmoothThreads, 0, st>>>(g, static_cast<const __nv_bfloat16*>(vt),
                                                       vmean, block_amax,
                                                       static_cast<uint8_t*>(vq), vexp);
  return cudaGetLastError();
}

}  // namespace sba
