// reorder.cu -- video-aware block organization (FVAttn: Adaptive Sparse
// Attention with Runtime Load Balancing for Video Generation, abstract):
// gather raster (t, h, w) tokens into spatio-temporal cube blocks and back,
// or, in Hilbert order (DFSAttn abstract: Hilbert-curve token reordering),
// into runs of tokens along a 3-D Hilbert curve through a slot->token table.
//
// One CTA moves one cube of one (tensor, b, h): bs rows of d elements, as
// 16-byte vectors. Cube-order rows are contiguous (bs*d*esize bytes per cube)
// and raster rows of one cube line (the cube's consecutive w) are contiguous
// too, so both sides stream in long coalesced runs. Inside an edge cube the
// real tokens take the first slots, row-major over the cube's real sub-box,
// and padding the tail. Pure bit copy; padding slots are written as zeros
// (reorder) or skipped (unreorder). HBM-bound: every byte is read once and
// written once.
#include "internal.h"
#include "ptx.cuh"

namespace sba {

namespace {

constexpr int kThreads = 256;

struct ReorderArgs {
  const char* src[3];
  char* dst[3];
  const int32_t* token_of_slot;  // Hilbert order: token of every slot (-1: padding)
};

// direction 0: raster -> cube order; 1: cube order -> raster.
template <int VPR_LOG2, int DIR>
__global__ void __launch_bounds__(kThreads) reorder_kernel(KGeom g, ReorderArgs a, int esize) {
  constexpr int VPR = 1 << VPR_LOG2;  // 16-byte vectors per row
  const int z = blockIdx.z;
  const int bh = blockIdx.y;
  const int j = blockIdx.x;
  const char* __restrict__ src = a.src[z];
  char* __restrict__ dst = a.dst[z];

  uint32_t bq, h;
  g.dv_H.divmod(static_cast<uint32_t>(bh), bq, h);
  uint32_t rest, tw, tt, th;
  g.dv_nW.divmod(static_cast<uint32_t>(j), rest, tw);
  g.dv_nH.divmod(rest, tt, th);
  const int t0 = tt * g.ct, h0 = th * g.ch, w0 = tw * g.cw;
  // real sub-box of this cube; its tokens fill slots [0, len) row-major
  const int vh = min(g.ch, g.Hh - h0), vw = min(g.cw, g.W - w0);
  const int len = min(g.ct, g.T - t0) * vh * vw;
  // in-cube offsets are ranks over the real sub-box: (vh*vw, vw) divisors
  const int he = static_cast<int>(th) == g.nH - 1, we = static_cast<int>(tw) == g.nW - 1;
  const DivMod dv_area = g.dv_area[he * 2 + we];
  const DivMod dv_w = g.dv_w[we];

  const int64_t row_bytes = static_cast<int64_t>(g.d) * esize;
  const int64_t packed_base = (static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(j) * g.bs) * row_bytes;
  const int64_t raster_base = (static_cast<int64_t>(bq) * g.sB + static_cast<int64_t>(h) * g.sH) * esize;
  const int64_t sN_bytes = g.sN * esize;

  const int total = g.bs * VPR;
  constexpr int kMaxPer = 16;  // bs*VPR / kThreads <= 128*32/256
  uint4 buf[kMaxPer];
  int64_t dst_off[kMaxPer];
  bool ok[kMaxPer];
  const int per = total / kThreads;

#pragma unroll
  for (int k = 0; k < kMaxPer; ++k) {
    if (k >= per) break;
    const int idx = threadIdx.x + k * kThreads;
    const int o = idx >> VPR_LOG2;
    const int c = idx & (VPR - 1);
    bool valid;
    int64_t n;
    if (a.token_of_slot != nullptr) {
      const int32_t tok = __ldg(&a.token_of_slot[j * g.bs + o]);
      valid = tok >= 0;
      n = tok;
    } else {
      uint32_t lt, r2, lh, lw;
      dv_area.divmod(static_cast<uint32_t>(o), lt, r2);
      dv_w.divmod(r2, lh, lw);
      valid = o < len;
      n = (static_cast<int64_t>(t0 + static_cast<int>(lt)) * g.Hh + (h0 + static_cast<int>(lh))) * g.W +
          (w0 + static_cast<int>(lw));
    }
    const int64_t raster = raster_base + n * sN_bytes + c * 16;
    const int64_t packed = packed_base + static_cast<int64_t>(o) * row_bytes + c * 16;
    ok[k] = valid;
    if (DIR == 0) {
      buf[k] = valid ? __ldg(reinterpret_cast<const uint4*>(src + raster)) : make_uint4(0, 0, 0, 0);
      dst_off[k] = packed;
    } else {
      if (valid) buf[k] = __ldg(reinterpret_cast<const uint4*>(src + packed));
      dst_off[k] = raster;
    }
  }
#pragma unroll
  for (int k = 0; k < kMaxPer; ++k) {
    if (k >= per) break;
    if (DIR == 0 || ok[k]) *reinterpret_cast<uint4*>(dst + dst_off[k]) = buf[k];
  }
}

template <int DIR>
cudaError_t launch_dir(const sba_plan* p, const KGeom& g, const ReorderArgs& a, int ntens,
                       cudaStream_t st) {
  const int vpr = p->g.d * p->esize / 16;
  dim3 grid(g.nb, g.B * g.H, ntens);
  switch (vpr) {
    case 8: reorder_kernel<3, DIR><<<grid, kThreads, 0, st>>>(g, a, p->esize); break;
    case 16: reorder_kernel<4, DIR><<<grid, kThreads, 0, st>>>(g, a, p->esize); break;
    case 32: reorder_kernel<5, DIR><<<grid, kThreads, 0, st>>>(g, a, p->esize); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_reorder(const sba_plan* p, int direction, const void* src[3], void* dst[3],
                           const int32_t* token_of_slot, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  ReorderArgs a{};
  a.token_of_slot = token_of_slot;
  int n = 0;
  for (int i = 0; i < 3; ++i) {
    if (src[i] == nullptr) continue;
    a.src[n] = static_cast<const char*>(src[i]);
    a.dst[n] = static_cast<char*>(dst[i]);
    ++n;
  }
  if (n == 0) return cudaSuccess;
  return direction == 0 ? launch_dir<0>(p, g, a, n, st) : launch_dir<1>(p, g, a, n, st);
}

}  // namespace sba
