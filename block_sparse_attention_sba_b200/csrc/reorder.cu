// reorder.cu -- video-aware block organization (FVAttn: Adaptive Sparse
// Attention with Runtime Load Balancing for Video Generation, abstract):
// gather raster (t, h, w) tokens into spatio-temporal cube blocks and back,
// or, in Hilbert order (DFSAttn abstract: Hilbert-curve token reordering),
// into runs of tokens along a 3-D Hilbert curve through a slot->token table.
//
// General strides (and Hilbert order): one CTA moves one cube of one
// (tensor, b, h): bs rows of d elements, as 16-byte vectors. Cube-order rows
// are contiguous (bs*d*esize bytes per cube) and raster rows of one cube line
// (the cube's consecutive w) are contiguous too. When the raster's token rows
// are contiguous ([B][H][N][d]) a CTA moves a whole row of cubes instead, so
// the raster side is whole lines of W tokens (reorder_rows_kernel). Inside an edge cube the
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
  // cube-row kernel: vectors per raster line (W * d * esize / 16), and the
  // cube heights along h (ch, and the last cube's)
  DivMod dv_line, dv_vh[2];
};

// direction 0: raster -> cube order; 1: cube order -> raster.
template <int VPR_LOG2, int DIR>
__global__ void __launch_bounds__(kThreads) reorder_kernel(KGeom g, ReorderArgs a, int esize) {
  constexpr int VPR = 1 << VPR_LOG2;  // 16-byte vectors per row
  const int z = blockIdx.z;
  const int bh = blockIdx.y;
  const int j = blockIdx.x;
  // (selects, not a dynamic index: that would copy the argument array to
  // local memory)
  const char* __restrict__ src = z == 0 ? a.src[0] : (z == 1 ? a.src[1] : a.src[2]);
  char* __restrict__ dst = z == 0 ? a.dst[0] : (z == 1 ? a.dst[1] : a.dst[2]);

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

// Cube order with token rows contiguous in the raster (sN == d, the
// [B][H][N][d] layout): one CTA moves one row of cubes (all cubes (tt, th, *))
// of one (tensor, b, h). On the raster side that is vt*vh whole raster lines
// of W tokens, each a contiguous run of W*d elements; on the cube side it is
// nW consecutive blocks. Thread k takes the 16-byte vectors k, k + 256, ... of
// the row's lines in raster order, so both sides stream in long runs (a warp
// covers 512 contiguous bytes on each side except where a line crosses into
// the next cube). reorder also zero-fills the cubes' padding slots.
template <int VPR_LOG2, int DIR>
__global__ void __launch_bounds__(kThreads) reorder_rows_kernel(KGeom g, ReorderArgs a, int esize) {
  constexpr int VPR = 1 << VPR_LOG2;
  constexpr int kUnroll = 8;
  const int z = blockIdx.z;
  const int bh = blockIdx.y;
  const int cr = blockIdx.x;  // cube row tt * nH + th
  // (selects, not a dynamic index: that would copy the argument array to
  // local memory)
  const char* __restrict__ src = z == 0 ? a.src[0] : (z == 1 ? a.src[1] : a.src[2]);
  char* __restrict__ dst = z == 0 ? a.dst[0] : (z == 1 ? a.dst[1] : a.dst[2]);
  uint32_t bq, h, tt, th;
  g.dv_H.divmod(static_cast<uint32_t>(bh), bq, h);
  g.dv_nH.divmod(static_cast<uint32_t>(cr), tt, th);
  const int t0 = tt * g.ct, h0 = th * g.ch;
  const int he = static_cast<int>(th) == g.nH - 1;
  const int vt = min(g.ct, g.T - t0), vh = min(g.ch, g.Hh - h0);
  const int vw_last = g.W - (g.nW - 1) * g.cw;
  const DivMod dv_vh = a.dv_vh[he];
  const int total = vt * vh * g.W * VPR;
  const int64_t row_bytes = static_cast<int64_t>(g.d) * esize;
  const char* src_head;
  char* dst_head;
  const int64_t packed_head = static_cast<int64_t>(bh) * g.Npad * row_bytes;
  const int64_t raster_head = (static_cast<int64_t>(bq) * g.sB + static_cast<int64_t>(h) * g.sH) * esize;
  src_head = src + (DIR == 0 ? raster_head : packed_head);
  dst_head = dst + (DIR == 0 ? packed_head : raster_head);
  const int jrow = cr * g.nW;
  for (int base = 0; base < total; base += kThreads * kUnroll) {
    uint4 buf[kUnroll];
    int64_t doff[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int idx = base + u * kThreads + static_cast<int>(threadIdx.x);
      doff[u] = -1;
      if (idx < total) {
        uint32_t line, rem, lt, lh, tw, lw;
        a.dv_line.divmod(static_cast<uint32_t>(idx), line, rem);
        const int w = static_cast<int>(rem >> VPR_LOG2), c = static_cast<int>(rem & (VPR - 1));
        dv_vh.divmod(line, lt, lh);
        g.dv_cw.divmod(static_cast<uint32_t>(w), tw, lw);
        const int vw = static_cast<int>(tw) == g.nW - 1 ? vw_last : g.cw;
        const int o = (static_cast<int>(lt) * vh + static_cast<int>(lh)) * vw + static_cast<int>(lw);
        const int64_t packed = (static_cast<int64_t>(jrow + static_cast<int>(tw)) * g.bs + o) * row_bytes + c * 16;
        const int64_t raster =
            ((static_cast<int64_t>(t0 + static_cast<int>(lt)) * g.Hh + h0 + static_cast<int>(lh)) * g.W + w) *
                row_bytes + c * 16;
        buf[u] = __ldg(reinterpret_cast<const uint4*>(src_head + (DIR == 0 ? raster : packed)));
        doff[u] = DIR == 0 ? packed : raster;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (doff[u] >= 0) *reinterpret_cast<uint4*>(dst_head + doff[u]) = buf[u];
  }
  if (DIR == 0) {
    // padding slots [len, bs) of every cube of the row, as zeros
    for (int tw = 0; tw < g.nW; ++tw) {
      const int vw = tw == g.nW - 1 ? vw_last : g.cw;
      const int len = vt * vh * vw;
      const int64_t blk = packed_head + static_cast<int64_t>(jrow + tw) * g.bs * row_bytes;
      for (int v = len * VPR + static_cast<int>(threadIdx.x); v < g.bs * VPR; v += kThreads)
        *reinterpret_cast<uint4*>(dst + blk + static_cast<int64_t>(v) * 16) = make_uint4(0, 0, 0, 0);
    }
  }
}

template <int DIR>
cudaError_t launch_rows(const sba_plan* p, const KGeom& g, ReorderArgs a, int ntens, cudaStream_t st) {
  const int vpr = p->g.d * p->esize / 16;
  a.dv_line = DivMod(static_cast<uint32_t>(g.W * vpr));
  a.dv_vh[0] = DivMod(static_cast<uint32_t>(g.ch));
  a.dv_vh[1] = DivMod(static_cast<uint32_t>(g.Hh - (g.nH - 1) * g.ch));
  dim3 grid(g.nT * g.nH, g.B * g.H, ntens);
  switch (vpr) {
    case 8: reorder_rows_kernel<3, DIR><<<grid, kThreads, 0, st>>>(g, a, p->esize); break;
    case 16: reorder_rows_kernel<4, DIR><<<grid, kThreads, 0, st>>>(g, a, p->esize); break;
    case 32: reorder_rows_kernel<5, DIR><<<grid, kThreads, 0, st>>>(g, a, p->esize); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
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
  // cube order over a raster whose token rows are contiguous: whole-line kernel
  const bool rows = token_of_slot == nullptr && g.sN == g.d;
  if (rows) return direction == 0 ? launch_rows<0>(p, g, a, n, st) : launch_rows<1>(p, g, a, n, st);
  return direction == 0 ? launch_dir<0>(p, g, a, n, st) : launch_dir<1>(p, g, a, n, st);
}

}  // namespace sba
