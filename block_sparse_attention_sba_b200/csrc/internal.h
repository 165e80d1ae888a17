// internal.h -- the plan and the launchers shared by the library's sources.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/sba.h"

struct sba_plan {
  sba_geometry g;
  sba_plan_info info;
  int esize;               // bytes per element (2 or 4)
  size_t ws_ctrl;          // offset of the control block (status, counters)
  size_t ws_qbar, ws_kbar; // offsets of the pooled means (fp64 [B*H][nb][d])
  size_t ws_scores, scores_bytes;  // pooled scores of a chunk of heads (fp64 [heads][nb][nb])
  size_t ws_perm;          // Hilbert order: offset of token_of_slot (int32 [Npad])
  size_t ws_heads;         // sba_smooth_v per-(b, h) words: counts, then maxima (uint32 [2][B*H], zero between calls)
  uint64_t wait_budget_ns; // bounded-wait limit for device waits
  std::vector<int32_t> slot_of_token;  // Hilbert order: int32 [N]
  std::vector<int32_t> token_of_slot;  // Hilbert order: int32 [Npad], -1 = padding
};

namespace sba {

// Control block at the start of every workspace (256 bytes, zero at rest).
struct Ctrl {
  uint32_t status;        // kStatusTimeout | kStatusCheck bits
  uint32_t work_next;     // persistent scheduler: next work_order index
  uint32_t cta_done;      // persistent scheduler: CTAs that finished
  uint32_t aux_next;      // sba_smooth_v: next work item
  uint32_t aux_done;      // sba_smooth_v: CTAs that finished
  uint32_t scan_done;     // mask: head-scan CTAs that finished
  uint32_t pad[58];
};
static_assert(sizeof(Ctrl) == 256, "control block is 256 bytes");

// Fast unsigned division by a runtime constant (multiply-high + shift),
// valid for dividends below 2^31.
struct DivMod {
  uint32_t d, mul, shr;
  __host__ __device__ DivMod() : d(1), mul(0), shr(0) {}
  __host__ explicit DivMod(uint32_t div) : d(div) {
    shr = 0;
    while ((1u << shr) < div) ++shr;
    // mul = ceil(2^(32+shr) / d) - 2^32 fits in 32 bits for d >= 1
    uint64_t m = ((1ull << (32 + shr)) + div - 1) / div;
    mul = static_cast<uint32_t>(m - (1ull << 32));
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    uint32_t t = __umulhi(n, mul);
    return (t + n) >> shr;  // (t + n) < 2^32 for n < 2^31
  }
  __device__ __forceinline__ void divmod(uint32_t n, uint32_t& q, uint32_t& r) const {
    q = div(n);
    r = n - q * d;
  }
};

// Geometry in the form the kernels take by value.
struct KGeom {
  int32_t B, H, T, Hh, W, d, ct, ch, cw, bs, nT, nH, nW, nb, Npad;
  int32_t order;  // sba_order
  int32_t N;      // tokens per head
  int32_t tail;   // Hilbert order: real tokens in the last block
  int64_t sB, sH, sN;
  DivMod dv_cw, dv_chcw, dv_nW, dv_nH, dv_H, dv_nb;
  // in-cube rank divisors of the cube kinds along h and w: index
  // (last cube along h) * 2 + (last cube along w); area = vh*vw, then vw
  DivMod dv_area[4], dv_w[2];
};

KGeom make_kgeom(const sba_plan* p);

// Real-token extents of cube block j (cube order): the cube's sub-box inside
// the grid.
__device__ __forceinline__ void cube_extents(const KGeom& g, int j, int& vt, int& vh, int& vw) {
  uint32_t rest, tw, tt, th;
  g.dv_nW.divmod(static_cast<uint32_t>(j), rest, tw);
  g.dv_nH.divmod(rest, tt, th);
  vt = min(g.ct, g.T - static_cast<int>(tt) * g.ct);
  vh = min(g.ch, g.Hh - static_cast<int>(th) * g.ch);
  vw = min(g.cw, g.W - static_cast<int>(tw) * g.cw);
}

// Number of real tokens of block j. In both orders they occupy the block's
// first slots (cube order: row-major over the cube's real sub-box; Hilbert
// order: only the last block is partial), so slot o of block j is real iff
// o < block_len(g, j).
__device__ __forceinline__ int block_len(const KGeom& g, int j) {
  if (g.order == SBA_ORDER_HILBERT) return j == g.nb - 1 ? g.tail : g.bs;
  int vt, vh, vw;
  cube_extents(g, j, vt, vh, vw);
  return vt * vh * vw;
}

// Launchers (return cudaError_t of the launch).
cudaError_t launch_reorder(const sba_plan* p, int direction, const void* src[3], void* dst[3],
                           const int32_t* token_of_slot, cudaStream_t st);
// The four mask launches with their scratch given: pooled means qbar, kbar
// (fp64 [B*H][nb][d] each) and the status word that device checks set.
cudaError_t launch_build_mask(const sba_plan* p, const void* qt, const void* kt,
                              const float* top_p, int top_k, uint32_t* bitmask, int32_t* row_cnt,
                              int32_t* row_ptr, int32_t* col_idx, int32_t* work_order,
                              double* qbar, double* kbar, double* scores, size_t scores_bytes,
                              Ctrl* ctrl, cudaStream_t st);
cudaError_t launch_build_stripe_mask(const sba_plan* p, const sba_stripe* params,
                                     uint32_t* bitmask, int32_t* row_cnt, int32_t* row_ptr,
                                     int32_t* col_idx, int32_t* work_order, void* workspace,
                                     cudaStream_t st);
cudaError_t launch_attention(const sba_plan* p, const void* qt, const void* kt, const void* vt,
                             const int32_t* row_ptr, const int32_t* col_idx,
                             const int32_t* work_order, void* ot, float* lse, int sched,
                             uint64_t* trace, void* workspace, cudaStream_t st);
cudaError_t launch_timeout_probe(void* workspace, uint64_t timeout_ns, cudaStream_t st);
cudaError_t launch_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t st);

cudaError_t launch_smooth_v(const sba_plan* p, const void* vt, void* vq, float* vmean,
                            int32_t* vexp, void* workspace, cudaStream_t st);
cudaError_t launch_attention_lowbit(const sba_plan* p, const void* qt, const void* kt, const void* vq,
                                    const float* vmean, const int32_t* vexp, const int32_t* row_ptr,
                                    const int32_t* col_idx, const int32_t* work_order, void* ot,
                                    float* lse, uint64_t* trace, void* workspace, cudaStream_t st);

// Set by launch_attention when it fails before a launch for a reason that is
// not a CUDA error (e.g. the tensor-map encoder is unavailable).
void set_error(const char* fmt, ...);

int attention_grid_size();

}  // namespace sba
