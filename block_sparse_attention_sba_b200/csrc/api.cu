// api.cu -- the C ABI of libsba: argument validation, plan geometry,
// workspace layout and the launches behind each entry point of sba.h.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <utility>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace sba {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

KGeom make_kgeom(const sba_plan* p) {
  const sba_geometry& G = p->g;
  KGeom k;
  k.B = G.B;
  k.H = G.H;
  k.T = G.T;
  k.Hh = G.Hh;
  k.W = G.W;
  k.d = G.d;
  k.ct = G.ct;
  k.ch = G.ch;
  k.cw = G.cw;
  k.bs = p->info.bs;
  k.nT = p->info.nT;
  k.nH = p->info.nH;
  k.nW = p->info.nW;
  k.nb = p->info.nb;
  k.Npad = p->info.Npad;
  k.order = G.order;
  k.N = G.T * G.Hh * G.W;
  k.tail = k.N - (k.nb - 1) * k.bs;
  k.sB = G.sB;
  k.sH = G.sH;
  k.sN = G.sN;
  k.dv_cw = DivMod(G.cw);
  k.dv_chcw = DivMod(G.ch * G.cw);
  k.dv_nW = DivMod(k.nW);
  k.dv_nH = DivMod(k.nH);
  k.dv_H = DivMod(G.H);
  k.dv_nb = DivMod(k.nb);
  const int vh_e = G.Hh - (k.nH - 1) * G.ch, vw_e = G.W - (k.nW - 1) * G.cw;
  for (int he = 0; he < 2; ++he)
    for (int we = 0; we < 2; ++we)
      k.dv_area[he * 2 + we] = DivMod((he ? vh_e : G.ch) * (we ? vw_e : G.cw));
  k.dv_w[0] = DivMod(G.cw);
  k.dv_w[1] = DivMod(vw_e);
  return k;
}

}  // namespace sba

using namespace sba;

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

static sba_status fail(sba_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

static sba_status cuda_fail(cudaError_t e, const char* what) {
  if (g_err[0] == '\0' || e != cudaErrorInvalidValue)
    snprintf(g_err, sizeof(g_err), "%s: %s", what, cudaGetErrorString(e));
  return SBA_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Position of (x, y, z) along a 3-D Hilbert curve over a 2^bits cube, after
// J. Skilling, "Programming the Hilbert curve" (2004): undo the curve's
// reflections and axis exchanges from the top bit down, Gray-encode across the
// axes, then interleave the transposed bits (top level first, axes in order).
static uint64_t hilbert3(uint32_t x, uint32_t y, uint32_t z, int bits) {
  uint32_t X[3] = {x, y, z};
  const uint32_t top = 1u << (bits - 1);
  for (uint32_t q = top; q > 1; q >>= 1) {
    const uint32_t low = q - 1;
    for (int i = 0; i < 3; ++i) {
      if (X[i] & q) {
        X[0] ^= low;
      } else {
        const uint32_t sw = (X[0] ^ X[i]) & low;
        X[0] ^= sw;
        X[i] ^= sw;
      }
    }
  }
  X[1] ^= X[0];
  X[2] ^= X[1];
  uint32_t flip = 0;
  for (uint32_t q = top; q > 1; q >>= 1)
    if (X[2] & q) flip ^= q - 1;
  for (int i = 0; i < 3; ++i) X[i] ^= flip;
  uint64_t h = 0;
  for (int b = bits - 1; b >= 0; --b)
    for (int i = 0; i < 3; ++i) h = (h << 1) | ((X[i] >> b) & 1u);
  return h;
}

// Hilbert-order tables: slot of every raster token and token of every slot.
static void build_hilbert_tables(sba_plan* p) {
  const sba_geometry& G = p->g;
  const int N = G.T * G.Hh * G.W;
  int side = std::max(G.T, std::max(G.Hh, G.W)), bits = 1;
  while ((1 << bits) < side) ++bits;
  std::vector<std::pair<uint64_t, int32_t>> key(N);
  int n = 0;
  for (int t = 0; t < G.T; ++t)
    for (int h = 0; h < G.Hh; ++h)
      for (int w = 0; w < G.W; ++w, ++n) key[n] = {hilbert3(t, h, w, bits), n};
  std::sort(key.begin(), key.end());
  p->slot_of_token.assign(N, 0);
  p->token_of_slot.assign(p->info.Npad, -1);
  for (int r = 0; r < N; ++r) {
    p->slot_of_token[key[r].second] = r;
    p->token_of_slot[r] = key[r].second;
  }
}

extern "C" {

sba_status sba_plan_create(const sba_geometry* geom, sba_plan** out) {
  g_err[0] = '\0';
  if (!geom || !out) return fail(SBA_ERR_INVALID_ARG, "geom and out must be non-NULL");
  *out = nullptr;
  const sba_geometry& G = *geom;
  if (G.B <= 0 || G.H <= 0 || G.T <= 0 || G.Hh <= 0 || G.W <= 0 || G.d <= 0 || G.ct <= 0 ||
      G.ch <= 0 || G.cw <= 0)
    return fail(SBA_ERR_INVALID_ARG, "all sizes must be positive");
  if (G.dtype != SBA_F32 && G.dtype != SBA_BF16)
    return fail(SBA_ERR_INVALID_ARG, "dtype must be SBA_F32 or SBA_BF16");
  if (G.order != SBA_ORDER_CUBE && G.order != SBA_ORDER_HILBERT)
    return fail(SBA_ERR_INVALID_ARG, "order must be SBA_ORDER_CUBE or SBA_ORDER_HILBERT");
  if (G.reserved != 0) return fail(SBA_ERR_INVALID_ARG, "reserved must be 0");
  const int64_t bs = static_cast<int64_t>(G.ct) * G.ch * G.cw;
  if (bs != 64 && bs != 128)
    return fail(SBA_ERR_UNSUPPORTED, "block size ct*ch*cw = %lld; supported: 64, 128", (long long)bs);
  if (G.dtype == SBA_BF16 && G.d != 64 && G.d != 128)
    return fail(SBA_ERR_UNSUPPORTED, "bf16 head dim %d; supported: 64, 128", G.d);
  if (G.dtype == SBA_F32 && G.d != 64)
    return fail(SBA_ERR_UNSUPPORTED, "f32 head dim %d; supported: 64", G.d);
  const int64_t nT = (G.T + G.ct - 1) / G.ct, nH = (G.Hh + G.ch - 1) / G.ch, nW = (G.W + G.cw - 1) / G.cw;
  const int64_t N = static_cast<int64_t>(G.T) * G.Hh * G.W;
  const int64_t nb = G.order == SBA_ORDER_HILBERT ? (N + bs - 1) / bs : nT * nH * nW;
  if (G.order == SBA_ORDER_HILBERT && std::max(G.T, std::max(G.Hh, G.W)) > (1 << 20))
    return fail(SBA_ERR_CAPACITY, "Hilbert order needs every grid side <= 2^20");
  if (nb > 1024) return fail(SBA_ERR_CAPACITY, "%lld blocks per head; at most 1024", (long long)nb);
  if (G.H > 256) return fail(SBA_ERR_CAPACITY, "H = %d; at most 256", G.H);
  const int64_t BH = static_cast<int64_t>(G.B) * G.H;
  if (BH > 8192) return fail(SBA_ERR_CAPACITY, "B*H = %lld; at most 8192", (long long)BH);
  const int64_t R = BH * nb;
  const int64_t Npad = nb * bs;
  if (R * nb >= (1ll << 31) || BH * Npad >= (1ll << 31) || N >= (1ll << 31))
    return fail(SBA_ERR_CAPACITY, "sizes exceed int32 indexing");
  if (G.sN < G.d || G.sH < 0 || G.sB < 0)
    return fail(SBA_ERR_INVALID_ARG, "strides must satisfy sN >= d, sH >= 0, sB >= 0");
  const int esize = G.dtype == SBA_BF16 ? 2 : 4;
  const int64_t epv = 16 / esize;
  if (G.sN % epv || G.sH % epv || G.sB % epv)
    return fail(SBA_ERR_INVALID_ARG, "strides must be multiples of %lld elements (16 bytes)", (long long)epv);

  sba_plan* p = new (std::nothrow) sba_plan();
  if (!p) return fail(SBA_ERR_CAPACITY, "out of host memory");
  p->g = G;
  p->esize = esize;
  p->info.nT = static_cast<int32_t>(nT);
  p->info.nH = static_cast<int32_t>(nH);
  p->info.nW = static_cast<int32_t>(nW);
  p->info.nb = static_cast<int32_t>(nb);
  p->info.bs = static_cast<int32_t>(bs);
  p->info.Npad = static_cast<int32_t>(Npad);
  p->info.rows = static_cast<int32_t>(R);
  p->info.words = static_cast<int32_t>((nb + 31) / 32);
  p->info.max_nnz = R * nb;
  p->ws_ctrl = 0;
  p->ws_qbar = 256;
  const size_t pooled = align256(static_cast<size_t>(R) * G.d * sizeof(double));
  p->ws_kbar = p->ws_qbar + pooled;
  // pooled scores: all heads, or as many as 48 MiB hold (at least one)
  const size_t per_head = static_cast<size_t>(nb) * nb * sizeof(double);
  const size_t all_heads = per_head * static_cast<size_t>(G.B) * G.H;
  p->scores_bytes = std::min(all_heads, std::max(per_head, size_t(48) << 20) / per_head * per_head);
  p->ws_scores = p->ws_kbar + pooled;
  p->ws_perm = p->ws_scores + align256(p->scores_bytes);
  p->info.workspace_bytes = p->ws_perm;
  if (G.order == SBA_ORDER_HILBERT) {
    build_hilbert_tables(p);
    p->info.workspace_bytes += align256(static_cast<size_t>(Npad) * sizeof(int32_t));
  }
  p->ws_heads = p->info.workspace_bytes;
  // V-Smooth's per-head words: completed-statistics counts, then maxima
  p->info.workspace_bytes += align256(2 * static_cast<size_t>(G.B) * G.H * sizeof(uint32_t));
  p->wait_budget_ns = 4000000000ull;  // 4 s: no healthy wait comes near it
  const char* env = getenv("SBA_WAIT_BUDGET_NS");
  if (env) {
    unsigned long long v = strtoull(env, nullptr, 10);
    if (v >= 1000ull && v <= 60000000000ull) p->wait_budget_ns = v;
  }
  *out = p;
  return SBA_OK;
}

void sba_plan_destroy(sba_plan* plan) { delete plan; }

sba_status sba_plan_query(const sba_plan* plan, sba_plan_info* info) {
  if (!plan || !info) return fail(SBA_ERR_INVALID_ARG, "plan and info must be non-NULL");
  *info = plan->info;
  return SBA_OK;
}

sba_status sba_workspace_init(const sba_plan* plan, void* workspace, void* stream) {
  g_err[0] = '\0';
  if (!plan || !workspace) return fail(SBA_ERR_INVALID_ARG, "plan and workspace must be non-NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(Ctrl), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  e = cudaMemsetAsync(static_cast<char*>(workspace) + plan->ws_heads, 0,
                      2 * static_cast<size_t>(plan->g.B) * plan->g.H * sizeof(uint32_t), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if (plan->g.order == SBA_ORDER_HILBERT) {
    // from pageable host memory: returns once the table has been staged
    e = cudaMemcpyAsync(static_cast<char*>(workspace) + plan->ws_perm, plan->token_of_slot.data(),
                        plan->token_of_slot.size() * sizeof(int32_t), cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(permutation)");
  }
  return SBA_OK;
}

static const int32_t* perm_table(const sba_plan* plan, const void* workspace) {
  if (plan->g.order != SBA_ORDER_HILBERT) return nullptr;
  return reinterpret_cast<const int32_t*>(static_cast<const char*>(workspace) + plan->ws_perm);
}

sba_status sba_reorder(const sba_plan* plan, const void* q, const void* k, const void* v, void* qt,
                       void* kt, void* vt, const void* workspace, void* stream) {
  g_err[0] = '\0';
  if (!plan) return fail(SBA_ERR_INVALID_ARG, "plan must be non-NULL");
  if (plan->g.order == SBA_ORDER_HILBERT && (!workspace || !aligned16(workspace)))
    return fail(SBA_ERR_INVALID_ARG, "Hilbert order needs the initialised workspace");
  const void* src[3] = {q, k, v};
  void* dst[3] = {qt, kt, vt};
  for (int i = 0; i < 3; ++i) {
    if ((src[i] == nullptr) != (dst[i] == nullptr))
      return fail(SBA_ERR_INVALID_ARG, "tensor %d: source and destination must both be NULL or both set", i);
    if (src[i] && (!aligned16(src[i]) || !aligned16(dst[i])))
      return fail(SBA_ERR_INVALID_ARG, "tensor %d: pointers must be 16-byte aligned", i);
  }
  cudaError_t e = launch_reorder(plan, 0, src, dst, perm_table(plan, workspace),
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "sba_reorder launch");
}

sba_status sba_unreorder(const sba_plan* plan, const void* ot, void* o, const void* workspace,
                         void* stream) {
  g_err[0] = '\0';
  if (!plan || !ot || !o) return fail(SBA_ERR_INVALID_ARG, "plan, ot and o must be non-NULL");
  if (plan->g.order == SBA_ORDER_HILBERT && (!workspace || !aligned16(workspace)))
    return fail(SBA_ERR_INVALID_ARG, "Hilbert order needs the initialised workspace");
  if (!aligned16(ot) || !aligned16(o)) return fail(SBA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const void* src[3] = {ot, nullptr, nullptr};
  void* dst[3] = {o, nullptr, nullptr};
  cudaError_t e = launch_reorder(plan, 1, src, dst, perm_table(plan, workspace),
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "sba_unreorder launch");
}

sba_status sba_build_mask(const sba_plan* plan, const void* qt, const void* kt, const float* top_p,
                          int32_t top_k, uint32_t* bitmask, int32_t* row_cnt, int32_t* row_ptr,
                          int32_t* col_idx, int32_t* work_order, void* workspace, void* stream) {
  g_err[0] = '\0';
  if (!plan || !qt || !kt || !top_p || !bitmask || !row_cnt || !row_ptr || !col_idx || !work_order ||
      !workspace)
    return fail(SBA_ERR_INVALID_ARG, "sba_build_mask: NULL argument");
  if (!aligned16(qt) || !aligned16(kt) || !aligned16(workspace))
    return fail(SBA_ERR_INVALID_ARG, "qt, kt and workspace must be 16-byte aligned");
  if (top_k < 0) return fail(SBA_ERR_INVALID_ARG, "top_k must be >= 0");
  for (int h = 0; h < plan->g.H; ++h) {
    const float p = top_p[h];
    if (!(p > 0.0f) || !(p <= 1.0f))
      return fail(SBA_ERR_INVALID_ARG, "top_p[%d] = %g; must lie in (0, 1]", h, (double)p);
  }
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = launch_build_mask(plan, qt, kt, top_p, top_k, bitmask, row_cnt, row_ptr, col_idx,
                                    work_order, reinterpret_cast<double*>(ws + plan->ws_qbar),
                                    reinterpret_cast<double*>(ws + plan->ws_kbar),
                                    reinterpret_cast<double*>(ws + plan->ws_scores), plan->scores_bytes,
                                    reinterpret_cast<Ctrl*>(ws + plan->ws_ctrl),
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "sba_build_mask launch");
}

sba_status sba_build_stripe_mask(const sba_plan* plan, const sba_stripe* params, uint32_t* bitmask,
                                 int32_t* row_cnt, int32_t* row_ptr, int32_t* col_idx,
                                 int32_t* work_order, void* workspace, void* stream) {
  g_err[0] = '\0';
  if (!plan || !params || !bitmask || !row_cnt || !row_ptr || !col_idx || !work_order || !workspace)
    return fail(SBA_ERR_INVALID_ARG, "sba_build_stripe_mask: NULL argument");
  if (!aligned16(workspace)) return fail(SBA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (plan->g.order != SBA_ORDER_CUBE)
    return fail(SBA_ERR_UNSUPPORTED, "stripe masks are defined on the cube grid (SBA_ORDER_CUBE)");
  for (int h = 0; h < plan->g.H; ++h) {
    const sba_stripe& q = params[h];
    const int32_t v[6] = {q.Tw, q.To, q.Ts, q.Sw, q.So, q.Ss};
    for (int k = 0; k < 6; ++k)
      if (v[k] < -32768 || v[k] > 32767)
        return fail(SBA_ERR_INVALID_ARG, "params[%d] field %d = %d; must lie in [-32768, 32767]", h, k,
                    v[k]);
    if (q.Tw < 0 || q.Ts < 0 || q.Sw < 0 || q.Ss < 0)
      return fail(SBA_ERR_INVALID_ARG, "params[%d]: widths and periods must be >= 0", h);
  }
  cudaError_t e = launch_build_stripe_mask(plan, params, bitmask, row_cnt, row_ptr, col_idx,
                                           work_order, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "sba_build_stripe_mask launch");
}

sba_status sba_smooth_v(const sba_plan* plan, const void* vt, void* vq, float* vmean, int32_t* vexp,
                        void* workspace, void* stream) {
  g_err[0] = '\0';
  if (!plan || !vt || !vq || !vmean || !vexp || !workspace)
    return fail(SBA_ERR_INVALID_ARG, "sba_smooth_v: NULL argument");
  if (plan->g.dtype != SBA_BF16 || plan->g.d > 128)
    return fail(SBA_ERR_UNSUPPORTED, "sba_smooth_v: bf16 plans with d <= 128 only");
  if (!aligned16(vt) || !aligned16(vq) || !aligned16(vmean) || !aligned16(workspace))
    return fail(SBA_ERR_INVALID_ARG, "vt, vq, vmean and workspace must be 16-byte aligned");
  cudaError_t e = launch_smooth_v(plan, vt, vq, vmean, vexp, workspace,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "sba_smooth_v launch");
}

sba_status sba_attention_lowbit(const sba_plan* plan, const void* qt, const void* kt, const void* vq,
                                const float* vmean, const int32_t* vexp, const int32_t* row_ptr,
                                const int32_t* col_idx, const int32_t* work_order, void* ot,
                                float* lse, uint64_t* trace, void* workspace, void* stream) {
  g_err[0] = '\0';
  if (!plan || !qt || !kt || !vq || !vmean || !vexp || !row_ptr || !col_idx || !work_order || !ot ||
      !workspace)
    return fail(SBA_ERR_INVALID_ARG, "sba_attention_lowbit: NULL argument");
  if (plan->g.dtype != SBA_BF16 || plan->g.d != 128 || plan->info.bs != 128)
    return fail(SBA_ERR_UNSUPPORTED, "sba_attention_lowbit: bf16 plans with d = bs = 128 only");
  if (!aligned16(qt) || !aligned16(kt) || !aligned16(vq) || !aligned16(vmean) || !aligned16(ot) ||
      !aligned16(workspace))
    return fail(SBA_ERR_INVALID_ARG, "qt, kt, vq, vmean, ot and workspace must be 16-byte aligned");
  cudaError_t e = launch_attention_lowbit(plan, qt, kt, vq, vmean, vexp, row_ptr, col_idx, work_order,
                                          ot, lse, trace, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "sba_attention_lowbit launch");
}

sba_status sba_attention(const sba_plan* plan, const void* qt, const void* kt, const void* vt,
                         const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work_order,
                         void* ot, float* lse, int32_t sched, uint64_t* trace, void* workspace,
                         void* stream) {
  g_err[0] = '\0';
  if (!plan || !qt || !kt || !vt || !row_ptr || !col_idx || !ot || !workspace)
    return fail(SBA_ERR_INVALID_ARG, "sba_attention: NULL argument");
  if (sched != SBA_SCHED_LPT && sched != SBA_SCHED_HEAD_MAJOR)
    return fail(SBA_ERR_INVALID_ARG, "sched must be SBA_SCHED_LPT or SBA_SCHED_HEAD_MAJOR");
  if (sched == SBA_SCHED_LPT && !work_order && plan->g.dtype == SBA_BF16)
    return fail(SBA_ERR_INVALID_ARG, "SBA_SCHED_LPT needs work_order");
  if (!aligned16(qt) || !aligned16(kt) || !aligned16(vt) || !aligned16(ot))
    return fail(SBA_ERR_INVALID_ARG, "qt, kt, vt and ot must be 16-byte aligned");
  cudaError_t e = launch_attention(plan, qt, kt, vt, row_ptr, col_idx, work_order, ot, lse, sched,
                                   trace, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "sba_attention launch");
}

sba_status sba_check_device_status(const sba_plan* plan, void* workspace, void* stream) {
  g_err[0] = '\0';
  if (!plan || !workspace) return fail(SBA_ERR_INVALID_ARG, "plan and workspace must be non-NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t word = 0;
  e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
  e = cudaMemset(workspace, 0, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status)");
  if (word & kStatusTimeout) return fail(SBA_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up");
  if (word & kStatusCheck) return fail(SBA_ERR_DEVICE_CHECK, "a device-side input check failed");
  return SBA_OK;
}

sba_status sba_debug_timeout_probe(const sba_plan* plan, void* workspace, uint64_t timeout_ns,
                                   void* stream) {
  g_err[0] = '\0';
  if (!plan || !workspace) return fail(SBA_ERR_INVALID_ARG, "plan and workspace must be non-NULL");
  if (timeout_ns < 1000ull || timeout_ns > 10000000000ull)
    return fail(SBA_ERR_INVALID_ARG, "timeout_ns must lie in [1e3, 1e10]");
  cudaError_t e = launch_timeout_probe(workspace, timeout_ns, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "timeout probe launch");
}

sba_status sba_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  g_err[0] = '\0';
  if (n < 0 || n > (int64_t(1) << 31)) return fail(SBA_ERR_INVALID_ARG, "n must lie in [0, 2^31]");
  if (n == 0) return SBA_OK;
  if (!x || !y) return fail(SBA_ERR_INVALID_ARG, "x and y must be non-NULL");
  cudaError_t e = launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SBA_OK : cuda_fail(e, "exp2 polynomial launch");
}

sba_status sba_perm_export(const sba_plan* plan, int32_t* slot_of_token) {
  if (!plan || !slot_of_token) return fail(SBA_ERR_INVALID_ARG, "plan and output must be non-NULL");
  const sba_geometry& G = plan->g;
  if (G.order == SBA_ORDER_HILBERT) {
    std::copy(plan->slot_of_token.begin(), plan->slot_of_token.end(), slot_of_token);
    return SBA_OK;
  }
  const int nH = plan->info.nH, nW = plan->info.nW, bs = plan->info.bs;
  int64_t n = 0;
  for (int t = 0; t < G.T; ++t)
    for (int h = 0; h < G.Hh; ++h)
      for (int w = 0; w < G.W; ++w, ++n) {
        const int th = h / G.ch, tw = w / G.cw;
        const int blk = ((t / G.ct) * nH + th) * nW + tw;
        // rank inside the cube's real sub-box (vh x vw in h and w)
        const int vh = std::min(G.ch, G.Hh - th * G.ch), vw = std::min(G.cw, G.W - tw * G.cw);
        const int off = ((t % G.ct) * vh + h % G.ch) * vw + w % G.cw;
        slot_of_token[n] = blk * bs + off;
      }
  return SBA_OK;
}

int32_t sba_attention_grid_size(void) { return attention_grid_size(); }

const char* sba_status_string(sba_status s) {
  switch (s) {
    case SBA_OK: return "SBA_OK";
    case SBA_ERR_INVALID_ARG: return "SBA_ERR_INVALID_ARG";
    case SBA_ERR_UNSUPPORTED: return "SBA_ERR_UNSUPPORTED";
    case SBA_ERR_CUDA: return "SBA_ERR_CUDA";
    case SBA_ERR_CAPACITY: return "SBA_ERR_CAPACITY";
    case SBA_ERR_DEVICE_TIMEOUT: return "SBA_ERR_DEVICE_TIMEOUT";
    case SBA_ERR_DEVICE_CHECK: return "SBA_ERR_DEVICE_CHECK";
  }
  return "SBA_ERR_UNKNOWN";
}

const char* sba_last_error(void) { return g_err; }

}  // extern "C"
