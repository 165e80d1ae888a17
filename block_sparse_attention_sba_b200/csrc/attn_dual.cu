// attn_dual.cu -- block-sparse attention forward on B200 tensor cores, two
// query tiles in flight per CTA (FVAttn: Adaptive Sparse Attention with
// Runtime Load Balancing for Video Generation, abstract: attention over the
// materialised Top-p / Top-k block mask, uneven per-head workloads taken by a
// longest-first scheduler; VC-Attention, abstract: on datacenter GPUs the
// exponential between the two products is a co-bottleneck of attention).
//
// Block size 128, head dim 64 or 128, bf16 operands, fp32 accumulation.
// Work item = one mask row (b, h, query block i): its 128-row query tile and
// the row's selected key blocks. A persistent CTA runs two items at once, one
// per "lane" L = 0, 1, each with its own query tile in shared memory and its
// own S and O accumulators in tensor memory (TMEM columns: S_L at 128*L, O_L
// at 256 + 128*L). Per key block j of a lane's row:
//   S_L = Q_L K_j^T      tcgen05.mma kind::f16, N cut to the block's real keys
//                        rounded up to 16
//   P = exp2(S*c - ref)  one TMEM lane (query row) per softmax thread, the
//                        whole row of S in registers; P rounded to bf16 and
//                        written back over S in TMEM
//   O_L += P V_j         tcgen05.mma with A = P from TMEM, K cut like N
// A lane's chain S -> softmax -> P.V is serial, and each lane's tensor-core
// work waits on its softmax; the other lane's products fill that gap: the
// issuer alternates between the lanes.
// Warp roles (384 threads, one CTA per SM):
//   warps 0-3 / 4-7   softmax and epilogue of lane 0 / lane 1 (one thread per
//                     query row: no exchange of row maxima between warps)
//   warp 8            MMA issuer of both lanes (one thread; it alternates
//                     between the lanes, which keeps one lane's products
//                     running while the other lane's softmax works) and
//                     TMEM owner
//   warps 9, 10       producer of lane 0 / lane 1 (one thread each): takes
//                     rows from the work order, TMA-loads the Q tile and the
//                     K and V tiles through the lane's ring of 16 KB slots
//                     (d = 128: per key block the two 64-column panels of K,
//                     then V in two halves of 64 keys; d = 64: K, then V). A
//                     slot is reused once the product that read it has
//                     completed; the S and P.V completions the issuer commits
//                     anyway tell the producer so (two commits per block).
// The reference max of a row is the first block's row max; a later block
// whose P may exceed 2^24 (its row sum exceeds 128 * 2^24) moves the
// reference up and scales O, the row sum and its own P down together (rare;
// bf16 P up to 2^24 keep O and the row sum far inside fp32 range, and the
// final normalisation uses the same reference, so the result is exact up to
// rounding). Every other
// pair of exponentials runs on the FMA pipe (a polynomial) to relieve MUFU.
// Padding keys (the tail of a partial block) are masked to -inf; padding
// query rows are written as 0. Every wait is bounded (status bit + clean
// exit).
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sba {

namespace {

constexpr int kDualSmemLimit = 232448;  // 227 KB: opt-in shared memory per CTA

template <int D>
struct DCfg {
  static constexpr int BS = 128;
  static constexpr int THREADS = 384;  // three warpgroups
  static constexpr int WARP_ISS = 8;   // MMA issuer of both lanes
  static constexpr int WARP_PROD = 9;  // producer of lane L: warp 9 + L (warp 11 idles)
  // Register split: launched at 168 per thread (384 x 168 = 64512 in the
  // CTA's pool), warpgroup 2 (issuer, producers) drops to 88, freeing
  // 128 x 80 = 10240; the two softmax warpgroups rise to 208, taking
  // 256 x 40 = 10240: the whole row of S stays in registers.
  static constexpr uint32_t REGS_LOW = 88, REGS_HIGH = 208;
  static_assert(128 * (168 - REGS_LOW) >= 256 * (REGS_HIGH - 168), "register split exceeds the pool");
  static constexpr int Q_BYTES = 128 * D * 2;   // one lane's query tile
  static constexpr int PANEL = 128 * 128;       // 128 rows x 64 bf16
  static constexpr int SLOT = 16384;            // ring unit
  static constexpr int NK = D / 64;             // K positions per key block
  static constexpr int PPB = 2 * NK;            // ring positions per key block
  // Slot reuse is told by the S / P.V completions of the block that read it.
  // The producer observes those completions in order; the depth below keeps
  // the next block's product from completing before the producer has seen
  // the one it waits for (so an mbarrier phase is never skipped).
  static constexpr int NSLOT = PPB + NK - 1;
  static constexpr int CTRL = 1024;
  static constexpr int SMEM = 1024 + 2 * Q_BYTES + 2 * NSLOT * SLOT + CTRL;
  // A block's P stay below 2^24 (its row sum below 128 * 2^24) while the
  // reference trails the row max by at most 24 (log2): bf16 P that large
  // keep O and the row sum far inside fp32 range. A block beyond that moves
  // the reference (rare).
  static constexpr float MAX_BLOCK_SUM = 128.0f * 16777216.0f;
  static constexpr uint32_t COL_O = 256;
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
  // per-lane barriers: item full (2), item empty (2), Q full, slot full
  // (NSLOT), S done, P.V done, P ready, O free, drain
  static constexpr int B_IF = 0, B_IE = 2, B_QF = 4, B_SF = 5, B_SD = B_SF + NSLOT, B_PD = B_SD + 1,
                       B_PF = B_PD + 1, B_OE = B_PF + 1, B_DR = B_OE + 1, NBL = B_DR + 1;
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static_assert(SMEM <= kDualSmemLimit, "shared memory budget");
  static_assert(2 * NBL * 8 + 128 <= CTRL, "control area");
};

struct DualParams {
  KGeom g;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* work_order;
  __nv_bfloat16* ot;
  float* lse;
  uint64_t* trace;
  Ctrl* ctrl;
  int R;
  int sched;
  int64_t max_nnz;
  uint64_t budget_ns;
  float scale_log2;
};

__device__ __forceinline__ bool dual_wait_drain(uint32_t bar, uint32_t parity, uint64_t budget_ns,
                                                uint32_t* status) {
  volatile int never = 0;
  return mbar_wait(bar, parity, budget_ns, &never, status);
}

template <int D>
__global__ void __launch_bounds__(DCfg<D>::THREADS, 1)
    attn_dual_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const DualParams P) {
  using C = DCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = sm;                          // [2][Q_BYTES]
  unsigned char* sRing = sm + 2 * C::Q_BYTES;      // [2][NSLOT][SLOT]
  unsigned char* ctl = sRing + 2 * C::NSLOT * C::SLOT;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctl);                 // [2][NBL]
  int* iring = reinterpret_cast<int*>(ctl + 2 * C::NBL * 8);          // [2 lanes][2][4]
  int* lenrec = iring + 16;  // [2 lanes][NSLOT]: real keys of the block whose K panel 0 is in the slot
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 2 * C::NBL * 8 + 112);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 2 * C::NBL * 8 + 116);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const KGeom& g = P.g;
  uint32_t* status = &P.ctrl->status;
  const uint64_t budget = P.budget_ns;
  auto bar = [&](int L, int i) -> uint32_t { return smem_u32(&bars[L * C::NBL + i]); };

  if (threadIdx.x == 0) {
    for (int L = 0; L < 2; ++L) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(bar(L, C::B_IF + b), 1);
        mbar_init(bar(L, C::B_IE + b), 1 + 4);  // the issuer and the four softmax warps
      }
      mbar_init(bar(L, C::B_QF), 1);
      for (int s = 0; s < C::NSLOT; ++s) mbar_init(bar(L, C::B_SF + s), 1);
      mbar_init(bar(L, C::B_SD), 1);
      mbar_init(bar(L, C::B_PD), 1);
      mbar_init(bar(L, C::B_PF), 4);
      mbar_init(bar(L, C::B_OE), 4);
      mbar_init(bar(L, C::B_DR), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::WARP_ISS) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= C::WARP_ISS) {
   regs_dec<C::REGS_LOW>();  // warpgroup 2: issuer, producers, one idle warp
   if (warp >= C::WARP_PROD) {
    // ------------------------------------------------ producer of lane L
    const int L = warp - C::WARP_PROD;
    if (lane == 0 && L < 2) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint32_t ring = smem_u32(sRing + L * C::NSLOT * C::SLOT);
      uint32_t items = 0, qloads = 0, gk = 0, pos = 0;
      int slot = 0;  // pos % NSLOT
      bool hm = P.sched == SBA_SCHED_HEAD_MAJOR && 2 * static_cast<int>(blockIdx.x) + L < P.R;
      bool ok = true;
      auto wait = [&](int b, uint32_t parity) -> bool {
        return mbar_wait(bar(L, b), parity, budget, abort_flag, status);
      };
      // one ring position: its slot and full barrier, then advance
      auto next_slot = [&](uint32_t& dst, uint32_t& fb) {
        dst = ring + slot * C::SLOT;
        fb = bar(L, C::B_SF + slot);
        ++pos;
        slot = slot + 1 == C::NSLOT ? 0 : slot + 1;
      };
      while (ok) {
        const int is = items & 1;
        if (items >= 2) {
          ok = wait(C::B_IE + is, ((items >> 1) - 1) & 1);
          if (!ok) break;
        }
        int row = -1;
        if (P.sched == SBA_SCHED_LPT) {
          const int idx = static_cast<int>(atomicAdd(&P.ctrl->work_next, 1u));
          if (idx < P.R) {
            row = __ldg(&P.work_order[idx]);
            if (row < 0 || row >= P.R) {
              atomicOr(status, kStatusCheck);
              continue;  // skip this entry
            }
          }
        } else if (hm) {
          row = 2 * static_cast<int>(blockIdx.x) + L;
          hm = false;
        }
        int start = 0, n = 0;
        if (row >= 0) {
          start = __ldg(&P.row_ptr[row]);
          n = __ldg(&P.row_ptr[row + 1]) - start;
          if (n < 0 || n > g.nb || start < 0 || static_cast<int64_t>(start) + n > P.max_nnz) {
            atomicOr(status, kStatusCheck);
            n = 0;  // a row that cannot be read is skipped (written as empty)
            start = 0;
          }
        }
        int* e = iring + (L * 2 + is) * 4;
        e[0] = row;
        e[1] = n;
        e[2] = start;
        mbar_arrive(bar(L, C::B_IF + is));
        ++items;
        if (row < 0) break;
        if (n == 0) continue;
        uint32_t bh, iq;
        g.dv_nb.divmod(static_cast<uint32_t>(row), bh, iq);
        const int hrow = static_cast<int>(bh) * g.Npad;
        int jn = __ldg(&P.col_idx[start]);
        for (int k = 0; k < n && ok; ++k) {
          int j = jn;
          if (j < 0 || j >= g.nb) {
            atomicOr(status, kStatusCheck);
            j = 0;
          }
          if (k + 1 < n) jn = __ldg(&P.col_idx[start + k + 1]);
          const int len = block_len(g, j);
          const int krow = hrow + j * C::BS;
          // Block gk's K panels (and, d = 128, its first V half) reuse the
          // slots of block gk-1's K panels: S(gk-1) must be done. Each
          // completion is waited for once, in order.
          if (gk >= 1) {
            ok = wait(C::B_SD, (gk - 1) & 1);
            if (!ok) break;
          }
          if (k == 0) {
            // every S product of the lane's previous rows is done: Q is free
            const uint32_t dq = smem_u32(sQ + L * C::Q_BYTES);
            mbar_arrive_expect_tx(bar(L, C::B_QF), C::Q_BYTES);
            const int qrow = hrow + static_cast<int>(iq) * C::BS;
            for (int p = 0; p < D / 64; ++p)
              for (int hf = 0; hf < 2; ++hf)
                tma_load_2d(dq + p * C::PANEL + hf * (C::PANEL / 2), &tmQ, p * 64, qrow + hf * 64,
                            bar(L, C::B_QF));
            ++qloads;
          }
          const bool two = len > 64;  // rows 64.. hold real keys
          uint32_t dst, fb;
          lenrec[L * C::NSLOT + slot] = len;  // published by the slot's full barrier
          for (int sub = 0; sub < C::NK; ++sub) {
            // K panel `sub` (columns 64*sub ..)
            next_slot(dst, fb);
            mbar_arrive_expect_tx(fb, two ? C::SLOT : C::SLOT / 2);
            tma_load_2d(dst, &tmK, sub * 64, krow, fb);
            if (two) tma_load_2d(dst + C::SLOT / 2, &tmK, sub * 64, krow + 64, fb);
          }
          if (D == 128) {
            // V keys 0..63, both column panels
            next_slot(dst, fb);
            mbar_arrive_expect_tx(fb, C::SLOT);
            tma_load_2d(dst, &tmV, 0, krow, fb);
            tma_load_2d(dst + C::SLOT / 2, &tmV, 64, krow, fb);
          }
          // the last V position reuses block gk-1's last V slot: P.V(gk-1) done
          if (gk >= 1) {
            ok = wait(C::B_PD, (gk - 1) & 1);
            if (!ok) break;
          }
          next_slot(dst, fb);
          if (D == 128) {
            // V keys 64..127
            if (two) {
              mbar_arrive_expect_tx(fb, C::SLOT);
              tma_load_2d(dst, &tmV, 0, krow + 64, fb);
              tma_load_2d(dst + C::SLOT / 2, &tmV, 64, krow + 64, fb);
            } else {
              mbar_arrive(fb);  // nothing to read
            }
          } else {
            mbar_arrive_expect_tx(fb, two ? C::SLOT : C::SLOT / 2);
            tma_load_2d(dst, &tmV, 0, krow, fb);
            if (two) tma_load_2d(dst + C::SLOT / 2, &tmV, 0, krow + 64, fb);
          }
          ++gk;
        }
      }
      if (*abort_flag) {
        // let every TMA load issued here land before shared memory goes away
        for (int s2 = 0; s2 < C::NSLOT; ++s2) {
          const uint32_t fills = pos / C::NSLOT + (static_cast<uint32_t>(s2) < pos % C::NSLOT ? 1u : 0u);
          if (fills) dual_wait_drain(bar(L, C::B_SF + s2), (fills - 1) & 1, budget, status);
        }
        if (qloads) dual_wait_drain(bar(L, C::B_QF), (qloads - 1) & 1, budget, status);
      }
    }
   } else {
    // --------------------------------------------- MMA issuer of both lanes
    // Per lane the products alternate S(k), P.V(k), S(k+1), ...; the issuer
    // serves the lanes in turn, P.V(k) and S(k+1) of one lane back to back
    // (the tensor core runs them in issue order, so S(k+1) overwrites P(k)
    // only after P.V(k) has read it), then the other lane. While one lane's
    // products run, the other lane's softmax works.
    if (lane == 0) {
      struct Lane {
        int id, n, start, k, len, slot, active;
        uint32_t items, qc, gk, oc;
      };
      Lane ln[2];
#pragma unroll
      for (int L = 0; L < 2; ++L) {
        Lane& x = ln[L];
        x.id = L;
        x.n = x.start = x.k = x.len = x.slot = x.active = 0;
        x.items = x.qc = x.gk = x.oc = 0;
      }
      // per-lane addresses, derived from the lane id
      const uint32_t bar0 = smem_u32(&bars[0]);
      auto lb = [&](const Lane& x, int i) -> uint32_t { return bar0 + (x.id * C::NBL + i) * 8; };
      auto dS = [&](const Lane& x) -> uint32_t { return tmem + static_cast<uint32_t>(x.id) * 128u; };
      const uint64_t dQ0 = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(smem_u32(sRing), 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(smem_u32(sRing), D == 128 ? C::SLOT / 2 : C::SLOT, 1024);
      bool ok = true;
      auto wt = [&](uint32_t b, uint32_t parity) -> bool {
        if (!ok) return false;
        ok = mbar_wait(b, parity, budget, abort_flag, status);
        return ok;
      };
      auto slot_at = [](int base, int s) -> int { const int t = base + s; return t >= C::NSLOT ? t - C::NSLOT : t; };
      // the phase of a slot's full barrier for ring position gk*PPB + s
      auto sf_parity = [](uint32_t gk, int s) -> uint32_t { return ((gk * C::PPB + s) / C::NSLOT) & 1; };
      // Next row of lane x with at least one key block (false: none left).
      auto fetch = [&](Lane& x) -> bool {
        while (ok) {
          const int is = x.items & 1;
          if (!wt(lb(x, C::B_IF + is), (x.items >> 1) & 1)) return false;
          const int* e = iring + (x.id * 2 + is) * 4;
          const int row = e[0], n = e[1], start = e[2];
          mbar_arrive(lb(x, C::B_IE + is));
          ++x.items;
          if (row < 0) return false;
          if (n == 0) continue;
          x.n = n;
          x.start = start;
          x.k = 0;
          if (!wt(lb(x, C::B_QF), x.qc & 1)) return false;
          ++x.qc;
          return true;
        }
        return false;
      };
      auto issue_s = [&](Lane& x) -> bool {
        for (int s2 = 0; s2 < C::NK; ++s2)
          if (!wt(lb(x, C::B_SF + slot_at(x.slot, s2)), sf_parity(x.gk, s2))) return false;
        x.len = lenrec[x.id * C::NSLOT + x.slot];
        const int n16 = (x.len + 15) & ~15;
        const uint32_t idesc_s = idesc_bf16_f32(128, n16, 0, 0);
        const uint64_t dK = dK0 + ((x.id * C::NSLOT * C::SLOT) >> 4);
        const uint64_t dQ = dQ0 + ((x.id * C::Q_BYTES) >> 4);
        const uint64_t bk0 = dK + ((x.slot * C::SLOT) >> 4);
        const uint64_t bk1 = dK + ((slot_at(x.slot, 1) * C::SLOT) >> 4);
        // all operand descriptors first: the issues then follow back to back
        uint64_t da[D / 16], db[D / 16];
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          da[kk] = dQ + (((kk >> 2) * C::PANEL + (kk & 3) * 32) >> 4);
          db[kk] = (kk < 4 ? bk0 : bk1) + ((kk & 3) * 32 >> 4);
        }
        const uint32_t ds = dS(x);
        tc_fence_after();
        mma_ss_c<false>(ds, da[0], db[0], idesc_s);
#pragma unroll
        for (int kk = 1; kk < D / 16; ++kk) mma_ss_c<true>(ds, da[kk], db[kk], idesc_s);
        mma_commit(lb(x, C::B_SD));
        return true;
      };
      auto issue_pv = [&](Lane& x) -> bool {
        if (!wt(lb(x, C::B_PF), x.gk & 1)) return false;
        for (int s2 = C::NK; s2 < C::PPB; ++s2)
          if (!wt(lb(x, C::B_SF + slot_at(x.slot, s2)), sf_parity(x.gk, s2))) return false;
        if (x.k == 0 && x.oc >= 1 && !wt(lb(x, C::B_OE), (x.oc - 1) & 1)) return false;
        const int nks = ((x.len + 15) & ~15) / 16;
        // descriptors of the two V positions (d = 128: keys 0..63 and 64..127)
        const uint64_t dV = dV0 + ((x.id * C::NSLOT * C::SLOT) >> 4);
        const uint64_t bv0 = dV + ((slot_at(x.slot, C::NK) * C::SLOT) >> 4);
        const uint64_t bv1 = dV + ((slot_at(x.slot, C::PPB - 1) * C::SLOT) >> 4);
        uint64_t db[8];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          db[kk] = D == 128 ? (kk < 4 ? bv0 : bv1) + ((kk & 3) * 2048 >> 4) : bv0 + (kk * 2048 >> 4);
        const uint32_t ds = dS(x), dO = ds + C::COL_O;
        tc_fence_after();
        if (x.k > 0) mma_ts_c<true>(dO, ds, db[0], C::IDESC_PV);
        else mma_ts_c<false>(dO, ds, db[0], C::IDESC_PV);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          if (kk < nks) mma_ts_c<true>(dO, ds + kk * 8, db[kk], C::IDESC_PV);
        mma_commit(lb(x, C::B_PD));
        ++x.gk;
        x.slot = slot_at(x.slot, C::PPB % C::NSLOT);
        if (++x.k == x.n) ++x.oc;
        return true;
      };
#pragma unroll
      for (int L = 0; L < 2; ++L) ln[L].active = fetch(ln[L]) && issue_s(ln[L]);
      while (ok && (ln[0].active || ln[1].active)) {
#pragma unroll
        for (int L = 0; L < 2; ++L) {
          Lane& x = ln[L];
          if (!x.active || !ok) continue;
          if (!issue_pv(x)) break;
          x.active = (x.k < x.n || fetch(x)) && issue_s(x);
        }
      }
      if (*abort_flag) {
        mma_commit(bar(0, C::B_DR));
        dual_wait_drain(bar(0, C::B_DR), 0, budget, status);
      }
    }
    __syncwarp();
   }
  } else {
    // ------------------------------------------------ softmax + epilogue
    regs_inc<C::REGS_HIGH>();
    const int L = warp >> 2;
    const int t = static_cast<int>(threadIdx.x) & 127;  // query row == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t scol = tmem + lane_off + static_cast<uint32_t>(L) * 128u;
    const uint32_t ocol = tmem + lane_off + C::COL_O + static_cast<uint32_t>(L) * 128u;
    const float sl2 = P.scale_log2;
    auto wwait = [&](int b, uint32_t parity) -> bool {
      const bool w = mbar_wait(bar(L, b), parity, budget, abort_flag, status);
      return __all_sync(0xffffffffu, w);
    };
    uint32_t items = 0, gk = 0;
    bool ok = true;
    while (ok) {
      const int is = items & 1;
      ok = wwait(C::B_IF + is, (items >> 1) & 1);
      if (!ok) break;
      const int* e = iring + (L * 2 + is) * 4;
      const int row = e[0], n = e[1], start = e[2];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L, C::B_IE + is));
      ++items;
      if (row < 0) break;
      const uint64_t t_start = globaltimer_ns();
      uint32_t bh, iq;
      g.dv_nb.divmod(static_cast<uint32_t>(row), bh, iq);
      const bool qvalid = t < block_len(g, static_cast<int>(iq));
      const int64_t orow = static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(iq) * C::BS + t;
      __nv_bfloat16* optr = P.ot + orow * D;
      if (n == 0) {
        for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(optr + c) = make_uint4(0u, 0u, 0u, 0u);
        if (P.lse) P.lse[orow] = qvalid ? -INFINITY : 0.f;
      } else {
        float ref = 0.f, l = 0.f;
        int jn = __ldg(&P.col_idx[start]);
        for (int k = 0; k < n; ++k) {
          const int j = (jn < 0 || jn >= g.nb) ? 0 : jn;
          if (k + 1 < n) jn = __ldg(&P.col_idx[start + k + 1]);
          const int len = block_len(g, j);
          const int nch = (len + 31) >> 5;  // 32-column chunks holding real keys
          ok = wwait(C::B_SD, gk & 1);
          if (!ok) break;
          tc_fence_after();
          // S of the block into registers (one TMEM load wait). Only the
          // last loaded 32-column chunk can hold columns past the real keys
          // (padding, and stale columns past the product's N): those become
          // -inf, and only when the key count is not a multiple of 32.
          uint32_t sr[128];
#define SBA_DUAL_LOAD_S()                                                                   \
  do {                                                                                      \
    _Pragma("unroll") for (int c = 0; c < 4; ++c) if (c < nch)                              \
        tmem_ld32(scol + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));           \
    tmem_ld_wait();                                                                         \
    if (len & 31) {                                                                         \
      const int vl = len & 31;                                                              \
      _Pragma("unroll") for (int e2 = 0; e2 < 32; ++e2) {                                   \
        const bool kill = e2 >= vl;                                                         \
        if (nch == 1 && kill) sr[e2] = 0xFF800000u;                                         \
        if (nch == 2 && kill) sr[32 + e2] = 0xFF800000u;                                    \
        if (nch == 3 && kill) sr[64 + e2] = 0xFF800000u;                                    \
        if (nch == 4 && kill) sr[96 + e2] = 0xFF800000u;                                    \
      }                                                                                     \
    }                                                                                       \
  } while (0)
          SBA_DUAL_LOAD_S();
          if (k == 0) {
            // the row's reference: the first block's row max
            float m0[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c)
              if (c < nch) {
#pragma unroll
                for (int e2 = 0; e2 < 32; e2 += 2)
                  m0[(e2 >> 1) & 3] =
                      fmax3(m0[(e2 >> 1) & 3], __uint_as_float(sr[c * 32 + e2]), __uint_as_float(sr[c * 32 + e2 + 1]));
              }
            ref = fmaxf(fmaxf(m0[0], m0[1]), fmaxf(m0[2], m0[3])) * sl2;
          }
          // P = exp2(S*c - ref) as bf16 pairs, packed into the first 16
          // registers of each chunk (their S values are used by then), and
          // the block's row sum. One pair in four runs on the FMA pipe, to
          // split the exponentials between MUFU and FMA.
          float lblk;
          {
            float2 acc[4];
            const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-ref, -ref);
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              if (c < nch) {
#pragma unroll
                for (int e2 = 0; e2 < 16; ++e2) {
                  const int i0 = c * 32 + 2 * e2;
                  const float2 x =
                      ffma2(make_float2(__uint_as_float(sr[i0]), __uint_as_float(sr[i0 + 1])), sc2, nm2);
                  const float2 pp =
                      ((e2 & 3) == 3) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
                  sr[c * 32 + e2] = pack_bf16x2(pp.x, pp.y);
                  acc[e2 & 3] = fadd2(acc[e2 & 3], pp);
                }
              }
            lblk = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
          }
          // After the first block the reference is used speculatively. A
          // block whose P may exceed 2^24 (its row sum says so) moves the
          // reference up (rare): O, the row sum and the block's P are scaled
          // down together. When P overflowed (row sum not finite), the block
          // is recomputed from S, still in TMEM.
          bool p_stored = false;
          if (__any_sync(0xffffffffu, !(lblk <= C::MAX_BLOCK_SUM))) {
            ok = wwait(C::B_PD, (gk - 1) & 1);  // O holds P.V up to block k-1 (k >= 1 here)
            if (!ok) break;
            tc_fence_after();
            float alpha = 1.f;
            if (__all_sync(0xffffffffu, isfinite(lblk))) {
              if (lblk > C::MAX_BLOCK_SUM) {
                alpha = 1.0f / lblk;  // the reference moves up by log2(lblk)
                ref += __log2f(lblk);
              }
#pragma unroll
              for (int c = 0; c < 4; ++c)
                if (c < nch) {
#pragma unroll
                  for (int e2 = 0; e2 < 16; ++e2) {
                    const uint32_t w = sr[c * 32 + e2];
                    sr[c * 32 + e2] = pack_bf16x2(__uint_as_float(w << 16) * alpha, __uint_as_float(w & 0xFFFF0000u) * alpha);
                  }
                }
              lblk *= alpha;
            } else {
              // P overflowed: reference = the block's row max, P again from S
              float mb = -INFINITY;
#pragma unroll 1
              for (int c = 0; c < nch; ++c) {
                uint32_t r[32];
                tmem_ld32(scol + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int e2 = 0; e2 < 32; ++e2)
                  if (c * 32 + e2 < len) mb = fmaxf(mb, __uint_as_float(r[e2]));
              }
              const float m_new = fmaxf(mb * sl2, ref);
              alpha = ex2_approx(ref - m_new);
              ref = m_new;
              lblk = 0.f;
#pragma unroll 1
              for (int c = 0; c < nch; ++c) {
                uint32_t r[32];
                tmem_ld32(scol + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int e2 = 0; e2 < 16; ++e2) {
                  const float a = c * 32 + 2 * e2 < len ? __uint_as_float(r[2 * e2]) * sl2 - ref : -INFINITY;
                  const float b = c * 32 + 2 * e2 + 1 < len ? __uint_as_float(r[2 * e2 + 1]) * sl2 - ref : -INFINITY;
                  const float pa = ex2_approx(a), pb = ex2_approx(b);
                  r[e2] = pack_bf16x2(pa, pb);
                  lblk += pa + pb;
                }
                // P of chunk c lands on columns of chunks already read
                tmem_st16(scol + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
              }
              p_stored = true;
            }
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tmem_ld32(ocol + c * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int e2 = 0; e2 < 32; ++e2) r[e2] = __float_as_uint(__uint_as_float(r[e2]) * alpha);
              tmem_st32(ocol + c * 32, r);
            }
            l *= alpha;
          }
#undef SBA_DUAL_LOAD_S
          // P over S: 16 TMEM columns per 32 keys
          if (!p_stored) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              if (c < nch) tmem_st16(scol + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[c * 32]));
          }
          l += lblk;
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L, C::B_PF));
          ++gk;
        }
        if (!ok) break;
        ok = wwait(C::B_PD, (gk - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const float inv = qvalid ? 1.0f / l : 0.f;
        // O out of TMEM 64 columns at a time, normalised, stored as bf16
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          uint32_t orr[64];
          tmem_ld32(ocol + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&orr[0]));
          tmem_ld32(ocol + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&orr[32]));
          tmem_ld_wait();
          if (h == D / 64 - 1) {
            // O is free for the lane's next item once all of it is read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L, C::B_OE));
          }
          auto o = [&](int i) -> float { return __uint_as_float(orr[i]) * inv; };
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            uint4 v;
            v.x = pack_bf16x2(o(c + 0), o(c + 1));
            v.y = pack_bf16x2(o(c + 2), o(c + 3));
            v.z = pack_bf16x2(o(c + 4), o(c + 5));
            v.w = pack_bf16x2(o(c + 6), o(c + 7));
            *reinterpret_cast<uint4*>(optr + h * 64 + c) = v;
          }
        }
        if (P.lse) P.lse[orow] = qvalid ? (ref * 0.69314718055994531f + logf(l)) : 0.f;
      }
      if (P.trace && t == 0) {
        P.trace[static_cast<int64_t>(row) * 3 + 0] = t_start;
        P.trace[static_cast<int64_t>(row) * 3 + 1] = globaltimer_ns();
        P.trace[static_cast<int64_t>(row) * 3 + 2] = smid();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::WARP_ISS) tmem_dealloc(tmem, 512);
  if (P.sched == SBA_SCHED_LPT && threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&P.ctrl->cta_done, 1u);
    if (prev == gridDim.x - 1) {
      atomicExch(&P.ctrl->work_next, 0u);
      atomicExch(&P.ctrl->cta_done, 0u);
      __threadfence();
    }
  }
}

template <int D>
cudaError_t launch_dual_d(const sba_plan* p, const void* qt, const void* kt, const void* vt,
                          const DualParams& dp, cudaStream_t st) {
  using C = DCfg<D>;
  const int64_t rows = static_cast<int64_t>(p->g.B) * p->g.H * p->info.Npad;
  CUtensorMap mq, mk, mv;
  if (!tma_map_bf16(&mq, qt, rows, D, 64) || !tma_map_bf16(&mk, kt, rows, D, 64) ||
      !tma_map_bf16(&mv, vt, rows, D, 64)) {
    set_error("cuTensorMapEncodeTiled unavailable or rejected the tensor");
    return cudaErrorInvalidValue;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int optin = 0, sms = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (optin < C::SMEM) {
    set_error("device offers %d bytes of shared memory per CTA, kernel needs %d", optin, C::SMEM);
    return cudaErrorInvalidConfiguration;
  }
  e = cudaFuncSetAttribute(attn_dual_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int pairs = (dp.R + 1) / 2;
  const int grid = dp.sched == SBA_SCHED_LPT ? std::min(sms, pairs) : pairs;
  if (dp.sched == SBA_SCHED_LPT) note_attention_grid_size(grid);
  attn_dual_kernel<D><<<grid, C::THREADS, C::SMEM, st>>>(mq, mk, mv, dp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_dual(const sba_plan* p, const void* qt, const void* kt, const void* vt,
                                  const int32_t* row_ptr, const int32_t* col_idx,
                                  const int32_t* work_order, void* ot, float* lse, int sched,
                                  uint64_t* trace, void* workspace, cudaStream_t st) {
  DualParams dp;
  dp.g = make_kgeom(p);
  dp.row_ptr = row_ptr;
  dp.col_idx = col_idx;
  dp.work_order = work_order;
  dp.ot = static_cast<__nv_bfloat16*>(ot);
  dp.lse = lse;
  dp.trace = trace;
  dp.ctrl = reinterpret_cast<Ctrl*>(static_cast<char*>(workspace) + p->ws_ctrl);
  dp.R = p->info.rows;
  dp.sched = sched;
  dp.max_nnz = p->info.max_nnz;
  dp.budget_ns = p->wait_budget_ns;
  dp.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(dp.g.d)));
  if (dp.g.d == 128) return launch_dual_d<128>(p, qt, kt, vt, dp, st);
  if (dp.g.d == 64) return launch_dual_d<64>(p, qt, kt, vt, dp, st);
  return cudaErrorInvalidValue;
}

}  // namespace sba
