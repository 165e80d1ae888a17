// attn_sm100.cu -- block-sparse attention forward on B200 tensor cores
// (FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for Video
// Generation, abstract: attention over the materialised Top-p / Top-k block
// mask; uneven per-head workloads absorbed by the scheduler).
//
// Work item = one mask row (b, h, query block i): a 128-row query tile and the
// row's selected key blocks, each a contiguous [bs x d] bf16 tile of the
// cube-ordered kt / vt. Per item and key block j:
//   S = Q K_j^T        tcgen05.mma kind::f16, A = Q (smem, K-major),
//                      B = K_j (smem, K-major), fp32 accumulator in TMEM
//   P = exp2(S*c - m)  online softmax in fp32 on CUDA cores, one TMEM lane
//                      (query row) per thread; P rounded to bf16 and written
//                      back over S in TMEM
//   O += P V_j         tcgen05.mma with A = P from TMEM, B = V_j (smem,
//                      MN-major), fp32 accumulator in TMEM
// Issuing a tcgen05.mma blocks the issuing thread at the tensor core's pace,
// and every commit / wait costs that thread tens of cycles, so one thread that
// alternates S and P.V products leaves the tensor core idle whenever it waits
// for the softmax. Two issuer warps keep it fed: one issues the S products up
// to three key blocks ahead (three S buffers in TMEM), the other issues P.V as
// soon as a block's P is ready.
// Warp roles (one CTA per SM):
//   warps 0 .. 4*NWG-1   softmax + epilogue in NWG column groups: warp w owns
//                        TMEM lanes 32*(w%4).. (query rows) and group w/4 owns
//                        bs/NWG columns of S and d/NWG columns of O; the
//                        groups combine their partial row maxima through
//                        shared memory once per key block
//   warp  4*NWG          producer: fetches work items; TMA-loads Q, the K
//                        tiles (ring of NK slots) and the V tiles (ring of NV
//                        slots), K running up to two blocks ahead of V
//   warp  4*NWG+1        S issuer (one thread) and TMEM owner
//   warp  4*NWG+2        P.V issuer (one thread)
// TMEM: S buffers at columns 0, 128, 256; O at 384.
// Rescaling of O is skipped while the running row max grows by less than
// 2^24 (the final normalisation uses the same reference max, so the result is
// exact up to rounding; bf16 P up to 2^24 stays far inside fp32 range for O
// and the row sum); padding keys (the tail of a partial block) are masked to
// -inf.
// Low-bit variant (LB, VC-Attention abstract): E4M3 probability codes from
// one multiply-add (ExpCast-FP8), O += P.V as an 8-bit tensor-core product
// on V-Smooth codes, and the block-mean term sum_j l_j mu_j added to O by a
// small tf32 product per block (A = the two groups' partial row sums, B = the
// block mean); the reference moves when a block exceeds it by 2^2.75.
// Scheduler: SBA_SCHED_LPT launches one persistent CTA per SM that takes rows
// in longest-first work order from an atomic counter (the counter resets
// itself when the last CTA exits); SBA_SCHED_HEAD_MAJOR launches one CTA per
// row in (b, h, i) order. Every wait is bounded (status bit + clean exit).
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace sba {

namespace {

constexpr int kSmemLimit = 232448;  // 227 KB: opt-in shared memory per CTA

template <int D, int BS, bool LB = false>
struct Cfg {
  static constexpr int M = 128;
  // softmax column groups: 2 (measured best for 128x128 tiles: 64 S columns
  // and 64 O columns per thread; 4 groups cost more in exchange and polling)
  static constexpr int NWG = 2;
  static constexpr int CPW = BS / NWG;  // S columns per group
  static constexpr int DPW = D / NWG;   // O columns per group
  static constexpr int SM_THREADS = NWG * 128;
  static constexpr int THREADS = SM_THREADS + 96;
  static constexpr int WARP_PROD = NWG * 4, WARP_SISS = NWG * 4 + 1, WARP_PVISS = NWG * 4 + 2;
  static_assert(CPW % 32 == 0 && DPW % 32 == 0, "column groups must be multiples of 32");
  static constexpr int NSB = 3;  // S buffers in TMEM
  static constexpr int PANELS = D / 64;  // 128-byte column panels along d
  static constexpr int Q_BYTES = M * D * 2;
  static constexpr int TILE_BYTES = BS * D * 2;  // a bf16 K (or V) tile
  // low-bit path (LB): a V tile is bs x d E4M3 codes stored [d][bs]
  static constexpr int VTILE_BYTES = LB ? BS * D : TILE_BYTES;
  // low-bit path: per V slot, the block-mean operand of the tf32 product
  // O += [l0 l1] [mu/2^e; mu/2^e]: 128 channels x 8 k, K-major, no swizzle
  static constexpr int MT_BYTES = LB ? 4096 : 0;
  static constexpr int CTRL_BYTES = 10240;  // barriers, ring, masks, row-max exchange
  static constexpr int NT_RAW = (kSmemLimit - 1024 - CTRL_BYTES - Q_BYTES) / TILE_BYTES;
  static constexpr int NT = NT_RAW > 8 ? 8 : NT_RAW;  // K + V slots
  static constexpr int NK = LB ? 3 : (NT + 1) / 2, NV = LB ? 4 : NT - NK;
  static constexpr int SMEM_USED =
      1024 + Q_BYTES + NK * TILE_BYTES + NV * (VTILE_BYTES + MT_BYTES) + CTRL_BYTES;
  // reference-max threshold (log2 units) beyond which O is rescaled. bf16
  // P up to 2^24 keeps O and the row sum far inside fp32 range and makes a
  // rescale rare (the running maximum of a row rarely jumps that far); E4M3
  // codes have 2.75 octaves of headroom above the reference (code 104 of 126).
  static constexpr float RESCALE = LB ? 2.75f : 24.0f;
  static constexpr float LB_BIAS = 104.0f;  // E4M3 code of the reference
  // bs = 64: a work item is a pair of query blocks (2i, 2i+1) of one head,
  // whose 128 rows fill the tile, over the union of their key sets
  static constexpr bool PAIR = BS == 64 && !LB;
  static_assert(!LB || (D == 128 && BS == 128), "low-bit path: d = bs = 128");
  // Request at least 120 KB so that only one CTA (one 512-column TMEM
  // allocation) is ever resident per SM.
  static constexpr int SMEM = SMEM_USED < 120 * 1024 ? 120 * 1024 : SMEM_USED;
  static constexpr uint32_t IDESC_PV = LB ? idesc_e4m3_f32(M, D) : idesc_bf16_f32(M, D, 0, 1);
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_O = 384;
  static constexpr uint32_t IDESC_MEAN = idesc_tf32_f32(M, D);
  // (the low-bit constants are referenced here so that the bf16
  // instantiations, which do not use them, compile without warnings)
  static_assert(LB_BIAS > 0.0f && RESCALE > 0.0f && IDESC_MEAN != 0u, "low-bit constants");
  // barrier indices
  static constexpr int B_QF = 0, B_QE = 1, B_KF = 2, B_KE = B_KF + NK, B_VF = B_KE + NK,
                       B_VE = B_VF + NV, B_SR = B_VE + NV, B_PR = B_SR + NSB, B_PD = B_PR + NSB,
                       B_OF = B_PD + NSB, B_OE = B_OF + 1, B_IF = B_OE + 1, B_IE = B_IF + 2,
                       B_X = B_IE + 2, B_L = B_X + NSB, B_DR = B_L + 1, NBAR = B_DR + 2;
  static_assert(NK >= 2 && NV >= 1, "need K and V slots");
  static_assert(D <= 128 && BS <= 128, "TMEM plan assumes d, bs <= 128");
  static_assert(NBAR * 8 <= 512, "barrier area");
  static_assert(NK <= 16 && NV <= 16, "slot length records");
  static_assert(1024 + (NSB * NWG + NWG) * 128 * 4 <= CTRL_BYTES, "control area");
  static_assert(SMEM <= kSmemLimit, "shared memory budget");
};

struct AttnParams {
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
  int64_t max_nnz;  // col_idx capacity the plan guarantees (B*H*nb*nb)
  uint64_t budget_ns;
  float scale_log2;
  // low-bit path only
  const float* vmean;    // [B*H][nb][d] block means of V
  const int32_t* vexp;   // [B*H] power-of-two exponent of the value codes
};

// 1.5 * 2^23: adding it to a float in [-2^22, 2^22) rounds the float to an
// integer (nearest even) held in the low mantissa bits.
constexpr float kCodeMagic = 12582912.0f;

// Next block of the ascending union of two sorted column lists (a pair's two
// mask rows): returns it and whether each row selects it. Past both ends it
// returns INT_MAX (only when the lists are inconsistent with the count).
__device__ __forceinline__ int union_next(const int32_t* __restrict__ col_idx, int& ia, int nA, int sA,
                                          int& ib, int nB, int sB, bool& inA, bool& inB) {
  const int a = ia < nA ? __ldg(&col_idx[sA + ia]) : 0x7fffffff;
  const int b = ib < nB ? __ldg(&col_idx[sB + ib]) : 0x7fffffff;
  const int j = min(a, b);
  inA = a == j;
  inB = b == j;
  ia += inA ? 1 : 0;
  ib += inB ? 1 : 0;
  return j;
}

// Wait that ignores the abort flag (used to drain in-flight async work).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t budget_ns,
                                                uint32_t* status) {
  volatile int never = 0;
  return mbar_wait(bar, parity, budget_ns, &never, status);
}

template <int D, int BS, bool LB>
__global__ void __launch_bounds__(Cfg<D, BS, LB>::THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams P) {
  using C = Cfg<D, BS, LB>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = sm;
  unsigned char* sK = sm + C::Q_BYTES;
  unsigned char* sV = sK + C::NK * C::TILE_BYTES;
  unsigned char* sMT = sV + C::NV * C::VTILE_BYTES;  // LB: block-mean operands
  unsigned char* ctl = sMT + C::NV * C::MT_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 516);
  // work item ring [2][8]: item, blocks, start, n (row or first row of a
  // pair), start and n of a pair's second row
  int* ring = reinterpret_cast<int*>(ctl + 528);
  // real keys of the block each K / V slot holds (written before the slot's
  // TMA arrive, read after its full barrier)
  int* klen_k = reinterpret_cast<int*>(ctl + 640);  // [NK]
  int* klen_v = reinterpret_cast<int*>(ctl + 704);  // [NV]
  float* xmax = reinterpret_cast<float*>(ctl + 1024);        // [NSB][NWG][128] partial row maxima
  float* xsum = xmax + C::NSB * C::NWG * 128;                // [NWG][128] partial row sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const KGeom& g = P.g;
  uint32_t* status = &P.ctrl->status;
  const uint64_t budget = P.budget_ns;
  auto bar = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_QF), 1);
    mbar_init(bar(C::B_QE), 1);
    for (int s = 0; s < C::NK; ++s) {
      mbar_init(bar(C::B_KF + s), 1);
      mbar_init(bar(C::B_KE + s), 1);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(bar(C::B_VF + s), 1);
      mbar_init(bar(C::B_VE + s), 1);
    }
    for (int b = 0; b < C::NSB; ++b) {
      mbar_init(bar(C::B_SR + b), 1);
      mbar_init(bar(C::B_PR + b), C::SM_THREADS);
      mbar_init(bar(C::B_PD + b), 1);
      mbar_init(bar(C::B_X + b), C::NWG * 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::B_IF + b), 1);
      mbar_init(bar(C::B_IE + b), 2 + C::NWG * 4);
      mbar_init(bar(C::B_DR + b), 1);
    }
    mbar_init(bar(C::B_OF), 1);
    mbar_init(bar(C::B_OE), C::NWG * 4);
    mbar_init(bar(C::B_L), C::NWG * 4);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::WARP_SISS) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // lane 0 waits, the warp follows
  auto wait1 = [&](int b, uint32_t parity) -> bool {
    int w = 0;
    if (lane == 0) w = mbar_wait(bar(b), parity, budget, abort_flag, status);
    return __shfl_sync(0xffffffffu, w, 0) != 0;
  };

  if (warp == C::WARP_PROD) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    uint32_t items = 0, kt = 0, vt = 0, qloads = 0;
    bool ok = true;
    while (ok) {
      int row = -1;
      if (P.sched == SBA_SCHED_LPT) {
        int idx = 0;
        if (lane == 0) idx = static_cast<int>(atomicAdd(&P.ctrl->work_next, 1u));
        idx = __shfl_sync(0xffffffffu, idx, 0);
        if (idx < P.R) {
          // pairs are taken in order (the work order ranks mask rows)
          row = C::PAIR ? idx : __ldg(&P.work_order[idx]);
          if (row < 0 || row >= P.R) {
            if (lane == 0) atomicOr(status, kStatusCheck);
            row = -1;
          }
        }
      } else {
        row = (items == 0) ? static_cast<int>(blockIdx.x) : -1;
      }
      // a mask row's selected blocks; a row that cannot be read is skipped
      // (written as empty)
      auto row_range = [&](int r, int& st0, int& cnt) {
        st0 = __ldg(&P.row_ptr[r]);
        cnt = __ldg(&P.row_ptr[r + 1]) - st0;
        if (cnt < 0 || cnt > g.nb || st0 < 0 || static_cast<int64_t>(st0) + cnt > P.max_nnz) {
          if (lane == 0) atomicOr(status, kStatusCheck);
          cnt = 0;
          st0 = 0;
        }
      };
      int start = 0, n = 0, nA = 0, startB = 0, nB = 0;
      if (row >= 0) {
        if constexpr (C::PAIR) {
          // item = pair index; rows 2i and 2i+1 (if it exists) of head bh
          const int hp = (g.nb + 1) >> 1;
          const int bhp = row / hp, ip = row - bhp * hp;
          const int rA = bhp * g.nb + 2 * ip;
          row_range(rA, start, nA);
          if (2 * ip + 1 < g.nb) row_range(rA + 1, startB, nB);
          // union size = nA + nB - |A and B| (binary search of A's blocks in B)
          int inter = 0;
          for (int a = lane; a < nA; a += 32) {
            const int x = __ldg(&P.col_idx[start + a]);
            int lo = 0, hi = nB;
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              if (__ldg(&P.col_idx[startB + mid]) < x) lo = mid + 1; else hi = mid;
            }
            inter += (lo < nB && __ldg(&P.col_idx[startB + lo]) == x) ? 1 : 0;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) inter += __shfl_xor_sync(0xffffffffu, inter, o);
          n = nA + nB - inter;
        } else {
          row_range(row, start, n);
          nA = n;
        }
      }
      const int rs = items & 1;
      if (items >= 2) {
        ok = wait1(C::B_IE + rs, ((items >> 1) - 1) & 1);
        if (!ok) break;
      }
      if (lane == 0) {
        ring[rs * 8 + 0] = row;
        ring[rs * 8 + 1] = n;
        ring[rs * 8 + 2] = start;
        ring[rs * 8 + 3] = nA;
        ring[rs * 8 + 4] = startB;
        ring[rs * 8 + 5] = nB;
        mbar_arrive(bar(C::B_IF + rs));
      }
      ++items;
      if (row < 0) break;
      if (n == 0) continue;
      uint32_t bh, iq;
      if constexpr (C::PAIR) {
        const int hp = (g.nb + 1) >> 1;
        bh = static_cast<uint32_t>(row / hp);
        iq = static_cast<uint32_t>(2 * (row - static_cast<int>(bh) * hp));
      } else {
        g.dv_nb.divmod(static_cast<uint32_t>(row), bh, iq);
      }
      const int rows_base = static_cast<int>(bh) * g.Npad;
      if (qloads >= 1) {
        ok = wait1(C::B_QE, (qloads - 1) & 1);
        if (!ok) break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(C::B_QF), C::Q_BYTES);
        for (int p = 0; p < C::PANELS; ++p)
          tma_load_2d(smem_u32(sQ) + p * C::M * 128, &tmQ, p * 64, rows_base + static_cast<int>(iq) * BS,
                      bar(C::B_QF));
      }
      ++qloads;
      // K runs up to NSB-1 blocks ahead of V (the S issuer works that far ahead)
      int nk = 0, nv = 0;
      int ck = 0, cv = 0, ckb = -32, cvb = -32;
      int iaK = 0, ibK = 0, iaV = 0, ibV = 0;  // pair: union cursors of K and V
      while (nv < n) {
        const bool isv = !(nk < n && nk <= nv + (C::NSB - 1));
        const int blk = isv ? nv : nk;
        const int cb = blk & ~31;
        int j;
        if constexpr (C::PAIR) {
          bool inA, inB;
          j = isv ? union_next(P.col_idx, iaV, nA, start, ibV, nB, startB, inA, inB)
                  : union_next(P.col_idx, iaK, nA, start, ibK, nB, startB, inA, inB);
          (void)cb;
        } else if (!isv) {
          if (cb != ckb) {
            ckb = cb;
            ck = (cb + lane < n) ? __ldg(&P.col_idx[start + cb + lane]) : 0;
          }
          j = __shfl_sync(0xffffffffu, ck, blk & 31);
        } else {
          if (cb != cvb) {
            cvb = cb;
            cv = (cb + lane < n) ? __ldg(&P.col_idx[start + cb + lane]) : 0;
          }
          j = __shfl_sync(0xffffffffu, cv, blk & 31);
        }
        if (j < 0 || j >= g.nb) {
          if (lane == 0) atomicOr(status, kStatusCheck);
          j = 0;
        }
        const uint32_t cnt = isv ? vt : kt;
        const int nslot = isv ? C::NV : C::NK;
        const int s = static_cast<int>(cnt % nslot);
        const uint32_t r = cnt / nslot;
        const int bfull = (isv ? C::B_VF : C::B_KF) + s, bempty = (isv ? C::B_VE : C::B_KE) + s;
        if (r >= 1) {
          ok = wait1(bempty, (r - 1) & 1);
          if (!ok) break;
        }
        if constexpr (LB) {
          if (isv) {
            // block j's mean / 2^e as the tf32 operand, K-major without
            // swizzle: core matrices of 8 channels x 16 bytes, 8-channel
            // groups 256 bytes apart and the two k-groups 128 bytes apart (so
            // every access of the product stays inside the 4 KB tile);
            // channel c's row is (v, 0, 0, 0) in both k-groups; 4 channels
            // per lane
            const float sinv = ldexpf(1.0f, -__ldg(&P.vexp[bh]));
            const float4 u = __ldg(reinterpret_cast<const float4*>(
                P.vmean + (static_cast<size_t>(bh) * g.nb + j) * D + lane * 4));
            const float uv[4] = {u.x * sinv, u.y * sinv, u.z * sinv, u.w * sinv};
            unsigned char* mt = sMT + s * C::MT_BYTES;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = lane * 4 + q;
              const int off = (c >> 3) * 256 + (c & 7) * 16;
              const float4 row = make_float4(uv[q], 0.f, 0.f, 0.f);
              *reinterpret_cast<float4*>(mt + off) = row;
              *reinterpret_cast<float4*>(mt + 128 + off) = row;
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
        }
        if (lane == 0) {
          // (not for the low-bit kernel: measured, the record slowed it by
          // 13 % and its S products run over whole blocks)
          if constexpr (!LB) (isv ? klen_v : klen_k)[s] = block_len(g, j);
          if (LB && isv) {
            // E4M3 codes of block j, [d][bs] bytes: one 128-byte-wide box
            const uint32_t dst = smem_u32(sV + s * C::VTILE_BYTES);
            mbar_arrive_expect_tx(bar(bfull), C::VTILE_BYTES);
            tma_load_2d(dst, &tmV, 0, (static_cast<int>(bh) * g.nb + j) * D, bar(bfull));
          } else {
            const uint32_t dst = smem_u32((isv ? sV : sK) + s * C::TILE_BYTES);
            mbar_arrive_expect_tx(bar(bfull), C::TILE_BYTES);
            for (int p = 0; p < C::PANELS; ++p)
              tma_load_2d(dst + p * BS * 128, isv ? &tmV : &tmK, p * 64, rows_base + j * BS, bar(bfull));
          }
        }
        if (isv) {
          ++vt;
          ++nv;
        } else {
          ++kt;
          ++nk;
        }
      }
    }
    if (*abort_flag && lane == 0) {
      // let every TMA load this CTA issued land before shared memory goes away
      for (int s = 0; s < C::NK; ++s) {
        const uint32_t uses = kt / C::NK + (static_cast<uint32_t>(s) < kt % C::NK ? 1u : 0u);
        if (uses) mbar_wait_drain(bar(C::B_KF + s), (uses - 1) & 1, budget, status);
      }
      for (int s = 0; s < C::NV; ++s) {
        const uint32_t uses = vt / C::NV + (static_cast<uint32_t>(s) < vt % C::NV ? 1u : 0u);
        if (uses) mbar_wait_drain(bar(C::B_VF + s), (uses - 1) & 1, budget, status);
      }
      if (qloads) mbar_wait_drain(bar(C::B_QF), (qloads - 1) & 1, budget, status);
    }
  } else if (warp == C::WARP_SISS) {
    // ------------------------------------------------------------ S issuer
    uint32_t items = 0, kc = 0, gs = 0, qloads = 0;
    bool ok = true;
    const uint32_t q_addr = smem_u32(sQ);
    while (ok) {
      const int rs = items & 1;
      ok = wait1(C::B_IF + rs, (items >> 1) & 1);
      if (!ok) break;
      const int row = ring[rs * 8 + 0], n = ring[rs * 8 + 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_IE + rs));
      ++items;
      if (row < 0) break;
      if (n == 0) continue;
      ok = wait1(C::B_QF, qloads & 1);
      ++qloads;
      if (!ok) break;
      for (int i = 0; i < n; ++i) {
        const int b = static_cast<int>(gs % C::NSB);
        if (gs >= static_cast<uint32_t>(C::NSB)) {
          // buffer b still holds P of block gs-NSB until its P.V is done
          ok = wait1(C::B_PD + b, (gs / C::NSB - 1) & 1);
          if (!ok) break;
        }
        const int s = static_cast<int>(kc % C::NK);
        ok = wait1(C::B_KF + s, (kc / C::NK) & 1);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t dS = tmem + static_cast<uint32_t>(b) * 128u;
          const uint32_t k_addr = smem_u32(sK + s * C::TILE_BYTES);
          // S over the block's real keys only, rounded up to the MMA's N step
          // of 16 (the softmax masks the rest of the row)
          const uint32_t idesc_s = idesc_bf16_f32(C::M, LB ? BS : ((klen_k[s] + 15) & ~15), 0, 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t a = smem_desc_sw128(q_addr + (kk >> 2) * (C::M * 128) + off, 16, 1024);
            const uint64_t bd = smem_desc_sw128(k_addr + (kk >> 2) * (BS * 128) + off, 16, 1024);
            mma_ss(dS, a, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::B_SR + b));
          mma_commit(bar(C::B_KE + s));
          if (i == n - 1) mma_commit(bar(C::B_QE));
        }
        __syncwarp();
        ++kc;
        ++gs;
      }
    }
    if (*abort_flag && lane == 0) {
      mma_commit(bar(C::B_DR + 0));
      mbar_wait_drain(bar(C::B_DR + 0), 0, budget, status);
    }
  } else if (warp == C::WARP_PVISS) {
    // ------------------------------------------------------------ P.V issuer
    uint32_t items = 0, vc = 0, gp = 0, ouses = 0;
    bool ok = true;
    while (ok) {
      const int rs = items & 1;
      ok = wait1(C::B_IF + rs, (items >> 1) & 1);
      if (!ok) break;
      const int row = ring[rs * 8 + 0], n = ring[rs * 8 + 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_IE + rs));
      ++items;
      if (row < 0) break;
      if (n == 0) continue;
      for (int i = 0; i < n; ++i) {
        const int b = static_cast<int>(gp % C::NSB);
        ok = wait1(C::B_PR + b, (gp / C::NSB) & 1);
        if (!ok) break;
        const int s = static_cast<int>(vc % C::NV);
        ok = wait1(C::B_VF + s, (vc / C::NV) & 1);
        if (!ok) break;
        if (i == 0 && ouses >= 1) {
          // the epilogue of the previous item has read O out of TMEM
          ok = wait1(C::B_OE, (ouses - 1) & 1);
          if (!ok) break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t aP = tmem + static_cast<uint32_t>(b) * 128u;
          if constexpr (LB) {
            // O += P.V in E4M3: A = P codes in TMEM (8 columns per 32 keys),
            // B = the block's codes, K-major [d][bs], 32 bytes per k-step
            const uint32_t v_addr = smem_u32(sV + s * C::VTILE_BYTES);
#pragma unroll
            for (int kk = 0; kk < BS / 32; ++kk) {
              const uint64_t bd = smem_desc_sw128(v_addr + kk * 32, 16, 1024);
              mma_ts_f8(tmem + C::COL_O, aP + kk * 8, bd, C::IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
            }
            // V-Smooth's mean term: O += [l0 0 0 0 l1 0 0 0] . [mu/2^e rows],
            // A = the groups' partial row sums in columns 32..39 of the S buffer
            const uint32_t mt_addr = smem_u32(sMT + s * C::MT_BYTES);
            mma_ts_tf32(tmem + C::COL_O, aP + 32, smem_desc_noswizzle(mt_addr, 128, 256),
                        C::IDESC_MEAN, 1u);
          } else {
            const uint32_t v_addr = smem_u32(sV + s * C::TILE_BYTES);
            // k-steps of 16 keys up to the block's last real key (P is zero
            // beyond it)
            const int nks = (klen_v[s] + 15) >> 4;
#pragma unroll
            for (int kk = 0; kk < BS / 16; ++kk) {
              if (kk < nks) {
                const uint64_t bd = smem_desc_sw128(v_addr + kk * 2048, BS * 128, 1024);
                mma_ts(tmem + C::COL_O, aP + kk * 8, bd, C::IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
              }
            }
          }
          mma_commit(bar(C::B_PD + b));
          mma_commit(bar(C::B_VE + s));
        }
        __syncwarp();
        ++vc;
        ++gp;
      }
      if (!ok) break;
      if (lane == 0) mma_commit(bar(C::B_OF));
      __syncwarp();
      ++ouses;
    }
    if (*abort_flag && lane == 0) {
      mma_commit(bar(C::B_DR + 1));
      mbar_wait_drain(bar(C::B_DR + 1), 0, budget, status);
    }
  } else {
    // ------------------------------------------------ softmax + epilogue
    constexpr int CPW = C::CPW, DPW = C::DPW, NWG = C::NWG, NSB = C::NSB;
    const int t = static_cast<int>(threadIdx.x) & 127;  // query row == TMEM lane
    const int wg = warp >> 2;                             // column group
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = P.scale_log2;
    auto wwait = [&](int b, uint32_t parity) -> bool {
      const bool w = mbar_wait(bar(b), parity, budget, abort_flag, status);
      return __all_sync(0xffffffffu, w);
    };
    uint32_t items = 0, gsm = 0, ouses = 0;
    bool ok = true;
    while (ok) {
      const int rs = items & 1;
      ok = wwait(C::B_IF + rs, (items >> 1) & 1);
      if (!ok) break;
      const int row = ring[rs * 8 + 0], n = ring[rs * 8 + 1], start = ring[rs * 8 + 2];
      const int nA = ring[rs * 8 + 3], startB = ring[rs * 8 + 4], nB = ring[rs * 8 + 5];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_IE + rs));
      ++items;
      if (row < 0) break;
      const uint64_t t_start = globaltimer_ns();
      uint32_t bh, iq;
      // pair items: rows t < 64 belong to query block iq, rows t >= 64 to
      // block iq + 1 (written only when it exists); otherwise rows t < BS
      bool has_rows = t < BS;
      if constexpr (C::PAIR) {
        const int hp = (g.nb + 1) >> 1;
        bh = static_cast<uint32_t>(row / hp);
        iq = static_cast<uint32_t>(2 * (row - static_cast<int>(bh) * hp));
        has_rows = t < BS || static_cast<int>(iq) + 1 < g.nb;
      } else {
        g.dv_nb.divmod(static_cast<uint32_t>(row), bh, iq);
      }
      // a block's real slots are its first block_len slots
      const bool qvalid = has_rows && (t < BS ? t < block_len(g, static_cast<int>(iq))
                                              : t - BS < block_len(g, static_cast<int>(iq) + 1));
      const int64_t orow = static_cast<int64_t>(bh) * g.Npad + static_cast<int64_t>(iq) * BS + t;
      __nv_bfloat16* optr = P.ot + orow * D + wg * DPW;
      // pair items: this warp's rows belong to the first (A) or second (B) row
      const bool half_b = C::PAIR && (warp & 3) >= 2;
      if (n == 0) {
        if (has_rows) {
          for (int c = 0; c < DPW; c += 8)
            *reinterpret_cast<uint4*>(optr + c) = make_uint4(0u, 0u, 0u, 0u);
          if (P.lse && wg == 0) P.lse[orow] = qvalid ? -INFINITY : 0.f;
        }
      } else {
        float m = -INFINITY, l = 0.f;  // l: this group's share of the row sum
        int jn = __ldg(&P.col_idx[start]);
        int ia = 0, ib = 0;  // pair: union cursors
        for (int i = 0; i < n; ++i) {
          int j;
          bool sel = true;  // this warp's rows select the block
          if constexpr (C::PAIR) {
            bool inA, inB;
            j = union_next(P.col_idx, ia, nA, start, ib, nB, startB, inA, inB);
            sel = half_b ? inB : inA;
            if (j < 0 || j >= g.nb) j = 0;
          } else {
            j = (jn < 0 || jn >= g.nb) ? 0 : jn;
            if (i + 1 < n) jn = __ldg(&P.col_idx[start + i + 1]);
          }
          const int b = static_cast<int>(gsm % NSB);
          const uint32_t ph = (gsm / NSB) & 1;
          ok = wwait(C::B_SR + b, ph);
          if (!ok) break;
          tc_fence_after();
          const uint32_t scol = tmem + lane_off + static_cast<uint32_t>(b) * 128u;
          if (C::PAIR && !sel) {
            // rows that do not select the block: P = 0 over this group's
            // columns, no maximum (-inf in the exchange), nothing added
            float* xm0 = xmax + (b * NWG) * 128;
            xm0[wg * 128 + t] = -INFINITY;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_X + b));
            uint32_t zero[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) zero[e] = 0u;
            tmem_st16(scol + wg * (CPW / 2), zero);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(C::B_PR + b));
            ++gsm;
            continue;
          }
          // the first block this row selects sets the reference
          const bool first = C::PAIR ? (m == -INFINITY) : (i == 0);
          const int klen = block_len(g, j);
          uint32_t sr[CPW];
#pragma unroll
          for (int c = 0; c < CPW / 32; ++c)
            tmem_ld32(scol + wg * CPW + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
          tmem_ld_wait();
          float s[CPW];
#pragma unroll
          for (int e = 0; e < CPW; ++e) s[e] = __uint_as_float(sr[e]);
          if (klen < BS) {
            // padding keys (slots klen .. BS-1) are masked
#pragma unroll
            for (int e = 0; e < CPW; ++e)
              if (wg * CPW + e >= klen) s[e] = -INFINITY;
          }
          // partial row max over this group's columns (independent chains)
          float mc[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) mc[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
          for (int e = 8; e < CPW; e += 8) {
#pragma unroll
            for (int k = 0; k < 4; ++k) mc[k] = fmax3(mc[k], s[e + 2 * k], s[e + 2 * k + 1]);
          }
          float* xm = xmax + (b * NWG) * 128;
          const float pm = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
          xm[wg * 128 + t] = pm;
          // publish this group's maximum; every group has also finished
          // loading its S columns before anyone overwrites S with P
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::B_X + b));
          uint32_t pk[LB ? CPW / 4 : CPW / 2];
          float2 acc[4];
          float alpha = 1.f;
          // Exponentials of this group's columns against the reference max.
          // After the first block the running max is used speculatively
          // (the usual case: no group's maximum exceeds it by more than RESCALE)
          // while the exchange completes; the rare block that does exceed it
          // rescales O and goes round once more with the new reference.
          float ref = m;
          if (first) {
            ok = wwait(C::B_X + b, ph);
            if (!ok) break;
            float mx = xm[t];
#pragma unroll
            for (int k = 1; k < NWG; ++k) mx = fmaxf(mx, xm[k * 128 + t]);
            ref = m = mx * sl2;
          }
#pragma unroll 1
          for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
            if constexpr (LB) {
              // ExpCast-FP8 (VC-Attention abstract): the E4M3 code of
              // 2^(x + 6), x = s*log2(e)/sqrt(d) - ref, is rint(8x + 104):
              // one multiply-add, the magic add's rounding, a clamp at 0,
              // and the low byte of each float is a code
              const float c8 = 8.0f * sl2, bb = C::LB_BIAS - 8.0f * ref;
              const float2 c82 = make_float2(c8, c8), b2 = make_float2(bb, bb);
              const float2 mg2 = make_float2(kCodeMagic, kCodeMagic);
#pragma unroll
              for (int e = 0; e < CPW / 4; ++e) {
                const float2 y0 = fadd2(ffma2(make_float2(s[4 * e], s[4 * e + 1]), c82, b2), mg2);
                const float2 y1 =
                    fadd2(ffma2(make_float2(s[4 * e + 2], s[4 * e + 3]), c82, b2), mg2);
                const uint32_t z0 = __float_as_uint(fmaxf(y0.x, kCodeMagic));
                const uint32_t z1 = __float_as_uint(fmaxf(y0.y, kCodeMagic));
                const uint32_t z2 = __float_as_uint(fmaxf(y1.x, kCodeMagic));
                const uint32_t z3 = __float_as_uint(fmaxf(y1.y, kCodeMagic));
                pk[e] = __byte_perm(__byte_perm(z0, z1, 0x0040), __byte_perm(z2, z3, 0x0040), 0x5410);
                // row sum of the decoded codes the P.V product uses
                add_e4m3x4_f32(pk[e], acc[e & 3].x, acc[e & 3].y);
              }
            } else {
              const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-ref, -ref);
#pragma unroll
              for (int e = 0; e < CPW / 2; ++e) {
                const float2 x = ffma2(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
                // one pair in eight runs on the FMA pipe to offload MUFU
                const float2 pp = ((e & 7) == 5) ? exp2_poly2(x)
                                                 : make_float2(ex2_approx(x.x), ex2_approx(x.y));
                pk[e] = pack_bf16x2(pp.x, pp.y);
                // row sum of the fp32 values (the bf16 rounding of P moves a
                // row's normalisation by ~2^-9 / sqrt(keys) relative)
                acc[e & 3] = fadd2(acc[e & 3], pp);
              }
            }
            if (first || pass == 1) break;
            ok = wwait(C::B_X + b, ph);
            if (!ok) break;
            float mx = xm[t];
#pragma unroll
            for (int k = 1; k < NWG; ++k) mx = fmaxf(mx, xm[k * 128 + t]);
            const float mblk = mx * sl2;
            const bool grow = mblk > m + C::RESCALE;
            if (!__any_sync(0xffffffffu, grow)) break;
            const float m_new = grow ? mblk : m;
            alpha = grow ? ex2_approx(m - m_new) : 1.f;
            // O holds P.V up to block i-1: wait for it, rescale this group's columns
            const uint32_t gp = gsm - 1;
            ok = wwait(C::B_PD + static_cast<int>(gp % NSB), (gp / NSB) & 1);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < DPW / 32; ++c) {
              uint32_t r[32];
              const uint32_t oc = tmem + lane_off + C::COL_O + wg * DPW + c * 32;
              tmem_ld32(oc, r);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              tmem_st32(oc, r);
            }
            tmem_st_wait();
            ref = m = m_new;
          }
          if (!ok) break;
          tc_fence_after();
          l *= alpha;
          const float lblk = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                             ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
          if constexpr (LB) {
            // E4M3 codes (4 per column) over this group's quarter of S
            tmem_st16(scol + wg * (CPW / 4), *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
            // this group's share of the block's row sum: k = 4 * group of
            // the tf32 mean product's A operand (columns 32..39)
            tmem_st4(scol + 32 + wg * 4, __float_as_uint(lblk), 0u, 0u, 0u);
          } else if constexpr (CPW >= 64) {
            // P (bf16 pairs) over the first half of this group's S columns
            const uint32_t pcol = scol + wg * (CPW / 2);
#pragma unroll
            for (int c = 0; c < CPW / 64; ++c)
              tmem_st32(pcol + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[c * 32]));
          } else {
            tmem_st16(scol + wg * (CPW / 2), *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
          }
          l += lblk;
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(C::B_PR + b));
          ++gsm;
        }
        if (!ok) break;
        ok = wwait(C::B_OF, ouses & 1);
        if (!ok) break;
        tc_fence_after();
        uint32_t orr[DPW];
#pragma unroll
        for (int c = 0; c < DPW / 32; ++c)
          tmem_ld32(tmem + lane_off + C::COL_O + wg * DPW + c * 32,
                    *reinterpret_cast<uint32_t(*)[32]>(&orr[c * 32]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_OE));
        ++ouses;
        xsum[wg * 128 + t] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_L));
        ok = wwait(C::B_L, (ouses - 1) & 1);
        if (!ok) break;
        float lt = xsum[t];
#pragma unroll
        for (int k = 1; k < NWG; ++k) lt += xsum[k * 128 + t];
        if constexpr (LB) {
          // O holds P.codes + sum_j l_j mu_j / 2^e: scale back by 2^e
          const float sig = ldexpf(1.0f, __ldg(&P.vexp[bh]));
#pragma unroll
          for (int c = 0; c < DPW; ++c) orr[c] = __float_as_uint(sig * __uint_as_float(orr[c]));
        }
        if (has_rows) {
          // (a pair's row that selects no block has lt = 0: O = 0, lse = -inf)
          const float inv = (qvalid && lt > 0.f) ? 1.0f / lt : 0.f;
#pragma unroll
          for (int c = 0; c < DPW; c += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(orr[c + 0]) * inv, __uint_as_float(orr[c + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(orr[c + 2]) * inv, __uint_as_float(orr[c + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(orr[c + 4]) * inv, __uint_as_float(orr[c + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(orr[c + 6]) * inv, __uint_as_float(orr[c + 7]) * inv);
            *reinterpret_cast<uint4*>(optr + c) = v;
          }
          // the low-bit codes carry a factor 2^6 (the reference maps to code 104)
          const float mref = LB ? m - 6.0f : m;
          if (P.lse && wg == 0)
            P.lse[orow] = qvalid ? (lt > 0.f ? mref * 0.69314718055994531f + logf(lt) : -INFINITY) : 0.f;
        }
      }
      if (P.trace && threadIdx.x == 0) {
        // the mask row (rows, for a pair) this item covered
        const int r0 = C::PAIR ? static_cast<int>(bh) * g.nb + static_cast<int>(iq) : row;
        const int nr = C::PAIR && static_cast<int>(iq) + 1 < g.nb ? 2 : 1;
        const uint64_t t_end = globaltimer_ns();
        for (int k = 0; k < nr; ++k) {
          P.trace[static_cast<int64_t>(r0 + k) * 3 + 0] = t_start;
          P.trace[static_cast<int64_t>(r0 + k) * 3 + 1] = t_end;
          P.trace[static_cast<int64_t>(r0 + k) * 3 + 2] = smid();
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::WARP_SISS) tmem_dealloc(tmem, C::TMEM_COLS);
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

// ---------------------------------------------------------------- fp32 path
// fp32 inputs keep fp32 arithmetic end to end (rounding them to bf16 would
// cost ~4e-2 max-abs on unit-scale data): one CTA per row, one thread per
// query slot, K/V tiles staged in shared memory, exact fp32 online softmax.
template <int D>
__global__ void __launch_bounds__(128)
    attn_f32_kernel(KGeom g, const float* __restrict__ qt, const float* __restrict__ kt,
                    const float* __restrict__ vt, const int32_t* __restrict__ row_ptr,
                    const int32_t* __restrict__ col_idx, float* __restrict__ ot,
                    float* __restrict__ lse, uint64_t* __restrict__ trace, uint32_t* status,
                    float scale_log2) {
  extern __shared__ float fsm[];
  const int BS = g.bs;
  float* Ks = fsm;                  // [BS][D+1]
  float* Vs = fsm + BS * (D + 1);   // [BS][D]
  const int row = blockIdx.x;
  const int t = threadIdx.x;
  const uint64_t t_start = globaltimer_ns();
  uint32_t bh, iq;
  g.dv_nb.divmod(static_cast<uint32_t>(row), bh, iq);
  const int64_t head = static_cast<int64_t>(bh) * g.Npad;

  const bool active = t < BS;
  const bool qvalid = active && t < block_len(g, static_cast<int>(iq));
  const int64_t qrow = head + static_cast<int64_t>(iq) * BS + t;
  float q[D], o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    q[c] = active ? qt[qrow * D + c] * scale_log2 : 0.f;
    o[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  int start = row_ptr[row];
  int n = row_ptr[row + 1] - start;
  if (n < 0 || n > g.nb || start < 0 || static_cast<int64_t>(start) + n > static_cast<int64_t>(g.nb) * g.nb * g.B * g.H) {
    // a row that cannot be read is skipped (written as empty)
    if (t == 0) atomicOr(status, kStatusCheck);
    n = 0;
    start = 0;
  }
  for (int i = 0; i < n; ++i) {
    int j = col_idx[start + i];
    if (j < 0 || j >= g.nb) {
      if (t == 0) atomicOr(status, kStatusCheck);
      j = 0;
    }
    __syncthreads();
    for (int e = t; e < BS * D; e += blockDim.x) {
      const int r = e / D, c = e % D;
      const int64_t src = (head + static_cast<int64_t>(j) * BS + r) * D + c;
      Ks[r * (D + 1) + c] = kt[src];
      Vs[r * D + c] = vt[src];
    }
    __syncthreads();
    if (!active) continue;
    const int klen = block_len(g, j);
    for (int c = 0; c < klen; ++c) {
      float s = 0.f;
#pragma unroll
      for (int x = 0; x < D; ++x) s = fmaf(q[x], Ks[c * (D + 1) + x], s);
      if (s > m) {
        const float a = exp2f(m - s);
        l *= a;
#pragma unroll
        for (int x = 0; x < D; ++x) o[x] *= a;
        m = s;
      }
      const float p = exp2f(s - m);
      l += p;
#pragma unroll
      for (int x = 0; x < D; ++x) o[x] = fmaf(p, Vs[c * D + x], o[x]);
    }
  }
  if (active) {
    const float inv = (qvalid && n > 0) ? 1.0f / l : 0.f;
#pragma unroll
    for (int c = 0; c < D; ++c) ot[qrow * D + c] = o[c] * inv;
    if (lse) lse[qrow] = !qvalid ? 0.f : (n > 0 ? m * 0.69314718055994531f + logf(l) : -INFINITY);
  }
  if (trace && t == 0) {
    trace[static_cast<int64_t>(row) * 3 + 0] = t_start;
    trace[static_cast<int64_t>(row) * 3 + 1] = globaltimer_ns();
    trace[static_cast<int64_t>(row) * 3 + 2] = smid();
  }
}

__global__ void timeout_probe_kernel(Ctrl* ctrl, uint64_t budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on this barrier: the bounded wait must give up.
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, budget_ns, &abort_flag, &ctrl->status);
}

// y = exp2_poly2(x) element-wise (the softmax's FMA-pipe exponential), for
// checking it against the exact 2^x.
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 r = exp2_poly2(v);
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

// ----------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map(CUtensorMap* map, const void* base, int64_t rows, int D, int box_rows) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 8-bit codes [rows][inner] (inner = 128 bytes), boxes of box_rows rows.
bool make_map_u8(CUtensorMap* map, const void* base, int64_t rows, int inner, int box_rows) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(inner), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int g_grid_size = 0;

template <int D, int BS, bool LB = false>
cudaError_t launch_tc(const sba_plan* p, const void* qt, const void* kt, const void* vt,
                      const AttnParams& ap, cudaStream_t st) {
  using C = Cfg<D, BS, LB>;
  const int64_t rows = static_cast<int64_t>(p->g.B) * p->g.H * p->info.Npad;
  CUtensorMap mq, mk, mv;
  const bool vmap = LB ? make_map_u8(&mv, vt, static_cast<int64_t>(p->g.B) * p->g.H * p->info.nb * D, BS, D)
                       : make_map(&mv, vt, rows, D, BS);
  if (!make_map(&mq, qt, rows, D, 128) || !make_map(&mk, kt, rows, D, BS) || !vmap) {
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
  e = cudaFuncSetAttribute(attn_tc_kernel<D, BS, LB>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = ap.sched == SBA_SCHED_LPT ? std::min(sms, ap.R) : ap.R;
  if (ap.sched == SBA_SCHED_LPT) g_grid_size = grid;
  attn_tc_kernel<D, BS, LB><<<grid, C::THREADS, C::SMEM, st>>>(mq, mk, mv, ap);
  return cudaGetLastError();
}

}  // namespace

int attention_grid_size() { return g_grid_size; }

cudaError_t launch_attention(const sba_plan* p, const void* qt, const void* kt, const void* vt,
                             const int32_t* row_ptr, const int32_t* col_idx,
                             const int32_t* work_order, void* ot, float* lse, int sched,
                             uint64_t* trace, void* workspace, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(static_cast<char*>(workspace) + p->ws_ctrl);
  const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(g.d)));
  if (p->g.dtype == SBA_F32) {
    const size_t smem = static_cast<size_t>(g.bs) * (2 * g.d + 1) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attn_f32_kernel<64><<<p->info.rows, 128, smem, st>>>(
        g, static_cast<const float*>(qt), static_cast<const float*>(kt), static_cast<const float*>(vt),
        row_ptr, col_idx, static_cast<float*>(ot), lse, trace, &ctrl->status, scale_log2);
    return cudaGetLastError();
  }
  AttnParams ap;
  ap.g = g;
  ap.row_ptr = row_ptr;
  ap.col_idx = col_idx;
  ap.work_order = work_order;
  ap.ot = static_cast<__nv_bfloat16*>(ot);
  ap.lse = lse;
  ap.trace = trace;
  ap.ctrl = ctrl;
  // block size 64 (bf16): work items are pairs of query blocks
  ap.R = (g.bs == 64 && p->g.dtype == SBA_BF16) ? g.B * g.H * ((g.nb + 1) / 2) : p->info.rows;
  ap.sched = sched;
  ap.max_nnz = p->info.max_nnz;
  ap.budget_ns = p->wait_budget_ns;
  ap.scale_log2 = scale_log2;
  ap.vmean = nullptr;
  ap.vexp = nullptr;
  if (g.d == 128 && g.bs == 128) return launch_tc<128, 128>(p, qt, kt, vt, ap, st);
  if (g.d == 128 && g.bs == 64) return launch_tc<128, 64>(p, qt, kt, vt, ap, st);
  if (g.d == 64 && g.bs == 128) return launch_tc<64, 128>(p, qt, kt, vt, ap, st);
  if (g.d == 64 && g.bs == 64) return launch_tc<64, 64>(p, qt, kt, vt, ap, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attention_lowbit(const sba_plan* p, const void* qt, const void* kt, const void* vq,
                                    const float* vmean, const int32_t* vexp, const int32_t* row_ptr,
                                    const int32_t* col_idx, const int32_t* work_order, void* ot,
                                    float* lse, uint64_t* trace, void* workspace, cudaStream_t st) {
  KGeom g = make_kgeom(p);
  AttnParams ap;
  ap.g = g;
  ap.row_ptr = row_ptr;
  ap.col_idx = col_idx;
  ap.work_order = work_order;
  ap.ot = static_cast<__nv_bfloat16*>(ot);
  ap.lse = lse;
  ap.trace = trace;
  ap.ctrl = reinterpret_cast<Ctrl*>(static_cast<char*>(workspace) + p->ws_ctrl);
  ap.R = p->info.rows;
  ap.sched = SBA_SCHED_LPT;
  ap.max_nnz = p->info.max_nnz;
  ap.budget_ns = p->wait_budget_ns;
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(g.d)));
  ap.vmean = vmean;
  ap.vexp = vexp;
  if (g.d == 128 && g.bs == 128) return launch_tc<128, 128, true>(p, qt, kt, vq, ap, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t st) {
  const int64_t pairs = (n + 1) / 2;
  const int threads = 256;
  exp2_poly_kernel<<<static_cast<unsigned>((pairs + threads - 1) / threads), threads, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(void* workspace, uint64_t timeout_ns, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(static_cast<Ctrl*>(workspace), timeout_ns);
  return cudaGetLastError();
}

}  // namespace sba
