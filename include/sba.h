/*
 * sba.h -- C ABI of libsba, training-free Top-p block-sparse self-attention
 * for video diffusion transformers, built for NVIDIA B200 (sm_100a).
 *
 * The method (FVAttn: Adaptive Sparse Attention with Runtime Load Balancing
 * for Video Generation, abstract): a sparse-routing front end made of
 * "video-aware block organization", "Top-p routing" and "a Top-k safety
 * floor" materialises a block mask, and attention then runs over the selected
 * blocks only; adaptive Top-p gives uneven per-head work, which a scheduler
 * has to absorb. The four calls below are the four steps of that path:
 *
 *   sba_reorder     raster (t,h,w) tokens -> spatio-temporal cube blocks
 *   sba_build_mask  pooled block scores -> Top-p / Top-k mask (bitmask + CSR)
 *                   and a longest-first work order
 *                   (sba_build_stripe_mask: the same outputs from a static
 *                   stripe pattern instead of scores)
 *   sba_attention   online-softmax attention over the selected key blocks
 *   sba_unreorder   cube blocks -> raster tokens
 *
 * Conventions shared by every call
 * --------------------------------
 * - Geometry: a latent grid of T x Hh x W tokens (N = T*Hh*W), cut into cubes
 *   of ct x ch x cw tokens; every cube is one block of bs = ct*ch*cw slots.
 *   The cube grid is nT x nH x nW with nT = ceil(T/ct) etc., nb = nT*nH*nW
 *   blocks per head and Npad = nb*bs slots per head. A grid that does not
 *   divide into whole cubes is padded: an edge cube's real tokens take its
 *   first slots and padding the rest, so the real slots of every block are a
 *   prefix of it. Padding slots hold zeros after sba_reorder, are never
 *   attended to as keys and produce zero output rows.
 * - Token order: raster token n = (t*Hh + h)*W + w lies in cube
 *   blk = ((t/ct)*nH + h/ch)*nW + w/cw (cubes row-major over the cube grid).
 *   With the cube's real extents vh = min(ch, Hh - (h/ch)*ch) and
 *   vw = min(cw, W - (w/cw)*cw), its slot is
 *   blk*bs + ((t%ct)*vh + h%ch)*vw + w%cw (tokens row-major inside the
 *   cube's real sub-box; ((t%ct)*ch + h%ch)*cw + w%cw for a complete cube).
 * - Hilbert order (DFSAttn: Hilbert-curve token reordering), when the
 *   geometry's order is SBA_ORDER_HILBERT: a token's slot is its rank along a
 *   3-D Hilbert curve (Skilling's construction, axes t, h, w) over the
 *   smallest power-of-two cube holding the grid; each run of bs = ct*ch*cw
 *   slots is one block, nb = ceil(N/bs), and only the last block has padding
 *   (slots N .. Npad-1).
 * - Tensors: raster q, k, v, o are [B][H][N][d] with element strides sB, sH,
 *   sN given in the geometry and d contiguous (so [B][N][H][d] storage is
 *   accepted). Reordered qt, kt, vt, ot are packed [B][H][Npad][d].
 * - Rows of the mask: r = (b*H + h)*nb + i for query block i; R = B*H*nb.
 * - Memory: every buffer is allocated and owned by the caller; the library
 *   never allocates device memory and never synchronises, except
 *   sba_check_device_status. Device pointers must be 16-byte aligned.
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *   default stream). Every call is asynchronous on it.
 * - Errors: arguments are validated on the host before any launch and a
 *   negative status is returned with a message in sba_last_error(). A failed
 *   launch returns SBA_ERR_CUDA. Checks that only the device can make (a
 *   column index out of range, a bounded wait that gave up) set bits in a
 *   status word inside the workspace; sba_check_device_status reads them.
 */
#ifndef SBA_H_
#define SBA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SBA_API __attribute__((visibility("default")))
#else
#define SBA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SBA_OK = 0,
  SBA_ERR_INVALID_ARG = -1,     /* bad pointer, size, stride or value */
  SBA_ERR_UNSUPPORTED = -2,     /* valid but not built (e.g. an untuned d) */
  SBA_ERR_CUDA = -3,            /* a CUDA runtime/driver call failed */
  SBA_ERR_CAPACITY = -4,        /* a size exceeds an int32 index or a limit */
  SBA_ERR_DEVICE_TIMEOUT = -5,  /* a bounded device-side wait gave up */
  SBA_ERR_DEVICE_CHECK = -6     /* a device-side input check failed */
} sba_status;

typedef enum { SBA_F32 = 0, SBA_BF16 = 1 } sba_dtype;

typedef enum {
  SBA_ORDER_CUBE = 0,       /* blocks are ct x ch x cw cubes of the grid */
  SBA_ORDER_HILBERT = 1     /* blocks are runs of bs tokens along a 3-D Hilbert curve */
} sba_order;

typedef enum {
  SBA_SCHED_LPT = 0,        /* persistent CTAs, rows taken longest first */
  SBA_SCHED_HEAD_MAJOR = 1  /* one CTA per row, rows in (b, h, i) order */
} sba_sched;

/* Geometry of one attention layer (see the conventions above). */
typedef struct {
  int32_t B, H;          /* batch, heads */
  int32_t T, Hh, W;      /* latent grid: frames, height, width */
  int32_t d;             /* head dimension */
  int32_t ct, ch, cw;    /* cube extents; bs = ct*ch*cw */
  int32_t dtype;         /* sba_dtype of q, k, v, o and their reordered forms */
  int64_t sB, sH, sN;    /* element strides of raster q/k/v/o; d is contiguous */
  int32_t order;         /* sba_order; SBA_ORDER_CUBE unless set */
  int32_t reserved;      /* must be 0 */
} sba_geometry;

/* Sizes derived from a geometry. */
typedef struct {
  int32_t nT, nH, nW;        /* cube grid */
  int32_t nb;                /* blocks per head (query and key) */
  int32_t bs;                /* slots per block */
  int32_t Npad;              /* slots per head = nb*bs */
  int32_t rows;              /* R = B*H*nb mask rows */
  int32_t words;             /* uint32 words per bitmask row = ceil(nb/32) */
  int64_t max_nnz;           /* worst-case length of col_idx = R*nb */
  size_t workspace_bytes;    /* size of the workspace every call below takes */
} sba_plan_info;

typedef struct sba_plan sba_plan;

/* Parameters of one head's stripe mask (sba_build_stripe_mask). */
typedef struct {
  int32_t Tw, To, Ts; /* temporal stripe: width, offset, period (0: once) */
  int32_t Sw, So, Ss; /* spatial stripe: width, offset, period (0: once) */
} sba_stripe;

/* Validate a geometry and build a host-side plan (no device memory, no CUDA
 * call). Supported: bs in {64, 128}; bf16 with d in {64, 128}; f32 with d = 64;
 * nb <= 1024; B*H <= 8192; H <= 256; R*nb < 2^31; strides multiples of 8
 * elements. Returns SBA_ERR_INVALID_ARG / SBA_ERR_UNSUPPORTED /
 * SBA_ERR_CAPACITY otherwise. The plan is immutable and may be shared by
 * threads. */
SBA_API sba_status sba_plan_create(const sba_geometry* geom, sba_plan** out);
SBA_API void sba_plan_destroy(sba_plan* plan);
SBA_API sba_status sba_plan_query(const sba_plan* plan, sba_plan_info* info);

/* Zero the control words at the start of a workspace (status word and the
 * scheduler's counters) and, for Hilbert-order plans, upload the plan's
 * permutation table into it. Call once after allocating a workspace, before
 * its first use (required for Hilbert order; for cube order a workspace
 * allocated zero-filled needs no call). */
SBA_API sba_status sba_workspace_init(const sba_plan* plan, void* workspace, void* stream);

/* Video-aware block organization (FVAttn abstract): gather raster q, k, v into
 * block order. Each of the three (src, dst) pairs may be (NULL, NULL) to skip
 * that tensor. Padding slots are written as zeros. Bit copy: no rounding.
 * workspace: may be NULL for cube order; for Hilbert order the workspace
 * initialised by sba_workspace_init (it holds the permutation table). */
SBA_API sba_status sba_reorder(const sba_plan* plan,
                       const void* q, const void* k, const void* v,
                       void* qt, void* kt, void* vt, const void* workspace, void* stream);

/* Inverse of sba_reorder for the output: ot [B][H][Npad][d] -> o, raster with
 * the geometry's strides. Padding slots are dropped. Bit copy. workspace as
 * for sba_reorder. */
SBA_API sba_status sba_unreorder(const sba_plan* plan, const void* ot, void* o,
                                 const void* workspace, void* stream);

/* Block scoring and routing (FVAttn abstract: Top-p routing, Top-k safety
 * floor). For every row r = (b, h, i):
 *   Qbar_i, Kbar_j = means of qt, kt over the real tokens of block i, j (fp64)
 *   P_ij = softmax_j(Qbar_i . Kbar_j / sqrt(d))   (fp64)
 *   sort j by P_ij descending (ties: lower j first); n_p = the shortest
 *   prefix whose cumulative mass reaches top_p[h] (all nb when it never does
 *   or top_p[h] >= 1); keep n = min(nb, max(top_k, n_p)) blocks.
 * Outputs (device, caller-owned):
 *   bitmask   uint32 [R][words]; bit j%32 of word j/32 set when block j kept
 *   row_cnt   int32 [R]; n of every row
 *   row_ptr   int32 [R+1]; exclusive prefix sum of row_cnt
 *   col_idx   int32 [>= row_ptr[R]]; kept j of each row, ascending (size it
 *             for max_nnz, or for a bound the caller knows)
 *   work_order int32 [R]; longest first, head by head: heads (b, h) by
 *             their total selected blocks descending (ties: lower head
 *             first), and inside each head its rows by row_cnt descending
 *             (ties: lower row first). Rows that run together then share one
 *             head's keys and values in L2.
 * top_p is a host array [H]; values in (0, 1] are meaningful, p >= 1 keeps
 * every block. top_k >= 0. Pooling, scores, softmax and the cumulative mass
 * are fp64 (the cut is found by bisection on the probabilities, not by a
 * sort), so a row can differ from another fp64 evaluation only where its
 * cumulative mass at the cut lies within rounding (~1e-15) of p.
 * The workspace holds the pooled means (2*B*H*nb*d doubles), the pooled
 * scores of a chunk of heads (nb*nb doubles per head; as many heads as 48 MiB
 * hold, at least one) and the status word that device-side checks set. */
SBA_API sba_status sba_build_mask(const sba_plan* plan, const void* qt, const void* kt,
                          const float* top_p, int32_t top_k,
                          uint32_t* bitmask, int32_t* row_cnt, int32_t* row_ptr,
                          int32_t* col_idx, int32_t* work_order,
                          void* workspace, void* stream);

/* Allocation-free sba_build_mask (the paper has no counterpart: this is a
 * deployment convenience). Same inputs, outputs and results as sba_build_mask,
 * but no workspace argument: its scratch (a 256-byte control block, the
 * pooled block means and the pooled scores of as many heads as fit in the
 * rest) lives in one 64 MiB array of static device memory
 * inside the library, which every GPU that loads libsba holds until the
 * process exits. For callers that cannot allocate device memory or carry a
 * workspace: plugin interfaces that pass only inputs and outputs, and services
 * that reserve all device memory at start-up and forbid cudaMalloc afterwards.
 * Limit: 256 + 2*B*H*nb*d*8 bytes (the two rounded up to 256 each) + one
 * head's nb*nb*8 bytes of scores <= 64 MiB (the Wan and HunyuanVideo-shaped
 * layers fit); larger plans return SBA_ERR_CAPACITY before anything is
 * launched.
 * Each call looks up the array's device address on the current device with
 * cudaGetSymbolAddress (a failed lookup is reported, not remembered); inside a
 * stream capture it reuses the last address found on that device, so make one
 * call on each device before capturing. Each call clears the control block
 * with cudaMemsetAsync and overwrites the means and scores; the array keeps the
 * last call's contents. All calls share the one array, so calls that overlap
 * on the GPU (other streams, other threads) race: serialise them. Device-side
 * check failures of the call land in the array's status word: read them with
 * sba_noalloc_status. Never calls cudaMalloc, cudaFree or any allocating
 * routine. */
SBA_API sba_status sba_build_mask_noalloc(const sba_plan* plan, const void* qt, const void* kt,
                                          const float* top_p, int32_t top_k,
                                          uint32_t* bitmask, int32_t* row_cnt, int32_t* row_ptr,
                                          int32_t* col_idx, int32_t* work_order, void* stream);

/* Status word of sba_build_mask_noalloc's static scratch (no counterpart in
 * the paper): synchronise `stream`, read and clear the word. Returns SBA_OK,
 * SBA_ERR_DEVICE_TIMEOUT or SBA_ERR_DEVICE_CHECK like
 * sba_check_device_status, or SBA_ERR_CUDA. */
SBA_API sba_status sba_noalloc_status(void* stream);

/* Stripe mask (Parameterized Stripe Attention for Efficient Video Generation,
 * Approach: a six-parameter mask M(Tw, To, Ts, Sw, So, Ss) of periodic
 * diagonal stripes). A static alternative to sba_build_mask that needs no
 * scores: rows, outputs and their layout are those of sba_build_mask, and
 * sba_attention consumes them unchanged. The page names the parameters but
 * prints no formula; this library reads them as follows. A block has cube
 * coordinates (tt, th, tw) and flattened spatial index sp = th*nW + tw; for
 * query block i and key block j
 *   dt = tt_j - tt_i,   ds = sp_j - sp_i,
 *   x lies in stripe (w, o, s) when 0 <= x - o < w (s == 0), or when
 *   ((x - o) mod s) < w with the non-negative remainder (s > 0);
 *   block j is kept for row i when dt lies in (Tw, To, Ts) and ds in
 *   (Sw, So, Ss) of the row's head.
 * A band of half-width r around the diagonal is (2r+1, -r, 0); s = nW
 * repeats a spatial stripe every cube row. Rows may come out empty (their
 * attention output is zero, lse -inf).
 * params: host array [H], one per head; every width and period >= 0 and
 * every field within [-32768, 32767], else SBA_ERR_INVALID_ARG. Cube order
 * only: plans with SBA_ORDER_HILBERT return SBA_ERR_UNSUPPORTED. Outputs
 * (device, caller-owned) as for sba_build_mask; workspace as for
 * sba_build_mask (its control block records device-side check failures).
 * Integer work only: results are exact. */
SBA_API sba_status sba_build_stripe_mask(const sba_plan* plan, const sba_stripe* params,
                                         uint32_t* bitmask, int32_t* row_cnt, int32_t* row_ptr,
                                         int32_t* col_idx, int32_t* work_order, void* workspace,
                                         void* stream);

/* Low-bit P.V path (VC-Attention: Value Smoothing and Softmax Casting for
 * Low-bit Attention, abstract: V-Smooth and ExpCast-FP8). Two calls beside
 * the bf16 path: sba_smooth_v quantises the values once per layer, and
 * sba_attention_lowbit runs the same block-sparse attention with E4M3
 * probabilities and E4M3 values in the P.V product (S = Q.K^T stays bf16).
 *
 * sba_smooth_v: V-Smooth. For every key block j of head (b, h):
 *   mu_j = mean of vt over the block's real tokens (summed in fp64, rounded
 *   once to fp32); R = vt - mu_j in fp32 (0 on padding slots); one
 *   power-of-two scale per head, 2^e with e the smallest integer such that
 *   max|R| <= 448 * 2^e (e = 0 when R is all zero); codes = E4M3(R * 2^-e),
 *   round to nearest even, saturating at +-448, the sign kept on a negative
 *   value that rounds to zero. (The page's online clustering of value tokens
 *   is not done: cube blocks already hold spatio-temporal neighbours.)
 * Inputs: vt, bf16 [B][H][Npad][d] from sba_reorder (16-byte aligned).
 * Outputs (device, caller-owned): vq uint8 [B][H][nb][d][bs] - each block's
 *   codes transposed, channel-major (16-byte aligned); vmean fp32
 *   [B][H][nb][d] (16-byte aligned); vexp int32 [B][H]. workspace as for
 *   sba_build_mask (two per-head words in it count finished blocks and hold
 *   the head's maximum meanwhile; zero again when the call completes).
 * bf16 plans with d <= 128 only (else SBA_ERR_UNSUPPORTED). Deterministic. */
SBA_API sba_status sba_smooth_v(const sba_plan* plan, const void* vt, void* vq, float* vmean,
                                int32_t* vexp, void* workspace, void* stream);

/* Block-sparse attention with ExpCast-FP8 probabilities and V-Smooth values.
 * Per row (query block i) and selected key block j, on real keys:
 *   x = q.k / sqrt(d) * log2(e) - m, with m the row's reference maximum: the
 *     first selected block's row maximum, replaced by a later block's when that
 *     exceeds it by more than 2.75 (accumulators rescaled);
 *   code = clamp(rint(8x + 104), 0, 126) (one multiply-add: the E4M3 code of
 *     ~2^(x+6), linear in the mantissa between powers of two), P = its value;
 *   A += P . (2^e * codes_j) on the tensor core (kind::f8f6f4, fp32
 *     accumulation), l_j = sum of P over the block, L += l_j;
 *   o = (A + sum_j l_j mu_j) / L, lse = ln(L) + (m - 6) ln(2).
 * Rows without blocks give o = 0 and lse = -inf; padding query slots 0.
 * Inputs as for sba_attention with vq, vmean, vexp from sba_smooth_v; the
 * longest-first persistent scheduler is always used (work_order required).
 * The block-mean term is accumulated in tensor memory; no scratch is needed.
 * bf16 plans with d = 128 and bs = 128 only (else SBA_ERR_UNSUPPORTED).
 * Results are not bit-identical to the bf16 path: E4M3 values carry ~3
 * mantissa bits, so the output departs from exact attention by a few
 * percent (measured and reported by the tests). */
SBA_API sba_status sba_attention_lowbit(const sba_plan* plan, const void* qt, const void* kt,
                                        const void* vq, const float* vmean, const int32_t* vexp,
                                        const int32_t* row_ptr, const int32_t* col_idx,
                                        const int32_t* work_order, void* ot, float* lse,
                                        uint64_t* trace, void* workspace, void* stream);

/* Block-sparse attention forward (FVAttn abstract: attention over the
 * materialised mask). For every real query slot q of block i:
 *   o_q = sum_{j in cols(i)} sum_{real keys k of j} softmax(q.k / sqrt(d)) v_k
 * with the softmax taken over exactly those keys; lse_q = log of its
 * denominator (natural log, scores already divided by sqrt(d)). bf16 inputs
 * run on tcgen05 tensor cores (bf16 operands, fp32 accumulation in tensor
 * memory, fp32 online softmax) and write bf16 ot; f32 inputs run in fp32 on
 * CUDA cores and write f32 ot. Padding query slots get o = 0 and lse = 0; a
 * row with no columns gets o = 0 and lse = -inf.
 *   row_ptr, col_idx  the CSR from sba_build_mask (or any CSR over [0, nb)
 *                     with at most nb columns per row)
 *   work_order        int32 [R], required for SBA_SCHED_LPT, ignored (may be
 *                     NULL) for SBA_SCHED_HEAD_MAJOR. bf16 plans with bs = 64
 *                     run pairs of query blocks (2i, 2i+1) of a head as one
 *                     128-row tile over the union of their columns, taken in
 *                     head order; work_order is then not read (it must still
 *                     be non-NULL for SBA_SCHED_LPT)
 *   lse               float [B][H][Npad] or NULL
 *   trace             NULL, or uint64 [R][3] receiving, per row, the
 *                     %globaltimer ns at which its CTA started and finished it
 *                     and the SM id (for the SM idle / tail measurement)
 * A column index outside [0, nb) is replaced by 0, and a row whose row_ptr
 * range is negative, longer than nb or past B*H*nb*nb is skipped (written as
 * empty); both flag SBA_ERR_DEVICE_CHECK in the workspace status word. */
SBA_API sba_status sba_attention(const sba_plan* plan, const void* qt, const void* kt, const void* vt,
                         const int32_t* row_ptr, const int32_t* col_idx,
                         const int32_t* work_order, void* ot, float* lse,
                         int32_t sched, uint64_t* trace, void* workspace, void* stream);

/* Synchronise `stream`, read and clear the workspace status word. Returns
 * SBA_OK, SBA_ERR_DEVICE_TIMEOUT or SBA_ERR_DEVICE_CHECK (timeouts win). */
SBA_API sba_status sba_check_device_status(const sba_plan* plan, void* workspace, void* stream);

/* Failure-detection probe: launch one CTA that waits, with the library's
 * bounded wait, on a barrier that nothing arrives at, for at most
 * timeout_ns nanoseconds (1e3..1e10). The wait gives up, flags
 * SBA_ERR_DEVICE_TIMEOUT in the status word and the kernel returns normally,
 * leaving the context usable. Used to test the timeout path without a hang. */
SBA_API sba_status sba_debug_timeout_probe(const sba_plan* plan, void* workspace,
                                   uint64_t timeout_ns, void* stream);

/* Numerical probe of the attention softmax's FMA-pipe exponential: y[i] =
 * 2^x[i] as the kernel computes it for one exponential pair in eight (range
 * reduction to f in [-1/2, 1/2], a degree-3 minimax polynomial for 2^f,
 * x clamped at -125). x, y: device fp32 [n], 0 <= n <= 2^31; asynchronous on
 * `stream`. The pages have no counterpart: it exists to test that
 * approximation against the exact 2^x. */
SBA_API sba_status sba_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* Host-only: write the slot of every raster token, int32 [N]. */
SBA_API sba_status sba_perm_export(const sba_plan* plan, int32_t* slot_of_token);

/* Number of SMs the persistent attention grid uses on the current device
 * (0 before the first sba_attention call in this process). */
SBA_API int32_t sba_attention_grid_size(void);

SBA_API const char* sba_status_string(sba_status status);
/* Message of the last failed call on this thread ("" if none). */
SBA_API const char* sba_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SBA_H_ */
