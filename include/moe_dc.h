/*
 * moe_dc.h — C ABI of the B200 (sm_100a) MoE token dispatch / combine library.
 *
 * One device, no collective: the expert-parallel alltoallv of the Ascend CANN
 * "low_latency_combine" page (Function: Description and Formula) collapses to a
 * local permute, and combine returns every row "along the same path".
 *
 * Conventions shared by every call below
 * --------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller, dense and
 *   row-major, 16-byte aligned where a row of 16-bit values is read or
 *   written. The library allocates nothing and keeps no state between calls.
 * - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *   stream. Work is enqueued asynchronously on it; nothing synchronises.
 * - Host-side checks run first and return a status before anything is
 *   launched: nothing is written when a call returns an error other than
 *   MOE_ERR_CUDA.
 * - Data errors found on the device (an id outside [0, N), an id repeated
 *   within a row) never fault: the pair is ignored and a bit is set in the
 *   layout's `dev_status` word.
 * - Every call is deterministic: no floating-point atomics, a fixed k order
 *   and fixed reduction trees ([combine] Deterministic Computation).
 *
 * Symbols: BS tokens, K experts per token, H hidden size, E routed experts,
 * Z zero, C copy, Q const experts, N = E + Z + C + Q ids, A expanded-row
 * capacity, R routed active pairs (R <= A).
 */
#ifndef MOE_DC_H
#define MOE_DC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,          /* bad size, null pointer, bad mode */
  MOE_ERR_UNSUPPORTED = 2,  /* a valid request this build does not implement */
  MOE_ERR_ALIGN = 3,        /* H * 2 not a multiple of 16, or a misaligned pointer */
  MOE_ERR_CAPACITY = 4,     /* a_capacity < BS * min(E, K), or workspace too small */
  MOE_ERR_CUDA = 5          /* a CUDA launch failed; see moe_last_cuda_error() */
} moe_status;

typedef enum { MOE_BF16 = 0, MOE_FP16 = 1 } moe_dtype;

/* Bits of the device status word written by moe_dispatch_layout. */
#define MOE_DEV_BAD_ID 1u  /* some id outside [0, N) */
#define MOE_DEV_DUP_ID 2u  /* some id repeated within a row; later copies ignored */

/*
 * Problem shape. [combine] Parameters table and Constraints:
 *   bs               tokens (BS >= 0; the page's BS <= 512 is not enforced)
 *   k                experts per token, 0 < K <= 16 and K <= N
 *   h                hidden size, H > 0 and H * 2 a multiple of 16
 *   num_experts      routed experts E, 1 <= E <= 1024
 *   zero/copy/const_expert_num   Z, C, Q >= 0; ids [E, E+Z) are zero experts,
 *                    [E+Z, E+Z+C) copy experts, [E+Z+C, N) const experts
 *   a_capacity       A, rows of expand_x; A >= BS * min(E, K)
 *   dtype            moe_dtype of x, expand_x and every 16-bit tensor
 *   mask_ndim        0: no x_active_mask; 1: mask (BS,); 2: mask (BS, K)
 */
typedef struct {
  int32_t bs, k, h, num_experts, zero_expert_num, copy_expert_num, const_expert_num,
      a_capacity;
  int32_t dtype;
  int32_t mask_ndim;
} moe_shape;

/* Text of a status code (static storage). */
const char* moe_status_string(int status);

/* The CUDA error (cudaError_t value) behind the last MOE_ERR_CUDA on this thread. */
int moe_last_cuda_error(void);

/*
 * Number of thread blocks on the current device that gave up a bounded wait
 * for an asynchronous copy since the library was loaded (0 in normal
 * operation; such a block leaves its part of the output unwritten).
 * Synchronises the device. Returns UINT32_MAX if the count cannot be read.
 */
uint32_t moe_async_wait_timeouts(void);

/* Elements of the int32 assist_info buffer: A + BS * K. */
size_t moe_assist_info_elems(const moe_shape* shape);

/* Bytes of device workspace moe_dispatch_layout needs (may be 0). */
size_t moe_layout_workspace_bytes(const moe_shape* shape);

/*
 * moe_dispatch_layout — [combine] Parameters (assist_info_for_combine,
 * ep_send_counts, x_active_mask) and Constraints.
 *
 * A pair (t, k) is routed when topk_idx[t, k] is in [0, E), is not a repeat of
 * an earlier id in row t, and is active in the mask. Routed pairs are laid out
 * expert by expert, and inside an expert by token (a stable order); pair
 * (t, k) gets slot s.
 *   topk_idx           int32 (BS, K), in
 *   x_active_mask      uint8 (BS,) or (BS, K) per shape->mask_ndim, or NULL
 *   expert_token_nums  int32 (E,), out: routed pairs per expert
 *   ep_send_counts     int32 (E + 1,), out: exclusive prefix sum of
 *                      expert_token_nums with the total R appended; expert e
 *                      owns slots [ep_send_counts[e], ep_send_counts[e + 1])
 *   assist_info        int32 (A + BS * K,), out, opaque to callers: entry s < A
 *                      holds t * K + k of the pair in slot s (-1 for s >= R);
 *                      entry A + t * K + k holds the slot of pair (t, k), or -1
 *   dev_status         uint32 (1,), out, or NULL: overwritten with the
 *                      MOE_DEV_* bits found in topk_idx
 *   workspace          device scratch of moe_layout_workspace_bytes() bytes
 *                      (NULL allowed when that is 0); its contents on entry do
 *                      not matter
 * Up to 16384 tokens (while the per-warp expert masks fit in shared memory)
 * the layout is one launch of a thread-block cluster of up to 16 blocks and
 * needs no workspace; a device that cannot hold such a cluster returns
 * MOE_ERR_CUDA (cudaErrorInvalidClusterSize) unless a workspace for the
 * tiled path is given (tile counts, expert totals and a status word per tile
 * of 256 tokens: 4 * (T * E + E + T) bytes, T = ceil(BS / 256)). Larger shapes
 * take the tiled path: three launches (count, column scan, scatter).
 */
moe_status moe_dispatch_layout(const moe_shape* shape, const int32_t* topk_idx,
                               const uint8_t* x_active_mask, int32_t* expert_token_nums,
                               int32_t* ep_send_counts, int32_t* assist_info,
                               uint32_t* dev_status, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * moe_dispatch_permute — the local stand-in for dispatch's alltoallv
 * ([combine] Function: Description) with the optional per-row int8
 * quantisation of comm_quant_mode / quant_mode 2 ([combine] Parameters,
 * Example).
 *   x                (BS, H) dtype, in
 *   assist_info      from moe_dispatch_layout, in
 *   ep_send_counts   accepted for interface parity with the page; not read
 *   comm_quant_mode  0: expand_x[s] = x[t] bit for bit, expand_x is (A, H) dtype
 *                    2: scale[t] = max_h |x[t, h]| / 127 (fp32, IEEE division),
 *                       expand_x[s] = int8(clamp(rne(x[t] / scale), -127, 127)),
 *                       dynamic_scales[s] = scale; expand_x is (A, H) int8 and
 *                       H must be a multiple of 16; all-zero rows give scale 0
 *   Rows s >= R of expand_x (and dynamic_scales) are not written.
 */
moe_status moe_dispatch_permute(const moe_shape* shape, const void* x,
                                const int32_t* assist_info, const int32_t* ep_send_counts,
                                int comm_quant_mode, void* expand_x, float* dynamic_scales,
                                void* stream);

/*
 * moe_dispatch_permute_smooth — int8 dispatch of smooth-scaled rows: the
 * graph-mode dispatch of the [combine] Example passes quant_mode 2 with a
 * scales tensor of shape (E, H), read here as one fp32 factor per expert and
 * hidden channel applied before the per-row quantisation.
 *   x                (BS, H) dtype, in
 *   topk_idx         int32 (BS, K), in: the ids moe_dispatch_layout was given
 *   assist_info      from moe_dispatch_layout, in
 *   ep_send_counts   from moe_dispatch_layout, in: the total R = ep_send_counts[E]
 *                    is read (clamped to [0, A])
 *   smooth_scales    fp32 (E, H), in, 16-byte aligned
 *   For slot s of pair (t, k) with expert e = topk_idx[t, k]:
 *     y = fp32(x[t] * smooth_scales[e]) (one rounding per element),
 *     scale = max_h |y| / 127 (IEEE division), expand_x[s] =
 *     int8(clamp(rne(y / scale), -127, 127)), dynamic_scales[s] = scale;
 *     an all-zero y gives scale 0 and zero codes.
 *   expand_x         int8 (A, H), out; dynamic_scales fp32 (A,), out. Rows
 *                    s >= R are not written. H must be a multiple of 16 and at
 *                    most 16384 (MOE_ERR_ALIGN / MOE_ERR_UNSUPPORTED).
 */
moe_status moe_dispatch_permute_smooth(const moe_shape* shape, const void* x,
                                       const int32_t* topk_idx, const int32_t* assist_info,
                                       const int32_t* ep_send_counts, const float* smooth_scales,
                                       void* expand_x, float* dynamic_scales, void* stream);

/*
 * moe_dispatch — moe_dispatch_layout followed by moe_dispatch_permute, in one
 * call (the dispatch of the [combine] Example: low_latency_dispatch returns
 * the expanded rows, the counts and assist_info together). For BS <= 1024
 * without quantisation (and E <= 640, whose lane masks fit in shared memory)
 * both run in one launch (every CTA
 * rebuilds the small layout in shared memory and copies its share of rows);
 * otherwise the launches of the two separate calls. Arguments and results as
 * in those calls; the workspace may be NULL when moe_layout_workspace_bytes()
 * is 0.
 */
moe_status moe_dispatch(const moe_shape* shape, const int32_t* topk_idx,
                        const uint8_t* x_active_mask, const void* x, int comm_quant_mode,
                        int32_t* expert_token_nums, int32_t* ep_send_counts,
                        int32_t* assist_info, uint32_t* dev_status, void* expand_x,
                        float* dynamic_scales, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * moe_combine_fwd — [combine] Function (Formula; special expert use cases),
 * Parameters, Return Value:
 *   out[t] = round16( sum_{k active, ascending} w[t,k] * M(t,k)  +  shared[t] )
 * with M = expand_x[slot(t,k)] for routed pairs, 0 for zero experts, ori_x[t]
 * for copy experts, alpha_1[j] * ori_x[t] + alpha_2[j] * v[j] for const expert
 * j = id - (E + Z + C). Everything is fp32 with each product and each sum
 * rounded on its own (no fused multiply-add), then one round-to-nearest-even
 * cast.
 *   expand_x         (A, H) dtype: the experts' outputs, in slot order
 *   topk_idx         int32 (BS, K); topk_weights fp32 (BS, K)
 *   assist_info      from moe_dispatch_layout; ep_send_counts: not read
 *   x_active_mask    as for the layout, or NULL
 *   shared_expert_x  (BS, H) dtype or NULL (added once, unweighted)
 *   ori_x            (BS, H) dtype; required when C > 0 or Q > 0
 *   const_alpha_1, const_alpha_2, const_v   (Q, H) dtype; required when Q > 0
 *   out              (BS, H) dtype
 */
moe_status moe_combine_fwd(const moe_shape* shape, const void* expand_x,
                           const int32_t* topk_idx, const float* topk_weights,
                           const int32_t* assist_info, const int32_t* ep_send_counts,
                           const uint8_t* x_active_mask, const void* shared_expert_x,
                           const void* ori_x, const void* const_alpha_1,
                           const void* const_alpha_2, const void* const_v, void* out,
                           void* stream);

/*
 * moe_combine_fwd_comm_quant — moe_combine_fwd with the combine side's
 * comm_quant_mode ([combine] Parameters: 0 no quantisation, 2 int8
 * quantisation of the communicated rows). At one device the expert-output
 * rows do not travel, so mode 2 is the round trip each routed row would make:
 * scale = max_h |y[s, h]| / 127 (fp32, IEEE division), q = clamp(rne(y / scale),
 * -127, 127), and the weighted sum uses the fp32 value q * scale (an all-zero
 * row contributes 0). Copy/const experts and shared_expert_x are local and are
 * not quantised. Mode 0 is exactly moe_combine_fwd. Other arguments as there.
 */
moe_status moe_combine_fwd_comm_quant(const moe_shape* shape, const void* expand_x,
                                      const int32_t* topk_idx, const float* topk_weights,
                                      const int32_t* assist_info, const int32_t* ep_send_counts,
                                      const uint8_t* x_active_mask, const void* shared_expert_x,
                                      const void* ori_x, const void* const_alpha_1,
                                      const void* const_alpha_2, const void* const_v,
                                      int comm_quant_mode, void* out, void* stream);

/*
 * moe_combine_fwd_comm_quant_ws — moe_combine_fwd_comm_quant with an optional
 * device workspace (same results, bit for bit). With a workspace of
 * moe_combine_fwd_comm_quant_workspace_bytes() bytes (16-byte aligned) and
 * mode 2, shapes without zero/copy/const experts whose rows are wide enough
 * (H / 8 >= 32 * U, with U = 4, 2, 1 for K <= 2, K <= 4, K > 4) run in two
 * passes: each slot row's scale and reciprocal into the workspace (one
 * streaming read of the rows, R = ep_send_counts[E] of them), then the
 * weighted gather with the round trip. Other shapes, or workspace NULL, take
 * the one-pass int8 combine: a warp-specialised kernel that stages each
 * token's rows in shared memory with bulk copies where its buffers fit, else a
 * kernel that reads each token's rows twice through L1.
 *   workspace        NULL or device scratch; its contents on entry do not
 *                    matter (MOE_ERR_CAPACITY if smaller than required,
 *                    MOE_ERR_ALIGN if not 16-byte aligned)
 *   ep_send_counts   from moe_dispatch_layout; required with a workspace
 */
size_t moe_combine_fwd_comm_quant_workspace_bytes(const moe_shape* shape);
moe_status moe_combine_fwd_comm_quant_ws(const moe_shape* shape, const void* expand_x,
                                         const int32_t* topk_idx, const float* topk_weights,
                                         const int32_t* assist_info,
                                         const int32_t* ep_send_counts,
                                         const uint8_t* x_active_mask,
                                         const void* shared_expert_x, const void* ori_x,
                                         const void* const_alpha_1, const void* const_alpha_2,
                                         const void* const_v, int comm_quant_mode, void* out,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_combine_bwd — gradient of the combine Formula for routed pairs (the
 * fused EP MoE layer of the Triton-distributed ep_moe_fused PR has a backward):
 *   grad_expand[slot(t,k)] = round16(w[t,k] * grad_out[t])     (fp32 product)
 *   grad_w[t,k]            = sum_h grad_out[t,h] * expand_x[slot(t,k),h] (fp32)
 * Pairs without a slot or masked get grad_w = 0 and write no row. The gradient
 * of shared_expert_x is grad_out itself (no call needed).
 *   grad_out (BS, H), expand_x (A, H), topk_weights fp32 (BS, K),
 *   grad_expand (A, H) out, grad_w fp32 (BS, K) out. topk_idx is not read.
 */
moe_status moe_combine_bwd(const moe_shape* shape, const void* grad_out, const void* expand_x,
                           const int32_t* topk_idx, const float* topk_weights,
                           const int32_t* assist_info, const uint8_t* x_active_mask,
                           void* grad_expand, float* grad_w, void* stream);

/*
 * moe_combine_bwd_comm_quant — the backward of moe_combine_fwd_comm_quant
 * ([combine] Parameters: comm_quant_mode). Mode 0 is moe_combine_bwd. Mode 2:
 * the forward summed each routed row's int8 round-trip values D(y) = fp32
 * q * scale (scale = max_h |y| / 127, IEEE division; q as in the forward), so
 *   grad_w[t,k]            = sum_h grad_out[t,h] * D(expand_x[slot(t,k)])[h]
 * and the round trip, piecewise constant, is passed straight through:
 *   grad_expand[slot(t,k)] = round16(w[t,k] * grad_out[t])  (as in mode 0).
 * Arguments, layouts and the pairs without a slot as in moe_combine_bwd;
 * MOE_ERR_ARG for a mode other than 0 or 2.
 */
moe_status moe_combine_bwd_comm_quant(const moe_shape* shape, const void* grad_out,
                                      const void* expand_x, const int32_t* topk_idx,
                                      const float* topk_weights, const int32_t* assist_info,
                                      const uint8_t* x_active_mask, int comm_quant_mode,
                                      void* grad_expand, float* grad_w, void* stream);

/*
 * moe_combine_bwd_special — gradient of the combine Formula through the copy
 * and const experts ([combine] Function, special expert use cases: copy
 * Moe(ori_x) = ori_x, const Moe(ori_x) = alpha_1 * ori_x + alpha_2 * v), the
 * part moe_combine_bwd leaves out. With g = grad_out[t], c = fl(w[t,k] * g):
 *   grad_w[t,k]     = sum_h g * M(t,k)   (fp32) for copy and const pairs only;
 *                     other entries of grad_w are not written (run
 *                     moe_combine_bwd first for the routed pairs)
 *   grad_ori_x[t]   = round16( sum over copy/const k, ascending, of c (copy)
 *                     or fl(c * alpha_1[j]) (const) ), (BS, H) dtype; 0 for
 *                     tokens without such pairs
 *   grad_alpha_1[j] = sum over pairs of const j of c * ori_x[t]  (Q, H) fp32
 *   grad_alpha_2[j] = S_j * v[j],  grad_v[j] = S_j * alpha_2[j],
 *                     S_j = sum over pairs of const j of c        (Q, H) fp32
 * Sums over tokens run in a fixed order (chunks of 64 tokens, then the
 * chunks in order), so results are deterministic. ori_x is required; the
 * const tensors and their gradients when Q > 0. workspace: device scratch of
 * moe_combine_bwd_special_workspace_bytes() bytes (0 when Q = 0).
 */
size_t moe_combine_bwd_special_workspace_bytes(const moe_shape* shape);
moe_status moe_combine_bwd_special(const moe_shape* shape, const void* grad_out,
                                   const int32_t* topk_idx, const float* topk_weights,
                                   const uint8_t* x_active_mask, const void* ori_x,
                                   const void* const_alpha_1, const void* const_alpha_2,
                                   const void* const_v, float* grad_w, void* grad_ori_x,
                                   float* grad_alpha_1, float* grad_alpha_2, float* grad_v,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_dispatch_bwd — gradient of the permute: every token gathers the
 * gradients of its slots, unweighted, summed in fp32 in ascending k:
 *   grad_x[t] = round16( sum_{k with a slot, active} grad_expand_in[slot(t,k)] )
 *   grad_expand_in (A, H), grad_x (BS, H) out.
 */
moe_status moe_dispatch_bwd(const moe_shape* shape, const void* grad_expand_in,
                            const int32_t* assist_info, const uint8_t* x_active_mask,
                            void* grad_x, void* stream);

/*
 * moe_dispatch_layout_noalloc — moe_dispatch_layout for callers that cannot
 * allocate device memory. No counterpart on the [combine] page: an addition of this
 * library. It is for code that runs where every byte of device memory is
 * owned by someone else — a plugin or kernel library handed buffers by a host
 * framework that exposes no allocator, or a latency-critical serving loop that
 * must not call cudaMalloc (which can synchronise the device) — and so cannot
 * provide the workspace moe_dispatch_layout wants.
 *
 * Same arguments and results as moe_dispatch_layout, minus the workspace: the
 * scratch is one fixed array of moe_layout_noalloc_max_workspace_bytes()
 * bytes (1 MiB) compiled into the library, which every GPU that loads the
 * library keeps until the process exits. A shape whose
 * moe_layout_workspace_bytes() exceeds that size returns MOE_ERR_CAPACITY
 * before anything runs (1 MiB covers, e.g., BS = 65 280 tokens with E = 1024,
 * or about a million tokens with E = 64).
 *
 * The call allocates nothing (no cudaMalloc, no cudaFree, no allocator of any
 * library). The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it for the
 * life of the process; make that first call before any stream capture. A
 * device reset (cudaDeviceReset, or anything else that destroys the primary
 * context) may move the array, so do not call this entry point in a process
 * after resetting the device it runs on. Every call shares the one array and
 * leaves its contents behind; nothing in it needs clearing, because every
 * entry the layout reads is written earlier in the same call. Calls whose
 * work can overlap on the GPU (other streams, other threads) race on the
 * array: serialise them, or give each its own workspace with
 * moe_dispatch_layout.
 */
moe_status moe_dispatch_layout_noalloc(const moe_shape* shape, const int32_t* topk_idx,
                                       const uint8_t* x_active_mask, int32_t* expert_token_nums,
                                       int32_t* ep_send_counts, int32_t* assist_info,
                                       uint32_t* dev_status, void* stream);

/* Bytes of the fixed scratch array moe_dispatch_layout_noalloc uses. */
size_t moe_layout_noalloc_max_workspace_bytes(void);

/*
 * Test hooks for the bounded waits (no counterpart on the pages). The staged
 * kernels (the one-pass int8 combine, the smooth-scaled int8 dispatch) wait on
 * mbarriers for their own bulk copies; every such wait gives up after a time
 * limit, counts the giving-up block (or warp) in moe_async_wait_timeouts(),
 * lets the copies it started land, and returns, leaving its part of the output
 * unwritten. These two calls run those kernels with a shorter limit and one
 * unit of work whose barrier is armed for 16 bytes that no copy delivers, so
 * that the give-up path runs while no copy is in flight for that unit. Not for
 * production use.
 *   wait_limit_ns   limit of the pipeline waits, in (0, 1e9] ns
 *   withhold_unit   >= 0: the int8 combine's first block's token number
 *                   withhold_unit (in that block's order), or the smooth
 *                   dispatch's first warp's slot number withhold_unit
 * Other arguments as moe_combine_fwd_comm_quant (mode 2) and
 * moe_dispatch_permute_smooth. MOE_ERR_UNSUPPORTED for shapes those calls run
 * on other kernels (K > 8, or rows whose buffers do not fit in shared memory).
 */
moe_status moe_test_combine_fwd_comm_quant_wait_timeout(
    const moe_shape* shape, const void* expand_x, const int32_t* topk_idx,
    const float* topk_weights, const int32_t* assist_info, const uint8_t* x_active_mask,
    const void* shared_expert_x, const void* ori_x, const void* const_alpha_1,
    const void* const_alpha_2, const void* const_v, void* out, uint64_t wait_limit_ns,
    int withhold_unit, void* stream);
moe_status moe_test_dispatch_permute_smooth_wait_timeout(
    const moe_shape* shape, const void* x, const int32_t* topk_idx, const int32_t* assist_info,
    const int32_t* ep_send_counts, const float* smooth_scales, void* expand_x,
    float* dynamic_scales, uint64_t wait_limit_ns, int withhold_unit, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DC_H */
