// C ABI of the dispatch/combine library: host-side argument checks, then the
// kernel launches of layout.cu, permute.cu and combine.cu. Declarations and
// the meaning of every argument are in include/moe_dc.h.
#include <cuda_runtime.h>

#include <cstdint>

#include "launch.cuh"
#include "moe_dc.h"

namespace {

thread_local int g_last_cuda_error = 0;

moe_status cuda_status(cudaError_t err) {
  if (err == cudaSuccess) return MOE_OK;
  g_last_cuda_error = static_cast<int>(err);
  return MOE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks shared by every call. [combine] Parameters and Constraints: K in
// (0, 16] and K <= N, E in [1, 1024], N < 2^31, A >= BS * min(E, K) at one
// device; H * 2 a multiple of 16 for 16-byte row vectors.
moe_status check_shape(const moe_shape* s) {
  if (s == nullptr) return MOE_ERR_ARG;
  if (s->dtype != MOE_BF16 && s->dtype != MOE_FP16) return MOE_ERR_ARG;
  if (s->bs < 0 || s->k <= 0 || s->k > 16 || s->h <= 0) return MOE_ERR_ARG;
  if (s->num_experts < 1 || s->num_experts > 1024) return MOE_ERR_ARG;
  if (s->zero_expert_num < 0 || s->copy_expert_num < 0 || s->const_expert_num < 0)
    return MOE_ERR_ARG;
  const int64_t n = static_cast<int64_t>(s->num_experts) + s->zero_expert_num +
                    s->copy_expert_num + s->const_expert_num;
  if (n >= (int64_t{1} << 31) || s->k > n) return MOE_ERR_ARG;
  if (s->mask_ndim < 0 || s->mask_ndim > 2) return MOE_ERR_ARG;
  if ((static_cast<int64_t>(s->h) * 2) % 16 != 0) return MOE_ERR_ALIGN;
  const int64_t pairs = static_cast<int64_t>(s->bs) * s->k;
  if (s->a_capacity < 0 || pairs + s->a_capacity >= (int64_t{1} << 31)) return MOE_ERR_ARG;
  // every index a kernel forms from a row and a 16-byte vector fits in int32
  const int64_t vecs = static_cast<int64_t>(s->h) / 8;
  if (static_cast<int64_t>(s->bs) * vecs >= (int64_t{1} << 31) ||
      static_cast<int64_t>(s->a_capacity) * vecs >= (int64_t{1} << 40))
    return MOE_ERR_UNSUPPORTED;
  const int64_t per_token = s->k < s->num_experts ? s->k : s->num_experts;
  if (s->a_capacity < static_cast<int64_t>(s->bs) * per_token) return MOE_ERR_CAPACITY;
  return MOE_OK;
}

moe_status check_mask(const moe_shape* s, const uint8_t* mask) {
  return (s->bs > 0 && s->mask_ndim > 0 && mask == nullptr) ? MOE_ERR_ARG : MOE_OK;
}

// Checks of the combine forward's arguments, then its launch arguments.
moe_status combine_args(const moe_shape* s, const void* expand_x, const int32_t* topk_idx,
                        const float* topk_weights, const int32_t* assist_info,
                        const uint8_t* x_active_mask, const void* shared_expert_x,
                        const void* ori_x, const void* const_alpha_1, const void* const_alpha_2,
                        const void* const_v, void* out, moe::CombineArgs* a) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if ((st = check_mask(s, x_active_mask)) != MOE_OK) return st;
  const bool special = s->zero_expert_num + s->copy_expert_num + s->const_expert_num > 0;
  if (s->bs > 0 && (expand_x == nullptr || topk_weights == nullptr || assist_info == nullptr ||
                    out == nullptr || (special && topk_idx == nullptr)))
    return MOE_ERR_ARG;
  // [combine] Parameters: ori_x is required with copy or const experts, and
  // the three const-expert tensors with const experts.
  if (s->bs > 0 && (s->copy_expert_num > 0 || s->const_expert_num > 0) && ori_x == nullptr)
    return MOE_ERR_ARG;
  if (s->bs > 0 && s->const_expert_num > 0 &&
      (const_alpha_1 == nullptr || const_alpha_2 == nullptr || const_v == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(expand_x) || !aligned16(out) || !aligned16(shared_expert_x) ||
      !aligned16(ori_x) || !aligned16(const_alpha_1) || !aligned16(const_alpha_2) ||
      !aligned16(const_v))
    return MOE_ERR_ALIGN;
  a->expand_x = expand_x;
  a->topk_idx = topk_idx;
  a->weights = topk_weights;
  a->assist = assist_info;
  a->mask = x_active_mask;
  a->mask_ndim = s->mask_ndim;
  a->shared = shared_expert_x;
  a->ori_x = ori_x;
  a->alpha1 = const_alpha_1;
  a->alpha2 = const_alpha_2;
  a->const_v = const_v;
  a->out = out;
  a->bs = s->bs;
  a->K = s->k;
  a->H = s->h;
  a->A = s->a_capacity;
  a->E = s->num_experts;
  a->Z = s->zero_expert_num;
  a->C = s->copy_expert_num;
  a->Q = s->const_expert_num;
  a->dtype = s->dtype;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_ALIGN: return "misaligned size or pointer";
    case MOE_ERR_CAPACITY: return "capacity or workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

uint32_t moe_async_wait_timeouts(void) {
  unsigned* p = moe::wait_timeout_counter();
  unsigned v = 0;
  if (p == nullptr || cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return UINT32_MAX;
  return v;
}

size_t moe_assist_info_elems(const moe_shape* s) {
  if (s == nullptr) return 0;
  return static_cast<size_t>(s->a_capacity) + static_cast<size_t>(s->bs) * s->k;
}

size_t moe_layout_workspace_bytes(const moe_shape* s) {
  if (s == nullptr || check_shape(s) != MOE_OK) return 0;
  return moe::layout_workspace_bytes(s->bs, s->num_experts, s->k);
}

moe_status moe_dispatch_layout(const moe_shape* s, const int32_t* topk_idx,
                               const uint8_t* x_active_mask, int32_t* expert_token_nums,
                               int32_t* ep_send_counts, int32_t* assist_info,
                               uint32_t* dev_status, void* workspace, size_t workspace_bytes,
                               void* stream) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if ((st = check_mask(s, x_active_mask)) != MOE_OK) return st;
  if ((s->bs > 0 && topk_idx == nullptr) || expert_token_nums == nullptr ||
      ep_send_counts == nullptr || (moe_assist_info_elems(s) > 0 && assist_info == nullptr))
    return MOE_ERR_ARG;
  const size_t need = moe::layout_workspace_bytes(s->bs, s->num_experts, s->k);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return MOE_ERR_CAPACITY;
  if (need > 0 && !aligned16(workspace)) return MOE_ERR_ALIGN;
  moe::LayoutArgs a;
  a.topk_idx = topk_idx;
  a.mask = x_active_mask;
  a.mask_ndim = s->mask_ndim;
  a.bs = s->bs;
  a.K = s->k;
  a.E = s->num_experts;
  a.N = s->num_experts + s->zero_expert_num + s->copy_expert_num + s->const_expert_num;
  a.A = s->a_capacity;
  a.expert_token_nums = expert_token_nums;
  a.ep_send_counts = ep_send_counts;
  a.assist = assist_info;
  a.dev_status = dev_status;
  a.workspace = workspace;
  a.workspace_bytes = workspace == nullptr ? 0 : workspace_bytes;
  return cuda_status(moe::launch_layout(a, static_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch_permute(const moe_shape* s, const void* x, const int32_t* assist_info,
                                const int32_t* ep_send_counts, int comm_quant_mode,
                                void* expand_x, float* dynamic_scales, void* stream) {
  (void)ep_send_counts;
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if (comm_quant_mode != 0 && comm_quant_mode != 2) return MOE_ERR_ARG;
  if (s->bs > 0 && (x == nullptr || assist_info == nullptr || expand_x == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(expand_x)) return MOE_ERR_ALIGN;
  if (comm_quant_mode == 2) {
    if (s->bs > 0 && dynamic_scales == nullptr) return MOE_ERR_ARG;
    if (s->h % 16 != 0) return MOE_ERR_ALIGN;
    if (s->h > 16384) return MOE_ERR_UNSUPPORTED;
  }
  moe::PermuteArgs a;
  a.x = x;
  a.assist = assist_info;
  a.expand_x = expand_x;
  a.scales = dynamic_scales;
  a.bs = s->bs;
  a.K = s->k;
  a.H = s->h;
  a.A = s->a_capacity;
  a.dtype = s->dtype;
  a.quant_mode = comm_quant_mode;
  return cuda_status(moe::launch_permute(a, static_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch_permute_smooth(const moe_shape* s, const void* x,
                                       const int32_t* topk_idx, const int32_t* assist_info,
                                       const int32_t* ep_send_counts, const float* smooth_scales,
                                       void* expand_x, float* dynamic_scales, void* stream) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if (s->bs > 0 && (x == nullptr || topk_idx == nullptr || assist_info == nullptr ||
                    ep_send_counts == nullptr || smooth_scales == nullptr ||
                    expand_x == nullptr || dynamic_scales == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(expand_x) || !aligned16(smooth_scales)) return MOE_ERR_ALIGN;
  if (s->h % 16 != 0) return MOE_ERR_ALIGN;
  if (s->h > 16384) return MOE_ERR_UNSUPPORTED;
  moe::PermuteArgs a;
  a.x = x;
  a.assist = assist_info;
  a.expand_x = expand_x;
  a.scales = dynamic_scales;
  a.bs = s->bs;
  a.K = s->k;
  a.H = s->h;
  a.A = s->a_capacity;
  a.dtype = s->dtype;
  a.quant_mode = 2;
  return cuda_status(moe::launch_permute_smooth(a, topk_idx, smooth_scales, ep_send_counts,
                                                s->num_experts,
                                                static_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch(const moe_shape* s, const int32_t* topk_idx, const uint8_t* x_active_mask,
                        const void* x, int comm_quant_mode, int32_t* expert_token_nums,
                        int32_t* ep_send_counts, int32_t* assist_info, uint32_t* dev_status,
                        void* expand_x, float* dynamic_scales, void* workspace,
                        size_t workspace_bytes, void* stream) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  const bool fused = comm_quant_mode == 0 && s->bs <= moe::kLayoutSmallMaxTokens &&
                     moe::dispatch_small_fits(s->num_experts, s->k);
  if (!fused) {
    st = moe_dispatch_layout(s, topk_idx, x_active_mask, expert_token_nums, ep_send_counts,
                             assist_info, dev_status, workspace, workspace_bytes, stream);
    if (st != MOE_OK) return st;
    return moe_dispatch_permute(s, x, assist_info, ep_send_counts, comm_quant_mode, expand_x,
                                dynamic_scales, stream);
  }
  if ((st = check_mask(s, x_active_mask)) != MOE_OK) return st;
  if ((s->bs > 0 && (topk_idx == nullptr || x == nullptr || expand_x == nullptr)) ||
      expert_token_nums == nullptr || ep_send_counts == nullptr ||
      (moe_assist_info_elems(s) > 0 && assist_info == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(expand_x)) return MOE_ERR_ALIGN;
  moe::LayoutArgs a;
  a.topk_idx = topk_idx;
  a.mask = x_active_mask;
  a.mask_ndim = s->mask_ndim;
  a.bs = s->bs;
  a.K = s->k;
  a.E = s->num_experts;
  a.N = s->num_experts + s->zero_expert_num + s->copy_expert_num + s->const_expert_num;
  a.A = s->a_capacity;
  a.expert_token_nums = expert_token_nums;
  a.ep_send_counts = ep_send_counts;
  a.assist = assist_info;
  a.dev_status = dev_status;
  a.workspace = nullptr;
  a.workspace_bytes = 0;
  return cuda_status(
      moe::launch_dispatch_small(a, x, expand_x, s->h, static_cast<cudaStream_t>(stream)));
}

moe_status moe_combine_fwd(const moe_shape* s, const void* expand_x, const int32_t* topk_idx,
                           const float* topk_weights, const int32_t* assist_info,
                           const int32_t* ep_send_counts, const uint8_t* x_active_mask,
                           const void* shared_expert_x, const void* ori_x,
                           const void* const_alpha_1, const void* const_alpha_2,
                           const void* const_v, void* out, void* stream) {
  return moe_combine_fwd_comm_quant(s, expand_x, topk_idx, topk_weights, assist_info,
                                    ep_send_counts, x_active_mask, shared_expert_x, ori_x,
                                    const_alpha_1, const_alpha_2, const_v, 0, out, stream);
}

moe_status moe_combine_fwd_comm_quant(const moe_shape* s, const void* expand_x,
                                      const int32_t* topk_idx, const float* topk_weights,
                                      const int32_t* assist_info, const int32_t* ep_send_counts,
                                      const uint8_t* x_active_mask, const void* shared_expert_x,
                                      const void* ori_x, const void* const_alpha_1,
                                      const void* const_alpha_2, const void* const_v,
                                      int comm_quant_mode, void* out, void* stream) {
  return moe_combine_fwd_comm_quant_ws(s, expand_x, topk_idx, topk_weights, assist_info,
                                       ep_send_counts, x_active_mask, shared_expert_x, ori_x,
                                       const_alpha_1, const_alpha_2, const_v, comm_quant_mode,
                                       out, nullptr, 0, stream);
}

size_t moe_combine_fwd_comm_quant_workspace_bytes(const moe_shape* s) {
  if (s == nullptr || s->a_capacity <= 0) return 0;
  return moe::combine_q8_workspace_bytes(s->a_capacity);
}

moe_status moe_combine_fwd_comm_quant_ws(const moe_shape* s, const void* expand_x,
                                         const int32_t* topk_idx, const float* topk_weights,
                                         const int32_t* assist_info,
                                         const int32_t* ep_send_counts,
                                         const uint8_t* x_active_mask,
                                         const void* shared_expert_x, const void* ori_x,
                                         const void* const_alpha_1, const void* const_alpha_2,
                                         const void* const_v, int comm_quant_mode, void* out,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  if (comm_quant_mode != 0 && comm_quant_mode != 2) return MOE_ERR_ARG;
  moe::CombineArgs a;
  moe_status st = combine_args(s, expand_x, topk_idx, topk_weights, assist_info, x_active_mask,
                               shared_expert_x, ori_x, const_alpha_1, const_alpha_2, const_v,
                               out, &a);
  if (st != MOE_OK) return st;
  if (!aligned16(workspace)) return MOE_ERR_ALIGN;
  if (workspace != nullptr &&
      workspace_bytes < moe::combine_q8_workspace_bytes(s->a_capacity > 0 ? s->a_capacity : 0))
    return MOE_ERR_CAPACITY;
  if (workspace != nullptr && s->bs > 0 && ep_send_counts == nullptr) return MOE_ERR_ARG;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return cuda_status(comm_quant_mode == 2
                         ? moe::launch_combine_fwd_q8(a, ep_send_counts, workspace, cs)
                         : moe::launch_combine_fwd(a, cs));
}

moe_status moe_test_combine_fwd_comm_quant_wait_timeout(
    const moe_shape* s, const void* expand_x, const int32_t* topk_idx, const float* topk_weights,
    const int32_t* assist_info, const uint8_t* x_active_mask, const void* shared_expert_x,
    const void* ori_x, const void* const_alpha_1, const void* const_alpha_2, const void* const_v,
    void* out, uint64_t wait_limit_ns, int withhold_unit, void* stream) {
  moe::CombineArgs a;
  moe_status st = combine_args(s, expand_x, topk_idx, topk_weights, assist_info, x_active_mask,
                               shared_expert_x, ori_x, const_alpha_1, const_alpha_2, const_v,
                               out, &a);
  if (st != MOE_OK) return st;
  if (withhold_unit < 0 || wait_limit_ns == 0 || wait_limit_ns > moe::kWaitLimitNs)
    return MOE_ERR_ARG;
  if (s->bs == 0 || s->h > 16384) return MOE_ERR_UNSUPPORTED;
  bool launched = false;
  const moe::WaitCfg wc = {wait_limit_ns, withhold_unit};
  const cudaError_t err = moe::launch_combine_fwd_q8s_test(a, wc, static_cast<cudaStream_t>(stream),
                                                           &launched);
  if (!launched) return MOE_ERR_UNSUPPORTED;
  return cuda_status(err);
}

moe_status moe_test_dispatch_permute_smooth_wait_timeout(
    const moe_shape* s, const void* x, const int32_t* topk_idx, const int32_t* assist_info,
    const int32_t* ep_send_counts, const float* smooth_scales, void* expand_x,
    float* dynamic_scales, uint64_t wait_limit_ns, int withhold_unit, void* stream) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if (s->bs > 0 && (x == nullptr || topk_idx == nullptr || assist_info == nullptr ||
                    ep_send_counts == nullptr || smooth_scales == nullptr ||
                    expand_x == nullptr || dynamic_scales == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(expand_x) || !aligned16(smooth_scales)) return MOE_ERR_ALIGN;
  if (s->h % 16 != 0) return MOE_ERR_ALIGN;
  if (withhold_unit < 0 || wait_limit_ns == 0 || wait_limit_ns > moe::kWaitLimitNs)
    return MOE_ERR_ARG;
  if (s->bs == 0 || s->h > 16384) return MOE_ERR_UNSUPPORTED;
  moe::PermuteArgs a;
  a.x = x;
  a.assist = assist_info;
  a.expand_x = expand_x;
  a.scales = dynamic_scales;
  a.bs = s->bs;
  a.K = s->k;
  a.H = s->h;
  a.A = s->a_capacity;
  a.dtype = s->dtype;
  a.quant_mode = 2;
  const moe::WaitCfg wc = {wait_limit_ns, withhold_unit};
  const cudaError_t err = moe::launch_permute_smooth(a, topk_idx, smooth_scales, ep_send_counts,
                                                     s->num_experts,
                                                     static_cast<cudaStream_t>(stream), wc, true);
  if (err == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return cuda_status(err);
}

moe_status moe_combine_bwd(const moe_shape* s, const void* grad_out, const void* expand_x,
                           const int32_t* topk_idx, const float* topk_weights,
                           const int32_t* assist_info, const uint8_t* x_active_mask,
                           void* grad_expand, float* grad_w, void* stream) {
  return moe_combine_bwd_comm_quant(s, grad_out, expand_x, topk_idx, topk_weights, assist_info,
                                    x_active_mask, 0, grad_expand, grad_w, stream);
}

moe_status moe_combine_bwd_comm_quant(const moe_shape* s, const void* grad_out,
                                      const void* expand_x, const int32_t* topk_idx,
                                      const float* topk_weights, const int32_t* assist_info,
                                      const uint8_t* x_active_mask, int comm_quant_mode,
                                      void* grad_expand, float* grad_w, void* stream) {
  (void)topk_idx;
  if (comm_quant_mode != 0 && comm_quant_mode != 2) return MOE_ERR_ARG;
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if ((st = check_mask(s, x_active_mask)) != MOE_OK) return st;
  if (s->bs > 0 && (grad_out == nullptr || expand_x == nullptr || topk_weights == nullptr ||
                    assist_info == nullptr || grad_expand == nullptr || grad_w == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(grad_out) || !aligned16(expand_x) || !aligned16(grad_expand))
    return MOE_ERR_ALIGN;
  moe::CombineBwdArgs a;
  a.grad_out = grad_out;
  a.expand_x = expand_x;
  a.weights = topk_weights;
  a.assist = assist_info;
  a.mask = x_active_mask;
  a.mask_ndim = s->mask_ndim;
  a.grad_expand = grad_expand;
  a.grad_w = grad_w;
  a.bs = s->bs;
  a.K = s->k;
  a.H = s->h;
  a.A = s->a_capacity;
  a.dtype = s->dtype;
  a.quant_mode = comm_quant_mode;
  return cuda_status(moe::launch_combine_bwd(a, static_cast<cudaStream_t>(stream)));
}

size_t moe_combine_bwd_special_workspace_bytes(const moe_shape* s) {
  if (s == nullptr || check_shape(s) != MOE_OK) return 0;
  return moe::special_bwd_workspace_bytes(s->bs, s->h, s->const_expert_num);
}

moe_status moe_combine_bwd_special(const moe_shape* s, const void* grad_out,
                                   const int32_t* topk_idx, const float* topk_weights,
                                   const uint8_t* x_active_mask, const void* ori_x,
                                   const void* const_alpha_1, const void* const_alpha_2,
                                   const void* const_v, float* grad_w, void* grad_ori_x,
                                   float* grad_alpha_1, float* grad_alpha_2, float* grad_v,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if ((st = check_mask(s, x_active_mask)) != MOE_OK) return st;
  const bool consts = s->const_expert_num > 0;
  if (s->bs > 0 && (grad_out == nullptr || topk_idx == nullptr || topk_weights == nullptr ||
                    ori_x == nullptr || grad_w == nullptr || grad_ori_x == nullptr))
    return MOE_ERR_ARG;
  if (consts && (const_alpha_1 == nullptr || const_alpha_2 == nullptr || const_v == nullptr ||
                 grad_alpha_1 == nullptr || grad_alpha_2 == nullptr || grad_v == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(grad_out) || !aligned16(ori_x) || !aligned16(grad_ori_x) ||
      !aligned16(const_alpha_1) || !aligned16(const_alpha_2) || !aligned16(const_v))
    return MOE_ERR_ALIGN;
  const size_t need = moe::special_bwd_workspace_bytes(s->bs, s->h, s->const_expert_num);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return MOE_ERR_CAPACITY;
  if (need > 0 && !aligned16(workspace)) return MOE_ERR_ALIGN;
  return cuda_status(moe::launch_special_bwd(
      grad_out, topk_idx, topk_weights, x_active_mask, s->mask_ndim, ori_x, const_alpha_1,
      const_alpha_2, const_v, grad_w, grad_ori_x, grad_alpha_1, grad_alpha_2, grad_v, workspace,
      s->bs, s->k, s->h, s->num_experts, s->zero_expert_num, s->copy_expert_num,
      s->const_expert_num, s->dtype, static_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch_bwd(const moe_shape* s, const void* grad_expand_in,
                            const int32_t* assist_info, const uint8_t* x_active_mask,
                            void* grad_x, void* stream) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if ((st = check_mask(s, x_active_mask)) != MOE_OK) return st;
  if (s->bs > 0 && (grad_expand_in == nullptr || assist_info == nullptr || grad_x == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(grad_expand_in) || !aligned16(grad_x)) return MOE_ERR_ALIGN;
  moe::CombineArgs a = {};
  a.expand_x = grad_expand_in;
  a.weights = nullptr;  // unit weights
  a.assist = assist_info;
  a.mask = x_active_mask;
  a.mask_ndim = s->mask_ndim;
  a.out = grad_x;
  a.bs = s->bs;
  a.K = s->k;
  a.H = s->h;
  a.A = s->a_capacity;
  a.E = s->num_experts;
  a.dtype = s->dtype;
  return cuda_status(moe::launch_combine_fwd(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace moe {

moe_status report_cuda_error(cudaError_t err) { return cuda_status(err); }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace moe
