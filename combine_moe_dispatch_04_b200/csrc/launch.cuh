// Internal launch interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "async.cuh"
#include "moe_dc.h"

namespace moe {

struct LayoutArgs {
  const int32_t* topk_idx;
  const uint8_t* mask;
  int mask_ndim;
  int bs, K, E, N, A;
  int32_t* expert_token_nums;
  int32_t* ep_send_counts;
  int32_t* assist;
  uint32_t* dev_status;  // may be null
  void* workspace;
  size_t workspace_bytes;
};

// Tokens per CTA in the multi-CTA layout, and the largest BS of the one-CTA layout.
constexpr int kLayoutTileTokens = 256;
constexpr int kLayoutSmallMaxTokens = 1024;

size_t layout_workspace_bytes(int bs, int E, int K);
cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t st);

struct PermuteArgs {
  const void* x;
  const int32_t* assist;
  void* expand_x;
  float* scales;
  int bs, K, H, A, dtype, quant_mode;
};
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st);
// int8 permute of x[t] * smooth[e] per slot (H <= 16384, multiple of 16; smooth 16-byte
// aligned); reads the total R from send[E].
cudaError_t launch_permute_smooth(const PermuteArgs& a, const int32_t* topk_idx,
                                  const float* smooth, const int32_t* send, int E,
                                  cudaStream_t st, const WaitCfg& wc = kProductWaits,
                                  bool staged_only = false);

// Layout and the plain (no quantisation) permute in one launch, BS <= kLayoutSmallMaxTokens
// and shared memory for E experts' masks (dispatch_small_fits).
bool dispatch_small_fits(int E, int K);
cudaError_t launch_dispatch_small(const LayoutArgs& a, const void* x, void* expand_x, int H,
                                  cudaStream_t st);

struct CombineArgs {
  const void* expand_x;  // (A, H): expert outputs, or slot gradients for dispatch bwd
  const int32_t* topk_idx;
  const float* weights;  // null: unit weights (dispatch backward)
  const int32_t* assist;
  const uint8_t* mask;
  int mask_ndim;
  const void* shared;
  const void* ori_x;
  const void* alpha1;
  const void* alpha2;
  const void* const_v;
  void* out;
  int bs, K, H, A, E, Z, C, Q, dtype;
};
cudaError_t launch_combine_fwd(const CombineArgs& a, cudaStream_t st);
// comm_quant_mode 2: every routed row through the per-row int8 round trip (H <= 16384).
// With a workspace of combine_q8_workspace_bytes(A) bytes and the total R in send[E], shapes
// with routed pairs only take two passes (per-row scales, then the gather); otherwise the
// staged kernel runs and the workspace is not touched.
size_t combine_q8_workspace_bytes(int A);
// The staged single-pass int8 combine with the given waits (test hook); *launched is
// false when the shape takes another kernel.
cudaError_t launch_combine_fwd_q8s_test(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st,
                                        bool* launched);
cudaError_t launch_combine_fwd_q8(const CombineArgs& a, const int32_t* send, void* workspace,
                                  cudaStream_t st);

struct CombineBwdArgs {
  const void* grad_out;
  const void* expand_x;
  const float* weights;
  const int32_t* assist;
  const uint8_t* mask;
  int mask_ndim;
  void* grad_expand;
  float* grad_w;
  int bs, K, H, A, dtype;
  int quant_mode;  // 0, or 2: the backward of the int8 round-trip combine
};
cudaError_t launch_combine_bwd(const CombineBwdArgs& a, cudaStream_t st);

size_t special_bwd_workspace_bytes(int bs, int H, int Q);
cudaError_t launch_special_bwd(const void* grad_out, const int32_t* topk_idx,
                               const float* weights, const uint8_t* mask, int mask_ndim,
                               const void* ori_x, const void* alpha1, const void* alpha2,
                               const void* const_v, float* grad_w, void* grad_ori_x,
                               float* grad_alpha1, float* grad_alpha2, float* grad_v,
                               void* workspace, int bs, int K, int H, int E, int Z, int C, int Q,
                               int dtype, cudaStream_t st);

int sm_count();

// Device address of the counter of CTAs that gave up a bounded wait on an
// asynchronous copy (this device's; null if it cannot be had).
unsigned* wait_timeout_counter();

// Records err as the thread's last CUDA error; returns MOE_ERR_CUDA (MOE_OK for success).
moe_status report_cuda_error(cudaError_t err);

}  // namespace moe
