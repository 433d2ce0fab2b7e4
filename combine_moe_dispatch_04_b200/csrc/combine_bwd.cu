// Combine backward: the gradient of the combine Formula for routed pairs, and
// of the combine with comm_quant_mode 2. [combine] Function (Formula),
// Parameters (comm_quant_mode); the fused EP MoE layer of the
// Triton-distributed ep_moe_fused PR has a backward.
//
// One warp per (token, k) pair on a persistent grid; the warp streams the
// pair's expand_x row against grad_out[t] (the K warps of a token share
// grad_out[t] through L1), writes grad_expand = round16(w * grad_out) and
// reduces grad_w with eight per-element accumulators per lane and a fixed
// butterfly, so the result does not depend on scheduling.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kBwdUnroll = 4;

// Q8: the backward of the combine with comm_quant_mode 2 (straight-through):
// grad_w takes the dot of grad_out with the row's int8 round-trip values
// fl(q * scale), scale = fl(max|y| / 127), the codes decided exactly as in
// the forward; grad_expand is unchanged. The row is read twice through L1:
// once for its max, once for the dot (holding it in registers instead was
// slower: 121 registers, half the warps).
template <typename T16, bool Q8>
__device__ __forceinline__ void combine_bwd_pair(const CombineBwdArgs& a, int pair, int lane) {
  const int t = pair / a.K;
  const int k = pair - t * a.K;
  const int s = __ldg(a.assist + static_cast<size_t>(a.A) + pair);
  if (s < 0 || !pair_active(a.mask, a.mask_ndim, t, k, a.K)) {
    if (lane == 0) a.grad_w[pair] = 0.0f;
    return;
  }
  const int V = a.H / kVecElems;
  const float w = __ldg(a.weights + pair);
  const uint4* g = static_cast<const uint4*>(a.grad_out) + static_cast<size_t>(t) * V;
  const uint4* y = static_cast<const uint4*>(a.expand_x) + static_cast<size_t>(s) * V;
  uint4* ge = static_cast<uint4*>(a.grad_expand) + static_cast<size_t>(s) * V;
  float mx = 0.0f, scale = 0.0f, inv = 0.0f;
  if (Q8) {
    uint32_t m2 = 0;
#pragma unroll 4
    for (int v = lane; v < V; v += 32) m2 = absmax_v4<T16>(m2, __ldg(y + v));
    mx = absmax_final<T16>(m2);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    scale = __fdiv_rn(mx, 127.0f);
    inv = 1.0f / scale;
  }
  float d[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i] = 0.0f;
  for (int v0 = lane; v0 < V; v0 += 32 * kBwdUnroll) {
    uint4 gv[kBwdUnroll], yv[kBwdUnroll];
#pragma unroll
    for (int u = 0; u < kBwdUnroll; ++u) {
      const int v = v0 + u * 32;
      if (v < V) {
        gv[u] = __ldg(g + v);  // kept in L1: the other K-1 warps of the token re-read it
        yv[u] = Q8 ? __ldg(y + v) : ld_nc_v4(y + v);
      }
    }
#pragma unroll
    for (int u = 0; u < kBwdUnroll; ++u) {
      const int v = v0 + u * 32;
      if (v >= V) continue;
      float gf[8], yf[8], o[8];
      widen8<T16>(gv[u], gf);
      if (Q8) {
        float yr[8];
        widen8<T16>(yv[u], yr);
        quant_roundtrip8<true>(yr, mx, scale, inv, yf);
      } else {
        widen8<T16>(yv[u], yf);
      }
      const float2 ww = f2(w, w);
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float2 g2 = f2(gf[i], gf[i + 1]);
        const float2 dd = __ffma2_rn(g2, f2(yf[i], yf[i + 1]), f2(d[i], d[i + 1]));
        d[i] = dd.x;
        d[i + 1] = dd.y;
        const float2 oo = __fmul2_rn(ww, g2);
        o[i] = oo.x;
        o[i + 1] = oo.y;
      }
      st_v4(ge + v, narrow8<T16>(o));
    }
  }
  float dot = ((d[0] + d[1]) + (d[2] + d[3])) + ((d[4] + d[5]) + (d[6] + d[7]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
  if (lane == 0) a.grad_w[pair] = dot;
}

template <typename T16, bool Q8>
__global__ void __launch_bounds__(kBwdThreads) combine_bwd_kernel(CombineBwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int n_pairs = a.bs * a.K;
  const int stride = gridDim.x * kBwdWarps;
  for (int pair = blockIdx.x * kBwdWarps + (threadIdx.x >> 5); pair < n_pairs; pair += stride)
    combine_bwd_pair<T16, Q8>(a, pair, lane);
}

template <typename T16, bool Q8>
cudaError_t launch_bwd(const CombineBwdArgs& a, cudaStream_t st) {
  constexpr auto kernel = combine_bwd_kernel<T16, Q8>;
  const long long pairs = static_cast<long long>(a.bs) * a.K;
  const long long want = (pairs + kBwdWarps - 1) / kBwdWarps;
  const long long cap = static_cast<long long>(sm_count()) * blocks_per_sm<kernel>(kBwdThreads, 0);
  const int blocks = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(kernel, dim3(blocks), dim3(kBwdThreads), 0, st, a);
}

}  // namespace

cudaError_t launch_combine_bwd(const CombineBwdArgs& a, cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  if (a.quant_mode == 2)
    return a.dtype == MOE_BF16 ? launch_bwd<Bf16, true>(a, st) : launch_bwd<Fp16, true>(a, st);
  return a.dtype == MOE_BF16 ? launch_bwd<Bf16, false>(a, st) : launch_bwd<Fp16, false>(a, st);
}

}  // namespace moe
