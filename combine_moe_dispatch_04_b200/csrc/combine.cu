// Combine forward, dispatch backward (the same gather with unit weights) and
// combine backward. [combine] Function (Formula; special expert use cases),
// Parameters, Return Value.
//
// Forward: one thread per 16-byte vector (8 values) of an output row. The
// thread issues the loads of all of its token's K slot rows first, then
// accumulates in fp32 in ascending k with every product and every sum rounded
// on its own (__fmul_rn / __fadd_rn: never contracted into an FMA), adds
// shared_expert_x once, and narrows with round-to-nearest-even.
//
// Backward: one warp per (token, k) pair; the warp streams the pair's
// expand_x row against grad_out[t] (the K warps of a token share grad_out[t]
// through L1), writes grad_expand = round16(w * grad_out) and reduces grad_w
// with eight per-element accumulators per lane and a fixed butterfly, so the
// result does not depend on scheduling.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kFwdThreads = 256;

enum PairKind : int { kSkip = 0, kRouted = 1, kZero = 2, kCopy = 3, kConst = 4 };

template <typename T16, int KMAX, bool SPECIAL, bool UNIT>
__global__ void __launch_bounds__(kFwdThreads) combine_fwd_kernel(CombineArgs a) {
  const int V = a.H / kVecElems;
  const int item = blockIdx.x * kFwdThreads + threadIdx.x;
  if (item >= a.bs * V) return;
  const int t = item / V;
  const int v = item - t * V;
  const int K = a.K;
  const uint4* Y = static_cast<const uint4*>(a.expand_x);
  const int32_t* slots = a.assist + static_cast<size_t>(a.A) + static_cast<size_t>(t) * K;
  const int32_t* ids = SPECIAL ? a.topk_idx + static_cast<size_t>(t) * K : nullptr;
  const int n_ids = a.E + a.Z + a.C + a.Q;

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;

  for (int k0 = 0; k0 < K; k0 += KMAX) {
    uint4 val[KMAX];
    int kind[KMAX];
    bool need_ori = false;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const int k = k0 + j;
      kind[j] = kSkip;
      if (k >= K) continue;
      if (!pair_active(a.mask, a.mask_ndim, t, k, K)) continue;
      if (!SPECIAL) {
        const int s = __ldg(slots + k);
        if (s >= 0) {
          val[j] = ld_nc_v4(Y + static_cast<size_t>(s) * V + v);
          kind[j] = kRouted;
        }
        continue;
      }
      const int id = __ldg(ids + k);
      if (id < 0 || id >= n_ids) continue;
      bool dup = false;
      for (int jj = 0; jj < k; ++jj) dup |= __ldg(ids + jj) == id;
      if (dup) continue;
      if (id < a.E) {
        const int s = __ldg(slots + k);
        if (s >= 0) {
          val[j] = ld_nc_v4(Y + static_cast<size_t>(s) * V + v);
          kind[j] = kRouted;
        }
      } else if (id < a.E + a.Z) {
        kind[j] = kZero;
      } else if (id < a.E + a.Z + a.C) {
        kind[j] = kCopy;
        need_ori = true;
      } else {
        const size_t q = static_cast<size_t>(id - (a.E + a.Z + a.C));
        // alpha_1[q], alpha_2[q], v[q] are combined below; stash row q here.
        val[j] = make_uint4(static_cast<uint32_t>(q), 0u, 0u, 0u);
        kind[j] = kConst;
        need_ori = true;
      }
    }
    float ori[8];
    if (SPECIAL && need_ori) {
      widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.ori_x) + item), ori);
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (kind[j] == kSkip) continue;
      float m[8];
      if (!SPECIAL || kind[j] == kRouted) {
        widen8<T16>(val[j], m);
      } else if (kind[j] == kZero) {
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = 0.0f;
      } else if (kind[j] == kCopy) {
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = ori[i];
      } else {
        const size_t row = static_cast<size_t>(val[j].x) * V + v;
        float a1[8], a2[8], cv[8];
        widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha1) + row), a1);
        widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha2) + row), a2);
        widen8<T16>(__ldg(static_cast<const uint4*>(a.const_v) + row), cv);
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = __fadd_rn(__fmul_rn(a1[i], ori[i]), __fmul_rn(a2[i], cv[i]));
      }
      if (UNIT) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], m[i]);
      } else {
        const float w = __ldg(a.weights + static_cast<size_t>(t) * K + k0 + j);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(w, m[i]));
      }
    }
  }
  if (!UNIT && a.shared != nullptr) {
    float sh[8];
    widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.shared) + item), sh);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], sh[i]);
  }
  st_v4(static_cast<uint4*>(a.out) + item, narrow8<T16>(acc));
}

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kBwdUnroll = 4;

template <typename T16>
__global__ void __launch_bounds__(kBwdThreads) combine_bwd_kernel(CombineBwdArgs a) {
  const int pair = blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (pair >= a.bs * a.K) return;
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
        yv[u] = ld_nc_v4(y + v);
      }
    }
#pragma unroll
    for (int u = 0; u < kBwdUnroll; ++u) {
      const int v = v0 + u * 32;
      if (v >= V) continue;
      float gf[8], yf[8], o[8];
      widen8<T16>(gv[u], gf);
      widen8<T16>(yv[u], yf);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        d[i] = __fmaf_rn(gf[i], yf[i], d[i]);
        o[i] = __fmul_rn(w, gf[i]);
      }
      st_v4(ge + v, narrow8<T16>(o));
    }
  }
  float dot = ((d[0] + d[1]) + (d[2] + d[3])) + ((d[4] + d[5]) + (d[6] + d[7]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
  if (lane == 0) a.grad_w[pair] = dot;
}

template <typename T16, bool SPECIAL, bool UNIT>
cudaError_t launch_fwd_k(const CombineArgs& a, cudaStream_t st) {
  const long long n = static_cast<long long>(a.bs) * (a.H / kVecElems);
  const int blocks = static_cast<int>((n + kFwdThreads - 1) / kFwdThreads);
  if (a.K <= 2)
    combine_fwd_kernel<T16, 2, SPECIAL, UNIT><<<blocks, kFwdThreads, 0, st>>>(a);
  else if (a.K <= 4)
    combine_fwd_kernel<T16, 4, SPECIAL, UNIT><<<blocks, kFwdThreads, 0, st>>>(a);
  else if (a.K <= 8)
    combine_fwd_kernel<T16, 8, SPECIAL, UNIT><<<blocks, kFwdThreads, 0, st>>>(a);
  else
    combine_fwd_kernel<T16, 16, SPECIAL, UNIT><<<blocks, kFwdThreads, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T16>
cudaError_t launch_fwd_t(const CombineArgs& a, cudaStream_t st) {
  if (a.weights == nullptr) return launch_fwd_k<T16, false, true>(a, st);
  if (a.Z + a.C + a.Q > 0) return launch_fwd_k<T16, true, false>(a, st);
  return launch_fwd_k<T16, false, false>(a, st);
}

}  // namespace

cudaError_t launch_combine_fwd(const CombineArgs& a, cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  return a.dtype == MOE_BF16 ? launch_fwd_t<Bf16>(a, st) : launch_fwd_t<Fp16>(a, st);
}

cudaError_t launch_combine_bwd(const CombineBwdArgs& a, cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  const long long pairs = static_cast<long long>(a.bs) * a.K;
  const int blocks = static_cast<int>((pairs + kBwdWarps - 1) / kBwdWarps);
  if (a.dtype == MOE_BF16)
    combine_bwd_kernel<Bf16><<<blocks, kBwdThreads, 0, st>>>(a);
  else
    combine_bwd_kernel<Fp16><<<blocks, kBwdThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
