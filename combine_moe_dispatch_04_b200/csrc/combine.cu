// Combine forward, dispatch backward (the same gather with unit weights) and
// combine backward. [combine] Function (Formula; special expert use cases),
// Parameters, Return Value.
//
// Forward: one thread per 16-byte vector (8 values) of an output row (or a
// few vectors when K is small), in one-shot blocks. The thread issues the
// loads of all of its token's K slot rows first, then accumulates in fp32 in
// ascending k with every product and every sum rounded on its own
// (__fmul_rn / __fadd_rn: never contracted into an FMA), adds shared_expert_x
// once, and narrows with round-to-nearest-even.
//
// Backward: one warp per (token, k) pair on a persistent grid; the warp
// streams the pair's expand_x row against grad_out[t] (the K warps of a token
// share grad_out[t] through L1), writes grad_expand = round16(w * grad_out)
// and reduces grad_w with eight per-element accumulators per lane and a fixed
// butterfly, so the result does not depend on scheduling.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kFwdThreads = 256;

enum PairKind : int { kSkip = 0, kRouted = 1, kZero = 2, kCopy = 3, kConst = 4 };

// The 8 values m of one pair for one vector: the routed row, 0, ori_x, or
// alpha_1 * ori_x + alpha_2 * v (each product and the sum rounded on its own).
template <typename T16, bool SPECIAL>
__device__ __forceinline__ void pair_values(const CombineArgs& a, int kind, int row, int V, int v,
                                            const uint4& val, const float (&ori)[8],
                                            float (&m)[8]) {
  if (!SPECIAL || kind == kRouted) {
    widen8<T16>(val, m);
  } else if (kind == kZero) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = 0.0f;
  } else if (kind == kCopy) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = ori[i];
  } else {
    const size_t r = static_cast<size_t>(row) * V + v;
    float a1[8], a2[8], cv[8];
    widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha1) + r), a1);
    widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha2) + r), a2);
    widen8<T16>(__ldg(static_cast<const uint4*>(a.const_v) + r), cv);
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = __fadd_rn(__fmul_rn(a1[i], ori[i]), __fmul_rn(a2[i], cv[i]));
  }
}

// Vectors per thread: enough that every thread keeps eight 16-byte row loads
// in flight when K is small.
template <int KMAX>
__host__ __device__ constexpr int fwd_vectors_per_thread() {
  return KMAX >= 8 ? 1 : 8 / KMAX;
}

// One thread per U output vectors (8 values each) spaced a block apart, so a
// warp's loads stay coalesced along the rows. For each vector the thread
// classifies its token's K pairs, issues the loads of all routed rows, then
// accumulates in ascending k.
template <typename T16, int KMAX, bool SPECIAL, bool UNIT>
__global__ void __launch_bounds__(kFwdThreads) combine_fwd_kernel(CombineArgs a) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int n = a.bs * V;
  const int n_ids = a.E + a.Z + a.C + a.Q;
  const uint4* Y = static_cast<const uint4*>(a.expand_x);
  const int base = blockIdx.x * (kFwdThreads * U) + threadIdx.x;
  uint4 val[U][KMAX];
  int kind[U][KMAX], row[U][KMAX];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int item = base + u * kFwdThreads;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) kind[u][j] = kSkip;
    if (item >= n) continue;
    const int t = item / V;
    const int v = item - t * V;
    const int32_t* slots = a.assist + static_cast<size_t>(a.A) + static_cast<size_t>(t) * K;
    int ids[KMAX];
    if (SPECIAL) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        ids[j] = j < K ? __ldg(a.topk_idx + static_cast<size_t>(t) * K + j) : -1;
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= K || !pair_active(a.mask, a.mask_ndim, t, j, K)) continue;
      int kd = kRouted, r = 0;
      if (SPECIAL) {
        const int id = ids[j];
        bool dup = false;
#pragma unroll
        for (int jj = 0; jj < j; ++jj) dup |= ids[jj] == id;
        if (dup || id < 0 || id >= n_ids) continue;
        if (id >= a.E) {
          kd = id < a.E + a.Z ? kZero : id < a.E + a.Z + a.C ? kCopy : kConst;
          r = id - (a.E + a.Z + a.C);
        }
      }
      if (kd == kRouted) {
        const int s = __ldg(slots + j);
        if (s < 0) continue;
        val[u][j] = ld_nc_v4(Y + static_cast<size_t>(s) * V + v);
      }
      kind[u][j] = kd;
      row[u][j] = r;
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int item = base + u * kFwdThreads;
    if (item >= n) continue;
    const int t = item / V;
    const int v = item - t * V;
    float ori[8];
    if (SPECIAL) {
      bool need = false;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) need |= kind[u][j] == kCopy || kind[u][j] == kConst;
      if (need) widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.ori_x) + item), ori);
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (kind[u][j] == kSkip) continue;
      float m[8];
      pair_values<T16, SPECIAL>(a, kind[u][j], row[u][j], V, v, val[u][j], ori, m);
      if (UNIT) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], m[i]);
      } else {
        const float w = __ldg(a.weights + static_cast<size_t>(t) * K + j);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(w, m[i]));
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
}

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kBwdUnroll = 4;

template <typename T16>
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

template <typename T16>
__global__ void __launch_bounds__(kBwdThreads) combine_bwd_kernel(CombineBwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int n_pairs = a.bs * a.K;
  const int stride = gridDim.x * kBwdWarps;
  for (int pair = blockIdx.x * kBwdWarps + (threadIdx.x >> 5); pair < n_pairs; pair += stride)
    combine_bwd_pair<T16>(a, pair, lane);
}

// Resident blocks per SM of a kernel (occupancy API), cached per kernel.
template <auto Kernel>
int blocks_per_sm(int threads, size_t smem) {
  static int cached = 0;
  if (cached == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, threads, smem) != cudaSuccess ||
        n < 1)
      n = 1;
    cached = n;
  }
  return cached;
}

template <typename T16, int KMAX, bool SPECIAL, bool UNIT>
cudaError_t launch_fwd_kmax(const CombineArgs& a, cudaStream_t st) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
  const long long n = static_cast<long long>(a.bs) * (a.H / kVecElems);
  const int blocks = static_cast<int>((n + kFwdThreads * U - 1) / (kFwdThreads * U));
  return launch_pdl(combine_fwd_kernel<T16, KMAX, SPECIAL, UNIT>, dim3(blocks), dim3(kFwdThreads),
                    0, st, a);
}

template <typename T16, bool SPECIAL, bool UNIT>
cudaError_t launch_fwd_k(const CombineArgs& a, cudaStream_t st) {
  if (a.K <= 2) return launch_fwd_kmax<T16, 2, SPECIAL, UNIT>(a, st);
  if (a.K <= 4) return launch_fwd_kmax<T16, 4, SPECIAL, UNIT>(a, st);
  if (a.K <= 8) return launch_fwd_kmax<T16, 8, SPECIAL, UNIT>(a, st);
  return launch_fwd_kmax<T16, 16, SPECIAL, UNIT>(a, st);
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
  auto kernel = a.dtype == MOE_BF16 ? combine_bwd_kernel<Bf16> : combine_bwd_kernel<Fp16>;
  const long long pairs = static_cast<long long>(a.bs) * a.K;
  const long long want = (pairs + kBwdWarps - 1) / kBwdWarps;
  const long long cap = static_cast<long long>(sm_count()) *
                        (a.dtype == MOE_BF16 ? blocks_per_sm<combine_bwd_kernel<Bf16>>(kBwdThreads, 0)
                                             : blocks_per_sm<combine_bwd_kernel<Fp16>>(kBwdThreads, 0));
  const int blocks = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(kernel, dim3(blocks), dim3(kBwdThreads), 0, st, a);
}

}  // namespace moe
