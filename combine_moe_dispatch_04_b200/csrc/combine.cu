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
constexpr int kFwdWarps = kFwdThreads / 32;

enum PairKind : int { kSkip = 0, kRouted = 1, kZero = 2, kCopy = 3, kConst = 4 };

// Metadata of pair (t, lane) held by lane k < K of the warp.
struct PairMeta {
  int kind;
  int slot;  // routed: expand_x row; const: row of alpha_1/alpha_2/v
  float w;
};

template <bool SPECIAL, bool UNIT>
__device__ __forceinline__ PairMeta load_meta(const CombineArgs& a, int t, int lane) {
  PairMeta m{kSkip, -1, 1.0f};
  const int K = a.K;
  int id = -1;
  if (lane < K) {
    const size_t tk = static_cast<size_t>(t) * K + lane;
    const bool act = pair_active(a.mask, a.mask_ndim, t, lane, K);
    const int s = __ldg(a.assist + static_cast<size_t>(a.A) + tk);
    if (!UNIT) m.w = __ldg(a.weights + tk);
    if (!SPECIAL) {
      if (act && s >= 0) {
        m.kind = kRouted;
        m.slot = s;
      }
    } else {
      id = __ldg(a.topk_idx + tk);
      const int n_ids = a.E + a.Z + a.C + a.Q;
      if (act && id >= 0 && id < n_ids) {
        if (id < a.E) {
          if (s >= 0) {
            m.kind = kRouted;
            m.slot = s;
          }
        } else if (id < a.E + a.Z) {
          m.kind = kZero;
        } else if (id < a.E + a.Z + a.C) {
          m.kind = kCopy;
        } else {
          m.kind = kConst;
          m.slot = id - (a.E + a.Z + a.C);
        }
      }
    }
  }
  if (SPECIAL) {  // a repeat of an earlier id in the row takes no part
    bool dup = false;
    for (int j = 0; j < K; ++j) {
      const int idj = __shfl_sync(0xFFFFFFFFu, id, j);
      dup |= j < lane && idj == id;
    }
    if (dup) m.kind = kSkip;
  }
  return m;
}

// The 8 values m of pair j for one vector: the routed row, 0, ori_x, or
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

// One warp per (token, chunk of 32 * U vectors) item, items strided over a
// persistent grid. Lane k < K holds pair k's metadata (broadcast by shuffle);
// every lane owns U vectors of the chunk and issues the loads of all K rows
// before accumulating, so K * U 16-byte loads are in flight per lane. The next
// item's metadata is fetched while the current rows are in flight.
template <typename T16, int KMAX, bool SPECIAL, bool UNIT>
__global__ void __launch_bounds__(kFwdThreads) combine_fwd_kernel(CombineArgs a, int chunks,
                                                                  int n_items) {
  constexpr int U = KMAX <= 4 ? 2 : 1;
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int lane = threadIdx.x & 31;
  const int stride = gridDim.x * kFwdWarps;
  const uint4* Y = static_cast<const uint4*>(a.expand_x);
  int item = blockIdx.x * kFwdWarps + (threadIdx.x >> 5);
  PairMeta meta;
  if (item < n_items) meta = load_meta<SPECIAL, UNIT>(a, item / chunks, lane);
  for (; item < n_items; item += stride) {
    const int t = item / chunks;
    const int v0 = (item - t * chunks) * 32 * U + lane;
    uint4 val[KMAX][U];
    int kind[KMAX], row[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      kind[j] = __shfl_sync(0xFFFFFFFFu, meta.kind, j);
      row[j] = __shfl_sync(0xFFFFFFFFu, meta.slot, j);
      if (j >= K) kind[j] = kSkip;
      if (kind[j] == kRouted) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * 32;
          if (v < V) val[j][u] = ld_nc_v4(Y + static_cast<size_t>(row[j]) * V + v);
        }
      }
    }
    float ori[U][8];
    if (SPECIAL) {
      bool need = false;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) need |= kind[j] == kCopy || kind[j] == kConst;
      if (need) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * 32;
          if (v < V)
            widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.ori_x) + static_cast<size_t>(t) * V + v),
                        ori[u]);
        }
      }
    }
    const float w_lane = meta.w;
    if (item + stride < n_items) meta = load_meta<SPECIAL, UNIT>(a, (item + stride) / chunks, lane);
    float acc[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const float w = UNIT ? 1.0f : __shfl_sync(0xFFFFFFFFu, w_lane, j);
      if (kind[j] == kSkip) continue;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * 32;
        if (v >= V) continue;
        float m[8];
        pair_values<T16, SPECIAL>(a, kind[j], row[j], V, v, val[j][u], ori[u], m);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          acc[u][i] = UNIT ? __fadd_rn(acc[u][i], m[i]) : __fadd_rn(acc[u][i], __fmul_rn(w, m[i]));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * 32;
      if (v >= V) continue;
      const size_t o = static_cast<size_t>(t) * V + v;
      if (!UNIT && a.shared != nullptr) {
        float sh[8];
        widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.shared) + o), sh);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = __fadd_rn(acc[u][i], sh[i]);
      }
      st_v4(static_cast<uint4*>(a.out) + o, narrow8<T16>(acc[u]));
    }
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
  constexpr int U = KMAX <= 4 ? 2 : 1;
  constexpr auto kernel = combine_fwd_kernel<T16, KMAX, SPECIAL, UNIT>;
  const int V = a.H / kVecElems;
  const int chunks = (V + 32 * U - 1) / (32 * U);
  const long long items = static_cast<long long>(a.bs) * chunks;
  const long long want = (items + kFwdWarps - 1) / kFwdWarps;
  const long long cap = static_cast<long long>(sm_count()) * blocks_per_sm<kernel>(kFwdThreads, 0);
  const int blocks = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(kernel, dim3(blocks), dim3(kFwdThreads), 0, st, a, chunks,
                    static_cast<int>(items));
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
