// Backward of the copy and const experts. [combine] Function (special expert
// use cases: copy Moe(ori_x) = ori_x, const Moe(ori_x) = alpha_1 ori_x +
// alpha_2 v) differentiated through the weighted sum of the Formula.
//
//   grad_w[t,k]      = <g[t], M(t,k)>, M = ori_x[t] or fl(fl(a1 x) + fl(a2 v))
//   grad_ori_x[t]    = round16( sum_{copy/const k, ascending} c  or  fl(c a1[j]) ),
//                      c = fl(w[t,k] g[t])
//   S[j]             = sum_{pairs of const j} c,   grad_alpha1[j] = sum c ori_x[t]
//   grad_alpha2[j]   = fl(S[j] v[j]),   grad_v[j] = fl(S[j] alpha2[j])
//
// Four launches: warp-per-pair dots (fixed butterfly), thread-per-vector
// grad_ori_x, per-(token chunk, const expert) partial sums into the workspace,
// and one fixed-order sum over the chunks. Every result is deterministic.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kChunkTokens = 256;  // tokens per partial sum of the alpha / v gradients

struct SpecialBwdArgs {
  const void* grad_out;
  const int32_t* topk_idx;
  const float* weights;
  const uint8_t* mask;
  int mask_ndim;
  const void* ori_x;
  const void* alpha1;
  const void* alpha2;
  const void* const_v;
  float* grad_w;
  void* grad_ori_x;
  float* grad_alpha1;
  float* grad_alpha2;
  float* grad_v;
  float* partials;  // [chunks][2][Q][H]: sum c * ori_x, sum c
  int bs, K, H, E, Z, C, Q;
};

// Kind of pair (t, k): 0 none (routed, zero, masked, invalid), 1 copy, 2 const
// (row q of the const tensors in *q).
__device__ __forceinline__ int special_kind(const SpecialBwdArgs& a, int t, int k, int* q) {
  const int32_t* ids = a.topk_idx + static_cast<size_t>(t) * a.K;
  const int id = __ldg(ids + k);
  const int lo = a.E + a.Z;
  if (id < lo || id >= lo + a.C + a.Q) return 0;
  for (int j = 0; j < k; ++j)
    if (__ldg(ids + j) == id) return 0;
  if (!pair_active(a.mask, a.mask_ndim, t, k, a.K)) return 0;
  if (id < lo + a.C) return 1;
  *q = id - lo - a.C;
  return 2;
}

template <typename T16>
__device__ __forceinline__ void const_m(const SpecialBwdArgs& a, int q, int V, int v,
                                        const float (&x)[8], float (&m)[8]) {
  const size_t r = static_cast<size_t>(q) * V + v;
  float a1[8], a2[8], cv[8];
  widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha1) + r), a1);
  widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha2) + r), a2);
  widen8<T16>(__ldg(static_cast<const uint4*>(a.const_v) + r), cv);
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = __fadd_rn(__fmul_rn(a1[i], x[i]), __fmul_rn(a2[i], cv[i]));
}

// grad_w of copy/const pairs: one warp per (token, k), persistent grid.
template <typename T16>
__global__ void __launch_bounds__(kThreads) special_dot_kernel(SpecialBwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int V = a.H / kVecElems;
  const int n_pairs = a.bs * a.K;
  for (int pair = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); pair < n_pairs;
       pair += gridDim.x * (kThreads / 32)) {
    const int t = pair / a.K, k = pair - t * a.K;
    int q = 0;
    const int kind = special_kind(a, t, k, &q);  // warp-uniform
    if (kind == 0) continue;
    const uint4* g = static_cast<const uint4*>(a.grad_out) + static_cast<size_t>(t) * V;
    const uint4* x = static_cast<const uint4*>(a.ori_x) + static_cast<size_t>(t) * V;
    float d[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = 0.0f;
    for (int v = lane; v < V; v += 32) {
      float gf[8], xf[8], m[8];
      widen8<T16>(__ldg(g + v), gf);
      widen8<T16>(__ldg(x + v), xf);
      if (kind == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = xf[i];
      } else {
        const_m<T16>(a, q, V, v, xf, m);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = __fmaf_rn(gf[i], m[i], d[i]);
    }
    float dot = ((d[0] + d[1]) + (d[2] + d[3])) + ((d[4] + d[5]) + (d[6] + d[7]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
    if (lane == 0) a.grad_w[pair] = dot;
  }
}

// grad_ori_x: one thread per 16-byte vector of (BS, H).
template <typename T16>
__global__ void __launch_bounds__(kThreads) special_ori_kernel(SpecialBwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int item = blockIdx.x * kThreads + threadIdx.x;
  if (item >= a.bs * V) return;
  const int t = item / V, v = item - t * V;
  float gf[8], acc[8];
  widen8<T16>(__ldg(static_cast<const uint4*>(a.grad_out) + item), gf);
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  for (int k = 0; k < a.K; ++k) {
    int q = 0;
    const int kind = special_kind(a, t, k, &q);
    if (kind == 0) continue;
    const float w = __ldg(a.weights + static_cast<size_t>(t) * a.K + k);
    float a1[8];
    if (kind == 2)
      widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha1) + static_cast<size_t>(q) * V + v), a1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float c = __fmul_rn(w, gf[i]);
      acc[i] = __fadd_rn(acc[i], kind == 1 ? c : __fmul_rn(c, a1[i]));
    }
  }
  st_v4(static_cast<uint4*>(a.grad_ori_x) + item, narrow8<T16>(acc));
}

// Partial sums over one chunk of tokens for one const expert q: thread per
// 16-byte vector of the row, tokens in ascending order.
template <typename T16>
__global__ void __launch_bounds__(kThreads) special_partial_kernel(SpecialBwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int chunk = blockIdx.x, q = blockIdx.y;
  const int v = blockIdx.z * kThreads + threadIdx.x;
  if (v >= V) return;
  float s1[8], sc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s1[i] = sc[i] = 0.0f;
  const int t1 = min(a.bs, (chunk + 1) * kChunkTokens);
  for (int t = chunk * kChunkTokens; t < t1; ++t) {
    for (int k = 0; k < a.K; ++k) {
      int qq = -1;
      if (special_kind(a, t, k, &qq) != 2 || qq != q) continue;
      const float w = __ldg(a.weights + static_cast<size_t>(t) * a.K + k);
      float gf[8], xf[8];
      widen8<T16>(__ldg(static_cast<const uint4*>(a.grad_out) + static_cast<size_t>(t) * V + v),
                  gf);
      widen8<T16>(__ldg(static_cast<const uint4*>(a.ori_x) + static_cast<size_t>(t) * V + v), xf);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float c = __fmul_rn(w, gf[i]);
        s1[i] = __fmaf_rn(c, xf[i], s1[i]);
        sc[i] = __fadd_rn(sc[i], c);
      }
    }
  }
  const size_t qh = static_cast<size_t>(a.Q) * a.H;
  float* p1 = a.partials + static_cast<size_t>(chunk) * 2 * qh + static_cast<size_t>(q) * a.H;
  float* pc = p1 + qh;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    p1[v * 8 + i] = s1[i];
    pc[v * 8 + i] = sc[i];
  }
}

// Sum of the partials over the chunks, in chunk order: grad_alpha1, and the
// alpha_2 / v gradients from S.
template <typename T16>
__global__ void __launch_bounds__(kThreads) special_final_kernel(SpecialBwdArgs a, int chunks) {
  pdl_trigger();
  pdl_wait();
  const size_t qh = static_cast<size_t>(a.Q) * a.H;
  const size_t i = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (i >= qh) return;
  float s1 = 0.0f, sc = 0.0f;
  for (int c = 0; c < chunks; ++c) {
    s1 = __fadd_rn(s1, a.partials[static_cast<size_t>(c) * 2 * qh + i]);
    sc = __fadd_rn(sc, a.partials[static_cast<size_t>(c) * 2 * qh + qh + i]);
  }
  const size_t vi = i / 8, e = i - vi * 8;  // 16-byte vector and lane of element i
  float a2[8], cv[8];
  widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha2) + vi), a2);
  widen8<T16>(__ldg(static_cast<const uint4*>(a.const_v) + vi), cv);
  a.grad_alpha1[i] = s1;
  a.grad_alpha2[i] = __fmul_rn(sc, cv[e]);
  a.grad_v[i] = __fmul_rn(sc, a2[e]);
}

template <typename T16>
cudaError_t launch_t(const SpecialBwdArgs& a, cudaStream_t st) {
  const int V = a.H / kVecElems;
  cudaError_t err = launch_pdl(special_dot_kernel<T16>, dim3(sm_count() * 4), dim3(kThreads), 0,
                               st, a);
  if (err != cudaSuccess) return err;
  const long long n = static_cast<long long>(a.bs) * V;
  err = launch_pdl(special_ori_kernel<T16>, dim3(static_cast<int>((n + kThreads - 1) / kThreads)),
                   dim3(kThreads), 0, st, a);
  if (err != cudaSuccess || a.Q == 0) return err;
  const int chunks = (a.bs + kChunkTokens - 1) / kChunkTokens;
  err = launch_pdl(special_partial_kernel<T16>,
                   dim3(chunks, a.Q, (V + kThreads - 1) / kThreads), dim3(kThreads), 0, st, a);
  if (err != cudaSuccess) return err;
  const long long qh = static_cast<long long>(a.Q) * a.H;
  return launch_pdl(special_final_kernel<T16>,
                    dim3(static_cast<int>((qh + kThreads - 1) / kThreads)), dim3(kThreads), 0, st,
                    a, chunks);
}

}  // namespace

size_t special_bwd_workspace_bytes(int bs, int H, int Q) {
  const size_t chunks = (static_cast<size_t>(bs) + kChunkTokens - 1) / kChunkTokens;
  return chunks * 2 * static_cast<size_t>(Q) * H * sizeof(float);
}

cudaError_t launch_special_bwd(const void* grad_out, const int32_t* topk_idx,
                               const float* weights, const uint8_t* mask, int mask_ndim,
                               const void* ori_x, const void* alpha1, const void* alpha2,
                               const void* const_v, float* grad_w, void* grad_ori_x,
                               float* grad_alpha1, float* grad_alpha2, float* grad_v,
                               void* workspace, int bs, int K, int H, int E, int Z, int C, int Q,
                               int dtype, cudaStream_t st) {
  if (bs == 0) return cudaSuccess;
  SpecialBwdArgs a;
  a.grad_out = grad_out;
  a.topk_idx = topk_idx;
  a.weights = weights;
  a.mask = mask;
  a.mask_ndim = mask_ndim;
  a.ori_x = ori_x;
  a.alpha1 = alpha1;
  a.alpha2 = alpha2;
  a.const_v = const_v;
  a.grad_w = grad_w;
  a.grad_ori_x = grad_ori_x;
  a.grad_alpha1 = grad_alpha1;
  a.grad_alpha2 = grad_alpha2;
  a.grad_v = grad_v;
  a.partials = static_cast<float*>(workspace);
  a.bs = bs;
  a.K = K;
  a.H = H;
  a.E = E;
  a.Z = Z;
  a.C = C;
  a.Q = Q;
  return dtype == MOE_BF16 ? launch_t<Bf16>(a, st) : launch_t<Fp16>(a, st);
}

}  // namespace moe
