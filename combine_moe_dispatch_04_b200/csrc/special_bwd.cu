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
// Three launches: warp-per-token grad_w dots (fixed butterfly) and grad_ori_x,
// per-(token chunk, const expert) partial sums into the workspace, and a
// fixed-order sum over the chunks. Every result is deterministic.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kChunkTokens = 64;  // tokens per partial sum of the alpha / v gradients

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

// grad_w of the copy/const pairs and grad_ori_x: one warp per token on a
// persistent grid. Lanes 0..K-1 classify the token's pairs (a repeat of an id
// held by an earlier lane takes no part). A token without such pairs only
// writes its zero grad_ori_x row. Otherwise the warp makes one pass over the
// row, kUV vectors per lane at a time with all their grad_out and ori_x loads
// issued first: per vector it adds the pairs' terms to grad_ori_x in ascending
// k and each pair's products to that pair's own dot accumulator (pair k in
// register k); the dots are reduced with a fixed butterfly at the end.
constexpr int kUV = 2;

template <typename T16, int KMAX>
__global__ void __launch_bounds__(kThreads) special_token_kernel(SpecialBwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int lo = a.E + a.Z;
  const int nw = gridDim.x * (kThreads / 32);
  for (int t = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t < a.bs; t += nw) {
    const int id = lane < K ? __ldg(a.topk_idx + static_cast<size_t>(t) * K + lane) : -1;
    bool dup = false;
#pragma unroll
    for (int jj = 0; jj < KMAX; ++jj) {
      const int other = __shfl_sync(0xFFFFFFFFu, id, jj);
      dup |= jj < lane && other == id;
    }
    int my_kind = 0, my_q = 0;
    float my_w = 0.0f;
    if (lane < K && !dup && id >= lo && id < lo + a.C + a.Q &&
        pair_active(a.mask, a.mask_ndim, t, lane, K)) {
      my_kind = id < lo + a.C ? 1 : 2;
      my_q = id - lo - a.C;
      my_w = __ldg(a.weights + static_cast<size_t>(t) * K + lane);
    }
    uint4* go = static_cast<uint4*>(a.grad_ori_x) + static_cast<size_t>(t) * V;
    const unsigned spec = __ballot_sync(0xFFFFFFFFu, my_kind != 0);
    if (spec == 0) {  // no copy/const pair: a zero grad_ori_x row
      for (int v = lane; v < V; v += 32) st_v4(go + v, make_uint4(0u, 0u, 0u, 0u));
      continue;
    }
    const uint4* g = static_cast<const uint4*>(a.grad_out) + static_cast<size_t>(t) * V;
    const uint4* x = static_cast<const uint4*>(a.ori_x) + static_cast<size_t>(t) * V;
    float d[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) d[j] = 0.0f;
    // every lane runs every iteration: the shuffles below need the whole warp
    for (int v0 = 0; v0 < V; v0 += 32 * kUV) {
      uint4 gv[kUV], xv[kUV];
#pragma unroll
      for (int u = 0; u < kUV; ++u) {
        const int v = v0 + 32 * u + lane;
        gv[u] = v < V ? ld_nc_v4(g + v) : make_uint4(0u, 0u, 0u, 0u);
        xv[u] = v < V ? ld_nc_v4(x + v) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kUV; ++u) {
        const int v = v0 + 32 * u + lane;
        const bool in = v < V;
        float gf[8], xf[8], acc[8];
        widen8<T16>(gv[u], gf);
        widen8<T16>(xv[u], xf);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (!((spec >> j) & 1u)) continue;  // warp-uniform
          const int kind = __shfl_sync(0xFFFFFFFFu, my_kind, j);
          const float w = __shfl_sync(0xFFFFFFFFu, my_w, j);
          const int q = __shfl_sync(0xFFFFFFFFu, my_q, j);
          if (kind == 1) {  // copy: c = fl(w g) into grad_ori_x, <g, ori_x> into the dot
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              acc[i] = __fadd_rn(acc[i], __fmul_rn(w, gf[i]));
              d[j] = __fmaf_rn(gf[i], xf[i], d[j]);
            }
          } else {  // const: fl(c alpha_1), and <g, fl(fl(a1 x) + fl(a2 v))>
            const size_t r = static_cast<size_t>(q) * V + (in ? v : 0);
            float a1[8], a2[8], cv[8];
            widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha1) + r), a1);
            widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha2) + r), a2);
            widen8<T16>(__ldg(static_cast<const uint4*>(a.const_v) + r), cv);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              acc[i] = __fadd_rn(acc[i], __fmul_rn(__fmul_rn(w, gf[i]), a1[i]));
              d[j] = __fmaf_rn(gf[i], __fadd_rn(__fmul_rn(a1[i], xf[i]), __fmul_rn(a2[i], cv[i])),
                               d[j]);
            }
          }
        }
        if (in) st_v4(go + v, narrow8<T16>(acc));
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (!((spec >> j) & 1u)) continue;
      float dj = d[j];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dj += __shfl_xor_sync(0xFFFFFFFFu, dj, off);
      if (lane == 0) a.grad_w[static_cast<size_t>(t) * K + j] = dj;
    }
  }
}

// Partial sums over one chunk of tokens for one const expert q. The first
// threads find, per token of the chunk, the pair of q (its first occurrence
// in the row, if active) and the CTA compacts those tokens in ascending order
// into shared memory; then every thread (one 16-byte vector of the row) walks
// the list, a few tokens' loads in flight at a time.
template <typename T16>
__global__ void __launch_bounds__(kThreads) special_partial_kernel(SpecialBwdArgs a) {
  __shared__ int s_tok[kChunkTokens];
  __shared__ float s_w[kChunkTokens];
  __shared__ int s_cnt[kChunkTokens / 32];
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int chunk = blockIdx.x, q = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = chunk * kChunkTokens;
  const int target = a.E + a.Z + a.C + q;
  bool hit = false;
  float wt = 0.0f;
  const int t = t0 + threadIdx.x;
  if (threadIdx.x < kChunkTokens && t < a.bs) {
    const int32_t* ids = a.topk_idx + static_cast<size_t>(t) * a.K;
    for (int k = 0; k < a.K; ++k) {
      if (__ldg(ids + k) != target) continue;
      if (pair_active(a.mask, a.mask_ndim, t, k, a.K)) {
        hit = true;
        wt = __ldg(a.weights + static_cast<size_t>(t) * a.K + k);
      }
      break;  // later occurrences are repeats
    }
  }
  const unsigned bal = __ballot_sync(0xFFFFFFFFu, hit);
  if (lane == 0 && warp < kChunkTokens / 32) s_cnt[warp] = __popc(bal);
  __syncthreads();
  int n = 0, base = 0;
#pragma unroll
  for (int w2 = 0; w2 < kChunkTokens / 32; ++w2) {
    if (w2 < warp) base += s_cnt[w2];
    n += s_cnt[w2];
  }
  if (hit) {
    const int pos = base + __popc(bal & lanemask_lt());
    s_tok[pos] = t;
    s_w[pos] = wt;
  }
  __syncthreads();
  const int v = blockIdx.z * kThreads + threadIdx.x;
  if (v >= V) return;
  float s1[8], sc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s1[i] = sc[i] = 0.0f;
  const uint4* G = static_cast<const uint4*>(a.grad_out);
  const uint4* X = static_cast<const uint4*>(a.ori_x);
  constexpr int kU = 4;
  for (int i0 = 0; i0 < n; i0 += kU) {
    uint4 gv[kU], xv[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (i0 + u < n) {
        const size_t r = static_cast<size_t>(s_tok[i0 + u]) * V + v;
        gv[u] = ld_nc_v4(G + r);
        xv[u] = ld_nc_v4(X + r);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (i0 + u >= n) break;
      const float w = s_w[i0 + u];
      float gf[8], xf[8];
      widen8<T16>(gv[u], gf);
      widen8<T16>(xv[u], xf);
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
  float4* p1v = reinterpret_cast<float4*>(p1 + static_cast<size_t>(v) * 8);
  float4* pcv = reinterpret_cast<float4*>(pc + static_cast<size_t>(v) * 8);
  p1v[0] = make_float4(s1[0], s1[1], s1[2], s1[3]);
  p1v[1] = make_float4(s1[4], s1[5], s1[6], s1[7]);
  pcv[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
  pcv[1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
}

// Sum of the partials over the chunks: grad_alpha1, and the alpha_2 / v
// gradients from S. A block takes 32 elements; its 8 warps sum the chunks
// c = w, w + 8, ... of each (lane = element), then one fixed-order pass over
// the 8 sums: the same order every run.
constexpr int kFinalParts = kThreads / 32;

template <typename T16>
__global__ void __launch_bounds__(kThreads) special_final_kernel(SpecialBwdArgs a, int chunks) {
  __shared__ float s1p[kFinalParts][32], scp[kFinalParts][32];
  pdl_trigger();
  pdl_wait();
  const size_t qh = static_cast<size_t>(a.Q) * a.H;
  const int lane = threadIdx.x & 31, part = threadIdx.x >> 5;
  const size_t i = static_cast<size_t>(blockIdx.x) * 32 + lane;
  float s1 = 0.0f, sc = 0.0f;
  if (i < qh) {
#pragma unroll 4
    for (int c = part; c < chunks; c += kFinalParts) {
      s1 = __fadd_rn(s1, a.partials[static_cast<size_t>(c) * 2 * qh + i]);
      sc = __fadd_rn(sc, a.partials[static_cast<size_t>(c) * 2 * qh + qh + i]);
    }
  }
  s1p[part][lane] = s1;
  scp[part][lane] = sc;
  __syncthreads();
  if (part != 0 || i >= qh) return;
  s1 = s1p[0][lane];
  sc = scp[0][lane];
#pragma unroll
  for (int p = 1; p < kFinalParts; ++p) {
    s1 = __fadd_rn(s1, s1p[p][lane]);
    sc = __fadd_rn(sc, scp[p][lane]);
  }
  // element i of alpha_2 and v: the pair of 16-bit values holding it, widened
  const size_t pi = i / 2;
  const float2 a2 = T16::widen2(__ldg(static_cast<const uint32_t*>(a.alpha2) + pi));
  const float2 cv = T16::widen2(__ldg(static_cast<const uint32_t*>(a.const_v) + pi));
  const bool hi = i & 1;
  a.grad_alpha1[i] = s1;
  a.grad_alpha2[i] = __fmul_rn(sc, hi ? cv.y : cv.x);
  a.grad_v[i] = __fmul_rn(sc, hi ? a2.y : a2.x);
}

template <typename T16, int KMAX>
cudaError_t launch_token(const SpecialBwdArgs& a, cudaStream_t st) {
  constexpr auto kernel = special_token_kernel<T16, KMAX>;
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
  if (err != cudaSuccess) return err;
  const long long want = (static_cast<long long>(a.bs) + kThreads / 32 - 1) / (kThreads / 32);
  const long long cap = static_cast<long long>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  return launch_pdl(kernel, dim3(static_cast<int>(want < cap ? want : cap)), dim3(kThreads), 0,
                    st, a);
}

template <typename T16>
cudaError_t launch_t(const SpecialBwdArgs& a, cudaStream_t st) {
  const int V = a.H / kVecElems;
  cudaError_t err = a.K <= 2   ? launch_token<T16, 2>(a, st)
                    : a.K <= 4 ? launch_token<T16, 4>(a, st)
                    : a.K <= 8 ? launch_token<T16, 8>(a, st)
                               : launch_token<T16, 16>(a, st);
  if (err != cudaSuccess || a.Q == 0) return err;
  const int chunks = (a.bs + kChunkTokens - 1) / kChunkTokens;
  err = launch_pdl(special_partial_kernel<T16>,
                   dim3(chunks, a.Q, (V + kThreads - 1) / kThreads), dim3(kThreads), 0, st, a);
  if (err != cudaSuccess) return err;
  const long long qh = static_cast<long long>(a.Q) * a.H;
  return launch_pdl(special_final_kernel<T16>, dim3(static_cast<int>((qh + 31) / 32)),
                    dim3(kThreads), 0, st, a, chunks);
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
