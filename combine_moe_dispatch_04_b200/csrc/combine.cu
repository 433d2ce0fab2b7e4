// Combine forward and dispatch backward (the same gather with unit weights).
// [combine] Function (Formula; special expert use cases), Parameters, Return
// Value.
//
// Forward: one thread per 16-byte vector (8 values) of an output row (or a
// few vectors when K is small), in one-shot blocks. The thread issues the
// loads of all of its token's K slot rows first, then accumulates in fp32 in
// ascending k with every product and every sum rounded on its own
// (__fmul_rn / __fadd_rn: never contracted into an FMA), adds shared_expert_x
// once, and narrows with round-to-nearest-even.

#include <mutex>

#include "async.cuh"
#include "common.cuh"
#include "launch.cuh"

namespace moe {

// CTAs that gave up a bounded wait on an asynchronous copy (0 in normal use).
__device__ unsigned g_wait_timeouts = 0;

unsigned* wait_timeout_counter() {
  static std::mutex mu;
  static unsigned* ptr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);  // host threads may make a device's first call together
  if (ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_wait_timeouts) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<unsigned*>(p);
  }
  return ptr[dev];
}

namespace {

// Threads per block of the weighted gathers: 128-thread blocks (at the same
// registers, so twice the blocks per SM) ran the special-expert combine in
// 62.6 us against 65.0 and the Mixtral-shaped one in 66.3 against 68.0.
constexpr int kFwdThreads = 128;

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

// Pair metadata of one (token, k): kind, expand_x row or const row, weight.
struct PairMeta {
  int kind;
  int row;
  float w;
};

// Classifies pair (t, k) (k < K, t < BS). With CHECK_REPEATS the ids of the
// same token's earlier k are read again (L1) for the repeat check; without it
// the caller does that check itself. With SRC_ROWS (combine_fwd_kernel) a copy
// or const pair's row is its token t, whose ori_x row it loads together with
// the routed rows, and a const pair keeps its const row j above the kind's
// low three bits (kind = kConst | j << 3).
template <bool SPECIAL, bool UNIT, bool CHECK_REPEATS = true, bool SRC_ROWS = false>
__device__ __forceinline__ PairMeta classify_pair(const CombineArgs& a, int t, int k) {
  PairMeta m{kSkip, 0, 1.0f};
  const size_t tk = static_cast<size_t>(t) * a.K + k;
  // With special experts the id and the slot are loaded together, so the pair
  // costs one round trip instead of two (the slot load would otherwise wait for
  // the id's range check). Without them the slot is loaded after the mask test,
  // which measured faster (8192-token step 195.8 vs 199.6 us; loading it with
  // the mask byte instead gained nothing on the masked Mixtral-shaped step and
  // cost the 8192-token one 2 us).
  if (!UNIT) m.w = __ldg(a.weights + tk);
  int s = -1;
  if (SPECIAL) s = __ldg(a.assist + static_cast<size_t>(a.A) + tk);
  const int32_t* ids = a.topk_idx + static_cast<size_t>(t) * a.K;
  const int id = SPECIAL ? __ldg(ids + k) : 0;
  if (!pair_active(a.mask, a.mask_ndim, t, k, a.K)) return m;
  if (!SPECIAL) s = __ldg(a.assist + static_cast<size_t>(a.A) + tk);
  if (SPECIAL) {
    if (id < 0 || id >= a.E + a.Z + a.C + a.Q) return m;
    if (CHECK_REPEATS)
      for (int j = 0; j < k; ++j)
        if (__ldg(ids + j) == id) return m;
    if (id >= a.E) {
      m.kind = id < a.E + a.Z ? kZero : id < a.E + a.Z + a.C ? kCopy : kConst;
      m.row = id - (a.E + a.Z + a.C);
      if (SRC_ROWS && m.kind == kConst) m.kind = kConst | (m.row << 3);
      if (SRC_ROWS && m.kind != kZero) m.row = t;
      return m;
    }
  }
  if (s >= 0) {
    m.kind = kRouted;
    m.row = s;
  }
  return m;
}

// Sixteen-byte vectors of zeros that skipped pairs read (branch-free sum).
constexpr int kZeroVecs = 64;
__device__ uint4 g_zero_vecs[kZeroVecs];

// Resident blocks per SM the forward kernel is compiled for, counted in
// 256-thread blocks (a register cap that avoids spills for each variant). For
// the special-expert variant with K <= 8: at 4 (64 registers, a few bytes of
// spill) it ran 67 us against 76 us at 3 (72 registers, no spill) on the
// 8192-token H 2048 special workload.
#ifndef MOE_FWD_SPECIAL_MIN_BLOCKS
#define MOE_FWD_SPECIAL_MIN_BLOCKS 4
#endif
template <int KMAX, bool SPECIAL>
__host__ __device__ constexpr int fwd_blocks_of_256() {
  return SPECIAL ? (KMAX <= 8 ? MOE_FWD_SPECIAL_MIN_BLOCKS : 2) : KMAX == 16 ? 2 : KMAX == 4 ? 3 : 4;
}
template <int KMAX, bool SPECIAL>
__host__ __device__ constexpr int fwd_min_blocks() {
  return fwd_blocks_of_256<KMAX, SPECIAL>() * (256 / kFwdThreads);
}

// Each warp owns a contiguous span of 32 * U output vectors (8 values each);
// lane l handles vectors l, l + 32, ... of the span, so every load of the warp
// is 32 consecutive 16-byte vectors. When a span fits in two tokens' rows
// (V >= 32 * U, the WARP_META variant), lanes 0..K-1 classify the first token's
// pairs and lanes 16..16+K-1 the second's, once for the whole span, and every
// lane takes its token's metadata by shuffle. (Narrower rows: every thread
// classifies its own token's pairs.) Every row a pair reads is loaded in one
// batch before the sum in ascending k.
// The rows of one warp span, from its pairs' kinds, rows and weights: every
// row a pair reads is loaded in one batch, then summed in ascending k and
// stored. SPECIAL: the pairs may be zero, copy or const experts.
template <typename T16, int KMAX, bool SPECIAL, bool UNIT, bool COPY = false>
__device__ __forceinline__ void gather_span(const CombineArgs& a, int span, int V, int n,
                                            int lane, int (&kind)[fwd_vectors_per_thread<KMAX>()][KMAX],
                                            const int (&row)[fwd_vectors_per_thread<KMAX>()][KMAX],
                                            float (&wt)[fwd_vectors_per_thread<KMAX>()][KMAX],
                                            const int (&col)[fwd_vectors_per_thread<KMAX>()]) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
  // the branch-free sum (below) where it measured faster: unit weights (DSv3-shaped
  // dispatch backward 87.7 -> 87.3 us, Mixtral-shaped 65.9 -> 62.5) and K > 4
  // without special experts (DSv3-shaped combine 101.4 -> 98.7); slower with
  // special experts (64.9 -> 66.9) and for the weighted K <= 4 gather (Mixtral
  // combine 67.9 -> 86.5)
  constexpr bool BRANCHFREE = UNIT || (!SPECIAL && KMAX > 4);
  const uint4* Y = static_cast<const uint4*>(a.expand_x);
  uint4 val[U][KMAX];
  // every row a pair reads (a routed row, or the ori_x row of a copy / const
  // pair) is loaded in one batch, before any is used
  const uint4* ORI = static_cast<const uint4*>(a.ori_x);
  if constexpr (BRANCHFREE) {
    // A sum that starts at +0 never becomes -0 (x + y is -0 only when both
    // are), so adding w * 0 never changes it: a skipped pair reads a vector of
    // zeros with weight 0 (its product is 0 whatever the weight held) and is
    // summed like the others, without a branch per pair. In the special-expert
    // kernel's plain spans a zero-expert pair reads the zeros with its own
    // weight (its term w * 0 is the oracle's) and, with COPY, a copy pair reads
    // its token's ori_x row like a routed row.
    static_assert(!SPECIAL, "routed, copy, zero-expert and skipped pairs only");
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = col[u];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        const int kd = kind[u][j];
        const uint4* src = g_zero_vecs + (v & (kZeroVecs - 1));
        if (kd == kRouted) src = Y + static_cast<size_t>(row[u][j]) * V + v;
        if (COPY && kd == kCopy) src = ORI + static_cast<size_t>(row[u][j]) * V + v;
        val[u][j] = ld_nc_v4(src);
        if (kd == kSkip) wt[u][j] = 0.0f;
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = col[u];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        const int kd = SPECIAL ? (kind[u][j] & 7) : kind[u][j];
        if (kd == kRouted)
          val[u][j] = ld_nc_v4(Y + static_cast<size_t>(row[u][j]) * V + v);
        else if (SPECIAL && (kd == kCopy || kd == kConst))
          val[u][j] = ld_nc_v4(ORI + static_cast<size_t>(row[u][j]) * V + v);
      }
    }
  }
  // the shared-expert row, added last, goes to L2 meanwhile (else it costs a
  // second DRAM round trip after the sum: DSv3-shaped step 443.9 -> 441.6 us)
  if (!UNIT && a.shared != nullptr) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int item = span + u * 32 + lane;
      if (item < n) prefetch_l2(static_cast<const uint4*>(a.shared) + item);
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int item = span + u * 32 + lane;
    if (item >= n) continue;
    const int v = col[u];
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const int kd = SPECIAL ? (kind[u][j] & 7) : kind[u][j];
      if (!BRANCHFREE && kd == kSkip) continue;
      float m[8];
      if (SPECIAL && kd == kConst) {  // alpha_1 * ori_x + alpha_2 * v, each product and the sum rounded
        const size_t r = static_cast<size_t>(kind[u][j] >> 3) * V + v;
        float o[8], a1[8], a2[8], cv[8];
        widen8<T16>(val[u][j], o);
        widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha1) + r), a1);
        widen8<T16>(__ldg(static_cast<const uint4*>(a.alpha2) + r), a2);
        widen8<T16>(__ldg(static_cast<const uint4*>(a.const_v) + r), cv);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          m[i] = __fadd_rn(__fmul_rn(a1[i], o[i]), __fmul_rn(a2[i], cv[i]));
      } else if (SPECIAL && !BRANCHFREE && kd == kZero) {
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = 0.0f;
      } else {  // a routed or ori_x row (or, branch-free, a vector of zeros)
        widen8<T16>(val[u][j], m);
      }
      if (UNIT)
        add8_rn(acc, m);
      else
        axpy8_rn(acc, wt[u][j], m);
    }
    if (!UNIT && a.shared != nullptr) {
      float sh[8];
      widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.shared) + item), sh);
      add8_rn(acc, sh);
    }
    st_v4(static_cast<uint4*>(a.out) + item, narrow8<T16>(acc));
  }
}


// Shuffles the classifying lanes' pair metadata to every lane of the span
// (lanes 0..15: the span's first token, 16..31: the next one).
template <int KMAX, bool UNIT>
__device__ __forceinline__ void spread_meta(const PairMeta& m, int span, int v0, int V, int K,
                                            int n, int lane,
                                            int (&kind)[fwd_vectors_per_thread<KMAX>()][KMAX],
                                            int (&row)[fwd_vectors_per_thread<KMAX>()][KMAX],
                                            float (&wt)[fwd_vectors_per_thread<KMAX>()][KMAX],
                                            int (&col)[fwd_vectors_per_thread<KMAX>()]) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int item = span + u * 32 + lane;
    // the span's first token, or the next one past its end (V >= 32 * U: at
    // most one wrap)
    int src_base = 0;
    col[u] = v0 + u * 32 + lane;
    if (col[u] >= V) {
      col[u] -= V;
      src_base = 16;
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      kind[u][j] = __shfl_sync(0xFFFFFFFFu, m.kind, src_base + j);
      row[u][j] = __shfl_sync(0xFFFFFFFFu, m.row, src_base + j);
      wt[u][j] = UNIT ? 1.0f : __shfl_sync(0xFFFFFFFFu, m.w, src_base + j);
      if (j >= K || item >= n) kind[u][j] = kSkip;
    }
  }
}

template <typename T16, int KMAX, bool SPECIAL, bool UNIT, bool WARP_META>
__global__ void __launch_bounds__(kFwdThreads, (fwd_min_blocks<KMAX, SPECIAL>()))
    combine_fwd_kernel(CombineArgs a) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int n = a.bs * V;
  const int lane = threadIdx.x & 31;
  const int span = blockIdx.x * (kFwdThreads * U) + (threadIdx.x >> 5) * (32 * U);
  if (span >= n) return;  // warp-uniform
  int kind[U][KMAX], row[U][KMAX];
  float wt[U][KMAX];
  int col[U];  // each vector's column in its row (one division per span)
  if (WARP_META) {  // the launcher picks WARP_META only when V >= 32 * U
    const int t0 = span / V;
    const int v0 = span - t0 * V;
    const int tm = t0 + (lane >> 4), km = lane & 15;
    const bool mine = km < K && tm < a.bs;
    PairMeta m{kSkip, 0, 1.0f};
    if (mine) m = classify_pair<SPECIAL, UNIT, false, true>(a, tm, km);
    if (SPECIAL) {
      // A span whose tokens have no const pair takes the plain gather
      // (warp-uniform): with routed (or skipped) pairs only for any K, and with
      // zero-expert and copy pairs too where the plain gather is branch-free
      // (K > 4), which sums them as zero vectors or ori_x rows with their
      // weights. A repeated routed id already has no slot, so the repeat check
      // is needed only where special ids are present.
      const int kd = m.kind & 7;
      const bool any_special = __any_sync(0xFFFFFFFFu, kd >= kZero);
      if (any_special) {
        // a repeat of an id held by an earlier lane of the same token takes no part
        const int id = mine ? __ldg(a.topk_idx + static_cast<size_t>(tm) * K + km) : -1;
        bool dup = false;
#pragma unroll
        for (int jj = 0; jj < KMAX - 1; ++jj) {  // km < K <= KMAX
          const int other = __shfl_sync(0xFFFFFFFFu, id, (lane & 16) | jj);
          dup |= jj < km && other == id;
        }
        if (dup) m.kind = kSkip;
      }
      const bool plain = KMAX > 4 ? !__any_sync(0xFFFFFFFFu, kd == kConst) : !any_special;
      spread_meta<KMAX, UNIT>(m, span, v0, V, K, n, lane, kind, row, wt, col);
      if (plain) {
        gather_span<T16, KMAX, false, UNIT, true>(a, span, V, n, lane, kind, row, wt, col);
        return;
      }
    } else {
      spread_meta<KMAX, UNIT>(m, span, v0, V, K, n, lane, kind, row, wt, col);
    }
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int item = span + u * 32 + lane;
      const int t = item / V;
      col[u] = item - t * V;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        kind[u][j] = kSkip;
        row[u][j] = 0;
        wt[u][j] = 1.0f;
        if (j >= K || item >= n) continue;
        const PairMeta m = classify_pair<SPECIAL, UNIT, true, true>(a, t, j);
        kind[u][j] = m.kind;
        row[u][j] = m.row;
        wt[u][j] = m.w;
      }
    }
  }
  gather_span<T16, KMAX, SPECIAL, UNIT>(a, span, V, n, lane, kind, row, wt, col);
}

// ---------------------------------------------------------------------------
// Combine forward with comm_quant_mode 2 in two passes over a caller workspace.
//
// Pass 1 (row_scale_kernel): one warp per slot row s < R, streaming the row
// once: max|y| on packed 16-bit pairs, a warp reduction, and then
// rscale[s] = (scale, reciprocal) with scale = fl(max / 127) (IEEE division);
// the reciprocal is 0 for an all-zero row (its codes are 0) and -1 marks a
// scale below 2^-100 (the codes then come from IEEE divisions).
template <typename T16>
__global__ void __launch_bounds__(256) row_scale_kernel(const uint4* __restrict__ Y,
                                                         const int32_t* __restrict__ send,
                                                         int E, int A, int V,
                                                         float2* __restrict__ rscale) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int R = min(max(__ldg(send + E), 0), A);
  const int nw = gridDim.x * (blockDim.x >> 5);
  for (int s = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); s < R; s += nw) {
    const uint4* row = Y + static_cast<size_t>(s) * V;
    uint32_t m2 = 0;
#pragma unroll 4
    for (int v = lane; v < V; v += 32) m2 = absmax_v4<T16>(m2, ld_nc_v4(row + v));
    float mx = absmax_final<T16>(m2);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
    if (lane == 0) {
      const float scale = __fdiv_rn(mx, 127.0f);
      const float inv = mx == 0.0f ? 0.0f : (scale >= kFastMinScale ? 1.0f / scale : -1.0f);
      rscale[s] = make_float2(scale, inv);
    }
  }
}

// Pass 2 (combine_fwd_rt_kernel): the one-shot gather of combine_fwd_kernel
// (routed pairs only, rows of at least 32 U vectors) with, per routed pair,
// the int8 codes of its values (quant_codes8) and their dequantisation
// fl(code * scale) before the same weighted fp32 sum. The lane that classified
// a pair also holds its (scale, reciprocal); every lane fetches them by
// shuffle when the pair's turn comes, so no per-pair array is kept.
template <typename T16, int KMAX>
__global__ void __launch_bounds__(kFwdThreads, (fwd_blocks_of_256<KMAX, false>() - 1) * (256 / kFwdThreads))
    combine_fwd_rt_kernel(CombineArgs a, const float2* __restrict__ rscale) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int n = a.bs * V;
  const int lane = threadIdx.x & 31;
  const int span = blockIdx.x * (kFwdThreads * U) + (threadIdx.x >> 5) * (32 * U);
  if (span >= n) return;  // warp-uniform
  const uint4* Y = static_cast<const uint4*>(a.expand_x);
  // lanes 0..K-1 classify the span's first token's pairs, lanes 16..16+K-1 the next one's
  const int t0 = span / V;
  const int v0 = span - t0 * V;
  const int tm = t0 + (lane >> 4), km = lane & 15;
  PairMeta pm{kSkip, 0, 1.0f};
  if (km < K && tm < a.bs) pm = classify_pair<false, false, false>(a, tm, km);
  const float2 ms = pm.kind == kRouted ? __ldg(rscale + pm.row) : make_float2(0.0f, 0.0f);
  uint4 val[U][KMAX];
  uint32_t routed[U];
  int src[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int item = span + u * 32 + lane;
    int v = v0 + u * 32 + lane;  // past the first token's row: the next one's
    src[u] = 0;
    if (v >= V) {
      v -= V;
      src[u] = 16;
    }
    routed[u] = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const int kind = __shfl_sync(0xFFFFFFFFu, pm.kind, src[u] + j);
      const int row = __shfl_sync(0xFFFFFFFFu, pm.row, src[u] + j);
      if (j < K && item < n && kind == kRouted) {
        routed[u] |= 1u << j;
        val[u][j] = ld_nc_v4(Y + static_cast<size_t>(row) * V + v);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int item = span + u * 32 + lane;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const float w = __shfl_sync(0xFFFFFFFFu, pm.w, src[u] + j);
      const float sc = __shfl_sync(0xFFFFFFFFu, ms.x, src[u] + j);
      const float iv = __shfl_sync(0xFFFFFFFFu, ms.y, src[u] + j);
      if ((routed[u] >> j) & 1u) {
        float y[8], q[8], b[8], m[8];
        widen8<T16>(val[u][j], y);
        quant_codes8<true>(y, sc, iv, iv >= 0.0f, q, b);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const float2 p = __fmul2_rn(f2(q[i], q[i + 1]), f2(sc, sc));
          m[i] = p.x;
          m[i + 1] = p.y;
        }
        axpy8_rn(acc, w, m);
      }
    }
    if (item >= n) continue;
    if (a.shared != nullptr) {
      float sh[8];
      widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.shared) + item), sh);
      add8_rn(acc, sh);
    }
    st_v4(static_cast<uint4*>(a.out) + item, narrow8<T16>(acc));
  }
}

// ---------------------------------------------------------------------------
// Combine forward with comm_quant_mode 2 ([combine] Parameters): every routed
// row returns through the per-row int8 round trip (scale = max|y| / 127 in
// fp32, q = clamp(rne(y / scale), -127, 127), value = q * scale) before the
// same weighted fp32 sum. One CTA per token, thread i owning vectors
// i, i + blockDim, ... of each row. Pass 1 reads the token's routed rows
// (through L1) and reduces each row's max|y| (shuffle + shared memory; a max
// does not depend on order); pass 2 reads them again, dequantises and
// accumulates in ascending k.
template <typename T16, int KMAX, bool SPECIAL>
__global__ void __launch_bounds__(1024) combine_fwd_q8_kernel(CombineArgs a) {
  __shared__ PairMeta meta[KMAX];
  __shared__ float red[32][KMAX];
  __shared__ float rmax[KMAX];
  pdl_trigger();
  pdl_wait();
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const uint4* Y = static_cast<const uint4*>(a.expand_x);
  for (int t = blockIdx.x; t < a.bs; t += gridDim.x) {
    if (threadIdx.x < K) meta[threadIdx.x] = classify_pair<SPECIAL, false>(a, t, threadIdx.x);
    __syncthreads();
    for (int j = 0; j < K; ++j) {  // meta is block-uniform: no divergence around the shuffles
      if (meta[j].kind != kRouted) continue;
      float mx = 0.0f;
      for (int v = threadIdx.x; v < V; v += blockDim.x) {
        float f[8];
        widen8<T16>(__ldg(Y + static_cast<size_t>(meta[j].row) * V + v), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(f[i]));
      }
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
      if (lane == 0) red[warp][j] = mx;
    }
    __syncthreads();
    if (threadIdx.x < K && meta[threadIdx.x].kind == kRouted) {
      float mx = 0.0f;
      for (int w = 0; w < nwarps; ++w) mx = fmaxf(mx, red[w][threadIdx.x]);
      rmax[threadIdx.x] = mx;
    }
    __syncthreads();
    bool need_ori = false;
    if (SPECIAL)
      for (int j = 0; j < K; ++j) need_ori |= meta[j].kind == kCopy || meta[j].kind == kConst;
    for (int v = threadIdx.x; v < V; v += blockDim.x) {
      const size_t item = static_cast<size_t>(t) * V + v;
      float ori[8];
      if (SPECIAL && need_ori) widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.ori_x) + item), ori);
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      for (int j = 0; j < K; ++j) {
        const PairMeta pm = meta[j];
        if (pm.kind == kSkip) continue;
        float m[8];
        if (pm.kind == kRouted) {
          const float mx = rmax[j];
          float y[8];
          widen8<T16>(__ldg(Y + static_cast<size_t>(pm.row) * V + v), y);
          const float scale = __fdiv_rn(mx, 127.0f);
          const float inv_scale = 1.0f / scale;
          quant_roundtrip8(y, mx, scale, inv_scale, m);
        } else {
          pair_values<T16, SPECIAL>(a, pm.kind, pm.row, V, v, make_uint4(0, 0, 0, 0), ori, m);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(pm.w, m[i]));
      }
      if (a.shared != nullptr) {
        float sh[8];
        widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.shared) + item), sh);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], sh[i]);
      }
      st_v4(static_cast<uint4*>(a.out) + item, narrow8<T16>(acc));
    }
    __syncthreads();  // meta, red and rmax are reused by the next token
  }
}

// The same round trip with the token's rows staged in shared memory: one CTA
// per token on a persistent grid, NBUF row buffers, warp-specialised. A
// producer warp classifies each token's pairs (lanes 0..K-1, repeats found by
// shuffle) ahead of time, waits until the consumers have released the
// buffer, records the pairs in shared memory and starts one bulk copy per
// routed row (cp.async.bulk, global -> shared, completing on the buffer's
// "full" mbarrier). Eight consumer warps wait for "full", take each row's
// max|y| on packed 16-bit pairs (the K reductions interleaved, then one
// consumer-only named barrier; the array is double-buffered by token parity),
// finish the K maxima from shared memory (lane j: row j, its scale and
// reciprocal), dequantise and accumulate in ascending k, and release the
// buffer on its "empty" mbarrier. The classification's global loads thus
// never sit on the consumers' path. Every wait is bounded: a block that gives
// up counts itself in *timeouts, lets its started copies land and returns.
constexpr int kQ8sConsumerWarps = 8;
constexpr int kQ8sConsumers = 32 * kQ8sConsumerWarps;
constexpr int kQ8sThreads = kQ8sConsumers + 32;  // the last warp is the producer
constexpr int kQ8sWarps = kQ8sConsumerWarps;

template <int KMAX, int NBUF>
struct Q8sLayout {  // byte offsets into the dynamic shared memory
  static constexpr size_t full = 0;    // NBUF mbarriers
  static constexpr size_t empty = 32;  // NBUF mbarriers
  static constexpr size_t meta = 64;
  static constexpr size_t red = meta + (NBUF * KMAX * sizeof(PairMeta) + 15) / 16 * 16;
  static constexpr size_t end = red + 2 * kQ8sWarps * KMAX * sizeof(float);
  static constexpr size_t rows = (end + 127) / 128 * 128;
  static size_t bytes(int V) { return rows + static_cast<size_t>(NBUF) * KMAX * V * 16; }
};

template <typename T16, int KMAX, bool SPECIAL, int NBUF>
__global__ void __launch_bounds__(kQ8sThreads, 2) combine_fwd_q8s_kernel(CombineArgs a,
                                                                         WaitCfg wc,
                                                                         unsigned* timeouts) {
  using L = Q8sLayout<KMAX, NBUF>;
  static_assert(NBUF >= 2 && NBUF <= 4, "buffers");
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::empty);
  PairMeta* meta = reinterpret_cast<PairMeta*>(smem + L::meta);
  float* red = reinterpret_cast<float*>(smem + L::red);
  uint4* rows = reinterpret_cast<uint4*>(smem + L::rows);
  const int V = a.H / kVecElems;
  const int K = a.K;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint4* Y = static_cast<const uint4*>(a.expand_x);
  if (threadIdx.x == 0) {
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, kQ8sConsumerWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  const int stride = gridDim.x;

  if (warp == kQ8sConsumerWarps) {  // producer
    int q = 0;
    for (int t = blockIdx.x; t < a.bs; t += stride, ++q) {
      const int b = q % NBUF;
      PairMeta pm{kSkip, 0, 1.0f};
      if (lane < K) pm = classify_pair<SPECIAL, false, false>(a, t, lane);
      if (SPECIAL) {
        const int id = lane < K ? __ldg(a.topk_idx + static_cast<size_t>(t) * K + lane) : -1;
        bool dup = false;
#pragma unroll
        for (int jj = 0; jj < KMAX; ++jj) {
          const int other = __shfl_sync(0xFFFFFFFFu, id, jj);
          dup |= jj < lane && other == id;
        }
        if (dup) pm.kind = kSkip;
      }
      const unsigned routed = __ballot_sync(0xFFFFFFFFu, pm.kind == kRouted);
      if (q >= NBUF) {  // wait until the consumers have released this buffer
        // (it gives up only after the consumers did: they count the block)
        const bool ok = mbar_wait_bounded(empty + b, ((q / NBUF) - 1) & 1, wc.limit_ns);
        if (__any_sync(0xFFFFFFFFu, !ok)) return;
      }
      if (lane < KMAX) meta[b * KMAX + lane] = pm;
      fence_proxy_async_smem();  // the buffer was last read by the consumers' loads
      if (q == wc.withhold && blockIdx.x == 0) {  // test hook: 16 bytes that never come
        if (lane == 0) mbar_arrive_expect_tx(full + b, 16u);
        continue;
      }
      if (lane == 0) mbar_arrive_expect_tx(full + b, __popc(routed) * static_cast<uint32_t>(V) * 16u);
      __syncwarp();
      if ((routed >> lane) & 1u)
        bulk_g2s(rows + (static_cast<size_t>(b) * KMAX + lane) * V,
                 Y + static_cast<size_t>(pm.row) * V, static_cast<uint32_t>(V) * 16u, full + b);
    }
    return;
  }

  int it = 0;
  for (int t = blockIdx.x; t < a.bs; t += stride, ++it) {
    const int b = it % NBUF;
    const int rb = it & 1;
    const bool ok = mbar_wait_bounded(full + b, (it / NBUF) & 1, wc.limit_ns);
    const PairMeta* pmeta = meta + b * KMAX;
    const uint4* brows = rows + static_cast<size_t>(b) * KMAX * V;
    // this warp's max |y| of every row, the K reductions interleaved
    // (rows of pairs that are not routed hold stale data: their maxima are
    // computed without a branch and never used)
    float mx[KMAX];
    {
      uint32_t m2[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) m2[j] = 0;
      for (int v = threadIdx.x; v < V; v += kQ8sConsumers)
#pragma unroll
        for (int j = 0; j < KMAX; ++j) m2[j] = absmax_v4<T16>(m2[j], brows[static_cast<size_t>(j) * V + v]);
#pragma unroll
      for (int j = 0; j < KMAX; ++j) mx[j] = absmax_final<T16>(m2[j]);
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1)
#pragma unroll
      for (int j = 0; j < KMAX; ++j) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xFFFFFFFFu, mx[j], d));
    if (lane == 0)
#pragma unroll
      for (int j = 0; j < KMAX; ++j) red[(rb * kQ8sWarps + warp) * KMAX + j] = mx[j];
    // consumers only; a block whose wait gave up leaves together
    if (named_barrier_or(1, kQ8sConsumers, !ok)) {
      if (threadIdx.x == 0) {
        atomicAdd(timeouts, 1u);
        for (int q = 0; q < NBUF; ++q)  // copies already started: let them land
          if (t + q * stride < a.bs && !(it + q == wc.withhold && blockIdx.x == 0))
            mbar_wait_bounded(full + (it + q) % NBUF, ((it + q) / NBUF) & 1);
      }
      return;
    }
    // every warp: lane j < K finishes row j's max and takes its scale and reciprocal
    float rm = 0.0f;
    if (lane < KMAX)
#pragma unroll
      for (int w = 0; w < kQ8sWarps; ++w) rm = fmaxf(rm, red[(rb * kQ8sWarps + w) * KMAX + lane]);
    const float rs = __fdiv_rn(rm, 127.0f);
    const float ri = 1.0f / rs;
    // the fast path's reciprocal: 0 for an all-zero row (its codes are then 0)
    const float rf = rm == 0.0f ? 0.0f : ri;
    // lane j also holds pair j's weight and kind; the warp takes them by shuffle
    const PairMeta lpm = pmeta[lane < KMAX ? lane : 0];
    const int lkind = lane < K ? lpm.kind : static_cast<int>(kSkip);
    const float lw = lpm.w;
    const uint32_t routed = __ballot_sync(0xFFFFFFFFu, lkind == kRouted);
    const uint32_t zerom = SPECIAL ? __ballot_sync(0xFFFFFFFFu, lkind == kZero) : 0u;
    const uint32_t copym = SPECIAL ? __ballot_sync(0xFFFFFFFFu, lkind == kCopy) : 0u;
    const uint32_t constm = SPECIAL ? __ballot_sync(0xFFFFFFFFu, lkind == kConst) : 0u;
    const uint32_t fastm = __ballot_sync(0xFFFFFFFFu, rm == 0.0f || rs >= kFastMinScale);
    // routed rows with a scale too small for the fast reciprocal take the
    // general path below (IEEE divisions); everything else the loop here
    const bool tiny = (routed & ~fastm) != 0u;
    // Whole warps walk the vectors (the shuffles below need every lane); a lane
    // past the row end works on vector 0 and stores nothing.
    for (int v0 = warp * 32; v0 < V; v0 += kQ8sConsumers) {
      const bool act = v0 + lane < V;
      const int v = act ? v0 + lane : 0;
      const size_t item = static_cast<size_t>(t) * V + v;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      if (!tiny) {
        // one pair at a time in ascending k, each term added as in the
        // oracle; the branches follow the token's pair kinds (warp-uniform)
        float ori[8];
        if (SPECIAL && (copym | constm) != 0u)  // requested before the loop
          widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.ori_x) + item), ori);
#pragma unroll 1
        for (int j = 0; j < KMAX; ++j) {
          const float rfj = __shfl_sync(0xFFFFFFFFu, rf, j);
          const float rsj = __shfl_sync(0xFFFFFFFFu, rs, j);
          const float wj = __shfl_sync(0xFFFFFFFFu, lw, j);
          float prod[8];
          if ((routed >> j) & 1u) {
            float y[8], n[8], b[8];
            widen8<T16>(brows[static_cast<size_t>(j) * V + v], y);
            quant_codes8<false>(y, rsj, rfj, true, n, b);  // exact, ties included
#pragma unroll
            for (int i = 0; i < 8; ++i) prod[i] = __fmul_rn(wj, __fmul_rn(n[i], rsj));
          } else if (SPECIAL && ((zerom | copym | constm) >> j) & 1u) {
            const int kind = (zerom >> j) & 1u ? kZero : (copym >> j) & 1u ? kCopy : kConst;
            float m[8];
            pair_values<T16, SPECIAL>(a, kind, pmeta[j].row, V, v, make_uint4(0, 0, 0, 0), ori, m);
#pragma unroll
            for (int i = 0; i < 8; ++i) prod[i] = __fmul_rn(wj, m[i]);
          } else {
            continue;
          }
          add8_rn(acc, prod);
        }
      }
      uint32_t redo = tiny ? 1u : 0u;
      // a routed row with a tiny scale: the general path (warp-uniform)
      if (redo != 0u) {
        float ori[8];
        if (SPECIAL && (copym | constm) != 0u)
          widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.ori_x) + item), ori);
        float acc2[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc2[i] = 0.0f;
#pragma unroll 1
        for (int j = 0; j < KMAX; ++j) {
          const int kind = __shfl_sync(0xFFFFFFFFu, lkind, j);
          const float wj = __shfl_sync(0xFFFFFFFFu, lw, j);
          const float rmj = __shfl_sync(0xFFFFFFFFu, rm, j);
          const float rsj = __shfl_sync(0xFFFFFFFFu, rs, j);
          const float rij = __shfl_sync(0xFFFFFFFFu, ri, j);
          if (kind == kSkip) continue;
          float m[8];
          if (kind == kRouted) {
            float y[8];
            widen8<T16>(brows[static_cast<size_t>(j) * V + v], y);
            quant_roundtrip8<true>(y, rmj, rsj, rij, m);
          } else {
            pair_values<T16, SPECIAL>(a, kind, pmeta[j].row, V, v, make_uint4(0, 0, 0, 0), ori, m);
          }
          axpy8_rn(acc2, wj, m);
        }
        if (redo != 0u)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = acc2[i];
      }
      if (!act) continue;
      if (a.shared != nullptr) {
        float sh[8];
        widen8<T16>(ld_nc_v4(static_cast<const uint4*>(a.shared) + item), sh);
        add8_rn(acc, sh);
      }
      st_v4(static_cast<uint4*>(a.out) + item, narrow8<T16>(acc));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + b);  // this warp is done with buffer b
  }
}

template <typename T16, int KMAX, bool SPECIAL, bool UNIT>
cudaError_t launch_fwd_kmax(const CombineArgs& a, cudaStream_t st) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
  const int V = a.H / kVecElems;
  const long long n = static_cast<long long>(a.bs) * V;
  const int blocks = static_cast<int>((n + kFwdThreads * U - 1) / (kFwdThreads * U));
  if (V >= 32 * U)
    return launch_pdl(combine_fwd_kernel<T16, KMAX, SPECIAL, UNIT, true>, dim3(blocks),
                      dim3(kFwdThreads), 0, st, a);
  return launch_pdl(combine_fwd_kernel<T16, KMAX, SPECIAL, UNIT, false>, dim3(blocks),
                    dim3(kFwdThreads), 0, st, a);
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

// Shared memory a CTA of the staged kernel may use: two CTAs per SM.
constexpr size_t kQ8sSmemBudget = 110 * 1024;

template <typename T16, bool SPECIAL, int KMAX, int NBUF>
cudaError_t launch_fwd_q8s(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st) {
  constexpr auto kernel = combine_fwd_q8s_kernel<T16, KMAX, SPECIAL, NBUF>;
  const int V = a.H / kVecElems;
  const size_t smem = Q8sLayout<KMAX, NBUF>::bytes(V);
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  unsigned* timeouts = wait_timeout_counter();
  if (timeouts == nullptr) return cudaErrorInvalidSymbol;
  int per_sm = 0;  // depends on the row size: not cached
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQ8sThreads, smem);
  if (err != cudaSuccess) return err;
  const int cap = sm_count() * (per_sm > 0 ? per_sm : 1);
  const int blocks = a.bs < cap ? a.bs : cap;
  return launch_pdl(kernel, dim3(blocks), dim3(kQ8sThreads), smem, st, a, wc, timeouts);
}

// Staged kernel with three buffers when they fit the budget, else two; false
// when even two do not fit (the caller then takes the two-pass kernel).
template <typename T16, bool SPECIAL, int KMAX>
bool try_launch_fwd_q8s(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st,
                        cudaError_t* err) {
  const int V = a.H / kVecElems;
  if (Q8sLayout<KMAX, 3>::bytes(V) <= kQ8sSmemBudget) {
    *err = launch_fwd_q8s<T16, SPECIAL, KMAX, 3>(a, wc, st);
    return true;
  }
  if (Q8sLayout<KMAX, 2>::bytes(V) <= kQ8sSmemBudget) {
    *err = launch_fwd_q8s<T16, SPECIAL, KMAX, 2>(a, wc, st);
    return true;
  }
  return false;
}

// The staged single-pass kernel when the shape allows it (false otherwise).
template <typename T16, bool SPECIAL>
bool try_launch_q8s_k(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st,
                      cudaError_t* err) {
  if (a.K <= 2) return try_launch_fwd_q8s<T16, SPECIAL, 2>(a, wc, st, err);
  if (a.K <= 4) return try_launch_fwd_q8s<T16, SPECIAL, 4>(a, wc, st, err);
  if (a.K <= 8) return try_launch_fwd_q8s<T16, SPECIAL, 8>(a, wc, st, err);
  return false;
}

template <typename T16, bool SPECIAL>
cudaError_t launch_fwd_q8_t(const CombineArgs& a, cudaStream_t st) {
  const int V = a.H / kVecElems;
  cudaError_t err = cudaSuccess;
  if (try_launch_q8s_k<T16, SPECIAL>(a, kProductWaits, st, &err)) return err;
  const int threads = V < 256 ? (V + 31) / 32 * 32 : 256;
  const int cap = sm_count() * (2048 / threads);
  const int blocks = a.bs < cap ? a.bs : cap;
  if (a.K <= 2)
    return launch_pdl(combine_fwd_q8_kernel<T16, 2, SPECIAL>, dim3(blocks), dim3(threads), 0, st, a);
  if (a.K <= 4)
    return launch_pdl(combine_fwd_q8_kernel<T16, 4, SPECIAL>, dim3(blocks), dim3(threads), 0, st, a);
  if (a.K <= 8)
    return launch_pdl(combine_fwd_q8_kernel<T16, 8, SPECIAL>, dim3(blocks), dim3(threads), 0, st, a);
  return launch_pdl(combine_fwd_q8_kernel<T16, 16, SPECIAL>, dim3(blocks), dim3(threads), 0, st, a);
}

template <typename T16>
cudaError_t launch_fwd_q8(const CombineArgs& a, cudaStream_t st) {
  if (a.Z + a.C + a.Q > 0) return launch_fwd_q8_t<T16, true>(a, st);
  return launch_fwd_q8_t<T16, false>(a, st);
}

template <typename T16, int KMAX>
cudaError_t launch_fwd_rt_k(const CombineArgs& a, const float2* rscale, cudaStream_t st) {
  constexpr int U = fwd_vectors_per_thread<KMAX>();
  const long long n = static_cast<long long>(a.bs) * (a.H / kVecElems);
  const int blocks = static_cast<int>((n + kFwdThreads * U - 1) / (kFwdThreads * U));
  return launch_pdl(combine_fwd_rt_kernel<T16, KMAX>, dim3(blocks), dim3(kFwdThreads), 0, st, a,
                    rscale);
}

// The two-pass path: whether it applies (routed pairs only, rows wide enough
// for the shared pair metadata), and its two launches.
bool rt_applies(const CombineArgs& a) {
  const int V = a.H / kVecElems;
  const int U = a.K <= 2 ? 4 : a.K <= 4 ? 2 : 1;
  return a.Z + a.C + a.Q == 0 && a.weights != nullptr && V >= 32 * U;
}

template <typename T16>
cudaError_t launch_fwd_rt(const CombineArgs& a, const int32_t* send, float2* rscale,
                          cudaStream_t st) {
  const int V = a.H / kVecElems;
  const long long want = (static_cast<long long>(a.A) + 7) / 8;  // 8 warps per CTA
  const long long cap = static_cast<long long>(sm_count()) * 8;
  const int blocks = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
  cudaError_t err = launch_pdl(row_scale_kernel<T16>, dim3(blocks), dim3(256), 0, st,
                               static_cast<const uint4*>(a.expand_x), send, a.E, a.A, V, rscale);
  if (err != cudaSuccess) return err;
  if (a.K <= 2) return launch_fwd_rt_k<T16, 2>(a, rscale, st);
  if (a.K <= 4) return launch_fwd_rt_k<T16, 4>(a, rscale, st);
  if (a.K <= 8) return launch_fwd_rt_k<T16, 8>(a, rscale, st);
  return launch_fwd_rt_k<T16, 16>(a, rscale, st);
}

}  // namespace

cudaError_t launch_combine_fwd(const CombineArgs& a, cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  return a.dtype == MOE_BF16 ? launch_fwd_t<Bf16>(a, st) : launch_fwd_t<Fp16>(a, st);
}

size_t combine_q8_workspace_bytes(int A) { return static_cast<size_t>(A) * sizeof(float2); }

cudaError_t launch_combine_fwd_q8s_test(const CombineArgs& a, const WaitCfg& wc, cudaStream_t st,
                                        bool* launched) {
  cudaError_t err = cudaSuccess;
  const bool special = a.Z + a.C + a.Q > 0;
  if (a.dtype == MOE_BF16)
    *launched = special ? try_launch_q8s_k<Bf16, true>(a, wc, st, &err)
                        : try_launch_q8s_k<Bf16, false>(a, wc, st, &err);
  else
    *launched = special ? try_launch_q8s_k<Fp16, true>(a, wc, st, &err)
                        : try_launch_q8s_k<Fp16, false>(a, wc, st, &err);
  return err;
}

cudaError_t launch_combine_fwd_q8(const CombineArgs& a, const int32_t* send, void* workspace,
                                  cudaStream_t st) {
  if (a.bs == 0) return cudaSuccess;
  if (workspace != nullptr && send != nullptr && a.A > 0 && rt_applies(a)) {
    float2* rscale = static_cast<float2*>(workspace);
    return a.dtype == MOE_BF16 ? launch_fwd_rt<Bf16>(a, send, rscale, st)
                               : launch_fwd_rt<Fp16>(a, send, rscale, st);
  }
  return a.dtype == MOE_BF16 ? launch_fwd_q8<Bf16>(a, st) : launch_fwd_q8<Fp16>(a, st);
}

}  // namespace moe
